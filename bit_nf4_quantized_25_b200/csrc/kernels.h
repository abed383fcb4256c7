// kernels.h -- internal launchers (host side) of the sm_100a kernels. Not part of the C ABI.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace qn {

struct WeightView {
    int64_t n, k;  // W is n x k, k % 64 == 0
    const uint8_t *codes;
    const uint8_t *q;      // double-quantised constants (absmax == nullptr)
    const float *sigma;
    const float *mu;
    int qtype;             // kQuantNF4 or kQuantFP4: the table of the code nibbles
    const float *absmax;   // fp32 block constants (no double quantisation), else nullptr
};

// LoRA dropout of the adapter's input (dropout.cuh): element e = offset + m k_in + k of the
// activation is kept when its Philox draw is >= thr; thr == 0 turns it off. The kernels take the
// adapter scale already divided by 1 - p.
struct DropoutArgs {
    uint64_t seed;
    uint64_t offset;
    uint32_t thr;
};

// Lookup used by the quantiser: the interval [-1, 1] split into 64 cells of
// width 1/32 plus the point 1.0; for cell j, `thr[j]` is the single decision
// threshold inside the cell (or 2.0 when there is none) and `codes[j]` the codes
// below and above it (low byte: x <= thr, second byte: x > thr). `zero_word`: eight
// copies of the code of an all-zero block.
struct QuantCells {
    float thr[65];
    int codes[65];
    uint32_t zero_word;
};

// Launch counter (per host thread).
void count_launch(int n = 1);

// nf4_quantize: two kernels plus a memset of the exponent bins.
// With absmax != nullptr the block absmaxes are stored there as fp32 (no double quantisation;
// q, sigma and mu are not written). qtype: kQuantNF4 or kQuantFP4.
cudaError_t launch_quantize(const uint16_t *W, int64_t n, int64_t k, int qtype, uint8_t *codes, uint8_t *q,
                            float *sigma, float *mu, float *absmax, void *ws, cudaStream_t s);
size_t quantize_workspace_bytes(int64_t n, int64_t k);
// Static scratch of the allocation-free quantiser entry point: size, and its device address on
// the current device (resolved once per device).
size_t static_scratch_bytes();
cudaError_t static_scratch_address(void **out);

// nf4_dequantize.
cudaError_t launch_dequant(const WeightView &w, uint16_t *out, cudaStream_t s);

// qlora_merge_bf16: out = bf16(fl32(NF4[code] c'_b) + s B A), A r x k, B n x r (r may be 0).
cudaError_t launch_merge(const WeightView &w, const uint16_t *A, const uint16_t *B, int r, float s, uint16_t *out,
                         cudaStream_t st);

// Token-count bound of the few-token path (M <= kDecodeMaxM tokens go there; the forward
// kernel takes kDecodeTokens tokens per launch and adapters of rank <= kDecodeMaxRank).
constexpr int kDecodeMaxM = 64;
constexpr int kDecodeTokens = 16;
constexpr int kDecodeMaxRank = 64;

// h = dequant(W) x + s B (A x) for M <= kDecodeTokens tokens and r <= kDecodeMaxRank (one
// launch, several for weights taller than one wave). err is the workspace (its first word the
// error word; it also holds the adapter product t and its ready flag, see
// decode_fwd_workspace_bytes); a timeout of a bounded wait is recorded in the error word.
cudaError_t launch_decode_fwd(const WeightView &w, const uint16_t *x, int M, const uint16_t *A,
                              const uint16_t *B, int r, float s, const DropoutArgs &drop, uint16_t *h, int *err,
                              cudaStream_t st);
// Workspace bytes launch_decode_fwd uses (zeroed once before the first call).
size_t decode_fwd_workspace_bytes();
// grad_x = dequant(W)^T grad_h + s A^T (B^T grad_h), streamed kernel: M <= kDecodeTokens tokens,
// r <= kDecodeMaxRank, shapes with decode_bwd_stream_supported(), one launch; err is the
// workspace (as for launch_decode_fwd).
cudaError_t launch_decode_bwd_stream(const WeightView &w, const uint16_t *gh, int M, const uint16_t *A,
                                     const uint16_t *B, int r, float s, const DropoutArgs &drop, uint16_t *gx,
                                     int *err, cudaStream_t st);
// n_out % 8 == 0, r % 8 == 0 (or r == 0) and few enough 256-feature chunks for one wave.
bool decode_bwd_stream_supported(int64_t n, int64_t k, int r);
// grad_x = dequant(W)^T grad_h + s A^T (B^T grad_h) for M <= kDecodeMaxM tokens.
cudaError_t launch_decode_bwd(const WeightView &w, const uint16_t *gh, int M, const uint16_t *A,
                              const uint16_t *B, int r, float s, uint16_t *gx, cudaStream_t st);

// Adapter down-projection for many tokens: out[m, j] = bf16(s * sum_i act[m,i] S(j,i)),
// S(j,i) = small[j*ldj + i*ldk]; out is M x RT with zeros for j >= r. With a dropout mask the
// activation element (m, i) enters only when it survives (element index offset + m red + i).
cudaError_t launch_lora_down(const uint16_t *act, int64_t M, int64_t red, const uint16_t *small, int64_t ldj,
                             int64_t ldk, int r, float s, uint16_t *out, int RT, cudaStream_t st,
                             const DropoutArgs *drop = nullptr);
// gx[m, k] = bf16(gx[m, k] + keep(m, k) sum_j u[m, j] A[j, k]): the adapter term of the input
// gradient under dropout, added to a base-only gradient (u: M x RT bf16, already scaled).
cudaError_t launch_adapter_up_masked(const uint16_t *u, int64_t M, int RT, const uint16_t *A, int r, int64_t k,
                                     const DropoutArgs &drop, uint16_t *gx, cudaStream_t st);

// Gradients of the adapter weights (fp32): grad_A (r x k), grad_B (n x r); workspace of
// lora_grads_workspace_bytes(M, r) bytes holds t = x A^T and u = grad_h B (bf16).
size_t lora_grads_workspace_bytes(int64_t M, int r);
cudaError_t launch_lora_grads(const uint16_t *x, const uint16_t *gh, int64_t M, int64_t n, int64_t k,
                              const uint16_t *A, const uint16_t *B, int r, float s, const DropoutArgs &drop,
                              float *grad_A, float *grad_B, void *ws, cudaStream_t st);

// tcgen05 fused dequant-GEMM for many tokens (the LoRA down-projection runs first, into
// the workspace). Workspace: a 256-byte header (error word) then the M x RT adapter operand.
size_t gemm_workspace_bytes(int64_t M, int r);
bool gemm_supported(int64_t n, int64_t k, int64_t M, bool bwd);
cudaError_t launch_gemm_fwd(const WeightView &w, const uint16_t *x, int64_t M, const uint16_t *A, const uint16_t *B,
                            int r, float s, uint16_t *h, void *ws, cudaStream_t st,
                            const DropoutArgs *drop = nullptr);
cudaError_t launch_gemm_bwd(const WeightView &w, const uint16_t *gh, int64_t M, const uint16_t *A, const uint16_t *B,
                            int r, float s, uint16_t *gx, void *ws, cudaStream_t st);

// One kernel whose bounded wait on a workspace word that nothing sets runs out and records the
// timeout in the workspace error word (the shared error path, checked by a test).
cudaError_t launch_wait_timeout_selftest(void *ws, cudaStream_t st);

}  // namespace qn
