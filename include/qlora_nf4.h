/*
 * qlora_nf4.h -- C ABI of the B200 (sm_100a) NF4 + double-quant + LoRA linear layer.
 *
 * The library quantises a frozen base weight W (n_out x k_in, bf16) to 4-bit
 * NormalFloat codes with one absmax per 64 consecutive weights, double-quantises
 * those absmaxes, and evaluates the QLoRA linear layer and its input gradient:
 *
 *   h      = dequant(W) x + s * B (A x)                       (forward)
 *   grad_x = dequant(W)^T grad_h + s * A^T (B^T grad_h)       (input gradient)
 *   s      = alpha / r
 *
 * Sources (page title, section):
 *   - NF4 table, 64-weight blocks, double quantisation of the block constants to
 *     FP8 in groups of 256 after subtracting their mean: "QLoRA paper notes"
 *     (tqpw.cn), sections "NormalFloat Quantization (NF4)" and
 *     "Double Quantization".
 *   - h = Wx + BAx and h = dequant(W_NF4) x + BAx, dequantisation to bf16 for the
 *     matmul: "Quantized LoRA (QLoRA) and 4-bit training" (apxml.com), the two
 *     forward equations and the list of the four configuration knobs.
 *   - Shapes W (d x k), B (d x r), A (r x k); one constant per 64 weights;
 *     gradients through the dequantised, frozen base: "How does QLoRA work for
 *     training?" (aivaro.ru), sections 2, 5 and 7.
 *   - lora_alpha as the adapter's scaling factor: LoRA/QLoRA talk summary
 *     (spark.aweffr.cn), "practice guide" configuration list.
 *
 * Conventions shared by every entry point
 *   - All tensors are row-major and contiguous. bf16 tensors are passed as
 *     `const void *` / `void *` pointing at 16-bit bf16 values.
 *   - Every tensor pointer is a DEVICE pointer (memory of the current CUDA
 *     device), except the `qn_nf4_weight` struct itself, which lives in host
 *     memory and holds device pointers. Sizes are element counts unless named
 *     *_bytes.
 *   - The caller owns and allocates every buffer, workspaces included. The
 *     library allocates no memory and keeps no per-call state.
 *   - `stream` is a cudaStream_t (NULL = legacy default stream). Every call only
 *     enqueues work on it and returns; results are ready when the stream is.
 *   - Argument errors are returned synchronously, before anything is enqueued.
 *     QN_ECUDA means a launch failed; faults inside a kernel surface at the
 *     caller's next synchronisation of the stream.
 *   - Calls are reentrant. Two calls that run concurrently on the GPU must not
 *     share an output buffer or a workspace.
 */
#ifndef QLORA_NF4_H
#define QLORA_NF4_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    QN_OK = 0,
    QN_EINVAL = 1,     /* null pointer, negative size, bad r or alpha          */
    QN_ESHAPE = 2,     /* k_in not a multiple of 64, or a size above the limits */
    QN_EALIGN = 3,     /* a tensor pointer is not 16-byte aligned               */
    QN_ECUDA = 4,      /* a CUDA launch or attribute call failed                */
    QN_EWORKSPACE = 5, /* workspace pointer null or smaller than required       */
    QN_ETIMEOUT = 6    /* a kernel stopped early: a bounded wait ran out (qlora_workspace_check) */
} qn_status;

/* Blocking of the format: one absmax per QN_BLOCK consecutive weights of the
 * row-major flattened W, one fp32 scale per QN_GROUP consecutive blocks. */
#define QN_BLOCK 64
#define QN_GROUP 256
/* Largest supported LoRA rank. */
#define QN_MAX_RANK 256

/* The two other settings of the 4-bit load ("Quantized LoRA (QLoRA) and 4-bit
 * training" (apxml.com), the four configuration knobs; "How does QLoRA work for
 * training?" (aivaro.ru) 6, bnb_4bit_quant_type and bnb_4bit_use_double_quant):
 *   quant type  : the table the code nibbles index. QN_QUANT_NF4 (the default):
 *                 NormalFloat4 as printed in "QLoRA paper notes" (tqpw.cn). QN_QUANT_FP4:
 *                 the standard 4-bit float, read as E2M1 (sign, two exponent bits with
 *                 bias 1, one mantissa bit; magnitudes 0, 0.5, 1, 1.5, 2, 3, 4, 6) divided
 *                 by 6 onto [-1, 1] and rounded to fp32; code = sign (bit 3) | magnitude
 *                 index (bits 0-2). "QLoRA paper notes", Experiments: NF4 does better.
 *   block constants: QN_CONST_DQ (the default): double quantised (absmax_q,
 *                 group_scale, absmax_mean). QN_CONST_F32: the exact fp32 block absmax
 *                 in `absmax` (0.5 bit per weight instead of 0.127; "QLoRA & PEFT family"
 *                 (ai-reference-codex) 3.3). */
#define QN_QUANT_NF4 0
#define QN_QUANT_FP4 1
#define QN_CONST_DQ 0
#define QN_CONST_F32 1

/* A quantised weight. The struct is host memory; the buffers are device memory
 * owned by the caller, with the sizes qn_weight_sizes() returns; codes,
 * absmax_q, group_scale and absmax start on 16-byte boundaries (QN_EALIGN
 * otherwise). A zero-initialised struct tail (quant_type, const_format, absmax)
 * is NF4 with double quantisation.
 *   codes        : n_out*k_in/2 bytes. Weight e = n*k_in + k (row-major) is the
 *                  low nibble of byte e/2 when e is even, the high nibble when e
 *                  is odd. A nibble is an index 0..15 into the quant type's table
 *                  (NF4: ascending values, index 7 is 0.0; FP4: see above).
 *   absmax_q     : nb = n_out*k_in/64 bytes, the FP8 E4M3 (finite variant,
 *                  max 448) code of d_b = absmax_b - mean, divided by the
 *                  group scale.
 *   group_scale  : ng = ceil(nb/256) floats; group g covers blocks
 *                  [256 g, 256 g + 256) of the flattened block index (groups may
 *                  straddle rows).
 *   absmax_mean  : 1 float, the exact mean of all nb block absmaxes, rounded
 *                  once to fp32.
 *   (absmax_q, group_scale and absmax_mean: QN_CONST_DQ only; NULL otherwise.)
 *   quant_type   : QN_QUANT_NF4 or QN_QUANT_FP4.
 *   const_format : QN_CONST_DQ or QN_CONST_F32.
 *   absmax       : QN_CONST_F32 only: nb floats, the block absmaxes c_b.
 * Block constant: c'_b = fma(e4m3_decode(absmax_q[b]), group_scale[b/256],
 * absmax_mean) in fp32 (QN_CONST_DQ), or c_b itself (QN_CONST_F32); dequantised
 * weight: T[code] * c'_b with T the quant type's table. */
typedef struct {
    int64_t n_out;
    int64_t k_in;
    uint8_t *codes;
    uint8_t *absmax_q;
    float *group_scale;
    float *absmax_mean;
    int32_t quant_type;
    int32_t const_format;
    float *absmax;
} qn_nf4_weight;

/* Byte sizes of the four buffers of a quantised n_out x k_in weight.
 * Errors: QN_EINVAL (null output pointer, negative size), QN_ESHAPE
 * (k_in % 64 != 0). Host-only; touches no GPU. */
qn_status qn_nf4_sizes(int64_t n_out, int64_t k_in, size_t *codes_bytes, size_t *absmax_bytes,
                       size_t *scale_bytes, size_t *mean_bytes);

/* Byte sizes of the buffers of a quantised n_out x k_in weight with block
 * constants const_format: QN_CONST_DQ gives qn_nf4_sizes()'s four sizes and
 * absmax_f32_bytes = 0; QN_CONST_F32 gives codes_bytes, absmax_f32_bytes = 4 nb
 * and zero for the three double-quantisation buffers.
 * Errors: as qn_nf4_sizes, QN_EINVAL for an unknown const_format. */
qn_status qn_weight_sizes(int64_t n_out, int64_t k_in, int const_format, size_t *codes_bytes, size_t *absmax_bytes,
                          size_t *scale_bytes, size_t *mean_bytes, size_t *absmax_f32_bytes);

/* Workspace bytes nf4_quantize needs for an n_out x k_in weight. Host-only. */
qn_status qn_quantize_workspace_size(int64_t n_out, int64_t k_in, size_t *ws_bytes);

/* nf4_quantize -- W (n_out x k_in bf16, device) -> the quantised weight `out`,
 * in out's quant type and constant format.
 * Per block of 64: absmax c_b, code = index of the table value nearest to
 * fl32(w / c_b) (ties to the lower index; c_b == 0 gives the lowest code of the
 * value 0: 7 for NF4, 0 for FP4), two codes per byte. QN_CONST_F32: absmax[b] =
 * c_b. QN_CONST_DQ: mean mu of all c_b (exact, rounded once), d_b = fl32(c_b - mu),
 * group scale sigma_g = fl32(max_b |d_b| / 448), absmax_q[b] =
 * e4m3_rn_satfinite(fl32(d_b / sigma_g)) (0 when sigma_g == 0).
 * Source: "QLoRA paper notes" (tqpw.cn), "NormalFloat Quantization (NF4)" and
 * "Double Quantization"; "How does QLoRA work for training?" (aivaro.ru) 5.
 * W must not contain NaN or Inf (the result is then unspecified).
 * ws: device workspace of at least qn_quantize_workspace_size() bytes, 256-byte
 * aligned; its contents on entry do not matter.
 * Errors: QN_EINVAL, QN_ESHAPE, QN_EALIGN (W, codes, absmax_q or group_scale not
 * 16-byte aligned), QN_EWORKSPACE, QN_ECUDA. */
qn_status nf4_quantize(const void *W, const qn_nf4_weight *out, void *ws, size_t ws_bytes, void *stream);

/* nf4_quantize_static_ws -- nf4_quantize without a caller workspace and without allocating.
 * No counterpart in the paper: this entry point exists for callers that cannot allocate
 * device memory when they quantise -- code running inside a global-mode stream capture (where
 * cudaMalloc is not permitted), runtimes whose device memory is entirely owned by another
 * allocator, and latency-critical paths that cannot afford cudaMalloc's implicit device
 * synchronisation. The scratch is a file-scope 16 MiB device array inside the library, which
 * every GPU that loads the library holds until the process exits; it fits weights of at most
 * 4,193,728 blocks of 64 (268,398,592 weights; 28672 x 8192 fits). Larger weights are
 * rejected with QN_EWORKSPACE before anything is enqueued.
 * Results are bit-identical to nf4_quantize. The first call in each CUDA context (on each
 * device, and again after a device reset, which loads the library's module anew) looks up the
 * scratch address (cudaGetSymbolAddress) with that device current, so make it before any
 * stream capture. Every call shares the one scratch array (the part that must start at zero is
 * cleared by each call): calls whose work overlaps on the GPU -- on different streams, or from
 * different host threads -- race and must be serialised by the caller.
 * No memory is allocated or freed (no cudaMalloc, cudaFree or allocating library call).
 * Errors: as nf4_quantize, with QN_EWORKSPACE for weights above the limit. */
qn_status nf4_quantize_static_ws(const void *W, const qn_nf4_weight *out, void *stream);

/* nf4_dequantize -- quantised weight -> W_out (n_out x k_in bf16, device):
 * W_out[e] = bf16_rn(fl32(T[code_e] * c'_b)).
 * Source: "Quantized LoRA (QLoRA) and 4-bit training" (apxml.com), the
 * dequantisation step to bf16 before the matmul.
 * Errors: QN_EINVAL, QN_ESHAPE, QN_EALIGN (codes or W_out not 16-byte
 * aligned), QN_ECUDA. */
qn_status nf4_dequantize(const qn_nf4_weight *w, void *W_out, void *stream);

/* qlora_merge_bf16 -- fold the adapter into a 16-bit weight (merge and unload):
 *   W_out[n, k] = bf16_rn( fl32(NF4[code] * c'_b) + s * sum_j B[n,j] A[j,k] ),  s = alpha / r.
 * A : r x k_in bf16, B : n_out x r bf16 (r == 0: A = B = NULL, W_out is the
 * dequantised weight); W_out : n_out x k_in bf16 (written; must not alias A or B).
 * The adapter product is accumulated in fp32 on the tensor cores and added to
 * the fp32 dequantised weight with one fp32 rounding before the bf16 rounding,
 * so a result may differ from the exactly rounded sum by one bf16 unit.
 * Source: "QLoRA & PEFT family" (ai-reference-codex) 3.6 (merge_and_unload);
 * "QLoRA paper notes" (tqpw.cn), Introduction (the merged weight is 16-bit:
 * it cannot be folded back into NF4).
 * Errors: QN_EINVAL, QN_ESHAPE, QN_EALIGN (codes, A, B or W_out not 16-byte
 * aligned), QN_ECUDA. */
qn_status qlora_merge_bf16(const qn_nf4_weight *w, const void *A, const void *B, int r, float alpha, void *W_out,
                           void *stream);

/* Workspace bytes qlora_linear_fwd / qlora_linear_bwd_x need for M tokens,
 * an n_out x k_in weight and rank r (0 <= r <= 256). Host-only.
 *
 * The linear-layer workspace: device memory of at least this many bytes,
 * 256-byte aligned. Zero all of it once when it is allocated. Its first 4
 * bytes are an error word: the kernels never clear it, they only set it when
 * a bounded wait inside them runs out (1) or the launch could not run (2), in
 * which case that call's output is incomplete; qlora_workspace_check reads and
 * clears it. The next bytes hold state the few-token kernels hand from one CTA
 * to another within a call (the adapter product and its ready flag); every
 * call leaves that state as it found it, so the workspace needs no clearing
 * between calls, but after an error (QN_ETIMEOUT) zero it all again before
 * reusing it. One workspace may serve any number of calls in stream order, of
 * any shapes, as long as it is large enough for each; calls that run
 * concurrently on the GPU need separate workspaces. */
qn_status qlora_workspace_size(int64_t M, int64_t n_out, int64_t k_in, int r, size_t *ws_bytes);

/* qlora_workspace_check -- read back and clear the workspace error word.
 * Synchronises `stream` (the stream the calls that used `ws` ran on).
 * Returns QN_OK when no kernel that used `ws` since the last check gave up a
 * bounded wait, QN_ETIMEOUT (and clears the word) otherwise.
 * No counterpart in the pages: this is the library's failure report.
 * Errors: QN_EINVAL (null ws), QN_ECUDA, QN_ETIMEOUT. */
qn_status qlora_workspace_check(void *ws, void *stream);

/* qn_selftest_wait_timeout -- a check of the error path above: enqueues one kernel that waits, with
 * the same bounded wait the library's kernels use, on a word of the (zeroed) linear workspace that
 * nothing ever sets. The wait runs out after its poll limit (about a second) and the kernel
 * records the timeout in the error word, so a following qlora_workspace_check returns
 * QN_ETIMEOUT and clears it. Nothing faults or hangs. No counterpart on the pages: it exists to
 * test the failure path of the hot-path kernels without breaking them.
 * ws: a linear workspace of at least 256 bytes, zeroed. Errors: QN_EWORKSPACE, QN_ECUDA. */
qn_status qn_selftest_wait_timeout(void *ws, size_t ws_bytes, void *stream);

/* qlora_linear_fwd -- h = dequant(W) x + (alpha/r) B (A x), per token row:
 *   h[m, n] = sum_k W'[n,k] x[m,k] + s * sum_j B[n,j] sum_k A[j,k] x[m,k].
 *   x : M x k_in bf16 (tokens x features); A : r x k_in bf16; B : n_out x r bf16;
 *   h : M x n_out bf16 (written, must not alias x, A or B).
 * fp32 accumulation; the block constant is applied in fp32; the adapter
 * product s (A x) is rounded to bf16 as the operand of the up-projection (for
 * M <= 64 per K-slice of the split reduction, whose partial up-projections are
 * then summed in fp32).
 * r == 0 means no adapter (A and B must then be NULL; alpha is ignored).
 * Source: "Quantized LoRA (QLoRA) and 4-bit training" (apxml.com), forward
 * equations; "How does QLoRA work for training?" (aivaro.ru) 2.
 * ws: the linear-layer workspace (see qlora_workspace_size: at least that many
 * bytes, 256-byte aligned, error word zeroed once). M may be 0 (nothing is
 * enqueued).
 * Ordering: the call may start reading the quantised weight (not x, A, B or h)
 * before the preceding kernel on the stream has finished when that kernel
 * signals its dependents early (griddepcontrol.launch_dependents); such a
 * kernel must not write the quantised weight. No kernel of this library that
 * signals early writes one.
 * Errors: QN_EINVAL, QN_ESHAPE, QN_EALIGN (x, h, codes, A or B not 16-byte
 * aligned), QN_EWORKSPACE, QN_ECUDA. */
qn_status qlora_linear_fwd(const qn_nf4_weight *w, const void *x, int64_t M, const void *A, const void *B,
                           int r, float alpha, void *h, void *ws, size_t ws_bytes, void *stream);

/* qlora_linear_bwd_x -- input gradient through the frozen base and the adapter:
 *   grad_x[m, k] = sum_n grad_h[m,n] W'[n,k] + s * sum_j A[j,k] sum_n grad_h[m,n] B[n,j].
 *   grad_h : M x n_out bf16; grad_x : M x k_in bf16 (written, no aliasing).
 * W is frozen: nothing is written to the quantised weight. fp32 accumulation;
 * u = s (B^T grad_h) is rounded to bf16 as the up-projection's MMA operand for
 * M > 64 and kept in fp32 for M <= 64.
 * Source: "How does QLoRA work for training?" (aivaro.ru) 7 (weights are
 * dequantised on the fly for the gradient and not updated).
 * Same workspace, alignment and error rules as qlora_linear_fwd. */
qn_status qlora_linear_bwd_x(const qn_nf4_weight *w, const void *grad_h, int64_t M, const void *A,
                             const void *B, int r, float alpha, void *grad_x, void *ws, size_t ws_bytes,
                             void *stream);

/* Workspace bytes qlora_lora_grads needs for M tokens and rank r (1..256).
 * Host-only. The workspace's contents on entry do not matter. */
qn_status qlora_lora_grads_workspace_size(int64_t M, int r, size_t *ws_bytes);

/* qlora_lora_grads -- gradients of the adapter weights, the only trained
 * parameters of the layer (W is frozen):
 *   grad_B[n, j] = s * sum_m grad_h[m,n] t[m,j],  t = x A^T        (n_out x r)
 *   grad_A[j, k] = s * sum_m u[m,j] x[m,k],       u = grad_h B     (r x k_in)
 * with s = alpha / r. x : M x k_in bf16, grad_h : M x n_out bf16, A : r x k_in
 * bf16, B : n_out x r bf16; grad_A, grad_B : fp32 device buffers (written).
 * t and u are rounded to bf16 (the tensor-core operands); all sums are fp32.
 * Source: "How does QLoRA work for training?" (aivaro.ru) 2 (only B and A are
 * trained) and 7 (gradients through the frozen base; only the adapters are
 * updated); the derivatives of the forward equation of "Quantized LoRA (QLoRA)
 * and 4-bit training" (apxml.com).
 * ws: at least qlora_lora_grads_workspace_size() bytes, 256-byte aligned.
 * Errors: QN_EINVAL (null pointer, r outside 1..256, alpha not finite),
 * QN_ESHAPE, QN_EALIGN, QN_EWORKSPACE, QN_ECUDA. */
qn_status qlora_lora_grads(const void *x, const void *grad_h, int64_t M, int64_t n_out, int64_t k_in,
                           const void *A, const void *B, int r, float alpha, float *grad_A, float *grad_B,
                           void *ws, size_t ws_bytes, void *stream);

/* LoRA dropout of the adapter's input (training). "QLoRA & PEFT family"
 * (ai-reference-codex) 3.4 gives the rate (0.05-0.1) and the configuration in
 * "How does QLoRA work for training?" (aivaro.ru) sets lora_dropout; the pages
 * say no more. This library's reading: inverted dropout of x on the adapter
 * branch only (the frozen base sees x unchanged). Element (m, k) of the M x
 * k_in activation has index e = offset + m * k_in + k; it survives when word
 * (e mod 4) of Philox4x32-10 (Salmon, Moraes, Dror and Shaw, SC 2011) at
 * counter (e / 4 low 32 bits, e / 4 high 32 bits, 0, 0) with key (seed low 32
 * bits, seed high 32 bits) is >= floor(p * 2^32); survivors are scaled by
 * 1 / (1 - p) (folded into the adapter scale: alpha / r / (1 - p)). The same
 * (seed, offset) in the forward, the input gradient and the adapter gradients
 * gives the same mask. A null pointer or p == 0 turns it off. */
typedef struct {
    float p;          /* drop rate, 0 <= p < 1 */
    uint64_t seed;    /* the generator's key */
    uint64_t offset;  /* added to every element index */
} qn_lora_dropout;

/* qlora_linear_fwd with LoRA dropout of the adapter's input:
 *   h = dequant(W) x + s / (1 - p) B (A (mask * x)).
 * Arguments, workspace and errors as qlora_linear_fwd; QN_EINVAL also for p
 * outside [0, 1). */
qn_status qlora_linear_fwd_dropout(const qn_nf4_weight *w, const void *x, int64_t M, const void *A, const void *B,
                                   int r, float alpha, const qn_lora_dropout *dropout, void *h, void *ws,
                                   size_t ws_bytes, void *stream);

/* qlora_linear_bwd_x under the forward's dropout mask:
 *   grad_x = dequant(W)^T grad_h + mask * (s / (1 - p) A^T (B^T grad_h)).
 * Arguments, workspace and errors as qlora_linear_bwd_x. */
qn_status qlora_linear_bwd_x_dropout(const qn_nf4_weight *w, const void *grad_h, int64_t M, const void *A,
                                     const void *B, int r, float alpha, const qn_lora_dropout *dropout, void *grad_x,
                                     void *ws, size_t ws_bytes, void *stream);

/* qlora_lora_grads under the forward's dropout mask (x replaced by mask * x,
 * s by s / (1 - p)). Arguments, workspace and errors as qlora_lora_grads. */
qn_status qlora_lora_grads_dropout(const void *x, const void *grad_h, int64_t M, int64_t n_out, int64_t k_in,
                                   const void *A, const void *B, int r, float alpha, const qn_lora_dropout *dropout,
                                   float *grad_A, float *grad_B, void *ws, size_t ws_bytes, void *stream);

/* Static description of a status code. */
const char *qn_status_string(qn_status s);

/* Detail of the last error returned on the calling host thread ("" if none). */
const char *qn_last_error(void);

/* Number of this library's kernels enqueued on the calling host thread since
 * the last reset (a launch counter for benchmarks). */
uint64_t qn_launch_count(int reset);

#ifdef __cplusplus
}
#endif

#endif /* QLORA_NF4_H */
