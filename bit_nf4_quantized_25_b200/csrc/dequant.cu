// dequant.cu -- nf4_dequantize on sm_100a: codes + block constants -> bf16 W.
//
// W'[e] = bf16_rn(fl32(T[code_e] * c'_b)), T the quant type's table (NF4 or the 4-bit float),
// c'_b = fma(e4m3(q_b), sigma_g, mu) with double quantisation, else the fp32 absmax c_b.
// "Quantized LoRA (QLoRA) and 4-bit training" (apxml.com): the 4-bit weights are
// dequantised to the bf16 compute type for the matmul.
//
// HBM-bound (0.52 B read, 2 B written per weight). Each thread takes one 32-bit word of
// codes (8 weights inside one 64-weight block) per step, computes the block constant (the 8
// lanes of a block load the same constant inputs), looks the values up in a 16-entry shared
// table and writes 16 bytes of bf16, so every warp load and store is fully contiguous.
#include "common.cuh"
#include "host_cache.h"
#include "kernels.h"

namespace qn {

namespace {

constexpr int kDeqThreads = 256;

__global__ void __launch_bounds__(kDeqThreads)
k_dequant(const uint32_t *__restrict__ codes, const uint8_t *__restrict__ q, const float *__restrict__ sigma,
          const float *__restrict__ mu_p, const float *__restrict__ absmax, int qtype, int64_t n_words,
          uint4 *__restrict__ out) {
    __shared__ float s_t[16];
    if (threadIdx.x < 16) s_t[threadIdx.x] = table_value(qtype, threadIdx.x);
    __syncthreads();
    const float mu = load_mu(mu_p, absmax);
    const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
    // A thread expands one 32-bit code word (8 weights, 16 bytes of bf16) per step, so a warp
    // reads 128 contiguous bytes and writes 512; two steps are loaded before either is expanded.
    auto expand = [&](uint32_t w, int64_t word) {
        const int64_t b = word >> 3;  // 8 words = 64 weights = one block
        const float cp = load_block_constant(q, sigma, mu, absmax, b);
        uint4 o;
        uint32_t *op = reinterpret_cast<uint32_t *>(&o);
#pragma unroll
        for (int p = 0; p < 4; ++p) {
            const uint32_t lo = (w >> (8 * p)) & 15u, hi = (w >> (8 * p + 4)) & 15u;
            op[p] = pack_bf16x2(__fmul_rn(s_t[lo], cp), __fmul_rn(s_t[hi], cp));
        }
        out[word] = o;
    };
    for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n_words; i += 2 * stride) {
        const int64_t i2 = i + stride;
        const uint32_t w0 = __ldcs(codes + i);
        const uint32_t w1 = i2 < n_words ? __ldcs(codes + i2) : 0u;
        expand(w0, i);
        if (i2 < n_words) expand(w1, i2);
    }
}

}  // namespace

cudaError_t launch_dequant(const WeightView &w, uint16_t *out, cudaStream_t s) {
    const int64_t n_words = w.n * w.k / 8;  // 4 bytes of codes each
    if (n_words == 0) return cudaSuccess;
    int sms = 148, occ = 4;
    cudaError_t e = device_sm_count(&sms);
    if (e != cudaSuccess) return e;
    e = resident_ctas(reinterpret_cast<const void *>(k_dequant), kDeqThreads, 0, &occ);
    if (e != cudaSuccess) return e;
    int64_t grid = (n_words + 2 * kDeqThreads - 1) / (2 * kDeqThreads);
    const int64_t cap = static_cast<int64_t>(sms) * occ;  // one wave
    if (grid > cap) grid = cap;
    k_dequant<<<static_cast<unsigned>(grid), kDeqThreads, 0, s>>>(reinterpret_cast<const uint32_t *>(w.codes), w.q,
                                                                   w.sigma, w.mu, w.absmax, w.qtype, n_words,
                                                                   reinterpret_cast<uint4 *>(out));
    count_launch();
    return cudaGetLastError();
}

}  // namespace qn
