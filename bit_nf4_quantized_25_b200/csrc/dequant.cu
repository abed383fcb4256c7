// dequant.cu -- nf4_dequantize on sm_100a: codes + double-quantised constants -> bf16 W.
//
// W'[e] = bf16_rn(fl32(NF4[code_e] * c'_b)), c'_b = fma(e4m3(q_b), sigma_g, mu).
// "Quantized LoRA (QLoRA) and 4-bit training" (apxml.com): the 4-bit weights are
// dequantised to the bf16 compute type for the matmul.
//
// HBM-bound (0.52 B read, 2 B written per weight). Each thread takes 16 bytes of codes
// (32 weights, always inside one 64-weight block), computes the block constant once,
// looks the 16 table values up in shared memory (16 distinct words: conflict-free) and
// writes 64 bytes of bf16.
#include "common.cuh"
#include "kernels.h"

namespace qn {

namespace {

constexpr int kDeqThreads = 256;

__global__ void __launch_bounds__(kDeqThreads)
k_dequant(const uint4 *__restrict__ codes, const uint8_t *__restrict__ q, const float *__restrict__ sigma,
          const float *__restrict__ mu_p, int64_t n_vec, uint4 *__restrict__ out) {
    __shared__ float s_t[16];
    if (threadIdx.x < 16) s_t[threadIdx.x] = nf4_value(threadIdx.x);
    __syncthreads();
    const float mu = __ldg(mu_p);
    const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
    for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n_vec; i += stride) {
        const uint4 c = ld_nc_v4(codes + i);
        const int64_t b = i >> 1;  // 16 bytes = 32 weights = half a block
        const float cp = block_constant(__ldg(q + b), __ldg(sigma + b / kGroup), mu);
        const uint32_t w[4] = {c.x, c.y, c.z, c.w};
        uint4 o[4];
        uint32_t *op = reinterpret_cast<uint32_t *>(o);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
#pragma unroll
            for (int p = 0; p < 4; ++p) {
                const uint32_t lo = (w[j] >> (8 * p)) & 15u, hi = (w[j] >> (8 * p + 4)) & 15u;
                op[j * 4 + p] = pack_bf16x2(__fmul_rn(s_t[lo], cp), __fmul_rn(s_t[hi], cp));
            }
        }
        uint4 *dst = out + i * 4;
#pragma unroll
        for (int j = 0; j < 4; ++j) dst[j] = o[j];
    }
}

}  // namespace

cudaError_t launch_dequant(const WeightView &w, uint16_t *out, cudaStream_t s) {
    const int64_t n_vec = w.n * w.k / 32;  // 16 bytes of codes each
    if (n_vec == 0) return cudaSuccess;
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    int64_t grid = (n_vec + kDeqThreads - 1) / kDeqThreads;
    const int64_t cap = static_cast<int64_t>(sms) * 16;
    if (grid > cap) grid = cap;
    k_dequant<<<static_cast<unsigned>(grid), kDeqThreads, 0, s>>>(reinterpret_cast<const uint4 *>(w.codes), w.q,
                                                                   w.sigma, w.mu, n_vec, reinterpret_cast<uint4 *>(out));
    count_launch();
    return cudaGetLastError();
}

}  // namespace qn
