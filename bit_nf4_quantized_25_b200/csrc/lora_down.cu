// lora_down.cu -- adapter down-projection for many tokens, the operand of the GEMM's
// extra up-projection steps:
//   fwd: t[m, j] = bf16(s * sum_k x[m,k] A[j,k])         (A: r x k)
//   bwd: u[m, j] = bf16(s * sum_n grad_h[m,n] B[n,j])    (B: n x r)
// written as a row-major M x RT bf16 matrix, RT = r rounded up to 64, zeros for j >= r.
// "How does QLoRA work for training?" (aivaro.ru), section 2: B (d x r), A (r x k).
//
// HBM-bound on the activations (read once). One CTA = 16 tokens; its 4 warps split the
// reduction, each running mma.sync m16n8k16 (tokens x adapter rank), and reduce through
// shared memory in a fixed order.
#include "common.cuh"
#include "dropout.cuh"
#include "kernels.h"

namespace qn {

namespace {

constexpr int kLdWarps = 4;

struct LoraDownParams {
    const uint16_t *act;  // M x red
    int64_t M, red;
    const uint16_t *small;  // element (j, kk) at small[j * ldj + kk * ldk]
    int64_t ldj, ldk;
    int r;
    float s;
    uint16_t *out;  // M x RT
    int RT;
    DropoutArgs drop;  // mask of act's elements (thr == 0: none)
};

// bf16 pair (v[i], v[i + 1]); kEven: i is even and v 4-byte aligned, so one 4-byte load.
template <bool kEven>
__device__ __forceinline__ uint32_t load_pair(const uint16_t *v) {
    if (kEven) return ld_ro_u32(v);
    return static_cast<uint32_t>(ld_ro_u16(v)) | (static_cast<uint32_t>(ld_ro_u16(v + 1)) << 16);
}

// kEven: the reduction length (the activation row stride) is even, so every activation pair
// and every pair of a row-major small operand is 4-byte aligned.
template <int NT, bool kEven>  // 8*NT adapter columns per pass
__global__ void __launch_bounds__(kLdWarps * 32) k_lora_down(const LoraDownParams p) {
    __shared__ float red[kLdWarps][16][8 * NT];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, t = lane & 3;
    const int64_t m0 = static_cast<int64_t>(blockIdx.x) * 16;
    const int64_t rowA = m0 + g, rowB = m0 + g + 8;
    const bool vA = rowA < p.M, vB = rowB < p.M;
    const uint16_t *aA = p.act + (vA ? rowA : 0) * p.red;
    const uint16_t *aB = p.act + (vB ? rowB : 0) * p.red;
    const int64_t steps = (p.red + 15) / 16;  // a partial last step reads zeros
    const int64_t s_lo = steps * warp / kLdWarps, s_hi = steps * (warp + 1) / kLdWarps;

    for (int j0 = 0; j0 < p.RT; j0 += 8 * NT) {
        float d[NT][4];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) d[nt][0] = d[nt][1] = d[nt][2] = d[nt][3] = 0.0f;
        if (j0 < p.r) {
            for (int64_t st = s_lo; st < s_hi; ++st) {
                const int64_t k0 = st * 16;
                const bool lo_ok = k0 + 2 * t < p.red, hi_ok = k0 + 2 * t + 8 < p.red;
                // a pair never straddles the row end: red is even, or (odd red) the last pair is
                // read element-wise below
                auto pair = [&](const uint16_t *row, int64_t kk) -> uint32_t {
                    if (kk + 1 < p.red) return load_pair<kEven>(row + kk);
                    return kk < p.red ? static_cast<uint32_t>(ld_ro_u16(row + kk)) : 0u;
                };
                uint32_t a0 = (vA && lo_ok) ? pair(aA, k0 + 2 * t) : 0u;
                uint32_t a1 = (vB && lo_ok) ? pair(aB, k0 + 2 * t) : 0u;
                uint32_t a2 = (vA && hi_ok) ? pair(aA, k0 + 2 * t + 8) : 0u;
                uint32_t a3 = (vB && hi_ok) ? pair(aB, k0 + 2 * t + 8) : 0u;
                if (p.drop.thr != 0u) {
                    // LoRA dropout of the activation: element (m, i) at index offset + m red + i
                    const uint64_t eA = p.drop.offset + static_cast<uint64_t>(rowA * p.red + k0 + 2 * t);
                    const uint64_t eB = p.drop.offset + static_cast<uint64_t>(rowB * p.red + k0 + 2 * t);
                    a0 = mask_pair(a0, dropout_keep_bits(p.drop, eA, 2));
                    a1 = mask_pair(a1, dropout_keep_bits(p.drop, eB, 2));
                    a2 = mask_pair(a2, dropout_keep_bits(p.drop, eA + 8, 2));
                    a3 = mask_pair(a3, dropout_keep_bits(p.drop, eB + 8, 2));
                }
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) {
                    const int j = j0 + nt * 8 + g;
                    uint32_t b0 = 0u, b1 = 0u;
                    if (j < p.r) {
                        const uint16_t *sp = p.small + static_cast<int64_t>(j) * p.ldj;
                        if (p.ldk == 1) {
                            if (lo_ok) b0 = pair(sp, k0 + 2 * t);
                            if (hi_ok) b1 = pair(sp, k0 + 2 * t + 8);
                        } else {
                            const int64_t L = p.ldk;
                            if (lo_ok)
                                b0 = ld_ro_u16(sp + (k0 + 2 * t) * L) |
                                     (k0 + 2 * t + 1 < p.red
                                          ? static_cast<uint32_t>(ld_ro_u16(sp + (k0 + 2 * t + 1) * L)) << 16
                                          : 0u);
                            if (hi_ok)
                                b1 = ld_ro_u16(sp + (k0 + 2 * t + 8) * L) |
                                     (k0 + 2 * t + 9 < p.red
                                          ? static_cast<uint32_t>(ld_ro_u16(sp + (k0 + 2 * t + 9) * L)) << 16
                                          : 0u);
                        }
                    }
                    mma_16816(d[nt], a0, a1, a2, a3, b0, b1);
                }
            }
        }
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            red[warp][g][nt * 8 + 2 * t] = d[nt][0];
            red[warp][g][nt * 8 + 2 * t + 1] = d[nt][1];
            red[warp][g + 8][nt * 8 + 2 * t] = d[nt][2];
            red[warp][g + 8][nt * 8 + 2 * t + 1] = d[nt][3];
        }
        __syncthreads();
        for (int i = threadIdx.x; i < 16 * 8 * NT; i += blockDim.x) {
            const int row = i / (8 * NT), col = i % (8 * NT);
            const int64_t m = m0 + row;
            const int j = j0 + col;
            if (m < p.M && j < p.RT) {
                float v = 0.0f;
                if (j < p.r) {
#pragma unroll
                    for (int w = 0; w < kLdWarps; ++w) v += red[w][row][col];
                    v *= p.s;
                }
                p.out[m * p.RT + j] = __bfloat16_as_ushort(__float2bfloat16_rn(v));
            }
        }
        __syncthreads();
    }
}

// Adapter term of the input gradient under dropout: gx[m, k] += keep(m, k) sum_j u[m, j] A[j, k].
// A CTA owns 32 tokens x 128 features; thread (ty, tx) accumulates tokens 4 ty .. + 4 and features
// 4 tx .. + 4 in fp32 over rank chunks of 64 staged in shared memory (u transposed, A row-major).
constexpr int kUpTok = 32, kUpFeat = 128, kUpRank = 64;

struct UpParams {
    const uint16_t *u;  // M x RT
    int64_t M;
    int RT;
    const uint16_t *A;  // r x k
    int r;
    int64_t k;
    DropoutArgs drop;
    uint16_t *gx;  // M x k
};

__global__ void __launch_bounds__(256) k_adapter_up_masked(const UpParams p) {
    __shared__ __align__(16) uint16_t uT[kUpRank][kUpTok];
    __shared__ __align__(16) uint16_t As[kUpRank][kUpFeat];
    const int ty = threadIdx.x >> 5, tx = threadIdx.x & 31;
    const int64_t m0 = static_cast<int64_t>(blockIdx.y) * kUpTok, f0 = static_cast<int64_t>(blockIdx.x) * kUpFeat;
    float acc[4][4] = {};
    for (int j0 = 0; j0 < p.RT && j0 < p.r; j0 += kUpRank) {
        for (int i = threadIdx.x; i < kUpRank * kUpTok; i += 256) {
            const int j = i / kUpTok, tk = i % kUpTok;
            const int64_t m = m0 + tk;
            uT[j][tk] = (m < p.M && j0 + j < p.RT) ? ld_ro_u16(p.u + m * p.RT + j0 + j) : static_cast<uint16_t>(0);
        }
        for (int i = threadIdx.x; i < kUpRank * kUpFeat; i += 256) {
            const int j = i / kUpFeat, f = i % kUpFeat;
            As[j][f] = (j0 + j < p.r && f0 + f < p.k) ? ld_ro_u16(p.A + static_cast<int64_t>(j0 + j) * p.k + f0 + f)
                                                      : static_cast<uint16_t>(0);
        }
        __syncthreads();
        for (int j = 0; j < kUpRank; ++j) {
            const uint2 uv = *reinterpret_cast<const uint2 *>(&uT[j][4 * ty]);
            const uint2 av = *reinterpret_cast<const uint2 *>(&As[j][4 * tx]);
            const float uu[4] = {bf16_lo(uv.x), bf16_hi(uv.x), bf16_lo(uv.y), bf16_hi(uv.y)};
            const float aa[4] = {bf16_lo(av.x), bf16_hi(av.x), bf16_lo(av.y), bf16_hi(av.y)};
#pragma unroll
            for (int a = 0; a < 4; ++a)
#pragma unroll
                for (int b = 0; b < 4; ++b) acc[a][b] = __fmaf_rn(uu[a], aa[b], acc[a][b]);
        }
        __syncthreads();
    }
#pragma unroll
    for (int a = 0; a < 4; ++a) {
        const int64_t m = m0 + 4 * ty + a;
        const int64_t f = f0 + 4 * tx;
        if (m >= p.M) continue;
        const uint32_t keep = dropout_keep_bits(p.drop, p.drop.offset + static_cast<uint64_t>(m * p.k + f), 4);
#pragma unroll
        for (int b = 0; b < 4; ++b) {
            if (f + b >= p.k || !(keep & (1u << b))) continue;
            uint16_t *dst = p.gx + m * p.k + f + b;
            const float v = __uint_as_float(static_cast<uint32_t>(*dst) << 16) + acc[a][b];
            *dst = __bfloat16_as_ushort(__float2bfloat16_rn(v));
        }
    }
}

}  // namespace

cudaError_t launch_adapter_up_masked(const uint16_t *u, int64_t M, int RT, const uint16_t *A, int r, int64_t k,
                                     const DropoutArgs &drop, uint16_t *gx, cudaStream_t st) {
    if (M <= 0 || k <= 0 || r <= 0) return cudaSuccess;
    UpParams p{u, M, RT, A, r, k, drop, gx};
    const dim3 grid(static_cast<unsigned>((k + kUpFeat - 1) / kUpFeat), static_cast<unsigned>((M + kUpTok - 1) / kUpTok));
    k_adapter_up_masked<<<grid, 256, 0, st>>>(p);
    count_launch();
    return cudaGetLastError();
}

cudaError_t launch_lora_down(const uint16_t *act, int64_t M, int64_t red, const uint16_t *small, int64_t ldj,
                             int64_t ldk, int r, float s, uint16_t *out, int RT, cudaStream_t st,
                             const DropoutArgs *drop) {
    LoraDownParams p{act, M, red, small, ldj, ldk, r, s, out, RT, drop ? *drop : DropoutArgs{0, 0, 0}};
    const unsigned grid = static_cast<unsigned>((M + 15) / 16);
    const bool even = (red & 1) == 0;
    auto go = [&](auto kern) { kern<<<grid, kLdWarps * 32, 0, st>>>(p); };
    if (r <= 8)
        even ? go(k_lora_down<1, true>) : go(k_lora_down<1, false>);
    else if (r <= 16)
        even ? go(k_lora_down<2, true>) : go(k_lora_down<2, false>);
    else if (r <= 32)
        even ? go(k_lora_down<4, true>) : go(k_lora_down<4, false>);
    else
        even ? go(k_lora_down<8, true>) : go(k_lora_down<8, false>);
    count_launch();
    return cudaGetLastError();
}

}  // namespace qn
