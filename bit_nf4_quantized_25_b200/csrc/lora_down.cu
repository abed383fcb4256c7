// lora_down.cu -- adapter down-projection for many tokens, the operand of the GEMM's
// extra up-projection steps:
//   fwd: t[m, j] = bf16(s * sum_k x[m,k] A[j,k])         (A: r x k)
//   bwd: u[m, j] = bf16(s * sum_n grad_h[m,n] B[n,j])    (B: n x r)
// written as a row-major M x RT bf16 matrix, RT = r rounded up to 64, zeros for j >= r.
// "How does QLoRA work for training?" (aivaro.ru), section 2: B (d x r), A (r x k).
//
// HBM-bound on the activations (read once). Main kernel (k_lora_down_tiled): a CTA takes 64
// tokens and a slice of the reduction; the activation tile (64 tokens x 64) and the adapter
// tile stream through a 4-stage ring of 16-byte asynchronous copies, four warps (16 tokens
// each) load their fragments with ldmatrix and run mma.sync m16n8k16 (tokens x adapter rank),
// and the slices of a cluster are summed through distributed shared memory in rank order, so
// the result does not depend on scheduling. Shapes whose rows are not 16-byte aligned take the
// per-element kernel (k_lora_down): 16 tokens per CTA, 4 warps splitting the reduction.
#include "common.cuh"
#include "dropout.cuh"
#include "host_cache.h"
#include "kernels.h"
#include "stream_common.cuh"

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

// ------------------------------------------------------------------ tiled kernel
constexpr int kTdTok = 64;          // tokens per CTA (4 warps x 16)
constexpr int kTdStages = 4;        // ring depth
constexpr int kTdThreads = 128;
constexpr int kTdMaxSplit = 8;      // reduction slices per cluster
constexpr uint32_t kTdTile = 8192;  // one 64 x 64 bf16 tile, 128-byte rows

struct TiledDownParams {
    const uint16_t *act;  // M x red, rows 16-byte aligned
    int64_t M, red;
    const uint16_t *small;  // col == 0: r x red row-major (element (j, kk) at small[j red + kk]);
                            // col == 1: red x r row-major (element (j, kk) at small[kk r + j])
    int col;
    int r, RT;
    float s;
    uint16_t *out;  // M x RT
    DropoutArgs drop;
    int nchunk;  // 64-element reduction chunks
};

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t &r0, uint32_t &r1, uint32_t &r2, uint32_t &r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t &r0, uint32_t &r1, uint32_t &r2, uint32_t &r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr));
}
__device__ __forceinline__ float ld_cluster_f32(uint32_t addr) {
    float v;
    asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(addr) : "memory");
    return v;
}

// Byte offset of 16-byte chunk c of row `row` in a tile of 128-byte rows (chunk ^ (row & 7)).
__device__ __forceinline__ uint32_t tswz(int row, int c) {
    return static_cast<uint32_t>(row * 128 + ((c ^ (row & 7)) << 4));
}

// RN adapter columns per pass (16, 32 or 64). Cluster (1, C, 1): rank c reduces chunks
// [nchunk c / C, nchunk (c + 1) / C) and finalises tokens [64 c / C, 64 (c + 1) / C).
template <int RN>
__global__ void __launch_bounds__(kTdThreads) k_lora_down_tiled(const TiledDownParams p) {
    extern __shared__ __align__(1024) uint8_t smem[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int C = static_cast<int>(gridDim.y);
    const int crank = static_cast<int>(blockIdx.y);
    const int64_t m0 = static_cast<int64_t>(blockIdx.x) * kTdTok;
    const int c_lo = p.nchunk * crank / C, c_hi = p.nchunk * (crank + 1) / C, nc = c_hi - c_lo;
    const uint32_t s_base = stream::saddr(smem);
    // stage s: the activation tile at 2 s kTdTile, the adapter tile after it
    auto x_tile = [&](int slot) { return s_base + static_cast<uint32_t>(slot) * 2u * kTdTile; };
    auto a_tile = [&](int slot) { return x_tile(slot) + kTdTile; };
    float *part = reinterpret_cast<float *>(smem);  // [64 tokens][RN] partial sums (the ring, reused)

    grid_dependency_wait();  // activations and adapters may come from the preceding kernel
    grid_dependents_launch();

    for (int j0 = 0; j0 < p.r; j0 += RN) {
        auto issue = [&](int ci, int slot) {
            const int64_t k0 = static_cast<int64_t>(c_lo + ci) * 64;
            // activations: 64 rows x 8 chunks
            for (int i = threadIdx.x; i < kTdTok * 8; i += kTdThreads) {
                const int row = i >> 3, c = i & 7;
                const int64_t m = m0 + row, kk = k0 + 8 * c;
                const bool v = m < p.M && kk < p.red;
                stream::cp_async16_zfill(x_tile(slot) + tswz(row, c), v ? p.act + m * p.red + kk : p.act,
                                         v ? 16u : 0u);
            }
            if (p.col == 0) {
                // adapter rows j0 .. j0 + RN, 8 chunks each
                for (int i = threadIdx.x; i < RN * 8; i += kTdThreads) {
                    const int jr = i >> 3, c = i & 7;
                    const int64_t kk = k0 + 8 * c;
                    const bool v = j0 + jr < p.r && kk < p.red;
                    stream::cp_async16_zfill(a_tile(slot) + tswz(jr, c),
                                             v ? p.small + static_cast<int64_t>(j0 + jr) * p.red + kk : p.small,
                                             v ? 16u : 0u);
                }
            } else {
                // 64 reduction rows x RN / 8 chunks of adapter columns
                for (int i = threadIdx.x; i < 64 * (RN / 8); i += kTdThreads) {
                    const int kr = i / (RN / 8), c = i % (RN / 8);
                    const int64_t kk = k0 + kr;
                    const bool v = kk < p.red && j0 + 8 * c < p.r;
                    stream::cp_async16_zfill(a_tile(slot) + tswz(kr, c), v ? p.small + kk * p.r + j0 + 8 * c : p.small,
                                             v ? 16u : 0u);
                }
            }
        };
        float acc[RN / 8][4];
#pragma unroll
        for (int nt = 0; nt < RN / 8; ++nt) acc[nt][0] = acc[nt][1] = acc[nt][2] = acc[nt][3] = 0.0f;
        for (int s = 0; s < kTdStages - 1; ++s) {
            if (s < nc) issue(s, s);
            stream::cp_async_commit();
        }
        for (int ci = 0; ci < nc; ++ci) {
            stream::cp_async_wait_n<kTdStages - 2>();
            __syncthreads();  // chunk ci has landed for every thread; the slot of chunk ci - 1 is free
            if (ci + kTdStages - 1 < nc) issue(ci + kTdStages - 1, (ci + kTdStages - 1) % kTdStages);
            stream::cp_async_commit();
            const int slot = ci % kTdStages;
            if (p.drop.thr != 0u) {
                // LoRA dropout: zero the dropped activations of the tile in place
                const int64_t k0 = static_cast<int64_t>(c_lo + ci) * 64;
                for (int i = threadIdx.x; i < kTdTok * 8; i += kTdThreads) {
                    const int row = i >> 3, c = i & 7;
                    const int64_t m = m0 + row, kk = k0 + 8 * c;
                    if (m >= p.M || kk >= p.red) continue;
                    const uint32_t a = x_tile(slot) + tswz(row, c);
                    const uint32_t keep =
                        dropout_keep_bits(p.drop, p.drop.offset + static_cast<uint64_t>(m * p.red + kk), 8);
                    uint4 v = stream::lds128(a);
                    v.x = mask_pair(v.x, keep);
                    v.y = mask_pair(v.y, keep >> 2);
                    v.z = mask_pair(v.z, keep >> 4);
                    v.w = mask_pair(v.w, keep >> 6);
                    asm volatile("st.shared.v4.b32 [%0], {%1,%2,%3,%4};" ::"r"(a), "r"(v.x), "r"(v.y), "r"(v.z),
                                 "r"(v.w)
                                 : "memory");
                }
                __syncthreads();
            }
            const uint32_t xa = x_tile(slot), aa = a_tile(slot);
            const int q = lane >> 3, rr = lane & 7;
#pragma unroll
            for (int k16 = 0; k16 < 4; ++k16) {
                uint32_t a0, a1, a2, a3;
                ldsm_x4(xa + tswz(16 * warp + (q & 1) * 8 + rr, 2 * k16 + (q >> 1)), a0, a1, a2, a3);
#pragma unroll
                for (int nt = 0; nt < RN / 8; nt += 2) {
                    uint32_t b0, b1, b2, b3;
                    if (p.col == 0)
                        ldsm_x4(aa + tswz(8 * (nt + (q >> 1)) + rr, 2 * k16 + (q & 1)), b0, b1, b2, b3);
                    else
                        ldsm_x4_t(aa + tswz(16 * k16 + (q & 1) * 8 + rr, nt + (q >> 1)), b0, b1, b2, b3);
                    mma_16816(acc[nt], a0, a1, a2, a3, b0, b1);
                    mma_16816(acc[nt + 1], a0, a1, a2, a3, b2, b3);
                }
            }
        }
        stream::cp_async_wait_n<0>();
        __syncthreads();  // every warp is done with the ring: it holds the partial sums now
        {
            const int g = lane >> 2, t = lane & 3;
#pragma unroll
            for (int nt = 0; nt < RN / 8; ++nt) {
                const int row = 16 * warp + g, cj = 8 * nt + 2 * t;
                part[row * RN + cj] = acc[nt][0];
                part[row * RN + cj + 1] = acc[nt][1];
                part[(row + 8) * RN + cj] = acc[nt][2];
                part[(row + 8) * RN + cj + 1] = acc[nt][3];
            }
        }
        if (C > 1) {
            stream::cluster_arrive_release();
            stream::cluster_wait_acquire();
        } else {
            __syncthreads();
        }
        // this rank's tokens: the C partial sums in rank order, scaled, as bf16; on the last pass
        // also the zero columns up to RT
        const bool last = j0 + RN >= p.r;
        const int t_lo = kTdTok * crank / C, t_hi = kTdTok * (crank + 1) / C;
        const int cols = last ? p.RT - j0 : RN;
        for (int i = threadIdx.x; i < (t_hi - t_lo) * cols; i += kTdThreads) {
            const int tl = t_lo + i / cols, cj = i % cols;
            const int64_t m = m0 + tl;
            if (m >= p.M) continue;
            float v = 0.0f;
            if (cj < RN && j0 + cj < p.r) {
                if (C > 1) {
                    const uint32_t a = stream::saddr(part + tl * RN + cj);
                    for (int src = 0; src < C; ++src) v += ld_cluster_f32(stream::mapa(a, static_cast<uint32_t>(src)));
                } else {
                    v = part[tl * RN + cj];
                }
                v *= p.s;
            }
            p.out[m * p.RT + j0 + cj] = __bfloat16_as_ushort(__float2bfloat16_rn(v));
        }
        // no CTA refills its ring (or exits) while another rank still reads its partial sums
        if (C > 1) {
            stream::cluster_arrive_release();
            stream::cluster_wait_acquire();
        } else {
            __syncthreads();
        }
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

namespace {

// The tiled kernel: rows of the activation and of the adapter 16-byte aligned (a row-major r x red
// adapter, or red x r with r % 8 == 0), RT a multiple of 64 (so every pass's columns exist).
cudaError_t launch_lora_down_tiled(const uint16_t *act, int64_t M, int64_t red, const uint16_t *small, int col, int r,
                                   float s, uint16_t *out, int RT, cudaStream_t st, const DropoutArgs &drop) {
    TiledDownParams p{act, M, red, small, col, r, RT, s, out, drop, static_cast<int>((red + 63) / 64)};
    const int RN = r <= 16 ? 16 : r <= 32 ? 32 : 64;
    const void *kern = RN == 16   ? reinterpret_cast<const void *>(k_lora_down_tiled<16>)
                       : RN == 32 ? reinterpret_cast<const void *>(k_lora_down_tiled<32>)
                                  : reinterpret_cast<const void *>(k_lora_down_tiled<64>);
    const size_t smem = static_cast<size_t>(kTdStages) * 2 * kTdTile;
    cudaError_t e = ensure_smem_limit(kern, smem);
    if (e != cudaSuccess) return e;
    int sms = 148;
    e = device_sm_count(&sms);
    if (e != cudaSuccess) return e;
    // reduction slices: about two CTAs per SM in all, at most 8, at most one per chunk
    const int64_t tiles = (M + kTdTok - 1) / kTdTok;
    int64_t C = (2 * sms + tiles - 1) / tiles;
    if (C > kTdMaxSplit) C = kTdMaxSplit;
    if (C > p.nchunk) C = p.nchunk;
    if (C < 1) C = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(tiles), static_cast<unsigned>(C), 1);
    cfg.blockDim = dim3(kTdThreads, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    attr[1].id = cudaLaunchAttributeClusterDimension;
    attr[1].val.clusterDim.x = 1;
    attr[1].val.clusterDim.y = static_cast<unsigned>(C);
    attr[1].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    if (RN == 16)
        e = cudaLaunchKernelEx(&cfg, k_lora_down_tiled<16>, p);
    else if (RN == 32)
        e = cudaLaunchKernelEx(&cfg, k_lora_down_tiled<32>, p);
    else
        e = cudaLaunchKernelEx(&cfg, k_lora_down_tiled<64>, p);
    count_launch();
    return e;
}

bool aligned16p(const void *q) { return (reinterpret_cast<uintptr_t>(q) & 15u) == 0; }

}  // namespace

cudaError_t launch_lora_down(const uint16_t *act, int64_t M, int64_t red, const uint16_t *small, int64_t ldj,
                             int64_t ldk, int r, float s, uint16_t *out, int RT, cudaStream_t st,
                             const DropoutArgs *drop) {
    if (M <= 0 || r <= 0) return cudaSuccess;
    const DropoutArgs dz = drop ? *drop : DropoutArgs{0, 0, 0};
    if (red % 8 == 0 && RT % 64 == 0 && aligned16p(act) && aligned16p(small)) {
        if (ldk == 1 && ldj == red) return launch_lora_down_tiled(act, M, red, small, 0, r, s, out, RT, st, dz);
        if (ldj == 1 && ldk == r && r % 8 == 0)
            return launch_lora_down_tiled(act, M, red, small, 1, r, s, out, RT, st, dz);
    }
    LoraDownParams p{act, M, red, small, ldj, ldk, r, s, out, RT, dz};
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
