// decode.cu -- QLoRA linear forward and input gradient for few tokens (M <= 64) on sm_100a.
//
//   fwd : h[m,n]      = sum_k W'[n,k] x[m,k]      + sum_j B[n,j] t[m,j],  t = s A x
//   bwd : grad_x[m,k] = sum_n grad_h[m,n] W'[n,k] + sum_j A[j,k] u[m,j],  u = s B^T grad_h
// with W'[n,k] = NF4[code] * c'_b ("Quantized LoRA (QLoRA) and 4-bit training", apxml.com,
// forward equations; "How does QLoRA work for training?", aivaro.ru, sections 2 and 7).
//
// Few tokens make this HBM-bound: each packed weight is read once and used M times. B200
// streams about 13e12 weights/s but its SMs issue only ~3.6e13 lane-instructions/s, so the
// whole per-weight budget is under three instructions. The multiply-accumulate therefore
// runs on the tensor cores (mma.sync m16n8k16: A = 16 weight rows, B = 8 tokens) and the
// dequantisation is one byte permute plus one shared-memory load per TWO weights: a
// 256-entry table maps a code byte (two nibbles) to a bf16 pair. The table is stored once
// per lane in 256-byte rows, so the permute that extracts the byte also forms the
// conflict-free address (byte << 8 | lane << 2).
//   - fwd: the table holds the unscaled NF4 values; every 64-weight block is reduced in its
//     own fp32 fragment and scaled by its constant c'_b (the same sum, constant applied after
//     the dot product). A lane computes the constants of one block per group of four and the
//     quad shares them with shuffles.
//   - bwd: the reduction runs over rows, whose constants differ, so the constants scale the
//     bf16 token operand (c'_b * grad_h), and the nibbles of neighbouring rows are
//     interleaved so that a byte again indexes a pair.
// The reduction is split across a thread-block cluster (<= 8 CTAs); partial sums and the
// LoRA down-projection are exchanged through distributed shared memory, so a layer is one
// launch with no workspace. Codes stream through a two-group register ring; before the
// programmatic-launch wait each warp asks L2 to prefetch its whole code slice (an L2
// prefetch cannot return stale data), so the DRAM latency overlaps the preceding kernel.
#include <cooperative_groups.h>

#include "common.cuh"
#include "kernels.h"

namespace cg = cooperative_groups;

namespace qn {

namespace {

constexpr int kDecWarps = 8;
constexpr int kDecThreads = kDecWarps * 32;
constexpr int kLutBytes = 256 * 256;  // 256 code bytes x 256-byte rows (32 lane copies used)
constexpr int kMaxCluster = 8;
constexpr int kFwdRows = 16 * kDecWarps;  // weight rows per forward CTA
constexpr int kBwdCols = 2;               // 64-feature block columns per input-gradient CTA
constexpr int kBwdSub = kDecWarps / kBwdCols;  // reduction sub-slices inside a CTA

struct DecodeParams {
    const uint8_t *codes;
    const uint8_t *q;
    const float *sigma;
    const float *mu;
    int64_t n, k;         // W is n x k
    const uint16_t *act;  // fwd: x (M x k); bwd: grad_h (M x n)
    int M;
    const uint16_t *A;  // r x k
    const uint16_t *B;  // n x r
    int r;
    float s;
    uint16_t *out;  // fwd: h (M x n); bwd: grad_x (M x k)
};

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
    uint32_t d;
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
    return d;
}

// Pair table: row e (a code byte) holds bf16x2(NF4[e & 15], NF4[e >> 4]) in its first 32
// words, one copy per lane.
__device__ __forceinline__ void build_pair_lut(uint8_t *lut) {
    uint4 *l4 = reinterpret_cast<uint4 *>(lut);
    for (int i = threadIdx.x; i < 256 * 8; i += blockDim.x) {
        const int e = i >> 3, c = i & 7;
        const uint32_t v = pack_bf16x2(nf4_value(e & 15), nf4_value(e >> 4));
        l4[e * 16 + c] = make_uint4(v, v, v, v);
    }
}

// Pair for byte i (0..3) of word w: the permute builds (byte << 8) | (lane << 2).
__device__ __forceinline__ uint32_t lut_pair(const uint8_t *lut, uint32_t w, uint32_t lane4, int i) {
    const uint32_t off = prmt(w, lane4, 0x5504u | (static_cast<uint32_t>(i) << 4));
    return *reinterpret_cast<const uint32_t *>(lut + off);
}

__device__ __forceinline__ float round_bf16(float v) { return __bfloat162float(__float2bfloat16_rn(v)); }

__device__ __forceinline__ void prefetch_l2(const void *p, uint32_t bytes) {
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(p), "r"(bytes) : "memory");
}

__device__ __forceinline__ void prefetch_line(const void *p) {
    asm volatile("prefetch.global.L2 [%0];" ::"l"(p) : "memory");
}

// L2 prefetch of an arbitrary byte range [p, p + bytes): 16-byte-aligned bulk part plus the
// cache lines at the ragged ends.
__device__ __forceinline__ void prefetch_range(const void *p, int64_t bytes) {
    if (bytes <= 0) return;
    const uintptr_t a = reinterpret_cast<uintptr_t>(p), e = a + static_cast<uintptr_t>(bytes);
    const uintptr_t a16 = (a + 15) & ~uintptr_t(15), e16 = e & ~uintptr_t(15);
    if (e16 > a16) prefetch_l2(reinterpret_cast<const void *>(a16), static_cast<uint32_t>(e16 - a16));
    prefetch_line(p);
    prefetch_line(reinterpret_cast<const void *>(e - 1));
}

// Split cluster barrier: arrive once this CTA has finished reading remote shared memory,
// wait (before exiting) until every CTA has.
__device__ __forceinline__ void cluster_arrive_release() {
    asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory");
}
__device__ __forceinline__ void cluster_wait_acquire() { asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory"); }

// L2 prefetch (before the dependency wait) of the activation slice, the adapter slice and the
// adapter rows the finalising CTA will read: with every operand already on its way to L2 the
// kernel pays one DRAM round trip instead of a chain of them.
__device__ __forceinline__ void prefetch_operands(const DecodeParams &p, int b_lo, int b_hi, int64_t row0, int rows,
                                                  int crank, int C) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t K = p.k;
    const int64_t kbytes = static_cast<int64_t>(b_hi - b_lo) * 128;  // 64 bf16 per block
    if (warp == 0 && lane < p.M && kbytes > 0)
        prefetch_l2(p.act + lane * K + static_cast<int64_t>(b_lo) * 64, static_cast<uint32_t>(kbytes));
    if (warp == 1 && p.r > 0) {
        for (int j = lane; j < p.r; j += 32)
            if (kbytes > 0) prefetch_l2(p.A + j * K + static_cast<int64_t>(b_lo) * 64, static_cast<uint32_t>(kbytes));
        const int r_lo = rows * crank / C, r_hi = rows * (crank + 1) / C;
        const int64_t n_lo = row0 + r_lo, n_hi = row0 + r_hi < p.n ? row0 + r_hi : p.n;
        if (lane == 0 && n_hi > n_lo) prefetch_range(p.B + n_lo * p.r, (n_hi - n_lo) * p.r * 2);
    }
}

// ------------------------------------------------------------------------- forward
// Registers of one group of four 64-weight blocks for rows A (g) and B (g + 8) of a lane.
struct FwdGroup {
    uint2 ca[4], cb[4];
    uint32_t qa, qb;  // this lane's block (t) of the group
    float sa, sb;
};

template <int NG>
__global__ void __launch_bounds__(kDecThreads)
k_decode_fwd(const DecodeParams p) {
    constexpr int MP = 8 * NG;  // padded token count
    extern __shared__ __align__(16) uint8_t smem[];
    uint8_t *lut = smem;
    float *part = reinterpret_cast<float *>(smem + kLutBytes);  // [kFwdRows][MP]
    const int rpad = (p.r + 15) & ~15;
    float *tpart = part + kFwdRows * MP;  // [rpad][MP] partial A x of this CTA's k-slice
    float *tfull = tpart + rpad * MP;     // [rpad][MP] s * A x, rounded to bf16

    cg::cluster_group cluster = cg::this_cluster();
    const int C = static_cast<int>(cluster.num_blocks());
    const int crank = static_cast<int>(cluster.block_rank());
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, t = lane & 3;
    const uint32_t lane4 = static_cast<uint32_t>(lane) << 2;

    const int64_t N = p.n, K = p.k;
    const int nbr = static_cast<int>(K / kBlock);
    const int b_lo = static_cast<int>(static_cast<int64_t>(nbr) * crank / C);
    const int b_hi = static_cast<int>(static_cast<int64_t>(nbr) * (crank + 1) / C);
    const int64_t row_base = static_cast<int64_t>(blockIdx.y) * kFwdRows + warp * 16;

    // Before the dependency wait: on-chip setup and an L2 prefetch of the weight codes.
    build_pair_lut(lut);
    for (int i = threadIdx.x; i < rpad * MP; i += blockDim.x) tpart[i] = 0.0f;
    if (lane < 16 && row_base + lane < N && b_hi > b_lo) {
        const int64_t row = row_base + lane;
        prefetch_l2(p.codes + row * (K / 2) + static_cast<int64_t>(b_lo) * 32, static_cast<uint32_t>(b_hi - b_lo) * 32u);
        prefetch_range(p.q + row * nbr + b_lo, b_hi - b_lo);
        prefetch_line(p.sigma + (row * nbr + b_lo) / kGroup);
    }
    prefetch_operands(p, b_lo, b_hi, static_cast<int64_t>(blockIdx.y) * kFwdRows, kFwdRows, crank, C);
    __syncthreads();
    grid_dependency_wait();

    const float mu = __ldg(p.mu);
    const int M = p.M;
    const int64_t rowA = row_base + g, rowB = rowA + 8;
    const bool vA = rowA < N, vB = rowB < N;
    const uint8_t *cA = p.codes + (vA ? rowA : 0) * (K / 2) + 8 * t;
    const uint8_t *cB = p.codes + (vB ? rowB : 0) * (K / 2) + 8 * t;
    const int64_t qA = (vA ? rowA : 0) * nbr, qB = (vB ? rowB : 0) * nbr;

    auto load_group = [&](int b0, FwdGroup &G) {
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int b = b0 + j;
            G.ca[j] = (vA && b < b_hi) ? __ldcs(reinterpret_cast<const uint2 *>(cA + static_cast<int64_t>(b) * 32))
                                       : make_uint2(0u, 0u);
            G.cb[j] = (vB && b < b_hi) ? __ldcs(reinterpret_cast<const uint2 *>(cB + static_cast<int64_t>(b) * 32))
                                       : make_uint2(0u, 0u);
        }
        const int bt = b0 + t;
        const bool ok = bt < b_hi;
        G.qa = (vA && ok) ? __ldg(p.q + qA + bt) : 0u;
        G.qb = (vB && ok) ? __ldg(p.q + qB + bt) : 0u;
        G.sa = (vA && ok) ? __ldg(p.sigma + (qA + bt) / kGroup) : 0.0f;
        G.sb = (vB && ok) ? __ldg(p.sigma + (qB + bt) / kGroup) : 0.0f;
    };

    // x rows of this lane's tokens: x[tg*8 + g][64b + 16t .. +16]
    const uint16_t *xrow[NG];
    bool xv[NG];
#pragma unroll
    for (int tg = 0; tg < NG; ++tg) {
        const int tok = tg * 8 + g;
        xv[tg] = tok < M;
        xrow[tg] = p.act + static_cast<int64_t>(xv[tg] ? tok : 0) * K + 16 * t;
    }

    float acc[NG][4];
#pragma unroll
    for (int tg = 0; tg < NG; ++tg) acc[tg][0] = acc[tg][1] = acc[tg][2] = acc[tg][3] = 0.0f;

    FwdGroup cur, nxt;
    if (b_lo < b_hi) load_group(b_lo, cur);

    // ---- LoRA down-projection over this CTA's k-slice (partial t = A x, fp32), while the
    // first codes are in flight. Item (j-tile, eighth of the slice) per warp.
    if (p.r > 0) {
        const int rt = rpad / 16;
        const int nsl = b_hi - b_lo;
        const int s_lo = b_lo + nsl * warp / kDecWarps, s_hi = b_lo + nsl * (warp + 1) / kDecWarps;
        for (int jt = 0; jt < rt; ++jt) {
            const int jA = jt * 16 + g, jB = jA + 8;
            const bool aA = jA < p.r, aB = jB < p.r;
            const uint16_t *pa = p.A + static_cast<int64_t>(aA ? jA : 0) * K + 16 * t;
            const uint16_t *pb = p.A + static_cast<int64_t>(aB ? jB : 0) * K + 16 * t;
            float d[NG][4];
#pragma unroll
            for (int tg = 0; tg < NG; ++tg) d[tg][0] = d[tg][1] = d[tg][2] = d[tg][3] = 0.0f;
            for (int b = s_lo; b < s_hi; ++b) {
                const int64_t o = static_cast<int64_t>(b) * 64;
                uint4 a0 = make_uint4(0u, 0u, 0u, 0u), a1 = a0, b0 = a0, b1 = a0;
                if (aA) {
                    a0 = ld_ro_v4(pa + o);
                    a1 = ld_ro_v4(pa + o + 8);
                }
                if (aB) {
                    b0 = ld_ro_v4(pb + o);
                    b1 = ld_ro_v4(pb + o + 8);
                }
                const uint32_t ra[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
                const uint32_t rb[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll
                for (int tg = 0; tg < NG; ++tg) {
                    uint4 x0 = make_uint4(0u, 0u, 0u, 0u), x1 = x0;
                    if (xv[tg]) {
                        x0 = ld_ro_v4(xrow[tg] + o);
                        x1 = ld_ro_v4(xrow[tg] + o + 8);
                    }
                    const uint32_t xw[8] = {x0.x, x0.y, x0.z, x0.w, x1.x, x1.y, x1.z, x1.w};
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        mma_16816(d[tg], ra[2 * kk], rb[2 * kk], ra[2 * kk + 1], rb[2 * kk + 1], xw[2 * kk],
                                  xw[2 * kk + 1]);
                }
            }
#pragma unroll
            for (int tg = 0; tg < NG; ++tg) {
                const int jl = jt * 16 + g;
                atomicAdd(&tpart[jl * MP + tg * 8 + 2 * t], d[tg][0]);
                atomicAdd(&tpart[jl * MP + tg * 8 + 2 * t + 1], d[tg][1]);
                atomicAdd(&tpart[(jl + 8) * MP + tg * 8 + 2 * t], d[tg][2]);
                atomicAdd(&tpart[(jl + 8) * MP + tg * 8 + 2 * t + 1], d[tg][3]);
            }
        }
    }

    // ---- base: blocks [b_lo, b_hi) of rows A and B, groups of four, double-buffered.
    for (int b0 = b_lo; b0 < b_hi; b0 += 4) {
        if (b0 + 4 < b_hi) load_group(b0 + 4, nxt);
        const float cA4 = vA ? block_constant(static_cast<uint8_t>(cur.qa), cur.sa, mu) : 0.0f;
        const float cB4 = vB ? block_constant(static_cast<uint8_t>(cur.qb), cur.sb, mu) : 0.0f;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int b = b0 + j;
            if (b >= b_hi) break;
            const float cpA = __shfl_sync(0xffffffffu, cA4, (lane & ~3) | j);
            const float cpB = __shfl_sync(0xffffffffu, cB4, (lane & ~3) | j);
            uint32_t af[4][4];
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
                const uint32_t wa = kk < 2 ? cur.ca[j].x : cur.ca[j].y, wb = kk < 2 ? cur.cb[j].x : cur.cb[j].y;
                const int i0 = (2 * kk) & 3;
                af[kk][0] = lut_pair(lut, wa, lane4, i0);
                af[kk][2] = lut_pair(lut, wa, lane4, i0 + 1);
                af[kk][1] = lut_pair(lut, wb, lane4, i0);
                af[kk][3] = lut_pair(lut, wb, lane4, i0 + 1);
            }
            const int64_t o = static_cast<int64_t>(b) * 64;
#pragma unroll
            for (int tg = 0; tg < NG; ++tg) {
                uint4 x0 = make_uint4(0u, 0u, 0u, 0u), x1 = x0;
                if (xv[tg]) {
                    x0 = ld_ro_v4(xrow[tg] + o);
                    x1 = ld_ro_v4(xrow[tg] + o + 8);
                }
                const uint32_t xw[8] = {x0.x, x0.y, x0.z, x0.w, x1.x, x1.y, x1.z, x1.w};
                float d[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    mma_16816(d, af[kk][0], af[kk][1], af[kk][2], af[kk][3], xw[2 * kk], xw[2 * kk + 1]);
                acc[tg][0] = __fmaf_rn(cpA, d[0], acc[tg][0]);
                acc[tg][1] = __fmaf_rn(cpA, d[1], acc[tg][1]);
                acc[tg][2] = __fmaf_rn(cpB, d[2], acc[tg][2]);
                acc[tg][3] = __fmaf_rn(cpB, d[3], acc[tg][3]);
            }
        }
        cur = nxt;
    }
    {
        const int rl = warp * 16 + g;
#pragma unroll
        for (int tg = 0; tg < NG; ++tg) {
            part[rl * MP + tg * 8 + 2 * t] = acc[tg][0];
            part[rl * MP + tg * 8 + 2 * t + 1] = acc[tg][1];
            part[(rl + 8) * MP + tg * 8 + 2 * t] = acc[tg][2];
            part[(rl + 8) * MP + tg * 8 + 2 * t + 1] = acc[tg][3];
        }
    }

    __syncthreads();
    cluster.sync();  // every CTA's partials are complete and visible in the cluster
    grid_dependents_launch();

    if (p.r > 0) {
        for (int i = threadIdx.x; i < rpad * MP; i += blockDim.x) {
            float sum = 0.0f;
            for (int cc = 0; cc < C; ++cc) sum += cluster.map_shared_rank(tpart, cc)[i];
            tfull[i] = round_bf16(sum * p.s);
        }
    }
    __syncthreads();

    // ---- this CTA finalises rows [kFwdRows*crank/C, kFwdRows*(crank+1)/C) of the row group
    const int r_lo = kFwdRows * crank / C, r_hi = kFwdRows * (crank + 1) / C, nr = r_hi - r_lo;
    for (int i = threadIdx.x; i < nr * M; i += blockDim.x) {
        const int rl = r_lo + i % nr, tok = i / nr;
        const int64_t n = static_cast<int64_t>(blockIdx.y) * kFwdRows + rl;
        if (n >= N) continue;
        float sum = 0.0f;
        for (int cc = 0; cc < C; ++cc) sum += cluster.map_shared_rank(part, cc)[rl * MP + tok];
        if (p.r > 0) {
            const uint16_t *brow = p.B + n * p.r;
            float lora = 0.0f;
            for (int j = 0; j < p.r; ++j)
                lora = __fmaf_rn(__uint_as_float(static_cast<uint32_t>(ld_ro_u16(brow + j)) << 16), tfull[j * MP + tok], lora);
            sum += lora;
        }
        p.out[static_cast<int64_t>(tok) * N + n] = __bfloat16_as_ushort(__float2bfloat16_rn(sum));
    }
    cluster.sync();  // keep this CTA's shared memory alive until the cluster is done reading it
}

// ------------------------------------------------------------------- input gradient
// Interleave the nibbles of two 8-code words of neighbouring rows: byte i of `even`
// holds (row a, k = 2i) | (row b, k = 2i) << 4, byte i of `odd` the same for k = 2i+1.
__device__ __forceinline__ void interleave_rows(uint32_t ra, uint32_t rb, uint32_t &even, uint32_t &odd) {
    even = (ra & 0x0f0f0f0fu) | ((rb & 0x0f0f0f0fu) << 4);
    odd = ((ra >> 4) & 0x0f0f0f0fu) | (rb & 0xf0f0f0f0u);
}

// 4 bf16 of row `tok` of grad_h at columns n0 .. n0+3 (zero beyond N).
__device__ __forceinline__ void load_g4(const uint16_t *gh, int64_t N, int tok, int64_t n0, float (&v)[4]) {
    const uint16_t *p = gh + static_cast<int64_t>(tok) * N + n0;
    if ((N & 3) == 0 && n0 + 3 < N) {
        const uint2 w = ld_ro_v2(p);
        v[0] = bf16_lo(w.x);
        v[1] = bf16_hi(w.x);
        v[2] = bf16_lo(w.y);
        v[3] = bf16_hi(w.y);
    } else {
#pragma unroll
        for (int i = 0; i < 4; ++i)
            v[i] = (n0 + i < N) ? __uint_as_float(static_cast<uint32_t>(ld_ro_u16(p + i)) << 16) : 0.0f;
    }
}

// Registers of one group of two 16-row steps: 4 rows (4t .. 4t+3) x 8 features per step,
// plus the constant inputs of row (4t + gq % 4) of each step.
struct BwdGroup {
    uint32_t w[2][4];
    uint32_t q[2];
    float s[2];
};

template <int NG>
__global__ void __launch_bounds__(kDecThreads)
k_decode_bwd(const DecodeParams p) {
    constexpr int MP = 8 * NG;
    extern __shared__ __align__(16) uint8_t smem[];
    uint8_t *lut = smem;
    float *part = reinterpret_cast<float *>(smem + kLutBytes);  // [warps][64 features][MP]
    const int rpad = (p.r + 15) & ~15;
    float *upart = part + kDecWarps * 64 * MP;  // [rpad][MP] partial B^T grad_h of this CTA
    float *ufull = upart + rpad * MP;           // [rpad][MP] s * B^T grad_h, rounded to bf16

    cg::cluster_group cluster = cg::this_cluster();
    const int C = static_cast<int>(cluster.num_blocks());
    const int crank = static_cast<int>(cluster.block_rank());
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int gq = lane >> 2, t = lane & 3;
    const uint32_t lane4 = static_cast<uint32_t>(lane) << 2;

    const int64_t N = p.n, K = p.k;
    const int64_t nbr = K / kBlock;
    const int col = warp % kBwdCols, sub = warp / kBwdCols;
    const int64_t kb = static_cast<int64_t>(blockIdx.y) * kBwdCols + col;  // output block column
    const bool vk = kb < nbr;
    const int64_t kbc = vk ? kb : 0;
    // reduction rows in 16-row steps: cluster slice, then this warp's sub-slice
    const int64_t n16 = (N + 15) / 16;
    const int64_t c_lo = n16 * crank / C, c_hi = n16 * (crank + 1) / C;
    const int64_t s_lo = c_lo + (c_hi - c_lo) * sub / kBwdSub, s_hi = c_lo + (c_hi - c_lo) * (sub + 1) / kBwdSub;

    build_pair_lut(lut);
    for (int i = threadIdx.x; i < rpad * MP; i += blockDim.x) upart[i] = 0.0f;
    // L2 prefetch of everything this CTA reads: the warp's codes (rows [16 s_lo, 16 s_hi) x
    // 32 bytes of column kb) and their constants, the grad_h slice, the adapter rows.
    if (vk) {
        for (int64_t rr = s_lo * 16 + lane; rr < s_hi * 16 && rr < N; rr += 32) {
            prefetch_l2(p.codes + rr * (K / 2) + kbc * 32, 32u);
            prefetch_line(p.q + rr * nbr + kbc);
            prefetch_line(p.sigma + (rr * nbr + kbc) / kGroup);
        }
    }
    if (warp == 0 && lane < p.M) {
        const int64_t n_lo = c_lo * 16, n_hi = c_hi * 16 < N ? c_hi * 16 : N;
        prefetch_range(p.act + lane * N + n_lo, (n_hi - n_lo) * 2);
    }
    if (warp == 1 && p.r > 0) {
        const int64_t n_lo = c_lo * 16, n_hi = c_hi * 16 < N ? c_hi * 16 : N;
        if (lane == 0) prefetch_range(p.B + n_lo * p.r, (n_hi - n_lo) * p.r * 2);
        const int64_t k0 = static_cast<int64_t>(blockIdx.y) * 64 * kBwdCols;
        const int64_t k1 = k0 + 64 * kBwdCols < K ? k0 + 64 * kBwdCols : K;
        for (int j = lane; j < p.r; j += 32) prefetch_range(p.A + j * K + k0, (k1 - k0) * 2);
    }
    __syncthreads();
    grid_dependency_wait();

    const float mu = __ldg(p.mu);
    const int M = p.M;

    auto load_group = [&](int64_t st0, BwdGroup &G) {
#pragma unroll
        for (int j = 0; j < 2; ++j) {
            const int64_t st = st0 + j;
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int64_t n = st * 16 + 4 * t + i;
                G.w[j][i] = (st < s_hi && n < N) ? ld_nc_u32(p.codes + n * (K / 2) + kbc * 32 + 4 * gq) : 0x77777777u;
            }
            const int64_t n = st * 16 + 4 * t + (gq & 3);
            const bool ok = st < s_hi && n < N;
            const int64_t bi = n * nbr + kbc;
            G.q[j] = ok ? __ldg(p.q + bi) : 0u;
            G.s[j] = ok ? __ldg(p.sigma + bi / kGroup) : 0.0f;
        }
    };

    float acc[4][NG][4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int tg = 0; tg < NG; ++tg) acc[i][tg][0] = acc[i][tg][1] = acc[i][tg][2] = acc[i][tg][3] = 0.0f;

    BwdGroup cur, nxt;
    if (vk && s_lo < s_hi) load_group(s_lo, cur);

    // ---- LoRA: partial u[j][tok] = sum_n B[n][j] grad_h[tok][n] over this CTA's slice.
    if (p.r > 0) {
        const int rt = rpad / 16;
        const int64_t ns = c_hi - c_lo;
        const int64_t q_lo = c_lo + ns * warp / kDecWarps, q_hi = c_lo + ns * (warp + 1) / kDecWarps;
        for (int jt = 0; jt < rt; ++jt) {
            const int jA = jt * 16 + gq, jB = jA + 8;
            float d[NG][4];
#pragma unroll
            for (int tg = 0; tg < NG; ++tg) d[tg][0] = d[tg][1] = d[tg][2] = d[tg][3] = 0.0f;
            for (int64_t st = q_lo; st < q_hi; ++st) {
                const int64_t n0 = st * 16;
                auto bval = [&](int64_t n, int j) -> uint32_t {
                    return (n < N && j < p.r) ? static_cast<uint32_t>(ld_ro_u16(p.B + n * p.r + j)) : 0u;
                };
                const uint32_t a0 = bval(n0 + 2 * t, jA) | (bval(n0 + 2 * t + 1, jA) << 16);
                const uint32_t a1 = bval(n0 + 2 * t, jB) | (bval(n0 + 2 * t + 1, jB) << 16);
                const uint32_t a2 = bval(n0 + 2 * t + 8, jA) | (bval(n0 + 2 * t + 9, jA) << 16);
                const uint32_t a3 = bval(n0 + 2 * t + 8, jB) | (bval(n0 + 2 * t + 9, jB) << 16);
#pragma unroll
                for (int tg = 0; tg < NG; ++tg) {
                    const int tok = tg * 8 + gq;
                    uint32_t b0 = 0u, b1 = 0u;
                    if (tok < M) {
                        const uint16_t *gr = p.act + static_cast<int64_t>(tok) * N + n0;
                        auto gval = [&](int64_t i) -> uint32_t {
                            return (n0 + i < N) ? static_cast<uint32_t>(ld_ro_u16(gr + i)) : 0u;
                        };
                        b0 = gval(2 * t) | (gval(2 * t + 1) << 16);
                        b1 = gval(2 * t + 8) | (gval(2 * t + 9) << 16);
                    }
                    mma_16816(d[tg], a0, a1, a2, a3, b0, b1);
                }
            }
#pragma unroll
            for (int tg = 0; tg < NG; ++tg) {
                const int jl = jt * 16 + gq;
                atomicAdd(&upart[jl * MP + tg * 8 + 2 * t], d[tg][0]);
                atomicAdd(&upart[jl * MP + tg * 8 + 2 * t + 1], d[tg][1]);
                atomicAdd(&upart[(jl + 8) * MP + tg * 8 + 2 * t], d[tg][2]);
                atomicAdd(&upart[(jl + 8) * MP + tg * 8 + 2 * t + 1], d[tg][3]);
            }
        }
    }

    // ---- base: block column kb, reduction over steps [s_lo, s_hi), groups of two steps
    if (vk) {
        for (int64_t st0 = s_lo; st0 < s_hi; st0 += 2) {
            if (st0 + 2 < s_hi) load_group(st0 + 2, nxt);
#pragma unroll
            for (int j = 0; j < 2; ++j) {
                const int64_t st = st0 + j;
                if (st >= s_hi) break;
                const int64_t n0 = st * 16 + 4 * t;  // this lane's 4 reduction rows
                // constant of row n0 + (gq & 3), shared with the lanes of the same t
                const float mine = block_constant(static_cast<uint8_t>(cur.q[j]), cur.s[j], mu);
                float cp[4];
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    cp[i] = __shfl_sync(0xffffffffu, mine, (i << 2) | t);
                    if (n0 + i >= N) cp[i] = 0.0f;
                }
                uint32_t e01, o01, e23, o23;
                interleave_rows(cur.w[j][0], cur.w[j][1], e01, o01);
                interleave_rows(cur.w[j][2], cur.w[j][3], e23, o23);
                uint32_t af[4][4];
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    af[i][0] = lut_pair(lut, e01, lane4, i);
                    af[i][1] = lut_pair(lut, o01, lane4, i);
                    af[i][2] = lut_pair(lut, e23, lane4, i);
                    af[i][3] = lut_pair(lut, o23, lane4, i);
                }
#pragma unroll
                for (int tg = 0; tg < NG; ++tg) {
                    const int tok = tg * 8 + gq;
                    float gv[4] = {0.0f, 0.0f, 0.0f, 0.0f};
                    if (tok < M) load_g4(p.act, N, tok, n0, gv);
                    const uint32_t b0 = pack_bf16x2(cp[0] * gv[0], cp[1] * gv[1]);
                    const uint32_t b1 = pack_bf16x2(cp[2] * gv[2], cp[3] * gv[3]);
#pragma unroll
                    for (int i = 0; i < 4; ++i)
                        mma_16816(acc[i][tg], af[i][0], af[i][1], af[i][2], af[i][3], b0, b1);
                }
            }
            cur = nxt;
        }
    }
    // D row gq of tile i is feature 8*gq + 2i, row gq+8 is feature 8*gq + 2i + 1.
    {
        float *wp = part + warp * 64 * MP;
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int tg = 0; tg < NG; ++tg) {
                const int f = 8 * gq + 2 * i, tok = tg * 8 + 2 * t;
                wp[f * MP + tok] = acc[i][tg][0];
                wp[f * MP + tok + 1] = acc[i][tg][1];
                wp[(f + 1) * MP + tok] = acc[i][tg][2];
                wp[(f + 1) * MP + tok + 1] = acc[i][tg][3];
            }
    }

    __syncthreads();
    cluster.sync();
    grid_dependents_launch();

    if (p.r > 0) {
        for (int i = threadIdx.x; i < rpad * MP; i += blockDim.x) {
            float sum = 0.0f;
            for (int cc = 0; cc < C; ++cc) sum += cluster.map_shared_rank(upart, cc)[i];
            ufull[i] = round_bf16(sum * p.s);
        }
    }
    __syncthreads();

    // ---- this CTA finalises features [F*crank/C, F*(crank+1)/C) of the CTA group's F features
    constexpr int F = 64 * kBwdCols;
    const int f_lo = F * crank / C, f_hi = F * (crank + 1) / C, nf = f_hi - f_lo;
    for (int i = threadIdx.x; i < nf * M; i += blockDim.x) {
        const int fl = f_lo + i % nf, tok = i / nf;
        const int64_t k = static_cast<int64_t>(blockIdx.y) * F + fl;
        if (k >= K) continue;
        const int c = fl / 64, f = fl % 64;
        float sum = 0.0f;
        for (int cc = 0; cc < C; ++cc) {
            const float *rp = cluster.map_shared_rank(part, cc);
#pragma unroll
            for (int sb = 0; sb < kBwdSub; ++sb) sum += rp[((sb * kBwdCols + c) * 64 + f) * MP + tok];
        }
        if (p.r > 0) {
            float lora = 0.0f;
            for (int j = 0; j < p.r; ++j)
                lora = __fmaf_rn(__uint_as_float(static_cast<uint32_t>(ld_ro_u16(p.A + static_cast<int64_t>(j) * K + k)) << 16),
                                 ufull[j * MP + tok], lora);
            sum += lora;
        }
        p.out[static_cast<int64_t>(tok) * K + k] = __bfloat16_as_ushort(__float2bfloat16_rn(sum));
    }
    cluster.sync();
}

template <typename Kern>
cudaError_t launch_cluster(Kern kern, dim3 grid, int cluster_x, size_t smem, cudaStream_t st, const DecodeParams &p) {
    // Raise the kernel's dynamic shared-memory limit only when a launch needs more than
    // any earlier one (the attribute call is skipped on the steady-state path).
    static thread_local const void *kerns[16];
    static thread_local size_t limits[16];
    static thread_local int nk = 0;
    int slot = -1;
    for (int i = 0; i < nk; ++i)
        if (kerns[i] == reinterpret_cast<const void *>(kern)) slot = i;
    if (slot < 0 || limits[slot] < smem) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
        if (e != cudaSuccess) return e;
        if (slot < 0 && nk < 16) {
            slot = nk++;
            kerns[slot] = reinterpret_cast<const void *>(kern);
        }
        if (slot >= 0) limits[slot] = smem;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = dim3(kDecThreads, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = cluster_x;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    // Programmatic dependent launch: the grid may start while the preceding kernel
    // finishes; the kernel reads no global memory before griddepcontrol.wait (only an L2
    // prefetch of the frozen weight codes is issued earlier).
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    cudaError_t e = cudaLaunchKernelEx(&cfg, kern, p);
    count_launch();
    return e;
}

int pick_groups(int M) { return M <= 8 ? 1 : M <= 16 ? 2 : M <= 32 ? 4 : 8; }

// Cluster size: the power of two (<= 8) that brings the CTA count closest to two per SM,
// keeping at least `min_units` units of reduction work per CTA.
int pick_cluster(int64_t tiles, int64_t red_units, int64_t min_units, int sms) {
    int best = 1;
    double best_score = 1e30;
    for (int C = 1; C <= kMaxCluster; C *= 2) {
        if (C > 1 && red_units / C < min_units) break;
        const double ratio = static_cast<double>(tiles * C) / (2.0 * sms);
        const double score = ratio > 1.0 ? ratio : 1.0 / ratio;
        if (score < best_score) {
            best_score = score;
            best = C;
        }
    }
    return best;
}

int num_sms() {
    static int sms = 0;
    if (sms == 0) {
        int dev = 0;
        cudaGetDevice(&dev);
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
        if (sms <= 0) sms = 148;
    }
    return sms;
}

}  // namespace

cudaError_t launch_decode_fwd(const WeightView &w, const uint16_t *x, int M, const uint16_t *A, const uint16_t *B,
                              int r, float s, uint16_t *h, cudaStream_t st) {
    if (M <= 0 || w.n == 0) return cudaSuccess;
    DecodeParams p{w.codes, w.q, w.sigma, w.mu, w.n, w.k, x, M, A, B, r, s, h};
    const int NG = pick_groups(M);
    const int rpad = (r + 15) & ~15;
    const size_t smem = kLutBytes + sizeof(float) * (kFwdRows * 8 * NG + 2 * rpad * 8 * NG);
    const int64_t tiles = (w.n + kFwdRows - 1) / kFwdRows;
    const int C = pick_cluster(tiles, w.k / kBlock, 4, num_sms());
    const dim3 grid(C, static_cast<unsigned>(tiles), 1);
    switch (NG) {
        case 1: return launch_cluster(k_decode_fwd<1>, grid, C, smem, st, p);
        case 2: return launch_cluster(k_decode_fwd<2>, grid, C, smem, st, p);
        case 4: return launch_cluster(k_decode_fwd<4>, grid, C, smem, st, p);
        default: return launch_cluster(k_decode_fwd<8>, grid, C, smem, st, p);
    }
}

cudaError_t launch_decode_bwd(const WeightView &w, const uint16_t *gh, int M, const uint16_t *A, const uint16_t *B,
                              int r, float s, uint16_t *gx, cudaStream_t st) {
    if (M <= 0 || w.k == 0) return cudaSuccess;
    DecodeParams p{w.codes, w.q, w.sigma, w.mu, w.n, w.k, gh, M, A, B, r, s, gx};
    const int NG = pick_groups(M);
    const int rpad = (r + 15) & ~15;
    const size_t smem = kLutBytes + sizeof(float) * (kDecWarps * 64 * 8 * NG + 2 * rpad * 8 * NG);
    const int64_t tiles = (w.k / kBlock + kBwdCols - 1) / kBwdCols;
    const int C = pick_cluster(tiles, (w.n + 15) / 16 / kBwdSub, 2, num_sms());
    const dim3 grid(C, static_cast<unsigned>(tiles), 1);
    switch (NG) {
        case 1: return launch_cluster(k_decode_bwd<1>, grid, C, smem, st, p);
        case 2: return launch_cluster(k_decode_bwd<2>, grid, C, smem, st, p);
        case 4: return launch_cluster(k_decode_bwd<4>, grid, C, smem, st, p);
        default: return cudaErrorInvalidValue;  // callers split tokens into chunks of 32
    }
}

}  // namespace qn
