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
// words, one copy per lane. One row per thread; the eight 16-byte stores of a row start at a
// column rotated by the row so that the lanes of a warp hit different banks.
__device__ __forceinline__ void build_pair_lut(uint8_t *lut) {
    uint4 *l4 = reinterpret_cast<uint4 *>(lut);
    for (int e = threadIdx.x; e < 256; e += blockDim.x) {
        const uint32_t v = pack_bf16x2(nf4_value(e & 15), nf4_value(e >> 4));
#pragma unroll
        for (int c = 0; c < 8; ++c) l4[e * 16 + ((c + e) & 7)] = make_uint4(v, v, v, v);
    }
}

// Low 24 bits of the shared-window address of dynamic shared memory when the driver reserves
// 1 KB per block and the kernel has no static shared memory; in a cluster launch the CTA's
// rank sits above them. The kernels check it at run time and otherwise take the generic path.
constexpr uint32_t kDynSmemBase = 1024;

__device__ __forceinline__ uint32_t smem_addr(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// Operand of the table permute: lane << 2 in byte 0 and, on the fixed-base path, the high
// byte (cluster rank) of the table's shared-window address in byte 3.
template <bool kFixedBase>
__device__ __forceinline__ uint32_t lut_lane_operand(const uint8_t *lut, int lane) {
    const uint32_t l4 = static_cast<uint32_t>(lane) << 2;
    return kFixedBase ? (l4 | (smem_addr(lut) & 0xff000000u)) : l4;
}

// Pair for byte i (0..3) of word w. The permute builds (byte << 8) | (lane << 2), plus the rank
// byte on the fixed-base path, where the table starts at the base of dynamic shared memory and
// its low address bits are an immediate of the load; otherwise the table address is added.
template <bool kFixedBase>
__device__ __forceinline__ uint32_t lut_pair(const uint8_t *lut, uint32_t w, uint32_t lane_op, int i) {
    if constexpr (kFixedBase) {
        const uint32_t a = prmt(w, lane_op, 0x7604u | (static_cast<uint32_t>(i) << 4));
        uint32_t v;
        asm volatile("ld.shared.b32 %0, [%1+%2];" : "=r"(v) : "r"(a), "n"(kDynSmemBase));
        return v;
    } else {
        const uint32_t off = prmt(w, lane_op, 0x5504u | (static_cast<uint32_t>(i) << 4));
        return *reinterpret_cast<const uint32_t *>(lut + off);
    }
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

// L2 prefetch (before the dependency wait) of the activation slice and the adapter slice of
// this CTA's k-range, so that their first reads after the wait are L2 hits.
__device__ __forceinline__ void prefetch_operands(const DecodeParams &p, int b_lo, int b_hi) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t K = p.k;
    const int64_t kbytes = static_cast<int64_t>(b_hi - b_lo) * 128;  // 64 bf16 per block
    if (kbytes <= 0) return;
    if (warp == 0 && lane < p.M)
        prefetch_l2(p.act + lane * K + static_cast<int64_t>(b_lo) * 64, static_cast<uint32_t>(kbytes));
    if (warp == 1)
        for (int j = lane; j < p.r; j += 32) prefetch_l2(p.A + j * K + static_cast<int64_t>(b_lo) * 64, static_cast<uint32_t>(kbytes));
}

__device__ __forceinline__ void cluster_arrive_relaxed() {
    asm volatile("barrier.cluster.arrive.relaxed.aligned;" ::: "memory");
}
__device__ __forceinline__ void cluster_wait() { asm volatile("barrier.cluster.wait.aligned;" ::: "memory"); }

// bf16 pair (B[row][j], B[row][j + 1]) of the row-major n x r adapter B, zero outside it.
__device__ __forceinline__ uint32_t load_b_pair(const DecodeParams &p, int64_t row, bool valid, int j) {
    if (!valid || j >= p.r) return 0u;
    const uint16_t *b = p.B + row * p.r + j;
    if ((p.r & 1) == 0) return ld_ro_u32(b);  // j even: 4-byte aligned
    const uint32_t lo = ld_ro_u16(b);
    const uint32_t hi = j + 1 < p.r ? ld_ro_u16(b + 1) : 0u;
    return lo | (hi << 16);
}

// MMA A-fragment of B rows (rowA, rowB) and adapter columns [j, j + 2) and [j + 8, j + 10).
__device__ __forceinline__ void load_b_frag(const DecodeParams &p, int64_t rowA, int64_t rowB, bool vA, bool vB, int j,
                                            uint32_t &a0, uint32_t &a1, uint32_t &a2, uint32_t &a3) {
    a0 = load_b_pair(p, rowA, vA, j);
    a1 = load_b_pair(p, rowB, vB, j);
    a2 = load_b_pair(p, rowA, vA, j + 8);
    a3 = load_b_pair(p, rowB, vB, j + 8);
}

// Copy columns [k0, k0 + nc) of the first `rows` rows of a row-major bf16 matrix with row
// stride `ld` to dst[row][c] (row stride nc), eight loads in flight per thread.
__device__ __forceinline__ void stage_cols(uint16_t *dst, const uint16_t *src, int64_t ld, int64_t k0, int rows,
                                           int nc) {
    constexpr int U = 8;
    const int n = rows * nc;
    for (int base = threadIdx.x; base < n; base += U * blockDim.x) {
        uint16_t v[U];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int i = base + u * blockDim.x;
            if (i < n) v[u] = ld_ro_u16(src + static_cast<int64_t>(i / nc) * ld + k0 + i % nc);
        }
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int i = base + u * blockDim.x;
            if (i < n) dst[i] = v[u];
        }
    }
}

// ------------------------------------------------------------------------- forward
// Registers of one group of four 64-weight blocks for rows A (g) and B (g + 8) of a lane.
struct FwdGroup {
    uint2 ca[4], cb[4];
    uint32_t qa, qb;  // this lane's block (t) of the group
    float sa, sb;
};

template <int NG, bool kFixedBase>
__device__ __forceinline__ void decode_fwd_body(const DecodeParams &p, uint8_t *smem) {
    constexpr int MP = 8 * NG;  // padded token count
    uint8_t *lut = smem;
    // recv[src][row - r_lo][MP]: the partial sums that cluster rank `src` pushes for the rows
    // this CTA finalises (at most kFwdRows + kMaxCluster rows in all).
    float *recv = reinterpret_cast<float *>(smem + kLutBytes);
    const int rpad = (p.r + 15) & ~15;
    float *tpart = recv + (kFwdRows + kMaxCluster) * MP;  // [rpad][MP] partial A x of this CTA's k-slice

    cg::cluster_group cluster = cg::this_cluster();
    const int C = static_cast<int>(cluster.num_blocks());
    const int crank = static_cast<int>(cluster.block_rank());
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, t = lane & 3;
    const uint32_t lane4 = lut_lane_operand<kFixedBase>(lut, lane);

    const int64_t N = p.n, K = p.k;
    const int nbr = static_cast<int>(K / kBlock);
    // nbr < 2^25 (k_in < 2^31), so the products fit 32 bits
    const int b_lo = static_cast<int>(static_cast<uint32_t>(nbr * crank) / static_cast<uint32_t>(C));
    const int b_hi = static_cast<int>(static_cast<uint32_t>(nbr * (crank + 1)) / static_cast<uint32_t>(C));
    const int64_t row_base = static_cast<int64_t>(blockIdx.y) * kFwdRows + warp * 16;

    // Before the dependency wait only an L2 prefetch of the operand slices. The weight codes are
    // not prefetched (per-row prefetches cost more to issue than they saved): the first two
    // groups of codes are requested right after the wait, and the pair table is built while
    // they are in flight.
    prefetch_operands(p, b_lo, b_hi);
    cluster_arrive_relaxed();  // phase 1: this CTA is running (its shared memory may be written)
    grid_dependency_wait();

    const float mu = __ldg(p.mu);
    const int M = p.M;
    const int64_t rowA = row_base + g, rowB = rowA + 8;
    const bool vA = rowA < N, vB = rowB < N;
    uint32_t bf[4] = {0u, 0u, 0u, 0u};  // B fragment of the first 16 adapter columns, loaded early
    if (p.r > 0) load_b_frag(p, rowA, rowB, vA, vB, 2 * t, bf[0], bf[1], bf[2], bf[3]);
    // Rows past N read row 0 (valid memory) and get a zero block constant; tokens past M read
    // token 0 and fill MMA columns that are never stored. The hot loop therefore only needs
    // the block count of the last (partial) group.
    const int nblk = b_hi - b_lo, ngrp = (nblk + 3) / 4;
    const uint2 *pa = reinterpret_cast<const uint2 *>(p.codes + (vA ? rowA : 0) * (K / 2) +
                                                      static_cast<int64_t>(b_lo) * 32 + 8 * t);
    const uint2 *pb = reinterpret_cast<const uint2 *>(p.codes + (vB ? rowB : 0) * (K / 2) +
                                                      static_cast<int64_t>(b_lo) * 32 + 8 * t);
    // flattened index of lane t's block in group 0 (the lane loads that block's constants)
    const int64_t eA = (vA ? rowA : 0) * nbr + b_lo + t, eB = (vB ? rowB : 0) * nbr + b_lo + t;

    auto load_group = [&](int gi, FwdGroup &G) {
        const int cnt = nblk - 4 * gi;  // blocks in this group (at least 1)
        const uint2 *ga = pa + 16 * gi, *gb = pb + 16 * gi;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            G.ca[j] = j < cnt ? __ldcs(ga + 4 * j) : make_uint2(0u, 0u);
            G.cb[j] = j < cnt ? __ldcs(gb + 4 * j) : make_uint2(0u, 0u);
        }
        const bool ok = t < cnt;
        const uint64_t ea = static_cast<uint64_t>(eA + 4 * gi), eb = static_cast<uint64_t>(eB + 4 * gi);
        G.qa = ok ? __ldg(p.q + ea) : 0u;
        G.qb = ok ? __ldg(p.q + eb) : 0u;
        G.sa = ok ? __ldg(p.sigma + ea / kGroup) : 0.0f;
        G.sb = ok ? __ldg(p.sigma + eb / kGroup) : 0.0f;
    };

    // x of this lane's tokens: x[tg*8 + g][64 b + 16 t .. + 16] is xq[tg][8 (b - b_lo)], [.. + 1]
    const uint4 *xq[NG];
#pragma unroll
    for (int tg = 0; tg < NG; ++tg) {
        const int tok = tg * 8 + g;
        xq[tg] = reinterpret_cast<const uint4 *>(p.act + static_cast<int64_t>(tok < M ? tok : 0) * K +
                                                 static_cast<int64_t>(b_lo) * 64 + 16 * t);
    }

    float acc[NG][4];
#pragma unroll
    for (int tg = 0; tg < NG; ++tg) acc[tg][0] = acc[tg][1] = acc[tg][2] = acc[tg][3] = 0.0f;

    FwdGroup G0, G1;  // ping-pong: two groups of codes in flight while one is consumed
    if (ngrp > 0) load_group(0, G0);
    if (ngrp > 1) load_group(1, G1);

    // ---- LoRA down-projection over this CTA's k-slice (partial t = A x, fp32), run after the
    // first group of codes has been consumed (its operands are L2 hits that would otherwise
    // queue behind the code loads). Item (j-tile, eighth of the slice) per warp.
    auto lora_down = [&]() {
        const int rt = rpad / 16;
        const int s_lo = nblk * warp / kDecWarps, s_hi = nblk * (warp + 1) / kDecWarps;  // relative to b_lo
        for (int jt = 0; jt < rt; ++jt) {
            const int jA = jt * 16 + g, jB = jA + 8;
            const bool aA = jA < p.r, aB = jB < p.r;
            const uint4 *ra = reinterpret_cast<const uint4 *>(p.A + static_cast<int64_t>(aA ? jA : 0) * K +
                                                             static_cast<int64_t>(b_lo) * 64 + 16 * t);
            const uint4 *rb = reinterpret_cast<const uint4 *>(p.A + static_cast<int64_t>(aB ? jB : 0) * K +
                                                             static_cast<int64_t>(b_lo) * 64 + 16 * t);
            float d[NG][4];
#pragma unroll
            for (int tg = 0; tg < NG; ++tg) d[tg][0] = d[tg][1] = d[tg][2] = d[tg][3] = 0.0f;
            for (int b = s_lo; b < s_hi; ++b) {
                uint4 a0 = make_uint4(0u, 0u, 0u, 0u), a1 = a0, b0 = a0, b1 = a0;
                if (aA) {
                    a0 = __ldg(ra + 8 * b);
                    a1 = __ldg(ra + 8 * b + 1);
                }
                if (aB) {
                    b0 = __ldg(rb + 8 * b);
                    b1 = __ldg(rb + 8 * b + 1);
                }
#pragma unroll
                for (int tg = 0; tg < NG; ++tg) {
                    const uint4 x0 = __ldg(xq[tg] + 8 * b), x1 = __ldg(xq[tg] + 8 * b + 1);
                    mma_16816(d[tg], a0.x, b0.x, a0.y, b0.y, x0.x, x0.y);
                    mma_16816(d[tg], a0.z, b0.z, a0.w, b0.w, x0.z, x0.w);
                    mma_16816(d[tg], a1.x, b1.x, a1.y, b1.y, x1.x, x1.y);
                    mma_16816(d[tg], a1.z, b1.z, a1.w, b1.w, x1.z, x1.w);
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
    };

    // The pair table is built while the first codes are in flight.
    build_pair_lut(lut);
    for (int i = threadIdx.x; i < rpad * MP; i += blockDim.x) tpart[i] = 0.0f;
    __syncthreads();

    // ---- base: group gi holds blocks b_lo + 4 gi .. + 4 of rows A and B.
    auto compute_group = [&](const FwdGroup &G, int gi) {
        const int cnt = nblk - 4 * gi;
        const bool ok = t < cnt;
        const float cA4 = (vA && ok) ? block_constant(static_cast<uint8_t>(G.qa), G.sa, mu) : 0.0f;
        const float cB4 = (vB && ok) ? block_constant(static_cast<uint8_t>(G.qb), G.sb, mu) : 0.0f;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            if (j >= cnt) break;
            const float cpA = __shfl_sync(0xffffffffu, cA4, (lane & ~3) | j);
            const float cpB = __shfl_sync(0xffffffffu, cB4, (lane & ~3) | j);
            uint32_t af[4][4];
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
                const uint32_t wa = kk < 2 ? G.ca[j].x : G.ca[j].y, wb = kk < 2 ? G.cb[j].x : G.cb[j].y;
                const int i0 = (2 * kk) & 3;
                af[kk][0] = lut_pair<kFixedBase>(lut, wa, lane4, i0);
                af[kk][2] = lut_pair<kFixedBase>(lut, wa, lane4, i0 + 1);
                af[kk][1] = lut_pair<kFixedBase>(lut, wb, lane4, i0);
                af[kk][3] = lut_pair<kFixedBase>(lut, wb, lane4, i0 + 1);
            }
            const int xo = 8 * (4 * gi + j);
#pragma unroll
            for (int tg = 0; tg < NG; ++tg) {
                const uint4 x0 = __ldg(xq[tg] + xo), x1 = __ldg(xq[tg] + xo + 1);
                float d[4] = {0.0f, 0.0f, 0.0f, 0.0f};
                mma_16816(d, af[0][0], af[0][1], af[0][2], af[0][3], x0.x, x0.y);
                mma_16816(d, af[1][0], af[1][1], af[1][2], af[1][3], x0.z, x0.w);
                mma_16816(d, af[2][0], af[2][1], af[2][2], af[2][3], x1.x, x1.y);
                mma_16816(d, af[3][0], af[3][1], af[3][2], af[3][3], x1.z, x1.w);
                acc[tg][0] = __fmaf_rn(cpA, d[0], acc[tg][0]);
                acc[tg][1] = __fmaf_rn(cpA, d[1], acc[tg][1]);
                acc[tg][2] = __fmaf_rn(cpB, d[2], acc[tg][2]);
                acc[tg][3] = __fmaf_rn(cpB, d[3], acc[tg][3]);
            }
        }
    };
    for (int gi = 0; gi < ngrp; gi += 2) {
        compute_group(G0, gi);
        if (gi == 0 && p.r > 0) lora_down();
        if (gi + 2 < ngrp) load_group(gi + 2, G0);
        if (gi + 1 < ngrp) {
            compute_group(G1, gi + 1);
            if (gi + 3 < ngrp) load_group(gi + 3, G1);
        }
    }
    if (ngrp == 0 && p.r > 0) lora_down();
    __syncthreads();  // tpart holds A x over this CTA's k-slice

    // ---- adapter up-projection of this CTA's k-slice, folded into the partial sums:
    // acc += B[rows, :] (s * t_c), with t_c = A x over the slice rounded to bf16 as the MMA operand.
    for (int jt = 0; jt < rpad / 16; ++jt) {
        uint32_t a0 = bf[0], a1 = bf[1], a2 = bf[2], a3 = bf[3];
        if (jt > 0) load_b_frag(p, rowA, rowB, vA, vB, jt * 16 + 2 * t, a0, a1, a2, a3);
        const int j0 = jt * 16 + 2 * t;
#pragma unroll
        for (int tg = 0; tg < NG; ++tg) {
            const int tok = tg * 8 + g;
            const uint32_t b0 = pack_bf16x2(p.s * tpart[j0 * MP + tok], p.s * tpart[(j0 + 1) * MP + tok]);
            const uint32_t b1 = pack_bf16x2(p.s * tpart[(j0 + 8) * MP + tok], p.s * tpart[(j0 + 9) * MP + tok]);
            mma_16816(acc[tg], a0, a1, a2, a3, b0, b1);
        }
    }

    // ---- push the partials of rows g and g + 8 of this warp to the CTAs that finalise them.
    const int nrmax = (kFwdRows + C - 1) / C;
    cluster_wait();  // phase 1: every CTA of the cluster is running
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        const int rl = warp * 16 + g + 8 * h;
        const int owner = (rl * C + C - 1) / kFwdRows;  // largest c with kFwdRows*c/C <= rl
        const int rr = rl - kFwdRows * owner / C;
        float *dst = cluster.map_shared_rank(recv, owner) + (crank * nrmax + rr) * MP + 2 * t;
#pragma unroll
        for (int tg = 0; tg < NG; ++tg)
            *reinterpret_cast<float2 *>(dst + tg * 8) = make_float2(acc[tg][2 * h], acc[tg][2 * h + 1]);
    }
    cluster_arrive_release();
    cluster_wait_acquire();  // phase 2: every partial has landed
    grid_dependents_launch();

    // ---- this CTA finalises rows [kFwdRows*crank/C, kFwdRows*(crank+1)/C) of the row group.
    const int r_lo = kFwdRows * crank / C, r_hi = kFwdRows * (crank + 1) / C, nr = r_hi - r_lo;
    const int64_t n_lo = static_cast<int64_t>(blockIdx.y) * kFwdRows + r_lo;
    const int nv = static_cast<int>(N - n_lo < nr ? (N - n_lo > 0 ? N - n_lo : 0) : nr);  // rows inside W
    for (int i = threadIdx.x; i < nv * M; i += blockDim.x) {
        const int rr = i % nv, tok = i / nv;
        float sum = 0.0f;
        for (int src = 0; src < C; ++src) sum += recv[(src * nrmax + rr) * MP + tok];
        p.out[static_cast<int64_t>(tok) * N + n_lo + rr] = __bfloat16_as_ushort(__float2bfloat16_rn(sum));
    }
}

template <int NG>
__global__ void __launch_bounds__(kDecThreads, NG <= 2 ? 2 : 1) k_decode_fwd(const DecodeParams p) {
    extern __shared__ __align__(16) uint8_t smem[];
    if ((smem_addr(smem) & 0x00ffffffu) == kDynSmemBase)
        decode_fwd_body<NG, true>(p, smem);
    else
        decode_fwd_body<NG, false>(p, smem);
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

template <int NG, bool kFixedBase>
__device__ __forceinline__ void decode_bwd_body(const DecodeParams &p, uint8_t *smem) {
    constexpr int MP = 8 * NG;
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
    const uint32_t lane4 = lut_lane_operand<kFixedBase>(lut, lane);

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

    // L2 prefetch of everything this CTA reads (first, so that DRAM streams while the CTA sets
    // up): the warp's codes (rows [16 s_lo, 16 s_hi) x 32 bytes of column kb) and their
    // constants, the grad_h slice, the adapter rows.
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
    build_pair_lut(lut);
    for (int i = threadIdx.x; i < rpad * MP; i += blockDim.x) upart[i] = 0.0f;
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
                    af[i][0] = lut_pair<kFixedBase>(lut, e01, lane4, i);
                    af[i][1] = lut_pair<kFixedBase>(lut, o01, lane4, i);
                    af[i][2] = lut_pair<kFixedBase>(lut, e23, lane4, i);
                    af[i][3] = lut_pair<kFixedBase>(lut, o23, lane4, i);
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

    __syncthreads();           // partials written; every warp is done with the pair table
    cluster_arrive_release();  // this CTA's partials (base and adapter) are ready for the cluster

    // ---- this CTA finalises features [F*crank/C, F*(crank+1)/C) of the CTA group's F features
    constexpr int F = 64 * kBwdCols;
    const int f_lo = F * crank / C, f_hi = F * (crank + 1) / C, nf = f_hi - f_lo;
    const int64_t k_lo = static_cast<int64_t>(blockIdx.y) * F + f_lo;
    const int nvf = static_cast<int>(K - k_lo < nf ? (K - k_lo > 0 ? K - k_lo : 0) : nf);  // features inside W
    // While the cluster barrier completes: stage the adapter columns A[:, k_lo, k_lo + nvf) as
    // as[j][f] in the (now unused) pair-table region, at most 256 x 128 bf16 = 64 KB.
    uint16_t *as = reinterpret_cast<uint16_t *>(lut);
    if (p.r > 0 && nvf > 0) stage_cols(as, p.A, K, k_lo, p.r, nvf);
    cluster_wait_acquire();  // every CTA's partials are visible in the cluster
    grid_dependents_launch();

    // Remote reads: adapter sums (ufull[j][tok] = bf16(s * B^T grad_h)) and, with more than one
    // CTA per cluster, the base sums of the owned features into red[f - f_lo][tok] (at most
    // 64 x 64 floats) behind the staged A columns.
    if (p.r > 0) {
        for (int i = threadIdx.x; i < p.r * M; i += blockDim.x) {
            const int j = i / M, tok = i % M;
            float sum = 0.0f;
#pragma unroll
            for (int cc = 0; cc < kMaxCluster; ++cc)
                if (cc < C) sum += cluster.map_shared_rank(upart, cc)[j * MP + tok];
            ufull[j * MP + tok] = round_bf16(sum * p.s);
        }
    }
    auto base_sum = [&](const float *rp, int fl, int tok) {
        const int c = fl / 64, f = fl % 64;
        float v = 0.0f;
#pragma unroll
        for (int sb = 0; sb < kBwdSub; ++sb) v += rp[((sb * kBwdCols + c) * 64 + f) * MP + tok];
        return v;
    };
    float *red = reinterpret_cast<float *>(lut + kLutBytes / 2);
    if (C > 1) {
        for (int i = threadIdx.x; i < nvf * M; i += blockDim.x) {
            const int ff = i % nvf, tok = i / nvf;
            float v[kMaxCluster];
#pragma unroll
            for (int cc = 0; cc < kMaxCluster; ++cc)
                v[cc] = cc < C ? base_sum(cluster.map_shared_rank(part, cc), f_lo + ff, tok) : 0.0f;
            float sum = 0.0f;
#pragma unroll
            for (int cc = 0; cc < kMaxCluster; ++cc)
                if (cc < C) sum += v[cc];
            red[ff * MP + tok] = sum;
        }
    }
    cluster_arrive_release();  // done reading other CTAs' shared memory
    __syncthreads();

    for (int i = threadIdx.x; i < nvf * M; i += blockDim.x) {
        const int ff = i % nvf, tok = i / nvf;
        float sum = C > 1 ? red[ff * MP + tok] : base_sum(part, f_lo + ff, tok);
        if (p.r > 0) {
            float lora = 0.0f;
            for (int j = 0; j < p.r; ++j)
                lora = __fmaf_rn(__uint_as_float(static_cast<uint32_t>(as[j * nvf + ff]) << 16), ufull[j * MP + tok], lora);
            sum += lora;
        }
        p.out[static_cast<int64_t>(tok) * K + k_lo + ff] = __bfloat16_as_ushort(__float2bfloat16_rn(sum));
    }
    cluster_wait_acquire();  // every CTA is done reading this CTA's shared memory
}

template <int NG>
__global__ void __launch_bounds__(kDecThreads) k_decode_bwd(const DecodeParams p) {
    extern __shared__ __align__(16) uint8_t smem[];
    if ((smem_addr(smem) & 0x00ffffffu) == kDynSmemBase)
        decode_bwd_body<NG, true>(p, smem);
    else
        decode_bwd_body<NG, false>(p, smem);
}

// Raise a kernel's dynamic shared-memory limit only when a launch needs more than any
// earlier one (the attribute call is skipped on the steady-state path).
cudaError_t ensure_smem(const void *kern, size_t smem) {
    static thread_local const void *kerns[16];
    static thread_local size_t limits[16];
    static thread_local int nk = 0;
    int slot = -1;
    for (int i = 0; i < nk; ++i)
        if (kerns[i] == kern) slot = i;
    if (slot >= 0 && limits[slot] >= smem) return cudaSuccess;
    const cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    if (slot < 0 && nk < 16) {
        slot = nk++;
        kerns[slot] = kern;
    }
    if (slot >= 0) limits[slot] = smem;
    return cudaSuccess;
}

cudaLaunchConfig_t cluster_config(dim3 grid, int cluster_x, size_t smem, cudaStream_t st, cudaLaunchAttribute *attr,
                                  bool pdl) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = dim3(kDecThreads, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
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
    cfg.numAttrs = pdl ? 2 : 1;
    return cfg;
}

// Clusters of `C` CTAs with `smem` bytes each that are resident at once on this device
// (the occupancy query accounts for GPC boundaries), cached per (device, kernel, C, smem).
int max_active_clusters(const void *kern, int C, size_t smem) {
    struct Entry {
        int dev;
        const void *kern;
        int C;
        size_t smem;
        int n;
    };
    static thread_local Entry cache[64];
    static thread_local int nc = 0;
    int dev = 0;
    cudaGetDevice(&dev);
    for (int i = 0; i < nc; ++i)
        if (cache[i].dev == dev && cache[i].kern == kern && cache[i].C == C && cache[i].smem == smem) return cache[i].n;
    int n = 0;
    if (ensure_smem(kern, smem) == cudaSuccess) {
        cudaLaunchAttribute attr[2];
        cudaLaunchConfig_t cfg = cluster_config(dim3(C, 1, 1), C, smem, nullptr, attr, false);
        if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) != cudaSuccess) {
            (void)cudaGetLastError();
            n = 0;
        }
    }
    if (nc < 64) cache[nc++] = Entry{dev, kern, C, smem, n};
    return n;
}

// Cluster size: the largest C <= 8 whose grid (tiles x C CTAs) is resident in one wave,
// keeping at least `min_units` units of reduction work per CTA; 1 when none fits.
int pick_cluster(const void *kern, size_t smem, int64_t tiles, int64_t red_units, int64_t min_units) {
    for (int C = kMaxCluster; C > 1; --C) {
        if (red_units / C < min_units) continue;
        if (tiles <= max_active_clusters(kern, C, smem)) return C;
    }
    return 1;
}

template <typename Kern>
cudaError_t launch_cluster(Kern kern, dim3 grid, int cluster_x, size_t smem, cudaStream_t st, const DecodeParams &p) {
    cudaError_t e = ensure_smem(reinterpret_cast<const void *>(kern), smem);
    if (e != cudaSuccess) return e;
    cudaLaunchAttribute attr[2];
    const cudaLaunchConfig_t cfg = cluster_config(grid, cluster_x, smem, st, attr, true);
    e = cudaLaunchKernelEx(&cfg, kern, p);
    count_launch();
    return e;
}

int pick_groups(int M) { return M <= 8 ? 1 : M <= 16 ? 2 : M <= 32 ? 4 : 8; }

template <typename Kern>
cudaError_t launch_picked(Kern kern, size_t smem, int64_t tiles, int64_t red_units, int64_t min_units, cudaStream_t st,
                          const DecodeParams &p) {
    const int C = pick_cluster(reinterpret_cast<const void *>(kern), smem, tiles, red_units, min_units);
    return launch_cluster(kern, dim3(C, static_cast<unsigned>(tiles), 1), C, smem, st, p);
}

}  // namespace

cudaError_t launch_decode_fwd(const WeightView &w, const uint16_t *x, int M, const uint16_t *A, const uint16_t *B,
                              int r, float s, uint16_t *h, cudaStream_t st) {
    if (M <= 0 || w.n == 0) return cudaSuccess;
    DecodeParams p{w.codes, w.q, w.sigma, w.mu, w.n, w.k, x, M, A, B, r, s, h};
    const int NG = pick_groups(M);
    const int rpad = (r + 15) & ~15;
    const size_t smem = kLutBytes + sizeof(float) * ((kFwdRows + kMaxCluster) * 8 * NG + rpad * 8 * NG);
    const int64_t tiles = (w.n + kFwdRows - 1) / kFwdRows;
    const int64_t red = w.k / kBlock;
    switch (NG) {
        case 1: return launch_picked(k_decode_fwd<1>, smem, tiles, red, 4, st, p);
        case 2: return launch_picked(k_decode_fwd<2>, smem, tiles, red, 4, st, p);
        case 4: return launch_picked(k_decode_fwd<4>, smem, tiles, red, 4, st, p);
        default: return launch_picked(k_decode_fwd<8>, smem, tiles, red, 4, st, p);
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
    const int64_t red = (w.n + 15) / 16 / kBwdSub;
    switch (NG) {
        case 1: return launch_picked(k_decode_bwd<1>, smem, tiles, red, 2, st, p);
        case 2: return launch_picked(k_decode_bwd<2>, smem, tiles, red, 2, st, p);
        case 4: return launch_picked(k_decode_bwd<4>, smem, tiles, red, 2, st, p);
        default: return cudaErrorInvalidValue;  // callers split tokens into chunks of 32
    }
}

}  // namespace qn
