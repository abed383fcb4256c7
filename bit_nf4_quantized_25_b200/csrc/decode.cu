// decode.cu -- QLoRA linear forward for few tokens (M <= 64) on sm_100a.
//
//   h[m,n] = sum_k W'[n,k] x[m,k] + sum_j B[n,j] t[m,j],  t = s A x,  W'[n,k] = NF4[code] * c'_b
// ("Quantized LoRA (QLoRA) and 4-bit training", apxml.com, forward equations; "How does QLoRA
// work for training?", aivaro.ru, section 2).
//
// Few tokens make this HBM-bound: each packed weight is read once and used M times. B200
// streams about 13e12 weights/s but its SMs issue only ~3.6e13 lane-instructions/s, so the
// whole per-weight budget is under three instructions. The multiply-accumulate therefore runs
// on the tensor cores (mma.sync m16n8k16: A = 16 weight rows, B = 8 tokens) and dequantisation
// is one byte permute plus one shared-memory load per TWO weights (the pair table of
// decode_common.cuh). The table holds the unscaled NF4 values; every 64-weight block is
// reduced in its own fp32 fragment and scaled by its constant c'_b (the same sum, constant
// applied after the dot product). A lane computes the constants of one block per group of four
// and the quad shares them with shuffles.
//
// A CTA owns 128 weight rows (8 warps x 16) over one K-slice; the K-slices of a row group form a
// thread-block cluster (<= 8 CTAs, sized so the grid is one wave). Each CTA adds the adapter
// term of its own K-slice (B (s t_c), t_c = A x over the slice) to its partial sums, pushes
// them into the shared memory of the CTA that finalises those rows, and one cluster barrier
// later that CTA sums and stores. Codes stream through two register groups (ping-pong);
// nothing is read from global memory before the programmatic-launch wait except L2 prefetches
// of the activation and adapter slices.
#include "decode_common.cuh"

namespace qn {

namespace {
// ------------------------------------------------------------------------- forward
// Registers of one group of GB (2 or 4) 64-weight blocks for rows A (g) and B (g + 8) of a lane.
template <int GB>
struct FwdGroup {
    uint2 ca[GB], cb[GB];
    uint32_t qa, qb;  // block t % GB of the group (the quad's lanes share them)
    float sa, sb;
};

// Blocks per register group, CTAs per SM and where the adapter down-projection runs. Groups of
// four blocks with two CTAs per SM (128 registers) measured faster than groups of two with three
// CTAs per SM (80 registers). With one token group the down-projection fits inside the loop,
// after the first group; with more tokens it runs after the loop to save registers.
template <int NG>
struct FwdShape {
    static constexpr int kGB = 4;
    static constexpr int kMinBlocks = NG <= 2 ? 2 : 1;
    static constexpr bool kAdapterInLoop = NG == 1;
};

template <int NG, bool kFixedBase>
__device__ __forceinline__ void decode_fwd_body(const DecodeParams &p, uint8_t *smem) {
    constexpr int MP = 8 * NG;  // padded token count
    constexpr int GB = FwdShape<NG>::kGB;
    using Group = FwdGroup<GB>;
    uint8_t *lut = smem;
    // recv[src][row - r_lo][MP]: the partial sums that cluster rank `src` pushes for the rows
    // this CTA finalises (at most kFwdRows + kMaxCluster rows in all).
    float *recv = reinterpret_cast<float *>(smem + kLutBytes);
    const int rpad = (p.r + 15) & ~15;
    float *tpart = recv + (kFwdRows + kMaxCluster) * MP;  // [rpad][MP] partial A x of this CTA's k-slice
    float *scratch = tpart + rpad * MP;                   // [kDecWarps / 2][16][MP] warp-sum tree

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
    // Rows past N read row 0 (valid memory) and get a zero block constant; tokens past M read
    // token 0 and fill MMA columns that are never stored. The hot loop therefore only needs
    // the block count of the last (partial) group.
    const int nblk = b_hi - b_lo, ngrp = (nblk + GB - 1) / GB;
    constexpr bool kAdapterInLoop = FwdShape<NG>::kAdapterInLoop;
    uint32_t bf[4] = {0u, 0u, 0u, 0u};  // B fragment of the first 16 adapter columns
    if (kAdapterInLoop && p.r > 0) load_b_frag(p, rowA, rowB, vA, vB, 2 * t, bf[0], bf[1], bf[2], bf[3]);
    const uint2 *pa = reinterpret_cast<const uint2 *>(p.codes + (vA ? rowA : 0) * (K / 2) +
                                                      static_cast<int64_t>(b_lo) * 32 + 8 * t);
    const uint2 *pb = reinterpret_cast<const uint2 *>(p.codes + (vB ? rowB : 0) * (K / 2) +
                                                      static_cast<int64_t>(b_lo) * 32 + 8 * t);
    // flattened index of lane t's block in group 0 (the lane loads that block's constants)
    const int tb = t % GB;  // the block of each group whose constants this lane loads
    const int64_t eA = (vA ? rowA : 0) * nbr + b_lo + tb, eB = (vB ? rowB : 0) * nbr + b_lo + tb;

    auto load_group = [&](int gi, Group &G) {
        const int cnt = nblk - GB * gi;  // blocks in this group (at least 1)
        const uint2 *ga = pa + 4 * GB * gi, *gb = pb + 4 * GB * gi;
#pragma unroll
        for (int j = 0; j < GB; ++j) {
            G.ca[j] = j < cnt ? __ldcs(ga + 4 * j) : make_uint2(0u, 0u);
            G.cb[j] = j < cnt ? __ldcs(gb + 4 * j) : make_uint2(0u, 0u);
        }
        const bool ok = tb < cnt;
        const uint64_t ea = static_cast<uint64_t>(eA + GB * gi), eb = static_cast<uint64_t>(eB + GB * gi);
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

    Group G0, G1;  // ping-pong: two groups of codes in flight while one is consumed
    if (ngrp > 0) load_group(0, G0);
    if (ngrp > 1) load_group(1, G1);

    // ---- LoRA down-projection over this CTA's k-slice (partial t = A x, fp32), run after the
    // first group (one token group) or after the loop: its operands are L2 hits that would
    // otherwise queue behind the first code loads. Item (j-tile, eighth of the slice) per warp.
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
            warp_tree_sum<NG>(d, scratch, tpart + jt * 16 * MP);  // fixed order: bit-reproducible
        }
    };

    // The pair table is built while the first codes are in flight.
    build_pair_lut(lut);
    __syncthreads();

    // ---- base: group gi holds blocks b_lo + GB gi .. + GB of rows A and B.
    auto compute_group = [&](const Group &G, int gi) {
        const int cnt = nblk - GB * gi;
        const bool ok = tb < cnt;
        const float cA4 = (vA && ok) ? block_constant(static_cast<uint8_t>(G.qa), G.sa, mu) : 0.0f;
        const float cB4 = (vB && ok) ? block_constant(static_cast<uint8_t>(G.qb), G.sb, mu) : 0.0f;
#pragma unroll
        for (int j = 0; j < GB; ++j) {
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
            const int xo = 8 * (GB * gi + j);
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
        if (kAdapterInLoop && gi == 0 && p.r > 0) lora_down();
        if (gi + 2 < ngrp) load_group(gi + 2, G0);
        if (gi + 1 < ngrp) {
            compute_group(G1, gi + 1);
            if (gi + 3 < ngrp) load_group(gi + 3, G1);
        }
    }
    // Adapter after the loop: the B fragment of the first 16 adapter columns is requested
    // before the down-projection so that both L2 round trips overlap.
    if (p.r > 0 && !kAdapterInLoop) load_b_frag(p, rowA, rowB, vA, vB, 2 * t, bf[0], bf[1], bf[2], bf[3]);
    if (p.r > 0 && (!kAdapterInLoop || ngrp == 0)) lora_down();
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
__global__ void __launch_bounds__(kDecThreads, FwdShape<NG>::kMinBlocks) k_decode_fwd(const DecodeParams p) {
    extern __shared__ __align__(16) uint8_t smem[];
    if ((smem_addr(smem) & 0x00ffffffu) == kDynSmemBase)
        decode_fwd_body<NG, true>(p, smem);
    else
        decode_fwd_body<NG, false>(p, smem);
}

}  // namespace

cudaError_t launch_decode_fwd(const WeightView &w, const uint16_t *x, int M, const uint16_t *A, const uint16_t *B,
                              int r, float s, uint16_t *h, cudaStream_t st) {
    if (M <= 0 || w.n == 0) return cudaSuccess;
    DecodeParams p{w.codes, w.q, w.sigma, w.mu, w.n, w.k, x, M, A, B, r, s, h};
    const int NG = pick_groups(M);
    const int rpad = (r + 15) & ~15;
    // table | recv | tpart | warp-sum scratch
    const size_t smem =
        kLutBytes + sizeof(float) * ((kFwdRows + kMaxCluster) * 8 * NG + rpad * 8 * NG + kDecWarps / 2 * 16 * 8 * NG);
    const int64_t tiles = (w.n + kFwdRows - 1) / kFwdRows;
    const int64_t red = w.k / kBlock;
    switch (NG) {
        case 1: return launch_picked(k_decode_fwd<1>, smem, tiles, red, 4, st, p);
        case 2: return launch_picked(k_decode_fwd<2>, smem, tiles, red, 4, st, p);
        case 4: return launch_picked(k_decode_fwd<4>, smem, tiles, red, 4, st, p);
        default: return launch_picked(k_decode_fwd<8>, smem, tiles, red, 4, st, p);
    }
}

}  // namespace qn
