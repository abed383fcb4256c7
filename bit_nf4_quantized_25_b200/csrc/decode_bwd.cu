// decode_bwd.cu -- QLoRA input gradient for few tokens (M <= 64) on sm_100a.
//
//   grad_x[m,k] = sum_n grad_h[m,n] W'[n,k] + sum_j A[j,k] u[m,j],  u = s B^T grad_h
// ("How does QLoRA work for training?", aivaro.ru, section 7: the frozen base is dequantised
// on the fly for the gradient and not updated).
//
// The reduction runs over weight rows, whose block constants differ, so the constants scale
// the bf16 token operand (c'_b * grad_h), and the nibbles of neighbouring rows are interleaved
// so that a byte again indexes a pair of the table in decode_common.cuh. A CTA owns two 64-
// feature block columns; the rows are split over a thread-block cluster and, inside a CTA,
// over four warp sub-slices.
#include "decode_common.cuh"

namespace qn {

namespace {
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

// Asynchronous 16-byte copy global -> shared (L2 only); src_bytes = 0 writes zeros.
__device__ __forceinline__ void cp_async16(void *dst, const void *src, uint32_t src_bytes) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_addr(dst)), "l"(src), "r"(src_bytes)
                 : "memory");
}
__device__ __forceinline__ void cp_async_commit_wait_all() {
    asm volatile("cp.async.commit_group;\ncp.async.wait_all;" ::: "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }

template <int NG, bool kFixedBase>
__device__ __forceinline__ void decode_bwd_body(const DecodeParams &p, uint8_t *smem) {
    constexpr int MP = 8 * NG;
    constexpr int F = 64 * kBwdCols;  // features (grad_x columns) of this CTA
    uint8_t *lut = smem;
    // After the main loop the table region holds part[warp][64 features][MP], each warp's sums.
    float *part = reinterpret_cast<float *>(smem);
    // recv[src][f - f_lo][MP]: the sums that cluster rank `src` pushes for the features this CTA
    // finalises (at most F + kMaxCluster rows in all).
    float *recv = reinterpret_cast<float *>(smem + kLutBytes);
    const int rpad = (p.r + 15) & ~15;
    float *upart = recv + (F + kMaxCluster) * MP;                   // [rpad][MP] partial B^T grad_h
    float *scratch = upart + rpad * MP;                              // [kDecWarps / 2][16][MP] warp-sum tree
    uint16_t *as = reinterpret_cast<uint16_t *>(scratch + kDecWarps / 2 * 16 * MP);  // [rpad][F] A[:, k0 .. k0 + F)

    cg::cluster_group cluster = cg::this_cluster();
    const int C = static_cast<int>(cluster.num_blocks());
    const int crank = static_cast<int>(cluster.block_rank());
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int gq = lane >> 2, t = lane & 3;
    const uint32_t lane4 = lut_lane_operand<kFixedBase>(lut, lane);

    const int64_t N = p.n, K = p.k;
    const int64_t nbr = K / kBlock;
    const int col = warp % kBwdCols, sub = warp / kBwdCols;
    const int64_t k0 = static_cast<int64_t>(blockIdx.y) * F;
    const int64_t kb = static_cast<int64_t>(blockIdx.y) * kBwdCols + col;  // this warp's block column
    const bool vk = kb < nbr;
    const int64_t kbc = vk ? kb : 0;
    // reduction rows in 16-row steps: cluster slice, then this warp's sub-slice
    const int64_t n16 = (N + 15) / 16;
    const int64_t c_lo = n16 * crank / C, c_hi = n16 * (crank + 1) / C;
    const int64_t s_lo = c_lo + (c_hi - c_lo) * sub / kBwdSub, s_hi = c_lo + (c_hi - c_lo) * (sub + 1) / kBwdSub;

    // Before the dependency wait only L2 prefetches of the grad_h slice and the adapter rows B.
    if (warp == 0 && lane < p.M) {
        const int64_t n_lo = c_lo * 16, n_hi = c_hi * 16 < N ? c_hi * 16 : N;
        prefetch_range(p.act + lane * N + n_lo, (n_hi - n_lo) * 2);
    }
    if (warp == 1 && lane == 0 && p.r > 0) {
        const int64_t n_lo = c_lo * 16, n_hi = c_hi * 16 < N ? c_hi * 16 : N;
        prefetch_range(p.B + n_lo * p.r, (n_hi - n_lo) * p.r * 2);
    }
    cluster_arrive_relaxed();  // phase 1: this CTA is running (its shared memory may be written)
    grid_dependency_wait();

    // Adapter columns A[j][k0 .. k0 + F) -> as[j][.], asynchronously (consumed at the end).
    for (int i = threadIdx.x; i < p.r * (F / 8); i += blockDim.x) {
        const int j = i / (F / 8), c = i % (F / 8);
        const bool ok = k0 + 8 * c < K;
        cp_async16(as + j * F + 8 * c, p.A + static_cast<int64_t>(j) * K + (ok ? k0 + 8 * c : 0), ok ? 16u : 0u);
    }
    cp_async_commit();

    const float mu = load_mu(p.mu, p.absmax);
    const int M = p.M;

    // Lane (gq, t) reads, per step st, the 4 code bytes [4 gq, 4 gq + 4) of block column kb of
    // rows 16 st + 4 t + i (i < 4), and the constant of row 16 st + 4 t + (gq & 3).
    const int64_t rstride = K / 2;  // bytes per weight row
    const uint8_t *cw = p.codes + (4 * t) * rstride + kbc * 32 + 4 * gq;
    const int64_t erow = (4 * t + (gq & 3)) * nbr + kbc;  // flattened block index, step 0
    const int nst = vk && s_hi > s_lo ? static_cast<int>(s_hi - s_lo) : 0, ngrp = (nst + 1) / 2;

    const int64_t nfull = N / 16;  // steps below this one have all 16 rows inside W
    auto load_group = [&](int gi, BwdGroup &G) {
        // both steps of the group complete and inside W: no per-row predicates (the common case)
        const bool gfull = 2 * gi + 2 <= nst && s_lo + 2 * gi + 2 <= nfull;
#pragma unroll
        for (int j = 0; j < 2; ++j) {
            const int64_t st = s_lo + 2 * gi + j;
            const bool sv = 2 * gi + j < nst;
            const uint8_t *rowp = cw + st * 16 * rstride;
            if (gfull) {
#pragma unroll
                for (int i = 0; i < 4; ++i) G.w[j][i] = ld_nc_u32(rowp + i * rstride);
            } else {
#pragma unroll
                for (int i = 0; i < 4; ++i)
                    G.w[j][i] = (sv && st * 16 + 4 * t + i < N) ? ld_nc_u32(rowp + i * rstride) : 0x77777777u;
            }
            const bool ok = sv && st * 16 + 4 * t + (gq & 3) < N;
            const uint64_t bi = static_cast<uint64_t>(erow + st * 16 * nbr);
            if (p.absmax) {  // the fp32 constant itself, in G.s
                G.q[j] = 0u;
                G.s[j] = ok ? __ldg(p.absmax + bi) : 0.0f;
            } else {
                G.q[j] = ok ? __ldg(p.q + bi) : 0u;
                G.s[j] = ok ? __ldg(p.sigma + bi / kGroup) : 0.0f;
            }
        }
    };

    float acc[4][NG][4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int tg = 0; tg < NG; ++tg) acc[i][tg][0] = acc[i][tg][1] = acc[i][tg][2] = acc[i][tg][3] = 0.0f;

    BwdGroup G0, G1;  // ping-pong: two groups of codes in flight while one is consumed
    if (ngrp > 0) load_group(0, G0);
    if (ngrp > 1) load_group(1, G1);

    // ---- LoRA: partial u[j][tok] = sum_n B[n][j] grad_h[tok][n] over this CTA's row slice, run
    // after the first group of codes has been consumed.
    auto lora_down = [&]() {
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
            warp_tree_sum<NG>(d, scratch, upart + jt * 16 * MP);  // fixed order: bit-reproducible
        }
    };

    // The pair table is built while the first codes are in flight.
    build_pair_lut(lut, p.qtype);
    __syncthreads();

    // ---- base: block column kb, group gi holds steps s_lo + 2 gi, + 1.
    auto compute_group = [&](const BwdGroup &G, int gi) {
#pragma unroll
        for (int j = 0; j < 2; ++j) {
            if (2 * gi + j >= nst) break;
            const int64_t n0 = (s_lo + 2 * gi + j) * 16 + 4 * t;  // this lane's 4 reduction rows
            // constant of row n0 + (gq & 3), shared with the lanes of the same t
            const float mine = p.absmax ? G.s[j] : block_constant(static_cast<uint8_t>(G.q[j]), G.s[j], mu);
            float cp[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) cp[i] = __shfl_sync(0xffffffffu, mine, (i << 2) | t);
            if (s_lo + 2 * gi + j >= nfull) {  // the step reaches past row N - 1
#pragma unroll
                for (int i = 0; i < 4; ++i)
                    if (n0 + i >= N) cp[i] = 0.0f;
            }
            uint32_t e01, o01, e23, o23;
            interleave_rows(G.w[j][0], G.w[j][1], e01, o01);
            interleave_rows(G.w[j][2], G.w[j][3], e23, o23);
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
                for (int i = 0; i < 4; ++i) mma_16816(acc[i][tg], af[i][0], af[i][1], af[i][2], af[i][3], b0, b1);
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
    __syncthreads();  // every warp is done with the pair table; upart holds this CTA's B^T grad_h

    // Each warp's sums into the (now free) table region. D row gq of tile i is feature
    // 8*gq + 2i, row gq+8 is feature 8*gq + 2i + 1.
    {
        float *wp = part + warp * 64 * MP;
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int tg = 0; tg < NG; ++tg) {
                const int f = 8 * gq + 2 * i, tok = tg * 8 + 2 * t;
                *reinterpret_cast<float2 *>(wp + f * MP + tok) = make_float2(acc[i][tg][0], acc[i][tg][1]);
                *reinterpret_cast<float2 *>(wp + (f + 1) * MP + tok) = make_float2(acc[i][tg][2], acc[i][tg][3]);
            }
    }
    cp_async_commit_wait_all();  // the adapter columns have landed
    __syncthreads();

    // ---- CTA sums (4 warp sub-slices + the adapter term of this CTA's row slice:
    // s * sum_j A[j][k] u_c[j][tok], fp32) pushed to the CTA that finalises the feature.
    const int nfmax = (F + C - 1) / C;
    cluster_wait();  // phase 1: every CTA of the cluster is running
    for (int i = threadIdx.x; i < F * M; i += blockDim.x) {
        const int fl = i % F, tok = i / F;
        const int c = fl / 64, f = fl % 64;
        float v = 0.0f;
#pragma unroll
        for (int sb = 0; sb < kBwdSub; ++sb) v += part[((sb * kBwdCols + c) * 64 + f) * MP + tok];
        if (p.r > 0) {
            float lora = 0.0f;
            for (int j = 0; j < p.r; ++j)
                lora = __fmaf_rn(__uint_as_float(static_cast<uint32_t>(as[j * F + fl]) << 16), upart[j * MP + tok], lora);
            v = __fmaf_rn(p.s, lora, v);
        }
        const int owner = (fl * C + C - 1) / F;  // largest c with F*c/C <= fl
        const int rr = fl - F * owner / C;
        cluster.map_shared_rank(recv, owner)[(crank * nfmax + rr) * MP + tok] = v;
    }
    cluster_arrive_release();
    cluster_wait_acquire();  // phase 2: every sum has landed
    grid_dependents_launch();

    // ---- this CTA finalises features [F*crank/C, F*(crank+1)/C) of the CTA's F features
    const int f_lo = F * crank / C, f_hi = F * (crank + 1) / C, nf = f_hi - f_lo;
    const int64_t k_lo = k0 + f_lo;
    const int nvf = static_cast<int>(K - k_lo < nf ? (K - k_lo > 0 ? K - k_lo : 0) : nf);  // features inside W
    for (int i = threadIdx.x; i < nvf * M; i += blockDim.x) {
        const int rr = i % nvf, tok = i / nvf;
        float sum = 0.0f;
        for (int src = 0; src < C; ++src) sum += recv[(src * nfmax + rr) * MP + tok];
        p.out[static_cast<int64_t>(tok) * K + k_lo + rr] = __bfloat16_as_ushort(__float2bfloat16_rn(sum));
    }
}

template <int NG>
__global__ void __launch_bounds__(kDecThreads) k_decode_bwd(const DecodeParams p) {
    extern __shared__ __align__(16) uint8_t smem[];
    if ((smem_addr(smem) & 0x00ffffffu) == kDynSmemBase)
        decode_bwd_body<NG, true>(p, smem);
    else
        decode_bwd_body<NG, false>(p, smem);
}

}  // namespace

cudaError_t launch_decode_bwd(const WeightView &w, const uint16_t *gh, int M, const uint16_t *A, const uint16_t *B,
                              int r, float s, uint16_t *gx, cudaStream_t st) {
    if (M <= 0 || w.k == 0) return cudaSuccess;
    DecodeParams p{w.codes, w.q, w.sigma, w.mu, w.absmax, w.qtype, w.n, w.k, gh, M, A, B, r, s, gx};
    const int NG = pick_groups(M);
    const int rpad = (r + 15) & ~15;
    // table (later the warps' sums) | recv | upart | warp-sum scratch | staged adapter columns
    const size_t smem =
        kLutBytes +
        sizeof(float) * ((64 * kBwdCols + kMaxCluster) * 8 * NG + rpad * 8 * NG + kDecWarps / 2 * 16 * 8 * NG) +
        sizeof(uint16_t) * rpad * 64 * kBwdCols;
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
