// decode_fwd.cu -- QLoRA linear forward for few tokens (M <= 16 per launch) on sm_100a.
//
//   h[m,n] = sum_k W'[n,k] x[m,k] + sum_j B[n,j] t[m,j],  t = s A x,  W'[n,k] = NF4[code] * c'_b
// ("Quantized LoRA (QLoRA) and 4-bit training", apxml.com, forward equations; "How does QLoRA
// work for training?", aivaro.ru, section 2).
//
// Few tokens make this HBM-bound: each packed weight is read once and used M times. The
// per-weight instruction budget is under three, so the multiply-accumulate runs on the tensor
// cores (mma.sync m16n8k16: A = 16 weight rows, B = 8 tokens) and dequantisation is one byte
// permute plus one shared-memory load per TWO weights (the pair table of stream_common.cuh).
// The table holds the unscaled NF4 values; every 64-weight block is reduced in its own fp32
// fragment and scaled by its constant c'_b.
//
// Work split. One CTA per SM. A CTA owns R = 16 m weight rows over one K-slice; the C K-slices
// of a row chunk form a thread-block cluster (R and C are chosen on the host so that the grid
// fills the SMs evenly). The CTA streams its (R rows x K-slice) tile through a ring of stages;
// a stage is R rows x 4 blocks of codes (one TMA box: one large box per stage keeps the copy
// engine near the HBM rate, several small boxes do not), the matching 4 x 64 columns of x and
// of the adapter A, and the inputs of the R x 4 block constants.
//   warp 0      : producer. Lane 0 issues the codes box; the 32 lanes copy x, A (16-byte
//                 cp.async into the 128-byte swizzled layout) and the constant inputs (the
//                 FP8 codes and group scales) with cp.async; every copy completes on the
//                 stage's full barrier.
//   warps 1..16 : consumers. Warp (kg, rg) takes block kg of every stage and the m-tiles
//                 rg, rg + 4, ... of the chunk: codes -> pair table -> mma.sync with x, one fp32
//                 fragment per block scaled by c'_b into the accumulators. The four lanes of a
//                 quad compute the block constants c'_b = fma(e4m3(q_b), sigma_g, mu) the quad
//                 needs and share them by shuffles. Each warp also runs a share of the adapter
//                 down-projection t_c = A x over the stage (mma.sync).
// After the loop the four block-warps of each m-tile are summed in a fixed order, the slice's
// adapter term B (s t_c) is added on the tensor cores, and the partial sums are pushed with DSMEM
// stores into the CTA of the cluster that finalises those rows; one cluster barrier later that
// CTA sums the slices in rank order and stores h. Results are bit-reproducible.
//
// Nothing is read from global memory before the programmatic-launch wait. Every mbarrier wait
// is bounded; a timeout records an error code in the workspace error word, stops the CTA's
// work (cluster and named barriers are still passed, so no CTA waits forever) and drains the
// loads already issued.
#include <cudaTypedefs.h>

#include "host_cache.h"
#include "stream_common.cuh"

namespace qn {

#ifdef QN_TIMELINE
// Per-CTA timestamps (globaltimer, ns) of the forward kernel's phases, for profiling builds only.
__device__ unsigned long long g_fwd_timeline[1024][8];
__device__ __forceinline__ void tl_mark(int slot) {
    unsigned long long t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    const unsigned cta = blockIdx.y * gridDim.x + blockIdx.x;
    if (cta < 1024) g_fwd_timeline[cta][slot] = t;
}
#define QN_TL(slot, cond) \
    do {                  \
        if (cond) tl_mark(slot); \
    } while (0)
#else
#define QN_TL(slot, cond) \
    do {                  \
    } while (0)
#endif

namespace {

using namespace sm100;
using namespace stream;

constexpr int kConsumers = 16;
constexpr int kThreads = 32 * (kConsumers + 1);
constexpr int kStageBlocks = 4;
constexpr int kMaxM = 16;           // m-tiles per chunk: R <= 256 rows (TMA box limit)
constexpr int kMaxStages = 8;
constexpr int kMaxCluster = 8;
constexpr size_t kSmemLimit = 227 * 1024;

struct FwdArgs {
    const uint8_t *q;
    const float *sigma;
    const float *mu;
    const uint16_t *B;  // n x r
    const uint16_t *x;  // M x k
    const uint16_t *A;  // r x k
    uint16_t *h;        // M x n
    int *err;
    int64_t n, k;
    int nbr;     // blocks per row (k / 64)
    int ncol;    // stage columns (ceil(nbr / 4))
    int M, r, rpad;  // rpad: r rounded up to 8, 16, 32 or 64 (0 without adapter)
    float s;
    int R, m;    // rows and m-tiles per chunk
    int C;       // K-slices (cluster size)
    int stages;
    // shared-memory layout (byte offsets from the start of dynamic shared memory)
    uint32_t slot_bytes, x_off, a_off, q_off, s_off;  // inside a slot
    uint32_t ring_off, recv_off, bar_off, post_off;
    uint32_t tx_bytes;
};

template <int NG, bool kFixedBase>
__device__ __forceinline__ void fwd_body(const CUtensorMap *tm_codes, const FwdArgs &p, uint8_t *smem) {
    constexpr int MP = 8 * NG;  // padded tokens
    constexpr int MW = 4 / NG;  // m-tiles per warp at most (m <= 4 MW)
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, t = lane & 3;
    const int C = p.C;
    const int crank = C > 1 ? static_cast<int>(cg::this_cluster().block_rank()) : 0;
    const int chunk = blockIdx.y;
    const int64_t row0 = static_cast<int64_t>(chunk) * p.R;
    const int col_lo = p.ncol * crank / C, col_hi = p.ncol * (crank + 1) / C;
    const int ns = col_hi - col_lo;
    const int S = p.stages;

    uint8_t *lut = smem;
    const uint32_t s_base = saddr(smem);
    const uint32_t s_ring = s_base + p.ring_off;
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + p.bar_off);
    uint64_t *empty = full + kMaxStages;
    volatile uint32_t *abort_flag = reinterpret_cast<volatile uint32_t *>(empty + kMaxStages);

    QN_TL(0, threadIdx.x == 0);
    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(&full[s], 32);  // the producer's 32 lanes (cp.async arrivals) + TMA bytes
            mbar_init(&empty[s], kConsumers);
        }
        *abort_flag = 0u;
        fence_barrier_init();
        tma_prefetch_desc(tm_codes);
    }
    build_pair_lut(lut, threadIdx.x, kThreads);
    // rows M .. MP-1 of x and r .. rpad-1 of A are read by the fragments but never copied: zero
    // them once in every slot
    for (int sidx = 0; sidx < S; ++sidx) {
        const uint32_t sl = s_ring + sidx * p.slot_bytes;
        const int xw = kStageBlocks * (MP - p.M) * 32, aw = kStageBlocks * (p.rpad - p.r) * 32;
        for (int i = threadIdx.x; i < xw; i += kThreads) {
            const int b = i / ((MP - p.M) * 32), rem = i % ((MP - p.M) * 32);
            asm volatile("st.shared.b32 [%0], %1;" ::"r"(sl + p.x_off + b * MP * 128 + (p.M + rem / 32) * 128 + (rem % 32) * 4),
                         "r"(0u)
                         : "memory");
        }
        for (int i = threadIdx.x; i < aw; i += kThreads) {
            const int b = i / ((p.rpad - p.r) * 32), rem = i % ((p.rpad - p.r) * 32);
            asm volatile("st.shared.b32 [%0], %1;" ::"r"(sl + p.a_off + b * p.rpad * 128 + (p.r + rem / 32) * 128 +
                                                      (rem % 32) * 4),
                         "r"(0u)
                         : "memory");
        }
    }
    __syncthreads();
    if (C > 1) cluster_arrive_relaxed();  // phase 1: this CTA runs (its shared memory may be written)
    grid_dependents_launch();
    grid_dependency_wait();  // x, A and B may come from the preceding kernel
    QN_TL(1, threadIdx.x == 0);

    auto fail = [&]() {
        if (atomicExch(const_cast<uint32_t *>(abort_flag), 1u) == 0u) record_error(p.err, kErrTimeout);
    };

    const int cw = warp - 1;  // consumer index
    const int kg = cw & 3, rg = cw >> 2;
    float acc[MW][NG][4];
#pragma unroll
    for (int i = 0; i < MW; ++i)
#pragma unroll
        for (int tg = 0; tg < NG; ++tg) acc[i][tg][0] = acc[i][tg][1] = acc[i][tg][2] = acc[i][tg][3] = 0.0f;
    float tacc[4] = {0.0f, 0.0f, 0.0f, 0.0f};
    const int NT = p.rpad / 8;  // adapter n-tiles of 8 ranks (1, 2, 4 or 8)

    if (warp == 0) {
        // ------------------------------------------------------------------ producer
        // Stage s: wait for its slot; lane 0 issues the TMA loads (codes, x, A); every lane copies
        // the constant inputs of its chunk rows (the aligned 8-byte window of q that holds the
        // stage's four FP8 codes, and the group scales of the first and last of the four blocks)
        // with cp.async, whose completion arrives on the same full barrier.
        const int RJ = (p.R + 31) >> 5;  // chunk rows per lane: lane + 32 j
        const int64_t nb = p.n * p.nbr;
        const int64_t ng = (nb + kGroup - 1) / kGroup;
        // the chunk's rows of B, read after the loop by the up-projection: into L2 now
        if (p.r > 0) {
            const int64_t nrows = (row0 + p.R <= p.n ? p.R : p.n - row0);
            const char *b0 = reinterpret_cast<const char *>(p.B + row0 * p.r);
            const int64_t bytes = nrows * p.r * 2;
            for (int64_t off = static_cast<int64_t>(lane) * 128; off < bytes; off += 32 * 128)
                asm volatile("prefetch.global.L2 [%0];" ::"l"(b0 + off) : "memory");
        }
        __syncwarp();
        int ni = 0;  // stages issued
        for (int s = 0; s < ns; ++s) {
            const int slot = s % S;
            if (*abort_flag) break;
            if (s >= S && !mbar_wait(&empty[slot], ((s / S) & 1) ^ 1)) {
                fail();
                break;
            }
            const int col = col_lo + s;
            const uint32_t sl = s_ring + slot * p.slot_bytes;
            if (lane == 0) {
                mbar_expect_tx(&full[slot], p.tx_bytes);
                tma_load_2d_saddr(sl, tm_codes, &full[slot], col * 128, static_cast<int32_t>(row0));
            }
            // x and A columns [256 col, 256 col + 256): row by row, lane j copies 16-byte chunk j & 7
            // of block j >> 3 into the 128-byte swizzled layout (chunk c of row rr at c ^ (rr & 7))
            {
                const int b = lane >> 3, c = lane & 7;
                const bool bvalid = 4 * col + b < p.nbr;
                const int64_t kcol = static_cast<int64_t>(4 * col + b) * 64 + 8 * c;
                for (int rr = 0; rr < p.M; ++rr) {
                    const uint32_t dst = sl + p.x_off + static_cast<uint32_t>(b * MP * 128 + rr * 128 + ((c ^ (rr & 7)) << 4));
                    cp_async16_zfill(dst, bvalid ? p.x + rr * p.k + kcol : p.x, bvalid ? 16u : 0u);
                }
                for (int rr = 0; rr < p.r; ++rr) {
                    const uint32_t dst =
                        sl + p.a_off + static_cast<uint32_t>(b * p.rpad * 128 + rr * 128 + ((c ^ (rr & 7)) << 4));
                    cp_async16_zfill(dst, bvalid ? p.A + rr * p.k + kcol : p.A, bvalid ? 16u : 0u);
                }
            }
            for (int j = 0; j < RJ; ++j) {
                const int i = lane + 32 * j;
                const int64_t row = row0 + i;
                if (i < p.R && row < p.n) {
                    const int64_t e0 = row * p.nbr + 4 * col;
                    const int64_t e3 = e0 + 3 < nb ? e0 + 3 : nb - 1;
                    const int64_t w0 = e0 & ~int64_t(3), w1 = w0 + 4;
                    const uint32_t qd = sl + p.q_off + static_cast<uint32_t>(i) * 8u;
                    const uint32_t sd = sl + p.s_off + static_cast<uint32_t>(i) * 8u;
                    cp_async4_zfill(qd, p.q + w0, 4);
                    const int64_t rest = nb - w1;
                    cp_async4_zfill(qd + 4, p.q + (rest > 0 ? w1 : w0), rest >= 4 ? 4u : (rest > 0 ? static_cast<uint32_t>(rest) : 0u));
                    cp_async4_zfill(sd, p.sigma + (e0 >> 8), 4);
                    cp_async4_zfill(sd + 4, p.sigma + ((e3 >> 8) < ng ? (e3 >> 8) : ng - 1), 4);
                }
            }
            cp_async_arrive_noinc(&full[slot]);  // one arrival per lane when its copies have landed
            ni = s + 1;
            QN_TL(2, lane == 0 && s == S - 1);
        }
        // drain: every copy this warp issued has landed before the CTA can exit
        cp_async_wait_all();
        if (lane == 0)
            for (int s = (ni > S ? ni - S : 0); s < ni; ++s) mbar_wait(&full[s % S], (s / S) & 1);
        __syncwarp();
    } else {
        // ------------------------------------------------------------------ consumers
        const uint32_t lane_op = lut_lane_operand<kFixedBase>(lut, lane);
        const uint32_t lut_base = s_base;
        const float mu = __ldg(p.mu);
        // x rows of this lane's tokens (tokens beyond M read a valid token; their columns of
        // the result are never stored), swizzle chunk offsets of x[tok][16 t .. 16 t + 16)
        uint32_t xr[NG], xc0[NG], xc1[NG];
#pragma unroll
        for (int tg = 0; tg < NG; ++tg) {
            int tok = tg * 8 + g;
            if (tok >= p.M) tok = tok % p.M;
            xr[tg] = static_cast<uint32_t>(tok) * 128u;
            xc0[tg] = static_cast<uint32_t>(((2 * t) ^ (tok & 7)) << 4);
            xc1[tg] = static_cast<uint32_t>(((2 * t + 1) ^ (tok & 7)) << 4);
        }
        const int nt_job = NT > 0 ? cw % NT : 0;
        const int kq_step = NT > 0 ? 16 / NT : 0;
        const int kq0 = NT > 0 ? cw / NT : 0;
        const int jrow = nt_job * 8 + g;  // adapter rank row of this lane's B fragment
        // The block constant this lane computes each stage: m-tile rg + 4 (t >> 1), row g + 8 (t & 1)
        // of it, block kg. The quad's four lanes cover the (up to) two m-tiles x two rows the quad
        // needs and share them with shuffles (MW = 4: a second pass for m-tiles rg + 8, rg + 12).
        int c_row[MW / 2 > 0 ? MW / 2 : 1];
        int64_t c_rowbase[MW / 2 > 0 ? MW / 2 : 1];
        uint32_t c_qoff[MW / 2 > 0 ? MW / 2 : 1];
#pragma unroll
        for (int pass = 0; pass < (MW + 1) / 2; ++pass) {
            const int mt = rg + 4 * (2 * pass + (t >> 1));
            const int i = 16 * mt + g + 8 * (t & 1);
            c_row[pass] = (mt < p.m && row0 + i < p.n) ? i : -1;
            c_rowbase[pass] = (row0 + i) * p.nbr;
            c_qoff[pass] = static_cast<uint32_t>(c_rowbase[pass] & 3);
        }

        for (int s = 0; s < ns; ++s) {
            const int slot = s % S;
            if (*abort_flag) break;
            if (!mbar_wait(&full[slot], (s / S) & 1)) {
                fail();
                break;
            }
            QN_TL(3, threadIdx.x == 32 && s == 0);
            QN_TL(4, threadIdx.x == 32 && s == ns - 1);
            const int col = col_lo + s;
            const uint32_t sl = s_ring + slot * p.slot_bytes;
            // block constants c'_b = fma(e4m3(q_b), sigma_g, mu) of this lane's rows, block kg
            float cmine[(MW + 1) / 2];
#pragma unroll
            for (int pass = 0; pass < (MW + 1) / 2; ++pass) {
                float c = 0.0f;
                const int i = c_row[pass];
                if (i >= 0 && 4 * col + kg < p.nbr) {
                    const uint32_t qw = lds32(sl + p.q_off + i * 8 + (((c_qoff[pass] + kg) >> 2) << 2));
                    const uint32_t qb = (qw >> (8 * ((c_qoff[pass] + kg) & 3))) & 0xffu;
                    const int64_t e = c_rowbase[pass] + 4 * col;
                    const bool same = ((e + kg) >> 8) == (e >> 8);
                    const float sg = __uint_as_float(lds32(sl + p.s_off + i * 8 + (same ? 0 : 4)));
                    c = block_constant(static_cast<uint8_t>(qb), sg, mu);
                }
                cmine[pass] = c;
            }
            const uint32_t xb = sl + p.x_off + kg * MP * 128;
            uint4 x0[NG], x1[NG];
#pragma unroll
            for (int tg = 0; tg < NG; ++tg) {
                x0[tg] = lds128(xb + xr[tg] + xc0[tg]);
                x1[tg] = lds128(xb + xr[tg] + xc1[tg]);
            }
#pragma unroll
            for (int i = 0; i < MW; ++i) {
                const int mt = rg + 4 * i;
                // constants of m-tile i: rows g and g + 8, held by quad lanes 2 (i & 1) and 2 (i & 1) + 1
                const float cA = __shfl_sync(0xffffffffu, cmine[i >> 1], (lane & ~3) | (2 * (i & 1)));
                const float cB = __shfl_sync(0xffffffffu, cmine[i >> 1], (lane & ~3) | (2 * (i & 1) + 1));
                if (mt < p.m) {
                    const uint32_t cr = sl + static_cast<uint32_t>(16 * mt + g) * 128u + kg * 32 + 8 * t;
                    const uint2 ca = lds64(cr), cb = lds64(cr + 8 * 128);
                    uint32_t af[4][4];
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk) {
                        const uint32_t wa = kk < 2 ? ca.x : ca.y, wb = kk < 2 ? cb.x : cb.y;
                        const int i0 = (2 * kk) & 3;
                        af[kk][0] = lut_pair<kFixedBase>(lut_base, wa, lane_op, i0);
                        af[kk][2] = lut_pair<kFixedBase>(lut_base, wa, lane_op, i0 + 1);
                        af[kk][1] = lut_pair<kFixedBase>(lut_base, wb, lane_op, i0);
                        af[kk][3] = lut_pair<kFixedBase>(lut_base, wb, lane_op, i0 + 1);
                    }
#pragma unroll
                    for (int tg = 0; tg < NG; ++tg) {
                        float d[4];
                        mma_16816_z(d, af[0][0], af[0][1], af[0][2], af[0][3], x0[tg].x, x0[tg].y);
                        mma_16816(d, af[1][0], af[1][1], af[1][2], af[1][3], x0[tg].z, x0[tg].w);
                        mma_16816(d, af[2][0], af[2][1], af[2][2], af[2][3], x1[tg].x, x1[tg].y);
                        mma_16816(d, af[3][0], af[3][1], af[3][2], af[3][3], x1[tg].z, x1[tg].w);
                        acc[i][tg][0] = __fmaf_rn(cA, d[0], acc[i][tg][0]);
                        acc[i][tg][1] = __fmaf_rn(cA, d[1], acc[i][tg][1]);
                        acc[i][tg][2] = __fmaf_rn(cB, d[2], acc[i][tg][2]);
                        acc[i][tg][3] = __fmaf_rn(cB, d[3], acc[i][tg][3]);
                    }
                }
            }
            // adapter down-projection jobs: n-tile nt_job, k16 steps kq0 + kq_step * j of the stage
            for (int j = 0; j < NT; ++j) {
                const int kq = kq0 + kq_step * j;
                const int blk = kq >> 2, q4 = kq & 3;
                const uint32_t xa = sl + p.x_off + blk * MP * 128;
                const uint32_t aa = sl + p.a_off + blk * p.rpad * 128;
                const uint32_t c0 = static_cast<uint32_t>(((2 * q4) ^ g) << 4) + 4 * t;
                const uint32_t c1 = static_cast<uint32_t>(((2 * q4 + 1) ^ g) << 4) + 4 * t;
                const uint32_t a0 = lds32(xa + g * 128 + c0), a2 = lds32(xa + g * 128 + c1);
                uint32_t a1 = 0u, a3 = 0u;
                if (NG > 1) {
                    a1 = lds32(xa + (g + 8) * 128 + c0);
                    a3 = lds32(xa + (g + 8) * 128 + c1);
                }
                const uint32_t jc0 = static_cast<uint32_t>(((2 * q4) ^ (jrow & 7)) << 4) + 4 * t;
                const uint32_t jc1 = static_cast<uint32_t>(((2 * q4 + 1) ^ (jrow & 7)) << 4) + 4 * t;
                const uint32_t b0 = lds32(aa + jrow * 128 + jc0), b1 = lds32(aa + jrow * 128 + jc1);
                mma_16816(tacc, a0, a1, a2, a3, b0, b1);
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[slot]);
        }
    }

    // ---------------------------------------------------------------------- reduction
    // The ring is idle from here on (every stage was consumed, the producer drained its loads):
    // its space holds the exchange buffers.
    QN_TL(5, threadIdx.x == 32);
    __syncthreads();
    QN_TL(6, threadIdx.x == 0);
    const uint32_t post = s_base + p.post_off;
    const uint32_t tbuf = post;                                  // [16 warps][32 lanes][4] f32
    const uint32_t tb = post + kConsumers * 32 * 16;             // [MP tokens][rk16] bf16 (s t_c)
    const int rk16 = (p.rpad + 15) & ~15;
    const uint32_t red = tb + ((MP * rk16 * 2 + 255) & ~255);    // [3][16 m-tiles][32 lanes][NG*4] f32
    if (warp > 0 && p.r > 0) {
        const uint32_t o = tbuf + static_cast<uint32_t>(cw * 32 + lane) * 16;
        asm volatile("st.shared.v4.f32 [%0], {%1,%2,%3,%4};" ::"r"(o), "f"(tacc[0]), "f"(tacc[1]), "f"(tacc[2]),
                     "f"(tacc[3])
                     : "memory");
    }
    if (warp > 0 && kg > 0) {
#pragma unroll
        for (int i = 0; i < MW; ++i) {
            const int mt = rg + 4 * i;
            if (mt < p.m) {
#pragma unroll
                for (int tg = 0; tg < NG; ++tg) {
                    const uint32_t o = red + static_cast<uint32_t>((((kg - 1) * kMaxM + mt) * 32 + lane) * NG + tg) * 16;
                    asm volatile("st.shared.v4.f32 [%0], {%1,%2,%3,%4};" ::"r"(o), "f"(acc[i][tg][0]),
                                 "f"(acc[i][tg][1]), "f"(acc[i][tg][2]), "f"(acc[i][tg][3])
                                 : "memory");
                }
            }
        }
    }
    __syncthreads();
    // t_c of n-tile cw (cw < NT): the warps cw, cw + NT, ... in that order; s t_c to bf16
    if (warp > 0 && cw < NT) {
        float tt[4] = {0.0f, 0.0f, 0.0f, 0.0f};
        for (int w = cw; w < kConsumers; w += NT) {
            const uint4 v = lds128(tbuf + static_cast<uint32_t>(w * 32 + lane) * 16);
            tt[0] += __uint_as_float(v.x);
            tt[1] += __uint_as_float(v.y);
            tt[2] += __uint_as_float(v.z);
            tt[3] += __uint_as_float(v.w);
        }
        // fragment: tokens g / g + 8, ranks 8 cw + 2 t (+1)
        const int j = 8 * cw + 2 * t;
        const uint32_t v0 = pack_bf16x2(p.s * tt[0], p.s * tt[1]);
        const uint32_t v1 = pack_bf16x2(p.s * tt[2], p.s * tt[3]);
        asm volatile("st.shared.b32 [%0], %1;" ::"r"(tb + static_cast<uint32_t>(g * rk16 + j) * 2), "r"(v0) : "memory");
        if (NG > 1)
            asm volatile("st.shared.b32 [%0], %1;" ::"r"(tb + static_cast<uint32_t>((g + 8) * rk16 + j) * 2), "r"(v1)
                         : "memory");
    }
    // ranks beyond rpad (up to the k16 boundary) read as zero
    if (p.r > 0 && rk16 > p.rpad) {
        for (int i = threadIdx.x; i < MP * (rk16 - p.rpad) / 2; i += kThreads) {
            const int tok = i / ((rk16 - p.rpad) / 2), jj = p.rpad + 2 * (i % ((rk16 - p.rpad) / 2));
            asm volatile("st.shared.b32 [%0], %1;" ::"r"(tb + static_cast<uint32_t>(tok * rk16 + jj) * 2), "r"(0u)
                         : "memory");
        }
    }
    __syncthreads();

    const int nrmax = (p.R + C - 1) / C;
    float *recv = reinterpret_cast<float *>(smem + p.recv_off);
    if (warp > 0 && kg == 0) {
        // sum the four block-warps of each m-tile (kg = 0, 1, 2, 3 in order), add B (s t_c)
#pragma unroll
        for (int i = 0; i < MW; ++i) {
            const int mt = rg + 4 * i;
            if (mt >= p.m) continue;
#pragma unroll
            for (int q = 0; q < 3; ++q) {
#pragma unroll
                for (int tg = 0; tg < NG; ++tg) {
                    const uint4 v = lds128(red + static_cast<uint32_t>(((q * kMaxM + mt) * 32 + lane) * NG + tg) * 16);
                    acc[i][tg][0] += __uint_as_float(v.x);
                    acc[i][tg][1] += __uint_as_float(v.y);
                    acc[i][tg][2] += __uint_as_float(v.z);
                    acc[i][tg][3] += __uint_as_float(v.w);
                }
            }
            const int64_t rA = row0 + 16 * mt + g, rB = rA + 8;
            const bool vA = rA < p.n, vB = rB < p.n;
            for (int kc = 0; kc < rk16 / 16 && p.r > 0; ++kc) {
                const int j = 16 * kc + 2 * t;
                const uint32_t a0 = load_pair_rowmajor(p.B, rA, vA, j, p.r);
                const uint32_t a1 = load_pair_rowmajor(p.B, rB, vB, j, p.r);
                const uint32_t a2 = load_pair_rowmajor(p.B, rA, vA, j + 8, p.r);
                const uint32_t a3 = load_pair_rowmajor(p.B, rB, vB, j + 8, p.r);
#pragma unroll
                for (int tg = 0; tg < NG; ++tg) {
                    const uint32_t tr = tb + static_cast<uint32_t>((tg * 8 + g) * rk16 + j) * 2;
                    mma_16816(acc[i][tg], a0, a1, a2, a3, lds32(tr), lds32(tr + 16));
                }
            }
            if (C == 1) {
                if (!*abort_flag) {
#pragma unroll
                    for (int tg = 0; tg < NG; ++tg) {
                        const int tok = tg * 8 + 2 * t;
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const int64_t row = (e < 2) ? rA : rB;
                            const int tk = tok + (e & 1);
                            if (row < p.n && tk < p.M)
                                p.h[static_cast<int64_t>(tk) * p.n + row] =
                                    __bfloat16_as_ushort(__float2bfloat16_rn(acc[i][tg][e]));
                        }
                    }
                }
            }
        }
    }
    if (C > 1) {
        cluster_wait();  // phase 1: every CTA of the cluster runs
        if (warp > 0 && kg == 0) {
            cg::cluster_group cluster = cg::this_cluster();
#pragma unroll
            for (int i = 0; i < MW; ++i) {
                const int mt = rg + 4 * i;
                if (mt >= p.m) continue;
#pragma unroll
                for (int hh = 0; hh < 2; ++hh) {
                    const int rl = 16 * mt + g + 8 * hh;
                    const int owner = (rl * C + C - 1) / p.R;
                    const int rr = rl - p.R * owner / C;
                    float *dst = cluster.map_shared_rank(recv, owner) + (crank * nrmax + rr) * MP + 2 * t;
#pragma unroll
                    for (int tg = 0; tg < NG; ++tg)
                        *reinterpret_cast<float2 *>(dst + tg * 8) = make_float2(acc[i][tg][2 * hh], acc[i][tg][2 * hh + 1]);
                }
            }
        }
        cluster_arrive_release();
        cluster_wait_acquire();  // phase 2: every partial has landed
        // rows [R crank / C, R (crank + 1) / C) of the chunk
        const int r_lo = p.R * crank / C, r_hi = p.R * (crank + 1) / C, nr = r_hi - r_lo;
        if (!*abort_flag) {
            for (int it = threadIdx.x; it < nr * p.M; it += kThreads) {
                const int rr = it % nr, tok = it / nr;
                const int64_t row = row0 + r_lo + rr;
                if (row >= p.n) continue;
                float sum = 0.0f;
                for (int src = 0; src < C; ++src) sum += recv[(src * nrmax + rr) * MP + tok];
                p.h[static_cast<int64_t>(tok) * p.n + row] = __bfloat16_as_ushort(__float2bfloat16_rn(sum));
            }
        }
    }
    QN_TL(7, threadIdx.x == 0);
}

template <int NG>
__global__ void __launch_bounds__(kThreads, 1)
k_decode_fwd(const __grid_constant__ CUtensorMap tm_codes, const FwdArgs p) {
    extern __shared__ __align__(1024) uint8_t smem[];
    if ((saddr(smem) & 0x00ffffffu) == kDynSmemBase)
        fwd_body<NG, true>(&tm_codes, p, smem);
    else
        fwd_body<NG, false>(&tm_codes, p, smem);
}

// ---------------------------------------------------------------------------- host side

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = [] {
        PFN_cuTensorMapEncodeTiled_v12000 f = nullptr;
        cudaDriverEntryPointQueryResult qres;
        void *ptr = nullptr;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &qres) == cudaSuccess &&
            qres == cudaDriverEntryPointSuccess)
            f = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
        (void)cudaGetLastError();
        return f;
    }();
    return fn;
}

bool encode_2d(CUtensorMap *m, CUtensorMapDataType dt, int esize, const void *base, uint64_t cols, uint64_t rows,
               uint32_t box_cols, uint32_t box_rows, CUtensorMapSwizzle sw) {
    auto fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[2] = {cols, rows};
    cuuint64_t strides[1] = {cols * static_cast<uint64_t>(esize)};
    cuuint32_t box[2] = {box_cols, box_rows};
    cuuint32_t estr[2] = {1, 1};
    return fn(m, dt, 2, const_cast<void *>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int round_rank(int r) { return r <= 0 ? 0 : r <= 8 ? 8 : r <= 16 ? 16 : r <= 32 ? 32 : 64; }

// Shared-memory layout of one launch shape; false if it does not fit with at least two stages.
bool layout(FwdArgs &a, int MP) {
    const uint32_t codes = static_cast<uint32_t>(a.R) * 128u;
    const uint32_t xb = kStageBlocks * MP * 128u;
    const uint32_t ab = kStageBlocks * a.rpad * 128u;
    const uint32_t qb = static_cast<uint32_t>(a.R) * 8u;  // q windows of the chunk rows
    const uint32_t sb = static_cast<uint32_t>(a.R) * 8u;  // group scales of the chunk rows
    a.x_off = codes;
    a.a_off = codes + xb;
    a.q_off = codes + xb + ab;
    a.s_off = a.q_off + qb;
    a.slot_bytes = (a.s_off + sb + 1023u) & ~1023u;
    a.tx_bytes = codes;
    const int rk16 = (a.rpad + 15) & ~15;
    const uint32_t post = kConsumers * 32 * 16 + ((MP * rk16 * 2 + 255) & ~255) + 3 * kMaxM * 32 * 16 * (MP / 8);
    const uint32_t recv = a.C > 1 ? (static_cast<uint32_t>(a.C * ((a.R + a.C - 1) / a.C) * MP * 4) + 1023u) & ~1023u : 0u;
    a.ring_off = kLutBytes;
    const uint32_t fixed = kLutBytes + recv + 1024;  // + barriers and flag
    if (fixed >= kSmemLimit) return false;
    int stages = static_cast<int>((kSmemLimit - fixed) / a.slot_bytes);
    if (stages > kMaxStages) stages = kMaxStages;
    if (stages < 2) return false;
    const uint32_t ring = static_cast<uint32_t>(stages) * a.slot_bytes;
    if (ring < post) {
        // the exchange buffers outgrow the ring: give them room of their own
        if (fixed + ring + post > kSmemLimit) {
            stages = static_cast<int>((kSmemLimit - fixed - post) / a.slot_bytes);
            if (stages < 2) return false;
        }
    }
    a.stages = stages;
    const uint32_t ring_bytes = static_cast<uint32_t>(a.stages) * a.slot_bytes;
    a.post_off = a.ring_off + (ring_bytes >= post ? 0u : ring_bytes);
    const uint32_t after = a.ring_off + (ring_bytes >= post ? ring_bytes : ring_bytes + post);
    a.recv_off = after;
    a.bar_off = after + recv;
    return true;
}

size_t smem_bytes(const FwdArgs &a) { return static_cast<size_t>(a.bar_off) + 2 * kMaxStages * 8 + 16; }

template <int NG>
cudaError_t launch_ng(const WeightView &w, const uint16_t *x, int M, const uint16_t *A, const uint16_t *B, int r,
                      float s, uint16_t *h, int *err, cudaStream_t st) {
    constexpr int MP = 8 * NG;
    const void *kern = reinterpret_cast<const void *>(k_decode_fwd<NG>);
    int sms = 148;
    cudaError_t e = device_sm_count(&sms);
    if (e != cudaSuccess) return e;

    FwdArgs a = {};
    a.q = w.q;
    a.sigma = w.sigma;
    a.mu = w.mu;
    a.B = B;
    a.x = x;
    a.A = A;
    a.h = h;
    a.err = err;
    a.n = w.n;
    a.k = w.k;
    a.nbr = static_cast<int>(w.k / kBlock);
    a.ncol = (a.nbr + kStageBlocks - 1) / kStageBlocks;
    a.M = M;
    a.r = r;
    a.rpad = round_rank(r);
    a.s = s;

    // Launch shape: R = 16 m rows per chunk and C K-slices per cluster with chunks x C <= SMs
    // and every cluster resident at once; per-CTA work is R x ceil(ncol / C) stage columns: take
    // the shape with the least of it (ties: smaller clusters, then shorter chunks).
    double best_work = 0.0;
    FwdArgs best = a;
    bool found = false;
    // m is a multiple of 4 (every consumer warp holds the same number of m-tiles) unless the
    // weight has fewer than 64 rows
    const int m_max = 16 / NG;  // four m-tile rows of warps, 4 / NG m-tiles each
    const int m_min = w.n < 64 ? static_cast<int>((w.n + 15) / 16) : 4;
    const int m_step = w.n < 64 ? 1 : 4;
    for (int C = 1; C <= kMaxCluster && C <= a.ncol; ++C) {
        for (int m = m_min; m <= m_max; m += m_step) {
            FwdArgs c = a;
            c.m = m;
            c.R = 16 * m;
            c.C = C;
            const int64_t chunks = (w.n + c.R - 1) / c.R;
            if (chunks * C > sms || chunks > 65535) continue;
            const double work = static_cast<double>(c.R) * ((a.ncol + C - 1) / C);
            if (found && work >= best_work * (1.0 - 1e-9)) continue;
            if (!layout(c, MP)) continue;
            if (C > 1) {
                int nc = 0;
                e = resident_clusters(kern, kThreads, C, smem_bytes(c), &nc);
                if (e != cudaSuccess) return e;
                if (nc < chunks) continue;
            }
            best = c;
            best_work = work;
            found = true;
        }
    }
    if (!found) {
        // more rows than one wave of the tallest chunks holds: several waves, no split
        best.m = m_max;
        best.R = 16 * m_max;
        best.C = 1;
        while (!layout(best, MP)) {
            if (best.m == 1) return cudaErrorInvalidConfiguration;
            best.m -= 1;
            best.R = 16 * best.m;
        }
    }
    a = best;
    const size_t smem = smem_bytes(a);

    CUtensorMap tm_codes;
    if (!encode_2d(&tm_codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, w.codes, static_cast<uint64_t>(w.k / 2),
                   static_cast<uint64_t>(w.n), 128, static_cast<uint32_t>(a.R), CU_TENSOR_MAP_SWIZZLE_NONE))
        return cudaErrorInvalidValue;
    e = ensure_smem_limit(kern, smem);
    if (e != cudaSuccess) return e;

    const int64_t chunks = (w.n + a.R - 1) / a.R;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(a.C), static_cast<unsigned>(chunks), 1);
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    attr[1].id = cudaLaunchAttributeClusterDimension;
    attr[1].val.clusterDim.x = a.C;
    attr[1].val.clusterDim.y = 1;
    attr[1].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = a.C > 1 ? 2 : 1;
    e = cudaLaunchKernelEx(&cfg, k_decode_fwd<NG>, tm_codes, a);
    count_launch();
    return e;
}

}  // namespace

cudaError_t launch_decode_fwd(const WeightView &w, const uint16_t *x, int M, const uint16_t *A, const uint16_t *B,
                              int r, float s, uint16_t *h, int *err, cudaStream_t st) {
    if (M <= 0 || w.n == 0) return cudaSuccess;
    if (M > kDecodeTokens || r > kDecodeMaxRank) return cudaErrorInvalidValue;
    if (M <= 8) return launch_ng<1>(w, x, M, A, B, r, s, h, err, st);
    return launch_ng<2>(w, x, M, A, B, r, s, h, err, st);
}

#ifdef QN_TIMELINE
extern "C" int qn_debug_fwd_timeline(unsigned long long *out, int n) {
    return cudaMemcpyFromSymbol(out, g_fwd_timeline, sizeof(unsigned long long) * 8 * (n < 1024 ? n : 1024)) ==
                   cudaSuccess
               ? 0
               : 1;
}
#endif

}  // namespace qn
