// decode_bwd2.cu -- QLoRA input gradient for few tokens (M <= 16 per launch) on sm_100a.
//
//   grad_x[m,k] = sum_n grad_h[m,n] W'[n,k] + s sum_j A[j,k] u[m,j],  u[m,j] = sum_n grad_h[m,n] B[n,j]
// ("How does QLoRA work for training?", aivaro.ru, section 7: the frozen base is dequantised on
// the fly for the gradient and not updated.)
//
// The reduction runs over weight rows n, whose block constants differ, so each block constant
// scales the bf16 token operand (c'_{n,b} grad_h[m,n]) instead of the product. A tensor-core tile
// (mma.sync m16n8k16) takes 16 features as its M rows and 16 weight rows as its K: the nibbles
// of two neighbouring weight rows are interleaved so that a byte again indexes a pair of the
// bf16-pair table (stream_common.cuh), and the 16 features of sub-tile f are chosen as the two
// nibbles of byte 4 g + f of each row segment, so a lane reads one 4-byte word per weight row.
//
// Work split. One CTA per SM. A CTA owns a 256-feature column chunk (4 blocks, one 128-byte TMA
// box column) over a slice of the weight rows; the C row slices of a chunk form a thread-block
// cluster. The CTA streams its rows through a ring of 64-row stages: the codes box, the stage's
// grad_h columns (swizzled), the stage's rows of B and the inputs of its block constants.
//   warp 0      : producer (codes by TMA, the rest by cp.async; all complete on the stage's full
//                 barrier).
//   warps 1..16 : consumers. Warp (kg, rg) takes block kg (64 features) and rows 16 rg .. + 16 of
//                 every stage; its accumulators hold the CTA's partial sums for those 64 features.
//                 Lanes compute the block constants of the warp's 16 rows and share them by
//                 shuffles. A share of the adapter term u_c = grad_h B over the stage's rows runs
//                 on the tensor cores too (B fragments by ldmatrix.trans).
// After the loop the four row-warps of each block are summed in a fixed order, the slice's
// adapter term A^T (s u_c) is added, and the partial sums are pushed with DSMEM stores into the
// CTA of the cluster that finalises those features; one cluster barrier later that CTA sums the
// slices in rank order and stores grad_x. Results are bit-reproducible.
// Nothing is read from global memory before the programmatic-launch wait; every mbarrier wait is
// bounded and a timeout is recorded in the workspace error word.
#include <cudaTypedefs.h>

#include "host_cache.h"
#include "stream_common.cuh"

namespace qn {

namespace {

using namespace sm100;
using namespace stream;

constexpr int kConsumers = 16;
constexpr int kThreads = 32 * (kConsumers + 1);
constexpr int kRowsPerStage = 64;
constexpr int kChunkFeat = 256;
constexpr int kMaxStages = 8;
constexpr int kMaxCluster = 8;
constexpr size_t kSmemLimit = 227 * 1024;

struct BwdArgs {
    const uint8_t *q;
    const float *sigma;
    const float *mu;
    const uint16_t *gh;  // M x n
    const uint16_t *A;   // r x k
    const uint16_t *B;   // n x r
    uint16_t *gx;        // M x k
    int *err;
    int64_t n, k;
    int nbr;   // blocks per row
    int nrs;   // row stages (ceil(n / 64))
    int M, r, rpad, rb;  // rpad: r rounded up to 8/16/32/64; rb: bytes per padded B row in smem
    float s;
    int C, stages;
    uint32_t slot_bytes, g_off, b_off, q_off, s_off;
    uint32_t ring_off, recv_off, bar_off, post_off;
    uint32_t tx_bytes;
};

__device__ __forceinline__ void ldm_x4_trans(uint32_t a, uint32_t &r0, uint32_t &r1, uint32_t &r2, uint32_t &r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(a));
}

// grad_h pair (rows 2 t, 2 t + 1 of 16 at column offset `row16`) of token `tok` in the stage's
// swizzled [token][64 rows] tile: 16-byte chunk c of token row tok sits at c ^ (tok & 7).
__device__ __forceinline__ uint32_t gh_pair(uint32_t gbase, int tok, int row) {
    const int c = row >> 3, w = (row & 7) >> 1;
    return lds32(gbase + static_cast<uint32_t>(tok * 128 + ((c ^ (tok & 7)) << 4) + w * 4));
}

template <int NG, bool kFixedBase>
__device__ __forceinline__ void bwd_body(const CUtensorMap *tm_codes, const BwdArgs &p, uint8_t *smem) {
    constexpr int MP = 8 * NG;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, t = lane & 3;
    const int C = p.C;
    const int crank = C > 1 ? static_cast<int>(cg::this_cluster().block_rank()) : 0;
    const int chunk = blockIdx.y;
    const int col = chunk;  // 128-byte code column = 4 blocks = 256 features
    const int64_t f0 = static_cast<int64_t>(chunk) * kChunkFeat;
    const int rs_lo = p.nrs * crank / C, rs_hi = p.nrs * (crank + 1) / C;
    const int ns = rs_hi - rs_lo;
    const int S = p.stages;

    uint8_t *lut = smem;
    const uint32_t s_base = saddr(smem);
    const uint32_t s_ring = s_base + p.ring_off;
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + p.bar_off);
    uint64_t *empty = full + kMaxStages;
    volatile uint32_t *abort_flag = reinterpret_cast<volatile uint32_t *>(empty + kMaxStages);

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
    // token rows M .. MP-1 of grad_h and the padding columns of the B rows are read but never
    // copied: zero every slot's tiles once
    for (int sidx = 0; sidx < S; ++sidx) {
        const uint32_t sl = s_ring + sidx * p.slot_bytes;
        for (int i = threadIdx.x; i < (MP - p.M) * 32; i += kThreads)
            asm volatile("st.shared.b32 [%0], %1;" ::"r"(sl + p.g_off + (p.M + i / 32) * 128 + (i % 32) * 4), "r"(0u)
                         : "memory");
        if (p.r > 0)
            for (int i = threadIdx.x; i < kRowsPerStage * (p.rb / 4); i += kThreads)
                asm volatile("st.shared.b32 [%0], %1;" ::"r"(sl + p.b_off + i * 4), "r"(0u) : "memory");
    }
    __syncthreads();
    if (C > 1) cluster_arrive_relaxed();  // phase 1: this CTA runs
    grid_dependents_launch();
    grid_dependency_wait();  // grad_h, A and B may come from the preceding kernel

    auto fail = [&]() {
        if (atomicExch(const_cast<uint32_t *>(abort_flag), 1u) == 0u) record_error(p.err, kErrTimeout);
    };

    const int cw = warp - 1;
    const int kg = cw & 3, rg = cw >> 2;
    const int NT = p.rpad / 8;
    float acc[4][NG][4];  // sub-tile f, token group, fragment
#pragma unroll
    for (int f = 0; f < 4; ++f)
#pragma unroll
        for (int tg = 0; tg < NG; ++tg) acc[f][tg][0] = acc[f][tg][1] = acc[f][tg][2] = acc[f][tg][3] = 0.0f;
    float uacc[2][4] = {{0.0f, 0.0f, 0.0f, 0.0f}, {0.0f, 0.0f, 0.0f, 0.0f}};

    if (warp == 0) {
        // ------------------------------------------------------------------ producer
        const int64_t nb = p.n * p.nbr;
        const int64_t ng = (nb + kGroup - 1) / kGroup;
        int ni = 0;
        for (int s = 0; s < ns; ++s) {
            const int slot = s % S;
            if (*abort_flag) break;
            if (s >= S && !mbar_wait(&empty[slot], ((s / S) & 1) ^ 1)) {
                fail();
                break;
            }
            const int rs = rs_lo + s;
            const int64_t n0 = static_cast<int64_t>(rs) * kRowsPerStage;
            const uint32_t sl = s_ring + slot * p.slot_bytes;
            if (lane == 0) {
                mbar_expect_tx(&full[slot], p.tx_bytes);
                tma_load_2d_saddr(sl, tm_codes, &full[slot], col * 128, static_cast<int32_t>(n0));
            }
            // grad_h[tok][n0 .. n0 + 64): 8 chunks of 16 bytes per token, lanes over (token, chunk)
            const bool rows16 = (p.n & 7) == 0;
            for (int i = lane; i < p.M * 8; i += 32) {
                const int tok = i >> 3, c = i & 7;
                const int64_t nn = n0 + 8 * c;
                const uint32_t dst = sl + p.g_off + static_cast<uint32_t>(tok * 128 + ((c ^ (tok & 7)) << 4));
                if (rows16) {
                    const int64_t left = p.n - nn;
                    cp_async16_zfill(dst, left > 0 ? p.gh + tok * p.n + nn : p.gh,
                                     left >= 8 ? 16u : (left > 0 ? static_cast<uint32_t>(2 * left) : 0u));
                } else {
                    // rows not 16-byte aligned: 4-byte pieces (n even) or element loads
                    for (int e = 0; e < 8; e += 2) {
                        uint32_t v = 0u;
                        if (nn + e < p.n) v = ld_ro_u16(p.gh + tok * p.n + nn + e);
                        if (nn + e + 1 < p.n) v |= static_cast<uint32_t>(ld_ro_u16(p.gh + tok * p.n + nn + e + 1)) << 16;
                        asm volatile("st.shared.b32 [%0], %1;" ::"r"(dst + e * 2), "r"(v) : "memory");
                    }
                }
            }
            // B rows n0 .. n0 + 64 (r ranks each) into [row][rb bytes]
            if (p.r > 0) {
                const int cpr = (p.r * 2 + 15) / 16;  // 16-byte chunks per row
                const bool r8 = (p.r & 7) == 0;
                for (int i = lane; i < kRowsPerStage * cpr; i += 32) {
                    const int row = i / cpr, c = i % cpr;
                    const int64_t nn = n0 + row;
                    const uint32_t dst = sl + p.b_off + static_cast<uint32_t>(row * p.rb + c * 16);
                    if (r8) {
                        cp_async16_zfill(dst, nn < p.n ? p.B + nn * p.r + 8 * c : p.B, nn < p.n ? 16u : 0u);
                    } else {
                        for (int e = 0; e < 8; e += 2) {
                            const int j = 8 * c + e;
                            uint32_t v = 0u;
                            if (nn < p.n && j < p.r) v = ld_ro_u16(p.B + nn * p.r + j);
                            if (nn < p.n && j + 1 < p.r) v |= static_cast<uint32_t>(ld_ro_u16(p.B + nn * p.r + j + 1)) << 16;
                            asm volatile("st.shared.b32 [%0], %1;" ::"r"(dst + e * 2), "r"(v) : "memory");
                        }
                    }
                }
            }
            // block-constant inputs of the stage's 64 rows: q window and group scales
            for (int j = 0; j < 2; ++j) {
                const int i = lane + 32 * j;
                const int64_t row = n0 + i;
                if (row < p.n) {
                    const int64_t e0 = row * p.nbr + 4 * col;
                    const int64_t e3 = e0 + 3 < nb ? e0 + 3 : nb - 1;
                    const int64_t w0 = e0 & ~int64_t(3), w1 = w0 + 4;
                    const uint32_t qd = sl + p.q_off + static_cast<uint32_t>(i) * 8u;
                    const uint32_t sd = sl + p.s_off + static_cast<uint32_t>(i) * 8u;
                    cp_async4_zfill(qd, p.q + w0, 4);
                    const int64_t rest = nb - w1;
                    cp_async4_zfill(qd + 4, p.q + (rest > 0 ? w1 : w0),
                                    rest >= 4 ? 4u : (rest > 0 ? static_cast<uint32_t>(rest) : 0u));
                    cp_async4_zfill(sd, p.sigma + (e0 >> 8), 4);
                    cp_async4_zfill(sd + 4, p.sigma + ((e3 >> 8) < ng ? (e3 >> 8) : ng - 1), 4);
                }
            }
            cp_async_arrive_noinc(&full[slot]);
            ni = s + 1;
        }
        cp_async_wait_all();
        if (lane == 0)
            for (int s = (ni > S ? ni - S : 0); s < ni; ++s) mbar_wait(&full[s % S], (s / S) & 1);
        __syncwarp();
    } else {
        // ------------------------------------------------------------------ consumers
        const uint32_t lane_op = lut_lane_operand<kFixedBase>(lut, lane);
        const uint32_t lut_base = s_base;
        const float mu = __ldg(p.mu);
        // the block constant this lane computes: row g + 8 (t & 1) of the warp's 16 rows, block kg
        const int my_row = 16 * rg + g + 8 * (t & 1);
        // source lanes of rows 2t, 2t+1, 2t+8, 2t+9 (row rho is computed by lane 4 (rho & 7) + (rho >> 3))
        const int src0 = 4 * ((2 * t) & 7) + 0, src1 = 4 * ((2 * t + 1) & 7) + 0;
        const int src8 = 4 * ((2 * t) & 7) + 1, src9 = 4 * ((2 * t + 1) & 7) + 1;
        const int nu_jobs = 4 * NT;  // (k16 step, rank tile) jobs of the adapter term per stage
        for (int s = 0; s < ns; ++s) {
            const int slot = s % S;
            if (*abort_flag) break;
            if (!mbar_wait(&full[slot], (s / S) & 1)) {
                fail();
                break;
            }
            const int rs = rs_lo + s;
            const int64_t n0 = static_cast<int64_t>(rs) * kRowsPerStage;
            const uint32_t sl = s_ring + slot * p.slot_bytes;
            // block constant of (row my_row, block kg)
            float cmine = 0.0f;
            {
                const int64_t row = n0 + my_row;
                if (row < p.n && 4 * col + kg < p.nbr) {
                    const int64_t e0 = row * p.nbr + 4 * col;
                    const uint32_t qo = static_cast<uint32_t>(e0 & 3) + kg;
                    const uint32_t qw = lds32(sl + p.q_off + my_row * 8 + ((qo >> 2) << 2));
                    const uint32_t qb = (qw >> (8 * (qo & 3))) & 0xffu;
                    const bool same = ((e0 + kg) >> 8) == (e0 >> 8);
                    const float sg = __uint_as_float(lds32(sl + p.s_off + my_row * 8 + (same ? 0 : 4)));
                    cmine = block_constant(static_cast<uint8_t>(qb), sg, mu);
                }
            }
            const float c0 = __shfl_sync(0xffffffffu, cmine, src0), c1 = __shfl_sync(0xffffffffu, cmine, src1);
            const float c8 = __shfl_sync(0xffffffffu, cmine, src8), c9 = __shfl_sync(0xffffffffu, cmine, src9);
            // token operand: grad_h of rows 2t, 2t+1 (b0) and 2t+8, 2t+9 (b1) of this warp's 16 rows,
            // scaled by their block constants
            const uint32_t gb = sl + p.g_off;
            uint32_t bop[NG][2];
#pragma unroll
            for (int tg = 0; tg < NG; ++tg) {
                const int tok = tg * 8 + g;
                const uint32_t v01 = gh_pair(gb, tok, 16 * rg + 2 * t);
                const uint32_t v89 = gh_pair(gb, tok, 16 * rg + 2 * t + 8);
                bop[tg][0] = pack_bf16x2(c0 * bf16_lo(v01), c1 * bf16_hi(v01));
                bop[tg][1] = pack_bf16x2(c8 * bf16_lo(v89), c9 * bf16_hi(v89));
            }
            // codes: byte 32 kg + 4 g .. + 4 of rows 2t, 2t+1, 2t+8, 2t+9
            const uint32_t cr = sl + static_cast<uint32_t>(16 * rg + 2 * t) * 128u + kg * 32 + 4 * g;
            const uint32_t w0 = lds32(cr), w1 = lds32(cr + 128), w8 = lds32(cr + 8 * 128), w9 = lds32(cr + 9 * 128);
            // interleave: byte f of ev holds (row a, even feature) | (row b, even feature) << 4
            const uint32_t ev01 = (w0 & 0x0f0f0f0fu) | ((w1 & 0x0f0f0f0fu) << 4);
            const uint32_t od01 = ((w0 >> 4) & 0x0f0f0f0fu) | (w1 & 0xf0f0f0f0u);
            const uint32_t ev89 = (w8 & 0x0f0f0f0fu) | ((w9 & 0x0f0f0f0fu) << 4);
            const uint32_t od89 = ((w8 >> 4) & 0x0f0f0f0fu) | (w9 & 0xf0f0f0f0u);
#pragma unroll
            for (int f = 0; f < 4; ++f) {
                const uint32_t a0 = lut_pair<kFixedBase>(lut_base, ev01, lane_op, f);
                const uint32_t a1 = lut_pair<kFixedBase>(lut_base, od01, lane_op, f);
                const uint32_t a2 = lut_pair<kFixedBase>(lut_base, ev89, lane_op, f);
                const uint32_t a3 = lut_pair<kFixedBase>(lut_base, od89, lane_op, f);
#pragma unroll
                for (int tg = 0; tg < NG; ++tg) mma_16816(acc[f][tg], a0, a1, a2, a3, bop[tg][0], bop[tg][1]);
            }
            // adapter: u_c[tok][j] += sum over the stage's rows of grad_h[tok][row] B[row][j]
            if (p.r > 0) {
#pragma unroll
                for (int jj = 0; jj < 2; ++jj) {
                    const int job = cw + 16 * jj;
                    if (job < nu_jobs) {
                        const int kq = job & 3, nt = job >> 2;
                        const uint32_t a0 = gh_pair(gb, g, 16 * kq + 2 * t);
                        const uint32_t a2 = gh_pair(gb, g, 16 * kq + 2 * t + 8);
                        uint32_t a1 = 0u, a3 = 0u;
                        if (NG > 1) {
                            a1 = gh_pair(gb, g + 8, 16 * kq + 2 * t);
                            a3 = gh_pair(gb, g + 8, 16 * kq + 2 * t + 8);
                        }
                        // B[16 kq .. + 16][8 nt .. + 8]: matrices (rows lo, rows hi) x (ranks 8 nt)
                        const int mi = lane >> 3, rr = lane & 7;
                        const uint32_t baddr =
                            sl + p.b_off + static_cast<uint32_t>((16 * kq + 8 * (mi & 1) + rr) * p.rb + 16 * nt);
                        uint32_t b0, b1, b2, b3;
                        ldm_x4_trans(baddr, b0, b1, b2, b3);  // matrices 2, 3 repeat 0, 1 (same addresses)
                        mma_16816(uacc[jj], a0, a1, a2, a3, b0, b1);
                    }
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[slot]);
        }
    }

    // ---------------------------------------------------------------------- reduction
    __syncthreads();
    const uint32_t post = s_base + p.post_off;
    const uint32_t ubuf = post;                                // [16 warps][2][32 lanes][4] f32
    const uint32_t sub = post + kConsumers * 2 * 32 * 16;      // [MP tokens][rk16] bf16: s u_c
    const int rk16 = (p.rpad + 15) & ~15;
    const uint32_t red = sub + ((MP * rk16 * 2 + 255) & ~255);  // [3][4 blocks][4 f][32 lanes][NG][4] f32
    if (warp > 0 && p.r > 0) {
#pragma unroll
        for (int jj = 0; jj < 2; ++jj) {
            const uint32_t o = ubuf + static_cast<uint32_t>(((cw * 2 + jj) * 32 + lane) * 16);
            asm volatile("st.shared.v4.f32 [%0], {%1,%2,%3,%4};" ::"r"(o), "f"(uacc[jj][0]), "f"(uacc[jj][1]),
                         "f"(uacc[jj][2]), "f"(uacc[jj][3])
                         : "memory");
        }
    }
    if (warp > 0 && rg > 0) {
#pragma unroll
        for (int f = 0; f < 4; ++f)
#pragma unroll
            for (int tg = 0; tg < NG; ++tg) {
                const uint32_t o = red + static_cast<uint32_t>(((((rg - 1) * 4 + kg) * 4 + f) * 32 + lane) * NG + tg) * 16;
                asm volatile("st.shared.v4.f32 [%0], {%1,%2,%3,%4};" ::"r"(o), "f"(acc[f][tg][0]), "f"(acc[f][tg][1]),
                             "f"(acc[f][tg][2]), "f"(acc[f][tg][3])
                             : "memory");
            }
    }
    __syncthreads();
    // u_c of rank tile nt: the jobs (kq = 0..3, nt) in order; job j lives in warp j % 16, slot j / 16
    if (warp > 0 && cw < NT) {
        const int nt = cw;
        float uu[4] = {0.0f, 0.0f, 0.0f, 0.0f};
        for (int kq = 0; kq < 4; ++kq) {
            const int job = 4 * nt + kq;
            const uint4 v = lds128(ubuf + static_cast<uint32_t>((((job % 16) * 2 + job / 16) * 32 + lane) * 16));
            uu[0] += __uint_as_float(v.x);
            uu[1] += __uint_as_float(v.y);
            uu[2] += __uint_as_float(v.z);
            uu[3] += __uint_as_float(v.w);
        }
        // fragment: tokens g / g + 8, ranks 8 nt + 2 t (+1)
        const int j = 8 * nt + 2 * t;
        asm volatile("st.shared.b32 [%0], %1;" ::"r"(sub + static_cast<uint32_t>(g * rk16 + j) * 2),
                     "r"(pack_bf16x2(p.s * uu[0], p.s * uu[1]))
                     : "memory");
        if (NG > 1)
            asm volatile("st.shared.b32 [%0], %1;" ::"r"(sub + static_cast<uint32_t>((g + 8) * rk16 + j) * 2),
                         "r"(pack_bf16x2(p.s * uu[2], p.s * uu[3]))
                         : "memory");
    }
    if (p.r > 0 && rk16 > p.rpad) {
        for (int i = threadIdx.x; i < MP * (rk16 - p.rpad) / 2; i += kThreads) {
            const int tok = i / ((rk16 - p.rpad) / 2), jj = p.rpad + 2 * (i % ((rk16 - p.rpad) / 2));
            asm volatile("st.shared.b32 [%0], %1;" ::"r"(sub + static_cast<uint32_t>(tok * rk16 + jj) * 2), "r"(0u)
                         : "memory");
        }
    }
    __syncthreads();

    // features of sub-tile f, fragment row g -> 64 kg + 8 g + 2 f, row g + 8 -> 64 kg + 8 g + 2 f + 1
    const int nrmax = (kChunkFeat + C - 1) / C;
    float *recv = reinterpret_cast<float *>(smem + p.recv_off);
    if (warp > 0 && rg == 0) {
#pragma unroll
        for (int q = 0; q < 3; ++q)
#pragma unroll
            for (int f = 0; f < 4; ++f)
#pragma unroll
                for (int tg = 0; tg < NG; ++tg) {
                    const uint4 v = lds128(red + static_cast<uint32_t>((((q * 4 + kg) * 4 + f) * 32 + lane) * NG + tg) * 16);
                    acc[f][tg][0] += __uint_as_float(v.x);
                    acc[f][tg][1] += __uint_as_float(v.y);
                    acc[f][tg][2] += __uint_as_float(v.z);
                    acc[f][tg][3] += __uint_as_float(v.w);
                }
        // adapter term of the slice: A^T (s u_c) for this warp's 64 features
        if (p.r > 0) {
            for (int kc = 0; kc < rk16 / 16; ++kc) {
                const int j = 16 * kc + 2 * t;
#pragma unroll
                for (int f = 0; f < 4; ++f) {
                    const int64_t fA = f0 + 64 * kg + 8 * g + 2 * f, fB = fA + 1;
                    auto a_pair = [&](int64_t feat, int jj) -> uint32_t {
                        if (feat >= p.k) return 0u;
                        const uint32_t lo = jj < p.r ? ld_ro_u16(p.A + static_cast<int64_t>(jj) * p.k + feat) : 0u;
                        const uint32_t hi = jj + 1 < p.r ? ld_ro_u16(p.A + static_cast<int64_t>(jj + 1) * p.k + feat) : 0u;
                        return lo | (hi << 16);
                    };
                    const uint32_t a0 = a_pair(fA, j), a1 = a_pair(fB, j), a2 = a_pair(fA, j + 8), a3 = a_pair(fB, j + 8);
#pragma unroll
                    for (int tg = 0; tg < NG; ++tg) {
                        const uint32_t tr = sub + static_cast<uint32_t>((tg * 8 + g) * rk16 + j) * 2;
                        mma_16816(acc[f][tg], a0, a1, a2, a3, lds32(tr), lds32(tr + 16));
                    }
                }
            }
        }
        if (C == 1 && !*abort_flag) {
#pragma unroll
            for (int f = 0; f < 4; ++f)
#pragma unroll
                for (int tg = 0; tg < NG; ++tg)
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int64_t feat = f0 + 64 * kg + 8 * g + 2 * f + (e >> 1);
                        const int tok = tg * 8 + 2 * t + (e & 1);
                        if (feat < p.k && tok < p.M)
                            p.gx[static_cast<int64_t>(tok) * p.k + feat] =
                                __bfloat16_as_ushort(__float2bfloat16_rn(acc[f][tg][e]));
                    }
        }
    }
    if (C > 1) {
        cluster_wait();  // phase 1: every CTA of the cluster runs
        if (warp > 0 && rg == 0) {
            cg::cluster_group cluster = cg::this_cluster();
#pragma unroll
            for (int f = 0; f < 4; ++f)
#pragma unroll
                for (int hh = 0; hh < 2; ++hh) {
                    const int fl = 64 * kg + 8 * g + 2 * f + hh;  // feature within the chunk
                    const int owner = (fl * C + C - 1) / kChunkFeat;
                    const int rr = fl - kChunkFeat * owner / C;
                    float *dst = cluster.map_shared_rank(recv, owner) + (crank * nrmax + rr) * MP + 2 * t;
#pragma unroll
                    for (int tg = 0; tg < NG; ++tg)
                        *reinterpret_cast<float2 *>(dst + tg * 8) =
                            make_float2(acc[f][tg][2 * hh], acc[f][tg][2 * hh + 1]);
                }
        }
        cluster_arrive_release();
        cluster_wait_acquire();  // phase 2: every partial has landed
        const int r_lo = kChunkFeat * crank / C, r_hi = kChunkFeat * (crank + 1) / C, nr = r_hi - r_lo;
        if (!*abort_flag) {
            for (int it = threadIdx.x; it < nr * p.M; it += kThreads) {
                const int rr = it % nr, tok = it / nr;
                const int64_t feat = f0 + r_lo + rr;
                if (feat >= p.k) continue;
                float sum = 0.0f;
                for (int src = 0; src < C; ++src) sum += recv[(src * nrmax + rr) * MP + tok];
                p.gx[static_cast<int64_t>(tok) * p.k + feat] = __bfloat16_as_ushort(__float2bfloat16_rn(sum));
            }
        }
    }
}

template <int NG>
__global__ void __launch_bounds__(kThreads, 1) k_decode_bwd(const __grid_constant__ CUtensorMap tm_codes,
                                                            const BwdArgs p) {
    extern __shared__ __align__(1024) uint8_t smem[];
    if ((saddr(smem) & 0x00ffffffu) == kDynSmemBase)
        bwd_body<NG, true>(&tm_codes, p, smem);
    else
        bwd_body<NG, false>(&tm_codes, p, smem);
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

int round_rank(int r) { return r <= 0 ? 0 : r <= 8 ? 8 : r <= 16 ? 16 : r <= 32 ? 32 : 64; }

bool layout(BwdArgs &a, int MP) {
    const uint32_t codes = kRowsPerStage * 128u;
    const uint32_t gb = static_cast<uint32_t>(MP) * 128u;
    const uint32_t bb = a.r > 0 ? kRowsPerStage * static_cast<uint32_t>(a.rb) : 0u;
    const uint32_t qb = kRowsPerStage * 8u, sb = kRowsPerStage * 8u;
    a.g_off = codes;
    a.b_off = codes + gb;
    a.q_off = a.b_off + bb;
    a.s_off = a.q_off + qb;
    a.slot_bytes = (a.s_off + sb + 1023u) & ~1023u;
    a.tx_bytes = codes;
    const int rk16 = (a.rpad + 15) & ~15;
    const uint32_t post = kConsumers * 2 * 32 * 16 + ((MP * rk16 * 2 + 255) & ~255) + 3 * 4 * 4 * 32 * 16 * (MP / 8);
    const uint32_t recv =
        a.C > 1 ? (static_cast<uint32_t>(a.C * ((kChunkFeat + a.C - 1) / a.C) * MP * 4) + 1023u) & ~1023u : 0u;
    a.ring_off = kLutBytes;
    const uint32_t fixed = kLutBytes + recv + 1024;
    if (fixed >= kSmemLimit) return false;
    int stages = static_cast<int>((kSmemLimit - fixed) / a.slot_bytes);
    if (stages > kMaxStages) stages = kMaxStages;
    if (stages < 2) return false;
    uint32_t ring = static_cast<uint32_t>(stages) * a.slot_bytes;
    if (ring < post && fixed + ring + post > kSmemLimit) {
        stages = static_cast<int>((kSmemLimit - fixed - post) / a.slot_bytes);
        if (stages < 2) return false;
        ring = static_cast<uint32_t>(stages) * a.slot_bytes;
    }
    a.stages = stages;
    a.post_off = a.ring_off + (ring >= post ? 0u : ring);
    const uint32_t after = a.ring_off + (ring >= post ? ring : ring + post);
    a.recv_off = after;
    a.bar_off = after + recv;
    return true;
}

size_t smem_bytes(const BwdArgs &a) { return static_cast<size_t>(a.bar_off) + 2 * kMaxStages * 8 + 16; }

template <int NG>
cudaError_t launch_ng(const WeightView &w, const uint16_t *gh, int M, const uint16_t *A, const uint16_t *B, int r,
                      float s, uint16_t *gx, int *err, cudaStream_t st) {
    constexpr int MP = 8 * NG;
    const void *kern = reinterpret_cast<const void *>(k_decode_bwd<NG>);
    int sms = 148;
    cudaError_t e = device_sm_count(&sms);
    if (e != cudaSuccess) return e;
    BwdArgs a = {};
    a.q = w.q;
    a.sigma = w.sigma;
    a.mu = w.mu;
    a.gh = gh;
    a.A = A;
    a.B = B;
    a.gx = gx;
    a.err = err;
    a.n = w.n;
    a.k = w.k;
    a.nbr = static_cast<int>(w.k / kBlock);
    a.nrs = static_cast<int>((w.n + kRowsPerStage - 1) / kRowsPerStage);
    a.M = M;
    a.r = r;
    a.rpad = round_rank(r);
    a.rb = r > 0 ? ((r * 2 + 15) / 16) * 16 + 16 : 0;  // padded row: conflict-free ldmatrix rows
    a.s = s;
    const int64_t chunks = (w.k + kChunkFeat - 1) / kChunkFeat;
    // cluster size: the largest C <= 8 with chunks x C <= SMs, every cluster resident and at least
    // one row stage per CTA
    BwdArgs best = a;
    bool found = false;
    for (int C = kMaxCluster; C >= 1; --C) {
        if (chunks * C > sms || C > a.nrs) continue;
        BwdArgs c = a;
        c.C = C;
        if (!layout(c, MP)) continue;
        if (C > 1) {
            int nc = 0;
            e = resident_clusters(kern, kThreads, C, smem_bytes(c), &nc);
            if (e != cudaSuccess) return e;
            if (nc < chunks) continue;
        }
        best = c;
        found = true;
        break;
    }
    if (!found) {
        best.C = 1;
        if (!layout(best, MP)) return cudaErrorInvalidConfiguration;
    }
    a = best;
    const size_t smem = smem_bytes(a);

    CUtensorMap tm_codes;
    {
        auto fn = encode_fn();
        if (!fn) return cudaErrorInvalidValue;
        cuuint64_t dims[2] = {static_cast<cuuint64_t>(w.k / 2), static_cast<cuuint64_t>(w.n)};
        cuuint64_t strides[1] = {static_cast<cuuint64_t>(w.k / 2)};
        cuuint32_t box[2] = {128, static_cast<cuuint32_t>(kRowsPerStage)};
        cuuint32_t estr[2] = {1, 1};
        if (fn(&tm_codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t *>(w.codes), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return cudaErrorInvalidValue;
    }
    e = ensure_smem_limit(kern, smem);
    if (e != cudaSuccess) return e;
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
    e = cudaLaunchKernelEx(&cfg, k_decode_bwd<NG>, tm_codes, a);
    count_launch();
    return e;
}

}  // namespace

cudaError_t launch_decode_bwd_stream(const WeightView &w, const uint16_t *gh, int M, const uint16_t *A,
                                     const uint16_t *B, int r, float s, uint16_t *gx, int *err, cudaStream_t st) {
    if (M <= 0 || w.k == 0) return cudaSuccess;
    if (M > kDecodeTokens || r > kDecodeMaxRank) return cudaErrorInvalidValue;
    if (M <= 8) return launch_ng<1>(w, gh, M, A, B, r, s, gx, err, st);
    return launch_ng<2>(w, gh, M, A, B, r, s, gx, err, st);
}

}  // namespace qn
