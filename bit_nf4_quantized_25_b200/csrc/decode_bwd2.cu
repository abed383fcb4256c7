// decode_bwd2.cu -- QLoRA input gradient for few tokens (M <= 16 per launch) on sm_100a.
//
//   grad_x[m,k] = sum_n grad_h[m,n] W'[n,k] + sum_j A[j,k] u[m,j],  u = bf16(s sum_n grad_h[m,n] B[n,j])
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
// Work split. One CTA per SM. A CTA owns a 256-feature column chunk (4 blocks, one 128-byte code
// column) over a slice of the weight rows; the C row slices of a chunk form a thread-block
// cluster. The CTA streams its rows through a ring of 128-row stages: the codes box (128-byte
// swizzled), the stage's grad_h columns (two swizzled boxes of 64 rows x the tokens), the stage's
// FP8 block codes (a 16-byte wide box, or per-row copies when the rows of FP8 codes are not
// 16-byte aligned) and its group scales.
//   warp 0      : producer.
//   warps 1..16 : consumers. Warp (kg, rg) takes block kg (64 features) and the rows
//                 16 rg + 64 j .. + 16 (j = 0, 1) of every stage; its accumulators hold the CTA's
//                 partial sums for those 64 features. Lanes compute the block constants of the
//                 warp's rows and share them by shuffles.
// The adapter product u = bf16(s B^T grad_h) is computed once per call by one more cluster (the
// first row of the grid): its CTAs stream grad_h and B over the same row slices, reduce into
// rank 0, which publishes u in the workspace and raises a flag (the protocol of the forward
// kernel). After the loop the four row-warps of each block are summed in a fixed order (rg =
// 0..3), sub-tile f of block kg by warp (kg, rg = f); in the CTA that owns a block's adapter term
// (block kg = crank mod C) the same warp adds A^T u for its sub-tile on the tensor cores from the
// A tile it staged; the partial sums go by asynchronous DSMEM stores to the CTA that finalises
// those features, which sums the slices in rank order and stores grad_x. Bit-reproducible.
//
// Programmatic launch: the packed weight is requested before the dependency wait; grad_h, A and
// B are read, and grad_x written, only after it (the caller's guarantee of the forward kernel
// applies). Every wait is bounded; a timeout records an error code in the workspace error word.
// Shapes: n_out % 8 == 0 and r % 8 == 0 (the grad_h and B rows are TMA rows); the host routes
// other shapes to the register-streaming kernel of decode_bwd.cu.
#include <cudaTypedefs.h>

#include "dropout.cuh"
#include "host_cache.h"
#include "stream_common.cuh"

namespace qn {

namespace {

using namespace sm100;
using namespace stream;

constexpr int kConsumers = 16;
constexpr int kThreads = 32 * (kConsumers + 1);
constexpr int kSR = 128;  // rows per stage
constexpr int kChunkFeat = 256;
constexpr int kMaxStages = 8;
constexpr int kMaxCluster = 8;
constexpr size_t kSmemLimit = 227 * 1024;
constexpr size_t kWsFlag = 64, kWsReaders = 128, kWsU = 256;

struct BwdArgs {
    const uint8_t *q;
    const float *sigma;
    const float *mu;
    const float *absmax;  // fp32 block constants (no double quantisation), else nullptr
    int qtype;            // table of the code nibbles
    uint16_t *gx;  // M x k
    int *err;
    uint16_t *u_ws;     // [MP][rk16] bf16 u, published by the adapter cluster
    unsigned *flag;     // 1 while u_ws holds this call's u
    unsigned *readers;  // CTAs that have copied u_ws
    int64_t n, k;
    int nbr;     // blocks per row
    int nrs;     // row stages (ceil(n / kSR))
    int chunks;  // feature chunks (ceil(k / 256)): grid rows 1 .. chunks when r > 0, else 0 ..
    int M, r, rpad, rk16;
    float s;           // adapter scale (divided by 1 - p under dropout)
    DropoutArgs drop;  // mask of the forward's adapter input (thr == 0: none); offset of token 0
    int C, stages;
    int q_tma;  // FP8 codes by a TMA box (rows of FP8 codes 16-byte aligned), else per-row copies
    uint32_t slot_bytes, g_off, q_off, s_off;  // chunk slot: codes, grad_h, FP8 codes (or fp32 constants),
                                               // group scales
    uint32_t b_off;                            // adapter slot: grad_h at 0, B at b_off
    uint32_t ring_off, ut_off, at_off, recv_off, bar_off, post_off;
    uint32_t codes_bytes, g_bytes, q_bytes, gb_bytes;  // transaction bytes
    int s_cap;  // group scales staged per stage (upper bound)
};

struct Bars {
    uint64_t *full, *empty, *recv, *atile;
    volatile uint32_t *abort_flag;
};

__device__ __forceinline__ Bars bars_of(uint8_t *smem, const BwdArgs &p) {
    Bars b;
    b.full = reinterpret_cast<uint64_t *>(smem + p.bar_off);
    b.empty = b.full + kMaxStages;
    b.recv = b.empty + kMaxStages;
    b.atile = b.recv + 1;
    b.abort_flag = reinterpret_cast<volatile uint32_t *>(b.atile + 1);
    return b;
}

__device__ __forceinline__ void ldm_x4_trans(uint32_t a, uint32_t &r0, uint32_t &r1, uint32_t &r2, uint32_t &r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(a));
}

// grad_h pair (rows `row`, row + 1 of the stage, row even) of token `tok`: two swizzled boxes of
// 64 rows, [token][64 rows], 16-byte chunk c of token row tok at c ^ (tok & 7).
template <int MP>
__device__ __forceinline__ uint32_t gh_pair(uint32_t gbase, int tok, int row) {
    const uint32_t box = gbase + static_cast<uint32_t>((row >> 6) * MP * 128);
    const int rr = row & 63;
    const int c = rr >> 3, w = (rr & 7) >> 1;
    return lds32(box + static_cast<uint32_t>(tok * 128 + ((c ^ (tok & 7)) << 4) + w * 4));
}

// ------------------------------------------------------------------------------ adapter cluster
// u_c = B^T grad_h over this CTA's row slice; rank 0 sums and publishes bf16(s u).
template <int NG>
__device__ __forceinline__ void adapter_body(const CUtensorMap *tm_g, const CUtensorMap *tm_b, const BwdArgs &p,
                                             uint8_t *smem) {
    constexpr int MP = 8 * NG;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, t = lane & 3;
    const int C = p.C;
    const int crank = C > 1 ? static_cast<int>(cg::this_cluster().block_rank()) : 0;
    const int rs_lo = p.nrs * crank / C, rs_hi = p.nrs * (crank + 1) / C;
    const int ns = rs_hi - rs_lo;
    const int S = p.stages;
    const uint32_t s_base = saddr(smem);
    const uint32_t s_ring = s_base + p.ring_off;
    const Bars bb = bars_of(smem, p);
    const int brow = 2 * p.rpad;  // bytes per B row in the box

    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(&bb.full[s], 1);
            mbar_init(&bb.empty[s], kConsumers);
        }
        mbar_init(bb.recv, 1);
        if (C > 1 && crank == 0) mbar_arrive_expect_tx(bb.recv, static_cast<uint32_t>(C * MP * p.rpad * 4));
        *bb.abort_flag = 0u;
        fence_barrier_init();
        tma_prefetch_desc(tm_g);
        tma_prefetch_desc(tm_b);
    }
    __syncthreads();
    if (C > 1) cluster_arrive_relaxed();
    grid_dependents_launch();
    grid_dependency_wait();  // grad_h and B may come from the preceding kernel

    auto fail = [&]() {
        if (atomicExch(const_cast<uint32_t *>(bb.abort_flag), 1u) == 0u) record_error(p.err, kErrTimeout);
    };
    const int cw = warp - 1;
    const int NT = p.rpad / 8;
    // jobs per stage: (k16 step kq = 0..7 over the 128 rows) x (rank tile nt) = 8 NT, split over
    // the 16 warps; warp cw takes jobs cw, cw + 16, cw + 32, cw + 48
    float uacc[4][4];
#pragma unroll
    for (int j = 0; j < 4; ++j) uacc[j][0] = uacc[j][1] = uacc[j][2] = uacc[j][3] = 0.0f;
    if (warp == 0) {
        int ni = 0;
        if (lane == 0) {
            for (int s = 0; s < ns; ++s) {
                const int slot = s % S;
                if (*bb.abort_flag) break;
                if (s >= S && !mbar_wait(&bb.empty[slot], ((s / S) & 1) ^ 1)) {
                    fail();
                    break;
                }
                const int32_t n0 = (rs_lo + s) * kSR;
                const uint32_t sl = s_ring + static_cast<uint32_t>(slot) * p.slot_bytes;
                mbar_arrive_expect_tx(&bb.full[slot], p.g_bytes + p.gb_bytes);
                tma_load_2d_saddr(sl, tm_g, &bb.full[slot], n0, 0);
                tma_load_2d_saddr(sl + MP * 128, tm_g, &bb.full[slot], n0 + 64, 0);
                tma_load_2d_saddr(sl + p.b_off, tm_b, &bb.full[slot], 0, n0);
                ni = s + 1;
            }
            for (int s = (ni > S ? ni - S : 0); s < ni; ++s) mbar_wait(&bb.full[s % S], (s / S) & 1);
        }
        __syncwarp();
    } else {
        for (int s = 0; s < ns; ++s) {
            const int slot = s % S;
            // every lane waits for the stage; the warp leaves together (mma.sync and shuffles below)
            const bool ok = !*bb.abort_flag && mbar_wait(&bb.full[slot], (s / S) & 1);
            if (!__all_sync(0xffffffffu, ok)) {
                if (!ok) fail();
                break;
            }
            const uint32_t sl = s_ring + static_cast<uint32_t>(slot) * p.slot_bytes;
#pragma unroll
            for (int jj = 0; jj < 4; ++jj) {
                const int job = cw + 16 * jj;
                if (job >= 8 * NT) break;
                const int kq = job & 7, nt = job >> 3;
                // A operand: grad_h[tok][rows 16 kq ..]; B operand: B[rows][ranks 8 nt ..] by
                // ldmatrix.trans from the swizzled [row][rpad] box
                const uint32_t a0 = gh_pair<MP>(sl, g, 16 * kq + 2 * t);
                const uint32_t a2 = gh_pair<MP>(sl, g, 16 * kq + 2 * t + 8);
                uint32_t a1 = 0u, a3 = 0u;
                if (NG > 1) {
                    a1 = gh_pair<MP>(sl, g + 8, 16 * kq + 2 * t);
                    a3 = gh_pair<MP>(sl, g + 8, 16 * kq + 2 * t + 8);
                }
                const int mi = lane >> 3, rr = lane & 7;
                const int row = 16 * kq + 8 * (mi & 1) + rr;  // lanes 16..31 repeat lanes 0..15
                // 16-byte chunk nt of the row, swizzled by the box's mode (chunk ^ key(row))
                uint32_t key;
                if (brow == 128) key = row & 7;
                else if (brow == 64) key = (row >> 1) & 3;
                else if (brow == 32) key = (row >> 2) & 1;
                else key = 0;
                const uint32_t baddr = sl + p.b_off + static_cast<uint32_t>(row * brow) + ((nt ^ key) << 4);
                uint32_t b0, b1, b2, b3;
                ldm_x4_trans(baddr, b0, b1, b2, b3);
                mma_16816(uacc[jj], a0, a1, a2, a3, b0, b1);
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&bb.empty[slot]);
        }
    }
    __syncthreads();
    // per-CTA sums of the rank tiles: tile nt collects jobs (kq = 0..7, nt) in kq order
    const uint32_t ubuf = s_base + p.post_off;  // [64 jobs][32 lanes][4] f32, in the idle ring
    if (warp > 0) {
#pragma unroll
        for (int jj = 0; jj < 4; ++jj) {
            const int job = cw + 16 * jj;
            if (job < 8 * NT)
                asm volatile("st.shared.v4.f32 [%0], {%1,%2,%3,%4};" ::"r"(ubuf + static_cast<uint32_t>(job * 32 + lane) * 16),
                             "f"(uacc[jj][0]), "f"(uacc[jj][1]), "f"(uacc[jj][2]), "f"(uacc[jj][3])
                             : "memory");
        }
    }
    __syncthreads();
    const uint32_t recv = s_base + p.recv_off;
    if (C > 1) cluster_wait();
    if (warp > 0 && cw < NT) {
        float uu[4] = {0.0f, 0.0f, 0.0f, 0.0f};
        for (int kq = 0; kq < 8; ++kq) {
            const uint4 v = lds128(ubuf + static_cast<uint32_t>((8 * cw + kq) * 32 + lane) * 16);
            uu[0] += __uint_as_float(v.x);
            uu[1] += __uint_as_float(v.y);
            uu[2] += __uint_as_float(v.z);
            uu[3] += __uint_as_float(v.w);
        }
        const int j = 8 * cw + 2 * t;  // fragment: tokens g / g + 8, ranks j, j + 1
        const uint32_t o0 = recv + static_cast<uint32_t>(((crank * MP + g) * p.rpad + j) * 4);
        const uint32_t o1 = recv + static_cast<uint32_t>(((crank * MP + g + 8) * p.rpad + j) * 4);
        if (C > 1) {
            const uint32_t bar = mapa(saddr(bb.recv), 0);
            st_async_v2(mapa(o0, 0), uu[0], uu[1], bar);
            if (NG > 1) st_async_v2(mapa(o1, 0), uu[2], uu[3], bar);
        } else {
            asm volatile("st.shared.v2.f32 [%0], {%1,%2};" ::"r"(o0), "f"(uu[0]), "f"(uu[1]) : "memory");
            if (NG > 1) asm volatile("st.shared.v2.f32 [%0], {%1,%2};" ::"r"(o1), "f"(uu[2]), "f"(uu[3]) : "memory");
        }
    }
    if (crank != 0) return;
    bool ok = true;
    if (C > 1) {
        ok = mbar_wait(bb.recv, 0);
        if (!ok && threadIdx.x == 0) record_error(p.err, kErrTimeout);
    } else {
        __syncthreads();
    }
    const int half = p.rk16 / 2;
    const float *rv = reinterpret_cast<const float *>(smem + p.recv_off);
    for (int i = threadIdx.x; i < MP * half; i += kThreads) {
        const int tok = i / half, j = 2 * (i - tok * half);
        float v0 = 0.0f, v1 = 0.0f;
        if (j < p.rpad)
            for (int src = 0; src < C; ++src) {
                v0 += rv[(src * MP + tok) * p.rpad + j];
                v1 += rv[(src * MP + tok) * p.rpad + j + 1];
            }
        reinterpret_cast<uint32_t *>(p.u_ws)[i] = pack_bf16x2(p.s * v0, p.s * v1);
    }
    __syncthreads();
    if (threadIdx.x == 0 && ok && !*bb.abort_flag) {
        __threadfence();
        st_release_u32(p.flag, 1u);
    }
}

// ------------------------------------------------------------------------------ chunk clusters
template <int NG, bool kFixedBase>
__device__ __forceinline__ void chunk_body(const CUtensorMap *tm_codes, const CUtensorMap *tm_g,
                                           const CUtensorMap *tm_q, const CUtensorMap *tm_a, const BwdArgs &p,
                                           uint8_t *smem) {
    constexpr int MP = 8 * NG;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, t = lane & 3;
    const int C = p.C;
    const int crank = C > 1 ? static_cast<int>(cg::this_cluster().block_rank()) : 0;
    const int col = static_cast<int>(blockIdx.y) - (p.r > 0 ? 1 : 0);  // 128-byte code column: 256 features
    const int64_t f0 = static_cast<int64_t>(col) * kChunkFeat;
    const int rs_lo = p.nrs * crank / C, rs_hi = p.nrs * (crank + 1) / C;
    const int ns = rs_hi - rs_lo;
    const int S = p.stages;
    const int npre = ns < S ? ns : S;
    // features [f_lo, f_hi) of the chunk are finalised by this CTA (C > 1)
    const int f_lo = kChunkFeat * crank / C, f_hi = kChunkFeat * (crank + 1) / C, nf = f_hi - f_lo;
    const int nfmax = (kChunkFeat + C - 1) / C;

    uint8_t *lut = smem;
    const uint32_t s_base = saddr(smem);
    const uint32_t s_ring = s_base + p.ring_off;
    const uint32_t ut = s_base + p.ut_off;  // [MP tokens][rk16] bf16 u
    const uint32_t at = s_base + p.at_off;  // A tile of the CTA's adapter blocks: [blk][rpad][128 B] swizzled
    const Bars bb = bars_of(smem, p);
    const int64_t nbq = p.n * p.nbr;
    const int64_t ngs = (nbq + kGroup - 1) / kGroup;

    // Stage s covers rows n0 = (rs_lo + s) * 128 ..; its group scales start at the chunk-aligned
    // index sg0(s) = ((n0 nbr + 4 col) >> 8) & ~3. Lane 0 requests the codes (and the FP8 codes by
    // TMA); all lanes copy the rest with cp.async, whose arrivals complete on the stage's barrier.
    auto stage_weights = [&](int s, uint64_t pol) {
        const int slot = s % S;
        const uint32_t sl = s_ring + static_cast<uint32_t>(slot) * p.slot_bytes;
        const int64_t n0 = static_cast<int64_t>(rs_lo + s) * kSR;
        if (lane == 0) {
            mbar_expect_tx(&bb.full[slot], p.codes_bytes + (p.q_tma ? p.q_bytes : 0u));
            tma_load_2d_saddr_hint(sl, tm_codes, &bb.full[slot], col * 128, static_cast<int32_t>(n0), pol);
            if (p.q_tma)
                tma_load_2d_saddr(sl + p.q_off, tm_q, &bb.full[slot], (4 * col) & ~15, static_cast<int32_t>(n0));
        }
        if (p.absmax) {
            // fp32 constants: per row the two 16-byte chunks from the one that holds block 4 col
            for (int i = lane; i < 2 * kSR; i += 32) {
                const int ri = i >> 1, h = i & 1;
                const int64_t row = n0 + ri;
                const int64_t cb = ((row < p.n ? row * p.nbr + 4 * col : 0) >> 2) + h;
                const int64_t avail = row < p.n ? 4 * (nbq - 4 * cb) : 0;
                const uint32_t bytes = avail >= 16 ? 16u : (avail > 0 ? static_cast<uint32_t>(avail) : 0u);
                cp_async16_zfill(sl + p.q_off + 32u * ri + 16u * h, p.absmax + (bytes ? 4 * cb : 0), bytes);
            }
            cp_async_arrive_noinc(&bb.full[slot]);
            return;
        }
        if (!p.q_tma) {
            // per row the 16-byte chunk that holds its four FP8 codes of this column
            for (int i = lane; i < kSR; i += 32) {
                const int64_t row = n0 + i;
                const int64_t cb = (row < p.n ? row * p.nbr + 4 * col : 0) >> 4;
                const int64_t avail = row < p.n ? nbq - 16 * cb : 0;
                const uint32_t bytes = avail >= 16 ? 16u : (avail > 0 ? static_cast<uint32_t>(avail) : 0u);
                cp_async16_zfill(sl + p.q_off + 16u * i, p.q + (bytes ? 16 * cb : 0), bytes);
            }
        }
        const int64_t last = n0 + kSR - 1 < p.n ? n0 + kSR - 1 : p.n - 1;
        const int64_t sg0 = ((n0 * p.nbr + 4 * col) >> 8) & ~int64_t(3);
        const int64_t elast = last * p.nbr + 4 * col + 3 < nbq ? last * p.nbr + 4 * col + 3 : nbq - 1;
        const int nch = static_cast<int>(((elast >> 8) - sg0) / 4 + 1);
        for (int c = lane; c < nch; c += 32) {
            const int64_t f = sg0 + 4 * c;
            const int64_t avail = 4 * (ngs - f);
            const uint32_t bytes = avail >= 16 ? 16u : (avail > 0 ? static_cast<uint32_t>(avail) : 0u);
            cp_async16_zfill(sl + p.s_off + 16u * c, p.sigma + (bytes ? f : 0), bytes);
        }
        cp_async_arrive_noinc(&bb.full[slot]);
    };

    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(&bb.full[s], 33);  // lane 0's arrive.expect_tx + 32 cp.async arrivals
            mbar_init(&bb.empty[s], kConsumers);
        }
        mbar_init(bb.recv, 1);
        if (C > 1) mbar_arrive_expect_tx(bb.recv, static_cast<uint32_t>(C * nf * MP * 4));
        mbar_init(bb.atile, 1);
        *bb.abort_flag = 0u;
        fence_barrier_init();
        tma_prefetch_desc(tm_codes);
        tma_prefetch_desc(tm_g);
        if (p.q_tma) tma_prefetch_desc(tm_q);
    }
    __syncthreads();  // barriers initialised
    if (warp == 0) {
        // weights of the first stages before the dependency wait; the producer then goes on to
        // the dependency wait and the grad_h requests while the consumers build the table
        const uint64_t pol = l2_policy_evict_first();
        for (int s = 0; s < npre; ++s) stage_weights(s, pol);
    } else {
        build_pair_lut(lut, threadIdx.x - 32, kThreads - 32, p.qtype);
        named_sync(1, kConsumers * 32);  // the table is complete
    }
    if (C > 1) cluster_arrive_relaxed();
    grid_dependents_launch();
    grid_dependency_wait();  // grad_h, A and B may come from the preceding kernel; grad_x may be read by it

    auto fail = [&]() {
        if (atomicExch(const_cast<uint32_t *>(bb.abort_flag), 1u) == 0u) record_error(p.err, kErrTimeout);
    };
    const int cw = warp - 1;
    const int kg = cw & 3, rg = cw >> 2;
    // blocks kg with kg % C == crank carry this CTA's adapter term
    const int nablk = p.r > 0 ? (4 - crank + C - 1) / C : 0;
    float acc[4][NG][4];  // sub-tile f, token group, fragment
#pragma unroll
    for (int f = 0; f < 4; ++f)
#pragma unroll
        for (int tg = 0; tg < NG; ++tg) acc[f][tg][0] = acc[f][tg][1] = acc[f][tg][2] = acc[f][tg][3] = 0.0f;

    if (warp == 0) {
        // ------------------------------------------------------------------ producer
        int ni = 0;
        if (lane == 0 && nablk > 0) {
            // A tile of the adapter blocks (one 3-D box per block: [rpad ranks][64 features])
            mbar_arrive_expect_tx(bb.atile, static_cast<uint32_t>(nablk * p.rpad * 128));
            for (int i = 0; i < nablk; ++i)
                tma_load_3d_saddr(at + static_cast<uint32_t>(i * p.rpad * 128), tm_a, bb.atile, 0, 0,
                                  4 * col + i * C + crank);
        }
        for (int s = 0; s < ns; ++s) {
            const int slot = s % S;
            // lane 0 decides (abort flag, slot wait) and the warp follows it as one
            int st = 0;  // 0 go on, 1 aborted elsewhere, 2 this wait ran out
            if (lane == 0) {
                if (*bb.abort_flag) st = 1;
                else if (s >= S && !mbar_wait(&bb.empty[slot], ((s / S) & 1) ^ 1)) st = 2;
            }
            st = __shfl_sync(0xffffffffu, st, 0);
            if (st != 0) {
                if (lane == 0 && st == 2) fail();
                break;
            }
            if (s >= S) stage_weights(s, l2_policy_evict_first());
            if (lane == 0) {
                const int32_t n0 = (rs_lo + s) * kSR;
                const uint32_t sl = s_ring + static_cast<uint32_t>(slot) * p.slot_bytes;
                mbar_arrive_expect_tx(&bb.full[slot], p.g_bytes);
                tma_load_2d_saddr(sl + p.g_off, tm_g, &bb.full[slot], n0, 0);
                tma_load_2d_saddr(sl + p.g_off + MP * 128, tm_g, &bb.full[slot], n0 + 64, 0);
            }
            ni = s + 1;
        }
        if (lane == 0) {
            // stages staged before the wait but never armed get lane 0's arrival; then every
            // requested stage lands before the CTA can exit
            for (int s = ni; s < npre; ++s) mbar_arrive(&bb.full[s]);
            const int hi = ni > npre ? ni : npre;
            for (int s = (hi > S ? hi - S : 0); s < hi; ++s) mbar_wait(&bb.full[s % S], (s / S) & 1);
            if (nablk > 0) mbar_wait(bb.atile, 0);
        }
        // u from the adapter cluster
        if (p.r > 0) {
            bool ok = true;
            if (lane == 0) ok = wait_flag(p.flag);
            ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
            if (!ok) {
                if (lane == 0) fail();
            } else {
                for (int i = lane; i < MP * p.rk16 / 2; i += 32)
                    asm volatile("st.shared.b32 [%0], %1;" ::"r"(ut + 4u * i), "r"(ld_cg_u32(p.u_ws + 2 * i))
                                 : "memory");
                __syncwarp();
                if (lane == 0) {
                    const unsigned old = atomicAdd(p.readers, 1u);
                    if (old == static_cast<unsigned>(p.chunks * C) - 1u) {
                        atomicExch(p.readers, 0u);
                        atomicExch(p.flag, 0u);
                    }
                }
            }
        }
        cp_async_wait_all();
        __syncwarp();
    } else {
        // ------------------------------------------------------------------ consumers
        const uint32_t lane_op = lut_lane_operand<kFixedBase>(lut, lane);
        const uint32_t lut_base = s_base;
        const float mu = load_mu(p.mu, p.absmax);
        // source lanes of rows 2t, 2t+1, 2t+8, 2t+9 (row rho of a 16-row tile is computed by lane
        // 4 (rho & 7) + (rho >> 3))
        const int src0 = 4 * ((2 * t) & 7) + 0, src1 = 4 * ((2 * t + 1) & 7) + 0;
        const int src8 = 4 * ((2 * t) & 7) + 1, src9 = 4 * ((2 * t + 1) & 7) + 1;
        const bool blk_ok = 4 * col + kg < p.nbr;
        for (int s = 0; s < ns; ++s) {
            const int slot = s % S;
            // every lane waits for the stage; the warp leaves together (mma.sync and shuffles below)
            const bool ok = !*bb.abort_flag && mbar_wait(&bb.full[slot], (s / S) & 1);
            if (!__all_sync(0xffffffffu, ok)) {
                if (!ok) fail();
                break;
            }
            const int64_t n0 = static_cast<int64_t>(rs_lo + s) * kSR;
            const uint32_t sl = s_ring + static_cast<uint32_t>(slot) * p.slot_bytes;
            const int64_t sg0 = ((n0 * p.nbr + 4 * col) >> 8) & ~int64_t(3);
#pragma unroll
            for (int j = 0; j < 2; ++j) {
                const int rt = 16 * rg + 64 * j;  // first row of this 16-row tile within the stage
                // block constant of (row rt + g + 8 (t & 1), block kg)
                float cmine = 0.0f;
                {
                    const int ri = rt + g + 8 * (t & 1);
                    const int64_t row = n0 + ri;
                    if (row < p.n && blk_ok) {
                        const int64_t e = row * p.nbr + 4 * col + kg;
                        if (p.absmax) {
                            cmine = __uint_as_float(
                                lds32(sl + p.q_off + 32u * ri + 4u * static_cast<uint32_t>(((e - kg) & 3) + kg)));
                        } else {
                            const uint32_t qb =
                                lds8(sl + p.q_off + 16u * ri + static_cast<uint32_t>((e - kg) & 15) + kg);
                            const float sg =
                                __uint_as_float(lds32(sl + p.s_off + 4u * static_cast<uint32_t>((e >> 8) - sg0)));
                            cmine = block_constant(static_cast<uint8_t>(qb), sg, mu);
                        }
                    }
                }
                const float c0 = __shfl_sync(0xffffffffu, cmine, src0), c1 = __shfl_sync(0xffffffffu, cmine, src1);
                const float c8 = __shfl_sync(0xffffffffu, cmine, src8), c9 = __shfl_sync(0xffffffffu, cmine, src9);
                // token operand: grad_h of rows 2t, 2t+1 (b0) and 2t+8, 2t+9 (b1) of the tile, scaled
                const uint32_t gb = sl + p.g_off;
                uint32_t bop[NG][2];
#pragma unroll
                for (int tg = 0; tg < NG; ++tg) {
                    const int tok = tg * 8 + g;
                    const uint32_t v01 = gh_pair<MP>(gb, tok, rt + 2 * t);
                    const uint32_t v89 = gh_pair<MP>(gb, tok, rt + 2 * t + 8);
                    bop[tg][0] = pack_bf16x2(c0 * bf16_lo(v01), c1 * bf16_hi(v01));
                    bop[tg][1] = pack_bf16x2(c8 * bf16_lo(v89), c9 * bf16_hi(v89));
                }
                // codes: bytes 32 kg + 4 g .. + 4 of rows rt + 2t, + 1, + 8, + 9; 16-byte chunk
                // 2 kg + (g >> 2) of the 128-byte row at chunk ^ (row & 7)
                const int ra = rt + 2 * t;
                auto code_word = [&](int row) {
                    return lds32(sl + static_cast<uint32_t>(row * 128 + (((2 * kg + (g >> 2)) ^ (row & 7)) << 4) +
                                                            4 * (g & 3)));
                };
                const uint32_t w0 = code_word(ra), w1 = code_word(ra + 1), w8 = code_word(ra + 8),
                               w9 = code_word(ra + 9);
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
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&bb.empty[slot]);
        }
    }

    // ---------------------------------------------------------------------- reduction
    __syncthreads();
    // Sub-tile f of block kg is summed, given its adapter term and stored or pushed by warp
    // (kg, rg = f), so that this work spreads over all the consumer warps.
    const uint32_t red = s_base + p.post_off;  // [4 rg][4 blocks][4 f][32 lanes][NG][4] f32, in the idle ring
    if (warp > 0) {
#pragma unroll
        for (int f = 0; f < 4; ++f) {
            if (f == rg) continue;
#pragma unroll
            for (int tg = 0; tg < NG; ++tg) {
                const uint32_t o = red + static_cast<uint32_t>((((rg * 4 + kg) * 4 + f) * 32 + lane) * NG + tg) * 16;
                asm volatile("st.shared.v4.f32 [%0], {%1,%2,%3,%4};" ::"r"(o), "f"(acc[f][tg][0]), "f"(acc[f][tg][1]),
                             "f"(acc[f][tg][2]), "f"(acc[f][tg][3])
                             : "memory");
            }
        }
    }
    __syncthreads();
    const bool run_ok = !*bb.abort_flag;
    const int fo = rg;  // the sub-tile this warp sums
    // features of sub-tile fo: fragment row g -> 64 kg + 8 g + 2 fo, row g + 8 -> 64 kg + 8 g + 2 fo + 1
    float sum[NG][4];
    if (warp > 0) {
        float own[NG][4];
#pragma unroll
        for (int f = 0; f < 4; ++f)
            if (f == fo)
#pragma unroll
                for (int tg = 0; tg < NG; ++tg)
#pragma unroll
                    for (int e = 0; e < 4; ++e) own[tg][e] = acc[f][tg][e];
        // the four row-group warps' partials in rg order
#pragma unroll
        for (int q = 0; q < 4; ++q)
#pragma unroll
            for (int tg = 0; tg < NG; ++tg) {
                float v[4];
                if (q == rg) {
                    v[0] = own[tg][0], v[1] = own[tg][1], v[2] = own[tg][2], v[3] = own[tg][3];
                } else {
                    const uint4 w4 = lds128(red + static_cast<uint32_t>((((q * 4 + kg) * 4 + fo) * 32 + lane) * NG + tg) * 16);
                    v[0] = __uint_as_float(w4.x), v[1] = __uint_as_float(w4.y);
                    v[2] = __uint_as_float(w4.z), v[3] = __uint_as_float(w4.w);
                }
#pragma unroll
                for (int e = 0; e < 4; ++e) sum[tg][e] = q == 0 ? v[e] : sum[tg][e] + v[e];
            }
        // adapter term of block kg (this CTA's when kg = crank mod C), sub-tile fo: A^T u from the
        // staged tile [rpad ranks][64 features] (128-byte swizzle: chunk c of rank row j at
        // c ^ (j & 7)); under dropout only the elements whose input survived the forward's mask
        // receive it
        if (p.r > 0 && kg % C == crank) {
            const uint32_t ab = at + static_cast<uint32_t>((kg / C) * p.rpad * 128);
            auto a_el = [&](int j, int feat) -> uint32_t {  // A[j][64 kg + feat] (bf16 bits)
                const uint32_t a = ab + static_cast<uint32_t>(j * 128 + (((feat >> 3) ^ (j & 7)) << 4) + (feat & 7) * 2);
                uint32_t v;
                asm volatile("ld.shared.u16 %0, [%1];" : "=r"(v) : "r"(a));
                return v;
            };
            auto pair = [&](int jj, int feat) -> uint32_t {
                if (jj >= p.rpad) return 0u;
                return a_el(jj, feat) | (a_el(jj + 1, feat) << 16);
            };
            const int fa = 8 * g + 2 * fo, fb = fa + 1;
            float ad[NG][4];
#pragma unroll
            for (int tg = 0; tg < NG; ++tg) ad[tg][0] = ad[tg][1] = ad[tg][2] = ad[tg][3] = 0.0f;
            for (int kc = 0; kc < p.rk16 / 16; ++kc) {
                const int j = 16 * kc + 2 * t;
                const uint32_t a0 = pair(j, fa), a1 = pair(j, fb), a2 = pair(j + 8, fa), a3 = pair(j + 8, fb);
#pragma unroll
                for (int tg = 0; tg < NG; ++tg) {
                    const uint32_t ur = ut + static_cast<uint32_t>((tg * 8 + g) * p.rk16 + j) * 2u;
                    mma_16816(ad[tg], a0, a1, a2, a3, lds32(ur), lds32(ur + 16));
                }
            }
#pragma unroll
            for (int tg = 0; tg < NG; ++tg) {
                // fragment element e: feature 64 kg + fa + (e >> 1), token tg 8 + 2 t + (e & 1)
                uint32_t keep = 0xfu;
                if (p.drop.thr != 0u) {
                    const int64_t feat = f0 + 64 * kg + fa;
                    const int tok = tg * 8 + 2 * t;
                    const uint32_t k0 =
                        dropout_keep_bits(p.drop, p.drop.offset + static_cast<uint64_t>(tok * p.k + feat), 2);
                    const uint32_t k1 =
                        dropout_keep_bits(p.drop, p.drop.offset + static_cast<uint64_t>((tok + 1) * p.k + feat), 2);
                    // e = 0: (fa, tok), 1: (fa, tok + 1), 2: (fb, tok), 3: (fb, tok + 1)
                    keep = (k0 & 1u) | ((k1 & 1u) << 1) | ((k0 & 2u) << 1) | ((k1 & 2u) << 2);
                }
#pragma unroll
                for (int e = 0; e < 4; ++e)
                    if (keep & (1u << e)) sum[tg][e] += ad[tg][e];
            }
        }
        if (C == 1 && run_ok) {
#pragma unroll
            for (int tg = 0; tg < NG; ++tg)
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int64_t feat = f0 + 64 * kg + 8 * g + 2 * fo + (e >> 1);
                    const int tok = tg * 8 + 2 * t + (e & 1);
                    if (feat < p.k && tok < p.M)
                        p.gx[static_cast<int64_t>(tok) * p.k + feat] =
                            __bfloat16_as_ushort(__float2bfloat16_rn(sum[tg][e]));
                }
        }
    }
    if (C > 1) {
        cluster_wait();  // phase 1: every CTA of the cluster runs (its barriers are initialised)
        if (warp > 0) {
            const uint32_t recv = s_base + p.recv_off;
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
                const int fl = 64 * kg + 8 * g + 2 * fo + hh;  // feature within the chunk
                const int owner = (fl * C + C - 1) / kChunkFeat;
                const int rr = fl - kChunkFeat * owner / C;
                const uint32_t dst = mapa(recv + static_cast<uint32_t>(((crank * nfmax + rr) * MP + 2 * t) * 4),
                                          static_cast<uint32_t>(owner));
                const uint32_t bar = mapa(saddr(bb.recv), static_cast<uint32_t>(owner));
#pragma unroll
                for (int tg = 0; tg < NG; ++tg)
                    st_async_v2(dst + 32u * tg, sum[tg][2 * hh], sum[tg][2 * hh + 1], bar);
            }
        }
        const bool ok = mbar_wait(bb.recv, 0);
        if (!ok && threadIdx.x == 0) record_error(p.err, kErrTimeout);
        if (ok && run_ok) {
            const float *recvf = reinterpret_cast<const float *>(smem + p.recv_off);
            for (int it = threadIdx.x; it < nf * p.M; it += kThreads) {
                const int rr = it % nf, tok = it / nf;
                const int64_t feat = f0 + f_lo + rr;
                if (feat >= p.k) continue;
                float tot = 0.0f;
                for (int src = 0; src < C; ++src) tot += recvf[(src * nfmax + rr) * MP + tok];
                p.gx[static_cast<int64_t>(tok) * p.k + feat] = __bfloat16_as_ushort(__float2bfloat16_rn(tot));
            }
        }
    }
}

template <int NG>
__global__ void __launch_bounds__(kThreads, 1)
k_decode_bwd(const __grid_constant__ CUtensorMap tm_codes, const __grid_constant__ CUtensorMap tm_g,
             const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_a,
             const __grid_constant__ CUtensorMap tm_b, const BwdArgs p) {
    extern __shared__ __align__(1024) uint8_t smem[];
    if (saddr(smem) & 1023u) {
        if (threadIdx.x == 0) record_error(p.err, kErrLayout);
        return;
    }
    if (p.r > 0 && blockIdx.y == 0) {
        adapter_body<NG>(&tm_g, &tm_b, p, smem);
    } else if ((saddr(smem) & 0x00ffffffu) == kDynSmemBase) {
        chunk_body<NG, true>(&tm_codes, &tm_g, &tm_q, &tm_a, p, smem);
    } else {
        chunk_body<NG, false>(&tm_codes, &tm_g, &tm_q, &tm_a, p, smem);
    }
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

bool encode(CUtensorMap *m, CUtensorMapDataType dt, int rank, const void *base, const uint64_t *dims,
            const uint64_t *strides, const uint32_t *box, CUtensorMapSwizzle sw) {
    auto fn = encode_fn();
    if (!fn) return false;
    cuuint64_t d[3], st[2];
    cuuint32_t b[3], es[3] = {1, 1, 1};
    for (int i = 0; i < rank; ++i) {
        d[i] = dims[i];
        b[i] = box[i];
        if (i + 1 < rank) st[i] = strides[i];
    }
    return fn(m, dt, static_cast<cuuint32_t>(rank), const_cast<void *>(base), d, st, b, es,
              CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int round_rank(int r) { return r <= 0 ? 0 : r <= 8 ? 8 : r <= 16 ? 16 : r <= 32 ? 32 : 64; }
uint32_t align_up(uint32_t v, uint32_t a) { return (v + a - 1) / a * a; }

bool layout(BwdArgs &a, int MP) {
    const uint32_t codes = kSR * 128u;
    const uint32_t gb = 2u * MP * 128u;  // two 64-row boxes
    // FP8 codes: one 16-byte chunk per row; fp32 constants: two
    const uint32_t qb = kSR * (a.absmax ? 32u : 16u);
    // a stage's scales: from an aligned index <= 3 below the first to the last, at most
    // (127 nbr + 3) / 256 + 1 apart, in whole 16-byte chunks (none with fp32 constants)
    a.s_cap = a.absmax ? 0 : static_cast<int>(static_cast<int64_t>(kSR) * a.nbr / 256 + 12);
    const uint32_t sb = align_up(static_cast<uint32_t>(a.s_cap) * 4u, 128);
    const uint32_t bb = a.r > 0 ? kSR * 2u * a.rpad : 0u;
    a.g_off = codes;
    a.q_off = codes + gb;
    a.s_off = a.q_off + qb;
    a.b_off = align_up(gb, 1024);
    const uint32_t chunk_slot = a.s_off + sb;
    const uint32_t adapter_slot = a.b_off + bb;
    a.slot_bytes = align_up(chunk_slot > adapter_slot ? chunk_slot : adapter_slot, 1024);
    a.codes_bytes = codes;
    a.g_bytes = gb;
    a.q_bytes = qb;
    a.gb_bytes = bb;
    const uint32_t utb = a.r > 0 ? align_up(static_cast<uint32_t>(MP * a.rk16 * 2), 128) : 0u;
    const int nablk_max = a.r > 0 ? (4 + a.C - 1) / a.C : 0;
    const uint32_t atb = static_cast<uint32_t>(nablk_max * a.rpad * 128);
    const uint32_t post_chunk = 4 * 4 * 4 * 32 * 16 * (MP / 8);
    const uint32_t post_adapter = 64 * 32 * 16;
    const uint32_t post = post_chunk > post_adapter ? post_chunk : post_adapter;
    const uint32_t recv_chunk = a.C > 1 ? static_cast<uint32_t>(a.C * ((kChunkFeat + a.C - 1) / a.C) * MP * 4) : 0u;
    const uint32_t recv_adapter = a.r > 0 ? static_cast<uint32_t>(a.C * MP * a.rpad * 4) : 0u;
    const uint32_t recv = align_up(recv_chunk > recv_adapter ? recv_chunk : recv_adapter, 128);
    const uint32_t bars = 256;
    const uint64_t fixed = static_cast<uint64_t>(kLutBytes) + align_up(atb, 1024) + utb + recv + bars + 1024;
    if (fixed + a.slot_bytes > kSmemLimit) return false;
    const int nsmax = (a.nrs + a.C - 1) / a.C;
    int stages = static_cast<int>((kSmemLimit - fixed) / a.slot_bytes);
    if (stages > kMaxStages) stages = kMaxStages;
    if (stages > nsmax) stages = nsmax;
    const int need = nsmax < 2 ? nsmax : 2;
    if (stages < need) return false;
    uint32_t ring = static_cast<uint32_t>(stages) * a.slot_bytes;
    bool post_in_ring = ring >= post;
    if (!post_in_ring && fixed + ring + post > kSmemLimit) {
        stages = static_cast<int>((kSmemLimit - fixed - post) / a.slot_bytes);
        if (stages < need) return false;
        ring = static_cast<uint32_t>(stages) * a.slot_bytes;
        post_in_ring = ring >= post;
    }
    a.stages = stages;
    a.ring_off = kLutBytes;
    uint32_t off = a.ring_off + ring;
    if (post_in_ring) {
        a.post_off = a.ring_off;
    } else {
        a.post_off = off;
        off += align_up(post, 128);
    }
    a.at_off = align_up(off, 1024);  // 128-byte-swizzled boxes
    off = a.at_off + align_up(atb, 1024);
    a.ut_off = off;
    off += utb;
    a.recv_off = off;
    off += recv;
    a.bar_off = off;
    return static_cast<uint64_t>(off) + bars <= kSmemLimit;
}

size_t smem_bytes(const BwdArgs &a) { return static_cast<size_t>(a.bar_off) + 256; }

template <int NG>
cudaError_t launch_ng(const WeightView &w, const uint16_t *gh, int M, const uint16_t *A, const uint16_t *B, int r,
                      float s, const DropoutArgs &drop, uint16_t *gx, int *err, cudaStream_t st) {
    constexpr int MP = 8 * NG;
    const void *kern = reinterpret_cast<const void *>(k_decode_bwd<NG>);
    int sms = 148;
    cudaError_t e = device_sm_count(&sms);
    if (e != cudaSuccess) return e;
    BwdArgs a = {};
    a.q = w.q;
    a.sigma = w.sigma;
    a.mu = w.mu;
    a.absmax = w.absmax;
    a.qtype = w.qtype;
    a.gx = gx;
    a.err = err;
    char *wsb = reinterpret_cast<char *>(err);
    a.flag = reinterpret_cast<unsigned *>(wsb + kWsFlag);
    a.readers = reinterpret_cast<unsigned *>(wsb + kWsReaders);
    a.u_ws = reinterpret_cast<uint16_t *>(wsb + kWsU);
    a.n = w.n;
    a.k = w.k;
    a.nbr = static_cast<int>(w.k / kBlock);
    a.nrs = static_cast<int>((w.n + kSR - 1) / kSR);
    a.chunks = static_cast<int>((w.k + kChunkFeat - 1) / kChunkFeat);
    a.M = M;
    a.r = r;
    a.rpad = round_rank(r);
    a.rk16 = (a.rpad + 15) & ~15;
    a.s = s;
    a.drop = drop;
    a.q_tma = (a.nbr % 16) == 0 && !w.absmax ? 1 : 0;
    const int extra = r > 0 ? 1 : 0;
    // cluster size: the largest C <= 8 with (chunks + 1) x C <= SMs, every cluster resident and
    // at least one row stage per CTA
    bool found = false;
    for (int C = kMaxCluster; C >= 1; --C) {
        if (static_cast<int64_t>(a.chunks + extra) * C > sms || C > a.nrs) continue;
        BwdArgs c = a;
        c.C = C;
        if (!layout(c, MP)) continue;
        if (C > 1) {
            int nc = 0;
            e = resident_clusters(kern, kThreads, C, smem_bytes(c), &nc);
            if (e != cudaSuccess) return e;
            if (nc < c.chunks + extra) continue;
        }
        a = c;
        found = true;
        break;
    }
    if (!found) return cudaErrorInvalidConfiguration;
    const size_t smem = smem_bytes(a);

    CUtensorMap tm_codes, tm_g, tm_q, tm_a, tm_b;
    {
        const uint64_t dims[2] = {static_cast<uint64_t>(w.k / 2), static_cast<uint64_t>(w.n)};
        const uint64_t strides[1] = {static_cast<uint64_t>(w.k / 2)};
        const uint32_t box[2] = {128, kSR};
        if (!encode(&tm_codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, w.codes, dims, strides, box,
                    CU_TENSOR_MAP_SWIZZLE_128B))
            return cudaErrorInvalidValue;
    }
    {
        const uint64_t dims[2] = {static_cast<uint64_t>(w.n), static_cast<uint64_t>(M)};
        const uint64_t strides[1] = {static_cast<uint64_t>(w.n) * 2};
        const uint32_t box[2] = {64, static_cast<uint32_t>(MP)};
        if (!encode(&tm_g, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, gh, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B))
            return cudaErrorInvalidValue;
    }
    tm_q = tm_codes;
    if (a.q_tma) {
        const uint64_t dims[2] = {static_cast<uint64_t>(a.nbr), static_cast<uint64_t>(w.n)};
        const uint64_t strides[1] = {static_cast<uint64_t>(a.nbr)};
        const uint32_t box[2] = {16, kSR};
        if (!encode(&tm_q, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, w.q, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_NONE))
            return cudaErrorInvalidValue;
    }
    tm_a = tm_codes;
    tm_b = tm_codes;
    if (r > 0) {
        const uint64_t dims[3] = {64, static_cast<uint64_t>(r), static_cast<uint64_t>(w.k / 64)};
        const uint64_t strides[2] = {static_cast<uint64_t>(w.k) * 2, 128};
        const uint32_t box[3] = {64, static_cast<uint32_t>(a.rpad), 1};
        if (!encode(&tm_a, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, A, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B))
            return cudaErrorInvalidValue;
        const uint64_t bdims[2] = {static_cast<uint64_t>(r), static_cast<uint64_t>(w.n)};
        const uint64_t bstrides[1] = {static_cast<uint64_t>(r) * 2};
        const uint32_t bbox[2] = {static_cast<uint32_t>(a.rpad), kSR};
        const CUtensorMapSwizzle sw = a.rpad == 64   ? CU_TENSOR_MAP_SWIZZLE_128B
                                      : a.rpad == 32 ? CU_TENSOR_MAP_SWIZZLE_64B
                                      : a.rpad == 16 ? CU_TENSOR_MAP_SWIZZLE_32B
                                                     : CU_TENSOR_MAP_SWIZZLE_NONE;
        if (!encode(&tm_b, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, B, bdims, bstrides, bbox, sw))
            return cudaErrorInvalidValue;
    }
    e = ensure_smem_limit(kern, smem);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(a.C), static_cast<unsigned>(a.chunks + extra), 1);
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
    e = cudaLaunchKernelEx(&cfg, k_decode_bwd<NG>, tm_codes, tm_g, tm_q, tm_a, tm_b, a);
    count_launch();
    return e;
}

}  // namespace

bool decode_bwd_stream_supported(int64_t n, int64_t k, int r) {
    return n % 8 == 0 && (r == 0 || r % 8 == 0) && (k + kChunkFeat - 1) / kChunkFeat + (r > 0 ? 1 : 0) <= 148;
}

cudaError_t launch_decode_bwd_stream(const WeightView &w, const uint16_t *gh, int M, const uint16_t *A,
                                     const uint16_t *B, int r, float s, const DropoutArgs &drop, uint16_t *gx,
                                     int *err, cudaStream_t st) {
    if (M <= 0 || w.k == 0) return cudaSuccess;
    if (M > kDecodeTokens || r > kDecodeMaxRank || !decode_bwd_stream_supported(w.n, w.k, r))
        return cudaErrorInvalidValue;
    if (M <= 8) return launch_ng<1>(w, gh, M, A, B, r, s, drop, gx, err, st);
    return launch_ng<2>(w, gh, M, A, B, r, s, drop, gx, err, st);
}

}  // namespace qn
