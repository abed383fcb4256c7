// decode_fwd.cu -- QLoRA linear forward for few tokens (M <= 16 per launch) on sm_100a.
//
//   h[m,n] = sum_k W'[n,k] x[m,k] + sum_j B[n,j] t[m,j],  t = bf16(s A x),  W'[n,k] = NF4[code] * c'_b
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
// fills the SMs and each CTA moves the fewest bytes; chunks of 128 rows run the k_decode_fwd<NG, 2>
// instantiation, every other R k_decode_fwd<NG, 0>). The CTA streams its (R rows x K-slice) codes
// through a ring of stages: a stage is R rows x 4 blocks (one TMA box, 128-byte swizzled so that
// the 8-byte reads of eight rows hit eight different bank groups). x of the whole K-slice
// ([stage][block][token][64 values], same swizzle) and the FP8 block codes and group scales of
// the slice are staged once, by the consumers' 16-byte cp.async copies.
//   warp 0      : producer (one lane issues the code boxes; all lanes stage the rows of B the CTA
//                 finalises, copy t, and compute B t of those rows on the tensor cores).
//   warps 1..16 : consumers. Warp (kg, rg) takes block kg of every stage and the m-tiles
//                 rg, rg + 4, ... of the chunk: codes -> pair table -> mma.sync with x, one fp32
//                 fragment per block scaled by c'_b = fma(e4m3(q_b), sigma_g, mu) into the
//                 accumulators (the four lanes of a quad compute the constants the quad needs and
//                 share them by shuffles). In <NG, 2> a warp runs both of its m-tiles at once.
// The adapter down-projection t = bf16(s A x) is computed once per call by one more cluster (the
// first row of the grid, so that it is dispatched first): its CTAs stream x and A over the same
// K-slices, reduce their partial sums into rank 0 (DSMEM), and rank 0 publishes t in the
// workspace and raises a flag. The other CTAs' producers wait for the flag after their last stage
// and copy t to shared memory; the last of them to do so lowers the flag again for the next call.
// After the loop the four block-warps of each m-tile are summed in a fixed order (kg = 0..3), each
// m-tile by one warp. With C > 1 the sums go by asynchronous DSMEM stores to the CTA of the
// cluster that finalises those rows, which waits on its own mbarrier for the bytes, sums the
// slices in rank order, adds B t and stores h; with C == 1 the summing warps add B t on the
// tensor cores and store h. Results are bit-reproducible.
//
// Programmatic launch: the packed weight (codes, FP8 codes, group scales) is requested BEFORE the
// dependency wait, so the first stages of the ring fill while the preceding kernel finishes; x,
// A and B are read, and h written, only after it. With x staged once, only two code stages are
// requested before the wait and the rest once x has landed: the x copies would otherwise queue
// behind every code request in flight. The caller guarantees that the preceding
// kernel on the stream, if it signals its dependents early, does not write the packed weight
// (no kernel of this library that signals early writes one). The codes are read with an L2
// evict-first policy: they are used once, and the activations and adapters should stay cached.
//
// Every wait is bounded; a timeout records an error code in the workspace error word, stops the
// CTA's work and drains the loads already issued.
#include <cudaTypedefs.h>

#include "dropout.cuh"
#include "host_cache.h"
#include "stream_common.cuh"

namespace qn {

#ifdef QN_TIMELINE
// Per-CTA timestamps (globaltimer, ns) of the forward kernel's phases, for profiling builds only.
// Two buffers, used by alternate launches, so that a chain's last two launches can be compared.
// Slots 0 and 1 (start, past the wait): globaltimer (ns); the other slots: SM cycles since the
// marking thread entered the kernel (clock64: one counter per SM, exact within a CTA).
__device__ unsigned long long g_fwd_timeline[2][1024][24];
__device__ __forceinline__ void tl_mark(int buf, int slot, long long c0) {
    const unsigned cta = blockIdx.y * gridDim.x + blockIdx.x;
    if (cta >= 1024) return;
    unsigned long long t;
    if (slot <= 1) {
        asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    } else {
        t = static_cast<unsigned long long>(clock64() - c0);
    }
    g_fwd_timeline[buf & 1][cta][slot] = t;
}
#define QN_TL(slot, cond) \
    do {                  \
        if (cond) tl_mark(p.tl_buf, slot, tl_c0); \
    } while (0)
static int g_last_plan[6];  // R, C, stages, chunks, shared bytes, bytes of the busiest CTA (KB)
static int g_launches_tl = 0;
__device__ int g_fwd_smid[2][1024];
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
constexpr int kPreWaitStages = 2;  // code stages requested before the dependency wait when x is staged once
constexpr int kMaxCluster = 8;
constexpr size_t kSmemLimit = 227 * 1024;

// Workspace of the few-token path: error word, t-ready flag, reader count, t.
constexpr size_t kWsFlag = 64, kWsReaders = 128, kWsT = 256;

struct FwdArgs {
    const uint8_t *q;
    const float *sigma;
    const float *mu;
    const float *absmax;  // fp32 block constants (no double quantisation), else nullptr
    int qtype;            // table of the code nibbles
    const uint16_t *B;  // n x r
    const uint16_t *x;  // M x k (the chunk CTAs' stage copies)
    uint16_t *h;        // M x n
    int *err;
    uint16_t *t_ws;     // [MP][rk16] bf16: bf16(s A x), published by the adapter cluster
    unsigned *flag;     // 1 while t_ws holds this call's t
    unsigned *readers;  // CTAs that have copied t_ws
    int64_t n, k;
    int64_t row_lo, row_hi;  // rows of W this launch covers (chunk c: row_lo + c R ..)
    int nbr;     // blocks per row (k / 64)
    int ncol;    // stage columns (ceil(nbr / 4))
    int M, r, rpad, rk16;  // rpad: r rounded up to 8, 16, 32 or 64; rk16: to 16 (0 without adapter)
    float s;     // adapter scale (divided by 1 - p under dropout)
    DropoutArgs drop;  // mask of the adapter's input x (thr == 0: none); offset of this launch's token 0
    int R, m;    // rows and m-tiles per chunk
    int C;       // K-slices (cluster size)
    int chunks;  // row chunks: grid rows 1 .. chunks when r > 0 (row 0 is the adapter cluster), else 0 .. chunks - 1
    int stages;
    int evict_first;  // the codes are read with an L2 evict-first policy
    // shared-memory layout (byte offsets from the start of dynamic shared memory)
    uint32_t slot_bytes, x_off;  // chunk CTAs: codes [R][128 B], x [4][M][128 B] at x_off (x_once == 0)
    int x_once;                  // chunk CTAs stage the x of every stage once, after the dependency wait
    uint32_t xs_off, xs_stage;   // ... at xs_off, xs_stage bytes per stage ([4][M][128 B])
    uint32_t a_off;              // adapter CTAs: x [4][MP][128 B] at 0, A [4][rpad][128 B] at a_off
    uint32_t ring_off, qs_off, ss_off, tb_off, bs_off, recv_off, bt_off, bar_off, post_off;
    uint32_t qs_stride;  // bytes per chunk row of the staged FP8 codes (or fp32 constants)
    uint32_t bs_stride;  // bytes per staged row of B
    uint32_t codes_bytes, x_bytes, xa_bytes;  // transaction bytes: codes box; x box; adapter x + A boxes
#ifdef QN_TIMELINE
    int tl_buf;
#endif
};

// Barrier block: full[kMaxStages], empty[kMaxStages], consts, recv, tready, abort flag.
struct Bars {
    uint64_t *full, *empty, *consts, *recv, *tready, *xready;
    volatile uint32_t *abort_flag;
};

__device__ __forceinline__ Bars bars_of(uint8_t *smem, const FwdArgs &p) {
    Bars b;
    b.full = reinterpret_cast<uint64_t *>(smem + p.bar_off);
    b.empty = b.full + kMaxStages;
    b.consts = b.empty + kMaxStages;
    b.recv = b.consts + 1;
    b.tready = b.recv + 1;
    b.xready = b.tready + 1;
    b.abort_flag = reinterpret_cast<volatile uint32_t *>(b.xready + 1);
    return b;
}

// ------------------------------------------------------------------------------ adapter cluster
// t_c = A x over this CTA's K-slice (mma.sync, the 16 consumer warps split the stage's (rank
// tile, k16 step) jobs), summed into rank 0, which publishes bf16(s t).
template <int NG>
__device__ __forceinline__ void adapter_body(const CUtensorMap *tm_xp, const CUtensorMap *tm_a, const FwdArgs &p,
                                             uint8_t *smem) {
    constexpr int MP = 8 * NG;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, t = lane & 3;
    const int C = p.C;
    const int crank = C > 1 ? static_cast<int>(cg::this_cluster().block_rank()) : 0;
    const int col_lo = p.ncol * crank / C, col_hi = p.ncol * (crank + 1) / C;
    const int ns = col_hi - col_lo;
    const int S = p.stages;
    const uint32_t s_base = saddr(smem);
    const uint32_t s_ring = s_base + p.ring_off;
    const Bars bb = bars_of(smem, p);
    const uint32_t recv_bytes = static_cast<uint32_t>(C * MP * p.rpad * 4);

    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(&bb.full[s], 1);
            mbar_init(&bb.empty[s], kConsumers);
        }
        mbar_init(bb.recv, 1);
        if (C > 1 && crank == 0) mbar_arrive_expect_tx(bb.recv, recv_bytes);
        *bb.abort_flag = 0u;
        fence_barrier_init();
        tma_prefetch_desc(tm_xp);
        tma_prefetch_desc(tm_a);
    }
    __syncthreads();
    if (C > 1) cluster_arrive_relaxed();  // phase 1: this CTA runs (its shared memory may be written)
    grid_dependents_launch();
    grid_dependency_wait();  // x and A may come from the preceding kernel

    auto fail = [&]() {
        if (atomicExch(const_cast<uint32_t *>(bb.abort_flag), 1u) == 0u) record_error(p.err, kErrTimeout);
    };
    const int cw = warp - 1;
    float tacc[4] = {0.0f, 0.0f, 0.0f, 0.0f};
    const int NT = p.rpad / 8;  // rank tiles of 8 (1, 2, 4 or 8); 16 NT jobs per stage
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
                mbar_arrive_expect_tx(&bb.full[slot], p.xa_bytes);
                const uint32_t sl = s_ring + static_cast<uint32_t>(slot) * p.slot_bytes;
                tma_load_3d_saddr(sl, tm_xp, &bb.full[slot], 0, 0, 4 * (col_lo + s));
                tma_load_3d_saddr(sl + p.a_off, tm_a, &bb.full[slot], 0, 0, 4 * (col_lo + s));
                ni = s + 1;
            }
            for (int s = (ni > S ? ni - S : 0); s < ni; ++s) mbar_wait(&bb.full[s % S], (s / S) & 1);
        }
        __syncwarp();
    } else {
        const int nt_job = cw % NT;
        const int kq_step = 16 / NT;
        const int kq0 = cw / NT;
        const int jrow = nt_job * 8 + g;  // rank row of this lane's B fragment
        for (int s = 0; s < ns; ++s) {
            const int slot = s % S;
            // every lane waits for the stage; the warp leaves together (mma.sync and shuffles below)
            const bool ok = !*bb.abort_flag && mbar_wait(&bb.full[slot], (s / S) & 1);
            if (!__all_sync(0xffffffffu, ok)) {
                if (!ok) fail();
                break;
            }
            const uint32_t sl = s_ring + static_cast<uint32_t>(slot) * p.slot_bytes;
            if (p.drop.thr != 0u) {
                // LoRA dropout: zero the dropped elements of the stage's x box in place, one
                // 16-byte chunk (8 elements of one token row) per consumer thread
                const int items = kStageBlocks * p.M * 8;
                for (int i = threadIdx.x - 32; i < items; i += kConsumers * 32) {
                    const int blk = i / (p.M * 8), rem = i - blk * (p.M * 8), tok = rem >> 3, c = rem & 7;
                    const int64_t kk0 = static_cast<int64_t>(4 * (col_lo + s) + blk) * 64 + 8 * c;
                    if (kk0 >= p.k) continue;
                    const uint32_t a = sl + static_cast<uint32_t>(blk * MP * 128 + tok * 128 + ((c ^ (tok & 7)) << 4));
                    const uint32_t keep =
                        dropout_keep_bits(p.drop, p.drop.offset + static_cast<uint64_t>(tok * p.k + kk0), 8);
                    uint4 v = lds128(a);
                    v.x = mask_pair(v.x, keep);
                    v.y = mask_pair(v.y, keep >> 2);
                    v.z = mask_pair(v.z, keep >> 4);
                    v.w = mask_pair(v.w, keep >> 6);
                    asm volatile("st.shared.v4.b32 [%0], {%1,%2,%3,%4};" ::"r"(a), "r"(v.x), "r"(v.y), "r"(v.z),
                                 "r"(v.w)
                                 : "memory");
                }
                // these writes precede the TMA that refills the slot (async proxy)
                fence_proxy_async_smem();
                named_sync(4, kConsumers * 32);
            }
            for (int j = 0; j < NT; ++j) {
                const int kq = kq0 + kq_step * j;
                const int blk = kq >> 2, q4 = kq & 3;
                const uint32_t xa = sl + blk * MP * 128;
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
            if (lane == 0) mbar_arrive(&bb.empty[slot]);
        }
    }
    __syncthreads();
    // Per-CTA sum of the rank tiles (warps cw, cw + NT, ... in that order) into rank 0's
    // receive buffer [src][MP tokens][rpad] fp32.
    const uint32_t tbuf = s_base + p.post_off;  // [16 warps][32 lanes][4] f32, in the idle ring
    if (warp > 0)
        asm volatile("st.shared.v4.f32 [%0], {%1,%2,%3,%4};" ::"r"(tbuf + static_cast<uint32_t>(cw * 32 + lane) * 16),
                     "f"(tacc[0]), "f"(tacc[1]), "f"(tacc[2]), "f"(tacc[3])
                     : "memory");
    __syncthreads();
    const uint32_t recv = s_base + p.recv_off;
    if (C > 1) cluster_wait();  // phase 1: every CTA of the cluster runs
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
        const uint32_t o0 = recv + static_cast<uint32_t>(((crank * MP + g) * p.rpad + j) * 4);
        const uint32_t o1 = recv + static_cast<uint32_t>(((crank * MP + g + 8) * p.rpad + j) * 4);
        if (C > 1) {
            const uint32_t bar = mapa(saddr(bb.recv), 0);
            st_async_v2(mapa(o0, 0), tt[0], tt[1], bar);
            if (NG > 1) st_async_v2(mapa(o1, 0), tt[2], tt[3], bar);
        } else {
            asm volatile("st.shared.v2.f32 [%0], {%1,%2};" ::"r"(o0), "f"(tt[0]), "f"(tt[1]) : "memory");
            if (NG > 1) asm volatile("st.shared.v2.f32 [%0], {%1,%2};" ::"r"(o1), "f"(tt[2]), "f"(tt[3]) : "memory");
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
    // t = bf16(s t) in rank order, [MP tokens][rk16] with zeros past rpad
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
        reinterpret_cast<uint32_t *>(p.t_ws)[i] = pack_bf16x2(p.s * v0, p.s * v1);
    }
    __syncthreads();
    if (threadIdx.x == 0 && ok && !*bb.abort_flag) {
        __threadfence();
        st_release_u32(p.flag, 1u);
    }
}

// ------------------------------------------------------------------------------ chunk clusters
// kMT: the m-tiles of every consumer warp (m = 4 kMT), fixed at compile time so that the tile
// loop has no branches (2: chunks of 128 rows); 0: up to MW, each checked against m.
template <int NG, bool kFixedBase, int kMT>
__device__ __forceinline__ void chunk_body(const CUtensorMap *tm_codes, const CUtensorMap *tm_x, const FwdArgs &p,
                                           uint8_t *smem) {
    constexpr int MP = 8 * NG;  // padded tokens
    constexpr int MW = 4;  // m-tiles per warp at most (m <= 4 MW)
    constexpr int MWL = kMT > 0 ? kMT : MW;  // m-tiles the stage loop visits
#ifdef QN_TIMELINE
    const long long tl_c0 = clock64();
#endif
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, t = lane & 3;
    const int C = p.C;
    const int crank = C > 1 ? static_cast<int>(cg::this_cluster().block_rank()) : 0;
    const int chunk = static_cast<int>(blockIdx.y) - (p.r > 0 ? 1 : 0);
    const int64_t row0 = p.row_lo + static_cast<int64_t>(chunk) * p.R;
    const int64_t nrow = p.row_hi;  // rows at or past nrow are not this launch's
    const int col_lo = p.ncol * crank / C, col_hi = p.ncol * (crank + 1) / C;
    const int ns = col_hi - col_lo;
    const int S = p.stages;
    // Stages whose codes are requested before the dependency wait. With x staged once, at most
    // kPreWaitStages: the x copies issued after the wait queue behind every request in flight, and
    // the remaining stages are requested only once x has landed.
    const int npre_all = ns < S ? ns : S;
    const int npre = p.x_once && npre_all > kPreWaitStages ? kPreWaitStages : npre_all;
    // rows [r_lo, r_hi) of the chunk are finalised by this CTA (C > 1)
    const int r_lo = p.R * crank / C, r_hi = p.R * (crank + 1) / C, nr = r_hi - r_lo;
    const int nrmax = (p.R + C - 1) / C;

    uint8_t *lut = smem;
    const uint32_t s_base = saddr(smem);
    const uint32_t s_ring = s_base + p.ring_off;
    const uint32_t s_qs = s_base + p.qs_off;
    const uint32_t s_ss = s_base + p.ss_off;
    const uint32_t s_xs = s_base + p.xs_off;  // x of every stage (x_once)
    const uint32_t tb = s_base + p.tb_off;  // [MP tokens][rk16] bf16 t
    const uint32_t bs = s_base + p.bs_off;  // [rows r_lo .. r_hi of the chunk][bs_stride] B rows
    const Bars bb = bars_of(smem, p);
    // the staged group scales start at index s_lo (that of the chunk's first block of the slice)
    const int64_t s_lo = (row0 * p.nbr + 4 * col_lo) >> 8;

    auto load_codes = [&](int s, uint64_t pol) {
        const int slot = s % S;
        const uint32_t dst = s_ring + static_cast<uint32_t>(slot) * p.slot_bytes;
        const int32_t c0 = (col_lo + s) * 128, c1 = static_cast<int32_t>(row0);
        if (p.evict_first)
            tma_load_2d_saddr_hint(dst, tm_codes, &bb.full[slot], c0, c1, pol);
        else
            tma_load_2d_saddr(dst, tm_codes, &bb.full[slot], c0, c1);
    };

    QN_TL(0, threadIdx.x == 0);
#ifdef QN_TIMELINE
    if (threadIdx.x == 0) {
        unsigned sm;
        asm volatile("mov.u32 %0, %%smid;" : "=r"(sm));
        const unsigned cta = blockIdx.y * gridDim.x + blockIdx.x;
        if (cta < 1024) g_fwd_smid[p.tl_buf & 1][cta] = static_cast<int>(sm);
    }
#endif
    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            // codes by bytes; one arrival, plus the producer lanes' x copies when x comes per stage
            mbar_init(&bb.full[s], p.x_once ? 1 : 33);
            mbar_init(&bb.empty[s], kConsumers);
        }
        mbar_init(bb.consts, kConsumers * 32);  // one cp.async arrival per consumer thread
        mbar_init(bb.recv, 1);
        if (C > 1) mbar_arrive_expect_tx(bb.recv, static_cast<uint32_t>(C * nr * MP * 4));
        mbar_init(bb.tready, 1);  // the producer: t and the B rows are in shared memory
        mbar_init(bb.xready, kConsumers * 32);  // one cp.async arrival per consumer thread: x has landed
        *bb.abort_flag = 0u;
        fence_barrier_init();
    }
    __syncthreads();  // barriers initialised
    float mu_pre = 0.0f;  // the weight's mean (consumers), read before the dependency wait
    if (warp == 0) {
        // ------------------------------------------ producer, before the dependency wait: weights
        if (lane == 0) {
            tma_prefetch_desc(tm_codes);
            const uint64_t pol = l2_policy_evict_first();
            for (int s = 0; s < npre; ++s) {
                // with x staged once, the stage is complete when its codes land: arm it now
                if (p.x_once)
                    mbar_arrive_expect_tx(&bb.full[s], p.codes_bytes);
                else
                    mbar_expect_tx(&bb.full[s], p.codes_bytes);
                load_codes(s, pol);
            }
        }
        __syncwarp();
        QN_TL(14, lane == 0);
    } else {
        // ------------------------------------------ consumers, before the wait: constants, table
        // FP8 codes of the slice: chunk row i holds the 16-byte aligned chunks from the one that
        // contains block 4 col_lo of that row on; the group scales of every block of the chunk
        // rows from the slice's first to its last, in whole 16-byte chunks. Bytes past the arrays
        // read as zero. With fp32 constants, chunk row i holds them (4 per chunk) instead.
        const int ct = threadIdx.x - 32;
        mu_pre = load_mu(p.mu, p.absmax);
        if (p.absmax) {
            const int64_t nbq = p.n * p.nbr;
            const int nch = static_cast<int>(p.qs_stride >> 4);
            for (int it = ct; it < p.R * nch; it += kConsumers * 32) {
                const int i = it / nch, c = it - (it / nch) * nch;
                const int64_t row = row0 + i;
                const int64_t cb = (((row < nrow ? row : row0) * p.nbr + 4 * col_lo) >> 2) + c;  // 16-byte chunk
                const int64_t avail = row < nrow ? 4 * (nbq - 4 * cb) : 0;
                const uint32_t bytes = avail >= 16 ? 16u : (avail > 0 ? static_cast<uint32_t>(avail) : 0u);
                cp_async16_zfill(s_qs + static_cast<uint32_t>(i) * p.qs_stride + 16u * c,
                                 p.absmax + (bytes ? 4 * cb : 0), bytes);
            }
        } else {
            const int64_t nbq = p.n * p.nbr;
            const int nch = static_cast<int>(p.qs_stride >> 4);
            const int items = p.R * nch;
            for (int it = ct; it < items; it += kConsumers * 32) {
                const int i = it / nch, c = it - (it / nch) * nch;
                const int64_t row = row0 + i;
                const int64_t cb = (((row < nrow ? row : row0) * p.nbr + 4 * col_lo) >> 4) + c;  // 16-byte chunk
                const int64_t avail = row < nrow ? nbq - 16 * cb : 0;
                const uint32_t bytes = avail >= 16 ? 16u : (avail > 0 ? static_cast<uint32_t>(avail) : 0u);
                cp_async16_zfill(s_qs + static_cast<uint32_t>(i) * p.qs_stride + 16u * c, p.q + (bytes ? 16 * cb : 0),
                                 bytes);
            }
            const int64_t ngs = (nbq + kGroup - 1) / kGroup;
            const int64_t rend = row0 + p.R < nrow ? row0 + p.R : nrow;
            const int64_t bend = 4 * col_hi < p.nbr ? 4 * col_hi : p.nbr;
            const int64_t s_hi = ((rend - 1) * p.nbr + bend - 1) >> 8;
            const int scnt = static_cast<int>((s_hi >> 2) - (s_lo >> 2) + 1);  // 16-byte chunks
            for (int c = ct; c < scnt; c += kConsumers * 32) {
                const int64_t f = ((s_lo >> 2) + c) * 4;  // first float of the chunk
                const int64_t avail = 4 * (ngs - f);
                const uint32_t bytes = avail >= 16 ? 16u : (avail > 0 ? static_cast<uint32_t>(avail) : 0u);
                cp_async16_zfill(s_ss + 16u * c, p.sigma + (bytes ? f : 0), bytes);
            }
        }
        cp_async_arrive_noinc(bb.consts);
        QN_TL(8, ct == 0);
    }
    if (C > 1) cluster_arrive_relaxed();  // phase 1: this CTA runs (its shared memory may be written)
    grid_dependents_launch();
    grid_dependency_wait();  // x, A and B may come from the preceding kernel; h may be read by it
    QN_TL(1, threadIdx.x == 0);

    auto fail = [&]() {
        if (atomicExch(const_cast<uint32_t *>(bb.abort_flag), 1u) == 0u) record_error(p.err, kErrTimeout);
    };

    const int cw = warp - 1;  // consumer index
    const int kg = cw & 3, rg = cw >> 2;
    float acc[MW][NG][4];
#pragma unroll
    for (int i = 0; i < MW; ++i)
#pragma unroll
        for (int tg = 0; tg < NG; ++tg) acc[i][tg][0] = acc[i][tg][1] = acc[i][tg][2] = acc[i][tg][3] = 0.0f;

    if (warp == 0) {
        // ------------------------------------------------------------------ producer
        // B rows r_lo .. r_hi of the chunk (all rows when C == 1), ranks 0 .. rk16 (zeros past r
        // and past the last row)
        auto stage_brows = [&]() {
            if (p.r == 0) return;
            const int cpr = p.rk16 / 8;  // 16-byte chunks per row
            const bool r8 = (p.r & 7) == 0;
            for (int i = lane; i < nr * cpr; i += 32) {
                const int rr = i / cpr, c = i - (i / cpr) * cpr;
                const int64_t row = row0 + r_lo + rr;
                const uint32_t dst = bs + static_cast<uint32_t>(rr) * p.bs_stride + 16u * c;
                if (r8) {
                    const bool v = row < nrow && 8 * c < p.r;
                    cp_async16_zfill(dst, v ? p.B + row * p.r + 8 * c : p.B, v ? 16u : 0u);
                } else {
                    uint32_t w[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int j = 8 * c + 2 * e;
                        const uint32_t lo = (row < nrow && j < p.r) ? ld_ro_u16(p.B + row * p.r + j) : 0u;
                        const uint32_t hi = (row < nrow && j + 1 < p.r) ? ld_ro_u16(p.B + row * p.r + j + 1) : 0u;
                        w[e] = lo | (hi << 16);
                    }
                    asm volatile("st.shared.v4.b32 [%0], {%1,%2,%3,%4};" ::"r"(dst), "r"(w[0]), "r"(w[1]), "r"(w[2]),
                                 "r"(w[3])
                                 : "memory");
                }
            }
        };
        int ni = 0;  // stages armed
        if (p.x_once) {
            // The stages requested before the wait were armed with their requests. Once x has
            // landed, lane 0 requests the next stages' codes, each when its slot is free.
            stage_brows();
            ni = npre;
            if (lane == 0) {
                const bool xok = npre >= ns || mbar_wait(bb.xready, 0);  // x first
                if (!xok) fail();
                for (int s = npre; xok && s < ns; ++s) {
                    const int slot = s % S;
                    if (*bb.abort_flag) break;
                    if (!mbar_wait(&bb.empty[slot], ((s / S) & 1) ^ 1)) {
                        fail();
                        break;
                    }
                    mbar_arrive_expect_tx(&bb.full[slot], p.codes_bytes);
                    load_codes(s, l2_policy_evict_first());
                    ni = s + 1;
                }
            }
            ni = __shfl_sync(0xffffffffu, ni, 0);
        } else {
            // Stage s: wait for its slot (from the second round on, then request its codes); arm
            // the full barrier (lane 0's arrival) and copy the stage's x. After the first round
            // is armed, stage the B rows.
            for (int s = 0; s < ns; ++s) {
                const int slot = s % S;
                // lane 0 decides (abort flag, slot wait) and the warp follows it as one
                bool ok = true;
                if (lane == 0) {
                    if (*bb.abort_flag) ok = false;
                    if (ok && s >= S) {
                        ok = mbar_wait(&bb.empty[slot], ((s / S) & 1) ^ 1);
                        if (!ok) fail();
                    }
                    if (ok && s >= npre) {
                        mbar_expect_tx(&bb.full[slot], p.codes_bytes);
                        load_codes(s, l2_policy_evict_first());
                    }
                    if (ok) mbar_arrive(&bb.full[slot]);
                }
                ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
                if (!ok) break;
                QN_TL(21, lane == 0 && s == 0);
                // x of the stage by the lanes' 16-byte copies (not TMA: these small loads must
                // not queue behind the code boxes): [block][token][64 values], 16-byte chunk c of
                // row b M + tok at c ^ (row & 7); blocks past the row read as zero
                {
                    const uint32_t sl = s_ring + static_cast<uint32_t>(slot) * p.slot_bytes + p.x_off;
                    const int items = kStageBlocks * p.M * 8;
                    for (int i = lane; i < items; i += 32) {
                        const int b = i / (p.M * 8), rem = i - b * (p.M * 8), tok = rem >> 3, c = rem & 7;
                        const int row = b * p.M + tok;
                        const int64_t kk = static_cast<int64_t>(4 * (col_lo + s) + b) * 64 + 8 * c;
                        const bool v = kk < p.k;
                        cp_async16_zfill(sl + static_cast<uint32_t>(row * 128 + ((c ^ (row & 7)) << 4)),
                                         v ? p.x + tok * p.k + kk : p.x, v ? 16u : 0u);
                    }
                    QN_TL(22, lane == 0 && s == 0);
                    cp_async_arrive_noinc(&bb.full[slot]);
                }
                QN_TL(16 + (s < 4 ? s : 3), lane == 0 && s < 4);
                ni = s + 1;
                QN_TL(2, lane == 0 && s == S - 1);
                if (s == npre - 1) stage_brows();
            }
        }
        // drain: in the per-stage mode, the stages whose codes were requested before the wait but
        // that were never armed get their 33 arrivals now; then every requested stage lands
        // before the CTA exits
        if (lane == 0) {
            if (!p.x_once)
                for (int s = ni; s < npre; ++s) mbar_arrive_cnt(&bb.full[s], 33);
            const int hi = ni > npre ? ni : npre;
            for (int s = (hi > S ? hi - S : 0); s < hi; ++s) mbar_wait(&bb.full[s % S], (s / S) & 1);
        }
        // t from the adapter cluster
        if (p.r > 0) {
            bool ok = true;
            if (lane == 0) ok = wait_flag(p.flag);
            ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
            if (!ok) {
                if (lane == 0) fail();
            } else {
                for (int i = lane; i < MP * p.rk16 / 2; i += 32)
                    asm volatile("st.shared.b32 [%0], %1;" ::"r"(tb + 4u * i), "r"(ld_cg_u32(p.t_ws + 2 * i))
                                 : "memory");
                __syncwarp();
                if (lane == 0) {
                    const unsigned old = atomicAdd(p.readers, 1u);
                    if (old == static_cast<unsigned>(p.chunks * C) - 1u) {
                        // every CTA has its copy: lower the flag for the next call
                        atomicExch(p.readers, 0u);
                        atomicExch(p.flag, 0u);
                    }
                }
            }
            QN_TL(12, lane == 0);
        }
        cp_async_wait_all();  // the B rows
        __syncwarp();
        if (C > 1 && p.r > 0 && !*bb.abort_flag) {
            // B t of the rows this CTA finalises, [nrmax][MP] fp32, while the consumers reduce:
            // 16-row tiles of the staged B rows times t on the tensor cores
            float *btf = reinterpret_cast<float *>(smem + p.bt_off);
            for (int rt = 0; rt < nr; rt += 16) {
                const int rA = min(rt + g, nr - 1), rB = min(rt + g + 8, nr - 1);
                float d[NG][4];
#pragma unroll
                for (int tg = 0; tg < NG; ++tg) d[tg][0] = d[tg][1] = d[tg][2] = d[tg][3] = 0.0f;
                for (int kc = 0; kc < p.rk16 / 16; ++kc) {
                    const uint32_t j2 = static_cast<uint32_t>(16 * kc + 2 * t) * 2u;
                    const uint32_t ba = bs + static_cast<uint32_t>(rA) * p.bs_stride + j2;
                    const uint32_t bb2 = bs + static_cast<uint32_t>(rB) * p.bs_stride + j2;
                    const uint32_t a0 = lds32(ba), a2 = lds32(ba + 16), a1 = lds32(bb2), a3 = lds32(bb2 + 16);
#pragma unroll
                    for (int tg = 0; tg < NG; ++tg) {
                        const uint32_t tr = tb + static_cast<uint32_t>((tg * 8 + g) * p.rk16) * 2u + j2;
                        mma_16816(d[tg], a0, a1, a2, a3, lds32(tr), lds32(tr + 16));
                    }
                }
#pragma unroll
                for (int tg = 0; tg < NG; ++tg)
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int row = rt + g + 8 * (e >> 1), tok = tg * 8 + 2 * t + (e & 1);
                        if (row < nr) btf[row * MP + tok] = d[tg][e];
                    }
            }
            __syncwarp();
        }
        if (lane == 0) mbar_arrive(bb.tready);
        if (C > 1) cluster_wait();  // phase 1 (every thread waits once)
    } else {
        // ------------------------------------------------------------------ consumers
        // Right after the dependency wait the x copies are issued; the pair table is built while
        // they are in flight. Their landing (one cp.async arrival per thread on xready) releases the
        // producer's requests for the code stages past the first kPreWaitStages.
        const int ct = threadIdx.x - 32;
        if (p.x_once) {
            // x of every stage of the slice, [stage][block][token][64 values] with 16-byte chunk c
            // of row b M + tok at c ^ (row & 7); blocks past the row read as zero
            const int per = kStageBlocks * p.M * 8;  // 16-byte chunks per stage
            for (int i = ct; i < ns * per; i += kConsumers * 32) {
                const int sx = i / per, j = i - sx * per;
                const int b = j / (p.M * 8), rem = j - b * (p.M * 8), tok = rem >> 3, c = rem & 7;
                const int row = b * p.M + tok;
                const int64_t kk = static_cast<int64_t>(4 * (col_lo + sx) + b) * 64 + 8 * c;
                const bool v = kk < p.k;
                cp_async16_zfill(s_xs + static_cast<uint32_t>(sx) * p.xs_stage +
                                     static_cast<uint32_t>(row * 128 + ((c ^ (row & 7)) << 4)),
                                 v ? p.x + tok * p.k + kk : p.x, v ? 16u : 0u);
            }
            cp_async_arrive_noinc(bb.xready);
        }
        build_pair_lut(lut, ct, kConsumers * 32, p.qtype);
        if (p.x_once) cp_async_wait_all();
        named_sync(1, kConsumers * 32);  // the table is complete and every consumer's x copies have landed
        QN_TL(22, ct == 0);
        const uint32_t lane_op = lut_lane_operand<kFixedBase>(lut, lane);
        const uint32_t lut_base = s_base;
        const float mu = mu_pre;
        // x rows of this lane's tokens (tokens beyond M read token tok % M; their columns of the
        // result are never stored): row kg M + tok of the x box, 16-byte chunks 2 t and 2 t + 1
        // of it, stored at chunk ^ (row & 7)
        uint32_t xr[NG], xc0[NG], xc1[NG];
#pragma unroll
        for (int tg = 0; tg < NG; ++tg) {
            const int tok = (tg * 8 + g) % p.M;
            const int row = kg * p.M + tok;
            xr[tg] = static_cast<uint32_t>(row) * 128u;
            xc0[tg] = static_cast<uint32_t>(((2 * t) ^ (row & 7)) << 4);
            xc1[tg] = static_cast<uint32_t>(((2 * t + 1) ^ (row & 7)) << 4);
        }
        // The block constant this lane computes each stage: m-tile rg + 4 (2 pass + (t >> 1)), row
        // g + 8 (t & 1) of it, block kg. The quad's four lanes cover the (up to) two m-tiles x two
        // rows the quad needs and share them with shuffles (MW = 4: a second pass for m-tiles
        // rg + 8, rg + 12). c_q: staged FP8 code of block kg of the first stage; c_e: its block
        // index relative to the first staged group scale (its scale is staged at c_e >> 8).
        constexpr int NP = (MWL + 1) / 2;
        bool c_ok[NP];
        uint32_t c_q[NP];
        int64_t c_e[NP];
#pragma unroll
        for (int pass = 0; pass < NP; ++pass) {
            const int mt = rg + 4 * (2 * pass + (t >> 1));
            const int i = 16 * mt + g + 8 * (t & 1);
            const int64_t e0 = (row0 + i) * p.nbr + 4 * col_lo;
            c_ok[pass] = mt < p.m && row0 + i < nrow;
            c_q[pass] = s_qs + static_cast<uint32_t>(i) * p.qs_stride +
                        (p.absmax ? 4u * static_cast<uint32_t>((e0 & 3) + kg) : static_cast<uint32_t>(e0 & 15) + kg);
            c_e[pass] = e0 + kg - ((s_lo & ~int64_t(3)) << 8);  // staged scales start at s_lo & ~3
        }
        int nsc = ns;
        if (!mbar_wait(bb.consts, 0)) {
            fail();
            nsc = 0;
        }

        for (int s = 0; s < nsc; ++s) {
            const int slot = s % S;
            // every lane waits for the stage; the warp leaves together (mma.sync and shuffles below)
            const bool ok = !*bb.abort_flag && mbar_wait(&bb.full[slot], (s / S) & 1);
            if (!__all_sync(0xffffffffu, ok)) {
                if (!ok) fail();
                break;
            }
            QN_TL(3, threadIdx.x == 32 && s == 0);
            QN_TL(4, threadIdx.x == 32 && s == ns - 1);
            const int col = col_lo + s;
            const uint32_t sl = s_ring + static_cast<uint32_t>(slot) * p.slot_bytes;
            const bool blk_ok = 4 * col + kg < p.nbr;
            // block constants c'_b = fma(e4m3(q_b), sigma_g, mu) of this lane's rows, block kg
            float cmine[NP];
#pragma unroll
            for (int pass = 0; pass < NP; ++pass) {
                float c = 0.0f;
                if (c_ok[pass] && blk_ok) {
                    if (p.absmax) {
                        c = __uint_as_float(lds32(c_q[pass] + 16u * s));
                    } else {
                        const uint32_t qb = lds8(c_q[pass] + 4u * s);
                        const int64_t si = (c_e[pass] + 4 * s) >> 8;
                        const float sg = __uint_as_float(lds32(s_ss + 4u * static_cast<uint32_t>(si)));
                        c = block_constant(static_cast<uint8_t>(qb), sg, mu);
                    }
                }
                cmine[pass] = c;
            }
            const uint32_t xb = p.x_once ? s_xs + static_cast<uint32_t>(s) * p.xs_stage : sl + p.x_off;
            uint4 x0[NG], x1[NG];
#pragma unroll
            for (int tg = 0; tg < NG; ++tg) {
                x0[tg] = lds128(xb + xr[tg] + xc0[tg]);
                x1[tg] = lds128(xb + xr[tg] + xc1[tg]);
            }
            // codes of row (16 mt + g), bytes 32 kg + 8 t .. + 8: 16-byte chunk 2 kg + (t >> 1) of
            // the 128-byte row, stored at chunk index ^ (row & 7) = ^ g
            const uint32_t cchunk = static_cast<uint32_t>(((2 * kg + (t >> 1)) ^ g) << 4) + 8u * (t & 1);
            if constexpr (kMT == 2 && NG == 1) {
                // both m-tiles of the warp at once: their table loads issue back to back and
                // their two MMA chains interleave (constants: quad lanes 0, 1 for m-tile rg,
                // 2, 3 for m-tile rg + 4)
                const float cA0 = __shfl_sync(0xffffffffu, cmine[0], (lane & ~3));
                const float cB0 = __shfl_sync(0xffffffffu, cmine[0], (lane & ~3) | 1);
                const float cA1 = __shfl_sync(0xffffffffu, cmine[0], (lane & ~3) | 2);
                const float cB1 = __shfl_sync(0xffffffffu, cmine[0], (lane & ~3) | 3);
                const uint32_t cr0 = sl + static_cast<uint32_t>(16 * rg + g) * 128u + cchunk;
                const uint32_t cr1 = cr0 + 64u * 128u;
                const uint2 ca0 = lds64(cr0), cb0 = lds64(cr0 + 8 * 128);
                const uint2 ca1 = lds64(cr1), cb1 = lds64(cr1 + 8 * 128);
                uint32_t af0[4][4], af1[4][4];
#pragma unroll
                for (int kk = 0; kk < 4; ++kk) {
                    const int i0 = (2 * kk) & 3;
                    const uint32_t wa0 = kk < 2 ? ca0.x : ca0.y, wb0 = kk < 2 ? cb0.x : cb0.y;
                    const uint32_t wa1 = kk < 2 ? ca1.x : ca1.y, wb1 = kk < 2 ? cb1.x : cb1.y;
                    af0[kk][0] = lut_pair<kFixedBase>(lut_base, wa0, lane_op, i0);
                    af0[kk][2] = lut_pair<kFixedBase>(lut_base, wa0, lane_op, i0 + 1);
                    af0[kk][1] = lut_pair<kFixedBase>(lut_base, wb0, lane_op, i0);
                    af0[kk][3] = lut_pair<kFixedBase>(lut_base, wb0, lane_op, i0 + 1);
                    af1[kk][0] = lut_pair<kFixedBase>(lut_base, wa1, lane_op, i0);
                    af1[kk][2] = lut_pair<kFixedBase>(lut_base, wa1, lane_op, i0 + 1);
                    af1[kk][1] = lut_pair<kFixedBase>(lut_base, wb1, lane_op, i0);
                    af1[kk][3] = lut_pair<kFixedBase>(lut_base, wb1, lane_op, i0 + 1);
                }
                float d0[4], d1[4];
                mma_16816_z(d0, af0[0][0], af0[0][1], af0[0][2], af0[0][3], x0[0].x, x0[0].y);
                mma_16816_z(d1, af1[0][0], af1[0][1], af1[0][2], af1[0][3], x0[0].x, x0[0].y);
                mma_16816(d0, af0[1][0], af0[1][1], af0[1][2], af0[1][3], x0[0].z, x0[0].w);
                mma_16816(d1, af1[1][0], af1[1][1], af1[1][2], af1[1][3], x0[0].z, x0[0].w);
                mma_16816(d0, af0[2][0], af0[2][1], af0[2][2], af0[2][3], x1[0].x, x1[0].y);
                mma_16816(d1, af1[2][0], af1[2][1], af1[2][2], af1[2][3], x1[0].x, x1[0].y);
                mma_16816(d0, af0[3][0], af0[3][1], af0[3][2], af0[3][3], x1[0].z, x1[0].w);
                mma_16816(d1, af1[3][0], af1[3][1], af1[3][2], af1[3][3], x1[0].z, x1[0].w);
                acc[0][0][0] = __fmaf_rn(cA0, d0[0], acc[0][0][0]);
                acc[0][0][1] = __fmaf_rn(cA0, d0[1], acc[0][0][1]);
                acc[0][0][2] = __fmaf_rn(cB0, d0[2], acc[0][0][2]);
                acc[0][0][3] = __fmaf_rn(cB0, d0[3], acc[0][0][3]);
                acc[1][0][0] = __fmaf_rn(cA1, d1[0], acc[1][0][0]);
                acc[1][0][1] = __fmaf_rn(cA1, d1[1], acc[1][0][1]);
                acc[1][0][2] = __fmaf_rn(cB1, d1[2], acc[1][0][2]);
                acc[1][0][3] = __fmaf_rn(cB1, d1[3], acc[1][0][3]);
            } else
#pragma unroll
            for (int i = 0; i < MWL; ++i) {
                const int mt = rg + 4 * i;
                // constants of m-tile i: rows g and g + 8, held by quad lanes 2 (i & 1) and 2 (i & 1) + 1
                const float cA = __shfl_sync(0xffffffffu, cmine[i >> 1], (lane & ~3) | (2 * (i & 1)));
                const float cB = __shfl_sync(0xffffffffu, cmine[i >> 1], (lane & ~3) | (2 * (i & 1) + 1));
                if (kMT > 0 || mt < p.m) {
                    const uint32_t cr = sl + static_cast<uint32_t>(16 * mt + g) * 128u + cchunk;
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
            __syncwarp();
            if (lane == 0) mbar_arrive(&bb.empty[slot]);
        }
        cp_async_wait_all();  // the constants' copies (complete already unless a wait ran out)
    }

    // ---------------------------------------------------------------------- reduction
    // The ring is idle once every consumer has left its loop (they waited for every stage, so
    // every box has landed): its space holds the exchange buffer of the four block-warps. The
    // consumers sum the block-warps of each m-tile in a fixed order (kg = 0, 1, 2, 3).
    QN_TL(5, threadIdx.x == 32);
    // [kg][m m-tiles][32 lanes][NG*4] f32 (kg 1..3 in slots 0..2 when C == 1, kg 0..3 otherwise)
    const uint32_t red = s_base + p.post_off;
    auto store_partials = [&]() {
#pragma unroll
        for (int i = 0; i < MW; ++i) {
            const int mt = rg + 4 * i;
            if (mt < p.m) {
#pragma unroll
                for (int tg = 0; tg < NG; ++tg) {
                    const uint32_t o = red + static_cast<uint32_t>((((kg - 1) * p.m + mt) * 32 + lane) * NG + tg) * 16;
                    asm volatile("st.shared.v4.f32 [%0], {%1,%2,%3,%4};" ::"r"(o), "f"(acc[i][tg][0]),
                                 "f"(acc[i][tg][1]), "f"(acc[i][tg][2]), "f"(acc[i][tg][3])
                                 : "memory");
                }
            }
        }
    };
    auto sum_partials = [&](int i) {
        const int mt = rg + 4 * i;
#pragma unroll
        for (int q = 0; q < 3; ++q) {
#pragma unroll
            for (int tg = 0; tg < NG; ++tg) {
                const uint4 v = lds128(red + static_cast<uint32_t>(((q * p.m + mt) * 32 + lane) * NG + tg) * 16);
                acc[i][tg][0] += __uint_as_float(v.x);
                acc[i][tg][1] += __uint_as_float(v.y);
                acc[i][tg][2] += __uint_as_float(v.z);
                acc[i][tg][3] += __uint_as_float(v.w);
            }
        }
    };

    if (C == 1) {
        // one CTA holds whole rows: add B t to the summed fragments on the tensor cores and store
        __syncthreads();  // every consumer has left its loop; the producer has t and the B rows
        QN_TL(6, threadIdx.x == 0);
        if (warp > 0 && kg > 0) store_partials();
        __syncthreads();
        QN_TL(9, threadIdx.x == 0);
        const bool run_ok = !*bb.abort_flag;
        if (warp > 0 && kg == 0) {
#pragma unroll
            for (int i = 0; i < MW; ++i) {
                const int mt = rg + 4 * i;
                if (mt >= p.m) continue;
                sum_partials(i);
                if (p.r > 0) {
                    const uint32_t brow = bs + static_cast<uint32_t>((16 * mt + g) * p.bs_stride);
                    for (int kc = 0; kc < p.rk16 / 16; ++kc) {
                        const uint32_t j2 = static_cast<uint32_t>(16 * kc + 2 * t) * 2u;
                        const uint32_t a0 = lds32(brow + j2), a2 = lds32(brow + j2 + 16);
                        const uint32_t a1 = lds32(brow + 8 * p.bs_stride + j2),
                                       a3 = lds32(brow + 8 * p.bs_stride + j2 + 16);
#pragma unroll
                        for (int tg = 0; tg < NG; ++tg) {
                            const uint32_t tr = tb + static_cast<uint32_t>((tg * 8 + g) * p.rk16) * 2u + j2;
                            mma_16816(acc[i][tg], a0, a1, a2, a3, lds32(tr), lds32(tr + 16));
                        }
                    }
                }
                if (run_ok) {
                    const int64_t rA = row0 + 16 * mt + g, rB = rA + 8;
#pragma unroll
                    for (int tg = 0; tg < NG; ++tg) {
                        const int tok = tg * 8 + 2 * t;
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const int64_t row = (e < 2) ? rA : rB;
                            const int tk = tok + (e & 1);
                            if (row < nrow && tk < p.M)
                                p.h[static_cast<int64_t>(tk) * p.n + row] =
                                    __bfloat16_as_ushort(__float2bfloat16_rn(acc[i][tg][e]));
                        }
                    }
                }
            }
        }
        QN_TL(10, threadIdx.x == 32);
    } else if (warp > 0) {
        // Cluster: the consumers reduce among themselves and push each row's partial sums (all MP
        // token columns) to the row's owner [src][row][MP] f32 right away; the owner adds B t while
        // it sums the C partials, so t from the adapter cluster is needed only there.
        // M-tile rg + 4 i is summed and pushed by warp (kg = i, rg), so that the sums and the
        // pushes of the chunk's m-tiles spread over all the consumer warps.
        named_sync(2, kConsumers * 32);  // every consumer has left its loop: the ring is idle
        QN_TL(6, threadIdx.x == 32);
#pragma unroll
        for (int i = 0; i < MW; ++i) {
            const int mt = rg + 4 * i;
            if (i == kg || mt >= p.m) continue;
#pragma unroll
            for (int tg = 0; tg < NG; ++tg) {
                const uint32_t o = red + static_cast<uint32_t>(((kg * p.m + mt) * 32 + lane) * NG + tg) * 16;
                asm volatile("st.shared.v4.f32 [%0], {%1,%2,%3,%4};" ::"r"(o), "f"(acc[i][tg][0]), "f"(acc[i][tg][1]),
                             "f"(acc[i][tg][2]), "f"(acc[i][tg][3])
                             : "memory");
            }
        }
        named_sync(3, kConsumers * 32);
        QN_TL(9, threadIdx.x == 32);
        const int mo = rg + 4 * kg;  // the m-tile this warp sums
        float own[NG][4], sum[NG][4];
#pragma unroll
        for (int i = 0; i < MW; ++i)
            if (i == kg)
#pragma unroll
                for (int tg = 0; tg < NG; ++tg)
#pragma unroll
                    for (int e = 0; e < 4; ++e) own[tg][e] = acc[i][tg][e];
        if (mo < p.m) {
            // the four block-warps' partials in kg order
#pragma unroll
            for (int q = 0; q < 4; ++q)
#pragma unroll
                for (int tg = 0; tg < NG; ++tg) {
                    float v[4];
                    if (q == kg) {
                        v[0] = own[tg][0], v[1] = own[tg][1], v[2] = own[tg][2], v[3] = own[tg][3];
                    } else {
                        const uint4 w4 =
                            lds128(red + static_cast<uint32_t>(((q * p.m + mo) * 32 + lane) * NG + tg) * 16);
                        v[0] = __uint_as_float(w4.x), v[1] = __uint_as_float(w4.y);
                        v[2] = __uint_as_float(w4.z), v[3] = __uint_as_float(w4.w);
                    }
#pragma unroll
                    for (int e = 0; e < 4; ++e) sum[tg][e] = q == 0 ? v[e] : sum[tg][e] + v[e];
                }
        }
        QN_TL(10, threadIdx.x == 32);
        cluster_wait();  // phase 1: every CTA of the cluster runs (its barriers are initialised)
        if (mo < p.m) {
            const uint32_t recv = s_base + p.recv_off;
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
                const int rl = 16 * mo + g + 8 * hh;
                const int owner = (rl * C + C - 1) / p.R;
                const int rr = rl - p.R * owner / C;
                const uint32_t dst = mapa(recv + static_cast<uint32_t>(((crank * nrmax + rr) * MP + 2 * t) * 4),
                                          static_cast<uint32_t>(owner));
                const uint32_t bar = mapa(saddr(bb.recv), static_cast<uint32_t>(owner));
#pragma unroll
                for (int tg = 0; tg < NG; ++tg)
                    st_async_v2(dst + 32u * tg, sum[tg][2 * hh], sum[tg][2 * hh + 1], bar);
            }
        }
        QN_TL(11, threadIdx.x == 32);
        // rows [r_lo, r_hi): the C partials in rank order, plus B t
        bool ok = mbar_wait(bb.recv, 0);
        if (ok && !mbar_wait(bb.tready, 0)) ok = false;
        if (!ok && threadIdx.x == 32) record_error(p.err, kErrTimeout);
        QN_TL(13, threadIdx.x == 32);
        if (ok && !*bb.abort_flag) {
            const float *recvf = reinterpret_cast<const float *>(smem + p.recv_off);
            for (int it = threadIdx.x - 32; it < nr * p.M; it += kConsumers * 32) {
                const int rr = it % nr, tok = it / nr;
                const int64_t row = row0 + r_lo + rr;
                if (row >= nrow) continue;
                float tot = 0.0f;
                for (int src = 0; src < C; ++src) tot += recvf[(src * nrmax + rr) * MP + tok];
                if (p.r > 0) tot += reinterpret_cast<const float *>(smem + p.bt_off)[rr * MP + tok];
                p.h[static_cast<int64_t>(tok) * p.n + row] = __bfloat16_as_ushort(__float2bfloat16_rn(tot));
            }
        }
        QN_TL(20, threadIdx.x == 32);
    }
    QN_TL(7, threadIdx.x == 0);
#ifdef QN_TIMELINE
    if (threadIdx.x == 0) {
        unsigned long long t;
        asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
        const unsigned cta = blockIdx.y * gridDim.x + blockIdx.x;
        if (cta < 1024) g_fwd_timeline[p.tl_buf & 1][cta][15] = t;  // end in ns: with slot 7 gives the clock
    }
#endif
}

// kMT: 2 for chunks of 128 rows (m = 8), whose tile loop is specialised; 0 for every other m.
template <int NG, int kMT>
__global__ void __launch_bounds__(kThreads, 1)
k_decode_fwd(const __grid_constant__ CUtensorMap tm_codes, const __grid_constant__ CUtensorMap tm_x,
             const __grid_constant__ CUtensorMap tm_xp, const __grid_constant__ CUtensorMap tm_a, const FwdArgs p) {
    extern __shared__ __align__(1024) uint8_t smem[];
    // the 128-byte-swizzled boxes need 1024-byte aligned slots (uniform over the grid: every CTA
    // leaves here together, before any barrier)
    if (saddr(smem) & 1023u) {
        if (threadIdx.x == 0) record_error(p.err, kErrLayout);
        return;
    }
    if (p.r > 0 && blockIdx.y == 0) {
        adapter_body<NG>(&tm_xp, &tm_a, p, smem);
    } else if ((saddr(smem) & 0x00ffffffu) == kDynSmemBase) {
        chunk_body<NG, true, kMT>(&tm_codes, &tm_x, p, smem);
    } else {
        chunk_body<NG, false, kMT>(&tm_codes, &tm_x, p, smem);
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

// Tiled tensor map of `rank` dimensions: dims[0] is contiguous; strides[i] is the byte stride of
// dimension i + 1.
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

// x (M x k) or A (r x k), bf16, as the stage boxes read it: 3-D {64 values, rows, blocks}, box
// {64, box_rows, 4} (rows past `rows` read as zero), 128-byte swizzle.
bool encode_operand(CUtensorMap *m, const uint16_t *base, int64_t rows, int64_t k, int box_rows) {
    const uint64_t dims[3] = {64, static_cast<uint64_t>(rows), static_cast<uint64_t>(k / 64)};
    const uint64_t strides[2] = {static_cast<uint64_t>(k) * 2, 128};
    const uint32_t box[3] = {64, static_cast<uint32_t>(box_rows), kStageBlocks};
    return encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, base, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B);
}

int round_rank(int r) { return r <= 0 ? 0 : r <= 8 ? 8 : r <= 16 ? 16 : r <= 32 ? 32 : 64; }

uint32_t align_up(uint32_t v, uint32_t a) { return (v + a - 1) / a * a; }

// Shared-memory layout of one launch shape, x staged once (x_once) or per stage in the ring
// slots; false if it does not fit.
bool layout_mode(FwdArgs &a, int MP, bool x_once) {
    const uint32_t codes = static_cast<uint32_t>(a.R) * 128u;  // multiple of 2048 (R = 16 m)
    const uint32_t xb = kStageBlocks * static_cast<uint32_t>(a.M) * 128u;
    const uint32_t xpb = kStageBlocks * MP * 128u;
    const uint32_t ab = a.r > 0 ? kStageBlocks * a.rpad * 128u : 0u;
    const int nsmax = (a.ncol + a.C - 1) / a.C;
    a.x_once = x_once ? 1 : 0;
    a.x_off = x_once ? 0u : codes;
    a.xs_stage = xb;
    const uint32_t chunk_slot = x_once ? codes : codes + xb;
    a.a_off = xpb;
    a.slot_bytes = align_up(chunk_slot > xpb + ab ? chunk_slot : xpb + ab, 1024);
    a.codes_bytes = codes;
    a.x_bytes = xb;
    a.xa_bytes = xpb + ab;
    const uint32_t xs = x_once ? align_up(static_cast<uint32_t>(nsmax) * xb, 128) : 0u;
    // staged FP8 codes (or fp32 constants): 16-byte chunks per chunk row, an odd count so that
    // rows fall on distinct bank groups
    const int nch = a.absmax ? (12 + 16 * nsmax + 15) / 16 : (15 + 4 * nsmax + 15) / 16;
    a.qs_stride = 16u * static_cast<uint32_t>(nch | 1);
    // staged group scales: at most R nbr / 256 + 2 of them, in whole 16-byte chunks (none with
    // fp32 constants)
    const int64_t s_max = a.absmax ? 0 : static_cast<int64_t>(a.R) * a.nbr / 256 + 8;
    if (s_max > (int64_t(1) << 20)) return false;
    const uint32_t qs = align_up(static_cast<uint32_t>(a.R) * a.qs_stride, 128);
    const uint32_t ss = align_up(static_cast<uint32_t>(s_max) * 4u, 128);
    const uint32_t tbb = a.r > 0 ? align_up(static_cast<uint32_t>(MP * a.rk16 * 2), 128) : 0u;
    // staged B rows: the rows the CTA finalises (all R when C == 1), padded so that the eight
    // fragment rows fall on distinct bank groups
    a.bs_stride = static_cast<uint32_t>(2 * a.rk16 + 16);
    const uint32_t bsb = a.r > 0 ? align_up(static_cast<uint32_t>((a.R + a.C - 1) / a.C) * a.bs_stride, 128) : 0u;
    const uint32_t post_chunk = static_cast<uint32_t>((a.C > 1 ? 4 : 3) * a.m * 32 * 16 * (MP / 8));
    const uint32_t post_adapter = kConsumers * 32 * 16;
    const uint32_t post = post_chunk > post_adapter ? post_chunk : post_adapter;
    const uint32_t recv_chunk = a.C > 1 ? static_cast<uint32_t>(a.C * ((a.R + a.C - 1) / a.C) * MP * 4) : 0u;
    const uint32_t recv_adapter = a.r > 0 ? static_cast<uint32_t>(a.C * MP * a.rpad * 4) : 0u;
    const uint32_t recv = align_up(recv_chunk > recv_adapter ? recv_chunk : recv_adapter, 128);
    // B t of the finalised rows (C > 1): [ceil(R / C)][MP] fp32
    const uint32_t bt = a.C > 1 && a.r > 0 ? align_up(static_cast<uint32_t>((a.R + a.C - 1) / a.C * MP * 4), 128) : 0u;
    const uint32_t bars = 256;
    const uint64_t fixed = static_cast<uint64_t>(kLutBytes) + qs + ss + tbb + bsb + xs + recv + bt + bars;
    if (fixed + a.slot_bytes > kSmemLimit) return false;
    int stages = static_cast<int>((kSmemLimit - fixed) / a.slot_bytes);
    if (stages > kMaxStages) stages = kMaxStages;
    if (stages > nsmax) stages = nsmax;
    const int need = nsmax < 2 ? nsmax : 2;
    if (stages < need) return false;
    uint32_t ring = static_cast<uint32_t>(stages) * a.slot_bytes;
    bool post_in_ring = ring >= post;
    if (!post_in_ring && fixed + ring + post > kSmemLimit) {
        // the exchange buffer outgrows the ring: give it room of its own
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
    a.qs_off = off;
    off += qs;
    a.ss_off = off;
    off += ss;
    a.tb_off = off;
    off += tbb;
    a.bs_off = off;
    off += bsb;
    a.xs_off = off;
    off += xs;
    a.recv_off = off;
    off += recv;
    a.bt_off = off;
    off += bt;
    a.bar_off = off;
    return static_cast<uint64_t>(off) + bars <= kSmemLimit;
}

bool layout(FwdArgs &a, int MP) {
#ifndef QN_FWD_NO_X_ONCE
    if (layout_mode(a, MP, true)) return true;
#endif
    return layout_mode(a, MP, false);
}

size_t smem_bytes(const FwdArgs &a) { return static_cast<size_t>(a.bar_off) + 256; }

// Bytes the busiest CTA moves: chunk CTAs codes + x per stage, adapter CTAs x + A per stage.
double cta_bytes(const FwdArgs &a) {
    const int nsmax = (a.ncol + a.C - 1) / a.C;
    const double chunk = static_cast<double>(a.codes_bytes + a.x_bytes) * nsmax;
    const double adapter = a.r > 0 ? static_cast<double>(a.xa_bytes) * nsmax : 0.0;
    return chunk > adapter ? chunk : adapter;
}

// The kernel that runs chunks of m m-tiles.
template <int NG>
const void *fwd_kernel(int m) {
    return m == 8 ? reinterpret_cast<const void *>(k_decode_fwd<NG, 2>)
                  : reinterpret_cast<const void *>(k_decode_fwd<NG, 0>);
}

// Launch shape for `rows` weight rows: R = 16 m rows per chunk and C K-slices per cluster with
// (chunks + 1) x C <= SMs and every cluster resident at once; the shape whose busiest CTA moves
// the fewest bytes (ties: the first found, i.e. smaller clusters, then shorter chunks).
template <int NG>
cudaError_t plan(FwdArgs &a, int64_t rows, int sms, bool &found) {
    constexpr int MP = 8 * NG;
    const int extra = a.r > 0 ? 1 : 0;  // the adapter cluster
    double best_cost = 0.0;
    FwdArgs best = a;
    found = false;
    // m is a multiple of 4 (every consumer warp holds the same number of m-tiles) unless the
    // weight has fewer than 64 rows
    const int m_max = kMaxM;  // four m-tile rows of warps, up to 4 m-tiles each
    const int m_min = rows < 64 ? static_cast<int>((rows + 15) / 16) : 4;
    const int m_step = rows < 64 ? 1 : 4;
    for (int C = 1; C <= kMaxCluster && C <= a.ncol; ++C) {
        for (int m = m_min; m <= m_max; m += m_step) {
            FwdArgs c = a;
            c.m = m;
            c.R = 16 * m;
            c.C = C;
            const int64_t chunks = (rows + c.R - 1) / c.R;
            if ((chunks + extra) * C > sms) continue;
            c.chunks = static_cast<int>(chunks);
            if (!layout(c, MP)) continue;
            const double cost = cta_bytes(c);
            if (found && cost >= best_cost * (1.0 - 1e-9)) continue;
            if (C > 1) {
                int nc = 0;
                const cudaError_t e = resident_clusters(fwd_kernel<NG>(m), kThreads, C, smem_bytes(c), &nc);
                if (e != cudaSuccess) return e;
                if (nc < c.chunks + extra) continue;
            }
            best = c;
            best_cost = cost;
            found = true;
        }
    }
    if (found) a = best;
    return cudaSuccess;
}

template <int NG>
cudaError_t launch_ng(const WeightView &w, const uint16_t *x, int M, const uint16_t *A, const uint16_t *B, int r,
                      float s, const DropoutArgs &drop, uint16_t *h, int *err, cudaStream_t st) {
    constexpr int MP = 8 * NG;
    int sms = 148;
    cudaError_t e = device_sm_count(&sms);
    if (e != cudaSuccess) return e;

    FwdArgs a = {};
    a.q = w.q;
    a.sigma = w.sigma;
    a.mu = w.mu;
    a.absmax = w.absmax;
    a.qtype = w.qtype;
    a.B = B;
    a.x = x;
    a.h = h;
    a.err = err;
    char *wsb = reinterpret_cast<char *>(err);
    a.flag = reinterpret_cast<unsigned *>(wsb + kWsFlag);
    a.readers = reinterpret_cast<unsigned *>(wsb + kWsReaders);
    a.t_ws = reinterpret_cast<uint16_t *>(wsb + kWsT);
    a.n = w.n;
    a.k = w.k;
    a.nbr = static_cast<int>(w.k / kBlock);
    a.ncol = (a.nbr + kStageBlocks - 1) / kStageBlocks;
    a.M = M;
    a.r = r;
    a.rpad = round_rank(r);
    a.rk16 = (a.rpad + 15) & ~15;
    a.s = s;
    a.drop = drop;
#ifdef QN_FWD_NO_EVICT_HINT
    a.evict_first = 0;
#else
    a.evict_first = 1;
#endif
    const int extra = r > 0 ? 1 : 0;  // the adapter cluster

    // Every CTA of a launch must be resident at once (the chunk CTAs wait for the adapter
    // cluster): a weight taller than one wave runs as several launches over row ranges of equal
    // size (multiples of 256 rows), each with its own adapter cluster.
    int64_t part = w.n;
    bool found = false;
    for (;;) {
        e = plan<NG>(a, part, sms, found);
        if (e != cudaSuccess) return e;
        if (found) break;
        if (part <= 256) return cudaErrorInvalidConfiguration;
        part = ((part + 1) / 2 + 255) / 256 * 256;
    }
    const size_t smem = smem_bytes(a);

    CUtensorMap tm_codes, tm_x, tm_xp, tm_a;
    {
        const uint64_t dims[2] = {static_cast<uint64_t>(w.k / 2), static_cast<uint64_t>(w.n)};
        const uint64_t strides[1] = {static_cast<uint64_t>(w.k / 2)};
        const uint32_t box[2] = {128, static_cast<uint32_t>(a.R)};
        if (!encode(&tm_codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, w.codes, dims, strides, box,
                    CU_TENSOR_MAP_SWIZZLE_128B))
            return cudaErrorInvalidValue;
    }
    if (!encode_operand(&tm_x, x, M, w.k, M)) return cudaErrorInvalidValue;
    if (r > 0) {
        if (!encode_operand(&tm_xp, x, M, w.k, MP) || !encode_operand(&tm_a, A, r, w.k, a.rpad))
            return cudaErrorInvalidValue;
    } else {
        tm_xp = tm_x;  // never read
        tm_a = tm_x;
    }
    e = ensure_smem_limit(fwd_kernel<NG>(a.m), smem);
    if (e != cudaSuccess) return e;

    for (int64_t lo = 0; lo < w.n; lo += part) {
        FwdArgs b = a;
#ifdef QN_TIMELINE
        b.tl_buf = g_launches_tl++ & 1;
#endif
        b.row_lo = lo;
        b.row_hi = lo + part < w.n ? lo + part : w.n;
        b.chunks = static_cast<int>((b.row_hi - lo + b.R - 1) / b.R);
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(static_cast<unsigned>(b.C), static_cast<unsigned>(b.chunks + extra), 1);
        cfg.blockDim = dim3(kThreads, 1, 1);
        cfg.dynamicSmemBytes = smem;
        cfg.stream = st;
        cudaLaunchAttribute attr[2];
        attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[0].val.programmaticStreamSerializationAllowed = 1;
        attr[1].id = cudaLaunchAttributeClusterDimension;
        attr[1].val.clusterDim.x = b.C;
        attr[1].val.clusterDim.y = 1;
        attr[1].val.clusterDim.z = 1;
        cfg.attrs = attr;
        cfg.numAttrs = b.C > 1 ? 2 : 1;
        if (b.m == 8)
            e = cudaLaunchKernelEx(&cfg, k_decode_fwd<NG, 2>, tm_codes, tm_x, tm_xp, tm_a, b);
        else
            e = cudaLaunchKernelEx(&cfg, k_decode_fwd<NG, 0>, tm_codes, tm_x, tm_xp, tm_a, b);
        count_launch();
        if (e != cudaSuccess) return e;
    }
#ifdef QN_TIMELINE
    g_last_plan[0] = a.R;
    g_last_plan[1] = a.C;
    g_last_plan[2] = a.stages;
    g_last_plan[3] = a.chunks;
    g_last_plan[4] = static_cast<int>(smem);
    g_last_plan[5] = static_cast<int>(cta_bytes(a) / 1024);
#endif
    return e;
}

}  // namespace

size_t decode_fwd_workspace_bytes() { return kWsT + 16 * 64 * 2; }

cudaError_t launch_decode_fwd(const WeightView &w, const uint16_t *x, int M, const uint16_t *A, const uint16_t *B,
                              int r, float s, const DropoutArgs &drop, uint16_t *h, int *err, cudaStream_t st) {
    if (M <= 0 || w.n == 0) return cudaSuccess;
    if (M > kDecodeTokens || r > kDecodeMaxRank) return cudaErrorInvalidValue;
    if (M <= 8) return launch_ng<1>(w, x, M, A, B, r, s, drop, h, err, st);
    return launch_ng<2>(w, x, M, A, B, r, s, drop, h, err, st);
}

#ifdef QN_TIMELINE
extern "C" void qn_debug_fwd_plan(int *out) {
    for (int i = 0; i < 6; ++i) out[i] = g_last_plan[i];
}
extern "C" int qn_debug_fwd_smid(int *out, int n, int buf) {
    const int which = (g_launches_tl - 1 - buf) & 1;
    return cudaMemcpyFromSymbol(out, g_fwd_smid, sizeof(int) * (n < 1024 ? n : 1024), sizeof(int) * 1024 * which) ==
                   cudaSuccess
               ? 0
               : 1;
}
// buf 0: the last launch's timeline, 1: the one before it
extern "C" int qn_debug_fwd_timeline(unsigned long long *out, int n, int buf) {
    const int which = (g_launches_tl - 1 - buf) & 1;
    return cudaMemcpyFromSymbol(out, g_fwd_timeline, sizeof(unsigned long long) * 24 * (n < 1024 ? n : 1024),
                                sizeof(unsigned long long) * 24 * 1024 * which) == cudaSuccess
               ? 0
               : 1;
}
#endif

}  // namespace qn
