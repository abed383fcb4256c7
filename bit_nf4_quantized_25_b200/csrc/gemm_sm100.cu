// gemm_sm100.cu -- fused NF4 dequant-GEMM on the 5th-generation tensor cores (tcgen05 + TMEM)
// for many tokens, forward and input gradient, with the LoRA up-projection accumulated into
// the same tile.
//
//   fwd : h^T[n, m]      = sum_k W'[n,k] x[m,k]       + sum_j B[n,j] t[m,j]    (t = s A x)
//   bwd : grad_x^T[k, m] = sum_n W'[n,k] grad_h[m,n]  + sum_j A[j,k] u[m,j]    (u = s B^T grad_h)
// "Quantized LoRA (QLoRA) and 4-bit training" (apxml.com): the 4-bit weights are
// dequantised to bf16 for the matmul and the adapter output is added; "How does QLoRA work
// for training?" (aivaro.ru), section 7: the same dequantisation feeds the gradient.
//
// One CTA computes a 128 x 512 tile: 128 weight rows (fwd) or 128 input features (bwd) as
// the MMA M dimension and two halves of 256 tokens as the MMA N dimension, each with its own
// fp32 accumulator in TMEM (512 columns). Each dequantised A tile feeds both halves, which
// halves the dequantisation work per flop.
//   warp 0      : TMA producer of the token operand (x / grad_h, then t / u), 64-wide K slabs
//                 in the 128-byte swizzled K-major layout (4-slot ring, one slot per k-slab and
//                 token half), and of the packed codes of each k-slab's weight tile (4 KB, one
//                 slot per dequant group).
//   warp 1      : TMEM allocator and the single MMA-issuing thread (tcgen05.mma kind::f16).
//   warps 2..13 : three groups of four dequant warps taking k-slabs round-robin. A thread owns one
//                 64-weight block per stage (fwd: one row; bwd: half of a reduction row),
//                 builds the 16 scaled bf16 values NF4[i] * c'_b in registers, expands the
//                 nibbles with byte permutes and writes the swizzled A tile (K-major for fwd,
//                 MN-major for bwd, so W is always read in its stored row-major order).
//                 The extra LoRA stages copy rows of B (fwd) / A (bwd) into the A tile.
//   epilogue    : the dequant warps read TMEM (tcgen05.ld) and store bf16, staged through shared
//                 memory for 16-byte stores when the output rows allow it.
// Every mbarrier wait is bounded; on a timeout the CTA records an error code, stops issuing
// work, drains what it issued and frees its TMEM.
#include <cudaTypedefs.h>

#include "common.cuh"
#include "kernels.h"
#include "sm100.cuh"

namespace qn {

namespace {

using namespace sm100;

constexpr int kTileM = 128;  // MMA M: weight rows / input features
constexpr int kTileN = 256;  // MMA N: tokens per accumulator
constexpr int kHalves = 2;   // accumulators per CTA: a CTA covers kHalves x 256 tokens
constexpr int kTileK = 64;   // reduction per stage: one 128-byte swizzle row of bf16
constexpr int kAStages = 3;  // dequantised A tiles and their code slots (one per dequant group)
constexpr int kBStages = 5;  // token-operand tiles (one per k-slab and half)
constexpr int kDqGroups = 3;               // dequant groups taking stages round-robin
constexpr int kDqWarps = 4 * kDqGroups;
constexpr int kGemmThreads = (2 + kDqWarps) * 32;
static_assert(kDqGroups == kAStages, "each dequant group owns one A slot");
constexpr uint32_t kABytes = kTileM * kTileK * 2;  // 16 KB
constexpr uint32_t kBBytes = kTileN * kTileK * 2;  // 32 KB
constexpr uint32_t kCBytes = kTileM * kTileK / 2;  // 4 KB of packed codes per stage
constexpr uint32_t kTmemCols = kTileN * kHalves;  // 512: the whole TMEM of the SM
constexpr size_t kGemmSmem = 1024 + kAStages * (kABytes + kCBytes) + kBStages * kBBytes + 256;

constexpr int kErrTimeout = 1;

struct GemmParams {
    const uint8_t *codes;
    const uint8_t *q;
    const float *sigma;
    const float *mu;
    const float *absmax;    // fp32 block constants (no double quantisation), else nullptr
    int64_t n, k;           // W is n x k
    int64_t M;              // tokens
    const uint16_t *lora;   // fwd: B (n x r); bwd: A (r x k)
    int r;
    uint16_t *out;          // fwd: h (M x n); bwd: grad_x (M x k)
    int *err;
};

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
    uint32_t d;
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
    return d;
}

// 16 scaled table values bf16(T[i] * cp) of quant type kQT, split into low-byte planes L0..L3
// and high-byte planes H0..H3 (4 entries per register) for byte-permute lookups.
struct Planes {
    uint32_t L0, L1, L2, L3, H0, H1, H2, H3;
};

template <int kQT>
__device__ __forceinline__ Planes make_planes(float cp) {
    uint32_t E[8];
#pragma unroll
    for (int i = 0; i < 8; ++i)
        E[i] = pack_bf16x2(__fmul_rn(table_value(kQT, 2 * i), cp), __fmul_rn(table_value(kQT, 2 * i + 1), cp));
    Planes P;
    P.L0 = prmt(E[0], E[1], 0x6420);
    P.H0 = prmt(E[0], E[1], 0x7531);
    P.L1 = prmt(E[2], E[3], 0x6420);
    P.H1 = prmt(E[2], E[3], 0x7531);
    P.L2 = prmt(E[4], E[5], 0x6420);
    P.H2 = prmt(E[4], E[5], 0x7531);
    P.L3 = prmt(E[6], E[7], 0x6420);
    P.H3 = prmt(E[6], E[7], 0x7531);
    return P;
}

// Four codes (nibbles of the low 16 bits of s) -> two bf16x2 words (codes 0,1 and 2,3).
__device__ __forceinline__ void lookup4(const Planes &P, uint32_t s, uint32_t &o0, uint32_t &o1) {
    const uint32_t s7 = s & 0x7777u;
    const uint32_t la = prmt(P.L0, P.L1, s7), lb = prmt(P.L2, P.L3, s7);
    const uint32_t ha = prmt(P.H0, P.H1, s7), hb = prmt(P.H2, P.H3, s7);
    // byte j = 0xff where code j >= 8 (bit 3 selects an odd byte of 0xff00ff00)
    const uint32_t m = prmt(0xff00ff00u, 0xff00ff00u, s >> 3);
    const uint32_t lo = (la & ~m) | (lb & m), hi = (ha & ~m) | (hb & m);
    o0 = prmt(lo, hi, 0x5140);
    o1 = prmt(lo, hi, 0x7362);
}

// 8 codes (one 32-bit word, element 0 in the low nibble) -> 8 bf16 (16 bytes).
__device__ __forceinline__ uint4 expand8(const Planes &P, uint32_t w) {
    uint4 o;
    lookup4(P, w, o.x, o.y);
    lookup4(P, w >> 16, o.z, o.w);
    return o;
}

__device__ __forceinline__ void sts128(uint32_t addr, uint4 v) {
    asm volatile("st.shared.v4.u32 [%0], {%1,%2,%3,%4};" ::"r"(addr), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w)
                 : "memory");
}

// Byte offset of 16-byte chunk j (elements 8j..8j+7) of the 64-element row `row` of a
// 128-byte-swizzled tile whose rows are 128 bytes apart (K-major) -- also the layout of one
// 64-element MN chunk of an MN-major tile whose K rows are 128 bytes apart.
__device__ __forceinline__ uint32_t swz(uint32_t row, uint32_t j) { return row * 128u + ((j ^ (row & 7u)) << 4); }

template <bool kBwd, int kQT>
__global__ void __launch_bounds__(kGemmThreads, 1)
k_gemm_nf4(const __grid_constant__ CUtensorMap tm_act, const __grid_constant__ CUtensorMap tm_lora,
           const __grid_constant__ CUtensorMap tm_codes, const GemmParams p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *sA = smem;                         // kAStages x 16 KB
    uint8_t *sB = smem + kAStages * kABytes;    // kBStages x 32 KB
    // packed codes of each k-slab: fwd 128 weight rows x 32 bytes (one block); bwd 64 reduction
    // rows x 64 bytes (the two blocks of the tile's 128 features)
    uint8_t *sC = sB + kBStages * kBBytes;      // kAStages x 4 KB
    uint64_t *bars = reinterpret_cast<uint64_t *>(sC + kAStages * kCBytes);
    uint64_t *full_a = bars, *empty_a = full_a + kAStages, *full_c = empty_a + kAStages;
    uint64_t *empty_c = full_c + kAStages;  // the dequant group has read the slot's codes
    uint64_t *full_b = empty_c + kAStages, *empty_b = full_b + kBStages, *acc_full = empty_b + kBStages;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(acc_full + 1);
    volatile uint32_t *abort_flag = tmem_slot + 1;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t N = p.n, K = p.k, nbr = K / kBlock;
    const int64_t row0 = static_cast<int64_t>(blockIdx.x) * kTileM;  // fwd: weight row; bwd: feature
    const int64_t tok0 = static_cast<int64_t>(blockIdx.y) * kTileN * kHalves;
    const int nh = tok0 + kTileN < p.M ? kHalves : 1;  // token halves with any token in range
    const int nred = kBwd ? static_cast<int>((N + kTileK - 1) / kTileK) : static_cast<int>(nbr);
    const int nlora = (p.r + kTileK - 1) / kTileK;
    const int T = nred + nlora;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kAStages; ++s) {
            mbar_init(&full_a[s], 4);
            mbar_init(&empty_a[s], 1);
            mbar_init(&full_c[s], 1);
            mbar_init(&empty_c[s], 4);
        }
        for (int s = 0; s < kBStages; ++s) {
            mbar_init(&full_b[s], 1);
            mbar_init(&empty_b[s], 1);
        }
        mbar_init(acc_full, 1);
        *abort_flag = 0u;
        fence_barrier_init();
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, kTmemCols);
        tmem_relinquish();
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(&tm_act);
        tma_prefetch_desc(&tm_lora);
        tma_prefetch_desc(&tm_codes);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_d = *tmem_slot;
    grid_dependency_wait();  // activations and adapters may come from the preceding kernel

    auto fail = [&]() {
        if (atomicExch(const_cast<uint32_t *>(abort_flag), 1u) == 0u && p.err) atomicExch(p.err, kErrTimeout);
    };

    if (warp == 0) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            // k-slab i: its codes (slot i % kAStages, refilled once the dequant group has read
            // the slot's previous codes), then one token-operand tile per half (B sequence
            // j = i nh + h).
            uint32_t c_phase[kAStages], b_phase[kBStages];
            bool c_issued[kAStages], b_issued[kBStages];
            for (int s = 0; s < kAStages; ++s) c_issued[s] = false;
            for (int s = 0; s < kBStages; ++s) b_issued[s] = false;
            bool stop = false;
            for (int i = 0; i < T && !stop && !*abort_flag; ++i) {
                if (i < nred) {
                    const int sa = i % kAStages;
                    const uint32_t pa = (i / kAStages) & 1u;
                    if (i >= kAStages && !mbar_wait(&empty_c[sa], pa ^ 1u)) {
                        fail();
                        break;
                    }
                    // codes: fwd rows [row0, row0 + 128) x bytes [32 i, 32 i + 32);
                    //        bwd rows [64 i, 64 i + 64) x bytes [row0 / 2, row0 / 2 + 64)
                    mbar_arrive_expect_tx(&full_c[sa], kCBytes);
                    if (kBwd)
                        tma_load_2d(sC + sa * kCBytes, &tm_codes, &full_c[sa], static_cast<int32_t>(row0 / 2), i * kTileK);
                    else
                        tma_load_2d(sC + sa * kCBytes, &tm_codes, &full_c[sa], i * (kBlock / 2), static_cast<int32_t>(row0));
                    c_issued[sa] = true;
                    c_phase[sa] = pa;
                }
                for (int h = 0; h < nh; ++h) {
                    const int j = i * nh + h;
                    const int sb = j % kBStages;
                    const uint32_t pb = (j / kBStages) & 1u;
                    if (j >= kBStages && !mbar_wait(&empty_b[sb], pb ^ 1u)) {
                        fail();
                        stop = true;
                        break;
                    }
                    mbar_arrive_expect_tx(&full_b[sb], kBBytes);
                    const int32_t tk = static_cast<int32_t>(tok0 + h * kTileN);
                    if (i < nred)
                        tma_load_2d(sB + sb * kBBytes, &tm_act, &full_b[sb], i * kTileK, tk);
                    else
                        tma_load_2d(sB + sb * kBBytes, &tm_lora, &full_b[sb], (i - nred) * kTileK, tk);
                    b_issued[sb] = true;
                    b_phase[sb] = pb;
                }
            }
            // drain: every load this thread issued has landed before the CTA can exit
            for (int s = 0; s < kAStages; ++s)
                if (c_issued[s]) mbar_wait(&full_c[s], c_phase[s]);
            for (int s = 0; s < kBStages; ++s)
                if (b_issued[s]) mbar_wait(&full_b[s], b_phase[s]);
        }
    } else if (warp == 1) {
        // --------------------------------------------------------------- MMA issuer
        if (lane == 0) {
            constexpr uint32_t idesc = idesc_bf16(kTileM, kTileN, kBwd ? 1 : 0, 0);
            bool stop = false;
            // phase of the last commit to each slot's release barrier (-1: none)
            int last_a[kAStages], last_b[kBStages];
            for (int s = 0; s < kAStages; ++s) last_a[s] = -1;
            for (int s = 0; s < kBStages; ++s) last_b[s] = -1;
            for (int i = 0; i < T && !stop && !*abort_flag; ++i) {
                const int sa = i % kAStages;
                const uint32_t pa = (i / kAStages) & 1u;
                if (!mbar_wait(&full_a[sa], pa)) {
                    fail();
                    break;
                }
                int nk = 4;
                if (i >= nred) {
                    const int rem = p.r - (i - nred) * kTileK;
                    nk = rem >= kTileK ? 4 : (rem + 15) / 16;
                }
                const uint32_t a_base = smem_u32(sA + sa * kABytes);
                for (int h = 0; h < nh; ++h) {
                    const int j = i * nh + h;
                    const int sb = j % kBStages;
                    const uint32_t pb = (j / kBStages) & 1u;
                    if (!mbar_wait(&full_b[sb], pb)) {
                        fail();
                        stop = true;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t b_base = smem_u32(sB + sb * kBBytes);
                    for (int kk = 0; kk < nk; ++kk) {
                        // fwd A: K-major, 16 elements = 32 bytes along the swizzled row.
                        // bwd A: MN-major, 16 reduction rows = two 8-row groups of 1024 bytes;
                        //        the two 64-feature chunks are 8192 bytes apart.
                        const uint64_t ad = kBwd ? smem_desc_sw128(a_base + kk * 2048, 8192, 1024)
                                                 : smem_desc_sw128(a_base + kk * 32, 16, 1024);
                        const uint64_t bd = smem_desc_sw128(b_base + kk * 32, 16, 1024);
                        mma_bf16_ss(tmem_d + static_cast<uint32_t>(h * kTileN), ad, bd, idesc,
                                    (i > 0 || kk > 0) ? 1u : 0u);
                    }
                    mma_commit(&empty_b[sb]);
                    last_b[sb] = static_cast<int>(pb);
                }
                if (stop) break;
                mma_commit(&empty_a[sa]);
                last_a[sa] = static_cast<int>(pa);
            }
            mma_commit(acc_full);  // arrives when every issued MMA has completed
            // The commits arrive asynchronously when the MMAs complete. Wait for the last one of
            // every slot: an arrival still in flight when the CTA exits could land on the
            // barriers of the next CTA that this SM runs.
            for (int s = 0; s < kAStages; ++s)
                if (last_a[s] >= 0) mbar_wait(&empty_a[s], static_cast<uint32_t>(last_a[s]));
            for (int s = 0; s < kBStages; ++s)
                if (last_b[s] >= 0) mbar_wait(&empty_b[s], static_cast<uint32_t>(last_b[s]));
        }
    } else {
        // ----------------------------------------------------------- dequant groups
        const int dw = warp - 2;
        const int grp = dw >> 2;                  // stages i with i % kDqGroups == grp
        const int tid = (dw & 3) * 32 + lane;     // 0..127 within the group
        const float mu = load_mu(p.mu, p.absmax);
        // fwd: thread = A row (weight row row0 + tid), 64 k per stage.
        // bwd: thread = (reduction row tid/2 of the stage, feature half tid%2).
        const uint32_t arow = kBwd ? static_cast<uint32_t>(tid >> 1) : static_cast<uint32_t>(tid);
        const uint32_t half = kBwd ? static_cast<uint32_t>(tid & 1) : 0u;
        const int64_t kf = row0 + 64 * half;  // bwd: first feature of this thread's block
        const bool bwd_kvalid = !kBwd || kf < K;

        // The block's codes arrive by TMA into sC; its constant inputs (one byte and one float, or
        // the fp32 constant itself in sg) are loaded one of this group's stages ahead.
        auto load_const = [&](int i, uint32_t &qb, float &sg, bool &valid) {
            valid = false;
            qb = 0u;
            sg = 0.0f;
            if (i >= nred) return;
            int64_t wrow, blk;
            if (kBwd) {
                wrow = static_cast<int64_t>(i) * kTileK + arow;
                if (wrow >= N || !bwd_kvalid) return;
                blk = wrow * nbr + kf / kBlock;
            } else {
                wrow = row0 + arow;
                if (wrow >= N) return;
                blk = wrow * nbr + i;
            }
            if (p.absmax) {
                sg = __ldg(p.absmax + blk);
            } else {
                qb = __ldg(p.q + blk);
                sg = __ldg(p.sigma + blk / kGroup);
            }
            valid = true;
        };
        const uint32_t c_off = kBwd ? arow * 64u + half * 32u : arow * 32u;  // this thread's block in sC

        uint32_t nq;
        float ns;
        bool nv;
        load_const(grp, nq, ns, nv);
        for (int i = grp; i < T; i += kDqGroups) {
            if (*abort_flag) break;
            const int s = i % kAStages;  // == grp: each group owns one A slot
            const uint32_t ph = (i / kAStages) & 1u;
            const uint32_t cq = nq;
            const float cs = ns;
            const bool cv = nv;
            load_const(i + kDqGroups, nq, ns, nv);  // prefetch this group's next stage
            if (i >= kAStages && !mbar_wait(&empty_a[s], ph ^ 1u)) {
                fail();
                break;
            }
            // every thread waits for the stage's codes, so the slot is never refilled while a
            // load into it is still in flight
            if (i < nred && !mbar_wait(&full_c[s], ph)) {
                fail();
                break;
            }
            uint4 c0 = make_uint4(0u, 0u, 0u, 0u), c1 = c0;
            if (i < nred) {
                if (cv) {
                    const uint4 *src = reinterpret_cast<const uint4 *>(sC + s * kCBytes + c_off);
                    c0 = src[0];
                    c1 = src[1];
                }
                __syncwarp();  // the whole warp has read its codes: the slot may be refilled
                if (lane == 0) mbar_arrive(&empty_c[s]);
            }
            const uint32_t a_base = smem_u32(sA + s * kABytes);
            // destination of chunk j (8 elements) of this thread's 64-element run
            auto dst = [&](uint32_t j) -> uint32_t {
                return kBwd ? a_base + half * 8192u + (arow >> 3) * 1024u + swz(arow & 7u, j)
                            : a_base + swz(arow, j);
            };
            if (i < nred) {
                if (cv) {
                    const Planes P =
                        make_planes<kQT>(p.absmax ? cs : block_constant(static_cast<uint8_t>(cq), cs, mu));
                    const uint32_t w[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
#pragma unroll
                    for (int j = 0; j < 8; ++j) sts128(dst(j), expand8(P, w[j]));
                } else {
#pragma unroll
                    for (int j = 0; j < 8; ++j) sts128(dst(j), make_uint4(0u, 0u, 0u, 0u));
                }
            } else {
                // adapter stage: fwd copies row (row0 + arow) of B (n x r), columns
                // [64c, 64c + 64); bwd copies row (64c + arow) of A (r x k), features [kf, kf + 64).
                const int c = i - nred;
                const uint16_t *src = nullptr;
                int count = 0;
                if (kBwd) {
                    const int j = c * kTileK + static_cast<int>(arow);
                    if (j < p.r && bwd_kvalid) {
                        src = p.lora + static_cast<int64_t>(j) * K + kf;
                        count = 64;
                    }
                } else {
                    const int64_t wrow = row0 + arow;
                    if (wrow < N) {
                        src = p.lora + wrow * p.r + c * kTileK;
                        const int rem = p.r - c * kTileK;
                        count = rem < 64 ? rem : 64;
                    }
                }
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    uint4 v = make_uint4(0u, 0u, 0u, 0u);
                    if (src && 8 * j < count) {
                        if (8 * j + 8 <= count && ((reinterpret_cast<uintptr_t>(src + 8 * j) & 15u) == 0)) {
                            v = __ldg(reinterpret_cast<const uint4 *>(src + 8 * j));
                        } else {
                            uint32_t e[8];
#pragma unroll
                            for (int x = 0; x < 8; ++x) e[x] = (8 * j + x < count) ? ld_ro_u16(src + 8 * j + x) : 0u;
                            v = make_uint4(e[0] | (e[1] << 16), e[2] | (e[3] << 16), e[4] | (e[5] << 16),
                                           e[6] | (e[7] << 16));
                        }
                    }
                    sts128(dst(j), v);
                }
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(&full_a[s]);
        }

        // --------------------------------------------------------------- epilogue
        grid_dependents_launch();
        const bool ok = mbar_wait(acc_full, 0) && !*abort_flag;
        if (!ok) fail();
        tc_fence_after();
        const uint32_t quarter = static_cast<uint32_t>(warp & 3);  // TMEM lanes this warp may access
        const int64_t orow = row0 + quarter * 32 + lane;           // fwd: n; bwd: feature k
        const int64_t ldo = kBwd ? K : N;
        const bool rvalid = orow < (kBwd ? K : N);
        // With 16-byte aligned output rows and a full 128-row tile, each 32-token chunk is staged
        // through the group's (now idle) A slot as [32 tokens][128 rows] bf16 and written with
        // 16-byte stores, 256 contiguous bytes per token; otherwise one 2-byte store per value.
        // (vec is the same for every thread of the CTA, so all four warps of a group reach the
        // group barrier equally often; `ok` only gates the global stores)
        const bool vec = (ldo % 8 == 0) && (row0 + kTileM <= (kBwd ? K : N));
        uint16_t *stage = reinterpret_cast<uint16_t *>(sA + grp * kABytes);  // 2 x [32][128] bf16
        int buf = 0;
        for (int cb = grp; cb < nh * kTileN / 32; cb += kDqGroups) {  // 32-column chunks of this group
            uint32_t v[32];
            tmem_ld32(tmem_d + ((quarter * 32u) << 16) + static_cast<uint32_t>(cb * 32), v);
            tmem_ld_wait();
            if (vec) {
                uint16_t *S = stage + buf * (32 * kTileM);
#pragma unroll
                for (int c = 0; c < 32; ++c)
                    S[c * kTileM + quarter * 32 + lane] = __bfloat16_as_ushort(__float2bfloat16_rn(__uint_as_float(v[c])));
                // the group's four warps (128 threads) hold the chunk's four quarters; double
                // buffering makes one barrier per chunk enough
                asm volatile("bar.sync %0, %1;" ::"r"(1 + grp), "r"(128) : "memory");
#pragma unroll
                for (int kq = 0; kq < 4; ++kq) {
                    const int e = tid + 128 * kq;  // 16-byte piece: token e / 16, rows 8 (e % 16) .. + 8
                    const int c = e >> 4, pr = (e & 15) * 8;
                    const int64_t m = tok0 + cb * 32 + c;
                    if (ok && m < p.M)
                        *reinterpret_cast<uint4 *>(p.out + m * ldo + row0 + pr) =
                            *reinterpret_cast<const uint4 *>(S + c * kTileM + pr);
                }
                buf ^= 1;
            } else if (ok && rvalid) {
#pragma unroll
                for (int c = 0; c < 32; ++c) {
                    const int64_t m = tok0 + cb * 32 + c;
                    if (m < p.M) p.out[m * ldo + orow] = __bfloat16_as_ushort(__float2bfloat16_rn(__uint_as_float(v[c])));
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) tmem_dealloc(tmem_d, kTmemCols);
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    if (!fn) {
        cudaDriverEntryPointQueryResult qres;
        void *ptr = nullptr;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &qres) == cudaSuccess &&
            qres == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
    }
    return fn;
}

// 2-D bf16 tensor map over a row-major rows x cols matrix, box 64 (cols) x 256 (rows),
// 128-byte swizzle, zero fill out of bounds.
bool make_map(CUtensorMap *m, const void *base, int64_t rows, int64_t cols) {
    auto fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
    cuuint64_t strides[1] = {static_cast<cuuint64_t>(cols) * 2};
    cuuint32_t box[2] = {static_cast<cuuint32_t>(kTileK), static_cast<cuuint32_t>(kTileN)};
    cuuint32_t estr[2] = {1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 2-D uint8 tensor map over the packed codes (n rows of k/2 bytes), no swizzle, zero fill out
// of bounds. Box: fwd 32 bytes (one block) x 128 rows; bwd 64 bytes (two blocks) x 64 rows.
bool make_codes_map(CUtensorMap *m, const void *codes, int64_t n, int64_t k, bool bwd) {
    auto fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[2] = {static_cast<cuuint64_t>(k / 2), static_cast<cuuint64_t>(n)};
    cuuint64_t strides[1] = {static_cast<cuuint64_t>(k / 2)};
    cuuint32_t box[2] = {bwd ? 64u : 32u, bwd ? 64u : 128u};
    cuuint32_t estr[2] = {1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void *>(codes), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <bool kBwd, int kQT>
cudaError_t launch_gemm_impl(const WeightView &w, const uint16_t *act, int64_t M, const uint16_t *lora_rows, int r,
                             const uint16_t *lora_act, int RT, uint16_t *out, int *err, cudaStream_t st) {
    CUtensorMap tm_act, tm_lora, tm_codes;
    const int64_t act_cols = kBwd ? w.n : w.k;
    if (!make_map(&tm_act, act, M, act_cols)) return cudaErrorInvalidValue;
    if (!make_codes_map(&tm_codes, w.codes, w.n, w.k, kBwd)) return cudaErrorInvalidValue;
    if (r > 0) {
        if (!make_map(&tm_lora, lora_act, M, RT)) return cudaErrorInvalidValue;
    } else {
        tm_lora = tm_act;  // never read
    }
    // The shared-memory limit is a per-device attribute: set once per (host thread, device).
    static thread_local uint64_t configured = 0;  // bit d: device d is configured
    int dev = 0;
    cudaError_t ge = cudaGetDevice(&dev);
    if (ge != cudaSuccess) return ge;
    const uint64_t bit = (dev >= 0 && dev < 64) ? (uint64_t(1) << dev) : 0;
    if (bit == 0 || !(configured & bit)) {
        cudaError_t e = cudaFuncSetAttribute(k_gemm_nf4<kBwd, kQT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             static_cast<int>(kGemmSmem));
        if (e != cudaSuccess) return e;
        configured |= bit;
    }
    GemmParams p{w.codes, w.q, w.sigma, w.mu, w.absmax, w.n, w.k, M, lora_rows, r, out, err};
    const int64_t tiles_m = ((kBwd ? w.k : w.n) + kTileM - 1) / kTileM;
    const int64_t tiles_n = (M + kTileN * kHalves - 1) / (kTileN * kHalves);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(tiles_m), static_cast<unsigned>(tiles_n), 1);
    cfg.blockDim = dim3(kGemmThreads, 1, 1);
    cfg.dynamicSmemBytes = kGemmSmem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cudaError_t e = cudaLaunchKernelEx(&cfg, k_gemm_nf4<kBwd, kQT>, tm_act, tm_lora, tm_codes, p);
    count_launch();
    return e;
}

}  // namespace

size_t gemm_workspace_bytes(int64_t M, int r) {
    const int64_t RT = (r + 63) / 64 * 64;
    return 256 + ((static_cast<size_t>(M * RT) * 2 + 255) & ~size_t(255));
}

bool gemm_supported(int64_t n, int64_t k, int64_t M, bool bwd) {
    // The token operand is read by TMA, whose row stride must be a multiple of 16 bytes:
    // x (M x k) always is (k % 64 == 0); grad_h (M x n) needs n % 8 == 0.
    return (k % 64 == 0) && M > 0 && (!bwd || n % 8 == 0);
}

cudaError_t launch_gemm_fwd(const WeightView &w, const uint16_t *x, int64_t M, const uint16_t *A, const uint16_t *B,
                            int r, float s, uint16_t *h, void *ws, cudaStream_t st, const DropoutArgs *drop) {
    int *err = static_cast<int *>(ws);
    uint16_t *t = reinterpret_cast<uint16_t *>(static_cast<char *>(ws) + 256);
    const int RT = (r + 63) / 64 * 64;
    // the error word is sticky: kernels only ever set it (qlora_workspace_check reads and clears it)
    if (r > 0) {
        cudaError_t e = launch_lora_down(x, M, w.k, A, w.k, 1, r, s, t, RT, st, drop);
        if (e != cudaSuccess) return e;
    }
    return w.qtype == kQuantFP4 ? launch_gemm_impl<false, kQuantFP4>(w, x, M, B, r, t, RT, h, err, st)
                                : launch_gemm_impl<false, kQuantNF4>(w, x, M, B, r, t, RT, h, err, st);
}

cudaError_t launch_gemm_bwd(const WeightView &w, const uint16_t *gh, int64_t M, const uint16_t *A, const uint16_t *B,
                            int r, float s, uint16_t *gx, void *ws, cudaStream_t st) {
    int *err = static_cast<int *>(ws);
    uint16_t *u = reinterpret_cast<uint16_t *>(static_cast<char *>(ws) + 256);
    const int RT = (r + 63) / 64 * 64;
    if (r > 0) {
        cudaError_t e = launch_lora_down(gh, M, w.n, B, 1, r, r, s, u, RT, st);
        if (e != cudaSuccess) return e;
    }
    return w.qtype == kQuantFP4 ? launch_gemm_impl<true, kQuantFP4>(w, gh, M, A, r, u, RT, gx, err, st)
                                : launch_gemm_impl<true, kQuantNF4>(w, gh, M, A, r, u, RT, gx, err, st);
}

}  // namespace qn
