// decode_common.cuh -- pieces shared by the few-token (M <= 64) kernels of decode.cu (forward)
// and decode_bwd.cu (input gradient): the parameter block, the bf16-pair table, prefetch and
// cluster-barrier helpers and the cluster-launch helpers. Everything sits in an anonymous
// namespace, so each translation unit has its own copy (and its own host-side caches).
//
// The table: a code byte (two nibbles) maps to a bf16 pair of NF4 values. It is stored once per
// lane in 256-byte rows, so the permute that extracts a byte also forms the conflict-free
// address (byte << 8 | lane << 2); 64 KB per CTA, of which the second half of every row is
// unused. NF4 table: "QLoRA paper notes" (tqpw.cn), "NormalFloat Quantization (NF4)".
#pragma once
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
    const float *absmax;  // fp32 block constants (no double quantisation), else nullptr
    int qtype;            // table of the code nibbles (kQuantNF4 or kQuantFP4)
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

// Pair table: row e (a code byte) holds bf16x2(T[e & 15], T[e >> 4]) in its first 32 words, one
// copy per lane (T: the table of quant type qtype). One row per thread; the eight 16-byte stores
// of a row start at a column rotated by the row so that the lanes of a warp hit different banks.
__device__ __forceinline__ void build_pair_lut(uint8_t *lut, int qtype) {
    uint4 *l4 = reinterpret_cast<uint4 *>(lut);
    for (int e = threadIdx.x; e < 256; e += blockDim.x) {
        const uint32_t v = pack_bf16x2(table_value(qtype, e & 15), table_value(qtype, e >> 4));
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

// Deterministic sum over the CTA's warps of one 16-row MMA accumulator tile d[NG][4] (row g or
// g + 8, token tg*8 + 2t (+1)): a pairwise tree in a fixed order (w += w + 4, w += w + 2,
// w += w + 1) through `scratch` (kDecWarps / 2 x 16 x MP floats); warp 0 writes the result to
// dst[row * MP + token]. Every warp of the CTA must call it (it contains __syncthreads).
template <int NG>
__device__ __forceinline__ void warp_tree_sum(float (&d)[NG][4], float *scratch, float *dst) {
    constexpr int MP = 8 * NG;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
#pragma unroll
    for (int half = kDecWarps / 2; half >= 1; half >>= 1) {
        if (warp >= half && warp < 2 * half) {
            float *sp = scratch + (warp - half) * 16 * MP;
#pragma unroll
            for (int tg = 0; tg < NG; ++tg) {
                *reinterpret_cast<float2 *>(sp + g * MP + tg * 8 + 2 * t) = make_float2(d[tg][0], d[tg][1]);
                *reinterpret_cast<float2 *>(sp + (g + 8) * MP + tg * 8 + 2 * t) = make_float2(d[tg][2], d[tg][3]);
            }
        }
        __syncthreads();
        if (warp < half) {
            const float *sp = scratch + warp * 16 * MP;
#pragma unroll
            for (int tg = 0; tg < NG; ++tg) {
                const float2 u = *reinterpret_cast<const float2 *>(sp + g * MP + tg * 8 + 2 * t);
                const float2 v = *reinterpret_cast<const float2 *>(sp + (g + 8) * MP + tg * 8 + 2 * t);
                d[tg][0] += u.x;
                d[tg][1] += u.y;
                d[tg][2] += v.x;
                d[tg][3] += v.y;
            }
        }
        __syncthreads();
    }
    if (warp == 0) {
#pragma unroll
        for (int tg = 0; tg < NG; ++tg) {
            *reinterpret_cast<float2 *>(dst + g * MP + tg * 8 + 2 * t) = make_float2(d[tg][0], d[tg][1]);
            *reinterpret_cast<float2 *>(dst + (g + 8) * MP + tg * 8 + 2 * t) = make_float2(d[tg][2], d[tg][3]);
        }
    }
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
}  // namespace qn
