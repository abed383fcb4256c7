// stream_common.cuh -- pieces shared by the streamed few-token kernels (forward in
// decode_fwd.cu, input gradient in decode_bwd.cu): the bf16-pair table, shared-memory loads,
// cluster barriers, the launch-shape planner and the error word.
//
// The pair table: a code byte (two nibbles) maps to a bf16 pair of table values (NF4 or the
// 4-bit float), bf16x2(T[byte & 15], T[byte >> 4]). It is stored once per lane in 256-byte rows, so the
// byte permute that extracts a byte also forms the conflict-free address (byte << 8 | lane << 2);
// 64 KB per CTA, of which the second half of every row is unused (a packed 32 KB table needs one
// more shift per lookup and measured slower). NF4 values: "QLoRA paper notes" (tqpw.cn),
// "NormalFloat Quantization (NF4)".
#pragma once

#include <cooperative_groups.h>

#include "common.cuh"
#include "kernels.h"
#include "sm100.cuh"

namespace qn {
namespace stream {

namespace cg = cooperative_groups;

constexpr int kLutBytes = 256 * 256;
// Low 24 bits of the shared-window address of dynamic shared memory when the driver reserves
// 1 KB per CTA and the kernel has no static shared memory; in a cluster launch the CTA's rank
// sits above them. Kernels check it at run time and otherwise take the generic table path.
constexpr uint32_t kDynSmemBase = 1024;
constexpr int kErrTimeout = 1;  // error word value: a bounded wait ran out
constexpr int kErrLayout = 2;   // error word value: dynamic shared memory not 1024-byte aligned

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
    uint32_t d;
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
    return d;
}

__device__ __forceinline__ uint32_t saddr(const void *p) { return static_cast<uint32_t>(__cvta_generic_to_shared(p)); }

// Shared-memory loads. Volatile, so that they stay behind the mbarrier waits that make the
// data they read valid.
__device__ __forceinline__ uint32_t lds32(uint32_t a) {
    uint32_t v;
    asm volatile("ld.shared.b32 %0, [%1];" : "=r"(v) : "r"(a));
    return v;
}
__device__ __forceinline__ uint32_t lds8(uint32_t a) {
    uint32_t v;
    asm volatile("ld.shared.u8 %0, [%1];" : "=r"(v) : "r"(a));
    return v;
}
__device__ __forceinline__ uint2 lds64(uint32_t a) {
    uint2 v;
    asm volatile("ld.shared.v2.b32 {%0,%1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(a));
    return v;
}
__device__ __forceinline__ uint4 lds128(uint32_t a) {
    uint4 v;
    asm volatile("ld.shared.v4.b32 {%0,%1,%2,%3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(a));
    return v;
}

// Row e of the pair table (a code byte) holds bf16x2(T[e & 15], T[e >> 4]) in its first 32
// words, one copy per lane (T: the table of quant type qtype). The eight 16-byte stores of a row
// start at a column rotated by the row so that the lanes of a warp hit different banks.
__device__ __forceinline__ void build_pair_lut(uint8_t *lut, int tid, int nthreads, int qtype) {
    uint4 *l4 = reinterpret_cast<uint4 *>(lut);
    for (int i = tid; i < 256 * 8; i += nthreads) {
        const int e = i >> 3, c = i & 7;
        const uint32_t v = pack_bf16x2(table_value(qtype, e & 15), table_value(qtype, e >> 4));
        l4[e * 16 + ((c + e) & 7)] = make_uint4(v, v, v, v);
    }
}

// Operand of the table permute: lane << 2 in byte 0 and, on the fixed-base path, the high
// byte (cluster rank) of the table's shared-window address in byte 3.
template <bool kFixedBase>
__device__ __forceinline__ uint32_t lut_lane_operand(const uint8_t *lut, int lane) {
    const uint32_t l4 = static_cast<uint32_t>(lane) << 2;
    return kFixedBase ? (l4 | (saddr(lut) & 0xff000000u)) : l4;
}

// Pair for byte i (0..3) of word w. The permute builds (byte << 8) | (lane << 2), plus the rank
// byte on the fixed-base path, where the table starts at the base of dynamic shared memory and
// its low address bits are an immediate of the load; otherwise the table address is added.
template <bool kFixedBase>
__device__ __forceinline__ uint32_t lut_pair(uint32_t lut_base, uint32_t w, uint32_t lane_op, int i) {
    if constexpr (kFixedBase) {
        const uint32_t a = prmt(w, lane_op, 0x7604u | (static_cast<uint32_t>(i) << 4));
        uint32_t v;
        asm volatile("ld.shared.b32 %0, [%1+%2];" : "=r"(v) : "r"(a), "n"(kDynSmemBase));
        return v;
    } else {
        const uint32_t off = prmt(w, lane_op, 0x5504u | (static_cast<uint32_t>(i) << 4));
        return lds32(lut_base + off);
    }
}

// First MMA of a chain: D = A * B with a zero accumulator.
__device__ __forceinline__ void mma_16816_z(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                            uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%10,%10,%10,%10};\n"
        : "=f"(d[0]), "=f"(d[1]), "=f"(d[2]), "=f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1), "f"(0.0f));
}

// 4-byte asynchronous copy global -> shared (the issuing thread reads it after a wait).
__device__ __forceinline__ void cp_async4(uint32_t dst, const void *src) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(dst), "l"(src) : "memory");
}
// 4-byte copy of which only the first `src_bytes` (0..4) are read; the rest is zero-filled.
__device__ __forceinline__ void cp_async4_zfill(uint32_t dst, const void *src, uint32_t src_bytes) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;" ::"r"(dst), "l"(src), "r"(src_bytes) : "memory");
}
// 16-byte copy global -> shared bypassing L1; only the first `src_bytes` (0 or 16) are read.
__device__ __forceinline__ void cp_async16_zfill(uint32_t dst, const void *src, uint32_t src_bytes) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(src_bytes) : "memory");
}
// Arrive on `bar` when every cp.async this thread issued so far has completed (the barrier's
// expected count includes this arrival).
__device__ __forceinline__ void cp_async_arrive_noinc(uint64_t *bar) {
    asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(saddr(bar)) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait_n() {
    asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}
// Wait until at most n (0 <= n <= 7) of this thread's committed copy groups are pending.
__device__ __forceinline__ void cp_async_wait_group(int n) {
    switch (n) {
        case 0: cp_async_wait_n<0>(); break;
        case 1: cp_async_wait_n<1>(); break;
        case 2: cp_async_wait_n<2>(); break;
        case 3: cp_async_wait_n<3>(); break;
        case 4: cp_async_wait_n<4>(); break;
        case 5: cp_async_wait_n<5>(); break;
        case 6: cp_async_wait_n<6>(); break;
        default: cp_async_wait_n<7>(); break;
    }
}

// Split cluster barrier.
__device__ __forceinline__ void cluster_arrive_relaxed() { asm volatile("barrier.cluster.arrive.relaxed.aligned;" ::: "memory"); }
__device__ __forceinline__ void cluster_arrive_release() { asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory"); }
__device__ __forceinline__ void cluster_wait() { asm volatile("barrier.cluster.wait.aligned;" ::: "memory"); }
__device__ __forceinline__ void cluster_wait_acquire() { asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory"); }

// Shared-window address `a` of this CTA mapped into the window of cluster rank `rank`.
__device__ __forceinline__ uint32_t mapa(uint32_t a, uint32_t rank) {
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(rank));
    return r;
}
// Asynchronous 8-byte store into a cluster CTA's shared memory; completes `bytes` on that
// CTA's mbarrier (both addresses from mapa).
__device__ __forceinline__ void st_async_v2(uint32_t addr, float a, float b, uint32_t mbar) {
    asm volatile("st.async.shared::cluster.mbarrier::complete_tx::bytes.v2.f32 [%0], {%1, %2}, [%3];" ::"r"(addr),
                 "f"(a), "f"(b), "r"(mbar)
                 : "memory");
}
// 4-byte global load that bypasses L1 (data another CTA published).
__device__ __forceinline__ uint32_t ld_cg_u32(const void *p) {
    uint32_t v;
    asm volatile("ld.global.cg.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}
__device__ __forceinline__ uint32_t ld_acquire_u32(const unsigned *p) {
    uint32_t v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}
__device__ __forceinline__ void st_release_u32(unsigned *p, uint32_t v) {
    asm volatile("st.release.gpu.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
// Bounded wait (nanosleep between polls, about a second in all) for a flag another CTA of the
// grid sets with release semantics; false when it runs out.
__device__ __forceinline__ bool wait_flag(const unsigned *flag) {
    for (uint32_t i = 0; i < (1u << 22); ++i) {
        if (ld_acquire_u32(flag) != 0u) return true;
        __nanosleep(128);
    }
    return false;
}

// Named barrier over `nthreads` threads (id 1..15; id 0 is __syncthreads).
__device__ __forceinline__ void named_sync(int id, int nthreads) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

// Record a failure in the caller's workspace error word (sticky until read back).
__device__ __forceinline__ void record_error(int *err, int code) {
    if (err) atomicExch(err, code);
}

// bf16 pair (B[row][j], B[row][j + 1]) of a row-major rows x r matrix, zero outside it.
__device__ __forceinline__ uint32_t load_pair_rowmajor(const uint16_t *B, int64_t row, bool valid, int j, int r) {
    if (!valid || j >= r) return 0u;
    const uint16_t *b = B + row * r + j;
    if ((r & 1) == 0) return ld_ro_u32(b);  // j even and r even: 4-byte aligned
    const uint32_t lo = ld_ro_u16(b);
    const uint32_t hi = j + 1 < r ? ld_ro_u16(b + 1) : 0u;
    return lo | (hi << 16);
}

}  // namespace stream
}  // namespace qn
