// common.cuh -- device helpers shared by the sm_100a kernels of the NF4 + LoRA linear layer.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace qn {

constexpr int kBlock = 64;   // weights per absmax block
constexpr int kGroup = 256;  // blocks per double-quantisation group

// The 16 NF4 values, ascending, as printed in "QLoRA paper notes" (tqpw.cn),
// section "NormalFloat Quantization (NF4)". Each is an exact fp32 value.
#define QN_NF4_VALUES                                                                       \
    {-1.0f, -0.6961928009986877f, -0.5250730514526367f, -0.39491748809814453f,              \
     -0.28444138169288635f, -0.18477343022823334f, -0.09105003625154495f, 0.0f,            \
     0.07958029955625534f, 0.16093020141124725f, 0.24611230194568634f, 0.33791524171829224f, \
     0.44070982933044434f, 0.5626170039176941f, 0.7229568362236023f, 1.0f}

// The other quant type, the 4-bit float E2M1 (sign, two exponent bits with bias 1, one
// mantissa bit): codes 0-7 are the magnitudes 0, 0.5, 1, 1.5, 2, 3, 4, 6 divided by the
// largest, 6, each the nearest fp32 value; codes 8-15 are their negatives (8 is -0, which the
// quantiser never produces). The quant-type knob: "Quantized LoRA (QLoRA) and 4-bit training"
// (apxml.com), the four configuration knobs; "QLoRA paper notes" (tqpw.cn), Experiments.
#define QN_FP4_VALUES                                                                                 \
    {0.0f,   0x1.555556p-4f,  0x1.555556p-3f,  0x1p-2f,  0x1.555556p-2f,  0x1p-1f,  0x1.555556p-1f,  1.0f, \
     -0.0f, -0x1.555556p-4f, -0x1.555556p-3f, -0x1p-2f, -0x1.555556p-2f, -0x1p-1f, -0x1.555556p-1f, -1.0f}

constexpr int kQuantNF4 = 0;
constexpr int kQuantFP4 = 1;

static __constant__ float c_tables[2][16] = {QN_NF4_VALUES, QN_FP4_VALUES};

// Value of code i (0..15) of quant type qtype (kQuantNF4 or kQuantFP4).
__host__ __device__ inline float table_value(int qtype, int i) {
#ifdef __CUDA_ARCH__
    return c_tables[qtype][i];
#else
    constexpr float T[2][16] = {QN_NF4_VALUES, QN_FP4_VALUES};
    return T[qtype][i];
#endif
}

__host__ __device__ inline float nf4_value(int i) { return table_value(kQuantNF4, i); }

// ---------------------------------------------------------------- loads

__device__ __forceinline__ uint4 ld_nc_v4(const void *p) {
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

__device__ __forceinline__ uint2 ld_nc_v2(const void *p) {
    uint2 v;
    asm volatile("ld.global.nc.L1::no_allocate.v2.u32 {%0,%1}, [%2];" : "=r"(v.x), "=r"(v.y) : "l"(p));
    return v;
}

__device__ __forceinline__ uint32_t ld_nc_u32(const void *p) {
    uint32_t v;
    asm volatile("ld.global.nc.L1::no_allocate.u32 %0, [%1];" : "=r"(v) : "l"(p));
    return v;
}

// Cached (L1) read-only loads for small operands that many warps re-read.
__device__ __forceinline__ uint4 ld_ro_v4(const void *p) { return __ldg(reinterpret_cast<const uint4 *>(p)); }
__device__ __forceinline__ uint2 ld_ro_v2(const void *p) { return __ldg(reinterpret_cast<const uint2 *>(p)); }
__device__ __forceinline__ uint32_t ld_ro_u32(const void *p) { return __ldg(reinterpret_cast<const unsigned int *>(p)); }
__device__ __forceinline__ uint16_t ld_ro_u16(const void *p) { return __ldg(reinterpret_cast<const unsigned short *>(p)); }

// ------------------------------------------------------------ numerics

// E4M3 (finite variant) -> fp32, exact. Exponent and mantissa bits are moved into the fp32
// fields, which reads the value scaled by 2^(7 - 127) (e4m3 bias 7, fp32 bias 127; a zero
// exponent gives an fp32 subnormal, matching the e4m3 subnormal); one exact multiply by 2^120
// restores the scale. The two NaN codes (0x7f, 0xff) are never produced by the quantiser.
__device__ __forceinline__ float e4m3_to_f32(uint8_t v) {
    const uint32_t u = v;
    return __uint_as_float(((u & 0x7fu) << 20) | ((u & 0x80u) << 24)) * 0x1p120f;
}

__device__ __forceinline__ uint8_t f32_to_e4m3_satfinite(float v) {
    return static_cast<uint8_t>(__nv_cvt_float_to_fp8(v, __NV_SATFINITE, __NV_E4M3));
}

// Block constant c'_b = fma(decode(q_b), sigma_g, mu), single rounding.
__device__ __forceinline__ float block_constant(uint8_t q, float sigma, float mu) {
    return __fmaf_rn(e4m3_to_f32(q), sigma, mu);
}

// Block constant b read from global memory: c'_b with double quantisation (mu already loaded),
// else the stored fp32 absmax (absmax != nullptr).
__device__ __forceinline__ float load_block_constant(const uint8_t *q, const float *sigma, float mu,
                                                     const float *absmax, int64_t b) {
    return absmax ? __ldg(absmax + b) : block_constant(__ldg(q + b), __ldg(sigma + b / kGroup), mu);
}
// mu of a weight with double-quantised constants (0 when they are fp32).
__device__ __forceinline__ float load_mu(const float *mu, const float *absmax) { return absmax ? 0.0f : __ldg(mu); }

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&v);
}

__device__ __forceinline__ float bf16_lo(uint32_t v) { return __uint_as_float(v << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t v) { return __uint_as_float(v & 0xffff0000u); }

// D = A(16x16, row) * B(16x8, col) + C, bf16 inputs, fp32 accumulate.
__device__ __forceinline__ void mma_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                          uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};\n"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// ------------------------------------------------------- programmatic launch
// Wait until the preceding grid on the stream has completed (no-op when the
// kernel was not launched as a programmatic dependent).
__device__ __forceinline__ void grid_dependency_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void grid_dependents_launch() { asm volatile("griddepcontrol.launch_dependents;"); }

}  // namespace qn
