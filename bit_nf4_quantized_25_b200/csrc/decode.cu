// decode.cu -- QLoRA linear forward and input gradient for few tokens (M <= 64) on sm_100a.
//
//   fwd : h[m,n]      = sum_k W'[n,k] x[m,k]      + s * sum_j B[n,j] t[m,j],  t = A x
//   bwd : grad_x[m,k] = sum_n grad_h[m,n] W'[n,k] + s * sum_j A[j,k] u[m,j],  u = B^T grad_h
// with W'[n,k] = NF4[code] * c'_b ("Quantized LoRA (QLoRA) and 4-bit training", apxml.com,
// forward equations; "How does QLoRA work for training?", aivaro.ru, sections 2 and 7).
//
// Few tokens make this HBM-bound: every packed weight is read once and used M times.
// B200 streams weights faster than CUDA cores can expand and multiply 4-bit codes, so
// the multiply-accumulate runs on the tensor cores (mma.sync m16n8k16, A = weights,
// B = tokens) and the per-weight work is one byte-indexed load from a shared-memory
// table that maps a code byte (two nibbles) straight to a bf16 pair:
//   - fwd: the table holds the unscaled NF4 values; each 64-weight block is reduced
//     into its own fp32 fragment and scaled by its constant c'_b in fp32 (the
//     block constant is applied after the dot product, which is the same sum).
//   - bwd: the reduction runs over rows, whose constants differ, so the constants are
//     folded into the bf16 token operand instead (c'_b * grad_h), and code nibbles of
//     neighbouring rows are interleaved so that a byte again indexes a bf16 pair.
// The contraction is split across a thread-block cluster (up to 8 CTAs); partial sums
// and the LoRA down-projection are exchanged through distributed shared memory, so the
// whole layer is one launch with no workspace.
#include <cooperative_groups.h>

#include "common.cuh"
#include "kernels.h"

namespace cg = cooperative_groups;

namespace qn {

namespace {

constexpr int kDecWarps = 4;
constexpr int kDecThreads = kDecWarps * 32;
constexpr int kLutBytes = 256 * 32 * 4;  // 256 code bytes x 32 lane copies x bf16 pair
constexpr int kMaxCluster = 8;
constexpr int kBatch = 8;      // 64-weight blocks per batch of loads (forward)
constexpr int kStepBatch = 4;  // 16-row steps per batch of loads (input gradient)

struct DecodeParams {
    const uint8_t *codes;
    const uint8_t *q;
    const float *sigma;
    const float *mu;
    int64_t n, k;         // W is n x k
    const uint16_t *act;  // fwd: x (M x k); bwd: grad_h (M x n)
    int M;
    const uint16_t *A;  // r x k
    const uint16_t *B;  // n x r
    int r;
    float s;
    uint16_t *out;  // fwd: h (M x n); bwd: grad_x (M x k)
};

// Pair table: entry e (a code byte) = bf16x2(NF4[e & 15], NF4[e >> 4]); each entry is
// stored once per lane so a warp's 32 random lookups hit 32 different banks.
__device__ __forceinline__ void build_pair_lut(uint32_t *lut) {
    __shared__ uint32_t s_t16[16];
    if (threadIdx.x < 16) s_t16[threadIdx.x] = __float_as_uint(nf4_value(threadIdx.x));
    __syncthreads();
    uint4 *l4 = reinterpret_cast<uint4 *>(lut);
    for (int i = threadIdx.x; i < 256 * 8; i += blockDim.x) {
        const int e = i >> 3;
        const uint32_t v = pack_bf16x2(__uint_as_float(s_t16[e & 15]), __uint_as_float(s_t16[e >> 4]));
        l4[i] = make_uint4(v, v, v, v);
    }
}

__device__ __forceinline__ uint32_t lut_get(const uint32_t *lut, uint32_t byte, int lane) {
    return lut[(byte << 5) | lane];
}

__device__ __forceinline__ uint32_t byte_of(uint32_t w, int i) { return (w >> (8 * i)) & 0xffu; }

__device__ __forceinline__ float round_bf16(float v) { return __bfloat162float(__float2bfloat16_rn(v)); }

// --------------------------------------------------------------------------- forward
template <int NG>
__global__ void __launch_bounds__(kDecThreads)
k_decode_fwd(const DecodeParams p) {
    constexpr int MP = 8 * NG;  // padded token count
    extern __shared__ __align__(16) uint8_t smem[];
    uint32_t *lut = reinterpret_cast<uint32_t *>(smem);
    float *part = reinterpret_cast<float *>(smem + kLutBytes);  // [64 rows][MP]
    const int rpad = (p.r + 15) & ~15;
    float *tpart = part + 64 * MP;     // [rpad][MP] partial A x of this CTA's k-slice
    float *tfull = tpart + rpad * MP;  // [rpad][MP] s * A x, rounded to bf16

    cg::cluster_group cluster = cg::this_cluster();
    const int C = static_cast<int>(cluster.num_blocks());
    const int crank = static_cast<int>(cluster.block_rank());
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, t = lane & 3;

    build_pair_lut(lut);
    for (int i = threadIdx.x; i < rpad * MP; i += blockDim.x) tpart[i] = 0.0f;
    __syncthreads();
    // Launched as a programmatic dependent: everything above overlaps the preceding
    // kernel; no global memory is read before this point.
    grid_dependency_wait();

    const int64_t N = p.n, K = p.k, nbr = K / kBlock;
    const int64_t b_lo = nbr * crank / C, b_hi = nbr * (crank + 1) / C;
    const float mu = __ldg(p.mu);
    const int M = p.M;

    // x fragments: lane (g, t) of token group tg holds x[tg*8+g][64b + 16t .. +16].
    const uint16_t *xrow[NG];
    bool xv[NG];
#pragma unroll
    for (int tg = 0; tg < NG; ++tg) {
        const int tok = tg * 8 + g;
        xv[tg] = tok < M;
        xrow[tg] = p.act + static_cast<int64_t>(xv[tg] ? tok : 0) * K + 16 * t;
    }

    // ---- base: rows n0+g and n0+g+8 of this warp's 16-row tile, blocks [b_lo, b_hi)
    {
        const int64_t rowA = static_cast<int64_t>(blockIdx.y) * 64 + warp * 16 + g;
        const int64_t rowB = rowA + 8;
        const bool vA = rowA < N, vB = rowB < N;
        const uint8_t *cA = p.codes + (vA ? rowA : 0) * (K / 2) + 8 * t;
        const uint8_t *cB = p.codes + (vB ? rowB : 0) * (K / 2) + 8 * t;
        const int64_t qA = (vA ? rowA : 0) * nbr, qB = (vB ? rowB : 0) * nbr;
        float acc[NG][4];
#pragma unroll
        for (int tg = 0; tg < NG; ++tg) acc[tg][0] = acc[tg][1] = acc[tg][2] = acc[tg][3] = 0.0f;

        // Batches of kBatch blocks: every load of a batch is issued before any use, so a
        // warp keeps 2 x kBatch x 8 bytes of codes per lane in flight.
        for (int64_t bb = b_lo; bb < b_hi; bb += kBatch) {
            const int nbk = static_cast<int>(b_hi - bb < kBatch ? b_hi - bb : kBatch);
            uint2 ca[kBatch], cb[kBatch];
            uint32_t qa[kBatch], qbv[kBatch];
#pragma unroll
            for (int j = 0; j < kBatch; ++j) {
                ca[j] = cb[j] = make_uint2(0u, 0u);
                qa[j] = qbv[j] = 0u;
                if (j < nbk) {
                    if (vA) {
                        ca[j] = __ldcs(reinterpret_cast<const uint2 *>(cA + (bb + j) * 32));
                        qa[j] = __ldg(p.q + qA + bb + j);
                    }
                    if (vB) {
                        cb[j] = __ldcs(reinterpret_cast<const uint2 *>(cB + (bb + j) * 32));
                        qbv[j] = __ldg(p.q + qB + bb + j);
                    }
                }
            }
            // a batch of <= 8 consecutive blocks touches at most two groups
            const int64_t gA0 = (qA + bb) / kGroup, gB0 = (qB + bb) / kGroup;
            const int64_t ng_all = (N * nbr + kGroup - 1) / kGroup;
            const float sA0 = __ldg(p.sigma + gA0), sA1 = __ldg(p.sigma + (gA0 + 1 < ng_all ? gA0 + 1 : gA0));
            const float sB0 = __ldg(p.sigma + gB0), sB1 = __ldg(p.sigma + (gB0 + 1 < ng_all ? gB0 + 1 : gB0));
#pragma unroll
            for (int j = 0; j < kBatch; ++j) {
                if (j >= nbk) break;
                const int64_t b = bb + j;
                const float cpA = vA ? block_constant(static_cast<uint8_t>(qa[j]),
                                                      (qA + b) / kGroup == gA0 ? sA0 : sA1, mu) : 0.0f;
                const float cpB = vB ? block_constant(static_cast<uint8_t>(qbv[j]),
                                                      (qB + b) / kGroup == gB0 ? sB0 : sB1, mu) : 0.0f;
                uint32_t af[4][4];
#pragma unroll
                for (int kk = 0; kk < 4; ++kk) {
                    const uint32_t wa = kk < 2 ? ca[j].x : ca[j].y, wb = kk < 2 ? cb[j].x : cb[j].y;
                    const int i0 = (2 * kk) & 3;
                    af[kk][0] = lut_get(lut, byte_of(wa, i0), lane);
                    af[kk][2] = lut_get(lut, byte_of(wa, i0 + 1), lane);
                    af[kk][1] = lut_get(lut, byte_of(wb, i0), lane);
                    af[kk][3] = lut_get(lut, byte_of(wb, i0 + 1), lane);
                }
#pragma unroll
                for (int tg = 0; tg < NG; ++tg) {
                    uint4 x0 = make_uint4(0u, 0u, 0u, 0u), x1 = x0;
                    if (xv[tg]) {
                        x0 = ld_ro_v4(xrow[tg] + b * 64);
                        x1 = ld_ro_v4(xrow[tg] + b * 64 + 8);
                    }
                    const uint32_t xw[8] = {x0.x, x0.y, x0.z, x0.w, x1.x, x1.y, x1.z, x1.w};
                    float d[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        mma_16816(d, af[kk][0], af[kk][1], af[kk][2], af[kk][3], xw[2 * kk], xw[2 * kk + 1]);
                    acc[tg][0] = __fmaf_rn(cpA, d[0], acc[tg][0]);
                    acc[tg][1] = __fmaf_rn(cpA, d[1], acc[tg][1]);
                    acc[tg][2] = __fmaf_rn(cpB, d[2], acc[tg][2]);
                    acc[tg][3] = __fmaf_rn(cpB, d[3], acc[tg][3]);
                }
            }
        }
        const int rl = warp * 16 + g;
#pragma unroll
        for (int tg = 0; tg < NG; ++tg) {
            part[rl * MP + tg * 8 + 2 * t] = acc[tg][0];
            part[rl * MP + tg * 8 + 2 * t + 1] = acc[tg][1];
            part[(rl + 8) * MP + tg * 8 + 2 * t] = acc[tg][2];
            part[(rl + 8) * MP + tg * 8 + 2 * t + 1] = acc[tg][3];
        }
    }

    // ---- LoRA down-projection over this CTA's k-slice: partial t = A x (fp32).
    // Work item (j-tile, quarter of the slice); warp w takes quarter w of every tile.
    if (p.r > 0) {
        const int rt = rpad / 16;
        const int64_t nb_sl = b_hi - b_lo;
        const int64_t s_lo = b_lo + nb_sl * warp / kDecWarps, s_hi = b_lo + nb_sl * (warp + 1) / kDecWarps;
        for (int jt = 0; jt < rt; ++jt) {
            const int jA = jt * 16 + g, jB = jA + 8;
            const bool vA = jA < p.r, vB = jB < p.r;
            const uint16_t *aA = p.A + static_cast<int64_t>(vA ? jA : 0) * K + 16 * t;
            const uint16_t *aB = p.A + static_cast<int64_t>(vB ? jB : 0) * K + 16 * t;
            float d[NG][4];
#pragma unroll
            for (int tg = 0; tg < NG; ++tg) d[tg][0] = d[tg][1] = d[tg][2] = d[tg][3] = 0.0f;
            for (int64_t b = s_lo; b < s_hi; ++b) {
                uint4 a0 = make_uint4(0u, 0u, 0u, 0u), a1 = a0, b0 = a0, b1 = a0;
                if (vA) {
                    a0 = ld_ro_v4(aA + b * 64);
                    a1 = ld_ro_v4(aA + b * 64 + 8);
                }
                if (vB) {
                    b0 = ld_ro_v4(aB + b * 64);
                    b1 = ld_ro_v4(aB + b * 64 + 8);
                }
                const uint32_t ra[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
                const uint32_t rb[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll
                for (int tg = 0; tg < NG; ++tg) {
                    uint4 x0 = make_uint4(0u, 0u, 0u, 0u), x1 = x0;
                    if (xv[tg]) {
                        x0 = ld_ro_v4(xrow[tg] + b * 64);
                        x1 = ld_ro_v4(xrow[tg] + b * 64 + 8);
                    }
                    const uint32_t xw[8] = {x0.x, x0.y, x0.z, x0.w, x1.x, x1.y, x1.z, x1.w};
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        mma_16816(d[tg], ra[2 * kk], rb[2 * kk], ra[2 * kk + 1], rb[2 * kk + 1], xw[2 * kk],
                                  xw[2 * kk + 1]);
                }
            }
#pragma unroll
            for (int tg = 0; tg < NG; ++tg) {
                const int jl = jt * 16 + g;
                atomicAdd(&tpart[jl * MP + tg * 8 + 2 * t], d[tg][0]);
                atomicAdd(&tpart[jl * MP + tg * 8 + 2 * t + 1], d[tg][1]);
                atomicAdd(&tpart[(jl + 8) * MP + tg * 8 + 2 * t], d[tg][2]);
                atomicAdd(&tpart[(jl + 8) * MP + tg * 8 + 2 * t + 1], d[tg][3]);
            }
        }
    }

    __syncthreads();
    cluster.sync();  // every CTA's partials are complete and visible in the cluster
    grid_dependents_launch();

    if (p.r > 0) {
        for (int i = threadIdx.x; i < rpad * MP; i += blockDim.x) {
            float sum = 0.0f;
            for (int cc = 0; cc < C; ++cc) sum += cluster.map_shared_rank(tpart, cc)[i];
            tfull[i] = round_bf16(sum * p.s);
        }
    }
    __syncthreads();

    // ---- this CTA finalises rows [64*crank/C, 64*(crank+1)/C) of the 64-row group
    const int r_lo = 64 * crank / C, r_hi = 64 * (crank + 1) / C, nr = r_hi - r_lo;
    for (int i = threadIdx.x; i < nr * M; i += blockDim.x) {
        const int rl = r_lo + i % nr, tok = i / nr;
        const int64_t n = static_cast<int64_t>(blockIdx.y) * 64 + rl;
        if (n >= N) continue;
        float sum = 0.0f;
        for (int cc = 0; cc < C; ++cc) sum += cluster.map_shared_rank(part, cc)[rl * MP + tok];
        if (p.r > 0) {
            const uint16_t *brow = p.B + n * p.r;
            float lora = 0.0f;
            for (int j = 0; j < p.r; ++j)
                lora = __fmaf_rn(__uint_as_float(static_cast<uint32_t>(ld_ro_u16(brow + j)) << 16), tfull[j * MP + tok], lora);
            sum += lora;
        }
        p.out[static_cast<int64_t>(tok) * N + n] = __bfloat16_as_ushort(__float2bfloat16_rn(sum));
    }
    cluster.sync();  // keep this CTA's shared memory alive until the cluster is done reading it
}

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

template <int NG>
__global__ void __launch_bounds__(kDecThreads)
k_decode_bwd(const DecodeParams p) {
    constexpr int MP = 8 * NG;
    extern __shared__ __align__(16) uint8_t smem[];
    uint32_t *lut = reinterpret_cast<uint32_t *>(smem);
    float *part = reinterpret_cast<float *>(smem + kLutBytes);  // [4 warps x 64 cols][MP]
    const int rpad = (p.r + 15) & ~15;
    float *upart = part + 256 * MP;    // [rpad][MP] partial B^T grad_h over this n-slice
    float *ufull = upart + rpad * MP;  // [rpad][MP] s * B^T grad_h, rounded to bf16

    cg::cluster_group cluster = cg::this_cluster();
    const int C = static_cast<int>(cluster.num_blocks());
    const int crank = static_cast<int>(cluster.block_rank());
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int gq = lane >> 2, t = lane & 3;

    build_pair_lut(lut);
    for (int i = threadIdx.x; i < rpad * MP; i += blockDim.x) upart[i] = 0.0f;
    __syncthreads();
    grid_dependency_wait();

    const int64_t N = p.n, K = p.k, nbr = K / kBlock;
    const int64_t n16 = (N + 15) / 16;
    const int64_t s_lo = n16 * crank / C, s_hi = n16 * (crank + 1) / C;  // 16-row steps of this slice
    const float mu = __ldg(p.mu);
    const int M = p.M;

    // ---- base: output block column kb (64 features), reduction over this slice's rows.
    {
        const int64_t kb = static_cast<int64_t>(blockIdx.y) * kDecWarps + warp;
        const bool vk = kb < nbr;
        const int64_t kbc = vk ? kb : 0;
        float acc[4][NG][4];
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int tg = 0; tg < NG; ++tg) acc[i][tg][0] = acc[i][tg][1] = acc[i][tg][2] = acc[i][tg][3] = 0.0f;

        if (vk) {
            // Batches of kStepBatch 16-row steps, all loads issued before use.
            for (int64_t sb = s_lo; sb < s_hi; sb += kStepBatch) {
                const int nst = static_cast<int>(s_hi - sb < kStepBatch ? s_hi - sb : kStepBatch);
                uint32_t w[kStepBatch][4], qv[kStepBatch][4];
                float sg[kStepBatch][4];
#pragma unroll
                for (int j = 0; j < kStepBatch; ++j)
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const int64_t n = (sb + j) * 16 + 4 * t + i;
                        w[j][i] = 0x77777777u;  // value 0
                        qv[j][i] = 0u;
                        sg[j][i] = 0.0f;
                        if (j < nst && n < N) {
                            const int64_t bi = n * nbr + kbc;
                            w[j][i] = ld_nc_u32(p.codes + n * (K / 2) + kbc * 32 + 4 * gq);
                            qv[j][i] = __ldg(p.q + bi);
                            sg[j][i] = __ldg(p.sigma + bi / kGroup);
                        }
                    }
#pragma unroll
                for (int j = 0; j < kStepBatch; ++j) {
                    if (j >= nst) break;
                    const int64_t n0 = (sb + j) * 16 + 4 * t;  // this lane's 4 reduction rows
                    float cp[4];
#pragma unroll
                    for (int i = 0; i < 4; ++i) cp[i] = block_constant(static_cast<uint8_t>(qv[j][i]), sg[j][i], mu);
                    uint32_t e01, o01, e23, o23;
                    interleave_rows(w[j][0], w[j][1], e01, o01);
                    interleave_rows(w[j][2], w[j][3], e23, o23);
                    uint32_t af[4][4];
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        af[i][0] = lut_get(lut, byte_of(e01, i), lane);
                        af[i][1] = lut_get(lut, byte_of(o01, i), lane);
                        af[i][2] = lut_get(lut, byte_of(e23, i), lane);
                        af[i][3] = lut_get(lut, byte_of(o23, i), lane);
                    }
#pragma unroll
                    for (int tg = 0; tg < NG; ++tg) {
                        const int tok = tg * 8 + gq;
                        float gv[4] = {0.0f, 0.0f, 0.0f, 0.0f};
                        if (tok < M) load_g4(p.act, N, tok, n0, gv);
                        const uint32_t b0 = pack_bf16x2(cp[0] * gv[0], cp[1] * gv[1]);
                        const uint32_t b1 = pack_bf16x2(cp[2] * gv[2], cp[3] * gv[3]);
#pragma unroll
                        for (int i = 0; i < 4; ++i)
                            mma_16816(acc[i][tg], af[i][0], af[i][1], af[i][2], af[i][3], b0, b1);
                    }
                }
            }
        }
        // D row gq of tile i is feature 8*gq + 2i, row gq+8 is feature 8*gq + 2i + 1.
        float *wp = part + warp * 64 * MP;
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int tg = 0; tg < NG; ++tg) {
                const int f = 8 * gq + 2 * i, tok = tg * 8 + 2 * t;
                wp[f * MP + tok] = acc[i][tg][0];
                wp[f * MP + tok + 1] = acc[i][tg][1];
                wp[(f + 1) * MP + tok] = acc[i][tg][2];
                wp[(f + 1) * MP + tok + 1] = acc[i][tg][3];
            }
    }

    // ---- LoRA: partial u[j][tok] = sum_n B[n][j] grad_h[tok][n] over this slice.
    if (p.r > 0) {
        const int rt = rpad / 16;
        const int64_t ns = s_hi - s_lo;
        const int64_t q_lo = s_lo + ns * warp / kDecWarps, q_hi = s_lo + ns * (warp + 1) / kDecWarps;
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
#pragma unroll
            for (int tg = 0; tg < NG; ++tg) {
                const int jl = jt * 16 + gq;
                atomicAdd(&upart[jl * MP + tg * 8 + 2 * t], d[tg][0]);
                atomicAdd(&upart[jl * MP + tg * 8 + 2 * t + 1], d[tg][1]);
                atomicAdd(&upart[(jl + 8) * MP + tg * 8 + 2 * t], d[tg][2]);
                atomicAdd(&upart[(jl + 8) * MP + tg * 8 + 2 * t + 1], d[tg][3]);
            }
        }
    }

    __syncthreads();
    cluster.sync();
    grid_dependents_launch();

    if (p.r > 0) {
        for (int i = threadIdx.x; i < rpad * MP; i += blockDim.x) {
            float sum = 0.0f;
            for (int cc = 0; cc < C; ++cc) sum += cluster.map_shared_rank(upart, cc)[i];
            ufull[i] = round_bf16(sum * p.s);
        }
    }
    __syncthreads();

    // ---- this CTA finalises features [256*crank/C, 256*(crank+1)/C) of the 256-feature group
    const int f_lo = 256 * crank / C, f_hi = 256 * (crank + 1) / C, nf = f_hi - f_lo;
    for (int i = threadIdx.x; i < nf * M; i += blockDim.x) {
        const int fl = f_lo + i % nf, tok = i / nf;
        const int64_t k = static_cast<int64_t>(blockIdx.y) * 256 + fl;
        if (k >= K) continue;
        float sum = 0.0f;
        for (int cc = 0; cc < C; ++cc) sum += cluster.map_shared_rank(part, cc)[fl * MP + tok];
        if (p.r > 0) {
            float lora = 0.0f;
            for (int j = 0; j < p.r; ++j)
                lora = __fmaf_rn(__uint_as_float(static_cast<uint32_t>(ld_ro_u16(p.A + static_cast<int64_t>(j) * K + k)) << 16),
                                 ufull[j * MP + tok], lora);
            sum += lora;
        }
        p.out[static_cast<int64_t>(tok) * K + k] = __bfloat16_as_ushort(__float2bfloat16_rn(sum));
    }
    cluster.sync();
}

template <typename Kern>
cudaError_t launch_cluster(Kern kern, dim3 grid, int cluster_x, size_t smem, cudaStream_t st, const DecodeParams &p) {
    // Raise the kernel's dynamic shared-memory limit only when a launch needs more than
    // any earlier one (the attribute call is skipped on the steady-state path).
    static thread_local const void *kerns[16];
    static thread_local size_t limits[16];
    static thread_local int nk = 0;
    int slot = -1;
    for (int i = 0; i < nk; ++i)
        if (kerns[i] == reinterpret_cast<const void *>(kern)) slot = i;
    if (slot < 0 || limits[slot] < smem) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
        if (e != cudaSuccess) return e;
        if (slot < 0 && nk < 16) {
            slot = nk++;
            kerns[slot] = reinterpret_cast<const void *>(kern);
        }
        if (slot >= 0) limits[slot] = smem;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = dim3(kDecThreads, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = cluster_x;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    // Programmatic dependent launch: the grid may start while the preceding kernel
    // finishes; the kernel reads no global memory before griddepcontrol.wait.
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    cudaError_t e;
    e = cudaLaunchKernelEx(&cfg, kern, p);
    count_launch();
    return e;
}

int pick_groups(int M) { return M <= 8 ? 1 : M <= 16 ? 2 : M <= 32 ? 4 : 8; }

// Cluster size: enough CTAs to fill the GPU, at most 8, at least 16 blocks of work per CTA.
int pick_cluster(int64_t tiles, int64_t red_units, int sms) {
    int C = 1;
    while (C < kMaxCluster && tiles * C < 2 * sms && red_units / (2 * C) >= 8) C *= 2;
    return C;
}

int num_sms() {
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    return sms;
}

}  // namespace

cudaError_t launch_decode_fwd(const WeightView &w, const uint16_t *x, int M, const uint16_t *A, const uint16_t *B,
                              int r, float s, uint16_t *h, cudaStream_t st) {
    if (M <= 0 || w.n == 0) return cudaSuccess;
    DecodeParams p{w.codes, w.q, w.sigma, w.mu, w.n, w.k, x, M, A, B, r, s, h};
    const int NG = pick_groups(M);
    const int rpad = (r + 15) & ~15;
    const size_t smem = kLutBytes + sizeof(float) * (64 * 8 * NG + 2 * rpad * 8 * NG);
    const int64_t tiles = (w.n + 63) / 64;
    const int C = pick_cluster(tiles, w.k / kBlock, num_sms());
    const dim3 grid(C, static_cast<unsigned>(tiles), 1);
    switch (NG) {
        case 1: return launch_cluster(k_decode_fwd<1>, grid, C, smem, st, p);
        case 2: return launch_cluster(k_decode_fwd<2>, grid, C, smem, st, p);
        case 4: return launch_cluster(k_decode_fwd<4>, grid, C, smem, st, p);
        default: return launch_cluster(k_decode_fwd<8>, grid, C, smem, st, p);
    }
}

cudaError_t launch_decode_bwd(const WeightView &w, const uint16_t *gh, int M, const uint16_t *A, const uint16_t *B,
                              int r, float s, uint16_t *gx, cudaStream_t st) {
    if (M <= 0 || w.k == 0) return cudaSuccess;
    DecodeParams p{w.codes, w.q, w.sigma, w.mu, w.n, w.k, gh, M, A, B, r, s, gx};
    const int NG = pick_groups(M);
    const int rpad = (r + 15) & ~15;
    const size_t smem = kLutBytes + sizeof(float) * (256 * 8 * NG + 2 * rpad * 8 * NG);
    const int64_t tiles = (w.k / kBlock + kDecWarps - 1) / kDecWarps;
    const int C = pick_cluster(tiles, (w.n + 15) / 16 / 4, num_sms());
    const dim3 grid(C, static_cast<unsigned>(tiles), 1);
    switch (NG) {
        case 1: return launch_cluster(k_decode_bwd<1>, grid, C, smem, st, p);
        case 2: return launch_cluster(k_decode_bwd<2>, grid, C, smem, st, p);
        case 4: return launch_cluster(k_decode_bwd<4>, grid, C, smem, st, p);
        default: return cudaErrorInvalidValue;  // callers split tokens into chunks of 32
    }
}

}  // namespace qn
