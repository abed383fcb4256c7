// merge.cu -- fold the adapter into a 16-bit weight on sm_100a:
//
//   W_merged[n, k] = bf16_rn( fl32(T[code] * c'_b) + s * sum_j B[n,j] A[j,k] )   (T: NF4 or the 4-bit float)
//
// ("QLoRA & PEFT family" (ai-reference-codex), 3.6 merge_and_unload; "QLoRA paper notes"
// (tqpw.cn), Introduction: the merged weight cannot stay NF4, so it is written as bf16.)
//
// HBM-bound (0.52 B read, 2 B written per weight; the adapter factors are small and stay in
// L2). A CTA takes a tile of 128 rows x 64 features (one block column): its eight warps form the
// rank-r product of 16 rows each on the tensor cores (mma.sync, fp32 accumulation; the tile's
// 64 columns of A are staged transposed in shared memory) and park it in shared memory; then
// every thread expands 8 codes of one row, adds s times the product and writes 16 bytes, so
// the code reads and the output writes are contiguous per row. Sum and rounding: the fp32
// dequantised weight plus s * (fp32 product), one fp32 rounding, then one bf16 rounding.
#include "common.cuh"
#include "host_cache.h"
#include "kernels.h"

namespace qn {

namespace {

constexpr int kMergeThreads = 256;
constexpr int kTileRows = 128;
constexpr int kTileCols = 64;
constexpr int kDPad = kTileCols + 4;  // floats per row of the parked product (bank spread)

struct MergeArgs {
    const uint32_t *codes;  // n * k / 8 words
    const uint8_t *q;
    const float *sigma;
    const float *mu;
    const float *absmax;  // fp32 block constants (no double quantisation), else nullptr
    int qtype;
    const uint16_t *A;  // r x k
    const uint16_t *B;  // n x r
    int64_t n, k;
    int r, rk;  // rk: r rounded up to 16
    float s;
    uint16_t *out;
};

// bf16 pair (M[row][j], M[row][j + 1]) of a row-major rows x r matrix, zero outside it.
__device__ __forceinline__ uint32_t pair_rowmajor(const uint16_t *M, int64_t row, bool valid, int j, int r) {
    if (!valid || j >= r) return 0u;
    const uint16_t *b = M + row * r + j;
    if ((r & 1) == 0) return ld_ro_u32(b);
    const uint32_t lo = ld_ro_u16(b);
    const uint32_t hi = j + 1 < r ? ld_ro_u16(b + 1) : 0u;
    return lo | (hi << 16);
}

__global__ void __launch_bounds__(kMergeThreads) k_merge(const MergeArgs p) {
    extern __shared__ __align__(16) uint8_t smem[];
    float *Dp = reinterpret_cast<float *>(smem);                                   // [128][kDPad]
    uint16_t *At = reinterpret_cast<uint16_t *>(smem + kTileRows * kDPad * 4);      // [64][rk] transposed A
    __shared__ float s_t[16];
    if (threadIdx.x < 16) s_t[threadIdx.x] = table_value(p.qtype, threadIdx.x);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
    const float mu = load_mu(p.mu, p.absmax);
    const int64_t nbr = p.k / kBlock;
    const int64_t row_tiles = (p.n + kTileRows - 1) / kTileRows;
    const int64_t tiles = row_tiles * nbr;
    int64_t cur_col = -1;
    for (int64_t tile = blockIdx.x; tile < tiles; tile += gridDim.x) {
        // column-major tile order: consecutive tiles of a CTA share their A columns
        const int64_t col = tile / row_tiles, rt = tile % row_tiles;
        const int64_t n0 = rt * kTileRows, k0 = col * kTileCols;
        __syncthreads();  // the previous tile's product (and A) are no longer read
        if (p.r > 0 && col != cur_col) {
            // A[:, k0 : k0 + 64] transposed into At[f][j] (ranks beyond r are zero)
            for (int i = threadIdx.x; i < kTileCols * p.rk; i += kMergeThreads) {
                const int j = i / kTileCols, f = i % kTileCols;
                At[f * p.rk + j] = j < p.r ? ld_ro_u16(p.A + static_cast<int64_t>(j) * p.k + k0 + f) : 0;
            }
            cur_col = col;
            __syncthreads();
        }
        if (p.r > 0) {
            // rows n0 + 16 warp .. + 16: D[16 x 64] = B rows x A columns
            const int64_t rA = n0 + 16 * warp + g, rB = rA + 8;
            const bool vA = rA < p.n, vB = rB < p.n;
            float d[8][4];
#pragma unroll
            for (int nt = 0; nt < 8; ++nt) d[nt][0] = d[nt][1] = d[nt][2] = d[nt][3] = 0.0f;
            for (int kc = 0; kc < p.rk / 16; ++kc) {
                const int j = 16 * kc + 2 * t;
                const uint32_t a0 = pair_rowmajor(p.B, rA, vA, j, p.r);
                const uint32_t a1 = pair_rowmajor(p.B, rB, vB, j, p.r);
                const uint32_t a2 = pair_rowmajor(p.B, rA, vA, j + 8, p.r);
                const uint32_t a3 = pair_rowmajor(p.B, rB, vB, j + 8, p.r);
#pragma unroll
                for (int nt = 0; nt < 8; ++nt) {
                    const uint32_t *col_f = reinterpret_cast<const uint32_t *>(At + (8 * nt + g) * p.rk + j);
                    mma_16816(d[nt], a0, a1, a2, a3, col_f[0], col_f[4]);
                }
            }
            float *drow = Dp + (16 * warp + g) * kDPad;
#pragma unroll
            for (int nt = 0; nt < 8; ++nt) {
                *reinterpret_cast<float2 *>(drow + 8 * nt + 2 * t) = make_float2(d[nt][0], d[nt][1]);
                *reinterpret_cast<float2 *>(drow + 8 * kDPad + 8 * nt + 2 * t) = make_float2(d[nt][2], d[nt][3]);
            }
        }
        __syncthreads();
        // expand: thread -> (row, 8-weight word) of the tile; 8 words per 64-feature row
        for (int i = threadIdx.x; i < kTileRows * 8; i += kMergeThreads) {
            const int rl = i >> 3, wd = i & 7;
            const int64_t row = n0 + rl;
            if (row >= p.n) continue;
            const int64_t blk = row * nbr + col;
            const uint32_t w = __ldcs(p.codes + blk * 8 + wd);
            const float cp = load_block_constant(p.q, p.sigma, mu, p.absmax, blk);
            const float *dv = Dp + rl * kDPad + 8 * wd;
            uint4 o;
            uint32_t *op = reinterpret_cast<uint32_t *>(&o);
#pragma unroll
            for (int pp = 0; pp < 4; ++pp) {
                const uint32_t lo = (w >> (8 * pp)) & 15u, hi = (w >> (8 * pp + 4)) & 15u;
                float v0 = __fmul_rn(s_t[lo], cp), v1 = __fmul_rn(s_t[hi], cp);
                if (p.r > 0) {
                    v0 = __fmaf_rn(p.s, dv[2 * pp], v0);
                    v1 = __fmaf_rn(p.s, dv[2 * pp + 1], v1);
                }
                op[pp] = pack_bf16x2(v0, v1);
            }
            *reinterpret_cast<uint4 *>(p.out + row * p.k + k0 + 8 * wd) = o;
        }
    }
}

}  // namespace

cudaError_t launch_merge(const WeightView &w, const uint16_t *A, const uint16_t *B, int r, float s, uint16_t *out,
                         cudaStream_t st) {
    if (w.n == 0 || w.k == 0) return cudaSuccess;
    MergeArgs p{reinterpret_cast<const uint32_t *>(w.codes), w.q, w.sigma, w.mu, w.absmax, w.qtype, A, B, w.n, w.k,
                r, (r + 15) / 16 * 16, s, out};
    const size_t smem = static_cast<size_t>(kTileRows) * kDPad * 4 + static_cast<size_t>(kTileCols) * p.rk * 2;
    const void *kern = reinterpret_cast<const void *>(k_merge);
    cudaError_t e = ensure_smem_limit(kern, smem);
    if (e != cudaSuccess) return e;
    int sms = 148, occ = 1;
    e = device_sm_count(&sms);
    if (e != cudaSuccess) return e;
    e = resident_ctas(kern, kMergeThreads, smem, &occ);
    if (e != cudaSuccess) return e;
    const int64_t tiles = (w.n + kTileRows - 1) / kTileRows * (w.k / kBlock);
    int64_t grid = static_cast<int64_t>(sms) * occ;
    if (grid > tiles) grid = tiles;
    k_merge<<<static_cast<unsigned>(grid), kMergeThreads, smem, st>>>(p);
    count_launch();
    return cudaGetLastError();
}

}  // namespace qn
