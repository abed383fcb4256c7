// quantize.cu -- nf4_quantize on sm_100a: 4-bit codes (NF4, or the 4-bit float E2M1) with
// blockwise absmax (64 weights) and double quantisation of the block absmaxes (tensor mean,
// FP8 E4M3 in groups of 256), or the absmaxes kept as fp32.
//
// "QLoRA paper notes" (tqpw.cn), sections "NormalFloat Quantization (NF4)" and
// "Double Quantization"; "How does QLoRA work for training?" (aivaro.ru), section 5.
//
// Kernel 1 (HBM-bound, one pass over W): each 4-lane group owns one 64-weight block (two 16-byte
// loads a lane, the warp's loads contiguous), takes the absmax with two shuffles, forms x = w / absmax,
// picks the code through a 65-cell lookup of the decision thresholds (the cell index
// floor(32 x + 32) is the low bits of one fma rounded toward -inf against 2^23 + 32, and the
// cell's threshold and its two codes are one 8-byte shared load), packs 8 codes per
// 32-bit word, writes the fp32 absmax to the workspace and adds it to 256 exponent bins
// (integer sums, so the tensor sum is exact and independent of scheduling).
// The codes are defined by the IEEE quotient fl32(w / c). The kernel multiplies by the
// correctly rounded reciprocal instead (|w*r - w/c| < 2^-22 for |w| <= c, c normal) and
// redoes the IEEE division, for the lane's sixteen weights, only when a product lies within
// 2^-21 of its cell's threshold -- the only case where the two can fall on different sides
// of it. Near a cell edge the two may pick neighbouring cells; both give the same code there
// because no threshold lies within 2^-19 of a cell edge (checked on the host; the 4-bit float
// has a threshold on a cell edge, 1/8, so it always takes the IEEE quotient).
// The last CTA of kernel 1 rebuilds the exact mean from the bins (once): one warp forms the exact
// 384-bit sum, one thread rounds the quotient.
// Kernel 2 (1/64 of the data): each warp double-quantises one group of 256 block absmaxes.
#include <mutex>
#include <vector>

#include "common.cuh"
#include "host_cache.h"
#include "kernels.h"

namespace qn {

namespace {

constexpr int kQuantThreads = 256;
constexpr int kDqThreads = 256;
constexpr size_t kBinsBytes = 256 * sizeof(unsigned long long);
constexpr size_t kHeaderBytes = kBinsBytes + 256;  // bins, then the finished-CTA counter

__device__ __forceinline__ uint32_t mag_max2(uint32_t u) {
    return max(u & 0x7fffu, (u >> 16) & 0x7fffu);
}

__device__ float mean_from_sum(const uint64_t (&S)[6], int64_t nb);
__device__ void bins_sum_warp(const unsigned long long *bins, int lane, uint64_t (&S)[6]);

// The last CTA to finish (counted with an atomic, no waiting) rebuilds the exact mean from
// the completed bins and stores it.
__global__ void __launch_bounds__(kQuantThreads)
k_quant_blocks(const uint4 *__restrict__ W, int64_t nb, uint32_t *__restrict__ codes, float *__restrict__ cblk,
               unsigned long long *__restrict__ bins, unsigned *__restrict__ done, float *__restrict__ mu_out,
               QuantCells cells, int fast_ok_flag) {
    __shared__ int2 s_cell[65];  // {threshold bits, code below | code above << 8} of each cell
    const bool fast_ok = fast_ok_flag != 0;  // reciprocal path allowed (checked on the host)
    __shared__ unsigned s_bins[256];
    for (int i = threadIdx.x; i < 65; i += blockDim.x) s_cell[i] = make_int2(__float_as_int(cells.thr[i]), cells.codes[i]);
    for (int i = threadIdx.x; i < 256; i += blockDim.x) s_bins[i] = 0u;
    __syncthreads();

    const int lane = threadIdx.x & 31;
    const int sub = lane >> 2;  // which of the warp's 8 blocks
    const int l4 = lane & 3;    // 16-byte chunks l4 and l4 + 4 of that block (8 weights each)
    const int64_t warp_global = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
    const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
    uint32_t cached_e = 0u, cached_sum = 0u;

    // software-pipelined: the next pass's 32 bytes are requested before this pass is processed
    auto load = [&](int64_t bb, uint4 &a, uint4 &bv) {
        if (bb < nb) {
            a = ld_nc_v4(W + bb * 8 + l4);
            bv = ld_nc_v4(W + bb * 8 + 4 + l4);
        } else {
            a = bv = make_uint4(0u, 0u, 0u, 0u);
        }
    };
    uint4 na, nbv;
    load(warp_global * 8 + sub, na, nbv);
    for (int64_t b0 = warp_global * 8; b0 < nb; b0 += nwarps * 8) {
        const int64_t b = b0 + sub;
        const bool valid = b < nb;
        const uint4 va = na, vb = nbv;
        load(b + nwarps * 8, na, nbv);
        uint32_t m = max(max(max(mag_max2(va.x), mag_max2(va.y)), max(mag_max2(va.z), mag_max2(va.w))),
                         max(max(mag_max2(vb.x), mag_max2(vb.y)), max(mag_max2(vb.z), mag_max2(vb.w))));
        m = max(m, __shfl_xor_sync(0xffffffffu, m, 1));
        m = max(m, __shfl_xor_sync(0xffffffffu, m, 2));
        const float c = __uint_as_float(m << 16);  // block absmax, exact (a bf16 value)
        uint32_t word_a = cells.zero_word, word_b = cells.zero_word;  // all-zero block: the code of 0
        if (c != 0.0f) {
            const uint32_t w[8] = {va.x, va.y, va.z, va.w, vb.x, vb.y, vb.z, vb.w};
            auto weight = [&](int i) {
                return __uint_as_float((i & 1) ? (w[i >> 1] & 0xffff0000u) : (w[i >> 1] << 16));
            };
            // For x in [-1, 1], 32 x + 32 + 2^23 rounded toward -inf is 2^23 + floor(32 x + 32): the
            // cell index in the mantissa, exactly. x leaves [-1, 1] only by a hair, when c > 2^126
            // makes fl(1/c) subnormal (the sum then drops below 2^23 and its bits below 2^23's), so
            // the index is clamped to [0, 64] as a signed integer; non-finite input lands in range too.
            auto code_of = [&](float x, float &dist) {
                const int j =
                    min(max(static_cast<int>(__float_as_uint(__fmaf_rd(x, 32.0f, 8388640.0f)) - 0x4B000000u), 0), 64);
                const int2 cell = s_cell[j];
                dist = x - __int_as_float(cell.x);
                return dist > 0.0f ? (cell.y >> 8) : (cell.y & 0xff);
            };
            // c is a bf16 value, so c >= 2^-126 exactly when its exponent field is non-zero
            const bool fast = fast_ok && (m >> 7) != 0u;
            const float r = __frcp_rn(c);
            word_a = word_b = 0u;
            bool redo = !fast;
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                float dist;
                const int code = code_of(__fmul_rn(weight(i), r), dist);
                if (i < 8)
                    word_a |= static_cast<uint32_t>(code) << (4 * i);
                else
                    word_b |= static_cast<uint32_t>(code) << (4 * (i - 8));
                redo |= fabsf(dist) <= 0x1p-21f;
            }
            if (redo) {  // rare: all sixteen weights of this lane again, by the IEEE quotient
                word_a = word_b = 0u;
                for (int i = 0; i < 16; ++i) {
                    float dist;
                    const int code = code_of(__fdiv_rn(weight(i), c), dist);
                    if (i < 8)
                        word_a |= static_cast<uint32_t>(code) << (4 * i);
                    else
                        word_b |= static_cast<uint32_t>(code) << (4 * (i - 8));
                }
            }
        }
        if (valid) {
            codes[b * 8 + l4] = word_a;
            codes[b * 8 + 4 + l4] = word_b;
            if (l4 == 0) {
                cblk[b] = c;
                const uint32_t e = m >> 7;
                const uint32_t sig = (e == 0u) ? (m & 0x7fu) : (0x80u | (m & 0x7fu));
                if (e == cached_e) {
                    cached_sum += sig;
                } else {
                    if (cached_sum) atomicAdd(&s_bins[cached_e], cached_sum);
                    cached_e = e;
                    cached_sum = sig;
                }
            }
        }
    }
    if (cached_sum) atomicAdd(&s_bins[cached_e], cached_sum);
    __syncthreads();
    for (int i = threadIdx.x; i < 256; i += blockDim.x)
        if (s_bins[i]) atomicAdd(&bins[i], static_cast<unsigned long long>(s_bins[i]));
    __threadfence();
    __syncthreads();
    __shared__ bool s_last;
    if (threadIdx.x == 0) s_last = atomicAdd(done, 1u) == gridDim.x - 1;
    __syncthreads();
    if (s_last && mu_out) {
        __threadfence();
        __shared__ unsigned long long s_all[256];
        for (int i = threadIdx.x; i < 256; i += blockDim.x) s_all[i] = __ldcg(bins + i);
        __syncthreads();
        if (threadIdx.x < 32) {
            uint64_t S[6];
            bins_sum_warp(s_all, threadIdx.x, S);
            if (threadIdx.x == 0) *mu_out = mean_from_sum(S, nb);
        }
    }
}

// a += b on 384-bit integers (six 64-bit limbs, least significant first).
__device__ __forceinline__ void add384(uint64_t (&a)[6], const uint64_t (&b)[6]) {
    uint64_t carry = 0;
#pragma unroll
    for (int i = 0; i < 6; ++i) {
        const uint64_t t = a[i] + b[i];
        const uint64_t c1 = t < b[i];
        const uint64_t t2 = t + carry;
        const uint64_t c2 = t2 < carry;
        a[i] = t2;
        carry = c1 + c2;
    }
}

// S (every lane of a warp) = sum over e of bins[e] * 2^p(e), p(e) = max(e - 1, 0): lane l adds the
// bins l, l + 32, ... into its own 384-bit sum (limb positions chosen by selects, so the limbs
// stay in registers), then five butterfly steps add the lanes' sums. The exact sum times 2^-133
// is the sum of the absmaxes.
__device__ void bins_sum_warp(const unsigned long long *bins, int lane, uint64_t (&S)[6]) {
#pragma unroll
    for (int i = 0; i < 6; ++i) S[i] = 0;
    for (int e = lane; e < 256; e += 32) {
        const uint64_t v = bins[e];
        if (v == 0) continue;
        const int p = e ? e - 1 : 0;
        const int li = p >> 6, sh = p & 63;
        const uint64_t lo = v << sh, hi = sh ? (v >> (64 - sh)) : 0ull;
        uint64_t add[6];
#pragma unroll
        for (int i = 0; i < 6; ++i) add[i] = (i == li) ? lo : ((i == li + 1) ? hi : 0ull);
        add384(S, add);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        uint64_t other[6];
#pragma unroll
        for (int i = 0; i < 6; ++i) other[i] = __shfl_xor_sync(0xffffffffu, S[i], o);
        add384(S, other);
    }
}

// Exact mean of the block absmaxes, rounded once to fp32, from their exact sum S * 2^-133
// (bins_sum_warp). Run by one thread.
__device__ float mean_from_sum(const uint64_t (&S)[6], int64_t nb) {
    int top = 5;
    while (top >= 0 && S[top] == 0) --top;
    if (top < 0 || nb <= 0) return 0.0f;
    const int L = top * 64 + (64 - __clzll(static_cast<long long>(S[top])));  // bit length
    // S64 = the top 64 bits of S (left-aligned), e2 = L - 64: S = S64 * 2^e2 + rest.
    uint64_t S64;
    bool sticky = false;
    const int e2 = L - 64;
    if (e2 <= 0) {
        S64 = S[0] << (-e2);  // L <= 64: S is limb 0
    } else {
        const int li = e2 >> 6, sh = e2 & 63;
        S64 = (sh == 0) ? S[li] : ((S[li] >> sh) | (S[li + 1] << (64 - sh)));
        for (int i = 0; i < li && !sticky; ++i) sticky = S[i] != 0;
        if (sh) sticky = sticky || (S[li] & ((1ull << sh) - 1)) != 0;
    }
    // Quotient with >= 40 significant bits: S64 / nb alone when that is wide enough,
    // else one more 64-bit division step on the remainder (nb < 2^40 keeps r1 << 24
    // and Q below 2^64). value = (Q + frac) * 2^eb.
    const uint64_t n = static_cast<uint64_t>(nb);
    const uint64_t q1 = S64 / n, r1 = S64 % n;
    uint64_t Q;
    int eb;  // exponent of Q's least significant bit
    if (q1 >> 39) {
        Q = q1;
        sticky = sticky || (r1 != 0);
        eb = e2 - 133;
    } else {
        const uint64_t q2 = (r1 << 24) / n, r2 = (r1 << 24) % n;
        Q = (q1 << 24) | q2;
        sticky = sticky || (r2 != 0);
        eb = e2 - 24 - 133;
    }
    const int lead = 63 - __clzll(static_cast<long long>(Q));
    const int lsb_exp = max(lead + eb - 23, -149);
    const int drop = lsb_exp - eb;
    uint64_t mant;
    int rbit;
    if (drop > 64) {
        mant = 0;
        rbit = 0;
        sticky = true;
    } else if (drop == 64) {
        mant = 0;
        rbit = static_cast<int>(Q >> 63);
        sticky = sticky || (Q & ~(1ull << 63)) != 0;
    } else {
        mant = Q >> drop;
        rbit = static_cast<int>((Q >> (drop - 1)) & 1ull);
        if (drop > 1) sticky = sticky || (Q & ((1ull << (drop - 1)) - 1)) != 0;
    }
    if (rbit && (sticky || (mant & 1ull))) mant += 1;
    return ldexpf(static_cast<float>(mant), lsb_exp);
}

__global__ void __launch_bounds__(kDqThreads)
k_double_quant(const float *__restrict__ cblk, int64_t nb, uint8_t *__restrict__ q, float *__restrict__ sigma,
               const float *__restrict__ mu_in) {
    const float mu = __ldcg(mu_in);
    const int lane = threadIdx.x & 31;
    const int64_t ng = (nb + kGroup - 1) / kGroup;
    const int64_t warp_global = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
    const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
    for (int64_t g = warp_global; g < ng; g += nwarps) {
        const int64_t b0 = g * kGroup;
        float d[8];
        float S = 0.0f;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const int64_t b = b0 + i * 32 + lane;
            d[i] = (b < nb) ? __fsub_rn(cblk[b], mu) : 0.0f;
            S = fmaxf(S, fabsf(d[i]));
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) S = fmaxf(S, __shfl_xor_sync(0xffffffffu, S, o));
        const float sg = __fdiv_rn(S, 448.0f);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const int64_t b = b0 + i * 32 + lane;
            if (b < nb) q[b] = (sg == 0.0f) ? static_cast<uint8_t>(0) : f32_to_e4m3_satfinite(__fdiv_rn(d[i], sg));
        }
        if (lane == 0) sigma[g] = sg;
    }
}

// Decision thresholds of a quant type: its distinct values ascending, each with the lowest code
// of that value (+0 before -0), and between neighbours v_j < v_j+1 with midpoint m_j (exact in
// fp64) a threshold t_j such that, for an fp32 x, "x > t_j" picks the upper neighbour exactly
// when x is nearer to it, or at equal distance and its code is the lower one: t_j = the largest
// fp32 not above m_j, one step lower still when m_j is an fp32 value and a tie goes up.
struct Thresholds {
    int nv;          // distinct values
    int code[16];    // their codes, ascending by value
    double mid[15];  // midpoints
    float t[15];
};

Thresholds make_thresholds(int qtype) {
    Thresholds th{};
    double v[16];
    for (int c = 0; c < 16; ++c) {
        const double val = table_value(qtype, c);
        bool seen = false;
        for (int j = 0; j < th.nv; ++j) seen = seen || v[j] == val;
        if (seen) continue;
        int j = th.nv++;
        for (; j > 0 && v[j - 1] > val; --j) {
            v[j] = v[j - 1];
            th.code[j] = th.code[j - 1];
        }
        v[j] = val;
        th.code[j] = c;
    }
    for (int j = 0; j + 1 < th.nv; ++j) {
        const double m = (v[j] + v[j + 1]) * 0.5;
        float f = static_cast<float>(m);
        if (static_cast<double>(f) > m) f = nextafterf(f, -2.0f);
        if (th.code[j + 1] < th.code[j] && static_cast<double>(f) == m) f = nextafterf(f, -2.0f);
        th.mid[j] = m;
        th.t[j] = f;
    }
    return th;
}

// The reciprocal path needs every decision threshold farther than 2^-19 from every cell edge.
int reciprocal_path_ok(int qtype) {
    const Thresholds th = make_thresholds(qtype);
    for (int i = 0; i + 1 < th.nv; ++i)
        for (int j = 0; j <= 64; ++j)
            if (fabs(th.mid[i] - (-1.0 + j / 32.0)) <= 0x1p-19) return 0;
    return 1;
}

// Cells of a quant type; false if two thresholds fall into one cell.
bool make_cells(int qtype, QuantCells *out) {
    const Thresholds th = make_thresholds(qtype);
    QuantCells c{};
    for (int j = 0; j <= 64; ++j) {
        const double lo = -1.0 + j / 32.0, hi = (j == 64) ? 1.0 : -1.0 + (j + 1) / 32.0;
        int base = 0, inside = 0;
        float thr = 2.0f;
        for (int i = 0; i + 1 < th.nv; ++i) {
            if (th.t[i] < lo) {
                ++base;
            } else if (th.t[i] < hi || (j == 64 && th.t[i] <= hi)) {
                thr = th.t[i];
                ++inside;
            }
        }
        if (inside > 1) return false;
        const int below = th.code[base], above = inside ? th.code[base + 1] : below;
        c.thr[j] = thr;
        c.codes[j] = below | (above << 8);
    }
    int zero = 7;
    for (int j = 0; j < th.nv; ++j)
        if (table_value(qtype, th.code[j]) == 0.0f) zero = th.code[j];
    c.zero_word = 0x11111111u * static_cast<uint32_t>(zero);
    *out = c;
    return true;
}

// Scratch for callers that cannot allocate device memory (nf4_quantize_static_ws): a
// file-scope device array that every GPU loading this library holds until exit.
constexpr size_t kStaticScratchBytes = size_t(16) << 20;
__device__ __align__(256) unsigned char g_quant_scratch[kStaticScratchBytes];

}  // namespace

size_t static_scratch_bytes() { return kStaticScratchBytes; }

// Device address of g_quant_scratch in the current context. The symbol's host-side name is not
// a device address, so it is resolved with cudaGetSymbolAddress (with the device current) and
// cached per context: a device reset creates a new context, where the module and its array are
// loaded again, so the address is looked up again there.
cudaError_t static_scratch_address(void **out) {
    struct Entry {
        uint64_t ctx;
        int dev;
        void *addr;
    };
    static std::mutex lock;
    static std::vector<Entry> cache;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    uint64_t ctx = current_context_id();
    std::lock_guard<std::mutex> guard(lock);
    if (ctx != 0)
        for (const Entry &c : cache)
            if (c.ctx == ctx && c.dev == dev) {
                *out = c.addr;
                return cudaSuccess;
            }
    void *p = nullptr;
    e = cudaGetSymbolAddress(&p, g_quant_scratch);
    if (e != cudaSuccess) return e;
    ctx = current_context_id();  // the lookup makes the device's primary context current
    if (ctx != 0) cache.push_back(Entry{ctx, dev, p});
    *out = p;
    return cudaSuccess;
}

size_t quantize_workspace_bytes(int64_t n, int64_t k) {
    const int64_t nb = n * k / kBlock;
    return kHeaderBytes + ((static_cast<size_t>(nb) * sizeof(float) + 255) & ~size_t(255));
}

cudaError_t launch_quantize(const uint16_t *W, int64_t n, int64_t k, int qtype, uint8_t *codes, uint8_t *q,
                            float *sigma, float *mu, float *absmax, void *ws, cudaStream_t s) {
    struct Tables {
        QuantCells cells[2];
        int fast_ok[2];
        bool ok;
    };
    static const Tables tables = [] {
        Tables t{};
        t.ok = make_cells(kQuantNF4, &t.cells[0]) && make_cells(kQuantFP4, &t.cells[1]);
        t.fast_ok[0] = reciprocal_path_ok(kQuantNF4);
        t.fast_ok[1] = reciprocal_path_ok(kQuantFP4);
        return t;
    }();
    if (!tables.ok || qtype < 0 || qtype > 1) return cudaErrorInvalidValue;
    const int64_t nb = n * k / kBlock;
    if (nb == 0) return cudaSuccess;
    auto *bins = static_cast<unsigned long long *>(ws);
    auto *done = reinterpret_cast<unsigned *>(static_cast<char *>(ws) + kBinsBytes);
    // without double quantisation the absmaxes go straight to the output and no mean is formed
    auto *cblk = absmax ? absmax : reinterpret_cast<float *>(static_cast<char *>(ws) + kHeaderBytes);
    float *mu_out = absmax ? nullptr : mu;
    cudaError_t e = cudaMemsetAsync(bins, 0, kHeaderBytes, s);
    if (e != cudaSuccess) return e;
    int sms = 148, occ = 4;
    e = device_sm_count(&sms);
    if (e != cudaSuccess) return e;
    e = resident_ctas(reinterpret_cast<const void *>(k_quant_blocks), kQuantThreads, 0, &occ);
    if (e != cudaSuccess) return e;
    // 64 blocks per CTA per pass; exactly one wave of resident CTAs, never more than needed,
    // and few enough blocks per CTA that the 32-bit smem bins cannot overflow.
    int64_t grid = (nb + 63) / 64;
    grid = grid < static_cast<int64_t>(sms) * occ ? grid : static_cast<int64_t>(sms) * occ;
    const int64_t min_grid = (nb + (1ll << 22) - 1) >> 22;
    if (grid < min_grid) grid = min_grid;
    k_quant_blocks<<<static_cast<unsigned>(grid), kQuantThreads, 0, s>>>(
        reinterpret_cast<const uint4 *>(W), nb, reinterpret_cast<uint32_t *>(codes), cblk, bins, done, mu_out,
        tables.cells[qtype], tables.fast_ok[qtype]);
    count_launch();
    e = cudaGetLastError();
    if (e != cudaSuccess || absmax) return e;
    const int64_t ng = (nb + kGroup - 1) / kGroup;
    int64_t grid2 = (ng + (kDqThreads / 32) - 1) / (kDqThreads / 32);
    grid2 = grid2 < static_cast<int64_t>(sms) * 4 ? grid2 : static_cast<int64_t>(sms) * 4;
    k_double_quant<<<static_cast<unsigned>(grid2), kDqThreads, 0, s>>>(cblk, nb, q, sigma, mu);
    count_launch();
    return cudaGetLastError();
}

}  // namespace qn
