// lora_grads.cu -- gradients of the adapter weights, the only trained parameters of the layer:
//
//   grad_B[n, j] = s * sum_m grad_h[m, n] t[m, j],   t = x A^T       (M x r)
//   grad_A[j, k] = s * sum_m u[m, j] x[m, k],        u = grad_h B    (M x r)
//
// ("How does QLoRA work for training?", aivaro.ru, sections 2 and 7: W is frozen, only B and A
// are updated; these are the derivatives of h = W'x + s B (A x).)
//
// Both are token reductions of the form C[p, q] = sum_m L[m, p] R[m, q] with L token-major
// (grad_h or x) and R = t or u (M x r, bf16, from the down-projection kernel). One CTA owns 64
// columns p of L and every q: its four warps take 16 p each. Chunks of 64 tokens of L and R are
// copied into shared memory (cp.async, double-buffered, padded rows) and read with
// ldmatrix.trans, which delivers the token-pair fragments mma.sync needs for both operands.
// fp32 accumulation over all M tokens in a fixed order (bit-reproducible); results are fp32,
// grad_A written transposed from its C = grad_A^T.
#include "common.cuh"
#include "dropout.cuh"
#include "host_cache.h"
#include "kernels.h"

namespace qn {

namespace {

constexpr int kGThreads = 128;  // 4 warps x 16 columns p
constexpr int kGP = 64;         // columns p per CTA
constexpr int kGM = 64;         // tokens per chunk
constexpr int kLRow = kGP + 8;  // bf16 per padded L row (144 B: conflict-free ldmatrix rows)

struct TnArgs {
    const uint16_t *L;  // M x P, row stride ldL
    int64_t ldL;
    const uint16_t *R;  // M x RT, row stride RT (columns >= r are zero)
    int RT;
    int64_t M, P;
    int r;
    float s;
    float *C;        // output
    int64_t ldC;     // C[p * ldC + q] (transpose = false) or C[q * ldC + p] (transpose = true)
    bool transpose;
    DropoutArgs drop;  // mask of L's elements (m, p) at index offset + m P + p (thr == 0: none)
};

__device__ __forceinline__ uint32_t saddr32(const void *p) { return static_cast<uint32_t>(__cvta_generic_to_shared(p)); }

__device__ __forceinline__ void cp16(uint32_t dst, const void *src, uint32_t bytes) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(bytes) : "memory");
}

__device__ __forceinline__ void ldm_x4_trans(uint32_t a, uint32_t &r0, uint32_t &r1, uint32_t &r2, uint32_t &r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(a));
}

template <int QT, bool kAligned>  // q tiles of 8 (r <= 8 QT); kAligned: L rows are 16-byte aligned
__global__ void __launch_bounds__(kGThreads) k_tn(const TnArgs p) {
    __shared__ __align__(16) uint16_t Ls[2][kGM][kLRow];
    __shared__ __align__(16) uint16_t Rs[2][kGM][8 * QT + 8];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
    const int64_t p0 = static_cast<int64_t>(blockIdx.x) * kGP;

    // chunk c of L (kGM tokens x kGP columns) and of R (kGM tokens x 8 QT columns)
    auto issue = [&](int64_t c, int buf) {
        const int64_t m0 = c * kGM;
        for (int i = threadIdx.x; i < kGM * (kGP / 8); i += kGThreads) {
            const int row = i / (kGP / 8), seg = i % (kGP / 8);
            const int64_t m = m0 + row, col = p0 + 8 * seg;
            if (kAligned) {
                uint32_t bytes = 0;
                const uint16_t *src = p.L;
                if (m < p.M && col < p.P) {
                    const int64_t left = p.P - col;
                    bytes = left >= 8 ? 16u : static_cast<uint32_t>(2 * left);
                    src = p.L + m * p.ldL + col;
                }
                cp16(saddr32(&Ls[buf][row][8 * seg]), src, bytes);
            } else {
                // rows not 16-byte aligned: element copies (synchronous; used for odd widths only)
#pragma unroll
                for (int e = 0; e < 8; ++e)
                    Ls[buf][row][8 * seg + e] =
                        (m < p.M && col + e < p.P) ? ld_ro_u16(p.L + m * p.ldL + col + e) : static_cast<uint16_t>(0);
            }
        }
        for (int i = threadIdx.x; i < kGM * QT; i += kGThreads) {
            const int row = i / QT, seg = i % QT;
            const int64_t m = m0 + row;
            const bool ok = m < p.M && 8 * seg < p.RT;
            cp16(saddr32(&Rs[buf][row][8 * seg]), ok ? p.R + m * p.RT + 8 * seg : p.R, ok ? 16u : 0u);
        }
        asm volatile("cp.async.commit_group;" ::: "memory");
    };

    float acc[QT][4];
#pragma unroll
    for (int q = 0; q < QT; ++q) acc[q][0] = acc[q][1] = acc[q][2] = acc[q][3] = 0.0f;
    const int64_t nchunks = (p.M + kGM - 1) / kGM;
    if (nchunks > 0) issue(0, 0);
    for (int64_t c = 0; c < nchunks; ++c) {
        const int buf = static_cast<int>(c & 1);
        if (c + 1 < nchunks) {
            issue(c + 1, buf ^ 1);
            asm volatile("cp.async.wait_group 1;" ::: "memory");
        } else {
            asm volatile("cp.async.wait_group 0;" ::: "memory");
        }
        __syncthreads();
        if (p.drop.thr != 0u) {
            // LoRA dropout: L is the forward's adapter input; zero its dropped elements in place
            for (int i = threadIdx.x; i < kGM * (kGP / 8); i += kGThreads) {
                const int row = i / (kGP / 8), seg = i % (kGP / 8);
                const int64_t m = c * kGM + row, col = p0 + 8 * seg;
                if (m >= p.M || col >= p.P) continue;
                const uint32_t keep = dropout_keep_bits(p.drop, p.drop.offset + static_cast<uint64_t>(m * p.P + col), 8);
                uint4 *v = reinterpret_cast<uint4 *>(&Ls[buf][row][8 * seg]);
                uint4 w = *v;
                w.x = mask_pair(w.x, keep);
                w.y = mask_pair(w.y, keep >> 2);
                w.z = mask_pair(w.z, keep >> 4);
                w.w = mask_pair(w.w, keep >> 6);
                *v = w;
            }
            __syncthreads();
        }
#pragma unroll
        for (int ks = 0; ks < kGM / 16; ++ks) {
            // A operand: L^T[p][m] for p = 16 warp .. + 16, m = 16 ks .. + 16 (matrix i: p half i & 1,
            // m half i >> 1; lanes 8 i .. 8 i + 7 give the rows m of matrix i)
            const int mi = lane >> 3, rr = lane & 7;
            const uint32_t aaddr =
                saddr32(&Ls[buf][16 * ks + 8 * (mi >> 1) + rr][16 * warp + 8 * (mi & 1)]);
            uint32_t a0, a1, a2, a3;
            ldm_x4_trans(aaddr, a0, a1, a2, a3);
#pragma unroll
            for (int q2 = 0; q2 < (QT + 1) / 2; ++q2) {
                // B operand: R[m][q] for two q tiles (matrices: (q tile 2 q2, m lo), (2 q2, m hi),
                // (2 q2 + 1, m lo), (2 q2 + 1, m hi))
                const uint32_t baddr =
                    saddr32(&Rs[buf][16 * ks + 8 * (mi & 1) + rr][8 * (2 * q2 + (mi >> 1))]);
                uint32_t b0, b1, b2, b3;
                ldm_x4_trans(baddr, b0, b1, b2, b3);
                mma_16816(acc[2 * q2], a0, a1, a2, a3, b0, b1);
                if (2 * q2 + 1 < QT) mma_16816(acc[2 * q2 + 1], a0, a1, a2, a3, b2, b3);
            }
        }
        __syncthreads();  // the buffer is refilled by the next issue
    }
    // acc[q]: rows p = 16 warp + g (+8), columns q = 8 q + 2 t (+1)
#pragma unroll
    for (int q = 0; q < QT; ++q)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const int64_t pp = p0 + 16 * warp + g + 8 * (e >> 1);
            const int qq = 8 * q + 2 * t + (e & 1);
            if (pp < p.P && qq < p.r) {
                const float v = p.s * acc[q][e];
                if (p.transpose)
                    p.C[static_cast<int64_t>(qq) * p.ldC + pp] = v;
                else
                    p.C[pp * p.ldC + qq] = v;
            }
        }
}

template <int QT>
cudaError_t launch_tn_q(const TnArgs &a, cudaStream_t st) {
    const unsigned grid = static_cast<unsigned>((a.P + kGP - 1) / kGP);
    if (a.ldL % 8 == 0)
        k_tn<QT, true><<<grid, kGThreads, 0, st>>>(a);
    else
        k_tn<QT, false><<<grid, kGThreads, 0, st>>>(a);
    count_launch();
    return cudaGetLastError();
}

// C = s L^T R for r columns of R, in chunks of at most 64 adapter columns per launch.
cudaError_t launch_tn(const TnArgs &a, cudaStream_t st) {
    if (a.P == 0 || a.r == 0) return cudaSuccess;
    for (int q0 = 0; q0 < a.r; q0 += 64) {
        TnArgs c = a;
        c.r = a.r - q0 < 64 ? a.r - q0 : 64;
        c.R = a.R + q0;
        c.C = a.transpose ? a.C + static_cast<int64_t>(q0) * a.ldC : a.C + q0;
        const int qt = (c.r + 7) / 8;
        cudaError_t e;
        if (qt <= 1)
            e = launch_tn_q<1>(c, st);
        else if (qt <= 2)
            e = launch_tn_q<2>(c, st);
        else if (qt <= 4)
            e = launch_tn_q<4>(c, st);
        else
            e = launch_tn_q<8>(c, st);
        if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
}

}  // namespace

size_t lora_grads_workspace_bytes(int64_t M, int r) {
    const int64_t RT = (r + 63) / 64 * 64;
    return 2 * ((static_cast<size_t>(M * RT) * 2 + 255) & ~size_t(255));
}

cudaError_t launch_lora_grads(const uint16_t *x, const uint16_t *gh, int64_t M, int64_t n, int64_t k,
                              const uint16_t *A, const uint16_t *B, int r, float s, const DropoutArgs &drop,
                              float *grad_A, float *grad_B, void *ws, cudaStream_t st) {
    if (r <= 0) return cudaSuccess;
    const int RT = (r + 63) / 64 * 64;
    const size_t half = (static_cast<size_t>(M * RT) * 2 + 255) & ~size_t(255);
    uint16_t *t = static_cast<uint16_t *>(ws);
    uint16_t *u = reinterpret_cast<uint16_t *>(static_cast<char *>(ws) + half);
    if (M > 0) {
        // t = (mask x) A^T and u = grad_h B (unscaled), bf16, M x RT
        cudaError_t e = launch_lora_down(x, M, k, A, k, 1, r, 1.0f, t, RT, st, &drop);
        if (e != cudaSuccess) return e;
        e = launch_lora_down(gh, M, n, B, 1, r, r, 1.0f, u, RT, st);
        if (e != cudaSuccess) return e;
    }
    // grad_B = s grad_h^T t   (n x r)
    TnArgs gb{gh, n, t, RT, M, n, r, s, grad_B, r, false, DropoutArgs{0, 0, 0}};
    cudaError_t e = launch_tn(gb, st);
    if (e != cudaSuccess) return e;
    // grad_A^T = s (mask x)^T u     (k x r), stored as grad_A (r x k)
    TnArgs ga{x, k, u, RT, M, k, r, s, grad_A, k, true, drop};
    return launch_tn(ga, st);
}

}  // namespace qn
