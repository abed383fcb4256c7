// api.cu -- the extern "C" boundary declared in include/qlora_nf4.h: argument checks,
// size queries, path selection (few-token decode kernels or the tcgen05 GEMM) and launches.
#include <math.h>
#include <stdarg.h>
#include <stdio.h>

#include <string>

#include "../../include/qlora_nf4.h"
#include "kernels.h"

namespace qn {

thread_local uint64_t g_launches = 0;
thread_local std::string g_err;

void count_launch(int n) { g_launches += static_cast<uint64_t>(n); }

namespace {

qn_status fail(qn_status s, const char *fmt, ...) {
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof buf, fmt, ap);
    va_end(ap);
    g_err = buf;
    return s;
}

qn_status cuda_status(cudaError_t e, const char *what) {
    if (e == cudaSuccess) {
        g_err.clear();
        return QN_OK;
    }
    return fail(QN_ECUDA, "%s: %s", what, cudaGetErrorString(e));
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

constexpr int64_t kMaxDim = (int64_t(1) << 31) - 1;

qn_status check_shape(int64_t n, int64_t k) {
    if (n < 0 || k < 0) return fail(QN_EINVAL, "negative size n_out=%lld k_in=%lld", (long long)n, (long long)k);
    if (k % QN_BLOCK != 0) return fail(QN_ESHAPE, "k_in=%lld is not a multiple of %d", (long long)k, QN_BLOCK);
    if (n > kMaxDim || k > kMaxDim) return fail(QN_ESHAPE, "n_out or k_in above 2^31-1");
    if (n > 0 && k > 0 && (n * k) / QN_BLOCK >= (int64_t(1) << 40))
        return fail(QN_ESHAPE, "more than 2^40 blocks");
    return QN_OK;
}

qn_status check_weight(const qn_nf4_weight *w) {
    if (!w) return fail(QN_EINVAL, "null weight struct");
    qn_status s = check_shape(w->n_out, w->k_in);
    if (s != QN_OK) return s;
    if (w->quant_type != QN_QUANT_NF4 && w->quant_type != QN_QUANT_FP4)
        return fail(QN_EINVAL, "unknown quant_type %d", w->quant_type);
    if (w->const_format != QN_CONST_DQ && w->const_format != QN_CONST_F32)
        return fail(QN_EINVAL, "unknown const_format %d", w->const_format);
    if (w->n_out == 0 || w->k_in == 0) return QN_OK;
    if (w->const_format == QN_CONST_F32) {
        if (!w->codes || !w->absmax) return fail(QN_EINVAL, "null pointer in the quantised weight");
        if (!aligned16(w->codes) || !aligned16(w->absmax)) return fail(QN_EALIGN, "codes or absmax not 16-byte aligned");
        return QN_OK;
    }
    if (!w->codes || !w->absmax_q || !w->group_scale || !w->absmax_mean)
        return fail(QN_EINVAL, "null pointer in the quantised weight");
    if (!aligned16(w->codes) || !aligned16(w->absmax_q) || !aligned16(w->group_scale))
        return fail(QN_EALIGN, "codes, absmax_q or group_scale not 16-byte aligned");
    return QN_OK;
}

WeightView view(const qn_nf4_weight *w) {
    const bool f32 = w->const_format == QN_CONST_F32;
    return WeightView{w->n_out,
                      w->k_in,
                      w->codes,
                      f32 ? nullptr : w->absmax_q,
                      f32 ? nullptr : w->group_scale,
                      f32 ? nullptr : w->absmax_mean,
                      w->quant_type == QN_QUANT_FP4 ? 1 : 0,
                      f32 ? w->absmax : nullptr};
}

qn_status launch_quantize_into(const void *W, const qn_nf4_weight *out, void *ws, cudaStream_t st) {
    const bool f32 = out->const_format == QN_CONST_F32;
    return cuda_status(launch_quantize(static_cast<const uint16_t *>(W), out->n_out, out->k_in,
                                       out->quant_type == QN_QUANT_FP4 ? 1 : 0, out->codes,
                                       f32 ? nullptr : out->absmax_q, f32 ? nullptr : out->group_scale,
                                       f32 ? nullptr : out->absmax_mean, f32 ? out->absmax : nullptr, ws, st),
                       "nf4_quantize");
}

qn_status check_lora(const void *A, const void *B, int r, float alpha) {
    if (r < 0 || r > QN_MAX_RANK) return fail(QN_EINVAL, "rank r=%d outside [0, %d]", r, QN_MAX_RANK);
    if (r == 0) {
        if (A || B) return fail(QN_EINVAL, "r == 0 requires A == B == NULL");
        return QN_OK;
    }
    if (!A || !B) return fail(QN_EINVAL, "null adapter pointer with r=%d", r);
    if (!aligned16(A) || !aligned16(B)) return fail(QN_EALIGN, "A or B not 16-byte aligned");
    if (!(alpha == alpha) || alpha - alpha != 0.0f) return fail(QN_EINVAL, "alpha is not finite");
    return QN_OK;
}

// The kernels' mask parameters and the adapter scale under dropout (s / (1 - p)); off when d is
// null, p == 0 or there is no adapter.
qn_status resolve_dropout(const qn_lora_dropout *d, int r, float sc, DropoutArgs *drop, float *sc_eff) {
    *drop = DropoutArgs{0, 0, 0};
    *sc_eff = sc;
    if (!d || d->p == 0.0f || r == 0) return QN_OK;
    if (!(d->p > 0.0f && d->p < 1.0f)) return fail(QN_EINVAL, "dropout rate p=%g outside [0, 1)", (double)d->p);
    const double thr = floor(static_cast<double>(d->p) * 4294967296.0);
    *drop = DropoutArgs{d->seed, d->offset, static_cast<uint32_t>(thr)};
    *sc_eff = static_cast<float>(static_cast<double>(sc) / (1.0 - static_cast<double>(d->p)));
    return QN_OK;
}

}  // namespace
}  // namespace qn

using namespace qn;

extern "C" {

const char *qn_status_string(qn_status s) {
    switch (s) {
        case QN_OK: return "ok";
        case QN_EINVAL: return "invalid argument";
        case QN_ESHAPE: return "unsupported shape";
        case QN_EALIGN: return "misaligned pointer";
        case QN_ECUDA: return "CUDA error";
        case QN_EWORKSPACE: return "workspace missing or too small";
        case QN_ETIMEOUT: return "a kernel gave up a bounded wait";
    }
    return "unknown status";
}

const char *qn_last_error(void) { return g_err.c_str(); }

uint64_t qn_launch_count(int reset) {
    const uint64_t v = g_launches;
    if (reset) g_launches = 0;
    return v;
}

qn_status qn_nf4_sizes(int64_t n_out, int64_t k_in, size_t *codes_bytes, size_t *absmax_bytes, size_t *scale_bytes,
                       size_t *mean_bytes) {
    if (!codes_bytes || !absmax_bytes || !scale_bytes || !mean_bytes) return fail(QN_EINVAL, "null output pointer");
    qn_status s = check_shape(n_out, k_in);
    if (s != QN_OK) return s;
    const int64_t nb = n_out * k_in / QN_BLOCK;
    *codes_bytes = static_cast<size_t>(n_out * k_in / 2);
    *absmax_bytes = static_cast<size_t>(nb);
    *scale_bytes = sizeof(float) * static_cast<size_t>((nb + QN_GROUP - 1) / QN_GROUP);
    *mean_bytes = sizeof(float);
    g_err.clear();
    return QN_OK;
}

qn_status qn_weight_sizes(int64_t n_out, int64_t k_in, int const_format, size_t *codes_bytes, size_t *absmax_bytes,
                          size_t *scale_bytes, size_t *mean_bytes, size_t *absmax_f32_bytes) {
    if (!absmax_f32_bytes) return fail(QN_EINVAL, "null output pointer");
    if (const_format != QN_CONST_DQ && const_format != QN_CONST_F32)
        return fail(QN_EINVAL, "unknown const_format %d", const_format);
    qn_status s = qn_nf4_sizes(n_out, k_in, codes_bytes, absmax_bytes, scale_bytes, mean_bytes);
    if (s != QN_OK) return s;
    *absmax_f32_bytes = 0;
    if (const_format == QN_CONST_F32) {
        *absmax_f32_bytes = sizeof(float) * *absmax_bytes;
        *absmax_bytes = *scale_bytes = *mean_bytes = 0;
    }
    return QN_OK;
}

qn_status qn_quantize_workspace_size(int64_t n_out, int64_t k_in, size_t *ws_bytes) {
    if (!ws_bytes) return fail(QN_EINVAL, "null output pointer");
    qn_status s = check_shape(n_out, k_in);
    if (s != QN_OK) return s;
    *ws_bytes = quantize_workspace_bytes(n_out, k_in);
    g_err.clear();
    return QN_OK;
}

qn_status nf4_quantize(const void *W, const qn_nf4_weight *out, void *ws, size_t ws_bytes, void *stream) {
    qn_status s = check_weight(out);
    if (s != QN_OK) return s;
    if (out->n_out == 0 || out->k_in == 0) return QN_OK;
    if (!W) return fail(QN_EINVAL, "null W");
    if (!aligned16(W)) return fail(QN_EALIGN, "W not 16-byte aligned");
    const size_t need = quantize_workspace_bytes(out->n_out, out->k_in);
    if (!ws || ws_bytes < need) return fail(QN_EWORKSPACE, "quantize workspace needs %zu bytes", need);
    if ((reinterpret_cast<uintptr_t>(ws) & 255u) != 0) return fail(QN_EALIGN, "workspace not 256-byte aligned");
    return launch_quantize_into(W, out, ws, static_cast<cudaStream_t>(stream));
}

qn_status nf4_quantize_static_ws(const void *W, const qn_nf4_weight *out, void *stream) {
    qn_status s = check_weight(out);
    if (s != QN_OK) return s;
    if (out->n_out == 0 || out->k_in == 0) return QN_OK;
    const size_t need = quantize_workspace_bytes(out->n_out, out->k_in);
    if (need > static_scratch_bytes())
        return fail(QN_EWORKSPACE,
                    "nf4_quantize_static_ws: a %lld x %lld weight needs %zu bytes of scratch, the static scratch holds "
                    "%zu (at most %lld weights); use nf4_quantize with a caller workspace",
                    (long long)out->n_out, (long long)out->k_in, need, static_scratch_bytes(),
                    (long long)((static_scratch_bytes() - 2304) / 4 * QN_BLOCK));
    if (!W) return fail(QN_EINVAL, "null W");
    if (!aligned16(W)) return fail(QN_EALIGN, "W not 16-byte aligned");
    void *ws = nullptr;
    cudaError_t e = static_scratch_address(&ws);
    if (e != cudaSuccess) return cuda_status(e, "nf4_quantize_static_ws: cudaGetSymbolAddress");
    return launch_quantize_into(W, out, ws, static_cast<cudaStream_t>(stream));
}

qn_status nf4_dequantize(const qn_nf4_weight *w, void *W_out, void *stream) {
    qn_status s = check_weight(w);
    if (s != QN_OK) return s;
    if (w->n_out == 0 || w->k_in == 0) return QN_OK;
    if (!W_out) return fail(QN_EINVAL, "null W_out");
    if (!aligned16(W_out)) return fail(QN_EALIGN, "W_out not 16-byte aligned");
    return cuda_status(launch_dequant(view(w), static_cast<uint16_t *>(W_out), static_cast<cudaStream_t>(stream)),
                       "nf4_dequantize");
}

qn_status qlora_merge_bf16(const qn_nf4_weight *w, const void *A, const void *B, int r, float alpha, void *W_out,
                           void *stream) {
    qn_status s = check_weight(w);
    if (s != QN_OK) return s;
    s = check_lora(A, B, r, alpha);
    if (s != QN_OK) return s;
    if (w->n_out == 0 || w->k_in == 0) return QN_OK;
    if (!W_out) return fail(QN_EINVAL, "null W_out");
    if (!aligned16(W_out)) return fail(QN_EALIGN, "W_out not 16-byte aligned");
    if (W_out == A || W_out == B) return fail(QN_EINVAL, "W_out aliases an adapter factor");
    const float sc = r > 0 ? alpha / static_cast<float>(r) : 0.0f;
    return cuda_status(launch_merge(view(w), static_cast<const uint16_t *>(A), static_cast<const uint16_t *>(B), r, sc,
                                    static_cast<uint16_t *>(W_out), static_cast<cudaStream_t>(stream)),
                       "qlora_merge_bf16");
}

qn_status qlora_lora_grads_workspace_size(int64_t M, int r, size_t *ws_bytes) {
    if (!ws_bytes) return fail(QN_EINVAL, "null output pointer");
    if (M < 0 || M > kMaxDim) return fail(QN_EINVAL, "M=%lld out of range", (long long)M);
    if (r < 1 || r > QN_MAX_RANK) return fail(QN_EINVAL, "rank r=%d outside [1, %d]", r, QN_MAX_RANK);
    *ws_bytes = lora_grads_workspace_bytes(M, r);
    g_err.clear();
    return QN_OK;
}

qn_status qlora_lora_grads(const void *x, const void *grad_h, int64_t M, int64_t n_out, int64_t k_in, const void *A,
                           const void *B, int r, float alpha, float *grad_A, float *grad_B, void *ws, size_t ws_bytes,
                           void *stream) {
    return qlora_lora_grads_dropout(x, grad_h, M, n_out, k_in, A, B, r, alpha, nullptr, grad_A, grad_B, ws, ws_bytes,
                                    stream);
}

qn_status qlora_lora_grads_dropout(const void *x, const void *grad_h, int64_t M, int64_t n_out, int64_t k_in,
                                   const void *A, const void *B, int r, float alpha, const qn_lora_dropout *dropout,
                                   float *grad_A, float *grad_B, void *ws, size_t ws_bytes, void *stream) {
    qn_status s = check_shape(n_out, k_in);
    if (s != QN_OK) return s;
    if (M < 0 || M > kMaxDim) return fail(QN_EINVAL, "M=%lld out of range", (long long)M);
    if (r < 1 || r > QN_MAX_RANK) return fail(QN_EINVAL, "rank r=%d outside [1, %d]", r, QN_MAX_RANK);
    s = check_lora(A, B, r, alpha);
    if (s != QN_OK) return s;
    if (!grad_A || !grad_B) return fail(QN_EINVAL, "null gradient output");
    if (n_out == 0 || k_in == 0) return QN_OK;
    if (M > 0 && (!x || !grad_h)) return fail(QN_EINVAL, "null activation pointer");
    if (M > 0 && (!aligned16(x) || !aligned16(grad_h))) return fail(QN_EALIGN, "x or grad_h not 16-byte aligned");
    const size_t need = lora_grads_workspace_bytes(M, r);
    if (!ws || ws_bytes < need) return fail(QN_EWORKSPACE, "adapter-gradient workspace needs %zu bytes", need);
    if ((reinterpret_cast<uintptr_t>(ws) & 255u) != 0) return fail(QN_EALIGN, "workspace not 256-byte aligned");
    DropoutArgs drop;
    float sc = alpha / static_cast<float>(r);
    s = resolve_dropout(dropout, r, sc, &drop, &sc);
    if (s != QN_OK) return s;
    return cuda_status(launch_lora_grads(static_cast<const uint16_t *>(x), static_cast<const uint16_t *>(grad_h), M,
                                         n_out, k_in, static_cast<const uint16_t *>(A),
                                         static_cast<const uint16_t *>(B), r, sc, drop, grad_A, grad_B, ws,
                                         static_cast<cudaStream_t>(stream)),
                       "qlora_lora_grads");
}

qn_status qlora_workspace_size(int64_t M, int64_t n_out, int64_t k_in, int r, size_t *ws_bytes) {
    if (!ws_bytes) return fail(QN_EINVAL, "null output pointer");
    qn_status s = check_shape(n_out, k_in);
    if (s != QN_OK) return s;
    if (M < 0 || M > kMaxDim) return fail(QN_EINVAL, "M=%lld out of range", (long long)M);
    if (r < 0 || r > QN_MAX_RANK) return fail(QN_EINVAL, "rank r=%d outside [0, %d]", r, QN_MAX_RANK);
    // The few-token kernels keep the error word, the adapter product and its ready flag there
    // (4 KB); the tensor-core path and the paths that add a dropout-masked adapter term after a
    // base-only pass the error word and the M x roundup(r, 64) adapter operand.
    const size_t few = decode_fwd_workspace_bytes() > 4096 ? decode_fwd_workspace_bytes() : 4096;
    const size_t op = gemm_workspace_bytes(M, r);
    *ws_bytes = op > few ? op : few;
    g_err.clear();
    return QN_OK;
}

static qn_status check_linear(const qn_nf4_weight *w, const void *in, int64_t M, const void *A, const void *B, int r,
                              float alpha, const void *out, void *ws, size_t ws_bytes) {
    qn_status s = check_weight(w);
    if (s != QN_OK) return s;
    if (M < 0 || M > kMaxDim) return fail(QN_EINVAL, "M=%lld out of range", (long long)M);
    s = check_lora(A, B, r, alpha);
    if (s != QN_OK) return s;
    if (M == 0 || w->n_out == 0 || w->k_in == 0) return QN_OK;
    if (!in || !out) return fail(QN_EINVAL, "null activation or output pointer");
    if (!aligned16(in) || !aligned16(out)) return fail(QN_EALIGN, "activation or output not 16-byte aligned");
    if (in == out) return fail(QN_EINVAL, "output aliases the input");
    size_t need = 0;
    qlora_workspace_size(M, w->n_out, w->k_in, r, &need);
    if (!ws || ws_bytes < need) return fail(QN_EWORKSPACE, "linear workspace needs %zu bytes", need);
    return QN_OK;
}

qn_status qlora_workspace_check(void *ws, void *stream) {
    if (!ws) return fail(QN_EINVAL, "null workspace");
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    int word = 0;
    cudaError_t e = cudaMemcpyAsync(&word, ws, sizeof(int), cudaMemcpyDeviceToHost, st);
    if (e == cudaSuccess) e = cudaStreamSynchronize(st);
    if (e != cudaSuccess) return cuda_status(e, "qlora_workspace_check");
    if (word == 0) return cuda_status(cudaSuccess, "");
    e = cudaMemsetAsync(ws, 0, sizeof(int), st);
    if (e == cudaSuccess) e = cudaStreamSynchronize(st);
    if (e != cudaSuccess) return cuda_status(e, "qlora_workspace_check");
    return fail(QN_ETIMEOUT,
                "a kernel that used this workspace stopped early (error word %d: %s); its output is incomplete", word,
                word == 2 ? "dynamic shared memory not 1024-byte aligned" : "a bounded wait ran out");
}

qn_status qn_selftest_wait_timeout(void *ws, size_t ws_bytes, void *stream) {
    if (!ws || ws_bytes < 256) return fail(QN_EWORKSPACE, "the self-test needs a zeroed workspace of 256 bytes");
    return cuda_status(launch_wait_timeout_selftest(ws, static_cast<cudaStream_t>(stream)), "qn_selftest_wait_timeout");
}

qn_status qlora_linear_fwd(const qn_nf4_weight *w, const void *x, int64_t M, const void *A, const void *B, int r,
                           float alpha, void *h, void *ws, size_t ws_bytes, void *stream) {
    return qlora_linear_fwd_dropout(w, x, M, A, B, r, alpha, nullptr, h, ws, ws_bytes, stream);
}

qn_status qlora_linear_fwd_dropout(const qn_nf4_weight *w, const void *x, int64_t M, const void *A, const void *B,
                                   int r, float alpha, const qn_lora_dropout *dropout, void *h, void *ws,
                                   size_t ws_bytes, void *stream) {
    qn_status s = check_linear(w, x, M, A, B, r, alpha, h, ws, ws_bytes);
    if (s != QN_OK) return s;
    DropoutArgs drop;
    float sc = r > 0 ? alpha / static_cast<float>(r) : 0.0f;
    s = resolve_dropout(dropout, r, sc, &drop, &sc);
    if (s != QN_OK) return s;
    if (M == 0 || w->n_out == 0) return QN_OK;
    const WeightView wv = view(w);
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const uint16_t *xp = static_cast<const uint16_t *>(x);
    uint16_t *hp = static_cast<uint16_t *>(h);
    const uint16_t *Ap = static_cast<const uint16_t *>(A), *Bp = static_cast<const uint16_t *>(B);
    // few tokens and adapters of rank <= 64: the streamed kernel, 16 tokens per launch;
    // otherwise the tensor-core GEMM (any token count; the forward operand always suits TMA)
    if (M <= kDecodeMaxM && r <= kDecodeMaxRank) {
        int *err = static_cast<int *>(ws);
        for (int64_t m0 = 0; m0 < M; m0 += kDecodeTokens) {
            const int mc = static_cast<int>(M - m0 < kDecodeTokens ? M - m0 : kDecodeTokens);
            DropoutArgs dc = drop;
            dc.offset += static_cast<uint64_t>(m0 * w->k_in);  // element index of token m0
            cudaError_t e =
                launch_decode_fwd(wv, xp + m0 * w->k_in, mc, Ap, Bp, r, sc, dc, hp + m0 * w->n_out, err, st);
            if (e != cudaSuccess) return cuda_status(e, "qlora_linear_fwd");
        }
        return cuda_status(cudaSuccess, "");
    }
    if ((reinterpret_cast<uintptr_t>(ws) & 255u) != 0) return fail(QN_EALIGN, "workspace not 256-byte aligned");
    return cuda_status(launch_gemm_fwd(wv, xp, M, Ap, Bp, r, sc, hp, ws, st, &drop), "qlora_linear_fwd");
}

qn_status qlora_linear_bwd_x(const qn_nf4_weight *w, const void *grad_h, int64_t M, const void *A, const void *B,
                             int r, float alpha, void *grad_x, void *ws, size_t ws_bytes, void *stream) {
    return qlora_linear_bwd_x_dropout(w, grad_h, M, A, B, r, alpha, nullptr, grad_x, ws, ws_bytes, stream);
}

qn_status qlora_linear_bwd_x_dropout(const qn_nf4_weight *w, const void *grad_h, int64_t M, const void *A,
                                     const void *B, int r, float alpha, const qn_lora_dropout *dropout, void *grad_x,
                                     void *ws, size_t ws_bytes, void *stream) {
    qn_status s = check_linear(w, grad_h, M, A, B, r, alpha, grad_x, ws, ws_bytes);
    if (s != QN_OK) return s;
    DropoutArgs drop;
    float sc = r > 0 ? alpha / static_cast<float>(r) : 0.0f;
    s = resolve_dropout(dropout, r, sc, &drop, &sc);
    if (s != QN_OK) return s;
    if (M == 0 || w->k_in == 0) return QN_OK;
    const WeightView wv = view(w);
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const uint16_t *gp = static_cast<const uint16_t *>(grad_h);
    uint16_t *xp = static_cast<uint16_t *>(grad_x);
    const uint16_t *Ap = static_cast<const uint16_t *>(A), *Bp = static_cast<const uint16_t *>(B);
    // few tokens, adapters of rank <= 64 and TMA-friendly rows: the streamed kernel, 16 tokens per
    // launch
    if (M <= kDecodeMaxM && r <= kDecodeMaxRank && decode_bwd_stream_supported(w->n_out, w->k_in, r)) {
        int *err = static_cast<int *>(ws);
        for (int64_t m0 = 0; m0 < M; m0 += kDecodeTokens) {
            const int mc = static_cast<int>(M - m0 < kDecodeTokens ? M - m0 : kDecodeTokens);
            DropoutArgs dc = drop;
            dc.offset += static_cast<uint64_t>(m0 * w->k_in);  // element index of token m0
            cudaError_t e =
                launch_decode_bwd_stream(wv, gp + m0 * w->n_out, mc, Ap, Bp, r, sc, dc, xp + m0 * w->k_in, err, st);
            if (e != cudaSuccess) return cuda_status(e, "qlora_linear_bwd_x");
        }
        return cuda_status(cudaSuccess, "");
    }
    // Under dropout the other paths run base-only and the masked adapter term is added after them
    // (u = s B^T grad_h into the workspace, then grad_x += mask * u A).
    const bool masked = drop.thr != 0u;
    const int ra = masked ? 0 : r;
    if ((reinterpret_cast<uintptr_t>(ws) & 255u) != 0) return fail(QN_EALIGN, "workspace not 256-byte aligned");
    if (M > kDecodeMaxM && gemm_supported(w->n_out, w->k_in, M, true)) {
        cudaError_t e = launch_gemm_bwd(wv, gp, M, Ap, Bp, ra, sc, xp, ws, st);
        if (e != cudaSuccess) return cuda_status(e, "qlora_linear_bwd_x");
    } else {
        // many tokens with n_out % 8 != 0 (the GEMM's TMA row-stride rule), or few tokens with a
        // rank above 64 or rows the streamed kernel's boxes cannot read: the register-streaming
        // few-token kernel in chunks of 32 tokens
        constexpr int kChunk = 32;
        for (int64_t m0 = 0; m0 < M; m0 += kChunk) {
            const int mc = static_cast<int>(M - m0 < kChunk ? M - m0 : kChunk);
            cudaError_t e = launch_decode_bwd(wv, gp + m0 * w->n_out, mc, Ap, Bp, ra, sc, xp + m0 * w->k_in, st);
            if (e != cudaSuccess) return cuda_status(e, "qlora_linear_bwd_x");
        }
    }
    if (masked) {
        const int RT = (r + 63) / 64 * 64;
        uint16_t *u = reinterpret_cast<uint16_t *>(static_cast<char *>(ws) + 256);
        cudaError_t e = launch_lora_down(gp, M, w->n_out, Bp, 1, r, r, sc, u, RT, st);
        if (e == cudaSuccess) e = launch_adapter_up_masked(u, M, RT, Ap, r, w->k_in, drop, xp, st);
        if (e != cudaSuccess) return cuda_status(e, "qlora_linear_bwd_x");
    }
    return cuda_status(cudaSuccess, "");
}

}  // extern "C"
