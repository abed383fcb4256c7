"""Parity of the CUDA path (through the C ABI) against the CPU oracle.

Codes, FP8 constants, group scales, the mean and the standalone dequantisation must
match bit for bit. h and grad_x (bf16, fp32 accumulation) must satisfy, per element,
|err| <= 1e-2 * |ref| + 1e-2 * rms(ref) against the fp64 oracle.
"""
import os

import numpy as np
import pytest
import torch

from bit_nf4_quantized_25_b200 import binding as qb
from bit_nf4_quantized_25_b200 import synth

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

DEV = "cuda"
RTOL = 1e-2  # relative part of the per-element bound
STOL = 1e-2  # part relative to the rms of the reference


def bits(t):
    return synth.bf16_bits(t)


def bf16_to_f64(u16):
    return (u16.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def assert_close(got_bf16: torch.Tensor, ref: np.ndarray, what: str):
    g = bf16_to_f64(bits(got_bf16)).reshape(ref.shape)
    rms = float(np.sqrt(np.mean(ref * ref))) if ref.size else 0.0
    err = np.abs(g - ref)
    bound = RTOL * np.abs(ref) + STOL * rms
    bad = err > bound
    assert not bad.any(), (f"{what}: {bad.sum()} of {bad.size} elements outside tolerance; "
                           f"worst err/bound = {np.max(err / np.maximum(bound, 1e-300)):.3g}")
    return float(np.max(err / np.maximum(bound, 1e-300))) if ref.size else 0.0


def quantize_both(oracle, W: torch.Tensor):
    n, k = W.shape
    w = qb.nf4_quantize(W)
    torch.cuda.synchronize()
    ref = oracle.nf4_quantize(bits(W), n, k)
    return w, ref


def assert_quant_equal(w, ref, what=""):
    codes = w.codes.cpu().numpy()
    q = w.absmax_q.cpu().numpy()
    sigma = w.group_scale.cpu().numpy()
    mu = w.absmax_mean.cpu().numpy()[0]
    assert mu.view(np.uint32) == np.float32(ref["mu"]).view(np.uint32), (what, mu, ref["mu"])
    nbad = int(np.sum(codes != ref["codes"]))
    assert nbad == 0, f"{what}: {nbad} code bytes differ"
    assert np.array_equal(q, ref["q"]), f"{what}: {int(np.sum(q != ref['q']))} FP8 constants differ"
    assert np.array_equal(sigma.view(np.uint32), ref["sigma"].view(np.uint32)), f"{what}: group scales differ"


def to_host_weight(w):
    d = dict(codes=w.codes.cpu().numpy(), qtype=w.quant_type, dq=w.double_quant)
    if w.double_quant:
        d.update(q=w.absmax_q.cpu().numpy(), sigma=w.group_scale.cpu().numpy(),
                 mu=np.float32(w.absmax_mean.cpu().numpy()[0]))
    else:
        d.update(absmax=w.absmax.cpu().numpy())
    return d


# ------------------------------------------------------------------ quantiser

def test_quantize_tiny_bit_exact(oracle):
    W, *_ = synth.layer_inputs(synth.tiny_case(), DEV)
    w, ref = quantize_both(oracle, W)
    assert_quant_equal(w, ref, "tiny")


@pytest.mark.parametrize("arrangement", ["shuffled", "sorted", "signed"])
def test_quantize_every_finite_bf16_pattern(oracle, arrangement):
    # Every finite bf16 weight, in blocks with absmaxes across the whole range:
    # exhaustive for the code decision, wide-range for the exact mean.
    u = np.arange(65536, dtype=np.uint32)
    finite = ((u >> 7) & 0xFF) != 0xFF
    pats = u[finite].astype(np.uint16)
    if arrangement == "shuffled":
        pats = np.random.default_rng(0).permutation(pats)
    elif arrangement == "signed":
        mag = pats[pats < 0x8000]
        pats = np.stack([mag, mag | 0x8000], 1).reshape(-1)
        pats = np.random.default_rng(1).permutation(pats.reshape(-1, 64)).reshape(-1)
    pad = (-pats.size) % (64 * 4)
    pats = np.concatenate([pats, np.zeros(pad, np.uint16)])
    n, k = pats.size // 256, 256
    W = torch.from_numpy(pats.view(np.int16).reshape(n, k).copy()).view(torch.bfloat16).to(DEV)
    w, ref = quantize_both(oracle, W)
    assert_quant_equal(w, ref, arrangement)


@pytest.mark.parametrize("n,k", [(1, 64), (3, 192), (200, 448), (5, 64 * 172), (4096, 4096), (11008, 4096),
                                 (4096, 11008), (8192, 8192), (28672, 8192), (8192, 28672)])
def test_quantize_shapes_bit_exact(oracle, n, k):
    W = synth.normal_bf16((n, k), 0.015 if max(n, k) > 11008 else 0.02, seed=n * 7 + k, device=DEV)
    w, ref = quantize_both(oracle, W)
    assert_quant_equal(w, ref, f"{n}x{k}")


def test_quantize_special_blocks(oracle):
    # all-zero blocks (code 7), blocks with equal absmax (sigma 0), a single non-zero
    W = torch.zeros(4, 1024, dtype=torch.bfloat16)
    W[1, ::64] = 0.375
    W[1, 5::64] = -0.1
    W[2, 7] = -3.0e-3
    W[3, :] = 1.0
    w, ref = quantize_both(oracle, W.to(DEV))
    assert_quant_equal(w, ref, "special")


def test_dequant_bit_exact(oracle):
    for n, k, seed in [(256, 256, 0), (3, 64 * 172, 5), (4096, 4096, 7)]:
        W = synth.student_t_bf16((n, k), 0.02, seed, device=DEV)
        w = qb.nf4_quantize(W)
        deq = qb.nf4_dequantize(w)
        torch.cuda.synchronize()
        ref = oracle.nf4_dequant_bf16(to_host_weight(w), n, k)
        got = bits(deq).reshape(n, k)
        assert np.array_equal(got, ref), f"{n}x{k}: {int(np.sum(got != ref))} dequantised weights differ"


def _bulk_layers():
    return int(os.environ.get("QN_BULK_LAYERS", "32"))


def test_bulk_quantize_roundtrip(oracle):
    # 32 layers of the 7B shapes (6.48e9 weights), Student-t(4) * 0.02 with 0.1 % outliers x 20.
    worst = 0.0
    for layer in range(_bulk_layers()):
        for name, (n, k) in synth.SHAPES_7B.items():
            W = synth.bulk_tensor(layer, name, device=DEV)
            w = qb.nf4_quantize(W)
            deq = qb.nf4_dequantize(w)
            torch.cuda.synchronize()
            Wh = bits(W)
            ref = oracle.nf4_quantize(Wh, n, k)
            assert_quant_equal(w, ref, f"layer {layer} {name}")
            got = bits(deq).reshape(n, k)
            rdq = oracle.nf4_dequant_bf16(ref, n, k)
            assert np.array_equal(got, rdq), f"layer {layer} {name}: dequant differs"
            # Round-trip error per block: first level within half the widest table gap of
            # c_b, second level within the FP8 rounding of d_b = c_b - mu (3 mantissa bits,
            # subnormal step 2^-9 sigma), then one bf16 rounding of the product.
            wf = bf16_to_f64(Wh).reshape(-1, 64)
            df = bf16_to_f64(got).reshape(-1, 64)
            c = ref["absmax"].astype(np.float64)
            mu = float(ref["mu"])
            sig = np.repeat(ref["sigma"].astype(np.float64), 256)[: c.size]
            dq = 2.0 ** -4 * np.abs(c - mu) + 2.0 ** -10 * sig + 2.0 ** -22 * (c + abs(mu))
            half_gap = float(np.max(np.diff(oracle.nf4_table()))) / 2  # (T[1] - T[0]) / 2
            bound = half_gap * c + dq + 2.0 ** -8 * (c + dq)
            err = np.max(np.abs(wf - df), axis=1)
            assert np.all(err <= bound * (1 + 1e-6)), f"layer {layer} {name}: round-trip bound"
            worst = max(worst, float(np.max(err / np.maximum(c, 1e-30))))
            del W, w, deq
    print(f"worst block round-trip error / absmax: {worst:.4f}")


# --------------------------------------------------------------- linear layer

def run_case(oracle, case: synth.LayerCase, rows=None, check_bwd=True, quant_type="nf4", double_quant=True):
    W, A, B, x, gh = synth.layer_inputs(case, DEV, need_grad=check_bwd)
    w = qb.nf4_quantize(W, quant_type=quant_type, double_quant=double_quant)
    r = case.r
    Ad, Bd = (A, B) if r > 0 else (None, None)
    h = qb.qlora_linear_fwd(w, x, Ad, Bd, case.alpha)
    gx = qb.qlora_linear_bwd_x(w, gh, Ad, Bd, case.alpha) if check_bwd else None
    torch.cuda.synchronize()
    hw = to_host_weight(w)
    n, k, M = case.n_out, case.k_in, case.M
    Ab, Bb = (bits(A), bits(B)) if r > 0 else (None, None)
    sel = np.arange(M) if rows is None else np.asarray(rows)
    ref_h = oracle.qlora_fwd(hw, n, k, bits(x), M, Ab, Bb, r, case.alpha, rows=sel)
    worst = assert_close(h[torch.as_tensor(sel, device=DEV)], ref_h, f"{case.name} fwd")
    if check_bwd:
        ref_g = oracle.qlora_bwd_x(hw, n, k, bits(gh), M, Ab, Bb, r, case.alpha, rows=sel)
        worst = max(worst, assert_close(gx[torch.as_tensor(sel, device=DEV)], ref_g, f"{case.name} bwd_x"))
    return worst


@pytest.mark.parametrize("n,k,M,r", [(128, 64, 65, 0), (128, 128, 256, 16), (256, 256, 300, 4), (200, 448, 129, 64),
                                     (384, 192, 513, 200), (136, 1024, 1000, 16)])
def test_gemm_small(oracle, n, k, M, r):
    # tensor-core path (M > 64): ragged rows, features, tokens and adapter ranks
    run_case(oracle, synth.LayerCase(f"gemm{n}x{k}M{M}r{r}", n, k, M, r, 2.0 * max(r, 1), 0.02, n * 3 + k + M))


@pytest.mark.parametrize("M", [300, 5])
def test_error_word_stays_clear(oracle, M):
    # tensor-core path (M > 64) and few-token path: a run without a timeout leaves the
    # workspace error word at zero, and qlora_workspace_check reports success
    case = synth.LayerCase("err_word", 256, 512, M, 16, 32.0, 0.02, 99)
    W, A, B, x, gh = synth.layer_inputs(case, DEV)
    w = qb.nf4_quantize(W)
    ws = qb.new_workspace(qb.linear_workspace_size(M, 256, 512, 16))
    qb.qlora_linear_fwd(w, x, A, B, 32.0, workspace=ws)
    qb.qlora_linear_bwd_x(w, gh, A, B, 32.0, workspace=ws)
    torch.cuda.synchronize()
    assert int(ws[:4].view(torch.int32).item()) == 0
    qb.workspace_check(ws)


def test_bounded_wait_runs_out_and_is_reported():
    # The shared failure path of the kernels, exercised without a fault: a kernel's bounded wait on a
    # workspace word that nothing sets runs out, the kernel records the timeout in the error word,
    # the check reports QN_ETIMEOUT and clears it, and the device stays usable.
    ws = qb.new_workspace(4096)
    qb.selftest_wait_timeout(ws)
    with pytest.raises(qb.QNError) as e:
        qb.workspace_check(ws)
    assert e.value.status == qb.QN_ETIMEOUT
    qb.workspace_check(ws)  # cleared
    W = synth.normal_bf16((256, 256), 0.02, 3, DEV)
    w = qb.nf4_quantize(W)
    x = synth.normal_bf16((4, 256), 1.0, 4, DEV)
    h = qb.qlora_linear_fwd(w, x, None, None, 0.0, workspace=ws)
    torch.cuda.synchronize()
    assert torch.isfinite(h.float()).all()
    qb.workspace_check(ws)


def test_error_word_is_reported_and_cleared():
    # a set error word (what a kernel writes when a bounded wait runs out) is reported as
    # QN_ETIMEOUT by the check, which clears it
    ws = qb.new_workspace(256)
    ws[:4].view(torch.int32).fill_(1)
    with pytest.raises(qb.QNError) as e:
        qb.workspace_check(ws)
    assert e.value.status == qb.QN_ETIMEOUT
    assert int(ws[:4].view(torch.int32).item()) == 0
    qb.workspace_check(ws)


def test_tiny_fwd_bwd(oracle):
    run_case(oracle, synth.tiny_case())


@pytest.mark.parametrize("case", synth.decode7b_cases(), ids=lambda c: c.name)
def test_decode7b_fwd_bwd(oracle, case):
    run_case(oracle, case, check_bwd=True)


@pytest.mark.parametrize("case", [c for c in synth.l70b_cases() if c.M <= 16], ids=lambda c: c.name)
def test_l70b_decode_fwd_bwd(oracle, case):
    run_case(oracle, case)


def _sample_rows(M, seed, n=128):
    rng = np.random.default_rng(seed)
    rows = set(rng.choice(M, size=min(n, M), replace=False).tolist())
    rows.update([0, M - 1])
    return sorted(rows)


@pytest.mark.parametrize("case", synth.train7b_cases(), ids=lambda c: c.name)
def test_train7b_sampled_rows(oracle, case):
    run_case(oracle, case, rows=_sample_rows(case.M, case.seed))


@pytest.mark.parametrize("case", [c for c in synth.l70b_cases() if c.M > 16], ids=lambda c: c.name)
def test_l70b_train_sampled_rows(oracle, case):
    run_case(oracle, case, rows=_sample_rows(case.M, case.seed, 64))


@pytest.mark.parametrize("M", [1, 3, 8, 13, 31, 33, 64, 65, 100, 257])
def test_ragged_token_counts(oracle, M):
    run_case(oracle, synth.LayerCase(f"ragged_M{M}", 320, 448, M, 16, 32.0, 0.02, 500 + M))


@pytest.mark.parametrize("r,alpha", [(0, 0.0), (1, 2.0), (4, 8.0), (64, 16.0), (200, 400.0), (256, 16.0)])
def test_lora_ranks(oracle, r, alpha):
    run_case(oracle, synth.LayerCase(f"rank{r}", 192, 512, 12, r, alpha, 0.02, 900 + r))


@pytest.mark.parametrize("n,k", [(1, 64), (17, 64), (200, 192), (130, 64 * 19), (4100, 320)])
def test_ragged_weight_shapes(oracle, n, k):
    run_case(oracle, synth.LayerCase(f"shape{n}x{k}", n, k, 5, 4, 8.0, 0.02, n + k))


@pytest.mark.parametrize("M", [1, 7, 12])
def test_ragged_rows_on_128_row_chunks(oracle, M):
    # 4160 rows: the few-token planner takes 128-row chunks here, so the last chunk holds 64 rows
    # and the specialised two-m-tile loop runs on rows past the weight (read as zero, not stored)
    run_case(oracle, synth.LayerCase(f"rows4160_M{M}", 4160, 4096, M, 16, 32.0, 0.02, 4160 + M), check_bwd=True)


def test_zero_adapter_and_zero_base(oracle):
    case = synth.LayerCase("zeroB", 256, 512, 9, 16, 32.0, 0.02, 77)
    W, A, B, x, gh = synth.layer_inputs(case, DEV)
    for Wz, Bz in ((W, torch.zeros_like(B)), (torch.zeros_like(W), B)):
        w = qb.nf4_quantize(Wz)
        h = qb.qlora_linear_fwd(w, x, A, Bz, case.alpha)
        gx = qb.qlora_linear_bwd_x(w, gh, A, Bz, case.alpha)
        torch.cuda.synchronize()
        hw = to_host_weight(w)
        assert_close(h, oracle.qlora_fwd(hw, 256, 512, bits(x), 9, bits(A), bits(Bz), 16, 32.0), "zero fwd")
        assert_close(gx, oracle.qlora_bwd_x(hw, 256, 512, bits(gh), 9, bits(A), bits(Bz), 16, 32.0), "zero bwd")


def test_adjoint_identity_on_gpu(oracle):
    # <grad_h, fwd(x)> = <bwd_x(grad_h), x> holds for the exact layer; the GPU results
    # satisfy it to the accuracy of bf16 outputs.
    case = synth.LayerCase("adjoint", 1024, 2048, 16, 16, 32.0, 0.02, 4242)
    W, A, B, x, gh = synth.layer_inputs(case, DEV)
    w = qb.nf4_quantize(W)
    h = qb.qlora_linear_fwd(w, x, A, B, case.alpha).double()
    gx = qb.qlora_linear_bwd_x(w, gh, A, B, case.alpha).double()
    lhs = float((gh.double() * h).sum())
    rhs = float((gx * x.double()).sum())
    scale = float(h.norm() * gh.double().norm())
    assert abs(lhs - rhs) <= 1e-2 * scale


def test_empty_token_batch_is_noop():
    W = synth.normal_bf16((128, 128), 0.02, 1, DEV)
    w = qb.nf4_quantize(W)
    x = torch.empty(0, 128, dtype=torch.bfloat16, device=DEV)
    h = qb.qlora_linear_fwd(w, x, None, None, 0.0)
    assert h.shape == (0, 128)


@pytest.mark.parametrize("n,k,M,bwd", [(11008, 4096, 4096, False), (4096, 11008, 4096, True), (11008, 4096, 16, False),
                                       (4096, 11008, 16, True)])
def test_repeat_runs_bit_identical(n, k, M, bwd):
    # The kernels have a fixed reduction order, so repeated calls on the same inputs must give
    # the same bits; a difference means a race (the many-token grids span several waves).
    case = synth.LayerCase(f"repeat{n}x{k}M{M}", n, k, M, 16, 32.0, 0.02, 4242 + M)
    W, A, B, x, gh = synth.layer_inputs(case, DEV, need_grad=bwd)
    w = qb.nf4_quantize(W)
    ws = torch.zeros(qb.linear_workspace_size(M, n, k, 16), dtype=torch.uint8, device=DEV)
    first = None
    for _ in range(8):
        out = (qb.qlora_linear_bwd_x(w, gh, A, B, 32.0, workspace=ws) if bwd
               else qb.qlora_linear_fwd(w, x, A, B, 32.0, workspace=ws))
        torch.cuda.synchronize()
        got = out.view(torch.int16).clone()
        if first is None:
            first = got
        else:
            assert torch.equal(got, first), f"run-to-run difference in {int((got != first).sum())} elements"
    assert int(ws[:4].view(torch.int32).item()) == 0


# ------------------------------------------------------------------------- merge

def _ulp_diff_bf16(a: np.ndarray, b: np.ndarray) -> np.ndarray:
    """Distance in bf16 units between two arrays of bf16 bit patterns (finite values)."""
    def key(u):
        u = u.astype(np.int32)
        return np.where(u & 0x8000, -(u & 0x7fff), u & 0x7fff)
    return np.abs(key(a) - key(b))


@pytest.mark.parametrize("n,k,r,alpha", [(256, 256, 4, 8.0), (200, 448, 5, 10.0), (4096, 4096, 16, 32.0),
                                         (1000, 64 * 19, 64, 16.0), (130, 256, 256, 16.0), (64, 128, 0, 0.0)])
def test_merge_matches_oracle(oracle, n, k, r, alpha):
    # "QLoRA & PEFT family" 3.6 (merge_and_unload): W' + s B A as bf16. The GPU adds the fp32
    # tensor-core product to the fp32 dequantised weight (one fp32 rounding) before rounding to
    # bf16, so it may differ from the exactly rounded oracle by one bf16 unit.
    case = synth.LayerCase(f"merge{n}x{k}r{r}", n, k, 1, max(r, 1), alpha, 0.02, 7 * n + k + r)
    W, A, B, _, _ = synth.layer_inputs(case, DEV, need_grad=False)
    w = qb.nf4_quantize(W)
    Ad, Bd = (A, B) if r > 0 else (None, None)
    got = bits(qb.qlora_merge_bf16(w, Ad, Bd, alpha)).reshape(n, k)
    torch.cuda.synchronize()
    hw = to_host_weight(w)
    ref = oracle.merge_bf16(hw, n, k, bits(A) if r > 0 else None, bits(B) if r > 0 else None, r, alpha)
    # within the stated tolerance everywhere; off by more than one bf16 unit only where the sum
    # cancels (the fp32 rounding of the product then spans several units of the small result)
    assert_close(torch.from_numpy(got.view(np.int16)).view(torch.bfloat16), bf16_to_f64(ref), "merge")
    d = _ulp_diff_bf16(got, ref)
    assert float(np.mean(d <= 1)) > 0.999, f"{int((d > 1).sum())} merged weights more than one bf16 unit off"
    assert float(np.mean(d == 0)) > 0.98
    if r == 0:
        assert np.array_equal(got, oracle.nf4_dequant_bf16(hw, n, k))


# --------------------------------------------------------- adapter weight gradients

def _assert_close_f32(got: torch.Tensor, ref: np.ndarray, what: str):
    g = got.detach().cpu().numpy().astype(np.float64).reshape(ref.shape)
    rms = float(np.sqrt(np.mean(ref * ref))) if ref.size else 0.0
    err = np.abs(g - ref)
    bound = RTOL * np.abs(ref) + STOL * rms
    bad = err > bound
    assert not bad.any(), (f"{what}: {bad.sum()} of {bad.size} elements outside tolerance; "
                           f"worst err/bound = {np.max(err / np.maximum(bound, 1e-300)):.3g}")


@pytest.mark.parametrize("n,k,M,r,alpha", [(256, 256, 8, 4, 8.0), (200, 448, 129, 5, 10.0), (17, 64, 33, 16, 32.0),
                                           (4096, 4096, 4096, 16, 32.0), (11008, 4096, 512, 16, 32.0),
                                           (8192, 28672, 256, 64, 16.0), (320, 192, 70, 200, 400.0)])
def test_lora_grads_match_oracle(oracle, n, k, M, r, alpha):
    # "How does QLoRA work for training?" 2 and 7: only B and A are trained; grad_B = s grad_h^T (x A^T),
    # grad_A = s (grad_h B)^T x, fp32 outputs within the stated tolerance of the fp64 oracle.
    case = synth.LayerCase(f"grads{n}x{k}M{M}r{r}", n, k, M, r, alpha, 0.02, 3 * n + k + M + r)
    _, A, B, x, gh = synth.layer_inputs(case, DEV)
    gA, gB = qb.qlora_lora_grads(x, gh, A, B, alpha)
    torch.cuda.synchronize()
    rA, rB = oracle.lora_grads(bits(x), bits(gh), M, n, k, bits(A), bits(B), r, alpha)
    _assert_close_f32(gA, rA, "grad_A")
    _assert_close_f32(gB, rB, "grad_B")


def test_lora_grads_repeat_bit_identical():
    case = synth.LayerCase("grads_repeat", 1024, 2048, 777, 16, 32.0, 0.02, 5)
    _, A, B, x, gh = synth.layer_inputs(case, DEV)
    ws = torch.empty(qb.lora_grads_workspace_size(777, 16), dtype=torch.uint8, device=DEV)
    first = None
    for _ in range(4):
        gA, gB = qb.qlora_lora_grads(x, gh, A, B, 32.0, workspace=ws)
        torch.cuda.synchronize()
        cur = (gA.clone(), gB.clone())
        if first is None:
            first = cur
        else:
            assert torch.equal(cur[0], first[0]) and torch.equal(cur[1], first[1])


@pytest.mark.parametrize("n,M,r", [(204, 129, 16), (200 + 4, 65, 4), (100, 70, 100)])
def test_bwd_many_tokens_with_unaligned_rows(oracle, n, M, r):
    # more than 64 tokens with n_out % 8 != 0 (the tensor-core path's TMA row-stride rule fails),
    # and few-token input gradients with a rank above 64: the fallback few-token kernel in chunks
    run_case(oracle, synth.LayerCase(f"bwd_unaligned{n}M{M}r{r}", n, 256, M, r, 2.0 * r, 0.02, 11 * n + M + r))


# ---------------------------------------------------------------- LoRA dropout
# "QLoRA & PEFT family" 3.4 and the lora_dropout setting of "How does QLoRA work for training?":
# dropout of the adapter's input. With a zero base and identity adapters the layer returns the
# masked, scaled input itself, so the mask is compared bit for bit with the oracle's generator;
# the other tests compare whole layers (adapter-dominated, so that a wrong mask shows).

def _zero_weight(n, k):
    return qb.nf4_quantize(torch.zeros(n, k, dtype=torch.bfloat16, device=DEV))


def _identity_adapters(r):
    eye = torch.eye(r, dtype=torch.bfloat16, device=DEV)
    return eye.contiguous(), eye.clone()


@pytest.mark.parametrize("M", [1, 5, 16, 40, 100])
def test_dropout_mask_is_the_generators(oracle, M):
    n = k = r = 64
    p, seed, offset = 0.25, 0x1234_5678_9ABC_DEF0, 12345
    w = _zero_weight(n, k)
    A, B = _identity_adapters(r)
    x = (torch.rand(M, k, generator=torch.Generator().manual_seed(M)) + 0.5).to(torch.bfloat16).to(DEV)
    # h = s / (1 - p) B (A (mask x)) = s / (1 - p) (mask x), s = alpha / r = 1
    h = qb.qlora_linear_fwd(w, x, A, B, float(r) * (1 - p), dropout=(p, seed, offset))
    gh = x.clone()
    gx = qb.qlora_linear_bwd_x(w, gh, A, B, float(r) * (1 - p), dropout=(p, seed, offset))
    torch.cuda.synchronize()
    keep = oracle.dropout_keep(seed, offset, p, M, k)
    for got, what in ((h, "fwd"), (gx, "bwd_x")):
        g = got.float().cpu().numpy()
        assert np.array_equal(g != 0, keep), f"{what}: {int(np.sum((g != 0) != keep))} mask bits differ"
        np.testing.assert_allclose(g[keep], x.float().cpu().numpy()[keep], rtol=1e-2)


@pytest.mark.parametrize("n,k,M,r,zero_base", [(4096, 4096, 1, 16, True), (4096, 4096, 5, 16, False),
                                               (11008, 4096, 16, 16, True), (4096, 11008, 3, 64, True),
                                               (256, 512, 300, 16, True), (204, 256, 40, 16, True),
                                               (200, 448, 129, 8, True)])
def test_dropout_layer_matches_oracle(oracle, n, k, M, r, zero_base):
    # few-token kernels (M <= 16 per launch), the tensor-core path (M > 64) and the fallback
    # paths (n_out % 8 != 0; M > 64 with n_out % 8 != 0): forward and input gradient vs the oracle
    p, seed, offset = 0.1, 987654321, 3 * n + k
    case = synth.LayerCase(f"drop{n}x{k}M{M}", n, k, M, r, 2.0 * r, 0.02, n + k + M)
    W, A, B, x, gh = synth.layer_inputs(case, DEV)
    if zero_base:
        W = torch.zeros_like(W)
    A, B = A * 30, B * 30  # an adapter term comparable to the base
    w = qb.nf4_quantize(W)
    h = qb.qlora_linear_fwd(w, x, A, B, case.alpha, dropout=(p, seed, offset))
    gx = qb.qlora_linear_bwd_x(w, gh, A, B, case.alpha, dropout=(p, seed, offset))
    torch.cuda.synchronize()
    hw = to_host_weight(w)
    ref_h = oracle.qlora_fwd(hw, n, k, bits(x), M, bits(A), bits(B), r, case.alpha, p_drop=p, seed=seed,
                             offset=offset)
    ref_g = oracle.qlora_bwd_x(hw, n, k, bits(gh), M, bits(A), bits(B), r, case.alpha, p_drop=p, seed=seed,
                               offset=offset)
    assert_close(h, ref_h, f"{case.name} fwd")
    assert_close(gx, ref_g, f"{case.name} bwd_x")


@pytest.mark.parametrize("n,k,M,r", [(256, 256, 8, 4), (1024, 2048, 300, 16), (512, 4096, 33, 64)])
def test_dropout_lora_grads_match_oracle(oracle, n, k, M, r):
    p, seed, offset = 0.2, 42, 7
    case = synth.LayerCase(f"dropgrads{n}x{k}M{M}", n, k, M, r, 2.0 * r, 0.02, 2 * n + k + M)
    _, A, B, x, gh = synth.layer_inputs(case, DEV)
    gA, gB = qb.qlora_lora_grads(x, gh, A, B, case.alpha, dropout=(p, seed, offset))
    torch.cuda.synchronize()
    rA, rB = oracle.lora_grads(bits(x), bits(gh), M, n, k, bits(A), bits(B), r, case.alpha, p, seed, offset)
    _assert_close_f32(gA, rA, "grad_A")
    _assert_close_f32(gB, rB, "grad_B")


def test_dropout_rate_zero_is_the_plain_call():
    case = synth.LayerCase("drop0", 1024, 2048, 9, 16, 32.0, 0.02, 5)
    W, A, B, x, gh = synth.layer_inputs(case, DEV)
    w = qb.nf4_quantize(W)
    a = qb.qlora_linear_fwd(w, x, A, B, 32.0)
    b = qb.qlora_linear_fwd(w, x, A, B, 32.0, dropout=(0.0, 11, 13))
    c = qb.qlora_linear_bwd_x(w, gh, A, B, 32.0)
    d = qb.qlora_linear_bwd_x(w, gh, A, B, 32.0, dropout=(0.0, 11, 13))
    torch.cuda.synchronize()
    assert torch.equal(a, b) and torch.equal(c, d)


# ------------------------------------------- quant type and constant format
# The other settings of the 4-bit load ("Quantized LoRA (QLoRA) and 4-bit training", the four
# configuration knobs): the 4-bit float (E2M1 / 6) instead of NF4, and fp32 block constants
# instead of double quantisation. Codes and constants bit-exact, the layer within tolerance, on
# every kernel path: few-token forward and input gradient (streamed and per-slice), the
# tensor-core GEMM and the merge.

FORMATS = [("fp4", True), ("fp4", False), ("nf4", False)]


def _fmt_id(f):
    return f"{f[0]}-{'dq' if f[1] else 'f32'}"


def assert_format_equal(w, ref, what):
    codes = w.codes.cpu().numpy()
    nbad = int(np.sum(codes != ref["codes"]))
    assert nbad == 0, f"{what}: {nbad} code bytes differ"
    if w.double_quant:
        assert_quant_equal(w, ref, what)
    else:
        got = w.absmax.cpu().numpy()
        assert np.array_equal(got.view(np.uint32), ref["absmax"].view(np.uint32)), f"{what}: fp32 constants differ"


@pytest.mark.parametrize("fmt", FORMATS, ids=_fmt_id)
@pytest.mark.parametrize("n,k", [(1, 64), (200, 448), (5, 64 * 172), (4096, 4096), (11008, 4096)])
def test_format_quantize_bit_exact(oracle, fmt, n, k):
    W = synth.student_t_bf16((n, k), 0.02, seed=n + 3 * k, device=DEV)
    w = qb.nf4_quantize(W, quant_type=fmt[0], double_quant=fmt[1])
    torch.cuda.synchronize()
    ref = oracle.quantize4(bits(W), n, k, fmt[0], fmt[1])
    assert_format_equal(w, ref, f"{_fmt_id(fmt)} {n}x{k}")


@pytest.mark.parametrize("dq", [True, False])
def test_fp4_every_finite_bf16_pattern(oracle, dq):
    # exhaustive for the 4-bit float's code decision (its ties and the IEEE-quotient path)
    u = np.arange(65536, dtype=np.uint32)
    pats = u[((u >> 7) & 0xFF) != 0xFF].astype(np.uint16)
    pats = np.random.default_rng(2).permutation(pats)
    pats = np.concatenate([pats, np.zeros((-pats.size) % 256, np.uint16)])
    n, k = pats.size // 256, 256
    W = torch.from_numpy(pats.view(np.int16).reshape(n, k).copy()).view(torch.bfloat16).to(DEV)
    w = qb.nf4_quantize(W, quant_type="fp4", double_quant=dq)
    torch.cuda.synchronize()
    assert_format_equal(w, oracle.quantize4(bits(W), n, k, "fp4", dq), "fp4 all bf16")


def test_fp4_special_blocks(oracle):
    # all-zero blocks (code 0), exact ties at representable midpoints, +-absmax
    W = torch.zeros(4, 1024, dtype=torch.bfloat16)
    W[1, ::64] = 1.0
    W[1, 1::64] = 0.125   # 1/8 of the absmax: a midpoint between 1/12 and 1/6
    W[1, 2::64] = -0.125
    W[2, 7] = -3.0e-3
    W[3, :] = -2.0
    for dq in (True, False):
        w = qb.nf4_quantize(W.to(DEV), quant_type="fp4", double_quant=dq)
        torch.cuda.synchronize()
        assert_format_equal(w, oracle.quantize4(bits(W), 4, 1024, "fp4", dq), f"fp4 special dq={dq}")


@pytest.mark.parametrize("fmt", FORMATS, ids=_fmt_id)
def test_format_dequant_bit_exact(oracle, fmt):
    for n, k, seed in [(256, 256, 0), (3, 64 * 172, 5), (4096, 4096, 7)]:
        W = synth.student_t_bf16((n, k), 0.02, seed, device=DEV)
        w = qb.nf4_quantize(W, quant_type=fmt[0], double_quant=fmt[1])
        deq = qb.nf4_dequantize(w)
        torch.cuda.synchronize()
        ref = oracle.nf4_dequant_bf16(to_host_weight(w), n, k)
        got = bits(deq).reshape(n, k)
        assert np.array_equal(got, ref), f"{n}x{k}: {int(np.sum(got != ref))} dequantised weights differ"


@pytest.mark.parametrize("fmt", FORMATS, ids=_fmt_id)
@pytest.mark.parametrize("n,k,M,r", [(4096, 4096, 1, 16), (11008, 4096, 16, 16), (4096, 11008, 5, 16),
                                     (200, 448, 7, 5), (136, 1024, 3, 0), (256, 256, 300, 4),
                                     (200, 448, 129, 64)])
def test_format_layer_matches_oracle(oracle, fmt, n, k, M, r):
    # M <= 16: streamed few-token kernels (r = 5 and n = 200 take the per-slice input gradient);
    # M > 64: the tensor-core GEMM
    case = synth.LayerCase(f"{_fmt_id(fmt)}{n}x{k}M{M}r{r}", n, k, M, r, 2.0 * max(r, 1), 0.02, n + k + M + r)
    run_case(oracle, case, quant_type=fmt[0], double_quant=fmt[1])


@pytest.mark.parametrize("fmt", FORMATS, ids=_fmt_id)
def test_format_merge_matches_oracle(oracle, fmt):
    n, k, r, alpha = 200, 448, 5, 10.0
    W = synth.normal_bf16((n, k), 0.02, 4, DEV)
    A = synth.normal_bf16((r, k), 0.01, 5, DEV)
    B = synth.normal_bf16((n, r), 0.01, 6, DEV)
    w = qb.nf4_quantize(W, quant_type=fmt[0], double_quant=fmt[1])
    got = qb.qlora_merge_bf16(w, A, B, alpha)
    torch.cuda.synchronize()
    ref = oracle.merge_bf16(to_host_weight(w), n, k, bits(A), bits(B), r, alpha)
    g = bits(got).reshape(n, k)
    assert_close(torch.from_numpy(g.view(np.int16)).view(torch.bfloat16), bf16_to_f64(ref), "merge")
    d = _ulp_diff_bf16(g, ref)
    assert float(np.mean(d <= 1)) > 0.999, f"{int((d > 1).sum())} merged weights more than one bf16 unit off"
