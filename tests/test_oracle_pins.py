"""Pins for the CPU oracle, each against something other than the oracle itself:
values printed on the pages, closed forms, library routines for the special
cases that reduce to them, invariants, and brute force on tiny inputs.

Page titles used in the citations:
  [apxml]  "Quantized LoRA (QLoRA) and 4-bit training" (apxml.com course page)
  [codex]  "QLoRA & PEFT family" (ai-reference-codex book notes)
  [aivaro] "How does QLoRA work for training?" (aivaro.ru answer 482)
  [tqpw]   "QLoRA paper notes" (tqpw.cn news 348736)
"""
import math
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden_table():
    vals = []
    with open(os.path.join(GOLDEN, "nf4_table.txt")) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                vals.append(float(line))
    return np.array(vals)


def _bf16_all_finite():
    bits = np.arange(65536, dtype=np.uint32)
    f = (bits << 16).view(np.float32)
    ok = np.isfinite(f)
    return bits[ok].astype(np.uint16), f[ok]


# --------------------------------------------------------------- NF4 table

def test_table_matches_printed_values(oracle):
    # [tqpw] "Method / NormalFloat Quantization (NF4)": the printed list.
    T = oracle.nf4_table()
    np.testing.assert_array_equal(T, _golden_table())


def test_table_invariants(oracle):
    # [tqpw] NF4: normalised to [-1, 1], asymmetric: 7 negative, 0, 8 positive.
    T = oracle.nf4_table()
    assert T.shape == (16,)
    assert np.all(np.diff(T) > 0)
    assert T[0] == -1.0 and T[7] == 0.0 and T[15] == 1.0
    assert np.sum(T < 0) == 7 and np.sum(T > 0) == 8
    # each printed value is exactly an fp32 value
    np.testing.assert_array_equal(T.astype(np.float32).astype(np.float64), T)


def test_table_follows_quantile_construction(oracle):
    # [tqpw] NF4 construction: quantiles of N(0,1) at equally spaced
    # probabilities, 2^(k-1)+1 points on the positive side and 2^(k-1) on the
    # negative side (both including 0), one zero dropped, normalised to [-1,1].
    # The tail offset delta is not printed; fit it and require the fit to
    # reproduce all 16 printed values to fp32 precision.
    from scipy.optimize import minimize_scalar
    from scipy.stats import norm

    T = oracle.nf4_table()

    def build(delta):
        pos = norm.ppf(np.linspace(0.5, 1.0 - delta, 9))  # 9 points incl. 0
        neg = norm.ppf(np.linspace(delta, 0.5, 8))  # 8 points incl. 0
        top = norm.ppf(1.0 - delta)
        v = np.concatenate([neg[:-1], [0.0], pos[1:]]) / top
        return v

    res = minimize_scalar(lambda d: np.max(np.abs(build(d) - T)), bounds=(0.01, 0.06),
                          method="bounded", options={"xatol": 1e-12})
    err = np.max(np.abs(build(res.x) - T))
    assert 0.031 < res.x < 0.034
    assert err < 2e-7, (res.x, err)


# ------------------------------------------------------------------ E4M3

def test_e4m3_decode_all_codes_vs_torch(oracle):
    # The FP8 format of the double-quantised constants ([tqpw] "Double
    # Quantization") is E4M3; torch.float8_e4m3fn is a library decoder.
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    ref = codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    mine = np.array([oracle.e4m3_decode(c) for c in range(256)])
    nan = np.isnan(ref)
    assert np.array_equal(nan, np.isnan(mine))
    np.testing.assert_array_equal(mine[~nan], ref[~nan])
    assert np.sum(nan) == 2  # 0x7f and 0xff


def _e4m3_probe_values():
    mags = sorted({oracle_mag for oracle_mag in
                   [math.ldexp(m, -9) for m in range(8)] +
                   [math.ldexp(1 + m / 8, e - 7) for e in range(1, 16) for m in range(8)
                    if not (e == 15 and m == 7)]})
    vals = set()
    for a, b in zip(mags[:-1], mags[1:]):
        mid = np.float32((a + b) / 2)  # exact in fp32
        for v in (mid, np.nextafter(mid, np.float32(0)), np.nextafter(mid, np.float32(1e9)),
                  np.float32(a), np.float32(b)):
            vals.add(float(v))
    rng = np.random.default_rng(7)
    vals.update(float(v) for v in np.exp(rng.uniform(np.log(2.0 ** -14), np.log(448.0), 4000)).astype(np.float32))
    vals.update(float(v) for v in rng.uniform(0, 448, 2000).astype(np.float32))
    vals.update([0.0, 1e-30, 2.0 ** -10, 448.0, float(np.float32(448.0 * (1 + 2 ** -22)))])
    out = []
    for v in sorted(vals):
        out.extend([v, -v])
    return np.array(out, dtype=np.float32)


def test_e4m3_encode_vs_torch(oracle):
    # Round to nearest even within the finite range; torch's cast is the library
    # reference for every value whose magnitude is at most 448 * (1 + 2^-22),
    # which bounds what the quantiser ever encodes (|d / sigma| <= 448 + rounding).
    v = _e4m3_probe_values()
    ref = torch.from_numpy(v).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    mine = np.array([oracle.e4m3_encode(float(x)) for x in v], dtype=np.uint8)
    bad = np.nonzero(mine != ref)[0]
    assert bad.size == 0, [(float(v[i]), int(mine[i]), int(ref[i])) for i in bad[:10]]


def test_e4m3_saturates(oracle):
    assert oracle.e4m3_encode(470.0) == 0x7E
    assert oracle.e4m3_encode(-1e6) == 0xFE
    assert oracle.e4m3_encode(448.0) == 0x7E


# ------------------------------------------------------------- exact mean

def _round_fraction_to_f32(F: Fraction) -> np.float32:
    """Correctly rounded (nearest, ties to even) fp32 of a non-negative rational."""
    if F == 0:
        return np.float32(0.0)
    c = np.float32(float(F))
    lo = c if Fraction(float(c)) <= F else np.nextafter(c, np.float32(0))
    hi = np.nextafter(lo, np.float32(np.inf))
    flo, fhi = Fraction(float(lo)), Fraction(float(hi))
    assert flo <= F <= fhi
    mid = (flo + fhi) / 2
    if F < mid:
        return lo
    if F > mid:
        return hi
    return lo if (lo.view(np.uint32) & 1) == 0 else hi


@pytest.mark.parametrize("kind", ["normal", "wide", "subnormal", "ties"])
def test_exact_mean_vs_fractions(oracle, kind):
    rng = np.random.default_rng({"normal": 1, "wide": 2, "subnormal": 3, "ties": 4}[kind])
    if kind == "normal":
        c = np.abs(rng.normal(0, 0.05, 5000))
    elif kind == "wide":
        c = np.exp2(rng.uniform(-130, 127, 3000)) * rng.uniform(1, 2, 3000)
    elif kind == "subnormal":
        c = np.exp2(rng.uniform(-133, -110, 2000))
    else:
        # exact halfway cases: (1 + 2^-24)/2 ties to the even 0.5, and
        # (1 + 1.5*2^-23)/2 ties up to the even 0.5 + 2^-23
        c = np.array([1.0, 2.0 ** -24]) if rng.integers(2) else np.array([1.0, 1.5 * 2.0 ** -23])
    bits = torch.from_numpy(np.asarray(c, dtype=np.float32)).to(torch.bfloat16)
    c32 = bits.to(torch.float32).numpy()  # every absmax is a bf16 value
    F = sum((Fraction(float(v)) for v in c32), Fraction(0)) / len(c32)
    assert oracle.exact_mean_f32(c32) == _round_fraction_to_f32(F)


def test_exact_mean_is_order_independent(oracle):
    rng = np.random.default_rng(11)
    c = torch.from_numpy(np.abs(rng.normal(0, 1, 20000)).astype(np.float32)).to(torch.bfloat16).float().numpy()
    m0 = oracle.exact_mean_f32(c)
    for s in range(3):
        assert oracle.exact_mean_f32(np.random.default_rng(s).permutation(c)) == m0


def test_exact_mean_closed_forms(oracle):
    assert oracle.exact_mean_f32(np.array([1.0, 2.0, 3.0], np.float32)) == np.float32(2.0)
    assert oracle.exact_mean_f32(np.array([0.0, 0.0], np.float32)) == np.float32(0.0)
    assert oracle.exact_mean_f32(np.full(1000, 0.375, np.float32)) == np.float32(0.375)
    assert oracle.exact_mean_f32(np.array([1.0, 2.0 ** -24], np.float32)) == np.float32(0.5)
    assert oracle.exact_mean_f32(np.array([1.0, 1.5 * 2.0 ** -23], np.float32)) == np.float32(0.5 + 2.0 ** -23)
    # 1/3 rounded once
    assert oracle.exact_mean_f32(np.array([1.0, 0.0, 0.0], np.float32)) == np.float32(1.0 / 3.0)


# ------------------------------------------------------------ NF4 codes

def test_code_special_cases(oracle):
    # w = +-absmax normalises to exactly +-1 -> codes 15 / 0; w = 0 -> code 7
    # (the value 0); an all-zero block -> code 7.
    for c in (1.0, 0.02, 3.0e-5, 2.0 ** -133, 1.5e38):
        c = float(np.float32(torch.tensor(c).to(torch.bfloat16).float()))
        assert oracle.nf4_code(c, c) == 15
        assert oracle.nf4_code(-c, c) == 0
        assert oracle.nf4_code(0.0, c) == 7
    assert oracle.nf4_code(0.0, 0.0) == 7


@pytest.mark.parametrize("c", [1.0, 0.0234375, 3.0, 1.0e-3])
def test_code_is_nearest_table_value_all_bf16(oracle, c):
    # Brute force over every finite bf16 weight with |w| <= c: the chosen code
    # is a nearest table value to fl32(w / c), and on a tie the lower index.
    c = np.float32(torch.tensor(c).to(torch.bfloat16).float().item())
    _, f = _bf16_all_finite()
    f = f[np.abs(f) <= c]
    T = oracle.nf4_table()
    x = (f / c).astype(np.float32).astype(np.float64)
    codes = np.array([oracle.nf4_code(float(w), float(c)) for w in f])
    err = np.abs(x[:, None] - T[None, :])
    best = err.min(axis=1)
    assert np.all(err[np.arange(len(x)), codes] == best)
    first = np.argmax(err == best[:, None], axis=1)
    assert np.array_equal(codes, first)


def test_quantize_roundtrip_bound_and_packing(oracle):
    # Tiny random blocks: every weight decodes (first level, exact absmax) to
    # within half the widest gap of the table; packing puts even elements in
    # the low nibble ([apxml]: W_NF4 held as 4-bit data).
    rng = np.random.default_rng(5)
    n, k = 3, 128
    w = torch.from_numpy(rng.normal(0, 0.02, (n, k)).astype(np.float32)).to(torch.bfloat16)
    bits = w.view(torch.int16).numpy().view(np.uint16)
    qw = oracle.nf4_quantize(bits, n, k)
    T = oracle.nf4_table()
    wf = w.float().numpy().reshape(-1)
    c = qw["absmax"]
    np.testing.assert_array_equal(c, np.abs(wf).reshape(-1, 64).max(axis=1))
    lo = qw["codes"] & 15
    hi = qw["codes"] >> 4
    codes = np.empty(n * k, dtype=np.int64)
    codes[0::2] = lo
    codes[1::2] = hi
    for e in range(n * k):
        assert codes[e] == oracle.nf4_code(float(wf[e]), float(c[e // 64]))
    half_gap = np.max(np.diff(T)) / 2
    recon = T[codes] * np.repeat(c, 64)
    assert np.all(np.abs(recon - wf) <= half_gap * np.repeat(c, 64) * (1 + 1e-6))


# ------------------------------------------------------ double quantisation

def _dq_case(oracle, n, k, seed, dist="normal"):
    rng = np.random.default_rng(seed)
    if dist == "normal":
        v = rng.normal(0, 0.02, (n, k))
    else:
        v = rng.standard_t(4, (n, k)) * 0.02
    w = torch.from_numpy(v.astype(np.float32)).to(torch.bfloat16)
    bits = w.view(torch.int16).numpy().view(np.uint16)
    return w, oracle.nf4_quantize(bits, n, k)


@pytest.mark.parametrize("n,k", [(4, 4096), (3, 64 * 172), (5, 64 * 7)])
def test_double_quant_invariants(oracle, n, k):
    # [tqpw] "Double Quantization": block constants minus their mean, then
    # symmetric FP8 quantisation per group of 256 with the group absmax mapped
    # to 448. Groups run over the flattened block index and may straddle rows
    # (k = 64 * 172 has 172 blocks per row).
    _, qw = _dq_case(oracle, n, k, seed=n * 1000 + k, dist="t")
    c, q, sigma, mu = qw["absmax"], qw["q"], qw["sigma"], qw["mu"]
    nb = n * k // 64
    assert q.size == nb and sigma.size == (nb + 255) // 256
    F = sum((Fraction(float(v)) for v in c), Fraction(0)) / nb
    assert mu == _round_fraction_to_f32(F)
    dec = np.array([oracle.e4m3_decode(int(b)) for b in q])
    for g in range(sigma.size):
        sl = slice(g * 256, min((g + 1) * 256, nb))
        d = (c[sl] - mu).astype(np.float32)
        S = np.max(np.abs(d))
        assert sigma[g] == np.float32(S / np.float32(448.0))
        if sigma[g] > 0:
            # the block holding the group absmax encodes to +-448
            assert np.max(np.abs(dec[sl])) == 448.0
            # per-block error of the second level
            approx = dec[sl] * np.float64(sigma[g])
            bound = np.where(np.abs(d) / sigma[g] >= 2.0 ** -6, np.abs(d) * 2.0 ** -4, 2.0 ** -10 * sigma[g])
            assert np.all(np.abs(approx - d) <= bound * (1 + 1e-5) + 1e-12 * abs(mu))


def test_block_constant_bound(oracle):
    # c'_b = fma(decode(q_b), sigma_g, mu) reconstructs c_b to within the FP8
    # rounding of d_b plus fp32 rounding.
    _, qw = _dq_case(oracle, 6, 4096, seed=9)
    c, q, sigma, mu = qw["absmax"], qw["q"], qw["sigma"], qw["mu"]
    for b in range(c.size):
        cp = oracle.block_constant(int(q[b]), float(sigma[b // 256]), float(mu))
        d = abs(float(c[b]) - float(mu))
        bound = 2.0 ** -4 * d + 2.0 ** -10 * float(sigma[b // 256]) + 2.0 ** -22 * (abs(float(c[b])) + abs(float(mu)))
        assert abs(float(cp) - float(c[b])) <= bound


def test_all_equal_absmax_is_exact(oracle):
    # Every block has the same absmax: mu = c, d = 0, sigma = 0, q = 0, c' = c.
    n, k = 2, 1024
    w = np.zeros((n, k), np.float32)
    w[:, ::64] = 0.375
    w[:, 5::64] = -0.1
    bits = torch.from_numpy(w).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    qw = oracle.nf4_quantize(bits, n, k)
    assert qw["mu"] == np.float32(0.375)
    assert np.all(qw["sigma"] == 0) and np.all(qw["q"] == 0)
    deq = oracle.nf4_dequant_f64(qw, n, k)
    assert np.all(deq[:, ::64] == 0.375)  # code 15 -> +c exactly
    assert np.all(deq[:, 1::64] == 0.0)  # code 7 -> 0 exactly


def test_dequant_bf16_special_codes(oracle):
    # Code 7 decodes to exactly 0, codes 15 and 0 to exactly +-c'.
    _, qw = _dq_case(oracle, 2, 256, seed=3)
    qw = dict(qw)
    nb = qw["q"].size
    codes = np.zeros(2 * 256 // 2, np.uint8)
    codes[0::2] = 7 | (15 << 4)
    codes[1::2] = 0 | (7 << 4)
    qw["codes"] = codes
    deq = oracle.nf4_dequant_bf16(qw, 2, 256).reshape(-1)
    f = (deq.astype(np.uint32) << 16).view(np.float32)
    cps = np.array([oracle.block_constant(int(qw["q"][b]), float(qw["sigma"][b // 256]), float(qw["mu"]))
                    for b in range(nb)])
    cpb = torch.from_numpy(cps.astype(np.float32)).to(torch.bfloat16).float().numpy()
    e = np.arange(512)
    assert np.all(f[e % 4 == 0] == 0.0)
    assert np.all(f[e % 4 == 1] == cpb[e[e % 4 == 1] // 64])
    assert np.all(f[e % 4 == 2] == -cpb[e[e % 4 == 2] // 64])
    assert np.all(f[e % 4 == 3] == 0.0)


# ------------------------------------------------------------ overhead

def test_overhead_bits_per_param(oracle):
    # [codex] 3.3: double quantisation lowers the constants from 0.5 to 0.127
    # bit per parameter; closed form 8/64 + 32/(64*256).
    vals = {}
    with open(os.path.join(GOLDEN, "overhead.txt")) as f:
        for line in f:
            if line.strip() and not line.startswith("#"):
                key, v = line.split()
                vals[key] = float(v)
    n, k = 4096, 4096
    nb, ng = oracle.num_blocks(n, k), oracle.num_groups(n, k)
    dq_bits = (8 * nb + 32 * ng) / (n * k)
    no_dq_bits = 32 * nb / (n * k)
    assert dq_bits == 8 / 64 + 32 / (64 * 256) == 0.126953125
    assert round(dq_bits, 3) == vals["dq_bits_per_param_rounded"]
    assert no_dq_bits == vals["no_dq_bits_per_param"]


# ------------------------------------------------------------- linear layer

def _bits(t):
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


def _layer(oracle, n, k, m, r, seed, zero_w=False, zero_b=False):
    g = torch.Generator().manual_seed(seed)
    W = (torch.randn(n, k, generator=g) * 0.02)
    if zero_w:
        W.zero_()
    W = W.to(torch.bfloat16)
    A = (torch.randn(r, k, generator=g) * 0.01).to(torch.bfloat16)
    B = (torch.randn(n, r, generator=g) * 0.01).to(torch.bfloat16)
    if zero_b:
        B.zero_()
    x = torch.randn(m, k, generator=g).to(torch.bfloat16)
    gh = torch.randn(m, n, generator=g).to(torch.bfloat16)
    qw = oracle.nf4_quantize(_bits(W), n, k)
    return qw, A, B, x, gh


def test_fwd_zero_lora_b_is_dequant_matmul(oracle):
    # [apxml] h = dequant(W_NF4) x + B A x; with B = 0 only the base remains.
    n, k, m, r = 96, 192, 5, 4
    qw, A, B, x, _ = _layer(oracle, n, k, m, r, 1, zero_b=True)
    h = oracle.qlora_fwd(qw, n, k, _bits(x), m, _bits(A), _bits(B), r, 8.0)
    Wd = oracle.nf4_dequant_f64(qw, n, k)
    ref = x.double().numpy() @ Wd.T
    np.testing.assert_allclose(h, ref, rtol=1e-12, atol=1e-12)


def test_fwd_zero_base_is_scaled_lora(oracle):
    # All-zero W: every block has absmax 0 -> code 7 -> W' = 0, so
    # h = (alpha/r) B (A x), shapes B (d x r), A (r x k) as in [aivaro] 2.
    n, k, m, r = 64, 128, 3, 4
    qw, A, B, x, _ = _layer(oracle, n, k, m, r, 2, zero_w=True)
    h = oracle.qlora_fwd(qw, n, k, _bits(x), m, _bits(A), _bits(B), r, 8.0)
    ref = 2.0 * (x.double().numpy() @ A.double().numpy().T) @ B.double().numpy().T
    np.testing.assert_allclose(h, ref, rtol=1e-12, atol=1e-14)


def test_bwd_zero_lora_b_is_transposed_matmul(oracle):
    # [aivaro] 7: gradients flow through the dequantised, frozen base.
    n, k, m, r = 96, 192, 5, 4
    qw, A, B, _, gh = _layer(oracle, n, k, m, r, 3, zero_b=True)
    gx = oracle.qlora_bwd_x(qw, n, k, _bits(gh), m, _bits(A), _bits(B), r, 8.0)
    Wd = oracle.nf4_dequant_f64(qw, n, k)
    ref = gh.double().numpy() @ Wd
    np.testing.assert_allclose(gx, ref, rtol=1e-12, atol=1e-12)


def test_bwd_zero_base_is_scaled_lora(oracle):
    n, k, m, r = 64, 128, 3, 4
    qw, A, B, _, gh = _layer(oracle, n, k, m, r, 4, zero_w=True)
    gx = oracle.qlora_bwd_x(qw, n, k, _bits(gh), m, _bits(A), _bits(B), r, 8.0)
    ref = 2.0 * (gh.double().numpy() @ B.double().numpy()) @ A.double().numpy()
    np.testing.assert_allclose(gx, ref, rtol=1e-12, atol=1e-14)


@pytest.mark.parametrize("alpha,r", [(8.0, 4), (32.0, 16), (16.0, 64)])
def test_adjoint_identity(oracle, alpha, r):
    # bwd_x is the adjoint of fwd in x: <g, fwd(x)> = <bwd_x(g), x> (exactly,
    # up to fp64 summation), for any W, A, B and scale.
    n, k, m = 80, 256, 4
    qw, A, B, x, gh = _layer(oracle, n, k, m, r, 10 + r)
    h = oracle.qlora_fwd(qw, n, k, _bits(x), m, _bits(A), _bits(B), r, alpha)
    gx = oracle.qlora_bwd_x(qw, n, k, _bits(gh), m, _bits(A), _bits(B), r, alpha)
    lhs = np.sum(gh.double().numpy() * h)
    rhs = np.sum(gx * x.double().numpy())
    assert abs(lhs - rhs) <= 1e-11 * (abs(lhs) + np.sqrt(np.sum(h * h)))


def test_row_selection_consistency(oracle):
    n, k, m, r = 64, 128, 9, 4
    qw, A, B, x, gh = _layer(oracle, n, k, m, r, 21)
    full = oracle.qlora_fwd(qw, n, k, _bits(x), m, _bits(A), _bits(B), r, 8.0)
    part = oracle.qlora_fwd(qw, n, k, _bits(x), m, _bits(A), _bits(B), r, 8.0, rows=[8, 0, 3])
    np.testing.assert_array_equal(part, full[[8, 0, 3]])
    fullb = oracle.qlora_bwd_x(qw, n, k, _bits(gh), m, _bits(A), _bits(B), r, 8.0)
    partb = oracle.qlora_bwd_x(qw, n, k, _bits(gh), m, _bits(A), _bits(B), r, 8.0, rows=[7, 1])
    np.testing.assert_array_equal(partb, fullb[[7, 1]])


def test_lora_scale_is_alpha_over_r(oracle):
    # lora_alpha is the scaling factor of the adapter branch: the branch is
    # linear in alpha and vanishes at alpha = 0.
    n, k, m, r = 64, 128, 2, 16
    qw, A, B, x, _ = _layer(oracle, n, k, m, r, 31)
    h0 = oracle.qlora_fwd(qw, n, k, _bits(x), m, _bits(A), _bits(B), r, 0.0)
    h1 = oracle.qlora_fwd(qw, n, k, _bits(x), m, _bits(A), _bits(B), r, 32.0)
    h2 = oracle.qlora_fwd(qw, n, k, _bits(x), m, _bits(A), _bits(B), r, 64.0)
    np.testing.assert_allclose(h2 - h0, 2 * (h1 - h0), rtol=1e-9, atol=1e-13)
    base = oracle.qlora_fwd(qw, n, k, _bits(x), m, None, None, 0, 0.0)
    np.testing.assert_array_equal(h0, base)


def test_code_ties_go_to_lower_index(oracle):
    # Pages are silent on ties; the reading is "lower index". A midpoint between
    # neighbouring table values that is itself an fp32 value (the midpoint
    # T[7..8] is T[8]/2, always exact) is an exact tie.
    T = oracle.nf4_table()
    n_ties = 0
    for i in range(15):
        m = (T[i] + T[i + 1]) / 2  # exact in fp64
        m32 = np.float32(m)
        if float(m32) != m:
            continue
        n_ties += 1
        assert oracle.nf4_code(float(m32), 1.0) == i
        assert oracle.nf4_code(float(np.nextafter(m32, np.float32(2))), 1.0) == i + 1
        assert oracle.nf4_code(float(np.nextafter(m32, np.float32(-2))), 1.0) == i
    assert n_ties >= 1


def test_block_constant_is_single_rounded_fma(oracle):
    # c' = dec(q) * sigma + mu computed exactly and rounded once to fp32.
    rng = np.random.default_rng(17)
    for _ in range(3000):
        qb = int(rng.integers(0, 256))
        if qb in (0x7F, 0xFF):
            continue
        sg = np.float32(rng.uniform(1e-6, 1e-3))
        mu = np.float32(rng.uniform(0.0, 0.2))
        F = Fraction(oracle.e4m3_decode(qb)) * Fraction(float(sg)) + Fraction(float(mu))
        want = _round_fraction_to_f32(abs(F))
        want = -want if F < 0 else want
        assert oracle.block_constant(qb, float(sg), float(mu)) == want


@pytest.mark.parametrize("n,k", [(3, 64 * 172), (9, 4096)])
def test_dequant_reconstructs_weights(oracle, n, k):
    # Two-level reconstruction bound, element by element, against the original
    # weights: first level within half the widest table gap of c_b, second
    # level within the FP8 rounding of d_b (groups straddle rows at k=64*172).
    w, qw = _dq_case(oracle, n, k, seed=77 + n, dist="t")
    wf = w.float().numpy().astype(np.float64).reshape(-1)
    T = oracle.nf4_table()
    c = qw["absmax"].astype(np.float64)
    mu = float(qw["mu"])
    sig = np.repeat(qw["sigma"].astype(np.float64), 256)[: c.size]
    half_gap = np.max(np.diff(T)) / 2
    dq_err = 2.0 ** -4 * np.abs(c - mu) + 2.0 ** -10 * sig + 2.0 ** -22 * (c + abs(mu))
    bound = np.repeat(half_gap * c + dq_err, 64) * (1 + 1e-6)
    d64 = oracle.nf4_dequant_f64(qw, n, k).reshape(-1)
    assert np.all(np.abs(d64 - wf) <= bound)
    d16 = oracle.nf4_dequant_bf16(qw, n, k).reshape(-1)
    f16 = (d16.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    assert np.all(np.abs(f16 - wf) <= bound + np.abs(d64) * 2.0 ** -8)


# ------------------------------------------------------ adapter weight gradients
# [aivaro] 2 and 7: W is frozen, only B and A are trained; their gradients are the
# derivatives of h = W'x + s B (A x). The pins below compare or_lora_grads with the
# forward oracle (h is linear in B and in A), with numpy on tiny shapes, and with the
# per-token decomposition.

def _grads(oracle, n, k, m, r, alpha, seed):
    qw, A, B, x, gh = _layer(oracle, n, k, m, r, seed)
    gA, gB = oracle.lora_grads(_bits(x), _bits(gh), m, n, k, _bits(A), _bits(B), r, alpha)
    return qw, A, B, x, gh, gA, gB


@pytest.mark.parametrize("alpha,r", [(8.0, 4), (32.0, 16), (16.0, 64)])
def test_grad_B_is_adjoint_of_forward_in_B(oracle, alpha, r):
    n, k, m = 48, 192, 5
    qw, A, B, x, gh, gA, gB = _grads(oracle, n, k, m, r, alpha, 70 + r)
    B2 = (torch.randn(n, r, generator=torch.Generator().manual_seed(5 + r)) * 0.01).to(torch.bfloat16)
    h1 = oracle.qlora_fwd(qw, n, k, _bits(x), m, _bits(A), _bits(B), r, alpha)
    h2 = oracle.qlora_fwd(qw, n, k, _bits(x), m, _bits(A), _bits(B2), r, alpha)
    lhs = np.sum(gh.double().numpy() * (h2 - h1))
    rhs = np.sum(gB * (B2.double().numpy() - B.double().numpy()))
    assert abs(lhs - rhs) <= 1e-10 * (abs(lhs) + 1e-300) + 1e-13


@pytest.mark.parametrize("alpha,r", [(8.0, 4), (32.0, 16), (16.0, 64)])
def test_grad_A_is_adjoint_of_forward_in_A(oracle, alpha, r):
    n, k, m = 48, 192, 5
    qw, A, B, x, gh, gA, gB = _grads(oracle, n, k, m, r, alpha, 80 + r)
    A2 = (torch.randn(r, k, generator=torch.Generator().manual_seed(9 + r)) * 0.01).to(torch.bfloat16)
    h1 = oracle.qlora_fwd(qw, n, k, _bits(x), m, _bits(A), _bits(B), r, alpha)
    h2 = oracle.qlora_fwd(qw, n, k, _bits(x), m, _bits(A2), _bits(B), r, alpha)
    lhs = np.sum(gh.double().numpy() * (h2 - h1))
    rhs = np.sum(gA * (A2.double().numpy() - A.double().numpy()))
    assert abs(lhs - rhs) <= 1e-10 * (abs(lhs) + 1e-300) + 1e-13


def test_lora_grads_match_numpy_on_tiny_shapes(oracle):
    n, k, m, r, alpha = 16, 64, 3, 4, 8.0
    qw, A, B, x, gh, gA, gB = _grads(oracle, n, k, m, r, alpha, 91)
    s = alpha / r
    xd, gd, Ad, Bd = (t.double().numpy() for t in (x, gh, A, B))
    np.testing.assert_allclose(gB, s * gd.T @ (xd @ Ad.T), rtol=1e-12, atol=1e-15)
    np.testing.assert_allclose(gA, s * (gd @ Bd).T @ xd, rtol=1e-12, atol=1e-15)


def test_lora_grads_sum_over_tokens(oracle):
    # the gradients of a batch are the sums of the per-token gradients
    n, k, m, r, alpha = 32, 128, 4, 8, 16.0
    qw, A, B, x, gh, gA, gB = _grads(oracle, n, k, m, r, alpha, 92)
    sA, sB = np.zeros_like(gA), np.zeros_like(gB)
    for i in range(m):
        a1, b1 = oracle.lora_grads(_bits(x[i:i + 1]), _bits(gh[i:i + 1]), 1, n, k, _bits(A), _bits(B), r, alpha)
        sA += a1
        sB += b1
    np.testing.assert_allclose(gA, sA, rtol=1e-12, atol=1e-15)
    np.testing.assert_allclose(gB, sB, rtol=1e-12, atol=1e-15)


# ------------------------------------------------------------------------- merge
# [codex] 3.6 merge_and_unload: the adapter is folded into a 16-bit weight W' + s B A
# ([tqpw] Introduction: it cannot stay NF4).

def test_f64_to_bf16_is_nearest_even(oracle):
    rng = np.random.default_rng(7)
    vals = np.concatenate([rng.standard_normal(3000) * 10.0 ** rng.integers(-40, 38, 3000),
                           np.ldexp(1.0 + np.arange(1, 256) / 256.0 + 2.0 ** -9, 0),  # exact ties
                           [2.0 ** -133, 2.0 ** -134, 3.0 * 2.0 ** -134, 1e-45, 3.39e38, -0.0, 0.0]])
    for v in vals:
        b = oracle.f64_to_bf16(float(v))
        got = float(np.array([b << 16], dtype=np.uint32).view(np.float32)[0])
        # brute force: the two bf16 neighbours of v (truncation and the next one up in magnitude)
        t32 = np.array([v], dtype=np.float64)
        lo_bits = int(np.float32(v).view(np.uint32)) >> 16 if np.isfinite(np.float32(v)) else None
        if lo_bits is None:
            continue
        cands = set()
        for d in (-1, 0, 1):
            c = (lo_bits + d) & 0xffff
            f = float(np.array([c << 16], dtype=np.uint32).view(np.float32)[0])
            if np.isfinite(f) and (f == 0 or np.sign(f) == np.sign(v) or v == 0):
                cands.add((abs(f - v), c & 1, c, f))
        best = min(cands)
        ties = [c for c in cands if c[0] == best[0]]
        want = min(ties, key=lambda c: c[1])[3] if len(ties) > 1 else best[3]
        assert got == want or (got == 0 and want == 0), (v, got, want)
        del t32


def test_f64_to_bf16_matches_torch_on_fp32_values(oracle):
    # for values exact in fp32 the one-step rounding equals torch's fp32 -> bf16 rounding
    x = torch.randn(4000, dtype=torch.float32) * 3.0
    want = x.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    got = np.array([oracle.f64_to_bf16(float(v)) for v in x.numpy()], dtype=np.uint16)
    assert np.array_equal(got, want)


def test_merge_without_adapter_is_the_dequantised_weight(oracle):
    n, k, m, r = 24, 192, 1, 4
    qw, A, B, x, _ = _layer(oracle, n, k, m, r, 93, zero_b=True)
    merged = oracle.merge_bf16(qw, n, k, _bits(A), _bits(B), r, 8.0)
    assert np.array_equal(merged, oracle.nf4_dequant_bf16(qw, n, k))
    assert np.array_equal(oracle.merge_bf16(qw, n, k, None, None, 0, 0.0), oracle.nf4_dequant_bf16(qw, n, k))


def test_merge_of_zero_base_is_rounded_scaled_product(oracle):
    n, k, m, r, alpha = 20, 128, 1, 8, 16.0
    qw, A, B, x, _ = _layer(oracle, n, k, m, r, 94, zero_w=True)
    merged = oracle.merge_bf16(qw, n, k, _bits(A), _bits(B), r, alpha)
    prod = (alpha / r) * (B.double().numpy() @ A.double().numpy())
    # r products of bf16 values sum exactly in fp64 here, so numpy's order cannot change them
    want = np.array([oracle.f64_to_bf16(float(v)) for v in prod.reshape(-1)], dtype=np.uint16).reshape(n, k)
    assert np.array_equal(merged, want)


def test_merged_weight_reproduces_the_forward_pass(oracle):
    # x W_merged^T agrees with the oracle forward within the bf16 rounding of the merged weight
    n, k, m, r, alpha = 40, 256, 3, 16, 32.0
    qw, A, B, x, _ = _layer(oracle, n, k, m, r, 95)
    merged = oracle.merge_bf16(qw, n, k, _bits(A), _bits(B), r, alpha)
    Wm = (merged.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    h = oracle.qlora_fwd(qw, n, k, _bits(x), m, _bits(A), _bits(B), r, alpha)
    hm = x.double().numpy() @ Wm.T
    bound = 2.0 ** -8 * (np.abs(x.double().numpy()) @ np.abs(Wm).T) + 1e-12
    assert np.all(np.abs(h - hm) <= bound)


def test_f64_to_bf16_overflow_threshold(oracle):
    # IEEE round to nearest: magnitudes from max_finite + half an ulp up overflow to infinity
    mx = (2.0 - 2.0 ** -7) * 2.0 ** 127
    half = 2.0 ** 119
    assert oracle.f64_to_bf16(mx) == 0x7f7f
    assert oracle.f64_to_bf16(mx + half * 0.999) == 0x7f7f
    assert oracle.f64_to_bf16(mx + half) == 0x7f80  # tie: the even neighbour is 2^128 -> inf
    assert oracle.f64_to_bf16(-(mx + 2 * half)) == 0xff80


# ---------------------------------------------------------------- LoRA dropout
# [codex] 3.4 and the lora_dropout setting in [aivaro]'s configuration: dropout on the adapter's
# input. Reading (the pages give only the rate): inverted dropout of x on the adapter branch only,
# element kept when the Philox4x32-10 output is >= floor(p 2^32), kept elements scaled 1 / (1 - p).
# Pins: the generator's published known-answer vectors; the threshold's closed form; the keep rate
# within a binomial bound; the counter/offset layout; p = 0 reducing to the plain layer exactly;
# the masked input gradient being the adjoint of the masked forward; the mean over seeds of the
# masked adapter term converging to the unmasked one; the gradients' adjointness with dropout.

def _kat():
    rows = []
    with open(os.path.join(GOLDEN, "philox4x32_10_kat.txt")) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                w = [int(v, 16) for v in line.split()]
                rows.append((w[0:4], w[4:6], w[6:10]))
    return rows


def test_philox_known_answers(oracle):
    for ctr, key, want in _kat():
        assert [int(v) for v in oracle.philox4x32_10(ctr, key)] == want


def test_dropout_threshold_closed_form(oracle):
    assert oracle.dropout_threshold(0.0) == 0
    assert oracle.dropout_threshold(0.5) == 2 ** 31
    assert oracle.dropout_threshold(0.25) == 2 ** 30
    assert oracle.dropout_threshold(0.05) == math.floor(0.05 * 2 ** 32)
    assert oracle.dropout_threshold(0.1) == math.floor(0.1 * 2 ** 32)


def test_dropout_bits_counter_layout(oracle):
    # element e draws word e % 4 of the block e // 4; the seed is the key (low, high word)
    seed = 0x0123456789ABCDEF
    for e in (0, 1, 2, 3, 4, 7, 1 << 33, (1 << 34) + 3):
        blk = e >> 2
        words = oracle.philox4x32_10([blk & 0xFFFFFFFF, blk >> 32, 0, 0], [seed & 0xFFFFFFFF, seed >> 32])
        assert oracle.dropout_bits(seed, e) == int(words[e & 3])


def test_dropout_keep_rate_and_offset(oracle):
    p, m, k = 0.1, 40, 1024
    keep = oracle.dropout_keep(1234, 0, p, m, k)
    n = keep.size
    rate = keep.mean()
    sd = math.sqrt(p * (1 - p) / n)
    assert abs(rate - (1 - p)) < 5 * sd
    # the offset shifts the element index: element (0, j) at offset d is element (0, j + d) at 0
    k2 = oracle.dropout_keep(1234, 5, p, 1, k - 5)
    assert np.array_equal(k2[0], keep[0, 5:])
    # another seed gives another mask
    assert not np.array_equal(oracle.dropout_keep(1235, 0, p, m, k), keep)


def test_dropout_zero_rate_is_the_plain_layer(oracle):
    n, k, m, r, alpha = 48, 192, 5, 8, 16.0
    qw, A, B, x, gh = _layer(oracle, n, k, m, r, 123)
    for fn, inp in ((oracle.qlora_fwd, x), (oracle.qlora_bwd_x, gh)):
        a = fn(qw, n, k, _bits(inp), m, _bits(A), _bits(B), r, alpha)
        b = fn(qw, n, k, _bits(inp), m, _bits(A), _bits(B), r, alpha, p_drop=0.0, seed=77, offset=9)
        assert np.array_equal(a, b)
    ga = oracle.lora_grads(_bits(x), _bits(gh), m, n, k, _bits(A), _bits(B), r, alpha)
    gb = oracle.lora_grads(_bits(x), _bits(gh), m, n, k, _bits(A), _bits(B), r, alpha, 0.0, 77, 9)
    assert np.array_equal(ga[0], gb[0]) and np.array_equal(ga[1], gb[1])


@pytest.mark.parametrize("p", [0.05, 0.3])
def test_dropout_adjoint_identity(oracle, p):
    # with one mask, the layer is linear in x and the input gradient is its adjoint
    n, k, m, r, alpha = 64, 256, 4, 16, 32.0
    qw, A, B, x, gh = _layer(oracle, n, k, m, r, 140)
    h = oracle.qlora_fwd(qw, n, k, _bits(x), m, _bits(A), _bits(B), r, alpha, p_drop=p, seed=9, offset=100)
    gx = oracle.qlora_bwd_x(qw, n, k, _bits(gh), m, _bits(A), _bits(B), r, alpha, p_drop=p, seed=9, offset=100)
    lhs = np.sum(gh.double().numpy() * h)
    rhs = np.sum(gx * x.double().numpy())
    assert abs(lhs - rhs) <= 1e-11 * (abs(lhs) + np.sqrt(np.sum(h * h)))
    # and the mask matters: without it the adapter part differs
    h0 = oracle.qlora_fwd(qw, n, k, _bits(x), m, _bits(A), _bits(B), r, alpha)
    assert not np.allclose(h, h0)


def test_dropout_adapter_term_is_the_masked_product(oracle):
    # zero base: h = s / (1 - p) B A (keep * x), keep from the generator (brute force, tiny shape)
    n, k, m, r, alpha, p = 16, 64, 3, 4, 8.0, 0.25
    zero, A, B, x, gh = _layer(oracle, n, k, m, r, 150, zero_w=True)
    keep = oracle.dropout_keep(31, 7, p, m, k)
    h = oracle.qlora_fwd(zero, n, k, _bits(x), m, _bits(A), _bits(B), r, alpha, p_drop=p, seed=31, offset=7)
    xd = x.double().numpy() * keep
    ref = (alpha / r) / (1 - p) * (xd @ A.double().numpy().T) @ B.double().numpy().T
    np.testing.assert_allclose(h, ref, rtol=1e-12, atol=1e-15)


def test_dropout_mean_over_seeds_is_the_plain_adapter(oracle):
    # inverted dropout is unbiased: the mean of the masked adapter term over independent masks
    # tends to the unmasked term (zero base isolates the adapter)
    n, k, m, r, alpha, p = 8, 64, 2, 4, 8.0, 0.3
    zero, A, B, x, gh = _layer(oracle, n, k, m, r, 160, zero_w=True)
    plain = oracle.qlora_fwd(zero, n, k, _bits(x), m, _bits(A), _bits(B), r, alpha)
    runs = np.stack([oracle.qlora_fwd(zero, n, k, _bits(x), m, _bits(A), _bits(B), r, alpha, p_drop=p, seed=s)
                     for s in range(400)])
    mean, sem = runs.mean(axis=0), runs.std(axis=0) / math.sqrt(runs.shape[0])
    assert np.all(np.abs(mean - plain) <= 5 * sem + 1e-12)


def test_dropout_grads_are_adjoint_of_forward(oracle):
    n, k, m, r, alpha, p = 48, 192, 5, 16, 32.0, 0.1
    qw, A, B, x, gh = _layer(oracle, n, k, m, r, 170)
    gA, gB = oracle.lora_grads(_bits(x), _bits(gh), m, n, k, _bits(A), _bits(B), r, alpha, p, 5, 11)
    B2 = (torch.randn(n, r, generator=torch.Generator().manual_seed(171)) * 0.01).to(torch.bfloat16)
    A2 = (torch.randn(r, k, generator=torch.Generator().manual_seed(172)) * 0.01).to(torch.bfloat16)
    fwd = lambda AA, BB: oracle.qlora_fwd(qw, n, k, _bits(x), m, _bits(AA), _bits(BB), r, alpha, p_drop=p, seed=5,
                                          offset=11)
    h1 = fwd(A, B)
    g = gh.double().numpy()
    lhs = np.sum(g * (fwd(A, B2) - h1))
    rhs = np.sum(gB * (B2.double().numpy() - B.double().numpy()))
    assert abs(lhs - rhs) <= 1e-10 * (abs(lhs) + 1e-300) + 1e-13
    lhs = np.sum(g * (fwd(A2, B) - h1))
    rhs = np.sum(gA * (A2.double().numpy() - A.double().numpy()))
    assert abs(lhs - rhs) <= 1e-10 * (abs(lhs) + 1e-300) + 1e-13


# ------------------------------------------- the 4-bit float and fp32 constants
# [apxml] (the four configuration knobs) and [aivaro] 6 (bnb_4bit_quant_type,
# bnb_4bit_use_double_quant): the quant type is NF4 or the standard 4-bit float, and
# double quantisation can be off; [tqpw] Experiments compares NF4 with FP4; [codex] 3.3
# gives the 0.5 bit per parameter of fp32 constants. The reading of "4-bit float": E2M1
# (sign, two exponent bits with bias 1, one mantissa bit), normalised by its largest
# magnitude 6 onto [-1, 1]. The pins derive the values from the bit fields here.

def _e2m1(code):
    s, e, m = code >> 3, (code >> 1) & 3, code & 1
    mag = m * 0.5 if e == 0 else 2.0 ** (e - 1) * (1.0 + m / 2.0)
    return -mag if s else mag


def test_fp4_table_from_e2m1_bit_fields(oracle):
    T = oracle.table("fp4")
    want = np.array([np.float32(_e2m1(c) / 6.0) for c in range(16)], dtype=np.float64)
    np.testing.assert_array_equal(T, want)
    assert sorted({abs(_e2m1(c)) for c in range(16)}) == [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]


def test_fp4_table_invariants(oracle):
    T = oracle.table("fp4")
    assert T[7] == 1.0 and T[15] == -1.0 and T[0] == 0.0 and T[8] == 0.0
    np.testing.assert_array_equal(T[8:], -T[:8])
    assert len(set(T.tolist())) == 15  # +0 and -0 are one value
    assert np.all(np.diff(T[:8]) > 0)
    np.testing.assert_array_equal(oracle.table("nf4"), oracle.nf4_table())


def test_fp4_code_special_cases(oracle):
    for c in (1.0, 0.02, 3.0e-5, 1.5e38):
        c = float(np.float32(torch.tensor(c).to(torch.bfloat16).float()))
        assert oracle.code4("fp4", c, c) == 7
        assert oracle.code4("fp4", -c, c) == 15
        assert oracle.code4("fp4", 0.0, c) == 0
        assert oracle.code4("fp4", -c * 2.0 ** -10, c) == 0  # rounds to zero: +0, never -0
    assert oracle.code4("fp4", 0.0, 0.0) == 0
    assert oracle.code4("nf4", 0.0, 0.0) == 7


@pytest.mark.parametrize("c", [1.0, 0.0234375, 3.0])
def test_fp4_code_is_nearest_table_value_all_bf16(oracle, c):
    # Brute force over every finite bf16 weight with |w| <= c against the values derived
    # from the bit fields: a nearest value, the lowest such code on a tie, never -0.
    c = np.float32(torch.tensor(c).to(torch.bfloat16).float().item())
    _, f = _bf16_all_finite()
    f = f[np.abs(f) <= c]
    T = np.array([np.float32(_e2m1(k) / 6.0) for k in range(16)], dtype=np.float64)
    x = (f / c).astype(np.float32).astype(np.float64)
    codes = np.array([oracle.code4("fp4", float(w), float(c)) for w in f])
    err = np.abs(x[:, None] - T[None, :])
    best = err.min(axis=1)
    assert np.all(err[np.arange(len(x)), codes] == best)
    assert np.array_equal(codes, np.argmax(err == best[:, None], axis=1))
    assert not np.any(codes == 8)


def test_fp4_ties_go_toward_zero(oracle):
    # Every midpoint of neighbouring values that an fp32 x can equal exactly: the code
    # of the smaller magnitude (the lower code index on both sides of zero).
    T = oracle.table("fp4")
    mags = T[:8]
    hits = 0
    for i in range(7):
        m = (mags[i] + mags[i + 1]) / 2.0
        if float(np.float32(m)) != m:
            continue
        hits += 1
        assert oracle.code4("fp4", float(m), 1.0) == i
        assert oracle.code4("fp4", -float(m), 1.0) == (i + 8 if i > 0 else 0)
    assert hits >= 1


def test_fp4_roundtrip_bound(oracle):
    # Every weight decodes (exact absmax) within half the widest gap, (1 - 2/3) / 2.
    rng = np.random.default_rng(11)
    n, k = 4, 256
    w = torch.from_numpy(rng.standard_t(4, (n, k)).astype(np.float32) * 0.02).to(torch.bfloat16)
    qw = oracle.quantize4(_bits(w), n, k, "fp4", False)
    wf = w.float().numpy().astype(np.float64).reshape(-1)
    c = np.abs(wf).reshape(-1, 64).max(axis=1)
    np.testing.assert_array_equal(qw["absmax"].astype(np.float64), c)
    codes = np.empty(n * k, dtype=np.int64)
    codes[0::2] = qw["codes"] & 15
    codes[1::2] = qw["codes"] >> 4
    T = np.array([np.float32(_e2m1(j) / 6.0) for j in range(16)], dtype=np.float64)
    recon = T[codes] * np.repeat(c, 64)
    assert np.all(np.abs(recon - wf) <= (1.0 / 6.0) * np.repeat(c, 64) * (1 + 1e-6))


@pytest.mark.parametrize("qtype", ["nf4", "fp4"])
def test_codes_do_not_depend_on_double_quant(oracle, qtype):
    # Codes are chosen against the exact block absmax; double quantisation only changes
    # how the constants are stored.
    rng = np.random.default_rng(3)
    n, k = 5, 64 * 9
    w = torch.from_numpy(rng.normal(0, 0.02, (n, k)).astype(np.float32)).to(torch.bfloat16)
    a = oracle.quantize4(_bits(w), n, k, qtype, True)
    b = oracle.quantize4(_bits(w), n, k, qtype, False)
    np.testing.assert_array_equal(a["codes"], b["codes"])
    np.testing.assert_array_equal(a["absmax"], b["absmax"])
    assert "q" not in b and "sigma" not in b


@pytest.mark.parametrize("qtype", ["nf4", "fp4"])
def test_fp32_constants_dequant_is_table_times_absmax(oracle, qtype):
    # Without double quantisation the dequantised weight is T[code] * c_b with c_b the
    # numpy block absmax; the bf16 form is its round-to-nearest-even (torch).
    rng = np.random.default_rng(8)
    n, k = 3, 64 * 5
    w = torch.from_numpy(rng.normal(0, 0.02, (n, k)).astype(np.float32)).to(torch.bfloat16)
    qw = oracle.quantize4(_bits(w), n, k, qtype, False)
    c = np.abs(w.float().numpy()).reshape(-1, 64).max(axis=1).astype(np.float64)
    codes = np.empty(n * k, dtype=np.int64)
    codes[0::2] = qw["codes"] & 15
    codes[1::2] = qw["codes"] >> 4
    T = oracle.table(qtype)
    want = T[codes] * np.repeat(c, 64)
    np.testing.assert_array_equal(oracle.nf4_dequant_f64(qw, n, k).reshape(-1), want)
    want16 = torch.from_numpy((T[codes].astype(np.float32) * np.repeat(c.astype(np.float32), 64))).to(torch.bfloat16)
    np.testing.assert_array_equal(oracle.nf4_dequant_bf16(qw, n, k).reshape(-1), _bits(want16))


@pytest.mark.parametrize("qtype,dq", [("fp4", True), ("fp4", False), ("nf4", False)])
def test_formats_layer_is_dequant_matmul_plus_adapter(oracle, qtype, dq):
    # The layer with another format is the same contraction: numpy over the independently
    # dequantised weight (fp32 constants) or the oracle's dequantisation (double quant),
    # plus s B (A x); and the adjoint identity between forward and input gradient.
    n, k, m, r, alpha = 24, 64 * 3, 3, 4, 8.0
    g = torch.Generator().manual_seed(21)
    W = (torch.randn(n, k, generator=g) * 0.02).to(torch.bfloat16)
    A = (torch.randn(r, k, generator=g) * 0.01).to(torch.bfloat16)
    B = (torch.randn(n, r, generator=g) * 0.01).to(torch.bfloat16)
    x = torch.randn(m, k, generator=g).to(torch.bfloat16)
    gh = torch.randn(m, n, generator=g).to(torch.bfloat16)
    qw = oracle.quantize4(_bits(W), n, k, qtype, dq)
    if dq:
        Wd = oracle.nf4_dequant_f64(qw, n, k)
    else:
        codes = np.empty(n * k, dtype=np.int64)
        codes[0::2] = qw["codes"] & 15
        codes[1::2] = qw["codes"] >> 4
        c = np.abs(W.float().numpy()).reshape(-1, 64).max(axis=1).astype(np.float64)
        Wd = (oracle.table(qtype)[codes] * np.repeat(c, 64)).reshape(n, k)
    xf, Af, Bf, gf = (t.double().numpy() for t in (x, A, B, gh))
    s = float(np.float32(alpha / r))
    h = oracle.qlora_fwd(qw, n, k, _bits(x), m, _bits(A), _bits(B), r, alpha)
    np.testing.assert_allclose(h, xf @ Wd.T + s * (xf @ Af.T) @ Bf.T, rtol=1e-12, atol=1e-12)
    gx = oracle.qlora_bwd_x(qw, n, k, _bits(gh), m, _bits(A), _bits(B), r, alpha)
    np.testing.assert_allclose(gx, gf @ Wd + s * (gf @ Bf) @ Af, rtol=1e-12, atol=1e-12)
    assert abs(np.sum(gf * h) - np.sum(gx * xf)) <= 1e-10 * (np.abs(gf * h).sum() + 1.0)
