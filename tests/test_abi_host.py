"""Host-side checks of the C ABI: the library loads without a GPU, exports every
function declared in include/*.h, answers size queries, and rejects bad arguments
before anything is enqueued (no call here reaches the GPU)."""
import ctypes
import glob
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
GOLDEN = os.path.join(ROOT, "tests", "golden")


@pytest.fixture(scope="module")
def lib():
    from bit_nf4_quantized_25_b200 import binding, build
    build.build()
    return binding.load()


def _declared_functions():
    names = set()
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        src = open(h).read()
        src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
        for m in re.finditer(r"^\s*(?:const\s+)?[A-Za-z_][A-Za-z0-9_]*\s*\*?\s*([A-Za-z_][A-Za-z0-9_]*)\s*\(",
                             src, flags=re.M):
            names.add(m.group(1))
    return sorted(names)


def test_header_declares_the_boundary():
    names = _declared_functions()
    for f in ("nf4_quantize", "qlora_linear_fwd", "qlora_linear_bwd_x", "nf4_dequantize"):
        assert f in names


def test_library_exports_every_declared_function(lib):
    for name in _declared_functions():
        assert hasattr(lib, name), name


def _sizes(lib, n, k):
    a, b, c, d = (ctypes.c_size_t() for _ in range(4))
    st = lib.qn_nf4_sizes(n, k, ctypes.byref(a), ctypes.byref(b), ctypes.byref(c), ctypes.byref(d))
    return st, (a.value, b.value, c.value, d.value)


def test_sizes_give_the_double_quant_overhead(lib):
    # "QLoRA & PEFT family" (ai-reference-codex) 3.3: 0.5 -> 0.127 bit per parameter.
    st, (cb, ab, sb, mb) = _sizes(lib, 4096, 4096)
    assert st == 0
    n = 4096 * 4096
    assert cb == n // 2 and ab == n // 64 and sb == 4 * (n // 64 // 256) and mb == 4
    assert (8 * ab + 8 * sb) / n == 0.126953125
    assert round((8 * ab + 8 * sb) / n, 3) == 0.127


def test_7b_stack_is_about_3p5_gb(lib):
    # "QLoRA & PEFT family" 3.1: a 7B base goes from 14 GB to about 3.5 GB in 4 bits.
    shapes = [(4096, 4096)] * 4 + [(11008, 4096)] * 2 + [(4096, 11008)]
    total = 0
    for n, k in shapes:
        st, s = _sizes(lib, n, k)
        assert st == 0
        total += sum(s)
    total *= 32
    assert 3.2e9 < total < 3.5e9


def test_size_errors(lib):
    st, _ = _sizes(lib, 4096, 100)
    assert st == 2  # QN_ESHAPE
    st, _ = _sizes(lib, -1, 64)
    assert st == 1  # QN_EINVAL


def _weight(n=128, k=128, base=0x100000):
    from bit_nf4_quantized_25_b200.binding import CWeight
    return CWeight(n, k, base, base + 0x10000, base + 0x20000, base + 0x30000)


def test_linear_argument_errors_before_launch(lib):
    from bit_nf4_quantized_25_b200.binding import QN_EALIGN, QN_EINVAL, QN_ESHAPE, QN_EWORKSPACE
    w = _weight()
    P = ctypes.c_void_p
    x, h, A, B, ws = P(0x200000), P(0x300000), P(0x400000), P(0x500000), P(0x600000)
    f = lib.qlora_linear_fwd
    assert f(ctypes.byref(w), x, 4, A, B, 300, 1.0, h, ws, 1 << 20, None) == QN_EINVAL  # r > 256
    assert f(ctypes.byref(w), x, 4, A, None, 4, 1.0, h, ws, 1 << 20, None) == QN_EINVAL  # null B
    assert f(ctypes.byref(w), x, 4, A, B, 0, 1.0, h, ws, 1 << 20, None) == QN_EINVAL  # r=0 with A, B
    assert f(ctypes.byref(w), P(0x200008), 4, A, B, 4, 1.0, h, ws, 1 << 20, None) == QN_EALIGN
    assert f(ctypes.byref(w), x, 4, A, B, 4, 1.0, x, ws, 1 << 20, None) == QN_EINVAL  # aliasing
    assert f(ctypes.byref(w), x, 4, A, B, 4, 1.0, h, None, 0, None) == QN_EWORKSPACE
    assert f(ctypes.byref(w), x, -1, A, B, 4, 1.0, h, ws, 1 << 20, None) == QN_EINVAL
    assert f(ctypes.byref(w), x, 4, A, B, 4, float("nan"), h, ws, 1 << 20, None) == QN_EINVAL
    bad = _weight(128, 100)
    assert f(ctypes.byref(bad), x, 4, A, B, 4, 1.0, h, ws, 1 << 20, None) == QN_ESHAPE
    assert lib.qn_last_error().decode() != ""
    g = lib.qlora_linear_bwd_x
    assert g(ctypes.byref(w), x, 4, A, B, 4, 1.0, h, None, 0, None) == QN_EWORKSPACE
    assert g(None, x, 4, A, B, 4, 1.0, h, ws, 1 << 20, None) == QN_EINVAL


def test_quantize_argument_errors_before_launch(lib):
    from bit_nf4_quantized_25_b200.binding import QN_EALIGN, QN_EINVAL, QN_EWORKSPACE
    w = _weight()
    P = ctypes.c_void_p
    q = lib.nf4_quantize
    assert q(None, ctypes.byref(w), P(0x700000), 1 << 20, None) == QN_EINVAL
    assert q(P(0x800004), ctypes.byref(w), P(0x700000), 1 << 20, None) == QN_EALIGN
    assert q(P(0x800000), ctypes.byref(w), P(0x700000), 16, None) == QN_EWORKSPACE
    assert q(P(0x800000), ctypes.byref(w), P(0x700010), 1 << 20, None) == QN_EALIGN
    ws = ctypes.c_size_t()
    assert lib.qn_quantize_workspace_size(128, 128, ctypes.byref(ws)) == 0 and ws.value >= 4 * 256
    d = lib.nf4_dequantize
    assert d(ctypes.byref(w), None, None) == QN_EINVAL
    assert d(ctypes.byref(w), P(0x900002), None) == QN_EALIGN


def test_empty_problems_enqueue_nothing(lib):
    w = _weight(0, 64)
    P = ctypes.c_void_p
    before = lib.qn_launch_count(0)
    assert lib.nf4_quantize(P(0x800000), ctypes.byref(w), None, 0, None) == 0
    w2 = _weight()
    assert lib.qlora_linear_fwd(ctypes.byref(w2), P(0x200000), 0, None, None, 0, 0.0, P(0x300000), None, 0, None) == 0
    assert lib.qn_launch_count(0) == before


def test_status_strings(lib):
    for s in range(6):
        assert lib.qn_status_string(s)


# ------------------------------------------------- binding: shapes refused before the call
# The library receives pointers and M only, so the binding refuses any tensor whose shape does
# not match the weight (it would be read or written out of bounds).

def _t(*shape):
    import torch
    return torch.empty(*shape, dtype=torch.bfloat16)


def test_binding_accepts_matching_linear_shapes():
    from bit_nf4_quantized_25_b200 import binding as qb
    n, k, M, r = 96, 128, 5, 16
    assert qb.check_linear_shapes(n, k, _t(M, k), _t(r, k), _t(n, r), _t(M, n), bwd=False) == r
    assert qb.check_linear_shapes(n, k, _t(M, n), _t(r, k), _t(n, r), _t(M, k), bwd=True) == r
    assert qb.check_linear_shapes(n, k, _t(M, k), None, None, None, bwd=False) == 0
    assert qb.check_linear_shapes(n, k, _t(0, k), _t(0, k), _t(n, 0), _t(0, n), bwd=False) == 0


@pytest.mark.parametrize("what", ["x_k", "x_1d", "out_fwd", "a_only", "a_cols", "b_rank", "b_rows", "gh_n",
                                  "out_bwd"])
def test_binding_refuses_mismatched_linear_shapes(what):
    from bit_nf4_quantized_25_b200 import binding as qb
    n, k, M, r = 96, 128, 5, 16
    x, A, B, h, gh, gx = _t(M, k), _t(r, k), _t(n, r), _t(M, n), _t(M, n), _t(M, k)
    bwd = what in ("gh_n", "out_bwd")
    act, out = (gh, gx) if bwd else (x, h)
    if what == "x_k":
        act = _t(M, k + 64)
    elif what == "x_1d":
        act = _t(M * k)
    elif what == "out_fwd":
        out = _t(M, n + 1)
    elif what == "a_only":
        B = None
    elif what == "a_cols":
        A = _t(r, k - 64)
    elif what == "b_rank":
        B = _t(n, r + 1)
    elif what == "b_rows":
        B = _t(n - 8, r)
    elif what == "gh_n":
        act = _t(M, k)
    elif what == "out_bwd":
        out = _t(M, n)
    with pytest.raises(ValueError):
        qb.check_linear_shapes(n, k, act, A, B, out, bwd=bwd)


def test_workspace_check_rejects_null(lib):
    # argument errors are returned before any GPU work
    assert lib.qlora_workspace_check(None, None) == 1  # QN_EINVAL
    assert "null workspace" in lib.qn_last_error().decode()


def test_timeout_status_has_a_description(lib):
    assert lib.qn_status_string(6).decode() == "a kernel gave up a bounded wait"


# ------------------------------------------- quant type and constant format (host checks)
# "Quantized LoRA (QLoRA) and 4-bit training" (apxml.com), the four configuration knobs: the
# quant type and double quantisation are settings of the weight; the struct carries them.

def test_weight_sizes_per_constant_format(lib):
    from bit_nf4_quantized_25_b200.binding import CONST_DQ, CONST_F32
    v = [ctypes.c_size_t() for _ in range(5)]
    n, k = 4096, 4096
    nb = n * k // 64
    assert lib.qn_weight_sizes(n, k, CONST_DQ, *(ctypes.byref(x) for x in v)) == 0
    assert [x.value for x in v] == [n * k // 2, nb, 4 * (nb // 256), 4, 0]
    assert lib.qn_weight_sizes(n, k, CONST_F32, *(ctypes.byref(x) for x in v)) == 0
    assert [x.value for x in v] == [n * k // 2, 0, 0, 0, 4 * nb]
    # 0.5 bit per weight of fp32 constants ("QLoRA & PEFT family" 3.3)
    assert 8 * v[4].value / (n * k) == 0.5
    assert lib.qn_weight_sizes(n, k, 7, *(ctypes.byref(x) for x in v)) == 1


def test_format_argument_errors_before_launch(lib):
    from bit_nf4_quantized_25_b200.binding import CONST_F32, CWeight, QN_EALIGN, QN_EINVAL
    P = ctypes.c_void_p
    d = lib.nf4_dequantize
    out = P(0x900000)
    w = _weight()
    w.quant_type = 5
    assert d(ctypes.byref(w), out, None) == QN_EINVAL
    w = _weight()
    w.const_format = 9
    assert d(ctypes.byref(w), out, None) == QN_EINVAL
    f32 = CWeight(128, 128, 0x100000, None, None, None, 1, CONST_F32, None)
    assert d(ctypes.byref(f32), out, None) == QN_EINVAL  # fp32 constants without absmax
    f32.absmax = 0x200004
    assert d(ctypes.byref(f32), out, None) == QN_EALIGN
    # fp32 constants need none of the double-quantisation buffers: argument checks pass and
    # only the missing W stops the quantiser
    f32.absmax = 0x200000
    assert lib.nf4_quantize(None, ctypes.byref(f32), P(0x700000), 1 << 20, None) == QN_EINVAL
    assert "W" in lib.qn_last_error().decode()
