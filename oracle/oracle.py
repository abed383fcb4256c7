"""CPU oracle for the NF4 + double-quant + LoRA linear layer (test infrastructure).

Quantised weights are dicts: ``codes`` and either ``q``, ``sigma``, ``mu`` (double
quantisation, ``dq`` True, the default) or ``absmax`` (fp32 block constants, ``dq``
False); ``qtype`` is "nf4" (default) or "fp4" (the 4-bit float, E2M1).

Only the tests, ``__graft_entry__.smoke()`` and ``bench.py``'s ``cpu_baseline``
leg and reference arm (``--impl reference``) may import this module. The product path (the CUDA library and its
Python binding) never imports, links or executes anything under ``oracle/``.

The arithmetic lives in ``nf4_oracle.c`` (plain C, fp64 sums, OpenMP over
independent outputs); this module only compiles it with gcc and marshals numpy
arrays through ctypes. Every function documents the passage it follows in the C
file's header.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "nf4_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile the C oracle into ``oracle/liboracle.so`` (gcc, OpenMP, strict IEEE)."""
    if not force and os.path.exists(_LIB) and os.path.getmtime(_LIB) >= os.path.getmtime(_SRC):
        return _LIB
    tmp = _LIB + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp", "-ffp-contract=off",
           "-fno-fast-math", "-Wall", "-o", tmp, _SRC, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, _LIB)
    return _LIB


QTYPES = {"nf4": 0, "fp4": 1}


class _Weight(ctypes.Structure):
    _fields_ = [("qtype", ctypes.c_int), ("dq", ctypes.c_int), ("codes", ctypes.c_void_p),
                ("q", ctypes.c_void_p), ("sigma", ctypes.c_void_p), ("mu", ctypes.c_float),
                ("absmax", ctypes.c_void_p)]


def _weight(qw: dict) -> _Weight:
    """The C view of a quantised-weight dict (its arrays stay owned by the dict)."""
    dq = bool(qw.get("dq", True))
    return _Weight(QTYPES[qw.get("qtype", "nf4")], int(dq), _ptr(qw["codes"]),
                   _ptr(qw["q"]) if dq else None, _ptr(qw["sigma"]) if dq else None,
                   float(qw["mu"]) if dq else 0.0, None if dq else _ptr(qw["absmax"]))


def _load():
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        lib = ctypes.CDLL(build())
        P = ctypes.c_void_p
        i64 = ctypes.c_int64
        lib.or_nf4_table.argtypes = [P]
        lib.or_4bit_table.argtypes = [ctypes.c_int, P]
        lib.or_4bit_code.argtypes = [ctypes.c_int, ctypes.c_float, ctypes.c_float]
        lib.or_4bit_code.restype = ctypes.c_int
        lib.or_quantize4.argtypes = [ctypes.c_int, ctypes.c_int, P, i64, i64, P, P, P, P, P]
        lib.or_quantize4.restype = ctypes.c_int
        WP = ctypes.POINTER(_Weight)
        lib.or_threads.restype = ctypes.c_int
        lib.or_f32_to_bf16.argtypes = [ctypes.c_float]
        lib.or_f32_to_bf16.restype = ctypes.c_uint16
        lib.or_e4m3_decode.argtypes = [ctypes.c_uint8]
        lib.or_e4m3_decode.restype = ctypes.c_double
        lib.or_e4m3_encode.argtypes = [ctypes.c_float]
        lib.or_e4m3_encode.restype = ctypes.c_uint8
        lib.or_exact_mean_f32.argtypes = [P, i64]
        lib.or_exact_mean_f32.restype = ctypes.c_float
        lib.or_nf4_code.argtypes = [ctypes.c_float, ctypes.c_float]
        lib.or_nf4_code.restype = ctypes.c_int
        lib.or_num_blocks.argtypes = [i64, i64]
        lib.or_num_blocks.restype = i64
        lib.or_num_groups.argtypes = [i64, i64]
        lib.or_num_groups.restype = i64
        lib.or_nf4_quantize.argtypes = [P, i64, i64, P, P, P, P, P]
        lib.or_nf4_quantize.restype = ctypes.c_int
        lib.or_block_constant.argtypes = [ctypes.c_uint8, ctypes.c_float, ctypes.c_float]
        lib.or_block_constant.restype = ctypes.c_float
        lib.or_dequant_bf16.argtypes = [WP, i64, i64, P]
        lib.or_dequant_f64.argtypes = [WP, i64, i64, P]
        u64, f64 = ctypes.c_uint64, ctypes.c_double
        lib.or_qlora_fwd.argtypes = [WP, i64, i64, P, P, i64, P, P, ctypes.c_int, ctypes.c_float, f64, u64, u64,
                                     P]
        lib.or_qlora_bwd_x.argtypes = lib.or_qlora_fwd.argtypes
        lib.or_lora_grads.argtypes = [P, P, i64, i64, i64, P, P, ctypes.c_int, ctypes.c_float, f64, u64, u64,
                                      P, P]
        lib.or_philox4x32_10.argtypes = [P, P, P]
        lib.or_dropout_threshold.argtypes = [f64]
        lib.or_dropout_threshold.restype = ctypes.c_uint32
        lib.or_dropout_bits.argtypes = [u64, u64]
        lib.or_dropout_bits.restype = ctypes.c_uint32
        lib.or_f64_to_bf16.argtypes = [ctypes.c_double]
        lib.or_f64_to_bf16.restype = ctypes.c_uint16
        lib.or_merge_bf16.argtypes = [WP, i64, i64, P, P, ctypes.c_int, ctypes.c_float, P]
        _lib = lib
        return lib


def _ptr(a: np.ndarray | None):
    if a is None:
        return None
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data_as(ctypes.c_void_p)


def _bits16(a: np.ndarray) -> np.ndarray:
    """bf16 payload as uint16 bits (accepts uint16 or int16 arrays)."""
    a = np.ascontiguousarray(a)
    assert a.dtype in (np.uint16, np.int16), a.dtype
    return a.view(np.uint16)


def threads() -> int:
    return int(_load().or_threads())


def nf4_table() -> np.ndarray:
    out = np.zeros(16, dtype=np.float64)
    _load().or_nf4_table(_ptr(out))
    return out


def table(qtype: str = "nf4") -> np.ndarray:
    """The 16 code values of a quant type, in code order (fp32 values as fp64)."""
    out = np.zeros(16, dtype=np.float64)
    _load().or_4bit_table(QTYPES[qtype], _ptr(out))
    return out


def code4(qtype: str, w: float, c: float) -> int:
    """Code of weight w in a block of absmax c under quant type qtype."""
    return int(_load().or_4bit_code(QTYPES[qtype], float(w), float(c)))


def f32_to_bf16(v: float) -> int:
    return int(_load().or_f32_to_bf16(float(v)))


def e4m3_decode(code: int) -> float:
    return float(_load().or_e4m3_decode(int(code)))


def e4m3_encode(v: float) -> int:
    return int(_load().or_e4m3_encode(float(v)))


def exact_mean_f32(c: np.ndarray) -> np.float32:
    c = np.ascontiguousarray(c, dtype=np.float32)
    return np.float32(_load().or_exact_mean_f32(_ptr(c), c.size))


def nf4_code(w: float, c: float) -> int:
    return int(_load().or_nf4_code(float(w), float(c)))


def num_blocks(n: int, k: int) -> int:
    return int(_load().or_num_blocks(n, k))


def num_groups(n: int, k: int) -> int:
    return int(_load().or_num_groups(n, k))


def block_constant(qb: int, sigma: float, mu: float) -> np.float32:
    return np.float32(_load().or_block_constant(int(qb), float(sigma), float(mu)))


def quantize4(W_bits: np.ndarray, n: int, k: int, qtype: str = "nf4", double_quant: bool = True):
    """Quantise a row-major n x k bf16 matrix (given as uint16 bits) with quant type qtype.

    Returns dict(codes=u8[n*k/2], absmax=f32[nb], qtype, dq) plus, with double quantisation,
    q=u8[nb], sigma=f32[ng], mu=f32.
    """
    W = _bits16(W_bits).reshape(-1)
    assert W.size == n * k
    nb, ng = num_blocks(n, k), num_groups(n, k)
    codes = np.zeros(n * k // 2, dtype=np.uint8)
    q = np.zeros(nb, dtype=np.uint8)
    sigma = np.zeros(ng, dtype=np.float32)
    mu = np.zeros(1, dtype=np.float32)
    absmax = np.zeros(nb, dtype=np.float32)
    rc = _load().or_quantize4(QTYPES[qtype], int(bool(double_quant)), _ptr(W), n, k, _ptr(codes), _ptr(q),
                              _ptr(sigma), _ptr(mu), _ptr(absmax))
    if rc != 0:
        raise ValueError(f"or_quantize4 failed: {rc} (k must be a multiple of 64)")
    out = dict(codes=codes, absmax=absmax, qtype=qtype, dq=bool(double_quant))
    if double_quant:
        out.update(q=q, sigma=sigma, mu=np.float32(mu[0]))
    return out


def nf4_quantize(W_bits: np.ndarray, n: int, k: int):
    """NF4 with double quantisation: dict(codes, q, sigma, mu, absmax)."""
    return quantize4(W_bits, n, k, "nf4", True)


def nf4_dequant_bf16(qw: dict, n: int, k: int) -> np.ndarray:
    """bf16 bits of the dequantised weight (any quant type and constant format)."""
    out = np.zeros(n * k, dtype=np.uint16)
    w = _weight(qw)
    _load().or_dequant_bf16(ctypes.byref(w), n, k, _ptr(out))
    return out.reshape(n, k)


def nf4_dequant_f64(qw: dict, n: int, k: int) -> np.ndarray:
    """The dequantised weight in fp64, unrounded (any quant type and constant format)."""
    out = np.zeros(n * k, dtype=np.float64)
    w = _weight(qw)
    _load().or_dequant_f64(ctypes.byref(w), n, k, _ptr(out))
    return out.reshape(n, k)


def _rows(m: int, rows) -> np.ndarray:
    if rows is None:
        return np.arange(m, dtype=np.int64)
    return np.ascontiguousarray(np.asarray(rows, dtype=np.int64))


def philox4x32_10(ctr, key) -> np.ndarray:
    """The four 32-bit words of Philox4x32-10 at counter `ctr` (4 words) and key `key` (2 words)."""
    c = np.ascontiguousarray(np.asarray(ctr, dtype=np.uint32))
    kk = np.ascontiguousarray(np.asarray(key, dtype=np.uint32))
    out = np.zeros(4, dtype=np.uint32)
    _load().or_philox4x32_10(_ptr(c), _ptr(kk), _ptr(out))
    return out


def dropout_threshold(p: float) -> int:
    return int(_load().or_dropout_threshold(float(p)))


def dropout_bits(seed: int, e: int) -> int:
    """The generator's 32-bit output for (offset) element index e."""
    return int(_load().or_dropout_bits(int(seed), int(e)))


def dropout_keep(seed: int, offset: int, p: float, m: int, k: int) -> np.ndarray:
    """m x k boolean mask of the adapter input's surviving elements (slow; small shapes)."""
    thr = dropout_threshold(p)
    return np.array([[thr == 0 or dropout_bits(seed, offset + i * k + j) >= thr for j in range(k)]
                     for i in range(m)], dtype=bool)


def qlora_fwd(qw: dict, n: int, k: int, x_bits: np.ndarray, m: int, A_bits, B_bits, r: int,
              alpha: float, rows=None, p_drop: float = 0.0, seed: int = 0, offset: int = 0) -> np.ndarray:
    """h (fp64) for the selected token rows of x (m x k bf16 bits); shape len(rows) x n.
    p_drop > 0: LoRA dropout of the adapter's input with generator (seed, offset)."""
    rows = _rows(m, rows)
    x = _bits16(x_bits).reshape(-1)
    assert x.size == m * k
    A = _bits16(A_bits).reshape(-1) if r > 0 else None
    B = _bits16(B_bits).reshape(-1) if r > 0 else None
    h = np.zeros(rows.size * n, dtype=np.float64)
    w = _weight(qw)
    _load().or_qlora_fwd(ctypes.byref(w), n, k, _ptr(x), _ptr(rows), rows.size, _ptr(A), _ptr(B), int(r),
                         float(alpha), float(p_drop), int(seed), int(offset), _ptr(h))
    return h.reshape(rows.size, n)


def qlora_bwd_x(qw: dict, n: int, k: int, gh_bits: np.ndarray, m: int, A_bits, B_bits, r: int,
                alpha: float, rows=None, p_drop: float = 0.0, seed: int = 0, offset: int = 0) -> np.ndarray:
    """grad_x (fp64) for the selected token rows of grad_h (m x n bf16 bits); shape len(rows) x k."""
    rows = _rows(m, rows)
    g = _bits16(gh_bits).reshape(-1)
    assert g.size == m * n
    A = _bits16(A_bits).reshape(-1) if r > 0 else None
    B = _bits16(B_bits).reshape(-1) if r > 0 else None
    gx = np.zeros(rows.size * k, dtype=np.float64)
    w = _weight(qw)
    _load().or_qlora_bwd_x(ctypes.byref(w), n, k, _ptr(g), _ptr(rows), rows.size, _ptr(A), _ptr(B), int(r),
                           float(alpha), float(p_drop), int(seed), int(offset), _ptr(gx))
    return gx.reshape(rows.size, k)


def lora_grads(x_bits: np.ndarray, gh_bits: np.ndarray, m: int, n: int, k: int, A_bits, B_bits, r: int,
               alpha: float, p_drop: float = 0.0, seed: int = 0, offset: int = 0):
    """(grad_A (r x k), grad_B (n x r)) in fp64 for all m token rows of x (m x k) and grad_h (m x n)."""
    x = _bits16(x_bits).reshape(-1)
    g = _bits16(gh_bits).reshape(-1)
    assert x.size == m * k and g.size == m * n
    A = _bits16(A_bits).reshape(-1)
    B = _bits16(B_bits).reshape(-1)
    gA = np.zeros(r * k, dtype=np.float64)
    gB = np.zeros(n * r, dtype=np.float64)
    _load().or_lora_grads(_ptr(x), _ptr(g), m, n, k, _ptr(A), _ptr(B), int(r), float(alpha), float(p_drop),
                          int(seed), int(offset), _ptr(gA), _ptr(gB))
    return gA.reshape(r, k), gB.reshape(n, r)


def f64_to_bf16(v: float) -> int:
    return int(_load().or_f64_to_bf16(float(v)))


def merge_bf16(qw: dict, n: int, k: int, A_bits, B_bits, r: int, alpha: float) -> np.ndarray:
    """bf16 bits (n x k) of the merged weight W' + s B A."""
    A = _bits16(A_bits).reshape(-1) if r > 0 else None
    B = _bits16(B_bits).reshape(-1) if r > 0 else None
    out = np.zeros(n * k, dtype=np.uint16)
    w = _weight(qw)
    _load().or_merge_bf16(ctypes.byref(w), n, k, _ptr(A), _ptr(B), int(r), float(alpha), _ptr(out))
    return out.reshape(n, k)
