"""Thin Python binding of ``libqlora_nf4.so`` (the C ABI in ``include/qlora_nf4.h``).

Argument marshalling only: torch tensors supply device memory and the current CUDA
stream; every step of the computation runs in the library's sm_100a kernels. There is
no fallback: if the library is missing or a call fails, an exception is raised.
"""
from __future__ import annotations

import ctypes
import dataclasses
import os
import threading

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libqlora_nf4.so")

QN_OK, QN_EINVAL, QN_ESHAPE, QN_EALIGN, QN_ECUDA, QN_EWORKSPACE, QN_ETIMEOUT = range(7)
BLOCK, GROUP, MAX_RANK = 64, 256, 256
QUANT_TYPES = {"nf4": 0, "fp4": 1}  # QN_QUANT_NF4, QN_QUANT_FP4
CONST_DQ, CONST_F32 = 0, 1           # QN_CONST_DQ, QN_CONST_F32

EXPORTED = ("qn_nf4_sizes", "qn_weight_sizes", "qn_quantize_workspace_size", "nf4_quantize", "nf4_quantize_static_ws", "nf4_dequantize",
            "qlora_workspace_size", "qlora_workspace_check", "qlora_linear_fwd", "qlora_linear_bwd_x",
            "qlora_merge_bf16", "qlora_lora_grads_workspace_size", "qlora_lora_grads", "qlora_linear_fwd_dropout",
            "qlora_linear_bwd_x_dropout", "qlora_lora_grads_dropout", "qn_status_string",
            "qn_last_error", "qn_launch_count", "qn_selftest_wait_timeout")


class QNError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(msg)
        self.status = status


class CWeight(ctypes.Structure):
    """qn_nf4_weight (see the header); fields left at zero mean NF4 with double quantisation."""
    _fields_ = [("n_out", ctypes.c_int64), ("k_in", ctypes.c_int64), ("codes", ctypes.c_void_p),
                ("absmax_q", ctypes.c_void_p), ("group_scale", ctypes.c_void_p),
                ("absmax_mean", ctypes.c_void_p), ("quant_type", ctypes.c_int32), ("const_format", ctypes.c_int32),
                ("absmax", ctypes.c_void_p)]


class CDropout(ctypes.Structure):
    """qn_lora_dropout (see the header): rate p, generator key and element-index offset."""
    _fields_ = [("p", ctypes.c_float), ("seed", ctypes.c_uint64), ("offset", ctypes.c_uint64)]


def _dropout_struct(dropout) -> CDropout:
    p, seed, offset = dropout
    return CDropout(float(p), int(seed) & 0xFFFFFFFFFFFFFFFF, int(offset) & 0xFFFFFFFFFFFFFFFF)


_lock = threading.Lock()
_lib = None


def load(path: str | None = None):
    """Load the library (once). Raises if it is missing: there is no other path."""
    global _lib
    with _lock:
        if _lib is not None and path is None:
            return _lib
        p = path or LIB_PATH
        if not os.path.exists(p):
            raise RuntimeError(f"{p} is missing: build it with `python -m bit_nf4_quantized_25_b200.build`")
        lib = ctypes.CDLL(p)
        P, i64, sz = ctypes.c_void_p, ctypes.c_int64, ctypes.POINTER(ctypes.c_size_t)
        W = ctypes.POINTER(CWeight)
        st = ctypes.c_int
        lib.qn_nf4_sizes.argtypes = [i64, i64, sz, sz, sz, sz]
        lib.qn_weight_sizes.argtypes = [i64, i64, ctypes.c_int, sz, sz, sz, sz, sz]
        lib.qn_quantize_workspace_size.argtypes = [i64, i64, sz]
        lib.nf4_quantize.argtypes = [P, W, P, ctypes.c_size_t, P]
        lib.nf4_dequantize.argtypes = [W, P, P]
        lib.nf4_quantize_static_ws.argtypes = [P, W, P]
        lib.qlora_workspace_size.argtypes = [i64, i64, i64, ctypes.c_int, sz]
        lib.qlora_workspace_check.argtypes = [P, P]
        lib.qn_selftest_wait_timeout.argtypes = [P, ctypes.c_size_t, P]
        lib.qlora_linear_fwd.argtypes = [W, P, i64, P, P, ctypes.c_int, ctypes.c_float, P, P, ctypes.c_size_t, P]
        lib.qlora_linear_bwd_x.argtypes = lib.qlora_linear_fwd.argtypes
        lib.qlora_merge_bf16.argtypes = [W, P, P, ctypes.c_int, ctypes.c_float, P, P]
        lib.qlora_lora_grads_workspace_size.argtypes = [i64, ctypes.c_int, sz]
        lib.qlora_lora_grads.argtypes = [P, P, i64, i64, i64, P, P, ctypes.c_int, ctypes.c_float, P, P, P,
                                         ctypes.c_size_t, P]
        D = ctypes.POINTER(CDropout)
        lib.qlora_linear_fwd_dropout.argtypes = [W, P, i64, P, P, ctypes.c_int, ctypes.c_float, D, P, P,
                                                 ctypes.c_size_t, P]
        lib.qlora_linear_bwd_x_dropout.argtypes = lib.qlora_linear_fwd_dropout.argtypes
        lib.qlora_lora_grads_dropout.argtypes = [P, P, i64, i64, i64, P, P, ctypes.c_int, ctypes.c_float, D, P, P,
                                                 P, ctypes.c_size_t, P]
        for f in ("qlora_merge_bf16", "qlora_lora_grads_workspace_size", "qlora_lora_grads", "qn_nf4_sizes", "qn_quantize_workspace_size", "nf4_quantize", "nf4_quantize_static_ws", "nf4_dequantize",
                  "qlora_workspace_size", "qlora_workspace_check", "qlora_linear_fwd", "qlora_linear_bwd_x",
                  "qlora_linear_fwd_dropout", "qlora_linear_bwd_x_dropout", "qlora_lora_grads_dropout"):
            getattr(lib, f).restype = st
        lib.qn_status_string.argtypes = [st]
        lib.qn_status_string.restype = ctypes.c_char_p
        lib.qn_last_error.restype = ctypes.c_char_p
        lib.qn_launch_count.argtypes = [ctypes.c_int]
        lib.qn_launch_count.restype = ctypes.c_uint64
        if path is None:
            _lib = lib
        return lib


def _check(status: int, what: str):
    if status != QN_OK:
        lib = load()
        raise QNError(status, f"{what}: {lib.qn_status_string(status).decode()} ({lib.qn_last_error().decode()})")


def _ptr(t: torch.Tensor | None):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _dev_bf16(t: torch.Tensor, name: str):
    if not t.is_cuda or t.dtype != torch.bfloat16 or not t.is_contiguous():
        raise ValueError(f"{name} must be a contiguous bf16 CUDA tensor")


def _expect_shape(t: torch.Tensor, shape, name: str):
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")


def check_linear_shapes(n_out: int, k_in: int, act: torch.Tensor, A, B, out, bwd: bool) -> int:
    """Shapes of a linear call; returns the adapter rank r. The library sees only pointers and
    M, so a tensor of the wrong shape would be read or written out of bounds: it is refused
    here. Forward: x (M, k_in) -> h (M, n_out); input gradient: grad_h (M, n_out) ->
    grad_x (M, k_in); A (r, k_in) and B (n_out, r) together, or neither."""
    name = "grad_h" if bwd else "x"
    if act.dim() != 2:
        raise ValueError(f"{name} must be 2-D (tokens x features)")
    M = act.shape[0]
    _expect_shape(act, (M, n_out if bwd else k_in), name)
    if (A is None) != (B is None):
        raise ValueError("A and B are given together or not at all")
    r = 0
    if A is not None:
        if A.dim() != 2:
            raise ValueError("A must be 2-D (r x k_in)")
        r = A.shape[0]
        _expect_shape(A, (r, k_in), "A")
        _expect_shape(B, (n_out, r), "B")
    if out is not None:
        _expect_shape(out, (M, k_in if bwd else n_out), "out")
    return r


def new_workspace(need: int, device="cuda") -> torch.Tensor:
    """A linear-layer workspace of `need` bytes, all zero as the header asks of a new workspace (see
    qlora_workspace_size there); reusable across calls in stream order."""
    return torch.zeros(max(need, 256), dtype=torch.uint8, device=device)


def workspace_check(ws: torch.Tensor, stream=None):
    """Raise QNError(QN_ETIMEOUT) if a kernel that used `ws` gave up a bounded wait since the last
    check (the error word is then cleared); synchronises the stream."""
    _check(load().qlora_workspace_check(_ptr(ws), _stream(stream)), "qlora_workspace_check")


def selftest_wait_timeout(ws: torch.Tensor, stream=None):
    """Enqueue the library's bounded-wait self-test on a zeroed workspace: its wait runs out and
    sets the error word (see qn_selftest_wait_timeout in the header)."""
    if not ws.is_cuda or not ws.is_contiguous():
        raise ValueError("workspace must be a contiguous CUDA tensor")
    _check(load().qn_selftest_wait_timeout(_ptr(ws), ws.numel() * ws.element_size(), _stream(stream)),
           "qn_selftest_wait_timeout")


def _workspace(ws: torch.Tensor | None, need: int, device) -> tuple[torch.Tensor, int]:
    """A caller workspace (contiguous CUDA memory, any dtype) or a fresh one; its size in bytes."""
    if ws is None:
        ws = new_workspace(need, device)
    elif not ws.is_cuda or not ws.is_contiguous():
        raise ValueError("workspace must be a contiguous CUDA tensor")
    return ws, ws.numel() * ws.element_size()


def _same_device(w, *ts):
    dev = w.codes.device
    for t in ts:
        if t is not None and t.device != dev:
            raise ValueError(f"tensor on {t.device}, the weight is on {dev}")


def sizes(n_out: int, k_in: int):
    """(codes, absmax_q, group_scale, absmax_mean) byte sizes of a quantised weight."""
    a, b, c, d = (ctypes.c_size_t() for _ in range(4))
    _check(load().qn_nf4_sizes(n_out, k_in, ctypes.byref(a), ctypes.byref(b), ctypes.byref(c), ctypes.byref(d)),
           "qn_nf4_sizes")
    return a.value, b.value, c.value, d.value


def weight_sizes(n_out: int, k_in: int, double_quant: bool = True):
    """(codes, absmax_q, group_scale, absmax_mean, absmax fp32) byte sizes for a constant format."""
    v = [ctypes.c_size_t() for _ in range(5)]
    _check(load().qn_weight_sizes(n_out, k_in, CONST_DQ if double_quant else CONST_F32, *(ctypes.byref(x) for x in v)),
           "qn_weight_sizes")
    return tuple(x.value for x in v)


def quantize_workspace_size(n_out: int, k_in: int) -> int:
    v = ctypes.c_size_t()
    _check(load().qn_quantize_workspace_size(n_out, k_in, ctypes.byref(v)), "qn_quantize_workspace_size")
    return v.value


def linear_workspace_size(M: int, n_out: int, k_in: int, r: int) -> int:
    v = ctypes.c_size_t()
    _check(load().qlora_workspace_size(M, n_out, k_in, r, ctypes.byref(v)), "qlora_workspace_size")
    return v.value


def launch_count(reset: bool = False) -> int:
    return int(load().qn_launch_count(1 if reset else 0))


@dataclasses.dataclass
class NF4Weight:
    """A quantised weight: its device buffers plus the shape and format (see include/qlora_nf4.h).
    quant_type "nf4" or "fp4"; double_quant True: absmax_q, group_scale, absmax_mean hold the
    constants; False: absmax (fp32 per block) does, and the other three are empty."""
    n_out: int
    k_in: int
    codes: torch.Tensor        # uint8 [n_out*k_in/2]
    absmax_q: torch.Tensor     # uint8 [nb], E4M3 bits
    group_scale: torch.Tensor  # float32 [ng]
    absmax_mean: torch.Tensor  # float32 [1]
    quant_type: str = "nf4"
    double_quant: bool = True
    absmax: torch.Tensor | None = None  # float32 [nb] (double_quant False)

    @staticmethod
    def empty(n_out: int, k_in: int, device="cuda", quant_type: str = "nf4", double_quant: bool = True) -> "NF4Weight":
        if quant_type not in QUANT_TYPES:
            raise ValueError(f"quant_type {quant_type!r} is not one of {sorted(QUANT_TYPES)}")
        cb, ab, sb, mb, fb = weight_sizes(n_out, k_in, double_quant)
        u8 = dict(dtype=torch.uint8, device=device)
        f32 = dict(dtype=torch.float32, device=device)
        return NF4Weight(n_out, k_in, torch.empty(cb, **u8), torch.empty(ab, **u8), torch.empty(sb // 4, **f32),
                         torch.empty(mb // 4, **f32), quant_type, bool(double_quant),
                         None if double_quant else torch.empty(fb // 4, **f32))

    def c_struct(self) -> CWeight:
        if self.double_quant:
            return CWeight(self.n_out, self.k_in, self.codes.data_ptr(), self.absmax_q.data_ptr(),
                           self.group_scale.data_ptr(), self.absmax_mean.data_ptr(), QUANT_TYPES[self.quant_type],
                           CONST_DQ, None)
        return CWeight(self.n_out, self.k_in, self.codes.data_ptr(), None, None, None, QUANT_TYPES[self.quant_type],
                       CONST_F32, self.absmax.data_ptr())

    def nbytes(self) -> int:
        ts = (self.codes, self.absmax_q, self.group_scale, self.absmax_mean) + (
            () if self.absmax is None else (self.absmax,))
        return sum(t.numel() * t.element_size() for t in ts)


def nf4_quantize(W: torch.Tensor, out: NF4Weight | None = None, workspace: torch.Tensor | None = None,
                 stream=None, quant_type: str = "nf4", double_quant: bool = True) -> NF4Weight:
    """Quantise a bf16 (n_out x k_in) CUDA tensor: NF4 (or "fp4") codes with double-quantised (or
    fp32) block constants; an `out` given keeps its own format."""
    _dev_bf16(W, "W")
    if W.dim() != 2:
        raise ValueError("W must be 2-D (n_out x k_in)")
    n, k = W.shape
    out = out or NF4Weight.empty(n, k, W.device, quant_type, double_quant)
    if (out.n_out, out.k_in) != (n, k):
        raise ValueError(f"out holds a {out.n_out} x {out.k_in} weight, W is {n} x {k}")
    _same_device(out, W)
    workspace, ws_bytes = _workspace(workspace, quantize_workspace_size(n, k), W.device)
    cw = out.c_struct()
    _check(load().nf4_quantize(_ptr(W), ctypes.byref(cw), _ptr(workspace), ws_bytes, _stream(stream)),
           "nf4_quantize")
    return out


def nf4_quantize_static_ws(W: torch.Tensor, out: NF4Weight, stream=None) -> NF4Weight:
    """nf4_quantize using the library's static device scratch instead of a workspace; the
    library allocates nothing (the output buffers are the caller's). See the header for the
    size limit and the rule that overlapping calls race."""
    _dev_bf16(W, "W")
    if W.dim() != 2 or (out.n_out, out.k_in) != tuple(W.shape):
        raise ValueError(f"W of shape {tuple(W.shape)} does not match a {out.n_out} x {out.k_in} weight")
    _same_device(out, W)
    cw = out.c_struct()
    _check(load().nf4_quantize_static_ws(_ptr(W), ctypes.byref(cw), _stream(stream)), "nf4_quantize_static_ws")
    return out


def nf4_dequantize(w: NF4Weight, out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    out = out if out is not None else torch.empty(w.n_out, w.k_in, dtype=torch.bfloat16, device=w.codes.device)
    _dev_bf16(out, "out")
    _expect_shape(out, (w.n_out, w.k_in), "out")
    _same_device(w, out)
    cw = w.c_struct()
    _check(load().nf4_dequantize(ctypes.byref(cw), _ptr(out), _stream(stream)), "nf4_dequantize")
    return out


def _lora(A, B, r):
    if r == 0:
        return None, None
    _dev_bf16(A, "A")
    _dev_bf16(B, "B")
    return A, B


def qlora_linear_fwd(w: NF4Weight, x: torch.Tensor, A: torch.Tensor | None, B: torch.Tensor | None,
                     alpha: float, out: torch.Tensor | None = None, workspace: torch.Tensor | None = None,
                     stream=None, dropout=None) -> torch.Tensor:
    """h = dequant(W) x + (alpha/r) B (A x); x is M x k_in, h is M x n_out (bf16).
    dropout = (p, seed, offset): LoRA dropout of the adapter's input (qlora_linear_fwd_dropout)."""
    _dev_bf16(x, "x")
    r = check_linear_shapes(w.n_out, w.k_in, x, A, B, out, bwd=False)
    M = x.shape[0]
    A, B = _lora(A, B, r)
    out = out if out is not None else torch.empty(M, w.n_out, dtype=torch.bfloat16, device=x.device)
    _dev_bf16(out, "out")
    _same_device(w, x, A, B, out)
    workspace, ws_bytes = _workspace(workspace, linear_workspace_size(M, w.n_out, w.k_in, r), x.device)
    cw = w.c_struct()
    if dropout is None:
        _check(load().qlora_linear_fwd(ctypes.byref(cw), _ptr(x), M, _ptr(A), _ptr(B), r, float(alpha), _ptr(out),
                                       _ptr(workspace), ws_bytes, _stream(stream)), "qlora_linear_fwd")
    else:
        d = _dropout_struct(dropout)
        _check(load().qlora_linear_fwd_dropout(ctypes.byref(cw), _ptr(x), M, _ptr(A), _ptr(B), r, float(alpha),
                                               ctypes.byref(d), _ptr(out), _ptr(workspace), ws_bytes,
                                               _stream(stream)), "qlora_linear_fwd_dropout")
    return out


def qlora_linear_bwd_x(w: NF4Weight, grad_h: torch.Tensor, A: torch.Tensor | None, B: torch.Tensor | None,
                       alpha: float, out: torch.Tensor | None = None, workspace: torch.Tensor | None = None,
                       stream=None, dropout=None) -> torch.Tensor:
    """grad_x = dequant(W)^T grad_h + (alpha/r) A^T (B^T grad_h); grad_h is M x n_out.
    dropout = (p, seed, offset): the forward's LoRA-dropout mask (qlora_linear_bwd_x_dropout)."""
    _dev_bf16(grad_h, "grad_h")
    r = check_linear_shapes(w.n_out, w.k_in, grad_h, A, B, out, bwd=True)
    M = grad_h.shape[0]
    A, B = _lora(A, B, r)
    out = out if out is not None else torch.empty(M, w.k_in, dtype=torch.bfloat16, device=grad_h.device)
    _dev_bf16(out, "out")
    _same_device(w, grad_h, A, B, out)
    workspace, ws_bytes = _workspace(workspace, linear_workspace_size(M, w.n_out, w.k_in, r), grad_h.device)
    cw = w.c_struct()
    if dropout is None:
        _check(load().qlora_linear_bwd_x(ctypes.byref(cw), _ptr(grad_h), M, _ptr(A), _ptr(B), r, float(alpha),
                                         _ptr(out), _ptr(workspace), ws_bytes, _stream(stream)),
               "qlora_linear_bwd_x")
    else:
        d = _dropout_struct(dropout)
        _check(load().qlora_linear_bwd_x_dropout(ctypes.byref(cw), _ptr(grad_h), M, _ptr(A), _ptr(B), r,
                                                 float(alpha), ctypes.byref(d), _ptr(out), _ptr(workspace),
                                                 ws_bytes, _stream(stream)), "qlora_linear_bwd_x_dropout")
    return out


def qlora_merge_bf16(w: NF4Weight, A: torch.Tensor | None, B: torch.Tensor | None, alpha: float,
                     out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """W' + (alpha/r) B A as a bf16 n_out x k_in tensor (merge and unload)."""
    if (A is None) != (B is None):
        raise ValueError("A and B are given together or not at all")
    r = 0
    if A is not None:
        _dev_bf16(A, "A")
        _dev_bf16(B, "B")
        if A.dim() != 2:
            raise ValueError("A must be 2-D (r x k_in)")
        r = A.shape[0]
        _expect_shape(A, (r, w.k_in), "A")
        _expect_shape(B, (w.n_out, r), "B")
    out = out if out is not None else torch.empty(w.n_out, w.k_in, dtype=torch.bfloat16, device=w.codes.device)
    _dev_bf16(out, "out")
    _expect_shape(out, (w.n_out, w.k_in), "out")
    _same_device(w, A, B, out)
    cw = w.c_struct()
    _check(load().qlora_merge_bf16(ctypes.byref(cw), _ptr(A), _ptr(B), r, float(alpha), _ptr(out), _stream(stream)),
           "qlora_merge_bf16")
    return out


def lora_grads_workspace_size(M: int, r: int) -> int:
    v = ctypes.c_size_t()
    _check(load().qlora_lora_grads_workspace_size(M, r, ctypes.byref(v)), "qlora_lora_grads_workspace_size")
    return v.value


def qlora_lora_grads(x: torch.Tensor, grad_h: torch.Tensor, A: torch.Tensor, B: torch.Tensor, alpha: float,
                     grad_A: torch.Tensor | None = None, grad_B: torch.Tensor | None = None,
                     workspace: torch.Tensor | None = None, stream=None, dropout=None):
    """(grad_A (r x k_in), grad_B (n_out x r)) in fp32 for x (M x k_in) and grad_h (M x n_out).
    dropout = (p, seed, offset): the forward's LoRA-dropout mask (qlora_lora_grads_dropout)."""
    for t, nm in ((x, "x"), (grad_h, "grad_h"), (A, "A"), (B, "B")):
        _dev_bf16(t, nm)
    if x.dim() != 2 or grad_h.dim() != 2 or A.dim() != 2 or B.dim() != 2:
        raise ValueError("x, grad_h, A and B must be 2-D")
    M, k = x.shape
    n = grad_h.shape[1]
    r = A.shape[0]
    _expect_shape(grad_h, (M, n), "grad_h")
    _expect_shape(A, (r, k), "A")
    _expect_shape(B, (n, r), "B")
    f32 = dict(dtype=torch.float32, device=x.device)
    grad_A = grad_A if grad_A is not None else torch.empty(r, k, **f32)
    grad_B = grad_B if grad_B is not None else torch.empty(n, r, **f32)
    for t, shp, nm in ((grad_A, (r, k), "grad_A"), (grad_B, (n, r), "grad_B")):
        if not t.is_cuda or t.dtype != torch.float32 or not t.is_contiguous():
            raise ValueError(f"{nm} must be a contiguous fp32 CUDA tensor")
        _expect_shape(t, shp, nm)
    if workspace is None:
        workspace = torch.empty(max(lora_grads_workspace_size(M, r), 256), dtype=torch.uint8, device=x.device)
    elif not workspace.is_cuda or not workspace.is_contiguous():
        raise ValueError("workspace must be a contiguous CUDA tensor")
    for t in (grad_h, A, B, grad_A, grad_B, workspace):
        if t.device != x.device:
            raise ValueError(f"tensor on {t.device}, x is on {x.device}")
    wsb = workspace.numel() * workspace.element_size()
    if dropout is None:
        _check(load().qlora_lora_grads(_ptr(x), _ptr(grad_h), M, n, k, _ptr(A), _ptr(B), r, float(alpha),
                                       _ptr(grad_A), _ptr(grad_B), _ptr(workspace), wsb, _stream(stream)),
               "qlora_lora_grads")
    else:
        d = _dropout_struct(dropout)
        _check(load().qlora_lora_grads_dropout(_ptr(x), _ptr(grad_h), M, n, k, _ptr(A), _ptr(B), r, float(alpha),
                                               ctypes.byref(d), _ptr(grad_A), _ptr(grad_B), _ptr(workspace), wsb,
                                               _stream(stream)), "qlora_lora_grads_dropout")
    return grad_A, grad_B
