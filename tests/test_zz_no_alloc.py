"""The allocation-free quantiser entry point, nf4_quantize_static_ws.

It serves callers that cannot allocate device memory when they quantise (inside a
global-mode stream capture, under an allocator that owns all device memory, or on paths
that cannot take cudaMalloc's implicit synchronisation): the scratch is a static device
array inside the library. Its results must equal those of nf4_quantize with a caller
workspace, bit for bit, on consecutive calls that reuse the same static scratch.

This file is collected last (test_zz_*) so that a run stopping at the first failure has
already run every other test; it passes on its own and after the others.
"""
import ctypes

import numpy as np
import pytest
import torch

from bit_nf4_quantized_25_b200 import binding as qb
from bit_nf4_quantized_25_b200 import synth

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)


def _same(a: qb.NF4Weight, b: qb.NF4Weight):
    assert torch.equal(a.codes, b.codes)
    assert torch.equal(a.absmax_q, b.absmax_q)
    assert torch.equal(a.group_scale.view(torch.int32), b.group_scale.view(torch.int32))
    assert torch.equal(a.absmax_mean.view(torch.int32), b.absmax_mean.view(torch.int32))


def test_static_scratch_matches_workspace_entry_point():
    lib = qb.load()
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    shapes = [(4096, 4096, 31), (11008, 4096, 32)]  # two calls in a row, different sizes
    for n, k, seed in shapes:
        W = synth.student_t_bf16((n, k), 0.02, seed, device="cuda")
        ref = qb.nf4_quantize(W)  # existing entry point, caller workspace
        out = qb.NF4Weight.empty(n, k)
        out.codes.fill_(0xEE)
        cw = out.c_struct()
        st = lib.nf4_quantize_static_ws(ctypes.c_void_p(W.data_ptr()), ctypes.byref(cw), stream)
        assert st == qb.QN_OK, lib.qn_last_error().decode()
        torch.cuda.synchronize()
        _same(out, ref)


def test_static_scratch_repeated_on_same_weight():
    W = synth.normal_bf16((1024, 2048), 0.02, 7, device="cuda")
    ref = qb.nf4_quantize(W)
    for _ in range(2):
        out = qb.nf4_quantize_static_ws(W, qb.NF4Weight.empty(1024, 2048))
        torch.cuda.synchronize()
        _same(out, ref)


def test_static_scratch_rejects_weights_above_the_limit():
    lib = qb.load()
    # 32768 x 16384 needs 32 MiB of scratch; rejected before anything is enqueued
    base = 0x10000000
    cw = qb.CWeight(32768, 16384, base, base + 0x1000000, base + 0x2000000, base + 0x3000000)
    st = lib.nf4_quantize_static_ws(ctypes.c_void_p(base + 0x4000000), ctypes.byref(cw), None)
    assert st == qb.QN_EWORKSPACE
    assert "static scratch" in lib.qn_last_error().decode()


def test_static_scratch_inside_a_stream_capture_allocates_nothing():
    # The case the entry point exists for: after one warm-up call (which resolves the scratch
    # address), a call captured into a CUDA graph and replayed gives the same bits as the
    # workspace entry point, and neither the capture nor the replays allocate device memory.
    n, k = 2048, 4096
    W = synth.student_t_bf16((n, k), 0.02, 41, device="cuda")
    ref = qb.nf4_quantize(W)
    out = qb.NF4Weight.empty(n, k)
    qb.nf4_quantize_static_ws(W, out)  # warm-up outside the capture
    torch.cuda.synchronize()
    out.codes.fill_(0)
    out.absmax_q.fill_(0)
    stream = torch.cuda.Stream()
    stream.wait_stream(torch.cuda.current_stream())
    graph = torch.cuda.CUDAGraph()
    free_before, _ = torch.cuda.mem_get_info()
    with torch.cuda.graph(graph, stream=stream):
        qb.nf4_quantize_static_ws(W, out, stream=stream)
    torch.cuda.synchronize()
    for _ in range(2):
        graph.replay()
        torch.cuda.synchronize()
        _same(out, ref)
    free_after, _ = torch.cuda.mem_get_info()
    # the graph's own bookkeeping may take a little device memory; the quantiser's scratch
    # (up to 16 MiB) must not appear as an allocation
    assert free_before - free_after < (8 << 20)
    del graph
