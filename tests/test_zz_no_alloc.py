"""gdr_prefill_static_workspace: the prefill for callers that cannot allocate
device memory (graph capture, host frameworks that own allocation, serving
paths where allocation is forbidden).  It uses a fixed array inside the
library instead of a caller workspace.

Called through the C ABI twice in a row with different inputs; each result
must equal gdr_prefill's on the same inputs bit for bit (both run the same
kernels on the same inputs), and gdr_prefill_static_status must report that
the kernels completed.  A CUDA graph captured around the call (after a first
call outside capture) replays on new inputs with the same results.  The file
sorts last so that a run stopping at the first failure has run every other
test before it.
"""
import ctypes

import numpy as np
import pytest
import torch

import workloads as wl

pytestmark = pytest.mark.gpu
TOL = 2e-2          # the prefill bound used by tests/test_prefill_gpu.py


def _lib():
    import gated_delta_rule_150_b200 as gdr
    L = gdr.lib()
    L.gdr_prefill_static_workspace.restype = ctypes.c_int
    L.gdr_prefill_static_workspace.argtypes = [ctypes.POINTER(gdr.PrefillArgs), ctypes.c_void_p]
    L.gdr_prefill_static_status.restype = ctypes.c_int
    L.gdr_prefill_static_status.argtypes = [ctypes.c_void_p]
    return gdr, L


def _args(gdr, d, out, fin, ws=None):
    a = gdr.PrefillArgs()
    T, H, dk = d["q"].shape
    a.n_seqs = d["cu_seqlens"].numel() - 1
    a.n_heads, a.d_k, a.d_v, a.total_tokens = H, dk, d["v"].shape[-1], T
    a.cu_seqlens = d["cu_seqlens"].data_ptr()
    a.qkv_dtype = 0 if d["q"].dtype == torch.bfloat16 else 1
    a.q, a.k, a.v = d["q"].data_ptr(), d["k"].data_ptr(), d["v"].data_ptr()
    a.beta, a.log_a = d["beta"].data_ptr(), d["log_a"].data_ptr()
    a.scalar_decay = int(d["scalar_decay"])
    a.scale = 1.0
    a.init_state = None if d["init_state"] is None else d["init_state"].data_ptr()
    a.o, a.final_state = out.data_ptr(), fin.data_ptr()
    if ws is not None:
        a.workspace, a.workspace_bytes = ws.data_ptr(), ws.numel()
    return a


def _inputs(seed, lengths, scalar):
    base = wl.GDN_LONG if scalar else wl.VARLEN
    w = wl.shrink(base, seed=seed, n_heads=3, d_k=64, d_v=64, lengths=lengths,
                  init_std=0.1, snap_interval=0)
    inp = wl.make_prefill_inputs(w, device="cuda")
    return inp


def _rel(x, ref):
    x, ref = x.double().cpu().numpy(), ref.double().cpu().numpy()
    return float(np.abs(x - ref).max() / np.abs(ref).max())


def test_static_workspace_matches_prefill_twice():
    gdr, L = _lib()
    st = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    cases = [_inputs(4242, (300, 1, 129), False), _inputs(4343, (77, 256, 0, 64), True)]
    for d in cases:
        T, H, dk = d["q"].shape
        n = d["cu_seqlens"].numel() - 1
        # the existing entry point, with a torch-allocated workspace
        o_ref = torch.empty(T, H, 64, dtype=d["q"].dtype, device="cuda")
        f_ref = torch.empty(n, H, 64, dk, device="cuda")
        ws = torch.empty(gdr.workspace_size(n, H, dk, 64, T, d["scalar_decay"]),
                         dtype=torch.uint8, device="cuda")
        assert L.gdr_prefill(ctypes.byref(_args(gdr, d, o_ref, f_ref, ws)), st) == 0
        # the no-allocation entry point
        o = torch.full_like(o_ref, float("nan"))
        f = torch.full_like(f_ref, float("nan"))
        assert L.gdr_prefill_static_workspace(ctypes.byref(_args(gdr, d, o, f)), st) == 0
        assert L.gdr_prefill_static_status(st) == 0          # no kernel gave up a wait
        torch.cuda.synchronize()
        assert not torch.isnan(o).any() and not torch.isnan(f).any()
        assert torch.equal(o, o_ref) and torch.equal(f, f_ref)
        assert _rel(o, o_ref) <= TOL and _rel(f, f_ref) <= TOL


def test_static_workspace_under_graph_capture():
    """The caller this entry point exists for: code captured into a CUDA
    graph, where no allocation may happen.  One call outside capture first,
    then capture, then replay on inputs copied into the captured buffers."""
    gdr, L = _lib()
    first = _inputs(4545, (300, 129), False)
    second = _inputs(4646, (300, 129), False)
    T, H, dk = first["q"].shape
    n = first["cu_seqlens"].numel() - 1
    o = torch.empty(T, H, 64, dtype=first["q"].dtype, device="cuda")
    f = torch.empty(n, H, 64, dk, device="cuda")
    a = _args(gdr, first, o, f)
    st = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    assert L.gdr_prefill_static_workspace(ctypes.byref(a), st) == 0
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        cap = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
        assert L.gdr_prefill_static_workspace(ctypes.byref(a), cap) == 0
    for name in ("q", "k", "v", "beta", "log_a", "init_state"):
        first[name].copy_(second[name])
    g.replay()
    torch.cuda.synchronize()
    assert L.gdr_prefill_static_status(st) == 0
    o_ref = torch.empty_like(o)
    f_ref = torch.empty_like(f)
    ws = torch.empty(gdr.workspace_size(n, H, dk, 64, T, 0), dtype=torch.uint8, device="cuda")
    assert L.gdr_prefill(ctypes.byref(_args(gdr, second, o_ref, f_ref, ws)), st) == 0
    torch.cuda.synchronize()
    assert torch.equal(o, o_ref) and torch.equal(f, f_ref)
    del g


def test_static_workspace_rejects_oversized_request():
    gdr, L = _lib()
    d = _inputs(4444, (64,), False)
    a = _args(gdr, d, torch.empty(1, device="cuda"), torch.empty(1, device="cuda"))
    a.total_tokens = 1 << 20              # needs far more than the fixed array
    assert L.gdr_prefill_static_workspace(ctypes.byref(a), None) == 3   # GDR_ERR_WORKSPACE
