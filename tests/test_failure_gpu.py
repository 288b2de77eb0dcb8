"""Failure detection without a GPU fault.

Every wait inside the prefill kernels is bounded; a wait that runs out sets
the workspace's error word, the CTA stops issuing work, waits (again with a
limit) for what it has in flight, releases its tensor memory and returns,
and gdr_prefill_status reports GDR_ERR_TIMEOUT.  Nothing here hangs or faults
the GPU:

* the status mapping is checked by writing the error word from the host;
* a test-only copy of the library (build.build_wait_test) makes the state-pass
  kernels wait for a barrier nothing arrives on, with a 1 ms limit, so the
  timeout path runs for real; its copy waits keep the regular limit, and a
  regular prefill on the same workspace afterwards must succeed with correct
  results (the context stays usable).
"""
import ctypes

import pytest
import torch

import oracle
import workloads as wl
from gpu_util import assert_close_rel

pytestmark = pytest.mark.gpu
TOL = 2e-2
TIMEOUT = 5


def _gdr():
    import gated_delta_rule_150_b200 as gdr
    gdr.lib()
    return gdr


def _wait_test_lib(gdr):
    from gated_delta_rule_150_b200 import build as gdr_build
    L = ctypes.CDLL(gdr_build.build_wait_test())
    L.gdr_prefill.restype = ctypes.c_int
    L.gdr_prefill.argtypes = [ctypes.POINTER(gdr.PrefillArgs), ctypes.c_void_p]
    L.gdr_prefill_status.restype = ctypes.c_int
    L.gdr_prefill_status.argtypes = [ctypes.c_void_p, ctypes.c_void_p]
    L.gdr_prefill_static_workspace.restype = ctypes.c_int
    L.gdr_prefill_static_workspace.argtypes = [ctypes.POINTER(gdr.PrefillArgs), ctypes.c_void_p]
    L.gdr_prefill_static_status.restype = ctypes.c_int
    L.gdr_prefill_static_status.argtypes = [ctypes.c_void_p]
    return L


def _case(lengths, heads, d=64):
    w = wl.shrink(wl.VARLEN, n_heads=heads, d_k=d, d_v=d, lengths=lengths, init_std=0.1,
                  snap_interval=0)
    inp = wl.make_prefill_inputs(w)
    dev = {k: (v.cuda() if torch.is_tensor(v) else v) for k, v in inp.items()}
    return inp, dev


def _buffers(gdr, dev):
    T, H, dk = dev["q"].shape
    n = dev["cu_seqlens"].numel() - 1
    o = torch.empty(T, H, dk, dtype=dev["q"].dtype, device="cuda")
    fin = torch.empty(n, H, dk, dk, device="cuda")
    ws = torch.empty(gdr.workspace_size(n, H, dk, dk, T), dtype=torch.uint8, device="cuda")
    return o, fin, ws


def _args(gdr, dev, o, fin, ws):
    return gdr._prefill_args(dev["q"], dev["k"], dev["v"], dev["beta"], dev["log_a"],
                             dev["cu_seqlens"], False, 1.0, dev["init_state"], 0, o, fin, None, ws)


def test_status_reads_the_error_word():
    gdr = _gdr()
    ws = torch.zeros(4096, dtype=torch.uint8, device="cuda")
    st = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    L = gdr.lib()
    assert L.gdr_prefill_status(ctypes.c_void_p(ws.data_ptr()), st) == 0
    ws[:4].view(torch.int32).fill_(1)
    assert L.gdr_prefill_status(ctypes.c_void_p(ws.data_ptr()), st) == TIMEOUT
    ws[:4].view(torch.int32).fill_(0)
    assert L.gdr_prefill_status(ctypes.c_void_p(ws.data_ptr()), st) == 0
    assert L.gdr_prefill_status(None, st) == 1


@pytest.mark.parametrize("lengths,heads,d", [((640, 300, 100), 4, 64),     # one pass (kFull)
                                             ((3000,), 1, 64),              # segmented pass
                                             ((640, 300, 100), 4, 128),    # d 128: records in two parts
                                             ((3000,), 1, 128)])
def test_timed_out_wait_is_reported_and_context_stays_usable(lengths, heads, d):
    gdr = _gdr()
    LW = _wait_test_lib(gdr)
    inp, dev = _case(lengths, heads, d)
    o, fin, ws = _buffers(gdr, dev)
    st = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    wsp = ctypes.c_void_p(ws.data_ptr())
    a = _args(gdr, dev, o, fin, ws)
    assert LW.gdr_prefill(ctypes.byref(a), st) == 0            # enqueued fine ...
    assert LW.gdr_prefill_status(wsp, st) == TIMEOUT           # ... but a wait gave up
    # the regular library on the same workspace: the error word is cleared
    # first, and the results are right
    L = gdr.lib()
    assert L.gdr_prefill(ctypes.byref(a), st) == 0
    assert L.gdr_prefill_status(wsp, st) == 0
    torch.cuda.synchronize()
    ref = oracle.prefill(inp["q"], inp["k"], inp["v"], inp["beta"], inp["log_a"],
                         inp["cu_seqlens"], init_state=inp["init_state"])
    assert_close_rel(o, ref["o"], TOL, "o after a timed-out call")
    assert_close_rel(fin, ref["final_state"], TOL, "final state after a timed-out call")


def test_static_workspace_status_reports_a_timeout():
    gdr = _gdr()
    LW = _wait_test_lib(gdr)
    inp, dev = _case((640, 300), 2)
    o, fin, ws = _buffers(gdr, dev)
    st = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    a = _args(gdr, dev, o, fin, ws)
    assert LW.gdr_prefill_static_workspace(ctypes.byref(a), st) == 0
    assert LW.gdr_prefill_static_status(st) == TIMEOUT
