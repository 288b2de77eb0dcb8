"""Prefix snapshots: per-sequence offsets and offload to host memory.

"Modele hybrydowe", section "Co stan rekurencyjny zmienia przy serwowaniu",
point 1: a request that extends a stored prompt prefix resumes from the state
snapshot taken at the prefix's end, and the fork keeps such checkpoints in
host memory, saved without stalling prefill.

* gdr_snapshot_offsets locates sequence n's m-th snapshot; passing the
  offsets to the kernels changes nothing (bitwise), and the snapshot found
  through them equals the oracle's state after that prefix.
* Snapshots written into page-locked host memory by the state-pass kernel
  are bitwise the ones written to device memory, and match the oracle.
"""
import pytest
import torch

import oracle
import workloads as wl
from gpu_util import assert_close_rel

pytestmark = pytest.mark.gpu
TOL = 2e-2


def _gdr():
    import gated_delta_rule_150_b200 as gdr
    gdr.lib()
    return gdr


def _run(gdr, d, inp, snaps, snap_offsets=None):
    cu_host = inp["cu_seqlens"]
    o, fin, s = gdr.prefill(d["q"], d["k"], d["v"], d["beta"], d["log_a"], d["cu_seqlens"],
                            scalar_decay=inp["scalar_decay"], init_state=d["init_state"],
                            snap_interval=inp["snap_interval"], cu_seqlens_host=cu_host,
                            snapshots=snaps, snap_offsets=snap_offsets)
    return o, fin, s


@pytest.mark.parametrize("d,scalar,heads,lengths", [
    (64, False, 3, (300, 0, 129, 1024, 64, 700)),       # one pass over many pairs
    (128, True, 1, (2000, 0, 700, 1536, 65)),           # segmented pass
])
def test_offsets_locate_each_sequences_snapshots(d, scalar, heads, lengths):
    gdr = _gdr()
    base = wl.GDN_LONG if scalar else wl.VARLEN
    w = wl.shrink(base, n_heads=heads, d_k=d, d_v=d, lengths=lengths, init_std=0.1,
                  snap_interval=128)
    inp = wl.make_prefill_inputs(w)
    dd = {k: (v.cuda() if torch.is_tensor(v) else v) for k, v in inp.items()}
    offs = gdr.snapshot_offsets(inp["cu_seqlens"], 128)
    ns = int(offs[-1])
    H, dk = inp["q"].shape[1], inp["q"].shape[2]
    a = torch.full((ns, H, d, dk), float("nan"), device="cuda")
    b = torch.full((ns, H, d, dk), float("nan"), device="cuda")
    o1, f1, _ = _run(gdr, dd, inp, a)
    o2, f2, _ = _run(gdr, dd, inp, b, snap_offsets=offs.cuda())
    torch.cuda.synchronize()
    assert torch.equal(a, b) and torch.equal(o1, o2) and torch.equal(f1, f2)
    # sequence n's m-th snapshot is the state after its first 128 m tokens
    cu = inp["cu_seqlens"].tolist()
    for n in range(len(lengths)):
        for m in range(1, lengths[n] // 128 + 1, 3):
            s, e = cu[n], cu[n] + 128 * m
            ref = oracle.prefill(*(inp[x][s:e] for x in ("q", "k", "v", "beta", "log_a")),
                                 torch.tensor([0, e - s], dtype=torch.int32),
                                 scalar_decay=scalar,
                                 init_state=inp["init_state"][n:n + 1])
            assert_close_rel(b[int(offs[n]) + m - 1], ref["final_state"][0], TOL,
                             f"sequence {n} snapshot {m}")


@pytest.mark.parametrize("d,scalar,heads,lengths,iv", [
    (64, False, 2, (640, 0, 1000, 64), 64),              # one pass
    (128, True, 1, (4096 + 100, 3000), 512),             # segmented pass
])
def test_snapshots_offloaded_to_pinned_host_memory(d, scalar, heads, lengths, iv):
    gdr = _gdr()
    base = wl.GDN_LONG if scalar else wl.VARLEN
    w = wl.shrink(base, n_heads=heads, d_k=d, d_v=d, lengths=lengths, init_std=0.1,
                  snap_interval=iv)
    inp = wl.make_prefill_inputs(w)
    dd = {k: (v.cuda() if torch.is_tensor(v) else v) for k, v in inp.items()}
    ns = gdr.snapshot_count(inp["cu_seqlens"], iv)
    H, dk = inp["q"].shape[1], inp["q"].shape[2]
    dev = torch.full((ns, H, d, dk), float("nan"), device="cuda")
    host = torch.full((ns, H, d, dk), float("nan")).pin_memory()
    _, fd, _ = _run(gdr, dd, inp, dev)
    _, fh, _ = _run(gdr, dd, inp, host)
    torch.cuda.synchronize()
    assert not torch.isnan(host).any()
    assert torch.equal(host, dev.cpu()) and torch.equal(fd, fh)
    ref = oracle.prefill(inp["q"], inp["k"], inp["v"], inp["beta"], inp["log_a"],
                         inp["cu_seqlens"], scalar_decay=scalar, init_state=inp["init_state"],
                         snap_interval=iv)
    assert_close_rel(host, ref["snapshots"], TOL, "offloaded snapshots")


def test_pageable_host_snapshots_rejected():
    gdr = _gdr()
    w = wl.shrink(wl.VARLEN, n_heads=1, d_k=64, d_v=64, lengths=(256,), init_std=0.0,
                  snap_interval=64)
    inp = wl.make_prefill_inputs(w)
    dd = {k: (v.cuda() if torch.is_tensor(v) else v) for k, v in inp.items()}
    a = gdr.PrefillArgs()
    T, H, dk = inp["q"].shape
    o = torch.empty(T, H, 64, dtype=inp["q"].dtype, device="cuda")
    fin = torch.empty(1, H, 64, dk, device="cuda")
    snaps = torch.empty(4, H, 64, dk)                      # pageable
    ws = torch.empty(gdr.workspace_size(1, H, dk, 64, T), dtype=torch.uint8, device="cuda")
    a = gdr._prefill_args(dd["q"], dd["k"], dd["v"], dd["beta"], dd["log_a"], dd["cu_seqlens"],
                          False, 1.0, None, 64, o, fin, snaps, ws)
    st = torch.cuda.current_stream().cuda_stream
    import ctypes
    assert gdr.lib().gdr_prefill(ctypes.byref(a), ctypes.c_void_p(st)) == 1


def test_snapshot_offload_on_copy_stream():
    """gdr_snapshot_offload: the copy runs on its own stream after the
    prefill that wrote the snapshots; the host copy equals the device
    snapshots bitwise and matches the oracle, while a second prefill (other
    buffers) is enqueued on the compute stream without waiting for it."""
    gdr = _gdr()
    w = wl.shrink(wl.GDN_LONG, n_heads=2, d_k=128, d_v=128, lengths=(4096 + 100, 3000),
                  init_std=0.1, snap_interval=512)
    inp = wl.make_prefill_inputs(w)
    dd = {k: (v.cuda() if torch.is_tensor(v) else v) for k, v in inp.items()}
    ns = gdr.snapshot_count(inp["cu_seqlens"], 512)
    H, dk = inp["q"].shape[1], inp["q"].shape[2]
    dev = [torch.full((ns, H, 128, dk), float("nan"), device="cuda") for _ in range(2)]
    host = torch.full((ns, H, 128, dk), float("nan")).pin_memory()
    copy_stream, ev = torch.cuda.Stream(), torch.cuda.Event()
    _run(gdr, dd, inp, dev[0])
    gdr.snapshot_offload(dev[0], host, copy_stream, ev)
    _run(gdr, dd, inp, dev[1])                   # does not wait for the copy
    copy_stream.synchronize()
    torch.cuda.synchronize()
    assert torch.equal(host, dev[0].cpu()) and torch.equal(dev[0], dev[1])
    ref = oracle.prefill(inp["q"], inp["k"], inp["v"], inp["beta"], inp["log_a"],
                         inp["cu_seqlens"], scalar_decay=True, init_state=inp["init_state"],
                         snap_interval=512)
    assert_close_rel(host, ref["snapshots"], TOL, "snapshots copied on the copy stream")
