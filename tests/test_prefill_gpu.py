"""Chunked prefill on the GPU against the fp64 oracle.

Bar (floating point, bf16 tensor-core operands, fp32 accumulation and state):
for each of o, final_state and snapshots, max |x - ref| <= 2e-2 * max |ref|.
Placement is exact: a token, chunk or snapshot written to the wrong place
shows up as an O(1) relative error, far above that bound, and canary-filled
outputs must be fully overwritten.

Small cases run the oracle on everything; the full-size workloads run the
whole batch on the GPU and the oracle on a sample of heads.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads as wl
from gpu_util import assert_close_rel, rel_err

pytestmark = pytest.mark.gpu
TOL = 2e-2


def _gdr():
    import gated_delta_rule_150_b200 as gdr
    gdr.lib()
    return gdr


def _to(inp, dev):
    return {k: (v.to(dev) if torch.is_tensor(v) else v) for k, v in inp.items()}


def _gpu_prefill(inp, canary=True):
    gdr = _gdr()
    d = _to(inp, "cuda")
    T, H, dk = d["q"].shape
    dv = d["v"].shape[-1]
    n = d["cu_seqlens"].numel() - 1
    out = torch.full((T, H, dv), float("nan"), device="cuda", dtype=d["q"].dtype)
    fin = torch.full((n, H, dv, dk), float("nan"), device="cuda")
    ns = gdr.snapshot_count(inp["cu_seqlens"].cpu(), inp["snap_interval"]) if inp["snap_interval"] else 0
    snaps = torch.full((max(ns, 1), H, dv, dk), float("nan"), device="cuda")[:ns] if ns else None
    ws = torch.empty(gdr.workspace_size(n, H, dk, dv, T, inp["scalar_decay"]), dtype=torch.uint8,
                     device="cuda")
    o, fin, snaps = gdr.prefill(d["q"], d["k"], d["v"], d["beta"], d["log_a"], d["cu_seqlens"],
                                scalar_decay=inp["scalar_decay"], scale=inp["scale"],
                                init_state=d["init_state"], snap_interval=inp["snap_interval"],
                                cu_seqlens_host=inp["cu_seqlens"].cpu(), out=out, final_state=fin,
                                snapshots=snaps, workspace=ws)
    gdr.prefill_status(ws)
    torch.cuda.synchronize()
    assert not torch.isnan(o).any(), "o not fully written"
    assert not torch.isnan(fin).any(), "final state not fully written"
    if snaps is not None:
        assert not torch.isnan(snaps).any(), "snapshots not fully written"
    return o, fin, snaps


def _check(inp, o, fin, snaps, heads=None, what=""):
    sel = slice(None) if heads is None else heads

    def host(x):
        return None if x is None else x[:, sel].cpu()
    ref = oracle.prefill(host(inp["q"]), host(inp["k"]), host(inp["v"]), host(inp["beta"]),
                         host(inp["log_a"]), inp["cu_seqlens"].cpu(),
                         scalar_decay=inp["scalar_decay"], scale=inp["scale"],
                         init_state=host(inp["init_state"]), snap_interval=inp["snap_interval"])
    e = {"o": assert_close_rel(o[:, sel], ref["o"], TOL, f"{what} o"),
         "final": assert_close_rel(fin[:, sel], ref["final_state"], TOL, f"{what} final_state")}
    if inp["snap_interval"]:
        assert snaps.shape[0] == ref["snapshots"].shape[0]
        if snaps.shape[0]:
            e["snap"] = assert_close_rel(snaps[:, sel], ref["snapshots"], TOL, f"{what} snapshots")
    print(what, {k: f"{v:.2e}" for k, v in e.items()})
    return e


# ---------------------------------------------------------------------------
# intra-chunk factors against the oracle's chunked form
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("d,dtype,scalar", [(64, torch.bfloat16, False), (128, torch.bfloat16, False),
                                            (64, torch.float32, True), (128, torch.bfloat16, True)])
def test_chunk_factors(d, dtype, scalar):
    gdr = _gdr()
    w = wl.shrink(wl.GDN_LONG if scalar else wl.VARLEN, n_heads=2, d_k=d, d_v=d,
                  lengths=(130, 1, 64, 63), qkv_dtype=dtype, init_std=0.0, snap_interval=0,
                  scale=0.5)
    inp = wl.make_prefill_inputs(w)
    dv = _to(inp, "cuda")
    f = gdr.chunk_factors(dv["q"], dv["k"], dv["v"], dv["beta"], dv["log_a"], dv["cu_seqlens"],
                          scalar_decay=scalar, scale=w.scale)
    torch.cuda.synchronize()
    cu = inp["cu_seqlens"].tolist()
    names = ("Qt", "PU", "BS", "NC", "gamma")
    got = {k_: [] for k_ in names}
    ref = {k_: [] for k_ in names}
    for n in range(len(cu) - 1):
        for j, s in enumerate(range(cu[n], cu[n + 1], 64)):
            e = min(s + 64, cu[n + 1])
            slot = cu[n] // 64 + j + n
            L = e - s
            for h in range(2):
                r = oracle.chunk_factors(inp["q"], inp["k"], inp["v"], inp["beta"], inp["log_a"],
                                         s, e, h, scalar, w.scale)
                for name in ("Qt", "PU"):
                    got[name].append(f[name][slot, h, :L].cpu().double().numpy())
                    ref[name].append(r[name])
                    assert (f[name][slot, h, L:] == 0).all(), f"{name} rows past the chunk end"
                for name in ("BS", "NC"):
                    got[name].append(f[name][slot, h].cpu().double().numpy())
                    ref[name].append(r[name])
                got["gamma"].append(f["gamma"][slot, h].cpu().double().numpy())
                ref["gamma"].append(r["gamma_C"])
    # bound relative to the largest reference value of each factor over all chunks
    for name in names:
        g_ = np.concatenate([x.ravel() for x in got[name]])
        r_ = np.concatenate([x.ravel() for x in ref[name]])
        assert_close_rel(g_, r_, 1e-5 if name == "gamma" else TOL, name)


def test_chunk_factors_extreme_decay():
    """Per-channel log decay far below -10 in some channels: the factored
    tensor-core form would overflow, the exact path must take over."""
    gdr = _gdr()
    w = wl.shrink(wl.VARLEN, n_heads=1, d_k=64, d_v=64, lengths=(64, 40), init_std=0.0,
                  snap_interval=0)
    inp = wl.make_prefill_inputs(w)
    inp["log_a"][:, :, :5] = -30.0
    dv = _to(inp, "cuda")
    f = gdr.chunk_factors(dv["q"], dv["k"], dv["v"], dv["beta"], dv["log_a"], dv["cu_seqlens"])
    torch.cuda.synchronize()
    for slot, (s, e) in ((0, (0, 64)), (2, (64, 104))):
        ref = oracle.chunk_factors(inp["q"], inp["k"], inp["v"], inp["beta"], inp["log_a"], s, e, 0)
        for name in ("Qt", "PU", "BS", "NC"):
            assert torch.isfinite(f[name][slot]).all()
        assert_close_rel(f["Qt"][slot, 0, :e - s], ref["Qt"], TOL, "Qt")
        assert_close_rel(f["PU"][slot, 0, :e - s], ref["PU"], TOL, "PU")
        assert_close_rel(f["BS"][slot, 0], ref["BS"], TOL, "BS")
        assert_close_rel(f["NC"][slot, 0], ref["NC"], TOL, "NC")
    o, fin, _ = _gpu_prefill(inp)
    _check(inp, o, fin, None, what="extreme decay")


@pytest.mark.parametrize("d,heads,chunks", [(64, 8, 150), (128, 4, 100)])
def test_extreme_decay_many_items_per_cta(d, heads, chunks):
    """More chunk-heads than CTAs, so each persistent CTA runs several, with
    every third chunk carrying a log decay of -30 in a few channels: the
    exact path and the flag carried from one item's scan to the next."""
    w = wl.shrink(wl.VARLEN, n_heads=heads, d_k=d, d_v=d, lengths=(64 * chunks,), init_std=0.1,
                  snap_interval=0)
    inp = wl.make_prefill_inputs(w)
    for c in range(0, chunks, 3):
        inp["log_a"][64 * c + 10: 64 * c + 20, :, 3:7] = -30.0
    o, fin, _ = _gpu_prefill(inp)
    _check(inp, o, fin, None, what=f"extreme decay d{d}")


# ---------------------------------------------------------------------------
# whole prefill
# ---------------------------------------------------------------------------
def test_tiny_kda_full():
    inp = wl.make_prefill_inputs(wl.TINY_KDA)
    o, fin, s = _gpu_prefill(inp)
    _check(inp, o, fin, s, what="tiny_kda")


def test_graft_layer_full():
    inp = wl.make_prefill_inputs(wl.GRAFT_LAYER)
    o, fin, s = _gpu_prefill(inp)
    _check(inp, o, fin, s, what="graft_layer")


@pytest.mark.parametrize("d,dtype,scalar,snap", [(64, torch.bfloat16, False, 128),
                                                 (128, torch.bfloat16, False, 64),
                                                 (128, torch.bfloat16, True, 192),
                                                 (64, torch.float32, True, 0),
                                                 (128, torch.float32, False, 128)])
def test_ragged_varlen(d, dtype, scalar, snap):
    """Several tiles, ragged tails, empty and one-token sequences, initial states."""
    base = wl.GDN_LONG if scalar else wl.VARLEN
    w = wl.shrink(base, n_heads=3, d_k=d, d_v=d, lengths=(300, 0, 1, 64, 129, 257, 63, 512),
                  qkv_dtype=dtype, init_std=0.1, snap_interval=snap, scale=0.8)
    inp = wl.make_prefill_inputs(w)
    o, fin, s = _gpu_prefill(inp)
    _check(inp, o, fin, s, what=f"ragged d{d} {dtype} scalar={scalar}")


@pytest.mark.parametrize("d,scalar,snap", [(64, False, 256), (128, False, 128), (128, True, 0),
                                           (64, True, 512)])
def test_segmented_pass(d, scalar, snap):
    """Few (sequence, head) pairs and long sequences: the sequential pass is
    cut into segments (zero-state pass with the identity, fp32 chaining of the
    segment maps, replay).  Ragged segment tails, an empty and a short
    sequence, initial states and snapshots across segment boundaries."""
    base = wl.GDN_LONG if scalar else wl.VARLEN
    w = wl.shrink(base, n_heads=1, d_k=d, d_v=d, lengths=(2000, 0, 700, 1536, 65),
                  init_std=0.1, snap_interval=snap, scale=0.9)
    inp = wl.make_prefill_inputs(w)
    import gated_delta_rule_150_b200 as gdr
    o, fin, s = _gpu_prefill(inp)
    _check(inp, o, fin, s, what=f"segmented d{d} scalar={scalar}")


def test_all_empty_sequences_copy_init():
    w = wl.shrink(wl.VARLEN, n_heads=2, d_k=64, d_v=64, lengths=(0, 0, 0), init_std=0.1,
                  snap_interval=0)
    inp = wl.make_prefill_inputs(w)
    o, fin, _ = _gpu_prefill(inp)
    assert torch.equal(fin.cpu(), inp["init_state"])


def test_init_may_alias_final():
    gdr = _gdr()
    w = wl.shrink(wl.VARLEN, n_heads=2, d_k=64, d_v=64, lengths=(200, 77), init_std=0.1,
                  snap_interval=0)
    inp = wl.make_prefill_inputs(w)
    d = _to(inp, "cuda")
    st = d["init_state"].clone()
    o, fin, _ = gdr.prefill(d["q"], d["k"], d["v"], d["beta"], d["log_a"], d["cu_seqlens"],
                            init_state=st, final_state=st)
    torch.cuda.synchronize()
    _check(inp, o, fin, None, what="aliased state")


def test_split_prefill_equals_one_shot():
    """Prefill of [0, N) then [N, T) with the carried state equals one prefill."""
    gdr = _gdr()
    w = wl.shrink(wl.GRAFT_LAYER, n_heads=4, lengths=(1000,))
    inp = wl.make_prefill_inputs(w)
    d = _to(inp, "cuda")
    o_full, f_full, _ = gdr.prefill(d["q"], d["k"], d["v"], d["beta"], d["log_a"], d["cu_seqlens"])
    N = 448
    cu1 = torch.tensor([0, N], dtype=torch.int32, device="cuda")
    cu2 = torch.tensor([0, 1000 - N], dtype=torch.int32, device="cuda")
    o1, f1, _ = gdr.prefill(d["q"][:N], d["k"][:N], d["v"][:N], d["beta"][:N], d["log_a"][:N], cu1)
    o2, f2, _ = gdr.prefill(d["q"][N:].contiguous(), d["k"][N:].contiguous(), d["v"][N:].contiguous(),
                            d["beta"][N:].contiguous(), d["log_a"][N:].contiguous(), cu2, init_state=f1)
    torch.cuda.synchronize()
    ref = oracle.prefill(inp["q"], inp["k"], inp["v"], inp["beta"], inp["log_a"], inp["cu_seqlens"])
    assert_close_rel(torch.cat([o1, o2]), ref["o"], TOL, "split o")
    assert_close_rel(f2, ref["final_state"], TOL, "split final")
    assert rel_err(torch.cat([o1, o2]), o_full.cpu().double().numpy()) < TOL


def test_chained_prefills_consume_previous_outputs():
    """Two prefills back to back on one stream, no host sync between: the
    second reads the first's o (as q and v) and final state (as its initial
    state), the way stacked layers would.  Its kernels may be scheduled while
    the first one drains, so this checks that they wait for its results."""
    gdr = _gdr()
    w = wl.shrink(wl.GRAFT_LAYER, n_heads=4, lengths=(700, 300))
    inp = wl.make_prefill_inputs(w)
    d = _to(inp, "cuda")
    o1, f1, _ = gdr.prefill(d["q"], d["k"], d["v"], d["beta"], d["log_a"], d["cu_seqlens"])
    o2, f2, _ = gdr.prefill(o1, d["k"], o1, d["beta"], d["log_a"], d["cu_seqlens"], init_state=f1)
    torch.cuda.synchronize()
    ref = oracle.prefill(o1.cpu(), inp["k"], o1.cpu(), inp["beta"], inp["log_a"], inp["cu_seqlens"],
                         init_state=f1.cpu())
    assert_close_rel(o2, ref["o"], TOL, "chained o")
    assert_close_rel(f2, ref["final_state"], TOL, "chained final")


def test_decode_steps_continue_prefill():
    """Decode steps after a prefill equal a longer prefill (same recurrence)."""
    gdr = _gdr()
    w = wl.shrink(wl.GRAFT_LAYER, n_heads=2, lengths=(200,))
    inp = wl.make_prefill_inputs(w)
    d = _to(inp, "cuda")
    P = 190
    cu = torch.tensor([0, P], dtype=torch.int32, device="cuda")
    _, S, _ = gdr.prefill(d["q"][:P], d["k"][:P], d["v"][:P], d["beta"][:P], d["log_a"][:P], cu)
    outs = []
    for t in range(P, 200):
        outs.append(gdr.decode_step(S, d["q"][t:t + 1], d["k"][t:t + 1], d["v"][t:t + 1],
                                    d["beta"][t:t + 1], d["log_a"][t:t + 1]))
    torch.cuda.synchronize()
    ref = oracle.prefill(inp["q"], inp["k"], inp["v"], inp["beta"], inp["log_a"], inp["cu_seqlens"])
    assert_close_rel(torch.cat(outs), ref["o"][P:], TOL, "decode o after prefill")
    assert_close_rel(S, ref["final_state"], TOL, "state after prefill + decode")


def test_gdn_long_full_size_sampled_heads():
    """65 536 tokens x 16 heads x d 128, scalar decay, snapshots every 4096."""
    inp = wl.make_prefill_inputs(wl.GDN_LONG, draw_device="cuda", device="cuda")
    o, fin, s = _gpu_prefill(inp)
    _check(inp, o, fin, s, heads=[0, 5, 11, 15], what="gdn_long")


def test_varlen_full_size_sampled_heads():
    """32 sequences of 1024..16384 tokens, 32 heads x d 128, initial states."""
    inp = wl.make_prefill_inputs(wl.VARLEN, draw_device="cuda", device="cuda")
    o, fin, s = _gpu_prefill(inp)
    _check(inp, o, fin, s, heads=[0, 5, 17, 31], what="varlen")


@pytest.mark.parametrize("dk,dv,scalar,lengths,heads,snap", [
    (64, 128, False, (300, 0, 129, 512, 64), 3, 128),     # one pass, wider values
    (128, 64, False, (300, 1, 257, 700), 3, 64),          # one pass, wider keys
    (64, 128, True, (2000, 700), 1, 256),                 # segmented, scalar gate
    (128, 64, True, (3000, 65), 1, 0),                    # segmented, scalar gate
    (128, 64, False, (1800, 0, 900), 1, 512),             # segmented, per-channel gate
])
def test_mixed_key_and_value_widths(dk, dv, scalar, lengths, heads, snap):
    """d_k != d_v: o [T, H, d_v], states [N, H, d_v, d_k], snapshots, against
    the oracle's rectangular recurrence."""
    base = wl.GDN_LONG if scalar else wl.VARLEN
    w = wl.shrink(base, n_heads=heads, d_k=dk, d_v=dv, lengths=lengths, init_std=0.1,
                  snap_interval=snap, scale=0.9)
    inp = wl.make_prefill_inputs(w)
    o, fin, s = _gpu_prefill(inp)
    assert tuple(o.shape) == (sum(lengths), heads, dv)
    assert tuple(fin.shape) == (len(lengths), heads, dv, dk)
    _check(inp, o, fin, s, what=f"d_k {dk} d_v {dv} scalar={scalar}")


@pytest.mark.parametrize("dk,dv", [(64, 128), (128, 64)])
def test_mixed_widths_with_output_epilogue(dk, dv):
    gdr = _gdr()
    w = wl.shrink(wl.VARLEN, n_heads=2, d_k=dk, d_v=dv, lengths=(300, 129), init_std=0.1,
                  snap_interval=0)
    inp = wl.make_prefill_inputs(w)
    g = wl.make_output_gate(inp["q"].shape[0], 2, dv, inp["q"].dtype, seed=88)
    d = _to(inp, "cuda")
    y, _, _ = gdr.prefill(d["q"], d["k"], d["v"], d["beta"], d["log_a"], d["cu_seqlens"],
                          init_state=d["init_state"], gate_raw=g["gate_raw"].cuda(),
                          norm_weight=g["norm_weight"].cuda(), norm_eps=1e-6)
    torch.cuda.synchronize()
    ref = oracle.prefill(inp["q"], inp["k"], inp["v"], inp["beta"], inp["log_a"],
                         inp["cu_seqlens"], init_state=inp["init_state"])
    y_ref = oracle.output_epilogue(ref["o"], g["gate_raw"], g["norm_weight"], 1e-6)
    assert_close_rel(y, y_ref, TOL, f"gated o, d_k {dk} d_v {dv}")
