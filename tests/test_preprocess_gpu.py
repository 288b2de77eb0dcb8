"""Input activations (conv-4, L2 norm, gates) on the GPU against the fp64
oracle.

Tolerances, per element, with M = max |ref| of the tensor: q, k, v within
2^-8 |ref| + 1e-5 M when they are bf16 (one bf16 rounding of an fp32 result)
and 1e-6 |ref| + 1e-5 M when fp32 (fp32 conv sums); beta and log a (fp32)
within 2e-6 |ref| + 2e-6 (fp32 rounding of the biased gate, expf / log1pf)."""
import numpy as np
import pytest
import torch

import oracle
import workloads as wl

pytestmark = pytest.mark.gpu


def _gdr():
    import gated_delta_rule_150_b200 as gdr
    gdr.lib()
    return gdr


ARGS = ("xq", "xk", "xv", "conv_q", "conv_k", "conv_v", "beta_raw", "a_raw", "a_bias",
        "cu_seqlens")


def _check(out, ref, bf16):
    for name in ("q", "k", "v"):
        x = out[name].double().cpu().numpy()
        r = ref[name]
        M = np.abs(r).max() if r.size else 0.0
        rel = 2.0 ** -8 if bf16 else 1e-6
        bad = np.abs(x - r) > rel * np.abs(r) + 1e-5 * M
        assert not bad.any(), f"{name}: {bad.sum()} elements out of bound, max err {np.abs(x - r).max():.3e}"
    for name in ("beta", "log_a"):
        x = out[name].double().cpu().numpy()
        r = ref[name]
        bad = np.abs(x - r) > 2e-6 * np.abs(r) + 2e-6
        assert not bad.any(), f"{name}: max err {np.abs(x - r).max():.3e}"


def _run(w, lengths=None):
    gdr = _gdr()
    inp = wl.make_preprocess_inputs(w, lengths=lengths)
    d = {k: (v.cuda() if torch.is_tensor(v) else v) for k, v in inp.items()}
    out = gdr.preprocess(*(d[a] for a in ARGS), scalar_decay=w.scalar_decay)
    torch.cuda.synchronize()
    ref = oracle.preprocess(*(inp[a] for a in ARGS), scalar_decay=w.scalar_decay)
    _check(out, ref, w.qkv_dtype == torch.bfloat16)
    return inp, out


def test_preprocess_graft_layer_full():
    """The graft layer's shape (8192 tokens x 14 heads x 64, bf16), every
    output element checked."""
    _run(wl.PREPROCESS)


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("scalar", [False, True])
def test_preprocess_ragged(d, dtype, scalar):
    """Sequences shorter than the conv (1, 2, 3 tokens), an empty one, one
    across a warp's worth of units, several heads."""
    w = wl.shrink(wl.PREPROCESS, n_heads=3, d_k=d, d_v=d, qkv_dtype=dtype, scalar_decay=scalar,
                  seed=1107)
    _run(w, lengths=[1, 2, 3, 0, 70, 5])


def test_preprocess_feeds_prefill():
    """The activations go straight into the prefill: the chain matches the
    oracle's prefill of the oracle's activations (cast to the kernel's
    dtype) within the prefill tolerance 2e-2 max |ref|."""
    gdr = _gdr()
    w = wl.shrink(wl.PREPROCESS, n_heads=2, seed=1108)
    lengths = [200, 77]
    inp = wl.make_preprocess_inputs(w, lengths=lengths)
    d = {k: (v.cuda() if torch.is_tensor(v) else v) for k, v in inp.items()}
    act = gdr.preprocess(*(d[a] for a in ARGS))
    o, fin, _ = gdr.prefill(act["q"], act["k"], act["v"], act["beta"], act["log_a"],
                            d["cu_seqlens"])
    torch.cuda.synchronize()
    ref_act = oracle.preprocess(*(inp[a] for a in ARGS))
    cast = {n: torch.from_numpy(ref_act[n]).to(torch.bfloat16) for n in ("q", "k", "v")}
    ref = oracle.prefill(cast["q"], cast["k"], cast["v"], ref_act["beta"], ref_act["log_a"],
                         inp["cu_seqlens"])
    for name, x, r in (("o", o, ref["o"]), ("final_state", fin, ref["final_state"])):
        err = np.abs(x.double().cpu().numpy() - r).max() / np.abs(r).max()
        assert err <= 2e-2, f"{name}: {err:.3e}"


def test_preprocess_no_tokens_is_noop():
    gdr = _gdr()
    w = wl.shrink(wl.PREPROCESS, n_heads=2, seed=1109)
    inp = wl.make_preprocess_inputs(w, lengths=[0, 0])
    d = {k: (v.cuda() if torch.is_tensor(v) else v) for k, v in inp.items()}
    out = gdr.preprocess(*(d[a] for a in ARGS))
    assert out["q"].shape == (0, 2, 64)


def _fused_vs_chain(w, lengths, snap=0, init=False, steep=None, minimal_ws=False):
    """The fused prefill from raw projections against (a) the oracle's prefill
    of the oracle's activations (cast to bf16) at the prefill bound 2e-2 max
    |ref|, and (b) the two-kernel chain preprocess -> prefill.  ``steep``:
    (tokens, channels) whose a_raw is set to -40 (log a near -35)."""
    gdr = _gdr()
    inp = wl.make_preprocess_inputs(w, lengths=lengths)
    if steep is not None:
        toks, chans = steep
        for t in toks:
            if w.scalar_decay:
                inp["a_raw"][t, :] = -40.0
            else:
                inp["a_raw"][t, :, chans] = -40.0
    d = {k: (v.cuda() if torch.is_tensor(v) else v) for k, v in inp.items()}
    H, dd = w.n_heads, w.d_k
    n = len(inp["lengths"])
    init_state = (0.1 * torch.randn(n, H, dd, dd, generator=torch.Generator().manual_seed(5))
                  if init else None)
    ini = None if init_state is None else init_state.cuda()
    kw = dict(scalar_decay=w.scalar_decay, init_state=ini, snap_interval=snap,
              cu_seqlens_host=inp["cu_seqlens"])
    ws = None
    if minimal_ws:
        # gdr_prefill's workspace: the fused first stage, also at d 128
        ws = torch.empty(gdr.workspace_size(n, H, dd, dd, inp["xq"].shape[0], w.scalar_decay),
                         dtype=torch.uint8, device="cuda")
    o, fin, snaps = gdr.prefill_from_projections(*(d[a] for a in ARGS), workspace=ws, **kw)
    act = gdr.preprocess(*(d[a] for a in ARGS), scalar_decay=w.scalar_decay)
    o2, fin2, snaps2 = gdr.prefill(act["q"], act["k"], act["v"], act["beta"], act["log_a"],
                                   d["cu_seqlens"], **kw)
    torch.cuda.synchronize()
    ref_act = oracle.preprocess(*(inp[a] for a in ARGS), scalar_decay=w.scalar_decay)
    cast = {m: torch.from_numpy(ref_act[m]).to(torch.bfloat16) for m in ("q", "k", "v")}
    ref = oracle.prefill(cast["q"], cast["k"], cast["v"], ref_act["beta"], ref_act["log_a"],
                         inp["cu_seqlens"], scalar_decay=w.scalar_decay, init_state=init_state,
                         snap_interval=snap)
    pairs = [("o", o, ref["o"]), ("final_state", fin, ref["final_state"])]
    if snap:
        pairs.append(("snapshots", snaps, ref["snapshots"]))
    for name, x, r in pairs:
        err = np.abs(x.double().cpu().numpy() - r).max() / np.abs(r).max()
        assert err <= 2e-2, f"fused {name}: {err:.3e}"
    # the chain of two kernels computes the same (up to the norms' summation order)
    for name, x, y in (("o", o, o2), ("final_state", fin, fin2)):
        err = (x.double() - y.double()).abs().max().item() / y.double().abs().max().item()
        assert err <= 2e-2, f"fused vs chain {name}: {err:.3e}"


@pytest.mark.parametrize("d,minimal_ws", [(64, False), (128, False), (128, True)])
@pytest.mark.parametrize("scalar", [False, True])
def test_fused_prefill_from_projections(d, minimal_ws, scalar):
    """Ragged sequences (1, 2, 3 tokens, empty, chunk-crossing lengths),
    initial states and snapshots: the conv's history restarts at each
    sequence start, including inside a chunk, and crosses chunk boundaries.
    At d 128 with a per-channel gate both the staged activations (default
    workspace) and the fused first stage (gdr_prefill's workspace)."""
    w = wl.shrink(wl.PREPROCESS, n_heads=3, d_k=d, d_v=d, scalar_decay=scalar, seed=1110)
    _fused_vs_chain(w, [1, 2, 3, 0, 130, 64, 200, 5], snap=64, init=True, minimal_ws=minimal_ws)


def test_fused_prefill_graft_layer_shape():
    """The graft layer's shape (8192 tokens x 14 heads x 64), one sequence."""
    _fused_vs_chain(wl.PREPROCESS, None)


@pytest.mark.parametrize("d,minimal_ws", [(64, False), (128, False), (128, True)])
@pytest.mark.parametrize("scalar", [False, True])
def test_fused_prefill_steep_decay(d, minimal_ws, scalar):
    """Decays below the factored range (log a < -10) inside the fused path,
    on enough chunks (6 heads x 64 chunks) that most CTAs take a second item,
    whose decay is scanned during the first item's solve: chunk j holds one
    steep row at position 3, 25 or 47 (j % 4 = 0, 1, 2; none for j % 4 = 3),
    so that each row range of that scan meets one, next to chunks without."""
    w = wl.shrink(wl.PREPROCESS, n_heads=6, d_k=d, d_v=d, scalar_decay=scalar, seed=1111)
    toks = [64 * j + (3, 25, 47)[j % 4] for j in range(64) if j % 4 != 3]
    _fused_vs_chain(w, [4096], steep=(toks, [1, d // 2 + 3, d - 1]), minimal_ws=minimal_ws)


@pytest.mark.parametrize("d,minimal_ws", [(64, False), (128, False), (128, True)])
def test_prefill_from_projections_output_epilogue(d, minimal_ws):
    """The output epilogue (RMSNorm and sigmoid gate) through the raw-projection
    path, fused first stage and staged activations alike, against the oracle's
    epilogue of the oracle's prefill of the oracle's activations."""
    gdr = _gdr()
    w = wl.shrink(wl.PREPROCESS, n_heads=3, d_k=d, d_v=d, seed=1112)
    inp = wl.make_preprocess_inputs(w, lengths=[300, 0, 77, 130])
    dd = {k: (v.cuda() if torch.is_tensor(v) else v) for k, v in inp.items()}
    T, H = inp["xq"].shape[0], w.n_heads
    n = len(inp["lengths"])
    g = wl.make_output_gate(T, H, d, torch.bfloat16, seed=91 + d)
    ws = None
    if minimal_ws:
        ws = torch.empty(gdr.workspace_size(n, H, d, d, T), dtype=torch.uint8, device="cuda")
    y = torch.full((T, H, d), float("nan"), dtype=torch.bfloat16, device="cuda")
    y, fin, _ = gdr.prefill_from_projections(*(dd[a] for a in ARGS), cu_seqlens_host=inp["cu_seqlens"],
                                             out=y, workspace=ws, gate_raw=g["gate_raw"].cuda(),
                                             norm_weight=g["norm_weight"].cuda(), norm_eps=1e-6)
    torch.cuda.synchronize()
    assert not torch.isnan(y).any()
    ref_act = oracle.preprocess(*(inp[a] for a in ARGS))
    cast = {m: torch.from_numpy(ref_act[m]).to(torch.bfloat16) for m in ("q", "k", "v")}
    ref = oracle.prefill(cast["q"], cast["k"], cast["v"], ref_act["beta"], ref_act["log_a"],
                         inp["cu_seqlens"])
    y_ref = oracle.output_epilogue(ref["o"], g["gate_raw"], g["norm_weight"], 1e-6)
    y_ref = np.asarray(y_ref, dtype=np.float64)
    err = np.abs(y.double().cpu().numpy() - y_ref).max() / np.abs(y_ref).max()
    assert err <= 2e-2, f"gated o: {err:.3e}"
    err = np.abs(fin.double().cpu().numpy() - ref["final_state"]).max() / np.abs(ref["final_state"]).max()
    assert err <= 2e-2, f"final state: {err:.3e}"
