"""Draft decode with per-token state retention, and rollback, on the GPU
against the fp64 oracle.

Tolerance: max |x - ref| <= 1e-4 * max |ref| for o and the kept states (fp32
state and arithmetic, as for the decode step).  The accept step is a copy, so
the state it leaves is compared bitwise with the GPU's own kept state."""
import numpy as np
import pytest
import torch

import oracle
import workloads as wl
from gpu_util import assert_close_rel

pytestmark = pytest.mark.gpu
TOL = 1e-4


def _gdr():
    import gated_delta_rule_150_b200 as gdr
    gdr.lib()
    return gdr


def _dev(inp):
    return {k: (v.cuda() if torch.is_tensor(v) else v) for k, v in inp.items()}


def _round(inp, r, sel=slice(None)):
    return [inp[n][r][sel] for n in ("q", "k", "v", "beta", "log_a")]


def test_draft_workload_sampled():
    """The draft workload at full size (256 sequences x 14 heads x 64 x 64,
    K = 4); the oracle follows all 256 sequences."""
    gdr = _gdr()
    w = wl.SPEC_DRAFT
    inp = wl.make_draft_inputs(w, rounds=1)
    d = _dev(inp)
    S = d["state"].clone()
    o, ts = gdr.decode_draft(S, *_round(d, 0), scalar_decay=inp["scalar_decay"],
                             scale=inp["scale"])
    torch.cuda.synchronize()
    assert torch.equal(S, d["state"]), "the draft must not modify the state"
    sel = slice(0, 256)
    ro, rts = oracle.decode_draft(inp["state"][sel], *_round(inp, 0, sel),
                                  scalar_decay=inp["scalar_decay"], scale=inp["scale"])
    eo = assert_close_rel(o[sel], ro, TOL, "draft o")
    es = assert_close_rel(ts[sel], rts, TOL, "kept states")
    print(f"draft K=4: rel err o {eo:.2e} states {es:.2e}")


@pytest.mark.parametrize("dk,dv,dtype,scalar,K", [(64, 64, torch.bfloat16, False, 1),
                                                  (64, 64, torch.float32, True, 8),
                                                  (128, 128, torch.bfloat16, False, 3),
                                                  (128, 64, torch.float32, False, 5),
                                                  (64, 128, torch.bfloat16, True, 2)])
def test_draft_shapes(dk, dv, dtype, scalar, K):
    gdr = _gdr()
    dw = wl.DecodeWorkload("small", 78, 5, 3, dk, dv, 1, qkv_dtype=dtype, scalar_decay=scalar,
                           log_a_mu=1.0, log_a_sd=2.0, scale=0.7)
    w = wl.DraftWorkload("small_draft", 79, dw, K, 1)
    inp = wl.make_draft_inputs(w)
    d = _dev(inp)
    o, ts = gdr.decode_draft(d["state"], *_round(d, 0), scalar_decay=scalar, scale=0.7)
    ro, rts = oracle.decode_draft(inp["state"], *_round(inp, 0), scalar_decay=scalar, scale=0.7)
    assert_close_rel(o, ro, TOL, "draft o")
    assert_close_rel(ts, rts, TOL, "kept states")


def test_accept_restores_the_accepted_prefix():
    """n = 0 leaves the state bitwise as it was; n in 1..K gives the state
    kept after token n; values outside [0, K] are clamped."""
    gdr = _gdr()
    dw = wl.DecodeWorkload("small", 80, 8, 2, 64, 64, 1)
    w = wl.DraftWorkload("small_draft", 81, dw, 4, 1)
    inp = wl.make_draft_inputs(w)
    d = _dev(inp)
    S = d["state"].clone()
    _, ts = gdr.decode_draft(S, *_round(d, 0))
    n_acc = torch.tensor([0, 1, 2, 3, 4, 7, -3, 2], dtype=torch.int32)
    gdr.decode_accept(S, ts, n_acc.cuda())
    torch.cuda.synchronize()
    for b, n in enumerate(n_acc.tolist()):
        n = min(max(n, 0), 4)
        want = d["state"][b] if n == 0 else ts[b, n - 1]
        assert torch.equal(S[b], want), f"sequence {b}, n = {n}"
    _, rts = oracle.decode_draft(inp["state"], *_round(inp, 0))
    ref = oracle.decode_accept(inp["state"], rts, n_acc)
    assert_close_rel(S, ref, TOL, "state after accept")


def test_speculative_rounds_follow_the_accepted_tokens():
    """Several draft / verify / accept rounds on the live state: the state
    after the rounds equals plain decode steps over the accepted tokens only
    (oracle), and so does every round's output of accepted tokens."""
    gdr = _gdr()
    dw = wl.DecodeWorkload("small", 82, 6, 3, 64, 64, 1, log_a_mu=2.0)
    w = wl.DraftWorkload("small_draft", 83, dw, 4, 5)
    inp = wl.make_draft_inputs(w)
    d = _dev(inp)
    S = d["state"].clone()
    ref_S = oracle.f64(inp["state"])
    for r in range(w.rounds):
        o, ts = gdr.decode_draft(S, *_round(d, r))
        gdr.decode_accept(S, ts, d["n_accept"][r])
        rq, rk, rv, rb, rl = (oracle.f64(x) for x in _round(inp, r))
        for b, n in enumerate(inp["n_accept"][r].tolist()):
            for t in range(n):
                sb, ob = oracle.decode_step(ref_S[b:b + 1], rq[b:b + 1, t], rk[b:b + 1, t],
                                            rv[b:b + 1, t], rb[b:b + 1, t], rl[b:b + 1, t])
                ref_S[b] = sb[0]
                assert_close_rel(o[b, t], ob[0], TOL, f"round {r} seq {b} token {t} o")
    torch.cuda.synchronize()
    assert_close_rel(S, ref_S, TOL, "state after the rounds")


def test_draft_of_one_token_matches_the_decode_step():
    gdr = _gdr()
    inp = wl.make_decode_inputs(wl.DecodeWorkload("small", 84, 7, 2, 64, 64, 1), steps=1)
    d = _dev(inp)
    S1 = d["state"].clone()
    o1 = gdr.decode_step(S1, d["q"][0], d["k"][0], d["v"][0], d["beta"][0], d["log_a"][0])
    o2, ts = gdr.decode_draft(d["state"], d["q"][0][:, None], d["k"][0][:, None],
                              d["v"][0][:, None], d["beta"][0][:, None], d["log_a"][0][:, None])
    torch.cuda.synchronize()
    assert_close_rel(o2[:, 0], o1.double().cpu().numpy(), 1e-6, "o")
    assert_close_rel(ts[:, 0], S1.double().cpu().numpy(), 1e-6, "state")


def test_empty_draft_and_accept_are_noops():
    gdr = _gdr()
    S = torch.randn(3, 2, 64, 64, device="cuda")
    S0 = S.clone()
    z = torch.zeros(3, 0, 2, 64, device="cuda", dtype=torch.bfloat16)
    o, ts = gdr.decode_draft(S, z, z, z, torch.zeros(3, 0, 2, device="cuda"),
                             torch.zeros(3, 0, 2, 64, device="cuda"))
    assert o.shape == (3, 0, 2, 64) and ts.shape == (3, 0, 2, 64, 64)
    gdr.decode_accept(S, ts, torch.full((3,), 2, dtype=torch.int32, device="cuda"))
    torch.cuda.synchronize()
    assert torch.equal(S, S0)
