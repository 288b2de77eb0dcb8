"""The seeded input generators (``workloads.py``): the same seed gives the
same bits, and each recipe has the shapes, dtypes and value ranges its
docstring states.  These inputs feed both the kernels and the oracle."""
import torch

import workloads as wl


def _same(a, b):
    assert a.keys() == b.keys()
    for k in a:
        if torch.is_tensor(a[k]):
            assert torch.equal(a[k], b[k]), k
        else:
            assert a[k] == b[k], k


def test_generators_are_deterministic():
    small = wl.shrink(wl.VARLEN, n_heads=2, d_k=64, d_v=64, n_seqs=3, len_range=(5, 40))
    _same(wl.make_prefill_inputs(small), wl.make_prefill_inputs(small))
    dec = wl.DecodeWorkload("d", 7, 4, 2, 64, 64, 3)
    _same(wl.make_decode_inputs(dec), wl.make_decode_inputs(dec))
    dr = wl.DraftWorkload("dr", 8, dec, 3, 2)
    _same(wl.make_draft_inputs(dr), wl.make_draft_inputs(dr))
    pw = wl.shrink(wl.PREPROCESS, n_heads=2)
    _same(wl.make_preprocess_inputs(pw, lengths=[7, 9]), wl.make_preprocess_inputs(pw, lengths=[7, 9]))
    other = wl.make_prefill_inputs(wl.shrink(small, seed=small.seed + 1))
    assert not torch.equal(other["beta"][:5], wl.make_prefill_inputs(small)["beta"][:5])


def test_prefill_recipe():
    w = wl.shrink(wl.VARLEN, n_heads=3, d_k=64, d_v=64, n_seqs=5, len_range=(10, 50))
    x = wl.make_prefill_inputs(w)
    cu = x["cu_seqlens"]
    assert cu.dtype == torch.int32 and int(cu[0]) == 0
    lens = (cu[1:] - cu[:-1]).tolist()
    assert lens == x["lengths"] and all(10 <= n <= 50 for n in lens)
    T = int(cu[-1])
    assert x["q"].shape == (T, 3, 64) and x["q"].dtype == torch.bfloat16
    for name in ("q", "k"):
        nrm = x[name].float().norm(dim=-1)
        assert torch.allclose(nrm, torch.ones_like(nrm), atol=1e-2)
    assert ((x["beta"] > 0) & (x["beta"] < 1)).all()
    assert (x["log_a"] <= 0).all() and (x["log_a"] >= -5).all()     # clamped recipe
    assert x["init_state"].shape == (5, 3, 64, 64)
    g = wl.make_prefill_inputs(wl.shrink(wl.GDN_LONG, lengths=(100,), snap_interval=0))
    assert g["log_a"].shape == (100, 16) and g["scalar_decay"]


def test_draft_and_preprocess_recipes():
    dec = wl.DecodeWorkload("d", 9, 5, 2, 64, 64, 1)
    dr = wl.make_draft_inputs(wl.DraftWorkload("dr", 10, dec, 4, 3))
    assert dr["q"].shape == (3, 5, 4, 2, 64) and dr["n_accept"].dtype == torch.int32
    assert dr["n_accept"].shape == (3, 5)
    assert int(dr["n_accept"].min()) >= 0 and int(dr["n_accept"].max()) <= 4
    p = wl.make_preprocess_inputs(wl.PREPROCESS, lengths=[300])
    assert p["xq"].shape == (300, 14, 64) and p["conv_q"].shape == (14 * 64, 4)
    assert torch.equal(p["a_bias"], torch.full((14, 64), 5.0))
    # taps: the identity tap plus N(0, 0.1)
    mean = p["conv_v"].mean(0)
    assert torch.allclose(mean, torch.tensor([0.0, 0.0, 0.0, 1.0]), atol=0.03)
    assert 0.08 < float(p["conv_v"].std(0).mean()) < 0.12
