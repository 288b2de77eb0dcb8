"""Chunk-local cumulative log decay on the GPU against the oracle's plain
prefix sums.  Chunk boundaries (restart at every sequence start and every 64
tokens, partial last chunk) must match exactly: an element summed into the
wrong chunk is off by at least one |log a| (> 1e-3 here), far above the
fp32 rounding bound used (rtol 1e-5 of the running sum of |log a|)."""
import numpy as np
import pytest
import torch

import oracle
import workloads as wl

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("scalar", [False, True])
@pytest.mark.parametrize("lengths", [[256], [1, 63, 64, 65, 130, 0, 200], [5000, 3]])
def test_cumdecay(scalar, lengths):
    import gated_delta_rule_150_b200 as gdr
    w = wl.shrink(wl.VARLEN if not scalar else wl.GDN_LONG, n_heads=3, d_k=64, d_v=64,
                  lengths=tuple(lengths), init_std=0.0, snap_interval=0)
    inp = wl.make_prefill_inputs(w)
    la = inp["log_a"]
    g = gdr.cumdecay(la.cuda(), inp["cu_seqlens"].cuda(), scalar_decay=scalar, d_k=64)
    torch.cuda.synchronize()
    ref = oracle.cumdecay(la, inp["cu_seqlens"])
    bound = oracle.cumdecay(np.abs(oracle.f64(la)), inp["cu_seqlens"])
    err = np.abs(g.cpu().double().numpy() - ref)
    assert (err <= 1e-5 * bound + 1e-7).all(), float(err.max())
