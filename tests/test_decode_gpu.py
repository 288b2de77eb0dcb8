"""Decode step on the GPU against the fp64 oracle.

Tolerance: max |x - ref| <= 1e-4 * max |ref| for o and the state (fp32 state
and arithmetic; the only rounding is fp32's), after 1 step and after the
decode workload's 1024 in-place steps on a sample of its sequences."""
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


def _run(w, steps, sample=None):
    gdr = _gdr()
    inp = wl.make_decode_inputs(w, steps=steps)
    dev = {k: (v.cuda() if torch.is_tensor(v) else v) for k, v in inp.items()}
    S = dev["state"].clone()
    o_last = None
    ref_S = inp["state"]
    sel = slice(None) if sample is None else sample
    ref_S = oracle.f64(ref_S)[sel]
    for t in range(steps):
        o_last = gdr.decode_step(S, dev["q"][t], dev["k"][t], dev["v"][t], dev["beta"][t],
                                 dev["log_a"][t], scalar_decay=w.scalar_decay, scale=w.scale)
        ref_S, ref_o = oracle.decode_step(ref_S, inp["q"][t][sel], inp["k"][t][sel],
                                          inp["v"][t][sel], inp["beta"][t][sel],
                                          inp["log_a"][t][sel], scalar_decay=w.scalar_decay,
                                          scale=w.scale)
        if t == 0:
            assert_close_rel(o_last[sel], ref_o, TOL, "o after step 1")
            assert_close_rel(S[sel], ref_S, TOL, "state after step 1")
    torch.cuda.synchronize()
    eo = assert_close_rel(o_last[sel], ref_o, TOL, f"o after step {steps}")
    es = assert_close_rel(S[sel], ref_S, TOL, f"state after step {steps}")
    return eo, es


def test_decode_workload_1024_steps_sampled():
    """The decode workload at full size (256 x 14 x 64 x 64, 1024 steps);
    the oracle follows 64 of the 256 sequences (every fourth)."""
    sample = slice(0, 256, 4)
    eo, es = _run(wl.DECODE, 1024, sample)
    print(f"decode 1024 steps: rel err o {eo:.2e} state {es:.2e}")


@pytest.mark.parametrize("dk,dv,dtype,scalar", [(64, 64, torch.float32, False),
                                                (128, 128, torch.bfloat16, False),
                                                (128, 64, torch.bfloat16, True),
                                                (64, 128, torch.float32, True)])
def test_decode_shapes(dk, dv, dtype, scalar):
    w = wl.DecodeWorkload("small", 77, 5, 3, dk, dv, 8, qkv_dtype=dtype, scalar_decay=scalar,
                          log_a_mu=1.0, log_a_sd=2.0, scale=0.7)
    _run(w, 8)


def test_decode_empty_batch_is_noop():
    gdr = _gdr()
    z = torch.zeros(0, 2, 64, device="cuda", dtype=torch.bfloat16)
    S = torch.zeros(0, 2, 64, 64, device="cuda")
    o = gdr.decode_step(S, z, z, z, torch.zeros(0, 2, device="cuda"),
                        torch.zeros(0, 2, 64, device="cuda"))
    assert o.shape == (0, 2, 64)
