"""Output epilogue (per-head RMSNorm with a shared weight, then the sigmoid
output gate; "kda-graft", section "Идея и архитектура") fused into the
prefill's output store and into the decode step, against the fp64 oracle:

* prefill: oracle.output_epilogue(oracle.prefill(...).o) at the prefill bound
  (2e-2 max |ref|), single-pass and segmented state passes, bf16 and fp32;
  and against the epilogue applied by the oracle to the GPU's own raw o (the
  epilogue's arithmetic alone, one bf16 rounding);
* decode: oracle.output_epilogue of the oracle decode step at 1e-4.
"""
import pytest
import torch

import oracle
import workloads as wl
from gpu_util import assert_close_rel

pytestmark = pytest.mark.gpu
TOL = 2e-2
EPS = 1e-6


def _gdr():
    import gated_delta_rule_150_b200 as gdr
    gdr.lib()
    return gdr


@pytest.mark.parametrize("d,dtype,scalar,lengths,heads", [
    (64, torch.bfloat16, False, (300, 0, 1, 129, 512), 3),      # one pass
    (128, torch.bfloat16, False, (300, 64, 257), 2),            # one pass, d 128
    (64, torch.bfloat16, False, (3000,), 1),                    # segmented
    (128, torch.bfloat16, True, (2000, 700), 1),                # segmented, scalar gate
    (64, torch.float32, False, (256,), 2),                      # fp32 (tiny workload's dtype)
    (128, torch.float32, True, (200, 77), 2),                   # fp32, d 128
])
def test_prefill_output_epilogue(d, dtype, scalar, lengths, heads):
    gdr = _gdr()
    base = wl.GDN_LONG if scalar else wl.VARLEN
    w = wl.shrink(base, n_heads=heads, d_k=d, d_v=d, lengths=lengths, qkv_dtype=dtype,
                  init_std=0.1, snap_interval=0)
    inp = wl.make_prefill_inputs(w)
    T = inp["q"].shape[0]
    g = wl.make_output_gate(T, heads, d, dtype, seed=77 + d)
    dv = {k: (v.cuda() if torch.is_tensor(v) else v) for k, v in inp.items()}
    gd = {k: v.cuda() for k, v in g.items()}
    args = (dv["q"], dv["k"], dv["v"], dv["beta"], dv["log_a"], dv["cu_seqlens"])
    kw = dict(scalar_decay=scalar, init_state=dv["init_state"])
    o_raw, f_raw, _ = gdr.prefill(*args, **kw)
    y = torch.full_like(o_raw, float("nan"))
    y, f, _ = gdr.prefill(*args, **kw, out=y, gate_raw=gd["gate_raw"],
                          norm_weight=gd["norm_weight"], norm_eps=EPS)
    torch.cuda.synchronize()
    assert not torch.isnan(y).any()
    assert torch.equal(f, f_raw)                          # the state is not touched
    ref = oracle.prefill(inp["q"], inp["k"], inp["v"], inp["beta"], inp["log_a"],
                         inp["cu_seqlens"], scalar_decay=scalar, init_state=inp["init_state"])
    y_ref = oracle.output_epilogue(ref["o"], g["gate_raw"], g["norm_weight"], EPS)
    assert_close_rel(y, y_ref, TOL, "gated o vs oracle")
    # the epilogue alone, on the GPU's own raw outputs
    y_own = oracle.output_epilogue(o_raw.cpu(), g["gate_raw"], g["norm_weight"], EPS)
    assert_close_rel(y, y_own, 1e-2 if dtype == torch.bfloat16 else 1e-4, "epilogue arithmetic")


@pytest.mark.parametrize("dk,dv,dtype,scalar", [(64, 64, torch.bfloat16, False),
                                                (128, 128, torch.bfloat16, True),
                                                (64, 128, torch.float32, False)])
def test_decode_output_epilogue(dk, dv, dtype, scalar):
    gdr = _gdr()
    w = wl.DecodeWorkload("decode_gate_case", 4242, 6, 3, dk, dv, 2, qkv_dtype=dtype,
                          scalar_decay=scalar)
    inp = wl.make_decode_inputs(w)
    g = wl.make_output_gate(w.batch, w.n_heads, dv, dtype, seed=91)
    S = inp["state"].cuda()
    S_ref = inp["state"].clone().double()
    for t in range(w.steps):
        x = {n: inp[n][t] for n in ("q", "k", "v", "beta", "log_a")}
        gate = g["gate_raw"] if t == 0 else g["gate_raw"].flip(0)
        y = gdr.decode_step(S, *(x[n].cuda() for n in ("q", "k", "v", "beta", "log_a")),
                            scalar_decay=scalar, gate_raw=gate.cuda(),
                            norm_weight=g["norm_weight"].cuda(), norm_eps=EPS)
        torch.cuda.synchronize()
        S_ref, o_ref = oracle.decode_step(S_ref, x["q"], x["k"], x["v"], x["beta"], x["log_a"],
                                          scalar_decay=scalar)
        y_ref = oracle.output_epilogue(o_ref, gate, g["norm_weight"], EPS)
        assert_close_rel(y, y_ref, 1e-4, f"decode step {t} gated o")
        assert_close_rel(S, S_ref, 1e-4, f"decode step {t} state")
