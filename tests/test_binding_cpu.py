"""Host-side checks of the Python binding, on CPU tensors: every call rejects
tensors whose shape or dtype does not match the layout the C ABI assumes
(the kernels would otherwise read or write past a buffer's end), and a call
with matching tensors gets as far as the device check."""
import pytest
import torch

import gated_delta_rule_150_b200 as gdr

bf16, f32 = torch.bfloat16, torch.float32


def _reaches_device_check(fn, *a, **kw):
    with pytest.raises(ValueError, match="CUDA tensors"):
        fn(*a, **kw)


def _prefill_inputs(T=10, H=2, d=64, scalar=False, lengths=(4, 6)):
    cu = torch.tensor([0] + list(torch.tensor(lengths).cumsum(0)), dtype=torch.int32)
    return dict(q=torch.zeros(T, H, d, dtype=bf16), k=torch.zeros(T, H, d, dtype=bf16),
                v=torch.zeros(T, H, d, dtype=bf16), beta=torch.zeros(T, H),
                log_a=torch.zeros((T, H) if scalar else (T, H, d)), cu_seqlens=cu)


def _prefill(x, **kw):
    return gdr.prefill(x["q"], x["k"], x["v"], x["beta"], x["log_a"], x["cu_seqlens"], **kw)


def test_prefill_shapes():
    x = _prefill_inputs()
    _reaches_device_check(_prefill, x)
    _reaches_device_check(_prefill, _prefill_inputs(scalar=True), scalar_decay=True)
    bad = dict(x, k=torch.zeros(10, 2, 32, dtype=bf16))
    with pytest.raises(ValueError, match="k must have shape"):
        _prefill(bad)
    with pytest.raises(TypeError, match="beta must be"):
        _prefill(dict(x, beta=torch.zeros(10, 2, dtype=torch.float16)))
    with pytest.raises(ValueError, match="log_a must have shape"):
        _prefill(x, scalar_decay=True)               # per-channel log_a with a scalar gate
    with pytest.raises(ValueError, match="cu_seqlens"):
        _prefill(dict(x, cu_seqlens=x["cu_seqlens"].long()))
    with pytest.raises(ValueError, match="end at the number of tokens"):
        _prefill(x, cu_seqlens_host=[0, 4, 11])
    with pytest.raises(ValueError, match="never decrease"):
        _prefill(x, cu_seqlens_host=[0, 11, 10])
    with pytest.raises(ValueError, match="init_state must have shape"):
        _prefill(x, init_state=torch.zeros(1, 2, 64, 64))
    with pytest.raises(ValueError, match="final_state must have shape"):
        _prefill(x, final_state=torch.zeros(2, 2, 64, 32))
    with pytest.raises(TypeError, match="out must be"):
        _prefill(x, out=torch.zeros(10, 2, 64))
    long = _prefill_inputs(T=192, lengths=(128, 64))
    with pytest.raises(ValueError, match="slots"):
        _prefill(long, snap_interval=64, cu_seqlens_host=[0, 128, 192],
                 snapshots=torch.zeros(2, 2, 64, 64))
    _reaches_device_check(_prefill, long, snap_interval=64, cu_seqlens_host=[0, 128, 192],
                          snapshots=torch.zeros(3, 2, 64, 64))


def test_prepared_prefill_needs_its_buffers():
    x = _prefill_inputs()
    args = (x["q"], x["k"], x["v"], x["beta"], x["log_a"], x["cu_seqlens"])
    with pytest.raises(ValueError, match="needs out"):
        gdr.PreparedPrefill(*args, out=None, final_state=torch.zeros(2, 2, 64, 64),
                            workspace=torch.zeros(16, dtype=torch.uint8))
    with pytest.raises(ValueError, match="snapshots buffer"):
        gdr.PreparedPrefill(*args, out=torch.zeros(10, 2, 64, dtype=bf16),
                            final_state=torch.zeros(2, 2, 64, 64),
                            workspace=torch.zeros(16, dtype=torch.uint8), snap_interval=64)


def test_cumdecay_and_chunk_factors_shapes():
    x = _prefill_inputs()
    with pytest.raises(ValueError, match="needs d_k"):
        gdr.cumdecay(torch.zeros(10, 2), x["cu_seqlens"], scalar_decay=True)
    with pytest.raises(ValueError, match="3 dimensions"):
        gdr.cumdecay(torch.zeros(10, 2), x["cu_seqlens"])
    with pytest.raises(ValueError, match="out must have shape"):
        gdr.cumdecay(x["log_a"], x["cu_seqlens"], out=torch.zeros(10, 2))
    _reaches_device_check(gdr.cumdecay, x["log_a"], x["cu_seqlens"])
    with pytest.raises(ValueError, match="v must have shape"):
        gdr.chunk_factors(x["q"], x["k"], torch.zeros(9, 2, 64, dtype=bf16), x["beta"],
                          x["log_a"], x["cu_seqlens"])
    _reaches_device_check(gdr.chunk_factors, x["q"], x["k"], x["v"], x["beta"], x["log_a"],
                          x["cu_seqlens"])


def test_decode_shapes():
    B, H, d = 3, 2, 64
    q = torch.zeros(B, H, d, dtype=bf16)
    S = torch.zeros(B, H, d, d)
    ok = (S, q, q, q, torch.zeros(B, H), torch.zeros(B, H, d))
    _reaches_device_check(gdr.decode_step, *ok)
    with pytest.raises(ValueError, match="state must have shape"):
        gdr.decode_step(torch.zeros(B, H, d, 32), *ok[1:])
    with pytest.raises(TypeError, match="state must be"):
        gdr.decode_step(S.double(), *ok[1:])
    with pytest.raises(ValueError, match="log_a must have shape"):
        gdr.decode_step(*ok, scalar_decay=True)
    with pytest.raises(ValueError, match="out must have shape"):
        gdr.decode_step(*ok, out=torch.zeros(B, H))


def test_draft_and_accept_shapes():
    B, K, H, d = 3, 4, 2, 64
    q = torch.zeros(B, K, H, d, dtype=bf16)
    S = torch.zeros(B, H, d, d)
    ok = (S, q, q, q, torch.zeros(B, K, H), torch.zeros(B, K, H, d))
    _reaches_device_check(gdr.decode_draft, *ok)
    with pytest.raises(ValueError, match="4 dimensions"):
        gdr.decode_draft(S, q[:, 0], q[:, 0], q[:, 0], torch.zeros(B, H), torch.zeros(B, H, d))
    with pytest.raises(ValueError, match="beta must have shape"):
        gdr.decode_draft(S, q, q, q, torch.zeros(B, H), ok[5])
    with pytest.raises(ValueError, match="token_states must have shape"):
        gdr.decode_draft(*ok, token_states=torch.zeros(B, K - 1, H, d, d))
    ts = torch.zeros(B, K, H, d, d)
    n = torch.zeros(B, dtype=torch.int32)
    _reaches_device_check(gdr.decode_accept, S, ts, n)
    with pytest.raises(TypeError, match="n_accept must be"):
        gdr.decode_accept(S, ts, n.long())
    with pytest.raises(ValueError, match="n_accept must have shape"):
        gdr.decode_accept(S, ts, torch.zeros(B + 1, dtype=torch.int32))
    with pytest.raises(ValueError, match="state must have shape"):
        gdr.decode_accept(S[:, :1], ts, n)


def test_preprocess_shapes():
    T, H, d = 10, 2, 64
    cu = torch.tensor([0, 4, 10], dtype=torch.int32)
    x = torch.zeros(T, H, d, dtype=bf16)
    w = torch.zeros(H * d, 4)
    ok = [x, x, x, w, w, w, torch.zeros(T, H), torch.zeros(T, H, d), torch.zeros(H, d), cu]
    _reaches_device_check(gdr.preprocess, *ok)
    sc = list(ok)
    sc[7], sc[8] = torch.zeros(T, H), torch.zeros(H)
    _reaches_device_check(gdr.preprocess, *sc, scalar_decay=True)
    bad = list(ok)
    bad[4] = torch.zeros(H * d, 3)
    with pytest.raises(ValueError, match="conv_k must have shape"):
        gdr.preprocess(*bad)
    with pytest.raises(ValueError, match="a_raw must have shape"):
        gdr.preprocess(*ok, scalar_decay=True)
    with pytest.raises(ValueError, match="out\\['q'\\] must have shape"):
        gdr.preprocess(*ok, out=dict(q=torch.zeros(T, H, 32, dtype=bf16)))
