"""Pins of the fp64 oracle against what the pages and the mathematics fix.

None of these re-types the oracle's own loop: each compares it with an
independent statement of the result (a closed form, a reduction to a simpler
rule, a dense product of transition matrices, a printed worked example, or an
invariance that any correct implementation must satisfy).  The last test
plants each of twelve plausible mistakes in the oracle (compile-time mutants of
the C source) and checks that at least one pin rejects every one of them.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rng(seed):
    return np.random.default_rng(seed)


def _unit(x):
    return x / np.linalg.norm(x, axis=-1, keepdims=True)


# --------------------------------------------------------------------------
# Individual pins.  Each takes the oracle mutant id (0 = the real oracle) and
# raises AssertionError when the oracle disagrees with the pin.
# --------------------------------------------------------------------------

def pin_exact_retrieval(mutant=0):
    """Modele hybrydowe, section "Reguła delta": with beta = 1, a = 1 and a
    unit key, the updated state maps k_t exactly to v_t (S_t k_t = v_t), and
    writing the same association again leaves the state unchanged."""
    r = _rng(1)
    T, H, d = 6, 2, 8
    k = _unit(r.standard_normal((T, H, d)))
    k[3] = k[2]                      # token 3 repeats token 2's key ...
    v = r.standard_normal((T, H, d))
    v[3] = v[2]                      # ... and its value
    q = k.copy()                     # o_t = S_t k_t
    beta = np.ones((T, H))
    la = np.zeros((T, H, d))
    S0 = r.standard_normal((1, H, d, d))
    out = oracle.prefill(q, k, v, beta, la, [0, T], init_state=S0, mutant=mutant)
    np.testing.assert_allclose(out["o"], v, rtol=0, atol=1e-12)
    # the repeated write changes nothing: state after token 3 == state after token 2
    s2 = oracle.prefill(q[:3], k[:3], v[:3], beta[:3], la[:3], [0, 3], init_state=S0,
                        mutant=mutant)["final_state"]
    s3 = oracle.prefill(q[:4], k[:4], v[:4], beta[:4], la[:4], [0, 4], init_state=S0,
                        mutant=mutant)["final_state"]
    np.testing.assert_allclose(s3, s2, rtol=0, atol=1e-12)


def pin_frozen_state(mutant=0):
    """beta = 0 removes both the erase and the write term of the gated rule
    (Modele hybrydowe, "Gated DeltaNet: dodaj zanik"), so the state only
    decays: S_T = S_0 Diag(prod_t a_t) and o_t = S_t q_t with that state."""
    r = _rng(2)
    T, H, d = 7, 2, 6
    q, k, v = (r.standard_normal((T, H, d)) for _ in range(3))
    beta = np.zeros((T, H))
    la = -0.3 * r.random((T, H, d))
    S0 = r.standard_normal((1, H, d, d))
    out = oracle.prefill(q, k, v, beta, la, [0, T], init_state=S0, mutant=mutant)
    G = np.cumsum(la, axis=0)                              # [T, H, d]
    S_t = S0[0][None] * np.exp(G)[:, :, None, :]           # [T, H, dv, dk]
    np.testing.assert_allclose(out["final_state"][0], S_t[-1], rtol=1e-13, atol=1e-13)
    o_ref = np.einsum("thjc,thc->thj", S_t, q)
    np.testing.assert_allclose(out["o"], o_ref, rtol=1e-12, atol=1e-12)


def pin_linear_attention(mutant=0):
    """Modele hybrydowe, section "Atencja liniowa": with orthonormal keys
    (T <= d_k), a = 1 and S_0 = 0 the erase term never fires, so the gated
    delta rule is additive linear attention with values beta_t v_t:
    S_T = sum_t beta_t v_t k_t^T and o_t = sum_{i<=t} beta_i v_i (k_i . q_t)."""
    r = _rng(3)
    T, H, d, dv = 5, 2, 8, 6
    k = np.stack([np.linalg.qr(r.standard_normal((d, d)))[0][:, :T].T for _ in range(H)], 1)
    q = r.standard_normal((T, H, d))
    v = r.standard_normal((T, H, dv))
    beta = r.random((T, H))
    la = np.zeros((T, H, d))
    out = oracle.prefill(q, k, v, beta, la, [0, T], mutant=mutant)
    S_ref = np.einsum("th,thj,thc->hjc", beta, v, k)
    np.testing.assert_allclose(out["final_state"][0], S_ref, rtol=0, atol=1e-12)
    causal = np.tril(np.ones((T, T)))
    o_ref = np.einsum("ih,ihj,ihc,thc,ti->thj", beta, v, k, q, causal)
    np.testing.assert_allclose(out["o"], o_ref, rtol=0, atol=1e-12)


def _brute(q, k, v, beta, la, S0, scalar):
    """Dense product of transition matrices:
    S_T = S_0 prod_t M_t + sum_t beta_t v_t k_t^T prod_{s>t} M_s,
    M_t = Diag(a_t) (I - beta_t k_t k_t^T)."""
    T, H, dk = q.shape
    dv = v.shape[2]
    o = np.zeros((T, H, dv))
    fin = np.zeros((H, dv, dk))
    for h in range(H):
        M = []
        for t in range(T):
            a = np.exp(np.full(dk, la[t, h]) if scalar else la[t, h])
            M.append(np.diag(a) @ (np.eye(dk) - beta[t, h] * np.outer(k[t, h], k[t, h])))
        for t in range(T):
            P = np.eye(dk)
            for s in range(t + 1):
                P = P @ M[s]
            S = S0[h] @ P
            for i in range(t + 1):
                R = np.eye(dk)
                for s in range(i + 1, t + 1):
                    R = R @ M[s]
                S = S + beta[i, h] * np.outer(v[i, h], k[i, h]) @ R
            o[t, h] = S @ q[t, h]
            if t == T - 1:
                fin[h] = S
    return o, fin


def pin_brute_force(mutant=0):
    """Tiny cases (T <= 6, d <= 4) against the dense transition-matrix
    expansion, per-channel and scalar decay, to 1e-12."""
    r = _rng(4)
    for scalar, (T, H, dk, dv) in ((False, (6, 2, 4, 3)), (True, (5, 3, 3, 4)), (False, (1, 2, 4, 4))):
        q = r.standard_normal((T, H, dk))
        k = r.standard_normal((T, H, dk))
        v = r.standard_normal((T, H, dv))
        beta = r.random((T, H))
        la = -r.random((T, H) if scalar else (T, H, dk))
        S0 = r.standard_normal((1, H, dv, dk))
        out = oracle.prefill(q, k, v, beta, la, [0, T], scalar_decay=scalar, init_state=S0,
                             mutant=mutant)
        o_ref, fin_ref = _brute(q, k, v, beta, la, S0[0], scalar)
        np.testing.assert_allclose(out["o"], o_ref, rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(out["final_state"][0], fin_ref, rtol=1e-12, atol=1e-12)


def pin_snapshots(mutant=0):
    """Modele hybrydowe, "Co stan rekurencyjny zmienia przy serwowaniu",
    point 1: the state at position N can only come from a snapshot taken at N.
    Snapshot m of a sequence must equal the final state of the same prefill
    cut after m * interval tokens; with L a multiple of the interval the last
    snapshot is the final state itself (bitwise)."""
    r = _rng(5)
    lengths = [24, 9, 16]
    iv = 8
    T, H, d = sum(lengths), 2, 4
    q, k, v = (r.standard_normal((T, H, d)) for _ in range(3))
    beta = r.random((T, H))
    la = -0.2 * r.random((T, H, d))
    cu = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int32)
    out = oracle.prefill(q, k, v, beta, la, cu, snap_interval=iv, mutant=mutant)
    assert out["snapshots"].shape[0] == sum(n // iv for n in lengths)
    slot = 0
    for n, L in enumerate(lengths):
        s = int(cu[n])
        for m in range(1, L // iv + 1):
            e = s + m * iv
            ref = oracle.prefill(q[s:e], k[s:e], v[s:e], beta[s:e], la[s:e], [0, e - s],
                                 mutant=mutant)["final_state"][0]
            np.testing.assert_array_equal(out["snapshots"][slot], ref)
            slot += 1
        if L % iv == 0:
            np.testing.assert_array_equal(out["snapshots"][slot - 1], out["final_state"][n])


def pin_split_and_varlen(mutant=0):
    """Any prefix split gives the same result when the state is carried over,
    and sequences packed by cu_seqlens are independent of one another."""
    r = _rng(6)
    T, H, d = 40, 2, 5
    q, k, v = (r.standard_normal((T, H, d)) for _ in range(3))
    beta = r.random((T, H))
    la = -0.5 * r.random((T, H, d))
    S0 = r.standard_normal((1, H, d, d))
    full = oracle.prefill(q, k, v, beta, la, [0, T], init_state=S0, mutant=mutant)
    N = 17
    a = oracle.prefill(q[:N], k[:N], v[:N], beta[:N], la[:N], [0, N], init_state=S0,
                       mutant=mutant)
    b = oracle.prefill(q[N:], k[N:], v[N:], beta[N:], la[N:], [0, T - N],
                       init_state=a["final_state"], mutant=mutant)
    np.testing.assert_allclose(np.concatenate([a["o"], b["o"]]), full["o"], rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(b["final_state"], full["final_state"], rtol=1e-12, atol=1e-12)
    # packing: [seq A | seq B] as two sequences == two separate calls
    S1 = r.standard_normal((2, H, d, d))
    pk = oracle.prefill(q, k, v, beta, la, [0, N, T], init_state=S1, mutant=mutant)
    a1 = oracle.prefill(q[:N], k[:N], v[:N], beta[:N], la[:N], [0, N], init_state=S1[:1],
                        mutant=mutant)
    b1 = oracle.prefill(q[N:], k[N:], v[N:], beta[N:], la[N:], [0, T - N], init_state=S1[1:],
                        mutant=mutant)
    np.testing.assert_array_equal(pk["o"], np.concatenate([a1["o"], b1["o"]]))
    np.testing.assert_array_equal(pk["final_state"],
                                  np.concatenate([a1["final_state"], b1["final_state"]]))


def pin_decay_magnitude(mutant=0):
    """kda-graft: the alpha gate starts at sigmoid(5) ~ 0.993 and its product
    over 950 tokens is ~ 1e-3.  With beta = 0 and v = 0 the oracle's state
    after 950 steps must be S_0 sigmoid(5)^950 (fp64), and that factor must
    round to the printed figures."""
    g = json.load(open(os.path.join(GOLDEN, "decay_magnitude.json")))
    bias, steps = g["gate_bias"], g["steps"]
    la_val = -math.log1p(math.exp(-bias))                  # logsigmoid(bias)
    sig = math.exp(la_val)
    assert round(sig, g["sigma_printed_digits"]) == g["sigma_printed"]
    H, d = 1, 3
    r = _rng(7)
    S0 = r.standard_normal((1, H, d, d))
    z = np.zeros((steps, H, d))
    out = oracle.prefill(z, z, z, np.zeros((steps, H)), np.full((steps, H), la_val), [0, steps],
                         scalar_decay=True, init_state=S0, mutant=mutant)
    factor = out["final_state"] / S0
    np.testing.assert_allclose(factor, sig ** steps, rtol=1e-12)
    assert round(math.log10(sig ** steps)) == g["product_order_of_magnitude"]


def pin_decode_equals_prefill(mutant=0):
    """T single-token decode steps equal one prefill of the same T tokens."""
    r = _rng(8)
    T, B, H, d = 5, 3, 2, 4
    q, k, v = (r.standard_normal((T, B, H, d)) for _ in range(3))
    beta = r.random((T, B, H))
    la = -0.3 * r.random((T, B, H, d))
    S = r.standard_normal((B, H, d, d))
    os_ = []
    St = S.copy()
    for t in range(T):
        St, o = oracle.decode_step(St, q[t], k[t], v[t], beta[t], la[t], mutant=mutant)
        os_.append(o)
    for b in range(B):
        ref = oracle.prefill(q[:, b], k[:, b], v[:, b], beta[:, b], la[:, b], [0, T],
                             init_state=S[b:b + 1], mutant=mutant)
        np.testing.assert_allclose(np.stack(os_)[:, b], ref["o"], rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(St[b], ref["final_state"][0], rtol=1e-12, atol=1e-12)


def pin_scalar_is_broadcast(mutant=0):
    """Modele hybrydowe, "Gated DeltaNet": the scalar gate alpha_t is the
    per-channel gate with every channel equal; the two forms agree bitwise."""
    r = _rng(9)
    T, H, d = 11, 3, 4
    q, k, v = (r.standard_normal((T, H, d)) for _ in range(3))
    beta = r.random((T, H))
    la = -r.random((T, H))
    a = oracle.prefill(q, k, v, beta, la, [0, T], scalar_decay=True, mutant=mutant)
    b = oracle.prefill(q, k, v, beta, np.repeat(la[:, :, None], d, 2), [0, T], mutant=mutant)
    np.testing.assert_array_equal(a["o"], b["o"])
    np.testing.assert_array_equal(a["final_state"], b["final_state"])


def _draft_inputs(r, B, K, H, dk, dv, scalar=False):
    q = r.standard_normal((B, K, H, dk))
    k = _unit(r.standard_normal((B, K, H, dk)))
    v = r.standard_normal((B, K, H, dv))
    beta = r.random((B, K, H))
    la = -0.4 * r.random((B, K, H) if scalar else (B, K, H, dk))
    S = r.standard_normal((B, H, dv, dk))
    return q, k, v, beta, la, S


def pin_draft_keeps_every_state(mutant=0):
    """Modele hybrydowe, "Co stan rekurencyjny zmienia przy serwowaniu",
    point 2: a draft of K tokens keeps the state after each token.  Draft
    sequence b must equal a prefill of its K tokens from state[b] with a
    snapshot after every token (the snapshot rule is pinned on its own above):
    the kept states are those snapshots and the outputs are the prefill's."""
    r = _rng(12)
    B, K, H, dk, dv = 3, 5, 2, 4, 3
    for scalar in (False, True):
        q, k, v, beta, la, S = _draft_inputs(r, B, K, H, dk, dv, scalar)
        o, ts = oracle.decode_draft(S, q, k, v, beta, la, scalar_decay=scalar, scale=0.5,
                                    mutant=mutant)
        assert o.shape == (B, K, H, dv) and ts.shape == (B, K, H, dv, dk)
        for b in range(B):
            ref = oracle.prefill(q[b], k[b], v[b], beta[b], la[b], [0, K], scalar_decay=scalar,
                                 scale=0.5, init_state=S[b:b + 1], snap_interval=1,
                                 mutant=mutant)
            np.testing.assert_allclose(ts[b], ref["snapshots"], rtol=1e-12, atol=1e-12)
            np.testing.assert_allclose(o[b], ref["o"], rtol=1e-12, atol=1e-12)


def pin_draft_frozen(mutant=0):
    """With beta = 0 every draft token only decays the state (as in
    pin_frozen_state): kept state t = S Diag(exp(sum_{i<=t} log a_i)) and
    o_t = (kept state t) (scale q_t), in closed form."""
    r = _rng(13)
    B, K, H, dk, dv = 2, 4, 3, 5, 4
    q, k, v, beta, la, S = _draft_inputs(r, B, K, H, dk, dv)
    beta[:] = 0.0
    o, ts = oracle.decode_draft(S, q, k, v, beta, la, scale=2.0, mutant=mutant)
    G = np.cumsum(la, axis=1)                                  # [B, K, H, dk]
    ts_ref = S[:, None] * np.exp(G)[:, :, :, None, :]          # [B, K, H, dv, dk]
    np.testing.assert_allclose(ts, ts_ref, rtol=1e-13, atol=1e-13)
    np.testing.assert_allclose(o, np.einsum("bthjc,bthc->bthj", ts_ref, 2.0 * q),
                               rtol=1e-12, atol=1e-12)


def pin_rollback(mutant=0):
    """Same passage: accepting n of the K draft tokens leaves exactly the
    state that n single decode steps give (decode steps are pinned against
    prefill above); n = 0 gives back the state before the draft bitwise;
    n outside [0, K] is clamped."""
    r = _rng(14)
    B, K, H, d = 6, 4, 2, 4
    q, k, v, beta, la, S = _draft_inputs(r, B, K, H, d, d)
    _, ts = oracle.decode_draft(S, q, k, v, beta, la, mutant=mutant)
    n_acc = np.array([0, 1, 2, K, K + 3, -2], dtype=np.int32)
    out = oracle.decode_accept(S, ts, n_acc, mutant=mutant)
    for b in range(B):
        n = min(max(int(n_acc[b]), 0), K)
        ref = S[b:b + 1].copy()
        for t in range(n):
            ref, _ = oracle.decode_step(ref, q[b:b + 1, t], k[b:b + 1, t], v[b:b + 1, t],
                                        beta[b:b + 1, t], la[b:b + 1, t], mutant=mutant)
        if n == 0:
            np.testing.assert_array_equal(out[b], S[b])
        else:
            np.testing.assert_allclose(out[b], ref[0], rtol=1e-12, atol=1e-12)


PINS = [pin_exact_retrieval, pin_frozen_state, pin_linear_attention, pin_brute_force,
        pin_snapshots, pin_split_and_varlen, pin_decay_magnitude, pin_decode_equals_prefill,
        pin_scalar_is_broadcast, pin_draft_keeps_every_state, pin_draft_frozen, pin_rollback]


@pytest.mark.parametrize("pin", PINS, ids=lambda p: p.__name__)
def test_pin(pin):
    pin(0)


def test_state_size_worked_example():
    """kda-graft, "Память — доказано точно" and Modele hybrydowe, "Atencja
    liniowa": the per-head state is d_v x d_k fp32 whatever the length.  The
    oracle's state for the graft's heads (14 x 64 x 64), times 18 KDA layers,
    reproduces the printed constant and the byte-exact cache figure."""
    g = json.load(open(os.path.join(GOLDEN, "state_size.json")))
    H, d = g["heads"], g["head_dim"]
    sizes = set()
    for T in (1, 37, 300):
        r = _rng(T)
        x = r.standard_normal((T, H, d))
        out = oracle.prefill(x, x, x, r.random((T, H)), -r.random((T, H, d)), [0, T])
        sizes.add(out["final_state"].shape)
    assert sizes == {(1, H, d, d)}
    per_layer = H * d * d * g["state_bytes_per_value"]
    assert per_layer * g["kda_layers"] == g["kda_state_bytes"]
    const = g["kda_state_bytes"] + g["conv_tail_bytes_inferred"]
    assert const == g["constant_bytes"]
    assert round(const / 2 ** 20, 2) == g["constant_mib_printed"]
    assert g["kv_bytes_per_token_after"] * g["context"] + const == g["measured_cache_bytes"]
    L_star = const / (g["kv_bytes_per_token_before"] - g["kv_bytes_per_token_after"])
    assert round(L_star / 10) * 10 == g["equal_memory_context_printed"]
    assert 128 * 128 == g["d128_state_values"]
    assert g["kv_values_per_token_d128"] * g["kv_context_262k"] // g["d128_state_values"] == \
        g["kv_over_state_at_262k"]


def test_chunk_form_matches_recurrence():
    """The chunked form (numpy, from its definition) equals the token
    recurrence: full and partial chunks, several sequences, scalar and
    per-channel decay, non-zero initial state."""
    r = _rng(10)
    lengths = [130, 64, 1, 63]
    T, H, d = sum(lengths), 2, 8
    cu = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int32)
    q = _unit(r.standard_normal((T, H, d)))
    k = _unit(r.standard_normal((T, H, d)))
    v = r.standard_normal((T, H, d))
    beta = 1 / (1 + np.exp(-r.standard_normal((T, H))))
    S0 = 0.1 * r.standard_normal((len(lengths), H, d, d))
    for scalar in (False, True):
        la = -np.log1p(np.exp(-(3 + 2 * r.standard_normal((T, H) if scalar else (T, H, d)))))
        ref = oracle.prefill(q, k, v, beta, la, cu, scalar_decay=scalar, scale=0.5, init_state=S0)
        for affine in (False, True):
            ch = oracle.chunked_prefill(q, k, v, beta, la, cu, scalar_decay=scalar, scale=0.5,
                                        init_state=S0, affine=affine)
            np.testing.assert_allclose(ch["o"], ref["o"], rtol=0, atol=1e-10)
            np.testing.assert_allclose(ch["final_state"], ref["final_state"], rtol=0, atol=1e-10)


def test_cumdecay_restarts_per_chunk():
    """exp of the chunk-local sum is the product of the gates since the
    chunk's first token; chunks start at every sequence start and every 64
    tokens after it."""
    r = _rng(11)
    lengths = [70, 5, 128]
    cu = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int32)
    la = -r.random((sum(lengths), 2, 3))
    g = oracle.cumdecay(la, cu)
    starts = {s for _, s, _ in oracle.chunk_bounds(cu)}
    assert starts == {0, 64, 70, 75, 139}
    for t in range(sum(lengths)):
        s = max(x for x in starts if x <= t)
        np.testing.assert_allclose(np.exp(g[t]), np.prod(np.exp(la[s:t + 1]), axis=0), rtol=1e-12)


MUTANTS = list(range(1, 13))


@pytest.mark.parametrize("mutant", MUTANTS)
def test_every_planted_mistake_is_caught(mutant):
    """Each compile-time mutant of the C oracle (wrong read order, decay on
    the wrong axis, sign, dropped beta, q/k swap, decay after the update,
    snapshot off by one, wrong head's gate, transposed state, draft keeping
    the state from before each token, rollback one token too far) must fail
    at least one pin."""
    caught = []
    for pin in PINS:
        try:
            pin(mutant)
        except AssertionError:
            caught.append(pin.__name__)
    assert caught, f"mutant {mutant} passed every pin"


def test_zero_channel_widening_is_exact():
    """Widening the key side (q = k = 0, log a = 0) or the value side (v = 0)
    with zero channels changes nothing in the original channels and leaves the
    extra state rows / columns at zero -- the property that lets a d_k != d_v
    prefill run on square D x D states, D = max(d_k, d_v)."""
    import workloads as wl

    def widen(x, D):
        y = torch.zeros(*x.shape[:-1], D, dtype=x.dtype)
        y[..., :x.shape[-1]] = x
        return y

    for dk, dv in ((64, 128), (128, 64)):
        w = wl.shrink(wl.VARLEN, n_heads=2, d_k=dk, d_v=dv, lengths=(70, 5, 64), init_std=0.1,
                      snap_interval=64)
        x = wl.make_prefill_inputs(w)
        ref = oracle.prefill(x["q"], x["k"], x["v"], x["beta"], x["log_a"], x["cu_seqlens"],
                             init_state=x["init_state"], snap_interval=64)
        D = max(dk, dv)
        init = torch.zeros(3, 2, D, D)
        init[:, :, :dv, :dk] = x["init_state"]
        wide = oracle.prefill(widen(x["q"], D), widen(x["k"], D), widen(x["v"], D), x["beta"],
                              widen(x["log_a"], D), x["cu_seqlens"], init_state=init,
                              snap_interval=64)
        assert np.array_equal(wide["o"][..., :dv], ref["o"])
        assert not wide["o"][..., dv:].any()
        for name in ("final_state", "snapshots"):
            assert np.array_equal(wide[name][..., :dv, :dk], ref[name])
            assert not wide[name][..., dv:, :].any() and not wide[name][..., :, dk:].any()
