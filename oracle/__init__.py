"""fp64 CPU oracle for the gated delta rule -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` /
``--impl reference`` legs of ``bench.py`` may import this package.  The CUDA
library never imports, links or calls it, and it imports nothing from the
CUDA library.

Contents
--------
* ``prefill`` / ``decode_step``: the token-by-token recurrence in plain C
  (``gdr_oracle.c``, fp64, OpenMP over (sequence, head)), wrapped with ctypes.
* ``output_epilogue``: the per-head RMSNorm of o and the sigmoid output gate
  that follow the mixer (numpy, fp64).
* ``decode_draft`` / ``decode_accept``: speculative decoding with rollback --
  K draft tokens that keep the state after each token, then the state of the
  accepted prefix (same C file).
* ``cumdecay``: chunk-local inclusive prefix sums of log a (numpy, fp64).
* ``preprocess``: the mixer's input activations from raw projections -- the
  causal depthwise conv of width 4 on q, k, v, L2 norm of q and k, beta as a
  sigmoid and log a as a log-sigmoid of the biased gate (numpy, fp64).
* ``chunk_factors`` / ``chunked_prefill``: the chunked form of the same
  recurrence written from its definition (numpy, fp64).  It is used to check
  the intermediate results of the intra-chunk kernel; it is itself pinned by
  equality with the token recurrence in the tests.

Every function states the passage it follows.  Inputs are widened to fp64
exactly (bf16 -> fp32 -> fp64 is exact), so the oracle sees the very bits the
GPU receives.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "gdr_oracle.c")
_BUILD = os.path.join(_HERE, "_build")
_LOCK = threading.Lock()
_LIBS: dict = {}

_dp = ctypes.POINTER(ctypes.c_double)
_ip = ctypes.POINTER(ctypes.c_int32)


def lib_path(mutant: int = 0) -> str:
    name = "liboracle.so" if mutant == 0 else f"liboracle_mutant{mutant}.so"
    return os.path.join(_BUILD, name)


def build(mutant: int = 0, force: bool = False) -> str:
    """Compile the C oracle with gcc (-O2 -fopenmp, strict IEEE fp64)."""
    path = lib_path(mutant)
    if not force and os.path.exists(path) and os.path.getmtime(path) >= os.path.getmtime(_SRC):
        return path
    os.makedirs(_BUILD, exist_ok=True)
    tmp = path + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c99",
           f"-DGDR_ORACLE_MUTANT={int(mutant)}", _SRC, "-o", tmp, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, path)
    return path


def _load(mutant: int = 0):
    with _LOCK:
        if mutant not in _LIBS:
            lib = ctypes.CDLL(build(mutant))
            lib.gdr_oracle_prefill.restype = ctypes.c_int
            lib.gdr_oracle_prefill.argtypes = [
                ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, _ip,
                _dp, _dp, _dp, _dp, _dp, ctypes.c_int, ctypes.c_double, _dp, _dp, _dp,
                ctypes.c_int, _dp]
            lib.gdr_oracle_decode_step.restype = ctypes.c_int
            lib.gdr_oracle_decode_step.argtypes = [
                ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                _dp, _dp, _dp, _dp, _dp, ctypes.c_int, ctypes.c_double, _dp, _dp]
            lib.gdr_oracle_decode_draft.restype = ctypes.c_int
            lib.gdr_oracle_decode_draft.argtypes = [
                ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                _dp, _dp, _dp, _dp, _dp, ctypes.c_int, ctypes.c_double, _dp, _dp, _dp]
            lib.gdr_oracle_decode_accept.restype = ctypes.c_int
            lib.gdr_oracle_decode_accept.argtypes = [
                ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                _ip, _dp, _dp]
            lib.gdr_oracle_snapshot_count.restype = ctypes.c_int64
            lib.gdr_oracle_snapshot_count.argtypes = [ctypes.c_int, _ip, ctypes.c_int]
            _LIBS[mutant] = lib
        return _LIBS[mutant]


def f64(x) -> np.ndarray:
    """Exact widening of a torch tensor (any float dtype) or array to fp64."""
    if x is None:
        return None
    if hasattr(x, "detach"):
        x = x.detach().cpu()
        if x.dtype != __import__("torch").float64:
            x = x.float().double()
        x = x.numpy()
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def _i32(x) -> np.ndarray:
    if hasattr(x, "detach"):
        x = x.detach().cpu().numpy()
    return np.ascontiguousarray(np.asarray(x, dtype=np.int32))


def _ptr(a):
    return None if a is None else a.ctypes.data_as(_dp)


def snapshot_count(cu_seqlens, snap_interval: int, mutant: int = 0) -> int:
    cu = _i32(cu_seqlens)
    return int(_load(mutant).gdr_oracle_snapshot_count(len(cu) - 1, cu.ctypes.data_as(_ip),
                                                        int(snap_interval)))


def prefill(q, k, v, beta, log_a, cu_seqlens, scalar_decay=False, scale=1.0,
            init_state=None, snap_interval=0, mutant: int = 0) -> dict:
    """Token-by-token recurrence over a packed batch (fp64).

    Follows "Modele hybrydowe: co Gated DeltaNet zastępuje w cache KV",
    sections "Atencja liniowa", "Reguła delta" and "Gated DeltaNet: dodaj
    zanik", with the per-key-channel decay of KDA; snapshots after every full
    ``snap_interval`` tokens per section "Co stan rekurencyjny zmienia przy
    serwowaniu", point 1.  Returns dict(o, final_state, snapshots).
    """
    q, k, v, beta, log_a = (f64(x) for x in (q, k, v, beta, log_a))
    cu = _i32(cu_seqlens)
    T, H, dk = q.shape
    dv = v.shape[2]
    n = len(cu) - 1
    init = f64(init_state)
    o = np.zeros((T, H, dv))
    fin = np.zeros((n, H, dv, dk))
    ns = snapshot_count(cu, snap_interval, mutant) if snap_interval > 0 else 0
    snaps = np.zeros((max(ns, 1), H, dv, dk))
    rc = _load(mutant).gdr_oracle_prefill(
        n, H, dk, dv, cu.ctypes.data_as(_ip), _ptr(q), _ptr(k), _ptr(v), _ptr(beta),
        _ptr(log_a), int(bool(scalar_decay)), float(scale), _ptr(init), _ptr(o), _ptr(fin),
        int(snap_interval), _ptr(snaps))
    if rc != 0:
        raise ValueError("oracle prefill rejected its arguments")
    return dict(o=o, final_state=fin, snapshots=snaps[:ns])


def decode_step(state, q, k, v, beta, log_a, scalar_decay=False, scale=1.0,
                mutant: int = 0):
    """One token of the recurrence for B independent sequences (fp64).

    Follows the same passages as ``prefill`` with T = 1 ("kda-graft", section
    "2. Decode: O(1) против O(L)": the step cost does not depend on context
    length).  Returns (new_state, o); the input state is not modified.
    """
    S = f64(state).copy()
    q, k, v, beta, log_a = (f64(x) for x in (q, k, v, beta, log_a))
    B, H, dk = q.shape
    dv = v.shape[2]
    o = np.zeros((B, H, dv))
    rc = _load(mutant).gdr_oracle_decode_step(
        B, H, dk, dv, _ptr(q), _ptr(k), _ptr(v), _ptr(beta), _ptr(log_a),
        int(bool(scalar_decay)), float(scale), _ptr(S), _ptr(o))
    if rc != 0:
        raise ValueError("oracle decode rejected its arguments")
    return S, o


def decode_draft(state, q, k, v, beta, log_a, scalar_decay=False, scale=1.0,
                 mutant: int = 0):
    """K draft tokens per sequence for speculative decoding (fp64).

    "Modele hybrydowe ...", section "Co stan rekurencyjny zmienia przy
    serwowaniu", point 2: the recurrent state absorbs draft tokens, so a
    rejected draft can only be undone from a state kept before it.  Runs the
    token update K times from ``state`` [B, H, dv, dk] (not modified) on
    q, k [B, K, H, dk], v [B, K, H, dv], beta [B, K, H], log_a [B, K, H, dk]
    (or [B, K, H]).  Returns (o [B, K, H, dv], token_states [B, K, H, dv, dk]),
    token_states[b, t] being the state after token t.
    """
    S = f64(state)
    q, k, v, beta, log_a = (f64(x) for x in (q, k, v, beta, log_a))
    B, K, H, dk = q.shape
    dv = v.shape[3]
    o = np.zeros((B, K, H, dv))
    ts = np.zeros((B, K, H, dv, dk))
    rc = _load(mutant).gdr_oracle_decode_draft(
        B, K, H, dk, dv, _ptr(q), _ptr(k), _ptr(v), _ptr(beta), _ptr(log_a),
        int(bool(scalar_decay)), float(scale), _ptr(S), _ptr(o), _ptr(ts))
    if rc != 0:
        raise ValueError("oracle draft decode rejected its arguments")
    return o, ts


def decode_accept(state, token_states, n_accept, mutant: int = 0) -> np.ndarray:
    """Rollback after verification (same passage as ``decode_draft``): the
    state of sequence b becomes token_states[b, n - 1] for n = n_accept[b] in
    1 .. K and stays ``state[b]`` for n = 0 (n clamped to [0, K]).  Returns
    the new state; the input is not modified."""
    S = f64(state).copy()
    ts = f64(token_states)
    n = _i32(n_accept)
    B, K, H, dv, dk = ts.shape
    rc = _load(mutant).gdr_oracle_decode_accept(B, K, H, dk, dv, n.ctypes.data_as(_ip),
                                                _ptr(ts), _ptr(S))
    if rc != 0:
        raise ValueError("oracle decode accept rejected its arguments")
    return S


# ---------------------------------------------------------------------------
# Chunked form (numpy, fp64), written from the recurrence's definition.
#
# "Modele hybrydowe ...", section "Co stan rekurencyjny zmienia przy
# serwowaniu", last paragraph: prefill runs in chunks; inside a chunk the
# updates are dense matrix products and only the step from chunk to chunk is
# sequential.  The pages print no formulas for it; the algebra below unrolls
# the token recurrence over one chunk with start state S0.
# ---------------------------------------------------------------------------

def chunk_bounds(cu_seqlens, chunk: int = 64):
    """List of (seq, start, end) per chunk: chunks restart at every sequence
    start and the last chunk of a sequence may be partial."""
    cu = _i32(cu_seqlens)
    out = []
    for n in range(len(cu) - 1):
        for s in range(int(cu[n]), int(cu[n + 1]), chunk):
            out.append((n, s, min(s + chunk, int(cu[n + 1]))))
    return out


def cumdecay(log_a, cu_seqlens, chunk: int = 64) -> np.ndarray:
    """g[t] = sum of log_a over the tokens of t's chunk up to and including t."""
    la = f64(log_a)
    g = np.zeros_like(la)
    for _, s, e in chunk_bounds(cu_seqlens, chunk):
        g[s:e] = np.cumsum(la[s:e], axis=0)
    return g


def chunk_factors(q, k, v, beta, log_a, start, end, h, scalar_decay=False, scale=1.0):
    """Per-chunk factors for tokens [start, end) of head h (fp64).

    With g_r the chunk-local cumulative log decay and Gamma_r = exp(g_r):
      A[r,i]  = beta_r sum_c k[r,c] k[i,c] exp(g[r,c]-g[i,c])   for i < r
      P[r,i]  = scale sum_c q[r,c] k[i,c] exp(g[r,c]-g[i,c])    for i <= r
      T       = (I + A)^-1
      W       = T diag(beta) (K * Gamma)       U = T diag(beta) V
      Qg      = scale Q * Gamma                Kd = K * exp(g_last - g)
      gamma_C = exp(g_last)
    so that, for start state S0, Delta = U - W S0^T, the outputs are
    O = Qg S0^T + P Delta and the end state is S0 Diag(gamma_C) + Delta^T Kd.
    Substituting Delta gives the same map with S0-free matrices
    Qt = Qg - P W, PU = P U, BS = -Kd^T W, NC = U^T Kd:
    O = Qt S0^T + PU and S_next = S0 Diag(gamma_C) + S0 BS^T + NC.
    """
    Q = f64(q)[start:end, h]
    K = f64(k)[start:end, h]
    V = f64(v)[start:end, h]
    b = f64(beta)[start:end, h]
    la = f64(log_a)[start:end, h]
    L, dk = Q.shape
    if scalar_decay:
        la = np.repeat(la[:, None], dk, axis=1)
    g = np.cumsum(la, axis=0)
    gam = np.exp(g)
    # decay-weighted products, term by term exp(g_r - g_i) (no factoring)
    # exp(g_r - g_i) for i <= r only (the other entries are masked out below)
    low = np.tril(np.ones((L, L), dtype=bool))[:, :, None]
    D = np.exp(np.where(low, g[:, None, :] - g[None, :, :], -np.inf))   # [r, i, c]
    KK = np.einsum("rc,ic,ric->ri", K, K, D)
    QK = np.einsum("rc,ic,ric->ri", Q, K, D)
    A = np.tril(b[:, None] * KK, -1)
    P = scale * np.tril(QK, 0)
    Tm = np.linalg.inv(np.eye(L) + A)
    W = Tm @ (b[:, None] * K * gam)
    U = Tm @ (b[:, None] * V)
    Qg = scale * Q * gam
    Kd = K * np.exp(g[-1][None, :] - g)
    # the chunk as an affine map of S0: S_next = S0 Diag(gamma_C) + S0 BS^T + NC,
    # O = Qt S0^T + PU (Delta = U - W S0^T substituted)
    return dict(A=A, P=P, T=Tm, W=W, U=U, Qg=Qg, Kd=Kd, gamma_C=gam[-1], g=g,
                Qt=Qg - P @ W, PU=P @ U, BS=-(Kd.T @ W), NC=U.T @ Kd)


def chunked_prefill(q, k, v, beta, log_a, cu_seqlens, scalar_decay=False, scale=1.0,
                    init_state=None, chunk: int = 64, affine: bool = False):
    """Prefill through the chunked form (fp64); must equal ``prefill``.
    ``affine`` uses the S0-free map (Qt, PU, BS, NC) instead of Delta."""
    q64, k64, v64 = f64(q), f64(k), f64(v)
    T, H, dk = q64.shape
    dv = v64.shape[2]
    cu = _i32(cu_seqlens)
    n = len(cu) - 1
    o = np.zeros((T, H, dv))
    fin = np.zeros((n, H, dv, dk)) if init_state is None else f64(init_state).copy()
    for s_idx, s, e in chunk_bounds(cu, chunk):
        for h in range(H):
            f = chunk_factors(q64, k64, v64, beta, log_a, s, e, h, scalar_decay, scale)
            S0 = fin[s_idx, h]
            if affine:
                o[s:e, h] = f["Qt"] @ S0.T + f["PU"]
                fin[s_idx, h] = S0 * f["gamma_C"][None, :] + S0 @ f["BS"].T + f["NC"]
            else:
                Delta = f["U"] - f["W"] @ S0.T
                o[s:e, h] = f["Qg"] @ S0.T + f["P"] @ Delta
                fin[s_idx, h] = S0 * f["gamma_C"][None, :] + Delta.T @ f["Kd"]
    return dict(o=o, final_state=fin)


# ---------------------------------------------------------------------------
# Input activations (numpy, fp64).
#
# "kda-graft: Qwen2.5-0.5B с трансплантированным KDA", section "Идея и
# архитектура": the graft adds a width-4 convolution (initialised as an
# identity tap), the alpha gate with bias +5 (sigma(5) ~ 0.993), the write
# strength beta, an output gate and an RMSNorm around the q/k/v projections.
# The page gives no formulas; the readings taken are stated per function.
# ---------------------------------------------------------------------------

def _conv4(x, w, cu):
    """Causal depthwise conv of width 4 per sequence: for token t of a
    sequence starting at s, y[t, h, c] = sum_{j=0..3} w[h*d + c, j] x[t-3+j, h, c]
    over the taps with t-3+j >= s (zero history at every sequence start; tap 3
    is the current token, so w = [0, 0, 0, 1] is the identity)."""
    T, H, d = x.shape
    W = w.reshape(H, d, 4)
    y = np.zeros_like(x)
    for n in range(len(cu) - 1):
        s, e = int(cu[n]), int(cu[n + 1])
        for t in range(s, e):
            for j in range(4):
                tt = t - 3 + j
                if tt >= s:
                    y[t] += W[:, :, j] * x[tt]
    return y


def _l2norm(y):
    """y / max(||y||_2, 1e-12) per (token, head)."""
    nrm = np.sqrt(np.sum(y * y, axis=-1, keepdims=True))
    return y / np.maximum(nrm, 1e-12)


def sigmoid(z):
    """1 / (1 + exp(-z)), written with exp(-|z|) so that it never overflows."""
    e = np.exp(-np.abs(z))
    return np.where(z >= 0, 1.0 / (1.0 + e), e / (1.0 + e))


def log_sigmoid(z):
    """log(1 / (1 + exp(-z))) = min(z, 0) - log1p(exp(-|z|)) (no overflow)."""
    return np.minimum(z, 0.0) - np.log1p(np.exp(-np.abs(z)))


def preprocess(xq, xk, xv, conv_q, conv_k, conv_v, beta_raw, a_raw, a_bias, cu_seqlens,
               scalar_decay=False) -> dict:
    """Inputs of the recurrence from raw per-head projections (fp64).

    q = L2norm(conv4(xq)), k = L2norm(conv4(xk)), v = conv4(xv),
    beta = sigmoid(beta_raw), log a = log_sigmoid(a_raw + a_bias).
    Readings: no activation after the conv (the page names none); q and k
    are L2-normalised per (token, head) after the conv; the bias is per
    (head, key channel), or per head with a scalar gate.  Shapes: xq, xk
    [T, H, d_k], xv [T, H, d_v], conv_* [H * d, 4], beta_raw [T, H], a_raw
    [T, H, d_k] with a_bias [H, d_k] (or [T, H] with [H]).
    """
    cu = _i32(cu_seqlens)
    xq, xk, xv = f64(xq), f64(xk), f64(xv)
    q = _l2norm(_conv4(xq, f64(conv_q), cu))
    k = _l2norm(_conv4(xk, f64(conv_k), cu))
    v = _conv4(xv, f64(conv_v), cu)
    beta = sigmoid(f64(beta_raw))
    z = f64(a_raw) + f64(a_bias)[None]
    return dict(q=q, k=k, v=v, beta=beta, log_a=log_sigmoid(z))


def output_epilogue(o, gate_raw, norm_weight, eps: float = 1e-6) -> np.ndarray:
    """The mixer's output after its RMSNorm and output gate (fp64).

    "kda-graft", section "Идея и архитектура": the graft adds an output gate
    and an RMSNorm to each KDA layer; the page gives no formulas.  Readings:
    the norm runs over the d_v channels of each (token, head) with one weight
    vector [d_v] shared by the heads and eps = 1e-6; the gate is the sigmoid of
    a raw gate projection [T, H, d_v]:
        y = o / sqrt(mean_c o_c^2 + eps) * norm_weight * sigmoid(gate_raw)
    """
    o = f64(o)
    ms = np.mean(o * o, axis=-1, keepdims=True)
    return o / np.sqrt(ms + eps) * f64(norm_weight) * sigmoid(f64(gate_raw))
