"""Gated delta-rule prefill and decode on B200 (sm_100a).

A thin ctypes binding over the C ABI in ``include/gdr.h``.  Every function
here only checks and marshals torch tensors (device pointers, sizes and the
current CUDA stream) into one library call; all arithmetic runs in the CUDA
kernels of ``libgdr.so``.  There is no CPU or PyTorch fallback: if the
library is missing, every call raises.

Layouts (token-major, sequences packed by ``cu_seqlens``):
  q, k [T, H, d_k]   v, o [T, H, d_v]   beta [T, H] fp32
  log_a [T, H, d_k] fp32 (per-channel decay) or [T, H] (scalar decay)
  state [N, H, d_v, d_k] fp32, row = value channel, column = key channel
"""
from __future__ import annotations

import ctypes
import os
import threading

import torch

__all__ = ["PrefillArgs", "PreparedPrefill", "prefill", "kernel_count", "decode_step",
           "decode_draft", "decode_accept", "PreprocessArgs", "preprocess", "Projections",
           "prefill_from_projections", "cumdecay", "chunk_factors", "workspace_size",
           "projections_workspace_size",
           "snapshot_count", "snapshot_offsets", "snapshot_offload", "prefill_status", "lib", "GdrError", "LIB_PATH"]

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "_build", "libgdr.so")

GDR_OK = 0
_STATUS = {0: "GDR_OK", 1: "GDR_ERR_INVALID_ARG", 2: "GDR_ERR_UNSUPPORTED",
           3: "GDR_ERR_WORKSPACE", 4: "GDR_ERR_CUDA", 5: "GDR_ERR_TIMEOUT"}
GDR_BF16, GDR_F32 = 0, 1


class GdrError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {_STATUS.get(status, status)}")


class PrefillArgs(ctypes.Structure):
    """Mirror of ``gdr_prefill_args`` (include/gdr.h)."""
    _fields_ = [
        ("n_seqs", ctypes.c_int), ("n_heads", ctypes.c_int), ("d_k", ctypes.c_int),
        ("d_v", ctypes.c_int), ("total_tokens", ctypes.c_int64),
        ("cu_seqlens", ctypes.c_void_p), ("qkv_dtype", ctypes.c_int),
        ("q", ctypes.c_void_p), ("k", ctypes.c_void_p), ("v", ctypes.c_void_p),
        ("beta", ctypes.c_void_p), ("log_a", ctypes.c_void_p), ("scalar_decay", ctypes.c_int),
        ("scale", ctypes.c_float), ("init_state", ctypes.c_void_p), ("o", ctypes.c_void_p),
        ("final_state", ctypes.c_void_p), ("snap_interval", ctypes.c_int),
        ("snapshots", ctypes.c_void_p), ("snap_offsets", ctypes.c_void_p),
        ("gate_raw", ctypes.c_void_p), ("norm_weight", ctypes.c_void_p),
        ("norm_eps", ctypes.c_float), ("workspace", ctypes.c_void_p),
        ("workspace_bytes", ctypes.c_size_t),
    ]


class Projections(ctypes.Structure):
    """Mirror of ``gdr_projections`` (include/gdr.h)."""
    _fields_ = [
        ("xq", ctypes.c_void_p), ("xk", ctypes.c_void_p), ("xv", ctypes.c_void_p),
        ("conv_q", ctypes.c_void_p), ("conv_k", ctypes.c_void_p), ("conv_v", ctypes.c_void_p),
        ("beta_raw", ctypes.c_void_p), ("a_raw", ctypes.c_void_p), ("a_bias", ctypes.c_void_p),
    ]


class PreprocessArgs(ctypes.Structure):
    """Mirror of ``gdr_preprocess_args`` (include/gdr.h)."""
    _fields_ = [
        ("n_seqs", ctypes.c_int), ("n_heads", ctypes.c_int), ("d", ctypes.c_int),
        ("total_tokens", ctypes.c_int64), ("cu_seqlens", ctypes.c_void_p),
        ("io_dtype", ctypes.c_int), ("xq", ctypes.c_void_p), ("xk", ctypes.c_void_p),
        ("xv", ctypes.c_void_p), ("conv_q", ctypes.c_void_p), ("conv_k", ctypes.c_void_p),
        ("conv_v", ctypes.c_void_p), ("beta_raw", ctypes.c_void_p), ("a_raw", ctypes.c_void_p),
        ("a_bias", ctypes.c_void_p), ("scalar_decay", ctypes.c_int), ("q", ctypes.c_void_p),
        ("k", ctypes.c_void_p), ("v", ctypes.c_void_p), ("beta", ctypes.c_void_p),
        ("log_a", ctypes.c_void_p),
    ]


_LOCK = threading.Lock()
_LIB = None


def lib():
    """Load libgdr.so (raises if it has not been built)."""
    global _LIB
    with _LOCK:
        if _LIB is None:
            if not os.path.exists(LIB_PATH):
                raise RuntimeError(f"CUDA library not built: {LIB_PATH} is missing "
                                   "(run python -m gated_delta_rule_150_b200.build)")
            L = ctypes.CDLL(LIB_PATH)
            vp, i, i64, f = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_float
            L.gdr_status_string.restype = ctypes.c_char_p
            L.gdr_status_string.argtypes = [i]
            L.gdr_version.restype = i
            L.gdr_prefill_workspace_size.restype = ctypes.c_size_t
            L.gdr_prefill_workspace_size.argtypes = [i, i, i, i, i64, i]
            L.gdr_prefill_from_projections_workspace_size.restype = ctypes.c_size_t
            L.gdr_prefill_from_projections_workspace_size.argtypes = [i, i, i, i64, i]
            L.gdr_prefill_kernel_count.restype = i
            L.gdr_prefill_kernel_count.argtypes = [i, i, i, i, i64, i]
            L.gdr_snapshot_count.restype = i64
            L.gdr_snapshot_count.argtypes = [vp, i, i]
            L.gdr_snapshot_offsets.restype = i
            L.gdr_snapshot_offsets.argtypes = [vp, i, i, vp]
            L.gdr_snapshot_offload.restype = i
            L.gdr_snapshot_offload.argtypes = [vp, vp, ctypes.c_size_t, vp, vp, vp]
            L.gdr_prefill_static_workspace.restype = i
            L.gdr_prefill_static_workspace.argtypes = [ctypes.POINTER(PrefillArgs), vp]
            L.gdr_prefill_static_status.restype = i
            L.gdr_prefill_static_status.argtypes = [vp]
            L.gdr_prefill.restype = i
            L.gdr_prefill.argtypes = [ctypes.POINTER(PrefillArgs), vp]
            L.gdr_prefill_stages.restype = i
            L.gdr_prefill_stages.argtypes = [ctypes.POINTER(PrefillArgs), i, i, vp]
            L.gdr_prefill_status.restype = i
            L.gdr_prefill_status.argtypes = [vp, vp]
            L.gdr_cumdecay.restype = i
            L.gdr_cumdecay.argtypes = [i, i, i, i64, vp, vp, i, vp, vp]
            L.gdr_chunk_factors.restype = i
            L.gdr_chunk_factors.argtypes = [ctypes.POINTER(PrefillArgs), vp, vp, vp, vp, vp, vp]
            L.gdr_decode_step.restype = i
            L.gdr_decode_step.argtypes = [i, i, i, i, i, vp, vp, vp, vp, vp, i, f, vp, vp, vp]
            L.gdr_decode_step_gated.restype = i
            L.gdr_decode_step_gated.argtypes = [i, i, i, i, i, vp, vp, vp, vp, vp, i, f, vp, vp,
                                                vp, f, vp, vp]
            L.gdr_prefill_from_projections.restype = i
            L.gdr_prefill_from_projections.argtypes = [ctypes.POINTER(PrefillArgs),
                                                       ctypes.POINTER(Projections), vp]
            L.gdr_preprocess.restype = i
            L.gdr_preprocess.argtypes = [ctypes.POINTER(PreprocessArgs), vp]
            L.gdr_decode_draft.restype = i
            L.gdr_decode_draft.argtypes = [i, i, i, i, i, i, vp, vp, vp, vp, vp, i, f, vp, vp,
                                           vp, vp]
            L.gdr_decode_accept.restype = i
            L.gdr_decode_accept.argtypes = [i, i, i, i, i, vp, vp, vp, vp]
            _LIB = L
        return _LIB


def _check(status: int, what: str):
    if status != GDR_OK:
        raise GdrError(status, what)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(device) -> ctypes.c_void_p:
    return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return GDR_BF16
    if t.dtype == torch.float32:
        return GDR_F32
    raise TypeError(f"q/k/v must be bfloat16 or float32, got {t.dtype}")


def _need_cuda(*ts):
    for t in ts:
        if t is not None:
            if not t.is_cuda:
                raise ValueError("all tensors must be CUDA tensors")
            if not t.is_contiguous():
                raise ValueError("all tensors must be contiguous")


def _check_snapshot_buffer(snapshots):
    """Snapshots go to device memory or, for offload, to page-locked host
    memory that the kernels write over the host link."""
    if snapshots is None:
        return
    if not snapshots.is_contiguous():
        raise ValueError("snapshots must be contiguous")
    if not (snapshots.is_cuda or snapshots.is_pinned()):
        raise ValueError("snapshots must be a CUDA tensor or pinned host memory")


def _expect(t, shape, dtype, name):
    """Raise unless ``t`` (when given) has exactly ``shape`` and ``dtype``.

    The C ABI receives bare pointers and sizes, so a tensor of the wrong shape
    would be read or written past its end by the kernels; every binding
    checks its tensors' shapes here, on the host, before anything else."""
    if t is None:
        return
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")


def _expect_dim(t, dim, name):
    if t.dim() != dim:
        raise ValueError(f"{name} must have {dim} dimensions, got shape {tuple(t.shape)}")


def _check_cu(cu_seqlens, total_tokens, cu_host=None):
    """cu_seqlens: int32, one dimension, N + 1 >= 1 entries; the host copy,
    when there is one, must start at 0, never decrease and end at T."""
    if cu_seqlens.dtype != torch.int32 or cu_seqlens.dim() != 1 or cu_seqlens.numel() < 1:
        raise ValueError("cu_seqlens must be a 1-D int32 tensor with N + 1 >= 1 entries")
    if cu_host is not None:
        c = torch.as_tensor(cu_host, dtype=torch.int64).reshape(-1)
        if c.numel() != cu_seqlens.numel():
            raise ValueError("cu_seqlens_host and cu_seqlens differ in length")
        if int(c[0]) != 0 or int(c[-1]) != total_tokens or bool((c[1:] < c[:-1]).any()):
            raise ValueError("cu_seqlens must start at 0, never decrease and end at the "
                             "number of tokens")


def _check_prefill_shapes(q, k, v, beta, log_a, cu_seqlens, scalar_decay, init_state=None,
                          out=None, final_state=None, snapshots=None, cu_host=None,
                          snap_interval=0):
    _expect_dim(q, 3, "q")
    _expect_dim(v, 3, "v")
    T, H, dk = q.shape
    dv = v.shape[-1]
    _dtype_code(q)
    _expect(k, (T, H, dk), q.dtype, "k")
    _expect(v, (T, H, dv), q.dtype, "v")
    _expect(beta, (T, H), torch.float32, "beta")
    _expect(log_a, (T, H) if scalar_decay else (T, H, dk), torch.float32, "log_a")
    _check_cu(cu_seqlens, T, cu_host)
    n = cu_seqlens.numel() - 1
    _expect(init_state, (n, H, dv, dk), torch.float32, "init_state")
    _expect(out, (T, H, dv), q.dtype, "out")
    _expect(final_state, (n, H, dv, dk), torch.float32, "final_state")
    if snapshots is not None:
        if snapshots.dim() != 4 or tuple(snapshots.shape[1:]) != (H, dv, dk) or \
                snapshots.dtype != torch.float32:
            raise ValueError(f"snapshots must be float32 [S, {H}, {dv}, {dk}]")
        if cu_host is not None and snap_interval:
            need = snapshot_count(cu_host, snap_interval)
            if snapshots.shape[0] < need:
                raise ValueError(f"snapshots holds {snapshots.shape[0]} slots, {need} needed")


def _host_cu(cu_seqlens, cu_seqlens_host):
    if cu_seqlens_host is not None:
        return torch.as_tensor(cu_seqlens_host, dtype=torch.int32).contiguous()
    return cu_seqlens.detach().to("cpu", torch.int32).contiguous()


def workspace_size(n_seqs, n_heads, d_k, d_v, total_tokens, scalar_decay=False) -> int:
    return int(lib().gdr_prefill_workspace_size(n_seqs, n_heads, d_k, d_v, total_tokens,
                                                int(bool(scalar_decay))))


def projections_workspace_size(n_seqs, n_heads, d, total_tokens, scalar_decay=False) -> int:
    """Workspace of ``prefill_from_projections`` with room for the staged
    activations (larger than ``workspace_size`` only at d 128 with a
    per-channel gate)."""
    return int(lib().gdr_prefill_from_projections_workspace_size(n_seqs, n_heads, d, total_tokens,
                                                                 int(bool(scalar_decay))))


def kernel_count(n_seqs, n_heads, d_k, d_v, total_tokens, scalar_decay=False) -> int:
    """Kernel launches one gdr_prefill enqueues for these sizes."""
    return int(lib().gdr_prefill_kernel_count(n_seqs, n_heads, d_k, d_v, total_tokens,
                                              int(bool(scalar_decay))))


def snapshot_count(cu_seqlens_host, snap_interval: int) -> int:
    cu = torch.as_tensor(cu_seqlens_host, dtype=torch.int32).contiguous()
    n = int(lib().gdr_snapshot_count(ctypes.c_void_p(cu.data_ptr()), cu.numel() - 1,
                                     int(snap_interval)))
    if n < 0:
        raise GdrError(1, "gdr_snapshot_count")
    return n


def snapshot_offsets(cu_seqlens_host, snap_interval: int) -> torch.Tensor:
    """First snapshot slot of every sequence (int64 [N+1], host); entry N is
    the slot count.  Sequence n's m-th snapshot is slot offsets[n] + m - 1."""
    cu = torch.as_tensor(cu_seqlens_host, dtype=torch.int32).contiguous()
    out = torch.empty(cu.numel(), dtype=torch.int64)
    _check(lib().gdr_snapshot_offsets(ctypes.c_void_p(cu.data_ptr()), cu.numel() - 1,
                                      int(snap_interval), ctypes.c_void_p(out.data_ptr())),
           "gdr_snapshot_offsets")
    return out


def _check_gate(gate_raw, norm_weight, norm_eps, o_shape, dtype):
    """The output epilogue's inputs: raw gate shaped like o (o's dtype),
    weight [d_v] fp32, eps >= 0; both or neither."""
    if gate_raw is None and norm_weight is None:
        return
    if gate_raw is None or norm_weight is None:
        raise ValueError("the output epilogue needs both gate_raw and norm_weight")
    _expect(gate_raw, o_shape, dtype, "gate_raw")
    _expect(norm_weight, (o_shape[-1],), torch.float32, "norm_weight")
    if not norm_eps >= 0.0:
        raise ValueError("norm_eps must be >= 0")
    _need_cuda(gate_raw, norm_weight)


def _prefill_args(q, k, v, beta, log_a, cu_seqlens, scalar_decay, scale, init_state,
                  snap_interval, o, final_state, snapshots, workspace, snap_offsets=None,
                  gate_raw=None, norm_weight=None, norm_eps=1e-6):
    T, H, dk = q.shape
    a = PrefillArgs()
    a.n_seqs = cu_seqlens.numel() - 1
    a.n_heads = H
    a.d_k = dk
    a.d_v = v.shape[-1]
    a.total_tokens = T
    a.cu_seqlens = cu_seqlens.data_ptr()
    a.qkv_dtype = _dtype_code(q)
    a.q, a.k, a.v = q.data_ptr(), k.data_ptr(), v.data_ptr()
    a.beta, a.log_a = beta.data_ptr(), log_a.data_ptr()
    a.scalar_decay = int(bool(scalar_decay))
    a.scale = float(scale)
    a.init_state = None if init_state is None else init_state.data_ptr()
    a.o = None if o is None else o.data_ptr()
    a.final_state = None if final_state is None else final_state.data_ptr()
    a.snap_interval = int(snap_interval)
    a.snapshots = None if snapshots is None else snapshots.data_ptr()
    a.snap_offsets = None if snap_offsets is None else snap_offsets.data_ptr()
    a.gate_raw = None if gate_raw is None else gate_raw.data_ptr()
    a.norm_weight = None if norm_weight is None else norm_weight.data_ptr()
    a.norm_eps = float(norm_eps)
    a.workspace = workspace.data_ptr()
    a.workspace_bytes = workspace.numel()
    return a


def prefill(q, k, v, beta, log_a, cu_seqlens, *, scalar_decay=False, scale=1.0,
            init_state=None, snap_interval=0, cu_seqlens_host=None, out=None,
            final_state=None, snapshots=None, workspace=None, stages=(0, 1),
            snap_offsets=None, gate_raw=None, norm_weight=None, norm_eps=1e-6):
    """Chunked prefill over a packed batch.  Returns (o, final_state, snapshots).

    ``cu_seqlens`` is a device int32 tensor [N+1]; its host copy (taken from
    ``cu_seqlens_host`` when given, else read back) sizes the snapshots.
    Output buffers and the workspace may be passed in to avoid allocation.
    ``snap_offsets`` (device int64 [N+1], from ``snapshot_offsets``) gives
    each sequence's first snapshot slot to the kernels; ``snapshots`` may be
    pinned host memory (written by the kernels over the host link).
    ``gate_raw`` [T, H, d_v] (q's dtype) with ``norm_weight`` [d_v] fp32 turns
    on the output epilogue: o = RMSNorm(o) * norm_weight * sigmoid(gate_raw).
    ``stages`` = (first, last) runs only that range of the two stages
    (0 intra-chunk factors with the cumulative decay, 1 state pass), for
    timing them apart.
    """
    if q.dtype != k.dtype or q.dtype != v.dtype:
        raise TypeError("q, k and v must share a dtype")
    _check_prefill_shapes(q, k, v, beta, log_a, cu_seqlens, scalar_decay, init_state, out,
                          final_state, snapshots, cu_seqlens_host, snap_interval)
    if snap_offsets is not None:
        _expect(snap_offsets, (cu_seqlens.numel(),), torch.int64, "snap_offsets")
    _check_gate(gate_raw, norm_weight, norm_eps, (q.shape[0], q.shape[1], v.shape[-1]), q.dtype)
    _need_cuda(q, k, v, beta, log_a, cu_seqlens, init_state, out, final_state, workspace,
               snap_offsets)
    _check_snapshot_buffer(snapshots)
    T, H, dk = q.shape
    dv = v.shape[-1]
    n = cu_seqlens.numel() - 1
    dev = q.device
    if out is None:
        out = torch.empty(T, H, dv, dtype=q.dtype, device=dev)
    if final_state is None:
        final_state = torch.empty(n, H, dv, dk, dtype=torch.float32, device=dev)
    if snap_interval and snapshots is None:
        ns = snapshot_count(_host_cu(cu_seqlens, cu_seqlens_host), snap_interval)
        snapshots = torch.empty(max(ns, 1), H, dv, dk, dtype=torch.float32, device=dev)[:ns]
    if workspace is None:
        nbytes = workspace_size(n, H, dk, dv, T, scalar_decay)
        if nbytes == 0:
            raise GdrError(2, "gdr_prefill_workspace_size")
        workspace = torch.empty(nbytes, dtype=torch.uint8, device=dev)
    snap_arg = snapshots if (snap_interval and snapshots is not None and snapshots.numel()) else None
    if snap_interval and snap_arg is None:
        # no full interval in any sequence: any valid aligned pointer will do
        snap_arg = final_state
    a = _prefill_args(q, k, v, beta, log_a, cu_seqlens, scalar_decay, scale, init_state,
                      snap_interval, out, final_state, snap_arg, workspace, snap_offsets,
                      gate_raw, norm_weight, norm_eps)
    first, last = stages
    if (first, last) == (0, 1):
        _check(lib().gdr_prefill(ctypes.byref(a), _stream(dev)), "gdr_prefill")
    else:
        _check(lib().gdr_prefill_stages(ctypes.byref(a), int(first), int(last), _stream(dev)),
               "gdr_prefill_stages")
    return out, final_state, snapshots


class PreparedPrefill:
    """A prefill whose argument block is built once and replayed.

    Holds references to every tensor it points at.  ``run()`` enqueues one
    gdr_prefill (or a stage range) on the current stream of the tensors' device.
    """

    def __init__(self, q, k, v, beta, log_a, cu_seqlens, *, out, final_state, workspace,
                 scalar_decay=False, scale=1.0, init_state=None, snap_interval=0,
                 snapshots=None, gate_raw=None, norm_weight=None, norm_eps=1e-6):
        _check_prefill_shapes(q, k, v, beta, log_a, cu_seqlens, scalar_decay, init_state, out,
                              final_state, snapshots)
        if out is None or final_state is None or workspace is None:
            raise ValueError("PreparedPrefill needs out, final_state and workspace")
        _check_gate(gate_raw, norm_weight, norm_eps, tuple(out.shape), q.dtype)
        if snap_interval and snapshots is None:
            raise ValueError("snap_interval > 0 needs a snapshots buffer")
        _need_cuda(q, k, v, beta, log_a, cu_seqlens, out, final_state, workspace, init_state)
        _check_snapshot_buffer(snapshots)
        self._keep = (q, k, v, beta, log_a, cu_seqlens, out, final_state, workspace,
                      init_state, snapshots, gate_raw, norm_weight)
        self.args = _prefill_args(q, k, v, beta, log_a, cu_seqlens, scalar_decay, scale,
                                  init_state, snap_interval, out, final_state,
                                  snapshots if snap_interval else None, workspace, None,
                                  gate_raw, norm_weight, norm_eps)
        self.device = q.device
        self.out, self.final_state, self.snapshots, self.workspace = out, final_state, snapshots, workspace
        lib()

    def run(self, stages=(0, 1), stream=None):
        st = ctypes.c_void_p(stream.cuda_stream) if stream is not None else _stream(self.device)
        if tuple(stages) == (0, 1):
            _check(_LIB.gdr_prefill(ctypes.byref(self.args), st), "gdr_prefill")
        else:
            _check(_LIB.gdr_prefill_stages(ctypes.byref(self.args), int(stages[0]), int(stages[1]), st),
                   "gdr_prefill_stages")


def prefill_status(workspace) -> None:
    """Raise if the device side of the last prefill on ``workspace`` timed out."""
    _check(lib().gdr_prefill_status(_ptr(workspace), _stream(workspace.device)),
           "gdr_prefill_status")


def cumdecay(log_a, cu_seqlens, *, scalar_decay=False, d_k=None, out=None):
    """Chunk-local cumulative log decay (the first prefill kernel on its own)."""
    _expect_dim(log_a, 2 if scalar_decay else 3, "log_a")
    if log_a.dtype != torch.float32:
        raise TypeError("log_a must be float32")
    T, H = log_a.shape[0], log_a.shape[1]
    if scalar_decay and d_k is None:
        raise ValueError("a scalar gate needs d_k")
    dk = d_k if scalar_decay else log_a.shape[2]
    _check_cu(cu_seqlens, T)
    _expect(out, tuple(log_a.shape), torch.float32, "out")
    _need_cuda(log_a, cu_seqlens, out)
    if out is None:
        out = torch.empty_like(log_a)
    _check(lib().gdr_cumdecay(cu_seqlens.numel() - 1, H, dk, T, _ptr(cu_seqlens), _ptr(log_a),
                              int(bool(scalar_decay)), _ptr(out), _stream(log_a.device)),
           "gdr_cumdecay")
    return out


def chunk_factors(q, k, v, beta, log_a, cu_seqlens, *, scalar_decay=False, scale=1.0):
    """Per-chunk affine map of the state (Qt, PU, BS, NC, gamma) per chunk slot, fp32."""
    if q.dtype != k.dtype or q.dtype != v.dtype:
        raise TypeError("q, k and v must share a dtype")
    _check_prefill_shapes(q, k, v, beta, log_a, cu_seqlens, scalar_decay)
    _need_cuda(q, k, v, beta, log_a, cu_seqlens)
    T, H, dk = q.shape
    dv = v.shape[-1]
    n = cu_seqlens.numel() - 1
    dev = q.device
    slots = T // 64 + n
    f = dict(Qt=torch.zeros(slots, H, 64, dk, device=dev), PU=torch.zeros(slots, H, 64, dv, device=dev),
             BS=torch.zeros(slots, H, dk, dk, device=dev), NC=torch.zeros(slots, H, dv, dk, device=dev),
             gamma=torch.zeros(slots, H, dk, device=dev))
    workspace = torch.empty(workspace_size(n, H, dk, dv, T, scalar_decay), dtype=torch.uint8,
                            device=dev)
    a = _prefill_args(q, k, v, beta, log_a, cu_seqlens, scalar_decay, scale, None, 0, None,
                      None, None, workspace)
    _check(lib().gdr_chunk_factors(ctypes.byref(a), _ptr(f["Qt"]), _ptr(f["PU"]), _ptr(f["BS"]),
                                   _ptr(f["NC"]), _ptr(f["gamma"]), _stream(dev)),
           "gdr_chunk_factors")
    return f


def decode_step(state, q, k, v, beta, log_a, *, scalar_decay=False, scale=1.0, out=None,
                gate_raw=None, norm_weight=None, norm_eps=1e-6):
    """One decode step; ``state`` [B, H, d_v, d_k] fp32 is updated in place.
    Returns o [B, H, d_v] fp32 (after the output epilogue when ``gate_raw``
    [B, H, d_v] and ``norm_weight`` [d_v] are given)."""
    if q.dtype != k.dtype or q.dtype != v.dtype:
        raise TypeError("q, k and v must share a dtype")
    _expect_dim(q, 3, "q")
    _expect_dim(v, 3, "v")
    B, H, dk = q.shape
    dv = v.shape[-1]
    _dtype_code(q)
    _expect(k, (B, H, dk), q.dtype, "k")
    _expect(beta, (B, H), torch.float32, "beta")
    _expect(log_a, (B, H) if scalar_decay else (B, H, dk), torch.float32, "log_a")
    _expect(state, (B, H, dv, dk), torch.float32, "state")
    _expect(out, (B, H, dv), torch.float32, "out")
    _need_cuda(state, q, k, v, beta, log_a, out)
    _check_gate(gate_raw, norm_weight, norm_eps, (B, H, dv), q.dtype)
    if out is None:
        out = torch.empty(B, H, dv, dtype=torch.float32, device=q.device)
    if gate_raw is None:
        _check(lib().gdr_decode_step(B, H, dk, dv, _dtype_code(q), _ptr(q), _ptr(k), _ptr(v),
                                     _ptr(beta), _ptr(log_a), int(bool(scalar_decay)), float(scale),
                                     _ptr(state), _ptr(out), _stream(q.device)),
               "gdr_decode_step")
    else:
        _check(lib().gdr_decode_step_gated(B, H, dk, dv, _dtype_code(q), _ptr(q), _ptr(k), _ptr(v),
                                           _ptr(beta), _ptr(log_a), int(bool(scalar_decay)),
                                           float(scale), _ptr(state), _ptr(gate_raw),
                                           _ptr(norm_weight), float(norm_eps), _ptr(out),
                                           _stream(q.device)),
               "gdr_decode_step_gated")
    return out


def decode_draft(state, q, k, v, beta, log_a, *, scalar_decay=False, scale=1.0, out=None,
                 token_states=None):
    """K draft tokens per sequence for speculative decoding.

    ``state`` [B, H, d_v, d_k] fp32 is read, not modified.  q, k [B, K, H, d_k],
    v [B, K, H, d_v], beta [B, K, H], log_a [B, K, H, d_k] (or [B, K, H]).
    Returns (o [B, K, H, d_v] fp32, token_states [B, K, H, d_v, d_k] fp32),
    token_states[b, t] being the state after token t of sequence b.
    """
    if q.dtype != k.dtype or q.dtype != v.dtype:
        raise TypeError("q, k and v must share a dtype")
    _expect_dim(q, 4, "q")
    _expect_dim(v, 4, "v")
    B, K, H, dk = q.shape
    dv = v.shape[-1]
    _dtype_code(q)
    _expect(k, (B, K, H, dk), q.dtype, "k")
    _expect(v, (B, K, H, dv), q.dtype, "v")
    _expect(beta, (B, K, H), torch.float32, "beta")
    _expect(log_a, (B, K, H) if scalar_decay else (B, K, H, dk), torch.float32, "log_a")
    _expect(state, (B, H, dv, dk), torch.float32, "state")
    _expect(out, (B, K, H, dv), torch.float32, "out")
    _expect(token_states, (B, K, H, dv, dk), torch.float32, "token_states")
    _need_cuda(state, q, k, v, beta, log_a, out, token_states)
    if out is None:
        out = torch.empty(B, K, H, dv, dtype=torch.float32, device=q.device)
    if token_states is None:
        token_states = torch.empty(B, K, H, dv, dk, dtype=torch.float32, device=q.device)
    _check(lib().gdr_decode_draft(B, K, H, dk, dv, _dtype_code(q), _ptr(q), _ptr(k), _ptr(v),
                                  _ptr(beta), _ptr(log_a), int(bool(scalar_decay)), float(scale),
                                  _ptr(state), _ptr(out), _ptr(token_states), _stream(q.device)),
           "gdr_decode_draft")
    return out, token_states


def decode_accept(state, token_states, n_accept):
    """Rollback after verification, in place: ``state[b]`` becomes
    ``token_states[b, n - 1]`` for n = n_accept[b] in 1 .. K and is left as it
    is for n = 0 (n clamped to [0, K]).  ``n_accept`` is a device int32 [B]."""
    _expect_dim(token_states, 5, "token_states")
    B, K, H, dv, dk = token_states.shape
    _expect(token_states, (B, K, H, dv, dk), torch.float32, "token_states")
    _expect(state, (B, H, dv, dk), torch.float32, "state")
    _expect(n_accept, (B,), torch.int32, "n_accept")
    _need_cuda(state, token_states, n_accept)
    _check(lib().gdr_decode_accept(B, K, H, dk, dv, _ptr(n_accept), _ptr(token_states),
                                   _ptr(state), _stream(state.device)),
           "gdr_decode_accept")
    return state


def preprocess(xq, xk, xv, conv_q, conv_k, conv_v, beta_raw, a_raw, a_bias, cu_seqlens, *,
               scalar_decay=False, out=None):
    """The recurrence's inputs from raw per-head projections, in one kernel.

    xq, xk, xv [T, H, d] (bf16 or fp32), conv_* [H * d, 4] fp32 taps (tap 3 =
    current token), beta_raw [T, H], a_raw [T, H, d] with a_bias [H, d] (or
    [T, H] with [H] for a scalar gate).  Returns dict(q, k, v, beta, log_a) in
    the layouts ``prefill`` takes: q = L2norm(conv(xq)), k = L2norm(conv(xk)),
    v = conv(xv), beta = sigmoid(beta_raw), log_a = log_sigmoid(a_raw + a_bias).
    ``out`` may hold preallocated outputs under the same keys.
    """
    if xq.dtype != xk.dtype or xq.dtype != xv.dtype:
        raise TypeError("xq, xk and xv must share a dtype")
    _expect_dim(xq, 3, "xq")
    T, H, d = xq.shape
    _dtype_code(xq)
    for name, t in (("xk", xk), ("xv", xv)):
        _expect(t, (T, H, d), xq.dtype, name)
    for name, t in (("conv_q", conv_q), ("conv_k", conv_k), ("conv_v", conv_v)):
        _expect(t, (H * d, 4), torch.float32, name)
    _expect(beta_raw, (T, H), torch.float32, "beta_raw")
    _expect(a_raw, (T, H) if scalar_decay else (T, H, d), torch.float32, "a_raw")
    _expect(a_bias, (H,) if scalar_decay else (H, d), torch.float32, "a_bias")
    _check_cu(cu_seqlens, T)
    if out:
        for name in ("q", "k", "v"):
            _expect(out.get(name), (T, H, d), xq.dtype, f"out[{name!r}]")
        _expect(out.get("beta"), (T, H), torch.float32, "out['beta']")
        _expect(out.get("log_a"), tuple(a_raw.shape), torch.float32, "out['log_a']")
    dev = xq.device
    out = dict(out or {})
    for name in ("q", "k", "v"):
        if out.get(name) is None:
            out[name] = torch.empty(T, H, d, dtype=xq.dtype, device=dev)
    if out.get("beta") is None:
        out["beta"] = torch.empty(T, H, device=dev)
    if out.get("log_a") is None:
        out["log_a"] = torch.empty(a_raw.shape, device=dev)
    _need_cuda(xq, xk, xv, conv_q, conv_k, conv_v, beta_raw, a_raw, a_bias, cu_seqlens,
               *out.values())
    a = PreprocessArgs()
    a.n_seqs, a.n_heads, a.d, a.total_tokens = cu_seqlens.numel() - 1, H, d, T
    a.cu_seqlens = cu_seqlens.data_ptr()
    a.io_dtype = _dtype_code(xq)
    a.xq, a.xk, a.xv = xq.data_ptr(), xk.data_ptr(), xv.data_ptr()
    a.conv_q, a.conv_k, a.conv_v = conv_q.data_ptr(), conv_k.data_ptr(), conv_v.data_ptr()
    a.beta_raw, a.a_raw, a.a_bias = beta_raw.data_ptr(), a_raw.data_ptr(), a_bias.data_ptr()
    a.scalar_decay = int(bool(scalar_decay))
    a.q, a.k, a.v = out["q"].data_ptr(), out["k"].data_ptr(), out["v"].data_ptr()
    a.beta, a.log_a = out["beta"].data_ptr(), out["log_a"].data_ptr()
    _check(lib().gdr_preprocess(ctypes.byref(a), _stream(dev)), "gdr_preprocess")
    return out


def prefill_from_projections(xq, xk, xv, conv_q, conv_k, conv_v, beta_raw, a_raw, a_bias,
                             cu_seqlens, *, scalar_decay=False, scale=1.0, init_state=None,
                             snap_interval=0, cu_seqlens_host=None, out=None, final_state=None,
                             snapshots=None, workspace=None, gate_raw=None, norm_weight=None,
                             norm_eps=1e-6):
    """``preprocess`` and ``prefill`` in one: the input activations (conv-4, L2
    norm of q and k, beta and log-decay gates) are applied inside the
    prefill's first kernel, or, at d 128 with a per-channel gate and a
    workspace of ``projections_workspace_size`` bytes (the default), by their
    own kernel into the workspace (faster there).  Raw projections as for
    ``preprocess`` (bf16); the other arguments and the result (o,
    final_state, snapshots) as for ``prefill``."""
    if xq.dtype != torch.bfloat16 or xk.dtype != xq.dtype or xv.dtype != xq.dtype:
        raise TypeError("the fused path takes bf16 projections")
    _expect_dim(xq, 3, "xq")
    T, H, d = xq.shape
    for name, t in (("xk", xk), ("xv", xv)):
        _expect(t, (T, H, d), xq.dtype, name)
    for name, t in (("conv_q", conv_q), ("conv_k", conv_k), ("conv_v", conv_v)):
        _expect(t, (H * d, 4), torch.float32, name)
    _expect(beta_raw, (T, H), torch.float32, "beta_raw")
    _expect(a_raw, (T, H) if scalar_decay else (T, H, d), torch.float32, "a_raw")
    _expect(a_bias, (H,) if scalar_decay else (H, d), torch.float32, "a_bias")
    _check_cu(cu_seqlens, T, cu_seqlens_host)
    n = cu_seqlens.numel() - 1
    _expect(init_state, (n, H, d, d), torch.float32, "init_state")
    _expect(out, (T, H, d), xq.dtype, "out")
    _expect(final_state, (n, H, d, d), torch.float32, "final_state")
    _check_gate(gate_raw, norm_weight, norm_eps, (T, H, d), xq.dtype)
    _need_cuda(xq, xk, xv, conv_q, conv_k, conv_v, beta_raw, a_raw, a_bias, cu_seqlens,
               init_state, out, final_state, workspace)
    _check_snapshot_buffer(snapshots)
    dev = xq.device
    if out is None:
        out = torch.empty(T, H, d, dtype=xq.dtype, device=dev)
    if final_state is None:
        final_state = torch.empty(n, H, d, d, dtype=torch.float32, device=dev)
    if snap_interval and snapshots is None:
        ns = snapshot_count(_host_cu(cu_seqlens, cu_seqlens_host), snap_interval)
        snapshots = torch.empty(max(ns, 1), H, d, d, dtype=torch.float32, device=dev)[:ns]
    if workspace is None:
        workspace = torch.empty(projections_workspace_size(n, H, d, T, scalar_decay),
                                dtype=torch.uint8, device=dev)
    snap_arg = snapshots if (snap_interval and snapshots is not None and snapshots.numel()) else None
    if snap_interval and snap_arg is None:
        snap_arg = final_state
    a = PrefillArgs()
    a.n_seqs, a.n_heads, a.d_k, a.d_v, a.total_tokens = n, H, d, d, T
    a.cu_seqlens = cu_seqlens.data_ptr()
    a.qkv_dtype = GDR_BF16
    a.scalar_decay = int(bool(scalar_decay))
    a.scale = float(scale)
    a.init_state = None if init_state is None else init_state.data_ptr()
    a.o, a.final_state = out.data_ptr(), final_state.data_ptr()
    a.snap_interval = int(snap_interval)
    a.snapshots = None if snap_arg is None else snap_arg.data_ptr()
    a.gate_raw = None if gate_raw is None else gate_raw.data_ptr()
    a.norm_weight = None if norm_weight is None else norm_weight.data_ptr()
    a.norm_eps = float(norm_eps)
    a.workspace, a.workspace_bytes = workspace.data_ptr(), workspace.numel()
    p = Projections()
    p.xq, p.xk, p.xv = xq.data_ptr(), xk.data_ptr(), xv.data_ptr()
    p.conv_q, p.conv_k, p.conv_v = conv_q.data_ptr(), conv_k.data_ptr(), conv_v.data_ptr()
    p.beta_raw, p.a_raw, p.a_bias = beta_raw.data_ptr(), a_raw.data_ptr(), a_bias.data_ptr()
    _check(lib().gdr_prefill_from_projections(ctypes.byref(a), ctypes.byref(p), _stream(dev)),
           "gdr_prefill_from_projections")
    return out, final_state, snapshots


def snapshot_offload(dev_snapshots, host_snapshots, copy_stream, event, compute_stream=None):
    """Copy the snapshots a prefill wrote (device) into pinned host memory on
    ``copy_stream`` (a torch.cuda.Stream), after the work enqueued so far on
    ``compute_stream`` (default: the current stream), ordered by ``event``
    (a torch.cuda.Event).  Later prefills on compute_stream do not wait."""
    if not dev_snapshots.is_cuda or not host_snapshots.is_pinned():
        raise ValueError("dev_snapshots must be a CUDA tensor and host_snapshots pinned host memory")
    if dev_snapshots.numel() != host_snapshots.numel() or dev_snapshots.dtype != torch.float32 or \
            host_snapshots.dtype != torch.float32:
        raise ValueError("snapshot buffers must be float32 of equal size")
    if not dev_snapshots.is_contiguous() or not host_snapshots.is_contiguous():
        raise ValueError("snapshot buffers must be contiguous")
    cs = compute_stream if compute_stream is not None else torch.cuda.current_stream(dev_snapshots.device)
    if not event.cuda_event:            # torch creates the event on its first record
        event.record(cs)
    _check(lib().gdr_snapshot_offload(_ptr(dev_snapshots), _ptr(host_snapshots),
                                      dev_snapshots.numel() * 4, ctypes.c_void_p(cs.cuda_stream),
                                      ctypes.c_void_p(copy_stream.cuda_stream),
                                      ctypes.c_void_p(event.cuda_event)),
           "gdr_snapshot_offload")
