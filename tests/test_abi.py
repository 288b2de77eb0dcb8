"""Host-side checks of the C ABI: the library loads without a GPU, exports
every function include/gdr.h declares, rejects bad arguments before any
launch, and sizes workspaces and snapshot buffers as documented."""
import ctypes
import os
import re

import pytest
import torch

import gated_delta_rule_150_b200 as gdr
from gated_delta_rule_150_b200 import build as gdr_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    gdr_build.build()
    return gdr.lib()


def declared_functions():
    names = []
    for h in os.listdir(os.path.join(ROOT, "include")):
        if h.endswith(".h"):
            src = open(os.path.join(ROOT, "include", h)).read()
            src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
            names += re.findall(r"^\s*[A-Za-z_][\w\s\*]*?\b(gdr_\w+)\s*\(", src, flags=re.M)
    return sorted(set(names))


def test_exports_every_declared_symbol(L):
    names = declared_functions()
    assert "gdr_prefill" in names and "gdr_decode_step" in names
    for n in names:
        assert hasattr(L, n), f"{n} declared in include/ but not exported"


def test_status_strings(L):
    for s, name in gdr._STATUS.items():
        assert L.gdr_status_string(s).decode() == name


def _fake(n):
    # 256-byte aligned fake device addresses: validation must fail before any use
    return ctypes.c_void_p(0x10000 * (n + 1))


def test_decode_rejects_bad_arguments(L):
    ok = [_fake(i) for i in range(7)]
    st = None
    def call(B=2, H=2, dk=64, dv=64, dt=0, ptrs=ok):
        return L.gdr_decode_step(B, H, dk, dv, dt, *ptrs[:5], 0, 1.0, ptrs[5], ptrs[6], st)
    assert call(B=-1) == 1
    assert call(dk=96) == 2
    assert call(dv=32) == 2
    assert call(dt=7) == 1
    bad = list(ok); bad[2] = None
    assert call(ptrs=bad) == 1
    mis = list(ok); mis[0] = ctypes.c_void_p(0x10008)
    assert call(ptrs=mis) == 1
    assert call(B=0) == 0


def test_draft_and_accept_reject_bad_arguments(L):
    ok = [_fake(i) for i in range(8)]
    def draft(B=2, K=4, H=2, dk=64, dv=64, dt=0, ptrs=ok):
        return L.gdr_decode_draft(B, K, H, dk, dv, dt, *ptrs[:5], 0, 1.0, *ptrs[5:8], None)
    assert draft(B=-1) == 1
    assert draft(K=-1) == 1
    assert draft(dk=96) == 2
    assert draft(dt=3) == 1
    for i in range(8):
        bad = list(ok); bad[i] = None
        assert draft(ptrs=bad) == 1, f"null pointer {i}"
    mis = list(ok); mis[7] = ctypes.c_void_p(0x10008)     # token_states not 16-byte aligned
    assert draft(ptrs=mis) == 1
    assert draft(B=0) == 0 and draft(K=0) == 0
    def accept(B=2, K=4, H=2, dk=64, dv=64, n=ok[0], ts=ok[1], st=ok[2]):
        return L.gdr_decode_accept(B, K, H, dk, dv, n, ts, st, None)
    assert accept(B=-1) == 1
    assert accept(dv=48) == 2
    assert accept(n=None) == 1
    assert accept(ts=ctypes.c_void_p(0x10004)) == 1
    assert accept(st=None) == 1
    assert accept(K=0) == 0 and accept(B=0) == 0


def _pre_args(**kw):
    a = gdr.PreprocessArgs()
    a.n_seqs, a.n_heads, a.d, a.total_tokens = 1, 2, 64, 128
    a.cu_seqlens = 0x10000
    a.io_dtype = 0
    names = ("xq", "xk", "xv", "conv_q", "conv_k", "conv_v", "beta_raw", "a_raw", "a_bias",
             "q", "k", "v", "beta", "log_a")
    for i, n in enumerate(names):
        setattr(a, n, 0x100000 * (i + 1))
    for k_, v_ in kw.items():
        setattr(a, k_, v_)
    return a


def test_preprocess_rejects_bad_arguments(L):
    pre = lambda a: L.gdr_preprocess(ctypes.byref(a), None)
    assert pre(_pre_args(n_heads=0)) == 1
    assert pre(_pre_args(d=96)) == 2
    assert pre(_pre_args(io_dtype=5)) == 1
    assert pre(_pre_args(total_tokens=-1)) == 1
    for n in ("xq", "conv_k", "beta_raw", "a_bias", "v", "log_a", "cu_seqlens"):
        assert pre(_pre_args(**{n: None})) == 1, n
    assert pre(_pre_args(xk=0x200008)) == 1                     # not 16-byte aligned
    assert pre(_pre_args(log_a=0x200004)) == 1                  # per-channel gate: 16 bytes
    assert pre(_pre_args(total_tokens=0)) == 0
    assert pre(_pre_args(total_tokens=0, xq=None)) == 0         # nothing to do, nothing read


def _args(**kw):
    a = gdr.PrefillArgs()
    a.n_seqs, a.n_heads, a.d_k, a.d_v, a.total_tokens = 1, 2, 64, 64, 128
    a.cu_seqlens = 0x10000
    a.qkv_dtype = 0
    a.q, a.k, a.v, a.beta, a.log_a = 0x20000, 0x30000, 0x40000, 0x50000, 0x60000
    a.scale = 1.0
    a.o, a.final_state = 0x70000, 0x80000
    a.workspace = 0x100000
    a.workspace_bytes = 1 << 40
    for k_, v_ in kw.items():
        setattr(a, k_, v_)
    return a


def test_prefill_rejects_bad_arguments(L):
    pre = lambda a: L.gdr_prefill(ctypes.byref(a), None)
    assert pre(_args(n_heads=0)) == 1
    assert pre(_args(d_k=96, d_v=96)) == 2
    assert pre(_args(d_v=96)) == 2
    assert pre(_args(d_k=128, d_v=32)) == 2
    assert pre(_args(q=None)) == 1
    assert pre(_args(k=0x30004)) == 1
    assert pre(_args(snap_interval=100, snapshots=0x90000)) == 1
    assert pre(_args(snap_interval=128, snapshots=None)) == 1
    assert pre(_args(workspace=None)) == 3
    assert pre(_args(workspace_bytes=16)) == 3
    assert pre(_args(workspace=0x100080)) == 3
    assert pre(_args(final_state=None)) == 1
    assert pre(_args(total_tokens=-1)) == 1
    assert pre(_args(n_seqs=0, total_tokens=0)) == 0


def test_workspace_size_grows_with_tokens(L):
    s1 = gdr.workspace_size(1, 14, 64, 64, 8192)
    s2 = gdr.workspace_size(1, 14, 64, 64, 16384)
    assert 0 < s1 < s2
    assert gdr.workspace_size(1, 14, 96, 96, 8192) == 0
    assert gdr.workspace_size(1, 14, 128, 128, 8192, True) <= gdr.workspace_size(1, 14, 128, 128, 8192, False)
    # d_k != d_v: the square layout at D = 128 plus the widened inputs
    sq = gdr.workspace_size(1, 14, 128, 128, 8192)
    assert gdr.workspace_size(1, 14, 64, 128, 8192) == sq + 3 * 8192 * 14 * 128 * 4
    assert gdr.workspace_size(1, 14, 64, 128, 8192, True) == \
        gdr.workspace_size(1, 14, 128, 128, 8192, True) + 2 * 8192 * 14 * 128 * 4
    assert gdr.workspace_size(1, 14, 128, 64, 8192) == sq + 8192 * 14 * 128 * 4
    assert gdr.kernel_count(32, 32, 64, 128, 278000) == 2 + 3
    assert gdr.kernel_count(32, 32, 128, 64, 278000) == 2 + 1


def test_projections_workspace_size(L):
    """The staged-activation workspace: larger only at d 128 with a per-channel
    gate, by q, k, v (bf16), beta and log a (fp32) of every token-head, each
    part rounded up to 256 bytes."""
    for d, scalar in ((64, False), (64, True), (128, True)):
        assert gdr.projections_workspace_size(1, 14, d, 8192, scalar) == \
            gdr.workspace_size(1, 14, d, d, 8192, scalar)
    base = gdr.workspace_size(2, 14, 128, 128, 8191)
    up = lambda x: (x + 255) // 256 * 256
    th = 8191 * 14
    assert gdr.projections_workspace_size(2, 14, 128, 8191) == \
        up(base) + 3 * up(th * 128 * 2) + up(th * 4) + up(th * 128 * 4)
    assert gdr.projections_workspace_size(1, 14, 96, 8192) == 0


def test_snapshot_count_matches_oracle(L):
    import oracle
    for lengths, iv in (([4096, 100, 8192, 0, 4095], 4096), ([64, 128, 1], 64), ([5, 7], 0)):
        cu = torch.tensor([0] + list(torch.tensor(lengths).cumsum(0)), dtype=torch.int32)
        assert gdr.snapshot_count(cu, iv) == oracle.snapshot_count(cu, iv)


def test_prefill_stage_range_and_kernel_count(L):
    pre = lambda a, f, l: L.gdr_prefill_stages(ctypes.byref(a), f, l, None)
    assert pre(_args(), -1, 1) == 1
    assert pre(_args(), 0, 2) == 1
    assert pre(_args(), 1, 0) == 1
    assert pre(_args(n_seqs=0, total_tokens=0), 0, 1) == 0
    # one intra-chunk kernel + one state pass, or + three when segmented
    assert gdr.kernel_count(1, 14, 64, 64, 8192) == 4          # 14 long heads: segmented
    assert gdr.kernel_count(32, 32, 128, 128, 278000) == 2     # many pairs: one pass
    assert gdr.kernel_count(300, 1, 64, 64, 300 * 4096) == 2   # more pairs than the CTA target
    assert gdr.kernel_count(1, 16, 128, 128, 65536, True) == 4  # 16 long heads: segmented
    assert gdr.kernel_count(1, 2, 64, 64, 256) == 2            # short: one pass
    assert gdr.kernel_count(1, 2, 64, 64, 0) == 1              # no tokens: state copy only
    assert gdr.kernel_count(1, 2, 96, 96, 256) == 0            # unsupported width


def test_static_workspace_is_declared_with_its_limit():
    src = open(os.path.join(ROOT, "include", "gdr.h")).read()
    assert "GDR_STATIC_WORKSPACE_BYTES" in src


def test_header_is_plain_c():
    """include/gdr.h is a C header: it compiles as C99 (and as C++17) with
    warnings enabled, with no CUDA or torch include."""
    import shutil
    import subprocess
    hdr = os.path.join(ROOT, "include", "gdr.h")
    src = open(hdr).read()
    includes = re.findall(r"#include\s*[<\"]([^>\"]+)", src.lower())
    assert not any("cuda" in inc or "torch" in inc for inc in includes), includes
    for cc, std, lang in (("gcc", "-std=c99", "c"), ("g++", "-std=c++17", "c++")):
        if shutil.which(cc) is None:
            pytest.skip(f"{cc} not available")
        subprocess.run([cc, std, "-Wall", "-Wextra", "-Werror", "-fsyntax-only", "-x", lang, hdr],
                       check=True)


def _enumerate_offsets(lengths, iv):
    """Host enumeration: walk every sequence's snapshot positions in order."""
    offsets, slot = [], 0
    for L in lengths:
        offsets.append(slot)
        for end in range(iv, L + 1, iv):
            slot += 1
    return offsets + [slot]


def test_snapshot_offsets_match_enumeration(L):
    for lengths, iv in (([4096, 100, 8192, 0, 4095], 4096), ([64, 128, 1, 0, 640], 64),
                        ([0], 128), ([], 64), ([300, 257, 1024], 128)):
        cu = torch.tensor([0] + [int(x) for x in torch.tensor(lengths, dtype=torch.int64).cumsum(0)],
                          dtype=torch.int32)
        got = gdr.snapshot_offsets(cu, iv)
        assert got.tolist() == _enumerate_offsets(lengths, iv)
        assert int(got[-1]) == gdr.snapshot_count(cu, iv)


def test_snapshot_offsets_reject_bad_arguments(L):
    cu = torch.tensor([0, 64, 32], dtype=torch.int32)             # decreasing
    out = torch.empty(3, dtype=torch.int64)
    call = lambda c, n, iv, o: L.gdr_snapshot_offsets(c, n, iv, o)
    p_cu, p_out = ctypes.c_void_p(cu.data_ptr()), ctypes.c_void_p(out.data_ptr())
    assert call(p_cu, 2, 64, p_out) == 1
    ok = torch.tensor([0, 64, 128], dtype=torch.int32)
    p_ok = ctypes.c_void_p(ok.data_ptr())
    assert call(p_ok, 2, 0, p_out) == 1
    assert call(p_ok, -1, 64, p_out) == 1
    assert call(None, 2, 64, p_out) == 1
    assert call(p_ok, 2, 64, None) == 1
    assert call(p_ok, 2, 64, p_out) == 0 and out.tolist() == [0, 1, 2]


def test_prefill_rejects_misaligned_snapshot_offsets(L):
    pre = lambda a: L.gdr_prefill(ctypes.byref(a), None)
    assert pre(_args(snap_interval=128, snapshots=0x90000, snap_offsets=0xA0004)) == 1


def test_snapshot_offload_rejects_bad_arguments(L):
    f = lambda d, h, n, cs, xs, ev: L.gdr_snapshot_offload(d, h, n, cs, xs, ev)
    d, h, ev = _fake(1), _fake(2), _fake(3)
    assert f(d, h, 1024, _fake(4), _fake(5), None) == 1          # no event
    assert f(d, h, 1024, _fake(4), _fake(4), ev) == 1            # same stream
    assert f(None, h, 1024, _fake(4), _fake(5), ev) == 1
    assert f(ctypes.c_void_p(0x10008), h, 1024, _fake(4), _fake(5), ev) == 1
