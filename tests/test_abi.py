"""The C-ABI library loads without a GPU, exports every function include/gdn.h
declares, and rejects bad arguments on the host before launching anything."""
import ctypes
import os
import re
import subprocess

import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "gdn.h")


def _declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(gdn_[a-z0-9_]+)\s*\(", text)))


@pytest.fixture(scope="module")
def lib():
    from gated_delta_rule_130_b200 import binding
    return binding.LIB


def test_header_declares_the_entry_points():
    names = _declared_functions()
    for n in ["gdn_chunk_fwd", "gdn_chunk_fwd_workspace_size", "gdn_chunk_fwd_path",
              "gdn_decode_step", "gdn_status_string"]:
        assert n in names


def test_library_exports_every_declared_symbol(lib):
    from gated_delta_rule_130_b200 import binding
    out = subprocess.run(["nm", "-D", "--defined-only", binding.library_path()],
                         capture_output=True, text=True, check=True).stdout
    exported = set(re.findall(r"\bT (gdn_[a-z0-9_]+)", out))
    for n in _declared_functions():
        assert n in exported, f"{n} declared in gdn.h but not exported"
        assert hasattr(lib, n)


def test_status_strings(lib):
    assert lib.gdn_status_string(0) == b"ok"
    assert lib.gdn_status_string(1) == b"invalid argument"
    assert lib.gdn_status_string(2) == b"unsupported size or type"
    assert lib.gdn_status_string(3) == b"CUDA launch failed"


def test_path_selection_and_workspace(lib):
    from gated_delta_rule_130_b200 import binding as b
    assert b.chunk_fwd_path(1, 64, 2, 16, 16, 16, torch.float32) == "simt"
    assert b.chunk_fwd_path(0, 64, 2, 16, 16, 16, torch.float32) == "none"
    assert b.chunk_fwd_path(1, 0, 2, 16, 16, 16, torch.float32) == "none"
    with pytest.raises(b.GdnError):
        b.chunk_fwd_path(1, 64, 2, 16, 16, 48, torch.float32)
    # the CUDA-core path stores T, P' (C x C each) and g (C) per chunk
    C, NT = 16, 4
    assert b.chunk_fwd_workspace_size(1, 64, 2, 16, 16, C, torch.float32) == \
        2 * NT * (2 * C * C + C) * 4
    assert b.chunk_fwd_workspace_size(1, 0, 2, 16, 16, C, torch.float32) == 0


def _chunk(lib, **kw):
    a = dict(q=16, k=16, v=16, la=16, beta=16, S0=None, o=4096, S_T=None, B=1, T=8, H=1, Dk=16,
             Dv=16, chunk=16, dtype=0, ws=1 << 40, ws_bytes=1 << 30, stream=None)
    a.update(kw)
    return lib.gdn_chunk_fwd(a["q"], a["k"], a["v"], a["la"], a["beta"], a["S0"], a["o"],
                             a["S_T"], a["B"], a["T"], a["H"], a["Dk"], a["Dv"], a["chunk"],
                             a["dtype"], a["ws"], a["ws_bytes"], a["stream"])


@pytest.mark.parametrize("kw,status", [
    (dict(q=None), 1), (dict(o=None), 1), (dict(la=None), 1),
    (dict(B=-1), 1), (dict(T=-3), 1), (dict(Dk=0), 1), (dict(Dv=-1), 1), (dict(dtype=7), 1),
    (dict(chunk=48), 2), (dict(chunk=128), 2), (dict(Dk=272), 2), (dict(Dv=528), 2),
    (dict(q=24), 1), (dict(S_T=4100), 1),                 # misaligned pointers
    (dict(ws=None), 1), (dict(ws_bytes=64), 1),           # short workspace
    (dict(ws=4096), 1), (dict(ws=32), 1),                 # workspace overlaps o / an input
    (dict(o=16), 1),                                      # output overlaps an input
    (dict(B=0), 0), (dict(H=0), 0),                       # empty: nothing to do
])
def test_chunk_fwd_rejects_before_launch(lib, kw, status):
    # every case returns from the host-side checks; no pointer is dereferenced
    assert _chunk(lib, **kw) == status


@pytest.mark.parametrize("kw,status", [
    (dict(q=None), 1), (dict(S=None), 1), (dict(B=-1), 1), (dict(Dk=0), 1), (dict(Dk=300), 2),
    (dict(dtype=5), 1), (dict(o=8), 1), (dict(o=16, S=16), 1), (dict(B=0), 0),
])
def test_decode_step_rejects_before_launch(lib, kw, status):
    a = dict(q=16, k=16, v=16, la=16, beta=16, S=1 << 20, o=16, B=2, H=2, Dk=16, Dv=16, dtype=1)
    a.update(kw)
    assert lib.gdn_decode_step(a["q"], a["k"], a["v"], a["la"], a["beta"], a["S"], a["o"], a["B"],
                               a["H"], a["Dk"], a["Dv"], a["dtype"], None) == status


def test_binding_fails_loudly_without_library(tmp_path):
    """Import of the binding from a copy of the package without libgdn.so raises."""
    import shutil
    pkg = os.path.join(ROOT, "gated_delta_rule_130_b200")
    dst = tmp_path / "gated_delta_rule_130_b200"
    shutil.copytree(pkg, dst, ignore=shutil.ignore_patterns("*.so", "__pycache__", "csrc"))
    code = ("import sys; sys.path.insert(0, %r)\n"
            "try:\n    import gated_delta_rule_130_b200.binding\nexcept ImportError as e:\n"
            "    print('RAISED', e)\n") % str(tmp_path)
    out = subprocess.run(["python", "-c", code], capture_output=True, text=True, timeout=120)
    assert "RAISED" in out.stdout and "libgdn.so not found" in out.stdout


def test_prologue_flags_checked_before_launch(lib):
    # unknown flag bits are rejected on the host (nothing is dereferenced)
    f = lib.gdn_chunk_fwd_ex
    f.argtypes = [ctypes.c_void_p] * 8 + [ctypes.c_int] * 7 + [ctypes.c_uint, ctypes.c_void_p,
                                                                 ctypes.c_size_t, ctypes.c_void_p]
    assert f(16, 16, 16, 16, 16, None, 4096, None, 1, 8, 1, 16, 16, 16, 0, 4, 1 << 40, 1 << 30,
             None) == 1
    d = lib.gdn_decode_step_ex
    d.argtypes = [ctypes.c_void_p] * 7 + [ctypes.c_int] * 5 + [ctypes.c_uint, ctypes.c_void_p]
    assert d(16, 16, 16, 16, 16, 1 << 20, 16, 2, 2, 16, 16, 1, 8, None) == 1
    assert d(16, 16, 16, 16, 16, 1 << 20, 16, 0, 2, 16, 16, 1, 3, None) == 0  # empty: nothing to do


def test_prologue_workspace_size_on_the_cuda_core_path(lib):
    from gated_delta_rule_130_b200 import binding as b
    C, NT, rows, Dk = 16, 4, 64 * 2, 16
    base = 2 * NT * (2 * C * C + C) * 4                     # 16896, a multiple of 256
    assert b.chunk_fwd_workspace_size(1, 64, 2, Dk, 16, C, torch.float32) == base
    # prepared q, k (float32) and gates follow the path's own scratch
    assert b.chunk_fwd_workspace_size(1, 64, 2, Dk, 16, C, torch.float32, l2norm_qk=True) == \
        base + 2 * rows * Dk * 4
    assert b.chunk_fwd_workspace_size(1, 64, 2, Dk, 16, C, torch.float32, gate_logits=True) == \
        base + 1024
    assert b.chunk_fwd_workspace_size(1, 64, 2, Dk, 16, C, torch.float32, True, True) == \
        base + 2 * rows * Dk * 4 + 2 * rows * 4


def _varlen(lib, cu, **kw):
    a = dict(q=16, k=16, v=16, la=16, beta=16, S0=None, o=1 << 24, S_T=None, cu_dev=1 << 28, H=1,
             Dk=16, Dv=16, chunk=16, dtype=0, flags=0, ws=1 << 40, ws_bytes=1 << 30)
    a.update(kw)
    N = a.pop("N") if "N" in a else len(cu) - 1
    host = (ctypes.c_int * len(cu))(*cu) if cu is not None else None
    return lib.gdn_chunk_fwd_varlen(a["q"], a["k"], a["v"], a["la"], a["beta"], a["S0"], a["o"],
                                    a["S_T"], a["cu_dev"], ctypes.cast(host, ctypes.c_void_p)
                                    if host is not None else None, N, a["H"], a["Dk"], a["Dv"],
                                    a["chunk"], a["dtype"], a["flags"], a["ws"], a["ws_bytes"], None)


@pytest.mark.parametrize("cu,kw,status", [
    ([1, 4, 8], {}, 1),                       # offsets must start at 0
    ([0, 6, 4, 9], {}, 1),                    # and never decrease
    (None, dict(N=2), 1),                     # no host offsets
    ([0, 4, 8], dict(N=-1), 1),
    ([0, 4, 8], dict(flags=8), 1),            # unknown prologue flag
    ([0, 4, 8], dict(q=None), 1),
    ([0, 4, 8], dict(cu_dev=None), 1),        # device offsets missing
    ([0, 4, 8], dict(ws=None), 1), ([0, 4, 8], dict(ws_bytes=16), 1),
    ([0, 4, 8], dict(o=16), 1),               # output overlaps q
    ([0, 4, 8], dict(ws=1 << 28), 1),         # workspace overlaps the device offsets
    ([0, 4, 8], dict(chunk=48), 2), ([0, 4, 8], dict(Dk=272), 2),
    ([0], {}, 0),                             # no sequences: nothing to do
    ([0, 0, 0], {}, 0),                       # empty sequences, no state asked for
    ([0] * 65537, {}, 2),                     # more sequences than one grid dimension holds
])
def test_chunk_fwd_varlen_rejects_before_launch(lib, cu, kw, status):
    assert _varlen(lib, cu, **kw) == status


def test_varlen_workspace_sizes(lib):
    from gated_delta_rule_130_b200 import binding as b
    # CUDA-core path: scratch for the longest sequence, reused by each in turn
    C, H = 16, 2
    cu = [0, 5, 45, 62]                       # lengths 5, 40, 17: longest has 3 chunks
    assert b.chunk_fwd_varlen_workspace_size(cu, H, 16, 16, C, torch.float32) == \
        H * 3 * (2 * C * C + C) * 4
    a256 = lambda n: (n + 255) // 256 * 256   # each part starts on a 256-byte boundary
    assert b.chunk_fwd_varlen_workspace_size(cu, H, 16, 16, C, torch.float32, True, True) == \
        a256(H * 3 * (2 * C * C + C) * 4) + a256(2 * 62 * H * 16 * 4 + 2 * 62 * H * 4)
    assert b.chunk_fwd_varlen_workspace_size([0, 0], H, 16, 16, C, torch.float32) == 0
    assert b.chunk_fwd_varlen_workspace_size([0, 3, 1], H, 16, 16, C, torch.float32) == 0


def test_varlen_binding_checks_the_offsets():
    from gated_delta_rule_130_b200 import binding as b
    q = torch.zeros(10, 2, 16)
    la = torch.zeros(10, 2)
    with pytest.raises(b.GdnError):          # offsets end before the packed tokens do
        b.chunk_fwd_varlen(q, q, q, la, la, [0, 4, 8])
    with pytest.raises(b.GdnError):
        b.chunk_fwd_varlen(q, q, q, la, la, [[0, 10]])


def _bwd(lib, **kw):
    a = dict(q=16, k=16, v=16, la=16, beta=16, S0=None, do=1 << 20, dS_T=None, dq=1 << 24,
             dk=1 << 25, dv=1 << 26, dla=1 << 27, dbeta=1 << 28, dS0=None, B=1, T=8, H=1, Dk=16,
             Dv=16, chunk=16, dtype=0, ws=1 << 40, ws_bytes=1 << 30)
    a.update(kw)
    return lib.gdn_chunk_bwd(a["q"], a["k"], a["v"], a["la"], a["beta"], a["S0"], a["do"],
                             a["dS_T"], a["dq"], a["dk"], a["dv"], a["dla"], a["dbeta"], a["dS0"],
                             a["B"], a["T"], a["H"], a["Dk"], a["Dv"], a["chunk"], a["dtype"],
                             a["ws"], a["ws_bytes"], None)


@pytest.mark.parametrize("kw,status", [
    (dict(q=None), 1), (dict(do=None), 1), (dict(dq=None), 1), (dict(dbeta=None), 1),
    (dict(Dk=0), 1), (dict(dtype=3), 1), (dict(chunk=48), 2),
    (dict(Dk=144), 2),                                     # the backward takes Dk <= 128
    (dict(dq=24), 1),                                      # misaligned
    (dict(dq=16), 1),                                      # a gradient overlaps q
    (dict(dk=1 << 24), 1),                                 # two gradients overlap
    (dict(ws=None), 1), (dict(ws_bytes=64), 1), (dict(ws=1 << 20), 1),
    (dict(B=0), 0), (dict(H=0), 0), (dict(T=0), 0),        # nothing to do (dS0 not asked)
])
def test_chunk_bwd_rejects_before_launch(lib, kw, status):
    assert _bwd(lib, **kw) == status


def test_chunk_bwd_workspace_size(lib):
    from gated_delta_rule_130_b200 import binding as b
    # recomputed T, P (C x C) and g (C), the chunk state and its gradient (Dv x Dk)
    C, NT, H, Dk, Dv = 16, 3, 2, 32, 8
    assert b.chunk_bwd_workspace_size(1, 40, H, Dk, Dv, C, torch.float32) == \
        H * NT * (2 * C * C + C + 2 * Dv * Dk) * 4
    assert b.chunk_bwd_workspace_size(1, 40, H, 256, Dv, C, torch.float32) == 0
    assert b.chunk_bwd_workspace_size(1, 0, H, Dk, Dv, C, torch.float32) == 0


def test_chunk_fwd_cw_checks(lib):
    from gated_delta_rule_130_b200 import binding as b
    f = lib.gdn_chunk_fwd_cw
    args = lambda **kw: dict(dict(q=16, k=16, v=16, la=16, bg=16, w=16, S0=None, o=1 << 24,
                                  S_T=None, B=1, T=8, H=1, Dk=16, Dv=16, chunk=16, dtype=0,
                                  ws=1 << 40, ws_bytes=1 << 30), **kw)
    call = lambda a: f(a["q"], a["k"], a["v"], a["la"], a["bg"], a["w"], a["S0"], a["o"],
                       a["S_T"], a["B"], a["T"], a["H"], a["Dk"], a["Dv"], a["chunk"],
                       a["dtype"], a["ws"], a["ws_bytes"], None)
    assert call(args(bg=None)) == 1 and call(args(w=None)) == 1
    assert call(args(Dk=144)) == 2 and call(args(chunk=48)) == 2
    assert call(args(o=16)) == 1 and call(args(ws=None)) == 1 and call(args(ws_bytes=8)) == 1
    assert call(args(B=0)) == 0 and call(args(T=0)) == 0
    # T, P' (C x C) and the running log-decay sums (C x Dk) per chunk and head
    assert b.chunk_fwd_cw_workspace_size(2, 40, 3, 16, 8, 16, torch.float32) == \
        2 * 3 * 3 * (2 * 16 * 16 + 16 * 16) * 4
    d = lib.gdn_decode_step_cw
    assert d(16, 16, 16, 16, 16, None, 1 << 20, 16, 1, 1, 16, 16, 0, None) == 1
    assert d(16, 16, 16, 16, 16, 16, 1 << 20, 16, 1, 1, 16, 16, 0, None) == 1   # o overlaps q
    assert d(16, 16, 16, 16, 16, 16, 1 << 20, 1 << 24, 0, 1, 16, 16, 0, None) == 0


def test_sizes_whose_byte_counts_would_overflow_are_refused(lib):
    from gated_delta_rule_130_b200 import binding as b
    B, H, T = 65535, 65535, 2 ** 31 - 1            # B H (T + 64) far above 2^40
    assert _chunk(lib, B=B, H=H, T=T) == 2
    assert _bwd(lib, B=B, H=H, T=T) == 2
    assert b.chunk_fwd_workspace_size(B, T, H, 16, 16, 16, torch.float32) == 0
    assert b.chunk_bwd_workspace_size(B, T, H, 16, 16, 16, torch.float32) == 0
    assert b.chunk_fwd_cw_workspace_size(B, T, H, 16, 16, 16, torch.float32) == 0
    with pytest.raises(b.GdnError):
        b.chunk_fwd_path(B, T, H, 16, 16, 16, torch.float32)
    # just inside the bound the checks pass on to the workspace test (short: 1)
    assert _chunk(lib, B=1, H=1, T=2 ** 31 - 1, ws_bytes=16) == 1


def test_binding_shape_checks_of_the_newer_entry_points():
    """Mismatched shapes are refused by the binding before any device work."""
    from gated_delta_rule_130_b200 import binding as b
    q = torch.zeros(1, 8, 2, 16)
    v = torch.zeros(1, 8, 2, 12)
    g = torch.zeros(1, 8, 2)
    with pytest.raises(b.GdnError):                      # d_o must be shaped like v
        b.chunk_bwd(q, q, v, g, g, None, torch.zeros(1, 8, 2, 16))
    with pytest.raises(b.GdnError):                      # dS_T must be [B,H,Dv,Dk]
        b.chunk_bwd(q, q, v, g, g, None, v, torch.zeros(1, 2, 16, 12))
    with pytest.raises(b.GdnError):                      # gates must be [B,T,H]
        b.chunk_bwd(q, q, v, torch.zeros(1, 8, 3), g, None, v)
    with pytest.raises(b.GdnError):                      # channel-wise decay is per key channel
        b.chunk_fwd_cw(q, q, v, g, q, v)
    with pytest.raises(b.GdnError):                      # the write gate is per value channel
        b.chunk_fwd_cw(q, q, v, q, q, q)
    with pytest.raises(b.GdnError):
        b.chunk_fwd_cw(q, q, v, q, q, v, S0=torch.zeros(1, 2, 16, 12))
    with pytest.raises(b.GdnError):                      # decode state must be [B,H,Dv,Dk]
        b.decode_step_cw(q[:, 0], q[:, 0], v[:, 0], q[:, 0], q[:, 0], v[:, 0],
                         torch.zeros(1, 2, 16, 12))
    with pytest.raises(b.GdnError):                      # packed q, k, v are [total,H,D]
        b.chunk_fwd_varlen(q, q, v, g, g, [0, 8])
