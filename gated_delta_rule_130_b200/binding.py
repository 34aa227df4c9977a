"""Thin ctypes binding of libgdn.so (C ABI in include/gdn.h).

Argument marshalling only: shape/dtype checks, device pointers, the current
torch stream, and workspace allocation through torch.  Every step of the
computation runs in the library's CUDA kernels.  Importing this module loads the
library and raises if it is missing -- there is no other implementation.
"""
from __future__ import annotations

import ctypes
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_PKG, "libgdn.so")

GDN_F32, GDN_BF16 = 0, 1
PATH_NONE, PATH_SIMT, PATH_TCGEN05 = 0, 1, 2
PATH_NAMES = {PATH_NONE: "none", PATH_SIMT: "simt", PATH_TCGEN05: "tcgen05"}


class GdnError(RuntimeError):
    pass


def library_path() -> str:
    return _LIB_PATH


def _load():
    if not os.path.exists(_LIB_PATH):
        raise ImportError(
            f"libgdn.so not found at {_LIB_PATH}: build it with "
            "`python -m gated_delta_rule_130_b200.build` (there is no fallback path)")
    lib = ctypes.CDLL(_LIB_PATH)
    vp, fp, I, Z = ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
    lib.gdn_chunk_fwd.argtypes = [vp, vp, vp, fp, fp, fp, vp, fp, I, I, I, I, I, I, I, vp, Z, vp]
    lib.gdn_chunk_fwd.restype = I
    lib.gdn_chunk_fwd_workspace_size.argtypes = [I, I, I, I, I, I, I]
    lib.gdn_chunk_fwd_workspace_size.restype = Z
    lib.gdn_chunk_fwd_path.argtypes = [I, I, I, I, I, I, I]
    lib.gdn_chunk_fwd_path.restype = I
    lib.gdn_chunk_fwd_variant.argtypes = [I, I, I, I, I, I, I]
    lib.gdn_chunk_fwd_variant.restype = I
    lib.gdn_decode_step.argtypes = [vp, vp, vp, fp, fp, fp, vp, I, I, I, I, I, vp]
    lib.gdn_decode_step.restype = I
    U = ctypes.c_uint
    lib.gdn_chunk_fwd_ex.argtypes = [vp, vp, vp, fp, fp, fp, vp, fp, I, I, I, I, I, I, I, U, vp,
                                     Z, vp]
    lib.gdn_chunk_fwd_ex.restype = I
    lib.gdn_chunk_fwd_workspace_size_ex.argtypes = [I, I, I, I, I, I, I, U]
    lib.gdn_chunk_fwd_workspace_size_ex.restype = Z
    lib.gdn_decode_step_ex.argtypes = [vp, vp, vp, fp, fp, fp, vp, I, I, I, I, I, U, vp]
    lib.gdn_decode_step_ex.restype = I
    lib.gdn_chunk_fwd_varlen.argtypes = [vp, vp, vp, fp, fp, fp, vp, fp, vp, vp, I, I, I, I, I, I,
                                         U, vp, Z, vp]
    lib.gdn_chunk_fwd_varlen.restype = I
    lib.gdn_chunk_fwd_varlen_workspace_size.argtypes = [vp, I, I, I, I, I, I, U]
    lib.gdn_chunk_fwd_varlen_workspace_size.restype = Z
    lib.gdn_chunk_bwd.argtypes = [vp, vp, vp, fp, fp, fp, vp, fp, vp, vp, vp, fp, fp, fp, I, I, I,
                                  I, I, I, I, vp, Z, vp]
    lib.gdn_chunk_bwd.restype = I
    lib.gdn_chunk_bwd_workspace_size.argtypes = [I, I, I, I, I, I, I]
    lib.gdn_chunk_bwd_workspace_size.restype = Z
    lib.gdn_chunk_bwd_path.argtypes = [I, I, I, I, I, I, I]
    lib.gdn_chunk_bwd_path.restype = I
    lib.gdn_chunk_fwd_cw.argtypes = [vp, vp, vp, fp, fp, fp, fp, vp, fp, I, I, I, I, I, I, I, vp,
                                     Z, vp]
    lib.gdn_chunk_fwd_cw.restype = I
    lib.gdn_chunk_fwd_cw_path.argtypes = [I, I, I, I, I, I, I]
    lib.gdn_chunk_fwd_cw_path.restype = I
    lib.gdn_chunk_fwd_cw_workspace_size.argtypes = [I, I, I, I, I, I, I]
    lib.gdn_chunk_fwd_cw_workspace_size.restype = Z
    lib.gdn_decode_step_cw.argtypes = [vp, vp, vp, fp, fp, fp, fp, vp, I, I, I, I, I, vp]
    lib.gdn_decode_step_cw.restype = I
    lib.gdn_debug_withhold_first_arrival.argtypes = [I]
    lib.gdn_debug_withhold_first_arrival.restype = I
    lib.gdn_check_device_status.argtypes = []
    lib.gdn_check_device_status.restype = I
    lib.gdn_status_string.argtypes = [I]
    lib.gdn_status_string.restype = ctypes.c_char_p
    return lib


LIB = _load()


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.float32:
        return GDN_F32
    if t.dtype == torch.bfloat16:
        return GDN_BF16
    raise GdnError(f"q/k/v must be float32 or bfloat16, got {t.dtype}")


def _check(status: int, what: str):
    if status != 0:
        raise GdnError(f"{what}: {LIB.gdn_status_string(status).decode()} (status {status})")


def _dev(t: torch.Tensor, name: str, dtype=None, device=None):
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise GdnError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise GdnError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise GdnError(f"{name} must be {dtype}, got {t.dtype}")
    if device is not None and t.device != device:
        raise GdnError(f"{name} is on {t.device}, expected {device}")
    return t.data_ptr()


def _stream_ptr(device) -> int:
    return torch.cuda.current_stream(device).cuda_stream


def check_device_status():
    """Synchronise and raise if a fused tensor-core kernel timed out since the last check."""
    _check(int(LIB.gdn_check_device_status()), "gdn_check_device_status")


# Input prologue flags of the _ex entry points (gdn_flag_t in include/gdn.h).
GDN_FLAG_L2NORM_QK = 1
GDN_FLAG_GATE_LOGITS = 2


def _flags(l2norm_qk: bool, gate_logits: bool) -> int:
    return (GDN_FLAG_L2NORM_QK if l2norm_qk else 0) | (GDN_FLAG_GATE_LOGITS if gate_logits else 0)


def chunk_fwd_workspace_size(B, T, H, Dk, Dv, chunk=64, dtype=torch.bfloat16,
                             l2norm_qk: bool = False, gate_logits: bool = False) -> int:
    code = GDN_BF16 if dtype == torch.bfloat16 else GDN_F32
    return int(LIB.gdn_chunk_fwd_workspace_size_ex(B, T, H, Dk, Dv, chunk, code,
                                                   _flags(l2norm_qk, gate_logits)))


def chunk_fwd_path(B, T, H, Dk, Dv, chunk=64, dtype=torch.bfloat16) -> str:
    code = GDN_BF16 if dtype == torch.bfloat16 else GDN_F32
    p = int(LIB.gdn_chunk_fwd_path(B, T, H, Dk, Dv, chunk, code))
    if p < 0:
        raise GdnError("invalid or unsupported sizes")
    return PATH_NAMES[p]


VARIANT_NAMES = {0: None, 1: "fused", 2: "precomputed", 3: "split"}


def chunk_fwd_variant(B, T, H, Dk, Dv, chunk=64, dtype=torch.bfloat16):
    """Which tcgen05 variant a chunk_fwd call with these sizes runs: "fused",
    "precomputed", or None off the tcgen05 path."""
    code = GDN_BF16 if dtype == torch.bfloat16 else GDN_F32
    return VARIANT_NAMES[int(LIB.gdn_chunk_fwd_variant(B, T, H, Dk, Dv, chunk, code))]


def chunk_fwd(q, k, v, log_alpha, beta, S0=None, chunk: int = 64, out=None, S_T=None,
              return_state: bool = True, workspace=None, l2norm_qk: bool = False,
              gate_logits: bool = False):
    """Chunkwise forward: returns (o [B,T,H,Dv], S_T [B,H,Dv,Dk] float32 or None).

    q, k [B,T,H,Dk] and v [B,T,H,Dv] in float32 or bfloat16 (same type);
    log_alpha, beta [B,T,H] float32; S0 [B,H,Dv,Dk] float32 or None (zeros).
    ``S_T`` may be passed (and may be ``S0`` itself for in-place continuation).
    ``l2norm_qk``: q and k are raw and get normalised per token and head in the
    kernels; ``gate_logits``: log_alpha and beta hold logits (log alpha =
    -softplus(x), beta = sigmoid(y)).
    """
    flags = _flags(l2norm_qk, gate_logits)
    if q.dim() != 4 or k.shape != q.shape or v.dim() != 4 or v.shape[:3] != q.shape[:3]:
        raise GdnError("q, k must be [B,T,H,Dk] and v [B,T,H,Dv]")
    B, T, H, Dk = q.shape
    Dv = v.shape[3]
    dev = q.device
    code = _dtype_code(q)
    args = [_dev(q, "q", q.dtype, dev), _dev(k, "k", q.dtype, dev), _dev(v, "v", q.dtype, dev)]
    if log_alpha.shape != (B, T, H) or beta.shape != (B, T, H):
        raise GdnError("log_alpha and beta must be [B,T,H]")
    args += [_dev(log_alpha, "log_alpha", torch.float32, dev),
             _dev(beta, "beta", torch.float32, dev)]
    if S0 is not None:
        if S0.shape != (B, H, Dv, Dk):
            raise GdnError("S0 must be [B,H,Dv,Dk]")
        args.append(_dev(S0, "S0", torch.float32, dev))
    else:
        args.append(None)
    o = out if out is not None else torch.empty((B, T, H, Dv), dtype=q.dtype, device=dev)
    if o.shape != (B, T, H, Dv):
        raise GdnError("out must be [B,T,H,Dv]")
    args.append(_dev(o, "out", q.dtype, dev))
    if S_T is None and return_state:
        S_T = torch.empty((B, H, Dv, Dk), dtype=torch.float32, device=dev)
    if S_T is not None:
        if S_T.shape != (B, H, Dv, Dk):
            raise GdnError("S_T must be [B,H,Dv,Dk]")
        args.append(_dev(S_T, "S_T", torch.float32, dev))
    else:
        args.append(None)
    need = int(LIB.gdn_chunk_fwd_workspace_size_ex(B, T, H, Dk, Dv, chunk, code, flags))
    ws_ptr, ws_bytes = None, 0
    if need:
        if workspace is None or workspace.numel() * workspace.element_size() < need:
            workspace = torch.empty(need, dtype=torch.uint8, device=dev)
        ws_ptr, ws_bytes = _dev(workspace, "workspace"), workspace.numel() * workspace.element_size()
    st = LIB.gdn_chunk_fwd_ex(*args, B, T, H, Dk, Dv, chunk, code, flags, ws_ptr, ws_bytes,
                              _stream_ptr(dev))
    _check(st, "gdn_chunk_fwd")
    return o, S_T


def chunk_bwd_workspace_size(B, T, H, Dk, Dv, chunk=64, dtype=torch.bfloat16) -> int:
    code = GDN_BF16 if dtype == torch.bfloat16 else GDN_F32
    return int(LIB.gdn_chunk_bwd_workspace_size(B, T, H, Dk, Dv, chunk, code))


def chunk_bwd(q, k, v, log_alpha, beta, S0, d_o, dS_T=None, chunk: int = 64, workspace=None,
              want_dS0: bool = True):
    """Chunkwise backward of ``chunk_fwd`` (plain gates, no prologue).

    Given the forward's inputs and d_o = dL/do [B,T,H,Dv] (q's dtype), dS_T =
    dL/dS_T [B,H,Dv,Dk] float32 or None, returns (dq, dk, dv, dlog_alpha, dbeta,
    dS0): dq, dk, dv in q's dtype, the rest float32 (dS0 None unless want_dS0).
    """
    if q.dim() != 4 or k.shape != q.shape or v.dim() != 4 or v.shape[:3] != q.shape[:3]:
        raise GdnError("q, k must be [B,T,H,Dk] and v [B,T,H,Dv]")
    B, T, H, Dk = q.shape
    Dv = v.shape[3]
    dev = q.device
    code = _dtype_code(q)
    if log_alpha.shape != (B, T, H) or beta.shape != (B, T, H):
        raise GdnError("log_alpha and beta must be [B,T,H]")
    if d_o.shape != v.shape:
        raise GdnError("d_o must be [B,T,H,Dv]")
    state = (B, H, Dv, Dk)
    for x, n in ((S0, "S0"), (dS_T, "dS_T")):
        if x is not None and x.shape != state:
            raise GdnError(f"{n} must be [B,H,Dv,Dk]")
    opt = lambda x, n: _dev(x, n, torch.float32, dev) if x is not None else None
    args = [_dev(q, "q", q.dtype, dev), _dev(k, "k", q.dtype, dev), _dev(v, "v", q.dtype, dev),
            _dev(log_alpha, "log_alpha", torch.float32, dev),
            _dev(beta, "beta", torch.float32, dev), opt(S0, "S0"),
            _dev(d_o, "d_o", q.dtype, dev), opt(dS_T, "dS_T")]
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    dla = torch.empty((B, T, H), dtype=torch.float32, device=dev)
    dbe = torch.empty((B, T, H), dtype=torch.float32, device=dev)
    dS0 = torch.empty(state, dtype=torch.float32, device=dev) if want_dS0 else None
    args += [dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), dla.data_ptr(), dbe.data_ptr(),
             dS0.data_ptr() if dS0 is not None else None]
    need = int(LIB.gdn_chunk_bwd_workspace_size(B, T, H, Dk, Dv, chunk, code))
    ws_ptr, ws_bytes = None, 0
    if need:
        if workspace is None or workspace.numel() * workspace.element_size() < need:
            workspace = torch.empty(need, dtype=torch.uint8, device=dev)
        ws_ptr, ws_bytes = _dev(workspace, "workspace"), workspace.numel() * workspace.element_size()
    st = LIB.gdn_chunk_bwd(*args, B, T, H, Dk, Dv, chunk, code, ws_ptr, ws_bytes,
                           _stream_ptr(dev))
    _check(st, "gdn_chunk_bwd")
    return dq, dk, dv, dla, dbe, dS0


def chunk_bwd_path(B, T, H, Dk, Dv, chunk=64, dtype=torch.bfloat16) -> str:
    """Which kernels chunk_bwd runs for these sizes: "tcgen05", "simt" or "none"."""
    code = GDN_BF16 if dtype == torch.bfloat16 else GDN_F32
    st = int(LIB.gdn_chunk_bwd_path(B, T, H, Dk, Dv, chunk, code))
    if st < 0:
        raise GdnError("gdn_chunk_bwd_path: invalid sizes")
    return PATH_NAMES[st]


def chunk_fwd_cw_path(B, T, H, Dk, Dv, chunk=64, dtype=torch.bfloat16) -> str:
    """Which kernels chunk_fwd_cw runs for these sizes: "tcgen05", "simt" or "none"."""
    code = GDN_BF16 if dtype == torch.bfloat16 else GDN_F32
    st = int(LIB.gdn_chunk_fwd_cw_path(B, T, H, Dk, Dv, chunk, code))
    if st < 0:
        raise GdnError("gdn_chunk_fwd_cw_path: invalid sizes")
    return PATH_NAMES[st]


def chunk_fwd_cw_workspace_size(B, T, H, Dk, Dv, chunk=64, dtype=torch.bfloat16) -> int:
    code = GDN_BF16 if dtype == torch.bfloat16 else GDN_F32
    return int(LIB.gdn_chunk_fwd_cw_workspace_size(B, T, H, Dk, Dv, chunk, code))


def chunk_fwd_cw(q, k, v, log_alpha, b, w, S0=None, chunk: int = 64, out=None, S_T=None,
                 return_state: bool = True, workspace=None):
    """Channel-wise gates: S_t = S_{t-1} Diag(alpha_t)(I - (b_t o k_t) k_t^T) + (w_t o v_t) k_t^T.

    q, k [B,T,H,Dk], v [B,T,H,Dv] (float32 or bfloat16); log_alpha, b
    [B,T,H,Dk] and w [B,T,H,Dv] float32; S0 [B,H,Dv,Dk] float32 or None.
    Returns (o [B,T,H,Dv], S_T or None).
    """
    if q.dim() != 4 or k.shape != q.shape or v.dim() != 4 or v.shape[:3] != q.shape[:3]:
        raise GdnError("q, k must be [B,T,H,Dk] and v [B,T,H,Dv]")
    B, T, H, Dk = q.shape
    Dv = v.shape[3]
    dev = q.device
    code = _dtype_code(q)
    if log_alpha.shape != q.shape or b.shape != q.shape or w.shape != v.shape:
        raise GdnError("log_alpha and b must be [B,T,H,Dk] and w [B,T,H,Dv]")
    args = [_dev(q, "q", q.dtype, dev), _dev(k, "k", q.dtype, dev), _dev(v, "v", q.dtype, dev),
            _dev(log_alpha, "log_alpha", torch.float32, dev), _dev(b, "b", torch.float32, dev),
            _dev(w, "w", torch.float32, dev)]
    state = (B, H, Dv, Dk)
    if S0 is not None and S0.shape != state:
        raise GdnError("S0 must be [B,H,Dv,Dk]")
    args.append(_dev(S0, "S0", torch.float32, dev) if S0 is not None else None)
    o = out if out is not None else torch.empty((B, T, H, Dv), dtype=q.dtype, device=dev)
    if o.shape != (B, T, H, Dv):
        raise GdnError("out must be [B,T,H,Dv]")
    args.append(_dev(o, "out", q.dtype, dev))
    if S_T is None and return_state:
        S_T = torch.empty(state, dtype=torch.float32, device=dev)
    if S_T is not None and S_T.shape != state:
        raise GdnError("S_T must be [B,H,Dv,Dk]")
    args.append(_dev(S_T, "S_T", torch.float32, dev) if S_T is not None else None)
    need = int(LIB.gdn_chunk_fwd_cw_workspace_size(B, T, H, Dk, Dv, chunk, code))
    ws_ptr, ws_bytes = None, 0
    if need:
        if workspace is None or workspace.numel() * workspace.element_size() < need:
            workspace = torch.empty(need, dtype=torch.uint8, device=dev)
        ws_ptr, ws_bytes = _dev(workspace, "workspace"), workspace.numel() * workspace.element_size()
    st = LIB.gdn_chunk_fwd_cw(*args, B, T, H, Dk, Dv, chunk, code, ws_ptr, ws_bytes,
                              _stream_ptr(dev))
    _check(st, "gdn_chunk_fwd_cw")
    return o, S_T


def decode_step_cw(q, k, v, log_alpha, b, w, S, out=None):
    """One channel-wise-gate step for every (b, h); S [B,H,Dv,Dk] updated in place.
    q, k, log_alpha, b [B,H,Dk]; v, w [B,H,Dv].  Returns o [B,H,Dv]."""
    if q.dim() != 3 or k.shape != q.shape or v.dim() != 3 or v.shape[:2] != q.shape[:2]:
        raise GdnError("q, k must be [B,H,Dk] and v [B,H,Dv]")
    B, H, Dk = q.shape
    Dv = v.shape[2]
    dev = q.device
    if log_alpha.shape != q.shape or b.shape != q.shape or w.shape != v.shape:
        raise GdnError("log_alpha and b must be [B,H,Dk] and w [B,H,Dv]")
    if S.shape != (B, H, Dv, Dk):
        raise GdnError("S must be [B,H,Dv,Dk]")
    o = out if out is not None else torch.empty((B, H, Dv), dtype=q.dtype, device=dev)
    st = LIB.gdn_decode_step_cw(
        _dev(q, "q", q.dtype, dev), _dev(k, "k", q.dtype, dev), _dev(v, "v", q.dtype, dev),
        _dev(log_alpha, "log_alpha", torch.float32, dev), _dev(b, "b", torch.float32, dev),
        _dev(w, "w", torch.float32, dev), _dev(S, "S", torch.float32, dev),
        _dev(o, "out", q.dtype, dev), B, H, Dk, Dv, _dtype_code(q), _stream_ptr(dev))
    _check(st, "gdn_decode_step_cw")
    return o


def _host_offsets(cu_seqlens) -> torch.Tensor:
    cu = torch.as_tensor(cu_seqlens, dtype=torch.int32).cpu().contiguous()
    if cu.dim() != 1 or cu.numel() < 1:
        raise GdnError("cu_seqlens must be a 1-D list of N + 1 offsets")
    return cu


def chunk_fwd_varlen_workspace_size(cu_seqlens, H, Dk, Dv, chunk=64, dtype=torch.bfloat16,
                                    l2norm_qk: bool = False, gate_logits: bool = False) -> int:
    cu = _host_offsets(cu_seqlens)
    code = GDN_BF16 if dtype == torch.bfloat16 else GDN_F32
    return int(LIB.gdn_chunk_fwd_varlen_workspace_size(cu.data_ptr(), cu.numel() - 1, H, Dk, Dv,
                                                       chunk, code, _flags(l2norm_qk, gate_logits)))


def chunk_fwd_varlen(q, k, v, log_alpha, beta, cu_seqlens, S0=None, chunk: int = 64, out=None,
                     S_T=None, return_state: bool = True, workspace=None, l2norm_qk: bool = False,
                     gate_logits: bool = False, cu_seqlens_device=None):
    """Chunkwise forward over N variable-length sequences packed without padding.

    q, k [total, H, Dk], v [total, H, Dv], log_alpha, beta [total, H]; ``cu_seqlens``
    the N + 1 token offsets (host list or tensor; sequence n is tokens
    cu_seqlens[n] .. cu_seqlens[n + 1] - 1).  S0 / S_T are [N, H, Dv, Dk] float32.
    ``cu_seqlens_device``: the same offsets as an int32 tensor on q's device (else
    they are copied there on every call, a synchronous copy).
    Returns (o [total, H, Dv], S_T or None).
    """
    cu = _host_offsets(cu_seqlens)
    N = cu.numel() - 1
    if q.dim() != 3 or k.shape != q.shape or v.dim() != 3 or v.shape[:2] != q.shape[:2]:
        raise GdnError("q, k must be [total,H,Dk] and v [total,H,Dv]")
    total, H, Dk = q.shape
    Dv = v.shape[2]
    if int(cu[-1]) != total:
        raise GdnError("cu_seqlens[-1] must equal the number of packed tokens")
    dev = q.device
    code = _dtype_code(q)
    flags = _flags(l2norm_qk, gate_logits)
    if log_alpha.shape != (total, H) or beta.shape != (total, H):
        raise GdnError("log_alpha and beta must be [total,H]")
    args = [_dev(q, "q", q.dtype, dev), _dev(k, "k", q.dtype, dev), _dev(v, "v", q.dtype, dev),
            _dev(log_alpha, "log_alpha", torch.float32, dev), _dev(beta, "beta", torch.float32, dev)]
    if S0 is not None:
        if S0.shape != (N, H, Dv, Dk):
            raise GdnError("S0 must be [N,H,Dv,Dk]")
        args.append(_dev(S0, "S0", torch.float32, dev))
    else:
        args.append(None)
    o = out if out is not None else torch.empty((total, H, Dv), dtype=q.dtype, device=dev)
    if o.shape != (total, H, Dv):
        raise GdnError("out must be [total,H,Dv]")
    args.append(_dev(o, "out", q.dtype, dev))
    if S_T is None and return_state:
        S_T = torch.empty((N, H, Dv, Dk), dtype=torch.float32, device=dev)
    if S_T is not None:
        if S_T.shape != (N, H, Dv, Dk):
            raise GdnError("S_T must be [N,H,Dv,Dk]")
        args.append(_dev(S_T, "S_T", torch.float32, dev))
    else:
        args.append(None)
    if cu_seqlens_device is not None:
        if cu_seqlens_device.shape != cu.shape:
            raise GdnError("cu_seqlens_device must hold the N + 1 offsets")
        _dev(cu_seqlens_device, "cu_seqlens_device", torch.int32, dev)
        cu_dev = cu_seqlens_device
    else:
        cu_dev = cu.to(dev)
    need = int(LIB.gdn_chunk_fwd_varlen_workspace_size(cu.data_ptr(), N, H, Dk, Dv, chunk, code,
                                                       flags))
    ws_ptr, ws_bytes = None, 0
    if need:
        if workspace is None or workspace.numel() * workspace.element_size() < need:
            workspace = torch.empty(need, dtype=torch.uint8, device=dev)
        ws_ptr, ws_bytes = _dev(workspace, "workspace"), workspace.numel() * workspace.element_size()
    st = LIB.gdn_chunk_fwd_varlen(*args, cu_dev.data_ptr(), cu.data_ptr(), N, H, Dk, Dv, chunk,
                                  code, flags, ws_ptr, ws_bytes, _stream_ptr(dev))
    _check(st, "gdn_chunk_fwd_varlen")
    return o, S_T


def decode_step(q, k, v, log_alpha, beta, S, out=None, l2norm_qk: bool = False,
                gate_logits: bool = False):
    """One recurrent step for every (b,h); S [B,H,Dv,Dk] float32 is updated in place.

    q, k [B,H,Dk], v [B,H,Dv] float32 or bfloat16; log_alpha, beta [B,H] float32.
    Returns o [B,H,Dv] in q's dtype.  ``l2norm_qk`` / ``gate_logits``: the input
    prologue, as in ``chunk_fwd``.
    """
    if q.dim() != 3 or k.shape != q.shape or v.dim() != 3 or v.shape[:2] != q.shape[:2]:
        raise GdnError("q, k must be [B,H,Dk] and v [B,H,Dv]")
    B, H, Dk = q.shape
    Dv = v.shape[2]
    dev = q.device
    code = _dtype_code(q)
    if log_alpha.shape != (B, H) or beta.shape != (B, H) or S.shape != (B, H, Dv, Dk):
        raise GdnError("log_alpha, beta must be [B,H] and S [B,H,Dv,Dk]")
    o = out if out is not None else torch.empty((B, H, Dv), dtype=q.dtype, device=dev)
    st = LIB.gdn_decode_step_ex(
        _dev(q, "q", q.dtype, dev), _dev(k, "k", q.dtype, dev), _dev(v, "v", q.dtype, dev),
        _dev(log_alpha, "log_alpha", torch.float32, dev), _dev(beta, "beta", torch.float32, dev),
        _dev(S, "S", torch.float32, dev), _dev(o, "out", q.dtype, dev), B, H, Dk, Dv, code,
        _flags(l2norm_qk, gate_logits), _stream_ptr(dev))
    _check(st, "gdn_decode_step")
    return o
