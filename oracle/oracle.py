"""Python binding of the float64 CPU oracle (``gdn_oracle.c``).

TEST INFRASTRUCTURE ONLY: the test suite, the smoke check and the benchmark's
CPU-baseline leg are the only callers.  The CUDA library never imports, links or
executes anything in this directory, and this module imports nothing from it.

The oracle is the gated delta rule applied token by token in float64,
    S_t = S_{t-1} (alpha_t (I - beta_t k_t k_t^T)) + beta_t v_t k_t^T,  o_t = S_t q_t,
and its exact reverse-mode gradient (``backward``); see the header of
``gdn_oracle.c`` for the pages it follows and the readings taken.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "gdn_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile ``gdn_oracle.c`` into ``liboracle.so`` next to it (plain gcc)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(
            ["gcc", "-O2", "-ffp-contract=off", "-fno-fast-math", "-Wall", "-shared", "-fPIC",
             "-pthread", _SRC, "-o", tmp, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _bind(path: str):
    lib = ctypes.CDLL(path)
    dp = ctypes.POINTER(ctypes.c_double)
    ip = ctypes.POINTER(ctypes.c_int)
    L = ctypes.c_long
    lib.gdn_oracle_forward.argtypes = [dp, dp, dp, dp, dp, dp, dp, dp, L, L, L, L, L,
                                       ip, ctypes.c_int, ctypes.c_int]
    lib.gdn_oracle_forward.restype = ctypes.c_int
    lib.gdn_oracle_decode.argtypes = [dp, dp, dp, dp, dp, dp, dp, L, L, L, L, L,
                                      ip, ctypes.c_int, ctypes.c_int]
    lib.gdn_oracle_decode.restype = ctypes.c_int
    lib.gdn_oracle_backward.argtypes = [dp] * 14 + [L, L, L, L, L, ip, ctypes.c_int,
                                                    ctypes.c_int]
    lib.gdn_oracle_backward.restype = ctypes.c_int
    lib.gdn_oracle_forward_cw.argtypes = [dp] * 9 + [L, L, L, L, L, ip, ctypes.c_int,
                                                     ctypes.c_int]
    lib.gdn_oracle_forward_cw.restype = ctypes.c_int
    return lib


def _load():
    global _lib
    with _lock:
        if _lib is None:
            _lib = _bind(build())
    return _lib


def _f64(x) -> np.ndarray:
    """Contiguous float64 copy of a numpy array or CPU torch tensor."""
    if hasattr(x, "detach"):  # torch tensor: widen on the torch side (handles bf16)
        x = x.detach().to("cpu").double().numpy()
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def _ptr(a: np.ndarray | None):
    if a is None:
        return None
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def _units(units, n_all):
    if units is None:
        return None, 0, None
    arr = np.ascontiguousarray(np.asarray(units, dtype=np.int32))
    if arr.ndim != 1 or (arr.size and (arr.min() < 0 or arr.max() >= n_all)):
        raise ValueError("units must be a 1-D list of (b*H + h) indices in range")
    return arr.ctypes.data_as(ctypes.POINTER(ctypes.c_int)), int(arr.size), arr


def default_threads() -> int:
    return os.cpu_count() or 1


def forward(q, k, v, log_alpha, beta, S0=None, units=None, nthreads=None, lib=None):
    """Token-by-token recurrence over a whole sequence.

    q,k [B,T,H,Dk]; v [B,T,H,Dv]; log_alpha, beta [B,T,H]; S0 [B,H,Dv,Dk] or None.
    Returns (o [B,T,H,Dv], S_T [B,H,Dv,Dk]) as float64 arrays.  With ``units`` (a
    list of b*H + h indices) only those heads are computed; the other slices of
    the outputs are NaN.  ``lib`` selects another build of the same source
    (the tests use it to check that the pins reject planted mistakes).
    """
    q, k, v, la, be = (_f64(x) for x in (q, k, v, log_alpha, beta))
    B, T, H, Dk = q.shape
    Dv = v.shape[-1]
    if k.shape != q.shape or v.shape[:3] != (B, T, H) or la.shape != (B, T, H) \
            or be.shape != (B, T, H):
        raise ValueError("shape mismatch")
    s0 = None if S0 is None else _f64(S0)
    if s0 is not None and s0.shape != (B, H, Dv, Dk):
        raise ValueError("S0 must be [B,H,Dv,Dk]")
    fill = np.nan if units is not None else 0.0
    o = np.full((B, T, H, Dv), fill)
    st = np.full((B, H, Dv, Dk), fill)
    up, nu, _keep = _units(units, B * H)
    rc = (lib or _load()).gdn_oracle_forward(
        _ptr(q), _ptr(k), _ptr(v), _ptr(la), _ptr(be), _ptr(s0), _ptr(o), _ptr(st),
        B, T, H, Dk, Dv, up, nu, int(nthreads or default_threads()))
    if rc != 0:
        raise RuntimeError(f"gdn_oracle_forward failed ({rc})")
    return o, st


def decode(q, k, v, log_alpha, beta, S, units=None, nthreads=None, lib=None):
    """``steps`` successive single-token updates.

    q,k [steps,B,H,Dk]; v [steps,B,H,Dv]; log_alpha, beta [steps,B,H];
    S [B,H,Dv,Dk] initial state.  Returns (o [steps,B,H,Dv], S_final) in float64.
    """
    q, k, v, la, be = (_f64(x) for x in (q, k, v, log_alpha, beta))
    steps, B, H, Dk = q.shape
    Dv = v.shape[-1]
    s = _f64(S).copy()
    if s.shape != (B, H, Dv, Dk):
        raise ValueError("S must be [B,H,Dv,Dk]")
    o = np.full((steps, B, H, Dv), np.nan if units is not None else 0.0)
    up, nu, _keep = _units(units, B * H)
    rc = (lib or _load()).gdn_oracle_decode(
        _ptr(q), _ptr(k), _ptr(v), _ptr(la), _ptr(be), _ptr(s), _ptr(o),
        steps, B, H, Dk, Dv, up, nu, int(nthreads or default_threads()))
    if rc != 0:
        raise RuntimeError(f"gdn_oracle_decode failed ({rc})")
    return o, s


def backward(q, k, v, log_alpha, beta, S0, d_o, dS_T=None, units=None, nthreads=None, lib=None):
    """Exact gradients of a scalar loss through the whole-sequence recurrence.

    Inputs as for ``forward`` plus d_o = dL/do [B,T,H,Dv] and dS_T = dL/dS_T
    [B,H,Dv,Dk] (None: zero).  Returns (dq, dk, dv, dlog_alpha, dbeta, dS0) as
    float64 arrays in the layouts of q, k, v, log_alpha, beta and S0.  With
    ``units`` only those heads are computed (NaN elsewhere).
    """
    q, k, v, la, be, do = (_f64(x) for x in (q, k, v, log_alpha, beta, d_o))
    B, T, H, Dk = q.shape
    Dv = v.shape[-1]
    if k.shape != q.shape or v.shape[:3] != (B, T, H) or la.shape != (B, T, H) \
            or be.shape != (B, T, H) or do.shape != v.shape:
        raise ValueError("shape mismatch")
    s0 = None if S0 is None else _f64(S0)
    ds = None if dS_T is None else _f64(dS_T)
    for x, n in ((s0, "S0"), (ds, "dS_T")):
        if x is not None and x.shape != (B, H, Dv, Dk):
            raise ValueError(f"{n} must be [B,H,Dv,Dk]")
    fill = np.nan if units is not None else 0.0
    out = [np.full(q.shape, fill), np.full(q.shape, fill), np.full(v.shape, fill),
           np.full(la.shape, fill), np.full(la.shape, fill), np.full((B, H, Dv, Dk), fill)]
    up, nu, _keep = _units(units, B * H)
    rc = (lib or _load()).gdn_oracle_backward(
        _ptr(q), _ptr(k), _ptr(v), _ptr(la), _ptr(be), _ptr(s0), _ptr(do), _ptr(ds),
        *(_ptr(a) for a in out), B, T, H, Dk, Dv, up, nu, int(nthreads or default_threads()))
    if rc != 0:
        raise RuntimeError(f"gdn_oracle_backward failed ({rc})")
    return tuple(out)


def forward_cw(q, k, v, log_alpha, b, w, S0=None, units=None, nthreads=None, lib=None):
    """Channel-wise gates (Gated DeltaNet-2 reading, see gdn_oracle.c):
    S_t = S_{t-1} Diag(alpha_t) (I - (b_t o k_t) k_t^T) + (w_t o v_t) k_t^T, o_t = S_t q_t.

    q, k, log_alpha, b [B,T,H,Dk]; v, w [B,T,H,Dv]; S0 [B,H,Dv,Dk] or None.
    Returns (o [B,T,H,Dv], S_T [B,H,Dv,Dk]) in float64 (NaN outside ``units``).
    """
    q, k, v, la, bb, ww = (_f64(x) for x in (q, k, v, log_alpha, b, w))
    B, T, H, Dk = q.shape
    Dv = v.shape[-1]
    if k.shape != q.shape or la.shape != q.shape or bb.shape != q.shape or \
            v.shape[:3] != (B, T, H) or ww.shape != v.shape:
        raise ValueError("shape mismatch")
    s0 = None if S0 is None else _f64(S0)
    if s0 is not None and s0.shape != (B, H, Dv, Dk):
        raise ValueError("S0 must be [B,H,Dv,Dk]")
    fill = np.nan if units is not None else 0.0
    o = np.full((B, T, H, Dv), fill)
    st = np.full((B, H, Dv, Dk), fill)
    up, nu, _keep = _units(units, B * H)
    rc = (lib or _load()).gdn_oracle_forward_cw(
        _ptr(q), _ptr(k), _ptr(v), _ptr(la), _ptr(bb), _ptr(ww), _ptr(s0), _ptr(o), _ptr(st),
        B, T, H, Dk, Dv, up, nu, int(nthreads or default_threads()))
    if rc != 0:
        raise RuntimeError(f"gdn_oracle_forward_cw failed ({rc})")
    return o, st


def load_variant(path: str):
    """Bind another build of ``gdn_oracle.c`` (for the tests' planted-mistake checks)."""
    return _bind(path)


SOURCE = _SRC
