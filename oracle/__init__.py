"""CPU oracle of the Mamba selective scan -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` /
``--impl reference`` legs of ``bench.py`` may import this package.  The
product (``selective_state_space_37_b200``) never imports it, and this package
imports nothing from the product.

The arithmetic lives in ``ss_oracle.c`` (plain loops, written from the
equations of "Understanding Mamba and Selective State Space Models (SSMs)",
§2.1, §2.2 first and second cut, §3.1 and §4.3); this module only marshals
numpy arrays through ctypes.

Array conventions (numpy, any float dtype; converted to float64 exactly):
  u, delta, z : [batch, L, d]      B, C : [batch, L, N]
  A : [d, N]    D, delta_bias : [d]
Returned outputs are float64: y [batch, L, d] and last_state [batch, d, N].
"""
import ctypes
import os

import numpy as np

from . import build as _build

_LIB = None
_DP = ctypes.POINTER(ctypes.c_double)
_I64 = ctypes.c_int64


def _lib():
    global _LIB
    if _LIB is None:
        path = _build.build()
        lib = ctypes.CDLL(path)
        fwd_args = [_DP, _DP, _DP, _DP, _DP, _DP, _DP, _DP, _DP, _DP,
                    _I64, _I64, _I64, _I64, ctypes.c_int]
        for name in ("ss_oracle_fwd_f64", "ss_oracle_fwd_f32"):
            fn = getattr(lib, name)
            fn.argtypes = fwd_args
            fn.restype = ctypes.c_int
        lib.ss_oracle_fwd_chunked_f64.argtypes = fwd_args + [_I64]
        lib.ss_oracle_fwd_chunked_f64.restype = ctypes.c_int
        step_args = [_DP, _DP, _DP, _DP, _DP, _DP, _DP, _DP, _DP, _DP,
                     _I64, _I64, _I64, ctypes.c_int]
        for name in ("ss_oracle_step_f64", "ss_oracle_step_f32"):
            fn = getattr(lib, name)
            fn.argtypes = step_args
            fn.restype = ctypes.c_int
        lib.ss_oracle_bwd_f64.argtypes = [_DP] * 18 + [_I64, _I64, _I64, _I64, ctypes.c_int]
        lib.ss_oracle_bwd_f64.restype = ctypes.c_int
        lib.ss_oracle_conv_silu_f64.argtypes = [_DP, _DP, _DP, _DP, _I64, _I64, _I64, _I64]
        lib.ss_oracle_conv_silu_f64.restype = ctypes.c_int
        lib.ss_oracle_ssd_f64.argtypes = [_DP] * 9 + [_I64, _I64, _I64, _I64, _I64, ctypes.c_int]
        lib.ss_oracle_ssd_f64.restype = ctypes.c_int
        lib.ss_oracle_set_mutation.argtypes = [ctypes.c_int]
        lib.ss_oracle_get_mutation.restype = ctypes.c_int
        lib.ss_oracle_max_threads.restype = ctypes.c_int
        lib.ss_oracle_set_threads.argtypes = [ctypes.c_int]
        _LIB = lib
    return _LIB


def _arr(x, shape=None):
    if x is None:
        return None, None
    a = np.ascontiguousarray(np.asarray(x, dtype=np.float64))
    if shape is not None and a.shape != tuple(shape):
        raise ValueError(f"oracle: expected shape {tuple(shape)}, got {a.shape}")
    return a, a.ctypes.data_as(_DP)


def _null():
    return ctypes.cast(None, _DP)


def _ptr(p):
    return p if p is not None else _null()


def _prep_fwd(u, delta, A, B, C, D, z, delta_bias):
    u = np.asarray(u)
    if u.ndim != 3:
        raise ValueError("oracle: u must be [batch, L, d]")
    batch, L, d = u.shape
    A_ = np.asarray(A)
    N = A_.shape[1]
    keep = []
    ptrs = []
    for x, shp in ((u, (batch, L, d)), (delta, (batch, L, d)), (delta_bias, (d,)),
                   (A, (d, N)), (B, (batch, L, N)), (C, (batch, L, N)), (D, (d,)),
                   (z, (batch, L, d))):
        a, p = _arr(x, shp)
        keep.append(a)
        ptrs.append(_ptr(p))
    return (batch, L, d, N), keep, ptrs


def fwd(u, delta, A, B, C, D=None, z=None, delta_bias=None, softplus=True,
        precision="f64"):
    """Sequential forward scan. Returns (y [b,L,d], last_state [b,d,N]) in float64."""
    (batch, L, d, N), keep, p = _prep_fwd(u, delta, A, B, C, D, z, delta_bias)
    y = np.empty((batch, L, d), dtype=np.float64)
    st = np.empty((batch, d, N), dtype=np.float64)
    fn = {"f64": _lib().ss_oracle_fwd_f64, "f32": _lib().ss_oracle_fwd_f32}[precision]
    rc = fn(p[0], p[1], p[2], p[3], p[4], p[5], p[6], p[7],
            y.ctypes.data_as(_DP), st.ctypes.data_as(_DP), batch, L, d, N, int(bool(softplus)))
    if rc != 0:
        raise ValueError(f"oracle fwd rejected sizes (rc={rc})")
    del keep
    return y, st


def fwd_chunked(u, delta, A, B, C, D=None, z=None, delta_bias=None, softplus=True,
                chunk=1):
    """Chunked (re-associated) forward scan in float64; same outputs as fwd()."""
    (batch, L, d, N), keep, p = _prep_fwd(u, delta, A, B, C, D, z, delta_bias)
    y = np.empty((batch, L, d), dtype=np.float64)
    st = np.empty((batch, d, N), dtype=np.float64)
    rc = _lib().ss_oracle_fwd_chunked_f64(p[0], p[1], p[2], p[3], p[4], p[5], p[6], p[7],
                                          y.ctypes.data_as(_DP), st.ctypes.data_as(_DP),
                                          batch, L, d, N, int(bool(softplus)), int(chunk))
    if rc != 0:
        raise ValueError(f"oracle fwd_chunked rejected sizes (rc={rc})")
    del keep
    return y, st


def step(state, u, delta, A, B, C, D=None, z=None, delta_bias=None, softplus=True,
         precision="f64"):
    """One decode step. state [b,d,N]; u, delta, z [b,d]; B, C [b,N].
    Returns (new_state [b,d,N], y [b,d]) in float64; the input is not modified."""
    st = np.array(state, dtype=np.float64, copy=True, order="C")
    batch, d, N = st.shape
    keep = []
    ptrs = []
    for x, shp in ((u, (batch, d)), (delta, (batch, d)), (delta_bias, (d,)), (A, (d, N)),
                   (B, (batch, N)), (C, (batch, N)), (D, (d,)), (z, (batch, d))):
        a, pp = _arr(x, shp)
        keep.append(a)
        ptrs.append(_ptr(pp))
    y = np.empty((batch, d), dtype=np.float64)
    fn = {"f64": _lib().ss_oracle_step_f64, "f32": _lib().ss_oracle_step_f32}[precision]
    rc = fn(st.ctypes.data_as(_DP), ptrs[0], ptrs[1], ptrs[2], ptrs[3], ptrs[4], ptrs[5],
            ptrs[6], ptrs[7], y.ctypes.data_as(_DP), batch, d, N, int(bool(softplus)))
    if rc != 0:
        raise ValueError(f"oracle step rejected sizes (rc={rc})")
    del keep
    return st, y


def bwd(u, delta, A, B, C, dy, D=None, z=None, delta_bias=None, dlast=None, softplus=True):
    """Backward of fwd() in float64: gradients of J = Σ dy·y + Σ dlast·last_state.

    Returns a dict with du, ddelta, dz [b,L,d] (dz only with z), dB, dC [b,L,N],
    dA [d,N], dD [d] (only with D) and dbias [d] (only with delta_bias)."""
    (batch, L, d, N), keep, p = _prep_fwd(u, delta, A, B, C, D, z, delta_bias)
    dya, dyp = _arr(dy, (batch, L, d))
    dla, dlp = _arr(dlast, (batch, d, N))
    out = {"du": np.empty((batch, L, d)), "ddelta": np.empty((batch, L, d)),
           "dA": np.empty((d, N)), "dB": np.empty((batch, L, N)), "dC": np.empty((batch, L, N))}
    if D is not None:
        out["dD"] = np.empty((d,))
    if z is not None:
        out["dz"] = np.empty((batch, L, d))
    if delta_bias is not None:
        out["dbias"] = np.empty((d,))

    def op(k):
        return out[k].ctypes.data_as(_DP) if k in out else _null()

    rc = _lib().ss_oracle_bwd_f64(p[0], p[1], p[2], p[3], p[4], p[5], p[6], p[7], dyp, _ptr(dlp),
                                  op("du"), op("ddelta"), op("dA"), op("dB"), op("dC"), op("dD"),
                                  op("dz"), op("dbias"), batch, L, d, N, int(bool(softplus)))
    if rc != 0:
        raise ValueError(f"oracle bwd rejected sizes (rc={rc})")
    del keep, dya, dla
    return out


def conv_silu(x, w, bias=None):
    """Causal depthwise conv1d (width w.shape[1]) then SiLU, float64.
    x [batch, L, d]; w [d, W]; bias [d] or None.  Returns u [batch, L, d]."""
    xa = np.ascontiguousarray(np.asarray(x, dtype=np.float64))
    if xa.ndim != 3:
        raise ValueError("oracle: x must be [batch, L, d]")
    batch, L, d = xa.shape
    wa, wp = _arr(w)
    if wa.ndim != 2 or wa.shape[0] != d:
        raise ValueError("oracle: w must be [d, W]")
    ba, bp = _arr(bias, (d,))
    u = np.empty_like(xa)
    rc = _lib().ss_oracle_conv_silu_f64(xa.ctypes.data_as(_DP), wp, _ptr(bp), u.ctypes.data_as(_DP),
                                        batch, L, d, wa.shape[1])
    if rc != 0:
        raise ValueError(f"oracle conv_silu rejected sizes (rc={rc})")
    del ba
    return u


def ssd(x, dt, A, B, C, D=None, dt_bias=None, softplus=True):
    """Multi-head scan with a scalar decay per head, float64, plain recurrence.
    x [b, L, H, P]; dt [b, L, H]; A, D, dt_bias [H]; B, C [b, L, N].
    Returns (y [b, L, H, P], final_state [b, H, P, N])."""
    xa = np.ascontiguousarray(np.asarray(x, dtype=np.float64))
    batch, L, H, P = xa.shape
    N = np.asarray(B).shape[-1]
    keep = []
    ptrs = []
    for v, shp in ((dt, (batch, L, H)), (dt_bias, (H,)), (A, (H,)), (B, (batch, L, N)), (C, (batch, L, N)),
                   (D, (H,))):
        a, pp = _arr(v, shp)
        keep.append(a)
        ptrs.append(_ptr(pp))
    y = np.empty_like(xa)
    st = np.empty((batch, H, P, N))
    rc = _lib().ss_oracle_ssd_f64(xa.ctypes.data_as(_DP), ptrs[0], ptrs[1], ptrs[2], ptrs[3], ptrs[4], ptrs[5],
                                  y.ctypes.data_as(_DP), st.ctypes.data_as(_DP), batch, L, H, P, N,
                                  int(bool(softplus)))
    if rc != 0:
        raise ValueError(f"oracle ssd rejected sizes (rc={rc})")
    del keep
    return y, st


def set_mutation(m: int) -> None:
    """Test-only: plant deliberate mistake number m (0 restores the oracle)."""
    _lib().ss_oracle_set_mutation(int(m))


def get_mutation() -> int:
    return _lib().ss_oracle_get_mutation()


def max_threads() -> int:
    return _lib().ss_oracle_max_threads()


def set_threads(n: int) -> None:
    _lib().ss_oracle_set_threads(int(n))


def library_path() -> str:
    return _build.LIB


__all__ = ["fwd", "fwd_chunked", "step", "bwd", "conv_silu", "ssd", "set_mutation", "get_mutation",
           "max_threads", "set_threads", "library_path"]

if os.environ.get("SS_ORACLE_THREADS"):
    set_threads(int(os.environ["SS_ORACLE_THREADS"]))
