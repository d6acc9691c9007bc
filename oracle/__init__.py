"""fp64 CPU oracle for ReplaySSM decode -- TEST INFRASTRUCTURE.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline /
reference arm may import this package.  The CUDA library never links, loads or
calls it, and it imports nothing from the CUDA package.

The arithmetic lives in ``oracle.c`` (double precision, libm ``exp``, no
fast-math, no contraction); this module only marshals numpy arrays.

Parity status of each function (what pins it is listed in the test-suite,
``tests/test_oracle_pins.py``):
  mamba2_eager / mamba2_eager_batch   pinned (closed forms, special cases)
  mamba2_replay                       pinned (== eager, brute force over L)
  gdn_eager / gdn_eager_batch         pinned (closed forms, special cases,
                                      autograd gradient step, golden fixture)
  gdn_replay                          pinned (== eager, brute force over L)
  bf16_rne, e4m3_rne_satfinite        pinned (torch casts, hand-derived codes)
  e4m3_quantize_tile                  pinned (format definition + decode bound)
"""
import ctypes
import os

import numpy as np

from . import build as _build

_HERE = os.path.dirname(os.path.abspath(__file__))
_lib = None

_dp = ctypes.POINTER(ctypes.c_double)


def _load():
    global _lib
    if _lib is None:
        path = _build.build()
        lib = ctypes.CDLL(path)
        i, d = ctypes.c_int, ctypes.c_double
        lib.oracle_mamba2_eager.argtypes = [i, i, i, d, d, _dp, _dp, _dp, _dp, _dp, _dp]
        lib.oracle_mamba2_replay.argtypes = [i, i, i, d, d, _dp, _dp, _dp, _dp, _dp, _dp]
        lib.oracle_gdn_eager.argtypes = [i, i, i, d, _dp, _dp, _dp, _dp, _dp, _dp, _dp]
        lib.oracle_gdn_replay.argtypes = [i, i, i, d, _dp, _dp, _dp, _dp, _dp, _dp, _dp]
        lib.oracle_mamba2_eager_batch.argtypes = [i, i, i, i, _dp, _dp, _dp, _dp, _dp, _dp,
                                                  _dp, _dp, i]
        lib.oracle_mamba2_eager_batch.restype = i
        lib.oracle_gdn_eager_batch.argtypes = [i, i, i, i, d, _dp, _dp, _dp, _dp, _dp, _dp,
                                               _dp, i]
        lib.oracle_gdn_eager_batch.restype = i
        vp, ll = ctypes.c_void_p, ctypes.c_longlong
        lib.oracle_bf16_rne_array.argtypes = [vp, vp, ll]
        lib.oracle_e4m3_rne_satfinite_array.argtypes = [vp, vp, ll]
        lib.oracle_e4m3_decode_array.argtypes = [vp, vp, ll]
        _lib = lib
    return _lib


def _d(a):
    """Contiguous float64 copy (or view) of ``a``."""
    return np.ascontiguousarray(np.asarray(a, dtype=np.float64))


def _p(a):
    return a.ctypes.data_as(_dp)


def default_threads() -> int:
    return os.cpu_count() or 1


# --------------------------------------------------------------------------
# Mamba-2
# --------------------------------------------------------------------------

def mamba2_eager(A, D, x, dt, B, C, h0=None):
    """Eager Mamba-2 over T steps for one (sequence, head).

    x [T,P], dt [T], B [T,N], C [T,N]; h0 [P,N] (zeros if None).
    Returns (y [T,P], h_T [P,N]).
    """
    x, dt, B, C = _d(x), _d(dt), _d(B), _d(C)
    T, P = x.shape
    N = B.shape[1]
    h = np.zeros((P, N)) if h0 is None else _d(h0).copy()
    y = np.empty((T, P))
    _load().oracle_mamba2_eager(P, N, T, float(A), float(D), _p(x), _p(dt), _p(B), _p(C),
                                _p(h), _p(y))
    return y, h


def mamba2_replay(A, D, S0, x, dt, B, C):
    """Replay-form output of the newest of L buffered entries (x [L,P], dt [L],
    B [L,N], C [L,N]; only C[L-1] enters) against checkpoint S0 [P,N]."""
    S0, x, dt, B, C = _d(S0), _d(x), _d(dt), _d(B), _d(C)
    L, P = x.shape
    N = B.shape[1]
    y = np.empty(P)
    _load().oracle_mamba2_replay(P, N, L, float(A), float(D), _p(S0), _p(x), _p(dt), _p(B),
                                 _p(C), _p(y))
    return y


def mamba2_eager_batch(A, D, x, dt, B, C, h=None, want_y=True, nthreads=None):
    """Independent pairs: A, D [n]; x [n,T,P]; dt [n,T]; B, C [n,T,N];
    h [n,P,N] in/out (zeros if None; the array passed is updated in place
    when it is already contiguous float64).  Returns (y [n,T,P] or None, h)."""
    A, D, x, dt, B, C = _d(A), _d(D), _d(x), _d(dt), _d(B), _d(C)
    n, T, P = x.shape
    N = B.shape[2]
    if h is None:
        h = np.zeros((n, P, N))
    elif not (isinstance(h, np.ndarray) and h.dtype == np.float64 and h.flags.c_contiguous):
        h = _d(h).copy()
    y = np.empty((n, T, P)) if want_y else None
    _load().oracle_mamba2_eager_batch(n, P, N, T, _p(A), _p(D), _p(x), _p(dt), _p(B), _p(C),
                                      _p(h), _p(y) if want_y else None,
                                      int(nthreads or default_threads()))
    return y, h


# --------------------------------------------------------------------------
# Gated DeltaNet
# --------------------------------------------------------------------------

def gdn_eager(q, k, v, alpha, beta, S0=None, scale=1.0):
    """Eager Gated DeltaNet over T steps for one (sequence, head).

    q, k [T,dk], v [T,dv], alpha, beta [T]; S0 [dv,dk] (zeros if None).
    Returns (o [T,dv], S_T [dv,dk])."""
    q, k, v, alpha, beta = _d(q), _d(k), _d(v), _d(alpha), _d(beta)
    T, DK = k.shape
    DV = v.shape[1]
    S = np.zeros((DV, DK)) if S0 is None else _d(S0).copy()
    o = np.empty((T, DV))
    _load().oracle_gdn_eager(DV, DK, T, float(scale), _p(q), _p(k), _p(v), _p(alpha), _p(beta),
                             _p(S), _p(o))
    return o, S


def gdn_replay(S0, k, v, alpha, beta, q, scale=1.0):
    """Replay-form output for the newest of L buffered entries (k [L,dk],
    v [L,dv], alpha, beta [L]) with query q [dk] against checkpoint S0 [dv,dk]."""
    S0, k, v, alpha, beta, q = _d(S0), _d(k), _d(v), _d(alpha), _d(beta), _d(q)
    L, DK = k.shape
    DV = v.shape[1]
    o = np.empty(DV)
    _load().oracle_gdn_replay(DV, DK, L, float(scale), _p(S0), _p(k), _p(v), _p(alpha),
                              _p(beta), _p(q), _p(o))
    return o


def gdn_eager_batch(q, k, v, alpha, beta, S=None, scale=1.0, want_o=True, nthreads=None):
    """Independent pairs: q, k [n,T,dk]; v [n,T,dv]; alpha, beta [n,T];
    S [n,dv,dk] in/out.  Returns (o [n,T,dv] or None, S)."""
    q, k, v, alpha, beta = _d(q), _d(k), _d(v), _d(alpha), _d(beta)
    n, T, DK = k.shape
    DV = v.shape[2]
    if S is None:
        S = np.zeros((n, DV, DK))
    elif not (isinstance(S, np.ndarray) and S.dtype == np.float64 and S.flags.c_contiguous):
        S = _d(S).copy()
    o = np.empty((n, T, DV)) if want_o else None
    _load().oracle_gdn_eager_batch(n, DV, DK, T, float(scale), _p(q), _p(k), _p(v), _p(alpha),
                                   _p(beta), _p(S), _p(o) if want_o else None,
                                   int(nthreads or default_threads()))
    return o, S


# --------------------------------------------------------------------------
# Number formats
# --------------------------------------------------------------------------

def bf16_rne(a):
    """float32 array -> uint16 bf16 codes, round to nearest even."""
    a = np.ascontiguousarray(np.asarray(a, dtype=np.float32))
    out = np.empty(a.shape, dtype=np.uint16)
    _load().oracle_bf16_rne_array(a.ctypes.data, out.ctypes.data, a.size)
    return out


def bf16_decode(codes):
    codes = np.ascontiguousarray(np.asarray(codes, dtype=np.uint16))
    return (codes.astype(np.uint32) << 16).view(np.float32)


def e4m3_rne_satfinite(a):
    """float32 array -> uint8 OCP E4M3 codes (RNE, satfinite)."""
    a = np.ascontiguousarray(np.asarray(a, dtype=np.float32))
    out = np.empty(a.shape, dtype=np.uint8)
    _load().oracle_e4m3_rne_satfinite_array(a.ctypes.data, out.ctypes.data, a.size)
    return out


def e4m3_decode(codes):
    codes = np.ascontiguousarray(np.asarray(codes, dtype=np.uint8))
    out = np.empty(codes.shape, dtype=np.float32)
    _load().oracle_e4m3_decode_array(codes.ctypes.data, out.ctypes.data, codes.size)
    return out


E4M3_MAX = 448.0


def e4m3_quantize_tile(master):
    """Quantise one (sequence, head) fp32 tile to the fp8 output copy.

    Reading of the pages (step 5 of the explainer names a low-precision copy
    but no format): one fp32 scale per tile, scale = absmax / 448 in fp32
    (1.0 when the tile is all zero), code = E4M3_RNE_satfinite(s / scale)
    with an IEEE fp32 division.  Returns (codes uint8, scale float32)."""
    m = np.asarray(master, dtype=np.float32)
    amax = np.float32(np.max(np.abs(m))) if m.size else np.float32(0.0)
    scale = np.float32(amax / np.float32(E4M3_MAX)) if amax > 0 else np.float32(1.0)
    return e4m3_rne_satfinite((m / scale).astype(np.float32)), scale


__all__ = [
    "mamba2_eager", "mamba2_replay", "mamba2_eager_batch",
    "gdn_eager", "gdn_replay", "gdn_eager_batch",
    "bf16_rne", "bf16_decode", "e4m3_rne_satfinite", "e4m3_decode", "e4m3_quantize_tile",
    "default_threads",
]
