"""CPU oracle for the decay-masked linear-attention (SSD) forward operator.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this package.  It is a plain,
slow, double-precision restatement of the method on the 2Mamba2Furious pages
(Algorithms 1-6) and shares no code with the CUDA library.

The arithmetic lives in ``ssd_oracle.c`` (plain C, double precision, OpenMP
over heads and rows); this module only compiles it with gcc and marshals numpy
arrays through ctypes.  Every function takes the same layouts as the CUDA
entry points: q, k, v are [B, H, N, d]; dt_p is [B, H, N]; A_log and dt_bias
are [H]; D is [H*d] or None.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Optional, Sequence

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "ssd_oracle.c")
_LIB = os.path.join(_HERE, "libssd_oracle.so")
_lib = None

_f32p = ctypes.POINTER(ctypes.c_float)
_f64p = ctypes.POINTER(ctypes.c_double)
_i32p = ctypes.POINTER(ctypes.c_int)


def build(force: bool = False) -> str:
    """Compile ssd_oracle.c into libssd_oracle.so next to it (gcc, -O2, OpenMP)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        cmd = ["gcc", "-O2", "-fno-fast-math", "-fopenmp", "-shared", "-fPIC",
               "-o", _LIB, _SRC, "-lm"]
        subprocess.check_call(cmd)
    return _LIB


def _load():
    global _lib
    if _lib is not None:
        return _lib
    build()
    lib = ctypes.CDLL(_LIB)
    lib.oracle_softplus.argtypes = [ctypes.c_double]
    lib.oracle_softplus.restype = ctypes.c_double
    lib.oracle_mask.argtypes = [_f64p, ctypes.c_int, ctypes.c_int]
    lib.oracle_mask.restype = ctypes.c_double
    lib.oracle_feature.argtypes = [_f64p, ctypes.c_int, ctypes.c_int, _f64p]
    lib.oracle_feature.restype = ctypes.c_int
    lib.oracle_log_decay.argtypes = [_f32p, _f32p, _f32p, _f32p, ctypes.c_int, ctypes.c_int,
                                     ctypes.c_int, _f64p]
    lib.oracle_log_decay.restype = None
    lib.oracle_ssd_quadratic.argtypes = [_f32p, _f32p, _f32p, _f32p, _f32p, _f32p, _f32p,
                                         _f32p, ctypes.c_int, _f64p, _f64p,
                                         ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                         ctypes.c_int, ctypes.c_int, _i32p, ctypes.c_int,
                                         _f64p, _f64p]
    lib.oracle_ssd_quadratic.restype = ctypes.c_int
    lib.oracle_ssd_recurrent.argtypes = [_f32p, _f32p, _f32p, _f32p, _f32p, _f32p, _f32p,
                                         _f32p, ctypes.c_int, _f64p, _f64p,
                                         ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                         ctypes.c_int, ctypes.c_int, _f64p, _f64p, _f64p, _f64p]
    lib.oracle_ssd_recurrent.restype = ctypes.c_int
    lib.oracle_silu.argtypes = [ctypes.c_double]
    lib.oracle_silu.restype = ctypes.c_double
    lib.oracle_conv1d.argtypes = [_f32p, _f32p, _f32p] + [ctypes.c_int] * 6 + [_f64p]
    lib.oracle_conv1d.restype = ctypes.c_int
    lib.oracle_num_threads.argtypes = []
    lib.oracle_num_threads.restype = ctypes.c_int
    _lib = lib
    return lib


def _f32(a) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(a, dtype=np.float32))


def _ptr(a: Optional[np.ndarray], typ):
    if a is None:
        return ctypes.cast(None, typ)
    return a.ctypes.data_as(typ)


def num_threads() -> int:
    """OpenMP threads the oracle uses (OMP_NUM_THREADS, else all cores)."""
    return int(_load().oracle_num_threads())


def softplus(x: float) -> float:
    """softplus(x) = log(1 + e^x) (Algorithm 3, the dt line)."""
    return float(_load().oracle_softplus(float(x)))


def mask(acs_row: np.ndarray, i: int, j: int) -> float:
    """A^M_ij * M_ij = exp(A^CS_i - A^CS_j) for i >= j, else 0 (Algorithm 4)."""
    a = np.ascontiguousarray(acs_row, dtype=np.float64)
    return float(_load().oracle_mask(_ptr(a, _f64p), int(i), int(j)))


def feature(x: np.ndarray, order: int) -> np.ndarray:
    """phi(x): x for order 1, x (x) x (index a*d+b) for order 2 (Algorithm 6)."""
    xd = np.ascontiguousarray(x, dtype=np.float64)
    d = xd.shape[0]
    out = np.zeros(d ** order, dtype=np.float64)
    _load().oracle_feature(_ptr(xd, _f64p), d, int(order), _ptr(out, _f64p))
    return out


def log_decay(dt_p, A_log, dt_bias, log_decay_in=None) -> np.ndarray:
    """A^CS = cumsum(-exp(A_log) * softplus(dt_p + dt_bias)) per (b, h), inclusive
    (Algorithm 3, last line), or cumsum(log_decay_in) when that [B, H, N] array
    is given (Algorithm 4).  Returns float64 [B, H, N]."""
    ld = None if log_decay_in is None else _f32(log_decay_in)
    dt_p = None if dt_p is None else _f32(dt_p)
    B, H, N = (ld if ld is not None else dt_p).shape
    A_log = None if A_log is None else _f32(A_log)
    dt_bias = None if dt_bias is None else _f32(dt_bias)
    out = np.zeros((B, H, N), dtype=np.float64)
    _load().oracle_log_decay(_ptr(dt_p, _f32p), _ptr(A_log, _f32p), _ptr(dt_bias, _f32p),
                             _ptr(ld, _f32p), B, H, N, _ptr(out, _f64p))
    return out


def _opt(a):
    return None if a is None else _f32(a)


def _f64(a):
    return None if a is None else np.ascontiguousarray(np.asarray(a, dtype=np.float64))


def _check_state(h0, z0, B, H, d, order):
    Dphi = d ** order
    if h0 is not None and h0.shape != (B, H, Dphi, d):
        raise ValueError(f"h0 must be [B, H, d^order, d] = {(B, H, Dphi, d)}")
    if z0 is not None and z0.shape != (B, H, Dphi):
        raise ValueError(f"z0 must be [B, H, d^order] = {(B, H, Dphi)}")


def ssd_quadratic(q, k, v, dt_p, A_log, dt_bias, D, order: int, normalize: bool,
                  rows: Optional[Sequence[int]] = None, return_norm: bool = False,
                  log_decay=None, value_dt: bool = False, h0=None, z0=None):
    """Masked-matrix form of the operator (Algorithms 1 and 5), in float64.

    ``log_decay`` ([B, H, N], optional) replaces A dt by a given per-token
    log-decay (Algorithm 4); ``value_dt`` contracts with V (.) dt instead of V
    (Algorithm 4, V_dt).  ``h0`` [B, H, d^order, d] and ``z0`` [B, H, d^order]
    are the states carried into token 0 (zero when None).  Returns y as
    [B, H, len(rows) or N, d] (and the row sums N_i when ``return_norm``)."""
    q, k, v = _f32(q), _f32(k), _f32(v)
    dt_p, A_log, dt_bias, ld = _opt(dt_p), _opt(A_log), _opt(dt_bias), _opt(log_decay)
    h0d, z0d = _f64(h0), _f64(z0)
    Dv = None if D is None else _f32(D)
    B, H, N, d = q.shape
    _check_state(h0d, z0d, B, H, d, order)
    if rows is None:
        r_arr = None
        n_rows = N
    else:
        r_arr = np.ascontiguousarray(np.asarray(rows, dtype=np.int32))
        n_rows = int(r_arr.shape[0])
    out = np.zeros((B, H, n_rows, d), dtype=np.float64)
    norm = np.zeros((B, H, n_rows), dtype=np.float64)
    rc = _load().oracle_ssd_quadratic(
        _ptr(q, _f32p), _ptr(k, _f32p), _ptr(v, _f32p), _ptr(dt_p, _f32p),
        _ptr(A_log, _f32p), _ptr(dt_bias, _f32p), _ptr(Dv, _f32p), _ptr(ld, _f32p),
        int(bool(value_dt)), _ptr(h0d, _f64p), _ptr(z0d, _f64p),
        B, H, N, d, int(order), int(bool(normalize)),
        _ptr(r_arr, _i32p), n_rows, _ptr(out, _f64p), _ptr(norm, _f64p))
    if rc != 0:
        raise ValueError("oracle_ssd_quadratic rejected its arguments")
    return (out, norm) if return_norm else out


def ssd_recurrent(q, k, v, dt_p, A_log, dt_bias, D, order: int, normalize: bool,
                  return_norm: bool = False, return_state: bool = False,
                  log_decay=None, value_dt: bool = False, h0=None, z0=None):
    """Token-by-token recurrent form (Algorithm 6), in float64.

    ``log_decay``, ``value_dt``, ``h0`` and ``z0`` as in ssd_quadratic.  Returns y
    [B, H, N, d]; optionally the row sums [B, H, N] and the final states
    H_up [B, H, d^order, d] and H_dn [B, H, d^order]."""
    q, k, v = _f32(q), _f32(k), _f32(v)
    dt_p, A_log, dt_bias, ld = _opt(dt_p), _opt(A_log), _opt(dt_bias), _opt(log_decay)
    h0d, z0d = _f64(h0), _f64(z0)
    Dv = None if D is None else _f32(D)
    B, H, N, d = q.shape
    _check_state(h0d, z0d, B, H, d, order)
    Dphi = d ** order
    out = np.zeros((B, H, N, d), dtype=np.float64)
    norm = np.zeros((B, H, N), dtype=np.float64)
    st = np.zeros((B, H, Dphi, d), dtype=np.float64) if return_state else None
    zst = np.zeros((B, H, Dphi), dtype=np.float64) if return_state else None
    rc = _load().oracle_ssd_recurrent(
        _ptr(q, _f32p), _ptr(k, _f32p), _ptr(v, _f32p), _ptr(dt_p, _f32p),
        _ptr(A_log, _f32p), _ptr(dt_bias, _f32p), _ptr(Dv, _f32p), _ptr(ld, _f32p),
        int(bool(value_dt)), _ptr(h0d, _f64p), _ptr(z0d, _f64p),
        B, H, N, d, int(order), int(bool(normalize)),
        _ptr(out, _f64p), _ptr(norm, _f64p), _ptr(st, _f64p), _ptr(zst, _f64p))
    if rc != 0:
        raise ValueError("oracle_ssd_recurrent rejected its arguments")
    res = [out]
    if return_norm:
        res.append(norm)
    if return_state:
        res.extend([st, zst])
    return res[0] if len(res) == 1 else tuple(res)


def silu(x: float) -> float:
    """SiLU(x) = x sigmoid(x) (Algorithm 3's sigma), in float64."""
    return float(_load().oracle_silu(float(x)))


def conv1d(x, w, bias=None, silu: bool = True) -> np.ndarray:
    """Causal depthwise convolution over tokens (+ SiLU), float64.

    x: [B, H, N, d]; w: [H*d, width], w[:, j] multiplies token t - j;
    bias: [H*d] or None.  Returns [B, H, N, d]."""
    x, w = _f32(x), _f32(w)
    bv = None if bias is None else _f32(bias)
    B, H, N, d = x.shape
    width = int(w.shape[1])
    if w.shape[0] != H * d:
        raise ValueError("w must be [H*d, width]")
    out = np.zeros((B, H, N, d), dtype=np.float64)
    rc = _load().oracle_conv1d(_ptr(x, _f32p), _ptr(w, _f32p), _ptr(bv, _f32p), B, H, N, d, width,
                               int(bool(silu)), _ptr(out, _f64p))
    if rc != 0:
        raise ValueError("oracle_conv1d rejected its arguments")
    return out
