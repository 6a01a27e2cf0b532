"""ctypes wrapper of the fp64 C oracle (``streamkl_oracle.c``).

TEST INFRASTRUCTURE ONLY (see the package docstring).  Arrays are numpy float64, dense
row-major: Q [B,Hq,NQ,d], K [B,Hkv,NK,d], per-row values [B,Hq,NQ].
"""
import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "streamkl_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lib = None
_lock = threading.Lock()

_D = ctypes.POINTER(ctypes.c_double)
_I64 = ctypes.POINTER(ctypes.c_int64)
_i = ctypes.c_int
_d = ctypes.c_double


def build(force=False):
    """Compile the oracle with gcc (-O2, OpenMP) into oracle/liboracle.so."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + ".tmp.%d" % os.getpid()
        subprocess.check_call(
            ["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11", "-o", tmp, _SRC, "-lm"]
        )
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    with _lock:
        if _lib is None:
            lib = ctypes.CDLL(build())
            shape = [_i, _i, _i, _i, _i, _i, _d, _i]
            lib.oracle_fwd.argtypes = [_D, _D, _D, _D] + shape + [_D, _D, _D]
            lib.oracle_fwd_rows.argtypes = [_D, _D, _D, _D] + shape + [_I64, ctypes.c_int64, _D, _D, _D]
            lib.oracle_fwd_streaming.argtypes = [_D, _D, _D, _D] + shape + [_i, _D, _D, _D]
            lib.oracle_bwd.argtypes = [_i, _D, _D, _D, _D, _D] + shape + [_D, _D]
            lib.oracle_bwd_dq_rows.argtypes = [_i, _D, _D, _D, _D, _D] + shape + [_I64, ctypes.c_int64, _D]
            lib.oracle_bwd_dk_keys.argtypes = [_i, _D, _D, _D, _D, _D] + shape + [_I64, ctypes.c_int64, _D]
            lib.oracle_bwd_dk_keys_stats.argtypes = ([_i, _D, _D, _D, _D, _D, _D, _D, _D] + shape +
                                                     [_I64, ctypes.c_int64, _D])
            for f in ("oracle_fwd", "oracle_fwd_rows", "oracle_fwd_streaming", "oracle_bwd",
                      "oracle_bwd_dq_rows", "oracle_bwd_dk_keys", "oracle_bwd_dk_keys_stats",
                      "oracle_num_threads"):
                getattr(lib, f).restype = _i
            lib.oracle_set_num_threads.argtypes = [_i]
            lib.oracle_set_num_threads.restype = None
            _lib = lib
    return _lib


def num_threads():
    return _load().oracle_num_threads()


def set_num_threads(n):
    _load().oracle_set_num_threads(int(n))


def _f64(a):
    a = np.ascontiguousarray(a, dtype=np.float64)
    return a, a.ctypes.data_as(_D)


def _shape(q1, k1, q2, k2):
    B, Hq, NQ, d = q1.shape
    Bk, Hkv, NK, dk = k1.shape
    if q2.shape != q1.shape or k2.shape != k1.shape or Bk != B or dk != d:
        raise ValueError("inconsistent shapes")
    return B, Hq, Hkv, NQ, NK, d


def _check(rc, name):
    if rc != 0:
        raise ValueError("%s failed with code %d" % (name, rc))


def _default_scale(d, scale):
    return 1.0 / np.sqrt(d) if scale is None else float(scale)


def fwd(q1, k1, q2, k2, scale=None, causal=False):
    """Per-row KL(P1||P2), LSE1, LSE2 of every row; each [B,Hq,NQ] float64."""
    lib = _load()
    B, Hq, Hkv, NQ, NK, d = _shape(q1, k1, q2, k2)
    arrs = [_f64(x) for x in (q1, k1, q2, k2)]
    out = [np.empty((B, Hq, NQ)) for _ in range(3)]
    rc = lib.oracle_fwd(*[p for _, p in arrs], B, Hq, Hkv, NQ, NK, d, _default_scale(d, scale),
                        int(bool(causal)), *[o.ctypes.data_as(_D) for o in out])
    _check(rc, "oracle_fwd")
    return tuple(out)


def fwd_rows(q1, k1, q2, k2, rows, scale=None, causal=False):
    """KL, LSE1, LSE2 for flat row indices ``rows`` into [B*Hq*NQ]; each [len(rows)]."""
    lib = _load()
    B, Hq, Hkv, NQ, NK, d = _shape(q1, k1, q2, k2)
    arrs = [_f64(x) for x in (q1, k1, q2, k2)]
    rows = np.ascontiguousarray(rows, dtype=np.int64)
    out = [np.empty(rows.shape[0]) for _ in range(3)]
    rc = lib.oracle_fwd_rows(*[p for _, p in arrs], B, Hq, Hkv, NQ, NK, d, _default_scale(d, scale),
                             int(bool(causal)), rows.ctypes.data_as(_I64), rows.shape[0],
                             *[o.ctypes.data_as(_D) for o in out])
    _check(rc, "oracle_fwd_rows")
    return tuple(out)


def fwd_streaming(q1, k1, q2, k2, scale=None, causal=False, tile=64):
    """The five-scalar online recurrence run in fp64 with key tiles of ``tile`` keys."""
    lib = _load()
    B, Hq, Hkv, NQ, NK, d = _shape(q1, k1, q2, k2)
    arrs = [_f64(x) for x in (q1, k1, q2, k2)]
    out = [np.empty((B, Hq, NQ)) for _ in range(3)]
    rc = lib.oracle_fwd_streaming(*[p for _, p in arrs], B, Hq, Hkv, NQ, NK, d,
                                  _default_scale(d, scale), int(bool(causal)), int(tile),
                                  *[o.ctypes.data_as(_D) for o in out])
    _check(rc, "oracle_fwd_streaming")
    return tuple(out)


def bwd(mode, q1, k1, q2, k2, dkl, scale=None, causal=False):
    """Gradients of sum g*KL.  mode 1 -> (dQ2, dK2); mode 2 -> (dQ1, dK1)."""
    lib = _load()
    B, Hq, Hkv, NQ, NK, d = _shape(q1, k1, q2, k2)
    arrs = [_f64(x) for x in (q1, k1, q2, k2)]
    g, gp = _f64(dkl)
    if g.shape != (B, Hq, NQ):
        raise ValueError("dkl must be [B,Hq,NQ]")
    dq = np.empty((B, Hq, NQ, d))
    dk = np.empty((B, Hkv, NK, d))
    rc = lib.oracle_bwd(int(mode), *[p for _, p in arrs], gp, B, Hq, Hkv, NQ, NK, d,
                        _default_scale(d, scale), int(bool(causal)), dq.ctypes.data_as(_D),
                        dk.ctypes.data_as(_D))
    _check(rc, "oracle_bwd")
    return dq, dk


def bwd_dq_rows(mode, q1, k1, q2, k2, dkl, rows, scale=None, causal=False):
    """dQ of the free distribution for flat rows ``rows``: [len(rows), d]."""
    lib = _load()
    B, Hq, Hkv, NQ, NK, d = _shape(q1, k1, q2, k2)
    arrs = [_f64(x) for x in (q1, k1, q2, k2)]
    g, gp = _f64(dkl)
    rows = np.ascontiguousarray(rows, dtype=np.int64)
    out = np.empty((rows.shape[0], d))
    rc = lib.oracle_bwd_dq_rows(int(mode), *[p for _, p in arrs], gp, B, Hq, Hkv, NQ, NK, d,
                                _default_scale(d, scale), int(bool(causal)),
                                rows.ctypes.data_as(_I64), rows.shape[0], out.ctypes.data_as(_D))
    _check(rc, "oracle_bwd_dq_rows")
    return out


def bwd_dk_keys(mode, q1, k1, q2, k2, dkl, keys, scale=None, causal=False):
    """dK of the free distribution for flat key indices ``keys`` into [B*Hkv*NK]: [len, d]."""
    lib = _load()
    B, Hq, Hkv, NQ, NK, d = _shape(q1, k1, q2, k2)
    arrs = [_f64(x) for x in (q1, k1, q2, k2)]
    g, gp = _f64(dkl)
    keys = np.ascontiguousarray(keys, dtype=np.int64)
    out = np.empty((keys.shape[0], d))
    rc = lib.oracle_bwd_dk_keys(int(mode), *[p for _, p in arrs], gp, B, Hq, Hkv, NQ, NK, d,
                                _default_scale(d, scale), int(bool(causal)),
                                keys.ctypes.data_as(_I64), keys.shape[0], out.ctypes.data_as(_D))
    _check(rc, "oracle_bwd_dk_keys")
    return out


def bwd_dk_keys_stats(mode, q1, k1, q2, k2, dkl, kl, lse1, lse2, keys, scale=None, causal=False):
    """dK for flat key indices with every row's (KL, LSE1, LSE2) given as inputs
    ([B,Hq,NQ] each) rather than recomputed: for sizes where the full statistics are out of
    reach.  Only as independent as the statistics passed in."""
    lib = _load()
    B, Hq, Hkv, NQ, NK, d = _shape(q1, k1, q2, k2)
    arrs = [_f64(x) for x in (q1, k1, q2, k2)]
    st = [_f64(x) for x in (dkl, kl, lse1, lse2)]
    for a, _ in st:
        if a.shape != (B, Hq, NQ):
            raise ValueError("row statistics must be [B,Hq,NQ]")
    keys = np.ascontiguousarray(keys, dtype=np.int64)
    out = np.empty((keys.shape[0], d))
    rc = lib.oracle_bwd_dk_keys_stats(int(mode), *[p for _, p in arrs], *[p for _, p in st], B, Hq,
                                      Hkv, NQ, NK, d, _default_scale(d, scale), int(bool(causal)),
                                      keys.ctypes.data_as(_I64), keys.shape[0], out.ctypes.data_as(_D))
    _check(rc, "oracle_bwd_dk_keys_stats")
    return out
