"""fp64 CPU oracle for S2-Attn (ctypes wrapper around ``s2attn_oracle.c``).

TEST INFRASTRUCTURE ONLY: the tests, the smoke check and the bench's CPU-baseline leg use
this package. The product path never imports it and shares no code with it.

Arrays follow the library's layouts: q/o/dO/dq [B,N,Hq,d], k/v/dk/dv [B,N,Hkv,d],
lse [B,Hq,N]. Inputs may be numpy uint16 (bf16 bit patterns), float32 or float64.
Unit functions return outputs in rolled local-row order for one (b, kv head, group).
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "s2attn_oracle.c")
_BUILD = os.path.join(_HERE, "_build")
_LIB = os.path.join(_BUILD, "libs2oracle.so")

IN_BF16, IN_F32, IN_F64 = 0, 1, 2

_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (plain -O2, no fast-math, OpenMP)."""
    os.makedirs(_BUILD, exist_ok=True)
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + ".tmp.%d" % os.getpid()
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp",
                               "-fno-fast-math", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        vp, i, d, dp = ctypes.c_void_p, ctypes.c_int, ctypes.c_double, ctypes.c_void_p
        lib.s2o_check.argtypes = [i] * 6
        lib.s2o_fwd_unit.argtypes = [vp, vp, vp, i] + [i] * 7 + [d, d] + [i, i, i] + [dp, dp]
        lib.s2o_bwd_unit.argtypes = [vp, vp, vp, vp, i] + [i] * 7 + [d, d] + [i, i, i] + [dp, dp, dp]
        lib.s2o_fwd.argtypes = [vp, vp, vp, i] + [i] * 7 + [d, d] + [dp, dp]
        lib.s2o_bwd.argtypes = [vp, vp, vp, vp, i] + [i] * 7 + [d, d] + [dp, dp, dp]
        lib.s2o_fwd_rows.argtypes = [vp, vp, vp, i] + [i] * 7 + [d, d] + [i, i, i] + \
            [i, vp, dp, dp]
        lib.s2o_bwd_rows.argtypes = [vp, vp, vp, vp, i] + [i] * 7 + [d, d] + [i, i, i] + \
            [i, vp, i, vp, dp, dp, dp]
        lib.s2o_rope.argtypes = [dp, dp, i, vp, i, d, d, i]
        lib.s2o_rope.restype = None
        lib.s2o_max_threads.restype = i
        lib.s2o_set_threads.argtypes = [i]
        lib.s2o_set_threads.restype = None
        _lib = lib
    return _lib


def _in(x: np.ndarray):
    x = np.ascontiguousarray(x)
    if x.dtype == np.uint16:
        return x, IN_BF16
    if x.dtype == np.float32:
        return x, IN_F32
    if x.dtype == np.float64:
        return x, IN_F64
    raise TypeError("oracle inputs must be uint16 (bf16 bits), float32 or float64")


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def max_threads() -> int:
    return _load().s2o_max_threads()


def set_threads(n: int) -> None:
    _load().s2o_set_threads(int(n))


def check(B, N, Hq, Hkv, d, G) -> bool:
    return _load().s2o_check(B, N, Hq, Hkv, d, G) == 0


def rope(x: np.ndarray, pos, s: float, base: float = 10000.0, inverse: bool = False) -> np.ndarray:
    """Rotate rows x [n, d] (fp64) at integer positions pos[n]."""
    x = np.ascontiguousarray(x, dtype=np.float64)
    n, d = x.shape
    pos = np.ascontiguousarray(np.asarray(pos, dtype=np.int64).reshape(n))
    y = np.empty_like(x)
    _load().s2o_rope(_ptr(x), _ptr(y), n, _ptr(pos), d, float(s), float(base), int(inverse))
    return y


# Shift patterns (which heads see the sequence rolled by -G/2); see shifted_head in
# s2attn_oracle.c: "half" = the second half of the heads, "alternate" = odd kv heads,
# "none" = no head.
SHIFT_PATTERNS = {"half": 0, "alternate": 1, "none": 2}


def _mode(causal, shift) -> int:
    return int(bool(causal)) | (SHIFT_PATTERNS[shift] << 4)


def head_is_shifted(h: int, Hq: int, Hkv: int, shift: str = "half") -> bool:
    """Whether query head h sees the rolled sequence under the given pattern."""
    R = Hq // Hkv
    if shift == "alternate":
        return (h // R) % 2 == 1
    if shift == "none":
        return False
    return h >= Hq // 2


def _dims(q, k):
    B, N, Hq, d = q.shape
    Hkv = k.shape[2]
    return B, N, Hq, Hkv, d


def fwd(q, k, v, G: int, s: float, base: float = 10000.0, causal: bool = True,
        shift: str = "half"):
    """Full forward. Returns (o [B,N,Hq,d] fp64, lse [B,Hq,N] fp64)."""
    (q, dt), (k, _), (v, _) = _in(q), _in(k), _in(v)
    B, N, Hq, Hkv, d = _dims(q, k)
    o = np.empty((B, N, Hq, d), dtype=np.float64)
    lse = np.empty((B, Hq, N), dtype=np.float64)
    rc = _load().s2o_fwd(_ptr(q), _ptr(k), _ptr(v), dt, B, N, Hq, Hkv, d, G,
                         _mode(causal, shift),
                         float(s), float(base), _ptr(o), _ptr(lse))
    if rc:
        raise ValueError("oracle fwd rejected the shape (rc=%d)" % rc)
    return o, lse


def bwd(q, k, v, dout, G: int, s: float, base: float = 10000.0, causal: bool = True,
        shift: str = "half"):
    """Full backward. Returns (dq, dk, dv) fp64 in the input layouts."""
    (q, dt), (k, _), (v, _), (dout, _) = _in(q), _in(k), _in(v), _in(dout)
    B, N, Hq, Hkv, d = _dims(q, k)
    dq = np.empty((B, N, Hq, d), dtype=np.float64)
    dk = np.empty((B, N, Hkv, d), dtype=np.float64)
    dv = np.empty((B, N, Hkv, d), dtype=np.float64)
    rc = _load().s2o_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(dout), dt, B, N, Hq, Hkv, d, G,
                         _mode(causal, shift), float(s), float(base), _ptr(dq), _ptr(dk),
                         _ptr(dv))
    if rc:
        raise ValueError("oracle bwd rejected the shape (rc=%d)" % rc)
    return dq, dk, dv


def fwd_unit(q, k, v, G: int, s: float, b: int, kvh: int, g: int, base: float = 10000.0,
             causal: bool = True, shift: str = "half"):
    """One unit's forward: (o_u [R,G,d], lse_u [R,G]) in rolled local-row order."""
    (q, dt), (k, _), (v, _) = _in(q), _in(k), _in(v)
    B, N, Hq, Hkv, d = _dims(q, k)
    R = Hq // Hkv
    o_u = np.empty((R, G, d), dtype=np.float64)
    lse_u = np.empty((R, G), dtype=np.float64)
    rc = _load().s2o_fwd_unit(_ptr(q), _ptr(k), _ptr(v), dt, B, N, Hq, Hkv, d, G,
                              _mode(causal, shift),
                              float(s), float(base), b, kvh, g, _ptr(o_u), _ptr(lse_u))
    if rc:
        raise ValueError("oracle fwd_unit rejected the arguments (rc=%d)" % rc)
    return o_u, lse_u


def bwd_unit(q, k, v, dout, G: int, s: float, b: int, kvh: int, g: int, base: float = 10000.0,
             causal: bool = True, shift: str = "half"):
    """One unit's backward: (dq_u [R,G,d], dk_u [G,d], dv_u [G,d]) in rolled local-row order."""
    (q, dt), (k, _), (v, _), (dout, _) = _in(q), _in(k), _in(v), _in(dout)
    B, N, Hq, Hkv, d = _dims(q, k)
    R = Hq // Hkv
    dq_u = np.empty((R, G, d), dtype=np.float64)
    dk_u = np.empty((G, d), dtype=np.float64)
    dv_u = np.empty((G, d), dtype=np.float64)
    rc = _load().s2o_bwd_unit(_ptr(q), _ptr(k), _ptr(v), _ptr(dout), dt, B, N, Hq, Hkv, d, G,
                              _mode(causal, shift), float(s), float(base), b, kvh, g, _ptr(dq_u),
                              _ptr(dk_u), _ptr(dv_u))
    if rc:
        raise ValueError("oracle bwd_unit rejected the arguments (rc=%d)" % rc)
    return dq_u, dk_u, dv_u


def unit_rows(N: int, G: int, Hq: int, kvh: int, Hkv: int, g: int,
              shift: str = "half") -> np.ndarray:
    """Original token index of each rolled local row of unit (kvh, g)."""
    R = Hq // Hkv
    shifted = head_is_shifted(kvh * R, Hq, Hkv, shift)
    r = g * G + np.arange(G)
    return (r + G // 2) % N if shifted else r


def fwd_rows(q, k, v, G: int, s: float, b: int, h: int, g: int, rows, base: float = 10000.0,
             causal: bool = True, shift: str = "half"):
    """Forward at chosen rolled local rows of query head h, group g: (o [n,d], lse [n])."""
    (q, dt), (k, _), (v, _) = _in(q), _in(k), _in(v)
    B, N, Hq, Hkv, d = _dims(q, k)
    rows = np.ascontiguousarray(np.asarray(rows, dtype=np.int32))
    o = np.empty((rows.size, d), dtype=np.float64)
    lse = np.empty(rows.size, dtype=np.float64)
    rc = _load().s2o_fwd_rows(_ptr(q), _ptr(k), _ptr(v), dt, B, N, Hq, Hkv, d, G,
                              _mode(causal, shift),
                              float(s), float(base), b, h, g, rows.size, _ptr(rows), _ptr(o),
                              _ptr(lse))
    if rc:
        raise ValueError("oracle fwd_rows rejected the arguments (rc=%d)" % rc)
    return o, lse


def bwd_rows(q, k, v, dout, G: int, s: float, b: int, kvh: int, g: int, qrows, krows,
             base: float = 10000.0, causal: bool = True, shift: str = "half"):
    """Backward of unit (b, kvh, g) at chosen rolled local rows:
    (dq [nq,R,d] for the R query heads of kvh, dk [nk,d], dv [nk,d])."""
    (q, dt), (k, _), (v, _), (dout, _) = _in(q), _in(k), _in(v), _in(dout)
    B, N, Hq, Hkv, d = _dims(q, k)
    R = Hq // Hkv
    qrows = np.ascontiguousarray(np.asarray(qrows, dtype=np.int32))
    krows = np.ascontiguousarray(np.asarray(krows, dtype=np.int32))
    dq = np.empty((qrows.size, R, d), dtype=np.float64)
    dk = np.empty((krows.size, d), dtype=np.float64)
    dv = np.empty((krows.size, d), dtype=np.float64)
    rc = _load().s2o_bwd_rows(_ptr(q), _ptr(k), _ptr(v), _ptr(dout), dt, B, N, Hq, Hkv, d, G,
                              _mode(causal, shift), float(s), float(base), b, kvh, g, qrows.size,
                              _ptr(qrows), krows.size, _ptr(krows), _ptr(dq), _ptr(dk), _ptr(dv))
    if rc:
        raise ValueError("oracle bwd_rows rejected the arguments (rc=%d)" % rc)
    return dq, dk, dv
