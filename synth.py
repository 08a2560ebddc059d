"""Seeded synthetic inputs for S2-Attn, shared by the oracle tests and the CUDA path.

This module holds none of the attention arithmetic. It only draws numbers:

* a counter-based generator: the SplitMix64 output function (Steele, Lea and Flood,
  "Fast splittable pseudorandom number generators", OOPSLA 2014) applied to
  ``key + i * 0x9E3779B97F4A7C15``, which is exactly the i-th SplitMix64 output of a
  generator seeded with ``key``. Every element is addressable by its index, so any
  slice can be regenerated alone;
* uniforms in (0, 1) from the top 53 bits, and standard normals by the Box-Muller
  transform (Box and Muller, 1958), two normals per pair of uniforms;
* rounding fp32 -> bfloat16 with round-to-nearest-even on the bit pattern.

Inputs are drawn in fp64, cast to fp32, multiplied by the (power-of-two) scale in fp32,
then optionally rounded to bf16. The result is returned as host numpy arrays; callers
copy them to the device, so both sides see the same bits.
"""
from __future__ import annotations

import os
from concurrent.futures import ThreadPoolExecutor

import numpy as np

_GAMMA = np.uint64(0x9E3779B97F4A7C15)
_M1 = np.uint64(0xBF58476D1CE4E5B9)
_M2 = np.uint64(0x94D049BB133111EB)

# Stream ids: one independent stream per tensor of a workload.
STREAM_Q, STREAM_K, STREAM_V, STREAM_DO = 1, 2, 3, 4

_CHUNK = 1 << 20  # pairs per worker task


def _mix64(z: np.ndarray) -> np.ndarray:
    z = (z ^ (z >> np.uint64(30))) * _M1
    z = (z ^ (z >> np.uint64(27))) * _M2
    return z ^ (z >> np.uint64(31))


def stream_key(seed: int, stream: int) -> np.uint64:
    """Per-(seed, stream) key: one SplitMix64 output of the pair packed into 64 bits."""
    with np.errstate(over="ignore"):
        x = np.array([(seed & 0xFFFFFFFF) << 32 | (stream & 0xFFFFFFFF)], dtype=np.uint64)
        return _mix64(x + _GAMMA)[0]


def uint64_stream(key: np.uint64, start: int, count: int) -> np.ndarray:
    """Outputs ``start .. start+count-1`` of the SplitMix64 sequence seeded with ``key``."""
    idx = np.arange(start + 1, start + count + 1, dtype=np.uint64)
    with np.errstate(over="ignore"):
        return _mix64(key + idx * _GAMMA)


def _uniform(z: np.ndarray) -> np.ndarray:
    # (z >> 11) is in [0, 2^53); adding one half keeps u strictly inside (0, 1).
    return ((z >> np.uint64(11)).astype(np.float64) + 0.5) * (1.0 / 9007199254740992.0)


def _normal_pairs(key: np.uint64, pair_start: int, npairs: int) -> np.ndarray:
    z = uint64_stream(key, 2 * pair_start, 2 * npairs)
    u1 = _uniform(z[0::2])
    u2 = _uniform(z[1::2])
    r = np.sqrt(-2.0 * np.log(u1))
    t = 2.0 * np.pi * u2
    out = np.empty(2 * npairs, dtype=np.float64)
    out[0::2] = r * np.cos(t)
    out[1::2] = r * np.sin(t)
    return out


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round fp32 to bf16 (round to nearest, ties to even); returns uint16 bit patterns."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    bias = ((u >> np.uint32(16)) & np.uint32(1)) + np.uint32(0x7FFF)
    return ((u + bias) >> np.uint32(16)).astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def _workers() -> int:
    return max(1, min(32, os.cpu_count() or 1))


def normal(seed: int, stream: int, shape, scale: float = 1.0, dtype: str = "bf16",
           threads: int | None = None) -> np.ndarray:
    """iid N(0,1) * scale of ``shape``.

    dtype "bf16" returns uint16 bf16 bit patterns; "f32" returns float32. ``scale`` must be a
    power of two (it is applied in fp32 and must be exact).
    """
    n = int(np.prod(shape))
    m, e = np.frexp(scale)
    if m != 0.5:
        raise ValueError("scale must be a power of two")
    key = stream_key(seed, stream)
    npairs = (n + 1) // 2
    out_dt = np.uint16 if dtype == "bf16" else np.float32
    out = np.empty(2 * npairs, dtype=out_dt)

    def work(c0: int) -> None:
        c1 = min(npairs, c0 + _CHUNK)
        v = _normal_pairs(key, c0, c1 - c0).astype(np.float32) * np.float32(scale)
        if dtype == "bf16":
            out[2 * c0:2 * c1] = f32_to_bf16_bits(v)
        else:
            out[2 * c0:2 * c1] = v

    starts = list(range(0, npairs, _CHUNK))
    nt = threads or _workers()
    if nt == 1 or len(starts) == 1:
        for c in starts:
            work(c)
    else:
        with ThreadPoolExecutor(nt) as ex:
            list(ex.map(work, starts))
    return out[:n].reshape(shape)


def s2attn_inputs(seed: int, B: int, N: int, Hq: int, Hkv: int, d: int, scale: float,
                  dtype: str = "bf16", with_dout: bool = True, dout_scale: float = 1.0):
    """q [B,N,Hq,d], k,v [B,N,Hkv,d], dO [B,N,Hq,d] as host arrays (see ``normal``)."""
    q = normal(seed, STREAM_Q, (B, N, Hq, d), scale, dtype)
    k = normal(seed, STREAM_K, (B, N, Hkv, d), scale, dtype)
    v = normal(seed, STREAM_V, (B, N, Hkv, d), scale, dtype)
    do = normal(seed, STREAM_DO, (B, N, Hq, d), dout_scale, dtype) if with_dout else None
    return q, k, v, do
