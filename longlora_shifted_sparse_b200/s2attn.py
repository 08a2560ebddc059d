"""Thin ctypes binding of libs2attn.so (argument marshalling only; every step runs in the
library's CUDA kernels).

Two layers:
* the C ABI under its own names (``s2attn_fwd``, ``s2attn_bwd``, ...), taking raw device
  pointers and sizes exactly like ``include/s2attn.h``;
* torch conveniences (``forward``, ``backward``, ``S2AttnFunction``) that allocate outputs
  and the workspace with torch and pass their pointers and the current CUDA stream.

Importing this module raises ImportError when the library has not been built: there is no
fallback implementation.
"""
from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libs2attn.so")

S2_OK, S2_ERR_NULL, S2_ERR_SHAPE, S2_ERR_DTYPE, S2_ERR_HEADDIM, S2_ERR_ALIGN, \
    S2_ERR_WORKSPACE, S2_ERR_CUDA, S2_ERR_DEVICE_TIMEOUT, S2_ERR_ARG, \
    S2_ERR_STALE_WORKSPACE = range(11)
S2_BF16, S2_FP32 = 0, 1
S2_CAUSAL, S2_SHIFT_HALF, S2_SHIFT_ALTERNATE, S2_SHIFT_NONE = 0x01, 0x00, 0x10, 0x20
S2_INJECT_FWD, S2_INJECT_DKDV = 1, 2
SHIFT_PATTERNS = {"half": S2_SHIFT_HALF, "alternate": S2_SHIFT_ALTERNATE, "none": S2_SHIFT_NONE}
NOALLOC_SCRATCH_BYTES = 32 * 1024 * 1024  # S2ATTN_NOALLOC_SCRATCH_BYTES

if not os.path.exists(LIB_PATH):
    raise ImportError(
        "libs2attn.so is not built (expected at %s); build it with "
        "`python -m longlora_shifted_sparse_b200.build`" % LIB_PATH)

_lib = ctypes.CDLL(LIB_PATH)

_vp, _i, _f, _sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
_SHAPE = [_i] * 7 + [_f, _f, _i]

_lib.s2attn_workspace_bytes.argtypes = [_i] * 6
_lib.s2attn_workspace_bytes.restype = _sz
_lib.s2attn_fwd.argtypes = [_vp] * 5 + _SHAPE + [_vp, _sz, _vp]
_lib.s2attn_fwd.restype = _i
_lib.s2attn_bwd.argtypes = [_vp] * 9 + _SHAPE + [_vp, _sz, _vp]
_lib.s2attn_bwd.restype = _i
_lib.s2attn_bwd_after_fwd.argtypes = [_vp] * 9 + _SHAPE + [_vp, _sz, _vp]
_lib.s2attn_bwd_after_fwd.restype = _i
_lib.s2attn_fwd_noalloc.argtypes = [_vp] * 5 + _SHAPE + [_vp]
_lib.s2attn_fwd_noalloc.restype = _i
_lib.s2attn_noalloc_device_status.argtypes = [_vp]
_lib.s2attn_noalloc_device_status.restype = _i
_lib.s2attn_kernel_path.argtypes = [_i] * 8
_lib.s2attn_kernel_path.restype = _i
_lib.s2attn_selftest_wait_timeout.argtypes = [_vp, _sz, _vp]
_lib.s2attn_selftest_wait_timeout.restype = _i
_lib.s2attn_selftest_inject.argtypes = [_i] + [_vp] * 9 + _SHAPE + [_vp, _sz, _vp]
_lib.s2attn_selftest_inject.restype = _i
_lib.s2attn_selftest_exp2.argtypes = [_vp, _vp, _i, _vp]
_lib.s2attn_selftest_exp2.restype = _i
_lib.s2attn_device_status.argtypes = [_vp, _sz, _vp]
_lib.s2attn_device_status.restype = _i
_lib.s2attn_status_string.argtypes = [_i]
_lib.s2attn_status_string.restype = ctypes.c_char_p
_lib.s2attn_profile_enable.argtypes = [_i]
_lib.s2attn_profile_enable.restype = _i
_lib.s2attn_profile_num_kernels.argtypes = []
_lib.s2attn_profile_num_kernels.restype = _i
_lib.s2attn_profile_query.argtypes = [_i, ctypes.POINTER(ctypes.c_char_p),
                                      ctypes.POINTER(_i), ctypes.POINTER(ctypes.c_double)]
_lib.s2attn_profile_query.restype = _i
_lib.s2attn_profile_dropped.argtypes = []
_lib.s2attn_profile_dropped.restype = _i

# C ABI, same names and argument order as include/s2attn.h
s2attn_workspace_bytes = _lib.s2attn_workspace_bytes
s2attn_fwd = _lib.s2attn_fwd
s2attn_bwd = _lib.s2attn_bwd
s2attn_bwd_after_fwd = _lib.s2attn_bwd_after_fwd
s2attn_fwd_noalloc = _lib.s2attn_fwd_noalloc
s2attn_noalloc_device_status = _lib.s2attn_noalloc_device_status
s2attn_kernel_path = _lib.s2attn_kernel_path
s2attn_device_status = _lib.s2attn_device_status
s2attn_selftest_wait_timeout = _lib.s2attn_selftest_wait_timeout
s2attn_selftest_inject = _lib.s2attn_selftest_inject
s2attn_selftest_exp2 = _lib.s2attn_selftest_exp2
s2attn_profile_enable = _lib.s2attn_profile_enable
s2attn_profile_num_kernels = _lib.s2attn_profile_num_kernels
s2attn_profile_dropped = _lib.s2attn_profile_dropped


def s2attn_status_string(status: int) -> str:
    return _lib.s2attn_status_string(int(status)).decode()


def s2attn_profile_query(kernel_id: int):
    """(name, launches, total_ms) of one kernel id."""
    name = ctypes.c_char_p()
    n = _i()
    ms = ctypes.c_double()
    rc = _lib.s2attn_profile_query(kernel_id, ctypes.byref(name), ctypes.byref(n),
                                   ctypes.byref(ms))
    check(rc)
    return name.value.decode(), n.value, ms.value


def profile_summary():
    """{kernel name: (launches, total_ms)} for every kernel that launched."""
    out = {}
    for i in range(s2attn_profile_num_kernels()):
        name, n, ms = s2attn_profile_query(i)
        if n:
            out[name] = (n, ms)
    return out


class S2Error(RuntimeError):
    def __init__(self, status: int):
        super().__init__("s2attn: %s (status %d)" % (s2attn_status_string(status), status))
        self.status = status


def check(status: int) -> None:
    if status != S2_OK:
        raise S2Error(status)


# ----------------------------------------------------------------------------- torch layer

def _dtype_code(t) -> int:
    import torch
    if t.dtype == torch.bfloat16:
        return S2_BF16
    if t.dtype == torch.float32:
        return S2_FP32
    raise TypeError("s2attn supports bfloat16 and float32 tensors, got %s" % t.dtype)


def _stream_ptr(device) -> int:
    import torch
    return torch.cuda.current_stream(device).cuda_stream


def mode(causal: bool = True, shift: str = "half") -> int:
    """The ABI's mode argument: the causal flag ORed with a shifted-head pattern."""
    if shift not in SHIFT_PATTERNS:
        raise ValueError("shift must be one of %s, got %r" % (sorted(SHIFT_PATTERNS), shift))
    return (S2_CAUSAL if causal else 0) | SHIFT_PATTERNS[shift]


def workspace(B, N, Hq, Hkv, d, dtype_code, device):
    import torch
    nbytes = s2attn_workspace_bytes(B, N, Hq, Hkv, d, dtype_code)
    if nbytes == 0:
        raise S2Error(S2_ERR_SHAPE)
    return torch.empty(nbytes, dtype=torch.uint8, device=device)


def forward(q, k, v, G: int, pi_scale: float, rope_base: float = 10000.0, causal: bool = True,
            ws=None, out=None, lse=None, shift: str = "half", check_status: bool = False):
    """q [B,N,Hq,d], k/v [B,N,Hkv,d] CUDA tensors -> (o, lse). shift picks the shifted
    heads: "half" (the method), "alternate" (odd kv heads) or "none".

    check_status=True waits for the stream after the launch and raises S2Error if a bounded
    wait in a kernel expired (the outputs are then undefined)."""
    import torch
    B, N, Hq, d = q.shape
    Hkv = k.shape[2]
    dt = _dtype_code(q)
    if ws is None:
        ws = workspace(B, N, Hq, Hkv, d, dt, q.device)
    o = out if out is not None else torch.empty_like(q)
    lse = lse if lse is not None else torch.empty((B, Hq, N), dtype=torch.float32, device=q.device)
    check(s2attn_fwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(),
                     B, N, Hq, Hkv, d, G, mode(causal, shift), pi_scale, rope_base, dt,
                     ws.data_ptr(), ws.numel(), _stream_ptr(q.device)))
    if check_status:
        check(device_status(ws))
    return o, lse


def backward(q, k, v, o, lse, dout, G: int, pi_scale: float, rope_base: float = 10000.0,
             causal: bool = True, ws=None, grads=None, after_forward: bool = False,
             shift: str = "half", check_status: bool = False):
    """Returns (dq, dk, dv) for the forward that produced (o, lse).

    after_forward=True calls s2attn_bwd_after_fwd: `ws` must then be the workspace the
    forward of these q, k used, unchanged since (it holds their rotation).
    check_status=True waits for the stream after the launch and raises S2Error if a bounded
    wait in a kernel expired (the gradients are then undefined)."""
    import torch
    B, N, Hq, d = q.shape
    Hkv = k.shape[2]
    dt = _dtype_code(q)
    if ws is None:
        if after_forward:
            raise ValueError("after_forward=True needs the forward's workspace")
        ws = workspace(B, N, Hq, Hkv, d, dt, q.device)
    if grads is None:
        grads = (torch.empty_like(q), torch.empty_like(k), torch.empty_like(v))
    dq, dk, dv = grads
    fn = s2attn_bwd_after_fwd if after_forward else s2attn_bwd
    check(fn(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(),
                     dout.data_ptr(), dq.data_ptr(), dk.data_ptr(), dv.data_ptr(),
                     B, N, Hq, Hkv, d, G, mode(causal, shift), pi_scale, rope_base, dt,
                     ws.data_ptr(), ws.numel(), _stream_ptr(q.device)))
    if check_status:
        check(device_status(ws))
    return dq, dk, dv


def device_status(ws) -> int:
    """Waits for the current stream, then reads and clears the status word of `ws`."""
    return s2attn_device_status(ws.data_ptr(), ws.numel(), _stream_ptr(ws.device))


def noalloc_device_status(device=None) -> int:
    """Status of the last s2attn_fwd_noalloc on `device` (waits for its current stream)."""
    import torch
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else device
    with torch.cuda.device(dev):
        return s2attn_noalloc_device_status(_stream_ptr(dev))


def _make_function():
    import torch

    class S2AttnFunction(torch.autograd.Function):
        """Autograd wrapper: o = S2Attn(q, k, v); backward through the library's kernels."""

        @staticmethod
        def forward(ctx, q, k, v, G, pi_scale, rope_base=10000.0, causal=True, shift="half"):
            q, k, v = q.contiguous(), k.contiguous(), v.contiguous()
            B, N, Hq, d = q.shape
            ws = workspace(B, N, Hq, k.shape[2], d, _dtype_code(q), q.device)
            o, lse = forward(q, k, v, G, pi_scale, rope_base, causal, ws=ws, shift=shift)
            # the workspace keeps the rotated q, k for the backward (q, k are saved too, so
            # autograd's version check catches an in-place change in between)
            ctx.save_for_backward(q, k, v, o, lse, ws)
            ctx.args = (G, pi_scale, rope_base, causal, shift)
            return o

        @staticmethod
        def backward(ctx, do):
            q, k, v, o, lse, ws = ctx.saved_tensors
            G, pi_scale, rope_base, causal, shift = ctx.args
            # The backward's first kernel resets the workspace's status word, so a bounded
            # wait that expired in the forward is read here, before it would be lost, and the
            # backward's own status right after it (the workspace is dropped afterwards):
            # two stream synchronisations per backward.
            check(device_status(ws))
            dq, dk, dv = backward(q, k, v, o, lse, do.contiguous(), G, pi_scale, rope_base, causal,
                                  ws=ws, after_forward=True, shift=shift, check_status=True)
            return dq, dk, dv, None, None, None, None, None

    return S2AttnFunction


_fn = None


def s2_attention(q, k, v, G: int, pi_scale: float, rope_base: float = 10000.0,
                 causal: bool = True, shift: str = "half"):
    """Differentiable S2-Attn on CUDA tensors."""
    global _fn
    if _fn is None:
        _fn = _make_function()
    return _fn.apply(q, k, v, G, pi_scale, rope_base, causal, shift)
