"""Host-side checks of the C ABI: the library loads, exports what include/s2attn.h declares,
and rejects bad arguments with the documented codes before touching the GPU."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    from longlora_shifted_sparse_b200 import build
    build.build()
    from longlora_shifted_sparse_b200 import s2attn
    return s2attn


def _declared_symbols():
    names = []
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            text = open(os.path.join(ROOT, "include", fn)).read()
            names += re.findall(r"S2_API\s+[\w\s\*]+?\b(s2attn_\w+)\s*\(", text)
    return sorted(set(names))


def test_library_exports_every_declared_symbol(lib):
    names = _declared_symbols()
    assert "s2attn_fwd" in names and "s2attn_bwd" in names
    raw = ctypes.CDLL(lib.LIB_PATH)
    for n in names:
        assert hasattr(raw, n), n


def test_status_strings(lib):
    for code in range(11):
        assert lib.s2attn_status_string(code) and lib.s2attn_status_string(code) != "unknown status"
    assert lib.s2attn_status_string(99) == "unknown status"


def test_workspace_bytes(lib):
    B, N, Hq, Hkv, d = 1, 32768, 32, 32, 128
    ws = lib.s2attn_workspace_bytes(B, N, Hq, Hkv, d, lib.S2_BF16)
    # rotated q, k; (cos, sin) table; D; the row terms (16 bf16 per query row)
    need = 2 * (B * Hq * N * d + B * Hkv * N * d) + N * (d // 2) * 8 + B * Hq * N * 4 + \
        B * Hq * N * 32
    assert need <= ws <= need + 6 * 256
    assert lib.s2attn_workspace_bytes(B, N, Hq, Hkv, d, lib.S2_FP32) > ws
    assert lib.s2attn_workspace_bytes(B, N, 3, 3, d, lib.S2_BF16) == 0
    assert lib.s2attn_workspace_bytes(B, N, Hq, Hkv, 100, lib.S2_BF16) == 0
    assert lib.s2attn_workspace_bytes(B, N, Hq, Hkv, d, 7) == 0
    assert lib.s2attn_workspace_bytes(0, N, Hq, Hkv, d, lib.S2_BF16) == 0


def test_kernel_path_rule(lib):
    assert lib.s2attn_kernel_path(1, 256, 4, 4, 64, 64, 1, lib.S2_FP32) == 0
    assert lib.s2attn_kernel_path(1, 256, 4, 4, 64, 60, 1, lib.S2_FP32) == -1
    assert lib.s2attn_kernel_path(1, 256, 4, 4, 64, 64, 2, lib.S2_FP32) == -1
    assert lib.s2attn_kernel_path(1, 256, 4, 4, 64, 64, 1, 5) == -1
    # mode: S2_CAUSAL or 0, ORed with one S2_SHIFT_* pattern
    for m in (0x00, 0x01, 0x10, 0x11, 0x20, 0x21):
        assert lib.s2attn_kernel_path(1, 1024, 4, 4, 128, 256, m, lib.S2_BF16) == 1
    for m in (0x30, 0x31, 0x02, 0x40, 0x100, -1):
        assert lib.s2attn_kernel_path(1, 1024, 4, 4, 128, 256, m, lib.S2_BF16) == -1


def test_largest_shape_limits(lib):
    # B * N * H_q must stay below 2^31 (row indices are 32-bit): the largest accepted shape
    # is sized and checked, one token more is rejected before anything is enqueued
    N = (1 << 31) // 32 // 2 - 128      # B = 2, H_q = 32: 2^31 - 8192 rows, G | N
    assert lib.s2attn_kernel_path(2, N, 32, 32, 128, 128, 1, lib.S2_BF16) == 0
    assert lib.s2attn_workspace_bytes(2, N, 32, 32, 128, lib.S2_BF16) > 0
    big = 1 << 26                       # 2 * 2^26 * 32 = 2^32 rows
    assert lib.s2attn_kernel_path(2, big, 32, 32, 128, 1 << 13, 1, lib.S2_BF16) == -1
    assert _fwd(lib, B=2, N=big, Hq=32, Hkv=32, d=128, G=1 << 13, dt=lib.S2_BF16) == 2


def test_mode_flags_match_header(lib):
    text = open(os.path.join(ROOT, "include", "s2attn.h")).read()
    defs = dict(re.findall(r"#define\s+(S2_(?:CAUSAL|SHIFT_\w+))\s+(0x[0-9a-fA-F]+)", text))
    assert set(defs) == {"S2_CAUSAL", "S2_SHIFT_HALF", "S2_SHIFT_ALTERNATE", "S2_SHIFT_NONE"}
    for name, val in defs.items():
        assert getattr(lib, name) == int(val, 16), name


def test_mode_helper(lib):
    assert lib.mode(True) == 1 and lib.mode(False) == 0
    assert lib.mode(True, "alternate") == 0x11 and lib.mode(False, "none") == 0x20
    with pytest.raises(ValueError):
        lib.mode(True, "odd")


# fake but aligned, non-null device addresses: the calls below must fail in validation,
# before any CUDA call could use them
P = 1 << 20


def _fwd(lib, **kw):
    a = dict(q=P, k=P, v=P, o=P, lse=P, B=1, N=256, Hq=4, Hkv=4, d=64, G=64, causal=1,
             s=2.0, base=10000.0, dt=lib.S2_FP32, ws=P, wsb=1 << 40, st=None)
    a.update(kw)
    return lib.s2attn_fwd(a["q"], a["k"], a["v"], a["o"], a["lse"], a["B"], a["N"], a["Hq"],
                          a["Hkv"], a["d"], a["G"], a["causal"], a["s"], a["base"], a["dt"],
                          a["ws"], a["wsb"], a["st"])


def _bwd(lib, **kw):
    a = dict(B=1, N=256, Hq=4, Hkv=4, d=64, G=64, causal=1, s=2.0, base=10000.0,
             dt=lib.S2_FP32, ws=P, wsb=1 << 40, dq=P)
    a.update(kw)
    return lib.s2attn_bwd(P, P, P, P, P, P, a["dq"], P, P, a["B"], a["N"], a["Hq"], a["Hkv"],
                          a["d"], a["G"], a["causal"], a["s"], a["base"], a["dt"], a["ws"],
                          a["wsb"], None)


@pytest.mark.parametrize("kw,code", [
    (dict(q=None), 1), (dict(lse=None), 1),
    (dict(B=0), 2), (dict(N=0), 2), (dict(G=60), 2), (dict(G=512), 2), (dict(G=63, N=252), 2),
    (dict(Hq=3, Hkv=3), 2), (dict(Hq=4, Hkv=3), 2), (dict(Hq=6, Hkv=3), 2), (dict(B=-1), 2),
    (dict(dt=2), 3), (dict(d=48), 4), (dict(d=512), 4), (dict(d=16), 4),
    (dict(q=P + 8), 5), (dict(o=P + 2), 5), (dict(ws=P + 4), 5),
    (dict(ws=None), 6), (dict(wsb=1000), 6),
    (dict(s=0.0), 9), (dict(s=float("nan")), 9), (dict(base=-1.0), 9), (dict(causal=3), 9),
    (dict(causal=0x31), 9), (dict(causal=0x41), 9), (dict(causal=0x30), 9),
])
def test_fwd_rejects_bad_arguments(lib, kw, code):
    assert _fwd(lib, **kw) == code


@pytest.mark.parametrize("kw,code", [
    (dict(dq=None), 1), (dict(N=100), 2), (dict(d=40), 4), (dict(dq=P + 4), 5), (dict(wsb=16), 6),
    (dict(s=float("inf")), 9)])
def test_bwd_rejects_bad_arguments(lib, kw, code):
    assert _bwd(lib, **kw) == code


def test_device_status_rejects_null(lib):
    assert lib.s2attn_device_status(None, 4096, None) == lib.S2_ERR_NULL
    assert lib.s2attn_device_status(P, 8, None) == lib.S2_ERR_WORKSPACE
    assert lib.s2attn_selftest_wait_timeout(None, 4096, None) == lib.S2_ERR_NULL
    assert lib.s2attn_selftest_wait_timeout(P, 8, None) == lib.S2_ERR_WORKSPACE
    assert lib.s2attn_selftest_wait_timeout(P + 4, 4096, None) == lib.S2_ERR_ALIGN


def test_profiler_host_side(lib):
    assert lib.s2attn_profile_num_kernels() >= 5
    assert lib.s2attn_profile_enable(1) == 0
    names = [lib.s2attn_profile_query(i)[0] for i in range(lib.s2attn_profile_num_kernels())]
    assert "rope_pi" in names
    assert all(lib.s2attn_profile_query(i)[1] == 0 for i in range(len(names)))
    assert lib.s2attn_profile_enable(0) == 0
    assert lib.s2attn_profile_dropped() == 0
    with pytest.raises(lib.S2Error):
        lib.s2attn_profile_query(99)


def test_flops_model():
    from longlora_shifted_sparse_b200 import flops
    # 32k headline workload: 4 * B * H * N * G * d / 2 forward, 2.5x backward
    f = flops.attention_fwd_flops(1, 32768, 32, 128, 8192, True)
    assert f == 4 * 32 * 32768 * 8192 * 128 / 2
    assert flops.attention_bwd_flops(1, 32768, 32, 128, 8192, True) == 2.5 * f


def test_bwd_after_fwd_rejects_bad_arguments(lib):
    a = (1, 256, 4, 4, 64, 64, 1, 2.0, 10000.0, lib.S2_FP32)
    f = lib.s2attn_bwd_after_fwd
    assert f(P, P, P, P, P, P, None, P, P, *a, P, 1 << 40, None) == lib.S2_ERR_NULL
    assert f(P, P, P, P, P, P, P, P, P, 1, 100, 4, 4, 64, 64, 1, 2.0, 10000.0, lib.S2_FP32,
             P, 1 << 40, None) == lib.S2_ERR_SHAPE
    assert f(P, P, P, P, P, P, P + 4, P, P, *a, P, 1 << 40, None) == lib.S2_ERR_ALIGN
    assert f(P, P, P, P, P, P, P, P, P, *a, P, 16, None) == lib.S2_ERR_WORKSPACE
