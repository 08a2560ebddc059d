"""Helpers of the GPU parity tests: move seeded host inputs to the device, run the library
through its C ABI, bring results back, and compare them with the oracle's."""
from __future__ import annotations

import json
import os

import numpy as np
import torch

import synth

# With S2_PARITY_REPORT=<path>, every comparison appends one JSON line (test, quantity,
# measured error, bound) to that file: the margins of each parity case against its bound.
_REPORT = os.environ.get("S2_PARITY_REPORT")


def _record(what: str, kind: str, err: float, bound: float) -> None:
    if not _REPORT:
        return
    test = os.environ.get("PYTEST_CURRENT_TEST", "").split(" ")[0]
    with open(_REPORT, "a") as f:
        f.write(json.dumps({"test": test, "what": what, "kind": kind, "err": err,
                            "bound": bound}) + "\n")


# Tolerances. bf16 inputs with fp32 accumulation: max-abs 2e-2 on O, relative L2 1e-2 on
# dq, dk, dv; LSE absolute 5e-3 (scores carry the bf16 rounding of the rotated q and k).
# fp32: relative L2 1e-5 and max-abs 1e-5 * max|ref| on every output, LSE absolute 1e-5.
TOL_BF16_O_MAXABS = 2e-2
TOL_BF16_GRAD_RELL2 = 1e-2
TOL_BF16_LSE_ABS = 5e-3
TOL_F32_REL = 1e-5
TOL_F32_LSE_ABS = 1e-5


def to_device(x: np.ndarray, dtype: str, device="cuda") -> torch.Tensor:
    if dtype == "bf16":
        t = torch.from_numpy(np.ascontiguousarray(x).view(np.int16)).to(device)
        return t.view(torch.bfloat16)
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(device)


def to_host_f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)


def inputs(w, with_dout=True):
    return synth.s2attn_inputs(w.seed, w.B, w.N, w.Hq, w.Hkv, w.d, w.in_scale, w.dtype,
                               with_dout=with_dout)


def rel_l2(a, b) -> float:
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))


def max_abs(a, b) -> float:
    return float(np.abs(np.asarray(a, np.float64) - np.asarray(b, np.float64)).max())


def assert_close_o(got, ref, dtype, what="o"):
    if dtype == "bf16":
        e = max_abs(got, ref)
        _record(what, "max-abs", e, TOL_BF16_O_MAXABS)
        assert e <= TOL_BF16_O_MAXABS, "%s max-abs %.3e" % (what, e)
    else:
        assert_close_f32(got, ref, what)


def assert_close_grad(got, ref, dtype, what):
    if dtype == "bf16":
        e = rel_l2(got, ref)
        _record(what, "rel-L2", e, TOL_BF16_GRAD_RELL2)
        assert e <= TOL_BF16_GRAD_RELL2, "%s rel-L2 %.3e" % (what, e)
    else:
        assert_close_f32(got, ref, what)


def assert_close_f32(got, ref, what):
    e = rel_l2(got, ref)
    m = max_abs(got, ref)
    bound = TOL_F32_REL * float(np.abs(ref).max())
    _record(what, "rel-L2", e, TOL_F32_REL)
    _record(what, "max-abs/max|ref|", m / max(float(np.abs(ref).max()), 1e-300), TOL_F32_REL)
    assert e <= TOL_F32_REL, "%s rel-L2 %.3e" % (what, e)
    assert m <= bound, "%s max-abs %.3e > %.3e" % (what, m, bound)


def assert_close_lse(got, ref, dtype, what="lse"):
    tol = TOL_BF16_LSE_ABS if dtype == "bf16" else TOL_F32_LSE_ABS
    e = max_abs(got, ref)
    _record(what, "abs", e, tol)
    assert e <= tol, "%s abs %.3e" % (what, e)


def sample_rows(G: int, extra: int = 6, seed: int = 0) -> np.ndarray:
    """Rolled local rows that cover tile edges (128-row tiles), the half-group boundary and
    the group's last rows, plus a few random ones."""
    cand = {0, 1, 2, 63, 64, 127, 128, 129, 255, 256, G // 2 - 1, G // 2, G // 2 + 1,
            G - 129, G - 128, G - 127, G - 2, G - 1}
    rng = np.random.default_rng(seed)
    cand |= set(int(x) for x in rng.integers(0, G, size=extra))
    return np.array(sorted(r for r in cand if 0 <= r < G), dtype=np.int64)
