"""GPU parity: the library (through its C ABI) against the fp64 oracle on identical seeded
inputs. Small shapes are compared element by element in full; the LLaMA2-sized workloads
run at full size in the configuration the bench times and are compared on sampled rows
(tile edges, the half-group boundary, the wrap group of the shifted heads)."""
import os

import numpy as np
import pytest
import torch

import oracle
import synth
from tests import gpu_helpers as H
from workloads import WORKLOADS, Workload

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def s2():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from longlora_shifted_sparse_b200 import s2attn  # raises if the library is missing
    return s2attn


def _run(s2, w, q, k, v, do):
    """Forward (and backward) through the library; every call's device status is checked, so
    an expired wait shows up as such rather than as wrong numbers."""
    tq, tk, tv = (H.to_device(x, w.dtype) for x in (q, k, v))
    o, lse = s2.forward(tq, tk, tv, w.G, w.pi_scale, w.rope_base, w.causal, shift=w.shift,
                        check_status=True)
    grads = None
    if do is not None:
        tdo = H.to_device(do, w.dtype)
        grads = s2.backward(tq, tk, tv, o, lse, tdo, w.G, w.pi_scale, w.rope_base, w.causal,
                            shift=w.shift, check_status=True)
    torch.cuda.synchronize()
    return o, lse, grads


def _full_compare(s2, w):
    q, k, v, do = H.inputs(w, with_dout=w.backward)
    o, lse, grads = _run(s2, w, q, k, v, do)
    o_ref, lse_ref = oracle.fwd(q, k, v, w.G, w.pi_scale, w.rope_base, w.causal, shift=w.shift)
    H.assert_close_o(H.to_host_f64(o), o_ref, w.dtype)
    H.assert_close_lse(H.to_host_f64(lse), lse_ref, w.dtype)
    if grads is not None:
        refs = oracle.bwd(q, k, v, do, w.G, w.pi_scale, w.rope_base, w.causal, shift=w.shift)
        for name, g, r in zip(("dq", "dk", "dv"), grads, refs):
            H.assert_close_grad(H.to_host_f64(g), r, w.dtype, name)


def test_tiny_fp32_workload_full(s2):
    """The tiny fp32 workload (N=256, H=4, d=64, G=64, s=2), fwd+bwd, every element."""
    _full_compare(s2, WORKLOADS["tiny_fp32"])


SMALL = [
    # name, B, N, Hq, Hkv, d, G, s, dtype, causal
    ("bf16_d128_g256", 1, 1024, 4, 4, 128, 256, 2.0, "bf16", True),
    ("bf16_gqa_b2", 2, 1024, 8, 2, 128, 512, 4.0, "bf16", True),
    ("bf16_one_group", 1, 512, 4, 4, 128, 512, 1.0, "bf16", True),
    ("bf16_noncausal", 1, 1024, 4, 4, 128, 256, 2.0, "bf16", False),
    ("bf16_d64_g64", 1, 512, 4, 4, 64, 64, 2.0, "bf16", True),
    ("bf16_d32_odd_tiles", 1, 600, 2, 2, 32, 200, 1.0, "bf16", True),
    ("f32_d128_g96", 1, 384, 4, 2, 128, 96, 3.0, "f32", True),
    ("f32_d256_noncausal", 1, 128, 2, 2, 256, 32, 1.0, "f32", False),
    ("f32_g2_minimal", 1, 8, 2, 2, 32, 2, 1.0, "f32", True),
    # several work items per CTA in the persistent kernels (forward 256 items, dQ 512, on
    # 148 CTAs), compared in full: the item-to-item hand-over of their rings
    ("bf16_multi_item_gqa", 1, 8192, 8, 4, 128, 1024, 2.0, "bf16", True),
    # the same with one query head per kv head (dQ 256 items; the last key tile of every
    # group has a single (query head, query tile) pair in the dK/dV pass)
    ("bf16_multi_item_mha", 1, 8192, 4, 4, 128, 1024, 2.0, "bf16", True),
    # and across batch entries: the unit number carries b (forward 256 items, dQ 512)
    ("bf16_multi_item_b2", 2, 4096, 8, 4, 128, 1024, 4.0, "bf16", True),
    # head dims of 3, 5, 6 and 7 elements per lane on the CUDA-core kernels
    ("bf16_d96_gqa", 1, 384, 4, 2, 96, 128, 2.0, "bf16", True),
    ("f32_d160_noncausal", 1, 256, 2, 2, 160, 64, 1.5, "f32", False),
    ("bf16_d192", 1, 256, 2, 2, 192, 64, 3.0, "bf16", True),
    ("f32_d224_b2", 2, 128, 2, 2, 224, 32, 1.0, "f32", True),
]


@pytest.mark.parametrize("case", SMALL, ids=[c[0] for c in SMALL])
def test_small_shapes_full(s2, case):
    name, B, N, Hq, Hkv, d, G, s, dt, causal = case
    w = Workload(name, B, N, Hq, Hkv, d, G, s, dt, 0.5 if dt == "bf16" else 1.0, True,
                 seed=100 + SMALL.index(case), causal=causal)
    expect_tc = dt == "bf16" and d == 128 and G % 256 == 0
    code = s2.S2_BF16 if dt == "bf16" else s2.S2_FP32
    assert s2.s2attn_kernel_path(B, N, Hq, Hkv, d, G, int(causal), code) == int(expect_tc)
    _full_compare(s2, w)


# The other head patterns, the full-group (no mask) reading and RoPE base scaling, on both
# kernel families: Workload(name, B, N, Hq, Hkv, d, G, s, dtype, in_scale, backward, seed, ...)
VARIANTS = [
    Workload("bf16_alternate", 1, 1024, 4, 4, 128, 256, 2.0, "bf16", 0.5, True, 120,
             shift="alternate"),
    Workload("bf16_alternate_gqa_b2", 2, 1024, 8, 4, 128, 512, 4.0, "bf16", 0.5, True, 121,
             shift="alternate"),
    Workload("bf16_alternate_noncausal", 1, 1024, 4, 2, 128, 256, 2.0, "bf16", 0.5, True, 122,
             causal=False, shift="alternate"),
    Workload("bf16_none_dense_causal", 1, 1024, 4, 4, 128, 1024, 1.0, "bf16", 0.5, True, 123,
             shift="none"),
    Workload("bf16_none_groups_gqa", 1, 1024, 4, 2, 128, 256, 2.0, "bf16", 0.5, True, 124,
             shift="none"),
    Workload("bf16_base_scaled", 1, 1024, 4, 4, 128, 256, 1.0, "bf16", 0.5, True, 125,
             rope_base=80000.0),
    Workload("bf16_d64_alternate", 1, 512, 4, 4, 64, 64, 2.0, "bf16", 0.5, True, 126,
             shift="alternate"),
    Workload("f32_alternate_gqa", 1, 384, 4, 2, 64, 96, 3.0, "f32", 1.0, True, 127,
             shift="alternate"),
    Workload("f32_none_dense_causal", 1, 256, 2, 2, 64, 256, 1.0, "f32", 1.0, True, 128,
             shift="none"),
    Workload("f32_base_scaled_noncausal", 1, 256, 4, 4, 64, 64, 1.0, "f32", 1.0, True, 129,
             causal=False, rope_base=40000.0),
    # edge cases of the persistent kernels: fewer work items than SMs, one group of two
    # tiles per batch entry, an 8:1 query-to-kv head ratio, one group holding everything
    Workload("bf16_b3_one_group_two_tiles", 3, 256, 2, 2, 128, 256, 1.0, "bf16", 0.5, True,
             131),
    Workload("bf16_gqa_8to1", 1, 512, 16, 2, 128, 256, 2.0, "bf16", 0.5, True, 132),
    Workload("bf16_one_group_alternate_noncausal", 1, 2048, 4, 2, 128, 2048, 1.0, "bf16",
             0.5, True, 133, causal=False, shift="alternate"),
]


@pytest.mark.parametrize("w", VARIANTS, ids=[w.name for w in VARIANTS])
def test_variants_full(s2, w):
    expect_tc = w.dtype == "bf16" and w.d == 128 and w.G % 256 == 0
    code = s2.S2_BF16 if w.dtype == "bf16" else s2.S2_FP32
    assert s2.s2attn_kernel_path(w.B, w.N, w.Hq, w.Hkv, w.d, w.G, s2.mode(w.causal, w.shift),
                                 code) == int(expect_tc)
    _full_compare(s2, w)


def test_no_shift_one_group_matches_sdpa(s2):
    """Pattern "none" with G = N on the tensor-core path against torch's causal SDPA (fp64,
    CPU) on the rotated inputs: a library routine, independent of the oracle's attention."""
    w = Workload("sdpa", 1, 1024, 4, 4, 128, 1024, 1.0, "bf16", 0.5, False, 130, shift="none")
    q, k, v, _ = H.inputs(w, with_dout=False)
    o, _, _ = _run(s2, w, q, k, v, None)
    pos = np.arange(w.N)

    def rotated(x):
        xf = synth.bf16_bits_to_f32(x).astype(np.float64)[0]
        return np.stack([oracle.rope(xf[:, h], pos, w.pi_scale, w.rope_base)
                         for h in range(xf.shape[1])])          # [H, N, d]

    vf = synth.bf16_bits_to_f32(v).astype(np.float64)[0].transpose(1, 0, 2)
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(rotated(q)), torch.from_numpy(rotated(k)), torch.from_numpy(vf),
        is_causal=True).numpy().transpose(1, 0, 2)[None]
    H.assert_close_o(H.to_host_f64(o), ref, "bf16")


def _sampled_fwd_check(w, q, k, v, o, lse):
    ng = w.N // w.G
    heads = sorted({0, w.Hq // 2 - 1, w.Hq // 2, w.Hq - 1})
    groups = sorted({0, ng // 2, ng - 1})
    rows = H.sample_rows(w.G)
    got_o, got_l, ref_o, ref_l = [], [], [], []
    for h in heads:
        kvh = h // (w.Hq // w.Hkv)
        for g in groups:
            tok = oracle.unit_rows(w.N, w.G, w.Hq, kvh, w.Hkv, g, shift=w.shift)[rows]
            o_r, l_r = oracle.fwd_rows(q, k, v, w.G, w.pi_scale, 0, h, g, rows, w.rope_base,
                                       w.causal, shift=w.shift)
            idx = torch.as_tensor(tok, device=o.device)
            got_o.append(H.to_host_f64(o[0, idx, h]))
            got_l.append(H.to_host_f64(lse[0, h, idx]))
            ref_o.append(o_r)
            ref_l.append(l_r)
    H.assert_close_o(np.concatenate(got_o), np.concatenate(ref_o), w.dtype)
    H.assert_close_lse(np.concatenate(got_l), np.concatenate(ref_l), w.dtype)


def _sampled_bwd_check(w, q, k, v, do, grads, units):
    """dq, dk, dv on sampled rows, each unit (b, kv head, group) against its own bound: one
    bad unit is not diluted by the norms of the others."""
    dq, dk, dv = grads
    R = w.Hq // w.Hkv
    rows = H.sample_rows(w.G, extra=4, seed=1)
    for (b, kvh, g) in units:
        tok = oracle.unit_rows(w.N, w.G, w.Hq, kvh, w.Hkv, g, shift=w.shift)[rows]
        dq_r, dk_r, dv_r = oracle.bwd_rows(q, k, v, do, w.G, w.pi_scale, b, kvh, g, rows, rows,
                                           w.rope_base, w.causal, shift=w.shift)
        idx = torch.as_tensor(tok, device=dq.device)
        unit = "(b=%d, kvh=%d, g=%d)" % (b, kvh, g)
        H.assert_close_grad(H.to_host_f64(dq[b, idx, kvh * R:(kvh + 1) * R]), dq_r, w.dtype,
                            "dq " + unit)
        H.assert_close_grad(H.to_host_f64(dk[b, idx, kvh]), dk_r, w.dtype, "dk " + unit)
        H.assert_close_grad(H.to_host_f64(dv[b, idx, kvh]), dv_r, w.dtype, "dv " + unit)


BIG = ["llama2_7b_8k_fwd", "llama2_7b_32k", "llama2_70b_gqa_32k", "llama2_7b_100k",
       "llama2_7b_32k_noncausal", "llama2_7b_32k_alternate", "llama2_7b_32k_base_scaled",
       "llama2_7b_32k_dense_infer"]


@pytest.mark.parametrize("name", BIG)
def test_llama2_workload_sampled(s2, name):
    """Full-size run; O/LSE on sampled rows of both head halves and first / middle / last
    (wrap) groups; dq/dk/dv on sampled rows of units in both halves incl. the wrap group."""
    w = WORKLOADS[name]
    # these shapes must take the tensor-core kernels
    assert s2.s2attn_kernel_path(w.B, w.N, w.Hq, w.Hkv, w.d, w.G, s2.mode(w.causal, w.shift),
                                 s2.S2_BF16) == 1
    q, k, v, do = H.inputs(w, with_dout=w.backward)
    o, lse, grads = _run(s2, w, q, k, v, do)
    _sampled_fwd_check(w, q, k, v, o, lse)
    if w.backward:
        # both head halves, first and last (for a shifted head, the wrap) group of each
        ng = w.N // w.G
        units = [(0, 0, 0), (0, w.Hkv - 1, ng - 1), (0, w.Hkv // 2, 0),
                 (0, w.Hkv // 2 - 1, ng - 1)]
        _sampled_bwd_check(w, q, k, v, do, grads, units)


def test_outputs_stay_inside_their_buffers(s2):
    """Canary bands (NaN patterns) around every output are untouched."""
    w = Workload("canary", 1, 1024, 4, 2, 128, 256, 2.0, "bf16", 0.5, True, seed=7)
    q, k, v, do = H.inputs(w)
    tq, tk, tv, tdo = (H.to_device(x, "bf16") for x in (q, k, v, do))
    pad = 64

    def padded(shape, dtype):
        n = int(np.prod(shape))
        buf = torch.empty(n + 2 * pad, dtype=dtype, device="cuda")
        buf.view(torch.int16 if dtype == torch.bfloat16 else torch.int32).fill_(-1)
        return buf, buf[pad:pad + n].view(shape)

    ob, o = padded(tq.shape, torch.bfloat16)
    lb, lse = padded((1, w.Hq, w.N), torch.float32)
    qb, dq = padded(tq.shape, torch.bfloat16)
    kb, dk = padded(tk.shape, torch.bfloat16)
    vb, dv = padded(tv.shape, torch.bfloat16)
    s2.forward(tq, tk, tv, w.G, w.pi_scale, out=o, lse=lse)
    s2.backward(tq, tk, tv, o, lse, tdo, w.G, w.pi_scale, grads=(dq, dk, dv))
    torch.cuda.synchronize()
    for buf in (ob, lb, qb, kb, vb):
        ints = buf.view(torch.int16 if buf.dtype == torch.bfloat16 else torch.int32)
        assert bool((ints[:pad] == -1).all()) and bool((ints[-pad:] == -1).all())
    assert bool(torch.isfinite(o).all()) and bool(torch.isfinite(dq).all())


def test_results_are_deterministic(s2):
    w = Workload("det", 1, 2048, 8, 2, 128, 512, 4.0, "bf16", 0.5, True, seed=8)
    q, k, v, do = H.inputs(w)
    a = _run(s2, w, q, k, v, do)
    b = _run(s2, w, q, k, v, do)
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])
    for x, y in zip(a[2], b[2]):
        assert torch.equal(x, y)


def test_autograd_function_matches_abi_calls(s2):
    w = Workload("ag", 1, 512, 4, 4, 64, 128, 2.0, "f32", 1.0, True, seed=9)
    q, k, v, do = H.inputs(w)
    tq, tk, tv = (H.to_device(x, "f32").requires_grad_(True) for x in (q, k, v))
    o = s2.s2_attention(tq, tk, tv, w.G, w.pi_scale)
    o.backward(H.to_device(do, "f32"))
    o2, lse2, (dq, dk, dv) = _run(s2, w, q, k, v, do)
    assert torch.equal(o.detach(), o2)
    assert torch.equal(tq.grad, dq) and torch.equal(tk.grad, dk) and torch.equal(tv.grad, dv)


def test_device_status_and_profiler(s2):
    w = Workload("prof", 1, 1024, 4, 4, 128, 256, 2.0, "bf16", 0.5, True, seed=10)
    q, k, v, do = H.inputs(w)
    tq, tk, tv = (H.to_device(x, "bf16") for x in (q, k, v))
    ws = s2.workspace(w.B, w.N, w.Hq, w.Hkv, w.d, s2.S2_BF16, tq.device)
    s2.check(s2.s2attn_profile_enable(1))
    o, lse = s2.forward(tq, tk, tv, w.G, w.pi_scale, ws=ws)
    s2.backward(tq, tk, tv, o, lse, H.to_device(do, "bf16"), w.G, w.pi_scale, ws=ws)
    assert s2.device_status(ws) == s2.S2_OK
    summary = s2.profile_summary()
    s2.check(s2.s2attn_profile_enable(0))
    assert summary["rope_table"][0] == summary["rope_pi"][0] == 2
    assert summary["bwd_rowsum"][0] == 1
    assert sum(n for n, _ in summary.values()) == 8
    assert all(ms > 0 for _, ms in summary.values())


@pytest.mark.parametrize("case", [
    # name, B, N, Hq, Hkv, d, G, s, dtype
    ("tcgen05_gqa", 1, 1024, 4, 2, 128, 256, 2.0, "bf16"),
    ("cuda_core_f32", 1, 256, 4, 4, 64, 64, 2.0, "f32"),
], ids=lambda c: c[0])
def test_backward_after_forward_is_bit_identical(s2, case):
    """s2attn_bwd_after_fwd reuses the rotated q, k that the forward left in its workspace;
    s2attn_bwd rotates them again into a fresh workspace. The rotation is deterministic and
    so are the backward kernels (no atomics), so the gradients must agree bit for bit; the
    autograd wrapper, which takes the first route, must agree as well."""
    name, B, N, Hq, Hkv, d, G, s, dt = case
    q, k, v, do = synth.s2attn_inputs(77, B, N, Hq, Hkv, d, 0.5 if dt == "bf16" else 1.0, dt)
    tq, tk, tv, tdo = (H.to_device(x, dt) for x in (q, k, v, do))
    code = s2.S2_BF16 if dt == "bf16" else s2.S2_FP32
    ws = s2.workspace(B, N, Hq, Hkv, d, code, tq.device)
    o, lse = s2.forward(tq, tk, tv, G, s, ws=ws)
    g_after = s2.backward(tq, tk, tv, o, lse, tdo, G, s, ws=ws, after_forward=True)
    g_fresh = s2.backward(tq, tk, tv, o, lse, tdo, G, s)
    torch.cuda.synchronize()
    assert s2.device_status(ws) == s2.S2_OK
    for a, b in zip(g_after, g_fresh):
        assert torch.equal(a, b)
    xs = [t.clone().requires_grad_(True) for t in (tq, tk, tv)]
    out = s2.s2_attention(xs[0], xs[1], xs[2], G, s)
    out.backward(tdo)
    assert torch.equal(out.detach(), o)
    for x, g in zip(xs, g_fresh):
        assert torch.equal(x.grad, g)


def test_softmax_rescale_paths(s2):
    """Scores whose running row max climbs by well over the forward's rescale threshold
    (2^8) along each group, so that the exact-max exchange, the power-of-two rescale of P
    already written and the O rescale all run, checked forward and backward against the
    oracle.

    Inputs: q, k, v ~ N(0,1)*0.5, then channel 0 of every q row set to 8 and channel 0 of
    every k row raised by 16 * (group-local position / G): the score gains ~11 nats from the
    first to the last key of a group (~1.4 nats per 128-key tile), while the keys of one tile
    stay within a few nats of each other, so the softmax rows are not one-hot and the
    backward tolerances keep their meaning. A position-interpolation factor of 1e30 makes
    every RoPE angle ~1e-27 rad: the rotation is the identity far below bf16 resolution on
    both sides, so channel 0 keeps its role in every head. The test first checks its own
    premise on the fp64 scores."""
    w = Workload("rescale", 1, 2048, 4, 2, 128, 1024, 1e30, "bf16", 0.5, True, seed=31)
    q, k, v, do = H.inputs(w, with_dout=True)
    qf = synth.bf16_bits_to_f32(q)
    kf = synth.bf16_bits_to_f32(k)
    qf[..., 0] = 8.0
    kf[..., 0] += (16.0 * (np.arange(w.N) % w.G) / w.G).astype(np.float32)[None, :, None]
    q, k = synth.f32_to_bf16_bits(qf), synth.f32_to_bf16_bits(kf)
    # premise: rows of the unshifted head 0, group 0 whose running max (log2 units) grows by
    # more than 8 after their first key tile
    qg = synth.bf16_bits_to_f32(q).astype(np.float64)[0, :w.G, 0]
    kg = synth.bf16_bits_to_f32(k).astype(np.float64)[0, :w.G, 0]
    sc = qg @ kg.T / np.sqrt(w.d) * np.log2(np.e)
    sc[np.triu_indices(w.G, 1)] = -np.inf
    grows = sum(sc[i, :i + 1].max() > sc[i, :128].max() + 8 for i in range(128, w.G))
    assert grows > 100, grows
    o, lse, grads = _run(s2, w, q, k, v, do)
    o_ref, lse_ref = oracle.fwd(q, k, v, w.G, w.pi_scale, w.rope_base, w.causal, shift=w.shift)
    H.assert_close_o(H.to_host_f64(o), o_ref, w.dtype)
    H.assert_close_lse(H.to_host_f64(lse), lse_ref, w.dtype)
    refs = oracle.bwd(q, k, v, do, w.G, w.pi_scale, w.rope_base, w.causal, shift=w.shift)
    for name, g, r in zip(("dq", "dk", "dv"), grads, refs):
        H.assert_close_grad(H.to_host_f64(g), r, w.dtype, name)


@pytest.mark.skipif(os.environ.get("S2_FULL_PARITY") != "1",
                    reason="minutes of host time: run with S2_FULL_PARITY=1")
def test_llama2_7b_32k_every_element(s2):
    """The bench's 32k workload compared element by element: every output of o, lse, dq,
    dk, dv against the full fp64 oracle (about 8e12 fp64 FLOPs on the host cores)."""
    _full_compare(s2, WORKLOADS["llama2_7b_32k"])
