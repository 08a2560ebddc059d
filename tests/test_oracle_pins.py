"""Pins of the fp64 oracle against facts that do not come from the oracle itself.

Each test names what fixes the expected value: a worked example printed on the pages
(tests/golden), a closed form, an invariant of the method, a special case that reduces
to a library routine (torch SDPA on rolled/folded tensors), or finite differences.
"""
import math
import os

import numpy as np
import pytest
import torch

import oracle
import synth
from tests import s2_torch_formulation as ref

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _inputs(seed, B, N, Hq, Hkv, d, dtype="f64"):
    q, k, v, do = synth.s2attn_inputs(seed, B, N, Hq, Hkv, d, 1.0, "f32")
    return tuple(x.astype(np.float64) for x in (q, k, v, do))


def _t(x):
    return torch.from_numpy(np.ascontiguousarray(x))


# ---------------------------------------------------------------- RoPE + PI (closed forms)

def test_rope_matches_complex_closed_form():
    """RoFormer's closed form: pair (x0, x1) -> (x0 + i x1) * exp(i (m/s) base^(-2i/d))."""
    rng = np.random.default_rng(1)
    d, n = 16, 40
    x = rng.standard_normal((n, d))
    pos = rng.integers(0, 100000, size=n)
    for s in (1.0, 2.0, 8.0, 25.0):
        y = oracle.rope(x, pos, s, 10000.0)
        z = x[:, 0::2] + 1j * x[:, 1::2]
        ang = (pos[:, None] / s) * 10000.0 ** (-np.arange(0, d, 2) / d)[None, :]
        w = z * np.exp(1j * ang)
        np.testing.assert_allclose(y[:, 0::2], w.real, rtol=0, atol=1e-9)
        np.testing.assert_allclose(y[:, 1::2], w.imag, rtol=0, atol=1e-9)


@pytest.mark.parametrize("base", [80000.0, 500000.0])
def test_rope_base_scaling_closed_form(base):
    """RoPE base scaling (a larger base, positions not interpolated): the closed form with
    that base; pair 0 keeps angle m for every base, every other pair turns more slowly."""
    rng = np.random.default_rng(4)
    d, n = 16, 24
    x = rng.standard_normal((n, d))
    pos = rng.integers(0, 100000, size=n)
    y = oracle.rope(x, pos, 1.0, base)
    z = (x[:, 0::2] + 1j * x[:, 1::2]) * np.exp(
        1j * pos[:, None] * base ** (-np.arange(0, d, 2) / d)[None, :])
    np.testing.assert_allclose(y[:, 0::2], z.real, rtol=0, atol=1e-9)
    np.testing.assert_allclose(y[:, 1::2], z.imag, rtol=0, atol=1e-9)
    e = np.zeros((d // 2, d))
    for i in range(d // 2):
        e[i, 2 * i] = 1.0
    one = np.ones(d // 2, dtype=np.int64)
    ang = lambda b: np.array([math.atan2(r[2 * i + 1], r[2 * i])
                              for i, r in enumerate(oracle.rope(e, one, 1.0, b))])
    a_ref, a_big = ang(10000.0), ang(base)
    assert a_big[0] == pytest.approx(1.0, abs=1e-15) and a_ref[0] == pytest.approx(1.0, abs=1e-15)
    assert np.all(a_big[1:] < a_ref[1:])


def test_rope_frequency_decreases_geometrically():
    """The angle of pair i at m = 1, s = 1 is theta_i = base^(-2i/d): a geometric sequence."""
    d = 8
    x = np.zeros((d // 2, d))
    for i in range(d // 2):
        x[i, 2 * i] = 1.0
    y = oracle.rope(x, np.ones(d // 2, dtype=np.int64), 1.0, 10000.0)
    ang = np.array([math.atan2(y[i, 2 * i + 1], y[i, 2 * i]) for i in range(d // 2)])
    np.testing.assert_allclose(ang, 10000.0 ** (-2.0 * np.arange(d // 2) / d), rtol=1e-12)
    np.testing.assert_allclose(ang[1:] / ang[:-1], 10000.0 ** (-2.0 / d), rtol=1e-12)


def test_rope_invariants():
    """Orthogonal (norm-preserving), identity at m = 0, inverse undoes it, relative position."""
    rng = np.random.default_rng(2)
    d, n = 32, 16
    x = rng.standard_normal((n, d))
    kx = rng.standard_normal((n, d))
    pos = rng.integers(0, 5000, size=n)
    y = oracle.rope(x, pos, 4.0)
    np.testing.assert_allclose(np.linalg.norm(y, axis=1), np.linalg.norm(x, axis=1), rtol=1e-12)
    np.testing.assert_array_equal(oracle.rope(x, np.zeros(n, np.int64), 4.0), x)
    np.testing.assert_allclose(oracle.rope(y, pos, 4.0, inverse=True), x, atol=1e-12)
    # <R(m) q, R(n) k> depends only on m - n.
    m, nn, shift = 700, 300, 1234
    a = oracle.rope(x[:1], [m], 4.0) @ oracle.rope(kx[:1], [nn], 4.0).T
    b = oracle.rope(x[:1], [m + shift], 4.0) @ oracle.rope(kx[:1], [nn + shift], 4.0).T
    np.testing.assert_allclose(a, b, rtol=1e-10)


def test_position_interpolation_divides_position():
    """PI: rotating at position m with scale s equals rotating at m/s with s = 1."""
    rng = np.random.default_rng(3)
    x = rng.standard_normal((5, 16))
    for s in (2, 8, 25):
        mp = rng.integers(0, 4096, size=5)
        np.testing.assert_allclose(oracle.rope(x, mp * s, float(s)), oracle.rope(x, mp, 1.0),
                                   atol=1e-12)


# ---------------------------------------------------------------- attention special cases

@pytest.mark.parametrize("Hq,Hkv", [(4, 4), (4, 2)])
def test_one_group_unshifted_heads_equal_dense_causal(Hq, Hkv):
    """G = N: the unshifted heads are textbook dense causal attention (torch SDPA)."""
    N, d = 32, 8
    q, k, v, _ = _inputs(4, 1, N, Hq, Hkv, d)
    o, _ = oracle.fwd(q, k, v, G=N, s=2.0)
    dense = ref.dense_causal(_t(q), _t(k), _t(v), 2.0).numpy()
    np.testing.assert_allclose(o[:, :, :Hq // 2], dense[:, :, :Hq // 2], atol=1e-12)


@pytest.mark.parametrize("B,N,Hq,Hkv,d,G,causal", [
    (1, 64, 4, 4, 8, 16, True), (2, 48, 4, 2, 8, 8, True), (1, 64, 8, 2, 16, 32, True),
    (1, 32, 4, 4, 8, 8, False), (1, 256, 4, 4, 64, 64, True)])
def test_oracle_equals_library_formulation(B, N, Hq, Hkv, d, G, causal):
    """Oracle == roll / fold / SDPA / roll-back built from torch routines, O and LSE."""
    q, k, v, _ = _inputs(5, B, N, Hq, Hkv, d)
    o, lse = oracle.fwd(q, k, v, G=G, s=2.0, causal=causal)
    o_r, lse_r = ref.s2attn(_t(q), _t(k), _t(v), G, 2.0, causal=causal, with_lse=True)
    np.testing.assert_allclose(o, o_r.numpy(), atol=1e-12)
    np.testing.assert_allclose(lse, lse_r.numpy(), atol=1e-12)


def test_unshifted_heads_are_block_diagonal():
    """Unshifted heads: each group alone is dense causal attention over its own rows."""
    N, G, d = 64, 16, 8
    q, k, v, _ = _inputs(6, 1, N, 2, 2, d)
    o, _ = oracle.fwd(q, k, v, G=G, s=1.0)
    qr = ref.rope_complex(_t(q), 1.0)
    kr = ref.rope_complex(_t(k), 1.0)
    for g in range(N // G):
        sl = slice(g * G, (g + 1) * G)
        og = torch.nn.functional.scaled_dot_product_attention(
            qr[0, sl, 0][None], kr[0, sl, 0][None], _t(v)[0, sl, 0][None], is_causal=True)
        np.testing.assert_allclose(o[0, sl, 0], og[0].numpy(), atol=1e-12)


def _read_shift_examples():
    rows = []
    with open(os.path.join(GOLDEN, "shift_groups.txt")) as f:
        for line in f:
            if line.strip() and not line.startswith("#"):
                rows.append(tuple(int(x) for x in line.split()))
    return rows


@pytest.mark.parametrize("G,first,last", _read_shift_examples())
def test_first_shifted_group_worked_example(G, first, last):
    """The shifted heads' first group is tokens G/2 .. 3G/2-1 (pages' worked examples).

    Perturbing any token outside that range leaves the shifted head's outputs at those
    tokens unchanged; the unit-row map of group 0 is exactly that range."""
    N = 2 * G
    rows = oracle.unit_rows(N, G, Hq=2, kvh=1, Hkv=2, g=0)
    assert rows[0] == first and rows[-1] == last
    np.testing.assert_array_equal(rows, np.arange(first, last + 1))
    if G > 64:
        return  # the index map is the pin at this size; the perturbation check runs small
    q, k, v, _ = _inputs(7, 1, N, 2, 2, 4)
    o, _ = oracle.fwd(q, k, v, G=G, s=1.0)
    outside = np.r_[0:first, last + 1:N]
    k2, v2 = k.copy(), v.copy()
    k2[:, outside] += 3.0
    v2[:, outside] -= 2.0
    o2, _ = oracle.fwd(q, k2, v2, G=G, s=1.0)
    np.testing.assert_array_equal(o2[0, first:last + 1, 1], o[0, first:last + 1, 1])
    assert np.abs(o2[0, :G, 0] - o[0, :G, 0]).max() > 1e-3  # unshifted head does see them


def test_wrap_group_mixes_end_and_start():
    """np.roll wraps: the last shifted group holds tokens N-G/2..N-1 then 0..G/2-1, so the
    shifted head's output at token 0 depends on the sequence's last tokens (and the
    unshifted head's does not)."""
    N, G, d = 32, 8, 4
    q, k, v, _ = _inputs(8, 1, N, 2, 2, d)
    o, _ = oracle.fwd(q, k, v, G=G, s=1.0)
    rows = oracle.unit_rows(N, G, 2, 1, 2, N // G - 1)
    np.testing.assert_array_equal(rows, np.r_[N - G // 2:N, 0:G // 2])
    v2 = v.copy()
    v2[0, N - 1] += 5.0
    o2, _ = oracle.fwd(q, k, v2, G=G, s=1.0)
    assert abs(o2[0, 0, 1] - o[0, 0, 1]).max() > 1e-6
    np.testing.assert_array_equal(o2[0, 0, 0], o[0, 0, 0])


def _read_alternate_examples():
    rows = []
    with open(os.path.join(GOLDEN, "alternate_heads.txt")) as f:
        for line in f:
            if line.strip() and not line.startswith("#"):
                rows.append(tuple(int(x) for x in line.split()))
    return rows


@pytest.mark.parametrize("G,head,first,last", _read_alternate_examples())
def test_alternate_head_pattern_worked_example(G, head, first, last):
    """Alternate-head shift pattern: even heads see tokens 0 .. G-1 in their first group,
    odd heads tokens G/2 .. 3G/2-1 (the pages' group figure, tests/golden)."""
    rows = oracle.unit_rows(2 * G, G, Hq=8, kvh=head, Hkv=8, g=0, shift="alternate")
    assert rows[0] == first and rows[-1] == last
    np.testing.assert_array_equal(rows, np.arange(first, last + 1))


@pytest.mark.parametrize("Hq,Hkv,causal", [(4, 4, True), (8, 4, True), (4, 4, False)])
def test_alternate_pattern_is_the_half_pattern_on_reordered_heads(Hq, Hkv, causal):
    """Heads are computed independently, so shifting the odd kv heads equals shifting the
    second half after reordering the kv heads as [even..., odd...] (query heads follow their
    kv head): the alternate pattern is pinned to the half pattern's pins, forward and
    backward."""
    B, N, d, G = 1, 32, 8, 8
    q, k, v, do = _inputs(21, B, N, Hq, Hkv, d)
    R = Hq // Hkv
    kv_perm = np.r_[0:Hkv:2, 1:Hkv:2]
    q_perm = np.concatenate([np.arange(h * R, (h + 1) * R) for h in kv_perm])
    o_a, l_a = oracle.fwd(q, k, v, G, 2.0, causal=causal, shift="alternate")
    o_h, l_h = oracle.fwd(q[:, :, q_perm], k[:, :, kv_perm], v[:, :, kv_perm], G, 2.0,
                          causal=causal)
    np.testing.assert_array_equal(o_a[:, :, q_perm], o_h)
    np.testing.assert_array_equal(l_a[:, q_perm], l_h)
    g_a = oracle.bwd(q, k, v, do, G, 2.0, causal=causal, shift="alternate")
    g_h = oracle.bwd(q[:, :, q_perm], k[:, :, kv_perm], v[:, :, kv_perm], do[:, :, q_perm], G,
                     2.0, causal=causal)
    np.testing.assert_array_equal(g_a[0][:, :, q_perm], g_h[0])
    np.testing.assert_array_equal(g_a[1][:, :, kv_perm], g_h[1])
    np.testing.assert_array_equal(g_a[2][:, :, kv_perm], g_h[2])


@pytest.mark.parametrize("Hq,Hkv", [(4, 4), (4, 2)])
def test_no_shift_one_group_is_dense_causal_on_every_head(Hq, Hkv):
    """Pattern "none" with G = N: every head is textbook dense causal attention (torch SDPA),
    the inference mode the guide's code falls back to ("Dual-Mode")."""
    N, d = 32, 8
    q, k, v, _ = _inputs(22, 1, N, Hq, Hkv, d)
    o, _ = oracle.fwd(q, k, v, G=N, s=2.0, shift="none")
    dense = ref.dense_causal(_t(q), _t(k), _t(v), 2.0).numpy()
    np.testing.assert_allclose(o, dense, atol=1e-12)


def test_no_shift_heads_are_block_diagonal():
    """Pattern "none", G < N: every head (also those the half pattern shifts) attends inside
    consecutive groups of its own rows only."""
    N, G, d = 64, 16, 8
    q, k, v, _ = _inputs(23, 1, N, 2, 2, d)
    o, _ = oracle.fwd(q, k, v, G=G, s=1.0, shift="none")
    qr = ref.rope_complex(_t(q), 1.0)
    kr = ref.rope_complex(_t(k), 1.0)
    for h in range(2):
        for g in range(N // G):
            sl = slice(g * G, (g + 1) * G)
            og = torch.nn.functional.scaled_dot_product_attention(
                qr[0, sl, h][None], kr[0, sl, h][None], _t(v)[0, sl, h][None], is_causal=True)
            np.testing.assert_allclose(o[0, sl, h], og[0].numpy(), atol=1e-12)


def test_roll_forward_then_back_is_identity():
    x = np.arange(40).reshape(1, 40, 1, 1)
    for G in (2, 8, 40):
        assert np.array_equal(np.roll(np.roll(x, -G // 2, axis=1), G // 2, axis=1), x)
        rows = np.concatenate([oracle.unit_rows(40, G, 2, 1, 2, g) for g in range(40 // G)])
        assert np.array_equal(np.sort(rows), np.arange(40))  # the roll is a bijection


def test_first_row_of_each_group_is_its_value_row():
    """Causal: local row 0 of every group sees one key, so O equals that token's v exactly."""
    N, G, d = 64, 16, 8
    q, k, v, _ = _inputs(9, 1, N, 4, 4, d)
    o, _ = oracle.fwd(q, k, v, G=G, s=2.0)
    for h in range(4):
        for g in range(N // G):
            t = oracle.unit_rows(N, G, 4, h, 4, g)[0]
            np.testing.assert_array_equal(o[0, t, h], v[0, t, h])


def test_lse_closed_forms():
    """LSE is the natural log of the sum of exp(q.k / sqrt(d)) over the visible keys.
    (1) Token 0 of an unshifted head sees only itself and RoPE at position 0 is the
    identity: LSE = q0.k0 / sqrt(d), computed here by hand. (2) With q = 0 every score is 0:
    local row i of a causal group sees i + 1 keys, so LSE = ln(i + 1) and O is the mean of
    the visible v rows; without the mask LSE = ln(G) on every row."""
    N, G, d, H = 64, 16, 8, 4
    q, k, v, _ = _inputs(31, 1, N, H, H, d)
    _, lse = oracle.fwd(q, k, v, G=G, s=2.0)
    for h in range(H // 2):   # unshifted heads
        assert lse[0, h, 0] == pytest.approx(float(q[0, 0, h] @ k[0, 0, h]) / math.sqrt(d),
                                             abs=1e-13)
    z = np.zeros_like(q)
    o, lse = oracle.fwd(z, k, v, G=G, s=2.0)
    for h in range(H):
        for g in range(N // G):
            rows = oracle.unit_rows(N, G, H, h, H, g)
            for i, t in enumerate(rows):
                assert lse[0, h, t] == pytest.approx(math.log(i + 1), abs=1e-13)
                np.testing.assert_allclose(o[0, t, h], v[0, rows[:i + 1], h].mean(axis=0),
                                           atol=1e-13)
    _, lse = oracle.fwd(z, k, v, G=G, s=2.0, causal=False)
    np.testing.assert_allclose(lse, math.log(G), atol=1e-13)


def test_output_in_convex_hull_of_visible_values():
    N, G, d = 64, 16, 8
    q, k, v, _ = _inputs(10, 1, N, 2, 2, d)
    o, _ = oracle.fwd(q, k, v, G=G, s=2.0)
    for h in range(2):
        for g in range(N // G):
            rows = oracle.unit_rows(N, G, 2, h, 2, g)
            for i, t in enumerate(rows):
                vis = v[0, rows[:i + 1], h]
                assert np.all(o[0, t, h] <= vis.max(0) + 1e-12)
                assert np.all(o[0, t, h] >= vis.min(0) - 1e-12)


def test_relative_position_invariance_across_groups():
    """With RoPE, a group whose rows repeat another group's rows at a constant offset gives
    the same outputs: input periodic with period G -> outputs periodic off the wrap group."""
    N, G, d = 64, 16, 8
    q, k, v, _ = _inputs(11, 1, N, 2, 2, d)
    for x in (q, k, v):
        for g in range(1, N // G):
            x[:, g * G:(g + 1) * G] = x[:, :G]
    o, _ = oracle.fwd(q, k, v, G=G, s=2.0)
    # unshifted head: every group equals group 0
    for g in range(1, N // G):
        np.testing.assert_allclose(o[0, g * G:(g + 1) * G, 0], o[0, :G, 0], atol=1e-12)
    # shifted head: non-wrap groups start at G/2 + gG
    a = o[0, G // 2:G // 2 + G, 1]
    for g in range(1, N // G - 1):
        b = o[0, G // 2 + g * G:G // 2 + (g + 1) * G, 1]
        np.testing.assert_allclose(b, a, atol=1e-12)


def test_gqa_equals_mha_with_repeated_kv_heads():
    N, G, d, Hq, Hkv = 32, 8, 8, 8, 2
    q, k, v, do = _inputs(12, 1, N, Hq, Hkv, d)
    R = Hq // Hkv
    kr, vr = np.repeat(k, R, axis=2), np.repeat(v, R, axis=2)
    o, lse = oracle.fwd(q, k, v, G=G, s=2.0)
    o2, lse2 = oracle.fwd(q, kr, vr, G=G, s=2.0)
    np.testing.assert_allclose(o, o2, atol=1e-13)
    np.testing.assert_allclose(lse, lse2, atol=1e-13)
    dq, dk, dv = oracle.bwd(q, k, v, do, G=G, s=2.0)
    dq2, dk2, dv2 = oracle.bwd(q, kr, vr, do, G=G, s=2.0)
    np.testing.assert_allclose(dq, dq2, atol=1e-12)
    np.testing.assert_allclose(dk, dk2.reshape(1, N, Hkv, R, d).sum(3), atol=1e-12)
    np.testing.assert_allclose(dv, dv2.reshape(1, N, Hkv, R, d).sum(3), atol=1e-12)


# ---------------------------------------------------------------- backward

@pytest.mark.parametrize("causal", [True, False])
def test_gradients_match_finite_differences(causal):
    """Central differences of L = sum(O * dO) match the oracle's analytic dq, dk, dv."""
    B, N, Hq, Hkv, d, G, s = 1, 16, 4, 2, 8, 8, 2.0
    q, k, v, do = _inputs(13, B, N, Hq, Hkv, d)
    dq, dk, dv = oracle.bwd(q, k, v, do, G=G, s=s, causal=causal)
    h = 1e-6

    def loss(q_, k_, v_):
        o, _ = oracle.fwd(q_, k_, v_, G=G, s=s, causal=causal)
        return float((o * do).sum())

    for name, x, g in (("q", q, dq), ("k", k, dk), ("v", v, dv)):
        num = np.empty_like(x)
        flat = x.reshape(-1)
        for idx in range(flat.size):
            old = flat[idx]
            flat[idx] = old + h
            lp = loss(q, k, v)
            flat[idx] = old - h
            lm = loss(q, k, v)
            flat[idx] = old
            num.reshape(-1)[idx] = (lp - lm) / (2 * h)
        err = np.abs(num - g).max() / np.abs(g).max()
        assert err < 1e-7, (name, err)


@pytest.mark.parametrize("B,N,Hq,Hkv,d,G", [(1, 64, 4, 4, 16, 16), (1, 64, 8, 2, 8, 32),
                                            (1, 256, 4, 4, 64, 64)])
def test_gradients_match_autograd_of_library_formulation(B, N, Hq, Hkv, d, G):
    q, k, v, do = _inputs(14, B, N, Hq, Hkv, d)
    tq, tk, tv = (_t(x).clone().requires_grad_(True) for x in (q, k, v))
    o = ref.s2attn(tq, tk, tv, G, 2.0)
    (o * _t(do)).sum().backward()
    dq, dk, dv = oracle.bwd(q, k, v, do, G=G, s=2.0)
    np.testing.assert_allclose(dq, tq.grad.numpy(), atol=1e-11)
    np.testing.assert_allclose(dk, tk.grad.numpy(), atol=1e-11)
    np.testing.assert_allclose(dv, tv.grad.numpy(), atol=1e-11)


def test_unit_functions_agree_with_full_functions():
    N, G, d, Hq, Hkv = 64, 16, 8, 8, 2
    q, k, v, do = _inputs(15, 2, N, Hq, Hkv, d)
    o, lse = oracle.fwd(q, k, v, G=G, s=2.0)
    dq, dk, dv = oracle.bwd(q, k, v, do, G=G, s=2.0)
    R = Hq // Hkv
    for b, kvh, g in ((0, 0, 0), (1, 1, N // G - 1), (0, 1, 1)):
        rows = oracle.unit_rows(N, G, Hq, kvh, Hkv, g)
        o_u, l_u = oracle.fwd_unit(q, k, v, G, 2.0, b, kvh, g)
        dq_u, dk_u, dv_u = oracle.bwd_unit(q, k, v, do, G, 2.0, b, kvh, g)
        for r in range(R):
            h = kvh * R + r
            np.testing.assert_array_equal(o_u[r], o[b, rows, h])
            np.testing.assert_array_equal(l_u[r], lse[b, h, rows])
            np.testing.assert_array_equal(dq_u[r], dq[b, rows, h])
        np.testing.assert_array_equal(dk_u, dk[b, rows, kvh])
        np.testing.assert_array_equal(dv_u, dv[b, rows, kvh])


@pytest.mark.parametrize("causal", [True, False])
def test_row_sampled_functions_agree_with_full_functions(causal):
    N, G, d, Hq, Hkv = 64, 16, 8, 8, 2
    q, k, v, do = _inputs(16, 2, N, Hq, Hkv, d)
    o, lse = oracle.fwd(q, k, v, G=G, s=2.0, causal=causal)
    dq, dk, dv = oracle.bwd(q, k, v, do, G=G, s=2.0, causal=causal)
    R = Hq // Hkv
    rows = np.array([0, 1, 7, 15, 3])
    for b, kvh, g in ((0, 0, 0), (1, 1, N // G - 1), (1, 1, 0)):
        tok = oracle.unit_rows(N, G, Hq, kvh, Hkv, g)[rows]
        for r in range(R):
            h = kvh * R + r
            o_r, l_r = oracle.fwd_rows(q, k, v, G, 2.0, b, h, g, rows, causal=causal)
            np.testing.assert_allclose(o_r, o[b, tok, h], rtol=0, atol=1e-14)
            np.testing.assert_allclose(l_r, lse[b, h, tok], rtol=0, atol=1e-14)
        dq_r, dk_r, dv_r = oracle.bwd_rows(q, k, v, do, G, 2.0, b, kvh, g, rows, rows[::-1],
                                           causal=causal)
        for r in range(R):
            np.testing.assert_allclose(dq_r[:, r], dq[b, tok, kvh * R + r], atol=1e-13)
        np.testing.assert_allclose(dk_r, dk[b, tok[::-1], kvh], atol=1e-13)
        np.testing.assert_allclose(dv_r, dv[b, tok[::-1], kvh], atol=1e-13)


def test_oracle_rejects_shapes_the_method_cannot_take():
    assert oracle.check(1, 64, 4, 4, 8, 16)
    assert not oracle.check(1, 60, 4, 4, 8, 16)   # N % G
    assert not oracle.check(1, 64, 3, 3, 8, 16)   # odd heads: no half split
    assert not oracle.check(1, 64, 4, 4, 8, 7)    # odd G: no G/2 shift
    assert not oracle.check(1, 64, 4, 3, 8, 16)   # Hq % Hkv
    assert not oracle.check(1, 16, 4, 4, 8, 32)   # G > N


# ---------------------------------------------------------------- FLOP model (worked example)

def _golden_flops():
    vals = {}
    with open(os.path.join(GOLDEN, "flop_counts.txt")) as f:
        for line in f:
            if "=" in line and not line.startswith("#"):
                key, val = line.strip().split("=")
                vals[key] = float(val)
    return vals


def test_flop_model_matches_pages_worked_example():
    from longlora_shifted_sparse_b200 import flops
    g = _golden_flops()
    L, G, D = int(g["L"]), int(g["G"]), int(g["D"])
    assert flops.toy_dense_ops(L, D) == int(g["dense_ops"])
    assert flops.toy_s2_ops(L, G, D) == int(g["s2_ops"])
    assert round((1 - flops.toy_s2_ops(L, G, D) / flops.toy_dense_ops(L, D)) * 100, 1) == \
        g["reduction_percent"]
    # The counted attention FLOPs scale the same way: dense / S2 = N / G, for any head split.
    for causal in (True, False):
        dense = flops.attention_fwd_flops(1, L, 8, D // 8, L, causal)
        s2 = flops.attention_fwd_flops(1, L, 8, D // 8, G, causal)
        assert dense / s2 == L / G


# ---------------------------------------------------------------- bf16 inputs (the format's definition)

def _bf16_by_definition(bits: int) -> float:
    """Value of a bfloat16 bit pattern from its fields alone: bfloat16 is the top half of an
    IEEE 754 binary32 (1 sign bit, 8 exponent bits with bias 127, 7 fraction bits), so a
    normal number is (-1)^s 2^(e-127) (1 + f/128) and a subnormal (-1)^s 2^(-126) (f/128).
    No bit reinterpretation is involved here."""
    s, e, f = bits >> 15, (bits >> 7) & 0xFF, bits & 0x7F
    assert e != 0xFF, "infinities and NaNs are not inputs of the method"
    mag = math.ldexp(1.0 + f / 128.0, e - 127) if e else math.ldexp(f / 128.0, -126)
    return -mag if s else mag


# Hand-decoded patterns: 1.0, -3.0, -0.0, the smallest subnormal 2^-133, the largest finite.
_BF16_PATTERNS = [(0x3F80, 1.0), (0xC040, -3.0), (0x8000, -0.0), (0x0001, 2.0 ** -133),
                  (0x7F7F, 3.3895313892515355e38)]


def test_bf16_decode_follows_the_binary32_definition():
    for bits, want in _BF16_PATTERNS:
        assert _bf16_by_definition(bits) == want
        got = float(synth.bf16_bits_to_f32(np.array([bits], dtype=np.uint16))[0])
        assert got == want and math.copysign(1.0, got) == math.copysign(1.0, want)
    finite = np.array([b for b in range(1 << 16) if (b >> 7) & 0xFF != 0xFF], dtype=np.uint16)
    want = np.array([_bf16_by_definition(int(b)) for b in finite])
    np.testing.assert_array_equal(synth.bf16_bits_to_f32(finite).astype(np.float64), want)


def test_oracle_reads_bf16_inputs_by_the_definition():
    """Local row 0 of a causal group sees one key, so O there is that token's v row exactly:
    the oracle's bf16 input path must hand v through unchanged. Row 0 of unshifted head 0 is
    token 0; with G = N = 2 row 0 of shifted head 1 is token 1 (rolled by -G/2)."""
    B, N, H, d, G = 1, 2, 2, 8, 2
    q, k, v, _ = synth.s2attn_inputs(17, B, N, H, H, d, 0.5, "bf16")
    pats = [b for b, _ in _BF16_PATTERNS] + [0x4049, 0xBE00, 0x0080]  # + 3.140625, -0.125, 2^-126
    v = v.copy()
    v[0, 0, 0, :] = pats
    v[0, 1, 1, :] = pats[::-1]
    o, _ = oracle.fwd(q, k, v, G=G, s=2.0)
    want = np.array([_bf16_by_definition(b) for b in pats])
    np.testing.assert_array_equal(o[0, 0, 0], want)
    np.testing.assert_array_equal(o[0, 1, 1], want[::-1])


@pytest.mark.parametrize("causal", [True, False])
def test_oracle_bf16_path_equals_decoded_fp64_inputs(causal):
    """The oracle reads bf16 bit patterns (every bf16 parity test) exactly as it reads the
    same values handed over in fp64: forward and backward agree bit for bit, GQA shape."""
    B, N, Hq, Hkv, d, G = 2, 48, 4, 2, 16, 16
    q, k, v, do = synth.s2attn_inputs(23, B, N, Hq, Hkv, d, 0.5, "bf16")
    dec = [synth.bf16_bits_to_f32(x).astype(np.float64) for x in (q, k, v, do)]
    o_b, lse_b = oracle.fwd(q, k, v, G=G, s=2.0, causal=causal)
    o_f, lse_f = oracle.fwd(*dec[:3], G=G, s=2.0, causal=causal)
    np.testing.assert_array_equal(o_b, o_f)
    np.testing.assert_array_equal(lse_b, lse_f)
    for gb, gf in zip(oracle.bwd(q, k, v, do, G=G, s=2.0, causal=causal),
                      oracle.bwd(*dec, G=G, s=2.0, causal=causal)):
        np.testing.assert_array_equal(gb, gf)
