"""Pins of the oracle's decode attention and low-plane selection.

The method's special cases reduce to textbook attention, which torch's
float64 ``scaled_dot_product_attention`` computes independently:
  * tau = 0: every token takes its full 4-bit value;
  * tau = +inf: every value is its high-plane midpoint;
  * 2-bit and bf16 cells: plain attention over the dequantised cache.
General tau is pinned by the decomposition o = attn(high) + sum over the
selected tokens of p_t * (full - high), with p from torch's softmax, and by
the invariants |S| <= 1/tau, S monotone in tau, o inside the value hull.
"""

import math

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle as O


def _bf16(rng, shape, scale=1.0):
    x = (rng.standard_normal(shape) * scale).astype(np.float32)
    return torch.from_numpy(x).to(torch.bfloat16).float().numpy()


def _case(seed, n=300, d=128, kind="q4", q_scale=1.0):
    rng = np.random.default_rng(seed)
    k = _bf16(rng, (n, d))
    k[:, rng.choice(d, 4, replace=False)] *= 10.0
    k = torch.from_numpy(k).to(torch.bfloat16).float().numpy()
    v = _bf16(rng, (n, d))
    q = _bf16(rng, (d,), q_scale)
    return q, k, v, O.StoredSequence(kind, k, v)


def _sdpa(q, k, v, sm_scale):
    t = lambda a: torch.from_numpy(np.asarray(a, np.float64))[None, None]
    return F.scaled_dot_product_attention(t(q)[:, :, None], t(k), t(v), scale=sm_scale)[0, 0, 0].numpy()


def _torch_p(q, k, sm_scale):
    s = torch.from_numpy(np.asarray(k, np.float64)) @ torch.from_numpy(np.asarray(q, np.float64))
    return torch.softmax(s * sm_scale, dim=0).numpy()


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_tau_zero_is_full_4bit_attention(seed):
    q, k, v, seq = _case(seed, q_scale=2.0)
    o, sel, _ = seq.attend(q, 0.0, 1.0)
    assert sel.all()
    ref = _sdpa(q, seq.qk.dequant(), seq.qv.dequant_full(), 1.0)
    np.testing.assert_allclose(o, ref, rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_tau_inf_is_high_plane_attention(seed):
    q, k, v, seq = _case(seed, q_scale=2.0)
    o, sel, _ = seq.attend(q, math.inf, 1.0)
    assert not sel.any()
    ref = _sdpa(q, seq.qk.dequant(), seq.qv.dequant_high(), 1.0)
    np.testing.assert_allclose(o, ref, rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("kind", ["q2", "bf16"])
def test_q2_and_bf16_are_plain_attention(kind):
    q, k, v, seq = _case(3, kind=kind, q_scale=0.5)
    o, sel, _ = seq.attend(q, 0.01, 0.7)
    assert not sel.any()
    if kind == "q2":
        ref = _sdpa(q, seq.qk.dequant(), seq.qv.dequant_full(), 0.7)
    else:
        ref = _sdpa(q, k, v, 0.7)
    np.testing.assert_allclose(o, ref, rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("tau", [1e-3, 1e-2, 5e-2])
def test_general_tau_decomposition(tau):
    q, k, v, seq = _case(4, n=517, q_scale=3.0)
    o, sel, p = seq.attend(q, tau, 1.0)
    kh, vf, vh = seq.qk.dequant(), seq.qv.dequant_full(), seq.qv.dequant_high()
    pt = _torch_p(q, kh, 1.0)
    np.testing.assert_allclose(p, pt, rtol=1e-12, atol=1e-15)
    want_sel = pt.astype(np.float32) >= np.float32(tau)
    np.testing.assert_array_equal(sel, want_sel)
    ref = _sdpa(q, kh, vh, 1.0) + (pt[want_sel, None] * (vf - vh)[want_sel]).sum(axis=0)
    np.testing.assert_allclose(o, ref, rtol=1e-10, atol=1e-12)
    assert 0 < sel.sum() < sel.size


def test_selection_invariants():
    q, k, v, seq = _case(5, n=1000, q_scale=4.0)
    prev = None
    for tau in [0.0, 1e-4, 1e-3, 3e-3, 1e-2, 5e-2, 0.2, 1.0, math.inf]:
        _, sel, _ = seq.attend(q, tau, 1.0)
        if 0 < tau < math.inf:
            assert sel.sum() <= math.floor(1 / tau)
        if prev is not None:
            assert np.all(sel <= prev)          # larger tau selects a subset
        prev = sel


def test_output_inside_value_hull():
    q, k, v, seq = _case(6, n=200, q_scale=2.0)
    o, sel, _ = seq.attend(q, 0.01, 1.0)
    vhat = np.where(sel[:, None], seq.qv.dequant_full(), seq.qv.dequant_high())
    assert np.all(o >= vhat.min(axis=0) - 1e-12) and np.all(o <= vhat.max(axis=0) + 1e-12)


def test_single_token_returns_its_full_value():
    q, k, v, seq = _case(7, n=1)
    o, sel, p = seq.attend(q, 0.5, 1.0)
    assert sel.tolist() == [True] and p.tolist() == [1.0]
    np.testing.assert_allclose(o, seq.qv.dequant_full()[0], rtol=0, atol=0)


def test_zero_query_is_uniform_average():
    q, k, v, seq = _case(8, n=64)
    q = np.zeros_like(q)
    o, sel, p = seq.attend(q, 1 / 64, 1.0)       # p = 1/64 >= tau: all selected
    assert sel.all()
    np.testing.assert_allclose(o, seq.qv.dequant_full().mean(axis=0), rtol=1e-12)
    o2, sel2, _ = seq.attend(q, 1 / 63, 1.0)     # p < tau: none selected
    assert not sel2.any()
    np.testing.assert_allclose(o2, seq.qv.dequant_high().mean(axis=0), rtol=1e-12)


def test_sm_scale_equals_scaled_query():
    q, k, v, seq = _case(9, n=100, kind="q2")
    o1, _, _ = seq.attend(q, 0.0, 0.25)
    o2, _, _ = seq.attend(q * np.float32(0.25), 0.0, 1.0)
    np.testing.assert_allclose(o1, o2, rtol=1e-12)


def test_empty_sequence_gives_zeros():
    o, sel, p = O.attend(np.ones(64), np.zeros((0, 64)), np.zeros((0, 64)), None, 0.1, 1.0)
    assert o.shape == (64,) and not o.any() and sel.size == 0


def test_reuse_reads_final_loop_with_own_query():
    rng = np.random.default_rng(10)
    L, N, H, B, n, d = 2, 2, 1, 1, 70, 64
    plan = ["reuse", "q2", "q4", "q4"]
    stored = {}
    for cell in (1, 2, 3):
        k, v = _bf16(rng, (n, d)), _bf16(rng, (n, d))
        stored[(cell, 0, 0)] = O.StoredSequence(plan[cell], k, v)
    q = _bf16(rng, (B, H, d), 2.0)
    got = O.decode_cell(plan, N, 0, stored, q, [n], 0.02, 1.0, pairs=[(0, 0)])[(0, 0)]
    want = stored[(2, 0, 0)].attend(q[0, 0], 0.02, 1.0)
    np.testing.assert_array_equal(got[0], want[0])
    np.testing.assert_array_equal(got[1], want[1])
    assert O.resolve_source(plan, 1, N) == 1
    with pytest.raises(ValueError):
        O.resolve_source(["q4", "reuse"], 1, 1)


def test_brute_force_tiny_loops():
    """Explicit scalar loops over tokens and channels (math.exp, Python
    floats) against the vectorised oracle on a tiny 4-bit case."""
    rng = np.random.default_rng(11)
    n, d, tau = 40, 32, 0.03
    k, v = _bf16(rng, (n, d)), _bf16(rng, (n, d))
    q = _bf16(rng, (d,), 2.0)
    seq = O.StoredSequence("q4", k, v)
    o, sel, _ = seq.attend(q, tau, 1.0)
    qk, qv = seq.qk, seq.qv
    logits = []
    for t in range(n):
        acc = 0.0
        for c in range(d):
            if t < 32:
                kv = float(qk.minv[0, c]) + float(qk.scale[0, c]) * int(qk.codes[t, c])
            else:
                kv = float(k[t, c])
            acc += float(q[c]) * kv
        logits.append(acc)
    m = max(logits)
    e = [math.exp(s - m) for s in logits]
    z = sum(e)
    out = [0.0] * d
    for t in range(n):
        p = e[t] / z
        take_low = np.float32(p) >= np.float32(tau)
        assert take_low == sel[t]
        for c in range(d):
            code = int(qv.codes[t, c])
            s, mn = float(qv.scale[t, 0]), float(qv.minv[t, 0])
            val = mn + s * (code if take_low else 4 * (code >> 2) + 1.5)
            out[c] += p * val
    np.testing.assert_allclose(o, out, rtol=1e-11, atol=1e-13)


def test_dequantised_cache_within_round_trip_bound():
    """Dequantised keys and values stay within the quantiser's closed-form
    error bound of the bf16 inputs (half a step, or the top overshoot)."""
    q, k, v, seq = _case(12, n=333, d=64)
    kh, vf = seq.qk.dequant(), seq.qv.dequant_full()
    ks = np.repeat(seq.qk.scale.astype(np.float64), 32, axis=0)      # [320, d]
    k_top = np.repeat((k[:320].reshape(10, 32, 64).max(axis=1)
                       - (seq.qk.minv + 15.0 * seq.qk.scale.astype(np.float64))), 32, axis=0)
    kb = np.maximum(ks / 2, k_top) * (1 + 1e-6) + 1e-6
    assert np.all(np.abs(kh[:320] - k[:320]) <= kb)
    np.testing.assert_array_equal(kh[320:], k[320:])
    vs = np.repeat(seq.qv.scale.astype(np.float64), 32, axis=1)
    v_top = np.repeat(v.reshape(333, 2, 32).max(axis=2)
                      - (seq.qv.minv + 15.0 * seq.qv.scale.astype(np.float64)), 32, axis=1)
    vb = np.maximum(vs / 2, v_top) * (1 + 1e-6) + 1e-6
    assert np.all(np.abs(vf - v) <= vb)


def test_high_plane_value_is_bucket_midpoint():
    """The high-plane-only value is the mean of the four full-precision
    values that share its high bits (unbiased for uniform low bits)."""
    q, k, v, seq = _case(13, n=50)
    qv = seq.qv
    s = np.repeat(qv.scale.astype(np.float64), 32, axis=1)
    m = np.repeat(qv.minv.astype(np.float64), 32, axis=1)
    hi = (qv.codes >> 2).astype(np.float64)
    bucket = np.mean([m + s * (4 * hi + lo) for lo in range(4)], axis=0)
    np.testing.assert_allclose(qv.dequant_high(), bucket, rtol=1e-15, atol=1e-15)
    assert np.all(np.abs(qv.dequant_full() - qv.dequant_high()) <= 1.5 * s + 1e-12)


# ---- coarser selection units (a granularity variant of the rule): pinned by
#      brute force over the units, nesting and the decomposition with torch

@pytest.mark.parametrize("unit", [16, 32])
@pytest.mark.parametrize("n", [1, 15, 16, 33, 517])
def test_unit_selection_is_any_token_of_the_unit(unit, n):
    q, k, v, seq = _case(7, n=n, q_scale=3.0)
    tau = 0.01
    _, tok, p = seq.attend(q, tau, 1.0)
    _, sel, _ = seq.attend(q, tau, 1.0, unit=unit)
    for t in range(n):
        u0 = (t // unit) * unit
        assert sel[t] == any(p[i].astype(np.float32) >= np.float32(tau) for i in range(u0, min(n, u0 + unit)))
    assert np.all(tok <= sel)


def test_units_nest_and_reduce_to_tokens():
    q, k, v, seq = _case(8, n=700, q_scale=4.0)
    for tau in [1e-3, 1e-2, 5e-2]:
        s1 = seq.attend(q, tau, 1.0)[1]
        s16 = seq.attend(q, tau, 1.0, unit=16)[1]
        s32 = seq.attend(q, tau, 1.0, unit=32)[1]
        assert np.all(s1 <= s16) and np.all(s16 <= s32)
        assert s32.sum() <= 32 * math.floor(1 / tau)
        np.testing.assert_array_equal(s1, seq.attend(q, tau, 1.0, unit=1)[1])
    for unit in (16, 32):
        assert seq.attend(q, 0.0, 1.0, unit=unit)[1].all()
        assert not seq.attend(q, math.inf, 1.0, unit=unit)[1].any()


@pytest.mark.parametrize("unit", [16, 32])
def test_unit_selection_decomposition(unit):
    q, k, v, seq = _case(9, n=300, q_scale=3.0)
    o, sel, _ = seq.attend(q, 0.01, 1.0, unit=unit)
    kh, vf, vh = seq.qk.dequant(), seq.qv.dequant_full(), seq.qv.dequant_high()
    pt = _torch_p(q, kh, 1.0)
    ref = _sdpa(q, kh, vh, 1.0) + (pt[sel, None] * (vf - vh)[sel]).sum(axis=0)
    np.testing.assert_allclose(o, ref, rtol=1e-10, atol=1e-12)


# ---- grouped queries (several query heads per KV head): the low plane of a
#      token is fetched when any head of the group selects it and then serves
#      every head.  Pinned by torch's attention per head, brute force over
#      the heads, the per-head bound |S_h| <= 1/tau and special cases.

def _queries(seed, g, d=128, scale=3.0):
    rng = np.random.default_rng(seed)
    return np.stack([_bf16(rng, (d,), scale) for _ in range(g)])


@pytest.mark.parametrize("kind", ["q4", "q2", "bf16"])
def test_grouped_single_head_is_attend(kind):
    q, k, v, seq = _case(21, n=257, kind=kind, q_scale=3.0)
    o, sel, p = seq.attend_grouped(q[None], 0.01, 1.0)
    o1, sel1, p1 = seq.attend(q, 0.01, 1.0)
    np.testing.assert_array_equal(o[0], o1)
    np.testing.assert_array_equal(sel, sel1)
    np.testing.assert_array_equal(p[0], p1)


@pytest.mark.parametrize("g", [2, 4, 8])
@pytest.mark.parametrize("unit", [1, 16, 32])
def test_grouped_union_decomposition(g, unit):
    """Each head: torch attention over the high-plane values plus, over the
    union of the heads' own selections, p_h(t) (full - high); the union is
    brute-forced token by token from torch's weights."""
    q, k, v, seq = _case(22, n=300)
    qs = _queries(23, g)
    tau = 0.01
    o, sel, p = seq.attend_grouped(qs, tau, 1.0, unit=unit)
    kh, vf, vh = seq.qk.dequant(), seq.qv.dequant_full(), seq.qv.dequant_high()
    pt = [_torch_p(qs[h], kh, 1.0) for h in range(g)]
    want = np.zeros(300, dtype=bool)
    for t in range(300):
        u0 = (t // unit) * unit
        want[t] = any(np.float32(pt[h][i]) >= np.float32(tau)
                      for h in range(g) for i in range(u0, min(300, u0 + unit)))
    np.testing.assert_array_equal(sel, want)
    for h in range(g):
        ref = _sdpa(qs[h], kh, vh, 1.0) + (pt[h][sel, None] * (vf - vh)[sel]).sum(axis=0)
        np.testing.assert_allclose(o[h], ref, rtol=1e-10, atol=1e-12)


def test_grouped_brute_force_tiny_loops():
    """Scalar loops (math.exp, Python floats) over heads, tokens and channels
    on a tiny 4-bit case with three query heads."""
    rng = np.random.default_rng(24)
    n, d, g, tau = 40, 32, 3, 0.04
    k, v = _bf16(rng, (n, d)), _bf16(rng, (n, d))
    qs = np.stack([_bf16(rng, (d,), 2.0) for _ in range(g)])
    seq = O.StoredSequence("q4", k, v)
    o, sel, _ = seq.attend_grouped(qs, tau, 1.0)
    qk, qv = seq.qk, seq.qv
    key = [[(float(qk.minv[0, c]) + float(qk.scale[0, c]) * int(qk.codes[t, c])) if t < 32 else float(k[t, c])
            for c in range(d)] for t in range(n)]
    probs = []
    for h in range(g):
        logits = [sum(float(qs[h][c]) * key[t][c] for c in range(d)) for t in range(n)]
        m = max(logits)
        e = [math.exp(s - m) for s in logits]
        z = sum(e)
        probs.append([x / z for x in e])
    union = [any(np.float32(probs[h][t]) >= np.float32(tau) for h in range(g)) for t in range(n)]
    assert list(sel) == union
    for h in range(g):
        out = [0.0] * d
        for t in range(n):
            for c in range(d):
                code = int(qv.codes[t, c])
                s, mn = float(qv.scale[t, 0]), float(qv.minv[t, 0])
                out[c] += probs[h][t] * (mn + s * (code if union[t] else 4 * (code >> 2) + 1.5))
        np.testing.assert_allclose(o[h], out, rtol=1e-11, atol=1e-13)


def test_grouped_special_cases_and_bounds():
    q, k, v, seq = _case(25, n=400, q_scale=3.0)
    qs = _queries(26, 4)
    kh, vf, vh = seq.qk.dequant(), seq.qv.dequant_full(), seq.qv.dequant_high()
    # tau = 0: full 4-bit values for every head; tau = inf: midpoints
    o0, s0, _ = seq.attend_grouped(qs, 0.0, 1.0)
    oi, si, _ = seq.attend_grouped(qs, math.inf, 1.0)
    assert s0.all() and not si.any()
    for h in range(4):
        np.testing.assert_allclose(o0[h], _sdpa(qs[h], kh, vf, 1.0), rtol=1e-10, atol=1e-12)
        np.testing.assert_allclose(oi[h], _sdpa(qs[h], kh, vh, 1.0), rtol=1e-10, atol=1e-12)
    for tau in [1e-3, 1e-2, 5e-2]:
        _, sel, _ = seq.attend_grouped(qs, tau, 1.0)
        own = [seq.attend(qs[h], tau, 1.0)[1] for h in range(4)]
        # the union holds every head's own set and at most G / tau tokens
        assert all(np.all(s <= sel) for s in own)
        assert sel.sum() <= 4 * math.floor(1 / tau)
        np.testing.assert_array_equal(sel, np.logical_or.reduce(own))
    # identical queries: the union is that head's own selection
    same = np.stack([qs[0]] * 3)
    o, sel, _ = seq.attend_grouped(same, 0.01, 1.0)
    o1, sel1, _ = seq.attend(qs[0], 0.01, 1.0)
    np.testing.assert_array_equal(sel, sel1)
    for h in range(3):
        np.testing.assert_array_equal(o[h], o1)
    # 2-bit and bf16 sources select nothing, whatever the group
    for kind in ("q2", "bf16"):
        _, _, _, s2 = _case(25, n=50, kind=kind)
        assert not s2.attend_grouped(_queries(27, 2), 0.01, 1.0)[1].any()
    # an empty sequence gives zeros for every head
    e = O.attend_grouped(qs, np.zeros((0, 128)), np.zeros((0, 128)), np.zeros((0, 128)), 0.01, 1.0)
    assert e[0].shape == (4, 128) and not e[0].any() and e[1].size == 0


# ---- the current token of a reuse cell's own loop: one exact extra entry of
#      the softmax after the stored tokens (no low plane).  Pinned by torch's
#      attention over the concatenated cache, the decomposition with torch's
#      softmax over n + 1 tokens, scalar loops and the one-token case.

def _current(seed, d=128, scale=1.0):
    rng = np.random.default_rng(seed)
    return _bf16(rng, (d,), scale), _bf16(rng, (d,))


@pytest.mark.parametrize("kind", ["q4", "q2", "bf16"])
@pytest.mark.parametrize("tau", [0.0, math.inf])
def test_current_token_limits_are_attention_over_concatenation(kind, tau):
    q, k, v, seq = _case(31, n=211, kind=kind, q_scale=2.0)
    kc, vc = _current(32, scale=3.0)
    o, sel, p = seq.attend(q, tau, 1.0, k_cur=kc, v_cur=vc)
    assert sel.size == 211 and p.size == 212
    if kind == "bf16":
        kh, vx = k, v
    else:
        kh = seq.qk.dequant()
        vx = seq.qv.dequant_full() if (kind == "q2" or tau == 0.0) else seq.qv.dequant_high()
    ref = _sdpa(q, np.vstack([kh, kc[None]]), np.vstack([vx, vc[None]]), 1.0)
    np.testing.assert_allclose(o, ref, rtol=1e-12, atol=1e-12)
    if kind == "q4":
        assert sel.all() == (tau == 0.0) and (not sel.any()) == (tau == math.inf)


@pytest.mark.parametrize("tau", [1e-3, 1e-2, 5e-2])
def test_current_token_general_tau_decomposition(tau):
    q, k, v, seq = _case(33, n=400, q_scale=3.0)
    kc, vc = _current(34, scale=2.0)
    o, sel, p = seq.attend(q, tau, 1.0, k_cur=kc, v_cur=vc)
    kh, vf, vh = seq.qk.dequant(), seq.qv.dequant_full(), seq.qv.dequant_high()
    keys = np.vstack([kh, kc[None]])
    pt = _torch_p(q, keys, 1.0)
    np.testing.assert_allclose(p, pt, rtol=1e-12, atol=1e-15)
    want = pt[:400].astype(np.float32) >= np.float32(tau)
    np.testing.assert_array_equal(sel, want)
    ref = _sdpa(q, keys, np.vstack([vh, vc[None]]), 1.0) + (pt[:400][want, None] * (vf - vh)[want]).sum(axis=0)
    np.testing.assert_allclose(o, ref, rtol=1e-10, atol=1e-12)
    # the extra entry takes weight: the stored tokens' weights sum to 1 - p_cur
    assert 0 < p[400] < 1 and abs(p[:400].sum() + p[400] - 1) < 1e-12


def test_current_token_alone_is_its_value():
    o, sel, p = O.attend(np.ones(64), np.zeros((0, 64)), np.zeros((0, 64)), np.zeros((0, 64)), 0.01, 1.0,
                         k_cur=np.full(64, 0.5), v_cur=np.arange(64.0))
    assert sel.size == 0 and p.tolist() == [1.0]
    np.testing.assert_array_equal(o, np.arange(64.0))


def test_current_token_brute_force_tiny_loops():
    """Scalar loops (math.exp, Python floats) over the stored tokens and the
    current one on a tiny 4-bit case."""
    rng = np.random.default_rng(35)
    n, d, tau = 37, 32, 0.03
    k, v = _bf16(rng, (n, d)), _bf16(rng, (n, d))
    q = _bf16(rng, (d,), 2.0)
    kc, vc = _bf16(rng, (d,), 2.0), _bf16(rng, (d,))
    seq = O.StoredSequence("q4", k, v)
    o, sel, _ = seq.attend(q, tau, 1.0, k_cur=kc, v_cur=vc)
    qk, qv = seq.qk, seq.qv
    logits = []
    for t in range(n):
        acc = 0.0
        for c in range(d):
            kv = float(qk.minv[0, c]) + float(qk.scale[0, c]) * int(qk.codes[t, c]) if t < 32 else float(k[t, c])
            acc += float(q[c]) * kv
        logits.append(acc)
    logits.append(sum(float(q[c]) * float(kc[c]) for c in range(d)))
    m = max(logits)
    e = [math.exp(s - m) for s in logits]
    z = sum(e)
    out = [0.0] * d
    for t in range(n):
        p = e[t] / z
        take_low = np.float32(p) >= np.float32(tau)
        assert take_low == sel[t]
        for c in range(d):
            code = int(qv.codes[t, c])
            s, mn = float(qv.scale[t, 0]), float(qv.minv[t, 0])
            out[c] += p * (mn + s * (code if take_low else 4 * (code >> 2) + 1.5))
    for c in range(d):
        out[c] += e[n] / z * float(vc[c])
    np.testing.assert_allclose(o, out, rtol=1e-11, atol=1e-13)


@pytest.mark.parametrize("g", [2, 4])
def test_current_token_grouped_union(g):
    q, k, v, seq = _case(36, n=300)
    qs = _queries(37, g)
    kc, vc = _current(38, scale=3.0)
    tau = 0.01
    o, sel, p = seq.attend_grouped(qs, tau, 1.0, k_cur=kc, v_cur=vc)
    kh, vf, vh = seq.qk.dequant(), seq.qv.dequant_full(), seq.qv.dequant_high()
    keys = np.vstack([kh, kc[None]])
    pt = [_torch_p(qs[h], keys, 1.0) for h in range(g)]
    want = np.array([any(np.float32(pt[h][t]) >= np.float32(tau) for h in range(g)) for t in range(300)])
    np.testing.assert_array_equal(sel, want)
    for h in range(g):
        ref = _sdpa(qs[h], keys, np.vstack([vh, vc[None]]), 1.0) + (pt[h][:300][sel, None] * (vf - vh)[sel]).sum(0)
        np.testing.assert_allclose(o[h], ref, rtol=1e-10, atol=1e-12)
    # one head: the grouped form is the single-query form
    o1, s1, p1 = seq.attend(qs[0], tau, 1.0, k_cur=kc, v_cur=vc)
    og, sg, pg = seq.attend_grouped(qs[:1], tau, 1.0, k_cur=kc, v_cur=vc)
    np.testing.assert_array_equal(o1, og[0])
    np.testing.assert_array_equal(s1, sg)


def test_reuse_cell_attends_the_current_token():
    rng = np.random.default_rng(39)
    N, n, d = 2, 70, 64
    plan = ["reuse", "q2", "q4", "q4"]
    stored = {(c, 0, 0): O.StoredSequence(plan[c], _bf16(rng, (n, d)), _bf16(rng, (n, d))) for c in (1, 2, 3)}
    q = _bf16(rng, (1, 1, d), 2.0)
    kc, vc = _bf16(rng, (d,), 2.0), _bf16(rng, (d,))
    got = O.decode_cell(plan, N, 0, stored, q, [n], 0.02, 1.0, pairs=[(0, 0)], current={(0, 0): (kc, vc)})
    want = stored[(2, 0, 0)].attend(q[0, 0], 0.02, 1.0, k_cur=kc, v_cur=vc)
    for a, b in zip(got[(0, 0)], want):
        np.testing.assert_array_equal(a, b)
    plain = stored[(2, 0, 0)].attend(q[0, 0], 0.02, 1.0)
    assert not np.allclose(got[(0, 0)][0], plain[0])
