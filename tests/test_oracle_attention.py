"""Pins of the oracle's attention values.

The pages print no numeric example, so the oracle is checked against a
library routine (torch's scaled_dot_product_attention on the CPU), closed
forms, and the invariants the rule implies ([picx] "Action-Aware Causal
Attention (Figure 6b)"): full bidirectional attention when every window
spans the segment, independence from dead tails and later segments, from
tails whose window excludes the query's frame, and from the order of keys.
"""
import math

import numpy as np
import pytest
import torch

from oracle import attention as oattn
from oracle import rule as orule
from segment_causal_masked_b200 import workloads as W


def _inputs(problem, seed, q_scale=1.0):
    t = W.make_inputs(problem, seed, q_scale)
    q = t["q"].float().numpy()
    k = torch.cat([t["cache_k"], t["k_cur"]]).float().numpy()
    v = torch.cat([t["cache_v"], t["v_cur"]]).float().numpy()
    return q, k, v


def _sdpa(q, k, v, mask, scale):
    qt = torch.from_numpy(np.ascontiguousarray(q.transpose(1, 0, 2))).double()
    kt = torch.from_numpy(np.ascontiguousarray(k.transpose(1, 0, 2))).double()
    vt = torch.from_numpy(np.ascontiguousarray(v.transpose(1, 0, 2))).double()
    o = torch.nn.functional.scaled_dot_product_attention(
        qt, kt, vt, attn_mask=torch.from_numpy(mask), scale=scale)
    return o.numpy().transpose(1, 0, 2)


@pytest.mark.parametrize("problem", [W.tiny_packed(), W.small_session(), W.small_packed()])
@pytest.mark.parametrize("q_scale", [1.0, 8.0])
def test_matches_torch_sdpa(problem, q_scale):
    lay = orule.Layout.of(problem)
    q, k, v = _inputs(problem, 5, q_scale)
    o, lse = oattn.attention(lay, q, k, v, problem.softmax_scale)
    ref = _sdpa(q, k, v, lay.mask(), problem.softmax_scale)
    assert np.abs(o - ref).max() < 1e-12
    # LSE against a direct log-sum-exp over the visible scores
    m = lay.mask()
    for h in range(problem.heads):
        s = (q[:, h, :].astype(np.float64) @ k[:, h, :].T.astype(np.float64)) * problem.softmax_scale
        s = np.where(m, s, -np.inf)
        ref_lse = np.log(np.exp(s - s.max(1, keepdims=True)).sum(1)) + s.max(1)
        assert np.abs(lse[h] - ref_lse).max() < 1e-10


def test_float32_agrees_with_float64():
    p = W.small_session()
    lay = orule.Layout.of(p)
    q, k, v = _inputs(p, 6)
    o64, l64 = oattn.attention(lay, q, k, v, p.softmax_scale)
    o32, l32 = oattn.attention(lay, q, k, v, p.softmax_scale, dtype=np.float32)
    assert np.abs(o64 - o32).max() < 1e-5
    assert np.abs(l64 - l32).max() < 1e-4


# ---------------------------------------------------------------------------
# closed forms
# ---------------------------------------------------------------------------

def test_zero_queries_give_mean_of_visible_values():
    """Q = 0 makes every visible score 0: O is the plain mean of the visible
    V rows and LSE = log(count). Visible sets are the hand-derived ones."""
    p = W.tiny_packed()
    lay = orule.Layout.of(p)
    q, k, v = _inputs(p, 7)
    q[:] = 0.0
    o, lse = oattn.attention(lay, q, k, v, p.softmax_scale)
    # seg1 head query (row 130) sees keys [80,144); seg1 video frame1 (row 110)
    # sees [0,64) + [80,144) + [152,160)
    np.testing.assert_allclose(o[130], v[80:144].astype(np.float64).mean(0), atol=1e-12)
    sel = np.r_[0:64, 80:144, 152:160]
    np.testing.assert_allclose(o[110], v[sel].astype(np.float64).mean(0), atol=1e-12)
    np.testing.assert_allclose(lse[:, 130], math.log(64), atol=1e-12)
    np.testing.assert_allclose(lse[:, 110], math.log(136), atol=1e-12)


def test_constant_values_are_reproduced():
    p = W.small_packed()
    lay = orule.Layout.of(p)
    q, k, v = _inputs(p, 8, 4.0)
    c = np.random.default_rng(0).standard_normal(v.shape[1:])
    v[:] = c[None]                                   # rounded to the float32 array
    o, _ = oattn.attention(lay, q, k, v, p.softmax_scale)
    assert np.abs(o - v[:1].astype(np.float64)).max() < 1e-12


def test_single_visible_key():
    """A one-token segment with no text: its only query sees only itself."""
    p = W.Problem("one", (), (W.Segment(1, 1, 0),), heads=2)
    lay = orule.Layout.of(p)
    q, k, v = _inputs(p, 9)
    o, lse = oattn.attention(lay, q, k, v, p.softmax_scale)
    assert np.array_equal(o[0], v[0].astype(np.float64))
    s = (q[0].astype(np.float64) * k[0].astype(np.float64)).sum(-1) * p.softmax_scale
    np.testing.assert_allclose(lse[:, 0], s, atol=1e-12)


# ---------------------------------------------------------------------------
# invariants
# ---------------------------------------------------------------------------

def _full_span_segment():
    return W.Segment(3, 20, 7, (W.Action(5, 0, 3), W.Action(9, 0, 3), W.Action(4, 0, 3)))


@pytest.mark.parametrize("policy", [W.TEXTQ_OWN_TAIL, W.TEXTQ_FULL_SEGMENT])
def test_full_window_segment_is_full_bidirectional(policy):
    p = W.Problem("full", (), (_full_span_segment(),), heads=3, textq_policy=policy)
    lay = orule.Layout.of(p)
    q, k, v = _inputs(p, 10)
    o, _ = oattn.attention(lay, q, k, v, p.softmax_scale)
    ref = _sdpa(q, k, v, np.ones((lay.n_queries, lay.n_keys), bool), p.softmax_scale)
    rows = np.arange(lay.n_queries) if policy == W.TEXTQ_FULL_SEGMENT else np.arange(60)
    assert np.abs(o[rows] - ref[rows]).max() < 1e-12
    if policy == W.TEXTQ_OWN_TAIL:        # head rows do not see the tails
        assert np.abs(o[60:67] - ref[60:67]).max() > 1e-3


def test_dead_tails_and_later_segments_do_not_matter():
    p = W.small_session()
    lay = orule.Layout.of(p)
    q, k, v = _inputs(p, 11)
    o, l = oattn.attention(lay, q, k, v, p.softmax_scale)
    k2, v2 = k.copy(), v.copy()
    for sp in lay.spans[:len(p.cached)]:            # every cached tail
        for a, b in sp.tails:
            k2[a:b] = 100.0
            v2[a:b] = -100.0
    o2, l2 = oattn.attention(lay, q, k2, v2, p.softmax_scale)
    assert np.array_equal(o, o2) and np.array_equal(l, l2)

    pk = W.small_packed()
    lay = orule.Layout.of(pk)
    q, k, v = _inputs(pk, 12)
    o, _ = oattn.attention(lay, q, k, v, pk.softmax_scale)
    cut = lay.spans[3].stop                          # perturb segments 4, 5
    k2, v2 = k.copy(), v.copy()
    k2[cut:] *= -3.0
    v2[cut:] += 1.0
    o2, _ = oattn.attention(lay, q, k2, v2, pk.softmax_scale)
    assert np.array_equal(o[:cut], o2[:cut])
    assert not np.array_equal(o[cut:], o2[cut:])


def test_frame_outside_window_ignores_tail():
    seg = W.Segment(4, 6, 3, (W.Action(5, 1, 3), W.Action(2, 0, 4)))
    p = W.Problem("win", (), (seg,), heads=2)
    lay = orule.Layout.of(p)
    q, k, v = _inputs(p, 13)
    o, _ = oattn.attention(lay, q, k, v, p.softmax_scale)
    a0 = lay.spans[0].tails[0]
    k2, v2 = k.copy(), v.copy()
    k2[a0[0]:a0[1]] += 5.0
    v2[a0[0]:a0[1]] -= 5.0
    o2, _ = oattn.attention(lay, q, k2, v2, p.softmax_scale)
    for f in range(4):
        rows = slice(6 * f, 6 * f + 6)
        if 1 <= f < 3:
            assert not np.array_equal(o[rows], o2[rows])
        else:
            assert np.array_equal(o[rows], o2[rows])


def test_key_permutation_within_visible_set():
    p = W.small_session()
    lay = orule.Layout.of(p)
    q, k, v = _inputs(p, 14)
    m = lay.mask()
    perm = np.random.default_rng(1).permutation(lay.n_keys)
    for h in range(p.heads):
        o, l = oattn.masked_attention(q[:, h], k[:, h], v[:, h], m, p.softmax_scale)
        o2, l2 = oattn.masked_attention(q[:, h], k[perm, h], v[perm, h], m[:, perm],
                                        p.softmax_scale)
        assert np.abs(o - o2).max() < 1e-12 and np.abs(l - l2).max() < 1e-12


def test_fully_masked_row_is_zero():
    q = np.ones((2, 4)); k = np.ones((3, 4)); v = np.ones((3, 4))
    mask = np.array([[True, False, False], [False, False, False]])
    o, lse = oattn.masked_attention(q, k, v, mask, 0.5)
    assert np.array_equal(o[1], np.zeros(4)) and lse[1] == -np.inf
    assert np.array_equal(o[0], np.ones(4))
