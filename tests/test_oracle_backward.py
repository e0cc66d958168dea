"""Pins of the oracle's attention gradients (oracle/backward.py).

Independent of the oracle's formulas: torch autograd through
scaled_dot_product_attention (a library routine), central finite differences
of the forward oracle (a different module), and identities that hold for any
softmax attention.
"""
import numpy as np
import pytest
import torch

from oracle import attention as oattn
from oracle import backward as obwd
from oracle import rule as orule
from segment_causal_masked_b200 import workloads as W


def _inputs(p, seed, q_scale=1.0):
    inp = W.make_inputs(p, seed, q_scale)
    q = inp["q"].double().numpy()
    k = torch.cat([inp["cache_k"], inp["k_cur"]]).double().numpy()
    v = torch.cat([inp["cache_v"], inp["v_cur"]]).double().numpy()
    rng = np.random.default_rng(seed + 17)
    d_o = rng.standard_normal(q.shape)
    return q, k, v, d_o


LAYOUTS = [W.tiny_packed(), W.small_session(heads=2),
           W.Problem("small-packed", (), W.small_packed(seed=3, n_segments=4).current, heads=2)]


@pytest.mark.parametrize("q_scale", [1.0, 6.0])
@pytest.mark.parametrize("p", LAYOUTS, ids=lambda p: p.name)
def test_matches_torch_autograd(p, q_scale):
    q, k, v, d_o = _inputs(p, 5, q_scale)
    lay = orule.Layout.of(p)
    dq, dk, dv = obwd.attention_backward(lay, q, k, v, d_o, p.softmax_scale)
    mask = torch.from_numpy(lay.mask())
    tq, tk, tv = (torch.from_numpy(np.ascontiguousarray(a.transpose(1, 0, 2))).requires_grad_()
                  for a in (q, k, v))
    o = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, attn_mask=mask,
                                                         scale=p.softmax_scale)
    o.backward(torch.from_numpy(np.ascontiguousarray(d_o.transpose(1, 0, 2))))
    for mine, ref in ((dq, tq.grad), (dk, tk.grad), (dv, tv.grad)):
        ref = ref.numpy().transpose(1, 0, 2)
        assert np.allclose(mine, ref, rtol=1e-9, atol=1e-11), np.abs(mine - ref).max()


def test_central_differences_of_the_forward_oracle():
    p = W.tiny_packed()
    q, k, v, d_o = _inputs(p, 6, 2.0)
    lay = orule.Layout.of(p)
    dq, dk, dv = obwd.attention_backward(lay, q, k, v, d_o, p.softmax_scale)

    def loss(qq, kk, vv):
        o, _ = oattn.attention(lay, qq, kk, vv, p.softmax_scale)
        return float((o * d_o).sum())

    rng = np.random.default_rng(0)
    eps = 1e-6
    for name, arr, grad in (("q", q, dq), ("k", k, dk), ("v", v, dv)):
        for _ in range(12):
            idx = tuple(int(rng.integers(0, n)) for n in arr.shape)
            plus, minus = arr.copy(), arr.copy()
            plus[idx] += eps
            minus[idx] -= eps
            args = {"q": q, "k": k, "v": v}
            fp = loss(*[plus if n == name else args[n] for n in ("q", "k", "v")])
            fm = loss(*[minus if n == name else args[n] for n in ("q", "k", "v")])
            fd = (fp - fm) / (2 * eps)
            assert abs(fd - grad[idx]) <= 1e-6 * max(1.0, abs(fd)), (name, idx, fd, grad[idx])


def test_identities():
    """Σ_k dK_k = 0 (each row of dS sums to zero); Σ_k dV_k = Σ_q dO_q (each
    row of P sums to one); keys no query sees (dead cached tails) get zero
    gradients; dO = 0 gives zero gradients."""
    p = W.small_session(heads=2)
    q, k, v, d_o = _inputs(p, 7, 3.0)
    lay = orule.Layout.of(p)
    dq, dk, dv = obwd.attention_backward(lay, q, k, v, d_o, p.softmax_scale)
    assert np.abs(dk.sum(axis=0)).max() <= 1e-10 * np.abs(dk).sum()
    assert np.allclose(dv.sum(axis=0), d_o.sum(axis=0), rtol=1e-10, atol=1e-10)
    unseen = ~lay.mask().any(axis=0)
    assert unseen.sum() > 0
    assert not dk[unseen].any() and not dv[unseen].any()
    z = obwd.attention_backward(lay, q, k, v, np.zeros_like(d_o), p.softmax_scale)
    assert all(not a.any() for a in z)


def test_sampled_rows_equal_full_rows():
    p = LAYOUTS[2]
    q, k, v, d_o = _inputs(p, 8)
    lay = orule.Layout.of(p)
    dq, _, _ = obwd.attention_backward(lay, q, k, v, d_o, p.softmax_scale)
    rows = [0, 5, p.n_query_tokens - 1]
    part = obwd.dq_rows(lay, q, k, v, d_o, rows, p.softmax_scale, heads=[1])
    assert np.allclose(part[:, 0], dq[rows, 1], rtol=1e-12, atol=1e-14)
