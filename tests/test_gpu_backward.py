"""GPU parity of the attention backward (dQ, dK, dV) against the oracle.

The CUDA forward gives O and LSE; the backward consumes them with an upstream
gradient dO drawn here. Expected values come from the oracle's gradients of
the same bf16 inputs (it recomputes P in float64 from q, k, v alone).

Bar (derived from the arithmetic, not stated by the pages): P and dS are
rounded to bf16 before their products (2^-9 relative each), the outputs are
bf16 (2^-9), accumulation is fp32; the relative L2 error of each gradient
must stay under 2e-2 and every element within 2e-2 of the reference scaled by
the gradient's largest magnitude. At full size, where the oracle cannot
produce dK and dV, sampled dQ rows are compared and two identities of any
softmax attention are checked on the whole result: Σ_keys dK = 0 and
Σ_keys dV = Σ_queries dO.
"""
import numpy as np
import pytest
import torch

from oracle import backward as obwd
from oracle import rule as orule
from segment_causal_masked_b200 import workloads as W

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

from segment_causal_masked_b200 import sca  # noqa: E402
from tests.gpu_session import GpuSession  # noqa: E402


class Bwd:
    """Forward + backward of a cacheless layout on the GPU."""

    def __init__(self, p, seed, q_scale=1.0):
        self.p = p
        self.inputs = W.make_inputs(p, seed, q_scale)
        g = torch.Generator().manual_seed(seed + 99)
        self.d_o_cpu = torch.randn(p.n_query_tokens, p.heads, 128, generator=g).bfloat16()
        self.s = GpuSession(p, self.inputs)
        self.o, self.lse = self.s.forward()
        self.d_o = self.d_o_cpu.cuda()

    def backward(self):
        p, s = self.p, self.s
        dq, dk, dv = (torch.full_like(s.q, float("nan")) for _ in range(3))
        ws = torch.empty(sca.attn_bwd_workspace_bytes(s.md, p.heads), dtype=torch.uint8,
                         device="cuda")
        sca.action_causal_attn_bwd(s.md, p.heads, s.q, s.k_cur, s.v_cur, self.o, self.lse,
                                   self.d_o, dq, dk, dv, p.softmax_scale, ws, None, s.status)
        torch.cuda.synchronize()
        assert int(s.status.item()) == 0
        return dq, dk, dv

    def oracle_inputs(self):
        f = lambda t: t.float().numpy()  # noqa: E731
        return (f(self.inputs["q"]), f(self.inputs["k_cur"]), f(self.inputs["v_cur"]),
                f(self.d_o_cpu))


def _check(name, got, ref):
    g = got.float().cpu().numpy().astype(np.float64)
    assert np.isfinite(g).all(), name
    scale = max(np.abs(ref).max(), 1e-30)
    rel = np.linalg.norm(g - ref) / max(np.linalg.norm(ref), 1e-30)
    worst = np.abs(g - ref).max() / scale
    assert rel <= 2e-2, f"{name}: relative L2 {rel:.3g}"
    assert worst <= 2e-2, f"{name}: max |d| / max |ref| = {worst:.3g}"
    return rel, worst


def _packed(name, seed, n_segments, heads=2, **kw):
    return W.Problem(name, (), W.small_packed(seed=seed, n_segments=n_segments).current,
                     heads=heads, **kw)


SMALL = [W.tiny_packed(),
         _packed("packed-4", 3, 4),
         _packed("packed-9", 21, 9, heads=3),
         _packed("packed-9-full", 21, 9, textq_policy=W.TEXTQ_FULL_SEGMENT),
         W.Problem("one-segment", (), (W.Segment(5, 60, 9, (W.Action(7, 0, 2), W.Action(5, 1, 5))),),
                   heads=2),
         W.Problem("one-token", (), (W.Segment(1, 1, 0),), heads=1),
         W.with_random_blocks(_packed("packed-6", 5, 6), 0.4, 13)]


@pytest.mark.parametrize("q_scale", [1.0, 6.0], ids=["normal", "sharp"])
@pytest.mark.parametrize("p", SMALL, ids=lambda p: p.name)
def test_backward_matches_oracle(p, q_scale):
    b = Bwd(p, 81, q_scale)
    dq, dk, dv = b.backward()
    q, k, v, d_o = b.oracle_inputs()
    r_dq, r_dk, r_dv = obwd.attention_backward(orule.Layout.of(p), q, k, v, d_o, p.softmax_scale)
    _check("dq", dq, r_dq)
    _check("dk", dk, r_dk)
    _check("dv", dv, r_dv)


def test_backward_is_deterministic():
    b = Bwd(_packed("packed-5", 8, 5), 82)
    first = b.backward()
    second = b.backward()
    for a, c in zip(first, second):
        assert torch.equal(a, c)


def test_backward_rejects_cache_and_missing_workspace():
    p = W.small_session(heads=2)
    s = GpuSession(p, W.make_inputs(p, 83))
    t = torch.zeros_like(s.q)
    lse = torch.zeros(p.heads, p.n_query_tokens, device="cuda")
    with pytest.raises(sca.ScaError) as e:
        sca.action_causal_attn_bwd(s.md, p.heads, s.q, s.k_cur, s.v_cur, t, lse, t, t, t, t,
                                   p.softmax_scale, None, 0, s.status)
    assert e.value.code == sca.ERR_UNSUPPORTED
    b = Bwd(W.tiny_packed(), 84)
    with pytest.raises(sca.ScaError) as e:
        sca.action_causal_attn_bwd(b.s.md, 2, b.s.q, b.s.k_cur, b.s.v_cur, b.o, b.lse, b.d_o,
                                   t, t, t, b.p.softmax_scale, None, 0, b.s.status)
    assert e.value.code == sca.ERR_CAPACITY


def test_pipeline_timeout_aborts_the_backward_cleanly():
    """The backward's three kernels with the pipeline-wait limit at 0: the
    call reports SCA_ERR_DEVICE_TIMEOUT, every CTA drains its own loads and
    products before it exits, and with the default limit restored the next
    backward on the same handles matches the oracle."""
    p = _packed("packed-14", 21, 14, heads=4)
    b = Bwd(p, 85)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    dq, dk, dv = (torch.empty_like(b.s.q) for _ in range(3))
    ws = torch.empty(sca.attn_bwd_workspace_bytes(b.s.md, p.heads), dtype=torch.uint8,
                     device="cuda")
    try:
        sca.set_pipeline_timeout_ns(0)
        # a wait whose phase completes within the hardware's own try-wait
        # window does not time out even at 0: repeat until one call gives up
        for _ in range(5):
            sca.action_causal_attn_bwd(b.s.md, p.heads, b.s.q, b.s.k_cur, b.s.v_cur, b.o, b.lse,
                                       b.d_o, dq, dk, dv, p.softmax_scale, ws, None, st)
            torch.cuda.synchronize()
            if int(st.item()) != 0:
                break
    finally:
        sca.set_pipeline_timeout_ns(2_000_000_000)
    assert int(st.item()) == sca.ERR_DEVICE_TIMEOUT
    x = torch.ones(4, device="cuda")
    assert float((x * 2).sum().item()) == 8.0
    dq, dk, dv = b.backward()
    q, k, v, d_o = b.oracle_inputs()
    refs = obwd.attention_backward(orule.Layout.of(p), q, k, v, d_o, p.softmax_scale)
    for name, got, ref in zip(("dq", "dk", "dv"), (dq, dk, dv), refs):
        _check(name, got, ref)


@pytest.mark.slow
def test_backward_packed_360k_sampled_rows_and_identities():
    p = W.packed_360k()
    b = Bwd(p, 85)
    dq, dk, dv = b.backward()
    for t in (dq, dk, dv):
        assert torch.isfinite(t.float()).all()
    rows = W.sample_rows(p.n_query_tokens, 24, seed=5)
    heads = [0, 11]
    q, k, v, d_o = b.oracle_inputs()
    lay = orule.Layout.of(p)
    ref = obwd.dq_rows(lay, q, k, v, d_o, rows, p.softmax_scale, heads=heads)
    _check("dq rows", dq[rows][:, heads], ref)
    # Σ_keys dK = 0 and Σ_keys dV = Σ_queries dO, per head and dimension (every
    # query sees at least itself); bf16 rounding of each term bounds the sums
    sk = dk.double().sum(0)
    assert (sk.abs() <= 1e-2 * dk.double().abs().sum(0) + 1e-3).all()
    sv, so = dv.double().sum(0), b.d_o.double().sum(0)
    assert ((sv - so).abs() <= 1e-2 * dv.double().abs().sum(0) + 1e-2).all()
