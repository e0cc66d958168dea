"""The allocation-free attention entry point (sca_action_causal_attn_fwd_static_ws).

It serves callers that must not allocate device memory, and takes its
key-split scratch from a fixed array inside the library instead of a caller
workspace. Each call through the C ABI must give what the regular entry point
gives with a workspace on the same inputs and the same split (the same
kernels and plan, so the same output within the parity tolerance). Two calls
in a row use different inputs and different splits, so a call that read the
partials the previous call left in the shared array would be caught. An
automatic plan that needs more scratch than the array holds runs unsplit; a
forced split that needs more is refused before launching anything.

This file is collected last on purpose; it must pass both on its own in a
fresh process and after the other tests.
"""
import pytest
import torch

from oracle import attention as oattn
from oracle import rule as orule
from segment_causal_masked_b200 import workloads as W

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

from segment_causal_masked_b200 import sca  # noqa: E402
from tests.gpu_session import GpuSession, compare, oracle_inputs  # noqa: E402


def _outputs(p):
    nq, h = p.n_query_tokens, p.heads
    return (torch.full((nq, h, 128), float("nan"), dtype=torch.bfloat16, device="cuda"),
            torch.full((h, nq), float("nan"), dtype=torch.float32, device="cuda"))


def _regular(s, p, q, extra_bytes=0, workspace=True):
    o, lse = _outputs(p)
    ws = None
    if workspace:
        nbytes = (sca.attn_workspace_bytes(s.md, p.heads) + 255) // 256 * 256 + extra_bytes
        ws = torch.empty(max(nbytes, 256), dtype=torch.uint8, device="cuda")
    sca.action_causal_attn_fwd(s.cache if p.cached else None, s.md, p.heads, q, s.k_cur,
                               s.v_cur, o, lse, p.softmax_scale, ws, None, s.status)
    return o, lse


def _static(s, p, q):
    o, lse = _outputs(p)
    sca.action_causal_attn_fwd_static_ws(s.cache if p.cached else None, s.md, p.heads, q,
                                         s.k_cur, s.v_cur, o, lse, p.softmax_scale, s.status)
    return o, lse


def _same(a, b):
    (o, lse), (o_ref, l_ref) = a, b
    assert int(torch.isnan(o.float()).sum().item()) == 0
    assert (o.float() - o_ref.float()).abs().max().item() <= 2e-2
    assert (lse - l_ref).abs().max().item() <= 1e-2


@pytest.mark.parametrize("splits", [(3, 5), (0, 0)], ids=["forced-3-then-5", "automatic"])
def test_static_workspace_matches_regular_entry_twice(splits):
    """Two calls in a row with different queries (and, forced, different key
    splits), each against the regular entry point on its own inputs."""
    p = W.small_session(heads=4)
    s = GpuSession(p, W.make_inputs(p, 51, 2.0))
    q2 = W.make_inputs(p, 53, 2.0)["q"].cuda()
    try:
        for q, chunks in zip((s.q, q2), splits):
            sca.set_split_override(chunks)      # k >= 2: force the key split; 0: automatic plan
            if chunks:
                assert 0 < sca.attn_workspace_bytes(s.md, p.heads) <= sca.STATIC_WORKSPACE_BYTES
            ref = _regular(s, p, q)
            got = _static(s, p, q)
            torch.cuda.synchronize()
            assert sca.read_device_status(s.status) == sca.OK
            _same(got, ref)
    finally:
        sca.set_split_override(0)


def test_static_workspace_int8_cache_holds_the_bf16_copy():
    """An INT8 cache small enough that the split partials and a bf16 copy of
    the cache fit the array: the call dequantises once into the array, like
    the regular entry point with a workspace that large (bit for bit), and
    matches the oracle over the dequantised cache."""
    p = W.small_session(heads=4)
    inputs = W.make_inputs(p, 54, 2.0)
    s = GpuSession(p, inputs, int8=True)
    extra = sca.attn_int8_scratch_bytes(s.md, p.heads)
    try:
        sca.set_split_override(3)
        need = (sca.attn_workspace_bytes(s.md, p.heads) + 255) // 256 * 256 + extra
        assert need <= sca.STATIC_WORKSPACE_BYTES
        ref = _regular(s, p, s.q, extra_bytes=extra)
        got = _static(s, p, s.q)
        torch.cuda.synchronize()
    finally:
        sca.set_split_override(0)
    assert sca.read_device_status(s.status) == sca.OK
    assert torch.equal(got[0], ref[0]) and torch.equal(got[1], ref[1])
    q, k, v = oracle_inputs(inputs, int8=True)
    o_ref, lse_ref = oattn.attention(orule.Layout.of(p), q, k, v, p.softmax_scale)
    compare(got[0], got[1], o_ref, lse_ref)


def test_static_workspace_runs_unsplit_when_the_plan_does_not_fit():
    """A layout whose automatic split plan needs more scratch than the array
    (33 MiB on a 148-SM B200): the call runs every work item whole, which is
    the regular entry point without a workspace, bit for bit."""
    seg = W.Segment(8, 390, 128, (W.Action(32, 0, 4), W.Action(32, 4, 8)))
    p = W.Problem("plan-over-32mib", (seg,), (seg,), heads=4)
    inputs = W.make_inputs(p, 55)
    s = GpuSession(p, inputs)
    if sca.attn_workspace_bytes(s.md, p.heads) <= sca.STATIC_WORKSPACE_BYTES:
        pytest.skip("this device's split plan for the layout fits the array")
    ref = _regular(s, p, s.q, workspace=False)
    got = _static(s, p, s.q)
    torch.cuda.synchronize()
    assert sca.read_device_status(s.status) == sca.OK
    assert torch.equal(got[0], ref[0]) and torch.equal(got[1], ref[1])
    rows = W.sample_rows(p.n_query_tokens, 32, seed=5)
    q, k, v = oracle_inputs(inputs)
    o_ref, lse_ref = oattn.attention_rows(orule.Layout.of(p), q, k, v, rows, p.softmax_scale)
    compare(got[0][rows], got[1][:, rows], o_ref, lse_ref)


def test_static_workspace_refuses_oversized_split():
    p = W.small_session(heads=4)
    s = GpuSession(p, W.make_inputs(p, 52))
    try:
        sca.set_split_override(64)          # 4 items x 64 chunks: ~34 MB of partials
        assert sca.attn_workspace_bytes(s.md, p.heads) > sca.STATIC_WORKSPACE_BYTES
        o, lse = _outputs(p)
        with pytest.raises(sca.ScaError) as e:
            sca.action_causal_attn_fwd_static_ws(s.cache, s.md, p.heads, s.q, s.k_cur, s.v_cur,
                                                 o, lse, p.softmax_scale, s.status)
        assert e.value.code == sca.ERR_CAPACITY and "static workspace" in str(e.value)
        torch.cuda.synchronize()
        assert torch.isnan(o.float()).all()   # nothing was launched
    finally:
        sca.set_split_override(0)
