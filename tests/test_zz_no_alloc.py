"""The allocation-free attention entry point (sca_action_causal_attn_fwd_static_ws).

It serves callers that must not allocate device memory, and takes its
key-split scratch from a fixed array inside the library instead of a caller
workspace. Two calls in a row through the C ABI must each give what the
regular entry point gives with a workspace (the same kernels and plan, so
the same output within the parity tolerance), and a call whose split needs
more scratch than the array holds must be refused before launching anything.

This file is collected last on purpose; it must pass both on its own in a
fresh process and after the other tests.
"""
import pytest
import torch

from segment_causal_masked_b200 import workloads as W

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

from segment_causal_masked_b200 import sca  # noqa: E402
from tests.gpu_session import GpuSession  # noqa: E402


def _outputs(p):
    nq, h = p.n_query_tokens, p.heads
    return (torch.full((nq, h, 128), float("nan"), dtype=torch.bfloat16, device="cuda"),
            torch.full((h, nq), float("nan"), dtype=torch.float32, device="cuda"))


def _regular(s, p):
    o, lse = _outputs(p)
    nbytes = sca.attn_workspace_bytes(s.md, p.heads)
    ws = torch.empty(max(nbytes, 256), dtype=torch.uint8, device="cuda")
    sca.action_causal_attn_fwd(s.cache if p.cached else None, s.md, p.heads, s.q, s.k_cur,
                               s.v_cur, o, lse, p.softmax_scale, ws, None, s.status)
    return o, lse


def _static(s, p):
    o, lse = _outputs(p)
    sca.action_causal_attn_fwd_static_ws(s.cache if p.cached else None, s.md, p.heads, s.q,
                                         s.k_cur, s.v_cur, o, lse, p.softmax_scale, s.status)
    return o, lse


@pytest.mark.parametrize("chunks", [3, 0])
def test_static_workspace_matches_regular_entry_twice(chunks):
    p = W.small_session(heads=4)
    s = GpuSession(p, W.make_inputs(p, 51, 2.0))
    try:
        sca.set_split_override(chunks)      # 3: force the key split; 0: automatic plan
        if chunks:
            assert 0 < sca.attn_workspace_bytes(s.md, p.heads) <= sca.STATIC_WORKSPACE_BYTES
        o_ref, l_ref = _regular(s, p)
        for _ in range(2):                  # the array keeps the last call's contents
            o, lse = _static(s, p)
            torch.cuda.synchronize()
            assert int(s.status.item()) == 0
            assert (o.float() - o_ref.float()).abs().max().item() <= 2e-2
            assert (lse - l_ref).abs().max().item() <= 1e-2
            assert torch.isfinite(o.float()).all() and torch.isfinite(lse).all()
    finally:
        sca.set_split_override(0)


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
