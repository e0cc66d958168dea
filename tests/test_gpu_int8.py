"""INT8 KV cache on the GPU against the oracle.

The append kernel quantises each (token, head) row of K and V to int8 codes
and one fp32 scale; the codes and scales must equal the oracle's bit for bit
(both take the integer decision in fp32 with correctly rounded divisions).
Attention over the INT8 cache must match the oracle's attention over the
dequantised cache (code x scale rounded to bf16) within the parity bar of the
bf16 path.
"""
import numpy as np
import pytest
import torch

from oracle import attention as oattn
from oracle import cache as ocache
from oracle import rule as orule
from segment_causal_masked_b200 import workloads as W

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

from segment_causal_masked_b200 import sca  # noqa: E402
from tests.gpu_session import GpuSession, compare, oracle_inputs  # noqa: E402


def _multi_pair(heads=3):
    return W.Problem("multi-pair", (W.Segment(4, 300, 33, (W.Action(20, 0, 2), W.Action(9, 1, 4))),),
                     (W.Segment(5, 230, 17, (W.Action(40, 0, 5), W.Action(7, 2, 3))),), heads=heads)


def _planted_inputs(p, seed):
    """Seeded inputs with special cache rows: a zero row, a row of one value,
    rows of huge and tiny magnitude, and values that land exactly half way
    between two codes."""
    inputs = W.make_inputs(p, seed)
    ck = inputs["cache_k"].clone()
    ck[0, 0] = 0
    ck[1, 0] = -3.0
    ck[2, 0] = ck[2, 0] * 1e30
    ck[3, 0] = ck[3, 0] * 1e-30
    row = torch.zeros(128)
    row[0], row[1], row[2] = 127.0, 2.5, -3.5        # scale 1: ties at 2.5 and -3.5
    ck[4, 0] = row.bfloat16()
    inputs["cache_k"] = ck
    return inputs


def test_append_codes_and_scales_bit_exact():
    p = W.Problem("two-cached", (W.Segment(3, 40, 5, (W.Action(6, 0, 2),)),
                                 W.Segment(2, 50, 0, (W.Action(3, 1, 2),))),
                  (W.Segment(1, 7, 0),), heads=5)
    inputs = _planted_inputs(p, 71)
    s = GpuSession(p, inputs, int8=True)
    torch.cuda.synchronize()
    nc = p.n_cache_tokens
    for buf, sc, name in ((s.k_buf, s.k_scale, "cache_k"), (s.v_buf, s.v_scale, "cache_v")):
        q_ref, s_ref = ocache.quantize_rows(inputs[name].float().numpy())   # [n, H, 128], [n, H]
        codes = buf[:, :nc].cpu().numpy().transpose(1, 0, 2).astype(np.int16) - 128  # offset binary
        scales = sc[:, :nc].cpu().numpy().T
        assert np.array_equal(codes, q_ref), name
        assert np.array_equal(scales.view(np.uint32), s_ref.view(np.uint32)), name
        assert not buf[:, nc:].any() and not sc[:, nc:].any()   # rows past the length untouched
    k_codes = s.k_buf.cpu().numpy().astype(np.int16) - 128
    assert not k_codes[0, 0].any() and s.k_scale[0, 0].item() == 0.0
    assert k_codes[0, 4, :3].tolist() == [127, 2, -4] and s.k_scale[0, 4].item() == 1.0


SMALL = [W.small_session(heads=4), _multi_pair(),
         W.Problem("small-session-full", W.small_session().cached, W.small_session().current,
                   heads=2, textq_policy=W.TEXTQ_FULL_SEGMENT),
         W.with_history(W.small_session(heads=2), 0),
         W.with_random_blocks(W.Problem("long-small", tuple(W.small_packed(seed=5, n_segments=7).current),
                                        (W.Segment(3, 60, 9, (W.Action(4, 0, 2), W.Action(6, 1, 3))),),
                                        heads=2), 0.4, 12)]


@pytest.mark.parametrize("q_scale", [1.0, 8.0], ids=["normal", "sharp"])
@pytest.mark.parametrize("p", SMALL, ids=lambda p: p.name)
def test_int8_attention_matches_oracle(p, q_scale):
    inputs = W.make_inputs(p, 72, q_scale)
    s = GpuSession(p, inputs, int8=True)
    o, lse = s.forward()
    q, k, v = oracle_inputs(inputs, int8=True)
    o_ref, lse_ref = oattn.attention(orule.Layout.of(p), q, k, v, p.softmax_scale)
    compare(o, lse, o_ref, lse_ref)


def test_int8_reads_the_quantised_cache():
    """With sharp attention the quantisation error of the cache shows in the
    output: the result must be nearer the oracle over the dequantised cache
    than the oracle over the bf16 cache (so the codes, not stale bf16 rows,
    reach the products)."""
    p = W.small_session(heads=4)
    inputs = W.make_inputs(p, 73, 8.0)
    s = GpuSession(p, inputs, int8=True)
    o, _ = s.forward()
    lay = orule.Layout.of(p)
    o8, _ = oattn.attention(lay, *oracle_inputs(inputs, int8=True), p.softmax_scale)
    o16, _ = oattn.attention(lay, *oracle_inputs(inputs), p.softmax_scale)
    og = o.float().cpu().numpy().astype(np.float64)
    e8, e16 = np.linalg.norm(og - o8), np.linalg.norm(og - o16)
    assert e8 < 0.5 * e16, (e8, e16)


@pytest.mark.parametrize("chunks", [2, 5])
def test_int8_split_keys_and_merge(chunks):
    p = _multi_pair()
    inputs = W.make_inputs(p, 74, 4.0)
    s = GpuSession(p, inputs, int8=True)
    try:
        sca.set_split_override(chunks)
        o, lse = s.forward()
    finally:
        sca.set_split_override(0)
    q, k, v = oracle_inputs(inputs, int8=True)
    o_ref, lse_ref = oattn.attention(orule.Layout.of(p), q, k, v, p.softmax_scale)
    compare(o, lse, o_ref, lse_ref)


def test_int8_planted_rows_and_later_segments():
    """Special cache rows (zero, constant, huge, tiny) in a cache built from
    several appended segments: still within the bar, and finite."""
    p = W.small_session(heads=2)
    inputs = _planted_inputs(p, 75)
    inputs["cache_k"][2, 0] = inputs["cache_k"][2, 0] * 1e-28   # 100x the others
    s = GpuSession(p, inputs, int8=True)
    o, lse = s.forward()
    q, k, v = oracle_inputs(inputs, int8=True)
    o_ref, lse_ref = oattn.attention(orule.Layout.of(p), q, k, v, p.softmax_scale)
    compare(o, lse, o_ref, lse_ref)
    assert torch.isfinite(o.float()).all()


@pytest.mark.slow
def test_int8_full_size_sampled_rows():
    p = W.session_480p_long()
    inputs = W.make_inputs(p, 76)
    s = GpuSession(p, inputs, int8=True)
    o, lse = s.forward()
    rows = W.sample_rows(p.n_query_tokens, 40, seed=4)
    heads = [2, 13]
    q, k, v = oracle_inputs(inputs, int8=True)
    lay = orule.Layout.of(p)
    o_ref, lse_ref = oattn.attention_rows(lay, q, k, v, rows, p.softmax_scale, heads=heads)
    compare(o[rows][:, heads], lse[heads][:, rows], o_ref, lse_ref)
    assert torch.isfinite(o.float()).all() and torch.isfinite(lse).all()


def _fwd(s, p, ws_bytes):
    o = torch.full((p.n_query_tokens, p.heads, 128), float("nan"), dtype=torch.bfloat16, device="cuda")
    lse = torch.full((p.heads, p.n_query_tokens), float("nan"), device="cuda")
    ws = torch.empty(max(ws_bytes, 256), dtype=torch.uint8, device="cuda")
    sca.action_causal_attn_fwd(s.cache, s.md, p.heads, s.q, s.k_cur, s.v_cur, o, lse,
                               p.softmax_scale, ws, ws_bytes, s.status)
    torch.cuda.synchronize()
    assert int(s.status.item()) == 0
    return o, lse


@pytest.mark.parametrize("chunks", [0, 3])
@pytest.mark.parametrize("p", [W.small_session(heads=4), _multi_pair(),
                               W.with_history(W.small_session(heads=2), 1)], ids=lambda p: p.name)
def test_int8_scratch_path_equals_tile_path(p, chunks):
    """With room for a bf16 copy of the cache, the call dequantises once and
    runs the bf16 kernel: the same values reach the products, so the result
    equals the tile-by-tile INT8 kernel's bit for bit; it matches the oracle."""
    s = GpuSession(p, W.make_inputs(p, 77, 3.0), int8=True)
    try:
        sca.set_split_override(chunks)
        split = (sca.attn_workspace_bytes(s.md, p.heads) + 255) // 256 * 256
        scratch = sca.attn_int8_scratch_bytes(s.md, p.heads)
        assert scratch == 2 * ((p.heads * p.n_cache_tokens * 256 + 255) // 256 * 256)
        o1, l1 = _fwd(s, p, split)               # tile by tile
        o2, l2 = _fwd(s, p, split + scratch)     # one bf16 copy first
    finally:
        sca.set_split_override(0)
    assert torch.equal(o1, o2) and torch.equal(l1, l2)   # the same values reach the products
    q, k, v = oracle_inputs(W.make_inputs(p, 77, 3.0), int8=True)
    o_ref, lse_ref = oattn.attention(orule.Layout.of(p), q, k, v, p.softmax_scale)
    compare(o2, l2, o_ref, lse_ref)
