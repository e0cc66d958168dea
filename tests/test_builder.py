"""Host-side parity of the C++ metadata builder against the oracle (no GPU).

The builder (sca_build_segment_mask_metadata) evaluates a predicate on
descriptor words; the oracle builds the explicit mask from sets of visible
key ranges and classifies tiles by brute force. Schedules, descriptors and the
unmasked-pair count must agree bit for bit.
"""
import os
import re

import numpy as np
import pytest

from oracle import cache as ocache
from oracle import rule as orule
from oracle import schedule as osched
from segment_causal_masked_b200 import workloads as W

sca = pytest.importorskip("segment_causal_masked_b200.sca")

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _builder(p):
    return sca.build_for(p)


def _overlap_problem():
    segs = (W.Segment(4, 3, 2, (W.Action(2, 0, 3), W.Action(3, 1, 2), W.Action(1, 3, 4))),
            W.Segment(3, 2, 0, (W.Action(2, 0, 1),)),
            W.Segment(1, 1, 0))
    return W.Problem("overlap", (), segs, heads=1)


SMALL = [
    W.tiny_packed(),
    W.small_session(),
    W.small_packed(),
    W.small_packed(seed=21, n_segments=14),
    W.Problem("small-session-full", W.small_session().cached, W.small_session().current, heads=2,
              textq_policy=W.TEXTQ_FULL_SEGMENT),
    _overlap_problem(),
    W.Problem("one-token", (), (W.Segment(1, 1, 0),), heads=1),
    W.Problem("no-text-cache", (W.Segment(3, 100, 0),), (W.Segment(2, 70, 5),), heads=1),
    W.Problem("32-actions", (), (W.Segment(32, 9, 4, tuple(W.Action(3, a, a + 1) for a in range(32))),),
              heads=1),
]


@pytest.mark.parametrize("p", SMALL, ids=lambda p: p.name)
def test_schedule_descriptors_and_count_small(p):
    lay = orule.Layout.of(p)
    md = _builder(p)
    c = md.counts()
    assert c["unmasked_pairs"] == int(lay.mask().sum()) == lay.unmasked_pairs()
    assert c["n_queries"] == lay.n_queries and c["n_cache_keys"] == lay.n_cache
    row_ptr, kv, flag = md.schedule()
    o_row_ptr, o_kv, o_flag = osched.schedule(lay)
    assert np.array_equal(row_ptr, o_row_ptr)
    assert np.array_equal(kv, o_kv)
    assert np.array_equal(flag, o_flag)
    assert c["n_full"] == int((o_flag == osched.FULL).sum())
    assert c["n_partial"] == int((o_flag == osched.PARTIAL).sum())
    kd, qd = md.descriptors()
    assert np.array_equal(kd, ocache.key_descriptors(p.current, len(p.cached)))
    assert np.array_equal(qd, ocache.query_descriptors(lay))


def _window_and_blocks():
    sess = W.small_session(heads=1)
    long_sess = W.Problem("long-small", tuple(W.small_packed(seed=5, n_segments=7).current),
                          (W.Segment(3, 60, 9, (W.Action(4, 0, 2), W.Action(6, 1, 3))),), heads=1)
    return [W.with_history(sess, 0), W.with_history(sess, 1), W.with_history(long_sess, 3),
            W.with_history(W.small_packed(seed=21, n_segments=14), 2),
            W.with_random_blocks(long_sess, 0.25, 7),
            W.with_random_blocks(W.with_history(long_sess, 4), 0.5, 8),
            W.with_random_blocks(W.small_packed(seed=21, n_segments=14), 0.3, 9),
            W.with_random_blocks(W.with_history(W.session_480p_single_turn(), 2), 0.25, 10)]


@pytest.mark.parametrize("p", _window_and_blocks(), ids=lambda p: p.name)
def test_window_and_dropped_blocks_schedule(p):
    """Sliding window and dropped video blocks: schedule, classes and A
    bit-exact against the oracle's brute-force tiles."""
    lay = orule.Layout.of(p)
    md = _builder(p)
    c = md.counts()
    assert c["unmasked_pairs"] == lay.unmasked_pairs()
    row_ptr, kv, flag = md.schedule()
    o_row_ptr, o_kv, o_flag = osched.schedule(lay)
    assert np.array_equal(row_ptr, o_row_ptr)
    assert np.array_equal(kv, o_kv) and np.array_equal(flag, o_flag)


def test_window_closed_form_and_bad_keep_blocks():
    p = W.with_history(W.session_480p_long(), 4)
    assert _builder(p).counts()["unmasked_pairs"] == 742_096_884
    with pytest.raises(sca.ScaError) as e:
        sca.build_segment_mask_metadata((), (W.Segment(2, 4, 1),), keep_blocks=np.ones((3, 3)))
    assert e.value.code == sca.ERR_INVALID_ARG and "keep_blocks" in str(e.value)


@pytest.mark.slow
@pytest.mark.parametrize("make", [W.session_480p_single_turn, W.session_480p_long, W.session_720p],
                         ids=["480p-single-turn", "480p-long-session", "720p-step"])
def test_schedule_full_size(make):
    p = make()
    lay = orule.Layout.of(p)
    md = _builder(p)
    c = md.counts()
    assert c["unmasked_pairs"] == lay.unmasked_pairs()
    row_ptr, kv, flag = md.schedule()
    o_row_ptr, o_kv, o_flag = osched.schedule(lay)
    assert np.array_equal(row_ptr, o_row_ptr)
    assert np.array_equal(kv, o_kv) and np.array_equal(flag, o_flag)
    kd, qd = md.descriptors()
    assert np.array_equal(kd, ocache.key_descriptors(p.current, len(p.cached)))
    assert np.array_equal(qd, ocache.query_descriptors(lay))


def test_480p_long_session_totals():
    """Closed forms: A = 1,923,821,844; 97 query tiles; 1158 + 97 key tiles."""
    md = _builder(W.session_480p_long())
    c = md.counts()
    assert c["unmasked_pairs"] == 1_923_821_844
    assert c["n_q_tiles"] == 97 and c["n_kv_tiles"] == 1158 + 97


@pytest.mark.slow
def test_packed_360k_sampled_tiles():
    p = W.packed_360k()
    lay = orule.Layout.of(p)
    md = _builder(p)
    c = md.counts()
    assert c["unmasked_pairs"] == lay.unmasked_pairs()
    assert c["n_queries"] == lay.n_queries <= 360_000
    row_ptr, kv, flag = md.schedule()
    rng = np.random.default_rng(0)
    n_qt = c["n_q_tiles"]
    for qt in sorted({0, n_qt - 1, *rng.choice(n_qt, 6, replace=False).tolist()}):
        cls = osched.classify_query_tile(lay, qt)
        nz = np.nonzero(cls)[0]
        assert np.array_equal(kv[row_ptr[qt]:row_ptr[qt + 1]], nz), qt
        assert np.array_equal(flag[row_ptr[qt]:row_ptr[qt + 1]], cls[nz]), qt


# ---------------------------------------------------------------------------
# the ABI itself
# ---------------------------------------------------------------------------

def test_library_exports_every_declared_symbol():
    with open(os.path.join(ROOT, "include", "sca.h")) as f:
        declared = set(re.findall(r"SCA_API\s+[\w\s\*]+?\b(sca_\w+)\s*\(", f.read()))
    assert declared == set(sca.EXPORTED)
    for name in declared:
        assert hasattr(sca._lib, name), name


@pytest.mark.parametrize("seg, msg", [
    (W.Segment(0, 4, 1), "num_frames"),
    (W.Segment(2, 0, 1), "tokens_per_frame"),
    (W.Segment(2, 4, -1), "head_len"),
    (W.Segment(2, 4, 1, (W.Action(3, 1, 1),)), "action 0"),
    (W.Segment(2, 4, 1, (W.Action(0, 0, 1),)), "action 0"),
    (W.Segment(2, 4, 1, (W.Action(3, 0, 3),)), "action 0"),
    (W.Segment(2, 4, 1, tuple(W.Action(1, 0, 1) for _ in range(33))), "num_actions"),
])
def test_builder_rejects_bad_layouts(seg, msg):
    with pytest.raises(sca.ScaError) as e:
        sca.build_segment_mask_metadata((), (seg,))
    assert e.value.code == sca.ERR_INVALID_ARG and msg in str(e.value)


def test_builder_rejects_empty_current_and_bad_policy():
    with pytest.raises(sca.ScaError):
        sca.build_segment_mask_metadata((), ())
    with pytest.raises(sca.ScaError):
        sca.build_segment_mask_metadata((), (W.Segment(1, 1, 0),), textq_policy=7)


def test_rebuild_replaces_contents():
    md = sca.build_segment_mask_metadata((), (W.Segment(1, 1, 0),))
    assert md.counts()["n_queries"] == 1
    md.build(W.small_session().cached, W.small_session().current)
    assert md.counts()["n_queries"] == W.small_session().n_query_tokens


def test_int8_cache_handle_checks():
    """The INT8 cache records caller buffers (no GPU work): capacity must be
    a multiple of 4, buffers 16-byte aligned."""
    base = 1 << 20   # fake, aligned device addresses: the handle never dereferences them
    with pytest.raises(sca.ScaError) as e:
        sca.kv_cache_create_int8(2, 6, base, base, base, base, base)
    assert e.value.code == sca.ERR_INVALID_ARG and "multiple of 4" in str(e.value)
    with pytest.raises(sca.ScaError) as e:
        sca.kv_cache_create_int8(2, 8, base, base, base + 4, base, base)
    assert e.value.code == sca.ERR_MISALIGNED
    c = sca.kv_cache_create_int8(2, 8, base, base, base, base, base)
    assert c.int8 and c.get() == (0, 0)


@pytest.mark.parametrize("p", [W.tiny_packed(), W.small_packed(), W.small_packed(seed=21, n_segments=14),
                               W.with_random_blocks(W.small_packed(seed=21, n_segments=14), 0.3, 9)],
                         ids=lambda p: p.name)
def test_backward_schedule_is_the_transposed_oracle_schedule(p):
    """The backward's key-major lists: for every key tile, the query tiles
    whose oracle class is not EMPTY, ascending, with that class; the order
    is a permutation of the key tiles."""
    lay = orule.Layout.of(p)
    md = _builder(p)
    kt_ptr, kt_list, kt_order = md.bwd_schedule()
    row_ptr, kv, flag = osched.schedule(lay)
    n_kt = md.counts()["n_kv_tiles"]
    expect = [[] for _ in range(n_kt)]
    for qt in range(len(row_ptr) - 1):
        for i in range(row_ptr[qt], row_ptr[qt + 1]):
            expect[int(kv[i])].append(qt | (int(flag[i]) << 24))
    assert kt_ptr[0] == 0 and len(kt_ptr) == n_kt + 1
    for t in range(n_kt):
        assert kt_list[kt_ptr[t]:kt_ptr[t + 1]].tolist() == expect[t], t
    assert sorted(kt_order.tolist()) == list(range(n_kt))


def test_backward_schedule_absent_with_a_cache():
    kt_ptr, kt_list, kt_order = _builder(W.small_session()).bwd_schedule()
    assert len(kt_ptr) == 0 and len(kt_list) == 0 and len(kt_order) == 0


def test_backward_and_int8_copy_workspace_sizes():
    """Host-only size queries: the backward's −D/−LSE rows per head padded to
    whole tiles, and the INT8 copy of the cached K and V (two halves, each
    256-byte aligned)."""
    p = W.small_packed()
    md = _builder(p)
    n_pad = md.counts()["n_q_tiles"] * 128
    assert sca.attn_bwd_workspace_bytes(md, 3) == 2 * 3 * n_pad * 4
    s = _builder(W.small_session())
    nc = W.small_session().n_cache_tokens
    half = (5 * nc * 256 + 255) // 256 * 256
    assert sca.attn_int8_scratch_bytes(s, 5) == 2 * half


def test_backward_refuses_metadata_not_uploaded():
    md = _builder(W.tiny_packed())
    with pytest.raises(sca.ScaError) as e:
        sca.action_causal_attn_bwd(md, 2, 16, 16, 16, 16, 16, 16, 16, 16, 16, workspace=256,
                                   workspace_bytes=1 << 20, stream=0)
    assert e.value.code == sca.ERR_INVALID_ARG and "uploaded" in str(e.value)


# ---------------------------------------------------------------------------
# the key-split plan (host-side; sca_attn_plan_for_sms needs no device)
# ---------------------------------------------------------------------------

SLOT_BYTES = 256 * 128 * 4 + 256 * 8   # one split chunk's fp32 partials: O rows, then (m, l)


@pytest.mark.parametrize("make, want", [
    (W.session_480p_long, (740, 44, 5)),
    (W.session_480p_single_turn, (740, 44, 4)),
])
def test_split_plan_of_the_480p_workloads_on_148_sms(make, want):
    """The plans the benchmark reported on a 148-SM B200: 49 query-tile pairs
    x 16 heads = 784 items, five whole waves kept and the 44 left cut into
    key chunks."""
    p = make()
    plan = sca.attn_plan_for_sms(_builder(p), p.heads, 148)
    assert (plan["n_full"], plan["n_split"], plan["chunks"]) == want
    assert plan["workspace_bytes"] == want[1] * want[2] * SLOT_BYTES


@pytest.mark.parametrize("sms", [1, 7, 132, 148, 160])
@pytest.mark.parametrize("p", [W.small_session(), W.small_packed(seed=21, n_segments=14),
                               W.session_480p_single_turn()], ids=lambda p: p.name)
def test_split_plan_properties(p, sms):
    md = _builder(p)
    n_items = (md.counts()["n_q_tiles"] + 1) // 2 * p.heads
    plan = sca.attn_plan_for_sms(md, p.heads, sms)
    assert plan["n_full"] + plan["n_split"] == n_items
    if plan["chunks"] == 1:
        assert plan["n_split"] == 0 and plan["workspace_bytes"] == 0
    else:
        assert plan["chunks"] in (2, 3, 4, 5, 6, 8)
        assert plan["n_full"] % sms == 0 and plan["n_split"] > 0
        assert plan["workspace_bytes"] == plan["n_split"] * plan["chunks"] * SLOT_BYTES


def test_split_plan_follows_the_override():
    p = W.session_480p_long()
    md = _builder(p)
    try:
        sca.set_split_override(1)
        plan = sca.attn_plan_for_sms(md, p.heads, 148)
        assert (plan["n_full"], plan["n_split"], plan["chunks"]) == (784, 0, 1)
        sca.set_split_override(3)        # keep all but the last whole wave, cut the rest in 3
        plan = sca.attn_plan_for_sms(md, p.heads, 148)
        assert (plan["n_full"], plan["n_split"], plan["chunks"]) == (4 * 148, 784 - 4 * 148, 3)
    finally:
        sca.set_split_override(0)
    with pytest.raises(sca.ScaError):
        sca.attn_plan_for_sms(md, p.heads, 0)


def test_cache_calls_refuse_before_any_gpu_work():
    """Every refusal of create / append / truncate happens on the host before
    anything is enqueued, and leaves the cache as it was (fake, aligned
    device addresses: nothing is dereferenced or launched)."""
    base = 1 << 20
    with pytest.raises(sca.ScaError) as e:
        sca.KVCache(2, 64, base, base + 8, base)
    assert e.value.code == sca.ERR_MISALIGNED
    with pytest.raises(sca.ScaError) as e:
        sca.KVCache(0, 64, base, base, base)
    assert e.value.code == sca.ERR_INVALID_ARG
    with pytest.raises(sca.ScaError) as e:
        sca.KVCache(2, 64, 0, base, base)
    assert e.value.code == sca.ERR_INVALID_ARG

    cache = sca.KVCache(2, 64, base, base, base)
    seg = W.Segment(2, 20, 8, (W.Action(4, 0, 1), W.Action(3, 1, 2)))   # 55 tokens
    big = W.Segment(3, 20, 8)                                           # 68 tokens
    cases = [
        (big, base, base, sca.ERR_CAPACITY, "does not fit"),
        (seg, base + 4, base, sca.ERR_MISALIGNED, "aligned"),
        (seg, 0, base, sca.ERR_INVALID_ARG, "null k"),
        (W.Segment(0, 20, 8), base, base, sca.ERR_INVALID_ARG, "num_frames"),
        (W.Segment(2, 20, 8, (W.Action(4, 1, 3),)), base, base, sca.ERR_INVALID_ARG, "[1, 3)"),
    ]
    for s, k, v, code, text in cases:
        with pytest.raises(sca.ScaError) as e:
            cache.append(s, k, v, stream=0)
        assert e.value.code == code and text in str(e.value), (code, str(e.value))
        assert cache.get() == (0, 0)
    with pytest.raises(sca.ScaError) as e:
        cache.truncate(1)
    assert e.value.code == sca.ERR_INVALID_ARG and cache.get() == (0, 0)
    cache.truncate(0)
    assert cache.get() == (0, 0)


def test_unbuilt_or_null_metadata_is_refused_by_every_accessor():
    md = sca.Metadata()
    calls = [md.counts, md.schedule, md.descriptors, md.bwd_schedule,
             lambda: sca.attn_workspace_bytes(md, 2), lambda: sca.attn_int8_scratch_bytes(md, 2),
             lambda: sca.attn_bwd_workspace_bytes(md, 2), lambda: sca.attn_plan_for_sms(md, 2, 148)]
    for call in calls:
        with pytest.raises(sca.ScaError) as e:
            call()
        assert e.value.code == sca.ERR_INVALID_ARG and "not built" in str(e.value)
    assert sca._lib.sca_metadata_get_counts(None, *([None] * 8)) == sca.ERR_INVALID_ARG
    sca._lib.sca_metadata_destroy(None)      # a no-op
    sca._lib.sca_kv_cache_destroy(None)
