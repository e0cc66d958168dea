"""Pins of the oracle's mask, pair count, descriptors and tile schedule.

Each check compares the oracle with something other than itself: a hand
derivation stored under tests/golden, closed-form counts worked out by hand
below, or a brute-force pairwise predicate written independently here.
"""
import json
import os

import numpy as np
import pytest

from oracle import cache as ocache
from oracle import rule as orule
from oracle import schedule as osched
from segment_causal_masked_b200 import workloads as W


def _golden(golden_dir, name):
    with open(os.path.join(golden_dir, name)) as f:
        return json.load(f)


# ---------------------------------------------------------------------------
# hand-derived visibility of the tiny packed layout
# ---------------------------------------------------------------------------

def test_tiny_visible_ranges_match_hand_derivation(golden_dir):
    g = _golden(golden_dir, "tiny_packed_visibility.json")
    lay = orule.Layout.of(W.tiny_packed())
    assert lay.n_keys == g["n_keys"] == lay.n_queries
    for cls in g["classes"]:
        q0, q1 = cls["queries"]
        want = np.zeros(lay.n_keys, dtype=bool)
        for a, b in cls["visible"]:
            want[a:b] = True
        assert int(want.sum()) == cls["count"], cls["name"]
        for q in range(q0, q1):
            assert np.array_equal(lay.mask_row(q), want), (cls["name"], q)


def test_tiny_unmasked_pairs(golden_dir):
    g = _golden(golden_dir, "tiny_packed_visibility.json")
    lay = orule.Layout.of(W.tiny_packed())
    assert lay.unmasked_pairs() == g["unmasked_pairs"] == int(lay.mask().sum())


def test_tiny_schedule(golden_dir):
    g = _golden(golden_dir, "tiny_packed_visibility.json")["schedule"]
    row_ptr, kv_tile, flag = osched.schedule(orule.Layout.of(W.tiny_packed()))
    assert row_ptr.tolist() == g["row_ptr"]
    assert kv_tile.tolist() == g["kv_tile"]
    assert flag.tolist() == g["flag"]


def test_tiny_descriptors(golden_dir):
    g = _golden(golden_dir, "tiny_packed_visibility.json")["descriptors"]
    p = W.tiny_packed()
    kd = ocache.key_descriptors(p.current)
    for idx, word in g["keys"]:
        assert int(kd[idx]) == word, idx
    qd = ocache.query_descriptors(orule.Layout.of(p))
    for idx, w0, w1 in g["queries"]:
        assert (int(qd[idx, 0]), int(qd[idx, 1])) == (w0, w1), idx


# ---------------------------------------------------------------------------
# closed-form pair counts (A of Eq. 6) of the 480p layouts, worked by hand
# ---------------------------------------------------------------------------
# A 480p segment: 31 frames x 390 = 12,090 video tokens, head 128, four
# 32-token tails whose windows cover every frame exactly once. Alive (video +
# head) tokens of a past segment: 12,218. Per current-segment query:
#   video : (cached alive) + own video + head + one tail = P + 12,090 + 160
#   head  : own video + head                            = 12,218
#   tail  : own video + head + its tail                 = 12,250

@pytest.mark.parametrize("n_cached, expect", [
    (3, 12_090 * (3 * 12_218 + 12_090 + 128 + 32) + 128 * 12_218 + 128 * 12_250),
    (12, 12_090 * (12 * 12_218 + 12_090 + 128 + 32) + 128 * 12_218 + 128 * 12_250),
])
def test_480p_unmasked_pairs_closed_form(n_cached, expect):
    s = W.seg_480p()
    lay = orule.Layout((s,) * n_cached, (s,))
    assert lay.unmasked_pairs() == expect
    assert expect in (594_381_264, 1_923_821_844)


def test_480p_key_and_tile_counts():
    lay = orule.Layout.of(W.session_480p_long())
    assert lay.n_cache == 148_152 and lay.n_keys == 160_498 and lay.n_queries == 12_346
    assert len(osched.key_tiles(lay)) == 1158 + 97
    assert osched.n_query_tiles(lay) == 97


# ---------------------------------------------------------------------------
# tile classes of the 480p layouts, derived by hand
# ---------------------------------------------------------------------------
# A cached 480p segment s occupies keys [12346 s, 12346 (s+1)); its dead tails
# are the last 128 keys, starting at 12346 s + 12218 = 58 (s+1) (mod 128),
# never tile-aligned for s < 63, so each dead run touches exactly two tiles:
# floor((12346 s + 12218)/128) and the next, both PARTIAL for a video query
# tile -- except for the last cached segment, whose second tile is the ragged
# last cache tile and lies wholly inside the dead run (it starts at
# 128 (n_tiles-1) >= 12346 n_cached - 128), so it is EMPTY. Current keys:
# video [0,12090), head [12090,12218), tails a0 [12218,12250) a1 [12250,12282) a2 [12282,12314) a3 [12314,12346).
# Query tile 0 = queries 0..127 = video of frame 0 (window of a0 only):
#   current tiles 0..94 (keys < 12160) are video/head -> FULL,
#   tile 95 (keys 12160..12287: head, a0, a1, a2) -> PARTIAL,
#   tile 96 (keys 12288..12345: a2, a3)            -> EMPTY.
# Query tile 96 = queries 12288..12345 (tails a2, a3; 58 rows): text queries
#   see no cache key; every current tile holds keys they see; all ragged ->
#   PARTIAL.

def _expected_cache_classes(n_cached):
    n_cache = 12_346 * n_cached
    n_tiles = (n_cache + 127) // 128
    assert 128 * (n_tiles - 1) >= n_cache - 128      # last tile wholly dead
    partial = set()
    for s in range(n_cached):
        first = (12_346 * s + 12_218) // 128
        partial.update({first, first + 1})
    partial.discard(n_tiles - 1)
    return n_tiles, partial


@pytest.mark.parametrize("problem", [W.session_480p_single_turn, W.session_480p_long])
def test_480p_tile_classes_by_hand(problem):
    p = problem()
    lay = orule.Layout.of(p)
    n_ct, partial = _expected_cache_classes(len(p.cached))
    cls0 = osched.classify_query_tile(lay, 0)
    want = np.full(n_ct + 97, osched.FULL, dtype=np.uint8)
    for t in partial:
        want[t] = osched.PARTIAL
    want[n_ct - 1] = osched.EMPTY
    want[n_ct + 95] = osched.PARTIAL
    want[n_ct + 96] = osched.EMPTY
    assert np.array_equal(cls0, want)
    assert int((cls0 == osched.FULL).sum()) == n_ct - 1 - len(partial) + 95
    assert int((cls0 == osched.PARTIAL).sum()) == 2 * len(p.cached) - 1 + 1

    cls96 = osched.classify_query_tile(lay, 96)
    want96 = np.full(n_ct + 97, osched.PARTIAL, dtype=np.uint8)
    want96[:n_ct] = osched.EMPTY
    assert np.array_equal(cls96, want96)


# ---------------------------------------------------------------------------
# brute-force pairwise predicate, written independently of the oracle
# ---------------------------------------------------------------------------

def _token_table(segments):
    """Per token: (segment, kind, frame, action, window-begin, window-end)."""
    rows = []
    for si, seg in enumerate(segments):
        for f in range(seg.num_frames):
            rows += [(si, "v", f, -1)] * seg.tokens_per_frame
        rows += [(si, "h", -1, -1)] * seg.head_len
        for a, act in enumerate(seg.actions):
            rows += [(si, "t", -1, a)] * act.length
    return rows


def _brute_mask(problem):
    segs = list(problem.cached) + list(problem.current)
    keys = _token_table(segs)
    queries = keys[problem.n_cache_tokens:]
    full = problem.textq_policy == W.TEXTQ_FULL_SEGMENT
    hist = problem.history_segments
    m = np.zeros((len(queries), len(keys)), dtype=bool)
    for i, (qs, qk, qf, qa) in enumerate(queries):
        for j, (ks, kk, kf, ka) in enumerate(keys):
            if ks > qs:
                ok = False
            elif ks < qs:
                ok = kk != "t" and (qk == "v" or full) and (hist < 0 or qs - ks <= hist)
            elif kk != "t":
                ok = True
            elif qk == "v":
                act = segs[ks].actions[ka]
                ok = act.begin <= qf < act.end
            else:
                ok = full or (qk == "t" and qa == ka)
            m[i, j] = ok
    if problem.keep_blocks is not None:                 # drop video-only key tiles
        nc = problem.n_cache_tokens
        starts = list(range(0, nc, 128)) + [nc + u for u in range(0, len(queries), 128)]
        ends = [min(nc, a + 128) for a in range(0, nc, 128)] + \
               [nc + min(len(queries), u + 128) for u in range(0, len(queries), 128)]
        for kt, (a, b) in enumerate(zip(starts, ends)):
            if all(keys[j][1] == "v" for j in range(a, b)):
                for i in range(len(queries)):
                    if not problem.keep_blocks[i // 128, kt]:
                        m[i, a:b] = False
    return m


@pytest.mark.parametrize("problem", [
    W.tiny_packed(),
    W.small_session(),
    W.small_packed(),
    W.Problem("small-session-full", W.small_session().cached, W.small_session().current,
              heads=2, textq_policy=W.TEXTQ_FULL_SEGMENT),
    W.Problem("overlap", (), (W.Segment(4, 3, 2, (W.Action(2, 0, 3), W.Action(3, 1, 2),
                                                     W.Action(1, 3, 4))),
                                W.Segment(3, 2, 0, (W.Action(2, 0, 1),))), heads=1),
])
def test_mask_matches_brute_force(problem):
    lay = orule.Layout.of(problem)
    m = lay.mask()
    assert np.array_equal(m, _brute_mask(problem))
    assert lay.unmasked_pairs() == int(m.sum())


def _window_and_blocks_problems():
    sess = W.small_session(heads=1)
    long_sess = W.Problem("long-small", tuple(W.small_packed(seed=5, n_segments=7).current),
                          (W.Segment(3, 60, 9, (W.Action(4, 0, 2), W.Action(6, 1, 3))),), heads=1)
    return [
        W.with_history(sess, 0), W.with_history(sess, 1), W.with_history(sess, 2),
        W.with_history(long_sess, 3),
        W.with_history(W.small_packed(seed=21, n_segments=14), 2),
        W.with_random_blocks(long_sess, 0.25, 7),
        W.with_random_blocks(W.with_history(long_sess, 4), 0.5, 8),
        W.with_random_blocks(W.small_packed(seed=21, n_segments=14), 0.3, 9),
    ]


@pytest.mark.parametrize("p", _window_and_blocks_problems(), ids=lambda p: p.name)
def test_window_and_dropped_blocks_match_brute_force(p):
    lay = orule.Layout.of(p)
    m = lay.mask()
    assert np.array_equal(m, _brute_mask(p))
    assert lay.unmasked_pairs() == int(m.sum())


def test_window_closed_form_480p():
    """Window of 4 segments over the 12-segment cache: a video query sees 4
    cached segments' video + head (4 x 12,218) plus its own 12,250; text
    queries are unaffected (they never look back)."""
    s = W.seg_480p()
    lay = orule.Layout((s,) * 12, (s,), history=4)
    expect = 12_090 * (4 * 12_218 + 12_250) + 128 * 12_218 + 128 * 12_250
    assert lay.unmasked_pairs() == expect == 742_096_884   # 12,090 x 61,122 + 1,563,904 + 1,568,000


def test_window_and_blocks_degenerate_cases():
    p = W.small_session(heads=1)
    full = orule.Layout.of(p).mask()
    assert np.array_equal(orule.Layout.of(W.with_history(p, 99)).mask(), full)
    keep_all = np.ones((W.n_query_tiles(p), W.n_key_tiles(p)), bool)
    import dataclasses
    assert np.array_equal(orule.Layout.of(dataclasses.replace(p, keep_blocks=keep_all)).mask(), full)


def test_schedule_matches_brute_force_tiles():
    p = W.small_session()
    lay = orule.Layout.of(p)
    m = _brute_mask(p)
    row_ptr, kv_tile, flag = osched.schedule(lay)
    tiles = osched.key_tiles(lay)
    for qt in range(osched.n_query_tiles(lay)):
        rows = m[qt * 128:(qt + 1) * 128]
        got = dict(zip(kv_tile[row_ptr[qt]:row_ptr[qt + 1]].tolist(),
                       flag[row_ptr[qt]:row_ptr[qt + 1]].tolist()))
        for t, (k0, nk) in enumerate(tiles):
            blk = rows[:, k0:k0 + nk]
            if not blk.any():
                assert t not in got
            elif blk.shape == (128, 128) and blk.all():
                assert got[t] == osched.FULL
            else:
                assert got[t] == osched.PARTIAL


def test_rejects_bad_layouts():
    with pytest.raises(ValueError):
        orule.Layout((), (W.Segment(0, 4, 1),))
    with pytest.raises(ValueError):
        orule.Layout((), (W.Segment(2, 4, 1, (W.Action(3, 1, 1),)),))
    with pytest.raises(ValueError):
        orule.Layout((), (W.Segment(2, 4, 1, (W.Action(3, 0, 3),)),))


# ---------------------------------------------------------------------------
# the cache after an append
# ---------------------------------------------------------------------------

def test_cache_append_layout_and_dead_tails():
    seg = W.Segment(2, 3, 2, (W.Action(2, 0, 1), W.Action(1, 1, 2)))
    n, h, d = seg.n_tokens, 3, 4
    rng = np.random.default_rng(0)
    k = rng.standard_normal((n, h, d))
    v = rng.standard_normal((n, h, d))
    ck = np.zeros((h, 16, d)); cv = np.zeros((h, 16, d)); cd = np.zeros(16, np.uint32)
    ck, cv, cd, length = ocache.append(ck, cv, cd, 5, 7, seg, k, v)
    assert length == 5 + n
    for i in range(n):
        for hh in range(h):
            assert np.array_equal(ck[hh, 5 + i], k[i, hh])
            assert np.array_equal(cv[hh, 5 + i], v[i, hh])
    # video 6 tokens, head 2, tails 2 + 1: hand-written words for segment 7
    want = [7 | 1 << 17] * 6 + [7 | 1 << 17 | 1 << 18] * 2 + [7 | 1 << 16] * 2 + [7 | 1 << 16 | 1 << 24]
    assert cd[5:5 + n].tolist() == want
    assert not cd[:5].any() and not cd[5 + n:].any()
