"""Sharpness of the oracle's pins.

A pin is only worth something if a plausible mistake in the oracle makes it
fail. Each case below plants one such mistake in the oracle (on the CPU,
through ``monkeypatch``, undone after the case): a dropped term, a wrong
sign, an off-by-one window end, a transposed or swapped operand, a wrong
rounding. It then runs the pins of that part of the oracle and requires at
least one of them to fail an assertion. The unmodified oracle passes every
pin (the rest of the suite); for the camera cross-attention, whose mistakes
are planted in a restatement of the oracle, the restatement left correct is
shown to pass the same pins.
"""
import functools
import os

import numpy as np
import pytest

from oracle import attention as oattn
from oracle import backward as obwd
from oracle import cache as ocache
from oracle import camera as ocam
from oracle import rule as orule
from oracle import schedule as osched
from segment_causal_masked_b200 import workloads as W
from tests import test_oracle_attention as ta
from tests import test_oracle_backward as tb
from tests import test_oracle_camera as tc
from tests import test_oracle_int8 as ti
from tests import test_oracle_rule as tr

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")
_p = functools.partial


def _mask_problems():
    return [W.tiny_packed(), W.small_session(), W.small_packed(),
            W.Problem("small-session-full", W.small_session().cached, W.small_session().current,
                      heads=2, textq_policy=W.TEXTQ_FULL_SEGMENT)]


def _rule_pins():
    pins = [_p(tr.test_tiny_visible_ranges_match_hand_derivation, GOLDEN),
            _p(tr.test_tiny_unmasked_pairs, GOLDEN),
            _p(tr.test_tiny_schedule, GOLDEN),
            _p(tr.test_tiny_descriptors, GOLDEN),
            tr.test_window_closed_form_480p]
    pins += [_p(tr.test_mask_matches_brute_force, p) for p in _mask_problems()]
    pins += [_p(tr.test_window_and_dropped_blocks_match_brute_force, p)
             for p in tr._window_and_blocks_problems()]
    return pins


def _attention_pins():
    return [_p(ta.test_matches_torch_sdpa, W.tiny_packed(), 1.0),
            _p(ta.test_matches_torch_sdpa, W.small_session(), 8.0),
            ta.test_zero_queries_give_mean_of_visible_values,
            ta.test_constant_values_are_reproduced,
            ta.test_single_visible_key,
            ta.test_fully_masked_row_is_zero]


def _backward_pins():
    return [_p(tb.test_matches_torch_autograd, tb.LAYOUTS[0], 1.0),
            _p(tb.test_matches_torch_autograd, tb.LAYOUTS[2], 6.0),
            tb.test_identities,
            tb.test_sampled_rows_equal_full_rows]


def _int8_pins():
    return [ti.test_hand_worked_row, ti.test_half_even_ties_and_extremes,
            ti.test_round_bf16_matches_torch_and_ties, ti.test_dequantized_values_by_hand,
            ti.test_error_bound_and_range]


def _schedule_pins():
    return [_p(tr.test_tiny_schedule, GOLDEN), tr.test_schedule_matches_brute_force_tiles,
            _p(tr.test_480p_tile_classes_by_hand, W.session_480p_single_turn),
            tr.test_480p_key_and_tile_counts]


def _descriptor_pins():
    return [_p(tr.test_tiny_descriptors, GOLDEN), tr.test_cache_append_layout_and_dead_tails]


def _first_failure(pins):
    """Name of the first pin whose assertion fails, or None. Only a failed
    assertion counts: a planted mistake that merely crashes a pin (a shape
    error) would show nothing about the pin's sharpness."""
    for pin in pins:
        try:
            pin()
        except AssertionError:
            f = pin.func if isinstance(pin, functools.partial) else pin
            return f.__name__
    return None


# ---------------------------------------------------------------------------
# planted mistakes: the visibility rule
# ---------------------------------------------------------------------------

_vkr = orule.visible_key_ranges


def _past_tails_visible(spans, run, policy=orule.OWN_TAIL, history=-1):
    out = _vkr(spans, run, policy, history)
    if run.kind == orule.VIDEO:
        out += [t for sp in spans if sp.segment < run.segment for t in sp.tails if t[1] > t[0]]
    return out


def _window_end_inclusive(spans, run, policy=orule.OWN_TAIL, history=-1):
    out = _vkr(spans, run, policy, history)
    if run.kind == orule.VIDEO:
        sp = spans[run.segment]
        out += [t for t, (b, e) in zip(sp.tails, sp.windows) if run.frame == e and t[1] > t[0]]
    return out


def _text_sees_past(spans, run, policy=orule.OWN_TAIL, history=-1):
    out = _vkr(spans, run, policy, history)
    if run.kind != orule.VIDEO and policy == orule.OWN_TAIL:
        for sp in spans:
            if sp.segment < run.segment:
                out += [r for r in (sp.video, sp.head) if r[1] > r[0]]
    return out


def _own_head_hidden(spans, run, policy=orule.OWN_TAIL, history=-1):
    head = spans[run.segment].head
    return [r for r in _vkr(spans, run, policy, history) if r != head]


def _later_segments_visible(spans, run, policy=orule.OWN_TAIL, history=-1):
    out = _vkr(spans, run, policy, history)
    return out + [sp.video for sp in spans if sp.segment > run.segment]


def _history_off_by_one(spans, run, policy=orule.OWN_TAIL, history=-1):
    return _vkr(spans, run, policy, history - 1 if history > 0 else history)


def _tail_sees_all_tails(spans, run, policy=orule.OWN_TAIL, history=-1):
    out = _vkr(spans, run, policy, history)
    if run.kind == orule.TAIL:
        out += [t for t in spans[run.segment].tails if t not in out and t[1] > t[0]]
    return out


_qruns = orule.query_runs


def _frames_from_one(cached, current):
    return [orule.QueryRun(r.start, r.stop, r.segment, r.kind, r.frame + 1 if r.frame >= 0 else -1,
                           r.action) for r in _qruns(cached, current)]


_spans = orule.spans


def _head_before_video(segments):
    out = []
    for sp in _spans(segments):
        nv = sp.video[1] - sp.video[0]
        nh = sp.head[1] - sp.head[0]
        h0 = sp.video[0]
        out.append(orule.Span(sp.segment, (h0 + nh, h0 + nh + nv), (h0, h0 + nh), sp.tails,
                              sp.windows, sp.num_frames, sp.tokens_per_frame, sp.stop))
    return out


def _unmasked_pairs_per_run(self):
    return sum(sum(b - a for a, b in orule.visible_key_ranges(self.spans, r, self.policy,
                                                              self.history))
               for r in self.runs)


RULE_MISTAKES = {
    "past tails visible": ("visible_key_ranges", _past_tails_visible),
    "window end inclusive": ("visible_key_ranges", _window_end_inclusive),
    "text queries see the past": ("visible_key_ranges", _text_sees_past),
    "own head hidden": ("visible_key_ranges", _own_head_hidden),
    "later segments visible": ("visible_key_ranges", _later_segments_visible),
    "history window off by one": ("visible_key_ranges", _history_off_by_one),
    "tail query sees every tail": ("visible_key_ranges", _tail_sees_all_tails),
    "frames counted from one": ("query_runs", _frames_from_one),
}


@pytest.mark.parametrize("name", list(RULE_MISTAKES))
def test_rule_mistake_is_caught(name, monkeypatch):
    attr, fn = RULE_MISTAKES[name]
    monkeypatch.setattr(orule, attr, fn)
    assert _first_failure(_rule_pins()) is not None, name


def test_token_order_mistake_is_caught(monkeypatch):
    """The head laid out before the video of its segment."""
    monkeypatch.setattr(orule, "spans", _head_before_video)
    assert _first_failure(_rule_pins()) is not None


def test_pair_count_mistake_is_caught(monkeypatch):
    """A of Eq. 6 summed once per run instead of once per query."""
    monkeypatch.setattr(orule.Layout, "unmasked_pairs", _unmasked_pairs_per_run)
    assert _first_failure(_rule_pins()) is not None


# ---------------------------------------------------------------------------
# planted mistakes: attention values
# ---------------------------------------------------------------------------

_ma = oattn.masked_attention


def _softmax(s, axis):
    m = np.max(s, axis=axis, keepdims=True, initial=-np.inf)
    m = np.where(np.isfinite(m), m, 0.0)
    e = np.exp(s - m)
    return e / e.sum(axis=axis, keepdims=True), m, e.sum(axis=axis, keepdims=True)


def _masked_scores_zero(q, k, v, mask, scale, dtype=np.float64):
    s = (np.asarray(q, dtype) @ np.asarray(k, dtype).T) * dtype(scale)
    p, m, z = _softmax(np.where(mask, s, 0.0), 1)
    return p @ np.asarray(v, dtype), (m + np.log(z))[:, 0]


def _softmax_over_queries(q, k, v, mask, scale, dtype=np.float64):
    s = (np.asarray(q, dtype) @ np.asarray(k, dtype).T) * dtype(scale)
    s = np.where(mask, s, -np.inf)
    with np.errstate(invalid="ignore"):
        p, _, _ = _softmax(s, 0)
    _, lse = _ma(q, k, v, mask, scale, dtype)
    return np.nan_to_num(p) @ np.asarray(v, dtype), lse


def _lse_without_max(q, k, v, mask, scale, dtype=np.float64):
    o, lse = _ma(q, k, v, mask, scale, dtype)
    s = np.where(mask, (np.asarray(q, dtype) @ np.asarray(k, dtype).T) * dtype(scale), -np.inf)
    m = s.max(axis=1, initial=-np.inf)
    return o, np.where(np.isfinite(m), lse - m, lse)


def _empty_rows_nan(q, k, v, mask, scale, dtype=np.float64):
    o, lse = _ma(q, k, v, mask, scale, dtype)
    o[~np.asarray(mask).any(axis=1)] = np.nan
    return o, lse


ATTENTION_MISTAKES = {
    "scale dropped": lambda q, k, v, mask, scale, dtype=np.float64: _ma(q, k, v, mask, 1.0, dtype),
    "scale applied twice": lambda q, k, v, mask, scale, dtype=np.float64: _ma(q, k, v, mask,
                                                                              scale * scale, dtype),
    "keys used as values": lambda q, k, v, mask, scale, dtype=np.float64: _ma(q, k, k, mask, scale,
                                                                              dtype),
    "masked scores set to zero": _masked_scores_zero,
    "softmax over the queries": _softmax_over_queries,
    "LSE without the row max": _lse_without_max,
    "rows that see nothing left undefined": _empty_rows_nan,
}


@pytest.mark.parametrize("name", list(ATTENTION_MISTAKES))
def test_attention_mistake_is_caught(name, monkeypatch):
    monkeypatch.setattr(oattn, "masked_attention", ATTENTION_MISTAKES[name])
    assert _first_failure(_attention_pins()) is not None, name


# ---------------------------------------------------------------------------
# planted mistakes: gradients
# ---------------------------------------------------------------------------

def _backward_with(mistake):
    """The oracle's backward with one planted mistake (same loop structure)."""

    def bwd(layout, q, k_all, v_all, d_o, scale):
        q, k_all, v_all, d_o = (np.asarray(a, dtype=np.float64) for a in (q, k_all, v_all, d_o))
        dq, dk, dv = np.zeros_like(q), np.zeros_like(k_all), np.zeros_like(v_all)
        mask = layout.mask_rows(range(q.shape[0]))
        for h in range(q.shape[1]):
            p = obwd._probs(q[:, h], k_all[:, h], mask, scale)
            dv[:, h] += p.T @ d_o[:, h]
            dp = d_o[:, h] @ (k_all if mistake == "dP from K" else v_all)[:, h].T
            d = (p * dp).sum(axis=1, keepdims=True)
            ds = {"D dropped": p * dp, "sign of dS": p * (d - dp)}.get(mistake, p * (dp - d))
            sq = 1.0 if mistake == "dQ scale dropped" else scale
            dq[:, h] = sq * (ds @ (v_all if mistake == "dQ from V" else k_all)[:, h])
            dk[:, h] += scale * (ds.T @ q[:, h])
        return dq, dk, dv

    return bwd


BACKWARD_MISTAKES = ["D dropped", "sign of dS", "dQ scale dropped", "dQ from V", "dP from K"]


@pytest.mark.parametrize("name", BACKWARD_MISTAKES)
def test_backward_mistake_is_caught(name, monkeypatch):
    monkeypatch.setattr(obwd, "attention_backward", _backward_with(name))
    assert _first_failure(_backward_pins()) is not None, name


# ---------------------------------------------------------------------------
# planted mistakes: INT8 cache, descriptors, tile schedule
# ---------------------------------------------------------------------------

def _scale_over_128(x):
    x = np.asarray(x, dtype=np.float32)
    scale = (np.abs(x).max(axis=-1) / np.float32(128.0)).astype(np.float32)
    safe = np.where(scale > 0, scale, np.float32(1.0)).astype(np.float32)
    q = np.clip(np.rint((x / safe[..., None]).astype(np.float32)), -127, 127).astype(np.int8)
    q[scale == 0] = 0
    return q, scale


def _round_half_away(x):
    x = np.asarray(x, dtype=np.float32)
    amax = np.abs(x).max(axis=-1)
    scale = (amax / np.float32(127.0)).astype(np.float32)
    safe = np.where(scale > 0, scale, np.float32(1.0)).astype(np.float32)
    r = (x / safe[..., None]).astype(np.float32)
    q = np.clip(np.sign(r) * np.floor(np.abs(r) + 0.5), -127, 127).astype(np.int8)
    q[scale == 0] = 0
    return q, scale


def _truncate_bf16(x):
    b = np.asarray(x, dtype=np.float32).view(np.uint32) & np.uint32(0xFFFF0000)
    return b.view(np.float32)


INT8_MISTAKES = {
    "scale = amax / 128": ("quantize_rows", _scale_over_128),
    "ties rounded away from zero": ("quantize_rows", _round_half_away),
    "bf16 by truncation": ("round_bf16", _truncate_bf16),
    "no bf16 rounding of the dequantised value": ("round_bf16", lambda x: np.asarray(x, np.float32)),
}


@pytest.mark.parametrize("name", list(INT8_MISTAKES))
def test_int8_mistake_is_caught(name, monkeypatch):
    attr, fn = INT8_MISTAKES[name]
    monkeypatch.setattr(ocache, attr, fn)
    assert _first_failure(_int8_pins()) is not None, name


_skd = ocache.segment_key_descriptors


def _tails_alive(segment, segment_index):
    w = _skd(segment, segment_index)
    return np.where(w & ocache.IS_TAIL, w | ocache.ALIVE, w).astype(np.uint32)


def _head_bit_missing(segment, segment_index):
    return (_skd(segment, segment_index) & ~np.uint32(ocache.IS_HEAD)).astype(np.uint32)


@pytest.mark.parametrize("fn", [_tails_alive, _head_bit_missing], ids=["tails alive", "no head bit"])
def test_descriptor_mistake_is_caught(fn, monkeypatch):
    monkeypatch.setattr(ocache, "segment_key_descriptors", fn)
    assert _first_failure(_descriptor_pins()) is not None


_ckt = osched.classify_query_tile


def _ragged_full(layout, qt):
    """FULL whenever every existing position is visible (ragged edges too)."""
    cls = _ckt(layout, qt)
    rows = np.arange(qt * 128, min((qt + 1) * 128, layout.n_queries))
    mask = layout.mask_rows(rows)
    for i, (k0, nk) in enumerate(osched.key_tiles(layout)):
        if mask[:, k0:k0 + nk].all():
            cls[i] = osched.FULL
    return cls


def _one_tiling(layout):
    """Key tiles laid over the whole key sequence, across the cache boundary."""
    return [(t0, min(128, layout.n_keys - t0)) for t0 in range(0, layout.n_keys, 128)]


@pytest.mark.parametrize("attr, fn", [("classify_query_tile", _ragged_full),
                                      ("key_tiles", _one_tiling)],
                         ids=["ragged tiles FULL", "one tiling across sources"])
def test_schedule_mistake_is_caught(attr, fn, monkeypatch):
    monkeypatch.setattr(osched, attr, fn)
    assert _first_failure(_schedule_pins()) is not None


# ---------------------------------------------------------------------------
# planted mistakes: camera cross-attention
# ---------------------------------------------------------------------------

def _camera_pins():
    pins = [_p(tc.test_matches_torch_sdpa, mode, n_cam, sharp)
            for mode in (ocam.CAM_ALL, ocam.CAM_UP_TO_FRAME) for n_cam in (1, 7, 31)
            for sharp in (1.0, 6.0)]
    return pins + [tc.test_own_frame_adds_that_frames_value_row, tc.test_single_camera_token,
                   tc.test_equal_keys_give_the_mean_of_the_visible_values,
                   tc.test_frames_outside_the_segment_keep_the_residual,
                   tc.test_all_mode_ignores_the_order_of_camera_tokens, tc.test_visibility_sets]


_vis = ocam.visible_camera_tokens
_cxa = ocam.camera_cross_attention


def _vis_with(fn):
    def vis(q_frame, n_cam, mode):
        q_frame = np.asarray(q_frame, dtype=np.int64)
        if mode == ocam.CAM_ALL:
            return _vis(q_frame, n_cam, mode)
        if mode not in (ocam.CAM_OWN_FRAME, ocam.CAM_UP_TO_FRAME):
            raise ValueError("unknown camera attention mode")
        return fn(q_frame[:, None], np.arange(n_cam)[None, :], n_cam, mode)
    return vis


CAMERA_VISIBILITY_MISTAKES = {
    "own frame off by one": _vis_with(
        lambda qf, f, n, mode: ((qf >= 0) & (qf < n)) & ((f == qf + 1) if mode == ocam.CAM_OWN_FRAME
                                                         else (f <= qf))),
    "frames up to the own one, exclusive": _vis_with(
        lambda qf, f, n, mode: ((qf >= 0) & (qf < n)) & ((f == qf) if mode == ocam.CAM_OWN_FRAME
                                                         else (f < qf))),
    "frames outside the segment see tokens": _vis_with(
        lambda qf, f, n, mode: (f == qf) if mode == ocam.CAM_OWN_FRAME else (f <= qf)),
    "every token for the whole segment": lambda q_frame, n_cam, mode: np.ones(
        (np.asarray(q_frame).shape[0], n_cam), dtype=bool),
}


def test_camera_visibility_restatement_without_a_mistake_passes(monkeypatch):
    monkeypatch.setattr(ocam, "visible_camera_tokens", _vis_with(
        lambda qf, f, n, mode: ((qf >= 0) & (qf < n)) & ((f == qf) if mode == ocam.CAM_OWN_FRAME
                                                         else (f <= qf))))
    assert _first_failure(_camera_pins()) is None


@pytest.mark.parametrize("name", list(CAMERA_VISIBILITY_MISTAKES))
def test_camera_visibility_mistake_is_caught(name, monkeypatch):
    monkeypatch.setattr(ocam, "visible_camera_tokens", CAMERA_VISIBILITY_MISTAKES[name])
    assert _first_failure(_camera_pins()) is not None, name


def _camera_with(mistake):
    def f(q, k_cam, v_cam, x, q_frame, mode, scale):
        q = np.asarray(q, dtype=np.float64)
        k = np.asarray(k_cam, dtype=np.float64)
        v = np.asarray(v_cam, dtype=np.float64)
        x = np.asarray(x, dtype=np.float64)
        vis = ocam.visible_camera_tokens(q_frame, k.shape[0], mode)
        return mistake(q, k, v, x, vis, scale)
    return f


def _camera_attn(q, k, v, x, vis, scale, masked_value=-np.inf, residual=True, axis=1):
    out = np.array(x) if residual else np.zeros_like(x)
    for h in range(q.shape[1]):
        s = (q[:, h, :] @ k[:, h, :].T) * scale
        s = np.where(vis, s, masked_value)
        m = s.max(axis=axis, keepdims=True, initial=-np.inf)
        m = np.where(np.isfinite(m), m, 0.0)
        e = np.exp(s - m)
        z = e.sum(axis=axis, keepdims=True)
        p = np.divide(e, z, out=np.zeros_like(e), where=z > 0)
        out[:, h, :] += p @ v[:, h, :]
    return out


CAMERA_MISTAKES = {
    "residual not added": _camera_with(lambda q, k, v, x, vis, scale: _camera_attn(
        q, k, v, x, vis, scale, residual=False)),
    "scale dropped": _camera_with(lambda q, k, v, x, vis, scale: _camera_attn(q, k, v, x, vis, 1.0)),
    "keys used as values": _camera_with(lambda q, k, v, x, vis, scale: _camera_attn(
        q, k, k, x, vis, scale)),
    "hidden tokens scored 0 instead of -inf": _camera_with(
        lambda q, k, v, x, vis, scale: _camera_attn(q, k, v, x, vis, scale, masked_value=0.0)),
    "softmax over the queries": _camera_with(lambda q, k, v, x, vis, scale: _camera_attn(
        q, k, v, x, vis, scale, axis=0)),
    "queries that see nothing get the mean value": _camera_with(
        lambda q, k, v, x, vis, scale: np.where(
            vis.any(axis=1)[:, None, None], _camera_attn(q, k, v, x, vis, scale),
            x + v.mean(axis=0)[None])),
}


def test_camera_restatement_without_a_mistake_passes(monkeypatch):
    """Control: the restatement the mistakes are planted in, left correct,
    passes every camera pin (so a caught mistake is the mistake's doing)."""
    monkeypatch.setattr(ocam, "camera_cross_attention",
                        _camera_with(lambda q, k, v, x, vis, scale: _camera_attn(q, k, v, x, vis,
                                                                                  scale)))
    assert _first_failure(_camera_pins()) is None


@pytest.mark.parametrize("name", list(CAMERA_MISTAKES))
def test_camera_mistake_is_caught(name, monkeypatch):
    monkeypatch.setattr(ocam, "camera_cross_attention", CAMERA_MISTAKES[name])
    assert _first_failure(_camera_pins()) is not None, name
