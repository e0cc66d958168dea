"""The growing KV cache after an append, and the ABI's descriptor words.

Test infrastructure (see the package docstring).

After a segment is generated its keys and values join a permanent cache that
every later segment attends to ([gpts24] "One World, Generated Segment by
Segment"). Its action tails stay in the cache but are never visible to a
later segment ([picx] "Action-Aware Causal Attention (Figure 6b)"), so the
appended tail keys are marked dead.

Cache layout (the library's documented format): K and V are head-major
``[heads, capacity, 128]``; the descriptor array holds one 32-bit word per
key:

    bits  0..15  segment index (cache order)
    bit  16      token is an action tail
    bit  17      alive: visible to later segments (video and head)
    bit  18      token is in the descriptive head
    bits 24..29  action index of a tail token (0 otherwise)

Query descriptors are two words per query:

    word 0: bits 0..15 segment index, bit 16 sees earlier segments,
            bit 17 valid query
    word 1: bit a set when the query sees tail a of its own segment
"""
from __future__ import annotations

from typing import Tuple

import numpy as np

from .rule import FULL_SEGMENT, TAIL, VIDEO, Layout

SEG_MASK = 0xFFFF
IS_TAIL = 1 << 16
ALIVE = 1 << 17
IS_HEAD = 1 << 18
ACTION_SHIFT = 24
Q_SEES_PAST = 1 << 16
Q_VALID = 1 << 17


def segment_key_descriptors(segment, segment_index: int) -> np.ndarray:
    """Descriptor word of each key of one segment, in token order."""
    words = []
    nv = segment.num_frames * segment.tokens_per_frame
    words += [segment_index | ALIVE] * nv                        # video
    words += [segment_index | ALIVE | IS_HEAD] * segment.head_len  # head
    for a, act in enumerate(segment.actions):                    # tails: dead later
        words += [segment_index | IS_TAIL | (a << ACTION_SHIFT)] * act.length
    return np.asarray(words, dtype=np.uint32)


def key_descriptors(segments, first_index: int = 0) -> np.ndarray:
    parts = [segment_key_descriptors(s, first_index + i) for i, s in enumerate(segments)]
    return np.concatenate(parts) if parts else np.zeros(0, np.uint32)


def query_descriptors(layout: Layout) -> np.ndarray:
    """[n_queries, 2] words describing what each query sees."""
    out = np.zeros((layout.n_queries, 2), dtype=np.uint32)
    for run in layout.runs:
        sees_past = run.kind == VIDEO or layout.policy == FULL_SEGMENT
        w0 = run.segment | Q_VALID | (Q_SEES_PAST if sees_past else 0)
        sp = layout.spans[run.segment]
        bits = 0
        for a, (b, e) in enumerate(sp.windows):
            if run.kind == VIDEO:
                seen = b <= run.frame < e
            else:
                seen = layout.policy == FULL_SEGMENT or (run.kind == TAIL and run.action == a)
            if seen:
                bits |= 1 << a
        out[run.start:run.stop, 0] = w0
        out[run.start:run.stop, 1] = bits
    return out


def append(cache_k: np.ndarray, cache_v: np.ndarray, cache_desc: np.ndarray,
           length: int, segment_index: int, segment, k: np.ndarray, v: np.ndarray
           ) -> Tuple[np.ndarray, np.ndarray, np.ndarray, int]:
    """Copy a segment's token-major K/V [n, H, d] into the head-major cache
    at rows [length, length+n) and write its descriptor words."""
    n = k.shape[0]
    ck, cv, cd = cache_k.copy(), cache_v.copy(), cache_desc.copy()
    if length + n > ck.shape[1]:
        raise ValueError("cache capacity exceeded")
    ck[:, length:length + n, :] = np.transpose(k, (1, 0, 2))
    cv[:, length:length + n, :] = np.transpose(v, (1, 0, 2))
    cd[length:length + n] = segment_key_descriptors(segment, segment_index)
    return ck, cv, cd, length + n


# ---------------------------------------------------------------------------
# INT8 cache
# ---------------------------------------------------------------------------
# The pages quantise the KV cache to INT8 for single-GPU inference ([picx]
# "Inference") without giving the scheme. Reading: every 128-value row of K
# or V (one token, one head) is quantised symmetrically with its own scale,
#     scale = max_d |x_d| / 127        (float32)
#     q_d   = round_half_even(x_d / scale), clamped to [-127, 127]   (int8)
# with x the bf16 value widened to float32 and both divisions in float32
# (a row of zeros has scale 0 and q = 0). The cached value is q * scale,
# formed in float32 and rounded to bf16: dequantisation gives back a tensor
# of the dtype the cache held before quantisation.

def quantize_rows(x: np.ndarray):
    """x: [..., 128] (bf16 values as float32). Returns (q int8 [..., 128],
    scale float32 [...])."""
    x = np.asarray(x, dtype=np.float32)
    amax = np.abs(x).max(axis=-1)
    scale = (amax / np.float32(127.0)).astype(np.float32)
    safe = np.where(scale > 0, scale, np.float32(1.0)).astype(np.float32)
    q = np.rint((x / safe[..., None]).astype(np.float32))
    q = np.clip(q, -127, 127).astype(np.int8)
    q[scale == 0] = 0
    return q, scale


def round_bf16(x: np.ndarray) -> np.ndarray:
    """float32 -> nearest bf16 (ties to even), returned as float32. bf16 keeps
    the top 16 bits of a float32; rounding adds half of the dropped range,
    minus one when the kept part is even, before truncating (finite x)."""
    b = np.asarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    b = (b + 0x7FFF + ((b >> 16) & 1)) & 0xFFFF0000
    return b.astype(np.uint32).view(np.float32)


def dequantize_rows(q: np.ndarray, scale: np.ndarray) -> np.ndarray:
    """bf16(float32(q * scale)), as float64."""
    v = q.astype(np.float32) * scale.astype(np.float32)[..., None]
    return round_bf16(v).astype(np.float64)


def append_int8(cache_q: np.ndarray, cache_scale: np.ndarray, length: int, k: np.ndarray):
    """Quantise token-major [n, H, 128] rows into the head-major int8 cache
    [H, capacity, 128] and its scales [H, capacity] at rows [length, length+n)."""
    q, s = quantize_rows(np.transpose(k, (1, 0, 2)))
    cq, cs = cache_q.copy(), cache_scale.copy()
    cq[:, length:length + k.shape[0], :] = q
    cs[:, length:length + k.shape[0]] = s
    return cq, cs
