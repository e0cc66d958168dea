"""Seeded synthetic workloads: segment layouts and bf16 Q/K/V tensors.

This module is the only code shared by the CUDA path and the CPU oracle. It
holds layouts and random numbers only, none of the attention arithmetic: the
oracle and the library each turn a layout into tokens, masks and schedules on
their own.

A layout follows the segment-autoregressive setting of the Hy-Nomas pages:
every segment has ``num_frames`` latent frames of ``tokens_per_frame`` video
tokens (the latent grid of Eq. 1 in the picx.dev summary, one token per
1x1x1 patch), a descriptive text head and action tails, each tail with a
half-open window of latent frames ("Action-Aware Causal Attention (Figure
6b)", picx.dev summary, Model Architecture).

Tensor shapes are token-major ``[tokens, heads, 128]`` bf16 drawn from
N(0, 1) in fp32 on the CPU with a seeded ``torch.Generator`` and rounded to
bf16, so that both sides of a parity test see bit-identical inputs.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Dict, List, Sequence, Tuple

import numpy as np

HEAD_DIM = 128
TEXTQ_OWN_TAIL = 0
TEXTQ_FULL_SEGMENT = 1


@dataclasses.dataclass(frozen=True)
class Action:
    """One action tail: ``length`` text tokens visible to frames [begin, end)."""

    length: int
    begin: int
    end: int


@dataclasses.dataclass(frozen=True)
class Segment:
    num_frames: int
    tokens_per_frame: int
    head_len: int
    actions: Tuple[Action, ...] = ()

    @property
    def n_tokens(self) -> int:
        return (self.num_frames * self.tokens_per_frame + self.head_len
                + sum(a.length for a in self.actions))


@dataclasses.dataclass(frozen=True)
class Problem:
    """One attention call: queries are the tokens of ``current``; keys are
    the tokens of ``cached`` followed by those of ``current``."""

    name: str
    cached: Tuple[Segment, ...]
    current: Tuple[Segment, ...]
    heads: int = 16
    textq_policy: int = TEXTQ_OWN_TAIL
    history_segments: int = -1          # sliding window over earlier segments (-1: all)
    keep_blocks: object = None          # [query tiles, key tiles] bools, or None

    @property
    def softmax_scale(self) -> float:
        return 1.0 / math.sqrt(HEAD_DIM)

    @property
    def n_cache_tokens(self) -> int:
        return sum(s.n_tokens for s in self.cached)

    @property
    def n_query_tokens(self) -> int:
        return sum(s.n_tokens for s in self.current)

    @property
    def n_key_tokens(self) -> int:
        return self.n_cache_tokens + self.n_query_tokens


# --------------------------------------------------------------------------
# the five workload shapes
# --------------------------------------------------------------------------

def _split_frames(num_frames: int, parts: int) -> List[Tuple[int, int]]:
    """Contiguous frame ranges with numpy.array_split's sizes (8,8,8,7 for 31/4)."""
    sizes = [len(c) for c in np.array_split(np.arange(num_frames), parts)]
    out, b = [], 0
    for n in sizes:
        out.append((b, b + n))
        b += n
    return out


def seg_480p() -> Segment:
    """31 latent frames of a 15x26 grid, a 128-token head and four 32-token
    tails whose windows split the 31 frames into four contiguous ranges."""
    acts = tuple(Action(32, b, e) for b, e in _split_frames(31, 4))
    return Segment(31, 15 * 26, 128, acts)


def tiny_packed() -> Problem:
    """2 segments of 2 frames x (4x6) tokens, head 16, tails 8+8 with windows
    [0,1) and [1,2); 2 heads; every token is a query."""
    seg = Segment(2, 24, 16, (Action(8, 0, 1), Action(8, 1, 2)))
    return Problem("tiny-packed", (), (seg, seg), heads=2)


def session_480p_single_turn() -> Problem:
    """Current 480p segment over a cache of 3 segments of the same layout."""
    s = seg_480p()
    return Problem("480p-single-turn", (s, s, s), (s,), heads=16)


def session_480p_long() -> Problem:
    """Current 480p segment over a cache of 12 segments (~148k cached keys)."""
    s = seg_480p()
    return Problem("480p-long-session", (s,) * 12, (s,), heads=16)


@dataclasses.dataclass(frozen=True)
class CameraProblem:
    """One camera cross-attention call: the video tokens of one segment
    (frame-major, ``tokens_per_frame`` per latent frame) as queries over the
    segment's camera tokens, one per latent frame ([onedev] "어떻게 쓰나")."""

    name: str
    num_frames: int
    tokens_per_frame: int
    heads: int = 16
    mode: int = 0                       # 0 every token, 1 own frame, 2 frames up to its own

    @property
    def n_q(self) -> int:
        return self.num_frames * self.tokens_per_frame

    @property
    def n_cam(self) -> int:
        return self.num_frames

    @property
    def softmax_scale(self) -> float:
        return 1.0 / math.sqrt(HEAD_DIM)

    def q_frame(self) -> np.ndarray:
        """int32 [n_q]: the latent frame of every query token."""
        return (np.arange(self.n_q) // self.tokens_per_frame).astype(np.int32)


def camera_480p(mode: int = 0) -> CameraProblem:
    """The 12,090 video tokens of a 480p segment (31 latent frames of 15 x 26)
    over its 31 camera tokens, 16 heads."""
    return CameraProblem("camera-xattn-480p", 31, 15 * 26, 16, mode)


def _windows_720p(rng: np.random.Generator, num_frames: int = 16,
                  n_actions: int = 6) -> Tuple[Tuple[int, int], ...]:
    """Random contiguous windows; redrawn until at least two overlap and at
    least one frame has no action."""
    while True:
        wins = []
        for _ in range(n_actions):
            b = int(rng.integers(0, num_frames))
            ln = int(rng.integers(1, 9))
            wins.append((b, min(num_frames, b + ln)))
        cover = np.zeros(num_frames, dtype=np.int64)
        for b, e in wins:
            cover[b:e] += 1
        if (cover > 1).any() and (cover == 0).any():
            return tuple(wins)


def session_720p(seed: int = 3) -> Problem:
    """16 frames x 22x40 grid, head 192, six 16-token tails with seeded
    windows (some overlapping, some frames uncovered); 6 cached segments."""
    rng = np.random.default_rng(seed)
    segs = []
    for _ in range(7):
        wins = _windows_720p(rng)
        segs.append(Segment(16, 22 * 40, 192, tuple(Action(16, b, e) for b, e in wins)))
    return Problem("720p-step", tuple(segs[:6]), (segs[6],), heads=16)


def packed_360k(seed: int = 4, budget: int = 360_000) -> Problem:
    """Training-shaped pack: segments with F~U{8..31} frames of 15x26 tokens,
    head 128, 1-6 tails of 16-48 tokens, windows b~U{0..F-1}, len~U{1..F};
    segments are drawn until the next one would overflow ``budget`` tokens."""
    rng = np.random.default_rng(seed)
    segs: List[Segment] = []
    total = 0
    while True:
        f = int(rng.integers(8, 32))
        n = int(rng.integers(1, 7))
        acts = []
        for _ in range(n):
            ln = int(rng.integers(16, 49))
            b = int(rng.integers(0, f))
            w = int(rng.integers(1, f + 1))
            acts.append(Action(ln, b, min(f, b + w)))
        seg = Segment(f, 390, 128, tuple(acts))
        if total + seg.n_tokens > budget:
            break
        segs.append(seg)
        total += seg.n_tokens
    return Problem("packed-360k", (), tuple(segs), heads=16)


# --------------------------------------------------------------------------
# small shapes for element-by-element parity (several tiles, ragged tails)
# --------------------------------------------------------------------------

def small_session(heads: int = 4, seed: int = 11) -> Problem:
    """3 cached + 1 current segment of 5 frames x 37 tokens; ragged tiles."""
    rng = np.random.default_rng(seed)
    segs = []
    for _ in range(4):
        acts = []
        for _ in range(3):
            b = int(rng.integers(0, 5))
            e = int(rng.integers(b + 1, 6))
            acts.append(Action(int(rng.integers(3, 12)), b, e))
        segs.append(Segment(5, 37, 19, tuple(acts)))
    return Problem("small-session", tuple(segs[:3]), (segs[3],), heads=heads)


def small_packed(heads: int = 3, seed: int = 12, n_segments: int = 6) -> Problem:
    """Packed small segments of varied shape, every token a query."""
    rng = np.random.default_rng(seed)
    segs = []
    for _ in range(n_segments):
        f = int(rng.integers(1, 7))
        g = int(rng.integers(5, 60))
        acts = []
        for _ in range(int(rng.integers(0, 5))):
            b = int(rng.integers(0, f))
            e = int(rng.integers(b + 1, f + 1))
            acts.append(Action(int(rng.integers(1, 20)), b, e))
        segs.append(Segment(f, g, int(rng.integers(0, 40)), tuple(acts)))
    return Problem("small-packed", (), tuple(segs), heads=heads)


def with_history(problem: Problem, segments: int) -> Problem:
    """The same call with a sliding window of ``segments`` earlier segments."""
    return dataclasses.replace(problem, name=f"{problem.name}-window{segments}",
                               history_segments=segments)


def n_query_tiles(problem: Problem) -> int:
    return (problem.n_query_tokens + 127) // 128


def n_key_tiles(problem: Problem) -> int:
    return (problem.n_cache_tokens + 127) // 128 + (problem.n_query_tokens + 127) // 128


def with_random_blocks(problem: Problem, keep: float, seed: int, group: int = 1) -> Problem:
    """The same call keeping a seeded random fraction ``keep`` of the key
    tiles, drawn once per ``group`` consecutive query tiles (neighbouring
    query tiles sharing their kept blocks, as a score-based selection
    tends to). Only video-only key tiles can be dropped; the others are kept
    whatever the draw."""
    rng = np.random.default_rng(seed)
    n_qt = n_query_tiles(problem)
    draw = rng.random(((n_qt + group - 1) // group, n_key_tiles(problem))) < keep
    mask = np.repeat(draw, group, axis=0)[:n_qt]
    return dataclasses.replace(problem, name=f"{problem.name}-blocks{int(round(100 * keep))}"
                                            + (f"g{group}" if group > 1 else ""),
                               keep_blocks=mask)


CONFIGS = {
    0: tiny_packed,
    1: session_480p_single_turn,
    2: session_480p_long,
    3: session_720p,
    4: packed_360k,
}


# --------------------------------------------------------------------------
# seeded tensors
# --------------------------------------------------------------------------

def randn_bf16(shape: Sequence[int], seed: int, scale: float = 1.0):
    """N(0, scale^2) drawn in fp32 on the CPU from ``seed``, rounded to bf16."""
    import torch

    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed))
    x = torch.randn(*shape, generator=g, dtype=torch.float32)
    if scale != 1.0:
        x.mul_(scale)
    return x.to(torch.bfloat16)


def make_inputs(problem: Problem, seed: int, q_scale: float = 1.0) -> Dict[str, object]:
    """Token-major bf16 tensors for one call.

    ``q``, ``k_cur``, ``v_cur``: [n_query_tokens, heads, 128].
    ``cache_k``, ``cache_v``: [n_cache_tokens, heads, 128], the K/V of the
    cached segments in time order (what was appended to the cache).
    Streams use seeds ``1000*seed + i``.
    """
    nq, nc, h = problem.n_query_tokens, problem.n_cache_tokens, problem.heads
    base = 1000 * int(seed)
    return {
        "q": randn_bf16((nq, h, HEAD_DIM), base + 0, q_scale),
        "k_cur": randn_bf16((nq, h, HEAD_DIM), base + 1),
        "v_cur": randn_bf16((nq, h, HEAD_DIM), base + 2),
        "cache_k": randn_bf16((nc, h, HEAD_DIM), base + 3),
        "cache_v": randn_bf16((nc, h, HEAD_DIM), base + 4),
    }


def sample_rows(n_rows: int, count: int, seed: int) -> np.ndarray:
    """Sorted distinct query rows: the first and last row, the last row of the
    last full 128-row tile, and a seeded uniform draw of the rest."""
    rng = np.random.default_rng(seed)
    fixed = {0, n_rows - 1, max(0, (n_rows // 128) * 128 - 1)}
    rest = rng.choice(n_rows, size=min(n_rows, count), replace=False)
    return np.array(sorted(fixed.union(int(r) for r in rest)), dtype=np.int64)
