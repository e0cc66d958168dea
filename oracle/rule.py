"""Token layout and the visibility rule, as explicit sets of visible keys.

Test infrastructure (see the package docstring). Float-free.

The rule, from the pages:

* Attention is bidirectional inside a segment and causal across segments:
  a query of segment j never sees a later segment ([picx] Model
  Architecture, "Segment-wise Causal Attention"; [xyznot] "Eyleme Duyarlı
  Nedensel Dikkat").
* The text of a segment is a descriptive head followed by action tails
  a_0..a_n, each with a window of frames. A query inside an action's window
  sees that action's tail and the head; heads stay visible to every later
  segment, tails never leave their own segment ([picx] "Action-Aware Causal
  Attention (Figure 6b)"; [onedev] "무엇과 다른가"; [gpts24] "Inside the
  Architecture").

Readings where the pages are silent (each is listed in the design notes):

* Token order inside a segment: video frame by frame (frame-major), then the
  head, then the tails in action order; segments in time order.
* A video query in a frame covered by several windows sees every covering
  tail; a frame no window covers sees no tail.
* Text queries, policy ``OWN_TAIL`` (the default): a head query sees its own
  segment's video and head; a query in tail a also sees tail a; neither sees
  an earlier segment. Policy ``FULL_SEGMENT``: text queries see their whole
  own segment and, like video queries, the video and heads of earlier
  segments.
* Windows are half-open latent-frame ranges local to the segment.

Two options for single-GPU inference, named on the pages without their rules
([picx] "Inference": sliding-window attention and sparse attention keeping a
quarter of the video blocks), read here as:

* ``history`` W >= 0: a query of segment s sees earlier segments s-W .. s-1
  only (its own segment as always); W < 0 keeps the whole history.
* ``keep_blocks`` [query tiles, key tiles]: a False entry drops, for the
  queries of that 128-query tile, every key of that 128-key tile when the key
  tile holds video tokens only ("a video block"); tiles with any text key are
  always kept. Tiles are those of the schedule (schedule.py).
"""
from __future__ import annotations

import dataclasses
from typing import Dict, List, Sequence, Tuple

import numpy as np

VIDEO, HEAD, TAIL = "video", "head", "tail"
OWN_TAIL, FULL_SEGMENT = 0, 1


@dataclasses.dataclass(frozen=True)
class Span:
    """Key-index ranges of one segment inside the key sequence."""

    segment: int
    video: Tuple[int, int]
    head: Tuple[int, int]
    tails: Tuple[Tuple[int, int], ...]
    windows: Tuple[Tuple[int, int], ...]
    num_frames: int
    tokens_per_frame: int
    stop: int           # one past the segment's last key


def _check_segment(seg) -> None:
    if seg.num_frames < 1 or seg.tokens_per_frame < 1 or seg.head_len < 0:
        raise ValueError("segment needs >= 1 frame, >= 1 token per frame, head >= 0")
    for a in seg.actions:
        if a.length < 1 or not (0 <= a.begin < a.end <= seg.num_frames):
            raise ValueError("action needs length >= 1 and 0 <= begin < end <= frames")


def spans(segments: Sequence) -> List[Span]:
    """Lay the segments end to end and return each one's key ranges."""
    out = []
    pos = 0
    for i, seg in enumerate(segments):
        _check_segment(seg)
        nv = seg.num_frames * seg.tokens_per_frame
        video = (pos, pos + nv)
        head = (video[1], video[1] + seg.head_len)
        tails = []
        t = head[1]
        for a in seg.actions:
            tails.append((t, t + a.length))
            t += a.length
        out.append(Span(i, video, head, tuple(tails),
                        tuple((a.begin, a.end) for a in seg.actions),
                        seg.num_frames, seg.tokens_per_frame, t))
        pos = t
    return out


@dataclasses.dataclass(frozen=True)
class QueryRun:
    """Consecutive queries that see the same keys (one frame, a head, a tail)."""

    start: int          # first query index (query sequence)
    stop: int
    segment: int        # global segment index (cache segments first)
    kind: str
    frame: int          # video frame, or -1
    action: int         # tail's action index, or -1


def query_runs(cached: Sequence, current: Sequence) -> List[QueryRun]:
    """Queries are the tokens of the current segments, in key order."""
    runs = []
    n_cached = len(cached)
    q = 0
    for j, seg in enumerate(current):
        g = n_cached + j
        for f in range(seg.num_frames):
            runs.append(QueryRun(q, q + seg.tokens_per_frame, g, VIDEO, f, -1))
            q += seg.tokens_per_frame
        if seg.head_len:
            runs.append(QueryRun(q, q + seg.head_len, g, HEAD, -1, -1))
            q += seg.head_len
        for a, act in enumerate(seg.actions):
            runs.append(QueryRun(q, q + act.length, g, TAIL, -1, a))
            q += act.length
    return runs


def visible_key_ranges(all_spans: Sequence[Span], run: QueryRun,
                       policy: int = OWN_TAIL, history: int = -1) -> List[Tuple[int, int]]:
    """The key ranges a query of ``run`` may attend to."""
    text_query = run.kind != VIDEO
    sees_past = (not text_query) or policy == FULL_SEGMENT
    out: List[Tuple[int, int]] = []
    for sp in all_spans:
        if sp.segment > run.segment:
            continue                                   # never a later segment
        if sp.segment < run.segment:
            in_window = history < 0 or run.segment - sp.segment <= history
            if sees_past and in_window:
                out += [sp.video, sp.head]             # past video + head; past tails never
            continue
        out += [sp.video, sp.head]                     # own segment: bidirectional
        for a, (tail, (b, e)) in enumerate(zip(sp.tails, sp.windows)):
            if run.kind == VIDEO:
                if b <= run.frame < e:
                    out.append(tail)                   # inside this action's window
            elif policy == FULL_SEGMENT or (run.kind == TAIL and a == run.action):
                out.append(tail)
    return [r for r in out if r[1] > r[0]]


class Layout:
    """Key spans and query runs of one call (cached segments, then current)."""

    def __init__(self, cached: Sequence, current: Sequence, policy: int = OWN_TAIL,
                 history: int = -1, keep_blocks=None):
        self.cached = tuple(cached)
        self.current = tuple(current)
        self.policy = policy
        self.history = history
        self.spans = spans(list(cached) + list(current))
        self.runs = query_runs(cached, current)
        self.n_keys = self.spans[-1].stop if self.spans else 0
        self.n_cache = self.spans[len(cached) - 1].stop if cached else 0
        self.n_queries = self.runs[-1].stop if self.runs else 0
        self._run_starts = np.array([r.start for r in self.runs], dtype=np.int64)
        self._row_cache: Dict[Tuple[int, int], np.ndarray] = {}
        self.keep_blocks = None if keep_blocks is None else np.asarray(keep_blocks, dtype=bool)
        if self.keep_blocks is not None:
            # key tiles of each source (128 keys, cache first), and which hold video only
            is_video = np.zeros(self.n_keys, dtype=bool)
            for sp in self.spans:
                is_video[sp.video[0]:sp.video[1]] = True
            self._tiles = []
            for base, n in ((0, self.n_cache), (self.n_cache, self.n_queries)):
                for t0 in range(0, n, 128):
                    a, b = base + t0, base + min(n, t0 + 128)
                    self._tiles.append((a, b, bool(is_video[a:b].all())))
            n_qt = (self.n_queries + 127) // 128
            if self.keep_blocks.shape != (n_qt, len(self._tiles)):
                raise ValueError("keep_blocks must be [query tiles, key tiles]")

    @classmethod
    def of(cls, problem) -> "Layout":
        return cls(problem.cached, problem.current, problem.textq_policy,
                   getattr(problem, "history_segments", -1), getattr(problem, "keep_blocks", None))

    def run_of(self, query: int) -> QueryRun:
        i = int(np.searchsorted(self._run_starts, query, side="right")) - 1
        return self.runs[i]

    def ranges(self, query: int) -> List[Tuple[int, int]]:
        """Visible key ranges of ``query`` (before any dropped video block)."""
        return visible_key_ranges(self.spans, self.run_of(query), self.policy, self.history)

    def mask_row(self, query: int) -> np.ndarray:
        """Boolean row of the explicit mask."""
        run = self.run_of(query)
        qt = query // 128 if self.keep_blocks is not None else -1
        key = (run.start, qt)
        row = self._row_cache.get(key)
        if row is None:
            row = np.zeros(self.n_keys, dtype=bool)
            for a, b in visible_key_ranges(self.spans, run, self.policy, self.history):
                row[a:b] = True
            if self.keep_blocks is not None:
                for kt, (a, b, video_only) in enumerate(self._tiles):
                    if video_only and not self.keep_blocks[qt, kt]:
                        row[a:b] = False             # a dropped video block
            if len(self._row_cache) < max(16, (1 << 28) // max(1, self.n_keys)):
                self._row_cache[key] = row
        return row

    def mask_rows(self, rows: Sequence[int]) -> np.ndarray:
        rows = np.asarray(rows, dtype=np.int64)
        out = np.empty((len(rows), self.n_keys), dtype=bool)
        for i, r in enumerate(rows):
            out[i] = self.mask_row(int(r))
        return out

    def mask(self) -> np.ndarray:
        """The whole explicit mask [n_queries, n_keys] (small layouts only)."""
        return self.mask_rows(np.arange(self.n_queries))

    def unmasked_pairs(self) -> int:
        """A of Eq. 6 ([picx] Training Infrastructure; [xyznot] "Dağıtık
        Paketleme FLOP Tahmini"): the number of (query, key) pairs whose mask
        entry is not -inf, summed run by run from the visible ranges (row by
        row from the explicit mask when video blocks are dropped)."""
        if self.keep_blocks is not None:
            return int(sum(int(self.mask_row(q).sum()) for q in range(self.n_queries)))
        total = 0
        for run in self.runs:
            seen = sum(b - a for a, b in
                       visible_key_ranges(self.spans, run, self.policy, self.history))
            total += (run.stop - run.start) * seen
        return total
