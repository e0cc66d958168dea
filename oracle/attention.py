"""Dense masked softmax attention on the explicit mask, in float64.

Test infrastructure (see the package docstring).

Each query row sees the keys its mask row allows ([picx] Model Architecture,
"Action-Aware Causal Attention (Figure 6b)"); the attention itself is the
joint softmax attention of the MMDiT blocks with 16 heads of width 128
([picx] "Theoretical Foundation"; [gpts24] "Inside the Architecture"). Per
head h and query row i:

    s_ik = scale * <q_i, k_k>          (scale = 1/sqrt(128))
    s_ik = -inf where the mask forbids (i, k)
    O_i  = sum_k softmax_k(s_i) v_k,   LSE_i = log sum_k exp(s_ik)

A row that sees no key gets O = 0 and LSE = -inf.
"""
from __future__ import annotations

from typing import Optional, Sequence, Tuple

import numpy as np

from .rule import Layout


def masked_attention(q: np.ndarray, k: np.ndarray, v: np.ndarray,
                     mask: np.ndarray, scale: float,
                     dtype=np.float64) -> Tuple[np.ndarray, np.ndarray]:
    """Softmax attention of one head.

    q: [m, d]; k, v: [n, d]; mask: [m, n] bool (True = visible).
    Returns O [m, d] and LSE [m] (natural log).
    """
    q = np.asarray(q, dtype=dtype)
    k = np.asarray(k, dtype=dtype)
    v = np.asarray(v, dtype=dtype)
    s = (q @ k.T) * dtype(scale)
    s = np.where(mask, s, -np.inf)
    m = s.max(axis=1, initial=-np.inf)
    empty = ~np.isfinite(m)
    m_safe = np.where(empty, 0.0, m)
    p = np.exp(s - m_safe[:, None])
    l = p.sum(axis=1)
    with np.errstate(invalid="ignore", divide="ignore"):
        o = (p @ v) / l[:, None]
        lse = m_safe + np.log(l)
    o[empty] = 0.0
    lse[empty] = -np.inf
    return o, lse


def attention_rows(layout: Layout, q: np.ndarray, k_all: np.ndarray, v_all: np.ndarray,
                   rows: Sequence[int], scale: float,
                   heads: Optional[Sequence[int]] = None, block: int = 256,
                   dtype=np.float64) -> Tuple[np.ndarray, np.ndarray]:
    """Outputs of the selected query rows.

    q: [n_queries, H, d]; k_all, v_all: [n_keys, H, d] (cache then current),
    any float dtype holding the bf16 inputs exactly.
    Returns O [len(rows), H', d] and LSE [H', len(rows)] for the heads listed.
    """
    rows = np.asarray(rows, dtype=np.int64)
    heads = list(range(q.shape[1])) if heads is None else list(heads)
    o = np.zeros((len(rows), len(heads), q.shape[2]), dtype=dtype)
    lse = np.zeros((len(heads), len(rows)), dtype=dtype)
    for hi, h in enumerate(heads):
        kh = np.asarray(k_all[:, h, :], dtype=dtype)
        vh = np.asarray(v_all[:, h, :], dtype=dtype)
        for b0 in range(0, len(rows), block):
            r = rows[b0:b0 + block]
            mask = layout.mask_rows(r)
            ob, lb = masked_attention(q[r, h, :], kh, vh, mask, scale, dtype)
            o[b0:b0 + len(r), hi, :] = ob
            lse[hi, b0:b0 + len(r)] = lb
    return o, lse


def attention(layout: Layout, q: np.ndarray, k_all: np.ndarray, v_all: np.ndarray,
              scale: float, dtype=np.float64) -> Tuple[np.ndarray, np.ndarray]:
    """All query rows and heads: O [n_queries, H, d], LSE [H, n_queries]."""
    return attention_rows(layout, q, k_all, v_all, np.arange(layout.n_queries), scale,
                          dtype=dtype)
