"""Gradients of the masked attention, in float64 (test infrastructure).

The pages train the model with this attention (the packed, FLOPs-balanced
training batches of [picx.dev summary, Methodology › Training Infrastructure,
Eq. 6]) but print no backward pass. Its gradients follow from the forward's
plain definition (attention.py), per head h, with S = scale · Q Kᵀ on the
visible pairs, P = row softmax of S (a row that sees nothing has P = 0) and
O = P V. For an upstream gradient dO:

    dV = Pᵀ dO
    dP = dO Vᵀ
    D_i = Σ_j P_ij dP_ij                    (= Σ_d dO_id O_id)
    dS = P ∘ (dP − D)                         (row-wise broadcast of D)
    dQ = scale · dS K,   dK = scale · dSᵀ Q

All arrays are [tokens, heads, 128]. Keys are the layout's keys (cache, then
current); queries are the current tokens.
"""
from __future__ import annotations

from typing import Optional, Sequence, Tuple

import numpy as np

from .rule import Layout

ROW_CHUNK = 2048


def _probs(q_h: np.ndarray, k_h: np.ndarray, mask: np.ndarray, scale: float) -> np.ndarray:
    """Row softmax of scale · q kᵀ over the visible keys (zero rows stay 0)."""
    s = scale * (q_h @ k_h.T)
    s = np.where(mask, s, -np.inf)
    m = s.max(axis=1, keepdims=True)
    m = np.where(np.isfinite(m), m, 0.0)
    e = np.where(mask, np.exp(s - m), 0.0)
    z = e.sum(axis=1, keepdims=True)
    return np.divide(e, z, out=np.zeros_like(e), where=z > 0)


def attention_backward(layout: Layout, q: np.ndarray, k_all: np.ndarray, v_all: np.ndarray,
                       d_o: np.ndarray, scale: float) -> Tuple[np.ndarray, np.ndarray, np.ndarray]:
    """dQ [n_q, H, 128], dK and dV [n_keys, H, 128] (float64)."""
    q, k_all, v_all, d_o = (np.asarray(a, dtype=np.float64) for a in (q, k_all, v_all, d_o))
    n_q, heads, _ = q.shape
    dq = np.zeros_like(q)
    dk = np.zeros_like(k_all)
    dv = np.zeros_like(v_all)
    for r0 in range(0, n_q, ROW_CHUNK):
        r1 = min(n_q, r0 + ROW_CHUNK)
        mask = layout.mask_rows(range(r0, r1))
        for h in range(heads):
            p = _probs(q[r0:r1, h], k_all[:, h], mask, scale)
            do_h = d_o[r0:r1, h]
            dv[:, h] += p.T @ do_h
            dp = do_h @ v_all[:, h].T
            d = (p * dp).sum(axis=1, keepdims=True)
            ds = p * (dp - d)
            dq[r0:r1, h] = scale * (ds @ k_all[:, h])
            dk[:, h] += scale * (ds.T @ q[r0:r1, h])
    return dq, dk, dv


def dq_rows(layout: Layout, q: np.ndarray, k_all: np.ndarray, v_all: np.ndarray,
            d_o: np.ndarray, rows: Sequence[int], scale: float,
            heads: Optional[Sequence[int]] = None) -> np.ndarray:
    """dQ of the given query rows only ([len(rows), len(heads), 128]): a row's
    gradient needs only that row's probabilities."""
    rows = np.asarray(rows, dtype=np.int64)
    heads = list(range(q.shape[1])) if heads is None else list(heads)
    out = np.zeros((len(rows), len(heads), q.shape[2]))
    for i, r in enumerate(rows):
        mask = layout.mask_row(int(r))[None, :]
        for j, h in enumerate(heads):
            qh = np.asarray(q[r:r + 1, h], dtype=np.float64)
            kh = np.asarray(k_all[:, h], dtype=np.float64)
            p = _probs(qh, kh, mask, scale)
            dp = np.asarray(d_o[r:r + 1, h], dtype=np.float64) @ np.asarray(v_all[:, h], dtype=np.float64).T
            ds = p * (dp - (p * dp).sum())
            out[i, j] = scale * (ds @ kh)[0]
    return out
