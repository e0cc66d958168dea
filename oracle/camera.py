"""Camera cross-attention of one segment, in float64.

Test infrastructure (see the package docstring).

Equation 3 of [picx] Methodology > Model Architecture, "Camera-Trajectory
Conditioning": the visual tokens V attend, as queries, to the camera tokens
C as keys and values, and the result is added back:

    V~ = V + CrossAttn(V, C)

[onedev] "어떻게 쓰나" adds that there is one camera token per VAE latent
frame (the relative poses of each group of four frames, flattened to 64
numbers), that the camera tokens are aligned in time with the latent
frames, and that the cross-attention is added in every MMDiT block; [xyznot]
"Eyleme Duyarlı Nedensel Dikkat ve Kamera Koşullandırması" restates Eq. 3
with 64-dimensional relative camera tokens.

What is computed here is the attention core of that cross-attention, per
head of width 128, on already projected inputs (the projections of V and C
and the output projection are model weights):

    s_if = scale * <q_i, k_f>    for the camera tokens f that query i sees
    out_i = x_i + sum_f softmax_f(s_i) v_f

where x is the residual (V of Eq. 3). Which camera tokens a query sees is
left open by the pages beyond "time-aligned"; three readings are offered:

    CAM_ALL        every camera token of the segment (the default);
    CAM_OWN_FRAME  only the token of the query's own latent frame;
    CAM_UP_TO_FRAME the tokens of latent frames 0 .. the query's own.

A query whose latent frame lies outside [0, n_cam) sees no camera token in
the two frame-aligned modes and keeps out_i = x_i.
"""
from __future__ import annotations

import numpy as np

CAM_ALL, CAM_OWN_FRAME, CAM_UP_TO_FRAME = 0, 1, 2


def visible_camera_tokens(q_frame: np.ndarray, n_cam: int, mode: int) -> np.ndarray:
    """Boolean [n_q, n_cam]: which camera tokens each query sees."""
    q_frame = np.asarray(q_frame, dtype=np.int64)
    f = np.arange(n_cam)[None, :]
    qf = q_frame[:, None]
    inside = (qf >= 0) & (qf < n_cam)
    if mode == CAM_ALL:
        return np.ones((q_frame.shape[0], n_cam), dtype=bool)
    if mode == CAM_OWN_FRAME:
        return inside & (f == qf)
    if mode == CAM_UP_TO_FRAME:
        return inside & (f <= qf)
    raise ValueError("unknown camera attention mode")


def camera_cross_attention(q, k_cam, v_cam, x, q_frame, mode: int, scale: float) -> np.ndarray:
    """q, x: [n_q, heads, d]; k_cam, v_cam: [n_cam, heads, d]; q_frame:
    [n_q] latent-frame index of each query. Returns out [n_q, heads, d]
    (float64)."""
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k_cam, dtype=np.float64)
    v = np.asarray(v_cam, dtype=np.float64)
    out = np.array(x, dtype=np.float64)
    vis = visible_camera_tokens(q_frame, k.shape[0], mode)
    for h in range(q.shape[1]):
        s = (q[:, h, :] @ k[:, h, :].T) * scale
        s = np.where(vis, s, -np.inf)
        m = s.max(axis=1, initial=-np.inf)
        seen = np.isfinite(m)
        p = np.zeros_like(s)
        p[seen] = np.exp(s[seen] - m[seen, None])
        p[seen] /= p[seen].sum(axis=1, keepdims=True)
        out[:, h, :] += p @ v[:, h, :]
    return out
