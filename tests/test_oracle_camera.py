"""Pins of the camera cross-attention oracle (Eq. 3, [picx] "Camera-Trajectory
Conditioning"; one camera token per latent frame, [onedev] "어떻게 쓰나").

The pages print no numeric example. The oracle is checked against torch's
scaled_dot_product_attention on the CPU (an independent routine), closed
forms (one visible token gives its value row; equal keys give the mean of
the visible values; no visible token keeps the residual) and invariants
(the order of camera tokens, in the mode where every token is seen).
"""
import numpy as np
import pytest
import torch

from oracle import camera as ocam

D = 128


def _inputs(n_q, n_cam, heads, seed, sharp=1.0):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((n_q, heads, D)) * sharp
    k = rng.standard_normal((n_cam, heads, D))
    v = rng.standard_normal((n_cam, heads, D))
    x = rng.standard_normal((n_q, heads, D))
    frame = rng.integers(0, n_cam, n_q)
    return q, k, v, x, frame


def _sdpa(q, k, v, mask, scale):
    qt = torch.from_numpy(np.ascontiguousarray(q.transpose(1, 0, 2)))
    kt = torch.from_numpy(np.ascontiguousarray(k.transpose(1, 0, 2)))
    vt = torch.from_numpy(np.ascontiguousarray(v.transpose(1, 0, 2)))
    o = torch.nn.functional.scaled_dot_product_attention(
        qt, kt, vt, attn_mask=torch.from_numpy(mask), scale=scale)
    return o.numpy().transpose(1, 0, 2)


@pytest.mark.parametrize("mode", [ocam.CAM_ALL, ocam.CAM_UP_TO_FRAME])
@pytest.mark.parametrize("n_cam", [1, 7, 31])
@pytest.mark.parametrize("sharp", [1.0, 6.0])
def test_matches_torch_sdpa(mode, n_cam, sharp):
    """Every query sees at least one token in these modes, so SDPA's masked
    softmax applies row by row."""
    q, k, v, x, frame = _inputs(53, n_cam, 3, 11, sharp)
    scale = 1.0 / np.sqrt(D)
    out = ocam.camera_cross_attention(q, k, v, x, frame, mode, scale)
    mask = ocam.visible_camera_tokens(frame, n_cam, mode)
    ref = x + _sdpa(q, k, v, mask, scale)
    assert np.abs(out - ref).max() < 1e-12


def test_own_frame_adds_that_frames_value_row():
    """One visible token: its softmax weight is exactly 1."""
    q, k, v, x, frame = _inputs(40, 9, 2, 12, 8.0)
    out = ocam.camera_cross_attention(q, k, v, x, frame, ocam.CAM_OWN_FRAME, 0.0883883)
    np.testing.assert_array_equal(out, x + v[frame])


def test_single_camera_token():
    q, k, v, x, frame = _inputs(17, 1, 4, 13)
    out = ocam.camera_cross_attention(q, k, v, x, frame, ocam.CAM_ALL, 0.0883883)
    np.testing.assert_array_equal(out, x + v[0][None])


def test_equal_keys_give_the_mean_of_the_visible_values():
    q, k, v, x, frame = _inputs(30, 12, 2, 14)
    k[:] = k[:1]
    out = ocam.camera_cross_attention(q, k, v, x, frame, ocam.CAM_UP_TO_FRAME, 0.0883883)
    for i in range(30):
        np.testing.assert_allclose(out[i], x[i] + v[: frame[i] + 1].mean(0), atol=1e-12)


def test_frames_outside_the_segment_keep_the_residual():
    q, k, v, x, _ = _inputs(6, 5, 2, 15)
    frame = np.array([-1, 5, 7, 0, 4, 2])
    for mode in (ocam.CAM_OWN_FRAME, ocam.CAM_UP_TO_FRAME):
        out = ocam.camera_cross_attention(q, k, v, x, frame, mode, 0.0883883)
        np.testing.assert_array_equal(out[:3], x[:3])
        assert not np.array_equal(out[3:], x[3:])


def test_all_mode_ignores_the_order_of_camera_tokens():
    q, k, v, x, frame = _inputs(25, 16, 2, 16, 3.0)
    perm = np.random.default_rng(1).permutation(16)
    a = ocam.camera_cross_attention(q, k, v, x, frame, ocam.CAM_ALL, 0.0883883)
    b = ocam.camera_cross_attention(q, k[perm], v[perm], x, frame, ocam.CAM_ALL, 0.0883883)
    assert np.abs(a - b).max() < 1e-12


def test_visibility_sets():
    frame = np.array([0, 3, 4, -2])
    vis = ocam.visible_camera_tokens(frame, 4, ocam.CAM_UP_TO_FRAME)
    assert vis.tolist() == [[1, 0, 0, 0], [1, 1, 1, 1], [0, 0, 0, 0], [0, 0, 0, 0]]
    vis = ocam.visible_camera_tokens(frame, 4, ocam.CAM_OWN_FRAME)
    assert vis.tolist() == [[1, 0, 0, 0], [0, 0, 0, 1], [0, 0, 0, 0], [0, 0, 0, 0]]
    assert ocam.visible_camera_tokens(frame, 4, ocam.CAM_ALL).all()
    with pytest.raises(ValueError):
        ocam.visible_camera_tokens(frame, 4, 3)
