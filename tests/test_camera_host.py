"""Argument checks of sca_camera_cross_attn, which the library makes on the
host before any CUDA call (include/sca.h documents each refusal). The
pointers are plain addresses that are never dereferenced: every case here is
refused before a launch."""
import math

import pytest

from segment_causal_masked_b200 import sca


class _T:
    """Stands in for a tensor: a shape and an address."""

    def __init__(self, shape, addr):
        self.shape = shape
        self.addr = addr

    def data_ptr(self):
        return self.addr


N_Q, N_CAM, H = 100, 8, 2
ROW = H * 128 * 2  # bytes of one query row
Q, X, OUT, K, V, FR = (0x100000, 0x200000, 0x300000, 0x400000, 0x500000, 0x600000)


def _call(q=Q, x=X, out=OUT, k=K, v=V, frame=FR, n_q=N_Q, n_cam=N_CAM, mode=sca.CAM_UP_TO_FRAME,
          scale=0.088):
    qs = (n_q, H, 128)
    ks = (n_cam, H, 128)
    with pytest.raises(sca.ScaError) as e:
        sca.camera_cross_attn(_T(qs, q), _T(ks, k), _T(ks, v), _T(qs, x), _T(qs, out),
                              None if frame is None else _T((n_q,), frame), mode, scale, stream=0)
    return e.value.code, str(e.value)


@pytest.mark.parametrize("n_cam", [0, -1, sca.MAX_CAMERA_TOKENS + 1])
def test_camera_token_count_is_bounded(n_cam):
    code, msg = _call(n_cam=n_cam)
    assert code == sca.ERR_INVALID_ARG and "n_cam" in msg


def test_unknown_mode_and_scale():
    assert _call(mode=3)[0] == sca.ERR_INVALID_ARG
    assert _call(scale=math.nan)[0] == sca.ERR_INVALID_ARG
    assert _call(scale=math.inf)[0] == sca.ERR_INVALID_ARG


def test_frame_modes_need_the_frame_index():
    for mode in (sca.CAM_OWN_FRAME, sca.CAM_UP_TO_FRAME):
        code, msg = _call(frame=None, mode=mode)
        assert code == sca.ERR_INVALID_ARG and "q_frame" in msg


@pytest.mark.parametrize("which", ["q", "x", "out", "k", "v"])
def test_misaligned_pointers_are_refused(which):
    code, _ = _call(**{which: {"q": Q, "x": X, "out": OUT, "k": K, "v": V}[which] + 8})
    assert code == sca.ERR_MISALIGNED


def test_null_pointers_are_refused():
    assert _call(k=0)[0] == sca.ERR_INVALID_ARG
    assert _call(q=0)[0] == sca.ERR_INVALID_ARG


@pytest.mark.parametrize("out", [Q + 16 * ROW, X + ROW, K - 16, V + 256])
def test_out_may_not_overlap_an_input_other_than_x(out):
    code, msg = _call(out=out)
    assert code == sca.ERR_INVALID_ARG and "overlaps" in msg


def test_row_count_is_bounded():
    assert _call(n_q=-1)[0] == sca.ERR_INVALID_ARG
    assert _call(n_q=2 ** 31 - 1)[0] == sca.ERR_UNSUPPORTED


def test_shapes_are_checked_by_the_binding():
    with pytest.raises(ValueError):
        sca.camera_cross_attn(_T((4, H, 128), Q), _T((3, H, 128), K), _T((3, H, 64), V),
                              _T((4, H, 128), X), _T((4, H, 128), OUT), stream=0)
