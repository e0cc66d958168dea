"""GPU parity of the camera cross-attention (sca_camera_cross_attn) against the
oracle (Eq. 3 of [picx] "Camera-Trajectory Conditioning"; one camera token
per latent frame, [onedev] "어떻게 쓰나").

Bar: every output element within 1e-2 · max(1, |ref|) of the float64 oracle
on the same bf16 inputs, and a relative L2 error <= 5e-3 (derived: P is
rounded to bf16 before its product, 2^-9 relative, and the output is one
bf16 rounding, 2^-9 relative, of x + the attention). Where a query sees a
single camera token its weight is exactly 1 and the output is the bf16
rounding of x + v, which the test checks bit for bit.
"""
import numpy as np
import pytest
import torch

from oracle import camera as ocam

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

from segment_causal_masked_b200 import sca  # noqa: E402

D = 128
SCALE = D ** -0.5


def _inputs(n_q, n_cam, heads, seed, sharp=1.0):
    g = torch.Generator().manual_seed(seed)
    q = (torch.randn(n_q, heads, D, generator=g) * sharp).bfloat16()
    k = torch.randn(n_cam, heads, D, generator=g).bfloat16()
    v = torch.randn(n_cam, heads, D, generator=g).bfloat16()
    x = torch.randn(n_q, heads, D, generator=g).bfloat16()
    frame = torch.randint(0, n_cam, (n_q,), generator=g, dtype=torch.int32)
    return q, k, v, x, frame


def _run(q, k, v, x, frame, mode, out=None):
    qd, kd, vd, xd, fd = (t.cuda() for t in (q, k, v, x, frame))
    od = torch.empty_like(xd) if out is None else out
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    sca.camera_cross_attn(qd, kd, vd, xd, od, fd, mode, SCALE, st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    return od.cpu()


def _ref(q, k, v, x, frame, mode):
    return ocam.camera_cross_attention(q.float().numpy(), k.float().numpy(), v.float().numpy(),
                                       x.float().numpy(), frame.numpy(), mode, SCALE)


def _check(out, ref):
    o = out.float().numpy().astype(np.float64)
    d = np.abs(o - ref)
    assert (d <= 1e-2 * np.maximum(1.0, np.abs(ref))).all(), f"max |d| = {d.max()}"
    assert np.linalg.norm(o - ref) <= 5e-3 * np.linalg.norm(ref)


@pytest.mark.parametrize("mode", [sca.CAM_ALL, sca.CAM_OWN_FRAME, sca.CAM_UP_TO_FRAME])
@pytest.mark.parametrize("n_cam", [1, 5, 16, 31, 48, 64])
def test_matches_oracle(mode, n_cam):
    q, k, v, x, frame = _inputs(301, n_cam, 3, 100 + n_cam + 7 * mode)
    _check(_run(q, k, v, x, frame, mode), _ref(q, k, v, x, frame, mode))


@pytest.mark.parametrize("n_q", [1, 15, 16, 17, 127, 128, 129, 255, 256, 257, 2048])
@pytest.mark.parametrize("sharp", [1.0, 8.0])
def test_ragged_rows_and_sharp_scores(n_q, sharp):
    q, k, v, x, frame = _inputs(n_q, 31, 16, 200 + n_q, sharp)
    _check(_run(q, k, v, x, frame, sca.CAM_ALL), _ref(q, k, v, x, frame, sca.CAM_ALL))


def test_own_frame_is_exact():
    """One visible token: out = bf16(x + v[frame]) bit for bit."""
    q, k, v, x, frame = _inputs(500, 31, 4, 300, 8.0)
    out = _run(q, k, v, x, frame, sca.CAM_OWN_FRAME)
    ref = torch.from_numpy(x.double().numpy() + v.double().numpy()[frame.long().numpy()]).bfloat16()
    assert torch.equal(out, ref)


def test_frames_outside_the_segment_keep_the_residual():
    q, k, v, x, _ = _inputs(64, 8, 2, 301)
    frame = torch.tensor([-3, 8, 9, 100] * 16, dtype=torch.int32)
    for mode in (sca.CAM_OWN_FRAME, sca.CAM_UP_TO_FRAME):
        assert torch.equal(_run(q, k, v, x, frame, mode), x)


def test_in_place_equals_out_of_place():
    q, k, v, x, frame = _inputs(777, 20, 16, 302)
    a = _run(q, k, v, x, frame, sca.CAM_UP_TO_FRAME)
    xd = x.cuda()
    sca.camera_cross_attn(q.cuda(), k.cuda(), v.cuda(), xd, xd, frame.cuda(),
                          sca.CAM_UP_TO_FRAME, SCALE)
    torch.cuda.synchronize()
    assert torch.equal(xd.cpu(), a)


def test_repeat_is_bit_identical_and_zero_rows_launch_nothing():
    q, k, v, x, frame = _inputs(129, 12, 2, 303)
    a = _run(q, k, v, x, frame, sca.CAM_ALL)
    b = _run(q, k, v, x, frame, sca.CAM_ALL)
    assert torch.equal(a, b)
    e = torch.empty(0, 2, D, dtype=torch.bfloat16, device="cuda")
    sca.camera_cross_attn(e, k.cuda(), v.cuda(), e, e, None, sca.CAM_ALL, SCALE)
    torch.cuda.synchronize()


def test_480p_segment_sampled_rows():
    """The bench's shape: the 12,090 video queries of a 480p segment (31
    latent frames of 390 tokens) over its 31 camera tokens, 16 heads;
    sampled rows against the oracle."""
    n_q, n_cam, heads = 31 * 390, 31, 16
    q, k, v, x, _ = _inputs(n_q, n_cam, heads, 304)
    frame = (torch.arange(n_q, dtype=torch.int32) // 390)
    out = _run(q, k, v, x, frame, sca.CAM_UP_TO_FRAME)
    rows = np.unique(np.r_[0, n_q - 1, np.random.default_rng(5).choice(n_q, 256, replace=False)])
    ref = _ref(q[rows], k, v, x[rows], frame[rows], sca.CAM_UP_TO_FRAME)
    _check(out[rows], ref)


@pytest.mark.parametrize("n_cam, mode", [(9, 1), (40, 2), (64, 0), (64, 2)])
def test_long_ranges_of_tiles_per_cta(n_cam, mode):
    """Enough rows that every CTA streams several 128-row tiles, across head
    changes, for each width of the camera tile; sampled rows."""
    n_q, heads = 9000, 16
    q, k, v, x, _ = _inputs(n_q, n_cam, heads, 400 + n_cam + mode)
    frame = (torch.arange(n_q, dtype=torch.int32) * n_cam // n_q)
    out = _run(q, k, v, x, frame, mode)
    rows = np.unique(np.r_[0, 127, 128, n_q - 1,
                           np.random.default_rng(n_cam).choice(n_q, 200, replace=False)])
    _check(out[rows], _ref(q[rows], k, v, x[rows], frame[rows], mode))


def test_unaligned_frame_index():
    """A q_frame view one element into its buffer (not 16-byte aligned)."""
    q, k, v, x, frame = _inputs(333, 24, 4, 305)
    buf = torch.zeros(frame.numel() + 1, dtype=torch.int32)
    buf[1:] = frame
    fd = buf.cuda()[1:]
    assert fd.data_ptr() % 16 != 0
    od = torch.empty(q.shape, dtype=torch.bfloat16, device="cuda")
    sca.camera_cross_attn(q.cuda(), k.cuda(), v.cuda(), x.cuda(), od, fd, sca.CAM_UP_TO_FRAME,
                          SCALE)
    torch.cuda.synchronize()
    _check(od.cpu(), _ref(q, k, v, x, frame, sca.CAM_UP_TO_FRAME))



def test_calls_replay_from_a_cuda_graph():
    """Captured in a CUDA graph (each call with its own tensor maps), the
    calls replay to the eager results bit for bit."""
    q, k, v, x, frame = _inputs(1000, 31, 16, 307)
    x2 = x.flip(0).contiguous()
    eager = [_run(q, k, v, xx, frame, sca.CAM_UP_TO_FRAME) for xx in (x, x2)]
    qd, kd, vd, fd = q.cuda(), k.cuda(), v.cuda(), frame.cuda()
    xs = [x.cuda(), x2.cuda()]
    outs = [torch.empty_like(xs[0]) for _ in range(2)]
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, capture_error_mode="relaxed"):
        for xx, oo in zip(xs, outs):
            sca.camera_cross_attn(qd, kd, vd, xx, oo, fd, sca.CAM_UP_TO_FRAME, SCALE, st,
                                  torch.cuda.current_stream().cuda_stream)
    for o in outs:
        o.zero_()
    graph.replay()
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    for o, e in zip(outs, eager):
        assert torch.equal(o.cpu(), e)


def test_pipeline_timeout_aborts_cleanly():
    """With the pipeline-wait limit at 0 a role gives up at its first wait
    that is not already complete: the status word reads
    SCA_ERR_DEVICE_TIMEOUT, every role lets its own copies and products land
    before the CTA frees its tensor memory and exits, and the device keeps
    answering: with the default limit back the next call is right. (A
    try-wait may itself block until the phase completes, so the call is
    repeated until one of them gives up.)"""
    q, k, v, x, frame = _inputs(32768, 31, 16, 306)
    qd, kd, vd, xd, fd = (t.cuda() for t in (q, k, v, x, frame))
    od = torch.empty_like(xd)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    try:
        sca.set_pipeline_timeout_ns(0)
        for _ in range(10):
            sca.camera_cross_attn(qd, kd, vd, xd, od, fd, sca.CAM_UP_TO_FRAME, SCALE, st)
            torch.cuda.synchronize()
            if int(st.item()) != 0:
                break
    finally:
        sca.set_pipeline_timeout_ns(2_000_000_000)
    assert int(st.item()) == sca.ERR_DEVICE_TIMEOUT
    assert float((torch.ones(4, device="cuda") * 2).sum().item()) == 8.0
    rows = np.arange(0, 32768, 61)
    out = _run(q, k, v, x, frame, sca.CAM_UP_TO_FRAME)
    _check(out[rows], _ref(q[rows], k, v, x[rows], frame[rows], sca.CAM_UP_TO_FRAME))


@pytest.mark.parametrize("mode", [sca.CAM_OWN_FRAME, sca.CAM_UP_TO_FRAME])
def test_random_frames_over_many_tiles_per_cta(mode):
    """Random frames (a stale row rarely matches) with 28 tiles of 128 rows
    per CTA, three calls: a warp that read another tile's x (the race of a
    shared x-stage ring) makes whole 32-row blocks wrong in some calls."""
    q, k, v, x, frame = _inputs(32768, 31, 16, 308 + mode)
    rows = np.arange(0, 32768, 37)
    ref = _ref(q[rows], k, v, x[rows], frame[rows], mode)
    qd, kd, vd, xd, fd = (t.cuda() for t in (q, k, v, x, frame))
    for _ in range(3):
        od = torch.empty_like(xd)
        st = torch.zeros(1, dtype=torch.int32, device="cuda")
        sca.camera_cross_attn(qd, kd, vd, xd, od, fd, mode, SCALE, st)
        torch.cuda.synchronize()
        assert int(st.item()) == 0
        _check(od.cpu()[rows], ref)
