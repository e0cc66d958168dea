"""Pins of the oracle's INT8 cache quantisation (the reading of the pages'
"INT8 KV-cache quantization"): hand-worked rows, error bounds, special cases."""
import numpy as np
import torch

from oracle import cache as ocache


def test_hand_worked_row():
    # max |x| = 2 -> scale = 2/127; 1 / (2/127) = 63.5 rounds half-even to 64,
    # 0.5 / (2/127) = 31.75 -> 32, -2 -> -127, 0 -> 0
    x = np.zeros(128, np.float32)
    x[:4] = [1.0, -2.0, 0.5, 0.0]
    q, s = ocache.quantize_rows(x[None])
    assert s[0] == np.float32(2.0) / np.float32(127.0)
    assert q[0, :4].tolist() == [64, -127, 32, 0]
    assert not q[0, 4:].any()


def test_half_even_ties_and_extremes():
    x = np.zeros((3, 128), np.float32)
    x[0, 0], x[0, 1] = 127.0, 2.5          # scale 1: 2.5 -> 2 (even), 127 -> 127
    x[0, 2] = 3.5                          # -> 4 (even)
    x[1, 5] = -0.25                        # lone value -> -127
    q, s = ocache.quantize_rows(x)
    assert s[0] == 1.0 and q[0, :3].tolist() == [127, 2, 4]
    assert q[1, 5] == -127 and s[1] == np.float32(0.25) / np.float32(127.0)
    assert s[2] == 0.0 and not q[2].any()   # a zero row stays zero


def test_round_bf16_matches_torch_and_ties():
    rng = np.random.default_rng(2)
    x = (rng.standard_normal(200_000) * np.exp(rng.uniform(-30, 30, 200_000))).astype(np.float32)
    # exact ties: the dropped 16 bits are 0x8000, kept part odd and even
    ties = np.array([0x3F808000, 0x3F818000, 0xBF808000, 0x40490000 | 0x8000], np.uint32).view(np.float32)
    x = np.concatenate([x, ties, np.float32([0.0, -0.0, 1.0, 65504.0, 1e-38])])
    ref = torch.from_numpy(x).bfloat16().float().numpy()
    assert np.array_equal(ocache.round_bf16(x).view(np.uint32), ref.view(np.uint32))
    assert ocache.round_bf16(ties).view(np.uint32).tolist() == [0x3F800000, 0x3F820000, 0xBF800000,
                                                                0x404A0000]


def test_dequantized_values_by_hand():
    # scale = fl32(2/127); 127 * scale rounds to 2.0 in bf16; 64 * scale =
    # 1.00787... lies 6.1e-5 above the bf16 neighbour 1 + 2^-7 (spacing 2^-7)
    x = np.zeros(128, np.float32)
    x[:3] = [2.0, 1.0, -0.5]
    q, s = ocache.quantize_rows(x[None])
    d = ocache.dequantize_rows(q, s)[0]
    assert q[0, :3].tolist() == [127, 64, -32]
    assert d[0] == 2.0 and d[1] == 1.0078125 and d[2] == -0.50390625
    assert not d[3:].any()


def test_error_bound_and_range():
    rng = np.random.default_rng(0)
    x = rng.standard_normal((64, 7, 128)).astype(np.float32) * rng.uniform(0.01, 30, (64, 7, 1))
    q, s = ocache.quantize_rows(x)
    assert q.dtype == np.int8 and np.abs(q.astype(int)).max() == 127
    # half a step of the code, plus the bf16 rounding of the result
    err = np.abs(ocache.dequantize_rows(q, s) - x)
    assert np.all(err <= s[..., None] * (0.5 + 1e-6) + np.abs(x) * 2.0 ** -8 + 1e-12)
    # the row maximum is represented exactly up to the scale's rounding
    amax = np.abs(x).max(-1)
    assert np.allclose(np.abs(q.astype(np.float64)).max(-1) * s, amax, rtol=1e-6)


def test_append_places_head_major_rows():
    rng = np.random.default_rng(1)
    k = rng.standard_normal((5, 3, 128)).astype(np.float32)
    cq = np.zeros((3, 10, 128), np.int8)
    cs = np.zeros((3, 10), np.float32)
    cq, cs = ocache.append_int8(cq, cs, 2, k)
    for i in range(5):
        for h in range(3):
            q, s = ocache.quantize_rows(k[i, h][None])
            assert np.array_equal(cq[h, 2 + i], q[0]) and cs[h, 2 + i] == s[0]
    assert not cq[:, :2].any() and not cq[:, 7:].any()
