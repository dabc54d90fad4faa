"""Pins of the oracle's e4m3 quantisation (FP8 attention variant), without a GPU.

The e4m3 format is the OCP 8-bit floating point specification's E4M3 ("fn": no infinities,
S.1111.111 is NaN, largest finite 1.75 * 2^8 = 448, smallest subnormal 2^-9). The oracle's
encoding is checked against values worked by hand from that definition, against PyTorch's
float8_e4m3fn conversion (a library routine, round to nearest even) everywhere in range,
including every tie, and for exact round trips of all finite codes; the saturation of the
variant (values beyond 448) against the definition only, since PyTorch maps them to NaN.
"""
import numpy as np
import pytest
import torch

from oracle import veda_oracle as O


def _torch_codes(x: np.ndarray) -> np.ndarray:
    return torch.from_numpy(x.astype(np.float32)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()


def test_e4m3_hand_worked_codes():
    cases = [
        (1.0, 0x38),            # exponent field 7 (2^0), mantissa 0
        (448.0, 0x7E),          # largest finite: 1.75 * 2^8
        (-448.0, 0xFE),
        (500.0, 0x7E),          # saturates (R23)
        (464.0, 0x7E),          # halfway to the non-existent 480: saturates
        (2.0 ** -6, 0x08),      # smallest normal
        (2.0 ** -9, 0x01),      # smallest subnormal
        (2.0 ** -10, 0x00),     # tie between 0 and 2^-9: even (0)
        (3 * 2.0 ** -10, 0x02),  # tie between 1 and 2 subnormal steps: even (2)
        (0.0, 0x00),
        (-0.0, 0x80),
        (1.0625, 0x38),         # tie between 1.0 (m 0) and 1.125 (m 1): even
        (1.1875, 0x3A),         # tie between 1.125 (m 1) and 1.25 (m 2): even
        (0.1, 0x1D),            # 0.1 = 1.6 * 2^-4 -> 1.625 * 2^-4 (exponent field 3, m 5)
        (-3.0, 0xC4),           # 1.5 * 2^1
    ]
    got = O.e4m3_codes(np.array([v for v, _ in cases]))
    assert [int(c) for c in got] == [c for _, c in cases]


def test_e4m3_all_finite_codes_round_trip():
    codes = np.array([c for c in range(256) if (c & 0x7F) != 0x7F], dtype=np.uint8)
    vals = O.e4m3_value(codes)
    assert np.array_equal(O.e4m3_codes(vals), codes)
    pos = np.sort(vals[vals > 0])
    assert pos[0] == 2.0 ** -9 and pos[-1] == 448.0 and len(pos) == 126
    with pytest.raises(ValueError):
        O.e4m3_value(np.array([0x7F], dtype=np.uint8))


def test_e4m3_matches_torch_in_range_and_on_every_tie():
    rng = np.random.default_rng(2301)
    mag = np.exp2(rng.uniform(-13, np.log2(448.0), 100000))
    x = (mag * rng.choice([-1.0, 1.0], mag.size)).astype(np.float32).astype(np.float64)
    assert np.array_equal(O.e4m3_codes(x), _torch_codes(x))
    # every midpoint between neighbouring finite values, and just beside it
    vals = np.sort(np.unique(np.abs(O.e4m3_value(np.arange(0, 0x7F, dtype=np.uint8)))))
    mids = (vals[:-1] + vals[1:]) / 2
    for y in (mids, np.nextafter(mids.astype(np.float32), np.float32(0)).astype(np.float64),
              np.nextafter(mids.astype(np.float32), np.float32(1e9)).astype(np.float64)):
        for sgn in (1.0, -1.0):
            assert np.array_equal(O.e4m3_codes(sgn * y), _torch_codes(sgn * y))


def test_quantize_fp8_scale_max_code_transpose_and_error():
    rng = np.random.default_rng(2302)
    x = rng.standard_normal((2, 3, 256, 128))
    x[1, 2] *= 40.0
    x[0, 1] = 0.0                                   # an all-zero tensor: scale 1, codes 0
    x = torch.from_numpy(x).to(torch.bfloat16).double().numpy()
    codes, scale = O.quantize_fp8(x)
    assert codes.dtype == np.uint8 and scale.dtype == np.float32
    assert scale[0, 1] == 1.0 and not codes[0, 1].any()
    for b in range(2):
        for h in range(3):
            if b == 0 and h == 1:
                continue
            amax = np.float32(np.abs(x[b, h]).max())
            assert scale[b, h] == amax / np.float32(448.0)
            i = np.unravel_index(np.argmax(np.abs(x[b, h])), x[b, h].shape)
            assert codes[b, h][i] & 0x7F == 0x7E          # the largest magnitude maps to 448
    deq = O.dequantize_fp8(codes, scale)
    y = np.abs(x) / scale.astype(np.float64)[:, :, None, None]
    normal = y >= 2.0 ** -6
    err = np.abs(deq - x)
    # relative 2^-4 (half a 3-bit mantissa step) for normals, 2^-10 of the scale for subnormals
    assert np.all(err[normal] <= 2.0 ** -4 * np.abs(x[normal]) * (1 + 1e-6))
    assert np.all(err[~normal] <= 2.0 ** -10 * np.broadcast_to(scale[:, :, None, None], x.shape)[~normal] * (1 + 1e-6))
    t_codes, t_scale = O.quantize_fp8(x, transpose_tiles=True)
    assert np.array_equal(t_scale, scale)
    assert np.array_equal(t_codes.reshape(2, 3, 2, 128, 128), codes.reshape(2, 3, 2, 128, 128).swapaxes(3, 4))
    assert np.array_equal(O.dequantize_fp8(t_codes, t_scale, transposed_tiles=True), deq)
