"""Pins of the FP8 (e4m3) quantisation oracle (CPU, no GPU).

The oracle writes e4m3 rounding out from the format's definition; it is
checked against PyTorch's float8_e4m3fn conversion (a library routine), against
the representable values themselves, hand-worked blocks, and the error bound
of a 3-bit mantissa.
"""
import numpy as np
import pytest
import torch

from oracle.sparse_attn_fp8 import E4M3_MAX, dequantize_blocks, e4m3_round, quantize_blocks


def _torch_e4m3(x):
    return torch.from_numpy(np.asarray(x, dtype=np.float32)).to(torch.float8_e4m3fn).float().numpy()


def test_every_e4m3_value_rounds_to_itself():
    allv = torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).float().numpy()
    fin = allv[np.isfinite(allv)]
    assert fin.size == 254 and fin.max() == E4M3_MAX
    assert np.array_equal(e4m3_round(fin), fin.astype(np.float64))


def test_rounding_matches_torch_in_range():
    g = np.random.default_rng(1)
    x = np.concatenate([g.standard_normal(300_000) * 40.0, g.standard_normal(100_000) * 0.01,
                        g.uniform(-448, 448, 100_000)]).astype(np.float32)
    # midpoints between neighbours: ties go to the even code
    allv = np.unique(np.abs(torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).float().numpy()))
    allv = allv[np.isfinite(allv)]
    mids = ((allv[:-1] + allv[1:]) / 2).astype(np.float32)
    x = np.concatenate([x, mids, -mids])
    x = x[np.abs(x) <= E4M3_MAX]
    assert np.array_equal(e4m3_round(x), _torch_e4m3(x).astype(np.float64))


def test_saturation_past_the_largest_value():
    # The reading saturates (satfinite); torch's conversion gives NaN there instead.
    for v in (448.0, 460.0, 464.0, 470.0, 1e6):
        assert e4m3_round(np.float32(v)) == 448.0
        assert e4m3_round(np.float32(-v)) == -448.0


def test_relative_error_bound_of_normal_codes():
    x = np.random.default_rng(2).uniform(2.0 ** -6, 448.0, 200_000)
    err = np.abs(e4m3_round(x) - x) / x
    assert err.max() <= 2.0 ** -4 + 1e-12


def test_hand_worked_block():
    # One block of 2 tokens x 2 channels: amax = 3, scale = 3/448; the largest
    # entry maps to 448 exactly, 1.5 to 224, -0.75 to -112, 0.01 to 1.4933 ->
    # 1.5 (step 2^-3 in [1, 2)).
    X = np.array([[[3.0, 1.5], [-0.75, 0.01]]], dtype=np.float32)
    codes, scales = quantize_blocks(X, 2)
    assert scales.shape == (1, 1) and scales[0, 0] == np.float32(3.0) / np.float32(448.0)
    assert codes[0].tolist() == [[448.0, 224.0], [-112.0, 1.5]]
    back = dequantize_blocks(codes, scales, 2)
    assert np.allclose(back[0, 0], [3.0, 1.5], rtol=1e-7)


def test_ragged_and_zero_blocks():
    X = np.zeros((1, 5, 4), dtype=np.float32)
    X[0, 4] = [1.0, -2.0, 0.5, 0.25]         # block 2 (tokens 4..) is ragged; blocks 0-1 are zero
    codes, scales = quantize_blocks(X, 2)
    assert scales.tolist() == [[0.0, 0.0, np.float32(2.0) / np.float32(448.0)]]
    assert np.all(codes[0, :4] == 0)
    assert codes[0, 4].tolist() == [224.0, -448.0, 112.0, 56.0]


@pytest.mark.parametrize("block", [64, 128])
def test_dequantised_blocks_are_within_the_format_error(block):
    g = torch.Generator().manual_seed(3)
    X = torch.randn(2, 3, 1000, 128, generator=g).to(torch.bfloat16).float().numpy()
    codes, scales = quantize_blocks(X, block)
    back = dequantize_blocks(codes, scales, block)
    # per block: |x - back| <= max(2^-4 |x|, half the subnormal step times the scale)
    for j in range(scales.shape[-1]):
        lo, hi = j * block, min(1000, (j + 1) * block)
        s = scales[..., j, None, None].astype(np.float64)
        bound = np.maximum(2.0 ** -4 * np.abs(X[..., lo:hi, :]), 2.0 ** -10 * s)
        assert np.all(np.abs(X[..., lo:hi, :] - back[..., lo:hi, :]) <= bound + 1e-12)
    assert np.all(np.abs(codes) <= 448.0)
