"""Pins for the oracle's e4m3 code book, encoder and block quantiser (CPU only)."""
import numpy as np
import pytest
import torch

from oracle import e4m3


def test_code_book_format_facts():
    v = e4m3.code_values()
    assert v[0x00] == 0.0
    assert v[0x01] == 2.0 ** -9            # smallest subnormal
    assert v[0x07] == 7 * 2.0 ** -9        # largest subnormal
    assert v[0x08] == 2.0 ** -6            # smallest normal
    assert v[0x38] == 1.0
    assert v[0x3C] == 1.5
    assert v[0x7E] == 448.0                # largest finite
    assert np.isnan(v[0x7F]) and np.isnan(v[0xFF])
    assert v[0xB8] == -1.0
    finite = v[:0x7F]
    assert np.all(np.diff(finite) > 0)     # code order is value order


def _torch_codes(x: np.ndarray) -> np.ndarray:
    t = torch.from_numpy(np.clip(x, -448.0, 448.0).astype(np.float32))
    return t.to(torch.float8_e4m3fn).view(torch.uint8).numpy()


def test_encoder_matches_torch_cast_with_clamp():
    rng = np.random.default_rng(0)
    grid = e4m3.code_values()[:0x7F]
    mids = (grid[1:] + grid[:-1]) / 2                  # exact ties
    xs = [grid, mids, np.nextafter(mids, 0), np.nextafter(mids, 1e9),
          rng.standard_normal(20000) * 30, rng.standard_normal(20000) * 1e-2,
          rng.uniform(-600, 600, 5000), np.array([0.0, 447.9, 448.0, 464.0, 470.0, 1e30])]
    x = np.concatenate(xs).astype(np.float32)
    x = np.concatenate([x, -x])
    np.testing.assert_array_equal(e4m3.encode(x), _torch_codes(x))


def test_roundtrip_and_saturation():
    grid = e4m3.code_values()[:0x7F]
    np.testing.assert_array_equal(e4m3.decode(e4m3.encode(grid)), grid)
    assert e4m3.encode(np.array([1000.0]))[0] == 0x7E
    assert e4m3.encode(np.array([-1e6]))[0] == 0xFE
    # ties go to the even code: 1 + 1/16 lies halfway between 1 (0x38) and 1.125 (0x39)
    assert e4m3.encode(np.array([1.0625]))[0] == 0x38
    assert e4m3.encode(np.array([1.1875]))[0] == 0x3A


def test_block_quantiser_properties():
    g = torch.Generator().manual_seed(1)
    x = torch.randn(2, 3, 300, 16, generator=g) * 3
    x[1, 2, 128:256] = 0.0
    codes, scales = e4m3.quantize_blocks(x)
    assert scales.shape == (2, 3, 3) and scales.dtype == np.float32
    xn = x.numpy()
    for b in range(2):
        for h in range(3):
            for blk in range(3):
                xb = xn[b, h, blk * 128:(blk + 1) * 128]
                a = np.abs(xb).max()
                cb = codes[b, h, blk * 128:(blk + 1) * 128]
                if a == 0:
                    assert scales[b, h, blk] == 1.0 and np.all(cb == 0)
                    continue
                assert scales[b, h, blk] == np.float32(a) / np.float32(448)
                # the block maximum lands on the largest finite code
                assert np.max(cb & 0x7F) == 0x7E
    deq = e4m3.dequantize_blocks(codes, scales)
    # relative error of e4m3 with round to nearest is at most 2^-4 for normal values
    big = np.abs(xn) > 1e-1
    rel = np.abs(deq[big] - xn[big]) / np.abs(xn[big])
    assert rel.max() <= 2.0 ** -4 + 1e-7


def test_block_quantiser_matches_torch_cast_on_scaled_values():
    g = torch.Generator().manual_seed(2)
    x = torch.randn(1, 2, 256, 32, generator=g)
    codes, scales = e4m3.quantize_blocks(x)
    xn = x.numpy()
    for blk in range(2):
        xb = xn[:, :, blk * 128:(blk + 1) * 128]
        a = np.abs(xb).max(axis=(2, 3)).astype(np.float32)
        mult = (np.float32(448) / a).astype(np.float32)
        y = (xb * mult[:, :, None, None]).astype(np.float32)
        np.testing.assert_array_equal(codes[:, :, blk * 128:(blk + 1) * 128], _torch_codes(y))
