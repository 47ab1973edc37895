"""The hardware conversions of the quantizer on exhaustive inputs, against the oracle.

Driven through nvfp4_quantize (1x16 rows) with crafted rows, so that each conversion
sees its input unchanged.  A first row holds 2688 (= 6 * 448), so the tensor scale
is g = 1 and the encode factor is 1.
- E2M1 codes (RNE and SR): every finite bf16 value in [-6, 6] sits in a block whose
  maximum is 6.  The block scale is then E4M3(6 / 6) = 1, the element multiplier is
  exactly 1, and each code is the conversion of the bf16 value itself.  Under SR each
  value meets its Philox draw, and the codes must equal the oracle's for the same
  draws.
- E4M3 block scales: every positive bf16 block maximum up to 2688 (the subnormal
  range included) heads a block of zeros.  Its scale byte is RNE_sat(amax_b / 6) with
  the same division, so all those maxima, the E4M3 ties and saturation among them,
  are compared with the oracle's scale bytes.
The oracle computes every expected value (its scalar encoders through its own
quantize); codes and swizzled scale bytes must match bit for bit."""
import numpy as np
import pytest

from gpu_util import gpu_quantize

pytestmark = pytest.mark.gpu

TOP = 0x4528  # bf16 2688.0


def bf16_in_unit_range():
    """Every finite bf16 bit pattern with |v| <= 6, both signs (zeros included)."""
    b = np.arange(1 << 16, dtype=np.uint32)
    mag = b & 0x7FFF
    v = (mag << 16).view(np.float32)
    keep = (mag < 0x7F80) & (v <= np.float32(6.0))
    return b[keep].astype(np.uint16)


def blocks_with_max_six(vals):
    """Rows of 16: element 0 is 6.0, elements 1..15 take the values in turn."""
    n = (len(vals) + 14) // 15
    body = np.zeros(n * 15, np.uint16)
    body[:len(vals)] = vals
    x = np.zeros((n, 16), np.uint16)
    x[:, 0] = 0x40C0  # 6.0
    x[:, 1:] = body.reshape(n, 15)
    return x


def with_top_row(x):
    top = np.zeros((1, 16), np.uint16)
    top[0, 0] = TOP
    x = np.concatenate([top, x])
    pad = (-x.shape[0]) % 16  # whole 16-row groups keep the shapes simple
    return np.concatenate([x, np.zeros((pad, 16), np.uint16)])


def compare(ora, x, rounding, seed, what):
    got_p, got_sf, got_g, st = gpu_quantize(x, 0, rounding, seed=seed)
    assert st == 0, what
    p, sf, g, _ = ora.quantize(x, 0, False, None, 0, rounding, seed)
    assert np.float32(got_g).view(np.uint32) == np.float32(g).view(np.uint32) == 0x3F800000, what
    bad = np.nonzero(got_p != p)
    assert bad[0].size == 0, f"{what}: {bad[0].size} code bytes differ, first row {bad[0][0]}"
    ref_sf = ora.sf_swizzle(sf, x.shape[1])
    badsf = np.nonzero(got_sf != ref_sf)[0]
    assert badsf.size == 0, f"{what}: {badsf.size} scale bytes differ"
    return got_p


@pytest.mark.parametrize("rounding", [0, 1])
def test_e2m1_every_bf16_in_range(ora, rounding):
    vals = bf16_in_unit_range()
    assert len(vals) > 30000
    x = with_top_row(blocks_with_max_six(vals))
    codes = compare(ora, x, rounding, 2024, f"E2M1 rounding={rounding}")
    if rounding == 0:
        # the block maxima (6.0) encode as code 7 in every block row
        assert (codes[1:1 + (len(vals) + 14) // 15, 0] & 0xF == 7).all()


@pytest.mark.parametrize("seed", [1, 77])
def test_sr_every_bf16_in_range_two_seeds(ora, seed):
    """Two more seeds: every value meets other draws."""
    x = with_top_row(blocks_with_max_six(bf16_in_unit_range()))
    compare(ora, x, 1, seed, f"SR seed={seed}")


def test_e4m3_block_scale_every_bf16_maximum(ora):
    b = np.arange(1, 1 << 15, dtype=np.uint32)  # positive patterns, zero excluded
    v = (b << 16).view(np.float32)
    maxima = b[(b < 0x7F80) & (v <= np.float32(2688.0))].astype(np.uint16)
    assert len(maxima) > 17000
    x = np.zeros((len(maxima), 16), np.uint16)
    x[:, 0] = maxima
    x[:, 5] = maxima ^ 0x8000  # the negative of the maximum too
    compare(ora, with_top_row(x), 0, 0, "E4M3 block scales")
