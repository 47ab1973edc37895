"""Pins of the oracle's MXFP4 (the comparison format of "Nemotron NVFP4" explainer,
"What NVFP4 actually is": E2M1 elements, one power-of-two E8M0 scale per 32
elements, 4.25 bits per element) and reading R15 (smallest power-of-two scale that
clips nothing)."""
import math

import numpy as np
import pytest

from nvfp4_bit_quantized_amax_b200 import synthetic as syn


def test_e8m0_codes(ora):
    for e in range(255):
        assert ora.e8m0_decode(e) == 2.0 ** (e - 127)
    assert math.isnan(ora.e8m0_decode(255))


@pytest.mark.parametrize("amax,code", [(6.0, 127), (3.0, 126), (6.0000005, 128), (1.5, 125),
                                       (0.0, 0), (12.0, 128), (4.0, 127), (3.0000002, 127)])
def test_mx_scale_closed_forms(ora, amax, code):
    assert ora.mx_scale_code(amax) == code


def test_mx_scale_is_smallest_unclipped_power(ora):
    rng = np.random.default_rng(3)
    for a in np.concatenate([rng.lognormal(0, 8, 2000), 6.0 * 2.0 ** rng.integers(-60, 60, 200)]):
        e = ora.mx_scale_code(a)
        assert 6.0 * 2.0 ** (e - 127) >= a
        assert e == 0 or 6.0 * 2.0 ** (e - 128) < a


def test_mx_storage_is_4_25_bits(ora):
    x = syn.normal_bf16((64, 256), 1)
    packed, sf = ora.mx_quantize(x)
    assert (packed.nbytes + sf.nbytes) * 8 / x.size == 4.25


def test_mx_quantize_invariants(ora):
    x = syn.normal_bf16((96, 320), 2, outlier_prob=0.02)
    packed, sf = ora.mx_quantize(x)
    xf = syn.bf16_bits_to_f32(x).astype(np.float64)
    codes = np.stack([packed & 15, packed >> 4], axis=-1).reshape(x.shape)
    mag = np.array([ora.e2m1_decode(c & 7) for c in range(16)])[codes]
    sign = np.where(codes & 8, -1.0, 1.0)
    scale = np.repeat(np.array([[ora.e8m0_decode(e) for e in row] for row in sf]), 32, axis=1)
    deq = sign * mag * scale
    # nothing clipped: the grid step at the top is 2, so RNE errs by at most one scale
    assert (np.abs(deq - xf) <= scale + 0.0).all()
    # the scale is minimal: each block's largest element lands on 3, 4 or 6
    blk = np.abs(xf).reshape(96, -1, 32).max(axis=2)
    top = np.abs(deq).reshape(96, -1, 32).max(axis=2) / scale[:, ::32]
    assert np.all((blk == 0) | np.isin(top, [3.0, 4.0, 6.0]))


def test_mx_single_element_blocks(ora):
    for v, want in ((5.0, 4.0), (6.0, 6.0), (0.75, 0.75), (7.0, 8.0), (-3.5, -4.0)):
        x = np.zeros((1, 32), dtype=np.float32)
        x[0, 7] = v
        packed, sf = ora.mx_quantize(syn.f32_to_bf16_bits(x))
        code = int(packed[0, 3] >> 4)
        got = (-1.0 if code & 8 else 1.0) * ora.e2m1_decode(code & 7) * ora.e8m0_decode(sf[0, 0])
        assert got == want, (v, got)


def test_mx_gemm_integer_special_case(ora):
    """All scales 2^0: 2 * E2M1 values are integers in [-12, 12], so D equals the
    integer GEMM exactly."""
    rng = np.random.default_rng(4)
    M, N, K = 8, 6, 256
    A = rng.integers(0, 256, (M, K // 2), dtype=np.uint8)
    B = rng.integers(0, 256, (N, K // 2), dtype=np.uint8)
    sA = np.full((M, K // 32), 127, np.uint8)
    sB = np.full((N, K // 32), 127, np.uint8)
    D, _ = ora.mx_gemm(A, sA, B, sB, 1.0)
    table = np.array([round(2 * ora.e2m1_decode(c & 7)) * (-1 if c & 8 else 1) for c in range(16)])
    ia = table[np.stack([A & 15, A >> 4], -1).reshape(M, K)]
    ib = table[np.stack([B & 15, B >> 4], -1).reshape(N, K)]
    assert np.array_equal(D * 4, (ia @ ib.T).astype(np.float64))
