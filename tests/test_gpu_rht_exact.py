"""The 16-point RHT at the edges of its fp32 fast path, against the oracle.

Both sides must produce the fp32 rounding of the exact sum: the oracle through an
fp64 16 x 16 product, the kernels through an fp32 butterfly when a chunk's nonzero
inputs span at most 13 binades (their partial sums are then exact) and an fp64
butterfly otherwise.  Crafted 16-element chunks straddle that boundary (spans 12,
13, 14, 15 and up to 41 binades), mix zeros, subnormals and values near the top of
the range, and random chunks with random spans exercise both paths side by side in
one warp.  Checked bit for bit: the standalone transform along both axes, and the
RHT column orientation of the quantizer (codes, scales, tensor scale, RNE and SR)."""
import numpy as np
import pytest
import torch

from gpu_util import DEV, f32_bits, to_dev_bf16
from nvfp4_bit_quantized_amax_b200 import capi
from nvfp4_bit_quantized_amax_b200 import synthetic as syn

pytestmark = pytest.mark.gpu


def bf16(sign, exp_field, mant):
    return np.uint16((int(sign) << 15) | (int(exp_field) << 7) | int(mant))


def crafted_chunks(rng):
    """A list of 16-value chunks (uint16 bf16 bits)."""
    chunks = []
    chunks.append(np.zeros(16, np.uint16))                                 # all zero
    one = np.zeros(16, np.uint16)
    one[5] = bf16(1, 130, 77)
    chunks.append(one)                                                    # one nonzero
    for span in (0, 1, 7, 12, 13, 14, 15, 20, 30, 41):                    # around the boundary
        for _ in range(6):
            top = int(rng.integers(100, 140))
            e = rng.integers(top - span, top + 1, 16)
            e[0], e[1] = top, top - span
            c = np.array([bf16(rng.integers(0, 2), ee, rng.integers(0, 128)) for ee in e], np.uint16)
            c[rng.integers(2, 16)] = 0                                     # a zero does not count
            chunks.append(rng.permutation(c))
    for _ in range(4):                                                    # subnormals
        c = np.array([bf16(rng.integers(0, 2), 0, rng.integers(1, 128)) for _ in range(16)], np.uint16)
        chunks.append(c)
        d = c.copy()
        d[:4] = [bf16(0, 1, 3), bf16(1, 13, 0), bf16(0, 14, 5), bf16(1, 12, 127)]
        chunks.append(d)                                                  # spans 12 .. 14 above them
    for top in (250, 251, 252):                                           # near the top of the range
        e = rng.integers(top - 3, top + 1, 16)
        chunks.append(np.array([bf16(rng.integers(0, 2), ee, rng.integers(0, 128)) for ee in e], np.uint16))
    # ties: equal magnitudes with alternating signs cancel exactly in most outputs
    chunks.append(np.array([bf16(i & 1, 127, 64) for i in range(16)], np.uint16))
    return chunks


def column_matrix(chunks, ncols, rng):
    """rows = 16 * len(chunks) / ncols ... : chunk k lands in column k % ncols, rows
    16 * (k // ncols) .. + 15; random N(0,1) chunks fill the rest."""
    nrow_chunks = (len(chunks) + ncols - 1) // ncols
    x = syn.normal_bf16((16 * nrow_chunks, ncols), 5)
    for k, c in enumerate(chunks):
        x[16 * (k // ncols): 16 * (k // ncols) + 16, k % ncols] = c
    return x


@pytest.mark.parametrize("seed", [0, 1])
def test_standalone_rht_edges_both_axes(ora, seed):
    rng = np.random.default_rng(seed)
    chunks = crafted_chunks(rng)
    signs = syn.rht_signs(seed + 3)
    x0 = column_matrix(chunks, 64, rng)                 # chunks down the columns (axis 0)
    x1 = np.ascontiguousarray(x0.T)                     # the same chunks along the rows (axis 1)
    for x, axis in ((x0, 0), (x1, 1)):
        y = torch.empty(x.shape, dtype=torch.float32, device=DEV)
        capi.nvfp4_rht(to_dev_bf16(x), signs, 16, y, axis=axis)
        got = y.cpu().numpy()
        ref = ora.rht(x, axis, signs)
        bad = np.nonzero(got.view(np.uint32) != ref.view(np.uint32))
        assert bad[0].size == 0, (axis, bad[0][:5], bad[1][:5])


def test_random_spans_mixed_paths(ora):
    """Every chunk draws its own exponent span in 0..24: about half take the fp32
    path and half the fp64 path, interleaved across the lanes of each warp."""
    rng = np.random.default_rng(9)
    rows, cols = 256, 128
    x = np.zeros((rows, cols), np.uint16)
    for j in range(rows // 16):
        for c in range(cols):
            span = int(rng.integers(0, 25))
            top = int(rng.integers(110, 140))
            e = rng.integers(top - span, top + 1, 16)
            x[16 * j: 16 * j + 16, c] = [bf16(rng.integers(0, 2), ee, rng.integers(0, 128)) for ee in e]
    signs = syn.rht_signs(4)
    y = torch.empty((rows, cols), dtype=torch.float32, device=DEV)
    capi.nvfp4_rht(to_dev_bf16(x), signs, 16, y, axis=0)
    assert np.array_equal(y.cpu().numpy().view(np.uint32), ora.rht(x, 0, signs).view(np.uint32))


@pytest.mark.parametrize("rounding", [0, 1])
def test_quantizer_rht_columns_at_the_edges(ora, rounding):
    """The fused RHT column orientation (amax pass + tile pass) on the crafted chunks:
    codes, scale bytes and the tensor scale bit for bit.  The top-of-range chunks are
    left out (their transform overflows to Inf, which the quantizer reports as an
    error instead of quantizing)."""
    rng = np.random.default_rng(2)
    chunks = [c for c in crafted_chunks(rng) if ((c >> 7) & 0xFF).max() < 200]
    x = column_matrix(chunks, 32, rng)
    rows, cols = x.shape
    signs = syn.rht_signs(6)
    seed = 77
    xd = to_dev_bf16(x)
    c = (torch.empty(rows * cols // 2, dtype=torch.uint8, device=DEV),
         torch.empty(capi.scale_bytes(cols, rows), dtype=torch.uint8, device=DEV),
         torch.empty(1, dtype=torch.float32, device=DEV))
    ws = torch.empty(capi.quantize_workspace_bytes(), dtype=torch.uint8, device=DEV)
    capi.nvfp4_quantize_2d(xd, 0, 0, rounding, seed, True, signs, None, c, ws)
    torch.cuda.synchronize()
    assert capi.nvfp4_read_status(ws) == 0
    p, sf, g, _ = ora.quantize(x, 1, True, signs, 0, rounding, seed)
    assert np.array_equal(c[0].cpu().numpy().reshape(cols, rows // 2), p)
    assert np.array_equal(c[1].cpu().numpy(), ora.sf_swizzle(sf, rows))
    assert f32_bits(c[2].item()) == f32_bits(g)
