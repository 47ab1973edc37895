"""The tensor amax of the rotated column orientation, bit for bit against the oracle.

The amax pass skips the rotation of a column whose rounded-up sum of |x| cannot
exceed the largest rotated magnitude already found for the same output word (every
entry of H16 is +-1, so no rotated value exceeds that sum).  The threshold only
comes into play once a warp has handled a unit, so these tensors are large enough
that every warp walks several units.  The cases target the bound: chunks whose
bound equals their rotated maximum, the maximum placed in the last units of the
tensor, subnormal-only inputs, both halves of a packed column pair, and (grouped)
experts of very different scales, where a threshold carried across a group
boundary would lose the small expert's maximum.  The amax words of the quantize
workspace (word 0: max |x|, word 1: max |RHT16 down the rows|) are read directly."""
import numpy as np
import pytest
import torch

from gpu_util import DEV, to_dev_bf16
from nvfp4_bit_quantized_amax_b200 import capi
from nvfp4_bit_quantized_amax_b200 import synthetic as syn

pytestmark = pytest.mark.gpu

SHAPE = (8192, 4096)   # 16384 units of 16 x 128: several per warp on a B200


def gpu_amax_words(x_bits, signs):
    """(max |x|, max |rotated column value|) as the quantizer's amax pass leaves them."""
    rows, cols = x_bits.shape
    c = (torch.empty(rows * cols // 2, dtype=torch.uint8, device=DEV),
         torch.empty(capi.scale_bytes(cols, rows), dtype=torch.uint8, device=DEV),
         torch.empty(1, dtype=torch.float32, device=DEV))
    ws = torch.empty(capi.quantize_workspace_bytes(), dtype=torch.uint8, device=DEV)
    capi.nvfp4_quantize_2d(to_dev_bf16(x_bits), 0, 0, 0, 5, True, signs, None, c, ws)
    torch.cuda.synchronize()
    w = ws[:8].cpu().numpy().view(np.uint32)
    return int(w[0]), int(w[1]), capi.nvfp4_read_status(ws)


def oracle_words(ora, x_bits, signs):
    a_row = ora.tensor_amax(x_bits, 0, False, signs)
    a_col = ora.tensor_amax(x_bits, 1, True, signs)
    return int(np.float32(a_row).view(np.uint32)), int(np.float32(a_col).view(np.uint32))


def bf16_bits(v):
    return syn.f32_to_bf16_bits(np.asarray(v, dtype=np.float32))


def tight_values(c, signs, j=0):
    """16 values c * s_i * H16[i][j] (float32): the rotation gathers them all into
    output j, so the chunk's largest rotated magnitude is 16|c|, its sum of |x|
    exactly."""
    h = np.array([1 - 2 * (bin(i & j).count("1") & 1) for i in range(16)], np.float32)
    return np.float32(c) * signs.astype(np.float32) * h


def tight_chunk(c, signs, j=0):
    return bf16_bits(tight_values(c, signs, j))


def plant(x, r0, col, chunk):
    x[r0:r0 + 16, col] = chunk


def check(ora, x, signs, *, status_ok=True, repeats=3):
    """Which columns a warp rotates depends on when the other warps publish, so the
    pass runs several times; every run must give the oracle's words."""
    ref_row, ref_col = oracle_words(ora, x, signs)
    for _ in range(repeats):
        got_row, got_col, st = gpu_amax_words(x, signs)
        if status_ok:
            assert st == 0
        assert got_row == ref_row, (hex(got_row), hex(ref_row))
        assert got_col == ref_col, (hex(got_col), hex(ref_col))


@pytest.mark.parametrize("kind", ["normal", "t3", "outlier"])
def test_amax_random(ora, kind):
    if kind == "normal":
        x = syn.normal_bf16(SHAPE, 21)
    elif kind == "t3":
        x = syn.student_t_bf16(SHAPE, 22)
    else:
        x = syn.normal_bf16(SHAPE, 23, outlier_prob=0.001)
    check(ora, x, syn.rht_signs(1))


@pytest.mark.parametrize("half", [0, 1])
def test_amax_tight_chunk_last_unit(ora, half):
    """The maximum sits in the last 16 rows of the last column pair (the last unit
    of the last warp), in a chunk whose bound equals its rotated maximum; a second
    tight chunk early in the tensor reaches one bf16 step less."""
    signs = syn.rht_signs(2)
    x = syn.normal_bf16(SHAPE, 24)
    rows, cols = SHAPE
    plant(x, 0, 6, tight_chunk(8.0, signs, 3))               # 128 after rotation
    plant(x, rows - 16, cols - 2 + half, tight_chunk(8.0625, signs, 5))  # 129
    check(ora, x, signs)


def test_amax_ties_at_the_threshold(ora):
    """Many chunks reach exactly the same rotated maximum as the first one found; one
    late chunk reaches it plus one bf16 step of an input."""
    signs = syn.rht_signs(3)
    x = syn.normal_bf16(SHAPE, 25, std=0.01)
    rows, cols = SHAPE
    rng = np.random.default_rng(5)
    for k in range(400):
        r0 = 16 * int(rng.integers(0, rows // 16))
        plant(x, r0, int(rng.integers(0, cols)), tight_chunk(2.0, signs, int(rng.integers(0, 16))))
    top = tight_values(2.0, signs, 7)
    top[9] *= np.float32(1.0078125)   # one bf16 step above 2: the chunk reaches 32 + 2^-6
    plant(x, rows - 32, cols - 1, bf16_bits(top))
    check(ora, x, signs)


def test_amax_single_values(ora):
    """A zero tensor with single nonzero values (bound = rotated maximum = |x|), in
    the low and high halves of the column pairs, growing towards the end."""
    signs = syn.rht_signs(4)
    x = np.zeros(SHAPE, np.uint16)
    rows, cols = SHAPE
    rng = np.random.default_rng(6)
    pos_r = np.sort(rng.integers(0, rows, 3000))
    pos_c = rng.integers(0, cols, 3000)
    vals = np.linspace(1.0, 3.0, 3000, dtype=np.float32)
    x[pos_r, pos_c] = bf16_bits(vals * np.where(rng.random(3000) < 0.5, -1, 1).astype(np.float32))
    check(ora, x, signs)


def test_amax_subnormal_inputs(ora):
    """bf16 subnormals only: the bound's sums keep subnormals (no flush to zero)."""
    signs = syn.rht_signs(5)
    rng = np.random.default_rng(7)
    mant = rng.integers(0, 128, SHAPE).astype(np.uint16)
    sign = (rng.integers(0, 2, SHAPE).astype(np.uint16) << 15)
    x = (sign | mant).astype(np.uint16)
    check(ora, x, signs, status_ok=False)   # the quantizer may report the tiny scale


@pytest.mark.parametrize("bits", [0x7F80, 0xFF80, 0x7FC1])
def test_amax_late_nonfinite(bits):
    """An Inf or NaN in the last unit of a large tensor, after every warp's threshold
    is set: the row word holds its pattern, the quantizer reports it, and an Inf's
    column (whose bound is Inf) is rotated, so the column word is Inf as well."""
    signs = syn.rht_signs(7)
    x = syn.normal_bf16(SHAPE, 26)
    x[SHAPE[0] - 3, SHAPE[1] - 5] = bits
    got_row, got_col, st = gpu_amax_words(x, signs)
    assert st == capi.ERR_NONFINITE
    if bits & 0x7F:  # NaN: its magnitude pattern sorts above Inf in the row word
        assert got_row == (bits & 0x7FFF) << 16
    else:
        assert got_row == 0x7F800000 and got_col == 0x7F800000


@pytest.mark.parametrize("gather", [False, True])
def test_grouped_amax_alternating_scales(ora, gather):
    """170 experts of 128 rows, hidden 1024: 10880 units, several per warp, so many
    warps cross an expert boundary.  Odd experts are zero except a few values in their
    first unit, 10^6 times smaller than the even experts' values: their tensor
    scales (the rotated column orientation of X) come out right only if each expert's
    threshold starts afresh."""
    E, K, N = 170, 1024, 128
    g = np.full(E, 128, dtype=np.int64)
    R = int(g.sum())
    x = syn.normal_bf16((R, K), 31)
    rng = np.random.default_rng(8)
    for e in range(1, E, 2):
        blk = np.zeros((128, K), np.float32)
        blk[:16, :128] = rng.standard_normal((16, 128)).astype(np.float32) * 1e-6 * (1 + e)
        x[128 * e:128 * (e + 1)] = bf16_bits(blk)
    W = to_dev_bf16(syn.normal_bf16((E * N, K), 32, std=0.02)).view(E, N, K)
    Y = torch.empty((R, N), dtype=torch.bfloat16, device=DEV)
    signs = syn.rht_signs(6)
    ws = torch.empty(capi.moe_grouped_workspace_bytes(g, K, N), dtype=torch.uint8, device=DEV)
    if gather:   # rows read through a routing table (reversed order of the source)
        src = np.ascontiguousarray(x[::-1])
        row_src = torch.arange(R - 1, -1, -1, dtype=torch.int32, device=DEV)
        capi.nvfp4_moe_grouped_fprop_gather(to_dev_bf16(src), row_src, W, Y, g, signs, ws)
    else:
        capi.nvfp4_moe_grouped_fprop(to_dev_bf16(x), W, Y, g, signs, ws)
    torch.cuda.synchronize()
    assert capi.nvfp4_read_status(ws) == 0
    v = capi.nvfp4_moe_grouped_operand(ws, g, K, N, capi.LIN_X_COL)
    base = ws.data_ptr()
    gs = ws[v.tensor_scale - base: v.tensor_scale - base + 4 * E].cpu().numpy().view(np.float32)
    for e in range(E):
        ref = ora.tensor_scale(ora.tensor_amax(x[128 * e:128 * (e + 1)], 1, True, signs))
        assert gs[e].view(np.uint32) == np.float32(ref).view(np.uint32), e
