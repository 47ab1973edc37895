"""GPU parity of the quantizer (nvfp4_quantize, nvfp4_quantize_2d) and the RHT
(nvfp4_rht) against the CPU oracle: codes, swizzled scale bytes and tensor
scales must match bit for bit; RHT outputs to the stated 1e-6 relative bound
(in fact bit for bit: both sides round the exact sum once)."""
import numpy as np
import pytest
import torch

from gpu_util import (DEV, empty_u8, f32_bits, fetch_operand, gpu_quantize, new_operand,
                      to_dev_bf16)
from nvfp4_bit_quantized_amax_b200 import capi
from nvfp4_bit_quantized_amax_b200 import synthetic as syn

pytestmark = pytest.mark.gpu


def oracle_full(ora, x, orient, rht, signs, block_mode, rounding, seed):
    packed, sf, g, amax = ora.quantize(x, orient, rht, signs, block_mode, rounding, seed)
    vcols = x.shape[0] if orient else x.shape[1]
    return packed, ora.sf_swizzle(sf, vcols), g


def assert_same(got, ref, what):
    gp, gs, gg = got[:3]
    rp, rs, rg = ref
    assert gp.shape == rp.shape, what
    bad = np.nonzero(gp != rp)
    assert bad[0].size == 0, f"{what}: {bad[0].size} code bytes differ, first at {bad[0][0]},{bad[1][0]}"
    badsf = np.nonzero(gs != rs)[0]
    assert badsf.size == 0, f"{what}: {badsf.size} scale bytes differ, first at {badsf[0]}"
    assert f32_bits(gg) == f32_bits(rg), f"{what}: tensor scale {gg} != {rg}"


def gen(kind, shape, seed):
    if kind == "normal":
        return syn.normal_bf16(shape, seed)
    if kind == "outlier":
        return syn.normal_bf16(shape, seed, outlier_prob=0.01)
    if kind == "t3":
        return syn.student_t_bf16(shape, seed)
    if kind == "laplace":
        return syn.laplace_bf16(shape, seed)
    if kind == "tiny":
        return syn.normal_bf16(shape, seed, std=1e-30)
    raise ValueError(kind)


SHAPES_1D = [(1, 16), (3, 48), (64, 128), (300, 272), (129, 1040)]
SHAPES_2D = [(16, 16), (48, 80), (304, 272), (256, 1024)]


@pytest.mark.parametrize("shape", SHAPES_1D)
@pytest.mark.parametrize("rounding", [0, 1])
@pytest.mark.parametrize("kind", ["normal", "outlier", "t3"])
def test_quantize_1x16(ora, shape, rounding, kind):
    x = gen(kind, shape, 11)
    got = gpu_quantize(x, 0, rounding, seed=1234)
    assert got[3] == 0
    assert_same(got, oracle_full(ora, x, 0, False, None, 0, rounding, 1234), f"{shape} {kind}")


@pytest.mark.parametrize("rounding", [0, 1])
def test_quantize_1x16_many_blocks_per_thread(ora, rounding):
    """The row quantizer walks its blocks grid-stride and advances each block's (row,
    block) position by counting: with 65 blocks per row (1040 columns), which no grid
    stride of 256-thread CTAs divides, and 266k blocks, every thread handles several
    blocks and the position wraps across rows.  Full comparison with the oracle."""
    x = syn.normal_bf16((4099, 1040), 31, outlier_prob=0.01)
    got = gpu_quantize(x, 0, rounding, seed=4321)
    assert got[3] == 0
    assert_same(got, oracle_full(ora, x, 0, False, None, 0, rounding, 4321), f"4099x1040 r{rounding}")


@pytest.mark.parametrize("shape", SHAPES_2D)
@pytest.mark.parametrize("rounding", [0, 1])
@pytest.mark.parametrize("kind", ["normal", "laplace", "tiny"])
def test_quantize_16x16(ora, shape, rounding, kind):
    x = gen(kind, shape, 5)
    got = gpu_quantize(x, 1, rounding, seed=77)
    assert_same(got, oracle_full(ora, x, 0, False, None, 1, rounding, 77), f"{shape} {kind}")


def crafted_codec_tensor():
    """Rows whose block scale is an exact power of two (block max 6 * 2^k, tensor max
    2688 so g = 1): the elements land exactly on E2M1 ties, near-ties, zeros of both
    signs, saturation and E4M3-subnormal scales."""
    ties = [0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 0.1, 0.0, 2.75, 4.5, 5.5, 0.5, 1.0, 6.0]
    rows = []
    rows.append([2688.0] + [0.0] * 15)
    for k in range(-3, 4):
        s = 2.0 ** k
        rows.append([6.0 * s] + [t * s for t in ties])
        rows.append([-6.0 * s] + [-t * s for t in ties])
    for s in (2.0 ** -8, 3.0 * 2.0 ** -9, 5.0 * 2.0 ** -10, 2.0 ** -14):  # E4M3-subnormal / zero scales
        rows.append([6.0 * s] + [t * s for t in ties])
    rows.append([-0.0] * 16)
    rows.append([0.0, -0.0] * 8)
    x = np.array(rows, dtype=np.float32)
    return syn.f32_to_bf16_bits(x)


@pytest.mark.parametrize("rounding", [0, 1])
def test_quantize_crafted_codec_cases(ora, rounding):
    x = crafted_codec_tensor()
    got = gpu_quantize(x, 0, rounding, seed=99)
    assert_same(got, oracle_full(ora, x, 0, False, None, 0, rounding, 99), "crafted")
    if rounding == 0:  # the ties, checked against hand-derived codes as well
        codes = got[0][1]
        assert codes[0] & 0xF == 7 and (codes[0] >> 4) == 0  # 6 -> code 7, 0.25 -> 0 (tie to even)
        assert codes[1] & 0xF == 2 and (codes[1] >> 4) == 2  # 0.75 -> 1.0, 1.25 -> 1.0


def test_quantize_zero_and_nonfinite(ora):
    x = np.zeros((32, 64), np.uint16)
    x[3, ::5] = 0x8000
    got = gpu_quantize(x, 0, 0)
    assert_same(got, oracle_full(ora, x, 0, False, None, 0, 0, 0), "zeros")
    x = syn.normal_bf16((32, 64), 1)
    x[7, 9] = 0x7F80  # +Inf
    _, _, g, status = gpu_quantize(x, 0, 0)
    assert status == capi.ERR_NONFINITE and np.isnan(g)
    x[7, 9] = 0x7FC1  # NaN
    _, _, g, status = gpu_quantize(x, 1, 0)
    assert status == capi.ERR_NONFINITE and np.isnan(g)


def gpu_quantize_2d(x_bits, block_mode, row_r, col_r, seed, col_rht, signs, want_row=True,
                    want_col=True):
    rows, cols = x_bits.shape
    x = to_dev_bf16(x_bits)
    ro = new_operand(rows, cols) if want_row else None
    co = new_operand(cols, rows) if want_col else None
    ws = empty_u8(capi.quantize_workspace_bytes())
    capi.nvfp4_quantize_2d(x, block_mode, row_r, col_r, seed, col_rht, signs, ro, co, ws)
    out_r = fetch_operand(ro, rows, cols) if want_row else None
    out_c = fetch_operand(co, cols, rows) if want_col else None
    assert capi.nvfp4_read_status(ws) == 0
    return out_r, out_c


@pytest.mark.parametrize("shape", [(16, 16), (64, 128), (160, 272), (512, 384), (1040, 96)])
@pytest.mark.parametrize("recipe", ["x", "dy", "w", "dy_col_only", "x_plain_col"])
def test_quantize_2d_orientations(ora, shape, recipe):
    rows, cols = shape
    signs = syn.rht_signs(7)
    x = syn.normal_bf16(shape, 21, outlier_prob=0.01)
    bm, rr, cr, rht, want_row = {
        "x": (0, 0, 0, True, True),
        "dy": (0, 1, 1, True, True),
        "w": (1, 0, 0, False, True),
        "dy_col_only": (0, 0, 1, True, False),
        "x_plain_col": (0, 0, 0, False, True),
    }[recipe]
    r, c = gpu_quantize_2d(x, bm, rr, cr, 4321, rht, signs, want_row=want_row)
    if want_row:
        assert_same(r, oracle_full(ora, x, 0, False, signs, bm, rr, 4321), f"{recipe} row")
    assert_same(c, oracle_full(ora, x, 1, rht, signs, bm, cr, 4321), f"{recipe} col")
    if recipe == "w":  # 16x16: the two orientations are exact transposes
        from test_oracle_quantize import unpack
        assert np.array_equal(unpack(r[0]), unpack(c[0]).T)


@pytest.mark.parametrize("shape,recipe", [((16384, 272), "dy"), ((8208, 1040), "w")])
def test_quantize_2d_many_units_ragged(ora, shape, recipe):
    """Enough work that every warp of the streamed amax pass walks several 16 x 128
    units (crossing rows, the last column unit partial: 272 columns), and many
    128 x 128 tiles of the 16x16 tile kernel with the last tile row and column partial
    (8208 rows, 1040 columns).  Full comparison with the oracle, both orientations."""
    signs = syn.rht_signs(5)
    x = syn.normal_bf16(shape, 23, outlier_prob=0.01)
    bm, rr, cr, rht = {"dy": (0, 1, 1, True), "w": (1, 0, 0, False)}[recipe]
    r, c = gpu_quantize_2d(x, bm, rr, cr, 987, rht, signs)
    assert_same(r, oracle_full(ora, x, 0, False, signs, bm, rr, 987), f"{recipe} {shape} row")
    assert_same(c, oracle_full(ora, x, 1, rht, signs, bm, cr, 987), f"{recipe} {shape} col")


@pytest.mark.parametrize("axis", [0, 1])
@pytest.mark.parametrize("shape", [(16, 16), (64, 48), (256, 1024)])
def test_rht(ora, axis, shape):
    signs = syn.rht_signs(3)
    x = syn.normal_bf16(shape, 8, outlier_prob=0.02)
    y = torch.empty(shape, dtype=torch.float32, device=DEV)
    capi.nvfp4_rht(to_dev_bf16(x), signs, 16, y, axis=axis)
    got = y.cpu().numpy()
    ref = ora.rht(x, axis, signs)
    rel = np.abs(got - ref) / np.maximum(np.abs(ref), 1e-30)
    assert rel.max() <= 1e-6
    assert np.array_equal(got.view(np.uint32), ref.view(np.uint32))


def test_deterministic_repeat(ora):
    x = syn.normal_bf16((512, 512), 3)
    a = gpu_quantize(x, 0, 1, seed=5)
    b = gpu_quantize(x, 0, 1, seed=5)
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])
    c = gpu_quantize(x, 0, 1, seed=6)
    assert not np.array_equal(a[0], c[0])


@pytest.mark.parametrize("kind", ["normal", "t3", "laplace"])
@pytest.mark.parametrize("mode", [(0, 0), (0, 1), (1, 0), (1, 1)])
def test_quantize_sweep_8192_sampled(ora, kind, mode):
    """The 8192 x 8192 quantization sweep at full size, in the launch configuration
    the bench uses; the oracle checks the full-tensor amax / tensor scale and 128
    sampled 16-row groups bit for bit."""
    block_mode, rounding = mode
    n = 8192
    seed = {"normal": 0, "t3": 1, "laplace": 2}[kind]
    x = gen(kind, (n, n), seed)
    packed, sf, g, status = gpu_quantize(x, block_mode, rounding, seed=2024)
    assert status == 0
    amax = ora.tensor_amax(x)
    assert f32_bits(g) == f32_bits(ora.tensor_scale(amax))
    rng = np.random.default_rng(seed)
    groups = np.sort(rng.choice(n // 16, 128, replace=False))
    # scale offsets of rows 0..127 from the oracle; 128-row groups repeat them
    inner = np.array([[ora.sf_offset(i, kb, n) for kb in range(n // 16)] for i in range(128)])
    group_bytes = ora.sf_offset(128, 0, n)
    for grp in groups:
        r0 = int(grp) * 16
        rp, rs = ora.quantize_rows(x, 0, False, None, block_mode, rounding, 2024, amax, r0, r0 + 16)
        assert np.array_equal(packed[r0:r0 + 16], rp), f"rows {r0}.."
        offs = (r0 // 128) * group_bytes + inner[r0 % 128: r0 % 128 + 16]
        assert np.array_equal(sf[offs], rs), f"scales rows {r0}.."
