"""The seeded synthetic inputs (CPU only), checked against the recipe they are
documented with.

- bf16 rounding is nearest-even, the same as torch's.
- Draws are deterministic per seed.
- The MLP tensors have the stated spreads (X ~ N(0,1), W ~ N(0, 0.02^2),
  dY ~ N(0, 1e-3^2)), and outliers (x50) come at the stated rate.
- MoE routing gives every token `topk` distinct experts with Zipf(1.1)
  popularity (p_e ~ (e+1)^-1.1, about a quarter of the routing mass on the top
  expert).
- The expert-contiguous layout places every routed copy exactly once, in token
  order, in segments padded with zero rows."""
import numpy as np
import pytest
import torch

from nvfp4_bit_quantized_amax_b200 import synthetic as syn


def test_bf16_rounding_matches_torch():
    rng = np.random.default_rng(0)
    x = np.concatenate([
        rng.standard_normal(20000).astype(np.float32),
        (rng.standard_normal(2000) * 1e-30).astype(np.float32),
        np.array([0.0, -0.0, 1.0 + 2.0 ** -8, 1.0 + 3 * 2.0 ** -8, 3.0e38, -3.0e38], dtype=np.float32),
    ])
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(syn.f32_to_bf16_bits(x), ref)
    back = syn.bf16_bits_to_f32(ref)
    assert np.array_equal(back, torch.from_numpy(ref.view(np.int16)).view(torch.bfloat16).float().numpy())


def test_draws_are_seeded():
    a, b, c = syn.normal_bf16((64, 64), 5), syn.normal_bf16((64, 64), 5), syn.normal_bf16((64, 64), 6)
    assert np.array_equal(a, b) and not np.array_equal(a, c)
    assert np.array_equal(syn.rht_signs(3), syn.rht_signs(3))
    s = syn.rht_signs(3)
    assert s.shape == (16,) and s.dtype == np.int8 and set(np.unique(s)) <= {-1, 1}


def test_mlp_spreads_and_outlier_rate():
    X, W, dY = syn.mlp_inputs(512, 640, 768, seed=1)
    assert X.shape == (512, 640) and W.shape == (768, 640) and dY.shape == (512, 768)
    for bits, std in ((X, 1.0), (W, 0.02), (dY, 1e-3)):
        v = syn.bf16_bits_to_f32(bits).astype(np.float64)
        assert abs(v.mean()) < 0.02 * std
        assert v.std() == pytest.approx(std, rel=0.02)
    z = syn.bf16_bits_to_f32(syn.normal_bf16((400, 500), 2, outlier_prob=0.01)).astype(np.float64)
    share = (np.abs(z) > 8.0).mean()   # N(0,1) almost never exceeds 8; x50 outliers mostly do
    assert 0.008 < share < 0.011


def test_moe_routing_zipf_top4():
    T, E, k = 16384, 64, 4
    ids = syn.moe_topk_ids(T, E, k, 1.1, seed=0)
    assert ids.shape == (T, k)
    assert all(len(set(row)) == k for row in ids[:2000].tolist())
    assert (np.sort(ids, axis=1)[:, 1:] != np.sort(ids, axis=1)[:, :-1]).all()
    counts = np.bincount(ids.ravel(), minlength=E)
    assert counts.sum() == T * k
    assert counts[0] == counts.max()             # the most popular expert is expert 0
    assert 11000 < counts[0] < 12300             # ~0.71 of the tokens pick it among their 4
    assert counts.min() > 100
    assert (np.diff(counts[:8]) < 0).all()       # popularity falls with the rank


def test_moe_layout_places_every_copy_once():
    ids = syn.moe_topk_ids(3000, 16, 4, 1.1, seed=4)
    for pad in (64, 128):
        group_rows, row_src, slots = syn.moe_layout(ids, 16, pad)
        counts = np.bincount(ids.ravel(), minlength=16)
        assert (group_rows % pad == 0).all() and (group_rows >= counts).all()
        assert (group_rows - counts < pad).all()
        assert row_src.size == group_rows.sum()
        t = np.repeat(np.arange(ids.shape[0]), 4).reshape(ids.shape)
        assert (row_src[slots] == t).all()       # the copy of token t lands on a row of t
        assert np.unique(slots).size == slots.size
        offs = np.concatenate([[0], np.cumsum(group_rows)])
        for e in range(16):
            seg = row_src[offs[e]: offs[e + 1]]
            real = seg[: counts[e]]
            assert (real >= 0).all() and (np.diff(real) > 0).all()   # its tokens, in order
            assert (seg[counts[e]:] == -1).all()                     # then padding
            assert set(real.tolist()) == set(np.nonzero((ids == e).any(axis=1))[0].tolist())


def test_moe_inputs_pad_rows_are_zero():
    d = syn.moe_inputs(512, 8, 128, 64, 2, 1.1, seed=0, pad=128)
    assert d["dY"].shape == (int(d["group_rows"].sum()), 64)
    assert (d["dY"][d["row_src"] < 0] == 0).all()
    assert (d["dY"][d["row_src"] >= 0] != 0).any()
    assert d["W"].shape == (8, 64, 128) and d["X"].shape == (512, 128)
