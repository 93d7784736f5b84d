"""Host-side checks of the seeded input generator (no method arithmetic involved)."""

import pytest
import numpy as np
import torch

import oracle as O
import synth as S


def test_splitmix64_reference_values():
    """SplitMix64 seeded with 1234567: published reference outputs of the generator."""
    got = [int(S.draw(1234567, n)) for n in range(3)]
    assert got == [6457827717110365317, 3203168211198807973, 9817491932198370423]


def test_bf16_rounding_matches_torch():
    rng = np.random.default_rng(0)
    x = (rng.standard_normal(100000) * np.exp(rng.uniform(-20, 20, 100000))).astype(np.float32)
    x[:4] = [1.00390625, 1.01171875, -1.00390625, 3.0]  # ties: to even
    ours = S.f32_to_bf16_bits(x)
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(ours, ref)


def test_normal_moments_and_bounds():
    z = S.fill_normal(7, S.PREFIX_K, (1, 1, 1, 1 << 18, 1), dtype="f32").ravel().astype(np.float64)
    assert abs(z.mean()) < 0.01 and abs(z.var() - 1.0) < 0.01
    assert np.abs(z).max() <= 2 * 65535 * float(S.INV_STD) + 1e-6


def test_blocks_are_consistent_slices():
    """A block drawn at an offset equals the same slice of a bigger block."""
    big = S.fill_normal(3, S.VERIFY_K, (2, 3, 2, 5, 16), head_dim=8)
    part = S.fill_normal(3, S.VERIFY_K, (1, 2, 1, 3, 16), r0=1, b0=1, l0=1, p0=2, head_dim=8)
    assert np.array_equal(big[1:2, 1:3, 1:2, 2:5], part)
    sub = S.fill_normal(3, S.VERIFY_K, (2, 3, 2, 5, 8), x0=8, head_dim=8)
    assert np.array_equal(big[..., 8:16], sub)


def test_head_scales_range():
    s = S.head_scales(2, 4, 8)
    assert s.dtype == np.float32 and s.shape == (4, 8)
    assert np.all(s >= 0.5) and np.all(s < 2.0)


def test_accept_lengths_means():
    for mean in (2.5, 3.5, 4.7, 5.0, 6.0):
        a = S.accept_lengths(11, 4000, 16, 16, mean)
        assert a.min() >= 0 and a.max() <= 16
        assert abs(a.mean() - mean) < 0.15
    u = S.accept_lengths(0, 4000, 1, 4, None)
    assert set(np.unique(u)) == {0, 1, 2, 3, 4}


def test_token_ids_yield_the_drawn_accepts():
    acc = S.accept_lengths(5, 50, 16, 16, 4.0)
    draft, target = S.token_ids(5, 50, 16, 16, acc, 151936)
    for r in range(50):
        for b in range(16):
            a, nxt = O.accept_scan(draft[r, b], target[r, b])
            assert a == acc[r, b] and nxt == target[r, b, a]


def test_prefix_lengths_range():
    p = S.prefix_lengths(3, 1000, 98304, 131072)
    assert p.min() >= 98304 and p.max() <= 131072 and len(np.unique(p)) > 900


def test_device_fill_refuses_scale_reads_past_the_array():
    """The device generator's wrapper checks, before any launch, that the per-head scale
    array covers every (layer, head) the block reads."""
    import synth as S
    with pytest.raises(ValueError):
        S.device_fill_normal(1, 0, S.PREFIX_K, (1, 1, 2, 4, 256), l0=3, head_dim=128, scale_ptr=1, scale_heads=8,
                             scale_layers=4)
    with pytest.raises(ValueError):
        S.device_fill_normal(1, 0, S.PREFIX_K, (1, 1, 1, 4, 256), x0=7 * 128, head_dim=128, scale_ptr=1,
                             scale_heads=8, scale_layers=4)
