"""The seeded input generator: determinism, counter-based access, rounding."""
import numpy as np
import torch

import moe_inputs as mi


def test_deterministic_and_counter_based():
    a = mi.normal(0, 3, (1000,), 1.0, "f32")
    b = mi.normal(0, 3, (1000,), 1.0, "f32")
    assert np.array_equal(a, b)
    # any window regenerates alone
    c = mi.normal(0, 3, (101,), 1.0, "f32", first=457)
    assert np.array_equal(a[457:558], c)
    # other seeds / streams differ
    assert not np.array_equal(a, mi.normal(1, 3, (1000,), 1.0, "f32"))
    assert not np.array_equal(a, mi.normal(0, 4, (1000,), 1.0, "f32"))


def test_normal_moments():
    a = mi.normal(0, 1, (1_000_000,), 2.0, "f32").astype(np.float64)
    assert abs(a.mean()) < 0.01
    assert abs(a.std() - 2.0) < 0.01
    # Box-Muller tails: about 0.27% beyond 3 sigma
    frac = np.mean(np.abs(a) > 6.0)
    assert 0.0015 < frac < 0.004


def test_bf16_is_round_to_nearest_even_of_f32():
    f = mi.normal(0, 5, (200_000,), 0.37, "f32")
    h = mi.normal(0, 5, (200_000,), 0.37, "bf16")
    ref = torch.from_numpy(f).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(h, ref)
    # widening is exact
    back = mi.bf16_bits_to_f32(h)
    assert np.array_equal(torch.from_numpy(back).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16), h)


def test_permutation_and_zipf_bias():
    p = mi.permutation(0, mi.STREAM_ZIPF_RANK, 256)
    assert sorted(p.tolist()) == list(range(256))
    inp = mi.make_inputs(mi.SMALL["fine_grained_e256_layer"])
    b = inp["router_b"]
    rank = np.rint(np.exp(-b.astype(np.float64) / 1.1)).astype(int)
    assert sorted(rank.tolist()) == list(range(1, 257))


def test_sample_tokens():
    s = mi.sample_tokens(0, 1000, 64)
    assert len(set(s.tolist())) == 64 and np.all(np.diff(s) > 0) and s.max() < 1000
    assert np.array_equal(mi.sample_tokens(0, 10, 64), np.arange(10))


def test_mxfp4_weights_are_seeded_uniform_codes_with_clustered_scales():
    b1, s1 = mi.mxfp4_weights(0, mi.STREAM_MX_GATE, mi.STREAM_MXS_GATE, 4, 64, 2880, 2880)
    b2, s2 = mi.mxfp4_weights(0, mi.STREAM_MX_GATE, mi.STREAM_MXS_GATE, 4, 64, 2880, 2880)
    assert b1.shape == (4, 64, 90, 16) and s1.shape == (4, 64, 90)
    assert np.array_equal(b1, b2) and np.array_equal(s1, s2)
    nib = np.concatenate([(b1 & 0xF).ravel(), (b1 >> 4).ravel()])
    hist = np.bincount(nib, minlength=16) / nib.size
    assert np.all(np.abs(hist - 1 / 16) < 0.01)
    # 2^(s - 127) * RMS(E2M1) ~ 1/sqrt(2880): the center byte is 120
    assert set(np.unique(s1).tolist()) == {119, 120, 121}
    # any sub-range regenerates alone
    assert np.array_equal(mi.random_bytes(0, 11, (100,), first=37), mi.random_bytes(0, 11, (137,))[37:])
