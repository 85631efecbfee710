"""Pins of the oracle's bits-lost proxy against closed forms and invariances.

"MiniMax-H3 NVFP4 -- what the smoothing scale should be calibrated on",
section "Why": a channel whose absmax is below its 16-channel group's absmax
loses log2(group_absmax / channel_absmax) bits, and lambda changes that profile
because the kernel sees X / lambda.  The values below are built from powers of
two so that every ratio, and so every logarithm, is an exact small integer.
"""
import numpy as np

from oracle import svdq_oracle as O


def test_powers_of_two_give_integer_bits():
    ax = np.empty(32, np.float32)
    ax[0] = 8.0
    ax[1:16] = 4.0              # 15 channels one bit below the group's absmax
    ax[16] = 1.0
    ax[17] = 0.125              # three bits below
    ax[18:32] = 0.5             # 14 channels one bit below
    # (15 * 1 + 3 + 14 * 1) / 32 channels
    assert O.bits_lost(ax, None)[0, 0] == 32.0 / 32.0


def test_flat_groups_lose_nothing():
    ax = np.repeat(np.float32([3.0, 0.7, 100.0]), 16)
    assert O.bits_lost(ax, None)[0, 0] == 0.0


def test_lambda_equal_to_the_absmax_flattens_every_group():
    rng = np.random.default_rng(0)
    ax = np.float32(2.0) ** rng.integers(-6, 7, size=64).astype(np.float32)
    assert O.bits_lost(ax, None)[0, 0] > 0.5
    # 1/lambda = 1/ax is exact for powers of two: every smoothed absmax is 1
    assert O.bits_lost(ax, (1.0 / ax).astype(np.float32))[0, 0] == 0.0
    # any absmax: the smoothed values are 1 within one fp32 rounding each
    ax2 = rng.uniform(0.01, 50.0, size=64).astype(np.float32)
    assert abs(O.bits_lost(ax2, (np.float32(1) / ax2).astype(np.float32))[0, 0]) < 4e-7


def test_zero_channels_are_left_out():
    ax = np.zeros(32, np.float32)
    ax[0] = 4.0
    ax[5] = 1.0                 # two bits; the 14 zero channels of the group do not count
    ax[16:32] = 0.0             # a group of zeros counts nothing
    assert O.bits_lost(ax, None)[0, 0] == (0.0 + 2.0) / 2
    assert O.bits_lost(np.zeros(16, np.float32), None)[0, 0] == 0.0


def test_invariances():
    rng = np.random.default_rng(1)
    ax = rng.lognormal(0.0, 1.5, size=(3, 160)).astype(np.float32)
    il = rng.uniform(0.2, 5.0, size=(2, 160)).astype(np.float32)
    base = O.bits_lost(ax, il)
    assert base.shape == (2, 3) and np.all(base > 0)
    # a power-of-two scale of all statistics (exact in fp32) changes nothing
    assert np.array_equal(O.bits_lost(ax * np.float32(8), il), base)
    assert np.array_equal(O.bits_lost(ax, il * np.float32(0.25)), base)
    # permuting channels inside every group changes nothing (the mean is order-free up to rounding)
    perm = np.concatenate([g * 16 + rng.permutation(16) for g in range(10)])
    np.testing.assert_allclose(O.bits_lost(ax[:, perm], il[:, perm]), base, rtol=1e-14)
    # modalities and candidates are independent rows of the result
    np.testing.assert_array_equal(O.bits_lost(ax[1:2], il[1:2])[0, 0], base[1, 1])


def test_uniform_group_profile_closed_form():
    # channel absmax a * 2^-j inside each group (j = 0..15): bits lost 0..15, mean 7.5
    ax = np.tile(np.float32(2.0) ** -np.arange(16, dtype=np.float32), 4) * np.float32(3.0)
    assert O.bits_lost(ax, None)[0, 0] == 7.5
