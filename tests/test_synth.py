"""The seeded generator: published splitmix64 vector, determinism, slices,
distribution and exact dtype rounding (CPU only)."""

import numpy as np
import torch

from io_aware_exact_30_b200 import synth


def test_splitmix64_published_vector():
    # splitmix64 seeded with state 0 yields 0xE220A8397B1DCDAF, 0x6E789E6AA1B965F4, ...
    g = int(synth.GAMMA)
    out = [int(synth.mix64(np.uint64((i * g) & (2**64 - 1)))) for i in (1, 2, 3)]
    assert out == [0xE220A8397B1DCDAF, 0x6E789E6AA1B965F4, 0x06C45D188009454F]


def test_deterministic_and_streams_differ():
    a = synth.tensor(7, 0, (3, 5, 8))
    b = synth.tensor(7, 0, (3, 5, 8))
    c = synth.tensor(7, 1, (3, 5, 8))
    d = synth.tensor(8, 0, (3, 5, 8))
    np.testing.assert_array_equal(a, b)
    assert (a != c).mean() > 0.9 and (a != d).mean() > 0.9


def test_counter_addressable_slices():
    n = 10_001
    full = synth.gaussian(3, 2, n)
    w = synth.words(3, 2, 0, 2 * ((n + 1) // 2))
    w2 = synth.words(3, 2, 100, 50)
    np.testing.assert_array_equal(w[100:150], w2)
    # chunked generation equals one pass
    old = synth._CHUNK
    try:
        synth._CHUNK = 1001
        np.testing.assert_array_equal(synth.gaussian(3, 2, n), full)
    finally:
        synth._CHUNK = old


def test_distribution_moments():
    z = synth.gaussian(0, 0, 400_000, sigma=0.5)
    assert abs(z.mean()) < 0.005
    assert abs(z.std() - 0.5) < 0.005
    assert abs((z ** 4).mean() / z.var() ** 2 - 3.0) < 0.05  # Gaussian kurtosis


def test_bf16_rounding_matches_torch():
    x = synth.gaussian(1, 0, 50_000, sigma=3.0)
    bits = synth.round_bf16_bits(x)
    ref = torch.from_numpy(x.astype(np.float32)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    np.testing.assert_array_equal(bits, ref)
    back = synth.bf16_bits_to_f64(bits)
    assert np.all(np.abs(back - x) <= np.abs(x) * 2.0 ** -8 + 1e-30)


def test_fp16_storage_upcast_exact():
    t = synth.tensor(5, 3, (4, 7), sigma=0.5, dtype="fp16")
    assert t.dtype == np.float16
    np.testing.assert_array_equal(synth.to_f64(t, "fp16"), t.astype(np.float64))
