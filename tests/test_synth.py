"""The seeded input generator: published SplitMix64 values, determinism and
the distribution of the synthetic workloads (CPU only)."""
import numpy as np

from ternary_weight_decoder_b200 import synth


def test_splitmix64_published_sequence():
    # SplitMix64 seeded with 0 (Steele, Lea & Flood 2014; the public-domain
    # reference implementation by S. Vigna) starts with these three outputs.
    got = synth.raw_outputs(0, 0, 3).tolist()
    assert got == [0xE220A8397B1DCDAF, 0x6E789E6AA1B965F4, 0x06C45D188009454F]


def test_deterministic_and_offset_consistent():
    k = synth.stream_key(3, 4, synth.KIND_W)
    a = synth.normal(k, 1000, 0.02)
    b = synth.normal(k, 1000, 0.02)
    assert (a == b).all()
    c = synth.normal(k, 300, 0.02, offset=700)
    assert (a[700:] == c).all()
    W = synth.weights(3, 4, 10, 100)
    Wr = synth.weights(3, 4, 10, 100, rows=slice(4, 7))
    assert (W[4:7] == Wr).all()


def test_streams_differ_by_label():
    a = synth.weights(0, 0, 4, 64)
    b = synth.weights(0, 1, 4, 64)
    c = synth.weights(1, 0, 4, 64)
    assert not np.array_equal(a, b) and not np.array_equal(a, c)


def test_normal_moments():
    z = synth.normal(synth.stream_key(9, 9, 9), 400_000, 1.0).astype(np.float64)
    assert abs(z.mean()) < 5 / np.sqrt(z.size)
    assert abs(z.std() - 1.0) < 0.01
    assert abs((np.abs(z) < 1).mean() - 0.6827) < 0.005


def test_outlier_channels():
    K = 1536
    ch = synth.outlier_channels(2, 5, K)
    assert len(ch) == 15 and len(set(ch.tolist())) == 15
    assert ch.min() >= 0 and ch.max() < K
    x = synth.activations(2, 5, 3, K)
    x0 = synth.activations(2, 5, 3, K, outliers=False)
    assert (x[:, ch] == x0[:, ch] * np.float32(20)).all()
    mask = np.ones(K, bool)
    mask[ch] = False
    assert (x[:, mask] == x0[:, mask]).all()
    assert len(synth.outlier_channels(0, 6, 8960)) == 89
