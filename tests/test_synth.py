"""Host-side generator checks (CPU only)."""
import os

import numpy as np

import lsa_synth as S

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "splitmix64_state0.txt")


def _golden_words():
    return [int(x, 16) for x in open(GOLDEN).read().split() if x.startswith("0x")]


def test_splitmix64_reference_outputs():
    # Element i of a stream is the (i+1)-th output from the stream key, so a
    # stream whose key is 0 reproduces SplitMix64 started from state 0.
    states = np.array([(S.GOLDEN * i) % 2**64 for i in (1, 2, 3)], dtype=np.uint64)
    assert [int(x) for x in S.mix64(states)] == _golden_words()


def test_hash_range_is_counter_based():
    a = S.hash_range(0, 5, 0, 1000)
    b = S.hash_range(0, 5, 400, 100)
    np.testing.assert_array_equal(a[400:500], b)
    assert not np.array_equal(S.hash_range(0, 6, 0, 100), a[:100])
    assert not np.array_equal(S.hash_range(1, 5, 0, 100), a[:100])


def test_bf16_rounding_nearest_even():
    x = np.array([1.0, 1.0 + 2**-8, 1.0 + 3 * 2**-8, 1.0 + 2**-7, -2.5, 1.0 + 2**-8 + 2**-20],
                 dtype=np.float32)
    got = S.bf16_bits_to_f32(S.f32_to_bf16_bits(x))
    # halfway 1+2^-8 ties to even (1.0); 1+3*2^-8 ties to even (1+2^-6);
    # just above halfway rounds up.
    np.testing.assert_array_equal(got, np.array([1.0, 1.0, 1.0 + 2**-6, 1.0 + 2**-7, -2.5, 1.0 + 2**-7],
                                                dtype=np.float32))


def test_normal_moments():
    x = S.normal_f32(0, 3, 0, 1 << 20).astype(np.float64)
    assert abs(x.mean()) < 5e-3
    assert abs(x.var() - 1.0) < 5e-3
    # 8-term Irwin-Hall: bounded at 4.90 sigma, but well past the 4-term 3.46
    assert np.abs(x).max() <= 4.90
    assert (np.abs(x) > 3.5).sum() > 100
    y = S.normal_f32(0, 4, 0, 1 << 18, sigma=S.W_SIGMA).astype(np.float64)
    assert abs(y.var() * 32 - 1.0) < 1e-2


def test_normal_is_one_fp32_multiply():
    # element i: the 16-bit fields of stream words 2i and 2i+1, summed, centred
    h = S.hash_range(9, 1, 0, 100)
    m = np.uint64(0xFFFF)
    f = sum(((h >> np.uint64(16 * q)) & m).astype(np.int64) for q in range(4))
    s = f[0::2] + f[1::2] - 4 * 65535
    scale = np.float32(1.0 / np.sqrt(8 * (65536.0 ** 2 - 1) / 12))
    expect = np.float32(s.astype(np.float32)) * scale
    np.testing.assert_array_equal(S.normal_f32(9, 1, 0, 50), expect)
    np.testing.assert_array_equal(S.normal_f32_at(9, 1, np.array([7, 3, 49])), expect[[7, 3, 49]])
    np.testing.assert_array_equal(S.normal_f32(9, 1, 20, 5), expect[20:25])


def test_rms_rows():
    bits = S.rms_rows_bf16(0, 2, 0, 64, 128)
    x = S.bf16_bits_to_f64(bits)
    rms = np.sqrt((x * x).mean(axis=1))
    assert np.all(np.abs(rms - 1.0) < 1e-2)


def test_decode_lengths_range():
    L = S.decode_lengths(0, 64, 16384, 32768)
    assert L.min() >= 16384 and L.max() <= 32768 and len(set(L.tolist())) > 50
