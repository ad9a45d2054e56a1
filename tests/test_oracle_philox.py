"""Pins for the oracle's Philox4x32-10 and its token draws (CPU only)."""

import os

import numpy as np
import pytest

from oracle import philox

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "philox4x32_10_kat.txt")


def _kat():
    rows = []
    for line in open(GOLDEN):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        lhs, rhs = line.split("->")
        a = [int(x, 16) for x in lhs.split()]
        b = [int(x, 16) for x in rhs.split()]
        rows.append((a[:4], a[4:], b))
    return rows


@pytest.mark.parametrize("ctr,key,want", _kat())
def test_known_answer_vectors(ctr, key, want):
    got = philox.philox4x32_10(ctr, key)
    assert [int(x) for x in got] == want


def test_vectorised_matches_scalar():
    rng = np.random.default_rng(0)
    ctr = rng.integers(0, 2**32, size=(64, 4), dtype=np.uint64)
    key = rng.integers(0, 2**32, size=(64, 2), dtype=np.uint64)
    vec = philox.philox4x32_10(ctr, key)
    for j in range(64):
        assert np.array_equal(vec[j], philox.philox4x32_10(ctr[j], key[j]))


def test_seed_key_split():
    k = philox.seed_key(0x0123456789ABCDEF)
    assert int(k[0]) == 0x89ABCDEF and int(k[1]) == 0x01234567


def test_injective_on_counters():
    # Philox is a bijection of the counter for a fixed key: 2^16 distinct counters
    # give 2^16 distinct 128-bit outputs.
    i = np.arange(1 << 16, dtype=np.uint64)
    w = philox.words(7, i, 3, 1, 0)
    packed = {tuple(r) for r in w.tolist()}
    assert len(packed) == 1 << 16


def test_stream_separation():
    # the four tags, steps and canvases give unrelated words for the same position
    i = np.arange(4096)
    base = philox.words(11, i, 5, 2, 0)[..., 0]
    for (s, c, tag) in [(5, 2, 1), (5, 2, 2), (5, 2, 3), (6, 2, 0), (5, 3, 0)]:
        other = philox.words(11, i, s, c, tag)[..., 0]
        assert np.mean(base == other) < 0.01
    assert np.mean(philox.words(12, i, 5, 2, 0)[..., 0] == base) < 0.01


def test_uniform_token_chi_square():
    V = 64
    n = 200_000
    t = philox.uniform_token(3, np.arange(n), 1, 0, 1, V)
    assert t.min() >= 0 and t.max() < V
    counts = np.bincount(t, minlength=V)
    exp = n / V
    chi2 = ((counts - exp) ** 2 / exp).sum()
    # 63 degrees of freedom: the 99.9% quantile is about 103
    assert chi2 < 103.0


def test_uniform_token_power_of_two_is_shift():
    i = np.arange(10000)
    w0 = philox.words(5, i, 2, 0, 1)[..., 0].astype(np.uint64)
    for logv in (12, 18):
        t = philox.uniform_token(5, i, 2, 0, 1, 1 << logv)
        assert np.array_equal(t, (w0 >> np.uint64(32 - logv)).astype(np.int64))


def test_uniform_token_general_vocab_in_range():
    V = 50257
    t = philox.uniform_token(9, np.arange(100000), 4, 1, 1, V)
    assert t.min() >= 0 and t.max() < V
    assert abs(t.mean() - (V - 1) / 2) < 0.01 * V


def test_words_bit_balance():
    # each output bit is set about half of the time
    w = philox.words(1, np.arange(50000), 0, 0, 0)
    bits = ((w[..., None] >> np.arange(32, dtype=np.uint32)) & 1).mean(axis=0)
    assert np.all(np.abs(bits - 0.5) < 0.02)
