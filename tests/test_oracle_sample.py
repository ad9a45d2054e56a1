"""Pins of the oracle's sampled acceptance (a draw from softmax(z / T) in two
levels: a Gumbel-max race between 64-entry chunks on their log-masses, then the
inverse CDF inside the winning chunk).

What fixes the sampler independently of its code: the Gumbel distribution's
closed-form mean, variance and CDF, the frequencies of its draws against
softmax(z) (chi-square), shift invariance, and the limits (a single finite logit;
a logit scale so large that the noise cannot reorder the entries).  Planted
mistakes - in the noise formula, and a draw inside the chunk that reuses the
chunk race's word - are shown to fail the frequency pin.
"""

import math

import numpy as np
import pytest
from scipy import stats as sps

from oracle import philox, stage

EULER_GAMMA = 0.5772156649015329
V256 = np.arange(256)
# four chunks of different mass (with two chunks a sign slip in the noise cannot be seen:
# the difference of two Gumbel variables is symmetric), probabilities spread over ~400x
Z256 = 1.5 * np.sin(0.37 * V256) + 1.0 * (V256 // 64)


def _frequencies(z, n_steps=40, n_canvas=2, seed=2024):
    z = np.asarray(z, np.float64)
    V = z.shape[0]
    counts = np.zeros(V, np.int64)
    rows = np.tile(z, (256, 1))
    for c in range(n_canvas):
        for s in range(1, n_steps + 1):
            smp, _, _ = stage.gumbel_sample(rows, seed, s, c, range(256))
            counts += np.bincount(smp, minlength=V)
    return counts


def _chi2_sf(counts, p):
    n = counts.sum()
    exp = n * p
    chi2 = float(((counts - exp) ** 2 / exp).sum())
    return sps.chi2.sf(chi2, len(p) - 1)


def _softmax(z):
    p = np.exp(z - z.max())
    return p / p.sum()


def test_gumbel_moments_and_cdf():
    """Standard Gumbel: mean = Euler's gamma, variance = pi^2 / 6, CDF exp(-exp(-x))."""
    w = np.concatenate([philox.chunk_words(7, i, 3, 1, 4096)[:, 0] for i in range(16)])   # 65536 words
    g = stage.gumbel_from_words(w)
    se = math.pi / math.sqrt(6.0) / math.sqrt(g.size)
    assert abs(g.mean() - EULER_GAMMA) < 5 * se
    assert abs(g.var() - math.pi ** 2 / 6.0) < 0.05
    for x in (-1.0, 0.0, 1.0, 3.0):
        assert abs((g <= x).mean() - math.exp(-math.exp(-x))) < 0.01


def test_sample_frequencies_match_softmax():
    counts = _frequencies(Z256)
    assert counts.sum() == 2 * 40 * 256
    assert _chi2_sf(counts, _softmax(Z256)) > 1e-4
    # also the chunk totals on their own (the first level of the draw)
    p = _softmax(Z256)
    assert _chi2_sf(counts.reshape(4, 64).sum(1), p.reshape(4, 64).sum(1)) > 1e-4


@pytest.mark.parametrize("wrong", ["exponential", "sign", "reused_word"])
def test_frequency_pin_catches_planted_mistakes(monkeypatch, wrong):
    """The same chi-square rejects plausible slips in the noise or the word use."""
    if wrong == "reused_word":
        real = philox.chunk_words

        def planted(seed, i, s, c, n):
            w = real(seed, i, s, c, n)
            return np.stack([w[:, 0], w[:, 0]], axis=1)     # the draw inside the chunk reuses word 0

        monkeypatch.setattr(philox, "chunk_words", planted)
    else:
        real = stage.gumbel_from_words

        def planted(w):
            g = real(w)
            return np.exp(-g) if wrong == "exponential" else -g   # -ln u, or +ln(-ln u)

        monkeypatch.setattr(stage, "gumbel_from_words", planted)
    counts = _frequencies(Z256, n_steps=20, n_canvas=1)
    p = _softmax(Z256)
    # either the per-entry test or the chunk-level one (the more powerful for the race's noise)
    assert min(_chi2_sf(counts, p), _chi2_sf(counts.reshape(4, 64).sum(1), p.reshape(4, 64).sum(1))) < 1e-6


def test_uniform_logits_give_uniform_samples():
    counts = _frequencies(np.zeros(64), n_steps=20, n_canvas=1)
    assert _chi2_sf(counts, np.full(64, 1 / 64)) > 1e-4


def test_shift_invariance():
    rng = np.random.default_rng(3)
    z = rng.normal(size=(32, 256))
    a, _, _ = stage.gumbel_sample(z, 11, 5, 2, range(32))
    b, _, _ = stage.gumbel_sample(z + 7.25, 11, 5, 2, range(32))
    assert np.array_equal(a, b)


def test_single_finite_logit_and_zero_temperature_limit():
    z = np.full((8, 128), -np.inf)
    z[:, 77] = 3.0
    smp, gap, _ = stage.gumbel_sample(z, 1, 1, 0, range(8))
    assert np.all(smp == 77) and np.all(np.isinf(gap))
    # logits scaled far beyond the noise range (|g| < 23 for 32-bit words): the sample is the argmax
    rng = np.random.default_rng(4)
    z = rng.permuted(np.tile(np.arange(128, dtype=np.float64), (16, 1)), axis=1)
    smp, _, _ = stage.gumbel_sample(z * 100.0, 9, 2, 1, range(16))
    assert np.array_equal(smp, z.argmax(1))


def test_noise_range_and_stream_separation():
    w = philox.chunk_words(5, 0, 1, 0, 1 << 15).reshape(-1)
    g = stage.gumbel_from_words(w)
    assert np.isfinite(g).all()
    assert g.max() < -math.log(0.5 / 2.0 ** 32) + 1e-9          # u < 1 - 2^-33
    assert g.min() > -math.log(-math.log(0.5 / 2.0 ** 32)) - 1e-9
    w00 = philox.chunk_words(5, 0, 1, 0, 32)
    assert not np.array_equal(w00, philox.chunk_words(5, 1, 1, 0, 32))
    assert not np.array_equal(w00, philox.chunk_words(5, 0, 2, 0, 32))
    assert not np.array_equal(w00, philox.chunk_words(5, 0, 1, 1, 32))


def test_step_rows_sampled_mode_accepts_the_sample():
    """accept_mode 1: accepted positions take the sample, the others the re-noise draw."""
    rng = np.random.default_rng(8)
    V, d = 256, 32
    W = stage.f64_to_bf16(rng.normal(size=(V, d)) * 0.5)
    Wd = stage.bf16_to_f64(W)
    k = rng.integers(0, V, 6)
    gains = np.array([40.0, 40.0, 40.0, 0.0, 0.0, 3.0])
    h = stage.f64_to_bf16(Wd[k] * (gains / (Wd[k] ** 2).sum(1))[:, None] * 0.8 * 4)
    pos = np.arange(6)
    o = stage.step_rows(h, W, W, 0.8, 0.1, 77, 4, 0, pos, V, want_selfcond=False, accept_mode=1)
    z = stage.logits_chunked(stage.bf16_to_f64(h), W, 0.8)
    smp, _, _ = stage.gumbel_sample(z, 77, 4, 0, pos)
    ren = philox.uniform_token(77, pos, 4, 0, philox.TAG_RENOISE, V)
    acc = o["H"] <= 0.1
    assert acc.any() and (~acc).any()
    assert np.array_equal(o["tokens"], np.where(acc, smp, ren))
    assert np.array_equal(o["sample"], smp)
