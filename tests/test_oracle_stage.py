"""Pins for the float64 oracle of one denoising step (CPU only).

Each test ties the oracle to something other than itself: a closed form,
a special case that reduces to a textbook quantity, an invariant of the
method, or brute force in pure Python on tiny inputs.
"""

import math

import numpy as np
import pytest

from oracle import stage, philox


def _rand_bf16(shape, scale, seed):
    rng = np.random.default_rng(seed)
    return stage.f64_to_bf16(rng.standard_normal(shape) * scale)


# ---------------------------------------------------------------- bf16 helpers
def test_bf16_roundtrip_exact():
    u = np.arange(0, 1 << 16, dtype=np.uint32).astype(np.uint16)
    x = stage.bf16_to_f64(u)
    finite = np.isfinite(x)
    assert np.array_equal(stage.f64_to_bf16(x[finite]), u[finite])


def test_bf16_round_to_nearest_even():
    # 1 + 2^-8 lies halfway between bf16 1.0 and 1 + 2^-7: ties go to the even mantissa (1.0)
    assert stage.bf16_to_f64(stage.f64_to_bf16(1.0 + 2.0 ** -8)) == 1.0
    # 1 + 3*2^-8 lies halfway between 1 + 2^-7 (odd) and 1 + 2^-6 (even)
    assert stage.bf16_to_f64(stage.f64_to_bf16(1.0 + 3 * 2.0 ** -8)) == 1.0 + 2.0 ** -6
    assert stage.bf16_to_f64(stage.f64_to_bf16(1.0 + 2.0 ** -8 + 2.0 ** -20)) == 1.0 + 2.0 ** -7


# ---------------------------------------------------------------- schedule
def test_temperature_endpoints_and_linearity():
    S = 48
    Ts = [stage.temperature(s, S) for s in range(1, S + 1)]
    assert Ts[0] == np.float32(0.8) and Ts[-1] == np.float32(0.4)
    d = np.diff(np.array(Ts, np.float64))
    assert np.all(d < 0) and np.allclose(d, -0.4 / 47, atol=1e-7)
    assert stage.temperature(1, 1) == np.float32(0.8)


# ---------------------------------------------------------------- closed forms
def test_uniform_logits_entropy_is_ln_V():
    V, d = 4096, 16
    W = stage.bf16_to_f64(_rand_bf16((V, d), 0.02, 1))
    h = np.zeros((3, d))
    st = stage.distribution_stats(stage.logits(h, W, 0.8))
    assert np.allclose(st["H"], math.log(V), atol=1e-12)
    assert np.allclose(st["lse"], math.log(V), atol=1e-12)
    assert np.all(st["argmax"] == 0)            # all tied: smallest index
    sc = stage.self_conditioning(st["p"], W)
    assert np.allclose(sc, W.mean(axis=0)[None, :], atol=1e-15)


def test_one_hot_spike_entropy_vanishes():
    V, d = 4096, 64
    W = stage.bf16_to_f64(_rand_bf16((V, d), 0.02, 2))
    k = 1234
    h = (200.0 * W[k] / (W[k] @ W[k]))[None, :]
    st = stage.distribution_stats(stage.logits(h, W, 0.8))
    assert st["argmax"][0] == k
    assert st["H"][0] < 1e-6
    assert abs(st["lse"][0] - st["max"][0]) < 1e-6


def test_two_way_tie_entropy_is_ln2():
    z = np.full((1, 100), -1e4)
    z[0, 7] = z[0, 42] = 50.0
    st = stage.distribution_stats(z)
    assert abs(st["H"][0] - math.log(2.0)) < 1e-12
    assert st["argmax"][0] == 7
    assert st["top2gap"][0] == 0.0


def test_k_way_uniform_entropy_is_ln_k():
    for k in (1, 3, 17):
        z = np.full((1, 64), -1e5)
        z[0, :k] = 3.0
        assert abs(stage.distribution_stats(z)["H"][0] - math.log(k)) < 1e-12


def test_zero_temperature_selfcond_is_argmax_row():
    V, d = 512, 32
    W = stage.bf16_to_f64(_rand_bf16((V, d), 0.02, 3))
    E = stage.bf16_to_f64(_rand_bf16((V, d), 0.02, 4))
    h = stage.bf16_to_f64(_rand_bf16((8, d), 1.0, 5))
    st = stage.distribution_stats(stage.logits(h, W, 1e-6))
    ok = st["top2gap"] > 40.0               # every other weight is below e^-40
    assert ok.sum() >= 6
    sc = stage.self_conditioning(st["p"], E)
    assert np.allclose(sc[ok], E[st["argmax"][ok]], atol=1e-12)


def test_entropy_shift_invariance_and_bounds():
    rng = np.random.default_rng(6)
    z = rng.standard_normal((20, 300)) * 3
    a = stage.distribution_stats(z)
    b = stage.distribution_stats(z + 123.25)
    assert np.allclose(a["H"], b["H"], atol=1e-11)
    assert np.all(a["H"] >= 0) and np.all(a["H"] <= math.log(300) + 1e-12)
    assert np.array_equal(a["argmax"], b["argmax"])


# ---------------------------------------------------------------- brute force
def _brute(h, W, E, T):
    """Pure-Python loops: logits, softmax, H = -sum p ln p, argmax, self-conditioning."""
    n, d = len(h), len(h[0])
    V = len(W)
    out = []
    for i in range(n):
        z = [sum(h[i][k] * W[v][k] for k in range(d)) / T for v in range(V)]
        m = max(z)
        e = [math.exp(x - m) for x in z]
        s = sum(e)
        p = [x / s for x in e]
        H = -sum(pi * math.log(pi) for pi in p if pi > 0)
        am = min(v for v in range(V) if z[v] == m)
        sc = [sum(p[v] * E[v][k] for v in range(V)) for k in range(d)]
        out.append((H, am, m + math.log(s), sc))
    return out


@pytest.mark.parametrize("V,d,T,seed", [(64, 8, 0.8, 10), (37, 5, 0.4, 11), (16, 8, 2.0, 12)])
def test_brute_force_tiny(V, d, T, seed):
    W = stage.bf16_to_f64(_rand_bf16((V, d), 0.5, seed))
    E = stage.bf16_to_f64(_rand_bf16((V, d), 0.5, seed + 100))
    h = stage.bf16_to_f64(_rand_bf16((6, d), 1.0, seed + 200))
    st = stage.distribution_stats(stage.logits(h, W, T))
    sc = stage.self_conditioning(st["p"], E)
    ref = _brute(h.tolist(), W.tolist(), E.tolist(), T)
    for i, (H, am, lse, scb) in enumerate(ref):
        assert abs(st["H"][i] - H) < 1e-12
        assert st["argmax"][i] == am
        assert abs(st["lse"][i] - lse) < 1e-12
        assert np.allclose(sc[i], scb, atol=1e-14)


def test_denoise_step_matches_pieces():
    V, d = 256, 16
    W = _rand_bf16((V, d), 0.3, 20)
    h = _rand_bf16((512, d), 1.0, 21)
    seeds = np.array([5, 9], np.uint64)
    r = stage.denoise_step(h, W, W, 0.8, 1.5, seeds, 4, V)
    for c in range(2):
        sl = slice(256 * c, 256 * (c + 1))
        st = stage.distribution_stats(stage.logits(stage.bf16_to_f64(h[sl]), stage.bf16_to_f64(W), 0.8))
        ren = philox.uniform_token(int(seeds[c]), np.arange(256), 4, c, 1, V)
        want = np.where(st["H"] <= 1.5, st["argmax"], ren)
        assert np.array_equal(r["tokens"][sl], want)
        assert abs(r["mean_H"][c] - st["H"].mean()) < 1e-12


# ---------------------------------------------------------------- split-vocabulary merge
def _stats_of(z, parts, order):
    pieces = []
    for a, b in parts:
        s = stage.partial_stats(z[:, a:b])
        pieces.append((s, a))
    acc, off = pieces[order[0]]
    acc = dict(acc)
    acc["a"] = np.asarray(acc["a"]) + off
    for j in order[1:]:
        s, o = pieces[j]
        acc = stage.merge_stats(acc, s, o)
    return stage.finish_stats(acc)


def test_merge_associative_commutative():
    rng = np.random.default_rng(30)
    z = rng.standard_normal((10, 1000)) * 4
    z[3, 500] = z[3, 200] = 40.0            # exact tie across ranges: smallest index must win
    direct = stage.distribution_stats(z)
    for trial in range(20):
        cuts = np.sort(rng.choice(np.arange(1, 1000), size=rng.integers(1, 9), replace=False))
        bounds = [0, *cuts.tolist(), 1000]
        parts = list(zip(bounds[:-1], bounds[1:]))
        order = rng.permutation(len(parts)).tolist()
        f = _stats_of(z, parts, order)
        assert np.allclose(f["H"], direct["H"], atol=1e-12)
        assert np.allclose(f["lse"], direct["lse"], atol=1e-12)
        assert np.array_equal(f["argmax"], direct["argmax"])
    assert direct["argmax"][3] == 200


# ---------------------------------------------------------------- sampler and stop rule
def test_accept_is_inclusive_at_bound():
    H = np.array([0.1, np.nextafter(0.1, 1.0), 0.0, 5.0])
    tok, acc = stage.eb_accept(H, np.array([1, 2, 3, 4]), 0.1, np.array([10, 20, 30, 40]))
    assert acc.tolist() == [1, 0, 1, 0]
    assert tok.tolist() == [1, 20, 3, 40]


def test_stop_rule_sequences():
    a = np.arange(256)
    b = a.copy()
    b[5] = 7
    # identical predictions and low entropy from step 1: earliest stop is step 3
    st, prev, stops = 0, None, []
    for s in range(1, 6):
        st, stop = stage.stop_update(0.001, a, prev, st, s)
        prev = a
        stops.append(stop)
    assert stops == [False, False, True, True, True]
    # a change resets the count
    seq = [a, a, b, b, b]
    st, prev, res = 0, None, []
    for s, x in enumerate(seq, 1):
        st, stop = stage.stop_update(0.0, x, prev, st, s)
        prev = x
        res.append((st, stop))
    assert res == [(0, False), (1, False), (0, False), (1, False), (2, True)]
    # stable but uncertain: never stops; threshold is strict
    st, prev = 0, None
    for s in range(1, 10):
        st, stop = stage.stop_update(0.005, a, prev, st, s)
        prev = a
        assert not stop
    assert st == 8


def test_init_tokens_uniform_stream():
    t = stage.init_tokens(123, 0, 262144)
    assert t.shape == (256,) and t.min() >= 0 and t.max() < 262144
    assert np.array_equal(t, philox.uniform_token(123, np.arange(256), 0, 0, 0, 262144))


# ---------------------------------------------------------------- stub hidden
def test_stub_exact_without_noise():
    V, d = 512, 16
    E = _rand_bf16((V, d), 0.02, 40)
    tok = np.arange(256) % V
    h, tgt = stage.stub_hidden(E, tok, 3, 8, 0, 8, gain=1.0, noise=0.0)     # a = 1
    assert np.array_equal(h, E[tgt])
    assert np.array_equal(tgt, philox.uniform_token(3, np.arange(256), 0, 0, 2, V))
    h0, _ = stage.stub_hidden(E, tok, 3, 0, 0, 8, gain=1.0, noise=0.0)      # a = 0
    assert np.array_equal(h0, E[tok])


def test_stub_noise_is_standard_normal():
    V, d = 64, 256
    E = np.zeros((V, d), np.uint16)
    h, _ = stage.stub_hidden(E, np.zeros(256, np.int64), 1, 1, 0, 4, gain=1.0, noise=1.0)
    x = stage.bf16_to_f64(h).ravel()
    assert abs(x.mean()) < 0.01 and abs(x.var() - 1.0) < 0.02
    # fourth moment of a normal is 3
    assert abs((x ** 4).mean() - 3.0) < 0.1


# ---------------------------------------------------------------- planted mistakes
def test_pins_catch_planted_mistakes(monkeypatch):
    """Plant plausible mistakes in the oracle and check that a pin fails."""
    W = stage.bf16_to_f64(_rand_bf16((64, 8), 0.5, 10))
    h = stage.bf16_to_f64(_rand_bf16((6, 8), 1.0, 210))
    ref = _brute(h.tolist(), W.tolist(), W.tolist(), 0.8)
    good = stage.distribution_stats

    def dropped_term(z):
        r = good(z)
        r["H"] = r["lse"] - (r["p"] * z).sum(1) + 0.0 * r["max"] - r["max"] * 0.0 + 1e-3 * r["lse"]
        return r

    def wrong_base(z):
        r = good(z)
        r["H"] = r["H"] / math.log(2.0)
        return r

    def last_index(z):
        r = good(z)
        r["argmax"] = z.shape[1] - 1 - z[:, ::-1].argmax(1)
        return r

    for bad in (dropped_term, wrong_base):
        st = bad(stage.logits(h, W, 0.8))
        assert any(abs(st["H"][i] - ref[i][0]) > 1e-9 for i in range(len(ref)))
    zt = np.zeros((1, 8))
    assert last_index(zt)["argmax"][0] != 0


def test_chunked_forms_equal_direct():
    """The chunked helpers only change memory use: same values as the direct forms."""
    V, d = 1000, 24
    W = _rand_bf16((V, d), 0.3, 70)
    E = _rand_bf16((V, d), 0.3, 71)
    h = stage.bf16_to_f64(_rand_bf16((7, d), 1.0, 72))
    z = stage.logits(h, stage.bf16_to_f64(W), 0.6)
    for Win in (W, stage.bf16_to_f64(W)):
        zc = stage.logits_chunked(h, Win, 0.6, chunk=97)
        assert np.array_equal(zc, z)
    p = stage.distribution_stats(z)["p"]
    sc = stage.self_conditioning(p, stage.bf16_to_f64(E))
    assert np.allclose(stage.self_conditioning_chunked(p, E, chunk=97), sc, rtol=1e-13, atol=1e-16)
