"""GPU parity of the group entropy-bounded accept (accept_rule 1: the longest
entropy-ordered prefix of a canvas whose cumulative entropy is within the bound).

The accepted set is decided from float32 entropies on the GPU and from float64
ones in the oracle, so a canvas is compared only when its cut is unambiguous: the
cumulative sums on either side of the cut are at least 1e-4 from the bound and the
entropies of the last accepted and first rejected positions differ by at least
1e-5.  Kept tokens are compared where the argmax (or sample) itself is not a
near-tie.  At full size the rule is re-applied exactly to the GPU's own entropies.
"""

import numpy as np
import pytest
import torch

import gpu_case as gc
import synth
from oracle import philox, stage

pytestmark = pytest.mark.gpu

CUT = 1e-4
ORDER = 1e-5


@pytest.fixture(scope="module")
def dg():
    from discrete_diffusion_decoding_b200 import build
    build.build()
    import discrete_diffusion_decoding_b200 as m
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    return m


def _expect(H, kept, bound, seed, s, c, V):
    ren = philox.uniform_token(seed, np.arange(256), s, c, philox.TAG_RENOISE, V)
    return stage.group_accept(H, kept, bound, ren)


def _check_canvas(g, c, H_ref, kept, kept_ok, bound, seed, s, V, tag, cut=CUT, order=ORDER):
    """Compare canvas c's accept flags and tokens; False when the cut is ambiguous."""
    sl = slice(c * 256, (c + 1) * 256)
    tok, acc, cm, og = _expect(H_ref, kept, bound, seed, s, c, V)
    if cm < cut or og < order:
        return False
    assert np.array_equal(g["accept"][sl], acc), f"{tag}: accept set differs"
    ok = kept_ok | (acc == 0)
    assert np.array_equal(g["tokens"][sl][ok], tok[ok]), f"{tag}: tokens differ"
    return True


@pytest.mark.parametrize("bound,mode", [(0.1, 0), (2.0, 0), (2.0, 1)])
def test_group_step_small(dg, bound, mode):
    V, d, C, s = 4096, 128, 3, 4
    W = synth.weights(V, d)
    h, _ = synth.spiked_hidden(W, C * 256, seed=80, gain_lo=0.5, gain_hi=30.0)
    p = dg.params(C, V, d, eb_bound=bound, accept_rule=1, accept_mode=mode)
    seeds = synth.canvas_seeds(C, base=300)
    Wd = W.cuda()
    g = gc.gpu_step(dg, p, s, h, Wd, Wd, seeds)
    T = dg.temperature(p, s)
    hb, Wb = gc.bits(h), gc.bits(W)
    checked = 0
    for c in range(C):
        rows = np.arange(c * 256, (c + 1) * 256)
        o = stage.step_rows(hb[rows], Wb, Wb, T, bound, int(seeds[c]), s, c, np.arange(256), V,
                            want_selfcond=False, accept_mode=mode)
        assert np.abs(g["H"][rows] - o["H"]).max() <= gc.H_TOL
        if mode == 1:
            kept, kept_ok = o["sample"], (o["keygap"] >= gc.EXCL) & (o["cdf_margin"] >= 1e-4)
        else:
            kept, kept_ok = o["argmax"], o["top2gap"] >= gc.EXCL
        checked += _check_canvas(g, c, o["H"], kept, kept_ok, bound, int(seeds[c]), s, V, f"c={c}")
    assert checked >= 2
    assert 0 < g["accept"].sum() < C * 256
    # the group rule never accepts a position the per-position rule would reject
    assert np.all(g["H"][g["accept"] == 1] <= bound + 1e-6)


def test_group_step_full_vocab_rule_on_gpu_entropies(dg):
    """V = 262144, d = 2816, 2 canvases: the accepted sets are the rule applied to the GPU's own H."""
    V, d, C, s, bound = 262144, 2816, 2, 6, 0.5
    W = synth.weights(V, d)
    h, _ = synth.spiked_hidden(W, C * 256, seed=81, gain_lo=2.0, gain_hi=40.0)
    p = dg.params(C, V, d, eb_bound=bound, accept_rule=1)
    seeds = synth.canvas_seeds(C, base=310)
    Wd = W.cuda()
    g = gc.gpu_step(dg, p, s, h, Wd, Wd, seeds)
    checked = 0
    for c in range(C):
        sl = slice(c * 256, (c + 1) * 256)
        checked += _check_canvas(g, c, g["H"][sl], g["argmax"][sl], np.ones(256, bool), bound, int(seeds[c]),
                                 s, V, f"full c={c}", cut=1e-5, order=0.0)
    assert checked >= 1
    assert 0 < g["accept"].sum() < C * 256


def test_group_lockstep_decode_small(dg):
    """Stub-driven decode with the group rule: every step's accepted sets and tokens against the oracle."""
    V, d, C, S, gain = 4096, 128, 2, 12, 300.0
    W = synth.weights(V, d)
    Wb = gc.bits(W)
    p = dg.params(C, V, d, max_steps=S, eb_bound=0.5, accept_rule=1)
    ws, bufs = dg.Workspace(p), dg.StepBuffers(p)
    seeds = synth.canvas_seeds(C, base=40)
    seeds_t = torch.tensor(np.asarray(seeds, np.uint64).view(np.int64), device="cuda")
    Wd = W.cuda()
    dg.dg_canvas_init(p, seeds_t, bufs.tokens, ws)
    checked = accepted = 0
    stopped = [False] * C
    for s in range(1, S + 1):
        dg.dg_stub_hidden(p, s, gain, 0.1, seeds_t, Wd, bufs.tokens, bufs.h, ws)
        dg.dg_denoise_step(p, s, bufs.h, Wd, Wd, seeds_t, bufs.tokens, bufs.entropy, bufs.argmax, bufs.accept,
                           bufs.lse, bufs.selfcond, ws)
        flags, _, _ = dg.dg_stop_check(p, ws)
        g = {"H": bufs.entropy.cpu().numpy().astype(np.float64), "argmax": bufs.argmax.cpu().numpy(),
             "tokens": bufs.tokens.cpu().numpy().astype(np.int64), "accept": bufs.accept.cpu().numpy()}
        hb = gc.bits(bufs.h)
        T = dg.temperature(p, s)
        for c in range(C):
            if stopped[c]:
                continue
            rows = np.arange(c * 256, (c + 1) * 256)
            o = stage.step_rows(hb[rows], Wb, Wb, T, p.eb_bound, int(seeds[c]), s, c, np.arange(256), V,
                                want_selfcond=False)
            checked += _check_canvas(g, c, o["H"], o["argmax"], o["top2gap"] >= gc.EXCL, p.eb_bound, int(seeds[c]),
                                     s, V, f"s={s} c={c}")
            accepted += int(g["accept"][rows].sum())
            stopped[c] = bool(flags[c])
        if all(stopped):
            break
    assert checked >= 6 and accepted > 0


def test_sampled_group_lockstep_decode_small(dg):
    """Both options at once over a stub-driven decode: the group rule picks the accepted set, accepted
    positions keep the two-level sample; every step against the oracle (lock-step on the GPU's h)."""
    V, d, C, S, gain = 4096, 128, 2, 12, 300.0
    W = synth.weights(V, d)
    Wb = gc.bits(W)
    p = dg.params(C, V, d, max_steps=S, eb_bound=10.0, accept_rule=1, accept_mode=1)   # wide: spread rows kept
    ws, bufs = dg.Workspace(p), dg.StepBuffers(p)
    seeds = synth.canvas_seeds(C, base=60)
    seeds_t = torch.tensor(np.asarray(seeds, np.uint64).view(np.int64), device="cuda")
    Wd = W.cuda()
    dg.dg_canvas_init(p, seeds_t, bufs.tokens, ws)
    checked = differ = 0
    stopped = [False] * C
    for s in range(1, S + 1):
        dg.dg_stub_hidden(p, s, gain, 0.1, seeds_t, Wd, bufs.tokens, bufs.h, ws)
        dg.dg_denoise_step(p, s, bufs.h, Wd, Wd, seeds_t, bufs.tokens, bufs.entropy, bufs.argmax, bufs.accept,
                           bufs.lse, bufs.selfcond, ws)
        flags, _, _ = dg.dg_stop_check(p, ws)
        g = {"H": bufs.entropy.cpu().numpy().astype(np.float64), "argmax": bufs.argmax.cpu().numpy(),
             "tokens": bufs.tokens.cpu().numpy().astype(np.int64), "accept": bufs.accept.cpu().numpy()}
        hb = gc.bits(bufs.h)
        T = dg.temperature(p, s)
        for c in range(C):
            if stopped[c]:
                continue
            rows = np.arange(c * 256, (c + 1) * 256)
            o = stage.step_rows(hb[rows], Wb, Wb, T, p.eb_bound, int(seeds[c]), s, c, np.arange(256), V,
                                want_selfcond=False, accept_mode=1)
            ok_arg = o["top2gap"] >= gc.EXCL
            assert np.array_equal(g["argmax"][rows][ok_arg], o["argmax"][ok_arg]), f"argmax s={s} c={c}"
            kept_ok = (o["keygap"] >= gc.EXCL) & (o["cdf_margin"] >= 1e-4)
            if _check_canvas(g, c, o["H"], o["sample"], kept_ok, p.eb_bound, int(seeds[c]), s, V, f"s={s} c={c}"):
                checked += 1
                differ += int(np.sum((g["accept"][rows] == 1) & (o["sample"] != o["argmax"])))
            stopped[c] = bool(flags[c])
        if all(stopped):
            break
    assert checked >= 6 and differ >= 3
