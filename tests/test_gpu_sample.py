"""GPU parity of the sampled acceptance mode (accept_mode 1: an accepted position
keeps a Gumbel-max draw from softmax(z / T) instead of the argmax).

The kept tokens are compared with the oracle's sample (bit-exact except where the
two best keys differ by less than 1e-3); H, argmax, LSE and the self-conditioning
vectors must equal those of the argmax mode exactly (the same arithmetic runs in
both kernels).  Bounds above the default 0.1 make accepted positions with spread
distributions, where the sample often differs from the argmax.
"""

import numpy as np
import pytest
import torch

import gpu_case as gc
import synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dg():
    from discrete_diffusion_decoding_b200 import build
    build.build()
    import discrete_diffusion_decoding_b200 as m
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    return m


def _both_modes(dg, C, V, d, group, bound, step, h, Wd, seeds):
    p1 = dg.params(C, V, d, group=group, eb_bound=bound, accept_mode=1)
    p0 = dg.params(C, V, d, group=group, eb_bound=bound, accept_mode=0)
    g1 = gc.gpu_step(dg, p1, step, h, Wd, Wd, seeds)
    g0 = gc.gpu_step(dg, p0, step, h, Wd, Wd, seeds)
    for k in ("H", "argmax", "lse", "accept"):
        assert np.array_equal(g0[k], g1[k]), f"{k} differs between the acceptance modes"
    assert np.array_equal(g0["selfcond"], g1["selfcond"])
    rej = g0["accept"] == 0
    assert np.array_equal(g0["tokens"][rej], g1["tokens"][rej])      # the same re-noise draws
    return p1, g1


@pytest.mark.parametrize("V,d,C,group,bound", [(4096, 128, 1, 0, 6.0), (8960, 512, 2, 2, 6.0),
                                               (4096, 1024, 3, 8, 6.0), (4096, 128, 2, 0, 0.1)])
def test_sampled_step_full_rows(dg, V, d, C, group, bound):
    W = synth.weights(V, d, seed=1234)
    h, _ = synth.spiked_hidden(W, C * 256, seed=70 + group, gain_lo=0.5, gain_hi=20.0)
    seeds = synth.canvas_seeds(C, base=200)
    Wd = W.cuda()
    p, g = _both_modes(dg, C, V, d, group, bound, 2, h, Wd, seeds)
    rows = np.arange(C * 256)
    o = gc.oracle_rows(gc.bits(h), gc.bits(W), gc.bits(W), dg.temperature(p, 2), bound, seeds, 2, rows, V,
                       accept_mode=1)
    excl, _, _ = gc.compare(g, o, rows, bound, tag=f"sample V={V} G={group}")
    assert len(excl) < C * 256 // 8
    acc = o["accept"] == 1
    assert 0 < acc.sum() < C * 256
    if bound > 1.0:
        # the mode is exercised: accepted positions keep a sample that is not the argmax
        assert np.sum(acc & (o["sample"] != o["argmax"])) >= 5


def test_sampled_step_full_vocab(dg):
    """V = 262144, d = 2816: sampled rows against the oracle's per-row Gumbel-max over the whole vocabulary."""
    V, d, C = 262144, 2816, 1
    W = synth.weights(V, d, seed=1234)
    h, _ = synth.spiked_hidden(W, 256, seed=71, gain_lo=2.0, gain_hi=40.0)
    seeds = synth.canvas_seeds(C, base=5)
    Wd = W.cuda()
    bound = 12.0                      # admits near-uniform rows (ln V = 12.48), where a sample differs
    p, g = _both_modes(dg, C, V, d, 0, bound, 9, h, Wd, seeds)
    rng = np.random.default_rng(21)
    rows = np.unique(np.concatenate([[0, 255], rng.choice(256, 30, replace=False)]))
    o = gc.oracle_rows(gc.bits(h), gc.bits(W), gc.bits(W), dg.temperature(p, 9), bound, seeds, 9, rows, V,
                       accept_mode=1, want_selfcond=False)
    gc.compare(g, o, rows, bound, check_selfcond=False, tag="sample full vocab")
    acc = o["accept"] == 1
    assert acc.sum() >= 5 and np.sum(acc & (o["sample"] != o["argmax"])) >= 2
