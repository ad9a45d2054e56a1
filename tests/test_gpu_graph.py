"""The step is capturable in a CUDA graph: after the first (set-up) call on the device,
dg_stub_hidden + dg_denoise_step launch kernels only (no allocation, no synchronisation), so
a whole decode of S steps can be captured once and replayed.  Stopped canvases are skipped
inside the kernels, so a captured decode needs no host decision between steps.  Replays
give the same bits as the same calls run eagerly."""

import numpy as np
import pytest
import torch

import synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dg():
    from discrete_diffusion_decoding_b200 import build
    build.build()
    import discrete_diffusion_decoding_b200 as m
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    return m


def _decode(dg, p, Wd, seeds_t, ws, b, S, gain, stream):
    for s in range(1, S + 1):
        dg.dg_stub_hidden(p, s, gain, 0.1, seeds_t, Wd, b.tokens, b.h, ws, stream)
        dg.dg_denoise_step(p, s, b.h, Wd, Wd, seeds_t, b.tokens, b.entropy, b.argmax, b.accept, b.lse, b.selfcond,
                           ws, stream)


@pytest.mark.parametrize("V,d,C,S,gain", [(4096, 128, 3, 16, 300.0), (8960, 512, 2, 8, 8.0)])
def test_captured_decode_replays_eager_bits(dg, V, d, C, S, gain):
    W = synth.weights(V, d)
    Wd = W.cuda()
    p = dg.params(C, V, d, max_steps=S)
    seeds_t = torch.tensor(synth.canvas_seeds(C, base=33).view(np.int64), device="cuda")
    # eager reference
    ws_e, b_e = dg.Workspace(p), dg.StepBuffers(p)
    dg.dg_canvas_init(p, seeds_t, b_e.tokens, ws_e)
    _decode(dg, p, Wd, seeds_t, ws_e, b_e, S, gain, torch.cuda.current_stream())
    flags_e, stable_e, _ = dg.dg_stop_check(p, ws_e, want_stable=True)
    # captured: canvas init eagerly, the S steps as one graph, replayed twice from a fresh canvas
    ws, b = dg.Workspace(p), dg.StepBuffers(p)
    side = torch.cuda.Stream()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(side):
        dg.dg_canvas_init(p, seeds_t, b.tokens, ws, side)
        side.synchronize()
        with torch.cuda.graph(g, stream=side):
            _decode(dg, p, Wd, seeds_t, ws, b, S, gain, side)
    for _ in range(2):
        dg.dg_canvas_init(p, seeds_t, b.tokens, ws)
        g.replay()
        torch.cuda.synchronize()
        flags, stable, _ = dg.dg_stop_check(p, ws, want_stable=True)
        assert flags == flags_e and stable == stable_e
        for k in ("tokens", "entropy", "argmax", "accept", "lse", "selfcond", "h"):
            assert torch.equal(getattr(b, k), getattr(b_e, k)), k
    if gain > 100:
        assert any(flags), "some canvas should stop inside the captured decode"
    del g
