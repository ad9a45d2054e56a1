"""The device half of the timeout path, on the GPU, without a fault: the fused kernel's
waits on other CTAs' progress counters get a limit short enough that they run out
(dg_debug_set_counter_wait_limit), as they would behind a stalled peer CTA.

The kernel must leave on its own, and promptly: its drain waits for the loads it issued
to land (on the pair leader's barriers, with the rounds the two CTAs issued unevenly
settled by the leader) rather than for stage releases that an aborted pass never makes,
so no load or tensor-core operation is in flight when a CTA leaves and no drain wait runs
out its 2 s limit.  dg_stop_check must report
DG_ETIMEOUT, the step's results must be poisoned, and after dg_canvas_init the same
context must run a normal step that matches the oracle on every position.
"""

import math
import time

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


def test_counter_wait_runs_out_then_context_recovers(dg):
    from discrete_diffusion_decoding_b200 import _abi
    V, d, C, group = 8960, 512, 1, 2          # groups of 2 pairs: every block needs the row-maximum exchange
    W = synth.weights(V, d, seed=1234)
    h, _ = synth.spiked_hidden(W, C * 256, seed=31, gain_lo=0.5, gain_hi=30.0)
    p = dg.params(C, V, d, group=group)
    ws, b = dg.Workspace(p), dg.StepBuffers(p)
    seeds = synth.canvas_seeds(C, base=900)
    seeds_t = torch.tensor(seeds.view(np.int64), device="cuda")
    Wd = W.cuda()
    b.h.copy_(h.cuda())
    dg.dg_canvas_init(p, seeds_t, b.tokens, ws)
    torch.cuda.synchronize()
    try:
        dg.dg_debug_set_counter_wait_limit(1)          # 1 ns: a wait not satisfied at once runs out
        t0 = time.time()
        dg.dg_denoise_step(p, 1, b.h, Wd, Wd, seeds_t, b.tokens, b.entropy, b.argmax, b.accept, b.lse, b.selfcond,
                           ws)
        with pytest.raises(_abi.DgError) as e:
            dg.dg_stop_check(p, ws)
        elapsed = time.time() - t0
    finally:
        dg.dg_debug_set_counter_wait_limit(0)
    assert e.value.status == _abi.DG_ETIMEOUT
    # well under one 2 s drain limit: every drain wait ended on its loads, none ran out
    assert elapsed < 1.0, f"the kernel took {elapsed:.2f} s to leave"
    # the failed step's results are poisoned, and the canvas stays valid
    assert torch.isnan(b.entropy).all() and (b.argmax == -1).all() and int(b.accept.sum()) == 0
    tok = b.tokens.cpu().numpy()
    assert tok.min() >= 0 and tok.max() < V
    # the context is usable: a fresh canvas and a normal step match the oracle everywhere
    g = gc.gpu_step(dg, p, 1, h, Wd, Wd, seeds, ws=ws, bufs=b)
    assert list(g["stop"]) == [0]
    rows = np.arange(C * 256)
    o = gc.oracle_rows(gc.bits(h), gc.bits(W), gc.bits(W), dg.temperature(p, 1), p.eb_bound, seeds, 1, rows, V)
    gc.compare(g, o, rows, p.eb_bound, tag=f"after a timed-out step ({elapsed:.2f} s to leave)")
    assert math.isfinite(float(g["H"].max()))
