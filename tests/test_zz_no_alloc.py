"""The allocation-free entry point (dg_denoise_stats_noalloc) against the regular one.

Some callers cannot allocate device memory when they call the library - a plugin
running inside a framework whose allocator it may not use, a process with a
memory budget fixed up front, or a latency-critical thread that must stay off
the allocator.  For them the library keeps the fused pass's scratch in a fixed
array in device memory.  This test checks, through the C ABI, that two calls in
a row of that entry point give the same entropies, argmax, log-sum-exp and
self-conditioning vectors as dg_denoise_step with a caller workspace (within the
tolerances the parity tests use), that no device memory is allocated by those
calls, and that a shape too large for the fixed scratch is refused.

This file is collected last on purpose, so that a run that stops at the first
failure has already run every other test.
"""

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


def _regular(dg, p, step, h, W, E):
    ws = dg.Workspace(p)
    b = dg.StepBuffers(p)
    seeds = torch.zeros(p.n_canvas, dtype=torch.int64, device="cuda")
    dg.dg_canvas_init(p, seeds, b.tokens, ws)
    b.h.copy_(h)
    dg.dg_denoise_step(p, step, b.h, W, E, seeds, b.tokens, b.entropy, b.argmax, b.accept, b.lse, b.selfcond, ws)
    dg.dg_stop_check(p, ws)
    return b.entropy.clone(), b.argmax.clone(), b.lse.clone(), b.selfcond.clone()


@pytest.mark.parametrize("tied", [True, False])
def test_noalloc_matches_workspace_path_on_two_calls(dg, tied):
    V, d, C = 32768, 2816, 2
    W = synth.weights(V, d).cuda()
    E = W if tied else synth.weights(V, d, seed=1235).cuda()
    h, _ = synth.spiked_hidden(W.cpu(), C * 256, seed=77, gain_lo=1.0, gain_hi=40.0)
    h = h.cuda()
    p = dg.params(C, V, d, tied=int(tied))
    N = C * 256
    H = torch.empty(N, dtype=torch.float32, device="cuda")
    am = torch.empty(N, dtype=torch.int32, device="cuda")
    lse = torch.empty(N, dtype=torch.float32, device="cuda")
    sc = torch.empty((N, d), dtype=torch.float32, device="cuda")
    for call, step in enumerate((1, 48)):
        want = _regular(dg, p, step, h, W, E)
        torch.cuda.synchronize()
        free_before = torch.cuda.mem_get_info()[0]
        H.fill_(float("nan"))
        am.fill_(-7)
        sc.fill_(float("nan"))
        dg.dg_denoise_stats_noalloc(p, step, h, W, E, H, am, lse, sc)
        assert dg.last_launch_count() == 3            # clear, fused pass, combine
        torch.cuda.synchronize()
        if call > 0:
            # the first call on a device is its set-up (the runtime may load the
            # library's device code, which holds the fixed scratch); later calls
            # must leave free device memory exactly as it was
            assert torch.cuda.mem_get_info()[0] == free_before, "the allocation-free call changed free device memory"
        assert torch.isfinite(H).all() and torch.isfinite(sc).all()
        assert (H - want[0]).abs().max().item() <= 1e-3
        assert torch.equal(am, want[1])
        assert (lse - want[2]).abs().max().item() <= 1e-3 * max(1.0, want[2].abs().max().item())
        rel = ((sc - want[3]).norm(dim=1) / want[3].norm(dim=1).clamp_min(1e-30)).max().item()
        assert rel <= 2e-2


def test_noalloc_refuses_shapes_beyond_its_scratch(dg):
    from discrete_diffusion_decoding_b200 import _abi
    V, d = 262144, 2816
    # the documented limit: up to 4 canvases of this head fit the 64 MiB scratch, 5 do not
    assert dg.workspace_size(dg.params(4, V, d)) <= 64 << 20 < dg.workspace_size(dg.params(5, V, d))
    x = torch.empty(16, dtype=torch.float32, device="cuda")
    with pytest.raises(_abi.DgError) as e:
        dg.dg_denoise_stats_noalloc(dg.params(5, V, d), 1, x, x, x, x, x, None, None)
    assert e.value.status == _abi.DG_ENOMEM
    assert dg.last_launch_count() == 0
    p = dg.params(64, V, d)                    # needs far more than the fixed scratch
    x = torch.empty(16, dtype=torch.float32, device="cuda")
    with pytest.raises(_abi.DgError) as e:
        dg.dg_denoise_stats_noalloc(p, 1, x, x, x, x, x, None, None)
    assert e.value.status == _abi.DG_ENOMEM
