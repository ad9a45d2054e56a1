"""Two independent decodes on two CUDA streams of one GPU at the same time.

The fused pass assumes the CTAs of a group can all be resident together; a second grid
launched on another stream may find most SMs taken, start part of its groups on the
free SMs and have them wait (boundedly) for their group-mates until the first grid
retires.  That must only delay it: both decodes, interleaved step by step on two streams
with separate workspaces, give the same bits as the same decodes run one after the
other, and no in-kernel wait runs out.
"""

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


def _decode(dg, p, W, seeds, ws, b, n_steps, stream):
    """n_steps of stub + denoise on `stream`; returns the step outputs (device clones)."""
    outs = []
    with torch.cuda.stream(stream):
        dg.dg_canvas_init(p, seeds, b.tokens, ws, stream)
        for s in range(1, n_steps + 1):
            dg.dg_stub_hidden(p, s, 4.0, 0.1, seeds, W, b.tokens, b.h, ws, stream)
            dg.dg_denoise_step(p, s, b.h, W, W, seeds, b.tokens, b.entropy, b.argmax, b.accept, b.lse, b.selfcond,
                               ws, stream)
            outs.append([t.clone() for t in (b.packed, b.lse, b.selfcond)])
    return outs


def test_two_streams_match_sequential(dg):
    V, d, n_steps = 262144, 2816, 6
    W = synth.weights(V, d, seed=1234).cuda()
    cfgs = [(1, [3]), (2, [4, 5])]
    runs = []
    for C, sd in cfgs:
        p = dg.params(C, V, d, max_steps=n_steps)
        runs.append((p, torch.tensor(sd, dtype=torch.int64, device="cuda"), dg.Workspace(p), dg.StepBuffers(p)))
    # one after the other on the default stream
    main = torch.cuda.current_stream()
    ref = [_decode(dg, p, W, seeds, ws, b, n_steps, main) for p, seeds, ws, b in runs]
    torch.cuda.synchronize()
    for p, _, ws, _ in runs:
        dg.dg_stop_check(p, ws)
    # both at once: the steps of the two decodes interleaved on two streams
    streams = [torch.cuda.Stream(), torch.cuda.Stream()]
    got = [[], []]
    for i, (p, seeds, ws, b) in enumerate(runs):
        with torch.cuda.stream(streams[i]):
            dg.dg_canvas_init(p, seeds, b.tokens, ws, streams[i])
    for s in range(1, n_steps + 1):
        for i, (p, seeds, ws, b) in enumerate(runs):
            with torch.cuda.stream(streams[i]):
                dg.dg_stub_hidden(p, s, 4.0, 0.1, seeds, W, b.tokens, b.h, ws, streams[i])
                dg.dg_denoise_step(p, s, b.h, W, W, seeds, b.tokens, b.entropy, b.argmax, b.accept, b.lse,
                                   b.selfcond, ws, streams[i])
                got[i].append([t.clone() for t in (b.packed, b.lse, b.selfcond)])
    torch.cuda.synchronize()
    for i, (p, _, ws, _) in enumerate(runs):
        dg.dg_stop_check(p, ws)                  # raises if a wait ran out
        for s in range(n_steps):
            for a, c in zip(ref[i][s], got[i][s]):
                assert torch.equal(a, c), f"decode {i} step {s + 1} differs when run concurrently"
