"""GPU tests of the tile-major head layout (dg_params.head_layout 1, dg_tile_head).

The layout only changes where the fused kernel's operand tiles come from: every
result must be bit-identical to the row-major run on the same inputs, at small
sizes spanning several tiles and a ragged vocabulary tail, with a separate
embedding, in the sampled acceptance mode, through the vocabulary split, the
allocation-free entry point and a whole decode.  At the full size the tiled run
is also checked against the oracle on sampled rows.
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


def _by_permute(W):
    """The tile-major order written with a reshape: [V/128, 128, d/64, 64] -> [V/128, d/64, 128, 64]."""
    V, d = W.shape
    return W.view(V // 128, 128, d // 64, 64).permute(0, 2, 1, 3).contiguous().view(V, d)


@pytest.mark.parametrize("V,d", [(1024, 128), (4096, 384), (262144, 2816)])
def test_tile_head_matches_reshape_and_round_trips(dg, V, d):
    W = synth.weights(V, d, seed=5).cuda()
    Wt = dg.tile_head(W)
    assert dg.last_launch_count() == 1
    assert torch.equal(Wt, _by_permute(W))
    back = torch.empty_like(W)
    dg.dg_tile_head(Wt, back, 1)
    torch.cuda.synchronize()
    assert torch.equal(back, W)


def test_tile_head_rejects_bad_shapes(dg):
    from discrete_diffusion_decoding_b200 import _abi
    W = torch.zeros(384, 128, dtype=torch.bfloat16, device="cuda")
    for bad in (W[:200], torch.zeros(256, 96, dtype=torch.bfloat16, device="cuda")):
        with pytest.raises(_abi.DgError) as e:
            dg.dg_tile_head(bad, torch.empty_like(bad), 0)
        assert e.value.status == _abi.DG_EINVAL
    with pytest.raises(_abi.DgError) as e:      # in place is not allowed
        dg.dg_tile_head(W, W, 0)
    assert e.value.status == _abi.DG_EINVAL


def test_fp8_with_tiled_head_is_unsupported(dg):
    from discrete_diffusion_decoding_b200 import _abi
    p = dg.params(1, 4096, 512, logits_format=1, head_layout=1)
    with pytest.raises(_abi.DgError) as e:
        dg.plan(p)
    assert e.value.status == _abi.DG_EUNSUPPORTED
    with pytest.raises(_abi.DgError):
        dg.plan(dg.params(1, 4096, 512, head_layout=2))


def _run_steps(dg, p, W, E, seeds_t, n_steps, gain=1.0, noise=0.2):
    """n_steps of stub + denoise; returns every step's outputs (host tensors)."""
    ws, b = dg.Workspace(p), dg.StepBuffers(p)
    dg.dg_canvas_init(p, seeds_t, b.tokens, ws)
    out = []
    for s in range(1, n_steps + 1):
        dg.dg_stub_hidden(p, s, gain, noise, seeds_t, E, b.tokens, b.h, ws)
        h = b.h.clone()
        dg.dg_denoise_step(p, s, b.h, W, E, seeds_t, b.tokens, b.entropy, b.argmax, b.accept, b.lse, b.selfcond,
                           ws)
        flags, stable, _ = dg.dg_stop_check(p, ws, want_stable=True)
        out.append({"h": h.cpu(), "H": b.entropy.cpu(), "argmax": b.argmax.cpu(), "accept": b.accept.cpu(),
                    "tokens": b.tokens.cpu(), "lse": b.lse.cpu(), "selfcond": b.selfcond.cpu(),
                    "stop": list(flags), "stable": list(stable)})
    return out


def _assert_identical(a, b, tag):
    for s, (x, y) in enumerate(zip(a, b), start=1):
        for k in x:
            if isinstance(x[k], torch.Tensor):
                assert torch.equal(x[k], y[k]), f"{tag}: step {s} {k} differs"
            else:
                assert x[k] == y[k], f"{tag}: step {s} {k} differs"


@pytest.mark.parametrize("C,V,d,tied,mode,rule", [
    (2, 4096 + 768, 512, True, 0, 0),      # ragged last group of vocabulary tiles
    (3, 8192, 768, False, 1, 0),           # separate embedding, sampled acceptance
    (1, 2048 + 256, 384, True, 0, 1),      # group acceptance, odd number of 128-column atoms
])
def test_tiled_equals_row_major(dg, C, V, d, tied, mode, rule):
    W = synth.weights(V, d, seed=11).cuda()
    E = W if tied else synth.weights(V, d, seed=12).cuda()
    seeds_t = torch.arange(100, 100 + C, dtype=torch.int64, device="cuda")
    kw = dict(max_steps=6, accept_mode=mode, accept_rule=rule)
    ref = _run_steps(dg, dg.params(C, V, d, **kw), W, E, seeds_t, 4)
    Wt = dg.tile_head(W)
    Et = Wt if tied else dg.tile_head(E)
    got = _run_steps(dg, dg.params(C, V, d, head_layout=1, **kw), Wt, Et, seeds_t, 4)
    _assert_identical(ref, got, f"C={C} V={V} d={d}")


def test_tiled_full_size_matches_row_major_and_oracle(dg):
    """One step at the full vocabulary and width: bits equal the row-major run; sampled rows
    agree with the oracle under the usual tolerances."""
    V, d, C = 262144, 2816, 2
    W = synth.weights(V, d, seed=1234)
    h = synth.gaussian_hidden(256 * C, d, seed=42)
    seeds = np.array([7, 8], np.uint64)
    Wd = W.cuda()
    ref = gc.gpu_step(dg, dg.params(C, V, d), 1, h, Wd, Wd, seeds)
    Wt = dg.tile_head(Wd)
    del Wd
    got = gc.gpu_step(dg, dg.params(C, V, d, head_layout=1), 1, h, Wt, Wt, seeds)
    for k in ("H", "argmax", "tokens", "accept", "lse", "selfcond", "stop", "stable"):
        assert np.array_equal(ref[k], got[k]), k
    rows = np.array([0, 1, 127, 128, 255, 256, 300, 511])
    p = dg.params(C, V, d)
    ora = gc.oracle_rows(gc.bits(h), gc.bits(W), gc.bits(W), dg.temperature(p, 1), p.eb_bound, seeds, 1, rows, V)
    gc.compare(got, ora, rows, p.eb_bound, tag="tiled full size")


def test_tiled_vocab_split_equals_row_major(dg):
    """Shards of a tiled head are the same sub-arrays as row-major shards (rows v0..v1)."""
    V, d, C = 8192, 512, 2
    W = synth.weights(V, d, seed=21).cuda()
    Wt = dg.tile_head(W)
    seeds_t = torch.tensor([3, 4], dtype=torch.int64, device="cuda")
    h = synth.gaussian_hidden(256 * C, d, seed=22).cuda()
    bounds = [(0, 2560), (2560, 5888), (5888, 8192)]
    outs = []
    for lay, Wl in ((0, W), (1, Wt)):
        p = dg.params(C, V, d, head_layout=lay)
        ws, b = dg.Workspace(p), dg.StepBuffers(p)
        dg.dg_canvas_init(p, seeds_t, b.tokens, ws)
        b.h.copy_(h)
        nb = dg.dg_partial_bytes(p)
        parts = torch.empty(len(bounds) * nb, dtype=torch.uint8, device="cuda")
        for k, (v0, v1) in enumerate(bounds):
            dg.dg_denoise_partial(p, 1, v0, v1 - v0, b.h, Wl[v0:v1], Wl[v0:v1], seeds_t, parts[k * nb:(k + 1) * nb],
                                  ws)
        dg.dg_denoise_merge(p, 1, len(bounds), parts, seeds_t, b.tokens, b.entropy, b.argmax, b.accept, b.lse,
                            b.selfcond, ws)
        torch.cuda.synchronize()
        outs.append([t.cpu() for t in (b.entropy, b.argmax, b.accept, b.tokens, b.lse, b.selfcond, parts)])
    for x, y in zip(*outs):
        assert torch.equal(x, y)


def test_tiled_no_alloc_equals_row_major(dg):
    V, d, C = 4096, 512, 1
    W = synth.weights(V, d, seed=31).cuda()
    Wt = dg.tile_head(W)
    h = synth.gaussian_hidden(256 * C, d, seed=32).cuda().to(torch.bfloat16)
    outs = []
    for lay, Wl in ((0, W), (1, Wt)):
        p = dg.params(C, V, d, head_layout=lay)
        H = torch.empty(256 * C, device="cuda")
        am = torch.empty(256 * C, dtype=torch.int32, device="cuda")
        lse = torch.empty(256 * C, device="cuda")
        sc = torch.empty(256 * C, d, device="cuda")
        dg.dg_denoise_stats_noalloc(p, 1, h, Wl, Wl, H, am, lse, sc)
        torch.cuda.synchronize()
        outs.append([t.cpu() for t in (H, am, lse, sc)])
    for x, y in zip(*outs):
        assert torch.equal(x, y)


def test_tiled_decode_equals_row_major(dg):
    V, d, C = 4096, 256, 2
    W = synth.weights(V, d, seed=41).cuda()
    seeds_t = torch.tensor([9, 10], dtype=torch.int64, device="cuda")
    p0 = dg.params(C, V, d, max_steps=16)
    p1 = dg.params(C, V, d, max_steps=16, head_layout=1)
    c0, s0 = dg.decode_batch(p0, W, W, seeds_t, gain=3.0, noise=0.05)
    Wt = dg.tile_head(W)
    c1, s1 = dg.decode_batch(p1, Wt, Wt, seeds_t, gain=3.0, noise=0.05)
    assert torch.equal(c0, c1) and s0 == s1
