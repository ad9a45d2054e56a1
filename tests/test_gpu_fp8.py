"""GPU parity of the E4M3 logits option (logits_format 1): the head as 8-bit E4M3 codes with
one power-of-two scale, the hidden states quantised per position at every step, the logits
GEMM on tcgen05 kind::f8f6f4, the self-conditioning GEMM on the bf16 embedding.

The quantisers are compared with oracle/fp8.py bit for bit; the step with the oracle fed
the same quantised values (decoded exactly), every position, under the usual tolerances.
"""

import math

import numpy as np
import pytest
import torch

import gpu_case as gc
import synth
from oracle import fp8, stage

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dg():
    from discrete_diffusion_decoding_b200 import build
    build.build()
    import discrete_diffusion_decoding_b200 as m
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    return m


def _bf16(x64):
    b = stage.f64_to_bf16(x64)
    return torch.from_numpy(b.view(np.int16)).view(torch.bfloat16)


def test_quantisers_bitexact(dg):
    rng = np.random.default_rng(7)
    rows, cols = 300, 512
    x = rng.standard_normal((rows, cols)) * np.exp2(rng.integers(-30, 30, (rows, 1)))
    x[5] = 0.0                                           # an all-zero row
    x[6, :] = 2.0 ** -130                                # bf16 subnormals
    x[7, ::3] *= 2.0 ** -12                              # values that fall to E4M3 subnormals
    xb = _bf16(x)
    x64 = stage.bf16_to_f64(synth.bf16_bits(xb))
    codes = torch.empty((rows, cols), dtype=torch.uint8, device="cuda")
    exps = torch.empty(rows, dtype=torch.int32, device="cuda")
    dg.dg_quantize_e4m3(xb.cuda(), codes, exps, 1)
    want_c, want_e = fp8.quantize_rows(x64)
    assert np.array_equal(exps.cpu().numpy(), want_e)
    assert np.array_equal(codes.cpu().numpy(), want_c)
    tc, te = dg.quantize_head_e4m3(xb.cuda())
    want_tc, want_te = fp8.quantize_tensor(x64)
    assert te == want_te and np.array_equal(tc.cpu().numpy(), want_tc)


def _fp8_head(dg, W):
    """Quantise the head on the GPU, check it against the oracle, and build the bf16 embedding
    of the tied head from the decoded codes (exact in bf16)."""
    codes, e = dg.quantize_head_e4m3(W.cuda())
    want_c, want_e = fp8.quantize_tensor(stage.bf16_to_f64(gc.bits(W)))
    assert e == want_e and np.array_equal(codes.cpu().numpy(), want_c)
    W64 = fp8.dequantize_tensor(want_c, want_e)
    E = _bf16(W64)
    assert np.array_equal(stage.bf16_to_f64(gc.bits(E)), W64)        # decoded codes are exact in bf16
    return codes, e, W64, E


def _oracle_fp8(h, W64, E, p, seeds, step, rows, V, accept_mode=0, want_selfcond=True):
    hq, eh = fp8.quantize_rows(stage.bf16_to_f64(gc.bits(h)))
    h_deq = stage.f64_to_bf16(fp8.dequantize_rows(hq, eh))
    return gc.oracle_rows(h_deq, W64, gc.bits(E), dg_temperature(p, step), p.eb_bound, seeds, step, rows, V,
                          accept_mode=accept_mode, want_selfcond=want_selfcond)


def dg_temperature(p, step):
    import discrete_diffusion_decoding_b200 as m
    return m.temperature(p, step)


@pytest.mark.parametrize("V,d,C,group,mode,rule,bound", [(8960, 512, 2, 2, 0, 0, 0.1), (4096, 1024, 3, 4, 0, 0, 0.1),
                                                         (4096, 256, 2, 0, 1, 0, 6.0), (4096, 256, 2, 0, 0, 1, 2.0)])
def test_fp8_step_every_row(dg, V, d, C, group, mode, rule, bound):
    W = synth.weights(V, d, seed=1234)
    codes, e, W64, E = _fp8_head(dg, W)
    h, _ = synth.spiked_hidden(W, C * 256, seed=60 + d, gain_lo=0.5, gain_hi=30.0)
    p = dg.params(C, V, d, group=group, logits_format=1, w_scale_exp=e, accept_mode=mode, accept_rule=rule,
                  eb_bound=bound, tied=0)
    seeds = synth.canvas_seeds(C, base=700)
    g = gc.gpu_step(dg, p, 4, h, codes, E.cuda(), seeds)
    rows = np.arange(C * 256)
    o = _oracle_fp8(h, W64, E, p, seeds, 4, rows, V, accept_mode=mode, want_selfcond=(rule == 0))
    if rule == 0:
        excl, dH, dsc = gc.compare(g, o, rows, bound, tag=f"fp8 V={V} d={d} G={group} mode={mode}")
    else:
        assert np.abs(g["H"] - o["H"]).max() <= gc.H_TOL
        ok = o["top2gap"] >= gc.EXCL
        assert np.array_equal(g["argmax"][ok], o["argmax"][ok])
        gc.report(f"fp8 group rule V={V}", C * 256, int((~ok).sum()))
    assert 0 < int(g["accept"].sum()) < C * 256


def test_fp8_full_vocab_every_row(dg):
    V, d, C = 262144, 2816, 1
    W = synth.weights(V, d, seed=1234)
    codes, e, W64, E = _fp8_head(dg, W)
    h, _ = synth.spiked_hidden(W, 256, seed=43, gain_lo=2.0, gain_hi=40.0)
    p = dg.params(C, V, d, logits_format=1, w_scale_exp=e, tied=0)
    seeds = synth.canvas_seeds(C)
    g = gc.gpu_step(dg, p, 12, h, codes, E.cuda(), seeds)
    rows = np.arange(256)
    o = _oracle_fp8(h, W64, E, p, seeds, 12, rows, V)
    gc.compare(g, o, rows, p.eb_bound, tag="fp8 full vocab V=262144 d=2816")
    assert np.all(g["H"] <= math.log(V) + 1e-3) and 0 < int(g["accept"].sum()) < 256


def test_fp8_unsupported_shapes_and_paths(dg):
    from discrete_diffusion_decoding_b200 import _abi
    with pytest.raises(_abi.DgError) as e:
        dg.plan(dg.params(1, 4096, 128, logits_format=1))          # 256 E4M3 values per pipeline stage
    assert e.value.status == _abi.DG_EUNSUPPORTED
    with pytest.raises(_abi.DgError) as e:
        dg.plan(dg.params(1, 4096, 256, logits_format=2))
    assert e.value.status == _abi.DG_EINVAL
    p = dg.params(1, 4096, 256, logits_format=1)
    x = torch.zeros(16, dtype=torch.float32, device="cuda")
    with pytest.raises(_abi.DgError) as e:
        dg.dg_denoise_stats_noalloc(p, 1, x, x, x, x, x, None, None)
    assert e.value.status == _abi.DG_EUNSUPPORTED
    with pytest.raises(_abi.DgError) as e:
        dg.dg_quantize_e4m3(torch.zeros((4, 3), dtype=torch.bfloat16, device="cuda"),
                            torch.zeros((4, 3), dtype=torch.uint8, device="cuda"),
                            torch.zeros(4, dtype=torch.int32, device="cuda"), 1)            # odd column count
    assert e.value.status == _abi.DG_EINVAL


def test_fp8_vocabulary_split_matches_single_call(dg):
    """Two E4M3 shards (the head quantised once, its codes split by rows) merged equal the single
    E4M3 call: the same logits, so the same argmax, accept flags and tokens."""
    V, d, C = 4096, 512, 2
    W = synth.weights(V, d, seed=1234)
    codes, e, W64, E = _fp8_head(dg, W)
    Ed = E.cuda()
    h, _ = synth.spiked_hidden(W, C * 256, seed=66, gain_lo=0.5, gain_hi=30.0)
    p = dg.params(C, V, d, logits_format=1, w_scale_exp=e, tied=0)
    seeds = synth.canvas_seeds(C, base=710)
    single = gc.gpu_step(dg, p, 3, h, codes, Ed, seeds)
    ws, b = dg.Workspace(p), dg.StepBuffers(p)
    seeds_t = torch.tensor(seeds.view(np.int64), device="cuda")
    dg.dg_canvas_init(p, seeds_t, b.tokens, ws)
    b.h.copy_(h.cuda())
    nb = dg.dg_partial_bytes(p)
    parts = torch.empty(2 * nb, dtype=torch.uint8, device="cuda")
    for k, (v0, v1) in enumerate([(0, 1536), (1536, 4096)]):
        dg.dg_denoise_partial(p, 3, v0, v1 - v0, b.h, codes[v0:v1], Ed[v0:v1], seeds_t, parts[k * nb:(k + 1) * nb], ws)
    dg.dg_denoise_merge(p, 3, 2, parts, seeds_t, b.tokens, b.entropy, b.argmax, b.accept, b.lse, b.selfcond, ws)
    dg.dg_stop_check(p, ws)
    assert np.array_equal(b.argmax.cpu().numpy(), single["argmax"])
    assert np.abs(b.entropy.cpu().numpy() - single["H"]).max() <= 1e-4
    near = np.abs(single["H"] - p.eb_bound) < 1e-4
    assert np.array_equal(b.accept.cpu().numpy()[~near], single["accept"][~near])
    assert np.array_equal(b.tokens.cpu().numpy()[~near], single["tokens"][~near])
    gc.report("fp8 vocabulary split 2 shards", C * 256, int(near.sum()))
