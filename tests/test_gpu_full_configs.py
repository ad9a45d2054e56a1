"""GPU parity on the full-size workloads (V = 262144, d = 2816), every row.

* single step, 1 canvas (both hidden recipes): every position against the oracle;
* 4 canvases of adversarial rows with untied W / E at both temperature endpoints:
  every position;
* one block of the block-autoregressive decode, lock-step: every position of every
  step against the oracle, and the stable counter and stop flag against the stop
  rule applied to the oracle's own full-canvas entropies and argmax; the oracle's
  free-running decode of the same block is run beside it and its stop step reported;
* the literal configurations (stub gain 1, nothing accepted, no stop): the block
  decode and 16 batched canvases over all 48 steps, every position at steps 1 and 48;
* 16 batched canvases with per-canvas stops (gain 10): every position of every
  active canvas at one step, the stop machinery at every step;
* the product's block-autoregressive loop (decode_block_ar) over 8 blocks, its first
  block equal to the lock-step run.

The oracle uses the GPU's canvas and hidden states at every step (lock-step), so
an excluded position cannot fork the trajectory; excluded counts are printed at
the end of the run.
"""

import math

import numpy as np
import pytest
import torch

import gpu_case as gc
import synth
from oracle import decode, stage

pytestmark = pytest.mark.gpu

V, D = 262144, 2816
STOP_AMBIG = 1e-3          # |mean H - stop threshold| below this leaves the stop flag unchecked


@pytest.fixture(scope="module")
def dg():
    from discrete_diffusion_decoding_b200 import build
    build.build()
    import discrete_diffusion_decoding_b200 as m
    assert torch.cuda.is_available()
    return m


@pytest.fixture(scope="module")
def head():
    """Tied head W = E: the bf16 tensor, its bits, the exact float64 widening and the device copy."""
    W = synth.weights(V, D, seed=1234)
    Wb = gc.bits(W)
    return {"W": W, "bits": Wb, "f64": stage.bf16_to_f64(Wb), "dev": W.cuda()}


@pytest.fixture(scope="module")
def untied_E():
    E = synth.weights(V, D, seed=1235)
    Eb = gc.bits(E)
    return {"E": E, "bits": Eb, "f64": stage.bf16_to_f64(Eb), "dev": E.cuda()}


def _all_rows(C):
    return np.arange(C * 256)


# ------------------------------------------------------------------ single step, one canvas
@pytest.mark.parametrize("hidden_kind,step", [("gaussian", 1), ("spiked", 48)])
def test_single_step_every_row(dg, head, hidden_kind, step):
    if hidden_kind == "gaussian":
        h = synth.gaussian_hidden(256, D, seed=42)
    else:
        h, _ = synth.spiked_hidden(head["W"], 256, seed=43, gain_lo=2.0, gain_hi=40.0)
    p = dg.params(1, V, D)
    seeds = synth.canvas_seeds(1)
    g = gc.gpu_step(dg, p, step, h, head["dev"], head["dev"], seeds)
    rows = _all_rows(1)
    o = gc.oracle_rows(gc.bits(h), head["f64"], head["f64"], dg.temperature(p, step), p.eb_bound, seeds, step,
                       rows, V)
    gc.compare(g, o, rows, p.eb_bound, tag=f"single step {hidden_kind} s={step}")
    assert np.all(g["H"] >= -1e-4) and np.all(g["H"] <= math.log(V) + 1e-3)
    if hidden_kind == "spiked":
        assert 0 < int(g["accept"].sum()) < 256


# ------------------------------------------------------------------ adversarial rows, untied
def _near_bound_row(Wf, Wb, k, base, T, target=0.1, tol=1e-4):
    """h = g W_k/||W_k||^2 + base with H(bf16(h)) close to target: a bisection on g whose search
    evaluates the entropy from float32 logits (input construction only; the float64 oracle decides
    the row's exclusion afterwards)."""
    Wk = stage.bf16_to_f64(Wb[k])
    lo, hi = 0.0, 60.0

    def H_of(g):
        hb = stage.f64_to_bf16(g * Wk / (Wk @ Wk) + base)
        hf = torch.from_numpy(stage.bf16_to_f64(hb).astype(np.float32))
        z = (Wf @ hf).double().numpy()[None, :] / T
        return stage.distribution_stats(z)["H"][0], hb

    for _ in range(40):
        mid = 0.5 * (lo + hi)
        Hm, hb = H_of(mid)
        if abs(Hm - target) < tol:
            return hb, Hm
        if Hm > target:
            lo = mid
        else:
            hi = mid
    return hb, Hm


@pytest.mark.parametrize("step", [1, 48])
def test_adversarial_rows_untied_every_row(dg, head, untied_E, step):
    """4 canvases (N = 1024): near-uniform, one-hot spikes, exact-tie and near-bound rows; E != W."""
    W, Wb = head["W"], head["bits"]
    C = 4
    p = dg.params(C, V, D, tied=0)
    T = dg.temperature(p, step)
    h, kind = synth.adversarial_rows(W, C * 256, seed=44)
    hb = gc.bits(h).copy()
    kind = kind.numpy()
    # replace a few kind-3 rows by rows whose entropy sits within 1e-4 of the bound
    rng = np.random.default_rng(5)
    near = np.nonzero(kind == 3)[0][:6]
    Wf = W.float()
    for i in near:
        base = rng.standard_normal(D) * 1e-3
        hb[i], _ = _near_bound_row(Wf, Wb, int(rng.integers(0, V)), base, T)
    del Wf
    h = torch.from_numpy(hb.view(np.int16)).view(torch.bfloat16)
    seeds = synth.canvas_seeds(C, base=300)
    g = gc.gpu_step(dg, p, step, h, head["dev"], untied_E["dev"], seeds)
    rows = _all_rows(C)
    o = gc.oracle_rows(hb, head["f64"], untied_E["f64"], T, p.eb_bound, seeds, step, rows, V)
    excl, _, _ = gc.compare(g, o, rows, p.eb_bound, tag=f"adversarial untied s={step}")
    # the exclusion machinery sees the constructed near-bound cases
    assert len([r for r in near if r in set(excl)]) >= len(near) - 1
    # exact closed forms on the h = 0 rows: all logits tie, H = ln V, argmax = 0
    zero_rows = [i for i in np.nonzero(kind == 0)[0] if (i // 4) % 2 == 0]
    assert np.abs(g["H"][zero_rows] - math.log(V)).max() < 1e-3
    assert np.all(g["argmax"][zero_rows] == 0)
    # one-hot spikes: H ~ 0 at every spike position
    assert np.all(g["H"][kind == 1] < 1e-3)


# ------------------------------------------------------------------ lock-step decodes
def _gpu_outputs(b):
    return {"H": b.entropy.cpu().numpy().astype(np.float64), "argmax": b.argmax.cpu().numpy().astype(np.int64),
            "tokens": b.tokens.cpu().numpy().astype(np.int64), "accept": b.accept.cpu().numpy(),
            "lse": b.lse.cpu().numpy().astype(np.float64),
            "selfcond": b.selfcond.cpu().numpy().astype(np.float64)}


def _excluded(o, bound):
    return (np.abs(o["H"] - bound) < gc.EXCL) | (o["top2gap"] < gc.EXCL)


def test_block_decode_lockstep_every_row_and_oracle_stop(dg, head):
    """One 256-token block (seed 0, stub gain 10, 48-step schedule): every position of every step
    against the oracle; stable counter and stop flag against the rule on the oracle's entropies."""
    Wb, W64, Wd = head["bits"], head["f64"], head["dev"]
    gain, noise = 10.0, 0.1
    p = dg.params(1, V, D)
    S = p.max_steps
    ws, b = dg.Workspace(p), dg.StepBuffers(p)
    seeds = synth.canvas_seeds(1)
    seeds_t = torch.tensor(seeds.view(np.int64), device="cuda")
    dg.dg_canvas_init(p, seeds_t, b.tokens, ws)
    assert np.array_equal(b.tokens.cpu().numpy(), stage.init_tokens(0, 0, V))
    stable_o, prev_o, prev_diff = 0, None, np.zeros(256, bool)
    stop_gpu = stop_checked = 0
    rows = _all_rows(1)
    for s in range(1, S + 1):
        tok_in = b.tokens.cpu().numpy().copy()
        dg.dg_stub_hidden(p, s, gain, noise, seeds_t, Wd, b.tokens, b.h, ws)
        hb = gc.bits(b.h)
        want_h, _ = stage.stub_hidden(Wb, tok_in, 0, s, 0, S, gain, noise)
        d = np.abs(stage.bf16_to_f64(hb) - stage.bf16_to_f64(want_h))
        assert (d == 0).mean() > 0.99 and d.max() < 1e-2, f"stub s={s}"
        dg.dg_denoise_step(p, s, b.h, Wd, Wd, seeds_t, b.tokens, b.entropy, b.argmax, b.accept, b.lse, b.selfcond,
                           ws)
        flags, st_gpu, _ = dg.dg_stop_check(p, ws, want_stable=True)
        g = _gpu_outputs(b)
        want_sc = s in (1, 2, 24) or flags[0]
        o = gc.oracle_rows(hb, W64, W64, dg.temperature(p, s), p.eb_bound, seeds, s, rows, V,
                           want_selfcond=want_sc)
        gc.compare(g, o, rows, p.eb_bound, check_selfcond=want_sc, tag=f"block decode s={s}")
        # the stop rule on the oracle's own full-canvas entropies and argmax vectors
        excl = _excluded(o, p.eb_bound)
        mean_H = float(o["H"].mean())
        stable_o, stop_o = stage.stop_update(mean_H, o["argmax"], prev_o, stable_o, s, p.stop_thresh, p.stability)
        # an excluded position whose argmax differs between the two sides (at this step or the
        # previous one) enters the stability comparison ambiguously: take the GPU's counter there
        # (lock-step) and check again once no such position is left in the comparison
        diff = excl & (g["argmax"] != o["argmax"])
        ambiguous = bool(np.any(diff) or np.any(prev_diff))
        if ambiguous:
            stable_o = int(st_gpu[0])
        else:
            assert st_gpu[0] == stable_o, f"stable counter s={s}: gpu {st_gpu[0]} oracle {stable_o}"
        if not ambiguous and abs(mean_H - p.stop_thresh) >= STOP_AMBIG:
            assert bool(flags[0]) == stop_o, f"stop flag s={s} (oracle mean H {mean_H:.4g})"
            stop_checked += 1
        prev_o, prev_diff = o["argmax"].copy(), diff
        if flags[0]:
            stop_gpu = s
            break
    assert stop_checked >= 10
    committed = b.argmax.cpu().numpy().copy()
    # the oracle's own free-running decode of the same block (its stub, its canvas)
    free = decode.decode_batch(Wb, Wb, seeds, decode.stub_hidden_fn(Wb, seeds, S, gain, noise), V, max_steps=S,
                               bound=p.eb_bound, stop_thresh=p.stop_thresh, stability=p.stability)
    stop_free = int(free["stop_step"][0])
    agree = float(np.mean(free["committed"][0] == committed))
    gc.report("block decode stop step", 256, 0,
              f"gpu lock-step {stop_gpu or S}, oracle free-running {stop_free}, committed agreement {agree:.3f}")
    assert stop_gpu and stop_gpu < S, "the block should stop before the step cap at gain 10"
    # the product's block-autoregressive loop reproduces this block exactly (same seed, deterministic kernels)
    out, steps = dg.decode_block_ar(dg.params(1, V, D), Wd, Wd, 8, seed0=0, gain=gain, noise=noise)
    assert steps[0] == stop_gpu
    assert np.array_equal(out[:256].cpu().numpy(), committed)
    assert out.shape == (8 * 256,) and int(out.min()) >= 0 and int(out.max()) < V
    assert all(3 <= st <= S for st in steps) and any(st < S for st in steps[1:])
    gc.report("decode_block_ar 8 blocks", 8 * 256, 0, f"stop steps {steps}")


def _literal_decode(dg, head, C, base_seed, check_steps):
    """The literal stub (gain 1, noise 0.1) over all 48 steps; every position at check_steps."""
    W64, Wd = head["f64"], head["dev"]
    p = dg.params(C, V, D)
    S = p.max_steps
    ws, b = dg.Workspace(p), dg.StepBuffers(p)
    seeds = synth.canvas_seeds(C, base=base_seed)
    seeds_t = torch.tensor(seeds.view(np.int64), device="cuda")
    dg.dg_canvas_init(p, seeds_t, b.tokens, ws)
    rows = _all_rows(C)
    for s in range(1, S + 1):
        dg.dg_stub_hidden(p, s, 1.0, 0.1, seeds_t, Wd, b.tokens, b.h, ws)
        dg.dg_denoise_step(p, s, b.h, Wd, Wd, seeds_t, b.tokens, b.entropy, b.argmax, b.accept, b.lse, b.selfcond,
                           ws)
        flags, st, n = dg.dg_stop_check(p, ws, want_stable=True)
        assert n == 0, f"a literal-gain canvas stopped at s={s}"
        if s in check_steps:
            g = _gpu_outputs(b)
            o = gc.oracle_rows(gc.bits(b.h), W64, W64, dg.temperature(p, s), p.eb_bound, seeds, s, rows, V)
            gc.compare(g, o, rows, p.eb_bound, tag=f"literal C={C} s={s}")
            # nothing is accepted and no canvas is near the stop threshold (oracle's mean H per canvas)
            assert int(g["accept"].sum()) == 0 and int(o["accept"].sum()) == 0
            assert o["H"].reshape(C, 256).mean(axis=1).min() > 10.0
            assert list(flags) == [0] * C


def test_literal_block_decode_48_steps(dg, head):
    _literal_decode(dg, head, 1, 0, (1, 48))


def test_literal_batched_16_canvases_48_steps(dg, head):
    _literal_decode(dg, head, 16, 100, (1, 48))


def test_batched_canvases_per_canvas_stop(dg, head):
    """16 canvases in one launch (N = 4096), gain 10: every position of every active canvas at one
    step against the oracle (its mean H and stop flag per canvas too); the stop machinery at every
    step; stopped canvases are frozen."""
    Wd, W64 = head["dev"], head["f64"]
    C, gain = 16, 10.0
    p = dg.params(C, V, D)
    ws, b = dg.Workspace(p), dg.StepBuffers(p)
    seeds = synth.canvas_seeds(C, base=100)
    seeds_t = torch.tensor(seeds.view(np.int64), device="cuda")
    dg.dg_canvas_init(p, seeds_t, b.tokens, ws)
    stopped = np.zeros(C, bool)
    stop_at = [p.max_steps] * C
    checked = False
    for s in range(1, p.max_steps + 1):
        tok_in = b.tokens.cpu().numpy().copy()
        am_in = b.argmax.cpu().numpy().copy()
        dg.dg_stub_hidden(p, s, gain, 0.1, seeds_t, Wd, b.tokens, b.h, ws)
        dg.dg_denoise_step(p, s, b.h, Wd, Wd, seeds_t, b.tokens, b.entropy, b.argmax, b.accept, b.lse, b.selfcond,
                           ws)
        flags, st_gpu, _ = dg.dg_stop_check(p, ws, want_stable=True)
        tok = b.tokens.cpu().numpy()
        am = b.argmax.cpu().numpy()
        for c in np.nonzero(stopped)[0]:
            sl = slice(c * 256, (c + 1) * 256)
            assert np.array_equal(tok[sl], tok_in[sl]) and np.array_equal(am[sl], am_in[sl])
        if not checked and s >= 30:
            act = np.nonzero(~stopped)[0]
            rows = np.concatenate([np.arange(c * 256, (c + 1) * 256) for c in act])
            g = _gpu_outputs(b)
            o = gc.oracle_rows(gc.bits(b.h), W64, W64, dg.temperature(p, s), p.eb_bound, seeds, s, rows, V)
            gc.compare(g, o, rows, p.eb_bound, tag=f"batched gain 10 s={s} ({len(act)} active)")
            mean_H = o["H"].reshape(len(act), 256).mean(axis=1)
            for k, c in enumerate(act):
                if flags[c] and abs(mean_H[k] - p.stop_thresh) >= STOP_AMBIG:
                    assert mean_H[k] < p.stop_thresh, f"canvas {c} stopped with oracle mean H {mean_H[k]:.4g}"
            checked = True
        for c in range(C):
            if flags[c] and not stopped[c]:
                stopped[c] = True
                stop_at[c] = s
        if stopped.all():
            break
    assert checked
    assert any(st < p.max_steps for st in stop_at) and all(st >= 3 for st in stop_at)
    gc.report("batched 16 canvases stop steps", C * 256, 0, f"{stop_at}")
