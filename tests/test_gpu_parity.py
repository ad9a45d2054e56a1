"""GPU parity: the CUDA path (through the C ABI) against the float64 oracle.

Every test here runs the library's sm_100a kernels on a B200 and compares with
the oracle on the same seeded inputs (see gpu_case.py for the tolerances).
"""

import ctypes
import math

import numpy as np
import pytest
import torch

import gpu_case as gc
import synth
from oracle import decode, philox, stage

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dg():
    from discrete_diffusion_decoding_b200 import build
    build.build()
    import discrete_diffusion_decoding_b200 as m
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    return m


def _assert_stub_close(got_bits, want_bits, gain):
    # one bf16 ulp of the result, plus the fp32 rounding of the sum's operands (which may cancel)
    a_got = stage.bf16_to_f64(got_bits)
    a_want = stage.bf16_to_f64(want_bits)
    ulp = 2.0 ** (np.floor(np.log2(np.maximum(np.abs(a_want), 2.0 ** -120))) - 7)
    err = np.abs(a_got - a_want)
    assert np.all(err <= ulp + 1e-6 * max(1.0, gain)), f"stub error {err.max():.3e}"
    assert (err == 0).mean() > 0.99


def _rows_all(n):
    return np.arange(n)


# ------------------------------------------------------------------ element-wise kernels
def test_canvas_init_bitexact(dg):
    V = 262144
    C = 256                                    # 4 calls x 65536 = 262144 Philox draws
    p = dg.params(C, V, 128)
    ws = dg.Workspace(p)
    tok = torch.empty(C * 256, dtype=torch.int32, device="cuda")
    for call in range(4):
        seeds = (np.arange(C, dtype=np.uint64) + np.uint64(C * call)) * np.uint64(0x9E3779B97F4A7C15) + np.uint64(7)
        dg.dg_canvas_init(p, torch.tensor(seeds.view(np.int64), device="cuda"), tok, ws)
        got = tok.cpu().numpy()
        want = np.concatenate([stage.init_tokens(int(seeds[c]), c, V) for c in range(C)])
        assert np.array_equal(got, want)


@pytest.mark.parametrize("V,d,C,gain,noise,step,S", [(4096, 128, 2, 300.0, 0.1, 5, 16),
                                                      (262144, 2816, 1, 8.0, 0.1, 48, 48)])
def test_stub_hidden_within_one_ulp(dg, V, d, C, gain, noise, step, S):
    W = synth.weights(V, d)
    Wb = gc.bits(W)
    p = dg.params(C, V, d, max_steps=S)
    seeds = synth.canvas_seeds(C, base=11)
    rng = np.random.default_rng(3)
    toks = rng.integers(0, V, size=C * 256).astype(np.int32)
    ws = dg.Workspace(p)
    Wd = W.cuda()
    seeds_t = torch.tensor(seeds.view(np.int64), device="cuda")
    tok_t = torch.tensor(toks, device="cuda")
    dg.dg_canvas_init(p, seeds_t, torch.empty_like(tok_t), ws)
    h = torch.empty((C * 256, d), dtype=torch.bfloat16, device="cuda")
    dg.dg_stub_hidden(p, step, gain, noise, seeds_t, Wd, tok_t, h, ws)
    got = gc.bits(h)
    for c in range(C):
        want, _ = stage.stub_hidden(Wb, toks[c * 256:(c + 1) * 256], int(seeds[c]), step, c, S, gain, noise)
        _assert_stub_close(got[c * 256:(c + 1) * 256], want, gain)


# ------------------------------------------------------------------ one step, small shapes
@pytest.mark.parametrize("kind", ["gaussian", "spiked"])
def test_step_small_tied(dg, kind):
    V, d, C = 4096, 128, 1
    W = synth.weights(V, d)
    h = synth.gaussian_hidden(C * 256, d, seed=42) if kind == "gaussian" else synth.spiked_hidden(W, C * 256, gain_lo=0.5, gain_hi=20.0)[0]
    p = dg.params(C, V, d)
    seeds = synth.canvas_seeds(C)
    Wd = W.cuda()
    g = gc.gpu_step(dg, p, 1, h, Wd, Wd, seeds)
    T = dg.temperature(p, 1)
    o = gc.oracle_rows(gc.bits(h), gc.bits(W), gc.bits(W), T, p.eb_bound, seeds, 1, _rows_all(C * 256), V)
    excl, dh, dsc = gc.compare(g, o, _rows_all(C * 256), p.eb_bound, tag=kind)
    assert len(excl) < 32
    if kind == "spiked":
        assert 0 < int(g["accept"].sum()) < C * 256           # both branches of the sampler taken


@pytest.mark.parametrize("group,tied,C,V,d", [(2, True, 2, 8960, 512), (4, False, 2, 8960, 512),
                                              (8, True, 3, 4096, 1024), (1, True, 2, 65536, 256)])
def test_step_groups_and_segments(dg, group, tied, C, V, d):
    """Multi-pair groups (P exchange, shared reference), multi-block pieces, ragged blocks."""
    W = synth.weights(V, d, seed=1234)
    E = W if tied else synth.weights(V, d, seed=1235)
    h, _ = synth.spiked_hidden(W, C * 256, seed=50 + group, gain_lo=0.5, gain_hi=30.0)
    p = dg.params(C, V, d, group=group, tied=int(tied))
    seeds = synth.canvas_seeds(C, base=100)
    Wd = W.cuda()
    Ed = Wd if tied else E.cuda()
    g = gc.gpu_step(dg, p, 3, h, Wd, Ed, seeds)
    T = dg.temperature(p, 3)
    o = gc.oracle_rows(gc.bits(h), gc.bits(W), gc.bits(E), T, p.eb_bound, seeds, 3, _rows_all(C * 256), V)
    gc.compare(g, o, _rows_all(C * 256), p.eb_bound, tag=f"G={group}")


@pytest.mark.parametrize("C,mode", [(1, 0), (5, 0), (5, 1)])
def test_smallest_shape(dg, C, mode):
    """The smallest accepted head (V = 256: one vocabulary tile; d = 128: one 128-column stage and
    slice) with one and several canvases, argmax and sampled acceptance, on every row."""
    V, d = 256, 128
    W = synth.weights(V, d, seed=81)
    h, _ = synth.spiked_hidden(W, C * 256, seed=82, gain_lo=0.5, gain_hi=60.0)
    p = dg.params(C, V, d, accept_mode=mode, eb_bound=4.0 if mode else 0.1)
    assert dg.plan(p)["group"] == 1
    seeds = synth.canvas_seeds(C, base=400)
    Wd = W.cuda()
    g = gc.gpu_step(dg, p, 1, h, Wd, Wd, seeds)
    o = gc.oracle_rows(gc.bits(h), gc.bits(W), gc.bits(W), dg.temperature(p, 1), p.eb_bound, seeds, 1,
                       _rows_all(C * 256), V, accept_mode=mode)
    excl, _, _ = gc.compare(g, o, _rows_all(C * 256), p.eb_bound, tag=f"V=256 d=128 C={C} mode={mode}")
    assert len(excl) < C * 256 // 4
    assert int(g["accept"].sum()) > 0


def _widest_hidden(dg, V):
    """The widest hidden size whose group (one pair per 256 columns) still fits on the device at once."""
    from discrete_diffusion_decoding_b200 import _abi
    for k in range(96, 0, -1):
        try:
            pl = dg.plan(dg.params(1, V, 256 * k))
        except _abi.DgError as e:
            assert e.status == _abi.DG_EUNSUPPORTED
            continue
        return 256 * k, pl
    raise AssertionError("no hidden size fits")


@pytest.mark.parametrize("which", ["d5376", "widest"])
def test_wide_hidden_groups(dg, which):
    """Wide hidden sizes: 21-pair groups (d = 5376, three groups), and the widest group the device holds
    at once (one group of every resident pair, a single ragged vocabulary block), on every row."""
    from discrete_diffusion_decoding_b200 import _abi
    if which == "d5376":
        V, d = 16384, 5376
        pl = dg.plan(dg.params(1, V, d))
        assert pl["group"] == 21 and pl["slice"] == 256
    else:
        V = 4096
        d, pl = _widest_hidden(dg, V)
        assert pl["n_groups"] == 1 and pl["group"] == d // 256 >= 64
        with pytest.raises(_abi.DgError) as e:                  # one more pair than fits
            dg.plan(dg.params(1, V, d + 256))
        assert e.value.status == _abi.DG_EUNSUPPORTED
    W = synth.weights(V, d, seed=71)
    h, _ = synth.spiked_hidden(W, 256, seed=72, gain_lo=0.5, gain_hi=30.0)
    p = dg.params(1, V, d)
    seeds = synth.canvas_seeds(1, base=300)
    Wd = W.cuda()
    g = gc.gpu_step(dg, p, 2, h, Wd, Wd, seeds)
    o = gc.oracle_rows(gc.bits(h), gc.bits(W), gc.bits(W), dg.temperature(p, 2), p.eb_bound, seeds, 2,
                       _rows_all(256), V)
    gc.compare(g, o, _rows_all(256), p.eb_bound, tag=f"d={d} G={pl['group']} groups={pl['n_groups']}")


def test_large_logits_rescale(dg):
    """Rows whose running maximum jumps late in the vocabulary force the lazy rescale of O."""
    V, d, C = 131072, 512, 1          # G = 2: 256 blocks per tile, several blocks per segment
    W = synth.weights(V, d, seed=9)
    Wf = W.to(torch.float64)
    h = torch.zeros((256, d), dtype=torch.float64)
    g = torch.Generator().manual_seed(5)
    for i in range(256):
        k = int(torch.randint(0, V, (1,), generator=g))       # the spike's block is usually not a segment's first
        h[i] = Wf[k] * ((10.0 + 0.3 * (i % 90)) / float(Wf[k] @ Wf[k]))
    h = h.to(torch.float32).to(torch.bfloat16)
    p = dg.params(C, V, d, group=2)
    seeds = synth.canvas_seeds(C)
    Wd = W.cuda()
    out = gc.gpu_step(dg, p, 1, h, Wd, Wd, seeds)
    o = gc.oracle_rows(gc.bits(h), gc.bits(W), gc.bits(W), dg.temperature(p, 1), p.eb_bound, seeds, 1,
                       _rows_all(256), V)
    gc.compare(out, o, _rows_all(256), p.eb_bound, tag="rescale")


def test_uniform_logits_closed_form(dg):
    """h = 0: every logit ties, H = ln V, argmax = 0, self-conditioning = column mean of E."""
    V, d, C = 8192, 512, 1
    W = synth.weights(V, d)
    p = dg.params(C, V, d)
    h = torch.zeros((256, d), dtype=torch.bfloat16)
    Wd = W.cuda()
    g = gc.gpu_step(dg, p, 1, h, Wd, Wd, synth.canvas_seeds(1))
    assert np.abs(g["H"] - math.log(V)).max() < 1e-4
    assert np.all(g["argmax"] == 0)
    mean = stage.bf16_to_f64(gc.bits(W)).mean(axis=0)
    rel = np.linalg.norm(g["selfcond"] - mean[None, :], axis=1) / np.linalg.norm(mean)
    assert rel.max() < 1e-3


# ------------------------------------------------------------------ multi-step, lock-step
def _lockstep(dg, V, d, C, S, gain, noise, seeds, W, sample=None, expect_stop=True):
    p = dg.params(C, V, d, max_steps=S)
    Wb = gc.bits(W)
    Wd = W.cuda()
    ws = dg.Workspace(p)
    bufs = dg.StepBuffers(p)
    seeds_t = torch.tensor(np.asarray(seeds, np.uint64).view(np.int64), device="cuda")
    dg.dg_canvas_init(p, seeds_t, bufs.tokens, ws)
    init = bufs.tokens.cpu().numpy()
    for c in range(C):
        assert np.array_equal(init[c * 256:(c + 1) * 256], stage.init_tokens(int(seeds[c]), c, V))
    prev = [None] * C
    stable = [0] * C
    stopped = [False] * C
    stop_at = [S] * C
    for s in range(1, S + 1):
        tok_in = bufs.tokens.cpu().numpy().copy()
        dg.dg_stub_hidden(p, s, gain, noise, seeds_t, Wd, bufs.tokens, bufs.h, ws)
        dg.dg_denoise_step(p, s, bufs.h, Wd, Wd, seeds_t, bufs.tokens, bufs.entropy, bufs.argmax, bufs.accept,
                           bufs.lse, bufs.selfcond, ws)
        flags, st_gpu, _ = dg.dg_stop_check(p, ws, want_stable=True)
        hb = gc.bits(bufs.h)
        g = {"H": bufs.entropy.cpu().numpy().astype(np.float64), "argmax": bufs.argmax.cpu().numpy().astype(np.int64),
             "tokens": bufs.tokens.cpu().numpy().astype(np.int64), "accept": bufs.accept.cpu().numpy(),
             "lse": bufs.lse.cpu().numpy().astype(np.float64), "selfcond": bufs.selfcond.cpu().numpy()}
        T = dg.temperature(p, s)
        for c in range(C):
            if stopped[c]:
                continue
            rows_c = np.arange(c * 256, (c + 1) * 256)
            # the stub is an input of the stage: check it, then hand its bytes to the oracle
            want_h, _ = stage.stub_hidden(Wb, tok_in[rows_c], int(seeds[c]), s, c, S, gain, noise)
            _assert_stub_close(hb[rows_c], want_h, gain)
            rows = rows_c if sample is None else rows_c[sample]
            o = gc.oracle_rows(hb, Wb, Wb, T, p.eb_bound, seeds, s, rows, V)
            excl, _, _ = gc.compare(g, o, rows, p.eb_bound, tag=f"s={s} c={c}")
            if sample is None:
                full = stage.distribution_stats(stage.logits_chunked(stage.bf16_to_f64(hb[rows_c]), Wb, T))
                mean_H = full["H"].mean()
                stable[c], stop = stage.stop_update(mean_H, g["argmax"][rows_c], prev[c], stable[c], s)
                prev[c] = g["argmax"][rows_c].copy()
                if not excl and abs(mean_H - p.stop_thresh) >= 1e-3:
                    assert st_gpu[c] == stable[c], f"stable counter s={s} c={c}"
                    assert bool(flags[c]) == stop, f"stop flag s={s} c={c}"
            if flags[c]:
                stopped[c] = True
                stop_at[c] = s
        if all(stopped):
            break
    if expect_stop:
        assert min(stop_at) < S, "no canvas stopped early: the stop path was not exercised"
    for c in range(C):
        if stop_at[c] < S:
            assert stop_at[c] >= 3
    return stop_at


def test_lockstep_decode_small(dg):
    W = synth.weights(4096, 128)
    stop_at = _lockstep(dg, 4096, 128, 1, 16, 300.0, 0.1, synth.canvas_seeds(1), W)
    assert stop_at[0] <= 16


def test_lockstep_batched_per_canvas_stop(dg):
    W = synth.weights(4096, 128)
    stop_at = _lockstep(dg, 4096, 128, 4, 16, 300.0, 0.1, synth.canvas_seeds(4, base=20), W)
    assert len(set(stop_at)) >= 1


def test_lockstep_literal_gain_never_accepts(dg):
    """The literal small configuration (gain 1, 16-step schedule, all 16 steps): entropies stay near
    ln V, nothing is accepted, no stop; every position of every step against the oracle."""
    W = synth.weights(4096, 128)
    stop_at = _lockstep(dg, 4096, 128, 1, 16, 1.0, 0.1, synth.canvas_seeds(1), W, expect_stop=False)
    assert stop_at == [16]


# ------------------------------------------------------------------ the product's decode loops
def _record_steps(dg):
    rec = {}

    def on_step(s, bufs):
        rec[s] = {"h": gc.bits(bufs.h).copy(), "tokens": bufs.tokens.cpu().numpy().astype(np.int64),
                  "argmax": bufs.argmax.cpu().numpy().astype(np.int64)}
    return rec, on_step


def _oracle_replay(Wb, seeds, V, S, rec, canvas_ids, C):
    """oracle.decode.decode_batch fed, at every step, the hidden states the GPU's stub produced for
    that step (lock-step) - after checking that the oracle's canvas equals the one the GPU stub read."""
    def hidden(tok, s, c):
        want_in = rec[s - 1]["tokens"][c * 256:(c + 1) * 256] if s > 1 else tok
        assert np.array_equal(tok, want_in), f"canvas {c} diverged before step {s}"
        return rec[s]["h"][c * 256:(c + 1) * 256]
    return decode.decode_batch(Wb, Wb, seeds, hidden, V, max_steps=S, record=True)


def test_product_decode_batch_matches_oracle(dg):
    """dg.decode_batch itself (stub inside, dg_stop_check every step, committed = the argmax of each
    canvas's last step) against oracle.decode.decode_batch in lock-step on the GPU stub's h."""
    V, d, C, S = 4096, 128, 3, 16
    W = synth.weights(V, d)
    Wb, Wd = gc.bits(W), W.cuda()
    p = dg.params(C, V, d, max_steps=S)
    seeds = synth.canvas_seeds(C, base=30)
    seeds_t = torch.tensor(seeds.view(np.int64), device="cuda")
    rec, on_step = _record_steps(dg)
    committed, stop_step = dg.decode_batch(p, Wd, Wd, seeds_t, gain=300.0, noise=0.1, on_step=on_step)
    ora = _oracle_replay(Wb, seeds, V, S, rec, None, C)
    assert list(ora["stop_step"]) == list(stop_step)
    assert min(stop_step) < S
    assert np.array_equal(committed.cpu().numpy(), ora["committed"])
    gc.report("decode_batch product loop", C * 256, 0, f"stop steps {stop_step}")


def test_product_decode_block_ar_matches_oracle(dg):
    """dg.decode_block_ar: 3 blocks one after another (seeds 7, 8, 9), each against the oracle's decode."""
    V, d, S, n_blocks = 4096, 128, 16, 3
    W = synth.weights(V, d)
    Wb, Wd = gc.bits(W), W.cuda()
    p1 = dg.params(1, V, d, max_steps=S)
    recs = {}

    def on_step(b, s, bufs):
        recs.setdefault(b, {})[s] = {"h": gc.bits(bufs.h).copy(),
                                     "tokens": bufs.tokens.cpu().numpy().astype(np.int64)}
    out, steps = dg.decode_block_ar(p1, Wd, Wd, n_blocks, seed0=7, gain=300.0, noise=0.1, on_step=on_step)
    out = out.cpu().numpy()
    for b in range(n_blocks):
        ora = _oracle_replay(Wb, np.array([7 + b], np.uint64), V, S, recs[b], None, 1)
        assert int(ora["stop_step"][0]) == steps[b]
        assert np.array_equal(out[b * 256:(b + 1) * 256], ora["committed"][0])
    gc.report("decode_block_ar product loop", n_blocks * 256, 0, f"stop steps {steps}")


# ------------------------------------------------------------------ argument checks
def test_argument_errors(dg):
    from discrete_diffusion_decoding_b200 import _abi
    p = dg.params(1, 4096, 128)
    ws = dg.Workspace(p)
    bufs = dg.StepBuffers(p)
    W = synth.weights(4096, 128).cuda()
    seeds = torch.zeros(1, dtype=torch.int64, device="cuda")
    with pytest.raises(_abi.DgError) as e:
        dg.dg_denoise_step(p, 0, bufs.h, W, W, seeds, bufs.tokens, bufs.entropy, bufs.argmax, bufs.accept, None,
                           None, ws)
    assert e.value.status == _abi.DG_EINVAL
    with pytest.raises(_abi.DgError) as e:
        dg.dg_denoise_step(p, 49, bufs.h, W, W, seeds, bufs.tokens, bufs.entropy, bufs.argmax, bufs.accept, None,
                           None, ws)
    assert e.value.status == _abi.DG_EINVAL
    with pytest.raises(_abi.DgError) as e:
        dg.dg_denoise_step(p, 1, None, W, W, seeds, bufs.tokens, bufs.entropy, bufs.argmax, bufs.accept, None, None,
                           ws)
    assert e.value.status == _abi.DG_EINVAL
    small = dg.Workspace(p)
    small.nbytes = 64
    with pytest.raises(_abi.DgError) as e:
        dg.dg_denoise_step(p, 1, bufs.h, W, W, seeds, bufs.tokens, bufs.entropy, bufs.argmax, bufs.accept, None,
                           None, small)
    assert e.value.status == _abi.DG_ENOMEM
    # every limit the header states for dg_params, with the status it names
    einval = [dict(n_canvas=0), dict(n_canvas=257), dict(canvas_len=128), dict(vocab=4000), dict(vocab=0),
              dict(hidden=100), dict(hidden=64), dict(hidden=192), dict(max_steps=0), dict(t_start=0.0),
              dict(t_end=-0.4), dict(stability=-1), dict(accept_mode=2), dict(accept_rule=-1)]
    for bad in einval:
        q = dg.params(1, 4096, 128)
        for k, v in bad.items():
            setattr(q, k, v)
        with pytest.raises(_abi.DgError) as e:
            dg.plan(q)
        assert e.value.status == _abi.DG_EINVAL, bad
        with pytest.raises(_abi.DgError):
            dg.workspace_size(q)
    eunsup = [(512, 3),        # the group does not divide hidden
              (384, 2),        # slice 192: not a multiple of 128
              (1280, 2),       # slice 640: wider than 256
              (128 * 75, 75)]  # 75 pairs of CTAs: more than a B200 holds at once
    for hidden, group in eunsup:
        with pytest.raises(_abi.DgError) as e:
            dg.plan(dg.params(1, 4096, hidden, group=group))
        assert e.value.status == _abi.DG_EUNSUPPORTED, (hidden, group)
    assert dg.plan(dg.params(256, 256, 128))["slice"] == 128       # the smallest accepted shape
    # the vocabulary split's arguments
    part = torch.empty(dg.dg_partial_bytes(p), dtype=torch.uint8, device="cuda")
    for vb, vc in [(128, 256), (0, 0), (0, 300), (3840, 512), (-256, 512)]:
        with pytest.raises(_abi.DgError) as e:
            dg.dg_denoise_partial(p, 1, vb, vc, bufs.h, W, W, seeds, part, ws)
        assert e.value.status == _abi.DG_EINVAL, (vb, vc)
    for n_parts in (0, 65):
        with pytest.raises(_abi.DgError) as e:
            dg.dg_denoise_merge(p, 1, n_parts, part, seeds, bufs.tokens, bufs.entropy, bufs.argmax, bufs.accept,
                                None, None, ws)
        assert e.value.status == _abi.DG_EINVAL
    assert dg.last_launch_count() == 0


def test_forced_error_word_reported_and_cleared(dg):
    """Host-side fault injection: a device error word (as a timed-out wait leaves it) makes the next
    dg_stop_check return DG_ETIMEOUT; dg_canvas_init clears it; steps in between still run."""
    from discrete_diffusion_decoding_b200 import _abi
    V, d = 4096, 128
    p = dg.params(1, V, d)
    ws, bufs = dg.Workspace(p), dg.StepBuffers(p)
    W = synth.weights(V, d).cuda()
    seeds = torch.zeros(1, dtype=torch.int64, device="cuda")
    dg.dg_canvas_init(p, seeds, bufs.tokens, ws)
    bufs.h.copy_(synth.gaussian_hidden(256, d).cuda())
    assert dg.dg_stop_check(p, ws)[2] == 0
    dg.dg_debug_set_error(p, ws, 301)
    dg.dg_denoise_step(p, 1, bufs.h, W, W, seeds, bufs.tokens, bufs.entropy, bufs.argmax, bufs.accept, bufs.lse,
                       bufs.selfcond, ws)
    with pytest.raises(_abi.DgError) as e:
        dg.dg_stop_check(p, ws)
    assert e.value.status == _abi.DG_ETIMEOUT
    # the step's results are poisoned, not plausible: NaN entropy / LSE / self-conditioning,
    # argmax -1, nothing accepted, every position re-noised (tokens stay in range)
    assert torch.isnan(bufs.entropy).all() and torch.isnan(bufs.lse).all() and torch.isnan(bufs.selfcond).all()
    assert (bufs.argmax == -1).all() and int(bufs.accept.sum()) == 0
    want = stage.renoise_tokens(0, 1, 0, V)
    assert np.array_equal(bufs.tokens.cpu().numpy(), want)
    with pytest.raises(_abi.DgError) as e:                 # the word stays set until the canvas is re-initialised
        dg.dg_stop_check(p, ws)
    assert e.value.status == _abi.DG_ETIMEOUT
    dg.dg_canvas_init(p, seeds, bufs.tokens, ws)
    dg.dg_denoise_step(p, 1, bufs.h, W, W, seeds, bufs.tokens, bufs.entropy, bufs.argmax, bufs.accept, None, None, ws)
    flags, _, n = dg.dg_stop_check(p, ws)
    assert flags == [0] and n == 0
    small = dg.Workspace(p)
    small.nbytes = 64
    with pytest.raises(_abi.DgError) as e:
        dg.dg_debug_set_error(p, small, 1)
    assert e.value.status == _abi.DG_ENOMEM


def test_last_sm_clock_telemetry(dg):
    """dg_last_sm_clock: 0 after dg_canvas_init, then the clock of the last fused pass, a value
    between the lowest and highest SM clocks a B200 runs at; argument errors are reported."""
    from discrete_diffusion_decoding_b200 import _abi
    V, d = 65536, 512
    p = dg.params(1, V, d)
    ws, bufs = dg.Workspace(p), dg.StepBuffers(p)
    W = synth.weights(V, d).cuda()
    seeds = torch.zeros(1, dtype=torch.int64, device="cuda")
    dg.dg_canvas_init(p, seeds, bufs.tokens, ws)
    assert dg.dg_last_sm_clock(p, ws) == 0.0
    bufs.h.copy_(synth.gaussian_hidden(256, d).cuda())
    dg.dg_denoise_step(p, 1, bufs.h, W, W, seeds, bufs.tokens, bufs.entropy, bufs.argmax, bufs.accept, bufs.lse,
                       bufs.selfcond, ws)
    mhz = dg.dg_last_sm_clock(p, ws)
    assert 300.0 < mhz < 2200.0, mhz
    dg.dg_canvas_init(p, seeds, bufs.tokens, ws)
    assert dg.dg_last_sm_clock(p, ws) == 0.0
    small = dg.Workspace(p)
    small.nbytes = 64
    with pytest.raises(_abi.DgError) as e:
        dg.dg_last_sm_clock(p, small)
    assert e.value.status == _abi.DG_ENOMEM
    mhz_c = ctypes.c_float()
    assert dg.lib().dg_last_sm_clock(ctypes.byref(p), None, ws.nbytes, ctypes.byref(mhz_c), None) == _abi.DG_EINVAL
    assert dg.lib().dg_last_sm_clock(ctypes.byref(p), ws.ptr, ws.nbytes, None, None) == _abi.DG_EINVAL


def test_all_canvases_stopped_step_is_a_no_op(dg):
    """Empty work: once every canvas has stopped, a further step (and the stub) leaves every output as it was."""
    V, d, C, S = 4096, 128, 2, 16
    W = synth.weights(V, d)
    Wd = W.cuda()
    p = dg.params(C, V, d, max_steps=S)
    ws, bufs = dg.Workspace(p), dg.StepBuffers(p)
    seeds = torch.tensor(np.asarray(synth.canvas_seeds(C, base=70), np.uint64).view(np.int64), device="cuda")
    dg.dg_canvas_init(p, seeds, bufs.tokens, ws)
    s_stop = None
    for s in range(1, S + 1):
        dg.dg_stub_hidden(p, s, 300.0, 0.1, seeds, Wd, bufs.tokens, bufs.h, ws)
        dg.dg_denoise_step(p, s, bufs.h, Wd, Wd, seeds, bufs.tokens, bufs.entropy, bufs.argmax, bufs.accept,
                           bufs.lse, bufs.selfcond, ws)
        _, _, n = dg.dg_stop_check(p, ws)
        if n == C:
            s_stop = s
            break
    assert s_stop is not None and s_stop < S, "both canvases should stop early at gain 300"
    before = {k: getattr(bufs, k).clone() for k in ("h", "tokens", "entropy", "argmax", "accept", "lse", "selfcond")}
    dg.dg_stub_hidden(p, s_stop + 1, 300.0, 0.1, seeds, Wd, bufs.tokens, bufs.h, ws)
    dg.dg_denoise_step(p, s_stop + 1, bufs.h, Wd, Wd, seeds, bufs.tokens, bufs.entropy, bufs.argmax, bufs.accept,
                       bufs.lse, bufs.selfcond, ws)
    flags, _, n = dg.dg_stop_check(p, ws)
    assert flags == [1] * C and n == C
    for k, v in before.items():
        assert torch.equal(getattr(bufs, k), v), f"{k} changed in a step with no active canvas"


def test_maximum_canvases_per_launch(dg):
    """256 canvases (N = 65536) in one launch: every position against the oracle; 257 is refused."""
    from discrete_diffusion_decoding_b200 import _abi
    V, d, C = 4096, 128, 256
    W = synth.weights(V, d)
    h, _ = synth.spiked_hidden(W, C * 256, seed=90, gain_lo=0.5, gain_hi=20.0)
    p = dg.params(C, V, d)
    seeds = synth.canvas_seeds(C, base=500)
    Wd = W.cuda()
    g = gc.gpu_step(dg, p, 2, h, Wd, Wd, seeds)
    rows = _rows_all(C * 256)
    o = gc.oracle_rows(gc.bits(h), gc.bits(W), gc.bits(W), dg.temperature(p, 2), p.eb_bound, seeds, 2, rows, V)
    gc.compare(g, o, rows, p.eb_bound, tag="256 canvases")
    assert np.all(g["stable"] == 0) and np.all(g["stop"] == 0)      # step 2 of a fresh run: nothing stable yet
    with pytest.raises(_abi.DgError) as e:
        dg.workspace_size(dg.params(C + 1, V, d))
    assert e.value.status == _abi.DG_EINVAL
