"""Multi-step canvas decoding loops built from ``stage`` (float64).

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``).

Follows the page flow of the deep dive (marrrang.tistory.com, "system
architecture" flow and "Block Diffusion"): a 256-token canvas is initialised
with uniform noise, denoised for at most S steps with the two-fold adaptive stop
checked after each step, then committed; block-autoregressive decoding repeats
this canvas after canvas.  The denoiser network itself is out of scope; a
``hidden(tokens, s, c)`` callable stands in for it.

Reading: the committed block is the argmax vector of the last executed step
(committing re-noised random tokens would contradict "keep confident tokens").
Stopped canvases of a batch are frozen: no further step touches them.
"""

import numpy as np

from . import stage


def decode_batch(W_u16, E_u16, seeds, hidden, vocab, max_steps=48, t_start=0.8, t_end=0.4,
                 bound=0.1, stop_thresh=0.005, stability=2, canvas_len=256,
                 want_selfcond=False, record=False, accept_rule=0):
    """Free-running decode of C independent canvases in one batch.

    hidden(tokens_of_canvas[int64 canvas_len], s, c) -> bf16 bits [canvas_len, d].
    Returns dict: stop_step[C], committed[C, canvas_len], tokens (final canvas),
    and, if record, a per-step trace.
    """
    C = len(seeds)
    tokens = np.stack([stage.init_tokens(int(seeds[c]), c, vocab, canvas_len) for c in range(C)])
    prev = [None] * C
    stable = [0] * C
    stopped = [False] * C
    stop_step = [max_steps] * C
    committed = np.zeros((C, canvas_len), np.int64)
    trace = []
    for s in range(1, max_steps + 1):
        T = stage.temperature(s, max_steps, t_start, t_end)
        rec = {"s": s, "T": T, "canvases": {}}
        for c in range(C):
            if stopped[c]:
                continue
            h = hidden(tokens[c].copy(), s, c)
            r = stage.denoise_step(h, W_u16, E_u16, T, bound, [seeds[c]], s, vocab,
                                   canvas_len, want_selfcond, canvas_ids=[c], accept_rule=accept_rule)
            tok, acc = r["tokens"], r["accept"]
            stable[c], stop = stage.stop_update(r["mean_H"][0], r["argmax"], prev[c], stable[c], s,
                                                stop_thresh, stability)
            prev[c] = r["argmax"].copy()
            if record:
                rec["canvases"][c] = {"h": h, "H": r["H"], "argmax": r["argmax"], "tokens_in": tokens[c].copy(),
                                      "tokens": tok, "accept": acc, "mean_H": r["mean_H"][0],
                                      "stable": stable[c], "stop": stop, "top2gap": r["top2gap"],
                                      "cut_margin": r["cut_margin"], "order_gap": r["order_gap"]}
            tokens[c] = tok
            if stop or s == max_steps:
                stopped[c] = True
                stop_step[c] = s
                committed[c] = r["argmax"]
        trace.append(rec)
        if all(stopped):
            break
    return {"stop_step": np.array(stop_step), "committed": committed, "tokens": tokens,
            "trace": trace if record else None}


def stub_hidden_fn(E_u16, seeds, max_steps, gain=1.0, noise=0.1):
    """The benchmark stub as a ``hidden`` callable for ``decode_batch``."""
    def hidden(tok, s, c):
        h, _ = stage.stub_hidden(E_u16, tok, int(seeds[c]), s, c, max_steps, gain, noise)
        return h
    return hidden
