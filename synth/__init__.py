"""Seeded synthetic inputs shared by the CUDA path's tests/bench and the oracle.

This module holds input recipes only - none of the sampling method's arithmetic.
Everything is generated on the CPU from fixed seeds with torch's CPU generator,
so both sides receive bit-identical bf16 tensors.

Shapes follow the workload the pages describe: a 256-token canvas (marrrang
deep dive, "Gemma based MoE backbone" table: canvas size 256 tokens) and a
Gemma-scale vocabulary head.  The pages give no vocabulary size or width; the
sizes used (V = 262144, d = 2816; V = 4096, d = 128 for the small case) are the
workload definitions of this project, not values from the pages.
"""

import math

import numpy as np
import torch

CANVAS = 256
ROWS_PER_CHUNK = 16384


def weights(vocab, hidden, seed=1234, std=0.02):
    """[V, d] bf16 embedding / vocabulary-head matrix, N(0, 1) * std rounded once.

    Generated in row chunks of 16384, chunk j from generator seed (seed * 1000003 + j),
    so the tensor is identical whatever the chunking of the consumer.
    """
    out = torch.empty((vocab, hidden), dtype=torch.bfloat16)
    for j, r0 in enumerate(range(0, vocab, ROWS_PER_CHUNK)):
        r1 = min(vocab, r0 + ROWS_PER_CHUNK)
        g = torch.Generator().manual_seed(seed * 1000003 + j)
        x = torch.empty((r1 - r0, hidden), dtype=torch.float32).normal_(generator=g)
        out[r0:r1] = (x * std).to(torch.bfloat16)
    return out


def gaussian_hidden(n, hidden, seed=42, scale=8.0):
    """[n, d] bf16 hidden states N(0, 1) / sqrt(d) * scale (single-step microbenchmark)."""
    g = torch.Generator().manual_seed(seed)
    x = torch.empty((n, hidden), dtype=torch.float32).normal_(generator=g)
    return (x * (scale / math.sqrt(hidden))).to(torch.bfloat16)


def spiked_hidden(W, n, seed=43, gain_lo=2.0, gain_hi=40.0, base_scale=8.0):
    """Hidden states whose entropies span 0 .. ln V.

    Row i = g_i * W[k_i] / ||W[k_i]||^2 + base noise, with k_i uniform over the
    vocabulary and g_i log-uniform in [gain_lo, gain_hi]; the spike makes logit
    k_i stand out by about g_i / T.  Recipe only; returns (h bf16 [n, d], k int64 [n]).
    """
    V, d = W.shape
    g = torch.Generator().manual_seed(seed)
    k = torch.randint(0, V, (n,), generator=g)
    gains = torch.exp(torch.empty(n).uniform_(math.log(gain_lo), math.log(gain_hi), generator=g))
    base = torch.empty((n, d)).normal_(generator=g) * (base_scale / math.sqrt(d))
    Wk = W[k].to(torch.float64)
    spike = Wk * (gains.to(torch.float64) / (Wk * Wk).sum(1))[:, None]
    return (spike + base.to(torch.float64)).to(torch.float32).to(torch.bfloat16), k


def canvas_seeds(n_canvas, base=0):
    """One 64-bit seed per canvas: canvas c gets seed base + c."""
    return np.arange(base, base + n_canvas, dtype=np.uint64)


def adversarial_rows(W, n, seed=44):
    """Row kinds by position mod 4 for the adversarial case (recipe only).

    0: near-uniform - h = 0 (even i/4) or 1e-3 * N(0, 1) (odd i/4);
    1: one-hot spike - h = g W_k / ||W_k||^2, g alternating 50 and 200;
    2: exact top-2 tie - h in span{W_a, W_b} with (h . W_a) = (h . W_b) in double
       before the bf16 rounding (after it the tie is a near-tie);
    3: placeholder spike rows (gain 8) that a test may replace by near-bound rows.
    Returns (h bf16 [n, d], kind int [n]).
    """
    V, d = W.shape
    g = torch.Generator().manual_seed(seed)
    Wd = W.to(torch.float64)
    h = torch.zeros((n, d), dtype=torch.float64)
    kind = torch.arange(n) % 4
    for i in range(n):
        q = i // 4
        if kind[i] == 0:
            if q % 2 == 1:
                h[i] = torch.empty(d, dtype=torch.float64).normal_(generator=g) * 1e-3
        elif kind[i] == 1 or kind[i] == 3:
            kk = int(torch.randint(0, V, (1,), generator=g))
            gain = (50.0 if q % 2 == 0 else 200.0) if kind[i] == 1 else 8.0
            h[i] = Wd[kk] * (gain / float(Wd[kk] @ Wd[kk]))
        else:
            a, b = [int(x) for x in torch.randint(0, V, (2,), generator=g)]
            wa, wb = Wd[a], Wd[b]
            # h = x wa + y wb with h.wa = h.wb = 20 (a large common logit)
            G = torch.tensor([[wa @ wa, wb @ wa], [wa @ wb, wb @ wb]], dtype=torch.float64)
            xy = torch.linalg.solve(G, torch.tensor([20.0, 20.0], dtype=torch.float64))
            h[i] = xy[0] * wa + xy[1] * wb
    return h.to(torch.float32).to(torch.bfloat16), kind


def bf16_bits(t):
    """bf16 tensor -> numpy uint16 bit patterns (what the oracle consumes)."""
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)
