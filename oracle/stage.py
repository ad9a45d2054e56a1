"""One denoising step of the sampling stage, in float64, written out directly.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``).

Sources (page title, section):
  [DD]  marrrang.tistory.com, "DiffusionGemma deep dive - Uniform State Diffusion
        and inference architecture": "Uniform State Diffusion" (x_t[i] ~ Uniform(V)),
        "reverse diffusion" steps 1-7, "standard sampling settings" table
        (48 steps, temperature linear 0.8 -> 0.4, entropy bound 0.1, stop 0.005),
        "Two-Fold Adaptive Stopping" (conditions 1 and 2, t-2 == t-1 == t).
  [JP]  juhoplayground.github.io, "DiffusionGemma - parallel text generation":
        "inference mechanism" (self-conditioning = softmax-probability-weighted
        token embedding; logits scheduler = temperature sharpening; entropy
        bounded sampler).
  [AX]  axbrief.com, "DiffusionGemma": --diffusion-eb-max-steps (default 48).

Everything is float64 on the exact bf16 inputs the GPU receives (bf16 bit
patterns widened to double).  The N x V logits block is formed explicitly: that
is allowed here, and only here.

The sampled-acceptance mode (``gumbel_from_words``, ``gumbel_sample``; the accepted
token is a draw from softmax(z / T) rather than the argmax) is a reading of the
same passages - [DD] step 4 keeps "high-confidence" tokens and [JP] names
temperature sharpening - that the pages leave open; the argmax mode stays the
default.

Parity status: every function below is pinned by tests/test_oracle_stage.py
(closed forms, brute force, invariants) and, for the sampler, by
tests/test_oracle_sample.py (Gumbel moments and CDF, chi-square of the draws
against softmax, planted mistakes, limits), except ``stub_hidden``'s realism as a
stand-in for a trained denoiser, which is "parity unpinned" by nature: the
pages print no sampler trajectory.
"""

import math

import numpy as np

from . import philox

LN2 = math.log(2.0)


# ----------------------------------------------------------------------------- bf16
def bf16_to_f64(u16):
    """Widen bf16 bit patterns (uint16) to float64 exactly."""
    u = np.asarray(u16, dtype=np.uint16).astype(np.uint32) << np.uint32(16)
    with np.errstate(invalid="ignore"):
        return u.view(np.float32).astype(np.float64)


def f32_to_bf16(x32):
    """Round float32 values to bf16 (round to nearest, ties to even); uint16 bits."""
    u = np.asarray(x32, dtype=np.float32).view(np.uint32).astype(np.uint64)
    lsb = (u >> np.uint64(16)) & np.uint64(1)
    r = (u + np.uint64(0x7FFF) + lsb) >> np.uint64(16)
    nan = np.isnan(np.asarray(x32, dtype=np.float32))
    r = np.where(nan, np.uint64(0x7FC0), r)
    return r.astype(np.uint16)


def f64_to_bf16(x):
    """float64 -> bf16 through float32 (the GPU rounds fp32 results the same way)."""
    return f32_to_bf16(np.asarray(x, dtype=np.float64).astype(np.float32))


# ----------------------------------------------------------------------- schedule
def temperature(s, max_steps, t_start=0.8, t_end=0.4):
    """Linear decay t_start -> t_end over the max-step schedule ([DD] settings table).

    Reading: T_1 = t_start, T_S = t_end, computed in double, handed to both sides
    as the float32 the kernels receive.
    """
    if max_steps <= 1:
        t = t_start
    else:
        t = t_start + (t_end - t_start) * (s - 1) / (max_steps - 1)
    return float(np.float32(t))


# ----------------------------------------------------------------- the step itself
def logits(h, W, T):
    """z[i, v] = (h_i . W_v) / T  in float64 ([JP]: logits for every canvas position)."""
    return (np.asarray(h, np.float64) @ np.asarray(W, np.float64).T) / float(T)


def distribution_stats(z):
    """Per position: max, log-sum-exp, probabilities, entropy (nats), argmax, top-2 gap.

    H = LSE - sum_v p_v z_v with p = softmax(z); argmax is the smallest index
    attaining the maximum; top2gap = max - (largest value at any other index).
    """
    z = np.asarray(z, np.float64)
    m = z.max(axis=1)
    e = np.exp(z - m[:, None])
    l = e.sum(axis=1)
    lse = m + np.log(l)
    p = e / l[:, None]
    H = lse - (p * z).sum(axis=1)
    am = z.argmax(axis=1)                 # numpy returns the first (smallest) index
    z2 = z.copy()
    z2[np.arange(z.shape[0]), am] = -np.inf
    gap = m - z2.max(axis=1)
    return {"max": m, "lse": lse, "p": p, "H": H, "argmax": am.astype(np.int64), "top2gap": gap}


def self_conditioning(p, E):
    """sc_i = sum_v p[i, v] E[v, :]  ([JP]: probability-weighted token embedding)."""
    return np.asarray(p, np.float64) @ np.asarray(E, np.float64)


def renoise_tokens(seed, s, c, vocab, n=256):
    """Uniform re-noise draws for every position of canvas c at step s (tag 1)."""
    return philox.uniform_token(seed, np.arange(n), s, c, philox.TAG_RENOISE, vocab)


def init_tokens(seed, c, vocab, n=256):
    """Canvas initialisation: every position uniform over the vocabulary (step 0, tag 0)."""
    return philox.uniform_token(seed, np.arange(n), 0, c, philox.TAG_INIT, vocab)


SAMPLE_CHUNK = 64      # vocabulary entries per chunk of the sampled acceptance


def uniform_open(w):
    """(u, 1 - u) for 32-bit words w: u = (w + 1/2) / 2^32 on (0, 1), both exact in double."""
    w = np.asarray(w, np.float64)
    return (w + 0.5) / 4294967296.0, (4294967295.0 - w + 0.5) / 4294967296.0


def gumbel_from_words(w):
    """Standard Gumbel noise g = -ln(-ln u), u from uniform_open; -ln u is taken as
    -log1p(-(1 - u)), so the noise keeps full relative precision as u -> 1."""
    _, one_minus_u = uniform_open(w)
    return -np.log(-np.log1p(-one_minus_u))


def gumbel_sample(z, seed, s, c, positions, chunk=SAMPLE_CHUNK):
    """Sampled acceptance: an exact draw from softmax(z_i) for each row, in two levels.

    The vocabulary is cut into chunks of 64 consecutive entries.  (1) A chunk q is
    chosen by the Gumbel-max trick on the chunk log-masses: argmax_q of
    ln(sum_{v in q} e^{z_v}) + g_q (smallest q on a tie), g_q from word 0 of Philox
    counter (q, s, c, 4 + 256 i) - so P(q) = mass_q / total (Gumbel 1954; the
    "Gumbel-max trick", Maddison, Tarlow and Minka 2014).  (2) Inside it the entry
    is the inverse CDF of the chunk's normalised probabilities at r = word 1 of the
    same counter mapped by uniform_open: the smallest v whose running sum exceeds
    r (the last entry with non-zero probability should rounding leave none).  The
    two words are independent, so P(v) = P(q) P(v | q) = softmax(z)_v.
    z are the temperature-scaled logits (the distribution whose entropy the bound
    tests).  Returns (sample int64 [n], keygap [n]: best chunk key minus the
    second best, cdf_margin [n]: min_k |running sum_k - r| in the chosen chunk),
    the last two for the near-tie exclusions.
    """
    z = np.asarray(z, np.float64)
    n, V = z.shape
    assert V % chunk == 0, "the vocabulary is a whole number of chunks"
    nq = V // chunk
    out = np.empty(n, np.int64)
    gap = np.empty(n)
    margin = np.empty(n)
    for row, i in enumerate(positions):
        zc = z[row].reshape(nq, chunk)
        mq = zc.max(axis=1)
        with np.errstate(invalid="ignore"):
            logmass = mq + np.log(np.exp(zc - mq[:, None]).sum(axis=1))
        logmass = np.where(np.isfinite(mq), logmass, -np.inf)
        w = philox.chunk_words(seed, int(i), s, c, nq)
        key = logmass + gumbel_from_words(w[:, 0])
        q = int(np.argmax(key))
        k2 = key.copy()
        k2[q] = -np.inf
        gap[row] = key[q] - k2.max() if nq > 1 else np.inf
        r, _ = uniform_open(w[q, 1])
        p = np.exp(zc[q] - logmass[q])
        cs = np.cumsum(p)
        hit = np.nonzero(cs > r)[0]
        j = int(hit[0]) if hit.size else int(np.nonzero(p > 0)[0][-1])
        out[row] = q * chunk + j
        margin[row] = np.min(np.abs(cs - r))
    return out, gap, margin


def eb_accept(H, argmax, bound, renoise):
    """Entropy-bounded accept / re-noise ([JP] sampler; [DD] steps 4-5, bound 0.1).

    Reading: per position, accept when H <= bound (inclusive) and keep the argmax;
    otherwise the position takes the uniform re-noise draw.
    """
    acc = np.asarray(H) <= bound
    tokens = np.where(acc, argmax, renoise).astype(np.int64)
    return tokens, acc.astype(np.uint8)


def group_accept(H, kept, bound, renoise):
    """Group entropy-bounded accept for the positions of one canvas ([JP] sampler: token
    groups are accepted by entropy-based confidence; [DD] settings table: bound 0.1).

    Reading: order the positions by entropy max(H, 0), ties by position, and accept the
    longest prefix whose cumulative entropy is <= bound - the largest set of positions
    whose entropies sum to at most the bound, and of the sets of that size the one with
    the least total; the other positions take their re-noise draw.  No position is
    forced through when even the smallest entropy exceeds the bound (as in the
    per-position rule).  kept is the token an accepted position keeps (the argmax, or
    the sample of the sampled mode).
    Returns (tokens, accept uint8, cut_margin, order_gap): the distance from the bound
    of the cumulative sums on either side of the cut, and the entropy gap between the
    last accepted and the first rejected position (for the parity exclusions).
    """
    H = np.maximum(np.asarray(H, np.float64), 0.0)
    n = H.size
    order = np.lexsort((np.arange(n), H))
    S = np.cumsum(H[order])
    k = int(np.count_nonzero(S <= bound))          # S is non-decreasing: the accepted prefix
    acc = np.zeros(n, bool)
    acc[order[:k]] = True
    tokens = np.where(acc, kept, renoise).astype(np.int64)
    cut = [abs(S[k - 1] - bound)] if k > 0 else []
    if k < n:
        cut.append(abs(S[k] - bound))
    cut_margin = min(cut) if cut else np.inf
    order_gap = H[order[k]] - H[order[k - 1]] if 0 < k < n else np.inf
    return tokens, acc.astype(np.uint8), float(cut_margin), float(order_gap)


def stop_update(mean_H, argmax, prev_argmax, stable, s, stop_thresh=0.005, stability=2):
    """Two-fold adaptive stop for one canvas ([DD] conditions 1 and 2).

    stable counts consecutive steps whose argmax vector equals the previous
    step's; it is 0 at step 1 and resets on any change.  Stop when the mean
    entropy is strictly below the threshold AND stable >= stability (with 2:
    three identical argmax vectors, so the earliest stop is step 3).
    """
    same = s > 1 and prev_argmax is not None and np.array_equal(argmax, prev_argmax)
    stable = stable + 1 if same else 0
    stop = bool(mean_H < stop_thresh and stable >= stability)
    return stable, stop


def denoise_step(h_u16, W_u16, E_u16, T, bound, seeds, s, vocab, canvas_len=256,
                 want_selfcond=True, canvas_ids=None, accept_rule=0):
    """One step over all canvases of a batch, from bf16 bit patterns.

    h_u16 [N, d], W_u16 / E_u16 [V, d] (uint16 bf16 bits, or their exact float64
    widening), seeds [C] (uint64),
    N = C * canvas_len; canvas_ids[c] (default c) is the canvas word of the
    Philox counter.  accept_rule 0 accepts per position (eb_accept), 1 by groups
    (group_accept; the cut margins are returned as cut_margin / order_gap per canvas).
    Returns dict with H, argmax, lse, top2gap, tokens, accept, selfcond (or None),
    mean_H per canvas.
    """
    h = bf16_to_f64(h_u16)
    W = _widen(np.asarray(W_u16))
    E = W if E_u16 is W_u16 else _widen(np.asarray(E_u16))
    n = h.shape[0]
    C = n // canvas_len
    out = {k: [] for k in ("H", "argmax", "lse", "top2gap", "tokens", "accept", "selfcond", "max",
                           "cut_margin", "order_gap")}
    for c in range(C):
        sl = slice(c * canvas_len, (c + 1) * canvas_len)
        st = distribution_stats(logits(h[sl], W, T))
        cid = c if canvas_ids is None else int(canvas_ids[c])
        ren = renoise_tokens(int(seeds[c]), s, cid, vocab, canvas_len)
        if accept_rule == 1:
            tok, acc, cm, og = group_accept(st["H"], st["argmax"], bound, ren)
            out["cut_margin"].append(np.array([cm]))
            out["order_gap"].append(np.array([og]))
        else:
            tok, acc = eb_accept(st["H"], st["argmax"], bound, ren)
        out["H"].append(st["H"])
        out["argmax"].append(st["argmax"])
        out["lse"].append(st["lse"])
        out["top2gap"].append(st["top2gap"])
        out["max"].append(st["max"])
        out["tokens"].append(tok)
        out["accept"].append(acc)
        if want_selfcond:
            out["selfcond"].append(self_conditioning(st["p"], E))
        del st
    res = {k: (np.concatenate(v) if v else None) for k, v in out.items()}
    res["mean_H"] = res["H"].reshape(C, canvas_len).mean(axis=1)
    return res


# ------------------------------------------------------------ large vocabularies
def _widen(block):
    """bf16 bit patterns are widened to float64; float64 input is used as it is."""
    return block if block.dtype == np.float64 else bf16_to_f64(block)


def logits_chunked(h, W, T, chunk=16384):
    """z = (h W^T) / T in float64, W (bf16 bits or float64) taken chunk by chunk (memory only)."""
    h = np.asarray(h, np.float64)
    V = W.shape[0]
    z = np.empty((h.shape[0], V))
    for v0 in range(0, V, chunk):
        v1 = min(V, v0 + chunk)
        z[:, v0:v1] = (h @ _widen(W[v0:v1]).T) / float(T)
    return z


def self_conditioning_chunked(p, E, chunk=16384):
    """sc = p E in float64, E (bf16 bits or float64) taken chunk by chunk (memory only)."""
    V, d = E.shape
    sc = np.zeros((p.shape[0], d))
    for v0 in range(0, V, chunk):
        v1 = min(V, v0 + chunk)
        sc += p[:, v0:v1] @ _widen(E[v0:v1])
    return sc


def step_rows(h_u16, W_u16, E_u16, T, bound, seed, s, c, positions, vocab, want_selfcond=True,
              accept_mode=0):
    """One step for selected positions of one canvas (rows of h_u16 are those positions).

    W_u16 / E_u16 may be bf16 bit patterns or their exact float64 widening.

    positions: index of each row within its canvas (for the re-noise and sample draws).
    accept_mode 0 keeps the argmax at accepted positions, 1 a Gumbel-max sample of
    softmax(z / T) (gumbel_sample).
    Returns dict with H, argmax, lse, top2gap, tokens, accept, selfcond, and with
    accept_mode 1 also sample, keygap and cdf_margin.
    """
    h = bf16_to_f64(h_u16)
    z = logits_chunked(h, W_u16, T)
    out = {}
    kept = None
    if accept_mode == 1:
        out["sample"], out["keygap"], out["cdf_margin"] = gumbel_sample(z, seed, s, c, positions)
        kept = out["sample"]
    st = distribution_stats(z)
    del z
    ren = philox.uniform_token(seed, np.asarray(positions), s, c, philox.TAG_RENOISE, vocab)
    tok, acc = eb_accept(st["H"], st["argmax"] if kept is None else kept, bound, ren)
    out.update({k: st[k] for k in ("H", "argmax", "lse", "top2gap", "max")})
    out["tokens"], out["accept"] = tok, acc
    out["selfcond"] = self_conditioning_chunked(st["p"], E_u16) if want_selfcond else None
    return out


# ------------------------------------------------------- split-vocabulary statistics
def partial_stats(z):
    """Statistics of one vocabulary range, relative to that range's own maximum.

    (m, l, u, a, zmax) with l = sum e^{z-m}, u = sum e^{z-m} (z-m), a = argmax
    (index within the range) - the quantities a streamed pass keeps per range.
    """
    z = np.asarray(z, np.float64)
    m = z.max(axis=1)
    e = np.exp(z - m[:, None])
    return {"m": m, "l": e.sum(1), "u": (e * (z - m[:, None])).sum(1), "a": z.argmax(1)}


def merge_stats(A, B, offset_b):
    """Merge the statistics of two disjoint ranges (B's indices shifted by offset_b).

    M = max(mA, mB); l = sum_r e^{m_r-M} l_r; u = sum_r e^{m_r-M} (u_r + (m_r-M) l_r);
    the argmax is the larger maximum, the smaller index on an exact tie.
    """
    M = np.maximum(A["m"], B["m"])
    fa, fb = np.exp(A["m"] - M), np.exp(B["m"] - M)
    l = fa * A["l"] + fb * B["l"]
    u = fa * (A["u"] + (A["m"] - M) * A["l"]) + fb * (B["u"] + (B["m"] - M) * B["l"])
    ia, ib = np.asarray(A["a"]), np.asarray(B["a"]) + offset_b
    take_b = (B["m"] > A["m"]) | ((B["m"] == A["m"]) & (ib < ia))
    return {"m": M, "l": l, "u": u, "a": np.where(take_b, ib, ia)}


def finish_stats(S):
    """LSE = m + ln l, H = ln l - u / l, from merged statistics."""
    return {"lse": S["m"] + np.log(S["l"]), "H": np.log(S["l"]) - S["u"] / S["l"], "argmax": S["a"]}


# ------------------------------------------------------------------ benchmark stub
def stub_hidden(E_u16, tokens, seed, s, c, max_steps, gain=1.0, noise=0.1):
    """Toy denoiser stand-in: h_i = g (a E[tgt_i] + (1-a) E[x_i]) + sigma n_i.

    a = s / max_steps; tgt_i uniform over V (tag 2, step 0); n_i standard normal
    from Philox tag 3 by Box-Muller: counter (i*d/4 + k//4, s, c, 3) gives words
    (w0, w1, w2, w3); u1 = (w0 + 1) 2^-32, u2 = w1 2^-32, r = sqrt(-2 ln u1),
    n_{4j} = r cos(2 pi u2), n_{4j+1} = r sin(2 pi u2); likewise (w2, w3) give
    n_{4j+2}, n_{4j+3}.  Computed in double, rounded to bf16 through float32.
    This stand-in is not on the pages; its realism is "parity unpinned".
    """
    E_u16 = np.asarray(E_u16)
    V, d = E_u16.shape
    tokens = np.asarray(tokens, np.int64)
    n = tokens.shape[0]
    a = s / max_steps
    tgt = philox.uniform_token(seed, np.arange(n), 0, c, philox.TAG_STUB_TARGET, V)
    j = np.arange(n)[:, None] * (d // 4) + np.arange(d // 4)[None, :]
    w = philox.words(seed, j, s, c, philox.TAG_STUB_NOISE).astype(np.float64)   # [n, d/4, 4]
    u1a = (w[..., 0] + 1.0) * 2.0 ** -32
    u2a = w[..., 1] * 2.0 ** -32
    u1b = (w[..., 2] + 1.0) * 2.0 ** -32
    u2b = w[..., 3] * 2.0 ** -32
    ra = np.sqrt(-2.0 * np.log(u1a))
    rb = np.sqrt(-2.0 * np.log(u1b))
    nz = np.stack([ra * np.cos(2 * np.pi * u2a), ra * np.sin(2 * np.pi * u2a),
                   rb * np.cos(2 * np.pi * u2b), rb * np.sin(2 * np.pi * u2b)], axis=-1)
    nz = nz.reshape(n, d)
    # only the gathered rows are widened (the values are those of the whole widened table)
    h = gain * (a * bf16_to_f64(E_u16[tgt]) + (1.0 - a) * bf16_to_f64(E_u16[tokens])) + noise * nz
    return f64_to_bf16(h), tgt
