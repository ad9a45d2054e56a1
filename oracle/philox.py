"""Philox4x32-10 counter-based generator and the draws the sampler makes from it.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``).

The pages say only that noised positions hold tokens drawn uniformly from the
vocabulary (marrrang.tistory.com deep dive, "Uniform State Diffusion":
x_t[i] ~ Uniform(V); juhoplayground overview, "Entropy Bounded Sampler":
initialise with uniform random tokens, re-noise with random alternatives).
They name no generator.  The generator used here is Philox4x32-10 as defined by
Salmon, Moraes, Dror and Shaw, "Parallel Random Numbers: As Easy as 1, 2, 3"
(SC'11), section 4: a 10-round bijection on a 128-bit counter under a 64-bit key,
each round two 32x32->64 multiplies with constants 0xD2511F53 and 0xCD9E8D57,
the key bumped between rounds by the Weyl constants 0x9E3779B9 and 0xBB67AE85.

Keying (a reading, the pages are silent): key = (lo32(seed), hi32(seed)) of the
per-canvas seed; counter = (position i, step s, canvas c, tag).  Tags separate
the streams: 0 canvas init, 1 re-noise, 2 stub target ids, 3 stub Gaussian noise.
A token is word 0 mapped to [0, V) by the multiply-high floor(r * V / 2^32).
The sampled-acceptance mode draws one counter per (position, chunk of 64
vocabulary entries): counter (floor(v / 64), s, c, 4 + 256 i), words 0 and 1 -
the fourth counter word is >= 4 there, so these streams never meet the four
above.

Pins: known-answer vectors of the SC'11 reference implementation
(tests/golden/philox4x32_10_kat.txt), bijectivity on a reduced counter set,
stream separation and a chi-square uniformity test (tests/test_oracle_philox.py).
"""

import numpy as np

PHILOX_M0 = 0xD2511F53
PHILOX_M1 = 0xCD9E8D57
PHILOX_W0 = 0x9E3779B9
PHILOX_W1 = 0xBB67AE85
MASK32 = 0xFFFFFFFF

TAG_INIT = 0
TAG_RENOISE = 1
TAG_STUB_TARGET = 2
TAG_STUB_NOISE = 3
TAG_SAMPLE = 4


def _round(c0, c1, c2, c3, k0, k1):
    """One Philox S-box round on uint64 arrays that hold 32-bit values."""
    p0 = c0 * np.uint64(PHILOX_M0)          # exact: both factors < 2^32
    p1 = c2 * np.uint64(PHILOX_M1)
    hi0, lo0 = p0 >> np.uint64(32), p0 & np.uint64(MASK32)
    hi1, lo1 = p1 >> np.uint64(32), p1 & np.uint64(MASK32)
    return (hi1 ^ c1 ^ k0, lo1, hi0 ^ c3 ^ k1, lo0)


def philox4x32_10(counter, key):
    """Philox4x32 with 10 rounds.

    counter: integer array [..., 4] of 32-bit words; key: integer array [..., 2].
    Returns uint32 array [..., 4].
    """
    ctr = np.asarray(counter, dtype=np.uint64) & np.uint64(MASK32)
    k = np.asarray(key, dtype=np.uint64) & np.uint64(MASK32)
    c0, c1, c2, c3 = ctr[..., 0], ctr[..., 1], ctr[..., 2], ctr[..., 3]
    k0, k1 = k[..., 0], k[..., 1]
    for r in range(10):
        if r > 0:
            k0 = (k0 + np.uint64(PHILOX_W0)) & np.uint64(MASK32)
            k1 = (k1 + np.uint64(PHILOX_W1)) & np.uint64(MASK32)
        c0, c1, c2, c3 = _round(c0, c1, c2, c3, k0, k1)
    return np.stack([c0, c1, c2, c3], axis=-1).astype(np.uint32)


def seed_key(seed):
    """Split a 64-bit seed into the (lo32, hi32) key words."""
    seed = int(seed) & 0xFFFFFFFFFFFFFFFF
    return np.array([seed & MASK32, seed >> 32], dtype=np.uint64)


def words(seed, i, s, c, tag):
    """The four output words for counter (i, s, c, tag) under the seed's key.

    i may be an array; s, c, tag are scalars or broadcastable arrays.
    """
    i = np.asarray(i, dtype=np.uint64)
    ctr = np.stack(np.broadcast_arrays(i, np.uint64(s), np.uint64(c), np.uint64(tag)), axis=-1)
    return philox4x32_10(ctr, seed_key(seed))


def uniform_token(seed, i, s, c, tag, vocab):
    """floor(word0 * V / 2^32): a token uniform on [0, V) (exact when V is a power of 2)."""
    w0 = words(seed, i, s, c, tag)[..., 0].astype(np.uint64)
    return ((w0 * np.uint64(vocab)) >> np.uint64(32)).astype(np.int64)



def chunk_words(seed, i, s, c, n_chunks):
    """Words 0 and 1 of counter (q, s, c, TAG_SAMPLE + 256 i) for every chunk q of position i.

    Returns uint32 [n_chunks, 2]: word 0 drives the chunk's Gumbel key, word 1 the
    draw inside the chunk."""
    w = words(seed, np.arange(n_chunks, dtype=np.uint64), s, c, TAG_SAMPLE + 256 * int(i))
    return w[:, :2]
