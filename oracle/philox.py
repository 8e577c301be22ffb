"""Philox4x32-10 counter-based random numbers and the sampler's uniform draws.

Philox4x32 is restated from its published definition (Philox, SC'11): a
4-word counter is put through R rounds; each round multiplies counter words
0 and 2 by two fixed 32-bit multipliers, splits each 64-bit product into its
high and low halves, and forms the new counter as
(hi1 ^ c1 ^ k0, lo1, hi0 ^ c3 ^ k1, lo0).  The two key words are advanced by
two fixed Weyl increments before every round except the first.  The
ten-round variant is the one the authors recommend.

The uniforms of the Psi-Spec sampler are one Philox block per draw:

* key     = (seed & 0xffffffff, seed >> 32)
* counter = (stream, position, kind, lane), where ``stream`` is the
  request's random stream id, ``position`` the absolute 0-based position of
  the token that the draw decides, ``kind`` one of the ``KIND_*`` values
  below and ``lane`` 0 (the tree sampler's chain index);
* u = ((x0 >> 9) * 2 + 1) * 2**-24 from output word 0, which lies strictly
  inside (0, 1) and is exact in float32.

Parity pin: the published known-answer vectors in
``tests/golden/philox4x32_10_kat.txt``.
"""

import numpy as np

_MASK32 = np.uint64(0xFFFFFFFF)
PHILOX_M0 = np.uint64(0xD2511F53)
PHILOX_M1 = np.uint64(0xCD9E8D57)
PHILOX_W0 = np.uint64(0x9E3779B9)
PHILOX_W1 = np.uint64(0xBB67AE85)

KIND_FIRST = 0   # first block token, sampled from the AR distribution
KIND_DRAFT = 1   # drafted tokens 2..B, sampled from the diffusion distribution
KIND_ACCEPT = 2  # accept test of a drafted token
KIND_RESID = 3   # token at the first rejected position (or the bonus token)
KIND_NOISE = 4   # optional uniform-noise prior of the noised block
KIND_PROMPT = 5  # reserved


def philox4x32_10(counter, key, rounds=10):
    """Philox4x32 with ``rounds`` rounds (default 10).

    ``counter`` is a sequence of four uint32 values or arrays (broadcast
    together); ``key`` a sequence of two.  Returns a tuple of four uint32
    numpy arrays.  Pinned by the published known-answer vectors.
    """
    c0, c1, c2, c3 = (np.asarray(w, dtype=np.uint64) & _MASK32 for w in counter)
    k0, k1 = (np.asarray(w, dtype=np.uint64) & _MASK32 for w in key)
    for r in range(rounds):
        if r > 0:
            k0 = (k0 + PHILOX_W0) & _MASK32
            k1 = (k1 + PHILOX_W1) & _MASK32
        p0 = PHILOX_M0 * c0          # both factors < 2**32: exact in uint64
        p1 = PHILOX_M1 * c2
        hi0, lo0 = p0 >> np.uint64(32), p0 & _MASK32
        hi1, lo1 = p1 >> np.uint64(32), p1 & _MASK32
        c0, c1, c2, c3 = hi1 ^ c1 ^ k0, lo1, hi0 ^ c3 ^ k1, lo0
    return tuple(np.asarray(w, dtype=np.uint32) for w in (c0, c1, c2, c3))


def bits_to_uniform(x):
    """Map a 32-bit word to u = ((x >> 9) * 2 + 1) / 2**24, in (0, 1).

    The result has at most 24 significant bits, so it is exact in float32 and
    float64 alike.  Closed forms: x = 0 gives 2**-24, x = 2**32 - 1 gives
    1 - 2**-24.
    """
    x = np.asarray(x, dtype=np.uint64)
    return ((x >> np.uint64(9)) * np.uint64(2) + np.uint64(1)).astype(np.float64) / float(1 << 24)


def uniform(seed, stream, position, kind, lane=0):
    """The uniform of draw ``kind`` for the token at ``position`` of ``stream``.

    ``lane`` is counter word 3: 0 for every draw of the linear sampler; the
    tree sampler numbers its drafted chains with it (chain 0 draws exactly
    the linear sampler's uniforms).  Any argument may be an array; the
    result broadcasts.
    """
    seed = int(seed)
    key = (seed & 0xFFFFFFFF, (seed >> 32) & 0xFFFFFFFF)
    x0, _, _, _ = philox4x32_10((stream, position, kind, lane), key)
    return bits_to_uniform(x0)
