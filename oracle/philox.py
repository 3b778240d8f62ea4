"""Philox4x32-10 counter-based random numbers, float64-free integer reference
(test infrastructure, like the rest of oracle/; the library has its own CUDA
implementation of the same published generator and shares no code with this).

Definition (Salmon, Moraes, Dror, Shaw, "Parallel random numbers: as easy as
1, 2, 3", SC 2011, the Philox-4x32 bijection): a 128-bit counter (c0, c1, c2, c3)
and a 64-bit key (k0, k1) go through 10 rounds. One round multiplies c0 and c2
by two fixed odd constants as full 32x32 -> 64-bit products and recombines
  (c0, c1, c2, c3) <- (hi(M1*c2) ^ c1 ^ k0,  lo(M1*c2),  hi(M0*c0) ^ c3 ^ k1,  lo(M0*c0));
between rounds the key is bumped by the Weyl constants (k0 += W0, k1 += W1,
modulo 2^32). The four words after round 10 are the output.

The draft noise of the sampled drafter uses it as follows (the definition both
sides follow): for request b, block position i (1..B-1) and vocabulary entry v,
the uniform is word (v mod 128) div 32 of Philox4x32-10 at counter
(v div 128, v mod 32, i, b) under key (seed_lo, seed_hi), mapped to
u = ((word >> 9) + 1/2) / 2^23, which lies strictly inside (0, 1) and is exact in
float32 (at most 24 significant bits).
"""
from __future__ import annotations

from typing import Sequence, Tuple

import numpy as np

M0, M1 = 0xD2511F53, 0xCD9E8D57   # round multipliers
W0, W1 = 0x9E3779B9, 0xBB67AE85   # key increments (golden ratio, sqrt(3) - 1, scaled to 2^32)
MASK = 0xFFFFFFFF


def _mulhilo(a: np.ndarray, b: int) -> Tuple[np.ndarray, np.ndarray]:
    p = a.astype(np.uint64) * np.uint64(b)
    return (p >> np.uint64(32)).astype(np.uint64), (p & np.uint64(MASK)).astype(np.uint64)


def philox4x32_10(counter: Sequence, key: Sequence) -> np.ndarray:
    """counter: 4 arrays (or ints) of uint32 words, broadcast together; key: 2 words.
    Returns a [4, ...] uint64 array holding the four 32-bit output words."""
    c = [np.asarray(x, dtype=np.uint64) & np.uint64(MASK) for x in counter]
    c = list(np.broadcast_arrays(*c))
    k0, k1 = np.uint64(int(key[0]) & MASK), np.uint64(int(key[1]) & MASK)
    for r in range(10):
        if r > 0:
            k0 = (k0 + np.uint64(W0)) & np.uint64(MASK)
            k1 = (k1 + np.uint64(W1)) & np.uint64(MASK)
        hi0, lo0 = _mulhilo(c[0], M0)
        hi1, lo1 = _mulhilo(c[2], M1)
        c = [hi1 ^ c[1] ^ k0, lo1, hi0 ^ c[3] ^ k1, lo0]
    return np.stack(c)


def word_to_uniform(w) -> np.ndarray:
    """A 32-bit word to a uniform strictly inside (0, 1): ((w >> 9) + 1/2) / 2^23."""
    w = np.asarray(w, dtype=np.uint64)
    return ((w >> np.uint64(9)).astype(np.float64) + 0.5) / float(1 << 23)


def draft_uniforms(seed: int, b: int, i: int, V: int) -> np.ndarray:
    """The draft noise uniforms u[v], v < V, of request b at block position i."""
    v = np.arange(V, dtype=np.uint64)
    words = philox4x32_10((v // np.uint64(128), v % np.uint64(32), np.uint64(i), np.uint64(b)),
                          (seed & MASK, (seed >> 32) & MASK))
    sel = (v % np.uint64(128)) // np.uint64(32)
    return word_to_uniform(np.take_along_axis(words, sel[None, :].astype(np.int64), axis=0)[0])
