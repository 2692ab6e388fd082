"""Oracle of the n-gram table row gather.

TEST INFRASTRUCTURE (see ``oracle/moe.py``): only ``tests/``,
``__graft_entry__.smoke()`` and the CPU legs of ``bench.py`` use it.

What it computes ([P3], pyshine Strata tour, "Understanding the
Architecture"): a large per-layer token-embedding table is kept outside the
expert packs; the last three token ids of a token are hashed into 16 row
indices, and only those rows are read.  The pages give neither the hash nor
the row format, so both are self-defined (the library header states the same
definition):

* ``mix64`` is SplitMix64's output finaliser (Steele, Lea & Flood, OOPSLA 2014);
  ``splitmix64(s, n)`` is the first ``n`` outputs of the generator seeded with
  state ``s``: output i = mix64(s + (i + 1) G), G = 0x9E3779B97F4A7C15.
* hash of the ids (a, b, c) of a token: h = splitmix64(seed, 1)[0], then
  h = mix64(h XOR u) for u = a, b, c in turn (each id's 32-bit pattern).
* row i = floor(x_i R / 2^64) with x_i = splitmix64(h, 16)[i]: the high word
  of the 128-bit product, a uniform map onto [0, R).
* the rows hold the library's Q4 block format (``moe.dequantize``).
"""
from __future__ import annotations

import numpy as np

from . import moe

MASK64 = (1 << 64) - 1
G = 0x9E3779B97F4A7C15
SLOTS = 16


def mix64(z: int) -> int:
    z &= MASK64
    z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & MASK64
    z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & MASK64
    return z ^ (z >> 31)


def splitmix64(state: int, n: int) -> list[int]:
    """The first ``n`` outputs of SplitMix64 started at ``state``."""
    return [mix64(state + (i + 1) * G) for i in range(n)]


def ngram_hash(seed: int, a: int, b: int, c: int) -> int:
    h = splitmix64(seed, 1)[0]
    for v in (a, b, c):
        h = mix64(h ^ (int(v) & 0xFFFFFFFF))
    return h


def reduce_rows(x: int, R: int) -> int:
    """floor(x R / 2^64) for a 64-bit x."""
    return (x * R) >> 64


def token_rows(seed: int, ids, R: int) -> list[int]:
    """The 16 row indices of one token whose last three ids are ``ids``."""
    h = ngram_hash(seed, *ids)
    return [reduce_rows(x, R) for x in splitmix64(h, SLOTS)]


def rows(seed: int, ngrams: np.ndarray, R: int) -> np.ndarray:
    """int64 [T, 16] row indices for int32 ``ngrams`` [T, 3] (pure-Python loops)."""
    ngrams = np.asarray(ngrams)
    return np.array([token_rows(seed, ngrams[t], R) for t in range(ngrams.shape[0])], dtype=np.int64)


def gather(codes: np.ndarray, scales: np.ndarray, row_idx: np.ndarray) -> np.ndarray:
    """float64 [..., D] dequantised rows ``row_idx`` of a Q4 table (codes uint8
    [R, D/2], scales uint16 [R, D/32, 2])."""
    r = np.asarray(row_idx).reshape(-1)
    w = moe.dequantize(np.asarray(codes)[r], np.asarray(scales)[r], 4)
    return w.reshape(np.asarray(row_idx).shape + (w.shape[-1],))
