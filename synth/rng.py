"""SplitMix64 used as a counter-based generator.

SplitMix64 (Steele, Lea & Flood, "Fast splittable pseudorandom number
generators", OOPSLA 2014; the 64-bit finaliser is Stafford's "Mix13") keeps a
64-bit state that advances by the golden-ratio increment and returns a mixed
copy of it.  Output ``i`` of a stream started at state ``key`` is therefore a
pure function of ``(key, i)``:

    out(key, i) = mix64(key + (i + 1) * GAMMA)      (mod 2**64)

which lets the host and the GPU draw any element independently.  The device
side (``synth/csrc/synth_fill.cu``) implements the same definition.

Stream keys fold the identifying words of a tensor into one 64-bit key:

    k = mix64(seed XOR KEY0)
    for w in words: k = mix64(k XOR ((w + 1) * GAMMA))
"""
from __future__ import annotations

import numpy as np

MASK64 = (1 << 64) - 1
GAMMA = 0x9E3779B97F4A7C15
MUL1 = 0xBF58476D1CE4E5B9
MUL2 = 0x94D049BB133111EB
KEY0 = 0x6A09E667F3BCC909  # first 64 fractional bits of sqrt(2)

_G = np.uint64(GAMMA)
_M1 = np.uint64(MUL1)
_M2 = np.uint64(MUL2)


def mix64(z: int) -> int:
    """Stafford Mix13 finaliser on a Python int (mod 2**64)."""
    z &= MASK64
    z = ((z ^ (z >> 30)) * MUL1) & MASK64
    z = ((z ^ (z >> 27)) * MUL2) & MASK64
    return z ^ (z >> 31)


def mix64_np(z: np.ndarray) -> np.ndarray:
    """Vectorised Mix13 on a uint64 array (wrapping arithmetic)."""
    z = z.astype(np.uint64, copy=True)
    with np.errstate(over="ignore"):
        z ^= z >> np.uint64(30)
        z *= _M1
        z ^= z >> np.uint64(27)
        z *= _M2
        z ^= z >> np.uint64(31)
    return z


def stream_key(seed: int, *words: int) -> int:
    """64-bit key of the stream named by ``(seed, *words)``."""
    k = mix64((seed & MASK64) ^ KEY0)
    for w in words:
        k = mix64(k ^ (((w + 1) * GAMMA) & MASK64))
    return k


def outputs(key: int, start: int, count: int) -> np.ndarray:
    """``out(key, i)`` for ``i`` in ``[start, start + count)`` as uint64."""
    i = np.arange(start + 1, start + count + 1, dtype=np.uint64)
    with np.errstate(over="ignore"):
        state = np.uint64(key & MASK64) + i * _G
    return mix64_np(state)


def uniform53(r: np.ndarray) -> np.ndarray:
    """Map uint64 outputs to float64 in [0, 1): (r >> 11) * 2**-53 (exact)."""
    return (r >> np.uint64(11)).astype(np.float64) * (2.0 ** -53)


def sequential(seed_state: int, n: int) -> list[int]:
    """The first ``n`` outputs of plain SplitMix64 started at ``seed_state``.

    Same numbers as ``outputs(seed_state, 0, n)``; kept as the textbook loop so
    the published test vectors can be checked against the generator's own
    definition.
    """
    s = seed_state & MASK64
    res = []
    for _ in range(n):
        s = (s + GAMMA) & MASK64
        res.append(mix64(s))
    return res
