"""Host generation of the synthetic workloads (canonical bytes + Gaussians).

Canonical (logical) layout of one expert matrix with ``rows`` outputs and
reduction length ``K`` (gate/up: rows = I, K = H; down: rows = H, K = I):

* codes  uint8  [rows, K*bits/8]; Q2 code j of a row sits in byte j//4 at bits
         2*(j%4); Q4 code j sits in byte j//2, low nibble for even j.
* scales uint16 [rows, K/32, 2] = fp16 bit patterns of (d, m) per block.

Codes are uniform i.i.d., so the code bytes are simply the little-endian
bytes of the stream ``out(codes_key, 0), out(codes_key, 1), ...``.

Scale ``d`` of block j (j = row * K/32 + block) is
``fp16_rne(lo + (hi - lo) * u_j)`` with ``u_j = (out(scales_key, j) >> 11) * 2**-53``
evaluated in float64 without fused multiply-add, and ``m = fp16_rne(-c * d)``
(c = 1.5 for Q2, 7.5 for Q4; the product is exact in float64).

Gaussians (router weights, biases, activations) are host-only: Box-Muller on
consecutive output pairs, ``u1 = ((r0 >> 11) + 1) * 2**-53`` in (0, 1],
``u2 = (r1 >> 11) * 2**-53``, ``z0 = sqrt(-2 ln u1) cos(2 pi u2)``,
``z1 = sqrt(-2 ln u1) sin(2 pi u2)``.
"""
from __future__ import annotations

import numpy as np

from . import rng
from .configs import (BLOCK, DOWN, GATE, UP, WHAT_BIAS, WHAT_CODES, WHAT_NGRAM_CODES, WHAT_NGRAM_IDS,
                      WHAT_NGRAM_SCALES, WHAT_NOISE, WHAT_ROUTER, WHAT_SCALES, WHAT_X, Config, FORMATS,
                      NgramConfig)


def matrix_shape(cfg: Config, mat: int) -> tuple[int, int]:
    """(rows, K) of an expert matrix: gate/up are [I, H], down is [H, I]."""
    return (cfg.I, cfg.H) if mat in (GATE, UP) else (cfg.H, cfg.I)


def codes_key(seed: int, cfg: Config, layer: int, expert: int, mat: int) -> int:
    return rng.stream_key(seed, cfg.cid, layer, expert, WHAT_CODES[mat])


def scales_key(seed: int, cfg: Config, layer: int, expert: int, mat: int) -> int:
    return rng.stream_key(seed, cfg.cid, layer, expert, WHAT_SCALES[mat])


def code_bytes(key: int, nbytes: int) -> np.ndarray:
    """Bytes ``[0, nbytes)`` of a code stream (nbytes a multiple of 8)."""
    assert nbytes % 8 == 0
    words = rng.outputs(key, 0, nbytes // 8)
    return words.astype("<u8").view(np.uint8)


def scale_pairs(key: int, nblocks: int, fmt: int) -> np.ndarray:
    """uint16 [nblocks, 2] fp16 bit patterns of (d, m)."""
    f = FORMATS[fmt]
    u = rng.uniform53(rng.outputs(key, 0, nblocks))
    d = np.float64(f.d_lo) + np.float64(f.d_hi - f.d_lo) * u
    d16 = d.astype(np.float16)
    m16 = (np.float64(-f.m_coef) * d16.astype(np.float64)).astype(np.float16)
    out = np.empty((nblocks, 2), dtype=np.uint16)
    out[:, 0] = d16.view(np.uint16)
    out[:, 1] = m16.view(np.uint16)
    return out


def expert_matrix(seed: int, cfg: Config, layer: int, expert: int, mat: int):
    """(codes uint8 [rows, K*bits/8], scales uint16 [rows, K/32, 2])."""
    cfg = cfg.for_layer(layer)
    rows, K = matrix_shape(cfg, mat)
    bits = cfg.format.bits
    codes = code_bytes(codes_key(seed, cfg, layer, expert, mat), rows * K * bits // 8)
    scales = scale_pairs(scales_key(seed, cfg, layer, expert, mat), rows * K // BLOCK, cfg.fmt)
    return codes.reshape(rows, K * bits // 8), scales.reshape(rows, K // BLOCK, 2)


def expert(seed: int, cfg: Config, layer: int, e: int) -> dict:
    """All three canonical matrices of expert ``e`` of ``layer``."""
    out = {}
    for mat, name in ((GATE, "gate"), (UP, "up"), (DOWN, "down")):
        c, s = expert_matrix(seed, cfg, layer, e, mat)
        out[name + "_codes"] = c
        out[name + "_scales"] = s
    return out


def gaussians(key: int, n: int) -> np.ndarray:
    """``n`` standard normals (float64) of stream ``key`` by Box-Muller."""
    npairs = (n + 1) // 2
    r = rng.outputs(key, 0, 2 * npairs)
    u1 = ((r[0::2] >> np.uint64(11)).astype(np.float64) + 1.0) * (2.0 ** -53)
    u2 = (r[1::2] >> np.uint64(11)).astype(np.float64) * (2.0 ** -53)
    rad = np.sqrt(-2.0 * np.log(u1))
    ang = 2.0 * np.pi * u2
    z = np.empty(2 * npairs, dtype=np.float64)
    z[0::2] = rad * np.cos(ang)
    z[1::2] = rad * np.sin(ang)
    return z[:n]


def router(seed: int, cfg: Config, layer: int) -> np.ndarray:
    """Router weight Wr [E, H] fp32 ~ N(0, router_std)."""
    z = gaussians(rng.stream_key(seed, cfg.cid, layer, 0, WHAT_ROUTER), cfg.E * cfg.H)
    return (cfg.router_std * z).astype(np.float32).reshape(cfg.E, cfg.H)


def bias(seed: int, cfg: Config, layer: int) -> np.ndarray | None:
    """Per-expert router logit bias [E] fp32 ~ N(0, 1), or None."""
    if not cfg.bias:
        return None
    z = gaussians(rng.stream_key(seed, cfg.cid, layer, 0, WHAT_BIAS), cfg.E)
    return z.astype(np.float32)


def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round-to-nearest-even fp32 -> bf16, returned as uint16 bit patterns."""
    b = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32).astype(np.uint64)
    b = (b + np.uint64(0x7FFF) + ((b >> np.uint64(16)) & np.uint64(1))) >> np.uint64(16)
    return b.astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (b.astype(np.uint32) << np.uint32(16)).view(np.float32)


def tokens(seed: int, cfg: Config, step: int = 0, T: int | None = None):
    """Activations of one step.

    Returns fp32 [T, H] for ``normal``/``correlated`` and uint16 bf16 bit
    patterns [T, H] for ``bf16``.  ``step`` selects an independent draw
    (benchmarks vary it so that routes change between iterations).
    """
    T = cfg.T if T is None else T
    H = cfg.H
    z = gaussians(rng.stream_key(seed, cfg.cid, step, 0, WHAT_X), T * H).reshape(T, H)
    if cfg.x_kind == "normal":
        return z.astype(np.float32)
    if cfg.x_kind == "correlated":
        n = gaussians(rng.stream_key(seed, cfg.cid, step, 0, WHAT_NOISE), T * H).reshape(T, H)
        x = np.empty((T, H), dtype=np.float64)
        x[0] = z[0]
        x[1:] = 0.8 * z[0][None, :] + 0.6 * n[1:]
        return x.astype(np.float32)
    if cfg.x_kind == "bf16":
        return f32_to_bf16_bits(z.astype(np.float32))
    raise ValueError(cfg.x_kind)


# ------------------------------------------------------- n-gram row tables --
def ngram_rows(seed: int, ncfg: NgramConfig, layer: int, rows) -> tuple[np.ndarray, np.ndarray]:
    """Canonical codes uint8 [n, D/2] and scales uint16 [n, D/32, 2] of table
    rows ``rows`` (row r is the stream pair keyed like expert r of an expert
    layer; the device fill draws the same bytes)."""
    rows = np.asarray(rows, dtype=np.int64).reshape(-1)
    D = ncfg.D
    codes = np.empty((len(rows), D * ncfg.format.bits // 8), dtype=np.uint8)
    scales = np.empty((len(rows), D // BLOCK, 2), dtype=np.uint16)
    for n, r in enumerate(rows):
        codes[n] = code_bytes(rng.stream_key(seed, ncfg.cid, layer, int(r), WHAT_NGRAM_CODES), codes.shape[1])
        scales[n] = scale_pairs(rng.stream_key(seed, ncfg.cid, layer, int(r), WHAT_NGRAM_SCALES), D // BLOCK,
                                ncfg.fmt).reshape(D // BLOCK, 2)
    return codes, scales


def ngram_ids(seed: int, ncfg: NgramConfig, step: int = 0, T: int | None = None) -> np.ndarray:
    """int32 [T, 3]: token t's ids (t-2, t-1, t) of a chunk of T + 2 ids drawn
    uniformly from the vocabulary (64-bit draws reduced by multiply-high)."""
    T = ncfg.T if T is None else T
    words = rng.outputs(rng.stream_key(seed, ncfg.cid, step, 0, WHAT_NGRAM_IDS), 0, T + 2)
    ids = np.array([(int(w) * ncfg.vocab) >> 64 for w in words], dtype=np.int32)
    return np.stack([ids[:-2], ids[1:-1], ids[2:]], axis=1)
