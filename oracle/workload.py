"""Feed the synthetic workloads to the float64 oracle.

TEST INFRASTRUCTURE (see ``oracle/moe.py``).  Weights are regenerated on the
host from the seeded streams of ``synth`` and dequantised here; only the
experts a route actually selects are generated.
"""
from __future__ import annotations

import numpy as np

from synth import gen
from synth.configs import Config

from . import moe


class Layer:
    """One layer of a workload: router, optional bias, lazily built experts."""

    def __init__(self, seed: int, cfg: Config, layer: int):
        self.seed, self.cfg, self.layer = seed, cfg, layer
        self.Wr = gen.router(seed, cfg, layer)
        self.bias = gen.bias(seed, cfg, layer)
        self._cache = {}

    def expert(self, e: int):
        """float64 (Wg [I,H], Wu [I,H], Wd [H,I]) of expert ``e``."""
        if e not in self._cache:
            raw = gen.expert(self.seed, self.cfg, self.layer, e)
            bits = self.cfg.for_layer(self.layer).format.bits
            self._cache[e] = tuple(
                moe.dequantize(raw[n + "_codes"], raw[n + "_scales"], bits)
                for n in ("gate", "up", "down"))
        return self._cache[e]

    def drop(self):
        self._cache.clear()


def x_float(seed: int, cfg: Config, step: int = 0, T: int | None = None) -> np.ndarray:
    """Step activations as float64 (bf16 inputs converted exactly)."""
    x = gen.tokens(seed, cfg, step, T)
    if cfg.x_kind == "bf16":
        x = gen.bf16_bits_to_f32(x)
    return x.astype(np.float64)


def run_layer(seed: int, cfg: Config, x: np.ndarray, layer: int = 0):
    """Route + FFN + combine of one layer on activations ``x`` [T, H].

    Returns (y float64 [T,H], idx int32 [T,k], gate float64 [T,k], logits).
    """
    L = Layer(seed, cfg, layer)
    idx, g, l = moe.route(x, L.Wr, L.bias, cfg.k)
    y = moe.moe_layer(x, idx, g, L.expert)
    return y, idx, g, l


def run_stack(seed: int, cfg: Config, x0: np.ndarray, n_layers: int | None = None):
    """Residual stack over the first ``n_layers`` layers (all by default).

    Returns the final activations and per-layer (x_in, idx, gate, y), as
    ``moe.stack`` computes them on the generated layers. Experts of a finished
    layer are dropped to bound host memory.
    """
    n = cfg.L if n_layers is None else n_layers

    def layers():
        for l in range(n):
            L = Layer(seed, cfg, l)
            yield L.Wr, L.bias, L.expert
            L.drop()
    return moe.stack(x0, layers(), cfg.k, cfg.eps, residual=cfg.residual)
