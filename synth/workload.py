"""Put a synthetic workload on the GPU: device-filled weights packed by libqmoe,
host-drawn router weights / biases / activations uploaded.

Glue between the generator (``synth``) and the library's public API; it holds
none of the method's arithmetic.
"""
from __future__ import annotations

import numpy as np
import torch

from . import device, gen
from .configs import Config


def device_layers(seed: int, cfg: Config, n_layers: int | None = None, dev="cuda", first: int = 0):
    """Packed expert layers, fp32 routers and biases of layers first .. first+n-1."""
    from quantised_expert_decode_b200.model import PackedLayer

    n = cfg.L if n_layers is None else n_layers
    canon, canon_fmt = None, None
    layers, routers, biases = [], [], []
    for l in range(first, first + n):
        lc = cfg.for_layer(l)
        if canon_fmt != lc.fmt:   # the canonical code buffers depend on the format
            canon, canon_fmt = device.alloc_canonical(lc, dev), lc.fmt
        device.fill_layer(seed, cfg, l, canon)
        layers.append(PackedLayer(lc.fmt, cfg.E, cfg.H, cfg.I, dev).pack(canon))
        routers.append(torch.from_numpy(gen.router(seed, cfg, l)).to(dev))
        b = gen.bias(seed, cfg, l)
        biases.append(None if b is None else torch.from_numpy(b).to(dev))
    torch.cuda.synchronize()
    del canon
    return layers, routers, (biases if cfg.bias else None)


def device_tokens(seed: int, cfg: Config, step: int = 0, dev="cuda", T: int | None = None):
    """Step activations on the device: fp32 [T,H] or bf16 [T,H]."""
    x = gen.tokens(seed, cfg, step, T)
    if cfg.x_kind == "bf16":
        return torch.from_numpy(x.view(np.int16)).to(dev).view(torch.bfloat16)
    return torch.from_numpy(x).to(dev)
