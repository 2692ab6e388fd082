"""GPU fill of the seeded code and scale streams (libqmoe_synth.so).

Same streams as ``synth.gen`` (bit-identical; checked by the GPU tests), so the
tens of gigabytes of expert weights never cross PCIe. Gaussians (router,
bias, activations) are generated on the host by ``synth.gen`` and uploaded.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

from . import gen, rng
from .configs import BLOCK, DOWN, GATE, UP, WHAT_CODES, WHAT_SCALES, Config

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libqmoe_synth.so")
_lib = None


def lib():
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: run `python quantised_expert_decode_b200/build.py`")
        h = ctypes.CDLL(LIB_PATH)
        h.synth_fill_codes.restype = ctypes.c_int
        h.synth_fill_codes.argtypes = [ctypes.c_uint64, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                       ctypes.c_int, ctypes.c_size_t, ctypes.c_void_p, ctypes.c_void_p]
        h.synth_fill_scales.restype = ctypes.c_int
        h.synth_fill_scales.argtypes = [ctypes.c_uint64, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                        ctypes.c_int, ctypes.c_size_t, ctypes.c_double, ctypes.c_double,
                                        ctypes.c_double, ctypes.c_void_p, ctypes.c_void_p]
        _lib = h
    return _lib


def _stream():
    import torch
    return torch.cuda.current_stream().cuda_stream


def fill_codes(seed: int, cfg: Config, layer: int, mat: int, dst, e0: int = 0) -> None:
    """dst: uint8 tensor [E, rows, K*bits/8] (experts e0 .. e0+E-1)."""
    E = dst.shape[0]
    per = dst[0].numel()
    rc = lib().synth_fill_codes(seed & rng.MASK64, cfg.cid, layer, e0, E, WHAT_CODES[mat], per, dst.data_ptr(),
                                _stream())
    if rc:
        raise RuntimeError(f"synth_fill_codes failed ({rc})")


def fill_scales(seed: int, cfg: Config, layer: int, mat: int, dst, e0: int = 0) -> None:
    """dst: uint16 tensor [E, rows, K/32, 2] (fp16 bit patterns of (d, m))."""
    f = cfg.for_layer(layer).format
    E = dst.shape[0]
    nblk = dst[0].numel() // 2
    rc = lib().synth_fill_scales(seed & rng.MASK64, cfg.cid, layer, e0, E, WHAT_SCALES[mat], nblk,
                                 float(np.float64(f.d_lo)), float(f.d_hi - f.d_lo), float(f.m_coef),
                                 dst.data_ptr(), _stream())
    if rc:
        raise RuntimeError(f"synth_fill_scales failed ({rc})")


def alloc_canonical(cfg: Config, device="cuda", E: int | None = None) -> dict:
    """Empty canonical buffers for one layer (or E experts of it)."""
    import torch
    E = cfg.E if E is None else E
    bits = cfg.format.bits
    out = {}
    for mat, name in ((GATE, "gate"), (UP, "up"), (DOWN, "down")):
        rows, K = gen.matrix_shape(cfg, mat)
        out[name + "_codes"] = torch.empty((E, rows, K * bits // 8), dtype=torch.uint8, device=device)
        out[name + "_scales"] = torch.empty((E, rows, K // BLOCK, 2), dtype=torch.int16, device=device)
    return out


def fill_layer(seed: int, cfg: Config, layer: int, bufs: dict, e0: int = 0) -> dict:
    """Fill canonical buffers with layer ``layer``'s experts e0 ..."""
    for mat, name in ((GATE, "gate"), (UP, "up"), (DOWN, "down")):
        fill_codes(seed, cfg, layer, mat, bufs[name + "_codes"], e0)
        fill_scales(seed, cfg, layer, mat, bufs[name + "_scales"], e0)
    return bufs


def ngram_table(seed: int, ncfg, layer: int = 0, device="cuda", R: int | None = None) -> tuple:
    """Device codes uint8 [R, D/2] and scales int16 [R, D/32, 2] of an n-gram
    row table (same bytes as ``gen.ngram_rows``)."""
    import torch
    from .configs import WHAT_NGRAM_CODES, WHAT_NGRAM_SCALES
    R = ncfg.R if R is None else R
    D, f = ncfg.D, ncfg.format
    codes = torch.empty((R, D * f.bits // 8), dtype=torch.uint8, device=device)
    scales = torch.empty((R, D // BLOCK, 2), dtype=torch.int16, device=device)
    rc = lib().synth_fill_codes(seed & rng.MASK64, ncfg.cid, layer, 0, R, WHAT_NGRAM_CODES, codes[0].numel(),
                                codes.data_ptr(), _stream())
    if rc:
        raise RuntimeError(f"synth_fill_codes failed ({rc})")
    rc = lib().synth_fill_scales(seed & rng.MASK64, ncfg.cid, layer, 0, R, WHAT_NGRAM_SCALES, D // BLOCK,
                                 float(np.float64(f.d_lo)), float(f.d_hi - f.d_lo), float(f.m_coef),
                                 scales.data_ptr(), _stream())
    if rc:
        raise RuntimeError(f"synth_fill_scales failed ({rc})")
    return codes, scales
