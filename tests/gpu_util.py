"""Helpers for the GPU parity tests: run the library's calls on device tensors."""
from __future__ import annotations

import numpy as np
import torch

import quantised_expert_decode_b200 as q
from quantised_expert_decode_b200 import _lib as L

DECODE_TOL = 1e-4     # rel-RMS bound for fp32-activation decode
GATE_TOL = 2e-6       # absolute bound on gate values (fp32 exp of float64 logit gaps)


def status_word():
    return torch.zeros(1, dtype=torch.int32, device="cuda")


def route(Wr, bias, x, k, dtype=L.F32):
    T, H = x.shape
    E = Wr.shape[0]
    idx = torch.empty((T, k), dtype=torch.int32, device="cuda")
    gate = torch.empty((T, k), dtype=torch.float32, device="cuda")
    ws = torch.zeros(q.qmoe_route_workspace_bytes(T, E), dtype=torch.uint8, device="cuda")
    st = status_word()
    q.qmoe_route(Wr, bias, x, dtype, T, H, E, k, idx, gate, ws, st)
    torch.cuda.synchronize()
    assert q.qmoe_read_status(st) == 0
    return idx, gate


def ffn(layer, x, idx, gate, k, ws=None, st=None, check=True):
    T, H = x.shape
    y = torch.full((T, H), float("nan"), dtype=torch.float32, device="cuda")
    if ws is None:
        ws = torch.zeros(q.qmoe_decode_workspace_bytes(T, k, layer.H, layer.I), dtype=torch.uint8, device="cuda")
    if st is None:
        st = status_word()
    q.qmoe_ffn_decode(layer.handle(), x, T, idx, gate, k, y, ws, st)
    torch.cuda.synchronize()
    if check:
        assert q.qmoe_read_status(st) == 0
    return y


def to_np(t):
    return t.detach().cpu().numpy()


def gap_report(l_row: np.ndarray, k: int) -> float:
    s = np.sort(l_row)[::-1]
    return float(np.min(s[:k] - s[1:k + 1]))
