"""Packed expert layers and the captured layer stack, on top of the C ABI.

Convenience objects that own torch device buffers and call libqmoe; every
step of the computation runs in the library's kernels.
"""
from __future__ import annotations

import ctypes

import torch

from . import _lib as L


class PackedLayer:
    """One layer's experts in the packed device layout (qmoe_pack)."""

    def __init__(self, fmt: int, E: int, H: int, I: int, device="cuda"):
        self.fmt, self.E, self.H, self.I = fmt, E, H, I
        self.gate_up = torch.empty(L.qmoe_packed_bytes(fmt, L.GATE_UP, E, H, I), dtype=torch.uint8, device=device)
        self.down = torch.empty(L.qmoe_packed_bytes(fmt, L.DOWN, E, H, I), dtype=torch.uint8, device=device)

    @property
    def nbytes(self) -> int:
        return self.gate_up.numel() + self.down.numel()

    def pack(self, canon: dict, stream=None) -> "PackedLayer":
        """Pack canonical tensors (gate/up/down _codes uint8 and _scales uint16)."""
        L.qmoe_pack(self.fmt, L.GATE_UP, self.E, self.H, self.I, canon["gate_codes"], canon["gate_scales"],
                    canon["up_codes"], canon["up_scales"], self.gate_up, stream)
        L.qmoe_pack(self.fmt, L.DOWN, self.E, self.H, self.I, canon["down_codes"], canon["down_scales"],
                    None, None, self.down, stream)
        return self

    def handle(self) -> L.qmoe_experts:
        return L.qmoe_experts(self.E, self.H, self.I, self.fmt, self.gate_up.data_ptr(), self.down.data_ptr(),
                              self.gate_up.numel(), self.down.numel())


class DecodeStack:
    """L layers of route -> FFN -> residual RMSNorm as one CUDA graph."""

    def __init__(self, layers, routers, biases, T: int, k: int, eps: float, stream=None, timing: bool = False,
                 layerwise: bool = False):
        self.layers, self.routers, self.biases = list(layers), list(routers), biases
        self.L, self.T, self.k = len(self.layers), T, k
        self.H = self.layers[0].H
        self._handles = (L.qmoe_experts * self.L)(*[l.handle() for l in self.layers])
        self._wr = (ctypes.c_void_p * self.L)(*[w.data_ptr() for w in self.routers])
        if biases is not None:
            self._bias = (ctypes.c_void_p * self.L)(*[None if b is None else b.data_ptr() for b in biases])
        else:
            self._bias = None
        self.desc = L.qmoe_stack_desc(self.L, T, k, eps, self._wr, self._bias, self._handles,
                                      (L.STACK_TIMING if timing else 0) | (L.STACK_LAYERWISE if layerwise else 0))
        nbytes = L.qmoe_stack_workspace_bytes(self.desc)
        if nbytes == 0:
            raise L.QmoeError("qmoe_stack_workspace_bytes", 1)
        dev = self.routers[0].device
        self.workspace = torch.zeros(nbytes, dtype=torch.uint8, device=dev)
        self.handle = L.qmoe_stack_create(self.desc, self.workspace, stream)
        bufs = L.qmoe_stack_buffers(self.handle)
        base = self.workspace.data_ptr()

        def view(ptr, n, dtype):
            off = ptr - base
            esz = torch.tensor([], dtype=dtype).element_size()
            return self.workspace[off:off + n * esz].view(dtype)

        TH = T * self.H
        self.x_in = view(bufs["x_in"], TH, torch.float32).view(T, self.H)
        self.x_out = view(bufs["x_out"], TH, torch.float32).view(T, self.H)
        self.idx = view(bufs["idx"], self.L * T * k, torch.int32).view(self.L, T, k)
        self.gate = view(bufs["gate"], self.L * T * k, torch.float32).view(self.L, T, k)
        self.dev_status = view(bufs["dev_status"], 1, torch.int32)
        self.kernels_per_replay = L.qmoe_stack_kernels_per_replay(self.handle)
        self.path = L.qmoe_stack_path(self.handle)

    def decode(self, stream=None) -> None:
        L.qmoe_stack_decode(self.handle, stream)

    def decode_host(self, x_host, x_out_host, stream=None) -> None:
        L.qmoe_stack_decode_host(self.handle, x_host, x_out_host, stream)

    def layer_times(self):
        """(route_ms, ffn_ms) per layer of the last completed replay (timing stacks)."""
        return L.qmoe_stack_layer_times(self.handle, self.L)

    def phase_trace(self):
        """Per-layer phase stamps of the last replay (fused timing stacks):
        int64 SM cycles [L, CTAs, points]."""
        return L.qmoe_stack_trace(self.handle, self.L)

    def status(self) -> int:
        return L.qmoe_read_status(self.dev_status)

    def close(self) -> None:
        if getattr(self, "handle", None):
            L.qmoe_stack_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass
