"""ctypes binding of libqmoe.so: the C ABI of include/qmoe.h under the same names.

Argument marshalling only. Tensor arguments are torch CUDA tensors (their data
pointers are passed); ``stream`` defaults to torch's current stream. A call
that returns a non-OK status raises :class:`QmoeError`. There is no fallback:
if the library is missing, importing this module's functions raises.
"""
from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libqmoe.so")

OK = 0
Q2, Q4 = 2, 4
F32, BF16 = 0, 1
GATE_UP, DOWN = 0, 1
STACK_TIMING = 1
STACK_LAYERWISE = 2
PATH_LAYERWISE, PATH_FUSED = 0, 1

STATUS_NAMES = {0: "OK", 1: "INVALID_ARG", 2: "GEOMETRY", 3: "UNSUPPORTED", 4: "WORKSPACE",
                5: "CUDA", 6: "TIMEOUT", 7: "DEVICE_STATUS", 8: "RANGE"}


class QmoeError(RuntimeError):
    def __init__(self, fn: str, code: int):
        self.code = code
        super().__init__(f"{fn} failed: {STATUS_NAMES.get(code, code)}")


class qmoe_experts(ctypes.Structure):
    _fields_ = [("E", ctypes.c_int), ("H", ctypes.c_int), ("I", ctypes.c_int), ("fmt", ctypes.c_int),
                ("gate_up", ctypes.c_void_p), ("down", ctypes.c_void_p),
                ("gate_up_bytes", ctypes.c_size_t), ("down_bytes", ctypes.c_size_t)]


class qmoe_stack_desc(ctypes.Structure):
    _fields_ = [("L", ctypes.c_int), ("T", ctypes.c_int), ("k", ctypes.c_int), ("eps", ctypes.c_float),
                ("Wr", ctypes.POINTER(ctypes.c_void_p)), ("bias", ctypes.POINTER(ctypes.c_void_p)),
                ("layers", ctypes.POINTER(qmoe_experts)), ("flags", ctypes.c_int)]


_VP, _I, _SZ, _F = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t, ctypes.c_float
_SIGS = {
    "qmoe_packed_bytes": (_SZ, [_I, _I, _I, _I, _I]),
    "qmoe_pack": (_I, [_I, _I, _I, _I, _I, _VP, _VP, _VP, _VP, _VP, _SZ, _VP]),
    "qmoe_route_workspace_bytes": (_SZ, [_I, _I]),
    "qmoe_route": (_I, [_VP, _VP, _VP, _I, _I, _I, _I, _I, _VP, _VP, _VP, _SZ, _VP, _VP]),
    "qmoe_route_fixed": (_I, [_VP, _VP, _VP, _I, _I, _I, _I, _VP, _VP, _VP, _VP]),
    "qmoe_residual_route": (_I, [_VP, _VP, _F, _VP, _VP, _VP, _I, _I, _I, _I, _VP, _VP, _VP, _SZ, _VP, _VP]),
    "qmoe_rmsnorm_residual": (_I, [_VP, _VP, _F, _VP, _I, _I, _VP]),
    "qmoe_decode_workspace_bytes": (_SZ, [_I, _I, _I, _I]),
    "qmoe_ffn_decode": (_I, [ctypes.POINTER(qmoe_experts), _VP, _I, _VP, _VP, _I, _VP, _VP, _SZ, _VP, _VP]),
    "qmoe_bucket_workspace_bytes": (_SZ, [_I, _I, _I]),
    "qmoe_bucket": (_I, [_VP, _I, _I, _I, _VP, _VP, _VP, _VP, _VP, _SZ, _VP, _VP]),
    "qmoe_prefill_workspace_bytes": (_SZ, [_I, _I, _I, _I, _I]),
    "qmoe_ffn_prefill": (_I, [ctypes.POINTER(qmoe_experts), _VP, _I, _VP, _VP, _I, _VP, _VP, _SZ, _VP, _VP]),
    "qmoe_ffn_prefill_timed": (_I, [ctypes.POINTER(qmoe_experts), _VP, _I, _VP, _VP, _I, _VP, _VP, _SZ, _VP, _VP,
                                    ctypes.POINTER(_VP), _I]),
    "qmoe_stack_workspace_bytes": (_SZ, [ctypes.POINTER(qmoe_stack_desc)]),
    "qmoe_stack_create": (_I, [ctypes.POINTER(qmoe_stack_desc), _VP, _SZ, _VP, ctypes.POINTER(_VP)]),
    "qmoe_stack_destroy": (_I, [_VP]),
    "qmoe_stack_buffers": (_I, [_VP, ctypes.POINTER(_VP), ctypes.POINTER(_VP), ctypes.POINTER(_VP),
                                ctypes.POINTER(_VP), ctypes.POINTER(_VP)]),
    "qmoe_stack_barrier_word": (_VP, [_VP]),
    "qmoe_stack_trace": (_I, [_VP, _VP, _SZ, _VP, _VP]),
    "qmoe_stack_kernels_per_replay": (_I, [_VP]),
    "qmoe_stack_path": (_I, [_VP]),
    "qmoe_stack_decode": (_I, [_VP, _VP]),
    "qmoe_stack_layer_times": (_I, [_VP, _VP, _VP]),
    "qmoe_stack_decode_host": (_I, [_VP, _VP, _VP, _VP]),
    "qmoe_ngram_gather": (_I, [_VP, _I, ctypes.c_uint64, _VP, _VP, ctypes.c_int64, _I, _VP, _VP, _VP]),
    "qmoe_read_status": (_I, [_VP]),
    "qmoe_status_string": (ctypes.c_char_p, [_I]),
    "qmoe_launch_count": (ctypes.c_uint64, []),
}

_lib = None


def lib() -> ctypes.CDLL:
    """Load libqmoe.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                               "`python quantised_expert_decode_b200/build.py` (there is no CPU fallback)")
        h = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in _SIGS.items():
            f = getattr(h, name)
            f.restype = res
            f.argtypes = args
        _lib = h
    return _lib


def exported_symbols() -> list[str]:
    return list(_SIGS)


# ------------------------------------------------------------------ helpers --
def _p(t) -> int | None:
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _s(stream) -> int | None:
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _check(name: str, code: int) -> None:
    if code != OK:
        raise QmoeError(name, code)


# ---------------------------------------------------------------- the ABI --
def qmoe_packed_bytes(fmt: int, kind: int, E: int, H: int, I: int) -> int:
    return lib().qmoe_packed_bytes(fmt, kind, E, H, I)


def qmoe_pack(fmt, kind, E, H, I, codes_a, scales_a, codes_up, scales_up, dst, stream=None) -> None:
    _check("qmoe_pack", lib().qmoe_pack(fmt, kind, E, H, I, _p(codes_a), _p(scales_a), _p(codes_up),
                                        _p(scales_up), _p(dst), dst.numel() * dst.element_size(), _s(stream)))


def qmoe_route_workspace_bytes(T: int, E: int) -> int:
    return lib().qmoe_route_workspace_bytes(T, E)


def qmoe_route(Wr, bias, x, x_dtype, T, H, E, k, idx, gate, workspace, dev_status, stream=None) -> None:
    _check("qmoe_route", lib().qmoe_route(_p(Wr), _p(bias), _p(x), x_dtype, T, H, E, k, _p(idx), _p(gate),
                                          _p(workspace), workspace.numel() * workspace.element_size(),
                                          _p(dev_status), _s(stream)))


def qmoe_route_fixed(Wr, bias, x, T, H, E, k, idx, gate, dev_status, stream=None) -> None:
    """The decode router with its scratch in a fixed device array (no workspace)."""
    _check("qmoe_route_fixed", lib().qmoe_route_fixed(_p(Wr), _p(bias), _p(x), T, H, E, k, _p(idx), _p(gate),
                                                      _p(dev_status), _s(stream)))


def qmoe_residual_route(x_in, y, eps, x_out, Wr, bias, T, H, E, k, idx, gate, workspace, dev_status,
                        stream=None) -> None:
    _check("qmoe_residual_route", lib().qmoe_residual_route(
        _p(x_in), _p(y), float(eps), _p(x_out), _p(Wr), _p(bias), T, H, E, k, _p(idx), _p(gate),
        _p(workspace), workspace.numel() * workspace.element_size(), _p(dev_status), _s(stream)))


def qmoe_rmsnorm_residual(x_in, y, eps, x_out, T, H, stream=None) -> None:
    _check("qmoe_rmsnorm_residual",
           lib().qmoe_rmsnorm_residual(_p(x_in), _p(y), float(eps), _p(x_out), T, H, _s(stream)))


def qmoe_decode_workspace_bytes(T: int, k: int, H: int, I: int) -> int:
    return lib().qmoe_decode_workspace_bytes(T, k, H, I)


def qmoe_ffn_decode(experts: qmoe_experts, x, T, idx, gate, k, y, workspace, dev_status, stream=None) -> None:
    _check("qmoe_ffn_decode", lib().qmoe_ffn_decode(
        ctypes.byref(experts), _p(x), T, _p(idx), _p(gate), k, _p(y), _p(workspace),
        workspace.numel() * workspace.element_size(), _p(dev_status), _s(stream)))


def qmoe_bucket_workspace_bytes(T: int, k: int, E: int) -> int:
    return lib().qmoe_bucket_workspace_bytes(T, k, E)


def qmoe_bucket(idx, T, k, E, offsets, perm, active, nactive, workspace, dev_status, stream=None) -> None:
    _check("qmoe_bucket", lib().qmoe_bucket(_p(idx), T, k, E, _p(offsets), _p(perm), _p(active), _p(nactive),
                                            _p(workspace), workspace.numel() * workspace.element_size(),
                                            _p(dev_status), _s(stream)))


def qmoe_prefill_workspace_bytes(T: int, k: int, E: int, H: int, I: int) -> int:
    return lib().qmoe_prefill_workspace_bytes(T, k, E, H, I)


def qmoe_ffn_prefill(experts: qmoe_experts, x, T, idx, gate, k, y, workspace, dev_status, stream=None) -> None:
    _check("qmoe_ffn_prefill", lib().qmoe_ffn_prefill(
        ctypes.byref(experts), _p(x), T, _p(idx), _p(gate), k, _p(y), _p(workspace),
        workspace.numel() * workspace.element_size(), _p(dev_status), _s(stream)))


def qmoe_ngram_gather(ngrams, T, seed, codes, scales, R, D, out, rows=None, stream=None) -> None:
    """``ngrams`` int32 [T, 3]; ``codes`` uint8 [R, D/2]; ``scales`` int16/uint16 [R, D/32, 2];
    ``out`` fp32 [T, 16, D]; ``rows`` int32 [T, 16] or None."""
    _check("qmoe_ngram_gather", lib().qmoe_ngram_gather(_p(ngrams), T, seed & ((1 << 64) - 1), _p(codes), _p(scales),
                                                        R, D, _p(out), _p(rows), _s(stream)))


PREFILL_ATOMIC_COMBINE = 1


def qmoe_ffn_prefill_timed(experts: qmoe_experts, x, T, idx, gate, k, y, workspace, dev_status, events,
                           stream=None, flags=0) -> None:
    """``events``: three torch.cuda.Event(enable_timing=True) objects."""
    for e in events:
        if not e.cuda_event:   # torch creates the CUDA event at its first record
            e.record()
    arr = (_VP * 3)(*[e.cuda_event for e in events])
    _check("qmoe_ffn_prefill_timed", lib().qmoe_ffn_prefill_timed(
        ctypes.byref(experts), _p(x), T, _p(idx), _p(gate), k, _p(y), _p(workspace),
        workspace.numel() * workspace.element_size(), _p(dev_status), _s(stream), arr, flags))


def qmoe_stack_workspace_bytes(desc: qmoe_stack_desc) -> int:
    return lib().qmoe_stack_workspace_bytes(ctypes.byref(desc))


def qmoe_stack_create(desc: qmoe_stack_desc, workspace, stream=None) -> int:
    out = ctypes.c_void_p()
    _check("qmoe_stack_create", lib().qmoe_stack_create(
        ctypes.byref(desc), _p(workspace), workspace.numel() * workspace.element_size(), _s(stream),
        ctypes.byref(out)))
    return out.value


def qmoe_stack_destroy(stack: int) -> None:
    _check("qmoe_stack_destroy", lib().qmoe_stack_destroy(stack))


def qmoe_stack_buffers(stack: int) -> dict:
    ptrs = [ctypes.c_void_p() for _ in range(5)]
    _check("qmoe_stack_buffers", lib().qmoe_stack_buffers(stack, *[ctypes.byref(p) for p in ptrs]))
    return dict(zip(("x_in", "x_out", "idx", "gate", "dev_status"), (p.value for p in ptrs)))


def qmoe_stack_kernels_per_replay(stack: int) -> int:
    return lib().qmoe_stack_kernels_per_replay(stack)


def qmoe_stack_trace(stack: int, L: int, max_ctas: int = 1024, points: int = 16):
    """Phase stamps (SM cycles) of the last replay: numpy int64 [L, ctas, points]."""
    import numpy as np
    buf = np.zeros(L * max_ctas * points, dtype=np.int64)
    g, p = ctypes.c_int(0), ctypes.c_int(0)
    _check("qmoe_stack_trace", lib().qmoe_stack_trace(stack, buf.ctypes.data, buf.size, ctypes.byref(g),
                                                      ctypes.byref(p)))
    return buf[:L * g.value * p.value].reshape(L, g.value, p.value)


def qmoe_stack_barrier_word(stack: int) -> int | None:
    return lib().qmoe_stack_barrier_word(stack)


def qmoe_stack_path(stack: int) -> int:
    return lib().qmoe_stack_path(stack)


def qmoe_stack_layer_times(stack: int, L: int):
    """(route_ms, ffn_ms) lists of the last completed replay of a timing stack."""
    r = (ctypes.c_float * L)()
    f = (ctypes.c_float * L)()
    _check("qmoe_stack_layer_times", lib().qmoe_stack_layer_times(stack, r, f))
    return list(r), list(f)


def qmoe_stack_decode(stack: int, stream=None) -> None:
    _check("qmoe_stack_decode", lib().qmoe_stack_decode(stack, _s(stream)))


def qmoe_stack_decode_host(stack: int, x_host, x_out_host, stream=None) -> None:
    _check("qmoe_stack_decode_host", lib().qmoe_stack_decode_host(stack, _p(x_host), _p(x_out_host), _s(stream)))


def qmoe_read_status(dev_status) -> int:
    return lib().qmoe_read_status(_p(dev_status))


def qmoe_status_string(code: int) -> str:
    return lib().qmoe_status_string(code).decode()


def qmoe_launch_count() -> int:
    return lib().qmoe_launch_count()
