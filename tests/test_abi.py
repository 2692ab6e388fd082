"""The C-ABI library loads and exports what include/qmoe.h declares; host-side
argument checks refuse bad calls before any GPU work (no GPU needed)."""
import ctypes
import os
import re

import pytest

from tests.conftest import ROOT

import quantised_expert_decode_b200 as q
from quantised_expert_decode_b200 import _lib as L


def _declared():
    with open(os.path.join(ROOT, "include", "qmoe.h")) as f:
        text = f.read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    names = set(re.findall(r"\b(qmoe_[a-z_0-9]+)\s*\(", text))
    return sorted(names)


def test_library_exports_every_declared_symbol():
    lib = q.lib()
    declared = _declared()
    assert len(declared) >= 18
    for name in declared:
        assert hasattr(lib, name), name
    assert set(declared) == set(L.exported_symbols())


def test_synth_library_exports():
    from synth import device
    h = device.lib()
    assert hasattr(h, "synth_fill_codes") and hasattr(h, "synth_fill_scales")


def test_packed_sizes_equal_canonical_sizes():
    E, H, I = 512, 2048, 768
    for fmt, bpb in ((L.Q2, 12), (L.Q4, 20)):
        total = q.qmoe_packed_bytes(fmt, L.GATE_UP, E, H, I) + q.qmoe_packed_bytes(fmt, L.DOWN, E, H, I)
        assert total == E * 3 * H * I // 32 * bpb
    assert q.qmoe_packed_bytes(3, L.GATE_UP, E, H, I) == 0


def test_workspace_sizes():
    assert q.qmoe_decode_workspace_bytes(1, 10, 2048, 768) >= 256 + 10 * 2 * 768 * 4 + 10 * 2048 * 4
    assert q.qmoe_route_workspace_bytes(1, 512) >= 512 * 8
    assert q.qmoe_route_workspace_bytes(0, 512) == 0


FAKE = 1 << 20  # aligned non-null address; never dereferenced by the host checks below


def test_route_argument_checks_without_gpu():
    lib = q.lib()
    ws = q.qmoe_route_workspace_bytes(1, 512)
    args = dict(Wr=FAKE, bias=None, x=FAKE, dt=L.F32, T=1, H=2048, E=512, k=10, idx=FAKE, gate=FAKE, ws=FAKE,
                wsb=ws, st=FAKE, stream=None)

    def call(**kw):
        a = dict(args, **kw)
        return lib.qmoe_route(a["Wr"], a["bias"], a["x"], a["dt"], a["T"], a["H"], a["E"], a["k"], a["idx"],
                              a["gate"], a["ws"], a["wsb"], a["st"], a["stream"])

    assert call(Wr=None) == 1
    assert call(x=FAKE + 4) == 1              # misaligned
    assert call(k=17) == 3
    assert call(k=600) == 3
    assert call(H=2000) == 1 or call(H=2000) == 3
    assert call(E=2048) == 3
    assert call(wsb=ws - 1) == 4
    assert call(dt=7) == 1


def test_ffn_decode_argument_checks_without_gpu():
    lib = q.lib()
    def ex_(E, H, I, fmt, gu, dn):
        return L.qmoe_experts(E, H, I, fmt, gu, dn, q.qmoe_packed_bytes(fmt, 0, E, H, I),
                              q.qmoe_packed_bytes(fmt, 1, E, H, I))
    ex = ex_(512, 2048, 768, L.Q2, FAKE, FAKE)
    wsb = q.qmoe_decode_workspace_bytes(1, 10, 2048, 768)

    def call(ex=ex, T=1, k=10, wsb=wsb, x=FAKE):
        return lib.qmoe_ffn_decode(ctypes.byref(ex), x, T, FAKE, FAKE, k, FAKE, FAKE, wsb, FAKE, None)

    assert call(T=9) == 3
    assert call(T=0) == 3
    assert call(k=17) == 3
    assert call(wsb=wsb - 16) == 4
    assert call(x=None) == 1
    assert call(ex=ex_(512, 2000, 768, L.Q2, FAKE, FAKE)) == 2
    assert call(ex=ex_(512, 2048, 768, 3, FAKE, FAKE)) == 2
    assert call(ex=ex_(512, 2048, 768, L.Q2, None, FAKE)) == 1
    bad = ex_(512, 2048, 768, L.Q2, FAKE, FAKE)
    bad.H = 1024                                    # sizes no longer match the geometry
    assert call(ex=bad) == 2


def test_prefill_argument_checks_without_gpu():
    lib = q.lib()
    def ex_(E, H, I, fmt, gu=FAKE, dn=FAKE):
        return L.qmoe_experts(E, H, I, fmt, gu, dn, q.qmoe_packed_bytes(fmt, 0, E, H, I),
                              q.qmoe_packed_bytes(fmt, 1, E, H, I))
    T, k = 4096, 10
    ex = ex_(512, 2048, 768, L.Q4)
    wsb = q.qmoe_prefill_workspace_bytes(T, k, 512, 2048, 768)
    # h rows (T*k + 15*E) x I bf16 dominate the workspace
    assert wsb >= (T * k + 15 * 512) * 768 * 2
    assert q.qmoe_prefill_workspace_bytes(0, k, 512, 2048, 768) == 0

    def call(ex=ex, T=T, k=k, wsb=wsb, x=FAKE, idx=FAKE, y=FAKE):
        return lib.qmoe_ffn_prefill(ctypes.byref(ex), x, T, idx, FAKE, k, y, FAKE, wsb, FAKE, None)

    assert call(x=None) == 1
    assert call(T=0) == 1
    assert call(x=FAKE + 8) == 1                            # bf16 rows must be 16-byte aligned
    assert call(idx=FAKE + 2) == 1
    assert call(ex=ex_(512, 2048, 768, L.Q2)) == 3          # Q2 prefill is not built
    assert call(ex=ex_(512, 2048 + 128, 768, L.Q4)) == 3    # H must be a multiple of 256
    assert call(k=600) == 3
    assert call(wsb=wsb - 256) == 4
    bad = ex_(512, 2048, 768, L.Q4)
    bad.I = 640                                             # sizes no longer match the geometry
    assert call(ex=bad) == 2


def test_bucket_argument_checks_without_gpu():
    lib = q.lib()
    ws = lib.qmoe_bucket_workspace_bytes(8, 2, 16)
    assert ws >= 16 * 4 and lib.qmoe_bucket_workspace_bytes(0, 2, 16) == 0
    # the table holds one row of E counts per CTA; CTAs cover at least 64 tokens each, 148 at most
    assert lib.qmoe_bucket_workspace_bytes(4096, 10, 512) >= 64 * 512 * 4
    assert lib.qmoe_bucket_workspace_bytes(1 << 20, 1, 1024) >= 148 * 1024 * 4
    assert lib.qmoe_bucket(None, 8, 2, 16, FAKE, FAKE, None, None, FAKE, ws, FAKE, None) == 1
    assert lib.qmoe_bucket(FAKE, 0, 2, 16, FAKE, FAKE, None, None, FAKE, ws, FAKE, None) == 1
    assert lib.qmoe_bucket(FAKE, 8, 2, 4096, FAKE, FAKE, None, None, FAKE, ws, FAKE, None) == 3
    assert lib.qmoe_bucket(FAKE + 2, 8, 2, 16, FAKE, FAKE, None, None, FAKE, ws, FAKE, None) == 1
    assert lib.qmoe_bucket(FAKE, 8, 2, 16, FAKE, FAKE, None, None, None, ws, FAKE, None) == 1
    assert lib.qmoe_bucket(FAKE, 8, 2, 16, FAKE, FAKE, None, None, FAKE + 4, ws, FAKE, None) == 1
    assert lib.qmoe_bucket(FAKE, 8, 2, 16, FAKE, FAKE, None, None, FAKE, ws - 4, FAKE, None) == 4


def test_pack_and_norm_argument_checks_without_gpu():
    lib = q.lib()
    assert lib.qmoe_pack(3, 0, 4, 256, 128, FAKE, FAKE, FAKE, FAKE, FAKE, 1 << 30, None) == 3
    assert lib.qmoe_pack(2, 0, 4, 250, 128, FAKE, FAKE, FAKE, FAKE, FAKE, 1 << 30, None) == 3
    assert lib.qmoe_pack(2, 0, 4, 256, 128, FAKE, FAKE, None, FAKE, FAKE, 1 << 30, None) == 1
    assert lib.qmoe_pack(2, 1, 4, 256, 128, FAKE, FAKE, None, None, FAKE, 16, None) == 1
    assert lib.qmoe_rmsnorm_residual(None, FAKE, ctypes.c_float(1e-6), FAKE, 1, 256, None) == 1
    assert lib.qmoe_residual_route(FAKE, FAKE, ctypes.c_float(1e-6), FAKE, FAKE, None, 1, 256, 64, 4,
                                   FAKE, FAKE, FAKE, 1 << 20, FAKE, None) == 1   # x_out aliases x_in


def test_stack_descriptor_checks_without_gpu():
    lib = q.lib()
    def ex_(E, H, I):
        return L.qmoe_experts(E, H, I, 2, FAKE, FAKE, q.qmoe_packed_bytes(2, 0, E, H, I),
                              q.qmoe_packed_bytes(2, 1, E, H, I))
    h = (L.qmoe_experts * 2)(ex_(64, 256, 128), ex_(64, 512, 128))
    wr = (ctypes.c_void_p * 2)(FAKE, FAKE)
    d = L.qmoe_stack_desc(2, 1, 4, 1e-6, wr, None, h)
    assert lib.qmoe_stack_workspace_bytes(ctypes.byref(d)) == 0     # mixed geometry refused
    h[1] = ex_(64, 256, 128)
    assert lib.qmoe_stack_workspace_bytes(ctypes.byref(d)) > 0
    h[1].down_bytes -= 16                                             # buffer size disagrees
    assert lib.qmoe_stack_workspace_bytes(ctypes.byref(d)) == 0
    h[1] = ex_(64, 256, 128)
    out = ctypes.c_void_p()
    assert lib.qmoe_stack_create(ctypes.byref(d), FAKE, 16, None, ctypes.byref(out)) == 4
    # layers of different block formats form one stack (mixed-bit)
    uniform = lib.qmoe_stack_workspace_bytes(ctypes.byref(d))
    h[1] = L.qmoe_experts(64, 256, 128, 4, FAKE, FAKE, q.qmoe_packed_bytes(4, 0, 64, 256, 128),
                          q.qmoe_packed_bytes(4, 1, 64, 256, 128))
    assert lib.qmoe_stack_workspace_bytes(ctypes.byref(d)) > 0
    h[1].down_bytes = q.qmoe_packed_bytes(2, 1, 64, 256, 128)          # Q2 size under a Q4 handle
    assert lib.qmoe_stack_workspace_bytes(ctypes.byref(d)) == 0
    h[1] = L.qmoe_experts(64, 256, 128, 3, FAKE, FAKE, 0, 0)             # no such format
    assert lib.qmoe_stack_workspace_bytes(ctypes.byref(d)) == 0
    assert lib.qmoe_stack_create(ctypes.byref(d), FAKE, uniform, None, ctypes.byref(out)) == 3


def test_ngram_gather_argument_checks_without_gpu():
    lib = q.lib()
    def call(ng=FAKE, T=2, codes=FAKE, scales=FAKE, R=4, D=32, out=FAKE, rows=None):
        return lib.qmoe_ngram_gather(ng, T, 0, codes, scales, R, D, out, rows, None)
    assert call(D=48) == 3 and call(D=0) == 3 and call(D=8192 + 32) == 3     # D outside the limits
    assert call(R=0) == 1 and call(R=2**31) == 1                              # table size
    assert call(T=0) == 1                                                     # no tokens
    assert call(codes=FAKE + 4) == 1 and call(out=FAKE + 8) == 1              # 16-byte alignment
    assert call(ng=FAKE + 2) == 1 and call(rows=FAKE + 1) == 1                # 4-byte alignment
    assert call(ng=None) == 1 and call(scales=None) == 1 and call(out=None) == 1


def test_status_strings():
    assert q.qmoe_status_string(0) == "ok"
    assert "geometry" in q.qmoe_status_string(2)
    assert q.qmoe_launch_count() >= 0


def test_binding_fails_loudly_without_library(monkeypatch, tmp_path):
    monkeypatch.setattr(L, "_lib", None)
    monkeypatch.setattr(L, "LIB_PATH", str(tmp_path / "missing.so"))
    with pytest.raises(RuntimeError, match="no CPU fallback"):
        L.lib()
