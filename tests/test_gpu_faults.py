"""Device-side failure detection without a GPU fault.

Every device wait of the decode kernels gives up after a bounded budget (about
one second of SM clocks), sets the caller's status word and returns. These
tests make a grid barrier run out on purpose: its counter is preset so that
some CTAs can never see it complete. The kernel must end on its own with
QMOE_ERR_TIMEOUT, and a fresh call afterwards must succeed and match the
oracle. Activations beyond the range of the exact router sums must be reported
as QMOE_ERR_RANGE, never read out of bounds."""
import numpy as np
import pytest
import torch

import quantised_expert_decode_b200 as q
from oracle import moe
from oracle import workload as W
from quantised_expert_decode_b200 import _lib as L
from quantised_expert_decode_b200.model import DecodeStack
from synth import configs, gen
from synth.workload import device_layers
from tests.gpu_util import DECODE_TOL, ffn, route, status_word, to_np

pytestmark = pytest.mark.gpu
SEED = 0
STUCK = 0x7FFFFFFF   # the first arrival flips bit 31; the CTAs after it wait for a flip that never comes
TIMEOUT, RANGE = 6, 8


def test_ffn_decode_grid_barrier_runs_out_then_a_fresh_call_passes():
    cfg = configs.get(0)
    layers, routers, _ = device_layers(SEED, cfg, 1)
    x_np = gen.tokens(SEED, cfg, 0)
    x = torch.from_numpy(x_np).cuda()
    idx, gate = route(routers[0], None, x, cfg.k)
    ws = torch.zeros(q.qmoe_decode_workspace_bytes(1, cfg.k, cfg.H, cfg.I), dtype=torch.uint8, device="cuda")
    ws[:4].view(torch.int32).fill_(STUCK)      # the grid-barrier counter is the workspace's first word
    st = status_word()
    ffn(layers[0], x, idx, gate, cfg.k, ws=ws, st=st, check=False)
    assert q.qmoe_read_status(st) == TIMEOUT
    # the context is still usable: a fresh workspace gives the oracle's answer
    y = ffn(layers[0], x, idx, gate, cfg.k)
    ref = W.run_layer(SEED, cfg, x_np.astype(np.float64), 0)[0]
    assert moe.rel_rms(to_np(y), ref) < DECODE_TOL


def test_fused_stack_grid_barrier_runs_out_then_a_fresh_stack_passes():
    cfg = configs.get(0).with_(L=2, residual=True)
    layers, routers, _ = device_layers(SEED, cfg, 2)
    x_np = gen.tokens(SEED, cfg, 0)
    stuck = DecodeStack(layers, routers, None, 1, cfg.k, cfg.eps)
    assert stuck.path == L.PATH_FUSED
    word = L.qmoe_stack_barrier_word(stuck.handle)
    off = word - stuck.workspace.data_ptr()
    assert 0 <= off < stuck.workspace.numel() and off % 4 == 0
    stuck.workspace[off:off + 4].view(torch.int32).fill_(STUCK)
    stuck.x_in.copy_(torch.from_numpy(x_np))
    stuck.decode()
    torch.cuda.synchronize()
    assert stuck.status() == TIMEOUT
    stuck.close()
    fresh = DecodeStack(layers, routers, None, 1, cfg.k, cfg.eps)
    fresh.x_in.copy_(torch.from_numpy(x_np))
    fresh.decode()
    torch.cuda.synchronize()
    assert fresh.status() == 0
    xo, _ = W.run_stack(SEED, cfg, x_np.astype(np.float64), 2)
    assert moe.rel_rms(to_np(fresh.x_out), xo) < DECODE_TOL
    fresh.close()


@pytest.mark.parametrize("layerwise", [False, True])
def test_activations_beyond_the_exact_sum_range_are_reported(layerwise):
    """x_0 of magnitude ~1e12: a router partial over one 16-element slice
    exceeds 2^19, so the stack reports QMOE_ERR_RANGE; every route it took is
    still a set of distinct experts in [0, E)."""
    cfg = configs.get(0).with_(L=3, residual=True)
    layers, routers, _ = device_layers(SEED, cfg, 3)
    stack = DecodeStack(layers, routers, None, 1, cfg.k, cfg.eps, layerwise=layerwise)
    stack.x_in.copy_(torch.from_numpy(gen.tokens(SEED, cfg, 0) * np.float32(1e12)))
    stack.decode()
    torch.cuda.synchronize()
    assert stack.status() == RANGE
    idx = to_np(stack.idx)
    assert ((idx >= 0) & (idx < cfg.E)).all()
    assert all(len(set(r.tolist())) == cfg.k for r in idx.reshape(-1, cfg.k))
    stack.close()
