"""GPU parity of the captured layer stack (route -> FFN -> residual RMSNorm per
layer, one CUDA graph) against the float64 oracle run free from the same x_0."""
import numpy as np
import pytest
import torch

from oracle import moe
from oracle import workload as W
from quantised_expert_decode_b200.model import DecodeStack
from synth import configs, gen
from synth.workload import device_layers
from tests.gpu_util import DECODE_TOL, GATE_TOL, gap_report, to_np

pytestmark = pytest.mark.gpu
SEED = 0


# Beyond the first layer the GPU and the oracle route slightly different
# activations (fp32 vs float64 arithmetic, 16-bit activation limbs), so two
# logits closer than this may legitimately order differently. A differing
# expert SET is accepted only as a reported near-tie below this gap.
NEAR_TIE = 1e-4


def _compare(cfg, stack, x0_np, n_layers):
    xo, recs = W.run_stack(SEED, cfg, x0_np.astype(np.float64), n_layers)
    idx = to_np(stack.idx)
    gate = to_np(stack.gate)
    for l, (x_in, oi, og, _) in enumerate(recs):
        if np.array_equal(idx[l], oi):
            assert np.max(np.abs(gate[l] - og)) < 50 * GATE_TOL, l
            continue
        L_ = W.Layer(SEED, cfg, l)
        lg = moe.logits(x_in, L_.Wr, L_.bias, cfg.k)
        for t in range(cfg.T):
            if set(idx[l, t].tolist()) != set(oi[t].tolist()):
                gap = gap_report(lg[t], cfg.k)
                if gap < NEAR_TIE:
                    pytest.xfail(f"layer {l} token {t}: near-tie route flip, oracle top-k gap {gap:.3g}")
                pytest.fail(f"layer {l} token {t}: expert sets differ; oracle top-k gap {gap:.3g}")
            for a, b in zip(idx[l, t], oi[t]):
                if a != b:
                    assert abs(lg[t, a] - lg[t, b]) < NEAR_TIE, (l, t, a, b)
            gm = dict(zip(idx[l, t].tolist(), gate[l, t].tolist()))
            for e, gv in zip(oi[t].tolist(), og[t].tolist()):
                assert abs(gm[e] - gv) < 50 * GATE_TOL, (l, t, e)
    err = moe.rel_rms(to_np(stack.x_out), xo)
    assert err < DECODE_TOL, err
    return err


def _run(cfg, n_layers, step=0, layerwise=False, built=None):
    layers, routers, biases = built if built else device_layers(SEED, cfg, n_layers)
    stack = DecodeStack(layers, routers, biases, cfg.T, cfg.k, cfg.eps, layerwise=layerwise)
    x0 = gen.tokens(SEED, cfg, step)
    stack.x_in.copy_(torch.from_numpy(x0))
    stack.decode()
    torch.cuda.synchronize()
    assert stack.status() == 0
    return stack, x0, layers


@pytest.mark.parametrize("layerwise", [False, True])
def test_stack_small_geometry(layerwise):
    cfg = configs.get(0).with_(L=6, residual=True)
    stack, x0, _ = _run(cfg, 6, layerwise=layerwise)
    _compare(cfg, stack, x0, 6)
    assert stack.path == (0 if layerwise else 1)
    assert stack.kernels_per_replay == (13 if layerwise else 1)
    # host-buffer entry point gives the same answer as the device-buffer replay
    xh = torch.from_numpy(x0).pin_memory()
    out = torch.empty_like(xh).pin_memory()
    ref = stack.x_out.clone()
    stack.decode_host(xh, out)
    torch.cuda.synchronize()
    assert torch.equal(out, ref.cpu())
    stack.close()


def test_stack_48_layers_q2_single_token():
    cfg = configs.get(2)
    stack, x0, layers = _run(cfg, cfg.L)
    assert sum(l.nbytes for l in layers) == cfg.L * cfg.E * cfg.expert_bytes()
    _compare(cfg, stack, x0, cfg.L)
    # replays are deterministic
    first = stack.x_out.clone()
    stack.decode()
    torch.cuda.synchronize()
    assert torch.equal(first, stack.x_out)
    # a second token through the same graph
    x1 = gen.tokens(SEED, cfg, 1)
    stack.x_in.copy_(torch.from_numpy(x1))
    stack.decode()
    torch.cuda.synchronize()
    _compare(cfg, stack, x1, cfg.L)
    # the per-layer kernel path routes identically and agrees to fp32 roundoff
    lw = DecodeStack(layers, stack.routers, None, cfg.T, cfg.k, cfg.eps, layerwise=True)
    lw.x_in.copy_(torch.from_numpy(x1))
    lw.decode()
    torch.cuda.synchronize()
    assert stack.path == 1 and lw.path == 0
    assert torch.equal(lw.idx, stack.idx)
    assert moe.rel_rms(to_np(lw.x_out), to_np(stack.x_out)) < 1e-5
    lw.close()
    stack.close()


def test_stack_48_layers_q4_verify_batch():
    cfg = configs.get(3)
    stack, x0, _ = _run(cfg, cfg.L)
    _compare(cfg, stack, x0, cfg.L)
    stack.close()


def test_verify_batch_equals_single_token_decoding_bit_for_bit():
    """A verify batch (8 correlated tokens, Q4 experts, per-layer path) reproduces
    every token decoded alone through the same per-layer path bit for bit:
    routes, gates and the final activations. A token's arithmetic (exact
    integer block sums, then one fixed floating-point order) does not depend on
    which other tokens of the batch share its experts."""
    cfg = configs.get(3)
    n_layers = 8
    layers, routers, biases = device_layers(SEED, cfg, n_layers)
    batch = DecodeStack(layers, routers, biases, cfg.T, cfg.k, cfg.eps, layerwise=True)
    one = DecodeStack(layers, routers, biases, 1, cfg.k, cfg.eps, layerwise=True)
    assert batch.path == 0 and one.path == 0
    x0 = torch.from_numpy(gen.tokens(SEED, cfg, 0)).cuda()
    batch.x_in.copy_(x0)
    batch.decode()
    torch.cuda.synchronize()
    assert batch.status() == 0
    # the batch does share experts, so the multi-token tile variants run
    idx = to_np(batch.idx)
    assert min(len(np.unique(idx[l])) for l in range(n_layers)) < cfg.T * cfg.k
    for t in range(cfg.T):
        one.x_in.copy_(x0[t:t + 1])
        one.decode()
        torch.cuda.synchronize()
        assert one.status() == 0
        assert torch.equal(one.idx[:, 0], batch.idx[:, t]), t
        assert torch.equal(one.gate[:, 0], batch.gate[:, t]), t
        assert torch.equal(one.x_out[0], batch.x_out[t]), t
    one.close()
    batch.close()
