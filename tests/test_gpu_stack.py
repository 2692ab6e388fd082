"""GPU parity of the captured layer stack (route -> FFN -> residual RMSNorm per
layer, one CUDA graph) against the float64 oracle run free from the same x_0,
and bit-for-bit agreement between the decode paths."""
import numpy as np
import pytest
import torch

from oracle import moe
from oracle import workload as W
from quantised_expert_decode_b200 import _lib as L
from quantised_expert_decode_b200.model import DecodeStack
from synth import configs, gen
from synth.workload import device_layers
from tests.gpu_util import DECODE_TOL, GATE_TOL, gap_report, to_np

pytestmark = pytest.mark.gpu
SEED = 0


def _flip_bound(cfg, built, x0, l, layerwise, x_oracle):
    """Certified bound on how far a GPU logit of layer l can sit from the
    oracle's own logit, from the actual input difference of that layer.

    The GPU's input to layer l is the output of the first l layers (a stack of
    l layers from the same x_0). A logit moves by at most
    ||Wr_e||_2 * ||x_gpu - x_oracle||_2 when its input moves, plus the GPU's own
    rounding of the normalised activations (2^-23 of sum_h |Wr_eh x_h|); two
    logits can swap only if their oracle gap is below twice that."""
    layers, routers, biases = built
    if l == 0:
        x_gpu = x0.astype(np.float64)
    else:
        part = DecodeStack(layers[:l], routers[:l], None if biases is None else biases[:l], cfg.T, cfg.k, cfg.eps,
                           layerwise=layerwise)
        part.x_in.copy_(torch.from_numpy(x0))
        part.decode()
        torch.cuda.synchronize()
        x_gpu = to_np(part.x_out).astype(np.float64)
        part.close()
    Wr = gen.router(SEED, cfg, l).astype(np.float64)
    delta = np.sqrt(np.sum((x_gpu - x_oracle) ** 2, axis=1))                     # per token
    rows = np.sqrt(np.sum(Wr * Wr, axis=1)).max()
    rnd = 2.0 ** -23 * (np.abs(x_gpu) @ np.abs(Wr).T).max(axis=1)
    return 2.0 * (rows * delta + rnd)


def _compare(cfg, stack, x0_np, n_layers, built, layerwise=False):
    xo, recs = W.run_stack(SEED, cfg, x0_np.astype(np.float64), n_layers)
    idx = to_np(stack.idx)
    gate = to_np(stack.gate)
    for l, (x_in, oi, og, _) in enumerate(recs):
        if np.array_equal(idx[l], oi):
            assert np.max(np.abs(gate[l] - og)) < 50 * GATE_TOL, l
            continue
        # A differing route is accepted only where the oracle's own top-k gap
        # lies below the bound derived from this layer's input difference;
        # the layers after it then follow another route, so the run stops here.
        L_ = W.Layer(SEED, cfg, l)
        lg = moe.logits(x_in, L_.Wr, L_.bias, cfg.k)
        bound = _flip_bound(cfg, built, x0_np, l, layerwise, x_in)
        for t in range(cfg.T):
            if np.array_equal(idx[l, t], oi[t]):
                continue
            gap = gap_report(lg[t], cfg.k)
            if gap >= bound[t]:
                pytest.fail(f"layer {l} token {t}: routes differ; oracle top-k gap {gap:.3g} "
                            f">= certified bound {bound[t]:.3g}")
        pytest.xfail(f"layer {l}: near-tie route flip within the certified input bound {bound.max():.3g}")
    err = moe.rel_rms(to_np(stack.x_out), xo)
    assert err < DECODE_TOL, err
    return err


def _run(cfg, n_layers, step=0, layerwise=False, built=None, scale=1.0):
    built = built if built else device_layers(SEED, cfg, n_layers)
    layers, routers, biases = built
    stack = DecodeStack(layers, routers, biases, cfg.T, cfg.k, cfg.eps, layerwise=layerwise)
    x0 = (gen.tokens(SEED, cfg, step) * np.float32(scale)).astype(np.float32)
    stack.x_in.copy_(torch.from_numpy(x0))
    stack.decode()
    torch.cuda.synchronize()
    assert stack.status() == 0
    return stack, x0, built


@pytest.mark.parametrize("layerwise", [False, True])
def test_stack_small_geometry(layerwise):
    cfg = configs.get(0).with_(L=6, residual=True)
    stack, x0, built = _run(cfg, 6, layerwise=layerwise)
    _compare(cfg, stack, x0, 6, built, layerwise)
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


def _same_bits(a, b):
    assert a.path != b.path
    assert torch.equal(a.idx, b.idx)
    assert torch.equal(a.gate, b.gate)
    assert torch.equal(a.x_out, b.x_out)


def test_stack_48_layers_q2_single_token():
    cfg = configs.get(2)
    stack, x0, built = _run(cfg, cfg.L)
    layers = built[0]
    assert sum(l.nbytes for l in layers) == cfg.L * cfg.E * cfg.expert_bytes()
    _compare(cfg, stack, x0, cfg.L, built)
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
    _compare(cfg, stack, x1, cfg.L, built)
    # the per-layer kernel path gives the same bits as the fused kernel
    lw = DecodeStack(layers, stack.routers, None, cfg.T, cfg.k, cfg.eps, layerwise=True)
    lw.x_in.copy_(torch.from_numpy(x1))
    lw.decode()
    torch.cuda.synchronize()
    assert stack.path == L.PATH_FUSED and lw.path == L.PATH_LAYERWISE
    _same_bits(stack, lw)
    lw.close()
    stack.close()


@pytest.mark.parametrize("scale", [1e3, 1e-4])
def test_stack_input_scale(scale):
    """x_0 scaled far from unit RMS (the first layer sees it raw): both paths
    match the oracle and each other bit for bit."""
    cfg = configs.get(2).with_(L=4)
    built = device_layers(SEED, cfg, 4)
    fused, x0, _ = _run(cfg, 4, built=built, scale=scale)
    assert fused.path == L.PATH_FUSED
    _compare(cfg, fused, x0, 4, built)
    lw, _, _ = _run(cfg, 4, built=built, scale=scale, layerwise=True)
    _same_bits(fused, lw)
    fused.close()
    lw.close()


def test_stack_48_layers_q4_verify_batch():
    cfg = configs.get(3)
    stack, x0, built = _run(cfg, cfg.L)
    _compare(cfg, stack, x0, cfg.L, built, layerwise=True)
    stack.close()


def test_verify_batch_equals_single_token_decoding_bit_for_bit():
    """A verify batch (8 correlated tokens, Q4 experts) reproduces every token
    decoded alone bit for bit - routes, gates and the final activations -
    against both single-token paths: the default one (the fused kernel) and
    the per-layer kernels. A token's arithmetic (exact integer block sums and
    router partials, then one fixed floating-point order) does not depend on
    which other tokens of the batch share its experts, nor on the path."""
    cfg = configs.get(3)
    n_layers = 8
    layers, routers, biases = device_layers(SEED, cfg, n_layers)
    batch = DecodeStack(layers, routers, biases, cfg.T, cfg.k, cfg.eps)
    one = DecodeStack(layers, routers, biases, 1, cfg.k, cfg.eps)
    one_lw = DecodeStack(layers, routers, biases, 1, cfg.k, cfg.eps, layerwise=True)
    assert batch.path == L.PATH_LAYERWISE and one.path == L.PATH_FUSED and one_lw.path == L.PATH_LAYERWISE
    x0 = torch.from_numpy(gen.tokens(SEED, cfg, 0)).cuda()
    batch.x_in.copy_(x0)
    batch.decode()
    torch.cuda.synchronize()
    assert batch.status() == 0
    # the batch does share experts, so the multi-token tile variants run
    idx = to_np(batch.idx)
    assert min(len(np.unique(idx[l])) for l in range(n_layers)) < cfg.T * cfg.k
    for t in range(cfg.T):
        for s in (one, one_lw):
            s.x_in.copy_(x0[t:t + 1])
            s.decode()
            torch.cuda.synchronize()
            assert s.status() == 0
            assert torch.equal(s.idx[:, 0], batch.idx[:, t]), (t, s.path)
            assert torch.equal(s.gate[:, 0], batch.gate[:, t]), (t, s.path)
            assert torch.equal(s.x_out[0], batch.x_out[t]), (t, s.path)
    one.close()
    one_lw.close()
    batch.close()


def test_fused_phase_trace_is_ordered_and_layer_times_add_up():
    """The fused kernel's phase stamps come in program order in every CTA and
    layer, and the per-layer times derived from them add up to the kernel's
    event-timed duration."""
    cfg = configs.get(0).with_(L=4, residual=True)
    layers, routers, _ = device_layers(SEED, cfg, 4)
    st = DecodeStack(layers, routers, None, 1, cfg.k, cfg.eps, timing=True)
    assert st.path == L.PATH_FUSED
    st.x_in.copy_(torch.from_numpy(gen.tokens(SEED, cfg, 0)))
    st.decode()
    torch.cuda.synchronize()
    assert st.status() == 0
    tr = st.phase_trace()
    assert tr.shape[0] == 4 and tr.shape[2] == 12
    assert (np.diff(tr[:, :, :7], axis=2) >= 0).all()
    assert ((tr[:, :, 0] <= tr[:, :, 7]) & (tr[:, :, 7] <= tr[:, :, 1])).all()   # logits ready, then the top-k
    busy = tr[:, :, 8] != 0                               # CTAs with gate/up tiles in the layer
    assert busy.any()
    assert ((tr[:, :, 2] <= tr[:, :, 8]) & (tr[:, :, 8] <= tr[:, :, 3]))[busy].all()   # a tile lands while C runs
    rows = np.arange(tr.shape[1]) < cfg.H // 16          # CTAs that own output rows run phase D
    d = tr[:, rows]
    assert ((d[:, :, 4] <= d[:, :, 9]) & (d[:, :, 9] <= d[:, :, 10]) & (d[:, :, 10] <= d[:, :, 11])
            & (d[:, :, 11] <= d[:, :, 5])).all()
    route_ms, ffn_ms = st.layer_times()
    assert all(r >= 0 for r in route_ms) and all(f > 0 for f in ffn_ms)
    plain = DecodeStack(layers, routers, None, 1, cfg.k, cfg.eps)
    plain.x_in.copy_(st.x_in)
    plain.decode()
    torch.cuda.synchronize()
    assert torch.equal(plain.x_out, st.x_out)     # stamping changes no result
    plain.close()
    st.close()



MIXED6 = (configs.Q2, configs.Q4, configs.Q4, configs.Q2, configs.Q4, configs.Q2)


@pytest.mark.parametrize("layerwise", [False, True])
def test_mixed_bit_stack_small_geometry(layerwise):
    """A stack whose layers use different block formats (Q2 and Q4 per layer)
    matches the oracle on both paths: the fused kernel takes each layer's
    format in turn, the per-layer kernels get each layer's handle."""
    cfg = configs.get(0).with_(L=6, residual=True, fmt_layers=MIXED6)
    stack, x0, built = _run(cfg, 6, layerwise=layerwise)
    assert [l.fmt for l in built[0]] == list(MIXED6)
    assert stack.path == (L.PATH_LAYERWISE if layerwise else L.PATH_FUSED)
    _compare(cfg, stack, x0, 6, built, layerwise)
    stack.close()


def test_mixed_bit_stack_decode_geometry_and_verify_batch():
    """Decode geometry (512 experts, H 2048, I 768, top-10) with a block
    format per layer: one token (fused kernel) and an 8-token verify batch
    (per-layer kernels) match the oracle; the per-layer path gives the fused
    path's bits, and every token of the batch equals that token decoded
    alone, bit for bit."""
    n = 4
    fl = (configs.Q4, configs.Q2, configs.Q2, configs.Q4)
    cfg1 = configs.get(2).with_(L=n, fmt_layers=fl)
    built = device_layers(SEED, cfg1, n)
    layers, routers, biases = built
    assert sum(l.nbytes for l in layers) == sum(cfg1.E * cfg1.for_layer(l).expert_bytes() for l in range(n))
    one, x0, _ = _run(cfg1, n, built=built)
    assert one.path == L.PATH_FUSED
    _compare(cfg1, one, x0, n, built)
    one_lw, _, _ = _run(cfg1, n, built=built, layerwise=True)
    _same_bits(one, one_lw)

    cfg8 = cfg1.with_(T=8, x_kind="correlated")   # same configuration id: same layers
    batch, xb, _ = _run(cfg8, n, built=built)
    assert batch.path == L.PATH_LAYERWISE
    _compare(cfg8, batch, xb, n, built, layerwise=True)
    x8 = torch.from_numpy(xb).cuda()
    for t in range(cfg8.T):
        for s in (one, one_lw):
            s.x_in.copy_(x8[t:t + 1])
            s.decode()
            torch.cuda.synchronize()
            assert s.status() == 0
            assert torch.equal(s.idx[:, 0], batch.idx[:, t]), (t, s.path)
            assert torch.equal(s.gate[:, 0], batch.gate[:, t]), (t, s.path)
            assert torch.equal(s.x_out[0], batch.x_out[t]), (t, s.path)
    for s in (one, one_lw, batch):
        s.close()
