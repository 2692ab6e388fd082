"""GPU parity of the decode path (router, bucketing, dequant-GEMV FFN, combine)
against the float64 oracle on the same seeded inputs."""
import numpy as np
import pytest
import torch

import quantised_expert_decode_b200 as q
from oracle import moe
from oracle import workload as W
from quantised_expert_decode_b200 import _lib as L
from quantised_expert_decode_b200.model import PackedLayer
from synth import configs, device, gen
from synth.workload import device_layers, device_tokens
from tests.gpu_util import DECODE_TOL, GATE_TOL, ffn, route, status_word, to_np

pytestmark = pytest.mark.gpu
SEED = 0


@pytest.fixture(scope="module")
def cfg1_layer():
    cfg = configs.get(1)
    layers, routers, _ = device_layers(SEED, cfg, 1)
    return cfg, layers[0], routers[0]


@pytest.fixture(scope="module")
def cfg3_layer():
    cfg = configs.get(3)
    layers, routers, _ = device_layers(SEED, cfg, 1)
    return cfg, layers[0], routers[0]


def test_device_fill_is_bit_identical_to_host_generator():
    for cid, experts in ((0, range(64)), (1, (0, 17, 511)), (3, (0, 300, 511))):
        cfg = configs.get(cid)
        for e in experts:
            bufs = device.alloc_canonical(cfg, "cuda", E=1)
            device.fill_layer(SEED, cfg, 0 if cid != 3 else 5, bufs, e0=e)
            torch.cuda.synchronize()
            ref = gen.expert(SEED, cfg, 0 if cid != 3 else 5, e)
            for name in ("gate", "up", "down"):
                assert np.array_equal(to_np(bufs[name + "_codes"][0]), ref[name + "_codes"]), (cid, e, name)
                got = to_np(bufs[name + "_scales"][0]).view(np.uint16)
                assert np.array_equal(got, ref[name + "_scales"]), (cid, e, name)


@pytest.mark.parametrize("cid", [0, 1])
def test_route_matches_oracle(cid):
    cfg = configs.get(cid)
    Wr_np = gen.router(SEED, cfg, 0)
    Wr = torch.from_numpy(Wr_np).cuda()
    for step in range(6):
        x_np = gen.tokens(SEED, cfg, step)
        idx, gate = route(Wr, None, torch.from_numpy(x_np).cuda(), cfg.k)
        oi, og, _ = moe.route(x_np.astype(np.float64), Wr_np, None, cfg.k)
        assert np.array_equal(to_np(idx), oi), step
        assert np.max(np.abs(to_np(gate) - og)) < GATE_TOL


def test_route_multi_token_matches_oracle():
    cfg = configs.get(3)
    Wr_np = gen.router(SEED, cfg, 2)
    Wr = torch.from_numpy(Wr_np).cuda()
    for T in (1, 2, 3, 5, 8):
        x_np = gen.tokens(SEED, cfg, 1, T=T)
        idx, gate = route(Wr, None, torch.from_numpy(x_np).cuda(), cfg.k)
        oi, og, _ = moe.route(x_np.astype(np.float64), Wr_np, None, cfg.k)
        assert np.array_equal(to_np(idx), oi), T
        assert np.max(np.abs(to_np(gate) - og)) < GATE_TOL


def test_route_special_activation_values():
    """Exact zeros, negative zeros, subnormals and large magnitudes in x: every
    value the router widens to float64 keeps its exact value."""
    cfg = configs.get(1)
    Wr_np = gen.router(SEED, cfg, 0)
    Wr = torch.from_numpy(Wr_np).cuda()
    rs = np.random.default_rng(3)
    for T in (1, 4, 8):
        x_np = gen.tokens(SEED, cfg, 2, T=T).copy()
        pick = rs.random(x_np.shape)
        x_np[pick < 0.05] = 0.0
        x_np[(pick >= 0.05) & (pick < 0.1)] = -0.0
        sub = (pick >= 0.1) & (pick < 0.15)
        x_np[sub] = np.float32(1e-40) * np.sign(rs.standard_normal(int(sub.sum()))).astype(np.float32)
        x_np[(pick >= 0.15) & (pick < 0.16)] *= np.float32(1e4)
        idx, gate = route(Wr, None, torch.from_numpy(x_np).cuda(), cfg.k)
        oi, og, _ = moe.route(x_np.astype(np.float64), Wr_np, None, cfg.k)
        assert np.array_equal(to_np(idx), oi), T
        assert np.max(np.abs(to_np(gate) - og)) < GATE_TOL


@pytest.mark.parametrize("E,H,T", [(100, 384, 3), (33, 128, 1), (1000, 640, 8)])
def test_route_ragged_geometry_with_bias(E, H, T):
    """Expert counts that leave lanes of the last 32-expert group idle and
    hidden sizes whose 16-element slices do not split evenly over the CTAs."""
    rs = np.random.default_rng(E + H + T)
    Wr_np = (0.05 * rs.standard_normal((E, H))).astype(np.float32)
    b_np = (0.1 * rs.standard_normal(E)).astype(np.float32)
    x_np = rs.standard_normal((T, H)).astype(np.float32)
    k = min(10, E)
    idx, gate = route(torch.from_numpy(Wr_np).cuda(), torch.from_numpy(b_np).cuda(), torch.from_numpy(x_np).cuda(), k)
    oi, og, _ = moe.route(x_np.astype(np.float64), Wr_np, b_np, k)
    assert np.array_equal(to_np(idx), oi)
    assert np.max(np.abs(to_np(gate) - og)) < GATE_TOL


def test_route_exact_ties_go_to_lower_index():
    cfg = configs.get(0)
    Wr_np = gen.router(SEED, cfg, 0).copy()
    x_np = gen.tokens(SEED, cfg, 0)
    best = int(moe.topk(moe.logits(x_np.astype(np.float64), Wr_np, None, 4)[0], 1)[0])
    for dup in (2, 40, 63):
        Wr_np[dup] = Wr_np[best]
    idx, gate = route(torch.from_numpy(Wr_np).cuda(), None, torch.from_numpy(x_np).cuda(), 4)
    oi, og, _ = moe.route(x_np.astype(np.float64), Wr_np, None, 4)
    assert np.array_equal(to_np(idx), oi)
    assert sorted(to_np(idx)[0].tolist()) == sorted([best, 2, 40, 63])
    assert np.allclose(to_np(gate), 0.25, atol=1e-7)


def test_route_degenerate_equal_logits():
    E, H, k = 512, 2048, 10
    Wr = torch.zeros((E, H), dtype=torch.float32, device="cuda")
    x = torch.randn((2, H), dtype=torch.float32, device="cuda")
    idx, gate = route(Wr, None, x, k)
    assert to_np(idx).tolist() == [list(range(k))] * 2
    assert np.allclose(to_np(gate), 1.0 / k, atol=1e-7)


def _oracle_layer(seed, cfg, layer, x64, idx, g):
    L_ = W.Layer(seed, cfg, layer)
    return moe.moe_layer(x64, idx, g, L_.expert)


def test_ffn_decode_cfg0_parity():
    cfg = configs.get(0)
    layers, routers, _ = device_layers(SEED, cfg, 1)
    for step in range(4):
        x_np = gen.tokens(SEED, cfg, step)
        x = torch.from_numpy(x_np).cuda()
        idx, gate = route(routers[0], None, x, cfg.k)
        y = ffn(layers[0], x, idx, gate, cfg.k)
        yo, oi, og, _ = W.run_layer(SEED, cfg, x_np.astype(np.float64), 0)
        assert np.array_equal(to_np(idx), oi)
        err = moe.rel_rms(to_np(y), yo)
        assert err < DECODE_TOL, err


def test_ffn_decode_cfg1_parity(cfg1_layer):
    cfg, layer, Wr = cfg1_layer
    for step in range(3):
        x_np = gen.tokens(SEED, cfg, step)
        x = torch.from_numpy(x_np).cuda()
        idx, gate = route(Wr, None, x, cfg.k)
        y = ffn(layer, x, idx, gate, cfg.k)
        yo, oi, og, _ = W.run_layer(SEED, cfg, x_np.astype(np.float64), 0)
        assert np.array_equal(to_np(idx), oi)
        err = moe.rel_rms(to_np(y), yo)
        assert err < DECODE_TOL, (step, err)


def test_ffn_decode_is_deterministic(cfg1_layer):
    cfg, layer, Wr = cfg1_layer
    x = device_tokens(SEED, cfg, 7)
    idx, gate = route(Wr, None, x, cfg.k)
    y1 = ffn(layer, x, idx, gate, cfg.k)
    y2 = ffn(layer, x, idx, gate, cfg.k)
    assert torch.equal(y1, y2)


@pytest.mark.parametrize("T", [1, 2, 3, 4, 5, 8])
def test_ffn_decode_q4_batches(cfg3_layer, T):
    cfg, layer, Wr = cfg3_layer
    x_np = gen.tokens(SEED, cfg, 0, T=T)
    x = torch.from_numpy(x_np).cuda()
    idx, gate = route(Wr, None, x, cfg.k)
    y = ffn(layer, x, idx, gate, cfg.k)
    oi, og, _ = moe.route(x_np.astype(np.float64), gen.router(SEED, cfg, 0), None, cfg.k)
    assert np.array_equal(to_np(idx), oi)
    yo = _oracle_layer(SEED, cfg, 0, x_np.astype(np.float64), oi, og)
    err = moe.rel_rms(to_np(y), yo)
    assert err < DECODE_TOL, (T, err)


@pytest.mark.parametrize("pattern", ["all_shared", "three_shared", "disjoint", "k1", "k16"])
def test_ffn_decode_crafted_routes(cfg3_layer, pattern):
    """Explicit routes exercising every token-per-expert width (1..8)."""
    cfg, layer, _ = cfg3_layer
    rng = np.random.default_rng(11)
    T, k = 8, 10
    if pattern == "all_shared":
        base = rng.permutation(cfg.E)[:k]
        idx_np = np.stack([rng.permutation(base) for _ in range(T)])
    elif pattern == "three_shared":
        base = rng.permutation(cfg.E)[:2 * k]
        idx_np = np.stack([rng.permutation(base[:k]) if t < 3 else rng.permutation(base[k:])
                           if t < 5 else rng.permutation(cfg.E)[:k] for t in range(T)])
    elif pattern == "disjoint":
        idx_np = rng.permutation(cfg.E)[:T * k].reshape(T, k)
    elif pattern == "k1":
        k = 1
        idx_np = np.array([[7], [7], [9], [7], [511], [0], [9], [7]])
    else:
        k = 16
        idx_np = np.stack([rng.permutation(cfg.E)[:k] for _ in range(T)])
    idx_np = idx_np.astype(np.int32)
    g = rng.dirichlet(np.ones(k), size=T).astype(np.float32)
    x_np = gen.tokens(SEED, cfg, 3, T=T)
    x = torch.from_numpy(x_np).cuda()
    y = ffn(layer, x, torch.from_numpy(idx_np).cuda(), torch.from_numpy(g).cuda(), k)
    yo = _oracle_layer(SEED, cfg, 0, x_np.astype(np.float64), idx_np, g.astype(np.float64))
    err = moe.rel_rms(to_np(y), yo)
    assert err < DECODE_TOL, (pattern, err)


def test_ffn_decode_zero_activation(cfg1_layer):
    cfg, layer, Wr = cfg1_layer
    x = torch.zeros((1, cfg.H), dtype=torch.float32, device="cuda")
    idx = torch.arange(cfg.k, dtype=torch.int32, device="cuda").view(1, cfg.k)
    gate = torch.full((1, cfg.k), 0.1, dtype=torch.float32, device="cuda")
    y = ffn(layer, x, idx, gate, cfg.k)
    assert torch.count_nonzero(y).item() == 0


def test_ffn_decode_refuses_bad_routes(cfg1_layer):
    cfg, layer, Wr = cfg1_layer
    x = device_tokens(SEED, cfg, 0)
    gate = torch.full((1, cfg.k), 0.1, dtype=torch.float32, device="cuda")
    for bad in ([3, 4, 5, 6, 7, 8, 9, 10, 11, 512], [3, 4, 5, 6, 7, 8, 9, 10, 11, -1],
                [3, 4, 5, 6, 7, 8, 9, 10, 11, 3]):
        st = status_word()
        idx = torch.tensor([bad], dtype=torch.int32, device="cuda")
        y = ffn(layer, x, idx, gate, cfg.k, st=st, check=False)
        assert q.qmoe_read_status(st) == 7
        assert torch.isnan(y).all()          # nothing written
    # a good call afterwards still works (the workspace was left consistent)
    idx, g2 = route(Wr, None, x, cfg.k)
    ffn(layer, x, idx, g2, cfg.k)


def test_ffn_decode_host_checks(cfg1_layer):
    cfg, layer, Wr = cfg1_layer
    x = device_tokens(SEED, cfg, 0)
    idx, gate = route(Wr, None, x, cfg.k)
    h = layer.handle()
    h.H = 1024
    y = torch.empty_like(x)
    ws = torch.zeros(q.qmoe_decode_workspace_bytes(1, cfg.k, cfg.H, cfg.I), dtype=torch.uint8, device="cuda")
    with pytest.raises(q.QmoeError) as e:
        q.qmoe_ffn_decode(h, x, 1, idx, gate, cfg.k, y, ws, status_word())
    assert e.value.code == 2
    with pytest.raises(q.QmoeError) as e:
        q.qmoe_ffn_decode(layer.handle(), x, 1, idx, gate, cfg.k, y, ws[:-512], status_word())
    assert e.value.code == 4


def test_rmsnorm_and_residual_route(cfg1_layer):
    cfg, layer, Wr = cfg1_layer
    x_np = gen.tokens(SEED, cfg, 2)
    y_np = (0.1 * gen.tokens(SEED, cfg, 3)).astype(np.float32)
    x, y = torch.from_numpy(x_np).cuda(), torch.from_numpy(y_np).cuda()
    out = torch.empty_like(x)
    q.qmoe_rmsnorm_residual(x, y, cfg.eps, out, 1, cfg.H)
    ref = moe.rmsnorm_residual(x_np, y_np, cfg.eps)
    assert moe.rel_rms(to_np(out), ref) < 1e-6
    idx = torch.empty((1, cfg.k), dtype=torch.int32, device="cuda")
    gate = torch.empty((1, cfg.k), dtype=torch.float32, device="cuda")
    ws = torch.zeros(q.qmoe_route_workspace_bytes(1, cfg.E), dtype=torch.uint8, device="cuda")
    xo = torch.empty_like(x)
    q.qmoe_residual_route(x, y, cfg.eps, xo, Wr, None, 1, cfg.H, cfg.E, cfg.k, idx, gate, ws, status_word())
    torch.cuda.synchronize()
    assert torch.equal(xo, out)
    oi, og, _ = moe.route(ref, gen.router(SEED, cfg, 0), None, cfg.k)
    assert np.array_equal(to_np(idx), oi)
    assert np.max(np.abs(to_np(gate) - og)) < GATE_TOL
