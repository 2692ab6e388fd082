"""GPU parity of the prefill path (bucketing, prefill router, tcgen05 grouped
GEMMs with the gate-weighted combine) against plain definitions and the
float64 oracle on the same seeded inputs."""
import numpy as np
import pytest
import torch

import quantised_expert_decode_b200 as q
from oracle import moe
from oracle import workload as W
from quantised_expert_decode_b200 import _lib as L
from synth import configs, gen
from synth.workload import device_layers, device_tokens
from tests.gpu_util import GATE_TOL, route, status_word, to_np

pytestmark = pytest.mark.gpu
SEED = 0
PREFILL_TOL = 2e-2     # rel-RMS bound for bf16 tensor-core prefill


# ------------------------------------------------------------- bucketing ----
def _bucket(idx_np, E, check=True):
    T, k = idx_np.shape
    idx = torch.from_numpy(np.ascontiguousarray(idx_np, dtype=np.int32)).cuda()
    off = torch.full((E + 1,), -1, dtype=torch.int32, device="cuda")
    perm = torch.full((T * k,), -1, dtype=torch.int32, device="cuda")
    act = torch.full((E,), -1, dtype=torch.int32, device="cuda")
    nact = torch.full((1,), -1, dtype=torch.int32, device="cuda")
    ws = torch.full((q.qmoe_bucket_workspace_bytes(T, k, E),), 0x5A, dtype=torch.uint8, device="cuda")
    st = status_word()
    q.qmoe_bucket(idx, T, k, E, off, perm, act, nact, ws, st)
    torch.cuda.synchronize()
    if check:
        assert q.qmoe_read_status(st) == 0
    return to_np(off), to_np(perm), to_np(act), int(to_np(nact)[0]), st


def _bucket_reference(idx_np, E):
    """Plain definition: counts, exclusive prefix, stable sort of pair ids by expert."""
    flat = idx_np.ravel()
    counts = np.bincount(flat, minlength=E)
    off = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    perm = np.argsort(flat, kind="stable").astype(np.int32)
    active = np.nonzero(counts)[0].astype(np.int32)
    return off, perm, active


@pytest.mark.parametrize("T,k,E", [(1, 1, 1), (1, 10, 512), (37, 4, 64), (4096, 10, 512), (1000, 8, 100),
                                   (333, 16, 1024), (9473, 3, 257), (148 * 64 + 1, 2, 33), (30000, 10, 1000)])
def test_bucket_is_the_stable_sort(T, k, E):
    rs = np.random.default_rng(T * 7 + k)
    # long-tailed loads: a few experts take most pairs (duplicates within a token allowed here)
    p = rs.pareto(1.2, size=E) + 1e-3
    idx = rs.choice(E, size=(T, k), p=p / p.sum()).astype(np.int32)
    off, perm, act, nact, _ = _bucket(idx, E)
    r_off, r_perm, r_act = _bucket_reference(idx, E)
    assert np.array_equal(off, r_off)
    assert np.array_equal(perm, r_perm)
    assert nact == len(r_act) and np.array_equal(act[:nact], r_act)


def test_bucket_all_pairs_to_one_expert_and_bad_index():
    idx = np.full((300, 3), 7, dtype=np.int32)
    off, perm, act, nact, _ = _bucket(idx, 16)
    assert off[7] == 0 and off[8] == 900 and off[16] == 900
    assert np.array_equal(perm, np.arange(900)) and nact == 1 and act[0] == 7
    idx[5, 1] = 16
    *_, st = _bucket(idx, 16, check=False)
    assert q.qmoe_read_status(st) == 7


def test_bucket_bad_index_in_a_late_cta_leaves_every_output_unwritten():
    rs = np.random.default_rng(11)
    idx = rs.integers(0, 64, size=(20000, 4)).astype(np.int32)
    idx[19990, 2] = -3
    off, perm, act, nact, st = _bucket(idx, 64, check=False)
    assert q.qmoe_read_status(st) == 7
    assert (off == -1).all() and (perm == -1).all() and (act == -1).all() and nact == -1


# ---------------------------------------------------------------- router ----
def test_prefill_router_matches_oracle_at_full_size():
    """4096 bf16 tokens, biased router: every index bit-exact, gates within GATE_TOL."""
    cfg = configs.get(4)
    Wr_np, b_np = gen.router(SEED, cfg, 0), gen.bias(SEED, cfg, 0)
    x_bits = gen.tokens(SEED, cfg, 0)
    x = torch.from_numpy(x_bits.view(np.int16)).cuda().view(torch.bfloat16)
    idx, gate = route(torch.from_numpy(Wr_np).cuda(), torch.from_numpy(b_np).cuda(), x, cfg.k, L.BF16)
    oi, og, _ = moe.route(gen.bf16_bits_to_f32(x_bits).astype(np.float64), Wr_np, b_np, cfg.k)
    assert np.array_equal(to_np(idx), oi)
    assert np.max(np.abs(to_np(gate) - og)) < GATE_TOL


def test_prefill_router_fp32_many_tokens_and_ties():
    cfg = configs.get(0)
    Wr_np = gen.router(SEED, cfg, 0).copy()
    Wr_np[9] = Wr_np[3]            # exact ties: equal logits, lower index wins
    Wr_np[40] = Wr_np[3]
    x_np = gen.tokens(SEED, cfg, 0, T=37)
    idx, gate = route(torch.from_numpy(Wr_np).cuda(), None, torch.from_numpy(x_np).cuda(), cfg.k)
    oi, og, _ = moe.route(x_np.astype(np.float64), Wr_np, None, cfg.k)
    assert np.array_equal(to_np(idx), oi)
    assert np.max(np.abs(to_np(gate) - og)) < GATE_TOL


def test_prefill_router_degenerate_equal_rows_take_the_exact_path():
    """Every router row equal: all logits tie, more experts are candidates than
    the candidate list holds, and the router falls back to float64 logits for
    every expert; ties go to the lower index, gates are uniform."""
    rs = np.random.default_rng(3)
    E, H, k, T = 128, 256, 8, 20
    row = (0.02 * rs.standard_normal(H)).astype(np.float32)
    Wr_np = np.tile(row, (E, 1))
    x_np = rs.standard_normal((T, H)).astype(np.float32)
    idx, gate = route(torch.from_numpy(Wr_np).cuda(), None, torch.from_numpy(x_np).cuda(), k)
    oi, og, _ = moe.route(x_np.astype(np.float64), Wr_np, None, k)
    assert np.array_equal(to_np(idx), oi)
    assert np.array_equal(oi, np.tile(np.arange(k, dtype=np.int32), (T, 1)))
    assert np.max(np.abs(to_np(gate) - 1.0 / k)) < GATE_TOL


def test_prefill_router_bf16_few_tokens_and_ragged_sizes():
    """bf16 activations with T <= 8 also take the prefill router; T and E not
    multiples of the GEMM tile."""
    rs = np.random.default_rng(4)
    for T, E, k in ((3, 200, 7), (70, 96, 16)):
        H = 384
        Wr_np = (0.02 * rs.standard_normal((E, H))).astype(np.float32)
        b_np = rs.standard_normal(E).astype(np.float32)
        x_bits = gen.f32_to_bf16_bits(rs.standard_normal((T, H)).astype(np.float32))
        x = torch.from_numpy(x_bits.view(np.int16)).cuda().view(torch.bfloat16)
        idx, gate = route(torch.from_numpy(Wr_np).cuda(), torch.from_numpy(b_np).cuda(), x, k, L.BF16)
        oi, og, _ = moe.route(gen.bf16_bits_to_f32(x_bits).astype(np.float64), Wr_np, b_np, k)
        assert np.array_equal(to_np(idx), oi), (T, E)
        assert np.max(np.abs(to_np(gate) - og)) < GATE_TOL


# ------------------------------------------------------------- prefill FFN --
def _prefill(layer, x, idx, gate, k, check=True):
    T = x.shape[0]
    y = torch.full((T, layer.H), float("nan"), dtype=torch.float32, device="cuda")
    ws = torch.empty(q.qmoe_prefill_workspace_bytes(T, k, layer.E, layer.H, layer.I), dtype=torch.uint8,
                     device="cuda")
    st = status_word()
    q.qmoe_ffn_prefill(layer.handle(), x, T, idx, gate, k, y, ws, st)
    torch.cuda.synchronize()
    if check:
        assert q.qmoe_read_status(st) == 0
    return y, st


def _oracle_rows(cfg, x64, idx, g, rows):
    """Oracle outputs of the given token rows on their given routes
    (``moe.moe_layer``), each expert generated once and not kept."""
    Lyr = W.Layer(SEED, cfg, 0)

    def get(e):
        w = Lyr.expert(e)
        Lyr.drop()
        return w
    rows = np.asarray(rows)
    return moe.moe_layer(x64[rows], idx[rows], g[rows], get)


def _row_errors(y, ref):
    """Relative error of every token row: ||y_t - ref_t|| / ||ref_t||."""
    y = np.asarray(y, dtype=np.float64)
    return np.sqrt(np.sum((y - ref) ** 2, axis=1)) / np.sqrt(np.sum(ref * ref, axis=1))


SMALL = configs.get(4).with_(E=64, H=512, I=256, k=4, T=300)


@pytest.fixture(scope="module")
def small_layer():
    layers, routers, biases = device_layers(SEED, SMALL, 1)
    return layers[0], routers[0], biases[0]


def _small_inputs(T, step=0):
    x_bits = gen.tokens(SEED, SMALL, step, T=T)
    x = torch.from_numpy(x_bits.view(np.int16)).cuda().view(torch.bfloat16)
    return x, gen.bf16_bits_to_f32(x_bits).astype(np.float64)


def test_prefill_small_layer_matches_oracle(small_layer):
    layer, Wr, bias = small_layer
    x, x64 = _small_inputs(SMALL.T)
    idx, gate = route(Wr, bias, x, SMALL.k, L.BF16)
    y, _ = _prefill(layer, x, idx, gate, SMALL.k)
    idx_np, g_np = to_np(idx), to_np(gate).astype(np.float64)
    ref = W.run_layer(SEED, SMALL, x64)[0]
    # every token row on its own: one wrong row cannot hide in an average
    errs = _row_errors(to_np(y), ref)
    assert errs.max() < PREFILL_TOL, (int(errs.argmax()), errs.max())
    # the route itself is the oracle's
    oi, og, _ = moe.route(x64, gen.router(SEED, SMALL, 0), gen.bias(SEED, SMALL, 0), SMALL.k)
    assert np.array_equal(idx_np, oi)


@pytest.mark.parametrize("T", [1, 17, 600])
def test_prefill_crafted_routes(small_layer, T):
    """One expert takes every token (T = 600: chunks of 256, 256 and a ragged 88),
    the other slots spread over the rest; gates arbitrary positive values."""
    layer, _, _ = small_layer
    k, E = SMALL.k, SMALL.E
    rs = np.random.default_rng(T)
    idx_np = np.empty((T, k), dtype=np.int32)
    for t in range(T):
        others = rs.choice(np.arange(1, E), size=k - 1, replace=False)
        idx_np[t] = np.concatenate([[0], others]) if t % 2 == 0 else np.concatenate([others, [0]])
    g_np = rs.uniform(0.05, 1.0, size=(T, k)).astype(np.float32)
    x, x64 = _small_inputs(T, step=3)
    y, _ = _prefill(layer, x, torch.from_numpy(idx_np).cuda(), torch.from_numpy(g_np).cuda(), k)
    rows = list(range(T)) if T <= 17 else list(range(0, T, 37))
    ref = _oracle_rows(SMALL, x64, idx_np, g_np.astype(np.float64), rows)
    errs = _row_errors(to_np(y)[rows], ref)
    assert errs.max() < PREFILL_TOL, (rows[int(errs.argmax())], errs.max())


def test_prefill_zero_activation_and_bad_routes(small_layer):
    layer, _, _ = small_layer
    T, k = 40, SMALL.k
    x = torch.zeros((T, SMALL.H), dtype=torch.bfloat16, device="cuda")
    idx_np = np.tile(np.arange(k, dtype=np.int32), (T, 1))
    g = torch.full((T, k), 0.25, dtype=torch.float32, device="cuda")
    y, _ = _prefill(layer, x, torch.from_numpy(idx_np).cuda(), g, k)
    assert torch.count_nonzero(y).item() == 0            # silu(0) * 0 = 0 everywhere
    idx_np[3, 2] = SMALL.E                                 # out of range
    y, st = _prefill(layer, x, torch.from_numpy(idx_np).cuda(), g, k, check=False)
    assert q.qmoe_read_status(st) == 7
    idx_np[3, 2] = idx_np[3, 0]                            # repeated within one token
    y, st = _prefill(layer, x, torch.from_numpy(idx_np).cuda(), g, k, check=False)
    assert q.qmoe_read_status(st) == 7


def test_prefill_full_size_rows_of_the_heaviest_expert():
    """The 4096-token chunk through one 512-expert Q4 layer with the biased
    router. The oracle checks, row by row, every token routed to the most
    loaded expert (its pairs span several 256-token chunks, so every chunk
    boundary of the grouped GEMMs is crossed) and 256 further random tokens.
    The routes fed to the oracle are the GPU's; the router's own parity is
    checked bit for bit in test_prefill_router_matches_oracle_at_full_size."""
    cfg = configs.get(4)
    layers, routers, biases = device_layers(SEED, cfg, 1)
    x = device_tokens(SEED, cfg, 0)
    idx, gate = route(routers[0], biases[0], x, cfg.k, L.BF16)
    y, _ = _prefill(layers[0], x, idx, gate, cfg.k)
    idx_np, g_np = to_np(idx), to_np(gate).astype(np.float64)
    counts = np.bincount(idx_np.ravel(), minlength=cfg.E)
    assert counts.max() > 512          # the skewed load spans several 256-token chunks
    x64 = W.x_float(SEED, cfg)
    heavy = int(counts.argmax())
    rows = set(np.nonzero((idx_np == heavy).any(axis=1))[0].tolist())
    rows |= set(np.random.default_rng(7).choice(cfg.T, size=256, replace=False).tolist())
    rows = sorted(rows | {0, cfg.T - 1})
    ref = _oracle_rows(cfg, x64, idx_np, g_np, rows)
    errs = _row_errors(to_np(y)[rows], ref)
    assert errs.max() < PREFILL_TOL, (rows[int(errs.argmax())], errs.max())
    assert np.isfinite(to_np(y)).all()


def test_prefill_combine_is_reproducible_and_matches_the_atomic_form(small_layer):
    """The slot-ordered combine gives the same bits on every run; the earlier
    atomic combine (kept behind a flag of the timed entry point) agrees to fp32
    rounding of the order of its additions."""
    layer, Wr, bias = small_layer
    x, x64 = _small_inputs(SMALL.T, step=1)
    idx, gate = route(Wr, bias, x, SMALL.k, L.BF16)
    y1, _ = _prefill(layer, x, idx, gate, SMALL.k)
    y2, _ = _prefill(layer, x, idx, gate, SMALL.k)
    assert torch.equal(y1, y2)
    T, k = SMALL.T, SMALL.k
    ya = torch.full((T, layer.H), float("nan"), dtype=torch.float32, device="cuda")
    ws = torch.empty(q.qmoe_prefill_workspace_bytes(T, k, layer.E, layer.H, layer.I), dtype=torch.uint8,
                     device="cuda")
    st = status_word()
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
    q.qmoe_ffn_prefill_timed(layer.handle(), x, T, idx, gate, k, ya, ws, st, ev, flags=L.PREFILL_ATOMIC_COMBINE)
    torch.cuda.synchronize()
    assert q.qmoe_read_status(st) == 0
    assert moe.rel_rms(to_np(ya), to_np(y1)) < 1e-6
    ref = W.run_layer(SEED, SMALL, x64)[0]
    assert _row_errors(to_np(y1), ref).max() < PREFILL_TOL
