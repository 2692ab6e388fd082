"""Pins of the float64 oracle to facts fixed outside it.

Each test checks the oracle against something it does not compute itself:
hand-worked values of the block format, brute-force enumeration, exact
rational arithmetic, closed forms and invariants.
"""
import itertools
import json
import math
import os
from fractions import Fraction

import numpy as np
import pytest

from oracle import moe

RNG = np.random.default_rng(12345)


def _fixture(golden_dir):
    with open(os.path.join(golden_dir, "block_format_examples.json")) as f:
        return json.load(f)


# ------------------------------------------------------------ block format --
def test_unpack_hand_examples(golden_dir):
    for case in _fixture(golden_dir)["byte_unpack"]:
        q = moe.unpack_codes(np.array([[case["byte"]]], dtype=np.uint8), case["bits"])
        assert q.ravel().tolist() == case["codes"]


def _const_bytes(bits, c, ncodes):
    per = 8 // bits
    byte = sum(c << (bits * p) for p in range(per))
    return np.full((1, ncodes // per), byte, dtype=np.uint8)


def _scale_bits(d, m, nblocks):
    s = np.empty((1, nblocks, 2), dtype=np.uint16)
    s[..., 0] = np.float16(d).view(np.uint16)
    s[..., 1] = np.float16(m).view(np.uint16)
    return s


def test_constant_block_closed_form(golden_dir):
    cb = _fixture(golden_dir)["constant_block"]
    for case in cb["cases"]:
        w = moe.dequantize(_const_bytes(case["bits"], case["c"], 32),
                           _scale_bits(cb["d"], cb["m"], 1), case["bits"])
        assert w.sum() == case["dot"]          # exact: every term is a dyadic rational


def _quantise_and_pack(w, d, m, bits):
    """Test-side inverse of the format: q = clamp(round((w-m)/d)), packed per the text."""
    rows, K = w.shape
    q = np.clip(np.rint((w - m.repeat(32, axis=1)) / d.repeat(32, axis=1)), 0, (1 << bits) - 1)
    q = q.astype(np.uint8)
    per = 8 // bits
    packed = np.zeros((rows, K // per), dtype=np.uint8)
    for j in range(K):
        packed[:, j // per] |= (q[:, j] << (bits * (j % per))).astype(np.uint8)
    s = np.empty((rows, K // 32, 2), dtype=np.uint16)
    s[..., 0] = d.astype(np.float16).view(np.uint16)
    s[..., 1] = m.astype(np.float16).view(np.uint16)
    return packed, s, q


@pytest.mark.parametrize("bits", [2, 4])
def test_quantise_dequantise_round_trip(bits):
    rows, K = 6, 128
    d = RNG.uniform(0.002, 0.02, size=(rows, K // 32)).astype(np.float16).astype(np.float64)
    m = (-1.5 * d).astype(np.float16).astype(np.float64)
    q_true = RNG.integers(0, 1 << bits, size=(rows, K))
    w = q_true * d.repeat(32, axis=1) + m.repeat(32, axis=1)
    packed, s, q = _quantise_and_pack(w, d, m, bits)
    assert np.array_equal(q, q_true)                    # codes recovered exactly
    assert np.array_equal(moe.dequantize(packed, s, bits), w)  # and the weights
    # an in-range w off the grid dequantises to within d/2
    w2 = w + RNG.uniform(-0.49, 0.49, size=w.shape) * d.repeat(32, axis=1)
    w2 = np.clip(w2, m.repeat(32, axis=1), m.repeat(32, axis=1) + ((1 << bits) - 1) * d.repeat(32, axis=1))
    p2, s2, _ = _quantise_and_pack(w2, d, m, bits)
    assert np.all(np.abs(moe.dequantize(p2, s2, bits) - w2) <= 0.5 * d.repeat(32, axis=1) + 1e-15)


def test_dequantised_weights_exact_in_fp32():
    # d has 11 significant bits and q <= 15, so d*q + m is an fp32 number
    d = RNG.uniform(0.002, 0.02, size=(64, 4)).astype(np.float16)
    m = (-7.5 * d.astype(np.float64)).astype(np.float16)
    s = np.stack([d.view(np.uint16), m.view(np.uint16)], axis=-1)
    codes = RNG.integers(0, 256, size=(64, 64), dtype=np.uint8)
    w = moe.dequantize(codes, s, 4)
    assert np.array_equal(w.astype(np.float32).astype(np.float64), w)


# ------------------------------------------------------------------ router --
def _brute_topk(l, k):
    """The unique k-subset S with (l_e > l_f) or (l_e == l_f and e < f) for e in S, f not in S."""
    E = len(l)
    found = []
    for S in itertools.combinations(range(E), k):
        rest = [f for f in range(E) if f not in S]
        if all(l[e] > l[f] or (l[e] == l[f] and e < f) for e in S for f in rest):
            found.append(S)
    assert len(found) == 1
    S = list(found[0])
    # slot order: larger logit first, then lower index
    S.sort(key=lambda e: (-l[e], e))
    return S


def test_topk_brute_force():
    for trial in range(300):
        E, k = 8, 3
        l = RNG.integers(-3, 4, size=E).astype(np.float64)  # many exact ties
        if trial % 2:
            l = RNG.standard_normal(E)
        assert moe.topk(l, k).tolist() == _brute_topk(l.tolist(), k)


def test_topk_all_equal_picks_lowest_indices():
    assert moe.topk(np.zeros(16), 5).tolist() == [0, 1, 2, 3, 4]


def test_duplicate_router_rows_tie_to_lower_index():
    H, E = 64, 12
    Wr = RNG.standard_normal((E, H)).astype(np.float32)
    x = RNG.standard_normal((3, H)).astype(np.float32)
    Wr[7] = Wr[2]
    Wr[9] = Wr[2]
    l = moe.logits(x, Wr, None, 4)
    assert np.all(l[:, 2] == l[:, 7]) and np.all(l[:, 2] == l[:, 9])
    for t in range(3):
        idx = moe.topk(l[t], 12).tolist()
        assert idx.index(2) < idx.index(7) < idx.index(9)


def _exact_logit(x, w, b=None):
    s = sum(Fraction(float(a)) * Fraction(float(c)) for a, c in zip(x, w))
    if b is not None:
        s += Fraction(float(b))
    return float(s)  # correctly rounded


def test_logits_match_exact_rationals_and_near_ties_are_exact():
    H, E, k = 48, 10, 3
    x = RNG.standard_normal((2, H)).astype(np.float32)
    Wr = RNG.standard_normal((E, H)).astype(np.float32)
    b = RNG.standard_normal(E).astype(np.float32)
    # row 4: same terms as row 3 with the last two coordinates' weights swapped
    # on a token whose x has equal entries there -> identical exact logit, which
    # a float64 matrix product may or may not reproduce; force a near tie too.
    x[:, -1] = x[:, -2]
    Wr[4] = Wr[3]
    Wr[4, -1], Wr[4, -2] = Wr[3, -2], Wr[3, -1]
    b[4] = b[3]
    Wr[3] *= 3.0
    Wr[4] *= 3.0
    b[3] = b[4] = 50.0
    l = moe.logits(x, Wr, b, k)
    for t in range(2):
        ex = [_exact_logit(x[t], Wr[e], b[e]) for e in range(E)]
        assert abs(l[t] - np.array(ex)).max() <= 1e-12 * max(1.0, np.abs(ex).max())
        assert l[t, 3] == ex[3] and l[t, 4] == ex[4]   # the near-tie was recomputed exactly
        assert l[t, 3] == l[t, 4]
        assert moe.topk(l[t], k)[:2].tolist() == [3, 4]


def test_bias_enters_selection_and_gates():
    H, E = 32, 6
    Wr = (0.01 * RNG.standard_normal((E, H))).astype(np.float32)
    x = RNG.standard_normal((1, H)).astype(np.float32)
    b = np.zeros(E, dtype=np.float32)
    b[5] = 100.0
    idx, g, _ = moe.route(x, Wr, b, 2)
    assert idx[0, 0] == 5 and g[0, 1] < math.exp(-90.0) and abs(g.sum() - 1) < 1e-15


def test_gates_sum_and_two_formulas():
    for _ in range(50):
        l = RNG.standard_normal(64) * 3
        idx = moe.topk(l, 10)
        g = moe.gates(l, idx)
        assert abs(g.sum() - 1.0) < 1e-15
        assert np.max(np.abs(g - moe.gates_via_full_softmax(l, idx))) < 1e-15
        assert np.all(np.diff(g) <= 0)


def test_gates_closed_form_k2():
    l = np.array([0.3, -1.2, 2.0, 0.7])
    idx = moe.topk(l, 2)
    assert idx.tolist() == [2, 3]
    g = moe.gates(l, idx)
    assert abs(g[0] - 1.0 / (1.0 + math.exp(0.7 - 2.0))) < 1e-16


# --------------------------------------------------------------------- FFN --
def test_silu_values():
    assert moe.silu(np.array([0.0]))[0] == 0.0
    assert abs(moe.silu(np.array([1.0]))[0] - 0.7310585786300049) < 1e-16
    assert abs(moe.silu(np.array([40.0]))[0] - 40.0) < 1e-12
    assert abs(moe.silu(np.array([-40.0]))[0]) < 1e-15
    assert moe.silu(np.array([-1000.0]))[0] == 0.0


def _const_expert(fx):
    H, I = fx["H"], fx["I"]
    gate = moe.dequantize(_const_bytes(2, fx["code"], H * I).reshape(I, H // 4),
                          _scale_bits(fx["d"], fx["m"], I * H // 32).reshape(I, H // 32, 2), 2)
    down = moe.dequantize(_const_bytes(2, fx["code"], H * I).reshape(H, I // 4),
                          _scale_bits(fx["d"], fx["m"], H * I // 32).reshape(H, I // 32, 2), 2)
    return gate, gate.copy(), down


def test_constant_expert_closed_form(golden_dir):
    fx = _fixture(golden_dir)["constant_expert"]
    Wg, Wu, Wd = _const_expert(fx)
    assert np.all(Wg == fx["w"]) and np.all(Wd == fx["w"])
    x = np.zeros((1, fx["H"]))
    x[0, 0] = 1.0
    y = moe.expert_ffn(x, Wg, Wu, Wd)
    w = fx["w"]
    closed = fx["I"] * w * (w / (1.0 + math.exp(-w))) * w
    assert abs(closed - fx["y_each"]) < 1e-20
    assert np.max(np.abs(y - closed)) < 1e-18


def _random_experts(E, H, I, bits):
    ex = []
    for _ in range(E):
        mats = []
        for rows, K in ((I, H), (I, H), (H, I)):
            codes = RNG.integers(0, 256, size=(rows, K * bits // 8), dtype=np.uint8)
            d = RNG.uniform(0.005, 0.02, size=(rows, K // 32)).astype(np.float16)
            m = (-1.5 * d.astype(np.float64)).astype(np.float16)
            s = np.stack([d.view(np.uint16), m.view(np.uint16)], axis=-1)
            mats.append(moe.dequantize(codes, s, bits))
        ex.append(tuple(mats))
    return ex


def test_one_hot_route_is_a_single_expert():
    ex = _random_experts(4, 64, 32, 2)
    x = RNG.standard_normal((3, 64))
    for e in range(4):
        idx = np.full((3, 1), e, dtype=np.int32)
        y = moe.moe_layer(x, idx, np.ones((3, 1)), lambda i: ex[i])
        assert np.array_equal(y, moe.expert_ffn(x, *ex[e]))


def test_routed_layer_equals_dense_mixture():
    E, H, I, k, T = 6, 64, 32, 3, 5
    ex = _random_experts(E, H, I, 4)
    x = RNG.standard_normal((T, H))
    idx = np.stack([RNG.permutation(E)[:k] for _ in range(T)]).astype(np.int32)
    g = RNG.uniform(0.1, 1.0, size=(T, k))
    y = moe.moe_layer(x, idx, g, lambda i: ex[i])
    # dense: every expert on every token (einsum over the stacked weights), then mix
    Wg = np.stack([e[0] for e in ex]); Wu = np.stack([e[1] for e in ex]); Wd = np.stack([e[2] for e in ex])
    a_g = np.einsum("eih,th->tei", Wg, x)
    a_u = np.einsum("eih,th->tei", Wu, x)
    hh = a_g * 0.5 * (1.0 + np.tanh(0.5 * a_g)) * a_u      # silu via tanh identity
    ye = np.einsum("ehi,tei->teh", Wd, hh)
    G = np.zeros((T, E))
    for t in range(T):
        G[t, idx[t]] = g[t]
    dense = np.einsum("te,teh->th", G, ye)
    assert moe.rel_rms(y, dense) < 1e-13


def test_combine_order_invariance():
    ys = RNG.standard_normal((10, 256))
    g = RNG.dirichlet(np.ones(10))
    base = moe.combine(ys, g)
    for _ in range(5):
        p = RNG.permutation(10)
        assert moe.rel_rms(moe.combine(ys[p], g[p]), base) < 1e-13


def test_rmsnorm_closed_form():
    z = RNG.standard_normal((4, 512)) * 3
    eps = 1e-6
    out = moe.rmsnorm_residual(z, np.zeros_like(z), eps)
    ms = np.mean(z * z, axis=1)
    assert np.allclose(np.mean(out * out, axis=1), ms / (ms + eps), rtol=1e-13, atol=0)
    # residual is added before the norm; the norm is scale-free up to eps
    out2 = moe.rmsnorm_residual(2.0 * z - 1.0, 1.0 + 0.0 * z, 0.0)
    assert np.allclose(out2, moe.rmsnorm_residual(z, 0 * z, 0.0), rtol=1e-14, atol=1e-15)


def test_stack_keeps_unit_rms():
    E, H, I, k = 8, 64, 32, 2
    layers = []
    for _ in range(3):
        ex = _random_experts(E, H, I, 2)
        Wr = (0.02 * RNG.standard_normal((E, H))).astype(np.float32)
        layers.append((Wr, None, (lambda ex: (lambda i: ex[i]))(ex)))
    x0 = RNG.standard_normal((2, H)).astype(np.float32)
    x, recs = moe.stack(x0, layers, k, 1e-6)
    assert len(recs) == 3
    assert np.allclose(np.sqrt(np.mean(x * x, axis=1)), 1.0, atol=1e-6)


# ----------------------------------------------------- stack composition --
# Two layers of four constant experts (every weight of a matrix equal) and
# constant router rows. With constant matrices the expert FFN collapses to a
# scalar of S = sum_h x_h: a_g = w_g S and a_u = w_u S on every row, so
# y_e = I w_d w_u S silu(w_g S) on every output element, and a constant router
# row alpha_e gives the logit alpha_e S. The residual stack is then a chain of
# plain scalar formulas, worked below in Python floats independently of the
# oracle's matrix code.
_SP_H, _SP_I = 64, 32
_SP_CODES = {0: (3, 2, 1), 1: (2, 3, 0), 2: (1, 3, 3), 3: (0, 0, 2)}   # expert -> (gate, up, down) Q2 code
_SP_ALPHA = ([2.0 ** -8, 2.0 ** -6, 2.0 ** -7, -2.0 ** -7], [-2.0 ** -6, 2.0 ** -8, 2.0 ** -7, 2.0 ** -6])
_SP_D, _SP_M = 2.0 ** -6, -1.5 * 2.0 ** -6     # w = d c + m = (c - 1.5) / 64


def _sp_layers():
    H, I = _SP_H, _SP_I

    def const(c, rows, K):
        return moe.dequantize(np.tile(_const_bytes(2, c, K), (rows, 1)),
                              np.tile(_scale_bits(_SP_D, _SP_M, K // 32), (rows, 1, 1)), 2)
    experts = {e: (const(g, I, H), const(u, I, H), const(d, H, I)) for e, (g, u, d) in _SP_CODES.items()}
    return [(np.tile(np.array(a, dtype=np.float32)[:, None], (1, H)), None, experts.__getitem__)
            for a in _SP_ALPHA]


def _sp_closed_form(x0, mistake=None):
    """Scalar walk of the stack; ``mistake`` switches in a plausible composition
    error: "norm_y" normalises y alone (residual dropped), "no_norm" passes
    x + y on without the norm."""
    w = lambda c: _SP_D * c + _SP_M
    silu = lambda a: a / (1.0 + math.exp(-a))
    x = [float(v) for v in x0]
    recs = []
    for alpha in _SP_ALPHA:
        S = sum(x)
        logit = [a * S for a in alpha]
        sel = sorted(range(4), key=lambda e: (-logit[e], e))[:2]      # 4 experts, by hand: value desc, index asc
        ex = [math.exp(logit[e] - logit[sel[0]]) for e in sel]
        g = [v / sum(ex) for v in ex]
        y = 0.0
        for gj, e in zip(g, sel):
            cg, cu, cd = _SP_CODES[e]
            y += gj * _SP_I * w(cd) * w(cu) * S * silu(w(cg) * S)
        recs.append((sel, g, y))
        z = [y] * len(x) if mistake == "norm_y" else [xi + y for xi in x]
        ms = sum(v * v for v in z) / len(z)
        x = z if mistake == "no_norm" else [v / math.sqrt(ms + 1e-6) for v in z]
    return np.array(x), recs


def test_stack_composition_closed_form():
    x0 = np.array([[0.5 + h / 64.0 for h in range(_SP_H)]], dtype=np.float32)
    x, recs = moe.stack(x0, _sp_layers(), 2, 1e-6)
    ref, ref_recs = _sp_closed_form(x0[0])
    for (x_in, idx, g, y), (sel, gs, ys) in zip(recs, ref_recs):
        assert idx[0].tolist() == sel
        assert np.allclose(g[0], gs, rtol=1e-13, atol=0)
        assert np.allclose(y[0], ys, rtol=1e-12, atol=1e-15)
    assert np.allclose(x[0], ref, rtol=1e-12, atol=0)
    # the pin discriminates: each plausible mistake moves the result far beyond the bound
    for bad in (_sp_closed_form(x0[0], "norm_y")[0], _sp_closed_form(x0[0], "no_norm")[0]):
        assert np.max(np.abs(bad - ref)) > 1e-2
    # routing layer 1 on the un-normalised residual sum changes its gates
    S_z = float(np.sum(x0[0] + ref_recs[0][2]))
    assert abs(S_z - float(np.sum(recs[1][0]))) > 1.0


def test_workload_stack_is_the_oracle_stack():
    """``oracle.workload.run_stack`` feeds generated layers to ``moe.stack``
    (one loop); the per-layer records agree with explicit single-layer calls."""
    from oracle import workload as W
    from synth import configs, gen
    cfg = configs.get(0).with_(L=2, residual=True)
    x0 = gen.tokens(0, cfg, 0).astype(np.float64)
    x, recs = W.run_stack(0, cfg, x0, 2)
    y0, i0, g0, _ = W.run_layer(0, cfg, x0, 0)
    assert np.array_equal(recs[0][1], i0) and np.array_equal(recs[0][3], y0)
    x1 = moe.rmsnorm_residual(x0, y0, cfg.eps)
    y1, i1, _, _ = W.run_layer(0, cfg, x1, 1)
    assert np.array_equal(recs[1][1], i1)
    assert np.array_equal(x, moe.rmsnorm_residual(x1, y1, cfg.eps))
