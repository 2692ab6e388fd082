"""The seeded generator against published vectors and its own stated definitions."""
import json
import os

import numpy as np

from synth import configs, gen, rng


def test_splitmix64_published_vectors(golden_dir):
    with open(os.path.join(golden_dir, "splitmix64_vectors.json")) as f:
        vec = json.load(f)["vectors"]
    a = vec[0]
    assert [f"{v:016x}" for v in rng.sequential(a["seed"], 3)] == a["outputs_hex"]
    b = vec[1]
    assert rng.sequential(b["seed"], 5) == b["outputs"]


def test_counter_form_equals_sequential_form():
    for key in (0, 1234567, 0xDEADBEEFCAFEF00D):
        seq = rng.sequential(key, 40)
        ctr = [int(v) for v in rng.outputs(key, 0, 40)]
        assert seq == ctr
        assert [int(v) for v in rng.outputs(key, 17, 5)] == seq[17:22]


def test_stream_keys_distinct():
    keys = {rng.stream_key(0, c, l, e, w) for c in range(5) for l in range(3)
            for e in range(4) for w in range(1, 11)}
    assert len(keys) == 5 * 3 * 4 * 10


def test_code_bytes_are_little_endian_words():
    key = rng.stream_key(7, 1, 2, 3, 1)
    b = gen.code_bytes(key, 32)
    w = rng.outputs(key, 0, 4)
    for i in range(4):
        assert int.from_bytes(bytes(b[8 * i:8 * i + 8]), "little") == int(w[i])


def test_codes_uniform():
    b = gen.code_bytes(rng.stream_key(1, 0, 0, 0, 1), 1 << 18)
    for bits in (2, 4):
        per = 8 // bits
        q = np.stack([(b >> (bits * p)) & ((1 << bits) - 1) for p in range(per)]).ravel()
        cnt = np.bincount(q, minlength=1 << bits)
        exp = q.size / (1 << bits)
        chi2 = float(np.sum((cnt - exp) ** 2 / exp))
        assert chi2 < 60.0, chi2


def test_scale_pairs_definition():
    for fmt in (configs.Q2, configs.Q4):
        f = configs.FORMATS[fmt]
        s = gen.scale_pairs(rng.stream_key(3, 0, 0, 0, 4), 4096, fmt)
        d = s[:, 0].view(np.float16).astype(np.float64)
        m = s[:, 1].view(np.float16).astype(np.float64)
        assert d.min() >= f.d_lo * (1 - 2 ** -10) and d.max() <= f.d_hi * (1 + 2 ** -10)
        # m is the fp16 rounding of -c*d; |m + c*d| within half an fp16 ulp of m
        ulp = np.spacing(np.abs(m).astype(np.float16)).astype(np.float64)
        assert np.all(np.abs(m + f.m_coef * d) <= 0.5 * ulp)
        assert abs(d.mean() - 0.5 * (f.d_lo + f.d_hi)) < 0.02 * f.d_hi


def test_gaussians_moments():
    z = gen.gaussians(rng.stream_key(5, 0, 0, 0, 9), 1_000_001)
    assert z.shape == (1_000_001,)
    assert abs(z.mean()) < 5e-3
    assert abs(z.std() - 1.0) < 5e-3
    assert abs(np.mean(z ** 4) - 3.0) < 0.05


def test_bf16_rounding():
    x = np.array([1.0, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -2.5, 1.0 + 2 ** -8 + 2 ** -20],
                 dtype=np.float32)
    b = gen.f32_to_bf16_bits(x)
    # 1+2^-8 is a tie -> even (1.0); 1+3*2^-8 is a tie -> even (1+2^-6... i.e. 0x3F82)
    assert [int(v) for v in b] == [0x3F80, 0x3F80, 0x3F82, 0xC020, 0x3F81]
    assert np.array_equal(gen.bf16_bits_to_f32(b)[[0, 3]], np.array([1.0, -2.5], np.float32))


def test_correlated_tokens():
    cfg = configs.get(3)
    x = gen.tokens(0, cfg).astype(np.float64)
    assert x.shape == (8, 2048)
    c = [np.corrcoef(x[0], x[i])[0, 1] for i in range(1, 8)]
    assert all(0.75 < v < 0.85 for v in c)


def test_expert_matrix_shapes():
    cfg = configs.get(0)
    raw = gen.expert(0, cfg, 0, 5)
    assert raw["gate_codes"].shape == (cfg.I, cfg.H // 4)
    assert raw["down_codes"].shape == (cfg.H, cfg.I // 4)
    assert raw["up_scales"].shape == (cfg.I, cfg.H // 32, 2)
    cfg4 = configs.get(4)
    assert cfg4.expert_bytes() == 2_949_120
    assert configs.get(1).expert_bytes() == 1_769_472


def test_mixed_bit_stack_layers_are_the_uniform_layers():
    """A mixed-bit stack (a block format per layer) draws layer l's codes and
    scales from the same streams as the uniform stack of layer l's format,
    and the oracle dequantises each layer with that layer's bits."""
    from oracle import workload as W
    base = configs.get(0).with_(L=3, residual=True)
    mixed = base.with_(fmt_layers=(configs.Q2, configs.Q4, configs.Q2))
    assert mixed.for_layer(1).fmt == configs.Q4 and mixed.for_layer(1).fmt_layers == ()
    assert base.for_layer(1) is base
    for l in range(3):
        uni = base.with_(fmt=mixed.fmt_layers[l])
        a, b = gen.expert(0, mixed, l, 7), gen.expert(0, uni, l, 7)
        assert a.keys() == b.keys()
        for n in a:
            assert np.array_equal(a[n], b[n]), (l, n)
        bits = 8 * a["gate_codes"].shape[1] // base.H
        assert bits == mixed.fmt_layers[l]
        for wa, wb in zip(W.Layer(0, mixed, l).expert(7), W.Layer(0, uni, l).expert(7)):
            assert np.array_equal(wa, wb)
    # the Q4 layer really is four-bit: 16 distinct code levels per block
    w = W.Layer(0, mixed, 1).expert(3)[0]
    blk = w[0, :32]
    assert len(np.unique(blk)) > 4


def test_ngram_inputs():
    """A chunk's triples are the sliding windows of one id sequence drawn over
    the vocabulary; table rows are streams keyed by their row index."""
    nc = configs.NGRAM.with_(T=500)
    ids = gen.ngram_ids(0, nc, 0)
    assert ids.shape == (500, 3) and ids.dtype == np.int32
    assert np.array_equal(ids[1:, 0], ids[:-1, 1]) and np.array_equal(ids[1:, 1], ids[:-1, 2])
    assert ids.min() >= 0 and ids.max() < nc.vocab
    assert not np.array_equal(ids, gen.ngram_ids(0, nc, 1))                 # steps differ
    codes, scales = gen.ngram_rows(0, nc, 0, [7, 7, 8])
    assert codes.shape == (3, nc.D // 2) and scales.shape == (3, nc.D // 32, 2)
    assert np.array_equal(codes[0], codes[1]) and not np.array_equal(codes[0], codes[2])
    d = scales[:, :, 0].view(np.float16).astype(np.float64)
    m = scales[:, :, 1].view(np.float16).astype(np.float64)
    assert np.all((d >= 0.002 * (1 - 2**-10)) & (d <= 0.01 * (1 + 2**-10)))
    assert np.array_equal(m, (-7.5 * d).astype(np.float16).astype(np.float64))
