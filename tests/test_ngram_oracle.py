"""Pins of the n-gram row-gather oracle (``oracle/ngram.py``): its generator
against SplitMix64's published outputs, the row reduction against closed
forms, and the hash's use of the ids (order, 32-bit patterns)."""
import json
import os

import numpy as np

from oracle import moe, ngram


def _vectors(golden_dir):
    with open(os.path.join(golden_dir, "splitmix64_vectors.json")) as f:
        return json.load(f)["vectors"]


def test_generator_matches_published_splitmix64_outputs(golden_dir):
    for v in _vectors(golden_dir):
        if "outputs_hex" in v:
            want = [int(h, 16) for h in v["outputs_hex"]]
        else:
            want = v["outputs"]
        assert ngram.splitmix64(v["seed"], len(want)) == want


def test_hash_starts_from_the_generators_first_output(golden_dir):
    # with the three mixing steps peeled off, the hash's start is output 0
    seed0 = next(v for v in _vectors(golden_dir) if v["seed"] == 0)
    h0 = int(seed0["outputs_hex"][0], 16)
    assert ngram.ngram_hash(0, 1, 2, 3) == ngram.mix64(ngram.mix64(ngram.mix64(h0 ^ 1) ^ 2) ^ 3)


def test_row_reduction_closed_forms():
    rs = np.random.default_rng(3)
    xs = [int(v) for v in rs.integers(0, 2**63, 200, dtype=np.int64)] + [0, 2**64 - 1, 2**63]
    for x in xs:
        assert ngram.reduce_rows(x, 1) == 0
        for k in (1, 7, 22, 31):
            assert ngram.reduce_rows(x, 1 << k) == x >> (64 - k)    # top k bits
        R = 1_000_003
        r = ngram.reduce_rows(x, R)
        assert 0 <= r < R and r * 2**64 <= x * R < (r + 1) * 2**64
    # boundaries for R = 3: the first x of row 1 is ceil(2^64 / 3)
    b = -(-2**64 // 3)
    assert ngram.reduce_rows(b - 1, 3) == 0 and ngram.reduce_rows(b, 3) == 1
    assert ngram.reduce_rows(2**64 - 1, 3) == 2


def test_rows_depend_on_every_id_in_order():
    base = ngram.token_rows(7, (11, 22, 33), 1 << 20)
    assert len(base) == 16 and all(0 <= r < (1 << 20) for r in base)
    assert ngram.token_rows(7, (11, 22, 33), 1 << 20) == base               # a function of its inputs
    for other in ((22, 11, 33), (11, 33, 22), (12, 22, 33), (11, 22, 34)):
        assert ngram.token_rows(7, other, 1 << 20) != base
    assert ngram.token_rows(8, (11, 22, 33), 1 << 20) != base               # the seed enters
    # an id is used as its 32-bit pattern: -1 and 2^32 - 1 are the same id
    assert ngram.token_rows(7, (-1, 5, 6), 1000) == ngram.token_rows(7, (2**32 - 1, 5, 6), 1000)
    # 16 distinct draws of one token spread over a large table
    assert len(set(base)) == 16


def test_row_draws_are_uniform():
    counts = np.zeros(8, dtype=np.int64)
    for t in range(2000):
        for r in ngram.token_rows(1, (t, t + 1, t + 2), 8):
            counts[r] += 1
    expected = 2000 * 16 / 8
    assert np.all(np.abs(counts - expected) < 5 * np.sqrt(expected))


def test_gather_is_the_block_format_of_the_selected_rows():
    rs = np.random.default_rng(4)
    R, D = 50, 64
    codes = rs.integers(0, 256, (R, D // 2), dtype=np.uint8)
    d = rs.uniform(0.002, 0.01, (R, D // 32)).astype(np.float16)
    m = (-7.5 * d.astype(np.float64)).astype(np.float16)
    scales = np.stack([d.view(np.uint16), m.view(np.uint16)], axis=-1)
    idx = np.array([[3, 49, 0], [7, 7, 1]])
    w = ngram.gather(codes, scales, idx)
    assert w.shape == (2, 3, D)
    full = moe.dequantize(codes, scales, 4)
    assert np.array_equal(w[0, 1], full[49]) and np.array_equal(w[1, 0], w[1, 1])
    # code j of a row is the low nibble of byte j/2 for even j
    assert w[0, 0, 0] == (codes[3, 0] & 15) * d[3, 0].astype(np.float64) + m[3, 0].astype(np.float64)
    assert w[0, 0, 1] == (codes[3, 0] >> 4) * d[3, 0].astype(np.float64) + m[3, 0].astype(np.float64)
