"""GPU parity of the n-gram row gather (``qmoe_ngram_gather``) against the
oracle: row indices bit for bit, dequantised values exactly (the block
format's values are exact in fp32)."""
import numpy as np
import pytest
import torch

from oracle import ngram
from quantised_expert_decode_b200 import _lib as L
from synth import configs, device, gen

pytestmark = pytest.mark.gpu
SEED = 0


def _table(R, D, rs):
    codes = rs.integers(0, 256, (R, D // 2), dtype=np.uint8)
    d = rs.uniform(0.002, 0.01, (R, D // 32)).astype(np.float16)
    m = (-7.5 * d.astype(np.float64)).astype(np.float16)
    scales = np.stack([d.view(np.uint16), m.view(np.uint16)], axis=-1)
    return codes, scales


def _run(ngrams, seed, codes_d, scales_d, R, D, want_rows=True):
    T = ngrams.shape[0]
    ng = torch.from_numpy(np.ascontiguousarray(ngrams, dtype=np.int32)).cuda()
    out = torch.full((T, 16, D), float("nan"), dtype=torch.float32, device="cuda")
    rows = torch.full((T, 16), -1, dtype=torch.int32, device="cuda") if want_rows else None
    L.qmoe_ngram_gather(ng, T, seed, codes_d, scales_d, R, D, out, rows)
    torch.cuda.synchronize()
    return out.cpu().numpy(), None if rows is None else rows.cpu().numpy()


@pytest.mark.parametrize("R,D,T", [(1000, 64, 37), (1, 32, 5), (4099, 288, 3), (257, 8192, 2)])
def test_gather_matches_oracle(R, D, T):
    rs = np.random.default_rng(R + D + T)
    codes, scales = _table(R, D, rs)
    ngrams = rs.integers(-2**31, 2**31, (T, 3), dtype=np.int64).astype(np.int32)
    ngrams[0] = (-1, 0, 2**31 - 1)
    cd = torch.from_numpy(codes).cuda()
    sd = torch.from_numpy(scales.view(np.int16)).cuda()
    seed = 0xDEADBEEFCAFEF00D
    out, rows = _run(ngrams, seed, cd, sd, R, D)
    want_rows = ngram.rows(seed, ngrams, R)
    assert np.array_equal(rows, want_rows)
    want = ngram.gather(codes, scales, want_rows)
    assert np.array_equal(out, want.astype(np.float32))          # exact values
    assert np.array_equal(out.astype(np.float64), want)
    # the row output is optional
    out2, _ = _run(ngrams, seed, cd, sd, R, D, want_rows=False)
    assert np.array_equal(out2, out)


def test_full_size_table():
    """2^22 rows of 256 (a billion elements, one layer of the pages' table)
    and a 4096-token chunk: every token's 16 rows bit for bit, and the values
    of 128 sampled (token, slot) pairs exactly against rows drawn on the host."""
    nc = configs.NGRAM
    codes_d, scales_d = device.ngram_table(SEED, nc)
    ngrams = gen.ngram_ids(SEED, nc, 0)
    out, rows = _run(ngrams, SEED, codes_d, scales_d, nc.R, nc.D)
    want_rows = ngram.rows(SEED, ngrams, nc.R)
    assert np.array_equal(rows, want_rows)
    rs = np.random.default_rng(1)
    picks = [(int(t), int(i)) for t, i in zip(rs.integers(0, nc.T, 128), rs.integers(0, 16, 128))]
    picks += [(0, 0), (nc.T - 1, 15)]
    sel = np.array([want_rows[t, i] for t, i in picks])
    codes, scales = gen.ngram_rows(SEED, nc, 0, sel)
    want = ngram.gather(codes, scales, np.arange(len(sel)))
    got = np.stack([out[t, i] for t, i in picks])
    assert np.array_equal(got.astype(np.float64), want)
    # the device table is the host generator's table
    assert np.array_equal(codes_d[sel[:8]].cpu().numpy(), codes[:8])
    assert np.array_equal(scales_d[sel[:8]].cpu().numpy().view(np.uint16), scales[:8])

