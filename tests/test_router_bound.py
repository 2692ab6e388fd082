"""The inequality the prefill router's candidate pass rests on, checked on the CPU
with its quantisation rule restated.

A token row x (bf16 or fp32 values) and a router row w (fp32) are quantised to
16-bit fixed point: s = fp32(max|row| / 32639), inv = fp32(1 / s), codes
X = rint(fp32(v * inv)) clamped to +-32639. The approximate logit
a = (sum X W) * (s_x * s_w) (+ b), formed from exact integer sums, differs from
the exact logit by at most
    B = 0.51 (s_x |w|_1 + s_w (|x|_1 + 0.51 H s_x))   (* (1 + 1e-9) + 1e-12 (|a| + 1)),
because every value lies within 0.51 of its scale from its quantised value.
With tau the k-th largest a of a token and B_max its largest bound, every expert
of the exact top-k then has a + B >= tau - B_max: the candidate set the float64
selection runs on contains the exact top-k.

The reference logits are float64 dot products of exact fp32 x fp32 products;
their own rounding is below 3e-13 sum|x w|, while B >= 1.5e-5 sum|x w|, so a
margin of 1e-7 B covers it."""
import numpy as np
import pytest

XMAX = 32639
SLACK = 1.0 - 1e-7


def quantise(rows):
    """Per-row scale (fp32) and int64 codes, in the router kernel's arithmetic."""
    rows = np.asarray(rows, dtype=np.float32)
    amax = np.max(np.abs(rows), axis=1).astype(np.float32)
    s = np.where(amax > 0, (amax / np.float32(XMAX)).astype(np.float32), np.float32(0)).astype(np.float32)
    with np.errstate(divide="ignore"):
        inv = np.where(s > 0, (np.float32(1) / s).astype(np.float32), np.float32(0)).astype(np.float32)
    prod = (rows * inv[:, None]).astype(np.float32)
    X = np.clip(np.rint(prod), -XMAX, XMAX).astype(np.int64)
    return s, X


def approx_and_bound(x, w, bias=None):
    x = np.asarray(x, dtype=np.float32)
    w = np.asarray(w, dtype=np.float32)
    H = x.shape[1]
    sx, X = quantise(x)
    sw, W = quantise(w)
    q = X @ W.T                                            # exact: |q| < 2048 * 32639^2 < 2^41
    a = q.astype(np.float64) * (sx.astype(np.float64)[:, None] * sw.astype(np.float64)[None, :])
    if bias is not None:
        a = a + np.asarray(bias, dtype=np.float32).astype(np.float64)[None, :]
    n1x = np.abs(x.astype(np.float64)).sum(axis=1)
    n1w = np.abs(w.astype(np.float64)).sum(axis=1)
    b = 0.51 * (sx.astype(np.float64)[:, None] * n1w[None, :]
                + sw.astype(np.float64)[None, :] * (n1x[:, None] + 0.51 * H * sx.astype(np.float64)[:, None]))
    B = b * (1.0 + 1e-9) + 1e-12 * (np.abs(a) + 1.0)
    exact = x.astype(np.float64) @ w.astype(np.float64).T
    if bias is not None:
        exact = exact + np.asarray(bias, dtype=np.float32).astype(np.float64)[None, :]
    return a, B, exact


def bf16(v):
    """Round float32 values to bf16 (nearest even), returned as float32."""
    u = np.asarray(v, dtype=np.float32).view(np.uint32).astype(np.uint64)
    u = ((u + 0x7FFF + ((u >> 16) & 1)) >> 16) << 16
    return u.astype(np.uint32).view(np.float32)


def test_bound_holds_on_router_shaped_rows():
    rs = np.random.default_rng(7)
    x = bf16(rs.standard_normal((64, 2048)))
    w = (0.02 * rs.standard_normal((96, 2048))).astype(np.float32)
    a, B, exact = approx_and_bound(x, w, bias=rs.standard_normal(96))
    assert np.all(np.abs(a - exact) <= SLACK * B)
    # the bound is not vacuous: well under 1 % of the logit spread (a typical
    # gap between the k-th and (k+1)-th logit of a token is several percent)
    assert np.median(B) < 1e-2 * np.std(exact)


@pytest.mark.parametrize("kind", ["heavy_tail", "cancel", "clamp_edge", "tiny_and_huge", "zeros"])
def test_bound_holds_on_adversarial_rows(kind):
    rs = np.random.default_rng(11)
    H = 2048
    if kind == "heavy_tail":
        x = (rs.standard_cauchy((16, H)) * 1e-2).astype(np.float32)
        w = (rs.standard_cauchy((16, H)) * 1e-3).astype(np.float32)
    elif kind == "cancel":
        # exact logit near zero from large terms of both signs
        x = np.tile(np.array([1.0, -1.0], dtype=np.float32), (16, H // 2)) * rs.uniform(0.5, 2.0, (16, 1)).astype(np.float32)
        w = np.tile(np.array([1.0, 1.0], dtype=np.float32), (16, H // 2)) + (1e-4 * rs.standard_normal((16, H))).astype(np.float32)
    elif kind == "clamp_edge":
        # values at and just below the row maximum (codes at +-32639)
        x = rs.choice(np.array([-3.0, 3.0, 2.9999998, -2.9999998], dtype=np.float32), (16, H))
        w = rs.choice(np.array([-0.5, 0.5, 0.49999997], dtype=np.float32), (16, H))
    elif kind == "tiny_and_huge":
        # one large value per row, the rest far below one quantisation step
        x = (1e-9 * rs.standard_normal((16, H))).astype(np.float32)
        x[:, 5] = 1e3
        w = (1e-9 * rs.standard_normal((16, H))).astype(np.float32)
        w[:, 7] = 1.0
    else:
        x = np.zeros((4, H), dtype=np.float32)
        w = (0.02 * rs.standard_normal((4, H))).astype(np.float32)
        w[1] = 0.0
    a, B, exact = approx_and_bound(x, w)
    assert np.all(np.abs(a - exact) <= SLACK * B), kind


@pytest.mark.parametrize("with_bias", [False, True])
def test_candidates_contain_the_exact_top_k(with_bias):
    """512 experts, top-10, the router's workload shape: the candidate rule keeps
    the exact top-k (value descending, lower index on ties) of every token, and
    the candidate sets stay small."""
    rs = np.random.default_rng(3)
    T, E, H, k = 48, 512, 2048, 10
    x = bf16(rs.standard_normal((T, H)))
    w = (0.02 * rs.standard_normal((E, H))).astype(np.float32)
    w[17] = w[300]                      # an exact tie between two experts
    bias = rs.standard_normal(E) if with_bias else None
    a, B, exact = approx_and_bound(x, w, bias)
    sizes = []
    for t in range(T):
        tau = np.sort(a[t])[::-1][k - 1]
        cand = set(np.nonzero(a[t] + B[t] >= tau - B[t].max())[0].tolist())
        top = sorted(range(E), key=lambda e: (-exact[t, e], e))[:k]
        assert set(top) <= cand, t
        sizes.append(len(cand))
    assert max(sizes) <= 64 and np.median(sizes) <= k + 4
