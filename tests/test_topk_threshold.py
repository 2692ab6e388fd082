"""The candidate threshold of the warp top-k, checked on the CPU with its rule
restated.

Expert e sits on lane e % 32 of a warp. Every float64 logit gets a 32-bit key:
the top 32 bits of its float64 pattern, made order-preserving as an unsigned
integer; a high word of 0x80000000 (-0 and the smallest negative subnormals)
is taken as that of +0, and NaN as -infinity (its rank). The threshold is the
k-th largest of the 32 per-lane maximum keys
(ties by lane); every key at or above it is a candidate, and the exact ranking
(logit descending, lower index on ties) runs on the candidates only. The
candidate set must contain the exact top-k for any logits; it should stay small
for router-like logits."""
import numpy as np
import pytest


def keys(logits):
    f = np.asarray(logits, dtype=np.float64)
    f = np.where(np.isnan(f), -np.inf, f)
    hi = (f.view(np.uint64) >> np.uint64(32)).astype(np.uint64)
    hi = np.where(hi == np.uint64(0x80000000), np.uint64(0), hi)
    return np.where(hi & np.uint64(0x80000000), ~hi & np.uint64(0xFFFFFFFF), hi | np.uint64(0x80000000))


def rank_key(v):
    """Selection order: value descending (NaN lowest), index ascending."""
    return -np.inf if np.isnan(v) else v


def candidates(logits, k):
    E = len(logits)
    M = (E + 31) // 32
    key = np.zeros(32 * M, dtype=np.uint64)    # 0 marks an empty slot
    key[:E] = keys(logits)
    lane_max = key.reshape(M, 32).max(axis=0)
    order = sorted(range(32), key=lambda l: (-int(lane_max[l]), l))
    thr = lane_max[order[k - 1]]
    return {e for e in range(E) if key[e] != 0 and key[e] >= thr}


def exact_top_k(logits, k):
    return sorted(range(len(logits)), key=lambda e: (-rank_key(logits[e]), e))[:k]


@pytest.mark.parametrize("kind", ["router", "ties", "degenerate", "signed_zero", "one_lane", "tiny", "nan"])
def test_candidates_contain_the_exact_top_k(kind):
    rs = np.random.default_rng(5)
    for trial in range(300):
        E = int(rs.choice([16, 33, 64, 100, 512, 1000, 1024]))
        k = int(rs.integers(1, min(16, E) + 1))
        if kind == "router":
            v = 0.9 * rs.standard_normal(E)
        elif kind == "ties":
            v = np.round(rs.standard_normal(E), 1)
        elif kind == "degenerate":
            v = np.zeros(E)
            v[rs.integers(0, E, 3)] = 1.0
        elif kind == "signed_zero":
            v = np.where(rs.random(E) < 0.5, -0.0, 0.0)
            v[rs.integers(0, E, 2)] = -1.0
        elif kind == "tiny":
            # negative subnormals whose high word is 0x80000000 share +0's key
            v = np.where(rs.random(E) < 0.5, -5e-324 * rs.integers(1, 1000, E), 0.0)
            v[rs.integers(0, E, 3)] = 1e-310
        elif kind == "nan":
            v = rs.standard_normal(E)
            v[rs.integers(0, E, max(1, E // 4))] = np.nan
        else:
            v = rs.standard_normal(E)
            v[np.arange(0, E, 32)] += 10.0       # the largest logits all on lane 0
        assert set(exact_top_k(v, k)) <= candidates(v, k), (kind, trial, E, k)


def test_router_logits_give_few_candidates():
    rs = np.random.default_rng(9)
    sizes = [len(candidates(0.9 * rs.standard_normal(512), 10)) for _ in range(500)]
    assert np.mean(sizes) < 14 and max(sizes) <= 64


def test_signed_zero_ties_go_to_the_lower_index():
    # -0.0 and +0.0 are equal logits: with keys that told them apart the
    # threshold would fall between them and drop the lower-index -0.0 expert
    v = np.array([-0.0] * 8 + [0.0] * 40 + [-1.0] * 16)
    assert exact_top_k(v, 10) == list(range(10))
    assert set(range(10)) <= candidates(v, 10)
