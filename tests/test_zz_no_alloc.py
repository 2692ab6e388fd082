"""The fixed-scratch router entry point (no workspace, nothing allocated)
against qmoe_route on the same inputs. Collected last on purpose: it must
also pass after every other GPU test has run in the same process."""
import numpy as np
import pytest
import torch

import quantised_expert_decode_b200 as q
from synth import configs, gen
from tests.gpu_util import route, status_word

pytestmark = pytest.mark.gpu
SEED = 0


def _fixed(Wr, bias, x, k):
    T, H = x.shape
    E = Wr.shape[0]
    idx = torch.full((T, k), -1, dtype=torch.int32, device="cuda")
    gate = torch.full((T, k), float("nan"), dtype=torch.float32, device="cuda")
    st = status_word()
    q.qmoe_route_fixed(Wr, bias, x, T, H, E, k, idx, gate, st)
    torch.cuda.synchronize()
    assert q.qmoe_read_status(st) == 0
    return idx, gate


@pytest.mark.parametrize("cid,T", [(1, 1), (3, 8), (0, 3)])
def test_fixed_scratch_router_matches_workspace_router(cid, T):
    cfg = configs.get(cid)
    Wr = torch.from_numpy(gen.router(SEED, cfg, 0)).cuda()
    for step in range(2):   # two calls in a row: each completed call leaves the ticket at zero
        x = torch.from_numpy(gen.tokens(SEED, cfg, step, T=T)).cuda()
        i1, g1 = _fixed(Wr, None, x, cfg.k)
        i0, g0 = route(Wr, None, x, cfg.k)
        assert torch.equal(i1, i0), (cid, step)
        assert torch.equal(g1, g0), (cid, step)


def test_fixed_scratch_router_at_its_maximum_size_with_bias():
    E, H, k, T = 1024, 256, 16, 8
    rs = np.random.default_rng(5)
    Wr = torch.from_numpy((0.02 * rs.standard_normal((E, H))).astype(np.float32)).cuda()
    bias = torch.from_numpy(rs.standard_normal(E).astype(np.float32)).cuda()
    for _ in range(2):
        x = torch.from_numpy(rs.standard_normal((T, H)).astype(np.float32)).cuda()
        i1, g1 = _fixed(Wr, bias, x, k)
        i0, g0 = route(Wr, bias, x, k)
        assert torch.equal(i1, i0)
        assert torch.equal(g1, g0)


def test_fixed_scratch_router_refuses_sizes_beyond_its_array():
    lib = q.lib()
    E, H, k = 1024, 256, 4
    Wr = torch.zeros((E + 1, H), dtype=torch.float32, device="cuda")
    x = torch.zeros((9, H), dtype=torch.float32, device="cuda")
    idx = torch.zeros((9, k), dtype=torch.int32, device="cuda")
    gate = torch.zeros((9, k), dtype=torch.float32, device="cuda")
    st = status_word()
    args = (Wr.data_ptr(), None, x.data_ptr())
    tail = (idx.data_ptr(), gate.data_ptr(), st.data_ptr(), None)
    assert lib.qmoe_route_fixed(*args, 9, H, E, k, *tail) == 3          # T > 8
    assert lib.qmoe_route_fixed(*args, 1, H, E + 1, k, *tail) == 3      # E > 1024
    assert lib.qmoe_route_fixed(*args, 1, H, E, 17, *tail) == 3         # k > 16
    assert lib.qmoe_route_fixed(None, None, x.data_ptr(), 1, H, E, k, *tail) == 1
