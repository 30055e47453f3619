"""GPU parity of nvfp4_gemm_grouped, the grouped expert decode (ignis,
"Models and artifacts", the model table: Flash-Next, 512 routed experts per
layer, ten chosen per token), against the oracle route by route."""
import numpy as np
import pytest
import torch

import oracle
from gpu_helpers import assert_gemm_close, x_from_dev
from nvfp4_weight_streaming_decode_b200 import abi, synth
from nvfp4_weight_streaming_decode_b200.workloads import make_matrix

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dev(cuda_device):
    from nvfp4_weight_streaming_decode_b200 import build
    build.build()
    abi.load()
    torch.cuda.set_device(cuda_device)
    return cuda_device


class Experts:
    """E experts of N x K as row blocks of one packed matrix (each block is a
    contiguous, aligned slice of both device planes)."""

    def __init__(self, dev, wid, E, N, K, exp=synth.EXP_UNIFORM_M4_2):
        assert N % 32 == 0
        self.E, self.N, self.K = E, N, K
        self.m = make_matrix(wid, 0, E * N, K, dev, exp)
        kc = -(-K // 64)
        qb, sb = (N // 32) * kc * 1024, (N // 32) * kc * 128
        self.gs = [synth.GSCALE * (1.0 + 0.125 * (e % 5)) for e in range(E)]
        mats = [(self.m.wq[e * qb:(e + 1) * qb], self.m.ws[e * sb:(e + 1) * sb], self.gs[e]) for e in range(E)]
        self.table = abi.expert_table(mats, dev)
        q, s = self.m.canonical(dev, wid)
        self.q, self.s = q.cpu().numpy(), s.cpu().numpy()

    def planes(self, e):
        return self.q[e * self.N:(e + 1) * self.N], self.s[e * self.N:(e + 1) * self.N]


def _routes(seed, M, T, E, distinct=True):
    rng = np.random.default_rng(seed)
    if distinct:
        return np.stack([rng.choice(E, T, replace=False) for _ in range(M)]).astype(np.int32)
    return rng.integers(0, E, (M, T)).astype(np.int32)


def _check(dev, ex, route, x_per_route, seed, rows_sample=None):
    M, T = route.shape
    X = synth.torch_activations(70, seed, M * T if x_per_route else M, ex.K, dev)
    r = torch.from_numpy(route).to(dev)
    Y = abi.gemm_grouped(X, r, ex.table, ex.E, ex.N, ex.K, x_per_route=x_per_route)
    torch.cuda.synchronize()
    Yh = Y.cpu().numpy()
    Xb = x_from_dev(X)
    sel = np.arange(ex.N) if rows_sample is None else rows_sample
    for m in range(M):
        for t in range(T):
            e = int(route[m, t])
            got = Yh[m, t][sel][None, :]
            if e < 0 or e >= ex.E:
                assert np.all(got == 0.0), (m, t, e)
                continue
            q, s = ex.planes(e)
            x = Xb[m * T + t if x_per_route else m][None, :]
            Yr, A = oracle.gemm_rows(x, q, s, ex.gs[e], sel)
            assert_gemm_close(got, Yr, A, f"route ({m},{t}) expert {e}")
    return Y


@pytest.mark.parametrize("M,T", [(1, 1), (1, 10), (3, 4), (8, 10), (8, 16)])
def test_grouped_matches_oracle(dev, M, T):
    ex = Experts(dev, 71, 40, 96, 320)
    _check(dev, ex, _routes(M * 100 + T, M, T, 40), False, M * 7 + T)


def test_grouped_per_route_inputs(dev):
    """x_per_route: each route has its own input row (the down projection)."""
    ex = Experts(dev, 72, 24, 64, 256)
    _check(dev, ex, _routes(5, 8, 6, 24), True, 9)


def test_grouped_shared_and_repeated_experts(dev):
    """Lanes sharing experts and a lane repeating one: one expert with more
    than 8 rows is cut into several groups."""
    ex = Experts(dev, 73, 8, 32, 128)
    route = np.zeros((8, 10), np.int32)
    route[:, 5:] = _routes(6, 8, 5, 8, distinct=False)
    _check(dev, ex, route, False, 10)


def test_grouped_invalid_routes(dev):
    ex = Experts(dev, 74, 6, 32, 64)
    route = _routes(7, 4, 3, 6)
    route[0, 1] = -1       # no expert: zero row, no flag
    assert abi.nvfp4_device_status() == 0
    _check(dev, ex, route, False, 11)
    assert abi.nvfp4_device_status() == 0
    route[2, 0] = 6        # id >= E: zero row, flagged
    _check(dev, ex, route, False, 12)
    assert abi.nvfp4_device_status() & 32


def test_grouped_flash_next_shape(dev):
    """512 experts of 768 x 2,048 (the gate/up shape read for Flash-Next),
    8 lanes x 10 picks, sampled rows; repeatable bit for bit."""
    ex = Experts(dev, 75, 512, 768, 2048)
    route = _routes(8, 8, 10, 512)
    rows = np.unique(np.concatenate([[0, 767], np.random.default_rng(3).integers(0, 768, 64)]))
    Y1 = _check(dev, ex, route, False, 13, rows)
    X = synth.torch_activations(70, 13, 8, 2048, dev)
    Y2 = abi.gemm_grouped(X, torch.from_numpy(route).to(dev), ex.table, 512, 768, 2048)
    torch.cuda.synchronize()
    assert torch.equal(Y1.view(torch.int32), Y2.view(torch.int32))


def test_grouped_errors(dev):
    ex = Experts(dev, 76, 4, 32, 64)
    X = synth.torch_activations(70, 1, 2, 64, dev)
    r = torch.zeros((2, 65), dtype=torch.int32, device=dev)
    Y = torch.empty((2, 65, 32), dtype=torch.float32, device=dev)
    s = torch.cuda.current_stream().cuda_stream
    assert abi.nvfp4_gemm_grouped(X.data_ptr(), 0, r.data_ptr(), 2, 65, ex.table.data_ptr(), 4, Y.data_ptr(), 32, 64, s) == abi.NVFP4_ERR_ARG
    assert abi.nvfp4_gemm_grouped(X.data_ptr(), 0, r.data_ptr(), 9, 2, ex.table.data_ptr(), 4, Y.data_ptr(), 32, 64, s) == abi.NVFP4_ERR_M
    assert abi.nvfp4_gemm_grouped(X.data_ptr() + 2, 0, r.data_ptr(), 2, 2, ex.table.data_ptr(), 4, Y.data_ptr(), 32, 64, s) == abi.NVFP4_ERR_ALIGN
