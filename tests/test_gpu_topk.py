"""GPU parity of nvfp4_topk (ignis README, "What sets it apart", "Speculative
decoding (DFlash2)": the row-split top-k after the output head, bit-identical
answer) against the oracle: indices exact, values bit for bit."""
import numpy as np
import pytest
import torch

import oracle
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


def _logits(seed, rows, V, ties=False):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((rows, V)).astype(np.float32)
    if ties:
        x = np.where(rng.random((rows, V)) < 0.5, (rng.integers(-8, 8, (rows, V)) / 2.0).astype(np.float32), x)
    return x


def _check(dev, x, k, V=None, ldv_pad=0):
    rows, V0 = x.shape
    V = V0 if V is None else V
    ldv = -(-(V0 + ldv_pad) // 4) * 4  # the row stride must be a multiple of 4 floats
    host = np.zeros((rows, ldv), np.float32)
    host[:, :V0] = x
    host[:, V0:] = np.float32(3e38)  # past V: never selected
    t = torch.from_numpy(host).to(dev)
    gv, gi = abi.topk(t, k, V)
    torch.cuda.synchronize()
    ov, oi = oracle.topk(host, k, V)
    gi, gv = gi.cpu().numpy(), gv.cpu().numpy()
    assert np.array_equal(gi, oi), (rows, V, k)
    assert np.array_equal(gv.view(np.uint32), ov.view(np.uint32)), (rows, V, k)
    return gv, gi


@pytest.mark.parametrize("rows,V,k", [
    (1, 1, 1), (1, 7, 7), (2, 64, 64), (3, 1000, 1), (3, 1000, 7), (8, 4099, 8), (1, 4097, 64),
    (8, 151936, 1), (8, 151936, 7), (8, 151936, 8), (8, 151936, 64), (1, 151936, 8), (1, 151936, 64),
    (4, 151937, 5), (64, 20000, 16), (1, 1 << 20, 8), (2, 300, 64), (1, 1025, 3),
])
def test_matches_oracle(dev, rows, V, k):
    _check(dev, _logits(rows * 1000003 + V * 7 + k, rows, V, ties=(V % 2 == 0)), k)


@pytest.mark.parametrize("rows,V,k", [(8, 151936, 8), (3, 5000, 64), (1, 70000, 33)])
def test_heavy_ties_at_threshold(dev, rows, V, k):
    """Values from a handful of levels: thousands tie at the k-th value, so the
    tie break by index (the second radix select) decides the answer."""
    rng = np.random.default_rng(V + k)
    x = rng.integers(0, 4, (rows, V)).astype(np.float32)
    _check(dev, x, k)


def test_constant_rows_take_lowest_indices(dev):
    x = np.full((8, 151936), -2.5, np.float32)
    gv, gi = _check(dev, x, 64)
    assert (gi == np.arange(64)).all()


def test_special_values(dev):
    """NaNs of both signs and payloads, infinities, signed zeros and
    subnormals scattered through rows of normal values."""
    rng = np.random.default_rng(17)
    rows, V = 4, 6000
    x = rng.standard_normal((rows, V)).astype(np.float32)
    specials = np.array([0x7FC00000, 0x7FC00001, 0x7F800001, 0xFFC00000, 0xFFC00003, 0x7F800000, 0xFF800000,
                         0x00000000, 0x80000000, 0x00000001, 0x80000001, 0x00800000], np.uint32).view(np.float32)
    for m in range(rows):
        pos = rng.choice(V, 200, replace=False)
        x[m, pos] = specials[rng.integers(0, len(specials), 200)]
    _check(dev, x, 64)
    _check(dev, x, 7)
    # all-special rows: zeros of both signs only -> ties broken by index, bits kept
    z = np.where(rng.random((2, 3000)) < 0.5, np.float32(0.0), np.float32(-0.0)).astype(np.float32)
    gv, gi = _check(dev, z, 40)
    assert (gi == np.arange(40)).all()


def test_ldv_larger_than_v(dev):
    _check(dev, _logits(5, 3, 10000), 8, V=9998, ldv_pad=8)


def test_head_logits(dev):
    """The head GEMM's own FP32 logits at M = 8 (151,936 columns), then top-k."""
    N, K = 151936, 5120
    m = make_matrix(3, 0, N, K, dev, synth.EXP_LOGU_M6_4)
    X = synth.torch_activations(3, 1, 8, K, dev)
    Y = abi.gemm_decode(X, m.wq, m.ws, synth.GSCALE, N, K)
    gv, gi = abi.topk(Y, 8)
    torch.cuda.synchronize()
    ov, oi = oracle.topk(Y.cpu().numpy(), 8)
    assert np.array_equal(gi.cpu().numpy(), oi)
    assert np.array_equal(gv.cpu().numpy().view(np.uint32), ov.view(np.uint32))


def test_repeatable_and_graph_capturable(dev):
    x = torch.from_numpy(_logits(9, 8, 151936)).to(dev)
    v0, i0 = abi.topk(x, 8)  # first call on the device: allocates the workspace
    v1 = torch.empty_like(v0)
    i1 = torch.empty_like(i0)
    s = torch.cuda.Stream()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        abi.topk(x, 8, values=v1, indices=i1, stream=s)
    for _ in range(3):
        v1.zero_()
        i1.zero_()
        g.replay()
        torch.cuda.synchronize()
        assert torch.equal(i0, i1) and torch.equal(v0.view(torch.int32), v1.view(torch.int32))
    del g


def test_errors(dev):
    x = torch.zeros((2, 1028), dtype=torch.float32, device=dev)
    v = torch.empty((2, 8), dtype=torch.float32, device=dev)
    i = torch.empty((2, 8), dtype=torch.int32, device=dev)
    s = torch.cuda.current_stream().cuda_stream
    assert abi.nvfp4_topk(x.data_ptr() + 4, 2, 1000, 1028, 8, v.data_ptr(), i.data_ptr(), s) == abi.NVFP4_ERR_ALIGN
    assert abi.nvfp4_topk(x.data_ptr(), 2, 1000, 1026, 8, v.data_ptr(), i.data_ptr(), s) == abi.NVFP4_ERR_ALIGN
    assert abi.nvfp4_topk(x.data_ptr(), 2, 1000, 1028, 65, v.data_ptr(), i.data_ptr(), s) == abi.NVFP4_ERR_SHAPE
    assert abi.nvfp4_topk(x.data_ptr(), 65, 1000, 1028, 8, v.data_ptr(), i.data_ptr(), s) == abi.NVFP4_ERR_M
    assert abi.nvfp4_topk(x.data_ptr(), 2, 5, 1028, 8, v.data_ptr(), i.data_ptr(), s) == abi.NVFP4_ERR_SHAPE
