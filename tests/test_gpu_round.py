"""GPU tests of the decode round: per-width graph replay against direct C-ABI
calls (bit-identical, the kernels being deterministic) and against the
oracle on the nodes' outputs."""
import numpy as np
import pytest
import torch

import oracle
from gpu_helpers import assert_gemm_close, x_from_dev
from nvfp4_weight_streaming_decode_b200 import abi, synth
from nvfp4_weight_streaming_decode_b200.workloads import SyntheticRound

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dev(cuda_device):
    from nvfp4_weight_streaming_decode_b200 import build
    build.build()
    abi.load()
    torch.cuda.set_device(cuda_device)
    return cuda_device


def _outputs(r):
    return {k: v.clone() for k, v in r.bufs.items() if k.startswith(("y", "H", "logits"))}


def _zero_outputs(r):
    for k, v in r.bufs.items():
        if k.startswith(("y", "H", "logits")):
            v.zero_()


def _check_node(r, name, M, rows=None):
    """Compare one node's output (first M rows) with the oracle, sampled on `rows`."""
    node = [n for n in r.nodes if n[0] == name][0]
    _, kind, xin, out, mkeys = node
    X = x_from_dev(r.bufs[xin][:M])
    mats = [r.mats[k] for k in mkeys]
    planes = []
    for m in mats:
        q, s = m.canonical(r.device, r.workload_id)
        planes.append((q.cpu().numpy(), s.cpu().numpy()))
    N = mats[0].N
    sel = np.arange(N) if rows is None else np.asarray(rows)
    got = r.bufs[out][:M].float().cpu().numpy()[:, sel].astype(np.float64)
    if kind == abi.NVFP4_DESC_GEMM:
        Yr, A = oracle.gemm_rows(X, planes[0][0], planes[0][1], r.gscale, sel)
        assert_gemm_close(got, Yr, A, f"{name} M={M}")
    else:
        G, AG = oracle.gemm_rows(X, planes[0][0], planes[0][1], r.gscale, sel)
        U, AU = oracle.gemm_rows(X, planes[1][0], planes[1][1], r.gscale, sel)
        h = G / (1.0 + np.exp(-G)) * U
        err = np.abs(got - h)
        assert np.all(err <= oracle.silu_tolerance(G, U, AG, AU)), f"{name} M={M}"


MODES = [abi.NVFP4_ROUND_PERSISTENT, abi.NVFP4_ROUND_CHAIN]


def _bit_exact_keys(mode, keys):
    """Outputs a replay must reproduce bit for bit against direct calls.  The
    chain mode runs the very kernels of the direct calls.  The persistent mode
    keeps every plain GEMM's partition (bit-identical) but computes the fused
    gate/up as a stacked GEMM plus a SiLU-multiply node, so H, and the down
    projection that reads it, are checked against the oracle instead."""
    if mode == abi.NVFP4_ROUND_CHAIN:
        return list(keys)
    return [k for k in keys if not k.startswith(("H", "ydown"))]


def _graph_nodes(mode, n):
    return 1 if mode == abi.NVFP4_ROUND_PERSISTENT else n


@pytest.mark.parametrize("mode", MODES)
def test_small_round_replay_matches_direct_calls_and_oracle(dev, mode):
    r = SyntheticRound.build(dev, layers=2, hidden=256, ffn=512, vocab=1000, workload_id=40)
    rnd = abi.Round(r.descs, mode)
    assert rnd.nodes == _graph_nodes(mode, 2 * 4 + 1)
    for M in range(1, 9):
        _zero_outputs(r)
        rnd.replay(M)
        torch.cuda.synchronize()
        replayed = _outputs(r)
        _zero_outputs(r)
        r.run_direct(M)
        torch.cuda.synchronize()
        direct = _outputs(r)
        for k in _bit_exact_keys(mode, replayed):
            a, b = replayed[k], direct[k]
            assert torch.equal(a.view(torch.int16) if a.dtype == torch.bfloat16 else a.view(torch.int32),
                               b.view(torch.int16) if b.dtype == torch.bfloat16 else b.view(torch.int32)), (k, M)
        rnd.replay(M)
        torch.cuda.synchronize()
        for name, *_ in r.nodes:
            _check_node(r, name, M)
    rnd.close()


@pytest.mark.parametrize("mode", MODES)
def test_round_replay_host_copies(dev, mode):
    r = SyntheticRound.build(dev, layers=1, hidden=128, ffn=256, vocab=320, workload_id=41)
    rnd = abi.Round(r.descs, mode)
    M = 8
    x_host = torch.empty((M, 128), dtype=torch.bfloat16).pin_memory()
    x_host.copy_(synth.torch_activations(41, 999, M, 128, "cpu"))
    y_host = torch.zeros((M, 320), dtype=torch.float32).pin_memory()
    rnd.replay_host(M, x_host, r.bufs["xhead"], r.bufs["logits"], y_host)
    torch.cuda.synchronize()
    assert torch.equal(r.bufs["xhead"].cpu(), x_host)
    assert torch.equal(y_host, r.bufs["logits"].cpu())
    _check_node(r, "head", M)
    rnd.close()


def test_full_round_sampled(dev):
    """The full 64-layer round plus head: replay equals direct calls at M = 1
    and 8, and sampled outputs of layers 0, 31, 63 and the head match the oracle."""
    w = synth.WORKLOADS[4]
    r = SyntheticRound.build(dev, layers=w["layers"], hidden=w["hidden"], ffn=w["ffn"], vocab=w["vocab"])
    rounds = {mode: abi.Round(r.descs, mode) for mode in MODES}
    assert rounds[abi.NVFP4_ROUND_CHAIN].nodes == 4 * w["layers"] + 1
    assert rounds[abi.NVFP4_ROUND_PERSISTENT].nodes == 1
    rng = np.random.default_rng(6)
    for M, mode in ((1, abi.NVFP4_ROUND_PERSISTENT), (8, abi.NVFP4_ROUND_PERSISTENT), (8, abi.NVFP4_ROUND_CHAIN)):
        rnd = rounds[mode]
        _zero_outputs(r)
        rnd.replay(M)
        torch.cuda.synchronize()
        replayed = _outputs(r)
        for l in (0, 31, 63):
            for nm, N in ((f"qkv{l}", 3 * w["hidden"]), (f"o{l}", w["hidden"]),
                          (f"gateup{l}", w["ffn"]), (f"down{l}", w["hidden"])):
                _check_node(r, nm, M, np.unique(np.concatenate([[0, N - 1], rng.integers(0, N, 48)])))
        _check_node(r, "head", M, np.unique(np.concatenate([[0, w["vocab"] - 1],
                                                             rng.integers(0, w["vocab"], 96)])))
        _zero_outputs(r)
        r.run_direct(M)
        torch.cuda.synchronize()
        direct = _outputs(r)
        for k in _bit_exact_keys(mode, replayed):
            a, b = replayed[k], direct[k]
            ia = a.view(torch.int16) if a.dtype == torch.bfloat16 else a.view(torch.int32)
            ib = b.view(torch.int16) if b.dtype == torch.bfloat16 else b.view(torch.int32)
            assert torch.equal(ia, ib), (k, M, mode)
    for rnd in rounds.values():
        rnd.close()
