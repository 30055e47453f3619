"""GPU parity of the CUDA path against the float64 oracle, through the C ABI.

Bars: byte-exact pack/unpack, bit-exact dequantisation (sign of zero
included), and for every GEMM output element
|Y_gpu - Y_oracle| <= 2e-3 * sum_k |x_k w_k| + 1e-6.
"""
import numpy as np
import pytest
import torch

import oracle
from gpu_helpers import assert_gemm_close, gemm_case, packed, to_dev, x_from_dev, x_to_dev
from nvfp4_weight_streaming_decode_b200 import abi, synth

pytestmark = pytest.mark.gpu

SHAPES = [(256, 512), (45, 80), (1, 16), (33, 208), (96, 1024), (7, 4096), (640, 64)]


@pytest.fixture(scope="module")
def dev(cuda_device):
    from nvfp4_weight_streaming_decode_b200 import build
    build.build()
    abi.load()
    torch.cuda.set_device(cuda_device)
    return cuda_device


# ------------------------------------------------------------------ layout

@pytest.mark.parametrize("N,K", SHAPES)
def test_pack_unpack_round_trip_is_byte_exact(dev, N, K):
    q, s = synth.matrix(30, N + K, N, K)
    wq, ws = packed(q, s, dev)
    q2, s2 = abi.unpack_debug(wq, ws, N, K)
    assert np.array_equal(q2.cpu().numpy(), q) and np.array_equal(s2.cpu().numpy(), s)


def test_single_nonzero_probes_cover_every_unit_position(dev):
    # row n sits at in-tile row n % 32 of tile n // 32; its one nonzero is at
    # column (n // 32) % 64, so the 2048 rows cover all 32 x 64 positions.
    N, K = 2048, 64
    q = np.zeros((N, K // 2), np.uint8)
    cols = (np.arange(N) // 32) % 64
    for n, k in enumerate(cols):
        q[n, k // 2] = 0x2 << (4 * (k % 2))
    s = np.full((N, K // 16), 0x38, np.uint8)
    wq, ws = packed(q, s, dev)
    W = abi.dequant_debug(wq, ws, 1.0, N, K).cpu().numpy()
    hot = np.zeros((N, K), np.float32)
    hot[np.arange(N), cols] = 1.0
    assert np.array_equal(W, hot)


@pytest.mark.parametrize("N,K", SHAPES + [(5120, 5120)])
def test_dequant_is_bit_exact(dev, N, K):
    q, s = synth.matrix(31, N * 3 + K, N, K)
    for gscale in (synth.GSCALE, 1.0, -3.0):
        wq, ws = packed(q, s, dev)
        W = abi.dequant_debug(wq, ws, gscale, N, K).cpu().numpy()
        ref = oracle.dequant(q, s, gscale)
        assert np.array_equal(W.view(np.uint32), ref.view(np.uint32)), gscale


def test_dequant_every_code_with_every_scale(dev):
    scales = np.array([b for b in range(256) if (b & 0x7F) != 0x7F], np.uint8)
    N, K = 256, 64
    codes = np.arange(K) % 16
    q = np.tile((codes[0::2] | (codes[1::2] << 4)).astype(np.uint8), (N, 1))
    s = np.repeat(scales[np.arange(N) % scales.size][:, None], K // 16, axis=1).astype(np.uint8)
    wq, ws = packed(q, s, dev)
    W = abi.dequant_debug(wq, ws, 1.0, N, K).cpu().numpy()
    ref = oracle.dequant(q, s, 1.0)
    assert np.array_equal(W.view(np.uint32), ref.view(np.uint32))


def test_head_dequant_sampled_rows(dev):
    N, K = 151936, 5120
    q, s = synth.matrix(3, 0, N, K, synth.EXP_LOGU_M6_4)
    wq, ws = packed(q, s, dev)
    W = abi.dequant_debug(wq, ws, synth.GSCALE, N, K)
    rows = np.unique(np.concatenate([[0, 1, 31, 32, N - 33, N - 1],
                                     np.random.default_rng(0).integers(0, N, 250)]))
    Ws = W[torch.from_numpy(rows).to(dev)].cpu().numpy()
    ref = oracle.dequant(np.ascontiguousarray(q[rows]), np.ascontiguousarray(s[rows]), synth.GSCALE)
    assert np.array_equal(Ws.view(np.uint32), ref.view(np.uint32))


def test_nan_scale_is_rejected(dev):
    N, K = 64, 128
    q, s = synth.matrix(32, 0, N, K)
    for bad in (0x7F, 0xFF):
        s2 = s.copy()
        s2[17, 3] = bad
        Q, S = to_dev(q, dev), to_dev(s2, dev)
        st, nq, ns = abi.nvfp4_packed_bytes(N, K)
        wq = torch.empty(nq, dtype=torch.uint8, device=dev)
        ws = torch.empty(ns, dtype=torch.uint8, device=dev)
        st = abi.nvfp4_pack_check(Q.data_ptr(), S.data_ptr(), N, K, wq.data_ptr(), ws.data_ptr(),
                                  torch.cuda.current_stream().cuda_stream)
        assert st == abi.NVFP4_ERR_BAD_SCALE
    # and a clean matrix after a rejected one packs fine
    packed(q, s, dev)


# ------------------------------------------------------------------ GEMM

@pytest.mark.parametrize("N,K", SHAPES)
@pytest.mark.parametrize("M", [1, 2, 3, 5, 8])
def test_gemm_matches_oracle(dev, M, N, K):
    q, s = synth.matrix(33, N * 11 + K, N, K)
    X = synth.activations(synth.rng(33, M * 100000 + N + K), M, K)
    Y = gemm_case(dev, q, s, X)
    Yr, A = oracle.gemm(X, q, s, synth.GSCALE)
    assert_gemm_close(Y, Yr, A, f"M={M} N={N} K={K}")


def test_gemm_workload_gemm_m1_n256_k512(dev):
    w = synth.WORKLOADS[0]
    q, s = synth.matrix(0, 0, w["N"], w["K"], w["exp"])
    for M in range(1, 9):
        X = synth.activations(synth.rng(0, 1), M, w["K"])
        Y = gemm_case(dev, q, s, X)
        Yr, A = oracle.gemm(X, q, s, synth.GSCALE)
        assert_gemm_close(Y, Yr, A, f"workload 0, M={M}")


@pytest.mark.parametrize("M", range(1, 9))
def test_gemm_workload_proj_5120(dev, M):
    w = synth.WORKLOADS[1]
    q, s = synth.matrix(1, 0, w["N"], w["K"], w["exp"])
    X = synth.activations(synth.rng(1, 100 + M), M, w["K"])
    Y = gemm_case(dev, q, s, X)
    Yr, A = oracle.gemm(X, q, s, synth.GSCALE)
    assert_gemm_close(Y, Yr, A, f"workload 1, M={M}")


def test_gemm_is_deterministic(dev):
    N, K, M = 5120, 5120, 8
    q, s = synth.matrix(34, 0, N, K)
    X = synth.activations(synth.rng(34, 1), M, K)
    wq, ws = packed(q, s, dev)
    Xd = x_to_dev(X, dev)
    Y1 = abi.gemm_decode(Xd, wq, ws, synth.GSCALE, N, K)
    Y2 = abi.gemm_decode(Xd, wq, ws, synth.GSCALE, N, K)
    torch.cuda.synchronize()
    assert torch.equal(Y1.view(torch.int32), Y2.view(torch.int32))


def _identity(K, perm=None):
    q = np.zeros((K, K // 2), np.uint8)
    cols = np.arange(K) if perm is None else perm
    for n in range(K):
        k = cols[n]
        q[n, k // 2] |= 0x2 << (4 * (k % 2))
    return q, np.full((K, K // 16), 0x38, np.uint8)


def test_gemm_identity_and_permutation_are_exact(dev):
    K = 512
    X = synth.activations(synth.rng(35, 0), 8, K)
    Xf = (X.astype(np.uint32) << 16).view(np.float32)
    q, s = _identity(K)
    Y = gemm_case(dev, q, s, X, gscale=1.0)
    assert np.array_equal(Y, Xf)
    perm = np.random.default_rng(1).permutation(K)
    q, s = _identity(K, perm)
    Y = gemm_case(dev, q, s, X, gscale=1.0)
    assert np.array_equal(Y, Xf[:, perm])


def test_gemm_constant_code_closed_form(dev):
    M, N, K = 4, 64, 1024
    q = np.full((N, K // 2), 0x77, np.uint8)  # 6.0
    s = np.full((N, K // 16), 0x30, np.uint8)  # 0.5
    X = synth.activations(synth.rng(36, 0), M, K)
    Y = gemm_case(dev, q, s, X, gscale=0.25)
    rowsum = (X.astype(np.uint32) << 16).view(np.float32).astype(np.float64).sum(axis=1)
    ref = np.repeat((6.0 * 0.5 * 0.25 * rowsum)[:, None], N, axis=1)
    _, A = oracle.gemm(X, q, s, 0.25)
    assert_gemm_close(Y, ref, A, "constant code")


def test_gemm_extreme_scales(dev):
    N, K, M = 64, 256, 8
    q, s = synth.matrix(37, 0, N, K)
    rng = np.random.default_rng(2)
    pool = np.array([0x01, 0x02, 0x07, 0x08, 0x7E, 0x00, 0x80, 0xFE, 0x81], np.uint8)
    s = pool[rng.integers(0, pool.size, s.shape)]
    X = synth.activations(synth.rng(37, 1), M, K)
    Y = gemm_case(dev, q, s, X, gscale=1.0)
    Yr, A = oracle.gemm(X, q, s, 1.0)
    assert_gemm_close(Y, Yr, A, "extreme scales")


def test_head_workload_sampled_rows(dev):
    w = synth.WORKLOADS[3]
    N, K = w["N"], w["K"]
    q, s = synth.matrix(3, 0, N, K, w["exp"])
    wq, ws = packed(q, s, dev)
    rows = np.unique(np.concatenate([[0, 1, 31, 32, N - 33, N - 1],
                                     np.random.default_rng(3).integers(0, N, 300)]))
    for M in w["M"]:
        X = synth.activations(synth.rng(3, 10 + M), M, K)
        Y = abi.gemm_decode(x_to_dev(X, dev), wq, ws, synth.GSCALE, N, K)
        torch.cuda.synchronize()
        Ys = Y.cpu().numpy()[:, rows]
        Yr, A = oracle.gemm_rows(X, q, s, synth.GSCALE, rows)
        assert_gemm_close(Ys, Yr, A, f"head M={M}")


# ------------------------------------------------------------------ fused MLP

def _gateup_check(dev, M, Nff, K, rows=None):
    qg, sg = synth.matrix(2, 0, Nff, K)
    qu, su = synth.matrix(2, 1, Nff, K)
    X = synth.activations(synth.rng(2, 10 + M), M, K)
    wg, sgd = packed(qg, sg, dev)
    wu, sud = packed(qu, su, dev)
    H = abi.gemm_gateup_silu(x_to_dev(X, dev), wg, sgd, synth.GSCALE, wu, sud, synth.GSCALE / 2, Nff, K)
    torch.cuda.synchronize()
    Hf = H.float().cpu().numpy().astype(np.float64)
    if rows is None:
        G, U, h, AG, AU = oracle.gateup_silu(X, qg, sg, synth.GSCALE, qu, su, synth.GSCALE / 2)
    else:
        Hf = Hf[:, rows]
        G, AG = oracle.gemm_rows(X, qg, sg, synth.GSCALE, rows)
        U, AU = oracle.gemm_rows(X, qu, su, synth.GSCALE / 2, rows)
        h = G / (1.0 + np.exp(-G)) * U
    bound = oracle.silu_tolerance(G, U, AG, AU)
    err = np.abs(Hf - h)
    assert np.all(err <= bound), f"gate/up M={M}: worst err/bound {np.max(err / bound):.3e}"
    return H, X


@pytest.mark.parametrize("M", [1, 3, 8])
@pytest.mark.parametrize("Nff,K", [(64, 256), (45, 80), (96, 5120)])
def test_gateup_silu_matches_oracle(dev, M, Nff, K):
    _gateup_check(dev, M, Nff, K)


@pytest.mark.parametrize("M", [1, 8])
def test_mlp_workload_sampled(dev, M):
    w = synth.WORKLOADS[2]
    Nff, K = w["Nff"], w["K"]
    rows = np.unique(np.concatenate([[0, 1, Nff - 1], np.random.default_rng(4).integers(0, Nff, 200)]))
    H, _ = _gateup_check(dev, M, Nff, K, rows)
    # down projection, checked stage-wise: its X is the GPU's own H
    qd, sd = synth.matrix(2, 2, K, Nff)
    wd, sdd = packed(qd, sd, dev)
    Y = abi.gemm_decode(H, wd, sdd, synth.GSCALE, K, Nff)
    torch.cuda.synchronize()
    Hbits = x_from_dev(H)
    drows = np.unique(np.concatenate([[0, K - 1], np.random.default_rng(5).integers(0, K, 200)]))
    Yr, A = oracle.gemm_rows(Hbits, qd, sd, synth.GSCALE, drows)
    assert_gemm_close(Y.cpu().numpy()[:, drows], Yr, A, f"down M={M}")
