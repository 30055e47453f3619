"""GPU parity of nvfp4_gemm_decode at verify widths, M = 9..64 (ignis README,
"What sets it apart", "Speculative decoding (DFlash2)": lanes x (1 + drafts)
rows verified in the same pass over the weights), against the oracle.  Widths
9..32 run on the register-MMA decode kernel with two to four blocks of 8
lanes, 33..64 on the tensor-memory (tcgen05) kernel."""
import numpy as np
import pytest
import torch

import oracle
from gpu_helpers import assert_gemm_close, gemm_case, packed, x_to_dev
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


@pytest.mark.parametrize("M", [9, 10, 12, 15, 16, 17, 24, 25, 31, 32, 33, 48, 63, 64])
@pytest.mark.parametrize("N,K", [(32, 64), (256, 512), (300, 1040), (1000, 2048), (5120, 5120)])
def test_verify_gemm_matches_oracle(dev, M, N, K):
    q, s = synth.matrix(50, N * 13 + K, N, K)
    X = synth.activations(synth.rng(50, M * 100003 + N + K), M, K)
    Y = gemm_case(dev, q, s, X)
    Yr, A = oracle.gemm(X, q, s, synth.GSCALE)
    assert_gemm_close(Y, Yr, A, f"M={M} N={N} K={K}")


@pytest.mark.parametrize("M", [9, 16, 24, 31, 64])
def test_verify_down_projection(dev, M):
    """K = 17,408 (the MLP down projection): long K ranges, many CTAs per tile pair."""
    N, K = 5120, 17408
    q, s = synth.matrix(51, M, N, K)
    X = synth.activations(synth.rng(51, M), M, K)
    Y = gemm_case(dev, q, s, X)
    Yr, A = oracle.gemm(X, q, s, synth.GSCALE)
    assert_gemm_close(Y, Yr, A, f"down M={M}")


@pytest.mark.parametrize("M", [12, 16, 25, 64])
def test_verify_head_sampled(dev, M):
    """The vocabulary head (151,936 x 5,120, log-uniform scales) at a verify
    width, checked against the oracle on sampled rows."""
    N, K = 151936, 5120
    m = make_matrix(3, 0, N, K, dev, synth.EXP_LOGU_M6_4)
    X = synth.torch_activations(3, 7, M, K, dev)
    Y = abi.gemm_decode(X, m.wq, m.ws, synth.GSCALE, N, K)
    torch.cuda.synchronize()
    q, s = m.canonical(dev, 3)
    rows = np.unique(np.concatenate([[0, 1, N - 1], np.random.default_rng(M).integers(0, N, 200)]))
    Xb = X.view(torch.int16).cpu().numpy().view(np.uint16)
    Yr, A = oracle.gemm_rows(Xb, q.cpu().numpy(), s.cpu().numpy(), synth.GSCALE, rows)
    assert_gemm_close(Y.cpu().numpy()[:, rows], Yr, A, f"head M={M}")


def test_verify_is_deterministic_and_agrees_with_decode_rows(dev):
    """Two calls are bit-identical; the first 8 rows agree with the M = 8
    decode kernel (another summation order) within the GEMM bound."""
    N, K = 5120, 5120
    q, s = synth.matrix(52, 0, N, K)
    X = synth.activations(synth.rng(52, 1), 40, K)
    wq, ws = packed(q, s, dev)
    Xd = x_to_dev(X, dev)
    Y1 = abi.gemm_decode(Xd, wq, ws, synth.GSCALE, N, K)
    Y2 = abi.gemm_decode(Xd, wq, ws, synth.GSCALE, N, K)
    Y8 = abi.gemm_decode(Xd[:8].contiguous(), wq, ws, synth.GSCALE, N, K)
    torch.cuda.synchronize()
    assert torch.equal(Y1.view(torch.int32), Y2.view(torch.int32))
    Yr, A = oracle.gemm(X[:8], q, s, synth.GSCALE)
    assert_gemm_close(Y1[:8].cpu().numpy(), Yr, A, "verify rows 0..7")
    assert_gemm_close(Y8.cpu().numpy(), Yr, A, "decode M=8")


def test_verify_identity_is_exact(dev):
    """Identity weights (code 1.0, scale 1.0): Y = X exactly at every width."""
    K = 512
    q = np.zeros((K, K // 2), np.uint8)
    for n in range(K):
        q[n, n // 2] |= 0x2 << (4 * (n % 2))
    s = np.full((K, K // 16), 0x38, np.uint8)
    for M in (9, 13, 16, 24, 64):
        X = synth.activations(synth.rng(53, M), M, K)
        Y = gemm_case(dev, q, s, X, gscale=1.0)
        assert np.array_equal(Y, (X.astype(np.uint32) << 16).view(np.float32)), M


def test_verify_status_clean(dev):
    assert abi.nvfp4_device_status() == 0


def test_wide_width_is_deterministic_and_matches_per_block_rows(dev):
    """M = 13 on the register-MMA kernel: bit-identical across calls, and each
    block of 8 lanes within the GEMM bound of the oracle (rows past M in the
    second block feed only dropped columns)."""
    N, K = 2048, 3072
    q, s = synth.matrix(54, 0, N, K)
    X = synth.activations(synth.rng(54, 1), 13, K)
    wq, ws = packed(q, s, dev)
    Xd = x_to_dev(X, dev)
    Y1 = abi.gemm_decode(Xd, wq, ws, synth.GSCALE, N, K)
    Y2 = abi.gemm_decode(Xd, wq, ws, synth.GSCALE, N, K)
    torch.cuda.synchronize()
    assert torch.equal(Y1.view(torch.int32), Y2.view(torch.int32))
    Yr, A = oracle.gemm(X, q, s, synth.GSCALE)
    assert_gemm_close(Y1[:8].cpu().numpy(), Yr[:8], A[:8], "lanes 0..7")
    assert_gemm_close(Y1[8:].cpu().numpy(), Yr[8:], A[8:], "lanes 8..12")


def test_verify_long_k_grows_the_x_buffer(dev):
    """K past 65,536 at a verify width: the first such call grows the buffer
    that holds X in the MMA's order (outside any capture), and both that call
    and a shorter one after it agree with the oracle."""
    N = 64
    for K in (65536 + 1024, 2048):
        q, s = synth.matrix(55, K, N, K)
        X = synth.activations(synth.rng(55, K), 40, K)
        Y = gemm_case(dev, q, s, X)
        Yr, A = oracle.gemm(X, q, s, synth.GSCALE)
        assert_gemm_close(Y, Yr, A, f"M=40 N={N} K={K}")
