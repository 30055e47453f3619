"""GPU parity at the edges of the activations' range.

The register kernels dequantise the weights exactly to bf16 ("Models and
artifacts", "The artifact": E2M1 elements, one E4M3 scale per 16 values; the
product carries at most 6 significant bits) and multiply X as it comes, in
bf16; the tcgen05 kernel does the same with the A operand in tensor memory.
Each case below puts X where a narrower format would not hold it exactly --
far above f16's range, far below it, in f16's subnormal range, and mixed chunk
by chunk with zeros -- and compares with the oracle; and since every product
is exact and the sums are FP32, scaling X by a power of two scales Y by it
exactly."""
import numpy as np
import pytest
import torch

import oracle
from gpu_helpers import assert_gemm_close, gemm_case, packed, x_to_dev
from nvfp4_weight_streaming_decode_b200 import abi, synth

pytestmark = pytest.mark.gpu

N, K = 512, 1024  # 16 chunks of 64 columns


@pytest.fixture(scope="module")
def dev(cuda_device):
    from nvfp4_weight_streaming_decode_b200 import build
    build.build()
    abi.load()
    torch.cuda.set_device(cuda_device)
    return cuda_device


def _x(kind, M, seed):
    g = synth.rng(61, seed)
    base = g.standard_normal((M, K))
    if kind == "f16_subnormal":
        # every magnitude in [2^-17, 2^-14): f16 would hold these only as subnormals
        x = np.sign(base) * (1.0 + g.random((M, K))) * 2.0 ** g.integers(-17, -14, (M, K))
    elif kind == "huge":
        x = base * 2.0 ** 20  # beyond f16's range
    elif kind == "tiny":
        x = base * 2.0 ** -40  # below f16's subnormals
    elif kind == "mixed":
        x = base.copy()
        x[:, 1 * 64 + 3] = 70000.0             # chunk 1: one value past 65,504
        x[:, 5 * 64 + 17] = -1.2345e-7         # chunk 5: one value below 2^-17
        x[:, 9 * 64:10 * 64] *= 2.0 ** -15     # chunk 9: f16 subnormals, exact
        x[:, 12 * 64 + 40] = 1.0e6             # chunk 12: one large value
        x[:, 14 * 64:15 * 64] = 0.0            # chunk 14: zeros
    else:
        raise ValueError(kind)
    return synth.bf16_bits_from_f64(x)


@pytest.mark.parametrize("M", [1, 8, 13, 40])
@pytest.mark.parametrize("kind", ["f16_subnormal", "huge", "tiny", "mixed"])
def test_gemm_x_range_matches_oracle(dev, M, kind):
    q, s = synth.matrix(61, M, N, K)
    X = _x(kind, M, M * 10 + len(kind))
    Y = gemm_case(dev, q, s, X)
    Yr, A = oracle.gemm(X, q, s, synth.GSCALE)
    assert np.all(np.isfinite(Y)), kind
    assert_gemm_close(Y, Yr, A, f"{kind} M={M}")


@pytest.mark.parametrize("M", [8, 40])
def test_power_of_two_scaling_is_exact(dev, M):
    """X and 2^8 X: Y scales by 2^8 bit for bit, because the products are exact
    and accumulate in FP32 in the same order."""
    q, s = synth.matrix(62, M, N, K)
    g = synth.rng(62, M)
    x = g.standard_normal((M, K))
    X1 = synth.bf16_bits_from_f64(x)
    X2 = synth.bf16_bits_from_f64(x * 2.0 ** 8)
    wq, ws = packed(q, s, dev)
    Y1 = abi.gemm_decode(x_to_dev(X1, dev), wq, ws, synth.GSCALE, N, K)
    Y2 = abi.gemm_decode(x_to_dev(X2, dev), wq, ws, synth.GSCALE, N, K)
    torch.cuda.synchronize()
    assert torch.equal((Y1 * 2.0 ** 8).view(torch.int32), Y2.view(torch.int32))


@pytest.mark.parametrize("M", [1, 8])
def test_gateup_silu_x_range(dev, M):
    Nff = 96
    qg, sg = synth.matrix(63, 0, Nff, K)
    qu, su = synth.matrix(63, 1, Nff, K)
    X = _x("mixed", M, 70 + M)
    wg, sgd = packed(qg, sg, dev)
    wu, sud = packed(qu, su, dev)
    # gate and up scaled so that silu(g) * u stays finite for the large values
    gs_g, gs_u = synth.GSCALE * 2.0 ** -20, synth.GSCALE * 2.0 ** -20
    H = abi.gemm_gateup_silu(x_to_dev(X, dev), wg, sgd, gs_g, wu, sud, gs_u, Nff, K)
    torch.cuda.synchronize()
    Hf = H.float().cpu().numpy().astype(np.float64)
    G, U, h, AG, AU = oracle.gateup_silu(X, qg, sg, gs_g, qu, su, gs_u)
    bound = oracle.silu_tolerance(G, U, AG, AU)
    err = np.abs(Hf - h)
    assert np.all(err <= bound), f"gate/up M={M}: worst err/bound {np.max(err / bound):.3e}"


def test_grouped_x_range(dev):
    from nvfp4_weight_streaming_decode_b200.workloads import make_matrix
    E, Ne = 6, 64
    m = make_matrix(64, 0, E * Ne, K, dev)
    kc = K // 64
    qb, sb = (Ne // 32) * kc * 1024, (Ne // 32) * kc * 128
    mats = [(m.wq[e * qb:(e + 1) * qb], m.ws[e * sb:(e + 1) * sb], synth.GSCALE) for e in range(E)]
    table = abi.expert_table(mats, dev)
    q, s = m.canonical(dev, 64)
    q, s = q.cpu().numpy(), s.cpu().numpy()
    M, T = 4, 3
    route = np.array([[0, 1, 2], [3, 4, 5], [5, 0, 2], [1, 3, 4]], np.int32)
    X = np.concatenate([_x(k, 1, 80 + i) for i, k in enumerate(["huge", "tiny", "mixed", "f16_subnormal"])])
    Y = abi.gemm_grouped(x_to_dev(X, dev), torch.from_numpy(route).to(dev), table, E, Ne, K)
    torch.cuda.synchronize()
    Yh = Y.cpu().numpy()
    for i in range(M):
        for t in range(T):
            e = int(route[i, t])
            Yr, A = oracle.gemm(X[i:i + 1], q[e * Ne:(e + 1) * Ne], s[e * Ne:(e + 1) * Ne], synth.GSCALE)
            assert_gemm_close(Yh[i, t][None, :], Yr, A, f"route ({i},{t})")
