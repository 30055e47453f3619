"""Helpers shared by the GPU tests: move seeded inputs to the device, run the
library through its C ABI, and compare with the oracle."""
import numpy as np
import torch

import oracle
from nvfp4_weight_streaming_decode_b200 import abi, synth


def to_dev(a: np.ndarray, dev):
    return torch.from_numpy(np.ascontiguousarray(a)).to(dev)


def x_to_dev(X_bits: np.ndarray, dev):
    return torch.from_numpy(np.ascontiguousarray(X_bits).view(np.int16)).to(dev).view(torch.bfloat16)


def x_from_dev(X) -> np.ndarray:
    return X.view(torch.int16).cpu().numpy().view(np.uint16)


def packed(q, s, dev):
    return abi.pack(to_dev(q, dev), to_dev(s, dev))


def assert_gemm_close(Y_gpu, Y_or, A, what=""):
    Yg = Y_gpu.astype(np.float64)
    err = np.abs(Yg - Y_or)
    bound = oracle.gemm_tolerance(A)
    bad = ~(err <= bound)
    assert not bad.any(), (f"{what}: {bad.sum()} elements out of bound; worst err/bound "
                           f"{np.nanmax(err / bound):.3e}")
    return float(np.max(err / bound)) if err.size else 0.0


def gemm_case(dev, q, s, X, gscale=synth.GSCALE, canary=True):
    """Run the GEMM on (q, s, X) and return Y as numpy float32 [M][N]."""
    N, K = q.shape[0], q.shape[1] * 2
    M = X.shape[0]
    wq, ws = packed(q, s, dev)
    Xd = x_to_dev(X, dev)
    pad = 64
    Ybuf = torch.full((M * N + pad,), 12345.0, dtype=torch.float32, device=dev)
    Y = Ybuf[:M * N].view(M, N)
    abi.gemm_decode(Xd, wq, ws, gscale, N, K, Y=Y)
    torch.cuda.synchronize()
    if canary:
        assert torch.all(Ybuf[M * N:] == 12345.0), "GEMM wrote past Y"
    return Y.cpu().numpy()
