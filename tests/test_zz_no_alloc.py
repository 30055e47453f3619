"""GPU test of nvfp4_gemm_decode_noalloc, the decode GEMM for callers that may
not allocate device memory (its split-K scratch is a static array inside the
library).  The same kernel runs with the same work split and a fixed combine
order, so its output must equal nvfp4_gemm_decode's bit for bit, on two calls
in a row (the second call sees the array exactly as the first left it): a
stale or misplaced partial sum of any size changes some bit.  Its output is
also checked against the oracle at the bound the other GEMM tests use.  This
file is collected last so that a run stopping at the first failure has run
every other test first.
"""
import numpy as np
import pytest
import torch

import oracle
from gpu_helpers import packed, x_to_dev
from nvfp4_weight_streaming_decode_b200 import abi, synth

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("M,N,K", [(8, 5120, 5120), (3, 45, 80), (1, 256, 512), (5, 96, 17408)])
def test_noalloc_matches_gemm_decode_on_two_calls(cuda_device, M, N, K):
    from nvfp4_weight_streaming_decode_b200 import build
    build.build()
    abi.load()
    torch.cuda.set_device(cuda_device)
    q, s = synth.matrix(50, N + K, N, K)
    X = synth.activations(synth.rng(50, M * 7 + N), M, K)
    wq, ws = packed(q, s, cuda_device)
    Xd = x_to_dev(X, cuda_device)
    Y_ref = abi.gemm_decode(Xd, wq, ws, synth.GSCALE, N, K)
    torch.cuda.synchronize()
    Yr, A = oracle.gemm(X, q, s, synth.GSCALE)
    bound = oracle.gemm_tolerance(A)
    stream = torch.cuda.current_stream().cuda_stream
    for call in range(2):
        Y = torch.full((M, N), float("nan"), dtype=torch.float32, device=cuda_device)
        st = abi.nvfp4_gemm_decode_noalloc(Xd.data_ptr(), M, wq.data_ptr(), ws.data_ptr(), synth.GSCALE,
                                           Y.data_ptr(), N, K, stream)
        assert st == abi.NVFP4_OK, abi.status_string(st)
        torch.cuda.synchronize()
        same = torch.equal(Y.view(torch.int32), Y_ref.view(torch.int32))
        assert same, f"call {call}: {int((Y.view(torch.int32) != Y_ref.view(torch.int32)).sum())} elements differ"
        err = np.abs(Y.cpu().numpy().astype(np.float64) - Yr)
        assert np.all(err <= bound), f"call {call}: worst err/bound vs oracle {np.nanmax(err / bound):.3e}"
