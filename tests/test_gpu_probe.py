"""GPU check of nvfp4_stream_read, the read-only bandwidth probe the bench
reports beside the copy peak: it must read every byte of the buffer once, so
the XOR of its per-CTA words equals the XOR of the buffer's 32-bit words
(computed here with numpy), for ragged sizes, a single word and grids larger
than the buffer."""
import numpy as np
import pytest
import torch

from nvfp4_weight_streaming_decode_b200 import abi

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dev(cuda_device):
    from nvfp4_weight_streaming_decode_b200 import build
    build.build()
    abi.load()
    torch.cuda.set_device(cuda_device)
    return cuda_device


@pytest.mark.parametrize("words16,ctas", [(1, 1), (1, 4), (7, 3), (512 * 4 * 3 + 7, 3), (100_003, 148),
                                          (4 * 1024 * 1024 + 5, 592), (2048, 4096)])
def test_stream_read_touches_every_byte(dev, words16, ctas):
    rng = np.random.default_rng(words16 * 31 + ctas)
    host = rng.integers(0, 2**32, size=words16 * 4, dtype=np.uint32)
    buf = torch.from_numpy(host.view(np.int32)).to(dev)
    out = abi.stream_read(buf, ctas)
    torch.cuda.synchronize()
    got = np.bitwise_xor.reduce(out.cpu().numpy().view(np.uint32))
    assert int(got) == int(np.bitwise_xor.reduce(host))


def test_stream_read_single_flipped_bit_is_seen(dev):
    host = np.zeros(64 * 1024, dtype=np.uint32)
    buf = torch.from_numpy(host.view(np.int32)).to(dev)
    assert int(np.bitwise_xor.reduce(abi.stream_read(buf, 148).cpu().numpy().view(np.uint32))) == 0
    host[-1] = 1 << 17   # the buffer's last word
    buf = torch.from_numpy(host.view(np.int32)).to(dev)
    assert int(np.bitwise_xor.reduce(abi.stream_read(buf, 148).cpu().numpy().view(np.uint32))) == 1 << 17
