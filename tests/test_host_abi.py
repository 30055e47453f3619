"""CPU tests of the C-ABI library: symbols, argument checks, and the host
model of the device layout against the oracle.  No GPU and no kernel launch:
every call here returns before the library touches CUDA."""
import ctypes
import os

import numpy as np
import pytest

import oracle
from nvfp4_weight_streaming_decode_b200 import abi, synth


@pytest.fixture(scope="module")
def lib():
    import __graft_entry__  # noqa: F401  (build helpers)
    from nvfp4_weight_streaming_decode_b200 import build
    build.build()
    return abi.load()


def _ptr(a):
    return a.ctypes.data_as(ctypes.c_void_p)


def test_library_exports_every_header_symbol(lib):
    names = abi.header_functions()
    assert len(names) >= 15
    for n in names:
        assert hasattr(lib, n), n
    assert set(abi._SIGNATURES) == set(names)


def test_status_strings(lib):
    for st in range(-8, 1):
        assert abi.status_string(st)
    assert "unknown" in abi.status_string(-99)
    assert abi.nvfp4_version() >= 100


@pytest.mark.parametrize("N,K,ok", [(1, 16, True), (5120, 5120, True), (0, 16, False), (8, 8, False),
                                    (8, 24, False), (-1, 64, False)])
def test_packed_bytes(lib, N, K, ok):
    st, nq, ns = abi.nvfp4_packed_bytes(N, K)
    if not ok:
        assert st == abi.NVFP4_ERR_SHAPE
        return
    assert st == abi.NVFP4_OK
    units = -(-N // 32) * -(-K // 64)
    assert nq == units * 1024 and ns == units * 128


def test_argument_errors_return_before_any_cuda_call(lib):
    p = 1 << 20  # a fake, aligned "device" pointer: never dereferenced on these paths
    assert abi.nvfp4_gemm_decode(p, 0, p, p, 1.0, p, 32, 64, None) == abi.NVFP4_ERR_M
    assert abi.nvfp4_gemm_decode(p, 65, p, p, 1.0, p, 32, 64, None) == abi.NVFP4_ERR_M
    assert abi.nvfp4_gemm_decode(p, 9, p, p, 1.0, p, 32, 40, None) == abi.NVFP4_ERR_SHAPE
    assert abi.nvfp4_gemm_decode(None, 20, p, p, 1.0, p, 32, 64, None) == abi.NVFP4_ERR_ARG
    assert abi.nvfp4_gemm_decode(p + 8, 64, p, p, 1.0, p, 32, 64, None) == abi.NVFP4_ERR_ALIGN
    assert abi.nvfp4_gemm_decode(p, 33, p, p, 1.0, p + 2, 32, 64, None) == abi.NVFP4_ERR_ALIGN
    assert abi.nvfp4_gemm_decode(p, 1, p, p, 1.0, p, 32, 40, None) == abi.NVFP4_ERR_SHAPE
    assert abi.nvfp4_gemm_decode(p, 1, p, p, 1.0, p, 0, 64, None) == abi.NVFP4_ERR_SHAPE
    assert abi.nvfp4_gemm_decode(None, 1, p, p, 1.0, p, 32, 64, None) == abi.NVFP4_ERR_ARG
    assert abi.nvfp4_gemm_decode(p + 8, 1, p, p, 1.0, p, 32, 64, None) == abi.NVFP4_ERR_ALIGN
    assert abi.nvfp4_gemm_decode(p, 1, p + 4, p, 1.0, p, 32, 64, None) == abi.NVFP4_ERR_ALIGN
    assert abi.nvfp4_gemm_decode(p, 1, p, p, 1.0, p + 2, 32, 64, None) == abi.NVFP4_ERR_ALIGN
    # widths 9..32 take the decode kernel's validation (lane blocks), 33..64 the tcgen05 kernel's
    assert abi.nvfp4_gemm_decode(p, 16, p, p, 1.0, p + 4, 32, 64, None) == abi.NVFP4_ERR_ALIGN
    assert abi.nvfp4_gemm_decode(p, 32, p + 8, p, 1.0, p, 32, 64, None) == abi.NVFP4_ERR_ALIGN
    assert abi.nvfp4_gemm_decode(p, 24, p, p, 1.0, p, 32, 0, None) == abi.NVFP4_ERR_SHAPE
    # the no-allocation entry point takes decode lanes only
    assert abi.nvfp4_gemm_decode_noalloc(p, 0, p, p, 1.0, p, 32, 64, None) == abi.NVFP4_ERR_M
    assert abi.nvfp4_gemm_decode_noalloc(p, 9, p, p, 1.0, p, 32, 64, None) == abi.NVFP4_ERR_M
    assert abi.nvfp4_gemm_decode_noalloc(p, 16, p, p, 1.0, p, 32, 64, None) == abi.NVFP4_ERR_M
    assert abi.nvfp4_gemm_gateup_silu(p, 1, p, p, 1.0, None, p, 1.0, p, 32, 64, None) == \
        abi.NVFP4_ERR_ARG
    assert abi.nvfp4_gemm_gateup_silu(p, 10, p, p, 1.0, p, p, 1.0, p, 32, 64, None) == abi.NVFP4_ERR_M
    assert abi.nvfp4_pack_check(None, p, 32, 64, p, p, None) == abi.NVFP4_ERR_ARG
    assert abi.nvfp4_pack_check(p, p, 32, 63, p, p, None) == abi.NVFP4_ERR_SHAPE
    assert abi.nvfp4_pack_check(p, p, 32, 64, p + 1, p, None) == abi.NVFP4_ERR_ALIGN
    assert abi.nvfp4_dequant_debug(p, p, 1.0, p + 4, 32, 64, None) == abi.NVFP4_ERR_ALIGN
    assert abi.nvfp4_round_replay(None, 1, None) == abi.NVFP4_ERR_ARG
    assert abi.nvfp4_round_destroy(None) == abi.NVFP4_OK
    bad = abi.Nvfp4GemmDesc(7, p, p, p, 1.0, None, None, 0.0, p, 32, 64)
    st, h = abi.nvfp4_round_create([bad])
    assert st == abi.NVFP4_ERR_ARG and not h
    badm = abi.Nvfp4GemmDesc(0, p, p, p, 1.0, None, None, 0.0, p, 32, 40)
    assert abi.nvfp4_round_create([badm])[0] == abi.NVFP4_ERR_SHAPE
    # grouped expert decode
    assert abi.nvfp4_gemm_grouped(None, 0, p, 2, 10, p, 512, p, 768, 2048, None) == abi.NVFP4_ERR_ARG
    assert abi.nvfp4_gemm_grouped(p, 0, p, 9, 10, p, 512, p, 768, 2048, None) == abi.NVFP4_ERR_M
    assert abi.nvfp4_gemm_grouped(p, 0, p, 8, 17, p, 512, p, 768, 2048, None) == abi.NVFP4_ERR_ARG
    assert abi.nvfp4_gemm_grouped(p, 0, p, 8, 10, p, 0, p, 768, 2048, None) == abi.NVFP4_ERR_ARG
    assert abi.nvfp4_gemm_grouped(p, 0, p, 8, 10, p, 512, p, 768, 2040, None) == abi.NVFP4_ERR_SHAPE
    assert abi.nvfp4_gemm_grouped(p, 0, p, 8, 10, p, 512, p, 131073, 2048, None) == abi.NVFP4_ERR_SHAPE
    assert abi.nvfp4_gemm_grouped(p + 8, 0, p, 8, 10, p, 512, p, 768, 2048, None) == abi.NVFP4_ERR_ALIGN
    assert abi.nvfp4_gemm_grouped(p, 0, p + 2, 8, 10, p, 512, p, 768, 2048, None) == abi.NVFP4_ERR_ALIGN
    assert abi.nvfp4_gemm_grouped(p, 0, p, 8, 10, p + 4, 512, p, 768, 2048, None) == abi.NVFP4_ERR_ALIGN
    # top-k over logits
    assert abi.nvfp4_topk(None, 1, 100, 100, 1, p, p, None) == abi.NVFP4_ERR_ARG
    assert abi.nvfp4_topk(p, 0, 100, 100, 1, p, p, None) == abi.NVFP4_ERR_M
    assert abi.nvfp4_topk(p, 65, 100, 100, 1, p, p, None) == abi.NVFP4_ERR_M
    assert abi.nvfp4_topk(p, 1, 100, 100, 0, p, p, None) == abi.NVFP4_ERR_SHAPE
    assert abi.nvfp4_topk(p, 1, 100, 100, 65, p, p, None) == abi.NVFP4_ERR_SHAPE
    assert abi.nvfp4_topk(p, 1, 5, 8, 6, p, p, None) == abi.NVFP4_ERR_SHAPE
    assert abi.nvfp4_topk(p, 1, 100, 96, 1, p, p, None) == abi.NVFP4_ERR_SHAPE
    assert abi.nvfp4_topk(p, 1, (1 << 24) + 4, (1 << 24) + 4, 1, p, p, None) == abi.NVFP4_ERR_SHAPE
    assert abi.nvfp4_topk(p + 4, 1, 100, 100, 1, p, p, None) == abi.NVFP4_ERR_ALIGN
    assert abi.nvfp4_topk(p, 1, 100, 102, 1, p, p, None) == abi.NVFP4_ERR_ALIGN
    assert abi.nvfp4_topk(p, 1, 100, 100, 1, p + 2, p, None) == abi.NVFP4_ERR_ALIGN
    # read-only stream probe
    assert abi.nvfp4_stream_read(None, 64, p, 4, None) == abi.NVFP4_ERR_ARG
    assert abi.nvfp4_stream_read(p, 64, None, 4, None) == abi.NVFP4_ERR_ARG
    assert abi.nvfp4_stream_read(p, 64, p, 0, None) == abi.NVFP4_ERR_ARG
    assert abi.nvfp4_stream_read(p, 64, p, (1 << 20) + 1, None) == abi.NVFP4_ERR_ARG
    assert abi.nvfp4_stream_read(p, 0, p, 4, None) == abi.NVFP4_ERR_SHAPE
    assert abi.nvfp4_stream_read(p, 72, p, 4, None) == abi.NVFP4_ERR_SHAPE
    assert abi.nvfp4_stream_read(p + 8, 64, p, 4, None) == abi.NVFP4_ERR_ALIGN
    assert abi.nvfp4_stream_read(p, 64, p + 2, 4, None) == abi.NVFP4_ERR_ALIGN


@pytest.mark.parametrize("rows", [1, 2, 3, 8, 13, 64])
@pytest.mark.parametrize("V", [1, 3, 4, 5, 63, 255, 256, 257, 1000, 4099, 12289, 151936, 151937, 1 << 20, 3_000_000])
@pytest.mark.parametrize("k", [1, 7, 8, 64])
def test_topk_row_split(lib, rows, V, k):
    """The row split of nvfp4_topk: slices a multiple of 4 long and at most
    12,288 elements, none empty, covering the row; the merge (splits * k)
    within 16,384 candidates; and an error exactly when no split fits."""
    st, S, slice_ = abi.nvfp4_topk_splits(rows, V, k, 148)
    if k > V:
        assert st == abi.NVFP4_ERR_SHAPE
        return
    fits = any(sl <= 12288 and -(-V // sl) * k <= 16384 for sl in range(4, 12289, 4))
    if not fits:
        assert st == abi.NVFP4_ERR_SHAPE
        return
    assert st == abi.NVFP4_OK
    assert slice_ % 4 == 0 and 4 <= slice_ <= 12288
    assert (S - 1) * slice_ < V <= S * slice_
    assert S * k <= 16384


def _host_dequant(q, s, gscale):
    """Dequantise a whole matrix through the library's host model, unit by unit."""
    N, K = q.shape[0], q.shape[1] * 2
    nt, kc = -(-N // 32), -(-K // 64)
    W = np.zeros((nt * 32, kc * 64), np.float32)
    qu = np.zeros(1024, np.uint8)
    su = np.zeros(128, np.uint8)
    Wu = np.zeros((32, 64), np.float32)
    for tile in range(nt):
        for chunk in range(kc):
            abi.check(abi.nvfp4_host_pack_unit(_ptr(q), _ptr(s), N, K, tile, chunk, _ptr(qu), _ptr(su)))
            abi.check(abi.nvfp4_host_dequant_unit(_ptr(qu), _ptr(su), gscale, _ptr(Wu)))
            W[tile * 32:(tile + 1) * 32, chunk * 64:(chunk + 1) * 64] = Wu
    return W[:N, :K], W


@pytest.mark.parametrize("N,K", [(32, 64), (256, 512), (45, 80), (7, 16), (33, 208)])
def test_host_layout_model_dequant_is_bit_exact(lib, N, K):
    q, s = synth.matrix(20, N * 7 + K, N, K)
    W, Wfull = _host_dequant(q, s, 1.0 / 64)
    ref = oracle.dequant(q, s, 1.0 / 64)
    assert np.array_equal(W.view(np.uint32), ref.view(np.uint32))
    # padding rows and columns dequantise to zero
    pad = Wfull.copy()
    pad[:N, :K] = 0
    assert not np.any(pad)


def test_host_layout_model_special_scales(lib):
    N, K = 32, 128
    q, s = synth.matrix(21, 0, N, K)
    specials = [0x00, 0x80, 0x01, 0x07, 0x08, 0x7E, 0xFE, 0xB9, 0x81, 0x3F]
    for i, b in enumerate(specials):
        s[i % N, i % (K // 16)] = b
    for gscale in (1.0, 1.0 / 64, 3.0, -0.5):
        W, _ = _host_dequant(q, s, gscale)
        ref = oracle.dequant(q, s, gscale)
        assert np.array_equal(W.view(np.uint32), ref.view(np.uint32)), gscale


def test_host_layout_model_every_code_with_every_scale(lib):
    # rows cycle the 254 non-NaN scale codes, columns cycle the 16 element codes
    scales = np.array([b for b in range(256) if (b & 0x7F) != 0x7F], np.uint8)
    N, K = 256, 64
    q = np.zeros((N, K // 2), np.uint8)
    codes = np.arange(K) % 16
    q[:] = (codes[0::2] | (codes[1::2] << 4)).astype(np.uint8)
    s = np.repeat(scales[np.arange(N) % scales.size][:, None], K // 16, axis=1).astype(np.uint8)
    W, _ = _host_dequant(q, s, 1.0)
    ref = oracle.dequant(q, s, 1.0)
    assert np.array_equal(W.view(np.uint32), ref.view(np.uint32))


@pytest.mark.parametrize("M", [9, 16, 17, 33, 48, 64])
@pytest.mark.parametrize("N,K", [(1, 16), (32, 64), (256, 512), (5120, 5120), (5120, 17408), (34816, 5120),
                                 (151936, 5120), (1000, 1040)])
def test_verify_geometry(lib, M, N, K):
    """Work split of the verify-width kernel: every CTA owns a non-empty range
    of (256-row group, pair of 64-column chunks) units, one CTA per SM at
    most, no more than 8 CTAs per group on average, and the MMA's N is M
    rounded up to 16."""
    st, ctas, units, nl = abi.nvfp4_verify_geometry(M, N, K, 148)
    assert st == abi.NVFP4_OK
    groups = -(-(-(-N // 32)) // 8)
    assert units == groups * -(-(-(-K // 64)) // 2)
    assert 1 <= ctas <= min(148, units, 8 * groups)
    assert nl % 16 == 0 and M <= nl < M + 16
    assert all(units * (i + 1) // ctas > units * i // ctas for i in range(ctas))


def test_verify_geometry_rejects():
    assert abi.nvfp4_verify_geometry(8, 32, 64, 148)[0] == abi.NVFP4_ERR_M
    assert abi.nvfp4_verify_geometry(65, 32, 64, 148)[0] == abi.NVFP4_ERR_M
    assert abi.nvfp4_verify_geometry(16, 32, 40, 148)[0] == abi.NVFP4_ERR_SHAPE
    assert abi.nvfp4_verify_geometry(16, 0, 64, 148)[0] == abi.NVFP4_ERR_SHAPE


def test_header_compiles_as_c99_and_links_from_c(lib, tmp_path):
    """include/nvfp4decode.h is a C header: a C99 program built with -Wall
    -Wextra -Werror against it links the library and gets the expected answers
    from its host-side calls (tests/abi_c_check.c)."""
    import subprocess
    here = os.path.dirname(os.path.abspath(__file__))
    root = os.path.dirname(here)
    libdir = os.path.dirname(abi.LIB_PATH)
    exe = str(tmp_path / "abi_c_check")
    subprocess.run(["gcc", "-std=c99", "-Wall", "-Wextra", "-Werror", "-pedantic", "-I", os.path.join(root, "include"),
                    os.path.join(here, "abi_c_check.c"), "-o", exe, "-L", libdir, "-lnvfp4decode",
                    "-Wl,-rpath," + libdir], check=True)
    out = subprocess.run([exe], capture_output=True, text=True, timeout=120)
    assert out.returncode == 0, out.stderr
    assert out.stdout.strip() == "ok"
