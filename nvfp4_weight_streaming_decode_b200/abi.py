"""ctypes binding of libnvfp4decode.so -- argument marshalling only.

Every function named ``nvfp4_*`` here has the C signature of the same name in
``include/nvfp4decode.h`` and returns its status (``NVFP4_OK`` = 0).  Device
pointers and streams are plain integers (``tensor.data_ptr()``,
``torch.cuda.current_stream().cuda_stream``).  The torch helpers at the end
only allocate device memory and pass pointers; all compute runs in the
library's CUDA kernels.  If the library is missing this module raises: there
is no fallback.
"""
from __future__ import annotations

import ctypes
import os
import re

HERE = os.path.dirname(os.path.abspath(__file__))
# NVFP4_LIB may name another build of the same library (same ABI).
LIB_PATH = os.environ.get("NVFP4_LIB") or os.path.join(HERE, "libnvfp4decode.so")
HEADER = os.path.join(os.path.dirname(HERE), "include", "nvfp4decode.h")

NVFP4_OK = 0
NVFP4_ERR_ARG = -1
NVFP4_ERR_M = -2
NVFP4_ERR_SHAPE = -3
NVFP4_ERR_ALIGN = -4
NVFP4_ERR_BAD_SCALE = -5
NVFP4_ERR_CUDA = -6
NVFP4_ERR_CAPTURE = -7
NVFP4_ERR_DEVICE = -8
NVFP4_ERR_SCRATCH = -9
NVFP4_ROUND_PERSISTENT = 0
NVFP4_ROUND_CHAIN = 1
NVFP4_DESC_GEMM = 0
NVFP4_DESC_GATEUP_SILU = 1
NVFP4_TOPK_MAX_ROWS = 64
NVFP4_TOPK_MAX_K = 64
NVFP4_TOPK_MAX_V = 1 << 24
NVFP4_GROUPED_MAX_ROUTES = 128
NVFP4_MAX_M = 64          # nvfp4_gemm_decode: 1..8 decode lanes, 9..64 verify rows

_P = ctypes.c_void_p
_I64 = ctypes.c_int64
_SZ = ctypes.c_size_t
_F = ctypes.c_float
_I = ctypes.c_int


class Nvfp4Expert(ctypes.Structure):
    _fields_ = [("wq", _P), ("ws", _P), ("gscale", _F), ("reserved", ctypes.c_int32)]


class Nvfp4GemmDesc(ctypes.Structure):
    _fields_ = [("kind", _I), ("X", _P), ("wq", _P), ("ws", _P), ("gscale", _F),
                ("wq2", _P), ("ws2", _P), ("gscale2", _F), ("out", _P), ("N", _I64), ("K", _I64)]


_SIGNATURES = {
    "nvfp4_packed_bytes": (_I, [_I64, _I64, ctypes.POINTER(_SZ), ctypes.POINTER(_SZ)]),
    "nvfp4_pack_check": (_I, [_P, _P, _I64, _I64, _P, _P, _P]),
    "nvfp4_gemm_decode": (_I, [_P, _I, _P, _P, _F, _P, _I64, _I64, _P]),
    "nvfp4_gemm_decode_noalloc": (_I, [_P, _I, _P, _P, _F, _P, _I64, _I64, _P]),
    "nvfp4_gemm_gateup_silu": (_I, [_P, _I, _P, _P, _F, _P, _P, _F, _P, _I64, _I64, _P]),
    "nvfp4_round_create": (_I, [ctypes.POINTER(Nvfp4GemmDesc), _I, ctypes.POINTER(_P)]),
    "nvfp4_round_create_ex": (_I, [ctypes.POINTER(Nvfp4GemmDesc), _I, _I, ctypes.POINTER(_P)]),
    "nvfp4_round_nodes": (_I, [_P, ctypes.POINTER(_I)]),
    "nvfp4_round_replay": (_I, [_P, _I, _P]),
    "nvfp4_round_replay_host": (_I, [_P, _I, _P, _P, _SZ, _P, _P, _SZ, _P]),
    "nvfp4_round_destroy": (_I, [_P]),
    "nvfp4_topk": (_I, [_P, _I, _I64, _I64, _I, _P, _P, _P]),
    "nvfp4_gemm_grouped": (_I, [_P, _I, _P, _I, _I, _P, _I, _P, _I64, _I64, _P]),
    "nvfp4_topk_splits": (_I, [_I, _I64, _I, _I, ctypes.POINTER(_I), ctypes.POINTER(_I)]),
    "nvfp4_verify_geometry": (_I, [_I, _I64, _I64, _I, ctypes.POINTER(_I64), ctypes.POINTER(_I64),
                                   ctypes.POINTER(_I)]),
    "nvfp4_dequant_debug": (_I, [_P, _P, _F, _P, _I64, _I64, _P]),
    "nvfp4_unpack_debug": (_I, [_P, _P, _I64, _I64, _P, _P, _P]),
    "nvfp4_host_dequant_unit": (_I, [_P, _P, _F, _P]),
    "nvfp4_host_pack_unit": (_I, [_P, _P, _I64, _I64, _I64, _I64, _P, _P]),
    "nvfp4_stream_read": (_I, [_P, _SZ, _P, _I, _P]),
    "nvfp4_status_string": (ctypes.c_char_p, [_I]),
    "nvfp4_last_cuda_error": (_I, []),
    "nvfp4_device_status": (_I, []),
    "nvfp4_version": (_I, []),
}

_lib = None


def load():
    """Load the library (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with __graft_entry__.build()")
        lib = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in _SIGNATURES.items():
            fn = getattr(lib, name)
            fn.restype = res
            fn.argtypes = args
        _lib = lib
    return _lib


def header_functions():
    """Names of the functions include/nvfp4decode.h declares."""
    with open(HEADER) as f:
        text = f.read()
    return sorted(set(re.findall(r"NVFP4_API\s+[\w\s\*]+?\b(nvfp4_\w+)\s*\(", text)))


class Nvfp4Error(RuntimeError):
    def __init__(self, status: int, what: str = ""):
        msg = status_string(status)
        if status == NVFP4_ERR_CUDA:
            msg += f" (cuda error {load().nvfp4_last_cuda_error()})"
        super().__init__(f"{what}: {msg} [{status}]" if what else f"{msg} [{status}]")
        self.status = status


def status_string(status: int) -> str:
    return load().nvfp4_status_string(int(status)).decode()


def check(status: int, what: str = "") -> int:
    if status != NVFP4_OK:
        raise Nvfp4Error(status, what)
    return status


def _s(stream):
    return None if stream is None else int(stream)


# ------------------------------------------------------- raw C-ABI calls

def nvfp4_packed_bytes(N, K):
    """(status, wq_bytes, ws_bytes)."""
    a, b = _SZ(), _SZ()
    st = load().nvfp4_packed_bytes(int(N), int(K), ctypes.byref(a), ctypes.byref(b))
    return st, a.value, b.value


def nvfp4_pack_check(wq_canon, ws_canon, N, K, wq_dev, ws_dev, stream):
    return load().nvfp4_pack_check(wq_canon, ws_canon, int(N), int(K), wq_dev, ws_dev, _s(stream))


def nvfp4_gemm_decode(X, M, wq_dev, ws_dev, gscale, Y, N, K, stream):
    return load().nvfp4_gemm_decode(X, int(M), wq_dev, ws_dev, float(gscale), Y, int(N), int(K),
                                    _s(stream))


def nvfp4_gemm_decode_noalloc(X, M, wq_dev, ws_dev, gscale, Y, N, K, stream):
    """nvfp4_gemm_decode without any device allocation (static scratch array in the library)."""
    return load().nvfp4_gemm_decode_noalloc(X, int(M), wq_dev, ws_dev, float(gscale), Y, int(N), int(K),
                                            _s(stream))


def nvfp4_gemm_gateup_silu(X, M, wq_gate, ws_gate, gscale_gate, wq_up, ws_up, gscale_up, H, Nff, K,
                           stream):
    return load().nvfp4_gemm_gateup_silu(X, int(M), wq_gate, ws_gate, float(gscale_gate), wq_up,
                                         ws_up, float(gscale_up), H, int(Nff), int(K), _s(stream))


def nvfp4_round_create(descs):
    """(status, handle) for a sequence of Nvfp4GemmDesc."""
    arr = (Nvfp4GemmDesc * len(descs))(*descs)
    h = _P()
    st = load().nvfp4_round_create(arr, len(descs), ctypes.byref(h))
    return st, h.value


def nvfp4_round_create_ex(descs, mode):
    """(status, handle) for a sequence of Nvfp4GemmDesc, with a round mode."""
    arr = (Nvfp4GemmDesc * len(descs))(*descs)
    h = _P()
    st = load().nvfp4_round_create_ex(arr, len(descs), int(mode), ctypes.byref(h))
    return st, h.value


def nvfp4_round_nodes(handle):
    n = _I()
    st = load().nvfp4_round_nodes(handle, ctypes.byref(n))
    return st, n.value


def nvfp4_round_replay(handle, M, stream):
    return load().nvfp4_round_replay(handle, int(M), _s(stream))


def nvfp4_round_replay_host(handle, M, x_host, x_dev, x_bytes, y_dev, y_host, y_bytes, stream):
    return load().nvfp4_round_replay_host(handle, int(M), x_host, x_dev, int(x_bytes), y_dev, y_host,
                                          int(y_bytes), _s(stream))


def nvfp4_round_destroy(handle):
    return load().nvfp4_round_destroy(handle)


def nvfp4_gemm_grouped(X, x_per_route, route, M, T, experts, E, Y, N, K, stream):
    return load().nvfp4_gemm_grouped(X, int(x_per_route), route, int(M), int(T), experts, int(E), Y, int(N), int(K),
                                     _s(stream))


def nvfp4_topk(logits, rows, V, ldv, k, values, indices, stream):
    return load().nvfp4_topk(logits, int(rows), int(V), int(ldv), int(k), values, indices, _s(stream))


def nvfp4_topk_splits(rows, V, k, sm_count):
    """(status, splits, slice) of the row split nvfp4_topk uses."""
    sp, sl = _I(0), _I(0)
    st = load().nvfp4_topk_splits(int(rows), int(V), int(k), int(sm_count), ctypes.byref(sp), ctypes.byref(sl))
    return st, sp.value, sl.value


def nvfp4_verify_geometry(M, N, K, sm_count):
    """(status, ctas, units, nl) of the verify-width work split."""
    c, u, nl = _I64(0), _I64(0), _I(0)
    st = load().nvfp4_verify_geometry(int(M), int(N), int(K), int(sm_count), ctypes.byref(c), ctypes.byref(u),
                                      ctypes.byref(nl))
    return st, c.value, u.value, nl.value


def nvfp4_dequant_debug(wq_dev, ws_dev, gscale, W, N, K, stream):
    return load().nvfp4_dequant_debug(wq_dev, ws_dev, float(gscale), W, int(N), int(K), _s(stream))


def nvfp4_unpack_debug(wq_dev, ws_dev, N, K, wq_canon, ws_canon, stream):
    return load().nvfp4_unpack_debug(wq_dev, ws_dev, int(N), int(K), wq_canon, ws_canon, _s(stream))


def nvfp4_host_dequant_unit(q_unit, s_unit, gscale, W):
    return load().nvfp4_host_dequant_unit(q_unit, s_unit, float(gscale), W)


def nvfp4_host_pack_unit(wq_canon, ws_canon, N, K, tile, chunk, q_unit, s_unit):
    return load().nvfp4_host_pack_unit(wq_canon, ws_canon, int(N), int(K), int(tile), int(chunk),
                                       q_unit, s_unit)


def nvfp4_stream_read(buf, nbytes, out, ctas, stream):
    return load().nvfp4_stream_read(buf, int(nbytes), out, int(ctas), _s(stream))


def nvfp4_status_string(status):
    return status_string(status)


def nvfp4_last_cuda_error():
    return load().nvfp4_last_cuda_error()


def nvfp4_device_status():
    return load().nvfp4_device_status()


def nvfp4_version():
    return load().nvfp4_version()


# ------------------------------------------------------- torch helpers

def _stream_ptr(stream=None):
    import torch
    s = torch.cuda.current_stream() if stream is None else stream
    return s.cuda_stream


def pack(q_canon, s_canon, stream=None):
    """Pack canonical device planes (torch uint8 [N][K/2], [N][K/16]) into
    freshly allocated device-layout planes; returns (wq_dev, ws_dev)."""
    import torch
    N, half_k = q_canon.shape
    K = half_k * 2
    st, nq, ns = nvfp4_packed_bytes(N, K)
    check(st, "nvfp4_packed_bytes")
    wq = torch.empty(nq, dtype=torch.uint8, device=q_canon.device)
    ws = torch.empty(ns, dtype=torch.uint8, device=q_canon.device)
    check(nvfp4_pack_check(q_canon.data_ptr(), s_canon.data_ptr(), N, K, wq.data_ptr(),
                           ws.data_ptr(), _stream_ptr(stream)), "nvfp4_pack_check")
    return wq, ws


def gemm_decode(X, wq, ws, gscale, N, K, Y=None, stream=None):
    """Y float32 [M][N] = gscale * X . dequant(W)^T (X: torch bf16 [M][K] on the device)."""
    import torch
    M = X.shape[0]
    if Y is None:
        Y = torch.empty((M, N), dtype=torch.float32, device=X.device)
    check(nvfp4_gemm_decode(X.data_ptr(), M, wq.data_ptr(), ws.data_ptr(), gscale, Y.data_ptr(), N,
                            K, _stream_ptr(stream)), "nvfp4_gemm_decode")
    return Y


def gemm_gateup_silu(X, wq_g, ws_g, gscale_g, wq_u, ws_u, gscale_u, Nff, K, H=None, stream=None):
    """H bf16 [M][Nff] = silu(X . Wg^T) * (X . Wu^T), one launch."""
    import torch
    M = X.shape[0]
    if H is None:
        H = torch.empty((M, Nff), dtype=torch.bfloat16, device=X.device)
    check(nvfp4_gemm_gateup_silu(X.data_ptr(), M, wq_g.data_ptr(), ws_g.data_ptr(), gscale_g,
                                 wq_u.data_ptr(), ws_u.data_ptr(), gscale_u, H.data_ptr(), Nff, K,
                                 _stream_ptr(stream)), "nvfp4_gemm_gateup_silu")
    return H


def expert_table(mats, device):
    """Device array of nvfp4_expert for a list of (wq, ws, gscale) device-layout planes."""
    import numpy as np
    import torch
    rec = np.zeros((len(mats), 3), dtype=np.uint64)
    for i, (wq, ws, gs) in enumerate(mats):
        rec[i, 0] = wq.data_ptr()
        rec[i, 1] = ws.data_ptr()
        rec[i, 2] = int(np.float32(gs).view(np.uint32))  # gscale in the low 32 bits, reserved = 0
    return torch.from_numpy(rec.view(np.int64)).to(device)


def gemm_grouped(X, route, experts, E, N, K, x_per_route=False, Y=None, stream=None):
    """Y float32 [M][T][N] for routes int32 [M][T] over the expert table (expert_table)."""
    import torch
    M, T = route.shape
    if Y is None:
        Y = torch.empty((M, T, N), dtype=torch.float32, device=X.device)
    check(nvfp4_gemm_grouped(X.data_ptr(), 1 if x_per_route else 0, route.data_ptr(), M, T, experts.data_ptr(), E,
                             Y.data_ptr(), N, K, _stream_ptr(stream)), "nvfp4_gemm_grouped")
    return Y


def topk(logits, k, V=None, values=None, indices=None, stream=None):
    """Top-k of each row of torch float32 [rows][ldv] device logits over the
    first V columns: (values float32 [rows][k], indices int32 [rows][k])."""
    import torch
    rows, ldv = logits.shape
    V = ldv if V is None else int(V)
    if logits.stride(1) != 1:
        raise ValueError("logits rows must be contiguous")
    if values is None:
        values = torch.empty((rows, k), dtype=torch.float32, device=logits.device)
    if indices is None:
        indices = torch.empty((rows, k), dtype=torch.int32, device=logits.device)
    check(nvfp4_topk(logits.data_ptr(), rows, V, logits.stride(0), k, values.data_ptr(), indices.data_ptr(),
                     _stream_ptr(stream)), "nvfp4_topk")
    return values, indices


def stream_read(buf, ctas, out=None, stream=None):
    """Read every byte of the contiguous device tensor `buf` once (nvfp4_stream_read);
    returns the uint32 [ctas] device tensor of per-CTA XORs (as int32)."""
    import torch
    if not buf.is_contiguous():
        raise ValueError("buf must be contiguous")
    if out is None:
        out = torch.empty((ctas,), dtype=torch.int32, device=buf.device)
    check(nvfp4_stream_read(buf.data_ptr(), buf.numel() * buf.element_size(), out.data_ptr(), ctas,
                            _stream_ptr(stream)), "nvfp4_stream_read")
    return out


def dequant_debug(wq, ws, gscale, N, K, stream=None):
    import torch
    W = torch.empty((N, K), dtype=torch.float32, device=wq.device)
    check(nvfp4_dequant_debug(wq.data_ptr(), ws.data_ptr(), gscale, W.data_ptr(), N, K,
                              _stream_ptr(stream)), "nvfp4_dequant_debug")
    return W


def unpack_debug(wq, ws, N, K, stream=None):
    import torch
    q = torch.empty((N, K // 2), dtype=torch.uint8, device=wq.device)
    s = torch.empty((N, K // 16), dtype=torch.uint8, device=wq.device)
    check(nvfp4_unpack_debug(wq.data_ptr(), ws.data_ptr(), N, K, q.data_ptr(), s.data_ptr(),
                             _stream_ptr(stream)), "nvfp4_unpack_debug")
    return q, s


class Round:
    """Owner of an nvfp4_round handle built from descriptors."""

    def __init__(self, descs, mode=None):
        if mode is None:
            st, h = nvfp4_round_create(descs)
        else:
            st, h = nvfp4_round_create_ex(descs, mode)
        check(st, "nvfp4_round_create")
        self.handle = h
        self._descs = list(descs)

    @property
    def nodes(self):
        st, n = nvfp4_round_nodes(self.handle)
        check(st, "nvfp4_round_nodes")
        return n

    def replay(self, M, stream=None):
        check(nvfp4_round_replay(self.handle, M, _stream_ptr(stream)), "nvfp4_round_replay")

    def replay_host(self, M, x_host, x_dev, y_dev, y_host, stream=None):
        """H2D copy of x_host -> x_dev, replay, D2H copy of y_dev -> y_host (torch tensors)."""
        xb = x_host.numel() * x_host.element_size()
        yb = y_host.numel() * y_host.element_size()
        check(nvfp4_round_replay_host(self.handle, M, x_host.data_ptr(), x_dev.data_ptr(), xb,
                                      y_dev.data_ptr(), y_host.data_ptr(), yb, _stream_ptr(stream)),
              "nvfp4_round_replay_host")

    def close(self):
        if self.handle:
            nvfp4_round_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def desc(kind, X, wq, ws, gscale, out, N, K, wq2=None, ws2=None, gscale2=0.0):
    """An Nvfp4GemmDesc from torch tensors."""
    return Nvfp4GemmDesc(kind, X.data_ptr(), wq.data_ptr(), ws.data_ptr(), float(gscale),
                         wq2.data_ptr() if wq2 is not None else None,
                         ws2.data_ptr() if ws2 is not None else None, float(gscale2),
                         out.data_ptr(), int(N), int(K))
