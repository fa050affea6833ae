"""Thin ctypes binding of the C ABI in ``include/rbw.h`` (librbw.so).

Argument marshalling only: every step of the computation runs in the CUDA
library.  Tensors must be CUDA tensors on the current device; the calls are
issued on torch's current stream.  A missing library raises immediately
(there is no fallback path).
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "librbw.so")

RB_OK, RB_ERR_ARG, RB_ERR_SHAPE, RB_ERR_ALIGN, RB_ERR_WORKSPACE, RB_ERR_UNSUPPORTED, RB_ERR_CUDA = range(7)
RB_DEV_NONFINITE, RB_DEV_RANGE, RB_DEV_TIMEOUT = 0x1, 0x2, 0x4
RB_F32, RB_BF16 = 0, 1
RB_LAUNCH_PDL = 0x1

# name -> (restype, argtypes); the full exported surface of include/rbw.h
_vp, _i32, _sz, _u32 = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t, ctypes.c_uint
SIGNATURES = {
    "rb_version": (_i32, []),
    "rb_status_string": (ctypes.c_char_p, [_i32]),
    "rb_packed_words": (_sz, [_i32, _i32, _i32]),
    "rb_pack": (_i32, [_vp, _vp, _vp, _i32, _i32, _i32, _vp, _vp, _vp, _vp, _vp]),
    "rb_gemv_workspace_bytes": (_sz, [_i32, _i32, _i32, _i32]),
    "rb_gemv": (_i32, [_vp, _vp, _i32, _vp, _i32, _vp, _sz, _vp, _u32, _vp]),
    "rb_gemv_batch": (_i32, [_vp, _vp, _vp, _i32, _i32, _i32, _vp, _u32, _vp]),
    "rb_gemm_workspace_bytes": (_sz, [_i32, _i32, _i32, _i32]),
    "rb_gemm": (_i32, [_vp, _vp, _i32, _vp, _i32, _vp, _sz, _vp, _u32, _vp]),
    "rb_gemm_wait_limit": (_i32, [_vp, _vp, _i32, _vp, _i32, _vp, _sz, _vp, _u32, ctypes.c_uint64, _vp]),
    "rb_gemm_noalloc": (_i32, [_vp, _vp, _i32, _vp, _i32, _vp, _u32, _vp]),
    "rb_transpose_planes": (_i32, [_vp, _vp, _vp]),
    "rb_rowmajor_words": (_sz, [_i32, _i32, _i32]),
    "rb_shard_rows": (_i32, [_vp, _i32, _i32, _vp, _vp, _vp]),
    "rb_planes_from_rowmajor": (_i32, [_vp, _i32, _i32, _i32, _vp, _vp]),
    "rb_planes_to_rowmajor": (_i32, [_vp, _i32, _i32, _i32, _vp, _vp]),
    "rb_qat_forward_workspace_bytes": (_sz, [_i32, _i32, _i32, _i32]),
    "rb_qat_forward": (_i32, [_vp, _vp, _vp, _i32, _i32, _i32, _vp, _i32, _vp, _i32, _vp, _sz, _vp, _u32, _vp]),
    "rb_qat_backward_workspace_bytes": (_sz, [_i32, _i32, _i32]),
    "rb_qat_backward": (_i32, [_vp, _vp, _vp, _i32, _i32, _i32, _vp, _vp, _i32, _vp, _vp, _vp, _vp, _sz, _vp, _vp]),
    "rb_btc_index_bits": (_i32, [_i32]),
    "rb_btc_row_words": (_sz, [_i32, _i32]),
    "rb_btc_encode_workspace_bytes": (_sz, [_i32]),
    "rb_btc_encode": (_i32, [_vp, _i32, _i32, _i32, _vp, _vp, _vp, _vp, _sz, _vp]),
    "rb_btc_gemv_workspace_bytes": (_sz, [_i32, _i32]),
    "rb_btc_gemv": (_i32, [_vp, _vp, _vp, _i32, _vp, _sz, _vp, _u32, _vp]),
    "rb_btc_gemv_batch_workspace_bytes": (_sz, [_i32, _i32, _i32]),
    "rb_btc_gemv_batch": (_i32, [_vp, _vp, _vp, _i32, _i32, _vp, _sz, _vp, _u32, _vp]),
    "rb_svid_workspace_bytes": (_sz, [_i32, _i32]),
    "rb_svid_greedy": (_i32, [_vp, _i32, _i32, _i32, _i32, _vp, _vp, _vp, _sz, _vp]),
    "rb_svid_iterative_workspace_bytes": (_sz, [_i32, _i32, _i32]),
    "rb_svid_iterative": (_i32, [_vp, _i32, _i32, _i32, _i32, _i32, _vp, _vp, _vp, _sz, _vp]),
    "rb_svid_pack_workspace_bytes": (_sz, [_i32, _i32, _i32]),
    "rb_svid_pack": (_i32, [_vp, _i32, _i32, _i32, _i32, _i32, _vp, _vp, _vp, _vp, _vp, _vp, _sz, _vp, _vp]),
}


class RbLayer(ctypes.Structure):
    _fields_ = [("n_out", ctypes.c_int32), ("k_in", ctypes.c_int32), ("k_planes", ctypes.c_int32),
                ("reserved", ctypes.c_int32), ("planes", _vp), ("g16", _vp), ("h16", _vp)]


class RbBtcLayer(ctypes.Structure):
    _fields_ = [("n_out", ctypes.c_int32), ("k_in", ctypes.c_int32), ("k_planes", ctypes.c_int32),
                ("c_max", ctypes.c_int32), ("index_bits", ctypes.c_int32), ("reserved", ctypes.c_int32),
                ("codebooks", _vp), ("indices", _vp), ("g16", _vp), ("h16", _vp)]


_lib = None


def lib():
    """Load librbw.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError("librbw.so not found at %s: run residual_binarized_weight_b200/build.py" % LIB_PATH)
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


class RbError(RuntimeError):
    def __init__(self, fn, status):
        self.status = status
        super().__init__("%s failed: %s" % (fn, lib().rb_status_string(status).decode()))


def _check(fn, status):
    if status != RB_OK:
        raise RbError(fn, status)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def packed_words(n_out, k_in, k_planes):
    return int(lib().rb_packed_words(n_out, k_in, k_planes))


class PackedLayer:
    """Device tensors of one packed layer (owns them) plus its rb_layer_t view."""

    def __init__(self, n_out, k_in, k_planes, device="cuda", g16=None, h16=None):
        """New planes; new scale tensors unless existing ones are passed to share."""
        nw = packed_words(n_out, k_in, k_planes)
        if nw == 0:
            raise ValueError("invalid layer shape")
        self.n_out, self.k_in, self.k_planes = n_out, k_in, k_planes
        self.planes = torch.empty(nw, dtype=torch.int32, device=device)
        self.g16 = torch.empty(k_planes, n_out, dtype=torch.float16, device=device) if g16 is None else g16
        self.h16 = torch.empty(k_planes, k_in, dtype=torch.float16, device=device) if h16 is None else h16
        if tuple(self.g16.shape) != (k_planes, n_out) or tuple(self.h16.shape) != (k_planes, k_in):
            raise ValueError("scale tensors do not match the layer shape")

    def struct(self):
        return RbLayer(self.n_out, self.k_in, self.k_planes, 0, self.planes.data_ptr(),
                       self.g16.data_ptr(), self.h16.data_ptr())

    def packed_bytes(self):
        return self.planes.numel() * 4


def pack(W, g, h, k_planes, out: PackedLayer | None = None, dev_status=None, stream=None):
    """rb_pack: W fp32 [N][K], g fp32 [k][N], h fp32 [k][K] (CUDA) -> PackedLayer."""
    N, K = W.shape
    out = out or PackedLayer(N, K, k_planes, W.device)
    st = lib().rb_pack(_ptr(W), _ptr(g), _ptr(h), N, K, k_planes, _ptr(out.planes), _ptr(out.g16),
                       _ptr(out.h16), _ptr(dev_status), _stream(stream))
    _check("rb_pack", st)
    return out


def gemv_workspace_bytes(n_out, k_in, k_planes, M):
    return int(lib().rb_gemv_workspace_bytes(n_out, k_in, k_planes, M))


def gemm_workspace_bytes(n_out, k_in, k_planes, M):
    return int(lib().rb_gemm_workspace_bytes(n_out, k_in, k_planes, M))


def svid_workspace_bytes(n_out, k_in):
    return int(lib().rb_svid_workspace_bytes(n_out, k_in))


def workspace(nbytes, device="cuda"):
    """Zero-filled device workspace (uint8) of at least nbytes (16-byte aligned)."""
    return torch.zeros(max(int(nbytes), 16), dtype=torch.uint8, device=device)


def _apply(fn_name, layer: PackedLayer, X, Y, ws, flags, dev_status, stream):
    M = X.shape[0]
    ydt = RB_BF16 if Y.dtype == torch.bfloat16 else RB_F32
    L = layer.struct()
    wsp, wsb = (None, 0) if ws is None else (_ptr(ws), ws.numel() * ws.element_size())
    st = getattr(lib(), fn_name)(ctypes.byref(L), _ptr(X), M, _ptr(Y), ydt, wsp, wsb,
                                 _ptr(dev_status), flags, _stream(stream))
    _check(fn_name, st)
    return Y


def gemv(layer: PackedLayer, X, Y=None, ws=None, flags=0, dev_status=None, stream=None, y_dtype=torch.float32):
    """rb_gemv: X bf16 [M][K] (M <= 64) -> Y [M][N] (fp32 or bf16)."""
    if Y is None:
        Y = torch.empty(X.shape[0], layer.n_out, dtype=y_dtype, device=X.device)
    return _apply("rb_gemv", layer, X, Y, ws, flags, dev_status, stream)


def gemv_batch(layers, Xs, Ys, flags=0, dev_status=None, stream=None):
    """rb_gemv_batch: independent layers of one shape; Xs[j] bf16 [M][K], Ys[j] [M][N] (CUDA tensors)."""
    n = len(layers)
    structs = (RbLayer * n)(*[L.struct() for L in layers])
    lp = (ctypes.POINTER(RbLayer) * n)(*[ctypes.pointer(structs[j]) for j in range(n)])
    xp = (ctypes.c_void_p * n)(*[X.data_ptr() for X in Xs])
    yp = (ctypes.c_void_p * n)(*[Y.data_ptr() for Y in Ys])
    M = Xs[0].shape[0]
    ydt = RB_BF16 if Ys[0].dtype == torch.bfloat16 else RB_F32
    st = lib().rb_gemv_batch(ctypes.cast(lp, ctypes.c_void_p), ctypes.cast(xp, ctypes.c_void_p),
                             ctypes.cast(yp, ctypes.c_void_p), n, M, ydt, _ptr(dev_status), flags, _stream(stream))
    _check("rb_gemv_batch", st)
    return Ys


def gemm(layer: PackedLayer, X, Y=None, ws=None, flags=0, dev_status=None, stream=None, y_dtype=torch.float32):
    """rb_gemm: X bf16 [M][K] -> Y [M][N] (fp32 or bf16) on the tcgen05 tensor cores."""
    if Y is None:
        Y = torch.empty(X.shape[0], layer.n_out, dtype=y_dtype, device=X.device)
    return _apply("rb_gemm", layer, X, Y, ws, flags, dev_status, stream)


def gemm_wait_limit(layer: PackedLayer, X, wait_limit_ns, Y=None, ws=None, flags=0, dev_status=None, stream=None,
                    y_dtype=torch.float32):
    """rb_gemm_wait_limit: rb_gemm with a caller-chosen bound (ns) on every device-side wait."""
    if Y is None:
        Y = torch.empty(X.shape[0], layer.n_out, dtype=y_dtype, device=X.device)
    L = layer.struct()
    ydt = RB_BF16 if Y.dtype == torch.bfloat16 else RB_F32
    wsp, wsb = (None, 0) if ws is None else (_ptr(ws), ws.numel() * ws.element_size())
    st = lib().rb_gemm_wait_limit(ctypes.byref(L), _ptr(X), X.shape[0], _ptr(Y), ydt, wsp, wsb, _ptr(dev_status),
                                  flags, int(wait_limit_ns), _stream(stream))
    _check("rb_gemm_wait_limit", st)
    return Y


def gemm_noalloc(layer: PackedLayer, X, Y=None, flags=0, dev_status=None, stream=None, y_dtype=torch.float32):
    """rb_gemm_noalloc: rb_gemm without a workspace (fixed 32 MiB library scratch; see include/rbw.h)."""
    if Y is None:
        Y = torch.empty(X.shape[0], layer.n_out, dtype=y_dtype, device=X.device)
    L = layer.struct()
    ydt = RB_BF16 if Y.dtype == torch.bfloat16 else RB_F32
    st = lib().rb_gemm_noalloc(ctypes.byref(L), _ptr(X), X.shape[0], _ptr(Y), ydt, _ptr(dev_status), flags,
                               _stream(stream))
    _check("rb_gemm_noalloc", st)
    return Y


def transpose(layer: PackedLayer, out: PackedLayer | None = None, stream=None):
    """rb_transpose_planes: the K x N layer of What^T (new planes, or out's; the
    scale tensors are shared with `layer`, exchanged).  Its forward product is
    the input gradient: gemv/gemm(transpose(layer), dY) = dY . What."""
    if out is None:
        out = PackedLayer(layer.k_in, layer.n_out, layer.k_planes, layer.planes.device, g16=layer.h16, h16=layer.g16)
    elif (out.n_out, out.k_in, out.k_planes) != (layer.k_in, layer.n_out, layer.k_planes):
        raise ValueError("out is not shaped as the transposed layer")
    else:
        out.g16, out.h16 = layer.h16, layer.g16
    L = layer.struct()
    st = lib().rb_transpose_planes(ctypes.byref(L), _ptr(out.planes), _stream(stream))
    _check("rb_transpose_planes", st)
    return out


def rowmajor_words(n_out, k_in, k_planes):
    return int(lib().rb_rowmajor_words(n_out, k_in, k_planes))


def planes_from_rowmajor(rowmajor, n_out, k_in, k_planes, out: PackedLayer | None = None, stream=None):
    """rb_planes_from_rowmajor: plain [k][N][K/32] LSB-first words (int32 CUDA tensor)
    -> a PackedLayer whose planes hold them in the storage layout (scales left to the caller)."""
    out = out or PackedLayer(n_out, k_in, k_planes, rowmajor.device)
    st = lib().rb_planes_from_rowmajor(_ptr(rowmajor), n_out, k_in, k_planes, _ptr(out.planes), _stream(stream))
    _check("rb_planes_from_rowmajor", st)
    return out


def planes_to_rowmajor(layer: PackedLayer, out=None, stream=None):
    """rb_planes_to_rowmajor: the layer's planes as plain [k][N][K/32] LSB-first words (int32)."""
    n = rowmajor_words(layer.n_out, layer.k_in, layer.k_planes)
    out = out if out is not None else torch.empty(n, dtype=torch.int32, device=layer.planes.device)
    st = lib().rb_planes_to_rowmajor(_ptr(layer.planes), layer.n_out, layer.k_in, layer.k_planes, _ptr(out),
                                     _stream(stream))
    _check("rb_planes_to_rowmajor", st)
    return out


def qat_forward_workspace_bytes(n_out, k_in, k_planes, M):
    return int(lib().rb_qat_forward_workspace_bytes(n_out, k_in, k_planes, M))


def qat_forward(W, g, h, k_planes, X, Y=None, ws=None, flags=0, dev_status=None, stream=None,
                y_dtype=torch.float32):
    """rb_qat_forward: Y = X What^T, planes derived from fp32 W into the workspace, fp32 scales (CUDA tensors)."""
    N, K = W.shape
    M = X.shape[0]
    if Y is None:
        Y = torch.empty(M, N, dtype=y_dtype, device=W.device)
    ws = ws if ws is not None else workspace(qat_forward_workspace_bytes(N, K, k_planes, M), W.device)
    ydt = RB_BF16 if Y.dtype == torch.bfloat16 else RB_F32
    st = lib().rb_qat_forward(_ptr(W), _ptr(g), _ptr(h), N, K, k_planes, _ptr(X), M, _ptr(Y), ydt, _ptr(ws),
                              ws.numel(), _ptr(dev_status), flags, _stream(stream))
    _check("rb_qat_forward", st)
    return Y


def qat_backward(layer: PackedLayer, g, h, X, dY, dW=None, dg=None, dh=None, ws=None, dev_status=None,
                 stream=None):
    """rb_qat_backward: (dW [N][K], dg [k][N], dh [k][K]) fp32 from the layer's planes, fp32 scales
    g [k][N], h [k][K], X bf16 [M][K] and dY bf16 [M][N] (CUDA tensors)."""
    N, K, k = layer.n_out, layer.k_in, layer.k_planes
    dev = layer.planes.device
    dW = dW if dW is not None else torch.empty(N, K, dtype=torch.float32, device=dev)
    dg = dg if dg is not None else torch.empty(k, N, dtype=torch.float32, device=dev)
    dh = dh if dh is not None else torch.empty(k, K, dtype=torch.float32, device=dev)
    nb = int(lib().rb_qat_backward_workspace_bytes(N, K, k))
    ws = ws if ws is not None else workspace(nb, dev)
    st = lib().rb_qat_backward(_ptr(layer.planes), _ptr(g), _ptr(h), N, K, k, _ptr(X), _ptr(dY), X.shape[0],
                               _ptr(dW), _ptr(dg), _ptr(dh), _ptr(ws), ws.numel(), _ptr(dev_status), _stream(stream))
    _check("rb_qat_backward", st)
    return dW, dg, dh


def svid_greedy(W, k_planes, iters=20, ws=None, stream=None):
    """rb_svid_greedy: fp32 W [N][K] (CUDA) -> (g [k][N], h [k][K]) fp32."""
    N, K = W.shape
    g = torch.empty(k_planes, N, dtype=torch.float32, device=W.device)
    h = torch.empty(k_planes, K, dtype=torch.float32, device=W.device)
    ws = ws if ws is not None else workspace(svid_workspace_bytes(N, K), W.device)
    st = lib().rb_svid_greedy(_ptr(W), N, K, k_planes, iters, _ptr(g), _ptr(h), _ptr(ws),
                              ws.numel(), _stream(stream))
    _check("rb_svid_greedy", st)
    return g, h


def svid_iterative(W, k_planes, sweeps=20, iters=20, ws=None, stream=None):
    """rb_svid_iterative: greedy scales refined by Gauss-Seidel sweeps; fp32 W [N][K] (CUDA)."""
    N, K = W.shape
    g = torch.empty(k_planes, N, dtype=torch.float32, device=W.device)
    h = torch.empty(k_planes, K, dtype=torch.float32, device=W.device)
    nbytes = int(lib().rb_svid_iterative_workspace_bytes(N, K, k_planes))
    ws = ws if ws is not None else workspace(nbytes, W.device)
    st = lib().rb_svid_iterative(_ptr(W), N, K, k_planes, sweeps, iters, _ptr(g), _ptr(h), _ptr(ws),
                                 ws.numel(), _stream(stream))
    _check("rb_svid_iterative", st)
    return g, h


def svid_pack(W, k_planes, sweeps=0, iters=20, out: PackedLayer | None = None, ws=None, dev_status=None,
              stream=None):
    """rb_svid_pack: fp32 W [N][K] (CUDA) -> (PackedLayer, g, h): SVID scales (greedy when sweeps = 0,
    else iterative) and the packed planes, in one device-side call."""
    N, K = W.shape
    out = out or PackedLayer(N, K, k_planes, W.device)
    g = torch.empty(k_planes, N, dtype=torch.float32, device=W.device)
    h = torch.empty(k_planes, K, dtype=torch.float32, device=W.device)
    nbytes = int(lib().rb_svid_pack_workspace_bytes(N, K, k_planes))
    ws = ws if ws is not None else workspace(nbytes, W.device)
    st = lib().rb_svid_pack(_ptr(W), N, K, k_planes, sweeps, iters, _ptr(g), _ptr(h), _ptr(out.planes),
                            _ptr(out.g16), _ptr(out.h16), _ptr(ws), ws.numel(), _ptr(dev_status), _stream(stream))
    _check("rb_svid_pack", st)
    return out, g, h


def shard_bounds(n_out, world, rank):
    """Rows [row0, row1) of rank `rank` in a row-parallel split of n_out rows over
    `world` ranks: contiguous ranges starting on 32-row tiles, as even as that allows."""
    tiles = (n_out + 31) // 32
    t0, t1 = tiles * rank // world, tiles * (rank + 1) // world
    return min(32 * t0, n_out), min(32 * t1, n_out)


def shard_rows(layer: PackedLayer, row0, rows, stream=None):
    """rb_shard_rows: rows [row0, row0 + rows) of `layer` as a PackedLayer sharing its h16."""
    out = PackedLayer(rows, layer.k_in, layer.k_planes, layer.planes.device, h16=layer.h16)
    L = layer.struct()
    st = lib().rb_shard_rows(ctypes.byref(L), row0, rows, _ptr(out.planes), _ptr(out.g16), _stream(stream))
    _check("rb_shard_rows", st)
    return out


# ---------------------------------------------------------------- binary codebook
class BtcLayer:
    """Device tensors of a binary-codebook layer (owns the codebooks and index streams; shares g16, h16)."""

    def __init__(self, n_out, k_in, k_planes, c_max, g16, h16, device="cuda"):
        self.n_out, self.k_in, self.k_planes, self.c_max = n_out, k_in, k_planes, c_max
        self.index_bits = int(lib().rb_btc_index_bits(c_max))
        self.row_words = int(lib().rb_btc_row_words(k_in, self.index_bits))
        if self.index_bits == 0 or self.row_words == 0:
            raise ValueError("invalid codebook layer shape")
        self.codebooks = torch.zeros(k_planes, c_max, dtype=torch.int16, device=device)
        self.indices = torch.zeros(k_planes, n_out, self.row_words, dtype=torch.int32, device=device)
        self.sizes = torch.zeros(k_planes, 4, dtype=torch.int32, device=device)   # c of each plane in column 0
        self.g16, self.h16 = g16, h16

    def struct(self):
        return RbBtcLayer(self.n_out, self.k_in, self.k_planes, self.c_max, self.index_bits, 0,
                          self.codebooks.data_ptr(), self.indices.data_ptr(), self.g16.data_ptr(),
                          self.h16.data_ptr())

    def index_bytes(self):
        return self.indices.numel() * 4


def btc_encode(layer: PackedLayer, c_max, iters=10, stream=None):
    """rb_btc_encode for every plane of a packed layer -> BtcLayer."""
    out = BtcLayer(layer.n_out, layer.k_in, layer.k_planes, c_max, layer.g16, layer.h16, layer.planes.device)
    ws = workspace(int(lib().rb_btc_encode_workspace_bytes(c_max)), layer.planes.device)
    L = layer.struct()
    for i in range(layer.k_planes):
        st = lib().rb_btc_encode(ctypes.byref(L), i, c_max, iters, _ptr(out.codebooks[i]), _ptr(out.sizes[i]),
                                 _ptr(out.indices[i]), _ptr(ws), ws.numel(), _stream(stream))
        _check("rb_btc_encode", st)
    return out


def btc_gemv(layer: BtcLayer, X, Y=None, ws=None, flags=0, stream=None, y_dtype=torch.float32):
    """rb_btc_gemv: X bf16 [1][K] (or [K]) -> Y [1][N]."""
    if Y is None:
        Y = torch.empty(1, layer.n_out, dtype=y_dtype, device=X.device)
    ws = ws if ws is not None else workspace(int(lib().rb_btc_gemv_workspace_bytes(layer.n_out, layer.k_in)),
                                             X.device)
    L = layer.struct()
    ydt = RB_BF16 if Y.dtype == torch.bfloat16 else RB_F32
    st = lib().rb_btc_gemv(ctypes.byref(L), _ptr(X), _ptr(Y), ydt, _ptr(ws), ws.numel(), None, flags,
                           _stream(stream))
    _check("rb_btc_gemv", st)
    return Y


def btc_gemv_batch(layers, Xs, Ys, ws=None, flags=0, stream=None):
    """rb_btc_gemv_batch: codebook layers of one shape; Xs[j] bf16 [1][K], Ys[j] [1][N] (CUDA tensors)."""
    n = len(layers)
    structs = (RbBtcLayer * n)(*[L.struct() for L in layers])
    lp = (ctypes.POINTER(RbBtcLayer) * n)(*[ctypes.pointer(structs[j]) for j in range(n)])
    xp = (ctypes.c_void_p * n)(*[X.data_ptr() for X in Xs])
    yp = (ctypes.c_void_p * n)(*[Y.data_ptr() for Y in Ys])
    L0 = layers[0]
    ws = ws if ws is not None else workspace(
        int(lib().rb_btc_gemv_batch_workspace_bytes(L0.n_out, L0.k_in, n)), Xs[0].device)
    ydt = RB_BF16 if Ys[0].dtype == torch.bfloat16 else RB_F32
    st = lib().rb_btc_gemv_batch(lp, xp, yp, n, ydt, _ptr(ws), ws.numel(), None, flags, _stream(stream))
    _check("rb_btc_gemv_batch", st)
    return Ys
