"""CPU oracle for the residual dual-scale binarized linear layer.

TEST INFRASTRUCTURE ONLY.  Only the test-suite, the smoke check and the
benchmark's CPU-baseline leg may import this package.  The product path (the
CUDA library and its binding) never imports it, and this package imports
nothing from the product.

The arithmetic lives in ``rb_oracle.c`` (plain C, fp32-exact derivation and
packing, float64 application, float64 greedy SVID).  This module only builds
that file with gcc and marshals numpy arrays through ctypes.

Method: RaBiT (Residual-Aware Binarization Training), "Residual binarization"
section (W ~= sum_i g_i . B_i . h_i with B_i in {-1,+1}) and Algorithm 2's
forward pass (B_i = sign(R_{i-1}), R_i = R_{i-1} - g_i . B_i . h_i).
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "rb_oracle.c")
_LIB = os.path.join(_HERE, "librb_oracle.so")
_CFLAGS = ["-O2", "-ffp-contract=off", "-fno-fast-math", "-fopenmp", "-shared", "-fPIC"]

_lib = None


def build(force: bool = False) -> str:
    """Compile rb_oracle.c into librb_oracle.so next to it (gcc, no fast-math)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + ".tmp%d" % os.getpid()
        subprocess.check_call(["gcc", *_CFLAGS, "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        i64, i32, vp, dbl = ctypes.c_int64, ctypes.c_int, ctypes.c_void_p, ctypes.c_double
        lib.oracle_pack.argtypes = [vp, vp, vp, i64, i64, i32, vp, vp, vp, vp]
        lib.oracle_pack.restype = i32
        lib.oracle_pack_rows.argtypes = [vp, vp, vp, i64, i64, i32, vp, i64, vp]
        lib.oracle_pack_rows.restype = i32
        lib.oracle_apply.argtypes = [vp, vp, vp, i64, i64, i32, vp, i64, vp, i64, vp, i64, vp]
        lib.oracle_apply.restype = None
        lib.oracle_qat_backward.argtypes = [vp, vp, vp, i64, i64, i32, vp, vp, i64, vp, vp, vp, vp]
        lib.oracle_qat_backward.restype = i32
        lib.oracle_qat_forward.argtypes = [vp, vp, vp, i64, i64, i32, vp, i64, vp, i64, vp, i64, vp]
        lib.oracle_qat_forward.restype = i32
        lib.oracle_set_threads.argtypes = [i32]
        lib.oracle_set_threads.restype = None
        lib.oracle_threads.argtypes = []
        lib.oracle_threads.restype = i32
        lib.oracle_transpose_planes.argtypes = [vp, i64, i64, i32, vp]
        lib.oracle_transpose_planes.restype = None
        lib.oracle_apply_t.argtypes = [vp, vp, vp, i64, i64, i32, vp, i64, vp]
        lib.oracle_apply_t.restype = None
        lib.oracle_svid_greedy.argtypes = [vp, i64, i64, i32, i32, vp, vp]
        lib.oracle_svid_greedy.restype = i32
        lib.oracle_svid_iterative.argtypes = [vp, i64, i64, i32, i32, i32, vp, vp]
        lib.oracle_svid_iterative.restype = i32
        lib.oracle_plane_words.argtypes = [i64, i64, i32]
        lib.oracle_plane_words.restype = i64
        lib.oracle_btc_index_bits.argtypes = [i32]
        lib.oracle_btc_index_bits.restype = i32
        lib.oracle_btc_row_words.argtypes = [i64, i32]
        lib.oracle_btc_row_words.restype = i64
        lib.oracle_btc_patterns.argtypes = [vp, i64, i64, i32, i32, vp]
        lib.oracle_btc_patterns.restype = None
        lib.oracle_btc_encode.argtypes = [vp, i64, i64, i32, i32, i32, i32, vp, vp, vp, vp]
        lib.oracle_btc_encode.restype = i32
        lib.oracle_btc_pack_indices.argtypes = [vp, i64, i64, i32, vp]
        lib.oracle_btc_pack_indices.restype = None
        lib.oracle_btc_apply.argtypes = [vp, i32, vp, vp, vp, i64, i64, i32, vp, i64, vp, i64, vp]
        lib.oracle_btc_apply.restype = None
        lib.oracle_f64_to_f16.argtypes = [dbl]
        lib.oracle_f64_to_f16.restype = ctypes.c_uint16
        lib.oracle_f16_to_f64.argtypes = [ctypes.c_uint16]
        lib.oracle_f16_to_f64.restype = dbl
        lib.oracle_f64_to_bf16.argtypes = [dbl]
        lib.oracle_f64_to_bf16.restype = ctypes.c_uint16
        lib.oracle_bf16_to_f64.argtypes = [ctypes.c_uint16]
        lib.oracle_bf16_to_f64.restype = dbl
        _lib = lib
    return _lib


def _p(a: np.ndarray | None):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


def threads() -> int:
    """OpenMP threads the oracle's parallel loops use."""
    return int(_load().oracle_threads())


def set_threads(n: int) -> None:
    """Thread count of the oracle's later parallel loops (from this thread)."""
    _load().oracle_set_threads(int(n))


def plane_words(N: int, K: int, k: int) -> int:
    """Number of uint32 words of the packed sign planes (layout in rb_oracle.c)."""
    return int(_load().oracle_plane_words(N, K, k))


class PackStatusError(RuntimeError):
    pass


def pack(W, g, h, k: int, want_residual: bool = False):
    """Derive and pack k sign planes (Algorithm 2 forward, fp32 recurrence).

    W float32 [N][K]; g float32 [k][N]; h float32 [k][K].
    Returns (planes uint32 [plane_words], g16 uint16 [k][N], h16 uint16 [k][K],
    status, R_k float32 [N][K] or None).  status: 0 ok, 1 non-finite input,
    2 a scale overflows fp16, -1 bad arguments.
    """
    W = _c(W, np.float32)
    N, K = W.shape
    g = _c(g, np.float32).reshape(k, N)
    h = _c(h, np.float32).reshape(k, K)
    lib = _load()
    nw = lib.oracle_plane_words(N, K, k) if K % 32 == 0 and K >= 32 and 1 <= k <= 8 else 0
    planes = np.zeros(max(nw, 1), np.uint32)
    g16 = np.zeros((k, N), np.uint16)
    h16 = np.zeros((k, K), np.uint16)
    R = np.zeros((N, K), np.float32) if want_residual else None
    st = lib.oracle_pack(_p(W), _p(g), _p(h), N, K, k, _p(planes), _p(g16), _p(h16), _p(R))
    return planes[:nw], g16, h16, int(st), R


def pack_rows(W, g, h, k: int, rows):
    """Pack only `rows`; returns uint32 [len(rows)][k][ceil(K/256)][8] (row-local order)."""
    W = _c(W, np.float32)
    N, K = W.shape
    g = _c(g, np.float32).reshape(k, N)
    h = _c(h, np.float32).reshape(k, K)
    rows = _c(rows, np.int64)
    S = (K + 255) // 256
    out = np.zeros((len(rows), k, S, 8), np.uint32)
    st = _load().oracle_pack_rows(_p(W), _p(g), _p(h), N, K, k, _p(rows), len(rows), _p(out))
    if st != 0:
        raise PackStatusError("oracle_pack_rows status %d" % st)
    return out


def apply(planes, g16, h16, N: int, K: int, k: int, X_bf16, rows=None, toks=None):
    """float64 Y = X . What^T from the stored representation.

    X_bf16 uint16 [M][K] (bfloat16 bit patterns). rows / toks optionally select
    output rows n and tokens m; the result is float64 [len(toks)][len(rows)].
    """
    planes = _c(planes, np.uint32)
    g16 = _c(g16, np.uint16)
    h16 = _c(h16, np.uint16)
    X = _c(X_bf16, np.uint16)
    M = X.shape[0]
    rows_a = None if rows is None else _c(rows, np.int64)
    toks_a = None if toks is None else _c(toks, np.int64)
    nr = N if rows_a is None else len(rows_a)
    nt = M if toks_a is None else len(toks_a)
    Y = np.zeros((nt, nr), np.float64)
    _load().oracle_apply(_p(planes), _p(g16), _p(h16), N, K, k, _p(X), M,
                         _p(rows_a), nr, _p(toks_a), nt, _p(Y))
    return Y


def transpose_planes(planes, N: int, K: int, k: int):
    """Sign planes of the transposed (K x N) layer in the same storage layout.

    The transposed layer's scales are the original ones exchanged (g' = h16,
    h' = g16).  Returns uint32 [plane_words(K, N, k)].
    """
    planes = _c(planes, np.uint32)
    out = np.zeros(max(plane_words(K, N, k), 1), np.uint32)
    _load().oracle_transpose_planes(_p(planes), N, K, k, _p(out))
    return out[:plane_words(K, N, k)]


def apply_t(planes, g16, h16, N: int, K: int, k: int, dY_bf16):
    """float64 input gradient dX = dY . What (dY bfloat16 bits [M][N]) -> [M][K]."""
    planes = _c(planes, np.uint32)
    g16 = _c(g16, np.uint16)
    h16 = _c(h16, np.uint16)
    dY = _c(dY_bf16, np.uint16)
    M = dY.shape[0]
    dX = np.zeros((M, K), np.float64)
    _load().oracle_apply_t(_p(planes), _p(g16), _p(h16), N, K, k, _p(dY), M, _p(dX))
    return dX


def qat_backward(W, g, h, k: int, X_bf16, dY_bf16):
    """float64 gradients of the coupled-training layer (signs derived from W by
    the fp32 recurrence and held constant): returns (status, dW [N][K],
    dg [k][N], dh [k][K], dX [M][K])."""
    W = _c(W, np.float32)
    N, K = W.shape
    g = _c(g, np.float32).reshape(k, N)
    h = _c(h, np.float32).reshape(k, K)
    X = _c(X_bf16, np.uint16)
    dY = _c(dY_bf16, np.uint16)
    M = X.shape[0]
    assert dY.shape == (M, N)
    dW = np.zeros((N, K), np.float64)
    dg = np.zeros((k, N), np.float64)
    dh = np.zeros((k, K), np.float64)
    dX = np.zeros((M, K), np.float64)
    st = _load().oracle_qat_backward(_p(W), _p(g), _p(h), N, K, k, _p(X), _p(dY), M,
                                     _p(dW), _p(dg), _p(dh), _p(dX))
    return int(st), dW, dg, dh, dX


def qat_forward(W, g, h, k: int, X_bf16, rows=None, toks=None):
    """float64 forward of the coupled-training layer: signs derived from W by the
    fp32 recurrence, fp32 scales; returns (status, Y [len(toks)][len(rows)])."""
    W = _c(W, np.float32)
    N, K = W.shape
    g = _c(g, np.float32).reshape(k, N)
    h = _c(h, np.float32).reshape(k, K)
    X = _c(X_bf16, np.uint16)
    M = X.shape[0]
    rows_a = None if rows is None else _c(rows, np.int64)
    toks_a = None if toks is None else _c(toks, np.int64)
    nr = N if rows_a is None else len(rows_a)
    nt = M if toks_a is None else len(toks_a)
    Y = np.zeros((nt, nr), np.float64)
    st = _load().oracle_qat_forward(_p(W), _p(g), _p(h), N, K, k, _p(X), M, _p(rows_a), nr, _p(toks_a), nt, _p(Y))
    return int(st), Y


def svid_greedy(W, k: int, iters: int = 20):
    """Greedy SVID scales: per plane the rank-1 of |R_{i-1}| by power iteration (fp64)."""
    W = _c(W, np.float32)
    N, K = W.shape
    g = np.zeros((k, N), np.float32)
    h = np.zeros((k, K), np.float32)
    st = _load().oracle_svid_greedy(_p(W), N, K, k, iters, _p(g), _p(h))
    if st != 0:
        raise ValueError("oracle_svid_greedy: bad arguments")
    return g, h


def svid_iterative(W, k: int, sweeps: int = 20, iters: int = 20):
    """Iterative residual SVID (Gauss-Seidel sweeps from the greedy scales), float64."""
    W = _c(W, np.float32)
    N, K = W.shape
    g = np.zeros((k, N), np.float32)
    h = np.zeros((k, K), np.float32)
    st = _load().oracle_svid_iterative(_p(W), N, K, k, sweeps, iters, _p(g), _p(h))
    if st != 0:
        raise ValueError("oracle_svid_iterative: bad arguments")
    return g, h


def f64_to_f16_bits(v: float) -> int:
    return int(_load().oracle_f64_to_f16(float(v)))


def f16_bits_to_f64(b: int) -> float:
    return float(_load().oracle_f16_to_f64(int(b)))


def f64_to_bf16_bits(v: float) -> int:
    return int(_load().oracle_f64_to_bf16(float(v)))


def bf16_bits_to_f64(b: int) -> float:
    return float(_load().oracle_bf16_to_f64(int(b)))


def f64_array_to_bf16_bits(a) -> np.ndarray:
    """Round each float64 to bfloat16 (nearest-even) with the oracle's encoder."""
    a = np.asarray(a, np.float64)
    lib = _load()
    out = np.fromiter((lib.oracle_f64_to_bf16(float(x)) for x in a.ravel()), np.uint16, a.size)
    return out.reshape(a.shape)


# ---------------------------------------------------------------- binary codebook (BTC-LLM)
def btc_index_bits(c_max: int) -> int:
    """Bits per stored index: ceil(log2 c_max), at least 1."""
    return int(_load().oracle_btc_index_bits(c_max))


def btc_row_words(K: int, w: int) -> int:
    return int(_load().oracle_btc_row_words(K, w))


def btc_patterns(planes, N: int, K: int, k: int, i: int):
    """uint16 [N][K/16]: the 16-column sign patterns of plane i (bit q = column 16j+q is +1)."""
    pat = np.zeros((N, K // 16), np.uint16)
    _load().oracle_btc_patterns(_p(_c(planes, np.uint32)), N, K, k, i, _p(pat))
    return pat


def btc_encode(planes, N: int, K: int, k: int, i: int, c_max: int, iters: int):
    """Binary k-means codebook of plane i: (codebook uint16 [c_max], c, idx uint16 [N][K/16],
    objective float64 [iters + 1])."""
    cb = np.zeros(c_max, np.uint16)
    idx = np.zeros((N, K // 16), np.uint16)
    obj = np.zeros(iters + 1, np.float64)
    c = ctypes.c_int(0)
    st = _load().oracle_btc_encode(_p(_c(planes, np.uint32)), N, K, k, i, c_max, iters, _p(cb),
                                   ctypes.byref(c), _p(idx), _p(obj))
    if st != 0:
        raise ValueError("oracle_btc_encode: bad arguments")
    return cb, int(c.value), idx, obj


def btc_pack_indices(idx, N: int, K: int, w: int):
    """uint32 [N][row_words]: index j of row r at bits [j w, j w + w) of the row's stream."""
    words = np.zeros((N, btc_row_words(K, w)), np.uint32)
    _load().oracle_btc_pack_indices(_p(_c(idx, np.uint16)), N, K, w, _p(words))
    return words


def btc_apply(codebooks, c_max: int, idx, g16, h16, N: int, K: int, k: int, X_bf16, rows=None):
    """float64 Y [M][len(rows)] of the codebook-reconstructed layer; codebooks [k][c_max],
    idx [k][N][K/16] plain indices."""
    X = _c(X_bf16, np.uint16)
    M = X.shape[0]
    rows_a = None if rows is None else _c(rows, np.int64)
    nr = N if rows_a is None else len(rows_a)
    Y = np.zeros((M, nr), np.float64)
    _load().oracle_btc_apply(_p(_c(codebooks, np.uint16)), c_max, _p(_c(idx, np.uint16)), _p(_c(g16, np.uint16)),
                             _p(_c(h16, np.uint16)), N, K, k, _p(X), M, _p(rows_a), nr, _p(Y))
    return Y
