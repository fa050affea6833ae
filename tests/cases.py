"""Shared test inputs: seeded workload layers with oracle-derived scales.

Only the oracle and the seeded generator produce these values; nothing here
comes from the CUDA library.  Results are memoised per test session.
"""
import functools

import numpy as np
import torch

import oracle
from residual_binarized_weight_b200 import synth


@functools.lru_cache(maxsize=None)
def layer_case(wl_index: int, layer_index: int, k: int, n_out=None, k_in=None):
    """(W fp32, g fp32 [k][N], h fp32 [k][K]) with greedy-SVID scales (20 iterations)."""
    wl = synth.workload(wl_index)
    W = synth.weights(wl.layers[layer_index], n_out, k_in)
    g, h = oracle.svid_greedy(W, k, iters=20)
    return W, g, h


@functools.lru_cache(maxsize=None)
def packed_case(wl_index: int, layer_index: int, k: int, n_out=None, k_in=None):
    W, g, h = layer_case(wl_index, layer_index, k, n_out, k_in)
    planes, g16, h16, st, _ = oracle.pack(W, g, h, k)
    assert st == 0
    return planes, g16, h16


def abs_bound(g16, h16, X_bf16, rows=None):
    """sum_i |g_i[r]| * sum_c |h_i[c] x_m[c]| per (token, row): scale of the fp32 error bound."""
    gq = np.abs(g16.view(np.float16).astype(np.float64))
    hq = np.abs(h16.view(np.float16).astype(np.float64))
    xq = np.abs(bf16_to_f64(X_bf16))
    hx = xq @ hq.T                                   # [M][k]
    if rows is not None:
        gq = gq[:, rows]
    return hx @ gq                                   # [M][rows]


def bf16_to_f64(bits):
    return torch.from_numpy(np.ascontiguousarray(bits, np.uint16).view(np.int16)).view(torch.bfloat16).double().numpy()


def to_dev(a: np.ndarray) -> torch.Tensor:
    a = np.ascontiguousarray(a)
    if a.dtype == np.uint32:
        a = a.view(np.int32)
    elif a.dtype == np.uint16:
        a = a.view(np.int16)
    return torch.from_numpy(a).cuda()


def to_host(t: torch.Tensor, dtype) -> np.ndarray:
    return t.detach().cpu().contiguous().numpy().view(dtype)


def upload_layer(planes, g16, h16, N, K, k):
    from residual_binarized_weight_b200 import rbw
    L = rbw.PackedLayer(N, K, k)
    L.planes.copy_(to_dev(planes))
    L.g16.copy_(to_dev(g16.reshape(k, N)).view(torch.float16))
    L.h16.copy_(to_dev(h16.reshape(k, K)).view(torch.float16))
    return L


def check_y(Y_gpu: np.ndarray, Y_ref: np.ndarray, bound: np.ndarray, bf16: bool, per_elem=1e-5):
    """Relative Frobenius error <= 2e-3 against the float64 oracle, plus a per-element
    gate: fp32 output within per_elem * sum|g h x| of the oracle; bf16 output
    within one bf16 step of the oracle value rounded to bf16."""
    num = np.linalg.norm(Y_gpu - Y_ref)
    den = np.linalg.norm(Y_ref)
    rel = num / den if den > 0 else num
    assert rel <= 2e-3, "relative Frobenius error %.3e" % rel
    if not bf16:
        err = np.abs(Y_gpu - Y_ref)
        lim = per_elem * bound + 1e-30
        bad = err > lim
        assert not bad.any(), "per-element: %d bad, worst ratio %.3g" % (bad.sum(), float((err / lim).max()))
    else:
        # bf16 output: one bf16 step of the exact value (the final rounding) plus the
        # fp32 accumulation error before it, per_elem * sum|g h x|.
        a = np.abs(Y_ref)
        ulp = np.where(a > 0, np.exp2(np.floor(np.log2(np.where(a > 0, a, 1.0))) - 7), 2.0 ** -133)
        err = np.abs(np.asarray(Y_gpu, np.float64) - Y_ref)
        lim = ulp + per_elem * bound
        bad = err > lim
        assert not bad.any(), "bf16 per-element: %d bad, worst ratio %.3g" % (bad.sum(), float((err / lim).max()))
    return rel
