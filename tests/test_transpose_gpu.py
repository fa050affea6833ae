"""rb_transpose_planes and the input gradient dX = dY . What on the GPU.

The transposed planes must equal the oracle's bit for bit (ragged shapes:
row-tile groups and column slices with fewer than 8 members, every k; and the
4096 x 4096 and 4096 x 11008 workload layers).  The input gradient, formed by
the forward kernels on the transposed layer, is checked against the oracle's
float64 dY . What on every decode path (byte tables at M = 1, mma.sync,
tcgen05 with a K split) and on rb_gemm.
"""
import numpy as np
import pytest
import torch

import oracle
from residual_binarized_weight_b200 import rbw, synth
from tests import cases, layout

pytestmark = pytest.mark.gpu


def gpu_transpose(L):
    LT = rbw.transpose(L)
    torch.cuda.synchronize()
    return LT, cases.to_host(LT.planes, np.uint32)


@pytest.mark.parametrize("N,K,k", [(32, 32, 1), (96, 320, 2), (288, 800, 3), (544, 288, 4),
                                   (64, 1056, 1), (256, 2304, 8), (4128, 96, 2)])
def test_transpose_bit_exact_ragged(N, K, k):
    rng = np.random.default_rng(N * 7 + K + k)
    planes = layout.pack_bits(rng.random((k, N, K)) < 0.5)
    g16 = np.zeros((k, N), np.uint16)
    h16 = np.zeros((k, K), np.uint16)
    L = cases.upload_layer(planes, g16, h16, N, K, k)
    LT, pt = gpu_transpose(L)
    assert (LT.n_out, LT.k_in, LT.k_planes) == (K, N, k)
    assert np.array_equal(pt, oracle.transpose_planes(planes, N, K, k))
    _, back = gpu_transpose(LT)                            # K is a multiple of 32: transposable
    assert np.array_equal(back, planes)


@pytest.mark.parametrize("wl,li", [(1, 0), (2, 2)])
def test_transpose_bit_exact_workload_layers(wl, li):
    k = 2
    W, _, _ = cases.layer_case(wl, li, k)
    N, K = W.shape
    planes, g16, h16 = cases.packed_case(wl, li, k)
    L = cases.upload_layer(planes, g16, h16, N, K, k)
    LT, pt = gpu_transpose(L)
    assert np.array_equal(pt, oracle.transpose_planes(planes, N, K, k))
    assert LT.g16.data_ptr() == L.h16.data_ptr() and LT.h16.data_ptr() == L.g16.data_ptr()


def _grad_case(N, K, k, seed):
    rng = np.random.default_rng(seed)
    W = (rng.standard_normal((N, K)) * 0.02).astype(np.float32)
    g, h = oracle.svid_greedy(W, k, iters=8)
    planes, g16, h16, st, _ = oracle.pack(W, g, h, k)
    assert st == 0
    return planes, g16, h16


@pytest.mark.parametrize("N,K,k", [(96, 320, 2), (288, 800, 3), (1024, 2048, 1), (512, 4128, 4)])
@pytest.mark.parametrize("M", [1, 4, 40])
def test_input_gradient_decode_paths(N, K, k, M):
    planes, g16, h16 = _grad_case(N, K, k, N + K + k)
    L = cases.upload_layer(planes, g16, h16, N, K, k)
    LT = rbw.transpose(L)
    dY = synth.activations(M, N, seed=M + 3)
    ws = rbw.workspace(rbw.gemv_workspace_bytes(K, N, k, M))
    dX = rbw.gemv(LT, cases.to_dev(dY), ws=ws)
    torch.cuda.synchronize()
    dXg = dX.cpu().numpy().astype(np.float64)
    ref = oracle.apply_t(planes, g16, h16, N, K, k, dY)
    bound = cases.abs_bound(h16, g16, dY)                  # sum_i |h_i[c]| sum_n |g_i[n] dY[m][n]|
    cases.check_y(dXg, ref, bound, bf16=False, per_elem=1e-5 if (M == 1 and k <= 4) else 1e-4)


@pytest.mark.parametrize("N,K,k,M", [(96, 320, 2, 300), (1024, 2048, 2, 130), (4096, 4096, 2, 48)])
@pytest.mark.parametrize("ydt", [torch.float32, torch.bfloat16])
def test_input_gradient_gemm(N, K, k, M, ydt):
    if (N, K) == (4096, 4096):
        planes, g16, h16 = cases.packed_case(1, 0, k)
    else:
        planes, g16, h16 = _grad_case(N, K, k, 3 * N + K)
    L = cases.upload_layer(planes, g16, h16, N, K, k)
    LT = rbw.transpose(L)
    dY = synth.activations(M, N, seed=M)
    ws = rbw.workspace(rbw.gemm_workspace_bytes(K, N, k, M))
    st = torch.zeros(4, dtype=torch.int32, device="cuda")
    dX = rbw.gemm(LT, cases.to_dev(dY), ws=ws, y_dtype=ydt, dev_status=st)
    torch.cuda.synchronize()
    assert int(st[0].item()) == 0
    ref = oracle.apply_t(planes, g16, h16, N, K, k, dY)
    bound = cases.abs_bound(h16, g16, dY)
    cases.check_y(dX.float().cpu().numpy().astype(np.float64), ref, bound,
                  bf16=ydt == torch.bfloat16, per_elem=1e-4)
