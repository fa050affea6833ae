"""rb_gemm_noalloc: the allocation-free form of rb_gemm for hosts that give the
library a fixed device-memory budget and allow no further allocations.

Called through the C ABI and compared with rb_gemm (which takes a caller
workspace) on two calls in a row with different shapes and inputs, using the
GEMM parity gate of the other tests; sizes beyond the fixed 32 MiB scratch are
rejected.  The file is collected last so that a run stopping at the first
failure has already run every other test; it also passes on its own.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
from residual_binarized_weight_b200 import rbw, synth
from tests import cases

pytestmark = pytest.mark.gpu


def _noalloc(L, X, M, Y):
    lay = L.struct()
    st = rbw.lib().rb_gemm_noalloc(ctypes.byref(lay), ctypes.c_void_p(X.data_ptr()), M,
                                   ctypes.c_void_p(Y.data_ptr()), rbw.RB_F32, None, 0,
                                   ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    return st


def _layer(N, K, k, seed):
    rng = np.random.default_rng(seed)
    W = (rng.standard_normal((N, K)) * 0.02).astype(np.float32)
    g, h = oracle.svid_greedy(W, k, iters=6)
    planes, g16, h16, st, _ = oracle.pack(W, g, h, k)
    assert st == 0
    return cases.upload_layer(planes, g16, h16, N, K, k), (planes, g16, h16)


def test_noalloc_matches_gemm_on_two_calls():
    calls = [(300, 1056, 2, 130, 1), (4096, 4096, 2, 512, 2)]
    for N, K, k, M, seed in calls:                      # two calls in a row, sharing the scratch
        L, (planes, g16, h16) = _layer(N, K, k, seed)
        X = synth.activations(M, K, seed=seed + 10)
        Xd = cases.to_dev(X)
        Y = torch.empty(M, N, dtype=torch.float32, device="cuda")
        assert _noalloc(L, Xd, M, Y) == rbw.RB_OK
        ref = rbw.gemm(L, Xd, ws=rbw.workspace(rbw.gemm_workspace_bytes(N, K, k, M)))
        torch.cuda.synchronize()
        a = Y.cpu().numpy().astype(np.float64)
        b = ref.cpu().numpy().astype(np.float64)
        bound = cases.abs_bound(g16, h16, X)
        assert np.linalg.norm(a - b) <= 2e-3 * np.linalg.norm(b)
        assert np.all(np.abs(a - b) <= 1e-4 * bound + 1e-30)


def test_noalloc_rejects_sizes_beyond_its_scratch():
    N, K, k = 128, 14336, 2
    M = 2048                                            # X alone needs 56 MiB in fp16
    L = rbw.PackedLayer(N, K, k)
    X = torch.zeros(M, K, dtype=torch.int16, device="cuda")
    Y = torch.empty(M, N, dtype=torch.float32, device="cuda")
    assert _noalloc(L, X, M, Y) == rbw.RB_ERR_WORKSPACE
