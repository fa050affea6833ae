"""rb_pack parity: packed sign planes and fp16 scales bit-exact with the oracle.

Workload layers run at their full sizes (greedy-SVID scales from the oracle);
edge cases cover sign(0) ties (zeros, -0.0, exact cancellation after a
subtraction), ragged tails (N not a multiple of 32, K not a multiple of 256),
one-row / one-word layers, every k from 1 to 8, negative scales, and the
device status bits for non-finite input and fp16 overflow.
"""
import numpy as np
import pytest
import torch

import oracle
from residual_binarized_weight_b200 import rbw, synth
from tests import cases, layout

pytestmark = pytest.mark.gpu


def gpu_pack(W, g, h, k):
    N, K = W.shape
    st = torch.zeros(4, dtype=torch.int32, device="cuda")
    L = rbw.pack(cases.to_dev(W), cases.to_dev(g), cases.to_dev(h), k, dev_status=st)
    torch.cuda.synchronize()
    return (cases.to_host(L.planes, np.uint32), cases.to_host(L.g16, np.uint16).reshape(k, N),
            cases.to_host(L.h16, np.uint16).reshape(k, K), int(st[0].item()))


def assert_pack_equal(W, g, h, k, expect_status=0):
    planes, g16, h16, st, _ = oracle.pack(W, g, h, k)
    gp, gg, gh, gst = gpu_pack(W, g, h, k)
    assert st == expect_status
    assert np.array_equal(gp, planes), "planes differ in %d words" % int((gp != planes).sum())
    assert np.array_equal(gg, g16) and np.array_equal(gh, h16)
    return gst


WORKLOAD_LAYERS = [(0, 0, 1), (1, 0, 2), (2, 0, 2), (2, 2, 2), (3, 0, 1), (3, 0, 2), (4, 0, 2), (4, 1, 2)]


@pytest.mark.parametrize("wl,li,k", WORKLOAD_LAYERS)
def test_pack_workload_layers_full_size(wl, li, k):
    W, g, h = cases.layer_case(wl, li, k)
    assert assert_pack_equal(W, g, h, k) == 0


@pytest.mark.parametrize("N,K,k", [(1, 32, 1), (33, 288, 2), (100, 800, 3), (65, 544, 8),
                                   (31, 256, 5), (7, 1056, 4), (129, 64, 6), (2, 4096, 7)])
def test_pack_ragged_and_all_k(N, K, k):
    rng = np.random.default_rng(N * 7 + K + k)
    W = (rng.standard_normal((N, K)) * 0.02).astype(np.float32)
    g, h = synth.positive_scales(k, N, K, seed=N + K, lo=0.001, hi=0.02)
    assert assert_pack_equal(W, g, h, k) == 0


def test_pack_sign_zero_ties():
    """Zeros, -0.0 and residuals that cancel exactly all take sign +1."""
    N, K, k = 40, 320, 3
    rng = np.random.default_rng(11)
    g, h = synth.positive_scales(k, N, K, seed=5)
    W = (rng.standard_normal((N, K)) * 0.3).astype(np.float32)
    W[rng.random((N, K)) < 0.05] = 0.0
    W[rng.random((N, K)) < 0.05] = -0.0
    # exact cancellation: W = fl(g1*h1) -> R_1 = 0 -> plane 2 sign +1; W = -fl(g1*h1) too
    t1 = (g[0][:, None] * h[0][None, :]).astype(np.float32)
    m = rng.random((N, K)) < 0.05
    W[m] = t1[m]
    m2 = rng.random((N, K)) < 0.05
    W[m2] = -t1[m2]
    assert assert_pack_equal(W, g, h, k) == 0
    planes, *_ = oracle.pack(W, g, h, k)
    B = layout.unpack_bits(planes, N, K, k)
    assert B[1][m & (W > 0)].all()


def test_pack_negative_scales():
    N, K, k = 64, 512, 2
    rng = np.random.default_rng(12)
    W = rng.standard_normal((N, K)).astype(np.float32)
    g = rng.standard_normal((k, N)).astype(np.float32)
    h = rng.standard_normal((k, K)).astype(np.float32)
    assert assert_pack_equal(W, g, h, k) == 0


def test_pack_nonfinite_and_range_status():
    N, K, k = 40, 256, 2
    rng = np.random.default_rng(13)
    W = rng.standard_normal((N, K)).astype(np.float32)
    g, h = synth.positive_scales(k, N, K, seed=1)
    W2 = W.copy()
    W2[3, 7] = np.nan
    W2[39, 255] = np.inf
    *_, st = gpu_pack(W2, g, h, k)
    assert st & rbw.RB_DEV_NONFINITE
    g2 = g.copy()
    g2[1, 5] = 1.0e5
    *_, st = gpu_pack(W, g2, h, k)
    assert st & rbw.RB_DEV_RANGE and not st & rbw.RB_DEV_NONFINITE
    assert oracle.pack(W, g2, h, k)[3] == 2


def test_pack_deterministic_and_overwrites_padding():
    N, K, k = 45, 288, 2
    W, g, h = cases.layer_case(1, 0, 2, N, K)
    L = rbw.PackedLayer(N, K, k)
    L.planes.fill_(-1)                       # garbage in the padding must be overwritten
    rbw.pack(cases.to_dev(W), cases.to_dev(g), cases.to_dev(h), k, out=L)
    a = cases.to_host(L.planes, np.uint32).copy()
    rbw.pack(cases.to_dev(W), cases.to_dev(g), cases.to_dev(h), k, out=L)
    b = cases.to_host(L.planes, np.uint32)
    assert np.array_equal(a, b)
    assert not layout.padding_words_and_bits(a, N, K, k).any()
    assert np.array_equal(a, oracle.pack(W, g, h, k)[0])
