"""rb_svid_greedy (device greedy SVID scales) against the oracle's float64 power
iteration.  Both run the same algorithm in float64 with different summation
orders, so the fp32 scales agree to a few ulps."""
import numpy as np
import pytest
import torch

import oracle
from residual_binarized_weight_b200 import rbw, synth
from tests import cases

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("wl,k,shape", [(0, 1, None), (1, 2, (512, 1024)), (1, 2, None), (4, 3, (300, 544))])
def test_svid_matches_oracle(wl, k, shape):
    layer = synth.workload(wl).layers[0]
    W = synth.weights(layer, *(shape or (None, None)))
    g_ref, h_ref = oracle.svid_greedy(W, k, iters=20)
    g, h = rbw.svid_greedy(cases.to_dev(W), k, iters=20)
    torch.cuda.synchronize()
    g, h = g.cpu().numpy(), h.cpu().numpy()
    for a, b in ((g, g_ref), (h, h_ref)):
        err = np.abs(a.astype(np.float64) - b) / np.maximum(np.abs(b).max(axis=1, keepdims=True), 1e-30)
        assert err.max() < 1e-5, err.max()
    assert (g >= 0).all() and (h >= 0).all()


def test_svid_zero_matrix():
    W = np.zeros((64, 256), np.float32)
    g, h = rbw.svid_greedy(cases.to_dev(W), 2)
    torch.cuda.synchronize()
    assert not g.any() and not h.any()


@pytest.mark.parametrize("wl,k,sweeps,shape", [(1, 2, 3, (256, 512)), (2, 2, 5, (512, 1024)), (4, 3, 2, (300, 544)),
                                               (0, 1, 4, None), (1, 2, 0, (128, 256))])
def test_svid_iterative_matches_oracle(wl, k, sweeps, shape):
    """rb_svid_iterative against the oracle's Gauss-Seidel sweeps: the signs are
    decided in float64 with the same operation order on both sides, the power
    iterations differ only in summation order."""
    layer = synth.workload(wl).layers[0]
    W = synth.weights(layer, *(shape or (None, None)))
    g_ref, h_ref = oracle.svid_iterative(W, k, sweeps=sweeps, iters=20)
    g, h = rbw.svid_iterative(cases.to_dev(W), k, sweeps=sweeps, iters=20)
    torch.cuda.synchronize()
    g, h = g.cpu().numpy(), h.cpu().numpy()
    for a, b in ((g, g_ref), (h, h_ref)):
        err = np.abs(a.astype(np.float64) - b) / np.maximum(np.abs(b).max(axis=1, keepdims=True), 1e-30)
        assert err.max() < 1e-5, err.max()
    assert (g >= 0).all() and (h >= 0).all()
    if sweeps == 0:                                       # the greedy pass itself
        g0, h0 = rbw.svid_greedy(cases.to_dev(W), k, iters=20)
        torch.cuda.synchronize()
        assert np.array_equal(g, g0.cpu().numpy()) and np.array_equal(h, h0.cpu().numpy())


def test_svid_iterative_lowers_the_packed_error():
    """The refined scales, packed by rb_pack's recurrence, reconstruct W at least
    as well as the greedy ones (the iteration's purpose)."""
    W = synth.weights(synth.workload(1).layers[0], 512, 1024)
    Wd = cases.to_dev(W)
    errs = []
    for g, h in (rbw.svid_greedy(Wd, 2), rbw.svid_iterative(Wd, 2, sweeps=10)):
        torch.cuda.synchronize()
        gn, hn = g.cpu().numpy(), h.cpu().numpy()
        planes, g16, h16, _, _ = oracle.pack(W, gn, hn, 2)
        eye = np.eye(1024, dtype=np.float32)
        What = oracle.apply(planes, g16, h16, 512, 1024, 2, synth.to_bf16_bits(eye))   # rows of What^T
        errs.append(np.linalg.norm(W.astype(np.float64) - What.T))
    assert errs[1] <= errs[0] * 1.001, errs


@pytest.mark.parametrize("wl,k,sweeps,shape", [(1, 2, 0, (512, 1024)), (1, 2, 3, (256, 512)), (4, 3, 0, (300, 544)),
                                               (2, 2, 0, None)])
def test_svid_pack_one_call(wl, k, sweeps, shape):
    """rb_svid_pack (SVID scales then the residual sign planes, one device-side
    call): the scales agree with the oracle's SVID, and the planes and fp16
    scales are bit-exact with the oracle's packer run on those scales."""
    layer = synth.workload(wl).layers[0]
    W = synth.weights(layer, *(shape or (None, None)))
    N, K = W.shape
    if sweeps:
        g_ref, h_ref = oracle.svid_iterative(W, k, sweeps=sweeps, iters=20)
    else:
        g_ref, h_ref = oracle.svid_greedy(W, k, iters=20)
    st = torch.zeros(4, dtype=torch.int32, device="cuda")
    L, g, h = rbw.svid_pack(cases.to_dev(W), k, sweeps=sweeps, iters=20, dev_status=st)
    torch.cuda.synchronize()
    assert int(st[0].item()) == 0
    g, h = g.cpu().numpy(), h.cpu().numpy()
    for a, b in ((g, g_ref), (h, h_ref)):
        err = np.abs(a.astype(np.float64) - b) / np.maximum(np.abs(b).max(axis=1, keepdims=True), 1e-30)
        assert err.max() < 1e-5, err.max()
    planes, g16, h16, st2, _ = oracle.pack(W, g, h, k)
    assert st2 == 0
    assert np.array_equal(cases.to_host(L.planes, np.uint32), planes)
    assert np.array_equal(cases.to_host(L.g16, np.uint16).reshape(k, N), g16)
    assert np.array_equal(cases.to_host(L.h16, np.uint16).reshape(k, K), h16)
