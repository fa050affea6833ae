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
