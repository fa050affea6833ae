"""rb_qat_backward (RaBiT, Algorithm 2 backward pass) against the float64
oracle's coupled-training gradients (oracle.qat_backward, pinned by exact
central differences): the latent-weight gradient G = dY^T X on the tcgen05
tensor cores, and the scale gradients dg, dh.

Tolerances, from the arithmetic: G's products are exact (bf16 x bf16 in fp32)
and only the fp32 accumulation over M tokens rounds, so |G - G_ref| <=
M * 2^-23 * sum_m |dY x| (taken with a factor 2); dg and dh add one fp32
summation over K (resp. N) terms of |G h| (|G g|), bounded the same way.
"""
import numpy as np
import pytest
import torch

import oracle
from residual_binarized_weight_b200 import rbw, synth
from tests import cases

pytestmark = pytest.mark.gpu

EPS = 2.0 ** -23


def bf16(a):
    return cases.bf16_to_f64(a)


def signs(planes, N, K, k, rows, cols):
    """+-1 float64 [k][len(rows)][len(cols)] read from packed planes with the
    storage-layout formula (test-side restatement, numpy only)."""
    S, Nt = (K + 255) // 256, (N + 31) // 32
    r = np.asarray(rows, np.int64)[:, None]
    c = np.asarray(cols, np.int64)[None, :]
    out = np.empty((k, r.shape[0], c.shape[1]))
    for i in range(k):
        w = (c % 256) // 32
        idx = ((i * S + c // 256) * Nt + r // 32) * 256 + (w ^ ((r % 32) // 4)) * 32 + r % 32
        out[i] = np.where((planes[idx] >> (c % 32).astype(np.uint32)) & 1, 1.0, -1.0)
    return out


@pytest.mark.parametrize("N,K,k,M", [(128, 256, 1, 64), (256, 512, 2, 100), (96, 800, 3, 33), (4096, 1024, 2, 256),
                                     (160, 4096, 4, 1), (64, 288, 8, 77), (1024, 2048, 2, 300)])
def test_qat_backward_matches_oracle(N, K, k, M):
    rng = np.random.default_rng(N + K + k + M)
    W = (rng.standard_normal((N, K)) * 0.02).astype(np.float32)
    g, h = oracle.svid_greedy(W, k, iters=6)
    X = synth.activations(M, K, seed=M + 1)
    dY = synth.activations(M, N, seed=M + 2)
    st, dW_r, dg_r, dh_r, _ = oracle.qat_backward(W, g, h, k, X, dY)
    assert st == 0
    planes, g16, h16, _, _ = oracle.pack(W, g, h, k)
    L = cases.upload_layer(planes, g16, h16, N, K, k)
    s = torch.zeros(4, dtype=torch.int32, device="cuda")
    dW, dg, dh = rbw.qat_backward(L, cases.to_dev(g), cases.to_dev(h), cases.to_dev(X), cases.to_dev(dY), dev_status=s)
    torch.cuda.synchronize()
    assert int(s[0].item()) == 0
    dW = dW.cpu().numpy().astype(np.float64)
    aG = np.abs(bf16(dY)).T @ np.abs(bf16(X))                     # sum_m |dY x| per element
    tolG = 2 * (M + 2) * EPS * aG + 1e-30
    assert np.all(np.abs(dW - dW_r) <= tolG), "G: worst %.3g" % float((np.abs(dW - dW_r) / tolG).max())
    # dg_i[n] = sum_c G B h: bound = G's error carried through plus the fp32 sum over K
    ah = np.abs(h.astype(np.float64))
    ag = np.abs(g.astype(np.float64))
    tol_g = (tolG @ ah.T).T + 2 * (K + 2) * EPS * (np.abs(dW_r) @ ah.T).T + 1e-30
    tol_h = ag @ tolG + 2 * (N + 2) * EPS * (ag @ np.abs(dW_r)) + 1e-30
    dg = dg.cpu().numpy().astype(np.float64)
    dh = dh.cpu().numpy().astype(np.float64)
    assert np.all(np.abs(dg - dg_r) <= tol_g), "dg: worst %.3g" % float((np.abs(dg - dg_r) / tol_g).max())
    assert np.all(np.abs(dh - dh_r) <= tol_h), "dh: worst %.3g" % float((np.abs(dh - dh_r) / tol_h).max())


def test_qat_backward_prefill_shape_sampled():
    """The prefill workload's up layer (14336 x 4096, k = 2, Laplace(0, 0.01)
    weights, M = 512 tokens with 1% heavy columns): G checked on sampled rows
    (numpy float64 dY[:, rows]^T X), dg on those rows and dh on sampled columns
    through the oracle's own sign planes."""
    wl = synth.workload(4)
    layer = wl.layers[0]
    W, g, h = cases.layer_case(4, 0, 2)
    N, K, k, M = W.shape[0], W.shape[1], 2, 512
    X = synth.activations_for(wl, M, K)
    dY = synth.activations(M, N, seed=77)
    planes, g16, h16 = cases.packed_case(4, 0, 2)
    L = cases.upload_layer(planes, g16, h16, N, K, k)
    dW, dg, dh = rbw.qat_backward(L, cases.to_dev(g), cases.to_dev(h), cases.to_dev(X), cases.to_dev(dY))
    torch.cuda.synchronize()
    rng = np.random.default_rng(5)
    rows = np.unique(np.concatenate([np.arange(32), np.arange(N - 32, N), rng.choice(N, 96, replace=False)]))
    cols = np.unique(np.concatenate([np.arange(16), np.arange(K - 16, K), rng.choice(K, 32, replace=False)]))
    Xf, dYf = bf16(X), bf16(dY)
    Grows = dYf[:, rows].T @ Xf
    dWr = dW[torch.from_numpy(rows).cuda()].cpu().numpy().astype(np.float64)
    tolG = 2 * (M + 2) * EPS * (np.abs(dYf[:, rows]).T @ np.abs(Xf)) + 1e-30
    assert np.all(np.abs(dWr - Grows) <= tolG)
    S_rows = signs(planes, N, K, k, rows, np.arange(K))               # oracle planes, +-1 [k][rows][K]
    S_cols = signs(planes, N, K, k, np.arange(N), cols)                # +-1 [k][N][cols]
    hf, gf = h.astype(np.float64), g.astype(np.float64)
    dg_ref = np.einsum("nc,inc,ic->in", Grows, S_rows, hf)
    tol_g = np.einsum("nc,ic->in", tolG, np.abs(hf)) + 2 * (K + 2) * EPS * np.einsum("nc,ic->in", np.abs(Grows), np.abs(hf))
    dgg = dg.cpu().numpy().astype(np.float64)[:, rows]
    assert np.all(np.abs(dgg - dg_ref) <= tol_g + 1e-30)
    Gcols = dYf.T @ Xf[:, cols]
    dh_ref = np.einsum("nc,in,inc->ic", Gcols, gf, S_cols)
    tolGc = 2 * (M + 2) * EPS * (np.abs(dYf).T @ np.abs(Xf[:, cols]))
    tol_h = np.einsum("nc,in->ic", tolGc, np.abs(gf)) + 2 * (N + 2) * EPS * np.einsum("nc,in->ic", np.abs(Gcols), np.abs(gf))
    dhh = dh.cpu().numpy().astype(np.float64)[:, cols]
    assert np.all(np.abs(dhh - dh_ref) <= tol_h + 1e-30)


def test_qat_backward_is_deterministic_and_checks_args():
    N, K, k, M = 256, 512, 2, 64
    rng = np.random.default_rng(1)
    W = (rng.standard_normal((N, K)) * 0.02).astype(np.float32)
    g, h = oracle.svid_greedy(W, k, iters=4)
    planes, g16, h16, _, _ = oracle.pack(W, g, h, k)
    L = cases.upload_layer(planes, g16, h16, N, K, k)
    X, dY = cases.to_dev(synth.activations(M, K, seed=1)), cases.to_dev(synth.activations(M, N, seed=2))
    gd, hd = cases.to_dev(g), cases.to_dev(h)
    a = rbw.qat_backward(L, gd, hd, X, dY)
    b = rbw.qat_backward(L, gd, hd, X, dY)
    torch.cuda.synchronize()
    for x, y in zip(a, b):
        assert torch.equal(x, y)
    L2 = rbw.PackedLayer(100, 512, 2)
    with pytest.raises(rbw.RbError) as e:
        rbw.qat_backward(L2, gd[:, :100].contiguous(), hd, X, cases.to_dev(synth.activations(M, 100, seed=3)))
    assert e.value.status == rbw.RB_ERR_SHAPE


@pytest.mark.parametrize("N,K,k,M", [(256, 512, 2, 100), (300, 800, 1, 64), (4096, 1024, 2, 2048), (128, 288, 2, 7),
                                     (1000, 4096, 1, 1500), (4097, 544, 2, 300), (640, 1024, 3, 1100),
                                     (256, 512, 4, 129), (160, 256, 8, 40)])
def test_qat_forward_matches_oracle(N, K, k, M):
    """rb_qat_forward (planes derived from fp32 W, then the tcgen05 GEMM with
    the fp32 g) against the oracle's float64 training forward.
    Gate from the arithmetic: the +-h operands are fp16(h) (relative error <=
    2^-11) and the MMA accumulates exact products in fp32, so each element is
    within (2^-11 + 1e-4) sum |g h x| (bf16 output: plus one bf16 step)."""
    rng = np.random.default_rng(N + K + k + M)
    W = (rng.standard_normal((N, K)) * 0.02).astype(np.float32)
    W[rng.random((N, K)) < 0.01] = 0.0
    g, h = oracle.svid_greedy(W, k, iters=6)
    X = synth.activations(M, K, seed=M + 3)
    rows = np.unique(np.concatenate([np.arange(min(N, 40)), np.arange(max(0, N - 40), N),
                                     rng.choice(N, min(N, 160), replace=False)]))
    toks = np.unique(np.concatenate([np.arange(min(M, 16)), np.arange(max(0, M - 16), M),
                                     rng.choice(M, min(M, 40), replace=False)]))
    st, Yr = oracle.qat_forward(W, g, h, k, X, rows=rows, toks=toks)
    assert st == 0
    Xf = np.abs(bf16(X[toks]))
    bound = Xf @ np.abs(h.astype(np.float64)).T @ np.abs(g.astype(np.float64)[:, rows])     # sum |g h x|
    for ydt in (torch.float32, torch.bfloat16):
        s = torch.zeros(4, dtype=torch.int32, device="cuda")
        Y = rbw.qat_forward(cases.to_dev(W), cases.to_dev(g), cases.to_dev(h), k, cases.to_dev(X), dev_status=s,
                            y_dtype=ydt)
        torch.cuda.synchronize()
        assert int(s[0].item()) == 0
        Yg = Y.float().cpu().numpy().astype(np.float64)[np.ix_(toks, rows)]
        cases.check_y(Yg, Yr, bound, bf16=ydt == torch.bfloat16, per_elem=2.0 ** -11 + 1e-4)


def test_qat_forward_equals_deployment_gemm_on_fp16_exact_scales():
    """With fp16-exact scales the training forward reaches the packed layer's
    product bit for bit: rb_qat_forward(W, g, h) equals rb_gemm on rb_pack's
    planes of the same W (the same MMA operands, the same accumulation), and
    the planes it leaves in its workspace are rb_pack's."""
    N, K, k, M = 512, 1024, 2, 256
    rng = np.random.default_rng(3)
    W = (rng.standard_normal((N, K)) * 0.02).astype(np.float32)
    g, h = oracle.svid_greedy(W, k, iters=6)
    g = g.astype(np.float16).astype(np.float32)
    h = h.astype(np.float16).astype(np.float32)
    Wd, gd, hd = cases.to_dev(W), cases.to_dev(g), cases.to_dev(h)
    X = cases.to_dev(synth.activations(M, K, seed=8))
    wsf = rbw.workspace(rbw.qat_forward_workspace_bytes(N, K, k, M))
    Yf = rbw.qat_forward(Wd, gd, hd, k, X, ws=wsf)
    L = rbw.pack(Wd, gd, hd, k)
    Yp = rbw.gemm(L, X, ws=rbw.workspace(rbw.gemm_workspace_bytes(N, K, k, M)))
    torch.cuda.synchronize()
    assert torch.equal(Yf, Yp)
    nw = int(rbw.lib().rb_packed_words(N, K, k))
    assert torch.equal(wsf.view(torch.int32)[:nw], L.planes.view(torch.int32)[:nw])


def test_qat_forward_flags_and_limits():
    """A NaN or infinite latent weight and a NaN h raise RB_DEV_NONFINITE (the
    run still completes); k = 9 and a workspace one byte short are refused."""
    N, K, k, M = 128, 256, 2, 64
    rng = np.random.default_rng(5)
    W = (rng.standard_normal((N, K)) * 0.02).astype(np.float32)
    g, h = oracle.svid_greedy(W, k, iters=4)
    X = cases.to_dev(synth.activations(M, K, seed=4))
    for bad in ("W_nan", "W_inf", "h_nan"):
        Wb, hb = W.copy(), h.copy()
        if bad == "W_nan":
            Wb[77, 130] = np.nan
        elif bad == "W_inf":
            Wb[3, 255] = -np.inf
        else:
            hb[1, 31] = np.nan
        s = torch.zeros(4, dtype=torch.int32, device="cuda")
        rbw.qat_forward(cases.to_dev(Wb), cases.to_dev(g), cases.to_dev(hb), k, X, dev_status=s)
        torch.cuda.synchronize()
        assert int(s[0].item()) & rbw.RB_DEV_NONFINITE, bad
    g9, h9 = np.concatenate([g] * 5)[:9], np.concatenate([h] * 5)[:9]
    with pytest.raises(rbw.RbError):
        rbw.qat_forward(cases.to_dev(W), cases.to_dev(g9), cases.to_dev(h9), 9, X)
    short = rbw.workspace(rbw.qat_forward_workspace_bytes(N, K, k, M) - 16)
    with pytest.raises(rbw.RbError):
        rbw.qat_forward(cases.to_dev(W), cases.to_dev(g), cases.to_dev(h), k, X, ws=short)
