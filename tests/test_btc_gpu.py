"""Binary-codebook layer (BTC-LLM, "Binary codebook" and "LUT-GEMM") on the
GPU against the oracle: rb_btc_encode is integer work and must reproduce the
oracle's codebook and index streams bit for bit; rb_btc_gemv forms h*x
exactly in fp32 and adds in fp32 like the byte-table decode path, so it takes
that path's gate (per element 1e-5 of sum |g h x|, relative Frobenius 2e-3)
against the float64 application of the reconstructed layer."""
import numpy as np
import pytest
import torch

import oracle
from residual_binarized_weight_b200 import rbw, synth
from tests import cases

pytestmark = pytest.mark.gpu


def make(N, K, k, seed, skew=False):
    rng = np.random.default_rng(seed)
    if skew:                                        # 16-column groups near a few prototypes
        protos = rng.integers(0, 65536, 12)
        pick = protos[rng.integers(0, 12, (N, K // 16))]
        noise = ((rng.random((N, K // 16, 16)) < 0.06) << np.arange(16)).sum(-1)
        pat = (pick ^ noise).astype(np.uint32)
        B = np.where((pat[..., None] >> np.arange(16)) & 1, 1.0, -1.0).reshape(N, K)
        W = (B * (0.5 + rng.random((N, K))) * 0.02).astype(np.float32)
    else:
        W = (rng.standard_normal((N, K)) * 0.02).astype(np.float32)
    g, h = oracle.svid_greedy(W, k, iters=4)
    planes, g16, h16, _, _ = oracle.pack(W, g, h, k)
    return planes, g16, h16


@pytest.mark.parametrize("N,K,k,c_max,iters,skew", [(96, 256, 1, 5, 4, True), (300, 800, 2, 40, 6, True),
                                                    (64, 512, 2, 65536, 2, False), (4096, 4096, 2, 256, 3, False),
                                                    (256, 512, 1, 7132, 1, False), (33, 96, 2, 1, 2, False)])
def test_encode_is_bit_exact(N, K, k, c_max, iters, skew):
    planes, g16, h16 = make(N, K, k, seed=N + K + k, skew=skew)
    L = cases.upload_layer(planes, g16, h16, N, K, k)
    B = rbw.btc_encode(L, c_max, iters)
    torch.cuda.synchronize()
    w = oracle.btc_index_bits(c_max)
    assert B.index_bits == w
    for i in range(k):
        cb, c, idx, _ = oracle.btc_encode(planes, N, K, k, i, c_max, iters)
        assert int(B.sizes[i, 0].item()) == c
        assert np.array_equal(B.codebooks[i].cpu().numpy().view(np.uint16), cb)
        streams = oracle.btc_pack_indices(idx, N, K, w)
        assert np.array_equal(B.indices[i].cpu().numpy().view(np.uint32), streams)


@pytest.mark.parametrize("N,K,k,c_max,skew", [(96, 256, 1, 5, True), (300, 800, 2, 40, True), (4097, 544, 2, 300, False),
                                              (4096, 4096, 2, 256, False), (1000, 4096, 1, 1024, False),
                                              (260, 8192, 2, 100, False)])
def test_gemv_matches_oracle(N, K, k, c_max, skew):
    """Ragged N and K, k = 1 and 2, up to 32 slices (K = 8192), fp32 and bf16
    output, with and without PDL (bit-identical)."""
    planes, g16, h16 = make(N, K, k, seed=N * 3 + K + k, skew=skew)
    L = cases.upload_layer(planes, g16, h16, N, K, k)
    B = rbw.btc_encode(L, c_max, iters=3)
    X = synth.activations(1, K, seed=N + 1)
    cbs = B.codebooks.cpu().numpy().view(np.uint16)
    idx = np.stack([oracle.btc_encode(planes, N, K, k, i, c_max, 3)[2] for i in range(k)])
    rows = np.unique(np.concatenate([np.arange(min(N, 64)), np.arange(max(0, N - 64), N),
                                     np.random.default_rng(1).choice(N, min(N, 300), replace=False)]))
    Yr = oracle.btc_apply(cbs, c_max, idx, g16, h16, N, K, k, X, rows=rows)
    bound = cases.abs_bound(g16, h16, X, rows=rows)
    Xd = cases.to_dev(X)
    for ydt in (torch.float32, torch.bfloat16):
        Y = rbw.btc_gemv(B, Xd, y_dtype=ydt)
        Y2 = rbw.btc_gemv(B, Xd, y_dtype=ydt, flags=rbw.RB_LAUNCH_PDL)
        torch.cuda.synchronize()
        assert torch.equal(Y, Y2)                    # deterministic, with and without PDL
        cases.check_y(Y.float().cpu().numpy().astype(np.float64)[:, rows], Yr, bound, bf16=ydt == torch.bfloat16)


def test_full_codebook_reproduces_the_plane_layer():
    """When every pattern fits in the codebook the layer is reproduced and
    rb_btc_gemv agrees with rb_gemv on the packed planes within the gate."""
    N, K, k = 512, 1024, 2
    planes, g16, h16 = make(N, K, k, seed=11)
    L = cases.upload_layer(planes, g16, h16, N, K, k)
    B = rbw.btc_encode(L, 65536, iters=1)
    X = synth.activations(1, K, seed=12)
    Xd = cases.to_dev(X)
    Yb = rbw.btc_gemv(B, Xd)
    Yg = rbw.gemv(L, Xd)
    torch.cuda.synchronize()
    Yr = oracle.apply(planes, g16, h16, N, K, k, X)
    bound = cases.abs_bound(g16, h16, X)
    for Y in (Yb, Yg):
        cases.check_y(Y.cpu().numpy().astype(np.float64), Yr, bound, bf16=False)


def test_errors():
    N, K, k = 64, 256, 2
    planes, g16, h16 = make(N, K, k, seed=2)
    L = cases.upload_layer(planes, g16, h16, N, K, k)
    B = rbw.btc_encode(L, 16, iters=1)
    Xd = cases.to_dev(synth.activations(1, K, seed=3))
    with pytest.raises(rbw.RbError) as e:
        rbw.btc_gemv(B, Xd, ws=rbw.workspace(rbw.lib().rb_btc_gemv_workspace_bytes(N, K) - 16))
    assert e.value.status == rbw.RB_ERR_WORKSPACE
    B.index_bits += 1
    with pytest.raises(rbw.RbError) as e:
        rbw.btc_gemv(B, Xd)
    assert e.value.status == rbw.RB_ERR_ARG
    B.index_bits -= 1
    B.k_planes = 3
    with pytest.raises(rbw.RbError) as e:
        rbw.btc_gemv(B, Xd)
    assert e.value.status == rbw.RB_ERR_UNSUPPORTED


def test_gemv_batch_equals_single_calls():
    """A batch of distinct codebook layers and tokens (70 layers: a group of 64
    and one of 6) reproduces each single-layer call bit for bit."""
    N, K, k = 200, 512, 2
    layers, Xs, singles = [], [], []
    for j in range(70):
        planes, g16, h16 = make(N, K, k, seed=100 + j % 5)
        L = cases.upload_layer(planes, g16, h16, N, K, k)
        layers.append(rbw.btc_encode(L, 32, iters=2))
        layers[-1].keep = L                           # the scales live in the packed layer
        Xs.append(cases.to_dev(synth.activations(1, K, seed=200 + j)))
    for B, X in zip(layers, Xs):
        singles.append(rbw.btc_gemv(B, X))
    Ys = [torch.empty(1, N, device="cuda") for _ in layers]
    rbw.btc_gemv_batch(layers, Xs, Ys, flags=rbw.RB_LAUNCH_PDL)
    torch.cuda.synchronize()
    for a, b in zip(Ys, singles):
        assert torch.equal(a, b)


def test_gemv_batch_of_full_size_layers_equals_single_calls():
    """48 layers of 4096 x 1024 in one batch (3072 CTAs): every output equals
    the single-layer call bit for bit."""
    N, K, k = 4096, 1024, 2
    planes, g16, h16 = make(N, K, k, seed=77)
    L = cases.upload_layer(planes, g16, h16, N, K, k)
    B = rbw.btc_encode(L, 512, iters=2)
    B.keep = L
    Xs = [cases.to_dev(synth.activations(1, K, seed=300 + j)) for j in range(48)]
    singles = [rbw.btc_gemv(B, X) for X in Xs]
    Ys = [torch.empty(1, N, device="cuda") for _ in Xs]
    rbw.btc_gemv_batch([B] * 48, Xs, Ys)
    torch.cuda.synchronize()
    for a, b in zip(Ys, singles):
        assert torch.equal(a, b)
