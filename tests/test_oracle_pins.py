"""Pins of the CPU oracle against facts fixed outside the oracle itself.

Each test names the passage or the mathematical fact it rests on:
  * RaBiT "Residual binarization": W ~= sum_i g_i . B_i . h_i, B_i in {-1,+1}.
  * RaBiT Algorithm 2 forward: R_0 = W, B_i = sign(R_{i-1}), R_i = R_{i-1} - W_i.
  * BTC-LLM, binary k-means M-step: a zero entry takes the sign +1.
  * BTC-LLM, "bit-compressed computation": the +-1 dot product equals
    n - 2*popcount(a XOR b) on packed vectors.
  * RaBiT, limitations paragraph: 2.02 effective bits per weight at k = 2.
No expected value here is computed by the CUDA library.
"""
import fractions
import itertools
import math
import os

import numpy as np
import pytest
import torch

import oracle
from residual_binarized_weight_b200 import synth
from tests import layout

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def bf16_to_f64(bits):
    return torch.from_numpy(np.asarray(bits, np.uint16).view(np.int16)).view(torch.bfloat16).double().numpy()


# ---------------------------------------------------------------- number formats

def test_f16_encoder_matches_numpy_float16():
    """The fp16 scale cast is IEEE binary16 round-to-nearest-even (numpy's astype)."""
    rng = np.random.default_rng(1)
    vals = np.concatenate([
        rng.standard_normal(20000) * 10.0 ** rng.uniform(-9, 5, 20000),
        np.array([0.0, -0.0, 65504.0, 65519.99, 65520.0, -65520.0, 1e-8, 2.0 ** -24,
                  2.0 ** -25, 3 * 2.0 ** -26, 2.0 ** -14, 1.0 + 2.0 ** -11, 1.0 + 3 * 2.0 ** -11,
                  np.inf, -np.inf]),
    ]).astype(np.float32)
    want = vals.astype(np.float16).view(np.uint16)
    got = np.array([oracle.f64_to_f16_bits(float(v)) for v in vals], np.uint16)
    assert np.array_equal(got, want)
    back = np.array([oracle.f16_bits_to_f64(int(b)) for b in want[:2000]])
    assert np.array_equal(back, want[:2000].view(np.float16).astype(np.float64))


def test_bf16_encoder_matches_torch():
    """bfloat16 outputs are round-to-nearest-even of the exact value (torch's cast)."""
    rng = np.random.default_rng(2)
    vals = (rng.standard_normal(20000) * 10.0 ** rng.uniform(-30, 30, 20000)).astype(np.float32)
    vals = np.concatenate([vals, np.float32([1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -0.0, 3e38])])
    want = torch.from_numpy(vals).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    got = np.array([oracle.f64_to_bf16_bits(float(v)) for v in vals], np.uint16)
    assert np.array_equal(got, want)
    assert np.array_equal(np.array([oracle.bf16_bits_to_f64(int(b)) for b in want]), bf16_to_f64(want))


# ---------------------------------------------------------------- layout, polarity, sign(0)

@pytest.mark.parametrize("N,K", [(8, 256), (6, 96), (13, 544), (4, 32)])
def test_k1_planes_are_sign_of_w(N, K):
    """k = 1: B_1 = sign(W) with sign(0) = +1 (zeros and -0.0 give bit 1)."""
    rng = np.random.default_rng(N * 1000 + K)
    W = rng.standard_normal((N, K)).astype(np.float32)
    W[0, :5] = [0.0, -0.0, 0.0, -0.0, 0.0]
    W[-1, -3:] = -0.0
    g = np.ones((1, N), np.float32)
    h = np.ones((1, K), np.float32)
    planes, g16, h16, st, _ = oracle.pack(W, g, h, 1)
    assert st == 0
    want = layout.pack_bits((W >= 0)[None])           # np.packbits in the stated layout
    assert np.array_equal(planes, want)
    assert not layout.padding_words_and_bits(planes, N, K, 1).any()
    assert np.all(g16 == 0x3C00) and np.all(h16 == 0x3C00)


def test_k1_unit_scales_apply_is_sign_matvec():
    """k = 1, g = h = 1: Y = X . sign(W)^T, a textbook matrix product (numpy)."""
    rng = np.random.default_rng(3)
    N, K, M = 40, 320, 3
    W = rng.standard_normal((N, K)).astype(np.float32)
    X = synth.activations(M, K, seed=9)
    planes, g16, h16, st, _ = oracle.pack(W, np.ones((1, N), np.float32), np.ones((1, K), np.float32), 1)
    Y = oracle.apply(planes, g16, h16, N, K, 1, X)
    S = np.where(W >= 0, 1.0, -1.0)
    want = bf16_to_f64(X) @ S.T
    np.testing.assert_allclose(Y, want, rtol=1e-12, atol=1e-12)


def test_popcount_identity():
    """+-1 dot = K - 2*popcount(a XOR b) on packed words (BTC-LLM Hamming step)."""
    rng = np.random.default_rng(4)
    N, K = 16, 512
    W = rng.standard_normal((N, K)).astype(np.float32)
    xs = np.where(rng.standard_normal(K) >= 0, 1.0, -1.0).astype(np.float32)
    X = synth.to_bf16_bits(xs[None])
    planes, g16, h16, _, _ = oracle.pack(W, np.ones((1, N), np.float32), np.ones((1, K), np.float32), 1)
    Y = oracle.apply(planes, g16, h16, N, K, 1, X)[0]
    xw = np.packbits(xs >= 0, bitorder="little").view("<u4")
    rows = layout.gather_rows(planes, N, K, 1, np.arange(N)).reshape(N, -1)
    for r in range(N):
        ham = sum(bin(int(a) ^ int(b)).count("1") for a, b in zip(rows[r], xw))
        assert Y[r] == K - 2 * ham


# ---------------------------------------------------------------- derivation

def _brute_best(R, T):
    """All B in {-1,+1}^{shape} minimising ||R - T.*B||_F (exhaustive)."""
    n = R.size
    best, arg = None, []
    for bits in itertools.product([1.0, -1.0], repeat=n):
        B = np.array(bits).reshape(R.shape)
        e = float(np.sum((R.astype(np.float64) - T * B) ** 2))
        if best is None or e < best - 1e-300:
            best, arg = e, [B]
        elif e == best:
            arg.append(B)
    return arg


@pytest.mark.parametrize("shape,seed", [((2, 32), 5), ((3, 32), 6)])
def test_plane_is_least_squares_sign_brute_force(shape, seed):
    """sign(R) minimises ||R - (g h^T).*B|| over all B (exhaustive over a 2x4/3x4 block);
    exact zeros are ties and take +1."""
    rng = np.random.default_rng(seed)
    N, K = shape
    W = rng.standard_normal((N, K)).astype(np.float32)
    W[0, 1] = 0.0
    W[1, 2] = -0.0
    g, h = synth.positive_scales(2, N, K, seed)
    planes2, _, _, _, _ = oracle.pack(W, g, h, 2)
    _, _, _, _, R1 = oracle.pack(W, g[:1], h[:1], 1, want_residual=True)
    Bs = np.where(layout.unpack_bits(planes2, N, K, 2), 1.0, -1.0)
    for i, Rprev in ((0, W), (1, R1)):
        T = np.outer(g[i], h[i]).astype(np.float64)
        blk = (slice(0, N), slice(0, 4))            # 2^(N*4) candidates
        cands = _brute_best(Rprev[blk], T[blk])
        assert any(np.array_equal(Bs[i][blk], c) for c in cands)
        if len(cands) > 1:                           # ties only at exact zeros -> +1
            zero = Rprev[blk] == 0
            assert np.all(Bs[i][blk][zero] == 1.0)
    assert Bs[0][0, 1] == 1.0 and Bs[0][1, 2] == 1.0


def test_residual_equals_w_minus_reconstruction():
    """R_k = W - sum_i g_i . B_i . h_i up to the fp32 roundings of the recurrence."""
    rng = np.random.default_rng(7)
    N, K, k = 24, 288, 3
    W = (rng.standard_normal((N, K)) * 0.02).astype(np.float32)
    g, h = oracle.svid_greedy(W, k)
    planes, _, _, st, R = oracle.pack(W, g, h, k, want_residual=True)
    assert st == 0
    B = np.where(layout.unpack_bits(planes, N, K, k), 1.0, -1.0)
    recon = sum(np.outer(g[i], h[i]).astype(np.float64) * B[i] for i in range(k))
    err = np.abs(R.astype(np.float64) - (W.astype(np.float64) - recon))
    bound = 2 * k * 2.0 ** -24 * (np.abs(W) + sum(np.outer(g[i], h[i]) for i in range(k)) * 2)
    assert np.all(err <= bound)


def test_no_fused_multiply_add_in_recurrence():
    """g*h is rounded to fp32 before the subtraction (worked by hand):
    g = h = 1 + 2^-12 -> fl(g*h) = 1 + 2^-11 (tie to even drops 2^-24);
    W = 1 + 2^-11 + 2^-23 -> R_1 = 2^-23 exactly (a fused form would give 2^-24)."""
    g = np.float32([[1.0 + 2.0 ** -12]])
    h = np.full((1, 32), 1.0 + 2.0 ** -12, np.float32)
    W = np.full((1, 32), 1.0 + 2.0 ** -11 + 2.0 ** -23, np.float32)
    _, _, _, st, R = oracle.pack(W, g, h, 1, want_residual=True)
    assert st == 0
    assert np.all(R == np.float32(2.0 ** -23))


@pytest.mark.parametrize("k", [1, 2, 3, 4])
def test_residual_norm_non_increasing(k):
    """||R_i||_F <= ||R_{i-1}||_F for rank-1 least-squares scales: |R_i| = | |R_{i-1}| - g h^T |
    and ||A - sigma u v^T||^2 = ||A||^2 - sigma^2 for sigma = u^T A v (any unit u, v)."""
    wl = synth.workload(1)
    W = synth.weights(wl.layers[0], 96, 512)
    g, h = oracle.svid_greedy(W, k)
    norms = [float(np.linalg.norm(W.astype(np.float64)))]
    for i in range(1, k + 1):
        _, _, _, _, R = oracle.pack(W, g[:i], h[:i], i, want_residual=True)
        norms.append(float(np.linalg.norm(R.astype(np.float64))))
    for a, b in zip(norms, norms[1:]):
        assert b <= a * (1 + 1e-6)
    assert norms[-1] < norms[0]


def test_svid_plane1_is_top_singular_pair_of_abs_w():
    """Plane-1 greedy SVID scales reproduce the top singular triple of |W| (numpy SVD)."""
    wl = synth.workload(0)
    W = synth.weights(wl.layers[0])
    g, h = oracle.svid_greedy(W, 1, iters=20)
    U, s, Vt = np.linalg.svd(np.abs(W.astype(np.float64)), full_matrices=False)
    ref = s[0] * np.outer(U[:, 0], Vt[0])
    ref *= np.sign(ref.sum())
    got = np.outer(g[0], h[0]).astype(np.float64)
    assert np.linalg.norm(got - ref) / np.linalg.norm(ref) < 1e-4
    assert np.all(g >= 0) and np.all(h >= 0)


@pytest.mark.parametrize("wl_index,shape", [(0, None), (1, (512, 1024))])
def test_svid_later_planes_are_top_singular_pair_of_abs_residual(wl_index, shape):
    """Greedy SVID (RaBiT, Technical novelty: the traditional greedy initialiser):
    plane i's scales reproduce the top singular triple of |R_{i-1}| (numpy SVD),
    with R_{i-1} the fp32 residual of the recurrence after the first i-1 planes
    (RaBiT Algorithm 2 forward).  Pins planes 2..4 directly: feeding plane i
    the wrong residual, or W itself, moves g_i h_i^T far from this triple."""
    W = synth.weights(synth.workload(wl_index).layers[0], *(shape or (None, None)))
    k = 4
    g, h = oracle.svid_greedy(W, k, iters=20)
    for i in range(2, k + 1):
        _, _, _, st, R = oracle.pack(W, g[:i - 1], h[:i - 1], i - 1, want_residual=True)
        assert st == 0
        U, s, Vt = np.linalg.svd(np.abs(R.astype(np.float64)), full_matrices=False)
        ref = s[0] * np.outer(U[:, 0], Vt[0])
        ref *= np.sign(ref.sum())
        got = np.outer(g[i - 1], h[i - 1]).astype(np.float64)
        assert np.linalg.norm(got - ref) / np.linalg.norm(ref) < 1e-4, "plane %d" % i
        assert np.all(g[i - 1] >= 0) and np.all(h[i - 1] >= 0)


def test_zero_weight_degenerate():
    """W = 0: every plane is all +1 (sign(0) = +1), greedy scales are 0, R stays 0."""
    N, K = 8, 64
    W = np.zeros((N, K), np.float32)
    g, h = oracle.svid_greedy(W, 2)
    assert np.all(g == 0) and np.all(h == 0)
    planes, _, _, st, R = oracle.pack(W, g, h, 2, want_residual=True)
    assert st == 0 and np.all(R == 0)
    assert layout.unpack_bits(planes, N, K, 2).all()


def test_bad_inputs_status():
    W = np.ones((4, 64), np.float32)
    g = np.ones((1, 4), np.float32)
    h = np.ones((1, 64), np.float32)
    W2 = W.copy()
    W2[1, 3] = np.nan
    assert oracle.pack(W2, g, h, 1)[3] == 1
    g2 = g.copy()
    g2[0, 0] = 70000.0
    assert oracle.pack(W, g2, h, 1)[3] == 2
    assert oracle.pack(np.ones((4, 48), np.float32), g, np.ones((1, 48), np.float32), 1)[3] == -1


# ---------------------------------------------------------------- application

def test_apply_equals_exact_matmul_free_form():
    """The dequantise-then-multiply oracle equals the matmul-free form
    Y = sum_i g_i . (B_i (h_i . x)) evaluated in exact rational arithmetic."""
    rng = np.random.default_rng(8)
    N, K, k, M = 5, 64, 2, 2
    W = (rng.standard_normal((N, K)) * 0.02).astype(np.float32)
    g, h = oracle.svid_greedy(W, k)
    planes, g16, h16, _, _ = oracle.pack(W, g, h, k)
    X = synth.activations(M, K, seed=11)
    Y = oracle.apply(planes, g16, h16, N, K, k, X)
    B = layout.unpack_bits(planes, N, K, k)
    F = fractions.Fraction
    gq = g16.view(np.float16).astype(np.float64)
    hq = h16.view(np.float16).astype(np.float64)
    xq = bf16_to_f64(X)
    for m in range(M):
        for n in range(N):
            tot = F(0)
            for i in range(k):
                acc = F(0)
                for c in range(K):
                    hx = F(hq[i, c]) * F(xq[m, c])
                    acc += hx if B[i, n, c] else -hx
                tot += F(gq[i, n]) * acc
            assert math.isclose(Y[m, n], float(tot), rel_tol=1e-12, abs_tol=1e-15)


def test_apply_row_and_token_subsets():
    rng = np.random.default_rng(10)
    N, K, k, M = 12, 256, 2, 4
    W = rng.standard_normal((N, K)).astype(np.float32)
    g, h = synth.positive_scales(k, N, K, 3)
    planes, g16, h16, _, _ = oracle.pack(W, g, h, k)
    X = synth.activations(M, K, seed=1)
    full = oracle.apply(planes, g16, h16, N, K, k, X)
    rows, toks = [11, 0, 5], [3, 1]
    sub = oracle.apply(planes, g16, h16, N, K, k, X, rows=rows, toks=toks)
    assert np.array_equal(sub, full[np.ix_(toks, rows)])
    packed_rows = oracle.pack_rows(W, g, h, k, rows)
    assert np.array_equal(packed_rows, layout.gather_rows(planes, N, K, k, rows))


# ---------------------------------------------------------------- sizes

def test_effective_bits_matches_page():
    """Stored bits per weight at 4096 x 4096, k = 2 with fp16 g, h (RaBiT: 2.02)."""
    with open(os.path.join(GOLDEN, "effective_bits.txt")) as f:
        rows = [l.split() for l in f if l.strip() and not l.startswith("#")]
    for N, K, k, want in rows:
        N, K, k = int(N), int(K), int(k)
        plane_bytes = 4 * oracle.plane_words(N, K, k)
        scale_bytes = 2 * k * (N + K)
        bpw = 8.0 * (plane_bytes + scale_bytes) / (N * K)
        assert round(bpw, 2) == float(want)


# ---------------------------------------------------------------- iterative residual SVID
def _numpy_iterative_svid(W, k, sweeps):
    """Independent restatement with exact rank-1 factors (numpy SVD), returning
    the scales and the reconstruction error after every Gauss-Seidel step."""
    W64 = W.astype(np.float64)
    N, K = W.shape

    def rank1_abs(A):
        U, s, Vt = np.linalg.svd(np.abs(A), full_matrices=False)
        u, v = np.abs(U[:, 0]), np.abs(Vt[0])            # Perron vectors of a nonnegative matrix
        return (np.sqrt(s[0]) * u).astype(np.float32), (np.sqrt(s[0]) * v).astype(np.float32)

    g = np.zeros((k, N), np.float32)
    h = np.zeros((k, K), np.float32)
    B = np.zeros((k, N, K), np.float64)
    R = W.copy()
    for i in range(k):                                    # greedy pass, fp32 recurrence
        g[i], h[i] = rank1_abs(R)
        b = R >= 0
        B[i] = np.where(b, 1.0, -1.0)
        t = (g[i][:, None] * h[i][None, :]).astype(np.float32)
        R = np.where(b, R - t, R + t).astype(np.float32)

    def err():
        What = sum(g[j].astype(np.float64)[:, None] * B[j] * h[j].astype(np.float64)[None, :] for j in range(k))
        return float(np.linalg.norm(W64 - What))

    errs = [err()]
    for _ in range(sweeps):
        for i in range(k):
            T = W64.copy()
            for j in range(k):
                if j != i:
                    T = T - B[j] * (g[j].astype(np.float64)[:, None] * h[j].astype(np.float64)[None, :])
            B[i] = np.where(T >= 0, 1.0, -1.0)
            g[i], h[i] = rank1_abs(T)
            errs.append(err())
    return g, h, errs


def test_iterative_svid_k1_is_greedy():
    """With one plane the target is W itself every sweep: the greedy scales."""
    W = synth.weights(synth.workload(1).layers[0], 64, 128)
    g0, h0 = oracle.svid_greedy(W, 1, iters=20)
    g1, h1 = oracle.svid_iterative(W, 1, sweeps=5, iters=20)
    assert np.array_equal(g0, g1) and np.array_equal(h0, h1)


def test_iterative_svid_zero_sweeps_is_greedy():
    W = synth.weights(synth.workload(1).layers[0], 48, 96)
    g0, h0 = oracle.svid_greedy(W, 3, iters=20)
    g1, h1 = oracle.svid_iterative(W, 3, sweeps=0, iters=20)
    assert np.array_equal(g0, g1) and np.array_equal(h0, h1)


@pytest.mark.parametrize("k,sweeps", [(2, 3), (3, 2)])
def test_iterative_svid_matches_exact_svd_restatement(k, sweeps):
    """The oracle (converged power iteration) agrees with an independent numpy
    restatement that takes the exact top singular pair; the restatement's
    error ||W - sum_i g_i B_i h_i|| never increases step by step (each step is
    the exact minimiser over one plane) and ends below the greedy pass."""
    rng = np.random.default_rng(5 + k)
    W = (rng.standard_normal((40, 96)) * 0.02).astype(np.float32)
    g_ref, h_ref, errs = _numpy_iterative_svid(W, k, sweeps)
    assert all(b <= a * (1 + 1e-12) for a, b in zip(errs, errs[1:])), errs
    assert errs[-1] < errs[0]
    g, h = oracle.svid_iterative(W, k, sweeps=sweeps, iters=400)
    for a, b in ((g, g_ref), (h, h_ref)):
        rel = np.abs(a.astype(np.float64) - b) / np.abs(b).max(axis=1, keepdims=True)
        assert rel.max() < 1e-5, rel.max()


# ---------------------------------------------------------------- transposed layer, input gradient
# shapes: N a multiple of 32 (the transposed layer's input width); N and K not
# multiples of 256 so both layouts have a ragged last slice and row-tile group.
_T_SHAPES = [(32, 32, 1), (96, 320, 2), (288, 800, 3), (64, 1056, 4)]


@pytest.mark.parametrize("N,K,k", _T_SHAPES)
def test_transposed_planes_equal_planes_of_transposed_weight(N, K, k):
    """The recurrence is element-wise and fl(g*h) = fl(h*g), so the planes of
    (W, g, h) transposed are exactly the planes derived from (W^T, h, g)."""
    rng = np.random.default_rng(N + K + k)
    W = (rng.standard_normal((N, K)) * 0.02).astype(np.float32)
    W[rng.random((N, K)) < 0.01] = 0.0                     # sign(0) ties take part too
    g, h = synth.positive_scales(k, N, K, seed=k)
    planes, g16, h16, st, _ = oracle.pack(W, g, h, k)
    planes_t2, g16_t, h16_t, st_t, _ = oracle.pack(np.ascontiguousarray(W.T), h, g, k)
    assert st == 0 and st_t == 0
    assert np.array_equal(oracle.transpose_planes(planes, N, K, k), planes_t2)
    assert np.array_equal(g16_t, h16) and np.array_equal(h16_t, g16)


@pytest.mark.parametrize("N,K,k", _T_SHAPES)
def test_transpose_is_the_bit_matrix_transpose(N, K, k):
    """Against the numpy layout helpers: unpacking the transposed planes gives
    the transposed sign matrices, padding stays zero, and a second transpose
    (allowed when K is a multiple of 32) restores the planes."""
    rng = np.random.default_rng(3 * N + K)
    B = rng.random((k, N, K)) < 0.5
    planes = layout.pack_bits(B)
    pt = oracle.transpose_planes(planes, N, K, k)
    assert np.array_equal(layout.unpack_bits(pt, K, N, k), B.transpose(0, 2, 1))
    assert not layout.padding_words_and_bits(pt, K, N, k).any()
    assert np.array_equal(oracle.transpose_planes(pt, K, N, k), planes)


def test_input_gradient_matches_dense_product_and_adjoint():
    """dX = dY . What: equal to numpy's product with the dense What built from
    the layout helpers; equal to the forward oracle on the transposed layer;
    and <dY, X What^T> = <dY What, X> (the adjoint identity)."""
    rng = np.random.default_rng(21)
    N, K, k, M = 96, 320, 2, 3
    W = (rng.standard_normal((N, K)) * 0.02).astype(np.float32)
    g, h = oracle.svid_greedy(W, k)
    planes, g16, h16, _, _ = oracle.pack(W, g, h, k)
    dY = synth.activations(M, N, seed=5)
    X = synth.activations(M, K, seed=6)
    dX = oracle.apply_t(planes, g16, h16, N, K, k, dY)
    B = np.where(layout.unpack_bits(planes, N, K, k), 1.0, -1.0)
    gq = g16.view(np.float16).astype(np.float64)
    hq = h16.view(np.float16).astype(np.float64)
    What = np.einsum("in,inc,ic->nc", gq, B, hq)
    assert np.allclose(dX, bf16_to_f64(dY) @ What, rtol=1e-12, atol=1e-15)
    via_t = oracle.apply(oracle.transpose_planes(planes, N, K, k), h16, g16, K, N, k, dY)
    assert np.allclose(dX, via_t, rtol=1e-12, atol=1e-15)
    Y = oracle.apply(planes, g16, h16, N, K, k, X)
    lhs = float(np.sum(bf16_to_f64(dY) * Y))
    rhs = float(np.sum(dX * bf16_to_f64(X)))
    assert math.isclose(lhs, rhs, rel_tol=1e-11, abs_tol=1e-14)


# ---------------------------------------------------------------- coupled-training gradients
def _loss_parts(W, g, h, k, X, dY):
    """Dense float64 pieces of L = <dY, X What^T> with the signs of the fp32
    recurrence (from oracle.pack through the numpy layout helpers)."""
    N, K = W.shape
    planes = oracle.pack(W, g, h, k)[0]
    S = np.where(layout.unpack_bits(planes, N, K, k), 1.0, -1.0)      # [k][N][K]
    xf, dyf = bf16_to_f64(X), bf16_to_f64(dY)

    def loss(gg, hh, xx=xf):
        What = np.einsum("in,inc,ic->nc", gg, S, hh)
        return float(np.sum(dyf * (xx @ What.T)))
    return S, xf, dyf, loss


def test_qat_gradients_match_central_differences():
    """L is linear in each g_i[n], each h_i[c], in What and in X, so central
    differences with a large step are exact up to rounding: they pin dg, dh,
    dW (= dL/dWhat, passed to the latent weight) and dX."""
    rng = np.random.default_rng(31)
    N, K, k, M = 12, 96, 3, 4
    W = (rng.standard_normal((N, K)) * 0.02).astype(np.float32)
    g, h = oracle.svid_greedy(W, k, iters=10)
    X = synth.activations(M, K, seed=2)
    dY = synth.activations(M, N, seed=3)
    st, dW, dg, dh, dX = oracle.qat_backward(W, g, h, k, X, dY)
    assert st == 0
    S, xf, dyf, loss = _loss_parts(W, g, h, k, X, dY)
    g64, h64 = g.astype(np.float64), h.astype(np.float64)
    scale = abs(loss(g64, h64)) + float(np.abs(dyf).sum() * np.abs(xf).max())
    d = 0.5
    for i, n in [(0, 0), (1, 5), (2, N - 1)]:
        e = np.zeros_like(g64)
        e[i, n] = d
        fd = (loss(g64 + e, h64) - loss(g64 - e, h64)) / (2 * d)
        assert math.isclose(dg[i, n], fd, rel_tol=1e-9, abs_tol=1e-12 * scale)
    for i, c in [(0, 0), (1, 40), (2, K - 1)]:
        e = np.zeros_like(h64)
        e[i, c] = d
        fd = (loss(g64, h64 + e) - loss(g64, h64 - e)) / (2 * d)
        assert math.isclose(dh[i, c], fd, rel_tol=1e-9, abs_tol=1e-12 * scale)
    What = np.einsum("in,inc,ic->nc", g64, S, h64)
    V = rng.standard_normal((N, K))
    fd = (np.sum(dyf * (xf @ (What + d * V).T)) - np.sum(dyf * (xf @ (What - d * V).T))) / (2 * d)
    assert math.isclose(float(np.sum(dW * V)), float(fd), rel_tol=1e-9, abs_tol=1e-12 * scale)
    U = rng.standard_normal((M, K))
    fd = (loss(g64, h64, xf + d * U) - loss(g64, h64, xf - d * U)) / (2 * d)
    assert math.isclose(float(np.sum(dX * U)), float(fd), rel_tol=1e-9, abs_tol=1e-12 * scale)


def test_qat_gradients_agree_with_the_deployment_oracle():
    """With scales exactly representable in fp16 the training-time gradients
    reach the same numbers through the stored representation: dX equals
    oracle.apply_t, and dg_i[n] = sum_m dY[m][n] * (B_i (h_i . x_m))[n], the
    latter from oracle.apply on plane i alone with unit g."""
    rng = np.random.default_rng(32)
    N, K, k, M = 32, 320, 2, 3
    W = (rng.standard_normal((N, K)) * 0.02).astype(np.float32)
    g, h = oracle.svid_greedy(W, k, iters=10)
    g = g.astype(np.float16).astype(np.float32)
    h = h.astype(np.float16).astype(np.float32)
    X = synth.activations(M, K, seed=4)
    dY = synth.activations(M, N, seed=5)
    st, _, dg, _, dX = oracle.qat_backward(W, g, h, k, X, dY)
    planes, g16, h16, st2, _ = oracle.pack(W, g, h, k)
    assert st == 0 and st2 == 0
    assert np.allclose(dX, oracle.apply_t(planes, g16, h16, N, K, k, dY), rtol=1e-12, atol=1e-15)
    per_plane = oracle.plane_words(N, K, 1)
    ones = np.full((1, N), oracle.f64_to_f16_bits(1.0), np.uint16)
    for i in range(k):
        Yi = oracle.apply(planes[i * per_plane:(i + 1) * per_plane], ones, h16[i:i + 1], N, K, 1, X)
        want = np.sum(bf16_to_f64(dY) * Yi, axis=0)
        assert np.allclose(dg[i], want, rtol=1e-12, atol=1e-15)


def test_qat_forward_is_the_adjoint_of_the_pinned_backward_and_the_deployment_apply():
    """The coupled-training forward (RaBiT, Algorithm 2 forward: signs derived
    from W on the fly, fp32 scales) is pinned three ways:
      * adjoint: <dY, Y(X)> = <dX, X> with dX from oracle.qat_backward, which is
        itself pinned by exact central differences;
      * with scales exactly representable in fp16 it equals oracle.apply of the
        packed planes (the deployment path);
      * rows and tokens selected by index give the same numbers as the full run.
    A dropped sign, a swapped scale index or a transposed X fails one of them."""
    rng = np.random.default_rng(41)
    N, K, k, M = 40, 288, 3, 5
    W = (rng.standard_normal((N, K)) * 0.02).astype(np.float32)
    W[rng.random((N, K)) < 0.02] = 0.0
    g, h = oracle.svid_greedy(W, k, iters=8)
    X = synth.activations(M, K, seed=6)
    dY = synth.activations(M, N, seed=7)
    st, Y = oracle.qat_forward(W, g, h, k, X)
    assert st == 0 and Y.shape == (M, N)
    st, _, _, _, dX = oracle.qat_backward(W, g, h, k, X, dY)
    lhs = float(np.sum(bf16_to_f64(dY) * Y))
    rhs = float(np.sum(dX * bf16_to_f64(X)))
    assert abs(lhs - rhs) <= 1e-12 * max(1.0, abs(lhs))
    g16e = g.astype(np.float16).astype(np.float32)
    h16e = h.astype(np.float16).astype(np.float32)
    _, Ye = oracle.qat_forward(W, g16e, h16e, k, X)
    planes, g16, h16, st2, _ = oracle.pack(W, g16e, h16e, k)
    assert st2 == 0
    assert np.allclose(Ye, oracle.apply(planes, g16, h16, N, K, k, X), rtol=1e-12, atol=1e-15)
    rows, toks = np.array([0, 7, 39]), np.array([4, 1])
    _, Ys = oracle.qat_forward(W, g, h, k, X, rows=rows, toks=toks)
    assert np.array_equal(Ys, Y[np.ix_(toks, rows)])
