"""Pins of the binary-codebook oracle (BTC-LLM, "Binary codebook": binary
k-means with majority-vote centroids and sign(0) = +1, dynamic codebook size;
"LUT-GEMM"; index width ceil(log2 c)).  Each check recomputes what the pages
fix with plain numpy on small inputs: nearest centroids by brute force over
+-1 dot products (Hamming distance = (16 - dot) / 2), majorities by counting,
the most frequent patterns by sorting, the dense product of the
reconstructed matrix by a matmul."""
import numpy as np
import pytest

import oracle
from residual_binarized_weight_b200 import synth


def bits16(p):
    """+-1 float64 [..., 16] of 16-bit patterns (bit q -> column q)."""
    p = np.asarray(p, np.uint32)
    return np.where((p[..., None] >> np.arange(16)) & 1, 1.0, -1.0)


def layer(N, K, k, seed):
    rng = np.random.default_rng(seed)
    W = (rng.standard_normal((N, K)) * 0.02).astype(np.float32)
    g, h = oracle.svid_greedy(W, k, iters=4)
    planes, g16, h16, _, _ = oracle.pack(W, g, h, k)
    return planes, g16, h16


def skewed_planes(N, K, seed, n_protos=6, flip=0.08):
    """Planes whose 16-column groups cluster around a few prototypes (so the
    codebook is smaller than the set of distinct patterns)."""
    rng = np.random.default_rng(seed)
    protos = rng.integers(0, 65536, n_protos)
    pick = protos[rng.integers(0, n_protos, (N, K // 16))]
    noise = (rng.random((N, K // 16, 16)) < flip) << np.arange(16)
    pat = (pick ^ noise.sum(-1)).astype(np.uint16)
    B = bits16(pat).reshape(N, K)
    W = (B * (0.5 + rng.random((N, K)))).astype(np.float32) * 0.02
    g, h = oracle.svid_greedy(W, 1, iters=4)
    planes, g16, h16, _, _ = oracle.pack(W, g, h, 1)
    assert np.array_equal(oracle.btc_patterns(planes, N, K, 1, 0), pat)   # sign(W) = B: one plane reproduces it
    return planes, g16, h16, pat


def test_hamming_is_the_pm1_dot_distance():
    """The identity the assignment step relies on: for +-1 vectors of length
    16, dot(a, b) = 16 - 2 popcount(a xor b)."""
    rng = np.random.default_rng(0)
    a, b = rng.integers(0, 65536, 500), rng.integers(0, 65536, 500)
    dot = (bits16(a) * bits16(b)).sum(-1)
    pop = np.array([bin(int(x) ^ int(y)).count("1") for x, y in zip(a, b)])
    assert np.array_equal(dot, 16 - 2 * pop)


def test_patterns_are_the_plane_bits():
    """btc_patterns reads the 16-column groups of the plane: the +-1 matrix
    they spell is sign(R_0) = sign(W) for plane 0."""
    rng = np.random.default_rng(1)
    N, K = 37, 96
    W = (rng.standard_normal((N, K)) * 0.02).astype(np.float32)
    g, h = oracle.svid_greedy(W, 1, iters=2)
    planes, _, _, _, _ = oracle.pack(W, g, h, 1)
    pat = oracle.btc_patterns(planes, N, K, 1, 0)
    assert np.array_equal(bits16(pat).reshape(N, K), np.where(W >= 0, 1.0, -1.0))


def test_initial_codebook_is_the_most_frequent_patterns():
    planes, _, _, pat = skewed_planes(64, 256, seed=2)
    u, cnt = np.unique(pat, return_counts=True)
    order = np.lexsort((u, -cnt))                     # count descending, then pattern ascending
    for c_max in (1, 5, 17):
        cb, c, _, _ = oracle.btc_encode(planes, 64, 256, 1, 0, c_max, iters=0)
        assert c == min(c_max, len(u))
        assert np.array_equal(cb[:c], u[order[:c]])
        assert not cb[c:].any()


@pytest.mark.parametrize("c_max,iters", [(3, 1), (6, 4), (9, 7)])
def test_assignment_is_nearest_and_centroids_are_majorities(c_max, iters):
    N, K = 48, 192
    planes, _, _, pat = skewed_planes(N, K, seed=c_max)
    cb, c, idx, obj = oracle.btc_encode(planes, N, K, 1, 0, c_max, iters)
    d = (16 - bits16(pat) @ bits16(cb[:c]).T) / 2    # Hamming distance of every vector to every centroid
    nearest = np.argmin(d, axis=-1)                  # first minimum: ties to the smaller index
    assert np.array_equal(idx, nearest)
    assert obj[-1] == pytest.approx(float(np.take_along_axis(d, idx[..., None].astype(np.int64), -1).sum()))
    assert np.all(np.diff(obj) <= 1e-9)              # each round can only lower the total distance
    # the next round's centroids are the majorities of this assignment's members
    cb2, _, _, _ = oracle.btc_encode(planes, N, K, 1, 0, c_max, iters + 1)
    vec = bits16(pat).reshape(-1, 16)
    for p in range(c):
        mem = vec[idx.reshape(-1) == p]
        if len(mem) == 0:
            assert cb2[p] == cb[p]
        else:
            want = int(((mem.sum(0) >= 0) << np.arange(16)).sum())
            assert cb2[p] == want


def test_codebook_is_exact_when_it_holds_every_pattern():
    """Dynamic size: with c_max >= the number of distinct patterns the
    codebook holds them all, the layer is reproduced bit for bit and the
    LUT application equals the plane application exactly."""
    N, K, k = 40, 128, 2
    planes, g16, h16 = layer(N, K, k, seed=3)
    X = synth.activations(3, K, seed=4)
    cbs, idxs = [], []
    for i in range(k):
        pat = oracle.btc_patterns(planes, N, K, k, i)
        cb, c, idx, obj = oracle.btc_encode(planes, N, K, k, i, 65536, iters=3)
        assert c == len(np.unique(pat)) and obj[-1] == 0.0
        assert np.array_equal(cb[idx], pat)
        cbs.append(cb)
        idxs.append(idx)
    Y = oracle.btc_apply(np.stack(cbs), 65536, np.stack(idxs), g16, h16, N, K, k, X)
    assert np.array_equal(Y, oracle.apply(planes, g16, h16, N, K, k, X))


def test_btc_apply_is_the_dense_product_of_the_reconstruction():
    N, K, k, c_max = 50, 160, 2, 7
    planes, g16, h16 = layer(N, K, k, seed=5)
    X = synth.activations(4, K, seed=6)
    cbs, idxs = [], []
    for i in range(k):
        cb, c, idx, _ = oracle.btc_encode(planes, N, K, k, i, c_max, iters=3)
        cbs.append(cb)
        idxs.append(idx)
    rows = np.array([0, 7, 49, 20])
    Y = oracle.btc_apply(np.stack(cbs), c_max, np.stack(idxs), g16, h16, N, K, k, X, rows=rows)
    g = g16.view(np.float16).astype(np.float64).reshape(k, N)
    h = h16.view(np.float16).astype(np.float64).reshape(k, K)
    What = sum(g[i][:, None] * bits16(cbs[i][idxs[i]]).reshape(N, K) * h[i][None, :] for i in range(k))
    Xf = (X.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    assert np.allclose(Y, (Xf @ What.T)[:, rows], rtol=1e-12, atol=1e-14)


def test_index_stream_and_sub_one_bit_width():
    """c = 7132 (the 7B configuration of the page) needs 13-bit indices:
    13 / 16 = 0.8125 bit per weight; the stream round-trips."""
    assert oracle.btc_index_bits(7132) == 13 and oracle.btc_index_bits(65536) == 16
    assert oracle.btc_index_bits(1) == 1 and oracle.btc_index_bits(2) == 1 and oracle.btc_index_bits(3) == 2
    rng = np.random.default_rng(7)
    N, K, w = 9, 4096, 13
    idx = rng.integers(0, 7132, (N, K // 16)).astype(np.uint16)
    words = oracle.btc_pack_indices(idx, N, K, w)
    assert words.shape == (N, 104)                   # 256 indices x 13 bits = 104 words per row
    bits = np.unpackbits(words.view(np.uint8), bitorder="little").reshape(N, -1)
    got = (bits[:, :256 * w].reshape(N, 256, w).astype(np.int64) << np.arange(w)).sum(-1)
    assert np.array_equal(got, idx)
