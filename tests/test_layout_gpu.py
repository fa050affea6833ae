"""Plain row-major packing <-> storage layout (rb_planes_from_rowmajor,
rb_planes_to_rowmajor), bit for bit against the oracle's planes.

The plain form is RaBiT's "32 columns packed into one uint32_t" read the
obvious way: words [k][N][K/32], column c at bit c % 32, bit 1 = +1.  The
expected plain words come from numpy's packbits of the sign matrix that the
oracle's planes hold (unpacked with the numpy layout helpers), never from the
library.
"""
import numpy as np
import pytest
import torch

import oracle
from residual_binarized_weight_b200 import rbw, synth
from tests import cases, layout

pytestmark = pytest.mark.gpu


def rowmajor_from_signs(B):
    """bool [k][N][K] -> uint32 [k][N][K/32], LSB first (numpy packbits)."""
    return np.ascontiguousarray(np.packbits(B, axis=-1, bitorder="little")).view("<u4")


@pytest.mark.parametrize("N,K,k", [(33, 288, 2), (100, 800, 3), (4096, 4096, 2), (257, 2080, 1), (64, 256, 8),
                                   (1, 32, 1), (4097, 544, 4)])
def test_rowmajor_round_trip_is_bit_exact(N, K, k):
    rng = np.random.default_rng(N * 7 + K + k)
    W = (rng.standard_normal((N, K)) * 0.02).astype(np.float32)
    W[rng.random((N, K)) < 0.01] = 0.0
    g, h = oracle.svid_greedy(W, k, iters=6)
    planes, g16, h16, st, _ = oracle.pack(W, g, h, k)
    assert st == 0
    B = layout.unpack_bits(planes, N, K, k)
    rm = rowmajor_from_signs(B)
    assert rm.shape == (k, N, K // 32) and rbw.rowmajor_words(N, K, k) == rm.size
    L = rbw.planes_from_rowmajor(cases.to_dev(rm.reshape(-1)), N, K, k)
    torch.cuda.synchronize()
    assert np.array_equal(cases.to_host(L.planes, np.uint32), planes)
    back = rbw.planes_to_rowmajor(cases.upload_layer(planes, g16, h16, N, K, k))
    torch.cuda.synchronize()
    assert np.array_equal(cases.to_host(back, np.uint32), rm.reshape(-1))


def test_planes_packed_elsewhere_apply_like_the_oracle():
    """A layer whose planes come from numpy's packbits of sign(R) (derived by
    the oracle's recurrence) goes through rb_planes_from_rowmajor into rb_gemv
    and matches the oracle's Y."""
    N, K, k = 1000, 2048, 2
    W, g, h = cases.layer_case(1, 0, k, N, K)
    planes, g16, h16 = cases.packed_case(1, 0, k, N, K)
    rm = rowmajor_from_signs(layout.unpack_bits(planes, N, K, k))
    L = rbw.PackedLayer(N, K, k)
    L.g16.copy_(cases.to_dev(g16).view(torch.float16))
    L.h16.copy_(cases.to_dev(h16).view(torch.float16))
    rbw.planes_from_rowmajor(cases.to_dev(rm.reshape(-1)), N, K, k, out=L)
    for M in (1, 4):
        X = synth.activations(M, K, seed=M)
        Y = rbw.gemv(L, cases.to_dev(X))
        torch.cuda.synchronize()
        Yr = oracle.apply(planes, g16, h16, N, K, k, X)
        cases.check_y(Y.cpu().numpy().astype(np.float64), Yr, cases.abs_bound(g16, h16, X), bf16=False,
                      per_elem=1e-5 if M == 1 else 1e-4)


def test_rowmajor_argument_errors():
    L = rbw.PackedLayer(64, 256, 2)
    buf = torch.zeros(rbw.packed_words(64, 256, 2) + 64, dtype=torch.int32, device="cuda")
    with pytest.raises(rbw.RbError) as e:                # overlapping buffers
        rbw.planes_from_rowmajor(buf[:rbw.rowmajor_words(64, 256, 2)], 64, 256, 2,
                                 out=type("P", (), {"planes": buf[4:]})())
    assert e.value.status == rbw.RB_ERR_ARG
    with pytest.raises(rbw.RbError) as e:
        rbw.planes_to_rowmajor(L, out=buf[1:])           # 4-byte offset
    assert e.value.status == rbw.RB_ERR_ALIGN


@pytest.mark.parametrize("N,K,k,world", [(4096, 4096, 2, 4), (300, 544, 3, 2), (11008, 4096, 2, 8), (100, 256, 1, 3)])
def test_row_shards_are_the_planes_of_the_row_ranges(N, K, k, world):
    """rb_shard_rows over a row-parallel split: each shard is bit for bit the
    oracle's packing of its rows (the recurrence is row-local), and the shards'
    outputs, concatenated along N, match the oracle's output of the whole layer."""
    rng = np.random.default_rng(N + K + k)
    W = (rng.standard_normal((N, K)) * 0.02).astype(np.float32)
    g, h = oracle.svid_greedy(W, k, iters=4)
    planes, g16, h16, _, _ = oracle.pack(W, g, h, k)
    L = cases.upload_layer(planes, g16, h16, N, K, k)
    X = synth.activations(2, K, seed=9)
    Xd = cases.to_dev(X)
    parts = []
    for r in range(world):
        r0, r1 = rbw.shard_bounds(N, world, r)
        if r1 == r0:
            continue
        Sh = rbw.shard_rows(L, r0, r1 - r0)
        torch.cuda.synchronize()
        sp, sg, _, _, _ = oracle.pack(W[r0:r1], g[:, r0:r1], h, k)
        assert np.array_equal(cases.to_host(Sh.planes, np.uint32), sp)
        assert np.array_equal(cases.to_host(Sh.g16, np.uint16).reshape(k, r1 - r0), sg)
        parts.append(rbw.gemv(Sh, Xd))
    Y = torch.cat(parts, dim=1)
    torch.cuda.synchronize()
    rows = np.unique(np.concatenate([np.arange(min(N, 64)), np.arange(max(0, N - 64), N),
                                     rng.choice(N, min(N, 200), replace=False)]))
    Yr = oracle.apply(planes, g16, h16, N, K, k, X, rows=rows)
    cases.check_y(Y.cpu().numpy().astype(np.float64)[:, rows], Yr, cases.abs_bound(g16, h16, X, rows), bf16=False,
                  per_elem=1e-4)


def test_shard_rows_argument_errors():
    L = rbw.PackedLayer(128, 256, 2)
    with pytest.raises(rbw.RbError) as e:
        rbw.shard_rows(L, 16, 32)                        # not on a 32-row tile
    assert e.value.status == rbw.RB_ERR_SHAPE
    with pytest.raises(rbw.RbError) as e:
        rbw.shard_rows(L, 96, 64)                        # past the last row
    assert e.value.status == rbw.RB_ERR_SHAPE
