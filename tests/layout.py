"""Numpy view of the packed sign-plane storage layout (test helper).

The layout (shared definition of the C-ABI and the oracle; stated in
``include/rbw.h``): plane i is cut into S = ceil(K/256) column slices, rows are
grouped in quads (Nq = ceil(N/4)), and the uint32 word

    word(i, s, r, w) = (((i*S + s)*Nq + r//4)*8 + w)*4 + r%4

holds columns 256*s + 32*w .. +31 of row r, column c at bit c % 32, bit = 1
meaning B = +1.  Padding bits/words are zero.

These helpers express that layout with numpy reshapes and ``np.packbits`` so
tests can check the oracle's packer against it and gather rows of a GPU
result.
"""
import numpy as np


def dims(N, K):
    return (K + 255) // 256, (N + 3) // 4


def pack_bits(B):
    """bool [k][N][K] (True = +1) -> uint32 words in the storage layout."""
    B = np.asarray(B, bool)
    k, N, K = B.shape
    S, Nq = dims(N, K)
    P = np.zeros((k, Nq * 4, S * 256), bool)
    P[:, :N, :K] = B
    P = P.reshape(k, Nq, 4, S, 8, 32).transpose(0, 3, 1, 4, 2, 5)  # k,S,Nq,8,4,32
    by = np.packbits(P, axis=-1, bitorder="little")                  # k,S,Nq,8,4,4 bytes
    return np.ascontiguousarray(by).view("<u4").reshape(-1)


def unpack_bits(words, N, K, k):
    """Inverse of pack_bits (padding dropped): bool [k][N][K]."""
    S, Nq = dims(N, K)
    w = np.ascontiguousarray(np.asarray(words, np.uint32)).reshape(k, S, Nq, 8, 4)
    by = w.view(np.uint8).reshape(k, S, Nq, 8, 4, 4)
    bits = np.unpackbits(by, axis=-1, bitorder="little").astype(bool)  # k,S,Nq,8,4,32
    full = bits.transpose(0, 2, 4, 1, 3, 5).reshape(k, Nq * 4, S * 256)
    return full[:, :N, :K]


def padding_words_and_bits(words, N, K, k):
    """All bits that must be zero (columns >= K, rows >= N) as a flat bool array."""
    S, Nq = dims(N, K)
    w = np.ascontiguousarray(np.asarray(words, np.uint32)).reshape(k, S, Nq, 8, 4)
    by = w.view(np.uint8).reshape(k, S, Nq, 8, 4, 4)
    bits = np.unpackbits(by, axis=-1, bitorder="little").astype(bool)
    full = bits.transpose(0, 2, 4, 1, 3, 5).reshape(k, Nq * 4, S * 256)
    pad = np.ones_like(full)
    pad[:, :N, :K] = False
    return full[pad]


def gather_rows(words, N, K, k, rows):
    """uint32 [len(rows)][k][S][8] words of the listed rows (row-local order)."""
    S, Nq = dims(N, K)
    w = np.asarray(words, np.uint32).reshape(k, S, Nq, 8, 4)
    rows = np.asarray(rows, np.int64)
    out = w[:, :, rows // 4, :, rows % 4]          # -> len(rows), k, S, 8 (advanced idx first)
    return np.ascontiguousarray(out)
