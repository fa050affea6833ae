"""Numpy view of the packed sign-plane storage layout (test helper).

The layout (the library's storage format, stated in ``include/rbw.h``): plane
i is cut into S = ceil(K/256) column slices and Nt = ceil(N/32) tiles of 32
rows; each (plane, slice, tile) block holds 256 uint32 words and

    word(i, s, r, w) = ((i*S + s)*Nt + r//32)*256 + (w ^ ((r%32)//4))*32 + r%32

holds columns 256*s + 32*w .. +31 of row r, column c at bit c % 32, bit = 1
meaning B = +1.  Padding bits and words are zero.

These helpers express that layout with numpy reshapes, fancy indexing and
``np.packbits`` so tests can check the oracle's packer against it and gather
rows of a GPU result.
"""
import numpy as np

_RHO = np.arange(32)
_SLOT = np.arange(8)[:, None] ^ (_RHO[None, :] >> 2)   # slot <-> logical word (an involution)


def dims(N, K):
    return (K + 255) // 256, (N + 31) // 32


def pack_bits(B):
    """bool [k][N][K] (True = +1) -> uint32 words in the storage layout."""
    B = np.asarray(B, bool)
    k, N, K = B.shape
    S, Nt = dims(N, K)
    P = np.zeros((k, Nt * 32, S * 256), bool)
    P[:, :N, :K] = B
    P = P.reshape(k, Nt, 32, S, 8, 32).transpose(0, 3, 1, 4, 2, 5)    # k,S,Nt,w,rho,bit
    logical = np.ascontiguousarray(np.packbits(P, axis=-1, bitorder="little")).view("<u4")[..., 0]
    stored = logical[:, :, :, _SLOT, _RHO[None, :]]                  # slot <- word slot^(rho/4)
    return np.ascontiguousarray(stored).reshape(-1)


def _logical_words(words, N, K, k):
    S, Nt = dims(N, K)
    stored = np.asarray(words, np.uint32).reshape(k, S, Nt, 8, 32)
    return stored[:, :, :, _SLOT, _RHO[None, :]]                     # k,S,Nt,w,rho


def _all_bits(words, N, K, k):
    S, Nt = dims(N, K)
    lw = np.ascontiguousarray(_logical_words(words, N, K, k))
    by = lw.view(np.uint8).reshape(k, S, Nt, 8, 32, 4)
    bits = np.unpackbits(by, axis=-1, bitorder="little").astype(bool)   # k,S,Nt,w,rho,32
    return bits.transpose(0, 2, 4, 1, 3, 5).reshape(k, Nt * 32, S * 256)


def unpack_bits(words, N, K, k):
    """Inverse of pack_bits (padding dropped): bool [k][N][K]."""
    return _all_bits(words, N, K, k)[:, :N, :K]


def padding_words_and_bits(words, N, K, k):
    """All bits that must be zero (columns >= K, rows >= N) as a flat bool array."""
    full = _all_bits(words, N, K, k)
    pad = np.ones_like(full)
    pad[:, :N, :K] = False
    return full[pad]


def gather_rows(words, N, K, k, rows):
    """uint32 [len(rows)][k][S][8] words of the listed rows (row-local order)."""
    S, Nt = dims(N, K)
    stored = np.asarray(words, np.uint32).reshape(k, S, Nt, 8, 32)
    rows = np.asarray(rows, np.int64)
    t, rho = rows // 32, rows % 32
    slots = np.arange(8)[None, :] ^ (rho[:, None] >> 2)             # [len(rows)][8]
    out = stored[:, :, t[:, None], slots, rho[:, None]]              # -> k, S, len(rows), 8
    return np.ascontiguousarray(out.transpose(2, 0, 1, 3))
