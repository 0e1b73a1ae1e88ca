"""Packed int4/int2 code storage.

KronQ README intro and "Model zoo": W4/W2 are stored as real packed int4 /
int2; W3 is fake-quant because 3-bit codes are not bit-packable.  The pages
give no layout; reading taken: per row, along n, codes fill uint32 words from
the least significant bits up (8 codes per word at 4 bits, 16 at 2 bits); a
ragged last word is zero-padded.
"""
from __future__ import annotations

import numpy as np


def words_per_row(n: int, bits: int) -> int:
    return -(-n * bits // 32)


def pack(codes, bits: int) -> np.ndarray:
    if bits not in (2, 4):
        raise ValueError("only 2- and 4-bit codes are packable")
    codes = np.asarray(codes, dtype=np.int64)
    m, n = codes.shape
    per = 32 // bits
    nw = words_per_row(n, bits)
    out = np.zeros((m, nw), dtype=np.uint64)
    for j in range(n):
        out[:, j // per] |= (codes[:, j].astype(np.uint64) & np.uint64(2 ** bits - 1)) << np.uint64(bits * (j % per))
    return out.astype(np.uint32)


def unpack(words, n: int, bits: int) -> np.ndarray:
    if bits not in (2, 4):
        raise ValueError("only 2- and 4-bit codes are packable")
    words = np.asarray(words, dtype=np.uint64)
    per = 32 // bits
    m = words.shape[0]
    out = np.zeros((m, n), dtype=np.uint8)
    for j in range(n):
        out[:, j] = ((words[:, j // per] >> np.uint64(bits * (j % per))) & np.uint64(2 ** bits - 1)).astype(np.uint8)
    return out
