"""Independent numpy decoder of the slot bit layout (test helper).

Written from the layout description (blocks of 128 inputs, 4 units of 32
codes, pair (even, odd) in the low/high 16-bit halves of a word; rows in
groups of 8 stored unit-major with a per-width lane permutation; gate/up rows
in blocks of 16), in a vectorised style unrelated to the oracle's per-bit C
loop, so that an index mistake in either one shows up as a mismatch.
"""
import numpy as np


def ceil128(k):
    return (k + 127) // 128 * 128


def _sigma(u, r, b):
    if b == 3:
        return r
    if b == 4:
        return (r + 2 * (u % 4)) % 8
    return (r + 4 * ((u // 2) % 2)) % 8


def _bit_positions(K, b):
    """For every input k < Kp and code bit j: (unit index u, word in unit, bit in word)."""
    Kp = ceil128(K)
    k = np.arange(Kp)
    blk, kk = k // 128, k % 128
    s, r16 = kk // 16, kk % 16
    h = r16 // 8
    p = (r16 % 8) // 2
    odd = k & 1
    i = 2 * s + h
    unit = 4 * blk + p
    U = np.zeros((Kp, b), np.int64)
    W = np.zeros((Kp, b), np.int64)
    B = np.zeros((Kp, b), np.int64)
    for j in range(b):
        if b == 4:
            wi, bi = i // 4, 4 * (i % 4) + j
        elif b == 3:
            wi = np.where(i < 15, i // 5, j)
            bi = np.where(i < 15, 3 * (i % 5) + j, 15)
        elif b == 6:
            m = i - 12
            if j < 4:
                wi = np.where(i < 12, i // 2, m)
                bi = np.where(i < 12, 6 * (i % 2) + j, 12 + j)
            else:
                wi = np.where(i < 12, i // 2, 4 + m // 2)
                bi = np.where(i < 12, 6 * (i % 2) + j, 12 + 2 * (m % 2) + (j - 4))
        else:
            raise ValueError(b)
        U[:, j] = unit
        W[:, j] = wi
        B[:, j] = bi + 16 * odd
    return U, W, B


def geometry(K, g, b):
    """(row bytes of codes, groups per row, tile bytes); b = 16 (BF16 experts)
    has no scale/bias words."""
    rb = ceil128(K) * b // 8
    ng = ceil128(K) // g
    return rb, ng, 16 * rb + (0 if b == 16 else 16 * ng * 4)


def decode_rows(proj, rows, K, g, b):
    """proj: a projection's bytes (tiles of 16 rows: codes, then scale/bias
    words) -> codes int64 [rows, K]."""
    rb, ng, tb = geometry(K, g, b)
    words = np.ascontiguousarray(proj, dtype=np.uint8).reshape(-1).view("<u4").astype(np.int64)
    U, W, B = _bit_positions(K, b)
    codes = np.zeros((rows, U.shape[0]), np.int64)
    for r in range(rows):
        grp_word = ((r // 16) * tb + ((r % 16) // 8) * 8 * rb) // 4
        for j in range(b):
            pos = 8 * U[:, j] + _sigma(U[:, j], r % 8, b)
            idx = grp_word + pos * b + W[:, j]
            codes[r] |= ((words[idx] >> B[:, j]) & 1) << j
    return codes[:, :K]


def sb_rows(proj, rows, K, g, b):
    """The (scale, bias) words of a projection as [rows, groups]."""
    rb, ng, tb = geometry(K, g, b)
    t = np.ascontiguousarray(proj, dtype=np.uint8).reshape(rows // 16, tb)[:, 16 * rb:]
    t = np.ascontiguousarray(t).view("<u4").reshape(rows // 16, ng, 16)
    return t.transpose(0, 2, 1).reshape(rows, ng)


def dequant_rows(proj, rows, K, g, b):
    """Closed form of fma(scale, q, bias) in fp32: the exact product-sum in
    float64 (exact for bf16 scale/bias and q < 64), rounded once to fp32.
    b = 16: the rows are bf16 values, row-major, each row padded to Kp."""
    if b == 16:
        v = np.ascontiguousarray(proj, dtype=np.uint8).reshape(-1).view("<u2").reshape(rows, ceil128(K))
        return (v[:, :K].astype(np.uint32) << 16).view(np.float32)
    codes = decode_rows(proj, rows, K, g, b).astype(np.float64)
    sb = sb_rows(proj, rows, K, g, b)
    s = ((sb & 0xFFFF).astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    bb = ((sb >> 16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    gi = np.arange(K) // g
    return (s[:, gi] * codes + bb[:, gi]).astype(np.float32)


def gate_up_storage_row(R, I):
    """Storage row of logical gate/up row R: blocks of 16 = 8 gate + 8 up rows."""
    j = R if R < I else R - I
    return 16 * (j // 8) + (0 if R < I else 8) + j % 8
