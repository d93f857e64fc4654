"""Plain FP64 oracle for the INT3/g128 embedding and the INT4/g128 LM head.

TEST INFRASTRUCTURE ONLY -- never called by the product path.

What it follows
---------------
The WAL-Ternary-8B card (Kazakh README, "Model format") lists the parts of
the model around the ternary body: the embedding is INT3 with groups of 128,
the LM head INT4 with groups of 128, norms and small tensors BF16.  A decode
step gathers one embedding row per token and ends with the LM-head product.

Readings where the card is silent (each one is listed in the design notes):
* "INTb/g128": integers q with a scale d per (row, group of 128 columns),
  w = d * q; q is a b-bit two's-complement range, [-8, 7] for INT4 and
  [-4, 3] for INT3; d is FP16 (the scale type of the body's cache);
* codes are offset binary, u = q + 8 (INT4) or u = q + 4 (INT3), as in
  GGUF's 4-bit blocks;
* INT4: two codes per byte, column 2i in the low nibble of byte i and 2i + 1
  in the high nibble; a row is K / 2 bytes;
* INT3: a group of 128 codes is a 384-bit little-endian bit string of 48
  bytes, code j at bits 3j .. 3j + 2; a row is 48 * H / 128 bytes;
* scales fp16 [rows][K / 128]; every plane is zero-padded to 16 bytes;
* the LM head computes logits y = W x (FP32 out); the embedding of token t
  is e = d[t] * q[t] in FP32 (exact: an FP16 scale times a 3-bit integer).
"""
from __future__ import annotations

import numpy as np

from .wal_oracle import FormatError, GROUP, widen_bf16, widen_fp16

INT4_OFFSET = 8
INT3_OFFSET = 4
INT4_HIGH_FIRST = False  # nibble order (a module constant for a planted mistake)


def _pad16(a) -> np.ndarray:
    b = np.ascontiguousarray(a).reshape(-1).view(np.uint8)
    out = np.zeros((b.size + 15) // 16 * 16, np.uint8)
    out[: b.size] = b
    return out


def _check(N, K):
    if N <= 0 or K <= 0 or K % GROUP:
        raise FormatError(f"bad shape {N} x {K} (columns must be a positive multiple of 128)")


# ---------------------------------------------------------------------------
# INT4 LM head
# ---------------------------------------------------------------------------

def int4_pack(q, d):
    """q int8 [N, K] in [-8, 7], d fp16 bits [N, K/128] -> (codes, scales) planes."""
    q = np.asarray(q)
    N, K = q.shape
    _check(N, K)
    if q.min(initial=0) < -8 or q.max(initial=0) > 7:
        raise FormatError("INT4 values must lie in [-8, 7]")
    u = (q.astype(np.int64) + INT4_OFFSET).reshape(N, K // 2, 2)
    lo, hi = (u[..., 1], u[..., 0]) if INT4_HIGH_FIRST else (u[..., 0], u[..., 1])
    codes = (lo | (hi << 4)).astype(np.uint8)
    return _pad16(codes), _pad16(np.asarray(d, np.uint16).reshape(N, K // GROUP).astype('<u2'))


def int4_unpack(codes, scales, N, K):
    """Planes -> (q int8 [N, K], d uint16 [N, G]); FormatError on sizes or padding."""
    _check(N, K)
    c = np.frombuffer(np.ascontiguousarray(codes).tobytes(), np.uint8)
    s = np.frombuffer(np.ascontiguousarray(scales).tobytes(), np.uint8)
    nc, ns = N * K // 2, N * (K // GROUP) * 2
    if c.size != (nc + 15) // 16 * 16 or s.size != (ns + 15) // 16 * 16:
        raise FormatError("wrong plane size")
    if np.any(c[nc:]) or np.any(s[ns:]):
        raise FormatError("nonzero padding")
    b = c[:nc].reshape(N, K // 2).astype(np.int64)
    lo, hi = b & 15, b >> 4
    first, second = (hi, lo) if INT4_HIGH_FIRST else (lo, hi)
    q = np.stack([first, second], axis=2).reshape(N, K) - INT4_OFFSET
    return q.astype(np.int8), s[:ns].view('<u2').reshape(N, K // GROUP).copy()


def int4_dense(q, d, rows=None) -> np.ndarray:
    q = np.asarray(q)
    N, K = q.shape
    rows = np.arange(N) if rows is None else np.asarray(rows)
    dd = widen_fp16(np.asarray(d).reshape(N, K // GROUP)[rows])
    return np.repeat(dd, GROUP, axis=1) * q[rows].astype(np.float64)


def int4_matmul_rows(q, d, X_bits, rows) -> np.ndarray:
    q = np.asarray(q)
    X = widen_bf16(np.asarray(X_bits).reshape(-1, q.shape[1]))
    return X @ int4_dense(q, d, rows).T


def int4_matmul(q, d, X_bits) -> np.ndarray:
    return int4_matmul_rows(q, d, X_bits, np.arange(np.asarray(q).shape[0]))


# ---------------------------------------------------------------------------
# INT3 embedding
# ---------------------------------------------------------------------------

def int3_pack(q, d):
    """q int8 [V, H] in [-4, 3], d fp16 bits [V, H/128] -> (codes, scales) planes."""
    q = np.asarray(q)
    V, H = q.shape
    _check(V, H)
    if q.min(initial=0) < -4 or q.max(initial=0) > 3:
        raise FormatError("INT3 values must lie in [-4, 3]")
    u = (q.astype(np.int64) + INT3_OFFSET).reshape(V, H // GROUP, GROUP)
    bits = ((u[..., None] >> np.arange(3)) & 1).reshape(V, H // GROUP, 3 * GROUP)  # bit 3j + i = bit i of code j
    codes = np.packbits(bits.astype(np.uint8), axis=2, bitorder="little")  # 48 bytes per group
    return _pad16(codes), _pad16(np.asarray(d, np.uint16).reshape(V, H // GROUP).astype('<u2'))


def int3_unpack(codes, scales, V, H):
    _check(V, H)
    c = np.frombuffer(np.ascontiguousarray(codes).tobytes(), np.uint8)
    s = np.frombuffer(np.ascontiguousarray(scales).tobytes(), np.uint8)
    nc, ns = V * H * 3 // 8, V * (H // GROUP) * 2
    if c.size != (nc + 15) // 16 * 16 or s.size != (ns + 15) // 16 * 16:
        raise FormatError("wrong plane size")
    if np.any(c[nc:]) or np.any(s[ns:]):
        raise FormatError("nonzero padding")
    bits = np.unpackbits(c[:nc].reshape(V, H // GROUP, 48), axis=2, bitorder="little").astype(np.int64)
    u = (bits.reshape(V, H // GROUP, GROUP, 3) << np.arange(3)).sum(axis=3)
    return (u.reshape(V, H) - INT3_OFFSET).astype(np.int8), s[:ns].view('<u2').reshape(V, H // GROUP).copy()


def int3_embed(q, d, ids) -> np.ndarray:
    """Rows of the dequantised table for the token ids: float64 [M, H]."""
    q = np.asarray(q)
    V, H = q.shape
    ids = np.asarray(ids).reshape(-1)
    if np.any(ids < 0) or np.any(ids >= V):
        raise FormatError("token id out of range")
    dd = widen_fp16(np.asarray(d).reshape(V, H // GROUP)[ids])
    return np.repeat(dd, GROUP, axis=1) * q[ids].astype(np.float64)
