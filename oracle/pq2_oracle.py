"""Plain FP64 oracle for the plain-ternary PQ2_0 block format.

TEST INFRASTRUCTURE ONLY -- never called by the product path.

What it follows
---------------
The WAL2-Ternary-27B card (section on bit widths) describes the format of
its fast native GGUF: PQ2_0 keeps 32 bytes of 2-bit codes plus a 2-byte FP16
scale for every 128 weights, 34 bytes or 2.125 bits per ternary weight, and
uses three of the four codes.  The weight is the scale times the trit:

    W[n, 128 g + j] = d[n, g] * T[n, 128 g + j],   y = W x.

This is the plain-ternary case of the direct-packed product (no residual
sites, no WALB2 pair) with the scale and the codes of a group stored side by
side.

Readings where the page is silent (each one is listed in the design notes):
* a block is the FP16 scale d (2 bytes, little endian) followed by its 32
  code bytes, the scale first as in GGUF's other block types;
* trit j of a block sits in code byte j // 4 at bits 2 (j % 4), code
  c = t + 1 (0 -> -1, 1 -> 0, 2 -> +1), code 3 reserved: the code and trit
  order of layout v1 of the direct-packed product;
* the G = K / 128 blocks of a row follow each other and rows follow each
  other: block (n, g) starts at byte 34 (n G + g);
* the buffer is zero-padded to a multiple of 16 bytes.

Every float is widened exactly (fp16 / bf16 -> float64) and W is formed
densely in float64; Y = X W^T is one float64 matrix product.
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np

from .wal_oracle import FormatError, GROUP, widen_bf16, widen_fp16

BLOCK_BYTES = 34
# byte offsets inside a block (module constants so the pins can be checked
# against planted mistakes)
SCALE_AT = 0
CODES_AT = 2


@dataclass
class Pq2:
    """Dense description of one PQ2_0 matrix: T int8 [N, K], d uint16 fp16 bits [N, G]."""
    N: int
    K: int
    T: np.ndarray
    d: np.ndarray


def _check(N, K):
    if N <= 0 or K <= 0 or K % GROUP:
        raise FormatError(f"bad shape N={N} K={K} (K must be a positive multiple of 128)")


def payload_bytes(N: int, K: int) -> int:
    _check(N, K)
    return N * (K // GROUP) * BLOCK_BYTES


def packed_bytes(N: int, K: int) -> int:
    return (payload_bytes(N, K) + 15) // 16 * 16


def pack(p: Pq2) -> np.ndarray:
    """Dense T and d -> the PQ2_0 byte buffer (uint8, zero-padded)."""
    N, K = p.N, p.K
    _check(N, K)
    G = K // GROUP
    T = np.asarray(p.T)
    if T.shape != (N, K) or T.min(initial=0) < -1 or T.max(initial=0) > 1:
        raise FormatError("T must be [N, K] with values in {-1, 0, +1}")
    code = (T.astype(np.int64) + 1).reshape(N, G, 32, 4)
    code_bytes = (code[..., 0] | (code[..., 1] << 2) | (code[..., 2] << 4) | (code[..., 3] << 6)).astype(np.uint8)
    d = np.asarray(p.d, dtype=np.uint16).reshape(N, G)
    blocks = np.zeros((N, G, BLOCK_BYTES), np.uint8)
    blocks[:, :, SCALE_AT] = (d & 0xFF).astype(np.uint8)
    blocks[:, :, SCALE_AT + 1] = (d >> 8).astype(np.uint8)
    blocks[:, :, CODES_AT:CODES_AT + 32] = code_bytes
    out = np.zeros(packed_bytes(N, K), np.uint8)
    out[: blocks.size] = blocks.reshape(-1)
    return out


def unpack(buf, N: int, K: int) -> Pq2:
    """PQ2_0 bytes -> dense T and d.  Raises FormatError on a wrong size,
    nonzero padding or the reserved code 3."""
    _check(N, K)
    G = K // GROUP
    raw = np.frombuffer(np.ascontiguousarray(buf).tobytes(), dtype=np.uint8)
    if raw.size != packed_bytes(N, K):
        raise FormatError(f"buffer has {raw.size} bytes, expected {packed_bytes(N, K)}")
    used = payload_bytes(N, K)
    if np.any(raw[used:]):
        raise FormatError("nonzero padding")
    blocks = raw[:used].reshape(N, G, BLOCK_BYTES)
    d = blocks[:, :, SCALE_AT].astype(np.uint16) | (blocks[:, :, SCALE_AT + 1].astype(np.uint16) << 8)
    cb = blocks[:, :, CODES_AT:CODES_AT + 32].astype(np.int64)
    code = np.stack([(cb >> (2 * i)) & 3 for i in range(4)], axis=3)  # [N, G, 32, 4]
    if np.any(code == 3):
        raise FormatError("reserved trit code 3")
    T = (code.reshape(N, K) - 1).astype(np.int8)
    return Pq2(N, K, T, d.astype(np.uint16))


def dense_weight(p: Pq2, rows=None) -> np.ndarray:
    """Dense float64 W[n, 128 g + j] = d[n, g] * T[n, 128 g + j] for the given rows."""
    rows = np.arange(p.N) if rows is None else np.asarray(rows)
    d = widen_fp16(np.asarray(p.d).reshape(p.N, p.K // GROUP)[rows])
    return np.repeat(d, GROUP, axis=1) * np.asarray(p.T)[rows].astype(np.float64)


def matmul_rows(p: Pq2, X_bits, rows) -> np.ndarray:
    """Y[m, i] = sum_j W[rows[i], j] x_m[j] in float64; X_bits bf16 [M, K]."""
    X = widen_bf16(np.asarray(X_bits).reshape(-1, p.K))
    return X @ dense_weight(p, rows).T


def matmul(p: Pq2, X_bits) -> np.ndarray:
    return matmul_rows(p, X_bits, np.arange(p.N))
