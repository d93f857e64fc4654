"""Plain oracle for the base-3 container and its conversion to layout v1.

TEST INFRASTRUCTURE ONLY -- never called by the product path.

What it follows
---------------
The WAL2-Ternary-27B card (section on bit widths) describes the base
container: a trit has three values (information bound log2 3 = 1.585 bits);
five trits are written into one byte, 8 / 5 = 1.6 bits per symbol before
scales and exceptions, and a BF16 scale per 128 weights adds 16 / 128 =
0.125 bits.  Before inference the runtime converts the canonical archive
into the compute layout (WAL-Ternary-27B-RC1 card, on the prepared cache:
the codes stay packed, scales are expanded to the kernels' format).

Readings where the pages are silent (each one is listed in the design notes):
* digit d = t + 1 in {0, 1, 2}; byte m of a row holds trits 5m .. 5m + 4 as
  sum_i d_i 3^i (trit 5m + i is digit i, the least significant first);
  bytes 243 .. 255 are invalid;
* each row starts on a byte: ceil(K / 5) bytes per row, rows back to back;
  digits past the row's last trit are 0 (the pages' 1.6 bits per symbol
  is the rate of a continuous stream; per row it costs at most one byte);
* the buffer is zero-padded to a multiple of 16 bytes;
* the BF16 scale of (row n, group g) becomes alpha of layout v1 (k = 0) by
  IEEE round-to-nearest-even to FP16; a scale that is not finite, or whose
  FP16 value is not finite, is a format error.

The conversion target is the layout-v1 code plane (code c = t + 1, trit j of
a row in 32-bit word j / 16 at bits 2 (j % 16)) and the k = 0 scale plane
(fp16 alpha [N][G]), each zero-padded to 16 bytes.
"""
from __future__ import annotations

import numpy as np

from .wal_oracle import FormatError, GROUP

# digit order inside a byte (a module constant so the pins can be checked
# against a planted mistake)
DIGIT_WEIGHTS = (1, 3, 9, 27, 81)


def _check(N, K):
    if N <= 0 or K <= 0 or K % GROUP:
        raise FormatError(f"bad shape N={N} K={K} (K must be a positive multiple of 128)")


def row_bytes(K: int) -> int:
    return (K + 4) // 5


def packed_bytes(N: int, K: int) -> int:
    _check(N, K)
    return (N * row_bytes(K) + 15) // 16 * 16


def pack(T) -> np.ndarray:
    """T int8 [N, K] in {-1, 0, 1} -> base-3 bytes (uint8, zero-padded)."""
    T = np.asarray(T)
    N, K = T.shape
    _check(N, K)
    if T.min(initial=0) < -1 or T.max(initial=0) > 1:
        raise FormatError("T must hold values in {-1, 0, +1}")
    P = row_bytes(K)
    d = np.zeros((N, 5 * P), np.int64)
    d[:, :K] = T.astype(np.int64) + 1
    d = d.reshape(N, P, 5)
    v = sum(d[:, :, i] * DIGIT_WEIGHTS[i] for i in range(5))
    out = np.zeros(packed_bytes(N, K), np.uint8)
    out[: N * P] = v.astype(np.uint8).reshape(-1)
    return out


def unpack(buf, N: int, K: int) -> np.ndarray:
    """Base-3 bytes -> T int8 [N, K].  Raises FormatError on a wrong size, a
    byte above 242, a nonzero digit past the row's end or nonzero padding."""
    _check(N, K)
    raw = np.frombuffer(np.ascontiguousarray(buf).tobytes(), dtype=np.uint8)
    if raw.size != packed_bytes(N, K):
        raise FormatError(f"buffer has {raw.size} bytes, expected {packed_bytes(N, K)}")
    P = row_bytes(K)
    if np.any(raw[N * P:]):
        raise FormatError("nonzero padding")
    v = raw[: N * P].reshape(N, P).astype(np.int64)
    if np.any(v > 242):
        raise FormatError("byte above 242")
    digits = np.stack([(v // w) % 3 for w in DIGIT_WEIGHTS], axis=2).reshape(N, 5 * P)
    if np.any(digits[:, K:]):
        raise FormatError("nonzero digit past the end of a row")
    return (digits[:, :K] - 1).astype(np.int8)


def bf16_to_fp16_bits(s_bits) -> np.ndarray:
    """BF16 bit patterns -> FP16 bit patterns by IEEE round-to-nearest-even
    (bf16 widens exactly to float32; numpy's float32 -> float16 cast rounds
    to nearest even).  FormatError when an input or a result is not finite."""
    f = (np.ascontiguousarray(s_bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)
    if not np.all(np.isfinite(f)):
        raise FormatError("scale is not finite")
    with np.errstate(over="ignore"):
        h = f.astype(np.float16)
    if not np.all(np.isfinite(h)):
        raise FormatError("scale overflows FP16")
    return h.view(np.uint16)


def convert(buf, scales_bf16, N: int, K: int):
    """The prepare step: base-3 bytes + BF16 scales [N][G] -> (layout-v1 code
    plane bytes, fp16 alpha plane bytes), each zero-padded to 16 bytes."""
    T = unpack(buf, N, K)
    code = (T.astype(np.uint32) + 1).reshape(N, K // 16, 16)
    words = np.bitwise_or.reduce(code << (2 * np.arange(16, dtype=np.uint32)), axis=2).astype('<u4')
    codes = np.zeros((N * K // 4 + 15) // 16 * 16, np.uint8)
    codes[: N * K // 4] = words.reshape(-1).view(np.uint8)
    G = K // GROUP
    alpha = bf16_to_fp16_bits(np.asarray(scales_bf16).reshape(N, G)).astype('<u2')
    aplane = np.zeros((N * G * 2 + 15) // 16 * 16, np.uint8)
    aplane[: N * G * 2] = alpha.reshape(-1).view(np.uint8)
    return codes, aplane
