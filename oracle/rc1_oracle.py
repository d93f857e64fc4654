"""Plain FP64 oracle for the RC1 storage of the direct-packed product.

TEST INFRASTRUCTURE ONLY -- never called by the product path.

What it follows
---------------
The WAL-Ternary-27B-RC1 card ("Representation") describes the matrices as
W ~ T3 + sparse + WALB2 with:
* the ternary base and the role-dependent k0/k2/k4/k8 sparse lane of the
  direct-packed product;
* WALB2 as two packed binary low-rank residual paths;
* body scales in a documented 24-bit float storage format that the prepared
  compute cache decodes to FP32 (the card stresses that the model is not
  "FP24": only the scales use it).
The prepared cache "keeps ternary and binary codes packed, expands 24-bit
scales to FP32" (same card, on building the cache).

    W = alpha (x) T + beta (x) R + U1 diag(s1) V1^T + U2 diag(s2) V2^T

Readings where the card is silent (each one is listed in the design notes;
the storage ABI it points to, docs/FORMAT.md, is not among the pages):
* a 24-bit float is the upper three bytes of an IEEE FP32 (sign, 8-bit
  exponent, 15 mantissa bits), stored little endian; decoding appends eight
  zero bits;
* alpha, beta, s1 and s2 all use it; alpha and beta are per (row, 128-group),
  interleaved {alpha, beta} per group when k > 0, alpha only when k = 0;
* each path is a WALB2 pair with its own rank r_p and per-rank scales, in the
  bit layout of layout v1 (u_bits [N][ceil(r_p/32)], v_bits [r_p][K/32],
  set bit = -1); r1 + r2 <= 32;
* the prepared matrix concatenates the paths into one rank block, path 1's
  ranks first: U = [U1 U2], V = [V1 V2], s = [s1 s2], and expands every scale
  to FP32 (the layout-v1 planes with FP32 in place of FP16).

Every value is widened exactly to float64 and W is formed densely; Y = X W^T
is one float64 matrix product.
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np

from .wal_oracle import FormatError, GROUP, widen_bf16

# bits appended by the decoder (a module constant so a planted mistake can change it)
F24_SHIFT = 8


def f24_to_f64(b) -> np.ndarray:
    """uint8 [..., 3] little-endian 24-bit floats -> float64, exactly."""
    b = np.asarray(b, dtype=np.uint32)
    u = b[..., 0] | (b[..., 1] << 8) | (b[..., 2] << 16)
    return (u << np.uint32(F24_SHIFT)).astype(np.uint32).view(np.float32).astype(np.float64)


def f24_to_f32_bits(b) -> np.ndarray:
    b = np.asarray(b, dtype=np.uint32)
    return ((b[..., 0] | (b[..., 1] << 8) | (b[..., 2] << 16)) << np.uint32(F24_SHIFT)).astype(np.uint32)


@dataclass
class Rc1:
    """Dense RC1 matrix: T int8 [N, K]; site_pos uint8 / site_sign int8 [N, G, k];
    alpha24, beta24 uint8 [N, G, 3]; per path p in (1, 2): U_p int8 [N, r_p],
    V_p int8 [K, r_p], s_p uint8 [r_p, 3]."""
    N: int
    K: int
    k: int
    T: np.ndarray
    site_pos: np.ndarray
    site_sign: np.ndarray
    alpha24: np.ndarray
    beta24: np.ndarray
    U1: np.ndarray
    V1: np.ndarray
    s1: np.ndarray
    U2: np.ndarray
    V2: np.ndarray
    s2: np.ndarray

    @property
    def r1(self):
        return int(np.asarray(self.U1).shape[1])

    @property
    def r2(self):
        return int(np.asarray(self.U2).shape[1])


def dense_weight(c: Rc1, rows=None) -> np.ndarray:
    """Dense float64 W for the given rows, straight from the definition."""
    N, K, k = c.N, c.K, c.k
    G = K // GROUP
    rows = np.arange(N) if rows is None else np.asarray(rows)
    n = rows.size
    alpha = f24_to_f64(np.asarray(c.alpha24).reshape(N, G, 3)[rows])
    W = np.repeat(alpha, GROUP, axis=1) * np.asarray(c.T)[rows].astype(np.float64)
    if k:
        beta = f24_to_f64(np.asarray(c.beta24).reshape(N, G, 3)[rows])
        R = np.zeros((n, K))
        pos = np.asarray(c.site_pos).reshape(N, G, k)[rows].astype(np.int64)
        sgn = np.asarray(c.site_sign).reshape(N, G, k)[rows].astype(np.float64)
        col = pos + (GROUP * np.arange(G))[None, :, None]
        rr = np.broadcast_to(np.arange(n)[:, None, None], col.shape)
        np.add.at(R, (rr.reshape(-1), col.reshape(-1)), sgn.reshape(-1))
        W += np.repeat(beta, GROUP, axis=1) * R
    for U, V, s in ((c.U1, c.V1, c.s1), (c.U2, c.V2, c.s2)):
        if np.asarray(U).shape[1]:
            sv = f24_to_f64(np.asarray(s).reshape(-1, 3))
            W += (np.asarray(U)[rows].astype(np.float64) * sv[None, :]) @ np.asarray(V).astype(np.float64).T
    return W


def matmul_rows(c: Rc1, X_bits, rows) -> np.ndarray:
    X = widen_bf16(np.asarray(X_bits).reshape(-1, c.K))
    return X @ dense_weight(c, rows).T


def matmul(c: Rc1, X_bits) -> np.ndarray:
    return matmul_rows(c, X_bits, np.arange(c.N))


# ---------------------------------------------------------------------------
# canonical RC1 scale planes and the prepared (expanded) buffers
# ---------------------------------------------------------------------------

def _pad16(a) -> np.ndarray:
    b = np.ascontiguousarray(a).reshape(-1).view(np.uint8)
    out = np.zeros((b.size + 15) // 16 * 16, np.uint8)
    out[: b.size] = b
    return out


def scales24_plane(c: Rc1) -> np.ndarray:
    """The 24-bit scale plane: {alpha, beta} per (row, group) as 6 bytes
    (k > 0) or alpha as 3 bytes (k = 0), zero-padded to 16 bytes."""
    N, G = c.N, c.K // GROUP
    a = np.asarray(c.alpha24, np.uint8).reshape(N, G, 3)
    if c.k:
        return _pad16(np.concatenate([a, np.asarray(c.beta24, np.uint8).reshape(N, G, 3)], axis=2))
    return _pad16(a)


def _ubits(U) -> np.ndarray:
    U = np.asarray(U)
    N, r = U.shape
    out = np.zeros((N, (r + 31) // 32), np.uint32)
    for rho in range(r):
        out[:, rho // 32] |= (U[:, rho] < 0).astype(np.uint32) << np.uint32(rho % 32)
    return out


def _vbits(V) -> np.ndarray:
    V = np.asarray(V)
    K, r = V.shape
    if not r:
        return np.zeros((0, K // 32), np.uint32)
    neg = (V.T < 0).astype(np.uint32).reshape(r, K // 32, 32)
    return np.bitwise_or.reduce(neg << np.arange(32, dtype=np.uint32), axis=2).astype(np.uint32)


def path_planes(U, V, s):
    """One path in the layout-v1 bit planes: (u_bits, v_bits, s24 bytes), each zero-padded."""
    return _pad16(_ubits(U)), _pad16(_vbits(V)), _pad16(np.asarray(s, np.uint8).reshape(-1, 3))


def prepared(c: Rc1):
    """The prepared matrix's scale and low-rank buffers: (scales32 [N][G][2|1]
    fp32, u_bits [N][ceil(r/32)], v_bits [r][K/32], lr32 [r] fp32) with
    r = r1 + r2, path 1's ranks first; each zero-padded to 16 bytes."""
    if c.r1 + c.r2 > 32:
        raise FormatError("r1 + r2 must be at most 32")
    N, G = c.N, c.K // GROUP
    a = f24_to_f32_bits(np.asarray(c.alpha24).reshape(N, G, 3))
    if c.k:
        sc = np.stack([a, f24_to_f32_bits(np.asarray(c.beta24).reshape(N, G, 3))], axis=2)
    else:
        sc = a
    U = np.concatenate([np.asarray(c.U1), np.asarray(c.U2)], axis=1)
    V = np.concatenate([np.asarray(c.V1), np.asarray(c.V2)], axis=1)
    s = np.concatenate([np.asarray(c.s1, np.uint8).reshape(-1, 3), np.asarray(c.s2, np.uint8).reshape(-1, 3)])
    return _pad16(sc.astype('<u4')), _pad16(_ubits(U)), _pad16(_vbits(V)), _pad16(f24_to_f32_bits(s).astype('<u4'))
