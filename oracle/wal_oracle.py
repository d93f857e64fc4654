"""Plain, slow FP64 oracle for y = (alpha*T + beta*R) x + sum_r U_r (V_r^T x).

TEST INFRASTRUCTURE ONLY -- never called by the product path.

What it follows
---------------
* The matrix model is the one printed on the WAL-Ternary-8B model card
  (section "Representation") and its Kazakh README (section "Model format"):
  W(x) = (alpha*T + beta*R) x + sum_r U_r (V_r^T x), T in {-1, 0, +1},
  R = exactly k signed residual sites per group of 128 weights.
* k may be 0, 2, 4 or 8 ("role- and depth-dependent k0/k2/k4/k8 corrections
  per group of 128 weights": WAL-Ternary-27B-RC1 card, "Representation").
* alpha and beta are FP16 per (output row, 128-group): FP16 scales are what
  the executable cache stores (WAL-Ternary-8B card, "Install": the cache
  holds packed ternary symbols, sparse positions/signs and FP16 scales); the
  group of 128 is the scale group of the WAL2-Ternary-27B card
  ("Архитектура").
* 2-bit codes, 32 bytes per 128 weights, three of the four codes used:
  PQ2_0 as described on the WAL2-Ternary-27B card ("Что означает битность").

Readings where the pages are silent (layout v1; each one is listed with its
reason in the design notes):
* code c = t + 1 (0 -> -1, 1 -> 0, 2 -> +1); code 3 is reserved and rejected.
* trit j of a row sits in 32-bit word j // 16 at bits 2*(j % 16), little endian.
* site byte = position (bits 0..6) | 0x80 if the sign is -1; exactly k distinct
  positions per group, stored ascending.  A site may coincide with a nonzero
  trit; both terms then add.
* k == 0 groups store alpha only; beta does not exist.
* WALB2: y += sum_r s_r * U[:, r] * (V[:, r]^T x) with one FP16 scale s_r per
  rank; U, V in {+1, -1}; a set bit means -1.  U is stored as
  u32[N][ceil(r/32)], V as u32[r][K/32].
* every buffer is zero-padded to a multiple of 16 bytes.

Every float is widened exactly (fp16 / bf16 -> float64) and W is formed
densely in float64; y = W x is one float64 matrix product.  There is no
blocking, fusion or reordering beyond that definition.
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np

GROUP = 128
VALID_K = (0, 2, 4, 8)
MAX_RANK = 32


class FormatError(ValueError):
    """Raised for any buffer that is not a valid layout-v1 matrix."""


# ---------------------------------------------------------------------------
# exact widening
# ---------------------------------------------------------------------------

def widen_fp16(bits) -> np.ndarray:
    """fp16 bit patterns -> float64, exactly (subnormals kept)."""
    return np.ascontiguousarray(bits, dtype=np.uint16).view(np.float16).astype(np.float64)


def widen_bf16(bits) -> np.ndarray:
    """bf16 bit patterns -> float64, exactly."""
    u = np.ascontiguousarray(bits, dtype=np.uint16).astype(np.uint32) << 16
    return u.view(np.float32).astype(np.float64)


# ---------------------------------------------------------------------------
# sizes
# ---------------------------------------------------------------------------

def _check_shape(N, K, k, r):
    if N <= 0 or K <= 0 or K % GROUP:
        raise FormatError(f"bad shape N={N} K={K} (K must be a positive multiple of 128)")
    if k not in VALID_K:
        raise FormatError(f"k={k} not in {VALID_K}")
    if not 0 <= r <= MAX_RANK:
        raise FormatError(f"r={r} outside [0, {MAX_RANK}]")


def payload_sizes(N: int, K: int, k: int, r: int):
    """Bytes of information in the six layout-v1 buffers: codes, sites, scales,
    U bits, V bits, s (before padding)."""
    _check_shape(N, K, k, r)
    G = K // GROUP
    codes = N * K // 4
    sites = N * G * k
    scales = N * G * (4 if k > 0 else 2)
    ubits = N * ((r + 31) // 32) * 4
    vbits = r * (K // 32) * 4
    lr = 2 * r
    return [codes, sites, scales, ubits, vbits, lr]


def packed_sizes(N: int, K: int, k: int, r: int):
    """Allocated size of each buffer: the payload zero-padded to a multiple of 16 bytes."""
    return [(s + 15) // 16 * 16 for s in payload_sizes(N, K, k, r)]


def bits_per_weight(N: int, K: int, k: int, r: int) -> float:
    return 8.0 * sum(payload_sizes(N, K, k, r)) / (N * K)


# ---------------------------------------------------------------------------
# pack / unpack (the oracle's own bit handling)
# ---------------------------------------------------------------------------

@dataclass
class Unpacked:
    N: int
    K: int
    k: int
    r: int
    T: np.ndarray          # int8 [N, K]
    site_pos: np.ndarray   # uint8 [N, G, k]
    site_sign: np.ndarray  # int8 [N, G, k]
    alpha: np.ndarray      # uint16 [N, G]
    beta: np.ndarray       # uint16 [N, G]
    U: np.ndarray          # int8 [N, r]
    V: np.ndarray          # int8 [K, r]
    lr_scale: np.ndarray   # uint16 [r]


def pack(c) -> list:
    """Components -> the six layout-v1 buffers (numpy uint8/uint16/uint32 arrays)."""
    N, K, k, r = c.N, c.K, c.k, c.r
    _check_shape(N, K, k, r)
    G = K // GROUP
    T = np.asarray(c.T)
    if T.shape != (N, K) or T.min(initial=0) < -1 or T.max(initial=0) > 1:
        raise FormatError("T must be [N, K] with values in {-1, 0, +1}")
    code = (T.astype(np.int64) + 1).astype(np.uint32).reshape(N, K // 16, 16)
    shifts = (2 * np.arange(16, dtype=np.uint32))
    codes = np.bitwise_or.reduce(code << shifts, axis=2).astype(np.uint32)

    pos = np.asarray(c.site_pos).reshape(N, G, k)
    sgn = np.asarray(c.site_sign).reshape(N, G, k)
    if k:
        if pos.max() >= GROUP:
            raise FormatError("site position outside the group")
        if np.any(np.diff(pos.astype(np.int16), axis=2) <= 0):
            raise FormatError("site positions must be distinct and ascending")
        if not np.all(np.abs(sgn) == 1):
            raise FormatError("site signs must be +1 or -1")
    sites = (pos.astype(np.uint8) | np.where(sgn < 0, 0x80, 0).astype(np.uint8)).astype(np.uint8)

    alpha = np.asarray(c.alpha, dtype=np.uint16).reshape(N, G)
    if k:
        scales = np.stack([alpha, np.asarray(c.beta, dtype=np.uint16).reshape(N, G)], axis=2)
    else:
        scales = alpha.copy()

    nw = (r + 31) // 32
    U = np.asarray(c.U).reshape(N, r)
    V = np.asarray(c.V).reshape(K, r)
    if r and not (np.all(np.abs(U) == 1) and np.all(np.abs(V) == 1)):
        raise FormatError("U and V must be +-1")
    ubits = np.zeros((N, nw), dtype=np.uint32)
    for rho in range(r):
        ubits[:, rho // 32] |= (U[:, rho] < 0).astype(np.uint32) << np.uint32(rho % 32)
    vneg = (V.T < 0).astype(np.uint32).reshape(r, K // 32, 32)
    vbits = np.bitwise_or.reduce(vneg << np.arange(32, dtype=np.uint32), axis=2).astype(np.uint32) \
        if r else np.zeros((0, K // 32), np.uint32)
    lr = np.asarray(c.lr_scale, dtype=np.uint16).reshape(r).copy()
    out = []
    for b, size in zip([codes, sites, scales, ubits, vbits, lr], packed_sizes(N, K, k, r)):
        raw = np.zeros(size, dtype=np.uint8)
        bb = np.ascontiguousarray(b).reshape(-1).view(np.uint8)
        raw[: bb.size] = bb
        out.append(raw)
    return out


def _as_u8(buf) -> np.ndarray:
    return np.frombuffer(np.ascontiguousarray(buf).tobytes(), dtype=np.uint8)


def unpack(bufs, N: int, K: int, k: int, r: int) -> Unpacked:
    """The six layout-v1 buffers (any integer dtype / raw bytes) -> dense components.

    Raises FormatError on reserved codes, out-of-order or duplicate sites and
    wrong buffer sizes."""
    _check_shape(N, K, k, r)
    G = K // GROUP
    sizes = packed_sizes(N, K, k, r)
    used = payload_sizes(N, K, k, r)
    raw = [_as_u8(b) for b in bufs]
    for i, (b, s, u) in enumerate(zip(raw, sizes, used)):
        if b.size != s:
            raise FormatError(f"buffer {i} has {b.size} bytes, expected {s}")
        if np.any(b[u:]):
            raise FormatError(f"buffer {i} has nonzero padding")
    raw = [b[:u] for b, u in zip(raw, used)]
    words = raw[0].view('<u4').reshape(N, K // 16, 1)
    code = (words >> (2 * np.arange(16, dtype=np.uint32))) & 3
    if np.any(code == 3):
        raise FormatError("reserved trit code 3")
    T = (code.reshape(N, K).astype(np.int8) - 1).astype(np.int8)

    sb = raw[1].reshape(N, G, k)
    pos = (sb & 0x7F).astype(np.uint8)
    sgn = np.where(sb & 0x80, -1, 1).astype(np.int8)
    if k and np.any(np.diff(pos.astype(np.int16), axis=2) <= 0):
        raise FormatError("site positions must be distinct and ascending")

    sc = raw[2].view('<u2')
    if k:
        sc = sc.reshape(N, G, 2)
        alpha, beta = sc[:, :, 0].copy(), sc[:, :, 1].copy()
    else:
        alpha, beta = sc.reshape(N, G).copy(), np.zeros((N, G), np.uint16)

    nw = (r + 31) // 32
    ub = raw[3].view('<u4').reshape(N, nw) if nw else np.zeros((N, 0), np.uint32)
    U = np.empty((N, r), np.int8)
    for rho in range(r):
        U[:, rho] = np.where((ub[:, rho // 32] >> np.uint32(rho % 32)) & 1, -1, 1)
    vb = raw[4].view('<u4').reshape(r, K // 32) if r else np.zeros((0, K // 32), np.uint32)
    vneg = (vb[:, :, None] >> np.arange(32, dtype=np.uint32)) & 1
    V = np.where(vneg.reshape(r, K).T, -1, 1).astype(np.int8) if r else np.zeros((K, 0), np.int8)
    lr = raw[5].view('<u2').copy() if r else np.zeros(0, np.uint16)
    return Unpacked(N, K, k, r, T, pos, sgn, alpha, beta, U, V, lr)


# ---------------------------------------------------------------------------
# the product
# ---------------------------------------------------------------------------

def dense_weight(c, rows=None) -> np.ndarray:
    """Dense float64 W = alpha (x) T + beta (x) R + U diag(s) V^T for the given rows.

    alpha and beta are expanded over the 128 columns of their group; R is
    zero except R[n, 128 g + pos] = sign at each residual site."""
    N, K, k, r = c.N, c.K, c.k, c.r
    G = K // GROUP
    rows = np.arange(N) if rows is None else np.asarray(rows)
    n = rows.size
    alpha = widen_fp16(np.asarray(c.alpha).reshape(N, G)[rows])
    W = np.repeat(alpha, GROUP, axis=1) * np.asarray(c.T)[rows].astype(np.float64)
    if k:
        beta = widen_fp16(np.asarray(c.beta).reshape(N, G)[rows])
        R = np.zeros((n, K), dtype=np.float64)
        pos = np.asarray(c.site_pos).reshape(N, G, k)[rows].astype(np.int64)
        sgn = np.asarray(c.site_sign).reshape(N, G, k)[rows].astype(np.float64)
        col = pos + (GROUP * np.arange(G))[None, :, None]
        rr = np.broadcast_to(np.arange(n)[:, None, None], col.shape)
        np.add.at(R, (rr.reshape(-1), col.reshape(-1)), sgn.reshape(-1))
        W += np.repeat(beta, GROUP, axis=1) * R
    if r:
        s = widen_fp16(c.lr_scale)
        U = np.asarray(c.U)[rows].astype(np.float64)
        V = np.asarray(c.V).astype(np.float64)
        W += (U * s[None, :]) @ V.T
    return W


def matmul_rows(c, X_bits, rows) -> np.ndarray:
    """Y[m, i] = sum_j W[rows[i], j] * x_m[j] in float64; X_bits is bf16 [M, K]."""
    X = widen_bf16(np.asarray(X_bits).reshape(-1, c.K))
    return X @ dense_weight(c, rows).T


def matmul(c, X_bits) -> np.ndarray:
    """Y = X W^T, float64 [M, N]."""
    return matmul_rows(c, X_bits, np.arange(c.N))


def matvec(c, x_bits) -> np.ndarray:
    """y = W x, float64 [N]."""
    return matmul(c, np.asarray(x_bits).reshape(1, c.K))[0]


# ---------------------------------------------------------------------------
# tolerance used by every parity test
# ---------------------------------------------------------------------------

REL_L2_TOL = 1e-5
MAX_ABS_FACTOR = 1e-3


def check_tolerance(Y, Y_ref, X_bits, alpha_bits):
    """rel-L2 = ||Y - Y*|| / ||Y*|| <= 1e-5 over the whole output, and for each
    activation row m: max |Y - Y*| <= 1e-3 * ||x_m||_2 * max |alpha|.
    Where Y* is exactly zero everywhere, Y must be exactly zero too.
    Returns (ok, rel_l2, worst_abs_ratio)."""
    Y = np.asarray(Y, dtype=np.float64).reshape(np.shape(Y_ref))
    Y_ref = np.asarray(Y_ref, dtype=np.float64)
    X = widen_bf16(X_bits).reshape(Y_ref.shape[0] if Y_ref.ndim > 1 else 1, -1)
    ref_norm = np.linalg.norm(Y_ref)
    if ref_norm == 0.0:
        ok = bool(np.all(Y == 0.0))
        return ok, 0.0 if ok else np.inf, 0.0 if ok else np.inf
    rel = float(np.linalg.norm(Y - Y_ref) / ref_norm)
    amax = float(np.max(np.abs(widen_fp16(alpha_bits)))) if np.size(alpha_bits) else 0.0
    Yr = Y_ref.reshape(X.shape[0], -1)
    Yd = np.abs(Y.reshape(X.shape[0], -1) - Yr)
    worst = 0.0
    for m in range(X.shape[0]):
        bound = MAX_ABS_FACTOR * np.linalg.norm(X[m]) * amax
        if Yd[m].size:
            worst = max(worst, float(Yd[m].max() / bound) if bound > 0 else (0.0 if Yd[m].max() == 0 else np.inf))
    return (rel <= REL_L2_TOL and worst <= 1.0), rel, worst
