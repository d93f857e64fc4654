"""Seeded generators for body-matrix components and activations.

Every stream is keyed by ``SeedSequence([0x57A1, workload_id, matrix_index,
stream])`` with streams 0 = T, 1 = residual sites, 2 = alpha/beta, 3 = U/V/s,
4 = x, 9 = selections.  The two bulk streams (T and the sites) are drawn by a
counter-based SplitMix64 in C (``csrc/synth.c``) seeded with the first 64-bit
word of that SeedSequence; the small streams use NumPy PCG64 directly.

Component arrays are the *dense, unpacked* description of one matrix
(what the WAL-Ternary-8B model card calls T, R, alpha, beta and the WALB2
pair); the packed byte layout is produced elsewhere.
"""
from __future__ import annotations

import ctypes
from dataclasses import dataclass

import numpy as np

from .build import build as _build_synth

_lib = None


def _synth_lib():
    global _lib
    if _lib is None:
        _lib = ctypes.CDLL(_build_synth())
        _lib.wal_synth_trits.argtypes = [ctypes.c_void_p, ctypes.c_int64, ctypes.c_uint64,
                                         ctypes.c_uint32, ctypes.c_uint32]
        _lib.wal_synth_sites.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int64,
                                         ctypes.c_int, ctypes.c_uint64]
    return _lib


def stream_seed(config_id: int, matrix_index: int, stream: int) -> int:
    ss = np.random.SeedSequence([CONFIG_SEED, int(config_id), int(matrix_index), int(stream)])
    return int(ss.generate_state(1, np.uint64)[0])

CONFIG_SEED = 0x57A1
GROUP = 128

S_T, S_SITES, S_SCALES, S_LOWRANK, S_X, S_SELECT = 0, 1, 2, 3, 4, 9


def rng_for(config_id: int, matrix_index: int, stream: int) -> np.random.Generator:
    ss = np.random.SeedSequence([CONFIG_SEED, int(config_id), int(matrix_index), int(stream)])
    return np.random.Generator(np.random.PCG64(ss))


def bf16_bits_from_f32(a) -> np.ndarray:
    """Round float32 values to bfloat16 (round to nearest, ties to even); returns uint16 bits."""
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32).astype(np.uint64)
    r = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return r.astype(np.uint16)


def bf16_bits_to_f32(b) -> np.ndarray:
    """Exact widening of bfloat16 bits to float32."""
    return (np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


@dataclass
class Components:
    """Dense description of one body matrix W (N outputs, K inputs).

    T         int8  [N, K]        ternary base, values in {-1, 0, +1}
    site_pos  uint8 [N, G, k]     residual positions inside each 128-group, distinct, ascending
    site_sign int8  [N, G, k]     residual signs, +1 / -1
    alpha     uint16[N, G]        fp16 bits of the T-scale per (row, group)
    beta      uint16[N, G]        fp16 bits of the R-scale per (row, group) (zeros when k == 0)
    U         int8  [N, r]        +1 / -1
    V         int8  [K, r]        +1 / -1
    lr_scale  uint16[r]           fp16 bits of the per-rank scale s_r
    """
    N: int
    K: int
    k: int
    r: int
    T: np.ndarray
    site_pos: np.ndarray
    site_sign: np.ndarray
    alpha: np.ndarray
    beta: np.ndarray
    U: np.ndarray
    V: np.ndarray
    lr_scale: np.ndarray

    @property
    def G(self) -> int:
        return self.K // GROUP


@dataclass
class MatrixSpec:
    name: str
    N: int
    K: int
    k: int
    r: int
    stage: int
    index: int = 0
    layer: int = 0


def _draw_sites(seed: int, n_groups: int, k: int):
    """k distinct uniform positions in [0, 128) per group (Floyd's subset
    sampling), ascending, plus fair +-1 signs."""
    pos = np.empty((n_groups, k), dtype=np.uint8)
    sign = np.empty((n_groups, k), dtype=np.int8)
    _synth_lib().wal_synth_sites(pos.ctypes.data, sign.ctypes.data, n_groups, k, seed)
    return pos, sign


def _fp16_bits(v: np.ndarray) -> np.ndarray:
    return v.astype(np.float16).view(np.uint16)


def gen_components(N: int, K: int, k: int, r: int, config_id: int = 0, matrix_index: int = 0,
                   p_neg: float = 0.3, p_zero: float = 0.4,
                   alpha_sd: float = 0.02, beta_sd: float = 0.005, s_sd: float = 0.01) -> Components:
    """Draw one matrix.  Defaults are the workload's distributions:
    T iid {-1: 0.3, 0: 0.4, +1: 0.3} (probabilities quantised to 1/65536); k distinct uniform sites per group with
    signs +-1 at p = 0.5; alpha = fp16(|N(0, 0.02)|), beta = fp16(|N(0, 0.005)|);
    U, V iid +-1; s = fp16(|N(0, 0.01)|)."""
    if K % GROUP:
        raise ValueError("K must be a multiple of 128")
    G = K // GROUP
    T = np.empty((N, K), dtype=np.int8)
    thr_neg = int(round(p_neg * 65536))
    thr_pos = int(round((p_neg + p_zero) * 65536))
    _synth_lib().wal_synth_trits(T.ctypes.data, N * K, stream_seed(config_id, matrix_index, S_T),
                                 thr_neg, thr_pos)
    if k > 0:
        pos, sgn = _draw_sites(stream_seed(config_id, matrix_index, S_SITES), N * G, k)
        site_pos = pos.reshape(N, G, k)
        site_sign = sgn.reshape(N, G, k)
    else:
        site_pos = np.zeros((N, G, 0), dtype=np.uint8)
        site_sign = np.zeros((N, G, 0), dtype=np.int8)
    rs = rng_for(config_id, matrix_index, S_SCALES)
    alpha = _fp16_bits(np.abs(rs.normal(0.0, alpha_sd, size=(N, G))))
    beta = _fp16_bits(np.abs(rs.normal(0.0, beta_sd, size=(N, G)))) if k > 0 else np.zeros((N, G), np.uint16)
    rl = rng_for(config_id, matrix_index, S_LOWRANK)
    U = (rl.integers(0, 2, size=(N, r), dtype=np.int8) * 2 - 1).astype(np.int8)
    V = (rl.integers(0, 2, size=(K, r), dtype=np.int8) * 2 - 1).astype(np.int8)
    lr_scale = _fp16_bits(np.abs(rl.normal(0.0, s_sd, size=r)))
    return Components(N, K, k, r, T, site_pos, site_sign, alpha, beta, U, V, lr_scale)


def gen_x(K: int, M: int = 1, config_id: int = 0, matrix_index: int = 0) -> np.ndarray:
    """Activations x ~ N(0, 1) rounded to bf16; uint16 bits, row-major [M, K]."""
    rx = rng_for(config_id, matrix_index, S_X)
    return bf16_bits_from_f32(rx.standard_normal((M, K), dtype=np.float32)).reshape(M, K)


# ---------------------------------------------------------------------------
# Model-shaped matrix lists
# ---------------------------------------------------------------------------

# (role, N out, K in) for a Qwen3-8B-shaped decoder layer
LAYER_8B = [("q", 4096, 4096), ("k", 1024, 4096), ("v", 1024, 4096), ("o", 4096, 4096),
            ("gate", 12288, 4096), ("up", 12288, 4096), ("down", 4096, 12288)]
# (role, N out, K in) for the 27B-shaped stand-in layer: hidden 5120, MLP 17408
LAYER_27B = [("q", 5120, 5120), ("k", 5120, 5120), ("v", 5120, 5120), ("o", 5120, 5120),
             ("gate", 17408, 5120), ("up", 17408, 5120), ("down", 5120, 17408)]
# dependency stage inside a layer: [q,k,v] -> [o] -> [gate,up] -> [down]
ROLE_STAGE = {"q": 0, "k": 0, "v": 0, "o": 1, "gate": 2, "up": 2, "down": 3}
ROLE_K_27B = {"q": 4, "k": 4, "v": 4, "o": 2, "gate": 8, "up": 8, "down": 8}


def body_plan(layers, layer_roles, k_by_role, r_default, config_id, n_lowrank=None,
              n_k0=0, r_value=8):
    """List of MatrixSpec in model order with seeded WALB2 / k=0 selections."""
    specs = []
    idx = 0
    for L in range(layers):
        for role, N, K in layer_roles:
            k = k_by_role[role] if isinstance(k_by_role, dict) else int(k_by_role)
            specs.append(MatrixSpec(f"L{L}.{role}", N, K, k, r_default, 4 * L + ROLE_STAGE[role], idx, L))
            idx += 1
    sel = rng_for(config_id, 0, S_SELECT)
    if n_lowrank is not None:
        chosen = set(int(i) for i in sel.choice(len(specs), n_lowrank, replace=False))
        for s in specs:
            s.r = r_value if s.index in chosen else 0
    if n_k0:
        chosen0 = set(int(i) for i in sel.choice(len(specs), n_k0, replace=False))
        for s in specs:
            if s.index in chosen0:
                s.k = 0
    return specs


# workload name -> seed id used in every SeedSequence of that workload
WORKLOAD_IDS = {"single": 0, "layer8b": 1, "body8b": 2, "body27b": 3, "sweep": 4, "pq2_body8b": 5}


def config_plan(workload):
    """Matrices of each named workload (name or its seed id).

    single : one matrix K=1024 -> N=512, k=8, r=4.
    layer8b: one Qwen3-8B-shaped layer (7 matrices), k=8, r=8.
    body8b : 36 such layers = 252 matrices, k=8, a seeded 213 carry r=8, the rest r=0.
    body27b: 64 layers x 7 = 448 27B-shaped matrices; k by role (MLP 8, q/k/v 4,
             o 2), a seeded 45 (10 %) forced to k=0, a seeded 152 carry r=8.
    sweep  : gate 4096->12288 and down 12288->4096, k=8, r=16 (batch sweep).
    pq2_body8b: the 252 matrices of body8b as plain ternary (k=0, r=0), the
             PQ2_0 block format's workload.
    """
    wid = WORKLOAD_IDS[workload] if isinstance(workload, str) else int(workload)
    if wid == 0:
        return [MatrixSpec("single", 512, 1024, 8, 4, 0, 0, 0)]
    if wid == 1:
        return body_plan(1, LAYER_8B, 8, 8, wid)
    if wid == 2:
        return body_plan(36, LAYER_8B, 8, 8, wid, n_lowrank=213)
    if wid == 3:
        return body_plan(64, LAYER_27B, ROLE_K_27B, 8, wid, n_lowrank=152, n_k0=45)
    if wid == 4:
        return [MatrixSpec("gate", 12288, 4096, 8, 16, 0, 0, 0),
                MatrixSpec("down", 4096, 12288, 8, 16, 1, 1, 0)]
    if wid == 5:
        return body_plan(36, LAYER_8B, 0, 0, wid)
    raise ValueError(f"unknown workload {workload}")


def workload_id(workload) -> int:
    return WORKLOAD_IDS[workload] if isinstance(workload, str) else int(workload)


def gen_matrix(workload, spec: MatrixSpec) -> Components:
    """Components of one matrix of a workload, seeded by (workload, matrix index)."""
    return gen_components(spec.N, spec.K, spec.k, spec.r, workload_id(workload), spec.index)


def gen_pq2(N: int, K: int, config_id: int = 0, matrix_index: int = 0):
    """One plain-ternary matrix for the PQ2_0 block format: T iid as in
    gen_components and one scale d = fp16(|N(0, 0.02)|) per (row, 128-group).
    Returns (T int8 [N, K], d uint16 fp16 bits [N, K/128])."""
    c = gen_components(N, K, 0, 0, config_id, matrix_index)
    return c.T, c.alpha


def gen_base3(N: int, K: int, config_id: int = 0, matrix_index: int = 0):
    """One plain-ternary matrix for the base-3 container: T iid as in
    gen_components and one BF16 scale per (row, 128-group), bf16(|N(0, 0.02)|).
    Returns (T int8 [N, K], s uint16 bf16 bits [N, K/128])."""
    c = gen_components(N, K, 0, 0, config_id, matrix_index)
    rs = rng_for(config_id, matrix_index, S_SCALES)
    s = bf16_bits_from_f32(np.abs(rs.normal(0.0, 0.02, size=(N, K // GROUP))).astype(np.float32))
    return c.T, s


S_LOWRANK2 = 6  # stream of the second WALB2 path of an RC1 matrix


def f24_bytes_from_f32(a) -> np.ndarray:
    """Round float32 values to the 24-bit float storage type (the upper three
    bytes of an FP32, round to nearest, ties to even); uint8 [..., 3] little endian."""
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32).astype(np.uint64)
    r = ((u + 0x7F + ((u >> 8) & 1)) >> 8).astype(np.uint32)
    return np.stack([(r >> (8 * i)) & 0xFF for i in range(3)], axis=-1).astype(np.uint8)


def gen_rc1(N: int, K: int, k: int, r1: int, r2: int, config_id: int = 0, matrix_index: int = 0):
    """One RC1-format matrix: T and sites as in gen_components; alpha, beta
    (|N(0, 0.02)|, |N(0, 0.005)|) and the per-rank scales (|N(0, 0.01)|) rounded
    to 24-bit floats; two WALB2 paths of ranks r1 and r2 with iid +-1 U, V.
    Returns a dict of arrays (T, site_pos, site_sign, alpha24, beta24, U1, V1,
    s1, U2, V2, s2) plus N, K, k."""
    G = K // GROUP
    c = gen_components(N, K, k, 0, config_id, matrix_index)
    rs = rng_for(config_id, matrix_index, S_SCALES)
    alpha = f24_bytes_from_f32(np.abs(rs.normal(0.0, 0.02, size=(N, G))).astype(np.float32))
    beta = f24_bytes_from_f32(np.abs(rs.normal(0.0, 0.005, size=(N, G))).astype(np.float32))
    paths = []
    for stream, r in ((S_LOWRANK, r1), (S_LOWRANK2, r2)):
        rl = rng_for(config_id, matrix_index, stream)
        U = (rl.integers(0, 2, size=(N, r), dtype=np.int8) * 2 - 1).astype(np.int8)
        V = (rl.integers(0, 2, size=(K, r), dtype=np.int8) * 2 - 1).astype(np.int8)
        s = f24_bytes_from_f32(np.abs(rl.normal(0.0, 0.01, size=r)).astype(np.float32)).reshape(r, 3)
        paths += [U, V, s]
    return dict(N=N, K=K, k=k, T=c.T, site_pos=c.site_pos, site_sign=c.site_sign, alpha24=alpha, beta24=beta,
                U1=paths[0], V1=paths[1], s1=paths[2], U2=paths[3], V2=paths[4], s2=paths[5])


def gen_int4(N: int, K: int, config_id: int = 0, matrix_index: int = 0):
    """An INT4/g128 matrix (the LM head): q iid uniform on [-8, 7] and one
    scale d = fp16(|N(0, 0.02)|) per (row, 128-group).  Returns (q int8 [N, K],
    d uint16 fp16 bits [N, K/128])."""
    rq = rng_for(config_id, matrix_index, S_T)
    q = rq.integers(-8, 8, size=(N, K), dtype=np.int8)
    rs = rng_for(config_id, matrix_index, S_SCALES)
    return q, _fp16_bits(np.abs(rs.normal(0.0, 0.02, size=(N, K // GROUP))))


def gen_int3(V: int, H: int, config_id: int = 0, matrix_index: int = 0):
    """An INT3/g128 table (the embedding): q iid uniform on [-4, 3] and one
    scale d = fp16(|N(0, 0.02)|) per (row, 128-group).  Returns (q int8 [V, H],
    d uint16 fp16 bits [V, H/128])."""
    rq = rng_for(config_id, matrix_index, S_T)
    q = rq.integers(-4, 4, size=(V, H), dtype=np.int8)
    rs = rng_for(config_id, matrix_index, S_SCALES)
    return q, _fp16_bits(np.abs(rs.normal(0.0, 0.02, size=(V, H // GROUP))))
