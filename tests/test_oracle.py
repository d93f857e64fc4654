"""Pins for the FP64 oracle (CPU only).

The oracle is checked against things other than itself:
  * hand-derived worked cases (tests/golden/*.txt, each with its derivation),
  * a pure-Python brute force over the unpacked generator arrays,
  * invariants of the definition (linearity, odd symmetry, scale doubling,
    row permutation, the plain-ternary special case via a separate numpy
    expression),
  * the PQ2_0 size of the WAL2-Ternary-27B card (34 bytes per 128 weights),
  * planted mistakes: each one must make at least one pin fail.
"""
import struct

import numpy as np
import pytest

import oracle
from oracle import wal_oracle as wo
from wal_synth import Components, gen_components, gen_x, bf16_bits_from_f32

from golden_io import fixture_names, load


# ---------------------------------------------------------------------------
# golden worked cases
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("name", fixture_names())
def test_golden_direct(name):
    c, x, y, _ = load(name)
    got = oracle.matvec(c, x)
    assert np.array_equal(got, y), (name, got, y)


@pytest.mark.parametrize("name", fixture_names())
def test_golden_through_packing(name):
    c, x, y, codes_hex = load(name)
    bufs = oracle.pack(c)
    u = oracle.unpack(bufs, c.N, c.K, c.k, c.r)
    assert np.array_equal(oracle.matvec(u, x), y)
    if codes_hex is not None:
        assert bufs[0].view(np.uint8)[: len(codes_hex)].tobytes() == codes_hex


def test_golden_codes_decode_by_hand():
    """Decode the fixture's hex bytes with the oracle and compare with the
    trits listed in the fixture."""
    c, _, _, codes_hex = load("codes_row16")
    raw = np.frombuffer(codes_hex, dtype=np.uint8)
    scales = np.zeros(16, np.uint8)
    scales[:2] = np.frombuffer(np.array([0x3C00], np.uint16).tobytes(), np.uint8)
    bufs = [raw, np.zeros(0, np.uint8), scales,
            np.zeros(0, np.uint8), np.zeros(0, np.uint8), np.zeros(0, np.uint8)]
    u = oracle.unpack(bufs, 1, 128, 0, 0)
    assert np.array_equal(u.T, c.T)


# ---------------------------------------------------------------------------
# brute force on tiny matrices
# ---------------------------------------------------------------------------

def _f16(b):
    return struct.unpack("<e", struct.pack("<H", int(b)))[0]


def _bf16(b):
    return struct.unpack("<f", struct.pack("<I", int(b) << 16))[0]


def brute_force(c, x_bits):
    """Per-element loops straight from the component arrays (no packing)."""
    x = [_bf16(b) for b in np.asarray(x_bits).reshape(-1)]
    y = []
    for n in range(c.N):
        total = 0.0
        for g in range(c.K // 128):
            t_acc = 0.0
            for j in range(128 * g, 128 * g + 128):
                t = int(c.T[n, j])
                if t == 1:
                    t_acc += x[j]
                elif t == -1:
                    t_acc -= x[j]
            r_acc = 0.0
            for i in range(c.k):
                p = 128 * g + int(c.site_pos[n, g, i])
                r_acc += x[p] if int(c.site_sign[n, g, i]) > 0 else -x[p]
            total += _f16(c.alpha[n, g]) * t_acc
            if c.k:
                total += _f16(c.beta[n, g]) * r_acc
        for rho in range(c.r):
            v = 0.0
            for j in range(c.K):
                v += x[j] if int(c.V[j, rho]) > 0 else -x[j]
            total += _f16(c.lr_scale[rho]) * int(c.U[n, rho]) * v
        y.append(total)
    return np.array(y)


@pytest.mark.parametrize("N,K,k,r", [(5, 256, 8, 3), (4, 128, 0, 0), (3, 256, 2, 1),
                                     (6, 128, 4, 4), (2, 384, 8, 0), (3, 128, 0, 2)])
def test_brute_force(N, K, k, r):
    c = gen_components(N, K, k, r, config_id=77, matrix_index=N * 1000 + K + k + r)
    x = gen_x(K, 1, 77, N + K)[0]
    want = brute_force(c, x)
    got = oracle.matvec(oracle.unpack(oracle.pack(c), N, K, k, r), x)
    np.testing.assert_allclose(got, want, rtol=1e-12, atol=1e-12 * np.abs(want).max())


# ---------------------------------------------------------------------------
# invariants
# ---------------------------------------------------------------------------

@pytest.fixture(scope="module")
def mid():
    c = gen_components(64, 1024, 8, 4, config_id=78, matrix_index=1)
    x = gen_x(1024, 1, 78, 1)[0]
    return c, x


def test_linearity_disjoint_support(mid):
    c, x = mid
    x1 = x.copy(); x1[1::2] = 0
    x2 = x.copy(); x2[0::2] = 0
    y = oracle.matvec(c, x)
    y12 = oracle.matvec(c, x1) + oracle.matvec(c, x2)
    np.testing.assert_allclose(y, y12, rtol=1e-13, atol=1e-13 * np.abs(y).max())


def test_odd_symmetry(mid):
    c, x = mid
    xn = x ^ np.uint16(0x8000)
    np.testing.assert_array_equal(oracle.matvec(c, xn), -oracle.matvec(c, x))


def test_alpha_doubling_doubles_ternary_part(mid):
    c, x = mid
    a = wo.widen_fp16(c.alpha)
    a2 = (2 * a).astype(np.float16).view(np.uint16)
    assert np.array_equal(wo.widen_fp16(a2), 2 * a)  # doubling is exact here
    c2 = Components(**{**c.__dict__, "alpha": a2})
    tpart = np.repeat(a, 128, axis=1) * c.T @ wo.widen_bf16(x)
    np.testing.assert_allclose(oracle.matvec(c2, x) - oracle.matvec(c, x), tpart,
                               rtol=1e-12, atol=1e-12 * np.abs(tpart).max())


def test_row_permutation(mid):
    c, x = mid
    perm = np.random.default_rng(5).permutation(c.N)
    cp = Components(c.N, c.K, c.k, c.r, c.T[perm], c.site_pos[perm], c.site_sign[perm],
                    c.alpha[perm], c.beta[perm], c.U[perm], c.V, c.lr_scale)
    np.testing.assert_array_equal(oracle.matvec(cp, x), oracle.matvec(c, x)[perm])


def test_plain_ternary_special_case():
    """beta = 0 and r = 0 reduce the method to plain group-scaled ternary:
    y = (alpha expanded over its 128 columns * T) @ x, written here with
    einsum over the group axis instead of a dense W."""
    c = gen_components(32, 512, 0, 0, config_id=79, matrix_index=2)
    x = gen_x(512, 1, 79, 2)[0]
    xs = wo.widen_bf16(x).reshape(4, 128)
    per_group = np.einsum("ngj,gj->ng", c.T.reshape(32, 4, 128).astype(np.float64), xs)
    want = (wo.widen_fp16(c.alpha) * per_group).sum(axis=1)
    np.testing.assert_allclose(oracle.matvec(c, x), want, rtol=1e-13, atol=1e-15)


def test_matmul_columns_equal_matvec(mid):
    c, _ = mid
    X = gen_x(1024, 3, 78, 9)
    Y = oracle.matmul(c, X)
    for m in range(3):
        np.testing.assert_array_equal(Y[m], oracle.matvec(c, X[m]))
    rows = np.array([0, 5, 63])
    np.testing.assert_array_equal(oracle.matmul_rows(c, X, rows), Y[:, rows])


# ---------------------------------------------------------------------------
# sizes
# ---------------------------------------------------------------------------

def test_pq2_size_per_group():
    """T + alpha (k = 0, r = 0) costs 32 B of codes + 2 B of FP16 scale per
    128 weights = 34 B = 2.125 bit/weight (PQ2_0 on the WAL2-Ternary-27B card)."""
    s = oracle.payload_sizes(1, 128, 0, 0)
    assert s[0] == 32 and s[2] == 2 and sum(s) == 34
    assert oracle.bits_per_weight(4096, 4096, 0, 0) == 2.125


@pytest.mark.parametrize("N,K,k,r", [(4096, 4096, 8, 8), (1024, 4096, 2, 0), (12288, 4096, 8, 16),
                                     (5120, 17408, 4, 8), (512, 1024, 0, 4)])
def test_bits_per_weight_formula(N, K, k, r):
    want = 2 + k / 16 + (0.25 if k else 0.125) + 32 * ((r + 31) // 32) / K \
        + r / N + 16 * r / (N * K)
    assert abs(oracle.bits_per_weight(N, K, k, r) - want) < 1e-12


# ---------------------------------------------------------------------------
# format rejection
# ---------------------------------------------------------------------------

def test_unpack_rejects_reserved_code():
    c = gen_components(2, 128, 2, 1, config_id=80)
    bufs = oracle.pack(c)
    bufs[0] = bufs[0].copy()
    bufs[0][5] |= np.uint8(3 << 2)
    with pytest.raises(oracle.FormatError):
        oracle.unpack(bufs, 2, 128, 2, 1)


def test_unpack_rejects_duplicate_sites():
    c = gen_components(2, 128, 4, 0, config_id=80)
    bufs = oracle.pack(c)
    bufs[1] = bufs[1].copy()
    bufs[1][1] = bufs[1][0]
    with pytest.raises(oracle.FormatError):
        oracle.unpack(bufs, 2, 128, 4, 0)


def test_unpack_rejects_wrong_size():
    c = gen_components(2, 128, 4, 0, config_id=80)
    bufs = oracle.pack(c)
    bufs[2] = bufs[2][:-1]
    with pytest.raises(oracle.FormatError):
        oracle.unpack(bufs, 2, 128, 4, 0)


def test_unpack_rejects_nonzero_padding():
    c = gen_components(3, 128, 2, 0, config_id=80)   # 12 site bytes padded to 16
    bufs = oracle.pack(c)
    bufs[1] = bufs[1].copy()
    bufs[1][-1] = 1
    with pytest.raises(oracle.FormatError):
        oracle.unpack(bufs, 3, 128, 2, 0)


def test_padding_to_16_bytes():
    assert oracle.packed_sizes(3, 128, 2, 1) == [96, 16, 16, 16, 16, 16]
    assert oracle.payload_sizes(3, 128, 2, 1) == [96, 6, 12, 12, 16, 2]


@pytest.mark.parametrize("shape", [(2, 100, 0, 0), (2, 128, 3, 0), (2, 128, 0, 33), (0, 128, 0, 0)])
def test_bad_shapes(shape):
    with pytest.raises(oracle.FormatError):
        oracle.packed_sizes(*shape)


def test_tolerance_check_catches_small_error(mid):
    c, x = mid
    y = oracle.matvec(c, x)
    ok, rel, _ = oracle.check_tolerance(y, y, x, c.alpha)
    assert ok and rel == 0.0
    bad = y * (1 + 3e-5)
    ok, rel, _ = oracle.check_tolerance(bad, y, x, c.alpha)
    assert not ok and rel > 1e-5
    ok, _, _ = oracle.check_tolerance(np.full(3, 1e-30), np.zeros(3), x, c.alpha)
    assert not ok


# ---------------------------------------------------------------------------
# planted mistakes in the oracle must be caught by the pins above
# ---------------------------------------------------------------------------

def _pins_pass():
    for name in fixture_names():
        c, x, y, _ = load(name)
        u = oracle.unpack(oracle.pack(c), c.N, c.K, c.k, c.r)
        if not np.array_equal(oracle.matvec(u, x), y):
            return False
    for N, K, k, r in [(5, 256, 8, 3), (3, 256, 2, 1)]:
        c = gen_components(N, K, k, r, config_id=77, matrix_index=N * 1000 + K + k + r)
        x = gen_x(K, 1, 77, N + K)[0]
        got = oracle.matvec(oracle.unpack(oracle.pack(c), N, K, k, r), x)
        want = brute_force(c, x)
        if not np.allclose(got, want, rtol=1e-12, atol=1e-12 * np.abs(want).max()):
            return False
    return True


def _plant_unpack(monkeypatch, mutate):
    real = wo.unpack

    def bad(bufs, N, K, k, r):
        u = real(bufs, N, K, k, r)
        mutate(u)
        return u
    monkeypatch.setattr(oracle, "unpack", bad)


def test_pins_pass_unplanted():
    assert _pins_pass()


def test_plant_dropped_residual(monkeypatch):
    _plant_unpack(monkeypatch, lambda u: setattr(u, "beta", np.zeros_like(u.beta)))
    assert not _pins_pass()


def test_plant_flipped_site_sign(monkeypatch):
    _plant_unpack(monkeypatch, lambda u: setattr(u, "site_sign", -u.site_sign))
    assert not _pins_pass()


def test_plant_reversed_v(monkeypatch):
    _plant_unpack(monkeypatch, lambda u: setattr(u, "V", u.V[::-1].copy()))
    assert not _pins_pass()


def test_plant_swapped_alpha_beta(monkeypatch):
    def swap(u):
        a = u.alpha.copy(); u.alpha = u.beta.copy(); u.beta = a
    _plant_unpack(monkeypatch, swap)
    assert not _pins_pass()


def test_plant_site_off_by_one(monkeypatch):
    _plant_unpack(monkeypatch, lambda u: setattr(u, "site_pos", ((u.site_pos.astype(int) + 1) % 128).astype(np.uint8)))
    assert not _pins_pass()


def test_plant_wrong_scale_widening(monkeypatch):
    real = wo.widen_fp16
    monkeypatch.setattr(wo, "widen_fp16", lambda b: real(b) * (1 + 2.0 ** -20))
    assert not _pins_pass()


def test_plant_code_offset(monkeypatch):
    _plant_unpack(monkeypatch, lambda u: setattr(u, "T", -u.T))
    assert not _pins_pass()
