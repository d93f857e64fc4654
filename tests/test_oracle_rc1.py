"""Pins for the RC1 oracle: 24-bit scales and two WALB2 paths (CPU only).

Checked against things other than the oracle itself:
  * hand-derived 24-bit decodings and a hand-derived two-path product
    (tests/golden/rc1/*.txt),
  * a pure-Python brute force (struct-decoded FP32 scales, per-element loops),
  * the layout-v1 oracle on the same matrix when every scale is an FP16 value
    (all ranks in one block there, split over two paths here),
  * invariants: the product is additive over the two paths, and a second
    path equal to the negated first one cancels it,
  * the prepared buffers: path 1's ranks first in U, V and s,
  * planted mistakes.
"""
import os
import struct

import numpy as np
import pytest

import oracle
from oracle import rc1_oracle as rc
from wal_synth import Components, gen_components, gen_rc1, gen_x, f24_bytes_from_f32

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "rc1")


def _lines(name):
    out = []
    with open(os.path.join(GOLDEN, name)) as fh:
        for raw in fh:
            line = raw.split("#", 1)[0].strip()
            if line:
                key, val = line.split(":", 1)
                out.append((key.strip(), val.split()))
    return out


def _b24(h):
    return np.frombuffer(bytes.fromhex(h), np.uint8)


def _num(tok):
    return float.fromhex(tok) if tok.lstrip("-").startswith("0x") else float(tok)


def load_product():
    lines = _lines("two_paths.txt")
    N, K, k, r1, r2 = [int(t) for key, v in lines if key == "shape" for t in v]
    G = K // 128
    T = np.zeros((N, K), np.int8)
    a24 = np.zeros((N, G, 3), np.uint8)
    b24 = np.zeros((N, G, 3), np.uint8)
    sites = {}
    U1, U2 = np.ones((N, r1), np.int8), np.ones((N, r2), np.int8)
    V1, V2 = np.ones((K, r1), np.int8), np.ones((K, r2), np.int8)
    s1, s2 = np.zeros((r1, 3), np.uint8), np.zeros((r2, 3), np.uint8)
    x = np.zeros(K, np.uint16)
    y = np.zeros(N)
    for key, v in lines:
        if key == "alpha24":
            a24[int(v[0]), int(v[1])] = _b24(v[2])
        elif key == "beta24":
            b24[int(v[0]), int(v[1])] = _b24(v[2])
        elif key == "trit":
            T[int(v[0]), int(v[1])] = int(v[2])
        elif key == "site":
            sites.setdefault((int(v[0]), int(v[1])), []).append((int(v[2]), int(v[3])))
        elif key == "s1":
            s1[int(v[0])] = _b24(v[1])
        elif key == "s2":
            s2[int(v[0])] = _b24(v[1])
        elif key == "u1neg":
            U1[int(v[0]), int(v[1])] = -1
        elif key == "u2neg":
            U2[int(v[0]), int(v[1])] = -1
        elif key == "v1neg":
            V1[int(v[0]), int(v[1])] = -1
        elif key == "v2neg":
            V2[int(v[0]), int(v[1])] = -1
        elif key == "x":
            x[int(v[0])] = int(v[1], 16)
        elif key == "y":
            y[int(v[0])] = float(v[1])
    pos = np.zeros((N, G, k), np.uint8)
    sgn = np.ones((N, G, k), np.int8)
    for (n, g), lst in sites.items():
        for i, (p, s) in enumerate(sorted(lst)):
            pos[n, g, i], sgn[n, g, i] = p, s
    return rc.Rc1(N, K, k, T, pos, sgn, a24, b24, U1, V1, s1, U2, V2, s2), x, y


def test_golden_decode():
    for key, v in _lines("decode.txt"):
        assert rc.f24_to_f64(_b24(v[0]))[()] == _num(v[1]), v


def test_golden_two_path_product():
    c, x, y = load_product()
    assert np.array_equal(rc.matmul(c, x.reshape(1, -1))[0], y)


def _f32(u):
    return struct.unpack("<f", struct.pack("<I", int(u)))[0]


def brute_force(d, x_bits):
    """Per-element loops; 24-bit values decoded with struct."""
    N, K, k = d["N"], d["K"], d["k"]
    dec = lambda b: _f32((int(b[0]) | int(b[1]) << 8 | int(b[2]) << 16) << 8)
    x = [_f32(int(b) << 16) for b in x_bits]
    y = []
    for n in range(N):
        tot = 0.0
        for g in range(K // 128):
            tx = sum(int(d["T"][n, j]) * x[j] for j in range(128 * g, 128 * g + 128))
            rx = sum(int(d["site_sign"][n, g, i]) * x[128 * g + int(d["site_pos"][n, g, i])] for i in range(k))
            tot += dec(d["alpha24"][n, g]) * tx + (dec(d["beta24"][n, g]) * rx if k else 0.0)
        for U, V, s in ((d["U1"], d["V1"], d["s1"]), (d["U2"], d["V2"], d["s2"])):
            for rho in range(U.shape[1]):
                z = sum(int(V[j, rho]) * x[j] for j in range(K))
                tot += dec(s[rho]) * int(U[n, rho]) * z
        y.append(tot)
    return np.array(y)


def _rc1(d):
    return rc.Rc1(d["N"], d["K"], d["k"], d["T"], d["site_pos"], d["site_sign"], d["alpha24"], d["beta24"],
                  d["U1"], d["V1"], d["s1"], d["U2"], d["V2"], d["s2"])


@pytest.mark.parametrize("N,K,k,r1,r2", [(2, 128, 8, 1, 2), (3, 256, 0, 2, 0), (1, 384, 4, 0, 3), (2, 256, 2, 2, 2)])
def test_brute_force(N, K, k, r1, r2):
    d = gen_rc1(N, K, k, r1, r2, 61, N + K + k)
    x = gen_x(K, 1, 61, K)[0]
    got = rc.matmul(_rc1(d), x.reshape(1, -1))[0]
    want = brute_force(d, x)
    np.testing.assert_allclose(got, want, rtol=1e-12, atol=1e-12 * np.abs(want).max())


def _f24_from_fp16(bits):
    """FP16 values are exact in the 24-bit format (the writer's rounding leaves them unchanged)."""
    return f24_bytes_from_f32(np.asarray(bits, np.uint16).view(np.float16).astype(np.float32))


@pytest.mark.parametrize("split", [(8, 0), (3, 5), (0, 8)])
def test_equals_layout_v1_with_fp16_scales(split):
    r1, r2 = split
    c = gen_components(6, 512, 4, r1 + r2, config_id=62, matrix_index=1)
    X = gen_x(512, 2, 62, 3)
    m = rc.Rc1(c.N, c.K, c.k, c.T, c.site_pos, c.site_sign, _f24_from_fp16(c.alpha), _f24_from_fp16(c.beta),
               c.U[:, :r1], c.V[:, :r1], _f24_from_fp16(c.lr_scale[:r1]), c.U[:, r1:], c.V[:, r1:],
               _f24_from_fp16(c.lr_scale[r1:]))
    np.testing.assert_array_equal(rc.dense_weight(m), oracle.dense_weight(c))
    np.testing.assert_array_equal(rc.matmul(m, X), oracle.matmul(c, X))


def test_additive_over_paths_and_cancellation():
    d = gen_rc1(5, 384, 8, 4, 3, 63, 1)
    m = _rc1(d)
    z = lambda r: (np.zeros((5, r), np.int8), np.zeros((384, r), np.int8), np.zeros((r, 3), np.uint8))
    base = rc.dense_weight(rc.Rc1(5, 384, 8, d["T"], d["site_pos"], d["site_sign"], d["alpha24"], d["beta24"],
                                  *z(0), *z(0)))
    only1 = rc.dense_weight(rc.Rc1(5, 384, 8, d["T"], d["site_pos"], d["site_sign"], d["alpha24"], d["beta24"],
                                   d["U1"], d["V1"], d["s1"], *z(0)))
    only2 = rc.dense_weight(rc.Rc1(5, 384, 8, d["T"], d["site_pos"], d["site_sign"], d["alpha24"], d["beta24"],
                                   *z(0), d["U2"], d["V2"], d["s2"]))
    np.testing.assert_allclose(rc.dense_weight(m), only1 + only2 - base, rtol=0, atol=1e-15)
    canc = rc.Rc1(5, 384, 8, d["T"], d["site_pos"], d["site_sign"], d["alpha24"], d["beta24"],
                  d["U1"], d["V1"], d["s1"], -d["U1"], d["V1"], d["s1"])
    np.testing.assert_array_equal(rc.dense_weight(canc), base)


def test_prepared_concatenation_by_hand():
    """Path 1's ranks come first: rank 0 from U1, ranks 1-2 from U2; s decoded to FP32."""
    U1 = np.array([[-1], [1]], np.int8)
    U2 = np.array([[1, -1], [-1, -1]], np.int8)
    V1 = np.ones((128, 1), np.int8)
    V2 = np.ones((128, 2), np.int8)
    V2[3, 1] = -1
    s1 = _b24("00803F")[None]
    s2 = np.stack([_b24("00003F"), _b24("00803E")])
    m = rc.Rc1(2, 128, 0, np.zeros((2, 128), np.int8), np.zeros((2, 1, 0), np.uint8), np.zeros((2, 1, 0), np.int8),
               np.stack([_b24("00803F")] * 2).reshape(2, 1, 3), np.zeros((2, 1, 3), np.uint8), U1, V1, s1, U2, V2, s2)
    sc, ub, vb, lr = rc.prepared(m)
    # row 0: U = [-1, +1, -1] -> bits 0 and 2 -> 0b101; row 1: [+1, -1, -1] -> bits 1, 2 -> 0b110
    assert list(ub[:8].view('<u4')) == [0b101, 0b110]
    # V bit rows (K / 32 = 4 words per rank): ranks 0 and 1 all +1; rank 2 has -1 at column 3
    assert list(vb[:48].view('<u4')) == [0, 0, 0, 0, 0, 0, 0, 0, 0b1000, 0, 0, 0]
    assert list(lr[:12].view('<f4')) == [1.0, 0.5, 0.25]
    assert list(sc[:8].view('<f4')) == [1.0, 1.0]


# ---------------------------------------------------------------------------
# planted mistakes
# ---------------------------------------------------------------------------

def _pins_pass():
    try:
        for key, v in _lines("decode.txt"):
            if rc.f24_to_f64(_b24(v[0]))[()] != _num(v[1]):
                return False
        c, x, y = load_product()
        if not np.array_equal(rc.matmul(c, x.reshape(1, -1))[0], y):
            return False
        d = gen_rc1(2, 256, 2, 2, 2, 64, 1)
        x = gen_x(256, 1, 64, 2)[0]
        got = rc.matmul(_rc1(d), x.reshape(1, -1))[0]
        want = brute_force(d, x)
        if not np.allclose(got, want, rtol=1e-12, atol=1e-12 * np.abs(want).max()):
            return False
        m = rc.Rc1(1, 128, 0, np.zeros((1, 128), np.int8), np.zeros((1, 1, 0), np.uint8), np.zeros((1, 1, 0), np.int8),
                   _b24("00803F").reshape(1, 1, 3), np.zeros((1, 1, 3), np.uint8), np.array([[-1]], np.int8),
                   np.ones((128, 1), np.int8), _b24("00803F")[None], np.array([[1]], np.int8),
                   np.ones((128, 1), np.int8), _b24("00003F")[None])
        _, ub, _, lr = rc.prepared(m)
        return int(ub[:4].view('<u4')[0]) == 1 and list(lr[:8].view('<f4')) == [1.0, 0.5]
    except Exception:
        return False


def test_pins_pass_unplanted():
    assert _pins_pass()


def test_plant_wrong_decode_shift(monkeypatch):
    monkeypatch.setattr(rc, "F24_SHIFT", 7)
    assert not _pins_pass()


def test_plant_dropped_second_path(monkeypatch):
    real = rc.dense_weight

    def bad(c, rows=None):
        z = np.zeros((c.N, 0), np.int8)
        return real(rc.Rc1(c.N, c.K, c.k, c.T, c.site_pos, c.site_sign, c.alpha24, c.beta24, c.U1, c.V1, c.s1,
                           z, np.zeros((c.K, 0), np.int8), np.zeros((0, 3), np.uint8)), rows)
    monkeypatch.setattr(rc, "dense_weight", bad)
    assert not _pins_pass()


def test_plant_paths_swapped_in_prepared(monkeypatch):
    real = rc.prepared

    def bad(c):
        return real(rc.Rc1(c.N, c.K, c.k, c.T, c.site_pos, c.site_sign, c.alpha24, c.beta24,
                           c.U2, c.V2, c.s2, c.U1, c.V1, c.s1))
    monkeypatch.setattr(rc, "prepared", bad)
    assert not _pins_pass()
