"""Pins for the INT4/g128 LM-head and INT3/g128 embedding oracle (CPU only).

Checked against things other than the oracle itself:
  * hand-derived bytes and results (tests/golden/head/*.txt),
  * pure-Python brute force (bit-by-bit decoding, per-element loops),
  * the layout-v1 oracle: an INT4 matrix whose values are in {-1, 0, 1} is a
    plain ternary matrix with alpha = d,
  * range and size checks, planted mistakes.
"""
import os
import struct

import numpy as np
import pytest

import oracle
from oracle import head_oracle as ho
from oracle.wal_oracle import FormatError
from wal_synth import Components, gen_int3, gen_int4, gen_x

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "head")


def _load(name):
    lines = []
    with open(os.path.join(GOLDEN, name + ".txt")) as fh:
        for raw in fh:
            line = raw.split("#", 1)[0].strip()
            if line:
                key, val = line.split(":", 1)
                lines.append((key.strip(), val.split()))
    N, K = [int(t) for k, v in lines if k == "shape" for t in v]
    q = np.zeros((N, K), np.int8)
    d = np.zeros((N, K // 128), np.uint16)
    x = np.zeros(K, np.uint16)
    out = {}
    hx = ""
    for k, v in lines:
        if k == "q":
            q[int(v[0]), int(v[1])] = int(v[2])
        elif k == "d":
            d[int(v[0]), int(v[1])] = int(v[2], 16)
        elif k == "x":
            x[int(v[0])] = int(v[1], 16)
        elif k in ("y", "e"):
            out[int(v[0])] = float(v[1])
        elif k == "codes_hex":
            hx += "".join(v)
    return q, d, x, out, bytes.fromhex(hx)


def test_int4_golden():
    q, d, x, y, raw = _load("int4_row")
    codes, scales = ho.int4_pack(q, d)
    assert codes[: len(raw)].tobytes() == raw
    q2, d2 = ho.int4_unpack(codes, scales, 1, 128)
    assert np.array_equal(q2, q) and np.array_equal(d2, d)
    assert ho.int4_matmul(q2, d2, x.reshape(1, -1))[0, 0] == y[0]


def test_int3_golden():
    q, d, _, e, raw = _load("int3_row")
    codes, scales = ho.int3_pack(q, d)
    assert codes[: len(raw)].tobytes() == raw
    q2, d2 = ho.int3_unpack(codes, scales, 1, 128)
    assert np.array_equal(q2, q)
    emb = ho.int3_embed(q2, d2, [0])[0]
    for j, v in e.items():
        assert emb[j] == v


def _f16(b):
    return struct.unpack("<e", struct.pack("<H", int(b)))[0]


def _bf16(b):
    return struct.unpack("<f", struct.pack("<I", int(b) << 16))[0]


@pytest.mark.parametrize("N,K", [(1, 128), (3, 256), (2, 384)])
def test_int4_brute_force(N, K):
    q, d = gen_int4(N, K, 51, N + K)
    x = gen_x(K, 1, 51, K)[0]
    codes, scales = ho.int4_pack(q, d)
    raw = codes.tobytes()
    xs = [_bf16(b) for b in x]
    want = []
    for n in range(N):
        tot = 0.0
        for g in range(K // 128):
            acc = 0.0
            for j in range(128 * g, 128 * g + 128):
                byte = raw[n * K // 2 + j // 2]
                u = (byte >> (4 * (j % 2))) & 15
                acc += (u - 8) * xs[j]
            tot += _f16(d[n, g]) * acc
        want.append(tot)
    got = ho.int4_matmul(*ho.int4_unpack(codes, scales, N, K), x.reshape(1, -1))[0]
    np.testing.assert_allclose(got, want, rtol=1e-12, atol=1e-12 * np.abs(want).max())


@pytest.mark.parametrize("V,H", [(2, 128), (3, 256)])
def test_int3_brute_force(V, H):
    q, d = gen_int3(V, H, 52, V + H)
    codes, scales = ho.int3_pack(q, d)
    raw = codes.tobytes()
    for t in range(V):
        for j in range(H):
            g, jj = divmod(j, 128)
            base = (t * (H // 128) + g) * 48
            u = 0
            for i in range(3):
                bit = 3 * jj + i
                u |= ((raw[base + bit // 8] >> (bit % 8)) & 1) << i
            assert u - 4 == q[t, j]
    e = ho.int3_embed(*ho.int3_unpack(codes, scales, V, H), [V - 1, 0])
    assert e[0, 5] == _f16(d[V - 1, 0]) * int(q[V - 1, 5])


def test_int4_ternary_values_equal_layout_v1():
    N, K = 5, 512
    rng = np.random.default_rng(53)
    q = rng.integers(-1, 2, size=(N, K)).astype(np.int8)
    _, d = gen_int4(N, K, 53, 1)
    G = K // 128
    c = Components(N, K, 0, 0, q, np.zeros((N, G, 0), np.uint8), np.zeros((N, G, 0), np.int8), d,
                   np.zeros((N, G), np.uint16), np.zeros((N, 0), np.int8), np.zeros((K, 0), np.int8),
                   np.zeros(0, np.uint16))
    X = gen_x(K, 2, 53, 2)
    np.testing.assert_array_equal(ho.int4_matmul(*ho.int4_unpack(*ho.int4_pack(q, d), N, K), X),
                                  oracle.matmul(oracle.unpack(oracle.pack(c), N, K, 0, 0), X))


def test_sizes_and_ranges():
    q, d = gen_int4(3, 256, 54, 1)
    codes, scales = ho.int4_pack(q, d)
    assert codes.size == 384 and scales.size == 16
    q3, d3 = gen_int3(3, 256, 54, 2)
    c3, s3 = ho.int3_pack(q3, d3)
    assert c3.size == 288  # 3 * 256 * 3 / 8
    with pytest.raises(FormatError):
        ho.int4_pack(np.full((1, 128), 8, np.int8), np.zeros((1, 1), np.uint16))
    with pytest.raises(FormatError):
        ho.int3_pack(np.full((1, 128), -5, np.int8), np.zeros((1, 1), np.uint16))
    with pytest.raises(FormatError):
        ho.int3_embed(q3, d3, [3])
    bad = codes.copy()
    with pytest.raises(FormatError):
        ho.int4_unpack(bad[:-16], scales, 3, 256)


# ---------------------------------------------------------------------------
# planted mistakes
# ---------------------------------------------------------------------------

def _pins_pass():
    try:
        q, d, x, y, raw = _load("int4_row")
        codes, scales = ho.int4_pack(q, d)
        if codes[: len(raw)].tobytes() != raw:
            return False
        if ho.int4_matmul(*ho.int4_unpack(np.frombuffer(raw, np.uint8).copy(), scales, 1, 128),
                          x.reshape(1, -1))[0, 0] != y[0]:
            return False
        q3, d3, _, e, raw3 = _load("int3_row")
        if ho.int3_pack(q3, d3)[0][: len(raw3)].tobytes() != raw3:
            return False
        c3 = np.frombuffer(raw3, np.uint8).copy()
        emb = ho.int3_embed(*ho.int3_unpack(c3, ho.int3_pack(q3, d3)[1], 1, 128), [0])[0]
        return all(emb[j] == v for j, v in e.items())
    except FormatError:
        return False


def test_pins_pass_unplanted():
    assert _pins_pass()


def test_plant_nibble_order(monkeypatch):
    monkeypatch.setattr(ho, "INT4_HIGH_FIRST", True)
    assert not _pins_pass()


def test_plant_int4_offset(monkeypatch):
    monkeypatch.setattr(ho, "INT4_OFFSET", 7)
    assert not _pins_pass()


def test_plant_int3_offset(monkeypatch):
    monkeypatch.setattr(ho, "INT3_OFFSET", 3)
    assert not _pins_pass()
