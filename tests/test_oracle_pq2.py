"""Pins for the PQ2_0 oracle (CPU only).

The PQ2_0 oracle is checked against things other than itself:
  * hand-derived worked cases (tests/golden/pq2/*.txt): the bytes of the
    packed buffer and the exact product,
  * a pure-Python brute force over the generator arrays,
  * the size the WAL2-Ternary-27B card gives (34 bytes per 128 weights),
  * the layout-v1 oracle on the same matrix with k = 0, r = 0 and
    alpha = d (a separate unpacker and a separate product), and the code bytes
    of each block against the layout-v1 code plane,
  * format rejections,
  * planted mistakes, each of which must make at least one pin fail.
"""
import os
import struct

import numpy as np
import pytest

import oracle
from oracle import pq2_oracle as pq
from oracle.wal_oracle import FormatError
from wal_synth import Components, gen_pq2, gen_x

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "pq2")


def _fixtures():
    return sorted(f[:-4] for f in os.listdir(GOLDEN) if f.endswith(".txt"))


def _load(name):
    lines = []
    with open(os.path.join(GOLDEN, name + ".txt")) as fh:
        for raw in fh:
            line = raw.split("#", 1)[0].strip()
            if line:
                key, val = line.split(":", 1)
                lines.append((key.strip(), val.split()))
    N, K = [int(t) for key, v in lines if key == "shape" for t in v]
    G = K // 128
    T = np.zeros((N, K), np.int8)
    d = np.zeros((N, G), np.uint16)
    x = np.zeros(K, np.uint16)
    y = np.zeros(N)
    hexs = ""
    for key, v in lines:
        if key == "d":
            d[int(v[0]), int(v[1])] = int(v[2], 16)
        elif key == "trit":
            T[int(v[0]), int(v[1])] = int(v[2])
        elif key == "x":
            x[int(v[0])] = int(v[1], 16)
        elif key == "y":
            y[int(v[0])] = float(v[1])
        elif key == "bytes_hex":
            hexs += "".join(v)
    return pq.Pq2(N, K, T, d), x, y, bytes.fromhex(hexs)


@pytest.mark.parametrize("name", _fixtures())
def test_golden_bytes(name):
    p, _, _, raw = _load(name)
    assert pq.pack(p).tobytes() == raw


@pytest.mark.parametrize("name", _fixtures())
def test_golden_product_from_bytes(name):
    p, x, y, raw = _load(name)
    u = pq.unpack(np.frombuffer(raw, np.uint8), p.N, p.K)
    assert np.array_equal(u.T, p.T) and np.array_equal(u.d, p.d)
    assert np.array_equal(pq.matmul(u, x.reshape(1, -1))[0], y)


def _f16(b):
    return struct.unpack("<e", struct.pack("<H", int(b)))[0]


def _bf16(b):
    return struct.unpack("<f", struct.pack("<I", int(b) << 16))[0]


def brute_force(T, d, x_bits):
    """Per-element loops over the generator arrays (no packing)."""
    N, K = T.shape
    x = [_bf16(b) for b in x_bits]
    y = []
    for n in range(N):
        tot = 0.0
        for g in range(K // 128):
            s = 0.0
            for j in range(128 * g, 128 * g + 128):
                t = int(T[n, j])
                if t == 1:
                    s += x[j]
                elif t == -1:
                    s -= x[j]
            tot += _f16(d[n, g]) * s
        y.append(tot)
    return np.array(y)


@pytest.mark.parametrize("N,K", [(1, 128), (3, 256), (5, 384), (2, 512)])
def test_brute_force(N, K):
    T, d = gen_pq2(N, K, 91, N * 1000 + K)
    x = gen_x(K, 1, 91, N + K)[0]
    got = pq.matmul(pq.unpack(pq.pack(pq.Pq2(N, K, T, d)), N, K), x.reshape(1, -1))[0]
    want = brute_force(T, d, x)
    np.testing.assert_allclose(got, want, rtol=1e-12, atol=1e-12 * np.abs(want).max())


def test_size_per_block():
    """32 B of codes + 2 B of FP16 scale per 128 weights = 34 B = 2.125 bit/weight
    (WAL2-Ternary-27B card, section on bit widths)."""
    assert pq.payload_bytes(1, 128) == 34
    assert 8 * pq.payload_bytes(4096, 4096) / (4096 * 4096) == 2.125
    assert pq.packed_bytes(1, 128) == 48


def test_equals_layout_v1_plain_ternary():
    """Same matrix through the layout-v1 oracle with k = 0, r = 0, alpha = d."""
    N, K = 6, 512
    T, d = gen_pq2(N, K, 92, 1)
    X = gen_x(K, 3, 92, 2)
    G = K // 128
    c = Components(N, K, 0, 0, T, np.zeros((N, G, 0), np.uint8), np.zeros((N, G, 0), np.int8), d,
                   np.zeros((N, G), np.uint16), np.zeros((N, 0), np.int8), np.zeros((K, 0), np.int8),
                   np.zeros(0, np.uint16))
    v1 = oracle.unpack(oracle.pack(c), N, K, 0, 0)
    p = pq.unpack(pq.pack(pq.Pq2(N, K, T, d)), N, K)
    np.testing.assert_array_equal(pq.matmul(p, X), oracle.matmul(v1, X))
    # the code bytes of block (n, g) are bytes 32 g .. 32 g + 31 of row n of the v1 code plane
    blocks = pq.pack(pq.Pq2(N, K, T, d))[: N * G * 34].reshape(N, G, 34)
    plane = oracle.pack(c)[0][: N * K // 4].reshape(N, G, 32)
    np.testing.assert_array_equal(blocks[:, :, 2:], plane)


def test_multi_row_activations():
    T, d = gen_pq2(4, 256, 93, 1)
    p = pq.Pq2(4, 256, T, d)
    X = gen_x(256, 5, 93, 2)
    Y = pq.matmul(p, X)
    for m in range(5):
        np.testing.assert_array_equal(Y[m], pq.matmul(p, X[m:m + 1])[0])


def test_rejects_reserved_code():
    T, d = gen_pq2(2, 128, 94, 1)
    buf = pq.pack(pq.Pq2(2, 128, T, d))
    buf[34 + 2 + 5] |= 0x03
    with pytest.raises(FormatError):
        pq.unpack(buf, 2, 128)


def test_rejects_padding_and_size():
    T, d = gen_pq2(1, 128, 94, 2)
    buf = pq.pack(pq.Pq2(1, 128, T, d))
    bad = buf.copy()
    bad[-1] = 1
    with pytest.raises(FormatError):
        pq.unpack(bad, 1, 128)
    with pytest.raises(FormatError):
        pq.unpack(buf[:-16], 1, 128)
    with pytest.raises(FormatError):
        pq.pack(pq.Pq2(1, 100, np.zeros((1, 100), np.int8), np.zeros((1, 1), np.uint16)))


# ---------------------------------------------------------------------------
# planted mistakes must be caught
# ---------------------------------------------------------------------------

def _pins_pass():
    for name in _fixtures():
        p, x, y, raw = _load(name)
        try:
            u = pq.unpack(np.frombuffer(raw, np.uint8), p.N, p.K)
        except FormatError:
            return False
        if pq.pack(p).tobytes() != raw or not np.array_equal(pq.matmul(u, x.reshape(1, -1))[0], y):
            return False
    T, d = gen_pq2(3, 256, 95, 1)
    x = gen_x(256, 1, 95, 2)[0]
    try:
        got = pq.matmul(pq.unpack(pq.pack(pq.Pq2(3, 256, T, d)), 3, 256), x.reshape(1, -1))[0]
    except FormatError:
        return False
    want = brute_force(T, d, x)
    return bool(np.allclose(got, want, rtol=1e-12, atol=1e-12 * np.abs(want).max()))


def test_pins_pass_unplanted():
    assert _pins_pass()


def test_plant_scale_after_codes(monkeypatch):
    monkeypatch.setattr(pq, "SCALE_AT", 32)
    monkeypatch.setattr(pq, "CODES_AT", 0)
    assert not _pins_pass()


def test_plant_codes_one_byte_late(monkeypatch):
    real = pq.unpack

    def bad(buf, N, K):
        p = real(buf, N, K)
        p.T = np.roll(p.T, 4, axis=1)
        return p
    monkeypatch.setattr(pq, "unpack", bad)
    assert not _pins_pass()


def test_plant_negated_code(monkeypatch):
    real = pq.unpack

    def bad(buf, N, K):
        p = real(buf, N, K)
        p.T = -p.T
        return p
    monkeypatch.setattr(pq, "unpack", bad)
    assert not _pins_pass()


def test_plant_scale_of_next_group(monkeypatch):
    real = pq.dense_weight

    def bad(p, rows=None):
        q = pq.Pq2(p.N, p.K, p.T, np.roll(np.asarray(p.d).reshape(p.N, -1), 1, axis=1))
        return real(q, rows)
    monkeypatch.setattr(pq, "dense_weight", bad)
    assert not _pins_pass()
