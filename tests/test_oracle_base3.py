"""Pins for the base-3 container oracle and its conversion (CPU only).

Checked against things other than the oracle itself:
  * hand-derived bytes (tests/golden/base3/row128.txt): base-3 bytes and the
    layout-v1 code plane of one row,
  * hand-derived BF16 -> FP16 roundings (tests/golden/base3/scales.txt),
  * a pure-Python digit expansion (divmod by 3) on tiny inputs,
  * the 8 / 5 bits per symbol of the WAL2-Ternary-27B card (section on bit widths),
  * the layout-v1 oracle's own packer for the converted code plane,
  * format rejections and planted mistakes.
"""
import os

import numpy as np
import pytest

import oracle
from oracle import base3_oracle as b3
from oracle.wal_oracle import FormatError
from wal_synth import Components, gen_base3

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "base3")


def _lines(name):
    out = []
    with open(os.path.join(GOLDEN, name)) as fh:
        for raw in fh:
            line = raw.split("#", 1)[0].strip()
            if line:
                key, val = line.split(":", 1)
                out.append((key.strip(), val.split()))
    return out


def load_row():
    lines = _lines("row128.txt")
    N, K = [int(t) for k, v in lines if k == "shape" for t in v]
    T = np.zeros((N, K), np.int8)
    for k, v in lines:
        if k == "trit":
            T[int(v[0]), int(v[1])] = int(v[2])
    hexes = {k: bytes.fromhex("".join("".join(v) for kk, v in lines if kk == k)) for k in ("bytes_hex", "codes_hex")}
    return T, hexes["bytes_hex"], hexes["codes_hex"]


def load_scales():
    lines = _lines("scales.txt")
    pairs = [(int(v[0], 16), int(v[1], 16)) for k, v in lines if k == "pair"]
    over = [int(v[0], 16) for k, v in lines if k == "overflow"]
    return pairs, over


def v1_codes(T):
    N, K = T.shape
    G = K // 128
    c = Components(N, K, 0, 0, T, np.zeros((N, G, 0), np.uint8), np.zeros((N, G, 0), np.int8),
                   np.zeros((N, G), np.uint16), np.zeros((N, G), np.uint16), np.zeros((N, 0), np.int8),
                   np.zeros((K, 0), np.int8), np.zeros(0, np.uint16))
    return oracle.pack(c)[0]


def test_golden_bytes():
    T, raw, _ = load_row()
    assert b3.pack(T).tobytes() == raw
    assert np.array_equal(b3.unpack(np.frombuffer(raw, np.uint8), *T.shape), T)


def test_golden_conversion():
    T, raw, codes_hex = load_row()
    codes, alpha = b3.convert(np.frombuffer(raw, np.uint8), np.array([[0x3F80]], np.uint16), 1, 128)
    assert codes.tobytes() == codes_hex
    assert alpha[:2].tobytes() == bytes([0x00, 0x3C]) and not alpha[2:].any()


def test_golden_scales():
    pairs, over = load_scales()
    got = b3.bf16_to_fp16_bits(np.array([p[0] for p in pairs], np.uint16))
    assert [int(g) for g in got] == [p[1] for p in pairs]
    for o in over:
        with pytest.raises(FormatError):
            b3.bf16_to_fp16_bits(np.array([o], np.uint16))
    with pytest.raises(FormatError):
        b3.bf16_to_fp16_bits(np.array([0x7FC0], np.uint16))  # a NaN scale


def _digits_by_hand(byte):
    out = []
    for _ in range(5):
        byte, r = divmod(byte, 3)
        out.append(r)
    return out


@pytest.mark.parametrize("N,K", [(1, 128), (2, 256), (3, 640), (2, 1152)])
def test_brute_force_digits(N, K):
    T, _ = gen_base3(N, K, 71, N + K)
    raw = b3.pack(T)
    P = (K + 4) // 5
    for n in range(N):
        trits = []
        for m in range(P):
            trits += [d - 1 for d in _digits_by_hand(int(raw[n * P + m]))]
        assert trits[:K] == [int(t) for t in T[n]]
        assert all(t == -1 for t in trits[K:])  # digits 0 past the row's end


def test_bits_per_symbol():
    """Five trits per byte: 8 / 5 = 1.6 bits per symbol (K a multiple of 5 here)."""
    assert b3.row_bytes(5120) * 8 / 5120 == 1.6
    assert b3.row_bytes(4096) == 820 and b3.row_bytes(128) == 26


@pytest.mark.parametrize("N,K", [(4, 128), (3, 4096), (2, 12288), (5, 5120), (1, 17408)])
def test_conversion_equals_layout_v1_packer(N, K):
    T, s = gen_base3(N, K, 72, N + K)
    codes, alpha = b3.convert(b3.pack(T), s, N, K)
    assert np.array_equal(codes, v1_codes(T))
    want = (s.astype(np.uint32) << 16).view(np.float32).astype(np.float16).view(np.uint16)
    assert np.array_equal(alpha[: want.size * 2].view('<u2').reshape(want.shape), want)


def test_rejections():
    T, _ = gen_base3(2, 128, 73, 1)
    raw = b3.pack(T)
    bad = raw.copy()
    bad[3] = 243
    with pytest.raises(FormatError):
        b3.unpack(bad, 2, 128)
    bad = raw.copy()
    bad[25] += 27  # digit 3 of the row's last byte: past the row's end
    with pytest.raises(FormatError):
        b3.unpack(bad, 2, 128)
    bad = raw.copy()
    bad[-1] = 1
    with pytest.raises(FormatError):
        b3.unpack(bad, 2, 128)
    with pytest.raises(FormatError):
        b3.unpack(raw[:-16], 2, 128)


# ---------------------------------------------------------------------------
# planted mistakes
# ---------------------------------------------------------------------------

def _pins_pass():
    T, raw, codes_hex = load_row()
    try:
        if b3.pack(T).tobytes() != raw:
            return False
        codes, _ = b3.convert(np.frombuffer(raw, np.uint8), np.array([[0x3F80]], np.uint16), 1, 128)
        if codes.tobytes() != codes_hex:
            return False
        pairs, _ = load_scales()
        got = b3.bf16_to_fp16_bits(np.array([p[0] for p in pairs], np.uint16))
        if [int(g) for g in got] != [p[1] for p in pairs]:
            return False
    except FormatError:
        return False
    T2, _ = gen_base3(2, 256, 74, 1)
    raw2 = b3.pack(T2)
    for n in range(2):
        trits = []
        for m in range(52):
            trits += [d - 1 for d in _digits_by_hand(int(raw2[n * 52 + m]))]
        if trits[:256] != [int(t) for t in T2[n]]:
            return False
    return True


def test_pins_pass_unplanted():
    assert _pins_pass()


def test_plant_reversed_digit_order(monkeypatch):
    monkeypatch.setattr(b3, "DIGIT_WEIGHTS", (81, 27, 9, 3, 1))
    assert not _pins_pass()


def test_plant_truncating_scale_conversion(monkeypatch):
    def trunc(s_bits):
        # the FP16 value next to the input on the side of zero (round toward zero)
        f = (np.asarray(s_bits, np.uint16).astype(np.uint32) << 16).view(np.float32)
        h = f.astype(np.float16)
        away = np.abs(h.astype(np.float32)) > np.abs(f)
        h[away] = np.nextafter(h[away], np.float16(0))
        return h.view(np.uint16)
    monkeypatch.setattr(b3, "bf16_to_fp16_bits", trunc)
    assert not _pins_pass()


def test_plant_digit_offset(monkeypatch):
    real = b3.unpack

    def bad(buf, N, K):
        return np.clip(real(buf, N, K) + 1, -1, 1).astype(np.int8)
    monkeypatch.setattr(b3, "unpack", bad)
    assert not _pins_pass()
