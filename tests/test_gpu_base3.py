"""GPU conversion of the base-3 container to layout v1 vs the oracle (needs a B200).

Integer and byte work: the code plane and the FP16 scale plane must equal
the oracle's bit for bit.
"""
import numpy as np
import pytest
import torch

import oracle
from oracle import base3_oracle as b3
from wal_synth import Components, gen_base3, gen_x

from gpu_util import needs_gpu, wal, stream, assert_parity
from test_oracle_base3 import load_row, load_scales

pytestmark = [pytest.mark.gpu, needs_gpu]


def _convert(raw, s, N, K):
    w = wal()
    sizes = w.wal_packed_sizes(N, K, 0, 0)
    b3d = torch.from_numpy(np.ascontiguousarray(raw)).cuda()
    sd = torch.from_numpy(np.ascontiguousarray(s, np.uint16).view(np.int16).reshape(-1)).cuda()
    codes = torch.full((sizes[0],), 0xA5, dtype=torch.uint8, device="cuda")
    alpha = torch.full((sizes[2],), 0xA5, dtype=torch.uint8, device="cuda")
    ws = torch.empty(512, dtype=torch.uint8, device="cuda")
    w.wal_base3_convert(b3d.data_ptr(), sd.data_ptr(), N, K, codes.data_ptr(), alpha.data_ptr(), ws.data_ptr(), 512,
                        stream())
    return codes.cpu().numpy(), alpha.cpu().numpy()


def _packed(T):
    N, K = T.shape
    out = np.empty(wal().wal_base3_bytes(N, K), np.uint8)
    wal().wal_base3_pack(T.ctypes.data, N, K, out.ctypes.data)
    return out


# K mod 5 = 3, 1, 4, 2, 0 and model widths
SHAPES = [(1, 128), (3, 256), (7, 384), (5, 512), (9, 640), (100, 4096), (33, 5120), (21, 12288), (4, 17408),
          (1000, 1152), (2048, 4096)]


@pytest.mark.parametrize("N,K", SHAPES)
def test_base3_convert_bit_exact(N, K):
    T, s = gen_base3(N, K, 76, N + K)
    raw = b3.pack(T)
    codes, alpha = _convert(raw, s, N, K)
    want_c, want_a = b3.convert(raw, s, N, K)
    assert np.array_equal(codes, want_c)
    assert np.array_equal(alpha, want_a)


def test_base3_golden_row():
    T, raw, codes_hex = load_row()
    codes, alpha = _convert(np.frombuffer(raw, np.uint8).copy(), np.array([[0x3F80]], np.uint16), 1, 128)
    assert codes.tobytes() == codes_hex
    assert alpha[:2].tobytes() == bytes([0x00, 0x3C]) and not alpha[2:].any()


def test_base3_golden_scales():
    pairs, _ = load_scales()
    G = len(pairs)
    T = np.zeros((1, 128 * G), np.int8)
    s = np.array([[p[0] for p in pairs]], np.uint16)
    _, alpha = _convert(_packed(T), s, 1, 128 * G)
    assert [int(v) for v in alpha[: 2 * G].view('<u2')] == [p[1] for p in pairs]


@pytest.mark.parametrize("what", ["byte", "tail", "overflow", "nan"])
def test_base3_rejections(what):
    w = wal()
    T, s = gen_base3(3, 256, 77, 1)
    raw = _packed(T)
    s = s.copy()
    if what == "byte":
        raw[60] = 250
    elif what == "tail":
        raw[51] += 81  # digit 4 of row 0's last byte (256 = 5 * 51 + 1)
    elif what == "overflow":
        s[1, 1] = 0x4780
    else:
        s[2, 0] = 0x7FC0
    with pytest.raises(w.WalError) as e:
        _convert(raw, s, 3, 256)
    assert e.value.status == w.WAL_ERR_FORMAT


def test_base3_prepared_matrix_runs_the_product():
    """Convert on the GPU, then run the batch-1 product of the prepared layout-v1
    matrix (k = 0, r = 0) and check it against the oracle's product of T and the
    converted scales."""
    w = wal()
    N, K = 3000, 4096
    T, s = gen_base3(N, K, 78, 1)
    codes, alpha = _convert(_packed(T), s, N, K)
    G = K // 128
    zero = np.zeros(16, np.uint8)
    pm = w.PackedMatrix([codes, zero[:0], alpha, zero[:0], zero[:0], zero[:0]], N, K, 0, 0)
    x = gen_x(K, 1, 78, 2)
    y = torch.empty(N, dtype=torch.float32, device="cuda")
    ws = torch.empty(pm.workspace_bytes(1), dtype=torch.uint8, device="cuda")
    xd = torch.from_numpy(x.view(np.int16)).cuda()
    w.wal_gemv(pm.desc, xd.data_ptr(), y.data_ptr(), ws.data_ptr(), ws.numel(), stream())
    torch.cuda.synchronize()
    a16 = b3.bf16_to_fp16_bits(s)
    c = Components(N, K, 0, 0, T, np.zeros((N, G, 0), np.uint8), np.zeros((N, G, 0), np.int8), a16,
                   np.zeros((N, G), np.uint16), np.zeros((N, 0), np.int8), np.zeros((K, 0), np.int8),
                   np.zeros(0, np.uint16))
    assert_parity(y.cpu().numpy().astype(np.float64), oracle.matvec(c, x[0]), x[0], a16, "prepared")
