"""INT4/g128 LM head and INT3/g128 embedding on the GPU vs the FP64 oracle (needs a B200).

LM head tolerance (oracle.check_tolerance, d in the role of alpha): rel-L2 <=
1e-5 and per activation row max-abs <= 1e-3 * ||x_m||_2 * max|d|.  The
embedding is exact: an FP16 scale times a 3-bit integer is an FP32 value.
"""
import numpy as np
import pytest
import torch

from oracle import head_oracle as ho
from wal_synth import gen_int3, gen_int4, gen_x

import oracle_pool
from gpu_util import needs_gpu, wal, device_bf16, stream, assert_parity
from test_oracle_head import _load

pytestmark = [pytest.mark.gpu, needs_gpu]


def _planes(pack, sizes, q, d):
    N, K = q.shape
    sc, ss = sizes(N, K)
    c, s = np.empty(sc, np.uint8), np.empty(ss, np.uint8)
    pack(np.ascontiguousarray(q).ctypes.data, np.ascontiguousarray(d).ctypes.data, N, K, c.ctypes.data, s.ctypes.data)
    return torch.from_numpy(c).cuda(), torch.from_numpy(s.view(np.int16)).cuda()


def _int4_device(q, d):
    w = wal()
    c, s = _planes(w.wal_int4_pack, w.wal_int4_sizes, q, d)
    return w.wal_int4_matrix(q.shape[0], q.shape[1], c.data_ptr(), s.data_ptr()), (c, s)


def _gemm(m, X):
    w = wal()
    M = X.shape[0]
    Y = torch.full((M, m.N), float("nan"), dtype=torch.float32, device="cuda")
    nb = w.wal_int4_workspace_bytes(m, M)
    ws = torch.empty(nb, dtype=torch.uint8, device="cuda")
    w.wal_int4_gemm(m, device_bf16(X).data_ptr(), M, m.K, Y.data_ptr(), m.N, ws.data_ptr(), nb, stream())
    torch.cuda.synchronize()
    w.wal_device_status(ws.data_ptr(), stream())
    return Y.cpu().numpy().astype(np.float64)


SHAPES = [(512, 1024), (37, 384), (1000, 2176), (64, 128), (4096, 4096), (9, 12288), (2051, 4224), (1, 128)]


@pytest.mark.parametrize("N,K", SHAPES)
@pytest.mark.parametrize("M", [1, 4])
def test_int4_parity(N, K, M):
    q, d = gen_int4(N, K, 41, N + K)
    X = gen_x(K, M, 41, N + K + M)
    m, keep = _int4_device(q, d)
    assert_parity(_gemm(m, X), ho.int4_matmul(q, d, X), X, d, f"INT4 {N}x{K} M={M}")


def test_int4_m16():
    q, d = gen_int4(3000, 4096, 42, 1)
    X = gen_x(4096, 16, 42, 2)
    m, keep = _int4_device(q, d)
    assert_parity(_gemm(m, X), ho.int4_matmul(q, d, X), X, d, "INT4 M=16")


def test_int4_golden_exact():
    q, d, x, y, _ = _load("int4_row")
    m, keep = _int4_device(q, d)
    assert _gemm(m, x.reshape(1, -1))[0, 0] == y[0]


def test_int4_extreme_codes():
    """Every code at -8 or +7 with the largest x in each group: the widest
    integer sums the 20-bit image can produce."""
    N, K = 256, 4096
    rng = np.random.default_rng(43)
    q = np.where(rng.random((N, K)) < 0.5, -8, 7).astype(np.int8)
    _, d = gen_int4(N, K, 43, 1)
    X = gen_x(K, 2, 43, 2)
    m, keep = _int4_device(q, d)
    assert_parity(_gemm(m, X), ho.int4_matmul(q, d, X), X, d, "INT4 extreme codes")


def test_int4_lm_head_qwen3_8b_full():
    """The full LM-head shape of an 8B model (vocabulary 151936 x hidden 4096):
    every logit of 2 activation rows checked against the oracle (process pool)."""
    N, K = 151936, 4096
    X = gen_x(K, 2, 44, 2)
    q, d = gen_int4(N, K, 44, 1)
    m, keep = _int4_device(q, d)
    del q
    Y = _gemm(m, X)
    ref = oracle_pool.int4_ref(N, K, 44, 1, X)
    assert_parity(Y, ref, X, d, "LM head")


def _embed(q, d, ids):
    w = wal()
    c, s = _planes(w.wal_int3_pack, w.wal_int3_sizes, q, d)
    t = w.wal_int3_table(q.shape[0], q.shape[1], c.data_ptr(), s.data_ptr())
    idd = torch.tensor(ids, dtype=torch.int32, device="cuda")
    out = torch.full((len(ids), q.shape[1]), float("nan"), dtype=torch.float32, device="cuda")
    ws = torch.empty(512, dtype=torch.uint8, device="cuda")
    w.wal_int3_embed(t, idd.data_ptr(), len(ids), out.data_ptr(), ws.data_ptr(), 512, stream())
    torch.cuda.synchronize()
    return out.cpu().numpy().astype(np.float64), ws


@pytest.mark.parametrize("V,H", [(1000, 4096), (37, 128), (5, 5120)])
def test_int3_embed_exact(V, H):
    q, d = gen_int3(V, H, 45, V + H)
    ids = [0, V - 1, V // 2, 3 % V, V - 1]
    out, ws = _embed(q, d, ids)
    wal().wal_device_status(ws.data_ptr(), stream())
    assert np.array_equal(out, ho.int3_embed(q, d, ids))


def test_int3_golden_row():
    q, d, _, e, _ = _load("int3_row")
    out, _ = _embed(q, d, [0])
    for j, v in e.items():
        assert out[0, j] == v


def test_int3_embed_full_vocab_table():
    """A table of the 8B model's shape (151936 x 4096) and 16 token ids."""
    V, H = 151936, 4096
    q, d = gen_int3(V, H, 46, 1)
    ids = list(np.random.default_rng(46).integers(0, V, 16))
    out, ws = _embed(q, d, ids)
    wal().wal_device_status(ws.data_ptr(), stream())
    assert np.array_equal(out, ho.int3_embed(q, d, ids))


def test_int3_bad_id_reported():
    w = wal()
    q, d = gen_int3(10, 128, 47, 1)
    out, ws = _embed(q, d, [3, 10, -1])
    assert np.array_equal(out[0], ho.int3_embed(q, d, [3])[0])
    assert not out[1].any() and not out[2].any()
    with pytest.raises(w.WalError) as e:
        w.wal_device_status(ws.data_ptr(), stream())
    assert e.value.status == w.WAL_ERR_ARG
