"""PQ2_0 plain-ternary products vs the FP64 oracle, through the C ABI (needs a B200).

Tolerance (applied by oracle.check_tolerance, with d in the role of alpha):
  rel-L2 = ||y - y*||_2 / ||y*||_2 <= 1e-5 over the whole output, and
  max |y_m - y*_m| <= 1e-3 * ||x_m||_2 * max|d| for every activation row m.
"""
import os

import numpy as np
import pytest
import torch

import oracle
from oracle import pq2_oracle as pq
from wal_synth import config_plan, gen_pq2, gen_x, body_plan, LAYER_8B

import oracle_pool
from gpu_util import needs_gpu, wal, device_bf16, stream, assert_parity

pytestmark = [pytest.mark.gpu, needs_gpu]

SHAPES = [
    (512, 1024),     # one K-slice, eight blocks per row
    (37, 384),       # ragged N, three blocks
    (1000, 2176),    # two K-slices, the second one a single block
    (64, 128),       # one block per row
    (4096, 4096),    # a q-shaped matrix: one full K-slice
    (9, 12288),      # three K-slices (down-shaped K)
    (2051, 4224),    # ragged rows and slices
    (1, 128),        # a single row
    (333, 5120),     # 27B hidden size: 40 blocks per row
    (130, 17408),    # 27B MLP width: 136 blocks per row, five K-slices
]


def _device(T, d, N, K):
    w = wal()
    return w.Pq2Matrix(w.pack_pq2_host(T, d, N, K), N, K)


def _gemm(pm, X_dev, M):
    w = wal()
    Y = torch.full((M, pm.N), float("nan"), dtype=torch.float32, device="cuda")
    nb = pm.workspace_bytes(M)
    ws = torch.empty(nb, dtype=torch.uint8, device="cuda")
    w.wal_pq2_gemm(pm.desc, X_dev.data_ptr(), M, pm.K, Y.data_ptr(), pm.N, ws.data_ptr(), nb, stream())
    torch.cuda.synchronize()
    w.wal_device_status(ws.data_ptr(), stream())
    return Y.cpu().numpy().astype(np.float64)


@pytest.mark.parametrize("N,K", SHAPES)
@pytest.mark.parametrize("M", [1, 3])
def test_pq2_parity(N, K, M):
    T, d = gen_pq2(N, K, 96, N + K)
    X = gen_x(K, M, 96, 7 * N + K + M)
    Y = _gemm(_device(T, d, N, K), device_bf16(X), M)
    assert_parity(Y, pq.matmul(pq.Pq2(N, K, T, d), X), X, d, f"PQ2_0 {N}x{K} M={M}")


def test_pq2_parity_m16():
    N, K = 700, 4096
    T, d = gen_pq2(N, K, 96, 1)
    X = gen_x(K, 16, 96, 2)
    Y = _gemm(_device(T, d, N, K), device_bf16(X), 16)
    assert_parity(Y, pq.matmul(pq.Pq2(N, K, T, d), X), X, d, "PQ2_0 M=16")


GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "pq2")


@pytest.mark.parametrize("name", sorted(f[:-4] for f in os.listdir(GOLDEN) if f.endswith(".txt")))
def test_pq2_golden_exact(name):
    """The hand-derived cases are dyadic: the kernel's result must be exact."""
    from test_oracle_pq2 import _load
    p, x, y, raw = _load(name)
    pm = wal().Pq2Matrix(np.frombuffer(raw, np.uint8).copy(), p.N, p.K)
    got = _gemm(pm, device_bf16(x.reshape(1, -1)), 1)[0]
    assert np.array_equal(got, y), (got, y)


def test_pq2_odd_symmetry_and_reruns():
    N, K = 1500, 4096
    T, d = gen_pq2(N, K, 97, 1)
    X = gen_x(K, 1, 97, 2)
    pm = _device(T, d, N, K)
    y1 = _gemm(pm, device_bf16(X), 1)
    y2 = _gemm(pm, device_bf16(X), 1)
    yn = _gemm(pm, device_bf16(X ^ np.uint16(0x8000)), 1)
    assert np.array_equal(y1, y2), "reruns differ"
    assert np.array_equal(yn, -y1), "y(-x) != -y(x)"


def test_pq2_matches_layout_v1_path():
    """The same plain-ternary matrix through the layout-v1 product (k = 0, r = 0)."""
    from gpu_util import device_matrix, run_gemm
    from wal_synth import Components
    N, K = 3000, 4096
    T, d = gen_pq2(N, K, 98, 1)
    G = K // 128
    c = Components(N, K, 0, 0, T, np.zeros((N, G, 0), np.uint8), np.zeros((N, G, 0), np.int8), d,
                   np.zeros((N, G), np.uint16), np.zeros((N, 0), np.int8), np.zeros((K, 0), np.int8),
                   np.zeros(0, np.uint16))
    X = gen_x(K, 2, 98, 2)
    y_pq2 = _gemm(_device(T, d, N, K), device_bf16(X), 2)
    y_v1 = run_gemm(device_matrix(c), device_bf16(X), 2)
    assert np.array_equal(y_pq2, y_v1)


def test_pq2_argument_errors():
    w = wal()
    T, d = gen_pq2(8, 256, 99, 1)
    pm = _device(T, d, 8, 256)
    X = device_bf16(gen_x(256, 1, 99, 2))
    Y = torch.empty(8, dtype=torch.float32, device="cuda")
    ws = torch.empty(512, dtype=torch.uint8, device="cuda")
    with pytest.raises(w.WalError) as e:
        w.wal_pq2_gemm(pm.desc, X.data_ptr(), 17, 256, Y.data_ptr(), 8, ws.data_ptr(), 512, stream())
    assert e.value.status == w.WAL_ERR_SHAPE
    with pytest.raises(w.WalError) as e:
        w.wal_pq2_gemm(pm.desc, X.data_ptr(), 1, 256, Y.data_ptr(), 8, ws.data_ptr(), 100, stream())
    assert e.value.status == w.WAL_ERR_WORKSPACE
    bad = w.wal_pq2_matrix(8, 256, pm.buf.data_ptr() + 2)
    with pytest.raises(w.WalError) as e:
        w.wal_pq2_gemm(bad, X.data_ptr(), 1, 256, Y.data_ptr(), 8, ws.data_ptr(), 512, stream())
    assert e.value.status == w.WAL_ERR_ARG


def _status(bp):
    wal().wal_device_status(bp.ws.data_ptr(), torch.cuda.current_stream().cuda_stream)


def test_pq2_body_two_layers_full():
    """Two 8B-shaped layers as PQ2_0 matrices, every output checked, two replays bitwise equal."""
    w = wal()
    specs = body_plan(2, LAYER_8B, 0, 0, 5)
    mats, xs, ys, refs = [], [], [], []
    for s in specs:
        T, d = gen_pq2(s.N, s.K, 5, 500 + s.index)
        X = gen_x(s.K, 1, 5, 500 + s.index)
        refs.append((s, pq.matmul(pq.Pq2(s.N, s.K, T, d), X), X, d))
        mats.append(_device(T, d, s.N, s.K))
        xs.append(device_bf16(X))
        ys.append(torch.full((s.N,), float("nan"), dtype=torch.float32, device="cuda"))
    bp = w.BodyPass(mats, [s.stage for s in specs], xs, ys, M=1)
    outs = []
    for _ in range(2):
        bp.run()
        torch.cuda.synchronize()
        _status(bp)
        outs.append([y.cpu().numpy().astype(np.float64) for y in ys])
    for (s, ref, X, d), y, y2 in zip(refs, outs[0], outs[1]):
        assert np.array_equal(y, y2)
        assert_parity(y.reshape(1, -1), ref, X, d, s.name)
    bp.close()


def test_pq2_body8b_full():
    """The 252-matrix PQ2_0 body pass in the configuration the benchmark times;
    every output checked against the oracle (all rows, process pool)."""
    w = wal()
    specs = config_plan("pq2_body8b")
    Xs = [gen_x(s.K, 1, 5, s.index) for s in specs]
    refs = oracle_pool.pq2_refs_async([(s.N, s.K, 5, s.index, X) for s, X in zip(specs, Xs)])
    mats, xs, ys = [], [], []
    for s, X in zip(specs, Xs):
        T, d = gen_pq2(s.N, s.K, 5, s.index)
        mats.append(_device(T, d, s.N, s.K))
        xs.append(device_bf16(X))
        ys.append(torch.full((s.N,), float("nan"), dtype=torch.float32, device="cuda"))
    bp = w.BodyPass(mats, [s.stage for s in specs], xs, ys, M=1)
    bp.run()
    torch.cuda.synchronize()
    _status(bp)
    for s, X, y, (ref, d) in zip(specs, Xs, ys, refs.get()):
        assert_parity(y.cpu().numpy().astype(np.float64).reshape(1, -1), ref, X, d, s.name)
    bp.close()
