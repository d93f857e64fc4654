"""Tensor-core path (8 or more activation rows) vs the FP64 oracle, through
the C ABI (needs a B200).

Tolerance as everywhere (oracle.check_tolerance): rel-L2 <= 1e-5 over Y and
max |y_m - y*_m| <= 1e-3 * ||x_m||_2 * max|alpha| per activation row m.
"""
import numpy as np
import pytest
import torch

import oracle
from wal_synth import gen_components, gen_x, config_plan, gen_matrix, bf16_bits_from_f32

from golden_io import fixture_names, load
import oracle_pool
from gpu_util import needs_gpu, wal, device_matrix, device_bf16, stream, run_gemm, assert_parity

pytestmark = [pytest.mark.gpu, needs_gpu]

TC_SHAPES = [  # N, K, k, r, M
    (256, 512, 8, 8, 64),
    (200, 384, 4, 16, 17),     # ragged second row tile
    (130, 256, 2, 0, 100),     # batch not a multiple of 16
    (128, 1024, 0, 32, 256),   # plain ternary + maximum rank, one full activation tile
    (384, 768, 8, 3, 300),     # two activation tiles, the second ragged
    (64, 128, 8, 1, 33),       # a single group, fewer rows than a tile
    (1000, 2176, 8, 8, 64),
    (1000, 2176, 8, 8, 8),
    (1000, 2176, 8, 8, 5),     # the smallest batch on this path
    (300, 4096, 4, 16, 12),
    (64, 128, 8, 1, 16),
    (12288, 4096, 8, 16, 16),  # the gate shape of the batch sweep
]


@pytest.mark.parametrize("N,K,k,r,M", TC_SHAPES)
def test_tc_parity(N, K, k, r, M):
    c = gen_components(N, K, k, r, config_id=80, matrix_index=N + M)
    X = gen_x(K, M, 80, N + M)
    Y = run_gemm(device_matrix(c), device_bf16(X), M)
    assert_parity(Y, oracle.matmul(c, X), X, c.alpha, f"{N}x{K} k={k} r={r} M={M}")


@pytest.mark.parametrize("name", fixture_names())
def test_tc_golden_exact(name):
    """The worked cases are dyadic: the FP16 operands and FP32 accumulation hold them exactly."""
    c, x, y_exp, _ = load(name)
    M = 20
    Y = run_gemm(device_matrix(c), device_bf16(np.tile(x, (M, 1))), M)
    for m in range(M):
        assert np.array_equal(Y[m], y_exp), (name, m, Y[m], y_exp)


def test_tc_odd_symmetry_bitwise():
    c = gen_components(300, 2048, 8, 8, config_id=81)
    X = gen_x(2048, 64, 81, 0)
    pm = device_matrix(c)
    Y1 = run_gemm(pm, device_bf16(X), 64)
    Y2 = run_gemm(pm, device_bf16(X ^ np.uint16(0x8000)), 64)
    assert np.array_equal(Y2, -Y1)


def test_tc_deterministic_reruns():
    c = gen_components(512, 4096, 8, 16, config_id=82)
    X = gen_x(4096, 128, 82, 0)
    pm = device_matrix(c)
    Xd = device_bf16(X)
    assert np.array_equal(run_gemm(pm, Xd, 128), run_gemm(pm, Xd, 128))


def test_tc_agrees_with_cuda_core_path():
    """Rows 0..3 of an M = 64 product (tensor path) against the CUDA-core path
    at M = 4 (the largest batch it takes): both within tolerance of the oracle
    and of each other."""
    c = gen_components(700, 4096, 8, 8, config_id=83)
    X = gen_x(4096, 64, 83, 0)
    pm = device_matrix(c)
    Yt = run_gemm(pm, device_bf16(X), 64)
    Yc = run_gemm(pm, device_bf16(X[:4]), 4)
    ref = oracle.matmul(c, X[:4])
    assert_parity(Yt[:4], ref, X[:4], c.alpha, "tensor")
    assert_parity(Yc, ref, X[:4], c.alpha, "cuda-core")
    assert_parity(Yt[:4], Yc, X[:4], c.alpha, "tensor vs cuda-core")


def test_tc_wide_dynamic_range_x():
    """Rows spanning 2^-40 .. 2^20: elements far below the row maximum are
    rounded by the FP16 image, which the tolerance absorbs."""
    c = gen_components(256, 1024, 8, 4, config_id=84)
    rng = np.random.default_rng(4)
    xf = (rng.standard_normal((40, 1024)) * 2.0 ** rng.integers(-40, 20, (40, 1024))).astype(np.float32)
    X = bf16_bits_from_f32(xf)
    Y = run_gemm(device_matrix(c), device_bf16(X), 40)
    assert_parity(Y, oracle.matmul(c, X), X, c.alpha, "wide range")


def test_tc_zero_rows():
    c = gen_components(100, 512, 8, 8, config_id=85)
    X = gen_x(512, 48, 85, 0)
    X[7] = 0
    X[40] = 0
    Y = run_gemm(device_matrix(c), device_bf16(X), 48)
    assert np.array_equal(Y[7], np.zeros(100)) and np.array_equal(Y[40], np.zeros(100))
    assert_parity(Y, oracle.matmul(c, X), X, c.alpha, "zero rows")


def test_tc_workspace_is_checked():
    w = wal()
    c = gen_components(128, 512, 8, 8, config_id=86)
    pm = device_matrix(c)
    M = 64
    need = pm.workspace_bytes(M)
    assert need > pm.workspace_bytes(16)
    X = device_bf16(gen_x(512, M, 86, 0))
    Y = torch.empty((M, 128), dtype=torch.float32, device="cuda")
    ws = torch.empty(need, dtype=torch.uint8, device="cuda")
    with pytest.raises(w.WalError) as e:
        w.wal_gemm_small_m(pm.desc, X.data_ptr(), M, 512, Y.data_ptr(), 128, ws.data_ptr(), need - 1024, stream())
    assert e.value.status == w.WAL_ERR_WORKSPACE


@pytest.mark.parametrize("M", [64, 256, 1024])
def test_sweep_full_size(M):
    """gate 4096->12288 and down 12288->4096 (k=8, r=16) at full size: every
    output checked against the oracle (all rows, process pool)."""
    specs = config_plan("sweep")
    Xs = [gen_x(s.K, M, 4, 100 + s.index) for s in specs]
    refs = oracle_pool.v1_refs_async("sweep", specs, Xs)
    Ys = [run_gemm(device_matrix(gen_matrix("sweep", s)), device_bf16(X), M) for s, X in zip(specs, Xs)]
    for spec, X, Y, (ref, alpha) in zip(specs, Xs, Ys, refs.get()):
        assert_parity(Y, ref, X, alpha, f"{spec.name} M={M}")
