"""The products' own decode, column by column, bit for bit (needs a B200).

wal_unpack_matrix pins the layout with the device's test decoder; this pins
the decode the products run (the masked dp4a slots, the site table, the
scale application, WALB2 phases 1 and 2, and the tensor path's FP16 planes).
With x = e_j the product returns column j of W.  The scales are chosen so that
every column value is exact in FP32 whatever the summation order: alpha = 1,
beta = 1/2 and s_r = 2^-(r+1), so W holds multiples of 1/32 below 8 in
magnitude.  Every column of W is read this way and compared with the oracle's
dense W (formed from the oracle's own unpacking of the packed bytes) for
equality.
"""
import numpy as np
import pytest
import torch

import oracle
from wal_synth import gen_components

from gpu_util import needs_gpu, device_matrix, device_bf16, run_gemm

pytestmark = [pytest.mark.gpu, needs_gpu]

ONE_BF16 = 0x3F80


def exact_components(N, K, k, r, seed):
    c = gen_components(N, K, k, r, config_id=98, matrix_index=seed)
    G = K // 128
    c.alpha = np.full((N, G), 0x3C00, np.uint16)                    # 1.0
    c.beta = np.full((N, G), 0x3800 if k else 0, np.uint16)          # 0.5
    c.lr_scale = np.array([0x3800 - 0x0400 * i for i in range(r)], np.uint16)  # 2^-1, 2^-2, ...
    return c


@pytest.mark.parametrize("N,K,k,r,M", [
    (100, 256, 8, 4, 7),     # CUDA-core decode, 7 one-hot rows per launch, ragged N
    (64, 384, 4, 2, 5),
    (40, 256, 2, 0, 3),
    (96, 256, 0, 3, 7),
    (130, 256, 8, 4, 16),    # tensor-core path (decode to FP16 planes + tcgen05)
])
def test_product_columns_equal_dense_w(N, K, k, r, M):
    c = exact_components(N, K, k, r, seed=N + K + M)
    u = oracle.unpack(oracle.pack(c), N, K, k, r)
    W = oracle.dense_weight(u)
    pm = device_matrix(c)
    for j0 in range(0, K, M):
        cols = list(range(j0, min(K, j0 + M)))
        X = np.zeros((M, K), np.uint16)
        for i, j in enumerate(cols):
            X[i, j] = ONE_BF16
        Y = run_gemm(pm, device_bf16(X), M)
        for i, j in enumerate(cols):
            assert np.array_equal(Y[i], W[:, j]), f"column {j}: {np.flatnonzero(Y[i] != W[:, j])[:8]} differ"
        for i in range(len(cols), M):  # rows of x that are all zero give exact zeros
            assert np.array_equal(Y[i], np.zeros(N))
