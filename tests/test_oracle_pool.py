"""The process pool that the full-size GPU tests use gives the same oracle
values as calling the oracle directly (CPU only)."""
import numpy as np

import oracle
import oracle_pool
from oracle import head_oracle as ho
from oracle import pq2_oracle as pq
from wal_synth import MatrixSpec, config_plan, gen_int4, gen_matrix, gen_pq2, gen_x


def test_v1_refs_match_direct_oracle():
    specs = config_plan("single") + [MatrixSpec("tall", 2100, 256, 4, 3, 1, 1, 0)]
    xs = [gen_x(s.K, 2, 9, s.index) for s in specs]
    old = oracle_pool.ROW_CHUNK
    oracle_pool.ROW_CHUNK = 1000  # several row blocks, the last ragged
    try:
        got = oracle_pool.v1_refs_async("single", specs, xs).get()
    finally:
        oracle_pool.ROW_CHUNK = old
    for s, x, (Y, alpha) in zip(specs, xs, got):
        c = gen_matrix("single", s)
        assert np.array_equal(Y, oracle.matmul(c, x))
        assert np.array_equal(alpha, c.alpha)


def test_pq2_and_int4_refs_match_direct_oracle():
    X = gen_x(256, 1, 9, 3)
    (Y, d), = oracle_pool.pq2_refs_async([(300, 256, 9, 3, X)]).get()
    T, d2 = gen_pq2(300, 256, 9, 3)
    assert np.array_equal(Y, pq.matmul(pq.Pq2(300, 256, T, d2), X))
    assert np.array_equal(d, d2)
    X4 = gen_x(256, 2, 9, 4)
    Y4 = oracle_pool.int4_ref(1000, 256, 9, 4, X4, chunk=300)
    q, d4 = gen_int4(1000, 256, 9, 4)
    assert np.array_equal(Y4, ho.int4_matmul_rows(q, d4, X4, np.arange(1000)))
