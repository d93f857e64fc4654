"""CUDA path vs the FP64 oracle, through the C ABI (needs a B200).

Tolerance (written out here, applied by oracle.check_tolerance):
  rel-L2 = ||y - y*||_2 / ||y*||_2 <= 1e-5 over the whole output, and
  max |y_m - y*_m| <= 1e-3 * ||x_m||_2 * max|alpha| for every activation row m.
Decoding is compared bit for bit.
"""
import numpy as np
import pytest
import torch

import oracle
from wal_synth import Components, gen_components, gen_x, config_plan, gen_matrix

from golden_io import fixture_names, load
import oracle_pool
from gpu_util import (needs_gpu, wal, device_matrix, device_bf16, stream, run_gemv, run_gemm,
                      assert_parity)

pytestmark = [pytest.mark.gpu, needs_gpu]

SHAPES = [
    (512, 1024, 8, 4),     # the single-matrix workload
    (37, 384, 2, 1),       # ragged N, three groups
    (1000, 2176, 8, 8),    # two K-slices, the second one ragged (one group)
    (64, 128, 0, 0),       # plain ternary, one group
    (300, 4096, 4, 16),
    (8, 12288, 8, 32),     # six K-slices, maximum rank
    (129, 1152, 0, 5),
    (1, 128, 8, 0),        # a single row
    (2051, 4224, 2, 3),    # ragged rows and slices
]


@pytest.mark.parametrize("N,K,k,r", SHAPES)
def test_decode_bit_exact(N, K, k, r):
    c = gen_components(N, K, k, r, config_id=90, matrix_index=N + K)
    pm = device_matrix(c)
    G = K // 128
    T = torch.empty((N, K), dtype=torch.int8, device="cuda")
    pos = torch.empty((N, G, max(k, 1)), dtype=torch.uint8, device="cuda")
    sgn = torch.empty((N, G, max(k, 1)), dtype=torch.int8, device="cuda")
    a = torch.empty((N, G), dtype=torch.int16, device="cuda")
    b = torch.empty((N, G), dtype=torch.int16, device="cuda")
    U = torch.empty((N, max(r, 1)), dtype=torch.int8, device="cuda")
    V = torch.empty((K, max(r, 1)), dtype=torch.int8, device="cuda")
    wal().wal_unpack_matrix(pm.desc, T.data_ptr(), pos.data_ptr(), sgn.data_ptr(), a.data_ptr(),
                            b.data_ptr(), U.data_ptr(), V.data_ptr(), stream())
    torch.cuda.synchronize()
    assert np.array_equal(T.cpu().numpy(), c.T)
    if k:
        assert np.array_equal(pos.cpu().numpy(), c.site_pos)
        assert np.array_equal(sgn.cpu().numpy(), c.site_sign)
        assert np.array_equal(b.cpu().numpy().view(np.uint16), c.beta)
    assert np.array_equal(a.cpu().numpy().view(np.uint16), c.alpha)
    if r:
        assert np.array_equal(U.cpu().numpy(), c.U)
        assert np.array_equal(V.cpu().numpy(), c.V)


@pytest.mark.parametrize("N,K,k,r", SHAPES)
def test_gemv_parity(N, K, k, r):
    c = gen_components(N, K, k, r, config_id=91, matrix_index=N + K)
    x = gen_x(K, 1, 91, N + K)[0]
    y = run_gemv(device_matrix(c), device_bf16(x))
    assert_parity(y, oracle.matvec(c, x), x, c.alpha, f"{N}x{K} k={k} r={r}")


@pytest.mark.parametrize("name", fixture_names())
def test_golden_exact_on_gpu(name):
    """The worked cases are dyadic and small: the GPU must reproduce them exactly."""
    c, x, y_exp, _ = load(name)
    y = run_gemv(device_matrix(c), device_bf16(x))
    assert np.array_equal(y, y_exp), (name, y, y_exp)


def test_odd_symmetry_bitwise():
    c = gen_components(700, 4096, 8, 8, config_id=92)
    x = gen_x(4096, 1, 92, 0)[0]
    pm = device_matrix(c)
    y1 = run_gemv(pm, device_bf16(x))
    y2 = run_gemv(pm, device_bf16(x ^ np.uint16(0x8000)))
    assert np.array_equal(y2, -y1)


def test_deterministic_reruns():
    c = gen_components(1024, 12288, 8, 8, config_id=93)
    x = gen_x(12288, 1, 93, 0)[0]
    pm = device_matrix(c)
    xd = device_bf16(x)
    assert np.array_equal(run_gemv(pm, xd), run_gemv(pm, xd))


def test_tall_matrix_both_row_reductions():
    """162800 x 128: a row block of 1100 rows, whose per-lane partials do not
    fit in shared memory beside the weight ring, so each row is reduced by a
    warp butterfly in the row loop.  Its first 1000 rows as a matrix of their
    own keep per-lane partials, summed in the combine by the same tree: the
    two must agree bit for bit, and the tall product must meet the oracle."""
    N, K, n = 148 * 1100, 128, 1000
    c = gen_components(N, K, 8, 4, config_id=97, matrix_index=1)
    x = gen_x(K, 1, 97, 1)[0]
    xd = device_bf16(x)
    y = run_gemv(device_matrix(c), xd)
    assert_parity(y, oracle.matvec(c, x), x, c.alpha, f"{N}x{K}")
    head = Components(n, K, 8, 4, c.T[:n], c.site_pos[:n], c.site_sign[:n], c.alpha[:n], c.beta[:n], c.U[:n],
                      c.V, c.lr_scale)
    assert np.array_equal(run_gemv(device_matrix(head), xd), y[:n])


def test_wide_dynamic_range_x():
    """x spanning 2^-40 .. 2^20 inside one group: small entries are rounded in
    the fixed-point image, which the tolerance absorbs."""
    c = gen_components(256, 1024, 8, 4, config_id=94)
    rng = np.random.default_rng(3)
    xf = (rng.standard_normal(1024) * 2.0 ** rng.integers(-40, 20, 1024)).astype(np.float32)
    from wal_synth import bf16_bits_from_f32
    x = bf16_bits_from_f32(xf)
    y = run_gemv(device_matrix(c), device_bf16(x))
    assert_parity(y, oracle.matvec(c, x), x, c.alpha, "wide range")


def test_zero_x_gives_zero():
    c = gen_components(100, 512, 8, 8, config_id=95)
    x = np.zeros(512, np.uint16)
    y = run_gemv(device_matrix(c), device_bf16(x))
    assert np.array_equal(y, np.zeros(100))


@pytest.mark.parametrize("M", [1, 2, 4, 5, 7, 8, 16])
def test_small_m_parity_and_columns(M):
    """M <= 4 runs M batch-1 products in one launch, each equal bit for bit to
    wal_gemv; from M = 5 the tensor-core path runs (checked against the oracle)."""
    c = gen_components(1000, 2176, 8, 8, config_id=96)
    X = gen_x(2176, M, 96, M)
    pm = device_matrix(c)
    Y = run_gemm(pm, device_bf16(X), M)
    assert_parity(Y, oracle.matmul(c, X), X, c.alpha, f"M={M}")
    if M < 5:
        for m in range(M):
            assert np.array_equal(Y[m], run_gemv(pm, device_bf16(X[m])))


def test_layer8b_full_size():
    """All seven Qwen3-8B-shaped matrices at full size; every output of the
    GPU product is checked against the oracle (all rows, process pool)."""
    specs = config_plan("layer8b")
    xs = [gen_x(s.K, 1, 1, s.index) for s in specs]
    refs = oracle_pool.v1_refs_async("layer8b", specs, xs)
    ys = []
    for spec, x in zip(specs, xs):
        ys.append(run_gemv(device_matrix(gen_matrix("layer8b", spec)), device_bf16(x[0])))
    for spec, x, y, (ref, alpha) in zip(specs, xs, ys, refs.get()):
        assert_parity(y.reshape(1, -1), ref, x, alpha, spec.name)


def test_validate_detects_corruption():
    w = wal()
    c = gen_components(64, 1024, 8, 4, config_id=97)
    bufs = w.pack_host(c)
    ws = torch.empty(4096, dtype=torch.uint8, device="cuda")
    pm = w.PackedMatrix(bufs, 64, 1024, 8, 4)
    w.wal_validate(pm.desc, ws.data_ptr(), ws.numel(), stream())
    bad = [b.copy() for b in bufs]
    bad[0][123] |= 0x0C      # a code field becomes 3
    pm2 = w.PackedMatrix(bad, 64, 1024, 8, 4)
    with pytest.raises(w.WalError) as e:
        w.wal_validate(pm2.desc, ws.data_ptr(), ws.numel(), stream())
    assert e.value.status == w.WAL_ERR_FORMAT
    bad = [b.copy() for b in bufs]
    bad[1][8:16] = bad[1][8:16][::-1].copy()   # sites of one group out of order
    pm3 = w.PackedMatrix(bad, 64, 1024, 8, 4)
    with pytest.raises(w.WalError) as e:
        w.wal_validate(pm3.desc, ws.data_ptr(), ws.numel(), stream())
    assert e.value.status == w.WAL_ERR_FORMAT


def test_argument_errors():
    w = wal()
    c = gen_components(64, 1024, 8, 4, config_id=98)
    pm = device_matrix(c)
    x = device_bf16(gen_x(1024)[0])
    y = torch.empty(64, dtype=torch.float32, device="cuda")
    nb = pm.workspace_bytes(1)
    ws = torch.empty(nb, dtype=torch.uint8, device="cuda")
    with pytest.raises(w.WalError) as e:
        w.wal_gemv(pm.desc, x.data_ptr(), y.data_ptr(), ws.data_ptr(), nb - 512, stream())
    assert e.value.status == w.WAL_ERR_WORKSPACE
    with pytest.raises(w.WalError) as e:
        w.wal_gemv(pm.desc, x.data_ptr() + 2, y.data_ptr(), ws.data_ptr(), nb, stream())
    assert e.value.status == w.WAL_ERR_ARG
    bad = w.wal_matrix(64, 1000, 8, 4, *[getattr(pm.desc, f) for f in ("codes", "sites", "scales", "u_bits", "v_bits", "lr_scale")])
    with pytest.raises(w.WalError) as e:
        w.wal_gemv(bad, x.data_ptr(), y.data_ptr(), ws.data_ptr(), nb, stream())
    assert e.value.status == w.WAL_ERR_SHAPE
