"""Body-pass driver (CUDA graph over many matrices) vs the oracle (needs a B200)."""
import numpy as np
import pytest
import torch

import oracle
from wal_synth import config_plan, gen_components, gen_matrix, gen_x, body_plan, bf16_bits_from_f32, LAYER_8B

from gpu_util import needs_gpu, wal, device_matrix, device_bf16, assert_parity
import oracle_pool

pytestmark = [pytest.mark.gpu, needs_gpu]


def _status(bp):
    wal().wal_device_status(bp.ws.data_ptr(), torch.cuda.current_stream().cuda_stream)


def _run_plan(workload, specs, sample=64, replays=2, M=1):
    w = wal()
    mats, xs, ys, comps, xbits = [], [], [], [], []
    for s in specs:
        c = gen_matrix(workload, s)
        x = gen_x(s.K, M, 2 if workload == "body8b" else 1, s.index)
        mats.append(device_matrix(c))
        xs.append(device_bf16(x))
        ys.append(torch.empty((M, s.N), dtype=torch.float32, device="cuda"))
        comps.append(c if sample else None)
        xbits.append(x)
    bp = w.BodyPass(mats, [s.stage for s in specs], xs, ys, M=M)
    outs = []
    for _ in range(replays):
        for y in ys:
            y.fill_(float("nan"))
        bp.run()
        torch.cuda.synchronize()
        _status(bp)
        outs.append([y.cpu().numpy().astype(np.float64) for y in ys])
    bp.close()
    return specs, comps, xbits, outs


def test_body_two_layers_sampled():
    specs = body_plan(2, LAYER_8B, 8, 8, 1, n_lowrank=10)
    specs, comps, xbits, outs = _run_plan("layer8b", specs)
    rng = np.random.default_rng(11)
    for s, c, x, y, y2 in zip(specs, comps, xbits, outs[0], outs[1]):
        assert np.array_equal(y, y2), "graph replays differ"
        rows = np.unique(np.concatenate([[0, s.N - 1], rng.choice(s.N, 64, replace=False)]))
        assert_parity(y[0][rows], oracle.matmul_rows(c, x, rows)[0], x, c.alpha, s.name)


def test_body_batch4_two_layers():
    """M = 4: four activation rows per matrix in one pass."""
    specs = body_plan(2, LAYER_8B, 8, 8, 1, n_lowrank=9)
    specs, comps, xbits, outs = _run_plan("layer8b", specs, replays=1, M=4)
    rng = np.random.default_rng(13)
    for s, c, X, Y in zip(specs, comps, xbits, outs[0]):
        rows = np.unique(rng.choice(s.N, 48, replace=False))
        assert_parity(Y[:, rows], oracle.matmul_rows(c, X, rows), X, c.alpha, s.name)


def test_body_stage_dependency():
    """Stage 1 reads what stage 0 writes.  Stage 0 is a selection matrix
    (y_A[n] = x_A[n mod K_A], alpha = 1), so its fp32 outputs are bf16 values
    exactly; read as bf16 pairs, y_A's bytes are (0, y_A[n]) for every n.
    Matrix B of stage 1 takes that buffer as its x.  The buffer starts as
    NaN, so a read before the grid barrier shows."""
    w = wal()
    NA, KA = 2048, 1024
    a = gen_components(NA, KA, 0, 0, config_id=60, matrix_index=0)
    a.T[:] = 0
    a.T[np.arange(NA), np.arange(NA) % KA] = 1
    a.alpha[:] = 0x3C00  # fp16 1.0
    # magnitudes in [1, 2): every x_A is exact in the fixed-point image, so
    # y_A holds bf16 values exactly
    rng = np.random.default_rng(60)
    xa = bf16_bits_from_f32((rng.uniform(1.0, 2.0, (1, KA)) * rng.choice([-1.0, 1.0], (1, KA))).astype(np.float32))
    b = gen_components(4096, 2 * NA, 8, 8, config_id=60, matrix_index=1)
    c2 = gen_components(1024, 4096, 4, 0, config_id=60, matrix_index=2)  # a second stage-1 matrix, own x
    xc = gen_x(4096, 1, 60, 2)
    ya = torch.full((NA,), float("nan"), dtype=torch.float32, device="cuda")
    xb = ya.view(torch.int16)  # the same bytes as 2 * NA bf16 values
    yb = torch.empty(4096, dtype=torch.float32, device="cuda")
    yc = torch.empty(1024, dtype=torch.float32, device="cuda")
    mats = [device_matrix(a), device_matrix(b), device_matrix(c2)]
    bp = w.BodyPass(mats, [0, 1, 1], [device_bf16(xa), xb, device_bf16(xc)], [ya, yb, yc], M=1)
    for _ in range(2):
        ya.fill_(float("nan"))
        bp.run()
        torch.cuda.synchronize()
        _status(bp)
        exp_a = oracle.matvec(a, xa[0])
        assert np.array_equal(ya.cpu().numpy().astype(np.float64), exp_a)
        xb_bits = ya.cpu().numpy().view(np.uint16)
        assert_parity(yb.cpu().numpy().astype(np.float64), oracle.matvec(b, xb_bits), xb_bits, b.alpha, "stage 1")
        assert_parity(yc.cpu().numpy().astype(np.float64), oracle.matvec(c2, xc[0]), xc[0], c2.alpha, "stage 1 other")
    bp.close()


def test_body8b_full():
    """The full 252-matrix 8B-shaped body pass in the launch configuration the
    benchmark times.  Every output is checked: the outputs start as NaN, and
    the oracle computes all rows of every matrix (in a process pool, while the
    GPU runs)."""
    w = wal()
    specs = config_plan("body8b")
    xbits = [gen_x(s.K, 1, 2, s.index) for s in specs]
    refs = oracle_pool.v1_refs_async("body8b", specs, xbits)
    mats, xs, ys = [], [], []
    for s, x in zip(specs, xbits):
        mats.append(device_matrix(gen_matrix("body8b", s)))
        xs.append(device_bf16(x))
        ys.append(torch.full((s.N,), float("nan"), dtype=torch.float32, device="cuda"))
    bp = w.BodyPass(mats, [s.stage for s in specs], xs, ys, M=1)
    bp.run()
    torch.cuda.synchronize()
    _status(bp)
    for s, x, y, (ref, alpha) in zip(specs, xbits, ys, refs.get()):
        assert_parity(y.cpu().numpy().astype(np.float64).reshape(1, -1), ref, x, alpha, s.name)
    bp.close()


@pytest.fixture(scope="module")
def body27b():
    """The 448 27B-shaped matrices on the device, with the oracle's outputs
    for every row of every matrix at M = 1 and M = 4 (computed in a process
    pool while the matrices are generated and uploaded)."""
    specs = config_plan("body27b")
    X = {M: [gen_x(s.K, M, 3, 1000 * M + s.index) for s in specs] for M in (1, 4)}
    refs = {M: oracle_pool.v1_refs_async("body27b", specs, X[M]) for M in (1, 4)}
    mats = [device_matrix(gen_matrix("body27b", s)) for s in specs]
    return specs, mats, X, refs


@pytest.mark.parametrize("M", [1, 4])
def test_body27b_full(body27b, M):
    """The full 448-matrix 27B-shaped body pass (k by role, 45 matrices with
    k = 0, 152 with WALB2 r = 8) at batch 1 and 4; every output checked."""
    w = wal()
    specs, mats, X, refs = body27b
    xs = [device_bf16(x) for x in X[M]]
    ys = [torch.full((M, s.N), float("nan"), dtype=torch.float32, device="cuda") for s in specs]
    bp = w.BodyPass(mats, [s.stage for s in specs], xs, ys, M=M)
    bp.run()
    torch.cuda.synchronize()
    _status(bp)
    for s, x, y, (ref, alpha) in zip(specs, X[M], ys, refs[M].get()):
        assert_parity(y.cpu().numpy().astype(np.float64), ref, x, alpha, f"{s.name} M={M}")
    bp.close()


def test_body_dependency_two_stages_back():
    """Stage 2 reads what stage 0 wrote, across a stage 1 that does not touch
    it.  The pass builds stage 2's x image while the barrier before it is
    still open (stage 1 writes no x of stage 2); stage 0's output is complete
    by then, since every CTA passed the barrier after stage 0.  The buffer
    starts as NaN, so a read before stage 0's writes shows."""
    w = wal()
    NA, KA = 2048, 1024
    a = gen_components(NA, KA, 0, 0, config_id=61, matrix_index=0)
    a.T[:] = 0
    a.T[np.arange(NA), np.arange(NA) % KA] = 1
    a.alpha[:] = 0x3C00  # fp16 1.0
    rng = np.random.default_rng(61)
    xa = bf16_bits_from_f32((rng.uniform(1.0, 2.0, (1, KA)) * rng.choice([-1.0, 1.0], (1, KA))).astype(np.float32))
    mid = gen_components(3000, 4096, 8, 8, config_id=61, matrix_index=1)   # stage 1, its own x
    xm = gen_x(4096, 1, 61, 1)
    b = gen_components(4096, 2 * NA, 8, 8, config_id=61, matrix_index=2)  # stage 2 reads y_A
    ya = torch.full((NA,), float("nan"), dtype=torch.float32, device="cuda")
    ym = torch.empty(3000, dtype=torch.float32, device="cuda")
    yb = torch.empty(4096, dtype=torch.float32, device="cuda")
    mats = [device_matrix(a), device_matrix(mid), device_matrix(b)]
    bp = w.BodyPass(mats, [0, 1, 2], [device_bf16(xa), device_bf16(xm), ya.view(torch.int16)], [ya, ym, yb], M=1)
    for _ in range(3):
        ya.fill_(float("nan"))
        bp.run()
        torch.cuda.synchronize()
        _status(bp)
        assert np.array_equal(ya.cpu().numpy().astype(np.float64), oracle.matvec(a, xa[0]))
        assert_parity(ym.cpu().numpy().astype(np.float64), oracle.matvec(mid, xm[0]), xm[0], mid.alpha, "stage 1")
        xb_bits = ya.cpu().numpy().view(np.uint16)
        assert_parity(yb.cpu().numpy().astype(np.float64), oracle.matvec(b, xb_bits), xb_bits, b.alpha, "stage 2")
    bp.close()
