"""Body-pass driver (CUDA graph over many matrices) vs the oracle (needs a B200)."""
import numpy as np
import pytest
import torch

import oracle
from wal_synth import config_plan, gen_matrix, gen_x, body_plan, LAYER_8B

from gpu_util import needs_gpu, wal, device_matrix, device_bf16, assert_parity

pytestmark = [pytest.mark.gpu, needs_gpu]


def _run_plan(workload, specs, sample=64, replays=2):
    w = wal()
    mats, xs, ys, comps, xbits = [], [], [], [], []
    for s in specs:
        c = gen_matrix(workload, s)
        x = gen_x(s.K, 1, 2 if workload == "body8b" else 1, s.index)
        mats.append(device_matrix(c))
        xs.append(device_bf16(x))
        ys.append(torch.empty(s.N, dtype=torch.float32, device="cuda"))
        comps.append(c if sample else None)
        xbits.append(x[0])
    bp = w.BodyPass(mats, [s.stage for s in specs], xs, ys, M=1)
    outs = []
    for _ in range(replays):
        for y in ys:
            y.fill_(float("nan"))
        bp.run()
        torch.cuda.synchronize()
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
        assert_parity(y[rows], oracle.matmul_rows(c, x, rows)[0], x, c.alpha, s.name)


def test_body8b_full_sampled():
    """The full 252-matrix 8B-shaped body pass in the launch configuration the
    benchmark times; 32 sampled rows of every matrix are checked."""
    w = wal()
    specs = config_plan("body8b")
    mats, xs, ys = [], [], []
    rng = np.random.default_rng(12)
    checks = []
    for s in specs:
        c = gen_matrix("body8b", s)
        x = gen_x(s.K, 1, 2, s.index)
        rows = np.unique(rng.choice(s.N, 32, replace=False))
        checks.append((s, rows, oracle.matmul_rows(c, x, rows)[0], x[0], c.alpha))
        mats.append(device_matrix(c))
        xs.append(device_bf16(x))
        ys.append(torch.empty(s.N, dtype=torch.float32, device="cuda"))
        del c
    bp = w.BodyPass(mats, [s.stage for s in specs], xs, ys, M=1)
    bp.run()
    torch.cuda.synchronize()
    for (s, rows, ref, x, alpha), y in zip(checks, ys):
        assert_parity(y.cpu().numpy().astype(np.float64)[rows], ref, x, alpha, s.name)
    bp.close()
