"""A bounded device wait that runs out (needs a B200).

The failure is made on the host: wal_debug_barrier_fault makes the next
body-pass plan's grid-barrier targets unreachable and gives each barrier wait
a 1 ms limit.  The pass must then end by itself, report WAL_ERR_TIMEOUT through
wal_device_status, leave the outputs of the stages after the first unwritten,
and leave the context usable: the same pass built afterwards without the fault
is correct.  No GPU fault, trap or endless wait is involved.
"""
import time

import numpy as np
import pytest
import torch

import oracle
from wal_synth import gen_components, gen_x

from gpu_util import needs_gpu, wal, device_matrix, device_bf16, assert_parity

pytestmark = [pytest.mark.gpu, needs_gpu]

# three dependency stages of two matrices each; K = 4096 spans several slices
SHAPES = [(512, 1024, 8, 4), (300, 4096, 4, 8), (1000, 2176, 8, 0), (640, 1024, 2, 16), (128, 4096, 8, 8),
          (2048, 1024, 0, 4)]
STAGES = [0, 0, 1, 1, 2, 2]


def _pass(mats, xs):
    ys = [torch.full((1, m.N), float("nan"), dtype=torch.float32, device="cuda") for m in mats]
    return wal().BodyPass(mats, STAGES, xs, ys, M=1), ys


def _status(bp):
    w = wal()
    try:
        w.wal_device_status(bp.ws.data_ptr(), torch.cuda.current_stream().cuda_stream)
        return w.WAL_OK
    except w.WalError as e:
        return e.status


def test_body_pass_barrier_wait_runs_out_then_recovers():
    w = wal()
    comps = [gen_components(N, K, k, r, config_id=97, matrix_index=i) for i, (N, K, k, r) in enumerate(SHAPES)]
    xbits = [gen_x(c.K, 1, 97, i) for i, c in enumerate(comps)]
    mats = [device_matrix(c) for c in comps]
    xs = [device_bf16(x) for x in xbits]

    prev = w.wal_debug_barrier_fault(1)
    try:
        bp, ys = _pass(mats, xs)
        t0 = time.perf_counter()
        bp.run()
        torch.cuda.synchronize()
        took = time.perf_counter() - t0
    finally:
        w.wal_debug_barrier_fault(prev)
    assert _status(bp) == w.WAL_ERR_TIMEOUT
    assert took < 10.0, f"the pass took {took:.1f} s to give up"
    got = [y.cpu().numpy().astype(np.float64) for y in ys]
    bp.close()
    for i, (c, x, y) in enumerate(zip(comps, xbits, got)):
        if STAGES[i] == 0:  # before the first barrier: complete and correct
            assert_parity(y, oracle.matmul(c, x), x, c.alpha, f"stage-0 matrix {i}")
        else:  # after it: nothing stored
            assert np.all(np.isnan(y)), f"matrix {i} of stage {STAGES[i]} was written after the wait gave up"

    # the context is usable and the same pass, built without the fault, is correct
    bp, ys = _pass(mats, xs)
    bp.run()
    torch.cuda.synchronize()
    assert _status(bp) == w.WAL_OK
    got = [y.cpu().numpy().astype(np.float64) for y in ys]
    bp.close()
    for i, (c, x, y) in enumerate(zip(comps, xbits, got)):
        assert_parity(y, oracle.matmul(c, x), x, c.alpha, f"matrix {i} after recovery")
