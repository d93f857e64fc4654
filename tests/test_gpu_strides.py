"""Row strides of X and Y, and the batch limits of the body pass (needs a B200).

wal_gemm_small_m takes X[M][ldx] and Y[M][ldy] with ldx >= K (a multiple of 8)
and ldy >= N.  Both paths (CUDA cores up to M = 4, the tensor path from
M = 5) must read only the first K entries of each X row and write only the
first N entries of each Y row.  The body pass takes 1 <= M <= 16.
"""
import numpy as np
import pytest
import torch

import oracle
from wal_synth import gen_components, gen_x

from gpu_util import needs_gpu, wal, device_matrix, device_bf16, stream, assert_parity

pytestmark = [pytest.mark.gpu, needs_gpu]


@pytest.mark.parametrize("M", [1, 3, 5, 20])
def test_strided_x_and_y(M):
    w = wal()
    N, K = 300, 1024
    ldx, ldy = K + 64, N + 3
    c = gen_components(N, K, 8, 8, config_id=99, matrix_index=M)
    X = gen_x(K, M, 99, M)
    Xp = np.full((M, ldx), 0x7FC0, np.uint16)  # NaN bf16 in the padding: any read of it would show
    Xp[:, :K] = X
    pm = device_matrix(c)
    Xd = device_bf16(Xp)
    Y = torch.full((M, ldy), float("nan"), dtype=torch.float32, device="cuda")
    nb = pm.workspace_bytes(M)
    ws = torch.empty(nb, dtype=torch.uint8, device="cuda")
    w.wal_gemm_small_m(pm.desc, Xd.data_ptr(), M, ldx, Y.data_ptr(), ldy, ws.data_ptr(), nb, stream())
    torch.cuda.synchronize()
    w.wal_device_status(ws.data_ptr(), stream())
    Yh = Y.cpu().numpy().astype(np.float64)
    assert np.all(np.isnan(Yh[:, N:])), "a write past N in a Y row"
    assert_parity(Yh[:, :N], oracle.matmul(c, X), X, c.alpha, f"M={M} ldx={ldx} ldy={ldy}")


def test_body_pass_largest_batch_and_limits():
    """M = 16 (the largest batch) over a short two-stage pass; M = 17 is refused."""
    w = wal()
    comps = [gen_components(N, K, k, r, config_id=99, matrix_index=100 + i)
             for i, (N, K, k, r) in enumerate([(256, 1024, 8, 4), (200, 4096, 4, 0), (512, 2048, 8, 8)])]
    M = 16
    xs_bits = [gen_x(c.K, M, 99, 200 + i) for i, c in enumerate(comps)]
    mats = [device_matrix(c) for c in comps]
    xs = [device_bf16(x) for x in xs_bits]
    ys = [torch.full((M, c.N), float("nan"), dtype=torch.float32, device="cuda") for c in comps]
    bp = w.BodyPass(mats, [0, 0, 1], xs, ys, M=M)
    bp.run()
    torch.cuda.synchronize()
    w.wal_device_status(bp.ws.data_ptr(), torch.cuda.current_stream().cuda_stream)
    for c, x, y in zip(comps, xs_bits, ys):
        assert_parity(y.cpu().numpy().astype(np.float64), oracle.matmul(c, x), x, c.alpha, f"{c.N}x{c.K} M=16")
    bp.close()
    ys17 = [torch.empty((17, c.N), dtype=torch.float32, device="cuda") for c in comps]
    xs17 = [device_bf16(gen_x(c.K, 17, 99, 300 + i)) for i, c in enumerate(comps)]
    bp = w.BodyPass(mats, [0, 0, 1], xs17, ys17, M=17)
    with pytest.raises(w.WalError) as e:
        bp.run()
    assert e.value.status == w.WAL_ERR_SHAPE
    bp.close()
