"""wal_gemm_tc_noalloc: the tensor-core product with its scratch in the
library's fixed device array, against the workspace entry point
wal_gemm_small_m (needs a B200).  Collected last on purpose: it must pass on
its own and after every other test has used the device."""
import numpy as np
import pytest
import torch

from wal_synth import gen_components, gen_x

from gpu_util import needs_gpu, wal, device_matrix, device_bf16, stream, run_gemm

pytestmark = [pytest.mark.gpu, needs_gpu]


def run_noalloc(pm, X_dev, M):
    w = wal()
    Y = torch.full((M, pm.N), float("nan"), dtype=torch.float32, device="cuda")
    w.wal_gemm_tc_noalloc(pm.desc, X_dev.data_ptr(), M, pm.K, Y.data_ptr(), pm.N, stream())
    torch.cuda.synchronize()
    return Y.cpu().numpy().astype(np.float64)


def test_two_calls_in_a_row_match_the_workspace_entry():
    c = gen_components(384, 1024, 8, 8, config_id=70)
    pm = device_matrix(c)
    X1 = gen_x(1024, 64, 70, 1)
    X2 = gen_x(1024, 100, 70, 2)
    Y1 = run_noalloc(pm, device_bf16(X1), 64)
    Y2 = run_noalloc(pm, device_bf16(X2), 100)
    assert np.array_equal(Y1, run_gemm(pm, device_bf16(X1), 64))
    assert np.array_equal(Y2, run_gemm(pm, device_bf16(X2), 100))


def test_second_matrix_after_first():
    """A different shape (k = 0, r = 0) right after: nothing stale in the scratch."""
    a = device_matrix(gen_components(256, 2048, 8, 16, config_id=71))
    b = device_matrix(gen_components(200, 512, 0, 0, config_id=72))
    Xa = gen_x(2048, 48, 71, 0)
    Xb = gen_x(512, 17, 72, 0)
    Ya = run_noalloc(a, device_bf16(Xa), 48)
    Yb = run_noalloc(b, device_bf16(Xb), 17)
    assert np.array_equal(Ya, run_gemm(a, device_bf16(Xa), 48))
    assert np.array_equal(Yb, run_gemm(b, device_bf16(Xb), 17))


def test_limits_are_enforced():
    w = wal()
    pm = device_matrix(gen_components(128, 12288, 8, 8, config_id=73))
    assert pm.workspace_bytes(1024) > w.WAL_NOALLOC_SCRATCH_BYTES
    X = torch.zeros((1024, 12288), dtype=torch.int16, device="cuda")
    Y = torch.empty((1024, 128), dtype=torch.float32, device="cuda")
    with pytest.raises(w.WalError) as e:
        w.wal_gemm_tc_noalloc(pm.desc, X.data_ptr(), 1024, 12288, Y.data_ptr(), 128, stream())
    assert e.value.status == w.WAL_ERR_WORKSPACE
    with pytest.raises(w.WalError) as e:
        w.wal_gemm_tc_noalloc(pm.desc, X.data_ptr(), 4, 12288, Y.data_ptr(), 128, stream())
    assert e.value.status == w.WAL_ERR_SHAPE


@pytest.mark.parametrize("M", [5, 8, 16])
def test_smallest_tensor_batches(M):
    """From M = 5 wal_gemm_small_m takes the tensor-core path; the no-alloc
    entry accepts the same batches and gives the same bits."""
    c = gen_components(300, 1024, 4, 8, config_id=74)
    pm = device_matrix(c)
    X = gen_x(1024, M, 74, M)
    assert np.array_equal(run_noalloc(pm, device_bf16(X), M), run_gemm(pm, device_bf16(X), M))


def test_status_reader():
    """wal_noalloc_status reads (and clears) the scratch status word: OK after
    calls that completed."""
    w = wal()
    pm = device_matrix(gen_components(256, 512, 8, 4, config_id=75))
    X = gen_x(512, 32, 75, 0)
    run_noalloc(pm, device_bf16(X), 32)
    w.wal_noalloc_status(stream())  # raises WalError on anything but WAL_OK
    w.wal_noalloc_status(stream())
