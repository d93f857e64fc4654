"""Helpers for the GPU tests: device copies of generator outputs, oracle comparison."""
import numpy as np
import pytest
import torch

import oracle

needs_gpu = pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")


def wal():
    import ternary_sparse_binary_b200 as w
    return w


def device_matrix(c):
    w = wal()
    return w.PackedMatrix(w.pack_host(c), c.N, c.K, c.k, c.r)


def device_bf16(x_bits):
    return torch.from_numpy(np.ascontiguousarray(x_bits).view(np.int16)).cuda()


def stream():
    return torch.cuda.current_stream().cuda_stream


def run_gemv(pm, x_dev):
    w = wal()
    y = torch.full((pm.N,), float("nan"), dtype=torch.float32, device="cuda")
    nb = pm.workspace_bytes(1)
    ws = torch.empty(nb, dtype=torch.uint8, device="cuda")
    w.wal_gemv(pm.desc, x_dev.data_ptr(), y.data_ptr(), ws.data_ptr(), nb, stream())
    torch.cuda.synchronize()
    w.wal_device_status(ws.data_ptr(), stream())
    return y.cpu().numpy().astype(np.float64)


def run_gemm(pm, X_dev, M):
    w = wal()
    Y = torch.full((M, pm.N), float("nan"), dtype=torch.float32, device="cuda")
    nb = pm.workspace_bytes(M)
    ws = torch.empty(nb, dtype=torch.uint8, device="cuda")
    w.wal_gemm_small_m(pm.desc, X_dev.data_ptr(), M, pm.K, Y.data_ptr(), pm.N, ws.data_ptr(), nb, stream())
    torch.cuda.synchronize()
    w.wal_device_status(ws.data_ptr(), stream())
    return Y.cpu().numpy().astype(np.float64)


def assert_parity(y, y_ref, x_bits, alpha_bits, what=""):
    """Every value finite (outputs start as NaN, so an unwritten one shows) and
    within the oracle tolerance."""
    assert np.all(np.isfinite(y)), f"{what}: {int(np.size(y) - np.count_nonzero(np.isfinite(y)))} outputs not finite"
    ok, rel, worst = oracle.check_tolerance(y, y_ref, x_bits, alpha_bits)
    assert ok, f"{what}: rel-L2 {rel:.3e} (<= 1e-5), max-abs ratio {worst:.3e} (<= 1)"
    return rel
