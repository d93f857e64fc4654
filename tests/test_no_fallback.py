"""There is no CPU fallback: without its CUDA library the package does not
import, and on a host without a GPU every device entry point fails with
WAL_ERR_CUDA instead of computing anything."""
import os
import subprocess
import sys

import numpy as np
import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_import_fails_loudly_without_the_library():
    # the package's build module is replaced before the package loads: the
    # library file does not exist and cannot be built
    code = ("import sys, types; sys.path.insert(0, %r)\n"
            "fake = types.ModuleType('ternary_sparse_binary_b200.build')\n"
            "fake.LIB = '/nonexistent/libwal.so'\n"
            "def nobuild(*a, **k):\n"
            "    raise RuntimeError('no compiler')\n"
            "fake.build = nobuild\n"
            "sys.modules['ternary_sparse_binary_b200.build'] = fake\n"
            "import ternary_sparse_binary_b200\n" % ROOT)
    r = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True, timeout=300)
    assert r.returncode != 0
    assert "no compiler" in r.stderr


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the behaviour on a host without a GPU")
def test_device_entry_points_refuse_without_a_gpu():
    import ternary_sparse_binary_b200 as wal
    from wal_synth import gen_components, gen_x
    c = gen_components(64, 256, 8, 2, config_id=3)
    bufs = [np.ascontiguousarray(b) for b in wal.pack_host(c)]
    ptrs = [b.ctypes.data if b.size else None for b in bufs]
    # host pointers stand in for device ones: the call must stop before any access
    m = wal.wal_matrix(64, 256, 8, 2, *ptrs)
    x = np.zeros(256, np.uint16)
    y = np.zeros(64, np.float32)
    ws = np.zeros(1024, np.uint8)
    with pytest.raises(wal.WalError) as e:
        wal.wal_gemv(m, x.ctypes.data, y.ctypes.data, ws.ctypes.data, ws.size, None)
    assert e.value.status == wal.WAL_ERR_CUDA
    assert not y.any()
