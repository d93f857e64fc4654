"""The C-ABI library loads on a CPU-only host and exports every declared entry point."""
import ctypes
import os
import re

import pytest

import ternary_sparse_binary_b200 as wal

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_functions():
    src = open(os.path.join(ROOT, "include", "wal.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(wal_[a-z0-9_]+)\s*\(", src)))


def test_header_declares_the_entry_points():
    names = declared_functions()
    for required in ("wal_pack_matrix", "wal_gemv", "wal_gemm_small_m", "wal_body_pass"):
        assert required in names


@pytest.mark.parametrize("name", declared_functions())
def test_symbol_exported(name):
    lib = ctypes.CDLL(wal.lib_path)
    assert hasattr(lib, name), name


def test_binding_covers_header():
    assert set(declared_functions()) <= set(wal.EXPORTED_SYMBOLS)


def test_status_strings():
    assert wal.wal_status_string(0) == "WAL_OK"
    assert wal.wal_status_string(-7) == "WAL_ERR_TIMEOUT"
    assert wal.wal_status_string(-99) == "WAL_ERR_UNKNOWN"


def test_device_calls_fail_cleanly_without_args():
    # argument checks run before any CUDA call
    with pytest.raises(wal.WalError) as e:
        wal.wal_gemv(wal.wal_matrix(4, 100, 0, 0), None, None, None, 0, None)
    assert e.value.status in (wal.WAL_ERR_SHAPE, wal.WAL_ERR_ARG)
