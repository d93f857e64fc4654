"""B200-native direct-packed body-matrix product (libwal.so) -- Python binding.

The binding only marshals arguments into the C ABI declared in include/wal.h;
every step of the product runs in the library's CUDA kernels.  PyTorch is
used for device memory and streams.  There is no CPU fallback: if libwal.so
cannot be loaded, importing this package raises.
"""
from ._abi import (  # noqa: F401
    WAL_OK, WAL_ERR_ARG, WAL_ERR_SHAPE, WAL_ERR_FORMAT, WAL_ERR_WORKSPACE, WAL_ERR_CUDA,
    WAL_ERR_UNSUPPORTED, WAL_ERR_TIMEOUT, WAL_MAX_RANK, WAL_MAX_SMALL_M, WAL_NOALLOC_SCRATCH_BYTES,
    WalError, wal_matrix, lib, lib_path, EXPORTED_SYMBOLS,
    wal_packed_sizes, wal_pack_matrix, wal_validate, wal_unpack_matrix, wal_workspace_bytes,
    wal_gemv, wal_gemm_small_m, wal_gemm_tc_noalloc, wal_noalloc_status, wal_device_status, wal_body_workspace_bytes, wal_body_pass,
    wal_body_plan_destroy, wal_debug_barrier_fault, wal_status_string, wal_last_error,
    wal_pq2_matrix, wal_pq2_bytes, wal_pq2_pack, wal_pq2_workspace_bytes, wal_pq2_gemm,
    wal_pq2_body_workspace_bytes, wal_pq2_body_pass,
    wal_base3_bytes, wal_base3_pack, wal_base3_convert,
    wal_rc1_matrix, wal_rc1_sizes, wal_rc1_prepare, wal_rc1_workspace_bytes, wal_rc1_gemm,
    wal_rc1_body_workspace_bytes, wal_rc1_body_pass,
    wal_int4_matrix, wal_int3_table, wal_int4_sizes, wal_int3_sizes, wal_int4_pack, wal_int3_pack,
    wal_int4_workspace_bytes, wal_int4_gemm, wal_int3_embed,
)
from .packed import PackedMatrix, Pq2Matrix, Rc1Matrix, pack_host, pack_pq2_host, to_device, BodyPass  # noqa: F401
