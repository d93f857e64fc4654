"""FP64 CPU oracle for the direct-packed body-matrix product.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path may import this
package: only the tests, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` /
``--impl reference`` legs of ``bench.py`` use it.  It shares no code with the
C++/CUDA library and imports nothing from it.
"""
from .wal_oracle import (  # noqa: F401
    pack,
    unpack,
    packed_sizes,
    payload_sizes,
    bits_per_weight,
    dense_weight,
    matvec,
    matmul,
    matmul_rows,
    widen_fp16,
    widen_bf16,
    check_tolerance,
    FormatError,
)
