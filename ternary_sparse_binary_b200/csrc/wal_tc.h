// Tensor-core product for larger batches (see wal_tc.cu).
#pragma once

#include <cuda_runtime.h>

#include <cstddef>
#include <cstdint>

#include "../../include/wal.h"

namespace wal {

// Products of this many activation rows or more take the tensor-core path.
// Its time hardly grows with M up to a 16-row tile, while the CUDA-core path
// streams the weights once per row: measured on the 8B gate (down) shape at
// k = 8, r = 16, M = 4 takes 35.8 (48.1) us on CUDA cores and 42.0 (46.2) on
// the tensor path, M = 5 42.0 (56.3) against 42.1 (46.1).
constexpr int kTcMinM = 5;

// Geometry of one tensor-core call.
struct TcPlan {
  int n_tiles_n;  // 128-row tiles of W
  int n_mt;       // activation tiles
  int M_tile;     // activation rows per tile (MMA N), multiple of 16, <= 256
  int M_pad;      // n_mt * M_tile
  int stages;     // pipeline depth
  int ks, gps;    // K splits and 128-column groups per split
  uint32_t smem;  // dynamic shared memory per CTA
  uint32_t tmem_cols;
  int per_sm;     // CTAs resident per SM (1 or 2)
  // workspace offsets from the 256-byte aligned base
  size_t off_scal, off_zt, off_xt, off_part, total;
};

int plan_tc(const wal_matrix* m, int M, TcPlan* out);
// Scratch bytes of the tensor-core path (including the 256-byte alignment slack).
size_t tc_ws_bytes(const wal_matrix* m, int M);
int launch_tc(const wal_matrix* m, const uint16_t* X, int M, int ldx, float* Y, int ldy, char* ws_base,
              cudaStream_t stream);

}  // namespace wal
