// ABI entry points of the PQ2_0 plain-ternary block format: sizes, the host
// packer, the small-M product and the body pass.  PQ2_0 is the fast native
// GGUF format of the WAL2-Ternary-27B card (section on bit widths): per 128
// weights an FP16 scale and 32 bytes of 2-bit codes.  The device work runs
// in the kFmtPq2 specialisation of the decode-GEMV (wal_stream.cu).
#include "wal_internal.h"
#include "wal_stream.h"

#include <cuda_runtime.h>

#include <algorithm>
#include <cstring>
#include <vector>

struct wal_body_plan;

namespace wal {
int launch_rows(const wal_matrix* m, const uint16_t* X, int ldx, float* Y, int ldy, int m0, int count,
                cudaStream_t stream, int32_t* status, int fmt);
size_t body_workspace_total(int n_mats, int M);
int body_pass_impl(wal_body_plan** plan, int fmt, const wal_matrix* mats, int n_mats, const int32_t* stage_of,
                   const uint16_t* const* xs, float* const* ys, int M, void* ws, size_t ws_bytes,
                   cudaStream_t stream);

namespace {

constexpr size_t kBlockBytes = 34;

size_t pq2_bytes(int N, int K) { return align_up((size_t)N * (K / kGroup) * kBlockBytes, 16); }

int check_pq2(const wal_pq2_matrix* m) {
  if (!m) return fail(WAL_ERR_ARG, "matrix descriptor is NULL");
  if (m->N <= 0 || m->K <= 0 || m->K % kGroup) return fail(WAL_ERR_SHAPE, "N must be > 0 and K a positive multiple of 128");
  if (m->K > kMaxK) return fail(WAL_ERR_UNSUPPORTED, "K above 24576 is not handled by this build");
  if ((int64_t)m->N * m->K > (int64_t)1 << 40) return fail(WAL_ERR_SHAPE, "matrix too large");
  if (!m->blocks) return fail(WAL_ERR_ARG, "blocks is NULL");
  if ((uintptr_t)m->blocks & 15u) return fail(WAL_ERR_ARG, "blocks must be 16-byte aligned");
  return WAL_OK;
}

// The decode-GEMV's view of a PQ2_0 matrix: the block buffer in place of the
// code plane, no sites, no scales plane, no low-rank pair.
wal_matrix as_matrix(const wal_pq2_matrix* m) {
  wal_matrix v = {};
  v.N = m->N;
  v.K = m->K;
  v.codes = reinterpret_cast<const uint32_t*>(m->blocks);
  return v;
}

int check_io(const wal_pq2_matrix* m, const void* X, int M, int ldx, const void* Y, int ldy) {
  int st = check_pq2(m);
  if (st) return st;
  if (!X || !Y) return fail(WAL_ERR_ARG, "activation and output pointers are required");
  if (((uintptr_t)X & 15u) || ((uintptr_t)Y & 3u)) return fail(WAL_ERR_ARG, "X must be 16-byte and Y 4-byte aligned");
  if (M < 1 || M > WAL_MAX_SMALL_M) return fail(WAL_ERR_SHAPE, "PQ2_0 products take 1 <= M <= 16");
  if (ldx < m->K || ldy < m->N || (ldx % 8)) return fail(WAL_ERR_ARG, "ldx must be >= K and a multiple of 8; ldy >= N");
  return stream_init();
}

}  // namespace
}  // namespace wal

using namespace wal;

extern "C" size_t wal_pq2_bytes(int N, int K) {
  if (N <= 0 || K <= 0 || K % kGroup || (int64_t)N * K > (int64_t)1 << 40) return 0;
  return pq2_bytes(N, K);
}

extern "C" int wal_pq2_pack(const int8_t* T, const uint16_t* d, int N, int K, void* out) {
  if (N <= 0 || K <= 0 || K % kGroup) return fail(WAL_ERR_SHAPE, "N must be > 0 and K a positive multiple of 128");
  if (!T || !d || !out) return fail(WAL_ERR_ARG, "T, d and out must be non-NULL");
  const int G = K / kGroup;
  uint8_t* o = static_cast<uint8_t*>(out);
  const size_t used = (size_t)N * G * kBlockBytes, total = pq2_bytes(N, K);
  std::memset(o + used, 0, total - used);
  int bad_rows = 0;
#pragma omp parallel for schedule(static) reduction(+ : bad_rows)
  for (int n = 0; n < N; ++n) {
    int bad = 0;
    for (int g = 0; g < G; ++g) {
      uint8_t* blk = o + ((size_t)n * G + g) * kBlockBytes;
      const uint16_t dv = d[(size_t)n * G + g];
      blk[0] = (uint8_t)(dv & 0xFFu);
      blk[1] = (uint8_t)(dv >> 8);
      const int8_t* t = T + (size_t)n * K + (size_t)g * kGroup;
      for (int b = 0; b < 32; ++b) {
        uint32_t byte = 0;
        for (int i = 0; i < 4; ++i) {
          const int v = t[4 * b + i];
          bad |= (v < -1) | (v > 1);
          byte |= (uint32_t)(v + 1) << (2 * i);
        }
        blk[2 + b] = (uint8_t)byte;
      }
    }
    bad_rows += bad;
  }
  if (bad_rows) return fail(WAL_ERR_FORMAT, "T outside {-1,0,1}");
  return WAL_OK;
}

extern "C" size_t wal_pq2_workspace_bytes(const wal_pq2_matrix* m, int M) {
  if (check_pq2(m) != WAL_OK || M < 1 || M > WAL_MAX_SMALL_M) return 0;
  return ws_layout(0, 0, 0, 0, 0).total;
}

extern "C" int wal_pq2_gemm(const wal_pq2_matrix* m, const uint16_t* X, int M, int ldx, float* Y, int ldy, void* ws,
                            size_t ws_bytes, wal_stream_t stream) {
  int st = check_io(m, X, M, ldx, Y, ldy);
  if (st) return st;
  if (!ws) return fail(WAL_ERR_ARG, "workspace is NULL");
  if (ws_bytes < wal_pq2_workspace_bytes(m, M)) return fail(WAL_ERR_WORKSPACE, "workspace too small");
  const wal_matrix v = as_matrix(m);
  int32_t* status = reinterpret_cast<int32_t*>(align_up((uintptr_t)ws, 256));
  return launch_rows(&v, X, ldx, Y, ldy, 0, M, (cudaStream_t)stream, status, kFmtPq2);
}

extern "C" size_t wal_pq2_body_workspace_bytes(const wal_pq2_matrix* mats, int n_mats, int M) {
  if (!mats || n_mats <= 0 || M < 1 || M > WAL_MAX_SMALL_M) return 0;
  for (int i = 0; i < n_mats; ++i)
    if (check_pq2(&mats[i]) != WAL_OK) return 0;
  return body_workspace_total(n_mats, M);
}

extern "C" int wal_pq2_body_pass(wal_body_plan** plan, const wal_pq2_matrix* mats, int n_mats,
                                 const int32_t* stage_of, const uint16_t* const* xs, float* const* ys, int M,
                                 void* ws, size_t ws_bytes, wal_stream_t stream) {
  if (!plan || !mats || !stage_of || !xs || !ys || n_mats <= 0)
    return fail(WAL_ERR_ARG, "plan, mats, stage_of, xs and ys are required and n_mats > 0");
  std::vector<wal_matrix> views((size_t)n_mats);
  for (int i = 0; i < n_mats; ++i) {
    int st = check_io(&mats[i], xs[i], M, mats[i].K, ys[i], mats[i].N);
    if (st) return st;
    if (i && stage_of[i] < stage_of[i - 1]) return fail(WAL_ERR_ARG, "stage_of must be non-decreasing");
    views[i] = as_matrix(&mats[i]);
  }
  if (!ws || ws_bytes < wal_pq2_body_workspace_bytes(mats, n_mats, M))
    return fail(WAL_ERR_WORKSPACE, "body-pass workspace too small");
  return body_pass_impl(plan, kFmtPq2, views.data(), n_mats, stage_of, xs, ys, M, ws, ws_bytes,
                        (cudaStream_t)stream);
}
