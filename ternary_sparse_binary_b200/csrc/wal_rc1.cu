// RC1 storage: 24-bit float scales and two WALB2 paths.
//
// The WAL-Ternary-27B-RC1 card ("Representation") keeps the body scales in a
// 24-bit float format that the prepared compute cache expands to FP32, and
// the WALB2 correction as two packed binary low-rank paths.  wal_rc1_prepare
// is that expansion on the GPU: every 24-bit scale (the upper three bytes of
// an FP32) becomes an FP32, and the two paths become one rank block, path
// 1's ranks first (U words merged by a shift, V bit rows and scales
// concatenated).  The prepared matrix runs in the kFmtF32 specialisation of
// the decode-GEMV (wal_stream.cu): layout v1 with FP32 scales.
#include "wal_internal.h"
#include "wal_stream.h"

#include <cuda_runtime.h>

#include <algorithm>
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

struct PrepParams {
  const uint8_t* s24;
  const uint32_t *u1, *v1, *u2, *v2;
  const uint8_t *p1, *p2;  // per-rank 24-bit scales of the paths
  float* s32;
  uint32_t *ub, *vb;
  float* lr;
  int N, K, k, r1, r2;
};

__device__ __forceinline__ uint32_t f24_bits(const uint8_t* b) {
  return ((uint32_t)b[0] | ((uint32_t)b[1] << 8) | ((uint32_t)b[2] << 16)) << 8;
}

__global__ void __launch_bounds__(256) rc1_prepare_kernel(PrepParams p) {
  const size_t stride = (size_t)gridDim.x * blockDim.x, t0 = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
  const size_t G = (size_t)p.K / kGroup;
  const size_t nsc = (size_t)p.N * G * (p.k > 0 ? 2 : 1);
  for (size_t i = t0; i < nsc; i += stride) p.s32[i] = __uint_as_float(f24_bits(p.s24 + 3 * i));
  const int r = p.r1 + p.r2;
  if (r > 0) {
    const uint32_t m1 = p.r1 >= 32 ? 0xFFFFFFFFu : ((1u << p.r1) - 1u);
    const uint32_t m2 = p.r2 >= 32 ? 0xFFFFFFFFu : ((1u << p.r2) - 1u);
    for (size_t n = t0; n < (size_t)p.N; n += stride) {
      uint32_t u = 0u;
      if (p.r1) u = p.u1[n] & m1;
      if (p.r2) u |= (p.u2[n] & m2) << (p.r1 & 31);  // r1 + r2 <= 32: r1 = 32 only with r2 = 0
      p.ub[n] = u;
    }
    const size_t wpr = (size_t)p.K / 32, n1 = (size_t)p.r1 * wpr, nv = (size_t)r * wpr;
    for (size_t i = t0; i < nv; i += stride) p.vb[i] = i < n1 ? p.v1[i] : p.v2[i - n1];
    for (size_t i = t0; i < (size_t)r; i += stride)
      p.lr[i] = __uint_as_float(f24_bits(i < (size_t)p.r1 ? p.p1 + 3 * i : p.p2 + 3 * (i - p.r1)));
  }
  // zero the 16-byte padding of the FP32 planes and of u_bits
  if (t0 < 4) {
    const size_t pad_s = (nsc + 3) & ~(size_t)3;
    if (nsc + t0 < pad_s) p.s32[nsc + t0] = 0.f;
    if (r > 0) {
      const size_t pad_u = ((size_t)p.N + 3) & ~(size_t)3;
      if ((size_t)p.N + t0 < pad_u) p.ub[p.N + t0] = 0u;
      const size_t pad_l = ((size_t)r + 3) & ~(size_t)3;
      if ((size_t)r + t0 < pad_l) p.lr[r + t0] = 0.f;
    }
  }
}

int check_rc1(const wal_rc1_matrix* m) {
  if (!m) return fail(WAL_ERR_ARG, "matrix descriptor is NULL");
  int st = check_shape(m->N, m->K, m->k, m->r);
  if (st) return st;
  if (m->K > kMaxK) return fail(WAL_ERR_UNSUPPORTED, "K above 24576 is not handled by this build");
  if (!m->codes || !m->scales) return fail(WAL_ERR_ARG, "codes and scales are required");
  if (m->k > 0 && !m->sites) return fail(WAL_ERR_ARG, "sites are required when k > 0");
  if (m->r > 0 && (!m->u_bits || !m->v_bits || !m->lr_scale))
    return fail(WAL_ERR_ARG, "u_bits, v_bits and lr_scale are required when r > 0");
  if (((uintptr_t)m->codes | (uintptr_t)m->sites | (uintptr_t)m->scales | (uintptr_t)m->u_bits |
       (uintptr_t)m->v_bits | (uintptr_t)m->lr_scale) & 15u)
    return fail(WAL_ERR_ARG, "matrix buffers must be 16-byte aligned");
  return WAL_OK;
}

// The decode-GEMV's view: the layout-v1 descriptor with the FP32 planes in
// place of the FP16 ones (the kernel reads them as floats in kFmtF32).
wal_matrix as_matrix(const wal_rc1_matrix* m) {
  wal_matrix v = {};
  v.N = m->N; v.K = m->K; v.k = m->k; v.r = m->r;
  v.codes = m->codes;
  v.sites = m->sites;
  v.scales = reinterpret_cast<const uint16_t*>(m->scales);
  v.u_bits = m->u_bits;
  v.v_bits = m->v_bits;
  v.lr_scale = reinterpret_cast<const uint16_t*>(m->lr_scale);
  return v;
}

int check_io(const wal_rc1_matrix* m, const void* X, int M, int ldx, const void* Y, int ldy) {
  int st = check_rc1(m);
  if (st) return st;
  if (!X || !Y) return fail(WAL_ERR_ARG, "activation and output pointers are required");
  if (((uintptr_t)X & 15u) || ((uintptr_t)Y & 3u)) return fail(WAL_ERR_ARG, "X must be 16-byte and Y 4-byte aligned");
  if (M < 1 || M > WAL_MAX_SMALL_M) return fail(WAL_ERR_SHAPE, "RC1 products take 1 <= M <= 16");
  if (ldx < m->K || ldy < m->N || (ldx % 8)) return fail(WAL_ERR_ARG, "ldx must be >= K and a multiple of 8; ldy >= N");
  return stream_init();
}

}  // namespace
}  // namespace wal

using namespace wal;

extern "C" int wal_rc1_sizes(int N, int K, int k, int r1, int r2, size_t canonical[7], size_t prepared[4]) {
  if (!canonical || !prepared) return fail(WAL_ERR_ARG, "output arrays are required");
  if (r1 < 0 || r2 < 0 || r1 + r2 > WAL_MAX_RANK) return fail(WAL_ERR_SHAPE, "r1, r2 >= 0 and r1 + r2 <= 32");
  int st = check_shape(N, K, k, r1 + r2);
  if (st) return st;
  const size_t G = (size_t)K / kGroup, per = k > 0 ? 2 : 1;
  canonical[0] = align_up((size_t)N * G * per * 3, 16);
  canonical[1] = align_up((size_t)N * ((r1 + 31) / 32) * 4, 16);
  canonical[2] = align_up((size_t)r1 * (K / 8), 16);
  canonical[3] = align_up((size_t)r1 * 3, 16);
  canonical[4] = align_up((size_t)N * ((r2 + 31) / 32) * 4, 16);
  canonical[5] = align_up((size_t)r2 * (K / 8), 16);
  canonical[6] = align_up((size_t)r2 * 3, 16);
  const int r = r1 + r2;
  prepared[0] = align_up((size_t)N * G * per * 4, 16);
  prepared[1] = align_up((size_t)N * ((r + 31) / 32) * 4, 16);
  prepared[2] = align_up((size_t)r * (K / 8), 16);
  prepared[3] = align_up((size_t)r * 4, 16);
  return WAL_OK;
}

extern "C" int wal_rc1_prepare(int N, int K, int k, const uint8_t* scales24, int r1, const uint32_t* u1,
                               const uint32_t* v1, const uint8_t* s1_24, int r2, const uint32_t* u2,
                               const uint32_t* v2, const uint8_t* s2_24, float* scales32, uint32_t* u_bits,
                               uint32_t* v_bits, float* lr32, wal_stream_t stream) {
  size_t can[7], prep[4];
  int st = wal_rc1_sizes(N, K, k, r1, r2, can, prep);
  if (st) return st;
  if (!scales24 || !scales32) return fail(WAL_ERR_ARG, "scale planes are required");
  if (r1 > 0 && (!u1 || !v1 || !s1_24)) return fail(WAL_ERR_ARG, "path 1 buffers are required when r1 > 0");
  if (r2 > 0 && (!u2 || !v2 || !s2_24)) return fail(WAL_ERR_ARG, "path 2 buffers are required when r2 > 0");
  if (r1 + r2 > 0 && (!u_bits || !v_bits || !lr32)) return fail(WAL_ERR_ARG, "low-rank outputs are required");
  if (((uintptr_t)scales24 | (uintptr_t)u1 | (uintptr_t)v1 | (uintptr_t)s1_24 | (uintptr_t)u2 | (uintptr_t)v2 |
       (uintptr_t)s2_24 | (uintptr_t)scales32 | (uintptr_t)u_bits | (uintptr_t)v_bits | (uintptr_t)lr32) & 15u)
    return fail(WAL_ERR_ARG, "buffers must be 16-byte aligned");
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return fail(WAL_ERR_CUDA, "no CUDA device");
  PrepParams p = {scales24, u1, v1, u2, v2, s1_24, s2_24, scales32, u_bits, v_bits, lr32, N, K, k, r1, r2};
  rc1_prepare_kernel<<<sms * 4, 256, 0, (cudaStream_t)stream>>>(p);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return fail(WAL_ERR_CUDA, std::string("rc1_prepare_kernel launch: ") + cudaGetErrorString(e));
  return WAL_OK;
}

extern "C" size_t wal_rc1_workspace_bytes(const wal_rc1_matrix* m, int M) {
  if (check_rc1(m) != WAL_OK || M < 1 || M > WAL_MAX_SMALL_M) return 0;
  return ws_layout(0, 0, 0, 0, 0).total;
}

extern "C" int wal_rc1_gemm(const wal_rc1_matrix* m, const uint16_t* X, int M, int ldx, float* Y, int ldy, void* ws,
                            size_t ws_bytes, wal_stream_t stream) {
  int st = check_io(m, X, M, ldx, Y, ldy);
  if (st) return st;
  if (!ws) return fail(WAL_ERR_ARG, "workspace is NULL");
  if (ws_bytes < wal_rc1_workspace_bytes(m, M)) return fail(WAL_ERR_WORKSPACE, "workspace too small");
  const wal_matrix v = as_matrix(m);
  int32_t* status = reinterpret_cast<int32_t*>(align_up((uintptr_t)ws, 256));
  return launch_rows(&v, X, ldx, Y, ldy, 0, M, (cudaStream_t)stream, status, kFmtF32);
}

extern "C" size_t wal_rc1_body_workspace_bytes(const wal_rc1_matrix* mats, int n_mats, int M) {
  if (!mats || n_mats <= 0 || M < 1 || M > WAL_MAX_SMALL_M) return 0;
  for (int i = 0; i < n_mats; ++i)
    if (check_rc1(&mats[i]) != WAL_OK) return 0;
  return body_workspace_total(n_mats, M);
}

extern "C" int wal_rc1_body_pass(wal_body_plan** plan, const wal_rc1_matrix* mats, int n_mats,
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
  if (!ws || ws_bytes < wal_rc1_body_workspace_bytes(mats, n_mats, M))
    return fail(WAL_ERR_WORKSPACE, "body-pass workspace too small");
  return body_pass_impl(plan, kFmtF32, views.data(), n_mats, stage_of, xs, ys, M, ws, ws_bytes,
                        (cudaStream_t)stream);
}
