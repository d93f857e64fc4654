// The decode step around the ternary body: the INT3/g128 embedding gather and
// the INT4/g128 LM-head product (WAL-Ternary-8B card, Kazakh README, "Model
// format": embedding INT3/g128, LM head INT4/g128).
//
// Codes are offset binary (u = q + 8 for INT4, q + 4 for INT3) with an FP16
// scale per (row, 128 columns).  INT4: two codes per byte, low nibble first.
// INT3: a group's 128 codes form a 48-byte little-endian bit string, code j
// at bits 3j .. 3j + 2.
//
// The LM head runs in the kFmtInt4 specialisation of the decode-GEMV
// (wal_stream.cu).  The embedding gather is its own small kernel: one CTA per
// token, one thread per 8 codes (3 bytes), dequantised exactly to FP32.
#include "wal_internal.h"
#include "wal_stream.h"

#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <cstring>

namespace wal {
int launch_rows(const wal_matrix* m, const uint16_t* X, int ldx, float* Y, int ldy, int m0, int count,
                cudaStream_t stream, int32_t* status, int fmt);

namespace {

constexpr size_t kInt3GroupBytes = 48;

int check_int4(const wal_int4_matrix* m) {
  if (!m) return fail(WAL_ERR_ARG, "matrix descriptor is NULL");
  if (m->N <= 0 || m->K <= 0 || m->K % kGroup) return fail(WAL_ERR_SHAPE, "N must be > 0 and K a positive multiple of 128");
  if (m->K > kMaxK) return fail(WAL_ERR_UNSUPPORTED, "K above 24576 is not handled by this build");
  if (!m->codes || !m->scales) return fail(WAL_ERR_ARG, "codes and scales are required");
  if (((uintptr_t)m->codes | (uintptr_t)m->scales) & 15u) return fail(WAL_ERR_ARG, "planes must be 16-byte aligned");
  return WAL_OK;
}

__global__ void __launch_bounds__(256) int3_embed_kernel(const uint8_t* __restrict__ codes,
                                                          const uint16_t* __restrict__ scales, int V, int H,
                                                          const int32_t* __restrict__ ids, float* __restrict__ out,
                                                          int32_t* status) {
  const int m = blockIdx.x;
  const int id = ids[m];
  const int G = H / kGroup, chunks = H / 8;
  float* o = out + (size_t)m * H;
  if (id < 0 || id >= V) {  // outside the table: zeros, and the status word says so
    for (int c = threadIdx.x; c < chunks; c += blockDim.x) {
      reinterpret_cast<float4*>(o + 8 * c)[0] = make_float4(0.f, 0.f, 0.f, 0.f);
      reinterpret_cast<float4*>(o + 8 * c)[1] = make_float4(0.f, 0.f, 0.f, 0.f);
    }
    if (threadIdx.x == 0 && status) atomicExch(status, (int32_t)WAL_ERR_ARG);
    return;
  }
  const uint8_t* row = codes + (size_t)id * G * kInt3GroupBytes;
  for (int c = threadIdx.x; c < chunks; c += blockDim.x) {
    const int g = c >> 4;  // 16 chunks of 8 codes per group
    const uint8_t* b = row + (size_t)g * kInt3GroupBytes + 3 * (c & 15);
    const uint32_t bits = (uint32_t)__ldg(b) | ((uint32_t)__ldg(b + 1) << 8) | ((uint32_t)__ldg(b + 2) << 16);
    const float d = __half2float(__ushort_as_half(__ldg(scales + (size_t)id * G + g)));
    float v[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) v[i] = d * (float)((int)((bits >> (3 * i)) & 7u) - 4);
    reinterpret_cast<float4*>(o + 8 * c)[0] = make_float4(v[0], v[1], v[2], v[3]);
    reinterpret_cast<float4*>(o + 8 * c)[1] = make_float4(v[4], v[5], v[6], v[7]);
  }
}

}  // namespace
}  // namespace wal

using namespace wal;

extern "C" int wal_int4_sizes(int N, int K, size_t out[2]) {
  if (!out) return fail(WAL_ERR_ARG, "out is NULL");
  if (N <= 0 || K <= 0 || K % kGroup || (int64_t)N * K > (int64_t)1 << 40)
    return fail(WAL_ERR_SHAPE, "N must be > 0 and K a positive multiple of 128");
  out[0] = align_up((size_t)N * K / 2, 16);
  out[1] = align_up((size_t)N * (K / kGroup) * 2, 16);
  return WAL_OK;
}

extern "C" int wal_int4_pack(const int8_t* q, const uint16_t* d, int N, int K, void* codes, void* scales) {
  size_t sz[2];
  int st = wal_int4_sizes(N, K, sz);
  if (st) return st;
  if (!q || !d || !codes || !scales) return fail(WAL_ERR_ARG, "q, d, codes and scales are required");
  uint8_t* c = static_cast<uint8_t*>(codes);
  const size_t nc = (size_t)N * K / 2, ns = (size_t)N * (K / kGroup) * 2;
  std::memset(c + nc, 0, sz[0] - nc);
  std::memset(static_cast<uint8_t*>(scales) + ns, 0, sz[1] - ns);
  std::memcpy(scales, d, ns);
  int bad = 0;
#pragma omp parallel for schedule(static) reduction(| : bad)
  for (long long i = 0; i < (long long)nc; ++i) {
    const int lo = q[2 * i], hi = q[2 * i + 1];
    bad |= (lo < -8) | (lo > 7) | (hi < -8) | (hi > 7);
    c[i] = (uint8_t)((lo + 8) | ((hi + 8) << 4));
  }
  if (bad) return fail(WAL_ERR_FORMAT, "INT4 values must lie in [-8, 7]");
  return WAL_OK;
}

extern "C" size_t wal_int4_workspace_bytes(const wal_int4_matrix* m, int M) {
  if (check_int4(m) != WAL_OK || M < 1 || M > WAL_MAX_SMALL_M) return 0;
  return ws_layout(0, 0, 0, 0, 0).total;
}

extern "C" int wal_int4_gemm(const wal_int4_matrix* m, const uint16_t* X, int M, int ldx, float* Y, int ldy,
                             void* ws, size_t ws_bytes, wal_stream_t stream) {
  int st = check_int4(m);
  if (st) return st;
  if (!X || !Y) return fail(WAL_ERR_ARG, "activation and output pointers are required");
  if (((uintptr_t)X & 15u) || ((uintptr_t)Y & 3u)) return fail(WAL_ERR_ARG, "X must be 16-byte and Y 4-byte aligned");
  if (M < 1 || M > WAL_MAX_SMALL_M) return fail(WAL_ERR_SHAPE, "INT4 products take 1 <= M <= 16");
  if (ldx < m->K || ldy < m->N || (ldx % 8)) return fail(WAL_ERR_ARG, "ldx must be >= K and a multiple of 8; ldy >= N");
  if (!ws) return fail(WAL_ERR_ARG, "workspace is NULL");
  if (ws_bytes < wal_int4_workspace_bytes(m, M)) return fail(WAL_ERR_WORKSPACE, "workspace too small");
  st = stream_init();
  if (st) return st;
  wal_matrix v = {};
  v.N = m->N;
  v.K = m->K;
  v.codes = reinterpret_cast<const uint32_t*>(m->codes);
  v.scales = m->scales;
  int32_t* status = reinterpret_cast<int32_t*>(align_up((uintptr_t)ws, 256));
  return launch_rows(&v, X, ldx, Y, ldy, 0, M, (cudaStream_t)stream, status, kFmtInt4);
}

extern "C" int wal_int3_sizes(int V, int H, size_t out[2]) {
  if (!out) return fail(WAL_ERR_ARG, "out is NULL");
  if (V <= 0 || H <= 0 || H % kGroup || (int64_t)V * H > (int64_t)1 << 40)
    return fail(WAL_ERR_SHAPE, "V must be > 0 and H a positive multiple of 128");
  out[0] = align_up((size_t)V * (H / kGroup) * kInt3GroupBytes, 16);
  out[1] = align_up((size_t)V * (H / kGroup) * 2, 16);
  return WAL_OK;
}

extern "C" int wal_int3_pack(const int8_t* q, const uint16_t* d, int V, int H, void* codes, void* scales) {
  size_t sz[2];
  int st = wal_int3_sizes(V, H, sz);
  if (st) return st;
  if (!q || !d || !codes || !scales) return fail(WAL_ERR_ARG, "q, d, codes and scales are required");
  const size_t G = (size_t)H / kGroup, nc = (size_t)V * G * kInt3GroupBytes, ns = (size_t)V * G * 2;
  uint8_t* c = static_cast<uint8_t*>(codes);
  std::memset(c, 0, sz[0]);
  std::memset(static_cast<uint8_t*>(scales) + ns, 0, sz[1] - ns);
  std::memcpy(scales, d, ns);
  int bad = 0;
#pragma omp parallel for schedule(static) reduction(| : bad)
  for (long long gi = 0; gi < (long long)(V * G); ++gi) {
    const int8_t* src = q + (size_t)gi * kGroup;
    uint8_t* dst = c + (size_t)gi * kInt3GroupBytes;
    for (int j = 0; j < kGroup; ++j) {
      const int v = src[j];
      bad |= (v < -4) | (v > 3);
      const uint32_t u = (uint32_t)(v + 4) & 7u;
      for (int i = 0; i < 3; ++i) {
        const int bit = 3 * j + i;
        dst[bit >> 3] |= (uint8_t)(((u >> i) & 1u) << (bit & 7));
      }
    }
  }
  (void)nc;
  if (bad) return fail(WAL_ERR_FORMAT, "INT3 values must lie in [-4, 3]");
  return WAL_OK;
}

extern "C" int wal_int3_embed(const wal_int3_table* t, const int32_t* ids, int M, float* out, void* ws,
                              size_t ws_bytes, wal_stream_t stream) {
  if (!t || !ids || !out) return fail(WAL_ERR_ARG, "table, ids and out are required");
  if (t->V <= 0 || t->H <= 0 || t->H % kGroup) return fail(WAL_ERR_SHAPE, "V must be > 0 and H a positive multiple of 128");
  if (!t->codes || !t->scales) return fail(WAL_ERR_ARG, "codes and scales are required");
  if (M < 1) return fail(WAL_ERR_SHAPE, "M must be >= 1");
  if (((uintptr_t)out & 15u) || ((uintptr_t)ids & 3u)) return fail(WAL_ERR_ARG, "out must be 16-byte and ids 4-byte aligned");
  if (!ws || ws_bytes < 512) return fail(WAL_ERR_WORKSPACE, "the gather needs a 512-byte workspace");
  int32_t* status = reinterpret_cast<int32_t*>(align_up((uintptr_t)ws, 256));
  cudaStream_t s = (cudaStream_t)stream;
  cudaError_t e = cudaMemsetAsync(status, 0, 4, s);
  if (e != cudaSuccess) return fail(WAL_ERR_CUDA, std::string("status clear: ") + cudaGetErrorString(e));
  int3_embed_kernel<<<M, 256, 0, s>>>(t->codes, t->scales, t->V, t->H, ids, out, status);
  e = cudaGetLastError();
  if (e != cudaSuccess) return fail(WAL_ERR_CUDA, std::string("int3_embed_kernel launch: ") + cudaGetErrorString(e));
  return WAL_OK;
}
