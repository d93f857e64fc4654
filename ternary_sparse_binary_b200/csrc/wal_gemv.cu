// ABI entry points of the product (wal_gemv, wal_gemm_small_m) and the test /
// validation kernels (wal_unpack_matrix, wal_validate).  The batch-1
// decode-GEMV itself lives in wal_stream.cu.
#include "wal_internal.h"
#include "wal_device.cuh"
#include "wal_stream.h"
#include "wal_tc.h"

#include <algorithm>
#include <mutex>

namespace wal {

using namespace dev;

// ----------------------------------------------------------------------------
// test entry: decode with the same routines
// ----------------------------------------------------------------------------
struct UnpackParams {
  const uint32_t* codes;
  const uint8_t* sites;
  const uint16_t* scales;
  const uint32_t* ubits;
  const uint32_t* vbits;
  int N, K, k, r, G, words;
  int8_t* T;
  uint8_t* pos;
  int8_t* sgn;
  uint16_t* alpha;
  uint16_t* beta;
  int8_t* U;
  int8_t* V;
};

__global__ void unpack_kernel(UnpackParams p) {
  for (int n = blockIdx.x; n < p.N; n += gridDim.x) {
    if (p.T)
      for (int w = threadIdx.x; w < p.words; w += blockDim.x) {
        const uint32_t word = p.codes[(size_t)n * p.words + w];
#pragma unroll
        for (int s = 0; s < 4; ++s) {
          const uint32_t c4 = slot_codes(word, s);
#pragma unroll
          for (int b = 0; b < 4; ++b)
            p.T[(size_t)n * p.K + 16 * w + 4 * b + s] = (int8_t)code_to_trit((c4 >> (8 * b)) & 0xFFu);
        }
      }
    for (int gi = threadIdx.x; gi < p.G; gi += blockDim.x) {
      const size_t i = (size_t)n * p.G + gi;
      if (p.k > 0) {
        if (p.alpha) p.alpha[i] = p.scales[2 * i];
        if (p.beta) p.beta[i] = p.scales[2 * i + 1];
        for (int q = 0; q < p.k; ++q) {
          const uint32_t b = p.sites[i * p.k + q];
          if (p.pos) p.pos[i * p.k + q] = (uint8_t)site_position(b);
          if (p.sgn) p.sgn[i * p.k + q] = site_negative(b) ? -1 : 1;
        }
      } else {
        if (p.alpha) p.alpha[i] = p.scales[i];
        if (p.beta) p.beta[i] = 0;
      }
    }
    if (p.U)
      for (int rho = threadIdx.x; rho < p.r; rho += blockDim.x)
        p.U[(size_t)n * p.r + rho] = ((p.ubits[(size_t)n * ((p.r + 31) / 32) + rho / 32] >> (rho % 32)) & 1u) ? -1 : 1;
  }
  if (p.V) {
    const size_t total = (size_t)p.K * p.r;
    for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < total; i += (size_t)gridDim.x * blockDim.x) {
      const int j = (int)(i / p.r), rho = (int)(i % p.r);
      p.V[i] = ((p.vbits[(size_t)rho * (p.K / 32) + j / 32] >> (j % 32)) & 1u) ? -1 : 1;
    }
  }
}

// flag bits: 1 = reserved code, 2 = site positions not strictly ascending
__global__ void validate_kernel(const uint32_t* codes, const uint8_t* sites, int N, int K, int k,
                                uint32_t* flags) {
  const size_t nwords = (size_t)N * (K / 16);
  uint32_t f = 0u;
  for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < nwords; i += (size_t)gridDim.x * blockDim.x) {
    const uint32_t w = codes[i];
    if (w & (w >> 1) & 0x55555555u) f |= 1u;
  }
  if (k > 0) {
    const size_t ngroups = (size_t)N * (K / kGroup);
    for (size_t gi = (size_t)blockIdx.x * blockDim.x + threadIdx.x; gi < ngroups; gi += (size_t)gridDim.x * blockDim.x) {
      int prev = -1;
      for (int q = 0; q < k; ++q) {
        const int pos = (int)site_position(sites[gi * k + q]);
        if (pos <= prev) f |= 2u;
        prev = pos;
      }
    }
  }
  if (f) atomicOr(flags, f);
}

// ----------------------------------------------------------------------------
// host side
// ----------------------------------------------------------------------------
WsLayout ws_layout(int N, int K, int M, int n_slices, int n_row_blocks) {
  (void)N; (void)K; (void)M; (void)n_slices; (void)n_row_blocks;
  WsLayout L = {};
  L.header = 0;
  L.total = 256 + 256;  // header + slack for aligning the caller's base pointer
  return L;
}

namespace {

bool aligned16(const void* p) { return ((uintptr_t)p & 15u) == 0; }

int cuda_fail(cudaError_t e, const char* what) {
  return fail(WAL_ERR_CUDA, std::string(what) + ": " + cudaGetErrorString(e));
}

char* ws_base(void* ws) { return reinterpret_cast<char*>(align_up((uintptr_t)ws, 256)); }

}  // namespace

int check_matrix(const wal_matrix* m) {
  if (!m) return fail(WAL_ERR_ARG, "matrix descriptor is NULL");
  int st = check_shape(m->N, m->K, m->k, m->r);
  if (st) return st;
  if (m->K > kMaxK) return fail(WAL_ERR_UNSUPPORTED, "K above 24576 is not handled by this build");
  if (!m->codes || !m->scales) return fail(WAL_ERR_ARG, "codes and scales are required");
  if (m->k > 0 && !m->sites) return fail(WAL_ERR_ARG, "sites are required when k > 0");
  if (m->r > 0 && (!m->u_bits || !m->v_bits || !m->lr_scale))
    return fail(WAL_ERR_ARG, "u_bits, v_bits and lr_scale are required when r > 0");
  if (!aligned16(m->codes) || !aligned16(m->sites) || !aligned16(m->scales) || !aligned16(m->u_bits) ||
      !aligned16(m->v_bits) || !aligned16(m->lr_scale))
    return fail(WAL_ERR_ARG, "matrix buffers must be 16-byte aligned");
  return WAL_OK;
}

StreamItem make_item(const wal_matrix* m, const uint16_t* x, float* y) {
  StreamItem it = {};
  it.codes = m->codes; it.sites = m->sites; it.scales = m->scales;
  it.ubits = m->u_bits; it.vbits = m->v_bits; it.lr = m->lr_scale;
  it.x = x; it.y = y;
  it.N = m->N; it.k = m->k; it.r = m->r;
  return it;
}

// Products of one matrix for activation rows [m0, m0 + count) in one launch
// (one group: every product shares K).  fmt kFmtPq2: m->codes is a PQ2_0
// block buffer and k = r = 0.
int launch_rows(const wal_matrix* m, const uint16_t* X, int ldx, float* Y, int ldy, int m0, int count,
                cudaStream_t stream, int32_t* status, int fmt) {
  StreamParams prm = {};
  prm.status = status;
  prm.fmt = fmt;
  for (int i = 0; i < count; ++i)
    prm.items[i] = make_item(m, X + (size_t)(m0 + i) * ldx, Y + (size_t)(m0 + i) * ldy);
  int st = plan_group(prm.items, count, m->K, &prm.group);
  if (st) return st;
  StreamLaunch L;
  st = plan_launch(&prm.group, 1, false, fmt, &L);
  if (st) return st;
  return launch_stream(prm, L, stream);
}

// From 8 activation rows on the tensor-core path is faster: it decodes each
// weight once for all rows (its time hardly grows with M up to a 256-row
// tile), while the CUDA-core path streams the weights once per row.  On the
// 8B gate and down shapes at k = 8, r = 16 the two cross between M = 6 and 8.

int current_device(int* dev) {
  const cudaError_t e = cudaGetDevice(dev);
  if (e != cudaSuccess) return fail(WAL_ERR_CUDA, std::string("cudaGetDevice: ") + cudaGetErrorString(e));
  if (*dev < 0 || *dev >= kMaxDevices) return fail(WAL_ERR_UNSUPPORTED, "device ordinal above 63");
  return WAL_OK;
}

size_t product_ws_bytes(const wal_matrix* m, int M) {
  if (M >= kTcMinM) return tc_ws_bytes(m, M);
  return ws_layout(0, 0, 0, 0, 0).total;
}

int check_product_args(const wal_matrix* m, const void* X, int M, int ldx, const void* Y, int ldy) {
  int st = check_matrix(m);
  if (st) return st;
  if (!X || !Y) return fail(WAL_ERR_ARG, "activation and output pointers are required");
  if (!aligned16(X) || ((uintptr_t)Y & 3u)) return fail(WAL_ERR_ARG, "X must be 16-byte and Y 4-byte aligned");
  if (M < 1) return fail(WAL_ERR_SHAPE, "M must be >= 1");
  if (ldx < m->K || ldy < m->N || (ldx % 8))
    return fail(WAL_ERR_ARG, "ldx must be >= K and a multiple of 8; ldy must be >= N");
  return stream_init();
}

}  // namespace wal

using namespace wal;

extern "C" size_t wal_workspace_bytes(const wal_matrix* m, int M) {
  if (check_matrix(m) != WAL_OK || M < 1) return 0;
  return product_ws_bytes(m, M);
}

static int ws_check(void* ws, size_t ws_bytes, size_t need) {
  if (!ws) return fail(WAL_ERR_ARG, "workspace is NULL");
  if (need == 0 || ws_bytes < need) return fail(WAL_ERR_WORKSPACE, "workspace too small");
  return WAL_OK;
}

extern "C" int wal_gemv(const wal_matrix* m, const uint16_t* x, float* y, void* ws, size_t ws_bytes,
                        wal_stream_t stream) {
  int st = check_product_args(m, x, 1, m ? m->K : 0, y, m ? m->N : 0);
  if (st) return st;
  st = ws_check(ws, ws_bytes, product_ws_bytes(m, 1));
  if (st) return st;
  return launch_rows(m, x, m->K, y, m->N, 0, 1, (cudaStream_t)stream, reinterpret_cast<int32_t*>(ws_base(ws)),
                     kFmtV1);
}

extern "C" int wal_gemm_small_m(const wal_matrix* m, const uint16_t* X, int M, int ldx, float* Y, int ldy,
                                void* ws, size_t ws_bytes, wal_stream_t stream) {
  int st = check_product_args(m, X, M, ldx, Y, ldy);
  if (st) return st;
  st = ws_check(ws, ws_bytes, product_ws_bytes(m, M));
  if (st) return st;
  // 8 or more activation rows: the product is a dense contraction (tensor cores)
  if (M >= kTcMinM) return launch_tc(m, X, M, ldx, Y, ldy, ws_base(ws), (cudaStream_t)stream);
  for (int m0 = 0; m0 < M; m0 += kMaxItems) {
    st = launch_rows(m, X, ldx, Y, ldy, m0, std::min(kMaxItems, M - m0), (cudaStream_t)stream,
                     reinterpret_cast<int32_t*>(ws_base(ws)), kFmtV1);
    if (st) return st;
  }
  return WAL_OK;
}

extern "C" int wal_unpack_matrix(const wal_matrix* m, int8_t* T, uint8_t* site_pos, int8_t* site_sign,
                                 uint16_t* alpha, uint16_t* beta, int8_t* U, int8_t* V, wal_stream_t stream) {
  int st = check_matrix(m);
  if (st) return st;
  st = stream_init();
  if (st) return st;
  UnpackParams p;
  p.codes = m->codes; p.sites = m->sites; p.scales = m->scales; p.ubits = m->u_bits; p.vbits = m->v_bits;
  p.N = m->N; p.K = m->K; p.k = m->k; p.r = m->r; p.G = m->K / kGroup; p.words = m->K / 16;
  p.T = T; p.pos = m->k ? site_pos : nullptr; p.sgn = m->k ? site_sign : nullptr;
  p.alpha = alpha; p.beta = beta; p.U = m->r ? U : nullptr; p.V = m->r ? V : nullptr;
  const int blocks = std::min(m->N, 148 * 8);
  unpack_kernel<<<blocks, 256, 0, (cudaStream_t)stream>>>(p);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "unpack_kernel launch");
  return WAL_OK;
}

extern "C" int wal_validate(const wal_matrix* m, void* ws, size_t ws_bytes, wal_stream_t stream) {
  int st = check_matrix(m);
  if (st) return st;
  if (!ws || ws_bytes < 512) return fail(WAL_ERR_WORKSPACE, "validate needs a 512-byte workspace");
  st = stream_init();
  if (st) return st;
  uint32_t* flags = reinterpret_cast<uint32_t*>(ws_base(ws)) + 1;
  cudaStream_t s = (cudaStream_t)stream;
  cudaError_t e = cudaMemsetAsync(flags, 0, 4, s);
  if (e != cudaSuccess) return cuda_fail(e, "validate memset");
  validate_kernel<<<148 * 4, 256, 0, s>>>(m->codes, m->sites, m->N, m->K, m->k, flags);
  e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "validate_kernel launch");
  uint32_t h = 0;
  e = cudaMemcpyAsync(&h, flags, 4, cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return cuda_fail(e, "validate readback");
  if (h & 1u) return fail(WAL_ERR_FORMAT, "reserved trit code 3 found");
  if (h & 2u) return fail(WAL_ERR_FORMAT, "residual site positions not strictly ascending");
  return WAL_OK;
}

extern "C" int wal_device_status(void* ws, wal_stream_t stream) {
  if (!ws) return fail(WAL_ERR_ARG, "workspace is NULL");
  int32_t* word = reinterpret_cast<int32_t*>(ws_base(ws));
  int32_t h = 0;
  cudaStream_t s = (cudaStream_t)stream;
  cudaError_t e = cudaMemcpyAsync(&h, word, 4, cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess) e = cudaMemsetAsync(word, 0, 4, s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return cuda_fail(e, "device status readback");
  if (h == WAL_ERR_ARG) return fail(WAL_ERR_ARG, "a token id is outside the embedding table");
  if (h != 0) return fail(WAL_ERR_TIMEOUT, "a bounded device wait gave up");
  return WAL_OK;
}
