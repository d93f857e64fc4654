// Decode-GEMV family for the direct-packed body-matrix product
//   y = (alpha*T + beta*R) x + sum_r s_r U_r (V_r^T x)
// (WAL-Ternary-8B model card, "Representation"), batch M = 1.
//
// Design (sm_100a, CUDA cores; the path is HBM-bound at batch 1):
//   * prep_x_kernel: x (bf16) -> per 128-group fixed-point image.  With
//     e_g = the largest exponent in group g, X_j = x_j * 2^(21 - e_g) is an
//     integer of at most 23 bits (exact whenever x_j is within 2^-14 of the
//     group maximum, round-to-nearest-even below that).  X_j is split into
//     three byte limbs lo, mid (unsigned) and hi (signed).  The kernel also
//     writes the per-word sums of X, the group weight 2^(e_g - 21), and the
//     WALB2 phase-1 vector z_r = s_r * V_r^T x (exact integer partial per
//     group, FP32 across groups).
//   * gemv_kernel: one warp covers a K-slice of 2048 columns, 64 per lane
//     (4 code words), and keeps its x limbs in registers while it walks rows.
//     Each lane streams its own 16-byte code chunk, residual-site bytes and
//     {alpha, beta} through a private cp.async ring in shared memory, so many
//     rows are in flight without spending registers.  The trit decode is
//     "mask the code word by slot" and the per-group dot is three byte-wise
//     dp4a products against the limbs (codes are t + 1, so the dot is
//     sum_j c_j X_j - sum_j X_j, exact in int32).  The group partial becomes
//     FP32 once (times 2^(e_g - 21)), then alpha and beta are applied in FP32.
//     Residual sites read +-x from a per-CTA shared-memory table indexed by
//     the site byte itself.  Lanes reduce by warp shuffles; K-slices combine
//     through a deterministic split-K pass (the last CTA of a row block sums
//     the slice partials in slice order), which also adds the WALB2 phase-2
//     term sum_r U[n, r] z_r and writes y once.
#include "wal_internal.h"
#include "wal_device.cuh"

#include <algorithm>
#include <mutex>

namespace wal {

using namespace dev;

// ----------------------------------------------------------------------------
// prep: x -> fixed-point limb image, word sums, group weights, WALB2 z
// ----------------------------------------------------------------------------
struct PrepParams {
  const uint16_t* X;
  int ldx, K, G, r, M;
  const uint32_t* vbits;
  const uint16_t* lr;
  uint32_t* limbs;
  int32_t* xsum;
  float* gscale;
  float* z;
  uint32_t* counters;
  int n_counters;
  int32_t* status;  // workspace header word 0
};

__device__ __forceinline__ uint32_t rne_shift_right(uint32_t m, int d) {
  if (d > 8) return 0u;  // m < 2^8, so m * 2^-d < 1/2
  const uint32_t q = m >> d, rem = m & ((1u << d) - 1u), half = 1u << (d - 1);
  return q + ((rem > half) || (rem == half && (q & 1u)) ? 1u : 0u);
}

__global__ void __launch_bounds__(512) prep_x_kernel(PrepParams p) {
  extern __shared__ int32_t prep_smem[];
  int32_t* zpart = prep_smem;                              // [r][G]
  float* gsc_s = reinterpret_cast<float*>(prep_smem + p.r * p.G);  // [G]
  const int m = blockIdx.x;
  const uint16_t* x = p.X + (size_t)m * p.ldx;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nwarps = blockDim.x >> 5;
  const int words = p.K / 16;
  if (m == 0) {
    for (int i = threadIdx.x; i < p.n_counters; i += blockDim.x) p.counters[i] = 0u;
    if (threadIdx.x == 0) *p.status = 0;  // the status word describes this product call
  }

  for (int g = warp; g < p.G; g += nwarps) {
    const int c0 = g * 128 + 4 * lane;
    const uint2 raw = *reinterpret_cast<const uint2*>(x + c0);
    const uint32_t b[4] = {raw.x & 0xFFFFu, raw.x >> 16, raw.y & 0xFFFFu, raw.y >> 16};
    uint32_t ep[4], emax = 1u;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const uint32_t e = (b[i] >> 7) & 0xFFu;
      ep[i] = e > 1u ? e : 1u;
      emax = ep[i] > emax ? ep[i] : emax;
    }
    emax = __reduce_max_sync(0xffffffffu, emax);
    int32_t X[4];
    int32_t sumx = 0;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const uint32_t e = (b[i] >> 7) & 0xFFu;
      const uint32_t mant = (b[i] & 0x7Fu) | (e ? 0x80u : 0u);
      const int sh = (int)ep[i] - (int)emax + 14;
      const uint32_t mag = sh >= 0 ? (mant << sh) : rne_shift_right(mant, -sh);
      X[i] = (b[i] & 0x8000u) ? -(int32_t)mag : (int32_t)mag;
      sumx += X[i];
    }
    // limb image: word w holds 12 uint32 = [limb L][slot s], byte b = column 16w + 4b + s
    const int word = g * 8 + (lane >> 2), bpos = lane & 3;
    uint8_t* img = reinterpret_cast<uint8_t*>(p.limbs + ((size_t)m * words + word) * kLimbWords);
#pragma unroll
    for (int s = 0; s < 4; ++s) {
      img[(0 * 4 + s) * 4 + bpos] = (uint8_t)(X[s] & 0xFF);
      img[(1 * 4 + s) * 4 + bpos] = (uint8_t)((X[s] >> 8) & 0xFF);
      img[(2 * 4 + s) * 4 + bpos] = (uint8_t)((X[s] >> 16) & 0xFF);
    }
    sumx += __shfl_xor_sync(0xffffffffu, sumx, 1);
    sumx += __shfl_xor_sync(0xffffffffu, sumx, 2);
    if (bpos == 0) p.xsum[(size_t)m * words + word] = sumx;
    // weight of one fixed-point unit: 2^(emax - 127 - 21)
    const float sc = emax >= 22u ? __uint_as_float((emax - 21u) << 23) : __uint_as_float(1u << (emax + 1u));
    if (lane == 0) {
      p.gscale[(size_t)m * p.G + g] = sc;
      gsc_s[g] = sc;
    }
    // WALB2 phase 1, exact per group: sum_j V[j, rho] X_j
    for (int rho = 0; rho < p.r; ++rho) {
      const uint32_t vw = p.vbits[(size_t)rho * (p.K / 32) + g * 4 + (lane >> 3)];
      const uint32_t nib = (vw >> (4 * (lane & 7))) & 0xFu;
      int32_t t = 0;
#pragma unroll
      for (int i = 0; i < 4; ++i) t += ((nib >> i) & 1u) ? -X[i] : X[i];
      t = __reduce_add_sync(0xffffffffu, t);
      if (lane == 0) zpart[rho * p.G + g] = t;
    }
  }
  __syncthreads();
  for (int rho = warp; rho < p.r; rho += nwarps) {
    float acc = 0.f;
    for (int g = lane; g < p.G; g += 32) acc = fmaf((float)zpart[rho * p.G + g], gsc_s[g], acc);
    acc = warp_sum(acc);
    if (lane == 0) p.z[m * 32 + rho] = fp16_bits_to_float(p.lr[rho]) * acc;
  }
}

// ----------------------------------------------------------------------------
// decode-GEMV, batch 1
// ----------------------------------------------------------------------------
constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kStages = 8;          // per-lane cp.async ring depth (rows in flight per lane)
constexpr int kSliceGroups = kSliceCols / kGroup;  // 16

struct GemvParams {
  const uint32_t* codes;
  const uint8_t* sites;
  const uint16_t* scales;
  const uint32_t* ubits;
  int N, K, k, r, G, words;
  const uint16_t* x;          // bf16 [K]
  const uint32_t* limbs;      // ws
  const int32_t* xsum;        // ws
  const float* gscale;        // ws
  const float* z;             // ws [32]
  float* part;                // ws [S][N]
  uint32_t* counters;         // ws [nRB]
  float* y;
  int S, RB, nRB;
};

__host__ __device__ constexpr size_t gemv_smem_bytes() {
  return (size_t)kSliceGroups * 256 * 4                    // +-x table
         + (size_t)kStages * kThreads * (16 + 4 + 4);       // rings: codes, sites, scales
}

template <int KS>
__global__ void __launch_bounds__(kThreads, 2) gemv_kernel(GemvParams p) {
  extern __shared__ __align__(16) unsigned char smem[];
  float* xt = reinterpret_cast<float*>(smem);
  uint4* ring_codes = reinterpret_cast<uint4*>(smem + kSliceGroups * 256 * 4);
  uint32_t* ring_site = reinterpret_cast<uint32_t*>(ring_codes + kStages * kThreads);
  uint32_t* ring_scale = ring_site + kStages * kThreads;
  __shared__ float s_z[32];
  __shared__ int s_last;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int sl = blockIdx.y, rb = blockIdx.x;
  const int n0 = rb * p.RB;
  const int rows = min(p.RB, p.N - n0);
  const int col_base = sl * kSliceCols;
  const int ncols = min(kSliceCols, p.K - col_base);
  const int col0 = col_base + lane * 64;
  const bool active = col0 < p.K;
  const int g = col0 >> 7;
  const int half = (col0 >> 6) & 1;
  const int gl = g - sl * kSliceGroups;

  // +-x table for the groups of this slice, indexed by the raw site byte
  for (int e = tid; e < ncols; e += kThreads) {
    const float v = bf16_bits_to_float(p.x[col_base + e]);
    xt[(e >> 7) * 256 + (e & 127)] = v;
    xt[(e >> 7) * 256 + 128 + (e & 127)] = -v;
  }
  if (tid < 32) s_z[tid] = tid < p.r ? p.z[tid] : 0.f;

  uint32_t lb[4][kLimbWords];
  int32_t xs = 0;
  float gsc = 0.f;
  if (active) {
    const uint4* src = reinterpret_cast<const uint4*>(p.limbs + (size_t)(col0 >> 4) * kLimbWords);
#pragma unroll
    for (int w = 0; w < 4; ++w) {
#pragma unroll
      for (int L = 0; L < 3; ++L) {
        const uint4 v = src[w * 3 + L];
        lb[w][L * 4 + 0] = v.x;
        lb[w][L * 4 + 1] = v.y;
        lb[w][L * 4 + 2] = v.z;
        lb[w][L * 4 + 3] = v.w;
      }
      xs += p.xsum[(col0 >> 4) + w];
    }
    gsc = p.gscale[g];
  } else {
#pragma unroll
    for (int w = 0; w < 4; ++w)
#pragma unroll
      for (int i = 0; i < kLimbWords; ++i) lb[w][i] = 0u;
  }
  __syncthreads();

  const int nmine = warp < rows ? (rows - warp + kWarps - 1) / kWarps : 0;
  auto issue = [&](int i) {
    const int rl = warp + kWarps * i;
    if (active && i < nmine) {
      const int n = n0 + rl;
      const int st = i % kStages;
      const size_t gi = (size_t)n * p.G + g;
      cp_async16(&ring_codes[st * kThreads + tid], p.codes + (size_t)n * p.words + (col0 >> 4));
      if (KS == 8) cp_async4(&ring_site[st * kThreads + tid], p.sites + gi * 8 + half * 4);
      if (KS == 4) cp_async4(&ring_site[st * kThreads + tid], p.sites + gi * 4);
      if (KS == 2) cp_async4(&ring_site[st * kThreads + tid], p.sites + ((gi * 2) & ~(size_t)3));
      if (KS > 0) cp_async4(&ring_scale[st * kThreads + tid], p.scales + gi * 2);
      else cp_async4(&ring_scale[st * kThreads + tid], p.scales + (gi & ~(size_t)1));
    }
    cp_async_commit();
  };

#pragma unroll 1
  for (int i = 0; i < kStages - 1; ++i) issue(i);

#pragma unroll 1
  for (int i = 0; i < nmine; ++i) {
    cp_async_wait<kStages - 2>();
    const int st = i % kStages;
    const int n = n0 + warp + kWarps * i;
    float part = 0.f;
    if (active) {
      const uint4 cw = ring_codes[st * kThreads + tid];
      const uint32_t words[4] = {cw.x, cw.y, cw.z, cw.w};
      uint32_t a0 = 0u, a1 = 0u;
      int32_t a2 = 0;
#pragma unroll
      for (int w = 0; w < 4; ++w) {
#pragma unroll
        for (int s = 0; s < 4; ++s) {
          const uint32_t msk = slot_codes(words[w], s);
          a0 = dp4a_uu(msk, lb[w][0 * 4 + s], a0);
          a1 = dp4a_uu(msk, lb[w][1 * 4 + s], a1);
          a2 = dp4a_us(msk, lb[w][2 * 4 + s], a2);
        }
      }
      const uint32_t acc = (uint32_t)a2 * 65536u + a1 * 256u + a0 - (uint32_t)xs;
      const float pf = (float)(int32_t)acc * gsc;
      const uint32_t sc = ring_scale[st * kThreads + tid];
      const size_t gi = (size_t)n * p.G + g;
      if (KS > 0) {
        const uint32_t sw = ring_site[st * kThreads + tid];
        const float* tab = xt + gl * 256;
        float q = 0.f;
        if (KS == 8) {
          q += tab[sw & 0xFFu];
          q += tab[(sw >> 8) & 0xFFu];
          q += tab[(sw >> 16) & 0xFFu];
          q += tab[sw >> 24];
        } else if (KS == 4) {
          const uint32_t two = sw >> (16 * half);
          q += tab[two & 0xFFu];
          q += tab[(two >> 8) & 0xFFu];
        } else {
          const uint32_t off = (uint32_t)((gi * 2) & 3) + (uint32_t)half;
          q += tab[(sw >> (8 * off)) & 0xFFu];
        }
        const float alpha = fp16_bits_to_float(sc & 0xFFFFu);
        const float beta = fp16_bits_to_float(sc >> 16);
        part = fmaf(alpha, pf, beta * q);
      } else {
        const float alpha = fp16_bits_to_float((sc >> (16 * (uint32_t)(gi & 1))) & 0xFFFFu);
        part = alpha * pf;
      }
    }
    if (p.S == 1 && p.r > 0) {
      const uint32_t uw = p.ubits[n];
      const float zl = s_z[lane];
      part += ((uw >> lane) & 1u) ? -zl : zl;   // lanes >= r hold z = 0
    }
    part = warp_sum(part);
    if (lane == 0) {
      if (p.S == 1) p.y[n] = part;
      else __stcg(&p.part[(size_t)sl * p.N + n], part);
    }
    issue(i + kStages - 1);
  }
  cp_async_wait<0>();

  if (p.S > 1) {
    __threadfence();
    __syncthreads();
    if (tid == 0) {
      const uint32_t prev = atomicAdd(&p.counters[rb], 1u);
      s_last = (prev == (uint32_t)(p.S - 1));
    }
    __syncthreads();
    if (s_last) {
      __threadfence();
      for (int rl = tid; rl < rows; rl += kThreads) {
        const int n = n0 + rl;
        float acc = 0.f;
        for (int s2 = 0; s2 < p.S; ++s2) acc += __ldcg(&p.part[(size_t)s2 * p.N + n]);
        if (p.r > 0) {
          const uint32_t uw = p.ubits[n];
          float lr = 0.f;
          for (int rho = 0; rho < p.r; ++rho) lr += ((uw >> rho) & 1u) ? -s_z[rho] : s_z[rho];
          acc += lr;
        }
        p.y[n] = acc;
      }
      if (tid == 0) p.counters[rb] = 0u;
    }
  }
}

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
  WsLayout L;
  const size_t words = (size_t)K / 16, G = (size_t)K / kGroup;
  size_t off = 0;
  auto take = [&](size_t bytes) { size_t o = off; off = align_up(off + bytes, 256); return o; };
  L.header = take(256);
  L.limbs = take((size_t)M * words * kLimbWords * 4);
  L.xsum = take((size_t)M * words * 4);
  L.gscale = take((size_t)M * G * 4);
  L.z = take((size_t)M * 32 * 4);
  L.part = take(n_slices > 1 ? (size_t)n_slices * M * N * 4 : 0);
  L.counters = take((size_t)(n_row_blocks > 0 ? n_row_blocks : 1) * 4);
  L.total = off + 256;  // slack for aligning the caller's base pointer
  return L;
}

namespace {

bool aligned16(const void* p) { return ((uintptr_t)p & 15u) == 0; }

int check_matrix(const wal_matrix* m) {
  if (!m) return fail(WAL_ERR_ARG, "matrix descriptor is NULL");
  int st = check_shape(m->N, m->K, m->k, m->r);
  if (st) return st;
  if (m->K > kMaxK) return fail(WAL_ERR_UNSUPPORTED, "K above 65536 is not handled by this build");
  if (!m->codes || !m->scales) return fail(WAL_ERR_ARG, "codes and scales are required");
  if (m->k > 0 && !m->sites) return fail(WAL_ERR_ARG, "sites are required when k > 0");
  if (m->r > 0 && (!m->u_bits || !m->v_bits || !m->lr_scale))
    return fail(WAL_ERR_ARG, "u_bits, v_bits and lr_scale are required when r > 0");
  if (!aligned16(m->codes) || !aligned16(m->sites) || !aligned16(m->scales) || !aligned16(m->u_bits) ||
      !aligned16(m->v_bits) || !aligned16(m->lr_scale))
    return fail(WAL_ERR_ARG, "matrix buffers must be 16-byte aligned");
  return WAL_OK;
}

int cuda_fail(cudaError_t e, const char* what) {
  return fail(WAL_ERR_CUDA, std::string(what) + ": " + cudaGetErrorString(e));
}

int g_num_sms = 0;
int g_gemv_occ[9] = {0};
std::once_flag g_init_flag;
cudaError_t g_init_err = cudaSuccess;

template <int KS>
cudaError_t init_gemv_kernel() {
  cudaError_t e = cudaFuncSetAttribute(gemv_kernel<KS>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)gemv_smem_bytes());
  if (e != cudaSuccess) return e;
  return cudaOccupancyMaxActiveBlocksPerMultiprocessor(&g_gemv_occ[KS], gemv_kernel<KS>, kThreads,
                                                       gemv_smem_bytes());
}

int ensure_init() {
  std::call_once(g_init_flag, [] {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&g_num_sms, cudaDevAttrMultiProcessorCount, dev);
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(prep_x_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               (kMaxK / kGroup) * (WAL_MAX_RANK + 1) * 4);
    if (e == cudaSuccess) e = init_gemv_kernel<0>();
    if (e == cudaSuccess) e = init_gemv_kernel<2>();
    if (e == cudaSuccess) e = init_gemv_kernel<4>();
    if (e == cudaSuccess) e = init_gemv_kernel<8>();
    g_init_err = e;
  });
  if (g_init_err != cudaSuccess) return cuda_fail(g_init_err, "device initialisation");
  return WAL_OK;
}

struct GemvPlan {
  int S, RB, nRB;
};

GemvPlan plan_gemv(int N, int K, int k) {
  GemvPlan g;
  g.S = (K + kSliceCols - 1) / kSliceCols;
  const int occ = std::max(1, g_gemv_occ[k]);
  const long slots = (long)std::max(1, g_num_sms) * occ;
  long rb = ((long)N * g.S + slots - 1) / slots;
  rb = std::max(8L, (rb + 7) / 8 * 8);
  g.RB = (int)rb;
  g.nRB = (N + g.RB - 1) / g.RB;
  return g;
}

char* ws_base(void* ws) { return reinterpret_cast<char*>(align_up((uintptr_t)ws, 256)); }

}  // namespace

// Launch prep + decode-GEMV for activation row `m_index` of X (X already
// prepped when `do_prep` is false).  Shared by wal_gemv, wal_gemm_small_m and
// the body-pass driver.
int launch_product_m1(const wal_matrix* m, const uint16_t* X, int M, int ldx, int m_index, float* y,
                      void* ws, size_t ws_bytes, cudaStream_t stream, bool do_prep) {
  const GemvPlan gp = plan_gemv(m->N, m->K, m->k);
  const WsLayout L = ws_layout(m->N, m->K, M, gp.S, gp.nRB);
  if (!ws) return fail(WAL_ERR_ARG, "workspace is NULL");
  if (ws_bytes < L.total) return fail(WAL_ERR_WORKSPACE, "workspace too small");
  char* base = ws_base(ws);
  const int G = m->K / kGroup, words = m->K / 16;
  if (do_prep) {
    PrepParams pp;
    pp.X = X; pp.ldx = ldx; pp.K = m->K; pp.G = G; pp.r = m->r; pp.M = M;
    pp.vbits = m->v_bits; pp.lr = m->lr_scale;
    pp.limbs = reinterpret_cast<uint32_t*>(base + L.limbs);
    pp.xsum = reinterpret_cast<int32_t*>(base + L.xsum);
    pp.gscale = reinterpret_cast<float*>(base + L.gscale);
    pp.z = reinterpret_cast<float*>(base + L.z);
    pp.counters = reinterpret_cast<uint32_t*>(base + L.counters);
    pp.n_counters = gp.nRB;
    pp.status = reinterpret_cast<int32_t*>(base + L.header);
    const size_t smem = (size_t)m->r * G * 4 + (size_t)G * 4;
    prep_x_kernel<<<M, 512, smem, stream>>>(pp);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e, "prep_x_kernel launch");
  }
  GemvParams p;
  p.codes = m->codes; p.sites = m->sites; p.scales = m->scales; p.ubits = m->u_bits;
  p.N = m->N; p.K = m->K; p.k = m->k; p.r = m->r; p.G = G; p.words = words;
  p.x = X + (size_t)m_index * ldx;
  p.limbs = reinterpret_cast<const uint32_t*>(base + L.limbs) + (size_t)m_index * words * kLimbWords;
  p.xsum = reinterpret_cast<const int32_t*>(base + L.xsum) + (size_t)m_index * words;
  p.gscale = reinterpret_cast<const float*>(base + L.gscale) + (size_t)m_index * G;
  p.z = reinterpret_cast<const float*>(base + L.z) + (size_t)m_index * 32;
  p.part = reinterpret_cast<float*>(base + L.part);
  p.counters = reinterpret_cast<uint32_t*>(base + L.counters);
  p.y = y;
  p.S = gp.S; p.RB = gp.RB; p.nRB = gp.nRB;
  const dim3 grid(gp.nRB, gp.S);
  switch (m->k) {
    case 0: gemv_kernel<0><<<grid, kThreads, gemv_smem_bytes(), stream>>>(p); break;
    case 2: gemv_kernel<2><<<grid, kThreads, gemv_smem_bytes(), stream>>>(p); break;
    case 4: gemv_kernel<4><<<grid, kThreads, gemv_smem_bytes(), stream>>>(p); break;
    default: gemv_kernel<8><<<grid, kThreads, gemv_smem_bytes(), stream>>>(p); break;
  }
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "gemv_kernel launch");
  return WAL_OK;
}

size_t product_ws_bytes(const wal_matrix* m, int M) {
  const GemvPlan gp = plan_gemv(m->N, m->K, m->k);
  return ws_layout(m->N, m->K, M, gp.S, gp.nRB).total;
}

int check_product_args(const wal_matrix* m, const void* X, int M, int ldx, const void* Y, int ldy) {
  int st = check_matrix(m);
  if (st) return st;
  if (!X || !Y) return fail(WAL_ERR_ARG, "activation and output pointers are required");
  if (!aligned16(X) || ((uintptr_t)Y & 3u)) return fail(WAL_ERR_ARG, "X must be 16-byte and Y 4-byte aligned");
  if (M < 1) return fail(WAL_ERR_SHAPE, "M must be >= 1");
  if (ldx < m->K || ldy < m->N || (ldx % 8))
    return fail(WAL_ERR_ARG, "ldx must be >= K and a multiple of 8; ldy must be >= N");
  return ensure_init();
}

}  // namespace wal

using namespace wal;

extern "C" size_t wal_workspace_bytes(const wal_matrix* m, int M) {
  if (check_matrix(m) != WAL_OK || M < 1) return 0;
  if (ensure_init() != WAL_OK) return 0;
  return product_ws_bytes(m, M);
}

extern "C" int wal_gemv(const wal_matrix* m, const uint16_t* x, float* y, void* ws, size_t ws_bytes,
                        wal_stream_t stream) {
  int st = check_product_args(m, x, 1, m ? m->K : 0, y, m ? m->N : 0);
  if (st) return st;
  return launch_product_m1(m, x, 1, m->K, 0, y, ws, ws_bytes, (cudaStream_t)stream, true);
}

extern "C" int wal_gemm_small_m(const wal_matrix* m, const uint16_t* X, int M, int ldx, float* Y, int ldy,
                                void* ws, size_t ws_bytes, wal_stream_t stream) {
  int st = check_product_args(m, X, M, ldx, Y, ldy);
  if (st) return st;
  for (int i = 0; i < M; ++i) {
    st = launch_product_m1(m, X, M, ldx, i, Y + (size_t)i * ldy, ws, ws_bytes, (cudaStream_t)stream, i == 0);
    if (st) return st;
  }
  return WAL_OK;
}

extern "C" int wal_unpack_matrix(const wal_matrix* m, int8_t* T, uint8_t* site_pos, int8_t* site_sign,
                                 uint16_t* alpha, uint16_t* beta, int8_t* U, int8_t* V, wal_stream_t stream) {
  int st = check_matrix(m);
  if (st) return st;
  st = ensure_init();
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
  st = ensure_init();
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
  if (h != 0) return fail(WAL_ERR_TIMEOUT, "a bounded device wait gave up");
  return WAL_OK;
}
