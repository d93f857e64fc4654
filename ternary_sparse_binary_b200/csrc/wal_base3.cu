// The base-3 container and its conversion to layout v1 on the GPU.
//
// The WAL2-Ternary-27B card (section on bit widths) stores the ternary base
// five trits to a byte (8 / 5 = 1.6 bits per symbol) with a BF16 scale per
// 128 weights.  Inference runs on a prepared compute layout (the RC1 card's
// prepared cache keeps the codes packed and expands the scales to the
// kernels' format); wal_base3_convert is that step for layout v1: each trit
// becomes its 2-bit code c = t + 1 and each BF16 scale becomes FP16 alpha.
//
// Byte m of a row holds trits 5m .. 5m + 4 as sum_i (t_i + 1) 3^i; rows start
// on a byte (ceil(K / 5) bytes each); digits past a row's end are 0.
//
// One thread converts a block of 80 trits = 16 input bytes = 5 output code
// words: the 16 bytes come in as five aligned 32-bit loads and a funnel
// shift, each byte is looked up in a 256-entry table of its five 2-bit codes
// (bit 15 marks bytes above 242), and the 10-bit pieces are concatenated at
// fixed offsets.  Scales are converted by the same launch, one per thread.
#include "wal_internal.h"

#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <cstring>

namespace wal {
namespace {

constexpr uint32_t kBadByte = 1u, kBadTail = 2u, kBadScale = 4u;

__device__ __forceinline__ uint32_t ld_nc32(const uint8_t* p) {
  uint32_t v;
  asm volatile("ld.global.nc.u32 %0, [%1];" : "=r"(v) : "l"(p));
  return v;
}

__global__ void __launch_bounds__(256) base3_convert_kernel(const uint8_t* __restrict__ b3,
                                                             const uint16_t* __restrict__ s, int N, int K,
                                                             uint32_t* __restrict__ codes,
                                                             uint16_t* __restrict__ alpha, size_t in_bytes,
                                                             uint32_t* flags) {
  __shared__ uint16_t lut[256];
  for (int v = threadIdx.x; v < 256; v += blockDim.x) {
    uint32_t e = 0u, u = (uint32_t)v;
    for (int i = 0; i < 5; ++i) {
      e |= (u % 3u) << (2 * i);
      u /= 3u;
    }
    lut[v] = (uint16_t)(v > 242 ? 0x8000u : e);
  }
  __syncthreads();

  const int P = (K + 4) / 5;  // bytes per row
  const int Q = (K + 79) / 80;  // 80-trit blocks per row
  const int W = K / 16;       // code words per row
  const int r5 = K % 5;       // trits in a row's last byte (0: five)
  uint32_t f = 0u;
  const size_t nblk = (size_t)N * Q;
  const size_t stride = (size_t)gridDim.x * blockDim.x;
  for (size_t t = (size_t)blockIdx.x * blockDim.x + threadIdx.x; t < nblk; t += stride) {
    const int n = (int)(t / Q), q = (int)(t % Q);
    const size_t start = (size_t)n * P + 16u * (size_t)q;
    uint32_t by[4];
    const size_t a = start & ~(size_t)3;
    if (a + 20 <= in_bytes) {
      uint32_t w[5];
#pragma unroll
      for (int i = 0; i < 5; ++i) w[i] = ld_nc32(b3 + a + 4 * i);
      const uint32_t sh = 8u * (uint32_t)(start & 3);
#pragma unroll
      for (int i = 0; i < 4; ++i) by[i] = __funnelshift_r(w[i], w[i + 1], sh);
    } else {  // the last blocks of the buffer: byte loads inside it
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        uint32_t v = 0u;
        for (int j = 0; j < 4; ++j) {
          const size_t o = start + 4 * i + j;
          if (o < in_bytes) v |= (uint32_t)b3[o] << (8 * j);
        }
        by[i] = v;
      }
    }
    const int row_bytes = min(16, P - 16 * q);  // bytes of this block that belong to row n
    uint32_t out[5];
    uint64_t acc = 0u;
#pragma unroll
    for (int b = 0; b < 16; ++b) {
      const uint32_t v = (by[b >> 2] >> (8 * (b & 3))) & 0xFFu;
      const uint32_t e = lut[v];
      if (b < row_bytes) {
        f |= (e >> 15) * kBadByte;
        if (r5 && 16 * q + b == P - 1 && ((e & 0x3FFu) >> (2 * r5))) f |= kBadTail;
      }
      // bits 10 b .. 10 b + 9 of the block's 160-bit code string
      acc |= (uint64_t)(e & 0x3FFu) << ((10 * b) % 32);
      if ((10 * b) % 32 + 10 >= 32) {  // a word is complete (compile-time test)
        out[(10 * b) / 32] = (uint32_t)acc;
        acc >>= 32;
      }
    }
    uint32_t* dst = codes + (size_t)n * W + 5 * (size_t)q;
#pragma unroll
    for (int i = 0; i < 5; ++i)
      if (5 * q + i < W) dst[i] = out[i];
  }

  // scales: BF16 -> FP16, round to nearest even; the plane's padding is zeroed
  const size_t ns = (size_t)N * (K / kGroup);
  for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < ns; i += stride) {
    const uint32_t bits = s[i];
    const float x = __uint_as_float(bits << 16);
    const __half h = __float2half_rn(x);
    if (((bits >> 7) & 0xFFu) == 0xFFu || __hisinf(h)) f |= kBadScale;
    alpha[i] = __half_as_ushort(h);
  }
  if (blockIdx.x == 0 && threadIdx.x < 8) {
    const size_t pad = (ns + 7) & ~(size_t)7;  // fp16 entries up to the 16-byte boundary
    if (ns + threadIdx.x < pad) alpha[ns + threadIdx.x] = 0;
  }
  if (f) atomicOr(flags, f);
}

}  // namespace
}  // namespace wal

using namespace wal;

extern "C" size_t wal_base3_bytes(int N, int K) {
  if (N <= 0 || K <= 0 || K % kGroup || (int64_t)N * K > (int64_t)1 << 40) return 0;
  return align_up((size_t)N * ((K + 4) / 5), 16);
}

extern "C" int wal_base3_pack(const int8_t* T, int N, int K, void* out) {
  const size_t total = wal_base3_bytes(N, K);
  if (!total) return fail(WAL_ERR_SHAPE, "N must be > 0 and K a positive multiple of 128");
  if (!T || !out) return fail(WAL_ERR_ARG, "T and out must be non-NULL");
  const int P = (K + 4) / 5;
  uint8_t* o = static_cast<uint8_t*>(out);
  std::memset(o + (size_t)N * P, 0, total - (size_t)N * P);
  int bad_rows = 0;
#pragma omp parallel for schedule(static) reduction(+ : bad_rows)
  for (int n = 0; n < N; ++n) {
    int bad = 0;
    const int8_t* t = T + (size_t)n * K;
    for (int m = 0; m < P; ++m) {
      uint32_t v = 0, w = 1;
      for (int i = 0; i < 5; ++i, w *= 3) {
        const int j = 5 * m + i;
        if (j >= K) break;  // digits past the row's end stay 0
        bad |= (t[j] < -1) | (t[j] > 1);
        v += (uint32_t)(t[j] + 1) * w;
      }
      o[(size_t)n * P + m] = (uint8_t)v;
    }
    bad_rows += bad;
  }
  if (bad_rows) return fail(WAL_ERR_FORMAT, "T outside {-1,0,1}");
  return WAL_OK;
}

extern "C" int wal_base3_convert(const uint8_t* b3, const uint16_t* scales_bf16, int N, int K, uint32_t* codes,
                                 uint16_t* alpha, void* ws, size_t ws_bytes, wal_stream_t stream) {
  const size_t in_bytes = wal_base3_bytes(N, K);
  if (!in_bytes) return fail(WAL_ERR_SHAPE, "N must be > 0 and K a positive multiple of 128");
  if (!b3 || !scales_bf16 || !codes || !alpha) return fail(WAL_ERR_ARG, "every buffer is required");
  if (((uintptr_t)b3 | (uintptr_t)scales_bf16 | (uintptr_t)codes | (uintptr_t)alpha) & 15u)
    return fail(WAL_ERR_ARG, "buffers must be 16-byte aligned");
  if (!ws || ws_bytes < 512) return fail(WAL_ERR_WORKSPACE, "the conversion needs a 512-byte workspace");
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return fail(WAL_ERR_CUDA, "no CUDA device");
  uint32_t* flags = reinterpret_cast<uint32_t*>(align_up((uintptr_t)ws, 256)) + 1;
  cudaStream_t st = (cudaStream_t)stream;
  cudaError_t e = cudaMemsetAsync(flags, 0, 4, st);
  if (e != cudaSuccess) return fail(WAL_ERR_CUDA, std::string("flag clear: ") + cudaGetErrorString(e));
  base3_convert_kernel<<<sms * 8, 256, 0, st>>>(b3, scales_bf16, N, K, codes, alpha, in_bytes, flags);
  e = cudaGetLastError();
  if (e != cudaSuccess) return fail(WAL_ERR_CUDA, std::string("base3_convert_kernel launch: ") + cudaGetErrorString(e));
  uint32_t h = 0;
  e = cudaMemcpyAsync(&h, flags, 4, cudaMemcpyDeviceToHost, st);
  if (e == cudaSuccess) e = cudaStreamSynchronize(st);
  if (e != cudaSuccess) return fail(WAL_ERR_CUDA, std::string("conversion readback: ") + cudaGetErrorString(e));
  if (h & kBadByte) return fail(WAL_ERR_FORMAT, "base-3 byte above 242");
  if (h & kBadTail) return fail(WAL_ERR_FORMAT, "nonzero digit past the end of a row");
  if (h & kBadScale) return fail(WAL_ERR_FORMAT, "scale not finite or beyond FP16");
  return WAL_OK;
}
