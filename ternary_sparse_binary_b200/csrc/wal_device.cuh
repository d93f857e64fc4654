// Device-side building blocks shared by every libwal kernel: the layout-v1
// decode routines and small PTX wrappers.  The test entry point
// wal_unpack_matrix decodes with exactly these routines.
#pragma once

#include <cstdint>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

namespace wal {
namespace dev {

// ---- layout-v1 decode ------------------------------------------------------
// A 32-bit code word holds 16 trits; trit i sits at bits 2i..2i+1 with code
// c = t + 1.  Slot s (0..3) gathers trits {s, 4+s, 8+s, 12+s}: masking the
// word shifted right by 2s leaves, in byte b, the code of trit 4b + s.  Those
// bytes are fed straight to byte-wise integer dot products.
__device__ __forceinline__ uint32_t slot_codes(uint32_t word, int s) {
  return (word >> (2 * s)) & 0x03030303u;
}
__device__ __forceinline__ int code_to_trit(uint32_t code) { return (int)code - 1; }
// Residual site byte: position in its group (bits 0..6), sign bit 7 (set = -1).
__device__ __forceinline__ uint32_t site_position(uint32_t b) { return b & 0x7Fu; }
__device__ __forceinline__ bool site_negative(uint32_t b) { return (b & 0x80u) != 0; }

__device__ __forceinline__ float bf16_bits_to_float(uint32_t b) { return __uint_as_float(b << 16); }
__device__ __forceinline__ float fp16_bits_to_float(uint32_t b) {
  return __half2float(__ushort_as_half((unsigned short)b));
}

// ---- integer dot products --------------------------------------------------
__device__ __forceinline__ uint32_t dp4a_uu(uint32_t a, uint32_t b, uint32_t c) {
  uint32_t d;
  asm("dp4a.u32.u32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}
__device__ __forceinline__ int32_t dp4a_us(uint32_t a, uint32_t b, int32_t c) {
  int32_t d;
  asm("dp4a.u32.s32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}

// ---- per-thread asynchronous copies (global -> shared) -----------------------
__device__ __forceinline__ uint32_t smem_addr(const void* p) {
  return (uint32_t)__cvta_generic_to_shared(p);
}
__device__ __forceinline__ void cp_async16(void* dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_addr(dst)), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async4(void* dst, const void* src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(smem_addr(dst)), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int off = 16; off; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
  return v;
}

}  // namespace dev
}  // namespace wal
