// Host side of libwal: layout-v1 sizes, the pack/layout converter and status text.
//
// The converter plays the role of the "prepare" step of the WAL runtimes
// (WAL-Ternary-8B card, "Install": the executable cache stores packed ternary
// symbols, sparse positions/signs and FP16 scales).  It writes the byte layout
// documented in include/wal.h and rejects every out-of-range input.
#include "wal_internal.h"

#include <cstring>
#include <string>

namespace wal {

thread_local std::string g_last_error;

int fail(int status, const std::string& msg) {
  g_last_error = msg;
  return status;
}

int check_shape(int N, int K, int k, int r) {
  if (N <= 0 || K <= 0 || K % kGroup != 0)
    return fail(WAL_ERR_SHAPE, "N must be > 0 and K a positive multiple of 128");
  if (k != 0 && k != 2 && k != 4 && k != 8) return fail(WAL_ERR_SHAPE, "k must be 0, 2, 4 or 8");
  if (r < 0 || r > WAL_MAX_RANK) return fail(WAL_ERR_SHAPE, "r must be in [0, 32]");
  if ((int64_t)N * K > (int64_t)1 << 40) return fail(WAL_ERR_SHAPE, "matrix too large");
  return WAL_OK;
}

// Every buffer is padded with zero bytes to a multiple of 16 so that the
// kernels may read any naturally aligned 4- or 16-byte word that overlaps it.
void sizes_of(int N, int K, int k, int r, size_t out[6]) {
  const size_t G = (size_t)K / kGroup;
  out[0] = align_up((size_t)N * K / 4, 16);
  out[1] = align_up((size_t)N * G * k, 16);
  out[2] = align_up((size_t)N * G * (k > 0 ? 4 : 2), 16);
  out[3] = align_up((size_t)N * ((r + 31) / 32) * 4, 16);
  out[4] = align_up((size_t)r * (K / 32) * 4, 16);
  out[5] = align_up((size_t)r * 2, 16);
}

}  // namespace wal

using namespace wal;

extern "C" int wal_packed_sizes(int N, int K, int k, int r, size_t out_bytes[6]) {
  if (!out_bytes) return fail(WAL_ERR_ARG, "out_bytes is NULL");
  int st = check_shape(N, K, k, r);
  if (st) return st;
  sizes_of(N, K, k, r, out_bytes);
  return WAL_OK;
}

extern "C" int wal_pack_matrix(const int8_t* T, const uint8_t* site_pos, const int8_t* site_sign,
                               const uint16_t* alpha, const uint16_t* beta, const int8_t* U,
                               const int8_t* V, const uint16_t* lr_scale, int N, int K, int k,
                               int r, void* const out[6]) {
  int st = check_shape(N, K, k, r);
  if (st) return st;
  if (!T || !alpha || !out) return fail(WAL_ERR_ARG, "T, alpha and out must be non-NULL");
  if (k > 0 && (!site_pos || !site_sign || !beta))
    return fail(WAL_ERR_ARG, "site_pos, site_sign and beta are required when k > 0");
  if (r > 0 && (!U || !V || !lr_scale)) return fail(WAL_ERR_ARG, "U, V and lr_scale are required when r > 0");
  size_t sz[6];
  sizes_of(N, K, k, r, sz);
  for (int i = 0; i < 6; ++i)
    if (sz[i] && !out[i]) return fail(WAL_ERR_ARG, "an output buffer is NULL");

  const int G = K / kGroup;
  const int words = K / 16;
  {
    // zero the padding tails
    const size_t used[6] = {(size_t)N * K / 4, (size_t)N * G * k, (size_t)N * G * (k > 0 ? 4 : 2),
                            (size_t)N * ((r + 31) / 32) * 4, (size_t)r * (K / 32) * 4, (size_t)r * 2};
    for (int i = 0; i < 6; ++i)
      if (sz[i] > used[i]) std::memset(static_cast<char*>(out[i]) + used[i], 0, sz[i] - used[i]);
  }
  uint32_t* codes = static_cast<uint32_t*>(out[0]);
  uint8_t* sites = static_cast<uint8_t*>(out[1]);
  uint16_t* scales = static_cast<uint16_t*>(out[2]);
  int bad_rows = 0;

#pragma omp parallel for schedule(static) reduction(+ : bad_rows)
  for (int n = 0; n < N; ++n) {
    int bad = 0;
    const int8_t* trow = T + (size_t)n * K;
    uint32_t* crow = codes + (size_t)n * words;
    for (int w = 0; w < words; ++w) {
      uint32_t word = 0;
      for (int i = 0; i < 16; ++i) {
        int t = trow[16 * w + i];
        bad |= (t < -1) | (t > 1);
        word |= (uint32_t)(t + 1) << (2 * i);
      }
      crow[w] = word;
    }
    for (int g = 0; g < G; ++g) {
      const size_t gi = (size_t)n * G + g;
      if (k > 0) {
        int prev = -1;
        for (int i = 0; i < k; ++i) {
          int p = site_pos[gi * k + i];
          int s = site_sign[gi * k + i];
          bad |= (p >= kGroup) | (p <= prev) | ((s != 1) & (s != -1));
          prev = p;
          sites[gi * k + i] = (uint8_t)(p | (s < 0 ? 0x80 : 0));
        }
        scales[2 * gi] = alpha[gi];
        scales[2 * gi + 1] = beta[gi];
      } else {
        scales[gi] = alpha[gi];
      }
    }
    bad_rows += bad;
  }
  if (bad_rows) return fail(WAL_ERR_FORMAT, "T outside {-1,0,1} or invalid residual sites");

  if (r > 0) {
    const int uw = (r + 31) / 32;
    uint32_t* ub = static_cast<uint32_t*>(out[3]);
    uint32_t* vb = static_cast<uint32_t*>(out[4]);
    int bad = 0;
    for (int n = 0; n < N; ++n) {
      for (int q = 0; q < uw; ++q) ub[(size_t)n * uw + q] = 0;
      for (int rho = 0; rho < r; ++rho) {
        int u = U[(size_t)n * r + rho];
        bad |= (u != 1) & (u != -1);
        if (u < 0) ub[(size_t)n * uw + rho / 32] |= 1u << (rho % 32);
      }
    }
    const int vw = K / 32;
    for (int rho = 0; rho < r; ++rho) {
      for (int q = 0; q < vw; ++q) {
        uint32_t word = 0;
        for (int b = 0; b < 32; ++b) {
          int v = V[(size_t)(32 * q + b) * r + rho];
          bad |= (v != 1) & (v != -1);
          if (v < 0) word |= 1u << b;
        }
        vb[(size_t)rho * vw + q] = word;
      }
    }
    std::memcpy(out[5], lr_scale, (size_t)r * 2);
    if (bad) return fail(WAL_ERR_FORMAT, "U or V entry outside {-1, +1}");
  }
  return WAL_OK;
}

extern "C" const char* wal_status_string(int status) {
  switch (status) {
    case WAL_OK: return "WAL_OK";
    case WAL_ERR_ARG: return "WAL_ERR_ARG";
    case WAL_ERR_SHAPE: return "WAL_ERR_SHAPE";
    case WAL_ERR_FORMAT: return "WAL_ERR_FORMAT";
    case WAL_ERR_WORKSPACE: return "WAL_ERR_WORKSPACE";
    case WAL_ERR_CUDA: return "WAL_ERR_CUDA";
    case WAL_ERR_UNSUPPORTED: return "WAL_ERR_UNSUPPORTED";
    case WAL_ERR_TIMEOUT: return "WAL_ERR_TIMEOUT";
    default: return "WAL_ERR_UNKNOWN";
  }
}

extern "C" const char* wal_last_error(void) { return g_last_error.c_str(); }
