// Internal declarations shared by the host and device translation units of libwal.
#pragma once

#include <cstddef>
#include <cstdint>
#include <string>

#include "../../include/wal.h"

namespace wal {

constexpr int kGroup = 128;        // weights per scale group
constexpr int kMaxK = 24576;       // largest K handled by this build
constexpr int kWordsPerLane = 8;   // one 128-group (8 code words) per lane in the decode-GEMV
constexpr int kSliceCols = 32 * kWordsPerLane * 16;  // 4096 columns per K-slice (one warp)
constexpr int kLimbWords = 12;     // 3 limbs x 4 slots of uint32 per 16-column code word

constexpr int kMaxDevices = 64;    // device ordinals with their own init state

int fail(int status, const std::string& msg);
// The current device's ordinal in *dev; WAL_ERR_CUDA or WAL_ERR_UNSUPPORTED (>= kMaxDevices) otherwise.
int current_device(int* dev);
int check_shape(int N, int K, int k, int r);
void sizes_of(int N, int K, int k, int r, size_t out[6]);

inline size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

// Scratch layout of one product call (offsets from the 256-byte aligned ws base).
struct WsLayout {
  size_t header;    // 256 B: [0] device status word
  size_t limbs;     // M * (K/16) * 12 uint32: fixed-point image of x, byte limbs per slot
  size_t xsum;      // M * (K/16) int32: sum of the fixed-point x over each 16-column word
  size_t gscale;    // M * G float: 2^(e_g - 21), the weight of one fixed-point unit in group g
  size_t z;         // M * 32 float: WALB2 phase-1 result s_r * V_r^T x
  size_t part;      // S * M * N float: split-K partial sums
  size_t counters;  // n_row_blocks uint32: split-K completion counters
  size_t total;
};

WsLayout ws_layout(int N, int K, int M, int n_slices, int n_row_blocks);

}  // namespace wal
