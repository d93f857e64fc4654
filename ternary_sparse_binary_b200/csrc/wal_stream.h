// Work-list launch of the batch-1 decode-GEMV (see wal_stream.cu).
#pragma once

#include <cuda_runtime.h>

#include <cstdint>

namespace wal {

constexpr int kMaxItems = 16;
constexpr int kMaxPrefetch = 24;

// One product y = W x inside a launch.
struct StreamItem {
  const uint32_t* codes;
  const uint8_t* sites;
  const uint16_t* scales;
  const uint32_t* ubits;
  const uint32_t* vbits;
  const uint16_t* lr;
  const uint16_t* x;  // bf16 [K]
  float* y;           // fp32 [N]
  int N, k, r;
  int tile_begin;     // first tile of this product (filled by launch_stream)
};

// A byte range to warm in L2 (16-byte aligned start, size a multiple of 16).
struct PrefetchRange {
  const void* ptr;
  unsigned long long bytes;
};

struct StreamParams {
  StreamItem items[kMaxItems];
  PrefetchRange pf[kMaxPrefetch];
  int n_items, n_pf;
  int K, S, P, RB, rmax, stage_v;
  int32_t* status;  // workspace status word, cleared by the launch (may be NULL)
};

struct StreamLaunch {
  int S, P, RB, threads, tiles, rmax, stages;
  bool signed_table, stage_v;
  unsigned smem;
};

int stream_init();
int num_sms();
int plan_stream(const StreamItem* items, int n, int K, StreamLaunch* out);
int launch_stream(StreamParams& prm, const StreamLaunch& L, cudaStream_t stream, bool pdl);

}  // namespace wal
