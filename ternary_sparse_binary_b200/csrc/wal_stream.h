// Work-list launch of the batch-1 decode-GEMV (see wal_stream.cu).
#pragma once

#include <cuda_runtime.h>

#include <cstdint>

namespace wal {

constexpr int kMaxItems = 16;

// Weight formats a launch can stream (one per launch):
//  kFmtV1  layout v1 of the direct-packed product (codes, sites, scales, WALB2);
//  kFmtPq2 PQ2_0 plain-ternary blocks (FP16 scale + 32 code bytes per 128
//          weights); `codes` then points at the block buffer, k = r = 0;
//  kFmtF32 layout v1 with FP32 scales: {alpha, beta} as two floats per
//          (row, group) (alpha alone when k = 0) and FP32 per-rank scales (a
//          prepared RC1 matrix); `scales` and `lr` then point at floats;
//  kFmtInt4 INT4/g128 (the LM head): `codes` points at the nibble plane
//          uint8 [N][K/2] (offset 8), `scales` at fp16 d [N][K/128], k = r = 0.
enum : int { kFmtV1 = 0, kFmtPq2 = 1, kFmtF32 = 2, kFmtInt4 = 3 };

// One product y = W x.
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
  int tile_begin;     // first tile of this product inside its group
};

// A group: up to 16 products that share K and run together, one tile of RB
// rows per CTA.  Groups of one dependency stage run back to back; between
// stages the CTAs meet at a grid barrier.
struct GroupDesc {
  int K, S, P, RB, rmax, tiles;
  int signed_table;  // +-X table (256 entries) or X table with the sign applied at lookup
  int xfree;         // the group's x is not written by the previous stage: its x image may be
                     // built while the grid barrier before it is still open
  int lane_parts;    // rows leave one partial per lane (summed in the combine) rather than a
                     // warp-reduced one; set where the 32x larger buffer fits shared memory
  int item0, n_items;
  int stage;         // dependency stage (non-decreasing along the group list)
};

enum : uint8_t { kTileSigned = 1, kTileXFree = 2, kTileLaneParts = 4 };

// What one CTA does in one group (16 bytes; a body pass keeps [CTA][group]
// of these in device memory and each CTA copies its row into shared memory).
struct TileRec {
  uint16_t item;   // index into the item table
  uint16_t rows;   // rows of the tile (0: the CTA has no tile in this group)
  int32_t n0;      // first output row of the tile
  uint8_t G, S, P, flags;  // K / 128, slices, phases, kTileSigned | kTileXFree | kTileLaneParts
  uint16_t RB;     // rows per tile of the group
  uint16_t stage;  // dependency stage
};

// Parameters of one launch: either one inline group (a single product call)
// or per-CTA schedules and an item table in device memory (a body pass).
struct StreamParams {
  StreamItem items[kMaxItems];
  GroupDesc group;
  const TileRec* t_sched;     // NULL: use the inline group; else [gridDim.x][n_groups]
  const StreamItem* t_items;
  int n_groups;
  int stages;                 // ring depth in chunks
  int rpc;                    // rows per ring chunk (2 or 3)
  uint32_t sched_off;         // shared-memory offset of the CTA's schedule
  uint32_t area_off;          // shared-memory offset of the per-group area
  unsigned int* barrier;      // grid-barrier counter (zeroed before the launch), body pass only
  unsigned int barrier_bias;  // added to every grid-barrier target (0; the fault-injection hook sets 2^30)
  unsigned long long wait_ns; // time limit of one grid-barrier wait (0: kGridWaitNs)
  int32_t* status;            // workspace status word (may be NULL)
  int fmt;                    // kFmtV1, kFmtPq2, kFmtF32 or kFmtInt4
};

struct StreamLaunch {
  int grid, threads, stages, rpc;
  unsigned smem;
  uint32_t sched_off, area_off;
};

// The schedule row of CTA `cta` for groups[0 .. n_groups) (items as planned).
void build_schedule(const GroupDesc* groups, int n_groups, const StreamItem* items, int cta, TileRec* out);

int stream_init();
int num_sms();
// Fill the geometry of group `g` (K, items) and return WAL_OK or an error.
int plan_group(StreamItem* items, int n, int K, GroupDesc* g);
// Shared memory and ring depth for a list of groups of format `fmt`.
int plan_launch(GroupDesc* groups, int n_groups, bool persistent, int fmt, StreamLaunch* out);
// Single group, items inline.
int launch_stream(StreamParams& prm, const StreamLaunch& L, cudaStream_t stream);
// Body pass: group and item tables already in device memory; cooperative launch.
int launch_body(StreamParams& prm, const StreamLaunch& L, cudaStream_t stream);

}  // namespace wal
