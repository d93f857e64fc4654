// Decode-GEMV for the direct-packed body-matrix product at batch 1
//   y = (alpha*T + beta*R) x + sum_r s_r U_r (V_r^T x)
// (WAL-Ternary-8B model card, "Representation").
//
// One launch runs a list of groups.  A group is up to kMaxItems products that
// share K; one CTA owns one tile of a group = RB consecutive output rows of
// one product and every K-slice of them, so nothing leaves the CTA before y
// is written.  A single product call is one group.  A body pass is one
// persistent, cooperative launch over all its groups, one CTA per SM: groups
// of one dependency stage follow each other directly, and between stages the
// CTAs meet at a grid barrier (stage s + 1 may read what stage s wrote).
//
// A lane owns one 128-group of a row (8 code words), a warp a K-slice of 4096
// columns; a group uses S slices x P phases warps.
//  - Weights stream through a per-warp TMA ring that runs ahead across group
//    and stage boundaries (the weights do not depend on x): lane 0 of each
//    warp keeps `stages` chunks of 2-3 rows in flight, one bulk copy each for
//    a row's code bytes (32 lanes x 32 B), residual-site bytes and
//    {alpha, beta} words, completing on an mbarrier per ring slot.  While a
//    CTA waits at the grid barrier its ring already fills with the next
//    stage's rows, and the x of its next tile is warmed in L2.
//  - Per group the CTA builds the fixed-point image of x: per 128-group g
//    with largest exponent e_g, X_j = round(x_j * 2^(21 - e_g)), an integer
//    below 2^22 in magnitude (exact when x_j is within 2^-14 of the group
//    maximum, round-to-nearest-even below that), as three byte limbs per
//    column, with the group sum of X, the group weight 2^(e_g - 21) and a
//    table of X (or X then -X) indexed by the residual-site byte,
//    group-major.  One pass over x and one CTA barrier.
//  - Each lane pulls its 96 limb words into registers.  The trit decode
//    masks each code word once per slot (word & (0x03030303 << 2s) leaves
//    4^s times the code t + 1 of trit 4b + s in byte b); three dp4a per slot
//    against the lo / mid / hi limbs accumulate per slot, and exact shifts
//    fold the slots, giving sum_j (t_j + 1) X_j; minus sum_j X_j that is T.x
//    of the group in int32.  The residual sites add +-X from the table
//    (exact).  alpha and beta are applied in FP32 and the group weight once.
//    The WALB2 phase-1 products V_r^T x go through the same path: a row of
//    V is a ternary row without zeros, its bits spread into 2-bit codes.
//  - Each lane stores its row partial to shared memory; after the rows one
//    thread per output row sums the row's 32 lane partials (the pairwise tree
//    of a xor-16 .. 1 butterfly) and the slices in order, and the WALB2
//    phase-2 term sum_r U[n, r] z_r joins in the single store.  Where the
//    lane buffer does not fit (very large row blocks), the row loop sums the
//    lanes with that butterfly itself; the bits are the same.
// Results are bitwise reproducible: no atomics in the arithmetic, fixed
// reduction orders.  Every wait (mbarrier, grid barrier) is bounded; one that
// gives up records WAL_ERR_TIMEOUT in the status word and the waiter moves on.
#include "wal_internal.h"
#include "wal_device.cuh"
#include "wal_ptx.cuh"
#include "wal_stream.h"

#include <algorithm>
#include <mutex>
#include <vector>

namespace wal {

using namespace dev;
using ptx::mbar_init;
using ptx::mbar_arrive_expect_tx;
using ptx::mbar_wait;
using ptx::bulk_g2s;

constexpr int kMaxRowsPerChunk = 3;  // rows per ring chunk: 3, or 2 where shared memory is short
constexpr int kMaxThreads = 384;
constexpr int kMaxWarps = kMaxThreads / 32;
constexpr int kMaxXChunks = 8;            // 8-column chunks of x per thread
constexpr uint32_t kMagic = 0x4B400000u;  // 1.5 * 2^23: adding it rounds |v| < 2^22 to an integer
constexpr uint32_t kLimbStride = 100;     // words per group in the limb image (96 + 4 pad)
constexpr unsigned long long kGridWaitNs = 2000000000ull;  // 2 s: far above any grid-barrier wait of a working pass
// One ring chunk of one warp: rpc rows of codes (32 lanes x 32 B each), then
// their site bytes (32 x 8 B each + 16 B alignment slack), then their
// {alpha, beta} words (32 x 4 B each + 16 B slack).  With a single K-slice
// (K <= 4096) the rows are contiguous in every buffer and arrive as one copy
// per buffer, packed at the buffers' own row pitch; otherwise each row is
// copied on its own at the fixed pitches below.
constexpr uint32_t kCodePitch = 1024, kSitePitch = 272, kScalePitch = 144, kScalePitch32 = 272;
// PQ2_0 rows (34-byte blocks: FP16 scale, then 32 code bytes) arrive as one
// byte range per chunk (one K-slice) or per row (several K-slices, at this
// pitch: 32 blocks plus the 16-byte widening at both ends).
constexpr uint32_t kPq2Block = 34, kPq2Pitch = 1152;
struct ChunkGeom {
  int rpc;                        // rows per chunk
  uint32_t sites, scales, bytes;  // offsets of the site and scale parts, chunk size
  uint32_t spitch;                // per-row pitch of the scale part (several K-slices)
};
// Code bytes of one 128-group: 2-bit codes, or 4-bit INT4 codes.
__host__ __device__ constexpr uint32_t code_group_bytes(int fmt) { return fmt == kFmtInt4 ? 64u : 32u; }
__host__ __device__ inline ChunkGeom chunk_geom(int rpc, int fmt) {
  ChunkGeom c;
  c.rpc = rpc;
  if (fmt == kFmtInt4) {  // codes (32 groups x 64 B per row), no sites, fp16 scales
    c.spitch = kScalePitch;
    c.sites = c.scales = (uint32_t)rpc * 32u * code_group_bytes(fmt);
    c.bytes = c.scales + (uint32_t)rpc * kScalePitch;
    return c;
  }
  if (fmt == kFmtPq2) {
    c.sites = c.scales = c.spitch = 0u;
    c.bytes = (uint32_t)rpc * kPq2Pitch;
    return c;
  }
  c.spitch = fmt == kFmtF32 ? kScalePitch32 : kScalePitch;  // 32 groups x (8 | 4) bytes + 16
  c.sites = (uint32_t)rpc * kCodePitch;
  c.scales = c.sites + (uint32_t)rpc * kSitePitch;
  c.bytes = c.scales + (uint32_t)rpc * c.spitch;
  return c;
}

__device__ __forceinline__ void prefetch_l2(const void* p, uint32_t bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(p), "r"(bytes) : "memory");
}
__device__ __forceinline__ void cp_async4_zfill(uint32_t dst, const void* src, uint32_t src_bytes) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;" ::"r"(dst), "l"(src), "r"(src_bytes) : "memory");
}
__device__ __forceinline__ uint4 lds128(uint32_t a) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(a));
  return v;
}
__device__ __forceinline__ uint32_t lds16(uint32_t a) {
  uint16_t v;
  asm volatile("ld.shared.u16 %0, [%1];" : "=h"(v) : "r"(a));
  return v;
}
__device__ __forceinline__ int32_t ldsi(uint32_t a) {
  int32_t v;
  asm volatile("ld.shared.s32 %0, [%1];" : "=r"(v) : "r"(a));
  return v;
}
// x may have been written by an earlier stage of the same launch: read it at
// L2 (coherent), never through the non-coherent or L1 path.
__device__ __forceinline__ uint4 ld_cg128(const void* p) {
  uint4 v;
  asm volatile("ld.global.cg.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "l"(p));
  return v;
}
__device__ __forceinline__ uint32_t ld_acquire(const unsigned int* p) {
  uint32_t v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ uint32_t byte_of(uint32_t w, int b) { return __byte_perm(w, 0u, 0x4440u | (uint32_t)b); }

// 16 bits -> the even bit positions of a 32-bit word.
__device__ __forceinline__ uint32_t spread16(uint32_t x) {
  x = (x | (x << 8)) & 0x00FF00FFu;
  x = (x | (x << 4)) & 0x0F0F0F0Fu;
  x = (x | (x << 2)) & 0x33333333u;
  x = (x | (x << 1)) & 0x55555555u;
  return x;
}

// Exact integer (T + 1).X over one lane's group (8 code words, 128 columns).
// Slot s of a word is masked in place, so its bytes carry 4^s times the code;
// the per-slot sums are multiples of 4^s and fold back by exact shifts.
__device__ __forceinline__ int32_t group_dot(const uint32_t (&wv)[8], const uint32_t (&lb)[8][kLimbWords]) {
  uint32_t a0[4] = {0u, 0u, 0u, 0u}, a1[4] = {0u, 0u, 0u, 0u};
  int32_t a2[4] = {0, 0, 0, 0};
#pragma unroll
  for (int w = 0; w < 8; ++w) {
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const uint32_t msk = wv[w] & (0x03030303u << (2 * q));
      a0[q] = dp4a_uu(msk, lb[w][0 * 4 + q], a0[q]);
      a1[q] = dp4a_uu(msk, lb[w][1 * 4 + q], a1[q]);
      a2[q] = dp4a_us(msk, lb[w][2 * 4 + q], a2[q]);
    }
  }
  const uint32_t t0 = a0[0] + (a0[1] >> 2) + (a0[2] >> 4) + (a0[3] >> 6);
  const uint32_t t1 = a1[0] + (a1[1] >> 2) + (a1[2] >> 4) + (a1[3] >> 6);
  const int32_t t2 = a2[0] + (a2[1] >> 2) + (a2[2] >> 4) + (a2[3] >> 6);
  return (int32_t)(((uint32_t)t2 << 16) + (t1 << 8) + t0);
}

// Exact integer sum_j u_j X_j over one lane's INT4 group (16 code words of
// eight 4-bit codes u = q + 8).  Word i of the group holds columns 8i..8i+7;
// its low nibbles (word & 0x0F0F0F0F) are the even columns and its high
// nibbles the odd ones, matched by limb slots 2h and 2h + 1 of 16-column
// word i / 2 (h = i % 2).  Both slots carry the code itself (no slot
// weight), so the three limb sums need no fold.  |X| < 2^20 keeps the true
// sum_j q_j X_j inside int32; the uint32 arithmetic wraps to it.
__device__ __forceinline__ uint32_t group_dot4(const uint32_t (&wv)[16], const uint32_t (&lb)[8][kLimbWords]) {
  uint32_t a0 = 0u, a1 = 0u;
  int32_t a2 = 0;
#pragma unroll
  for (int w = 0; w < 8; ++w) {
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const uint32_t word = wv[2 * w + h];
      const uint32_t lo = word & 0x0F0F0F0Fu, hi = (word >> 4) & 0x0F0F0F0Fu;
      a0 = dp4a_uu(lo, lb[w][0 * 4 + 2 * h], a0);
      a0 = dp4a_uu(hi, lb[w][0 * 4 + 2 * h + 1], a0);
      a1 = dp4a_uu(lo, lb[w][1 * 4 + 2 * h], a1);
      a1 = dp4a_uu(hi, lb[w][1 * 4 + 2 * h + 1], a1);
      a2 = dp4a_us(lo, lb[w][2 * 4 + 2 * h], a2);
      a2 = dp4a_us(hi, lb[w][2 * 4 + 2 * h + 1], a2);
    }
  }
  return a0 + (a1 << 8) + ((uint32_t)a2 << 16);
}

// ---------------------------------------------------------------------------
// shared memory: [ring | mbarriers | producer states] then the per-group area
// ---------------------------------------------------------------------------
// Site table: per group, the X of its 128 columns (and, in the signed
// table, their negations after them), group-major.  The row stride is a
// multiple of 4 words, so the build writes 16-byte vectors; the site bytes
// of a warp's lanes are random, so no stride spreads their banks better.
__host__ __device__ inline uint32_t table_stride(bool signed_table) { return signed_table ? 260u : 132u; }

__host__ __device__ inline uint32_t ring_bytes(int warps, int stages, int rpc, int fmt) {
  return (uint32_t)warps * stages * chunk_geom(rpc, fmt).bytes;
}
struct ProdState;  // defined below
__host__ __device__ inline uint32_t area_offset(int warps, int stages, int rpc, int fmt);

struct AreaPlan {
  uint32_t table, limbs, part, xgsum, gsc, partz, ubuf, vstage, lrs, total;
};
// Row pitch of the lane partials: RB rounded up to odd, so that the 32 lanes'
// stores of one row (stride pitch words) fall in 32 different banks.
// Partials of a tile: [slice][lane][pitch] with lane partials (a row's 32
// lanes are summed in the combine), else [slice][RB] (summed by a warp
// butterfly in the row loop).
__host__ __device__ inline uint32_t part_pitch(int RB) { return (uint32_t)RB | 1u; }
// Carve-up of the per-group area (offsets relative to the area base).  A
// PQ2_0 group has no site table and no WALB2 pair.
__host__ __device__ inline AreaPlan area_plan(int K, int S, int RB, bool signed_table, int fmt, bool lanes) {
  AreaPlan p;
  uint32_t off = 0;
  auto take = [&](uint32_t bytes) { uint32_t o = off; off = (off + bytes + 15u) & ~15u; return o; };
  const uint32_t G = (uint32_t)K / kGroup;
  const bool v1 = fmt == kFmtV1 || fmt == kFmtF32;
  p.table = take(v1 ? G * table_stride(signed_table) * 4u : 0u);
  p.limbs = take(G * kLimbStride * 4u);
  p.part = take((uint32_t)S * (lanes ? 32u * part_pitch(RB) : (uint32_t)RB) * 4u);
  p.xgsum = take(G * 4u);
  p.gsc = take(G * 4u);
  p.partz = take(v1 ? (uint32_t)S * WAL_MAX_RANK * 4u : 0u);
  p.ubuf = take(v1 ? (uint32_t)RB * 4u : 0u);
  // V bit planes of the first P ranks (each of the P phases of a slice takes one): P * K / 8 bytes
  p.vstage = take(v1 ? (uint32_t)(kMaxWarps / S) * (uint32_t)K / 8u : 0u);
  p.lrs = take(v1 ? WAL_MAX_RANK * 4u : 0u);  // the per-rank scales (FP16 or FP32)
  p.total = off;
  return p;
}

// Rows of one warp in one group: a contiguous block, row i of the warp is
// output row nb + i of one product (tile row r0 + i), columns of K-slice s.
struct WarpRing {
  const uint32_t* codes;
  const uint8_t* sites;
  const uint16_t* scales;
  int nmine;
  int s, nb, r0, G, K, k;
  __device__ __forceinline__ bool one_slice() const { return G <= 32; }
  __device__ __forceinline__ int ngroups() const { return min(32, G - 32 * s); }
};

// What warp `warp` does for tile record t of product `it` (nmine = 0: nothing).
// `it` is read only when this warp has rows.  The P warps of a slice take
// contiguous blocks of ceil(rows / P) rows.
__device__ __forceinline__ void warp_work(const TileRec& t, const StreamItem* it, int warp, WarpRing& W) {
  W.codes = nullptr; W.sites = nullptr; W.scales = nullptr;
  W.nmine = 0;
  W.s = W.r0 = 0;
  W.nb = t.n0;
  W.G = t.G; W.K = (int)t.G * kGroup; W.k = 0;
  if (t.rows == 0 || warp >= (int)t.S * t.P) return;
  W.s = warp % t.S;
  const int p = warp / t.S, m = ((int)t.rows + t.P - 1) / t.P;
  W.r0 = p * m;
  W.nb = t.n0 + W.r0;
  W.nmine = max(0, min(m, (int)t.rows - W.r0));
  // the producer skips the groups where this warp has no rows without a
  // round trip to memory
  if (W.nmine == 0) return;
  W.codes = it->codes; W.sites = it->sites; W.scales = it->scales; W.k = it->k;
}

// Host and device: the tile record of CTA `cta` in group g.
__host__ __device__ inline TileRec tile_record(const GroupDesc& g, const StreamItem* items, int cta) {
  TileRec t = {};
  t.G = (uint8_t)(g.K / kGroup); t.S = (uint8_t)g.S; t.P = (uint8_t)g.P;
  t.flags = (uint8_t)((g.signed_table ? kTileSigned : 0) | (g.xfree ? kTileXFree : 0) |
                      (g.lane_parts ? kTileLaneParts : 0));
  t.RB = (uint16_t)g.RB;
  t.stage = (uint16_t)g.stage;
  if (cta >= g.tiles) return t;
  int i = 0;
  while (i + 1 < g.n_items && cta >= items[i + 1].tile_begin) ++i;
  const int n0 = (cta - items[i].tile_begin) * g.RB;
  const int rows = items[i].N - n0 < g.RB ? items[i].N - n0 : g.RB;
  t.item = (uint16_t)(g.item0 + i);
  t.n0 = n0;
  t.rows = (uint16_t)rows;
  return t;
}

__device__ __forceinline__ uint32_t site_bytes(int k) { return (uint32_t)k; }
// bytes of one (row, group) in the scale plane: {alpha, beta} or alpha, FP16 or FP32
template <int FMT>
__device__ __forceinline__ uint32_t scale_bytes(int k) {
  return (k > 0 ? 4u : 2u) * (FMT == kFmtF32 ? 2u : 1u);
}

// Byte range of PQ2_0 blocks [b0, b0 + nb) widened to 16-byte boundaries
// (the block buffer is zero-padded to a multiple of 16 bytes, so the widened
// range stays inside it).
__device__ __forceinline__ void pq2_range(size_t b0, size_t nb, size_t& a, size_t& e) {
  a = (b0 * kPq2Block) & ~(size_t)15;
  e = ((b0 + nb) * kPq2Block + 15) & ~(size_t)15;
}

// Queue the rows of chunk `chunk` of W into ring slot `sl` with mbarrier
// `bar`.  Site and scale ranges are widened to 16-byte boundaries (every
// buffer is zero-padded to a multiple of 16 bytes, so the widened range stays
// inside).
template <int FMT>
__device__ __forceinline__ void issue_chunk(const WarpRing& W, uint32_t sl, uint32_t bar, int chunk,
                                            const ChunkGeom& C) {
  const int i0 = chunk * C.rpc;
  const int un = min(C.rpc, W.nmine - i0);
  if (un <= 0) return;
  if (FMT == kFmtPq2) {
    const unsigned char* bbase = reinterpret_cast<const unsigned char*>(W.codes);
    const size_t G = (size_t)W.G;
    size_t a, e;
    if (W.one_slice()) {  // the chunk's rows are one contiguous range
      pq2_range((size_t)(W.nb + i0) * G, (size_t)un * G, a, e);
      mbar_arrive_expect_tx(bar, (uint32_t)(e - a));
      bulk_g2s(sl, bbase + a, (uint32_t)(e - a), bar);
      return;
    }
    const size_t ng = (size_t)W.ngroups();
    uint32_t bytes = 0;
    for (int u = 0; u < un; ++u) {
      pq2_range((size_t)(W.nb + i0 + u) * G + 32 * (size_t)W.s, ng, a, e);
      bytes += (uint32_t)(e - a);
    }
    mbar_arrive_expect_tx(bar, bytes);
    for (int u = 0; u < un; ++u) {
      pq2_range((size_t)(W.nb + i0 + u) * G + 32 * (size_t)W.s, ng, a, e);
      bulk_g2s(sl + (uint32_t)u * kPq2Pitch, bbase + a, (uint32_t)(e - a), bar);
    }
    return;
  }
  const uint32_t kb = site_bytes(W.k), sb = scale_bytes<FMT>(W.k);
  const unsigned char* cbase = reinterpret_cast<const unsigned char*>(W.codes);
  const unsigned char* abase = reinterpret_cast<const unsigned char*>(W.scales);
  constexpr uint32_t cgb = code_group_bytes(FMT);  // code bytes per group
  if (W.one_slice()) {
    const size_t n = (size_t)(W.nb + i0), G = (size_t)W.G;
    const uint32_t clen = (uint32_t)un * (uint32_t)W.G * cgb;
    const size_t sa = (n * G * kb) & ~(size_t)15, se = ((n + un) * G * kb + 15) & ~(size_t)15;
    const size_t aa = (n * G * sb) & ~(size_t)15, ae = ((n + un) * G * sb + 15) & ~(size_t)15;
    mbar_arrive_expect_tx(bar, clen + (uint32_t)(se - sa) + (uint32_t)(ae - aa));
    bulk_g2s(sl, cbase + n * G * cgb, clen, bar);
    if (se > sa) bulk_g2s(sl + C.sites, W.sites + sa, (uint32_t)(se - sa), bar);
    bulk_g2s(sl + C.scales, abase + aa, (uint32_t)(ae - aa), bar);
    return;
  }
  // several K-slices: each row on its own (lengths first for the expected bytes)
  const int ng = W.ngroups();
  auto site_range = [&](size_t gb, size_t& a, size_t& e) {
    a = (gb * kb) & ~(size_t)15;
    e = ((gb + ng) * kb + 15) & ~(size_t)15;
  };
  auto scale_range = [&](size_t gb, size_t& a, size_t& e) {
    a = (gb * sb) & ~(size_t)15;
    e = ((gb + ng) * sb + 15) & ~(size_t)15;
  };
  uint32_t bytes = 0;
  for (int u = 0; u < un; ++u) {
    const size_t gb = (size_t)(W.nb + i0 + u) * W.G + 32 * W.s;
    size_t a, e, a2, e2;
    site_range(gb, a, e);
    scale_range(gb, a2, e2);
    bytes += (uint32_t)ng * cgb + (uint32_t)(e - a) + (uint32_t)(e2 - a2);
  }
  mbar_arrive_expect_tx(bar, bytes);
  for (int u = 0; u < un; ++u) {
    const size_t n = (size_t)(W.nb + i0 + u);
    const size_t gb = n * W.G + 32 * W.s;
    size_t a, e, a2, e2;
    site_range(gb, a, e);
    scale_range(gb, a2, e2);
    bulk_g2s(sl + (uint32_t)u * 32u * cgb, cbase + n * (size_t)W.G * cgb + (size_t)W.s * 32u * cgb, (uint32_t)ng * cgb,
             bar);
    if (e > a) bulk_g2s(sl + C.sites + (uint32_t)u * kSitePitch, W.sites + a, (uint32_t)(e - a), bar);
    bulk_g2s(sl + C.scales + (uint32_t)u * C.spitch, abase + a2, (uint32_t)(e2 - a2), bar);
  }
}

// The producer side of a warp's ring (kept in shared memory, used by lane 0):
// the next chunk to issue, which may lie in a later group.
struct ProdState {
  int j, c, nc;
  uint32_t issued;    // chunks issued so far
  uint32_t consumed;  // chunks consumed so far
  uint32_t slot;      // ring slot of the next chunk to issue (issued mod stages)
  WarpRing W;
};
__host__ __device__ inline uint32_t area_offset(int warps, int stages, int rpc, int fmt) {
  const uint32_t o = ring_bytes(warps, stages, rpc, fmt) + (uint32_t)warps * stages * 8u +
                     (uint32_t)warps * (uint32_t)((sizeof(ProdState) + 15) & ~(size_t)15);
  return (o + 127u) & ~127u;
}

// Move the producer to the first group at or after ps.j with rows for this warp.
__device__ __forceinline__ void prod_seek(ProdState& ps, const TileRec* sched, int n_groups, const StreamItem* items,
                                          int warp, int rpc) {
  while (ps.j < n_groups) {
    const TileRec t = sched[ps.j];
    if (t.rows && warp < (int)t.S * t.P) {
      warp_work(t, items + t.item, warp, ps.W);
      ps.nc = (ps.W.nmine + rpc - 1) / rpc;
      ps.c = 0;
      if (ps.nc > 0) return;
    }
    ++ps.j;
  }
}

// Keep up to `stages` chunks in flight: issue the producer's next chunks (in
// order, chunk n into slot n mod stages) while fewer are outstanding and, if
// j_limit >= 0, while they belong to groups up to j_limit.
template <int FMT>
__device__ __forceinline__ void prod_topup(ProdState& ps, uint32_t ring, uint32_t mbar, int stages,
                                           const TileRec* sched, int n_groups, const StreamItem* items, int warp,
                                           const ChunkGeom& C, int j_limit) {
  while (ps.j < n_groups && ps.issued - ps.consumed < (uint32_t)stages && (j_limit < 0 || ps.j <= j_limit)) {
    issue_chunk<FMT>(ps.W, ring + ps.slot * C.bytes, mbar + ps.slot * 8u, ps.c, C);
    ++ps.issued;
    if (++ps.slot == (uint32_t)stages) ps.slot = 0;
    if (++ps.c == ps.nc) {
      ++ps.j;
      prod_seek(ps, sched, n_groups, items, warp, C.rpc);
    }
  }
}

// tab = shared address of this lane's group in the site table
template <bool SIGNED_TABLE>
__device__ __forceinline__ int32_t site_at(uint32_t tab, uint32_t byte) {
  if (SIGNED_TABLE) return ldsi(tab + byte * 4u);
  const int32_t v = ldsi(tab + (byte & 0x7Fu) * 4u);
  return (byte & 0x80u) ? -v : v;
}

// One row's contribution of this lane's group: 2^(e_g - 21) * (alpha * T.X +
// beta * R.X).  crow, srow, arow: shared addresses of the row's codes, site
// bytes and scale words for lane 0 of the warp.  `hsw` swaps the two 16-byte
// halves of the lane's code chunk (matching the limb registers), so that the
// 32-byte-strided reads of a warp never share a bank.
template <int KS, bool SIGNED_TABLE, int FMT>
__device__ __forceinline__ float row_value(uint32_t crow, uint32_t srow, uint32_t arow, int lane, uint32_t hsw,
                                           const uint32_t (&lb)[8][kLimbWords], int32_t xs, float gsc,
                                           uint32_t tab) {
  if (FMT == kFmtInt4) {
    // the lane's 64 code bytes as four 16-byte reads starting at chunk
    // (lane / 2) % 4, so that the 8 lanes of each quarter-warp hit 8
    // different 16-byte bank groups; the limb image is rotated to match
    const uint32_t cd = crow + (uint32_t)lane * 64u, rot = ((uint32_t)lane >> 1) & 3u;
    uint32_t wv[16];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const uint4 c = lds128(cd + 16u * (((uint32_t)j + rot) & 3u));
      wv[4 * j] = c.x; wv[4 * j + 1] = c.y; wv[4 * j + 2] = c.z; wv[4 * j + 3] = c.w;
    }
    const int32_t tdot = (int32_t)(group_dot4(wv, lb) - 8u * (uint32_t)xs);
    return fp16_bits_to_float(lds16(arow + (uint32_t)lane * 2u)) * ((float)tdot * gsc);
  }
  const uint32_t cd = crow + (uint32_t)lane * 32u;
  const uint4 c0 = lds128(cd + hsw), c1 = lds128(cd + (hsw ^ 16u));
  const uint32_t wv[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
  const int32_t tdot = group_dot(wv, lb) - xs;
  int32_t q = 0;
  if (KS == 8) {
    const uint2 sw = ptx::lds64(srow + (uint32_t)lane * 8u);
    q = site_at<SIGNED_TABLE>(tab, byte_of(sw.x, 0)) + site_at<SIGNED_TABLE>(tab, byte_of(sw.x, 1)) +
        site_at<SIGNED_TABLE>(tab, byte_of(sw.x, 2));
    q += site_at<SIGNED_TABLE>(tab, byte_of(sw.x, 3)) + site_at<SIGNED_TABLE>(tab, byte_of(sw.y, 0)) +
         site_at<SIGNED_TABLE>(tab, byte_of(sw.y, 1));
    q += site_at<SIGNED_TABLE>(tab, byte_of(sw.y, 2)) + site_at<SIGNED_TABLE>(tab, byte_of(sw.y, 3));
  } else if (KS == 4) {
    const uint32_t sw = ptx::lds32(srow + (uint32_t)lane * 4u);
    q = site_at<SIGNED_TABLE>(tab, byte_of(sw, 0)) + site_at<SIGNED_TABLE>(tab, byte_of(sw, 1)) +
        site_at<SIGNED_TABLE>(tab, byte_of(sw, 2)) + site_at<SIGNED_TABLE>(tab, byte_of(sw, 3));
  } else if (KS == 2) {
    const uint32_t sw = lds16(srow + (uint32_t)lane * 2u);
    q = site_at<SIGNED_TABLE>(tab, sw & 0xFFu) + site_at<SIGNED_TABLE>(tab, sw >> 8);
  }
  if (FMT == kFmtF32) {  // FP32 scales
    if (KS == 0) return __uint_as_float(ptx::lds32(arow + (uint32_t)lane * 4u)) * ((float)tdot * gsc);
    const uint2 sc = ptx::lds64(arow + (uint32_t)lane * 8u);
    return fmaf(__uint_as_float(sc.x), (float)tdot, __uint_as_float(sc.y) * (float)q) * gsc;
  }
  if (KS == 0) {
    const float alpha = fp16_bits_to_float(lds16(arow + (uint32_t)lane * 2u));
    return alpha * ((float)tdot * gsc);
  }
  const uint32_t sc = ptx::lds32(arow + (uint32_t)lane * 4u);
  const float alpha = fp16_bits_to_float(sc & 0xFFFFu), beta = fp16_bits_to_float(sc >> 16);
  return fmaf(alpha, (float)tdot, beta * (float)q) * gsc;
}

// One PQ2_0 row's contribution of this lane's block at shared address A
// (2-byte aligned): d * T.x over the block's 128 columns.  The block is read
// as nine aligned words from A rounded down to 4 bytes; each code word is
// then a byte permute of two neighbours (bytes 2..5 when A is 4-byte
// aligned, bytes 4..7 when it is not), and d is the block's first two bytes.
__device__ __forceinline__ float pq2_row_value(uint32_t A, const uint32_t (&lb)[8][kLimbWords], int32_t xs,
                                               float gsc) {
  const uint32_t B = A & ~3u;
  uint32_t w[9];
#pragma unroll
  for (int i = 0; i < 9; ++i) w[i] = ptx::lds32(B + 4u * (uint32_t)i);
  const bool odd = (A & 2u) != 0u;
  const uint32_t sel = odd ? 0x7654u : 0x5432u;
  uint32_t wv[8];
#pragma unroll
  for (int q = 0; q < 8; ++q) wv[q] = __byte_perm(w[q], w[q + 1], sel);
  const uint32_t dbits = __byte_perm(w[0], 0u, odd ? 0x4432u : 0x4410u);
  const int32_t tdot = group_dot(wv, lb) - xs;
  return fp16_bits_to_float(dbits) * ((float)tdot * gsc);
}

// Everything a warp needs to walk its ring.
struct RingCtx {
  uint32_t ring, mbar;  // this warp's ring slots and mbarriers (shared window)
  int stages;
  ProdState* ps;        // this warp's producer state
  const TileRec* sched; // this CTA's schedule (shared memory)
  const StreamItem* items;
  int n_groups, warp;
  ChunkGeom C;          // ring chunk geometry
  bool items_global;    // items live in device memory (not kernel parameters)
  int32_t* status;
  unsigned int* barrier;  // grid-barrier counter (body pass)
  unsigned long long wait_ns;  // limit of one grid-barrier wait
};

// Consume this warp's rows of the current group (ring positions q, q+1, ...);
// after each chunk lane 0 refills the slot with the producer's next chunk.
// False when a wait gave up.
// A row's value leaves the row loop as this lane's partial (summed in the
// combine, no dependent chain in the loop) or, where the lane buffer does not
// fit, as the warp's butterfly sum stored by lane 0.  Both give the same bits.
__device__ __forceinline__ void store_row(float* dst, float v, bool lanes, int lane) {
  if (lanes) {
    *dst = v;
  } else {
    v = warp_sum(v);
    if (lane == 0) *dst = v;
  }
}

template <int KS, bool SIGNED_TABLE, int FMT>
__device__ __forceinline__ bool run_rows(const WarpRing& W, const RingCtx& R, uint32_t& st, uint32_t& parity, int RB,
                                         int lane, bool active, uint32_t hsw, const uint32_t (&lb)[8][kLimbWords],
                                         int32_t xs, float gsc, uint32_t tab, float* part, bool lanes) {
  const ChunkGeom& C = R.C;
  const int nc = (W.nmine + C.rpc - 1) / C.rpc;
  // row i of this warp: lane partials at mine[i], or the warp's sum at mine[i] (lane 0)
  float* mine = lanes ? part + (uint32_t)(W.s * 32 + lane) * part_pitch(RB) + W.r0 : part + W.s * RB + W.r0;
  const uint32_t kb = site_bytes(KS), sb = scale_bytes<FMT>(KS);
  const bool one = W.one_slice();
  const uint32_t G = (uint32_t)W.G;
  // one slice: pitches of the packed rows; otherwise the fixed pitches
  constexpr uint32_t cgb = code_group_bytes(FMT);
  const uint32_t cp = one ? G * cgb : 32u * cgb, sp = one ? G * kb : kSitePitch, ap = one ? G * sb : C.spitch;
#pragma unroll 1
  for (int j = 0; j < nc; ++j) {
    const uint32_t sl = R.ring + st * C.bytes;
    if (!mbar_wait(R.mbar + st * 8u, parity, R.status)) return false;
    // group index of the chunk's first row (this slice's first group)
    const uint32_t gb0 = (uint32_t)(W.nb + j * C.rpc) * G + 32u * (uint32_t)W.s;
    // rows one at a time (not unrolled): the loop body stays small enough for
    // the instruction caches, which measured faster than three unrolled rows
#pragma unroll 1
    for (int u = 0; u < kMaxRowsPerChunk; ++u) {
      const int i = j * C.rpc + u;
      if (u < C.rpc && i < W.nmine) {  // uniform across the warp
        const uint32_t gb = one ? gb0 : gb0 + (uint32_t)u * G;
        const uint32_t srow = sl + C.sites + (uint32_t)u * sp + ((gb * kb) & 15u);
        const uint32_t arow = sl + C.scales + (uint32_t)u * ap + ((gb * sb) & 15u);
        const float v =
            row_value<KS, SIGNED_TABLE, FMT>(sl + (uint32_t)u * cp, srow, arow, lane, hsw, lb, xs, gsc, tab);
        store_row(mine + i, active ? v : 0.f, lanes, lane);
      }
    }
    __syncwarp();  // every lane has consumed the slot before it is refilled
    if (lane == 0) {
      ++R.ps->consumed;
      prod_topup<FMT>(*R.ps, R.ring, R.mbar, R.stages, R.sched, R.n_groups, R.items, R.warp, C, -1);
    }
    if (++st == (uint32_t)R.stages) {
      st = 0;
      parity ^= 1u;
    }
  }
  return true;
}

// run_rows for PQ2_0 rows: lane l takes block l of the warp's K-slice.
__device__ __forceinline__ bool run_rows_pq2(const WarpRing& W, const RingCtx& R, uint32_t& st, uint32_t& parity,
                                             int RB, int lane, bool active, const uint32_t (&lb)[8][kLimbWords],
                                             int32_t xs, float gsc, float* part, bool lanes) {
  const ChunkGeom& C = R.C;
  const int nc = (W.nmine + C.rpc - 1) / C.rpc;
  float* mine = lanes ? part + (uint32_t)(W.s * 32 + lane) * part_pitch(RB) + W.r0 : part + W.s * RB + W.r0;
  const bool one = W.one_slice();
  const uint32_t G = (uint32_t)W.G, rowb = G * kPq2Block;
#pragma unroll 1
  for (int j = 0; j < nc; ++j) {
    const uint32_t sl = R.ring + st * C.bytes;
    if (!mbar_wait(R.mbar + st * 8u, parity, R.status)) return false;
#pragma unroll 1
    for (int u = 0; u < kMaxRowsPerChunk; ++u) {
      const int i = j * C.rpc + u;
      if (u < C.rpc && i < W.nmine) {  // uniform across the warp
        // where the widened copy put the row (only the low 4 bits of the byte offset matter)
        const uint32_t row = one ? sl + (((uint32_t)(W.nb + j * C.rpc) * rowb) & 15u) + (uint32_t)u * rowb
                                 : sl + (uint32_t)u * kPq2Pitch +
                                       ((((uint32_t)(W.nb + i) * G + 32u * (uint32_t)W.s) * kPq2Block) & 15u);
        const float v = pq2_row_value(row + kPq2Block * (uint32_t)lane, lb, xs, gsc);
        store_row(mine + i, active ? v : 0.f, lanes, lane);
      }
    }
    __syncwarp();
    if (lane == 0) {
      ++R.ps->consumed;
      prod_topup<kFmtPq2>(*R.ps, R.ring, R.mbar, R.stages, R.sched, R.n_groups, R.items, R.warp, C, -1);
    }
    if (++st == (uint32_t)R.stages) {
      st = 0;
      parity ^= 1u;
    }
  }
  return true;
}

// This thread's 8-column chunks of x (chunk tid + i * blockDim.x).
__device__ __forceinline__ void load_x(const uint16_t* x, int K, uint4 (&xr)[kMaxXChunks]) {
  const int n8 = K / 8;
#pragma unroll
  for (int i = 0; i < kMaxXChunks; ++i) {
    const int c8 = (int)threadIdx.x + i * (int)blockDim.x;
    xr[i] = c8 < n8 ? ld_cg128(reinterpret_cast<const uint4*>(x) + c8) : make_uint4(0u, 0u, 0u, 0u);
  }
}

// Layout v1 (and its FP32-scale form): the site table and the half-swapped
// limb image below.  PQ2_0: no site table, and the image keeps every group in
// natural word order (its code words are read one by one).  INT4: no site
// table, X scaled to 20 bits (X = round(x * 2^(19 - e_g))), the limb slots of
// each 16-column word are (8-column half, even / odd column), and a group's
// words are stored rotated by 2 * ((g / 2) % 4) to match its lane's reads.
template <bool SIGNED_TABLE, int FMT>
__device__ __forceinline__ void build_image(const uint4 (&xr)[kMaxXChunks], int K, unsigned char* area,
                                            const AreaPlan& ap) {
  constexpr bool NO_TABLE = FMT == kFmtPq2 || FMT == kFmtInt4, INT4 = FMT == kFmtInt4;
  constexpr uint32_t kOff = INT4 ? 19u : 21u;  // X = round(x * 2^(kOff - e_g))
  const int threads = blockDim.x, tid = threadIdx.x, lane = tid & 31;
  const uint32_t tstride = table_stride(SIGNED_TABLE);
  int32_t* table = reinterpret_cast<int32_t*>(area + ap.table);
  uint32_t* limbs = reinterpret_cast<uint32_t*>(area + ap.limbs);
  int32_t* xgsum = reinterpret_cast<int32_t*>(area + ap.xgsum);
  float* gsc_s = reinterpret_cast<float*>(area + ap.gsc);
  const int n8 = K / 8;
#pragma unroll
  for (int i = 0; i < kMaxXChunks; ++i) {
    // chunk c8 = tid + i * threads, as loaded; the 16 chunks of one group sit
    // on 16 aligned lanes of one warp, so the test below is uniform across
    // each half-warp and its shuffles stay complete
    const int c8 = tid + i * threads;
    if (c8 >= n8) continue;
    const unsigned gmask = (lane & 16) ? 0xFFFF0000u : 0x0000FFFFu;
    const int c = 8 * c8;
    const uint4 raw = xr[i];
    const uint32_t pr[4] = {raw.x, raw.y, raw.z, raw.w};
    uint32_t m2 = 0u;  // largest |x| bit pattern, two bf16 lanes
#pragma unroll
    for (int q = 0; q < 4; ++q) m2 = __vmaxu2(m2, pr[q] & 0x7FFF7FFFu);
    uint32_t mx = __reduce_max_sync(gmask, max(m2 & 0xFFFFu, m2 >> 16));
    uint32_t emax = mx >> 7;
    emax = emax > 1u ? emax : 1u;  // exponent field of the group maximum (denormals as 1)
    // X = round(x * 2^(127 + kOff - emax)); tiny groups are pre-scaled by 2^64 so the factor stays finite
    const float pre = emax < 64u ? 18446744073709551616.0f : 1.0f;
    const float scl = __uint_as_float((254u + kOff - emax - (emax < 64u ? 64u : 0u)) << 23);
    int32_t X[8];
    int32_t sum8 = 0;
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      const float xv = bf16_bits_to_float((pr[q >> 1] >> (16 * (q & 1))) & 0xFFFFu);
      X[q] = (int32_t)(__float_as_uint(fmaf(xv * pre, scl, __uint_as_float(kMagic))) - kMagic);
      sum8 += X[q];
    }
    sum8 = __reduce_add_sync(gmask, sum8);
    const int gg = c >> 7, pos = c & 127, h = (c >> 3) & 1;
    // limb image [group][word-in-group][limb][slot] (+4 words of padding per
    // group): byte b of (word wl, limb L, slot q) = limb L of column 16 wl + 4 b + q.
    // A group read by a lane with bit 2 set is stored with its halves swapped
    // (words 0-3 <-> 4-7), the order in which that lane holds its limbs, so
    // that every lane reads its image front to back without bank conflicts.
    if (INT4) {
      // byte b of (word wl, limb L, slot 2h + p) = limb L of column 16 wl + 8h + 2b + p
      const int wl = (((c >> 4) & 7) - 2 * ((gg >> 1) & 3)) & 7;
      uint32_t* img32 = limbs + (size_t)gg * kLimbStride;
#pragma unroll
      for (int L2 = 0; L2 < 3; ++L2)
#pragma unroll
        for (int p = 0; p < 2; ++p) {
          const uint32_t sel = (uint32_t)(L2 | ((4 + L2) << 4));
          const uint32_t b01 = __byte_perm((uint32_t)X[p], (uint32_t)X[2 + p], sel);
          const uint32_t b23 = __byte_perm((uint32_t)X[4 + p], (uint32_t)X[6 + p], sel);
          img32[(wl * 3 + L2) * 4 + 2 * h + p] = __byte_perm(b01, b23, 0x5410u);
        }
    } else {
      const int wl = ((c >> 4) & 7) ^ ((!NO_TABLE && (gg & 4)) ? 4 : 0);
      uint16_t* img16 = reinterpret_cast<uint16_t*>(limbs + (size_t)gg * kLimbStride);
#pragma unroll
      for (int L2 = 0; L2 < 3; ++L2)
#pragma unroll
        for (int q = 0; q < 4; ++q)
          img16[((wl * 3 + L2) * 4 + q) * 2 + h] =
              (uint16_t)__byte_perm((uint32_t)X[q], (uint32_t)X[4 + q], (uint32_t)(L2 | ((4 + L2) << 4)));
    }
    if ((c8 & 15) == 0) {
      xgsum[gg] = sum8;
      // 2^(emax - 127 - kOff), a subnormal float for the smallest exponents
      gsc_s[gg] = emax > kOff ? __uint_as_float((emax - kOff) << 23) : __uint_as_float(1u << (emax + 22u - kOff));
    }
    // site table: entry e of group gg (e = site byte) at gg * stride + e
    if (!NO_TABLE) {  // rows of the table are 16-byte aligned (stride a multiple of 4 words)
      int4* trow = reinterpret_cast<int4*>(table + (size_t)gg * tstride + pos);
      trow[0] = make_int4(X[0], X[1], X[2], X[3]);
      trow[1] = make_int4(X[4], X[5], X[6], X[7]);
      if (SIGNED_TABLE) {
        trow[32] = make_int4(-X[0], -X[1], -X[2], -X[3]);
        trow[33] = make_int4(-X[4], -X[5], -X[6], -X[7]);
      }
    }
  }
  __syncthreads();
}

// Sum of the 32 lane partials of one row (lane l at p[l * pitch]) as the
// pairwise tree of a xor-16, 8, 4, 2, 1 butterfly, so that a row's value is
// the same as a warp butterfly would give lane 0.
__device__ __forceinline__ float lane_sum(const float* p, uint32_t pitch) {
  float v[32];
#pragma unroll
  for (int l = 0; l < 32; ++l) v[l] = p[(uint32_t)l * pitch];
#pragma unroll
  for (int w = 16; w; w >>= 1)
#pragma unroll
    for (int l = 0; l < w; ++l) v[l] += v[l + w];
  return v[0];
}

__device__ __forceinline__ void prefetch_l1(const void* p) {
  asm volatile("prefetch.global.L1 [%0];" ::"l"(p));
}

// One group on this CTA (which owns the tile t of it).  Returns false (on
// every thread) when some wait of the CTA gave up.
// All CTAs of the launch meet at a grid barrier, in two halves.  Arrive:
// thread 0 adds one with release semantics (the CTA barrier before it carries
// the CTA's writes).  Wait: thread 0 polls with acquire loads until `target`
// = CTAs x barriers so far, and the CTA barrier after it hands the acquired
// view to every thread.  Between the halves a CTA may do work that reads
// nothing the other CTAs write before the barrier.  A CTA always waits before
// it arrives at the next barrier.
__device__ __forceinline__ void grid_arrive(unsigned int* ctr) {
  __syncthreads();
  if (threadIdx.x == 0) asm volatile("red.release.gpu.global.add.u32 [%0], 1;" ::"l"(ctr) : "memory");
}
// The wait is bounded in time (%globaltimer); false on every thread of the CTA
// when it ran out (WAL_ERR_TIMEOUT recorded).
__device__ __forceinline__ bool grid_wait(unsigned int* ctr, unsigned int target, int32_t* status,
                                          unsigned long long limit_ns) {
  int timed_out = 0;
  if (threadIdx.x == 0) {
    const unsigned long long t0 = ptx::global_ns();
    while (ld_acquire(ctr) < target)
      if (ptx::global_ns() - t0 > limit_ns) {
        if (status) atomicExch(status, (int32_t)WAL_ERR_TIMEOUT);
        timed_out = 1;
        break;
      }
  }
  return !__syncthreads_or(timed_out);
}


// wait_target != 0: the grid barrier before this group is still open (this
// CTA has arrived); the x image and the WALB2 phase-1 products are built
// first, and the barrier is waited for before the rows.
template <int FMT, bool SIGNED_TABLE>
__device__ __forceinline__ bool do_group(const TileRec& t, const RingCtx& R, int j, uint32_t& st, uint32_t& parity,
                                         unsigned char* area, float* s_z, unsigned int wait_target) {
  const int threads = blockDim.x, tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int K = (int)t.G * kGroup, S = t.S, P = t.P, RB = t.RB, rows = t.rows, n0 = t.n0;
  const StreamItem& it = R.items[t.item];
  WarpRing W;
  warp_work(t, &it, warp, W);
  constexpr bool PQ2 = FMT == kFmtPq2;
  constexpr bool PLAIN = PQ2 || FMT == kFmtInt4;  // no residual sites, no WALB2 pair
  const int r = PLAIN ? 0 : it.r, ks = PLAIN ? 0 : it.k;
  const bool worker = warp < S * P;
  const bool lanes = (t.flags & kTileLaneParts) != 0;
  const AreaPlan ap = area_plan(K, S, RB, SIGNED_TABLE, FMT, lanes);
  float* partz = reinterpret_cast<float*>(area + ap.partz);
  float* part = reinterpret_cast<float*>(area + ap.part);
  uint32_t* ubuf = reinterpret_cast<uint32_t*>(area + ap.ubuf);

  // x first (it may be the previous stage's output), then the U words of the
  // tile's rows and the V bit planes of the first P ranks
  uint4 xr[kMaxXChunks];
  load_x(it.x, K, xr);
  const int rv = min(r, P);  // ranks staged in shared memory
  if (r > 0) {
    for (int rl = tid; rl < rows; rl += threads)
      cp_async4_zfill(ptx::smem_u32(ubuf + rl), it.ubits + (size_t)(n0 + rl) * ((r + 31) / 32), 4u);
    for (int i = tid; i < rv * (K / 128); i += threads)
      cp_async16(reinterpret_cast<void*>(area + ap.vstage + 16u * i), it.vbits + 4 * i);
    // per-rank scales for the combine (the buffer is padded to 16 bytes)
    if (tid < (r * (FMT == kFmtF32 ? 4 : 2) + 15) / 16)
      cp_async16(reinterpret_cast<void*>(area + ap.lrs + 16u * tid), reinterpret_cast<const char*>(it.lr) + 16 * tid);
  }
  cp_async_commit();

  // the item records of the next groups into L1 (the producer reads them when it moves on)
  if (R.items_global && tid < 4 && j + 1 + tid < R.n_groups) {
    const TileRec tn = R.sched[j + 1 + tid];
    if (tn.rows) prefetch_l1(R.items + tn.item);
  }
  build_image<SIGNED_TABLE, FMT>(xr, K, area, ap);

  // the 96 limb words of this lane's group into registers; on lanes with bit
  // 2 set register word w holds group word w ^ 4 (stored so in the image), as
  // their code reads do
  const int col0 = W.s * kSliceCols + lane * kGroup;
  const bool active = worker && col0 < K;
  const int g = active ? col0 >> 7 : 0;
  const uint32_t hsw = (lane & 4) ? 16u : 0u;
  uint32_t lb[8][kLimbWords];
  int32_t xs = 0;
  float gsc = 0.f;
  if (active) {
    const uint32_t img = ptx::smem_u32(area + ap.limbs) + (uint32_t)g * kLimbStride * 4u;
#pragma unroll
    for (int w = 0; w < 8; ++w) {
#pragma unroll
      for (int L2 = 0; L2 < 3; ++L2) {
        const uint4 v = lds128(img + (uint32_t)(w * 3 + L2) * 16u);
        lb[w][L2 * 4 + 0] = v.x; lb[w][L2 * 4 + 1] = v.y; lb[w][L2 * 4 + 2] = v.z; lb[w][L2 * 4 + 3] = v.w;
      }
    }
    xs = reinterpret_cast<const int32_t*>(area + ap.xgsum)[g];
    gsc = reinterpret_cast<const float*>(area + ap.gsc)[g];
  } else {
#pragma unroll
    for (int w = 0; w < 8; ++w)
#pragma unroll
      for (int qq = 0; qq < kLimbWords; ++qq) lb[w][qq] = 0u;
  }

  cp_async_wait<0>();
  __syncthreads();  // staged U / V complete
  // WALB2 phase 1: rows of V (no zeros: bit set -> code 0, clear -> code 2)
  if (worker)
    for (int rho = warp / S; rho < r; rho += P) {
      float val = 0.f;
      if (active) {
        const uint4 vb = rho < rv ? *reinterpret_cast<const uint4*>(area + ap.vstage + (size_t)rho * (K / 8) + (size_t)g * 16)
                                  : __ldg(reinterpret_cast<const uint4*>(it.vbits + (size_t)rho * (K / 32) + (size_t)g * 4));
        const uint32_t vw[4] = {vb.x, vb.y, vb.z, vb.w};
        uint32_t wv[8];
#pragma unroll
        for (int w = 0; w < 8; ++w) {
          const int wsw = hsw ? (w ^ 4) : w;  // limb registers are in swapped order on these lanes
          wv[w] = spread16(~(vw[wsw >> 1] >> (16 * (wsw & 1))) & 0xFFFFu) << 1;
        }
        val = (float)(group_dot(wv, lb) - xs) * gsc;
      }
      val = warp_sum(val);
      if (lane == 0) partz[W.s * WAL_MAX_RANK + rho] = val;
    }
  // the rows run only after the grid barrier before them (if it is still open) has passed
  const bool passed = !wait_target || grid_wait(R.barrier, wait_target, R.status, R.wait_ns);
  const uint32_t tab = ptx::smem_u32(area + ap.table) + (uint32_t)g * table_stride(SIGNED_TABLE) * 4u;
  bool ok = passed;
  if (!passed) {
  } else if (PQ2) {
    if (worker) ok = run_rows_pq2(W, R, st, parity, RB, lane, active, lb, xs, gsc, part, lanes);
  } else if (worker) {
    switch (ks) {
      case 8: ok = run_rows<8, SIGNED_TABLE, FMT>(W, R, st, parity, RB, lane, active, hsw, lb, xs, gsc, tab, part, lanes); break;
      case 4: ok = run_rows<4, SIGNED_TABLE, FMT>(W, R, st, parity, RB, lane, active, hsw, lb, xs, gsc, tab, part, lanes); break;
      case 2: ok = run_rows<2, SIGNED_TABLE, FMT>(W, R, st, parity, RB, lane, active, hsw, lb, xs, gsc, tab, part, lanes); break;
      default: ok = run_rows<0, SIGNED_TABLE, FMT>(W, R, st, parity, RB, lane, active, hsw, lb, xs, gsc, tab, part, lanes); break;
    }
  }

  // keep this warp's ring full (a warp with no rows here has issued nothing since the first fill)
  if (lane == 0) prod_topup<FMT>(*R.ps, R.ring, R.mbar, R.stages, R.sched, R.n_groups, R.items, R.warp, R.C, -1);
  // the last warp (fewest rows) warms L2 with the x of the CTA's next tile
  if (warp == (int)(blockDim.x / 32) - 1 && lane == 0)
    for (int jn = j + 1; jn < R.n_groups; ++jn) {
      const TileRec tn = R.sched[jn];
      if (tn.rows) {
        prefetch_l2(R.items[tn.item].x, (uint32_t)tn.G * kGroup * 2u);
        break;
      }
    }
  const bool all_ok = !__syncthreads_or(!ok);
  // a group whose wait gave up stores nothing (all_ok is the same on every thread)
  if (!all_ok) return false;

  // slices in order, WALB2 phase 2, one store per output
  if (tid < r) {
    float a = 0.f;
    for (int s2 = 0; s2 < S; ++s2) a += partz[s2 * WAL_MAX_RANK + tid];
    const float s = FMT == kFmtF32 ? reinterpret_cast<const float*>(area + ap.lrs)[tid]
                                   : fp16_bits_to_float(reinterpret_cast<const uint16_t*>(area + ap.lrs)[tid]);
    s_z[tid] = s * a;
  }
  __syncthreads();
  const uint32_t pp = part_pitch(RB);
  for (int rl = tid; rl < rows; rl += threads) {
    float acc = 0.f;
    for (int s2 = 0; s2 < S; ++s2) acc += lanes ? lane_sum(part + (uint32_t)s2 * 32u * pp + rl, pp) : part[s2 * RB + rl];
    if (r > 0) {
      const uint32_t uw = ubuf[rl];
      float lr = 0.f;
      for (int rho = 0; rho < r; ++rho) lr += ((uw >> rho) & 1u) ? -s_z[rho] : s_z[rho];
      acc += lr;
    }
    it.y[n0 + rl] = acc;
  }
  __syncthreads();  // the area is rebuilt by the next group
  return all_ok;
}


template <int FMT>
__global__ void __launch_bounds__(kMaxThreads, 1) stream_kernel(const __grid_constant__ StreamParams prm) {
  extern __shared__ __align__(128) unsigned char smem[];
  __shared__ float s_z[WAL_MAX_RANK];
  const bool table_mode = prm.t_sched != nullptr;
  const StreamItem* items = table_mode ? prm.t_items : prm.items;
  const int n_groups = table_mode ? prm.n_groups : 1;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, warps = (int)blockDim.x / 32;
  const int stages = prm.stages;
  if (!table_mode && blockIdx.x == 0 && tid == 0 && prm.status) *prm.status = 0;  // no timeout seen yet

  // this CTA's schedule into shared memory
  TileRec* sched = reinterpret_cast<TileRec*>(smem + prm.sched_off);
  if (table_mode) {
    const TileRec* src = prm.t_sched + (size_t)blockIdx.x * n_groups;
    for (int jj = tid; jj < n_groups; jj += blockDim.x) sched[jj] = src[jj];
  } else if (tid == 0) {
    sched[0] = tile_record(prm.group, prm.items, blockIdx.x);
  }
  __syncthreads();

  RingCtx R;
  const uint32_t base = ptx::smem_u32(smem);
  R.C = chunk_geom(prm.rpc, FMT);
  R.ring = base + (uint32_t)warp * stages * R.C.bytes;
  R.mbar = base + ring_bytes(warps, stages, prm.rpc, FMT) + (uint32_t)warp * stages * 8u;
  R.ps = reinterpret_cast<ProdState*>(smem + ring_bytes(warps, stages, prm.rpc, FMT) + (uint32_t)warps * stages * 8u +
                                      (uint32_t)warp * (uint32_t)((sizeof(ProdState) + 15) & ~(size_t)15));
  R.stages = stages;
  R.sched = sched;
  R.items = items;
  R.n_groups = n_groups;
  R.warp = warp;
  R.items_global = table_mode;
  R.status = prm.status;
  R.barrier = prm.barrier;
  R.wait_ns = prm.wait_ns ? prm.wait_ns : kGridWaitNs;
  if (lane == 0) {
    for (int st = 0; st < stages; ++st) mbar_init(R.mbar + 8u * st, 1u);
    ptx::mbar_init_fence();
    R.ps->j = 0;
    R.ps->issued = 0;
    R.ps->consumed = 0;
    R.ps->slot = 0;
    prod_seek(*R.ps, sched, n_groups, items, warp, R.C.rpc);
    // the first fill stays inside the CTA's first group with rows; the
    // run-ahead into later groups starts once that group is under way
    int j0 = 0;
    while (j0 + 1 < n_groups && sched[j0].rows == 0) ++j0;
    prod_topup<FMT>(*R.ps, R.ring, R.mbar, stages, sched, n_groups, items, warp, R.C, j0);
  }
  __syncwarp();

  unsigned char* area = smem + prm.area_off;
  uint32_t st = 0, parity = 0;  // this warp's ring slot and its phase parity
  unsigned int nbar = 0;
  bool dead = false;
  for (int j = 0; j < n_groups; ++j) {
    const TileRec t = sched[j];
    // a CTA whose wait gave up takes no further part: it neither arrives nor
    // waits (the CTAs that wait for it give up in turn, each after one limit)
    if (dead) break;
    unsigned int pending = 0;  // target of a grid barrier this CTA has arrived at but not passed
    if (j > 0 && t.stage != sched[j - 1].stage) {
      ++nbar;
      grid_arrive(prm.barrier);
      pending = nbar * gridDim.x + prm.barrier_bias;
      // the x image may be built before the barrier only when the previous
      // stage does not write this group's x (decided on the host)
      if (t.rows == 0 || !(t.flags & kTileXFree)) {
        dead = !grid_wait(prm.barrier, pending, prm.status, R.wait_ns);
        pending = 0;
      }
    }
    if (t.rows == 0 || dead) continue;  // uniform across the CTA
    bool ok;
    if (FMT == kFmtPq2 || FMT == kFmtInt4) ok = do_group<FMT, false>(t, R, j, st, parity, area, s_z, pending);
    else ok = (t.flags & kTileSigned) ? do_group<FMT, true>(t, R, j, st, parity, area, s_z, pending)
                                      : do_group<FMT, false>(t, R, j, st, parity, area, s_z, pending);
    dead = !ok;
  }
  // never leave with bulk copies in flight: after a wait gave up, wait for
  // every chunk this warp issued but did not consume (they sit in consecutive
  // slots from the current one).  Each is a copy of in-bounds global memory
  // into this CTA's ring, so its mbarrier phase completes by itself; the wait
  // is bounded all the same and goes on to the next chunk either way.
  if (lane == 0 && dead)
    for (uint32_t k = R.ps->consumed; k < R.ps->issued; ++k) {
      ptx::mbar_drain(R.mbar + st * 8u, parity, prm.status);
      if (++st == (uint32_t)stages) {
        st = 0;
        parity ^= 1u;
      }
    }
}

// ----------------------------------------------------------------------------
// host side
// ----------------------------------------------------------------------------
namespace {
// per device: SM count, shared-memory opt-in limit, and the kernels' attribute set once
struct StreamDev {
  std::once_flag once;
  cudaError_t err = cudaSuccess;
  int sms = 0, max_smem = 0;
};
StreamDev g_dev[kMaxDevices];

const StreamDev* dev_state() {
  int dev = 0;
  return current_device(&dev) == WAL_OK ? &g_dev[dev] : nullptr;
}
}  // namespace

int stream_init() {
  int dev = 0;
  int st = current_device(&dev);
  if (st) return st;
  StreamDev& d = g_dev[dev];
  std::call_once(d.once, [&d, dev] {
    cudaError_t e = cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&d.max_smem, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
    const int lim = d.max_smem - 1024;
    if (e == cudaSuccess) e = cudaFuncSetAttribute(stream_kernel<kFmtV1>, cudaFuncAttributeMaxDynamicSharedMemorySize, lim);
    if (e == cudaSuccess) e = cudaFuncSetAttribute(stream_kernel<kFmtPq2>, cudaFuncAttributeMaxDynamicSharedMemorySize, lim);
    if (e == cudaSuccess) e = cudaFuncSetAttribute(stream_kernel<kFmtF32>, cudaFuncAttributeMaxDynamicSharedMemorySize, lim);
    if (e == cudaSuccess) e = cudaFuncSetAttribute(stream_kernel<kFmtInt4>, cudaFuncAttributeMaxDynamicSharedMemorySize, lim);
    d.err = e;
  });
  if (d.err != cudaSuccess) return fail(WAL_ERR_CUDA, std::string("device initialisation: ") + cudaGetErrorString(d.err));
  return WAL_OK;
}

int num_sms() {
  const StreamDev* d = dev_state();
  return d && d->sms > 0 ? d->sms : 148;
}

int plan_group(StreamItem* items, int n, int K, GroupDesc* out) {
  if (n < 1 || n > kMaxItems) return fail(WAL_ERR_ARG, "a group takes 1..16 products");
  GroupDesc g = {};
  g.K = K;
  g.S = (K + kSliceCols - 1) / kSliceCols;
  if (g.S > kMaxWarps) return fail(WAL_ERR_UNSUPPORTED, "K above 49152 is not handled by this build");
  g.P = std::max(1, kMaxWarps / g.S);
  const int threads = 32 * g.S * g.P;
  if (K / 8 > kMaxXChunks * threads) return fail(WAL_ERR_UNSUPPORTED, "K too large for the x-chunk registers");
  int rmax = 0;
  for (int i = 0; i < n; ++i) rmax = std::max(rmax, items[i].r);
  g.rmax = rmax;
  // smallest row block that keeps the group in one wave
  const int sms = num_sms();
  int total_rows = 0;
  for (int i = 0; i < n; ++i) total_rows += items[i].N;
  int RB = std::max(1, (total_rows + sms - 1) / sms);
  for (;; ++RB) {
    int tiles = 0;
    for (int i = 0; i < n; ++i) tiles += (items[i].N + RB - 1) / RB;
    if (tiles <= sms) break;
  }
  if (RB > 65535) return fail(WAL_ERR_UNSUPPORTED, "row block above 65535 rows");
  g.RB = RB;
  int t = 0;
  for (int i = 0; i < n; ++i) {
    items[i].tile_begin = t;
    t += (items[i].N + RB - 1) / RB;
  }
  g.tiles = t;
  g.n_items = n;
  g.signed_table = 1;
  g.xfree = 0;
  g.lane_parts = 1;
  *out = g;
  return WAL_OK;
}

int plan_launch(GroupDesc* groups, int n_groups, bool persistent, int fmt, StreamLaunch* out) {
  StreamLaunch L = {};
  int warps = 0;
  for (int j = 0; j < n_groups; ++j) warps = std::max(warps, groups[j].S * groups[j].P);
  if (persistent) warps = kMaxWarps;
  L.threads = 32 * warps;
  const StreamDev* dv = dev_state();
  const uint32_t limit = (uint32_t)(dv && dv->max_smem > 0 ? dv->max_smem : 232448) - 1024u;
  const uint32_t sched_bytes = (uint32_t)align_up((size_t)n_groups * sizeof(TileRec), 128);
  // deepest ring first (rows in flight per warp), fewer copies on a tie
  static const int kRing[6][2] = {{3, 4}, {3, 3}, {2, 4}, {3, 2}, {2, 3}, {2, 2}};
  for (const auto& rs : kRing) {
    const int rpc = rs[0], stages = rs[1];
    const uint32_t soff = area_offset(warps, stages, rpc, fmt);
    const uint32_t off = soff + sched_bytes;
    uint32_t need = off;
    bool fits = true;
    // per group, the first area that fits: lane partials before the signed
    // table (the lane partials take the dependent reduction out of every row)
    std::vector<int> pick((size_t)n_groups, 0);
    for (int j = 0; j < n_groups && fits; ++j) {
      const GroupDesc& g = groups[j];
      const bool v1 = fmt == kFmtV1 || fmt == kFmtF32;
      int chosen = -1;
      for (int c = 0; c < 4 && chosen < 0; ++c) {  // c: bit 1 = warp sums, bit 0 = unsigned table
        if (v1 || !(c & 1)) {
          const uint32_t a = area_plan(g.K, g.S, g.RB, v1 && !(c & 1), fmt, !(c & 2)).total;
          if (off + a <= limit) {
            chosen = c;
            need = std::max(need, off + a);
          }
        }
      }
      if (chosen < 0) fits = false;
      else pick[j] = chosen;
    }
    if (!fits) continue;
    for (int j = 0; j < n_groups; ++j) {
      groups[j].signed_table = (fmt == kFmtV1 || fmt == kFmtF32) && !(pick[j] & 1) ? 1 : 0;
      groups[j].lane_parts = !(pick[j] & 2);
    }
    L.stages = stages;
    L.rpc = rpc;
    L.sched_off = soff;
    L.area_off = off;
    L.smem = need;
    int tiles = 0;
    for (int j = 0; j < n_groups; ++j) tiles = std::max(tiles, groups[j].tiles);
    L.grid = persistent ? num_sms() : tiles;
    *out = L;
    return WAL_OK;
  }
  return fail(WAL_ERR_UNSUPPORTED, "K too large for the shared-memory plan");
}

void build_schedule(const GroupDesc* groups, int n_groups, const StreamItem* items, int cta, TileRec* out) {
  for (int j = 0; j < n_groups; ++j) out[j] = tile_record(groups[j], items + groups[j].item0, cta);
}

static int launch(StreamParams& prm, const StreamLaunch& L, cudaStream_t stream, bool cooperative) {
  prm.stages = L.stages;
  prm.rpc = L.rpc;
  prm.sched_off = L.sched_off;
  prm.area_off = L.area_off;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(L.grid);
  cfg.blockDim = dim3(L.threads);
  cfg.dynamicSmemBytes = L.smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = cooperative ? 1 : 0;
  const cudaError_t e = prm.fmt == kFmtPq2    ? cudaLaunchKernelEx(&cfg, stream_kernel<kFmtPq2>, prm)
                        : prm.fmt == kFmtF32  ? cudaLaunchKernelEx(&cfg, stream_kernel<kFmtF32>, prm)
                        : prm.fmt == kFmtInt4 ? cudaLaunchKernelEx(&cfg, stream_kernel<kFmtInt4>, prm)
                                              : cudaLaunchKernelEx(&cfg, stream_kernel<kFmtV1>, prm);
  if (e != cudaSuccess) return fail(WAL_ERR_CUDA, std::string("stream_kernel launch: ") + cudaGetErrorString(e));
  return WAL_OK;
}

int launch_stream(StreamParams& prm, const StreamLaunch& L, cudaStream_t stream) {
  prm.t_sched = nullptr;
  prm.t_items = nullptr;
  prm.n_groups = 1;
  prm.barrier = nullptr;
  return launch(prm, L, stream, false);
}

int launch_body(StreamParams& prm, const StreamLaunch& L, cudaStream_t stream) {
  if (!prm.t_sched || !prm.t_items || !prm.barrier) return fail(WAL_ERR_ARG, "body launch without tables");
  int per_sm = 0;
  const void* fn = prm.fmt == kFmtPq2    ? reinterpret_cast<const void*>(stream_kernel<kFmtPq2>)
                   : prm.fmt == kFmtF32  ? reinterpret_cast<const void*>(stream_kernel<kFmtF32>)
                   : prm.fmt == kFmtInt4 ? reinterpret_cast<const void*>(stream_kernel<kFmtInt4>)
                                         : reinterpret_cast<const void*>(stream_kernel<kFmtV1>);
  cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, fn, L.threads, L.smem);
  if (e != cudaSuccess) return fail(WAL_ERR_CUDA, std::string("occupancy query: ") + cudaGetErrorString(e));
  if (per_sm < 1 || L.grid > per_sm * num_sms())
    return fail(WAL_ERR_UNSUPPORTED, "the persistent launch does not fit on the device at once");
  return launch(prm, L, stream, true);
}

}  // namespace wal
