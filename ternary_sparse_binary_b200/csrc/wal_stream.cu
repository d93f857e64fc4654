// Decode-GEMV for the direct-packed body-matrix product at batch 1
//   y = (alpha*T + beta*R) x + sum_r s_r U_r (V_r^T x)
// (WAL-Ternary-8B model card, "Representation").
//
// One launch processes a work list of up to kMaxItems products that share K
// (for example the q, k and v matrices of one dependency stage).  One CTA owns
// one tile = RB consecutive output rows of one product and every K-slice of
// them, so nothing leaves the CTA before y is written.
//
// A lane owns one 128-group of a row (8 code words), a warp a K-slice of 4096
// columns; the CTA has S slices x P phases warps.
//  1. x first: every thread requests its chunks of x (after the dependent-
//     launch wait, since x may be the previous stage's output).  Then lane 0
//     of each warp starts the warp's TMA ring: per row of the warp, one bulk
//     copy of the slice's code bytes (32 lanes x 32 B), one of its residual-
//     site bytes and one of its {alpha, beta} words, completing on an
//     mbarrier per ring stage (two rows).  The WALB2 bit planes (V) and bit
//     words (U) of the tile follow by cp.async.
//  2. The CTA builds the fixed-point image of x: per group g with largest
//     exponent e_g, X_j = round(x_j * 2^(21 - e_g)), an integer below 2^22 in
//     magnitude (exact when x_j is within 2^-14 of the group maximum, round-
//     to-nearest-even below that), as three byte limbs per column, with the
//     group sum of X, the group weight 2^(e_g - 21) and a +-X table indexed
//     by the raw residual-site byte.  The table is interleaved by group so
//     that the lanes of a warp (one group each) never share a bank when they
//     look up their sites; it is filled through a padded transpose.
//  3. Each lane pulls its 96 limb words into registers.  The trit decode masks
//     each code word once per slot (word & (0x03030303 << 2s) leaves 4^s times
//     the code t + 1 of trit 4b + s in byte b); three dp4a per slot against
//     the lo / mid / hi limbs accumulate per slot, and exact shifts fold the
//     slots, giving sum_j (t_j + 1) X_j; minus sum_j X_j that is T.x of the
//     group in int32.  The residual sites add +-X from the table (exact).
//     alpha and beta are applied in FP32 and the group weight once.  The
//     WALB2 phase-1 products V_r^T x go through the same path: a row of V is
//     a ternary row without zeros, its bits spread into 2-bit codes.
//  4. Each lane leaves its group's partial in shared memory; after the rows
//     one thread per output row sums the slices and lanes in a fixed order,
//     and the WALB2 phase-2 term sum_r U[n, r] z_r joins in the single store.
// Results are bitwise reproducible: no atomics, fixed reduction orders.
// Every mbarrier wait is bounded; a wait that gives up records
// WAL_ERR_TIMEOUT in the status word and the warp skips the rest of its rows.
#include "wal_internal.h"
#include "wal_device.cuh"
#include "wal_stream.h"

#include <algorithm>
#include <mutex>

namespace wal {

using namespace dev;

constexpr int kRowsPerStage = 2;
constexpr int kMaxThreads = 384;
constexpr int kMaxXChunks = 8;            // 8-column chunks of x per thread
constexpr uint32_t kMagic = 0x4B400000u;  // 1.5 * 2^23: adding it rounds |v| < 2^22 to an integer
constexpr uint32_t kSpinLimit = 1u << 22; // try_wait polls before a wait gives up
constexpr uint32_t kLimbStride = 100;     // words per group in the limb image (96 + 4 pad)
// one row of one warp in the ring: codes 32 x 32 B, sites 32 x 8 B (+16 B
// alignment slack), scales 32 x 4 B (+16 B slack)
constexpr uint32_t kSlotCodes = 0, kSlotSites = 1024, kSlotScales = 1024 + 272, kSlotBytes = 1024 + 272 + 144;

__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }
__device__ __forceinline__ void prefetch_l2(const void* p, uint32_t bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(p), "r"(bytes) : "memory");
}

// ---- raw shared-memory access (32-bit shared-window addresses) -------------
__device__ __forceinline__ void cp_async16_zfill(uint32_t dst, const void* src, uint32_t src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(src_bytes) : "memory");
}
__device__ __forceinline__ void cp_async4_zfill(uint32_t dst, const void* src, uint32_t src_bytes) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;" ::"r"(dst), "l"(src), "r"(src_bytes) : "memory");
}
__device__ __forceinline__ uint4 lds128(uint32_t a) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(a));
  return v;
}
__device__ __forceinline__ uint2 lds64(uint32_t a) {
  uint2 v;
  asm volatile("ld.shared.v2.u32 {%0, %1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(a));
  return v;
}
__device__ __forceinline__ uint32_t lds32(uint32_t a) {
  uint32_t v;
  asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(a));
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
__device__ __forceinline__ uint32_t byte_of(uint32_t w, int b) { return __byte_perm(w, 0u, 0x4440u | (uint32_t)b); }

// ---- mbarrier + bulk copies (one CTA is its own cluster) -------------------
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t done;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(done)
      : "r"(bar), "r"(parity)
      : "memory");
  return done != 0;
}
// Bounded wait: false (and the status word set) if the phase never completes.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, int32_t* status) {
  for (uint32_t it = 0; it < kSpinLimit; ++it)
    if (mbar_try_wait(bar, parity)) return true;
  if (status) atomicExch(status, (int32_t)WAL_ERR_TIMEOUT);
  return false;
}
__device__ __forceinline__ void bulk_g2s(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
               "l"(src), "r"(bytes), "r"(bar)
               : "memory");
}

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

struct SmemPlan {
  uint32_t table, limbs, xgsum, gsc, partz, part, vstage, ubuf, scratch, ring, mbar, total;
};

// Groups rounded up to a multiple of 32: the +-X table is interleaved as
// [entry][group], so lane l of a warp (group 32 s + l) always reads bank l.
__host__ __device__ inline uint32_t group_stride(int K) { return (uint32_t)((K / kGroup + 31) / 32 * 32); }

// Shared-memory carve-up of one CTA.
__host__ __device__ inline SmemPlan smem_plan(int K, int threads, int S, int RB, int rmax, bool signed_table,
                                              int stages, bool stage_v) {
  SmemPlan p;
  uint32_t off = 0;
  auto take = [&](uint32_t bytes) { uint32_t o = off; off = (off + bytes + 15u) & ~15u; return o; };
  const uint32_t G = (uint32_t)K / kGroup;
  p.table = take(group_stride(K) * (signed_table ? 256u : 128u) * 4u);
  p.limbs = take(G * kLimbStride * 4u);
  p.xgsum = take(G * 4u);
  p.gsc = take(G * 4u);
  p.partz = take((uint32_t)S * WAL_MAX_RANK * 4u);
  p.part = take((uint32_t)S * RB * 32u * 4u);  // per-lane partials [slice][row][lane]
  p.vstage = take(stage_v ? (uint32_t)rmax * (uint32_t)(K / 8) : 0u);
  p.ubuf = take((uint32_t)RB * 4u);             // U bit words of the tile's rows
  p.scratch = take(32u * 129u * 4u);            // X of 32 groups, rows padded to 129 words
  p.ring = take((uint32_t)(threads / 32) * stages * kRowsPerStage * kSlotBytes);
  p.mbar = take((uint32_t)(threads / 32) * stages * 8u);
  p.total = off;
  return p;
}

// One warp's view of its rows: row i of the warp is output row n0 + p + P i.
struct WarpRing {
  uint32_t ring;   // warp's ring base (shared window)
  uint32_t mbar;   // warp's mbarriers
  int stages;
  int nmine;
  int s, p, P, n0, G, K, k;
  const StreamItem* it;
  __device__ __forceinline__ uint32_t slot(int stage, int u) const {
    return ring + ((uint32_t)stage * kRowsPerStage + (uint32_t)u) * kSlotBytes;
  }
  __device__ __forceinline__ uint32_t bar(int stage) const { return mbar + (uint32_t)stage * 8u; }
  // groups of the warp's slice, and the group index of the slice's first group in row i
  __device__ __forceinline__ int ngroups() const { return min(32, G - 32 * s); }
  __device__ __forceinline__ size_t gbase(int i) const { return (size_t)(n0 + p + P * i) * G + 32 * s; }
};

__device__ __forceinline__ uint32_t site_bytes(int k) { return (uint32_t)k; }
__device__ __forceinline__ uint32_t scale_bytes(int k) { return k > 0 ? 4u : 2u; }

// Lane 0: queue the rows of chunk `chunk` (two rows) into ring stage `stage`.
// Site and scale ranges are widened to 16-byte boundaries (every buffer is
// zero-padded to a multiple of 16 bytes, so the widened range stays inside).
__device__ __forceinline__ void issue_chunk(const WarpRing& W, int stage, int chunk) {
  const int ng = W.ngroups();
  const uint32_t kb = site_bytes(W.k), sb = scale_bytes(W.k);
  const unsigned char* src[kRowsPerStage][3];
  uint32_t len[kRowsPerStage][3];
  uint32_t bytes = 0;
#pragma unroll
  for (int u = 0; u < kRowsPerStage; ++u) {
    const int i = chunk * kRowsPerStage + u;
    len[u][0] = len[u][1] = len[u][2] = 0u;
    src[u][0] = src[u][1] = src[u][2] = nullptr;
    if (i < W.nmine) {
      const size_t n = (size_t)(W.n0 + W.p + W.P * i);
      const size_t gb = W.gbase(i);
      src[u][0] = reinterpret_cast<const unsigned char*>(W.it->codes) + n * (size_t)(W.K / 4) + (size_t)W.s * 1024;
      len[u][0] = (uint32_t)ng * 32u;
      if (W.k > 0) {
        const size_t a = (gb * kb) & ~(size_t)15, e = ((gb + ng) * kb + 15) & ~(size_t)15;
        src[u][1] = W.it->sites + a;
        len[u][1] = (uint32_t)(e - a);
      }
      const size_t a = (gb * sb) & ~(size_t)15, e = ((gb + ng) * sb + 15) & ~(size_t)15;
      src[u][2] = reinterpret_cast<const unsigned char*>(W.it->scales) + a;
      len[u][2] = (uint32_t)(e - a);
      bytes += len[u][0] + len[u][1] + len[u][2];
    }
  }
  if (bytes == 0) return;
  const uint32_t bar = W.bar(stage);
  mbar_arrive_expect_tx(bar, bytes);
#pragma unroll
  for (int u = 0; u < kRowsPerStage; ++u) {
    if (len[u][0] == 0u) continue;
    const uint32_t sl = W.slot(stage, u);
    bulk_g2s(sl + kSlotCodes, src[u][0], len[u][0], bar);
    if (len[u][1]) bulk_g2s(sl + kSlotSites, src[u][1], len[u][1], bar);
    bulk_g2s(sl + kSlotScales, src[u][2], len[u][2], bar);
  }
}

// tab = table base + 4 * group; entries of one group are gstride4 bytes apart
template <bool SIGNED_TABLE>
__device__ __forceinline__ int32_t site_at(uint32_t tab, uint32_t gstride4, uint32_t byte) {
  if (SIGNED_TABLE) return ldsi(tab + byte * gstride4);
  const int32_t v = ldsi(tab + (byte & 0x7Fu) * gstride4);
  return (byte & 0x80u) ? -v : v;
}

// One row's contribution of this lane's group, read from the ring slot:
// 2^(e_g - 21) * (alpha * T.X + beta * R.X).  `hsw` swaps the two 16-byte
// halves of the lane's code chunk (matching the limb registers), so that the
// 32-byte-strided reads of a warp never share a bank.
template <int KS, bool SIGNED_TABLE>
__device__ __forceinline__ float row_value(uint32_t sl, uint32_t site_off, uint32_t scale_off, int lane,
                                           uint32_t hsw, const uint32_t (&lb)[8][kLimbWords], int32_t xs,
                                           float gsc, uint32_t tab, uint32_t gs4) {
  const uint32_t cd = sl + kSlotCodes + (uint32_t)lane * 32u;
  const uint4 c0 = lds128(cd + hsw), c1 = lds128(cd + (hsw ^ 16u));
  const uint32_t wv[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
  const int32_t tdot = group_dot(wv, lb) - xs;
  int32_t q = 0;
  if (KS == 8) {
    const uint2 sw = lds64(sl + kSlotSites + site_off + (uint32_t)lane * 8u);
    q = site_at<SIGNED_TABLE>(tab, gs4, byte_of(sw.x, 0)) + site_at<SIGNED_TABLE>(tab, gs4, byte_of(sw.x, 1)) +
        site_at<SIGNED_TABLE>(tab, gs4, byte_of(sw.x, 2));
    q += site_at<SIGNED_TABLE>(tab, gs4, byte_of(sw.x, 3)) + site_at<SIGNED_TABLE>(tab, gs4, byte_of(sw.y, 0)) +
         site_at<SIGNED_TABLE>(tab, gs4, byte_of(sw.y, 1));
    q += site_at<SIGNED_TABLE>(tab, gs4, byte_of(sw.y, 2)) + site_at<SIGNED_TABLE>(tab, gs4, byte_of(sw.y, 3));
  } else if (KS == 4) {
    const uint32_t sw = lds32(sl + kSlotSites + site_off + (uint32_t)lane * 4u);
    q = site_at<SIGNED_TABLE>(tab, gs4, byte_of(sw, 0)) + site_at<SIGNED_TABLE>(tab, gs4, byte_of(sw, 1)) +
        site_at<SIGNED_TABLE>(tab, gs4, byte_of(sw, 2)) + site_at<SIGNED_TABLE>(tab, gs4, byte_of(sw, 3));
  } else if (KS == 2) {
    const uint32_t sw = lds16(sl + kSlotSites + site_off + (uint32_t)lane * 2u);
    q = site_at<SIGNED_TABLE>(tab, gs4, sw & 0xFFu) + site_at<SIGNED_TABLE>(tab, gs4, sw >> 8);
  }
  if (KS == 0) {
    const float alpha = fp16_bits_to_float(lds16(sl + kSlotScales + scale_off + (uint32_t)lane * 2u));
    return alpha * ((float)tdot * gsc);
  }
  const uint32_t sc = lds32(sl + kSlotScales + scale_off + (uint32_t)lane * 4u);
  const float alpha = fp16_bits_to_float(sc & 0xFFFFu), beta = fp16_bits_to_float(sc >> 16);
  return fmaf(alpha, (float)tdot, beta * (float)q) * gsc;
}

template <int KS, bool SIGNED_TABLE>
__device__ __forceinline__ void run_rows(const WarpRing& W, int RB, int lane, bool active, uint32_t hsw,
                                         const uint32_t (&lb)[8][kLimbWords], int32_t xs, float gsc, uint32_t tab,
                                         uint32_t gs4, float* part, int32_t* status) {
  const int nc = (W.nmine + kRowsPerStage - 1) / kRowsPerStage;
  float* mine = part + ((size_t)W.s * RB + W.p) * 32 + lane;  // partial of row p + P i at mine[P i * 32]
  const uint32_t kb = site_bytes(KS), sb = scale_bytes(KS);
  int stage = 0;
  uint32_t parity = 0;
#pragma unroll 1
  for (int j = 0; j < nc; ++j) {
    if (!mbar_wait(W.bar(stage), parity, status)) return;
#pragma unroll
    for (int u = 0; u < kRowsPerStage; ++u) {
      const int i = j * kRowsPerStage + u;
      if (i < W.nmine) {  // uniform across the warp
        const size_t gb = W.gbase(i);
        const uint32_t site_off = (uint32_t)((gb * kb) & 15), scale_off = (uint32_t)((gb * sb) & 15);
        mine[(size_t)W.P * i * 32] =
            active ? row_value<KS, SIGNED_TABLE>(W.slot(stage, u), site_off, scale_off, lane, hsw, lb, xs, gsc, tab, gs4)
                   : 0.f;
      }
    }
    __syncwarp();  // every lane has consumed the stage before it is refilled
    if (lane == 0) issue_chunk(W, stage, j + W.stages);
    if (++stage == W.stages) {
      stage = 0;
      parity ^= 1u;
    }
  }
}

template <bool SIGNED_TABLE, int STAGES>
__global__ void __launch_bounds__(kMaxThreads, 1) stream_kernel(const __grid_constant__ StreamParams prm) {
  extern __shared__ __align__(16) unsigned char smem[];
  __shared__ float s_z[WAL_MAX_RANK];
  const int K = prm.K, S = prm.S, P = prm.P, RB = prm.RB;
  const int G = K / kGroup;
  const int threads = blockDim.x;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const SmemPlan sp = smem_plan(K, threads, S, RB, prm.rmax, SIGNED_TABLE, STAGES, prm.stage_v != 0);
  int32_t* table = reinterpret_cast<int32_t*>(smem + sp.table);
  uint32_t* limbs = reinterpret_cast<uint32_t*>(smem + sp.limbs);
  int32_t* xgsum = reinterpret_cast<int32_t*>(smem + sp.xgsum);
  float* gsc_s = reinterpret_cast<float*>(smem + sp.gsc);
  float* partz = reinterpret_cast<float*>(smem + sp.partz);
  float* part = reinterpret_cast<float*>(smem + sp.part);
  uint32_t* vst = reinterpret_cast<uint32_t*>(smem + sp.vstage);
  uint32_t* ubuf = reinterpret_cast<uint32_t*>(smem + sp.ubuf);
  int32_t* scratch = reinterpret_cast<int32_t*>(smem + sp.scratch);
  if (blockIdx.x == 0 && tid == 0 && prm.status) *prm.status = 0;  // this launch has seen no timeout

  // which product and which rows
  int item = 0;
  while (item + 1 < prm.n_items && (int)blockIdx.x >= prm.items[item + 1].tile_begin) ++item;
  const StreamItem& it = prm.items[item];
  const int n0 = ((int)blockIdx.x - it.tile_begin) * RB;
  const int rows = min(RB, it.N - n0);
  const int s = warp % S, p = warp / S;
  const int col0 = s * kSliceCols + lane * kGroup;
  const bool active = col0 < K;
  const int g = active ? col0 >> 7 : 0;
  const int nmine = p < rows ? (rows - p + P - 1) / P : 0;
  const int r = it.r;
  const int ks = it.k;

  WarpRing W;
  W.ring = smem_addr(smem + sp.ring) + (uint32_t)warp * STAGES * kRowsPerStage * kSlotBytes;
  W.mbar = smem_addr(smem + sp.mbar) + (uint32_t)warp * STAGES * 8u;
  W.stages = STAGES;
  W.nmine = nmine;
  W.s = s; W.p = p; W.P = P; W.n0 = n0; W.G = G; W.K = K; W.k = ks;
  W.it = &it;
  if (lane == 0) {
    for (int st = 0; st < STAGES; ++st) mbar_init(W.bar(st), 1u);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncwarp();

  // 1. x first (x may be the output of the previous stage: dependent-launch wait)
  pdl_wait();
  uint4 xr[kMaxXChunks];
  {
    const int n8 = K / 8;
#pragma unroll
    for (int i = 0; i < kMaxXChunks; ++i) {
      const int c8 = tid + i * threads;
      xr[i] = c8 < n8 ? __ldg(reinterpret_cast<const uint4*>(it.x) + c8) : make_uint4(0u, 0u, 0u, 0u);
    }
  }
  // the warp's TMA ring: every stage queued at once
  if (lane == 0)
    for (int st = 0; st < STAGES; ++st) issue_chunk(W, st, st);
  // WALB2 bit planes (V) and the tile's U words, by cp.async (one group)
  if (prm.stage_v && r > 0) {
    const int n16 = r * (K / 128);  // 16-byte pieces of the [r][K/32] bit planes
    for (int i = tid; i < n16; i += threads) cp_async16_zfill(smem_addr(vst) + 16u * i, it.vbits + 4 * i, 16u);
  }
  if (r > 0)
    for (int rl = tid; rl < rows; rl += threads)
      cp_async4_zfill(smem_addr(ubuf + rl), it.ubits + (size_t)(n0 + rl) * ((r + 31) / 32), 4u);
  cp_async_commit();
  pdl_trigger();
  // warm L2 with the next stage's weights, spread over all CTAs
  if (tid == 0 && prm.n_pf > 0) {
    for (int j = 0; j < prm.n_pf; ++j) {
      const unsigned long long bytes = prm.pf[j].bytes;
      const unsigned long long chunk = ((bytes / gridDim.x) + 4095ull) & ~4095ull;
      const unsigned long long b0 = chunk * blockIdx.x;
      if (b0 >= bytes) continue;
      const unsigned long long b1 = b0 + chunk < bytes ? b0 + chunk : bytes;
      for (unsigned long long o = b0; o < b1; o += 65536ull) {
        const unsigned long long len = (b1 - o) < 65536ull ? (b1 - o) : 65536ull;
        prefetch_l2(static_cast<const char*>(prm.pf[j].ptr) + o, (uint32_t)len);
      }
    }
  }

  // 2. fixed-point image of x
  const uint32_t Gp = group_stride(K);
  // blocks of 32 groups: phase A converts x (16 threads per group), phase B
  // transposes the block's X into the interleaved +-X table (lanes = groups)
  for (int gb = 0; gb < G; gb += 32) {
    const int nblk = min(32, G - gb);
#pragma unroll
    for (int i = 0; i < kMaxXChunks; ++i) {
      // chunk c8 = tid + i * threads, as loaded above; the 16 threads of one
      // group are 16 aligned lanes of one warp, so the test below is uniform
      // across each half-warp and the half-warp shuffles stay complete
      const int c8 = tid + i * threads;
      if (c8 < gb * 16 || c8 >= (gb + nblk) * 16) continue;
      const unsigned gmask = (lane & 16) ? 0xFFFF0000u : 0x0000FFFFu;
      const int c = 8 * c8;
      const uint4 raw = xr[i];
      const uint32_t pr[4] = {raw.x, raw.y, raw.z, raw.w};
      uint32_t m2 = 0u;  // largest |x| bit pattern, two bf16 lanes
#pragma unroll
      for (int q = 0; q < 4; ++q) m2 = __vmaxu2(m2, pr[q] & 0x7FFF7FFFu);
      uint32_t mx = max(m2 & 0xFFFFu, m2 >> 16);
#pragma unroll
      for (int off = 8; off; off >>= 1) mx = max(mx, __shfl_xor_sync(gmask, mx, off));
      uint32_t emax = mx >> 7;
      emax = emax > 1u ? emax : 1u;  // exponent field of the group maximum (denormals as 1)
      // X = round(x * 2^(148 - emax)); tiny groups are pre-scaled by 2^64 so the factor stays finite
      const float pre = emax < 64u ? 18446744073709551616.0f : 1.0f;
      const float scl = __uint_as_float((275u - emax - (emax < 64u ? 64u : 0u)) << 23);
      int32_t X[8];
      int32_t sum8 = 0;
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        const float xv = bf16_bits_to_float((pr[q >> 1] >> (16 * (q & 1))) & 0xFFFFu);
        X[q] = (int32_t)(__float_as_uint(fmaf(xv * pre, scl, __uint_as_float(kMagic))) - kMagic);
        sum8 += X[q];
      }
#pragma unroll
      for (int off = 8; off; off >>= 1) sum8 += __shfl_xor_sync(gmask, sum8, off);
      const int gg = c >> 7, pos = c & 127, wl = (c >> 4) & 7, h = (c >> 3) & 1;
      // limb image [group][word-in-group][limb][slot] (+4 words of padding per
      // group): byte b of (word wl, limb L, slot q) = limb L of column 16 wl + 4 b + q
      uint16_t* img16 = reinterpret_cast<uint16_t*>(limbs + (size_t)gg * kLimbStride);
#pragma unroll
      for (int L2 = 0; L2 < 3; ++L2)
#pragma unroll
        for (int q = 0; q < 4; ++q)
          img16[((wl * 3 + L2) * 4 + q) * 2 + h] =
              (uint16_t)__byte_perm((uint32_t)X[q], (uint32_t)X[4 + q], (uint32_t)(L2 | ((4 + L2) << 4)));
      if ((c8 & 15) == 0) {
        xgsum[gg] = sum8;
        gsc_s[gg] = emax >= 22u ? __uint_as_float((emax - 21u) << 23) : __uint_as_float(1u << (emax + 1u));
      }
      int32_t* srow = scratch + (gg - gb) * 129 + pos;
#pragma unroll
      for (int q = 0; q < 8; ++q) srow[q] = X[q];
    }
    __syncthreads();
    // phase B: entry e of group gg at table[e * Gp + gg]; lane = group
    if (lane < nblk)
      for (int pos = warp; pos < 128; pos += threads / 32) {
        const int32_t v = scratch[lane * 129 + pos];
        table[(size_t)pos * Gp + gb + lane] = v;
        if (SIGNED_TABLE) table[(size_t)(128 + pos) * Gp + gb + lane] = -v;
      }
    __syncthreads();
  }

  // 3. the 96 limb words of this lane's group into registers; lanes with bit 2
  // set swap the halves of their group (words 0-3 <-> 4-7), like their code reads
  const uint32_t hsw = (lane & 4) ? 16u : 0u;
  uint32_t lb[8][kLimbWords];
  int32_t xs = 0;
  float gsc = 0.f;
  if (active) {
    const uint4* img = reinterpret_cast<const uint4*>(limbs + (size_t)g * kLimbStride);
#pragma unroll
    for (int w = 0; w < 8; ++w) {
      const int wsw = hsw ? (w ^ 4) : w;
#pragma unroll
      for (int L2 = 0; L2 < 3; ++L2) {
        const uint4 v = img[wsw * 3 + L2];
        lb[w][L2 * 4 + 0] = v.x; lb[w][L2 * 4 + 1] = v.y; lb[w][L2 * 4 + 2] = v.z; lb[w][L2 * 4 + 3] = v.w;
      }
    }
    xs = xgsum[g];
    gsc = gsc_s[g];
  } else {
#pragma unroll
    for (int w = 0; w < 8; ++w)
#pragma unroll
      for (int q = 0; q < kLimbWords; ++q) lb[w][q] = 0u;
  }

  // WALB2 phase 1: rows of V (no zeros: bit set -> code 0, clear -> code 2)
  if (r > 0) {
    cp_async_wait<0>();  // V planes and U words
    __syncthreads();
  }
  for (int rho = p; rho < r; rho += P) {
    float val = 0.f;
    if (active) {
      const uint32_t* vrow = (prm.stage_v ? vst : it.vbits) + (size_t)rho * (K / 32) + (size_t)g * 4;
      const uint4 vb = *reinterpret_cast<const uint4*>(vrow);
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
    if (lane == 0) partz[s * WAL_MAX_RANK + rho] = val;
  }

  const uint32_t tab = smem_addr(table) + (uint32_t)g * 4u;
  const uint32_t gs4 = Gp * 4u;
  switch (ks) {
    case 8: run_rows<8, SIGNED_TABLE>(W, RB, lane, active, hsw, lb, xs, gsc, tab, gs4, part, prm.status); break;
    case 4: run_rows<4, SIGNED_TABLE>(W, RB, lane, active, hsw, lb, xs, gsc, tab, gs4, part, prm.status); break;
    case 2: run_rows<2, SIGNED_TABLE>(W, RB, lane, active, hsw, lb, xs, gsc, tab, gs4, part, prm.status); break;
    default: run_rows<0, SIGNED_TABLE>(W, RB, lane, active, hsw, lb, xs, gsc, tab, gs4, part, prm.status); break;
  }
  __syncthreads();

  // 4. slices and lanes in order, WALB2 phase 2, one store per output
  if (tid < r) {
    float a = 0.f;
    for (int s2 = 0; s2 < S; ++s2) a += partz[s2 * WAL_MAX_RANK + tid];
    s_z[tid] = fp16_bits_to_float(it.lr[tid]) * a;
  }
  __syncthreads();
  for (int rl = tid; rl < rows; rl += threads) {
    const float* pr = part + (size_t)rl * 32;
    float acc = 0.f;
    for (int s2 = 0; s2 < S; ++s2) {
      float a = 0.f;
#pragma unroll
      for (int l = 0; l < 32; ++l) a += pr[(size_t)s2 * RB * 32 + l];
      acc += a;
    }
    if (r > 0) {
      const uint32_t uw = ubuf[rl];
      float lr = 0.f;
      for (int rho = 0; rho < r; ++rho) lr += ((uw >> rho) & 1u) ? -s_z[rho] : s_z[rho];
      acc += lr;
    }
    it.y[n0 + rl] = acc;
  }
}

// ----------------------------------------------------------------------------
// host side
// ----------------------------------------------------------------------------
namespace {
int g_sms = 0;
int g_max_smem = 0;
std::once_flag g_once;
cudaError_t g_err = cudaSuccess;
constexpr int kStageChoices[2] = {4, 2};
}  // namespace

int stream_init() {
  std::call_once(g_once, [] {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&g_sms, cudaDevAttrMultiProcessorCount, dev);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&g_max_smem, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
    const int lim = g_max_smem - 1024;
    if (e == cudaSuccess) e = cudaFuncSetAttribute(stream_kernel<true, 4>, cudaFuncAttributeMaxDynamicSharedMemorySize, lim);
    if (e == cudaSuccess) e = cudaFuncSetAttribute(stream_kernel<false, 4>, cudaFuncAttributeMaxDynamicSharedMemorySize, lim);
    if (e == cudaSuccess) e = cudaFuncSetAttribute(stream_kernel<true, 2>, cudaFuncAttributeMaxDynamicSharedMemorySize, lim);
    if (e == cudaSuccess) e = cudaFuncSetAttribute(stream_kernel<false, 2>, cudaFuncAttributeMaxDynamicSharedMemorySize, lim);
    g_err = e;
  });
  if (g_err != cudaSuccess) return fail(WAL_ERR_CUDA, std::string("device initialisation: ") + cudaGetErrorString(g_err));
  return WAL_OK;
}

int num_sms() { return g_sms > 0 ? g_sms : 148; }

// Plan one launch over `n` products that share K.
int plan_stream(const StreamItem* items, int n, int K, StreamLaunch* out) {
  if (n < 1 || n > kMaxItems) return fail(WAL_ERR_ARG, "a stream launch takes 1..16 products");
  StreamLaunch L;
  L.S = (K + kSliceCols - 1) / kSliceCols;
  if (L.S > kMaxThreads / 32) return fail(WAL_ERR_UNSUPPORTED, "K above 49152 is not handled by this build");
  L.P = std::max(1, (kMaxThreads / 32) / L.S);
  L.threads = 32 * L.S * L.P;
  if (K / 8 > kMaxXChunks * L.threads) return fail(WAL_ERR_UNSUPPORTED, "K too large for the x-chunk registers");
  int rmax = 0;
  long total_rows = 0;
  for (int i = 0; i < n; ++i) {
    rmax = std::max(rmax, items[i].r);
    total_rows += items[i].N;
  }
  const int sms = num_sms();
  // one tile per SM where possible: the smallest RB whose tile count fits one wave
  int RB = (int)std::max(1L, (total_rows + sms - 1) / sms);
  for (;;) {
    long tiles = 0;
    for (int i = 0; i < n; ++i) tiles += (items[i].N + RB - 1) / RB;
    if (tiles <= sms || RB >= 4096) break;
    ++RB;
  }
  L.RB = RB;
  L.rmax = rmax;
  // richest configuration that fits: deeper ring, +-X table, staged V planes
  const int limit = g_max_smem - 1024;
  bool found = false;
  SmemPlan sp = {};
  for (int trial = 0; trial < 8 && !found; ++trial) {
    L.stages = kStageChoices[(trial >> 2) & 1];
    L.signed_table = !(trial & 2);
    L.stage_v = !(trial & 1) && rmax > 0;
    sp = smem_plan(K, L.threads, L.S, L.RB, rmax, L.signed_table, L.stages, L.stage_v);
    found = (int)sp.total <= limit;
  }
  while (!found && L.RB > 1) {
    L.RB = std::max(1, L.RB / 2);
    sp = smem_plan(K, L.threads, L.S, L.RB, rmax, L.signed_table, L.stages, L.stage_v);
    found = (int)sp.total <= limit;
  }
  if (!found) return fail(WAL_ERR_UNSUPPORTED, "K too large for the shared-memory plan");
  L.smem = sp.total;
  int tiles = 0;
  for (int i = 0; i < n; ++i) tiles += (items[i].N + L.RB - 1) / L.RB;
  L.tiles = tiles;
  *out = L;
  return WAL_OK;
}

int launch_stream(StreamParams& prm, const StreamLaunch& L, cudaStream_t stream, bool pdl) {
  prm.S = L.S;
  prm.P = L.P;
  prm.RB = L.RB;
  prm.rmax = L.rmax;
  prm.stage_v = L.stage_v ? 1 : 0;
  int t = 0;
  for (int i = 0; i < prm.n_items; ++i) {
    prm.items[i].tile_begin = t;
    t += (prm.items[i].N + L.RB - 1) / L.RB;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(L.tiles);
  cfg.blockDim = dim3(L.threads);
  cfg.dynamicSmemBytes = L.smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  cudaError_t e;
  if (L.stages == 4)
    e = L.signed_table ? cudaLaunchKernelEx(&cfg, stream_kernel<true, 4>, prm)
                       : cudaLaunchKernelEx(&cfg, stream_kernel<false, 4>, prm);
  else
    e = L.signed_table ? cudaLaunchKernelEx(&cfg, stream_kernel<true, 2>, prm)
                       : cudaLaunchKernelEx(&cfg, stream_kernel<false, 2>, prm);
  if (e != cudaSuccess) return fail(WAL_ERR_CUDA, std::string("stream_kernel launch: ") + cudaGetErrorString(e));
  return WAL_OK;
}

}  // namespace wal
