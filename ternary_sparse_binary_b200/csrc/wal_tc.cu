// Tensor-core product for batches of 8 or more activation rows
//   Y[M][N] = X[M][K] W^T,   W = alpha*T + beta*R + U diag(s) V^T
// (WAL-Ternary-8B model card, "Representation").  Only here is the product a
// dense contraction, so only here do the 5th-generation tensor cores run.
//
// Exact FP16 operands.  alpha*t and beta*r (t, r in {-1, 0, +1}, alpha and beta
// FP16) are FP16 values exactly, so W's ternary and residual planes are
// decoded to FP16 with the group scales folded in: A_T = alpha (x) T and
// A_R = beta (x) R, two MMAs into one FP32 accumulator in tensor memory (their
// sum alpha*t + beta*r would not be exact in FP16 where a site falls on a
// nonzero trit, so the planes stay apart).  X is BF16; scaled by a power of
// two per activation row it is FP16 exactly (see tc_prep_kernel), and the
// power of two comes off again in the epilogue.
//
// Launch 1, tc_prep_kernel (one CTA per activation row m):
//   - 2^sc_m puts max|x_m| in [2^14, 2^15); x_m * 2^sc_m is written as FP16,
//     exact for every element down to 2^-31 of the row maximum and rounded to
//     nearest-even below that, into the pre-tiled B operand: per 64-column
//     K-block and tile of activation rows, M_tile rows of 128 bytes in the
//     tensor core's 128-byte-swizzled K-major layout, so one bulk copy moves a
//     whole B tile.  Inside every 16 columns the order is the 4 x 4 transpose
//     (column 16b + 4i + j goes to position 16b + 4j + i), which is the order
//     the trit decode below produces.
//   - WALB2 phase 1: z_r = sum_j V[j][r] x_j 2^sc_m in FP32 (fixed order), then
//     2^t_m puts max_r |z_r| in [2^14, 2^15) and z_r 2^-t_m is split into an
//     FP16 pair hi + lo (about 22 significant bits), stored as the B operand
//     of one more MMA: columns 0..r-1 hi, r..2r-1 lo, zero to 64.
// Launch 2, tc_kernel: one CTA per (128-row tile of W, tile of activation
// rows), 10 warps:
//   warp 0    lane 0 streams the B tiles (bulk copies, mbarrier ring);
//   warp 1    allocates tensor memory; lane 0 issues the MMAs:
//             D  += A_T B + A_R B          per 64-column K-block,
//             D2  = A_lr B_lr              once, A_lr[n] = (+-s_r, +-s_r) from U;
//   warps 2-9 decode: two teams of 128 threads, one output row per thread,
//             team h taking the K-blocks 2g + h of every group g.  Per 16
//             trits (one code word) four masks give the byte codes of slots
//             {s, 4+s, 8+s, 12+s}; a multiply-add turns each code c into the
//             byte-permute selector (2c, 2c+1), and byte permutes pick
//             {-alpha, 0, +alpha} as FP16 pairs from two table registers.  The
//             residual plane is zeroed and the k sites scattered as +-beta.
//             Then the same warps run the epilogue:
//             y[m][n] = (D + D2 2^t_m) 2^-sc_m.
// With few row tiles the K range is split over CTAs (ks splits of whole
// 128-column groups); each split writes its raw sums and a third launch adds
// the splits in order and applies 2^-sc_m.  The WALB2 MMA belongs to split 0.
// Launches 2 and 3 are programmatic dependent launches: launch 2 starts while
// launch 1 runs (the decoders need only the weights), and only its B
// producer and epilogue wait for launch 1's grid (griddepcontrol.wait);
// launch 3 is scheduled early and waits for launch 2's whole grid.
// All mbarrier waits are bounded; one that gives up records WAL_ERR_TIMEOUT in
// the status word and its role stops issuing work.
#include "wal_internal.h"
#include "wal_device.cuh"
#include "wal_ptx.cuh"
#include "wal_tc.h"

#include <algorithm>
#include <mutex>

namespace wal {

using namespace ptx;

namespace {

constexpr int kRows = 128;           // MMA M: rows of W per tile
constexpr int kBlockK = 64;          // K per pipeline stage: one 128-byte row of FP16
constexpr int kMaxTileM = 256;       // MMA N limit
constexpr int kThreads = 320;        // 10 warps
constexpr int kPrepThreads = 256;
constexpr uint32_t kATile = kRows * 128u;  // 16 KB: one FP16 plane of a stage
constexpr int kMaxStages = 4;

struct TcPrepParams {
  const uint16_t* X;
  int ldx, M, K, r, M_tile;
  const uint32_t* vbits;
  char* xt;      // [n_mt][K/64][M_tile x 128 B]
  char* zt;      // [n_mt][M_tile x 128 B]
  float2* scal;  // [M_pad] {2^-sc_m, 2^t_m}
  int32_t* status;
};

struct TcParams {
  const uint32_t* codes;
  const uint8_t* sites;
  const uint16_t* scales;
  const uint32_t* ubits;
  const uint16_t* lr;
  const char* xt;
  const char* zt;
  const float2* scal;
  float* Y;
  int ldy, N, K, r, M, M_tile, stages, n_tiles_n;
  int ks, gps;         // K splits and 128-column groups per split
  float* part;         // ks > 1: raw partial sums [ks][M][N]
  uint32_t d2_col;     // tensor-memory column of D2
  uint32_t tmem_cols;  // allocated tensor-memory columns
  int32_t* status;
};

// 2^e as a double, e in [-1022, 1023].
__device__ __forceinline__ double pow2d(int e) { return __longlong_as_double((long long)(e + 1023) << 52); }

// floor(log2(v)) of a finite nonzero float bit pattern (sign ignored).
__device__ __forceinline__ int ilog2f_bits(uint32_t b) {
  const uint32_t ex = (b >> 23) & 0xFFu;
  if (ex) return (int)ex - 127;
  return -149 + (31 - __clz((int)(b & 0x7FFFFFu)));
}

// ---------------------------------------------------------------------------
// launch 1: FP16 image of X (pre-tiled B operand) and WALB2 phase 1
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(kPrepThreads) tc_prep_kernel(const TcPrepParams p) {
  const int m = blockIdx.x, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  if (m == 0 && tid == 0 && p.status) *p.status = 0;
  // the product launch may start now: its decoders need only the weights
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  const bool live = m < p.M;
  const int KB = p.K / kBlockK, n16 = p.K / 16;
  const int mt = m / p.M_tile, row = m % p.M_tile;
  const uint16_t* xrow = p.X + (size_t)(live ? m : 0) * p.ldx;
  __shared__ uint32_t s_red[kPrepThreads / 32];
  __shared__ float s_z[kPrepThreads / 32][WAL_MAX_RANK];
  __shared__ float s_zr[WAL_MAX_RANK];
  __shared__ int s_t;

  // largest |x| as a bit pattern (monotonic for finite values)
  uint32_t mx = 0;
  if (live)
    for (int c = tid; c < p.K / 8; c += kPrepThreads) {
      const uint4 v = __ldg(reinterpret_cast<const uint4*>(xrow) + c);
      const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int q = 0; q < 4; ++q) mx = max(mx, max(w[q] & 0x7FFFu, (w[q] >> 16) & 0x7FFFu));
    }
#pragma unroll
  for (int off = 16; off; off >>= 1) mx = max(mx, __shfl_xor_sync(0xffffffffu, mx, off));
  if (lane == 0) s_red[warp] = mx;
  __syncthreads();
  mx = 0;
#pragma unroll
  for (int w = 0; w < kPrepThreads / 32; ++w) mx = max(mx, s_red[w]);
  const int sc = mx ? 14 - ilog2f_bits(mx << 16) : 0;
  const double f = pow2d(sc);

  // the V bit planes in shared memory (coalesced), read per 16 columns below
  extern __shared__ __align__(16) uint32_t s_v[];  // [r][K/32]
  const int vwords = p.r * (p.K / 32);
  for (int i = tid; i < vwords / 4; i += kPrepThreads)
    reinterpret_cast<uint4*>(s_v)[i] = __ldg(reinterpret_cast<const uint4*>(p.vbits) + i);
  __syncthreads();

  float acc[WAL_MAX_RANK];
#pragma unroll
  for (int q = 0; q < WAL_MAX_RANK; ++q) acc[q] = 0.f;
  for (int b = tid; b < n16; b += kPrepThreads) {
    float xs[16];
    if (live) {
      const uint4 v0 = __ldg(reinterpret_cast<const uint4*>(xrow) + 2 * b);
      const uint4 v1 = __ldg(reinterpret_cast<const uint4*>(xrow) + 2 * b + 1);
      const uint32_t w[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
#pragma unroll
      for (int j = 0; j < 16; ++j)
        xs[j] = (float)((double)dev::bf16_bits_to_float((w[j >> 1] >> (16 * (j & 1))) & 0xFFFFu) * f);
    } else {
#pragma unroll
      for (int j = 0; j < 16; ++j) xs[j] = 0.f;
    }
    // FP16, 4 x 4 transposed inside the 16 columns
    uint32_t hw[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int i0 = 2 * i, i1 = 2 * i + 1;
      const int j0 = 4 * (i0 & 3) + (i0 >> 2), j1 = 4 * (i1 & 3) + (i1 >> 2);
      hw[i] = (uint32_t)__half_as_ushort(__float2half_rn(xs[j0])) |
              ((uint32_t)__half_as_ushort(__float2half_rn(xs[j1])) << 16);
    }
    const int kb = b >> 2, bq = b & 3;
    char* tile = p.xt + ((size_t)mt * KB + kb) * ((size_t)p.M_tile * 128u);
    *reinterpret_cast<uint4*>(tile + sw128((uint32_t)row, 2u * bq)) = make_uint4(hw[0], hw[1], hw[2], hw[3]);
    *reinterpret_cast<uint4*>(tile + sw128((uint32_t)row, 2u * bq + 1u)) = make_uint4(hw[4], hw[5], hw[6], hw[7]);
    // WALB2 phase 1 partials: sum_j V[j][rho] x_j, V = -1 where the bit is set
    if (p.r > 0) {
#pragma unroll
      for (int q = 0; q < WAL_MAX_RANK; ++q) {
        if (q < p.r) {
          const uint32_t bits = (s_v[q * (p.K / 32) + (b >> 1)] >> (16 * (b & 1))) & 0xFFFFu;
          float s = 0.f;
#pragma unroll
          for (int j = 0; j < 16; ++j) s += __uint_as_float(__float_as_uint(xs[j]) ^ (((bits >> j) & 1u) << 31));
          acc[q] += s;
        }
      }
    }
  }
  if (tid == 0) p.scal[m] = make_float2((float)pow2d(-sc), 1.f);
  if (p.r == 0) return;

#pragma unroll
  for (int q = 0; q < WAL_MAX_RANK; ++q) {
    float v = acc[q];
#pragma unroll
    for (int off = 16; off; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
    if (lane == 0) s_z[warp][q] = v;
  }
  __syncthreads();
  if (tid < 32) {
    float z = 0.f;
    if (tid < p.r)
#pragma unroll
      for (int w = 0; w < kPrepThreads / 32; ++w) z += s_z[w][tid];
    s_zr[tid] = z;
    uint32_t zm = __float_as_uint(z) & 0x7FFFFFFFu;
#pragma unroll
    for (int off = 16; off; off >>= 1) zm = max(zm, __shfl_xor_sync(0xffffffffu, zm, off));
    if (tid == 0) {
      int t = zm ? ilog2f_bits(zm) - 14 : 0;
      t = max(-120, min(t, 120));
      s_t = t;
      p.scal[m] = make_float2((float)pow2d(-sc), (float)pow2d(t));
    }
  }
  __syncthreads();
  if (tid < 64) {
    // column kk of the WALB2 B operand: hi of rank kk, lo of rank kk - r, else 0
    float hv = 0.f;
    if (live && tid < 2 * p.r) {
      const int q = tid < p.r ? tid : tid - p.r;
      const float v = (float)((double)s_zr[q] * pow2d(-s_t));
      const float hi = __half2float(__float2half_rn(v));
      hv = tid < p.r ? hi : __half2float(__float2half_rn(v - hi));
    }
    char* tile = p.zt + (size_t)mt * ((size_t)p.M_tile * 128u);
    *reinterpret_cast<__half*>(tile + sw128((uint32_t)row, (uint32_t)tid >> 3) + 2 * (tid & 7)) = __float2half_rn(hv);
  }
}

// ---------------------------------------------------------------------------
// launch 2: decode + tcgen05 MMA + epilogue
// ---------------------------------------------------------------------------

// 16 trits (one code word) -> two 16-byte chunks of FP16 {-a, 0, +a} in the
// 4 x 4 transposed order.  ta = (-a, 0), tb = (+a, 0) as FP16 pairs; code c
// selects bytes 2c, 2c+1 of (ta, tb).
__device__ __forceinline__ void decode_word(uint32_t w, uint32_t ta, uint32_t tb, uint4& c0, uint4& c1) {
  const uint32_t s0 = (w & 0x03030303u) * 0x22u + 0x10101010u;
  const uint32_t s1 = ((w >> 2) & 0x03030303u) * 0x22u + 0x10101010u;
  const uint32_t s2 = ((w >> 4) & 0x03030303u) * 0x22u + 0x10101010u;
  const uint32_t s3 = ((w >> 6) & 0x03030303u) * 0x22u + 0x10101010u;
  c0.x = __byte_perm(ta, tb, s0);        // trits 0, 4
  c0.y = __byte_perm(ta, tb, s0 >> 16);  // 8, 12
  c0.z = __byte_perm(ta, tb, s1);        // 1, 5
  c0.w = __byte_perm(ta, tb, s1 >> 16);  // 9, 13
  c1.x = __byte_perm(ta, tb, s2);        // 2, 6
  c1.y = __byte_perm(ta, tb, s2 >> 16);  // 10, 14
  c1.z = __byte_perm(ta, tb, s3);        // 3, 7
  c1.w = __byte_perm(ta, tb, s3 >> 16);  // 11, 15
}

template <int KS>
struct GroupLoad {
  uint4 codes;
  uint32_t sites_lo, sites_hi;
  uint32_t scales;
};

template <int KS>
__device__ __forceinline__ GroupLoad<KS> load_group(const TcParams& p, int n, int g, int h, int G) {
  GroupLoad<KS> v;
  const size_t rg = (size_t)n * G + g;
  v.codes = __ldg(reinterpret_cast<const uint4*>(p.codes + (size_t)n * (p.K / 16) + 8 * g + 4 * h));
  v.sites_lo = v.sites_hi = 0u;
  if (KS == 8) {
    const uint2 s = __ldg(reinterpret_cast<const uint2*>(p.sites + rg * 8));
    v.sites_lo = s.x; v.sites_hi = s.y;
  } else if (KS == 4) {
    v.sites_lo = __ldg(reinterpret_cast<const uint32_t*>(p.sites + rg * 4));
  } else if (KS == 2) {
    v.sites_lo = __ldg(reinterpret_cast<const uint16_t*>(p.sites + rg * 2));
  }
  v.scales = KS ? __ldg(reinterpret_cast<const uint32_t*>(p.scales) + rg) : (uint32_t)__ldg(p.scales + rg);
  return v;
}

template <int KS>
__global__ void __launch_bounds__(kThreads, 2) tc_kernel(const TcParams p) {
  extern __shared__ uint8_t smem_raw[];
  constexpr bool kHasR = KS > 0;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  // the split-sum launch may be scheduled now; it waits for this whole grid
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  const uint32_t base = (smem_u32(smem_raw) + 1023u) & ~1023u;
  const uint32_t b_bytes = (uint32_t)p.M_tile * 128u;
  const uint32_t stage_bytes = kATile * (kHasR ? 2u : 1u) + b_bytes;
  const int S = p.stages;
  const uint32_t bars = base + (uint32_t)S * stage_bytes;
  // barriers: b_full[S], a_full[S], empty[S], acc_full.  a_full(s) completes
  // when the 128 decoders of the stage's team have arrived, b_full(s) when the
  // B tile's bulk copy has landed (its own barrier, so that the producer can
  // wait for every copy it issued whatever the decoders do).
  auto b_full = [&](int s) { return bars + 8u * s; };
  auto a_full = [&](int s) { return bars + 8u * (S + s); };
  auto empty = [&](int s) { return bars + 8u * (2 * S + s); };
  const uint32_t acc_full = bars + 8u * (3 * S);
  const uint32_t tmem_slot = acc_full + 8u;
  const uint32_t scal_s = (tmem_slot + 4u + 15u) & ~15u;
  auto a_t = [&](int s) { return base + (uint32_t)s * stage_bytes; };
  auto a_r = [&](int s) { return base + (uint32_t)s * stage_bytes + kATile; };
  auto b_t = [&](int s) { return base + (uint32_t)s * stage_bytes + kATile * (kHasR ? 2u : 1u); };

  // CTA -> (row tile, K split, activation tile); row tiles vary fastest so
  // that concurrent CTAs share B tiles in L2
  const int n_tile = blockIdx.x % p.n_tiles_n;
  const int split = (blockIdx.x / p.n_tiles_n) % p.ks, mt = blockIdx.x / (p.n_tiles_n * p.ks);
  const int KB = p.K / kBlockK;
  const int g0 = split * p.gps, G = min(p.K / 128, g0 + p.gps);  // this split's groups [g0, G)
  const int KBl = 2 * (G - g0), kb0 = 2 * g0;                     // its K-blocks [kb0, kb0 + KBl)
  const bool has_lr = p.r > 0 && split == 0;                       // the WALB2 MMA belongs to split 0
  const int n_iter = KBl + (has_lr ? 1 : 0);
  const uint32_t ncols = p.tmem_cols;

  if (tid == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(a_full(s), 128);  // the 128 decoders of the stage's team
      mbar_init(b_full(s), 1);    // the producer's arrival with the B tile's bytes
      mbar_init(empty(s), 1);
    }
    mbar_init(acc_full, 1);
    mbar_init_fence();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, ncols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = lds32(tmem_slot);

  if (warp == 0) {
    // ---- B producer ----
    if (lane == 0) {
      // the B tiles are the prep launch's output
      asm volatile("griddepcontrol.wait;" ::: "memory");
      int issued = 0;
      for (int i = 0; i < n_iter; ++i) {
        const int s = i % S;
        const uint32_t ph = (uint32_t)(i / S) & 1u;
        if (!mbar_wait(empty(s), ph ^ 1u, p.status)) break;
        const char* src = i < KBl ? p.xt + ((size_t)mt * KB + kb0 + i) * b_bytes : p.zt + (size_t)mt * b_bytes;
        mbar_arrive_expect_tx(b_full(s), b_bytes);
        bulk_g2s(b_t(s), src, b_bytes, b_full(s));
        issued = i + 1;
      }
      // every copy issued lands before the CTA leaves (a slot is refilled only
      // after its previous copy was consumed, so at most the last S can be
      // outstanding)
      for (int i = max(0, issued - S); i < issued; ++i) mbar_drain(b_full(i % S), (uint32_t)(i / S) & 1u, p.status);
    }
  } else if (warp == 1) {
    // ---- MMA issuer ----
    // The whole warp runs the loop, so its addresses and counters stay
    // warp-uniform; one elected lane issues the MMAs and commits.  A wait
    // ends the loop for every lane together (__all_sync).
    const uint32_t idesc = idesc_f16_f32(kRows, (uint32_t)p.M_tile);
    // descriptors of stage 0; a stage step or a 16-column step only moves
    // the 14-bit start-address field (address / 16), which never carries
    const uint64_t da0 = sdesc_sw128(a_t(0)), dr0 = sdesc_sw128(a_r(0)), db0 = sdesc_sw128(b_t(0));
    const uint32_t dstage = stage_bytes >> 4;
    bool ok = true;
    int s = 0;
    uint32_t ph = 0u;
    for (int i = 0; i < KBl && ok; ++i) {
      ok = __all_sync(0xffffffffu, mbar_wait(a_full(s), ph, p.status) && mbar_wait(b_full(s), ph, p.status));
      if (!ok) break;
      tc_fence_after();
      if (elect_one()) {
        const uint64_t so = (uint64_t)((uint32_t)s * dstage);
#pragma unroll
        for (int kk = 0; kk < kBlockK / 16; ++kk) {
          const uint64_t bd = db0 + so + 2u * kk;
          mma_f16(tmem, da0 + so + 2u * kk, bd, idesc, (i | kk) != 0);
          if (kHasR) mma_f16(tmem, dr0 + so + 2u * kk, bd, idesc, 1u);
        }
        mma_commit(empty(s));
      }
      __syncwarp();
      if (++s == S) {
        s = 0;
        ph ^= 1u;
      }
    }
    if (ok && has_lr) {
      const int s2 = KBl % S;
      const uint32_t ph2 = (uint32_t)(KBl / S) & 1u;
      ok = __all_sync(0xffffffffu, mbar_wait(a_full(s2), ph2, p.status) && mbar_wait(b_full(s2), ph2, p.status));
      if (ok) {
        tc_fence_after();
        if (elect_one()) {
          for (int kk = 0; kk < (2 * p.r + 15) / 16; ++kk)
            mma_f16(tmem + p.d2_col, sdesc_sw128(a_t(s2) + 32u * kk), sdesc_sw128(b_t(s2) + 32u * kk), idesc,
                    kk != 0);
          mma_commit(empty(s2));
        }
        __syncwarp();
      }
    }
    // acc_full tracks every MMA issued before it, also after a wait gave up;
    // tensor memory is released only once they have completed
    if (elect_one()) mma_commit(acc_full);
    __syncwarp();
    if (lane == 0) mbar_drain(acc_full, 0u, p.status);
    __syncwarp();
  } else {
    // ---- decoders, then epilogue ----
    const int h = (warp - 2) >> 2;      // team
    const int q = warp & 3;             // tensor-memory lane quarter
    const int row = 32 * q + lane;
    const int n = n_tile * kRows + row;
    const bool live = n < p.N;
    const uint32_t rowoff = (uint32_t)(row >> 3) * 1024u + (uint32_t)(row & 7) * 128u;
    const uint32_t r7 = (uint32_t)row & 7u;
    bool ok = true;

    const int GK = p.K / 128;
    GroupLoad<KS> cur = {}, nxt = {};
    if (live) cur = load_group<KS>(p, n, g0, h, GK);
    if (live && g0 + 1 < G) nxt = load_group<KS>(p, n, g0 + 1, h, GK);
    for (int g = g0; g < G && ok; ++g) {
      GroupLoad<KS> nn = {};
      if (live && g + 2 < G) nn = load_group<KS>(p, n, g + 2, h, GK);
      const int i = 2 * (g - g0) + h, s = i % S;
      const uint32_t ph = (uint32_t)(i / S) & 1u;
      ok = mbar_wait(empty(s), ph ^ 1u, p.status);
      if (!ok) break;
      const uint32_t at = a_t(s) + rowoff;
      // ternary plane: alpha (x) T
      const uint32_t alpha = cur.scales & 0xFFFFu;
      const uint32_t ta = live ? (alpha ^ 0x8000u) : 0u, tb = alpha;
      const uint32_t cw[4] = {cur.codes.x, cur.codes.y, cur.codes.z, cur.codes.w};
#pragma unroll
      for (int w = 0; w < 4; ++w) {
        uint4 c0, c1;
        decode_word(cw[w], ta, tb, c0, c1);
        sts128(at + ((((uint32_t)(2 * w)) ^ r7) << 4), c0);
        sts128(at + ((((uint32_t)(2 * w + 1)) ^ r7) << 4), c1);
      }
      if (kHasR) {
        // residual plane: zero the row, scatter +-beta at this half's sites
        const uint32_t ar = a_r(s) + rowoff;
#pragma unroll
        for (int c = 0; c < 8; ++c) sts128(ar + (((uint32_t)c ^ r7) << 4), make_uint4(0u, 0u, 0u, 0u));
        const uint32_t beta = cur.scales >> 16;
        // straight-line code with a predicated store per site: the sites of
        // a warp's rows fall in either half at random, and a branch per site
        // diverged on every one
#pragma unroll
        for (int j = 0; j < KS; ++j) {
          const uint32_t b = ((j < 4 ? cur.sites_lo : cur.sites_hi) >> (8 * (j & 3))) & 0xFFu;
          const uint32_t pos = b & 63u, jj = pos & 15u;
          const uint32_t col = (pos & 48u) | ((jj & 3u) << 2) | (jj >> 2);
          sts16_if(live && ((b >> 6) & 1u) == (uint32_t)h, ar + ((((col >> 3) ^ r7) & 7u) << 4) + 2u * (col & 7u),
                   beta ^ ((b & 0x80u) << 8));
        }
      }
      fence_proxy_async_smem();
      mbar_arrive(a_full(s));
      cur = nxt;
      nxt = nn;
    }
    // WALB2 phase-2 operand A_lr[n] = (+-s_0 .. +-s_{r-1}, +-s_0 .. +-s_{r-1}, 0 ...)
    if (ok && has_lr && h == (KBl & 1)) {
      const int s = KBl % S;
      const uint32_t ph = (uint32_t)(KBl / S) & 1u;
      ok = mbar_wait(empty(s), ph ^ 1u, p.status);
      if (ok) {
        const uint32_t u = live ? __ldg(p.ubits + (size_t)n * ((p.r + 31) / 32)) : 0u;
        const uint32_t at = a_t(s) + rowoff;
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          uint32_t hw[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            uint32_t v2 = 0u;
#pragma unroll
            for (int hlf = 0; hlf < 2; ++hlf) {
              const int kk = 8 * c + 2 * e + hlf;
              const int rho = kk < p.r ? kk : kk - p.r;
              uint32_t v = 0u;
              if (live && kk < 2 * p.r) v = (uint32_t)__ldg(p.lr + rho) ^ (((u >> rho) & 1u) << 15);
              v2 |= v << (16 * hlf);
            }
            hw[e] = v2;
          }
          sts128(at + (((uint32_t)c ^ r7) << 4), make_uint4(hw[0], hw[1], hw[2], hw[3]));
        }
        fence_proxy_async_smem();
        mbar_arrive(a_full(s));
      }
    }

    // ---- epilogue ----
    asm volatile("griddepcontrol.wait;" ::: "memory");  // the row scales are the prep launch's output
    for (int j = tid - 64; j < p.M_tile; j += 256) {
      const int m = mt * p.M_tile + j;
      const float2 v = m < p.M ? p.scal[m] : make_float2(0.f, 0.f);
      sts64(scal_s + 8u * j, make_uint2(__float_as_uint(v.x), __float_as_uint(v.y)));
    }
    named_bar_sync(1, 256);
    if (mbar_wait(acc_full, 0u, p.status)) {
      tc_fence_after();
      const uint32_t lane_base = tmem + ((uint32_t)(32 * q) << 16);
      for (int c16 = h; c16 < p.M_tile / 16; c16 += 2) {
        uint32_t d[16], e[16];
        tmem_ld16(lane_base + 16u * c16, d);
        if (has_lr) tmem_ld16(lane_base + p.d2_col + 16u * c16, e);
        tmem_ld_wait();
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          const int col = 16 * c16 + j, m = mt * p.M_tile + col;
          const uint2 sv = lds64(scal_s + 8u * col);
          float y = __uint_as_float(d[j]);
          if (has_lr) y = fmaf(__uint_as_float(e[j]), __uint_as_float(sv.y), y);
          if (p.ks == 1) {
            y *= __uint_as_float(sv.x);
            if (live && m < p.M) p.Y[(size_t)m * p.ldy + n] = y;
          } else if (live && m < p.M) {
            p.part[((size_t)split * p.M + m) * p.N + n] = y;  // raw: scaled by 2^-sc_m after the sum
          }
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, ncols);
  }
}

// Split-K: y[m][n] = 2^-sc_m * sum over splits (in order) of the raw partials.
__global__ void __launch_bounds__(256) tc_reduce_kernel(const float* __restrict__ part, const float2* __restrict__ scal,
                                                        float* Y, int ldy, int M, int N, int ks) {
  asm volatile("griddepcontrol.wait;" ::: "memory");  // the partial sums are the product launch's output
  const size_t total = (size_t)M * N;
  for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < total; i += (size_t)gridDim.x * blockDim.x) {
    const int m = (int)(i / N), n = (int)(i % N);
    float acc = 0.f;
    for (int s2 = 0; s2 < ks; ++s2) acc += __ldg(part + (size_t)s2 * total + i);
    Y[(size_t)m * ldy + n] = acc * __ldg(&scal[m].x);
  }
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------
// per device: the shared-memory opt-in limit and the kernels' attribute set once
struct TcDev {
  std::once_flag once;
  cudaError_t err = cudaSuccess;
  int smem_limit = 0;
};
TcDev g_tc_dev[kMaxDevices];

int tc_init() {
  int dev = 0;
  int st = current_device(&dev);
  if (st) return st;
  TcDev& d = g_tc_dev[dev];
  std::call_once(d.once, [&d, dev] {
    cudaError_t e = cudaDeviceGetAttribute(&d.smem_limit, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
    const int lim = d.smem_limit;
    if (e == cudaSuccess) e = cudaFuncSetAttribute(tc_prep_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, 100 * 1024);
    if (e == cudaSuccess) e = cudaFuncSetAttribute(tc_kernel<0>, cudaFuncAttributeMaxDynamicSharedMemorySize, lim);
    if (e == cudaSuccess) e = cudaFuncSetAttribute(tc_kernel<2>, cudaFuncAttributeMaxDynamicSharedMemorySize, lim);
    if (e == cudaSuccess) e = cudaFuncSetAttribute(tc_kernel<4>, cudaFuncAttributeMaxDynamicSharedMemorySize, lim);
    if (e == cudaSuccess) e = cudaFuncSetAttribute(tc_kernel<8>, cudaFuncAttributeMaxDynamicSharedMemorySize, lim);
    d.err = e;
  });
  if (d.err != cudaSuccess)
    return fail(WAL_ERR_CUDA, std::string("tensor-core path initialisation: ") + cudaGetErrorString(d.err));
  return WAL_OK;
}

int tc_smem_limit() {
  int dev = 0;
  return current_device(&dev) == WAL_OK && g_tc_dev[dev].smem_limit > 0 ? g_tc_dev[dev].smem_limit : 232448;
}

uint32_t pow2_ceil(uint32_t v) {
  uint32_t p = 1;
  while (p < v) p <<= 1;
  return p;
}

}  // namespace

int plan_tc(const wal_matrix* m, int M, TcPlan* out) {
  TcPlan P = {};
  P.n_tiles_n = (m->N + kRows - 1) / kRows;
  P.n_mt = (M + kMaxTileM - 1) / kMaxTileM;
  P.M_tile = ((M + P.n_mt - 1) / P.n_mt + 15) / 16 * 16;
  P.M_pad = P.n_mt * P.M_tile;
  const uint32_t b_bytes = (uint32_t)P.M_tile * 128u;
  const uint32_t stage_bytes = kATile * (m->k > 0 ? 2u : 1u) + b_bytes;
  const uint32_t extra = 1024u /*alignment*/ + 8u * (3 * kMaxStages + 1) + 16u + 8u * kMaxTileM;
  const uint32_t d2 = pow2_ceil((uint32_t)P.M_tile);
  P.tmem_cols = std::max(32u, d2 * (m->r > 0 ? 2u : 1u));
  // Two CTAs per SM when half the tensor memory and half the shared memory
  // (of the B200's 228 KB per SM, less 1 KB per CTA) hold a CTA with at least
  // two stages: the two MMA-issuing loops then overlap.  The registers allow
  // it (launch bounds).  Otherwise one CTA per SM with all the shared memory.
  const uint32_t limit = (uint32_t)tc_smem_limit();
  constexpr uint32_t kPairSmem = 233472u / 2u - 1024u;
  const bool pair = P.tmem_cols <= 256u && kPairSmem >= extra + 2u * stage_bytes;
  const uint32_t budget = pair ? std::min(limit, kPairSmem) : limit;
  P.stages = (int)std::min<uint32_t>(kMaxStages, (budget - extra) / stage_bytes);
  if (P.stages < 2) return fail(WAL_ERR_UNSUPPORTED, "tensor-core tile does not fit in shared memory");
  P.smem = extra + (uint32_t)P.stages * stage_bytes;
  P.per_sm = pair ? 2 : 1;
  // K splits: with few row tiles, split K so the grid fills the SMs.  Cost
  // model in microseconds: waves x (K-blocks per split + about 4 of fixed
  // work) x about 1 us per K-block, plus the split sums' traffic (ks partial
  // planes read, one written) at about 3 TB/s.  The B200's 148 SMs are a
  // constant here so the plan (and the workspace size) do not depend on
  // device queries.
  const int G = m->K / 128, tiles = P.n_tiles_n * P.n_mt;
  constexpr int kPlanSms = 148;
  double best = 1e30;
  P.ks = 1;
  P.gps = G;
  for (int ks = 1; ks <= std::min(G, 16); ++ks) {
    const int gps = (G + ks - 1) / ks, eff = (G + gps - 1) / gps;
    if (eff != ks) continue;
    const int waves = (tiles * ks + kPlanSms * P.per_sm - 1) / (kPlanSms * P.per_sm);
    const double reduce_us = ks > 1 ? (double)(ks + 1) * M * m->N * 4.0 / 3.0e6 : 0.0;
    const double est = (double)waves * (2.0 * gps + 4.0) + reduce_us;
    if (est < best - 1e-9) {
      best = est;
      P.ks = ks;
      P.gps = gps;
    }
  }
  P.off_scal = 0;
  P.off_zt = align_up(256 + (size_t)P.M_pad * 8, 1024);
  P.off_xt = align_up(P.off_zt + (m->r > 0 ? (size_t)P.n_mt * b_bytes : 0), 1024);
  P.off_part = align_up(P.off_xt + (size_t)P.M_pad * m->K * 2, 1024);
  P.total = P.off_part + (P.ks > 1 ? (size_t)P.ks * M * m->N * 4 : 0);
  *out = P;
  return WAL_OK;
}

size_t tc_ws_bytes(const wal_matrix* m, int M) {
  TcPlan P;
  if (plan_tc(m, M, &P) != WAL_OK) return 0;
  return 256 /*alignment slack*/ + 256 /*header*/ + P.total;
}

int launch_tc(const wal_matrix* m, const uint16_t* X, int M, int ldx, float* Y, int ldy, char* ws,
              cudaStream_t stream) {
  int st = tc_init();
  if (st) return st;
  TcPlan P;
  st = plan_tc(m, M, &P);
  if (st) return st;
  int32_t* status = reinterpret_cast<int32_t*>(ws);
  char* data = ws + 256;  // header occupies the first 256 bytes
  TcPrepParams pp;
  pp.X = X; pp.ldx = ldx; pp.M = M; pp.K = m->K; pp.r = m->r; pp.M_tile = P.M_tile;
  pp.vbits = m->v_bits;
  pp.xt = data + P.off_xt;
  pp.zt = data + P.off_zt;
  pp.scal = reinterpret_cast<float2*>(data + P.off_scal);
  pp.status = status;
  const size_t vbytes = (size_t)m->r * (m->K / 8);  // <= 32 * 24576 / 8 = 96 KB
  tc_prep_kernel<<<P.M_pad, kPrepThreads, vbytes, stream>>>(pp);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return fail(WAL_ERR_CUDA, std::string("tc_prep_kernel launch: ") + cudaGetErrorString(e));

  TcParams tp;
  tp.codes = m->codes; tp.sites = m->sites; tp.scales = m->scales; tp.ubits = m->u_bits; tp.lr = m->lr_scale;
  tp.xt = pp.xt; tp.zt = pp.zt; tp.scal = pp.scal;
  tp.Y = Y; tp.ldy = ldy; tp.N = m->N; tp.K = m->K; tp.r = m->r; tp.M = M; tp.M_tile = P.M_tile;
  tp.stages = P.stages; tp.n_tiles_n = P.n_tiles_n;
  tp.ks = P.ks; tp.gps = P.gps;
  tp.part = reinterpret_cast<float*>(data + P.off_part);
  tp.d2_col = m->r > 0 ? P.tmem_cols / 2 : P.tmem_cols;
  tp.tmem_cols = P.tmem_cols;
  tp.status = status;
  // programmatic dependent launch: the product launch starts while the prep
  // launch runs; its B producer and epilogue wait for the prep grid
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(P.n_tiles_n * P.ks * P.n_mt);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = P.smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  switch (m->k) {
    case 0: e = cudaLaunchKernelEx(&cfg, tc_kernel<0>, tp); break;
    case 2: e = cudaLaunchKernelEx(&cfg, tc_kernel<2>, tp); break;
    case 4: e = cudaLaunchKernelEx(&cfg, tc_kernel<4>, tp); break;
    default: e = cudaLaunchKernelEx(&cfg, tc_kernel<8>, tp); break;
  }
  if (e == cudaSuccess) e = cudaGetLastError();
  if (e != cudaSuccess) return fail(WAL_ERR_CUDA, std::string("tc_kernel launch: ") + cudaGetErrorString(e));
  if (P.ks > 1) {
    const size_t total = (size_t)M * m->N;
    const int blocks = (int)std::min<size_t>((total + 255) / 256, 148 * 8);
    cudaLaunchConfig_t rc = {};
    rc.gridDim = dim3(blocks);
    rc.blockDim = dim3(256);
    rc.stream = stream;
    rc.attrs = attr;
    rc.numAttrs = 1;
    e = cudaLaunchKernelEx(&rc, tc_reduce_kernel, (const float*)tp.part, (const float2*)tp.scal, Y, ldy, M, m->N,
                           P.ks);
    if (e == cudaSuccess) e = cudaGetLastError();
    if (e != cudaSuccess) return fail(WAL_ERR_CUDA, std::string("tc_reduce_kernel launch: ") + cudaGetErrorString(e));
  }
  return WAL_OK;
}

}  // namespace wal
