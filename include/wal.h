/* wal.h -- C ABI of libwal.so: the direct-packed body-matrix product on B200.
 *
 *   y = (alpha * T + beta * R) x + sum_r s_r U_r (V_r^T x)
 *
 * The product, its parts and their names follow the WAL-Ternary-8B model card
 * (section "Representation"; the Kazakh README, section "Model format", prints
 * the same formula):
 *   T      ternary base, T in {-1, 0, +1}, stored as packed 2-bit codes
 *          (32 bytes per 128 weights with three of four codes used, like PQ2_0
 *          on the WAL2-Ternary-27B card, section on bit widths);
 *   R      exactly k signed residual sites per group of 128 weights, k in
 *          {0, 2, 4, 8} (WAL-Ternary-27B-RC1 card, "Representation": k0/k2/k4/k8);
 *   alpha, beta  FP16 scales per (output row, 128-group) (WAL-Ternary-8B card,
 *          "Install": the cache keeps FP16 scales; the 128-weight scale group
 *          is the WAL2-Ternary-27B card's, "Архитектура");
 *   U, V   the WALB2 binary low-rank pair, entries +-1, with one FP16 scale per
 *          rank (WAL-Ternary-8B card, "Representation": packed binary low-rank
 *          WALB2 correction).
 *
 * Layout v1 (the byte format every entry point reads), N outputs, K inputs,
 * G = K / 128 groups, k sites per group, rank r:
 *   codes    uint32[N][K/16]   trit j of row n in word j/16, bits 2*(j%16)..+1;
 *                              code c = t + 1 (0 -> -1, 1 -> 0, 2 -> +1), 3 reserved
 *   sites    uint8 [N][G][k]   byte = position in group (bits 0..6) | 0x80 if the
 *                              site's sign is -1; positions distinct, ascending
 *   scales   uint16[N][G][2]   fp16 bits {alpha, beta} when k > 0;
 *            uint16[N][G]      fp16 bits alpha when k == 0
 *   u_bits   uint32[N][ceil(r/32)]  bit (rho % 32) of word rho/32 set <=> U[n][rho] = -1
 *   v_bits   uint32[r][K/32]   bit (j % 32) of word j/32 set <=> V[j][rho] = -1
 *   lr_scale uint16[r]         fp16 bits of s_rho
 * Each buffer spans the size wal_packed_sizes returns (its payload rounded
 * up to a multiple of 16 bytes) and its padding bytes are zero: the kernels
 * read whole aligned 16-byte words of every buffer.
 * Activations are bf16 bit patterns, row-major X[M][ldx]; outputs are fp32,
 * row-major Y[M][ldy], overwritten (never accumulated into).
 *
 * Conventions for every entry point:
 *   - Ownership: the caller owns every buffer.  The library never allocates
 *     device memory; scratch comes from the caller as (ws, ws_bytes), sized by
 *     the matching *_workspace_bytes call.  Plans own only a CUDA graph.
 *   - Matrix buffers and activations must be 16-byte aligned, outputs 4-byte
 *     aligned; otherwise WAL_ERR_ARG.
 *   - Stream semantics: device work is enqueued on `stream` and returns at
 *     once; argument and shape errors are returned synchronously before any
 *     launch.  Launch failures return WAL_ERR_CUDA.  A bounded wait inside a
 *     kernel that gives up records WAL_ERR_TIMEOUT in the workspace header,
 *     which wal_device_status() reads.
 *   - No exceptions and no aborts cross the ABI.  wal_last_error() returns a
 *     thread-local text for the last non-OK status of the calling thread.
 *   - There is no CPU fallback: every device entry point runs CUDA kernels
 *     built for sm_100a and fails with WAL_ERR_CUDA when no such device exists.
 */
#ifndef WAL_H
#define WAL_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same object as cudaStream_t; NULL means the legacy default stream. */
typedef struct CUstream_st* wal_stream_t;

enum {
  WAL_OK = 0,
  WAL_ERR_ARG = -1,         /* null / misaligned pointer, bad count */
  WAL_ERR_SHAPE = -2,       /* K % 128 != 0, k not in {0,2,4,8}, r > 32, N <= 0, M out of range */
  WAL_ERR_FORMAT = -3,      /* buffer content violates layout v1 */
  WAL_ERR_WORKSPACE = -4,   /* ws_bytes smaller than required */
  WAL_ERR_CUDA = -5,        /* a CUDA runtime call failed */
  WAL_ERR_UNSUPPORTED = -6, /* valid but not handled by this build */
  WAL_ERR_TIMEOUT = -7      /* a bounded device wait gave up */
};

#define WAL_MAX_RANK 32
#define WAL_MAX_SMALL_M 16

/* One packed matrix.  All pointers are device pointers into caller-owned
 * buffers laid out as described above; `sites` may be NULL when k == 0 and
 * `u_bits`, `v_bits`, `lr_scale` may be NULL when r == 0. */
typedef struct wal_matrix {
  int32_t N, K, k, r;
  const uint32_t* codes;
  const uint8_t* sites;
  const uint16_t* scales;
  const uint32_t* u_bits;
  const uint32_t* v_bits;
  const uint16_t* lr_scale;
} wal_matrix;

/* Byte sizes of the six layout-v1 buffers, in the order codes, sites, scales,
 * u_bits, v_bits, lr_scale.  Host only.  WAL_ERR_SHAPE on a bad shape. */
int wal_packed_sizes(int N, int K, int k, int r, size_t out_bytes[6]);

/* Pack dense components (host arrays) into the six layout-v1 buffers (host
 * memory, sizes from wal_packed_sizes).  Inputs:
 *   T [N][K] int8 in {-1,0,1}; site_pos [N][G][k] uint8 < 128, strictly
 *   ascending per group; site_sign [N][G][k] int8 +-1; alpha, beta [N][G]
 *   fp16 bits (beta ignored and may be NULL when k == 0); U [N][r] and
 *   V [K][r] int8 +-1; lr_scale [r] fp16 bits.
 * Host only, multi-threaded.  WAL_ERR_FORMAT on any out-of-range value;
 * nothing is guaranteed about out[] then. */
int wal_pack_matrix(const int8_t* T, const uint8_t* site_pos, const int8_t* site_sign,
                    const uint16_t* alpha, const uint16_t* beta, const int8_t* U,
                    const int8_t* V, const uint16_t* lr_scale, int N, int K, int k, int r,
                    void* const out[6]);

/* Scan a packed matrix on the device for layout-v1 violations (reserved code
 * 3, site positions not strictly ascending).  Synchronises `stream`.
 * Returns WAL_OK or WAL_ERR_FORMAT (wal_last_error names the first kind found).
 * ws must hold at least 256 bytes. */
int wal_validate(const wal_matrix* m, void* ws, size_t ws_bytes, wal_stream_t stream);

/* Test entry point: decode a packed matrix on the device into dense device
 * arrays with the same decode routines the product kernels use.
 *   T [N][K] int8; site_pos, site_sign [N][G][k]; alpha, beta [N][G] fp16 bits
 *   (beta zero-filled when k == 0); U [N][r] int8; V [K][r] int8.
 * Any output pointer may be NULL to skip it.  Asynchronous. */
int wal_unpack_matrix(const wal_matrix* m, int8_t* T, uint8_t* site_pos, int8_t* site_sign,
                      uint16_t* alpha, uint16_t* beta, int8_t* U, int8_t* V,
                      wal_stream_t stream);

/* Scratch bytes wal_gemv (M = 1) / wal_gemm_small_m (any M) need: the
 * 256-byte header for M <= 4, the tensor path's X image, WALB2 operand and
 * split sums from M = 5 on. */
size_t wal_workspace_bytes(const wal_matrix* m, int M);

/* y[N] = W x for one bf16 activation x[K] (batch 1): the decode-GEMV.
 * Streams the packed planes once, FP32 output. */
int wal_gemv(const wal_matrix* m, const uint16_t* x, float* y, void* ws, size_t ws_bytes,
             wal_stream_t stream);

/* Y[M][ldy] = X[M][ldx] W^T for 1 <= M.  M <= 4 runs the CUDA-core
 * decode-GEMV, one product per activation row in one launch; M >= 5 runs the
 * tensor-core path (bulk copies + tcgen05), which decodes each weight once for
 * up to 256 rows.  ldx >= K and a multiple of 8; ldy >= N. */
int wal_gemm_small_m(const wal_matrix* m, const uint16_t* X, int M, int ldx, float* Y, int ldy,
                     void* ws, size_t ws_bytes, wal_stream_t stream);

/* Y[M][ldy] = X[M][ldx] W^T on the tensor-core path (M >= 5) without a
 * workspace argument.  The model cards have no counterpart to this entry
 * point: it exists for callers that cannot hand the library scratch memory.
 * Its scratch is a fixed array of WAL_NOALLOC_SCRATCH_BYTES in the library's
 * own device memory (one per device; its address is looked up on every call,
 * so it always belongs to the current device and context); a call whose
 * scratch need, wal_workspace_bytes(m, M), is larger returns
 * WAL_ERR_WORKSPACE, and M < 5 returns WAL_ERR_SHAPE.  Nothing is allocated.
 * Every call on a device uses the same array, so calls that overlap in time
 * on one device (other streams, other host threads) race on it: the caller
 * must order them.  Asynchronous on `stream`.  A bounded device wait that
 * gives up is recorded in the array's status word: wal_noalloc_status reads
 * it. */
#define WAL_NOALLOC_SCRATCH_BYTES (16u << 20)
int wal_gemm_tc_noalloc(const wal_matrix* m, const uint16_t* X, int M, int ldx, float* Y, int ldy,
                        wal_stream_t stream);

/* Read and clear the status word of the current device's no-alloc scratch
 * (synchronises `stream`): WAL_OK, or WAL_ERR_TIMEOUT when a bounded device
 * wait of a wal_gemm_tc_noalloc call since the last read gave up.  Every
 * wal_gemm_tc_noalloc call clears the word when it starts. */
int wal_noalloc_status(wal_stream_t stream);

/* Read and clear the device status word in a workspace header (synchronises
 * `stream`).  Every product call clears the word when it starts, so it reports
 * on the last call that used this workspace.  WAL_OK, WAL_ERR_TIMEOUT, or
 * WAL_ERR_ARG for a token id outside the table (wal_int3_embed). */
int wal_device_status(void* ws, wal_stream_t stream);

/* Whole body pass: n_mats products, matrix i reading xs[i] (bf16 [M][K_i]) and
 * writing ys[i] (fp32 [M][N_i]).  stage_of[i] is the dependency stage of
 * matrix i: all matrices of stage s may run concurrently, and stage s + 1
 * starts only after every product of stage s has finished (a matrix of a
 * later stage may read an output of an earlier one).  Stages must be
 * non-decreasing along the array.  mats, stage_of, xs and ys are host arrays
 * (of device pointers).  1 <= M <= 16.
 * The first call builds *plan: launch tables (kept in ws) and a CUDA graph of
 * the pass on `stream` (a header clear plus one persistent cooperative launch
 * with a grid barrier between stages).  Later calls with identical arguments
 * replay it; a call whose arguments differ rebuilds it (synchronising
 * `stream` first).  ws belongs to the plan while the plan is in use: nothing
 * else may write it between calls.  wal_body_workspace_bytes gives its size.
 * A bounded wait that gives up records WAL_ERR_TIMEOUT in the ws header
 * (wal_device_status). */
typedef struct wal_body_plan wal_body_plan;
size_t wal_body_workspace_bytes(const wal_matrix* mats, int n_mats, int M);
int wal_body_pass(wal_body_plan** plan, const wal_matrix* mats, int n_mats,
                  const int32_t* stage_of, const uint16_t* const* xs, float* const* ys, int M,
                  void* ws, size_t ws_bytes, wal_stream_t stream);
void wal_body_plan_destroy(wal_body_plan* plan);

/* Fault injection for tests of the timeout path (host side only; no GPU fault
 * is involved).  While the setting is nonzero, body-pass plans built
 * afterwards (wal_body_pass, wal_pq2_body_pass, wal_rc1_body_pass) get grid
 * barrier targets that no CTA ever reaches and a 1 ms limit per barrier
 * wait.  Such a pass ends early: each CTA gives up at its first wait, stops
 * taking part, waits for its own copies in flight and exits, and
 * wal_device_status() then returns WAL_ERR_TIMEOUT.  Plans built while the
 * setting is zero are not affected.  Returns the previous setting. */
int wal_debug_barrier_fault(int on);

/* ---- PQ2_0: the plain-ternary block format ---------------------------------
 * The WAL2-Ternary-27B card (section on bit widths) describes PQ2_0, the
 * format of its fast native GGUF: 32 bytes of 2-bit codes plus a 2-byte FP16
 * scale for every 128 weights (34 bytes, 2.125 bits per weight), three of
 * the four codes in use.  W[n][128 g + j] = d[n][g] * T[n][128 g + j]: the
 * direct-packed product with k = 0 and r = 0, scale and codes side by side.
 * This library's reading of the block (the card does not give the order):
 *   block (n, g) at byte 34 * (n * G + g): uint16 fp16 bits d (little
 *   endian), then 32 code bytes, trit j of the block in code byte j / 4 at
 *   bits 2 * (j % 4), code c = t + 1 (3 reserved), as in layout v1.
 *   The buffer is zero-padded to a multiple of 16 bytes (wal_pq2_bytes).
 * The product streams it with its own specialisation of the decode-GEMV (no
 * site table, no low-rank term); decode errors are not checked at run time. */
typedef struct wal_pq2_matrix {
  int32_t N, K;              /* K a positive multiple of 128, at most 24576 */
  const uint8_t* blocks;     /* device pointer, 16-byte aligned */
} wal_pq2_matrix;

/* Bytes of a PQ2_0 buffer for an N x K matrix (34 * N * K / 128 rounded up
 * to 16); 0 on a bad shape.  Host only. */
size_t wal_pq2_bytes(int N, int K);

/* Pack T [N][K] int8 in {-1,0,1} and d [N][K/128] fp16 bits into the PQ2_0
 * buffer `out` (host memory, wal_pq2_bytes(N, K) bytes, padding zeroed).
 * Host only, multi-threaded.  WAL_ERR_FORMAT when T leaves {-1,0,1}. */
int wal_pq2_pack(const int8_t* T, const uint16_t* d, int N, int K, void* out);

/* Scratch bytes of wal_pq2_gemm (1 <= M <= 16); 0 on a bad argument. */
size_t wal_pq2_workspace_bytes(const wal_pq2_matrix* m, int M);

/* Y[M][ldy] = X[M][ldx] W^T for a PQ2_0 matrix, 1 <= M <= 16 (one product
 * per activation row in one launch; the batch-1 decode-GEMV).  X bf16 bits,
 * 16-byte aligned, ldx >= K and a multiple of 8; Y fp32, ldy >= N.
 * Asynchronous; a bounded wait that gives up records WAL_ERR_TIMEOUT in the
 * workspace header (wal_device_status). */
int wal_pq2_gemm(const wal_pq2_matrix* m, const uint16_t* X, int M, int ldx, float* Y, int ldy, void* ws,
                 size_t ws_bytes, wal_stream_t stream);

/* Body pass over PQ2_0 matrices: the same contract as wal_body_pass (stages,
 * plan, graph replay, workspace ownership), with every matrix in PQ2_0. */
size_t wal_pq2_body_workspace_bytes(const wal_pq2_matrix* mats, int n_mats, int M);
int wal_pq2_body_pass(wal_body_plan** plan, const wal_pq2_matrix* mats, int n_mats, const int32_t* stage_of,
                      const uint16_t* const* xs, float* const* ys, int M, void* ws, size_t ws_bytes,
                      wal_stream_t stream);

/* ---- the base-3 container and its conversion (the prepare step) -----------
 * The WAL2-Ternary-27B card (section on bit widths) keeps its canonical
 * ternary base five trits to a byte (8 / 5 = 1.6 bits per symbol) with a
 * BF16 scale per 128 weights.  This library's reading of the bytes: byte m
 * of a row holds trits 5m .. 5m + 4 as sum_i (t_i + 1) * 3^i (trit 5m + i is
 * digit i, least significant first); values 243..255 are invalid; each row
 * starts on a byte (ceil(K / 5) bytes per row, rows back to back); digits
 * past a row's last trit are 0; the buffer is zero-padded to 16 bytes.
 * Scales: bf16 bits [N][K/128]. */

/* Bytes of the base-3 buffer of an N x K matrix; 0 on a bad shape. */
size_t wal_base3_bytes(int N, int K);

/* Pack T [N][K] int8 in {-1,0,1} into the base-3 buffer `out` (host memory,
 * wal_base3_bytes(N, K) bytes, padding zeroed).  Host only, multi-threaded.
 * WAL_ERR_FORMAT when T leaves {-1,0,1}. */
int wal_base3_pack(const int8_t* T, int N, int K, void* out);

/* The prepare step on the GPU: base-3 bytes b3 and BF16 scales [N][K/128]
 * become the layout-v1 code plane `codes` (uint32 [N][K/16], code c = t + 1)
 * and the k = 0 scale plane `alpha` (fp16 bits [N][K/128], BF16 rounded to
 * nearest even; its 16-byte padding is zeroed).  All device pointers,
 * 16-byte aligned; output sizes as wal_packed_sizes(N, K, 0, r) gives for
 * buffers 0 and 2.  ws: at least 512 bytes.  Synchronises `stream` and
 * returns WAL_ERR_FORMAT when a byte is above 242, a digit past a row's end
 * is nonzero, or a scale is not finite or overflows FP16 (the outputs are
 * then incomplete). */
int wal_base3_convert(const uint8_t* b3, const uint16_t* scales_bf16, int N, int K, uint32_t* codes,
                      uint16_t* alpha, void* ws, size_t ws_bytes, wal_stream_t stream);

/* ---- RC1 storage: 24-bit float scales and two WALB2 paths ------------------
 * The WAL-Ternary-27B-RC1 card ("Representation") keeps the body scales in a
 * 24-bit float format that its prepared compute cache expands to FP32, and
 * WALB2 as two packed binary low-rank paths:
 *   W = alpha (x) T + beta (x) R + U1 diag(s1) V1^T + U2 diag(s2) V2^T.
 * This library's reading (the card's storage ABI is not among its pages):
 * a 24-bit float is the upper three bytes of an IEEE FP32, little endian;
 * alpha, beta, s1 and s2 use it; the canonical planes are
 *   scales24 uint8 [N][G][2][3] ({alpha, beta}) when k > 0, [N][G][3] when k = 0;
 *   u_p uint32 [N][ceil(r_p/32)], v_p uint32 [r_p][K/32] (set bit = -1),
 *   s_p uint8 [r_p][3];  r1 + r2 <= 32;
 * each zero-padded to 16 bytes (wal_rc1_sizes).  The prepared matrix is
 * layout v1 with FP32 in place of FP16: scales float {alpha, beta} [N][G]
 * (alpha [N][G] when k = 0), one rank block r = r1 + r2 with path 1's ranks
 * first, lr_scale float [r]. */
typedef struct wal_rc1_matrix {  /* a prepared RC1 matrix; device pointers, 16-byte aligned */
  int32_t N, K, k, r;
  const uint32_t* codes;         /* layout v1 code plane */
  const uint8_t* sites;          /* layout v1 site bytes (NULL when k == 0) */
  const float* scales;           /* FP32 {alpha, beta} [N][G], or alpha [N][G] when k == 0 */
  const uint32_t* u_bits;        /* [N][ceil(r/32)] */
  const uint32_t* v_bits;        /* [r][K/32] */
  const float* lr_scale;         /* FP32 [r] */
} wal_rc1_matrix;

/* Byte sizes of the canonical RC1 planes (scales24, u1, v1, s1, u2, v2, s2)
 * and of the prepared planes (scales32, u_bits, v_bits, lr32).  Host only.
 * WAL_ERR_SHAPE on a bad shape or r1 + r2 > 32. */
int wal_rc1_sizes(int N, int K, int k, int r1, int r2, size_t canonical[7], size_t prepared[4]);

/* The prepare step on the GPU: decode every 24-bit scale to FP32 and merge
 * the two paths into one rank block (U words: path 2's bits shifted up by
 * r1; V bit rows and per-rank scales concatenated, path 1 first).  Device
 * pointers, 16-byte aligned; a path with r_p = 0 may pass NULL buffers.  The
 * code plane and the site bytes are layout v1 already and are used as they
 * are.  Asynchronous. */
int wal_rc1_prepare(int N, int K, int k, const uint8_t* scales24, int r1, const uint32_t* u1, const uint32_t* v1,
                    const uint8_t* s1_24, int r2, const uint32_t* u2, const uint32_t* v2, const uint8_t* s2_24,
                    float* scales32, uint32_t* u_bits, uint32_t* v_bits, float* lr32, wal_stream_t stream);

/* Products of a prepared RC1 matrix, 1 <= M <= 16, with the same contract as
 * wal_gemm_small_m (the FP32-scale specialisation of the decode-GEMV), and
 * the body pass over prepared RC1 matrices with the contract of
 * wal_body_pass. */
size_t wal_rc1_workspace_bytes(const wal_rc1_matrix* m, int M);
int wal_rc1_gemm(const wal_rc1_matrix* m, const uint16_t* X, int M, int ldx, float* Y, int ldy, void* ws,
                 size_t ws_bytes, wal_stream_t stream);
size_t wal_rc1_body_workspace_bytes(const wal_rc1_matrix* mats, int n_mats, int M);
int wal_rc1_body_pass(wal_body_plan** plan, const wal_rc1_matrix* mats, int n_mats, const int32_t* stage_of,
                      const uint16_t* const* xs, float* const* ys, int M, void* ws, size_t ws_bytes,
                      wal_stream_t stream);

/* ---- around the body: INT3/g128 embedding, INT4/g128 LM head --------------
 * The WAL-Ternary-8B card (Kazakh README, "Model format") keeps the
 * embedding as INT3 and the LM head as INT4, both with groups of 128.  This
 * library's reading: w = d * q with an FP16 scale d per (row, 128 columns);
 * codes are offset binary, u = q + 8 (INT4, q in [-8, 7]) or u = q + 4
 * (INT3, q in [-4, 3]).  INT4 rows: K / 2 bytes, column 2i in the low nibble
 * of byte i.  INT3 rows: 48 bytes per group, code j of the group at bits
 * 3j .. 3j + 2 of its little-endian 384-bit string.  Scales fp16 [rows][K/128].
 * Every plane is zero-padded to a multiple of 16 bytes. */
typedef struct wal_int4_matrix {  /* device pointers, 16-byte aligned */
  int32_t N, K;                   /* K a positive multiple of 128, at most 24576 */
  const uint8_t* codes;           /* [N][K/2] */
  const uint16_t* scales;         /* fp16 [N][K/128] */
} wal_int4_matrix;
typedef struct wal_int3_table {   /* device pointers, 16-byte aligned */
  int32_t V, H;                   /* rows (vocabulary) and row length */
  const uint8_t* codes;           /* [V][H/128][48] */
  const uint16_t* scales;         /* fp16 [V][H/128] */
} wal_int3_table;

/* Plane sizes (codes, scales) in bytes.  Host only; WAL_ERR_SHAPE on a bad shape. */
int wal_int4_sizes(int N, int K, size_t out[2]);
int wal_int3_sizes(int V, int H, size_t out[2]);

/* Host packers: q int8 [rows][cols], d fp16 bits [rows][cols/128] into the
 * two planes (host memory of the wal_*_sizes sizes, padding zeroed).
 * WAL_ERR_FORMAT when a value leaves its range. */
int wal_int4_pack(const int8_t* q, const uint16_t* d, int N, int K, void* codes, void* scales);
int wal_int3_pack(const int8_t* q, const uint16_t* d, int V, int H, void* codes, void* scales);

/* LM head: Y[M][ldy] = X[M][ldx] W^T for 1 <= M <= 16 (logits, FP32), with
 * the contract of wal_gemm_small_m.  Runs the INT4 specialisation of the
 * decode-GEMV. */
size_t wal_int4_workspace_bytes(const wal_int4_matrix* m, int M);
int wal_int4_gemm(const wal_int4_matrix* m, const uint16_t* X, int M, int ldx, float* Y, int ldy, void* ws,
                  size_t ws_bytes, wal_stream_t stream);

/* Embedding gather: out[m][0..H) = d[ids[m]] * q[ids[m]] in FP32 (exact),
 * for M >= 1 token ids (int32, device memory).  out is device memory [M][H],
 * 16-byte aligned.  An id outside [0, V) gives a zero row and records
 * WAL_ERR_ARG in the workspace status word (wal_device_status); ws: at least
 * 512 bytes.  Asynchronous. */
int wal_int3_embed(const wal_int3_table* t, const int32_t* ids, int M, float* out, void* ws, size_t ws_bytes,
                   wal_stream_t stream);

const char* wal_status_string(int status);
const char* wal_last_error(void);

#ifdef __cplusplus
}
#endif

#endif /* WAL_H */
