/*
 * losa.h - C ABI of the LoSA retained-mass block-sparse attention library
 * (B200, sm_100a).
 *
 * The method (LoSA: Near-Lossless Sparse Attention for Training-Free Video
 * Diffusion Acceleration, arXiv 2608.12032) runs in three phases, and each
 * phase is one call here:
 *
 *   losa_dense_mass   one early dense attention step that also measures the
 *                     exact attention mass of every (head, query block, key
 *                     block) pair (ubos.tech LoSA post, "How It Works in
 *                     Practice", Phase 1 - Dense Calibration; LoSA abstract:
 *                     "measures exact block attention masses at one early
 *                     dense step").
 *   losa_select       per head and query block, the smallest key-block set
 *                     whose cumulative mass reaches tau (Phase 2 - Block
 *                     Mask Generation; legiblepapers.com LoSA page, "Summary
 *                     & Methodology Analysis": default tau = 0.99), frozen
 *                     into a CSR pattern the library owns.
 *   losa_dense_mass_select  the first two phases in one call, the per-row
 *                     cut fused into the construction kernel.
 *   losa_sparse_attn  every later step: attention of fresh Q/K/V over the
 *                     frozen retained key blocks only (Phase 3 - Repeated
 *                     Sparse Inference; legiblepapers.com: Q, K, V are
 *                     recomputed, the indices are not).
 *   losa_free         releases a pattern.
 *
 * Conventions shared by every call:
 *   - Tensors are caller-owned DEVICE memory on the current CUDA device,
 *     contiguous, row-major. Q, K, V, O are [B, H, L_pad, d]; lse is
 *     [B, H, L_pad]; the mass map is [B, H, n, n] with n = L_pad / block.
 *     Base pointers of Q, K, V must be 16-byte aligned.
 *   - Token rows i >= L are padding: keys there take no weight, and query
 *     rows there get O = 0 and lse = -inf and are left out of the masses.
 *     L_pad must be a multiple of the block size, and L_pad - L < block.
 *   - Attention is bidirectional: softmax(scale * q k^T) over the valid keys.
 *   - `stream` is a cudaStream_t (NULL = legacy default stream). Calls are
 *     stream-ordered and return without a host synchronisation, except
 *     losa_select and losa_dense_mass_select (one synchronisation, to size
 *     the CSR),
 *     losa_pattern_export / losa_pattern_import (they finish their copies
 *     before returning) and losa_check_status.
 *   - Every call returns LOSA_OK (0) or a negative losa_status; it checks
 *     its arguments on the host before touching the device and then leaves
 *     outputs untouched on LOSA_ERR_ARG.
 *   - Supported: d in {64, 128}; block in {32, 64, 128}; n <= 2047;
 *     B*H <= 65535; an sm_100 device.
 *   - The library keeps no global state besides, per device, one status
 *     word (set by a kernel that ran out of a bounded wait, or by a bad mass
 *     value), one stream-ordered memory pool (patterns and scratch), the
 *     fixed scratch array of losa_select_noalloc, and its CUDA function
 *     handles; and, per process, the wait limit of losa_set_wait_limit.
 *     Calls on different streams are independent, except that overlapping
 *     losa_select_noalloc calls share that scratch array.
 */
#ifndef LOSA_H_
#define LOSA_H_

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  LOSA_BF16 = 0, /* bfloat16: the attention runs on kind::f16 tensor cores
                    (bf16 operands, bf16 weights P, fp32 accumulation) */
  LOSA_FP32 = 1  /* float32: inputs are rounded to tf32 (nearest even, 10
                    mantissa bits) on entry into pool temporaries and the
                    attention runs on kind::tf32 tensor cores (the weights P
                    stay fp32 and are read as tf32); as an output dtype,
                    float32 */
} losa_dtype;

typedef enum {
  LOSA_OK = 0,
  LOSA_ERR_ARG = -1,         /* bad argument: shape, dtype, null pointer, tau */
  LOSA_ERR_CUDA = -2,        /* a CUDA runtime call failed */
  LOSA_ERR_NOMEM = -3,       /* device allocation failed */
  LOSA_ERR_TIMEOUT = -4,     /* a kernel gave up a bounded wait (see losa_check_status) */
  LOSA_ERR_MASS = -5,        /* a mass entry is NaN, Inf, negative or >= 2 */
  LOSA_ERR_UNSUPPORTED = -6  /* the current device is not sm_100 */
} losa_status;

/* A frozen block pattern: opaque, owned by the library, freed by losa_free. */
typedef struct losa_pattern losa_pattern;

/* Read-only view of a pattern. All pointers are DEVICE pointers owned by the
 * pattern and valid until losa_free. Rows are ordered (b, h, I) row-major,
 * R = B*H*n rows. */
typedef struct {
  int B, H, n_blocks, block;
  int64_t nnz;                 /* retained (query block, key block) pairs */
  const int32_t* row_ptr;      /* [R + 1], row_ptr[0] = 0, row_ptr[R] = nnz */
  const int32_t* col_idx;      /* [nnz], ascending key-block index within a row */
  const int64_t* retained_fx;  /* [R], sum of the kept fixed-point masses */
  const int64_t* total_fx;     /* [R], sum of all fixed-point masses of the row */
  /* Work list of the sparse kernel: 128-query-row tiles (128/block query
   * blocks each). A tile's entries are the union of its query blocks'
   * retained key blocks, ascending; entry = J | (m << 16), bit q of m set
   * when the tile's q-th query block keeps key block J. */
  int64_t n_tiles;
  int64_t tile_entries;
  const int32_t* tile_ptr;     /* [n_tiles + 1] */
  const int32_t* tile_entry;   /* [tile_entries] */
  const int32_t* tile_order;   /* [n_tiles], tiles by entry count, largest first */
} losa_pattern_view;

/*
 * losa_dense_mass - construction step: dense attention plus the exact block
 * attention mass (Phase 1 - Dense Calibration, ubos.tech LoSA post; LoSA
 * abstract).
 *
 *   q, k, v    [B, H, L_pad, d] device, dtype in_dtype (LOSA_FP32 takes
 *              the tf32 path: see losa_dtype).
 *   o          [B, H, L_pad, d] device, dtype out_dtype:
 *              O = softmax(scale * Q K^T over keys j < L) V.
 *   lse        [B, H, L_pad] fp32 device: lse_i = log sum_{j<L} exp(scale q_i.k_j).
 *   mass       [B, H, n, n] fp32 device, n = L_pad / block:
 *              mass[b,h,I,J] = (1/|I|) sum_{i in I, i<L} sum_{j in J}
 *                              exp(scale q_i.k_j - lse_i),
 *              |I| = valid query rows of block I; each row sums to 1.
 *   One kernel with two passes over the key tiles: a flash forward that
 *   leaves O and lse, then a recompute of Q K^T that sums exp(s - lse) into
 *   the block masses. o, lse and mass must not alias the inputs.
 *   Returns LOSA_ERR_ARG for: a null pointer, B, H < 1, L < 1, L > L_pad,
 *   L_pad % block != 0, L_pad - L >= block, d not in {64, 128}, block not in
 *   {32, 64, 128}, n > 2047, B*H > 65535, a dtype out of range, scale not
 *   finite and > 0.
 */
int losa_dense_mass(const void* q, const void* k, const void* v, int in_dtype,
                    int B, int H, int L, int L_pad, int d, int block, float scale,
                    void* o, int out_dtype, float* lse, float* mass, void* stream);

/*
 * losa_select - smallest key-block set per (b, h, query block) whose
 * cumulative mass reaches tau (Phase 2 - Block Mask Generation; LoSA
 * abstract; legiblepapers.com FAQ Q4).
 *
 *   mass      [B, H, n, n] fp32 device (as written by losa_dense_mass).
 *   tau       in (0, 1]; the method's default is 0.99.
 *   out       receives a new pattern on LOSA_OK, else NULL.
 *
 *   Per row: x_J = round(mass_J * 2^48) as int64 (ties to even); order the
 *   key blocks by (x desc, J asc); C_k = prefix sums; S = sum x; keep the
 *   first k >= 1 blocks with 2^48 * C_k >= round(tau * 2^48) * S, compared
 *   exactly in 128-bit integers. The kept set is stored ascending. Integer
 *   work throughout, so the result is bit-exact.
 *   Allocates the pattern (and its scratch) stream-ordered on `stream` from
 *   the library's own memory pool, and synchronises the stream once to learn
 *   the CSR size.
 *   Returns LOSA_ERR_ARG (null pointer, sizes, tau outside (0, 1]),
 *   LOSA_ERR_MASS (a mass entry NaN, Inf, < 0 or >= 2), LOSA_ERR_NOMEM,
 *   LOSA_ERR_CUDA.
 */
int losa_select(const float* mass, int B, int H, int n_blocks, int block, double tau,
                losa_pattern** out, void* stream);

/*
 * losa_dense_mass_select - losa_dense_mass and losa_select in one call, with
 * the selection's per-row cut run inside the construction kernel: a CTA of
 * that kernel computes every key block of its query blocks' mass rows, so
 * once its mass pass is over it sorts and cuts those rows itself (Phase 1
 * and Phase 2 of the ubos.tech LoSA post, "How It Works in Practice"; the
 * LoSA abstract's "smallest key/value block set" per head and query block).
 * The tile lists and the tile order are then built as losa_select builds
 * them.
 *
 *   Arguments as for losa_dense_mass (q, k, v, o, lse, mass and their
 *   dtypes, shapes, alignment) plus tau and out as for losa_select.
 *   o, lse and mass are written exactly as losa_dense_mass writes them, and
 *   the pattern is bit-identical to losa_select(mass, ..., tau) on that
 *   mass map (the same integer cut, run by one warpgroup per row instead
 *   of one CTA or warp per row).
 *   Synchronises the stream once (to size the CSR), like losa_select, and
 *   allocates from the library's pool on `stream`.
 *   Returns LOSA_ERR_ARG (as for losa_dense_mass, a null out, or tau outside
 *   (0, 1]), LOSA_ERR_NOMEM, LOSA_ERR_CUDA, LOSA_ERR_TIMEOUT (the
 *   construction kernel gave up a bounded wait; the status word is cleared
 *   and no pattern is returned), LOSA_ERR_UNSUPPORTED.
 */
int losa_dense_mass_select(const void* q, const void* k, const void* v, int in_dtype,
                           int B, int H, int L, int L_pad, int d, int block, float scale,
                           double tau, void* o, int out_dtype, float* lse, float* mass,
                           losa_pattern** out, void* stream);

/* Fills *view from a pattern. Returns LOSA_ERR_ARG on NULL. */
int losa_pattern_info(const losa_pattern* p, losa_pattern_view* view);

/*
 * losa_pattern_export - copies the pattern's arrays into caller buffers
 * (host or device memory; cudaMemcpyDefault) so a frozen pattern can be
 * stored for reuse (ubos.tech LoSA post, Phase 2: the mask "is stored for
 * reuse"). Any destination may be NULL to skip it; sizes are those of
 * losa_pattern_view. The copies are ordered on `stream`; the call
 * synchronises the stream before returning, so host buffers are filled.
 */
int losa_pattern_export(const losa_pattern* p, int32_t* row_ptr, int32_t* col_idx,
                        int64_t* retained_fx, int64_t* total_fx, int32_t* tile_ptr,
                        int32_t* tile_entry, int32_t* tile_order, void* stream);

/*
 * losa_pattern_import - rebuilds a pattern from a stored CSR, the inverse of
 * losa_pattern_export (ubos.tech LoSA post, Phase 2: the mask "is stored
 * for reuse"), so a frozen pattern can outlive the process that selected it
 * or come from elsewhere.
 *
 *   row_ptr      [B*H*n_blocks + 1] int32, HOST memory; row r = (b*H + h)*n
 *                + I lists query block I's kept key blocks.
 *   col_idx      [row_ptr[last]] int32, HOST memory.
 *   retained_fx, total_fx
 *                [B*H*n_blocks] int64 HOST memory or NULL; copied into the
 *                pattern as given, or set to -1 (unknown) when NULL.
 *   out          receives a new pattern on LOSA_OK, else NULL.
 *
 *   The CSR is checked on the host before any device work: row_ptr[0] = 0,
 *   every row holds 1..n_blocks entries, and each row's columns are strictly
 *   ascending in [0, n_blocks) (as losa_select writes them). The sparse
 *   kernel's tile lists are then rebuilt on the device from the CSR; a
 *   pattern exported from losa_select and imported again gives the same
 *   row_ptr, col_idx, tile_ptr and tile_entry, and tile_order up to the order
 *   of tiles with equal keys. The host arrays are read before the call
 *   returns (it synchronises `stream`) and stay the caller's.
 *   Returns LOSA_ERR_ARG (null pointer, sizes as for losa_select, an invalid
 *   CSR), LOSA_ERR_NOMEM, LOSA_ERR_CUDA, LOSA_ERR_UNSUPPORTED.
 */
int losa_pattern_import(const int32_t* row_ptr, const int32_t* col_idx,
                        const int64_t* retained_fx, const int64_t* total_fx, int B, int H,
                        int n_blocks, int block, losa_pattern** out, void* stream);

/*
 * losa_sparse_attn - later steps: attention of fresh Q/K/V restricted to the
 * frozen retained key blocks (Phase 3 - Repeated Sparse Inference, ubos.tech
 * LoSA post; legiblepapers.com "Summary & Methodology Analysis").
 *
 *   q, k, v   [B, H, L_pad, d] device, L_pad = p->n_blocks * p->block.
 *   o         [B, H, L_pad, d], out_dtype: for i in query block I,
 *             O_i = sum_{j in R(I), j<L} softmax_j(scale q_i.k_j) v_j with the
 *             softmax renormalised over the retained keys R(I) only.
 *   lse       [B, H, L_pad] fp32, may be NULL: log-sum-exp over the retained keys.
 *   Returns LOSA_ERR_ARG for a null pointer, a bad dtype, d not in {64, 128},
 *   L < 1, L > L_pad, L_pad - L >= block, or a current device other than the
 *   one the pattern was built on.
 */
int losa_sparse_attn(const void* q, const void* k, const void* v, int in_dtype, int d,
                     int L, float scale, const losa_pattern* p,
                     void* o, int out_dtype, float* lse, void* stream);

/* Largest B*H*n_blocks that losa_select_noalloc accepts. */
#define LOSA_NOALLOC_MAX_ROWS 65536

/*
 * losa_select_noalloc - the same selection as losa_select, for callers that
 * cannot allocate device memory, written straight into buffers the caller
 * owns. The LoSA pages have no counterpart to this call; it exists for
 * callers such as serving engines that reserve all device memory at
 * start-up and forbid allocation while requests run, code that lives inside
 * another framework's allocator, and latency-critical loops that cannot
 * afford cudaMalloc's implicit device synchronisation.
 *
 *   mass         [B, H, n, n] fp32 device.
 *   row_ptr      [R + 1] int32 device, R = B*H*n: CSR row offsets
 *                (row_ptr[R] = number of kept blocks).
 *   col_idx      [col_capacity] int32 device: kept key blocks, ascending
 *                per row. Entries at offsets >= col_capacity are dropped;
 *                col_capacity >= R*n always suffices. Compare row_ptr[R]
 *                with col_capacity to see whether everything fit.
 *   retained_fx, total_fx  [R] int64 device, as in losa_pattern_view.
 *
 * It allocates nothing: its scratch (one 64-bit cut key and one count per
 * row, 768 KB in all) is a fixed array inside the library that every GPU
 * which loads the library holds until the process exits. Hence R must not
 * exceed LOSA_NOALLOC_MAX_ROWS (LOSA_ERR_ARG otherwise). Every call shares
 * that array, so calls that overlap on the GPU (on different streams, or
 * from different threads) race and must be serialised by the caller. The
 * first call on a device looks up the array's device address; make that
 * first call before any stream capture. The call does not synchronise, so a
 * bad mass value (NaN, Inf, negative or >= 2) cannot be returned: it raises
 * the device status word, which the caller reads and clears with
 * losa_check_status (LOSA_ERR_MASS) after the call. Until it is cleared, the
 * next losa_select on that device reports LOSA_ERR_MASS too, whatever its
 * own input, so check the status before the next losa_select.
 * Returns LOSA_OK, LOSA_ERR_ARG (null pointer, sizes, tau outside (0, 1],
 * col_capacity < 0), LOSA_ERR_UNSUPPORTED (not an sm_100 device) or
 * LOSA_ERR_CUDA.
 */
int losa_select_noalloc(const float* mass, int B, int H, int n_blocks, double tau,
                        int32_t* row_ptr, int32_t* col_idx, int64_t col_capacity,
                        int64_t* retained_fx, int64_t* total_fx, void* stream);

/* Frees a pattern. The memory returns to the library's pool in stream order
 * on the stream the pattern was built on, so work on that stream that uses
 * the pattern may still be in flight; work on OTHER streams that uses it must
 * be complete (or ordered before that stream) first. NULL is a no-op. */
void losa_free(losa_pattern* p);

/*
 * losa_check_status - synchronises `stream`, then reads and clears the
 * device status word of the current device. Returns LOSA_ERR_TIMEOUT when a
 * kernel since the last check gave up a bounded wait (its outputs are then
 * undefined), LOSA_ERR_MASS when a losa_select_noalloc call since the last
 * check met a bad mass value (its outputs are then undefined), else LOSA_OK
 * or LOSA_ERR_CUDA. The word records the first event only.
 */
int losa_check_status(void* stream);

/*
 * losa_set_wait_limit - diagnostic of the attention kernels' failure path:
 * sets, for the whole process, how many SM cycles a wait inside the
 * attention kernels spins before it gives up (1 <= limit_cycles <= 2^33),
 * or restores the default (about 2 s at the B200's clock) when limit_cycles
 * is 0. It applies to the losa_dense_mass and losa_sparse_attn launches made
 * after the call. A kernel whose wait runs out records LOSA_ERR_TIMEOUT in
 * the device status word, and every warp of the CTA then leaves its loop,
 * lets the copies and MMAs it issued finish, frees its tensor memory and
 * returns, so the CUDA context stays usable. With a limit of a few cycles a
 * launch times out on purpose (its outputs are then undefined). Not for use
 * while other threads launch. Returns LOSA_ERR_ARG for a limit out of range.
 */
int losa_set_wait_limit(int64_t limit_cycles);

/*
 * losa_selftest_wait - diagnostic of the failure path every kernel uses:
 * launches one wait on a barrier that nothing completes. The wait gives up
 * after limit_cycles SM cycles (0 < limit_cycles <= 2^33), records a
 * timeout in the device status word and the kernel returns normally, so the
 * CUDA context stays usable; the next losa_check_status on that stream
 * returns LOSA_ERR_TIMEOUT and clears the word. Returns LOSA_ERR_ARG for a
 * limit out of range.
 */
int losa_selftest_wait(int64_t limit_cycles, void* stream);

/*
 * losa_exp2_eval - diagnostic: y[i] = 2^x[i] computed with the FMA-pipe
 * exponential the attention kernels use for part of their softmax
 * exponentials (Cody-Waite range reduction and a degree-5 minimax
 * polynomial; relative error below 4e-7 for x in [-125, 127]; x below -125
 * gives a value under 3e-38). x, y: n fp32 device values. Stream-ordered.
 * Returns LOSA_ERR_ARG for null pointers or n < 0.
 */
int losa_exp2_eval(const float* x, float* y, int64_t n, void* stream);

/* Short English text for a status code. Never NULL. */
const char* losa_strerror(int status);

/* Library version, "major.minor.patch". */
const char* losa_version(void);

#ifdef __cplusplus
}
#endif

#endif /* LOSA_H_ */
