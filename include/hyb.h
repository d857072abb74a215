/*
 * hyb.h -- C ABI of libhyb: tile-hybrid (dense | 2:4) weight GEMV for decode,
 * CUDA for NVIDIA B200 (sm_100a).
 *
 * What is computed
 * ----------------
 * A weight matrix W (n outputs x k inputs, row-major, bf16) is cut into
 * b1 x b2 tiles (b1 rows along n, b2 columns along k).  Every tile is either
 * dense or 2:4 sparse: in a 2:4 tile every group of four consecutive
 * elements along k keeps two.  ("PATCH: Learnable Tile-level Hybrid Sparsity
 * for LLMs", §2 Methodology, core mechanism; §1 Problem statement for 2:4.)
 * The kept values of a 2:4 group are stored at a fixed stride with a 4-bit
 * mask telling which columns they came from ("SparseDecoding: decoding-aware
 * pruning ...", authors' abstract: bitmask indexing, fixed-stride traversal).
 * An optional low-rank term adds U (V^T x) ("3BASiL: An Algorithmic
 * Framework for Sparse plus Low-Rank Compression of LLMs", §1: W ~ S + L).
 *
 *   Y[b][i] = sum_k W_hat[i][k] X[b][k]  (+ sum_j U[i][j] sum_k V[k][j] X[b][k])
 *
 * with W_hat the masked matrix, bf16 inputs and fp32 accumulation.
 *
 * Packed format (produced by hyb_pack)
 * ------------------------------------
 *  - Tiles are numbered row-major, t = tr * (k / b2) + tc; tile_map[t] is 1
 *    for a 2:4 tile and 0 for a dense tile.
 *  - val_off[t] / meta_off[t] (t = 0..num_tiles) are the element / byte
 *    offsets of tile t in vals / meta: a dense tile takes b1*b2 values and no
 *    meta, a 2:4 tile b1*b2/2 values and b1*b2/8 meta bytes.
 *  - Dense tile: b1 rows of b2 values.  2:4 tile: b1 rows of b2/2 values; the
 *    two kept values of group g of row i sit at i*(b2/2) + 2g and +1 in
 *    ascending column order; their mask is the nibble of meta byte
 *    i*(b2/8) + g/2 (low nibble for even g), bit j set iff column 4g+j kept.
 *  - Selection keeps the two largest |w| of each group (key = bits & 0x7FFF;
 *    ties go to the lower column; values are copied bit-exactly).
 *
 * Conventions
 * -----------
 *  - bf16 crosses the ABI as uint16_t bit patterns.  All data pointers are
 *    DEVICE pointers unless the argument name ends in _host.  The caller owns
 *    every buffer; the library never allocates or frees device memory and
 *    keeps no global mutable state except a per-device SM-count cache.
 *  - Every call is asynchronous on `stream` (0 = legacy default stream).
 *    Argument, shape and alignment checks are synchronous: a failing check
 *    returns a negative hyb_status and launches nothing.  A failed launch
 *    returns HYB_ERR_CUDA.  Problems only the device can see (a NaN weight,
 *    a tile_map byte other than 0/1) set a status word in the workspace, read
 *    and cleared by hyb_check_status.  No device code traps.
 *  - Workspaces: size them with the *_workspace_bytes queries and zero them
 *    once (hyb_workspace_init) before first use.  The library leaves them
 *    ready for the next call.  Two calls that run concurrently must not share
 *    a workspace.
 *  - X is [batch][k] bf16 with leading dimension ldx >= k; Y is [batch][n]
 *    (fp32 or bf16) with ldy >= n.  X and meta must be 16-byte aligned and
 *    ldx a multiple of 8 (rows of X 16-byte aligned); vals 32-byte aligned;
 *    Y aligned to its element size; workspaces 256-byte aligned.
 *  - Shapes: n % b1 == 0, k % b2 == 0, b2 % 8 == 0, (b1 * b2) % 128 == 0.
 *    Any batch 1..16.  Tiles of 64 or 128 rows by 64 or 128 columns run the
 *    tuned streaming kernel; other legal tilings (b2 = 8, 16, 24, ...) run a
 *    simpler one-warp-per-row CUDA kernel (never a CPU fallback).
 */
#ifndef HYB_H
#define HYB_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define HYB_API __attribute__((visibility("default")))
#else
#define HYB_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st *hyb_stream_t; /* same type as cudaStream_t */

typedef enum {
  HYB_OK = 0,
  HYB_ERR_INVALID_ARG = -1,  /* bad shape, null pointer, bad enum */
  HYB_ERR_UNSUPPORTED = -2,  /* valid request the library does not handle */
  HYB_ERR_ALIGNMENT = -3,    /* pointer or leading dimension misaligned */
  HYB_ERR_WORKSPACE = -4,    /* workspace null or smaller than required */
  HYB_ERR_CUDA = -5,         /* a CUDA runtime call failed */
  HYB_ERR_DEVICE_CHECK = -6, /* the device flagged bad data (see above) */
  HYB_ERR_TIMEOUT = -7       /* a bounded wait inside a kernel ran out (status bit 4);
                                that call's outputs are incomplete, the context is usable */
} hyb_status;

typedef enum { HYB_F32 = 0, HYB_BF16 = 1 } hyb_dtype;

/* A packed hybrid matrix; every pointer is a device pointer. */
typedef struct {
  int64_t n, k;          /* outputs, inputs */
  int32_t b1, b2;        /* tile rows (along n), tile columns (along k) */
  int64_t num_tiles;     /* (n / b1) * (k / b2) */
  const uint8_t *tile_map;  /* [num_tiles], 1 = 2:4 tile, 0 = dense tile */
  const uint16_t *vals;     /* packed values, bf16 bits */
  const uint8_t *meta;      /* packed 4-bit masks (never NULL: pass any valid
                               device byte when the map has no 2:4 tile) */
  const int64_t *val_off;   /* [num_tiles + 1] */
  const int64_t *meta_off;  /* [num_tiles + 1] */
  int64_t n_vals;           /* val_off[num_tiles], as given by hyb_packed_sizes */
  int64_t n_meta_bytes;     /* meta_off[num_tiles], as given by hyb_packed_sizes */
  const int64_t *plan;      /* optional, HOST memory (may be NULL): the work
                               split hyb_make_plan made for this matrix on this
                               device; saves the products their start-up search */
  int32_t plan_ctas;        /* the CTA count hyb_make_plan reported for plan */
} hyb_matrix;

/* Low-rank factors of y += U (V^T x): U is [n][rank] (row stride ldu),
 * V is [k][rank] (row stride ldv), bf16, device pointers.  rank 1..256. */
typedef struct {
  int32_t rank;
  const uint16_t *U;
  int64_t ldu;
  const uint16_t *V;
  int64_t ldv;
} hyb_lowrank;

/* ---- format ----------------------------------------------------------- */

/* Host-only: number of packed values and meta bytes for a tile map held in
 * HOST memory (PATCH §2: dense tiles keep b1*b2 values, 2:4 tiles half of
 * them plus one 4-bit mask per group).  Rejects map bytes other than 0/1. */
HYB_API int hyb_packed_sizes(int64_t n, int64_t k, int b1, int b2,
                     const uint8_t *tile_map_host, int64_t *n_vals,
                     int64_t *n_meta_bytes);

/* Workspace bytes hyb_pack needs (status word only). */
HYB_API size_t hyb_pack_workspace_bytes(void);

/* Pack W ([n][k] bf16, row stride ldw, device) with the device tile_map into
 * vals / meta / val_off / meta_off (device buffers of the sizes given by
 * hyb_packed_sizes; offsets num_tiles + 1 entries each; meta never NULL, a
 * 1-byte buffer will do when the map has no 2:4 tile).  The selection rule
 * is the magnitude projection of 3BASiL §2A applied per 2:4 group (two
 * largest |w|, ties to the lower column).  A group holding a NaN, or a map
 * byte other than 0/1, sets the workspace status word; the pack still
 * completes deterministically.  W must be 16-byte aligned with ldw % 8 == 0. */
HYB_API int hyb_pack(int64_t n, int64_t k, int b1, int b2, const uint16_t *W,
             int64_t ldw, const uint8_t *tile_map, uint16_t *vals,
             uint8_t *meta, int64_t *val_off, int64_t *meta_off, void *ws,
             size_t ws_bytes, hyb_stream_t stream);

/* ---- work split -------------------------------------------------------- */

/* Entries (int64_t) of each of hyb_make_plan's two buffers on the current
 * device. */
HYB_API size_t hyb_plan_entries(void);

/* Work out, once per matrix, how the streaming kernel splits A's packed bytes
 * over its CTAs on the current device: CTA c takes the tiles whose packed byte
 * offset falls in [c, c+1) * total / G.  `scratch` is a device buffer and
 * `plan_host` a host buffer, both of hyb_plan_entries() int64_t; on return
 * plan_host holds, for every CTA, its first tile, the packed offsets of that
 * tile, the 2:4 bits of its first 31 tiles and the stage boundaries of that
 * first window (and one closing record with the tile count), and *plan_ctas
 * holds G (0 when the tiling has no streaming kernel).  Synchronises
 * `stream`.  Point A->plan / A->plan_ctas at the result: the products copy
 * it into the kernel's launch parameters and start streaming without any
 * global-memory load.  A plan whose CTA count differs from the one the
 * product would use, or whose ranges are malformed, is ignored (the kernel
 * then finds its range itself); results do not depend on whether a plan is
 * used. */
HYB_API int hyb_make_plan(const hyb_matrix *A, int64_t *scratch, int64_t *plan_host,
                          int32_t *plan_ctas, hyb_stream_t stream);

/* ---- products ---------------------------------------------------------- */

/* Workspace bytes for hyb_spmv / hyb_spmm_skinny on matrix A with this
 * batch and low-rank rank (0 = none); 0 if the arguments are invalid.  The
 * answer depends on the current device (its SM count). */
HYB_API size_t hyb_workspace_bytes(const hyb_matrix *A, int batch, int rank);

/* Zero a workspace before its first use (asynchronous memset on stream). */
HYB_API int hyb_workspace_init(void *ws, size_t ws_bytes, hyb_stream_t stream);

/* Y = W_hat x (+ U (V^T x)) for one input vector (batch 1).  The decode-time
 * sparse matrix-vector product of SparseDecoding (authors' abstract) applied
 * to PATCH's hybrid tiles, with the sparse-plus-low-rank form of 3BASiL §1.
 * ydt selects fp32 or bf16 (round-to-nearest-even from fp32) output; lr may
 * be NULL. */
HYB_API int hyb_spmv(const hyb_matrix *A, const uint16_t *X, int64_t ldx, void *Y,
             int64_t ldy, hyb_dtype ydt, const hyb_lowrank *lr, void *ws,
             size_t ws_bytes, hyb_stream_t stream);

/* Same for a skinny batch of 1..16 input vectors, X [batch][k]. */
HYB_API int hyb_spmm_skinny(const hyb_matrix *A, int batch, const uint16_t *X,
                    int64_t ldx, void *Y, int64_t ldy, hyb_dtype ydt,
                    const hyb_lowrank *lr, void *ws, size_t ws_bytes,
                    hyb_stream_t stream);

/* Launch options of the _ex entry points (bit set; unknown bits are
 * rejected with HYB_ERR_INVALID_ARG). */
#define HYB_LAUNCH_OVERLAP_PREV 1u
/* HYB_LAUNCH_OVERLAP_PREV: launch the streaming kernel as a programmatic
 * dependent of the kernel queued before it on the stream, so that a chain of
 * products (one decode step's layers, back to back) does not drain the GPU
 * between them: while the preceding kernel's last CTAs finish, this product's
 * CTAs start on the SMs it frees and request their first ring of weight
 * bytes.  They read X, and read or write Y, the workspace and the low-rank
 * intermediates, only after the preceding kernel has completed and its
 * writes are visible (griddepcontrol.wait), so results are identical with
 * and without the flag.  The caller guarantees that the weights -- A's tile
 * map, values, masks and offsets, the low-rank factors U and V (or W for
 * hyb_gemv_dense_ex) -- are not written by the work queued before the call on
 * the stream that has not finished by then.  Tilings served by the
 * one-warp-per-row kernel ignore the flag.
 * Low-rank term: with the tuned tilings the term is computed inside the
 * streaming kernel (one launch per call).  One warp per CTA computes V^T x
 * over a slice of V's rows, then t by slices, then U t for a slice of the
 * output rows.  Bounded grid barriers separate the steps; the CTAs are
 * never more than the SMs and there is one per SM, so all of them can be
 * resident.  If other work on the GPU kept some of them from starting for
 * seconds, the wait runs out and hyb_check_status reports HYB_ERR_TIMEOUT.
 * Batches of 8 and 16, and other tilings, run three kernels (V^T x, U t,
 * the product) one after another; the flag applies to the first. */

/* hyb_spmm_skinny with launch options `flags` (0 = hyb_spmm_skinny). */
HYB_API int hyb_spmm_skinny_ex(const hyb_matrix *A, int batch, const uint16_t *X,
                               int64_t ldx, void *Y, int64_t ldy, hyb_dtype ydt,
                               const hyb_lowrank *lr, uint32_t flags, void *ws,
                               size_t ws_bytes, hyb_stream_t stream);

/* ---- row sharding for tensor-parallel decode ---------------------------
 * Host only.  The tile-row bands [*band_begin, *band_end) that rank `rank` of
 * `world` holds when a packed matrix is split by rows for tensor-parallel
 * decode: contiguous bands, balanced by packed bytes (rank i takes the bands
 * whose first packed byte b satisfies i * total <= b * world < (i + 1) *
 * total), every band on exactly one rank; a rank may get none when there are
 * fewer bands than ranks.  Each rank then applies its bands (rows band_begin
 * * b1 .. band_end * b1) to the full X and the ranks' outputs are gathered.
 * The bands of one rank are a contiguous slice of the packed buffers, so a
 * shard needs no repacking: its values, masks and tile map are views, its
 * offsets the matrix's minus those of its first tile.  Errors:
 * HYB_ERR_INVALID_ARG for a bad tiling, map byte, world or rank. */
HYB_API int hyb_shard_bands(int64_t n, int64_t k, int b1, int b2,
                            const uint8_t *tile_map_host, int world, int rank,
                            int64_t *band_begin, int64_t *band_end);

/* ---- prefill / large batch on the tensor cores ---------------------------
 * Y[m][i] = sum_k W_hat[i][k] X[m][k] for a block of M tokens (PATCH: dense
 * tiles on dense tensor-core kernels, 2:4 tiles on sparse ones, §2 Method):
 * one tcgen05 pipeline per CTA of one or two 128-row bands and a block of
 * tokens, fp32 accumulators in tensor memory, the tile's operands moved by TMA in the
 * 128-byte swizzle layout.  Dense tiles run tcgen05.mma; 2:4 tiles run the
 * sparse tensor cores (tcgen05.mma.sp): their packed kept values are the
 * compressed operand as stored, and their masks are converted to the sparse
 * MMA's metadata inside the kernel.
 *   A: 128 x 128 tiles (HYB_ERR_UNSUPPORTED otherwise), k <= 131072.
 *   X: [m][k] bf16, row stride ldx (>= k, multiple of 8), 16-byte aligned;
 *      m >= 1 (any; the last block's missing tokens read as zeros).
 *   Y: [m][n] fp32, row stride ldy >= n, 4-byte aligned; written, not
 *      accumulated.
 *   ws: at least hyb_prefill_workspace_bytes() bytes, 256-byte aligned, its
 *      status word zeroed before the first call (hyb_check_status reads and
 *      clears it).  Nothing is allocated.  Asynchronous on `stream`.
 * hyb_spmm_prefill takes the CTA shape hyb_prefill_block_shape(n, m)
 * returns; hyb_spmm_prefill_blocked takes it from (block_rows, block_tokens):
 * (128, 128), (128, 256), (256, 240) or (256, 208) (two bands sharing each X
 * tile); (0, 0) = the same choice; anything else is HYB_ERR_INVALID_ARG.  Every
 * shape adds the same products in the same order: Y is bit-identical. */
HYB_API size_t hyb_prefill_workspace_bytes(void);
/* The CTA shape for an n-row weight and m tokens on the current device: of
 * the four above, the one with the fewest modelled bytes per SM (CTAs
 * stream their operands from L2 at about the same rate, so a launch takes
 * its waves of CTAs times the bytes one CTA moves per tile).  Writes
 * *block_rows and *block_tokens; HYB_ERR_INVALID_ARG for n < 128, m < 1 or a
 * null pointer (both set to 0). */
HYB_API int hyb_prefill_block_shape(int64_t n, int64_t m, int *block_rows, int *block_tokens);
HYB_API int hyb_spmm_prefill(const hyb_matrix *A, int64_t m, const uint16_t *X, int64_t ldx,
                             float *Y, int64_t ldy, void *ws, size_t ws_bytes,
                             hyb_stream_t stream);
HYB_API int hyb_spmm_prefill_blocked(const hyb_matrix *A, int64_t m, const uint16_t *X,
                                     int64_t ldx, float *Y, int64_t ldy, int block_rows,
                                     int block_tokens, void *ws, size_t ws_bytes,
                                     hyb_stream_t stream);

/* ---- gate and up projections sharing one low-rank factor V ---------------
 * 3BASiL §1-§2: a weight is approximated by S + L with L = U V^T of
 * rank r.  The gate and up projections of an FFN
 * read the same input x; when their low-rank terms share V, t = V^T x is one
 * vector for both:
 *     Yg = Ag X + Ug (V^T X),   Yu = Au X + Uu (V^T X)
 * (X [batch][k] bf16, row stride ldx; Yg [batch][Ag->n] and Yu [batch][Au->n]
 * with row strides ldyg, ldyu, in ydt).  lr_g gives the rank, Ug (ldu) and V
 * (ldv); Uu ([Au->n][rank] bf16, row stride lduu) is the up projection's U.
 * The gate product runs as hyb_spmm_skinny_ex would and leaves t in its part
 * of the workspace; the up product then computes only Uu t (no second pass
 * over V, no second V^T x reduction).  Ag->k must equal Au->k.  Yg is
 * bit-identical to a hyb_spmm_skinny_ex call with (Ug, V); Yu differs from a
 * call with (Uu, V) only by the rounding of t, which the gate product reduces
 * over its own split of k (identical when both products split over the same
 * number of CTAs, and always for batches above 4).
 * flags: as for hyb_spmm_skinny_ex (the up product is a programmatic
 * dependent of the gate product when HYB_LAUNCH_OVERLAP_PREV is set).
 * Workspace: at least hyb_gate_up_workspace_bytes(Ag, Au, batch, rank) bytes,
 * 256-byte aligned; errors as hyb_spmm_skinny. */
HYB_API size_t hyb_gate_up_workspace_bytes(const hyb_matrix *Ag, const hyb_matrix *Au,
                                           int batch, int rank);
HYB_API int hyb_spmm_skinny_gate_up(const hyb_matrix *Ag, const hyb_matrix *Au, int batch,
                                    const uint16_t *X, int64_t ldx, void *Yg, int64_t ldyg,
                                    void *Yu, int64_t ldyu, hyb_dtype ydt,
                                    const hyb_lowrank *lr_g, const uint16_t *Uu, int64_t lduu,
                                    uint32_t flags, void *ws, size_t ws_bytes,
                                    hyb_stream_t stream);

/* Workspace bytes for hyb_lowrank_add. */
HYB_API size_t hyb_lowrank_workspace_bytes(int64_t k, int batch, int rank);

/* Y[b][i] += sum_j U[i][j] sum_k V[k][j] X[b][k]  (fp32 Y, in place): the
 * low-rank term of 3BASiL §1 on its own. */
HYB_API int hyb_lowrank_add(int64_t n, int64_t k, int batch, const hyb_lowrank *lr,
                    const uint16_t *X, int64_t ldx, float *Y, int64_t ldy,
                    void *ws, size_t ws_bytes, hyb_stream_t stream);

/* Workspace bytes for hyb_gemv_dense. */
HYB_API size_t hyb_dense_workspace_bytes(int64_t n, int64_t k, int batch);

/* Plain dense Y = W X for W [n][k] bf16 row-major (row stride ldw), the
 * dense baseline the pages compare the hybrid format against (PATCH §4,
 * SparseDecoding abstract).  Same streaming design as hyb_spmv.  Needs
 * k % 16 == 0.  When n and k are both multiples of 64 the tuned kernel runs
 * and W must be 32-byte aligned with ldw % 16 == 0; otherwise a one-warp-
 * per-row kernel runs and W must be 16-byte aligned with ldw % 8 == 0. */
HYB_API int hyb_gemv_dense(int64_t n, int64_t k, int batch, const uint16_t *W,
                   int64_t ldw, const uint16_t *X, int64_t ldx, void *Y,
                   int64_t ldy, hyb_dtype ydt, void *ws, size_t ws_bytes,
                   hyb_stream_t stream);

/* hyb_gemv_dense with launch options `flags` (see HYB_LAUNCH_OVERLAP_PREV;
 * 0 = hyb_gemv_dense). */
HYB_API int hyb_gemv_dense_ex(int64_t n, int64_t k, int batch, const uint16_t *W,
                              int64_t ldw, const uint16_t *X, int64_t ldx, void *Y,
                              int64_t ldy, hyb_dtype ydt, uint32_t flags, void *ws,
                              size_t ws_bytes, hyb_stream_t stream);

/* ---- general N:M tiles ---------------------------------------------------- */

/* Tiles that are dense or N:M sparse for a general N:M: nk kept of every m
 * consecutive columns, m in {4, 8, 16}, 0 < nk < m, b2 a multiple of m (and
 * the tiling rules of hyb_pack).  PATCH, "Future direction": the tile-level
 * scheme extends to other N:M patterns such as 4:8; SparseDecoding (authors'
 * abstract): N:M with bitmask indexing and fixed-stride traversal.
 * Layout: a sparse tile row keeps, in every group of m columns, the nk values
 * with the largest key (bits & 0x7FFF, ties to the lower column), stored in
 * ascending column order, nk per group (group g at nk*g of the row), and a
 * b2-bit mask stream, bit c of the row's b2/8 bytes set iff column c is kept.
 * A sparse tile holds b1*b2*nk/m values and b1*b2/8 mask bytes.  nk = 2,
 * m = 4 is hyb_pack's layout bit for bit.  Unsupported m, or b2 not a
 * multiple of 16, returns HYB_ERR_UNSUPPORTED; other bad arguments
 * HYB_ERR_INVALID_ARG. */

/* hyb_packed_sizes for nk:m tiles (host only). */
HYB_API int hyb_packed_sizes_nm(int64_t n, int64_t k, int b1, int b2, int nk, int m,
                                const uint8_t *tile_map_host, int64_t *n_vals,
                                int64_t *n_meta_bytes);

/* hyb_pack for nk:m tiles: same arguments, buffers, workspace (status word:
 * NaN weight, bad map byte) and asynchrony as hyb_pack. */
HYB_API int hyb_pack_nm(int64_t n, int64_t k, int b1, int b2, int nk, int m,
                        const uint16_t *W, int64_t ldw, const uint8_t *tile_map,
                        uint16_t *vals, uint8_t *meta, int64_t *val_off,
                        int64_t *meta_off, void *ws, size_t ws_bytes,
                        hyb_stream_t stream);

/* Y = W_hat X for a matrix packed by hyb_pack_nm with the same nk, m; X
 * [batch][k] bf16, batch 1..16, Y [batch][n] fp32 or bf16 (ydt), no low-rank
 * term.  2 of 4 and 4 of 8 with 64- or 128-row by 64- or 128-column tiles run
 * the streaming kernel of hyb_spmm_skinny (the same split, plan -- A->plan is
 * used -- and stage packing: these patterns keep half of a tile's values
 * with b1*b2/8 mask bytes); other patterns and tilings run a one-warp-per-row
 * kernel.  The workspace needs hyb_workspace_bytes(A, batch, 0) bytes and is
 * zeroed once, as for hyb_spmm_skinny (its status word: a bounded wait that
 * ran out; a tile whose offsets do not fit the buffers is skipped and
 * flagged, read by hyb_check_status as HYB_ERR_DEVICE_CHECK).  Asynchronous on
 * stream; results are deterministic. */
HYB_API int hyb_spmm_skinny_nm(const hyb_matrix *A, int nk, int m, int batch,
                               const uint16_t *X, int64_t ldx, void *Y, int64_t ldy,
                               hyb_dtype ydt, void *ws, size_t ws_bytes,
                               hyb_stream_t stream);

/* ---- product without any allocation ------------------------------------ */

/* hyb_spmv for callers that cannot allocate device memory -- an engine that
 * hands out all device memory from one arena sized at start-up, code that
 * runs while a CUDA graph is being captured (cudaMalloc is not allowed
 * there), a host whose memory pool refuses allocations after set-up.  The
 * pages have no counterpart of this entry point; it is a library facility.
 *
 * Same operation, arguments and output as hyb_spmv with batch 1 and no
 * low-rank term, but no workspace argument: the scratch (band tickets and
 * split partial sums) lives in one static device array of
 * hyb_spmv_noalloc_max_scratch_bytes() bytes (1 MiB), which every GPU that
 * loads the library holds until the process exits.  The call allocates and
 * frees nothing.  A matrix whose scratch would exceed the array (with
 * 128-row tiles: more than about 1,600 tile-row bands) is rejected with
 * HYB_ERR_WORKSPACE before anything is queued.
 *  - The first call in each CUDA context looks up the array's device address
 *    (cudaGetSymbolAddress) with that context current and caches it per
 *    context; make that first call outside any stream capture.
 *  - All calls on a device share the one array.  Each call clears the part
 *    that must start at zero (the band tickets), but two calls whose work
 *    overlaps on the GPU (different streams, no ordering between them) race
 *    on it: order them, for instance by using one stream.
 *  - Problems the device detects (a bounded wait that ran out, a tile map
 *    that does not fit its buffers) set the array's status word, which is
 *    kept across calls until hyb_spmv_noalloc_check_status reads and clears
 *    it. */
HYB_API int hyb_spmv_noalloc(const hyb_matrix *A, const uint16_t *X,
                             int64_t ldx, void *Y, int64_t ldy, hyb_dtype ydt,
                             hyb_stream_t stream);

/* Size in bytes of the static scratch array behind hyb_spmv_noalloc. */
HYB_API size_t hyb_spmv_noalloc_max_scratch_bytes(void);

/* hyb_check_status for the static array behind hyb_spmv_noalloc on the
 * current device: synchronise `stream`, read and clear the status word that
 * the noalloc calls since the last query have set.  Same return values and
 * flag bits as hyb_check_status.  Allocates nothing. */
HYB_API int hyb_spmv_noalloc_check_status(hyb_stream_t stream, uint32_t *flags);

/* ---- status ------------------------------------------------------------ */

/* Synchronise `stream`, read and clear the workspace status word.  Returns
 * HYB_OK, HYB_ERR_TIMEOUT (a pipeline wait gave up), HYB_ERR_DEVICE_CHECK (a
 * data check fired) or HYB_ERR_CUDA. If flags is not NULL it receives the raw
 * status bits (1 = NaN weight seen by hyb_pack, 2 = tile_map byte other than
 * 0/1 or a tile map that does not fit the buffers, 4 = a bounded wait ran
 * out). */
HYB_API int hyb_check_status(void *ws, hyb_stream_t stream, uint32_t *flags);

/* Failure-path self test: launch on `stream` a one-CTA kernel whose mbarrier
 * wait can never complete (nothing arrives), bounded by `wait_limit` tries of
 * the same wait loop the products use.  The wait runs out, the kernel sets
 * status bit 4 in the workspace (`ws`, >= 256 bytes, device) and returns; the
 * next hyb_check_status then returns HYB_ERR_TIMEOUT.  Nothing faults or
 * traps.  wait_limit must be in [1, 1 << 20]. */
HYB_API int hyb_selftest_wait_timeout(void *ws, size_t ws_bytes, uint32_t wait_limit,
                                      hyb_stream_t stream);

/* Static description of a status code. */
HYB_API const char *hyb_status_string(int status);

#ifdef __cplusplus
}
#endif

#endif /* HYB_H */
