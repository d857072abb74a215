/*
 * hyb_oracle.h -- CPU oracle for the tile-hybrid (dense | 2:4) weight format
 * and its matrix-vector product.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the library's product path may
 * include, link or call this code: only the test-suite, the smoke check and
 * the CPU-baseline leg of the benchmark use it.  It shares no header, helper
 * or table with the CUDA sources, and never the other way round.
 *
 * Every routine is a plain loop over the definitions, with fp64 arithmetic
 * for the products.  bf16 values travel as their raw 16-bit patterns.
 *
 * Sources (the pages are summaries of the papers below):
 *  - "PATCH: Learnable Tile-level Hybrid Sparsity for LLMs", §2 Methodology,
 *    core mechanism: the weight matrix is cut into b1 x b2 tiles and every
 *    tile is either dense or 2:4 sparse (two non-zeros in every four
 *    consecutive elements, §1 Problem statement; six possible patterns,
 *    §2 "pattern selection").
 *  - "SparseDecoding: decoding-aware pruning ...", authors' abstract: the N:M
 *    sparse matrix-vector kernel indexes kept values with a bitmask and walks
 *    them with a fixed stride.
 *  - "3BASiL: An Algorithmic Framework for Sparse plus Low-Rank Compression of
 *    LLMs", §1 Problem and §2A: W ~ S + L with L of rank r; the sparse block
 *    is obtained by magnitude projection.
 *
 * Readings fixed here where the pages are silent (each is also listed in the
 * design notes):
 *  - b1 counts rows (outputs, N), b2 counts columns (inputs, K); the 2:4 groups
 *    run along K.  Tiles are numbered row-major: t = tr*(K/b2) + tc.
 *  - tile_map[t] == 1 marks a 2:4 tile, 0 a dense tile; other bytes are
 *    rejected.
 *  - Selection: key(w) = bits(w) & 0x7FFF (exact |w| order for every bf16
 *    that is not NaN; +0 and -0 tie).  The two largest keys are kept; on a
 *    tie the lower column wins.
 *  - Packed layout: tile t starts at vals[val_off[t]] and meta[meta_off[t]].
 *    Dense tile: b1 rows of b2 values.  2:4 tile: b1 rows of b2/2 values,
 *    group g of row i stores its two kept values (ascending column) at
 *    i*(b2/2) + 2g and +1 (fixed stride 2 per group); its 4-bit mask sits in
 *    byte i*(b2/8) + g/2, low nibble for even g, bit j set iff column 4g+j
 *    is kept.  Dense tiles own no meta bytes.
 *  - A NaN weight is a data error: the pack still completes with the same key
 *    rule (NaN keys exceed +/-inf) and the number of groups holding a NaN is
 *    returned so the caller can report it.
 */
#ifndef HYB_ORACLE_H
#define HYB_ORACLE_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Return codes (the oracle's own; unrelated to the library's). */
#define ORC_OK 0
#define ORC_BAD_ARG (-1)

/* Sizes of the packed arrays for a tile map held in host memory. */
int oracle_packed_sizes(int64_t n, int64_t k, int b1, int b2,
                        const uint8_t *tile_map, int64_t *n_vals,
                        int64_t *n_meta_bytes);

/* val_off / meta_off (each num_tiles+1 entries) from the tile map. */
int oracle_offsets(int64_t n, int64_t k, int b1, int b2,
                   const uint8_t *tile_map, int64_t *val_off,
                   int64_t *meta_off);

/* Pack W (row-major, leading dimension ldw) into vals/meta/offsets.
 * Returns the number of 2:4 groups that held a NaN (>= 0), or ORC_BAD_ARG. */
int64_t oracle_pack(int64_t n, int64_t k, int b1, int b2, const uint16_t *W,
                    int64_t ldw, const uint8_t *tile_map, uint16_t *vals,
                    uint8_t *meta, int64_t *val_off, int64_t *meta_off);

/* Decode the packed arrays back to the masked dense matrix W_hat (n x k,
 * row-major, bf16 bits; dropped positions become +0). */
int oracle_unpack(int64_t n, int64_t k, int b1, int b2,
                  const uint8_t *tile_map, const uint16_t *vals,
                  const uint8_t *meta, const int64_t *val_off,
                  const int64_t *meta_off, uint16_t *W_hat);

/* Y[b][i] = sum_k A[i][k] * X[b][k]  (+ sum_j U[i][j] * sum_k V[k][j] X[b][k])
 * in fp64, ascending k then ascending j.  A is n x k bf16 (lda), X is
 * batch x k bf16 (ldx), U is n x rank (ldu), V is k x rank (ldv); rank 0 or
 * U == NULL skips the low-rank term.  Y is batch x n fp64 (ldy).  When env
 * is not NULL it receives the error envelope
 * (|A||x| + |U|(|V|^T |x|))[b][i] with the same layout as Y. */
int oracle_matvec_f64(int64_t n, int64_t k, const uint16_t *A, int64_t lda,
                      int batch, const uint16_t *X, int64_t ldx,
                      const uint16_t *U, int64_t ldu, const uint16_t *V,
                      int64_t ldv, int rank, double *Y, int64_t ldy,
                      double *env);

/* Hybrid product straight from the packed arrays: unpack, then the fp64
 * matvec above. */
int oracle_spmv_f64(int64_t n, int64_t k, int b1, int b2,
                    const uint8_t *tile_map, const uint16_t *vals,
                    const uint8_t *meta, const int64_t *val_off,
                    const int64_t *meta_off, int batch, const uint16_t *X,
                    int64_t ldx, const uint16_t *U, int64_t ldu,
                    const uint16_t *V, int64_t ldv, int rank, double *Y,
                    int64_t ldy, double *env);

/* Hybrid product for a list of rows only, straight from the dense W and the
 * tile map (selection applied on the fly).  Row r of the result (for batch b)
 * is Y[b*nrows + r] and corresponds to output row rows[r].  Used to check
 * sampled outputs of matrices too large for the full oracle. */
int oracle_rows_f64(int64_t n, int64_t k, int b1, int b2, const uint16_t *W,
                    int64_t ldw, const uint8_t *tile_map, int batch,
                    const uint16_t *X, int64_t ldx, const uint16_t *U,
                    int64_t ldu, const uint16_t *V, int64_t ldv, int rank,
                    const int64_t *rows, int64_t nrows, double *Y,
                    double *env);

/* fp64 value of a bf16 bit pattern, exposed for the tests. */
double oracle_bf16_to_f64(uint16_t h);

/* General N:M tiles (nk kept of every m consecutive columns; m in {4, 8, 16},
 * 0 < nk < m, b2 a multiple of m and 8).  A sparse tile row stores its kept
 * values in ascending column order, nk per group, and a b2-bit mask stream
 * (bit c of the row's b2/8 bytes set iff column c is kept); nk = 2, m = 4 is
 * the 2:4 layout above, bit for bit.  Same conventions and return codes as
 * the 2:4 routines. */
int oracle_offsets_nm(int64_t n, int64_t k, int b1, int b2, int nk, int m,
                      const uint8_t *tile_map, int64_t *val_off,
                      int64_t *meta_off);
int64_t oracle_pack_nm(int64_t n, int64_t k, int b1, int b2, int nk, int m,
                       const uint16_t *W, int64_t ldw, const uint8_t *tile_map,
                       uint16_t *vals, uint8_t *meta, int64_t *val_off,
                       int64_t *meta_off);
int oracle_unpack_nm(int64_t n, int64_t k, int b1, int b2, int nk, int m,
                     const uint8_t *tile_map, const uint16_t *vals,
                     const uint8_t *meta, const int64_t *val_off,
                     const int64_t *meta_off, uint16_t *W_hat);
int oracle_spmv_nm_f64(int64_t n, int64_t k, int b1, int b2, int nk, int m,
                       const uint8_t *tile_map, const uint16_t *vals,
                       const uint8_t *meta, const int64_t *val_off,
                       const int64_t *meta_off, int batch, const uint16_t *X,
                       int64_t ldx, const uint16_t *U, int64_t ldu,
                       const uint16_t *V, int64_t ldv, int rank, double *Y,
                       int64_t ldy, double *env);

#ifdef __cplusplus
}
#endif

#endif /* HYB_ORACLE_H */
