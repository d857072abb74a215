/*
 * hyb_oracle.c -- plain CPU oracle for the tile-hybrid (dense | 2:4) format.
 *
 * TEST INFRASTRUCTURE ONLY (see hyb_oracle.h): the test-suite, the smoke check
 * and the benchmark's CPU-baseline leg are its only users.
 *
 * Written for a reader who checks it against the definitions by eye: no
 * blocking, no fusion, no reordering.  Products are formed in fp64, where a
 * bf16 x bf16 product is exact.
 *
 * ORACLE_MUTANT (compile-time, default 0) plants one deliberate mistake; the
 * test-suite builds those variants to show that its pins catch each of them.
 * The default build contains none of them.
 */
#include "hyb_oracle.h"

#include <math.h>
#include <stdlib.h>
#include <string.h>

#ifndef ORACLE_MUTANT
#define ORACLE_MUTANT 0
#endif

/* ------------------------------------------------------------------ */
/* bf16 helpers                                                        */
/* ------------------------------------------------------------------ */

/* A bf16 number is the upper half of an IEEE-754 binary32. */
double oracle_bf16_to_f64(uint16_t h) {
  uint32_t u = (uint32_t)h << 16;
  float f;
  memcpy(&f, &u, sizeof f);
  return (double)f;
}

/* Magnitude key used to rank the four members of a 2:4 group.  Clearing the
 * sign bit leaves exponent:mantissa, whose unsigned order is |w| order for
 * every non-NaN bf16 (+0 and -0 both give 0, +/-inf give 0x7F80, NaN keys are
 * above that). */
static unsigned key_of(uint16_t w) {
#if ORACLE_MUTANT == 4
  /* planted mistake: rank by signed value instead of magnitude */
  return (unsigned)(w & 0x8000 ? 0x7FFF - (w & 0x7FFF) : 0x8000 + w);
#else
  return (unsigned)(w & 0x7FFF);
#endif
}

static int is_nan_bf16(uint16_t w) {
  return (w & 0x7F80) == 0x7F80 && (w & 0x007F) != 0;
}

/* ------------------------------------------------------------------ */
/* argument checks shared by the entry points                          */
/* ------------------------------------------------------------------ */

static int check_shape(int64_t n, int64_t k, int b1, int b2,
                       const uint8_t *tile_map) {
  if (n <= 0 || k <= 0 || b1 <= 0 || b2 <= 0) return ORC_BAD_ARG;
  if (b2 % 8 != 0) return ORC_BAD_ARG; /* whole meta bytes per tile row */
  if (n % b1 != 0 || k % b2 != 0) return ORC_BAD_ARG;
  if (tile_map == NULL) return ORC_BAD_ARG;
  int64_t T = (n / b1) * (k / b2);
  for (int64_t t = 0; t < T; ++t)
    if (tile_map[t] > 1) return ORC_BAD_ARG;
  return ORC_OK;
}

/* ------------------------------------------------------------------ */
/* tile offsets                                                        */
/* ------------------------------------------------------------------ */

/* A dense tile stores all b1*b2 values; a 2:4 tile stores half of them plus
 * one 4-bit mask per group of four, i.e. b1*b2/8 bytes. */
int oracle_offsets(int64_t n, int64_t k, int b1, int b2,
                   const uint8_t *tile_map, int64_t *val_off,
                   int64_t *meta_off) {
  if (check_shape(n, k, b1, b2, tile_map) != ORC_OK) return ORC_BAD_ARG;
  int64_t T = (n / b1) * (k / b2);
  int64_t tile_elems = (int64_t)b1 * b2;
  val_off[0] = 0;
  meta_off[0] = 0;
  for (int64_t t = 0; t < T; ++t) {
    int sparse = tile_map[t] == 1;
    val_off[t + 1] = val_off[t] + (sparse ? tile_elems / 2 : tile_elems);
    meta_off[t + 1] = meta_off[t] + (sparse ? tile_elems / 8 : 0);
  }
  return ORC_OK;
}

int oracle_packed_sizes(int64_t n, int64_t k, int b1, int b2,
                        const uint8_t *tile_map, int64_t *n_vals,
                        int64_t *n_meta_bytes) {
  if (check_shape(n, k, b1, b2, tile_map) != ORC_OK) return ORC_BAD_ARG;
  int64_t T = (n / b1) * (k / b2);
  int64_t *vo = (int64_t *)malloc(sizeof(int64_t) * (size_t)(T + 1));
  int64_t *mo = (int64_t *)malloc(sizeof(int64_t) * (size_t)(T + 1));
  if (!vo || !mo) {
    free(vo);
    free(mo);
    return ORC_BAD_ARG;
  }
  oracle_offsets(n, k, b1, b2, tile_map, vo, mo);
  *n_vals = vo[T];
  *n_meta_bytes = mo[T];
  free(vo);
  free(mo);
  return ORC_OK;
}

/* ------------------------------------------------------------------ */
/* 2:4 selection                                                       */
/* ------------------------------------------------------------------ */

/* Keep the two members of w[0..3] with the largest magnitude; among equal
 * magnitudes the lower column wins.  Returns the 4-bit mask (bit j = column
 * j kept); *p0 < *p1 are the kept columns. */
static unsigned select_two(const uint16_t w[4], int *p0, int *p1) {
  int first = 0;
  for (int j = 1; j < 4; ++j) {
#if ORACLE_MUTANT == 1
    /* planted mistake: ties go to the higher column */
    if (key_of(w[j]) >= key_of(w[first])) first = j;
#else
    if (key_of(w[j]) > key_of(w[first])) first = j;
#endif
  }
  int second = -1;
  for (int j = 0; j < 4; ++j) {
    if (j == first) continue;
#if ORACLE_MUTANT == 1
    if (second < 0 || key_of(w[j]) >= key_of(w[second])) second = j;
#else
    if (second < 0 || key_of(w[j]) > key_of(w[second])) second = j;
#endif
  }
  *p0 = first < second ? first : second;
  *p1 = first < second ? second : first;
  return (1u << *p0) | (1u << *p1);
}

/* ------------------------------------------------------------------ */
/* pack / unpack                                                       */
/* ------------------------------------------------------------------ */

/* Byte index, inside a 2:4 tile's meta block, of group g of tile row i, and
 * the shift of its nibble inside that byte. */
static int64_t meta_byte(int64_t i, int64_t g, int b2) {
  return i * (b2 / 8) + g / 2;
}
static int meta_shift(int64_t g) {
#if ORACLE_MUTANT == 2
  /* planted mistake: odd groups in the low nibble */
  return (g % 2 == 1) ? 0 : 4;
#else
  return (g % 2 == 0) ? 0 : 4;
#endif
}
/* Element index, inside a 2:4 tile's value block, of the first kept value of
 * group g of tile row i (the second follows it). */
static int64_t sparse_val_index(int64_t i, int64_t g, int b2) {
  return i * (b2 / 2) + 2 * g;
}

/* Slot (0 or 1) of the kept value from column p0 of a group; the value from
 * p1 > p0 takes the other slot, so values keep ascending column order. */
static int slot_of_first(void) {
#if ORACLE_MUTANT == 6
  return 1; /* planted mistake: kept values stored in descending column order */
#else
  return 0;
#endif
}

int64_t oracle_pack(int64_t n, int64_t k, int b1, int b2, const uint16_t *W,
                    int64_t ldw, const uint8_t *tile_map, uint16_t *vals,
                    uint8_t *meta, int64_t *val_off, int64_t *meta_off) {
  if (check_shape(n, k, b1, b2, tile_map) != ORC_OK) return ORC_BAD_ARG;
  if (W == NULL || ldw < k) return ORC_BAD_ARG;
  oracle_offsets(n, k, b1, b2, tile_map, val_off, meta_off);
  int64_t tiles_per_row = k / b2;
  int64_t T = (n / b1) * tiles_per_row;
  int64_t nan_groups = 0;
  for (int64_t t = 0; t < T; ++t) {
    int64_t tr = t / tiles_per_row, tc = t % tiles_per_row;
    const uint16_t *Wt = W + tr * b1 * ldw + tc * b2;
    uint16_t *vt = vals + val_off[t];
    if (tile_map[t] == 0) {
      for (int64_t i = 0; i < b1; ++i)
        for (int64_t j = 0; j < b2; ++j) vt[i * b2 + j] = Wt[i * ldw + j];
      continue;
    }
    uint8_t *mt = meta + meta_off[t];
    for (int64_t i = 0; i < (int64_t)b1 * (b2 / 8); ++i) mt[i] = 0;
    for (int64_t i = 0; i < b1; ++i) {
      for (int64_t g = 0; g < b2 / 4; ++g) {
        const uint16_t *w = Wt + i * ldw + 4 * g;
        int p0, p1;
        unsigned mask = select_two(w, &p0, &p1);
        if (is_nan_bf16(w[0]) || is_nan_bf16(w[1]) || is_nan_bf16(w[2]) ||
            is_nan_bf16(w[3]))
          nan_groups++;
        vt[sparse_val_index(i, g, b2) + slot_of_first()] = w[p0];
        vt[sparse_val_index(i, g, b2) + 1 - slot_of_first()] = w[p1];
        mt[meta_byte(i, g, b2)] |= (uint8_t)(mask << meta_shift(g));
      }
    }
  }
  return nan_groups;
}

int oracle_unpack(int64_t n, int64_t k, int b1, int b2,
                  const uint8_t *tile_map, const uint16_t *vals,
                  const uint8_t *meta, const int64_t *val_off,
                  const int64_t *meta_off, uint16_t *W_hat) {
  if (check_shape(n, k, b1, b2, tile_map) != ORC_OK) return ORC_BAD_ARG;
  int64_t tiles_per_row = k / b2;
  int64_t T = (n / b1) * tiles_per_row;
  for (int64_t t = 0; t < T; ++t) {
    int64_t tr = t / tiles_per_row, tc = t % tiles_per_row;
    uint16_t *Wt = W_hat + tr * b1 * k + tc * b2;
    const uint16_t *vt = vals + val_off[t];
    if (tile_map[t] == 0) {
      for (int64_t i = 0; i < b1; ++i)
        for (int64_t j = 0; j < b2; ++j) Wt[i * k + j] = vt[i * b2 + j];
      continue;
    }
    const uint8_t *mt = meta + meta_off[t];
    for (int64_t i = 0; i < b1; ++i) {
      for (int64_t g = 0; g < b2 / 4; ++g) {
        unsigned mask = (mt[meta_byte(i, g, b2)] >> meta_shift(g)) & 0xF;
        int taken = 0;
        for (int j = 0; j < 4; ++j) {
          uint16_t v = 0;
          if ((mask >> j) & 1) {
            /* a malformed mask with more than two bits set reads nothing past
             * this group's two slots */
            int slot = taken == 0 ? slot_of_first() : 1 - slot_of_first();
            v = taken < 2 ? vt[sparse_val_index(i, g, b2) + slot] : 0;
            taken++;
          }
          Wt[i * k + 4 * g + j] = v;
        }
      }
    }
  }
  return ORC_OK;
}

/* ------------------------------------------------------------------ */
/* fp64 products                                                       */
/* ------------------------------------------------------------------ */

/* Low-rank inner factor for one input vector: t[j] = sum_k V[k][j] x[k]
 * (and |V|^T |x| into tabs). */
static void lowrank_inner(int64_t k, const uint16_t *x, const uint16_t *V,
                          int64_t ldv, int rank, double *t, double *tabs) {
  for (int j = 0; j < rank; ++j) {
    double s = 0.0, sa = 0.0;
    for (int64_t c = 0; c < k; ++c) {
#if ORACLE_MUTANT == 3
      /* planted mistake: V read transposed */
      double v = oracle_bf16_to_f64(V[(int64_t)j * ldv + c]);
#else
      double v = oracle_bf16_to_f64(V[c * ldv + j]);
#endif
      double xv = oracle_bf16_to_f64(x[c]);
      s += v * xv;
      sa += fabs(v) * fabs(xv);
    }
    t[j] = s;
    tabs[j] = sa;
  }
}

/* One output row: sum_k a[k] x[k] (+ sum_j u[j] t[j]). */
static void row_product(int64_t k, const uint16_t *a, const uint16_t *x,
                        const uint16_t *u, int rank, const double *t,
                        const double *tabs, double *y, double *env) {
  double s = 0.0, sa = 0.0;
#if ORACLE_MUTANT == 5
  int64_t kend = k - 1; /* planted mistake: last column dropped */
#else
  int64_t kend = k;
#endif
  for (int64_t c = 0; c < kend; ++c) {
    double av = oracle_bf16_to_f64(a[c]);
    double xv = oracle_bf16_to_f64(x[c]);
    s += av * xv;
    sa += fabs(av) * fabs(xv);
  }
  for (int j = 0; j < rank; ++j) {
    double uv = oracle_bf16_to_f64(u[j]);
    s += uv * t[j];
    sa += fabs(uv) * tabs[j];
  }
  *y = s;
  if (env) *env = sa;
}

int oracle_matvec_f64(int64_t n, int64_t k, const uint16_t *A, int64_t lda,
                      int batch, const uint16_t *X, int64_t ldx,
                      const uint16_t *U, int64_t ldu, const uint16_t *V,
                      int64_t ldv, int rank, double *Y, int64_t ldy,
                      double *env) {
  if (n <= 0 || k <= 0 || batch <= 0 || lda < k || ldx < k || ldy < n)
    return ORC_BAD_ARG;
  if (U == NULL || V == NULL) rank = 0;
  if (rank < 0) return ORC_BAD_ARG;
  double *t = (double *)calloc((size_t)(rank > 0 ? rank : 1), sizeof(double));
  double *tabs = (double *)calloc((size_t)(rank > 0 ? rank : 1), sizeof(double));
  if (!t || !tabs) {
    free(t);
    free(tabs);
    return ORC_BAD_ARG;
  }
  for (int b = 0; b < batch; ++b) {
    const uint16_t *x = X + (int64_t)b * ldx;
    if (rank > 0) lowrank_inner(k, x, V, ldv, rank, t, tabs);
    for (int64_t i = 0; i < n; ++i) {
      row_product(k, A + i * lda, x, rank > 0 ? U + i * ldu : NULL, rank, t,
                  tabs, &Y[(int64_t)b * ldy + i],
                  env ? &env[(int64_t)b * ldy + i] : NULL);
    }
  }
  free(t);
  free(tabs);
  return ORC_OK;
}

int oracle_spmv_f64(int64_t n, int64_t k, int b1, int b2,
                    const uint8_t *tile_map, const uint16_t *vals,
                    const uint8_t *meta, const int64_t *val_off,
                    const int64_t *meta_off, int batch, const uint16_t *X,
                    int64_t ldx, const uint16_t *U, int64_t ldu,
                    const uint16_t *V, int64_t ldv, int rank, double *Y,
                    int64_t ldy, double *env) {
  uint16_t *W_hat = (uint16_t *)malloc(sizeof(uint16_t) * (size_t)(n * k));
  if (!W_hat) return ORC_BAD_ARG;
  int rc = oracle_unpack(n, k, b1, b2, tile_map, vals, meta, val_off, meta_off,
                         W_hat);
  if (rc == ORC_OK)
    rc = oracle_matvec_f64(n, k, W_hat, k, batch, X, ldx, U, ldu, V, ldv,
                           rank, Y, ldy, env);
  free(W_hat);
  return rc;
}

int oracle_rows_f64(int64_t n, int64_t k, int b1, int b2, const uint16_t *W,
                    int64_t ldw, const uint8_t *tile_map, int batch,
                    const uint16_t *X, int64_t ldx, const uint16_t *U,
                    int64_t ldu, const uint16_t *V, int64_t ldv, int rank,
                    const int64_t *rows, int64_t nrows, double *Y,
                    double *env) {
  if (check_shape(n, k, b1, b2, tile_map) != ORC_OK) return ORC_BAD_ARG;
  if (W == NULL || ldw < k || batch <= 0 || ldx < k || nrows < 0)
    return ORC_BAD_ARG;
  if (U == NULL || V == NULL) rank = 0;
  int64_t tiles_per_row = k / b2;
  uint16_t *a = (uint16_t *)malloc(sizeof(uint16_t) * (size_t)k);
  double *t = (double *)calloc((size_t)(rank > 0 ? rank : 1), sizeof(double));
  double *tabs = (double *)calloc((size_t)(rank > 0 ? rank : 1), sizeof(double));
  if (!a || !t || !tabs) {
    free(a);
    free(t);
    free(tabs);
    return ORC_BAD_ARG;
  }
  for (int b = 0; b < batch; ++b) {
    const uint16_t *x = X + (int64_t)b * ldx;
    if (rank > 0) lowrank_inner(k, x, V, ldv, rank, t, tabs);
    for (int64_t r = 0; r < nrows; ++r) {
      int64_t i = rows[r];
      if (i < 0 || i >= n) {
        free(a);
        free(t);
        free(tabs);
        return ORC_BAD_ARG;
      }
      /* the masked row of W_hat, tile by tile */
      for (int64_t tc = 0; tc < tiles_per_row; ++tc) {
        int64_t tidx = (i / b1) * tiles_per_row + tc;
        const uint16_t *w = W + i * ldw + tc * b2;
        for (int64_t g = 0; g < b2 / 4; ++g) {
          if (tile_map[tidx] == 0) {
            for (int j = 0; j < 4; ++j) a[tc * b2 + 4 * g + j] = w[4 * g + j];
          } else {
            int p0, p1;
            unsigned mask = select_two(w + 4 * g, &p0, &p1);
            for (int j = 0; j < 4; ++j)
              a[tc * b2 + 4 * g + j] = ((mask >> j) & 1) ? w[4 * g + j] : 0;
          }
        }
      }
      row_product(k, a, x, rank > 0 ? U + i * ldu : NULL, rank, t, tabs,
                  &Y[(int64_t)b * nrows + r],
                  env ? &env[(int64_t)b * nrows + r] : NULL);
    }
  }
  free(a);
  free(t);
  free(tabs);
  return ORC_OK;
}

/* ------------------------------------------------------------------ */
/* general N:M tiles (N kept of every M consecutive columns)           */
/* ------------------------------------------------------------------ */
/*
 * The pages name other N:M patterns (4:8) as the natural extension of the
 * tile-level scheme (PATCH, "Future direction"), and SparseDecoding's kernel
 * is an N:M sparse matrix-vector product with a bitmask and a fixed stride.
 * Reading used here, which for N = 2, M = 4 is exactly the 2:4 layout above:
 *  - a sparse tile row keeps N of every M consecutive columns, chosen by the
 *    same magnitude key, ties to the lower column;
 *  - its kept values are stored in ascending column order, N per group (group
 *    g of row i at i*(b2*N/M) + N*g, fixed stride N);
 *  - its mask is a bit stream of b2 bits, bit c (byte c/8, bit c%8 of the
 *    row's b2/8 bytes) set iff column c is kept, so a tile costs
 *    b1*b2*N/M values and b1*b2/8 mask bytes whatever N and M are.
 * Supported: M in {4, 8, 16}, 0 < N < M, b2 a multiple of M and of 8.
 */

static int check_nm(int b2, int nk, int m) {
  if (!(m == 4 || m == 8 || m == 16)) return ORC_BAD_ARG;
  if (nk <= 0 || nk >= m) return ORC_BAD_ARG;
  if (b2 % m != 0) return ORC_BAD_ARG;
  return ORC_OK;
}

/* Member j of w[0..m-1] is kept iff fewer than nk members rank above it; a
 * member ranks above j when its key is larger, or equal with a lower column.
 * Returns the m-bit mask (bit j = column j kept). */
static unsigned select_n_of_m(const uint16_t *w, int nk, int m) {
  unsigned mask = 0;
  for (int j = 0; j < m; ++j) {
    int above = 0;
    for (int i = 0; i < m; ++i) {
      if (i == j) continue;
#if ORACLE_MUTANT == 7
      /* planted mistake: among equal keys the higher column ranks above */
      if (key_of(w[i]) > key_of(w[j]) || (key_of(w[i]) == key_of(w[j]) && i > j))
        above++;
#else
      if (key_of(w[i]) > key_of(w[j]) || (key_of(w[i]) == key_of(w[j]) && i < j))
        above++;
#endif
    }
    if (above < nk) mask |= 1u << j;
  }
  return mask;
}

/* Byte and bit, inside a sparse tile's mask block, of column c of row i. */
static int64_t nm_mask_byte(int64_t i, int64_t c, int b2) {
  return i * (b2 / 8) + c / 8;
}
static int nm_mask_bit(int64_t c) {
#if ORACLE_MUTANT == 8
  return 7 - (int)(c % 8); /* planted mistake: bits numbered from the top */
#else
  return (int)(c % 8);
#endif
}

int oracle_offsets_nm(int64_t n, int64_t k, int b1, int b2, int nk, int m,
                      const uint8_t *tile_map, int64_t *val_off,
                      int64_t *meta_off) {
  if (check_shape(n, k, b1, b2, tile_map) != ORC_OK) return ORC_BAD_ARG;
  if (check_nm(b2, nk, m) != ORC_OK) return ORC_BAD_ARG;
  int64_t T = (n / b1) * (k / b2);
  int64_t tile_elems = (int64_t)b1 * b2;
  val_off[0] = 0;
  meta_off[0] = 0;
  for (int64_t t = 0; t < T; ++t) {
    int sparse = tile_map[t] == 1;
    val_off[t + 1] = val_off[t] + (sparse ? tile_elems / m * nk : tile_elems);
    meta_off[t + 1] = meta_off[t] + (sparse ? tile_elems / 8 : 0);
  }
  return ORC_OK;
}

int64_t oracle_pack_nm(int64_t n, int64_t k, int b1, int b2, int nk, int m,
                       const uint16_t *W, int64_t ldw, const uint8_t *tile_map,
                       uint16_t *vals, uint8_t *meta, int64_t *val_off,
                       int64_t *meta_off) {
  if (oracle_offsets_nm(n, k, b1, b2, nk, m, tile_map, val_off, meta_off) != ORC_OK)
    return ORC_BAD_ARG;
  if (W == NULL || ldw < k) return ORC_BAD_ARG;
  int64_t tiles_per_row = k / b2;
  int64_t T = (n / b1) * tiles_per_row;
  int64_t row_vals = (int64_t)b2 / m * nk;
  int64_t nan_groups = 0;
  for (int64_t t = 0; t < T; ++t) {
    int64_t tr = t / tiles_per_row, tc = t % tiles_per_row;
    const uint16_t *Wt = W + tr * b1 * ldw + tc * b2;
    uint16_t *vt = vals + val_off[t];
    if (tile_map[t] == 0) {
      for (int64_t i = 0; i < b1; ++i)
        for (int64_t j = 0; j < b2; ++j) vt[i * b2 + j] = Wt[i * ldw + j];
      continue;
    }
    uint8_t *mt = meta + meta_off[t];
    for (int64_t i = 0; i < (int64_t)b1 * (b2 / 8); ++i) mt[i] = 0;
    for (int64_t i = 0; i < b1; ++i) {
      for (int64_t g = 0; g < b2 / m; ++g) {
        const uint16_t *w = Wt + i * ldw + (int64_t)m * g;
        unsigned mask = select_n_of_m(w, nk, m);
        int has_nan = 0;
        int s = 0;
        for (int j = 0; j < m; ++j) {
          if (is_nan_bf16(w[j])) has_nan = 1;
          if (!((mask >> j) & 1)) continue;
          int64_t c = (int64_t)m * g + j;
          vt[i * row_vals + (int64_t)nk * g + s] = w[j];
          s++;
          mt[nm_mask_byte(i, c, b2)] |= (uint8_t)(1u << nm_mask_bit(c));
        }
        nan_groups += has_nan;
      }
    }
  }
  return nan_groups;
}

int oracle_unpack_nm(int64_t n, int64_t k, int b1, int b2, int nk, int m,
                     const uint8_t *tile_map, const uint16_t *vals,
                     const uint8_t *meta, const int64_t *val_off,
                     const int64_t *meta_off, uint16_t *W_hat) {
  if (check_shape(n, k, b1, b2, tile_map) != ORC_OK) return ORC_BAD_ARG;
  if (check_nm(b2, nk, m) != ORC_OK) return ORC_BAD_ARG;
  int64_t tiles_per_row = k / b2;
  int64_t T = (n / b1) * tiles_per_row;
  int64_t row_vals = (int64_t)b2 / m * nk;
  for (int64_t t = 0; t < T; ++t) {
    int64_t tr = t / tiles_per_row, tc = t % tiles_per_row;
    uint16_t *Wt = W_hat + tr * b1 * k + tc * b2;
    const uint16_t *vt = vals + val_off[t];
    if (tile_map[t] == 0) {
      for (int64_t i = 0; i < b1; ++i)
        for (int64_t j = 0; j < b2; ++j) Wt[i * k + j] = vt[i * b2 + j];
      continue;
    }
    const uint8_t *mt = meta + meta_off[t];
    for (int64_t i = 0; i < b1; ++i) {
      for (int64_t g = 0; g < b2 / m; ++g) {
        int s = 0;
        for (int j = 0; j < m; ++j) {
          int64_t c = (int64_t)m * g + j;
          uint16_t v = 0;
          if ((mt[nm_mask_byte(i, c, b2)] >> nm_mask_bit(c)) & 1) {
            /* a malformed mask with more than nk bits set reads nothing past
             * this group's nk slots */
            v = s < nk ? vt[i * row_vals + (int64_t)nk * g + s] : 0;
            s++;
          }
          Wt[i * k + c] = v;
        }
      }
    }
  }
  return ORC_OK;
}

int oracle_spmv_nm_f64(int64_t n, int64_t k, int b1, int b2, int nk, int m,
                       const uint8_t *tile_map, const uint16_t *vals,
                       const uint8_t *meta, const int64_t *val_off,
                       const int64_t *meta_off, int batch, const uint16_t *X,
                       int64_t ldx, const uint16_t *U, int64_t ldu,
                       const uint16_t *V, int64_t ldv, int rank, double *Y,
                       int64_t ldy, double *env) {
  uint16_t *W_hat = (uint16_t *)malloc(sizeof(uint16_t) * (size_t)(n * k));
  if (!W_hat) return ORC_BAD_ARG;
  int rc = oracle_unpack_nm(n, k, b1, b2, nk, m, tile_map, vals, meta, val_off,
                            meta_off, W_hat);
  if (rc == ORC_OK)
    rc = oracle_matvec_f64(n, k, W_hat, k, batch, X, ldx, U, ldu, V, ldv,
                           rank, Y, ldy, env);
  free(W_hat);
  return rc;
}
