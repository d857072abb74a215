// hyb_nm.cu -- tiles that are dense or N:M sparse for a general N:M (N kept of
// every M consecutive columns, M in {4, 8, 16}): pack and skinny product.
//
// "PATCH: Learnable Tile-level Hybrid Sparsity for LLMs", "Future direction":
// the tile-level scheme is pattern-agnostic and extends to other N:M patterns
// such as 4:8.  "SparseDecoding" (authors' abstract): an N:M sparse
// matrix-vector product with bitmask indexing and fixed-stride traversal.
//
// Layout (N = 2, M = 4 is the layout of hyb_pack, bit for bit): a sparse tile
// row keeps the N largest-magnitude values of every group of M columns (key =
// bits & 0x7FFF, ties to the lower column), stored in ascending column order,
// N per group (group g at N*g of the row: a fixed stride), and a b2-bit mask
// stream (bit c of the row's b2/8 bytes set iff column c is kept).  A sparse
// tile holds b1*b2*N/M values and b1*b2/8 mask bytes; a dense tile b1*b2
// values.
//
// The product here is the first, plain form of the path: one warp per output
// row, plain loads, fp32 accumulation, a fixed reduction order.
#include "hyb_internal.cuh"

namespace hyb {

int check_tiling(int64_t n, int64_t k, int b1, int b2);  // hyb_pack.cu
int stream_product_nm(const hyb_matrix *A, int nk, int m, int batch, const uint16_t *X,
                      int64_t ldx, void *Y, int64_t ldy, hyb_dtype ydt, void *ws,
                      size_t ws_bytes, cudaStream_t s);  // hyb_spmv.cu

namespace {

constexpr int kNmScanThreads = 1024;
constexpr int kNmPackThreads = 256;
constexpr int kNmWarps = 8;

int check_nm(int b2, int nk, int m) {
  if (!(m == 4 || m == 8 || m == 16)) return HYB_ERR_UNSUPPORTED;
  if (nk <= 0 || nk >= m) return HYB_ERR_INVALID_ARG;
  if (b2 % m != 0) return HYB_ERR_INVALID_ARG;
  // the N:M pack works on 16-column units of a tile row
  if (b2 % 16 != 0) return HYB_ERR_UNSUPPORTED;
  return HYB_OK;
}

// Exclusive prefix sums of the per-tile value and mask sizes, one CTA.
__global__ void __launch_bounds__(kNmScanThreads)
    offsets_nm_kernel(const uint8_t *__restrict__ map, int64_t T, int64_t tile_elems,
                      int64_t sparse_vals, int64_t *__restrict__ val_off,
                      int64_t *__restrict__ meta_off, uint32_t *status) {
  __shared__ int64_t s_v[kNmScanThreads];
  __shared__ int64_t s_m[kNmScanThreads];
  const int tid = threadIdx.x;
  const int64_t per = (T + kNmScanThreads - 1) / kNmScanThreads;
  const int64_t t0 = min(T, (int64_t)tid * per);
  const int64_t t1 = min(T, t0 + per);
  int64_t sv = 0, sm = 0;
  bool bad = false;
  for (int64_t t = t0; t < t1; ++t) {
    const uint8_t b = map[t];
    bad |= b > 1;
    sv += b == 1 ? sparse_vals : tile_elems;
    sm += b == 1 ? tile_elems / 8 : 0;
  }
  s_v[tid] = sv;
  s_m[tid] = sm;
  __syncthreads();
  for (int d = 1; d < kNmScanThreads; d <<= 1) {  // inclusive scan
    int64_t av = 0, am = 0;
    if (tid >= d) {
      av = s_v[tid - d];
      am = s_m[tid - d];
    }
    __syncthreads();
    s_v[tid] += av;
    s_m[tid] += am;
    __syncthreads();
  }
  int64_t rv = s_v[tid] - sv, rm = s_m[tid] - sm;
  for (int64_t t = t0; t < t1; ++t) {
    val_off[t] = rv;
    meta_off[t] = rm;
    const bool sparse = map[t] == 1;
    rv += sparse ? sparse_vals : tile_elems;
    rm += sparse ? tile_elems / 8 : 0;
  }
  if (tid == kNmScanThreads - 1) {
    val_off[T] = s_v[tid];
    meta_off[T] = s_m[tid];
  }
  if (__syncthreads_or(bad) && tid == 0) atomicOr(status, kStatusBadMap);
}

__device__ __forceinline__ bool nan_bf16(uint32_t w) {
  return (w & 0x7F80u) == 0x7F80u && (w & 0x007Fu) != 0;
}

// A thread takes 16 consecutive columns of one tile row (whole groups for
// every M, two mask bytes): dense tiles copy them; N:M tiles keep, in every
// group, the members that fewer than nk others rank above (a larger key, or an
// equal key in a lower column), and write them in column order.
__global__ void __launch_bounds__(kNmPackThreads)
    pack_nm_kernel(int64_t T, int64_t tpr, int b1, int b2, int nk, int m,
                   const uint16_t *__restrict__ W, int64_t ldw,
                   const uint8_t *__restrict__ map, const int64_t *__restrict__ val_off,
                   const int64_t *__restrict__ meta_off, uint16_t *__restrict__ vals,
                   uint8_t *__restrict__ meta, uint32_t *status) {
  const int upr = b2 / 16;  // 16-column units per tile row
  const int units = b1 * upr;
  const int64_t row_vals = (int64_t)b2 / m * nk;
  bool nan_seen = false;
  for (int64_t t = blockIdx.x; t < T; t += gridDim.x) {
    const int64_t tr = t / tpr, tc = t - tr * tpr;
    const uint16_t *Wt = W + tr * b1 * ldw + tc * b2;
    uint16_t *vt = vals + val_off[t];
    const bool sparse = map[t] == 1;
    for (int u = threadIdx.x; u < units; u += kNmPackThreads) {
      const int i = u / upr, q = u - i * upr;
      const uint4 a = *reinterpret_cast<const uint4 *>(Wt + (int64_t)i * ldw + 16 * q);
      const uint4 b = *reinterpret_cast<const uint4 *>(Wt + (int64_t)i * ldw + 16 * q + 8);
      if (!sparse) {
        *reinterpret_cast<uint4 *>(vt + (int64_t)i * b2 + 16 * q) = a;
        *reinterpret_cast<uint4 *>(vt + (int64_t)i * b2 + 16 * q + 8) = b;
        continue;
      }
      const uint32_t pk[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
      uint32_t w[16];
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        w[2 * e] = pk[e] & 0xFFFFu;
        w[2 * e + 1] = pk[e] >> 16;
      }
      uint32_t mask = 0;
#pragma unroll
      for (int c = 0; c < 16; ++c) {
        nan_seen |= nan_bf16(w[c]);
        const int g0 = c / m * m;  // first column of c's group
        const uint32_t kc = w[c] & 0x7FFFu;
        int above = 0;
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          if (j < g0 || j >= g0 + m || j == c) continue;
          const uint32_t kj = w[j] & 0x7FFFu;
          above += (kj > kc || (kj == kc && j < c)) ? 1 : 0;
        }
        if (above < nk) mask |= 1u << c;
      }
      // kept values of this unit's 16/m groups, in column order
      uint16_t *dst = vt + (int64_t)i * row_vals + (int64_t)(16 * q / m) * nk;
      int s = 0;
#pragma unroll
      for (int c = 0; c < 16; ++c)
        if ((mask >> c) & 1u) dst[s++] = (uint16_t)w[c];
      uint8_t *mt = meta + meta_off[t] + (int64_t)i * (b2 / 8) + 2 * q;
      mt[0] = (uint8_t)(mask & 0xFFu);
      mt[1] = (uint8_t)(mask >> 8);
    }
  }
  if (__syncthreads_or(nan_seen) && threadIdx.x == 0) atomicOr(status, kStatusNaN);
}

struct NmParams {
  const uint8_t *map;
  const uint16_t *vals;
  const uint8_t *meta;
  const int64_t *val_off;
  const int64_t *meta_off;
  int64_t n, k, tpr, n_vals, n_meta;
  int b1, b2, nk, m;
  const uint16_t *X;
  int64_t ldx;
  int batch;
  void *Y;
  int64_t ldy;
  int ydt;
  uint32_t *status;
};

// One warp per output row.  Dense tiles: a lane takes 8 consecutive columns
// per step (16-byte loads of values and x).  N:M tiles: a lane takes whole
// groups; the group's mask bits give the columns of its N values, in order.
// A tile whose offsets do not fit the buffers, or are not a multiple of 8
// values, is skipped and flagged (a corrupted matrix is reported, never read
// out of bounds or misaligned).
template <int BP>
__global__ void __launch_bounds__(kNmWarps * 32) spmm_nm_kernel(const NmParams p) {
  const int lane = threadIdx.x & 31;
  const int64_t warps = (int64_t)gridDim.x * kNmWarps;
  const int64_t te = (int64_t)p.b1 * p.b2;
  const int64_t row_vals = (int64_t)p.b2 / p.m * p.nk;
  const int groups = p.b2 / p.m;
  const uint32_t gmask = p.m == 16 ? 0xFFFFu : (1u << p.m) - 1u;
  for (int64_t r = (int64_t)blockIdx.x * kNmWarps + (threadIdx.x >> 5); r < p.n; r += warps) {
    const int64_t band = r / p.b1;
    const int i = (int)(r - band * p.b1);
    float acc[BP];
#pragma unroll
    for (int b = 0; b < BP; ++b) acc[b] = 0.f;
    bool bad = false;
    for (int64_t tc = 0; tc < p.tpr; ++tc) {
      const int64_t t = band * p.tpr + tc;
      const bool sparse = p.map[t] == 1;
      const int64_t vo = p.val_off[t], mo = p.meta_off[t];
      // (every tile starts on a multiple of 8 values: the dense path reads
      // 16-byte pieces)
      if (vo < 0 || (vo & 7) != 0 || vo + (sparse ? te / p.m * p.nk : te) > p.n_vals ||
          (sparse && (mo < 0 || mo + te / 8 > p.n_meta))) {
        bad = true;
        continue;
      }
      const uint16_t *xt = p.X + tc * p.b2;
      if (!sparse) {
        const uint16_t *wr = p.vals + vo + (int64_t)i * p.b2;
        for (int c8 = lane; c8 < p.b2 / 8; c8 += 32) {
          const uint4 wv = ld_stream16(wr + 8 * c8);
          const uint32_t w[4] = {wv.x, wv.y, wv.z, wv.w};
#pragma unroll
          for (int b = 0; b < BP; ++b) {
            if (b >= p.batch) break;
            const uint4 xv = ld_keep16(xt + (int64_t)b * p.ldx + 8 * c8);
            const uint32_t x[4] = {xv.x, xv.y, xv.z, xv.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              acc[b] = fmaf(bf16_lo(w[e]), bf16_lo(x[e]), acc[b]);
              acc[b] = fmaf(bf16_hi(w[e]), bf16_hi(x[e]), acc[b]);
            }
          }
        }
      } else {
        const uint16_t *vr = p.vals + vo + (int64_t)i * row_vals;
        const uint8_t *mr = p.meta + mo + (int64_t)i * (p.b2 / 8);
        for (int g = lane; g < groups; g += 32) {
          const int c0 = g * p.m;  // first column of the group
          // the group's m bits of the row's mask stream (never across a
          // 16-bit boundary: m divides 16)
          const uint32_t two = (uint32_t)mr[c0 / 8] |
                               ((c0 / 8 + 1 < p.b2 / 8) ? (uint32_t)mr[c0 / 8 + 1] << 8 : 0u);
          uint32_t mg = (two >> (c0 % 8)) & gmask;
          for (int s = 0; s < p.nk && mg != 0u; ++s) {
            const int c = __ffs(mg) - 1;
            mg &= mg - 1u;
            const float v = __uint_as_float((uint32_t)vr[(int64_t)g * p.nk + s] << 16);
#pragma unroll
            for (int b = 0; b < BP; ++b) {
              if (b >= p.batch) break;
              const float xv =
                  __uint_as_float((uint32_t)__ldg(xt + (int64_t)b * p.ldx + c0 + c) << 16);
              acc[b] = fmaf(v, xv, acc[b]);
            }
          }
        }
      }
    }
    if (__any_sync(0xffffffffu, bad) && lane == 0) atomicOr(p.status, kStatusBadMap);
#pragma unroll
    for (int b = 0; b < BP; ++b) {
      float v = acc[b];
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
      if (lane == 0 && b < p.batch) {
        if (p.ydt == HYB_BF16)
          reinterpret_cast<uint16_t *>(p.Y)[(int64_t)b * p.ldy + r] = f32_to_bf16_rne(v);
        else
          reinterpret_cast<float *>(p.Y)[(int64_t)b * p.ldy + r] = v;
      }
    }
  }
}

void *pick_spmm_nm(int batch) {
  if (batch <= 1) return reinterpret_cast<void *>(&spmm_nm_kernel<1>);
  if (batch <= 2) return reinterpret_cast<void *>(&spmm_nm_kernel<2>);
  if (batch <= 4) return reinterpret_cast<void *>(&spmm_nm_kernel<4>);
  if (batch <= 8) return reinterpret_cast<void *>(&spmm_nm_kernel<8>);
  return reinterpret_cast<void *>(&spmm_nm_kernel<16>);
}

}  // namespace
}  // namespace hyb

extern "C" {

int hyb_packed_sizes_nm(int64_t n, int64_t k, int b1, int b2, int nk, int m,
                        const uint8_t *tile_map_host, int64_t *n_vals,
                        int64_t *n_meta_bytes) {
  int rc = hyb::check_tiling(n, k, b1, b2);
  if (rc != HYB_OK) return rc;
  rc = hyb::check_nm(b2, nk, m);
  if (rc != HYB_OK) return rc;
  if (!tile_map_host || !n_vals || !n_meta_bytes) return HYB_ERR_INVALID_ARG;
  const int64_t T = (n / b1) * (k / b2);
  const int64_t te = (int64_t)b1 * b2;
  int64_t v = 0, mb = 0;
  for (int64_t t = 0; t < T; ++t) {
    if (tile_map_host[t] > 1) return HYB_ERR_INVALID_ARG;
    v += tile_map_host[t] ? te / m * nk : te;
    mb += tile_map_host[t] ? te / 8 : 0;
  }
  *n_vals = v;
  *n_meta_bytes = mb;
  return HYB_OK;
}

int hyb_pack_nm(int64_t n, int64_t k, int b1, int b2, int nk, int m, const uint16_t *W,
                int64_t ldw, const uint8_t *tile_map, uint16_t *vals, uint8_t *meta,
                int64_t *val_off, int64_t *meta_off, void *ws, size_t ws_bytes,
                hyb_stream_t stream) {
  int rc = hyb::check_tiling(n, k, b1, b2);
  if (rc != HYB_OK) return rc;
  rc = hyb::check_nm(b2, nk, m);
  if (rc != HYB_OK) return rc;
  if (!W || !tile_map || !vals || !meta || !val_off || !meta_off) return HYB_ERR_INVALID_ARG;
  if (ldw < k) return HYB_ERR_INVALID_ARG;
  if (!ws || ws_bytes < hyb::kHeaderBytes) return HYB_ERR_WORKSPACE;
  if (((uintptr_t)W | (uintptr_t)vals) % 16 != 0 || ldw % 8 != 0) return HYB_ERR_ALIGNMENT;
  const int64_t T = (n / b1) * (k / b2);
  const int64_t te = (int64_t)b1 * b2;
  cudaStream_t s = (cudaStream_t)stream;
  uint32_t *status = reinterpret_cast<uint32_t *>(ws);
  hyb::offsets_nm_kernel<<<1, hyb::kNmScanThreads, 0, s>>>(tile_map, T, te, te / m * nk,
                                                           val_off, meta_off, status);
  if (cudaGetLastError() != cudaSuccess) return HYB_ERR_CUDA;
  int sms = 0;
  rc = hyb::device_sm_count(&sms);
  if (rc != HYB_OK) return rc;
  const int64_t grid = T < (int64_t)sms * 16 ? T : (int64_t)sms * 16;
  hyb::pack_nm_kernel<<<(unsigned)grid, hyb::kNmPackThreads, 0, s>>>(
      T, k / b2, b1, b2, nk, m, W, ldw, tile_map, val_off, meta_off, vals, meta, status);
  if (cudaGetLastError() != cudaSuccess) return HYB_ERR_CUDA;
  return HYB_OK;
}

int hyb_spmm_skinny_nm(const hyb_matrix *A, int nk, int m, int batch, const uint16_t *X,
                       int64_t ldx, void *Y, int64_t ldy, hyb_dtype ydt, void *ws,
                       size_t ws_bytes, hyb_stream_t stream) {
  if (!A) return HYB_ERR_INVALID_ARG;
  int rc = hyb::check_tiling(A->n, A->k, A->b1, A->b2);
  if (rc != HYB_OK) return rc;
  rc = hyb::check_nm(A->b2, nk, m);
  if (rc != HYB_OK) return rc;
  if (A->num_tiles != (A->n / A->b1) * (A->k / A->b2)) return HYB_ERR_INVALID_ARG;
  if (!A->tile_map || !A->vals || !A->meta || !A->val_off || !A->meta_off)
    return HYB_ERR_INVALID_ARG;
  const int64_t te = (int64_t)A->b1 * A->b2;
  if (A->n_vals < A->num_tiles * (te / m * nk) || A->n_vals > A->num_tiles * te ||
      A->n_meta_bytes < 0 || A->n_meta_bytes > A->num_tiles * te / 8)
    return HYB_ERR_INVALID_ARG;
  if (((uintptr_t)A->vals) % 16 != 0) return HYB_ERR_ALIGNMENT;
  if (!X || !Y) return HYB_ERR_INVALID_ARG;
  if (batch < 1 || batch > 16) return HYB_ERR_INVALID_ARG;
  if (ydt != HYB_F32 && ydt != HYB_BF16) return HYB_ERR_INVALID_ARG;
  if (ldx < A->k || ldy < A->n) return HYB_ERR_INVALID_ARG;
  if ((uintptr_t)X % 16 != 0 || ldx % 8 != 0) return HYB_ERR_ALIGNMENT;
  if ((uintptr_t)Y % (ydt == HYB_F32 ? 4 : 2) != 0) return HYB_ERR_ALIGNMENT;
  if (!ws || ws_bytes < hyb::kHeaderBytes) return HYB_ERR_WORKSPACE;
  // 2 of 4 and 4 of 8 with the tuned tilings: the streaming kernel
  rc = hyb::stream_product_nm(A, nk, m, batch, X, ldx, Y, ldy, ydt, ws, ws_bytes,
                              (cudaStream_t)stream);
  if (rc != HYB_ERR_UNSUPPORTED) return rc;
  hyb::NmParams prm{};
  prm.map = A->tile_map;
  prm.vals = A->vals;
  prm.meta = A->meta;
  prm.val_off = A->val_off;
  prm.meta_off = A->meta_off;
  prm.n = A->n;
  prm.k = A->k;
  prm.tpr = A->k / A->b2;
  prm.n_vals = A->n_vals;
  prm.n_meta = A->n_meta_bytes;
  prm.b1 = A->b1;
  prm.b2 = A->b2;
  prm.nk = nk;
  prm.m = m;
  prm.X = X;
  prm.ldx = ldx;
  prm.batch = batch;
  prm.Y = Y;
  prm.ldy = ldy;
  prm.ydt = ydt;
  prm.status = reinterpret_cast<uint32_t *>(ws);
  int sms = 0;
  rc = hyb::device_sm_count(&sms);
  if (rc != HYB_OK) return rc;
  const int64_t need = (A->n + hyb::kNmWarps - 1) / hyb::kNmWarps;
  const int64_t grid = need < (int64_t)sms * 8 ? need : (int64_t)sms * 8;
  void *args[] = {&prm};
  if (cudaLaunchKernel(hyb::pick_spmm_nm(batch), dim3((unsigned)grid), dim3(hyb::kNmWarps * 32),
                       args, 0, (cudaStream_t)stream) != cudaSuccess)
    return HYB_ERR_CUDA;
  return HYB_OK;
}

}  // extern "C"
