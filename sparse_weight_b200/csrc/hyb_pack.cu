// hyb_pack.cu -- dense bf16 W + tile map -> packed tile-hybrid format.
//
// "PATCH: Learnable Tile-level Hybrid Sparsity for LLMs", §2 Methodology:
// every b1 x b2 tile is kept dense or made 2:4 sparse.  Inside a 2:4 tile each
// group of four consecutive columns keeps its two largest-magnitude values
// (the magnitude projection of "3BASiL", §2A), stored at a fixed stride with a
// 4-bit mask ("SparseDecoding", authors' abstract: bitmask indexing).
// Offline step (once per weight); bandwidth-bound.
#include "hyb_internal.cuh"

namespace hyb {
namespace {

constexpr int kScanThreads = 1024;
constexpr int kPackThreads = 256;

// Exclusive prefix sums of the per-tile value and meta sizes, one CTA.
__global__ void __launch_bounds__(kScanThreads)
    offsets_kernel(const uint8_t *__restrict__ map, int64_t T,
                   int64_t tile_elems, int64_t *__restrict__ val_off,
                   int64_t *__restrict__ meta_off, uint32_t *status) {
  __shared__ int64_t s_v[kScanThreads];
  __shared__ int64_t s_m[kScanThreads];
  const int tid = threadIdx.x;
  const int64_t per = (T + kScanThreads - 1) / kScanThreads;
  const int64_t t0 = min(T, (int64_t)tid * per);
  const int64_t t1 = min(T, t0 + per);
  int64_t sv = 0, sm = 0;
  bool bad = false;
  for (int64_t t = t0; t < t1; ++t) {
    const uint8_t m = map[t];
    bad |= m > 1;
    const bool sparse = m == 1;
    sv += sparse ? tile_elems / 2 : tile_elems;
    sm += sparse ? tile_elems / 8 : 0;
  }
  s_v[tid] = sv;
  s_m[tid] = sm;
  __syncthreads();
  // Hillis-Steele inclusive scan.
  for (int d = 1; d < kScanThreads; d <<= 1) {
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
    rv += sparse ? tile_elems / 2 : tile_elems;
    rm += sparse ? tile_elems / 8 : 0;
  }
  if (tid == kScanThreads - 1) {
    val_off[T] = s_v[tid];
    meta_off[T] = s_m[tid];
  }
  if (__syncthreads_or(bad) && tid == 0) atomicOr(status, kStatusBadMap);
}

__device__ __forceinline__ bool is_nan_bf16(uint32_t w) {
  return (w & 0x7F80u) == 0x7F80u && (w & 0x007Fu) != 0;
}

// One 2:4 group: keep the two largest keys (bits & 0x7FFF), lower column on
// ties.  Returns the 4-bit mask and the two kept values, ascending column.
__device__ __forceinline__ uint32_t select_group(const uint32_t w[4],
                                                 uint32_t &out_pair) {
  uint32_t key[4];
#pragma unroll
  for (int j = 0; j < 4; ++j) key[j] = w[j] & 0x7FFFu;
  int first = 0;
#pragma unroll
  for (int j = 1; j < 4; ++j)
    if (key[j] > key[first]) first = j;
  int second = first == 0 ? 1 : 0;
#pragma unroll
  for (int j = 0; j < 4; ++j)
    if (j != first && j > second && key[j] > key[second]) second = j;
  const int lo = min(first, second), hi = max(first, second);
  out_pair = w[lo] | (w[hi] << 16);
  return (1u << lo) | (1u << hi);
}

// One CTA per tile (grid-stride).  A thread handles 8 consecutive columns of
// one tile row: 16 bytes in; dense tiles copy them, 2:4 tiles emit two groups
// (4 values, 8 bytes) and one meta byte.
__global__ void __launch_bounds__(kPackThreads)
    pack_kernel(int64_t T, int64_t tpr, int b1, int b2,
                const uint16_t *__restrict__ W, int64_t ldw,
                const uint8_t *__restrict__ map,
                const int64_t *__restrict__ val_off,
                const int64_t *__restrict__ meta_off, uint16_t *__restrict__ vals,
                uint8_t *__restrict__ meta, uint32_t *status) {
  const int upr = b2 / 8;  // 8-column units per tile row
  const int units = b1 * upr;
  bool nan_seen = false;
  for (int64_t t = blockIdx.x; t < T; t += gridDim.x) {
    const int64_t tr = t / tpr, tc = t - tr * tpr;
    const uint16_t *Wt = W + tr * b1 * ldw + tc * b2;
    uint16_t *vt = vals + val_off[t];
    const bool sparse = map[t] == 1;
    uint8_t *mt = sparse ? meta + meta_off[t] : nullptr;
    for (int u = threadIdx.x; u < units; u += kPackThreads) {
      const int i = u / upr, q = u - i * upr;
      const uint4 src =
          *reinterpret_cast<const uint4 *>(Wt + (int64_t)i * ldw + 8 * q);
      if (!sparse) {
        *reinterpret_cast<uint4 *>(vt + (int64_t)i * b2 + 8 * q) = src;
        continue;
      }
      const uint32_t wv[8] = {src.x & 0xFFFFu, src.x >> 16, src.y & 0xFFFFu,
                              src.y >> 16,     src.z & 0xFFFFu, src.z >> 16,
                              src.w & 0xFFFFu, src.w >> 16};
#pragma unroll
      for (int e = 0; e < 8; ++e) nan_seen |= is_nan_bf16(wv[e]);
      uint32_t pair0, pair1;
      const uint32_t m0 = select_group(wv, pair0);
      const uint32_t m1 = select_group(wv + 4, pair1);
      *reinterpret_cast<uint2 *>(vt + (int64_t)i * (b2 / 2) + 4 * q) =
          make_uint2(pair0, pair1);
      mt[(int64_t)i * (b2 / 8) + q] = (uint8_t)(m0 | (m1 << 4));
    }
  }
  if (__syncthreads_or(nan_seen) && threadIdx.x == 0)
    atomicOr(status, kStatusNaN);
}

}  // namespace

// Shape rule shared by every entry point of the library.
int check_tiling(int64_t n, int64_t k, int b1, int b2) {
  if (n <= 0 || k <= 0 || b1 <= 0 || b2 <= 0) return HYB_ERR_INVALID_ARG;
  if (n % b1 != 0 || k % b2 != 0) return HYB_ERR_INVALID_ARG;
  if (b2 % 8 != 0) return HYB_ERR_INVALID_ARG;  // whole mask bytes per 2:4 tile row
  if (((int64_t)b1 * b2) % 128 != 0) return HYB_ERR_INVALID_ARG;
  return HYB_OK;
}

}  // namespace hyb

extern "C" {

size_t hyb_pack_workspace_bytes(void) { return hyb::kHeaderBytes; }

int hyb_packed_sizes(int64_t n, int64_t k, int b1, int b2,
                     const uint8_t *tile_map_host, int64_t *n_vals,
                     int64_t *n_meta_bytes) {
  int rc = hyb::check_tiling(n, k, b1, b2);
  if (rc != HYB_OK) return rc;
  if (!tile_map_host || !n_vals || !n_meta_bytes) return HYB_ERR_INVALID_ARG;
  const int64_t T = (n / b1) * (k / b2);
  const int64_t te = (int64_t)b1 * b2;
  int64_t v = 0, m = 0;
  for (int64_t t = 0; t < T; ++t) {
    if (tile_map_host[t] > 1) return HYB_ERR_INVALID_ARG;
    v += tile_map_host[t] ? te / 2 : te;
    m += tile_map_host[t] ? te / 8 : 0;
  }
  *n_vals = v;
  *n_meta_bytes = m;
  return HYB_OK;
}

int hyb_shard_bands(int64_t n, int64_t k, int b1, int b2, const uint8_t *tile_map_host,
                    int world, int rank, int64_t *band_begin, int64_t *band_end) {
  int rc = hyb::check_tiling(n, k, b1, b2);
  if (rc != HYB_OK) return rc;
  if (!tile_map_host || !band_begin || !band_end || world < 1 || rank < 0 || rank >= world)
    return HYB_ERR_INVALID_ARG;
  const int64_t R = n / b1, tpr = k / b2;
  const int64_t dense = 2LL * b1 * b2, sparse = (int64_t)b1 * b2 + (int64_t)b1 * b2 / 8;
  // packed bytes before each band; rank i takes the bands whose first byte
  // b satisfies i * total <= b * world < (i + 1) * total (contiguous bands,
  // balanced by bytes, every band on exactly one rank)
  int64_t total = 0;
  for (int64_t t = 0; t < R * tpr; ++t) {
    if (tile_map_host[t] > 1) return HYB_ERR_INVALID_ARG;
    total += tile_map_host[t] ? sparse : dense;
  }
  int64_t before = 0, lo = -1, hi = -1;
  for (int64_t r = 0; r <= R; ++r) {
    const int64_t b = r < R ? before : total;
    if (lo < 0 && (r == R || b * world >= (int64_t)rank * total)) lo = r;
    if (hi < 0 && (r == R || b * world >= (int64_t)(rank + 1) * total)) hi = r;
    if (r < R)
      for (int64_t t = r * tpr; t < (r + 1) * tpr; ++t) before += tile_map_host[t] ? sparse : dense;
  }
  if (rank == world - 1) hi = R;
  *band_begin = lo;
  *band_end = hi < lo ? lo : hi;
  return HYB_OK;
}

int hyb_pack(int64_t n, int64_t k, int b1, int b2, const uint16_t *W,
             int64_t ldw, const uint8_t *tile_map, uint16_t *vals,
             uint8_t *meta, int64_t *val_off, int64_t *meta_off, void *ws,
             size_t ws_bytes, hyb_stream_t stream) {
  int rc = hyb::check_tiling(n, k, b1, b2);
  if (rc != HYB_OK) return rc;
  if (!W || !tile_map || !vals || !meta || !val_off || !meta_off)
    return HYB_ERR_INVALID_ARG;
  if (ldw < k) return HYB_ERR_INVALID_ARG;
  if (!ws || ws_bytes < hyb::kHeaderBytes) return HYB_ERR_WORKSPACE;
  if (((uintptr_t)W | (uintptr_t)vals) % 16 != 0 || ldw % 8 != 0)
    return HYB_ERR_ALIGNMENT;
  const int64_t T = (n / b1) * (k / b2);
  cudaStream_t s = (cudaStream_t)stream;
  uint32_t *status = reinterpret_cast<uint32_t *>(ws);
  hyb::offsets_kernel<<<1, hyb::kScanThreads, 0, s>>>(
      tile_map, T, (int64_t)b1 * b2, val_off, meta_off, status);
  if (cudaGetLastError() != cudaSuccess) return HYB_ERR_CUDA;
  int sms = 0;
  rc = hyb::device_sm_count(&sms);
  if (rc != HYB_OK) return rc;
  const int64_t grid = T < (int64_t)sms * 16 ? T : (int64_t)sms * 16;
  hyb::pack_kernel<<<(unsigned)grid, hyb::kPackThreads, 0, s>>>(
      T, k / b2, b1, b2, W, ldw, tile_map, val_off, meta_off, vals, meta,
      status);
  if (cudaGetLastError() != cudaSuccess) return HYB_ERR_CUDA;
  return HYB_OK;
}

}  // extern "C"
