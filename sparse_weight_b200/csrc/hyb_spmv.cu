// hyb_spmv.cu -- Y = W_hat X (+ U (V^T X)) for the tile-hybrid format, plus
// the dense GEMV baseline and the stand-alone low-rank term.
//
// Decode-time products are memory-bound ("SparseDecoding: decoding-aware
// pruning ...", authors' abstract: the decode phase is limited by memory
// access and is dominated by sparse matrix-vector products), so every kernel
// here is a single streaming pass over the weight bytes with no tensor cores.
//
//  * hybrid_tma_kernel (packed matrices, tilings 128x128, 128x64, 64x64,
//    64x128): the packed stream is row-major over tiles, so every tile-row
//    band is contiguous.  CTA c of G takes the tiles whose byte offset falls
//    in [c, c+1) * total / G -- a split by bytes, not by tiles, because a
//    dense tile costs 2 B/weight and a 2:4 tile 1.125 B/weight ("PATCH:
//    Learnable Tile-level Hybrid Sparsity for LLMs", §2: tiles are dense or
//    2:4).  A producer warp moves the bytes into a shared-memory ring with
//    bulk copies; consumer warps compute from it; two epilogue warps finish
//    the bands.
//  * hybrid_rowwarp_kernel (any other legal tiling, packed or row-major): one
//    warp per output row, plain loads.
//  * dense_gemv_kernel (row-major bf16 W, the baseline the format is measured
//    against): the same byte split over uniform tiles, register double
//    buffering instead of a ring.
//  * Band results cross CTAs through fp32 partial slots; the last CTA to
//    arrive at a band (atomic ticket, no spinning) sums the slots in CTA order
//    -- deterministic -- and applies the epilogue: the low-rank term
//    ("3BASiL", §1: W ~ S + L) and the fp32 or bf16 store.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <mutex>

#include "hyb_internal.cuh"

namespace hyb {

int check_tiling(int64_t n, int64_t k, int b1, int b2);  // hyb_pack.cu

namespace {

constexpr int kWarps = 8;
constexpr int kThreads = kWarps * 32;
constexpr int kMaxRank = 256;

struct Params {
  // matrix (packed) or dense W (strided mode)
  const uint8_t *map;
  const uint8_t *vals;  // bytes
  const uint8_t *meta;
  const int64_t *val_off;
  const int64_t *meta_off;
  const uint16_t *Wd;
  int64_t ldw;
  int64_t n, k, tpr, T;
  int R;  // tile-row bands
  // operands
  const uint16_t *X;
  int64_t ldx;
  int batch;
  void *Y;
  int64_t ldy;
  int ydt;
  // low rank: t = V^T x and then ut = U t (fp32 [batch][n]) are computed by
  // two small kernels before the product; the product's epilogue adds ut
  const uint16_t *U;
  int64_t ldu;
  int rank;
  const float *lr_t;
  const float *lr_ut;
  // split
  int G;
  int64_t total;  // packed bytes of the whole matrix
  float *partials;
  uint32_t *counters;
  uint32_t *status;  // workspace status word
  int64_t nvb, nmb;  // bytes of the value and mask buffers
  // 1: launched as a programmatic dependent of the preceding kernel on the
  // stream.  The weights (packed matrix or row-major W) may then be read
  // before that kernel has finished; X, Y, the workspace and the low-rank
  // intermediates are touched only after griddepcontrol.wait.
  // 2: the same, behind the low-rank kernels of the same call, which start
  // only once all work before the call has finished: X may be read at once,
  // and only the epilogue (Y, workspace, U t) waits.
  int pdl;
};

// Programmatic dependent launch (sm_90+): let the next grid on the stream, if
// it was launched as a programmatic dependent, start its CTAs as this grid's
// CTAs exit; and wait until the preceding grid has completed and its memory
// is visible.  Both are no-ops for a grid launched without the attribute.
__device__ __forceinline__ void grid_dep_trigger() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
__device__ __forceinline__ void grid_dep_wait() {
  asm volatile("griddepcontrol.wait;" ::: "memory");
}

// Work split made once per matrix (hyb_make_plan) and handed to the streaming
// kernel as launch parameters, so that a CTA issues its first copy without
// any global-memory load.  Host layout (int64): [0] = G, [1] = kind (1),
// [2..7] reserved, then G + 1 records {t0, val_off[t0], meta_off[t0], 2:4
// bits of tiles t0 .. t0 + 30 (low word) and the stage starts of that first
// window (high word)}, t0 being the CTA's first tile; record G holds the end
// (T).
constexpr int kMaxCtas = 160;
constexpr int kPlanHead = 8;
constexpr int32_t kPlanTiles = 1;
struct LaunchPlan {
  int32_t kind;  // 0: none (the kernel searches for its range)
  int32_t ctas;
  int64_t rec[4 * (kMaxCtas + 1)];
};

// ---------------------------------------------------------------------------
// helpers
// ---------------------------------------------------------------------------

template <int BP>
struct XRegs {
  uint4 v[BP][2];  // 16 bf16 per batch column
};

// Select x[p0] and x[p1] of one group from its 4-bit mask (two bits set):
// p0 is the lowest set bit, p1 the highest.
__device__ __forceinline__ void pick2(uint32_t nib, float x0, float x1,
                                      float x2, float x3, float &xa,
                                      float &xb) {
  xa = (nib & 1u) ? x0 : ((nib & 2u) ? x1 : x2);
  xb = (nib & 8u) ? x3 : ((nib & 4u) ? x2 : x1);
}

__device__ __forceinline__ void unpack16(const uint4 &a, const uint4 &b,
                                         float f[16]) {
  const uint32_t w[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    f[2 * i] = bf16_lo(w[i]);
    f[2 * i + 1] = bf16_hi(w[i]);
  }
}

__device__ __forceinline__ int owner_of(int64_t P, const Params &p) {
  int64_t o = (P * p.G) / p.total;
  return (int)(o < p.G - 1 ? o : p.G - 1);
}

// Epilogue for one (row, batch) output: add the low-rank term, store.
__device__ __forceinline__ void store_out(const Params &p, int64_t row, int b,
                                          float y) {
  if (p.lr_ut != nullptr) y += p.lr_ut[(int64_t)b * p.n + row];
  if (p.ydt == HYB_BF16)
    reinterpret_cast<uint16_t *>(p.Y)[(int64_t)b * p.ldy + row] =
        f32_to_bf16_rne(y);
  else
    reinterpret_cast<float *>(p.Y)[(int64_t)b * p.ldy + row] = y;
}

// ---------------------------------------------------------------------------
// dense GEMV baseline: row-major bf16 W, CTA c takes tiles
// [c, c+1) * T / G (all tiles cost the same); warp w owns rows [w*R, (w+1)*R)
// of a tile and a lane 16 columns of one row per step; the next tile is
// loaded into registers while the current one computes
// ---------------------------------------------------------------------------

template <int BP, int B1, int B2>
struct Cfg {
  static constexpr int RW = B1 / kWarps;    // rows per warp per tile
  static constexpr int CPR = B2 / 16;       // lanes per row (16 columns each)
  static constexpr int RPS = 32 / CPR;      // rows per warp step
  static constexpr int JS = RW / RPS;       // steps per warp per tile
  static constexpr int XB = BP < 4 ? BP : 4;  // batch columns per x sub-block
  static constexpr int64_t kDenseCost = 2LL * B1 * B2;
  static constexpr int kMinBlocks = BP <= 1 ? 2 : 1;
  static_assert(RW * kWarps == B1, "b1 must split over the warps");
  static_assert(RPS * CPR == 32 && JS * RPS == RW, "tile shape");
};

// Registers of one tile in flight: 32 B (16 bf16) per lane per step.
template <int JS>
struct TileRegs {
  uint4 a[JS];
  uint4 b[JS];
};

template <int BP, int B1, int B2>
__global__ void __launch_bounds__(kThreads, (Cfg<BP, B1, B2>::kMinBlocks))
    dense_gemv_kernel(const Params p) {
  using C = Cfg<BP, B1, B2>;
  constexpr int JS = C::JS;
  extern __shared__ int s_owner[];  // [2 * R]: owner CTA of each band's first / last tile
  __shared__ float s_acc[B1 * BP];
  __shared__ int64_t s_range[2];
  __shared__ int s_last;

  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  const int cp = lane % C::CPR;  // 16-column part
  const int rs = lane / C::CPR;  // row inside a step
  const int c = blockIdx.x;
  const int G = p.G;
  if (p.pdl) grid_dep_trigger();

  // ---- 1. this CTA's tile range [t0, t1) -----------------------------------
  const int64_t tgtA = (int64_t)c * p.total;
  const int64_t tgtB = (int64_t)(c + 1) * p.total;
  // uniform tiles: the split is a closed form
  const int64_t unit = C::kDenseCost * G;
  int64_t t0 = (tgtA + unit - 1) / unit;
  int64_t t1 = (c == G - 1) ? p.T : (tgtB + unit - 1) / unit;
  for (int i = tid; i < p.R; i += kThreads) {
    s_owner[2 * i] = owner_of((int64_t)i * p.tpr * C::kDenseCost, p);
    s_owner[2 * i + 1] = owner_of(((int64_t)(i + 1) * p.tpr - 1) * C::kDenseCost, p);
  }
  if (tid == 0) {
    s_range[0] = t0;
    s_range[1] = t1;
  }
  __syncthreads();
  t0 = s_range[0];
  t1 = s_range[1];

  // ---- 2. stream the tiles --------------------------------------------------
  float acc[JS][BP];
#pragma unroll
  for (int j = 0; j < JS; ++j)
#pragma unroll
    for (int b = 0; b < BP; ++b) acc[j][b] = 0.f;

  const int wrow = warp * C::RW;  // first row of this warp inside a tile

  // a lane's 16 columns of JS rows of a tile of the row-major W
  auto load_tile = [&](int64_t t, TileRegs<JS> &r) {
    const int64_t tr = t / p.tpr, tc = t - tr * p.tpr;
    const uint16_t *base = p.Wd + (tr * B1 + wrow + rs) * p.ldw + tc * B2 + 16 * cp;
#pragma unroll
    for (int j = 0; j < JS; ++j) ld_stream32(base + (int64_t)j * C::RPS * p.ldw, r.a[j], r.b[j]);
  };
  auto load_x = [&](int64_t t, int b0, XRegs<C::XB> &xr) {
    const int64_t tc = t % p.tpr;
    const uint16_t *xp = p.X + tc * B2 + 16 * cp;
#pragma unroll
    for (int b = 0; b < C::XB; ++b) {
      if (b0 + b < p.batch) {
        xr.v[b][0] = ld_keep16(xp + (int64_t)(b0 + b) * p.ldx);
        xr.v[b][1] = ld_keep16(xp + (int64_t)(b0 + b) * p.ldx + 8);
      } else {
        xr.v[b][0] = make_uint4(0, 0, 0, 0);
        xr.v[b][1] = make_uint4(0, 0, 0, 0);
      }
    }
  };

  // flush the accumulators of band r: lanes -> shared -> slot or epilogue
  auto flush = [&](int r) {
#pragma unroll
    for (int j = 0; j < JS; ++j)
#pragma unroll
      for (int b = 0; b < BP; ++b) {
        float v = acc[j][b];
#pragma unroll
        for (int o = 1; o < C::CPR; o <<= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
        acc[j][b] = v;
      }
    if (cp == 0) {
#pragma unroll
      for (int j = 0; j < JS; ++j)
#pragma unroll
        for (int b = 0; b < BP; ++b)
          s_acc[(wrow + j * C::RPS + rs) * BP + b] = acc[j][b];
    }
#pragma unroll
    for (int j = 0; j < JS; ++j)
#pragma unroll
      for (int b = 0; b < BP; ++b) acc[j][b] = 0.f;
    __syncthreads();
    const int oA = s_owner[2 * r], oB = s_owner[2 * r + 1];
    const int64_t row0 = (int64_t)r * B1;
    if (oA == oB) {
      // this CTA owns the whole band
      for (int i = tid; i < B1 * BP; i += kThreads) {
        const int row = i % B1, b = i / B1;
        if (b < p.batch) store_out(p, row0 + row, b, s_acc[row * BP + b]);
      }
    } else {
      float *slot = p.partials + (int64_t)(c + r) * (B1 * BP);
      for (int i = tid; i < B1 * BP; i += kThreads) __stcg(slot + i, s_acc[i]);
      __threadfence();
      __syncthreads();
      if (tid == 0) {
        const uint32_t prev = atomicAdd(p.counters + r, 1u);
        s_last = prev == (uint32_t)(oB - oA);
      }
      __syncthreads();
      if (s_last) {
        __threadfence();
        for (int i = tid; i < B1 * BP; i += kThreads) {
          const int row = i % B1, b = i / B1;
          if (b >= p.batch) continue;
          float y = 0.f;
          for (int cc = oA; cc <= oB; ++cc)
            y += __ldcg(p.partials + (int64_t)(cc + r) * (B1 * BP) + row * BP + b);
          store_out(p, row0 + row, b, y);
        }
        if (tid == 0) p.counters[r] = 0;  // ready for the next call
      }
    }
    __syncthreads();
  };

  if (t0 < t1) {
    TileRegs<JS> cur;
    load_tile(t0, cur);
    // the first tile of W is on its way; X and everything written below may
    // belong to the preceding grid
    if (p.pdl) grid_dep_wait();
    XRegs<C::XB> xcur;
    if (BP <= 4) load_x(t0, 0, xcur);
    for (int64_t t = t0; t < t1; ++t) {
      TileRegs<JS> nxt;
      XRegs<C::XB> xnxt;
      if (t + 1 < t1) {
        load_tile(t + 1, nxt);
        if (BP <= 4) load_x(t + 1, 0, xnxt);
      }
      // ---- compute tile t ----
#pragma unroll
      for (int b0 = 0; b0 < BP; b0 += C::XB) {
        XRegs<C::XB> xs;
        if (BP <= 4) {
          xs = xcur;
        } else {
          load_x(t, b0, xs);
        }
        float xf[C::XB][16];
#pragma unroll
        for (int b = 0; b < C::XB; ++b) unpack16(xs.v[b][0], xs.v[b][1], xf[b]);
#pragma unroll
        for (int j = 0; j < JS; ++j) {
          float wf[16];
          unpack16(cur.a[j], cur.b[j], wf);
#pragma unroll
          for (int e = 0; e < 16; ++e)
#pragma unroll
            for (int b = 0; b < C::XB; ++b)
              acc[j][b0 + b] = fmaf(wf[e], xf[b][e], acc[j][b0 + b]);
        }
      }
      // band boundary or end of range: flush
      if (t + 1 == t1 || (t + 1) % p.tpr == 0) flush((int)(t / p.tpr));
      cur = nxt;
      xcur = xnxt;
    }
  }
}

// ---------------------------------------------------------------------------
// the TMA-ring kernel for packed hybrid matrices
// ---------------------------------------------------------------------------
//
// One CTA per SM.  CTA c owns the tiles whose packed byte offset falls in
// [c, c+1) * total / G -- a contiguous piece of the packed stream, taken from
// the launch-parameter plan (or, without one, found by two rounds of parallel
// search over the tile offsets at start-up).  A producer warp copies that
// piece stage by stage (the values and masks of one to TPX tiles and the
// matching slice of X) from HBM into a ring of shared-memory stages with 1-D
// bulk copies (cp.async.bulk; X through a 2-D tensor map at batch >= 4;
// completion counted on an mbarrier), so the bytes in flight are set by the
// ring, not by registers.  B1/RW consumer warps, RW tile rows each, compute
// from shared memory and keep fp32 row sums in registers until their piece of
// a tile-row band ends.
//
// A band piece goes to one of two epilogue warps (alternating), which stores
// a band this CTA owns outright, or writes the piece to fp32 slot c + r; a
// ticket per band finds the last of its CTAs, whose epilogue warp sums the
// band's slots in CTA order (deterministic; nothing spins, and the consumers
// go on with the next piece meanwhile).
//
// Products use the mixed-precision FMA of sm_100 (bf16 x bf16 + fp32 -> fp32,
// exact product) straight on packed bf16 pairs, and PRMT picks the two x
// values of a 2:4 group from its 4-bit mask ("SparseDecoding", authors'
// abstract: bitmask-indexed N:M SpMV); the PRMT selector comes from two more
// PRMTs at batch <= 4 and from a 16-entry shared table above.  Masks are
// expected to have two bits set (as hyb_pack writes them); any other mask
// still selects within the group's four values.

constexpr uint32_t kWaitLimit = 1u << 22;

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
  return (uint32_t)__cvta_generic_to_shared(p);
}
__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count)
               : "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t tx) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
               "r"(tx)
               : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}
// Every wait is bounded: on expiry the caller records kStatusTimeout and
// leaves the pipeline instead of waiting for ever.
__device__ __forceinline__ bool mbar_wait_limit(uint64_t *bar, uint32_t parity,
                                                uint32_t limit) {
  for (uint32_t i = 0; i < limit; ++i)
    if (mbar_try_wait(bar, parity)) return true;
  return false;
}
__device__ __forceinline__ bool mbar_wait(uint64_t *bar, uint32_t parity) {
  return mbar_wait_limit(bar, parity, kWaitLimit);
}
__device__ __forceinline__ int64_t ld_volatile_nc64(const int64_t *addr) {
  int64_t v;
  asm volatile("ld.global.nc.s64 %0, [%1];" : "=l"(v) : "l"(addr));
  return v;
}
__device__ __forceinline__ uint32_t ld_volatile_nc8(const uint8_t *addr) {
  uint32_t v;
  asm volatile("ld.global.nc.u8 %0, [%1];" : "=r"(v) : "l"(addr));
  return v;
}
__device__ __forceinline__ uint32_t atom_add_acq_rel(uint32_t *addr, uint32_t v) {
  uint32_t old;
  asm volatile("atom.acq_rel.gpu.global.add.u32 %0, [%1], %2;" : "=r"(old) : "l"(addr), "r"(v)
               : "memory");
  return old;
}
__device__ __forceinline__ void bulk_g2s(void *dst, const void *src, uint32_t bytes,
                                         uint64_t *bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::
          "r"(smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}
// 2-D tiled TMA load of box (x, y) of the tensor map into shared memory,
// completion counted on the mbarrier (no multicast).
__device__ __forceinline__ void tma_load_2d(void *dst, const CUtensorMap *map, int x, int y,
                                            uint64_t *bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3}], [%4];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_u32(bar))
      : "memory");
}
// acc += lo(w) * lo(x) + hi(w) * hi(x) on two packed bf16 pairs.
__device__ __forceinline__ void fma_bf16x2(float &acc, uint32_t w, uint32_t x) {
  unsigned short wl, wh, xl, xh;
  asm("mov.b32 {%0,%1}, %2;" : "=h"(wl), "=h"(wh) : "r"(w));
  asm("mov.b32 {%0,%1}, %2;" : "=h"(xl), "=h"(xh) : "r"(x));
  asm("fma.rn.f32.bf16 %0, %1, %2, %0;" : "+f"(acc) : "h"(wl), "h"(xl));
  asm("fma.rn.f32.bf16 %0, %1, %2, %0;" : "+f"(acc) : "h"(wh), "h"(xh));
}

template <int BP, int B1, int B2>
struct TmaCfg {
  // rows per consumer warp: 8, or 16 for wide batches so that the 17-warp
  // register budget (96 per thread) is not exceeded by the accumulators
  static constexpr int RW = BP >= 8 ? 16 : 8;
  static constexpr int NC = B1 / RW;                // consumer warps
  static constexpr int CPR = B2 / 16;               // lanes per row, 16 columns each
  static constexpr int RPS = 32 / CPR;              // rows per warp step
  static constexpr int JS = RW / RPS;               // steps per warp per tile
  static constexpr int XB = BP < 4 ? BP : 4;        // batch columns per pass
  // A stage holds 32 KB of values: TPD dense tiles, or up to 2*TPD tiles
  // when some are 2:4 (a 2:4 tile has half the bytes), so that every stage
  // in the ring carries about the same number of bytes.
  static constexpr int TPD = (16384 / (B1 * B2)) > 0 ? 16384 / (B1 * B2) : 1;
  static constexpr int TPX = 2 * TPD;                         // tiles per stage, at most
  static constexpr int WIN = 31;                    // tiles per producer offset window
  static constexpr int kValsBytes = 2 * B1 * B2 * TPD;        // 32 KB
  static constexpr int kMetaBytes = B1 * B2 / 8 * TPX;        // 4 KB
  // X slices of a stage: with XTM (batch >= 4) one 2-D tensor copy fetches
  // XT tiles' columns for all BP batch rows at once (box [BP][XT B2]);
  // otherwise one 1-D copy per batch row.  Layout [copy][batch][XT B2].
  static constexpr bool XTM = BP >= 4;
  static constexpr int XT0 = 256 / B2 < TPX ? 256 / B2 : TPX;
  static constexpr int XT = XTM ? XT0 : TPX;                 // tiles per X copy
  static constexpr int kXBatch = 2 * B2 * XT;                // bytes between batch rows
  static constexpr int kXCopy = BP * kXBatch;                // bytes of one X copy group
  static constexpr int kXRegion = (TPX / XT) * kXCopy;       // = BP * 2 * B2 * TPX
  static constexpr int kStageBytes = kValsBytes + kMetaBytes + kXRegion;
  static constexpr int kStages =
      (200 * 1024 / kStageBytes) < 6 ? (200 * 1024 / kStageBytes) : 6;
  static constexpr int kThreads = (NC + 3) * 32;  // consumers, producer, 2 epilogue warps
  static constexpr size_t kSmem = (size_t)kStages * kStageBytes + 1024;
  static_assert(RPS * CPR == 32 && JS * RPS == RW && JS >= 1, "tile shape");
  static_assert(kStages >= 3, "ring too short");
  static_assert(TPX <= 8 && WIN < 32, "stage / offset window");
  static_assert(TPX % XT == 0 && (!XTM || XT * B2 <= 256), "X copy groups");
};

// Stage starts of a window of nw tiles beginning at tile w0 (bit i: a stage
// starts at tile w0 + i): greedy packing by value bytes, in units of a 2:4
// tile (a dense tile is 2), at most 2 tpd units and tpx tiles per stage, and
// a new stage at every band start.  Used by the streaming kernel for every
// window and by the plan for each CTA's first window.
__device__ __forceinline__ uint32_t stage_starts(uint32_t spm, int nw, int64_t w0, int tpr,
                                                int tpd, int tpx) {
  int nb = (int)((tpr - w0 % tpr) % tpr);  // first band start at or after w0, relative
  uint32_t starts = 0;
  int fill = 2 * tpx, cnt = tpx;  // force a start at tile 0
  for (int i = 0; i < nw; ++i) {
    const int sz = (spm >> i & 1u) ? 1 : 2;
    const bool band_start = i == nb;
    if (band_start) nb += tpr;
    if (band_start || fill + sz > 2 * tpd || cnt == tpx) {
      starts |= 1u << i;
      fill = 0;
      cnt = 0;
    }
    fill += sz;
    ++cnt;
  }
  return starts;
}

struct StageDesc {
  int64_t t0;       // first tile of the stage
  uint16_t ntiles;  // tiles in the stage (<= TPX, never across a band)
  uint8_t sparse;   // bit i: tile i is 2:4
  uint8_t flags;    // 1: last stage of this CTA's piece of a band, 2: end of work
};

template <int BP, int B1, int B2>
__global__ void __launch_bounds__(TmaCfg<BP, B1, B2>::kThreads, 1)
    hybrid_tma_kernel(const Params p, const LaunchPlan lp, const __grid_constant__ CUtensorMap xmap) {
  using C = TmaCfg<BP, B1, B2>;
  constexpr int S = C::kStages;
  extern __shared__ __align__(1024) uint8_t smem[];
  __shared__ __align__(8) uint64_t full_bar[S];
  __shared__ __align__(8) uint64_t empty_bar[S];
  __shared__ StageDesc desc[S];
  __shared__ uint32_t sel_lut[16];
  __shared__ uint32_t s_cnt[2];
  __shared__ int64_t s_range[2];
  // a CTA's piece of a band: row sums handed from the consumer warps to the
  // epilogue warp through a 2-slot ring, [slot][warp][b * RW + row]
  __shared__ float s_rows[2][C::NC][C::RW * BP];
  __shared__ __align__(8) uint64_t piece_full[2];
  __shared__ __align__(8) uint64_t piece_empty[2];

  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  const int c = blockIdx.x;
  const int G = p.G;
  const int tpr = (int)p.tpr;
  // The plan record is read first thing and parked in shared memory before
  // the first barrier, so that its constant-bank line is fetched while the
  // barriers are set up rather than when the producer first needs it.
  __shared__ int64_t s_rec[5];
  const bool planned = lp.kind == kPlanTiles;
  if (p.pdl) grid_dep_trigger();
  if (planned && tid == 32 * C::NC + 1) {
    s_rec[0] = lp.rec[4 * c];
    s_rec[1] = lp.rec[4 * (c + 1)];
    s_rec[2] = lp.rec[4 * c + 1];
    s_rec[3] = lp.rec[4 * c + 2];
    s_rec[4] = lp.rec[4 * c + 3];
  }
  if (tid == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&full_bar[s], 1);
      mbar_init(&empty_bar[s], C::NC);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&piece_full[s], C::NC);
      mbar_init(&piece_empty[s], 1);
    }
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    s_cnt[0] = 0;
    s_cnt[1] = 0;
  }
  if (tid < 16) {
    // PRMT selector moving bf16 x[p0] to the low and x[p1] to the high half,
    // p0 < p1 the set bits of the mask (x0x1 in bytes 0-3, x2x3 in 4-7)
    const uint32_t m = tid;
    uint32_t p0 = 0, p1 = 0;
    if (m) {
      p0 = __ffs(m) - 1;
      p1 = 31 - __clz(m);
    }
    sel_lut[m] = (2 * p0) | ((2 * p0 + 1) << 4) | ((2 * p1) << 8) | ((2 * p1 + 1) << 12);
  }
  __syncthreads();

  // ---- this CTA's tiles [t0, t1): tiles whose packed offset P(t) satisfies
  // c*total <= P(t)*G < (c+1)*total.  With a plan the producer and the
  // epilogue warp take them from the launch parameters; otherwise round 1
  // brackets both ends between band starts and round 2 counts inside the
  // bracketing band. ----
  if (!planned) {
      const int64_t tgtA = (int64_t)c * p.total, tgtB = (int64_t)(c + 1) * p.total;
      uint32_t ca = 0, cb = 0;
      for (int i = tid; i <= p.R; i += blockDim.x) {
        const int64_t t = (int64_t)i * tpr;
        const int64_t P = 2 * __ldg(p.val_off + t) + __ldg(p.meta_off + t);
        ca += P * G < tgtA;
        cb += P * G < tgtB;
      }
      ca = __reduce_add_sync(0xffffffffu, ca);
      cb = __reduce_add_sync(0xffffffffu, cb);
      if (lane == 0) {
        atomicAdd(&s_cnt[0], ca);
        atomicAdd(&s_cnt[1], cb);
      }
      __syncthreads();
      const uint32_t bA = s_cnt[0], bB = s_cnt[1];  // band starts below each target
      __syncthreads();
      if (tid == 0) {
        s_cnt[0] = 0;
        s_cnt[1] = 0;
      }
      __syncthreads();
      ca = 0;
      cb = 0;
      const int64_t baseA = bA > 0 ? (int64_t)(bA - 1) * tpr : 0;
      const int64_t baseB = bB > 0 ? (int64_t)(bB - 1) * tpr : 0;
      for (int i = tid; i < tpr; i += blockDim.x) {
        if (bA > 0) {
          const int64_t t = baseA + i;
          ca += (2 * __ldg(p.val_off + t) + __ldg(p.meta_off + t)) * G < tgtA;
        }
        if (bB > 0) {
          const int64_t t = baseB + i;
          cb += (2 * __ldg(p.val_off + t) + __ldg(p.meta_off + t)) * G < tgtB;
        }
      }
      ca = __reduce_add_sync(0xffffffffu, ca);
      cb = __reduce_add_sync(0xffffffffu, cb);
      if (lane == 0) {
        atomicAdd(&s_cnt[0], ca);
        atomicAdd(&s_cnt[1], cb);
      }
      __syncthreads();
      if (tid == 0) {
        s_range[0] = bA > 0 ? baseA + s_cnt[0] : 0;
        s_range[1] = (c == G - 1) ? p.T : (bB > 0 ? baseB + s_cnt[1] : 0);
      }
      __syncthreads();
  }
  // consumers never need the range; the producer and the epilogue warp take
  // it from the plan record when there is one
  int64_t t0 = 0, t1 = 0;
  if (!planned) {
    t0 = s_range[0];
    t1 = s_range[1];
  } else if (warp >= C::NC) {
    t0 = s_rec[0];
    t1 = s_rec[1];
  }

  if (warp == C::NC) {
    // ------------------------------ producer ------------------------------
    if constexpr (C::XTM) {
      // bring the X tensor map's descriptor into the TMA unit's cache once
      if (lane == 0)
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&xmap))
                     : "memory");
    }
    // Tiles are taken in windows of WIN: lane i holds the packed offsets of
    // tile w0 + i (and lane WIN those of the window's end), the next window
    // is loaded while this one is issued.  Stages are packed greedily inside
    // a window: a new stage starts at a band start or when the next tile no
    // longer fits in the 32 KB value buffer; every lane runs the same packing
    // over the window's 2:4 bitmask, so all agree on the stage starts.
    struct Win {
      int64_t vo, mo;
      uint32_t sp;
    };
    // (volatile loads: the compiler may not turn the window load that a
    // plan makes unnecessary into a speculative load the first window waits on)
    auto load_win = [&](int64_t w0) -> Win {
      Win o{0, 0, 0};
      const int64_t t = w0 + lane;
      if (lane <= C::WIN && t <= t1) {
        o.vo = ld_volatile_nc64(p.val_off + t);
        o.mo = ld_volatile_nc64(p.meta_off + t);
      }
      if (lane < C::WIN && t < t1) o.sp = ld_volatile_nc8(p.map + t) == 1;
      return o;
    };
    int stage = 0;
    uint32_t phase = 0;
    bool ok = true;
    uint32_t armed = 0, armed_parity = 0;  // per stage: copies issued / phase parity
    // X of a stage: whole tensor-map boxes (rows past the batch and columns
    // past k are zero-filled and counted in the transaction bytes), or one
    // 1-D copy per batch row
    auto issue_x = [&](int st_i, int64_t xcol, int nt) {
      uint8_t *xdst = smem + (size_t)st_i * C::kStageBytes + C::kValsBytes + C::kMetaBytes;
      if constexpr (C::XTM) {
        const int ngx = (nt + C::XT - 1) / C::XT;
        for (int q = 0; q < ngx; ++q)
          tma_load_2d(xdst + q * C::kXCopy, &xmap, (int)(xcol + q * C::XT * B2), 0,
                      &full_bar[st_i]);
      } else {
        const uint32_t xrow = (uint32_t)(2 * B2 * nt);
        for (int b = 0; b < p.batch; ++b)
          bulk_g2s(xdst + b * C::kXBatch, p.X + xcol + (int64_t)b * p.ldx, xrow, &full_bar[st_i]);
      }
    };
    // As a programmatic dependent, the first ring's worth of stages gets its
    // weight bytes requested at once and its X only after the preceding grid
    // has finished (it may have written X); the lane that armed a stage keeps
    // the stage's X request until then.  Warp-uniform: pend, issued.
    bool pend = p.pdl == 1;
    int issued = 0;
    int dx_stage = -1, dx_nt = 0;
    int64_t dx_col = 0;
    auto release_x = [&]() {
      grid_dep_wait();
      if (dx_stage >= 0) issue_x(dx_stage, dx_col, dx_nt);
      dx_stage = -1;
      pend = false;
    };
    Win cur;
    bool derived = false;
    if (planned) {
      // first window from the plan: offsets of tile t0 + lane follow from
      // those of t0 and the 2:4 bits of the tiles before it
      constexpr int64_t TE = (int64_t)B1 * B2;
      const uint32_t bits = (uint32_t)s_rec[4];
      const int nb = __popc(bits & ((1u << lane) - 1u));
      cur.vo = s_rec[2] + (int64_t)lane * TE - nb * (TE / 2);
      cur.mo = s_rec[3] + nb * (TE / 8);
      cur.sp = lane < C::WIN ? (bits >> lane) & 1u : 0u;
      // a plan that does not fit the buffers is not used
      const int nw = (int)min((int64_t)C::WIN, t1 - t0);
      derived = 2 * __shfl_sync(0xffffffffu, cur.vo, nw) <= p.nvb &&
                __shfl_sync(0xffffffffu, cur.mo, nw) <= p.nmb && cur.vo >= 0;
      derived = __all_sync(0xffffffffu, derived);
    }
    if (!derived) cur = load_win(t0);
    for (int64_t w0 = t0; ok && w0 < t1; w0 += C::WIN) {
      const Win nxt = load_win(w0 + C::WIN);  // in flight while this window issues
      const int nw = (int)min((int64_t)C::WIN, t1 - w0);
      const uint32_t spm = __ballot_sync(0xffffffffu, cur.sp != 0);
      // stage starts: the plan's for the first window (checked against the
      // stage limits lane by lane), else the greedy packing
      uint32_t starts = 0;
      bool have = false;
      if (derived && w0 == t0) {
        starts = (uint32_t)((uint64_t)s_rec[4] >> 32);
        const uint32_t nxt_s = lane < 31 ? starts >> (lane + 1) : 0u;
        const int e = nxt_s ? lane + __ffs(nxt_s) : nw;  // end of the stage starting here
        const uint32_t in = e > lane ? ((e - lane >= 32 ? ~0u : (1u << (e - lane)) - 1u)) : 0u;
        const int units = 2 * (e - lane) - __popc((spm >> lane) & in);
        const bool good = lane >= nw || !(starts >> lane & 1u) ||
                          (e - lane <= C::TPX && units <= 2 * C::TPD);
        const bool band_ok = lane >= nw || (w0 + lane) % tpr != 0 || (starts >> lane & 1u);
        have = __all_sync(0xffffffffu, good && band_ok) && (starts & 1u) && (starts >> nw) == 0;
      }
      if (!have) starts = stage_starts(spm, nw, w0, tpr, C::TPD, C::TPX);
      // the stage that starts at this lane: tiles [w0 + lane, w0 + e)
      const bool is_start = lane < nw && (starts >> lane & 1u);
      const uint32_t later = lane < 31 ? (starts >> (lane + 1)) : 0u;
      const int e = later ? lane + 1 + __ffs(later) - 1 : nw;
      const int64_t v_end = __shfl_sync(0xffffffffu, cur.vo, e & 31);
      const int64_t m_end = __shfl_sync(0xffffffffu, cur.mo, e & 31);
      // (e == 32 only when nw == 32, which WIN < 32 rules out)
      uint32_t todo = starts;
      while (todo) {
        const int k = __ffs(todo) - 1;
        todo &= todo - 1;
        if (pend && issued == S) release_x();  // the ring is armed: X can wait no longer
        if (lane == k && is_start) {
          if (!mbar_wait(&empty_bar[stage], phase ^ 1u)) {
            ok = false;
          } else {
            uint8_t *st = smem + (size_t)stage * C::kStageBytes;
            const int64_t ts = w0 + k, te = w0 + e;
            const uint32_t vbytes = (uint32_t)(2 * (v_end - cur.vo));
            const uint32_t mbytes = (uint32_t)(m_end - cur.mo);
            const int nt = e - k;
            const uint32_t xrow = (uint32_t)(2 * B2 * nt);
            const int ngx = (nt + C::XT - 1) / C::XT;  // X copy groups (tensor path)
            const uint32_t xbytes =
                C::XTM ? (uint32_t)(ngx * C::kXCopy) : xrow * (uint32_t)p.batch;
            const int64_t band = ts / tpr;
            StageDesc d;
            d.t0 = ts;
            d.ntiles = (uint16_t)nt;
            d.sparse = (uint8_t)((spm >> k) & ((1u << nt) - 1u));
            d.flags = (te == (band + 1) * tpr || te == t1) ? 1 : 0;
            desc[stage] = d;
            armed |= 1u << stage;
            armed_parity = (armed_parity & ~(1u << stage)) | (phase << stage);
            mbar_arrive_expect_tx(&full_bar[stage], vbytes + mbytes + xbytes);
            bulk_g2s(st, p.vals + 2 * cur.vo, vbytes, &full_bar[stage]);
            if (mbytes) bulk_g2s(st + C::kValsBytes, p.meta + cur.mo, mbytes, &full_bar[stage]);
            const int64_t xcol = (ts - band * tpr) * B2;  // first X column of the stage
            if (pend) {
              dx_stage = stage;
              dx_col = xcol;
              dx_nt = nt;
            } else {
              issue_x(stage, xcol, nt);
            }
          }
        }
        // every lane keeps the ring position
        ++issued;
        if (++stage == S) {
          stage = 0;
          phase ^= 1u;
        }
      }
      if (pend) release_x();  // at the latest after the first window
      ok = __all_sync(0xffffffffu, ok);
      cur = nxt;
    }
    if (pend) release_x();  // (no window at all)
    // lanes kept identical ring positions; lane 0 closes the ring
    if (lane == 0) {
      if (ok && mbar_wait(&empty_bar[stage], phase ^ 1u)) {
        StageDesc d{};
        d.flags = 2;
        desc[stage] = d;
        mbar_arrive(&full_bar[stage]);
      } else {
        ok = false;
      }
    }
    if (!__all_sync(0xffffffffu, ok)) {
      if (lane == 0) atomicOr(p.status, kStatusTimeout);
      // let every copy already issued land before the CTA's shared memory
      // goes away (bounded, like every other wait); each lane drains the
      // stages it armed
      for (int s2 = 0; s2 < S; ++s2)
        if (armed >> s2 & 1u) mbar_wait(&full_bar[s2], armed_parity >> s2 & 1u);
    }
    return;
  }

  if (warp >= C::NC + 1) {
    // ------------------------------ epilogue ------------------------------
    // Takes every piece of band this CTA finishes, in band order, pieces
    // alternating between the two epilogue warps so that one piece's ticket
    // round trip does not hold up the next: a whole band goes straight to Y
    // (with the low-rank term); a band shared with other CTAs goes to slot
    // c + r, and a ticket per band finds the last of its CTAs, which sums the
    // band's slots in CTA order (deterministic).  All global-memory ordering
    // (release, acquire) happens here, off the consumer warps' path.
    // Y, the slots, the tickets and the low-rank term may belong to the
    // preceding grid until it has finished.
    if (p.pdl) grid_dep_wait();
    auto owner_of_p = [&](int64_t P) -> int {
      const int64_t o = (P * G) / p.total;
      return (int)(o < G - 1 ? o : G - 1);
    };
    constexpr int OPL = 4, QMAX = 8;  // outputs per lane, contributors per load round
    const int ew = warp - (C::NC + 1);
    const int r_first = (int)(t0 / tpr), r_last = t1 > t0 ? (int)((t1 - 1) / tpr) : r_first - 1;
    for (int r = r_first + ew; r <= r_last; r += 2) {
      const int piece = r - r_first;
      const int slot = piece & 1;
      const uint32_t ph = (uint32_t)(piece >> 1) & 1u;
      const bool whole = t0 <= (int64_t)r * tpr && t1 >= (int64_t)(r + 1) * tpr;
      // owners of the band's first and last tile, fetched before the wait
      int oA = 0, oB = 0;
      if (!whole && lane == 0) {
        const int64_t ta = (int64_t)r * tpr, tb = ta + tpr - 1;
        oA = owner_of_p(2 * __ldg(p.val_off + ta) + __ldg(p.meta_off + ta));
        oB = owner_of_p(2 * __ldg(p.val_off + tb) + __ldg(p.meta_off + tb));
      }
      if (!mbar_wait(&piece_full[slot], ph)) {
        if (lane == 0) atomicOr(p.status, kStatusTimeout);
        break;
      }
      const float(*rows)[C::RW * BP] = s_rows[slot];
      const int64_t row0 = (int64_t)r * B1;
      if (whole) {
        for (int o = lane; o < B1 * BP; o += 32) {
          const int row = o % B1, b = o / B1;
          if (b < p.batch) store_out(p, row0 + row, b, rows[row / C::RW][b * C::RW + row % C::RW]);
        }
      } else {
        float *slotp = p.partials + (int64_t)(c + r) * BP * B1;
        for (int o = lane; o < B1 * BP; o += 32) {
          const int row = o % B1, b = o / B1;
          __stcg(slotp + b * B1 + row, rows[row / C::RW][b * C::RW + row % C::RW]);
        }
        // The warp barrier orders every lane's slot stores before lane 0's
        // ticket; the ticket's release side (acq_rel, cumulative) publishes
        // them at gpu scope, and its acquire side covers the reads of the
        // other CTAs' slots if this CTA turns out to be last -- the pattern of
        // a split-K semaphore, with no full fence per lane.
        __syncwarp();
        uint32_t last = 0;
        if (lane == 0) last = atom_add_acq_rel(p.counters + r, 1u) == (uint32_t)(oB - oA);
        last = __shfl_sync(0xffffffffu, last, 0);
        oA = __shfl_sync(0xffffffffu, oA, 0);
        oB = __shfl_sync(0xffffffffu, oB, 0);
        if (last) {
          __syncwarp();
          // sum the band's slots in CTA order; the loads of 4 outputs x 8
          // contributors are issued together, then added in a fixed order
          for (int o0 = 0; o0 < B1 * BP; o0 += 32 * OPL) {
            float y[OPL];
#pragma unroll
            for (int u = 0; u < OPL; ++u) y[u] = 0.f;
            for (int q0 = oA; q0 <= oB; q0 += QMAX) {
              float v[OPL][QMAX];
#pragma unroll
              for (int u = 0; u < OPL; ++u) {
                const int o = o0 + u * 32 + lane;
                const int row = o % B1, b = o / B1;
#pragma unroll
                for (int q = 0; q < QMAX; ++q)
                  v[u][q] = (o < B1 * BP && q0 + q <= oB)
                                ? __ldcg(p.partials + ((int64_t)(q0 + q + r) * BP + b) * B1 + row)
                                : 0.f;
              }
#pragma unroll
              for (int u = 0; u < OPL; ++u)
#pragma unroll
                for (int q = 0; q < QMAX; ++q) y[u] += v[u][q];
            }
#pragma unroll
            for (int u = 0; u < OPL; ++u) {
              const int o = o0 + u * 32 + lane;
              const int row = o % B1, b = o / B1;
              if (o < B1 * BP && b < p.batch) store_out(p, row0 + row, b, y[u]);
            }
          }
          if (lane == 0) p.counters[r] = 0;  // ready for the next call
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&piece_empty[slot]);
    }
    return;
  }

  // -------------------------------- consumers --------------------------------
  const int cp = lane % C::CPR;
  const int rs = lane / C::CPR;
  const int wrow = warp * C::RW;
  float acc[C::JS][BP];
#pragma unroll
  for (int j = 0; j < C::JS; ++j)
#pragma unroll
    for (int b = 0; b < BP; ++b) acc[j][b] = 0.f;
  int piece = 0;

  int stage = 0;
  uint32_t phase = 0;
  for (;;) {
    if (!mbar_wait(&full_bar[stage], phase)) {
      if (lane == 0) atomicOr(p.status, kStatusTimeout);
      break;
    }
    const StageDesc d = desc[stage];
    if (d.flags & 2) break;
    const uint8_t *st = smem + (size_t)stage * C::kStageBytes;
    int voff = 0, moff = 0;
    for (int i = 0; i < d.ntiles; ++i) {
      const bool sp = (d.sparse >> i) & 1;
      // a lane covers columns [16cp, 16cp+16) of a 2:4 tile row, and columns
      // [8cp, 8cp+8) + [B2/2 + 8cp, B2/2 + 8cp + 8) of a dense tile row (so
      // that 8 lanes read 128 contiguous bytes of shared memory)
      const uint8_t *xs = st + C::kValsBytes + C::kMetaBytes + (i / C::XT) * C::kXCopy +
                          (i % C::XT) * 2 * B2;
      const int xo0 = sp ? 32 * cp : 16 * cp;
      const int xo1 = sp ? 32 * cp + 16 : B2 + 16 * cp;
#pragma unroll
      for (int b0 = 0; b0 < BP; b0 += C::XB) {
        uint32_t xr[C::XB][8];
#pragma unroll
        for (int b = 0; b < C::XB; ++b) {
          const uint4 lo = *reinterpret_cast<const uint4 *>(xs + (b0 + b) * C::kXBatch + xo0);
          const uint4 hi = *reinterpret_cast<const uint4 *>(xs + (b0 + b) * C::kXBatch + xo1);
          xr[b][0] = lo.x; xr[b][1] = lo.y; xr[b][2] = lo.z; xr[b][3] = lo.w;
          xr[b][4] = hi.x; xr[b][5] = hi.y; xr[b][6] = hi.z; xr[b][7] = hi.w;
        }
        if (sp) {
#pragma unroll
          for (int j = 0; j < C::JS; ++j) {
            const int row = wrow + j * C::RPS + rs;
            const uint4 v = *reinterpret_cast<const uint4 *>(st + voff + row * B2 + 16 * cp);
            const uint32_t m = *reinterpret_cast<const uint16_t *>(
                st + C::kValsBytes + moff + row * (B2 / 8) + 2 * cp);
            const uint32_t w[4] = {v.x, v.y, v.z, v.w};
            // PRMT selector of each group: (p0, p1) -- the lowest and highest
            // kept column -- becomes bytes {2p0, 2p0+1, 2p1, 2p1+1} of the
            // group's x quad.  Narrow batches, where a selector serves one or
            // two products, build it in registers: one PRMT looks up (p0, p1)
            // of two groups at once from a byte table indexed by the low three
            // bits of each 4-bit mask (distinct for the six masks with two bits
            // set), a second expands them to byte pairs.  Wide batches reuse a
            // selector across four columns and take it from the shared table.
            uint32_t selw[4];
            if constexpr (BP <= 4) {
              constexpr uint32_t kPairLo = 0x10313010u, kPairHi = 0x10212032u;
              const uint32_t s01 = __byte_perm(kPairLo, kPairHi, m & 0x77u);
              const uint32_t s23 = __byte_perm(kPairLo, kPairHi, (m >> 8) & 0x77u);
              const uint32_t a01 = __byte_perm(0x76543210u, 0u, s01);
              const uint32_t a23 = __byte_perm(0x76543210u, 0u, s23);
              selw[0] = a01;
              selw[1] = a01 >> 16;
              selw[2] = a23;
              selw[3] = a23 >> 16;
            } else {
#pragma unroll
              for (int g = 0; g < 4; ++g) selw[g] = sel_lut[(m >> (4 * g)) & 0xFu];
            }
#pragma unroll
            for (int g = 0; g < 4; ++g) {
              const uint32_t sel = selw[g];
#pragma unroll
              for (int b = 0; b < C::XB; ++b) {
                const uint32_t xp = __byte_perm(xr[b][2 * g], xr[b][2 * g + 1], sel);
                fma_bf16x2(acc[j][b0 + b], w[g], xp);
              }
            }
          }
        } else {
#pragma unroll
          for (int j = 0; j < C::JS; ++j) {
            const int row = wrow + j * C::RPS + rs;
            const uint4 a = *reinterpret_cast<const uint4 *>(st + voff + row * 2 * B2 + 16 * cp);
            const uint4 c2 =
                *reinterpret_cast<const uint4 *>(st + voff + row * 2 * B2 + B2 + 16 * cp);
            const uint32_t w[8] = {a.x, a.y, a.z, a.w, c2.x, c2.y, c2.z, c2.w};
#pragma unroll
            for (int e = 0; e < 8; ++e)
#pragma unroll
              for (int b = 0; b < C::XB; ++b) fma_bf16x2(acc[j][b0 + b], w[e], xr[b][e]);
          }
        }
      }
      voff += sp ? B1 * B2 : 2 * B1 * B2;
      moff += sp ? B1 * B2 / 8 : 0;
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty_bar[stage]);
    if (++stage == S) {
      stage = 0;
      phase ^= 1u;
    }
    if (!(d.flags & 1)) continue;

    // ---- end of this CTA's piece of a band: row sums to the epilogue warp ----
    const int slot = piece & 1;
    const uint32_t ph = (uint32_t)(piece >> 1) & 1u;
    if (!mbar_wait(&piece_empty[slot], ph ^ 1u)) {
      if (lane == 0) atomicOr(p.status, kStatusTimeout);
      break;
    }
    float *rows_s = s_rows[slot][warp];
#pragma unroll
    for (int j = 0; j < C::JS; ++j)
#pragma unroll
      for (int b = 0; b < BP; ++b) {
        float v = acc[j][b];
#pragma unroll
        for (int o = 1; o < C::CPR; o <<= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
        if (cp == 0) rows_s[b * C::RW + j * C::RPS + rs] = v;
        acc[j][b] = 0.f;
      }
    __syncwarp();
    if (lane == 0) mbar_arrive(&piece_full[slot]);
    ++piece;
  }
}

// ---------------------------------------------------------------------------
// work-split plan: one thread per CTA boundary c in [0, G], by the same rules
// the streaming kernels apply when they search for their own range
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(128)
    plan_kernel(const int64_t *__restrict__ val_off, const int64_t *__restrict__ meta_off,
                const uint8_t *__restrict__ map, int64_t T, int G, int64_t total, int tpr,
                int tpd, int64_t *__restrict__ plan) {
  const int c = blockIdx.x * blockDim.x + threadIdx.x;
  if (c > G) return;
  auto P = [&](int64_t t) -> int64_t { return 2 * val_off[t] + meta_off[t]; };
  if (c == 0) {
    plan[0] = G;
    plan[1] = kPlanTiles;
    for (int i = 2; i < kPlanHead; ++i) plan[i] = 0;
  }
  auto first_tile = [&](int64_t tg) -> int64_t {  // first t with P(t) G >= tg
    int64_t lo = 0, hi = T;
    while (lo < hi) {
      const int64_t mid = (lo + hi) / 2;
      if (P(mid) * G < tg) lo = mid + 1;
      else hi = mid;
    }
    return lo;
  };
  const int64_t tgt = (int64_t)c * total;
  const int64_t t0 = c == G ? T : first_tile(tgt);
  const int64_t t1 = c >= G - 1 ? T : first_tile(tgt + total);
  uint32_t bits = 0;
  const int nw = (int)min((int64_t)31, t1 - t0);
  for (int i = 0; i < nw; ++i) bits |= (uint32_t)(map[t0 + i] == 1) << i;
  const uint32_t starts = nw > 0 ? stage_starts(bits, nw, t0, tpr, tpd, 2 * tpd) : 0u;
  int64_t *rec = plan + kPlanHead + 4 * (int64_t)c;
  rec[0] = t0;
  rec[1] = val_off[t0];
  rec[2] = meta_off[t0];
  rec[3] = (int64_t)(((uint64_t)starts << 32) | bits);
}

// ---------------------------------------------------------------------------
// simple kernel for other legal tilings: one warp per output row
// ---------------------------------------------------------------------------
template <int BP, bool STRIDED>
__global__ void __launch_bounds__(kThreads)
    hybrid_rowwarp_kernel(const Params p, int b1, int b2) {
  const int lane = threadIdx.x & 31;
  const int64_t warps = (int64_t)gridDim.x * kWarps;
  const int cpr = b2 / 16;  // 16-column chunks per tile row
  for (int64_t row = (int64_t)blockIdx.x * kWarps + (threadIdx.x >> 5); row < p.n;
       row += warps) {
    const int64_t r = row / b1, i = row - r * b1;
    float acc[BP];
#pragma unroll
    for (int b = 0; b < BP; ++b) acc[b] = 0.f;
    for (int64_t q = lane; q < p.tpr * cpr; q += 32) {
      const int64_t tc = q / cpr;
      const int cpart = (int)(q - tc * cpr);
      const int64_t t = r * p.tpr + tc;
      float xf[BP][16];
#pragma unroll
      for (int b = 0; b < BP; ++b) {
        if (b < p.batch) {
          const uint16_t *xp = p.X + (int64_t)b * p.ldx + tc * b2 + 16 * cpart;
          unpack16(ld_keep16(xp), ld_keep16(xp + 8), xf[b]);
        } else {
#pragma unroll
          for (int e = 0; e < 16; ++e) xf[b][e] = 0.f;
        }
      }
      const bool sparse = !STRIDED && __ldg(p.map + t) == 1;
      if (sparse) {
        const uint8_t *vp =
            p.vals + 2 * __ldg(p.val_off + t) + i * b2 + 16 * cpart;
        const uint8_t *mp = p.meta + __ldg(p.meta_off + t) + i * (b2 / 8) + 2 * cpart;
        const uint4 v = ld_stream16(vp);
        const uint32_t m = ld_stream_u16(mp);
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int g = 0; g < 4; ++g) {
          const uint32_t nib = (m >> (4 * g)) & 0xFu;
#pragma unroll
          for (int b = 0; b < BP; ++b) {
            float xa, xb;
            pick2(nib, xf[b][4 * g], xf[b][4 * g + 1], xf[b][4 * g + 2],
                  xf[b][4 * g + 3], xa, xb);
            acc[b] = fmaf(bf16_lo(w[g]), xa, acc[b]);
            acc[b] = fmaf(bf16_hi(w[g]), xb, acc[b]);
          }
        }
      } else {
        const uint8_t *vp =
            STRIDED ? reinterpret_cast<const uint8_t *>(p.Wd + row * p.ldw + tc * b2 + 16 * cpart)
                    : p.vals + 2 * __ldg(p.val_off + t) + i * 2 * b2 + 32 * cpart;
        float wf[16];
        unpack16(ld_stream16(vp), ld_stream16(vp + 16), wf);
#pragma unroll
        for (int e = 0; e < 16; ++e)
#pragma unroll
          for (int b = 0; b < BP; ++b) acc[b] = fmaf(wf[e], xf[b][e], acc[b]);
      }
    }
#pragma unroll
    for (int b = 0; b < BP; ++b)
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) acc[b] += __shfl_xor_sync(0xffffffffu, acc[b], o);
    if (lane == 0)
      for (int b = 0; b < p.batch; ++b) store_out(p, row, b, acc[b]);
  }
}

// ---------------------------------------------------------------------------
// low rank: t[b][j] = sum_k V[k][j] x[b][k]  (3BASiL §1: the L = U V^T term)
// ---------------------------------------------------------------------------
// CTA c sums k in its slice; partials go to lr_part[c][b][j]; the last CTA to
// arrive sums them into t in a fixed order (deterministic).  With pdl (it is a
// programmatic dependent itself) it waits for its predecessor before touching
// anything, and only then lets its own dependents launch.
template <int BP>
__global__ void __launch_bounds__(kThreads)
    lowrank_t_kernel(const uint16_t *__restrict__ V, int64_t ldv, int rank,
                     int64_t k, const uint16_t *__restrict__ X, int64_t ldx,
                     int batch, float *__restrict__ t_out,
                     float *__restrict__ lr_part, uint32_t *counter, int pdl) {
  __shared__ float s_sum[BP * kMaxRank];
  __shared__ float4 s_red[kThreads];
  __shared__ int s_last;
  if (pdl) grid_dep_wait();
  // Dependents (the U pass, then the product) may launch from here on: all
  // work queued before this kernel has finished, so they may read X at once.
  grid_dep_trigger();
  const int tid = threadIdx.x;
  const int jg_count = rank / 8;          // 8 columns of V per thread
  const int rows_par = kThreads / jg_count;  // k rows in parallel
  const int jg = tid % jg_count, rg = tid / jg_count;
  const int G2 = gridDim.x, c = blockIdx.x;
  const int64_t k0 = k * c / G2, k1 = k * (c + 1) / G2;
  float acc[BP][8];
#pragma unroll
  for (int b = 0; b < BP; ++b)
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[b][e] = 0.f;
  if (rg < rows_par) {
    for (int64_t kk = k0 + rg; kk < k1; kk += rows_par) {
      const uint4 v = ld_stream16(V + kk * ldv + 8 * jg);
      const float vf[8] = {bf16_lo(v.x), bf16_hi(v.x), bf16_lo(v.y), bf16_hi(v.y),
                           bf16_lo(v.z), bf16_hi(v.z), bf16_lo(v.w), bf16_hi(v.w)};
#pragma unroll
      for (int b = 0; b < BP; ++b) {
        if (b >= batch) break;
        const float xv = __uint_as_float((uint32_t)__ldg(X + b * ldx + kk) << 16);
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[b][e] = fmaf(vf[e], xv, acc[b][e]);
      }
    }
  }
  // fixed-order reduction over the row groups of this CTA
  for (int i = tid; i < BP * rank; i += kThreads) s_sum[i] = 0.f;
  __syncthreads();
  for (int g = 0; g < rows_par; ++g) {
    if (rg == g) {
#pragma unroll
      for (int b = 0; b < BP; ++b)
#pragma unroll
        for (int e = 0; e < 8; ++e) s_sum[b * rank + 8 * jg + e] += acc[b][e];
    }
    __syncthreads();
  }
  float *mine = lr_part + (int64_t)c * BP * rank;
  for (int i = tid; i < BP * rank; i += kThreads) __stcg(mine + i, s_sum[i]);
  __threadfence();
  __syncthreads();
  if (tid == 0) s_last = atomicAdd(counter, 1u) == (uint32_t)(G2 - 1);
  __syncthreads();
  if (s_last) {
    __threadfence();
    // Every thread takes part: a column of four outputs is split over `per`
    // threads, thread `sub` adding the partials of CTAs sub, sub + per, ...
    // in ascending order with four loads in flight, and the `per` sums are
    // then added in sub order.  (BP * rank is a multiple of 8.)
    const int O4 = BP * rank / 4;
    const int per = O4 >= kThreads ? 1 : kThreads / O4;
    const float4 *part4 = reinterpret_cast<const float4 *>(lr_part);
    float4 *t4 = reinterpret_cast<float4 *>(t_out);
    auto add4 = [](float4 &a, const float4 &v) {
      a.x += v.x;
      a.y += v.y;
      a.z += v.z;
      a.w += v.w;
    };
    for (int item = tid; item < O4 * per; item += kThreads) {
      const int col = item % O4, sub = item / O4;
      float4 a = make_float4(0.f, 0.f, 0.f, 0.f);
      int cc = sub;
      for (; cc + 3 * per < G2; cc += 4 * per) {
        const float4 v0 = __ldcg(part4 + (int64_t)cc * O4 + col);
        const float4 v1 = __ldcg(part4 + (int64_t)(cc + per) * O4 + col);
        const float4 v2 = __ldcg(part4 + (int64_t)(cc + 2 * per) * O4 + col);
        const float4 v3 = __ldcg(part4 + (int64_t)(cc + 3 * per) * O4 + col);
        add4(a, v0);
        add4(a, v1);
        add4(a, v2);
        add4(a, v3);
      }
      for (; cc < G2; cc += per) add4(a, __ldcg(part4 + (int64_t)cc * O4 + col));
      if (per == 1)
        t4[col] = a;
      else
        s_red[sub * O4 + col] = a;
    }
    if (per > 1) {
      __syncthreads();
      for (int col = tid; col < O4; col += kThreads) {
        float4 a = s_red[col];
        for (int sub = 1; sub < per; ++sub) add4(a, s_red[sub * O4 + col]);
        t4[col] = a;
      }
    }
    if (tid == 0) *counter = 0;
  }
}

// Y[b][i] += sum_j U[i][j] t[b][j]  (fp32 Y), one thread per row.
template <int BP>
__global__ void __launch_bounds__(kThreads)
    lowrank_apply_kernel(int64_t n, const uint16_t *__restrict__ U, int64_t ldu,
                         int rank, const float *__restrict__ t, int batch,
                         float *__restrict__ Y, int64_t ldy, int pdl) {
  grid_dep_trigger();
  const int64_t i = (int64_t)blockIdx.x * kThreads + threadIdx.x;
  // the first 16 bytes of this row of U are requested before t and Y, which
  // the preceding grid writes, may be read
  const uint4 u0 = i < n ? __ldg(reinterpret_cast<const uint4 *>(U + i * ldu)) : make_uint4(0, 0, 0, 0);
  if (pdl) grid_dep_wait();
  if (i >= n) return;
  float acc[BP];
#pragma unroll
  for (int b = 0; b < BP; ++b) acc[b] = 0.f;
  for (int j = 0; j < rank; j += 8) {
    const uint4 uv = j == 0 ? u0 : __ldg(reinterpret_cast<const uint4 *>(U + i * ldu + j));
    const float uf[8] = {bf16_lo(uv.x), bf16_hi(uv.x), bf16_lo(uv.y), bf16_hi(uv.y),
                         bf16_lo(uv.z), bf16_hi(uv.z), bf16_lo(uv.w), bf16_hi(uv.w)};
#pragma unroll
    for (int b = 0; b < BP; ++b)
#pragma unroll
      for (int e = 0; e < 8; ++e) acc[b] = fmaf(uf[e], t[b * rank + j + e], acc[b]);
  }
  for (int b = 0; b < batch; ++b) Y[b * ldy + i] += acc[b];
}

// ut[b][i] = sum_j U[i][j] t[b][j] (fp32), one thread per row; U is read once.
template <int BP>
__global__ void __launch_bounds__(kThreads)
    lowrank_ut_kernel(int64_t n, const uint16_t *__restrict__ U, int64_t ldu, int rank,
                      const float *__restrict__ t, int batch, float *__restrict__ ut, int pdl) {
  grid_dep_trigger();  // the product that follows may start streaming its weights
  const int64_t i = (int64_t)blockIdx.x * kThreads + threadIdx.x;
  const bool live = i < n;
  auto load_chunk = [&](int j0, uint4 (&uv)[8]) {
#pragma unroll
    for (int q = 0; q < 8; ++q)
      uv[q] = live && j0 + 8 * q < rank
                  ? __ldg(reinterpret_cast<const uint4 *>(U + i * ldu + j0 + 8 * q))
                  : make_uint4(0, 0, 0, 0);
  };
  // the first 128 bytes of this row of U are requested before t, which the
  // preceding grid writes, may be read
  uint4 first[8];
  load_chunk(0, first);
  if (pdl) grid_dep_wait();
  if (!live) return;
  float acc[BP];
#pragma unroll
  for (int b = 0; b < BP; ++b) acc[b] = 0.f;
  for (int j0 = 0; j0 < rank; j0 += 64) {
    uint4 uv[8];
    if (j0 == 0) {
#pragma unroll
      for (int q = 0; q < 8; ++q) uv[q] = first[q];
    } else {
      load_chunk(j0, uv);
    }
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      if (j0 + 8 * q >= rank) break;
      const float uf[8] = {bf16_lo(uv[q].x), bf16_hi(uv[q].x), bf16_lo(uv[q].y), bf16_hi(uv[q].y),
                           bf16_lo(uv[q].z), bf16_hi(uv[q].z), bf16_lo(uv[q].w), bf16_hi(uv[q].w)};
#pragma unroll
      for (int b = 0; b < BP; ++b)
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[b] = fmaf(uf[e], t[b * rank + j0 + 8 * q + e], acc[b]);
    }
  }
  for (int b = 0; b < batch; ++b) ut[(int64_t)b * n + i] = acc[b];
}

// ---------------------------------------------------------------------------
// failure-path self test: a wait that nothing completes runs out
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(32) selftest_wait_timeout_kernel(uint32_t *status,
                                                                   uint32_t limit) {
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncwarp();
  // nothing ever arrives on bar, so phase 0 never completes
  const bool done = mbar_wait_limit(&bar, 0u, limit);
  if (!done && threadIdx.x == 0) atomicOr(status, kStatusTimeout);
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------

int pad_batch(int batch) {
  if (batch <= 1) return 1;
  if (batch <= 2) return 2;
  if (batch <= 4) return 4;
  if (batch <= 8) return 8;
  return 16;
}

enum Shape { kS128x128, kS128x64, kS64x64, kS64x128, kGeneric };

Shape shape_of(int b1, int b2) {
  if (b1 == 128 && b2 == 128) return kS128x128;
  if (b1 == 128 && b2 == 64) return kS128x64;
  if (b1 == 64 && b2 == 64) return kS64x64;
  if (b1 == 64 && b2 == 128) return kS64x128;
  return kGeneric;
}

template <int BP, int B1, int B2>
void *dense_kernel_ptr() {
  return reinterpret_cast<void *>(&dense_gemv_kernel<BP, B1, B2>);
}

void *pick_dense_kernel(int bp, Shape s) {
#define HYB_CASE(BP_)                                                  \
  case BP_:                                                            \
    switch (s) {                                                       \
      case kS128x128: return dense_kernel_ptr<BP_, 128, 128>(); \
      case kS128x64: return dense_kernel_ptr<BP_, 128, 64>();   \
      case kS64x64: return dense_kernel_ptr<BP_, 64, 64>();     \
      case kS64x128: return dense_kernel_ptr<BP_, 64, 128>();   \
      default: return nullptr;                                         \
    }
  switch (bp) {
    HYB_CASE(1)
    HYB_CASE(2)
    HYB_CASE(4)
    HYB_CASE(8)
    HYB_CASE(16)
    default: return nullptr;
  }
#undef HYB_CASE
}

struct TmaKernel {
  void *fn;
  int threads;
  size_t smem;
  int tps;
  bool xtm;    // X slices by 2-D tensor copies (box xcols x bp)
  int xcols;
  int bp;
};

template <int BP, int B1, int B2>
TmaKernel tma_kernel_info() {
  using C = TmaCfg<BP, B1, B2>;
  return TmaKernel{reinterpret_cast<void *>(&hybrid_tma_kernel<BP, B1, B2>), C::kThreads,
                   C::kSmem, C::TPX, C::XTM, C::XT * B2, BP};
}

bool pick_tma_kernel(int bp, Shape s, TmaKernel *out) {
#define HYB_TCASE(BP_)                                                         \
  case BP_:                                                                    \
    switch (s) {                                                               \
      case kS128x128: *out = tma_kernel_info<BP_, 128, 128>(); return true;    \
      case kS128x64: *out = tma_kernel_info<BP_, 128, 64>(); return true;      \
      case kS64x64: *out = tma_kernel_info<BP_, 64, 64>(); return true;        \
      case kS64x128: *out = tma_kernel_info<BP_, 64, 128>(); return true;      \
      default: return false;                                                   \
    }
  switch (bp) {
    HYB_TCASE(1)
    HYB_TCASE(2)
    HYB_TCASE(4)
    HYB_TCASE(8)
    HYB_TCASE(16)
    default: return false;
  }
#undef HYB_TCASE
}

template <bool STRIDED>
void *pick_rowwarp_kernel(int bp) {
  switch (bp) {
    case 1: return reinterpret_cast<void *>(&hybrid_rowwarp_kernel<1, STRIDED>);
    case 2: return reinterpret_cast<void *>(&hybrid_rowwarp_kernel<2, STRIDED>);
    case 4: return reinterpret_cast<void *>(&hybrid_rowwarp_kernel<4, STRIDED>);
    case 8: return reinterpret_cast<void *>(&hybrid_rowwarp_kernel<8, STRIDED>);
    default: return reinterpret_cast<void *>(&hybrid_rowwarp_kernel<16, STRIDED>);
  }
}

void *pick_lowrank_t(int bp) {
  switch (bp) {
    case 1: return reinterpret_cast<void *>(&lowrank_t_kernel<1>);
    case 2: return reinterpret_cast<void *>(&lowrank_t_kernel<2>);
    case 4: return reinterpret_cast<void *>(&lowrank_t_kernel<4>);
    case 8: return reinterpret_cast<void *>(&lowrank_t_kernel<8>);
    default: return reinterpret_cast<void *>(&lowrank_t_kernel<16>);
  }
}

void *pick_lowrank_ut(int bp) {
  switch (bp) {
    case 1: return reinterpret_cast<void *>(&lowrank_ut_kernel<1>);
    case 2: return reinterpret_cast<void *>(&lowrank_ut_kernel<2>);
    case 4: return reinterpret_cast<void *>(&lowrank_ut_kernel<4>);
    case 8: return reinterpret_cast<void *>(&lowrank_ut_kernel<8>);
    default: return reinterpret_cast<void *>(&lowrank_ut_kernel<16>);
  }
}

void *pick_lowrank_apply(int bp) {
  switch (bp) {
    case 1: return reinterpret_cast<void *>(&lowrank_apply_kernel<1>);
    case 2: return reinterpret_cast<void *>(&lowrank_apply_kernel<2>);
    case 4: return reinterpret_cast<void *>(&lowrank_apply_kernel<4>);
    case 8: return reinterpret_cast<void *>(&lowrank_apply_kernel<8>);
    default: return reinterpret_cast<void *>(&lowrank_apply_kernel<16>);
  }
}

// Resident CTAs per SM of a kernel instance (cached; the answer only depends
// on the instance and the device).
int blocks_per_sm(void *fn, size_t dyn_smem, int threads = kThreads) {
  static std::mutex mu;
  struct Entry {
    void *fn;
    int dev;
    size_t smem;
    int blocks;
  };
  static Entry cache[256];
  static int used = 0;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return -1;
  // dynamic shared memory is small; bucket it so the cache stays tiny
  const size_t bucket = align_up(dyn_smem, 4096);
  std::lock_guard<std::mutex> lock(mu);
  for (int i = 0; i < used; ++i)
    if (cache[i].fn == fn && cache[i].dev == dev && cache[i].smem == bucket)
      return cache[i].blocks;
  int nb = 0;
  if (bucket > 48 * 1024 &&
      cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bucket) !=
          cudaSuccess)
    return -1;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&nb, fn, threads, bucket) != cudaSuccess)
    return -1;
  if (used < 256) cache[used++] = Entry{fn, dev, bucket, nb};
  return nb;
}

// Work split and workspace layout of one product call.
struct Plan {
  bool tma;        // TMA-ring kernel (packed hybrid, tuned tile shapes)
  TmaKernel tk;
  bool stream;     // tuned kernel (else one warp per row)
  int bp;          // padded batch
  int b1, b2;
  int G;           // CTAs of the stream split
  int R;           // bands
  int64_t total;   // packed bytes
  int lr_ctas;     // CTAs of the low-rank reduction
  size_t off_counters, off_lr_t, off_lr_part, off_lr_counter, off_lr_ut, off_partials,
      bytes;
  size_t dyn_smem;
};

// CTAs of the TMA-ring kernels: one per SM (the ring takes most of shared
// memory), at most kMaxCtas (the size of the launch-parameter plan), and no
// more than there are dense tiles' worth of bytes.
int tma_ctas(int sms, int64_t total_bytes, int b1, int b2) {
  const int64_t gcap = std::max<int64_t>(1, total_bytes / (2LL * b1 * b2));
  return (int)std::min<int64_t>(std::min(sms, kMaxCtas), gcap);
}

int make_plan(int64_t n, int64_t k, int b1, int b2, int64_t total_bytes,
              int batch, int rank, bool strided, Plan *pl) {
  Plan P{};
  P.bp = pad_batch(batch);
  P.b1 = b1;
  P.b2 = b2;
  P.R = (int)(n / b1);
  P.total = total_bytes;
  const Shape s = shape_of(b1, b2);
  int sms = 0;
  int rc = device_sm_count(&sms);
  if (rc != HYB_OK) return rc;
  P.tma = !strided && s != kGeneric;
  if (P.tma) {
    P.G = tma_ctas(sms, total_bytes, b1, b2);
    if (!pick_tma_kernel(P.bp, s, &P.tk)) return HYB_ERR_UNSUPPORTED;
  }
  P.stream = strided && s != kGeneric && P.R <= 8192;
  P.dyn_smem = P.tma ? P.tk.smem : (P.stream ? (size_t)2 * P.R * sizeof(int) : 0);
  if (P.tma) {
    const int nb = blocks_per_sm(P.tk.fn, P.tk.smem, P.tk.threads);
    if (nb <= 0) return HYB_ERR_CUDA;
  } else if (P.stream) {
    void *fn = pick_dense_kernel(P.bp, s);
    if (P.dyn_smem > 48 * 1024) {
      if (cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               (int)P.dyn_smem) != cudaSuccess)
        return HYB_ERR_CUDA;
    }
    const int nb = blocks_per_sm(fn, P.dyn_smem);
    if (nb <= 0) return HYB_ERR_CUDA;
    const int64_t max_cost = 2LL * b1 * b2;  // a dense tile
    int64_t G = (int64_t)nb * sms;
    // every CTA must own at least one tile: total / G >= largest tile
    const int64_t gcap = std::max<int64_t>(1, total_bytes / max_cost);
    P.G = (int)std::min(G, gcap);
  } else {
    P.G = 0;
  }
  P.lr_ctas = rank > 0 ? (int)std::max<int64_t>(1, std::min<int64_t>(sms, k / 64)) : 0;
  size_t off = kHeaderBytes;
  P.off_counters = off;
  if (P.tma) off = align_up(off + (size_t)P.R * (b1 / 8) * sizeof(uint32_t), 256);
  else if (P.stream) off = align_up(off + (size_t)P.R * sizeof(uint32_t), 256);
  P.off_lr_t = off;
  off = align_up(off + (size_t)P.bp * (rank > 0 ? rank : 0) * sizeof(float), 256);
  P.off_lr_part = off;
  off = align_up(off + (size_t)P.lr_ctas * P.bp * (rank > 0 ? rank : 0) * sizeof(float), 256);
  P.off_lr_counter = off;
  off = align_up(off + sizeof(uint32_t), 256);
  P.off_lr_ut = off;
  off = align_up(off + (size_t)P.bp * (rank > 0 ? n : 0) * sizeof(float), 256);
  P.off_partials = off;
  if (P.tma || P.stream) off += (size_t)(P.G + P.R) * b1 * P.bp * sizeof(float);
  P.bytes = align_up(off, 256);
  *pl = P;
  return HYB_OK;
}

int check_lowrank(const hyb_lowrank *lr, int64_t n, int64_t k) {
  if (!lr) return HYB_OK;
  if (lr->rank < 0 || lr->rank > kMaxRank) return HYB_ERR_INVALID_ARG;
  if (lr->rank == 0) return HYB_OK;
  if (lr->rank % 8 != 0) return HYB_ERR_UNSUPPORTED;
  if (!lr->U || !lr->V || lr->ldu < lr->rank || lr->ldv < lr->rank)
    return HYB_ERR_INVALID_ARG;
  if (((uintptr_t)lr->U | (uintptr_t)lr->V) % 16 != 0 || lr->ldu % 8 != 0 ||
      lr->ldv % 8 != 0)
    return HYB_ERR_ALIGNMENT;
  (void)n;
  (void)k;
  return HYB_OK;
}

// A launch, as a programmatic dependent of the preceding kernel on the stream
// when pdl is set (the kernel then orders its own accesses with
// griddepcontrol.wait).
cudaError_t launch_kernel(const void *fn, dim3 grid, dim3 block, void **args, size_t smem,
                          cudaStream_t s, bool pdl) {
  if (!pdl) return cudaLaunchKernel(fn, grid, block, args, smem, s);
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelExC(&cfg, fn, args);
}

int launch_lowrank_t(const Plan &P, const hyb_lowrank *lr, int64_t k,
                     const uint16_t *X, int64_t ldx, int batch, uint8_t *ws,
                     cudaStream_t s, bool pdl) {
  void *fn = pick_lowrank_t(P.bp);
  const uint16_t *V = lr->V;
  int64_t ldv = lr->ldv;
  int rank = lr->rank;
  float *t_out = reinterpret_cast<float *>(ws + P.off_lr_t);
  float *part = reinterpret_cast<float *>(ws + P.off_lr_part);
  uint32_t *counter = reinterpret_cast<uint32_t *>(ws + P.off_lr_counter);
  int pdl_i = pdl ? 1 : 0;
  void *args[] = {&V, &ldv, &rank, &k, &X, &ldx, &batch, &t_out, &part, &counter, &pdl_i};
  if (launch_kernel(fn, dim3(P.lr_ctas), dim3(kThreads), args, 0, s, pdl) != cudaSuccess)
    return HYB_ERR_CUDA;
  return HYB_OK;
}

// Shared driver of hyb_spmv / hyb_spmm_skinny / hyb_gemv_dense.
// Tensor map of X ([batch][k] bf16, row stride ldx) with box [bp][xcols]:
// rows past the batch and columns past k read as zeros.  The encoder is the
// driver's, found once through the runtime.
int encode_x_map(const uint16_t *X, int64_t k, int batch, int64_t ldx, int xcols, int bp,
                 CUtensorMap *map) {
  static PFN_cuTensorMapEncodeTiled_v12000 encode = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void *fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  });
  if (!encode) return HYB_ERR_CUDA;
  const cuuint64_t dims[2] = {(cuuint64_t)k, (cuuint64_t)batch};
  const cuuint64_t strides[1] = {(cuuint64_t)ldx * 2};
  const cuuint32_t box[2] = {(cuuint32_t)xcols, (cuuint32_t)bp};
  const cuuint32_t estr[2] = {1, 1};
  const CUresult r = encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
                            const_cast<uint16_t *>(X), dims, strides, box, estr,
                            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                            CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? HYB_OK : HYB_ERR_CUDA;
}

// Copies a host plan made for this split into the launch parameters, after
// checking that its ranges are well formed (a plan for another split, kind or
// size is ignored and the kernel searches for its own range).
void fill_launch_plan(const int64_t *plan, int32_t plan_ctas, const Plan &P, const Params &prm,
                      LaunchPlan *lp) {
  lp->kind = 0;
  lp->ctas = 0;
  const int32_t kind = kPlanTiles;
  if (!plan || !P.tma || plan_ctas != P.G || plan[0] != P.G || plan[1] != kind) return;
  const int64_t *rec = plan + kPlanHead;
  const int64_t end = prm.T;
  if (rec[0] != 0 || rec[4 * P.G] != end) return;
  for (int c = 0; c <= P.G; ++c) {
    const int64_t *r = rec + 4 * c;
    if (r[0] < 0 || r[0] > end || (c > 0 && r[0] < r[-4])) return;
    if (r[1] < 0 || 2 * r[1] > prm.nvb || r[2] < 0 || r[2] > prm.nmb) return;
  }
  std::copy(rec, rec + 4 * (P.G + 1), lp->rec);
  lp->kind = kind;
  lp->ctas = P.G;
}

int run_product(Params prm, int b1, int b2, int batch, const hyb_lowrank *lr,
                bool strided, void *ws, size_t ws_bytes, cudaStream_t s,
                const int64_t *plan = nullptr, int32_t plan_ctas = 0, uint32_t flags = 0) {
  const int rank = (lr && lr->rank > 0) ? lr->rank : 0;
  Plan P;
  int rc = make_plan(prm.n, prm.k, b1, b2, prm.total, batch, rank, strided, &P);
  if (rc != HYB_OK) return rc;
  if (!ws || ws_bytes < P.bytes) return HYB_ERR_WORKSPACE;
  if ((uintptr_t)ws % 256 != 0) return HYB_ERR_ALIGNMENT;
  uint8_t *w = reinterpret_cast<uint8_t *>(ws);
  prm.R = P.R;
  prm.G = P.G;
  prm.partials = reinterpret_cast<float *>(w + P.off_partials);
  prm.counters = reinterpret_cast<uint32_t *>(w + P.off_counters);
  prm.rank = rank;
  prm.U = rank ? lr->U : nullptr;
  prm.ldu = rank ? lr->ldu : 0;
  prm.lr_t = reinterpret_cast<const float *>(w + P.off_lr_t);
  prm.lr_ut = nullptr;
  const bool overlap = (flags & HYB_LAUNCH_OVERLAP_PREV) != 0;
  if (rank) {
    // V^T x, then U t, then the product: the two later kernels always launch
    // as programmatic dependents of the one before.  V^T x lets them launch
    // only after everything queued before the call has finished (with the
    // caller's leave it starts early itself, and waits), so their early
    // loads -- of U, the weights and X -- see finished data; what they wait
    // for is t, U t and the workspace.
    rc = launch_lowrank_t(P, lr, prm.k, prm.X, prm.ldx, batch, w, s, overlap);
    if (rc != HYB_OK) return rc;
    int64_t nn = prm.n, ldu = lr->ldu;
    const uint16_t *U = lr->U;
    int rk = rank, bt = batch;
    const float *tp = prm.lr_t;
    float *ut = reinterpret_cast<float *>(w + P.off_lr_ut);
    int one = 1;
    void *uargs[] = {&nn, &U, &ldu, &rk, &tp, &bt, &ut, &one};
    const int64_t grid = (prm.n + kThreads - 1) / kThreads;
    if (launch_kernel(pick_lowrank_ut(P.bp), dim3((unsigned)grid), dim3(kThreads), uargs, 0, s,
                      true) != cudaSuccess)
      return HYB_ERR_CUDA;
    prm.lr_ut = ut;
  }
  prm.status = reinterpret_cast<uint32_t *>(w);
  const bool pdl = (overlap || rank > 0) && (P.tma || P.stream);
  prm.pdl = !pdl ? 0 : (rank > 0 ? 2 : 1);
  void *args[] = {&prm};
  if (P.tma) {
    LaunchPlan lp;
    fill_launch_plan(plan, plan_ctas, P, prm, &lp);
    alignas(64) CUtensorMap xmap{};
    if (P.tk.xtm) {
      rc = encode_x_map(prm.X, prm.k, batch, prm.ldx, P.tk.xcols, P.tk.bp, &xmap);
      if (rc != HYB_OK) return rc;
    }
    void *targs[] = {&prm, &lp, &xmap};
    if (launch_kernel(P.tk.fn, dim3(P.G), dim3(P.tk.threads), targs, P.tk.smem, s, pdl) !=
        cudaSuccess)
      return HYB_ERR_CUDA;
  } else if (P.stream) {
    void *fn = pick_dense_kernel(P.bp, shape_of(b1, b2));
    if (launch_kernel(fn, dim3(P.G), dim3(kThreads), args, P.dyn_smem, s, pdl) != cudaSuccess)
      return HYB_ERR_CUDA;
  } else {
    void *fn = strided ? pick_rowwarp_kernel<true>(P.bp)
                       : pick_rowwarp_kernel<false>(P.bp);
    int sms = 0;
    rc = device_sm_count(&sms);
    if (rc != HYB_OK) return rc;
    const int64_t need = (prm.n + kWarps - 1) / kWarps;
    const int64_t grid = std::min<int64_t>(need, (int64_t)sms * 8);
    int b1v = b1, b2v = b2;
    void *args2[] = {&prm, &b1v, &b2v};
    if (cudaLaunchKernel(fn, dim3((unsigned)grid), dim3(kThreads), args2, 0, s) !=
        cudaSuccess)
      return HYB_ERR_CUDA;
  }
  return HYB_OK;
}

int check_io(const uint16_t *X, int64_t ldx, void *Y, int64_t ldy, int64_t n,
             int64_t k, int batch, int ydt) {
  if (!X || !Y) return HYB_ERR_INVALID_ARG;
  if (batch < 1 || batch > 16) return HYB_ERR_INVALID_ARG;
  if (ydt != HYB_F32 && ydt != HYB_BF16) return HYB_ERR_INVALID_ARG;
  if (ldx < k || ldy < n) return HYB_ERR_INVALID_ARG;
  // X is read in 16-byte pieces; Y is written one element at a time
  if ((uintptr_t)X % 16 != 0 || ldx % 8 != 0) return HYB_ERR_ALIGNMENT;
  if ((uintptr_t)Y % (ydt == HYB_F32 ? 4 : 2) != 0) return HYB_ERR_ALIGNMENT;
  return HYB_OK;
}

int spmm_impl(const hyb_matrix *A, int batch, const uint16_t *X, int64_t ldx,
              void *Y, int64_t ldy, hyb_dtype ydt, const hyb_lowrank *lr,
              void *ws, size_t ws_bytes, cudaStream_t s, uint32_t flags = 0) {
  if (!A) return HYB_ERR_INVALID_ARG;
  if (flags & ~HYB_LAUNCH_OVERLAP_PREV) return HYB_ERR_INVALID_ARG;
  int rc = check_tiling(A->n, A->k, A->b1, A->b2);
  if (rc != HYB_OK) return rc;
  if (A->num_tiles != (A->n / A->b1) * (A->k / A->b2)) return HYB_ERR_INVALID_ARG;
  if (!A->tile_map || !A->vals || !A->meta || !A->val_off || !A->meta_off)
    return HYB_ERR_INVALID_ARG;
  const int64_t te = (int64_t)A->b1 * A->b2;
  if (A->n_vals < A->num_tiles * te / 2 || A->n_vals > A->num_tiles * te ||
      A->n_meta_bytes < 0 || A->n_meta_bytes > A->num_tiles * te / 8)
    return HYB_ERR_INVALID_ARG;
  if (((uintptr_t)A->vals) % 32 != 0 || ((uintptr_t)A->meta) % 16 != 0)
    return HYB_ERR_ALIGNMENT;
  rc = check_io(X, ldx, Y, ldy, A->n, A->k, batch, ydt);
  if (rc != HYB_OK) return rc;
  rc = check_lowrank(lr, A->n, A->k);
  if (rc != HYB_OK) return rc;
  Params prm{};
  prm.map = A->tile_map;
  prm.vals = reinterpret_cast<const uint8_t *>(A->vals);
  prm.meta = A->meta;
  prm.val_off = A->val_off;
  prm.meta_off = A->meta_off;
  prm.n = A->n;
  prm.k = A->k;
  prm.tpr = A->k / A->b2;
  prm.T = A->num_tiles;
  prm.X = X;
  prm.ldx = ldx;
  prm.batch = batch;
  prm.Y = Y;
  prm.ldy = ldy;
  prm.ydt = ydt;
  prm.total = 2 * A->n_vals + A->n_meta_bytes;  // packed bytes
  prm.nvb = 2 * A->n_vals;
  prm.nmb = A->n_meta_bytes;
  return run_product(prm, A->b1, A->b2, batch, lr, false, ws, ws_bytes, s, A->plan,
                     A->plan_ctas, flags);
}

// Virtual tiling of a plain row-major W for the dense baseline.
void dense_tiling(int64_t n, int64_t k, int *b1, int *b2) {
  if (n % 128 == 0 && k % 128 == 0) {
    *b1 = 128;
    *b2 = 128;
  } else if (n % 64 == 0 && k % 64 == 0) {
    *b1 = 64;
    *b2 = 64;
  } else {
    *b1 = 1;
    *b2 = 16;
  }
}

size_t lowrank_ws_layout(int64_t k, int batch, int rank, size_t *off_t,
                         size_t *off_part, size_t *off_counter, int *ctas) {
  int sms = 0;
  if (device_sm_count(&sms) != HYB_OK) return 0;
  const int bp = pad_batch(batch);
  *ctas = (int)std::max<int64_t>(1, std::min<int64_t>(sms, k / 64));
  size_t off = kHeaderBytes;
  *off_t = off;
  off = align_up(off + (size_t)bp * rank * sizeof(float), 256);
  *off_part = off;
  off = align_up(off + (size_t)(*ctas) * bp * rank * sizeof(float), 256);
  *off_counter = off;
  off = align_up(off + sizeof(uint32_t), 256);
  return off;
}

}  // namespace
}  // namespace hyb

using namespace hyb;

extern "C" {

size_t hyb_plan_entries(void) { return (size_t)kPlanHead + 4 * (size_t)(kMaxCtas + 1); }

int hyb_make_plan(const hyb_matrix *A, int64_t *scratch, int64_t *plan_host,
                  int32_t *plan_ctas, hyb_stream_t stream) {
  if (!A || !scratch || !plan_host || !plan_ctas) return HYB_ERR_INVALID_ARG;
  *plan_ctas = 0;
  int rc = check_tiling(A->n, A->k, A->b1, A->b2);
  if (rc != HYB_OK) return rc;
  if (!A->val_off || !A->meta_off || !A->tile_map ||
      A->num_tiles != (A->n / A->b1) * (A->k / A->b2))
    return HYB_ERR_INVALID_ARG;
  if ((uintptr_t)scratch % 8 != 0 || (uintptr_t)plan_host % 8 != 0) return HYB_ERR_ALIGNMENT;
  int sms = 0;
  rc = device_sm_count(&sms);
  if (rc != HYB_OK) return rc;
  std::fill(plan_host, plan_host + hyb_plan_entries(), 0);
  const int64_t total = 2 * A->n_vals + A->n_meta_bytes;
  if (shape_of(A->b1, A->b2) == kGeneric || total <= 0) return HYB_OK;  // no TMA kernel: G = 0
  // the same split as the products: make_plan's CTA count
  const int G = tma_ctas(sms, total, A->b1, A->b2);
  cudaStream_t s = (cudaStream_t)stream;
  // stage limits of the streaming kernel (a 32 KB value buffer per stage)
  const int tpd = std::max(1, 16384 / (A->b1 * A->b2));
  plan_kernel<<<(G + 1 + 127) / 128, 128, 0, s>>>(A->val_off, A->meta_off, A->tile_map,
                                                  A->num_tiles, G, total,
                                                  (int)(A->k / A->b2), tpd, scratch);
  if (cudaGetLastError() != cudaSuccess) return HYB_ERR_CUDA;
  const size_t bytes = sizeof(int64_t) * (kPlanHead + 4 * (size_t)(G + 1));
  if (cudaMemcpyAsync(plan_host, scratch, bytes, cudaMemcpyDeviceToHost, s) != cudaSuccess ||
      cudaStreamSynchronize(s) != cudaSuccess)
    return HYB_ERR_CUDA;
  *plan_ctas = G;
  return HYB_OK;
}

size_t hyb_workspace_bytes(const hyb_matrix *A, int batch, int rank) {
  if (!A || check_tiling(A->n, A->k, A->b1, A->b2) != HYB_OK) return 0;
  if (batch < 1 || batch > 16 || rank < 0 || rank > kMaxRank) return 0;
  Plan P;
  if (make_plan(A->n, A->k, A->b1, A->b2, 2 * A->n_vals + A->n_meta_bytes,
                batch, rank, false, &P) != HYB_OK)
    return 0;
  return P.bytes;
}

int hyb_spmv(const hyb_matrix *A, const uint16_t *X, int64_t ldx, void *Y,
             int64_t ldy, hyb_dtype ydt, const hyb_lowrank *lr, void *ws,
             size_t ws_bytes, hyb_stream_t stream) {
  return spmm_impl(A, 1, X, ldx, Y, ldy, ydt, lr, ws, ws_bytes,
                   (cudaStream_t)stream);
}

int hyb_spmm_skinny(const hyb_matrix *A, int batch, const uint16_t *X,
                    int64_t ldx, void *Y, int64_t ldy, hyb_dtype ydt,
                    const hyb_lowrank *lr, void *ws, size_t ws_bytes,
                    hyb_stream_t stream) {
  return spmm_impl(A, batch, X, ldx, Y, ldy, ydt, lr, ws, ws_bytes,
                   (cudaStream_t)stream);
}

int hyb_spmm_skinny_ex(const hyb_matrix *A, int batch, const uint16_t *X, int64_t ldx,
                       void *Y, int64_t ldy, hyb_dtype ydt, const hyb_lowrank *lr,
                       uint32_t flags, void *ws, size_t ws_bytes, hyb_stream_t stream) {
  return spmm_impl(A, batch, X, ldx, Y, ldy, ydt, lr, ws, ws_bytes, (cudaStream_t)stream,
                   flags);
}

size_t hyb_lowrank_workspace_bytes(int64_t k, int batch, int rank) {
  if (k <= 0 || batch < 1 || batch > 16 || rank < 1 || rank > kMaxRank) return 0;
  size_t a, b, c;
  int ctas;
  return lowrank_ws_layout(k, batch, rank, &a, &b, &c, &ctas);
}

int hyb_lowrank_add(int64_t n, int64_t k, int batch, const hyb_lowrank *lr,
                    const uint16_t *X, int64_t ldx, float *Y, int64_t ldy,
                    void *ws, size_t ws_bytes, hyb_stream_t stream) {
  if (n <= 0 || k <= 0 || !lr || lr->rank < 1) return HYB_ERR_INVALID_ARG;
  int rc = check_io(X, ldx, Y, ldy, n, k, batch, HYB_F32);
  if (rc != HYB_OK) return rc;
  rc = check_lowrank(lr, n, k);
  if (rc != HYB_OK) return rc;
  size_t off_t, off_part, off_counter;
  int ctas;
  const size_t need =
      lowrank_ws_layout(k, batch, lr->rank, &off_t, &off_part, &off_counter, &ctas);
  if (need == 0) return HYB_ERR_CUDA;
  if (!ws || ws_bytes < need) return HYB_ERR_WORKSPACE;
  if ((uintptr_t)ws % 256 != 0) return HYB_ERR_ALIGNMENT;
  cudaStream_t s = (cudaStream_t)stream;
  uint8_t *w = reinterpret_cast<uint8_t *>(ws);
  const int bp = pad_batch(batch);
  {
    const uint16_t *V = lr->V;
    int64_t ldv = lr->ldv, kk = k, ldxx = ldx;
    int rank = lr->rank, bt = batch;
    const uint16_t *Xp = X;
    float *t_out = reinterpret_cast<float *>(w + off_t);
    float *part = reinterpret_cast<float *>(w + off_part);
    uint32_t *counter = reinterpret_cast<uint32_t *>(w + off_counter);
    int zero = 0;
    void *args[] = {&V, &ldv, &rank, &kk, &Xp, &ldxx, &bt, &t_out, &part, &counter, &zero};
    if (cudaLaunchKernel(pick_lowrank_t(bp), dim3(ctas), dim3(kThreads), args, 0, s) !=
        cudaSuccess)
      return HYB_ERR_CUDA;
  }
  {
    int64_t nn = n, ldu = lr->ldu, ldyy = ldy;
    const uint16_t *U = lr->U;
    int rank = lr->rank, bt = batch;
    const float *t = reinterpret_cast<const float *>(w + off_t);
    float *Yp = Y;
    // a programmatic dependent of the V^T x pass, launched plainly just above
    int one = 1;
    void *args[] = {&nn, &U, &ldu, &rank, &t, &bt, &Yp, &ldyy, &one};
    const int64_t grid = (n + kThreads - 1) / kThreads;
    if (launch_kernel(pick_lowrank_apply(bp), dim3((unsigned)grid), dim3(kThreads), args, 0, s,
                      true) != cudaSuccess)
      return HYB_ERR_CUDA;
  }
  return HYB_OK;
}

size_t hyb_dense_workspace_bytes(int64_t n, int64_t k, int batch) {
  if (n <= 0 || k <= 0 || k % 16 != 0 || batch < 1 || batch > 16) return 0;
  int b1, b2;
  dense_tiling(n, k, &b1, &b2);
  Plan P;
  if (make_plan(n, k, b1, b2, 2 * n * k, batch, 0, true, &P) != HYB_OK) return 0;
  return P.bytes;
}

int hyb_gemv_dense(int64_t n, int64_t k, int batch, const uint16_t *W,
                   int64_t ldw, const uint16_t *X, int64_t ldx, void *Y,
                   int64_t ldy, hyb_dtype ydt, void *ws, size_t ws_bytes,
                   hyb_stream_t stream) {
  return hyb_gemv_dense_ex(n, k, batch, W, ldw, X, ldx, Y, ldy, ydt, 0, ws, ws_bytes, stream);
}

int hyb_gemv_dense_ex(int64_t n, int64_t k, int batch, const uint16_t *W, int64_t ldw,
                      const uint16_t *X, int64_t ldx, void *Y, int64_t ldy, hyb_dtype ydt,
                      uint32_t flags, void *ws, size_t ws_bytes, hyb_stream_t stream) {
  if (flags & ~HYB_LAUNCH_OVERLAP_PREV) return HYB_ERR_INVALID_ARG;
  if (n <= 0 || k <= 0 || !W || ldw < k) return HYB_ERR_INVALID_ARG;
  if (k % 16 != 0) return HYB_ERR_INVALID_ARG;
  int rc = check_io(X, ldx, Y, ldy, n, k, batch, ydt);
  if (rc != HYB_OK) return rc;
  int b1, b2;
  dense_tiling(n, k, &b1, &b2);
  // the tuned kernel reads 32-byte pieces of W; the row-per-warp one 16
  const bool wide = b1 > 1;
  if ((uintptr_t)W % (wide ? 32 : 16) != 0 || ldw % (wide ? 16 : 8) != 0)
    return HYB_ERR_ALIGNMENT;
  Params prm{};
  prm.Wd = W;
  prm.ldw = ldw;
  prm.n = n;
  prm.k = k;
  prm.tpr = k / b2;
  prm.T = (n / b1) * (k / b2);
  prm.X = X;
  prm.ldx = ldx;
  prm.batch = batch;
  prm.Y = Y;
  prm.ldy = ldy;
  prm.ydt = ydt;
  prm.total = 2 * n * k;
  return run_product(prm, b1, b2, batch, nullptr, true, ws, ws_bytes,
                     (cudaStream_t)stream, nullptr, 0, flags);
}

}  // extern "C"

// ---------------------------------------------------------------------------
// hyb_spmv_noalloc: the batch-1 product with its scratch in a fixed array.
//
// For callers that may not allocate device memory at all: engines that carve
// every byte out of one arena at start-up, code running while a CUDA graph is
// being captured (where cudaMalloc is not permitted), or hosts whose memory
// pool forbids allocation after initialisation.  hyb_spmv needs a workspace
// from the caller; this variant takes its split partials and band tickets from
// a file-scope device array instead and allocates nothing.
// ---------------------------------------------------------------------------
namespace hyb {
namespace {

// 1 MiB per device, held from module load until the process exits.
constexpr size_t kNoAllocScratchBytes = size_t(1) << 20;
static __device__ __align__(256) uint8_t g_noalloc_scratch[kNoAllocScratchBytes];

// Device address of the array in the current CUDA context.  The name of a
// __device__ variable in host code is only a host-side stand-in, so the
// address is looked up (with the context current) and cached.  The cache is
// keyed on the context, not on the device ordinal: after cudaDeviceReset, or
// in another context on the same device, the module is loaded anew and the
// array lives at another address.
int noalloc_scratch_ptr(void **out) {
  using GetCtx = CUresult (*)(CUcontext *);
  static GetCtx get_ctx = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void *fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &fn, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_ctx = reinterpret_cast<GetCtx>(fn);
  });
  if (!get_ctx) return HYB_ERR_CUDA;
  CUcontext ctx = nullptr;
  if (get_ctx(&ctx) != CUDA_SUCCESS) return HYB_ERR_CUDA;
  if (ctx == nullptr) {
    // no context current yet: the runtime's symbol lookup makes the device's
    // primary context current
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess) return HYB_ERR_CUDA;
    if (get_ctx(&ctx) != CUDA_SUCCESS || ctx == nullptr) return HYB_ERR_CUDA;
  }
  static std::mutex mu;
  struct Entry {
    CUcontext ctx;
    void *addr;
  };
  static Entry cache[64];
  static int used = 0, next = 0;
  std::lock_guard<std::mutex> lock(mu);
  for (int i = 0; i < used; ++i)
    if (cache[i].ctx == ctx) {
      *out = cache[i].addr;
      return HYB_OK;
    }
  void *p = nullptr;
  if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr)
    return HYB_ERR_CUDA;
  // a full table recycles its oldest entry
  const int slot = used < 64 ? used++ : (next++ % 64);
  cache[slot] = Entry{ctx, p};
  *out = p;
  return HYB_OK;
}

// The argument checks of the batch-1 product, run before anything is queued.
int noalloc_validate(const hyb_matrix *A, const uint16_t *X, int64_t ldx,
                     void *Y, int64_t ldy, int ydt) {
  if (!A) return HYB_ERR_INVALID_ARG;
  int rc = check_tiling(A->n, A->k, A->b1, A->b2);
  if (rc != HYB_OK) return rc;
  if (A->num_tiles != (A->n / A->b1) * (A->k / A->b2)) return HYB_ERR_INVALID_ARG;
  if (!A->tile_map || !A->vals || !A->meta || !A->val_off || !A->meta_off)
    return HYB_ERR_INVALID_ARG;
  const int64_t te = (int64_t)A->b1 * A->b2;
  if (A->n_vals < A->num_tiles * te / 2 || A->n_vals > A->num_tiles * te ||
      A->n_meta_bytes < 0 || A->n_meta_bytes > A->num_tiles * te / 8)
    return HYB_ERR_INVALID_ARG;
  if (((uintptr_t)A->vals) % 32 != 0 || ((uintptr_t)A->meta) % 16 != 0)
    return HYB_ERR_ALIGNMENT;
  return check_io(X, ldx, Y, ldy, A->n, A->k, 1, ydt);
}

}  // namespace
}  // namespace hyb

extern "C" {

size_t hyb_spmv_noalloc_max_scratch_bytes(void) {
  return hyb::kNoAllocScratchBytes;
}

int hyb_spmv_noalloc(const hyb_matrix *A, const uint16_t *X, int64_t ldx,
                     void *Y, int64_t ldy, hyb_dtype ydt, hyb_stream_t stream) {
  int rc = hyb::noalloc_validate(A, X, ldx, Y, ldy, ydt);
  if (rc != HYB_OK) return rc;
  hyb::Plan P;
  rc = hyb::make_plan(A->n, A->k, A->b1, A->b2, 2 * A->n_vals + A->n_meta_bytes,
                      1, 0, false, &P);
  if (rc != HYB_OK) return rc;
  if (P.bytes > hyb::kNoAllocScratchBytes) return HYB_ERR_WORKSPACE;
  void *scratch = nullptr;
  rc = hyb::noalloc_scratch_ptr(&scratch);
  if (rc != HYB_OK) return rc;
  cudaStream_t s = (cudaStream_t)stream;
  // The array keeps whatever the previous call left.  The band tickets must
  // start at zero (the partial slots are always written before they are
  // read), so clear everything between the header and the slots.  The status
  // word at the head is not cleared: it collects the flags of every call
  // until hyb_spmv_noalloc_check_status reads and clears it.
  if (cudaMemsetAsync(static_cast<uint8_t *>(scratch) + hyb::kHeaderBytes, 0,
                      P.off_partials - hyb::kHeaderBytes, s) != cudaSuccess)
    return HYB_ERR_CUDA;
  return hyb::spmm_impl(A, 1, X, ldx, Y, ldy, ydt, nullptr, scratch,
                        hyb::kNoAllocScratchBytes, s);
}

int hyb_spmv_noalloc_check_status(hyb_stream_t stream, uint32_t *flags) {
  void *scratch = nullptr;
  const int rc = hyb::noalloc_scratch_ptr(&scratch);
  if (rc != HYB_OK) return rc;
  return hyb_check_status(scratch, stream, flags);
}

int hyb_selftest_wait_timeout(void *ws, size_t ws_bytes, uint32_t wait_limit,
                              hyb_stream_t stream) {
  if (ws == nullptr || ws_bytes < hyb::kHeaderBytes) return HYB_ERR_WORKSPACE;
  if ((uintptr_t)ws % 256 != 0) return HYB_ERR_ALIGNMENT;
  if (wait_limit < 1 || wait_limit > (1u << 20)) return HYB_ERR_INVALID_ARG;
  hyb::selftest_wait_timeout_kernel<<<1, 32, 0, (cudaStream_t)stream>>>(
      reinterpret_cast<uint32_t *>(ws), wait_limit);
  return cudaGetLastError() == cudaSuccess ? HYB_OK : HYB_ERR_CUDA;
}

}  // extern "C"
