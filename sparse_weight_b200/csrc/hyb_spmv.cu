// hyb_spmv.cu -- Y = W_hat X (+ U (V^T X)) for the tile-hybrid format, the
// dense GEMV baseline and the stand-alone low-rank term.
//
// Decode-time products are memory-bound ("SparseDecoding: decoding-aware
// pruning ...", authors' abstract: the decode phase is limited by memory
// access and is dominated by sparse matrix-vector products), so every kernel
// here is a single streaming pass over the weight bytes with no tensor cores.
//
//  * hybrid_tma_kernel (tilings 128x128, 128x64, 64x64, 64x128): the packed
//    stream is row-major over tiles, so every tile-row band is contiguous.
//    CTA c of G takes the tiles whose byte offset falls in [c, c+1) * total /
//    G -- a split by bytes, not by tiles, because a dense tile costs
//    2 B/weight and a 2:4 tile 1.125 B/weight ("PATCH: Learnable Tile-level
//    Hybrid Sparsity for LLMs", §2: tiles are dense or 2:4).  A producer warp
//    moves the bytes into a shared-memory ring with bulk copies; consumer
//    warps compute from it; two epilogue warps finish the bands; a low-rank
//    warp computes the L = U V^T term ("3BASiL", §1: W ~ S + L) in the same
//    pass.  The same kernel streams a plain row-major W (every tile dense,
//    each tile one 2-D tensor copy): the dense baseline the format is
//    measured against.
//  * hybrid_rowwarp_kernel (any other legal tiling, packed or row-major): one
//    warp per output row, plain loads.
//  * Band results cross CTAs through fp32 partial slots; the last CTA to
//    arrive at a band (atomic ticket, no spinning) sums the slots in CTA order
//    -- deterministic -- and applies the epilogue: the low-rank term and the
//    fp32 or bf16 store.
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
  // matrix: packed, or (rowmajor) a plain row-major bf16 W read through the
  // kernel's W tensor map, every b1 x b2 tile dense
  int rowmajor;
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
  // low rank: t = V^T x (fp32 [BP][rank]) and ut = U t (fp32 [BP][n]); the
  // product's epilogue adds ut.  Fused (streaming kernel): the kernel's
  // low-rank warp computes both, with lr_part ([G][BP][rank] partials of t),
  // lr_epoch (the calls' barrier epoch) and lr_flags (one barrier flag per
  // CTA) in the workspace.  Not fused (other tilings): two small kernels
  // compute them before the product.
  const uint16_t *U;
  int64_t ldu;
  const uint16_t *V;
  int64_t ldv;
  int rank;
  int fused_lr;
  float *lr_t;
  // t computed by an earlier call that shares V (gate and up of one input):
  // the fused low-rank warp, or the call's kernels, then compute U t only
  const float *lr_t_in;
  float *lr_ut;
  float *lr_part;
  uint32_t *lr_epoch;
  uint32_t *lr_flags;
  // split
  int G;
  int nst;        // ring stages this launch uses (at most the kernel's compile-time count)
  int64_t total;  // packed bytes of the whole matrix
  float *partials;
  uint32_t *counters;
  uint32_t *status;  // workspace status word
  int64_t nvb, nmb;  // bytes of the value and mask buffers
  // 1: launched as a programmatic dependent of the preceding kernel on the
  // stream.  The weights (packed matrix or row-major W, and U, V) may then be
  // read before that kernel has finished; X, Y and the workspace are touched
  // only after griddepcontrol.wait.
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

// Select x[p0] and x[p1] of one group from its 4-bit mask (two bits set):
// p0 is the lowest set bit, p1 the highest.
__device__ __forceinline__ void pick2(uint32_t nib, float x0, float x1,
                                      float x2, float x3, float &xa,
                                      float &xb) {
  xa = (nib & 1u) ? x0 : ((nib & 2u) ? x1 : x2);
  xb = (nib & 8u) ? x3 : ((nib & 4u) ? x2 : x1);
}

// Epilogue for one (row, batch) output: add the low-rank term, store.
__device__ __forceinline__ void store_out(const Params &p, int64_t row, int b,
                                          float y) {
  if (p.lr_ut != nullptr) y += __ldcg(p.lr_ut + (int64_t)b * p.n + row);
  if (p.ydt == HYB_BF16)
    reinterpret_cast<uint16_t *>(p.Y)[(int64_t)b * p.ldy + row] =
        f32_to_bf16_rne(y);
  else
    reinterpret_cast<float *>(p.Y)[(int64_t)b * p.ldy + row] = y;
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

// The low-rank warp's chunk buffer after the ring: two halves (16 KB of
// dynamic shared memory, requested only by launches with a low-rank term;
// such launches may use one ring stage fewer to make room).
constexpr int kLrHalf = 8192;
constexpr int kLrBufBytes = 2 * kLrHalf;

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
__device__ __forceinline__ uint32_t ld_acquire_u32(const uint32_t *addr) {
  uint32_t v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(addr) : "memory");
  return v;
}
__device__ __forceinline__ void st_release_u32(uint32_t *addr, uint32_t v) {
  asm volatile("st.release.gpu.global.u32 [%0], %1;" ::"l"(addr), "r"(v) : "memory");
}

// Grid barrier over the G CTAs of a launch, called by one whole warp per CTA.
// Every CTA has a flag word; arriving CTA c publishes flags[c] = target with
// a release store (after a warp barrier, so that it covers everything the
// warp wrote before), and the warp's lanes then poll all G flags until each
// has reached target.  No atomics, so arrivals do
// not queue on one address.  Targets are per call: the call's epoch (read
// from the workspace at the start) plus the barrier's number, so flags left
// by earlier calls are always behind.  Needs every CTA of the grid to be
// resident at some point while the others wait: the streaming kernel runs at
// most one CTA per SM and no more CTAs than SMs.  The wait is bounded: false
// when it ran out.
constexpr uint32_t kGridWaitLimit = 1u << 20;
__device__ __forceinline__ bool flag_barrier(uint32_t *flags, int G, int c, uint32_t target,
                                             int lane) {
  __syncwarp();
  if (lane == 0) st_release_u32(flags + c, target);
  // each lane polls the flags of CTAs lane, lane + 32, ... with acquire
  // loads, so what a CTA published before its flag is visible after the wait
  bool done = false;
  for (uint32_t i = 0; i < kGridWaitLimit && !done; ++i) {
    bool mine = true;
    for (int q = lane; q < G; q += 32) mine &= (int32_t)(ld_acquire_u32(flags + q) - target) >= 0;
    done = __all_sync(0xffffffffu, mine);
    if (!done) __nanosleep(32);
  }
  __syncwarp();
  return done;
}

// 16-byte asynchronous copy global -> shared through the load/store path
// (L2 only), completion tracked per thread by commit / wait groups.  Used for
// the low-rank warp's small chunks so they do not queue in the TMA engine
// behind the ring's stage copies.
__device__ __forceinline__ void cp_async16(void *dst, const void *src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(dst)), "l"(src)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
  asm volatile("cp.async.commit_group;" ::: "memory");
}
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// acc += lo(w) * lo(x) + hi(w) * hi(x) on two packed bf16 pairs.
__device__ __forceinline__ void fma_bf16x2(float &acc, uint32_t w, uint32_t x) {
  unsigned short wl, wh, xl, xh;
  asm("mov.b32 {%0,%1}, %2;" : "=h"(wl), "=h"(wh) : "r"(w));
  asm("mov.b32 {%0,%1}, %2;" : "=h"(xl), "=h"(xh) : "r"(x));
  asm("fma.rn.f32.bf16 %0, %1, %2, %0;" : "+f"(acc) : "h"(wl), "h"(xl));
  asm("fma.rn.f32.bf16 %0, %1, %2, %0;" : "+f"(acc) : "h"(wh), "h"(xh));
}

// D (16 x 8, fp32) += A (16 x 16, bf16, row-major) B (16 x 8, bf16, "col"):
// one warp-wide tensor-core product.  Lane (g, c) = (lane / 4, lane % 4)
// holds A rows g and g + 8 at k = 2c, 2c + 1 (a0, a1) and 2c + 8, 2c + 9
// (a2, a3), B column g at the same k (b0, b1), and D rows g, g + 8 at
// columns 2c, 2c + 1.
__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], uint32_t a0, uint32_t a1,
                                               uint32_t a2, uint32_t a3, uint32_t b0,
                                               uint32_t b1) {
  asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, "
      "{%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

template <int BP, int B1, int B2, bool LR = false, int PAT = 0>
struct TmaCfg {
  // From batch 4 on, dense and 2:4 tiles go through the tensor cores (the
  // batch is the product's M side, padded to 16; a 2:4 tile row is expanded
  // to dense bf16 pairs in registers); narrower batches, and 4:8 tiles, use
  // scalar FMAs.
  static constexpr bool MMA = BP >= 4 && PAT == 0;
  // rows per consumer warp: 8; 16 from batch 4 on (scalar: fewer warps,
  // each reusing its X registers over more rows; tensor cores: two 8-row
  // product columns per warp, eight warps for a 128-row tile -- four warps
  // leave the tensor products too little overlap, sixteen re-read X too often)
  static constexpr int RW = BP >= 4 ? 16 : 8;
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
  // consumers, producer, 2 epilogue warps (and, in the instances for calls
  // with a low-rank term, the low-rank warp: the others carry none of its
  // code)
  static constexpr int kThreads = (NC + 3 + (LR ? 1 : 0)) * 32;
  static constexpr size_t kSmem = (size_t)kStages * kStageBytes + 1024;
  static_assert(MMA || (RPS * CPR == 32 && JS * RPS == RW && JS >= 1), "tile shape");
  static_assert(!MMA || (B2 % 64 == 0 && B1 % RW == 0), "tensor-core tile shape");
  static_assert(kStages >= 3, "ring too short");
  static_assert(TPX <= 8 && WIN < 32, "stage / offset window");
  static_assert(TPX % XT == 0 && (!XTM || XT * B2 <= 256), "X copy groups");
};

// Stage starts of a window of nw tiles beginning at tile w0 (bit i: a stage
// starts at tile w0 + i): greedy packing by value bytes, in units of a 2:4
// tile (a dense tile is 2), at most 2 tpd units and tpx tiles per stage, and
// a new stage at every band start.  Used by the streaming kernel for every
// window and by the plan for each CTA's first window.
__device__ __forceinline__ uint32_t stage_starts(uint32_t spm, int nw, uint32_t w0_col, int tpr,
                                                int tpd, int tpx) {
  // (w0_col = w0 mod tpr: the tile column of w0 within its band)
  int nb = (int)(((uint32_t)tpr - w0_col) % (uint32_t)tpr);  // first band start at or after w0
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

// U t for up to `rows` rows of a U chunk in shared memory (rows of r bf16),
// CPL = r / 8 lanes per row, 32 / CPL rows side by side, one batch column at
// a time.  Each lane adds its 16-byte chunk's products for CPL rows of its
// group, then a butterfly over the group's lanes (halving the rows at each
// step: CPL - 1 shuffles) leaves lane c of the group with the whole dot
// product of the group's row c, which it stores (consecutive lanes,
// consecutive rows).  The sum over the lanes has a fixed order.  tv holds
// the lane's 8 columns of t for LB batch columns.  ut: the chunk's first
// output row (row stride 1, batch stride n).
template <int CPL, int LB>
__device__ __forceinline__ bool ut_block(const uint8_t *src, int rows, int r,
                                         const float (&tv)[LB][8], int lane, float *ut, int64_t n,
                                         int b0) {
  constexpr int RG = 32 / CPL;
  const int g = lane / CPL, c = lane % CPL;
  for (int blk = 0; blk < rows; blk += RG * CPL) {
#pragma unroll
    for (int b = 0; b < LB; ++b) {
      float v[CPL];
#pragma unroll
      for (int i = 0; i < CPL; ++i) {
        const int row = blk + g * CPL + i;
        float part = 0.f;
        if (row < rows) {
          const uint4 u = *reinterpret_cast<const uint4 *>(src + (size_t)row * r * 2 + 16 * c);
          part = fmaf(bf16_lo(u.x), tv[b][0], part);
          part = fmaf(bf16_hi(u.x), tv[b][1], part);
          part = fmaf(bf16_lo(u.y), tv[b][2], part);
          part = fmaf(bf16_hi(u.y), tv[b][3], part);
          part = fmaf(bf16_lo(u.z), tv[b][4], part);
          part = fmaf(bf16_hi(u.z), tv[b][5], part);
          part = fmaf(bf16_lo(u.w), tv[b][6], part);
          part = fmaf(bf16_hi(u.w), tv[b][7], part);
        }
        v[i] = part;
      }
      // butterfly: at stride s a lane keeps the half of its 2s rows whose
      // index has bit s equal to its own and adds its partner's copy of them
#pragma unroll
      for (int s = CPL / 2; s >= 1; s /= 2) {
        const bool hi = (c & s) != 0;
#pragma unroll
        for (int i = 0; i < s; ++i) {
          const float send = hi ? v[i] : v[i + s];
          const float keep = hi ? v[i + s] : v[i];
          v[i] = keep + __shfl_xor_sync(0xffffffffu, send, s);
        }
      }
      const int row = blk + g * CPL + c;
      if (row < rows) __stcg(ut + (int64_t)(b0 + b) * n + row, v[0]);
    }
  }
  return true;
}

// Selectors of a 4:8 mask byte for the two-PRMT x pairs of the consumers:
// x[c0], x[c1] through T = PRMT(X0, X1, s1) and PRMT(T, X2, s2); x[c2], x[c3]
// through T' = PRMT(X2, X3, s3) and PRMT(X1, T', s4).  Entry .x = s1 | s2 << 16,
// .y = s3 | s4 << 16; 0 for a byte without exactly four bits set.
__device__ __forceinline__ uint2 lut48_entry(uint32_t m) {
  if (__popc(m) != 4) return make_uint2(0u, 0u);
  int c[4], n = 0;
  for (int i = 0; i < 8; ++i)
    if ((m >> i) & 1u) c[n++] = i;
  auto pair = [](int lo, int hi) -> uint32_t {  // nibbles of the bytes lo, lo+1, hi, hi+1
    return (uint32_t)lo | (uint32_t)(lo + 1) << 4 | (uint32_t)hi << 8 | (uint32_t)(hi + 1) << 12;
  };
  // T: x[c0], x[c1] from X0:X1 when below column 4 (bytes 2c, 2c+1)
  const uint32_t s1 = pair(c[0] < 4 ? 2 * c[0] : 0, c[1] < 4 ? 2 * c[1] : 0);
  // pair A from T (bytes 0..3) or X2 (bytes 4..7 hold x4, x5)
  const uint32_t s2 = pair(c[0] < 4 ? 0 : 4 + 2 * (c[0] - 4), c[1] < 4 ? 2 : 4 + 2 * (c[1] - 4));
  // T': x[c2], x[c3] from X2:X3 when at or above column 4
  const uint32_t s3 = pair(c[2] >= 4 ? 2 * (c[2] - 4) : 0, c[3] >= 4 ? 2 * (c[3] - 4) : 0);
  // pair B from X1 (bytes 0..3 hold x2, x3) or T' (bytes 4..7)
  const uint32_t s4 = pair(c[2] < 4 ? 2 * (c[2] - 2) : 4, c[3] < 4 ? 2 * (c[3] - 2) : 6);
  return make_uint2(s1 | s2 << 16, s3 | s4 << 16);
}

// PAT 0: 2:4 tiles (hyb_pack); PAT 1: 4:8 tiles (hyb_pack_nm with 4 of 8).
// LR: the instance for calls with a low-rank term (an extra warp computes it).
template <int BP, int B1, int B2, int PAT, bool LR>
__global__ void __launch_bounds__(TmaCfg<BP, B1, B2, LR, PAT>::kThreads, 1)
    hybrid_tma_kernel(const Params p, const LaunchPlan lp, const __grid_constant__ CUtensorMap xmap,
                      const __grid_constant__ CUtensorMap wmap) {
  using C = TmaCfg<BP, B1, B2, LR, PAT>;
  constexpr int S = C::kStages;
  extern __shared__ __align__(1024) uint8_t smem[];
  __shared__ __align__(8) uint64_t full_bar[S];
  __shared__ __align__(8) uint64_t empty_bar[S];
  __shared__ StageDesc desc[S];
  __shared__ uint32_t sel_lut[16];
  __shared__ uint32_t sel_dense[16];
  __shared__ uint2 lut48[PAT == 1 ? 256 : 1];
  __shared__ uint32_t s_cnt[2];
  __shared__ int64_t s_range[2];
  // a CTA's piece of a band: row sums handed from the consumer warps to the
  // epilogue warp through a 2-slot ring, [slot][warp][b * RW + row]
  __shared__ float s_rows[2][C::NC][C::RW * BP];
  __shared__ __align__(8) uint64_t piece_full[2];
  __shared__ __align__(8) uint64_t piece_empty[2];
  // the low-rank warp's U t is complete (or its wait ran out, which it
  // records in the status word)
  __shared__ __align__(8) uint64_t lr_done;

  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  const int c = blockIdx.x;
  const int G = p.G;
  const int tpr = (int)p.tpr;
  __shared__ int64_t s_rec[5];
  const bool planned = lp.kind == kPlanTiles;
  // With a plan, or a row-major W, the CTA's range needs no search.  Then the
  // producer warp sets up the mbarriers itself, signals the other warps with
  // a non-blocking arrive on named barrier 1 and goes straight on to request
  // its first ring of stages; the other warps wait on that barrier.  (Without
  // a plan every thread takes part in the search, behind __syncthreads.)
  const bool fast = planned || p.rowmajor;
  if (p.pdl) grid_dep_trigger();
  auto init_barriers = [&]() {
    for (int s = 0; s < S; ++s) {
      mbar_init(&full_bar[s], 1);
      mbar_init(&empty_bar[s], C::NC);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&piece_full[s], C::NC);
      mbar_init(&piece_empty[s], 1);
    }
    mbar_init(&lr_done, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  };
  if (fast && warp == C::NC) {
    if (lane == 0) {
      init_barriers();
      if (planned) {
        s_rec[0] = lp.rec[4 * c];
        s_rec[1] = lp.rec[4 * (c + 1)];
        s_rec[2] = lp.rec[4 * c + 1];
        s_rec[3] = lp.rec[4 * c + 2];
        s_rec[4] = lp.rec[4 * c + 3];
      } else {
        // every tile costs the same: CTA c takes tiles [ceil(c T / G), ceil((c+1) T / G))
        s_range[0] = ((int64_t)c * p.T + G - 1) / G;
        s_range[1] = ((int64_t)(c + 1) * p.T + G - 1) / G;
      }
    }
    // this warp's entries of the 4:8 selector table (the other warps fill
    // theirs below); like the barriers, they are published by bar.arrive 1
    if constexpr (PAT == 1) {
      for (int m = tid; m < 256; m += blockDim.x) lut48[m] = lut48_entry((uint32_t)m);
    }
    __syncwarp();
    asm volatile("bar.arrive 1, %0;" ::"r"(C::kThreads) : "memory");
  } else {
    if (tid == 0 && !fast) {
      init_barriers();
      s_cnt[0] = 0;
      s_cnt[1] = 0;
      if (planned) {  // (a plan always takes the fast path; kept for robustness)
        s_rec[0] = lp.rec[4 * c];
        s_rec[1] = lp.rec[4 * (c + 1)];
        s_rec[2] = lp.rec[4 * c + 1];
        s_rec[3] = lp.rec[4 * c + 2];
        s_rec[4] = lp.rec[4 * c + 3];
      }
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
      // PRMT selectors expanding a kept pair (v_p0 in bytes 0-1, v_p1 in
      // bytes 2-3, zero bytes 4-7) to the group's dense columns 0-1 (low
      // half) and 2-3 (high half); a column not kept takes zero bytes
      uint32_t sd = 0;
      for (int j = 0; j < 4; ++j) {
        const uint32_t lo = !m ? 4u : (j == (int)p0 ? 0u : (j == (int)p1 ? 2u : 4u));
        const uint32_t hi = lo == 4u ? 4u : lo + 1u;
        sd |= (lo | hi << 4) << (8 * j);
      }
      sel_dense[m] = sd;
    }
    if constexpr (PAT == 1) {
      for (int m = tid; m < 256; m += blockDim.x) lut48[m] = lut48_entry((uint32_t)m);
    }
    if (fast) asm volatile("bar.sync 1, %0;" ::"r"(C::kThreads) : "memory");
  }
  if (!fast) __syncthreads();

  // ---- this CTA's tiles [t0, t1): tiles whose packed offset P(t) satisfies
  // c*total <= P(t)*G < (c+1)*total.  With a plan the producer and the
  // epilogue warp take them from the launch parameters; a row-major W has
  // them in closed form; otherwise round 1 brackets both ends between band
  // starts and round 2 counts inside the bracketing band. ----
  if (!fast && !planned) {
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
      // band starts below each target (at most R: the bracketing band is a
      // real one even when a corrupted matrix puts the end below a target)
      const uint32_t bA = min(s_cnt[0], (uint32_t)p.R), bB = min(s_cnt[1], (uint32_t)p.R);
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
    if (p.rowmajor && lane == 1)
      asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&wmap))
                   : "memory");
    // Tiles are taken in windows of WIN: lane i holds the packed offsets of
    // tile w0 + i (and lane WIN those of the window's end), the next window
    // is loaded while this one is issued.  Stages are packed greedily inside
    // a window: a new stage starts at a band start or when the next tile no
    // longer fits in the 32 KB value buffer; every lane runs the same packing
    // over the window's 2:4 bitmask, so all agree on the stage starts.
    struct Win {
      int64_t vo, mo;
      uint32_t sp;  // the tile's map byte (1: a 2:4 tile)
    };
    // (volatile loads: the compiler may not turn the window load that a
    // plan makes unnecessary into a speculative load the first window waits
    // on; and nothing here inspects the loaded values, so the next window's
    // loads stay in flight while this one issues)
    auto load_win = [&](int64_t w0) -> Win {
      Win o{0, 0, 0};
      const int64_t t = w0 + lane;
      if (p.rowmajor) {  // dense tiles, offsets in closed form, nothing to load
        o.vo = t * ((int64_t)B1 * B2);
        return o;
      }
      if (lane <= C::WIN && t <= t1) {
        o.vo = ld_volatile_nc64(p.val_off + t);
        o.mo = ld_volatile_nc64(p.meta_off + t);
      }
      if (lane < C::WIN && t < t1) o.sp = ld_volatile_nc8(p.map + t);
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
      const uint32_t spm = __ballot_sync(0xffffffffu, cur.sp == 1u);
      // band and tile column of w0 (tile indices fit 32 bits on this path)
      const uint32_t tpu = (uint32_t)tpr;
      const uint32_t wband = (uint32_t)w0 / tpu, wcol = (uint32_t)w0 - wband * tpu;
      if (!p.rowmajor && !(derived && w0 == t0)) {
        // offsets read from the matrix must step by each tile's size (a
        // corrupted matrix is flagged; the copies are bounded either way)
        constexpr int64_t TE = (int64_t)B1 * B2;
        const int64_t nvo = __shfl_down_sync(0xffffffffu, cur.vo, 1);
        const int64_t nmo = __shfl_down_sync(0xffffffffu, cur.mo, 1);
        const bool sp = cur.sp == 1u;
        const bool bad = lane < nw && (nvo - cur.vo != (sp ? TE / 2 : TE) ||
                                       nmo - cur.mo != (sp ? TE / 8 : 0));
        if (__any_sync(0xffffffffu, bad) && lane == 0) atomicOr(p.status, kStatusBadMap);
      }
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
        const bool band_ok = lane >= nw || (wcol + lane) % tpu != 0 || (starts >> lane & 1u);
        have = __all_sync(0xffffffffu, good && band_ok) && (starts & 1u) && (starts >> nw) == 0;
      }
      if (!have) starts = stage_starts(spm, nw, wcol, tpr, C::TPD, C::TPX);
      // the stage that starts at this lane: tiles [w0 + lane, w0 + e).  Every
      // start lane works out its stage here, all at once, so that the serial
      // part below (one stage after the other, as ring slots free up) only
      // waits and issues.
      const bool is_start = lane < nw && (starts >> lane & 1u);
      const uint32_t later = lane < 31 ? (starts >> (lane + 1)) : 0u;
      const int e = later ? lane + 1 + __ffs(later) - 1 : nw;
      const int64_t v_end = __shfl_sync(0xffffffffu, cur.vo, e & 31);
      const int64_t m_end = __shfl_sync(0xffffffffu, cur.mo, e & 31);
      // (e == 32 only when nw == 32, which WIN < 32 rules out)
      const int nt = e - lane;
      const int64_t ts = w0 + lane, te = w0 + e;
      // the stage's byte ranges, from the tile offsets: a range that does not
      // fit the buffers, the stage or 16-byte alignment (a corrupted matrix)
      // is not copied and is flagged; the consumers then read stale stage
      // bytes, never outside the stage
      const int64_t vb = 2 * (v_end - cur.vo), mb = m_end - cur.mo;
      const bool fits = p.rowmajor || (cur.vo >= 0 && cur.mo >= 0 && vb > 0 && mb >= 0 &&
                                       vb <= C::kValsBytes && mb <= C::kMetaBytes &&
                                       2 * cur.vo + vb <= p.nvb && cur.mo + mb <= p.nmb &&
                                       ((2 * cur.vo) | vb | cur.mo | mb) % 16 == 0);
      if (__any_sync(0xffffffffu, is_start && !fits) && lane == 0) atomicOr(p.status, kStatusBadMap);
      const uint32_t vbytes = fits ? (uint32_t)vb : 0u;
      const uint32_t mbytes = fits ? (uint32_t)mb : 0u;
      const int ngx = (nt + C::XT - 1) / C::XT;  // X copy groups (tensor path)
      const uint32_t xbytes =
          C::XTM ? (uint32_t)(ngx * C::kXCopy) : (uint32_t)(2 * B2 * nt) * (uint32_t)p.batch;
      const int64_t band = wband + (wcol + lane) / tpu;  // = ts / tpr
      StageDesc dl;
      dl.t0 = ts;
      dl.ntiles = (uint16_t)nt;
      dl.sparse = (uint8_t)((spm >> lane) & ((1u << (nt & 31)) - 1u));
      dl.flags = (te == (band + 1) * tpr || te == t1) ? 1 : 0;
      const int64_t xcol = (ts - band * tpr) * B2;  // first X column of the stage
      uint32_t todo = starts;
      while (todo) {
        const int k = __ffs(todo) - 1;
        todo &= todo - 1;
        if (pend && issued == p.nst) release_x();  // the ring is armed: X can wait no longer
        if (lane == k && is_start) {
          if (!mbar_wait(&empty_bar[stage], phase ^ 1u)) {
            ok = false;
          } else {
            uint8_t *st = smem + (size_t)stage * C::kStageBytes;
            desc[stage] = dl;
            armed |= 1u << stage;
            armed_parity = (armed_parity & ~(1u << stage)) | (phase << stage);
            mbar_arrive_expect_tx(&full_bar[stage], vbytes + mbytes + xbytes);
            if (p.rowmajor) {
              // one 2-D tensor copy per tile: box [B1 rows][B2 columns] of W,
              // which lands in the packed dense tile layout
              int64_t tr = band, tc = ts - band * tpr;
              for (int q = 0; q < nt; ++q) {
                tma_load_2d(st + (size_t)q * 2 * B1 * B2, &wmap, (int)(tc * B2), (int)(tr * B1),
                            &full_bar[stage]);
                if (++tc == tpr) {
                  tc = 0;
                  ++tr;
                }
              }
            } else {
              if (vbytes) bulk_g2s(st, p.vals + 2 * cur.vo, vbytes, &full_bar[stage]);
              if (mbytes) bulk_g2s(st + C::kValsBytes, p.meta + cur.mo, mbytes, &full_bar[stage]);
            }
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
        if (++stage == p.nst) {
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

  if (LR && warp == C::NC + 3) {
    // ------------------------------ low rank ------------------------------
    // The L = U V^T term of "3BASiL" (§1: W ~ S + L), fused into the pass:
    // (1) a partial t = V^T x over this CTA's slice of V's rows; (2) once
    // every CTA has written its partial, elements [E c / G, E (c+1) / G) of
    // t, each the sum of the G partials in CTA order; (3) once t is whole,
    // U t for this CTA's slice of the output rows.  A grid barrier separates
    // the steps; the epilogue warps wait for the last one (lr_done) before
    // their first final store, and add U t there.  The V and U rows (and the
    // X slice) come in by bulk copies into two 8 KB halves of a buffer after
    // the ring, one chunk in flight while the other is used.  Every sum has a
    // fixed order, so results do not depend on timing.
    if (!p.fused_lr) return;
    if (p.pdl) grid_dep_wait();  // X and the workspace may belong to the preceding grid
    constexpr int LB = BP < 4 ? BP : 4;  // batch columns per pass
    const uint32_t full = 0xffffffffu;
    const int r = p.rank;
    const int cpl = r / 8;                          // 16-byte chunks of a V or U row
    const int rg = (32 % cpl == 0) ? 32 / cpl : 1;  // rows handled side by side
    const int chunk = lane % cpl, rgrp = lane / cpl;
    const bool active = lane < cpl * rg;
    const int64_t E = (int64_t)BP * r;  // elements of t (padded batch)
    uint8_t *lrbuf = smem + (size_t)p.nst * C::kStageBytes;
    bool ok = true;
    // this call's barrier epoch (every CTA reads it before its first arrival;
    // CTA 0 advances it after the last barrier)
    const uint32_t epoch = __shfl_sync(full, lane == 0 ? ld_acquire_u32(p.lr_epoch) : 0u, 0);
    // Copy chunks [0, nch) through the two halves, calling use(j, half) on
    // each once it has landed; issue(j, half) has every lane request its
    // 16-byte pieces of chunk j.  Two chunks in flight, one commit group each.
    auto pipeline = [&](int nch, auto &&issue, auto &&use) {
      if (nch > 0) issue(0, lrbuf);
      cp_async_commit();
      if (nch > 1) issue(1, lrbuf + kLrHalf);
      cp_async_commit();
      for (int j = 0; j < nch; ++j) {
        cp_async_wait<1>();  // chunk j has landed (at most chunk j + 1 pending)
        __syncwarp();
        use(j, lrbuf + (j & 1) * kLrHalf);
        __syncwarp();
        if (j + 2 < nch) issue(j + 2, lrbuf + (j & 1) * kLrHalf);
        cp_async_commit();
      }
      cp_async_wait<0>();
      __syncwarp();
    };
    // lanes copy `bytes` contiguous bytes (a multiple of 16) in 16-byte pieces
    auto copy_span = [&](uint8_t *dst, const void *src, uint32_t bytes) {
      const uint8_t *g = reinterpret_cast<const uint8_t *>(src);
      for (uint32_t o = 16u * lane; o < bytes; o += 512u) cp_async16(dst + o, g + o);
    };
    // (1) partial t over rows [k0, k1) of V, multiples of 8 so that the X
    // rows' copies start on 16-byte boundaries; a chunk holds rc rows of V
    // and the same rows of X for four batch columns
    if (!p.lr_t_in) {  // V^T x here (else t comes from an earlier call)
      const int64_t k8 = p.k / 8;
      const int64_t k0 = 8 * (k8 * c / G), k1 = 8 * (k8 * (c + 1) / G);
      const int rc = max(8, (kLrHalf / (2 * r + 2 * 4)) / 8 * 8);
      const int nch = (int)((k1 - k0 + rc - 1) / rc);
      float *mine = p.lr_part + (int64_t)c * E;
#pragma unroll 1
      for (int b0 = 0; b0 < BP && ok; b0 += 4) {
        const int nb = min(4, p.batch - b0);  // batch rows of X in this pass (<= 0: none)
        float acc[4][8];
#pragma unroll
        for (int b = 0; b < 4; ++b)
#pragma unroll
          for (int e = 0; e < 8; ++e) acc[b][e] = 0.f;
        auto issue = [&](int j, uint8_t *dst) {
          const int64_t row0 = k0 + (int64_t)j * rc;
          const int rows = (int)min((int64_t)rc, k1 - row0);
          const uint32_t vb = (uint32_t)rows * r * 2, xb = (uint32_t)rows * 2;
          if (p.ldv == r)
            copy_span(dst, p.V + row0 * p.ldv, vb);
          else
            for (int i = 0; i < rows; ++i)
              copy_span(dst + (size_t)i * r * 2, p.V + (row0 + i) * p.ldv, (uint32_t)r * 2);
          for (int b = 0; b < nb; ++b)
            copy_span(dst + (size_t)rc * r * 2 + (size_t)b * rc * 2,
                      p.X + (int64_t)(b0 + b) * p.ldx + row0, xb);
        };
        auto use = [&](int j, const uint8_t *src) {
          const int64_t row0 = k0 + (int64_t)j * rc;
          const int rows = (int)min((int64_t)rc, k1 - row0);
          if (!active) return;
          const uint16_t *xsm = reinterpret_cast<const uint16_t *>(src + (size_t)rc * r * 2);
          for (int i = rgrp; i < rows; i += rg) {
            const uint4 v = *reinterpret_cast<const uint4 *>(src + (size_t)i * r * 2 + 16 * chunk);
            const float vf[8] = {bf16_lo(v.x), bf16_hi(v.x), bf16_lo(v.y), bf16_hi(v.y),
                                 bf16_lo(v.z), bf16_hi(v.z), bf16_lo(v.w), bf16_hi(v.w)};
#pragma unroll
            for (int b = 0; b < 4; ++b) {
              if (b < nb) {
                const float xv = __uint_as_float((uint32_t)xsm[b * rc + i] << 16);
#pragma unroll
                for (int e = 0; e < 8; ++e) acc[b][e] = fmaf(vf[e], xv, acc[b][e]);
              }
            }
          }
        };
        if (nb > 0) pipeline(nch, issue, use);
        if (rg > 1) {  // lanes chunk + cpl g hold the same columns: a fixed xor tree
#pragma unroll 1
          for (int o = cpl; o < 32; o <<= 1)
#pragma unroll
            for (int b = 0; b < 4; ++b)
#pragma unroll
              for (int e = 0; e < 8; ++e) acc[b][e] += __shfl_xor_sync(full, acc[b][e], o);
        }
        if (active && rgrp == 0) {
#pragma unroll
          for (int b = 0; b < 4; ++b)
            if (b0 + b < BP)
#pragma unroll
              for (int e = 0; e < 8; ++e) __stcg(mine + (b0 + b) * r + 8 * chunk + e, acc[b][e]);
        }
      }
    }
    if (!p.lr_t_in) {
      __syncwarp();
      if (ok) ok = flag_barrier(p.lr_flags, G, c, epoch + 1u, lane);
      if (ok) {
        // 8 lanes per element, each adding the partials of CTAs sub, sub + 8,
        // ... in order (all loads issued first); the 8 sums then combined by a
        // fixed xor tree
        const int64_t e0 = E * c / G, e1 = E * (c + 1) / G;
        const int sub = lane % 8;
        constexpr int QL = 10;  // partials per lane in flight (two rounds cover 160 CTAs)
        for (int64_t eb = e0; eb < e1; eb += 4) {
          const int64_t e = eb + lane / 8;
          float a = 0.f;
#pragma unroll 1
          for (int q0 = 0; q0 < G; q0 += 8 * QL) {
            float v[QL];
#pragma unroll
            for (int q = 0; q < QL; ++q) {
              const int cq = q0 + sub + 8 * q;
              v[q] = (e < e1 && cq < G) ? __ldcg(p.lr_part + (int64_t)cq * E + e) : 0.f;
            }
#pragma unroll
            for (int q = 0; q < QL; ++q) a += v[q];
          }
          a += __shfl_xor_sync(full, a, 1);
          a += __shfl_xor_sync(full, a, 2);
          a += __shfl_xor_sync(full, a, 4);
          if (e < e1 && sub == 0) __stcg(p.lr_t + e, a);
        }
        ok = flag_barrier(p.lr_flags, G, c, epoch + 2u, lane);
      }
    }
    if (ok) {
      // (3) U t for rows [i0, i1); a chunk holds rc3 rows of U
      const float *tsrc = p.lr_t_in ? p.lr_t_in : p.lr_t;
      const int64_t i0 = p.n * c / G, i1 = p.n * (c + 1) / G;
      const int rc3 = kLrHalf / (2 * r);
      const int nch = (int)((i1 - i0 + rc3 - 1) / rc3);
#pragma unroll 1
      for (int b0 = 0; b0 < BP && ok; b0 += LB) {
        float tv[LB][8];
#pragma unroll
        for (int b = 0; b < LB; ++b)
#pragma unroll
          for (int e = 0; e < 8; ++e)
            tv[b][e] = active ? __ldcg(tsrc + (b0 + b) * r + 8 * chunk + e) : 0.f;
        auto issue = [&](int j, uint8_t *dst) {
          const int64_t row0 = i0 + (int64_t)j * rc3;
          const int rows = (int)min((int64_t)rc3, i1 - row0);
          if (p.ldu == r)
            copy_span(dst, p.U + row0 * p.ldu, (uint32_t)rows * r * 2);
          else
            for (int i = 0; i < rows; ++i)
              copy_span(dst + (size_t)i * r * 2, p.U + (row0 + i) * p.ldu, (uint32_t)r * 2);
        };
        auto use = [&](int j, const uint8_t *src) {
          const int64_t row0 = i0 + (int64_t)j * rc3;
          const int rows = (int)min((int64_t)rc3, i1 - row0);
          // 16-byte chunks of a row per lane: 4 to 16 (ranks 32 to 128) take
          // rows a block at a time and a butterfly over the lanes of a row
          // (ut_block); other ranks one row per lane group and a shuffle sum
          bool done = false;
          switch (cpl) {
            case 4: done = ut_block<4, LB>(src, rows, r, tv, lane, p.lr_ut + row0, p.n, b0); break;
            case 8: done = ut_block<8, LB>(src, rows, r, tv, lane, p.lr_ut + row0, p.n, b0); break;
            case 16: done = ut_block<16, LB>(src, rows, r, tv, lane, p.lr_ut + row0, p.n, b0); break;
            default: break;
          }
          if (done) return;
          for (int ib = 0; ib < rows; ib += rg) {
            const int i = ib + rgrp;
            float part[LB];
#pragma unroll
            for (int b = 0; b < LB; ++b) part[b] = 0.f;
            if (active && i < rows) {
              const uint4 u = *reinterpret_cast<const uint4 *>(src + (size_t)i * r * 2 + 16 * chunk);
              const float uf[8] = {bf16_lo(u.x), bf16_hi(u.x), bf16_lo(u.y), bf16_hi(u.y),
                                   bf16_lo(u.z), bf16_hi(u.z), bf16_lo(u.w), bf16_hi(u.w)};
#pragma unroll
              for (int b = 0; b < LB; ++b)
#pragma unroll
                for (int e = 0; e < 8; ++e) part[b] = fmaf(uf[e], tv[b][e], part[b]);
            }
            // the row's cpl lanes: a fixed xor tree, or (cpl not a power of
            // two, lanes 0 .. cpl-1) a sum in lane order
#pragma unroll
            for (int b = 0; b < LB; ++b) {
              if (rg > 1 || (cpl & (cpl - 1)) == 0) {
                for (int o = 1; o < cpl; o <<= 1) part[b] += __shfl_xor_sync(full, part[b], o);
              } else {
                float t = 0.f;
                for (int q = 0; q < cpl; ++q) t += __shfl_sync(full, part[b], q);
                part[b] = t;
              }
            }
            if (active && i < rows && chunk == 0) {
#pragma unroll
              for (int b = 0; b < LB; ++b)
                __stcg(p.lr_ut + (int64_t)(b0 + b) * p.n + row0 + i, part[b]);
            }
          }
        };
        pipeline(nch, issue, use);
      }
      __syncwarp();
      if (ok) ok = flag_barrier(p.lr_flags, G, c, epoch + 3u, lane);
      // the next call's epoch: every CTA has read this one (they all arrived)
      if (ok && c == 0 && lane == 0) st_release_u32(p.lr_epoch, epoch + 3u);
    }
    if (lane == 0) {
      if (!ok) atomicOr(p.status, kStatusTimeout);
      mbar_arrive(&lr_done);
    }
    return;
  }

  if (warp == C::NC + 1 || warp == C::NC + 2) {
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
    // (clamped to [0, G): offsets of a corrupted matrix never index slots
    // outside the workspace)
    auto owner_of_p = [&](int64_t P) -> int {
      const int64_t o = (P * G) / p.total;
      return (int)(o < 0 ? 0 : (o < G - 1 ? o : G - 1));
    };
    constexpr int OPL = 4, QMAX = 8;  // outputs per lane, contributors per load round
    const int ew = warp - (C::NC + 1);
    // the fused low-rank term must be complete before a final store adds it
    bool lr_wait = LR && p.fused_lr != 0;
    auto wait_lowrank = [&]() {
      if (!lr_wait) return;
      lr_wait = false;
      if (!mbar_wait(&lr_done, 0u) && lane == 0) atomicOr(p.status, kStatusTimeout);
    };
    const int r_first = (int)((uint32_t)t0 / (uint32_t)tpr);
    const int r_last = t1 > t0 ? (int)((uint32_t)(t1 - 1) / (uint32_t)tpr) : r_first - 1;
    for (int r = r_first + ew; r <= r_last; r += 2) {
      const int piece = r - r_first;
      const int slot = piece & 1;
      const uint32_t ph = (uint32_t)(piece >> 1) & 1u;
      const bool whole = t0 <= (int64_t)r * tpr && t1 >= (int64_t)(r + 1) * tpr;
      // owners of the band's first and last tile, fetched before the wait
      int oA = 0, oB = 0;
      if (!whole && lane == 0) {
        const int64_t ta = (int64_t)r * tpr, tb = ta + tpr - 1;
        if (p.rowmajor) {
          oA = owner_of_p(ta * 2 * B1 * B2);
          oB = owner_of_p(tb * 2 * B1 * B2);
        } else {
          oA = owner_of_p(2 * __ldg(p.val_off + ta) + __ldg(p.meta_off + ta));
          oB = owner_of_p(2 * __ldg(p.val_off + tb) + __ldg(p.meta_off + tb));
        }
      }
      if (!mbar_wait(&piece_full[slot], ph)) {
        if (lane == 0) atomicOr(p.status, kStatusTimeout);
        break;
      }
      const float(*rows)[C::RW * BP] = s_rows[slot];
      const int64_t row0 = (int64_t)r * B1;
      if (whole) {
        wait_lowrank();
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
          wait_lowrank();
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
  // scalar consumers: acc[j][b], row j RPS + rs of the warp, batch column b
  float acc[C::MMA ? 1 : C::JS][BP];
#pragma unroll
  for (int j = 0; j < (C::MMA ? 1 : C::JS); ++j)
#pragma unroll
    for (int b = 0; b < BP; ++b) acc[j][b] = 0.f;
  // tensor-core consumers: dacc[nb] is the D fragment of the warp's rows
  // 8 nb .. 8 nb + 7 (lane (g, c): batch g and g + 8, rows 2c and 2c + 1)
  constexpr int NB = C::MMA ? C::RW / 8 : 1;
  float dacc[NB][4];
#pragma unroll
  for (int nb = 0; nb < NB; ++nb)
#pragma unroll
    for (int q = 0; q < 4; ++q) dacc[nb][q] = 0.f;
  const int mg = lane >> 2, mc = lane & 3;
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
      // a lane covers columns [16cp, 16cp+16) of a sparse tile row, and
      // columns [8cp, 8cp+8) + [B2/2 + 8cp, B2/2 + 8cp + 8) of a dense tile
      // row (so that 8 lanes read 128 contiguous bytes of shared memory)
      const uint8_t *xs = st + C::kValsBytes + C::kMetaBytes + (i / C::XT) * C::kXCopy +
                          (i % C::XT) * 2 * B2;
      if constexpr (C::MMA) {
        // Columns of a 64-column block are spread over the four products of
        // the block so that every lane reads contiguous bytes: lane (g, c)
        // covers columns 16c .. 16c + 15, product j taking 16c + 4j .. 16c +
        // 4j + 3 as its k = 2c, 2c + 1, 2c + 8, 2c + 9.  A is X (batch rows
        // g and g + 8, zero past the batch), B the tile rows.
#pragma unroll
        for (int kb = 0; kb < B2 / 64; ++kb) {
          uint32_t xa[2][8];
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const int b = mg + 8 * h;
            if (b < BP) {
              const uint8_t *xp = xs + b * C::kXBatch + (kb * 64 + 16 * mc) * 2;
              const uint4 lo = *reinterpret_cast<const uint4 *>(xp);
              const uint4 hi = *reinterpret_cast<const uint4 *>(xp + 16);
              xa[h][0] = lo.x; xa[h][1] = lo.y; xa[h][2] = lo.z; xa[h][3] = lo.w;
              xa[h][4] = hi.x; xa[h][5] = hi.y; xa[h][6] = hi.z; xa[h][7] = hi.w;
            } else {
#pragma unroll
              for (int q = 0; q < 8; ++q) xa[h][q] = 0u;
            }
          }
#pragma unroll
          for (int nb = 0; nb < NB; ++nb) {
            const int row = wrow + 8 * nb + mg;
            uint32_t wv[8];
            if (sp) {
              // 8 kept values (4 groups of 4 columns) and their 4 masks
              const uint4 v = *reinterpret_cast<const uint4 *>(st + voff + row * B2 + kb * 64 +
                                                              16 * mc);
              const uint32_t m = *reinterpret_cast<const uint16_t *>(
                  st + C::kValsBytes + moff + row * (B2 / 8) + kb * 8 + 2 * mc);
              const uint32_t kv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
              for (int q = 0; q < 4; ++q) {
                const uint32_t sd = sel_dense[(m >> (4 * q)) & 0xFu];
                wv[2 * q] = __byte_perm(kv[q], 0u, sd);
                wv[2 * q + 1] = __byte_perm(kv[q], 0u, sd >> 16);
              }
            } else {
              const uint8_t *wp = st + voff + row * 2 * B2 + (kb * 64 + 16 * mc) * 2;
              const uint4 lo = *reinterpret_cast<const uint4 *>(wp);
              const uint4 hi = *reinterpret_cast<const uint4 *>(wp + 16);
              wv[0] = lo.x; wv[1] = lo.y; wv[2] = lo.z; wv[3] = lo.w;
              wv[4] = hi.x; wv[5] = hi.y; wv[6] = hi.z; wv[7] = hi.w;
            }
#pragma unroll
            for (int j = 0; j < 4; ++j)
              mma_bf16_16816(dacc[nb], xa[0][2 * j], xa[1][2 * j], xa[0][2 * j + 1],
                             xa[1][2 * j + 1], wv[2 * j], wv[2 * j + 1]);
          }
        }
      } else {
        const int xo0 = sp ? 32 * cp : 16 * cp;
        const int xo1 = sp ? 32 * cp + 16 : B2 + 16 * cp;
#pragma unroll
        for (int b0 = 0; b0 < BP; b0 += C::XB) {
          uint32_t xr[C::XB][8];
#pragma unroll
          for (int b = 0; b < C::XB; ++b) {
            const uint4 lo = *reinterpret_cast<const uint4 *>(xs + (b0 + b) * C::kXBatch + xo0);
            const uint4 hi = *reinterpret_cast<const uint4 *>(xs + (b0 + b) * C::kXBatch + xo1);
            xr[b][0] = lo.x;
            xr[b][1] = lo.y;
            xr[b][2] = lo.z;
            xr[b][3] = lo.w;
            xr[b][4] = hi.x;
            xr[b][5] = hi.y;
            xr[b][6] = hi.z;
            xr[b][7] = hi.w;
          }
          if (sp) {
#pragma unroll
            for (int j = 0; j < C::JS; ++j) {
              const int row = wrow + j * C::RPS + rs;
              const uint4 v = *reinterpret_cast<const uint4 *>(st + voff + row * B2 + 16 * cp);
              const uint32_t m = *reinterpret_cast<const uint16_t *>(
                  st + C::kValsBytes + moff + row * (B2 / 8) + 2 * cp);
              const uint32_t w[4] = {v.x, v.y, v.z, v.w};
              if constexpr (PAT == 1) {
                // 4:8: two groups of 8 columns, 4 kept each (c0 < c1 < c2 <
                // c3); (v0, v1) meet x[c0], x[c1] and (v2, v3) x[c2], x[c3].
                // As c0 <= 4, c1 <= 5, c2 >= 2 and c3 >= 3, each x pair comes
                // from three of the group's four x registers in two PRMTs,
                // with selectors from the mask byte's lut48 entry.
#pragma unroll
                for (int gb = 0; gb < 2; ++gb) {
                  const uint2 sl = lut48[(m >> (8 * gb)) & 0xFFu];
                  const uint32_t s1 = sl.x, s2 = sl.x >> 16, s3 = sl.y, s4 = sl.y >> 16;
#pragma unroll
                  for (int b = 0; b < C::XB; ++b) {
                    const uint32_t *X4 = &xr[b][4 * gb];
                    const uint32_t pa = __byte_perm(__byte_perm(X4[0], X4[1], s1), X4[2], s2);
                    const uint32_t pb = __byte_perm(X4[1], __byte_perm(X4[2], X4[3], s3), s4);
                    fma_bf16x2(acc[j][b0 + b], w[2 * gb], pa);
                    fma_bf16x2(acc[j][b0 + b], w[2 * gb + 1], pb);
                  }
                }
              } else {
                // 2:4: the PRMT selector of each group moves x[p0] to the low
                // and x[p1] to the high half (p0 < p1 the kept columns).
                // Narrow batches, where a selector serves one to four products,
                // build it in registers: one PRMT looks up (p0, p1) of two
                // groups at once in a byte table indexed by the low three bits
                // of each 4-bit mask (distinct for the six masks with two bits
                // set), a second PRMT expands them to byte pairs.  Wide batches
                // take it from a 16-entry shared table (one load serves eight or
                // sixteen products).
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
      }
      voff += sp ? B1 * B2 : 2 * B1 * B2;
      moff += sp ? B1 * B2 / 8 : 0;
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty_bar[stage]);
    if (++stage == p.nst) {
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
    if constexpr (C::MMA) {
#pragma unroll
      for (int nb = 0; nb < NB; ++nb) {
        const int r0 = 8 * nb + 2 * mc;
        if (mg < BP) {
          rows_s[mg * C::RW + r0] = dacc[nb][0];
          rows_s[mg * C::RW + r0 + 1] = dacc[nb][1];
        }
        if (mg + 8 < BP) {
          rows_s[(mg + 8) * C::RW + r0] = dacc[nb][2];
          rows_s[(mg + 8) * C::RW + r0 + 1] = dacc[nb][3];
        }
#pragma unroll
        for (int q = 0; q < 4; ++q) dacc[nb][q] = 0.f;
      }
    } else {
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
  const uint32_t starts = nw > 0 ? stage_starts(bits, nw, (uint32_t)(t0 % tpr), tpr, tpd, 2 * tpd) : 0u;
  int64_t *rec = plan + kPlanHead + 4 * (int64_t)c;
  rec[0] = t0;
  rec[1] = val_off[t0];
  rec[2] = meta_off[t0];
  rec[3] = (int64_t)(((uint64_t)starts << 32) | bits);
}

// ---------------------------------------------------------------------------
// simple kernel for other legal tilings: one warp per output row.  A lane
// takes 8-column chunks of the row (b2 is a multiple of 8): 16 bytes of a
// dense tile row, or 4 kept values (8 bytes) and one mask byte (two groups)
// of a 2:4 tile row, with the chunk's 8 x values.
// ---------------------------------------------------------------------------
template <int BP, bool STRIDED>
__global__ void __launch_bounds__(kThreads)
    hybrid_rowwarp_kernel(const Params p, int b1, int b2) {
  const int lane = threadIdx.x & 31;
  const int64_t warps = (int64_t)gridDim.x * kWarps;
  const int cpr = b2 / 8;  // 8-column chunks per tile row
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
      uint32_t xr[BP][4];
#pragma unroll
      for (int b = 0; b < BP; ++b) {
        if (b < p.batch) {
          const uint4 xv = ld_keep16(p.X + (int64_t)b * p.ldx + tc * b2 + 8 * cpart);
          xr[b][0] = xv.x;
          xr[b][1] = xv.y;
          xr[b][2] = xv.z;
          xr[b][3] = xv.w;
        } else {
#pragma unroll
          for (int e = 0; e < 4; ++e) xr[b][e] = 0u;
        }
      }
      const bool sparse = !STRIDED && __ldg(p.map + t) == 1;
      if (sparse) {
        // groups 2 cpart and 2 cpart + 1 of the row: kept values 4 cpart ..
        // 4 cpart + 3, mask byte cpart
        const uint8_t *vp = p.vals + 2 * __ldg(p.val_off + t) + i * b2 + 8 * cpart;
        const uint8_t *mp = p.meta + __ldg(p.meta_off + t) + i * (b2 / 8) + cpart;
        const uint2 v = ld_stream8(vp);
        const uint32_t m = ld_stream_u8(mp);
        const uint32_t w[2] = {v.x, v.y};
#pragma unroll
        for (int g = 0; g < 2; ++g) {
          const uint32_t nib = (m >> (4 * g)) & 0xFu;
#pragma unroll
          for (int b = 0; b < BP; ++b) {
            float xa, xb;
            pick2(nib, bf16_lo(xr[b][2 * g]), bf16_hi(xr[b][2 * g]), bf16_lo(xr[b][2 * g + 1]),
                  bf16_hi(xr[b][2 * g + 1]), xa, xb);
            acc[b] = fmaf(bf16_lo(w[g]), xa, acc[b]);
            acc[b] = fmaf(bf16_hi(w[g]), xb, acc[b]);
          }
        }
      } else {
        const uint8_t *vp =
            STRIDED ? reinterpret_cast<const uint8_t *>(p.Wd + row * p.ldw + tc * b2 + 8 * cpart)
                    : p.vals + 2 * __ldg(p.val_off + t) + i * 2 * b2 + 16 * cpart;
        const uint4 wv = ld_stream16(vp);
        const uint32_t w[4] = {wv.x, wv.y, wv.z, wv.w};
#pragma unroll
        for (int e = 0; e < 4; ++e)
#pragma unroll
          for (int b = 0; b < BP; ++b) {
            acc[b] = fmaf(bf16_lo(w[e]), bf16_lo(xr[b][e]), acc[b]);
            acc[b] = fmaf(bf16_hi(w[e]), bf16_hi(xr[b][e]), acc[b]);
          }
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

struct TmaKernel {
  void *fn;
  int threads;
  size_t smem;       // dynamic shared memory with every stage of the ring
  int stage_bytes;
  int stages;        // the ring's compile-time stage count
  int tps;
  bool xtm;    // X slices by 2-D tensor copies (box xcols x bp)
  int xcols;
  int bp;
};

template <int BP, int B1, int B2, int PAT, bool LR = false>
TmaKernel tma_kernel_info() {
  using C = TmaCfg<BP, B1, B2, LR, PAT>;
  return TmaKernel{reinterpret_cast<void *>(&hybrid_tma_kernel<BP, B1, B2, PAT, LR>), C::kThreads,
                   C::kSmem, C::kStageBytes, C::kStages, C::TPX, C::XTM, C::XT * B2, BP};
}

bool pick_tma_kernel(int bp, Shape s, int pat, bool lr, TmaKernel *out) {
#define HYB_TCASE(BP_, PAT_, LR_)                                                            \
  case BP_:                                                                                  \
    switch (s) {                                                                             \
      case kS128x128: *out = tma_kernel_info<BP_, 128, 128, PAT_, LR_>(); return true;       \
      case kS128x64: *out = tma_kernel_info<BP_, 128, 64, PAT_, LR_>(); return true;         \
      case kS64x64: *out = tma_kernel_info<BP_, 64, 64, PAT_, LR_>(); return true;           \
      case kS64x128: *out = tma_kernel_info<BP_, 64, 128, PAT_, LR_>(); return true;         \
      default: return false;                                                                 \
    }
#define HYB_TSET(PAT_, LR_)  \
  switch (bp) {              \
    HYB_TCASE(1, PAT_, LR_)  \
    HYB_TCASE(2, PAT_, LR_)  \
    HYB_TCASE(4, PAT_, LR_)  \
    HYB_TCASE(8, PAT_, LR_)  \
    HYB_TCASE(16, PAT_, LR_) \
    default: return false;   \
  }
  // the low-rank term exists for 2:4 tiles only (the N:M entry point has none)
  if (pat == 1) {
    if (lr) return false;
    HYB_TSET(1, false)
  }
  if (lr) {
    switch (bp) {  // (only narrow batches fuse the low-rank term)
      HYB_TCASE(1, 0, true)
      HYB_TCASE(2, 0, true)
      HYB_TCASE(4, 0, true)
      default: return false;
    }
  }
  HYB_TSET(0, false)
#undef HYB_TSET
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

// Static shared memory of a kernel instance and the dynamic shared memory it
// may be launched with (the device's opt-in maximum less the static part);
// the first query for an instance also raises its dynamic limit to that
// maximum.  Cached per instance and device.
int kernel_smem_limits(void *fn, size_t *static_bytes, size_t *max_dynamic) {
  static std::mutex mu;
  struct Entry {
    void *fn;
    int dev;
    size_t stat, dyn;
  };
  static Entry cache[256];
  static int used = 0;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return HYB_ERR_CUDA;
  std::lock_guard<std::mutex> lock(mu);
  for (int i = 0; i < used; ++i)
    if (cache[i].fn == fn && cache[i].dev == dev) {
      *static_bytes = cache[i].stat;
      *max_dynamic = cache[i].dyn;
      return HYB_OK;
    }
  cudaFuncAttributes attr{};
  int optin = 0;
  if (cudaFuncGetAttributes(&attr, fn) != cudaSuccess ||
      cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) != cudaSuccess)
    return HYB_ERR_CUDA;
  if ((size_t)optin <= attr.sharedSizeBytes) return HYB_ERR_UNSUPPORTED;
  const size_t dyn = (size_t)optin - attr.sharedSizeBytes;
  if (cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)dyn) !=
      cudaSuccess)
    return HYB_ERR_CUDA;
  if (used < 256) cache[used++] = Entry{fn, dev, attr.sharedSizeBytes, dyn};
  *static_bytes = attr.sharedSizeBytes;
  *max_dynamic = dyn;
  return HYB_OK;
}

// Resident CTAs per SM of a kernel instance with this much dynamic shared
// memory (cached; the answer only depends on the instance, the size and the
// device).
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
  size_t stat = 0, maxdyn = 0;
  if (kernel_smem_limits(fn, &stat, &maxdyn) != HYB_OK || dyn_smem > maxdyn) return -1;
  std::lock_guard<std::mutex> lock(mu);
  for (int i = 0; i < used; ++i)
    if (cache[i].fn == fn && cache[i].dev == dev && cache[i].smem == dyn_smem)
      return cache[i].blocks;
  int nb = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&nb, fn, threads, dyn_smem) != cudaSuccess)
    return -1;
  if (used < 256) cache[used++] = Entry{fn, dev, dyn_smem, nb};
  return nb;
}

// Work split and workspace layout of one product call.
struct Plan {
  bool tma;        // TMA-ring kernel (tuned tile shapes, packed or row-major)
  bool fused;      // a low-rank term computed inside the streaming kernel
  TmaKernel tk;
  int bp;          // padded batch
  int b1, b2;
  int G;           // CTAs of the stream split
  int nst;         // ring stages of the launch
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
              int batch, int rank, bool strided, Plan *pl, int pat = 0) {
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
  (void)strided;  // packed and row-major matrices take the same kernels
  // (tile indices are 32-bit in the streaming kernel's band arithmetic)
  P.tma = s != kGeneric && (n / b1) * (k / b2) < (int64_t(1) << 31);
  // A low-rank term rides in the streaming kernel for narrow batches, where
  // it is a few percent more bytes and little arithmetic; for batch 8 and 16
  // its arithmetic (2 batch r (n + k) flops) is better spread over the whole
  // GPU by the separate kernels than left to one warp of each CTA.
  P.fused = P.tma && rank > 0 && P.bp <= 4;
  if (P.tma) {
    P.G = tma_ctas(sms, total_bytes, b1, b2);
    if (!pick_tma_kernel(P.bp, s, pat, P.fused, &P.tk)) return HYB_ERR_UNSUPPORTED;
    // a low-rank term adds the low-rank warp's chunk buffer after the ring,
    // and the ring gives up stages if both do not fit
    size_t stat = 0, maxdyn = 0;
    rc = kernel_smem_limits(P.tk.fn, &stat, &maxdyn);
    if (rc != HYB_OK) return rc;
    const size_t extra = P.tk.smem - (size_t)P.tk.stages * P.tk.stage_bytes;  // alignment slack
    const size_t lrb = P.fused ? (size_t)kLrBufBytes : 0;
    const int fit = maxdyn > extra + lrb ? (int)((maxdyn - extra - lrb) / P.tk.stage_bytes) : 0;
    P.nst = std::min(P.tk.stages, fit);
    if (P.nst < 3) return HYB_ERR_UNSUPPORTED;
    P.dyn_smem = (size_t)P.nst * P.tk.stage_bytes + extra + lrb;
    const int nb = blocks_per_sm(P.tk.fn, P.dyn_smem, P.tk.threads);
    if (nb <= 0) return HYB_ERR_CUDA;
  } else {
    P.G = 0;
    P.nst = 0;
    P.dyn_smem = 0;
  }
  // partials of t: one per CTA of the streaming kernel (fused), else one per
  // CTA of the separate V^T x kernel
  P.lr_ctas = rank <= 0 ? 0
              : P.fused  ? P.G
                         : (int)std::max<int64_t>(1, std::min<int64_t>(sms, k / 64));
  size_t off = kTicketsOffset;
  P.off_counters = off;
  if (P.tma) off = align_up(off + (size_t)P.R * (b1 / 8) * sizeof(uint32_t), 256);
  P.off_lr_t = off;
  off = align_up(off + (size_t)P.bp * (rank > 0 ? rank : 0) * sizeof(float), 256);
  P.off_lr_part = off;
  off = align_up(off + (size_t)P.lr_ctas * P.bp * (rank > 0 ? rank : 0) * sizeof(float), 256);
  // ticket of the V^T x kernel (the fused term's epoch and flags have their
  // own fixed places)
  P.off_lr_counter = kLowrankTicketOffset;
  P.off_lr_ut = off;
  off = align_up(off + (size_t)P.bp * (rank > 0 ? n : 0) * sizeof(float), 256);
  P.off_partials = off;
  if (P.tma) off += (size_t)(P.G + P.R) * b1 * P.bp * sizeof(float);
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
// rows past the batch and columns past k read as zeros.
int encode_x_map(const uint16_t *X, int64_t k, int batch, int64_t ldx, int xcols, int bp,
                 CUtensorMap *map) {
  PFN_cuTensorMapEncodeTiled_v12000 encode = tensor_map_encoder();
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

// Tensor map of a row-major bf16 W ([n][k], row stride ldw) with box
// [b1 rows][b2 columns]: one box is one dense tile, in the packed dense
// tile layout.
int encode_w_map(const uint16_t *W, int64_t n, int64_t k, int64_t ldw, int b1, int b2,
                 CUtensorMap *map) {
  PFN_cuTensorMapEncodeTiled_v12000 encode = tensor_map_encoder();
  if (!encode) return HYB_ERR_CUDA;
  const cuuint64_t dims[2] = {(cuuint64_t)k, (cuuint64_t)n};
  const cuuint64_t strides[1] = {(cuuint64_t)ldw * 2};
  const cuuint32_t box[2] = {(cuuint32_t)b2, (cuuint32_t)b1};
  const cuuint32_t estr[2] = {1, 1};
  const CUresult r = encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<uint16_t *>(W),
                            dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                            CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
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
                const int64_t *plan = nullptr, int32_t plan_ctas = 0, uint32_t flags = 0,
                int pat = 0, const float *t_in = nullptr, const float **t_out = nullptr) {
  const int rank = (lr && lr->rank > 0) ? lr->rank : 0;
  Plan P;
  int rc = make_plan(prm.n, prm.k, b1, b2, prm.total, batch, rank, strided, &P, pat);
  if (rc != HYB_OK) return rc;
  if (!ws || ws_bytes < P.bytes) return HYB_ERR_WORKSPACE;
  if ((uintptr_t)ws % 256 != 0) return HYB_ERR_ALIGNMENT;
  uint8_t *w = reinterpret_cast<uint8_t *>(ws);
  prm.R = P.R;
  prm.G = P.G;
  prm.nst = P.nst;
  prm.partials = reinterpret_cast<float *>(w + P.off_partials);
  prm.counters = reinterpret_cast<uint32_t *>(w + P.off_counters);
  prm.rank = rank;
  prm.U = rank ? lr->U : nullptr;
  prm.ldu = rank ? lr->ldu : 0;
  prm.V = rank ? lr->V : nullptr;
  prm.ldv = rank ? lr->ldv : 0;
  prm.lr_t = reinterpret_cast<float *>(w + P.off_lr_t);
  prm.lr_part = reinterpret_cast<float *>(w + P.off_lr_part);
  prm.lr_epoch = reinterpret_cast<uint32_t *>(w + kLowrankEpochOffset);
  prm.lr_flags = reinterpret_cast<uint32_t *>(w + kLowrankFlagsOffset);
  prm.lr_t_in = rank ? t_in : nullptr;
  if (t_out) *t_out = rank && !t_in ? prm.lr_t : nullptr;
  prm.lr_ut = nullptr;
  prm.fused_lr = 0;
  const bool overlap = (flags & HYB_LAUNCH_OVERLAP_PREV) != 0;
  if (rank && P.fused) {
    // the streaming kernel's low-rank warp computes V^T x and U t itself
    prm.fused_lr = 1;
    prm.lr_ut = reinterpret_cast<float *>(w + P.off_lr_ut);
  } else if (rank) {
    // wide batches and other tilings: V^T x, then U t, then the product,
    // launched one after the other (the first as a programmatic dependent
    // with the caller's overlap flag; the one-warp-per-row product ignores
    // the flag)
    if (!t_in) {
      rc = launch_lowrank_t(P, lr, prm.k, prm.X, prm.ldx, batch, w, s, overlap);
      if (rc != HYB_OK) return rc;
    }
    int64_t nn = prm.n, ldu = lr->ldu;
    const uint16_t *U = lr->U;
    int rk = rank, bt = batch;
    const float *tp = t_in ? t_in : prm.lr_t;
    float *ut = reinterpret_cast<float *>(w + P.off_lr_ut);
    int zero = 0;
    void *uargs[] = {&nn, &U, &ldu, &rk, &tp, &bt, &ut, &zero};
    const int64_t grid = (prm.n + kThreads - 1) / kThreads;
    if (cudaLaunchKernel(pick_lowrank_ut(P.bp), dim3((unsigned)grid), dim3(kThreads), uargs, 0,
                         s) != cudaSuccess)
      return HYB_ERR_CUDA;
    prm.lr_ut = ut;
  }
  prm.status = reinterpret_cast<uint32_t *>(w);
  const bool pdl = overlap && P.tma;
  prm.pdl = pdl ? 1 : 0;
  prm.rowmajor = strided ? 1 : 0;
  if (P.tma) {
    LaunchPlan lp;
    fill_launch_plan(strided ? nullptr : plan, plan_ctas, P, prm, &lp);
    alignas(64) CUtensorMap xmap{};
    alignas(64) CUtensorMap wmap{};
    if (P.tk.xtm) {
      rc = encode_x_map(prm.X, prm.k, batch, prm.ldx, P.tk.xcols, P.tk.bp, &xmap);
      if (rc != HYB_OK) return rc;
    }
    if (strided) {
      rc = encode_w_map(prm.Wd, prm.n, prm.k, prm.ldw, b1, b2, &wmap);
      if (rc != HYB_OK) return rc;
    }
    void *targs[] = {&prm, &lp, &xmap, &wmap};
    if (launch_kernel(P.tk.fn, dim3(P.G), dim3(P.tk.threads), targs, P.dyn_smem, s, pdl) !=
        cudaSuccess)
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
              void *ws, size_t ws_bytes, cudaStream_t s, uint32_t flags = 0, int pat = 0,
              const float *t_in = nullptr, const float **t_out = nullptr) {
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
                     A->plan_ctas, flags, pat, t_in, t_out);
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
  *off_counter = kLowrankTicketOffset;  // in the header, the same place for every call
  return off;
}

}  // namespace

// The streaming product of a matrix packed by hyb_pack_nm with nk = 2 of
// m = 4 (hyb_pack's layout) or nk = 4 of m = 8: both keep half of a sparse
// tile's values with b1 * b2 / 8 mask bytes, so the split, the plan and the
// stage packing are the 2:4 ones; only the mask decode differs.  Returns
// HYB_ERR_UNSUPPORTED when the tiling has no streaming kernel.
int stream_product_nm(const hyb_matrix *A, int nk, int m, int batch, const uint16_t *X,
                      int64_t ldx, void *Y, int64_t ldy, hyb_dtype ydt, void *ws,
                      size_t ws_bytes, cudaStream_t s) {
  if (shape_of(A->b1, A->b2) == kGeneric) return HYB_ERR_UNSUPPORTED;
  int pat;
  if (nk == 2 && m == 4) pat = 0;
  else if (nk == 4 && m == 8) pat = 1;
  else return HYB_ERR_UNSUPPORTED;
  return spmm_impl(A, batch, X, ldx, Y, ldy, ydt, nullptr, ws, ws_bytes, s, 0, pat);
}

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

size_t hyb_gate_up_workspace_bytes(const hyb_matrix *Ag, const hyb_matrix *Au, int batch,
                                   int rank) {
  if (rank < 1) return 0;
  const size_t a = hyb_workspace_bytes(Ag, batch, rank);
  const size_t b = hyb_workspace_bytes(Au, batch, rank);
  if (a == 0 || b == 0) return 0;
  return (a + 255) / 256 * 256 + b;
}

int hyb_spmm_skinny_gate_up(const hyb_matrix *Ag, const hyb_matrix *Au, int batch,
                            const uint16_t *X, int64_t ldx, void *Yg, int64_t ldyg, void *Yu,
                            int64_t ldyu, hyb_dtype ydt, const hyb_lowrank *lr_g,
                            const uint16_t *Uu, int64_t lduu, uint32_t flags, void *ws,
                            size_t ws_bytes, hyb_stream_t stream) {
  if (!Ag || !Au || !lr_g || lr_g->rank < 1 || !Uu) return HYB_ERR_INVALID_ARG;
  if (Ag->k != Au->k) return HYB_ERR_INVALID_ARG;  // one input x for both
  const hyb_lowrank lr_u{lr_g->rank, Uu, lduu, lr_g->V, lr_g->ldv};
  int rc = check_lowrank(&lr_u, Au->n, Au->k);
  if (rc != HYB_OK) return rc;
  const size_t need = hyb_gate_up_workspace_bytes(Ag, Au, batch, lr_g->rank);
  if (need == 0) return HYB_ERR_INVALID_ARG;
  if (!ws || ws_bytes < need) return HYB_ERR_WORKSPACE;
  const size_t wa = (hyb_workspace_bytes(Ag, batch, lr_g->rank) + 255) / 256 * 256;
  uint8_t *w = static_cast<uint8_t *>(ws);
  cudaStream_t s = (cudaStream_t)stream;
  // gate: the full product, which leaves t = V^T x in its workspace
  const float *t = nullptr;
  rc = hyb::spmm_impl(Ag, batch, X, ldx, Yg, ldyg, ydt, lr_g, w, wa, s, flags, 0, nullptr, &t);
  if (rc != HYB_OK) return rc;
  if (!t) return HYB_ERR_CUDA;
  // up: the same t, only U_up t (launched after the gate product on the
  // stream; as a programmatic dependent when the caller asked for overlap)
  return hyb::spmm_impl(Au, batch, X, ldx, Yu, ldyu, ydt, &lr_u, w + wa, ws_bytes - wa, s,
                        flags, 0, t, nullptr);
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
  // the streaming kernel reads W by tensor copies (16-byte aligned start and
  // row stride), the row-per-warp one in 16-byte pieces
  if ((uintptr_t)W % 16 != 0 || ldw % 8 != 0) return HYB_ERR_ALIGNMENT;
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
