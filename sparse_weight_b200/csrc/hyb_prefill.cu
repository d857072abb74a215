// hyb_spmm_prefill: a hybrid (dense | 2:4) weight times a tall block of
// activations on the 5th-generation tensor cores,
//
//     Y[m][i] = sum_k W_hat[i][k] X[m][k]     (m < M tokens, i < n rows)
//
// the prefill / large-batch form of the product.  PATCH ("PATCH: Learnable
// Tile-level Hybrid Sparsity for LLMs", §2 Method) runs its dense tiles on
// dense tensor-core kernels and its 2:4 tiles on the sparse tensor cores; here
// both kinds of tile feed one tcgen05 pipeline, dense tiles through
// tcgen05.mma and 2:4 tiles through tcgen05.mma.sp:
//
//   * A CTA owns NB 128-row bands (1 or 2) and PN tokens (128 or 256 for one
//     band, 240 or 208 for two): one 128 x PN fp32 accumulator per band in tensor
//     memory (TMEM, band b from column 256 b), M = 128 weight rows per MMA,
//     N = PN tokens, K looped over the bands' tiles (128 columns each, in two
//     halves of 64).  hyb_prefill_block_shape picks the shape per call.
//   * warp 0 moves the operands with TMA into a ring of 192 KB: 3 slots of a
//     whole tile (one band, 128 tokens), else slots of a half-tile (4 x 48 KB
//     for one band and 256 tokens, 3 x 62 KB for two bands): a dense tile's
//     half as a 2-D box of 64 columns x 128 rows with the 128-byte swizzle
//     (the K-major layout tcgen05.mma reads), a 2:4 tile's kept values (already
//     the sparse MMA's compressed A operand: 2 kept values per group of 4,
//     ascending) as a box of 64 values x 128 rows, or of 32 values x 128 rows
//     in the 64-byte swizzle per half in the half-tile rings, X as a box of 64
//     columns x PN tokens per half.  Its lanes load a window of 32 tiles'
//     value offsets into shared memory; lane 0 alone walks the tiles.
//   * warps 4-11 turn each 2:4 tile's masks into the sparse MMA's metadata
//     (the two kept positions of a group as a nibble, laid out by tensor-
//     memory lane and column), fence it for the async proxy and signal the
//     MMA warp.
//   * warp 1 owns the TMEM allocation; its lane 0 issues per band and half-tile
//     4 tcgen05.mma (dense: kind::f16, bf16 x bf16 -> fp32, K = 16 each) or,
//     for a 2:4 tile, a tcgen05.cp of the metadata and 2 tcgen05.mma.sp (K =
//     32 each) per half, and frees each ring slot with tcgen05.commit.
//   * warps 4-11 then read the accumulators with tcgen05.ld (warp w: TMEM
//     lanes 32 (w % 4) .., half of the token columns of one band, or every
//     column of band w / 8 - 1) and store Y (a warp writes 32 consecutive
//     rows of one token: 128 contiguous bytes).
//
// A CTA's operand bytes per tile are its bands' A (16 KB per band and half)
// and PN x 256 bytes of X, against NB x PN x 128 x 128 multiply-adds: the
// two-band shape moves the fewest bytes per product, one band x 128 tokens
// the most; the choice weighs that against the number of CTA waves.  A 2:4
// tile moves the hybrid format's bytes and costs half a dense tile's tensor
// work.  Every wait is bounded; one that runs out sets kStatusTimeout in the
// status word and the CTA leaves its pipeline.
#include "hyb_internal.cuh"

namespace hyb {
namespace {

constexpr int kPM = 128;                      // weight rows per CTA (b1), MMA M
constexpr int kPK = 128;                      // columns per tile (b2)
constexpr int kAtomBytes = 128 * 128;         // 128 rows x 128 bytes (64 bf16), swizzled
constexpr int kSValBytes = kPM * kPK;         // a 2:4 tile's kept values (bf16)
constexpr int kSMetaBytes = kPM * kPK / 8;    // and masks
constexpr int kEBytes = kPM * kPK / 8;      // a 2:4 tile's sparse-MMA metadata, 2 KB
constexpr int kRingBytes = 192 * 1024;        // the half-tile ring
constexpr int kESlots = 8;                      // metadata ring: 2:4 tiles converted ahead
constexpr int kMaxSlots = 4;
constexpr int kPThreads = 384;  // warp 0 TMA, warp 1 MMA + TMEM, warps 4-11 expand + epilogue
constexpr int kExpThreads = 256;  // two per tile row (columns 0-63, 64-127)
constexpr int kMaxBandTiles = 1024;           // tiles per band (k <= 131072)
static_assert(kSValBytes == kAtomBytes, "a 2:4 tile's kept values fill one swizzle box");

// The shape of one CTA's pipeline: NB row bands of 128 rows (1 or 2) and PN
// tokens.  A ring slot holds HS half-tiles (64 columns each), a half-tile
// being the bands' A halves (16 KB each) and then X's (PN x 128 bytes): a
// whole tile per slot for one band and 128 tokens (3 slots of 64 KB), a half
// per slot otherwise (4 slots of 48 KB for one band and 256 tokens, 3 slots of
// 62 or 58 KB for two bands and 240 or 208 tokens).  TMEM holds the bands' PN-column fp32
// accumulators (band b from column 256 b), then 4 metadata columns per
// metadata slot (8 slots for one band, 4 in the last 16 columns for two).
template <int PN, int NB>
struct PrefillShape {
  static constexpr int HS = (NB == 1 && PN == 128) ? 2 : 1;  // half-tiles per ring slot
  static constexpr int kXHalfBytes = PN * 128;
  static constexpr int kHalfBytes = NB * kAtomBytes + kXHalfBytes;
  static constexpr int kSlotBytes = HS * kHalfBytes;
  static constexpr int kSlots = kRingBytes / kSlotBytes;
  static constexpr int kAccStride = 256;                         // band b's accumulator: column 256 b
  static constexpr int kEsl = NB == 1 ? kESlots : 4;             // metadata slots in use
  static constexpr int kTmemE = NB == 1 ? PN : 512 - 4 * kEsl;  // first metadata column
  static constexpr int kTmemCols = kTmemE + 4 * kEsl <= 256 ? 256 : 512;
  static_assert(NB == 1 || NB == 2, "one or two bands per CTA");
  static_assert(PN % 16 == 0 && PN >= 16 && PN <= 256, "MMA N: a multiple of 16 up to 256");
  static_assert(kSlots >= 3 && kSlots <= kMaxSlots, "ring depth");
  static_assert(kHalfBytes % 1024 == 0, "slots keep the 1024-byte swizzle alignment");
  static_assert((NB - 1) * kAccStride + PN <= kTmemE, "accumulators before the metadata");
  static_assert(kTmemE + 4 * kEsl <= kTmemCols && kTmemCols <= 512, "TMEM columns");
};

// tcgen05.mma instruction descriptor: D fp32, A and B bf16, both K-major,
// N tokens, M = kPM (bit layout of the sm_100 instruction descriptor); the
// sparse form adds bit 2 and selects its metadata half with bits 0-1.
template <int PN>
__host__ __device__ constexpr uint32_t idesc_f16() {
  return (1u << 4)                         // D format: f32
         | (1u << 7)                       // A format: bf16
         | (1u << 10)                      // B format: bf16
         | ((uint32_t)(PN >> 3) << 17)     // N / 8
         | ((uint32_t)(kPM >> 4) << 24);   // M / 16
}

// Shared-memory matrix descriptor of the metadata for tcgen05.cp (128 rows of
// 16 bytes, no swizzle: 8-row core matrices of 128 contiguous bytes, 128
// bytes apart).
__device__ __forceinline__ uint64_t e_desc(uint32_t saddr) {
  uint64_t d = (uint64_t)((saddr >> 4) & 0x3FFFu);
  d |= (uint64_t)(128 >> 4) << 16;    // leading byte offset (one 16-byte column: unused)
  d |= (uint64_t)(128 >> 4) << 32;    // stride byte offset: next 8 rows
  d |= (uint64_t)1 << 46;             // version; layout type 0 (no swizzle)
  return d;
}

// Shared-memory matrix descriptor of a K-major operand in the 128-byte
// swizzle layout: rows 128 bytes apart, 8-row groups 1024 bytes apart
// (stride byte offset), descriptor version 1, layout type 2 (128B swizzle).
__device__ __forceinline__ uint64_t sw128_desc(uint32_t saddr) {
  uint64_t d = (uint64_t)((saddr >> 4) & 0x3FFFu);
  d |= (uint64_t)1 << 16;             // leading byte offset (unused by swizzled K-major)
  d |= (uint64_t)(1024 >> 4) << 32;   // stride byte offset
  d |= (uint64_t)1 << 46;             // version
  d |= (uint64_t)2 << 61;             // 128-byte swizzle
  return d;
}

// The same for the 64-byte swizzle layout: rows 64 bytes apart, 8-row groups
// 512 bytes apart, layout type 4 (a 2:4 tile's half: 32 kept values per row).
__device__ __forceinline__ uint64_t sw64_desc(uint32_t saddr) {
  uint64_t d = (uint64_t)((saddr >> 4) & 0x3FFFu);
  d |= (uint64_t)1 << 16;             // leading byte offset (unused by swizzled K-major)
  d |= (uint64_t)(512 >> 4) << 32;    // stride byte offset
  d |= (uint64_t)1 << 46;             // version
  d |= (uint64_t)4 << 61;             // 64-byte swizzle
  return d;
}

__device__ __forceinline__ void umma_bf16(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc,
                                          uint32_t accumulate, uint32_t idesc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %3, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %4, p;\n\t}" ::"r"(tmem_d),
      "l"(adesc), "l"(bdesc), "r"(accumulate), "r"(idesc)
      : "memory");
}
// D += A (2:4 compressed, K = 32 per instruction, 16 stored) x B, metadata
// from tensor memory column `tmem_e` (even) and half `id2`
__device__ __forceinline__ void umma_sp_bf16(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc,
                                             uint32_t tmem_e, uint32_t id2,
                                             uint32_t accumulate, uint32_t idesc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.sp.cta_group::1.kind::f16 [%0], %1, %2, [%3], %5, p;\n\t}" ::"r"(tmem_d),
      "l"(adesc), "l"(bdesc), "r"(tmem_e), "r"(accumulate), "r"(idesc | (1u << 2) | id2)
      : "memory");
}
// copy 128 lanes x 16 bytes of metadata from shared to tensor memory
__device__ __forceinline__ void tmem_cp_128x128b(uint32_t taddr, uint64_t sdesc) {
  asm volatile("tcgen05.cp.cta_group::1.128x128b [%0], %1;" ::"r"(taddr), "l"(sdesc) : "memory");
}
// arrives on the mbarrier once every tcgen05.mma this thread issued before
// has completed
__device__ __forceinline__ void umma_commit(uint64_t *bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::
                   "r"(smem_u32(bar))
               : "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
// 16 consecutive fp32 columns of this thread's TMEM lane
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float (&v)[16]) {
  uint32_t r[16];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
      "%11, %12, %13, %14, %15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int q = 0; q < 16; ++q) v[q] = __uint_as_float(r[q]);
}

// Waits for the mbarrier phase of the given parity.  The thread sleeps in
// mbarrier.try_wait with an explicit suspend-time hint: in this pipeline a
// blocked try_wait without one woke up late enough to cost most of a
// microsecond per ring slot.  Gives up (returns false) after about 2^31 SM
// clocks, so a phase that never completes ends the CTA's pipeline.
__device__ __forceinline__ bool ring_wait(uint64_t *bar, uint32_t parity) {
  const long long t0 = clock64();
  do {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity), "r"(200000u)  // hint: 200 us
        : "memory");
    if (ok) return true;
  } while (clock64() - t0 < (1ll << 31));
  return false;
}

struct PrefillParams {
  const uint8_t *map;
  const uint16_t *vals;
  const uint8_t *meta;
  const int64_t *val_off;
  const int64_t *meta_off;
  int64_t n, k, m;
  int tpr;
  int bands;         // n / 128
  int64_t nvb, nmb;  // bytes of the value and mask buffers
  float *Y;
  int64_t ldy;
  uint32_t *status;
};

constexpr uint32_t kNoMeta = 0xFFFFFFFFu;  // a mask offset that cannot be used

template <int PN, int NB>
__global__ void __launch_bounds__(kPThreads, 1)
    hybrid_prefill_kernel(const PrefillParams p, const __grid_constant__ CUtensorMap xmap,
                          const __grid_constant__ CUtensorMap wmap,
                          const __grid_constant__ CUtensorMap spmap) {
  using Sh = PrefillShape<PN, NB>;
  constexpr int NS = Sh::kSlots, HS = Sh::HS;
  constexpr uint32_t kIdesc = idesc_f16<PN>();
  extern __shared__ uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t full_bar[kMaxSlots];
  __shared__ __align__(8) uint64_t empty_bar[kMaxSlots];
  // the metadata ring: slot q holds the metadata of every kEsl-th 2:4 tile
  // of the CTA, taken in (tile, band) order (efull: written; eempty: the MMAs
  // that read it completed).  The converting warps and the MMA warp take the
  // 2:4 tiles in the same order, and each waits for the other's previous use
  // of the slot, so neither barrier runs two phases ahead of a waiting thread.
  __shared__ __align__(8) uint64_t efull_bar[kESlots];
  __shared__ __align__(8) uint64_t eempty_bar[kESlots];
  __shared__ __align__(8) uint64_t acc_bar;
  __shared__ uint32_t s_tmem;
  __shared__ uint8_t s_map[NB][kMaxBandTiles];
  __shared__ uint32_t s_mo[NB][kMaxBandTiles];  // the bands' mask offsets / 16, or kNoMeta
  __shared__ int64_t s_vo[NB][32];               // the producer's window of value offsets

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int r0 = blockIdx.x * NB;                  // first tile-row band
  // A CTA always runs NB bands: past the last band (an odd band count, two
  // bands per CTA) the second one repeats the last band's loads and products
  // and stores nothing, so that no loop below tests how many bands there are.
  const int rlast = p.bands - 1;
  auto band_of = [&](int b) { return min(r0 + b, rlast); };
  const int64_t m0 = (int64_t)blockIdx.y * PN;     // first token
  const int tpr = p.tpr;
  // ring slots at a 1024-byte boundary (the swizzle pattern repeats every 1024)
  uint8_t *smem =
      smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);

  if (tid == 0) {
    for (int s = 0; s < NS; ++s) {
      mbar_init(&full_bar[s], 1);
      mbar_init(&empty_bar[s], 1);
    }
    for (int q = 0; q < kESlots; ++q) {
      mbar_init(&efull_bar[q], kExpThreads);
      mbar_init(&eempty_bar[q], 1);
    }
    mbar_init(&acc_bar, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  for (int i = tid; i < NB * tpr; i += kPThreads) {
    const int b = i / tpr, j = i - b * tpr;
    uint8_t sp = 0;
    uint32_t mo16 = kNoMeta;
    {
      const int64_t t = (int64_t)band_of(b) * tpr + j;
      sp = p.map[t];
      const int64_t mo = p.meta_off[t];
      if (mo >= 0 && mo % 16 == 0 && mo + kSMetaBytes <= p.nmb && mo / 16 < (int64_t)kNoMeta)
        mo16 = (uint32_t)(mo / 16);
    }
    s_map[b][j] = sp;
    s_mo[b][j] = mo16;
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(&s_tmem)),
                 "r"(Sh::kTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = s_tmem;

  if (warp == 0) {
    // ------------------------------ producer ------------------------------
    // Windows of 32 tiles: lane l loads the value offsets of tile w0 + l of
    // each band (the next window's loads stay in flight while this one is
    // issued) and leaves them in shared memory, where lane 0 alone takes them
    // tile by tile (the warp meets once per window, not once per tile).
    bool ok = true;
    auto load = [&](int w0, int64_t (&vo)[NB]) {
#pragma unroll
      for (int b = 0; b < NB; ++b)
        vo[b] = w0 + lane < tpr ? __ldg(p.val_off + (int64_t)band_of(b) * tpr + w0 + lane) : 0;
    };
    int64_t nvo[NB];
    load(0, nvo);
    for (int w0 = 0; w0 < tpr && ok; w0 += 32) {
#pragma unroll
      for (int b = 0; b < NB; ++b) s_vo[b][lane] = nvo[b];
      __syncwarp();
      load(w0 + 32, nvo);
      const int nw = min(32, tpr - w0);
      for (int l = 0; l < nw && ok && lane == 0; ++l) {
        const int j = w0 + l;
        int64_t tvo[NB];
#pragma unroll
        for (int b = 0; b < NB; ++b) tvo[b] = s_vo[b][l];
        {
          if constexpr (HS == 2) {
            // one band, a whole tile per slot: both halves of A and of X
            const int s = j % NS;
            if (!ring_wait(&empty_bar[s], ((uint32_t)(j / NS) & 1u) ^ 1u)) {
              ok = false;
            } else {
              uint8_t *st = smem + (size_t)s * Sh::kSlotBytes;
              const bool sp = s_map[0][j] == 1;
              // a range outside the buffers (a corrupted matrix) is not copied
              const bool fits = sp ? (tvo[0] >= 0 && 2 * tvo[0] + kSValBytes <= p.nvb &&
                                      tvo[0] % (kPK / 2) == 0 && s_mo[0][j] != kNoMeta)
                                   : (tvo[0] >= 0 && 2 * tvo[0] + 2 * kAtomBytes <= p.nvb &&
                                      tvo[0] % kPK == 0);
              if (!fits) atomicOr(p.status, kStatusBadMap);
              const uint32_t abytes = !fits ? 0u : (sp ? (uint32_t)kAtomBytes : 2u * kAtomBytes);
              mbar_arrive_expect_tx(&full_bar[s], 2u * Sh::kXHalfBytes + abytes);
              // X: tokens m0 .. m0 + PN - 1 (rows past M read as zeros), tile j's columns
              tma_load_2d(st + kAtomBytes, &xmap, j * kPK, (int)m0, &full_bar[s]);
              tma_load_2d(st + Sh::kHalfBytes + kAtomBytes, &xmap, j * kPK + 64, (int)m0,
                          &full_bar[s]);
              if (fits && !sp) {  // the tile's first row in the 128-wide view of the values
                tma_load_2d(st, &wmap, 0, (int)(tvo[0] / kPK), &full_bar[s]);
                tma_load_2d(st + Sh::kHalfBytes, &wmap, 64, (int)(tvo[0] / kPK), &full_bar[s]);
              } else if (fits) {  // 64 kept values x 128 rows (128-byte swizzle)
                tma_load_2d(st, &spmap, 0, (int)(tvo[0] / (kPK / 2)), &full_bar[s]);
              }
            }
          } else {
            // half a tile per slot
            bool sp[NB], fits[NB];
#pragma unroll
            for (int b = 0; b < NB; ++b) {
              sp[b] = s_map[b][j] == 1;
              // a range outside the buffers (a corrupted matrix) is not copied
              fits[b] = sp[b] ? (tvo[b] >= 0 && 2 * tvo[b] + kSValBytes <= p.nvb &&
                                 tvo[b] % (kPK / 2) == 0 && s_mo[b][j] != kNoMeta)
                              : (tvo[b] >= 0 && 2 * tvo[b] + 2 * kAtomBytes <= p.nvb &&
                                 tvo[b] % kPK == 0);
              if (!fits[b]) atomicOr(p.status, kStatusBadMap);
            }
            // both halves unrolled (straight-line code: measured faster than a
            // loop that stops early)
#pragma unroll
            for (int h0 = 0; h0 < 2; ++h0) {
              if (!ok) break;
              const int idx = 2 * j + h0;  // ring position of half h0
              const int s = idx % NS;
              if (!ring_wait(&empty_bar[s], ((uint32_t)(idx / NS) & 1u) ^ 1u)) {
                ok = false;
                break;
              }
              uint8_t *st = smem + (size_t)s * Sh::kSlotBytes;
              // A's bytes in this slot: each band's half tile, 16 KB dense or
              // 8 KB of kept values
              uint32_t bytes = (uint32_t)Sh::kXHalfBytes;
#pragma unroll
              for (int b = 0; b < NB; ++b)
                if (fits[b]) bytes += sp[b] ? (uint32_t)(kAtomBytes / 2) : (uint32_t)kAtomBytes;
              mbar_arrive_expect_tx(&full_bar[s], bytes);
              // X: tokens m0 .. m0 + PN - 1 (rows past M read as zeros), columns
              // 64 h0 .. 64 h0 + 63 of tile j
              tma_load_2d(st + NB * kAtomBytes, &xmap, j * kPK + 64 * h0, (int)m0, &full_bar[s]);
#pragma unroll
              for (int b = 0; b < NB; ++b) {
                if (!fits[b]) continue;
                if (sp[b])  // kept values 32 h0 .. 32 h0 + 31 of 128 rows (64-byte swizzle)
                  tma_load_2d(st + b * kAtomBytes, &spmap, 32 * h0, (int)(tvo[b] / (kPK / 2)),
                              &full_bar[s]);
                else        // the tile's first row in the 128-wide view of the values
                  tma_load_2d(st + b * kAtomBytes, &wmap, 64 * h0, (int)(tvo[b] / kPK), &full_bar[s]);
              }
            }
          }
        }
      }
      ok = __shfl_sync(0xffffffffu, ok, 0);
      __syncwarp();  // lane 0 is done with this window's offsets
    }
    if (!ok && lane == 0) atomicOr(p.status, kStatusTimeout);
  } else if (warp == 1) {
    // ------------------------------- MMA --------------------------------
    bool ok = true;
    uint32_t nsp = 0;  // 2:4 tiles multiplied so far
    const uint32_t eb0 = smem_u32(smem + (size_t)kRingBytes);  // metadata ring
    // lane 0 alone walks the tiles (the other lanes wait at the end: no warp
    // convergence per tile, measured faster)
    for (int j = 0; j < tpr && ok && lane == 0; ++j) {
      if constexpr (HS == 2) {
        // one band, a whole tile per slot: 8 dense products, or the metadata
        // copy and 4 sparse ones
        if (lane == 0) {
          const int s = j % NS;
          const bool sp = s_map[0][j] == 1;
          const uint32_t q = nsp % Sh::kEsl;
          ok = ring_wait(&full_bar[s], (uint32_t)(j / NS) & 1u);
          if (ok && sp) ok = ring_wait(&efull_bar[q], (nsp / Sh::kEsl) & 1u);
          if (ok) {
            tc_fence_after();
            const uint32_t st = smem_u32(smem + (size_t)s * Sh::kSlotBytes);
            if (sp) {
              // A advancing 16 stored values (32 B) per K = 32 product, B 32
              // columns (64 B) of the product's half
              const uint32_t te = tmem + Sh::kTmemE + 4 * q;
              tmem_cp_128x128b(te, e_desc(eb0 + q * kEBytes));
#pragma unroll
              for (int kb = 0; kb < 4; ++kb) {
                const uint32_t ecol = te + kb;
                umma_sp_bf16(tmem, sw128_desc(st + kb * 32),
                             sw128_desc(st + (kb >> 1) * Sh::kHalfBytes + kAtomBytes + (kb & 1) * 64),
                             ecol & ~1u, ecol & 1u, (j | kb) != 0 ? 1u : 0u, kIdesc);
              }
            } else {
#pragma unroll
              for (int h = 0; h < 2; ++h)
#pragma unroll
                for (int kk = 0; kk < 4; ++kk) {
                  // K = 16 columns (32 bytes) at a time inside the 128-byte row
                  const uint32_t hb = st + h * Sh::kHalfBytes;
                  umma_bf16(tmem, sw128_desc(hb + kk * 32), sw128_desc(hb + kAtomBytes + kk * 32),
                            (j | h | kk) != 0 ? 1u : 0u, kIdesc);
                }
            }
            umma_commit(&empty_bar[s]);
            if (sp) {
              umma_commit(&eempty_bar[q]);  // the metadata slot is free once these completed
              ++nsp;
            }
          }
        }
      } else if (lane == 0) {
        // half a tile per slot, every band's products for that half
        bool sp[NB];
        uint32_t qn[NB];  // metadata ring positions of the 2:4 bands
        uint32_t c = nsp;
#pragma unroll
        for (int b = 0; b < NB; ++b) {
          sp[b] = s_map[b][j] == 1;
          qn[b] = sp[b] ? c++ : 0u;
        }
#pragma unroll
        for (int h = 0; h < 2; ++h) {  // both halves unrolled, as in the producer
          if (!ok) break;
          const int idx = 2 * j + h;
          const int s = idx % NS;
          ok = ring_wait(&full_bar[s], (uint32_t)(idx / NS) & 1u);
          if (h == 0) {
#pragma unroll
            for (int b = 0; b < NB; ++b)
              if (ok && sp[b]) ok = ring_wait(&efull_bar[qn[b] % Sh::kEsl], (qn[b] / Sh::kEsl) & 1u);
          }
          if (!ok) break;
          tc_fence_after();
          const uint32_t st = smem_u32(smem + (size_t)s * Sh::kSlotBytes);
          const uint32_t b0 = st + NB * kAtomBytes;  // X of this half
          if (h == 0) {
            // metadata to tensor memory (4 columns: one per K = 32 product)
#pragma unroll
            for (int b = 0; b < NB; ++b)
              if (sp[b])
                tmem_cp_128x128b(tmem + Sh::kTmemE + 4 * (qn[b] % Sh::kEsl),
                                 e_desc(eb0 + (qn[b] % Sh::kEsl) * kEBytes));
          }
#pragma unroll
          for (int b = 0; b < NB; ++b) {
            const uint32_t d = tmem + b * Sh::kAccStride;  // band b's accumulator
            if (sp[b]) {
              // products 2h, 2h + 1: A (this half's 32 kept values per row)
              // advancing 16 stored values (32 B), B 32 columns (64 B) each
              const uint32_t te = tmem + Sh::kTmemE + 4 * (qn[b] % Sh::kEsl);
#pragma unroll
              for (int kk = 0; kk < 2; ++kk) {
                const int kb = 2 * h + kk;
                const uint32_t ecol = te + kb;
                umma_sp_bf16(d, sw64_desc(st + b * kAtomBytes + kk * 32), sw128_desc(b0 + kk * 64),
                             ecol & ~1u, ecol & 1u, (j | kb) != 0 ? 1u : 0u, kIdesc);
              }
            } else {
#pragma unroll
              for (int kk = 0; kk < 4; ++kk)
                // K = 16 columns (32 bytes) at a time inside the 128-byte row
                umma_bf16(d, sw128_desc(st + b * kAtomBytes + kk * 32), sw128_desc(b0 + kk * 32),
                          (j | h | kk) != 0 ? 1u : 0u, kIdesc);
            }
          }
          umma_commit(&empty_bar[s]);  // the slot is free once its products completed
          if (h == 1) {
#pragma unroll
            for (int b = 0; b < NB; ++b)
              if (sp[b]) umma_commit(&eempty_bar[qn[b] % Sh::kEsl]);  // metadata slot free
            nsp = c;
          }
        }
      }
    }
    if (lane == 0) {
      if (!ok) atomicOr(p.status, kStatusTimeout);
      // the accumulators are final once every MMA issued above has completed
      // (also after a timeout, so that nothing is in flight at the end)
      umma_commit(&acc_bar);
      if (!ring_wait(&acc_bar, 0u)) atomicOr(p.status, kStatusTimeout);
    }
    __syncwarp();
  } else if (warp >= 4) {
    // ------------- 2:4 metadata for the sparse MMA, then the epilogue -------------
    // The sparse MMA reads, per K = 32 product kb, a tensor-memory column in
    // which lane L = r0 + 8 k1 + 16 r2 holds rows r = r0 + 8 r1 + 16 r2
    // (r1 = 0, 1) in its 16-bit halves r1: the four 4-column chunks c of the
    // product's columns 16 k1 .. 16 k1 + 15, one nibble each (c = 0 lowest),
    // a nibble being the two kept positions p0 < p1 as p0 | p1 << 2.  The
    // buffer is copied to tensor memory by tcgen05.cp (lane L: bytes 16 L ..
    // 16 L + 15, column kb: bytes 4 kb .. 4 kb + 3).
    const int e = tid - 128;
    const int row = e & 127;  // tile row
    const int hf = e >> 7;    // half of the row: products 2 hf, 2 hf + 1
    const int q0 = row & 7, q1 = (row >> 3) & 1, q2 = row >> 4;
    bool ok = true;
    uint32_t nsp = 0;  // 2:4 tiles converted so far
    // the half-row's 16 mask nibbles (8 bytes) of 2:4 tile (position pos =
    // NB j + b); an offset that is unusable reads nothing (the producer flags it)
    auto load_masks = [&](int pos) -> uint2 {
      const uint32_t mo16 = s_mo[pos % NB][pos / NB];
      return mo16 != kNoMeta
                 ? __ldg(reinterpret_cast<const uint2 *>(p.meta + (int64_t)mo16 * 16 +
                                                         (int64_t)row * (kPK / 8) + hf * (kPK / 16)))
                 : make_uint2(0, 0);
    };
    // kept positions of a mask nibble as p0 | p1 << 2 (masks with two bits set;
    // any other mask gives 0)
    constexpr uint64_t kIdx = (0x4ull << 12) | (0x8ull << 20) | (0x9ull << 24) | (0xCull << 36) |
                              (0xDull << 40) | (0xEull << 48);
    const int npos = NB * tpr;
    auto next_sparse = [&](int pos) {
      int q = pos < npos ? pos + 1 : npos;
      while (q < npos && s_map[q % NB][q / NB] != 1) ++q;
      return q;
    };
    auto masks_at = [&](int pos) { return pos < npos ? load_masks(pos) : make_uint2(0, 0); };
    // the masks of the next four 2:4 tiles are in flight (a load from global
    // memory takes about as long as a tile's products)
    int pos = next_sparse(-1);
    int pos1 = next_sparse(pos), pos2 = next_sparse(pos1), pos3 = next_sparse(pos2);
    uint2 cur = masks_at(pos), m1 = masks_at(pos1), m2 = masks_at(pos2), m3 = masks_at(pos3);
    while (pos < npos) {
      const int pn = next_sparse(pos3);
      const uint2 mn = masks_at(pn);
      const int q = (int)(nsp % Sh::kEsl);
      // the slot's previous tile has been multiplied
      if (!ring_wait(&eempty_bar[q], ((nsp / Sh::kEsl) & 1u) ^ 1u)) {
        ok = false;
        break;
      }
      ++nsp;
      uint8_t *eb = smem + (size_t)kRingBytes + (size_t)q * kEBytes;
#pragma unroll
      for (int kk = 0; kk < 2; ++kk) {
        const int kb = 2 * hf + kk;
        const uint32_t w = kk ? cur.y : cur.x;  // chunks 8 kb .. 8 kb + 7 (2 per byte)
#pragma unroll
        for (int k1 = 0; k1 < 2; ++k1) {
          const uint32_t m16 = (w >> (16 * k1)) & 0xFFFFu;
          uint32_t v = 0;
#pragma unroll
          for (int c = 0; c < 4; ++c) v |= (uint32_t)((kIdx >> (4 * ((m16 >> (4 * c)) & 0xFu))) & 0xFu) << (4 * c);
          const int L = q0 + 8 * k1 + 16 * q2;
          *reinterpret_cast<uint16_t *>(eb + L * 16 + 4 * kb + 2 * q1) = (uint16_t)v;
        }
      }
      // generic-proxy writes, read next by tcgen05.cp (async proxy)
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      mbar_arrive(&efull_bar[q]);
      cur = m1;
      m1 = m2;
      m2 = m3;
      m3 = mn;
      pos = pos1;
      pos1 = pos2;
      pos2 = pos3;
      pos3 = pn;
    }
    if (!ok && lane == 0) atomicOr(p.status, kStatusTimeout);
    // epilogue: TMEM lanes 32 (warp % 4) .. + 31 are this warp's weight rows;
    // one band: warps 4-7 store the block's first PN / 2 tokens, warps 8-11
    // the rest; two bands: warps 4-7 band 0, warps 8-11 band 1, every token
    if (ring_wait(&acc_bar, 0u)) {
      tc_fence_after();
      const int qw = warp & 3;
      const int b = NB == 2 && warp >= 8 ? 1 : 0;
      const int cb = NB == 1 && warp >= 8 ? PN / 2 : 0;
      const int ce = NB == 1 ? cb + PN / 2 : PN;
      if (r0 + b < p.bands) {
        const int64_t yrow = (int64_t)(r0 + b) * kPM + 32 * qw + lane;
#pragma unroll 1
        for (int c0 = cb; c0 < ce; c0 += 16) {
          float v[16];
          tmem_ld16(tmem + ((uint32_t)(32 * qw) << 16) + (uint32_t)(b * Sh::kAccStride + c0), v);
#pragma unroll
          for (int jj = 0; jj < 16; ++jj) {
            const int64_t tok = m0 + c0 + jj;
            if (tok < p.m) p.Y[tok * p.ldy + yrow] = v[jj];
          }
        }
      }
    } else if (lane == 0) {
      atomicOr(p.status, kStatusTimeout);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                 "r"(Sh::kTmemCols)
                 : "memory");
  }
}

// 2-D tensor map, bf16, box box_cols x box_rows, 128- or 64-byte swizzle
// (box_cols 64 or 32).
int encode_swz(const void *base, uint64_t cols, uint64_t rows, uint64_t row_bytes,
               uint32_t box_cols, uint32_t box_rows, CUtensorMap *map) {
  PFN_cuTensorMapEncodeTiled_v12000 encode = tensor_map_encoder();
  if (!encode) return HYB_ERR_CUDA;
  const cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  const cuuint64_t strides[1] = {(cuuint64_t)row_bytes};
  const cuuint32_t box[2] = {box_cols, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  const CUresult res = encode(
      map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims, strides, box, estr,
      CU_TENSOR_MAP_INTERLEAVE_NONE,
      box_cols == 64 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B,
      CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return res == CUDA_SUCCESS ? HYB_OK : HYB_ERR_CUDA;
}

template <int PN, int NB>
int launch_prefill(const PrefillParams &prm, const CUtensorMap &xmap, const CUtensorMap &wmap,
                   const CUtensorMap &spmap, int64_t m, cudaStream_t stream) {
  const size_t dyn = (size_t)kRingBytes + (size_t)kESlots * kEBytes + 1024;
  if (cudaFuncSetAttribute(hybrid_prefill_kernel<PN, NB>,
                           cudaFuncAttributeMaxDynamicSharedMemorySize, (int)dyn) != cudaSuccess)
    return HYB_ERR_CUDA;
  const dim3 grid((unsigned)((prm.bands + NB - 1) / NB), (unsigned)((m + PN - 1) / PN));
  hybrid_prefill_kernel<PN, NB><<<grid, kPThreads, dyn, stream>>>(prm, xmap, wmap, spmap);
  return cudaGetLastError() == cudaSuccess ? HYB_OK : HYB_ERR_CUDA;
}

// The CTA shapes (rows, tokens) the kernel is built for.
constexpr int kShapes[4][2] = {{128, 128}, {128, 256}, {256, 240}, {256, 208}};

}  // namespace
}  // namespace hyb

using namespace hyb;

size_t hyb_prefill_workspace_bytes(void) { return kHeaderBytes; }

int hyb_prefill_block_shape(int64_t n, int64_t m, int *block_rows, int *block_tokens) {
  if (!block_rows || !block_tokens) return HYB_ERR_INVALID_ARG;
  *block_rows = *block_tokens = 0;
  if (n < kPM || m < 1) return HYB_ERR_INVALID_ARG;
  int sms = 148;
  int dev = 0;
  if (cudaGetDevice(&dev) == cudaSuccess)
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (sms < 1) sms = 148;
  // Every shape streams its operands from L2 at about the same rate per SM,
  // so a CTA's time goes with the bytes it moves per tile (its bands' A and
  // its tokens' X), and the launch's with that times its waves of CTAs.
  const int64_t bands = (n + kPM - 1) / kPM;
  int64_t best = -1;
  for (const auto &sh : kShapes) {
    const int nb = sh[0] / kPM, pn = sh[1];
    if (nb > bands) continue;
    const int64_t ctas = ((bands + nb - 1) / nb) * ((m + pn - 1) / pn);
    const int64_t cost = ((ctas + sms - 1) / sms) * ((int64_t)nb * 2 * kAtomBytes + (int64_t)pn * 256);
    if (best < 0 || cost < best) {
      best = cost;
      *block_rows = sh[0];
      *block_tokens = pn;
    }
  }
  return HYB_OK;
}

int hyb_spmm_prefill_blocked(const hyb_matrix *A, int64_t m, const uint16_t *X, int64_t ldx,
                             float *Y, int64_t ldy, int block_rows, int block_tokens, void *ws,
                             size_t ws_bytes, hyb_stream_t stream) {
  if (!A || !X || !Y || m < 1) return HYB_ERR_INVALID_ARG;
  if (A->b1 != kPM || A->b2 != kPK) return HYB_ERR_UNSUPPORTED;
  if (A->n <= 0 || A->k <= 0 || A->n % kPM != 0 || A->k % kPK != 0)
    return HYB_ERR_INVALID_ARG;
  int rows = block_rows, pn = block_tokens;
  if (rows == 0 && pn == 0) {
    const int rc = hyb_prefill_block_shape(A->n, m, &rows, &pn);
    if (rc != HYB_OK) return rc;
  }
  bool known = false;
  for (const auto &sh : kShapes) known = known || (sh[0] == rows && sh[1] == pn);
  if (!known) return HYB_ERR_INVALID_ARG;
  const int64_t tpr = A->k / kPK;
  if (tpr > kMaxBandTiles || A->n / kPM > INT32_MAX || (m + pn - 1) / pn > 65535 ||
      m > INT32_MAX)
    return HYB_ERR_UNSUPPORTED;
  if (A->num_tiles != (A->n / kPM) * tpr) return HYB_ERR_INVALID_ARG;
  if (!A->tile_map || !A->vals || !A->meta || !A->val_off || !A->meta_off)
    return HYB_ERR_INVALID_ARG;
  const int64_t te = (int64_t)kPM * kPK;
  if (A->n_vals < A->num_tiles * te / 2 || A->n_vals > A->num_tiles * te ||
      A->n_vals % kPK != 0 || A->n_meta_bytes < 0 || A->n_meta_bytes > A->num_tiles * te / 8)
    return HYB_ERR_INVALID_ARG;
  if (ldx < A->k || ldy < A->n) return HYB_ERR_INVALID_ARG;
  if ((uintptr_t)A->vals % 16 != 0 || (uintptr_t)A->meta % 16 != 0 || (uintptr_t)X % 16 != 0 ||
      ldx % 8 != 0 || (uintptr_t)Y % 4 != 0)
    return HYB_ERR_ALIGNMENT;
  if (!ws || ws_bytes < kHeaderBytes) return HYB_ERR_WORKSPACE;
  if ((uintptr_t)ws % 256 != 0) return HYB_ERR_ALIGNMENT;

  alignas(64) CUtensorMap xmap{};
  alignas(64) CUtensorMap wmap{};
  // X: a box of 64 columns x one token block
  int rc = encode_swz(X, (uint64_t)A->k, (uint64_t)m, (uint64_t)ldx * 2, 64, (uint32_t)pn, &xmap);
  if (rc != HYB_OK) return rc;
  // the value buffer seen as rows of 128 bf16: a dense tile at element offset
  // vo is rows vo / 128 .. + 127
  rc = encode_swz(A->vals, (uint64_t)kPK, (uint64_t)(A->n_vals / kPK), (uint64_t)kPK * 2, 64,
                  (uint32_t)kPM, &wmap);
  if (rc != HYB_OK) return rc;
  // and as rows of 64 bf16: a 2:4 tile's 128 rows of kept values at element
  // offset vo are rows vo / 64 .. + 127, loaded whole (a box of 64 values,
  // 128-byte swizzle) where a ring slot holds a whole tile, else by halves (a
  // box of 32 values, 64-byte swizzle)
  alignas(64) CUtensorMap spmap{};
  const bool whole_tiles = rows == 128 && pn == 128;
  rc = encode_swz(A->vals, (uint64_t)(kPK / 2), (uint64_t)(A->n_vals / (kPK / 2)), (uint64_t)kPK,
                  whole_tiles ? 64u : 32u, (uint32_t)kPM, &spmap);
  if (rc != HYB_OK) return rc;

  PrefillParams prm{};
  prm.map = A->tile_map;
  prm.vals = A->vals;
  prm.meta = A->meta;
  prm.val_off = A->val_off;
  prm.meta_off = A->meta_off;
  prm.n = A->n;
  prm.k = A->k;
  prm.m = m;
  prm.tpr = (int)tpr;
  prm.bands = (int)(A->n / kPM);
  prm.nvb = 2 * A->n_vals;
  prm.nmb = A->n_meta_bytes;
  prm.Y = Y;
  prm.ldy = ldy;
  prm.status = static_cast<uint32_t *>(ws);

  cudaStream_t st = (cudaStream_t)stream;
  if (rows == 256)
    return pn == 240 ? launch_prefill<240, 2>(prm, xmap, wmap, spmap, m, st)
                     : launch_prefill<208, 2>(prm, xmap, wmap, spmap, m, st);
  return pn == 256 ? launch_prefill<256, 1>(prm, xmap, wmap, spmap, m, st)
                   : launch_prefill<128, 1>(prm, xmap, wmap, spmap, m, st);
}

int hyb_spmm_prefill(const hyb_matrix *A, int64_t m, const uint16_t *X, int64_t ldx, float *Y,
                     int64_t ldy, void *ws, size_t ws_bytes, hyb_stream_t stream) {
  return hyb_spmm_prefill_blocked(A, m, X, ldx, Y, ldy, 0, 0, ws, ws_bytes, stream);
}
