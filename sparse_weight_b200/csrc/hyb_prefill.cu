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
//   * CTA (band r, token block mb) owns Y[PN mb .. +PN][128 r .. +128]: a
//     128 x PN fp32 accumulator in tensor memory (TMEM), M = 128 weight rows,
//     N = PN tokens (128 or 256), K looped over the band's tiles (128 columns
//     each), every tile in two halves of 64 columns.
//   * warp 0 (one lane) moves the operands with TMA into a ring of 192 KB
//     (3 slots of a whole tile at N = 128, 4 slots of a half-tile at N =
//     256): a dense tile's half as a 2-D box of 64 columns x 128 rows with
//     128-byte swizzle (the K-major layout tcgen05.mma reads), a 2:4 tile's
//     kept values with its first half as one box of 64 values x 128 rows
//     (already the sparse MMA's compressed A operand: 2 kept values per group
//     of 4, ascending), X as a box of 64 columns x PN tokens per half.
//   * warps 4-11 turn each 2:4 tile's masks into the sparse MMA's metadata
//     (the two kept positions of a group as a nibble, laid out by tensor-
//     memory lane and column), fence it for the async proxy and signal the
//     MMA warp.
//   * warp 1 owns the TMEM allocation; one lane issues per half-tile 4
//     tcgen05.mma (dense: kind::f16, bf16 x bf16 -> fp32, K = 16 each) or, for
//     a 2:4 tile, a tcgen05.cp of the metadata and 2 tcgen05.mma.sp (K = 32
//     each) per half, and frees each ring slot with tcgen05.commit (a 2:4
//     tile's first half-tile slot only after its second half's products: it
//     holds A).
//   * warps 4-11 then read the accumulator with tcgen05.ld (warp w: TMEM lanes
//     32 (w % 4) .., half of the token columns each) and store Y (a warp
//     writes 32 consecutive rows of one token: 128 contiguous bytes).
//
// Every half-tile moves 16 KB of A and PN x 128 bytes of X into shared
// memory for PN x 128 x 64 multiply-adds, so N = 256 halves the operand bytes
// per product of N = 128; it is taken when the grid still fills the SMs.
// A 2:4 tile moves the hybrid format's bytes and costs half a dense tile's
// tensor work.  Every wait is bounded; one that runs out sets kStatusTimeout
// in the status word and the CTA leaves its pipeline.
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

// The shape of one CTA's pipeline at PN tokens.  A ring slot holds HS
// half-tiles (64 columns each): A's halves (16 KB each), then X's (PN x 128
// bytes each); a whole tile per slot at N = 128 (3 slots of 64 KB), a half
// per slot at N = 256 (4 slots of 48 KB).  TMEM holds the PN-column fp32
// accumulator, then 4 metadata columns per metadata slot.
template <int PN>
struct PrefillShape {
  static constexpr int HS = PN == 256 ? 1 : 2;  // half-tiles per ring slot
  static constexpr int kXHalfBytes = PN * 128;
  static constexpr int kSlotBytes = HS * (kAtomBytes + kXHalfBytes);
  static constexpr int kSlots = kRingBytes / kSlotBytes;
  static constexpr int kTmemCols = PN == 256 ? 512 : 256;
  static constexpr int kTmemE = PN;  // first metadata column
  static_assert(PN == 128 || PN == 256, "N = 128 or 256 tokens per CTA");
  static_assert(kSlots >= 3 && kSlots <= kMaxSlots, "ring depth");
  static_assert(kSlotBytes % 1024 == 0, "slots keep the 1024-byte swizzle alignment");
  static_assert(kTmemE + 4 * kESlots <= kTmemCols, "metadata columns fit the allocation");
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
  int64_t nvb, nmb;  // bytes of the value and mask buffers
  float *Y;
  int64_t ldy;
  uint32_t *status;
};

template <int PN>
__global__ void __launch_bounds__(kPThreads, 1)
    hybrid_prefill_kernel(const PrefillParams p, const __grid_constant__ CUtensorMap xmap,
                          const __grid_constant__ CUtensorMap wmap,
                          const __grid_constant__ CUtensorMap spmap) {
  using Sh = PrefillShape<PN>;
  constexpr int NS = Sh::kSlots, HS = Sh::HS;
  constexpr uint32_t kIdesc = idesc_f16<PN>();
  extern __shared__ uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t full_bar[kMaxSlots];
  __shared__ __align__(8) uint64_t empty_bar[kMaxSlots];
  // the metadata ring: slot q holds the metadata of every kESlots-th 2:4 tile
  // of the band (efull: written; eempty: the MMAs that read it completed).
  // The converting warps and the MMA warp take the 2:4 tiles in the same
  // order, and each waits for the other's previous use of the slot, so
  // neither barrier runs two phases ahead of a thread waiting on it.
  __shared__ __align__(8) uint64_t efull_bar[kESlots];
  __shared__ __align__(8) uint64_t eempty_bar[kESlots];
  __shared__ __align__(8) uint64_t acc_bar;
  __shared__ uint32_t s_tmem;
  __shared__ uint8_t s_map[kMaxBandTiles];
  __shared__ int64_t s_mo[kMaxBandTiles];  // the band's mask offsets

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int r = blockIdx.x;                  // tile-row band
  const int64_t m0 = (int64_t)blockIdx.y * PN;  // first token
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
  for (int j = tid; j < tpr; j += kPThreads) {
    const int64_t t = (int64_t)r * tpr + j;
    s_map[j] = p.map[t];
    s_mo[j] = p.meta_off[t];
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
    // lane l holds the offsets of tile w0 + l of the band (a window of 32,
    // the next window loaded while this one is issued)
    bool ok = true;
    const int64_t t_band = (int64_t)r * tpr;
    auto load = [&](int w0, int64_t &vo, int64_t &mo) {
      vo = mo = 0;
      if (w0 + lane < tpr) {
        vo = __ldg(p.val_off + t_band + w0 + lane);
        mo = __ldg(p.meta_off + t_band + w0 + lane);
      }
    };
    int64_t vo, mo, nvo, nmo;
    load(0, vo, mo);
    for (int w0 = 0; w0 < tpr && ok; w0 += 32) {
      load(w0 + 32, nvo, nmo);
      const int nw = min(32, tpr - w0);
      for (int l = 0; l < nw && ok; ++l) {
        const int j = w0 + l;
        const int64_t tvo = __shfl_sync(0xffffffffu, vo, l);
        const int64_t tmo = __shfl_sync(0xffffffffu, mo, l);
        if (lane == 0) {
          const bool sp = s_map[j] == 1;
          // a range outside the buffers (a corrupted matrix) is not copied
          const bool fits = sp ? (tvo >= 0 && tmo >= 0 && 2 * tvo + kSValBytes <= p.nvb &&
                                  tmo + kSMetaBytes <= p.nmb && tvo % (kPK / 2) == 0 &&
                                  tmo % 16 == 0)
                               : (tvo >= 0 && 2 * tvo + 2 * kAtomBytes <= p.nvb &&
                                  tvo % kPK == 0);
          if (!fits) atomicOr(p.status, kStatusBadMap);
          for (int h0 = 0; h0 < 2 && ok; h0 += HS) {
            const int idx = (2 * j + h0) / HS;  // ring position of halves h0 .. h0 + HS - 1
            const int s = idx % NS;
            if (!ring_wait(&empty_bar[s], ((uint32_t)(idx / NS) & 1u) ^ 1u)) {
              ok = false;
              break;
            }
            uint8_t *st = smem + (size_t)s * Sh::kSlotBytes;
            // A's bytes in this slot: a dense tile's halves, or a 2:4 tile's
            // whole compressed operand with its first half
            const uint32_t abytes =
                !fits ? 0u : (sp ? (h0 == 0 ? (uint32_t)kAtomBytes : 0u) : (uint32_t)(HS * kAtomBytes));
            mbar_arrive_expect_tx(&full_bar[s], (uint32_t)(HS * Sh::kXHalfBytes) + abytes);
            for (int hh = 0; hh < HS; ++hh) {
              const int h = h0 + hh;
              // X: tokens m0 .. m0 + PN - 1 (rows past M read as zeros),
              // columns 64 h .. 64 h + 63 of tile j
              tma_load_2d(st + HS * kAtomBytes + hh * Sh::kXHalfBytes, &xmap, j * kPK + 64 * h,
                          (int)m0, &full_bar[s]);
              if (fits && !sp)  // the tile's first row in the 128-wide view of the values
                tma_load_2d(st + hh * kAtomBytes, &wmap, 64 * h, (int)(tvo / kPK), &full_bar[s]);
            }
            if (fits && sp && h0 == 0)  // 64 kept values x 128 rows (128-byte swizzle)
              tma_load_2d(st, &spmap, 0, (int)(tvo / (kPK / 2)), &full_bar[s]);
          }
        }
        ok = __shfl_sync(0xffffffffu, ok, 0);
      }
      vo = nvo;
      mo = nmo;
    }
    if (!ok && lane == 0) atomicOr(p.status, kStatusTimeout);
  } else if (warp == 1) {
    // ------------------------------- MMA --------------------------------
    bool ok = true;
    uint32_t nsp = 0;  // 2:4 tiles multiplied so far
    const uint32_t eb0 = smem_u32(smem + (size_t)kRingBytes);  // metadata ring
    for (int j = 0; j < tpr && ok; ++j) {
      if (lane == 0) {
        const bool sp = s_map[j] == 1;
        const int q = (int)(nsp % kESlots);
        const uint32_t te = tmem + Sh::kTmemE + 4 * q;
        uint32_t a_sp = 0;  // a 2:4 tile's compressed A (in its first half's slot)
        int s_first = 0;
        for (int h0 = 0; h0 < 2 && ok; h0 += HS) {
          const int idx = (2 * j + h0) / HS;
          const int s = idx % NS;
          ok = ring_wait(&full_bar[s], (uint32_t)(idx / NS) & 1u);
          if (ok && sp && h0 == 0) ok = ring_wait(&efull_bar[q], (nsp / kESlots) & 1u);
          if (!ok) break;
          tc_fence_after();
          const uint32_t st = smem_u32(smem + (size_t)s * Sh::kSlotBytes);
          if (sp && h0 == 0) {
            // metadata to tensor memory (4 columns: one per K = 32 product)
            tmem_cp_128x128b(te, e_desc(eb0 + (uint32_t)q * kEBytes));
            a_sp = st;
            s_first = s;
          }
#pragma unroll
          for (int hh = 0; hh < HS; ++hh) {
            const int h = h0 + hh;
            const uint32_t a0 = st + hh * kAtomBytes;
            const uint32_t b0 = st + HS * kAtomBytes + hh * Sh::kXHalfBytes;
            if (sp) {
              // products 2h, 2h + 1: A advancing 16 stored values (32 B), B 32
              // columns (64 B) of this half each
#pragma unroll
              for (int kk = 0; kk < 2; ++kk) {
                const int kb = 2 * h + kk;
                const uint32_t ecol = te + kb;
                umma_sp_bf16(tmem, sw128_desc(a_sp + kb * 32), sw128_desc(b0 + kk * 64),
                             ecol & ~1u, ecol & 1u, (j | kb) != 0 ? 1u : 0u, kIdesc);
              }
            } else {
#pragma unroll
              for (int kk = 0; kk < 4; ++kk)
                // K = 16 columns (32 bytes) at a time inside the 128-byte row
                umma_bf16(tmem, sw128_desc(a0 + kk * 32), sw128_desc(b0 + kk * 32),
                          (j | h | kk) != 0 ? 1u : 0u, kIdesc);
            }
          }
          // the slot is free once its products completed; a 2:4 tile's first
          // slot holds A for the second half too
          if (!sp || HS == 2) {
            umma_commit(&empty_bar[s]);
          } else if (h0 == 1) {
            umma_commit(&empty_bar[s_first]);
            umma_commit(&empty_bar[s]);
          }
          if (sp && h0 + HS == 2) {
            umma_commit(&eempty_bar[q]);  // the metadata slot is free once these completed
            ++nsp;
          }
        }
      }
      ok = __shfl_sync(0xffffffffu, ok, 0);
    }
    if (lane == 0) {
      if (!ok) atomicOr(p.status, kStatusTimeout);
      // the accumulator is final once every MMA issued above has completed
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
    const int r0 = row & 7, r1 = (row >> 3) & 1, r2 = row >> 4;
    bool ok = true;
    uint32_t nsp = 0;  // 2:4 tiles converted so far
    // the half-row's 16 mask nibbles (8 bytes); a range outside the buffer (a
    // corrupted matrix) reads nothing (the producer flags it)
    auto load_masks = [&](int j) -> uint2 {
      const int64_t mo = s_mo[j];
      const bool fits = mo >= 0 && mo + kSMetaBytes <= p.nmb && mo % 16 == 0;
      return fits ? __ldg(reinterpret_cast<const uint2 *>(p.meta + mo + (int64_t)row * (kPK / 8) +
                                                         hf * (kPK / 16)))
                  : make_uint2(0, 0);
    };
    // kept positions of a mask nibble as p0 | p1 << 2 (masks with two bits set;
    // any other mask gives 0)
    constexpr uint64_t kIdx = (0x4ull << 12) | (0x8ull << 20) | (0x9ull << 24) | (0xCull << 36) |
                              (0xDull << 40) | (0xEull << 48);
    auto next_sparse = [&](int j) {
      int q = j + 1;
      while (q < tpr && s_map[q] != 1) ++q;
      return q;
    };
    int j = next_sparse(-1);
    uint2 cur = j < tpr ? load_masks(j) : make_uint2(0, 0);
    while (j < tpr) {
      const int jn = next_sparse(j);
      const uint2 nxt = jn < tpr ? load_masks(jn) : make_uint2(0, 0);
      const int q = (int)(nsp % kESlots);
      // the slot's previous tile has been multiplied
      if (!ring_wait(&eempty_bar[q], ((nsp / kESlots) & 1u) ^ 1u)) {
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
          const int L = r0 + 8 * k1 + 16 * r2;
          *reinterpret_cast<uint16_t *>(eb + L * 16 + 4 * kb + 2 * r1) = (uint16_t)v;
        }
      }
      // generic-proxy writes, read next by tcgen05.cp (async proxy)
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      mbar_arrive(&efull_bar[q]);
      cur = nxt;
      j = jn;
    }
    if (!ok && lane == 0) atomicOr(p.status, kStatusTimeout);
    // epilogue: TMEM lanes 32 (warp % 4) .. + 31 are this warp's weight rows;
    // warps 4-7 store the block's first PN / 2 tokens, warps 8-11 the rest
    if (ring_wait(&acc_bar, 0u)) {
      tc_fence_after();
      const int q = warp & 3;
      const int64_t yrow = (int64_t)r * kPM + 32 * q + lane;
      const int cb = warp >= 8 ? PN / 2 : 0;
#pragma unroll 1
      for (int c0 = cb; c0 < cb + PN / 2; c0 += 16) {
        float v[16];
        tmem_ld16(tmem + ((uint32_t)(32 * q) << 16) + (uint32_t)c0, v);
#pragma unroll
        for (int jj = 0; jj < 16; ++jj) {
          const int64_t tok = m0 + c0 + jj;
          if (tok < p.m) p.Y[tok * p.ldy + yrow] = v[jj];
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

// 2-D tensor map, bf16, 128-byte swizzle, box 64 columns x box_rows rows.
int encode_sw128(const void *base, uint64_t cols, uint64_t rows, uint64_t row_bytes,
                 uint32_t box_rows, CUtensorMap *map) {
  PFN_cuTensorMapEncodeTiled_v12000 encode = tensor_map_encoder();
  if (!encode) return HYB_ERR_CUDA;
  const cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  const cuuint64_t strides[1] = {(cuuint64_t)row_bytes};
  const cuuint32_t box[2] = {64, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  const CUresult res =
      encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims, strides,
             box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return res == CUDA_SUCCESS ? HYB_OK : HYB_ERR_CUDA;
}

template <int PN>
int launch_prefill(const PrefillParams &prm, const CUtensorMap &xmap, const CUtensorMap &wmap,
                   const CUtensorMap &spmap, int64_t bands, int64_t m, cudaStream_t stream) {
  const size_t dyn = (size_t)kRingBytes + (size_t)kESlots * kEBytes + 1024;
  if (cudaFuncSetAttribute(hybrid_prefill_kernel<PN>,
                           cudaFuncAttributeMaxDynamicSharedMemorySize, (int)dyn) != cudaSuccess)
    return HYB_ERR_CUDA;
  const dim3 grid((unsigned)bands, (unsigned)((m + PN - 1) / PN));
  hybrid_prefill_kernel<PN><<<grid, kPThreads, dyn, stream>>>(prm, xmap, wmap, spmap);
  return cudaGetLastError() == cudaSuccess ? HYB_OK : HYB_ERR_CUDA;
}

}  // namespace
}  // namespace hyb

using namespace hyb;

size_t hyb_prefill_workspace_bytes(void) { return kHeaderBytes; }

int hyb_prefill_block_tokens(int64_t n, int64_t m) {
  if (n <= 0 || m <= 0) return 0;
  int sms = 148;
  int dev = 0;
  if (cudaGetDevice(&dev) == cudaSuccess)
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  // 256 tokens per CTA when that grid still gives every SM a CTA
  const int64_t ctas256 = ((n + kPM - 1) / kPM) * ((m + 255) / 256);
  return ctas256 >= sms ? 256 : 128;
}

int hyb_spmm_prefill_blocked(const hyb_matrix *A, int64_t m, const uint16_t *X, int64_t ldx,
                             float *Y, int64_t ldy, int block_tokens, void *ws, size_t ws_bytes,
                             hyb_stream_t stream) {
  if (!A || !X || !Y || m < 1) return HYB_ERR_INVALID_ARG;
  if (block_tokens != 0 && block_tokens != 128 && block_tokens != 256)
    return HYB_ERR_INVALID_ARG;
  if (A->b1 != kPM || A->b2 != kPK) return HYB_ERR_UNSUPPORTED;
  if (A->n <= 0 || A->k <= 0 || A->n % kPM != 0 || A->k % kPK != 0)
    return HYB_ERR_INVALID_ARG;
  const int64_t tpr = A->k / kPK;
  const int pn = block_tokens ? block_tokens : hyb_prefill_block_tokens(A->n, m);
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
  int rc = encode_sw128(X, (uint64_t)A->k, (uint64_t)m, (uint64_t)ldx * 2, (uint32_t)pn, &xmap);
  if (rc != HYB_OK) return rc;
  // the value buffer seen as rows of 128 bf16: a dense tile at element offset
  // vo is rows vo / 128 .. + 127
  rc = encode_sw128(A->vals, (uint64_t)kPK, (uint64_t)(A->n_vals / kPK), (uint64_t)kPK * 2,
                    (uint32_t)kPM, &wmap);
  if (rc != HYB_OK) return rc;
  // and as rows of 64 bf16: a 2:4 tile's 128 rows of kept values at element
  // offset vo are rows vo / 64 .. + 127
  alignas(64) CUtensorMap spmap{};
  rc = encode_sw128(A->vals, (uint64_t)(kPK / 2), (uint64_t)(A->n_vals / (kPK / 2)),
                    (uint64_t)kPK, (uint32_t)kPM, &spmap);
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
  prm.nvb = 2 * A->n_vals;
  prm.nmb = A->n_meta_bytes;
  prm.Y = Y;
  prm.ldy = ldy;
  prm.status = static_cast<uint32_t *>(ws);

  const int64_t bands = A->n / kPM;
  return pn == 256
             ? launch_prefill<256>(prm, xmap, wmap, spmap, bands, m, (cudaStream_t)stream)
             : launch_prefill<128>(prm, xmap, wmap, spmap, bands, m, (cudaStream_t)stream);
}

int hyb_spmm_prefill(const hyb_matrix *A, int64_t m, const uint16_t *X, int64_t ldx, float *Y,
                     int64_t ldy, void *ws, size_t ws_bytes, hyb_stream_t stream) {
  return hyb_spmm_prefill_blocked(A, m, X, ldx, Y, ldy, 0, ws, ws_bytes, stream);
}
