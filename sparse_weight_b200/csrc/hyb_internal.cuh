// hyb_internal.cuh -- device helpers shared by the libhyb CUDA sources.
//
// Nothing here is part of the C ABI (include/hyb.h is).  Target: sm_100a.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>
#include <stdint.h>

#include <mutex>

#include "hyb.h"

namespace hyb {

// Status bits kept in the first word of every workspace.
constexpr uint32_t kStatusNaN = 1u;      // hyb_pack saw a NaN weight
constexpr uint32_t kStatusBadMap = 2u;   // tile_map byte other than 0 / 1
constexpr uint32_t kStatusTimeout = 4u;  // a bounded wait inside a kernel ran out

// Workspace header: status word, padded so that what follows is aligned.
constexpr size_t kHeaderBytes = 256;
// At fixed places whatever the call's shape, batch or rank (so that calls of
// different shapes can share a workspace): in the header, the epoch of the
// fused low-rank term's grid barriers and the ticket of the separate V^T x
// kernel; after the header, one barrier flag per CTA of the fused term.
constexpr size_t kLowrankEpochOffset = 16;
constexpr size_t kLowrankTicketOffset = 24;
constexpr size_t kLowrankFlagsOffset = kHeaderBytes;
constexpr int kLowrankFlags = 256;  // at least the most CTAs a streaming launch has
constexpr size_t kTicketsOffset = kLowrankFlagsOffset + 4 * kLowrankFlags;

__host__ __device__ inline size_t align_up(size_t v, size_t a) {
  return (v + a - 1) / a * a;
}

// ---- bf16 <-> fp32 --------------------------------------------------------
// A bf16 value is the upper half of a binary32: widening is a shift.
__device__ __forceinline__ float bf16_lo(uint32_t pair) {
  return __uint_as_float(pair << 16);
}
__device__ __forceinline__ float bf16_hi(uint32_t pair) {
  return __uint_as_float(pair & 0xFFFF0000u);
}
// fp32 -> bf16, round-to-nearest-even (CUDA's conversion intrinsic).
__device__ __forceinline__ uint16_t f32_to_bf16_rne(float f) {
  return __bfloat16_as_ushort(__float2bfloat16_rn(f));
}

// ---- streaming loads -------------------------------------------------------
// Weights are read exactly once per call: read-only path, no L1 allocation;
// the 32-byte form also carries an L2 evict-first hint so streamed weights do
// not push the reused operands (X, the low-rank factors, partial sums) out.
__device__ __forceinline__ uint4 ld_stream16(const void *p) {
  uint4 r;
  asm volatile(
      "ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
      : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
      : "l"(p));
  return r;
}
// 32-byte load (sm_100 256-bit global load).
__device__ __forceinline__ void ld_stream32(const void *p, uint4 &a, uint4 &b) {
  asm volatile(
      "ld.global.nc.L1::no_allocate.L2::evict_first.v8.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
      : "=r"(a.x), "=r"(a.y), "=r"(a.z), "=r"(a.w), "=r"(b.x), "=r"(b.y),
        "=r"(b.z), "=r"(b.w)
      : "l"(p));
}
// 8-byte load, same hints as ld_stream16.
__device__ __forceinline__ uint2 ld_stream8(const void *p) {
  uint2 r;
  asm volatile("ld.global.nc.L1::no_allocate.v2.u32 {%0,%1}, [%2];"
               : "=r"(r.x), "=r"(r.y)
               : "l"(p));
  return r;
}
__device__ __forceinline__ uint32_t ld_stream_u8(const void *p) {
  uint16_t r;
  asm volatile("ld.global.nc.L1::no_allocate.u8 %0, [%1];" : "=h"(r) : "l"(p));
  return r;
}
__device__ __forceinline__ uint16_t ld_stream_u16(const void *p) {
  uint16_t r;
  asm volatile("ld.global.nc.L1::no_allocate.u16 %0, [%1];"
               : "=h"(r)
               : "l"(p));
  return r;
}
// Reused operand (X): read-only path, cached in L1.
__device__ __forceinline__ uint4 ld_keep16(const void *p) {
  return __ldg(reinterpret_cast<const uint4 *>(p));
}

// ---- host helpers -----------------------------------------------------------
int device_sm_count(int *out);  // cached per device


// ---- shared-memory barriers and bulk / tensor copies (sm_90+) -------------
// Every wait is bounded: a wait that runs out returns false, and the caller
// records kStatusTimeout and leaves its pipeline instead of waiting for ever.
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
__device__ __forceinline__ bool mbar_wait_limit(uint64_t *bar, uint32_t parity,
                                                uint32_t limit) {
  for (uint32_t i = 0; i < limit; ++i)
    if (mbar_try_wait(bar, parity)) return true;
  return false;
}
__device__ __forceinline__ bool mbar_wait(uint64_t *bar, uint32_t parity) {
  return mbar_wait_limit(bar, parity, kWaitLimit);
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

// The driver's tensor-map encoder, found once through the runtime.
inline PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
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
  return encode;
}

}  // namespace hyb
