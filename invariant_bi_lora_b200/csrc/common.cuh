// common.cuh -- shared device helpers for libbi (sm_100a).
//
// All fp32 arithmetic that is part of a canonical reduction order is written
// with the _rn intrinsics (__fadd_rn, __fmul_rn, __fdiv_rn, __fsqrt_rn), which
// the compiler never contracts into FMAs or reassociates.  The library is
// built without --use_fast_math.
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "bi.h"

#define BI_DEV __device__ __forceinline__

namespace bi {

// ----------------------------------------------------------------------
// Device status word: the first error a kernel meets is recorded here
// (atomicCAS from 0), the host reads and clears it.  Kernels receive its
// address as a parameter so that every translation unit can use it.
// ----------------------------------------------------------------------
BI_DEV void flag_error(unsigned *status, unsigned code) {
  if (status) atomicCAS(status, 0u, code);
}

// Host side: address of the status word on the current device.
unsigned *status_word();
// Host side: SM count of the current device.
int num_sms();

// ----------------------------------------------------------------------
// bf16 <-> fp32.  A bf16 value is the top half of an fp32 value, so the
// widening is exact bit placement.
// ----------------------------------------------------------------------
BI_DEV float bf16lo(uint32_t pair) { return __uint_as_float(pair << 16); }
BI_DEV float bf16hi(uint32_t pair) { return __uint_as_float(pair & 0xffff0000u); }

// fp32 -> bf16, round to nearest even (the hardware cvt.rn.bf16.f32).
BI_DEV uint16_t f32_to_bf16(float f) {
  return __bfloat16_as_ushort(__float2bfloat16_rn(f));
}
BI_DEV uint32_t pack_bf16x2(float lo, float hi) {
  return (uint32_t)f32_to_bf16(lo) | ((uint32_t)f32_to_bf16(hi) << 16);
}

// 128-bit read-only load through the non-coherent path.
BI_DEV uint4 ldg128(const void *p) { return __ldg(reinterpret_cast<const uint4 *>(p)); }

// 128-bit load that should not displace reused lines (data read once).
BI_DEV uint4 ldg128_stream(const void *p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

// ----------------------------------------------------------------------
// Warp-level mma.sync m16n8k16, bf16 inputs, fp32 accumulate:
//   d = a . b + c
// Not volatile: the compiler may move it past other instructions (it has no
// effect beyond its outputs), so independent chains can be interleaved.
// ----------------------------------------------------------------------
BI_DEV void mma_bf16_16816(float d[4], const uint32_t a[4], const uint32_t b[2],
                           const float c[4]) {
  asm(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 "
      "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%10,%11,%12,%13};"
      : "=f"(d[0]), "=f"(d[1]), "=f"(d[2]), "=f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]),
        "f"(c[0]), "f"(c[1]), "f"(c[2]), "f"(c[3]));
}

// Warp butterfly over 32 lanes.  Offsets 1, 2, 4, 8, 16 pair lanes
// (2i, 2i+1), then pairs of pairs, ...: exactly the canonical tree over the
// 32 lane values (IEEE addition is commutative, so both partners of a pair
// hold the same bits).
BI_DEV float warp_tree_sum(float v) {
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) v = __fadd_rn(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

BI_DEV float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// Largest adapter count of a plan (segment n_ad holds the tokens without
// an adapter).
constexpr int kMaxAdapters = 256;

// ----------------------------------------------------------------------
// Plan layout (int32 words), written by bi_lora_plan:
//   perm[M]                 token indices grouped by adapter
//   offsets[n_ad + 2]       segment starts in perm
//   (zero to three words of padding: the table starts on 16 bytes)
//   table[plan_tiles(M, n_ad)][kPlanRec]
// Table record i describes the i-th 64-row tile of the segments taken in
// order (segment a's tiles are its positions offsets[a] + 64j ...):
//   {adapter (n_ad = no adapter, -1 = past the last tile), rows (1..64),
//    first perm position, 0, token ids[64]} -- ids past `rows` are -1.
// A kernel finds its tile's adapter and every token row in one read of
// 272 bytes, instead of reading the offsets, then perm, then x.
// ----------------------------------------------------------------------
constexpr int kPlanTile = 64;
constexpr int kPlanRec = 4 + kPlanTile;
__host__ __device__ constexpr long plan_table_word(long M, int n_ad) { return (M + n_ad + 2 + 3) & ~3L; }
__host__ __device__ constexpr long plan_tiles(long M, int n_ad) { return (M + kPlanTile - 1) / kPlanTile + n_ad + 1; }
__host__ __device__ constexpr long plan_words(long M, int n_ad) {
  return plan_table_word(M, n_ad) + kPlanRec * plan_tiles(M, n_ad);
}

}  // namespace bi

// Host-side helpers shared by the launch code.
#define BI_CUDA_TRY(expr)                          \
  do {                                             \
    cudaError_t _e = (expr);                       \
    if (_e != cudaSuccess) return BI_ERR_CUDA;     \
  } while (0)

static inline bool bi_aligned16(const void *p) { return (((uintptr_t)p) & 15u) == 0; }
static inline bool bi_pow2(long v) { return v > 0 && (v & (v - 1)) == 0; }
