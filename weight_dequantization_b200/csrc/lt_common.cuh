// lt_common.cuh -- device helpers shared by the decode kernels (sm_100a).
#pragma once

#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "lt_decode.h"

#define LT_API extern "C" __attribute__((visibility("default")))

namespace lt {

// ---------------------------------------------------------------------------
// device status: first error wins
// ---------------------------------------------------------------------------
__device__ __forceinline__ void report(int32_t *d_status, int32_t code) {
  if (d_status != nullptr) atomicCAS(d_status, 0, code);
}

// ---------------------------------------------------------------------------
// global memory access
// ---------------------------------------------------------------------------
// Read-only, streamed once: do not keep in L1.
__device__ __forceinline__ uint32_t ld_stream_u32(const void *p) {
  uint32_t v;
  asm volatile("ld.global.nc.L1::no_allocate.u32 %0, [%1];" : "=r"(v) : "l"(p));
  return v;
}
__device__ __forceinline__ uint2 ld_stream_u64(const void *p) {
  uint2 v;
  asm volatile("ld.global.nc.L1::no_allocate.v2.u32 {%0, %1}, [%2];" : "=r"(v.x), "=r"(v.y) : "l"(p));
  return v;
}
__device__ __forceinline__ uint4 ld_stream_u128(const void *p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}
// 8 little-endian bytes at p, any alignment, inside a caller's buffer
// [lo, hi): two aligned 8-byte loads when both aligned words lie inside the
// buffer, byte loads at its edges (never a byte outside [lo, hi)).
struct GlobalBytes {
  const uint8_t *lo, *hi;
  __device__ __forceinline__ uint64_t rd64(const uint8_t *p) const {
    const uintptr_t a = reinterpret_cast<uintptr_t>(p) & ~uintptr_t(7);
    const uint32_t sh = (uint32_t)(reinterpret_cast<uintptr_t>(p) & 7) * 8;
    const uint64_t *w = reinterpret_cast<const uint64_t *>(a);
    if (sh == 0) return __ldg(reinterpret_cast<const unsigned long long *>(w));
    if (a >= reinterpret_cast<uintptr_t>(lo) && a + 16 <= reinterpret_cast<uintptr_t>(hi)) {
      const uint64_t x = __ldg(reinterpret_cast<const unsigned long long *>(w));
      const uint64_t y = __ldg(reinterpret_cast<const unsigned long long *>(w + 1));
      return (x >> sh) | (y << (64 - sh));
    }
    uint64_t v = 0;
#pragma unroll
    for (int i = 0; i < 8; ++i) v |= (uint64_t)__ldg(p + i) << (8 * i);
    return v;
  }
};

// Output written once and not read back by this kernel.
__device__ __forceinline__ void st_u128(void *p, uint4 v) {
  asm volatile("st.global.v4.u32 [%0], {%1, %2, %3, %4};" ::"l"(p), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w)
               : "memory");
}

// ---------------------------------------------------------------------------
// exact (q - z) * s in binary16
// ---------------------------------------------------------------------------
// Both halves of a half2 are formed exactly from small integers with the
// "magic number" construction: OR-ing an integer m into the fraction of a
// binary16 with a fixed exponent gives base + m * ulp(base). For the low half
// base 1024 (ulp 1), for the high half base 64 (ulp 1/16) with the code
// placed 4 bits higher -- so one byte b = lo | hi << 4 becomes
// (1024 + lo, 64 + hi) with a single PRMT + LOP3. Subtracting
// (1024 + z, 64 + z) leaves (lo - z, hi - z) exactly (integers of magnitude
// <= 255), and one correctly rounded binary16 multiply by s gives
// fp16_rn((q - z) * s): the product of an exact integer and s rounded once.
__device__ __forceinline__ uint32_t hsub2_rn(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("sub.rn.f16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}
__device__ __forceinline__ uint32_t hmul2_rn(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}
// byte j of w -> half2 (1024 + low nibble, 64 + high nibble)
template <int J>
__device__ __forceinline__ uint32_t int4_pair_magic(uint32_t w) {
  constexpr uint32_t sel = (uint32_t)J | 0x40u | ((uint32_t)J << 8) | 0x4000u;  // [bJ, 0, bJ, 0]
  uint32_t x = __byte_perm(w, 0u, sel);
  uint32_t r;
  asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(r) : "r"(x), "r"(0x00F0000Fu), "r"(0x54006400u));  // (a & b) | c
  return r;
}
// the subtrahend (1024 + z, 64 + z) for an unsigned zero point z <= 255
__device__ __forceinline__ uint32_t int4_zero_magic(uint32_t z) {
  __half lo = __float2half_rn(1024.0f + (float)z);
  __half hi = __float2half_rn(64.0f + (float)z);
  return (uint32_t)__half_as_ushort(lo) | ((uint32_t)__half_as_ushort(hi) << 16);
}
// 4 packed bytes (8 codes) -> 8 binary16 (uint4), codes in memory order
__device__ __forceinline__ uint4 int4x8_dequant(uint32_t w, uint32_t zmagic, uint32_t s2) {
  uint4 o;
  o.x = hmul2_rn(hsub2_rn(int4_pair_magic<0>(w), zmagic), s2);
  o.y = hmul2_rn(hsub2_rn(int4_pair_magic<1>(w), zmagic), s2);
  o.z = hmul2_rn(hsub2_rn(int4_pair_magic<2>(w), zmagic), s2);
  o.w = hmul2_rn(hsub2_rn(int4_pair_magic<3>(w), zmagic), s2);
  return o;
}

// INT8: bytes J and J+1 of w (two int8 codes) -> half2 (1152 + q0, 1152 + q1):
// flipping bit 7 maps q in [-128, 127] to q + 128 in [0, 255], OR-ed into
// the fraction of 1024.
template <int J>
__device__ __forceinline__ uint32_t int8_pair_magic(uint32_t w) {
  constexpr uint32_t sel = (uint32_t)J | 0x40u | ((uint32_t)(J + 1) << 8) | 0x4000u;  // [bJ, 0, bJ+1, 0]
  uint32_t x = __byte_perm(w, 0u, sel);
  uint32_t r;
  asm("lop3.b32 %0, %1, %2, %3, 0x6A;" : "=r"(r) : "r"(x), "r"(0x00FF00FFu), "r"(0x64806480u));  // (a & b) ^ c
  return r;
}
// (1152 + z) in both halves for a signed zero point z in [-128, 127]
__device__ __forceinline__ uint32_t int8_zero_magic(int32_t z) {
  uint32_t h = (uint32_t)__half_as_ushort(__float2half_rn(1152.0f + (float)z));
  return h | (h << 16);
}
// 8 int8 codes (uint2) -> 8 binary16 (uint4)
__device__ __forceinline__ uint4 int8x8_dequant(uint2 w, uint32_t zmagic, uint32_t s2) {
  uint4 o;
  o.x = hmul2_rn(hsub2_rn(int8_pair_magic<0>(w.x), zmagic), s2);
  o.y = hmul2_rn(hsub2_rn(int8_pair_magic<2>(w.x), zmagic), s2);
  o.z = hmul2_rn(hsub2_rn(int8_pair_magic<0>(w.y), zmagic), s2);
  o.w = hmul2_rn(hsub2_rn(int8_pair_magic<2>(w.y), zmagic), s2);
  return o;
}

// scalar reference path on the device (unaligned / ragged cases): the exact
// integer times s in fp32 (exact), then one rounding to binary16.
__device__ __forceinline__ uint16_t dequant_scalar(int32_t q_minus_z, uint16_t s_bits) {
  float s = __half2float(__ushort_as_half(s_bits));
  return __half_as_ushort(__float2half_rn((float)q_minus_z * s));
}

__device__ __forceinline__ uint32_t bcast_half(uint16_t h) { return (uint32_t)h | ((uint32_t)h << 16); }

// ---------------------------------------------------------------------------
// host helpers
// ---------------------------------------------------------------------------
__host__ __device__ inline bool aligned(const void *p, uintptr_t a) { return ((uintptr_t)p & (a - 1)) == 0; }

int num_sms();
// resident blocks per SM of a kernel (cached per kernel and device)
int blocks_per_sm(const void *kernel, int threads, size_t dyn_smem);
lt_status launch_status();
// a CUDA driver API function by name (nullptr if unavailable)
void *driver_fn(const char *name);
// unique id of the calling thread's current CUDA context (false if none):
// a context destroyed and created again (cudaDeviceReset) gets a new id
bool current_context_id(unsigned long long *id);

}  // namespace lt
