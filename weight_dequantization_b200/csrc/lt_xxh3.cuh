// lt_xxh3.cuh -- the 64-bit XXH3 hash (xxHash 0.8) with a caller-given
// secret and seed 0, as one sequential function over a byte range, for the
// per-block checksums of an HCT v2 container ("GPU Compression Pipeline -
// TDD Roadmap", Phase 6.1 HCT Format V2: XXH3 checksum support).
//
// The input is cut by length into the classes 0, 1-3, 4-8, 9-16, 17-128,
// 129-240 and longer. Short classes mix a few input words with secret words;
// longer inputs run 8 accumulators over 64-byte stripes, the secret
// advancing 8 bytes per stripe, scrambled after every (secret_len - 64) / 8
// stripes, then merged. All arithmetic is modulo 2^64 on little-endian
// words; every read stays inside [in, in + len) and [sec, sec + sec_len)
// for sec_len >= 136.
#pragma once

#include <stdint.h>

#ifdef __CUDACC__
#define LT_HD __host__ __device__ __forceinline__
#else
#define LT_HD inline
#endif

namespace lt {
namespace xxh3 {

constexpr uint64_t kP32_1 = 0x9E3779B1u, kP32_2 = 0x85EBCA77u, kP32_3 = 0xC2B2AE3Du;
constexpr uint64_t kP64_1 = 0x9E3779B185EBCA87ull, kP64_2 = 0xC2B2AE3D27D4EB4Full, kP64_3 = 0x165667B19E3779F9ull;
constexpr uint64_t kP64_4 = 0x85EBCA77C2B2AE63ull, kP64_5 = 0x27D4EB2F165667C5ull;
constexpr uint64_t kMx1 = 0x165667919E3779F9ull, kMx2 = 0x9FB21C651E98DF25ull;
constexpr uint32_t kSecretMin = 136;

// byte loads: the ranges start at any byte
LT_HD uint64_t rd64(const uint8_t *p) {
  uint64_t v = 0;
#pragma unroll
  for (int i = 0; i < 8; ++i) v |= (uint64_t)p[i] << (8 * i);
  return v;
}
LT_HD uint32_t rd32(const uint8_t *p) {
  return (uint32_t)p[0] | ((uint32_t)p[1] << 8) | ((uint32_t)p[2] << 16) | ((uint32_t)p[3] << 24);
}
LT_HD uint64_t rotl(uint64_t x, int r) { return (x << r) | (x >> (64 - r)); }
LT_HD uint64_t swap64(uint64_t x) {
  x = ((x & 0x00FF00FF00FF00FFull) << 8) | ((x >> 8) & 0x00FF00FF00FF00FFull);
  x = ((x & 0x0000FFFF0000FFFFull) << 16) | ((x >> 16) & 0x0000FFFF0000FFFFull);
  return (x << 32) | (x >> 32);
}
// low and high halves of the 128-bit product, XORed
LT_HD uint64_t mul_fold(uint64_t a, uint64_t b) {
#ifdef __CUDA_ARCH__
  return (a * b) ^ __umul64hi(a, b);
#else
  const unsigned __int128 p = (unsigned __int128)a * b;
  return (uint64_t)p ^ (uint64_t)(p >> 64);
#endif
}
LT_HD uint64_t avalanche64(uint64_t h) {
  h ^= h >> 33;
  h *= kP64_2;
  h ^= h >> 29;
  h *= kP64_3;
  return h ^ (h >> 32);
}
LT_HD uint64_t avalanche3(uint64_t h) {
  h ^= h >> 37;
  h *= kMx1;
  return h ^ (h >> 32);
}
LT_HD uint64_t rrmxmx(uint64_t h, uint64_t len) {
  h ^= rotl(h, 49) ^ rotl(h, 24);
  h *= kMx2;
  h ^= (h >> 35) + len;
  h *= kMx2;
  return h ^ (h >> 28);
}
LT_HD uint64_t mix16(const uint8_t *in, const uint8_t *sec) {
  return mul_fold(rd64(in) ^ rd64(sec), rd64(in + 8) ^ rd64(sec + 8));
}
LT_HD void stripe(uint64_t acc[8], const uint8_t *in, const uint8_t *sec) {
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const uint64_t v = rd64(in + 8 * i);
    const uint64_t k = v ^ rd64(sec + 8 * i);
    acc[i ^ 1] += v;
    acc[i] += (k & 0xFFFFFFFFull) * (k >> 32);
  }
}

LT_HD uint64_t hash64(const uint8_t *in, uint64_t len, const uint8_t *sec, uint64_t sec_len) {
  if (len == 0) return avalanche64(rd64(sec + 56) ^ rd64(sec + 64));
  if (len <= 3) {
    const uint32_t c = ((uint32_t)in[0] << 16) | ((uint32_t)in[len >> 1] << 24) | (uint32_t)in[len - 1] |
                       ((uint32_t)len << 8);
    return avalanche64((uint64_t)c ^ (uint64_t)(rd32(sec) ^ rd32(sec + 4)));
  }
  if (len <= 8) {
    const uint64_t v = (uint64_t)rd32(in + len - 4) | ((uint64_t)rd32(in) << 32);
    return rrmxmx(v ^ (rd64(sec + 8) ^ rd64(sec + 16)), len);
  }
  if (len <= 16) {
    const uint64_t lo = rd64(in) ^ rd64(sec + 24) ^ rd64(sec + 32);
    const uint64_t hi = rd64(in + len - 8) ^ rd64(sec + 40) ^ rd64(sec + 48);
    return avalanche3(len + swap64(lo) + hi + mul_fold(lo, hi));
  }
  if (len <= 128) {
    uint64_t acc = len * kP64_1;
    if (len > 32) {
      if (len > 64) {
        if (len > 96) {
          acc += mix16(in + 48, sec + 96);
          acc += mix16(in + len - 64, sec + 112);
        }
        acc += mix16(in + 32, sec + 64);
        acc += mix16(in + len - 48, sec + 80);
      }
      acc += mix16(in + 16, sec + 32);
      acc += mix16(in + len - 32, sec + 48);
    }
    acc += mix16(in, sec);
    acc += mix16(in + len - 16, sec + 16);
    return avalanche3(acc);
  }
  if (len <= 240) {
    uint64_t acc = len * kP64_1;
    for (int i = 0; i < 8; ++i) acc += mix16(in + 16 * i, sec + 16 * i);
    acc = avalanche3(acc);
    const int rounds = (int)(len / 16);
    for (int i = 8; i < rounds; ++i) acc += mix16(in + 16 * i, sec + 16 * (i - 8) + 3);
    acc += mix16(in + len - 16, sec + kSecretMin - 17);
    return avalanche3(acc);
  }
  uint64_t acc[8] = {kP32_3, kP64_1, kP64_2, kP64_3, kP64_4, kP32_2, kP64_5, kP32_1};
  const uint64_t per_block = (sec_len - 64) / 8;  // stripes between scrambles
  const uint64_t block_len = 64 * per_block;
  const uint64_t n_blocks = (len - 1) / block_len;
  const uint8_t *scr = sec + sec_len - 64;
  for (uint64_t b = 0; b < n_blocks; ++b) {
    for (uint64_t s = 0; s < per_block; ++s) stripe(acc, in + b * block_len + 64 * s, sec + 8 * s);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      uint64_t a = acc[i];
      a ^= a >> 47;
      a ^= rd64(scr + 8 * i);
      acc[i] = a * kP32_1;
    }
  }
  const uint64_t tail = ((len - 1) - block_len * n_blocks) / 64;
  for (uint64_t s = 0; s < tail; ++s) stripe(acc, in + n_blocks * block_len + 64 * s, sec + 8 * s);
  stripe(acc, in + len - 64, sec + sec_len - 64 - 7);
  uint64_t h = len * kP64_1;
#pragma unroll
  for (int i = 0; i < 4; ++i) h += mul_fold(acc[2 * i] ^ rd64(sec + 11 + 16 * i), acc[2 * i + 1] ^ rd64(sec + 19 + 16 * i));
  return avalanche3(h);
}

#ifdef __CUDACC__
// ---------------------------------------------------------------------------
// The long class (len > 240) computed by one warp. Within one scramble
// interval the accumulator updates of the stripes are plain sums modulo
// 2^64, so they can be split among lanes and added up: lane l takes the
// 8-byte word i = l % 8 of stripes l / 8, l / 8 + 4, ...; a butterfly over
// the four lanes with the same i adds their terms; acc[i] takes its product
// terms and the data terms of word i ^ 1 (one shuffle). The scramble, the
// tail stripes, the last stripe and the merge then follow the sequential
// definition above, each lane holding acc[l % 8]. `rd(off)` returns the 8
// input bytes at offset off (little-endian, any alignment); `rk(off)` the 8
// secret bytes at offset off. Every lane returns the hash.
// ---------------------------------------------------------------------------

// the initial accumulator i: kP32_3, kP64_1, kP64_2, kP64_3, kP64_4, kP32_2, kP64_5, kP32_1
__device__ __forceinline__ uint64_t acc_init(int i) {
  return (i & 4) ? ((i & 2) ? ((i & 1) ? kP32_1 : kP64_5) : ((i & 1) ? kP32_2 : kP64_4))
                 : ((i & 2) ? ((i & 1) ? kP64_3 : kP64_2) : ((i & 1) ? kP64_1 : kP32_3));
}

// what stripes [0, ns) starting at input offset base (stripe s keyed at
// secret offset key0 + 8 s) add to acc[lane % 8]; every lane returns its sum
template <typename RD, typename RK>
__device__ __forceinline__ uint64_t stripe_terms(RD &rd, RK &rk, uint64_t base, uint64_t ns, uint64_t key0,
                                                 int lane) {
  const uint64_t i = (uint64_t)(lane & 7);
  uint64_t m = 0, d = 0;
  for (uint64_t st = (uint64_t)(lane >> 3); st < ns; st += 4) {
    const uint64_t v = rd(base + 64 * st + 8 * i);
    const uint64_t k = v ^ rk(key0 + 8 * st + 8 * i);
    d += v;
    m += (k & 0xFFFFFFFFull) * (k >> 32);
  }
  m += __shfl_xor_sync(0xFFFFFFFFu, m, 8);
  m += __shfl_xor_sync(0xFFFFFFFFu, m, 16);
  d += __shfl_xor_sync(0xFFFFFFFFu, d, 8);
  d += __shfl_xor_sync(0xFFFFFFFFu, d, 16);
  return m + __shfl_xor_sync(0xFFFFFFFFu, d, 1);
}

__device__ __forceinline__ uint64_t scramble(uint64_t acc, uint64_t scr) {
  acc ^= acc >> 47;
  acc ^= scr;
  return acc * kP32_1;
}

// tail stripes, last stripe and merge, after the n_blocks full scramble
// intervals have been added into acc (lane l holds acc[l % 8])
template <typename RD, typename RK>
__device__ __forceinline__ uint64_t finish_long(RD &rd, RK &rk, uint64_t acc, uint64_t len, uint64_t sec_len,
                                                uint64_t n_blocks, int lane) {
  const uint64_t block_len = 64 * ((sec_len - 64) / 8);
  acc += stripe_terms(rd, rk, n_blocks * block_len, ((len - 1) - block_len * n_blocks) / 64, 0, lane);
  acc += stripe_terms(rd, rk, len - 64, 1, sec_len - 64 - 7, lane);
  // merge: term j (lanes 0..3) from acc[2j] and acc[2j + 1]
  const uint64_t a_even = __shfl_sync(0xFFFFFFFFu, acc, (2 * lane) & 7);
  const uint64_t a_odd = __shfl_sync(0xFFFFFFFFu, acc, (2 * lane + 1) & 7);
  uint64_t t = lane < 4 ? mul_fold(a_even ^ rk(11 + 16 * (uint64_t)lane), a_odd ^ rk(19 + 16 * (uint64_t)lane)) : 0;
  t += __shfl_xor_sync(0xFFFFFFFFu, t, 1);
  t += __shfl_xor_sync(0xFFFFFFFFu, t, 2);
  return avalanche3(len * kP64_1 + __shfl_sync(0xFFFFFFFFu, t, 0));
}

template <typename RD, typename RK>
__device__ __forceinline__ uint64_t hash64_long_warp(RD rd, RK rk, uint64_t len, uint64_t sec_len, int lane) {
  uint64_t acc = acc_init(lane & 7);
  const uint64_t per_block = (sec_len - 64) / 8;
  const uint64_t block_len = 64 * per_block;
  const uint64_t n_blocks = (len - 1) / block_len;
  const uint64_t scr = rk(sec_len - 64 + 8 * (uint64_t)(lane & 7));
  for (uint64_t b = 0; b < n_blocks; ++b) acc = scramble(acc + stripe_terms(rd, rk, b * block_len, per_block, 0, lane), scr);
  return finish_long(rd, rk, acc, len, sec_len, n_blocks, lane);
}
#endif

}  // namespace xxh3
}  // namespace lt
