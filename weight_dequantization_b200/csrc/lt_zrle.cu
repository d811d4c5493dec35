// lt_zrle.cu -- zero-run decoding of mostly-zero binary16 activations
// ("LoreToken-powered GPU memory layer", compression strategies: zero-run
// encoding for ReLU outputs).
//
// The work of a chunk is a serial walk over its records (where a record's
// header sits depends on every literal count before it) plus a dense fp16
// output that is mostly zeros. So each LANE walks one chunk, and each warp
// writes its 32 chunks' output together:
//  - lane l of a warp owns chunk 32 w + l and a 256-element stripe tile in
//    shared memory that starts out zero;
//  - round r: every lane walks its records until its output position reaches
//    the end of stripe r of its chunk, skipping zero runs (the tile is
//    already zero) and writing literals into its tile; a zero run or literal
//    run that crosses the stripe end carries over to the next round;
//  - then the warp stores the 32 stripes one after the other, each as 32
//    16-byte pieces (512 contiguous bytes per store instruction), zeroing the
//    tile behind it.
// So a record costs a few instructions of one lane (32 chunks walk side by
// side) and the output leaves with fully coalesced 16-byte stores. Every
// walk is bounded by its chunk's bytes; the checks are the oracle's, in its
// order.
#include "lt_common.cuh"

namespace lt {
namespace {

constexpr int kZWarps = 2;                 // warps per CTA (33 KB of tiles: six CTAs per SM)
constexpr int kZThreads = kZWarps * 32;
constexpr uint32_t kStripe = 256;          // elements per stripe
constexpr uint32_t kPitch = 2 * kStripe + 16;  // bytes per lane tile (padded: lanes' tiles start on different banks)

// the little-endian u16 at chunk byte p (the chunk may start at an odd address)
__device__ __forceinline__ uint32_t rd16(const uint8_t *__restrict__ base, uint64_t p, bool even) {
  if (even) {
    uint16_t v;
    asm volatile("ld.global.nc.u16 %0, [%1];" : "=h"(v) : "l"(base + p));
    return v;
  }
  return (uint32_t)__ldg(base + p) | ((uint32_t)__ldg(base + p + 1) << 8);
}

// A lane's sequential reader over its chunk: three aligned 16-byte windows in
// registers, the two after the current one loaded ahead of use, so a lane
// issues one 16-byte load per 16 bytes it consumes (not one per field) and
// its next loads are in flight while it works. Windows that reach outside
// the encoded buffer are read byte by byte, inside it only.
struct LaneReader {
  uintptr_t lo, hi;  // the encoded buffer [enc, enc + enc_bytes)
  uintptr_t wb;      // address of window 0 (16-byte aligned)
  uint4 w0, w1, w2;
  __device__ __forceinline__ uint4 load(uintptr_t a) const {
    if (a >= lo && a + 16 <= hi) return ld_stream_u128(reinterpret_cast<const void *>(a));
    uint32_t b0 = 0, b1 = 0, b2 = 0, b3 = 0;
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      const uintptr_t x = a + (uintptr_t)i;
      const uint32_t v = (x >= lo && x < hi) ? (uint32_t)__ldg(reinterpret_cast<const uint8_t *>(x)) : 0u;
      const uint32_t sh = 8u * (uint32_t)(i & 3);
      if (i < 4) b0 |= v << sh;
      else if (i < 8) b1 |= v << sh;
      else if (i < 12) b2 |= v << sh;
      else b3 |= v << sh;
    }
    return make_uint4(b0, b1, b2, b3);
  }
  __device__ __forceinline__ void start(uintptr_t a) {
    wb = a & ~uintptr_t(15);
    w0 = load(wb);
    w1 = load(wb + 16);
    w2 = load(wb + 32);
  }
  // the little-endian u16 at even address a (a >= the current window)
  __device__ __forceinline__ uint32_t get16(uintptr_t a) {
    uintptr_t off = a - wb;
    if (off >= 48) {  // a jump past the windows held (a long literal run): start again there
      start(a);
      off = a - wb;
    }
    while (off >= 16) {
      w0 = w1;
      w1 = w2;
      w2 = load(wb + 48);
      wb += 16;
      off -= 16;
    }
    const uint32_t word = (off & 8) ? ((off & 4) ? w0.w : w0.z) : ((off & 4) ? w0.y : w0.x);
    return (off & 2) ? (word >> 16) : (word & 0xFFFFu);
  }
};

template <bool VEC>
__global__ void __launch_bounds__(kZThreads) k_zrle(const uint8_t *__restrict__ enc, uint64_t enc_bytes,
                                                      const uint64_t *__restrict__ offsets, int64_t n, int32_t chunk,
                                                      int64_t n_chunks, uint16_t *__restrict__ out,
                                                      int32_t *d_status) {
  __shared__ __align__(16) uint8_t tiles[kZWarps][32 * kPitch];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  uint8_t *wt = tiles[warp];
  uint16_t *mine = reinterpret_cast<uint16_t *>(wt + lane * kPitch);
  const int64_t c0 = ((int64_t)blockIdx.x * kZWarps + warp) * 32;  // the warp's first chunk
  const int64_t c = c0 + lane;

  for (uint32_t i = (uint32_t)lane; i < 32 * kPitch / 16; i += 32)
    reinterpret_cast<uint4 *>(wt)[i] = make_uint4(0u, 0u, 0u, 0u);

  // this lane's chunk
  uint32_t len = 0;
  uint64_t b0 = 0, nb = 0;
  int err = 0;
  if (c < n_chunks) {
    const int64_t e0 = c * (int64_t)chunk;
    len = (uint32_t)((n - e0) < chunk ? (n - e0) : chunk);
    b0 = offsets[c];
    const uint64_t b1 = offsets[c + 1];
    if (b1 < b0 || b1 > enc_bytes) err = LT_ERR_CORRUPT_STREAM;
    else nb = b1 - b0;
  }
  const uint8_t *src = enc + b0;
  const bool even = ((reinterpret_cast<uintptr_t>(src)) & 1) == 0;
  LaneReader rdr;
  rdr.lo = reinterpret_cast<uintptr_t>(enc);
  rdr.hi = reinterpret_cast<uintptr_t>(enc) + enc_bytes;
  if (even && nb) rdr.start(reinterpret_cast<uintptr_t>(src));
  // the u16 at chunk byte q: through the window reader, or byte by byte for
  // a chunk at an odd address
  auto field = [&](uint64_t q) -> uint32_t {
    return even ? rdr.get16(reinterpret_cast<uintptr_t>(src) + (uintptr_t)q) : rd16(src, q, false);
  };
  uint64_t p = 0;          // next unread byte of the chunk
  uint32_t pos = 0;        // elements produced
  uint32_t zrem = 0, lrem = 0;  // zeros / literals of the current record still to produce
  uint64_t lsrc = 0;       // byte of the next literal
  bool walking = err == 0 && len > 0;
  const uint32_t stripes = (len + kStripe - 1) / kStripe;
  const uint32_t rounds = __reduce_max_sync(0xFFFFFFFFu, stripes);
  __syncwarp();

  for (uint32_t r = 0; r < rounds; ++r) {
    const uint32_t s0 = r * kStripe;
    const uint32_t s_end = (s0 + kStripe) < len ? (s0 + kStripe) : len;
    // 1. walk this lane's records up to the end of its stripe r
    while (walking && pos < s_end) {
      if (zrem) {  // zeros: the tile is zero already
        const uint32_t t = zrem < s_end - pos ? zrem : s_end - pos;
        pos += t;
        zrem -= t;
        if (zrem) break;
      }
      if (lrem) {
        const uint32_t t = lrem < s_end - pos ? lrem : s_end - pos;
        for (uint32_t i = 0; i < t; ++i) mine[pos - s0 + i] = (uint16_t)field(lsrc + 2 * i);
        lsrc += 2 * (uint64_t)t;
        pos += t;
        lrem -= t;
        if (lrem) break;
      }
      if (pos >= len) {
        walking = false;
        break;
      }
      if (pos >= s_end) break;
      // the next record's header (the oracle's checks, in its order)
      if (p + 4 > nb) {
        err = LT_ERR_SIZE_MISMATCH;
        walking = false;
        break;
      }
      const uint32_t zr = field(p);
      const uint32_t nl = field(p + 2);
      p += 4;
      if ((uint64_t)pos + zr + nl > len || p + 2 * (uint64_t)nl > nb) {
        err = LT_ERR_CORRUPT_STREAM;
        walking = false;
        break;
      }
      zrem = zr;
      lrem = nl;
      lsrc = p;
      p += 2 * (uint64_t)nl;
    }
    __syncwarp();
    // 2. the warp stores stripe r of each of its 32 chunks: 32 x 16 bytes each
    for (int j = 0; j < 32; ++j) {
      const uint32_t len_j = __shfl_sync(0xFFFFFFFFu, len, j);
      if (s0 >= len_j) continue;  // warp-uniform
      const uint32_t m = (len_j - s0) < kStripe ? (len_j - s0) : kStripe;
      uint16_t *dst = out + (c0 + j) * (int64_t)chunk + s0;
      uint4 *tv = reinterpret_cast<uint4 *>(wt + j * kPitch) + lane;
      const uint32_t e = 8 * (uint32_t)lane;
      if (e < m) {
        const uint4 v = *tv;
        if (VEC && e + 8 <= m) {
          st_u128(dst + e, v);
        } else {
          const uint16_t *h = reinterpret_cast<const uint16_t *>(&v);
          for (uint32_t q = 0; q < 8 && e + q < m; ++q) dst[e + q] = h[q];
        }
        *tv = make_uint4(0u, 0u, 0u, 0u);
      }
    }
    __syncwarp();
  }
  if (err) report(d_status, err);
}

}  // namespace
}  // namespace lt

using namespace lt;

LT_API lt_status lt_zrle_decode(const uint8_t *enc, uint64_t enc_bytes, const uint64_t *chunk_offsets,
                                int64_t n_elements, int32_t chunk_elems, lt_half *out, int32_t *d_status,
                                lt_stream_t stream) {
  if (n_elements < 0) return LT_ERR_INVALID_ARG;
  if (chunk_elems < 1 || chunk_elems > 65535) return LT_ERR_UNSUPPORTED;
  if (n_elements == 0) return LT_OK;
  if (!chunk_offsets || !out || (!enc && enc_bytes != 0)) return LT_ERR_INVALID_ARG;
  if (!aligned(chunk_offsets, 8) || !aligned(out, 2) || !aligned(d_status, 4)) return LT_ERR_MISALIGNED;
  cudaStream_t st = (cudaStream_t)stream;
  const int64_t n_chunks = (n_elements + chunk_elems - 1) / chunk_elems;
  const int64_t grid = (n_chunks + kZThreads - 1) / kZThreads;  // one chunk per lane
  if (grid > INT32_MAX) return LT_ERR_UNSUPPORTED;
  // 16-byte stores when every chunk's output starts on a 16-byte boundary
  if (aligned(out, 16) && chunk_elems % 8 == 0)
    k_zrle<true><<<(int)grid, kZThreads, 0, st>>>(enc, enc_bytes, chunk_offsets, n_elements, chunk_elems, n_chunks,
                                                  out, d_status);
  else
    k_zrle<false><<<(int)grid, kZThreads, 0, st>>>(enc, enc_bytes, chunk_offsets, n_elements, chunk_elems, n_chunks,
                                                   out, d_status);
  return launch_status();
}
