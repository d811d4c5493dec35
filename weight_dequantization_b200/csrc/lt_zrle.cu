// lt_zrle.cu -- zero-run decoding of mostly-zero binary16 activations
// ("LoreToken-powered GPU memory layer", compression strategies: zero-run
// encoding for ReLU outputs).
//
// One warp per chunk, no shared memory (so up to 64 warps per SM keep the
// HBM streams busy):
//  1. the chunk's output is zero-filled with 16-byte stores;
//  2. the encoded bytes are read 128 at a time into registers (4 bytes per
//     lane = two 16-bit fields per lane), realigned to the chunk's 16-bit
//     grid with funnel shifts;
//  3. the records are walked in the registers -- each step reads a
//     record's (zero run, literal count) pair with two warp shuffles -- and
//     the lanes holding a record's literals store them to their output
//     positions (L2 merges these with the zero fill before HBM sees them).
// A record whose literals run past the 128-byte window carries over into
// the next window. Every loop is bounded by the chunk's byte range.
#include "lt_common.cuh"

namespace lt {
namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr uint32_t kWin = 128;  // bytes per window = 64 u16 slots, 2 per lane

// aligned 4-byte word at byte address a (a % 4 == 0) of enc; bytes past
// `limit` (the end of the encoded buffer) read as 0
__device__ __forceinline__ uint32_t load_word(const uint8_t *__restrict__ enc, uint64_t a, uint64_t limit) {
  if (a + 4 <= limit) return __ldg(reinterpret_cast<const uint32_t *>(enc + a));
  uint32_t v = 0;
  for (int j = 0; j < 4; ++j)
    if (a + j < limit) v |= (uint32_t)__ldg(enc + a + j) << (8 * j);
  return v;
}

// zero-fill out[0, len)
__device__ __forceinline__ void zero_fill(uint16_t *out, uint32_t len, int lane) {
  uint32_t i0 = 0;
  const uintptr_t mis = reinterpret_cast<uintptr_t>(out) & 15;
  if (mis & 1) {  // not even 2-byte aligned cannot happen (checked on the host)
    for (uint32_t i = lane; i < len; i += 32) out[i] = 0;
    return;
  }
  // elements up to the first 16-byte boundary
  const uint32_t head = mis ? (uint32_t)((16 - mis) / 2) : 0u;
  for (uint32_t i = lane; i < head && i < len; i += 32) out[i] = 0;
  i0 = head < len ? head : len;
  const uint32_t n16 = (len - i0) / 8;
  uint4 *o4 = reinterpret_cast<uint4 *>(out + i0);
  for (uint32_t i = lane; i < n16; i += 32) st_u128(o4 + i, make_uint4(0u, 0u, 0u, 0u));
  for (uint32_t i = i0 + 8 * n16 + lane; i < len; i += 32) out[i] = 0;
}

__global__ void __launch_bounds__(kThreads) k_zrle(const uint8_t *__restrict__ enc, uint64_t enc_bytes,
                                                   const uint64_t *__restrict__ offsets, int64_t n, int32_t chunk,
                                                   int64_t n_chunks, uint16_t *__restrict__ out,
                                                   int32_t *d_status) {
  const int lane = threadIdx.x & 31;
  const int64_t warp_global = (int64_t)blockIdx.x * kWarps + (threadIdx.x >> 5);
  const int64_t warps_total = (int64_t)gridDim.x * kWarps;

  for (int64_t c = warp_global; c < n_chunks; c += warps_total) {
    const int64_t e0 = c * (int64_t)chunk;
    const uint32_t len = (uint32_t)((n - e0) < chunk ? (n - e0) : chunk);
    uint16_t *o = out + e0;
    zero_fill(o, len, lane);
    __syncwarp();  // the literal stores below land after the zero fill

    const uint64_t b0 = offsets[c], b1 = offsets[c + 1];
    if (b1 < b0 || b1 > enc_bytes) {
      if (lane == 0) report(d_status, LT_ERR_CORRUPT_STREAM);
      continue;
    }
    const uint64_t nbytes = b1 - b0;  // the chunk's bytes
    uint32_t done = 0;                // elements produced
    uint64_t q = 0;                   // byte offset of the window in the chunk (even)
    uint32_t p = 0;                   // next record start, in 16-bit slots from q
    uint32_t lit_rem = 0, lit_out = 0;  // literals carried over from the previous window
    int err = 0;
    // every iteration moves q forward by at least 4 bytes: bounded by nbytes
    while (done < len || lit_rem) {
      if (q >= nbytes) {
        err = LT_ERR_SIZE_MISMATCH;
        break;
      }
      // window: chunk bytes [q, q + 128) as 64 u16 slots; lane l holds slots
      // 2l (low half) and 2l + 1 (high half)
      const uint64_t A = b0 + q;  // absolute byte index of slot 0
      const uint64_t al = A & ~uint64_t(3);
      const uint32_t sh = (uint32_t)(A & 3) * 8;
      const uint32_t w0 = load_word(enc, al + 4 * (uint64_t)lane, enc_bytes);
      const uint32_t w33 = (lane == 31) ? load_word(enc, al + 128, enc_bytes) : 0u;
      uint32_t w1 = __shfl_down_sync(0xFFFFFFFFu, w0, 1);
      if (lane == 31) w1 = w33;
      const uint32_t pair = __funnelshift_r(w0, w1, sh);  // slots 2*lane, 2*lane + 1
      // slots that exist in the chunk's bytes
      const uint64_t win_bytes = (nbytes - q) < kWin ? (nbytes - q) : kWin;
      const uint32_t win_slots = (uint32_t)(win_bytes / 2);

      // 1. literals carried over from a record that began in an earlier window
      if (lit_rem) {
        const uint32_t take = lit_rem < win_slots ? lit_rem : win_slots;
        for (int h = 0; h < 2; ++h) {
          const uint32_t s = 2 * (uint32_t)lane + h;
          if (s < take) o[lit_out + s] = (uint16_t)(h ? (pair >> 16) : (pair & 0xFFFFu));
        }
        lit_rem -= take;
        lit_out += take;
        if (lit_rem) {  // the whole window was literals
          if (win_slots < 64) {
            err = LT_ERR_CORRUPT_STREAM;
            break;
          }
          q += kWin;
          p -= 64;
          continue;
        }
      }
      // 2. records starting in this window (header fully inside it)
      while (done < len && p + 1 < 64) {
        if (p + 1 >= win_slots) {  // the chunk's bytes end before the next header: too few records
          err = LT_ERR_SIZE_MISMATCH;
          break;
        }
        const uint32_t zp = __shfl_sync(0xFFFFFFFFu, pair, p >> 1);
        const uint32_t np = __shfl_sync(0xFFFFFFFFu, pair, (p + 1) >> 1);
        const uint32_t zrun = (p & 1) ? (zp >> 16) : (zp & 0xFFFFu);
        const uint32_t nlit = ((p + 1) & 1) ? (np >> 16) : (np & 0xFFFFu);
        if ((uint64_t)done + zrun + nlit > len || q + 2 * ((uint64_t)p + 2 + nlit) > nbytes) {
          err = LT_ERR_CORRUPT_STREAM;
          break;
        }
        done += zrun;
        const uint32_t ls = p + 2;  // first literal slot
        for (int h = 0; h < 2; ++h) {
          const uint32_t s = 2 * (uint32_t)lane + h;
          if (s >= ls && s < ls + nlit && s < 64) o[done + (s - ls)] = (uint16_t)(h ? (pair >> 16) : (pair & 0xFFFFu));
        }
        if (ls + nlit > 64) {  // literals continue in the next window(s)
          const uint32_t in_win = ls < 64 ? 64 - ls : 0u;
          lit_rem = nlit - in_win;
          lit_out = done + in_win;
        }
        done += nlit;
        p = ls + nlit;
      }
      if (err) break;
      if (done >= len && !lit_rem) break;
      // next window: at the next record's header (or past the carried literals)
      if (p < 64) {
        q += 2 * (uint64_t)p;
        p = 0;
      } else {
        q += kWin;
        p -= 64;
      }
    }
    if (err && lane == 0) report(d_status, err);
  }
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
  const int64_t need = (n_chunks + kWarps - 1) / kWarps;
  const int64_t cap = (int64_t)num_sms() * blocks_per_sm((const void *)k_zrle, kThreads, 0);
  const int grid = (int)(need < cap ? need : cap);
  k_zrle<<<grid, kThreads, 0, st>>>(enc, enc_bytes, chunk_offsets, n_elements, chunk_elems, n_chunks, out,
                                    d_status);
  return launch_status();
}
