// lt_zrle.cu -- zero-run decoding of mostly-zero binary16 activations
// ("LoreToken-powered GPU memory layer", compression strategies: zero-run
// encoding for ReLU outputs).
//
// One warp per chunk, no shared memory (so up to 64 warps per SM keep the
// HBM streams busy):
//  1. the chunk's output is zero-filled with 16-byte stores;
//  2. the encoded bytes are read 128 at a time into registers (two 16-bit
//     fields per lane), realigned to the chunk's 16-bit grid with funnel
//     shifts;
//  3. in each window the warp walks the record chain -- one shuffle per
//     record reads its (zero run, literal count) -- and parks record k's
//     position and header in lane k; then all records of the window are
//     finished in parallel: a warp scan gives each record's output offset,
//     a vote finds the first bad record (the oracle's checks, in its order),
//     and every lane stores the literals it holds (L2 merges them with the
//     zero fill before HBM sees them).
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

__global__ void __launch_bounds__(kThreads, 6) k_zrle(const uint8_t *__restrict__ enc, uint64_t enc_bytes,
                                                   const uint64_t *__restrict__ offsets, int64_t n, int32_t chunk,
                                                   int64_t n_chunks, uint16_t *__restrict__ out,
                                                   int32_t *d_status) {
  const uint32_t lane = threadIdx.x & 31;
  const int64_t warp_global = (int64_t)blockIdx.x * kWarps + (threadIdx.x >> 5);
  const int64_t warps_total = (int64_t)gridDim.x * kWarps;

  for (int64_t c = warp_global; c < n_chunks; c += warps_total) {
    const int64_t e0 = c * (int64_t)chunk;
    const uint32_t len = (uint32_t)((n - e0) < chunk ? (n - e0) : chunk);
    uint16_t *o = out + e0;
    zero_fill(o, len, (int)lane);
    __syncwarp();  // the literal stores below land after the zero fill

    const uint64_t b0 = offsets[c], b1 = offsets[c + 1];
    if (b1 < b0 || b1 > enc_bytes) {
      if (lane == 0) report(d_status, LT_ERR_CORRUPT_STREAM);
      continue;
    }
    const uint64_t nbytes = b1 - b0;  // the chunk's bytes
    uint32_t done = 0;                // elements accounted for (zero runs and literals)
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
      // 2l, 2l + 1 in `pair` and slots 2l + 1, 2l + 2 in `podd`
      const uint64_t A = b0 + q;  // absolute byte index of slot 0
      const uint64_t al = A & ~uint64_t(3);
      const uint32_t sh = (uint32_t)(A & 3) * 8;
      const uint32_t w0 = load_word(enc, al + 4 * (uint64_t)lane, enc_bytes);
      const uint32_t w33 = (lane == 31) ? load_word(enc, al + 128, enc_bytes) : 0u;
      const uint32_t w34 = (lane == 31) ? load_word(enc, al + 132, enc_bytes) : 0u;
      uint32_t w1 = __shfl_down_sync(0xFFFFFFFFu, w0, 1);
      if (lane == 31) w1 = w33;
      const uint32_t pair = __funnelshift_r(w0, w1, sh);  // slots 2*lane, 2*lane + 1
      uint32_t pnext = __shfl_down_sync(0xFFFFFFFFu, pair, 1);
      if (lane == 31) pnext = __funnelshift_r(w33, w34, sh);  // slots 64, 65
      const uint32_t podd = __funnelshift_r(pair, pnext, 16);  // slots 2*lane + 1, 2*lane + 2
      const uint64_t win_bytes = (nbytes - q) < kWin ? (nbytes - q) : kWin;
      const uint32_t win_slots = (uint32_t)(win_bytes / 2);

      // 1. literals carried over from a record that began in an earlier window
      if (lit_rem) {
        const uint32_t take = lit_rem < win_slots ? lit_rem : win_slots;
        for (int h = 0; h < 2; ++h) {
          const uint32_t s = 2 * lane + h;
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
      // 2. walk the records whose header lies in this window and in the
      //    chunk's bytes, until the chunk is accounted for; record k's slot
      //    and header go to lane k
      const int32_t lim = nbytes >= q + 4 ? (int32_t)((nbytes - q - 4) / 2 < 62 ? (nbytes - q - 4) / 2 : 62) : -1;
      const uint32_t rem = len - done;
      // Record r of the window (at most 32: each takes >= 2 slots) goes to
      // lane r by pointer jumping instead of a serial walk: for every slot s,
      // the next record would start at nxt(s) = s + 2 + n_lit(s); jump[b]
      // holds nxt^(2^b) for this lane's slots 2 lane and 2 lane + 1 (low and
      // high halves; positions past the window saturate at 64), and lane r
      // follows the binary digits of r from p.
      uint32_t jump[5];
      jump[0] = min(2 * lane + 2 + (pair >> 16), 64u) | (min(2 * lane + 3 + (podd >> 16), 64u) << 16);
#pragma unroll
      for (int b = 1; b < 5; ++b) {
        const uint32_t q0 = jump[b - 1] & 0xFFFFu, q1 = jump[b - 1] >> 16;
        const uint32_t t0 = __shfl_sync(0xFFFFFFFFu, jump[b - 1], (int)(q0 < 64 ? q0 >> 1 : 0));
        const uint32_t t1 = __shfl_sync(0xFFFFFFFFu, jump[b - 1], (int)(q1 < 64 ? q1 >> 1 : 0));
        const uint32_t r0 = q0 < 64 ? ((q0 & 1) ? t0 >> 16 : t0 & 0xFFFFu) : 64u;
        const uint32_t r1 = q1 < 64 ? ((q1 & 1) ? t1 >> 16 : t1 & 0xFFFFu) : 64u;
        jump[b] = r0 | (r1 << 16);
      }
      uint32_t myP = p < 64 ? p : 64u;
#pragma unroll
      for (int b = 0; b < 5; ++b) {
        const uint32_t t = __shfl_sync(0xFFFFFFFFu, jump[b], (int)(myP < 64 ? myP >> 1 : 0));
        const uint32_t nx = myP < 64 ? ((myP & 1) ? t >> 16 : t & 0xFFFFu) : 64u;
        if ((lane >> b) & 1) myP = nx;
      }
      const uint32_t vsrc = myP < 64 ? myP >> 1 : 0;
      const uint32_t vp = __shfl_sync(0xFFFFFFFFu, pair, (int)vsrc), vo = __shfl_sync(0xFFFFFFFFu, podd, (int)vsrc);
      const bool inwin = (int32_t)myP <= lim;  // a header in the window and in the chunk's bytes
      uint32_t myV = inwin ? ((myP & 1) ? vo : vp) : 0u;
      // the records before the chunk is full (the serial walk's stop rule)
      const uint32_t lk0 = (myV & 0xFFFFu) + (myV >> 16);
      uint32_t incl = lk0;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const uint32_t t = __shfl_up_sync(0xFFFFFFFFu, incl, off);
        if ((int)lane >= off) incl += t;
      }
      const unsigned validm = __ballot_sync(0xFFFFFFFFu, inwin && incl - lk0 < rem);
      const uint32_t k = (~validm) ? (uint32_t)(__ffs(~validm) - 1) : 32u;  // leading valid records
      uint32_t dsum = 0, pp = p;
      if (k) {
        dsum = __shfl_sync(0xFFFFFFFFu, incl, (int)k - 1);
        const uint32_t lp = __shfl_sync(0xFFFFFFFFu, myP, (int)k - 1), lv = __shfl_sync(0xFFFFFFFFu, myV, (int)k - 1);
        pp = lp + 2 + (lv >> 16);
      }
      // 3. the walked records, in parallel
      const bool rec = lane < k;
      if (!rec) myV = 0;
      const uint32_t zr = myV & 0xFFFFu, nl = myV >> 16;
      const uint32_t lk = rec ? zr + nl : 0u;
      const uint32_t before = incl - lk0;  // elements of the window's earlier records
      const bool bad = rec && ((uint64_t)done + before + lk > len || q + 2 * ((uint64_t)myP + 2 + nl) > nbytes);
      const unsigned badm = __ballot_sync(0xFFFFFFFFu, bad);
      const uint32_t ok = badm ? (uint32_t)(__ffs(badm) - 1) : k;  // records before the first bad one
      const bool live = lane < ok;
      const uint32_t mlo = __reduce_or_sync(0xFFFFFFFFu, live && myP < 32 ? 1u << myP : 0u);
      const uint32_t mhi = __reduce_or_sync(0xFFFFFFFFu, live && myP >= 32 ? 1u << (myP - 32) : 0u);
      const uint32_t lend = myP + 2 + nl < 64 ? myP + 2 + nl : 64u;
      const uint32_t span = (myP + 2) | (lend << 16);     // the record's literal slots in this window
      const uint32_t obase = done + before + zr - (myP + 2);  // output index of literal slot s: obase + s
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const uint32_t s = 2 * lane + h;  // the slot this lane holds
        const uint32_t cnt = __popc(mlo & (s >= 31 ? 0xFFFFFFFFu : (2u << s) - 1u)) +
                             (s >= 32 ? __popc(mhi & (s == 63 ? 0xFFFFFFFFu : (2u << (s - 32)) - 1u)) : 0);
        const int r = cnt ? (int)cnt - 1 : 0;  // the last record starting at or before s
        const uint32_t sp = __shfl_sync(0xFFFFFFFFu, span, r);
        const uint32_t ob = __shfl_sync(0xFFFFFFFFu, obase, r);
        if (cnt && s >= (sp & 0xFFFFu) && s < (sp >> 16)) o[ob + s] = (uint16_t)(h ? (pair >> 16) : (pair & 0xFFFFu));
      }
      if (badm) {
        err = LT_ERR_CORRUPT_STREAM;
        break;
      }
      // 4. carry-over from the window's last record, and the next window
      if (k) {
        const uint32_t lastP = __shfl_sync(0xFFFFFFFFu, myP, (int)k - 1);
        const uint32_t lastV = __shfl_sync(0xFFFFFFFFu, myV, (int)k - 1);
        const uint32_t lastB = __shfl_sync(0xFFFFFFFFu, before, (int)k - 1);
        const uint32_t lend_all = lastP + 2 + (lastV >> 16);
        if (lend_all > 64) {
          lit_rem = lend_all - 64;
          lit_out = done + lastB + (lastV & 0xFFFFu) + (64 - lastP - 2);
        }
      }
      done += dsum;
      if (done >= len && !lit_rem) break;
      if (done < len && (int32_t)pp <= 62 && (int32_t)pp > lim) {  // the next header does not fit in the chunk's bytes
        err = LT_ERR_SIZE_MISMATCH;
        break;
      }
      if (lit_rem) {
        q += kWin;
        p = pp - 64;
      } else {
        q += 2 * (uint64_t)pp;
        p = 0;
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
