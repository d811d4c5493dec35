// lt_lz4.cu -- LZ4 block decompression on chip, fused with INT4 unpack and
// group scaling to binary16 ("GPU Compression Pipeline - TDD Roadmap",
// Phase 2.1 LZ4 + INT4 Fused Kernel; 64 KB independent blocks as in
// Phase 3.1 / Phase 6.1), plus the same decoder writing raw bytes.
//
// One CTA decodes one 64 KB block at a time (persistent CTAs, grid-stride
// over the blocks of up to LT_LZ4_BATCH_MAX matrices); three CTAs fit per
// SM. The decompressed bytes (the packed INT4 codes) live only in a 64 KB
// window in shared memory and never reach HBM. The four warps of a CTA form
// a pipeline, each stage handing over through counters in shared memory
// (release stores, acquire loads, bounded waits):
//  * warp 0, the parser, streams the block's compressed bytes into an 8 KB
//    shared-memory ring with cp.async (2 KB chunks, up to four in flight)
//    and walks the sequence headers -- the one serial part of LZ4 -- pushing
//    one descriptor (literal position and length, match offset and length)
//    per sequence into a queue. It validates every field against the block
//    bounds, so what it pushes is always in range.
//  * warp 1, the copier, executes the descriptors in order with all 32
//    lanes: literal runs and non-overlapping matches four bytes per lane
//    (funnel shifts align source to destination); a match of offset d that
//    overlaps itself repeats its last d bytes, copied in rounds of d bytes
//    (d >= 16), as a byte fill (d == 1) or byte by byte with
//    win[p + i] = win[p - d + (i mod d)] (other d). Every ~1 KB it publishes
//    how many window bytes are final.
//  * warps 2 and 3 follow that progress and turn each 128-byte unit of the
//    window into 256 binary16 values: one 4-byte word (8 codes) per lane and
//    one 16-byte store per lane, so fp16 writes overlap the serial parse.

#include "lt_common.cuh"

namespace lt {
namespace {

constexpr int kWarps = 4;  // parser, copier, two dequantizers
constexpr int kThreads = kWarps * 32;
constexpr int kConsumers = kWarps - 2;
constexpr int kMaxWindow = 65536;
constexpr int kPad = 16;               // guard bytes before and after the window
constexpr uint32_t kPublishBytes = 1024;
constexpr uint32_t kUnit = 128;        // window bytes per dequantizer-warp step
constexpr uint32_t kRing = 8192;       // shared-memory ring for the compressed stream
constexpr uint32_t kChunk = 2048;      // ring refill granularity (one cp.async group)
constexpr uint32_t kChunks = kRing / kChunk;
constexpr uint32_t kQueue = 64;        // sequence descriptors in flight
constexpr uint32_t kEnd = 0xFFFFFFFFu; // descriptor literal length marking the end
constexpr long kSpinLimit = 1L << 23;  // ~0.5 s of polling, then give up

struct Job {
  const uint8_t *comp;
  uint64_t comp_bytes;
  const uint64_t *offsets;
  const uint16_t *scales;
  const uint8_t *zeros;
  void *out;
  int64_t n_codes;       // INT4 codes (fused) ; output bytes (raw)
  int64_t packed_bytes;  // decompressed bytes of the whole matrix
  int64_t first_block;   // index of this job's first block in the batch
  int64_t group_size;
  int32_t block_bytes;
  int32_t group_shift;   // log2(group_size) when a power of two, else -1
};

struct Batch {
  Job job[LT_LZ4_BATCH_MAX];
  int32_t n_jobs;
  int32_t max_block_bytes;
  int64_t total_blocks;
};

// hand-over counters of one CTA (reset for every block)
struct Ctl {
  uint32_t avail;     // parser -> copier: ring bytes (rel) that have landed
  uint32_t kc;        // copier -> parser: ring bytes (rel) the copier is done with
  uint32_t qhead;     // parser -> copier: descriptors pushed
  uint32_t qtail;     // copier -> parser: descriptors taken
  uint32_t progress;  // copier -> dequantizers: window bytes that are final
  uint32_t abort;     // set when a wait ran out: every stage stops waiting
};

__device__ __forceinline__ uint32_t ld_acquire_shared(const uint32_t *p) {
  uint32_t v;
  asm volatile("ld.acquire.cta.shared::cta.u32 %0, [%1];"
               : "=r"(v)
               : "r"((uint32_t)__cvta_generic_to_shared(p))
               : "memory");
  return v;
}
__device__ __forceinline__ void st_release_shared(uint32_t *p, uint32_t v) {
  asm volatile("st.release.cta.shared::cta.u32 [%0], %1;" ::"r"((uint32_t)__cvta_generic_to_shared(p)), "r"(v)
               : "memory");
}

// Wait (whole warp) until *c >= target. Lane 0 polls; the value is
// broadcast. Returns false if the wait ran out or another stage gave up.
__device__ __forceinline__ bool wait_ge(const uint32_t *c, uint32_t target, uint32_t &seen, Ctl *ctl, int lane,
                                        int32_t *d_status) {
  uint32_t v = 0, ok = 1;
  if (lane == 0) {
    v = ld_acquire_shared(c);
    long spins = 0;
    while (v < target) {
      ++spins;
      if ((spins & 15) == 0) {
        if (ld_acquire_shared(&ctl->abort)) {
          ok = 0;
          break;
        }
        if (spins > kSpinLimit) {
          report(d_status, LT_ERR_TIMEOUT);
          st_release_shared(&ctl->abort, 1u);
          ok = 0;
          break;
        }
      }
      if (spins > 64) __nanosleep(64);
      v = ld_acquire_shared(c);
    }
  }
  v = __shfl_sync(0xFFFFFFFFu, v, 0);
  ok = __shfl_sync(0xFFFFFFFFu, ok, 0);
  __syncwarp();
  seen = v;
  return ok != 0;
}

// ---------------------------------------------------------------------------
// compressed-stream ring (parser side). Positions are "rel" = address - a0,
// a0 = the block's first byte rounded down to a 16-byte boundary; rel r lives
// at ring[r mod kRing]. A chunk's slot is reused once the copier is past the
// chunk kChunks before it.
// ---------------------------------------------------------------------------
struct Ring {
  uint8_t *buf;
  const uint8_t *a0;   // rel 0 (absolute address, 16-byte aligned)
  const uint8_t *beg;  // the block's first byte
  const uint8_t *end;  // one past the block's last byte
  uint32_t total;      // chunks covering [a0, end)
  uint32_t issued;     // chunks whose copies were issued
  uint32_t done;       // chunks known complete and visible to the parser
};

__device__ __forceinline__ void cp_async16(void *smem, const void *gmem, uint32_t src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"((uint32_t)__cvta_generic_to_shared(smem)),
               "l"(gmem), "r"(src_bytes)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// Issue the copies of the next chunk, 16 bytes per lane per step. Only bytes
// of [beg, end) are read from HBM; the rest of the chunk is zero-filled or
// stale and never used. A 16-byte piece that starts before `beg` (the block
// does not start on a 16-byte boundary) is copied byte by byte.
__device__ __forceinline__ void ring_issue(Ring &r, int lane) {
  const uint32_t k = r.issued;
#pragma unroll
  for (uint32_t j = 0; j < kChunk / 512; ++j) {
    const uint32_t rel = k * kChunk + j * 512 + (uint32_t)lane * 16;
    const uint8_t *src = r.a0 + rel;
    uint8_t *dst = r.buf + (rel & (kRing - 1));
    if (src >= r.beg) {
      const uint32_t n = src < r.end ? (uint32_t)((r.end - src) < 16 ? (r.end - src) : 16) : 0u;
      cp_async16(dst, n ? (const void *)src : (const void *)r.beg, n);
    } else {
      for (uint32_t i = 0; i < 16; ++i)
        if (src + i >= r.beg && src + i < r.end) dst[i] = __ldg(src + i);
    }
  }
  cp_async_commit();
  r.issued = k + 1;
}

// wait until every chunk up to `c` (< issued) has landed and is visible
__device__ __forceinline__ void ring_wait(Ring &r, uint32_t c) {
  if (c < r.done) return;
  const uint32_t pending_after = r.issued - 1 - c;
  switch (pending_after) {
    case 0: cp_async_wait<0>(); break;
    case 1: cp_async_wait<1>(); break;
    case 2: cp_async_wait<2>(); break;
    default: cp_async_wait<3>(); break;
  }
  r.done = c + 1;
  __syncwarp();
}

// 4 bytes at rel position s (little-endian) from the ring
__device__ __forceinline__ uint32_t ring_gather4(const uint8_t *ring, uint32_t s) {
  const uint32_t *w = reinterpret_cast<const uint32_t *>(ring);
  const uint32_t i = s >> 2;
  return __funnelshift_r(w[i & (kRing / 4 - 1)], w[(i + 1) & (kRing / 4 - 1)], 8u * (s & 3));
}

// 4 bytes at window byte index s (may be slightly negative or past the end:
// the window has kPad guard bytes on both sides)
__device__ __forceinline__ uint32_t gather4_window(const uint8_t *win, int32_t s) {
  const int32_t al = s & ~3;  // floor to a multiple of 4 (two's complement)
  const uint32_t *w = reinterpret_cast<const uint32_t *>(win + al);
  return __funnelshift_r(w[0], w[1], 8u * (uint32_t)(s & 3));
}

// store word w (window bytes [4w, 4w+4)) keeping the bytes below `keep_below`
__device__ __forceinline__ void store_word(uint8_t *win, uint32_t w, uint32_t v, uint32_t keep_below) {
  uint32_t *dst = reinterpret_cast<uint32_t *>(win) + w;
  const uint32_t x = 4 * w;
  if (x < keep_below) {
    const uint32_t keep = 0xFFFFFFFFu >> (8u * (4u - (keep_below - x)));  // low (keep_below - x) bytes
    v = (*dst & keep) | (v & ~keep);
  }
  *dst = v;
}

// Copy L bytes from ring rel [src, src + L) to win[op, op + L). Bytes of the
// last word past op + L may receive garbage: they lie beyond everything
// decoded so far and will be written again.
__device__ __forceinline__ void copy_from_ring(const uint8_t *ring, uint32_t src, uint8_t *win, uint32_t op,
                                               uint32_t L, int lane) {
  const uint32_t w0 = op >> 2, w1 = (op + L + 3) >> 2;
  const uint32_t sbase = src - op;  // ring rel of window byte x is sbase + x (mod 2^32)
  for (uint32_t w = w0 + lane; w < w1; w += 32) store_word(win, w, ring_gather4(ring, sbase + 4 * w), op);
}

// Copy M bytes win[op - d + i] -> win[op + i] for d >= M (no overlap).
__device__ __forceinline__ void copy_window(uint8_t *win, uint32_t op, uint32_t d, uint32_t M, int lane) {
  const uint32_t w0 = op >> 2, w1 = (op + M + 3) >> 2;
  for (uint32_t w = w0 + lane; w < w1; w += 32)
    store_word(win, w, gather4_window(win, (int32_t)(4 * w) - (int32_t)d), op);
}

// ---------------------------------------------------------------------------
// warp 0: parser
// ---------------------------------------------------------------------------
struct Parser {
  Ring r;
  uint8_t *ring;
  uint4 *queue;
  Ctl *ctl;
  int32_t *d_status;
  int lane;
  uint32_t avail_pub;  // last published ring availability
  uint32_t kc_seen;    // copier consumption last observed
  uint32_t qhead, qtail_seen, qhead_pub;
  uint32_t iend;
  uint32_t pushed_end;  // input position up to which pushed descriptors reach

  // make everything issued so far land, and tell the copier
  __device__ __forceinline__ void publish_all() {
    if (r.issued > r.done) ring_wait(r, r.issued - 1);
    const uint32_t a = r.done * kChunk < iend ? r.done * kChunk : iend;
    if (a > avail_pub) {
      if (lane == 0) st_release_shared(&ctl->avail, a);
      avail_pub = a;
    }
  }

  // make ring rel bytes [.., q) readable by parser and copier (q <= iend)
  __device__ __forceinline__ bool need(uint32_t q) {
    if (q <= avail_pub) return true;
    const uint32_t c = (q - 1) / kChunk;
    if (c >= r.issued) kc_seen = ld_acquire_shared(&ctl->kc);  // refresh (lane-uniform enough: see below)
    kc_seen = __shfl_sync(0xFFFFFFFFu, kc_seen, 0);
    while (c >= r.issued) {
      if (r.issued < kc_seen / kChunk + kChunks) {
        ring_issue(r, lane);
        continue;
      }
      publish_all();  // the copier may be waiting for bytes already issued
      flush();        // ... or for descriptors not yet handed over
      if (!wait_ge(&ctl->kc, (r.issued - kChunks + 1) * kChunk, kc_seen, ctl, lane, d_status)) return false;
    }
    // top up while slots are free, then wait for chunk c
    while (r.issued < r.total && r.issued < kc_seen / kChunk + kChunks) ring_issue(r, lane);
    ring_wait(r, c);
    const uint32_t a = r.done * kChunk < iend ? r.done * kChunk : iend;
    if (a > avail_pub) {
      if (lane == 0) st_release_shared(&ctl->avail, a);
      avail_pub = a;
    }
    return true;
  }

  // The copier's position in the input only advances through pushed
  // descriptors (each marks the input up to the end of its literals), so
  // the ring can only be refilled up to ~3 chunks past `pushed_end`.
  __device__ __forceinline__ bool push(uint32_t src, uint32_t lit, uint32_t d, uint32_t m) {
    if (lit != kEnd && src + lit > pushed_end) pushed_end = src + lit;
    if (qhead - qtail_seen >= kQueue) {
      flush();
      if (!wait_ge(&ctl->qtail, qhead - kQueue + 1, qtail_seen, ctl, lane, d_status)) return false;
    }
    if (lane == 0) queue[qhead & (kQueue - 1)] = make_uint4(src, lit, d, m);
    ++qhead;
    // hand over in groups of 4 (and whenever the parser is about to wait)
    if ((qhead & 3) == 0 || lit == kEnd || d == 0) flush();
    return true;
  }

  __device__ __forceinline__ void flush() {
    if (qhead != qhead_pub) {
      if (lane == 0) st_release_shared(&ctl->qhead, qhead);
      qhead_pub = qhead;
    }
  }

  __device__ __forceinline__ uint32_t byte_at(uint32_t s) const { return ring[s & (kRing - 1)]; }

  // read a length-extension chain (bytes of 255 continue it) starting at
  // rel `ip`; slow path, taken only for runs of 270+ bytes
  __device__ __forceinline__ int ext_chain(uint32_t &ip, uint32_t &len, uint32_t olen) {
    uint32_t b;
    do {
      if (ip >= iend || len > olen) return LT_ERR_CORRUPT_STREAM;
      if (!need(ip + 1)) return -1;
      b = byte_at(ip);
      ip += 1;
      len += b;
    } while (b == 255);
    return 0;
  }

  // returns 0, a stream status, or -1 when a wait gave up
  __device__ int run(uint64_t s0, uint64_t s1, uint32_t olen) {
    const uint64_t ilen = s1 - s0;
    if (ilen == 0) return olen == 0 ? 0 : LT_ERR_SIZE_MISMATCH;
    if (ilen > 0x7FFFFFFFull) return LT_ERR_CORRUPT_STREAM;  // no valid block of <= 64 KB is this long
    const uint32_t lead = (uint32_t)(r.beg - r.a0);
    iend = lead + (uint32_t)ilen;
    uint32_t ip = lead, op = 0;
    for (;;) {
      // token and up to 3 length bytes
      if (ip + 4 > avail_pub) {
        if (ip >= iend) return LT_ERR_CORRUPT_STREAM;
        if (!need(ip + 4 < iend ? ip + 4 : iend)) return -1;
      }
      const uint32_t h = ring_gather4(ring, ip);
      const uint32_t token = h & 0xFFu;
      uint32_t lit = token >> 4;
      uint32_t ls = ip + 1;  // first literal byte
      if (lit == 15) {
        const uint32_t b = (h >> 8) & 0xFFu;
        if (ls >= iend) return LT_ERR_CORRUPT_STREAM;
        lit += b;
        ls += 1;
        if (b == 255) {
          const int e = ext_chain(ls, lit, olen);
          if (e) return e;
        }
      }
      const uint32_t le = ls + lit;  // end of the literals = offset position
      if (le > iend || op + lit > olen) return LT_ERR_CORRUPT_STREAM;
      if (le == iend) {
        // last sequence: literals only; feed the ring to the end of the block
        if (!push(ls, lit, 0, 0) || !need(iend)) return -1;
        return op + lit == olen ? 0 : LT_ERR_SIZE_MISMATCH;
      }
      // if the offset bytes lie too far past what the copier can reach,
      // hand the literals over first so that it can make room in the ring
      uint32_t lsrc = ls, llen = lit;
      if ((le + 3) / kChunk > pushed_end / kChunk + (kChunks - 1)) {
        if (!push(ls, lit, 0, 0)) return -1;
        lsrc = le;
        llen = 0;
      }
      if (le + 4 > avail_pub) {
        if (le + 2 > iend) return LT_ERR_CORRUPT_STREAM;
        if (!need(le + 4 < iend ? le + 4 : iend)) return -1;
      }
      const uint32_t m = ring_gather4(ring, le);  // offset and up to 2 length bytes
      const uint32_t d = m & 0xFFFFu;
      uint32_t mlen = (token & 15u) + 4;
      uint32_t nip = le + 2;  // next token
      if ((token & 15u) == 15u) {
        const uint32_t b = (m >> 16) & 0xFFu;
        if (nip >= iend) return LT_ERR_CORRUPT_STREAM;
        mlen += b;
        nip += 1;
        if (b == 255) {
          const int e = ext_chain(nip, mlen, olen);
          if (e) return e;
        }
      }
      op += lit;
      if (le + 2 > iend || d == 0 || d > op || op + mlen > olen) return LT_ERR_CORRUPT_STREAM;
      if (!push(lsrc, llen, d, mlen)) return -1;
      op += mlen;
      ip = nip;
    }
  }
};

// ---------------------------------------------------------------------------
// warp 1: copier
// ---------------------------------------------------------------------------
__device__ void copier(const uint8_t *ring, uint8_t *win, const uint4 *queue, Ctl *ctl, uint32_t olen, int lane,
                       int32_t *d_status) {
  uint32_t op = 0, qtail = 0, qhead_seen = 0, avail_seen = 0, kc_pub = 0, published = 0;
  for (;;) {
    if (qtail == qhead_seen) {
      if (!wait_ge(&ctl->qhead, qtail + 1, qhead_seen, ctl, lane, d_status)) break;
    }
    const uint4 e = queue[qtail & (kQueue - 1)];
    ++qtail;
    if ((qtail & 7) == 0 && lane == 0) st_release_shared(&ctl->qtail, qtail);
    if (e.y == kEnd) break;
    uint32_t src = e.x, L = e.y;
    const uint32_t d = e.z, M = e.w;
    bool ok = true;
    while (L) {
      if (src + L > avail_seen) {
        if (!wait_ge(&ctl->avail, src + 1, avail_seen, ctl, lane, d_status)) {
          ok = false;
          break;
        }
      }
      const uint32_t piece = (avail_seen - src) < L ? (avail_seen - src) : L;
      copy_from_ring(ring, src, win, op, piece, lane);
      src += piece;
      op += piece;
      L -= piece;
      if (L) {
        __syncwarp();
        if (src / kChunk != kc_pub / kChunk) {  // a chunk fully consumed: the parser may refill it
          if (lane == 0) st_release_shared(&ctl->kc, src);
          kc_pub = src;
        }
      }
    }
    if (!ok) break;
    __syncwarp();
    if (src / kChunk != kc_pub / kChunk && src > kc_pub) {
      if (lane == 0) st_release_shared(&ctl->kc, src);
      kc_pub = src;
    }
    if (M) {
      if (d >= M) {
        copy_window(win, op, d, M, lane);
      } else if (d == 1) {
        const uint32_t v = 0x01010101u * (uint32_t)win[op - 1];
        const uint32_t w0 = op >> 2, w1 = (op + M + 3) >> 2;
        for (uint32_t w = w0 + lane; w < w1; w += 32) store_word(win, w, v, op);
      } else if (d >= 16) {
        for (uint32_t done = 0; done < M; done += d) {  // rounds of d bytes: sources precede them
          const uint32_t n = (M - done) < d ? (M - done) : d;
          copy_window(win, op + done, d, n, lane);
          __syncwarp();
        }
      } else {
        const uint32_t src0 = op - d;
        uint32_t rr = (uint32_t)lane % d;
        const uint32_t step = 32u % d;
        for (uint32_t i = lane; i < M; i += 32) {
          win[op + i] = win[src0 + rr];
          rr += step;
          if (rr >= d) rr -= d;
        }
      }
      __syncwarp();
      op += M;
    }
    if (op - published >= kPublishBytes) {
      if (lane == 0) st_release_shared(&ctl->progress, op);
      published = op;
    }
  }
  __syncwarp();
  if (lane == 0) {
    // release everyone: dequantizers finish the block (content unspecified
    // after an error); the parser never waits on the copier again
    st_release_shared(&ctl->progress, olen);
    st_release_shared(&ctl->qtail, 0x7FFFFFFFu);
    st_release_shared(&ctl->kc, 0x7FFFFFFFu);
  }
}

template <bool FUSED>
__global__ void __launch_bounds__(kThreads) k_lz4(const __grid_constant__ Batch batch, int32_t *d_status) {
  extern __shared__ uint4 smem_u4[];
  uint8_t *ring = reinterpret_cast<uint8_t *>(smem_u4);
  uint8_t *win = ring + kRing + kPad;
  __shared__ uint4 queue[kQueue];
  __shared__ Ctl ctl;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  for (int64_t blk = blockIdx.x; blk < batch.total_blocks; blk += gridDim.x) {
    int j = 0;
    while (j + 1 < batch.n_jobs && blk >= batch.job[j + 1].first_block) ++j;
    const Job &jb = batch.job[j];
    const int64_t b = blk - jb.first_block;
    const int64_t d0 = b * (int64_t)jb.block_bytes;
    const uint32_t olen =
        (uint32_t)((jb.packed_bytes - d0) < jb.block_bytes ? (jb.packed_bytes - d0) : jb.block_bytes);

    if (threadIdx.x == 0) {
      ctl.avail = 0;
      ctl.kc = 0;
      ctl.qhead = 0;
      ctl.qtail = 0;
      ctl.progress = 0;
      ctl.abort = 0;
    }
    __syncthreads();

    if (warp == 0) {
      const uint64_t s0 = jb.offsets[b], s1 = jb.offsets[b + 1];
      int err;
      if (s1 < s0 || s1 > jb.comp_bytes) {
        err = LT_ERR_CORRUPT_STREAM;
        if (lane == 0) {  // nothing to parse: stop the copier at once
          queue[0] = make_uint4(0, kEnd, (uint32_t)err, 0);
          st_release_shared(&ctl.qhead, 1u);
        }
      } else {
        Parser P;
        P.ring = ring;
        P.queue = queue;
        P.ctl = &ctl;
        P.d_status = d_status;
        P.lane = lane;
        P.avail_pub = 0;
        P.kc_seen = 0;
        P.qhead = 0;
        P.qtail_seen = 0;
        P.qhead_pub = 0;
        P.pushed_end = 0;
        P.r.buf = ring;
        P.r.beg = jb.comp + s0;
        P.r.end = jb.comp + s1;
        P.r.a0 = reinterpret_cast<const uint8_t *>(reinterpret_cast<uintptr_t>(P.r.beg) & ~uintptr_t(15));
        P.r.total = (uint32_t)((P.r.end - P.r.a0 + kChunk - 1) / kChunk);
        P.r.issued = 0;
        P.r.done = 0;
        P.iend = 0;
        err = P.run(s0, s1, olen);
        if (err != 0 && lane == 0) {
          // a literal run the copier is still waiting for may never be fed:
          // let it copy whatever the ring holds (the output is unspecified)
          st_release_shared(&ctl.avail, 0x7FFFFFFFu);
        }
        if (err >= 0) P.push(0, kEnd, (uint32_t)err, 0);
        cp_async_wait<0>();  // nothing may land in the ring after this block
      }
      __syncwarp();
      if (lane == 0 && err > 0) report(d_status, err);
    } else if (warp == 1) {
      copier(ring, win, queue, &ctl, olen, lane, d_status);
    } else {
      const uint32_t n_units = (olen + kUnit - 1) / kUnit;
      uint32_t seen = 0;
      if (FUSED) {
        uint16_t *out = reinterpret_cast<uint16_t *>(jb.out);
        const int64_t k0 = 2 * d0;  // first code of the block
        const int64_t k_end = (k0 + 2 * (int64_t)olen) < jb.n_codes ? (k0 + 2 * (int64_t)olen) : jb.n_codes;
        const int64_t G = jb.group_size;
        const bool vec = (G % 8 == 0) && aligned(out + k0, 16);
        const uint32_t *win32 = reinterpret_cast<const uint32_t *>(win);
        for (uint32_t u = warp - 2; u < n_units; u += kConsumers) {
          const uint32_t need = (u + 1) * kUnit < olen ? (u + 1) * kUnit : olen;
          if (seen < need && !wait_ge(&ctl.progress, need, seen, &ctl, lane, d_status)) break;
          const uint32_t wi = u * (kUnit / 4) + lane;  // window word
          const int64_t k = k0 + 8 * (int64_t)wi;      // its first code
          if (k >= k_end) continue;
          if (vec && k + 8 <= k_end) {
            const int64_t g = jb.group_shift >= 0 ? (k >> jb.group_shift) : k / G;
            const uint32_t s2 = bcast_half(__ldg(jb.scales + g));
            const uint32_t zm = jb.zeros ? int4_zero_magic(__ldg(jb.zeros + g)) : 0x54006400u;
            st_u128(out + k, int4x8_dequant(win32[wi], zm, s2));
          } else {
            const int64_t ke = (k + 8) < k_end ? (k + 8) : k_end;
            for (int64_t kk = k; kk < ke; ++kk) {
              const uint8_t byte = win[(kk - k0) >> 1];
              const int32_t q = (kk & 1) ? (byte >> 4) : (byte & 0x0F);
              const int64_t g = kk / G;
              const int32_t z = jb.zeros ? jb.zeros[g] : 0;
              out[kk] = dequant_scalar(q - z, jb.scales[g]);
            }
          }
        }
      } else {
        uint8_t *out = reinterpret_cast<uint8_t *>(jb.out) + d0;
        const bool vec = aligned(out, 4);
        for (uint32_t u = warp - 2; u < n_units; u += kConsumers) {
          const uint32_t need = (u + 1) * kUnit < olen ? (u + 1) * kUnit : olen;
          if (seen < need && !wait_ge(&ctl.progress, need, seen, &ctl, lane, d_status)) break;
          const uint32_t x = u * kUnit + 4 * lane;
          if (x >= olen) continue;
          if (vec && x + 4 <= olen) {
            *reinterpret_cast<uint32_t *>(out + x) = *reinterpret_cast<const uint32_t *>(win + x);
          } else {
            for (uint32_t i = x; i < olen && i < x + 4; ++i) out[i] = win[i];
          }
        }
      }
    }
    __syncthreads();
  }
}

lt_status launch(const Batch &batch, bool fused, int32_t *d_status, cudaStream_t st) {
  if (batch.total_blocks == 0) return LT_OK;
  const size_t smem = kRing + (size_t)((batch.max_block_bytes + 15) / 16 * 16) + 2 * kPad;
  const void *k = fused ? (const void *)k_lz4<true> : (const void *)k_lz4<false>;
  static int attr_set[2][64] = {{0}};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev >= 0 && dev < 64 && !attr_set[fused][dev]) {
    cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, kRing + kMaxWindow + 2 * kPad);
    attr_set[fused][dev] = 1;
  }
  const int64_t cap = (int64_t)num_sms() * blocks_per_sm(k, kThreads, smem);
  const int grid = (int)(batch.total_blocks < cap ? batch.total_blocks : cap);
  if (fused)
    k_lz4<true><<<grid, kThreads, smem, st>>>(batch, d_status);
  else
    k_lz4<false><<<grid, kThreads, smem, st>>>(batch, d_status);
  return launch_status();
}

bool block_bytes_ok(int32_t bb) { return bb >= 16 && bb <= kMaxWindow && bb % 16 == 0; }

// validate one fused descriptor and append it to the batch
lt_status add_fused_job(Batch &batch, const uint8_t *comp, uint64_t comp_bytes, const uint64_t *offsets,
                        int32_t block_bytes, const lt_half *scales, const uint8_t *zeros, int64_t rows, int64_t cols,
                        int32_t group_size, lt_half *out) {
  if (rows < 0 || cols < 0 || group_size < 1) return LT_ERR_INVALID_ARG;
  if (cols % group_size != 0) return LT_ERR_INVALID_ARG;
  if (rows != 0 && cols > INT64_MAX / rows) return LT_ERR_INVALID_ARG;
  if (!block_bytes_ok(block_bytes)) return LT_ERR_UNSUPPORTED;
  const int64_t n = rows * cols;
  if (n == 0) return LT_OK;
  if (!offsets || !scales || !out || (!comp && comp_bytes != 0)) return LT_ERR_INVALID_ARG;
  if (!aligned(offsets, 8) || !aligned(scales, 2) || !aligned(out, 2)) return LT_ERR_MISALIGNED;
  if (batch.n_jobs >= LT_LZ4_BATCH_MAX) return LT_ERR_UNSUPPORTED;
  Job &j = batch.job[batch.n_jobs++];
  j.comp = comp;
  j.comp_bytes = comp_bytes;
  j.offsets = offsets;
  j.scales = scales;
  j.zeros = zeros;
  j.out = out;
  j.n_codes = n;
  j.packed_bytes = (n + 1) / 2;
  j.first_block = batch.total_blocks;
  j.group_size = group_size;
  j.block_bytes = block_bytes;
  j.group_shift = -1;
  for (int sh = 0; sh < 62; ++sh)
    if ((int64_t)1 << sh == (int64_t)group_size) j.group_shift = sh;
  batch.total_blocks += (j.packed_bytes + block_bytes - 1) / block_bytes;
  if (block_bytes > batch.max_block_bytes) batch.max_block_bytes = block_bytes;
  return LT_OK;
}

Batch empty_batch() {
  Batch b;
  memset(&b, 0, sizeof(b));
  return b;
}

}  // namespace
}  // namespace lt

using namespace lt;

LT_API lt_status lt_lz4_int4_decode(const uint8_t *comp, uint64_t comp_bytes, const uint64_t *block_offsets,
                                    int32_t block_bytes, const lt_half *scales, const uint8_t *zeros, int64_t rows,
                                    int64_t cols, int32_t group_size, lt_half *out, int32_t *d_status,
                                    lt_stream_t stream) {
  if (!aligned(d_status, 4)) return LT_ERR_MISALIGNED;
  Batch batch = empty_batch();
  lt_status s = add_fused_job(batch, comp, comp_bytes, block_offsets, block_bytes, scales, zeros, rows, cols,
                              group_size, out);
  if (s != LT_OK) return s;
  return launch(batch, true, d_status, (cudaStream_t)stream);
}

LT_API lt_status lt_lz4_int4_decode_batch(const lt_lz4_int4_desc *descs, int32_t n_desc, int32_t *d_status,
                                          lt_stream_t stream) {
  if (n_desc < 1 || !descs) return LT_ERR_INVALID_ARG;
  if (n_desc > LT_LZ4_BATCH_MAX) return LT_ERR_UNSUPPORTED;
  if (!aligned(d_status, 4)) return LT_ERR_MISALIGNED;
  Batch batch = empty_batch();
  for (int32_t i = 0; i < n_desc; ++i) {
    const lt_lz4_int4_desc &d = descs[i];
    lt_status s = add_fused_job(batch, d.comp, d.comp_bytes, d.block_offsets, d.block_bytes, d.scales, d.zeros,
                                d.rows, d.cols, d.group_size, d.out);
    if (s != LT_OK) return s;
  }
  return launch(batch, true, d_status, (cudaStream_t)stream);
}

LT_API lt_status lt_lz4_decode(const uint8_t *comp, uint64_t comp_bytes, const uint64_t *block_offsets,
                               int32_t block_bytes, uint8_t *out, uint64_t out_bytes, int32_t *d_status,
                               lt_stream_t stream) {
  if (!block_bytes_ok(block_bytes)) return LT_ERR_UNSUPPORTED;
  if (out_bytes == 0) return LT_OK;
  if (!block_offsets || !out || (!comp && comp_bytes != 0)) return LT_ERR_INVALID_ARG;
  if (!aligned(block_offsets, 8) || !aligned(d_status, 4)) return LT_ERR_MISALIGNED;
  if (out_bytes > (uint64_t)INT64_MAX) return LT_ERR_INVALID_ARG;
  Batch batch = empty_batch();
  Job &j = batch.job[0];
  batch.n_jobs = 1;
  j.comp = comp;
  j.comp_bytes = comp_bytes;
  j.offsets = block_offsets;
  j.out = out;
  j.n_codes = (int64_t)out_bytes;
  j.packed_bytes = (int64_t)out_bytes;
  j.first_block = 0;
  j.group_size = 1;
  j.group_shift = 0;
  j.block_bytes = block_bytes;
  batch.total_blocks = ((int64_t)out_bytes + block_bytes - 1) / block_bytes;
  batch.max_block_bytes = block_bytes;
  return launch(batch, false, d_status, (cudaStream_t)stream);
}
