// lt_lz4.cu -- LZ4 block decompression fused with INT4 unpack and group
// scaling to binary16 ("GPU Compression Pipeline - TDD Roadmap", Phase 2.1
// LZ4 + INT4 Fused Kernel; 64 KB independent blocks as in Phase 3.1 /
// Phase 6.1), plus the same decoder writing raw bytes.
//
// The one serial part of LZ4 is the walk over sequence headers: where a
// sequence's literals and match are depends on every length before it.
// Everything else is parallel once that walk has produced an index, so a
// call is two kernels:
//  1. k_lz4_parse: one warp per block walks its token stream (through a
//     small cp.async ring in shared memory), validates every field against
//     the block bounds in the oracle's order, gives each match a dependency
//     level, and writes a sequence index -- literal source and level,
//     output position, literal length, match offset and length, 16 bytes per
//     sequence -- to a caller-provided workspace. Thousands of blocks walk
//     side by side.
//  2. k_lz4_expand: one CTA per block (persistent, three per SM) rebuilds the
//     block in a 64 KB shared-memory window -- decompressed bytes never reach
//     HBM: it stages the compressed block at the end of the window, copies
//     all literal runs in parallel rounds, copies the matches one dependency
//     level at a time, then turns the window into binary16 (8 codes per
//     4-byte word, 16-byte stores).
// The two kernels can also be launched separately: lt_lz4_index_batch runs
// the parse over many matrices at once, lt_lz4_int4_expand_batch expands a
// slice of its index. Blocks with more than kCap sequences, calls without a
// workspace, blocks that cannot be staged in place, and blocks indexed for a
// different window size are decoded by warp 0 walking the block itself
// (slower, same result).

#include <mutex>

#include "lt_common.cuh"
#include "lt_xxh3.cuh"

namespace lt {
namespace {

constexpr int kWarps = 8;
constexpr int kThreads = kWarps * 32;
constexpr uint32_t kMaxWindow = 65536;
constexpr int kPad = 16;                 // guard bytes before and after the window
constexpr uint32_t kCap = 2 * kThreads; // sequence descriptors per block in the workspace (two per thread)
constexpr uint32_t kOverflow = 0x100;    // parse status: more than kCap sequences
constexpr uint32_t kNoIndex = 0x101;     // no workspace: every block takes the fallback
constexpr uint32_t kNoInPlace = 0x102;   // parse status: the block cannot be staged in its window
constexpr uint32_t kWinSlack = 512;      // window bytes past the largest block, for in-place staging
constexpr uint32_t kLevelCap = 255;      // match levels saturate here (the block is then replayed in order)
constexpr uint32_t kTailMatches = 32;    // matches left when warp 0 finishes the levels alone

// Window bytes a CTA holds for blocks of up to max_block_bytes: the block
// plus room to stage its compressed bytes at the end.
__host__ __device__ constexpr uint32_t win_cap(int32_t max_block_bytes) {
  return ((uint32_t)max_block_bytes + 15u) / 16u * 16u + kWinSlack;
}

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
  // checked decode (one job): each compressed block's XXH3-64 with this
  // secret must equal expected[block] before the block is decoded
  const uint8_t *secret;
  uint32_t secret_len;
  const uint64_t *expected;
  unsigned long long *first_bad;
};

__device__ __forceinline__ const Job &find_job(const Batch &batch, int64_t blk, int64_t &b) {
  int j = 0;
  while (j + 1 < batch.n_jobs && blk >= batch.job[j + 1].first_block) ++j;
  b = blk - batch.job[j].first_block;
  return batch.job[j];
}

__device__ __forceinline__ uint32_t block_len(const Job &jb, int64_t b) {
  const int64_t d0 = b * (int64_t)jb.block_bytes;
  return (uint32_t)((jb.packed_bytes - d0) < jb.block_bytes ? (jb.packed_bytes - d0) : jb.block_bytes);
}


// 4 bytes at window byte index s (may be slightly negative or past the end:
// the window has kPad guard bytes on both sides)
__device__ __forceinline__ uint32_t gather4_window(const uint8_t *win, int32_t s) {
  const int32_t al = s & ~3;  // floor to a multiple of 4 (two's complement)
  const uint32_t *w = reinterpret_cast<const uint32_t *>(win + al);
  return __funnelshift_r(w[0], w[1], 8u * (uint32_t)(s & 3));
}

// Write window bytes [a, b) with NL cooperating lanes (lid in [0, NL)):
// whole aligned words in the middle, single bytes at the (at most 3-byte)
// edges; the value of window byte x is src1(x), of the aligned word at x
// src4(x). Never writes a byte outside [a, b), so spans written by
// different warps never clobber each other.
template <int NL, typename S1, typename S4>
__device__ __forceinline__ void write_span(uint8_t *win, uint32_t a, uint32_t b, int lid, S1 src1, S4 src4) {
  const uint32_t wa = (a + 3) & ~3u, wb = b & ~3u;
  const uint32_t he = wa < b ? wa : b;    // head bytes [a, he)
  const uint32_t ts = wb > he ? wb : he;  // tail bytes [ts, b)
  if (wa < wb) {
    uint32_t *w32 = reinterpret_cast<uint32_t *>(win);
    for (uint32_t x = wa + 4 * (uint32_t)lid; x < wb; x += 4 * NL) w32[x >> 2] = src4(x);
  }
  if (lid < 8) {
    const uint32_t x = lid < 4 ? a + (uint32_t)lid : ts + (uint32_t)(lid - 4);
    if (lid < 4 ? x < he : x < b) win[x] = src1(x);
  }
}

// Replay one match with NL cooperating lanes (lid in [0, NL), syncing with
// `mask`): window bytes [op, op + M) from [op - d, ...).
template <int NL>
__device__ __forceinline__ void copy_match(uint8_t *win, uint32_t op, uint32_t d, uint32_t M, int lid,
                                           unsigned mask) {
  if (d >= M) {
    write_span<NL>(
        win, op, op + M, lid, [&](uint32_t x) { return win[x - d]; },
        [&](uint32_t x) { return gather4_window(win, (int32_t)x - (int32_t)d); });
  } else if (d == 1) {
    const uint32_t bv = win[op - 1];
    const uint32_t v = 0x01010101u * bv;
    write_span<NL>(
        win, op, op + M, lid, [&](uint32_t) { return (uint8_t)bv; }, [&](uint32_t) { return v; });
  } else if (d >= 16) {
    for (uint32_t done = 0; done < M; done += d) {  // rounds of d bytes: each round's source precedes it
      const uint32_t n = (M - done) < d ? (M - done) : d;
      write_span<NL>(
          win, op + done, op + done + n, lid, [&](uint32_t x) { return win[x - d]; },
          [&](uint32_t x) { return gather4_window(win, (int32_t)x - (int32_t)d); });
      __syncwarp(mask);
    }
  } else {
    const uint32_t src0 = op - d;
    uint32_t rr = (uint32_t)lid % d;
    const uint32_t step = (uint32_t)NL % d;
    for (uint32_t i = lid; i < M; i += NL) {
      win[op + i] = win[src0 + rr];
      rr += step;
      if (rr >= d) rr -= d;
    }
  }
}

// ---------------------------------------------------------------------------
// 1. parse: one warp walks one block
// ---------------------------------------------------------------------------
// One warp walks one block: its compressed bytes stream through a 2 KB
// shared-memory ring (cp.async, one 16-byte copy per lane = one 512-byte
// chunk per instruction, four chunks in flight ahead of the walk) and every
// lane reads the same header bytes from there (broadcast), so the walk is
// warp-uniform -- no divergence -- at two dependent shared-memory reads per
// sequence. 64 warps per SM walk 64 blocks side by side.
constexpr int kParseWarps = 4;
constexpr uint32_t kPRing = 2048;
constexpr uint32_t kPChunk = 512;
constexpr uint32_t kPChunks = kPRing / kPChunk;

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

struct WarpRing {
  uint8_t *buf;        // this warp's kPRing bytes
  const uint8_t *a0;   // rel 0: the block's first byte rounded down to 16 bytes
  const uint8_t *beg;  // the block's first byte
  const uint8_t *end;  // one past its last byte
  uint32_t total;      // chunks covering [a0, end)
  uint32_t issued;     // chunks issued (each one cp.async group, in order)
  uint32_t done;       // chunks known landed and visible to the warp
  int lane;

  // copies of chunk `issued`, 16 bytes per lane; only bytes of [beg, end)
  // are read from HBM (a piece starting before `beg` is copied byte by byte)
  __device__ __forceinline__ void issue() {
    const uint32_t rel = issued * kPChunk + 16u * (uint32_t)lane;
    const uint8_t *src = a0 + rel;
    uint8_t *dst = buf + (rel & (kPRing - 1));
    if (src >= beg) {
      const uint32_t nb = src < end ? (uint32_t)((end - src) < 16 ? (end - src) : 16) : 0u;
      cp_async16(dst, nb ? (const void *)src : (const void *)beg, nb);
    } else {
      for (uint32_t i = 0; i < 16; ++i)
        if (src + i >= beg && src + i < end) dst[i] = __ldg(src + i);
    }
    cp_async_commit();
    ++issued;
  }
  // wait until every chunk up to c (< issued) has landed
  __device__ __forceinline__ void wait_for(uint32_t c) {
    if (c < done) return;
    switch (issued - 1 - c) {  // groups allowed to stay in flight
      case 0: cp_async_wait<0>(); break;
      case 1: cp_async_wait<1>(); break;
      case 2: cp_async_wait<2>(); break;
      default: cp_async_wait<3>(); break;
    }
    done = c + 1;
    __syncwarp();  // every lane's copies are visible to every lane
  }
  // keep kPChunks chunks in flight ahead of rel position `pos`. A slot is
  // refilled only after the chunk it held has landed: copies of different
  // groups may complete in any order.
  __device__ __forceinline__ void top_up(uint32_t pos) {
    const uint32_t lim = pos / kPChunk + kPChunks;
    while (issued < total && issued < lim) {
      if (issued >= kPChunks) wait_for(issued - kPChunks);
      issue();
    }
  }
  // make rel bytes [pos, q) readable (pos < q <= pos + 32)
  __device__ __forceinline__ void need(uint32_t pos, uint32_t q) {
    const uint32_t c = (q - 1) / kPChunk;
    if (c < done) return;
    const uint32_t cmin = pos / kPChunk;
    if (cmin > issued) {  // the walk skipped everything fetched (a long literal run): restart there
      cp_async_wait<0>();
      issued = done = cmin;
    }
    top_up(pos);
    wait_for(c);
  }
  __device__ __forceinline__ uint32_t at(uint32_t rel) const { return buf[rel & (kPRing - 1)]; }
};

// Sequence descriptors leave the parse one per lane, 32 at a time.
struct DescOut {
  uint4 *out;
  uint4 held = make_uint4(0u, 0u, 0u, 0u);  // descriptor n with n % 32 == lane
  uint32_t n = 0;
  uint32_t lane;
  __device__ __forceinline__ void push(const uint4 &e) {
    if (lane == (n & 31)) held = e;
    ++n;
    if ((n & 31) == 0) out[n - 32 + lane] = held;
  }
  __device__ __forceinline__ void flush() {
    if (lane < (n & 31)) out[(n & ~31u) + lane] = held;
  }
};

// Match levels: a match's level is one more than the highest level of any
// match that wrote bytes it reads (literals are level 0), tracked per
// 16-byte output granule in `lmap` (4096 bytes). A granule's level is the
// highest level of the matches writing into it, so a match that reads a
// byte another match wrote always has the higher level, and matches of one
// level never read each other's output: they can be copied in parallel.
// Levels saturate at kLevelCap (the expansion then replays in order).
struct Leveler {
  uint8_t *lmap;
  uint32_t lane, lmax = 0;
  // level of the match writing [dst, dst + M) from offset d (warp-wide)
  __device__ __forceinline__ uint32_t level(uint32_t dst, uint32_t d, uint32_t M) {
    const uint32_t lo = dst - d, hi = lo + (d < M ? d : M);
    const uint32_t s0 = lo >> 4, ns = ((hi - 1) >> 4) - s0;  // source granules s0 .. s0 + ns
    const uint32_t d0 = dst >> 4, nd = ((dst + M - 1) >> 4) - d0;
    uint32_t mx = lane <= ns ? lmap[s0 + lane] : 0u;
    const uint32_t old0 = lmap[d0];
    for (uint32_t g = 32 + lane; g <= ns; g += 32) mx = mx > lmap[s0 + g] ? mx : lmap[s0 + g];  // long sources
    mx = __reduce_max_sync(0xFFFFFFFFu, mx);
    const uint32_t lvl = mx + 1 < kLevelCap ? mx + 1 : kLevelCap;
    if (lane <= nd) lmap[d0 + lane] = (uint8_t)(lane == 0 && old0 > lvl ? old0 : lvl);
    for (uint32_t g = 32 + lane; g <= nd; g += 32) lmap[d0 + g] = (uint8_t)lvl;  // long matches
    __syncwarp();
    lmax = lmax > lvl ? lmax : lvl;
    return lvl;
  }
};

// Walk LZ4 block [beg, end) that must decode to exactly olen bytes; write
// descriptors {literal source | level << 17, output position, literal
// length, match offset | (match length - 4) << 16} (offset 0: no match).
// Returns 0, a stream status, kOverflow or kNoInPlace. Warp-uniform: every
// lane reads the same header bytes (broadcast).
//
// Most sequences take the fast path: all header bytes readable, at most one
// extra length byte each for the literal and the match length, and every
// bound satisfied -- tested with flags, no branch per check. Any other
// sequence (the last one, long lengths, anything out of bounds) is walked
// by the slow path, which checks the bounds the oracle checks in the same
// order, so statuses agree. A match's level is worked out one sequence
// later, right after the next token is read, so it overlaps that read.
template <typename R>
__device__ __forceinline__ uint32_t parse_block(R &r, uint32_t olen, uint32_t wcap, uint8_t *lmap,
                                                uint4 *__restrict__ out, uint32_t &n_out, uint32_t &lmax_out) {
  n_out = 0;
  lmax_out = 0;
  const uint64_t ilen = (uint64_t)(r.end - r.beg);
  if (ilen == 0) return olen == 0 ? 0u : (uint32_t)LT_ERR_SIZE_MISMATCH;
  if (ilen > 0x7FFFFFFFull) return LT_ERR_CORRUPT_STREAM;  // no valid block of <= 64 KB is this long
  const uint32_t lead = (uint32_t)(r.beg - r.a0);
  const uint32_t iend = lead + (uint32_t)ilen;
  // In-place staging: the expanding CTA puts rel byte p at window index
  // so16 + p. That works if no literal byte's output position lies past its
  // staged position (checked per run below).
  bool inplace = iend <= wcap;
  const uint32_t so16 = inplace ? (wcap - iend) & ~15u : 0u;
  for (uint32_t i = (uint32_t)r.lane; i < kMaxWindow / 16 / 16; i += 32)
    reinterpret_cast<uint4 *>(lmap)[i] = make_uint4(0u, 0u, 0u, 0u);
  __syncwarp();
  DescOut dout;
  dout.out = out;
  dout.lane = (uint32_t)r.lane;
  Leveler lv;
  lv.lmap = lmap;
  lv.lane = (uint32_t)r.lane;
  bool pend = false;  // a match whose level is still to be worked out
  uint4 pe = make_uint4(0u, 0u, 0u, 0u);
  uint32_t ip = lead, op = 0, n = 0, st = 0;
  for (;;) {
    // --- fast path ---
    const uint32_t ic = ip < iend ? ip : iend - 1;  // clamped: reads stay inside the block
    r.need(ic, ic + 3 < iend ? ic + 3 : iend);
    const uint32_t token = r.at(ic), t1 = r.at(ic + 1), t2 = r.at(ic + 2);
    if (pend) {  // the previous match
      pe.x |= lv.level(pe.y + pe.z, pe.w & 0xFFFFu, (pe.w >> 16) + 4) << 17;
      dout.push(pe);
      pend = false;
    }
    const uint32_t lx = (token >> 4) == 15 ? 1u : 0u;  // one extra literal-length byte
    const uint32_t lit = (token >> 4) + (lx ? t1 : 0u);
    const uint32_t ls = ip + 1 + lx;  // first literal
    const uint32_t mp = ls + lit;     // match offset bytes
    // The literal side is settled before the offset bytes are fetched: that
    // fetch may move the ring past the token, and the slow path below then
    // uses the token and its first length byte from registers.
    if (ip + 3 <= iend && !(lx && t1 == 255u) && mp + 3 <= iend && op + lit <= olen && n < kCap) {
      r.need(mp, mp + 3);
      const uint32_t o0 = r.at(mp), o1 = r.at(mp + 1), o2 = r.at(mp + 2);
      const uint32_t d = o0 | (o1 << 8);
      const uint32_t mx = (token & 15u) == 15u ? 1u : 0u;  // one extra match-length byte
      const uint32_t mlen = (token & 15u) + 4 + (mx ? o2 : 0u);
      if (!(mx && o2 == 255u) && d != 0 && d <= op + lit && op + lit + mlen <= olen) {
        if (lit && op > so16 + ls) inplace = false;
        pe = make_uint4(ls - lead, op, lit, d | ((mlen - 4) << 16));
        pend = true;
        ++n;
        op += lit + mlen;
        ip = mp + 2 + mx;
        r.top_up(ip);
        continue;
      }
    }
    // --- slow path: one sequence, every check in the oracle's order; the
    // bytes after the first length byte are read from the ring, which
    // still holds them (see above) ---
    if (ip >= iend) { st = LT_ERR_CORRUPT_STREAM; break; }
    uint32_t b = ip + 1 < iend ? t1 : 0u;
    ip += 1;
    uint32_t slit = token >> 4;
    if (slit == 15) {
      for (;;) {
        if (ip >= iend || slit > olen) { st = LT_ERR_CORRUPT_STREAM; break; }
        ip += 1;
        slit += b;
        if (b != 255) break;
        if (ip < iend) {
          r.need(ip, ip + 1);
          b = r.at(ip);
        }
      }
      if (st) break;
    }
    if ((uint64_t)ip + slit > iend || (uint64_t)op + slit > olen) { st = LT_ERR_CORRUPT_STREAM; break; }
    if (slit && op > so16 + ip) inplace = false;
    const uint32_t sls = ip - lead;
    ip += slit;
    if (ip == iend) {  // the last sequence has literals only
      if (n >= kCap) { st = kOverflow; break; }
      dout.push(make_uint4(sls, op, slit, 0u));
      ++n;
      op += slit;
      if (op != olen) st = LT_ERR_SIZE_MISMATCH;
      break;
    }
    if (ip + 2 > iend) { st = LT_ERR_CORRUPT_STREAM; break; }
    r.need(ip, ip + 3 < iend ? ip + 3 : iend);
    const uint32_t sd = r.at(ip) | (r.at(ip + 1) << 8);
    b = ip + 2 < iend ? r.at(ip + 2) : 0u;
    ip += 2;
    if (sd == 0 || sd > op + slit) { st = LT_ERR_CORRUPT_STREAM; break; }
    uint32_t smlen = (token & 15u) + 4;
    if ((token & 15u) == 15u) {
      for (;;) {
        if (ip >= iend || smlen > olen) { st = LT_ERR_CORRUPT_STREAM; break; }
        ip += 1;
        smlen += b;
        if (b != 255) break;
        if (ip < iend) {
          r.need(ip, ip + 1);
          b = r.at(ip);
        }
      }
      if (st) break;
    }
    if ((uint64_t)op + slit + smlen > olen) { st = LT_ERR_CORRUPT_STREAM; break; }
    if (n >= kCap) { st = kOverflow; break; }
    pe = make_uint4(sls, op, slit, sd | ((smlen - 4) << 16));
    pend = true;
    ++n;
    op += slit + smlen;
    r.top_up(ip);
  }
  if (st == 0) dout.flush();  // (a valid block ends with a literal-only sequence: nothing is pending)
  cp_async_wait<0>();  // nothing may land in the ring after this block
  __syncwarp();
  n_out = n;
  lmax_out = lv.lmax;
  if (st == 0 && !inplace) st = kNoInPlace;
  return st;
}

__global__ void __launch_bounds__(kParseWarps * 32) k_lz4_parse(const __grid_constant__ Batch batch,
                                                                uint4 *__restrict__ hdr, uint4 *__restrict__ desc) {
  __shared__ __align__(16) uint8_t rings[kParseWarps][kPRing];
  __shared__ __align__(16) uint8_t lmaps[kParseWarps][kMaxWindow / 16];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int64_t blk = (int64_t)blockIdx.x * kParseWarps + warp; blk < batch.total_blocks;
       blk += (int64_t)gridDim.x * kParseWarps) {
    int64_t b;
    const Job &jb = find_job(batch, blk, b);
    const uint32_t olen = block_len(jb, b);
    const uint64_t s0 = jb.offsets[b], s1 = jb.offsets[b + 1];
    uint32_t n = 0, st, lmax = 0;
    if (s1 < s0 || s1 > jb.comp_bytes) {
      st = LT_ERR_CORRUPT_STREAM;
    } else {
      WarpRing r;
      r.buf = rings[warp];
      r.lane = lane;
      r.beg = jb.comp + s0;
      r.end = jb.comp + s1;
      r.a0 = reinterpret_cast<const uint8_t *>(reinterpret_cast<uintptr_t>(r.beg) & ~uintptr_t(15));
      r.total = (uint32_t)((r.end - r.a0 + kPChunk - 1) / kPChunk);
      r.issued = 0;
      r.done = 0;
      r.top_up(0);
      st = parse_block(r, olen, win_cap(batch.max_block_bytes), lmaps[warp], desc + blk * kCap, n, lmax);
    }
    if (lane == 0) hdr[blk] = make_uint4(n, st, lmax, win_cap(batch.max_block_bytes));  // the window checked against
  }
}

// The whole compressed block staged in shared memory: the same walk with
// none of the ring's bookkeeping (every byte is readable from the start).
// For launches with few blocks per SM, where each warp's walk is a latency
// chain and the ring's per-sequence work sits on it.
struct StagedBlock {
  const uint8_t *buf;  // rel byte x at buf[x] (rel 0 = a0)
  const uint8_t *a0, *beg, *end;
  int lane;
  __device__ __forceinline__ void need(uint32_t, uint32_t) const {}
  __device__ __forceinline__ void top_up(uint32_t) const {}
  __device__ __forceinline__ uint32_t at(uint32_t rel) const { return buf[rel]; }
};

// Staging buffer of a CTA of k_lz4_parse_staged: 51 KB, so that four CTAs
// (with their level maps) fit in an SM's shared memory. Compressible 64 KB
// blocks fit (the INT4 workloads' largest is 50.5 KB); a block that does not
// (e.g. incompressible data) streams through the first 2 KB of the buffer as
// the ring of k_lz4_parse instead.
constexpr uint32_t kStageCap = 51 * 1024;

__global__ void __launch_bounds__(32) k_lz4_parse_staged(const __grid_constant__ Batch batch, uint4 *__restrict__ hdr,
                                                          uint4 *__restrict__ desc) {
  extern __shared__ __align__(16) uint8_t psm[];
  uint8_t *lmap = psm;                      // kMaxWindow / 16 level granules
  uint8_t *buf = psm + kMaxWindow / 16;     // the staged block (kStageCap bytes)
  const int lane = threadIdx.x;
  for (int64_t blk = blockIdx.x; blk < batch.total_blocks; blk += gridDim.x) {
    int64_t b;
    const Job &jb = find_job(batch, blk, b);
    const uint32_t olen = block_len(jb, b);
    const uint64_t s0 = jb.offsets[b], s1 = jb.offsets[b + 1];
    uint32_t n = 0, st, lmax = 0;
    if (s1 < s0 || s1 > jb.comp_bytes) {
      st = LT_ERR_CORRUPT_STREAM;
    } else {
      StagedBlock r;
      r.buf = buf;
      r.lane = lane;
      r.beg = jb.comp + s0;
      r.end = jb.comp + s1;
      r.a0 = reinterpret_cast<const uint8_t *>(reinterpret_cast<uintptr_t>(r.beg) & ~uintptr_t(15));
      const uint64_t span = (uint64_t)(r.end - r.a0);
      if (span > kStageCap) {  // too long to stage: the ring walk, in the buffer's first 2 KB
        WarpRing w;
        w.buf = buf;
        w.lane = lane;
        w.beg = r.beg;
        w.end = r.end;
        w.a0 = r.a0;
        w.total = (uint32_t)((w.end - w.a0 + kPChunk - 1) / kPChunk);
        w.issued = 0;
        w.done = 0;
        w.top_up(0);
        st = parse_block(w, olen, win_cap(batch.max_block_bytes), lmap, desc + blk * kCap, n, lmax);
      } else {
        const uint32_t nch = (uint32_t)((span + 15) / 16);
        for (uint32_t c = (uint32_t)lane; c < nch; c += 32) {
          const uint8_t *src = r.a0 + 16 * c;
          uint8_t *dst = buf + 16 * c;
          if (src >= r.beg) {
            const uint32_t nb = (uint32_t)((r.end - src) < 16 ? (r.end - src) : 16);
            cp_async16(dst, src, nb);  // the rest of the 16 bytes is zero-filled
          } else {
            for (uint32_t i = 0; i < 16; ++i)
              if (src + i >= r.beg && src + i < r.end) dst[i] = __ldg(src + i);
          }
        }
        cp_async_commit();
        cp_async_wait<0>();
        __syncwarp();
        st = parse_block(r, olen, win_cap(batch.max_block_bytes), lmap, desc + blk * kCap, n, lmax);
      }
    }
    if (lane == 0) hdr[blk] = make_uint4(n, st, lmax, win_cap(batch.max_block_bytes));
    __syncwarp();  // the buffer is refilled for the next block only after every lane is done with it
  }
}

// ---------------------------------------------------------------------------
// fallback: warp 0 walks the block from global memory itself (lockstep,
// warp-uniform control flow). Returns 0 or a stream status.
// ---------------------------------------------------------------------------
__device__ int walk_block_warp(const uint8_t *__restrict__ src, uint64_t ilen, uint8_t *win, uint32_t olen,
                               int lane) {
  if (ilen == 0) return olen == 0 ? 0 : LT_ERR_SIZE_MISMATCH;
  uint64_t ip = 0;
  uint32_t op = 0;
  for (;;) {
    if (ip >= ilen) return LT_ERR_CORRUPT_STREAM;
    const uint32_t token = __ldg(src + ip++);
    uint64_t lit = token >> 4;
    if (lit == 15) {
      uint32_t bb;
      do {
        if (ip >= ilen || lit > olen) return LT_ERR_CORRUPT_STREAM;
        bb = __ldg(src + ip++);
        lit += bb;
      } while (bb == 255);
    }
    if (ip + lit > ilen || (uint64_t)op + lit > olen) return LT_ERR_CORRUPT_STREAM;
    for (uint32_t i = lane; i < (uint32_t)lit; i += 32) win[op + i] = __ldg(src + ip + i);
    ip += lit;
    op += (uint32_t)lit;
    __syncwarp();
    if (ip == ilen) break;
    if (ip + 2 > ilen) return LT_ERR_CORRUPT_STREAM;
    const uint32_t d = (uint32_t)__ldg(src + ip) | ((uint32_t)__ldg(src + ip + 1) << 8);
    ip += 2;
    if (d == 0 || d > op) return LT_ERR_CORRUPT_STREAM;
    uint64_t mlen = (token & 15u) + 4;
    if ((token & 15u) == 15u) {
      uint32_t bb;
      do {
        if (ip >= ilen || mlen > olen) return LT_ERR_CORRUPT_STREAM;
        bb = __ldg(src + ip++);
        mlen += bb;
      } while (bb == 255);
    }
    if ((uint64_t)op + mlen > olen) return LT_ERR_CORRUPT_STREAM;
    copy_match<32>(win, op, d, (uint32_t)mlen, lane, 0xFFFFFFFFu);
    __syncwarp();
    op += (uint32_t)mlen;
  }
  return op == olen ? 0 : LT_ERR_SIZE_MISMATCH;
}

// ---------------------------------------------------------------------------
// 2. expand
// ---------------------------------------------------------------------------

// first k in [0, n) with a[k] > v (n if none); a non-decreasing
__device__ __forceinline__ uint32_t upper_bound(const uint32_t *a, uint32_t n, int64_t v) {
  uint32_t lo = 0, hi = n;
  while (lo < hi) {
    const uint32_t mid = (lo + hi) >> 1;
    if ((int64_t)a[mid] > v) hi = mid;
    else lo = mid + 1;
  }
  return lo;
}

constexpr int kResolved = 0, kResolveFallback = 1, kResolveSkip = 2;

// Per-block state of the expansion, in shared memory.
struct Seqs {
  uint32_t op[kCap + 1];  // output position of sequence k's literals; op[n] = block length
  uint32_t md[kCap];      // output position of its match (op[k + 1] is the match's end)
  uint32_t le[kCap];      // end of its literal run in the block
  uint16_t dist[kCap];    // its match offset (0: no match)
  uint16_t lvl[kCap];     // its match level (0: no match)
  union alignas(16) {  // (16-byte aligned: the checked decode keeps 8-byte hash terms in it)
    uint16_t seg[kMaxWindow / 256];  // literals: last sequence starting at or before byte 256 s
    struct {
      uint32_t start[kLevelCap + 1];  // matches: first slot of each level in `order` (level counts first)
      uint16_t order[kCap];           // sequences with a match, by level
    } m;
  } u;
  uint32_t tail_level;  // levels from here on hold at most kTailMatches matches in all
};

// Rebuild one block whose sequence index is in the workspace (n <= kCap
// sequences, staged in place by the parse's rule). All threads of the CTA.
//  a. stage: the compressed bytes go to the end of the window (16-byte
//     cp.async copies), the index into Seqs;
//  b. literals: in rounds of 32 output bytes per thread, in output order.
//     Each thread reads the staged literal bytes of its eight output words
//     (one 4-byte gather per word), the CTA syncs, and the thread stores
//     them (bytes of a match are written too, with junk: the matches
//     overwrite them).
//     The parse checked that a literal's output position never lies past
//     its staged position, so a round's stores only hit staged bytes whose
//     output lies in this round or earlier ones -- bytes already read;
//  c. matches, one level at a time (levels come from the parse: a match
//     reads only literals and matches of lower levels), 8 lanes per match,
//     a CTA barrier between levels.
// Returns kResolveFallback before any output byte is written if the index is
// not one the parse can have written (the caller then walks the block
// itself), kResolveSkip if `check_staged` (given the window index of the
// staged block's first byte and its length, called by every thread once the
// block is staged) says the block is not to be decoded, else kResolved.
template <typename Check>
__device__ __forceinline__ int resolve_block(uint8_t *win, Seqs &S, const uint8_t *beg, uint32_t ilen, uint32_t olen,
                                             uint32_t n, uint32_t lmax, uint32_t wcap, const uint4 *__restrict__ dsc,
                                             Check &&check_staged) {
  const uint32_t tid = threadIdx.x;
  const int lane = tid & 31;
  // a. stage
  const uint32_t lead = (uint32_t)(reinterpret_cast<uintptr_t>(beg) & 15);
  const uint32_t iend = lead + ilen;
  const uint32_t so16 = (wcap - iend) & ~15u;
  const uint32_t S0 = so16 + lead;  // window index of staged block byte 0
  const uint8_t *a0 = beg - lead;
  const uint8_t *end = beg + ilen;
  const uint32_t nch = (iend + 15) / 16;
  for (uint32_t c = tid; c < nch; c += kThreads) {
    const uint8_t *src = a0 + 16 * c;
    uint8_t *dst = win + so16 + 16 * c;
    if (src >= beg) {
      const uint32_t nb = (uint32_t)((end - src) < 16 ? (end - src) : 16);
      cp_async16(dst, src, nb);  // the rest of the 16 bytes is zero-filled
    } else {
      for (uint32_t i = 0; i < 16; ++i)
        if (src + i >= beg && src + i < end) dst[i] = __ldg(src + i);
    }
  }
  cp_async_commit();
  // every index the expansion reads or writes stays inside the window if,
  // for all k: op[k] <= md[k] <= op[k + 1] <= olen, the literal run lies in
  // the block, and a match's offset reaches no further back than byte 0
  bool bad = false;
  if (lmax > kLevelCap) bad = true;
  for (uint32_t j = tid; j < n; j += kThreads) {
    const uint4 e = dsc[j];
    const uint32_t d = e.w & 0xFFFFu, ls = e.x & 0x1FFFFu, lv = e.x >> 17;
    const uint32_t md = e.y + e.z;
    if (e.y > olen || e.z > olen - e.y || ls > ilen || e.z > ilen - ls || d > md || (d != 0) != (lv != 0) ||
        lv > lmax)
      bad = true;
    S.op[j] = e.y;
    S.md[j] = md;
    S.le[j] = ls + e.z;
    S.dist[j] = (uint16_t)d;
    S.lvl[j] = (uint16_t)lv;
  }
  if (tid == 0) S.op[n] = olen;
  __syncthreads();
  for (uint32_t j = tid; j < n; j += kThreads)
    if (S.md[j] > S.op[j + 1]) bad = true;
  const uint32_t nseg = (olen + 255) / 256;
  for (uint32_t sg = tid; sg < nseg; sg += kThreads) {
    const uint32_t u = upper_bound(S.op, n, 256 * sg);
    S.u.seg[sg] = (uint16_t)(u ? u - 1 : 0u);
  }
  cp_async_wait<0>();
  if (__syncthreads_or(bad)) return kResolveFallback;
  // checked decode: the staged copy of the block is hashed here, before the
  // literal rounds overwrite it
  if (check_staged(S0, ilen)) return kResolveSkip;

  // b. literals. A 4-byte output word holds literals of at most one run
  // (two runs are separated by a match of at least 4 bytes), so each word
  // is one 4-byte gather from the staged bytes at that run's offset.
  for (uint32_t r0 = 0; r0 < olen; r0 += 32 * kThreads) {
    const uint32_t p0 = r0 + 32 * tid;
    uint32_t w[8] = {0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u};
    bool any = false;
    if (p0 < olen) {
      uint32_t k = S.u.seg[p0 >> 8];
      uint32_t o = S.op[k], m = S.md[k], nx = S.op[k + 1];
      int32_t delta = (int32_t)(S0 + S.le[k] - m);  // staged index of output byte p is p + delta (within k's literals)
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        const uint32_t p = p0 + 4 * q;
        if (p < olen) {
          while (nx <= p + 3 && k + 1 < n) {  // k: the last sequence starting at or before the word's last byte
            ++k;
            o = nx;
            m = S.md[k];
            nx = S.op[k + 1];
            delta = (int32_t)(S0 + S.le[k] - m);
          }
          if (p < m && p + 4 > o) {
            w[q] = gather4_window(win, (int32_t)p + delta);
            any = true;
          }
        }
      }
    }
    __syncthreads();
    if (any) {
      if (p0 + 32 <= olen) {
        *reinterpret_cast<uint4 *>(win + p0) = make_uint4(w[0], w[1], w[2], w[3]);
        *reinterpret_cast<uint4 *>(win + p0 + 16) = make_uint4(w[4], w[5], w[6], w[7]);
      } else {
#pragma unroll
        for (uint32_t i = 0; i < 32; ++i)
          if (p0 + i < olen) win[p0 + i] = (uint8_t)(w[i >> 2] >> (8 * (i & 3)));
      }
    }
  }

  // c. matches, one level at a time
  if (lmax >= kLevelCap) {  // levels saturated: warp 0 replays every match in order
    __syncthreads();
    if (tid < 32) {
      for (uint32_t j0 = 0; j0 < n; j0 += 32) {
        const uint32_t jl = j0 + (uint32_t)lane;
        unsigned pm = __ballot_sync(0xFFFFFFFFu, jl < n && S.dist[jl] != 0);
        while (pm) {
          const uint32_t j = j0 + (uint32_t)(__ffs(pm) - 1);
          pm &= pm - 1;
          const uint32_t md = S.md[j];
          copy_match<32>(win, md, S.dist[j], S.op[j + 1] - md, lane, 0xFFFFFFFFu);
          __syncwarp();
        }
      }
    }
    return kResolved;
  }
  // counting sort of the matches by level into S.u.m.order
  for (uint32_t i = tid; i <= kLevelCap; i += kThreads) S.u.m.start[i] = 0;
  __syncthreads();
  uint32_t rank[2];
#pragma unroll
  for (int q = 0; q < 2; ++q) {
    const uint32_t j = tid + (uint32_t)q * kThreads;
    rank[q] = (j < n && S.lvl[j]) ? atomicAdd(&S.u.m.start[S.lvl[j]], 1u) : 0u;
  }
  __syncthreads();
  if (tid < 32) {  // exclusive scan of the level counts (levels 1..lmax; 8 per lane)
    uint32_t c[8], sum = 0;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const uint32_t lv = 8 * (uint32_t)lane + (uint32_t)i;
      c[i] = lv <= kLevelCap ? S.u.m.start[lv] : 0u;
      sum += c[i];
    }
    uint32_t incl = sum;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t v = __shfl_up_sync(0xFFFFFFFFu, incl, o);
      if (lane >= o) incl += v;
    }
    uint32_t run = incl - sum;
    const uint32_t total = __shfl_sync(0xFFFFFFFFu, incl, 31);
    uint32_t tail = lmax + 1;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const uint32_t lv = 8 * (uint32_t)lane + (uint32_t)i;
      if (lv <= kLevelCap) S.u.m.start[lv] = run;
      if (lv >= 1 && lv <= lmax && total - run <= kTailMatches && lv < tail) tail = lv;
      run += c[i];
    }
    tail = __reduce_min_sync(0xFFFFFFFFu, tail);
    if (lane == 0) S.tail_level = tail;
  }
  __syncthreads();
#pragma unroll
  for (int q = 0; q < 2; ++q) {
    const uint32_t j = tid + (uint32_t)q * kThreads;
    if (j < n && S.lvl[j]) S.u.m.order[S.u.m.start[S.lvl[j]] + rank[q]] = (uint16_t)j;
  }
  __syncthreads();
  // level by level: 8 lanes per match, four matches per warp at a time;
  // the last few matches by warp 0 alone (no CTA barriers)
  const int warp = (int)(tid >> 5), sub = lane >> 3;
  const uint32_t tail = S.tail_level;
  for (uint32_t lv = 1; lv < tail; ++lv) {
    const uint32_t a = S.u.m.start[lv], end = S.u.m.start[lv + 1];  // lmax < kLevelCap: start[lmax + 1] = all matches
    for (uint32_t base = a + 4 * (uint32_t)warp; base < end; base += 4 * kWarps) {
      const uint32_t i = base + (uint32_t)sub;
      if (i < end) {
        const uint32_t j = S.u.m.order[i];
        const uint32_t md = S.md[j];
        copy_match<8>(win, md, S.dist[j], S.op[j + 1] - md, lane & 7, 0xFFu << (8 * sub));
      }
      __syncwarp();
    }
    __syncthreads();
  }
  if (tid < 32) {
    for (uint32_t lv = tail; lv <= lmax; ++lv) {
      const uint32_t a = S.u.m.start[lv], end = S.u.m.start[lv + 1];
      for (uint32_t base = a; base < end; base += 4) {
        const uint32_t i = base + (uint32_t)sub;
        if (i < end) {
          const uint32_t j = S.u.m.order[i];
          const uint32_t md = S.md[j];
          copy_match<8>(win, md, S.dist[j], S.op[j + 1] - md, lane & 7, 0xFFu << (8 * sub));
        }
        __syncwarp();
      }
    }
  }
  return kResolved;
}

// Checked decode: does block b's XXH3-64 (batch's secret) differ from the
// expected value? One warp; every lane returns the answer. An offset pair
// outside the stream is not hashed (the decode reports it). Kept out of
// line so that the hash's registers do not weigh on the expand loop.
__device__ __noinline__ bool block_hash_differs(const Batch &batch, const Job &jb, int64_t b, int64_t blk, int lane) {
  const uint64_t c0 = jb.offsets[b], c1 = jb.offsets[b + 1];
  if (c0 > c1 || c1 > jb.comp_bytes) return false;
  const uint64_t len = c1 - c0;
  const uint8_t *in = jb.comp + c0;
  const GlobalBytes din{jb.comp, jb.comp + jb.comp_bytes}, dsec{batch.secret, batch.secret + batch.secret_len};
  uint64_t h;
  if (len > 240)
    h = xxh3::hash64_long_warp([&](uint64_t off) { return din.rd64(in + off); },
                               [&](uint64_t off) { return dsec.rd64(batch.secret + off); }, len, batch.secret_len,
                               lane);
  else
    h = __shfl_sync(0xFFFFFFFFu, lane == 0 ? xxh3::hash64(in, len, batch.secret, batch.secret_len) : 0ull, 0);
  return h != batch.expected[blk];
}

// The same check on the block's staged copy in shared memory: window bytes
// [S0, S0 + ilen), by the whole CTA (every thread calls it and gets the
// answer). The terms of up to kHashChunk scramble intervals are computed by
// the eight warps side by side into `terms` (kHashChunk x 8 words of shared
// memory), then warp 0 applies them in order. Out of line for the same
// reason as above.
constexpr int kHashChunk = 24;
__device__ __noinline__ bool staged_hash_differs(const Batch &batch, const uint8_t *win, uint32_t S0, uint32_t ilen,
                                                 int64_t blk, uint64_t *terms, uint32_t *flag) {
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  // 8 bytes of the staged block at offset off: two aligned 8-byte loads (the
  // window is 16-byte aligned and padded past its end)
  auto rd = [&](uint64_t off) -> uint64_t {
    const uint32_t x = S0 + (uint32_t)off, sh = (x & 7u) * 8u;
    const uint64_t *w = reinterpret_cast<const uint64_t *>(win + (x & ~7u));
    return sh ? (w[0] >> sh) | (w[1] << (64u - sh)) : w[0];
  };
  const GlobalBytes dsec{batch.secret, batch.secret + batch.secret_len};
  auto rk = [&](uint64_t off) { return dsec.rd64(batch.secret + off); };
  uint64_t h = 0;
  if (ilen <= 240) {
    if (tid == 0) h = xxh3::hash64(win + S0, ilen, batch.secret, batch.secret_len);
  } else {
    const uint64_t per_block = (batch.secret_len - 64) / 8, block_len = 64 * per_block;
    const uint64_t nb = ((uint64_t)ilen - 1) / block_len;
    uint64_t acc = xxh3::acc_init(lane & 7);
    const uint64_t scr = rk(batch.secret_len - 64 + 8 * (uint64_t)(lane & 7));
    for (uint64_t c0 = 0; c0 < nb; c0 += kHashChunk) {
      const uint64_t cn = (nb - c0) < (uint64_t)kHashChunk ? (nb - c0) : (uint64_t)kHashChunk;
      for (uint64_t j = (uint64_t)warp; j < cn; j += kWarps) {
        const uint64_t t = xxh3::stripe_terms(rd, rk, (c0 + j) * block_len, per_block, 0, lane);
        if (lane < 8) terms[8 * j + lane] = t;
      }
      __syncthreads();
      if (warp == 0)
        for (uint64_t j = 0; j < cn; ++j) acc = xxh3::scramble(acc + terms[8 * j + (lane & 7)], scr);
      __syncthreads();
    }
    if (warp == 0) h = xxh3::finish_long(rd, rk, acc, ilen, batch.secret_len, nb, lane);
  }
  if (tid == 0) *flag = h != batch.expected[blk] ? 1u : 0u;
  __syncthreads();
  return *flag != 0;
}

template <bool FUSED, bool CHECKED>
__global__ void __launch_bounds__(kThreads, 3) k_lz4_expand(const __grid_constant__ Batch batch,
                                                          const uint4 *__restrict__ hdr,
                                                          const uint4 *__restrict__ desc, int32_t *d_status) {
  extern __shared__ uint4 smem_u4[];
  uint8_t *win = reinterpret_cast<uint8_t *>(smem_u4) + kPad;
  __shared__ Seqs S;
  __shared__ uint32_t s_n, s_st, s_lmax, s_badsum, s_hashflag;
  const uint32_t wcap = win_cap(batch.max_block_bytes);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  for (int64_t blk = blockIdx.x; blk < batch.total_blocks; blk += gridDim.x) {
    int64_t b;
    const Job &jb = find_job(batch, blk, b);
    const int64_t d0 = b * (int64_t)jb.block_bytes;
    const uint32_t olen = block_len(jb, b);
    if (threadIdx.x == 0) {
      const uint4 h = hdr ? hdr[blk] : make_uint4(0u, kNoIndex, 0u, 0u);
      s_n = h.x;
      s_st = h.y;
      s_lmax = h.z;
      if (h.y == 0 && h.w != wcap) s_st = kNoIndex;  // indexed for another window size: walk the block instead
    }
    __syncthreads();
    const uint32_t n = s_n, lmax = s_lmax;
    uint32_t st = s_st;
    const uint64_t s0 = jb.offsets[b], s1 = jb.offsets[b + 1];
    const uint32_t lead = (uint32_t)(reinterpret_cast<uintptr_t>(jb.comp + s0) & 15);
    if (st == 0 && (n > kCap || s1 < s0 || s1 > jb.comp_bytes || s1 - s0 + lead > wcap))
      st = kNoIndex;  // never from the parse
    // Checked decode: each block's checksum comes first, so that a damaged
    // block is reported as a checksum mismatch (and not decoded) whatever
    // else is wrong with it. A block that is staged for decoding is hashed
    // from its staged copy (resolve_block); any other from global memory here.
    auto mismatch = [&](bool bad) {
      if (lane == 0) {
        s_badsum = bad ? 1u : 0u;
        if (bad) {
          report(d_status, LT_ERR_CHECKSUM);
          if (batch.first_bad) atomicMin(batch.first_bad, (unsigned long long)blk);
        }
      }
    };
    if (CHECKED && st != 0) {
      if (warp == 0) mismatch(block_hash_differs(batch, jb, b, blk, lane));
      __syncthreads();
      if (s_badsum) {  // not decoded (output unspecified)
        __syncthreads();
        continue;
      }
    }
    if (st != 0 && st != kOverflow && st != kNoIndex && st != kNoInPlace) {
      // the parse found a malformed block: report it; its output stays unwritten
      if (threadIdx.x == 0) report(d_status, (int32_t)st);
      __syncthreads();
      continue;
    }
    if (st == 0) {
      auto check_staged = [&](uint32_t S0, uint32_t ilen) -> bool {
        if (!CHECKED) return false;
        // the hash terms use the part of S.u that the literal rounds' segment
        // table (its first 512 bytes) leaves free until the match phase
        uint64_t *terms = reinterpret_cast<uint64_t *>(reinterpret_cast<uint8_t *>(&S.u) + 512);
        const bool bad = staged_hash_differs(batch, win, S0, ilen, blk, terms, &s_hashflag);
        if (warp == 0) mismatch(bad);
        __syncthreads();
        return bad;
      };
      const int rs = resolve_block(win, S, jb.comp + s0, (uint32_t)(s1 - s0), olen, n, lmax, wcap,
                                   desc + blk * kCap, check_staged);
      if (rs == kResolveSkip) {  // checksum mismatch: not decoded (output unspecified)
        __syncthreads();
        continue;
      }
      if (rs == kResolveFallback) st = kNoIndex;
    }
    if (st != 0 && warp == 0) {
      int err = LT_ERR_CORRUPT_STREAM;
      if (s0 <= s1 && s1 <= jb.comp_bytes) err = walk_block_warp(jb.comp + s0, s1 - s0, win, olen, lane);
      if (err && lane == 0) report(d_status, err);  // content unspecified after an error
    }
    __syncthreads();
    if (FUSED) {
      uint16_t *out = reinterpret_cast<uint16_t *>(jb.out);
      const int64_t k0 = 2 * d0;  // first code of the block
      const int64_t k_end = (k0 + 2 * (int64_t)olen) < jb.n_codes ? (k0 + 2 * (int64_t)olen) : jb.n_codes;
      const uint32_t nk = (uint32_t)(k_end - k0);  // codes in this block (<= 131072)
      const int64_t G = jb.group_size;
      const int gs = jb.group_shift;
      const bool vec = (G % 8 == 0) && aligned(out + k0, 16);
      const int64_t g0 = gs >= 0 ? (k0 >> gs) : 0;
      const uint32_t koff = gs >= 0 ? (uint32_t)(k0 - (g0 << gs)) : 0u;
      const uint32_t nw = (nk + 7) / 8;  // window words (8 codes each)
      const uint32_t nq = (nw + 3) / 4;  // units of 4 words = 32 codes
      if (vec && G % 32 == 0 && gs >= 0) {
        // a unit lies in one group (units start at multiples of 32 codes);
        // the scales and zero points of 8 units are loaded before any is used
        for (uint32_t q0 = threadIdx.x; q0 < nq; q0 += 8 * kThreads) {
          uint32_t sc[8], zr[8];
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const uint32_t q = q0 + (uint32_t)i * kThreads;
            const int64_t g = g0 + (int64_t)((koff + 32 * (q < nq ? q : 0u)) >> gs);
            sc[i] = q < nq ? __ldg(jb.scales + g) : 0u;
            zr[i] = q < nq && jb.zeros ? __ldg(jb.zeros + g) : 0u;
          }
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const uint32_t q = q0 + (uint32_t)i * kThreads;
            if (q >= nq) break;
            const uint32_t kr = 32 * q;
            const uint32_t s2 = bcast_half((uint16_t)sc[i]);
            const uint32_t zm = jb.zeros ? int4_zero_magic((uint8_t)zr[i]) : 0x54006400u;
            if (kr + 32 <= nk) {
              const uint4 v = reinterpret_cast<const uint4 *>(win)[q];
              uint16_t *o = out + k0 + kr;
              st_u128(o, int4x8_dequant(v.x, zm, s2));
              st_u128(o + 8, int4x8_dequant(v.y, zm, s2));
              st_u128(o + 16, int4x8_dequant(v.z, zm, s2));
              st_u128(o + 24, int4x8_dequant(v.w, zm, s2));
            } else {  // the block's last, partial unit
              for (uint32_t kk = kr; kk < nk; ++kk) {
                const uint8_t byte = win[kk >> 1];
                const int32_t qv = (kk & 1) ? (byte >> 4) : (byte & 0x0F);
                const int64_t g = (k0 + kk) / G;
                const int32_t z = jb.zeros ? jb.zeros[g] : 0;
                out[k0 + kk] = dequant_scalar(qv - z, jb.scales[g]);
              }
            }
          }
        }
      } else {
        for (uint32_t wi = threadIdx.x; wi < nw; wi += kThreads) {
          const uint32_t kw = 8 * wi;
          if (vec && kw + 8 <= nk) {
            const int64_t g = gs >= 0 ? g0 + (int64_t)((koff + kw) >> gs) : (k0 + kw) / G;
            const uint32_t s2 = bcast_half(__ldg(jb.scales + g));
            const uint32_t zm = jb.zeros ? int4_zero_magic(__ldg(jb.zeros + g)) : 0x54006400u;
            st_u128(out + k0 + kw, int4x8_dequant(reinterpret_cast<const uint32_t *>(win)[wi], zm, s2));
          } else {
            const uint32_t ke = (kw + 8) < nk ? (kw + 8) : nk;
            for (uint32_t kk = kw; kk < ke; ++kk) {
              const uint8_t byte = win[kk >> 1];
              const int32_t qv = (kk & 1) ? (byte >> 4) : (byte & 0x0F);
              const int64_t g = (k0 + kk) / G;
              const int32_t z = jb.zeros ? jb.zeros[g] : 0;
              out[k0 + kk] = dequant_scalar(qv - z, jb.scales[g]);
            }
          }
        }
      }
    } else {
      uint8_t *out = reinterpret_cast<uint8_t *>(jb.out) + d0;
      if (aligned(out, 16)) {
        const uint32_t n16 = olen / 16;
        for (uint32_t i = threadIdx.x; i < n16; i += kThreads)
          st_u128(reinterpret_cast<uint4 *>(out) + i, reinterpret_cast<const uint4 *>(win)[i]);
        for (uint32_t i = 16 * n16 + threadIdx.x; i < olen; i += kThreads) out[i] = win[i];
      } else {
        for (uint32_t i = threadIdx.x; i < olen; i += kThreads) out[i] = win[i];
      }
    }
    __syncthreads();
  }
}

uint64_t workspace_need(int64_t total_blocks) { return (uint64_t)total_blocks * (16ull + 16ull * kCap) + 256; }

// The sequence index of `total` blocks in a workspace: a header per block,
// then kCap descriptors per block, from the first 256-byte boundary.
void index_arrays(const void *ws, int64_t total, uint4 *&hdr, uint4 *&desc) {
  uintptr_t p = (reinterpret_cast<uintptr_t>(ws) + 255) & ~uintptr_t(255);
  hdr = reinterpret_cast<uint4 *>(p);
  desc = hdr + total;
}

void launch_parse(const Batch &batch, uint4 *hdr, uint4 *desc, cudaStream_t st) {
  // Few blocks per SM (e.g. one 4096 x 14336 matrix: 448 blocks): each
  // block's walk is a latency chain, so the lean walk over a fully staged
  // block wins. Many blocks per SM (a whole model's layers): the walks are
  // issue-bound and the ring's small footprint keeps 36 of them per SM.
  const int64_t sms = num_sms();
  if (batch.total_blocks <= 4 * sms) {
    const size_t smem = kMaxWindow / 16 + kStageCap;
    static int attr_set[64] = {0};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev >= 0 && dev < 64 && !attr_set[dev]) {
      cudaFuncSetAttribute(k_lz4_parse_staged, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
      attr_set[dev] = 1;
    }
    k_lz4_parse_staged<<<(int)batch.total_blocks, 32, smem, st>>>(batch, hdr, desc);
    return;
  }
  const int64_t need = (batch.total_blocks + kParseWarps - 1) / kParseWarps;
  const int64_t cap = (int64_t)num_sms() * blocks_per_sm((const void *)k_lz4_parse, kParseWarps * 32, 0);
  k_lz4_parse<<<(int)(need < cap ? need : cap), kParseWarps * 32, 0, st>>>(batch, hdr, desc);
}

lt_status launch_expand(const Batch &batch, bool fused, const uint4 *hdr, const uint4 *desc, int32_t *d_status,
                        cudaStream_t st);

lt_status launch(const Batch &batch, bool fused, void *workspace, uint64_t workspace_bytes, int32_t *d_status,
                 cudaStream_t st) {
  if (batch.total_blocks == 0) return LT_OK;
  uint4 *hdr = nullptr, *desc = nullptr;
  if (workspace && workspace_bytes >= workspace_need(batch.total_blocks)) {
    index_arrays(workspace, batch.total_blocks, hdr, desc);
    launch_parse(batch, hdr, desc, st);
  }
  return launch_expand(batch, fused, hdr, desc, d_status, st);
}

lt_status launch_expand(const Batch &batch, bool fused, const uint4 *hdr, const uint4 *desc, int32_t *d_status,
                        cudaStream_t st) {
  if (batch.total_blocks == 0) return LT_OK;
  const size_t smem = (size_t)win_cap(batch.max_block_bytes) + 2 * kPad;
  const bool checked = fused && batch.secret != nullptr;
  const int variant = checked ? 2 : (fused ? 1 : 0);
  const void *k = checked ? (const void *)k_lz4_expand<true, true>
                          : (fused ? (const void *)k_lz4_expand<true, false> : (const void *)k_lz4_expand<false, false>);
  static int attr_set[3][64] = {{0}};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev >= 0 && dev < 64 && !attr_set[variant][dev]) {
    cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)win_cap(kMaxWindow) + 2 * kPad);
    attr_set[variant][dev] = 1;
  }
  const int64_t cap = (int64_t)num_sms() * blocks_per_sm(k, kThreads, smem);
  const int grid = (int)(batch.total_blocks < cap ? batch.total_blocks : cap);
  if (checked)
    k_lz4_expand<true, true><<<grid, kThreads, smem, st>>>(batch, hdr, desc, d_status);
  else if (fused)
    k_lz4_expand<true, false><<<grid, kThreads, smem, st>>>(batch, hdr, desc, d_status);
  else
    k_lz4_expand<false, false><<<grid, kThreads, smem, st>>>(batch, hdr, desc, d_status);
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

LT_API uint64_t lt_lz4_workspace_bytes(int64_t n_blocks) { return n_blocks > 0 ? workspace_need(n_blocks) : 0; }

LT_API lt_status lt_lz4_int4_decode(const uint8_t *comp, uint64_t comp_bytes, const uint64_t *block_offsets,
                                    int32_t block_bytes, const lt_half *scales, const uint8_t *zeros, int64_t rows,
                                    int64_t cols, int32_t group_size, lt_half *out, void *workspace,
                                    uint64_t workspace_bytes, int32_t *d_status, lt_stream_t stream) {
  if (!aligned(d_status, 4) || !aligned(workspace, 16)) return LT_ERR_MISALIGNED;
  Batch batch = empty_batch();
  lt_status s = add_fused_job(batch, comp, comp_bytes, block_offsets, block_bytes, scales, zeros, rows, cols,
                              group_size, out);
  if (s != LT_OK) return s;
  return launch(batch, true, workspace, workspace_bytes, d_status, (cudaStream_t)stream);
}

LT_API lt_status lt_lz4_int4_decode_batch(const lt_lz4_int4_desc *descs, int32_t n_desc, void *workspace,
                                          uint64_t workspace_bytes, int32_t *d_status, lt_stream_t stream) {
  if (n_desc < 1 || !descs) return LT_ERR_INVALID_ARG;
  if (n_desc > LT_LZ4_BATCH_MAX) return LT_ERR_UNSUPPORTED;
  if (!aligned(d_status, 4) || !aligned(workspace, 16)) return LT_ERR_MISALIGNED;
  Batch batch = empty_batch();
  for (int32_t i = 0; i < n_desc; ++i) {
    const lt_lz4_int4_desc &d = descs[i];
    lt_status s = add_fused_job(batch, d.comp, d.comp_bytes, d.block_offsets, d.block_bytes, d.scales, d.zeros,
                                d.rows, d.cols, d.group_size, d.out);
    if (s != LT_OK) return s;
  }
  return launch(batch, true, workspace, workspace_bytes, d_status, (cudaStream_t)stream);
}

LT_API lt_status lt_lz4_int4_decode_checked(const uint8_t *comp, uint64_t comp_bytes, const uint64_t *block_offsets,
                                            int32_t block_bytes, const lt_half *scales, const uint8_t *zeros,
                                            int64_t rows, int64_t cols, int32_t group_size, lt_half *out,
                                            void *workspace, uint64_t workspace_bytes, const uint8_t *secret,
                                            int32_t secret_len, const uint64_t *expected_hashes, int32_t *d_status,
                                            uint64_t *d_first_bad, lt_stream_t stream) {
  if (!aligned(d_status, 4) || !aligned(workspace, 16) || !aligned(d_first_bad, 8)) return LT_ERR_MISALIGNED;
  if (!secret || secret_len < (int32_t)xxh3::kSecretMin || !expected_hashes) return LT_ERR_INVALID_ARG;
  if (!aligned(expected_hashes, 8)) return LT_ERR_MISALIGNED;
  Batch batch = empty_batch();
  lt_status s = add_fused_job(batch, comp, comp_bytes, block_offsets, block_bytes, scales, zeros, rows, cols,
                              group_size, out);
  if (s != LT_OK) return s;
  batch.secret = secret;
  batch.secret_len = (uint32_t)secret_len;
  batch.expected = expected_hashes;
  batch.first_bad = reinterpret_cast<unsigned long long *>(d_first_bad);
  return launch(batch, true, workspace, workspace_bytes, d_status, (cudaStream_t)stream);
}

namespace lt {
namespace {
lt_status batch_from(const lt_lz4_int4_desc *descs, int32_t n_desc, Batch &batch) {
  if (n_desc < 1 || !descs) return LT_ERR_INVALID_ARG;
  if (n_desc > LT_LZ4_BATCH_MAX) return LT_ERR_UNSUPPORTED;
  for (int32_t i = 0; i < n_desc; ++i) {
    const lt_lz4_int4_desc &d = descs[i];
    lt_status s = add_fused_job(batch, d.comp, d.comp_bytes, d.block_offsets, d.block_bytes, d.scales, d.zeros,
                                d.rows, d.cols, d.group_size, d.out);
    if (s != LT_OK) return s;
  }
  return LT_OK;
}
}  // namespace
}  // namespace lt

LT_API lt_status lt_lz4_index_batch(const lt_lz4_int4_desc *descs, int32_t n_desc, void *index, uint64_t index_bytes,
                                    lt_stream_t stream) {
  Batch batch = empty_batch();
  lt_status s = batch_from(descs, n_desc, batch);
  if (s != LT_OK) return s;
  if (batch.total_blocks == 0) return LT_OK;
  if (!index || index_bytes < workspace_need(batch.total_blocks)) return LT_ERR_INVALID_ARG;
  if (!aligned(index, 16)) return LT_ERR_MISALIGNED;
  uint4 *hdr, *desc;
  index_arrays(index, batch.total_blocks, hdr, desc);
  launch_parse(batch, hdr, desc, (cudaStream_t)stream);
  return launch_status();
}

LT_API lt_status lt_lz4_int4_expand_batch(const lt_lz4_int4_desc *descs, int32_t n_desc, const void *index,
                                          uint64_t index_bytes, int64_t index_blocks, int64_t first_block,
                                          int32_t *d_status, lt_stream_t stream) {
  if (!aligned(d_status, 4)) return LT_ERR_MISALIGNED;
  Batch batch = empty_batch();
  lt_status s = batch_from(descs, n_desc, batch);
  if (s != LT_OK) return s;
  if (batch.total_blocks == 0) return LT_OK;
  if (!index || index_blocks < 1 || index_blocks > ((int64_t)1 << 40) || first_block < 0 ||
      first_block > index_blocks - batch.total_blocks || index_bytes < workspace_need(index_blocks))
    return LT_ERR_INVALID_ARG;
  if (!aligned(index, 16)) return LT_ERR_MISALIGNED;
  uint4 *hdr, *desc;
  index_arrays(index, index_blocks, hdr, desc);
  return launch_expand(batch, true, hdr + first_block, desc + first_block * kCap, d_status, (cudaStream_t)stream);
}

LT_API lt_status lt_lz4_decode(const uint8_t *comp, uint64_t comp_bytes, const uint64_t *block_offsets,
                               int32_t block_bytes, uint8_t *out, uint64_t out_bytes, void *workspace,
                               uint64_t workspace_bytes, int32_t *d_status, lt_stream_t stream) {
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
  if (workspace && !aligned(workspace, 16)) return LT_ERR_MISALIGNED;
  batch.max_block_bytes = block_bytes;
  return launch(batch, false, workspace, workspace_bytes, d_status, (cudaStream_t)stream);
}

// ---------------------------------------------------------------------------
// Entry point that allocates nothing: the fused decode with its sequence
// index kept in a fixed scratch array compiled into this library, for
// callers that may not allocate device memory themselves (see the header).
// ---------------------------------------------------------------------------
namespace lt {
namespace {

constexpr uint64_t kNoAllocBytes = (uint64_t)LT_NOALLOC_MAX_BLOCKS * (16ull + 16ull * kCap) + 256;

// One copy per GPU that loads the library, resident until the process
// exits. Host code only ever sees its address through the lookup below.
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocBytes];

std::mutex g_noalloc_mu;
struct NoAllocAddr {
  unsigned long long ctx_id;  // the context the address belongs to
  void *addr;
};
NoAllocAddr g_noalloc_addr[64] = {};

// Device address of g_noalloc_scratch in the current context. It is looked
// up on the first call in a context (with that device current) and kept per
// device together with the context's id; a call from a new context on that
// device -- e.g. after cudaDeviceReset, which destroys the primary context
// and with it this module's copy of the array -- looks it up again instead
// of using the old address.
lt_status noalloc_scratch(void **out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) {
    cudaGetLastError();
    return LT_ERR_CUDA;
  }
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  unsigned long long ctx = 0;
  const bool have_ctx = current_context_id(&ctx);
  if (!g_noalloc_addr[dev].addr || !have_ctx || g_noalloc_addr[dev].ctx_id != ctx) {
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) {
      cudaGetLastError();
      return LT_ERR_CUDA;
    }
    // cudaGetSymbolAddress made the primary context current if none was:
    // record the id of the context the address was taken in
    if (!have_ctx && !current_context_id(&ctx)) ctx = 0;
    g_noalloc_addr[dev] = NoAllocAddr{ctx, p};
  }
  *out = g_noalloc_addr[dev].addr;
  return LT_OK;
}

}  // namespace
}  // namespace lt

LT_API lt_status lt_lz4_int4_decode_noalloc(const uint8_t *comp, uint64_t comp_bytes, const uint64_t *block_offsets,
                                            int32_t block_bytes, const lt_half *scales, const uint8_t *zeros,
                                            int64_t rows, int64_t cols, int32_t group_size, lt_half *out,
                                            int32_t *d_status, lt_stream_t stream) {
  if (!aligned(d_status, 4)) return LT_ERR_MISALIGNED;
  Batch batch = empty_batch();
  lt_status s = add_fused_job(batch, comp, comp_bytes, block_offsets, block_bytes, scales, zeros, rows, cols,
                              group_size, out);
  if (s != LT_OK) return s;
  if (batch.total_blocks > LT_NOALLOC_MAX_BLOCKS) return LT_ERR_UNSUPPORTED;  // larger than the built-in scratch
  if (batch.total_blocks == 0) return LT_OK;
  void *scratch = nullptr;
  s = noalloc_scratch(&scratch);
  if (s != LT_OK) return s;
  // the parse pass writes every index entry the expand pass reads, so the
  // scratch needs no clearing between calls
  return launch(batch, true, scratch, kNoAllocBytes, d_status, (cudaStream_t)stream);
}
