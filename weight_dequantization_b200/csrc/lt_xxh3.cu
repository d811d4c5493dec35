// lt_xxh3.cu -- per-block XXH3-64 checksums of a compressed stream, and
// their verification ("GPU Compression Pipeline - TDD Roadmap", Phase 6.1
// HCT Format V2: XXH3 checksums that report a flipped byte as a mismatch).
//
// One CTA hashes one block: for blocks longer than 240 bytes its warps
// compute the terms of many scramble intervals side by side (lanes take the
// 8-byte words of 4 stripes at a time, a butterfly adds them), then warp 0
// applies them in order; shorter blocks by one thread with the sequential
// definition. The same hash, fused into the LZ4 decode, checks a
// block while it is staged for decoding (lt_lz4_int4_decode_checked).
#include "lt_common.cuh"
#include "lt_xxh3.cuh"

namespace lt {
namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kChunk = 64;  // scramble intervals whose terms are staged in shared memory at a time

// One CTA per block. The terms each scramble interval adds to the eight
// accumulators depend only on the data, so the warps compute them for up to
// kChunk intervals side by side (many loads in flight), then warp 0 applies
// them in order, scrambling after each; the tail, the last stripe and the
// merge follow.
__global__ void __launch_bounds__(kThreads)
    k_xxh3_blocks(const uint8_t *__restrict__ data, uint64_t data_bytes, const uint64_t *__restrict__ offsets,
                  int64_t n_blocks, const uint8_t *__restrict__ secret, uint32_t secret_len,
                  uint64_t *__restrict__ hashes, const uint64_t *__restrict__ expected, int32_t *d_status,
                  unsigned long long *d_first_bad) {
  __shared__ uint64_t terms[kChunk][8];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const GlobalBytes din{data, data + data_bytes}, dsec{secret, secret + secret_len};
  auto rk = [&](uint64_t off) { return dsec.rd64(secret + off); };
  const uint64_t per_block = (secret_len - 64) / 8, block_len = 64 * per_block;
  for (int64_t b = blockIdx.x; b < n_blocks; b += gridDim.x) {
    const uint64_t s0 = offsets[b], s1 = offsets[b + 1];
    if (s1 < s0 || s1 > data_bytes) {  // (uniform: every thread read the same offsets)
      if (threadIdx.x == 0) report(d_status, LT_ERR_CORRUPT_STREAM);
      continue;
    }
    const uint64_t len = s1 - s0;
    const uint8_t *in = data + s0;
    auto rd = [&](uint64_t off) { return din.rd64(in + off); };
    uint64_t h = 0;
    if (len <= 240) {
      if (threadIdx.x == 0) h = xxh3::hash64(in, len, secret, secret_len);
    } else {
      const uint64_t nb = (len - 1) / block_len;  // full scramble intervals
      uint64_t acc = xxh3::acc_init(lane & 7);
      const uint64_t scr = rk(secret_len - 64 + 8 * (uint64_t)(lane & 7));
      for (uint64_t c0 = 0; c0 < nb; c0 += kChunk) {
        const uint64_t cn = (nb - c0) < (uint64_t)kChunk ? (nb - c0) : (uint64_t)kChunk;
        for (uint64_t j = (uint64_t)warp; j < cn; j += kWarps) {
          const uint64_t t = xxh3::stripe_terms(rd, rk, (c0 + j) * block_len, per_block, 0, lane);
          if (lane < 8) terms[j][lane] = t;
        }
        __syncthreads();
        if (warp == 0)
          for (uint64_t j = 0; j < cn; ++j) acc = xxh3::scramble(acc + terms[j][lane & 7], scr);
        __syncthreads();
      }
      if (warp == 0) h = xxh3::finish_long(rd, rk, acc, len, secret_len, nb, lane);
    }
    if (threadIdx.x == 0) {
      if (hashes != nullptr) hashes[b] = h;
      if (expected != nullptr && expected[b] != h) {
        report(d_status, LT_ERR_CHECKSUM);
        if (d_first_bad != nullptr) atomicMin(d_first_bad, (unsigned long long)b);
      }
    }
  }
}

}  // namespace
}  // namespace lt

using namespace lt;

LT_API lt_status lt_xxh3_blocks(const uint8_t *data, uint64_t data_bytes, const uint64_t *offsets, int64_t n_blocks,
                                const uint8_t *secret, int32_t secret_len, uint64_t *hashes, const uint64_t *expected,
                                int32_t *d_status, uint64_t *d_first_bad, lt_stream_t stream) {
  if (n_blocks < 0 || secret_len < (int32_t)xxh3::kSecretMin) return LT_ERR_INVALID_ARG;
  if (n_blocks == 0) return LT_OK;
  if (!offsets || !secret || (!data && data_bytes != 0)) return LT_ERR_INVALID_ARG;
  if (!hashes && !expected) return LT_ERR_INVALID_ARG;
  if (!aligned(offsets, 8) || (hashes && !aligned(hashes, 8)) || (expected && !aligned(expected, 8)) ||
      (d_first_bad && !aligned(d_first_bad, 8)) || (d_status && !aligned(d_status, 4)))
    return LT_ERR_MISALIGNED;
  int64_t blocks = n_blocks;
  const int64_t cap = (int64_t)num_sms() * 8;
  if (blocks > cap) blocks = cap;
  k_xxh3_blocks<<<(int)blocks, kThreads, 0, (cudaStream_t)stream>>>(
      data, data_bytes, offsets, n_blocks, secret, (uint32_t)secret_len, hashes, expected, d_status,
      reinterpret_cast<unsigned long long *>(d_first_bad));
  return launch_status();
}
