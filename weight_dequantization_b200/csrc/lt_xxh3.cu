// lt_xxh3.cu -- per-block XXH3-64 checksums of a compressed stream, and
// their verification ("GPU Compression Pipeline - TDD Roadmap", Phase 6.1
// HCT Format V2: XXH3 checksums that report a flipped byte as a mismatch).
//
// One warp hashes one block: blocks longer than 240 bytes with the
// warp-cooperative long-input hash of lt_xxh3.cuh (lanes take the 8-byte
// words of 4 stripes at a time, 8-byte loads, a butterfly adds their terms
// within each scramble interval), shorter ones by lane 0 with the
// sequential definition. The same hash, fused into the LZ4 decode, checks a
// block while it is staged for decoding (lt_lz4_int4_decode_checked).
#include "lt_common.cuh"
#include "lt_xxh3.cuh"

namespace lt {
namespace {

constexpr int kThreads = 128;
constexpr int kWarps = kThreads / 32;

__global__ void __launch_bounds__(kThreads)
    k_xxh3_blocks(const uint8_t *__restrict__ data, uint64_t data_bytes, const uint64_t *__restrict__ offsets,
                  int64_t n_blocks, const uint8_t *__restrict__ secret, uint32_t secret_len,
                  uint64_t *__restrict__ hashes, const uint64_t *__restrict__ expected, int32_t *d_status,
                  unsigned long long *d_first_bad) {
  const int lane = threadIdx.x & 31;
  const GlobalBytes din{data, data + data_bytes}, dsec{secret, secret + secret_len};
  for (int64_t b = (int64_t)blockIdx.x * kWarps + (threadIdx.x >> 5); b < n_blocks;
       b += (int64_t)gridDim.x * kWarps) {
    const uint64_t s0 = offsets[b], s1 = offsets[b + 1];
    if (s1 < s0 || s1 > data_bytes) {
      if (lane == 0) report(d_status, LT_ERR_CORRUPT_STREAM);
      continue;
    }
    const uint64_t len = s1 - s0;
    uint64_t h;
    if (len > 240) {
      const uint8_t *in = data + s0;
      h = xxh3::hash64_long_warp([&](uint64_t off) { return din.rd64(in + off); },
                                 [&](uint64_t off) { return dsec.rd64(secret + off); }, len, secret_len, lane);
    } else {
      h = lane == 0 ? xxh3::hash64(data + s0, len, secret, secret_len) : 0;
    }
    if (lane == 0) {
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
  int64_t blocks = (n_blocks + kWarps - 1) / kWarps;
  const int64_t cap = (int64_t)num_sms() * 16;
  if (blocks > cap) blocks = cap;
  k_xxh3_blocks<<<(int)blocks, kThreads, 0, (cudaStream_t)stream>>>(
      data, data_bytes, offsets, n_blocks, secret, (uint32_t)secret_len, hashes, expected, d_status,
      reinterpret_cast<unsigned long long *>(d_first_bad));
  return launch_status();
}
