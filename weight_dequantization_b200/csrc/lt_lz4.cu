// lt_lz4.cu -- LZ4 block decompression on chip, fused with INT4 unpack and
// group scaling to binary16 ("GPU Compression Pipeline - TDD Roadmap",
// Phase 2.1 LZ4 + INT4 Fused Kernel; 64 KB independent blocks as in
// Phase 3.1 / Phase 6.1), plus the same decoder writing raw bytes.
//
// One CTA per 64 KB block (a grid-stride loop over the blocks of up to
// LT_LZ4_BATCH_MAX matrices). Warp 0 walks the block's sequences; the
// decompressed bytes (the packed INT4 codes) go to a window in shared memory,
// never to HBM. Literal runs are copied by the 32 lanes; a match of length
// M at offset d is copied in one parallel pass with
// win[p + i] = win[p - d + (i mod d)], which is what the format's byte-by-byte
// overlapping copy produces. Then all warps of the CTA dequantize the window
// and write binary16 to HBM with 16-byte stores.
#include "lt_common.cuh"

namespace lt {
namespace {

constexpr int kThreads = 256;
constexpr int kMaxWindow = 65536;

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
  int32_t pad_;
};

struct Batch {
  Job job[LT_LZ4_BATCH_MAX];
  int32_t n_jobs;
  int32_t max_block_bytes;
  int64_t total_blocks;
};

// Walk one LZ4 block src[0, ilen) into win[0, olen). Executed by all 32 lanes
// of a warp in lockstep (the control flow is warp-uniform). Returns 0 or a
// status code; bounded by ilen on any input.
__device__ int lz4_block_to_window(const uint8_t *__restrict__ src, uint64_t ilen, uint8_t *win, uint32_t olen,
                                   int lane) {
  if (ilen == 0) return olen == 0 ? 0 : LT_ERR_SIZE_MISMATCH;
  uint64_t ip = 0;
  uint32_t op = 0;
  for (;;) {
    if (ip >= ilen) return LT_ERR_CORRUPT_STREAM;
    const uint32_t token = src[ip++];
    uint64_t lit = token >> 4;
    if (lit == 15) {
      uint32_t b;
      do {
        if (ip >= ilen) return LT_ERR_CORRUPT_STREAM;
        b = src[ip++];
        lit += b;
      } while (b == 255 && lit <= olen);
    }
    if (ip + lit > ilen || (uint64_t)op + lit > olen) return LT_ERR_CORRUPT_STREAM;
    for (uint32_t i = lane; i < (uint32_t)lit; i += 32) win[op + i] = src[ip + i];
    ip += lit;
    op += (uint32_t)lit;
    if (ip == ilen) break;  // the last sequence has literals only
    if (ip + 2 > ilen) return LT_ERR_CORRUPT_STREAM;
    const uint32_t off = (uint32_t)src[ip] | ((uint32_t)src[ip + 1] << 8);
    ip += 2;
    if (off == 0 || off > op) return LT_ERR_CORRUPT_STREAM;
    uint64_t mlen = (token & 15u) + 4;
    if ((token & 15u) == 15u) {
      uint32_t b;
      do {
        if (ip >= ilen) return LT_ERR_CORRUPT_STREAM;
        b = src[ip++];
        mlen += b;
      } while (b == 255 && mlen <= olen);
    }
    if ((uint64_t)op + mlen > olen) return LT_ERR_CORRUPT_STREAM;
    __syncwarp();  // literals written by other lanes become visible
    const uint32_t src0 = op - off;
    for (uint32_t i = lane; i < (uint32_t)mlen; i += 32) win[op + i] = win[src0 + (i < off ? i : i % off)];
    __syncwarp();
    op += (uint32_t)mlen;
  }
  return op == olen ? 0 : LT_ERR_SIZE_MISMATCH;
}

template <bool FUSED>
__global__ void __launch_bounds__(kThreads) k_lz4(const __grid_constant__ Batch batch, int32_t *d_status) {
  extern __shared__ uint4 smem_u4[];
  uint8_t *win = reinterpret_cast<uint8_t *>(smem_u4);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  for (int64_t blk = blockIdx.x; blk < batch.total_blocks; blk += gridDim.x) {
    int j = 0;
    while (j + 1 < batch.n_jobs && blk >= batch.job[j + 1].first_block) ++j;
    const Job &jb = batch.job[j];
    const int64_t b = blk - jb.first_block;
    const int64_t d0 = b * (int64_t)jb.block_bytes;
    const uint32_t olen = (uint32_t)((jb.packed_bytes - d0) < jb.block_bytes ? (jb.packed_bytes - d0) : jb.block_bytes);

    if (warp == 0) {
      const uint64_t s0 = jb.offsets[b], s1 = jb.offsets[b + 1];
      int err;
      if (s1 < s0 || s1 > jb.comp_bytes)
        err = LT_ERR_CORRUPT_STREAM;
      else
        err = lz4_block_to_window(jb.comp + s0, s1 - s0, win, olen, lane);
      if (err && lane == 0) report(d_status, err);
    }
    __syncthreads();

    if (FUSED) {
      // window byte i holds codes 2i (low nibble) and 2i+1 (high nibble) of
      // the block; the block's first code is 2 * d0
      uint16_t *out = reinterpret_cast<uint16_t *>(jb.out);
      const int64_t k0 = 2 * d0;
      const int64_t k_end_blk = (k0 + 2 * (int64_t)olen) < jb.n_codes ? (k0 + 2 * (int64_t)olen) : jb.n_codes;
      const int64_t G = jb.group_size;
      const bool vec = (G % 8 == 0) && aligned(out + k0, 16);
      int64_t k_vec_end = k0;
      if (vec) {
        const uint32_t n_words = (uint32_t)((k_end_blk - k0) / 8);
        const uint32_t *win32 = reinterpret_cast<const uint32_t *>(win);
        for (uint32_t i = threadIdx.x; i < n_words; i += kThreads) {
          const int64_t k = k0 + 8 * (int64_t)i;
          const int64_t g = k / G;
          const uint32_t s2 = bcast_half(__ldg(jb.scales + g));
          const uint32_t zm = jb.zeros ? int4_zero_magic(__ldg(jb.zeros + g)) : 0x54006400u;
          st_u128(out + k, int4x8_dequant(win32[i], zm, s2));
        }
        k_vec_end = k0 + 8 * (int64_t)n_words;
      }
      for (int64_t k = k_vec_end + threadIdx.x; k < k_end_blk; k += kThreads) {
        const uint8_t byte = win[(k - k0) >> 1];
        const int32_t q = (k & 1) ? (byte >> 4) : (byte & 0x0F);
        const int64_t g = k / G;
        const int32_t z = jb.zeros ? jb.zeros[g] : 0;
        out[k] = dequant_scalar(q - z, jb.scales[g]);
      }
    } else {
      uint8_t *out = reinterpret_cast<uint8_t *>(jb.out) + d0;
      if (aligned(out, 16) && (olen & 15) == 0) {
        const uint4 *w4 = reinterpret_cast<const uint4 *>(win);
        uint4 *o4 = reinterpret_cast<uint4 *>(out);
        for (uint32_t i = threadIdx.x; i < olen / 16; i += kThreads) st_u128(o4 + i, w4[i]);
      } else {
        for (uint32_t i = threadIdx.x; i < olen; i += kThreads) out[i] = win[i];
      }
    }
    __syncthreads();
  }
}

lt_status launch(const Batch &batch, bool fused, int32_t *d_status, cudaStream_t st) {
  if (batch.total_blocks == 0) return LT_OK;
  const size_t smem = (size_t)((batch.max_block_bytes + 15) / 16 * 16);
  const void *k = fused ? (const void *)k_lz4<true> : (const void *)k_lz4<false>;
  static int attr_set[2][64] = {{0}};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev >= 0 && dev < 64 && !attr_set[fused][dev]) {
    cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, kMaxWindow);
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
  j.pad_ = 0;
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
  j.block_bytes = block_bytes;
  batch.total_blocks = ((int64_t)out_bytes + block_bytes - 1) / block_bytes;
  batch.max_block_bytes = block_bytes;
  return launch(batch, false, d_status, (cudaStream_t)stream);
}
