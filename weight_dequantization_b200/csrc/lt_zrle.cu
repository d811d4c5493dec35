// lt_zrle.cu -- zero-run decoding of mostly-zero binary16 activations
// ("LoreToken-powered GPU memory layer", compression strategies: zero-run
// encoding for ReLU outputs).
//
// One warp per chunk. The chunk's output is built in a shared-memory tile
// that is zeroed with 16-byte stores; the warp walks the chunk's records
// (the walk is serial: each record's position depends on the previous
// literal count) and its lanes scatter each record's literals into the
// tile; the tile then leaves with 16-byte coalesced stores. Chunks larger
// than the tile limit are decoded straight into global memory.
#include "lt_common.cuh"

namespace lt {
namespace {

constexpr int kWarps = 4;
constexpr int kTileMaxElems = 8192;  // 16 KB per warp

__device__ __forceinline__ uint32_t rd_u16le(const uint8_t *__restrict__ p) {
  return (uint32_t)p[0] | ((uint32_t)p[1] << 8);
}

template <bool TILE>
__global__ void __launch_bounds__(kWarps * 32) k_zrle(const uint8_t *__restrict__ enc, uint64_t enc_bytes,
                                                      const uint64_t *__restrict__ offsets, int64_t n,
                                                      int32_t chunk, int64_t n_chunks, int32_t tile_elems,
                                                      uint16_t *__restrict__ out, int32_t *d_status) {
  extern __shared__ uint4 smem_u4[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  uint16_t *tile = reinterpret_cast<uint16_t *>(smem_u4) + (size_t)warp * tile_elems;

  for (int64_t c = (int64_t)blockIdx.x * kWarps + warp; c < n_chunks; c += (int64_t)gridDim.x * kWarps) {
    const int64_t e0 = c * (int64_t)chunk;
    const int32_t len = (int32_t)((n - e0) < chunk ? (n - e0) : chunk);
    uint16_t *dst = TILE ? tile : out + e0;

    // zero fill
    if (TILE) {
      uint4 *t4 = reinterpret_cast<uint4 *>(tile);
      for (int i = lane; i < tile_elems / 8; i += 32) t4[i] = make_uint4(0u, 0u, 0u, 0u);
    } else {
      for (int i = lane; i < len; i += 32) dst[i] = 0;
    }
    __syncwarp();

    const uint64_t b0 = offsets[c], b1 = offsets[c + 1];
    if (b1 < b0 || b1 > enc_bytes) {
      if (lane == 0) report(d_status, LT_ERR_CORRUPT_STREAM);
    } else {
      uint64_t p = b0;
      int32_t done = 0;
      while (done < len) {
        if (p + 4 > b1) {
          if (lane == 0) report(d_status, LT_ERR_SIZE_MISMATCH);
          break;
        }
        const uint32_t zrun = rd_u16le(enc + p);
        const uint32_t nlit = rd_u16le(enc + p + 2);
        p += 4;
        if ((int64_t)done + zrun + nlit > len || p + 2ull * nlit > b1) {
          if (lane == 0) report(d_status, LT_ERR_CORRUPT_STREAM);
          break;
        }
        done += (int32_t)zrun;
        for (uint32_t i = lane; i < nlit; i += 32) dst[done + i] = (uint16_t)rd_u16le(enc + p + 2ull * i);
        done += (int32_t)nlit;
        p += 2ull * nlit;
      }
    }
    __syncwarp();

    if (TILE) {
      uint16_t *o = out + e0;
      if (aligned(o, 16) && (len & 7) == 0) {
        const uint4 *t4 = reinterpret_cast<const uint4 *>(tile);
        uint4 *o4 = reinterpret_cast<uint4 *>(o);
        for (int i = lane; i < len / 8; i += 32) st_u128(o4 + i, t4[i]);
      } else {
        for (int i = lane; i < len; i += 32) o[i] = tile[i];
      }
      __syncwarp();
    }
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
  if (chunk_elems <= kTileMaxElems) {
    const int32_t tile_elems = (chunk_elems + 7) / 8 * 8;
    const size_t smem = (size_t)kWarps * tile_elems * 2;
    auto k = k_zrle<true>;
    static int attr_set[64] = {0};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev >= 0 && dev < 64 && !attr_set[dev]) {
      cudaFuncSetAttribute((const void *)k, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           kWarps * kTileMaxElems * 2);
      attr_set[dev] = 1;
    }
    const int64_t cap = (int64_t)num_sms() * blocks_per_sm((const void *)k, kWarps * 32, smem);
    const int grid = (int)(need < cap ? need : cap);
    k<<<grid, kWarps * 32, smem, st>>>(enc, enc_bytes, chunk_offsets, n_elements, chunk_elems, n_chunks, tile_elems,
                                       out, d_status);
  } else {
    auto k = k_zrle<false>;
    const int64_t cap = (int64_t)num_sms() * blocks_per_sm((const void *)k, kWarps * 32, 0);
    const int grid = (int)(need < cap ? need : cap);
    k<<<grid, kWarps * 32, 0, st>>>(enc, enc_bytes, chunk_offsets, n_elements, chunk_elems, n_chunks, 0, out,
                                    d_status);
  }
  return launch_status();
}
