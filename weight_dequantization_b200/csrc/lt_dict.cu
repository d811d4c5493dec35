// lt_dict.cu -- value-dictionary decoding: out[k] = dict[index k]
// ("LoreToken-powered GPU memory layer", compression strategies: value
// dictionary compression of tensors that hold few distinct values; the
// "GPU sidecar brain" explanation, its strategy list: small integer codes
// plus a tiny lookup table).
//
// A pure HBM stream (bits/8 B in, 2 B out per element) with no arithmetic:
// the entries are copied bit for bit. Each CTA first expands the 2^bits
// dictionary into a byte table in shared memory -- for each of the 256 byte
// values, the binary16 entries of the 8/bits indices that byte holds, in
// element order -- so one 4-byte word of indices becomes its output with
// four shared-memory loads and no per-index unpacking. A warp's loads cover
// 128 contiguous bytes of indices and its stores 8 * 8/bits * 32 contiguous
// bytes of output; the grid is at most one resident wave, walking the words
// in tiles of 256 threads x 4 words.
#include "lt_common.cuh"

namespace lt {
namespace {

constexpr int kThreads = 256;
constexpr int kUnroll = 4;

// 32-bit words of byte table: 4/BITS per byte value for BITS <= 4 (one half
// per index, two halves per word); for BITS == 8 the table is the dictionary
// itself (one half per byte value).
template <int BITS>
struct Table {
  static constexpr int kWords = BITS == 8 ? 128 : 256 * (4 / BITS);
};

template <int BITS>
__device__ __forceinline__ void build_table(const uint16_t *__restrict__ dict, uint32_t *tab) {
  constexpr uint32_t M = (1u << BITS) - 1u;
  if constexpr (BITS == 8) {
    uint16_t *t16 = reinterpret_cast<uint16_t *>(tab);
    for (int v = threadIdx.x; v < 256; v += kThreads) t16[v] = __ldg(dict + v);
  } else {
    constexpr int W = 4 / BITS;
    for (int j = threadIdx.x; j < 256 * W; j += kThreads) {
      const uint32_t v = (uint32_t)j / W, m = (uint32_t)j % W;
      const uint32_t lo = __ldg(dict + ((v >> (2 * m * BITS)) & M));
      const uint32_t hi = __ldg(dict + ((v >> ((2 * m + 1) * BITS)) & M));
      tab[j] = lo | (hi << 16);
    }
  }
}

// word i of indices (packed bytes 4i .. 4i+3) -> its 4 * 8/BITS outputs
template <int BITS>
__device__ __forceinline__ void expand_word(const uint32_t *tab, uint32_t w, void *__restrict__ out, int64_t i) {
  const uint32_t b0 = w & 0xFFu, b1 = (w >> 8) & 0xFFu, b2 = (w >> 16) & 0xFFu, b3 = w >> 24;
  if constexpr (BITS == 8) {
    const uint16_t *t16 = reinterpret_cast<const uint16_t *>(tab);
    const uint32_t a = (uint32_t)t16[b0] | ((uint32_t)t16[b1] << 16);
    const uint32_t b = (uint32_t)t16[b2] | ((uint32_t)t16[b3] << 16);
    reinterpret_cast<uint2 *>(out)[i] = make_uint2(a, b);
  } else if constexpr (BITS == 4) {
    st_u128(reinterpret_cast<uint4 *>(out) + i, make_uint4(tab[b0], tab[b1], tab[b2], tab[b3]));
  } else if constexpr (BITS == 2) {
    const uint2 *t2 = reinterpret_cast<const uint2 *>(tab);
    const uint2 e0 = t2[b0], e1 = t2[b1], e2 = t2[b2], e3 = t2[b3];
    uint4 *o = reinterpret_cast<uint4 *>(out) + 2 * i;
    st_u128(o, make_uint4(e0.x, e0.y, e1.x, e1.y));
    st_u128(o + 1, make_uint4(e2.x, e2.y, e3.x, e3.y));
  } else {
    const uint4 *t4 = reinterpret_cast<const uint4 *>(tab);
    const uint4 e0 = t4[b0], e1 = t4[b1], e2 = t4[b2], e3 = t4[b3];
    uint4 *o = reinterpret_cast<uint4 *>(out) + 4 * i;
    st_u128(o, e0);
    st_u128(o + 1, e1);
    st_u128(o + 2, e2);
    st_u128(o + 3, e3);
  }
}

// n_words whole 4-byte words of indices; out is 16-byte aligned (8-byte for
// BITS == 8) and receives n_words * 4 * (8/BITS) elements
template <int BITS>
__global__ void __launch_bounds__(kThreads) k_dict_vec(const uint32_t *__restrict__ packed,
                                                       const uint16_t *__restrict__ dict, int64_t n_words,
                                                       void *__restrict__ out) {
  __shared__ __align__(16) uint32_t tab[Table<BITS>::kWords];
  const int64_t tile = (int64_t)kThreads * kUnroll;
  const int64_t stride = (int64_t)gridDim.x * tile;
  int64_t base = (int64_t)blockIdx.x * tile;
  uint32_t w[kUnroll];
  // the first tile's loads are in flight while the table is built
#pragma unroll
  for (int u = 0; u < kUnroll; ++u) {
    const int64_t i = base + u * kThreads + threadIdx.x;
    w[u] = i < n_words ? ld_stream_u32(packed + i) : 0u;
  }
  build_table<BITS>(dict, tab);
  __syncthreads();
  while (base < n_words) {
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const int64_t i = base + u * kThreads + threadIdx.x;
      if (i < n_words) expand_word<BITS>(tab, w[u], out, i);
    }
    base += stride;
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const int64_t i = base + u * kThreads + threadIdx.x;
      w[u] = i < n_words ? ld_stream_u32(packed + i) : 0u;
    }
  }
}

// one thread per element; any alignment, any element range
__global__ void __launch_bounds__(kThreads) k_dict_scalar(const uint8_t *__restrict__ packed, int bits,
                                                          const uint16_t *__restrict__ dict, int64_t k_begin,
                                                          int64_t k_end, uint16_t *__restrict__ out) {
  const uint32_t mask = (1u << bits) - 1u;
  for (int64_t k = k_begin + (int64_t)blockIdx.x * blockDim.x + threadIdx.x; k < k_end;
       k += (int64_t)gridDim.x * blockDim.x) {
    const uint64_t bit = (uint64_t)k * (uint64_t)bits;
    const uint32_t idx = ((uint32_t)packed[bit >> 3] >> (bit & 7)) & mask;
    out[k] = dict[idx];
  }
}

template <int BITS>
void launch_vec(const uint8_t *packed, const uint16_t *dict, int64_t n_words, void *out, cudaStream_t st) {
  auto k = k_dict_vec<BITS>;
  const int64_t need = (n_words + (int64_t)kThreads * kUnroll - 1) / ((int64_t)kThreads * kUnroll);
  // one CTA per tile (the kernel loops, so any grid is correct): as for the
  // dequant streams, fresh CTAs keep more loads in flight than one resident
  // wave that loops; the table build is 256 shared-memory stores per CTA
  const int64_t cap = 1ll << 30;
  const int64_t g = need < cap ? need : cap;
  k<<<(int)(g < 1 ? 1 : g), kThreads, 0, st>>>(reinterpret_cast<const uint32_t *>(packed), dict, n_words, out);
}

}  // namespace
}  // namespace lt

using namespace lt;

LT_API lt_status lt_value_dict_decode(const uint8_t *packed, int32_t bits, const lt_half *dict, int64_t n,
                                      lt_half *out, lt_stream_t stream) {
  if (n < 0) return LT_ERR_INVALID_ARG;
  if (bits != 1 && bits != 2 && bits != 4 && bits != 8) return LT_ERR_INVALID_ARG;
  if (n > INT64_MAX / 8) return LT_ERR_INVALID_ARG;
  if (n == 0) return LT_OK;
  if (!packed || !dict || !out) return LT_ERR_INVALID_ARG;
  if (!aligned(dict, 2) || !aligned(out, 2)) return LT_ERR_MISALIGNED;
  cudaStream_t st = (cudaStream_t)stream;

  const int64_t per_word = 4 * (8 / bits);  // elements per 4-byte word of indices
  const bool vec_ok = aligned(packed, 4) && aligned(out, bits == 8 ? 8 : 16);
  int64_t k_vec_end = 0;
  if (vec_ok) {
    const int64_t n_words = n / per_word;
    k_vec_end = n_words * per_word;
    if (n_words > 0) {
      switch (bits) {
        case 1: launch_vec<1>(packed, dict, n_words, out, st); break;
        case 2: launch_vec<2>(packed, dict, n_words, out, st); break;
        case 4: launch_vec<4>(packed, dict, n_words, out, st); break;
        default: launch_vec<8>(packed, dict, n_words, out, st); break;
      }
    }
  }
  if (k_vec_end < n) {
    int64_t blocks = (n - k_vec_end + kThreads - 1) / kThreads;
    const int64_t cap = (int64_t)num_sms() * 8;
    if (blocks > cap) blocks = cap;
    k_dict_scalar<<<(int)blocks, kThreads, 0, st>>>(packed, bits, dict, k_vec_end, n, out);
  }
  return launch_status();
}
