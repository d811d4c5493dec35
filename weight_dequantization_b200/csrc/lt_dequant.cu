// lt_dequant.cu -- INT4 group and INT8 per-tensor / per-row dequantization
// to binary16 ("GPU Compression Pipeline - TDD Roadmap", Phases 1.1 and 1.2).
//
// Both are pure HBM streams (INT4: 0.5 B in, 2 B out per element; INT8: 1 B
// in, 2 B out). Vector path: each thread reads one 4-byte (INT4, 8 codes) or
// 8-byte (INT8, 8 codes) word and writes the 8 binary16 results with one
// 16-byte store, so a warp's loads cover 128 / 256 contiguous bytes and its
// stores 512 contiguous bytes. U independent words per thread keep enough
// loads in flight; the grid has one CTA per tile of U words per thread.
// (16-byte loads with four 16-byte stores per thread at a 64-byte stride
// measured 35-65 % slower: a warp's stores then scatter; 16-byte loads with
// the stores regrouped through shared memory measured the same as this.)
#include "lt_common.cuh"

namespace lt {
namespace {

constexpr int kThreads = 256;
constexpr int kUnroll = 4;

// ----------------------------------------------------------------------------
// INT4
// ----------------------------------------------------------------------------
template <bool HAS_Z, bool POW2>
__global__ void __launch_bounds__(kThreads) k_int4_vec(const uint32_t *__restrict__ packed,
                                                       const uint16_t *__restrict__ scales,
                                                       const uint8_t *__restrict__ zeros, int64_t n_words,
                                                       uint32_t words_per_group, uint32_t wpg_shift,
                                                       uint4 *__restrict__ out) {
  const int64_t tile = (int64_t)kThreads * kUnroll;
  const uint32_t zm0 = 0x54006400u;  // (1024, 64): zero point 0
  for (int64_t base = (int64_t)blockIdx.x * tile; base < n_words; base += (int64_t)gridDim.x * tile) {
    uint32_t w[kUnroll];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const int64_t i = base + u * kThreads + threadIdx.x;
      w[u] = i < n_words ? ld_stream_u32(packed + i) : 0u;
    }
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const int64_t i = base + u * kThreads + threadIdx.x;
      if (i < n_words) {
        const int64_t g = POW2 ? (i >> wpg_shift) : (i / (int64_t)words_per_group);
        const uint32_t s2 = bcast_half(__ldg(scales + g));
        const uint32_t zm = HAS_Z ? int4_zero_magic(__ldg(zeros + g)) : zm0;
        st_u128(out + i, int4x8_dequant(w[u], zm, s2));
      }
    }
  }
}

// one thread per code; any alignment, any group size
__global__ void __launch_bounds__(kThreads) k_int4_scalar(const uint8_t *__restrict__ packed,
                                                          const uint16_t *__restrict__ scales,
                                                          const uint8_t *__restrict__ zeros, int64_t k_begin,
                                                          int64_t k_end, int64_t group_size,
                                                          uint16_t *__restrict__ out) {
  for (int64_t k = k_begin + (int64_t)blockIdx.x * blockDim.x + threadIdx.x; k < k_end;
       k += (int64_t)gridDim.x * blockDim.x) {
    const uint8_t b = packed[k >> 1];
    const int32_t q = (k & 1) ? (b >> 4) : (b & 0x0F);
    const int64_t g = k / group_size;
    const int32_t z = zeros ? zeros[g] : 0;
    out[k] = dequant_scalar(q - z, scales[g]);
  }
}

// ----------------------------------------------------------------------------
// INT8
// ----------------------------------------------------------------------------
template <bool PER_ROW, bool HAS_Z>
__global__ void __launch_bounds__(kThreads) k_int8_vec(const uint2 *__restrict__ q, const uint16_t *__restrict__ scales,
                                                       const int8_t *__restrict__ zeros, int64_t n_vec,
                                                       int64_t vec_per_row, uint4 *__restrict__ out) {
  const int64_t tile = (int64_t)kThreads * kUnroll;
  uint32_t s2_t = 0, zm_t = 0;
  if (!PER_ROW) {
    s2_t = bcast_half(__ldg(scales));
    zm_t = int8_zero_magic(HAS_Z ? (int32_t)__ldg(zeros) : 0);
  }
  for (int64_t base = (int64_t)blockIdx.x * tile; base < n_vec; base += (int64_t)gridDim.x * tile) {
    uint2 w[kUnroll];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const int64_t i = base + u * kThreads + threadIdx.x;
      w[u] = i < n_vec ? ld_stream_u64(q + i) : make_uint2(0u, 0u);
    }
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const int64_t i = base + u * kThreads + threadIdx.x;
      if (i < n_vec) {
        uint32_t s2 = s2_t, zm = zm_t;
        if (PER_ROW) {
          const int64_t r = i / vec_per_row;
          s2 = bcast_half(__ldg(scales + r));
          zm = int8_zero_magic(HAS_Z ? (int32_t)__ldg(zeros + r) : 0);
        }
        st_u128(out + i, int8x8_dequant(w[u], zm, s2));
      }
    }
  }
}

__global__ void __launch_bounds__(kThreads) k_int8_scalar(const int8_t *__restrict__ q,
                                                          const uint16_t *__restrict__ scales,
                                                          const int8_t *__restrict__ zeros, int per_row,
                                                          int64_t k_begin, int64_t k_end, int64_t cols,
                                                          uint16_t *__restrict__ out) {
  for (int64_t k = k_begin + (int64_t)blockIdx.x * blockDim.x + threadIdx.x; k < k_end;
       k += (int64_t)gridDim.x * blockDim.x) {
    const int64_t r = per_row ? k / cols : 0;
    const int32_t z = zeros ? zeros[r] : 0;
    out[k] = dequant_scalar((int32_t)q[k] - z, scales[r]);
  }
}

// grid: one CTA per tile of work (the kernels loop, so any grid is
// correct). Measured on B200 with these pure streams: a grid of one CTA per
// tile beats one resident wave that loops (INT8 8192 x 8192: 36.9 vs
// 38.9 us; INT4 4096 x 14336: 28.7 vs 30.8 us), as freshly started CTAs
// issue their loads together instead of after the previous tile's stores.
int grid_for(const void *, int64_t n_blocks_needed) {
  const int64_t cap = 1ll << 30;
  const int64_t g = n_blocks_needed < cap ? n_blocks_needed : cap;
  return (int)(g < 1 ? 1 : g);
}

int scalar_grid(int64_t n) {
  int64_t b = (n + kThreads - 1) / kThreads;
  const int64_t cap = (int64_t)num_sms() * 8;
  return (int)(b < 1 ? 1 : (b > cap ? cap : b));
}

}  // namespace
}  // namespace lt

using namespace lt;

LT_API lt_status lt_dequant_int4(const uint8_t *packed, const lt_half *scales, const uint8_t *zeros, int64_t rows,
                                 int64_t cols, int32_t group_size, lt_half *out, lt_stream_t stream) {
  if (rows < 0 || cols < 0 || group_size < 1) return LT_ERR_INVALID_ARG;
  if (cols % group_size != 0) return LT_ERR_INVALID_ARG;
  if (rows != 0 && cols > INT64_MAX / rows) return LT_ERR_INVALID_ARG;
  const int64_t n = rows * cols;
  if (n == 0) return LT_OK;
  if (!packed || !scales || !out) return LT_ERR_INVALID_ARG;
  if (!aligned(scales, 2) || !aligned(out, 2)) return LT_ERR_MISALIGNED;
  cudaStream_t st = (cudaStream_t)stream;

  const bool vec_ok = (group_size % 8 == 0) && aligned(packed, 4) && aligned(out, 16);
  int64_t k_vec_end = 0;
  if (vec_ok) {
    const int64_t n_words = n / 8;
    k_vec_end = n_words * 8;
    if (n_words > 0) {
      const uint32_t wpg = (uint32_t)(group_size / 8);
      const bool pow2 = (wpg & (wpg - 1)) == 0;
      uint32_t shift = 0;
      while (pow2 && (1u << shift) < wpg) ++shift;
      const int64_t need = (n_words + (int64_t)kThreads * kUnroll - 1) / ((int64_t)kThreads * kUnroll);
      const uint32_t *pw = (const uint32_t *)packed;
      uint4 *po = (uint4 *)out;
      if (zeros) {
        if (pow2) {
          auto k = k_int4_vec<true, true>;
          k<<<grid_for((const void *)k, need), kThreads, 0, st>>>(pw, scales, zeros, n_words, wpg, shift, po);
        } else {
          auto k = k_int4_vec<true, false>;
          k<<<grid_for((const void *)k, need), kThreads, 0, st>>>(pw, scales, zeros, n_words, wpg, shift, po);
        }
      } else {
        if (pow2) {
          auto k = k_int4_vec<false, true>;
          k<<<grid_for((const void *)k, need), kThreads, 0, st>>>(pw, scales, zeros, n_words, wpg, shift, po);
        } else {
          auto k = k_int4_vec<false, false>;
          k<<<grid_for((const void *)k, need), kThreads, 0, st>>>(pw, scales, zeros, n_words, wpg, shift, po);
        }
      }
    }
  }
  if (k_vec_end < n) {
    k_int4_scalar<<<scalar_grid(n - k_vec_end), kThreads, 0, st>>>(packed, scales, zeros, k_vec_end, n, group_size,
                                                                    out);
  }
  return launch_status();
}

LT_API lt_status lt_dequant_int8(const int8_t *q, const lt_half *scales, const int8_t *zeros, int32_t scale_mode,
                                 int64_t rows, int64_t cols, lt_half *out, lt_stream_t stream) {
  if (rows < 0 || cols < 0) return LT_ERR_INVALID_ARG;
  if (scale_mode != LT_SCALE_PER_TENSOR && scale_mode != LT_SCALE_PER_ROW) return LT_ERR_INVALID_ARG;
  if (rows != 0 && cols > INT64_MAX / rows) return LT_ERR_INVALID_ARG;
  const int64_t n = rows * cols;
  if (n == 0) return LT_OK;
  if (!q || !scales || !out) return LT_ERR_INVALID_ARG;
  if (!aligned(scales, 2) || !aligned(out, 2)) return LT_ERR_MISALIGNED;
  cudaStream_t st = (cudaStream_t)stream;
  const bool per_row = scale_mode == LT_SCALE_PER_ROW;

  const bool vec_ok = aligned(q, 8) && aligned(out, 16) && (!per_row || cols % 8 == 0);
  int64_t k_vec_end = 0;
  if (vec_ok) {
    const int64_t n_vec = n / 8;
    k_vec_end = n_vec * 8;
    if (n_vec > 0) {
      const int64_t need = (n_vec + (int64_t)kThreads * kUnroll - 1) / ((int64_t)kThreads * kUnroll);
      const int64_t vpr = per_row ? cols / 8 : 1;
      const uint2 *pq = (const uint2 *)q;
      uint4 *po = (uint4 *)out;
      if (per_row) {
        if (zeros) {
          auto k = k_int8_vec<true, true>;
          k<<<grid_for((const void *)k, need), kThreads, 0, st>>>(pq, scales, zeros, n_vec, vpr, po);
        } else {
          auto k = k_int8_vec<true, false>;
          k<<<grid_for((const void *)k, need), kThreads, 0, st>>>(pq, scales, zeros, n_vec, vpr, po);
        }
      } else {
        if (zeros) {
          auto k = k_int8_vec<false, true>;
          k<<<grid_for((const void *)k, need), kThreads, 0, st>>>(pq, scales, zeros, n_vec, vpr, po);
        } else {
          auto k = k_int8_vec<false, false>;
          k<<<grid_for((const void *)k, need), kThreads, 0, st>>>(pq, scales, zeros, n_vec, vpr, po);
        }
      }
    }
  }
  if (k_vec_end < n) {
    k_int8_scalar<<<scalar_grid(n - k_vec_end), kThreads, 0, st>>>(q, scales, zeros, per_row ? 1 : 0, k_vec_end, n,
                                                                    cols, out);
  }
  return launch_status();
}
