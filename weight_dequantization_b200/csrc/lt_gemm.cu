// lt_gemm.cu -- fused INT4 decode -> matrix multiply on the 5th-generation
// tensor cores ("LoreToken-powered GPU memory layer": decode + GEMM, the
// decoded weights feeding a matrix multiply; "GPU Compression Pipeline - TDD
// Roadmap", Phase 4.1: a decoded weight tensor used in input.matmul(weights)).
//
//   out[M, N] = x[M, K] . W[K, N],  W = the INT4 group dequantization of a
//   [K, N] code matrix exactly as lt_dequant_int4 computes it (groups of G
//   along each row of W), x and out binary16, products summed in fp32.
//
// One CTA computes a 128 x 256 tile of out over a range of K (the whole of
// K, or a split of it whose fp32 partial sums a second kernel adds in a
// fixed order). Warp roles:
//   warp 0      packed-W producer: for each 64-wide K step one tiled bulk
//               copy (TMA) of the packed INT4 tile (64 rows x 128 bytes,
//               128-byte swizzle) into a 6-deep ring, completion counted on
//               an mbarrier; a slot is refilled as soon as the decoders are
//               done with it, so this stream runs well ahead of the MMAs;
//   warp 2      x producer: the x tile (128 x 64 fp16, 128-byte swizzle) of
//               each step into a 3-deep ring, refilled when the MMAs that
//               read a slot have completed;
//   warps 3..18 decoders: turn the packed tile into the fp16 B operand in
//               shared memory (N-major, 128-byte swizzle), with the exact
//               half2 arithmetic of lt_dequant_int4 (bit-identical to it), in
//               a 4-deep ring; scales and zero points are loaded three steps
//               before their use;
//   warp 1      MMA issuer: one thread issues tcgen05.mma kind::f16 (fp32
//               accumulator in tensor memory, 128 x 256 = 256 columns), four
//               K = 16 instructions per step, and tcgen05.commit releases the
//               ring slots;
//   warps 3..18 epilogue: tcgen05.ld of the accumulator (warp w reads lanes
//               32 (w % 4) ... and a quarter of the columns), conversion to
//               binary16 (or the fp32 partial of a split), 16-byte stores.
// Every mbarrier wait is bounded (about a second of clock); a wait that runs
// out sets LT_ERR_TIMEOUT in the status word and the CTA winds down: the
// producer waits (bounded) for its copies in flight, the tensor memory is
// freed, nothing more is written.
#include "lt_common.cuh"

#include <cuda.h>
#include <mutex>
#include <type_traits>

namespace lt {
namespace {

constexpr int kBM = 128, kBN = 256, kBK = 64;
constexpr int kStagesW = 6;  // packed-W slots (TMA; freed by the decoders)
constexpr int kStagesX = 3;  // x slots (TMA; freed by the MMAs)
constexpr int kStagesB = 4;  // decoded-B slots: the decoders run up to three steps ahead of the MMAs
constexpr int kDecWarps = 16;
constexpr int kDec0 = 3;     // first decoder warp (0: packed-W producer, 1: MMA, 2: x producer)
constexpr int kUnits = (kBK * kBN / 32) / (kDecWarps * 32);  // 16-byte packed chunks per decoder thread per step
static_assert(kUnits * kDecWarps * 32 == kBK * kBN / 32, "decoder units must cover a packed tile");
constexpr int kGemmThreads = (kDec0 + kDecWarps) * 32;
constexpr uint32_t kABytes = kBM * kBK * 2;   // 16384
constexpr uint32_t kWBytes = kBK * kBN / 2;   // 8192
constexpr uint32_t kBBytes = kBN * kBK * 2;   // 32768
constexpr uint32_t kSmemA = 0;
constexpr uint32_t kSmemW = kSmemA + kStagesX * kABytes;
constexpr uint32_t kSmemB = kSmemW + kStagesW * kWBytes;
constexpr uint32_t kSmemTotal = kSmemB + kStagesB * kBBytes;  // 224 KB
constexpr uint32_t kSmemDyn = kSmemTotal + 1024;              // + alignment slack
constexpr uint32_t kTmemCols = 256;
// B operand (N-major, 128-byte swizzle): 1 KB atoms of 64 n x 8 k; atoms
// along N are kBAtomN bytes apart, atoms along K 1 KB apart.
constexpr uint32_t kBAtomN = (kBK / 8) * 1024;  // 8192
constexpr uint32_t kBAtomK = 1024;
constexpr long long kWaitCycles = 2000000000LL;  // ~1 s at the boost clock

__device__ __forceinline__ uint32_t smem_u32(const void *p) { return (uint32_t)__cvta_generic_to_shared(p); }

// shared-memory matrix descriptor (tcgen05): start, leading and stride byte
// offsets (16-byte units), descriptor version 1, 128-byte swizzle
__device__ __forceinline__ uint64_t smem_desc(uint32_t addr, uint32_t lbo, uint32_t sbo) {
  return (uint64_t)((addr & 0x3FFFFu) >> 4) | ((uint64_t)(lbo >> 4) << 16) | ((uint64_t)(sbo >> 4) << 32) |
         (1ull << 46) | (2ull << 61);
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}
// bounded wait for the phase with the given parity to complete
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  if (ok) return true;
  const long long t0 = clock64();
  for (;;) {
    asm volatile(
        "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    if (ok) return true;
    if (clock64() - t0 > kWaitCycles) return false;
  }
}

__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap *map, int32_t c0, int32_t c1,
                                            uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::"r"(
          dst),
      "l"(map), "r"(c0), "r"(c1), "r"(bar)
      : "memory");
}

__device__ __forceinline__ void mma_f16(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                        uint32_t accumulate) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}" ::"r"(
          tmem_d),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate));
}
__device__ __forceinline__ void mma_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar) : "memory");
}

// 32 consecutive fp32 columns of this warp's 32 accumulator lanes
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,%17,%18,"
      "%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]),
        "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]),
        "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
        "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

struct GemmArgs {
  const uint16_t *scales;  // [K, N / G]
  const uint8_t *zeros;    // [K, N / G] or nullptr
  uint16_t *out;           // [M, N] binary16 (one split)
  float *partial;          // [splits, M, N] fp32 (several splits)
  int32_t *d_status;
  int64_t M, N, K;
  int32_t group_size;
  int32_t k_iters;  // K / 64
  int32_t splits;
};

__global__ void __launch_bounds__(kGemmThreads, 1) k_int4_gemm(const __grid_constant__ CUtensorMap map_x,
                                                                 const __grid_constant__ CUtensorMap map_w,
                                                                 const __grid_constant__ GemmArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  __shared__ __align__(8) uint64_t bar_wfull[kStagesW], bar_wempty[kStagesW], bar_xfull[kStagesX],
      bar_xempty[kStagesX], bar_bfull[kStagesB], bar_bempty[kStagesB], bar_acc;
  __shared__ uint32_t s_tmem;
  __shared__ int s_abort;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int n_tile = blockIdx.x, m_tile = blockIdx.y, split = blockIdx.z;
  const int64_t n0 = (int64_t)n_tile * kBN, m0 = (int64_t)m_tile * kBM;
  const int it_begin = (int)((int64_t)a.k_iters * split / a.splits);
  const int it_end = (int)((int64_t)a.k_iters * (split + 1) / a.splits);
  const int n_it = it_end - it_begin;

  if (tid == 0) {
    for (int s = 0; s < kStagesW; ++s) {
      mbar_init(smem_u32(&bar_wfull[s]), 1);
      mbar_init(smem_u32(&bar_wempty[s]), kDecWarps);
    }
    for (int s = 0; s < kStagesX; ++s) {
      mbar_init(smem_u32(&bar_xfull[s]), 1);
      mbar_init(smem_u32(&bar_xempty[s]), 1);
    }
    for (int b = 0; b < kStagesB; ++b) {
      mbar_init(smem_u32(&bar_bfull[b]), kDecWarps);
      mbar_init(smem_u32(&bar_bempty[b]), 1);
    }
    mbar_init(smem_u32(&bar_acc), 1);
    s_abort = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&s_tmem)),
                 "r"(kTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
  __syncthreads();
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
  const uint32_t tmem = s_tmem;
  const uint32_t sbase = smem_u32(sm);

  auto fail = [&]() {
    s_abort = 1;
    report(a.d_status, LT_ERR_TIMEOUT);
  };
  // one TMA stream: step it's tile into slot it % STAGES once that slot is
  // free again (its empty barrier completed STAGES steps earlier); on an abort,
  // wait (bounded) for the copies in flight before the CTA exits
  auto produce = [&](auto stages_c, uint64_t *full, uint64_t *empty, uint32_t slot0, uint32_t bytes, auto issue) {
    constexpr int STAGES = decltype(stages_c)::value;
    int issued = 0;
    for (int it = 0; it < n_it; ++it) {
      const int s = it % STAGES;
      if (it >= STAGES && !mbar_wait(smem_u32(&empty[s]), ((it / STAGES) - 1) & 1)) {
        fail();
        break;
      }
      if (*(volatile int *)&s_abort) break;
      mbar_expect_tx(smem_u32(&full[s]), bytes);
      issue(slot0 + s * bytes, (it_begin + it) * kBK, smem_u32(&full[s]));
      issued = it + 1;
    }
    if (*(volatile int *)&s_abort)
      for (int it = issued > STAGES ? issued - STAGES : 0; it < issued; ++it)
        mbar_wait(smem_u32(&full[it % STAGES]), (it / STAGES) & 1);
  };

  if (warp == 0) {
    // ---------------- packed-W producer: runs up to 8 steps ahead ----------------
    if (lane == 0)
      produce(std::integral_constant<int, kStagesW>{}, bar_wfull, bar_wempty, sbase + kSmemW, kWBytes,
              [&](uint32_t dst, int32_t kk, uint32_t bar) { tma_load_2d(dst, &map_w, (int32_t)(n0 / 2), kk, bar); });
  } else if (warp == 2) {
    // ---------------- x producer ----------------
    if (lane == 0)
      produce(std::integral_constant<int, kStagesX>{}, bar_xfull, bar_xempty, sbase + kSmemA, kABytes,
              [&](uint32_t dst, int32_t kk, uint32_t bar) { tma_load_2d(dst, &map_x, kk, (int32_t)m0, bar); });
  } else if (warp == 1) {
    // ---------------- MMA issuer ----------------
    if (lane == 0) {
      // kind::f16, fp32 accumulator, A and B fp16, A K-major, B N-major, N = 256, M = 128
      const uint32_t idesc = (1u << 4) | (1u << 16) | ((uint32_t)(kBN >> 3) << 17) | ((uint32_t)(kBM >> 4) << 24);
      for (int it = 0; it < n_it; ++it) {
        const int sx = it % kStagesX, b = it % kStagesB;
        if (!mbar_wait(smem_u32(&bar_xfull[sx]), (it / kStagesX) & 1) ||
            !mbar_wait(smem_u32(&bar_bfull[b]), (it / kStagesB) & 1)) {
          fail();
          break;
        }
        if (*(volatile int *)&s_abort) break;
        asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
        const uint32_t a0 = sbase + kSmemA + sx * kABytes, b0 = sbase + kSmemB + b * kBBytes;
#pragma unroll
        for (int ks = 0; ks < kBK / 16; ++ks) {
          // A: K-major 128-byte swizzle, 8-row atoms 1 KB apart, K = 16 slice at +32 bytes;
          // B: N-major 128-byte swizzle, K = 16 slice = two 1 KB atoms along K
          const uint64_t ad = smem_desc(a0 + 32u * ks, 16, 1024);
          const uint64_t bd = smem_desc(b0 + 2u * kBAtomK * ks, kBAtomN, kBAtomK);
          mma_f16(tmem, ad, bd, idesc, (it | ks) != 0);
        }
        mma_commit(smem_u32(&bar_xempty[sx]));
        mma_commit(smem_u32(&bar_bempty[b]));
      }
      mma_commit(smem_u32(&bar_acc));  // the accumulator is final (or abandoned) once this arrives
    }
  } else {
    // ---------------- decoders (then epilogue) ----------------
    const int dt = tid - 32 * kDec0;  // 0 .. 32 kDecWarps - 1
    const int klo = dt & 7, h = (dt >> 3) & 7, khi0 = dt >> 6;  // unit i: row klo + 8 (khi0 + (kDecWarps / 2) i)
    const int64_t NG = a.N / a.group_size;
    const int64_t gcol = (n0 + 32 * h) / a.group_size;  // this thread's group column
    // scales / zero points of this thread's 4 rows of step `it`
    auto load_sz = [&](int it, uint32_t (&sc)[kUnits], uint32_t (&zr)[kUnits]) {
#pragma unroll
      for (int i = 0; i < kUnits; ++i) {
        const int64_t k = (int64_t)(it_begin + it) * kBK + klo + 8 * (khi0 + (kDecWarps / 2) * i);
        sc[i] = __ldg(a.scales + k * NG + gcol);
        zr[i] = a.zeros ? __ldg(a.zeros + k * NG + gcol) : 0u;
      }
    };
    // Scales and zero points arrive through three register sets, each loaded
    // three steps before its use and reloaded right after it (no register
    // moves: a move would wait for the load it copies).
    uint32_t scA[kUnits], zrA[kUnits], scB[kUnits], zrB[kUnits], scC[kUnits], zrC[kUnits];
    if (n_it > 0) load_sz(0, scA, zrA);
    if (n_it > 1) load_sz(1, scB, zrB);
    if (n_it > 2) load_sz(2, scC, zrC);
    bool ok = true;
    // one K step: wait for its packed tile and a free B slot, decode with
    // (sc, zr), refill (sc, zr) for step it + 3, hand the slot to the MMA
    auto step = [&](int it, uint32_t(&sc)[kUnits], uint32_t(&zr)[kUnits]) -> bool {
      const int s = it % kStagesW, b = it % kStagesB;
      if (!mbar_wait(smem_u32(&bar_wfull[s]), (it / kStagesW) & 1) ||
          (it >= kStagesB && !mbar_wait(smem_u32(&bar_bempty[b]), ((it / kStagesB) - 1) & 1))) {
        fail();
        return false;
      }
      if (*(volatile int *)&s_abort) return false;
      const uint8_t *wsrc = sm + kSmemW + s * kWBytes;
      uint8_t *bdst = sm + kSmemB + b * kBBytes;
#pragma unroll
      for (int i = 0; i < kUnits; ++i) {
        const int kk = klo + 8 * (khi0 + (kDecWarps / 2) * i);  // row of the step, 0..63
        // packed row kk: 128 bytes (256 codes), 16-byte chunk h at chunk h ^ (kk & 7)
        const uint4 v = *reinterpret_cast<const uint4 *>(wsrc + kk * 128 + ((h ^ klo) << 4));
        const uint32_t s2 = bcast_half((uint16_t)sc[i]);
        const uint32_t zm = a.zeros ? int4_zero_magic(zr[i]) : 0x54006400u;
        const uint4 o[4] = {int4x8_dequant(v.x, zm, s2), int4x8_dequant(v.y, zm, s2), int4x8_dequant(v.z, zm, s2),
                            int4x8_dequant(v.w, zm, s2)};
        // codes n = 32 h + 8 j .. + 7 of row kk: atom (n / 64, kk / 8), row kk % 8, chunk (n % 64) / 8
        uint8_t *atom = bdst + (h >> 1) * kBAtomN + (kk >> 3) * kBAtomK + klo * 128;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int c = 4 * (h & 1) + j;
          *reinterpret_cast<uint4 *>(atom + ((c ^ klo) << 4)) = o[j];
        }
      }
      if (it + 3 < n_it) load_sz(it + 3, sc, zr);
      // generic-proxy writes of B become visible to the tensor core's async proxy
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(smem_u32(&bar_wempty[s]));
        mbar_arrive(smem_u32(&bar_bfull[b]));
      }
      return true;
    };
    for (int it = 0; it < n_it && ok; it += 3) {
      ok = step(it, scA, zrA);
      if (ok && it + 1 < n_it) ok = step(it + 1, scB, zrB);
      if (ok && it + 2 < n_it) ok = step(it + 2, scC, zrC);
    }
    // ---------------- epilogue ----------------
    const bool acc_ok = mbar_wait(smem_u32(&bar_acc), 0);
    if (!acc_ok) fail();
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
    if (acc_ok && !*(volatile int *)&s_abort && n_it > 0) {
      const int quarter = warp & 3;  // tensor-memory lanes 32 quarter .. + 31
      const int64_t m = m0 + 32 * quarter + lane;
      // each quarter's 256 columns split among its kDecWarps / 4 decoder warps
      constexpr int kCols = kBN / (kDecWarps / 4);
      const int cbeg = ((warp - kDec0) / 4) * kCols;
      for (int c0 = cbeg; c0 < cbeg + kCols; c0 += 32) {
        uint32_t r[32];
        tmem_ld32(tmem + ((uint32_t)(32 * quarter) << 16) + (uint32_t)c0, r);
        if (m < a.M) {
          if (a.splits == 1) {
            uint4 *o = reinterpret_cast<uint4 *>(a.out + m * a.N + n0 + c0);
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              uint32_t w[4];
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                const __half2 hv = __floats2half2_rn(__uint_as_float(r[8 * q + 2 * e]),
                                                     __uint_as_float(r[8 * q + 2 * e + 1]));
                w[e] = *reinterpret_cast<const uint32_t *>(&hv);
              }
              st_u128(o + q, make_uint4(w[0], w[1], w[2], w[3]));
            }
          } else {
            uint4 *o = reinterpret_cast<uint4 *>(a.partial + ((int64_t)split * a.M + m) * a.N + n0 + c0);
#pragma unroll
            for (int q = 0; q < 8; ++q) st_u128(o + q, make_uint4(r[4 * q], r[4 * q + 1], r[4 * q + 2], r[4 * q + 3]));
          }
        }
      }
    }
  }
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
  __syncthreads();
  if (warp == 1) {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols) : "memory");
  }
}

// ---------------------------------------------------------------------------
// Small batches (M <= 8): the same product on the CUDA cores. With a few rows
// of x, the 128-row MMA tile is mostly padding while its operands still flow
// through shared memory; here each code is decoded in registers and used
// straight away, so the codes stream from HBM once and nothing is staged
// but x. One CTA: 256 columns [n0, n0 + 256) over a range of K rows (a split
// of K); lane l of every warp takes columns n0 + 8 l .. + 7 (one 4-byte word
// of codes per row, a warp's loads 128 contiguous bytes), warp w rows w,
// w + 8, ... of each chunk of 512 rows. W is decoded with the exact half2
// arithmetic (lt_dequant_int4's values) and widened to fp32; products with x
// are exact in fp32 and summed in fp32 per thread, then the 8 warps' sums in
// order through shared memory.
// ---------------------------------------------------------------------------
constexpr int kVThreads = 256;
constexpr int kVCols = 256;
constexpr int kVChunk = 512;  // x rows staged per chunk
constexpr int kVUnroll = 8;   // code words in flight per thread

template <int MT>
__global__ void __launch_bounds__(kVThreads) k_int4_gemv(const uint16_t *__restrict__ x, int64_t M, int64_t K,
                                                          const uint32_t *__restrict__ packed,
                                                          const uint16_t *__restrict__ scales,
                                                          const uint8_t *__restrict__ zeros, int64_t N, int32_t G,
                                                          uint16_t *__restrict__ out, float *__restrict__ partial,
                                                          int splits) {
  __shared__ float xs[MT][kVChunk];
  __shared__ float red[MT][kVCols];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int64_t n0 = (int64_t)blockIdx.x * kVCols;
  const int split = blockIdx.y;
  const int64_t k_begin = K * split / splits, k_end = K * (split + 1) / splits;
  const int64_t NG = N / G, wpr = N / 8;  // groups and code words per row
  const int64_t col = n0 + 8 * lane;
  const int64_t gcol = col / G;
  float acc[MT][8];
#pragma unroll
  for (int m = 0; m < MT; ++m)
#pragma unroll
    for (int j = 0; j < 8; ++j) acc[m][j] = 0.f;
  for (int64_t c0 = k_begin; c0 < k_end; c0 += kVChunk) {
    const int rows = (int)((k_end - c0) < kVChunk ? (k_end - c0) : kVChunk);
    __syncthreads();  // the previous chunk's x is no longer read
    for (int i = tid; i < MT * kVChunk; i += kVThreads) {
      const int m = i / kVChunk, r = i % kVChunk;
      xs[m][r] = (m < M && r < rows) ? __half2float(__ushort_as_half(x[(int64_t)m * K + c0 + r])) : 0.f;
    }
    __syncthreads();
    for (int r0 = warp; r0 < rows; r0 += 8 * kVUnroll) {
      uint32_t w[kVUnroll], sc[kVUnroll], zr[kVUnroll];
#pragma unroll
      for (int u = 0; u < kVUnroll; ++u) {
        const int r = r0 + 8 * u;
        const int64_t k = c0 + (r < rows ? r : 0);
        w[u] = r < rows ? ld_stream_u32(packed + k * wpr + col / 8) : 0u;
        sc[u] = r < rows ? __ldg(scales + k * NG + gcol) : 0u;
        zr[u] = (r < rows && zeros) ? __ldg(zeros + k * NG + gcol) : 0u;
      }
#pragma unroll
      for (int u = 0; u < kVUnroll; ++u) {
        const int r = r0 + 8 * u;
        if (r < rows) {
          const uint4 h = int4x8_dequant(w[u], zeros ? int4_zero_magic(zr[u]) : 0x54006400u, bcast_half((uint16_t)sc[u]));
          const uint32_t hw[4] = {h.x, h.y, h.z, h.w};
          float wv[8];
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const float2 f = __half22float2(*reinterpret_cast<const __half2 *>(&hw[q]));
            wv[2 * q] = f.x;
            wv[2 * q + 1] = f.y;
          }
#pragma unroll
          for (int m = 0; m < MT; ++m) {
            const float xm = xs[m][r];
#pragma unroll
            for (int j = 0; j < 8; ++j) acc[m][j] = fmaf(xm, wv[j], acc[m][j]);
          }
        }
      }
    }
  }
  // the 8 warps' sums, added in warp order
  for (int wv = 0; wv < 8; ++wv) {
    __syncthreads();
    if (warp == wv) {
#pragma unroll
      for (int m = 0; m < MT; ++m)
#pragma unroll
        for (int j = 0; j < 8; ++j) red[m][8 * lane + j] = (wv == 0 ? 0.f : red[m][8 * lane + j]) + acc[m][j];
    }
  }
  __syncthreads();
  for (int i = tid; i < MT * kVCols; i += kVThreads) {
    const int m = i / kVCols, c = i % kVCols;
    if (m >= M) continue;
    if (splits == 1)
      out[m * N + n0 + c] = __half_as_ushort(__float2half_rn(red[m][c]));
    else
      partial[((int64_t)split * M + m) * N + n0 + c] = red[m][c];
  }
}

// K splits of the small-batch kernel: about two CTAs per SM, each split at
// least 256 rows
int gemv_splits(int64_t N, int64_t K) {
  const int64_t tiles = N / kVCols;
  int64_t s = (2 * (int64_t)num_sms() + tiles - 1) / tiles;
  if (s > K / 256) s = K / 256;
  if (s > 64) s = 64;
  return (int)(s < 1 ? 1 : s);
}

// out[m, n] = fp16_rn(sum over splits s = 0, 1, ... of partial[s, m, n]), in that order
__global__ void __launch_bounds__(256) k_gemm_reduce(const float4 *__restrict__ partial, int64_t mn4, int splits,
                                                     uint2 *__restrict__ out) {
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < mn4; i += (int64_t)gridDim.x * blockDim.x) {
    float4 acc = partial[i];
    for (int s = 1; s < splits; ++s) {
      const float4 p = partial[(int64_t)s * mn4 + i];
      acc.x += p.x;
      acc.y += p.y;
      acc.z += p.z;
      acc.w += p.w;
    }
    const __half2 lo = __floats2half2_rn(acc.x, acc.y), hi = __floats2half2_rn(acc.z, acc.w);
    out[i] = make_uint2(*reinterpret_cast<const uint32_t *>(&lo), *reinterpret_cast<const uint32_t *>(&hi));
  }
}

typedef CUresult (*encode_tiled_t)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                   const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

encode_tiled_t encoder() {
  static encode_tiled_t fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] { fn = (encode_tiled_t)driver_fn("cuTensorMapEncodeTiled"); });
  return fn;
}

// split count for a grid of `tiles` output tiles and k_iters K steps: as
// many CTAs as fit in one wave over the SMs (one CTA per SM), each split at
// least 4 steps
int choose_splits(int64_t tiles, int64_t k_iters) {
  const int64_t sms = num_sms();
  if (tiles >= sms || k_iters < 8) return 1;
  int64_t s = sms / tiles;
  const int64_t max_s = k_iters / 4;
  if (s > max_s) s = max_s;
  if (s > 32) s = 32;
  return (int)(s < 1 ? 1 : s);
}

bool gemm_shape_ok(int64_t M, int64_t N, int64_t K, int32_t G) {
  return M >= 1 && M <= (1ll << 31) && N >= kBN && N % kBN == 0 && N <= (1ll << 30) && K >= kBK && K % kBK == 0 &&
         K <= (1ll << 30) && G >= 32 && G % 32 == 0 && N % G == 0;
}

}  // namespace
}  // namespace lt

using namespace lt;

LT_API uint64_t lt_int4_gemm_workspace_bytes(int64_t M, int64_t N, int64_t K) {
  if (M < 1 || N < kBN || K < kBK || N % kBN != 0 || K % kBK != 0) return 0;
  int s;
  if (M <= 8) {
    s = gemv_splits(N, K);
  } else {
    const int64_t tiles = ((M + kBM - 1) / kBM) * (N / kBN);
    s = choose_splits(tiles, K / kBK);
  }
  return s > 1 ? (uint64_t)s * (uint64_t)M * (uint64_t)N * 4ull : 0;
}

LT_API lt_status lt_int4_gemm(const lt_half *x, int64_t M, int64_t K, const uint8_t *packed, const lt_half *scales,
                              const uint8_t *zeros, int64_t N, int32_t group_size, lt_half *out, void *workspace,
                              uint64_t workspace_bytes, int32_t *d_status, lt_stream_t stream) {
  if (M < 0 || N < 0 || K < 0) return LT_ERR_INVALID_ARG;
  if (M == 0 || N == 0) return LT_OK;
  if (!gemm_shape_ok(M, N, K, group_size)) return LT_ERR_UNSUPPORTED;
  if (!x || !packed || !scales || !out) return LT_ERR_INVALID_ARG;
  if (!aligned(x, 16) || !aligned(packed, 16) || !aligned(out, 16) || !aligned(scales, 2) ||
      !aligned(workspace, 16) || !aligned(d_status, 4))
    return LT_ERR_MISALIGNED;
  cudaStream_t st = (cudaStream_t)stream;
  auto reduce_splits = [&](int splits) {
    const int64_t mn4 = M * N / 4;
    int64_t g = (mn4 + 255) / 256;
    const int64_t cap = (int64_t)num_sms() * 8;
    if (g > cap) g = cap;
    k_gemm_reduce<<<(int)g, 256, 0, st>>>(reinterpret_cast<const float4 *>(workspace), mn4, splits,
                                          reinterpret_cast<uint2 *>(out));
  };
  if (M <= 8) {  // small batch: the CUDA-core kernel
    int splits = gemv_splits(N, K);
    if (splits > 1 && (!workspace || workspace_bytes < (uint64_t)splits * (uint64_t)M * (uint64_t)N * 4ull)) splits = 1;
    const dim3 grid((unsigned)(N / kVCols), (unsigned)splits);
    const uint32_t *pw = reinterpret_cast<const uint32_t *>(packed);
    float *part = reinterpret_cast<float *>(workspace);
    if (M == 1)
      k_int4_gemv<1><<<grid, kVThreads, 0, st>>>(x, M, K, pw, scales, zeros, N, group_size, out, part, splits);
    else if (M == 2)
      k_int4_gemv<2><<<grid, kVThreads, 0, st>>>(x, M, K, pw, scales, zeros, N, group_size, out, part, splits);
    else if (M <= 4)
      k_int4_gemv<4><<<grid, kVThreads, 0, st>>>(x, M, K, pw, scales, zeros, N, group_size, out, part, splits);
    else
      k_int4_gemv<8><<<grid, kVThreads, 0, st>>>(x, M, K, pw, scales, zeros, N, group_size, out, part, splits);
    if (splits > 1) reduce_splits(splits);
    return launch_status();
  }
  encode_tiled_t enc = encoder();
  if (!enc) return LT_ERR_CUDA;
  CUtensorMap map_x, map_w;
  {
    const cuuint64_t dims[2] = {(cuuint64_t)K, (cuuint64_t)M};
    const cuuint64_t strides[1] = {(cuuint64_t)K * 2};
    const cuuint32_t box[2] = {(cuuint32_t)kBK, (cuuint32_t)kBM};
    const cuuint32_t es[2] = {1, 1};
    if (enc(&map_x, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, (void *)x, dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return LT_ERR_CUDA;
  }
  {
    const cuuint64_t dims[2] = {(cuuint64_t)(N / 2), (cuuint64_t)K};
    const cuuint64_t strides[1] = {(cuuint64_t)(N / 2)};
    const cuuint32_t box[2] = {(cuuint32_t)(kBN / 2), (cuuint32_t)kBK};
    const cuuint32_t es[2] = {1, 1};
    if (enc(&map_w, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, (void *)packed, dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return LT_ERR_CUDA;
  }
  const int64_t tiles_m = (M + kBM - 1) / kBM, tiles_n = N / kBN;
  int splits = choose_splits(tiles_m * tiles_n, K / kBK);
  if (splits > 1 && (!workspace || workspace_bytes < (uint64_t)splits * (uint64_t)M * (uint64_t)N * 4ull)) splits = 1;
  if (tiles_m > 65535) return LT_ERR_UNSUPPORTED;
  GemmArgs ga;
  ga.scales = scales;
  ga.zeros = zeros;
  ga.out = out;
  ga.partial = reinterpret_cast<float *>(workspace);
  ga.d_status = d_status;
  ga.M = M;
  ga.N = N;
  ga.K = K;
  ga.group_size = group_size;
  ga.k_iters = (int32_t)(K / kBK);
  ga.splits = splits;
  static int attr_set[64] = {0};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev >= 0 && dev < 64 && !attr_set[dev]) {
    if (cudaFuncSetAttribute(k_int4_gemm, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemDyn) != cudaSuccess)
      return LT_ERR_CUDA;
    attr_set[dev] = 1;
  }
  k_int4_gemm<<<dim3((unsigned)tiles_n, (unsigned)tiles_m, (unsigned)splits), kGemmThreads, kSmemDyn, st>>>(map_x,
                                                                                                         map_w, ga);
  if (splits > 1) reduce_splits(splits);
  return launch_status();
}
