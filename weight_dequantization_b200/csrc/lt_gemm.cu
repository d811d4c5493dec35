// lt_gemm.cu -- fused INT4 decode -> matrix multiply on the 5th-generation
// tensor cores ("LoreToken-powered GPU memory layer": decode + GEMM, the
// decoded weights feeding a matrix multiply; "GPU Compression Pipeline - TDD
// Roadmap", Phase 4.1: a decoded weight tensor used in input.matmul(weights)).
//
//   out[M, N] = x[M, K] . W[K, N],  W = the INT4 group dequantization of a
//   [K, N] code matrix exactly as lt_dequant_int4 computes it (groups of G
//   along each row of W), x and out binary16, products summed in fp32.
//
// Batches of more than 16 rows: one CTA computes MT x 128 rows (MT = 1, or
// 2 when M > 128) by 256 columns of out over a range of K (the whole of K,
// or a split of it whose fp32 partial sums a second kernel adds in a fixed
// order). Warp roles:
//   warp 0      packed-W producer: for each 64-wide K step one tiled bulk
//               copy (TMA) of the packed INT4 tile (64 rows x 128 bytes,
//               128-byte swizzle) into a 6-deep (MT = 2: 4-deep) ring,
//               completion counted on an mbarrier; a slot is refilled as soon
//               as the decoders are done with it, so this stream runs well
//               ahead of the MMAs;
//   warp 2      x producer: the x tile (MT x 128 rows x 64 fp16, 128-byte
//               swizzle) of each step into a 3-deep ring, refilled when the
//               MMAs that read a slot have completed;
//   warps 3..18 decoders: turn the packed tile into the fp16 B operand in
//               shared memory (N-major, 128-byte swizzle), with the exact
//               half2 arithmetic of lt_dequant_int4 (bit-identical to it), in
//               a 4-deep (MT = 2: 3-deep) ring; scales and zero points are
//               loaded three steps before their use;
//   warp 1      MMA issuer: one thread issues tcgen05.mma kind::f16 (fp32
//               accumulators in tensor memory, MT x (128 x 256) = 256 MT
//               columns), 4 MT K = 16 instructions per step, every B tile
//               shared by the MT accumulators, and tcgen05.commit releases
//               the ring slots;
//   warps 3..18 epilogue: tcgen05.ld of the accumulators (warp w reads lanes
//               32 (w % 4) ... and a quarter of the columns), conversion to
//               binary16 (or the fp32 partial of a split), 16-byte stores.
// Every mbarrier wait is bounded (about a second of clock); a wait that runs
// out sets LT_ERR_TIMEOUT in the status word and the CTA winds down: the
// producer waits (bounded) for its copies in flight, the tensor memory is
// freed, nothing more is written.
#include "lt_common.cuh"

#include <cuda.h>
#include <algorithm>
#include <mutex>
#include <type_traits>

namespace lt {
namespace {

constexpr int kBM = 128, kBN = 256, kBK = 64;
constexpr int kDecWarps = 16;
constexpr int kDec0 = 3;     // first decoder warp (0: packed-W producer, 1: MMA, 2: x producer)
constexpr int kUnits = (kBK * kBN / 32) / (kDecWarps * 32);  // 16-byte packed chunks per decoder thread per step
static_assert(kUnits * kDecWarps * 32 == kBK * kBN / 32, "decoder units must cover a packed tile");
constexpr int kGemmThreads = (kDec0 + kDecWarps) * 32;
constexpr uint32_t kWBytes = kBK * kBN / 2;   // 8192
constexpr uint32_t kBBytes = kBN * kBK * 2;   // 32768
// A CTA of the tcgen05 kernel computes MT 128-row tiles of out (MT = 1 or
// 2) against one 256-column tile: its MT accumulators (256 tensor-memory
// columns each) share every decoded B tile, so with MT = 2 the decode and the
// shared-memory round trip of B are spent once per 256 rows of x.
template <int MT>
struct Tile {
  static constexpr int kStagesW = MT == 1 ? 6 : 4;  // packed-W slots (TMA; freed by the decoders)
  static constexpr int kStagesX = 3;                // x slots (TMA; freed by the MMAs)
  static constexpr int kStagesB = MT == 1 ? 4 : 3;  // decoded-B slots (the decoders run ahead of the MMAs)
  static constexpr uint32_t kABytes = MT * kBM * kBK * 2;  // x tile: 16 or 32 KB
  static constexpr uint32_t kSmemA = 0;
  static constexpr uint32_t kSmemW = kSmemA + kStagesX * kABytes;
  static constexpr uint32_t kSmemB = kSmemW + kStagesW * kWBytes;
  static constexpr uint32_t kSmemTotal = kSmemB + kStagesB * kBBytes;  // 224 KB either way
  static constexpr uint32_t kSmemDyn = kSmemTotal + 1024;              // + alignment slack
  static constexpr uint32_t kTmemCols = 256 * MT;
};
static_assert(Tile<1>::kSmemDyn <= 227 * 1024 - 256 && Tile<2>::kSmemDyn <= 227 * 1024 - 256, "shared memory");
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

// explicit shared-window accesses (32-bit shared addresses)
__device__ __forceinline__ uint2 lds64(uint32_t a) {
  uint2 v;
  asm volatile("ld.shared.v2.u32 {%0, %1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(a));
  return v;
}
__device__ __forceinline__ uint32_t lds32(uint32_t a) {
  uint32_t v;
  asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(a));
  return v;
}
__device__ __forceinline__ uint32_t lds16(uint32_t a) {
  uint16_t v;
  asm volatile("ld.shared.u16 %0, [%1];" : "=h"(v) : "r"(a));
  return v;
}
__device__ __forceinline__ uint32_t lds8(uint32_t a) {
  uint16_t v;
  asm volatile("ld.shared.u8 %0, [%1];" : "=h"(v) : "r"(a));
  return v;
}

__device__ __forceinline__ uint4 lds128(uint32_t a) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(a));
  return v;
}
__device__ __forceinline__ void sts128(uint32_t a, uint4 v) {
  asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(a), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w) : "memory");
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
  // small-batch kernel: TMA box widths (elements) of the scale and zero-point
  // tiles, 0 where that tensor is copied word by word instead
  int32_t sc_box, z_box;
};

template <int MT>
__global__ void __launch_bounds__(kGemmThreads, 1) k_int4_gemm(const __grid_constant__ CUtensorMap map_x,
                                                                 const __grid_constant__ CUtensorMap map_w,
                                                                 const __grid_constant__ GemmArgs a) {
  using T = Tile<MT>;
  constexpr int kStagesW = T::kStagesW, kStagesX = T::kStagesX, kStagesB = T::kStagesB;
  constexpr uint32_t kABytes = T::kABytes, kSmemA = T::kSmemA, kSmemW = T::kSmemW, kSmemB = T::kSmemB;
  constexpr uint32_t kTmemCols = T::kTmemCols;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  __shared__ __align__(8) uint64_t bar_wfull[kStagesW], bar_wempty[kStagesW], bar_xfull[kStagesX],
      bar_xempty[kStagesX], bar_bfull[kStagesB], bar_bempty[kStagesB], bar_acc;
  __shared__ uint32_t s_tmem;
  __shared__ int s_abort;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int n_tile = blockIdx.x, m_tile = blockIdx.y, split = blockIdx.z;
  const int64_t n0 = (int64_t)n_tile * kBN, m0 = (int64_t)m_tile * kBM * MT;
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
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");  // see k_gemm_reduce

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
          // A: K-major 128-byte swizzle, 8-row atoms 1 KB apart, K = 16 slice at +32 bytes
          // (rows 128 mt ... of the x tile start 16 KB further per mt);
          // B: N-major 128-byte swizzle, K = 16 slice = two 1 KB atoms along K
          const uint64_t bd = smem_desc(b0 + 2u * kBAtomK * ks, kBAtomN, kBAtomK);
#pragma unroll
          for (int mt = 0; mt < MT; ++mt) {
            const uint64_t ad = smem_desc(a0 + (uint32_t)mt * (kBM * 128u) + 32u * ks, 16, 1024);
            mma_f16(tmem + 256u * mt, ad, bd, idesc, (it | ks) != 0);
          }
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
      const bool got = mbar_wait(smem_u32(&bar_wfull[s]), (it / kStagesW) & 1) &&
                       (it < kStagesB || mbar_wait(smem_u32(&bar_bempty[b]), ((it / kStagesB) - 1) & 1));
      // the warp goes on only together: it meets at __syncwarp below
      if (!__all_sync(0xffffffffu, got)) {
        fail();
        return false;
      }
      if (*(volatile int *)&s_abort) return false;
      const uint32_t wsrc = sbase + kSmemW + s * kWBytes;
      const uint32_t bdst = sbase + kSmemB + b * kBBytes;
#pragma unroll
      for (int i = 0; i < kUnits; ++i) {
        const int kk = klo + 8 * (khi0 + (kDecWarps / 2) * i);  // row of the step, 0..63
        // packed row kk: 128 bytes (256 codes), 16-byte chunk h at chunk h ^ (kk & 7)
        const uint4 v = lds128(wsrc + kk * 128 + ((h ^ klo) << 4));
        const uint32_t s2 = bcast_half((uint16_t)sc[i]);
        const uint32_t zm = a.zeros ? int4_zero_magic(zr[i]) : 0x54006400u;
        const uint4 o[4] = {int4x8_dequant(v.x, zm, s2), int4x8_dequant(v.y, zm, s2), int4x8_dequant(v.z, zm, s2),
                            int4x8_dequant(v.w, zm, s2)};
        // codes n = 32 h + 8 j .. + 7 of row kk: atom (n / 64, kk / 8), row kk % 8, chunk (n % 64) / 8
        const uint32_t atom = bdst + (h >> 1) * kBAtomN + (kk >> 3) * kBAtomK + klo * 128;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int c = 4 * (h & 1) + j;
          sts128(atom + ((c ^ klo) << 4), o[j]);
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
    const bool acc_ok = __all_sync(0xffffffffu, mbar_wait(smem_u32(&bar_acc), 0));  // tcgen05.ld is warp-wide
    if (!acc_ok) fail();
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
    if (acc_ok && !*(volatile int *)&s_abort && n_it > 0) {
      const int quarter = warp & 3;  // tensor-memory lanes 32 quarter .. + 31
      // each quarter's 256 columns split among its kDecWarps / 4 decoder warps
      constexpr int kCols = kBN / (kDecWarps / 4);
      const int cbeg = ((warp - kDec0) / 4) * kCols;
      for (int cm = 0; cm < MT * kCols; cm += 32) {
        const int mt = cm / kCols, c0 = cbeg + cm % kCols;  // accumulator mt, columns c0 .. c0 + 31
        const int64_t m = m0 + kBM * mt + 32 * quarter + lane;
        uint32_t r[32];
        tmem_ld32(tmem + ((uint32_t)(32 * quarter) << 16) + 256u * mt + (uint32_t)c0, r);
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
// Small batches (M <= 16). With a few rows of x the 128-row tcgen05 tile is
// mostly padding, while its decoded operand still makes a round trip through
// shared memory; the product is bound by streaming the codes from HBM. Here
// the codes stream through a TMA ring and each thread decodes them straight
// into the register operands of mma.sync.m16n8k16 (fp16 in, fp32
// accumulate), computing out^T = W^T . x^T: the MMA's 16 rows are 16 columns
// of W, its 16-deep reduction 16 rows of K, its 8 columns 8 rows of the
// batch (two MMAs per A fragment for 9 .. 16 rows).
//
// One CTA: 256 columns [n0, n0 + 256) over a range of 64-row K tiles (a
// split of K). Warp 0 is the producer: per tile one TMA copy of the packed
// codes (64 rows x 128 bytes, 128-byte swizzle), one of x (8 or 16 batch
// rows x 64 fp16, rows past M zero-filled) and the tile's scales and zero
// points (TMA boxes or word copies, below) into a 7-deep ring, completion
// counted on the slot's full barrier. Warps 1..8: warp 1 + 2 q + h takes
// column half h (128 columns) and rows 16 q .. 16 q + 15 of every tile.
// Lane (g, t) = (lane / 4, lane % 4) holds, for the 8 MMAs j = 0..7 of a
// tile, code byte j of its 8-byte slice (columns 16 g + 2 j and + 1 of the
// half) in rows 2t, 2t+1, 2t+8, 2t+9 of the slot: a byte of row k and the
// same byte of row k + 1 make two half2 A registers, (W[k][c], W[k+1][c])
// for the low nibbles and for the high ones, with the exact arithmetic of
// lt_dequant_int4 (so W is bit-identical to its output). The products are
// exact in fp32; sums are in fp32. At the end the four K slots' sums are
// added in slot order through shared memory.
// ---------------------------------------------------------------------------
constexpr int kVWarps = 8;                       // consumer warps
constexpr int kVThreads = 32 * (kVWarps + 1);    // + the producer warp
constexpr int kVStages = 7;
constexpr int kVPerSM = 2;                       // resident CTAs per SM (launch bounds, shared memory)
constexpr uint32_t kVXBytes = 16 * kBK * 2;      // x tile: up to 16 rows x 64 fp16
// each row's scales and zero points of the strip: a TMA box of 8 or 16
// scales / 16 or 32 zero points per row starting at a 16-byte boundary at or
// below the strip's first group, or (where the tensors' row pitch is not a
// multiple of 16 bytes) the 4-byte words holding them (a strip of 256
// columns spans at most 9 groups of >= 32: <= 5 words of scales, <= 3 of
// zero points)
constexpr uint32_t kVScRow = 20, kVZRow = 12;  // word-copy row pitches
constexpr uint32_t kVScOff = kWBytes + kVXBytes, kVZOff = kVScOff + kBK * 32;
constexpr uint32_t kVStage = kVZOff + kBK * 32;  // 14336, a multiple of 1 KB (swizzle atoms stay aligned)
static_assert(kVStage % 1024 == 0, "stage size");
constexpr uint32_t kVRing = kVStages * kVStage;
constexpr int kVRedPitch = 290;                  // fp32 words per batch row of the reduction buffer
constexpr uint32_t kVRedBytes = 4u * 16u * kVRedPitch * 4u;
static_assert(kVRedBytes <= kVRing, "the reduction buffer reuses the ring");
constexpr uint32_t kVSmemDyn = kVRing + 1024;

// byte JJ of wa (row k) and of wb (row k + 1), columns c (low nibble) and
// c + 1 (high nibble): lo = (W[k][c], W[k+1][c]), hi = (W[k][c+1], W[k+1][c+1])
// as half2, each fp16_rn((q - z) * s) exactly as in lt_dequant_int4: the
// low nibbles OR-ed into the fraction of 1024 (ulp 1), the high ones into
// that of 64 (ulp 1/16) four bits up, the zero points' magic subtracted
// exactly, one rounded multiply by the row's scale.
template <int JJ>
__device__ __forceinline__ void int4_rowpair(uint32_t wa, uint32_t wb, uint32_t zlo, uint32_t zhi, uint32_t s2,
                                             uint32_t &lo, uint32_t &hi) {
  constexpr uint32_t sel = (uint32_t)JJ | ((uint32_t)JJ << 4) | ((uint32_t)(4 + JJ) << 8) | ((uint32_t)(4 + JJ) << 12);
  const uint32_t x = __byte_perm(wa, wb, sel);  // [wa.bJJ, wa.bJJ, wb.bJJ, wb.bJJ]
  uint32_t l, h;
  asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(l) : "r"(x), "r"(0x000F000Fu), "r"(0x64006400u));  // (a & b) | c
  asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(h) : "r"(x), "r"(0x00F000F0u), "r"(0x54005400u));
  lo = hmul2_rn(hsub2_rn(l, zlo), s2);
  hi = hmul2_rn(hsub2_rn(h, zhi), s2);
}
__device__ __forceinline__ uint32_t hadd2_rn(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("add.rn.f16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}
__device__ __forceinline__ void mma_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                          uint32_t b0, uint32_t b1) {
  asm("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// 4-byte copy global -> shared (only the first `bytes` bytes read, the rest
// zero), completion tracked by the thread's next cp.async mbarrier arrive
__device__ __forceinline__ void cp_async4(uint32_t dst, const void *src, uint32_t bytes) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;" ::"r"(dst), "l"(src), "r"(bytes) : "memory");
}
__device__ __forceinline__ void cp_async_arrive(uint32_t bar) {
  asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(bar) : "memory");
}

template <int NB>  // batch rows in blocks of 8 (the MMA's N): 1 or 2
__global__ void __launch_bounds__(kVThreads, kVPerSM) k_int4_gemv(const __grid_constant__ CUtensorMap map_x,
                                                                   const __grid_constant__ CUtensorMap map_w,
                                                                   const __grid_constant__ CUtensorMap map_s,
                                                                   const __grid_constant__ CUtensorMap map_z,
                                                                   const __grid_constant__ GemmArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  __shared__ __align__(8) uint64_t bar_full[kVStages], bar_empty[kVStages];
  __shared__ int s_abort;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int64_t n0 = (int64_t)blockIdx.x * kBN;
  const int split = blockIdx.y;
  const int it_begin = (int)((int64_t)a.k_iters * split / a.splits);
  const int n_it = (int)((int64_t)a.k_iters * (split + 1) / a.splits) - it_begin;
  const int64_t NG = a.N / a.group_size;

  if (tid == 0) {
    for (int s = 0; s < kVStages; ++s) {
      mbar_init(smem_u32(&bar_full[s]), 1 + 32);  // the TMA's arrive + each producer lane's copies
      mbar_init(smem_u32(&bar_empty[s]), kVWarps);
    }
    s_abort = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();
  // the split-sum kernel that follows on the stream may start launching now;
  // it waits for this grid's completion before reading anything
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  const uint32_t sbase = smem_u32(sm);
  auto fail = [&]() {
    s_abort = 1;
    report(a.d_status, LT_ERR_TIMEOUT);
  };

  float acc[NB][8][4];
#pragma unroll
  for (int nb = 0; nb < NB; ++nb)
#pragma unroll
    for (int j = 0; j < 8; ++j)
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[nb][j][e] = 0.f;
  const int cw = warp - 1, h = cw & 1, q = cw >> 1, g = lane >> 2, t = lane & 3;

  if (warp == 0) {
    // ---------------- producer ----------------
    const int64_t gc0 = n0 / a.group_size, gc1 = (n0 + kBN - 1) / a.group_size;
    const uint64_t sc_bytes = 2ull * (uint64_t)a.K * (uint64_t)NG, z_bytes = (uint64_t)a.K * (uint64_t)NG;
    const uint8_t *sc8 = reinterpret_cast<const uint8_t *>(a.scales);
    // per row of a tile (lane, lane + 32): the first word and the word counts
    // do not depend on the tile (k0 is a multiple of 64)
    uint64_t sw0[2], zw0[2];
    uint32_t nws[2], nwz[2];
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      const uint64_t e = (uint64_t)(lane + 32 * r) * (uint64_t)NG;
      const uint64_t sb = 2 * (e + gc0), se = 2 * (e + gc1) + 2, zb = e + gc0, ze = e + gc1 + 1;
      sw0[r] = sb & ~uint64_t(3);
      zw0[r] = zb & ~uint64_t(3);
      nws[r] = a.sc_box ? 0u : (uint32_t)((se - sw0[r] + 3) / 4);
      nwz[r] = (a.zeros && !a.z_box) ? (uint32_t)((ze - zw0[r] + 3) / 4) : 0u;
    }
    const int64_t xs = (gc0 / 8) * 8, xz = (gc0 / 16) * 16;  // TMA boxes start at 16-byte boundaries
    const uint32_t tx_bytes = kWBytes + (uint32_t)(NB * 8 * kBK * 2) + (uint32_t)(kBK * 2 * a.sc_box) + (uint32_t)(kBK * a.z_box);
    int issued = 0;
    for (int it = 0; it < n_it; ++it) {
      const int s = it % kVStages;
      bool ok = true;
      if (it >= kVStages && lane == 0) ok = mbar_wait(smem_u32(&bar_empty[s]), ((it / kVStages) - 1) & 1);
      if (!__shfl_sync(0xffffffffu, (int)ok, 0)) {
        if (lane == 0) fail();
        break;
      }
      if (*(volatile int *)&s_abort) break;
      const int32_t k0 = (it_begin + it) * kBK;
      const uint32_t dst = sbase + s * kVStage, bar = smem_u32(&bar_full[s]);
      if (lane == 0) {
        mbar_expect_tx(bar, tx_bytes);
        tma_load_2d(dst, &map_w, (int32_t)(n0 / 2), k0, bar);
        tma_load_2d(dst + kWBytes, &map_x, k0, 0, bar);
        if (a.sc_box) tma_load_2d(dst + kVScOff, &map_s, (int32_t)xs, k0, bar);
        if (a.z_box) tma_load_2d(dst + kVZOff, &map_z, (int32_t)xz, k0, bar);
      }
      // the tile's scales and zero points: rows lane and lane + 32, the
      // 4-byte words covering groups gc0 .. gc1 (a word reaching past a
      // tensor's end is read only up to it: the last tile of K)
      const uint64_t step_sc = 2ull * (uint64_t)(it_begin + it) * kBK * (uint64_t)NG;
      const uint64_t step_z = (uint64_t)(it_begin + it) * kBK * (uint64_t)NG;
      const bool last = it_begin + it == a.k_iters - 1;
#pragma unroll
      for (int r = 0; r < 2; ++r) {
        const int rr = lane + 32 * r;
        for (uint32_t j = 0; j < nws[r]; ++j) {  // (nws = 0 when the scales come by TMA; nwz likewise)
          const uint64_t o = sw0[r] + step_sc + 4 * j;
          cp_async4(dst + kVScOff + rr * kVScRow + 4 * j, sc8 + o, last && sc_bytes - o < 4 ? (uint32_t)(sc_bytes - o) : 4u);
        }
        for (uint32_t j = 0; j < nwz[r]; ++j) {
          const uint64_t o = zw0[r] + step_z + 4 * j;
          cp_async4(dst + kVZOff + rr * kVZRow + 4 * j, a.zeros + o, last && z_bytes - o < 4 ? (uint32_t)(z_bytes - o) : 4u);
        }
      }
      cp_async_arrive(bar);
      issued = it + 1;
    }
    // on an abort, let the copies in flight land before the CTA exits
    if (*(volatile int *)&s_abort && lane == 0)
      for (int it = issued > kVStages ? issued - kVStages : 0; it < issued; ++it)
        mbar_wait(smem_u32(&bar_full[it % kVStages]), (it / kVStages) & 1);
  } else {
    // ---------------- consumers ----------------
    const int r0 = 16 * q + 2 * t;  // rows r0, r0 + 1, r0 + 8, r0 + 9 of every tile
    // 128-byte swizzle: 16-byte chunk c of row r sits at chunk c ^ (r % 8)
    const uint32_t chunk = 4 * h + (g >> 1), within = 8 * (g & 1);
    const uint32_t off0 = r0 * 128 + ((chunk ^ (uint32_t)(2 * t)) << 4) + within;
    const uint32_t off1 = (r0 + 1) * 128 + ((chunk ^ (uint32_t)(2 * t + 1)) << 4) + within;
    const uint32_t xo0 = kWBytes + g * 128 + (((uint32_t)(2 * q) ^ (uint32_t)g) << 4) + 4 * t;
    const uint32_t xo1 = kWBytes + g * 128 + (((uint32_t)(2 * q + 1) ^ (uint32_t)g) << 4) + 4 * t;
    const int64_t gcol = (n0 + 128 * h + 16 * g) / a.group_size, gc0 = n0 / a.group_size;
    const bool has_z = a.zeros != nullptr;
    // where this thread's scale and zero point sit in a row's words: row k's
    // words start at 4-byte boundary below element k NG + gc0; the offset
    // depends on k only through k mod 4, and the thread's rows r0 + {0, 1,
    // 8, 9} of a tile (k0 a multiple of 64) have k mod 4 = (r0 + {0, 1}) mod 4
    // (from a TMA box: the offset of gcol from the box's first element, the
    // same in every row)
    uint32_t soff[2], zoff[2];
#pragma unroll
    for (int p = 0; p < 2; ++p) {
      const uint64_t e = (uint64_t)((r0 + p) & 3) * (uint64_t)(NG & 3) + (uint64_t)gc0;
      soff[p] = a.sc_box ? 2u * (uint32_t)(gcol - (gc0 / 8) * 8) : 2u * (uint32_t)(e & 1) + 2u * (uint32_t)(gcol - gc0);
      zoff[p] = a.z_box ? (uint32_t)(gcol - (gc0 / 16) * 16) : (uint32_t)(e & 3) + (uint32_t)(gcol - gc0);
    }
    const uint32_t sp = a.sc_box ? 2u * (uint32_t)a.sc_box : kVScRow, zp = a.z_box ? (uint32_t)a.z_box : kVZRow;
    const uint32_t srow0 = kVScOff + r0 * sp, zrow0 = kVZOff + r0 * zp;
    bool ok = true;
    for (int it = 0; it < n_it && ok; ++it) {
      const int s = it % kVStages;
      // the warp goes on only together (a wait that ran out in one lane ends the whole warp's loop)
      if (!__all_sync(0xffffffffu, mbar_wait(smem_u32(&bar_full[s]), (it / kVStages) & 1))) {
        if (lane == 0) fail();
        ok = false;
        break;
      }
      if (*(volatile int *)&s_abort) break;
      const uint32_t st = sbase + s * kVStage;  // shared-window address of the slot
      const uint2 w0 = lds64(st + off0);
      const uint2 w1 = lds64(st + off1);
      const uint2 w2 = lds64(st + off0 + 8 * 128);
      const uint2 w3 = lds64(st + off1 + 8 * 128);
      uint32_t b0[NB], b1[NB];
#pragma unroll
      for (int nb = 0; nb < NB; ++nb) {  // batch rows g + 8 nb: 8 x rows (1 KB) further, the same swizzle
        b0[nb] = lds32(st + xo0 + 1024 * nb);
        b1[nb] = lds32(st + xo1 + 1024 * nb);
      }
      uint32_t sc[4], zr[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const uint32_t row = (i & 1) + 8 * (i >> 1);
        sc[i] = lds16(st + srow0 + row * sp + soff[i & 1]);
        zr[i] = has_z ? lds8(st + zrow0 + row * zp + zoff[i & 1]) : 0u;
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&bar_empty[s]));  // the slot is in registers now
      // zero-point magics (1024 + z, 64 + z) and scales of the row pairs (r0, r0 + 1), (r0 + 8, r0 + 9)
      const uint32_t zloA = 0x64006400u | zr[0] | (zr[1] << 16), zloB = 0x64006400u | zr[2] | (zr[3] << 16);
      const uint32_t zhiA = has_z ? hadd2_rn(hsub2_rn(zloA, 0x64006400u), 0x54005400u) : 0x54005400u;
      const uint32_t zhiB = has_z ? hadd2_rn(hsub2_rn(zloB, 0x64006400u), 0x54005400u) : 0x54005400u;
      const uint32_t sA = sc[0] | (sc[1] << 16), sB = sc[2] | (sc[3] << 16);
      uint32_t a0, a1, a2, a3;
#define LT_GEMV_MMA(J, WA, WB, WC, WD)                  \
  int4_rowpair<(J) & 3>(WA, WB, zloA, zhiA, sA, a0, a1); \
  int4_rowpair<(J) & 3>(WC, WD, zloB, zhiB, sB, a2, a3); \
  for (int nb = 0; nb < NB; ++nb) mma_16816(acc[nb][J], a0, a1, a2, a3, b0[nb], b1[nb]);
      LT_GEMV_MMA(0, w0.x, w1.x, w2.x, w3.x)
      LT_GEMV_MMA(1, w0.x, w1.x, w2.x, w3.x)
      LT_GEMV_MMA(2, w0.x, w1.x, w2.x, w3.x)
      LT_GEMV_MMA(3, w0.x, w1.x, w2.x, w3.x)
      LT_GEMV_MMA(4, w0.y, w1.y, w2.y, w3.y)
      LT_GEMV_MMA(5, w0.y, w1.y, w2.y, w3.y)
      LT_GEMV_MMA(6, w0.y, w1.y, w2.y, w3.y)
      LT_GEMV_MMA(7, w0.y, w1.y, w2.y, w3.y)
#undef LT_GEMV_MMA
    }
  }
  __syncthreads();  // every tile consumed (or the CTA aborted): the ring is free
  if (*(volatile int *)&s_abort || n_it <= 0) return;
  // ---------------- the four K slots' sums, in slot order ----------------
  // red[q][m][c + c / 32] (m < 16): the padding and the pitch (290 = 2 mod 32) make
  // both the scattered stores below and the row reads after them conflict-free
  float *red = reinterpret_cast<float *>(sm);
  if (warp > 0) {
#pragma unroll
    for (int nb = 0; nb < NB; ++nb)
#pragma unroll
      for (int j = 0; j < 8; ++j)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int c = 128 * h + 16 * g + 2 * j + (e >> 1), m = 8 * nb + 2 * t + (e & 1);
          red[(q * 16 + m) * kVRedPitch + c + (c >> 5)] = acc[nb][j][e];
        }
  }
  __syncthreads();
  if (warp > 0) {
    const int c = tid - 32;  // 0 .. 255
    for (int m = 0; m < 8 * NB && m < a.M; ++m) {
      float v = red[(0 * 16 + m) * kVRedPitch + c + (c >> 5)];
#pragma unroll
      for (int qq = 1; qq < 4; ++qq) v += red[(qq * 16 + m) * kVRedPitch + c + (c >> 5)];
      if (a.splits == 1)
        a.out[(int64_t)m * a.N + n0 + c] = __half_as_ushort(__float2half_rn(v));
      else
        a.partial[((int64_t)split * a.M + m) * a.N + n0 + c] = v;
    }
  }
}

// K splits of the small-batch kernel: the fewest that fill at least 90 % of
// the resident CTA slots of the waves they take (else the best fill), each
// split at least one tile
int gemv_splits(int64_t N, int64_t K) {
  const int64_t strips = N / kBN, k_tiles = K / kBK, slots = (int64_t)kVPerSM * num_sms();
  int best = 1;
  double best_fill = 0.0;
  for (int64_t s = 1; s <= 64 && s <= k_tiles; ++s) {
    const int64_t ctas = strips * s, waves = (ctas + slots - 1) / slots;
    const double fill = (double)ctas / (double)(waves * slots);
    if (fill >= 0.9) return (int)s;
    if (fill > best_fill + 1e-9) {
      best_fill = fill;
      best = (int)s;
    }
  }
  return best;
}

// out[m, n] = fp16_rn(sum over splits s = 0, 1, ... of partial[s, m, n]), in that order
__global__ void __launch_bounds__(256) k_gemm_reduce(const float4 *__restrict__ partial, int64_t mn4, int splits,
                                                     uint2 *__restrict__ out) {
  asm volatile("griddepcontrol.wait;" ::: "memory");  // the partials are complete (no-op in a plain launch)
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
  if (M <= 16) {
    s = gemv_splits(N, K);
  } else {
    const int64_t rows = M > kBM ? 2 * kBM : kBM;  // rows of out per CTA (the tcgen05 kernel's MT)
    const int64_t tiles = ((M + rows - 1) / rows) * (N / kBN);
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
  const bool small = M <= 16;  // the mma.sync kernel (x tile of 8 or 16 rows) instead of the tcgen05 one (128 rows)
  const int nb = M <= 8 ? 1 : 2;
  const int mt = M > kBM ? 2 : 1;  // tcgen05 kernel: 128-row tiles of out per CTA
  encode_tiled_t enc = encoder();
  if (!enc) return LT_ERR_CUDA;
  CUtensorMap map_x, map_w;
  {
    const cuuint64_t dims[2] = {(cuuint64_t)K, (cuuint64_t)M};
    const cuuint64_t strides[1] = {(cuuint64_t)K * 2};
    const cuuint32_t box[2] = {(cuuint32_t)kBK, (cuuint32_t)(small ? 8 * nb : kBM * mt)};
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
  const int64_t tiles_m = (M + kBM * mt - 1) / (kBM * mt), tiles_n = N / kBN;
  if (tiles_m > 65535) return LT_ERR_UNSUPPORTED;
  int splits = small ? gemv_splits(N, K) : choose_splits(tiles_m * tiles_n, K / kBK);
  if (splits > 1 && (!workspace || workspace_bytes < (uint64_t)splits * (uint64_t)M * (uint64_t)N * 4ull)) splits = 1;
  // small batch: scale / zero-point tiles by TMA where the row pitch is a
  // multiple of 16 bytes and a box of the chosen width, started at the
  // 16-byte boundary at or below each strip's first group, covers the
  // strip's last group (else word copies)
  int sc_box = 0, z_box = 0;
  CUtensorMap map_s = map_w, map_z = map_w;
  if (small) {
    const int64_t NG = N / group_size, strips = N / kBN;
    int64_t span_s = 0, span_z = 0;  // max over strips of last group - box start
    for (int64_t j = 0; j < strips; ++j) {
      const int64_t g0 = j * kBN / group_size, g1 = (j * kBN + kBN - 1) / group_size;
      span_s = std::max(span_s, g1 - (g0 / 8) * 8);
      span_z = std::max(span_z, g1 - (g0 / 16) * 16);
    }
    if (aligned(scales, 16) && (NG * 2) % 16 == 0 && span_s < 16) sc_box = span_s < 8 ? 8 : 16;
    if (zeros && aligned(zeros, 16) && NG % 16 == 0 && span_z < 32) z_box = span_z < 16 ? 16 : 32;
    const cuuint32_t es[2] = {1, 1};
    if (sc_box) {
      const cuuint64_t dims[2] = {(cuuint64_t)NG, (cuuint64_t)K};
      const cuuint64_t strides[1] = {(cuuint64_t)NG * 2};
      const cuuint32_t box[2] = {(cuuint32_t)sc_box, (cuuint32_t)kBK};
      if (enc(&map_s, CU_TENSOR_MAP_DATA_TYPE_UINT16, 2, (void *)scales, dims, strides, box, es,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
        return LT_ERR_CUDA;
    }
    if (z_box) {
      const cuuint64_t dims[2] = {(cuuint64_t)NG, (cuuint64_t)K};
      const cuuint64_t strides[1] = {(cuuint64_t)NG};
      const cuuint32_t box[2] = {(cuuint32_t)z_box, (cuuint32_t)kBK};
      if (enc(&map_z, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, (void *)zeros, dims, strides, box, es,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
        return LT_ERR_CUDA;
    }
  }
  GemmArgs ga;
  ga.sc_box = sc_box;
  ga.z_box = z_box;
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
  static int attr_set[4][64] = {{0}};
  int dev = 0;
  cudaGetDevice(&dev);
  const int which = small ? nb : 2 + mt;  // 1, 2: k_int4_gemv<nb>; 3, 4: k_int4_gemm<mt>
  if (dev >= 0 && dev < 64 && !attr_set[which - 1][dev]) {
    const void *fn = which == 1   ? (const void *)k_int4_gemv<1>
                     : which == 2 ? (const void *)k_int4_gemv<2>
                     : which == 3 ? (const void *)k_int4_gemm<1>
                                  : (const void *)k_int4_gemm<2>;
    const int bytes = (int)(small ? kVSmemDyn : (mt == 1 ? Tile<1>::kSmemDyn : Tile<2>::kSmemDyn));
    if (cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) != cudaSuccess)
      return LT_ERR_CUDA;
    attr_set[which - 1][dev] = 1;
  }
  cudaStream_t st = (cudaStream_t)stream;
  const dim3 grid_tc((unsigned)tiles_n, (unsigned)tiles_m, (unsigned)splits);
  if (small) {
    if (nb == 1)
      k_int4_gemv<1><<<dim3((unsigned)tiles_n, (unsigned)splits), kVThreads, kVSmemDyn, st>>>(map_x, map_w, map_s,
                                                                                              map_z, ga);
    else
      k_int4_gemv<2><<<dim3((unsigned)tiles_n, (unsigned)splits), kVThreads, kVSmemDyn, st>>>(map_x, map_w, map_s,
                                                                                              map_z, ga);
  } else if (mt == 1) {
    k_int4_gemm<1><<<grid_tc, kGemmThreads, Tile<1>::kSmemDyn, st>>>(map_x, map_w, ga);
  } else {
    k_int4_gemm<2><<<grid_tc, kGemmThreads, Tile<2>::kSmemDyn, st>>>(map_x, map_w, ga);
  }
  if (splits > 1) {
    // the split sums in order; launched as a programmatic dependent of the
    // product kernel, so its launch overlaps that kernel's tail (it waits for
    // the kernel's completion and memory before reading a partial)
    const int64_t mn4 = M * N / 4;
    int64_t g = (mn4 + 255) / 256;
    const int64_t cap = (int64_t)num_sms() * 8;
    if (g > cap) g = cap;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)g);
    cfg.blockDim = dim3(256);
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, k_gemm_reduce, reinterpret_cast<const float4 *>(workspace), mn4, splits,
                           reinterpret_cast<uint2 *>(out)) != cudaSuccess)
      return launch_status();
  }
  return launch_status();
}
