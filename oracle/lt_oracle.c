/*
 * lt_oracle.c -- TEST INFRASTRUCTURE ONLY.
 *
 * A plain, slow, element-by-element CPU statement of what the on-device
 * decoders compute. It exists so that the CUDA library can be checked
 * against it; no product code path may call, link or load it. It shares no
 * code, header, table or constant generator with the CUDA library or with
 * the input generator; only the bytes those produce pass through it.
 *
 * Sources it follows (web pages, cited by title and section):
 *   [R]  "GPU Compression Pipeline - TDD Roadmap" (abaddon docs):
 *        Phase 1.1 INT4 Dequantization (test_int4_dequant_basic: packed
 *        [0x10,0x32,0x54,0x76] are codes 0..7, low nibble first; scale f16,
 *        zero point; "block-level dequantization (GPTQ/AWQ compatible)"),
 *        Phase 1.2 INT8 Dequantization ("Expected: values * scale";
 *        per-tensor and per-channel scales), Phase 2.1 LZ4 + INT4 Fused
 *        Kernel (cpu_lz4_decompress_then_dequant: decompress, then
 *        dequantize), Phase 3.1 (64 KB LZ4 blocks), Phase 6.1 (block_size
 *        65536).
 *   [L]  "LoreToken-powered GPU memory layer" (freemwiki ChatGPT export):
 *        compression strategies, "Zero-run encoding - extremely effective on
 *        ReLU activations that are mostly zero"; "Value dictionary
 *        compression" for tensors that hold few distinct values (a
 *        dictionary plus small indices).
 *   [S]  "GPU sidecar brain" explanation (freemwiki ChatGPT export), its
 *        list of strategies: value dictionaries store small integer codes
 *        plus a tiny lookup table.
 *   LZ4 block format: the public description of the LZ4 block layout
 *        (token, literal run, 2-byte little-endian offset, match length
 *        with minimum 4, 255-continuation length bytes, literal-only last
 *        sequence). The pages name LZ4 but do not restate its format.
 *   IEEE 754-2008 binary16 for the fp16 encoding and round-to-nearest-even.
 *   XXH3: the 64-bit XXH3 hash of xxHash 0.8 as its author publishes it,
 *        for the checksums [R] Phase 6.1 (HCT Format V2) asks for; the
 *        HCT v2 byte layout is this oracle's reading (the page lists the
 *        header as a task without designing it).
 *
 * Readings where the pages are silent (each stated again in the design
 * notes): the dequantized value is (q - z) * s with one rounding to fp16
 * (round to nearest, ties to even, subnormals kept, overflow to infinity);
 * groups run along the contiguous row of a row-major [rows, cols] tensor;
 * per-channel means per row; the zero-run chunk format is the
 * (u16 zero run, u16 literal count, fp16 literals)* record list with
 * little-endian fields; a value dictionary is one table of 2^bits fp16
 * entries per tensor, indexed by bits-wide fields packed least-significant
 * bits first (the INT4 nibble order); decode -> GEMM multiplies an fp16
 * input by the decoded [K, N] weight.
 *
 * Parity unpinned by the pages (the tests pin this code's arithmetic, but
 * the pages fix no value for these readings): the zero point for z != 0,
 * the zero-run byte layout, the value-dictionary layout beyond the 4-bit
 * order, and the HCT v2 byte layout.
 *
 * Status values returned by the decoders: 0 ok, 4 corrupt stream, 5 decoded
 * size differs from the declared size, 1 invalid argument. The container
 * validator has its own (HCT_*, below).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORACLE_EXPORT __attribute__((visibility("default")))

enum { ORACLE_OK = 0, ORACLE_INVALID = 1, ORACLE_CORRUPT = 4, ORACLE_SIZE = 5 };

/* ------------------------------------------------------------------ */
/* IEEE 754 binary16                                                   */
/* ------------------------------------------------------------------ */

/* binary16 bits -> exact double value. Layout: 1 sign bit, 5 exponent bits
 * (bias 15), 10 fraction bits; exponent 0 is zero/subnormal (f * 2^-24),
 * exponent 31 is infinity (f == 0) or NaN. */
ORACLE_EXPORT double oracle_f16_to_f64(uint16_t h) {
  int sign = (h >> 15) & 1;
  int e = (h >> 10) & 0x1F;
  int f = h & 0x3FF;
  double v;
  if (e == 0) {
    v = ldexp((double)f, -24);
  } else if (e == 31) {
    v = f ? NAN : INFINITY;
  } else {
    v = ldexp((double)(1024 + f), e - 25);
  }
  return sign ? -v : v;
}

/* double -> binary16 bits, round to nearest, ties to even.
 * Method: the representable binary16 values near |x| are the integer
 * multiples of the quantum 2^(max(E, -14) - 10), E = floor(log2 |x|); round
 * |x| / quantum to the nearest integer (ties to the even integer), which is
 * exact arithmetic in double, then encode that multiple. Results at or above
 * 2^16 are infinity (the largest finite value is 65504). NaN becomes the
 * quiet NaN 0x7E00 with the input's sign. */
ORACLE_EXPORT uint16_t oracle_f16_from_f64(double x) {
  uint16_t sign = signbit(x) ? 0x8000 : 0;
  if (isnan(x)) return (uint16_t)(sign | 0x7E00);
  double a = fabs(x);
  if (isinf(a)) return (uint16_t)(sign | 0x7C00);
  if (a == 0.0) return sign;
  int e2;
  frexp(a, &e2); /* a = m * 2^e2, m in [0.5, 1) -> floor(log2 a) = e2 - 1 */
  int E = e2 - 1;
  if (E < -14) E = -14; /* subnormal range: fixed quantum 2^-24 */
  double quantum = ldexp(1.0, E - 10);
  double k = a / quantum; /* exact: division by a power of two */
  double kf = floor(k);
  double rem = k - kf;
  if (rem > 0.5 || (rem == 0.5 && fmod(kf, 2.0) != 0.0)) kf += 1.0;
  double v = kf * quantum; /* the rounded magnitude */
  if (v >= 65536.0) return (uint16_t)(sign | 0x7C00);
  if (v < ldexp(1.0, -14)) {
    /* subnormal (or +-0): fraction = v / 2^-24 */
    return (uint16_t)(sign | (uint16_t)ldexp(v, 24));
  }
  int ev2;
  double m = frexp(v, &ev2); /* v = m * 2^ev2, m in [0.5, 1) */
  int exp_field = (ev2 - 1) + 15;
  uint16_t frac = (uint16_t)(ldexp(m, 11) - 1024.0); /* (2m - 1) * 1024 */
  return (uint16_t)(sign | (uint16_t)(exp_field << 10) | frac);
}

ORACLE_EXPORT void oracle_f16_from_f64_array(const double *x, int64_t n, uint16_t *out) {
  for (int64_t i = 0; i < n; ++i) out[i] = oracle_f16_from_f64(x[i]);
}

ORACLE_EXPORT void oracle_f16_to_f64_array(const uint16_t *h, int64_t n, double *out) {
  for (int64_t i = 0; i < n; ++i) out[i] = oracle_f16_to_f64(h[i]);
}

/* ------------------------------------------------------------------ */
/* INT4 group dequantization   [R] Phase 1.1                          */
/* ------------------------------------------------------------------ */

/* Code k of the packed array: byte k/2, low nibble for even k, high nibble
 * for odd k (the worked example lists [0x10,0x32,0x54,0x76] as 0..7). */
static int int4_code(const uint8_t *packed, int64_t k) {
  uint8_t b = packed[k / 2];
  return (k % 2 == 0) ? (b & 0x0F) : (b >> 4);
}

/* out[r, c] = fp16_rn((q[r, c] - z[g]) * s[g]), g = r * (cols / G) + c / G:
 * groups of G consecutive codes along each row of a row-major
 * [rows, cols] tensor. zeros == NULL means zero point 0. */
ORACLE_EXPORT int oracle_dequant_int4(const uint8_t *packed, const uint16_t *scales, const uint8_t *zeros,
                                      int64_t rows, int64_t cols, int64_t group_size, uint16_t *out) {
  if (rows < 0 || cols < 0 || group_size < 1 || (cols % group_size) != 0) return ORACLE_INVALID;
  int64_t groups_per_row = cols / group_size;
  for (int64_t r = 0; r < rows; ++r) {
    for (int64_t c = 0; c < cols; ++c) {
      int64_t k = r * cols + c;
      int64_t g = r * groups_per_row + c / group_size;
      int q = int4_code(packed, k);
      int z = zeros ? zeros[g] : 0;
      double s = oracle_f16_to_f64(scales[g]);
      out[k] = oracle_f16_from_f64((double)(q - z) * s);
    }
  }
  return ORACLE_OK;
}

/* ------------------------------------------------------------------ */
/* INT8 dequantization   [R] Phase 1.2                                 */
/* ------------------------------------------------------------------ */

/* per_row == 0: one scale (and zero point) for the tensor;
 * per_row == 1: one per row (output channel).
 * out[r, c] = fp16_rn((q[r, c] - z) * s). zeros == NULL means 0. */
ORACLE_EXPORT int oracle_dequant_int8(const int8_t *q, const uint16_t *scales, const int8_t *zeros, int per_row,
                                      int64_t rows, int64_t cols, uint16_t *out) {
  if (rows < 0 || cols < 0 || (per_row != 0 && per_row != 1)) return ORACLE_INVALID;
  for (int64_t r = 0; r < rows; ++r) {
    int64_t i = per_row ? r : 0;
    double s = oracle_f16_to_f64(scales[i]);
    int z = zeros ? zeros[i] : 0;
    for (int64_t c = 0; c < cols; ++c) {
      int64_t k = r * cols + c;
      out[k] = oracle_f16_from_f64((double)((int)q[k] - z) * s);
    }
  }
  return ORACLE_OK;
}

/* ------------------------------------------------------------------ */
/* Value-dictionary decoding   [L] compression strategies, [S]         */
/* ------------------------------------------------------------------ */

/* Index k: the bits-wide field that starts at bit k * bits of the packed
 * byte stream, bit 0 being the least significant bit of byte 0 (for
 * bits == 4 this is the INT4 order above: even k in the low nibble). A
 * field never straddles two bytes because bits divides 8. */
static unsigned dict_index(const uint8_t *packed, int64_t k, int bits) {
  uint64_t bit = (uint64_t)k * (uint64_t)bits;
  unsigned byte = packed[bit / 8];
  return (byte >> (bit % 8)) & ((1u << bits) - 1u);
}

/* out[k] = dict[index k] for k in [0, n): the entry's fp16 bit pattern is
 * copied as it is (no arithmetic, so NaN payloads and -0 survive). dict
 * holds 2^bits entries; bits is 1, 2, 4 or 8. */
ORACLE_EXPORT int oracle_value_dict_decode(const uint8_t *packed, int bits, const uint16_t *dict, int64_t n,
                                           uint16_t *out) {
  if (n < 0 || !(bits == 1 || bits == 2 || bits == 4 || bits == 8)) return ORACLE_INVALID;
  for (int64_t k = 0; k < n; ++k) out[k] = dict[dict_index(packed, k, bits)];
  return ORACLE_OK;
}

/* ------------------------------------------------------------------ */
/* Zero-run decoding   [L] compression strategies                      */
/* ------------------------------------------------------------------ */

static unsigned rd_u16le(const uint8_t *p) { return (unsigned)p[0] | ((unsigned)p[1] << 8); }

/* Chunk c covers elements [c * chunk_elems, min(n, (c + 1) * chunk_elems)).
 * Its bytes are enc[offsets[c], offsets[c + 1]), a list of records
 * (u16 zero_run, u16 literal_count, literal_count fp16 bit patterns).
 * Each record emits zero_run elements equal to +0 (0x0000) and then the
 * literals as they are. Decoding stops once the chunk is full; remaining
 * bytes are padding. A record that would overrun the chunk, or a record
 * that does not fit in the chunk's bytes, is a corrupt stream; running out
 * of bytes before the chunk is full is a size mismatch. */
ORACLE_EXPORT int oracle_zrle_decode(const uint8_t *enc, uint64_t enc_bytes, const uint64_t *offsets, int64_t n,
                                     int64_t chunk_elems, uint16_t *out) {
  if (n < 0 || chunk_elems < 1) return ORACLE_INVALID;
  int status = ORACLE_OK;
  int64_t n_chunks = (n + chunk_elems - 1) / chunk_elems;
  for (int64_t c = 0; c < n_chunks; ++c) {
    int64_t e0 = c * chunk_elems;
    int64_t len = n - e0 < chunk_elems ? n - e0 : chunk_elems;
    for (int64_t i = 0; i < len; ++i) out[e0 + i] = 0;
    uint64_t b0 = offsets[c], b1 = offsets[c + 1];
    if (b1 < b0 || b1 > enc_bytes) {
      if (!status) status = ORACLE_CORRUPT;
      continue;
    }
    uint64_t p = b0;
    int64_t done = 0;
    while (done < len) {
      if (p + 4 > b1) {
        if (!status) status = ORACLE_SIZE;
        break;
      }
      int64_t zrun = rd_u16le(enc + p);
      int64_t nlit = rd_u16le(enc + p + 2);
      p += 4;
      if (done + zrun + nlit > len || p + 2 * (uint64_t)nlit > b1) {
        if (!status) status = ORACLE_CORRUPT;
        break;
      }
      for (int64_t i = 0; i < zrun; ++i) out[e0 + done + i] = 0;
      done += zrun;
      for (int64_t i = 0; i < nlit; ++i) out[e0 + done + i] = (uint16_t)rd_u16le(enc + p + 2 * i);
      done += nlit;
      p += 2 * (uint64_t)nlit;
    }
  }
  return status;
}

/* ------------------------------------------------------------------ */
/* LZ4 block decoding   (public LZ4 block format; [R] Phases 2.1, 3.1) */
/* ------------------------------------------------------------------ */

/* Decode one raw LZ4 block src[0, src_len) into dst, which must come out
 * exactly dst_len bytes long. Sequence: token; literal count = high nibble,
 * extended by following bytes while they are 255 (the first byte below 255
 * ends it) when the nibble is 15; the literals; unless the input ends right
 * after the literals: 2-byte little-endian offset (1..65535, not beyond the
 * bytes already produced), match length = low nibble + 4, extended the same
 * way; the match copies byte by byte from dst[pos - offset], so an offset
 * smaller than the length repeats the last `offset` bytes. */
ORACLE_EXPORT int oracle_lz4_block_decode(const uint8_t *src, uint64_t src_len, uint8_t *dst, uint64_t dst_len) {
  uint64_t ip = 0, op = 0;
  if (src_len == 0) return dst_len == 0 ? ORACLE_OK : ORACLE_SIZE;
  for (;;) {
    if (ip >= src_len) return ORACLE_CORRUPT;
    unsigned token = src[ip++];
    uint64_t lit = token >> 4;
    if (lit == 15) {
      unsigned b;
      do {
        if (ip >= src_len) return ORACLE_CORRUPT;
        b = src[ip++];
        lit += b;
      } while (b == 255);
    }
    if (ip + lit > src_len) return ORACLE_CORRUPT;
    if (op + lit > dst_len) return ORACLE_CORRUPT;
    for (uint64_t i = 0; i < lit; ++i) dst[op + i] = src[ip + i];
    ip += lit;
    op += lit;
    if (ip == src_len) break; /* the last sequence holds literals only */
    if (ip + 2 > src_len) return ORACLE_CORRUPT;
    uint64_t off = (uint64_t)src[ip] | ((uint64_t)src[ip + 1] << 8);
    ip += 2;
    if (off == 0 || off > op) return ORACLE_CORRUPT;
    uint64_t mlen = (token & 0x0F) + 4;
    if ((token & 0x0F) == 15) {
      unsigned b;
      do {
        if (ip >= src_len) return ORACLE_CORRUPT;
        b = src[ip++];
        mlen += b;
      } while (b == 255);
    }
    if (op + mlen > dst_len) return ORACLE_CORRUPT;
    for (uint64_t i = 0; i < mlen; ++i) dst[op + i] = dst[op - off + i];
    op += mlen;
  }
  return op == dst_len ? ORACLE_OK : ORACLE_SIZE;
}

/* Independent blocks: block b decodes enc[offsets[b], offsets[b + 1]) into
 * dst[b * block_bytes, ...) (the last block holds the remainder of
 * dst_len). Decodes every block; returns the first failing status. */
ORACLE_EXPORT int oracle_lz4_decode_blocks(const uint8_t *comp, uint64_t comp_bytes, const uint64_t *offsets,
                                           int64_t block_bytes, uint8_t *dst, uint64_t dst_len) {
  if (block_bytes < 1) return ORACLE_INVALID;
  int status = ORACLE_OK;
  uint64_t n_blocks = (dst_len + (uint64_t)block_bytes - 1) / (uint64_t)block_bytes;
  for (uint64_t b = 0; b < n_blocks; ++b) {
    uint64_t d0 = b * (uint64_t)block_bytes;
    uint64_t dl = dst_len - d0 < (uint64_t)block_bytes ? dst_len - d0 : (uint64_t)block_bytes;
    uint64_t s0 = offsets[b], s1 = offsets[b + 1];
    int st;
    if (s1 < s0 || s1 > comp_bytes)
      st = ORACLE_CORRUPT;
    else
      st = oracle_lz4_block_decode(comp + s0, s1 - s0, dst + d0, dl);
    if (st && !status) status = st;
  }
  return status;
}

/* [R] Phase 2.1 cpu_lz4_decompress_then_dequant: decompress all blocks into
 * the packed INT4 bytes, then dequantize them as oracle_dequant_int4. */
ORACLE_EXPORT int oracle_lz4_int4_decode(const uint8_t *comp, uint64_t comp_bytes, const uint64_t *offsets,
                                         int64_t block_bytes, const uint16_t *scales, const uint8_t *zeros,
                                         int64_t rows, int64_t cols, int64_t group_size, uint16_t *out) {
  if (rows < 0 || cols < 0) return ORACLE_INVALID;
  int64_t n = rows * cols;
  uint64_t packed_len = (uint64_t)((n + 1) / 2);
  uint8_t *packed = (uint8_t *)calloc(packed_len ? packed_len : 1, 1);
  if (!packed) return ORACLE_INVALID;
  int st = oracle_lz4_decode_blocks(comp, comp_bytes, offsets, block_bytes, packed, packed_len);
  int st2 = oracle_dequant_int4(packed, scales, zeros, rows, cols, group_size, out);
  free(packed);
  return st ? st : st2;
}

/* ------------------------------------------------------------------ */
/* XXH3 64-bit hash with a caller-given secret   [R] Phase 6.1         */
/* ------------------------------------------------------------------ */
/* [R] Phase 6.1 (HCT Format V2, Checksums & Validation) asks for XXH3
 * checksums. This is the XXH3 64-bit hash of xxHash 0.8, written from the
 * algorithm's published description, in its "with secret" form: the secret
 * (at least 136 bytes) is an input, the seed is 0. The input is cut by
 * length into the classes 0, 1-3, 4-8, 9-16, 17-128, 129-240 and longer;
 * each class mixes input words with secret words by 64x64->128-bit
 * multiplies folded to 64 bits, and ends in an avalanche. Everything is
 * arithmetic modulo 2^64 on little-endian words. */

#define XXH_P32_1 0x9E3779B1u
#define XXH_P32_2 0x85EBCA77u
#define XXH_P32_3 0xC2B2AE3Du
#define XXH_P64_1 0x9E3779B185EBCA87ull
#define XXH_P64_2 0xC2B2AE3D27D4EB4Full
#define XXH_P64_3 0x165667B19E3779F9ull
#define XXH_P64_4 0x85EBCA77C2B2AE63ull
#define XXH_P64_5 0x27D4EB2F165667C5ull
#define XXH_MX1 0x165667919E3779F9ull
#define XXH_MX2 0x9FB21C651E98DF25ull

static uint64_t le64(const uint8_t *p) {
  uint64_t v = 0;
  for (int i = 7; i >= 0; --i) v = (v << 8) | p[i];
  return v;
}
static uint32_t le32(const uint8_t *p) {
  return (uint32_t)p[0] | ((uint32_t)p[1] << 8) | ((uint32_t)p[2] << 16) | ((uint32_t)p[3] << 24);
}
static uint64_t rotl64(uint64_t x, int r) { return (x << r) | (x >> (64 - r)); }
static uint64_t bswap64(uint64_t x) {
  uint64_t r = 0;
  for (int i = 0; i < 8; ++i) r = (r << 8) | ((x >> (8 * i)) & 0xFF);
  return r;
}

/* the 128-bit product of a and b, its two halves XORed */
static uint64_t mul_fold(uint64_t a, uint64_t b) {
  unsigned __int128 p = (unsigned __int128)a * b;
  return (uint64_t)p ^ (uint64_t)(p >> 64);
}

static uint64_t xxh64_avalanche(uint64_t h) {
  h ^= h >> 33;
  h *= XXH_P64_2;
  h ^= h >> 29;
  h *= XXH_P64_3;
  h ^= h >> 32;
  return h;
}
static uint64_t xxh3_avalanche(uint64_t h) {
  h ^= h >> 37;
  h *= XXH_MX1;
  h ^= h >> 32;
  return h;
}
static uint64_t xxh3_rrmxmx(uint64_t h, uint64_t len) {
  h ^= rotl64(h, 49) ^ rotl64(h, 24);
  h *= XXH_MX2;
  h ^= (h >> 35) + len;
  h *= XXH_MX2;
  h ^= h >> 28;
  return h;
}

/* 16 input bytes against 16 secret bytes (seed 0) */
static uint64_t mix16(const uint8_t *in, const uint8_t *sec) {
  return mul_fold(le64(in) ^ le64(sec), le64(in + 8) ^ le64(sec + 8));
}

/* one 64-byte stripe into the 8 accumulators */
static void accumulate_stripe(uint64_t acc[8], const uint8_t *in, const uint8_t *sec) {
  for (int i = 0; i < 8; ++i) {
    uint64_t v = le64(in + 8 * i);
    uint64_t k = v ^ le64(sec + 8 * i);
    acc[i ^ 1] += v;
    acc[i] += (uint64_t)(uint32_t)k * (k >> 32);
  }
}
static void scramble(uint64_t acc[8], const uint8_t *sec) {
  for (int i = 0; i < 8; ++i) {
    uint64_t a = acc[i];
    a ^= a >> 47;
    a ^= le64(sec + 8 * i);
    a *= XXH_P32_1;
    acc[i] = a;
  }
}

ORACLE_EXPORT uint64_t oracle_xxh3_64_secret(const uint8_t *in, uint64_t len, const uint8_t *sec,
                                             uint64_t sec_len) {
  if (len == 0) return xxh64_avalanche(le64(sec + 56) ^ le64(sec + 64));
  if (len <= 3) {
    uint32_t c1 = in[0], c2 = in[len >> 1], c3 = in[len - 1];
    uint32_t combined = (c1 << 16) | (c2 << 24) | c3 | ((uint32_t)len << 8);
    uint64_t bitflip = (uint64_t)(le32(sec) ^ le32(sec + 4));
    return xxh64_avalanche((uint64_t)combined ^ bitflip);
  }
  if (len <= 8) {
    uint64_t bitflip = le64(sec + 8) ^ le64(sec + 16);
    uint64_t v = (uint64_t)le32(in + len - 4) + ((uint64_t)le32(in) << 32);
    return xxh3_rrmxmx(v ^ bitflip, len);
  }
  if (len <= 16) {
    uint64_t lo = le64(in) ^ (le64(sec + 24) ^ le64(sec + 32));
    uint64_t hi = le64(in + len - 8) ^ (le64(sec + 40) ^ le64(sec + 48));
    uint64_t acc = len + bswap64(lo) + hi + mul_fold(lo, hi);
    return xxh3_avalanche(acc);
  }
  if (len <= 128) {
    uint64_t acc = len * XXH_P64_1;
    /* pairs of 16-byte pieces from both ends, the outer pairs first in the
       secret: (0, len-16), (16, len-32), (32, len-48), (48, len-64) */
    int pairs = len > 96 ? 4 : len > 64 ? 3 : len > 32 ? 2 : 1;
    for (int j = pairs - 1; j >= 0; --j) {
      acc += mix16(in + 16 * j, sec + 32 * j);
      acc += mix16(in + len - 16 * (j + 1), sec + 32 * j + 16);
    }
    return xxh3_avalanche(acc);
  }
  if (len <= 240) {
    uint64_t acc = len * XXH_P64_1;
    uint64_t rounds = len / 16;
    for (uint64_t i = 0; i < 8; ++i) acc += mix16(in + 16 * i, sec + 16 * i);
    acc = xxh3_avalanche(acc);
    for (uint64_t i = 8; i < rounds; ++i) acc += mix16(in + 16 * i, sec + 16 * (i - 8) + 3);
    acc += mix16(in + len - 16, sec + 136 - 17);
    return xxh3_avalanche(acc);
  }
  /* longer inputs: 8 accumulators over 64-byte stripes; the secret advances
     8 bytes per stripe, and after (sec_len - 64) / 8 stripes (a block) the
     accumulators are scrambled with the secret's last 64 bytes */
  uint64_t acc[8] = {XXH_P32_3, XXH_P64_1, XXH_P64_2, XXH_P64_3, XXH_P64_4, XXH_P32_2, XXH_P64_5, XXH_P32_1};
  uint64_t stripes_per_block = (sec_len - 64) / 8;
  uint64_t block_len = 64 * stripes_per_block;
  uint64_t n_blocks = (len - 1) / block_len;
  for (uint64_t b = 0; b < n_blocks; ++b) {
    for (uint64_t s = 0; s < stripes_per_block; ++s) accumulate_stripe(acc, in + b * block_len + 64 * s, sec + 8 * s);
    scramble(acc, sec + sec_len - 64);
  }
  uint64_t last_stripes = ((len - 1) - block_len * n_blocks) / 64;
  for (uint64_t s = 0; s < last_stripes; ++s) accumulate_stripe(acc, in + n_blocks * block_len + 64 * s, sec + 8 * s);
  accumulate_stripe(acc, in + len - 64, sec + sec_len - 64 - 7);
  uint64_t h = len * XXH_P64_1;
  for (int i = 0; i < 4; ++i) h += mul_fold(acc[2 * i] ^ le64(sec + 11 + 16 * i), acc[2 * i + 1] ^ le64(sec + 11 + 16 * i + 8));
  return xxh3_avalanche(h);
}

/* ------------------------------------------------------------------ */
/* HCT v2 container: validation and metadata   [R] Phase 6.1          */
/* ------------------------------------------------------------------ */
/* [R] Phase 6.1 asks for a v2 header with XXH3 checksums, compression and
 * quantization metadata and the block size, such that a flipped byte is
 * reported as a checksum mismatch. The page leaves the header undesigned;
 * the layout read here (all fields little-endian) is:
 *
 *   0  "HCT2"          4  version (u16) = 2   6  reserved (u16) = 0
 *   8  compression u8: 0 none, 1 LZ4 raw blocks
 *   9  quantization u8: 0 none (fp16), 1 INT4, 2 INT8
 *   10 checksum u8: 1 XXH3-64        11 reserved u8 = 0
 *   12 block_size u32 (decompressed bytes per block)
 *   16 rows u64   24 cols u64   32 group_size u32   36 secret_len u32
 *   40 n_blocks u64   48 payload_bytes u64   56 meta_hash u64
 *   64 the XXH3 secret (secret_len >= 136 bytes)
 *   then, each section starting at a multiple of 16 bytes (zero padding):
 *   block offsets u64[n_blocks + 1] (relative to the payload; offsets[0] =
 *   0, offsets[n_blocks] = payload_bytes, non-decreasing), block hashes
 *   u64[n_blocks], scales fp16[n_groups], zero points u8[n_groups], and the
 *   payload (the compressed blocks) last, ending the container.
 *   n_groups = rows * cols / group_size for INT4, rows for INT8, 0 for none.
 *
 * meta_hash is XXH3-64 (with the container's secret) of every byte before
 * the payload with the meta_hash field read as zero; block hash b is
 * XXH3-64 of the payload bytes [offsets[b], offsets[b + 1]). Together they
 * cover every byte. */

enum { HCT_OK = 0, HCT_BAD_HEADER = 1, HCT_TRUNCATED = 2, HCT_META_MISMATCH = 3, HCT_BLOCK_MISMATCH = 4 };

static uint64_t round16(uint64_t x) { return (x + 15) & ~(uint64_t)15; }

/* section offsets of a container; 0 if the header is not a v2 header */
typedef struct {
  uint64_t offsets_at, hashes_at, scales_at, zeros_at, payload_at, end;
} hct_layout;

static int hct_parse(const uint8_t *buf, uint64_t len, hct_layout *L, uint64_t meta[12]) {
  if (len < 64 || memcmp(buf, "HCT2", 4) != 0) return HCT_BAD_HEADER;
  uint32_t version = (uint32_t)buf[4] | ((uint32_t)buf[5] << 8);
  uint32_t compression = buf[8], quantization = buf[9], checksum = buf[10];
  uint32_t block_size = le32(buf + 12), group_size = le32(buf + 32), secret_len = le32(buf + 36);
  uint64_t rows = le64(buf + 16), cols = le64(buf + 24), n_blocks = le64(buf + 40), payload = le64(buf + 48);
  if (version != 2 || compression > 1 || quantization > 2 || checksum != 1 || secret_len < 136) return HCT_BAD_HEADER;
  if (block_size == 0 || n_blocks > (1ull << 40)) return HCT_BAD_HEADER;
  if (cols != 0 && rows > (1ull << 50) / cols) return HCT_BAD_HEADER; /* at most 2^50 elements */
  uint64_t n = rows * cols, n_groups = 0;
  if (quantization == 1) {
    if (group_size == 0 || cols % group_size != 0) return HCT_BAD_HEADER;
    n_groups = n / group_size;
  } else if (quantization == 2) {
    n_groups = rows;
  }
  uint64_t at = round16(64 + (uint64_t)secret_len);
  L->offsets_at = at;
  at = round16(at + 8 * (n_blocks + 1));
  L->hashes_at = at;
  at = round16(at + 8 * n_blocks);
  L->scales_at = at;
  at = round16(at + 2 * n_groups);
  L->zeros_at = at;
  at = round16(at + (quantization == 1 ? n_groups : 0));
  L->payload_at = at;
  L->end = at + payload;
  if (L->end < at || L->end != len) return HCT_TRUNCATED;
  if (meta) {
    uint64_t m[12] = {version, compression, quantization, checksum, block_size, rows,
                      cols,    group_size,  secret_len,   n_blocks, payload,    n_groups};
    memcpy(meta, m, sizeof m);
  }
  return HCT_OK;
}

/* Status of a container: HCT_OK, or the first failure in the order header,
 * size, meta_hash, block hashes (the first mismatching block in *bad_block),
 * with offsets out of order counted as a meta failure. */
ORACLE_EXPORT int oracle_hct2_validate(const uint8_t *buf, uint64_t len, uint64_t *bad_block) {
  hct_layout L;
  int st = hct_parse(buf, len, &L, NULL);
  if (st) return st;
  uint32_t secret_len = le32(buf + 36);
  const uint8_t *secret = buf + 64;
  uint64_t n_blocks = le64(buf + 40), payload = le64(buf + 48);

  uint8_t *meta = (uint8_t *)malloc(L.payload_at ? L.payload_at : 1);
  if (!meta) return HCT_BAD_HEADER;
  memcpy(meta, buf, L.payload_at);
  memset(meta + 56, 0, 8);
  uint64_t h = oracle_xxh3_64_secret(meta, L.payload_at, secret, secret_len);
  free(meta);
  if (h != le64(buf + 56)) return HCT_META_MISMATCH;

  const uint8_t *offs = buf + L.offsets_at;
  if (le64(offs) != 0 || le64(offs + 8 * n_blocks) != payload) return HCT_META_MISMATCH;
  for (uint64_t b = 0; b < n_blocks; ++b)
    if (le64(offs + 8 * (b + 1)) < le64(offs + 8 * b)) return HCT_META_MISMATCH;
  for (uint64_t b = 0; b < n_blocks; ++b) {
    uint64_t s0 = le64(offs + 8 * b), s1 = le64(offs + 8 * (b + 1));
    uint64_t hb = oracle_xxh3_64_secret(buf + L.payload_at + s0, s1 - s0, secret, secret_len);
    if (hb != le64(buf + L.hashes_at + 8 * b)) {
      if (bad_block) *bad_block = b;
      return HCT_BLOCK_MISMATCH;
    }
  }
  return HCT_OK;
}

/* The header's fields (version, compression, quantization, checksum,
 * block_size, rows, cols, group_size, secret_len, n_blocks, payload_bytes,
 * n_groups) and the byte offsets of the sections (offsets, hashes, scales,
 * zeros, payload, end); no checksum is checked. */
ORACLE_EXPORT int oracle_hct2_meta(const uint8_t *buf, uint64_t len, uint64_t meta[12], uint64_t sections[6]) {
  hct_layout L;
  int st = hct_parse(buf, len, &L, meta);
  if (st) return st;
  uint64_t s[6] = {L.offsets_at, L.hashes_at, L.scales_at, L.zeros_at, L.payload_at, L.end};
  memcpy(sections, s, sizeof s);
  return HCT_OK;
}

/* ------------------------------------------------------------------ */
/* Decode -> matrix multiply   [R] Phase 4.1, [L] decode + GEMM        */
/* ------------------------------------------------------------------ */
/* [R] Phase 4.1 (test_tensor_usable_in_matmul) multiplies an input by a
 * decoded weight tensor, input.matmul(weights); [L] lists "decode + GEMM"
 * benchmarks (decompress, then multiply). Two plain steps: W = the INT4
 * dequant of oracle_dequant_int4 as a [K, N] matrix (rows = K, cols = N,
 * groups along each row), then out[m, n] = sum over k of x[m, k] * W[k, n]
 * with x a row-major [M, K] binary16 matrix. Products of two binary16
 * values are exact in double, and the sum is taken in double in order of
 * k; absum[m, n] = sum of |x[m, k] * W[k, n]| bounds the rounding error
 * of any other summation order. */
ORACLE_EXPORT int oracle_int4_matmul(const uint16_t *x, int64_t M, const uint8_t *packed, const uint16_t *scales,
                                     const uint8_t *zeros, int64_t K, int64_t N, int64_t group_size, double *out,
                                     double *absum) {
  if (M < 0 || K < 0 || N < 0) return ORACLE_INVALID;
  uint16_t *w = (uint16_t *)malloc((size_t)(K * N > 0 ? K * N : 1) * sizeof(uint16_t));
  double *wd = (double *)malloc((size_t)(K * N > 0 ? K * N : 1) * sizeof(double));
  double *xd = (double *)malloc((size_t)(M * K > 0 ? M * K : 1) * sizeof(double));
  if (!w || !wd || !xd) {
    free(w);
    free(wd);
    free(xd);
    return ORACLE_INVALID;
  }
  int st = oracle_dequant_int4(packed, scales, zeros, K, N, group_size, w);
  if (st == ORACLE_OK) {
    for (int64_t i = 0; i < K * N; ++i) wd[i] = oracle_f16_to_f64(w[i]);
    for (int64_t i = 0; i < M * K; ++i) xd[i] = oracle_f16_to_f64(x[i]);
    for (int64_t m = 0; m < M; ++m) {
      for (int64_t n = 0; n < N; ++n) {
        double s = 0.0, a = 0.0;
        for (int64_t k = 0; k < K; ++k) {
          double p = xd[m * K + k] * wd[k * N + n];
          s += p;
          a += fabs(p);
        }
        out[m * N + n] = s;
        if (absum) absum[m * N + n] = a;
      }
    }
  }
  free(w);
  free(wd);
  free(xd);
  return st;
}
