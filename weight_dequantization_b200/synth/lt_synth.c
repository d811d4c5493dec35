/*
 * lt_synth.c -- seeded synthetic inputs for the compressed-tensor decode path.
 *
 * This module makes the *inputs* of the decoders: random codes, scales and
 * zero points drawn from the value laws of the workloads, the INT4 packing of
 * codes into bytes, an LZ4 block-format compressor and a zero-run encoder.
 * It holds no decoding arithmetic: it never dequantizes, never parses an LZ4
 * or zero-run stream, and shares no code with either the CUDA library or the
 * CPU oracle. Both of those only consume what it writes.
 *
 * Random numbers: xoshiro256** (Blackman & Vigna, "Scrambled linear
 * pseudorandom number generators", 2018) seeded through SplitMix64
 * (Steele, Lea & Flood, "Fast splittable pseudorandom number generators",
 * 2014). Every independent unit (a span of codes, a row, a block) draws from
 * its own substream keyed by (seed, stream id, unit index), so the output is
 * the same whatever the number of threads. Normals use the Box-Muller
 * transform (cosine branch only) on top of libm.
 *
 * fp16 rounding of drawn values uses the compiler's _Float16 conversion
 * (IEEE round-to-nearest-even).
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#include <unistd.h>

#define SYNTH_EXPORT __attribute__((visibility("default")))

/* ------------------------------------------------------------------ */
/* PRNG                                                                */
/* ------------------------------------------------------------------ */

static inline uint64_t splitmix64_next(uint64_t *x) {
  uint64_t z = (*x += 0x9E3779B97F4A7C15ull);
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

typedef struct {
  uint64_t s[4];
} xo256;

static inline uint64_t rotl64(uint64_t x, int k) { return (x << k) | (x >> (64 - k)); }

/* Substream for (seed, stream, unit): SplitMix64 walks from a key that mixes
 * all three through SplitMix64 itself, then fills the xoshiro state. */
static void xo_seed(xo256 *g, uint64_t seed, uint64_t stream, uint64_t unit) {
  uint64_t k = seed;
  uint64_t a = splitmix64_next(&k);
  k = a ^ (stream * 0xD1B54A32D192ED03ull);
  uint64_t b = splitmix64_next(&k);
  k = b ^ (unit * 0xAEF17502108EF2D9ull);
  for (int i = 0; i < 4; ++i) g->s[i] = splitmix64_next(&k);
  if ((g->s[0] | g->s[1] | g->s[2] | g->s[3]) == 0) g->s[0] = 1;
}

static inline uint64_t xo_next(xo256 *g) {
  uint64_t *s = g->s;
  const uint64_t result = rotl64(s[1] * 5, 7) * 9;
  const uint64_t t = s[1] << 17;
  s[2] ^= s[0];
  s[3] ^= s[1];
  s[1] ^= s[2];
  s[0] ^= s[3];
  s[2] ^= t;
  s[3] = rotl64(s[3], 45);
  return result;
}

/* uniform double in [0, 1) with 53 random bits */
static inline double xo_u01(xo256 *g) { return (double)(xo_next(g) >> 11) * 0x1.0p-53; }

/* standard normal, Box-Muller (cosine branch) */
static inline double xo_normal(xo256 *g) {
  double u1 = 1.0 - xo_u01(g); /* (0, 1] */
  double u2 = xo_u01(g);
  return sqrt(-2.0 * log(u1)) * cos(6.283185307179586 * u2);
}

/* geometric on {1, 2, ...} with success probability p (mean 1/p) */
static inline int64_t xo_geometric(xo256 *g, double p) {
  double u = 1.0 - xo_u01(g); /* (0, 1] */
  double k = floor(log(u) / log1p(-p)) + 1.0;
  if (k < 1.0) k = 1.0;
  if (k > 1e15) k = 1e15;
  return (int64_t)k;
}

static inline uint16_t f16_bits(double v) {
  _Float16 h = (_Float16)v;
  uint16_t b;
  memcpy(&b, &h, 2);
  return b;
}

/* ------------------------------------------------------------------ */
/* Parallel-for over independent units                                 */
/* ------------------------------------------------------------------ */

typedef void (*unit_fn)(void *ctx, int64_t unit);

typedef struct {
  unit_fn fn;
  void *ctx;
  int64_t n_units;
  int64_t next;
  pthread_mutex_t mu;
} pfor_state;

static void *pfor_worker(void *arg) {
  pfor_state *st = (pfor_state *)arg;
  for (;;) {
    pthread_mutex_lock(&st->mu);
    int64_t u = st->next++;
    pthread_mutex_unlock(&st->mu);
    if (u >= st->n_units) break;
    st->fn(st->ctx, u);
  }
  return NULL;
}

static int g_threads = 0; /* 0 = all online cores */

SYNTH_EXPORT void synth_set_threads(int n) { g_threads = n; }

static void parallel_for(int64_t n_units, unit_fn fn, void *ctx) {
  int nt = g_threads > 0 ? g_threads : (int)sysconf(_SC_NPROCESSORS_ONLN);
  if (nt < 1) nt = 1;
  if (nt > 256) nt = 256;
  if ((int64_t)nt > n_units) nt = (int)(n_units > 0 ? n_units : 1);
  pfor_state st = {fn, ctx, n_units, 0, PTHREAD_MUTEX_INITIALIZER};
  if (nt == 1) {
    for (int64_t u = 0; u < n_units; ++u) fn(ctx, u);
    return;
  }
  pthread_t th[256];
  for (int i = 0; i < nt; ++i) pthread_create(&th[i], NULL, pfor_worker, &st);
  for (int i = 0; i < nt; ++i) pthread_join(th[i], NULL);
}

/* ------------------------------------------------------------------ */
/* Value laws                                                          */
/* ------------------------------------------------------------------ */

/* Codes are generated in spans of SPAN codes, one substream per span. */
#define SPAN 131072

typedef struct {
  uint64_t seed, stream;
  int64_t n;
  uint8_t *packed;
} int4_uniform_ctx;

static void int4_uniform_unit(void *c, int64_t u) {
  int4_uniform_ctx *x = (int4_uniform_ctx *)c;
  xo256 g;
  xo_seed(&g, x->seed, x->stream, (uint64_t)u);
  int64_t k0 = u * SPAN, k1 = k0 + SPAN;
  if (k1 > x->n) k1 = x->n;
  for (int64_t k = k0; k < k1; ++k) {
    uint8_t q = (uint8_t)(xo_next(&g) >> 60);
    if ((k & 1) == 0)
      x->packed[k >> 1] = q; /* even code: low nibble */
    else
      x->packed[k >> 1] |= (uint8_t)(q << 4); /* odd code: high nibble */
  }
}

/* n codes uniform on {0..15}, packed two per byte, even code in the low
 * nibble. packed must hold ceil(n/2) bytes. */
SYNTH_EXPORT void synth_int4_uniform(uint64_t seed, uint64_t stream, int64_t n, uint8_t *packed) {
  int4_uniform_ctx c = {seed, stream, n, packed};
  parallel_for((n + SPAN - 1) / SPAN, int4_uniform_unit, &c);
}

typedef struct {
  uint64_t seed, stream;
  int64_t n;
  int32_t group;
  double p_const;
  uint32_t cdf[16]; /* P(code <= c) * 2^32 (saturating), c = 0..14; cdf[15] unused */
  uint8_t *packed;
} int4_gauss_ctx;

/* clip(round(N(mu, sigma)), 0, 15) has P(code <= c) = Phi((c + 0.5 - mu) / sigma)
 * for c < 15 (rounding ties have probability zero). Sampling by inverting
 * this CDF with a 32-bit uniform draws exactly that law (to 2^-32). */
static void gauss_code_cdf(double mu, double sigma, uint32_t cdf[16]) {
  for (int c = 0; c < 16; ++c) {
    double p = (c == 15) ? 1.0 : 0.5 * erfc(-((c + 0.5 - mu) / sigma) / sqrt(2.0));
    double v = p * 4294967296.0;
    cdf[c] = v >= 4294967295.0 ? 0xFFFFFFFFu : (uint32_t)v;
  }
}

static inline uint8_t gauss_code(uint32_t u, const uint32_t cdf[16]) {
  uint8_t c = 0;
  while (c < 15 && u >= cdf[c]) ++c;
  return c;
}

static void int4_gauss_unit(void *c, int64_t u) {
  int4_gauss_ctx *x = (int4_gauss_ctx *)c;
  xo256 g;
  xo_seed(&g, x->seed, x->stream, (uint64_t)u);
  int64_t k0 = u * SPAN, k1 = k0 + SPAN;
  if (k1 > x->n) k1 = x->n;
  int64_t k = k0;
  while (k < k1) {
    /* one value-law group starts here (groups are aligned to multiples of
     * `group` codes; SPAN is a multiple of every group size allowed) */
    int64_t gend = (k / x->group + 1) * x->group;
    if (gend > k1) gend = k1;
    uint64_t r = xo_next(&g);
    int is_const = (double)(r >> 11) * 0x1.0p-53 < x->p_const;
    uint8_t cval = gauss_code((uint32_t)xo_next(&g), x->cdf);
    uint64_t bits = 0;
    int avail = 0;
    for (; k < gend; ++k) {
      uint8_t q = cval;
      if (!is_const) {
        if (avail == 0) {
          bits = xo_next(&g);
          avail = 2;
        }
        q = gauss_code((uint32_t)bits, x->cdf);
        bits >>= 32;
        --avail;
      }
      if ((k & 1) == 0)
        x->packed[k >> 1] = q;
      else
        x->packed[k >> 1] |= (uint8_t)(q << 4);
    }
  }
}

/* n codes ~ clip(round(N(mu, sigma)), 0, 15); each aligned run of `group`
 * codes is, with probability p_const, one repeated draw. Packed as above. */
SYNTH_EXPORT void synth_int4_gauss_groups(uint64_t seed, uint64_t stream, int64_t n, int32_t group,
                                          double p_const, double mu, double sigma, uint8_t *packed) {
  int4_gauss_ctx c;
  c.seed = seed;
  c.stream = stream;
  c.n = n;
  c.group = group;
  c.p_const = p_const;
  c.packed = packed;
  gauss_code_cdf(mu, sigma, c.cdf);
  parallel_for((n + SPAN - 1) / SPAN, int4_gauss_unit, &c);
}

typedef struct {
  uint64_t seed, stream;
  int64_t n;
  double lo, hi;
  void *out;
  int kind; /* 0: fp16 uniform, 1: u8 uniform int, 2: int8 normal */
} simple_ctx;

static void simple_unit(void *c, int64_t u) {
  simple_ctx *x = (simple_ctx *)c;
  xo256 g;
  xo_seed(&g, x->seed, x->stream, (uint64_t)u);
  int64_t k0 = u * SPAN, k1 = k0 + SPAN;
  if (k1 > x->n) k1 = x->n;
  for (int64_t k = k0; k < k1; ++k) {
    if (x->kind == 0) {
      double v = x->lo + (x->hi - x->lo) * xo_u01(&g);
      ((uint16_t *)x->out)[k] = f16_bits(v);
    } else if (x->kind == 1) {
      int64_t span = (int64_t)x->hi - (int64_t)x->lo + 1;
      ((uint8_t *)x->out)[k] = (uint8_t)((int64_t)x->lo + (int64_t)(xo_u01(&g) * (double)span));
    } else {
      double v = nearbyint(x->hi * xo_normal(&g)); /* hi carries sigma */
      if (v < -128) v = -128;
      if (v > 127) v = 127;
      ((int8_t *)x->out)[k] = (int8_t)v;
    }
  }
}

/* n fp16 bit patterns, fp16_rn(U[lo, hi]) */
SYNTH_EXPORT void synth_fp16_uniform(uint64_t seed, uint64_t stream, int64_t n, double lo, double hi,
                                     uint16_t *out) {
  simple_ctx c = {seed, stream, n, lo, hi, out, 0};
  parallel_for((n + SPAN - 1) / SPAN, simple_unit, &c);
}

/* n bytes uniform on the integers {lo..hi} */
SYNTH_EXPORT void synth_u8_uniform(uint64_t seed, uint64_t stream, int64_t n, int32_t lo, int32_t hi,
                                   uint8_t *out) {
  simple_ctx c = {seed, stream, n, (double)lo, (double)hi, out, 1};
  parallel_for((n + SPAN - 1) / SPAN, simple_unit, &c);
}

/* n int8 values clip(round(N(0, sigma)), -128, 127) */
SYNTH_EXPORT void synth_int8_normal(uint64_t seed, uint64_t stream, int64_t n, double sigma, int8_t *out) {
  simple_ctx c = {seed, stream, n, 0.0, sigma, out, 2};
  parallel_for((n + SPAN - 1) / SPAN, simple_unit, &c);
}

/* ReLU-like activations: alternating runs over the flat tensor. Zero runs
 * have lengths ~ Geometric(1/mean_zero_run), non-zero runs ~ Geometric(p_nz);
 * the first run is a zero run with probability p_first_zero. Non-zeros are
 * fp16_rn(|N(0,1)|), redrawn while they round to +0. The run process is
 * restarted (fresh substream, fresh first-run draw) every `restart`
 * elements so that spans can be generated in parallel. */
typedef struct {
  uint64_t seed, stream;
  int64_t n, restart;
  double mean_zero_run, p_nz, p_first_zero;
  uint16_t *out;
} relu_ctx;

static void relu_unit(void *c, int64_t u) {
  relu_ctx *x = (relu_ctx *)c;
  xo256 g;
  xo_seed(&g, x->seed, x->stream, (uint64_t)u);
  int64_t k = u * x->restart, k1 = k + x->restart;
  if (k1 > x->n) k1 = x->n;
  int zero = xo_u01(&g) < x->p_first_zero;
  while (k < k1) {
    int64_t len = zero ? xo_geometric(&g, 1.0 / x->mean_zero_run) : xo_geometric(&g, x->p_nz);
    if (len > k1 - k) len = k1 - k;
    for (int64_t i = 0; i < len; ++i) {
      if (zero) {
        x->out[k + i] = 0;
      } else {
        uint16_t b;
        do {
          b = f16_bits(fabs(xo_normal(&g)));
        } while (b == 0);
        x->out[k + i] = b;
      }
    }
    k += len;
    zero = !zero;
  }
}

SYNTH_EXPORT void synth_relu_runs(uint64_t seed, uint64_t stream, int64_t n, double mean_zero_run,
                                  double p_nz, double p_first_zero, int64_t restart, uint16_t *out) {
  if (restart <= 0) restart = n > 0 ? n : 1;
  relu_ctx c = {seed, stream, n, restart, mean_zero_run, p_nz, p_first_zero, out};
  parallel_for((n + restart - 1) / restart, relu_unit, &c);
}

/* ------------------------------------------------------------------ */
/* LZ4 block-format compressor                                         */
/* ------------------------------------------------------------------ */
/*
 * Written from the public LZ4 block format: a block is a run of sequences;
 * a sequence is a token (high nibble = literal count, low nibble = match
 * length - 4, each nibble 15 meaning "more length bytes follow, each adding
 * its value, stopping after the first byte below 255"), the literals, a
 * two-byte little-endian back offset and the match-length extension. The
 * last sequence carries literals only. End-of-block rules the encoder
 * keeps: the last 5 bytes are literals and no match starts within the last
 * 12 bytes.
 *
 * Matcher: greedy, single 4096-entry hash table of 4-byte prefixes, no
 * backward extension, no lazy matching. Any valid encoding decodes to the
 * same bytes; this one is simple and deterministic.
 */

#define LZ4_MINMATCH 4
#define LZ4_LASTLITERALS 5
#define LZ4_MFLIMIT 12
#define LZ4_HASH_LOG 12

static inline uint32_t rd32(const uint8_t *p) {
  uint32_t v;
  memcpy(&v, p, 4);
  return v;
}

static inline uint32_t lz4_hash(uint32_t v) { return (v * 2654435761u) >> (32 - LZ4_HASH_LOG); }

static uint8_t *put_len(uint8_t *op, int64_t len) {
  /* length extension bytes after a nibble of 15 */
  while (len >= 255) {
    *op++ = 255;
    len -= 255;
  }
  *op++ = (uint8_t)len;
  return op;
}

static uint8_t *emit_seq(uint8_t *op, const uint8_t *lit, int64_t nlit, int64_t off, int64_t mlen) {
  uint8_t *tok = op++;
  uint8_t t = 0;
  if (nlit >= 15) {
    t = 15 << 4;
    op = put_len(op, nlit - 15);
  } else {
    t = (uint8_t)(nlit << 4);
  }
  memcpy(op, lit, (size_t)nlit);
  op += nlit;
  if (mlen > 0) {
    *op++ = (uint8_t)(off & 0xFF);
    *op++ = (uint8_t)(off >> 8);
    int64_t m = mlen - LZ4_MINMATCH;
    if (m >= 15) {
      t |= 15;
      op = put_len(op, m - 15);
    } else {
      t |= (uint8_t)m;
    }
  }
  *tok = t;
  return op;
}

/* worst-case compressed size of an n-byte block */
SYNTH_EXPORT int64_t synth_lz4_bound(int64_t n) { return n + n / 255 + 16; }

/* Compress one block; returns the compressed size. dst must hold
 * synth_lz4_bound(n) bytes. If force_literals, emit a single literal-only
 * sequence. */
SYNTH_EXPORT int64_t synth_lz4_compress_block(const uint8_t *src, int64_t n, uint8_t *dst, int force_literals) {
  uint8_t *op = dst;
  int64_t anchor = 0;
  if (!force_literals && n > LZ4_MFLIMIT) {
    uint32_t table[1 << LZ4_HASH_LOG];
    for (int i = 0; i < (1 << LZ4_HASH_LOG); ++i) table[i] = 0xFFFFFFFFu;
    const int64_t match_start_limit = n - LZ4_MFLIMIT; /* last match starts before this */
    const int64_t match_end_limit = n - LZ4_LASTLITERALS;
    int64_t ip = 0;
    while (ip < match_start_limit) {
      uint32_t v = rd32(src + ip);
      uint32_t h = lz4_hash(v);
      uint32_t ref = table[h];
      table[h] = (uint32_t)ip;
      if (ref != 0xFFFFFFFFu && ip - (int64_t)ref <= 65535 && rd32(src + ref) == v) {
        int64_t mlen = LZ4_MINMATCH;
        while (ip + mlen < match_end_limit && src[ref + mlen] == src[ip + mlen]) ++mlen;
        op = emit_seq(op, src + anchor, ip - anchor, ip - (int64_t)ref, mlen);
        /* seed the table inside the match so that later repeats find it */
        if (ip + mlen - 2 > ip) table[lz4_hash(rd32(src + ip + mlen - 2))] = (uint32_t)(ip + mlen - 2);
        ip += mlen;
        anchor = ip;
      } else {
        ++ip;
      }
    }
  }
  op = emit_seq(op, src + anchor, n - anchor, 0, 0);
  return (int64_t)(op - dst);
}

typedef struct {
  const uint8_t *src;
  int64_t src_len;
  int32_t block_bytes;
  uint8_t *tmp;
  int64_t bound;
  int64_t *sizes;
  int force_literals;
} lz4_ctx;

static void lz4_unit(void *c, int64_t b) {
  lz4_ctx *x = (lz4_ctx *)c;
  int64_t s0 = b * (int64_t)x->block_bytes;
  int64_t len = x->src_len - s0;
  if (len > x->block_bytes) len = x->block_bytes;
  x->sizes[b] = synth_lz4_compress_block(x->src + s0, len, x->tmp + b * x->bound, x->force_literals);
}

/* Compress src in independent blocks of block_bytes (last block = the
 * remainder). Writes the concatenated blocks to dst and n_blocks + 1 byte
 * offsets (offsets[0] = 0, offsets[n_blocks] = total). dst must hold
 * n_blocks * synth_lz4_bound(block_bytes) bytes (it is also the scratch).
 * Returns the total compressed size. */
SYNTH_EXPORT int64_t synth_lz4_compress_blocks(const uint8_t *src, int64_t src_len, int32_t block_bytes,
                                               uint8_t *dst, uint64_t *offsets, int force_literals) {
  int64_t n_blocks = (src_len + block_bytes - 1) / block_bytes;
  int64_t bound = synth_lz4_bound(block_bytes);
  int64_t *sizes = (int64_t *)malloc(sizeof(int64_t) * (size_t)(n_blocks > 0 ? n_blocks : 1));
  lz4_ctx c = {src, src_len, block_bytes, dst, bound, sizes, force_literals};
  parallel_for(n_blocks, lz4_unit, &c);
  int64_t pos = 0;
  offsets[0] = 0;
  for (int64_t b = 0; b < n_blocks; ++b) {
    if (b * bound != pos) memmove(dst + pos, dst + b * bound, (size_t)sizes[b]);
    pos += sizes[b];
    offsets[b + 1] = (uint64_t)pos;
  }
  free(sizes);
  return pos;
}

/* ------------------------------------------------------------------ */
/* Zero-run encoder                                                    */
/* ------------------------------------------------------------------ */
/*
 * Chunk stream: records (u16 zero_run, u16 literal_count, literal_count
 * fp16 bit patterns), little-endian, in output order. Canonical form: each
 * record takes the maximal run of +0 (0x0000) bit patterns, then the
 * maximal run of anything else. Each chunk's bytes are padded with zero
 * bytes to a multiple of `pad` (16 for vector loads).
 */

static int64_t zrle_chunk_size(const uint16_t *x, int64_t len) {
  int64_t i = 0, bytes = 0;
  while (i < len) {
    int64_t z = 0;
    while (i < len && x[i] == 0 && z < 65535) ++i, ++z;
    int64_t l = 0;
    while (i < len && x[i] != 0 && l < 65535) ++i, ++l;
    bytes += 4 + 2 * l;
  }
  return bytes;
}

static void zrle_chunk_write(const uint16_t *x, int64_t len, uint8_t *dst) {
  int64_t i = 0;
  uint8_t *op = dst;
  while (i < len) {
    int64_t z = 0;
    while (i < len && x[i] == 0 && z < 65535) ++i, ++z;
    int64_t l0 = i, l = 0;
    while (i < len && x[i] != 0 && l < 65535) ++i, ++l;
    op[0] = (uint8_t)(z & 0xFF);
    op[1] = (uint8_t)(z >> 8);
    op[2] = (uint8_t)(l & 0xFF);
    op[3] = (uint8_t)(l >> 8);
    op += 4;
    memcpy(op, x + l0, (size_t)(2 * l));
    op += 2 * l;
  }
}

typedef struct {
  const uint16_t *x;
  int64_t n;
  int32_t chunk;
  int32_t pad;
  int64_t *sizes;
  uint8_t *dst;
  const uint64_t *offsets;
} zrle_ctx;

static void zrle_size_unit(void *c, int64_t u) {
  zrle_ctx *z = (zrle_ctx *)c;
  int64_t k0 = u * z->chunk, len = z->n - k0;
  if (len > z->chunk) len = z->chunk;
  int64_t b = zrle_chunk_size(z->x + k0, len);
  z->sizes[u] = (b + z->pad - 1) / z->pad * z->pad;
}

static void zrle_write_unit(void *c, int64_t u) {
  zrle_ctx *z = (zrle_ctx *)c;
  int64_t k0 = u * z->chunk, len = z->n - k0;
  if (len > z->chunk) len = z->chunk;
  uint8_t *d = z->dst + z->offsets[u];
  memset(d, 0, (size_t)(z->offsets[u + 1] - z->offsets[u]));
  zrle_chunk_write(z->x + k0, len, d);
}

/* Pass 1: fills offsets[n_chunks + 1] and returns the total encoded size. */
SYNTH_EXPORT int64_t synth_zrle_plan(const uint16_t *x, int64_t n, int32_t chunk, int32_t pad, uint64_t *offsets) {
  if (pad < 1) pad = 1;
  int64_t n_chunks = (n + chunk - 1) / chunk;
  int64_t *sizes = (int64_t *)malloc(sizeof(int64_t) * (size_t)(n_chunks > 0 ? n_chunks : 1));
  zrle_ctx c = {x, n, chunk, pad, sizes, NULL, NULL};
  parallel_for(n_chunks, zrle_size_unit, &c);
  offsets[0] = 0;
  for (int64_t u = 0; u < n_chunks; ++u) offsets[u + 1] = offsets[u] + (uint64_t)sizes[u];
  free(sizes);
  return (int64_t)offsets[n_chunks];
}

/* Pass 2: writes the chunks at the planned offsets. */
SYNTH_EXPORT void synth_zrle_write(const uint16_t *x, int64_t n, int32_t chunk, const uint64_t *offsets,
                                   uint8_t *dst) {
  int64_t n_chunks = (n + chunk - 1) / chunk;
  zrle_ctx c = {x, n, chunk, 1, NULL, dst, offsets};
  parallel_for(n_chunks, zrle_write_unit, &c);
}
