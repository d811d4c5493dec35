// lt_hct.cpp -- HCT v2 container header: layout, parse and write, on the
// host ("GPU Compression Pipeline - TDD Roadmap", Phase 6.1 HCT Format V2:
// a v2 header carrying compression, quantization and block size, with XXH3
// checksums). The page lists the header as a task without designing it; the
// byte layout is this library's and is documented with lt_hct2_header.
#include <string.h>

#include "lt_decode.h"

#define LT_API extern "C" __attribute__((visibility("default")))

namespace {

uint64_t r16(uint64_t x) { return (x + 15) & ~(uint64_t)15; }

uint64_t get(const uint8_t *p, int n) {
  uint64_t v = 0;
  for (int i = n - 1; i >= 0; --i) v = (v << 8) | p[i];
  return v;
}

void put(uint8_t *p, uint64_t v, int n) {
  for (int i = 0; i < n; ++i) p[i] = (uint8_t)(v >> (8 * i));
}

}  // namespace

LT_API lt_status lt_hct2_layout(lt_hct2_header *h) {
  if (!h) return LT_ERR_INVALID_ARG;
  if (h->version != LT_HCT2_VERSION || h->compression > 1 || h->quantization > 2 || h->checksum != 1 ||
      h->secret_len < LT_HCT2_SECRET_MIN)
    return LT_ERR_INVALID_ARG;
  if (h->block_size == 0 || h->n_blocks > (1ull << 40)) return LT_ERR_INVALID_ARG;
  if (h->cols != 0 && h->rows > (1ull << 50) / h->cols) return LT_ERR_INVALID_ARG;
  uint64_t n_groups = 0;
  if (h->quantization == 1) {
    if (h->group_size == 0 || h->cols % h->group_size != 0) return LT_ERR_INVALID_ARG;
    n_groups = h->rows * h->cols / h->group_size;
  } else if (h->quantization == 2) {
    n_groups = h->rows;
  }
  h->n_groups = n_groups;
  uint64_t at = r16(LT_HCT2_HEADER_BYTES + (uint64_t)h->secret_len);
  h->offsets_at = at;
  at = r16(at + 8 * (h->n_blocks + 1));
  h->hashes_at = at;
  at = r16(at + 8 * h->n_blocks);
  h->scales_at = at;
  at = r16(at + 2 * n_groups);
  h->zeros_at = at;
  at = r16(at + (h->quantization == 1 ? n_groups : 0));
  h->payload_at = at;
  if (h->payload_bytes > UINT64_MAX - at) return LT_ERR_INVALID_ARG;
  h->total_bytes = at + h->payload_bytes;
  return LT_OK;
}

LT_API lt_status lt_hct2_read_header(const uint8_t *buf, uint64_t buf_bytes, lt_hct2_header *h) {
  if (!buf || !h) return LT_ERR_INVALID_ARG;
  if (buf_bytes < LT_HCT2_HEADER_BYTES || memcmp(buf, "HCT2", 4) != 0) return LT_ERR_INVALID_ARG;
  lt_hct2_header r;
  memset(&r, 0, sizeof r);
  r.version = (uint16_t)get(buf + 4, 2);
  r.compression = buf[8];
  r.quantization = buf[9];
  r.checksum = buf[10];
  r.block_size = (uint32_t)get(buf + 12, 4);
  r.rows = get(buf + 16, 8);
  r.cols = get(buf + 24, 8);
  r.group_size = (uint32_t)get(buf + 32, 4);
  r.secret_len = (uint32_t)get(buf + 36, 4);
  r.n_blocks = get(buf + 40, 8);
  r.payload_bytes = get(buf + 48, 8);
  r.meta_hash = get(buf + 56, 8);
  const lt_status st = lt_hct2_layout(&r);
  if (st != LT_OK) return st;
  if (r.total_bytes != buf_bytes) return LT_ERR_SIZE_MISMATCH;
  *h = r;
  return LT_OK;
}

LT_API lt_status lt_hct2_write_header(const lt_hct2_header *h, uint8_t *out) {
  if (!h || !out) return LT_ERR_INVALID_ARG;
  lt_hct2_header r = *h;
  const lt_status st = lt_hct2_layout(&r);
  if (st != LT_OK) return st;
  memset(out, 0, LT_HCT2_HEADER_BYTES);
  memcpy(out, "HCT2", 4);
  put(out + 4, r.version, 2);
  out[8] = r.compression;
  out[9] = r.quantization;
  out[10] = r.checksum;
  put(out + 12, r.block_size, 4);
  put(out + 16, r.rows, 8);
  put(out + 24, r.cols, 8);
  put(out + 32, r.group_size, 4);
  put(out + 36, r.secret_len, 4);
  put(out + 40, r.n_blocks, 8);
  put(out + 48, r.payload_bytes, 8);
  put(out + 56, r.meta_hash, 8);
  return LT_OK;
}
