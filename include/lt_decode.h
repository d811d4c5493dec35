/*
 * lt_decode.h -- C ABI of liblt_decode.so: on-device decoding of compressed
 * tensors on NVIDIA B200 (sm_100a).
 *
 * Operations (sources are web pages, cited by title and section):
 *   INT4 group dequantization   "GPU Compression Pipeline - TDD Roadmap",
 *                               Phase 1.1 INT4 Dequantization
 *   INT8 dequantization         same page, Phase 1.2 INT8 Dequantization
 *   zero-run decoding           "LoreToken-powered GPU memory layer",
 *                               compression strategies (zero-run encoding of
 *                               mostly-zero ReLU activations)
 *   fused LZ4 -> INT4 -> fp16   "GPU Compression Pipeline - TDD Roadmap",
 *                               Phase 2.1 LZ4 + INT4 Fused Kernel, with the
 *                               64 KB blocks of Phase 3.1 / Phase 6.1
 *   block checksums             "GPU Compression Pipeline - TDD Roadmap",
 *                               Phase 6.1 HCT Format V2 (XXH3 checksums)
 *   decode -> matrix multiply   "LoreToken-powered GPU memory layer", decode
 *                               + GEMM; "GPU Compression Pipeline - TDD
 *                               Roadmap", Phase 4.1
 *   value-dictionary decoding   "LoreToken-powered GPU memory layer",
 *                               compression strategies (value dictionary
 *                               compression), and the "GPU sidecar brain"
 *                               explanation's strategy list (small integer
 *                               codes plus a tiny lookup table)
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *  - Every data pointer is a DEVICE pointer owned by the caller, except the
 *    descriptor arrays of the LZ4 batch calls (host arrays read during the
 *    call) and the buffers of the lt_hct2_* header functions, which are
 *    host-only and touch no device. The library allocates no memory, frees nothing, never
 *    synchronizes and keeps no pointer after it returns.
 *  - All work is enqueued on `stream` (NULL = the legacy default stream).
 *    A call returns as soon as its kernel is enqueued.
 *  - lt_half is an IEEE 754 binary16 bit pattern (the storage of __half /
 *    torch.float16). lt_half pointers must be 2-byte aligned and
 *    uint64_t pointers 8-byte aligned, else LT_ERR_MISALIGNED. Wider
 *    alignment (16 bytes) of the large buffers selects vectorized kernels;
 *    any other alignment is still decoded correctly, just more slowly.
 *  - Dequantized values are (q - z) * s rounded once to binary16: round to
 *    nearest, ties to even, subnormals kept, overflow to infinity. |q - z|
 *    is at most 255, so the product is exact before that single rounding.
 *  - Host-checkable argument errors are returned synchronously and nothing is
 *    enqueued. Launch failures return LT_ERR_CUDA.
 *  - Data-dependent errors of the stream decoders (a corrupt stream, a
 *    decoded size that differs from the declared one) are asynchronous: if
 *    `d_status` is not NULL the first error code is stored there (the caller
 *    zeroes it beforehand and reads it after synchronizing the stream).
 *    After such an error the output content is unspecified, but every write
 *    stays inside the output buffer. Decoders never trap, assert or loop
 *    unboundedly on corrupt input.
 *  - Sizes of zero are valid and enqueue nothing.
 */
#ifndef LT_DECODE_H_
#define LT_DECODE_H_

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define LT_ABI_VERSION 6

/* Same type as cudaStream_t. */
typedef struct CUstream_st *lt_stream_t;

/* IEEE 754 binary16 bit pattern. */
typedef uint16_t lt_half;

typedef enum {
  LT_OK = 0,
  LT_ERR_INVALID_ARG = 1,    /* NULL pointer with a non-zero size, negative size, bad shape */
  LT_ERR_MISALIGNED = 2,     /* pointer not aligned to its element type */
  LT_ERR_UNSUPPORTED = 3,    /* valid request outside what the kernels implement */
  LT_ERR_CORRUPT_STREAM = 4, /* (device status) malformed LZ4 / zero-run data */
  LT_ERR_SIZE_MISMATCH = 5,  /* (device status) stream decodes to a different length */
  LT_ERR_CUDA = 6,           /* a CUDA launch failed */
  LT_ERR_TIMEOUT = 7,        /* (device status) an internal on-chip wait ran out (lt_int4_gemm) */
  LT_ERR_CHECKSUM = 8        /* (device status) a block's checksum differs from the stored one */
} lt_status;

typedef enum { LT_SCALE_PER_TENSOR = 0, LT_SCALE_PER_ROW = 1 } lt_scale_mode;

/*
 * INT4 group dequantization ("GPU Compression Pipeline - TDD Roadmap",
 * Phase 1.1; block-level, GPTQ/AWQ-style groups).
 *
 *   packed  ceil(rows*cols/2) bytes: code k = rows-major element index k is
 *           the low nibble of byte k/2 when k is even, the high nibble when
 *           odd (the page's example: bytes 0x10,0x32,0x54,0x76 are codes
 *           0..7). An odd element count ignores the last high nibble.
 *   scales  rows*cols/group_size binary16 scales, group g covers codes
 *           [g*group_size, (g+1)*group_size): groups run along each row of a
 *           row-major [rows, cols] tensor and never cross a row.
 *   zeros   one uint8 zero point per group, or NULL for zero point 0.
 *   out     rows*cols binary16 values, out[k] = fp16_rn((q[k] - z[g]) * s[g]).
 *   group_size >= 1 and divides cols, else LT_ERR_INVALID_ARG.
 */
lt_status lt_dequant_int4(const uint8_t *packed, const lt_half *scales, const uint8_t *zeros, int64_t rows,
                          int64_t cols, int32_t group_size, lt_half *out, lt_stream_t stream);

/*
 * INT8 dequantization ("GPU Compression Pipeline - TDD Roadmap", Phase 1.2:
 * "values * scale", per-tensor and per-channel scales).
 *
 *   q           rows*cols int8 values, row-major [rows, cols].
 *   scales      1 binary16 scale (LT_SCALE_PER_TENSOR) or one per row
 *               (LT_SCALE_PER_ROW, the output channel).
 *   zeros       int8 zero points laid out like scales, or NULL for 0.
 *   out         rows*cols binary16, out[r, c] = fp16_rn((q[r, c] - z) * s).
 */
lt_status lt_dequant_int8(const int8_t *q, const lt_half *scales, const int8_t *zeros, int32_t scale_mode,
                          int64_t rows, int64_t cols, lt_half *out, lt_stream_t stream);

/*
 * Zero-run decoding of mostly-zero activations ("LoreToken-powered GPU
 * memory layer", compression strategies: zero-run encoding).
 *
 *   enc, enc_bytes   the encoded stream.
 *   chunk_offsets    n_chunks + 1 byte offsets into enc (uint64, device),
 *                    n_chunks = ceil(n_elements / chunk_elems). Chunk c
 *                    covers elements [c*chunk_elems, min(n, (c+1)*chunk_elems))
 *                    and its bytes are enc[offsets[c], offsets[c+1]).
 *   Chunk bytes: records (u16 zero_run, u16 literal_count, literal_count
 *   binary16 literals), little-endian; each record emits zero_run elements
 *   equal to +0 (0x0000), then the literals bit for bit. Decoding of a chunk
 *   stops once it is full; bytes after that are padding. Offsets may be any
 *   byte position; 16-byte-aligned offsets (the generator pads chunks to 16
 *   bytes) take the fast path.
 *   Device status: LT_ERR_CORRUPT_STREAM if a record overruns its chunk or
 *   its bytes, or an offset pair lies outside enc; LT_ERR_SIZE_MISMATCH if a
 *   chunk's bytes end before the chunk is full.
 *   chunk_elems in [1, 65535], else LT_ERR_UNSUPPORTED.
 */
lt_status lt_zrle_decode(const uint8_t *enc, uint64_t enc_bytes, const uint64_t *chunk_offsets, int64_t n_elements,
                         int32_t chunk_elems, lt_half *out, int32_t *d_status, lt_stream_t stream);

/*
 * Value-dictionary decoding ("LoreToken-powered GPU memory layer",
 * compression strategies: a tensor that holds few distinct values stored as
 * a dictionary plus small indices).
 *
 *   packed  ceil(n*bits/8) bytes of indices: index k is the bits-wide field
 *           that starts at bit k*bits of the byte stream, bit 0 being the
 *           least significant bit of byte 0 (for bits == 4, the nibble
 *           order of lt_dequant_int4: even k in the low nibble). Unused high
 *           bits of the last byte are ignored.
 *   bits    1, 2, 4 or 8, else LT_ERR_INVALID_ARG.
 *   dict    2^bits binary16 entries (one dictionary for the tensor).
 *   out     n binary16 values, out[k] = dict[index k], copied bit for bit
 *           (no arithmetic: -0 and NaN payloads are kept).
 *   A 4-byte-aligned `packed` with a 16-byte-aligned `out` (8-byte for
 *   bits == 8) takes the vectorized kernel.
 */
lt_status lt_value_dict_decode(const uint8_t *packed, int32_t bits, const lt_half *dict, int64_t n, lt_half *out,
                               lt_stream_t stream);

/*
 * Per-block XXH3-64 checksums ("GPU Compression Pipeline - TDD Roadmap",
 * Phase 6.1 HCT Format V2: XXH3 checksums; a flipped byte must be reported
 * as a checksum mismatch).
 *
 *   data, data_bytes  the byte stream (e.g. the LZ4 payload of a container).
 *   offsets           n_blocks + 1 byte offsets into data (uint64, device);
 *                     block b is data[offsets[b], offsets[b+1]).
 *   secret            the XXH3 secret (device), secret_len >= 136 bytes; the
 *                     hash is XXH3-64 (xxHash 0.8) with this secret, seed 0.
 *   hashes            n_blocks uint64 outputs, or NULL.
 *   expected          n_blocks uint64 stored checksums, or NULL. A block
 *                     whose hash differs sets LT_ERR_CHECKSUM in *d_status
 *                     and lowers *d_first_bad (caller-initialised, e.g. to
 *                     UINT64_MAX) to its index.
 *   At least one of hashes / expected, else LT_ERR_INVALID_ARG.
 *   Device status: LT_ERR_CORRUPT_STREAM for an offset pair out of order or
 *   past data_bytes (that block is not hashed).
 */
lt_status lt_xxh3_blocks(const uint8_t *data, uint64_t data_bytes, const uint64_t *offsets, int64_t n_blocks,
                         const uint8_t *secret, int32_t secret_len, uint64_t *hashes, const uint64_t *expected,
                         int32_t *d_status, uint64_t *d_first_bad, lt_stream_t stream);

/*
 * HCT v2 container header ("GPU Compression Pipeline - TDD Roadmap",
 * Phase 6.1 HCT Format V2: compression / quantization metadata, block size
 * and XXH3 checksums; the page leaves the header's design open, so this
 * layout is this library's). HOST functions: buf / out / h are host memory,
 * nothing touches a device.
 *
 * Bytes 0..63, little-endian: "HCT2", version u16 (= 2), reserved u16,
 * compression u8 (0 none, 1 raw LZ4 blocks), quantization u8 (0 none = fp16,
 * 1 INT4, 2 INT8), checksum u8 (1 = XXH3-64), reserved u8, block_size u32,
 * rows u64, cols u64, group_size u32, secret_len u32, n_blocks u64,
 * payload_bytes u64, meta_hash u64. Then the XXH3 secret (secret_len >= 136
 * bytes) and, each from a 16-byte boundary: block offsets u64[n_blocks + 1]
 * (relative to the payload), block hashes u64[n_blocks] (lt_xxh3_blocks of
 * the payload), scales fp16[n_groups], zero points u8[n_groups] (INT4 only),
 * and the payload, which ends the container. n_groups is rows*cols /
 * group_size for INT4, rows for INT8, 0 otherwise. meta_hash is XXH3-64 of
 * every byte before the payload with the meta_hash field read as zero.
 */
#define LT_HCT2_VERSION 2
#define LT_HCT2_HEADER_BYTES 64
#define LT_HCT2_SECRET_MIN 136
typedef struct {
  /* the stored fields */
  uint16_t version;
  uint8_t compression;
  uint8_t quantization;
  uint8_t checksum;
  uint32_t block_size;
  uint64_t rows;
  uint64_t cols;
  uint32_t group_size;
  uint32_t secret_len;
  uint64_t n_blocks;
  uint64_t payload_bytes;
  uint64_t meta_hash;
  /* derived by lt_hct2_layout: group count and byte offsets of the sections */
  uint64_t n_groups;
  uint64_t offsets_at;
  uint64_t hashes_at;
  uint64_t scales_at;
  uint64_t zeros_at;
  uint64_t payload_at;
  uint64_t total_bytes;
} lt_hct2_header;

/* Check the stored fields of *h and fill in the derived ones.
 * LT_ERR_INVALID_ARG for an unknown version, compression, quantization or
 * checksum kind, a secret shorter than 136 bytes, block_size 0, more than
 * 2^40 blocks or 2^50 elements, or an INT4 group size that does not divide
 * cols. */
lt_status lt_hct2_layout(lt_hct2_header *h);

/* Parse the header of a container of buf_bytes bytes (host memory) into *h
 * (stored and derived fields). LT_ERR_INVALID_ARG for a bad magic or fields
 * as in lt_hct2_layout, LT_ERR_SIZE_MISMATCH if the sections do not end at
 * buf_bytes. No checksum is checked here (lt_xxh3_blocks does that). */
lt_status lt_hct2_read_header(const uint8_t *buf, uint64_t buf_bytes, lt_hct2_header *h);

/* Write the 64 header bytes of *h's stored fields to out (host memory),
 * after the checks of lt_hct2_layout. */
lt_status lt_hct2_write_header(const lt_hct2_header *h, uint8_t *out);

/*
 * Workspace of the LZ4 decoders. The serial part of LZ4 -- walking the
 * sequence headers of a block -- runs as a separate pass, one warp per
 * block, that writes a small sequence index (a 16-byte header per block,
 * then 16 bytes per sequence, at most 512 sequences per block) into a
 * caller-provided device workspace; the expansion then runs with the index
 * in hand. lt_lz4_workspace_bytes(n)
 * is the size needed for n blocks in one call (the sum over a batch). A
 * call given NULL or a smaller workspace still decodes correctly, each
 * block walked by the expanding CTA itself (much slower), and so is a block
 * with more than 512 sequences. The workspace must be 16-byte aligned, is
 * owned by the caller, and may be reused by the next call on the same
 * stream; calls that run concurrently need their own.
 */
uint64_t lt_lz4_workspace_bytes(int64_t n_blocks);

/*
 * Fused LZ4 block decompression -> INT4 unpack -> scale -> binary16
 * ("GPU Compression Pipeline - TDD Roadmap", Phase 2.1: decompress
 * directly to dequantized F16 with no intermediate buffer).
 *
 *   comp, comp_bytes   raw LZ4 blocks (block format, no frame), independent
 *                      (no block refers to another).
 *   block_offsets      n_blocks + 1 byte offsets into comp (uint64, device).
 *   block_bytes        decompressed bytes per block, in [16, 65536] and a
 *                      multiple of 16 (65536 in the workloads); the last
 *                      block holds the remainder of ceil(rows*cols/2).
 *                      n_blocks = ceil(ceil(rows*cols/2) / block_bytes).
 *   The decompressed bytes are the `packed` array of lt_dequant_int4, and
 *   scales / zeros / rows / cols / group_size / out mean what they mean
 *   there. Decompressed bytes live only in on-chip shared memory; the
 *   workspace holds the sequence index (see lt_lz4_workspace_bytes).
 *   Device status: LT_ERR_CORRUPT_STREAM for a malformed block (offset 0 or
 *   before the block start, literal or match past the block end, input
 *   overrun, an offset pair outside comp), LT_ERR_SIZE_MISMATCH for a block
 *   that decodes to fewer bytes than it must. A malformed block's output is
 *   left unspecified (possibly unwritten).
 */
lt_status lt_lz4_int4_decode(const uint8_t *comp, uint64_t comp_bytes, const uint64_t *block_offsets,
                             int32_t block_bytes, const lt_half *scales, const uint8_t *zeros, int64_t rows,
                             int64_t cols, int32_t group_size, lt_half *out, void *workspace,
                             uint64_t workspace_bytes, int32_t *d_status, lt_stream_t stream);

/*
 * The fused decode of lt_lz4_int4_decode with each compressed block checked
 * first ("GPU Compression Pipeline - TDD Roadmap", Phase 6.1 HCT Format V2:
 * XXH3 checksums; a flipped byte is reported as a checksum mismatch).
 *
 * Before decoding block b, the kernel computes the XXH3-64 (seed 0, the
 * given secret, as lt_xxh3_blocks) of comp[block_offsets[b],
 * block_offsets[b + 1]) and compares it with expected_hashes[b]. A block
 * that differs is not decoded (its output is left unspecified), sets
 * LT_ERR_CHECKSUM in *d_status (which then takes precedence over any other
 * error of that block) and lowers *d_first_bad (caller-initialised, e.g. to
 * UINT64_MAX; may be NULL) to b. Other blocks decode as in
 * lt_lz4_int4_decode. The hash is computed while the block is read for
 * decoding (one warp of the expanding CTA), so the compressed stream is not
 * read by a separate pass.
 *   secret, secret_len  device, secret_len >= 136; expected_hashes: n_blocks
 *                       uint64 (device, 8-byte aligned). All other arguments
 *                       as lt_lz4_int4_decode.
 */
lt_status lt_lz4_int4_decode_checked(const uint8_t *comp, uint64_t comp_bytes, const uint64_t *block_offsets,
                                     int32_t block_bytes, const lt_half *scales, const uint8_t *zeros, int64_t rows,
                                     int64_t cols, int32_t group_size, lt_half *out, void *workspace,
                                     uint64_t workspace_bytes, const uint8_t *secret, int32_t secret_len,
                                     const uint64_t *expected_hashes, int32_t *d_status, uint64_t *d_first_bad,
                                     lt_stream_t stream);

/*
 * Several fused LZ4 -> INT4 decodes in one launch (the weight matrices of a
 * transformer layer decoded into one reused buffer). Each descriptor has
 * the meaning of the lt_lz4_int4_decode arguments of the same name. The
 * descriptor array itself is a HOST array, read during the call; the
 * workspace covers the blocks of all descriptors together.
 * 1 <= n_desc <= LT_LZ4_BATCH_MAX, else LT_ERR_INVALID_ARG / UNSUPPORTED.
 */
#define LT_LZ4_BATCH_MAX 64
typedef struct {
  const uint8_t *comp;
  uint64_t comp_bytes;
  const uint64_t *block_offsets;
  const lt_half *scales;
  const uint8_t *zeros;
  lt_half *out;
  int64_t rows;
  int64_t cols;
  int32_t group_size;
  int32_t block_bytes;
} lt_lz4_int4_desc;

lt_status lt_lz4_int4_decode_batch(const lt_lz4_int4_desc *descs, int32_t n_desc, void *workspace,
                                   uint64_t workspace_bytes, int32_t *d_status, lt_stream_t stream);

/*
 * The same decode in two steps, so that the serial part -- the walk over
 * each block's sequence headers -- can run over many more blocks in one
 * launch than one decode call covers (e.g. every layer of a model, while
 * the layers are still decoded one at a time into one reused buffer).
 *
 * lt_lz4_index_batch walks every block of descs[0 .. n_desc) and writes its
 * sequence index (and any stream error it finds) to `index`, a device
 * buffer of at least lt_lz4_workspace_bytes(total blocks) bytes laid out
 * like the workspace of the one-step calls. Blocks are numbered across the
 * descriptors in order: descriptor i's block b is block
 * (blocks of descriptors 0 .. i-1) + b, where a descriptor has
 * ceil(ceil(rows*cols/2) / block_bytes) blocks. It writes no output and
 * reports nothing to a status word.
 *
 * lt_lz4_int4_expand_batch decodes descs[0 .. n_desc) -- which must be
 * consecutive descriptors of an earlier lt_lz4_index_batch call, with the
 * same compressed streams, starting at its block `first_block` -- from that
 * index: `index` and `index_bytes` are the buffer given to the index call,
 * `index_blocks` the total block count of that call. Stream errors found by
 * the index call, and errors found now, go to *d_status as in
 * lt_lz4_int4_decode. The index must be complete (the same stream, or an
 * event) and unchanged since. first_block + the descriptors' blocks >
 * index_blocks, or an index buffer too small for index_blocks, returns
 * LT_ERR_INVALID_ARG.
 * 1 <= n_desc <= LT_LZ4_BATCH_MAX for both, else LT_ERR_INVALID_ARG /
 * UNSUPPORTED.
 */
lt_status lt_lz4_index_batch(const lt_lz4_int4_desc *descs, int32_t n_desc, void *index, uint64_t index_bytes,
                             lt_stream_t stream);
lt_status lt_lz4_int4_expand_batch(const lt_lz4_int4_desc *descs, int32_t n_desc, const void *index,
                                   uint64_t index_bytes, int64_t index_blocks, int64_t first_block,
                                   int32_t *d_status, lt_stream_t stream);

/*
 * Plain LZ4 block decompression to bytes (the same decoder as the fused
 * path, writing the decompressed bytes instead of dequantizing them). Used
 * to check the LZ4 stage bit for bit, and as a general decoder.
 *   out        out_bytes bytes; block b fills [b*block_bytes, ...).
 *   block_bytes in [16, 65536], a multiple of 16.
 */
lt_status lt_lz4_decode(const uint8_t *comp, uint64_t comp_bytes, const uint64_t *block_offsets, int32_t block_bytes,
                        uint8_t *out, uint64_t out_bytes, void *workspace, uint64_t workspace_bytes,
                        int32_t *d_status, lt_stream_t stream);

/*
 * The fused decode of lt_lz4_int4_decode for callers that cannot allocate
 * device memory. (No counterpart on the pages: this entry point exists for
 * how the library is called, not for what it computes.)
 *
 * Some callers may not allocate device memory at the time they decode: a
 * plugin running inside an inference engine or server that hands out a fixed
 * device-memory budget at start-up and forbids allocations afterwards, or
 * any code whose device allocator belongs to another component. They cannot
 * provide the workspace the other LZ4 entry points take. This entry point
 * keeps that workspace in a scratch array built into the library instead:
 * every GPU that loads the library holds LT_NOALLOC_MAX_BLOCKS blocks'
 * worth of it (about 4 MiB) until the process exits, and the call itself
 * allocates and frees nothing.
 *
 * Arguments, results and device status are those of lt_lz4_int4_decode,
 * without the workspace. Limits and rules:
 *  - At most LT_NOALLOC_MAX_BLOCKS LZ4 blocks per call
 *    (ceil(ceil(rows*cols/2) / block_bytes)); larger requests return
 *    LT_ERR_UNSUPPORTED and enqueue nothing.
 *  - The first call on each device looks up the scratch array's device
 *    address (cudaGetSymbolAddress) with that device current; make that
 *    first call before any stream capture. A failed lookup returns
 *    LT_ERR_CUDA. The address is kept with the id of the CUDA context it
 *    was taken in: after the context is destroyed and created again (e.g.
 *    cudaDeviceReset), the next call is again a first call in the new
 *    context and looks the address up again.
 *  - All calls on a device share the one scratch array and it keeps the
 *    last call's contents (nothing in it needs to start at zero). Calls whose
 *    work overlaps on the GPU -- on different streams, or from different host
 *    threads -- race on it and may decode wrongly: run them one after
 *    another, e.g. on one stream.
 */
#define LT_NOALLOC_MAX_BLOCKS 512
lt_status lt_lz4_int4_decode_noalloc(const uint8_t *comp, uint64_t comp_bytes, const uint64_t *block_offsets,
                                     int32_t block_bytes, const lt_half *scales, const uint8_t *zeros, int64_t rows,
                                     int64_t cols, int32_t group_size, lt_half *out, int32_t *d_status,
                                     lt_stream_t stream);

/*
 * Fused INT4 decode -> matrix multiply on the tensor cores
 * ("LoreToken-powered GPU memory layer": decode + GEMM, decoded weights
 * feeding a matrix multiply; "GPU Compression Pipeline - TDD Roadmap",
 * Phase 4.1: a decoded weight tensor used in input.matmul(weights)).
 *
 *   out[M, N] = x[M, K] . W[K, N]
 *
 *   x        M x K binary16, row-major (row stride K), 16-byte aligned.
 *   packed, scales, zeros, group_size
 *            W in the layout of lt_dequant_int4 with rows = K, cols = N:
 *            ceil(K*N/2) bytes of codes (16-byte aligned), K*N/group_size
 *            binary16 scales and uint8 zero points (or NULL) laid out
 *            [K, N/group_size]. W[k, n] is exactly lt_dequant_int4's output
 *            element k*N + n; it is never written to memory: each tile is
 *            decoded on chip and fed to the tensor cores (for M > 16 into
 *            shared memory as the B operand of tcgen05.mma; for M <= 16
 *            straight into the registers of mma.sync).
 *   out      M x N binary16, row-major, 16-byte aligned: the fp32 sum of the
 *            exact products x[m, k] * W[k, n] over k, rounded once to
 *            binary16. The order of the fp32 additions is the hardware's
 *            (and, with a split of K, partial sums are added in split
 *            order), so out differs from the exact sum by at most about
 *            K * 2^-23 * sum_k |x[m, k] W[k, n]| plus half an ulp of out.
 *   workspace, workspace_bytes
 *            optional fp32 scratch for splitting K across CTAs when the
 *            output has few tiles (small M): lt_int4_gemm_workspace_bytes
 *            gives the size the call would use (0: no split). NULL or a
 *            smaller workspace computes without splitting (correct, fewer
 *            CTAs). 16-byte aligned, caller-owned, reusable by the next
 *            call on the same stream.
 *   Shapes: M >= 1, K a multiple of 64, N a multiple of 256, group_size a
 *   multiple of 32 that divides N, else LT_ERR_UNSUPPORTED.
 *   Device status: LT_ERR_TIMEOUT if an on-chip wait of the kernel ran out
 *   (an internal error; the output is then unspecified).
 */
uint64_t lt_int4_gemm_workspace_bytes(int64_t M, int64_t N, int64_t K);
lt_status lt_int4_gemm(const lt_half *x, int64_t M, int64_t K, const uint8_t *packed, const lt_half *scales,
                       const uint8_t *zeros, int64_t N, int32_t group_size, lt_half *out, void *workspace,
                       uint64_t workspace_bytes, int32_t *d_status, lt_stream_t stream);

/* Static, human-readable name of a status code. */
const char *lt_status_string(lt_status s);

/* LT_ABI_VERSION of the built library. */
int32_t lt_abi_version(void);

#ifdef __cplusplus
}
#endif

#endif /* LT_DECODE_H_ */
