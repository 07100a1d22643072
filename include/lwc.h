/*
 * lwc.h — C ABI of liblwc: lossless compression of BF16 weight tensors and
 * their decompression to bit-exact BF16 in GPU memory (NVIDIA B200, sm_100a).
 *
 * Two codecs, both lossless:
 *
 *  - DFloat11-style ("Koniec z kompromisami! DFloat11 ratuje dokładność
 *    modeli AI, czyli kompresja, na którą czekałem", section "Przełom:
 *    DFloat11 – bezstratna kompresja z wydajnością GPU"): each BF16 weight is
 *    split into its 8-bit exponent, which is Huffman coded per tensor, and one
 *    raw byte holding its sign and 7 mantissa bits. About 10.6–11 bits/weight.
 *    The decoder is the GPU kernel of section "Jak to działa w praktyce? Magia
 *    na poziomie GPU" of the same page: small linked lookup tables in shared
 *    memory, two phases (threads count their codes, a block scan gives each
 *    thread its output position, threads decode again and write), and one
 *    launch for all matrices of a transformer block.
 *
 *  - Codebook ("Codebook Lossless Compression: когда 25% памяти значат
 *    больше, чем кажется", section "Как работает эта магия?"; and
 *    "無損 LLM 壓縮減少 10-25% RAM", key points): the table of the tensor's U
 *    distinct 16-bit patterns plus ceil(log2 U)-bit packed indices, decoded by
 *    table lookup.
 *
 * Memory and ownership
 *  - The host encoders malloc the blob; release it with lwc_free. (The
 *    device encoders below write into caller-owned device memory instead.)
 *  - The caller copies the blob, byte for byte, to a device buffer it owns
 *    (d_in) and keeps the lwc_desc (a plain struct in host memory).
 *  - Decoders run asynchronously on the caller's CUDA stream and write n
 *    BF16 values (2n bytes) to the caller's device buffer d_out_bf16
 *    (for DFloat11 blobs of another element type: n elements of that type,
 *    4n bytes for FP32).
 *    They allocate no memory (host or device) and never synchronise.
 *  - d_in and d_out_bf16 must be 16-byte aligned (else LWC_ERR_MISALIGNED).
 *
 * Errors
 *  - Return values report synchronous checks: arguments, descriptor
 *    consistency, and cudaGetLastError() after the launch (LWC_ERR_CUDA).
 *    lwc_last_error() gives a message for the calling thread's last failure.
 *  - Corrupt device data (a damaged blob whose header is still valid) cannot
 *    make a decoder read or write outside its buffers or hang; the affected
 *    outputs are unspecified and, in the *_checked variants, a bit is OR-ed
 *    into the caller's device status word (LWC_DEVICE_* below). The library
 *    never traps or asserts on the device.
 *
 * Thread safety: all entry points may be called concurrently from several
 * host threads (the decoders keep only per-device launch configuration,
 * set once under a lock).
 */
#ifndef LWC_H
#define LWC_H

#include <stdint.h>

#if defined(__GNUC__)
#define LWC_API __attribute__((visibility("default")))
#else
#define LWC_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t; NULL means the legacy default stream. */
typedef struct CUstream_st *lwc_stream_t;

typedef enum lwc_status {
    LWC_OK = 0,
    LWC_ERR_INVALID_ARG = 1,  /* NULL pointer, bad size or parameter */
    LWC_ERR_MISALIGNED = 2,   /* device pointer not 16-byte aligned */
    LWC_ERR_CORRUPT = 3,      /* blob header/descriptor inconsistent */
    LWC_ERR_UNSUPPORTED = 4,  /* valid but outside what this library decodes */
    LWC_ERR_NOMEM = 5,        /* host allocation failed (encoders) */
    LWC_ERR_CUDA = 6          /* CUDA runtime error at launch */
} lwc_status;

enum {
    LWC_CODEC_DFLOAT11 = 1,
    LWC_CODEC_CODEBOOK = 2
};

/* Element types of a DFloat11 blob (lwc_desc.elem). The DFloat11 idea --
 * entropy-code the exponent, keep sign and mantissa raw -- carried from BF16
 * to the other float formats. Each element becomes a 16-bit pattern laid out
 * like BF16 (sign, exponent field, 7 mantissa bits), coded as a BF16 tensor,
 * plus the mantissa bits that do not fit, kept raw in the "lo" section:
 *   FP32: the top 16 bits are a BF16 pattern; low 16 bits raw (uint16[n]).
 *   FP16: sign | 5-bit exponent | top 7 mantissa bits; the low 3 mantissa
 *         bits packed 3 per weight, least significant bits first.
 * Decoders write n elements of the blob's type (4 bytes each for FP32). */
enum {
    LWC_ELEM_BF16 = 0,
    LWC_ELEM_FP32 = 1,
    LWC_ELEM_FP16 = 2
};

/* Bits OR-ed into the optional device status word by the decoders. */
enum {
    LWC_DEVICE_BAD_COUNT = 1u,   /* a block decoded a different number of codes than blkoff says */
    LWC_DEVICE_BAD_CODE = 2u,    /* a lookup-table path that no valid code takes */
    LWC_DEVICE_BAD_OFFSET = 4u,  /* blkoff out of order, past n, or above max_block_count */
    LWC_DEVICE_TIMEOUT = 8u      /* a bounded wait on an asynchronous copy gave up */
};

/* Descriptor of one compressed tensor: a host-side copy of the blob header
 * (layout of the blob itself: 256-byte little-endian header, then sections at
 * 16-byte aligned offsets; see the field comments). Plain data, owned by the
 * caller; fill it with an encoder or with lwc_desc_from_blob. */
typedef struct lwc_desc {
    uint32_t magic;            /* 0x3143574C */
    uint32_t version;          /* 1 */
    uint32_t codec;            /* LWC_CODEC_* */
    uint32_t flags;            /* DFloat11: bit 0 one exponent value only;
                                  bit 1 per-chunk code counts stored (off_counts) */
    uint64_t n;                /* number of weights */
    uint64_t total_bytes;      /* blob size */
    /* DFloat11 */
    uint32_t chunk_bytes;      /* bitstream bytes per chunk = per decoding thread */
    uint32_t threads_per_block;/* chunks per block = threads per CUDA block */
    uint32_t max_len;          /* longest code length (<= 32) */
    uint32_t n_tables;         /* 256-entry lookup tables */
    uint64_t n_chunks;
    uint64_t n_blocks;
    uint64_t total_bits;       /* Huffman bitstream length */
    uint32_t max_block_count;  /* most weights decoded by one block */
    uint32_t const_exp;        /* exponent when flags bit 0 is set */
    uint64_t off_lengths;      /* u8[256] code length per exponent value */
    uint64_t off_lut;          /* u16[n_tables][256] */
    uint64_t off_gaps;         /* u8[n_blocks * threads_per_block] */
    uint64_t off_blkoff;       /* u64[n_blocks + 1] */
    uint64_t off_stream;       /* u32 words, MSB-first codes */
    uint64_t stream_bytes;
    uint64_t off_sm;           /* u8[n] sign|mantissa bytes */
    /* codebook */
    uint32_t U;                /* table entries */
    uint32_t k;                /* index bits = ceil(log2 U) */
    uint64_t off_table;        /* u16[U], ascending */
    uint64_t off_packed;       /* k-bit indices, LSB first */
    uint64_t packed_bytes;
    /* DFloat11 element type (header bytes 136..159; zero in BF16 blobs) */
    uint32_t elem;             /* LWC_ELEM_* */
    uint32_t reserved;
    uint64_t off_lo;           /* raw low mantissa bits (FP32, FP16) */
    uint64_t lo_bytes;
    /* DFloat11, flags bit 1 (header bytes 160..167; zero otherwise):
     * u8[n_blocks * threads_per_block], the number of codes that start in
     * each chunk -- what the first phase of the two-phase decoder (DF11
     * page, section "Jak to działa w praktyce?") counts, stored by the
     * encoder so that a decoder can go straight to the scan and the writes.
     * Chunks past the stream end count 0. */
    uint64_t off_counts;
} lwc_desc;

/* DFloat11 encoder parameters; pass NULL for the defaults
 * (chunk_bytes 36, threads_per_block 32, max_len 32, chunk_counts 1).
 * chunk_bytes: multiple of 4 in [8, 1024]; threads_per_block: multiple of 32
 * in [32, 1024]; max_len: code length limit in [9, 32]; chunk_counts: 1 =
 * store the per-chunk code counts (flags bit 1) whenever every count fits in
 * a byte, which the code guarantees when ceil(8 chunk_bytes / shortest code
 * length) <= 255 (with 36-byte chunks: no 1-bit code); 0 = never. Blobs with
 * the counts decode faster; both kinds decode to the same tensor. */
typedef struct lwc_df11_params {
    uint32_t chunk_bytes;
    uint32_t threads_per_block;
    uint32_t max_len;
    uint32_t chunk_counts;
} lwc_df11_params;

/* ---- host encoders -------------------------------------------------------- */

/* Compress n BF16 bit patterns (h_src, host memory, read only) with the
 * DFloat11 codec. On LWC_OK, *h_blob_out is a malloc'ed blob of
 * *blob_bytes_out bytes (release with lwc_free) and *desc_out describes it.
 * n = 0 gives a header-only blob. Fails only on bad arguments or
 * LWC_ERR_NOMEM. */
LWC_API lwc_status lwc_encode_dfloat11(const uint16_t *h_src, uint64_t n, const lwc_df11_params *params,
                               lwc_desc *desc_out, void **h_blob_out, uint64_t *blob_bytes_out);

/* DFloat11 compression of n elements of type `elem` (LWC_ELEM_*): h_src
 * holds uint32 patterns for FP32, uint16 patterns for FP16 and BF16 (BF16 is
 * exactly lwc_encode_dfloat11). Same ownership and errors; LWC_ERR_INVALID_ARG
 * for an unknown element type. Not part of the pages' method, which is
 * defined for BF16. */
LWC_API lwc_status lwc_encode_dfloat11_elements(const void *h_src, uint64_t n, uint32_t elem,
                                                const lwc_df11_params *params, lwc_desc *desc_out,
                                                void **h_blob_out, uint64_t *blob_bytes_out);

/* Compress n BF16 bit patterns with the codebook codec (table of the U
 * distinct patterns in ascending order + k = ceil(log2 U)-bit indices).
 * Same ownership and errors as lwc_encode_dfloat11. */
LWC_API lwc_status lwc_encode_codebook(const uint16_t *h_src, uint64_t n,
                               lwc_desc *desc_out, void **h_blob_out, uint64_t *blob_bytes_out);

/* Release a blob returned by an encoder (NULL is ignored). */
LWC_API void lwc_free(void *h_blob);

/* Parse and check the header of a blob held in host memory (h_blob, bytes
 * long) into *desc_out. LWC_ERR_CORRUPT if the header is inconsistent with
 * itself or with `bytes`. */
LWC_API lwc_status lwc_desc_from_blob(const void *h_blob, uint64_t bytes, lwc_desc *desc_out);

/* ---- device decoders (asynchronous on `stream`) --------------------------- */

/* Decode a DFloat11 blob: d_in = the blob in device memory (16-byte aligned),
 * d_out_bf16 = n outputs (2n bytes, 16-byte aligned). */
LWC_API lwc_status lwc_decode_dfloat11(const lwc_desc *desc, const void *d_in, uint16_t *d_out_bf16,
                               lwc_stream_t stream);

/* Decode a codebook blob; arguments as lwc_decode_dfloat11. */
LWC_API lwc_status lwc_decode_codebook(const lwc_desc *desc, const void *d_in, uint16_t *d_out_bf16,
                               lwc_stream_t stream);

/* As above, plus d_status: a device uint32 the caller owns (and zeroes); the
 * decoder ORs LWC_DEVICE_* bits into it when it meets corrupt data. NULL is
 * allowed. */
LWC_API lwc_status lwc_decode_dfloat11_checked(const lwc_desc *desc, const void *d_in, uint16_t *d_out_bf16,
                                       uint32_t *d_status, lwc_stream_t stream);
LWC_API lwc_status lwc_decode_codebook_checked(const lwc_desc *desc, const void *d_in, uint16_t *d_out_bf16,
                                       uint32_t *d_status, lwc_stream_t stream);

/* Decode `count` DFloat11 tensors — e.g. all matrices of one transformer
 * block (DF11 page, section "Jak to działa w praktyce?", third pillar) — in
 * as few launches as possible (one per distinct (chunk_bytes,
 * threads_per_block) pair among them, plus one for tensors with a single
 * exponent value). descs[i], d_ins[i], d_outs[i] as for lwc_decode_dfloat11;
 * d_status optional. */
LWC_API lwc_status lwc_decode_dfloat11_batched(const lwc_desc *descs, const void *const *d_ins,
                                       uint16_t *const *d_outs, int count, uint32_t *d_status,
                                       lwc_stream_t stream);

/* Decode `count` codebook tensors in as few launches as possible (one per
 * distinct index width k among them, plus one fill per single-entry table).
 * Arguments as lwc_decode_dfloat11_batched. */
LWC_API lwc_status lwc_decode_codebook_batched(const lwc_desc *descs, const void *const *d_ins,
                                               uint16_t *const *d_outs, int count, uint32_t *d_status,
                                               lwc_stream_t stream);

/* ---- decode fused into the linear layer that consumes the weights --------- */

/* y = x W^T without writing W out: the decoded weights stay in registers.
 * The DF11 page ("Koniec z kompromisami! DFloat11 ratuje dokładność modeli
 * AI ...", section "Jak to działa w praktyce? Magia na poziomie GPU") has the
 * weights decompressed on the GPU during inference for the model's use, and
 * measures token-generation throughput (section "Realne korzyści, które
 * zmieniają zasady gry"); token generation runs the linear layers on a few
 * activation rows, where the product is bound by reading the weights.
 *
 *   y[m * rows + r] = sum over c < cols of W[r * cols + c] * x[m * cols + c]
 *
 * for m < M, r < rows = n / cols, W the n weights the blob decodes to (BF16),
 * read as rows x cols row-major (out_features x in_features).
 *   - d_blob: the blob in device memory, 16-byte aligned (not modified).
 *   - cols: 1 .. 2^31 - 1, and n must be a multiple of it.
 *   - d_x: M x cols BF16 activations, row-major, 16-byte aligned (not modified).
 *   - M: 1 .. 8.
 *   - d_y: M x rows FP32 outputs, 4-byte aligned; every output is written
 *     (overwritten, not accumulated into). The caller owns all buffers.
 *   - d_status: optional, as for the checked decoders.
 * Products of two BF16 values are exact in FP32; the sums are FP32, and
 * every output is a summation tree of height at most h, so that
 * |y - exact| <= gamma_h * sum |W x|, gamma_h = h u / (1 - h u), u = 2^-24:
 *   codebook: h = ceil(cols / 1024) + 37 (ceil(cols / 32) + 5 for a
 *     one-entry table); the result does not depend on the launch shape;
 *   DFloat11: h = ceil(cols / 512) + ceil(cols / 32) + 32 when cols is a
 *     multiple of 16, else h = cols; blocks that share an output row add
 *     their parts atomically, so the last bits may vary from run to run.
 * Errors as for the decoders (LWC_ERR_INVALID_ARG for a bad M or cols). */
LWC_API lwc_status lwc_linear_codebook(const lwc_desc *desc, const void *d_blob, uint64_t cols, const uint16_t *d_x,
                                       int M, float *d_y, uint32_t *d_status, lwc_stream_t stream);

/* `count` codebook tensors, each with its own cols[i], activations d_xs[i]
 * and outputs d_ys[i] (all with the same M), in one launch per index width. */
LWC_API lwc_status lwc_linear_codebook_batched(const lwc_desc *descs, const void *const *d_blobs,
                                               const uint64_t *cols, const uint16_t *const *d_xs, int M,
                                               float *const *d_ys, int count, uint32_t *d_status,
                                               lwc_stream_t stream);

/* As lwc_linear_codebook, for a DFloat11 blob of BF16 elements whose blocks
 * hold 32 chunks (threads_per_block = 32, the encoder's default), or with a
 * single exponent value; other blobs give LWC_ERR_UNSUPPORTED (re-encode). */
LWC_API lwc_status lwc_linear_dfloat11(const lwc_desc *desc, const void *d_blob, uint64_t cols, const uint16_t *d_x,
                                       int M, float *d_y, uint32_t *d_status, lwc_stream_t stream);

/* `count` DFloat11 tensors as lwc_linear_codebook_batched, in one launch per
 * distinct chunk_bytes (at most 16 tensors each), after zeroing the outputs. */
LWC_API lwc_status lwc_linear_dfloat11_batched(const lwc_desc *descs, const void *const *d_blobs,
                                               const uint64_t *cols, const uint16_t *const *d_xs, int M,
                                               float *const *d_ys, int count, uint32_t *d_status,
                                               lwc_stream_t stream);

/* ---- decode fused into a tensor-core matrix product ------------------------ */

/* Tile order: the order in which lwc_gemm_dfloat11 expects a matrix's
 * weights. W (rows x cols, row-major, rows % 128 == 0, cols % 64 == 0) is cut
 * into 128 x 64 tiles; tile (i, j) holds rows 128 i .. 128 i + 127 and
 * columns 64 j .. 64 j + 63; tiles follow each other by i, then j, and each
 * tile is row-major. Writes that order of d_src (rows x cols BF16 on the
 * device) to d_dst (same size, not overlapping); both 16-byte aligned. Encode
 * the result with any DFloat11 encoder to get a blob for lwc_gemm_dfloat11
 * (its plain decode then yields the tile order, not the source order).
 * LWC_ERR_INVALID_ARG for other shapes, NULL or equal pointers. */
LWC_API lwc_status lwc_tile_order(const uint16_t *d_src, uint64_t rows, uint64_t cols, uint16_t *d_dst,
                                  lwc_stream_t stream);

/* y = x W^T on the tensor cores (tcgen05, sm_100 only), with W decoded from
 * a DFloat11 blob straight into shared-memory operand tiles; the BF16 matrix
 * is never written to device memory. This is the decompression the DFloat11
 * page places just before a layer's use ("Koniec z kompromisami! DFloat11
 * ratuje dokładność modeli AI ...", section "Jak to działa w praktyce? Magia
 * na poziomie GPU"), fused with the layer for batches of 1 to 256 rows.
 *   - desc / d_blob: a DFloat11 blob of BF16 weights in tile order (see
 *     lwc_tile_order), blocks of 32 chunks, stored chunk counts (the
 *     encoder's defaults) and more than one exponent value; else
 *     LWC_ERR_UNSUPPORTED. d_blob 16-byte aligned.
 *   - cols: W's columns (a multiple of 64, at most 2^24); rows = n / cols
 *     must be a multiple of 128 (at most 2^20); else LWC_ERR_INVALID_ARG.
 *   - d_x: M x cols BF16 activations, row-major, 16-byte aligned.
 *   - M: 1 .. 256.
 *   - d_y: M x rows FP32 outputs (row-major), 4-byte aligned; every output
 *     is written (not accumulated into). The caller owns all buffers.
 *   - d_status: optional, as for the checked decoders; on a nonzero status
 *     d_y is undefined.
 * Products of two BF16 values are exact in FP32; the tensor cores add them
 * into an FP32 accumulator in steps of 16, in an order and with an internal
 * rounding the hardware fixes: |y - exact| <= gamma_cols * sum |W x| with
 * gamma_k = k u / (1 - k u) and u = 2^-23 (twice FP32's unit roundoff, to
 * cover truncating internal additions). Results repeat bit for bit from run
 * to run. */
LWC_API lwc_status lwc_gemm_dfloat11(const lwc_desc *desc, const void *d_blob, uint64_t cols, const uint16_t *d_x,
                                     int M, float *d_y, uint32_t *d_status, lwc_stream_t stream);

/* `count` (at most 8) such matrices in one launch, each with its own cols[i],
 * activations d_xs[i] and outputs d_ys[i], all with the same M and
 * chunk_bytes; at most 4096 units of 128 rows in all. */
LWC_API lwc_status lwc_gemm_dfloat11_batched(const lwc_desc *descs, const void *const *d_blobs,
                                             const uint64_t *cols, const uint16_t *const *d_xs, int M,
                                             float *const *d_ys, int count, uint32_t *d_status,
                                             lwc_stream_t stream);

/* As lwc_gemm_dfloat11, for a codebook blob of tile-ordered weights (codebook
 * page: "Codebook Lossless Compression: когда 25% памяти значат больше, чем
 * кажется", section "Как работает эта магия?": out[i] = table[index i]):
 * each 1024-index run of a tile's packed indices is copied, unpacked and
 * looked up into the shared-memory operand. Index widths k = 1..16 (a
 * one-entry table, k = 0, gives LWC_ERR_UNSUPPORTED); at k = 16 the 128 KB
 * table may leave no room for larger M (LWC_ERR_UNSUPPORTED). Same bound and
 * repeatability as lwc_gemm_dfloat11. */
LWC_API lwc_status lwc_gemm_codebook(const lwc_desc *desc, const void *d_blob, uint64_t cols, const uint16_t *d_x,
                                     int M, float *d_y, uint32_t *d_status, lwc_stream_t stream);

/* `count` (at most 8) codebook matrices with one index width in one launch. */
LWC_API lwc_status lwc_gemm_codebook_batched(const lwc_desc *descs, const void *const *d_blobs,
                                             const uint64_t *cols, const uint16_t *const *d_xs, int M,
                                             float *const *d_ys, int count, uint32_t *d_status,
                                             lwc_stream_t stream);

/* ---- device encoders ------------------------------------------------------ */

/* Compression of a tensor that is already in GPU memory, into a blob in GPU
 * memory. The blob is byte-for-byte the one the host encoder makes from the
 * same weights and parameters. The codebook page ("Codebook Lossless
 * Compression: когда 25% памяти значат больше, чем кажется", trade-offs)
 * notes that building the dictionary and index map lengthens model loading;
 * these entry points keep every pass over the weights on the GPU and leave
 * only the code construction (from a 256-bin histogram or a 65536-bit
 * presence map) to the host.
 *
 * Two calls per tensor, sharing one device workspace the caller owns
 * (lwc_encode_device_workspace_bytes(n) bytes, 256-byte aligned):
 *   1. *_device_plan reads d_src (n BF16 patterns, device, 16-byte aligned)
 *      and fills *desc_out; desc_out->total_bytes is the blob size to
 *      allocate. (max_block_count is still 0 here.)
 *   2. lwc_encode_device_write reads d_src again and writes the blob to d_blob
 *      (device, 16-byte aligned, at least total_bytes long); *desc_out then
 *      holds the final descriptor, equal to the blob's header.
 * d_src must hold the same weights in both calls (else LWC_ERR_INVALID_ARG,
 * with nothing written outside d_blob's total_bytes); the workspace must not
 * be used by another encode in between. Work is issued on `stream`, after
 * whatever the caller has queued there, and both calls synchronise `stream`
 * before returning (the host needs the histogram, and the blob is complete on
 * return). They allocate nothing. Limit: n <= 2^36. */
LWC_API uint64_t lwc_encode_device_workspace_bytes(uint64_t n);

/* Plan a DFloat11 blob (params as for lwc_encode_dfloat11; NULL = defaults). */
LWC_API lwc_status lwc_encode_dfloat11_device_plan(const void *d_src, uint64_t n, const lwc_df11_params *params,
                                                   void *d_work, uint64_t work_bytes, lwc_desc *desc_out,
                                                   lwc_stream_t stream);

/* Plan a DFloat11 blob of n elements of type `elem` (LWC_ELEM_*; d_src holds
 * uint32 patterns for FP32, uint16 otherwise); lwc_encode_device_write then
 * writes the same bytes lwc_encode_dfloat11_elements makes on the host.
 * lwc_encode_dfloat11_device_plan is this with LWC_ELEM_BF16. */
LWC_API lwc_status lwc_encode_dfloat11_elements_device_plan(const void *d_src, uint64_t n, uint32_t elem,
                                                            const lwc_df11_params *params, void *d_work,
                                                            uint64_t work_bytes, lwc_desc *desc_out,
                                                            lwc_stream_t stream);

/* Plan a codebook blob. */
LWC_API lwc_status lwc_encode_codebook_device_plan(const void *d_src, uint64_t n, void *d_work,
                                                   uint64_t work_bytes, lwc_desc *desc_out, lwc_stream_t stream);

/* Write the blob the workspace's plan describes (either codec). */
LWC_API lwc_status lwc_encode_device_write(const void *d_src, uint64_t n, void *d_work, uint64_t work_bytes,
                                           void *d_blob, uint64_t blob_bytes, lwc_desc *desc_out,
                                           lwc_stream_t stream);

/* DFloat11 device encode that allocates nothing, for callers that cannot
 * call cudaMalloc when they compress a tensor: e.g. a serving process whose
 * memory manager has reserved the device memory for weights and KV cache up
 * front and permits no further cudaMalloc/cudaFree (a late cudaMalloc can
 * fail or fragment that pool; cudaFree synchronises the whole device).
 * The pages have no counterpart to this entry point.
 *
 * Does lwc_encode_dfloat11_device_plan + lwc_encode_device_write in one call,
 * with a fixed scratch array inside the library (3,154,432 bytes of device
 * memory, created when the library's device code is loaded on a GPU and
 * held by every GPU that loads it until the process exits) in place of the
 * caller's workspace. It calls no cudaMalloc or cudaFree and no allocating
 * library routine.
 *   - n must be <= 2^30 weights (the scratch's limit; every matrix of
 *     Llama-3-8B and -70B fits), else LWC_ERR_UNSUPPORTED before any device
 *     work.
 *   - d_src, d_blob, params, *desc_out and the stream behave as for the
 *     two-call device encoder; if blob_bytes is below the blob's size the
 *     call fails with LWC_ERR_INVALID_ARG and *desc_out holds the plan, whose
 *     total_bytes is the size needed.
 *   - The first call on a device (per process) looks up the scratch array's
 *     device address for that device (cudaGetSymbolAddress, with that device
 *     current).
 *   - Every call on a device shares the one scratch array, which keeps the
 *     last call's contents (each call clears what must start at zero). Calls
 *     whose GPU work overlaps — from several host threads, or on several
 *     streams of one device — race on it and give wrong blobs: serialise
 *     them. */
LWC_API lwc_status lwc_encode_dfloat11_device_noalloc(const void *d_src, uint64_t n, const lwc_df11_params *params,
                                                      void *d_blob, uint64_t blob_bytes, lwc_desc *desc_out,
                                                      lwc_stream_t stream);

/* Self-test of the bounded wait every kernel above uses on its asynchronous
 * copies (failure detection without a GPU fault): one thread waits, for at
 * most `polls` (1 .. 2^24) polls, on a shared-memory mbarrier phase that
 * completes only if `arrive` is non-zero (the thread's own arrival). A wait
 * that gives up ORs LWC_DEVICE_TIMEOUT into *d_status (device, 4-byte
 * aligned, owned and zeroed by the caller) and the kernel returns normally,
 * so the context stays usable. No copy, trap or fault is involved. */
LWC_API lwc_status lwc_selftest_bounded_wait(uint32_t *d_status, uint32_t polls, int arrive, lwc_stream_t stream);

/* ---- helpers -------------------------------------------------------------- */

/* Static string naming a status code. */
LWC_API const char *lwc_status_string(lwc_status s);

/* Message describing the calling thread's last failed call ("" if none). */
LWC_API const char *lwc_last_error(void);

/* Library version as 10000*major + 100*minor + patch. */
LWC_API int lwc_version(void);

#ifdef __cplusplus
}
#endif

#endif /* LWC_H */
