/*
 * df11.h -- C ABI of the DFloat11 (DF11) codec library, libdf11.so.
 *
 * DF11 stores a BF16 weight as a Huffman code of its 8-bit exponent plus one
 * raw byte holding its sign and 7-bit mantissa, about 11 bits per weight, and
 * rebuilds the exact BF16 bits on the GPU right before the weight is used.
 *
 * Sources (web pages on DFloat11; cited by title and section):
 *  - "DFloat11 : compression sans perte pour l'inference GPU qui reduit les
 *    LLM a 70 % de leur taille" (fr.news.hada.io).  Sections used:
 *      << La marge de compression restante dans l'exposant BFloat16 >>
 *      << Le format DFloat11 >>
 *      << Decompression adaptee a l'inference GPU >>
 *      << Decodage fonde sur des LUT hierarchiques >>
 *      << Noyau GPU en deux etapes et metadonnees auxiliaires >>
 *      << Decompression par bloc transformer >>
 *  - "70% Size, 100% Accuracy: Lossless LLM Compression for Efficient GPU
 *    Inference via Dynamic-Length Float" (chatpaper.ai), abstract.
 *
 * Conventions for every call:
 *  - Plain C types only.  Streams are passed as `void *` holding a
 *    cudaStream_t (NULL = the legacy default stream).
 *  - The caller owns every buffer.  The library never allocates device
 *    memory; host encoding uses a size-then-fill pattern.
 *  - Errors are returned as df11_status; nothing is thrown across the ABI.
 *  - Device calls are asynchronous on the given stream and return launch /
 *    argument errors immediately.  Data corruption found by a kernel is
 *    reported by OR-ing bits into a caller-owned device word (err_word).
 *  - Thread safety: calls share no mutable global state, except the
 *    no-allocation encoder calls, which share one fixed scratch array per
 *    device (see there).
 *  - CUDA graphs: df11_decode, df11_decode_block, df11_decode_gemv and
 *    df11_gemm_bf16 only enqueue work on the given stream (kernels, and a
 *    memset for split-K GEMMs), so they can be captured into a CUDA graph
 *    and replayed.  The first call on a device must come before any capture
 *    (it makes one-time settings), and df11_read_error synchronises the
 *    stream, so it stays outside the graph.
 */
#ifndef DF11_H
#define DF11_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum df11_status {
    DF11_OK = 0,
    DF11_ERR_INVALID_ARG = 1, /* NULL pointer, bad size, bad alignment, bad params */
    DF11_ERR_UNSUPPORTED = 2, /* a parameter value this build does not implement */
    DF11_ERR_TOO_LARGE = 3,   /* more than 2^32 - 1 elements in one stream */
    DF11_ERR_CORRUPT = 4,     /* inconsistent stream / aux data (host checks) */
    DF11_ERR_CUDA = 5,        /* a CUDA runtime call failed */
    DF11_ERR_NOMEM = 6        /* host allocation failed */
} df11_status;

/* Bits a decode kernel ORs into err_word when the data is inconsistent. */
#define DF11_KERR_COUNT_MISMATCH 0x1u /* codes in a thread block != its span  */
#define DF11_KERR_BAD_CODE 0x2u       /* a bit pattern that is no code        */
#define DF11_KERR_BAD_BLOCK 0x4u      /* block_start not monotone / too big   */
#define DF11_KERR_OVERRUN 0x8u        /* a thread's codes run past its end    */
#define DF11_KERR_BAD_ROW 0x40u       /* a requested row index is out of range */

/* Encoder parameters.
 *  max_code_len      -- length cap L_MAX for the exponent code, 1..32.  The
 *                       pages give 32 as the bound implied by 5-bit gaps
 *                       and observe 24..32 in LLMs ("Decodage fonde sur des
 *                       LUT hierarchiques", "Noyau GPU en deux etapes...").
 *                       Default 12: every code then resolves in one table
 *                       lookup, for about 0.004 more bits per weight on
 *                       LLM-like weights than an uncapped code.
 *  bytes_per_thread  -- n, bytes of the exponent stream owned by one decode
 *                       thread.  The pages use n = 8; this build supports 8.
 *  threads_per_block -- T, threads that share one stored output position.
 *                       The pages do not give T; this build supports 256. */
typedef struct df11_params {
    uint32_t max_code_len;
    uint32_t bytes_per_thread;
    uint32_t threads_per_block;
    uint32_t reserved; /* must be 0 */
} df11_params;

/* A compressed tensor (or a whole transformer block encoded with one shared
 * table).  Plain data: the struct never owns the arrays it points to.
 *
 * Format ("Le format DFloat11", "Noyau GPU en deux etapes et metadonnees
 * auxiliaires"), with the readings this library takes where the pages are
 * silent:
 *  enc         EncodedExponent: canonical Huffman codes of the exponents in
 *              element order, packed MSB-first; zero-padded to enc_bytes
 *              = n_blocks * T * n + 16.
 *  sm          PackedSignMantissa: byte i = (sign_i << 7) | mantissa_i;
 *              zero-padded to sm_bytes = round_up(n_elems, 16) + 16.
 *  gaps        Gaps: one 5-bit field per thread (MSB-first, thread order):
 *              bit offset, from the thread's first byte, of the first code
 *              that starts in its n bytes (the end of the stream counts as
 *              a start).  n_blocks * T fields, zero-padded to gaps_bytes.
 *  block_start u32 per thread block: index of the first element decoded by
 *              that block, plus a final entry equal to n_elems; zero-padded
 *              to block_start_bytes = round_up(4 * (n_blocks + 1), 16) + 16.
 *  counts      OPTIONAL per-thread code counts, one byte per thread: how
 *              many codes start in the thread's n bytes (0..64; threads past
 *              the stream 0), n_blocks * T bytes, zero-padded to
 *              counts_bytes = n_blocks * T + 16.  This is the number the
 *              first pass of the two-step kernel finds ("Noyau GPU en deux
 *              etapes et metadonnees auxiliaires"); stored, it lets the
 *              decoder skip that pass (one decoding pass, then the block
 *              prefix sum of the stored counts).  It is derived data: the
 *              encoders write it when counts is non-NULL, and a decode with
 *              counts == NULL runs the two passes of the pages.
 *  lut         decode tables derived from code_len (layout private to the
 *              library, lut_bytes long): a multi-code LUT on the first W
 *              bits of a window, a code-count LUT, and canonical limits for
 *              codes longer than W bits.
 *  code_len    the table: code length of every exponent value (0 = absent).
 *              Codes are canonical: ordered by (length, exponent value).
 *  max_block_codes  the largest block_start[b + 1] - block_start[b]; the
 *              decoder picks its on-chip buffer size from it (a block whose
 *              span exceeds the buffer is reported as DF11_KERR_BAD_BLOCK).
 *
 * For the encode calls the pointers are HOST arrays the caller allocated
 * with the *_bytes sizes returned by the size call (counts may be NULL:
 * not written).  For the decode calls they are DEVICE arrays holding the
 * same bytes, each 16-byte aligned (counts may be NULL). */
typedef struct df11_tensor {
    uint64_t n_elems;
    uint64_t total_bits; /* bits of code in enc (padding excluded) */
    uint64_t n_threads;  /* ceil(total_bits / (8 * n)) */
    uint64_t n_blocks;   /* ceil(n_threads / T) */
    df11_params params;
    uint32_t max_block_codes; /* most codes in one thread block (set by the encoder) */
    uint32_t reserved2;       /* 0 */
    uint8_t code_len[256];
    uint64_t enc_bytes;
    uint64_t sm_bytes;
    uint64_t gaps_bytes;
    uint64_t block_start_bytes;
    uint64_t lut_bytes;
    uint64_t counts_bytes;
    uint8_t *enc;
    uint8_t *sm;
    uint8_t *gaps;
    uint32_t *block_start;
    uint8_t *lut;
    uint8_t *counts; /* optional (NULL) */
} df11_tensor;

/* ------------------------------------------------------------------ host */

/* ABI version of this header (bumped on any layout change) and
 * sizeof(df11_tensor) as compiled into the library, so that bindings can
 * check their mirror of the struct. */
#define DF11_ABI_VERSION 3u
uint32_t df11_abi_version(void);
size_t df11_sizeof_tensor(void);

/* Default parameters: max_code_len 12, bytes_per_thread 8, T 256. */
void df11_default_params(df11_params *p);

/* Human-readable name of a status code (static string). */
const char *df11_status_str(df11_status s);

/* Exponent histogram of k matrices taken as one sequence ("Le format
 * DFloat11": the tree is built from the exponent distribution).
 * mats[i] points to sizes[i] BF16 values (as uint16 bits).  count[256] out. */
df11_status df11_exponent_histogram(const uint16_t *const *mats, const uint64_t *sizes,
                                    uint32_t k, uint64_t count[256]);

/* Size pass of the encoder for one matrix of n BF16 values: computes the
 * histogram, the length-limited optimal code lengths (canonical code), the
 * stream size, the aux sizes and every *_bytes field of *t.  The pointer
 * fields of *t are left untouched.  params may be NULL (defaults). */
df11_status df11_encode_size(const uint16_t *bf16, uint64_t n, const df11_params *params,
                             df11_tensor *t);

/* Fill pass: writes enc, sm, gaps, block_start, lut and (when non-NULL)
 * counts into the caller's host arrays *t points to (sizes from
 * df11_encode_size on the same data).  Arrays are fully written, padding
 * included. */
df11_status df11_encode(const uint16_t *bf16, uint64_t n, df11_tensor *t);

/* Same two passes for k matrices encoded as ONE stream with ONE shared table
 * ("Decompression par bloc transformer": every matrix of a transformer block
 * is decompressed in one batch).  Element i of matrix j sits at element
 * offset (sizes[0] + ... + sizes[j-1]) + i of the decoded block. */
df11_status df11_encode_multi_size(const uint16_t *const *mats, const uint64_t *sizes, uint32_t k,
                                   const df11_params *params, df11_tensor *t);
df11_status df11_encode_multi(const uint16_t *const *mats, const uint64_t *sizes, uint32_t k,
                              df11_tensor *t);

/* Host-side consistency check of a tensor's scalar fields and sizes
 * (no array contents are read; counts_bytes is checked only when counts is
 * non-NULL). */
df11_status df11_validate(const df11_tensor *t);

/* --------------------------------------------------------- device encoder */

/* The encoder for weights already in device memory: the exponent histogram
 * and the packing (EncodedExponent, PackedSignMantissa, Gaps, block output
 * positions: "Le format DFloat11", "Noyau GPU en deux etapes et metadonnees
 * auxiliaires") run on the GPU; the code lengths (<= 256 symbols) and the
 * decode tables are computed on the host by the same planner as
 * df11_encode, so the arrays are byte-identical to the host encoder's.
 *
 * Scratch: caller-owned device memory of df11_encode_device_scratch_bytes(n)
 * bytes, 16-byte aligned (the library allocates no device memory). */
uint64_t df11_encode_device_scratch_bytes(uint64_t n);

/* Size pass: w is a DEVICE array of n BF16 values (16-byte aligned; a block's
 * matrices concatenated) on the current device (else DF11_ERR_INVALID_ARG).
 * Runs the histogram on `stream`, synchronises it, plans the code and fills
 * *hdr (sizes, code lengths) as df11_encode_size does; array pointers are
 * left NULL. */
df11_status df11_encode_device_size(const uint16_t *w, uint64_t n, const df11_params *params, df11_tensor *hdr,
                                    void *scratch, uint64_t scratch_bytes, void *stream);

/* Fill pass: io from df11_encode_device_size with its array pointers set to
 * caller-allocated DEVICE buffers of the planned sizes (16-byte aligned;
 * counts may stay NULL, and is then not written).
 * Packs everything on `stream` (the decode tables are copied from the host)
 * and synchronises it; sets io->max_block_codes.  DF11_ERR_INVALID_ARG if
 * w no longer matches the planned code (e.g. changed since the size pass). */
df11_status df11_encode_device(const uint16_t *w, uint64_t n, df11_tensor *io, void *scratch, uint64_t scratch_bytes,
                               void *stream);

/* The device encoder without caller scratch.  The pages describe no
 * counterpart of these calls: they are a convenience of this library for
 * callers that must not allocate device memory around an encode -- e.g. a
 * runtime that owns all device memory through a fixed pool, or a serving
 * process re-encoding weights in place on a full GPU, where cudaMalloc would
 * fail or synchronise the device.  The scratch is a fixed array inside
 * libdf11 (264,224 B = 258 KiB on every device that loads the library,
 * held until exit), so:
 *  - n is limited to df11_encode_device_noalloc_max_elems() (2^28 weights, a
 *    whole Llama-3.1-8B block); larger inputs return DF11_ERR_TOO_LARGE
 *    before any GPU work;
 *  - every call looks up the array's address in the current device's
 *    context (cudaGetSymbolAddress), so a device reset or a re-created
 *    context is picked up; the first call on a device also loads the
 *    library's device code, so make it before any stream capture;
 *  - w must be device memory of the current device (else
 *    DF11_ERR_INVALID_ARG);
 *  - calls that overlap on one device (other host threads or streams) share
 *    that array and race: serialise them per device.
 * Everything the encoder needs cleared is cleared by each call.  Otherwise
 * as df11_encode_device_size / df11_encode_device. */
uint64_t df11_encode_device_noalloc_max_elems(void);
df11_status df11_encode_device_size_noalloc(const uint16_t *w, uint64_t n, const df11_params *params,
                                            df11_tensor *hdr, void *stream);
df11_status df11_encode_device_noalloc(const uint16_t *w, uint64_t n, df11_tensor *io, void *stream);

/* ---------------------------------------------------------------- device */

/* Decodes one compressed tensor into out (n_elems BF16 values, as uint16,
 * 16-byte aligned device memory).  One kernel launch on `stream`; the whole
 * decode (table staging, per-thread decode, block scan, sign/mantissa merge,
 * stores) runs on the GPU.  err_word: caller-owned device uint32 that the
 * kernel ORs DF11_KERR_* bits into (it is not cleared here); may be NULL,
 * in which case corruption is not reported.  n_elems == 0 is a no-op. */
df11_status df11_decode(const df11_tensor *t, uint16_t *out, uint32_t *err_word, void *stream);

/* Decodes every matrix of a transformer block, encoded with
 * df11_encode_multi, in ONE launch into a reusable BF16 scratch buffer of at
 * least t->n_elems elements ("Decompression par bloc transformer").
 * mat_offsets[0..k] are the element offsets of the k matrices in the
 * scratch (mat_offsets[0] == 0, mat_offsets[k] == n_elems, non-decreasing);
 * they are validated and matrix j is then the view
 * scratch[mat_offsets[j] .. mat_offsets[j+1]).  err_word as in df11_decode. */
df11_status df11_decode_block(const df11_tensor *blk, const uint64_t *mat_offsets, uint32_t k,
                              uint16_t *scratch, uint32_t *err_word, void *stream);

/* Row gather: decodes only rows rows[0..n_rows) of a compressed [R, row_len]
 * matrix (an embedding table: the rows a batch of token ids needs) into out,
 * row i of out = row rows[i] of the matrix (n_rows x row_len BF16 values,
 * row-major, 2-byte aligned device memory).  The pages name the embedding and
 * LM-head matrices among those DF11 compresses ("Le format DFloat11"); the
 * format keeps only each thread block's first output index ("Noyau GPU en deux
 * etapes et metadonnees auxiliaires"), so the kernel finds the thread blocks
 * covering a row by searching those indices, decodes them in full (count
 * pass or stored counts, scan, decoding pass) and writes only the row's elements.
 *  rows: DEVICE uint32 row indices (repeats allowed); an index >= R sets
 *        DF11_KERR_BAD_ROW and leaves that output row unwritten.
 *  row_len: > 0 and dividing t->n_elems; else DF11_ERR_INVALID_ARG.
 *  n_rows == 0 is a no-op.  err_word as in df11_decode.  One launch. */
df11_status df11_decode_rows(const df11_tensor *t, uint64_t row_len, const uint32_t *rows, uint32_t n_rows,
                             uint16_t *out, uint32_t *err_word, void *stream);

/* One matrix of a compressed tensor for df11_decode_gemv. */
typedef struct df11_gemv_mat {
    uint64_t elem_offset; /* first element of the [rows, cols] row-major matrix
                             in the tensor (e.g. a df11_decode_block offset);
                             a multiple of 16 */
    uint32_t rows;        /* out features, >= 1 */
    uint32_t cols;        /* in features, a multiple of 16 */
    const uint16_t *x;    /* DEVICE [T, cols] BF16 activations, row-major,
                             16-byte aligned */
    float *y;             /* DEVICE [T, rows] FP32, row-major: x * W^T is ADDED
                             (zero it first for a plain product), 4-byte
                             aligned */
} df11_gemv_mat;

/* Fused decode and matrix-vector products for small batches (1 <= T <= 4):
 * for each listed matrix, y += x * W^T, with W decoded on the fly and never
 * written to memory.  The pages decompress each matrix right before its
 * multiplication and discard it after ("Decompression adaptee a l'inference
 * GPU"); here the merge step multiplies every decoded 16-weight chunk by x
 * instead of storing it, so only the compressed arrays are read.  Only the
 * thread blocks that hold the listed matrices are decoded.
 *  mats: HOST array of n_mats descriptors (<= 16), ordered by elem_offset,
 *        not overlapping, each inside [0, t->n_elems); n_mats == 0 is a
 *        no-op.  Elements outside the listed matrices are decoded (where
 *        they share a thread block) but not used.
 *  FP32 accumulation (BF16 x BF16 products are exact); each warp's partial
 *  sum of a row is added into y with an FP32 atomic, so the last bits of y
 *  may differ run to run.
 *  Errors: DF11_ERR_UNSUPPORTED for T outside 1..4 or more than 16 matrices;
 *  DF11_ERR_INVALID_ARG for a bad descriptor (size, order, alignment, NULL).
 *  err_word as in df11_decode.  One launch, asynchronous on `stream`. */
df11_status df11_decode_gemv(const df11_tensor *t, const df11_gemv_mat *mats, uint32_t n_mats, uint32_t T,
                             uint32_t *err_word, void *stream);

/* Fused decode and matrix multiplication on the tensor cores (any batch
 * 1 <= T <= 256; meant for T > 4, where df11_decode_gemv's CUDA-core product
 * stops paying): for each listed matrix, y += x * W^T with W decoded on the
 * fly into shared-memory operand tiles of tcgen05.mma and never written to
 * memory.  The pages decompress each matrix right before its multiplication
 * and discard it after ("Decompression adaptee a l'inference GPU"); here the
 * decoded tiles go straight from the decoder to the tensor cores, so only the
 * compressed arrays are read from HBM.
 *  The listed matrices must be encoded in TILE ORDER (df11_to_tile_order):
 *  the same DF11 format, with each matrix's elements ordered as its 128 x 64
 *  tiles (row tiles in order, the 64-column tiles of a row tile in order, each
 *  tile row-major), so that every tile is a contiguous piece of the stream.
 *  mats: as for df11_decode_gemv (HOST array, <= 16 descriptors ordered by
 *        elem_offset, not overlapping; x [T, cols] BF16 16-byte aligned; y
 *        [T, rows] FP32 4-byte aligned, ADDED INTO: zero it first for a plain
 *        product), with rows a multiple of 128 and cols a multiple of 64.
 *  The tensor must carry its per-thread counts (t->counts), and its blocks
 *  must be LLM-like (at most 7137 codes per thread block, df11_tensor's
 *  max_block_codes); otherwise DF11_ERR_UNSUPPORTED.  So are T outside
 *  1..256, more than 16 matrices, and rows / cols off those multiples.
 *  FP32 accumulation in tensor memory; the partial sums of a row tile that two
 *  CTAs share are added with FP32 atomics, so the last bits of y may differ
 *  run to run.  A wait that timed out sets bit 0x20 of err_word.  One launch,
 *  asynchronous on `stream`; n_mats == 0 is a no-op. */
df11_status df11_decode_gemm(const df11_tensor *t, const df11_gemv_mat *mats, uint32_t n_mats, uint32_t T,
                             uint32_t *err_word, void *stream);

/* Tile order for df11_decode_gemm (host, plain copies): df11_to_tile_order
 * writes the row-major [rows, cols] BF16 matrix w (rows a multiple of 128,
 * cols of 64) into out as its 128 x 64 tiles (row tiles in order, the
 * 64-column tiles of a row tile in order, each tile row-major);
 * df11_from_tile_order is the inverse.  w and out must not overlap;
 * DF11_ERR_INVALID_ARG for NULL pointers, DF11_ERR_UNSUPPORTED for other
 * shapes. */
df11_status df11_to_tile_order(const uint16_t *w, uint32_t rows, uint32_t cols, uint16_t *out);
df11_status df11_from_tile_order(const uint16_t *tiled, uint32_t rows, uint32_t cols, uint16_t *out);

/* Consumer of a decoded weight matrix: Y = X * W^T with BF16 inputs and FP32
 * accumulation, the matrix multiplication the decompressed weights feed
 * ("Decompression adaptee a l'inference GPU": a matrix is decompressed right
 * before its multiplication and discarded after).  T > 4 runs on the tensor
 * cores (tcgen05; split-K partial sums are added with FP32 atomics, so the
 * last bits may differ run to run); T <= 4 is a matrix-vector stream on the
 * CUDA cores (bound by reading W; deterministic).
 *  x: DEVICE [T, in] BF16 (uint16 bits), row-major, 16-byte aligned
 *  w: DEVICE [out, in] BF16, row-major (nn.Linear layout; e.g. a view of a
 *     decoded block's scratch buffer), 16-byte aligned
 *  y: DEVICE [T, out] FP32, row-major; fully overwritten
 *  Limits: 1 <= T <= 256, out a multiple of 128, in a multiple of 64;
 *  otherwise DF11_ERR_UNSUPPORTED.  err_word as in df11_decode (a wait that
 *  timed out sets bit 0x20); may be NULL.  Asynchronous on `stream`. */
df11_status df11_gemm_bf16(const uint16_t *x, const uint16_t *w, float *y, uint32_t T, uint32_t out,
                           uint32_t in, uint32_t *err_word, void *stream);

/* One product of df11_gemm_bf16_multi: Y = X * W^T with
 *  x: DEVICE [T, in] BF16 (uint16 bits), row-major, 16-byte aligned
 *  w: DEVICE [out, in] BF16, row-major, 16-byte aligned
 *  y: DEVICE [T, out] FP32, row-major, 4-byte aligned; fully overwritten
 *  out a multiple of 128, in a multiple of 64. */
typedef struct df11_gemm_mat {
    const uint16_t *x;
    const uint16_t *w;
    float *y;
    uint32_t out, in;
} df11_gemm_mat;

/* Several consumer products of decoded weights, e.g. the seven matrices of a
 * decoded transformer block ("Decompression adaptee a l'inference GPU": each
 * matrix is multiplied right after its decompression), in ONE persistent
 * tensor-core launch for T > 4: the 128 x 64 weight tiles of all products
 * are split evenly over the SMs (no per-matrix launch tail), partial sums
 * are added into Y with FP32 atomics after the Y buffers are zeroed on the
 * stream (the last bits may differ run to run).  T <= 4: one matrix-vector
 * launch per product, as df11_gemm_bf16.  1 <= n_mats <= 16, 1 <= T <= 256
 * (else DF11_ERR_UNSUPPORTED; shape and alignment faults as for
 * df11_gemm_bf16).  err_word: bit 0x20 when a wait timed out; may be NULL.
 * Asynchronous on `stream`; `mats` is read before the call returns. */
df11_status df11_gemm_bf16_multi(const df11_gemm_mat *mats, uint32_t n_mats, uint32_t T, uint32_t *err_word,
                                 void *stream);

/* Copies *err_word to the host after the stream's work so far completes
 * (synchronises the stream) and returns DF11_ERR_CORRUPT if any bit is set. */
df11_status df11_read_error(const uint32_t *err_word, void *stream, uint32_t *host_value);

/* Number of SMs the decode kernel sizes its persistent grid to on the
 * current device (for reporting). */
df11_status df11_device_sm_count(int *sm_count);

#ifdef __cplusplus
}
#endif

#endif /* DF11_H */
