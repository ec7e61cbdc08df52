/*
 * df11.h -- C ABI of the DF11 (DFloat11) decode library, libdf11.so.
 *
 * DF11 stores a BF16 weight tensor as
 *   - its 8-bit exponents, Huffman coded with a canonical code of at most
 *     32-bit codewords and packed into one MSB-first bitstream, and
 *   - its sign and 7 mantissa bits, kept as they are, one byte per element
 *     (sign in bit 7, mantissa in bits 0-6).
 * Sources: "DFloat11无损压缩技术：基于哈夫曼编码的BFloat16大模型显存优化方案"
 * (jsqmd.com), §2.1 (BF16 fields) and §2.2 items 1-3 (Huffman-coded
 * exponents, sign/mantissa kept, aligned blocks, decode on the GPU right
 * before the matmul, no CPU decompression, discard after use);
 * "DFloat11：用于高效 GPU 推理的 LLM 和扩散模型无损压缩" (gittoolsai.com),
 * section "工作原理" (bit-identical output, weights stay compressed in GPU
 * memory); "DFloat11重新定义LLM无损压缩的技术边界" (ocdem.com), §2.2
 * (multi-level lookup tables in shared memory, two-phase locate /
 * reconstruct, parallel prefix sum).
 *
 * Layout of one encoded tensor (written by df11_build):
 *   bitstream      the codewords of elements 0..n-1, one after another,
 *                  first bit = bit 7 of byte 0.  Cut into chunks of C bytes
 *                  (one per decoding thread) and blocks of T chunks (one per
 *                  thread block).  num_blocks*T*C bytes + 16 zero bytes.
 *   gaps           per chunk, the distance in bits (0..31) from the chunk's
 *                  first bit to the first codeword that starts at or after
 *                  it (to the end of the stream if none does; 0 for chunks
 *                  past the end).  5-bit fields packed MSB-first;
 *                  num_blocks*T*5/8 + 16 bytes.
 *   block_out_pos  num_blocks+1 uint32: index of the first element whose
 *                  codeword starts in each block; the last entry is n.
 *   chunk_counts   per chunk, the number of codewords that start in it
 *                  (uint8; num_blocks*T + 16 bytes).  Derived metadata the
 *                  pages do not have: with it a decoding thread knows where
 *                  its output goes before it decodes; without it (NULL) the
 *                  thread counts by decoding first.
 *   luts           num_luts tables of 256 uint32, table 0 first:
 *                  table 0, indexed by the next 8 bits: up to three whole
 *                  codewords in those bits -- bits 0-23 their exponents
 *                  (first in bits 0-7, unused bytes 0), bits 24-27 the bits
 *                  they use (1..8), bits 28-29 how many (1..3); or, when the
 *                  first codeword is longer than 8 bits, bits 0-23 the number
 *                  of the next-level table and bits 24-31 zero.
 *                  tables 1.. (levels 1..3), indexed by the following 8
 *                  bits: bits 0-7 the exponent and bits 28-29 = 1, or a
 *                  pointer as above.  0 marks a bit pattern no codeword
 *                  starts with.  Tables are numbered level by level and by
 *                  prefix value within a level.
 *   code_lengths   256 bytes, codeword length of each exponent (0 = absent).
 *   sign_mantissa  n bytes, readable up to a multiple of 16 bytes.
 *
 * Every decode call is asynchronous on the given stream, allocates nothing,
 * never synchronises the host and has no CPU fallback.  Argument errors are
 * returned at once; errors the GPU finds in the data are written to the
 * optional device word d_err (first error wins) and never trap.
 */
#ifndef DF11_H
#define DF11_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* The CUDA runtime's cudaStream_t; NULL is the legacy default stream. */
typedef struct CUstream_st *df11_stream_t;

typedef enum df11_status {
  DF11_OK = 0,
  DF11_ERR_NULL = 1,        /* a required pointer is NULL */
  DF11_ERR_ALIGN = 2,       /* a pointer misses its required alignment */
  DF11_ERR_FORMAT = 3,      /* parameters inconsistent with each other */
  DF11_ERR_UNSUPPORTED = 4, /* (chunk_bytes, threads_per_block) not built */
  DF11_ERR_CUDA = 5,        /* a CUDA runtime call failed */
  DF11_ERR_TOO_LARGE = 6,   /* n >= 2^32, or a batch over DF11_MAX_BATCH */
  DF11_ERR_INVALID = 7,     /* other invalid argument */
  DF11_ERR_NOMEM = 8,       /* host allocation failed (df11_build) */
  DF11_ERR_DEVICE = 9       /* a device pointer is not memory of the current
                               device (checked before anything is queued) */
} df11_status;

/* Values the GPU writes to *d_err.  A device word that is not 0 means the
 * output of the call is not to be trusted. */
#define DF11_DEV_OK 0
#define DF11_DEV_ERR_COUNT 1    /* a block decoded a different element count
                                   than block_out_pos says */
#define DF11_DEV_ERR_OVERRUN 2  /* a thread's last codeword ran past the
                                   start of the next thread's first one */
#define DF11_DEV_ERR_TABLE 3    /* the stream reached an invalid table entry
                                   or a zero code length */
#define DF11_DEV_ERR_TIMEOUT 4  /* an asynchronous copy into shared memory
                                   did not complete in time */
#define DF11_DEV_ERR_CAPACITY 5 /* a block holds more elements than
                                   max_block_elems */

/* Largest number of tensors one df11_decode_batched launch takes. */
#define DF11_MAX_BATCH 16

/* Per-tensor format parameters, written by df11_build. */
typedef struct df11_params {
  uint64_t n;                 /* elements (< 2^32) */
  uint64_t total_bits;        /* meaningful bits of the bitstream */
  uint32_t chunk_bytes;       /* C: bitstream bytes per thread */
  uint32_t threads_per_block; /* T: threads (chunks) per block */
  uint32_t num_blocks;        /* ceil(total_bits / (8*C*T)) */
  uint32_t num_luts;          /* 256-entry tables (>= 1) */
  uint32_t max_block_elems;   /* max over blocks of elements per block */
  uint32_t max_len;           /* longest codeword in bits (<= 32) */
  uint32_t max_chunk_elems;   /* max over chunks of codewords starting in it */
  uint32_t max_warp_elems;    /* max over groups of 32 consecutive chunks of
                                 the codewords starting in them (one warp's
                                 share of a block in the decode kernel;
                                 sizes its shared-memory buffers) */
} df11_params;

/* Bytes of the decode table that df11_build_decode_table writes. */
#define DF11_DECODE_TABLE_BYTES 17664

/* One tensor to decode: device pointers plus its parameters. */
typedef struct df11_tensor {
  const uint8_t *bitstream;      /* 16-byte aligned */
  const uint8_t *gaps;           /* 16-byte aligned */
  const uint8_t *chunk_counts;   /* 16-byte aligned, or NULL */
  const uint32_t *block_out_pos; /* 4-byte aligned */
  const uint32_t *luts;          /* 16-byte aligned */
  const uint8_t *code_lengths;   /* any alignment */
  const uint8_t *sign_mantissa;  /* 16-byte aligned */
  uint16_t *out_bf16;            /* 16-byte aligned, n elements, caller-owned */
  const void *decode_table;      /* 16-byte aligned, DF11_DECODE_TABLE_BYTES
                                    written by df11_build_decode_table from
                                    this tensor's luts and code_lengths; or
                                    NULL: every thread block derives it */
  df11_params params;
} df11_tensor;

/*
 * Decode one tensor into out_bf16 (bit-identical to the BF16 tensor that was
 * encoded), from the format the pages describe (no chunk counts: every
 * thread counts its codewords by decoding, then places them after the scan).
 * All pointers are device pointers owned by the caller and laid out as
 * described at the top of this file; `params` is a host pointer.
 * n must equal params->n.  d_err is a device int32 (may be NULL) that the
 * caller zeroes; the kernel writes a DF11_DEV_ERR_* code into it when the
 * data are inconsistent.  Returns DF11_OK once the work is queued on
 * `stream`.  n == 0 queues nothing.
 */
df11_status df11_decode(const uint8_t *bitstream, const uint8_t *gaps,
                        const uint32_t *block_out_pos, const uint32_t *luts,
                        const uint8_t *code_lengths,
                        const uint8_t *sign_mantissa, uint16_t *out_bf16,
                        uint64_t n, const df11_params *params, int32_t *d_err,
                        df11_stream_t stream);

/*
 * Launches use programmatic dependent launch: a decode kernel may start
 * while the previous kernel in the stream finishes, and waits for it to
 * complete before its first store to out_bf16 (which that kernel may still
 * read or write); the compressed inputs must not be written by it.  Setting
 * DF11_PDL=0 in the environment before the first call launches plainly.
 */

/*
 * Decode `count` tensors (a layer's weights, say) with one kernel launch per
 * DF11_MAX_BATCH tensors.  `tensors` is a host array; every tensor must use
 * the same chunk_bytes and threads_per_block.  A tensor whose chunk_counts is
 * not NULL is decoded in one pass straight to its output places; the others
 * as in df11_decode.  Same conventions as df11_decode.
 */
df11_status df11_decode_batched(const df11_tensor *tensors, int count,
                                int32_t *d_err, df11_stream_t stream);

/* Largest batch (activation rows) one df11_decode_gemv operation takes. */
#define DF11_GEMV_MAX_BATCH 8

/* The matrix-vector product applied to one decoded tensor. */
typedef struct df11_gemv {
  const uint16_t *x;   /* BF16 activations (device, 16-byte aligned): `batch` rows of
                          `cols` elements, row b at x + b*x_stride */
  float *y;            /* fp32 outputs (device, 4-byte aligned): `batch` rows of
                          n/cols elements, row b at y + b*y_stride */
  uint32_t cols;       /* in-features: the decoded tensor is (n/cols) x cols, row-major;
                          a multiple of 16 that divides n */
  uint32_t batch;      /* 1 .. DF11_GEMV_MAX_BATCH */
  uint32_t x_stride;   /* elements between activation rows: >= cols, a multiple of 8 */
  uint32_t y_stride;   /* elements between output rows: >= n/cols */
  int32_t accumulate;  /* 0: y = W x (the call clears y first, in stream order);
                          otherwise y += W x */
  uint32_t interleave; /* the tensor's element order: R rows interleaved per 16 columns
                          (R = 1 or 0: row-major; else a power of two up to 32 that
                          divides n/cols).  With R rows interleaved the compressed
                          stream holds, for each block of R rows and each group of 16
                          columns, the R rows' 16 elements one after another; lanes that
                          share a column group then share activations, which makes
                          batches above 1 cheaper (see df11_decode_gemv). */
} df11_gemv;

/*
 * Decode-and-multiply without writing the decoded tensor anywhere: for each
 * tensor W (rows x cols) and its df11_gemv op, y[b][r] (+)= sum over c of
 * W[r][c] * x[b][c], the decoded BF16 weights taken straight from the decode
 * kernel's registers into fp32 fused multiply-adds.  This is the pages'
 * "decode just before the matmul" ("DFloat11无损压缩技术" (jsqmd.com) §2.2
 * item 3; "DFloat11重新定义LLM无损压缩的技术边界" (ocdem.com) §2.2) for
 * batch-1 and small-batch matrix-vector products, without the round trip of
 * the BF16 weights through memory.  Needs chunk counts and T = 256 with
 * C = 8, 16 or 24; out_bf16 is not used (may be NULL).  Every product
 * w*x is exact in fp32; the sums run in fp32 in an order that depends on
 * scheduling (atomic adds per row segment), so y may differ from run to
 * run in the last bits, within the usual bound for an fp32 sum of cols
 * terms.  Same conventions as df11_decode_batched otherwise (asynchronous,
 * no allocation, device-detected errors in d_err); the activations may be
 * written by the previous kernel in the stream.  DF11_ERR_INVALID for a
 * cols, batch or stride outside the rules above.
 */
df11_status df11_decode_gemv(const df11_tensor *tensors, const df11_gemv *ops, int count,
                             int32_t *d_err, df11_stream_t stream);

/* Largest batch one df11_decode_gemm operation takes. */
#define DF11_GEMM_MAX_BATCH 128

/*
 * The same product for batches of activation rows, on the tensor cores: for
 * each tensor W (rows x cols) and its df11_gemv op, y[b][r] (+)= sum over c
 * of W[r][c] * x[b][c], with W decoded inside the kernel into shared memory
 * in 128 x 16 tiles that tcgen05.mma multiplies (BF16 operands, fp32
 * accumulation in tensor memory); the decoded weights never reach global
 * memory.  This is the pages' decode right before the matmul
 * ("DFloat11无损压缩技术" (jsqmd.com) §2.2 item 3: the cost of decoding is
 * spread over the batch, so the gap to BF16 shrinks as the batch grows;
 * "DFloat11重新定义LLM无损压缩的技术边界" (ocdem.com) §3.2) for batches
 * from 1 to DF11_GEMM_MAX_BATCH.
 * Requirements beyond df11_decode_gemv's: the tensor encoded with 128 rows
 * interleaved per 16 columns (interleave = 128, rows a multiple of 128),
 * chunk counts and a decode table present, T = 256 and C = 8 or 16 (the
 * tile ring and the accumulators must fit one thread block's shared and
 * tensor memory), at most DF11_MAX_BATCH tensors per call, all of one C.
 * The sums run in fp32 in an order that depends on the tiling and on
 * scheduling (atomic adds per 128-row block and K range), within the usual
 * bound for an fp32 sum of cols terms.  Same conventions as
 * df11_decode_gemv otherwise.  DF11_ERR_UNSUPPORTED for a tensor without
 * counts or table or of another chunk size; DF11_ERR_INVALID for a layout,
 * batch or stride outside the rules.
 */
df11_status df11_decode_gemm(const df11_tensor *tensors, const df11_gemv *ops, int count,
                             int32_t *d_err, df11_stream_t stream);

/*
 * Derive, on the device, the decode table of one tensor from its luts and
 * code_lengths (device pointers, as in df11_tensor) into `out` (device,
 * 16-byte aligned, DF11_DECODE_TABLE_BYTES, caller-owned).  The table is an
 * acceleration structure of this library (no counterpart in the format the
 * pages describe): the format's first table and code lengths with every
 * exponent byte rotated right by one bit, and a table of 2^11 entries each
 * holding the codewords that lie wholly inside an 11-bit window.  Passing it
 * in df11_tensor.decode_table saves every thread block of every decode call
 * from deriving it.  Asynchronous on `stream`; DF11_ERR_NULL / _ALIGN /
 * _FORMAT (num_luts outside 1 .. 2^24-1) are returned before anything is
 * queued.
 */
df11_status df11_build_decode_table(const uint32_t *luts, const uint8_t *code_lengths,
                                    uint32_t num_luts, void *out, df11_stream_t stream);

/* Bytes of dynamic shared memory one thread block of a decode launch for
 * these parameters may use: the larger of the two kernels' needs (with and
 * without chunk counts), for occupancy planning; 0 if unsupported. */
size_t df11_shared_bytes(const df11_params *params);

/* 1 if the library has a kernel for this (chunk_bytes, threads_per_block). */
int df11_supported(uint32_t chunk_bytes, uint32_t threads_per_block);

const char *df11_status_string(df11_status status);
const char *df11_device_error_string(int32_t code);

/* Testing hook for the decode's failure detection (no counterpart in the
 * pages).  Every wait of the decode kernels is bounded: a thread block that
 * has waited too long for its own copies reports DF11_DEV_ERR_TIMEOUT in
 * d_err and stops, and the context stays usable.  After this call, the next
 * `launches` decode launches of tensors with chunk counts are made with the
 * producer issuing no stage copy, so that the consumers' waits run out after
 * `spin_limit` polls (each suspends for up to about a microsecond; 1 ..
 * 2^20, the default bound).  No copy is then in flight and nothing faults:
 * the failure is a withheld message, injected from the host.  Returns
 * DF11_ERR_INVALID for arguments out of range.  Process-wide; not for use
 * alongside real decodes in other threads. */
df11_status df11_test_withhold_copies(int launches, uint32_t spin_limit);

/* ---------------------------------------------------------------------- */
/* Host-side format builder ("compression"; offline, host memory only).   */

typedef struct df11_host_tensor {
  df11_params params;
  uint8_t code_lengths[256];
  uint8_t *bitstream;
  uint64_t bitstream_bytes;   /* num_blocks*T*C + 16 */
  uint8_t *gaps;
  uint64_t gaps_bytes;        /* num_blocks*T*5/8 + 16 */
  uint32_t *block_out_pos;    /* num_blocks + 1 */
  uint32_t *luts;             /* num_luts * 256 */
  uint8_t *sign_mantissa;
  uint64_t sign_mantissa_bytes; /* n rounded up to 16 */
  uint8_t *chunk_counts;
  uint64_t chunk_counts_bytes;  /* num_blocks*T + 16 */
} df11_host_tensor;

/*
 * Encode n BF16 words (host memory) with chunk_bytes C (a multiple of 4,
 * 4..28) and threads_per_block T (a multiple of 128, 128..1024), using up
 * to num_threads host threads (<= 0: all cores).  The exponent code is the
 * Huffman code of the exponent histogram, limited to 32-bit codewords by
 * package-merge when needed, in canonical form; ties are broken by symbol
 * value so the output is deterministic.  On success the buffers in *out
 * belong to the caller and are released with df11_host_tensor_free.
 */
df11_status df11_build(const uint16_t *bf16, uint64_t n, uint32_t chunk_bytes,
                       uint32_t threads_per_block, int num_threads,
                       df11_host_tensor *out);
void df11_host_tensor_free(df11_host_tensor *t);

/* ---------------------------------------------------------------------- */
/* Device-side format builder: the same encoding, byte for byte, of BF16  */
/* words already in device memory.                                        */
/*                                                                        */
/* The pages build the format offline on the host ("DFloat11无损压缩技术"  */
/* (jsqmd.com) §2.2 items 1-2).  Here histogram, bit offsets, packing,    */
/* gaps, block positions and counts run on the device; the codebook (256  */
/* symbols) on the host.  Two calls, so that the caller allocates the     */
/* output buffers once their sizes are known.                             */

typedef struct df11_gpu_build df11_gpu_build;

/*
 * Phase 1.  d_bf16: n BF16 words in device memory (2-byte aligned; 16-byte
 * alignment lets the kernels load 8 words at a time and must then hold in
 * phase 2 too).  Same chunk_bytes / threads_per_block rules as df11_build.
 * Computes the histogram and the code, waits for the counts (everything
 * queued on `stream` before them has then run), and on success fills *params (n, total_bits, chunk_bytes, threads_per_block,
 * num_blocks, num_luts, max_len; the max_* counts are filled by phase 2),
 * code_lengths (host, 256 bytes) and *handle, which holds device scratch
 * until phase 2 or df11_gpu_build_free.  The scratch comes from a memory
 * pool the library keeps per device (allocated and freed in stream order;
 * what the pool has reserved stays reserved for the process, so repeated
 * builds allocate nothing new).  The buffers phase 2 writes, with
 * C = chunk_bytes, T = threads_per_block, B = num_blocks:
 *   bitstream      B*T*C + 16 bytes       gaps           B*T*5/8 + 16 bytes
 *   chunk_counts   B*T + 16 bytes         block_out_pos  (B + 1) uint32
 *   luts           num_luts*256 uint32    code_lengths   256 bytes
 *   sign_mantissa  n rounded up to 16 bytes
 * Errors: DF11_ERR_NULL, _INVALID, _TOO_LARGE, _ALIGN, _NOMEM before any
 * device work; DF11_ERR_CUDA if a CUDA call fails.  *handle is NULL on
 * every error.  Small transfers between host and device go through a pinned
 * buffer the library keeps; concurrent build calls take turns on it.
 */
df11_status df11_gpu_build_begin(const uint16_t *d_bf16, uint64_t n, uint32_t chunk_bytes,
                                 uint32_t threads_per_block, df11_stream_t stream,
                                 df11_params *params, uint8_t code_lengths[256],
                                 df11_gpu_build **handle);

/*
 * Phase 2.  Writes the encoded tensor into caller-owned device buffers of
 * the sizes above (bitstream, gaps, chunk_counts, luts, sign_mantissa
 * 16-byte aligned; block_out_pos 4-byte aligned), from the same d_bf16,
 * on `stream`, and synchronises it.  On success *params is complete and
 * equal to what df11_build returns for the same words.  Releases the
 * handle in every case (success or error).
 */
df11_status df11_gpu_build_finish(df11_gpu_build *handle, const uint16_t *d_bf16,
                                  uint8_t *bitstream, uint8_t *gaps, uint8_t *chunk_counts,
                                  uint32_t *block_out_pos, uint32_t *luts,
                                  uint8_t *code_lengths, uint8_t *sign_mantissa,
                                  df11_params *params, df11_stream_t stream);

/*
 * Exponent histogram of n BF16 words in device memory, with no allocation:
 * hist[e] (host array of 256) = how many words have exponent field e (bits
 * 7-14).  The paper has no counterpart to this entry point.  It is the
 * builder's histogram kernel on its own, for callers that cannot allocate
 * device memory -- code that runs where the CUDA allocator must not be
 * entered (an allocator hook, a memory pool in the middle of a resize), or
 * a program that has handed all device memory to its own allocator -- and
 * still want the exponent statistics (entropy, the size a tensor will
 * compress to).  It calls no cudaMalloc, cudaFree or other allocating
 * routine: its counters are a fixed array of 256 64-bit counters (2 KB) in
 * the library's device memory, one per device, held until the process
 * exits.  The first call on a device looks up that array's device address
 * (set-up, with the device current); make that first call before any
 * stream capture.  All calls on a device share the array and it keeps the
 * last call's counts, so every call clears it first; calls whose work
 * overlapped on the GPU would race on it, so the library takes one call at
 * a time per device and waits for each call's counts.  Queues its work on
 * `stream` (of the current device) and synchronises it; the counts are
 * copied straight into `hist` (pinned memory makes that a DMA).  d_bf16
 * must be 2-byte aligned memory of the current device (16-byte alignment
 * lets the kernel load 8 words at a time).  Errors: DF11_ERR_NULL,
 * _TOO_LARGE (n >= 2^32: beyond the counters' and the kernel's index
 * range), _ALIGN, _DEVICE (d_bf16 not memory of the current device) before
 * any device work; DF11_ERR_CUDA if a CUDA call fails.
 */
df11_status df11_exponent_histogram(const uint16_t *d_bf16, uint64_t n, uint64_t hist[256],
                                    df11_stream_t stream);

/* The output buffers of one tensor's phase 2 (sizes and alignment as for
 * df11_gpu_build_finish). */
typedef struct df11_gpu_build_out {
  uint8_t *bitstream;
  uint8_t *gaps;
  uint8_t *chunk_counts;
  uint32_t *block_out_pos;
  uint32_t *luts;
  uint8_t *code_lengths;
  uint8_t *sign_mantissa;
} df11_gpu_build_out;

/*
 * Both phases for `count` tensors at once (d_bf16[i], n[i]; params and
 * handles arrays of count, code_lengths count*256 bytes, all host arrays).
 * Phase 1 counts up to 32 tensors per launch, the last quarter of the
 * elements (the shortest run of last tensors that holds it) in a launch of
 * its own, and waits for each launch's counts as they arrive (computing
 * their codes while the device works on the later tensors); phase 2
 * synchronises the stream once.  Same conventions as the
 * single-tensor calls; on an error in phase 1 no handle is returned (all
 * NULL), and phase 2 releases every handle in all cases.  The
 * single-tensor calls are these with count 1.
 */
df11_status df11_gpu_build_begin_batched(const uint16_t *const *d_bf16, const uint64_t *n,
                                         int count, uint32_t chunk_bytes,
                                         uint32_t threads_per_block, df11_stream_t stream,
                                         df11_params *params, uint8_t *code_lengths,
                                         df11_gpu_build **handles);
df11_status df11_gpu_build_finish_batched(df11_gpu_build *const *handles, int count,
                                          const uint16_t *const *d_bf16,
                                          const df11_gpu_build_out *outs, df11_params *params,
                                          df11_stream_t stream);

/*
 * Where the phase-2 outputs of `count` tensors go in one device allocation
 * (params as phase 1 filled them): tensor after tensor, each tensor's seven
 * buffers in the order of df11_gpu_build_out with the sizes listed at
 * df11_gpu_build_begin, every buffer at a 256-byte offset and given at
 * least 16 bytes.  Writes buffer j of tensor i's byte offset to
 * offsets[7 i + j] and its size to sizes[7 i + j] (either array may be
 * NULL) and returns the allocation's size in bytes; 0 for a NULL params or
 * a negative count.  Host only: touches no device.
 */
uint64_t df11_gpu_build_layout(const df11_params *params, int count, uint64_t *offsets,
                               uint64_t *sizes);

/* Release a phase-1 handle without running phase 2 (NULL is a no-op); its
 * scratch is freed in order on the stream phase 1 ran on, which must still
 * exist. */
void df11_gpu_build_free(df11_gpu_build *handle);

#ifdef __cplusplus
}
#endif
#endif /* DF11_H */
