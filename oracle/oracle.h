/*
 * oracle.h -- plain, slow, single-threaded CPU oracle for DFloat11 (DF11)
 * Huffman-coded BF16 weights.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may include, link
 * or call this code: only the tests, the smoke check and the CPU-baseline
 * leg of the benchmark do.  It shares no source with the CUDA library.
 *
 * What it computes, and where the pages say so:
 *  - BF16 = 1 sign bit, 8 exponent bits, 7 mantissa bits; only the exponent
 *    is entropy coded, sign and mantissa are kept as they are
 *    ("DFloat11无损压缩技术" (jsqmd.com), §2.1 and §2.2 items 1-2).
 *  - Exponent histogram -> Huffman code lengths, frequent exponents short
 *    (same page, §2.2 item 1), limited to 32 bits and made canonical
 *    (the format statement of the decode path; the pages are silent on the
 *    limit, so the optimal length-limited code is built with package-merge).
 *  - Codewords packed into one bitstream, cut into fixed-size per-thread
 *    chunks with the bit offset ("gap") of each chunk's first codeword and the
 *    first output index of each block of chunks (same page, §2.2 item 2,
 *    "aligned memory blocks"; per-thread/per-block layout from the format
 *    statement of the decode path).
 *  - Hierarchical 256-entry lookup tables ("DFloat11 ... 三重编码机制",
 *    ocdem.com, §2.2, "multi-level compact lookup tables").
 *  - Decoding is a bit-serial canonical decode that never looks at the
 *    lookup tables, so it shares no logic with the GPU path.
 *
 * Parity status of each function is stated in the oracle's Python header
 * (oracle/__init__.py) and in the tests that pin it.
 */
#ifndef DF11_ORACLE_H
#define DF11_ORACLE_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define ORACLE_MAX_LEN 32

/* Everything the encoder produces.  All buffers are malloc'd by
 * oracle_encode and released by oracle_format_free. */
typedef struct oracle_format {
  uint64_t n;                 /* elements */
  uint64_t total_bits;        /* meaningful bits in the bitstream */
  uint32_t chunk_bytes;       /* C: bitstream bytes per thread */
  uint32_t threads_per_block; /* T: chunks per block */
  uint32_t num_blocks;        /* ceil(total_bits / (8*C*T)) */
  uint32_t num_luts;          /* 256-entry tables, level 0 first */
  uint32_t max_block_elems;   /* max over blocks of its element count */
  uint32_t max_len;           /* longest codeword */
  uint32_t max_chunk_elems;   /* max over chunks of codewords starting in it */
  uint32_t max_warp_elems;    /* max over groups of 32 consecutive chunks of
                                 the codewords starting in them */
  uint8_t code_lengths[256];  /* 0 = exponent absent */
  uint32_t codes[256];        /* canonical codeword, right-aligned */
  uint8_t *bitstream;         /* num_blocks*T*C + 16 bytes, MSB-first */
  uint64_t bitstream_bytes;
  uint8_t *gaps;              /* one value 0..31 per chunk (unpacked) */
  uint8_t *gaps_packed;       /* 5-bit fields, MSB-first */
  uint64_t gaps_bytes;        /* num_blocks*T*5/8 + 16 */
  uint32_t *block_out_pos;    /* num_blocks + 1 entries, last == n */
  uint32_t *luts;             /* num_luts * 256 entries */
  uint8_t *sign_mantissa;     /* n bytes, buffer padded to a multiple of 16 */
  uint64_t sm_bytes;
  uint8_t *chunk_counts;      /* codewords starting in each chunk; chunks+16 */
  uint64_t chunk_counts_bytes;
} oracle_format;

/* Field split of one BF16 word. */
void oracle_split(const uint16_t *w, uint64_t n, uint8_t *exps, uint8_t *sm);
void oracle_histogram(const uint8_t *exps, uint64_t n, uint64_t hist[256]);

/* Unconstrained Huffman code lengths (depth of each leaf).  Ties are broken
 * by (weight, smallest symbol in the subtree).  Returns the longest length
 * (which may exceed 32), 0 when no symbol is present. */
int oracle_huffman_lengths(const uint64_t hist[256], uint8_t len[256]);

/* Optimal code lengths limited to max_len bits by package-merge.  Returns the
 * longest length, 0 when no symbol is present, -1 when 2^max_len < symbols. */
int oracle_package_merge_lengths(const uint64_t hist[256], int max_len,
                                 uint8_t len[256]);

/* The code lengths the format uses: Huffman, or package-merge with a 32-bit
 * limit when Huffman is deeper than that.  A lone symbol gets length 1. */
int oracle_code_lengths(const uint64_t hist[256], uint8_t len[256]);

/* Canonical codewords for the given lengths. */
void oracle_canonical_codes(const uint8_t len[256], uint32_t codes[256]);

/* Hierarchical tables.  Writes at most max_tables*256 entries into luts (may
 * be NULL to count) and returns the number of tables. */
int oracle_build_luts(const uint8_t len[256], const uint32_t codes[256],
                      uint32_t *luts, int max_tables);

/* Full encoder.  Returns 0 on success. */
int oracle_encode(const uint16_t *w, uint64_t n, uint32_t chunk_bytes,
                  uint32_t threads_per_block, oracle_format *out);
void oracle_format_free(oracle_format *f);

/* Bit-serial canonical decode of `count` codewords starting at bit
 * `start_bit`, each fused with its sign/mantissa byte sm[i].  Writes the
 * start bit of every codeword to starts (may be NULL).  Returns the bit
 * position after the last codeword, or UINT64_MAX on an invalid stream. */
uint64_t oracle_decode(const uint8_t *bitstream, uint64_t bitstream_bytes,
                       uint64_t start_bit, const uint8_t len[256],
                       const uint8_t *sm, uint64_t count, uint16_t *out,
                       uint64_t *starts);

/* Chunk gaps and block output positions recomputed from the list of codeword
 * start bits.  gaps gets num_blocks*T values, block_out_pos num_blocks+1. */
void oracle_metadata_from_starts(const uint64_t *starts, uint64_t n,
                                 uint64_t total_bits, uint32_t chunk_bytes,
                                 uint32_t threads_per_block,
                                 uint32_t num_blocks, uint8_t *gaps,
                                 uint32_t *block_out_pos);

/* Pack one 5-bit value per chunk, MSB-first. */
void oracle_pack_gaps(const uint8_t *gaps, uint64_t count, uint8_t *packed);

#ifdef __cplusplus
}
#endif
#endif
