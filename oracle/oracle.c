/*
 * oracle.c -- plain, slow, single-threaded CPU oracle for DF11 (see oracle.h).
 *
 * TEST INFRASTRUCTURE ONLY: used by tests/, the smoke check and the
 * benchmark's CPU-baseline leg, never by the product path.  Written for
 * obviousness, not speed: bits are written and read one at a time and every
 * table entry is found by trying every codeword.
 */
#include "oracle.h"

#include <stdlib.h>
#include <string.h>

/* ------------------------------------------------------------------------ */
/* Field split.  "DFloat11无损压缩技术" (jsqmd.com) §2.1: a BF16 word is one
 * sign bit, eight exponent bits and seven mantissa bits.  §2.2 item 2: the
 * sign bit and the 7 mantissa bits are kept unchanged.  They are stored as
 * one byte, sign in bit 7 and mantissa in bits 0-6.                         */
void oracle_split(const uint16_t *w, uint64_t n, uint8_t *exps, uint8_t *sm) {
  for (uint64_t i = 0; i < n; i++) {
    uint16_t x = w[i];
    uint8_t sign = (uint8_t)((x >> 15) & 1);
    uint8_t exponent = (uint8_t)((x >> 7) & 0xFF);
    uint8_t mantissa = (uint8_t)(x & 0x7F);
    if (exps) exps[i] = exponent;
    if (sm) sm[i] = (uint8_t)((sign << 7) | mantissa);
  }
}

/* Same page, §2.2 item 1: count how often each exponent value occurs.      */
void oracle_histogram(const uint8_t *exps, uint64_t n, uint64_t hist[256]) {
  for (int s = 0; s < 256; s++) hist[s] = 0;
  for (uint64_t i = 0; i < n; i++) hist[exps[i]]++;
}

/* ------------------------------------------------------------------------ */
/* Huffman code lengths (same page, §2.2 item 1: frequent exponents get short
 * codewords).  Textbook construction: repeatedly merge the two lightest
 * nodes.  Ties go to the node whose smallest symbol is smaller, so the result
 * is unique.  Quadratic scans; at most 256 leaves.                          */
int oracle_huffman_lengths(const uint64_t hist[256], uint8_t len[256]) {
  uint64_t weight[511];
  int minsym[511], parent[511], alive[511];
  int leaf_of[256];
  int nodes = 0;
  for (int s = 0; s < 256; s++) {
    len[s] = 0;
    leaf_of[s] = -1;
    if (hist[s] > 0) {
      weight[nodes] = hist[s];
      minsym[nodes] = s;
      parent[nodes] = -1;
      alive[nodes] = 1;
      leaf_of[s] = nodes;
      nodes++;
    }
  }
  int leaves = nodes;
  if (leaves == 0) return 0;
  if (leaves == 1) {
    for (int s = 0; s < 256; s++)
      if (leaf_of[s] >= 0) len[s] = 1;
    return 1;
  }
  for (int round = 0; round < leaves - 1; round++) {
    int a = -1, b = -1;
    for (int i = 0; i < nodes; i++) {
      if (!alive[i]) continue;
      if (a < 0 || weight[i] < weight[a] ||
          (weight[i] == weight[a] && minsym[i] < minsym[a])) {
        b = a;
        a = i;
      } else if (b < 0 || weight[i] < weight[b] ||
                 (weight[i] == weight[b] && minsym[i] < minsym[b])) {
        b = i;
      }
    }
    alive[a] = alive[b] = 0;
    weight[nodes] = weight[a] + weight[b];
    minsym[nodes] = minsym[a] < minsym[b] ? minsym[a] : minsym[b];
    parent[nodes] = -1;
    alive[nodes] = 1;
    parent[a] = parent[b] = nodes;
    nodes++;
  }
  int longest = 0;
  for (int s = 0; s < 256; s++) {
    if (leaf_of[s] < 0) continue;
    int depth = 0;
    for (int v = leaf_of[s]; parent[v] >= 0; v = parent[v]) depth++;
    len[s] = (uint8_t)depth;
    if (depth > longest) longest = depth;
  }
  return longest;
}

/* ------------------------------------------------------------------------ */
/* Package-merge (Larmore & Hirschberg, 1990), the optimal length-limited
 * prefix code.  Coin-collector form: the leaves, sorted by (weight, symbol),
 * are the coins of the smallest denomination 2^-L.  For each larger
 * denomination, adjacent pairs of the previous list are packaged and merged
 * with the leaves (a leaf goes first when weights tie).  The cheapest 2m-2
 * items of the list for denomination 2^-1 are kept; a symbol's length is the
 * number of kept items that contain it.  Every item carries its full count
 * vector, so no bookkeeping trick is needed to read the lengths back.       */
typedef struct {
  uint64_t w;
  uint8_t cnt[256];
} pm_item;

int oracle_package_merge_lengths(const uint64_t hist[256], int max_len,
                                 uint8_t len[256]) {
  int sym[256];
  int m = 0;
  for (int s = 0; s < 256; s++) {
    len[s] = 0;
    if (hist[s] > 0) sym[m++] = s;
  }
  if (m == 0) return 0;
  if (m == 1) {
    len[sym[0]] = 1;
    return 1;
  }
  if (max_len < 31 && (1ull << max_len) < (uint64_t)m) return -1;
  /* insertion sort of the leaves by (weight, symbol) */
  for (int i = 1; i < m; i++) {
    int v = sym[i], j = i - 1;
    while (j >= 0 && (hist[sym[j]] > hist[v] ||
                      (hist[sym[j]] == hist[v] && sym[j] > v))) {
      sym[j + 1] = sym[j];
      j--;
    }
    sym[j + 1] = v;
  }
  pm_item *leaves = (pm_item *)calloc((size_t)(unsigned)m, sizeof(pm_item));
  pm_item *cur = (pm_item *)calloc(2 * (size_t)(unsigned)m, sizeof(pm_item));
  pm_item *next = (pm_item *)calloc(2 * (size_t)(unsigned)m, sizeof(pm_item));
  for (int i = 0; i < m; i++) {
    leaves[i].w = hist[sym[i]];
    leaves[i].cnt[sym[i]] = 1;
    cur[i] = leaves[i];
  }
  int cur_count = m;
  for (int level = max_len - 1; level >= 1; level--) {
    int packages = cur_count / 2;
    int li = 0, pi = 0, k = 0;
    while (li < m || pi < packages) {
      int take_leaf;
      if (li >= m) take_leaf = 0;
      else if (pi >= packages) take_leaf = 1;
      else take_leaf = leaves[li].w <= cur[2 * pi].w + cur[2 * pi + 1].w;
      if (take_leaf) {
        next[k++] = leaves[li++];
      } else {
        pm_item p;
        p.w = cur[2 * pi].w + cur[2 * pi + 1].w;
        for (int s = 0; s < 256; s++)
          p.cnt[s] = (uint8_t)(cur[2 * pi].cnt[s] + cur[2 * pi + 1].cnt[s]);
        next[k++] = p;
        pi++;
      }
    }
    pm_item *t = cur;
    cur = next;
    next = t;
    cur_count = k;
  }
  int longest = 0;
  for (int i = 0; i < 2 * m - 2; i++)
    for (int s = 0; s < 256; s++) len[s] = (uint8_t)(len[s] + cur[i].cnt[s]);
  for (int s = 0; s < 256; s++)
    if (len[s] > longest) longest = len[s];
  free(leaves);
  free(cur);
  free(next);
  return longest;
}

int oracle_code_lengths(const uint64_t hist[256], uint8_t len[256]) {
  int longest = oracle_huffman_lengths(hist, len);
  if (longest > ORACLE_MAX_LEN)
    longest = oracle_package_merge_lengths(hist, ORACLE_MAX_LEN, len);
  return longest;
}

/* ------------------------------------------------------------------------ */
/* Canonical code: symbols in order of (length, symbol value); the first
 * codeword is all zeros and each next one is the previous plus one, shifted
 * left by the growth in length (the assignment of RFC 1951 §3.2.2).         */
void oracle_canonical_codes(const uint8_t len[256], uint32_t codes[256]) {
  uint64_t code = 0;
  int prev_len = 0, first = 1;
  for (int s = 0; s < 256; s++) codes[s] = 0;
  for (int l = 1; l <= 255; l++) {
    for (int s = 0; s < 256; s++) {
      if (len[s] != l) continue;
      if (first) {
        code = 0;
        first = 0;
      } else {
        code = (code + 1) << (l - prev_len);
      }
      prev_len = l;
      codes[s] = (uint32_t)code;
    }
  }
}

/* ------------------------------------------------------------------------ */
/* Bit helpers: bit k of a byte array is bit (7 - k%8) of byte k/8.         */
static void put_bit(uint8_t *buf, uint64_t k, int bit) {
  if (bit) buf[k >> 3] |= (uint8_t)(0x80u >> (k & 7));
}
static int get_bit(const uint8_t *buf, uint64_t k) {
  return (buf[k >> 3] >> (7 - (k & 7))) & 1;
}

/* Does codeword `code` of length `l` equal the first l bits of the
 * `width`-bit string `bits`?                                                */
static int is_prefix(uint32_t code, int l, uint64_t bits, int width) {
  if (l > width) return 0;
  return (uint64_t)code == (bits >> (width - l));
}

/* ------------------------------------------------------------------------ */
/* Hierarchical lookup tables ("multi-level compact lookup tables",
 * "DFloat11 ... 三重编码机制" (ocdem.com) §2.2).  Every table has 256 entries
 * indexed by the next 8 bits of the stream.
 *
 *   table 0 (level 0), indexed by bits 0-7 of the window:
 *     the codewords that fit in those 8 bits, taken greedily from the
 *     start, at most three:  bits 0-23 = the exponents (first in bits 0-7,
 *     unused bytes zero), bits 24-27 = bits they use (1..8), bits 28-29 =
 *     how many (1..3).
 *     If the first codeword is longer than 8 bits: bits 0-23 = the number
 *     of the level-1 table for these 8 bits, all other bits zero.
 *   a level-k table (k = 1..3) for the 8k-bit prefix p, indexed by bits
 *   8k..8k+7: the codeword of length 8k+1..8k+8 that starts with the 8k+8
 *     bits p.i: bits 0-7 = exponent, bits 28-29 = 1;  or a pointer to the
 *     level-(k+1) table of prefix p.i as above.
 *   An entry no codeword matches is 0.
 * Tables are numbered level by level, by prefix value within a level.      */
typedef struct {
  int level;
  uint64_t prefix;
} lut_key;

static int find_table(const lut_key *keys, int count, int level,
                      uint64_t prefix) {
  for (int i = 0; i < count; i++)
    if (keys[i].level == level && keys[i].prefix == prefix) return i;
  return -1;
}

int oracle_build_luts(const uint8_t len[256], const uint32_t codes[256],
                      uint32_t *luts, int max_tables) {
  lut_key keys[1 + 3 * 256];
  int count = 1;
  keys[0].level = 0;
  keys[0].prefix = 0;
  /* enumerate tables: level k exists for every 8k-bit prefix of a codeword
   * longer than 8k bits; ascending prefix within a level                   */
  for (int k = 1; k <= 3; k++) {
    for (uint64_t p = 0; p < (1ull << (8 * k)); ) {
      /* find the smallest prefix >= p of a long codeword, by brute force
       * over the symbols (the prefix space at level 3 is too big to walk) */
      uint64_t best = UINT64_MAX;
      for (int s = 0; s < 256; s++) {
        if (len[s] <= 8 * k) continue;
        uint64_t pre = (uint64_t)codes[s] >> (len[s] - 8 * k);
        if (pre >= p && pre < best) best = pre;
      }
      if (best == UINT64_MAX) break;
      keys[count].level = k;
      keys[count].prefix = best;
      count++;
      p = best + 1;
    }
  }
  if (luts == NULL) return count;
  for (int t = 0; t < count && t < max_tables; t++) {
    int k = keys[t].level;
    for (int i = 0; i < 256; i++) {
      uint32_t entry = 0;
      if (k == 0) {
        /* greedy multi-codeword decode of the 8-bit string i */
        int used = 0, nsym = 0;
        uint32_t syms = 0;
        while (nsym < 3) {
          int found = -1;
          for (int s = 0; s < 256 && found < 0; s++) {
            if (len[s] == 0 || len[s] > 8 - used) continue;
            uint64_t rest = (uint64_t)i & ((1u << (8 - used)) - 1);
            if (is_prefix(codes[s], len[s], rest, 8 - used)) found = s;
          }
          if (found < 0) break;
          syms |= (uint32_t)found << (8 * nsym);
          nsym++;
          used += len[found];
        }
        if (nsym > 0) {
          entry = syms | ((uint32_t)used << 24) | ((uint32_t)nsym << 28);
        } else {
          int next = find_table(keys, count, 1, (uint64_t)i);
          if (next > 0) entry = (uint32_t)next;
        }
      } else {
        int width = 8 * k + 8;
        uint64_t q = (keys[t].prefix << 8) | (uint64_t)i;
        int found = -1;
        for (int s = 0; s < 256 && found < 0; s++) {
          if (len[s] <= 8 * k || len[s] > width) continue;
          if (is_prefix(codes[s], len[s], q, width)) found = s;
        }
        if (found >= 0) {
          entry = (uint32_t)found | (1u << 28);
        } else if (k < 3) {
          int next = find_table(keys, count, k + 1, q);
          if (next > 0) entry = (uint32_t)next;
        }
      }
      luts[(size_t)t * 256 + (size_t)i] = entry;
    }
  }
  return count;
}

/* ------------------------------------------------------------------------ */
/* Chunk gaps and block output positions, from their definitions:
 *   chunk c covers bits [8*C*c, 8*C*(c+1)); its gap is the distance from its
 *   first bit to the first codeword starting at or after it (or to the end
 *   of the stream when none does), 0 for chunks past the end;
 *   block b holds chunks [b*T, (b+1)*T); its output position is the number
 *   of codewords that start before its first bit; the last entry is n.     */
void oracle_metadata_from_starts(const uint64_t *starts, uint64_t n,
                                 uint64_t total_bits, uint32_t chunk_bytes,
                                 uint32_t threads_per_block,
                                 uint32_t num_blocks, uint8_t *gaps,
                                 uint32_t *block_out_pos) {
  uint64_t chunk_bits = 8ull * chunk_bytes;
  uint64_t chunks = (uint64_t)num_blocks * threads_per_block;
  uint64_t i = 0; /* first codeword with start >= chunk start */
  for (uint64_t c = 0; c < chunks; c++) {
    uint64_t begin = c * chunk_bits;
    while (i < n && starts[i] < begin) i++;
    if (begin >= total_bits) {
      gaps[c] = 0;
    } else {
      uint64_t first = i < n ? starts[i] : total_bits;
      if (first > total_bits) first = total_bits;
      gaps[c] = (uint8_t)(first - begin);
    }
  }
  uint64_t block_bits = chunk_bits * threads_per_block;
  uint64_t j = 0;
  for (uint32_t b = 0; b < num_blocks; b++) {
    while (j < n && starts[j] < (uint64_t)b * block_bits) j++;
    block_out_pos[b] = (uint32_t)j;
  }
  block_out_pos[num_blocks] = (uint32_t)n;
}

void oracle_pack_gaps(const uint8_t *gaps, uint64_t count, uint8_t *packed) {
  for (uint64_t c = 0; c < count; c++)
    for (int j = 0; j < 5; j++)
      put_bit(packed, 5 * c + (uint64_t)j, (gaps[c] >> (4 - j)) & 1);
}

/* ------------------------------------------------------------------------ */
int oracle_encode(const uint16_t *w, uint64_t n, uint32_t chunk_bytes,
                  uint32_t threads_per_block, oracle_format *f) {
  memset(f, 0, sizeof(*f));
  if (chunk_bytes < 4 || chunk_bytes > 28 || chunk_bytes % 4 != 0) return 1;
  if (threads_per_block == 0 || threads_per_block % 128 != 0) return 1;
  if (n >= (1ull << 32)) return 1;
  f->n = n;
  f->chunk_bytes = chunk_bytes;
  f->threads_per_block = threads_per_block;

  uint8_t *exps = (uint8_t *)malloc(n ? n : 1);
  f->sm_bytes = (n + 15) / 16 * 16;
  f->sign_mantissa = (uint8_t *)calloc(f->sm_bytes ? f->sm_bytes : 16, 1);
  oracle_split(w, n, exps, f->sign_mantissa);

  uint64_t hist[256];
  oracle_histogram(exps, n, hist);
  int longest = oracle_code_lengths(hist, f->code_lengths);
  f->max_len = (uint32_t)(longest > 0 ? longest : 0);
  oracle_canonical_codes(f->code_lengths, f->codes);

  uint64_t total = 0;
  for (uint64_t i = 0; i < n; i++) total += f->code_lengths[exps[i]];
  f->total_bits = total;
  uint64_t block_bits = 8ull * chunk_bytes * threads_per_block;
  f->num_blocks = (uint32_t)((total + block_bits - 1) / block_bits);
  uint64_t chunks = (uint64_t)f->num_blocks * threads_per_block;

  /* "codewords are packed one after another": MSB-first, element order */
  f->bitstream_bytes = chunks * chunk_bytes + 16;
  f->bitstream = (uint8_t *)calloc(f->bitstream_bytes, 1);
  uint64_t *starts = (uint64_t *)malloc((n ? n : 1) * sizeof(uint64_t));
  uint64_t pos = 0;
  for (uint64_t i = 0; i < n; i++) {
    int l = f->code_lengths[exps[i]];
    uint32_t c = f->codes[exps[i]];
    starts[i] = pos;
    for (int b = l - 1; b >= 0; b--) put_bit(f->bitstream, pos++, (c >> b) & 1);
  }

  f->gaps = (uint8_t *)calloc(chunks ? chunks : 1, 1);
  f->block_out_pos = (uint32_t *)calloc((size_t)f->num_blocks + 1, 4);
  oracle_metadata_from_starts(starts, n, total, chunk_bytes, threads_per_block,
                              f->num_blocks, f->gaps, f->block_out_pos);
  f->gaps_bytes = chunks * 5 / 8 + 16;
  f->gaps_packed = (uint8_t *)calloc(f->gaps_bytes, 1);
  oracle_pack_gaps(f->gaps, chunks, f->gaps_packed);

  /* codewords starting in each chunk, counted one start at a time, and in
     each group of 32 consecutive chunks */
  f->max_chunk_elems = 0;
  f->max_warp_elems = 0;
  f->chunk_counts_bytes = chunks + 16;
  f->chunk_counts = (uint8_t *)calloc(f->chunk_counts_bytes, 1);
  if (chunks) {
    uint32_t *per_chunk = (uint32_t *)calloc(chunks, 4);
    for (uint64_t i = 0; i < n; i++) per_chunk[starts[i] / (8ull * chunk_bytes)]++;
    for (uint64_t c = 0; c < chunks; c++) {
      if (per_chunk[c] > f->max_chunk_elems) f->max_chunk_elems = per_chunk[c];
      f->chunk_counts[c] = (uint8_t)per_chunk[c];
    }
    for (uint64_t g = 0; g < chunks; g += 32) {
      uint32_t sum = 0;
      for (uint64_t c = g; c < g + 32 && c < chunks; c++) sum += per_chunk[c];
      if (sum > f->max_warp_elems) f->max_warp_elems = sum;
    }
    free(per_chunk);
  }

  f->max_block_elems = 0;
  for (uint32_t b = 0; b < f->num_blocks; b++) {
    uint32_t e = f->block_out_pos[b + 1] - f->block_out_pos[b];
    if (e > f->max_block_elems) f->max_block_elems = e;
  }

  int tables = oracle_build_luts(f->code_lengths, f->codes, NULL, 0);
  f->num_luts = (uint32_t)tables;
  f->luts = (uint32_t *)calloc((size_t)tables * 256, 4);
  oracle_build_luts(f->code_lengths, f->codes, f->luts, tables);

  free(starts);
  free(exps);
  return 0;
}

void oracle_format_free(oracle_format *f) {
  free(f->bitstream);
  free(f->gaps);
  free(f->gaps_packed);
  free(f->block_out_pos);
  free(f->luts);
  free(f->sign_mantissa);
  free(f->chunk_counts);
  memset(f, 0, sizeof(*f));
}

/* ------------------------------------------------------------------------ */
/* Bit-serial canonical decode: grow the candidate codeword one bit at a time
 * until it lies in the range of codewords of its length.  Uses only the code
 * lengths, never the lookup tables.  The exponent is put back between the
 * sign bit and the mantissa ("DFloat11无损压缩技术" §2.1).                  */
uint64_t oracle_decode(const uint8_t *bitstream, uint64_t bitstream_bytes,
                       uint64_t start_bit, const uint8_t len[256],
                       const uint8_t *sm, uint64_t count, uint16_t *out,
                       uint64_t *starts) {
  uint32_t codes[256];
  oracle_canonical_codes(len, codes);
  /* per length: first codeword value, how many, and the symbols in order */
  uint64_t first_code[ORACLE_MAX_LEN + 1];
  int how_many[ORACLE_MAX_LEN + 1];
  int symbols[ORACLE_MAX_LEN + 1][256];
  for (int l = 0; l <= ORACLE_MAX_LEN; l++) {
    how_many[l] = 0;
    first_code[l] = 0;
  }
  for (int l = 1; l <= ORACLE_MAX_LEN; l++)
    for (int s = 0; s < 256; s++)
      if (len[s] == l) {
        if (how_many[l] == 0) first_code[l] = codes[s];
        symbols[l][how_many[l]++] = s;
      }
  uint64_t limit = bitstream_bytes * 8;
  uint64_t pos = start_bit;
  for (uint64_t i = 0; i < count; i++) {
    if (starts) starts[i] = pos;
    uint64_t code = 0;
    int sym = -1;
    for (int l = 1; l <= ORACLE_MAX_LEN; l++) {
      if (pos >= limit) return UINT64_MAX;
      code = (code << 1) | (uint64_t)get_bit(bitstream, pos++);
      if (how_many[l] > 0 && code >= first_code[l] &&
          code - first_code[l] < (uint64_t)how_many[l]) {
        sym = symbols[l][code - first_code[l]];
        break;
      }
    }
    if (sym < 0) return UINT64_MAX;
    uint16_t sign = (uint16_t)((sm[i] >> 7) & 1);
    uint16_t mantissa = (uint16_t)(sm[i] & 0x7F);
    out[i] = (uint16_t)((sign << 15) | ((uint16_t)sym << 7) | mantissa);
  }
  return pos;
}
