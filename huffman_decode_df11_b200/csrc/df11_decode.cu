// df11_decode.cu -- DF11 decode on sm_100a (B200) and the C ABI around it.
//
// One kernel, with persistent thread blocks: every thread block is assigned
// to one tensor of the launch (one wave, split by format blocks) and walks
// that tensor's format blocks (T chunks of C bitstream bytes) with a stride.
// It uses a decode table in shared memory: table 0 of the format and the
// code lengths with every exponent byte rotated right by one bit, and a
// derived table of 2^11 entries, each holding up to five whole codewords of
// the next 11 bits (built once per tensor by df11_table_kernel, or by every
// thread block when none is passed).  Deeper format tables (codewords longer
// than 8 bits) are read from global memory.
//
// df11_decode_ws_kernel: warp-specialised, one producer warp and T/32
// consumer warps per thread block, no block-wide barrier per format block.
// With chunk counts (the default path):
//   stage    the producer's lane 0 keeps two stage slots filled with bulk
//            copies (cp.async.bulk, no multicast) of a block's bitstream
//            slice, gap fields and chunk counts, and its sign/mantissa bytes
//            (or those go to per-warp buffers, or stay in L2), each slot
//            guarded by a full and an empty mbarrier.
//   locate   every consumer warp sums the stored chunk counts before its 32
//            chunks (warp reductions) and scans its lanes' counts: each lane
//            knows where its exponents go before it decodes.
//   decode   each lane walks its chunk once ("locate" and "reconstruct" of
//            "DFloat11重新定义LLM无损压缩的技术边界" (ocdem.com) §2.2 in one
//            pass) with a shifting bit window, stopping on its element
//            count; every lookup ORs its up to five exponents into the
//            warp's zeroed exponent region (two shared reductions).
//   output   the warp fuses 16 exponents with 16 sign/mantissa bytes per
//            lane and step (two selects, two byte permutes per four
//            elements), writes two 16-byte stores, re-zeroes what it read,
//            and writes the two ragged 16-element groups one element per
//            lane; then releases the slot.
//
// Without chunk counts (the format as the pages state it): each lane decodes
// its chunk into its own column of the warp's column area, counting
// ("locate"); the warps of the block post their totals and wait for each
// other (one bounded mbarrier wait per block); each lane then moves its
// bytes to their place in the warp's exponent region ("reconstruct"), and
// the output runs as above.
//
// Why the rotation: with e' = e>>1 | (e&1)<<7, the high byte of a BF16 word
// is (sm & 0x80) | (e' & 0x7F) and the low byte (e' & 0x80) | (sm & 0x7F), so
// four output words cost two bitwise selects and two byte permutes.
//
// Nothing here waits on another thread block of the same grid, so nothing
// can hang: the waits are on this block's own copies and barriers, bounded,
// reporting DF11_DEV_ERR_TIMEOUT, and (programmatic dependent launch) for
// the previous grid in the stream to complete.  Every data-dependent access is bounds-checked;
// inconsistent data are reported through the error word, never by a trap.
#include <cuda_runtime.h>

#include <atomic>
#include <cstdlib>
#include <cstdint>

#include "df11.h"
#include "df11_device_check.h"

namespace {

constexpr uint32_t kSpinLimit = 1u << 20;  // x ~1 us suspend hint: ~1 s
constexpr uint32_t kSuspendHintNs = 1000;
constexpr int kWideBits = 11;              // index bits of the derived table

struct KTensor {
  const uint8_t *bitstream;
  const uint8_t *gaps;
  const uint8_t *chunk_counts;  // NULL: count by decoding
  const uint32_t *block_out_pos;
  const uint32_t *luts;
  const uint8_t *code_lengths;
  const uint8_t *sign_mantissa;
  uint16_t *out;
  const void *decode_table;  // NULL: derived by every thread block
  uint64_t total_bits;
  uint32_t n;
  uint32_t num_blocks;
  uint32_t num_luts;
  uint32_t max_block_elems;
  uint32_t max_chunk_elems;
  uint32_t max_warp_elems;   // sizes the per-warp regions of the warp-specialised kernel
  uint32_t masked;     // longest codeword > kWideBits: bits past a region may be set
  uint32_t cta_begin;  // first thread block of this tensor
  uint32_t pad;
  // fused matrix-vector product (df11_decode_gemv): y[b][r] += sum_c W[r][c] x[b][c]
  // with W the decoded tensor as rows x cols, row-major
  const uint16_t *x;  // BF16 activations, batch rows of x_stride elements
  float *y;           // batch rows of y_stride floats
  uint32_t cols, batch, x_stride, y_stride;
  uint32_t interleave_log2;  // rows interleaved per 16-column group: 2^this (0: row-major)
  uint32_t pad2;
};

struct KBatch {
  KTensor t[DF11_MAX_BATCH];
  int32_t *err;
  int count;
  uint32_t cta_end;      // total thread blocks
  uint32_t stage_bytes;  // bytes of the exponent array
  uint32_t sm_bytes;     // sign/mantissa bytes per stage slot (warp-specialised kernel;
                         // 0: read from global memory)
  uint32_t spin_limit;   // polls of every bounded wait (kSpinLimit unless a test lowers it)
  uint32_t withhold;     // test hook: the producer issues no stage copy, so the
                         // consumers' waits run out (df11_test_withhold_copies)
  uint32_t col_bytes;    // without chunk counts: bytes of each warp's column area
  uint32_t col_cap;      // without chunk counts: most bytes a column takes (max_chunk_elems)
  uint32_t sub_bytes;    // room for a tensor's deeper tables in shared memory (0: read from
                         // global memory); tensors whose tables do not fit read them there
};

// ---- shared memory layout --------------------------------------------------
// [0,304)      mbarriers (full and empty per stage slot, per-warp copies, the
//              decode table's copy, the page layout's counted barriers)
// [304,560)    code lengths by rotated exponent
// [560,1584)   table 0 (rotated)
// [1584, ...)  wide table (2^WB x 8 bytes)
// then         the stage slots, the warps' exponent regions, their
//              sign/mantissa buffers and column areas (see the kernel)
constexpr uint32_t kOffLens = 304;
constexpr uint32_t kOffLut0 = 560;
constexpr uint32_t kOffWide = 1584;
constexpr uint32_t kWideBytes = 8u << kWideBits;
constexpr uint32_t kOffStages = kOffWide + kWideBytes;
// a decode table (df11_build_decode_table) is the image of [kOffLens, kOffStages)
static_assert(kOffStages - kOffLens == DF11_DECODE_TABLE_BYTES, "decode table layout");
static_assert(kOffLut0 - kOffLens == 256 && kOffWide - kOffLut0 == 1024, "decode table layout");

__device__ __forceinline__ uint32_t rot8x3(uint32_t v) {
  // rotate each of the low three bytes right by one bit
  return ((v >> 1) & 0x007F7F7Fu) | ((v << 7) & 0x00808080u);
}

__device__ __forceinline__ void report(int32_t *err, int32_t code) {
  if (err) atomicCAS(err, 0, code);
}

__device__ __forceinline__ uint32_t smem_addr(const void *p) {
  return (uint32_t)__cvta_generic_to_shared(p);
}

// Shared-memory accesses through 32-bit shared-window addresses.
__device__ __forceinline__ uint2 lds64(uint32_t a) {
  uint2 v;
  asm volatile("ld.shared.v2.u32 {%0, %1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(a) : "memory");
  return v;
}
__device__ __forceinline__ uint32_t lds32(uint32_t a) {
  uint32_t v;
  asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(a) : "memory");
  return v;
}
__device__ __forceinline__ void sts32(uint32_t a, uint32_t v) {
  asm volatile("st.shared.u32 [%0], %1;" ::"r"(a), "r"(v) : "memory");
}
__device__ __forceinline__ uint4 lds128(uint32_t a) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "r"(a)
               : "memory");
  return v;
}
__device__ __forceinline__ void sts128_zero(uint32_t a) {
  asm volatile("st.shared.v4.u32 [%0], {%1, %1, %1, %1};" ::"r"(a), "r"(0u) : "memory");
}
__device__ __forceinline__ uint32_t lds8(uint32_t a) {
  uint32_t v;
  asm volatile("ld.shared.u8 %0, [%1];" : "=r"(v) : "r"(a) : "memory");
  return v;
}
__device__ __forceinline__ void sts8_zero(uint32_t a) {
  asm volatile("st.shared.u8 [%0], %1;" ::"r"(a), "h"((unsigned short)0) : "memory");
}
__device__ __forceinline__ void red_or32(uint32_t a, uint32_t v) {
  asm volatile("red.shared.or.b32 [%0], %1;" ::"r"(a), "r"(v) : "memory");
}

// Programmatic dependent launch: a launch of this library may start while
// the previous kernel in the stream is still running.  Each thread block
// lets the next launch start once it has queued its last block
// (launch_dependents; the next grid starts when every block has, so its
// thread blocks take the places of this grid's as they finish, and set up
// their tables and first blocks meanwhile), and waits for the previous grid
// to finish, and its writes to be visible, only before its first store to
// the output (wait): the output buffer may be one that the previous kernel
// wrote or still reads, while the compressed inputs are read-only.  Letting
// the next grid start at once measured slower on sequences of different
// launches.  Without the launch attribute both are no-ops.
__device__ __forceinline__ void pdl_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
               : "memory");
}

__device__ __forceinline__ void bulk_g2s(uint32_t dst, const void *src, uint32_t bytes,
                                         uint32_t bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
      "l"(src), "r"(bytes), "r"(bar)
      : "memory");
}

// Bounded wait for phase `parity` of an mbarrier: at most `limit` polls,
// each suspending for up to about a microsecond; false on timeout.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity,
                                          uint32_t limit = kSpinLimit) {
  for (uint32_t i = 0; i < limit; ++i) {
    uint32_t done;
    asm volatile(
        "{\n .reg .pred p;\n"
        " mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n"
        " selp.u32 %0, 1, 0, p;\n}\n"
        : "=r"(done)
        : "r"(bar), "r"(parity), "r"(kSuspendHintNs)
        : "memory");
    if (done) return true;
  }
  return false;
}

// One codeword at the start of a 32-bit window through the format's tables:
// the (rotated) exponent and the codeword length; false for an invalid one.
__device__ __forceinline__ bool decode_one(uint32_t win, const uint32_t *__restrict__ lut0,
                                           const uint8_t *__restrict__ lens,
                                           const uint32_t *sub, uint32_t num_luts,
                                           uint32_t &sym, uint32_t &len) {
  const uint32_t e = lut0[win >> 24];
  if ((e >> 24) & 15u) {
    sym = e & 0xFFu;
  } else {
    uint32_t t = e & 0xFFFFFFu, f = 0;
#pragma unroll 1
    for (int level = 1; level <= 3; ++level) {
      if (t == 0 || t >= num_luts) break;
      const uint32_t e2 = sub[(t - 1) * 256 + ((win >> (24 - 8 * level)) & 0xFFu)];
      if (e2 >> 28) {
        f = e2;
        break;
      }
      t = e2 & 0xFFFFFFu;
    }
    if (f == 0) return false;
    sym = rot8x3(f & 0xFFu);
  }
  len = lens[sym];
  return len != 0;
}

// Table 0 of the format and the code lengths into shared memory, every
// exponent byte rotated right by one bit (code lengths indexed by the
// rotated exponent).
__device__ __forceinline__ void load_tables(int tid, int nthreads, const uint32_t *luts,
                                            const uint8_t *code_lengths, uint32_t *lut0_s,
                                            uint8_t *lens_s) {
  for (int i = tid; i < 256; i += nthreads) {
    uint32_t e = luts[i] & 0x3FFFFFFFu;
    if ((e >> 24) & 15u) e = (e & 0xFF000000u) | rot8x3(e);
    lut0_s[i] = e;
    lens_s[((uint32_t)i >> 1) | (((uint32_t)i & 1u) << 7)] = code_lengths[i];
  }
}

// Derived table: entry i holds the codewords that lie wholly inside the WB
// bits i, at most MS of them: x = the first four exponents (first in bits
// 0-7), y = bits used | 8 * count << 16 | fifth exponent << 24, so that one
// add of y's low 24 bits moves both the bit position and the output bit
// offset of a packed (bit, output bit) register, and the five exponent
// bytes shift into two words with two funnel shifts.
// y == 0: the first codeword is longer than WB bits (or invalid) and takes
// the slow path.
template <int T, int MS>
__device__ void build_wide(uint2 *wide, const uint32_t *lut0, const uint8_t *lens,
                           const uint32_t *sub, uint32_t num_luts) {
  static_assert(MS >= 1 && MS <= 5, "at most five exponent bytes per entry");
  for (uint32_t i = threadIdx.x; i < (1u << kWideBits); i += T) {
    const uint32_t bits = i << (32 - kWideBits);
    uint32_t used = 0, n = 0;
    uint64_t syms = 0;
    while (n < MS) {
      const uint32_t win = bits << used;
      const uint32_t e = lut0[win >> 24];
      const uint32_t ns = e >> 28;
      if (((e >> 24) & 15u) == 0) {
        uint32_t s, l;
        if (!decode_one(win, lut0, lens, sub, num_luts, s, l) || used + l > kWideBits) break;
        syms |= (uint64_t)s << (8 * n);
        ++n;
        used += l;
        continue;
      }
      bool stop = ns == 0;
      for (uint32_t j = 0; j < ns && n < MS; ++j) {
        const uint32_t s = (e >> (8 * j)) & 0xFFu, l = lens[s];
        if (l == 0 || used + l > kWideBits) {
          stop = true;
          break;
        }
        syms |= (uint64_t)s << (8 * n);
        ++n;
        used += l;
      }
      if (stop || used >= kWideBits) break;
    }
    wide[i] = n ? make_uint2((uint32_t)syms, used | (n << 19) | ((uint32_t)(syms >> 32) << 24))
                : make_uint2(0, 0);
  }
}

// 32 stream bits starting at bit `pos` of a chunk held as big-endian words
// (the chunk and the 4 bytes after it).  Codeword starts lie below 8*C (the
// next chunk's gap covers the rest), so for C = 8 the window comes from words
// (0,1) or (1,2).
template <int C>
__device__ __forceinline__ uint32_t window(const uint32_t (&w)[C / 4 + 1], uint32_t pos) {
  if (C == 4) return __funnelshift_l(w[1], w[0], pos);
  if (C == 8) {
    const bool up = pos & 32u;
    return __funnelshift_l(up ? w[2] : w[1], up ? w[1] : w[0], pos);
  }
  const uint32_t k = pos >> 5;
  uint32_t hi = w[0], lo = w[1];
#pragma unroll
  for (int j = 1; j < C / 4; ++j)
    if (k == (uint32_t)j) {
      hi = w[j];
      lo = w[j + 1];
    }
  return __funnelshift_l(lo, hi, pos);
}

// The same walk when the thread's output place is known before it decodes
// (the format's chunk count): exponents go straight into the block's
// (zeroed) exponent array from byte d on.  Every lookup ORs its up to five
// bytes into the word that holds the next byte and the word after it (the
// part that spills over; zero when nothing does), which also merges the
// words a thread shares with its neighbours.  `pk` packs the bit position
// (bits 0-15) with the bit offset of the next byte (bits 16-31, so d stays
// below 8192); `limit` is the last word the thread may touch.  Returns the
// number of codewords decoded.
template <int T, int C, bool MASKED>
__device__ __forceinline__ uint32_t decode_direct(const uint32_t (&w)[C / 4 + 1], int start,
                                                  const int end, uint32_t wide,
                                                  const uint32_t *__restrict__ lut0,
                                                  const uint8_t *__restrict__ lens,
                                                  const uint32_t *sub, uint32_t num_luts,
                                                  uint32_t ex, uint32_t d, uint32_t limit,
                                                  int &bad) {
  uint32_t pk = (uint32_t)start | (d << 19);
  while ((int)(pk & 0xFFFFu) < end) {
    const uint32_t win = window<C>(w, pk & 0xFFFFu);
    uint2 e = lds64(wide + ((win >> (32 - kWideBits)) << 3));
    if (e.y == 0 || (!MASKED && (int)(e.y & 0xFFFFu) > end - (int)(pk & 0xFFFFu))) {
      uint32_t sym, len;
      if (!decode_one(win, lut0, lens, sub, num_luts, sym, len)) {
        bad = DF11_DEV_ERR_TABLE;
        return 0;
      }
      e = make_uint2(sym, len | (8u << 16));
    }
    const uint32_t sh = (pk >> 16) & 24u;
    const uint32_t a = min(ex + ((pk >> 21) << 2), limit);
    red_or32(a, e.x << sh);
    red_or32(a + 4u, __funnelshift_l(e.x, e.y >> 24, sh));  // with the fifth exponent
    pk += e.y & 0x00FFFFFFu;
  }
  if ((int)(pk & 0xFFFFu) != end) bad = DF11_DEV_ERR_OVERRUN;
  return (pk >> 19) - d;
}

// The direct walk for masked streams when the chunk's count is known, with
// fewer operations per lookup:
//   - the chunk's bits sit in a shifting window of NW words (next bit at the
//     top of s[0]), moved on by funnel shifts whose amount is the entry's
//     second word itself: funnel shifts use only its low five bits, which
//     hold the bits used (at most kWideBits here), and ones come in from the
//     right, so the stream stays masked past its last word;
//   - the loop ends on the element count, not the bit position: it runs
//     while the output bit offset (bits 16-31 of `pk`, bit position in bits
//     0-15) is below 8*(d+cnt).  Every iteration emits at least one element,
//     so a corrupt stream stops within cnt lookups and writes at most four
//     bytes past the thread's range (the last lookup's five bytes stay in two
//     words), which the region's slack absorbs: no clamp on the address.  Bits past `end` are ones, so
//     on valid data the last lookup stops exactly at `end` (checked after).
// Returns the number of elements written.
template <int C>
__device__ __forceinline__ uint32_t decode_counted(const uint32_t (&w)[C / 4 + 1], int start,
                                                   const int end, uint32_t wide,
                                                   const uint32_t *__restrict__ lut0,
                                                   const uint8_t *__restrict__ lens,
                                                   const uint32_t *sub, uint32_t num_luts,
                                                   uint32_t ex, uint32_t d, uint32_t cnt,
                                                   int &bad) {
  constexpr int NW = C / 4 + 1;
  uint32_t s[NW];
#pragma unroll
  for (int j = 0; j < NW - 1; ++j) s[j] = __funnelshift_l(w[j + 1], w[j], (uint32_t)start);
  s[NW - 1] = __funnelshift_l(0xFFFFFFFFu, w[NW - 1], (uint32_t)start);
  uint32_t pk = (uint32_t)start | ((8u * d) << 16);
  const uint32_t lim = (8u * (d + cnt)) << 16;
  while (pk < lim) {
    uint2 e = lds64(wide + ((s[0] >> (32 - kWideBits)) << 3));
    if (e.y == 0) {
      // rare: a codeword longer than the derived table's index.  Shift by
      // half its length here and the rest below (both at most 16 bits, in
      // the funnel shifts' range).
      uint32_t sym, len;
      if (!decode_one(s[0], lut0, lens, sub, num_luts, sym, len)) {
        bad = DF11_DEV_ERR_TABLE;
        return 0;
      }
      const uint32_t half = len >> 1;
#pragma unroll
      for (int j = 0; j < NW - 1; ++j) s[j] = __funnelshift_l(s[j + 1], s[j], half);
      s[NW - 1] = __funnelshift_l(0xFFFFFFFFu, s[NW - 1], half);
      pk += half;
      e = make_uint2(sym, (len - half) | (8u << 16));
    }
    const uint32_t sh = pk >> 16;  // funnel shifts use sh & 31: the bit offset in the word
    const uint32_t a = ex + ((pk >> 21) << 2);
    red_or32(a, __funnelshift_l(0u, e.x, sh));
    red_or32(a + 4u, __funnelshift_l(e.x, e.y >> 24, sh));  // with the fifth exponent
#pragma unroll
    for (int j = 0; j < NW - 1; ++j) s[j] = __funnelshift_l(s[j + 1], s[j], e.y);
    s[NW - 1] = __funnelshift_l(0xFFFFFFFFu, s[NW - 1], e.y);
    pk += e.y & 0x00FFFFFFu;
  }
  // a count that disagrees with the stream ends the walk short of `end`
  // (too small) or past it (too large, or a corrupt stream)
  const int pos = (int)(pk & 0xFFFFu);
  if (pos != end) bad = pos < end ? DF11_DEV_ERR_COUNT : DF11_DEV_ERR_OVERRUN;
  return (pk >> 19) - d;
}

// The walk of the format as the pages state it (no chunk counts): a thread
// learns where its output goes only once every warp of the block has
// counted, so it decodes into its own column of the warp's column area
// (its byte j at word (j/4)*32 + lane: the lanes' reductions never share a
// bank) and counts.  The window moves as in decode_counted; the walk stops
// at the chunk's end bit, or when `cap` bytes (the format's
// max_chunk_elems) are written, beyond which the data are inconsistent.
// Unmasked streams (every codeword within the derived table's index) check
// each entry against the end.  Returns the number of codewords.
template <int C, bool MASKED>
__device__ __forceinline__ uint32_t decode_column(const uint32_t (&w)[C / 4 + 1], int start,
                                                  const int end, uint32_t wide,
                                                  const uint32_t *__restrict__ lut0,
                                                  const uint8_t *__restrict__ lens,
                                                  const uint32_t *sub, uint32_t num_luts,
                                                  uint32_t col, uint32_t cap, int &bad) {
  constexpr int NW = C / 4 + 1;
  uint32_t s[NW];
#pragma unroll
  for (int j = 0; j < NW - 1; ++j) s[j] = __funnelshift_l(w[j + 1], w[j], (uint32_t)start);
  s[NW - 1] = __funnelshift_l(0xFFFFFFFFu, w[NW - 1], (uint32_t)start);
  uint32_t pk = (uint32_t)start;          // bit position | 8 * bytes written << 16
  const uint32_t lim = (8u * cap) << 16;  // pk < lim: fewer than cap bytes written
  while ((int)(pk & 0xFFFFu) < end && pk < lim) {
    uint2 e = lds64(wide + ((s[0] >> (32 - kWideBits)) << 3));
    if (e.y == 0 || (!MASKED && (int)(e.y & 0xFFFFu) > end - (int)(pk & 0xFFFFu))) {
      // a codeword longer than the derived table's index, or (unmasked
      // streams) an entry that runs past the end: one codeword through the
      // format's own tables, the window moved by half its length here
      uint32_t sym, len;
      if (!decode_one(s[0], lut0, lens, sub, num_luts, sym, len)) {
        bad = DF11_DEV_ERR_TABLE;
        return 0;
      }
      const uint32_t half = len >> 1;
#pragma unroll
      for (int j = 0; j < NW - 1; ++j) s[j] = __funnelshift_l(s[j + 1], s[j], half);
      s[NW - 1] = __funnelshift_l(0xFFFFFFFFu, s[NW - 1], half);
      pk += half;
      e = make_uint2(sym, (len - half) | (8u << 16));
    }
    const uint32_t sh = pk >> 16;
    const uint32_t a = col + ((pk >> 21) << 7);
    red_or32(a, __funnelshift_l(0u, e.x, sh));
    red_or32(a + 128u, __funnelshift_l(e.x, e.y >> 24, sh));
#pragma unroll
    for (int j = 0; j < NW - 1; ++j) s[j] = __funnelshift_l(s[j + 1], s[j], e.y);
    s[NW - 1] = __funnelshift_l(0xFFFFFFFFu, s[NW - 1], e.y);
    pk += e.y & 0x00FFFFFFu;
  }
  const int pos = (int)(pk & 0xFFFFu);
  if (pos != end) bad = pos < end ? DF11_DEV_ERR_COUNT : DF11_DEV_ERR_OVERRUN;
  return pk >> 19;
}

// A lane's `cnt` exponent bytes, from its column (word k at col + 128k),
// into the warp's element-order region from byte d on: whole words are
// stored, the first and last (shared with the neighbouring lanes' ranges)
// ORed into the zeroed region.  Column bytes past cnt are zero.  Each column
// word is zeroed once read, for the next block.
__device__ __forceinline__ void column_to_region(uint32_t col, uint32_t cnt, uint32_t region,
                                                 uint32_t d) {
  if (!cnt) return;
  const uint32_t r8 = (d & 3u) * 8u;
  const uint32_t words = ((d & 3u) + cnt + 3u) >> 2;  // destination words
  const uint32_t held = (cnt + 3u) >> 2;              // column words with bytes
  uint32_t prev = 0, dst = region + (d & ~3u);
  for (uint32_t j = 0; j < words; ++j, dst += 4u) {
    uint32_t cur = 0;
    if (j < held) {
      cur = lds32(col + 128u * j);
      sts32(col + 128u * j, 0u);
    }
    const uint32_t v = __funnelshift_l(prev, cur, r8);  // bytes 4j - (d & 3) ..
    if (j == 0 || j + 1 == words) red_or32(dst, v);
    else sts32(dst, v);
    prev = cur;
  }
}

// four sign/mantissa bytes and four rotated exponents -> four BF16 words:
// the four low bytes (E0 | mantissa) and the four high bytes (sign | E7..E1)
// are two bitwise selects, then two byte permutes interleave them
__device__ __forceinline__ uint2 fuse4(uint32_t sm4, uint32_t er4) {
  const uint32_t lo = (sm4 & 0x7F7F7F7Fu) | (er4 & 0x80808080u);
  const uint32_t hi = (er4 & 0x7F7F7F7Fu) | (sm4 & 0x80808080u);
  return make_uint2(__byte_perm(lo, hi, 0x5140), __byte_perm(lo, hi, 0x7362));
}

__device__ __forceinline__ uint16_t fuse1(uint32_t sm, uint32_t er) {
  const uint32_t lo = (sm & 0x7Fu) | (er & 0x80u), hi = (er & 0x7Fu) | (sm & 0x80u);
  return (uint16_t)__byte_perm(lo, hi, 0x3340);
}

__device__ __forceinline__ void bulk_prefetch_l2(const void *src, uint32_t bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(src), "r"(bytes) : "memory");
}

// ---------------------------------------------------------------------------
// Warp-specialised decode for tensors that carry chunk counts.
//
// With the counts in shared memory every warp can work out where its output
// goes on its own, so the thread block needs no block-wide barrier per format
// block.  One producer warp (one lane) keeps kWsStages stage slots filled
// (bitstream slice, gap fields, chunk counts, positions and the block's
// sign/mantissa bytes), each guarded by a "full" mbarrier (completed by the
// bulk copies) and an "empty" mbarrier (one arrival per consumer warp when it
// is done with the block).  Each of the T/32 consumer warps, per format block:
//   - sums the block's chunk counts before its own chunks and over the whole
//     block (two warp reductions over T bytes) and scans its lanes' counts;
//   - decodes straight into its private exponent region (zeroed; words shared
//     by two lanes merged with OR) and checks every count;
//   - writes its own output range from shared memory: whole 16-element
//     groups with 16-byte stores, the two ragged edge groups one element per
//     lane; then releases the slot.
constexpr int kWsStages = 2;

// Where the output of the warp-specialised kernel finds a block's sign/
// mantissa bytes: in the stage slot (one bulk copy per block by the
// producer), in global memory (L2-prefetched by the producer), or in a
// buffer of the warp's own, filled by one bulk copy of the warp's output
// range that the warp issues before it decodes.  The host takes the first
// that keeps the most thread blocks resident.
enum SmMode { kSmSlot = 0, kSmGlobal = 1, kSmWarp = 2 };

// ---- fused matrix-vector product -------------------------------------------
// a BF16 word (low 16 bits) widened to fp32, exactly
__device__ __forceinline__ float bf16_lo(uint32_t u) { return __uint_as_float(u << 16); }

// sum over 16 elements of w * x, both BF16, two per word, in fp32: the
// mixed-precision fused multiply-add of PTX takes the BF16 halves of a
// register as they are (no widening instructions); its product is exact
// and the sum rounds once, as fmaf on the widened values would
__device__ __forceinline__ float dot16(const uint32_t (&w)[8], const uint4 &x0, const uint4 &x1) {
  const uint32_t xv[8] = {x0.x, x0.y, x0.z, x0.w, x1.x, x1.y, x1.z, x1.w};
  float a = 0.f, b = 0.f;
#pragma unroll
  for (int k = 0; k < 8; ++k)
    asm("{\n\t.reg .b16 wl, wh, xl, xh;\n\t"
        "mov.b32 {wl, wh}, %2;\n\tmov.b32 {xl, xh}, %3;\n\t"
        "fma.rn.f32.bf16 %0, wl, xl, %0;\n\tfma.rn.f32.bf16 %1, wh, xh, %1;\n\t}"
        : "+f"(a), "+f"(b)
        : "r"(w[k]), "r"(xv[k]));
  return a + b;
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, o);
  return v;
}

// Add the warp's partial sums p (lane l: row `row`, only where `act`) into
// y[row].  When the active lanes' rows take at most two values, each row
// takes one warp sum and one atomic add; otherwise (matrices narrower than
// 512 columns) every active lane adds its own.
__device__ __forceinline__ void warp_row_add(float p, uint32_t row, bool act, float *y,
                                             int lane) {
  if (!__any_sync(0xFFFFFFFFu, act)) return;
  const uint32_t r0 = __reduce_min_sync(0xFFFFFFFFu, act ? row : 0xFFFFFFFFu);
  const uint32_t r1 = __reduce_max_sync(0xFFFFFFFFu, act ? row : 0u);
  if (r0 == r1) {
    const float s = warp_sum(act ? p : 0.f);
    if (lane == 0) atomicAdd(y + r0, s);
  } else if (__all_sync(0xFFFFFFFFu, !act || row == r0 || row == r1)) {
    const float s0 = warp_sum(act && row == r0 ? p : 0.f);
    const float s1 = warp_sum(act && row == r1 ? p : 0.f);
    if (lane == 0) {
      atomicAdd(y + r0, s0);
      atomicAdd(y + r1, s1);
    }
  } else if (act) {
    atomicAdd(y + row, p);
  }
}

// y = W x: the outputs of a launch's products cleared by one small kernel
// before it (the product kernel adds into them only after its
// dependent-launch wait, which waits for this grid to complete)
struct ClearArgs {
  float *y[DF11_MAX_BATCH];
  uint32_t rows[DF11_MAX_BATCH], batch[DF11_MAX_BATCH], stride[DF11_MAX_BATCH];
  int count;
};

__global__ void __launch_bounds__(256) clear_rows_kernel(const __grid_constant__ ClearArgs c) {
  asm volatile("griddepcontrol.wait;" ::: "memory");  // the previous kernel may still read y
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  for (int t = 0; t < c.count; ++t) {
    const uint64_t all = (uint64_t)c.rows[t] * c.batch[t];
    for (uint64_t i = blockIdx.x * 256ull + threadIdx.x; i < all; i += (uint64_t)gridDim.x * 256) {
      const uint64_t b = i / c.rows[t], r = i - b * c.rows[t];
      c.y[t][b * c.stride[t] + r] = 0.f;
    }
  }
}

template <int T, int C>
struct WsLayout {
  static constexpr uint32_t bits_bytes = T * C + 16;
  static constexpr uint32_t gaps_bytes = T * 5 / 8 + 16;
  static constexpr uint32_t counts_bytes = T;
  static constexpr uint32_t meta_bytes = 16;
  // the block's sign/mantissa bytes follow (KBatch::sm_bytes of them)
  static constexpr uint32_t head_bytes = bits_bytes + gaps_bytes + counts_bytes + meta_bytes;
  static_assert(head_bytes % 16 == 0, "alignment");
};

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

template <int T, int C, int SM, bool COUNTS>
__device__ __forceinline__ void ws_issue(const KTensor &tk, uint32_t b, uint8_t *slot,
                                         uint32_t full, uint32_t sm_capacity) {
  using L = WsLayout<T, C>;
  const uint32_t P0 = tk.block_out_pos[b], P1 = tk.block_out_pos[b + 1];
  const uint32_t expected = P1 - P0;
  // a warp's exponents fit its region whatever the block: every chunk count
  // is checked against max_chunk_elems before decoding
  const bool ok = P1 >= P0 && P1 <= tk.n && expected <= tk.max_block_elems &&
                  (SM != kSmSlot || expected + 32 <= sm_capacity);
  // bits of the stream inside this block: all of them but in the last block
  const uint64_t bit0 = (uint64_t)b * (T * C * 8);
  const uint32_t valid_bits = tk.total_bits - bit0 < (uint64_t)(T * C * 8)
                                  ? (uint32_t)(tk.total_bits - bit0)
                                  : 0xFFFFFFFFu;
  *reinterpret_cast<uint4 *>(slot + L::bits_bytes + L::gaps_bytes + L::counts_bytes) =
      make_uint4(P0, P1, ok ? 1u : 0u, valid_bits);
  if (!ok) {
    mbar_arrive_expect_tx(full, 0);
    return;
  }
  const uint32_t sm_begin = P0 & ~15u;
  const uint32_t sm_bytes = ((P1 + 15u) & ~15u) - sm_begin;
  mbar_arrive_expect_tx(full, L::bits_bytes + L::gaps_bytes + (COUNTS ? L::counts_bytes : 0u) +
                                  (SM == kSmSlot ? sm_bytes : 0u));
  bulk_g2s(smem_addr(slot), tk.bitstream + (size_t)b * (T * C), L::bits_bytes, full);
  bulk_g2s(smem_addr(slot + L::bits_bytes), tk.gaps + (size_t)b * (T * 5 / 8), L::gaps_bytes,
           full);
  if (COUNTS)
    bulk_g2s(smem_addr(slot + L::bits_bytes + L::gaps_bytes), tk.chunk_counts + (size_t)b * T,
             L::counts_bytes, full);
  if (SM == kSmGlobal) {
    if (sm_bytes) bulk_prefetch_l2(tk.sign_mantissa + sm_begin, sm_bytes);
  } else if (SM == kSmSlot && sm_bytes) {
    bulk_g2s(smem_addr(slot + L::head_bytes), tk.sign_mantissa + sm_begin, sm_bytes, full);
  }
}

// Where 16-element group q of the stream (q = element / 16) sits in the
// rows x cols weight: with R = 2^s rows interleaved, the stream holds, per
// block of R rows and per 16-column group, the R rows' 16 elements one after
// another (R = 1: row-major).  Returns the row; *cg = the column group.
__device__ __forceinline__ uint32_t group_row(uint32_t q, uint32_t groups_per_row, uint32_t s,
                                              uint32_t *cg) {
  const uint32_t t = q >> s, r = q & ((1u << s) - 1u);
  const uint32_t rb = t / groups_per_row;
  *cg = t - rb * groups_per_row;
  return (rb << s) + r;
}

// The whole 16-element groups [g_begin, g_end) of a warp's range into
// y += W x (batch rows nb <= NB): each lane sums its groups of one row in
// registers and hands the sums over (warp sums per row, one atomic add each)
// when it moves to another row, and at the end.  With R rows interleaved
// a lane keeps one row of each block of R rows and the lanes that share
// a column group read the same activations.
template <int SM, int NB>
__device__ __forceinline__ void gemv_groups(const KTensor &tk, int lane, uint32_t base,
                                            uint32_t g_begin, uint32_t g_end, uint32_t sm,
                                            uint32_t region, const uint8_t *smg, uint32_t cols,
                                            uint32_t nb) {
  const uint32_t s = tk.interleave_log2, gpr = cols >> 4;  // column groups per row
  const uint32_t step = 32u >> s;                         // column groups per iteration
  uint32_t cg;
  uint32_t row = group_row((base >> 4) + g_begin + (uint32_t)lane, gpr, s, &cg);
  float acc[NB];
#pragma unroll
  for (int bi = 0; bi < NB; ++bi) acc[bi] = 0.f;
  uint32_t acc_row = row;
  bool has = false;
  for (uint32_t gg = g_begin; gg < g_end; gg += 32) {
    const uint32_t g = gg + (uint32_t)lane;
    const bool act = g < g_end;
    const bool moved = act && has && row != acc_row;
    if (__any_sync(0xFFFFFFFFu, moved)) {
#pragma unroll
      for (int bi = 0; bi < NB; ++bi) {
        if ((uint32_t)bi < nb) {
          warp_row_add(acc[bi], acc_row, moved, tk.y + (size_t)bi * tk.y_stride, lane);
          acc[bi] = moved ? 0.f : acc[bi];
        }
      }
    }
    if (act) {
      const uint4 sv = SM == kSmGlobal ? __ldg(reinterpret_cast<const uint4 *>(smg) + g)
                                       : lds128(sm + 16u * g);
      const uint4 rv = lds128(region + 16u * g);
      sts128_zero(region + 16u * g);
      const uint2 a = fuse4(sv.x, rv.x), c = fuse4(sv.y, rv.y);
      const uint2 e2 = fuse4(sv.z, rv.z), f = fuse4(sv.w, rv.w);
      const uint32_t wv[8] = {a.x, a.y, c.x, c.y, e2.x, e2.y, f.x, f.y};
#pragma unroll
      for (int bi = 0; bi < NB; ++bi) {
        if ((uint32_t)bi < nb) {
          const uint4 *xp =
              reinterpret_cast<const uint4 *>(tk.x + (size_t)bi * tk.x_stride + 16u * cg);
          acc[bi] += dot16(wv, __ldg(xp), __ldg(xp + 1));
        }
      }
      acc_row = row;
      has = true;
    }
    // the next group of this lane: `step` column groups on, in the same rows
    // or, past the row's end, in the next block of rows
    cg += step;
    while (cg >= gpr) {
      cg -= gpr;
      row += 1u << s;
    }
  }
#pragma unroll
  for (int bi = 0; bi < NB; ++bi)
    if ((uint32_t)bi < nb) warp_row_add(acc[bi], acc_row, has, tk.y + (size_t)bi * tk.y_stride, lane);
}

// Register budget from the resident thread blocks the shared memory allows:
// five at 8-byte chunks, at most four from 16 bytes on (more registers there
// measured about 1% faster) and for the fused matrix-vector product.
//
// COUNTS = false decodes the format as the pages state it (no chunk
// counts): each lane decodes into its own column and counts, the warps of a
// block exchange their totals (one bounded mbarrier wait per block), and
// each lane then moves its bytes into the warp's element-order region, from
// which the output runs as with counts.
template <int T, int C, int SM, bool GEMV, bool COUNTS = true>
__global__ void __launch_bounds__(T + 32, (T + 32) <= 160 ? 8
                                          : ((C >= 16 || GEMV) && T == 256 ? 4 : 1280 / T))
    df11_decode_ws_kernel(const __grid_constant__ KBatch kb) {
  using L = WsLayout<T, C>;
  constexpr int NW = C / 4 + 1;
  constexpr int CONSUMERS = T / 32;
  extern __shared__ __align__(128) uint8_t smem[];
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem);  // full[S], empty[S]
  uint8_t *lens_s = smem + kOffLens;
  uint32_t *lut0_s = reinterpret_cast<uint32_t *>(smem + kOffLut0);
  uint2 *wide_s = reinterpret_cast<uint2 *>(smem + kOffWide);
  uint8_t *stages = smem + kOffStages;
  const uint32_t slot_bytes = L::head_bytes + kb.sm_bytes;
  uint8_t *regions = stages + kWsStages * slot_bytes;
  // kSmWarp: each warp's sign/mantissa buffer (region-sized) follows the regions
  uint8_t *warp_sm = regions + CONSUMERS * kb.stage_bytes;
  // without counts: each warp's column area (kb.col_bytes) follows
  uint8_t *columns = warp_sm + (SM == kSmWarp ? CONSUMERS * kb.stage_bytes : 0u);
  // the tensor's deeper tables (codewords longer than 8 bits), when room was left
  uint32_t *subs_s = reinterpret_cast<uint32_t *>(columns + CONSUMERS * kb.col_bytes);

  int ti = 0;
  for (int i = 1; i < kb.count; ++i)
    if (blockIdx.x >= kb.t[i].cta_begin) ti = i;
  const KTensor &tk = kb.t[ti];
  const uint32_t ctas = (ti + 1 < kb.count ? kb.t[ti + 1].cta_begin : kb.cta_end) - tk.cta_begin;
  const uint32_t first = blockIdx.x - tk.cta_begin;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  if (first >= tk.num_blocks) return;

  // barriers: full[S], empty[S], per-warp (kSmWarp), tables, and without
  // counts counted[S] (every consumer warp has posted its total)
  const uint32_t tbar = smem_addr(&bars[2 * kWsStages + 16]);
  if (tid == 0) {
    for (int i = 0; i < kWsStages; ++i) {
      mbar_init(smem_addr(&bars[i]), 1);
      mbar_init(smem_addr(&bars[kWsStages + i]), CONSUMERS);
      if (!COUNTS) mbar_init(smem_addr(&bars[2 * kWsStages + 17 + i]), CONSUMERS);
    }
    if (SM == kSmWarp)
      for (int i = 0; i < CONSUMERS; ++i) mbar_init(smem_addr(&bars[2 * kWsStages + i]), 1);
    mbar_init(tbar, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();
  // the producer queues the decode table and the first blocks before
  // anything else, so that they arrive while the tables are set up
  const bool have_table = tk.decode_table != nullptr;
  // the tensor's deeper tables come into shared memory with its decode table
  // when the launch left room for them
  const uint32_t sub_bytes = have_table && tk.num_luts > 1 &&
                                     (tk.num_luts - 1) * 1024u <= kb.sub_bytes
                                 ? (tk.num_luts - 1) * 1024u
                                 : 0u;
  uint32_t issued = 0;
  if (warp == CONSUMERS && lane == 0) {
    if (have_table) {
      mbar_arrive_expect_tx(tbar, DF11_DECODE_TABLE_BYTES + sub_bytes);
      bulk_g2s(smem_addr(lens_s), tk.decode_table, DF11_DECODE_TABLE_BYTES, tbar);
      if (sub_bytes) bulk_g2s(smem_addr(subs_s), tk.luts + 256, sub_bytes, tbar);
    }
    if (!kb.withhold)
      for (uint32_t b = first; b < tk.num_blocks && issued < kWsStages; b += ctas, ++issued)
        ws_issue<T, C, SM, COUNTS>(tk, b, stages + issued * slot_bytes,
                                   smem_addr(&bars[issued]), kb.sm_bytes);
  }
  // deeper tables: in shared memory when they came with the decode table
  const uint32_t *sub = sub_bytes ? subs_s : tk.luts + 256;
  for (uint32_t i = tid; i < CONSUMERS * kb.stage_bytes / 16; i += T + 32)
    reinterpret_cast<uint4 *>(regions)[i] = make_uint4(0, 0, 0, 0);
  if (!COUNTS)
    for (uint32_t i = tid; i < CONSUMERS * kb.col_bytes / 16; i += T + 32)
      reinterpret_cast<uint4 *>(columns)[i] = make_uint4(0, 0, 0, 0);
  bool tables_ok = true;
  if (have_table) {
    tables_ok = mbar_wait(tbar, 0, kb.spin_limit);
  } else {
    load_tables(tid, T + 32, tk.luts, tk.code_lengths, lut0_s, lens_s);
    __syncthreads();
    build_wide<T + 32, 5>(wide_s, lut0_s, lens_s, sub, tk.num_luts);
  }
  if (!__syncthreads_and(tables_ok)) {
    if (tid == 0) report(kb.err, DF11_DEV_ERR_TIMEOUT);
    return;
  }

  if (warp == CONSUMERS) {  // producer
    if (lane == 0) {
      uint32_t k = issued;
      if (!kb.withhold) {
        for (uint32_t b = first + issued * ctas; b < tk.num_blocks; b += ctas, ++k) {
          const uint32_t s = k % kWsStages, par = (k / kWsStages) & 1u;
          if (!mbar_wait(smem_addr(&bars[kWsStages + s]), par ^ 1u, kb.spin_limit)) {
            report(kb.err, DF11_DEV_ERR_TIMEOUT);
            break;
          }
          ws_issue<T, C, SM, COUNTS>(tk, b, stages + s * slot_bytes, smem_addr(&bars[s]),
                                     kb.sm_bytes);
        }
      }
      pdl_launch_dependents();  // every block of this thread block is queued
      // Stay until the last copy into each slot has landed, so that no copy
      // is in flight into this thread block's shared memory when it exits,
      // even when consumers gave up waiting (bounded as well).
      for (uint32_t j = k > kWsStages ? k - kWsStages : 0; j < k; ++j)
        if (!mbar_wait(smem_addr(&bars[j % kWsStages]), (j / kWsStages) & 1u, kb.spin_limit))
          report(kb.err, DF11_DEV_ERR_TIMEOUT);
    }
    return;
  }

  const uint32_t region = smem_addr(regions + warp * kb.stage_bytes);
  uint8_t *region_p = regions + warp * kb.stage_bytes;
  const uint32_t wide = smem_addr(wide_s);
  const uint32_t wsm = smem_addr(warp_sm + warp * kb.stage_bytes);  // kSmWarp
  const uint32_t wbar = smem_addr(&bars[2 * kWsStages + warp]);     // kSmWarp
  uint32_t wph = 0;  // kSmWarp: copies issued so far (phase parity)
  bool waited = false;  // for the previous grid (programmatic dependent launch)
  uint32_t k = 0;
  for (uint32_t b = first; b < tk.num_blocks; b += ctas, ++k) {
    const uint32_t s = k % kWsStages, par = (k / kWsStages) & 1u;
    const uint8_t *slot = stages + s * slot_bytes;
    if (!__all_sync(0xFFFFFFFFu, mbar_wait(smem_addr(&bars[s]), par, kb.spin_limit))) {
      if (lane == 0) report(kb.err, DF11_DEV_ERR_TIMEOUT);
      return;  // whole warp
    }
    // everything this warp needs from the slot, into registers (32-bit
    // shared-window addresses throughout)
    const uint32_t slot_sa = smem_addr(slot);
    const uint32_t counts_sa = slot_sa + L::bits_bytes + L::gaps_bytes;
    const uint4 m = lds128(counts_sa + L::counts_bytes);
    const uint32_t P0 = m.x, P1 = m.y, expected = P1 - P0;
    const uint32_t release = smem_addr(&bars[kWsStages + s]);
    int start, end;
    {
      const uint32_t bit = 5u * (uint32_t)tid;
      const uint32_t ga = slot_sa + L::bits_bytes + 4u * (bit >> 5);
      const uint32_t v = __funnelshift_l(__byte_perm(lds32(ga + 4u), 0, 0x0123),
                                         __byte_perm(lds32(ga), 0, 0x0123), bit);
      start = (int)(v >> 27);
      end = C * 8 + (int)((v >> 22) & 31u);
    }
    uint32_t w[NW];
#pragma unroll
    for (int j = 0; j < NW; ++j)
      w[j] = __byte_perm(lds32(slot_sa + (uint32_t)tid * C + 4u * j), 0, 0x0123);
    uint32_t cnt, before, incl, warp_total;
    int bad = 0;
    if constexpr (COUNTS) {
      uint32_t lsum;
      if (T == 128) {
        lsum = __dp4a(lds32(counts_sa + 4u * lane), 0x01010101u, 0u);
      } else if (T == 256) {
        const uint2 v = lds64(counts_sa + 8u * lane);
        lsum = __dp4a(v.x, 0x01010101u, __dp4a(v.y, 0x01010101u, 0u));
      } else {
        const uint4 v = lds128(counts_sa + 16u * lane);
        lsum = __dp4a(v.x, 0x01010101u, __dp4a(v.y, 0x01010101u,
                      __dp4a(v.z, 0x01010101u, __dp4a(v.w, 0x01010101u, 0u))));
      }
      cnt = lds8(counts_sa + tid);
      before = __reduce_add_sync(0xFFFFFFFFu, lane < warp * 32 / (T / 32) ? lsum : 0u);
      const uint32_t total = __reduce_add_sync(0xFFFFFFFFu, lsum);
      if (!m.z || total != expected ||
          __any_sync(0xFFFFFFFFu, cnt > tk.max_chunk_elems)) {
        if (warp == 0 && lane == 0)
          report(kb.err, m.z ? (total != expected ? DF11_DEV_ERR_COUNT : DF11_DEV_ERR_CAPACITY)
                             : DF11_DEV_ERR_CAPACITY);
        __syncwarp();
        if (lane == 0) mbar_arrive(release);
        continue;
      }
    }
    if (m.w != 0xFFFFFFFFu) {  // the block that holds the end of the stream
      const uint32_t b0 = (uint32_t)tid * (C * 8);
      if (b0 >= m.w) start = end = 0;
      else if ((uint32_t)end > m.w - b0) end = (int)(m.w - b0);
    }
    if (tk.masked) {  // ones from bit `end` on; mostly only the last word has any
      if (end >= C * 8) {
        w[NW - 1] |= __funnelshift_rc(0xFFFFFFFFu, 0u, (uint32_t)(end - C * 8));
      } else {
#pragma unroll
        for (int j = 0; j < NW; ++j)
          w[j] |= __funnelshift_rc(0xFFFFFFFFu, 0u, (uint32_t)max(end - 32 * j, 0));
      }
    }
    const uint32_t col = smem_addr(columns + warp * kb.col_bytes) + 4u * lane;  // !COUNTS
    if constexpr (!COUNTS) {
      // locate: decode into the lane's column, counting
      cnt = 0;
      if (m.z)
        cnt = tk.masked ? decode_column<C, true>(w, start, end, wide, lut0_s, lens_s, sub,
                                                 tk.num_luts, col, kb.col_cap, bad)
                        : decode_column<C, false>(w, start, end, wide, lut0_s, lens_s, sub,
                                                  tk.num_luts, col, kb.col_cap, bad);
    }
    incl = cnt;
#pragma unroll
    for (int dd = 1; dd < 32; dd <<= 1) {
      const uint32_t v = __shfl_up_sync(0xFFFFFFFFu, incl, dd);
      if (lane >= dd) incl += v;
    }
    warp_total = __shfl_sync(0xFFFFFFFFu, incl, 31);
    if constexpr (!COUNTS) {
      // scan across the block: every warp posts its total (bit 31: a lane
      // found bad data) in the slot's unused chunk-count bytes, then waits
      // (bounded) until all have
      const bool warp_bad = __any_sync(0xFFFFFFFFu, bad != 0);
      const uint32_t cbar = smem_addr(&bars[2 * kWsStages + 17 + s]);
      if (lane == 0) {
        sts32(counts_sa + 4u * warp, warp_total | (warp_bad ? 0x80000000u : 0u));
        mbar_arrive(cbar);
      }
      if (!__all_sync(0xFFFFFFFFu, mbar_wait(cbar, par, kb.spin_limit))) {
        if (lane == 0) report(kb.err, DF11_DEV_ERR_TIMEOUT);
        return;  // whole warp
      }
      const uint32_t v = lane < CONSUMERS ? lds32(counts_sa + 4u * lane) : 0u;
      const uint32_t any_bad = __reduce_or_sync(0xFFFFFFFFu, v) >> 31;
      before = __reduce_add_sync(0xFFFFFFFFu, lane < warp ? v & 0x7FFFFFFFu : 0u);
      const uint32_t total = __reduce_add_sync(0xFFFFFFFFu, v & 0x7FFFFFFFu);
      const bool block_bad = !m.z || any_bad || total != expected;
      if (block_bad || warp_total > tk.max_warp_elems) {
        if (bad) {
          report(kb.err, bad);  // the lane's own finding
        } else if (lane == 0 && !any_bad) {
          if (!block_bad)  // this warp's range would not fit its region
            report(kb.err, DF11_DEV_ERR_CAPACITY);
          else if (warp == 0)
            report(kb.err, !m.z || total == expected ? DF11_DEV_ERR_CAPACITY : DF11_DEV_ERR_COUNT);
        }
        for (uint32_t j = 0; j < kb.col_bytes / 128u; ++j) sts32(col + 128u * j, 0u);
        __syncwarp();
        if (lane == 0) mbar_arrive(release);
        continue;
      }
    } else {
      if (warp_total > tk.max_warp_elems) {  // would not fit the region (uniform)
        if (lane == 0) report(kb.err, DF11_DEV_ERR_CAPACITY);
        __syncwarp();
        if (lane == 0) mbar_arrive(release);
        continue;
      }
    }
    const uint32_t G0 = P0 + before;            // first element of this warp
    const uint32_t head = G0 & 15u, span = head + warp_total;
    const uint32_t d = head + incl - cnt;       // my first byte in the region
    // kSmGlobal: the sign/mantissa bytes of the lane's first whole group of
    // the output, loaded now so that they arrive from L2 during the walk (or
    // the move into the region) instead of stalling the output
    uint4 sv_first = make_uint4(0, 0, 0, 0);
    if (SM == kSmGlobal && !GEMV) {
      const uint32_t g0 = (head ? 1u : 0u) + (uint32_t)lane;
      if (g0 < (span >> 4))
        sv_first = __ldg(reinterpret_cast<const uint4 *>(tk.sign_mantissa + (G0 & ~15u)) + g0);
    }
    // kSmWarp: the warp's sign/mantissa bytes, elements [G0 & ~15,
    // round16(G0 + warp_total)), inside the block's range, copied while it
    // decodes (or, without counts, while it moves its bytes into place);
    // every path below waits for the copy before going on
    const uint32_t wsm_bytes = SM == kSmWarp ? (span + 15u) & ~15u : 0u;
    if (SM == kSmWarp && wsm_bytes && lane == 0) {
      mbar_arrive_expect_tx(wbar, wsm_bytes);
      bulk_g2s(wsm, tk.sign_mantissa + (G0 & ~15u), wsm_bytes, wbar);
    }
    if constexpr (COUNTS) {
      uint32_t got;
      if (tk.masked) {
        got = decode_counted<C>(w, start, end, wide, lut0_s, lens_s, sub, tk.num_luts, region,
                                d, cnt, bad);
      } else {
        const uint32_t limit = region + ((d + (cnt ? cnt : 1u) - 1u) & ~3u);
        got = decode_direct<T, C, false>(w, start, end, wide, lut0_s, lens_s, sub, tk.num_luts,
                                         region, d, limit, bad);
      }
      if (!bad && got != cnt) bad = DF11_DEV_ERR_COUNT;
    } else {
      // reconstruct: the column's bytes to their place in element order
      column_to_region(col, cnt, region, d);
    }
    if (SM == kSmWarp && wsm_bytes) {
      const bool landed = __all_sync(0xFFFFFFFFu, mbar_wait(wbar, wph & 1u, kb.spin_limit));
      ++wph;
      if (!landed) {
        if (lane == 0) report(kb.err, DF11_DEV_ERR_TIMEOUT);
        return;  // whole warp; the buffer may still be written
      }
    }
    if (COUNTS && __any_sync(0xFFFFFFFFu, bad != 0)) {
      if (bad) report(kb.err, bad);
      __syncwarp();
      // a counted walk over corrupt data may write up to 7 bytes past `span`
      for (uint32_t i = lane; i < (span + 8u + 15u) >> 4; i += 32)
        reinterpret_cast<uint4 *>(region_p)[i] = make_uint4(0, 0, 0, 0);
      __syncwarp();
      if (lane == 0) mbar_arrive(release);
      continue;
    }
    __syncwarp();
    if (!waited) {
      pdl_wait();
      waited = true;
    }

    // output of this warp's elements [G0, G0 + warp_total); its sign/mantissa
    // bytes are in the slot, which starts at element P0 & ~15.  Group g (16
    // elements) is at byte 16g of the region and of `sm` and at element 16g of
    // `out`.
    const uint32_t base = G0 & ~15u;
    uint16_t *out = tk.out + base;
    const uint8_t *smg = tk.sign_mantissa + base;  // kSmGlobal
    const uint32_t sm = SM == kSmWarp   ? wsm
                        : SM == kSmSlot ? smem_addr(slot + L::head_bytes) + (base - (P0 & ~15u))
                                        : 0u;
    const uint32_t g_begin = head ? 1u : 0u, g_end = span >> 4;
    if constexpr (GEMV) {
      // the decoded weights go into y += W x instead of to memory: per
      // 16-element group (within one row, since cols is a multiple of 16)
      // one partial sum per batch row, summed over the warp per row
      const uint32_t cols = tk.cols, nb = tk.batch;
      if (nb == 1)
        gemv_groups<SM, 1>(tk, lane, base, g_begin, g_end, sm, region, smg, cols, nb);
      else
        gemv_groups<SM, DF11_GEMV_MAX_BATCH>(tk, lane, base, g_begin, g_end, sm, region, smg,
                                             cols, nb);
      // every lane is done with the whole groups (it may have read one that
      // a ragged lane zeroes next) before the ragged groups are touched
      __syncwarp();
      if (span) {
        // the elements outside whole groups, one per lane: lanes 0-15 the
        // first group, 16-31 the last one when it is another group
        const uint32_t last_g = (span - 1) >> 4;
        const uint32_t i = ((uint32_t)lane & 15u) + (lane >> 4 ? last_g << 4 : 0u);
        const bool act = i >= head && i < span && (i < (g_begin << 4) || i >= (g_end << 4)) &&
                         (lane < 16 || last_g != 0);
        const uint32_t wbits = act ? fuse1(SM == kSmGlobal ? (uint32_t)__ldg(smg + i) : lds8(sm + i),
                                           lds8(region + i))
                                   : 0u;
        sts8_zero(region + i);  // the loop zeroed whole groups; this does the rest
        uint32_t cgi;
        const uint32_t r = group_row((base + i) >> 4, cols >> 4, tk.interleave_log2, &cgi);
        const uint32_t ci = 16u * cgi + (i & 15u);
        const uint32_t half = __ballot_sync(0xFFFFFFFFu, act) >> (lane & 16);
        for (uint32_t bi = 0; bi < nb; ++bi) {
          float p = act ? bf16_lo(wbits) * bf16_lo(tk.x[(size_t)bi * tk.x_stride + ci]) : 0.f;
#pragma unroll
          for (int o = 8; o; o >>= 1) p += __shfl_xor_sync(0xFFFFFFFFu, p, o);
          if ((lane & 15) == 0 && (half & 0xFFFFu)) atomicAdd(tk.y + (size_t)bi * tk.y_stride + r, p);
        }
      }
    } else {
      {
        uint32_t g = g_begin + (uint32_t)lane;
        uint32_t sa_sm = sm + 16u * g, sa_rg = region + 16u * g;
        uint4 *o = reinterpret_cast<uint4 *>(out) + 2u * g;
        const uint4 *sp = reinterpret_cast<const uint4 *>(smg) + g;
        uint4 sv_next = sv_first;  // kSmGlobal: one group ahead
        for (; g < g_end; g += 32, sa_sm += 512u, sa_rg += 512u, o += 64, sp += 32) {
          uint4 sv;
          if (SM == kSmGlobal) {
            sv = sv_next;
            if (g + 32 < g_end) sv_next = __ldg(sp + 32);
          } else {
            sv = lds128(sa_sm);
          }
          const uint4 rv = lds128(sa_rg);
          sts128_zero(sa_rg);  // leave the region zeroed for the next block
          const uint2 a = fuse4(sv.x, rv.x), c = fuse4(sv.y, rv.y);
          const uint2 e2 = fuse4(sv.z, rv.z), f = fuse4(sv.w, rv.w);
          o[0] = make_uint4(a.x, a.y, c.x, c.y);
          o[1] = make_uint4(e2.x, e2.y, f.x, f.y);
        }
      }
      // every lane is done with the whole groups (it may have read one that
      // a ragged lane zeroes next) before the ragged groups are touched
      __syncwarp();
      if (span) {
        // the elements outside whole groups [g_begin, g_end), one per lane:
        // lanes 0-15 take the first group, 16-31 the last one (the same group
        // when there is only one: both lanes then write the same value)
        const uint32_t i = ((uint32_t)lane & 15u) + (lane >> 4 ? ((span - 1) >> 4) << 4 : 0u);
        if (i >= head && i < span && (i < (g_begin << 4) || i >= (g_end << 4)))
          out[i] = fuse1(SM == kSmGlobal ? (uint32_t)__ldg(smg + i) : lds8(sm + i),
                         lds8(region + i));
        sts8_zero(region + i);  // the loop zeroed whole groups; this does the rest
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(release);  // slot free for refill
  }
}

// ---------------------------------------------------------------------------
// Fused decode and matrix product on the tensor cores (df11_decode_gemm):
// y[b][r] (+)= sum_c W[r][c] x[b][c] for a batch of BF16 activation rows,
// with W decoded inside the kernel and never written to memory.
//
// W is encoded with 128 rows interleaved per 16 columns (interleave 128), so
// that the stream holds, per block of 128 rows and per 16-column group, a
// 128 x 16 tile: the A operand of one tcgen05.mma of M = 128, K = 16.  The
// work is cut into tiles: every thread block takes an equal, contiguous
// range of the launch's tiles, in pieces of at most one row block.  Per
// piece:
//   - the producer warp stages the format blocks that overlap the piece (as
//     the decode kernel does; a block at a piece's edge is staged for each
//     of the two pieces);
//   - the consumer warps decode them as the decode kernel does (lanes whose
//     codewords all lie outside the piece skip their walk) and write the
//     piece's BF16 weights, 16 bytes at a time, into a ring of A tiles in
//     shared memory, in the canonical K-major layout without swizzle (8-row
//     x 16-byte core matrices; K halves 128 bytes apart, 8-row groups 256
//     bytes apart); then they post the block (mbarrier);
//   - one MMA warp loads the activation tile of every completed weight tile
//     (N = batch rounded up to 16 rows x 16 columns, zero rows past the
//     batch; fetched with cp.async one block ahead) into the same layout and
//     issues tcgen05.mma into one of two (one at batches over 64) fp32
//     accumulators in tensor memory
//     (128 lanes x N columns), then commits to an mbarrier that the writers
//     of the ring wait on before they overwrite tiles;
//   - consumer warps 0-3 (one per 32 tensor-memory lanes) move a finished
//     piece's accumulator to registers (tcgen05.ld) and add it to y with
//     fp32 atomics, while the next piece accumulates in the other one.
// Every wait is bounded (DF11_DEV_ERR_TIMEOUT); no warp leaves early, so
// the MMA warp frees the tensor memory after a final barrier in every case.
constexpr int kGemmM = 128;                    // rows of a weight tile (MMA M)
constexpr uint32_t kGemmTileBytes = 128u * 16u * 2u;  // one 128 x 16 BF16 tile

struct GBatch {
  KTensor t[DF11_MAX_BATCH];                  // decode fields, x, y, cols, batch, strides
  uint32_t tile_begin[DF11_MAX_BATCH + 1];    // first tile of each tensor; [count] = all tiles
  int32_t *err;
  int count;
  uint32_t ctas;         // thread blocks of the launch
  uint32_t stage_bytes;  // bytes of each consumer warp's exponent region
  uint32_t ring;         // A tile (and activation tile) slots
  uint32_t n_mma;        // N of every MMA: the batch rounded up to 16
  uint32_t tmem_cols;    // tensor-memory columns allocated (accs accumulators)
  uint32_t accs;         // accumulators: 2 (a finished piece's is moved out while the
                         // next accumulates) when they fit beside three others, else 1
  uint32_t spin_limit;
};

// A piece of a thread block's tile range: the tiles from global tile t on
// that lie in one row block of one tensor (and below t_end): its tensor, its
// element range [u0, u1) of that tensor's stream, its row block, its first
// 16-column group and its tiles.
struct GUnit {
  int ti;
  uint32_t u0, u1, rb, cg0, tiles;
};

__device__ __forceinline__ GUnit gemm_piece(const GBatch &gb, uint32_t t, uint32_t t_end) {
  GUnit g;
  g.ti = 0;
  for (int i = 1; i < gb.count; ++i)
    if (t >= gb.tile_begin[i]) g.ti = i;
  const KTensor &tk = gb.t[g.ti];
  const uint32_t tpr = tk.cols >> 4;  // tiles per row block
  const uint32_t lt = t - gb.tile_begin[g.ti];
  g.rb = lt / tpr;
  g.cg0 = lt - g.rb * tpr;
  g.tiles = min(tpr - g.cg0, t_end - t);
  g.u0 = lt * 2048u;  // the tiles of a tensor follow one another in its stream
  g.u1 = g.u0 + g.tiles * 2048u;
  return g;
}

// Format blocks overlapping [u0, u1): the last block starting at or before
// u0 and the first block whose range reaches u1 (block_out_pos is the
// positions' ascending table; a corrupt table gives some range inside
// [0, num_blocks), which the per-block checks then flag).
__device__ __forceinline__ void gemm_blocks(const KTensor &tk, uint32_t u0, uint32_t u1,
                                            uint32_t &bf, uint32_t &bl) {
  uint32_t lo = 0, hi = tk.num_blocks;  // bf: largest b with pos[b] <= u0
  while (hi - lo > 1) {
    const uint32_t mid = (lo + hi) >> 1;
    if (__ldg(tk.block_out_pos + mid) <= u0) lo = mid;
    else hi = mid;
  }
  bf = lo;
  lo = bf;
  hi = tk.num_blocks - 1;  // bl: smallest b >= bf with pos[b + 1] >= u1
  while (lo < hi) {
    const uint32_t mid = (lo + hi) >> 1;
    if (__ldg(tk.block_out_pos + mid + 1) >= u1) hi = mid;
    else lo = mid + 1;
  }
  bl = lo;
}

// Byte offset of weight (r, c) of a 128 x 16 tile in the canonical K-major
// layout without swizzle.
__device__ __forceinline__ uint32_t umma_offset(uint32_t r, uint32_t c) {
  return (r >> 3) * 256u + (c >> 3) * 128u + (r & 7u) * 16u + (c & 7u) * 2u;
}

// Shared-memory matrix descriptor: K-major, no swizzle, leading (K-half)
// and stride (8-row group) byte offsets, version 1.
__device__ __forceinline__ uint64_t umma_desc(uint32_t addr, uint32_t lbo, uint32_t sbo) {
  return (uint64_t)((addr >> 4) & 0x3FFFu) | ((uint64_t)((lbo >> 4) & 0x3FFFu) << 16) |
         ((uint64_t)((sbo >> 4) & 0x3FFFu) << 32) | (1ull << 46);
}

__device__ __forceinline__ void fence_proxy_async() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

template <int T, int C>
__global__ void __launch_bounds__(T + 64, 4) df11_decode_gemm_kernel(const __grid_constant__ GBatch gb) {
  static_assert(T == 256, "eight consumer warps, eight chunk counts per lane");
  using L = WsLayout<T, C>;
  constexpr int NW = C / 4 + 1;
  constexpr int CONSUMERS = T / 32;
  constexpr int PRODUCER = CONSUMERS, MMA = CONSUMERS + 1;
  static_assert(CONSUMERS >= 4, "four consumer warps read the accumulator");
  extern __shared__ __align__(1024) uint8_t gsmem[];
  uint64_t *bars = reinterpret_cast<uint64_t *>(gsmem);
  // barriers: full[2] 0-1, empty[2] 2-3, table, staged[2], mma_done[2],
  // d_free[2]; the tensor-memory address after them
  constexpr int kTableBar = 4, kStaged = kTableBar + 1,
                kMmaDone = kStaged + 2, kDFree = kMmaDone + 2, kBars = kDFree + 2;
  static_assert(kBars * 8 + 8 <= (int)kOffLens, "barriers fit below the tables");
  uint32_t *taddr_s = reinterpret_cast<uint32_t *>(gsmem + kBars * 8);
  uint8_t *lens_s = gsmem + kOffLens;
  uint32_t *lut0_s = reinterpret_cast<uint32_t *>(gsmem + kOffLut0);
  uint2 *wide_s = reinterpret_cast<uint2 *>(gsmem + kOffWide);
  uint8_t *stages = gsmem + kOffStages;
  uint8_t *regions = stages + 2 * L::head_bytes;
  const uint32_t ring_a = smem_addr(gsmem) +
                          ((kOffStages + 2 * L::head_bytes + CONSUMERS * gb.stage_bytes + 1023u) &
                           ~1023u);
  const uint32_t x_tile_bytes = gb.n_mma * 32u;
  const uint32_t ring_x = ring_a + gb.ring * kGemmTileBytes;

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  // this thread block's tiles: an equal share of all tiles of the launch
  const uint32_t ub = (uint32_t)(((uint64_t)blockIdx.x * gb.tile_begin[gb.count]) / gb.ctas);
  const uint32_t ue = (uint32_t)(((uint64_t)(blockIdx.x + 1) * gb.tile_begin[gb.count]) / gb.ctas);
  auto bar = [&](int i) { return smem_addr(&bars[i]); };

  if (tid == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(bar(i), 1);
      mbar_init(bar(2 + i), CONSUMERS);
      mbar_init(bar(kStaged + i), CONSUMERS);
      mbar_init(bar(kMmaDone + i), 1);
      mbar_init(bar(kDFree + i), 4);
    }
    mbar_init(bar(kTableBar), 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == MMA) {  // tensor memory: gb.accs accumulators of n_mma columns
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_addr(taddr_s)),
                 "r"(gb.tmem_cols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  for (uint32_t i = tid; i < CONSUMERS * gb.stage_bytes / 16; i += T + 64)
    reinterpret_cast<uint4 *>(regions)[i] = make_uint4(0, 0, 0, 0);
  for (uint32_t i = tid; i < gb.ring * x_tile_bytes / 16; i += T + 64)  // activation rows past
    sts128_zero(ring_x + 16u * i);                                    // the batch stay zero
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *taddr_s;
  int32_t *err = gb.err;
  bool failed = false;  // this thread gave up on a wait: it skips to the end

  // a tensor's decode table: fetched by the producer before the first piece
  // of each tensor in this thread block's range (a range is contiguous, so
  // rarely), waited for by everyone through the table barrier's phases
  uint32_t k = 0;  // block instances so far (stage slot k & 1)

  if (warp == PRODUCER) {
    if (lane == 0) {
      int cur_t = -1;
      uint32_t tphase = 0;
      for (uint32_t u = ub; u < ue && !failed;) {
        const GUnit g = gemm_piece(gb, u, ue);
        u += g.tiles;
        const KTensor &tk = gb.t[g.ti];
        if (g.ti != cur_t) {
          // the table is read by the consumers of the previous piece until
          // they release its last block: wait for every slot to be free
          for (uint32_t j = k > 2 ? k - 2 : 0; j < k && !failed; ++j)
            failed = !mbar_wait(bar(2 + (j & 1)), (j >> 1) & 1u, gb.spin_limit);
          if (failed) break;
          mbar_arrive_expect_tx(bar(kTableBar), DF11_DECODE_TABLE_BYTES);
          bulk_g2s(smem_addr(lens_s), tk.decode_table, DF11_DECODE_TABLE_BYTES, bar(kTableBar));
          cur_t = g.ti;
          ++tphase;
        }
        uint32_t bf, bl;
        gemm_blocks(tk, g.u0, g.u1, bf, bl);
        for (uint32_t b = bf; b <= bl; ++b, ++k) {
          if (k >= 2 && !mbar_wait(bar(2 + (k & 1)), ((k >> 1) - 1) & 1u, gb.spin_limit)) {
            failed = true;
            break;
          }
          // the block's sign/mantissa bytes stay in global memory, prefetched to L2
          ws_issue<T, C, kSmGlobal, true>(tk, b, stages + (k & 1) * L::head_bytes, bar(k & 1), 0);
        }
      }
      if (failed) report(err, DF11_DEV_ERR_TIMEOUT);
      pdl_launch_dependents();
      // no copy of this thread block in flight when it ends
      for (uint32_t j = k > 2 ? k - 2 : 0; j < k; ++j)
        if (!mbar_wait(bar(j & 1), (j >> 1) & 1u, gb.spin_limit)) report(err, DF11_DEV_ERR_TIMEOUT);
      if (tphase && !mbar_wait(bar(kTableBar), (tphase - 1) & 1u, gb.spin_limit))
        report(err, DF11_DEV_ERR_TIMEOUT);
    }
  } else if (warp == MMA) {
    // idesc: D fp32, A and B BF16, both K-major, N = n_mma, M = 128
    const uint32_t idesc = (1u << 4) | (1u << 7) | (1u << 10) | ((gb.n_mma >> 3) << 17) |
                           ((uint32_t)(kGemmM >> 4) << 24);
    pdl_wait();  // the activations may come from the previous kernel
    uint32_t t_run = 0;  // tiles of this thread block's pieces so far (ring position)
    uint32_t seg = 0, seg_tiles = 0;  // pieces so far (accumulator seg % accs), their tiles
    int prev_ti = -1;
    uint32_t prev_rb = 0;
    // The activation tile of column group cg, rows below the batch (the
    // rows past it stay zero from the start), into ring slot `slot`: K half
    // h of row n at byte h * 16 * n_mma + 16 n, by 16-byte asynchronous
    // copies that land while the consumers decode.
    auto fetch_x = [&](const KTensor &tk, uint32_t cg, uint32_t slot) {
      const uint32_t xs = ring_x + slot * x_tile_bytes;
      for (uint32_t p = lane; p < 2u * tk.batch; p += 32) {
        const uint32_t n = p >> 1, h = p & 1u;
        asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(xs + h * 16u * gb.n_mma +
                                                                     16u * n),
                     "l"(tk.x + (size_t)n * tk.x_stride + 16u * cg + 8u * h)
                     : "memory");
      }
    };
    for (uint32_t u = ub; u < ue && !failed;) {
      const GUnit g = gemm_piece(gb, u, ue);
      u += g.tiles;
      const KTensor &tk = gb.t[g.ti];
      uint32_t bf, bl;
      gemm_blocks(tk, g.u0, g.u1, bf, bl);
      if (prev_ti >= 0 && (g.ti != prev_ti || g.rb != prev_rb)) {
        ++seg;  // a new row block: the other accumulator
        seg_tiles = 0;
        // flushed two segments ago
        // the accumulator it takes was emptied (the piece gb.accs before)
        if (seg >= gb.accs &&
            !__all_sync(0xFFFFFFFFu, mbar_wait(bar(kDFree + seg % gb.accs),
                                                ((seg / gb.accs) - 1) & 1u, gb.spin_limit))) {
          failed = true;
          break;
        }
        tc_fence_after();
      }
      prev_ti = g.ti;
      prev_rb = g.rb;
      const uint32_t d_tmem = tmem + (seg % gb.accs) * gb.n_mma;
      // tiles of the piece complete once block b is decoded
      auto ready_after = [&](uint32_t b) {
        if (b >= bl) return g.tiles;
        const uint32_t p1 = min(max(__ldg(tk.block_out_pos + b + 1), g.u0), g.u1);
        return min((p1 - g.u0) >> 11, g.tiles);
      };
      // the first block's activation tiles (every earlier product is done:
      // each block below waits for its own products before it goes on)
      uint32_t done = 0, fetched = ready_after(bf);
      for (uint32_t j = 0; j < fetched; ++j) fetch_x(tk, g.cg0 + j, (t_run + j) % gb.ring);
      asm volatile("cp.async.commit_group;" ::: "memory");
      for (uint32_t b = bf; b <= bl; ++b, ++k) {
        if (!__all_sync(0xFFFFFFFFu, mbar_wait(bar(kStaged + (k & 1)), (k >> 1) & 1u,
                                                gb.spin_limit))) {
          failed = true;
          break;
        }
        tc_fence_after();
        const uint32_t ready = ready_after(b);
        for (uint32_t j = fetched; j < ready; ++j)  // not fetched ahead (inconsistent positions)
          fetch_x(tk, g.cg0 + j, (t_run + j) % gb.ring);
        fetched = fetched > ready ? fetched : ready;
        asm volatile("cp.async.commit_group;\n\tcp.async.wait_all;" ::: "memory");
        fence_proxy_async();  // the activation tiles are read by the tensor cores
        __syncwarp();
        if (lane == 0) {
          for (; done < ready; ++done) {
            const uint32_t slot = (t_run + done) % gb.ring;
            const uint64_t ad = umma_desc(ring_a + slot * kGemmTileBytes, 128u, 256u);
            const uint64_t bd = umma_desc(ring_x + slot * x_tile_bytes, 16u * gb.n_mma, 128u);
            const uint32_t acc = seg_tiles + done > 0 ? 1u : 0u;
            asm volatile(
                "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
                " tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}\n" ::"r"(d_tmem),
                "l"(ad), "l"(bd), "r"(idesc), "r"(acc)
                : "memory");
          }
          asm volatile(
              "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                  bar(kMmaDone + (k & 1)))
              : "memory");
        }
        done = __shfl_sync(0xFFFFFFFFu, done, 0);
        // these products done, their slots take the next block's activation
        // tiles, which land while the consumers decode it
        if (!__all_sync(0xFFFFFFFFu, mbar_wait(bar(kMmaDone + (k & 1)), (k >> 1) & 1u,
                                                gb.spin_limit))) {
          failed = true;
          ++k;  // this block's commit was made
          break;
        }
        if (b < bl) {
          const uint32_t next = ready_after(b + 1);
          for (; fetched < next; ++fetched) fetch_x(tk, g.cg0 + fetched, (t_run + fetched) % gb.ring);
          asm volatile("cp.async.commit_group;" ::: "memory");
        }
      }
      asm volatile("cp.async.wait_all;" ::: "memory");  // nothing in flight past the piece
      t_run += g.tiles;
      seg_tiles += g.tiles;
    }
    asm volatile("cp.async.wait_all;" ::: "memory");
    if (failed && lane == 0) report(err, DF11_DEV_ERR_TIMEOUT);
    // no product in flight when the tensor memory goes: its last commit
    if (k >= 1 && !mbar_wait(bar(kMmaDone + ((k - 1) & 1)), ((k - 1) >> 1) & 1u, gb.spin_limit) &&
        lane == 0)
      report(err, DF11_DEV_ERR_TIMEOUT);
  } else {
    // ---- consumer warps ----
    const uint32_t region = smem_addr(regions + warp * gb.stage_bytes);
    uint8_t *region_p = regions + warp * gb.stage_bytes;
    const uint32_t wide = smem_addr(wide_s);
    uint32_t tphase = 0, t_run = 0, seg = 0;
    int cur_t = -1;
    bool waited = false;
    int32_t flush_seg = -1;  // segment whose accumulator waits to be added to y (warps 0-3)
    uint32_t flush_rb = 0, flush_k = 0, prev_rb = 0;
    int flush_ti = 0, prev_ti = -1;
    auto flush = [&]() {  // warps 0-3: accumulator of segment `flush_seg` into y
      const KTensor &ft = gb.t[flush_ti];
      if (!__all_sync(0xFFFFFFFFu, mbar_wait(bar(kMmaDone + (flush_k & 1)), (flush_k >> 1) & 1u,
                                              gb.spin_limit))) {
        failed = true;
        return;
      }
      tc_fence_after();
      if (!waited) {
        pdl_wait();  // y may still be cleared or read by the previous kernel
        waited = true;
      }
      const uint32_t row = flush_rb * kGemmM + 32u * warp + lane;
      const uint32_t base = tmem + ((32u * warp) << 16) + (flush_seg % gb.accs) * gb.n_mma;
      for (uint32_t c = 0; c < gb.n_mma; c += 8) {
        uint32_t v[8];
        asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
                     : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]),
                       "=r"(v[6]), "=r"(v[7])
                     : "r"(base + c)
                     : "memory");
        asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
        for (int j = 0; j < 8; ++j)
          if (c + j < ft.batch) atomicAdd(ft.y + (size_t)(c + j) * ft.y_stride + row, __uint_as_float(v[j]));
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(kDFree + flush_seg % gb.accs));
      flush_seg = -1;
    };
    for (uint32_t u = ub; u < ue && !failed;) {
      const GUnit g = gemm_piece(gb, u, ue);
      u += g.tiles;
      const KTensor &tk = gb.t[g.ti];
      if (prev_ti >= 0 && (g.ti != prev_ti || g.rb != prev_rb)) {
        // the previous segment is complete after its last block instance;
        // warps 0-3 add it to y during this segment's first block
        flush_seg = (int32_t)seg;
        flush_rb = prev_rb;
        flush_ti = prev_ti;
        flush_k = k - 1;
        ++seg;
      }
      prev_ti = g.ti;
      prev_rb = g.rb;
      if (g.ti != cur_t) {  // this tensor's decode table
        if (!__all_sync(0xFFFFFFFFu, mbar_wait(bar(kTableBar), tphase & 1u, gb.spin_limit))) {
          failed = true;
          break;
        }
        ++tphase;
        cur_t = g.ti;
      }
      uint32_t bf, bl;
      gemm_blocks(tk, g.u0, g.u1, bf, bl);
      for (uint32_t b = bf; b <= bl && !failed; ++b, ++k) {
        const uint32_t s = k & 1u, par = (k >> 1) & 1u;
        const uint32_t slot_sa = smem_addr(stages + s * L::head_bytes);
        const uint32_t release = bar(2 + s);
        if (!__all_sync(0xFFFFFFFFu, mbar_wait(bar(s), par, gb.spin_limit))) {
          failed = true;
          break;
        }
        const uint32_t counts_sa = slot_sa + L::bits_bytes + L::gaps_bytes;
        const uint4 m = lds128(counts_sa + L::counts_bytes);
        const uint32_t P0 = m.x, P1 = m.y, expected = P1 - P0;
        const uint2 cv = lds64(counts_sa + 8u * lane);  // T == 256: 8 counts per lane
        const uint32_t lsum = __dp4a(cv.x, 0x01010101u, __dp4a(cv.y, 0x01010101u, 0u));
        const uint32_t cnt = lds8(counts_sa + tid);
        const uint32_t before = __reduce_add_sync(0xFFFFFFFFu,
                                                  lane < warp * 32 / CONSUMERS ? lsum : 0u);
        const uint32_t total = __reduce_add_sync(0xFFFFFFFFu, lsum);
        bool ok = m.z && total == expected && !__any_sync(0xFFFFFFFFu, cnt > tk.max_chunk_elems);
        int start, end;
        {
          const uint32_t bit = 5u * (uint32_t)tid;
          const uint32_t ga = slot_sa + L::bits_bytes + 4u * (bit >> 5);
          const uint32_t v = __funnelshift_l(__byte_perm(lds32(ga + 4u), 0, 0x0123),
                                             __byte_perm(lds32(ga), 0, 0x0123), bit);
          start = (int)(v >> 27);
          end = C * 8 + (int)((v >> 22) & 31u);
        }
        if (m.w != 0xFFFFFFFFu) {
          const uint32_t b0 = (uint32_t)tid * (C * 8);
          if (b0 >= m.w) start = end = 0;
          else if ((uint32_t)end > m.w - b0) end = (int)(m.w - b0);
        }
        uint32_t w[NW];
#pragma unroll
        for (int j = 0; j < NW; ++j) {
          w[j] = __byte_perm(lds32(slot_sa + (uint32_t)tid * C + 4u * j), 0, 0x0123);
          if (tk.masked) w[j] |= __funnelshift_rc(0xFFFFFFFFu, 0u, (uint32_t)max(end - 32 * j, 0));
        }
        uint32_t incl = cnt;
#pragma unroll
        for (int dd = 1; dd < 32; dd <<= 1) {
          const uint32_t v = __shfl_up_sync(0xFFFFFFFFu, incl, dd);
          if (lane >= dd) incl += v;
        }
        const uint32_t warp_total = __shfl_sync(0xFFFFFFFFu, incl, 31);
        ok = ok && warp_total <= tk.max_warp_elems;
        int bad = 0;
        const uint32_t G0 = P0 + before;
        const uint32_t head = G0 & 15u, span = head + warp_total;
        const uint32_t d = head + incl - cnt;
        if (ok) {
          // lanes whose codewords all lie outside the piece skip their walk
          const uint32_t e0 = G0 + incl - cnt;
          const bool inside = cnt && e0 < g.u1 && e0 + cnt > g.u0;
          uint32_t got = cnt;
          if (inside) {
            if (tk.masked)
              got = decode_counted<C>(w, start, end, wide, lut0_s, lens_s, tk.luts + 256,
                                      tk.num_luts, region, d, cnt, bad);
            else
              got = decode_direct<T, C, false>(w, start, end, wide, lut0_s, lens_s, tk.luts + 256,
                                               tk.num_luts, region, d,
                                               region + ((d + cnt - 1u) & ~3u), bad);
          }
          if (!bad && got != cnt) bad = DF11_DEV_ERR_COUNT;
        }
        if (!ok || __any_sync(0xFFFFFFFFu, bad != 0)) {
          if (bad) report(err, bad);
          else if (lane == 0 && warp == 0) report(err, m.z ? DF11_DEV_ERR_COUNT : DF11_DEV_ERR_CAPACITY);
          ok = false;
        }
        // the ring's tiles that this block writes held tiles of blocks up
        // to the previous one: their products must be done
        if (k >= 1 && !__all_sync(0xFFFFFFFFu, mbar_wait(bar(kMmaDone + ((k - 1) & 1)),
                                                          ((k - 1) >> 1) & 1u, gb.spin_limit))) {
          failed = true;
          break;
        }
        tc_fence_after();
        if (flush_seg >= 0 && warp < 4) flush();  // the previous segment's accumulator
        if (failed) break;
        __syncwarp();
        const uint32_t base = G0 & ~15u;
        const uint8_t *smg = tk.sign_mantissa + base;  // this warp's sign/mantissa bytes
        if (ok) {
          // whole 16-element groups inside the piece: row r of tile j, two
          // 16-byte halves
          const uint32_t g_begin = head ? 1u : 0u, g_end = span >> 4;
          for (uint32_t gi = g_begin + lane; gi < g_end; gi += 32) {
            const uint32_t q = base + 16u * gi;  // first element of the group
            const uint32_t rv_a = region + 16u * gi;
            if (q >= g.u0 && q < g.u1) {
              const uint32_t e = q - g.u0, r = (e >> 4) & 127u;
              const uint32_t dst = ring_a + ((t_run + (e >> 11)) % gb.ring) * kGemmTileBytes +
                                   (r >> 3) * 256u + (r & 7u) * 16u;
              const uint4 sv = __ldg(reinterpret_cast<const uint4 *>(smg) + gi);
              const uint4 rv = lds128(rv_a);
              const uint2 a = fuse4(sv.x, rv.x), c2 = fuse4(sv.y, rv.y);
              const uint2 e2 = fuse4(sv.z, rv.z), f = fuse4(sv.w, rv.w);
              asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(dst), "r"(a.x),
                           "r"(a.y), "r"(c2.x), "r"(c2.y)
                           : "memory");
              asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(dst + 128u), "r"(e2.x),
                           "r"(e2.y), "r"(f.x), "r"(f.y)
                           : "memory");
            }
            sts128_zero(rv_a);
          }
          // every lane is done with the whole groups (it may have read one that
          // a ragged lane zeroes next) before the ragged groups are touched
          __syncwarp();
          if (span) {  // the ragged first and last groups, one element per lane
            const uint32_t i = ((uint32_t)lane & 15u) + (lane >> 4 ? ((span - 1) >> 4) << 4 : 0u);
            const uint32_t q = base + i;
            if (i >= head && i < span && (i < (g_begin << 4) || i >= (g_end << 4)) && q >= g.u0 &&
                q < g.u1) {
              const uint32_t e = q - g.u0;
              const uint32_t dst = ring_a + ((t_run + (e >> 11)) % gb.ring) * kGemmTileBytes +
                                   umma_offset((e >> 4) & 127u, e & 15u);
              const uint16_t v = fuse1(__ldg(smg + i), lds8(region + i));
              asm volatile("st.shared.u16 [%0], %1;" ::"r"(dst), "h"(v) : "memory");
            }
            sts8_zero(region + i);
          }
        } else {
          for (uint32_t i = lane; i < (span + 8u + 15u) >> 4 && 16u * i < gb.stage_bytes; i += 32)
            reinterpret_cast<uint4 *>(region_p)[i] = make_uint4(0, 0, 0, 0);
        }
        fence_proxy_async();  // the tiles are read by the tensor cores
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(bar(kStaged + s));
          mbar_arrive(release);
        }
      }
      if (failed) break;
      t_run += g.tiles;
    }
    if (!failed && prev_ti >= 0 && warp < 4) {  // the last segment
      flush_seg = (int32_t)seg;
      flush_rb = prev_rb;
      flush_ti = prev_ti;
      flush_k = k - 1;
      flush();
    }
    if (failed && lane == 0) report(err, DF11_DEV_ERR_TIMEOUT);
  }
  // every warp is here before the tensor memory goes
  tc_fence_before();
  __syncthreads();
  if (warp == MMA) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                 "r"(gb.tmem_cols)
                 : "memory");
  }
}

// ---------------------------------------------------------------------------
// The decode table of one tensor (df11_build_decode_table): the shared-memory
// image of table 0, the code lengths and the derived table, as the decode
// kernels set them up, written to global memory once.
__global__ void __launch_bounds__(256) df11_table_kernel(const uint32_t *luts,
                                                         const uint8_t *code_lengths,
                                                         uint32_t num_luts, uint4 *out) {
  __shared__ __align__(16) uint8_t t[DF11_DECODE_TABLE_BYTES];
  uint8_t *lens_s = t;
  uint32_t *lut0_s = reinterpret_cast<uint32_t *>(t + (kOffLut0 - kOffLens));
  uint2 *wide_s = reinterpret_cast<uint2 *>(t + (kOffWide - kOffLens));
  load_tables(threadIdx.x, 256, luts, code_lengths, lut0_s, lens_s);
  __syncthreads();
  build_wide<256, 5>(wide_s, lut0_s, lens_s, luts + 256, num_luts);
  __syncthreads();
  for (uint32_t i = threadIdx.x; i < DF11_DECODE_TABLE_BYTES / 16; i += 256)
    out[i] = reinterpret_cast<const uint4 *>(t)[i];
}

// ---------------------------------------------------------------------------
// host side

bool supported(uint32_t C, uint32_t T) {
  if (T == 256) return C == 4 || C == 8 || C == 16 || C == 24;
  if (T == 128 || T == 512) return C == 8;
  return false;
}

uint32_t stage_bytes_for(uint32_t max_block_elems) {
  return (max_block_elems + 32u + 15u) & ~15u;
}

bool aligned(const void *p, uintptr_t a) { return ((uintptr_t)p & (a - 1)) == 0; }

df11_status validate(const df11_tensor &t) {
  const df11_params &p = t.params;
  if (p.n == 0) return DF11_OK;
  if (p.n >= (1ull << 32)) return DF11_ERR_TOO_LARGE;
  if (!t.bitstream || !t.gaps || !t.block_out_pos || !t.luts || !t.code_lengths ||
      !t.sign_mantissa || !t.out_bf16)
    return DF11_ERR_NULL;
  if (!aligned(t.bitstream, 16) || !aligned(t.gaps, 16) || !aligned(t.luts, 16) ||
      !aligned(t.chunk_counts, 16) || !aligned(t.decode_table, 16) ||
      !aligned(t.sign_mantissa, 16) || !aligned(t.out_bf16, 16) || !aligned(t.block_out_pos, 4))
    return DF11_ERR_ALIGN;
  if (!supported(p.chunk_bytes, p.threads_per_block)) return DF11_ERR_UNSUPPORTED;
  const uint64_t block_bits = 8ull * p.chunk_bytes * p.threads_per_block;
  if (p.total_bits < p.n || p.total_bits > 32ull * p.n) return DF11_ERR_FORMAT;
  if ((uint64_t)p.num_blocks != (p.total_bits + block_bits - 1) / block_bits) return DF11_ERR_FORMAT;
  if (p.num_luts < 1 || p.num_luts >= (1u << 24)) return DF11_ERR_FORMAT;
  if (p.max_block_elems == 0 || p.max_block_elems > 8ull * p.chunk_bytes * p.threads_per_block)
    return DF11_ERR_FORMAT;
  if (p.max_chunk_elems == 0 || p.max_chunk_elems > 8ull * p.chunk_bytes) return DF11_ERR_FORMAT;
  if (p.max_warp_elems == 0 || p.max_warp_elems > 32ull * p.max_chunk_elems)
    return DF11_ERR_FORMAT;
  if (t.chunk_counts && 8ull * p.chunk_bytes > 255) return DF11_ERR_FORMAT;
  if (p.max_len < 1 || p.max_len > 32) return DF11_ERR_FORMAT;
  return DF11_OK;
}

// Per-device launch state, indexed by kernel instance: the warp-specialised
// kernels use 3 * i + mode with i = 3-8 (decode with counts), 12-14 (fused
// matrix-vector product) and 15-20 (decode without counts); the
// tensor-core product 64-65.
constexpr int kInstances = 80;
struct DeviceInfo {
  int sms = 0;
  std::atomic<size_t> configured[kInstances];  // shared-memory limit set, per kernel instance
  // (smem << 8 | blocks per SM) of the last two shared-memory sizes, per instance
  std::atomic<uint64_t> occupancy[kInstances][2];
};

DeviceInfo &device_info(int dev) {
  static DeviceInfo info[64];
  DeviceInfo &d = info[dev & 63];
  if (d.sms == 0) {
    int v = 0;
    cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev);
    d.sms = v > 0 ? v : 1;
  }
  return d;
}

// Thread blocks per tensor: one wave (at most `budget`, the resident
// count), at least one per tensor, and as few format blocks per thread block
// as possible, since a launch lasts as long as its busiest thread block.
// Shares in proportion to the format blocks, rounded down, then thread
// blocks moved to where the most format blocks per thread block remain.
uint32_t split_grid(KBatch &kb, const uint32_t *blocks, uint64_t budget) {
  const int n = kb.count;
  uint64_t total = 0;
  for (int i = 0; i < n; ++i) total += blocks[i];
  if (budget < (uint64_t)n) budget = n;
  uint64_t c[DF11_MAX_BATCH], sum = 0;
  for (int i = 0; i < n; ++i) {
    c[i] = budget * blocks[i] / total;
    if (c[i] < 1) c[i] = 1;
    if (c[i] > blocks[i]) c[i] = blocks[i];
    sum += c[i];
  }
  auto per = [&](int i, uint64_t ci) { return (blocks[i] + ci - 1) / ci; };
  while (sum > budget) {  // only from the at-least-one rule: take from the idlest
    int best = -1;
    for (int i = 0; i < n; ++i)
      if (c[i] > 1 && (best < 0 || per(i, c[i] - 1) < per(best, c[best] - 1))) best = i;
    if (best < 0) break;
    --c[best];
    --sum;
  }
  while (sum < budget) {  // the rest to the busiest tensor that can use one
    int best = -1;
    for (int i = 0; i < n; ++i)
      if (c[i] < blocks[i] && (best < 0 || per(i, c[i]) > per(best, c[best]))) best = i;
    if (best < 0) break;
    ++c[best];
    ++sum;
  }
  uint32_t begin = 0;
  for (int i = 0; i < n; ++i) {
    kb.t[i].cta_begin = begin;
    begin += (uint32_t)c[i];
  }
  kb.cta_end = begin;
  return begin;
}

// Launch with programmatic stream serialization: the kernel may begin while
// the previous one in the stream finishes (see pdl_wait).  DF11_PDL=0 in the
// environment launches without it.
bool pdl_enabled() {
  static const bool on = [] {
    const char *v = std::getenv("DF11_PDL");
    return !(v && v[0] == '0');
  }();
  return on;
}

template <typename... Args>
df11_status launch_pdl(void (*kern)(Args...), uint32_t grid, uint32_t threads, size_t smem,
                       cudaStream_t s, Args... args) {
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(threads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl_enabled() ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kern, args...) == cudaSuccess ? DF11_OK : DF11_ERR_CUDA;
}

template <typename K>
df11_status prepare(K kern, int threads, size_t smem, int instance, uint64_t &budget) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return DF11_ERR_CUDA;
  DeviceInfo &di = device_info(dev);
  if (instance < 0 || instance >= kInstances) return DF11_ERR_INVALID;
  if (smem > 48 * 1024 && di.configured[instance].load() < smem) {
    // all of the unified L1 as shared memory: these kernels keep their
    // working set there, and the occupancy query assumes this split
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
            cudaSuccess ||
        cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout, 100) !=
            cudaSuccess)
      return DF11_ERR_CUDA;
    di.configured[instance].store(smem);
  }
  // occupancy queries cost microseconds of host time: one per instance and
  // shared-memory size (a layer-by-layer decode loop repeats the sizes)
  int per_sm = 0;
  const uint64_t c0 = di.occupancy[instance][0].load(), c1 = di.occupancy[instance][1].load();
  if (c0 && (c0 >> 8) == (uint64_t)smem) {
    per_sm = (int)(c0 & 0xFF);
  } else if (c1 && (c1 >> 8) == (uint64_t)smem) {
    per_sm = (int)(c1 & 0xFF);
  } else {
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, threads, smem) !=
        cudaSuccess)
      return DF11_ERR_CUDA;
    // keep the most recent size in slot 0, the one before in slot 1
    di.occupancy[instance][1].store(c0);
    di.occupancy[instance][0].store(((uint64_t)smem << 8) | (uint64_t)(per_sm & 0xFF));
  }
  if (per_sm < 1) return DF11_ERR_TOO_LARGE;
  budget = (uint64_t)di.sms * per_sm;
  return DF11_OK;
}

size_t ws_shared_bytes(uint32_t C, uint32_t T, uint32_t sm_bytes, uint32_t region,
                       uint32_t columns, bool warp_sm);

// Sign/mantissa bytes staged per block in the stage slot or per warp in the
// warp's own buffer, whichever keeps more thread blocks resident (the slot
// on a tie); read from global memory (L2) only when neither fits, or, without
// chunk counts, when that keeps more blocks resident.  Measured: at equal
// residency the slot beats the warp buffer, which beats global reads.
template <int T, int C, bool GEMV = false, bool COUNTS = true>
df11_status launch_ws(KBatch &kb, const uint32_t *blocks, uint32_t sm_stage, cudaStream_t s,
                      int instance) {
  uint32_t sub_need = 0;  // bytes of the largest set of deeper tables of the launch
  for (int i = 0; i < kb.count; ++i)
    if (kb.t[i].num_luts > 1 && (kb.t[i].num_luts - 1) * 1024u > sub_need)
      sub_need = (kb.t[i].num_luts - 1) * 1024u;
  void (*kern[3])(KBatch) = {df11_decode_ws_kernel<T, C, kSmSlot, GEMV, COUNTS>,
                             df11_decode_ws_kernel<T, C, kSmGlobal, GEMV, COUNTS>,
                             df11_decode_ws_kernel<T, C, kSmWarp, GEMV, COUNTS>};
  const size_t smem[3] = {ws_shared_bytes(C, T, sm_stage, kb.stage_bytes, kb.col_bytes, false),
                          ws_shared_bytes(C, T, 0, kb.stage_bytes, kb.col_bytes, false),
                          ws_shared_bytes(C, T, 0, kb.stage_bytes, kb.col_bytes, true)};
  const int order[3] = {kSmSlot, kSmWarp, kSmGlobal};
  uint64_t best = 0;
  int pick = -1;
  for (int m : order) {
    // with chunk counts, global reads only when nothing else fits (measured
    // slower at C = 24 even with a fourth resident block); without counts
    // also when they keep more blocks resident (the column areas leave room
    // for two blocks per SM with staged bytes, three without)
    if (m == kSmGlobal && pick >= 0 && COUNTS) break;
    if (smem[m] > 227 * 1024) continue;
    uint64_t budget = 0;
    const df11_status st = prepare(kern[m], T + 32, smem[m], 3 * instance + m, budget);
    if (st != DF11_OK && st != DF11_ERR_TOO_LARGE) return st;
    if (budget > best) {
      best = budget;
      pick = m;
    }
  }
  if (pick < 0) return DF11_ERR_TOO_LARGE;
  kb.sm_bytes = pick == kSmSlot ? sm_stage : 0u;
  // the deeper tables (read on codewords longer than the derived table's
  // index) in shared memory too, when they fit in what the resident blocks
  // leave of the SM's shared memory
  size_t use = smem[pick];
  kb.sub_bytes = 0;
  if (sub_need && kb.col_bytes == 0) {
    int dev = 0, smem_sm = 0, reserved = 0;
    if (cudaGetDevice(&dev) == cudaSuccess &&
        cudaDeviceGetAttribute(&smem_sm, cudaDevAttrMaxSharedMemoryPerMultiprocessor, dev) ==
            cudaSuccess &&
        cudaDeviceGetAttribute(&reserved, cudaDevAttrReservedSharedMemoryPerBlock, dev) ==
            cudaSuccess) {
      const uint64_t per_sm = best / (uint64_t)device_info(dev).sms;
      if (per_sm && use + sub_need + (size_t)reserved <= (size_t)smem_sm / per_sm &&
          use + sub_need <= 227 * 1024) {
        uint64_t b2 = 0;
        const df11_status st = prepare(kern[pick], T + 32, use + sub_need, 3 * instance + pick, b2);
        if (st == DF11_OK && b2 == best) {
          kb.sub_bytes = sub_need;
          use += sub_need;
        }
      }
    }
  }
  const uint32_t grid = split_grid(kb, blocks, best);
  return launch_pdl(kern[pick], grid, T + 32, use, s, kb);
}

// Per-warp exponent region of the warp-specialised kernel: the warp's head
// (< 16), up to max_warp_elems exponents (checked per block before
// decoding), and slack for the last lookup: it touches bytes up to 6 past
// the warp's last element (the spill word, or up to three extra exponents of
// a corrupt stream).
uint32_t region_bytes_for(uint32_t max_warp_elems) {
  return (15u + max_warp_elems + 8u + 15u) & ~15u;
}

// Without chunk counts, each warp's column area: the lane's byte j at word
// (j/4)*32 + lane, for up to the bytes a walk may write (max_chunk_elems,
// plus the four past it that its last lookup may reach, plus the word the
// last lookup's bytes spill into).
uint32_t column_bytes_for(uint32_t max_chunk_elems) {
  return 128u * ((max_chunk_elems + 3u) / 4u + 1u);
}

size_t ws_shared_bytes(uint32_t C, uint32_t T, uint32_t sm_bytes, uint32_t region,
                       uint32_t columns, bool warp_sm) {
  const size_t slot = (size_t)T * C + 16 + (size_t)T * 5 / 8 + 16 + T + 16 + sm_bytes;
  return (size_t)kOffStages + kWsStages * slot +
         (size_t)(T / 32) * ((size_t)region * (warp_sm ? 2 : 1) + columns);
}

// Test hook (df11_test_withhold_copies): launches left to make with the
// producer issuing no copies, and the wait limit they use.
std::atomic<int> g_withhold_launches{0};
std::atomic<uint32_t> g_withhold_spin_limit{kSpinLimit};

df11_status launch_group(const df11_tensor *ts, int count, int32_t *d_err, cudaStream_t s,
                         bool ws, const df11_gemv *ops = nullptr) {
  KBatch kb{};
  kb.err = d_err;
  kb.spin_limit = kSpinLimit;
  if (ws && g_withhold_launches.load() > 0 && g_withhold_launches.fetch_sub(1) > 0) {
    kb.withhold = 1;
    kb.spin_limit = g_withhold_spin_limit.load();
  }
  uint32_t blocks[DF11_MAX_BATCH];
  uint32_t max_elems = 0, max_chunk = 0, max_warp = 0, C = 0, T = 0;
  for (int i = 0; i < count; ++i) {
    const df11_params &p = ts[i].params;
    if (p.n == 0) continue;
    KTensor &k = kb.t[kb.count];
    k.bitstream = ts[i].bitstream;
    k.gaps = ts[i].gaps;
    k.chunk_counts = ts[i].chunk_counts;
    k.block_out_pos = ts[i].block_out_pos;
    k.luts = ts[i].luts;
    k.code_lengths = ts[i].code_lengths;
    k.sign_mantissa = ts[i].sign_mantissa;
    k.out = ts[i].out_bf16;
    k.decode_table = ts[i].decode_table;
    k.total_bits = p.total_bits;
    k.n = (uint32_t)p.n;
    k.num_blocks = p.num_blocks;
    k.num_luts = p.num_luts;
    k.max_block_elems = p.max_block_elems;
    k.max_chunk_elems = p.max_chunk_elems;
    k.max_warp_elems = p.max_warp_elems;
    k.masked = p.max_len > (uint32_t)kWideBits ? 1u : 0u;
    if (ops) {
      k.x = ops[i].x;
      k.y = ops[i].y;
      k.cols = ops[i].cols;
      k.batch = ops[i].batch;
      k.x_stride = ops[i].x_stride;
      k.y_stride = ops[i].y_stride;
      k.interleave_log2 = ops[i].interleave > 1 ? (uint32_t)__builtin_ctz(ops[i].interleave) : 0u;
    }
    blocks[kb.count] = p.num_blocks;
    ++kb.count;
    max_elems = max_elems > p.max_block_elems ? max_elems : p.max_block_elems;
    max_chunk = max_chunk > p.max_chunk_elems ? max_chunk : p.max_chunk_elems;
    max_warp = max_warp > p.max_warp_elems ? max_warp : p.max_warp_elems;
    C = p.chunk_bytes;
    T = p.threads_per_block;
  }
  if (kb.count == 0) return DF11_OK;
  kb.stage_bytes = region_bytes_for(max_warp);  // bytes of each warp's region
  // deeper tables only serve codewords longer than the derived table's
  // index (about one lookup in a thousand): they are read from global
  // memory, and the shared memory goes to resident thread blocks
  const uint32_t sm_stage = stage_bytes_for(max_elems);
  if (ops) {
    if (T == 256 && C == 8) return launch_ws<256, 8, true>(kb, blocks, sm_stage, s, 12);
    if (T == 256 && C == 16) return launch_ws<256, 16, true>(kb, blocks, sm_stage, s, 13);
    if (T == 256 && C == 24) return launch_ws<256, 24, true>(kb, blocks, sm_stage, s, 14);
    return DF11_ERR_UNSUPPORTED;
  }
  if (ws) {
    if (T == 256 && C == 8) return launch_ws<256, 8>(kb, blocks, sm_stage, s, 3);
    if (T == 256 && C == 4) return launch_ws<256, 4>(kb, blocks, sm_stage, s, 4);
    if (T == 256 && C == 16) return launch_ws<256, 16>(kb, blocks, sm_stage, s, 5);
    if (T == 256 && C == 24) return launch_ws<256, 24>(kb, blocks, sm_stage, s, 8);
    if (T == 128 && C == 8) return launch_ws<128, 8>(kb, blocks, sm_stage, s, 6);
    if (T == 512 && C == 8) return launch_ws<512, 8>(kb, blocks, sm_stage, s, 7);
    return DF11_ERR_UNSUPPORTED;
  }
  // the format as the pages state it: each lane decodes into its column
  kb.col_cap = max_chunk;
  kb.col_bytes = column_bytes_for(max_chunk);
  if (T == 256 && C == 8) return launch_ws<256, 8, false, false>(kb, blocks, sm_stage, s, 15);
  if (T == 256 && C == 4) return launch_ws<256, 4, false, false>(kb, blocks, sm_stage, s, 16);
  if (T == 256 && C == 16) return launch_ws<256, 16, false, false>(kb, blocks, sm_stage, s, 17);
  if (T == 256 && C == 24) return launch_ws<256, 24, false, false>(kb, blocks, sm_stage, s, 18);
  if (T == 128 && C == 8) return launch_ws<128, 8, false, false>(kb, blocks, sm_stage, s, 19);
  if (T == 512 && C == 8) return launch_ws<512, 8, false, false>(kb, blocks, sm_stage, s, 20);
  return DF11_ERR_UNSUPPORTED;
}

// The buffers of a call's non-empty tensors must be memory of the current
// device, where its kernels run (checked for every tensor of the call before
// anything is queued): the stream, the sign/mantissa bytes and the output
// (or the product's activations and results).
df11_status check_devices(const df11_tensor *ts, int count, const df11_gemv *ops = nullptr) {
  for (int i = 0; i < count; ++i) {
    if (ts[i].params.n == 0) continue;
    const void *ptrs[5] = {ts[i].bitstream, ts[i].sign_mantissa, ts[i].decode_table,
                           ops ? (const void *)ops[i].x : (const void *)ts[i].out_bf16,
                           ops ? (const void *)ops[i].y : nullptr};
    const df11_status st = df11_internal::check_device_pointers(ptrs, 5);
    if (st != DF11_OK) return st;
  }
  return DF11_OK;
}

// Tensors with chunk counts go to the warp-specialised kernel, the others to
// the count-by-decoding kernel (one launch each, same stream).
df11_status launch_batch(const df11_tensor *ts, int count, int32_t *d_err, cudaStream_t s) {
  df11_tensor with[DF11_MAX_BATCH], without[DF11_MAX_BATCH];
  int nw = 0, nwo = 0;
  for (int i = 0; i < count; ++i) {
    if (ts[i].chunk_counts) with[nw++] = ts[i];
    else without[nwo++] = ts[i];
  }
  df11_status st = DF11_OK;
  if (nwo) st = launch_group(without, nwo, d_err, s, false);
  if (st == DF11_OK && nw) st = launch_group(with, nw, d_err, s, true);
  return st;
}

// The fused product on tensor cores for up to DF11_MAX_BATCH tensors (one
// launch): the launch's tiles spread over one wave of thread blocks in
// equal contiguous ranges.

template <int C>
df11_status launch_gemm(GBatch &gb, cudaStream_t s, int instance) {
  constexpr int T = 256;
  auto kern = df11_decode_gemm_kernel<T, C>;
  using L = WsLayout<T, C>;
  const size_t head = (kOffStages + 2 * L::head_bytes + (T / 32) * (size_t)gb.stage_bytes +
                       1023) & ~(size_t)1023;
  size_t smem = head + (size_t)gb.ring * (kGemmTileBytes + 32u * gb.n_mma);
  if (smem > 227 * 1024) return DF11_ERR_TOO_LARGE;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return DF11_ERR_CUDA;
  // Resident thread blocks per SM, from the kernel's registers and shared
  // memory and the SM's limits; and tensor memory: each resident block
  // holds tmem_cols of the SM's 512 columns.  When tensor memory allows
  // fewer blocks than the rest, the launch asks for more shared memory than
  // it uses, so that no SM takes more blocks than its tensor memory holds
  // (an allocation would otherwise wait for a neighbour to finish).
  cudaFuncAttributes fa{};
  int smem_sm = 0, regs_sm = 0, reserved = 0;
  if (cudaFuncGetAttributes(&fa, kern) != cudaSuccess ||
      cudaDeviceGetAttribute(&smem_sm, cudaDevAttrMaxSharedMemoryPerMultiprocessor, dev) !=
          cudaSuccess ||
      cudaDeviceGetAttribute(&regs_sm, cudaDevAttrMaxRegistersPerMultiprocessor, dev) !=
          cudaSuccess ||
      cudaDeviceGetAttribute(&reserved, cudaDevAttrReservedSharedMemoryPerBlock, dev) !=
          cudaSuccess)
    return DF11_ERR_CUDA;
  const uint64_t regs_block = (uint64_t)((fa.numRegs + 7) & ~7) * (T + 64);
  uint64_t per_sm = (uint64_t)smem_sm / (smem + (size_t)reserved);
  if (regs_block && (uint64_t)regs_sm / regs_block < per_sm) per_sm = (uint64_t)regs_sm / regs_block;
  if (2048u / (T + 64) < per_sm) per_sm = 2048u / (T + 64);
  const uint64_t tmem_fit = 512u / gb.tmem_cols;
  if (tmem_fit < per_sm) {
    per_sm = tmem_fit;
    const size_t want = ((size_t)smem_sm / per_sm - (size_t)reserved) & ~(size_t)127;
    if (want > smem) smem = want < 227 * 1024 ? want : 227 * 1024;
  }
  if (per_sm < 1) return DF11_ERR_TOO_LARGE;
  uint64_t budget = 0;  // prepare() sets the kernel's shared-memory limit; its count is not used
  const df11_status st = prepare(kern, T + 64, smem, instance, budget);
  if (st != DF11_OK && st != DF11_ERR_TOO_LARGE) return st;
  budget = (uint64_t)device_info(dev).sms * per_sm;
  const uint32_t tiles = gb.tile_begin[gb.count];
  gb.ctas = (uint32_t)(tiles < budget ? tiles : budget);
  return launch_pdl(kern, gb.ctas, T + 64, smem, s, gb);
}

}  // namespace

extern "C" {

df11_status df11_decode(const uint8_t *bitstream, const uint8_t *gaps,
                        const uint32_t *block_out_pos, const uint32_t *luts,
                        const uint8_t *code_lengths, const uint8_t *sign_mantissa,
                        uint16_t *out_bf16, uint64_t n, const df11_params *params,
                        int32_t *d_err, df11_stream_t stream) {
  if (!params) return DF11_ERR_NULL;
  if (params->n != n) return DF11_ERR_INVALID;
  if (d_err && !aligned(d_err, 4)) return DF11_ERR_ALIGN;
  df11_tensor t{bitstream, gaps, nullptr, block_out_pos, luts, code_lengths, sign_mantissa,
                out_bf16, nullptr, *params};
  df11_status st = validate(t);
  if (st != DF11_OK || n == 0) return st;
  st = check_devices(&t, 1);
  if (st != DF11_OK) return st;
  return launch_batch(&t, 1, d_err, (cudaStream_t)stream);
}

df11_status df11_decode_batched(const df11_tensor *tensors, int count, int32_t *d_err,
                                df11_stream_t stream) {
  if (count < 0) return DF11_ERR_INVALID;
  if (count == 0) return DF11_OK;
  if (!tensors) return DF11_ERR_NULL;
  if (d_err && !aligned(d_err, 4)) return DF11_ERR_ALIGN;
  uint32_t C = 0, T = 0;
  for (int i = 0; i < count; ++i) {
    df11_status st = validate(tensors[i]);
    if (st != DF11_OK) return st;
    if (tensors[i].params.n == 0) continue;
    if (C == 0) {
      C = tensors[i].params.chunk_bytes;
      T = tensors[i].params.threads_per_block;
    } else if (C != tensors[i].params.chunk_bytes || T != tensors[i].params.threads_per_block) {
      return DF11_ERR_INVALID;
    }
  }
  const df11_status dst = check_devices(tensors, count);
  if (dst != DF11_OK) return dst;
  for (int i = 0; i < count; i += DF11_MAX_BATCH) {
    const int c = count - i < DF11_MAX_BATCH ? count - i : DF11_MAX_BATCH;
    df11_status st = launch_batch(tensors + i, c, d_err, (cudaStream_t)stream);
    if (st != DF11_OK) return st;
  }
  return DF11_OK;
}

df11_status df11_decode_gemv(const df11_tensor *tensors, const df11_gemv *ops, int count,
                             int32_t *d_err, df11_stream_t stream) {
  if (count < 0) return DF11_ERR_INVALID;
  if (count == 0) return DF11_OK;
  if (!tensors || !ops) return DF11_ERR_NULL;
  if (d_err && !aligned(d_err, 4)) return DF11_ERR_ALIGN;
  cudaStream_t s = (cudaStream_t)stream;
  uint32_t C = 0, T = 0;
  for (int i = 0; i < count; ++i) {
    const df11_tensor &t = tensors[i];
    const df11_gemv &g = ops[i];
    const df11_params &p = t.params;
    if (!g.y || (p.n && !g.x)) return DF11_ERR_NULL;
    if (g.cols == 0 || g.cols % 16 || p.n % g.cols) return DF11_ERR_INVALID;
    const uint64_t rows = p.n / g.cols;
    if (g.batch < 1 || g.batch > DF11_GEMV_MAX_BATCH) return DF11_ERR_INVALID;
    if (g.x_stride < g.cols || g.x_stride % 8 || g.y_stride < rows) return DF11_ERR_INVALID;
    const uint32_t il = g.interleave ? g.interleave : 1u;
    if (il > 32 || (il & (il - 1)) || rows % il) return DF11_ERR_INVALID;
    if (!aligned(g.x, 16) || !aligned(g.y, 4)) return DF11_ERR_ALIGN;
    df11_tensor v = t;
    v.out_bf16 = reinterpret_cast<uint16_t *>(16);  // not written; passes the output checks
    const df11_status st = validate(v);
    if (st != DF11_OK) return st;
    if (p.n == 0) continue;
    if (!t.chunk_counts) return DF11_ERR_UNSUPPORTED;
    if (C == 0) {
      C = p.chunk_bytes;
      T = p.threads_per_block;
    } else if (C != p.chunk_bytes || T != p.threads_per_block) {
      return DF11_ERR_INVALID;
    }
  }
  if (C && !(T == 256 && (C == 8 || C == 16 || C == 24))) return DF11_ERR_UNSUPPORTED;
  const df11_status dst = check_devices(tensors, count, ops);
  if (dst != DF11_OK) return dst;
  // y = W x: clear the outputs first, in stream order, one launch per 16
  for (int i = 0; i < count; i += DF11_MAX_BATCH) {
    ClearArgs ca{};
    for (int j = i; j < count && j < i + DF11_MAX_BATCH; ++j) {
      const df11_gemv &g = ops[j];
      if (g.accumulate || tensors[j].params.n == 0) continue;
      ca.y[ca.count] = g.y;
      ca.rows[ca.count] = (uint32_t)(tensors[j].params.n / g.cols);
      ca.batch[ca.count] = g.batch;
      ca.stride[ca.count] = g.y_stride;
      ++ca.count;
    }
    if (ca.count && launch_pdl(clear_rows_kernel, 148u, 256u, 0, s, ca) != DF11_OK)
      return DF11_ERR_CUDA;
  }
  for (int i = 0; i < count; i += DF11_MAX_BATCH) {
    const int c = count - i < DF11_MAX_BATCH ? count - i : DF11_MAX_BATCH;
    df11_tensor ts[DF11_MAX_BATCH];
    df11_gemv gs[DF11_MAX_BATCH];
    int m = 0;
    for (int j = 0; j < c; ++j) {
      if (tensors[i + j].params.n == 0) continue;
      ts[m] = tensors[i + j];
      gs[m] = ops[i + j];
      ++m;
    }
    if (!m) continue;
    const df11_status st = launch_group(ts, m, d_err, s, true, gs);
    if (st != DF11_OK) return st;
  }
  return DF11_OK;
}

df11_status df11_decode_gemm(const df11_tensor *tensors, const df11_gemv *ops, int count,
                             int32_t *d_err, df11_stream_t stream) {
  if (count < 0 || count > DF11_MAX_BATCH) return count < 0 ? DF11_ERR_INVALID : DF11_ERR_TOO_LARGE;
  if (count == 0) return DF11_OK;
  if (!tensors || !ops) return DF11_ERR_NULL;
  if (d_err && !aligned(d_err, 4)) return DF11_ERR_ALIGN;
  cudaStream_t s = (cudaStream_t)stream;
  GBatch gb{};
  gb.err = d_err;
  gb.spin_limit = kSpinLimit;
  uint32_t C = 0, max_warp = 0, max_block = 0, max_batch = 0, tiles = 0;
  df11_tensor ts[DF11_MAX_BATCH];
  df11_gemv gs[DF11_MAX_BATCH];
  int m = 0;
  for (int i = 0; i < count; ++i) {
    const df11_tensor &t = tensors[i];
    const df11_gemv &g = ops[i];
    const df11_params &p = t.params;
    if (!g.y || (p.n && !g.x)) return DF11_ERR_NULL;
    if (g.cols == 0 || g.cols % 16 || p.n % g.cols) return DF11_ERR_INVALID;
    const uint64_t rows = p.n / g.cols;
    if (rows % kGemmM || g.interleave != kGemmM) return DF11_ERR_INVALID;
    if (g.batch < 1 || g.batch > DF11_GEMM_MAX_BATCH) return DF11_ERR_INVALID;
    if (g.x_stride < g.cols || g.x_stride % 8 || g.y_stride < rows) return DF11_ERR_INVALID;
    if (!aligned(g.x, 16) || !aligned(g.y, 4)) return DF11_ERR_ALIGN;
    df11_tensor v = t;
    v.out_bf16 = reinterpret_cast<uint16_t *>(16);  // not written; passes the output checks
    const df11_status st = validate(v);
    if (st != DF11_OK) return st;
    if (p.n == 0) continue;
    if (!t.chunk_counts || !t.decode_table) return DF11_ERR_UNSUPPORTED;
    if (p.threads_per_block != 256 || (p.chunk_bytes != 8 && p.chunk_bytes != 16))
      return DF11_ERR_UNSUPPORTED;
    if (C && C != p.chunk_bytes) return DF11_ERR_INVALID;
    C = p.chunk_bytes;
    ts[m] = t;
    gs[m] = g;
    ++m;
  }
  if (m == 0) return DF11_OK;
  {
    const df11_status st = check_devices(ts, m, gs);
    if (st != DF11_OK) return st;
  }
  for (int i = 0; i < m; ++i) {
    const df11_params &p = ts[i].params;
    KTensor &k = gb.t[i];
    k.bitstream = ts[i].bitstream;
    k.gaps = ts[i].gaps;
    k.chunk_counts = ts[i].chunk_counts;
    k.block_out_pos = ts[i].block_out_pos;
    k.luts = ts[i].luts;
    k.code_lengths = ts[i].code_lengths;
    k.sign_mantissa = ts[i].sign_mantissa;
    k.decode_table = ts[i].decode_table;
    k.total_bits = p.total_bits;
    k.n = (uint32_t)p.n;
    k.num_blocks = p.num_blocks;
    k.num_luts = p.num_luts;
    k.max_block_elems = p.max_block_elems;
    k.max_chunk_elems = p.max_chunk_elems;
    k.max_warp_elems = p.max_warp_elems;
    k.masked = p.max_len > (uint32_t)kWideBits ? 1u : 0u;
    k.x = gs[i].x;
    k.y = gs[i].y;
    k.cols = gs[i].cols;
    k.batch = gs[i].batch;
    k.x_stride = gs[i].x_stride;
    k.y_stride = gs[i].y_stride;
    const uint32_t rows = (uint32_t)(p.n / gs[i].cols), tpr = gs[i].cols / 16;
    gb.tile_begin[i] = tiles;
    tiles += rows / kGemmM * tpr;
    max_warp = max_warp > p.max_warp_elems ? max_warp : p.max_warp_elems;
    max_block = max_block > p.max_block_elems ? max_block : p.max_block_elems;
    max_batch = max_batch > gs[i].batch ? max_batch : gs[i].batch;
  }
  gb.count = m;
  gb.tile_begin[m] = tiles;
  gb.stage_bytes = region_bytes_for(max_warp);
  // a block's elements touch at most ceil(max_block / 2048) + 1 tiles (one
  // of them the tile the block before it began); the ring holds them
  gb.ring = (max_block + 2047u) / 2048u + 1u;
  gb.n_mma = (max_batch + 15u) & ~15u;
  // two accumulators up to 128 columns (room for four resident blocks),
  // one above: a thread block's range holds one or two pieces, so waiting
  // for the one accumulator to be emptied costs little
  gb.accs = 2 * gb.n_mma <= 128 ? 2u : 1u;
  gb.tmem_cols = 32;
  while (gb.tmem_cols < gb.accs * gb.n_mma) gb.tmem_cols <<= 1;
  // y = W x: clear the outputs first, in stream order
  ClearArgs ca{};
  for (int i = 0; i < m; ++i) {
    if (gs[i].accumulate) continue;
    ca.y[ca.count] = gs[i].y;
    ca.rows[ca.count] = (uint32_t)(ts[i].params.n / gs[i].cols);
    ca.batch[ca.count] = gs[i].batch;
    ca.stride[ca.count] = gs[i].y_stride;
    ++ca.count;
  }
  if (ca.count && launch_pdl(clear_rows_kernel, 148u, 256u, 0, s, ca) != DF11_OK)
    return DF11_ERR_CUDA;
  if (C == 8) return launch_gemm<8>(gb, s, 64);
  return launch_gemm<16>(gb, s, 65);
}

df11_status df11_build_decode_table(const uint32_t *luts, const uint8_t *code_lengths,
                                    uint32_t num_luts, void *out, df11_stream_t stream) {
  if (!luts || !code_lengths || !out) return DF11_ERR_NULL;
  if (!aligned(luts, 16) || !aligned(out, 16)) return DF11_ERR_ALIGN;
  if (num_luts < 1 || num_luts >= (1u << 24)) return DF11_ERR_FORMAT;
  const void *ptrs[3] = {luts, code_lengths, out};
  const df11_status st = df11_internal::check_device_pointers(ptrs, 3);
  if (st != DF11_OK) return st;
  df11_table_kernel<<<1, 256, 0, (cudaStream_t)stream>>>(luts, code_lengths, num_luts,
                                                           reinterpret_cast<uint4 *>(out));
  return cudaGetLastError() == cudaSuccess ? DF11_OK : DF11_ERR_CUDA;
}

df11_status df11_test_withhold_copies(int launches, uint32_t spin_limit) {
  if (launches < 0 || spin_limit < 1 || spin_limit > kSpinLimit) return DF11_ERR_INVALID;
  g_withhold_spin_limit.store(spin_limit);
  g_withhold_launches.store(launches);
  return DF11_OK;
}

size_t df11_shared_bytes(const df11_params *p) {
  if (!p || !supported(p->chunk_bytes, p->threads_per_block)) return 0;
  const uint32_t C = p->chunk_bytes, T = p->threads_per_block;
  const uint32_t region = region_bytes_for(p->max_warp_elems);
  const uint32_t stage = stage_bytes_for(p->max_block_elems);
  const uint32_t cols = column_bytes_for(p->max_chunk_elems);
  size_t most = 0;  // over both layouts and the three sign/mantissa stagings
  for (uint32_t c : {0u, cols}) {
    const size_t v[3] = {ws_shared_bytes(C, T, stage, region, c, false),
                         ws_shared_bytes(C, T, 0, region, c, false),
                         ws_shared_bytes(C, T, 0, region, c, true)};
    for (size_t x : v) most = x > most ? x : most;
  }
  return most;
}

int df11_supported(uint32_t chunk_bytes, uint32_t threads_per_block) {
  return supported(chunk_bytes, threads_per_block) ? 1 : 0;
}

const char *df11_status_string(df11_status s) {
  switch (s) {
    case DF11_OK: return "ok";
    case DF11_ERR_NULL: return "a required pointer is NULL";
    case DF11_ERR_ALIGN: return "a pointer misses its required alignment";
    case DF11_ERR_FORMAT: return "format parameters are inconsistent";
    case DF11_ERR_UNSUPPORTED: return "no kernel for this (chunk_bytes, threads_per_block)";
    case DF11_ERR_CUDA: return "a CUDA runtime call failed";
    case DF11_ERR_TOO_LARGE: return "size beyond the supported range";
    case DF11_ERR_INVALID: return "invalid argument";
    case DF11_ERR_NOMEM: return "host allocation failed";
    case DF11_ERR_DEVICE: return "a device pointer is not memory of the current device";
  }
  return "unknown status";
}

const char *df11_device_error_string(int32_t code) {
  switch (code) {
    case DF11_DEV_OK: return "ok";
    case DF11_DEV_ERR_COUNT: return "a block decoded a different element count than block_out_pos";
    case DF11_DEV_ERR_OVERRUN: return "a codeword ran past the next chunk's first codeword";
    case DF11_DEV_ERR_TABLE: return "invalid lookup-table entry or zero code length";
    case DF11_DEV_ERR_TIMEOUT: return "shared-memory copy did not complete in time";
    case DF11_DEV_ERR_CAPACITY: return "block or chunk holds more elements than its parameters allow";
  }
  return "unknown device error";
}

}  // extern "C"
