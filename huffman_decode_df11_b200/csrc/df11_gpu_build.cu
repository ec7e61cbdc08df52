// df11_gpu_build.cu -- the DF11 format builder on the GPU: compression of
// BF16 words already in device memory, byte for byte the output of the host
// builder (df11_build.cpp) on the same words.
//
// The pages compress offline on the host ("DFloat11无损压缩技术" (jsqmd.com)
// §2.2 items 1-2 give the recipe; "DFloat11重新定义LLM无损压缩的技术边界"
// (ocdem.com) §2.2 the lookup tables).  Here every step that touches the n
// elements runs on the device.  The codebook, a function of 256 counts, is
// computed on the host (df11_codebook.h, shared with the host builder), and
// with it the stream's length, the sum over exponents of count x code
// length, which sizes the outputs.  The device reads the elements twice,
// in tiles of 16384:
//   histogram  (phase 1) exponent counts per tile and in all, for up to 32
//              tensors a launch: four-bit counters in registers for a
//              window of 16 exponents around the mode of a first sample,
//              spread into byte counters after every 8 elements and summed
//              over the warp at the end of the tile; shared counters for
//              exponents outside the window.  Each tile's 256 counts are
//              kept (16 bits each);
//   tile bits  (phase 2) each tile's bit count, the dot product of its
//              counts with the code lengths, and an exclusive scan of them:
//              every tile's first bit, with no second pass over the
//              elements and no wait between thread blocks;
//   pack       one thread block per tile, in four steps of 4096 elements:
//              a block scan of the code lengths, the codewords ORed into a
//              shared-memory image of the step's words, written out
//              coalesced (the word two steps share is carried to the next
//              step; the first and last words of a tile, which it may share
//              with its neighbours, go to a side array).  Also written: the
//              sign/mantissa bytes, and for every chunk and block whose
//              first codeword start is one of the tile's elements, its gap,
//              first element and block position;
//   finish     the shared words from the side array, chunk counts from
//              first-element differences (n past the last codeword start),
//              the gaps packed eight to five bytes, block positions past
//              the last start, the paddings, the tables into the caller's
//              buffers, and the largest block, chunk and group of 32
//              chunks.
#include <cuda_runtime.h>

#include <atomic>
#include <cstdint>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <new>
#include <vector>

#include "df11.h"
#include "df11_device_check.h"
#include "df11_codebook.h"

namespace {

constexpr int kThreads = 256;
constexpr int kPerThread = 8;
constexpr int kPerCta = kThreads * kPerThread;  // elements per histogram step of a block

__device__ __forceinline__ uint32_t bswap32(uint32_t x) { return __byte_perm(x, 0, 0x0123); }
__device__ __forceinline__ uint32_t exponent(uint32_t x) { return (x >> 7) & 0xFFu; }

// The 8 words of elements i0 .. i0+7, two per 32-bit lane (element i0+2k in
// the low half of the k-th of .x .y .z .w); zero past n.
__device__ __forceinline__ uint4 load8(const uint16_t *w, uint64_t n, uint64_t i0, bool vec) {
  if (vec && i0 + kPerThread <= n) return __ldg(reinterpret_cast<const uint4 *>(w + i0));
  uint32_t u[4];
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const uint32_t a = i0 + 2 * k < n ? w[i0 + 2 * k] : 0u;
    const uint32_t b = i0 + 2 * k + 1 < n ? w[i0 + 2 * k + 1] : 0u;
    u[k] = a | (b << 16);
  }
  return make_uint4(u[0], u[1], u[2], u[3]);
}

__device__ __forceinline__ uint32_t word_of(const uint4 &v, int q) {
  return q == 0 ? v.x : q == 1 ? v.y : q == 2 ? v.z : v.w;
}

__device__ __forceinline__ uint32_t exponent_of(const uint4 &v, int k) {
  return (word_of(v, k >> 1) >> ((k & 1) ? 23 : 7)) & 0xFFu;
}

// entry e of a 256-entry table of 32-bit words, e the exponent of element k:
// the exponent field times 4 is the byte offset
__device__ __forceinline__ uint32_t entry_of(const uint32_t *table, const uint4 &v, int k) {
  const uint32_t off = (word_of(v, k >> 1) >> ((k & 1) ? 21 : 5)) & 0x3FCu;
  return *reinterpret_cast<const uint32_t *>(reinterpret_cast<const char *>(table) + off);
}

// how many of elements i0 .. i0+7 exist (0..8)
__device__ __forceinline__ uint32_t live_of(uint64_t i0, uint64_t n) {
  return i0 >= n ? 0u : (n - i0 >= (uint64_t)kPerThread ? (uint32_t)kPerThread : (uint32_t)(n - i0));
}

// ---- histogram -----------------------------------------------------------
// One launch counts the exponents of a batch of tensors (jobs): their tiles
// are numbered job after job, and block b takes tiles b, b + gridDim.x, and
// so on.  A tile
// is kTileSteps steps of 2048 elements (8 per thread of a 256-thread
// block), loaded in two halves so that one half is in flight while the
// other is counted: the tile's second half during the count of its first,
// the next tile's first half during the count of its second.  Per lane, 16
// four-bit counters in two registers (bins 0-7 and 8-15 of the warp's
// window, mode - 11 .. mode + 4, the mode taken over the first elements of
// the warp's lanes in the tile) take the 8 elements of a step; after each
// step they are spread into byte counters (four registers), which are
// summed over the warp at the end of the tile and added to the block's
// shared counters, one bin per lane (at most 64 counts per byte).
// Exponents outside the window go to the shared counters at once.  The
// shared counters alternate between two arrays from tile to tile, so that
// one barrier per tile separates a tile's adds from the reads of the tile
// before.
constexpr int kWindowBelow = 11;
constexpr int kTileSteps = 8;
constexpr int kHalfSteps = kTileSteps / 2;
constexpr uint32_t kTile = kTileSteps * kPerCta;  // elements per tile (16384)
constexpr int kHistJobs = 32;                     // jobs per histogram launch

struct HistJob {
  const uint16_t *w;
  uint64_t n;
  uint64_t tile_base;        // its first tile's number in the launch
  unsigned long long *hist;  // 256 counts, added to
  unsigned long long *last;  // its last element (its codeword ends the stream), or null
  uint16_t *tile_hist;       // 256 counts per tile (16 bits: at most 16384), or null
  uint32_t vec;              // w is 16-byte aligned
};

struct HistBatch {
  HistJob job[kHistJobs];
  int count;
  uint64_t tiles;  // of all its jobs
};

// The window's byte counters summed over the warp and added to the shared
// counters h, lane b (0-15) taking window bin b.  Byte j of counter
// register r holds bin (r >> 1) * 8 + 2 j + (r & 1): bin b is byte
// (b & 7) >> 1 of register (b >> 3) * 2 + (b & 1).
__device__ __forceinline__ void flush_window(uint32_t (&c)[4], int lo, uint32_t *h, int lane) {
  uint32_t even[4], odd[4];
#pragma unroll
  for (int r = 0; r < 4; ++r) {
    // two 16-bit sums per word (bytes 0 and 2, or 1 and 3): 32 lanes x 64 < 2^16
    even[r] = __reduce_add_sync(0xFFFFFFFFu, c[r] & 0x00FF00FFu);
    odd[r] = __reduce_add_sync(0xFFFFFFFFu, (c[r] >> 8) & 0x00FF00FFu);
    c[r] = 0;
  }
  const int b = lane & 15;
  const int r = ((b >> 3) << 1) | (b & 1), j = (b & 7) >> 1;
  const uint32_t ev = r == 0 ? even[0] : r == 1 ? even[1] : r == 2 ? even[2] : even[3];
  const uint32_t od = r == 0 ? odd[0] : r == 1 ? odd[1] : r == 2 ? odd[2] : odd[3];
  const uint32_t v = (((j & 1) ? od : ev) >> ((j & 2) ? 16 : 0)) & 0xFFFFu;
  const int e = lo + b;
  if (lane < 16 && v && e >= 0 && e < 256) atomicAdd(&h[e], v);
}

// One element whose exponent times 4 is e4: the window offset times 4 is
// sh = e4 - lo4 (wrapping below the window), and 1 << sh lands in the
// counter pair's low register for sh < 32, in the high one for 32 <= sh <
// 64; the clamped funnel shifts give 0 elsewhere.  `oow` collects the
// offsets: at least 64 once an element lies outside the window.
__device__ __forceinline__ void count_one(uint32_t e4, uint32_t lo4, uint32_t &n_lo,
                                          uint32_t &n_hi, uint32_t &oow) {
  const uint32_t sh = e4 - lo4;
  n_lo += __funnelshift_lc(0u, 1u, sh);
  n_hi += __funnelshift_lc(0u, 1u, sh - 32u);
  oow |= sh;
}

template <bool FULL>
__device__ __forceinline__ void count8(const uint4 &v, uint32_t live, uint32_t lo4,
                                       uint32_t (&c)[4], uint32_t *h) {
  uint32_t n_lo = 0, n_hi = 0, oow = 0;
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const uint32_t u = word_of(v, q);
    if (FULL || (uint32_t)(2 * q) < live) count_one((u >> 5) & 0x3FCu, lo4, n_lo, n_hi, oow);
    if (FULL || (uint32_t)(2 * q + 1) < live)
      count_one((u >> 21) & 0x3FCu, lo4, n_lo, n_hi, oow);
  }
  if (oow >= 64u) {  // rare: an exponent outside the window goes to the shared counters
#pragma unroll
    for (int k = 0; k < kPerThread; ++k) {
      const uint32_t e4 = (word_of(v, k >> 1) >> ((k & 1) ? 21 : 5)) & 0x3FCu;
      if ((FULL || (uint32_t)k < live) && e4 - lo4 >= 64u) atomicAdd(&h[e4 >> 2], 1u);
    }
  }
  c[0] += n_lo & 0x0F0F0F0Fu;
  c[1] += (n_lo >> 4) & 0x0F0F0F0Fu;
  c[2] += n_hi & 0x0F0F0F0Fu;
  c[3] += (n_hi >> 4) & 0x0F0F0F0Fu;
}

// Steps s0 .. s0 + kHalfSteps - 1 of the tile at element t0 of a job
__device__ __forceinline__ void load_half(uint4 (&v)[kHalfSteps], const HistJob &J, uint64_t t0,
                                          int s0, uint32_t me) {
#pragma unroll
  for (int st = 0; st < kHalfSteps; ++st)
    v[st] = load8(J.w, J.n, t0 + (uint64_t)(s0 + st) * kPerCta + me, J.vec != 0);
}

__device__ __forceinline__ void count_half(const uint4 (&v)[kHalfSteps], bool full, uint64_t t0,
                                           int s0, uint64_t n, uint32_t me, uint32_t lo4,
                                           uint32_t (&c)[4], uint32_t *h) {
  if (full) {
#pragma unroll
    for (int st = 0; st < kHalfSteps; ++st) count8<true>(v[st], kPerThread, lo4, c, h);
  } else {
#pragma unroll
    for (int st = 0; st < kHalfSteps; ++st)
      count8<false>(v[st], live_of(t0 + (uint64_t)(s0 + st) * kPerCta + me, n), lo4, c, h);
  }
}

// Per job: hist[e] += the count of exponent e (64-bit, device-wide);
// tile_hist, if not null, each tile's 256 counts; last, if not null, the
// last element.
__global__ void __launch_bounds__(kThreads, 4) hist_kernel(const __grid_constant__ HistBatch hb) {
  __shared__ uint32_t h[2][256];
  static_assert(kThreads == 256, "a thread per exponent value");
  const int lane = threadIdx.x & 31;
  const uint32_t me = threadIdx.x * kPerThread;
  if (blockIdx.x == 0 && threadIdx.x < (unsigned)hb.count) {
    const HistJob &J = hb.job[threadIdx.x];
    if (J.last && J.n) *J.last = J.w[J.n - 1];
  }
  h[0][threadIdx.x] = 0;
  h[1][threadIdx.x] = 0;
  __syncthreads();
  uint64_t t = blockIdx.x;  // the grid has at most as many blocks as tiles
  int ji = 0;
  while (ji + 1 < hb.count && t >= hb.job[ji + 1].tile_base) ++ji;
  uint4 va[kHalfSteps], vb[kHalfSteps];
  load_half(va, hb.job[ji], (t - hb.job[ji].tile_base) * kTile, 0, me);
  uint32_t total = 0;  // exponent threadIdx.x over the block's tiles of job ji
  for (int p = 0;; p ^= 1) {
    const HistJob &J = hb.job[ji];
    const uint64_t t0 = (t - J.tile_base) * kTile;
    const bool full = t0 + kTile <= J.n;
    load_half(vb, J, t0, kHalfSteps, me);
    const uint64_t tn = t + gridDim.x;
    int jn = ji;
    while (jn + 1 < hb.count && tn >= hb.job[jn + 1].tile_base) ++jn;
    // the window: around the most frequent exponent among the lanes' first
    // elements (256 for a lane past the end: no exponent)
    int lo;
    {
      const uint32_t key = t0 + me < J.n ? exponent(va[0].x) : 256u;
      const uint32_t peers = __match_any_sync(0xFFFFFFFFu, key);
      const uint32_t best = __reduce_max_sync(0xFFFFFFFFu, ((uint32_t)__popc(peers) << 16) | key);
      lo = (int)(best & 0x1FFu) - kWindowBelow;
    }
    const uint32_t lo4 = (uint32_t)(4 * lo);
    uint32_t *hp = h[p];
    uint32_t c[4] = {0, 0, 0, 0};
    count_half(va, full, t0, 0, J.n, me, lo4, c, hp);
    if (tn < hb.tiles) load_half(va, hb.job[jn], (tn - hb.job[jn].tile_base) * kTile, 0, me);
    count_half(vb, full, t0, kHalfSteps, J.n, me, lo4, c, hp);
    flush_window(c, lo, hp, lane);
    __syncthreads();
    const uint32_t v = hp[threadIdx.x];
    hp[threadIdx.x] = 0;
    if (J.tile_hist) J.tile_hist[(t - J.tile_base) * 256 + threadIdx.x] = (uint16_t)v;
    total += v;
    if (tn >= hb.tiles || jn != ji) {
      if (total) atomicAdd(&J.hist[threadIdx.x], (unsigned long long)total);
      total = 0;
    }
    if (tn >= hb.tiles) break;
    t = tn;
    ji = jn;
  }
}

// ---- phase 2 jobs --------------------------------------------------------
// Phase 2 of a batch runs as one launch per kernel over all its tensors;
// each tensor is a job, described in device memory (copied there with the
// code tables).  Tiles are numbered through the batch, job after job.

// {codeword << 8 | length} for codes of up to 24 bits; 0x80 | length for
// longer ones, whose codewords are in a second table
constexpr uint32_t kLongCode = 0x80u;
constexpr int kPackedCodeBits = 24;

struct Job {
  const uint16_t *w;  // the elements
  uint64_t n;
  uint32_t vec;       // w is 16-byte aligned
  uint32_t longs;     // the code has codewords above 24 bits
  uint64_t tiles, tile_base;  // tiles, and the first one's number in the batch
  const uint16_t *tile_hist;  // phase 1: 256 counts per tile
  uint32_t *tile_bits;
  unsigned long long *tile_start;  // tiles + 1 (the total last)
  uint32_t *edge;                  // per tile: its first and last word when shared
  const uint32_t *tab;  // 256 packed entries, 256 codewords, the luts, 256 code lengths
  // outputs
  uint32_t *bs32;
  uint8_t *sm, *gaps_packed, *counts, *code_lengths;
  uint32_t *bpos, *luts;
  // scratch: per chunk its first element and gap; the largest block, chunk
  // and group of 32 chunks
  uint32_t *first_elem;
  uint8_t *gap;
  unsigned int *maxima;
  uint64_t chunks, total, last_start;
  uint32_t num_blocks, luts_vec4;
  uint32_t chunk_bits, block_bits;    // 8 C and 8 C T
  uint32_t chunk_words, block_words;  // chunk_bits / 32, block_bits / 32
  uint64_t chunk_magic, block_magic;  // ceil(2^64 / words) (words >= 2)
  uint64_t fin_threads;               // threads of the finish kernel
  uint8_t *zero[4];                   // byte ranges to clear: the paddings
  uint32_t zero_bytes[4];
};

// floor(x / d) for x < 2^32 by a multiply-high with ceil(2^64 / d): the
// error, below x / 2^64 < 2^-32, never crosses an integer (d < 2^32)
__device__ __forceinline__ uint64_t div_words(uint32_t x, uint32_t d, uint64_t magic) {
  return d == 1 ? x : __umul64hi((uint64_t)x, magic);
}

// ---- tile bits -----------------------------------------------------------
// Grid (x, job): one warp per tile, lane l takes exponents 8l .. 8l+7.
__global__ void __launch_bounds__(256) tile_bits_kernel(const Job *jobs) {
  const Job &J = jobs[blockIdx.y];
  __shared__ uint32_t len_s[256];
  len_s[threadIdx.x] = J.tab[threadIdx.x] & 0x3Fu;
  __syncthreads();
  const int lane = threadIdx.x & 31;
  const uint64_t t = blockIdx.x * 8ull + (threadIdx.x >> 5);
  if (t >= J.tiles) return;
  const uint4 hv = reinterpret_cast<const uint4 *>(J.tile_hist + t * 256)[lane];
  uint32_t sum = 0;
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const uint32_t x = word_of(hv, q);
    sum += (x & 0xFFFFu) * len_s[8 * lane + 2 * q] + (x >> 16) * len_s[8 * lane + 2 * q + 1];
  }
  sum = __reduce_add_sync(0xFFFFFFFFu, sum);  // at most 16384 x 32 bits
  if (lane == 0) J.tile_bits[t] = sum;
}

// Exclusive scan of a job's tile bits into their first bits, the total at
// tile_start[tiles]; one thread block per job, each thread a contiguous run.
constexpr int kScanThreads = 1024;

__global__ void __launch_bounds__(kScanThreads) scan_kernel(const Job *jobs) {
  const Job &J = jobs[blockIdx.x];
  __shared__ unsigned long long warp_tot[kScanThreads / 32];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const uint64_t count = J.tiles;
  const uint64_t per = (count + kScanThreads - 1) / kScanThreads;
  const uint64_t b = threadIdx.x * per;
  const uint64_t e = b + per < count ? b + per : count;
  unsigned long long mine = 0;
  for (uint64_t i = b; i < e; ++i) mine += J.tile_bits[i];
  unsigned long long incl = mine;
#pragma unroll
  for (int d = 1; d < 32; d <<= 1) {
    const unsigned long long v = __shfl_up_sync(0xFFFFFFFFu, incl, d);
    if (lane >= d) incl += v;
  }
  if (lane == 31) warp_tot[warp] = incl;
  __syncthreads();
  unsigned long long run = incl - mine;
  for (int j = 0; j < warp; ++j) run += warp_tot[j];
  for (uint64_t i = b; i < e; ++i) {
    J.tile_start[i] = run;
    run += J.tile_bits[i];
  }
  if (threadIdx.x == kScanThreads - 1) J.tile_start[count] = run;
}

// ---- pack ----------------------------------------------------------------
// A thread block packs a tile in steps of 16 units of 256 elements; warp w
// packs units w and w + 8 of a step, a unit being 8 consecutive elements
// per lane.  Bits are counted relative to the step's origin, the first bit
// of the word its first codeword begins in; a step spans at most 4096 x 32
// bits plus the 31 before its start.
constexpr int kUnit = 32 * kPerThread;           // elements per unit
constexpr int kStepUnits = 2 * (kThreads / 32);  // units per step
constexpr uint32_t kStep = kStepUnits * kUnit;   // elements per step (4096)
constexpr int kStepsPerTile = kTile / kStep;
constexpr int kStepWords = kStep + 2;            // words a step's codewords can touch
static_assert(kTile % kStep == 0, "a tile is whole steps");

// the job whose tiles hold batch tile t (jobs in tile order)
__device__ __forceinline__ int job_of(const Job *jobs, int count, uint64_t t) {
  int lo = 0, hi = count - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (jobs[mid].tile_base <= t) lo = mid;
    else hi = mid - 1;
  }
  return lo;
}

// What a lane knows of its 8 elements of one unit.
struct Seg {
  uint4 v;           // the words
  uint32_t tt[8];    // packed table entries (0 past n)
  uint32_t live;     // elements that exist
  uint32_t mine;     // their bits
  bool longs;        // one of them has a codeword above 24 bits
};

// Table entries of the lane's elements (0 past n), their bits and, when the
// code has them, whether one is above 24 bits.
template <bool FULL, bool LONGS>
__device__ __forceinline__ void seg_lengths(Seg &g, const uint32_t *tab_s) {
  uint32_t mine = 0, any = 0;
#pragma unroll
  for (int k = 0; k < kPerThread; ++k) {
    const uint32_t t = (FULL || (uint32_t)k < g.live) ? entry_of(tab_s, g.v, k) : 0u;
    g.tt[k] = t;
    mine += t & 0x3Fu;
    if (LONGS) any |= t;
  }
  g.mine = mine;
  g.longs = LONGS && (any & kLongCode) != 0;
}

// The lane's codewords, MSB first, ORed into the image from bit `rel` on:
// up to 64 bits (the usual case) gathered in two registers and placed with
// up to three ORs, longer runs word by word.
__device__ __forceinline__ void seg_pack(const Seg &g, uint32_t rel, bool any_long,
                                         const uint32_t *code_s, uint32_t *image) {
  if (!g.mine) return;
  uint32_t cw[kPerThread], ln[kPerThread];
#pragma unroll
  for (int k = 0; k < kPerThread; ++k) {
    ln[k] = g.tt[k] & 0x3Fu;
    cw[k] = g.tt[k] >> 8;
  }
  if (any_long) {  // warp-uniform; rare
#pragma unroll
    for (int k = 0; k < kPerThread; ++k)
      if (ln[k] > (uint32_t)kPackedCodeBits) cw[k] = entry_of(code_s, g.v, k);
  }
  const uint32_t o = rel & 31u, wk = rel >> 5;
  if (g.mine <= 64) {
    uint32_t hi = 0, lo = 0;
#pragma unroll
    for (int k = 0; k < kPerThread; ++k) {  // (hi:lo) = (hi:lo) << ln | cw, ln <= 32
      hi = __funnelshift_lc(lo, hi, ln[k]);
      lo = __funnelshift_lc(0u, lo, ln[k]) | cw[k];
    }
    // left-align the `mine` bits: first bit at bit 63
    const uint32_t s = 64u - g.mine;
    uint32_t ah, al;
    if (s >= 32) {
      ah = lo << (s - 32);
      al = 0;
    } else {
      ah = __funnelshift_l(lo, hi, s);
      al = lo << s;
    }
    atomicOr(&image[wk], ah >> o);
    if (o + g.mine > 32) atomicOr(&image[wk + 1], __funnelshift_r(al, ah, o));
    if (o + g.mine > 64) atomicOr(&image[wk + 2], al << (32 - o));
  } else {
    // `cur` holds the pending bits left-aligned, `nb` of them
    uint32_t w = wk, nb = o, cur = 0;
    bool first = true;
#pragma unroll
    for (int k = 0; k < kPerThread; ++k) {
      if (ln[k]) {
        const uint32_t tot = nb + ln[k];
        if (tot >= 32) {
          const uint32_t t = cur | (cw[k] >> (tot - 32));
          if (first) atomicOr(&image[w], t);  // the previous lane may own its first bits
          else image[w] = t;
          first = false;
          ++w;
          nb = tot - 32;
          cur = __funnelshift_lc(0u, cw[k], 32 - nb);  // 0 when nb == 0
        } else {
          cur |= cw[k] << (32 - tot);
          nb = tot;
        }
      }
    }
    if (nb) atomicOr(&image[w], cur);  // the last, partial word, which the next lane may share
  }
}

// Sign/mantissa bytes of the lane's elements: bit 15 -> bit 7, bits 0-6
// kept; two per word.
__device__ __forceinline__ void seg_sign_mantissa(uint8_t *sm, const Seg &g, uint64_t i0) {
  if (!g.live) return;
  uint32_t sm2[4];
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const uint32_t t = word_of(g.v, q);
    sm2[q] = (t & 0x007F007Fu) | ((t >> 8) & 0x00800080u);  // bytes 0 and 2
  }
  const uint2 smv = make_uint2(__byte_perm(sm2[0], sm2[1], 0x6420),
                               __byte_perm(sm2[2], sm2[3], 0x6420));
  if (g.live == kPerThread) {
    *reinterpret_cast<uint2 *>(sm + i0) = smv;
  } else {
    for (uint32_t k = 0; k < g.live; ++k)
      sm[i0 + k] = (uint8_t)((k < 4 ? smv.x : smv.y) >> (8 * (k & 3)));
  }
}

// The element a boundary goes to: the first of the step whose codeword
// starts at or after bit r (from the step's origin), and that start.  The
// step's 512 lane segments of 8 elements, in element order, have their
// first bits in seg_start and their words in seg_words: a binary search
// finds the last segment that starts before r, a walk over its lengths the
// element.  The caller guarantees that some element of the step starts at
// or after r.
__device__ __forceinline__ uint32_t boundary_element(int r, const int *seg_start,
                                                     const uint4 *seg_words,
                                                     const uint32_t *tab_s, int *start) {
  int s = 0;
#pragma unroll
  for (int d = kStepUnits * 32 / 2; d; d >>= 1)
    if (seg_start[s + d] < r) s += d;
  int p = seg_start[s];
  uint32_t k = 0;
  if (p < r) {  // else s is 0 and the step's first element takes the boundary
    const uint4 v = seg_words[s];
#pragma unroll
    for (int j = 0; j < kPerThread; ++j) {
      if (p < r) {
        p += (int)(entry_of(tab_s, v, j) & 0x3Fu);
        ++k;
      }
    }
  }
  *start = p;
  return (uint32_t)s * kPerThread + k;  // k = 8: the next segment's first element
}

// The chunks and blocks whose first codeword start is in a step: those
// that begin after the start of the element before the step (any, for the
// first step of the tensor) and at or before the start of its last
// element.  The first boundary after a start p is floor(p / chunk bits) +
// 1; bit offsets stay below 2^37, so p / 32 fits 32 bits and floor(p / (32
// m)) = floor(floor(p / 32) / m).  r0 and rq0 are the first chunk and block
// boundary from the step's origin.
struct StepRanges {
  unsigned long long c_lo, q_lo;
  uint32_t nc, nq;
  int r0, rq0;
};

__device__ __forceinline__ StepRanges step_ranges(const Job &J, unsigned long long origin,
                                                  uint32_t lead, uint32_t bits,
                                                  uint32_t prev_len, uint32_t last_len,
                                                  bool tensor_first) {
  const unsigned long long pos = origin + lead;
  const uint32_t hi_w = (uint32_t)((pos + bits - last_len) >> 5);
  const uint32_t lo_w = (uint32_t)((pos - prev_len) >> 5);
  StepRanges r;
  r.c_lo = tensor_first ? 0 : div_words(lo_w, J.chunk_words, J.chunk_magic) + 1;
  r.q_lo = tensor_first ? 0 : div_words(lo_w, J.block_words, J.block_magic) + 1;
  const unsigned long long c_hi = div_words(hi_w, J.chunk_words, J.chunk_magic);
  const unsigned long long q_hi = div_words(hi_w, J.block_words, J.block_magic);
  r.nc = (uint32_t)(c_hi + 1 - r.c_lo);
  r.nq = q_hi + 1 > r.q_lo ? (uint32_t)(q_hi + 1 - r.q_lo) : 0u;
  r.r0 = (int)((long long)(r.c_lo * J.chunk_bits) - (long long)origin);
  r.rq0 = (int)((long long)(r.q_lo * J.block_bits) - (long long)origin);
  return r;
}

// Tiles are claimed one at a time from a counter, in batch order, so that
// the blocks finish together.  A tile is packed in steps of 4096 elements,
// each with its own image; two images alternate, so that the one a step
// writes out is cleared during the next step, before the step after that
// packs into it.  A step whose last word is partial (and not the tile's
// last step) hands it to the next step, which ORs it into its first word.
// The block keeps its job's descriptor and code tables in shared memory
// and reloads them when a claimed tile belongs to another job.
__global__ void __launch_bounds__(kThreads, 3) pack_kernel(const Job *jobs, int count,
                                                        uint64_t all_tiles,
                                                        unsigned long long *counter) {
  __shared__ uint32_t tab_s[256];
  __shared__ uint32_t code_s[256];
  __shared__ uint32_t images[2][kStepWords];
  __shared__ uint32_t unit_bits[kStepUnits];  // bits of each unit
  __shared__ int seg_start[kStepUnits * 32];  // first bit of each lane segment
  __shared__ uint4 seg_words[kStepUnits * 32];
  __shared__ uint32_t carry[2];               // a step's partial last word
  __shared__ uint32_t prev_len;               // codeword length of the element before the step
  __shared__ StepRanges ranges;               // of a whole step, from its last thread
  __shared__ unsigned long long claim;
  __shared__ Job J;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  if (tid == 0) claim = atomicAdd(counter, 1ull);
  for (int j = tid; j < 2 * kStepWords; j += kThreads) (&images[0][0])[j] = 0;
  __syncthreads();
  uint64_t g = claim;  // the tile, numbered through the batch
  if (g >= all_tiles) return;
  int job = job_of(jobs, count, g);
  static_assert(sizeof(Job) % 8 == 0, "descriptor copied in 8-byte words");
  for (int j = tid; j < (int)(sizeof(Job) / 8); j += kThreads)
    reinterpret_cast<unsigned long long *>(&J)[j] =
        reinterpret_cast<const unsigned long long *>(&jobs[job])[j];
  __syncthreads();
  tab_s[tid] = J.tab[tid];
  code_s[tid] = J.tab[256 + tid];
  uint64_t t = g - J.tile_base;  // the tile within its job
  int q = 0;                     // the step within the tile
  const uint32_t lane_off = (uint32_t)warp * kUnit + (uint32_t)lane * kPerThread;
  // the step's words (units w and w + 8), and for thread 0 the element before
  uint4 na, nb;
  uint32_t nprev = 0;
  {
    const uint64_t i = t * kTile + lane_off;
    na = load8(J.w, J.n, i, J.vec);
    nb = load8(J.w, J.n, i + kStep / 2, J.vec);
    if (tid == kThreads - 1 && t) nprev = J.w[t * kTile - 1];
  }
  int cur = 0;
  uint32_t stale = 0;  // words the other image holds from the step before
  unsigned long long pos = J.tile_start[t];  // the step's first bit
  __syncthreads();  // the tables
  for (;;) {
    uint32_t *image = images[cur];
    // element indices fit 32 bits (n < 2^32); a lane's index may wrap only
    // in the step that ends the tensor, where such a lane has no elements
    const uint32_t step_first = (uint32_t)(t * kTile) + (uint32_t)q * kStep;
    const uint32_t n = (uint32_t)J.n;
    Seg A, B;
    A.v = na;
    B.v = nb;
    const uint32_t prev_word = nprev;
    const uint32_t i_a = step_first + lane_off, i_b = i_a + kStep / 2;
    const bool whole = n - step_first >= kStep;  // uniform
    A.live = whole ? kPerThread : live_of((uint64_t)step_first + lane_off, n);
    B.live = whole ? kPerThread : live_of((uint64_t)step_first + lane_off + kStep / 2, n);
    if (whole) {
      if (J.longs) {
        seg_lengths<true, true>(A, tab_s);
        seg_lengths<true, true>(B, tab_s);
      } else {
        seg_lengths<true, false>(A, tab_s);
        seg_lengths<true, false>(B, tab_s);
      }
    } else {
      seg_lengths<false, true>(A, tab_s);
      seg_lengths<false, true>(B, tab_s);
    }
    // both units' bits scanned over the warp at once, 16 bits each (a unit
    // holds at most 8192)
    const uint32_t both = A.mine | (B.mine << 16);
    uint32_t incl = both;
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
      const uint32_t y = __shfl_up_sync(0xFFFFFFFFu, incl, d);
      if (lane >= d) incl += y;
    }
    const uint32_t excl = incl - both;
    if (lane == 31) {
      unit_bits[warp] = incl & 0xFFFFu;
      unit_bits[warp + 8] = incl >> 16;
    }
    __syncthreads();
    {
      uint32_t *other = images[cur ^ 1];
      for (uint32_t j = tid; j < stale; j += kThreads) other[j] = 0;
    }
    // every warp scans the 16 unit counts
    const uint32_t ub = lane < kStepUnits ? unit_bits[lane] : 0u;
    uint32_t ui = ub;
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
      const uint32_t y = __shfl_up_sync(0xFFFFFFFFu, ui, d);
      if (lane >= d) ui += y;
    }
    const uint32_t bits = __shfl_sync(0xFFFFFFFFu, ui, 31);
    const uint32_t off_a = __shfl_sync(0xFFFFFFFFu, ui - ub, warp);
    const uint32_t off_b = __shfl_sync(0xFFFFFFFFu, ui - ub, warp + 8);
    const unsigned long long origin = pos & ~31ull;
    const uint32_t lead = (uint32_t)(pos & 31u);
    if (tid == kThreads - 1) {
      // the element before the step; for a whole step this thread's last
      // element is the step's last
      const uint32_t pl = step_first ? tab_s[exponent(prev_word)] & 0x3Fu : 0u;
      prev_len = pl;
      if (whole) ranges = step_ranges(J, origin, lead, bits, pl, B.tt[kPerThread - 1] & 0x3Fu,
                                      step_first == 0);
    }
    const uint32_t rel_a = lead + off_a + (excl & 0xFFFFu), rel_b = lead + off_b + (excl >> 16);
    seg_pack(A, rel_a, J.longs && __any_sync(0xFFFFFFFFu, A.longs), code_s, image);
    seg_pack(B, rel_b, J.longs && __any_sync(0xFFFFFFFFu, B.longs), code_s, image);
    seg_start[warp * 32 + lane] = (int)rel_a;
    seg_start[(warp + 8) * 32 + lane] = (int)rel_b;
    seg_words[warp * 32 + lane] = A.v;
    seg_words[(warp + 8) * 32 + lane] = B.v;
    seg_sign_mantissa(J.sm, A, i_a);
    seg_sign_mantissa(J.sm, B, i_b);
    const bool last_step = q + 1 == kStepsPerTile || n - step_first <= kStep;
    if (last_step && tid == 0) claim = atomicAdd(counter, 1ull);
    __syncthreads();  // the image is complete; the step's starts and words are in place
    // the next step: of this tile, or the next claimed tile
    const uint64_t gn = last_step ? claim : g;
    const int jn = !last_step ? job : gn < all_tiles ? job_of(jobs, count, gn) : job;
    const uint64_t tn = !last_step ? t : gn - jobs[jn].tile_base;
    const int qn = last_step ? 0 : q + 1;
    if (gn < all_tiles) {  // in flight while this step is finished
      const Job &N = jobs[jn];
      const uint16_t *w = last_step ? N.w : J.w;
      const uint64_t n = last_step ? N.n : J.n;
      const bool vec = last_step ? N.vec != 0 : J.vec != 0;
      const uint64_t first_n = tn * kTile + (uint64_t)qn * kStep;
      const uint64_t i = first_n + lane_off;
      na = load8(w, n, i, vec);
      nb = load8(w, n, i + kStep / 2, vec);
      if (tid == kThreads - 1 && first_n) nprev = w[first_n - 1];
    }
    // the chunks and blocks whose first codeword start is in this step, one
    // thread each (a step that ends the tensor works out its ranges here)
    {
      StepRanges rg;
      if (whole) {
        rg = ranges;
      } else {
        const uint32_t e_last = n - step_first - 1;
        const uint32_t last_len =
            tab_s[exponent_of(seg_words[e_last / kPerThread], e_last % kPerThread)] & 0x3Fu;
        rg = step_ranges(J, origin, lead, bits, prev_len, last_len, step_first == 0);
      }
      for (uint32_t b = tid; b < rg.nc + rg.nq; b += kThreads) {
        const bool chunk = b < rg.nc;
        const int r = chunk ? rg.r0 + (int)(b * J.chunk_bits)
                            : rg.rq0 + (int)((b - rg.nc) * J.block_bits);
        int start;
        const uint32_t e = boundary_element(r, seg_start, seg_words, tab_s, &start);
        const uint32_t elem = (uint32_t)step_first + e;
        if (chunk) {
          const uint64_t idx = rg.c_lo + b;
          if (idx < J.chunks) {
            J.gap[idx] = (uint8_t)(start - r);
            J.first_elem[idx] = elem;
          }
        } else {
          const uint64_t idx = rg.q_lo + (b - rg.nc);
          if (idx < J.num_blocks) J.bpos[idx] = elem;
        }
      }
    }
    // words out; the first word of a step after the first holds the
    // previous step's partial last word too
    const uint32_t end_bits = lead + bits;
    const uint32_t nwords = (end_bits + 31) >> 5;
    const bool end_partial = (end_bits & 31u) != 0;
    const uint64_t base = origin >> 5;
    // the step's first and last words, which it may share, by the first
    // and last thread; the rest stored plainly
    const uint32_t last_w = nwords - 1;
    if (tid == 0 || tid == kThreads - 1) {
      const uint32_t j = tid == 0 ? 0u : last_w;
      if (tid == 0 || last_w != 0) {  // one word: thread 0 takes it
        uint32_t val = image[j];
        if (j == 0 && q && lead) val |= carry[cur ^ 1];
        const bool head = j == 0 && q == 0 && lead, tail = j == last_w && end_partial;
        if (tail && !last_step) {
          carry[cur] = val;
        } else {
          if (head) J.edge[2 * t] = val;  // shared with the tile before
          if (tail) J.edge[2 * t + 1] = val;  // shared with the tile after
          if (!head && !tail) J.bs32[base + j] = bswap32(val);
        }
      }
    }
    {
      uint32_t *dst = J.bs32 + base;
      for (uint32_t j = tid + 1; j < last_w; j += kThreads) dst[j] = bswap32(image[j]);
    }
    if (gn >= all_tiles) break;  // uniform
    if (jn != job) {  // another tensor: its descriptor and tables
      __syncthreads();
      for (int j = tid; j < (int)(sizeof(Job) / 8); j += kThreads)
        reinterpret_cast<unsigned long long *>(&J)[j] =
            reinterpret_cast<const unsigned long long *>(&jobs[jn])[j];
      __syncthreads();
      tab_s[tid] = J.tab[tid];
      code_s[tid] = J.tab[256 + tid];
      __syncthreads();
      job = jn;
    }
    stale = nwords;
    cur ^= 1;
    pos = last_step ? J.tile_start[tn] : pos + bits;
    g = gn;
    t = tn;
    q = qn;
  }
}

// ---- finish --------------------------------------------------------------
// first element of chunk c: n for the chunks that begin after the last
// codeword start (no element starts at or after them) and for the end entry
__device__ __forceinline__ uint32_t chunk_first(const Job &J, uint64_t c) {
  return c * J.chunk_bits > J.last_start ? (uint32_t)J.n : J.first_elem[c];
}

// entry b of block_out_pos as the format stores it: n for the blocks after
// the last codeword start and for the end entry
__device__ __forceinline__ uint32_t block_pos(const Job &J, uint64_t b) {
  if (b >= J.num_blocks || b * (uint64_t)J.block_bits > J.last_start) return (uint32_t)J.n;
  return J.bpos[b];
}

// Grid (x, job).  A job's threads in three ranges: one per group of 8 chunks
// (5 packed gap bytes; chunks is a multiple of 128), one per entry of
// block_out_pos, one per tile; then all of them over the paddings and
// tables.  Rewriting an entry of block_out_pos with its block_pos leaves its
// block_pos unchanged, so a neighbour may read it before or after the
// rewrite.
__global__ void finish_kernel(const Job *jobs) {
  const Job &J = jobs[blockIdx.y];
  const uint64_t i = blockIdx.x * 256ull + threadIdx.x;
  const uint64_t groups = J.chunks / 8;
  if (i < groups) {
    const uint64_t c0 = i * 8;
    unsigned long long v = 0;
    uint32_t mc = 0;
    const uint32_t f0 = chunk_first(J, c0);
    uint32_t f = f0;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const uint64_t c = c0 + j, cb = c * J.chunk_bits;
      // a chunk that begins inside the last codeword: the distance to the end
      const uint32_t gv =
          cb > J.last_start ? (cb < J.total ? (uint32_t)(J.total - cb) : 0u) : J.gap[c];
      const uint32_t fn = chunk_first(J, c + 1);
      const uint32_t k = fn - f;
      f = fn;
      J.counts[c] = (uint8_t)k;
      mc = mc > k ? mc : k;
      v = (v << 5) | gv;
    }
#pragma unroll
    for (int j = 0; j < 5; ++j) J.gaps_packed[i * 5 + j] = (uint8_t)(v >> (32 - 8 * j));
    atomicMax(&J.maxima[1], mc);
    if (c0 % 32 == 0) {
      const uint64_t e = c0 + 32 < J.chunks ? c0 + 32 : J.chunks;
      atomicMax(&J.maxima[2], chunk_first(J, e) - f0);
    }
  } else if (i - groups <= J.num_blocks) {
    const uint64_t b = i - groups;
    const uint32_t here = block_pos(J, b);
    if (b < J.num_blocks) atomicMax(&J.maxima[0], block_pos(J, b + 1) - here);
    J.bpos[b] = here;
  } else if (i - groups - J.num_blocks - 1 < J.tiles) {
    // the word a tile shares with the one before it, and the stream's last
    // word when it is partial (unless that is the same word)
    const uint64_t t = i - groups - J.num_blocks - 1;
    const unsigned long long s = J.tile_start[t], e = J.tile_start[t + 1];
    const bool head = (s & 31u) != 0;
    if (head) J.bs32[s >> 5] = bswap32(J.edge[2 * (t - 1) + 1] | J.edge[2 * t]);
    if (t + 1 == J.tiles && (e & 31u) && !(head && (s >> 5) == (e >> 5)))
      J.bs32[e >> 5] = bswap32(J.edge[2 * t + 1]);
  }
  const uint64_t all = (uint64_t)gridDim.x * 256;
  const uint4 *luts_src = reinterpret_cast<const uint4 *>(J.tab + 512);
  for (uint64_t j = i; j < J.luts_vec4; j += all) reinterpret_cast<uint4 *>(J.luts)[j] = luts_src[j];
  if (i < 256) J.code_lengths[i] = reinterpret_cast<const uint8_t *>(J.tab + 512 + 4 * J.luts_vec4)[i];
  // paddings: each at most a block of the bitstream plus 16 bytes
  for (int k = 0; k < 4; ++k)
    for (uint64_t j = i; j < J.zero_bytes[k]; j += all) J.zero[k][j] = 0;
}

bool grid_for(uint64_t items, uint64_t per_cta, unsigned *grid) {
  const uint64_t g = (items + per_cta - 1) / per_cta;
  if (g >= (1ull << 31)) return false;
  *grid = (unsigned)(g ? g : 1);
  return true;
}

uint64_t round256(uint64_t x) { return (x + 255) & ~255ull; }

constexpr int kMaxDevices = 64;

// resident thread blocks of kThreads on the current device (at least 1),
// queried once per kernel and device
template <class K>
uint64_t resident(K kernel) {
  static std::atomic<uint64_t> known[kMaxDevices];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) dev = -1;
  if (dev >= 0) {
    const uint64_t v = known[dev].load(std::memory_order_relaxed);
    if (v) return v;
  }
  int sms = 0, per_sm = 0;
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev < 0 ? 0 : dev) !=
          cudaSuccess ||
      sms < 1)
    sms = 1;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, kThreads, 0) != cudaSuccess ||
      per_sm < 1)
    per_sm = 1;
  const uint64_t v = (uint64_t)sms * per_sm;
  if (dev >= 0) known[dev].store(v, std::memory_order_relaxed);
  return v;
}

// The builder's device scratch comes from a memory pool of the library's
// own per device, allocated and freed in stream order; the pool keeps what
// it has reserved, so repeated builds neither map memory nor synchronise
// the device to release it.
cudaError_t scratch_alloc(void **p, size_t bytes, cudaStream_t s) {
  static std::mutex mu;
  static cudaMemPool_t pools[kMaxDevices] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaMalloc(p, bytes);
  cudaMemPool_t pool;
  {
    std::lock_guard<std::mutex> lock(mu);
    if (!pools[dev]) {
      cudaMemPoolProps props = {};
      props.allocType = cudaMemAllocationTypePinned;
      props.location.type = cudaMemLocationTypeDevice;
      props.location.id = dev;
      if ((e = cudaMemPoolCreate(&pools[dev], &props)) != cudaSuccess) {
        pools[dev] = nullptr;
        return e;
      }
      uint64_t keep = UINT64_MAX;
      cudaMemPoolSetAttribute(pools[dev], cudaMemPoolAttrReleaseThreshold, &keep);
    }
    pool = pools[dev];
  }
  return cudaMallocFromPoolAsync(p, bytes, pool, s);
}

}  // namespace

struct df11_gpu_build {
  uint64_t n = 0;
  uint32_t C = 0, T = 0;
  int longest = 0;
  uint8_t len[256];
  uint32_t code[256];
  std::vector<uint32_t> luts;
  uint64_t total = 0, last_start = 0, num_blocks = 0, chunks = 0;
  uint64_t tiles = 0;
  bool vec = false;
  cudaStream_t stream = nullptr;  // the stream the scratch was allocated on
  // device scratch, phase 1: each tile's counts
  void *scratch1 = nullptr;
  uint16_t *d_tile_hist = nullptr;
  // device scratch, phase 2: per tile its bits, first bit and shared
  // words, per chunk first element and gap
  void *scratch2 = nullptr;
  uint32_t *d_tile_bits = nullptr;
  unsigned long long *d_tile_start = nullptr;
  uint32_t *d_edge = nullptr, *d_first = nullptr;
  uint8_t *d_gap = nullptr;
};

namespace {

void fill_params(const df11_gpu_build *h, df11_params *p) {
  std::memset(p, 0, sizeof(*p));
  p->n = h->n;
  p->total_bits = h->total;
  p->chunk_bytes = h->C;
  p->threads_per_block = h->T;
  p->num_blocks = (uint32_t)h->num_blocks;
  p->num_luts = (uint32_t)(h->luts.size() / 256);
  p->max_len = (uint32_t)h->longest;
}

// Small host<->device transfers go through one pinned buffer of the
// library's (grown on demand, kept for the process), so that they queue
// without synchronising the stream the way pageable copies do.  A build call
// holds it from its first copy to its last synchronisation.
struct Staging {
  std::mutex mu;
  void *p = nullptr;
  size_t bytes = 0;
  // caller holds mu
  void *get(size_t want) {
    if (want <= bytes) return p;
    if (p) cudaFreeHost(p);
    p = nullptr;
    bytes = 0;
    if (cudaHostAlloc(&p, want, cudaHostAllocDefault) != cudaSuccess) {
      p = nullptr;
      return nullptr;
    }
    bytes = want;
    return p;
  }
};
Staging g_staging;

df11_status check_begin_args(const uint16_t *d_bf16, uint64_t n, uint32_t C, uint32_t T) {
  if (n && !d_bf16) return DF11_ERR_NULL;
  if (C < 4 || C > 28 || C % 4) return DF11_ERR_INVALID;
  if (T < 128 || T > 1024 || T % 128) return DF11_ERR_INVALID;
  if (n >= (1ull << 32)) return DF11_ERR_TOO_LARGE;
  if ((uintptr_t)d_bf16 & 1) return DF11_ERR_ALIGN;
  return DF11_OK;
}

// phase 1's counts and last element of one tensor, one after another for
// the call's tensors (as in the host staging array)
constexpr uint64_t kHistWords = 257;

// A stream per device for phase 1's copies of the counts, so that they do
// not queue between the histogram kernels on the caller's stream (created
// once, non-blocking, kept for the process).
cudaStream_t side_stream() {
  static std::mutex mu;
  static cudaStream_t streams[kMaxDevices] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lock(mu);
  if (!streams[dev] && cudaStreamCreateWithFlags(&streams[dev], cudaStreamNonBlocking) != cudaSuccess)
    streams[dev] = nullptr;
  return streams[dev];
}

}  // namespace

extern "C" {

void df11_gpu_build_free(df11_gpu_build *h) {
  if (!h) return;
  // after the work queued on the handle's stream, which may read the scratch
  if (h->scratch1) cudaFreeAsync(h->scratch1, h->stream);
  if (h->scratch2) cudaFreeAsync(h->scratch2, h->stream);
  delete h;
}

df11_status df11_gpu_build_begin_batched(const uint16_t *const *d_bf16, const uint64_t *n,
                                         int count, uint32_t C, uint32_t T,
                                         df11_stream_t stream, df11_params *params,
                                         uint8_t *code_lengths, df11_gpu_build **handles) {
  if (count < 0) return DF11_ERR_INVALID;
  if (count == 0) return DF11_OK;
  if (!handles) return DF11_ERR_NULL;
  for (int i = 0; i < count; ++i) handles[i] = nullptr;
  if (!d_bf16 || !n || !params || !code_lengths) return DF11_ERR_NULL;
  for (int i = 0; i < count; ++i) {
    const df11_status st = check_begin_args(d_bf16[i], n[i], C, T);
    if (st != DF11_OK) return st;
  }
  for (int i = 0; i < count; ++i) {  // after every host-side check
    const void *p = n[i] ? d_bf16[i] : nullptr;
    const df11_status st = df11_internal::check_device_pointers(&p, 1);
    if (st != DF11_OK) return st;
  }
  cudaStream_t s = (cudaStream_t)stream;
  cudaStream_t side = side_stream();
  if (!side) return DF11_ERR_CUDA;
  std::vector<df11_gpu_build *> hs(count, nullptr);
  void *hblk = nullptr;  // the call's counts
  auto fail = [&](df11_status st) {
    // copies into the staging buffer may still be queued: let them land
    // before the buffer is released to another call
    cudaStreamSynchronize(s);
    cudaStreamSynchronize(side);
    if (hblk) cudaFreeAsync(hblk, s);
    for (auto *h : hs) df11_gpu_build_free(h);
    return st;
  };
  const uint64_t hist_slots = resident(hist_kernel);
  std::lock_guard<std::mutex> lock(g_staging.mu);
  auto *stage = static_cast<unsigned long long(*)[kHistWords]>(
      g_staging.get(sizeof(unsigned long long[kHistWords]) * count));
  if (!stage) return DF11_ERR_NOMEM;
  for (int i = 0; i < count; ++i) {
    df11_gpu_build *h = hs[i] = new (std::nothrow) df11_gpu_build();
    if (!h) return fail(DF11_ERR_NOMEM);
    h->n = n[i];
    h->C = C;
    h->T = T;
    h->vec = ((uintptr_t)d_bf16[i] & 15) == 0;
    h->stream = s;
    h->tiles = (h->n + kTile - 1) / kTile;
  }
  // The launches: the jobs in order, at most kHistJobs per launch, and the
  // shortest run of last jobs that holds a quarter of the tiles in a launch
  // of its own, so that the codebooks of the jobs before it are computed
  // while it runs.
  uint64_t all_tiles = 0;
  for (int i = 0; i < count; ++i) all_tiles += hs[i]->tiles;
  int tail = count - 1;
  uint64_t tail_tiles = hs[tail]->tiles;
  while (tail > 0 && count - tail < kHistJobs && 4 * tail_tiles < all_tiles)
    tail_tiles += hs[--tail]->tiles;
  std::vector<int> cut;  // launch k takes jobs cut[k] .. cut[k + 1] - 1
  for (int i = 0; i < tail; i += kHistJobs) cut.push_back(i);
  cut.push_back(tail);
  cut.push_back(count);
  const int launches = (int)cut.size() - 1;
  // per launch: its kernel is done (caller's stream), its counts are back
  // (side stream)
  struct Events {
    std::vector<cudaEvent_t> e;
    ~Events() {
      for (cudaEvent_t x : e)
        if (x) cudaEventDestroy(x);
    }
  } ev;
  ev.e.assign(2 * (size_t)launches, nullptr);
  for (auto &x : ev.e)
    if (cudaEventCreateWithFlags(&x, cudaEventDisableTiming) != cudaSuccess)
      return fail(DF11_ERR_CUDA);
  cudaEvent_t *done = ev.e.data(), *back = ev.e.data() + launches;
  const size_t hist_bytes = sizeof(unsigned long long) * kHistWords * count;
  if (scratch_alloc(&hblk, hist_bytes, s) != cudaSuccess) {
    hblk = nullptr;
    return fail(DF11_ERR_CUDA);
  }
  if (cudaMemsetAsync(hblk, 0, hist_bytes, s) != cudaSuccess) return fail(DF11_ERR_CUDA);
  unsigned long long *hist = static_cast<unsigned long long *>(hblk);
  for (int i = 0; i < count; ++i) {
    df11_gpu_build *h = hs[i];
    // the per-tile counts are written whole by the kernel
    if (scratch_alloc(&h->scratch1, round256(h->tiles * 512) + 256, s) != cudaSuccess)
      return fail(DF11_ERR_CUDA);
    h->d_tile_hist = static_cast<uint16_t *>(h->scratch1);
  }
  // histograms, and each tensor's last element (its codeword ends the stream)
  for (int k = 0; k < launches; ++k) {
    HistBatch hb;
    std::memset(&hb, 0, sizeof(hb));
    hb.count = cut[k + 1] - cut[k];
    for (int j = 0; j < hb.count; ++j) {
      const int i = cut[k] + j;
      HistJob &J = hb.job[j];
      J.w = d_bf16[i];
      J.n = hs[i]->n;
      J.tile_base = hb.tiles;
      J.hist = hist + kHistWords * i;
      J.last = hist + kHistWords * i + 256;
      J.tile_hist = hs[i]->d_tile_hist;
      J.vec = hs[i]->vec;
      hb.tiles += hs[i]->tiles;
    }
    if (hb.tiles) {
      const unsigned grid = (unsigned)(hb.tiles < hist_slots ? hb.tiles : hist_slots);
      hist_kernel<<<grid, kThreads, 0, s>>>(hb);
      if (cudaGetLastError() != cudaSuccess) return fail(DF11_ERR_CUDA);
    }
    if (cudaEventRecord(done[k], s) != cudaSuccess ||
        cudaStreamWaitEvent(side, done[k], 0) != cudaSuccess ||
        cudaMemcpyAsync(stage[cut[k]], hist + kHistWords * cut[k],
                        sizeof(stage[0]) * hb.count, cudaMemcpyDeviceToHost, side) !=
            cudaSuccess ||
        cudaEventRecord(back[k], side) != cudaSuccess)
      return fail(DF11_ERR_CUDA);
  }

  // codebooks (host: 256 symbols each), each as soon as its launch's
  // counts are back, while the device counts the later tensors; the
  // stream's length is the sum of count x code length
  for (int i = 0, k = 0; i < count; ++i) {
    df11_gpu_build *h = hs[i];
    if (i == cut[k]) {
      if (cudaEventSynchronize(back[k]) != cudaSuccess) return fail(DF11_ERR_CUDA);
      ++k;
    }
    uint64_t hist64[256];
    for (int k = 0; k < 256; ++k) hist64[k] = stage[i][k];
    h->longest = df11_internal::codebook(hist64, h->len, h->code, h->luts);
    uint64_t total = 0;
    for (int k = 0; k < 256; ++k) total += hist64[k] * h->len[k];
    h->total = total;
    if (h->n) h->last_start = h->total - h->len[(stage[i][256] >> 7) & 0xFF];
    const uint64_t block_bits = 8ull * C * T;
    h->num_blocks = (h->total + block_bits - 1) / block_bits;
    h->chunks = h->num_blocks * T;
    const uint64_t o_start = round256(h->tiles * 4);  // tile bits first
    const uint64_t o_edge = o_start + round256((h->tiles + 1) * 8);
    const uint64_t o_first = o_edge + round256(h->tiles * 8);
    const uint64_t o_gap = o_first + round256((h->chunks + 1) * sizeof(uint32_t));
    const uint64_t bytes2 = o_gap + round256(h->chunks + 1);
    if (scratch_alloc(&h->scratch2, bytes2, s) != cudaSuccess) return fail(DF11_ERR_CUDA);
    char *base2 = static_cast<char *>(h->scratch2);
    h->d_tile_bits = reinterpret_cast<uint32_t *>(base2);
    h->d_tile_start = reinterpret_cast<unsigned long long *>(base2 + o_start);
    h->d_edge = reinterpret_cast<uint32_t *>(base2 + o_edge);
    h->d_first = reinterpret_cast<uint32_t *>(base2 + o_first);
    h->d_gap = reinterpret_cast<uint8_t *>(base2 + o_gap);
    fill_params(h, &params[i]);
    std::memcpy(code_lengths + 256 * (size_t)i, h->len, 256);
  }
  cudaFreeAsync(hblk, s);  // every copy of it is done
  for (int i = 0; i < count; ++i) handles[i] = hs[i];
  return DF11_OK;
}

df11_status df11_gpu_build_begin(const uint16_t *d_bf16, uint64_t n, uint32_t C, uint32_t T,
                                 df11_stream_t stream, df11_params *params,
                                 uint8_t code_lengths[256], df11_gpu_build **handle) {
  if (handle) *handle = nullptr;
  if (!params || !code_lengths || !handle || (n && !d_bf16)) return DF11_ERR_NULL;
  return df11_gpu_build_begin_batched(&d_bf16, &n, 1, C, T, stream, params, code_lengths,
                                      handle);
}

df11_status df11_gpu_build_finish_batched(df11_gpu_build *const *handles, int count,
                                          const uint16_t *const *d_bf16,
                                          const df11_gpu_build_out *outs, df11_params *params,
                                          df11_stream_t stream) {
  if (count < 0) return DF11_ERR_INVALID;
  if (count == 0) return DF11_OK;
  if (!handles) return DF11_ERR_NULL;
  df11_status st = DF11_OK;
  cudaStream_t s = (cudaStream_t)stream;
  for (int i = 0; i < count && st == DF11_OK; ++i) {
    const df11_gpu_build *h = handles[i];
    if (!h || !d_bf16 || !outs || !params) {
      st = DF11_ERR_NULL;
      break;
    }
    const df11_gpu_build_out &o = outs[i];
    if (!o.bitstream || !o.gaps || !o.chunk_counts || !o.block_out_pos || !o.luts ||
        !o.code_lengths || !o.sign_mantissa || (h->n && !d_bf16[i])) {
      st = DF11_ERR_NULL;
    } else if (((uintptr_t)o.bitstream & 15) || ((uintptr_t)o.gaps & 15) ||
               ((uintptr_t)o.luts & 15) || ((uintptr_t)o.chunk_counts & 15) ||
               ((uintptr_t)o.sign_mantissa & 15) || ((uintptr_t)o.block_out_pos & 3) ||
               (h->n && h->vec != (((uintptr_t)d_bf16[i] & 15) == 0))) {
      st = DF11_ERR_ALIGN;
    }
  }
  for (int i = 0; i < count && st == DF11_OK; ++i) {  // after every host-side check
    const df11_gpu_build_out &o = outs[i];
    const void *ptrs[8] = {o.bitstream, o.gaps, o.chunk_counts, o.block_out_pos,
                           o.luts, o.code_lengths, o.sign_mantissa,
                           handles[i]->n ? (const void *)d_bf16[i] : nullptr};
    st = df11_internal::check_device_pointers(ptrs, 8);
  }
  // One staging area and one device block for the whole call: the job
  // descriptors, each job's tables (packed codes, codewords, luts, code
  // lengths), the tile counter and the maxima (zeros on the way in, the
  // results on the way out).
  std::unique_lock<std::mutex> lock(g_staging.mu, std::defer_lock);
  std::vector<size_t> tab_off(count > 0 ? count : 0);
  const size_t jobs_bytes = sizeof(Job) * (size_t)count;
  size_t bytes = (jobs_bytes + 255) & ~(size_t)255;
  for (int i = 0; i < count && st == DF11_OK; ++i) {
    tab_off[i] = bytes;
    bytes += (512 * 4 + handles[i]->luts.size() * 4 + 256 + 255) & ~(size_t)255;
  }
  const size_t ctl_off = bytes;  // counter, then 3 maxima per job
  bytes += 8 + 12 * (size_t)count;
  if (st == DF11_OK) lock.lock();
  uint8_t *stage = st == DF11_OK ? static_cast<uint8_t *>(g_staging.get(bytes)) : nullptr;
  if (st == DF11_OK && !stage) st = DF11_ERR_NOMEM;
  void *blk = nullptr;
  if (st == DF11_OK && scratch_alloc(&blk, bytes, s) != cudaSuccess) {
    blk = nullptr;
    st = DF11_ERR_CUDA;
  }
  uint8_t *dev = static_cast<uint8_t *>(blk);
  uint64_t all_tiles = 0, max_tiles = 0, max_fin = 0;
  if (st == DF11_OK) {
    Job *jobs = reinterpret_cast<Job *>(stage);
    std::memset(stage + ctl_off, 0, 8 + 12 * (size_t)count);
    for (int i = 0; i < count; ++i) {
      df11_gpu_build *h = handles[i];
      const df11_gpu_build_out &o = outs[i];
      const uint64_t chunks = h->chunks, n = h->n;
      const uint64_t bs_bytes = chunks * h->C + 16, gaps_bytes = chunks * 5 / 8 + 16;
      const uint64_t sm_bytes = (n + 15) / 16 * 16;
      const uint64_t bs_written = (h->total + 31) / 32 * 4;  // the stream's words
      const size_t lut_bytes = h->luts.size() * 4;
      uint32_t *st_tab = reinterpret_cast<uint32_t *>(stage + tab_off[i]);
      for (int e = 0; e < 256; ++e) {
        const uint32_t l = h->len[e];
        st_tab[e] = l <= (uint32_t)kPackedCodeBits ? (h->code[e] << 8) | l : kLongCode | l;
        st_tab[256 + e] = h->code[e];
      }
      std::memcpy(st_tab + 512, h->luts.data(), lut_bytes);
      std::memcpy(reinterpret_cast<uint8_t *>(st_tab + 512) + lut_bytes, h->len, 256);
      Job &J = jobs[i];
      std::memset(&J, 0, sizeof(J));
      J.w = d_bf16[i];
      J.n = n;
      J.vec = h->vec;
      J.longs = h->longest > kPackedCodeBits;
      J.tiles = h->tiles;
      J.tile_base = all_tiles;
      J.tile_hist = h->d_tile_hist;
      J.tile_bits = h->d_tile_bits;
      J.tile_start = h->d_tile_start;
      J.edge = h->d_edge;
      J.tab = reinterpret_cast<const uint32_t *>(dev + tab_off[i]);
      J.bs32 = reinterpret_cast<uint32_t *>(o.bitstream);
      J.sm = o.sign_mantissa;
      J.gaps_packed = o.gaps;
      J.counts = o.chunk_counts;
      J.code_lengths = o.code_lengths;
      J.bpos = o.block_out_pos;
      J.luts = o.luts;
      J.first_elem = h->d_first;
      J.gap = h->d_gap;
      J.maxima = reinterpret_cast<unsigned int *>(dev + ctl_off + 8) + 3 * i;
      J.chunks = chunks;
      J.total = h->total;
      J.last_start = h->last_start;
      J.num_blocks = (uint32_t)h->num_blocks;
      J.luts_vec4 = (uint32_t)(lut_bytes / 16);
      J.chunk_bits = 8 * h->C;
      J.block_bits = 8 * h->C * h->T;
      J.chunk_words = h->C / 4;
      J.block_words = h->C / 4 * h->T;
      J.chunk_magic = J.chunk_words > 1 ? UINT64_MAX / J.chunk_words + 1 : 0;
      J.block_magic = J.block_words > 1 ? UINT64_MAX / J.block_words + 1 : 0;
      // every byte no kernel writes otherwise: the padding after each buffer
      J.zero[0] = o.bitstream + bs_written;
      J.zero[1] = o.gaps + chunks * 5 / 8;
      J.zero[2] = o.chunk_counts + chunks;
      J.zero[3] = o.sign_mantissa + n;
      J.zero_bytes[0] = (uint32_t)(bs_bytes - bs_written);
      J.zero_bytes[1] = (uint32_t)(gaps_bytes - chunks * 5 / 8);
      J.zero_bytes[2] = 16u;
      J.zero_bytes[3] = (uint32_t)(sm_bytes - n);
      J.fin_threads = chunks / 8 + h->num_blocks + 1 + h->tiles;
      all_tiles += h->tiles;
      max_tiles = h->tiles > max_tiles ? h->tiles : max_tiles;
      max_fin = J.fin_threads > max_fin ? J.fin_threads : max_fin;
    }
    if (cudaMemcpyAsync(dev, stage, bytes, cudaMemcpyHostToDevice, s) != cudaSuccess)
      st = DF11_ERR_CUDA;
  }
  if (st == DF11_OK) {
    const Job *jobs = reinterpret_cast<const Job *>(dev);
    unsigned long long *counter = reinterpret_cast<unsigned long long *>(dev + ctl_off);
    unsigned fin_x;
    if (count > 65535 || !grid_for(max_fin, 256, &fin_x)) st = DF11_ERR_TOO_LARGE;
    if (st == DF11_OK && all_tiles) {
      // each tile's first bit, then the tiles packed
      tile_bits_kernel<<<dim3((unsigned)((max_tiles + 7) / 8), (unsigned)count), 256, 0, s>>>(
          jobs);
      scan_kernel<<<(unsigned)count, kScanThreads, 0, s>>>(jobs);
      const uint64_t slots = resident(pack_kernel);
      pack_kernel<<<(unsigned)(all_tiles < slots ? all_tiles : slots), kThreads, 0, s>>>(
          jobs, count, all_tiles, counter);
    }
    if (st == DF11_OK) {
      finish_kernel<<<dim3(fin_x, (unsigned)count), 256, 0, s>>>(jobs);
      if (cudaGetLastError() != cudaSuccess ||
          cudaMemcpyAsync(stage + ctl_off + 8, dev + ctl_off + 8, 12 * (size_t)count,
                          cudaMemcpyDeviceToHost, s) != cudaSuccess)
        st = DF11_ERR_CUDA;
    }
  }
  // the parameters' host-side fields, while the handles exist
  for (int i = 0; i < count && st == DF11_OK; ++i) fill_params(handles[i], &params[i]);
  // the scratch is freed in stream order after this call's work; the frees
  // are queued before the wait, so that their host time overlaps the kernels
  if (blk) cudaFreeAsync(blk, s);
  for (int i = 0; i < count; ++i) {
    if (!handles[i]) continue;
    handles[i]->stream = s;
    df11_gpu_build_free(handles[i]);
  }
  // the maxima come back (the staging buffer is read until then in any case)
  if (cudaStreamSynchronize(s) != cudaSuccess && st == DF11_OK) st = DF11_ERR_CUDA;
  for (int i = 0; i < count && st == DF11_OK; ++i) {
    unsigned int mx[3];
    std::memcpy(mx, stage + ctl_off + 8 + 12 * (size_t)i, sizeof(mx));
    params[i].max_block_elems = mx[0];
    params[i].max_chunk_elems = mx[1];
    params[i].max_warp_elems = mx[2];
  }
  if (lock.owns_lock()) lock.unlock();
  return st;
}

uint64_t df11_gpu_build_layout(const df11_params *params, int count, uint64_t *offsets,
                               uint64_t *sizes) {
  if (!params || count < 0) return 0;
  uint64_t total = 0;
  for (int i = 0; i < count; ++i) {
    const df11_params &p = params[i];
    const uint64_t chunks = (uint64_t)p.num_blocks * p.threads_per_block;
    const uint64_t sz[7] = {chunks * p.chunk_bytes + 16, chunks * 5 / 8 + 16, chunks + 16,
                            4ull * p.num_blocks + 4,     1024ull * p.num_luts, 256,
                            (p.n + 15) / 16 * 16};
    for (int j = 0; j < 7; ++j) {
      if (offsets) offsets[7 * (size_t)i + j] = total;
      if (sizes) sizes[7 * (size_t)i + j] = sz[j];
      total += round256(sz[j] > 16 ? sz[j] : 16);
    }
  }
  return total;
}

df11_status df11_gpu_build_finish(df11_gpu_build *h, const uint16_t *d_bf16, uint8_t *bitstream,
                                  uint8_t *gaps, uint8_t *chunk_counts, uint32_t *block_out_pos,
                                  uint32_t *luts, uint8_t *code_lengths, uint8_t *sign_mantissa,
                                  df11_params *params, df11_stream_t stream) {
  if (!h) return DF11_ERR_NULL;
  const df11_gpu_build_out o{bitstream, gaps, chunk_counts, block_out_pos, luts, code_lengths,
                             sign_mantissa};
  return df11_gpu_build_finish_batched(&h, 1, &d_bf16, &o, params, stream);
}

}  // extern "C"
// ---- exponent histogram with no allocation --------------------------------
// Some callers cannot allocate device memory: code running where the CUDA
// allocator must not be entered (inside an allocator hook, or a pool that is
// being resized), or a caller that has handed all device memory to its own
// allocator and has none to spare.  For them df11_exponent_histogram runs
// the builder's histogram kernel with its counters in this file-scope array
// instead of scratch the builder takes from its memory pool.  Its size is
// fixed: 256 64-bit counters (2 KB), held by every device that loads the
// library until the process exits.  All calls on a device share it and it
// keeps the last call's counts, so every call clears it first; two calls
// whose work overlaps on the GPU would race on it, which the library
// prevents within a process by taking one call at a time per device and
// waiting for each call's counts to come back before the next starts.
static __device__ __align__(256) unsigned long long g_exponent_hist[256];

namespace {
struct HistDevice {
  std::mutex mu;                       // one call at a time on this device's array
  unsigned long long *addr = nullptr;  // device address of g_exponent_hist (set-up)
};
HistDevice g_hist_device[kMaxDevices];
}  // namespace

extern "C" df11_status df11_exponent_histogram(const uint16_t *d_bf16, uint64_t n,
                                               uint64_t hist[256], df11_stream_t stream) {
  static_assert(sizeof(uint64_t) == sizeof(unsigned long long), "counter width");
  if (!hist || (n && !d_bf16)) return DF11_ERR_NULL;
  if (n >= (1ull << 32)) return DF11_ERR_TOO_LARGE;
  if ((uintptr_t)d_bf16 & 1) return DF11_ERR_ALIGN;
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return DF11_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return DF11_ERR_INVALID;
  if (n) {
    const void *p = d_bf16;
    const df11_status st = df11_internal::check_device_pointers(&p, 1);
    if (st != DF11_OK) return st;
  }
  HistDevice &hd = g_hist_device[dev];
  std::lock_guard<std::mutex> lock(hd.mu);
  if (!hd.addr) {
    // set-up, once per device, with that device current: in host code the
    // array's name stands for a host-side shadow, not a device address
    void *sym = nullptr;
    if (cudaGetSymbolAddress(&sym, g_exponent_hist) != cudaSuccess || !sym) return DF11_ERR_CUDA;
    hd.addr = static_cast<unsigned long long *>(sym);
  }
  cudaStream_t s = (cudaStream_t)stream;
  if (cudaMemsetAsync(hd.addr, 0, sizeof(g_exponent_hist), s) != cudaSuccess) return DF11_ERR_CUDA;
  if (n) {
    const uint64_t tiles = (n + kTile - 1) / kTile, slots = resident(hist_kernel);
    HistBatch hb;
    std::memset(&hb, 0, sizeof(hb));
    hb.count = 1;
    hb.tiles = tiles;
    hb.job[0].w = d_bf16;
    hb.job[0].n = n;
    hb.job[0].hist = hd.addr;  // no last element, no per-tile counts
    hb.job[0].vec = ((uintptr_t)d_bf16 & 15) == 0;
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3((unsigned)(tiles < slots ? tiles : slots));
    cfg.blockDim = dim3(kThreads);
    cfg.stream = s;
    // the launch's own status (not an earlier error of the calling thread)
    if (cudaLaunchKernelEx(&cfg, hist_kernel, hb) != cudaSuccess) return DF11_ERR_CUDA;
  }
  // straight into the caller's array (a DMA if the caller pinned it)
  if (cudaMemcpyAsync(hist, hd.addr, sizeof(g_exponent_hist), cudaMemcpyDeviceToHost, s) !=
          cudaSuccess ||
      cudaStreamSynchronize(s) != cudaSuccess)
    return DF11_ERR_CUDA;
  return DF11_OK;
}
