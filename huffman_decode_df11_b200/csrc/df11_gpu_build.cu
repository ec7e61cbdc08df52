// df11_gpu_build.cu -- the DF11 format builder on the GPU: compression of
// BF16 words already in device memory, byte for byte the output of the host
// builder (df11_build.cpp) on the same words.
//
// The pages compress offline on the host ("DFloat11无损压缩技术" (jsqmd.com)
// §2.2 items 1-2 give the recipe; "DFloat11重新定义LLM无损压缩的技术边界"
// (ocdem.com) §2.2 the lookup tables).  Here every step that touches the n
// elements runs on the device; only the codebook, a function of 256 counts,
// is computed on the host (df11_codebook.h, shared with the host builder).
// The elements are cut into pack blocks of 2048 (8 per thread of a
// 256-thread block); the kernels, in stream order:
//   histogram  exponent counts, one pass: counters in registers for a
//              window of 16 exponents around the mode of a first sample,
//              summed over the warp now and then; shared counters for the
//              rest;
//   sums       the code-length total of every pack block.  Each thread
//              block walks a contiguous range of pack blocks and keeps a
//              running total, so it writes every pack block's first bit
//              relative to its range, and the range's total;
//   scan       the ranges' first bits (one thread block; at most a few
//              thousand ranges) and the stream's total, which the host
//              reads to size the outputs;
//   prepare    chunk first elements preset to n, gaps and maxima cleared,
//              the bitstream words two pack blocks share cleared;
//   pack       persistent: per pack block, a block scan of the threads' bit
//              counts, every codeword ORed into a shared-memory image of the
//              block's words, the words written out coalesced (atomic OR
//              for the first and last word when a neighbour owns part of
//              it), the sign/mantissa bytes, and for every chunk and block
//              whose first codeword start is one of the thread's elements
//              the gap, first element and block position; the next pack
//              block's words are loaded while this one is packed;
//   finish     the chunks and blocks after the last codeword start, chunk
//              counts from first-element differences, the gaps packed
//              eight to five bytes, and the largest block, chunk and group
//              of 32 chunks.
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
constexpr int kPerCta = kThreads * kPerThread;  // elements per pack block

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

__device__ __forceinline__ uint32_t exponent_of(const uint4 &v, int k) {
  const uint32_t u = (k >> 1) == 0 ? v.x : (k >> 1) == 1 ? v.y : (k >> 1) == 2 ? v.z : v.w;
  return (u >> ((k & 1) ? 23 : 7)) & 0xFFu;
}

// how many of elements i0 .. i0+7 exist (0..8)
__device__ __forceinline__ uint32_t live_of(uint64_t i0, uint64_t n) {
  return i0 >= n ? 0u : (n - i0 >= (uint64_t)kPerThread ? (uint32_t)kPerThread : (uint32_t)(n - i0));
}

// ---- histogram -----------------------------------------------------------
// Per lane, 16 four-bit counters in one 64-bit register take the 8 elements
// of a tile whose exponent falls in the warp's window (mode - 11 .. mode + 4);
// after each tile they are spread into byte counters (four registers), and
// those are summed over the warp into shared counters every 31 tiles
// (at most 248 counts per byte).  Exponents outside the window go to the
// shared counters at once.
constexpr int kWindow = 16;
constexpr int kWindowBelow = 11;
constexpr int kFlushTiles = 31;

// byte j of counter register r holds window bin (r >> 1) * 8 + 2 j + (r & 1)
__device__ __forceinline__ void flush_window(uint32_t (&c)[4], int lo, uint32_t *h, int lane) {
#pragma unroll
  for (int r = 0; r < 4; ++r) {
    // two 16-bit sums per word: 32 lanes x 248 < 2^16
    const uint32_t even = __reduce_add_sync(0xFFFFFFFFu, c[r] & 0x00FF00FFu);
    const uint32_t odd = __reduce_add_sync(0xFFFFFFFFu, (c[r] >> 8) & 0x00FF00FFu);
    if (lane == 0) {
      const uint32_t v[4] = {even & 0xFFFFu, odd & 0xFFFFu, even >> 16, odd >> 16};
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int e = lo + (r >> 1) * 8 + 2 * j + (r & 1);
        if (v[j] && e >= 0 && e < 256) atomicAdd(&h[e], v[j]);
      }
    }
    c[r] = 0;
  }
}

__device__ __forceinline__ void count8(const uint4 &v, uint32_t live, int lo, uint32_t (&c)[4],
                                       uint32_t *h) {
  unsigned long long nib = 0;
#pragma unroll
  for (int k = 0; k < kPerThread; ++k) {
    if ((uint32_t)k < live) {
      const uint32_t e = exponent_of(v, k);
      const uint32_t d = (uint32_t)((int)e - lo);
      if (d < (uint32_t)kWindow) nib += 1ull << (4 * d);
      else atomicAdd(&h[e], 1u);
    }
  }
  const uint32_t n_lo = (uint32_t)nib, n_hi = (uint32_t)(nib >> 32);
  c[0] += n_lo & 0x0F0F0F0Fu;
  c[1] += (n_lo >> 4) & 0x0F0F0F0Fu;
  c[2] += n_hi & 0x0F0F0F0Fu;
  c[3] += (n_hi >> 4) & 0x0F0F0F0Fu;
}

__global__ void __launch_bounds__(kThreads) hist_kernel(const uint16_t *w, uint64_t n, bool vec,
                                                        unsigned long long *hist,
                                                        unsigned long long *last) {
  // the last element (its codeword ends the stream), for the builder
  if (last && blockIdx.x == 0 && threadIdx.x == 0 && n) *last = w[n - 1];
  __shared__ uint32_t h[kThreads / 32][256];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  for (int j = threadIdx.x; j < (kThreads / 32) * 256; j += kThreads) (&h[0][0])[j] = 0;
  const uint64_t stride = (uint64_t)gridDim.x * kPerCta;
  uint64_t base = (uint64_t)blockIdx.x * kPerCta;
  const uint64_t me = (uint64_t)threadIdx.x * kPerThread;
  uint4 next = load8(w, n, base + me, vec);
  // the window: around the most frequent exponent among the warp's lanes'
  // first elements
  int lo;
  {
    const uint32_t key = base + me < n ? exponent(next.x & 0xFFFFu) : 256u;
    const uint32_t peers = __match_any_sync(0xFFFFFFFFu, key);
    const uint32_t best = __reduce_max_sync(0xFFFFFFFFu, ((uint32_t)__popc(peers) << 16) | key);
    lo = (int)(best & 0x1FFu) - kWindowBelow;
  }
  __syncthreads();
  uint32_t c[4] = {0, 0, 0, 0};
  int tiles = 0;
  // `base` is the same for every thread of the block: whole warps iterate
  for (; base < n; base += stride) {
    const uint4 v = next;
    if (base + stride < n) next = load8(w, n, base + stride + me, vec);
    count8(v, live_of(base + me, n), lo, c, h[warp]);
    if (++tiles == kFlushTiles) {
      flush_window(c, lo, h[warp], lane);
      tiles = 0;
    }
  }
  flush_window(c, lo, h[warp], lane);
  __syncthreads();
  uint32_t s = 0;
  for (int j = 0; j < kThreads / 32; ++j) s += h[j][threadIdx.x];
  if (s) atomicAdd(&hist[threadIdx.x], (unsigned long long)s);
}

// ---- bit offsets ---------------------------------------------------------
// The pack kernel works in units of 256 elements (one warp, 8 per lane).  A
// sums thread block walks a contiguous range of units, 32 per iteration
// (four per warp), and keeps a running total, so it writes each unit's first
// bit relative to its range, and the range's total.
constexpr int kUnit = 32 * kPerThread;        // elements per unit
constexpr int kUnitWords = kUnit + 1;         // words a unit's codewords can touch
constexpr int kUnitsPerWarp = 4;              // per iteration of the sums kernel
constexpr int kUnitsPerIter = (kThreads / 32) * kUnitsPerWarp;
static_assert(kUnitsPerIter == 32, "one warp scans an iteration's units");

struct Ranges {
  uint64_t units;  // units of the tensor
  uint64_t per;    // units per range (one range per sums thread block)
  uint32_t *local; // first bit of each unit within its range
  unsigned long long *range_start;  // first bit of each range; the total after the last
};

// units and ranges number below 2^24: 32-bit division
__device__ __forceinline__ unsigned long long unit_start(const Ranges &r, uint64_t u) {
  return r.range_start[(uint32_t)u / (uint32_t)r.per] + r.local[u];
}

__global__ void __launch_bounds__(kThreads, 4) sums_kernel(const uint16_t *w, uint64_t n, bool vec,
                                                           const uint2 *tab, const Ranges r,
                                                           unsigned long long *range_total) {
  __shared__ uint8_t len[256];
  __shared__ uint32_t part[kUnitsPerIter];
  len[threadIdx.x] = (uint8_t)tab[threadIdx.x].y;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const uint64_t u_begin = (uint64_t)blockIdx.x * r.per;
  const uint64_t u_end = u_begin + r.per < r.units ? u_begin + r.per : r.units;
  const uint64_t me = (uint64_t)lane * kPerThread;
  uint4 next[kUnitsPerWarp];
#pragma unroll
  for (int j = 0; j < kUnitsPerWarp; ++j) {
    const uint64_t u = u_begin + warp * kUnitsPerWarp + j;
    next[j] = u < u_end ? load8(w, n, u * kUnit + me, vec) : make_uint4(0, 0, 0, 0);
  }
  __syncthreads();
  unsigned long long running = 0;  // warp 0: bits of the range so far (uniform)
  for (uint64_t u0 = u_begin; u0 < u_end; u0 += kUnitsPerIter) {
    uint4 v[kUnitsPerWarp];
#pragma unroll
    for (int j = 0; j < kUnitsPerWarp; ++j) {
      v[j] = next[j];
      const uint64_t u = u0 + kUnitsPerIter + warp * kUnitsPerWarp + j;
      if (u < u_end) next[j] = load8(w, n, u * kUnit + me, vec);
    }
#pragma unroll
    for (int j = 0; j < kUnitsPerWarp; ++j) {
      const uint64_t u = u0 + warp * kUnitsPerWarp + j;
      const uint32_t live = u < u_end ? live_of(u * kUnit + me, n) : 0u;
      uint32_t s = 0;
#pragma unroll
      for (int k = 0; k < kPerThread; ++k)
        if ((uint32_t)k < live) s += len[exponent_of(v[j], k)];
      s = __reduce_add_sync(0xFFFFFFFFu, s);
      if (lane == 0) part[warp * kUnitsPerWarp + j] = s;
    }
    __syncthreads();
    if (warp == 0) {  // the iteration's 32 units in order, one per lane
      const uint32_t mine = part[lane];
      uint32_t incl = mine;
#pragma unroll
      for (int d = 1; d < 32; d <<= 1) {
        const uint32_t t = __shfl_up_sync(0xFFFFFFFFu, incl, d);
        if (lane >= d) incl += t;
      }
      const uint64_t u = u0 + lane;
      if (u < u_end) r.local[u] = (uint32_t)(running + incl - mine);
      running += __shfl_sync(0xFFFFFFFFu, incl, 31);
    }
    __syncthreads();  // part is rewritten next iteration
  }
  if (threadIdx.x == 0) range_total[blockIdx.x] = running;
}

// Exclusive scan of the range totals into the ranges' first bits, the total
// at starts[count]; one thread block, each thread a contiguous run.
constexpr int kScanThreads = 1024;

__global__ void __launch_bounds__(kScanThreads) scan_kernel(const unsigned long long *totals,
                                                            uint64_t count,
                                                            unsigned long long *starts) {
  __shared__ unsigned long long warp_tot[kScanThreads / 32];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const uint64_t per = (count + kScanThreads - 1) / kScanThreads;
  const uint64_t b = threadIdx.x * per;
  const uint64_t e = b + per < count ? b + per : count;
  unsigned long long mine = 0;
  for (uint64_t i = b; i < e; ++i) mine += totals[i];
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
    starts[i] = run;
    run += totals[i];
  }
  if (threadIdx.x == kScanThreads - 1) starts[count] = run;
}

// Before packing: first elements preset to n, gaps cleared, the bitstream
// words that two units share cleared (they are ORed into), maxima cleared;
// also the output paddings no kernel writes cleared, and the tables copied
// from the device staging area into the caller's buffers.
struct PrepareArgs {
  uint32_t *first_elem;
  uint8_t *gap;
  uint64_t chunks;
  uint32_t n;
  Ranges r;
  uint32_t *bs32;
  unsigned int *maxima;
  uint8_t *zero[4];        // byte ranges to clear
  uint32_t zero_bytes[4];
  const uint4 *luts_src;   // num_luts * 1 KB
  uint4 *luts_dst;         // 16-byte aligned
  uint32_t luts_vec4;      // 16-byte words of the tables
  const uint8_t *lens_src;
  uint8_t *lens_dst;       // 256 bytes, any alignment
};

__global__ void prepare_kernel(const PrepareArgs a) {
  uint64_t all = a.chunks + 1 > a.r.units ? a.chunks + 1 : a.r.units;
  all = all > a.luts_vec4 ? all : a.luts_vec4;
  all = all > 256 ? all : 256;  // the code lengths, the paddings, the maxima
  for (uint64_t i = blockIdx.x * 256ull + threadIdx.x; i < all; i += (uint64_t)gridDim.x * 256) {
    if (i <= a.chunks) {
      a.first_elem[i] = a.n;
      a.gap[i] = 0;
    }
    if (i >= 1 && i < a.r.units) {
      const unsigned long long st = unit_start(a.r, i);
      if (st & 31u) a.bs32[st >> 5] = 0;
    }
    if (i < 3) a.maxima[i] = 0;
    if (i < a.luts_vec4) a.luts_dst[i] = a.luts_src[i];
    if (i < 256) a.lens_dst[i] = a.lens_src[i];
  }
  // paddings: each at most a block of the bitstream plus 16 bytes
  for (int k = 0; k < 4; ++k)
    for (uint32_t i = blockIdx.x * 256u + threadIdx.x; i < a.zero_bytes[k]; i += gridDim.x * 256u)
      a.zero[k][i] = 0;
}

// ---- pack ----------------------------------------------------------------
struct PackArgs {
  const uint16_t *w;
  uint64_t n;
  bool vec;             // w is 16-byte aligned
  const uint2 *tab;     // {codeword, length} per exponent
  Ranges r;
  uint32_t *bs32;       // bitstream as 32-bit words
  uint8_t *sm;          // 16-byte aligned
  uint8_t *gap;         // one byte per chunk
  uint32_t *first_elem; // chunks + 1, preset to n
  uint32_t *bpos;
  uint64_t chunks;
  uint32_t num_blocks;
  uint32_t chunk_bits, block_bits;  // 8 C and 8 C T
  uint32_t chunk_words, block_words;  // chunk_bits / 32, block_bits / 32
  uint64_t chunk_magic, block_magic;  // ceil(2^64 / words) (words >= 2)
  uint32_t chunk_m32;                 // ceil(2^32 / chunk_bits): floor(x / chunk_bits)
                                      // = umulhi(x, chunk_m32) for x < 2^16
};

// floor(x / d) for x < 2^32 by a multiply-high with ceil(2^64 / d): the
// error, below x / 2^64 < 2^-32, never crosses an integer (d < 2^32)
__device__ __forceinline__ uint64_t div_words(uint32_t x, uint32_t d, uint64_t magic) {
  return d == 1 ? x : __umul64hi((uint64_t)x, magic);
}

__global__ void __launch_bounds__(kThreads) pack_kernel(const PackArgs a) {
  __shared__ uint2 tab_s[256];
  __shared__ uint32_t words_s[kThreads / 32][kUnitWords];
  tab_s[threadIdx.x] = a.tab[threadIdx.x];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint32_t *words = words_s[warp];
  for (int j = lane; j < kUnitWords; j += 32) words[j] = 0;
  const uint64_t me = (uint64_t)lane * kPerThread;
  const uint64_t units = a.r.units;
  const uint64_t stride = (uint64_t)gridDim.x * (kThreads / 32);
  uint64_t u = (uint64_t)blockIdx.x * (kThreads / 32) + warp;
  // unit u's words, first bit and previous element (lane 0)
  uint4 nx = make_uint4(0, 0, 0, 0);
  unsigned long long nstart = 0;
  uint32_t nprev = 0;
  if (u < units) {
    nx = load8(a.w, a.n, u * kUnit + me, a.vec);
    nstart = unit_start(a.r, u);
    if (lane == 0 && u) nprev = a.w[u * kUnit - 1];
  }
  __syncthreads();  // the table
  for (; u < units; u += stride) {
    const uint4 v = nx;
    const unsigned long long start = nstart;
    const uint32_t prev_word = nprev;
    const uint64_t un = u + stride;
    if (un < units) {
      nx = load8(a.w, a.n, un * kUnit + me, a.vec);
      nstart = unit_start(a.r, un);
      if (lane == 0) nprev = a.w[un * kUnit - 1];
    }
    const uint64_t i0 = u * kUnit + me;
    const uint32_t live = live_of(i0, a.n);
    uint32_t e[kPerThread], l[kPerThread], cw[kPerThread];
    uint32_t mine = 0, last = 0;
#pragma unroll
    for (int k = 0; k < kPerThread; ++k) {
      e[k] = exponent_of(v, k);
      const uint2 t = tab_s[e[k]];
      const bool in = (uint32_t)k < live;
      l[k] = in ? t.y : 0u;
      cw[k] = in ? t.x : 0u;
      mine += l[k];
      last = in ? l[k] : last;
    }
    uint32_t incl = mine;
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
      const uint32_t t = __shfl_up_sync(0xFFFFFFFFu, incl, d);
      if (lane >= d) incl += t;
    }
    const uint32_t total = __shfl_sync(0xFFFFFFFFu, incl, 31);
    // length of element i0 - 1's codeword: the previous lane's last, or
    // for lane 0 the previous unit's last element (0 for element 0)
    const uint32_t up = __shfl_up_sync(0xFFFFFFFFu, last, 1);
    const uint32_t prev_len = lane ? up : (u ? tab_s[exponent(prev_word)].y : 0u);
    // positions below are relative to `origin`, the first bit of the word
    // this unit begins in
    const unsigned long long origin = start & ~31ull;
    const uint32_t lead = (uint32_t)(start & 31u);
    const uint32_t rel = lead + incl - mine;  // this lane's first bit

    // codewords, MSB first, ORed into the warp's image of the unit's words:
    // up to 32 bits (the usual case) gathered in one register and placed
    // with one or two ORs, up to 64 in two registers, longer runs word by word
    __syncwarp();  // the previous unit's words are written out and cleared
    if (mine && mine <= 32) {
      uint32_t acc = 0;
#pragma unroll
      for (int k = 0; k < kPerThread; ++k) acc = (acc << l[k]) | cw[k];
      const uint32_t o = rel & 31u, wk = rel >> 5;
      const uint32_t left = acc << (32 - mine);  // first bit at bit 31
      atomicOr(&words[wk], left >> o);
      if (o + mine > 32) atomicOr(&words[wk + 1], left << (32 - o));
    } else if (mine) {
      if (mine <= 64) {
        unsigned long long acc = 0;
#pragma unroll
        for (int k = 0; k < kPerThread; ++k) acc = (acc << l[k]) | cw[k];
        const uint32_t o = rel & 31u, wk = rel >> 5;
        const unsigned long long left = acc << (64 - mine);
        const uint32_t hi = (uint32_t)(left >> 32), lo = (uint32_t)left;
        atomicOr(&words[wk], hi >> o);
        atomicOr(&words[wk + 1], __funnelshift_r(lo, hi, o));
        if (o + mine > 64) atomicOr(&words[wk + 2], __funnelshift_lc(0u, lo, 32 - o));
      } else {
        // `cur` holds the pending bits left-aligned, `nb` of them
        uint32_t wk = rel >> 5, nb = rel & 31u, cur = 0;
        bool first = true;
#pragma unroll
        for (int k = 0; k < kPerThread; ++k) {
          if (l[k]) {
            const uint32_t tot = nb + l[k];
            if (tot >= 32) {
              const uint32_t t = cur | (cw[k] >> (tot - 32));
              if (first) atomicOr(&words[wk], t);  // the previous lane may own its first bits
              else words[wk] = t;
              first = false;
              ++wk;
              nb = tot - 32;
              cur = __funnelshift_lc(0u, cw[k], 32 - nb);  // 0 when nb == 0
            } else {
              cur |= cw[k] << (32 - tot);
              nb = tot;
            }
          }
        }
        if (nb) atomicOr(&words[wk], cur);  // the last, partial word, which the next lane may share
      }
    }
    __syncwarp();
    // words out, and cleared for the next unit: ORed where a neighbouring
    // unit owns part of the word (cleared beforehand), stored otherwise
    const uint64_t base = origin >> 5;
    const uint32_t end_bits = lead + total;
    const uint32_t nwords = (end_bits + 31) >> 5;
    const bool shared_last = (end_bits & 31u) && u + 1 < units;
    for (uint32_t j = lane; j < nwords; j += 32) {
      const uint32_t t = bswap32(words[j]);
      words[j] = 0;
      if ((j == 0 && lead) || (j == nwords - 1 && shared_last)) atomicOr(&a.bs32[base + j], t);
      else a.bs32[base + j] = t;
    }
    // chunks and blocks whose first codeword start is one of these
    // elements: those that begin after element i0 - 1's codeword start and
    // at or before element i0 + live - 1's.  The first chunk (block) after
    // that start is floor(start / chunk bits) + 1; bit offsets stay below
    // 2^37, so offset / 32 fits 32 bits and floor(p / (32 m)) =
    // floor(floor(p / 32) / m).  Blocks are skipped unless one begins
    // inside this unit (warp-wide test, before any lane leaves).
    const int p_last = (int)(rel + mine - last);
    const uint32_t pw = (uint32_t)((origin + rel - prev_len) >> 5);  // element i0 - 1's start / 32
    // chunk c_base begins o_c bits before `origin` (0 <= o_c < chunk bits)
    const uint64_t c_base = div_words((uint32_t)(origin >> 5), a.chunk_words, a.chunk_magic);
    const int o_c = (int)(origin - c_base * a.chunk_bits);
    const uint32_t pw0 = __shfl_sync(0xFFFFFFFFu, pw, 0);
    const int p_end = __shfl_sync(0xFFFFFFFFu, p_last, 31);
    const uint64_t q0 = u ? div_words(pw0, a.block_words, a.block_magic) + 1 : 0;
    const bool blocks_here = (long long)(q0 * a.block_bits) - (long long)origin <= p_end;
    if (!live) continue;

    // sign/mantissa bytes: bit 15 -> bit 7, bits 0-6 kept; two per word
    uint32_t sm2[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const uint32_t t = q == 0 ? v.x : q == 1 ? v.y : q == 2 ? v.z : v.w;
      sm2[q] = (t & 0x007F007Fu) | ((t >> 8) & 0x00800080u);  // bytes 0 and 2
    }
    const uint2 smv = make_uint2(__byte_perm(sm2[0], sm2[1], 0x6420),
                                 __byte_perm(sm2[2], sm2[3], 0x6420));
    if (live == kPerThread) {
      *reinterpret_cast<uint2 *>(a.sm + i0) = smv;
    } else {
      for (uint32_t k = 0; k < live; ++k)
        a.sm[i0 + k] = (uint8_t)((k < 4 ? smv.x : smv.y) >> (8 * (k & 3)));
    }

    // the first chunk boundary after element i0 - 1's start; then, while
    // it lies at or before this lane's last start, the first element
    // starting at or after it (counted without branches) takes it
    const uint32_t x = (uint32_t)((int)rel - (int)prev_len + o_c + (int)a.chunk_bits);
    const uint32_t jc = i0 ? __umulhi(x, a.chunk_m32) : 0u;  // floor(x / chunk_bits)
    int cb = (int)(jc * a.chunk_bits) - o_c;
    if (cb <= p_last) {
      uint64_t c = c_base + jc;
      do {
        uint32_t k = 0, bits = 0;
        int pj = (int)rel;
#pragma unroll
        for (int j = 0; j < kPerThread; ++j) {
          const bool before = l[j] && pj < cb;
          k += before ? 1u : 0u;
          bits += before ? l[j] : 0u;
          pj += (int)l[j];
        }
        if (c < a.chunks) {
          a.gap[c] = (uint8_t)((int)(rel + bits) - cb);
          a.first_elem[c] = (uint32_t)(i0 + k);
        }
        ++c;
        cb += (int)a.chunk_bits;
      } while (cb <= p_last);
    }
    if (blocks_here) {  // the same for block boundaries (about one unit in 25)
      uint64_t q = i0 ? div_words(pw, a.block_words, a.block_magic) + 1 : 0;
      int qb = (int)((long long)(q * a.block_bits) - (long long)origin);
      int pk = (int)rel;
#pragma unroll
      for (int k = 0; k < kPerThread; ++k) {
        if (l[k]) {
          for (; qb <= pk; qb += (int)a.block_bits, ++q)
            if (q < a.num_blocks) a.bpos[q] = (uint32_t)(i0 + k);
          pk += (int)l[k];
        }
      }
    }
  }
}

// ---- finish --------------------------------------------------------------
struct FinishArgs {
  const uint8_t *gap;
  const uint32_t *first_elem;
  uint8_t *gaps_packed;
  uint8_t *counts;
  uint32_t *bpos;
  unsigned int *maxima;  // block, chunk, group of 32 chunks
  uint64_t chunk_bits, chunks, block_bits, total, last_start;
  uint32_t num_blocks, n;
};

// one thread per group of 8 chunks (5 packed gap bytes); chunks is a
// multiple of 128
__global__ void finish_chunks(const FinishArgs a) {
  const uint64_t g = blockIdx.x * 256ull + threadIdx.x;
  const uint64_t c0 = g * 8;
  if (c0 >= a.chunks) return;
  unsigned long long v = 0;
  uint32_t mc = 0;
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const uint64_t c = c0 + j, cb = c * a.chunk_bits;
    uint32_t gv = a.gap[c];
    // a chunk that begins inside the last codeword: the distance to the end
    if (a.n && cb > a.last_start && cb < a.total) gv = (uint32_t)(a.total - cb);
    const uint32_t k = a.first_elem[c + 1] - a.first_elem[c];
    a.counts[c] = (uint8_t)k;
    mc = mc > k ? mc : k;
    v = (v << 5) | gv;
  }
#pragma unroll
  for (int j = 0; j < 5; ++j) a.gaps_packed[g * 5 + j] = (uint8_t)(v >> (32 - 8 * j));
  atomicMax(&a.maxima[1], mc);
  if (c0 % 32 == 0) {
    const uint64_t e = c0 + 32 < a.chunks ? c0 + 32 : a.chunks;
    atomicMax(&a.maxima[2], a.first_elem[e] - a.first_elem[c0]);
  }
}

// entry b of block_out_pos as the format stores it: n for the blocks after
// the last codeword start and for the end entry
__device__ __forceinline__ uint32_t block_pos(const FinishArgs &a, uint64_t b) {
  if (b >= a.num_blocks || (a.n && b * a.block_bits > a.last_start)) return a.n;
  return a.bpos[b];
}

// one thread per entry of block_out_pos.  Rewriting an entry with its
// block_pos leaves its block_pos unchanged, so a neighbour may read it
// before or after the rewrite.
__global__ void finish_blocks(const FinishArgs a) {
  const uint64_t b = blockIdx.x * 256ull + threadIdx.x;
  if (b > a.num_blocks) return;
  const uint32_t here = block_pos(a, b);
  if (b < a.num_blocks) atomicMax(&a.maxima[0], block_pos(a, b + 1) - here);
  a.bpos[b] = here;
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
  bool vec = false;
  Ranges r{};
  uint64_t ranges = 0;
  // device scratch, phase 1: histogram, {codeword, length} per exponent,
  // range totals and first bits, pack-block first bits within their range
  cudaStream_t stream = nullptr;  // the stream the scratch was allocated on
  void *scratch1 = nullptr;
  unsigned long long *d_hist = nullptr, *d_range_total = nullptr;
  uint2 *d_tab = nullptr;
  // device scratch, phase 2: per-chunk first element and gap, the maxima
  void *scratch2 = nullptr;
  uint32_t *d_first = nullptr;
  unsigned int *d_max = nullptr;
  uint8_t *d_gap = nullptr;
  uint8_t *d_tables = nullptr;  // the luts, then the code lengths, for the prepare kernel
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

// what one tensor's phase 1 reads back and sends
struct BeginSlot {
  unsigned long long hist[257];  // the counts, then the last element
  uint2 tab[256];
  unsigned long long total;
};

df11_status check_begin_args(const uint16_t *d_bf16, uint64_t n, uint32_t C, uint32_t T) {
  if (n && !d_bf16) return DF11_ERR_NULL;
  if (C < 4 || C > 28 || C % 4) return DF11_ERR_INVALID;
  if (T < 128 || T > 1024 || T % 128) return DF11_ERR_INVALID;
  if (n >= (1ull << 32)) return DF11_ERR_TOO_LARGE;
  if ((uintptr_t)d_bf16 & 1) return DF11_ERR_ALIGN;
  return DF11_OK;
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
  std::vector<df11_gpu_build *> hs(count, nullptr);
  auto fail = [&](df11_status st) {
    // copies into the staging buffer may still be queued: let them land
    // before the buffer is released to another call
    cudaStreamSynchronize(s);
    for (auto *h : hs) df11_gpu_build_free(h);
    return st;
  };
  const uint64_t slots = resident(sums_kernel), hist_slots = resident(hist_kernel);
  std::lock_guard<std::mutex> lock(g_staging.mu);
  BeginSlot *stage = static_cast<BeginSlot *>(g_staging.get(sizeof(BeginSlot) * count));
  if (!stage) return DF11_ERR_NOMEM;
  // one event per tensor: its counts are back
  struct Events {
    std::vector<cudaEvent_t> e;
    ~Events() {
      for (cudaEvent_t x : e)
        if (x) cudaEventDestroy(x);
    }
  } ev;
  ev.e.assign(count, nullptr);
  for (int i = 0; i < count; ++i)
    if (cudaEventCreateWithFlags(&ev.e[i], cudaEventDisableTiming) != cudaSuccess)
      return DF11_ERR_CUDA;
  const std::vector<cudaEvent_t> &events = ev.e;

  // histograms, and each tensor's last element (its codeword ends the stream)
  for (int i = 0; i < count; ++i) {
    df11_gpu_build *h = hs[i] = new (std::nothrow) df11_gpu_build();
    if (!h) return fail(DF11_ERR_NOMEM);
    h->n = n[i];
    h->C = C;
    h->T = T;
    h->vec = ((uintptr_t)d_bf16[i] & 15) == 0;
    h->stream = s;
    // contiguous ranges of units, one per resident sums thread block.  A
    // range's bits fit 32 bits: at most 2^24 units over at least
    // min(units, SMs) ranges, at most 8192 bits per unit.
    h->r.units = (h->n + kUnit - 1) / kUnit;
    h->ranges = h->r.units < slots ? h->r.units : slots;
    h->r.per = h->ranges ? (h->r.units + h->ranges - 1) / h->ranges : 1;
    if (h->ranges) h->ranges = (h->r.units + h->r.per - 1) / h->r.per;
    const uint64_t o_tab = round256(257 * sizeof(unsigned long long));
    const uint64_t o_tot = o_tab + round256(256 * sizeof(uint2));
    const uint64_t o_rs = o_tot + round256(h->ranges * sizeof(unsigned long long) + 8);
    const uint64_t o_loc = o_rs + round256((h->ranges + 1) * sizeof(unsigned long long));
    const uint64_t bytes1 = o_loc + round256(h->r.units * sizeof(uint32_t) + 4);
    if (scratch_alloc(&h->scratch1, bytes1, s) != cudaSuccess) return fail(DF11_ERR_CUDA);
    char *base1 = static_cast<char *>(h->scratch1);
    h->d_hist = reinterpret_cast<unsigned long long *>(base1);
    h->d_tab = reinterpret_cast<uint2 *>(base1 + o_tab);
    h->d_range_total = reinterpret_cast<unsigned long long *>(base1 + o_tot);
    h->r.range_start = reinterpret_cast<unsigned long long *>(base1 + o_rs);
    h->r.local = reinterpret_cast<uint32_t *>(base1 + o_loc);
    if (cudaMemsetAsync(h->d_hist, 0, 257 * sizeof(unsigned long long), s) != cudaSuccess)
      return fail(DF11_ERR_CUDA);
    if (h->n) {
      const uint64_t tiles = (h->n + kPerCta - 1) / kPerCta;
      const unsigned grid = (unsigned)(tiles < hist_slots ? tiles : hist_slots);
      hist_kernel<<<grid, kThreads, 0, s>>>(d_bf16[i], h->n, h->vec, h->d_hist, h->d_hist + 256);
      if (cudaGetLastError() != cudaSuccess) return fail(DF11_ERR_CUDA);
    }
    if (cudaMemcpyAsync(stage[i].hist, h->d_hist, sizeof(stage[i].hist), cudaMemcpyDeviceToHost,
                        s) != cudaSuccess ||
        cudaEventRecord(events[i], s) != cudaSuccess)
      return fail(DF11_ERR_CUDA);
  }

  // codebooks (host: 256 symbols each), each as soon as its counts are
  // back, while the device computes the previous tensors' bit offsets; then
  // every unit's first bit and the totals
  for (int i = 0; i < count; ++i) {
    df11_gpu_build *h = hs[i];
    if (cudaEventSynchronize(events[i]) != cudaSuccess) return fail(DF11_ERR_CUDA);
    uint64_t hist64[256];
    for (int k = 0; k < 256; ++k) hist64[k] = stage[i].hist[k];
    h->longest = df11_internal::codebook(hist64, h->len, h->code, h->luts);
    for (int k = 0; k < 256; ++k) stage[i].tab[k] = make_uint2(h->code[k], h->len[k]);
    stage[i].total = 0;
    if (cudaMemcpyAsync(h->d_tab, stage[i].tab, sizeof(stage[i].tab), cudaMemcpyHostToDevice,
                        s) != cudaSuccess)
      return fail(DF11_ERR_CUDA);
    if (h->ranges) {
      sums_kernel<<<(unsigned)h->ranges, kThreads, 0, s>>>(d_bf16[i], h->n, h->vec, h->d_tab,
                                                           h->r, h->d_range_total);
      scan_kernel<<<1, kScanThreads, 0, s>>>(h->d_range_total, h->ranges, h->r.range_start);
      if (cudaGetLastError() != cudaSuccess ||
          cudaMemcpyAsync(&stage[i].total, h->r.range_start + h->ranges,
                          sizeof(stage[i].total), cudaMemcpyDeviceToHost, s) != cudaSuccess)
        return fail(DF11_ERR_CUDA);
    }
  }
  if (cudaStreamSynchronize(s) != cudaSuccess) return fail(DF11_ERR_CUDA);

  for (int i = 0; i < count; ++i) {
    df11_gpu_build *h = hs[i];
    h->total = stage[i].total;
    if (h->n) h->last_start = h->total - h->len[(stage[i].hist[256] >> 7) & 0xFF];
    const uint64_t block_bits = 8ull * C * T;
    h->num_blocks = (h->total + block_bits - 1) / block_bits;
    h->chunks = h->num_blocks * T;
    const uint64_t o_max = round256((h->chunks + 1) * sizeof(uint32_t));
    const uint64_t o_gap = o_max + 256;
    const uint64_t o_tables = o_gap + round256(h->chunks + 1);
    const uint64_t table_bytes = h->luts.size() * 4 + 256;
    if (scratch_alloc(&h->scratch2, o_tables + round256(table_bytes), s) != cudaSuccess)
      return fail(DF11_ERR_CUDA);
    char *base2 = static_cast<char *>(h->scratch2);
    h->d_first = reinterpret_cast<uint32_t *>(base2);
    h->d_max = reinterpret_cast<unsigned int *>(base2 + o_max);
    h->d_gap = reinterpret_cast<uint8_t *>(base2 + o_gap);
    h->d_tables = reinterpret_cast<uint8_t *>(base2 + o_tables);
    fill_params(h, &params[i]);
    std::memcpy(code_lengths + 256 * (size_t)i, h->len, 256);
  }
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
  std::unique_lock<std::mutex> lock(g_staging.mu, std::defer_lock);
  size_t stage_bytes = 0;
  std::vector<size_t> off(count > 0 ? count : 0);
  if (st == DF11_OK) {
    for (int i = 0; i < count; ++i) {
      off[i] = stage_bytes;  // luts, code lengths, then the maxima read back
      stage_bytes += (handles[i]->luts.size() * 4 + 256 + 16 + 15) & ~(size_t)15;
    }
    lock.lock();
  }
  uint8_t *stage = st == DF11_OK ? static_cast<uint8_t *>(g_staging.get(stage_bytes)) : nullptr;
  if (st == DF11_OK && !stage) st = DF11_ERR_NOMEM;
  for (int i = 0; i < count && st == DF11_OK; ++i) {
    df11_gpu_build *h = handles[i];
    const df11_gpu_build_out &o = outs[i];
    const uint64_t chunks = h->chunks, n = h->n;
    const uint64_t bs_bytes = chunks * h->C + 16, gaps_bytes = chunks * 5 / 8 + 16;
    const uint64_t sm_bytes = (n + 15) / 16 * 16;
    const uint64_t bs_written = (h->total + 31) / 32 * 4;  // the units' words
    const size_t lut_bytes = h->luts.size() * 4;
    uint8_t *st_luts = stage + off[i], *st_lens = st_luts + lut_bytes;
    std::memcpy(st_luts, h->luts.data(), lut_bytes);
    std::memcpy(st_lens, h->len, 256);
    if (cudaMemcpyAsync(h->d_tables, st_luts, lut_bytes + 256, cudaMemcpyHostToDevice, s) !=
        cudaSuccess) {
      st = DF11_ERR_CUDA;
      break;
    }
    uint32_t *bs32 = reinterpret_cast<uint32_t *>(o.bitstream);
    // every byte the kernels do not write: the padding after each buffer
    PrepareArgs pr{h->d_first, h->d_gap, chunks, (uint32_t)n, h->r, bs32, h->d_max,
                   {o.bitstream + bs_written, o.gaps + chunks * 5 / 8, o.chunk_counts + chunks,
                    o.sign_mantissa + n},
                   {(uint32_t)(bs_bytes - bs_written), (uint32_t)(gaps_bytes - chunks * 5 / 8), 16u,
                    (uint32_t)(sm_bytes - n)},
                   reinterpret_cast<const uint4 *>(h->d_tables), reinterpret_cast<uint4 *>(o.luts),
                   (uint32_t)(lut_bytes / 16), h->d_tables + lut_bytes, o.code_lengths};
    prepare_kernel<<<148 * 4, 256, 0, s>>>(pr);
    const uint32_t chunk_bits = 8 * h->C, block_bits = 8 * h->C * h->T;
    const uint32_t chunk_words = h->C / 4, block_words = h->C / 4 * h->T;
    const PackArgs pa{d_bf16[i], n, h->vec, h->d_tab, h->r, bs32, o.sign_mantissa, h->d_gap,
                      h->d_first, o.block_out_pos, chunks, (uint32_t)h->num_blocks,
                      chunk_bits, block_bits, chunk_words, block_words,
                      chunk_words > 1 ? UINT64_MAX / chunk_words + 1 : 0,
                      block_words > 1 ? UINT64_MAX / block_words + 1 : 0,
                      (uint32_t)(((1ull << 32) + chunk_bits - 1) / chunk_bits)};
    if (h->r.units) {
      const uint64_t want = resident(pack_kernel), ctas = (h->r.units + 7) / 8;
      const unsigned grid = (unsigned)(ctas < want ? ctas : want);
      pack_kernel<<<grid, kThreads, 0, s>>>(pa);
    }
    const FinishArgs fa{h->d_gap, h->d_first, o.gaps, o.chunk_counts, o.block_out_pos,
                        h->d_max, 8ull * h->C, chunks, 8ull * h->C * h->T, h->total,
                        h->last_start, (uint32_t)h->num_blocks, (uint32_t)n};
    unsigned grid;
    if (chunks) {
      if (!grid_for(chunks / 8, 256, &grid)) {
        st = DF11_ERR_TOO_LARGE;
        break;
      }
      finish_chunks<<<grid, 256, 0, s>>>(fa);
    }
    grid_for(h->num_blocks + 1, 256, &grid);
    finish_blocks<<<grid, 256, 0, s>>>(fa);
    if (cudaGetLastError() != cudaSuccess ||
        cudaMemcpyAsync(st_lens + 256, h->d_max, 3 * sizeof(unsigned int), cudaMemcpyDeviceToHost,
                        s) != cudaSuccess) {
      st = DF11_ERR_CUDA;
      break;
    }
  }
  if (st == DF11_OK && cudaStreamSynchronize(s) != cudaSuccess) st = DF11_ERR_CUDA;
  for (int i = 0; i < count && st == DF11_OK; ++i) {
    const df11_gpu_build *h = handles[i];
    unsigned int mx[3];
    std::memcpy(mx, stage + off[i] + h->luts.size() * 4 + 256, sizeof(mx));
    fill_params(h, &params[i]);
    params[i].max_block_elems = mx[0];
    params[i].max_chunk_elems = mx[1];
    params[i].max_warp_elems = mx[2];
  }
  if (st != DF11_OK) cudaStreamSynchronize(s);  // the staging buffer is read until then
  if (lock.owns_lock()) lock.unlock();
  for (int i = 0; i < count; ++i) {
    if (!handles[i]) continue;
    handles[i]->stream = s;  // frees follow this call's work
    df11_gpu_build_free(handles[i]);
  }
  return st;
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
    const uint64_t tiles = (n + kPerCta - 1) / kPerCta, slots = resident(hist_kernel);
    const bool vec = ((uintptr_t)d_bf16 & 15) == 0;
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3((unsigned)(tiles < slots ? tiles : slots));
    cfg.blockDim = dim3(kThreads);
    cfg.stream = s;
    unsigned long long *no_last = nullptr;
    // the launch's own status (not an earlier error of the calling thread)
    if (cudaLaunchKernelEx(&cfg, hist_kernel, d_bf16, n, vec, hd.addr, no_last) != cudaSuccess)
      return DF11_ERR_CUDA;
  }
  // straight into the caller's array (a DMA if the caller pinned it)
  if (cudaMemcpyAsync(hist, hd.addr, sizeof(g_exponent_hist), cudaMemcpyDeviceToHost, s) !=
          cudaSuccess ||
      cudaStreamSynchronize(s) != cudaSuccess)
    return DF11_ERR_CUDA;
  return DF11_OK;
}
