// df11_decode.cu -- DF11 decode on sm_100a (B200) and the C ABI around it.
//
// One thread block decodes one block of T chunks of C bitstream bytes:
//
//   stage    one thread issues bulk asynchronous copies (cp.async.bulk, no
//            multicast) of the block's bitstream slice and gap fields, and of
//            its sign/mantissa bytes, into shared memory; meanwhile all
//            threads copy table 0 and the code lengths into shared memory.
//   phase 1  "locate" ("DFloat11重新定义LLM无损压缩的技术边界" (ocdem.com)
//            §2.2): each thread walks its chunk from its gap with the
//            table and counts the codewords that start in it.
//   scan     exclusive prefix sum of the counts (warp shuffles, then across
//            warps) gives every thread its first output index; the block's
//            total must equal its block_out_pos difference.
//   phase 2  "reconstruct": each thread decodes its chunk again and writes
//            its exponents to their final places in a shared-memory array.
//   output   every thread fuses 16 exponents with 16 sign/mantissa bytes
//            into 16 BF16 words with byte permutes and writes them with two
//            16-byte stores; the block's ragged ends use 2-byte stores.
//
// Tables: table 0 lives in shared memory with its exponent bytes rotated
// right by one bit (e>>1 | (e&1)<<7), which turns the BF16 rebuild into two
// byte permutes and one bitwise select per output word.  Deeper tables (only
// codewords longer than 8 bits reach them) are read from shared memory when
// few, from global memory otherwise.
//
// Nothing here waits on another block, so nothing can hang: the only waits
// are on this block's own copies, bounded, reporting DF11_DEV_ERR_TIMEOUT.
#include <cuda_runtime.h>

#include <atomic>
#include <cstdint>

#include "df11.h"

namespace {

constexpr int kSubTablesInSmem = 8;     // deeper tables kept in shared memory
constexpr uint32_t kSpinLimit = 1u << 20;  // x ~1 us suspend hint: ~1 s
constexpr uint32_t kSuspendHintNs = 1000;

struct KTensor {
  const uint8_t *bitstream;
  const uint8_t *gaps;
  const uint32_t *block_out_pos;
  const uint32_t *luts;
  const uint8_t *code_lengths;
  const uint8_t *sign_mantissa;
  uint16_t *out;
  uint64_t total_bits;
  uint32_t n;
  uint32_t num_blocks;
  uint32_t num_luts;
  uint32_t max_block_elems;
  uint32_t block_begin;  // first grid block of this tensor
  uint32_t pad;
};

struct KBatch {
  KTensor t[DF11_MAX_BATCH];
  int32_t *err;
  int count;
  uint32_t stage_bytes;  // bytes of each of the sign/mantissa and exponent stages
  uint32_t sub_in_smem;  // deeper tables copied to shared memory
};

// shared memory layout (bytes); every buffer starts on a 16-byte boundary
constexpr uint32_t kOffMbar = 0;      // 2 mbarriers
constexpr uint32_t kOffScan = 16;     // 36 ints
constexpr uint32_t kOffLens = 160;    // 256 code lengths, by rotated exponent
constexpr uint32_t kOffLut0 = 416;    // 256 x u32
constexpr uint32_t kOffBits = 1440;   // T*C + 16 bitstream bytes, then gaps ...

template <int T, int C>
struct Layout {
  static constexpr uint32_t bits_bytes = T * C + 16;
  static constexpr uint32_t gaps_bytes = T * 5 / 8 + 16;
  static constexpr uint32_t off_gaps = kOffBits + bits_bytes;
  static constexpr uint32_t off_sm = off_gaps + gaps_bytes;
  static_assert(bits_bytes % 16 == 0 && gaps_bytes % 16 == 0, "alignment");
};

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

// Bounded wait for phase `parity` of an mbarrier; false on timeout.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity) {
  for (uint32_t i = 0; i < kSpinLimit; ++i) {
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

// 5-bit gap field k of a block's gap bytes (MSB-first packing)
__device__ __forceinline__ int read_gap(const uint8_t *g, int k) {
  const int bit = 5 * k;
  const uint32_t v = ((uint32_t)g[bit >> 3] << 8) | g[(bit >> 3) + 1];
  return (int)((v >> (11 - (bit & 7))) & 31u);
}

// Walk one thread's codewords [pos, end) (bit positions relative to its
// chunk's first bit) through the tables; count them and, when EMIT, write
// their (rotated) exponents to dst.  w holds the chunk and the 8 bytes after
// it as big-endian 32-bit words.  Sets *bad on inconsistent data.
template <int C, bool EMIT>
__device__ __forceinline__ int decode_run(const uint32_t (&w)[C / 4 + 2], int pos,
                                          const int end, const uint32_t *__restrict__ lut0,
                                          const uint8_t *__restrict__ lens,
                                          const uint32_t *sub, uint32_t num_luts,
                                          uint8_t *dst, int &bad) {
  constexpr int NW = C / 4 + 2;
  int count = 0;
#pragma unroll
  for (int k = 0; k < NW - 1; ++k) {
    const int lim = min(32 * (k + 1), end);
    const uint32_t hi = w[k], lo = w[k + 1];
    while (pos < lim) {
      const uint32_t win = __funnelshift_l(lo, hi, (uint32_t)pos);  // bits [pos, pos+32)
      uint32_t e = lut0[win >> 24];
      uint32_t nbits = (e >> 24) & 15u;
      if (nbits - 1u >= (uint32_t)(end - pos)) {
        // rare: a codeword longer than 8 bits (nbits == 0: pointer), or the
        // entry's codewords run past the end of this thread's region
        uint32_t sym;
        if (nbits == 0) {
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
          if (f == 0) {
            bad = DF11_DEV_ERR_TABLE;
            return count;
          }
          sym = rot8x3(f & 0xFFu);
        } else {
          sym = e & 0xFFu;
        }
        nbits = lens[sym];
        if (nbits == 0) {
          bad = DF11_DEV_ERR_TABLE;
          return count;
        }
        e = sym | (1u << 28);
      }
      const uint32_t nsym = e >> 28;
      if (EMIT) {
        dst[0] = (uint8_t)e;
        if (nsym >= 2) dst[1] = (uint8_t)(e >> 8);
        if (nsym >= 3) dst[2] = (uint8_t)(e >> 16);
        dst += nsym;
      }
      count += (int)nsym;
      pos += (int)nbits;
    }
  }
  if (pos != end) bad = DF11_DEV_ERR_OVERRUN;
  return count;
}

// four sign/mantissa bytes and four rotated exponents -> four BF16 words
__device__ __forceinline__ uint2 fuse4(uint32_t sm4, uint32_t er4) {
  const uint32_t p0 = __byte_perm(sm4, er4, 0x5140), q0 = __byte_perm(sm4, er4, 0x1504);
  const uint32_t p1 = __byte_perm(sm4, er4, 0x7362), q1 = __byte_perm(sm4, er4, 0x3726);
  return make_uint2((p0 & 0x7F7F7F7Fu) | (q0 & 0x80808080u),
                    (p1 & 0x7F7F7F7Fu) | (q1 & 0x80808080u));
}

__device__ __forceinline__ uint16_t fuse1(uint32_t sm, uint32_t er) {
  return (uint16_t)(((sm & 0x80u) << 8) | ((er & 0x7Fu) << 8) | (er & 0x80u) | (sm & 0x7Fu));
}

template <int T, int C>
__global__ void __launch_bounds__(T) df11_decode_kernel(const __grid_constant__ KBatch kb) {
  using L = Layout<T, C>;
  constexpr int NW = C / 4 + 2;
  extern __shared__ __align__(128) uint8_t smem[];
  uint64_t *mbar = reinterpret_cast<uint64_t *>(smem + kOffMbar);
  int *scan = reinterpret_cast<int *>(smem + kOffScan);
  uint8_t *lens_s = smem + kOffLens;
  uint32_t *lut0_s = reinterpret_cast<uint32_t *>(smem + kOffLut0);
  uint8_t *bits_s = smem + kOffBits;
  uint8_t *gaps_s = smem + L::off_gaps;
  uint8_t *sm_s = smem + L::off_sm;
  uint8_t *ex_s = sm_s + kb.stage_bytes;
  uint32_t *sub_s = reinterpret_cast<uint32_t *>(ex_s + kb.stage_bytes);

  int ti = 0;
  for (int i = 1; i < kb.count; ++i)
    if (blockIdx.x >= kb.t[i].block_begin) ti = i;
  const KTensor &tk = kb.t[ti];
  const uint32_t b = blockIdx.x - tk.block_begin;
  const int tid = threadIdx.x;

  const uint32_t P0 = tk.block_out_pos[b], P1 = tk.block_out_pos[b + 1];
  const uint32_t expected = P1 - P0;
  if (P1 < P0 || P1 > tk.n || expected > tk.max_block_elems || expected + 32 > kb.stage_bytes) {
    if (tid == 0) report(kb.err, DF11_DEV_ERR_CAPACITY);
    return;
  }
  const uint32_t bar_in = smem_addr(&mbar[0]), bar_sm = smem_addr(&mbar[1]);
  const uint32_t sm_begin = P0 & ~15u;
  const uint32_t sm_bytes = ((P1 + 15u) & ~15u) - sm_begin;
  if (tid == 0) {
    mbar_init(bar_in, 1);
    mbar_init(bar_sm, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    mbar_arrive_expect_tx(bar_in, L::bits_bytes + L::gaps_bytes);
    bulk_g2s(smem_addr(bits_s), tk.bitstream + (size_t)b * (T * C), L::bits_bytes, bar_in);
    bulk_g2s(smem_addr(gaps_s), tk.gaps + (size_t)b * (T * 5 / 8), L::gaps_bytes, bar_in);
    mbar_arrive_expect_tx(bar_sm, sm_bytes);
    if (sm_bytes) bulk_g2s(smem_addr(sm_s), tk.sign_mantissa + sm_begin, sm_bytes, bar_sm);
  }
  // tables: level 0 with rotated exponent bytes, code lengths by rotated
  // exponent, deeper tables verbatim
  for (int i = tid; i < 256; i += T) {
    uint32_t e = tk.luts[i] & 0x3FFFFFFFu;
    if ((e >> 24) & 15u) e = (e & 0xFF000000u) | rot8x3(e);
    lut0_s[i] = e;
    lens_s[((uint32_t)i >> 1) | (((uint32_t)i & 1u) << 7)] = tk.code_lengths[i];
  }
  const uint32_t *sub = tk.luts + 256;
  if (kb.sub_in_smem) {
    const uint32_t words = (tk.num_luts - 1) * 256;
    for (uint32_t i = tid; i < words; i += T) sub_s[i] = sub[i];
    sub = sub_s;
  }
  __syncthreads();  // tables and barrier initialisation visible to all

  int bad = 0;
  if (!mbar_wait(bar_in, 0)) bad = DF11_DEV_ERR_TIMEOUT;

  // this thread's region of the stream, relative to its chunk's first bit
  const uint64_t chunk_bit = ((uint64_t)b * T + tid) * (uint64_t)(C * 8);
  int start = read_gap(gaps_s, tid);
  int end = C * 8 + read_gap(gaps_s, tid + 1);
  if (chunk_bit >= tk.total_bits) {
    start = end = 0;
  } else if ((uint64_t)end > tk.total_bits - chunk_bit) {
    end = (int)(tk.total_bits - chunk_bit);
  }
  uint32_t w[NW];
#pragma unroll
  for (int k = 0; k < NW; ++k)
    w[k] = __byte_perm(*reinterpret_cast<const uint32_t *>(bits_s + tid * C + 4 * k), 0, 0x0123);

  // phase 1: count
  int cnt = 0;
  if (!bad) cnt = decode_run<C, false>(w, start, end, lut0_s, lens_s, sub, tk.num_luts, nullptr, bad);

  // block exclusive scan of the counts
  const int lane = tid & 31, warp = tid >> 5;
  int incl = cnt;
#pragma unroll
  for (int d = 1; d < 32; d <<= 1) {
    const int v = __shfl_up_sync(0xFFFFFFFFu, incl, d);
    if (lane >= d) incl += v;
  }
  if (lane == 31) scan[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    const int v = lane < T / 32 ? scan[lane] : 0;
    int s = v;
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
      const int u = __shfl_up_sync(0xFFFFFFFFu, s, d);
      if (lane >= d) s += u;
    }
    if (lane < T / 32) scan[lane] = s - v;
    if (lane == 31) scan[32] = s;
  }
  const int any_bad = __syncthreads_or(bad);
  const int excl = scan[warp] + incl - cnt;
  const uint32_t total = (uint32_t)scan[32];
  if (any_bad || total != expected) {
    if (bad) report(kb.err, bad);
    else if (tid == 0 && !any_bad) report(kb.err, DF11_DEV_ERR_COUNT);
    mbar_wait(bar_sm, 0);  // never leave with a copy in flight
    return;
  }

  // phase 2: exponents to their final places (index i <-> element sm_begin+i)
  const uint32_t head = P0 & 15u;
  decode_run<C, true>(w, start, end, lut0_s, lens_s, sub, tk.num_luts, ex_s + head + excl, bad);
  __syncthreads();
  if (!mbar_wait(bar_sm, 0)) {
    if (tid == 0) report(kb.err, DF11_DEV_ERR_TIMEOUT);
    return;
  }

  // output: fuse and store, 16 elements per thread per step
  uint16_t *out = tk.out + sm_begin;
  const uint32_t span = head + expected;
  const uint32_t groups = (span + 15u) >> 4;
  for (uint32_t g = tid; g < groups; g += T) {
    const uint32_t i0 = g << 4;
    if (i0 >= head && i0 + 16u <= span) {
      const uint4 s = *reinterpret_cast<const uint4 *>(sm_s + i0);
      const uint4 r = *reinterpret_cast<const uint4 *>(ex_s + i0);
      const uint2 a = fuse4(s.x, r.x), c = fuse4(s.y, r.y);
      const uint2 d = fuse4(s.z, r.z), f = fuse4(s.w, r.w);
      uint4 *o = reinterpret_cast<uint4 *>(out + i0);
      o[0] = make_uint4(a.x, a.y, c.x, c.y);
      o[1] = make_uint4(d.x, d.y, f.x, f.y);
    } else {
      const uint32_t lo = i0 > head ? i0 : head, hi = i0 + 16u < span ? i0 + 16u : span;
      for (uint32_t i = lo; i < hi; ++i) out[i] = fuse1(sm_s[i], ex_s[i]);
    }
  }
}

// ---------------------------------------------------------------------------
// host side

bool supported(uint32_t C, uint32_t T) {
  if (T == 256) return C == 4 || C == 8 || C == 16;
  if (T == 128 || T == 512) return C == 8;
  return false;
}

uint32_t stage_bytes_for(uint32_t max_block_elems) {
  return (max_block_elems + 32u + 15u) & ~15u;
}

size_t shared_bytes(uint32_t C, uint32_t T, uint32_t stage, uint32_t sub_tables) {
  return (size_t)kOffBits + (T * C + 16) + (T * 5 / 8 + 16) + 2 * (size_t)stage +
         (size_t)sub_tables * 1024;
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
      !aligned(t.sign_mantissa, 16) || !aligned(t.out_bf16, 16) || !aligned(t.block_out_pos, 4))
    return DF11_ERR_ALIGN;
  if (!supported(p.chunk_bytes, p.threads_per_block)) return DF11_ERR_UNSUPPORTED;
  const uint64_t block_bits = 8ull * p.chunk_bytes * p.threads_per_block;
  if (p.total_bits < p.n || p.total_bits > 32ull * p.n) return DF11_ERR_FORMAT;
  if ((uint64_t)p.num_blocks != (p.total_bits + block_bits - 1) / block_bits) return DF11_ERR_FORMAT;
  if (p.num_luts < 1 || p.num_luts >= (1u << 24)) return DF11_ERR_FORMAT;
  if (p.max_block_elems > 8ull * p.chunk_bytes * p.threads_per_block) return DF11_ERR_FORMAT;
  if (p.max_block_elems == 0) return DF11_ERR_FORMAT;
  return DF11_OK;
}

template <int T, int C>
df11_status launch(const KBatch &kb, uint32_t grid, size_t smem, cudaStream_t s) {
  static std::atomic<size_t> configured[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return DF11_ERR_CUDA;
  auto kern = df11_decode_kernel<T, C>;
  if (smem > 48 * 1024 && dev < 64 && configured[dev].load() < smem) {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
        cudaSuccess)
      return DF11_ERR_CUDA;
    configured[dev].store(smem);
  }
  kern<<<grid, T, smem, s>>>(kb);
  return cudaGetLastError() == cudaSuccess ? DF11_OK : DF11_ERR_CUDA;
}

df11_status launch_batch(const df11_tensor *ts, int count, int32_t *d_err, cudaStream_t s) {
  KBatch kb{};
  kb.err = d_err;
  uint32_t grid = 0, max_elems = 0, max_luts = 1, C = 0, T = 0;
  for (int i = 0; i < count; ++i) {
    const df11_params &p = ts[i].params;
    if (p.n == 0) continue;
    KTensor &k = kb.t[kb.count++];
    k.bitstream = ts[i].bitstream;
    k.gaps = ts[i].gaps;
    k.block_out_pos = ts[i].block_out_pos;
    k.luts = ts[i].luts;
    k.code_lengths = ts[i].code_lengths;
    k.sign_mantissa = ts[i].sign_mantissa;
    k.out = ts[i].out_bf16;
    k.total_bits = p.total_bits;
    k.n = (uint32_t)p.n;
    k.num_blocks = p.num_blocks;
    k.num_luts = p.num_luts;
    k.max_block_elems = p.max_block_elems;
    k.block_begin = grid;
    if ((uint64_t)grid + p.num_blocks > 0x7FFFFFFFu) return DF11_ERR_TOO_LARGE;
    grid += p.num_blocks;
    max_elems = max_elems > p.max_block_elems ? max_elems : p.max_block_elems;
    max_luts = max_luts > p.num_luts ? max_luts : p.num_luts;
    C = p.chunk_bytes;
    T = p.threads_per_block;
  }
  if (kb.count == 0 || grid == 0) return DF11_OK;
  kb.stage_bytes = stage_bytes_for(max_elems);
  kb.sub_in_smem = (max_luts - 1) <= (uint32_t)kSubTablesInSmem ? 1u : 0u;
  const size_t smem = shared_bytes(C, T, kb.stage_bytes, kb.sub_in_smem ? max_luts - 1 : 0);
  if (smem > 227 * 1024) return DF11_ERR_TOO_LARGE;
  if (T == 256 && C == 8) return launch<256, 8>(kb, grid, smem, s);
  if (T == 256 && C == 4) return launch<256, 4>(kb, grid, smem, s);
  if (T == 256 && C == 16) return launch<256, 16>(kb, grid, smem, s);
  if (T == 128 && C == 8) return launch<128, 8>(kb, grid, smem, s);
  if (T == 512 && C == 8) return launch<512, 8>(kb, grid, smem, s);
  return DF11_ERR_UNSUPPORTED;
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
  df11_tensor t{bitstream, gaps, block_out_pos, luts, code_lengths, sign_mantissa, out_bf16, *params};
  df11_status st = validate(t);
  if (st != DF11_OK || n == 0) return st;
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
  for (int i = 0; i < count; i += DF11_MAX_BATCH) {
    const int c = count - i < DF11_MAX_BATCH ? count - i : DF11_MAX_BATCH;
    df11_status st = launch_batch(tensors + i, c, d_err, (cudaStream_t)stream);
    if (st != DF11_OK) return st;
  }
  return DF11_OK;
}

size_t df11_shared_bytes(const df11_params *p) {
  if (!p || !supported(p->chunk_bytes, p->threads_per_block)) return 0;
  const uint32_t subs = p->num_luts - 1 <= (uint32_t)kSubTablesInSmem ? p->num_luts - 1 : 0;
  return shared_bytes(p->chunk_bytes, p->threads_per_block, stage_bytes_for(p->max_block_elems),
                      subs);
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
    case DF11_DEV_ERR_CAPACITY: return "block holds more elements than max_block_elems";
  }
  return "unknown device error";
}

}  // extern "C"
