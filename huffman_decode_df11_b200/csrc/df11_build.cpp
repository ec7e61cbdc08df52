// df11_build.cpp -- host-side DF11 format builder (the offline "compress"
// step).  Multithreaded C++; host memory only.
//
// Steps (the pages' compression recipe, "DFloat11无损压缩技术" (jsqmd.com)
// §2.2 items 1-2):
//   1. split every BF16 word into its exponent and a sign/mantissa byte;
//   2. histogram the exponents;
//   3. Huffman code lengths (binary heap, ties by smallest symbol), reduced
//      to a 32-bit limit by package-merge when the tree is deeper;
//   4. canonical codewords from the lengths (count per length, first code
//      per length -- the bl_count/next_code construction of RFC 1951);
//   5. the hierarchical 256-entry tables ("multi-level compact lookup
//      tables", "DFloat11重新定义LLM无损压缩的技术边界" (ocdem.com) §2.2),
//      filled range by range from the codewords;
//   6. the bitstream, packed in parallel over element ranges, with the gap
//      of every chunk and the output position of every block recorded as
//      the codeword starts go by.
#include <algorithm>
#include <array>
#include <atomic>
#include <cstdint>
#include <cstdlib>
#include <cstring>
#include <map>
#include <queue>
#include <thread>
#include <tuple>
#include <vector>

#include "df11.h"
#include "df11_codebook.h"

namespace {

constexpr int kMaxLen = 32;

template <class F>
void parallel_for(int workers, uint64_t n, F &&fn) {
  // fn(worker, begin, end) on `workers` contiguous slices of [0, n)
  if (workers <= 1 || n < (1u << 16)) {
    fn(0, 0, n);
    return;
  }
  std::vector<std::thread> pool;
  pool.reserve(workers);
  for (int w = 0; w < workers; ++w) {
    uint64_t b = n * w / workers, e = n * (w + 1) / workers;
    pool.emplace_back([&, w, b, e] { fn(w, b, e); });
  }
  for (auto &t : pool) t.join();
}

// ---- 3. code lengths --------------------------------------------------
// Huffman with a binary heap keyed on (weight, smallest symbol).
int huffman_depths(const uint64_t hist[256], uint8_t len[256]) {
  struct Node {
    uint64_t w;
    int minsym;
    int id;
  };
  auto heavier = [](const Node &a, const Node &b) {
    return std::tie(a.w, a.minsym) > std::tie(b.w, b.minsym);
  };
  std::priority_queue<Node, std::vector<Node>, decltype(heavier)> heap(heavier);
  std::vector<int> parent;
  std::vector<int> leaf(256, -1);
  for (int s = 0; s < 256; ++s) {
    len[s] = 0;
    if (hist[s]) {
      leaf[s] = (int)parent.size();
      heap.push({hist[s], s, (int)parent.size()});
      parent.push_back(-1);
    }
  }
  int leaves = (int)parent.size();
  if (leaves == 0) return 0;
  if (leaves == 1) {
    for (int s = 0; s < 256; ++s)
      if (leaf[s] >= 0) len[s] = 1;
    return 1;
  }
  while (heap.size() > 1) {
    Node a = heap.top();
    heap.pop();
    Node b = heap.top();
    heap.pop();
    int id = (int)parent.size();
    parent.push_back(-1);
    parent[a.id] = id;
    parent[b.id] = id;
    heap.push({a.w + b.w, std::min(a.minsym, b.minsym), id});
  }
  // depth of every node, parents are created after their children
  std::vector<int> depth(parent.size(), 0);
  for (int v = (int)parent.size() - 2; v >= 0; --v) depth[v] = depth[parent[v]] + 1;
  int longest = 0;
  for (int s = 0; s < 256; ++s)
    if (leaf[s] >= 0) {
      len[s] = (uint8_t)std::min(depth[leaf[s]], 255);
      longest = std::max(longest, depth[leaf[s]]);
    }
  return longest;
}

// Package-merge with the lengths read back through item back-pointers:
// every list item is a leaf or a package of two items of the list below;
// a selected package adds one to the lengths of all leaves inside it.
// Order rules: leaves by (weight, symbol); when a leaf and a package weigh
// the same, the leaf comes first; adjacent pairs are packaged.
int package_merge(const uint64_t hist[256], int limit, uint8_t len[256]) {
  std::vector<int> syms;
  for (int s = 0; s < 256; ++s) {
    len[s] = 0;
    if (hist[s]) syms.push_back(s);
  }
  const int m = (int)syms.size();
  if (m == 0) return 0;
  if (m == 1) {
    len[syms[0]] = 1;
    return 1;
  }
  std::stable_sort(syms.begin(), syms.end(), [&](int a, int b) {
    return std::tie(hist[a], a) < std::tie(hist[b], b);
  });
  struct Item {
    uint64_t w;
    int sym;    // >= 0 for a leaf
    int child;  // index of the first of two items in the lower list
  };
  std::vector<std::vector<Item>> lists(limit);
  for (int s : syms) lists[limit - 1].push_back({hist[s], s, -1});
  for (int lv = limit - 2; lv >= 0; --lv) {
    const auto &lower = lists[lv + 1];
    auto &cur = lists[lv];
    size_t packages = lower.size() / 2, li = 0, pi = 0;
    cur.reserve(m + packages);
    while (li < (size_t)m || pi < packages) {
      uint64_t pw = pi < packages ? lower[2 * pi].w + lower[2 * pi + 1].w : 0;
      if (pi >= packages || (li < (size_t)m && hist[syms[li]] <= pw)) {
        cur.push_back({hist[syms[li]], syms[li], -1});
        ++li;
      } else {
        cur.push_back({pw, -1, (int)(2 * pi)});
        ++pi;
      }
    }
  }
  // walk down: in list 0 the first 2m-2 items are selected; a selected
  // package selects its two children in the next list
  std::vector<int> lens(256, 0);
  size_t take = 2 * (size_t)m - 2;
  for (int lv = 0; lv < limit; ++lv) {
    size_t next_take = 0;
    for (size_t i = 0; i < take; ++i) {
      const Item &it = lists[lv][i];
      if (it.sym >= 0) {
        lens[it.sym]++;
      } else {
        next_take = std::max(next_take, (size_t)it.child + 2);
      }
    }
    take = next_take;
    if (take == 0) break;
  }
  int longest = 0;
  for (int s = 0; s < 256; ++s) {
    len[s] = (uint8_t)lens[s];
    longest = std::max(longest, lens[s]);
  }
  return longest;
}

// ---- 4. canonical codes (RFC 1951 bl_count / next_code) ---------------
void canonical(const uint8_t len[256], uint32_t code[256]) {
  uint32_t count[kMaxLen + 2] = {0};
  for (int s = 0; s < 256; ++s)
    if (len[s]) count[len[s]]++;
  uint64_t next[kMaxLen + 2] = {0};
  uint64_t c = 0;
  for (int l = 1; l <= kMaxLen; ++l) {
    c = (c + count[l - 1]) << 1;
    next[l] = c;
  }
  // with count[0] == 0 the first length's first code is 0
  for (int s = 0; s < 256; ++s) code[s] = len[s] ? (uint32_t)next[len[s]]++ : 0;
}

// ---- 5. lookup tables ---------------------------------------------------
constexpr uint32_t kSymbolsShift = 28;
constexpr uint32_t kBitsShift = 24;

std::vector<uint32_t> build_tables(const uint8_t len[256], const uint32_t code[256]) {
  // table keys: level k >= 1 and the 8k-bit prefix; numbered level by level,
  // ascending prefix within a level
  std::map<std::pair<int, uint64_t>, uint32_t> index;
  for (int k = 1; k <= 3; ++k)
    for (int s = 0; s < 256; ++s)
      if (len[s] > 8 * k) index[{k, (uint64_t)code[s] >> (len[s] - 8 * k)}] = 0;
  uint32_t next_id = 1;
  for (auto &kv : index) kv.second = next_id++;  // std::map iterates (k, prefix) ascending
  std::vector<uint32_t> luts((size_t)next_id * 256, 0);

  // single-codeword view of the first 8 bits: symbol and length per index
  int16_t first_sym[256];
  uint8_t first_len[256];
  for (int i = 0; i < 256; ++i) {
    first_sym[i] = -1;
    first_len[i] = 0;
  }
  for (int s = 0; s < 256; ++s) {
    if (!len[s] || len[s] > 8) continue;
    uint32_t lo = code[s] << (8 - len[s]), hi = (code[s] + 1) << (8 - len[s]);
    for (uint32_t i = lo; i < hi; ++i) {
      first_sym[i] = (int16_t)s;
      first_len[i] = len[s];
    }
  }
  // level 0: up to three whole codewords per 8-bit index
  for (int i = 0; i < 256; ++i) {
    int used = 0, nsym = 0;
    uint32_t syms = 0;
    while (nsym < 3 && used < 8) {
      int j = (i << used) & 0xFF;  // remaining bits, left-aligned
      if (first_sym[j] < 0 || first_len[j] > 8 - used) break;
      syms |= (uint32_t)first_sym[j] << (8 * nsym);
      ++nsym;
      used += first_len[j];
    }
    if (nsym)
      luts[i] = syms | ((uint32_t)used << kBitsShift) | ((uint32_t)nsym << kSymbolsShift);
  }
  // pointers out of level 0 and of every sub-table, and sub-table symbols
  for (int s = 0; s < 256; ++s) {
    if (len[s] <= 8) continue;
    uint64_t c = code[s];
    int L = len[s];
    for (int k = 0; k <= 3; ++k) {
      uint32_t table = k == 0 ? 0 : index.at({k, c >> (L - 8 * k)});
      uint32_t *t = &luts[(size_t)table * 256];
      if (L <= 8 * k + 8) {
        // the codeword ends in this table: fill its index range
        uint32_t rest = (uint32_t)(c & ((1ull << (L - 8 * k)) - 1));
        uint32_t lo = rest << (8 * k + 8 - L), hi = (rest + 1) << (8 * k + 8 - L);
        for (uint32_t i = lo; i < hi; ++i) t[i] = (uint32_t)s | (1u << kSymbolsShift);
        break;
      }
      uint32_t i = (uint32_t)((c >> (L - 8 * k - 8)) & 0xFF);
      t[i] = index.at({k + 1, c >> (L - 8 * k - 8)});
    }
  }
  return luts;
}

}  // namespace

int df11_internal::codebook(const uint64_t hist[256], uint8_t len[256], uint32_t code[256],
                            std::vector<uint32_t> &luts) {
  int longest = huffman_depths(hist, len);
  if (longest > kMaxLen) longest = package_merge(hist, kMaxLen, len);
  canonical(len, code);
  luts = build_tables(len, code);
  return longest;
}

extern "C" df11_status df11_build(const uint16_t *w, uint64_t n, uint32_t C,
                                  uint32_t T, int num_threads,
                                  df11_host_tensor *out) {
  if (!out || (n && !w)) return DF11_ERR_NULL;
  std::memset(out, 0, sizeof(*out));
  if (C < 4 || C > 28 || C % 4) return DF11_ERR_INVALID;  // counts fit a byte
  if (T < 128 || T > 1024 || T % 128) return DF11_ERR_INVALID;
  if (n >= (1ull << 32)) return DF11_ERR_TOO_LARGE;
  int workers = num_threads > 0 ? num_threads : (int)std::thread::hardware_concurrency();
  workers = std::max(1, std::min(workers, 64));

  // 1-2. split and histogram
  out->sign_mantissa_bytes = (n + 15) / 16 * 16;
  out->sign_mantissa = (uint8_t *)std::calloc(out->sign_mantissa_bytes + 16, 1);
  if (!out->sign_mantissa) return DF11_ERR_NOMEM;
  std::vector<std::array<uint64_t, 256>> part(workers);
  for (auto &p : part) p.fill(0);
  parallel_for(workers, n, [&](int wk, uint64_t b, uint64_t e) {
    auto &h = part[wk];
    for (uint64_t i = b; i < e; ++i) {
      uint16_t x = w[i];
      h[(x >> 7) & 0xFF]++;
      out->sign_mantissa[i] = (uint8_t)(((x >> 8) & 0x80) | (x & 0x7F));
    }
  });
  uint64_t hist[256] = {0};
  for (auto &p : part)
    for (int s = 0; s < 256; ++s) hist[s] += p[s];

  // 3-5. code and tables
  uint8_t len[256];
  uint32_t code[256];
  std::vector<uint32_t> luts;
  const int longest = df11_internal::codebook(hist, len, code, luts);
  std::memcpy(out->code_lengths, len, 256);
  df11_params &p = out->params;
  p.n = n;
  p.chunk_bytes = C;
  p.threads_per_block = T;
  p.num_luts = (uint32_t)(luts.size() / 256);
  p.max_len = (uint32_t)longest;
  out->luts = (uint32_t *)std::malloc(luts.size() * 4);
  if (!out->luts) {
    df11_host_tensor_free(out);
    return DF11_ERR_NOMEM;
  }
  std::memcpy(out->luts, luts.data(), luts.size() * 4);

  // 6. bitstream, gaps, block positions
  // bit offset of every worker's first element
  std::vector<uint64_t> range_bits(workers + 1, 0);
  std::vector<uint64_t> bounds(workers + 1, 0);
  for (int k = 0; k <= workers; ++k) bounds[k] = n * k / workers;
  parallel_for(workers, (uint64_t)workers, [&](int, uint64_t b, uint64_t e) {
    for (uint64_t k = b; k < e; ++k) {
      uint64_t s = 0;
      for (uint64_t i = bounds[k]; i < bounds[k + 1]; ++i) s += len[(w[i] >> 7) & 0xFF];
      range_bits[k + 1] = s;
    }
  });
  for (int k = 0; k < workers; ++k) range_bits[k + 1] += range_bits[k];
  const uint64_t total = range_bits[workers];
  p.total_bits = total;
  const uint64_t chunk_bits = 8ull * C, block_bits = chunk_bits * T;
  p.num_blocks = (uint32_t)((total + block_bits - 1) / block_bits);
  const uint64_t chunks = (uint64_t)p.num_blocks * T;
  out->bitstream_bytes = chunks * C + 16;
  out->gaps_bytes = chunks * 5 / 8 + 16;
  out->bitstream = (uint8_t *)std::calloc(out->bitstream_bytes, 1);
  out->gaps = (uint8_t *)std::calloc(out->gaps_bytes, 1);
  out->block_out_pos = (uint32_t *)std::calloc((size_t)p.num_blocks + 1, 4);
  std::vector<uint8_t> gap(chunks ? chunks : 1, 0);
  // index of the first element whose codeword starts at or after each chunk
  std::vector<uint32_t> first_elem(chunks + 1, (uint32_t)n);
  if (!out->bitstream || !out->gaps || !out->block_out_pos) {
    df11_host_tensor_free(out);
    return DF11_ERR_NOMEM;
  }
  uint8_t *bs = out->bitstream;
  uint32_t *bpos = out->block_out_pos;
  parallel_for(workers, (uint64_t)workers, [&](int, uint64_t kb, uint64_t ke) {
    for (uint64_t k = kb; k < ke; ++k) {
      uint64_t i0 = bounds[k], i1 = bounds[k + 1];
      if (i0 == i1) continue;
      uint64_t bit = range_bits[k];
      // start of the previous codeword (or "none" for element 0)
      int64_t prev = i0 == 0 ? -1 : (int64_t)(bit - len[(w[i0 - 1] >> 7) & 0xFF]);
      uint64_t acc = 0;
      int pending = (int)(bit & 7);  // leading bits owned by the previous range
      uint64_t byte = bit >> 3;
      bool first_byte = true;
      for (uint64_t i = i0; i < i1; ++i) {
        int sym = (w[i] >> 7) & 0xFF;
        // chunks and blocks whose first codeword start is this one
        for (uint64_t c = prev < 0 ? 0 : (uint64_t)prev / chunk_bits + 1;
             c * chunk_bits <= bit && c < chunks; ++c) {
          gap[c] = (uint8_t)(bit - c * chunk_bits);
          first_elem[c] = (uint32_t)i;
        }
        for (uint64_t b = prev < 0 ? 0 : (uint64_t)prev / block_bits + 1;
             b * block_bits <= bit && b < p.num_blocks; ++b)
          bpos[b] = (uint32_t)i;
        prev = (int64_t)bit;
        int l = len[sym];
        acc = (acc << l) | code[sym];
        pending += l;
        bit += l;
        while (pending >= 8) {
          uint8_t v = (uint8_t)(acc >> (pending - 8));
          if (first_byte)
            __atomic_fetch_or(&bs[byte], v, __ATOMIC_RELAXED);
          else
            bs[byte] = v;
          first_byte = false;
          ++byte;
          pending -= 8;
        }
        acc &= (1ull << pending) - 1;
      }
      if (pending > 0) __atomic_fetch_or(&bs[byte], (uint8_t)(acc << (8 - pending)), __ATOMIC_RELAXED);
    }
  });
  // the stream's tail: chunks that begin inside the last codeword, blocks
  // that hold no codeword start
  if (n) {
    uint64_t last_start = total - len[(w[n - 1] >> 7) & 0xFF];
    for (uint64_t c = last_start / chunk_bits + 1; c * chunk_bits < total && c < chunks; ++c)
      gap[c] = (uint8_t)(total - c * chunk_bits);
    for (uint64_t b = last_start / block_bits + 1; b < p.num_blocks; ++b) bpos[b] = (uint32_t)n;
  }
  bpos[p.num_blocks] = (uint32_t)n;
  // pack the gaps, 8 chunks (40 bits = 5 bytes) per group
  parallel_for(workers, (chunks + 7) / 8, [&](int, uint64_t gb, uint64_t ge) {
    for (uint64_t g = gb; g < ge; ++g) {
      uint64_t v = 0;
      for (int j = 0; j < 8; ++j) {
        uint64_t c = g * 8 + j;
        v = (v << 5) | (c < chunks ? gap[c] : 0);
      }
      for (int j = 0; j < 5; ++j) out->gaps[g * 5 + j] = (uint8_t)(v >> (32 - 8 * j));
    }
  });
  uint32_t mx = 0;
  for (uint32_t b = 0; b < p.num_blocks; ++b) mx = std::max(mx, bpos[b + 1] - bpos[b]);
  p.max_block_elems = mx;
  out->chunk_counts_bytes = chunks + 16;
  out->chunk_counts = (uint8_t *)std::calloc(out->chunk_counts_bytes, 1);
  if (!out->chunk_counts) {
    df11_host_tensor_free(out);
    return DF11_ERR_NOMEM;
  }
  uint32_t mc = 0, mw = 0;
  for (uint64_t c = 0; c < chunks; ++c) {
    const uint32_t k = first_elem[c + 1] - first_elem[c];
    out->chunk_counts[c] = (uint8_t)k;
    mc = std::max(mc, k);
  }
  for (uint64_t g = 0; g < chunks; g += 32) {  // groups of 32 consecutive chunks
    const uint64_t e = std::min<uint64_t>(g + 32, chunks);
    mw = std::max(mw, first_elem[e] - first_elem[g]);
  }
  p.max_chunk_elems = mc;
  p.max_warp_elems = mw;
  return DF11_OK;
}

extern "C" void df11_host_tensor_free(df11_host_tensor *t) {
  if (!t) return;
  std::free(t->bitstream);
  std::free(t->gaps);
  std::free(t->block_out_pos);
  std::free(t->luts);
  std::free(t->sign_mantissa);
  std::free(t->chunk_counts);
  std::memset(t, 0, sizeof(*t));
}
