// df11_codebook.h -- the codebook half of the DF11 format builder, shared by
// the host builder (df11_build.cpp) and the device builder
// (df11_gpu_build.cu): from an exponent histogram to code lengths, canonical
// codewords and the hierarchical 256-entry tables.  Internal to the library.
#pragma once
#include <cstdint>
#include <vector>

namespace df11_internal {

// Code lengths (Huffman, limited to 32 bits by package-merge when deeper),
// canonical codewords and lookup tables of a histogram.  Returns the longest
// code length.
int codebook(const uint64_t hist[256], uint8_t len[256], uint32_t code[256],
             std::vector<uint32_t> &luts);

}  // namespace df11_internal
