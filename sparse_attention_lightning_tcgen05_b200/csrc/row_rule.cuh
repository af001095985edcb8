// row_rule.cuh -- where a decode-style score row stops being valid.
//
// POSITIONS (DeepSeek-V3.2 Sparse Indexer Kernel API Reference, positions):
// slot s of token t is valid iff s <= positions[t].
// COMPRESSED (NeMo AutoModel optimized_kernels, dsv4_indexer_scores, read as
// a causal pool): pooled slot j holds raw tokens [j*r, (j+1)*r) and is valid
// for the token at absolute position query_start + t once all of them have
// been seen, (j+1)*r <= query_start + t + 1, i.e. j <= (query_start+t+1)/r - 1.
#pragma once

#include <cstdint>

namespace dsa {

// The row's "position": the largest valid slot, before clamping to the row.
// Negative: nothing is valid; >= S: every slot is. `positions` NULL selects
// the compressed rule. `positions` may point to global or shared memory.
__device__ __forceinline__ int64_t row_position(const int *positions, int64_t query_start,
                                                int ratio, int t) {
  if (positions) return positions[t];
  return (query_start + t + 1) / ratio - 1;
}

}  // namespace dsa
