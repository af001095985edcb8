// row_rule.cuh -- where a decode-style score row stops being valid.
//
// POSITIONS (DeepSeek-V3.2 Sparse Indexer Kernel API Reference, positions):
// slot s of token t is valid iff s <= positions[t].
// COMPRESSED (NeMo AutoModel optimized_kernels, dsv4_indexer_scores, read as
// a causal pool): pooled slot j holds raw tokens [j*r, (j+1)*r) and is valid
// for the token at absolute position query_start + t once all of them have
// been seen, (j+1)*r <= query_start + t + 1, i.e.
//     j <= floor((query_start + t + 1) / r) - 1.
// The host keeps query_start + T below 2^31, so that numerator is a 31-bit
// unsigned integer and the division by r (fixed for a launch) becomes one
// multiplication and one shift.
#pragma once

#include <cstdint>

#if !defined(__CUDACC__)
#define __host__
#define __device__
#define __forceinline__ inline
#endif

namespace dsa {

// Floor division by a divisor d fixed for a whole launch (Granlund and
// Montgomery, "Division by Invariant Integers using Multiplication", PLDI
// 1994, Theorem 4.2, for N = 31-bit numerators): with l = ceil(log2 d) and
// m = ceil(2^(31+l) / d), 2^(31+l) <= m*d < 2^(31+l) + 2^l, hence
// floor(n / d) = floor(m*n / 2^(31+l)) for every 0 <= n < 2^31. For
// 1 <= d < 2^31, m < 2^32.
struct DivMagic {
  uint32_t m;
  int shift;    // 31 + l
};

inline DivMagic div_magic(uint32_t d) {
  int l = 0;
  while ((uint64_t{1} << l) < d) ++l;
  const uint64_t two = uint64_t{1} << (31 + l);
  return {static_cast<uint32_t>((two + d - 1) / d), 31 + l};
}

__host__ __device__ __forceinline__ uint32_t div_by(uint32_t n, DivMagic g) {
  return static_cast<uint32_t>((static_cast<uint64_t>(g.m) * n) >> g.shift);
}

// The compressed rule's parameters: base = query_start + 1.
struct CompressedRule {
  int32_t base;
  DivMagic div;
};

// Largest valid pooled slot of token t (-1: none), for t < T.
__host__ __device__ __forceinline__ int compressed_last_slot(const CompressedRule &c, int t) {
  return static_cast<int>(div_by(static_cast<uint32_t>(c.base + t), c.div)) - 1;
}

}  // namespace dsa
