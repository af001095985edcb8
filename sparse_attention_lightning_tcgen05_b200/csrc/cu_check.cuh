// cu_check.cuh -- device-side check of the packed-sequence offsets of a
// CAUSAL call.
//
// The score and top-k kernels derive every row's place in the packed score
// buffer from cu_seqlens (sequence i's [L_i, L_i] block at float offset
// sum_{j<i} L_j^2). An array that is not what the descriptor promises
// (cu[0] = 0, non-decreasing, cu[num_seqs] = T) would send their stores
// outside the caller's buffers. The array lives in device memory, so the
// host cannot look at it without a synchronisation; this one-CTA kernel runs
// first on the stream and writes a flag that the later kernels of the call
// read after their dependency wait: when it is set they write nothing.
#pragma once

#include <cstdint>

#include "sm100_ptx.cuh"

namespace dsa {

constexpr unsigned int kStatusInvalidArg = 1;   // == DSA_ERR_INVALID_ARG

// cap_elems >= 0: the score rows must also fit in that many floats (the
// workspace holds them). Writes *cu_bad (0 or 1) every call; a bad array
// also records kStatusInvalidArg in *err unless an earlier failure is there.
template <int NT>
__global__ void __launch_bounds__(NT) cu_seqlens_check_kernel(const int *cu, int num_seqs, int T,
                                                             long long cap_elems,
                                                             unsigned int *cu_bad,
                                                             unsigned int *err) {
  __shared__ unsigned long long total;
  grid_dep_wait();                 // cu_seqlens may come from earlier work
  grid_dep_launch_dependents();
  if (threadIdx.x == 0) total = 0ull;
  __syncthreads();
  int bad = 0;
  unsigned long long part = 0;
  for (int i = threadIdx.x; i < num_seqs; i += NT) {
    const int a = __ldg(cu + i), b = __ldg(cu + i + 1);
    if (b < a) bad = 1;
    const long long L = static_cast<long long>(b) - a;
    part += static_cast<unsigned long long>(L * L);
  }
  if (threadIdx.x == 0 && (__ldg(cu) != 0 || __ldg(cu + num_seqs) != T)) bad = 1;
  if (part) atomicAdd(&total, part);
  bad = __syncthreads_or(bad);
  if (threadIdx.x == 0) {
    if (!bad && cap_elems >= 0 && total > static_cast<unsigned long long>(cap_elems)) bad = 1;
    *cu_bad = bad ? 1u : 0u;
    if (bad) atomicCAS(err, 0u, kStatusInvalidArg);
  }
}

}  // namespace dsa
