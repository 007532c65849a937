// Deterministic block top-k inside one CTA: keeps the k largest scores of a
// row of nb scores (a tie goes to the smaller block index) and writes the kept
// block indices in ascending order.  This is the selection of the critical
// set S_i (PISA §2 "Algoritmo Central") / SLA2's top-k router (§2B).
#pragma once

#include "common.cuh"

namespace sa {

constexpr int kMaxRouteBlocks = 4096;

// Ascending bitonic sort of n (a power of two) 64-bit keys in shared memory.
__device__ __forceinline__ void bitonic_sort_u64(unsigned long long* keys, int n) {
  for (int size = 2; size <= n; size <<= 1) {
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      __syncthreads();
      for (int i = threadIdx.x; i < (n >> 1); i += blockDim.x) {
        const int lo = 2 * i - (i & (stride - 1));
        const int hi = lo + stride;
        const bool asc = (lo & size) == 0;
        const unsigned long long a = keys[lo], b = keys[hi];
        if ((a > b) == asc) {
          keys[lo] = b;
          keys[hi] = a;
        }
      }
    }
  }
  __syncthreads();
}

// scores: nb floats in shared memory (read only); keys: scratch of
// next_pow2(nb) 64-bit words in shared memory; out: k int32 (global).
// All threads of the CTA must call it.
__device__ __forceinline__ void block_topk_ascending(const float* scores, int nb, int k,
                                                     unsigned long long* keys, int32_t* out) {
  int n = 1;
  while (n < nb) n <<= 1;
  // key = (descending score, ascending index): high word ~order(score)
  for (int j = threadIdx.x; j < n; j += blockDim.x) {
    keys[j] = j < nb ? ((unsigned long long)(~order_key(scores[j])) << 32) | (unsigned)j
                     : ~0ull;
  }
  bitonic_sort_u64(keys, n);
  // second pass: the first k indices, ascending (each thread rewrites only
  // the entries it reads)
  for (int j = threadIdx.x; j < n; j += blockDim.x)
    keys[j] = j < k ? (keys[j] & 0xffffffffull) : ~0ull;
  bitonic_sort_u64(keys, n);
  for (int j = threadIdx.x; j < k; j += blockDim.x) out[j] = (int32_t)keys[j];
  __syncthreads();
}

}  // namespace sa
