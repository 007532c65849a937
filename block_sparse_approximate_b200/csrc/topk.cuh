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


// Shared memory of radix_topk_cta.
struct RadixTopkSmem {
  unsigned hist[256];
  uint32_t bits[kMaxRouteBlocks / 32];
  unsigned prefix, rank, cnt;
  unsigned mn[32], mx[32];
};

// radix_topk_cta: the top k of one row of nb <= kMaxRouteBlocks scores `sc`
// (global or shared memory) by a whole CTA of NTH threads (all of them call
// it), the kept indices written to `out` in ascending order.  Radix select
// over the 32-bit order keys of the scores (higher score = smaller key).  The
// keys of one row share their high bits (the scores span
// a narrow range), so the select starts below the highest bit in which the
// row's smallest and largest keys differ, and takes 8-bit digits from there:
// each pass histograms the digit of the keys that still match the prefix
// found so far, and the bin holding the k-th key extends the prefix.  Once
// that bin holds exactly the places left, every key in it is kept and the
// lower bits do not matter (usually after two passes); otherwise the passes
// run down to bit 0 and, of the keys equal to the k-th, the smallest indices
// fill the places left.  The kept indices are emitted in ascending order from
// a bitmap.
template <int NTH>
__device__ __forceinline__ void radix_topk_cta(const float* sc, int nb, int topk, int32_t* out, RadixTopkSmem& sm) {
  constexpr int KPT = (kMaxRouteBlocks + NTH - 1) / NTH;   // keys per thread
  constexpr int NW = NTH / 32;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  unsigned* hist = sm.hist;
  uint32_t* bits = sm.bits;
  unsigned& sh_prefix = sm.prefix;
  unsigned& sh_rank = sm.rank;
  unsigned& sh_cnt = sm.cnt;
  unsigned* sh_min = sm.mn;
  unsigned* sh_max = sm.mx;
  const int nwords = (nb + 31) / 32;

  uint32_t key[KPT];
  unsigned kmin = 0xffffffffu, kmax = 0u;
#pragma unroll
  for (int e = 0; e < KPT; ++e) {
    const int j = tid + e * NTH;
    key[e] = j < nb ? ~order_key(sc[j]) : 0xffffffffu;
    if (j < nb) {
      kmin = min(kmin, key[e]);
      kmax = max(kmax, key[e]);
    }
  }
  for (int x = tid; x < nwords; x += NTH) bits[x] = 0u;
  kmin = __reduce_min_sync(0xffffffffu, kmin);
  kmax = __reduce_max_sync(0xffffffffu, kmax);
  if (lane == 0) {
    sh_min[warp] = kmin;
    sh_max[warp] = kmax;
  }
  __syncthreads();
  kmin = sh_min[0];
  kmax = sh_max[0];
#pragma unroll
  for (int w = 1; w < NW; ++w) {
    kmin = min(kmin, sh_min[w]);
    kmax = max(kmax, sh_max[w]);
  }
  // bits above `hi` are common to every key of the row
  const unsigned diff = kmin ^ kmax;
  int hi = diff ? 31 - __clz(diff) : -1;
  unsigned mask = diff == 0u ? 0xffffffffu : (hi >= 31 ? 0u : ~((2u << hi) - 1u));
  unsigned prefix = kmin & mask;
  unsigned rank = (unsigned)topk, cnt = (unsigned)nb;
  while (hi >= 0 && cnt != rank) {
    const int lo = max(hi - 7, 0);
    const unsigned dmask = (2u << (hi - lo)) - 1u;      // the digit's bits, shifted down
    for (int x = tid; x < 256; x += NTH) hist[x] = 0u;
    __syncthreads();
#pragma unroll
    for (int e = 0; e < KPT; ++e) {
      const int j = tid + e * NTH;
      if (j < nb && (key[e] & mask) == prefix) atomicAdd(&hist[(key[e] >> lo) & dmask], 1u);
    }
    __syncthreads();
    if (warp == 0) {
      // the bin holding the rank-th smallest key among those matching prefix
      unsigned c[8], tot = 0;
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        c[e] = hist[lane * 8 + e];
        tot += c[e];
      }
      unsigned incl = tot;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const unsigned y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
      }
      const unsigned excl = incl - tot;
      if (excl < rank && rank <= incl) {
        unsigned run = excl;
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          if (run < rank && rank <= run + c[e]) {
            sh_prefix = prefix | ((unsigned)(lane * 8 + e) << lo);
            sh_rank = rank - run;
            sh_cnt = c[e];
          }
          run += c[e];
        }
      }
    }
    __syncthreads();
    prefix = sh_prefix;
    rank = sh_rank;
    cnt = sh_cnt;
    mask |= dmask << lo;
    hi = lo - 1;
  }
  // keep every key whose determined bits are below the prefix, and of the
  // keys matching it: all of them when they fill the places left exactly,
  // else (all bits determined: ties) the smallest indices
  const bool all_eq = cnt == rank;
#pragma unroll
  for (int e = 0; e < KPT; ++e) {
    const int j = tid + e * NTH;
    if (j < nb) {
      const unsigned km = key[e] & mask;
      if (km < prefix || (all_eq && km == prefix)) atomicOr(&bits[j >> 5], 1u << (j & 31));
    }
  }
  if (!all_eq && warp == 0) {
    // ties at the threshold key (mask covers every bit): the smallest indices first
    unsigned left = rank;
    for (int j0 = 0; j0 < nb && left > 0; j0 += 32) {
      const int j = j0 + lane;
      const bool eq = j < nb && ~order_key(sc[j]) == prefix;
      const unsigned bal = __ballot_sync(0xffffffffu, eq);
      const unsigned before = __popc(bal & ((1u << lane) - 1u));
      if (eq && before < left) atomicOr(&bits[j >> 5], 1u << (j & 31));
      const unsigned n = __popc(bal);
      left = n >= left ? 0u : left - n;
    }
  }
  __syncthreads();
  if (warp == 0) {
    int base = 0;
    for (int x0 = 0; x0 < nwords; x0 += 32) {
      const int x = x0 + lane;
      const uint32_t word = x < nwords ? bits[x] : 0u;
      const int cnt_w = __popc(word);
      int pre = cnt_w;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, pre, o);
        if (lane >= o) pre += y;
      }
      int pos = base + pre - cnt_w;
      uint32_t m = word;
      while (m) {
        const int bpos = __ffs(m) - 1;
        out[pos++] = x * 32 + bpos;
        m &= m - 1;
      }
      base += __shfl_sync(0xffffffffu, pre, 31);
    }
  }
}

}  // namespace sa
