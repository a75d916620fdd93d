// Key set of one 16-token query block under hierarchical KV enrichment
// (Step 3 of the howistudyai explainer of "Trainable Log-linear Sparse
// Attention for Efficient Diffusion Transformers"): the 16 fine tokens of
// each block kept in I(1)[b], then for l = 2..L the pooled tokens kept in
// I(l)[b >> 4(l-1)].  Built by warp 0 of the CTA into shared memory.
#pragma once

#include "llsa_internal.cuh"

namespace llsa {

constexpr int kMaxKeys = kBlock * kMaxK + (kMaxL - 1) * kMaxK;  // 672

struct KeyList {
  int n;                   // number of keys
  int nfine;               // the first nfine keys are fine tokens
  int tok[kMaxKeys];       // fine token index, or coarse token index at its level
  signed char lvl[kMaxKeys];   // 0 fine, l >= 2 coarse
  signed char slot[kMaxKeys];  // coarse: position in its index row
};

// Must be called by all 32 lanes of one warp; returns the status flags seen
// (lane 0's copy is complete).  `b` is the level-1 block (query block).
__device__ __forceinline__ int build_key_list(KeyList& kl, const AttnParams& p, int bh, int b) {
  const int lane = threadIdx.x & 31;
  const int K = p.K;
  int flags = 0;
  int n = 0;
  {
    const int n1 = p.N / kBlock;
    const int c = (lane < K) ? p.idx[1][((size_t)bh * n1 + b) * K + lane] : -1;
    const bool u = warp_row_used(c, lane, n1, lane < K, flags);
    const unsigned m = __ballot_sync(0xffffffffu, u);
    if (u) {
      const int pos = __popc(m & ((1u << lane) - 1u)) * kBlock;
      for (int j = 0; j < kBlock; ++j) {
        kl.tok[pos + j] = c * kBlock + j;
        kl.lvl[pos + j] = 0;
        kl.slot[pos + j] = (signed char)lane;
      }
    }
    n = __popc(m) * kBlock;
  }
  const int nfine = n;
  for (int l = 2; l <= p.L; ++l) {
    const int nl = p.N >> (4 * l);
    const int a = b >> (4 * (l - 1));
    const int Kl = p.Kl[l];
    const int c = (lane < Kl) ? p.idx[l][((size_t)bh * nl + a) * Kl + lane] : -1;
    const bool u = warp_row_used(c, lane, nl, lane < Kl, flags);
    const unsigned m = __ballot_sync(0xffffffffu, u);
    if (u) {
      const int pos = n + __popc(m & ((1u << lane) - 1u));
      kl.tok[pos] = c;
      kl.lvl[pos] = (signed char)l;
      kl.slot[pos] = (signed char)lane;
    }
    n += __popc(m);
  }
  if (lane == 0) {
    kl.n = n;
    kl.nfine = nfine;
  }
  return __reduce_or_sync(0xffffffffu, flags);
}

}  // namespace llsa

namespace llsa {

// Ascending bitonic sort of 32*E ints held by one warp, element i = lane + 32*e
// in v[e] (E a power of two).  All 32 lanes must call it.
template <int E>
__device__ __forceinline__ void warp_bitonic_sort(int (&v)[E], int lane) {
  constexpr int n = 32 * E;
#pragma unroll
  for (int k = 2; k <= n; k <<= 1) {
#pragma unroll
    for (int j = k >> 1; j > 0; j >>= 1) {
      if (j < 32) {
#pragma unroll
        for (int e = 0; e < E; ++e) {
          const int i = lane + 32 * e;
          const int other = __shfl_xor_sync(0xffffffffu, v[e], j);
          const bool lower = (lane & j) == 0;
          const bool asc = (i & k) == 0;
          v[e] = (asc == lower) ? min(v[e], other) : max(v[e], other);
        }
      } else {
        const int je = j / 32;
#pragma unroll
        for (int e = 0; e < E; ++e) {
          if ((e & je) == 0) {
            const int i = lane + 32 * e;
            const bool asc = (i & k) == 0;
            const int a = v[e], b = v[e + je];
            v[e] = asc ? min(a, b) : max(a, b);
            v[e + je] = asc ? max(a, b) : min(a, b);
          }
        }
      }
    }
  }
}

// Sorted, de-duplicated union of `cnt` entries in[0..cnt) (cnt <= 32*E) into
// out[0..u); returns u.  One warp; entries >= 0x7fffffff are ignored.
template <int E>
__device__ __forceinline__ int warp_sorted_union(const int* in, int cnt, int* out, int lane) {
  int v[E];
#pragma unroll
  for (int e = 0; e < E; ++e) {
    const int i = lane + 32 * e;
    v[e] = (i < cnt) ? in[i] : 0x7fffffff;
  }
  warp_bitonic_sort<E>(v, lane);
  int base = 0;
  int prev_last = -1;  // last element of the previous column (e - 1), lane 31
#pragma unroll
  for (int e = 0; e < E; ++e) {
    int prev = __shfl_up_sync(0xffffffffu, v[e], 1);
    if (lane == 0) prev = prev_last;
    const bool first = v[e] != 0x7fffffff && v[e] != prev;
    const unsigned m = __ballot_sync(0xffffffffu, first);
    if (first) out[base + __popc(m & ((1u << lane) - 1u))] = v[e];
    base += __popc(m);
    prev_last = __shfl_sync(0xffffffffu, v[e], 31);
  }
  return base;
}

// Position of `x` in the sorted array a[0..n) (x must be present).
__device__ __forceinline__ int sorted_find(const int* a, int n, int x) {
  int lo = 0, hi = n - 1;
  while (lo < hi) {
    const int mid = (lo + hi) >> 1;
    if (a[mid] < x) lo = mid + 1;
    else hi = mid;
  }
  return lo;
}

}  // namespace llsa
