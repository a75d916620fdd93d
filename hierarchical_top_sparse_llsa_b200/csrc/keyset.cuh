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
    const int c = (lane < K) ? p.idx[l][((size_t)bh * nl + a) * K + lane] : -1;
    const bool u = warp_row_used(c, lane, nl, lane < K, flags);
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
