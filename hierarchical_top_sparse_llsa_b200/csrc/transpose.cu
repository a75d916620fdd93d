// Sparse index transpose (Step 4 of the howistudyai explainer of "Trainable
// Log-linear Sparse Attention for Efficient Diffusion Transformers";
// Building Blocks: Sparse Index Transpose): query-major index lists I(l) to
// key-major CSR lists, by counting, prefix-summing and filling, with no dense
// mask and no global atomics.
//
// One launch covers every level.  A CTA owns (level, b*h, a range of 256 key
// tokens) and walks all index rows of its (level, b, h) twice:
//   pass 1 counts, per warp, the used entries that fall in its key range
//          (warp-private shared-memory histograms) and those below it;
//   scan   turns the counts into row offsets: keys below the range come
//          first, then an exclusive scan over the range, then per-warp bases;
//   pass 2 writes each query token at its key's cursor.  Warps own
//          contiguous query slices in order, rows are walked in order inside
//          a warp, and lanes that share a key in one step are ranked by
//          __match_any_sync, so each key's list comes out ascending.
// The whole result is deterministic.  Entries are screened with the same
// used-entry rule as the attention kernels.

#include "llsa_internal.cuh"

namespace llsa {

namespace {

constexpr int kTrWarps = 16;
constexpr int kTrRange = 256;
constexpr int kBatch = 8;  // row steps whose index loads are in flight together

__global__ void __launch_bounds__(kTrWarps * 32)
transpose_kernel(TransposeParams p) {
  __shared__ int hist[kTrWarps][kTrRange];
  __shared__ int below[kTrWarps];
  __shared__ int scan_buf[kTrRange];
  __shared__ int below_total;

  // which level this CTA works on
  int lvl = 0;
  while (lvl + 1 < p.nlev && (int)blockIdx.x >= p.lv[lvl + 1].cta_begin) ++lvl;
  const TransposeLevel L = p.lv[lvl];
  const int local = blockIdx.x - L.cta_begin;
  const int bh = local / L.ranges;
  const int c0 = (local % L.ranges) * kTrRange;
  const int c1 = min(L.n, c0 + kTrRange);
  const int K = p.K;
  const int n = L.n;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  const int32_t* I = L.idx + (size_t)bh * n * K;
  int32_t* row_ptr = L.row_ptr + (size_t)bh * (n + 1);
  int32_t* col = L.col + (size_t)bh * n * K;

  for (int e = threadIdx.x; e < kTrWarps * kTrRange; e += blockDim.x) (&hist[0][0])[e] = 0;
  __syncthreads();

  const int rows_per_step = 32 / K;  // K <= 32
  const int sub = lane / K;
  const bool lane_on = sub < rows_per_step;
  const int slot = lane_on ? lane % K : lane;  // lanes past the last row never feed a row
  const int rpw = (n + kTrWarps - 1) / kTrWarps;  // rows per warp
  const int r_begin = min(n, warp * rpw), r_end = min(n, r_begin + rpw);

  // pass 1: counts (entries of kBatch steps are loaded before any is used,
  // so their latencies overlap)
  int flags = 0, my_below = 0;
  for (int rb = r_begin; rb < r_end; rb += kBatch * rows_per_step) {
    int cb[kBatch];
#pragma unroll
    for (int i = 0; i < kBatch; ++i) {
      const int q = rb + i * rows_per_step + sub;
      cb[i] = (lane_on && q < r_end) ? I[(size_t)q * K + slot] : -1;
    }
#pragma unroll
    for (int i = 0; i < kBatch; ++i) {
      const int q = rb + i * rows_per_step + sub;
      const bool on = lane_on && q < r_end;
      const int c = cb[i];
      const bool u = warp_row_used(c, slot, n, on, flags);
      if (u && c >= c0 && c < c1) atomicAdd(&hist[warp][c - c0], 1);
      if (u && c < c0) ++my_below;
    }
  }
  my_below = __reduce_add_sync(0xffffffffu, my_below);
  if (lane == 0) below[warp] = my_below;
  __syncthreads();

  // scan: offsets of the keys in [c0, c1)
  if (threadIdx.x == 0) {
    int b = 0;
    for (int w = 0; w < kTrWarps; ++w) b += below[w];
    below_total = b;
  }
  if (threadIdx.x < kTrRange) {
    int tot = 0;
    for (int w = 0; w < kTrWarps; ++w) tot += hist[w][threadIdx.x];
    scan_buf[threadIdx.x] = tot;
  }
  __syncthreads();
  // inclusive Hillis-Steele scan over 256 entries
  for (int off = 1; off < kTrRange; off <<= 1) {
    int v = 0;
    if (threadIdx.x < kTrRange && threadIdx.x >= off) v = scan_buf[threadIdx.x - off];
    __syncthreads();
    if (threadIdx.x < kTrRange) scan_buf[threadIdx.x] += v;
    __syncthreads();
  }
  if (threadIdx.x < kTrRange) {
    const int t = threadIdx.x;
    const int c = c0 + t;
    const int excl = (t == 0) ? 0 : scan_buf[t - 1];
    if (c < c1) {
      const int start = below_total + excl;
      row_ptr[c] = start;
      int run = start;
      for (int w = 0; w < kTrWarps; ++w) {
        const int h = hist[w][t];
        hist[w][t] = run;  // becomes warp w's cursor for key c
        run += h;
      }
    }
  }
  const bool last_range = (c1 == n);
  const int total = below_total + scan_buf[kTrRange - 1];
  if (last_range && threadIdx.x == 0) row_ptr[n] = total;
  __syncthreads();
  if (last_range)
    for (int e = total + threadIdx.x; e < n * K; e += blockDim.x) col[e] = -1;

  // pass 2: fill
  int dummy = 0;
  for (int rb = r_begin; rb < r_end; rb += kBatch * rows_per_step) {
    int cb[kBatch];
#pragma unroll
    for (int i = 0; i < kBatch; ++i) {
      const int q = rb + i * rows_per_step + sub;
      cb[i] = (lane_on && q < r_end) ? I[(size_t)q * K + slot] : -1;
    }
#pragma unroll
    for (int i = 0; i < kBatch; ++i) {
      const int q = rb + i * rows_per_step + sub;
      const bool on = lane_on && q < r_end;
      const int c = cb[i];
      const bool u = warp_row_used(c, slot, n, on, dummy);
      const int key = (u && c >= c0 && c < c1) ? c : -2 - lane;  // -2 - lane matches nobody
      const unsigned peers = __match_any_sync(0xffffffffu, key);
      if (key >= 0) {
        const unsigned lower = peers & ((1u << lane) - 1u);
        col[hist[warp][key - c0] + __popc(lower)] = q;
      }
      __syncwarp();
      if (key >= 0 && lane == 31 - __clz(peers)) hist[warp][key - c0] += __popc(peers);
      __syncwarp();
    }
  }
  if (local % L.ranges == 0) {
    flags = __reduce_or_sync(0xffffffffu, flags);
    if (lane == 0) report_status(p.status, flags);
  }
}

}  // namespace

cudaError_t launch_transpose(const TransposeParams& p, cudaStream_t s) {
  const int total = p.lv[p.nlev - 1].cta_begin + p.BH * p.lv[p.nlev - 1].ranges;
  transpose_kernel<<<total, kTrWarps * 32, 0, s>>>(p);
  return cudaGetLastError();
}

}  // namespace llsa
