// Sparse index transpose (Step 4 of the howistudyai explainer of "Trainable
// Log-linear Sparse Attention for Efficient Diffusion Transformers";
// Building Blocks: Sparse Index Transpose): query-major index lists I(l) to
// key-major CSR lists, with no dense mask and no global atomics.
//
// A stable counting sort of the (key, query) pairs by key, in four launches
// that each cover every level.  The query rows of a (level, b, h) are cut
// into nchunk chunks of consecutive rows; the workspace holds one count per
// (chunk, key).
//   count   one CTA per chunk: shared-memory histogram of the chunk's used
//           entries, written out as that chunk's row of counts;
//   prefix  one CTA per 1024 keys: per key, the running sum over chunks (in
//           place: each count becomes the chunk's first slot relative to the
//           key's list) and the key's total, parked in row_ptr;
//   scan    one CTA per (level, b, h): the exclusive scan of the totals into
//           row_ptr, and -1 in the unused tail of col;
//   fill    one CTA per chunk: the cursors row_ptr[c] + first slot are staged
//           in shared memory, then the chunk's rows go in super-steps of 32
//           consecutive rows spread over the CTA's warps: each row holding
//           key c sets its bit in c's row mask (order-free), and after a
//           barrier each entry's slot is c's cursor plus the number of lower
//           bits, the highest bit's entry advancing the cursor.
// Chunks are filled in row order from the slots the prefix gave them, so
// every key's list comes out ascending and the result is deterministic.
// Entries are screened with the same used-entry rule as the attention
// kernels; the count launch reports the status bits.

#include "llsa_internal.cuh"

namespace llsa {

namespace {

constexpr int kCountThreads = 256;
constexpr int kPrefixThreads = 256;
constexpr int kPrefixKeys = 4 * kPrefixThreads;  // keys per prefix CTA
constexpr int kScanThreads = 1024;
constexpr int kFillThreads = 256;  // 8 warps: each fills whole rows of a super-step
constexpr int kSuperRows = 32;     // rows per fill super-step (one bit each in a key's row mask)
constexpr int kMaxChunks = 128;    // row chunks per (level, b, h); see transpose_chunking
constexpr int kRangeKeys = 8192;   // keys per shared-memory histogram / cursor range
constexpr int kBatch = 8;          // row steps whose index loads are in flight together

enum Grid { kChunkGrid, kTileGrid, kScanGrid };

__device__ __forceinline__ int grid_begin(const TransposeLevel& t, Grid g) {
  return g == kChunkGrid ? t.cta_begin : (g == kTileGrid ? t.tile_begin : t.scan_begin);
}

__device__ __forceinline__ int level_of(const TransposeParams& p, int blk, Grid g) {
  int lvl = 0;
  while (lvl + 1 < p.nlev && blk >= grid_begin(p.lv[lvl + 1], g)) ++lvl;
  return lvl;
}

// How one warp lays index rows across its lanes: rows_per_step rows of K
// slots side by side; lanes past the last full row stay idle.
struct RowLanes {
  int rows_per_step, sub, slot;
  bool on;
  __device__ __forceinline__ RowLanes(int K, int lane) {
    rows_per_step = 32 / K;  // K <= 32
    sub = lane / K;
    on = sub < rows_per_step;
    slot = on ? lane % K : lane;  // idle lanes never feed a row
  }
};

__global__ void __launch_bounds__(kCountThreads)
tr_count_kernel(TransposeParams p) {
  __shared__ int hist[kRangeKeys];
  const TransposeLevel L = p.lv[level_of(p, blockIdx.x, kChunkGrid)];
  const int local = blockIdx.x - L.cta_begin;
  const int bh = local / L.nchunk, ch = local % L.nchunk;
  const int n = L.n, K = L.K;
  const int r0 = ch * L.rows, r1 = min(n, r0 + L.rows);
  const int32_t* I = L.idx + (size_t)bh * n * K;
  int32_t* cnt = L.cnt + ((size_t)bh * L.nchunk + ch) * n;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const RowLanes rl(K, lane);
  const int stride = (kCountThreads / 32) * rl.rows_per_step * kBatch;

  int flags = 0;
  for (int k0 = 0; k0 < n; k0 += kRangeKeys) {
    const int k1 = min(n, k0 + kRangeKeys);
    for (int e = threadIdx.x; e < k1 - k0; e += blockDim.x) hist[e] = 0;
    __syncthreads();
    for (int rb = r0 + warp * rl.rows_per_step * kBatch; rb < r1; rb += stride) {
      int cb[kBatch];
#pragma unroll
      for (int i = 0; i < kBatch; ++i) {
        const int q = rb + i * rl.rows_per_step + rl.sub;
        cb[i] = (rl.on && q < r1) ? I[(size_t)q * K + rl.slot] : -1;
      }
#pragma unroll
      for (int i = 0; i < kBatch; ++i) {
        const int q = rb + i * rl.rows_per_step + rl.sub;
        const int c = cb[i];
        const bool u = warp_row_used(c, rl.slot, n, rl.on && q < r1, flags, K);
        if (u && c >= k0 && c < k1) atomicAdd(&hist[c - k0], 1);
      }
    }
    __syncthreads();
    for (int e = threadIdx.x; e < k1 - k0; e += blockDim.x) cnt[k0 + e] = hist[e];
    __syncthreads();
  }
  flags = __reduce_or_sync(0xffffffffu, flags);
  if (lane == 0) report_status(p.status, flags);
}

__global__ void __launch_bounds__(kPrefixThreads)
tr_prefix_kernel(TransposeParams p) {
  const TransposeLevel L = p.lv[level_of(p, blockIdx.x, kTileGrid)];
  const int n = L.n, nch = L.nchunk;
  const int tiles = (n + kPrefixKeys - 1) / kPrefixKeys;
  const int local = blockIdx.x - L.tile_begin;
  const int bh = local / tiles;
  const int c0 = (local % tiles) * kPrefixKeys + 4 * threadIdx.x;
  if (c0 >= n) return;
  int32_t* cnt = L.cnt + (size_t)bh * nch * n;
  int32_t* tot = L.row_ptr + (size_t)bh * (n + 1);
  if ((n & 3) == 0) {
    // four keys per thread as one int4; 8 chunks' loads in flight at a time
    int4 run = make_int4(0, 0, 0, 0);
    for (int ch0 = 0; ch0 < nch; ch0 += 8) {
      int4 v[8];
#pragma unroll
      for (int i = 0; i < 8; ++i)
        if (ch0 + i < nch) v[i] = *reinterpret_cast<const int4*>(cnt + (size_t)(ch0 + i) * n + c0);
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        if (ch0 + i < nch) {
          *reinterpret_cast<int4*>(cnt + (size_t)(ch0 + i) * n + c0) = run;
          run.x += v[i].x;
          run.y += v[i].y;
          run.z += v[i].z;
          run.w += v[i].w;
        }
      }
    }
    tot[c0] = run.x;
    tot[c0 + 1] = run.y;
    tot[c0 + 2] = run.z;
    tot[c0 + 3] = run.w;
  } else {
    for (int j = 0; j < 4 && c0 + j < n; ++j) {
      int run = 0;
      for (int ch = 0; ch < nch; ++ch) {
        int32_t* a = cnt + (size_t)ch * n + c0 + j;
        const int v = *a;
        *a = run;
        run += v;
      }
      tot[c0 + j] = run;
    }
  }
}

__global__ void __launch_bounds__(kScanThreads)
tr_scan_kernel(TransposeParams p) {
  __shared__ int warp_tot[kScanThreads / 32];
  const TransposeLevel L = p.lv[level_of(p, blockIdx.x, kScanGrid)];
  const int bh = blockIdx.x - L.scan_begin;
  const int n = L.n, K = L.K;
  int32_t* row_ptr = L.row_ptr + (size_t)bh * (n + 1);
  int32_t* col = L.col + (size_t)bh * n * K;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  int carry = 0;  // entries of the keys before this tile
  for (int t0 = 0; t0 < n; t0 += 4 * kScanThreads) {
    const int c0 = t0 + 4 * threadIdx.x;
    int tot[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) tot[j] = (c0 + j < n) ? row_ptr[c0 + j] : 0;
    const int mine = tot[0] + tot[1] + tot[2] + tot[3];
    int incl = mine;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    if (lane == 31) warp_tot[warp] = incl;
    __syncthreads();
    int before = 0, tile_total = 0;
    for (int w = 0; w < kScanThreads / 32; ++w) {
      const int x = warp_tot[w];
      if (w < warp) before += x;
      tile_total += x;
    }
    int run = carry + before + incl - mine;  // first slot of key c0
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      if (c0 + j < n) row_ptr[c0 + j] = run;
      run += tot[j];
    }
    carry += tile_total;
    __syncthreads();  // warp_tot is rewritten by the next tile
  }
  if (threadIdx.x == 0) row_ptr[n] = carry;
  for (int e = carry + threadIdx.x; e < n * K; e += blockDim.x) col[e] = -1;
}

__global__ void __launch_bounds__(kFillThreads)
tr_fill_kernel(TransposeParams p) {
  // cur[e]: next free slot of key k0 + e; rowmask[e]: which rows of the
  // current super-step hold key k0 + e (bit b = row R0 + b)
  extern __shared__ int fill_smem[];
  int* cur = fill_smem;
  unsigned* rowmask = reinterpret_cast<unsigned*>(fill_smem + kRangeKeys);
  const TransposeLevel L = p.lv[level_of(p, blockIdx.x, kChunkGrid)];
  const int local = blockIdx.x - L.cta_begin;
  const int bh = local / L.nchunk, ch = local % L.nchunk;
  const int n = L.n, K = L.K;
  const int r0 = ch * L.rows, r1 = min(n, r0 + L.rows);
  const int32_t* I = L.idx + (size_t)bh * n * K;
  const int32_t* start = L.cnt + ((size_t)bh * L.nchunk + ch) * n;
  const int32_t* row_ptr = L.row_ptr + (size_t)bh * (n + 1);
  int32_t* col = L.col + (size_t)bh * n * K;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const RowLanes rl(K, lane);
  // a super-step is kSuperRows consecutive rows, rows_per_step per warp
  const int warp_rows = rl.rows_per_step;
  const int active_warps = min(kFillThreads / 32, kSuperRows / warp_rows);
  const int super_rows = active_warps * warp_rows;

  for (int k0 = 0; k0 < n; k0 += kRangeKeys) {
    const int len = min(n, k0 + kRangeKeys) - k0;
    // cursors: the key's first slot plus this chunk's offset in its list,
    // 8 pairs of loads in flight per thread; masks cleared
    for (int e0 = threadIdx.x; e0 < len; e0 += 8 * kFillThreads) {
      int t[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int e = e0 + i * kFillThreads;
        t[i] = (e < len) ? start[k0 + e] + row_ptr[k0 + e] : 0;
      }
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int e = e0 + i * kFillThreads;
        if (e < len) {
          cur[e] = t[i];
          rowmask[e] = 0u;
        }
      }
    }
    __syncthreads();
    // this lane's entry is row R0 + b of each super-step; the next
    // super-step's entry is loaded while the current one is placed
    const int b = warp * warp_rows + rl.sub;
    auto entry = [&](int R0) {
      const int q = R0 + b;
      return (warp < active_warps && rl.on && q < r1) ? I[(size_t)q * K + rl.slot] : -1;
    };
    int c_next = entry(r0);
    for (int R0 = r0; R0 < r1; R0 += super_rows) {
      const int q = R0 + b;
      const bool row_on = warp < active_warps && rl.on && q < r1;
      const int c = c_next;
      if (R0 + super_rows < r1) c_next = entry(R0 + super_rows);
      int dummy = 0;
      const bool u = warp_row_used(c, rl.slot, n, row_on, dummy, K);
      const int key = (u && c >= k0 && c < k0 + len) ? c - k0 : -1;
      // 1. every row that holds a key marks its bit (order-free)
      if (key >= 0) atomicOr(&rowmask[key], 1u << b);
      __syncthreads();
      // 2. slot = cursor + the rows before this one in the super-step that
      //    hold the key; the last such row advances the cursor after all reads
      bool last = false;
      unsigned m = 0u;
      if (key >= 0) {
        m = rowmask[key];
        col[cur[key] + __popc(m & ((1u << b) - 1u))] = q;
        last = (31 - __clz(m)) == b;
      }
      __syncthreads();
      if (last) {
        cur[key] += __popc(m);
        rowmask[key] = 0u;
      }
      __syncthreads();
    }
  }
}

}  // namespace

// Rows per chunk for a level of n query rows: 128 rows per chunk (one warp
// fills a chunk in row order, so the chunk length bounds the fill's critical
// path), at most kMaxChunks chunks (the workspace holds nchunk * n counts per
// (b, h)).
void transpose_chunking(int n, int* nchunk, int* rows) {
  int c = (n + 127) / 128;
  if (c > kMaxChunks) c = kMaxChunks;
  if (c < 1) c = 1;
  *rows = (n + c - 1) / c;
  *nchunk = (n + *rows - 1) / *rows;
}

cudaError_t launch_transpose(const TransposeParams& p, cudaStream_t s) {
  const TransposeLevel& last = p.lv[p.nlev - 1];
  const int chunks = last.cta_begin + p.BH * last.nchunk;
  const int tiles = last.tile_begin + p.BH * ((last.n + kPrefixKeys - 1) / kPrefixKeys);
  const int scans = last.scan_begin + p.BH;
  tr_count_kernel<<<chunks, kCountThreads, 0, s>>>(p);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  tr_prefix_kernel<<<tiles, kPrefixThreads, 0, s>>>(p);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  tr_scan_kernel<<<scans, kScanThreads, 0, s>>>(p);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const size_t fill_smem = (size_t)kRangeKeys * (sizeof(int) + sizeof(unsigned));
  e = cudaFuncSetAttribute(tr_fill_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)fill_smem);
  if (e != cudaSuccess) return e;
  tr_fill_kernel<<<chunks, kFillThreads, fill_smem, s>>>(p);
  return cudaGetLastError();
}

int transpose_prefix_tiles(int n) { return (n + kPrefixKeys - 1) / kPrefixKeys; }

}  // namespace llsa
