// Internal helpers shared by the LLSA CUDA kernels (not part of the C ABI).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "llsa.h"

namespace llsa {

typedef __nv_bfloat16 bf16;

constexpr int kBlock = LLSA_BLOCK;  // tokens per block, pooling factor
constexpr int kMaxL = LLSA_MAX_LEVELS;
constexpr int kMaxK = LLSA_MAX_TOPK;

// ------------------------------------------------------------ conversions
__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ float to_f32(bf16 x) { return __bfloat162float(x); }
__device__ __forceinline__ void store_elem(float* p, float v) { *p = v; }
__device__ __forceinline__ void store_elem(bf16* p, float v) { *p = __float2bfloat16_rn(v); }

// 16-byte vector of T loaded as floats.
template <typename T>
struct Vec16;

template <>
struct Vec16<float> {
  static constexpr int N = 4;
  __device__ __forceinline__ static void unpack(uint4 u, float* o) {
    o[0] = __uint_as_float(u.x); o[1] = __uint_as_float(u.y);
    o[2] = __uint_as_float(u.z); o[3] = __uint_as_float(u.w);
  }
  __device__ __forceinline__ static void load(const float* p, float* o) {
    unpack(__ldg(reinterpret_cast<const uint4*>(p)), o);
  }
};

template <>
struct Vec16<bf16> {
  static constexpr int N = 8;
  // bf16 -> fp32 is exact: the bf16 bits are the high half of the fp32 bits
  __device__ __forceinline__ static void unpack(uint4 u, float* o) {
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      o[2 * i] = __uint_as_float(w[i] << 16);
      o[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
    }
  }
  __device__ __forceinline__ static void load(const bf16* p, float* o) {
    unpack(__ldg(reinterpret_cast<const uint4*>(p)), o);
  }
};

// --------------------------------------------------- index-row entry rule
// An entry v of a row of I(l) is used iff 0 <= v < n and v is larger than the
// last used entry.  Anything else is skipped; -1 is padding, other values
// outside [0, n) are bad, and skipped in-range values or a valid entry after a
// pad are non-canonical.  Every kernel that reads index rows applies exactly
// this rule, so forward, transpose and backward see the same key sets.
struct RowRule {
  int last = -1;
  bool seen_pad = false;
  int flags = 0;
  __device__ __forceinline__ bool use(int v, int n) {
    if (v == -1) { seen_pad = true; return false; }
    if (v < -1 || v >= n) { flags |= LLSA_DEV_BAD_INDEX; return false; }
    if (v <= last) { flags |= LLSA_DEV_NONCANONICAL; return false; }
    if (seen_pad) flags |= LLSA_DEV_NONCANONICAL;
    last = v;
    return true;
  }
};

// The same rule for rows laid side by side across a warp: this lane holds
// entry `slot` of a row whose entry 0 sits `slot` lanes lower; `on` is false
// for lanes outside every row (their results are ignored and they are never
// read by lanes inside a row).  Segmented shuffle scans give, for each entry,
// the largest in-range entry before it and whether a pad came before it.
// Must be called by all 32 lanes; seg, the same on every lane, is at least
// the row length (the scans stop once they span that many slots).
__device__ __forceinline__ bool warp_row_used(int v, int slot, int n, bool on, int& flags, int seg = 32) {
  const bool inr = on && v >= 0 && v < n;
  int mx = inr ? v : -1;
  int pad = (on && v == -1) ? 1 : 0;
#pragma unroll
  for (int o = 1; o < seg; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, mx, o);
    const int z = __shfl_up_sync(0xffffffffu, pad, o);
    if (slot >= o) {
      mx = max(mx, y);
      pad |= z;
    }
  }
  int mx_before = __shfl_up_sync(0xffffffffu, mx, 1);
  int pad_before = __shfl_up_sync(0xffffffffu, pad, 1);
  if (slot < 1) {
    mx_before = -1;
    pad_before = 0;
  }
  const bool used = inr && v > mx_before;
  if (on) {
    if (v < -1 || v >= n) flags |= LLSA_DEV_BAD_INDEX;
    else if (inr && !used) flags |= LLSA_DEV_NONCANONICAL;
    else if (used && pad_before) flags |= LLSA_DEV_NONCANONICAL;
  }
  return used;
}

__device__ __forceinline__ void report_status(int32_t* st, int flags) {
  if (st != nullptr && flags != 0) atomicOr(st, flags);
}

// --------------------------------------------------------- launch params
struct PoolParams {
  const void* x[3];          // q, k, v fine tensors
  float* lvl[3][kMaxL + 1];  // [tensor][level] outputs (V level 1 unused)
  int BH, N, D, L;
};

struct SelectParams {
  const float* ql;       // Q(l) [BH, n, D]
  const float* kl;       // K(l) [BH, n, D]
  const int32_t* parent; // I(l+1) [BH, n/16, Kp] or nullptr at level L
  int32_t* out;          // I(l) [BH, n, K]
  int n;                 // N_l
  int K;                 // K_l, kept keys per row at this level
  int Kp;                // K_{l+1}, the parent row's width
};

struct TransposeLevel {
  const int32_t* idx;
  int32_t* row_ptr;
  int32_t* col;
  int32_t* cnt;    // workspace [BH][nchunk][n]: per-chunk key counts, then cursors
  int n;           // N_l (queries == keys at level l)
  int K;           // K_l, the width of an index row
  int nchunk;      // row chunks per (b, h)
  int rows;        // rows per chunk
  int cta_begin;   // first CTA of this level in the count and fill grids
  int tile_begin;  // first CTA of this level in the chunk-prefix grid
  int scan_begin;  // first CTA of this level in the row_ptr scan grid
};

struct TransposeParams {
  TransposeLevel lv[kMaxL];
  int nlev;
  int BH;
  int32_t* status;
};

struct AttnParams {
  const void* q;
  const void* k;
  const void* v;
  const void* o;
  const void* dout;
  const float* lse_in;
  const float* pk[kMaxL + 1];  // coarse keys, levels 2..L
  const float* pv[kMaxL + 1];
  const int32_t* idx[kMaxL + 1];
  const int32_t* row_ptr[kMaxL + 1];
  const int32_t* col[kMaxL + 1];
  float logw[kMaxL + 1];  // ln of the level weights (0 for weight 1)
  void* out;              // O (fwd)
  void* o_res;            // bf16 rounding residual of O: written by the fwd, read by the bwd (null: none)
  float* lse;             // LSE (fwd)
  void* dq;
  void* dk;
  void* dv;
  float* delta;                 // [BH, N]
  float* part[kMaxL + 1];       // [BH, N/128, K_l, 2, D] per coarse level (groups of 8 query blocks)
  float* coarse[kMaxL + 1];     // [BH, N_l, 2, D] per coarse level
  int32_t* work;                // pass-3 work counter (zeroed by pass 1)
  int32_t* status;
  int B, H, N, D, L, K;  // L: top key level (Lc); K = K_1, the fine blocks per query block
  int Kl[kMaxL + 1];      // K_l, the width of I(l) (Kl[1] == K)
  int Kc;                 // coarse keys per query block at most: sum of K_l, l = 2..L
  float scale;
};

// ------------------------------------------------------ kernel launchers
// Each returns cudaSuccess or the launch error.
cudaError_t launch_pool(const PoolParams& p, int dtype, cudaStream_t s);
cudaError_t launch_pool_up(const PoolParams& p, cudaStream_t s);  // levels 3..L from level 2
cudaError_t launch_select_level(const SelectParams& p, int BH, int D, cudaStream_t s);
cudaError_t launch_transpose(const TransposeParams& p, cudaStream_t s);
void transpose_chunking(int n, int* nchunk, int* rows);
int transpose_prefix_tiles(int n);
cudaError_t launch_coarse_reduce(const AttnParams& p, cudaStream_t s);
cudaError_t launch_reorder(const void* src, void* dst, long long rows, int N, int side_log2, int row_bytes,
                           int to_zorder, cudaStream_t s);

}  // namespace llsa
