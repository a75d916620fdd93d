// Hierarchical Top-K selection (Step 2 of the howistudyai explainer of
// "Trainable Log-linear Sparse Attention for Efficient Diffusion
// Transformers"; Building Blocks: Hierarchical Top-K Selection).
//
// One launch per level, coarsest first.  A CTA owns the 16 sibling query
// tokens under one parent (level l < L), or 16 consecutive query tokens at
// the top level, so they share one candidate list: the children of the keys
// their parent kept, or every top-level key.  Candidate K(l) rows are staged
// in shared memory once per CTA in chunks of 128 and scored by 16 warps, one
// query per warp, one candidate per lane.
//
// Score: fp32, d = 0..D-1 left to right, one rounding per multiply and per
// add (explicit __fmul_rn/__fadd_rn: no contraction into FMA), so scores are
// reproducible bit for bit and the selected indices are exact.
// Top-K: each (score, index) pair is packed into one 64-bit key that orders
// by score (with -0 == +0) and then by lower index; K rounds of a warp-wide
// maximum (two redux.sync on 32-bit halves) pick the winners, merging the
// running list of earlier chunks.  Rows are then sorted ascending by index.

#include "llsa_internal.cuh"

namespace llsa {

namespace {

constexpr int kSelWarps = 16;
constexpr int kSelChunk = 128;
constexpr int kSelItems = kSelChunk / 32;

__device__ __forceinline__ uint64_t pack_key(float s, int idx) {
  s = __fadd_rn(s, 0.0f);  // -0 -> +0, so that equal scores compare equal
  uint32_t b = __float_as_uint(s);
  uint32_t ord = (b & 0x80000000u) ? ~b : (b | 0x80000000u);
  return ((uint64_t)ord << 32) | (uint32_t)(~(uint32_t)idx);
}

__device__ __forceinline__ uint64_t warp_max_u64(uint64_t x) {
  const uint32_t hi = __reduce_max_sync(0xffffffffu, (uint32_t)(x >> 32));
  const uint32_t lo_c = ((uint32_t)(x >> 32) == hi) ? (uint32_t)x : 0u;
  const uint32_t lo = __reduce_max_sync(0xffffffffu, lo_c);
  return ((uint64_t)hi << 32) | lo;
}

template <int D>
__global__ void __launch_bounds__(kSelWarps * 32)
select_kernel(SelectParams p) {
  constexpr int LD = D + 4;  // row stride (floats): conflict-free 16-byte loads
  extern __shared__ float4 smem4[];
  float* qs = reinterpret_cast<float*>(smem4);     // [16][LD]
  float* ks = qs + kSelWarps * LD;                 // [kSelChunk][LD]
  int* cid = reinterpret_cast<int*>(ks + kSelChunk * LD);  // [kSelChunk]
  __shared__ int parents[kMaxK];
  __shared__ int n_par;

  const int bh = blockIdx.y;
  const int grp = blockIdx.x;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int n = p.n;
  const int K = p.K;
  const bool top = (p.parent == nullptr);

  if (threadIdx.x == 0) {
    int m = 0;
    if (!top) {
      RowRule rr;
      const int32_t* prow = p.parent + ((size_t)bh * (n / kBlock) + grp) * K;
      for (int s = 0; s < K; ++s) {
        const int c = prow[s];
        if (rr.use(c, n / kBlock)) parents[m++] = c;
      }
    }
    n_par = m;
  }
  // the 16 query rows
  const float* qbase = p.ql + ((size_t)bh * n + (size_t)grp * kSelWarps) * D;
  for (int e = threadIdx.x; e < kSelWarps * (D / 4); e += blockDim.x) {
    const int r = e / (D / 4), c4 = e % (D / 4);
    float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
    if (grp * kSelWarps + r < n) v = *reinterpret_cast<const float4*>(qbase + (size_t)r * D + c4 * 4);
    *reinterpret_cast<float4*>(qs + r * LD + c4 * 4) = v;
  }
  __syncthreads();
  const int C = top ? n : n_par * kBlock;
  const int q = grp * kSelWarps + warp;

  uint64_t run = 0;  // lane r < K holds the r-th best so far (0 = none)
  const float* kbase = p.kl + (size_t)bh * n * D;
  for (int c0 = 0; c0 < C; c0 += kSelChunk) {
    const int cn = min(kSelChunk, C - c0);
    __syncthreads();
    for (int e = threadIdx.x; e < cn * (D / 4); e += blockDim.x) {
      const int r = e / (D / 4), c4 = e % (D / 4);
      const int j = c0 + r;
      const int c = top ? j : parents[j / kBlock] * kBlock + (j % kBlock);
      *reinterpret_cast<float4*>(ks + r * LD + c4 * 4) =
          *reinterpret_cast<const float4*>(kbase + (size_t)c * D + c4 * 4);
      if (c4 == 0) cid[r] = c;
    }
    __syncthreads();
    uint64_t item[kSelItems + 1];
#pragma unroll
    for (int it = 0; it < kSelItems; ++it) {
      const int j = lane + 32 * it;
      item[it] = 0;
      if (j < cn) {
        const float* qr = qs + warp * LD;
        const float* kr = ks + j * LD;
        float s = 0.f;
#pragma unroll
        for (int d = 0; d < D; d += 4) {
          const float4 a = *reinterpret_cast<const float4*>(qr + d);
          const float4 b = *reinterpret_cast<const float4*>(kr + d);
          s = (d == 0) ? __fmul_rn(a.x, b.x) : __fadd_rn(s, __fmul_rn(a.x, b.x));
          s = __fadd_rn(s, __fmul_rn(a.y, b.y));
          s = __fadd_rn(s, __fmul_rn(a.z, b.z));
          s = __fadd_rn(s, __fmul_rn(a.w, b.w));
        }
        item[it] = pack_key(s, cid[j]);
      }
    }
    item[kSelItems] = (lane < K) ? run : 0;
    uint64_t next = 0;
    for (int r = 0; r < K; ++r) {
      uint64_t mine = 0;
      int arg = 0;
#pragma unroll
      for (int it = 0; it <= kSelItems; ++it)
        if (item[it] > mine) { mine = item[it]; arg = it; }
      const uint64_t best = warp_max_u64(mine);
      if (best == 0) break;  // uniform: no candidates left
      if (mine == best) {
#pragma unroll
        for (int it = 0; it <= kSelItems; ++it)
          if (it == arg) item[it] = 0;
      }
      if (lane == r) next = best;
    }
    run = next;
  }
  if (q >= n) return;
  // ascending index order; the kept entries are lanes 0..cnt-1
  const bool valid = (lane < K) && (run != 0);
  const int id = valid ? (int)(~(uint32_t)run) : 0x7fffffff;
  int pos = 0;
  for (int r = 0; r < K; ++r) {
    const int other = __shfl_sync(0xffffffffu, id, r);
    pos += (other < id) ? 1 : 0;
  }
  if (lane < K) {
    int32_t* orow = p.out + ((size_t)bh * n + q) * K;
    if (valid) orow[pos] = id;
    else orow[lane] = -1;  // unfilled rounds are the last K - cnt lanes
  }
}

template <int D>
cudaError_t launch_sel(const SelectParams& p, int BH, cudaStream_t s) {
  constexpr int LD = D + 4;
  const size_t smem = (size_t)(kSelWarps + kSelChunk) * LD * sizeof(float) + kSelChunk * sizeof(int);
  // set on every call: the attribute is per device and the call is cheap
  cudaError_t e = cudaFuncSetAttribute(select_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const int groups = (p.parent == nullptr) ? (p.n + kSelWarps - 1) / kSelWarps : p.n / kBlock;
  select_kernel<D><<<dim3(groups, BH), kSelWarps * 32, smem, s>>>(p);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_select_level(const SelectParams& p, int BH, int D, cudaStream_t s) {
  return (D == 64) ? launch_sel<64>(p, BH, s) : launch_sel<128>(p, BH, s);
}

}  // namespace llsa
