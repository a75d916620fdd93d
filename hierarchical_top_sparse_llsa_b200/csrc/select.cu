// Hierarchical Top-K selection (Step 2 of the howistudyai explainer of
// "Trainable Log-linear Sparse Attention for Efficient Diffusion
// Transformers"; Building Blocks: Hierarchical Top-K Selection).
//
// One launch per level, coarsest first.  A CTA owns the 16 sibling query
// tokens under one parent (level l < L), or 16 consecutive query tokens at
// the top level, so they share one candidate list: the children of the keys
// their parent kept, or every top-level key.  Query rows and candidate K(l)
// rows (in chunks of 128) are staged transposed in shared memory, and each
// thread scores a 4 x 4 block of (query, candidate) pairs, so a candidate row
// is read from shared memory 4 times rather than 16.
//
// Score: fp32, d = 0..D-1 left to right, one rounding per multiply and per
// add (no contraction into FMA), so scores are reproducible bit for bit and
// the selected indices are exact.  The products and sums run as packed pairs
// (sm_100 mul/add .f32x2: each half rounded exactly as the scalar .rn op),
// two candidates per instruction.
// Top-K: each (score, index) pair is packed into one 64-bit key that orders
// by score (with -0 == +0) and then by lower index; K rounds of a warp-wide
// maximum (two redux.sync on 32-bit halves) pick the winners, merging the
// running list of earlier chunks.  Rows are then sorted ascending by index.

#include "select_core.cuh"

namespace llsa {

namespace {

template <int D>
__global__ void __launch_bounds__(kSelThreads)
select_kernel(SelectParams p) {
  extern __shared__ float4 smem4[];
  select_group<D>(p, blockIdx.y, blockIdx.x, reinterpret_cast<float*>(smem4));
}

template <int D>
cudaError_t launch_sel(const SelectParams& p, int BH, cudaStream_t s) {
  static_assert(kSelQ * kSelChunk <= 64 * (kSelChunk + 4), "scores fit over the candidate tile");
  const size_t smem = select_scratch_bytes<D>();
  // set on every call: the attribute is per device and the call is cheap
  cudaError_t e = cudaFuncSetAttribute(select_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(select_kernel<D>, cudaFuncAttributePreferredSharedMemoryCarveout, (int)cudaSharedmemCarveoutMaxShared);
  if (e != cudaSuccess) return e;
  const int groups = (p.parent == nullptr) ? (p.n + kSelQ - 1) / kSelQ : p.n / kBlock;
  select_kernel<D><<<dim3(groups, BH), kSelThreads, smem, s>>>(p);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_select_level(const SelectParams& p, int BH, int D, cudaStream_t s) {
  return (D == 64) ? launch_sel<64>(p, BH, s) : launch_sel<128>(p, BH, s);
}

}  // namespace llsa
