// Hierarchical compression: mean pooling by 16 per level (Step 1 of the
// howistudyai explainer of "Trainable Log-linear Sparse Attention for
// Efficient Diffusion Transformers"; Building Blocks: Hierarchical
// Compression).
//
// Kernel 1 reads the fine Q, K, V once (16-byte vector loads, every 128-byte
// line fully used) and writes levels 1 and 2.  One CTA owns 256 fine tokens of
// one (b, h, tensor): thread (t1, v) sums the 16 rows of level-1 token t1 for
// one 16-byte vector of channels, left to right in fp32; the 16 level-1 means
// are staged in shared memory and summed again for level 2.  Kernel 2 forms
// levels 3..L from the level below (a few hundred KB at most).
// Every sum runs left to right with one rounding per addition and is then
// scaled by 1/16, so the pyramid is reproducible bit for bit.

#include "llsa_internal.cuh"

namespace llsa {

namespace {

template <typename T, int D>
__global__ void __launch_bounds__(16 * D * sizeof(T) / 16)
pool_l12_kernel(PoolParams p) {
  constexpr int VEC = Vec16<T>::N;
  constexpr int NV = D / VEC;  // vectors per row
  __shared__ float m1[16][D];

  const int tensor = blockIdx.z;
  const int bh = blockIdx.y;
  const int chunk = blockIdx.x;  // 256 fine tokens
  const int t1 = threadIdx.x / NV;
  const int vv = threadIdx.x % NV;
  const int n1 = p.N / kBlock;
  const int g1 = chunk * 16 + t1;  // level-1 token

  const T* x = static_cast<const T*>(p.x[tensor]);
  float acc[VEC];
  if (g1 < n1) {
    const T* row = x + ((size_t)bh * p.N + (size_t)g1 * kBlock) * D + vv * VEC;
    uint4 raw[16];  // all 16 loads in flight before the first add
#pragma unroll
    for (int j = 0; j < 16; ++j) raw[j] = __ldg(reinterpret_cast<const uint4*>(row + (size_t)j * D));
    float r[VEC];
    Vec16<T>::unpack(raw[0], acc);
#pragma unroll
    for (int j = 1; j < 16; ++j) {
      Vec16<T>::unpack(raw[j], r);
#pragma unroll
      for (int e = 0; e < VEC; ++e) acc[e] = __fadd_rn(acc[e], r[e]);
    }
#pragma unroll
    for (int e = 0; e < VEC; ++e) acc[e] = __fmul_rn(acc[e], 0.0625f);
    float* o1 = p.lvl[tensor][1];
    if (o1 != nullptr) {
      float* dst = o1 + ((size_t)bh * n1 + g1) * D + vv * VEC;
#pragma unroll
      for (int e = 0; e < VEC; e += 4)
        *reinterpret_cast<float4*>(dst + e) = make_float4(acc[e], acc[e + 1], acc[e + 2], acc[e + 3]);
    }
#pragma unroll
    for (int e = 0; e < VEC; ++e) m1[t1][vv * VEC + e] = acc[e];
  }
  if (p.L < 2) return;
  __syncthreads();
  // level 2: one level-2 token per CTA (N is a multiple of 256 when L >= 2)
  for (int d = threadIdx.x; d < D; d += blockDim.x) {
    float a = m1[0][d];
#pragma unroll
    for (int t = 1; t < 16; ++t) a = __fadd_rn(a, m1[t][d]);
    p.lvl[tensor][2][((size_t)bh * (p.N >> 8) + chunk) * D + d] = __fmul_rn(a, 0.0625f);
  }
}

// Level l (>= 3) from level l-1, thread per (token, channel).
__global__ void pool_up_kernel(PoolParams p, int l) {
  const int tensor = blockIdx.z;
  const int n_out = p.N >> (4 * l);
  const size_t total = (size_t)p.BH * n_out * p.D;
  const float* in = p.lvl[tensor][l - 1];
  float* out = p.lvl[tensor][l];
  for (size_t e = (size_t)blockIdx.x * blockDim.x + threadIdx.x; e < total;
       e += (size_t)gridDim.x * blockDim.x) {
    const size_t d = e % p.D;
    const size_t tok = e / p.D;  // bh * n_out + t
    const float* src = in + tok * 16 * p.D + d;
    float a = src[0];
#pragma unroll
    for (int j = 1; j < 16; ++j) a = __fadd_rn(a, src[(size_t)j * p.D]);
    out[e] = __fmul_rn(a, 0.0625f);
  }
}

template <typename T, int D>
cudaError_t launch_l12(const PoolParams& p, cudaStream_t s) {
  constexpr int threads = 16 * D * (int)sizeof(T) / 16;
  const int n1 = p.N / kBlock;
  dim3 grid((n1 + 15) / 16, p.BH, p.L >= 2 ? 3 : 2);  // V has no level-1 output
  pool_l12_kernel<T, D><<<grid, threads, 0, s>>>(p);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_pool(const PoolParams& p, int dtype, cudaStream_t s) {
  cudaError_t e;
  if (dtype == LLSA_BF16)
    e = (p.D == 64) ? launch_l12<bf16, 64>(p, s) : launch_l12<bf16, 128>(p, s);
  else
    e = (p.D == 64) ? launch_l12<float, 64>(p, s) : launch_l12<float, 128>(p, s);
  if (e != cudaSuccess) return e;
  return launch_pool_up(p, s);
}

cudaError_t launch_pool_up(const PoolParams& p, cudaStream_t s) {
  cudaError_t e;
  for (int l = 3; l <= p.L; ++l) {
    const size_t total = (size_t)p.BH * (p.N >> (4 * l)) * p.D;
    int blocks = (int)((total + 255) / 256);
    if (blocks > 148 * 8) blocks = 148 * 8;
    pool_up_kernel<<<dim3(blocks, 1, 3), 256, 0, s>>>(p, l);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

}  // namespace llsa
