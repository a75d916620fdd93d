// Sparse attention forward with hierarchical KV enrichment and KV
// reweighting, CUDA-core (SIMT) fp32 kernel (Step 3 of the howistudyai
// explainer of "Trainable Log-linear Sparse Attention for Efficient Diffusion
// Transformers").
//
// This kernel serves fp32 inputs, whose 1e-4 accuracy the bf16 tensor-core
// path cannot give.  One CTA (256 threads) owns one 16-token query block;
// 16 threads share a query.  The block's key list (fine tokens of the kept
// level-1 blocks, then the kept coarse tokens of levels 2..L) is walked in
// tiles of 32 keys with an online softmax; a coarse key of level l adds
// ln(w_l) to its score, which multiplies its exponential by w_l.

#include <math.h>

#include "keyset.cuh"

namespace llsa {

namespace {

constexpr int kTile = 32;

template <typename T, int D>
__global__ void __launch_bounds__(256)
attn_fwd_simt_kernel(AttnParams p) {
  constexpr int DPT = D / 16;
  __shared__ KeyList kl;
  __shared__ float qs[16][D + 1];
  __shared__ float ks[kTile][D + 1];
  __shared__ float vs[kTile][D];
  __shared__ float lw[kTile];
  __shared__ float ps[16][kTile];

  const int b = blockIdx.x;
  const int bh = blockIdx.y;
  const int tid = threadIdx.x;
  const int i = tid >> 4, sub = tid & 15;
  const T* Q = static_cast<const T*>(p.q);
  const T* Kf = static_cast<const T*>(p.k);
  const T* Vf = static_cast<const T*>(p.v);

  if (tid < 32) {
    const int f = build_key_list(kl, p, bh, b);
    if (tid == 0) report_status(p.status, f);
  }
  const size_t qrow0 = (size_t)bh * p.N + (size_t)b * kBlock;
  for (int e = tid; e < 16 * D; e += 256) qs[e / D][e % D] = to_f32(Q[qrow0 * D + e]);
  __syncthreads();

  const int nkeys = kl.n;
  float m = -INFINITY, l = 0.f;
  float acc[DPT];
#pragma unroll
  for (int dd = 0; dd < DPT; ++dd) acc[dd] = 0.f;

  for (int t0 = 0; t0 < nkeys; t0 += kTile) {
    const int tn = min(kTile, nkeys - t0);
    for (int e = tid; e < tn * D; e += 256) {
      const int j = e / D, d = e % D;
      const int key = t0 + j;
      const int lv = kl.lvl[key];
      const int tok = kl.tok[key];
      float kv, vv;
      if (lv == 0) {
        const size_t off = ((size_t)bh * p.N + tok) * D + d;
        kv = to_f32(Kf[off]);
        vv = to_f32(Vf[off]);
      } else {
        const size_t off = ((size_t)bh * (p.N >> (4 * lv)) + tok) * D + d;
        kv = p.pk[lv][off];
        vv = p.pv[lv][off];
      }
      ks[j][d] = kv;
      vs[j][d] = vv;
      if (d == 0) lw[j] = (lv == 0) ? 0.f : p.logw[lv];
    }
    __syncthreads();
    float s[2];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int j = sub + 16 * h;
      s[h] = -INFINITY;
      if (j < tn) {
        float a = 0.f;
#pragma unroll 8
        for (int d = 0; d < D; ++d) a = fmaf(qs[i][d], ks[j][d], a);
        s[h] = a * p.scale + lw[j];
      }
    }
    float mx = fmaxf(s[0], s[1]);
#pragma unroll
    for (int o = 8; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    const float m_new = fmaxf(m, mx);
    const float corr = expf(m - m_new);
    const float p0 = expf(s[0] - m_new), p1 = expf(s[1] - m_new);
    float psum = p0 + p1;
#pragma unroll
    for (int o = 8; o > 0; o >>= 1) psum += __shfl_xor_sync(0xffffffffu, psum, o);
    l = l * corr + psum;
    ps[i][sub] = p0;
    ps[i][sub + 16] = p1;
    __syncwarp();
#pragma unroll
    for (int dd = 0; dd < DPT; ++dd) {
      const int d = sub + 16 * dd;
      float a = acc[dd] * corr;
      for (int j = 0; j < tn; ++j) a = fmaf(ps[i][j], vs[j][d], a);
      acc[dd] = a;
    }
    m = m_new;
    __syncthreads();
  }
  T* O = static_cast<T*>(p.out);
  const size_t orow = (qrow0 + i) * D;
  const bool has = l > 0.f;
  const float inv = has ? 1.f / l : 0.f;
#pragma unroll
  for (int dd = 0; dd < DPT; ++dd) store_elem(&O[orow + sub + 16 * dd], acc[dd] * inv);
  if (sub == 0) p.lse[qrow0 + i] = has ? m + logf(l) : -INFINITY;
}

}  // namespace

cudaError_t launch_attn_fwd_simt(const AttnParams& p, int dtype, cudaStream_t s) {
  dim3 grid(p.N / kBlock, p.B * p.H);
  if (dtype == LLSA_BF16) {
    if (p.D == 64) attn_fwd_simt_kernel<bf16, 64><<<grid, 256, 0, s>>>(p);
    else attn_fwd_simt_kernel<bf16, 128><<<grid, 256, 0, s>>>(p);
  } else {
    if (p.D == 64) attn_fwd_simt_kernel<float, 64><<<grid, 256, 0, s>>>(p);
    else attn_fwd_simt_kernel<float, 128><<<grid, 256, 0, s>>>(p);
  }
  return cudaGetLastError();
}

}  // namespace llsa
