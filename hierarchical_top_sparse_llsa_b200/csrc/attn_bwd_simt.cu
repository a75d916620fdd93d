// Backward of the enriched sparse attention, CUDA-core (SIMT) fp32 kernels
// (the key-major backward of Step 4 of the howistudyai explainer of
// "Trainable Log-linear Sparse Attention for Efficient Diffusion
// Transformers"; Building Blocks: Sparse Index Transpose).
//
// Three launches, no global atomics, every sum in a fixed order:
//   1. query-major: one CTA per 8 consecutive query blocks (they share every
//      coarse key set; one CTA per block when L = 1).  It forms
//      Delta_i = sum_j P_ij dP_ij (equal to dO_i . O_i, but taken from the
//      unrounded terms: O itself is stored rounded to its dtype), dQ, and the
//      coarse-key partials
//      sum_i dS_ij q_i and sum_i P_ij dO_i over its 256 queries, one slot per
//      kept coarse key, in a workspace region that only this CTA touches.
//   2. coarse reduce: for every coarse token c of level l >= 2, the partials
//      of the level-l query tokens in row c of the level-l key-major lists
//      (ascending), over their level-2 descendants (ascending).
//   3. key-major: one CTA per 16-token key block walks the query blocks of
//      its row of the level-1 key-major lists (ascending) and accumulates
//      dK, dV of its fine tokens; the epilogue adds each coarse gradient
//      divided by 16^l, the derivative of the mean pooling.

#include <math.h>

#include "keyset.cuh"

namespace llsa {

namespace {

template <typename T, int D>
__global__ void __launch_bounds__(256)
bwd_query_simt_kernel(AttnParams p, int G) {
  constexpr int DPT = D / 16;
  constexpr int kTile = (D == 64) ? 32 : 16;  // keeps static shared memory under 48 KB
  __shared__ KeyList kl;
  __shared__ float qs[16][D + 1];
  __shared__ float dos[16][D + 1];
  __shared__ float ks[kTile][D + 1];
  __shared__ float vs[kTile][D + 1];
  __shared__ float lw[kTile];
  __shared__ float ps[16][kTile];
  __shared__ float dss[16][kTile];
  __shared__ float lse_s[16], delta_s[16];

  const int g = blockIdx.x;  // group of G query blocks
  const int bh = blockIdx.y;
  const int tid = threadIdx.x;
  const int i = tid >> 4, sub = tid & 15;
  const int NG = p.N >> 7;  // partial groups of 8 query blocks per (b, h)
  const T* Q = static_cast<const T*>(p.q);
  const T* Kf = static_cast<const T*>(p.k);
  const T* Vf = static_cast<const T*>(p.v);
  const T* dO = static_cast<const T*>(p.dout);
  T* dQ = static_cast<T*>(p.dq);

  // key tile loader (fine rows from K/V, coarse rows from the pyramid)
  auto load_tile = [&](int t0, int tn) {
    for (int e = tid; e < tn * D; e += 256) {
      const int j = e / D, d = e % D;
      const int key = t0 + j;
      const int lv = kl.lvl[key];
      const int tok = kl.tok[key];
      if (lv == 0) {
        const size_t off = ((size_t)bh * p.N + tok) * D + d;
        ks[j][d] = to_f32(Kf[off]);
        vs[j][d] = to_f32(Vf[off]);
      } else {
        const size_t off = ((size_t)bh * (p.N >> (4 * lv)) + tok) * D + d;
        ks[j][d] = p.pk[lv][off];
        vs[j][d] = p.pv[lv][off];
      }
      if (d == 0) lw[j] = (lv == 0) ? 0.f : p.logw[lv];
    }
  };

  // zero this CTA's partial slots (levels 2..L)
  for (int l = 2; l <= p.L; ++l) {
    float* part = p.part[l] + ((size_t)bh * NG + g) * p.Kl[l] * 2 * D;
    for (int e = tid; e < p.Kl[l] * 2 * D; e += 256) part[e] = 0.f;
  }
  int flags = 0;
  for (int bb = 0; bb < G; ++bb) {
    const int b = g * G + bb;
    __syncthreads();
    if (tid < 32) flags |= build_key_list(kl, p, bh, b);
    const size_t row0 = (size_t)bh * p.N + (size_t)b * kBlock;
    for (int e = tid; e < 16 * D; e += 256) {
      qs[e / D][e % D] = to_f32(Q[row0 * D + e]);
      dos[e / D][e % D] = to_f32(dO[row0 * D + e]);
    }
    if (tid < 16) lse_s[tid] = p.lse_in[row0 + tid];
    __syncthreads();
    const float lse_i = lse_s[i];
    const bool live = lse_i > -INFINITY;
    // Sweep 1 over every key: Delta_i = sum_j P_ij dP_ij (exact, not dO . O
    // from the rounded output), A_i = sum_j P_ij dP_ij k_j, B_i = sum_j P_ij k_j,
    // so that dQ_i = scale * (A_i - Delta_i B_i).
    float accA[DPT], accB[DPT];
#pragma unroll
    for (int dd = 0; dd < DPT; ++dd) accA[dd] = accB[dd] = 0.f;
    float dpart = 0.f;
    const int nkeys = kl.n;
    for (int t0 = 0; t0 < nkeys; t0 += kTile) {
      const int tn = min(kTile, nkeys - t0);
      __syncthreads();
      load_tile(t0, tn);
      __syncthreads();
#pragma unroll
      for (int h = 0; h < kTile / 16; ++h) {
        const int j = sub + 16 * h;
        float P = 0.f, PdP = 0.f;
        if (j < tn && live) {
          float s = 0.f, dp = 0.f;
          for (int d = 0; d < D; ++d) {
            s = fmaf(qs[i][d], ks[j][d], s);
            dp = fmaf(dos[i][d], vs[j][d], dp);
          }
          P = expf(s * p.scale + lw[j] - lse_i);
          PdP = P * dp;
        }
        dpart += PdP;
        ps[i][j] = P;
        dss[i][j] = PdP;
      }
      __syncthreads();
#pragma unroll
      for (int dd = 0; dd < DPT; ++dd) {
        const int d = sub + 16 * dd;
        float a = accA[dd], bsum = accB[dd];
        for (int j = 0; j < tn; ++j) {
          a = fmaf(dss[i][j], ks[j][d], a);
          bsum = fmaf(ps[i][j], ks[j][d], bsum);
        }
        accA[dd] = a;
        accB[dd] = bsum;
      }
    }
#pragma unroll
    for (int o = 8; o > 0; o >>= 1) dpart += __shfl_xor_sync(0xffffffffu, dpart, o);
    const float delta_i = dpart;
    if (sub == 0) {
      delta_s[i] = delta_i;
      p.delta[row0 + i] = delta_i;
    }
#pragma unroll
    for (int dd = 0; dd < DPT; ++dd)
      store_elem(&dQ[(row0 + i) * D + sub + 16 * dd], (accA[dd] - delta_i * accB[dd]) * p.scale);
    // Sweep 2 over the coarse keys only: dS_ij = P_ij (dP_ij - Delta_i) and
    // the partials sum_i dS_ij q_i, sum_i P_ij dO_i over this block's queries.
    for (int t0 = kl.nfine; t0 < nkeys; t0 += kTile) {
      const int tn = min(kTile, nkeys - t0);
      __syncthreads();
      load_tile(t0, tn);
      __syncthreads();
#pragma unroll
      for (int h = 0; h < kTile / 16; ++h) {
        const int j = sub + 16 * h;
        float P = 0.f, dS = 0.f;
        if (j < tn && live) {
          float s = 0.f, dp = 0.f;
          for (int d = 0; d < D; ++d) {
            s = fmaf(qs[i][d], ks[j][d], s);
            dp = fmaf(dos[i][d], vs[j][d], dp);
          }
          P = expf(s * p.scale + lw[j] - lse_i);
          dS = P * (dp - delta_i);
        }
        ps[i][j] = P;
        dss[i][j] = dS;
      }
      __syncthreads();
      for (int e = tid; e < tn * D; e += 256) {
        const int j = e / D, d = e % D;
        const int lv = kl.lvl[t0 + j];
        float gk = 0.f, gv = 0.f;
        for (int r = 0; r < 16; ++r) {
          gk = fmaf(dss[r][j], qs[r][d], gk);
          gv = fmaf(ps[r][j], dos[r][d], gv);
        }
        float* part = p.part[lv] + (((size_t)bh * NG + g) * p.Kl[lv] + kl.slot[t0 + j]) * 2 * D;
        part[d] += gk * p.scale;
        part[D + d] += gv;
      }
    }
  }
  if (tid < 32) {
    flags = __reduce_or_sync(0xffffffffu, flags);
    if (tid == 0) report_status(p.status, flags);
  }
}

// Coarse gradient of token c at level l: thread per (kv, d).  The (query
// token, slot) pairs of row c of the level-l key-major lists are found first,
// in parallel, then every thread sums its column over them in order.
constexpr int kReduceChunk = 128;
__global__ void bwd_coarse_reduce_kernel(AttnParams p, int l) {
  __shared__ int s_q[kReduceChunk], s_slot[kReduceChunk];
  const int c = blockIdx.x;
  const int bh = blockIdx.y;
  const int D = p.D, K = p.Kl[l];
  const int nl = p.N >> (4 * l);
  const int NG = p.N >> 7;
  const int span = 2 << (4 * (l - 2));  // groups of 8 query blocks under a level-l token
  const int nsum = (l >= 3) ? 1 : span;  // levels >= 3 were pre-added into the first group
  const int t = threadIdx.x;            // kv * D + d
  const int32_t* rp = p.row_ptr[l] + (size_t)bh * (nl + 1);
  const int32_t* col = p.col[l] + (size_t)bh * nl * K;
  const float* part = p.part[l] + (size_t)bh * NG * K * 2 * D + t;
  const int beg = rp[c], end = rp[c + 1];
  float acc = 0.f;
  for (int e0 = beg; e0 < end; e0 += kReduceChunk) {
    const int cnt = min(kReduceChunk, end - e0);
    __syncthreads();
    for (int e = t; e < cnt; e += blockDim.x) {
      const int ql = col[e0 + e];
      const int32_t* row = p.idx[l] + ((size_t)bh * nl + ql) * K;
      RowRule rr;
      int slot = -1;
      for (int s = 0; s < K; ++s)
        if (rr.use(row[s], nl) && row[s] == c) slot = s;
      s_q[e] = ql;
      s_slot[e] = slot;
    }
    __syncthreads();
    // entries in batches of 8 whose loads are all in flight before the sums,
    // which still run in entry order, then group order (nsum is 2 at level 2
    // and 1 above)
    const size_t stride = (size_t)K * 2 * D;  // next group, same slot
    for (int eb = 0; eb < cnt; eb += 8) {
      float x0[8], x1[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int e = eb + i;
        const int slot = (e < cnt) ? s_slot[e] : -1;
        const float* src = part + ((size_t)(slot >= 0 ? s_q[e] : 0) * span * K + (slot >= 0 ? slot : 0)) * 2 * D;
        x0[i] = (slot >= 0) ? src[0] : 0.f;
        x1[i] = (slot >= 0 && nsum > 1) ? src[stride] : 0.f;
      }
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        acc += x0[i];
        acc += x1[i];
      }
    }
  }
  p.coarse[l][((size_t)bh * nl + c) * 2 * D + t] = acc;
}

template <typename T, int D>
__global__ void __launch_bounds__(256)
bwd_kv_simt_kernel(AttnParams p) {
  constexpr int DPT = D / 16;
  __shared__ float kc[16][D + 1];
  __shared__ float vc[16][D + 1];
  __shared__ float qs[16][D + 1];
  __shared__ float dos[16][D + 1];
  __shared__ float ps[16][17];
  __shared__ float dss[16][17];
  __shared__ float lse_s[16], delta_s[16];

  const int c = blockIdx.x;  // key block (level-1 token)
  const int bh = blockIdx.y;
  const int tid = threadIdx.x;
  const int j = tid >> 4, sub = tid & 15;  // key j of the block; sub = query in the score step
  const int K = p.K;
  const int n1 = p.N / kBlock;
  const T* Q = static_cast<const T*>(p.q);
  const T* Kf = static_cast<const T*>(p.k);
  const T* Vf = static_cast<const T*>(p.v);
  const T* dO = static_cast<const T*>(p.dout);

  const size_t krow0 = (size_t)bh * p.N + (size_t)c * kBlock;
  for (int e = tid; e < 16 * D; e += 256) {
    kc[e / D][e % D] = to_f32(Kf[krow0 * D + e]);
    vc[e / D][e % D] = to_f32(Vf[krow0 * D + e]);
  }
  float ak[DPT], av[DPT];
#pragma unroll
  for (int dd = 0; dd < DPT; ++dd) ak[dd] = av[dd] = 0.f;
  const int32_t* rp = p.row_ptr[1] + (size_t)bh * (n1 + 1);
  const int32_t* col = p.col[1] + (size_t)bh * n1 * K;
  const int beg = rp[c], end = rp[c + 1];
  for (int e = beg; e < end; ++e) {
    const int b = col[e];
    const size_t qrow0 = (size_t)bh * p.N + (size_t)b * kBlock;
    __syncthreads();
    for (int x = tid; x < 16 * D; x += 256) {
      qs[x / D][x % D] = to_f32(Q[qrow0 * D + x]);
      dos[x / D][x % D] = to_f32(dO[qrow0 * D + x]);
    }
    if (tid < 16) {
      lse_s[tid] = p.lse_in[qrow0 + tid];
      delta_s[tid] = p.delta[qrow0 + tid];
    }
    __syncthreads();
    {
      const int qi = sub;
      float P = 0.f, dS = 0.f;
      if (lse_s[qi] > -INFINITY) {
        float s = 0.f, dp = 0.f;
        for (int d = 0; d < D; ++d) {
          s = fmaf(qs[qi][d], kc[j][d], s);
          dp = fmaf(dos[qi][d], vc[j][d], dp);
        }
        P = expf(s * p.scale - lse_s[qi]);
        dS = P * (dp - delta_s[qi]);
      }
      ps[j][qi] = P;
      dss[j][qi] = dS;
    }
    __syncthreads();
#pragma unroll
    for (int dd = 0; dd < DPT; ++dd) {
      const int d = sub + 16 * dd;
      float a = ak[dd], v = av[dd];
      for (int r = 0; r < 16; ++r) {
        a = fmaf(dss[j][r], qs[r][d], a);
        v = fmaf(ps[j][r], dos[r][d], v);
      }
      ak[dd] = a;
      av[dd] = v;
    }
  }
  // epilogue: fine gradient plus each coarse gradient spread over its tokens
  T* dK = static_cast<T*>(p.dk);
  T* dV = static_cast<T*>(p.dv);
  const size_t tok = (size_t)c * kBlock + j;
#pragma unroll
  for (int dd = 0; dd < DPT; ++dd) {
    const int d = sub + 16 * dd;
    float gk = ak[dd] * p.scale, gv = av[dd];
    for (int l = 2; l <= p.L; ++l) {
      const int nl = p.N >> (4 * l);
      const float inv = 1.0f / (float)(1u << (4 * l));
      const float* cg = p.coarse[l] + ((size_t)bh * nl + (tok >> (4 * l))) * 2 * D;
      gk += cg[d] * inv;
      gv += cg[D + d] * inv;
    }
    store_elem(&dK[(krow0 + j) * D + d], gk);
    store_elem(&dV[(krow0 + j) * D + d], gv);
  }
}

template <typename T, int D>
cudaError_t launch_typed(const AttnParams& p, cudaStream_t s) {
  const int BH = p.B * p.H;
  const int n1 = p.N / kBlock;
  const int G = (p.L >= 2) ? 8 : 1;
  bwd_query_simt_kernel<T, D><<<dim3(n1 / G, BH), 256, 0, s>>>(p, G);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  e = launch_coarse_reduce(p, s);
  if (e != cudaSuccess) return e;
  bwd_kv_simt_kernel<T, D><<<dim3(n1, BH), 256, 0, s>>>(p);
  return cudaGetLastError();
}

}  // namespace

// For levels >= 3, first add each level-l query token's groups into its first
// group (thread per (token, slot, kv, d); the groups in ascending order), so
// the key-major gather reads one group per entry.
__global__ void bwd_span_reduce_kernel(AttnParams p, int l) {
  const int D = p.D, K = p.Kl[l];
  const int nl = p.N >> (4 * l);
  const int NG = p.N >> 7;
  const int span = 2 << (4 * (l - 2));
  const size_t per_tok = (size_t)K * 2 * D;
  const size_t total = (size_t)p.B * p.H * nl * per_tok;
  for (size_t e = (size_t)blockIdx.x * blockDim.x + threadIdx.x; e < total;
       e += (size_t)gridDim.x * blockDim.x) {
    const size_t w = e % per_tok;
    const size_t tok = e / per_tok;  // bh * nl + ql
    const size_t bh = tok / nl, ql = tok % nl;
    float* first = p.part[l] + ((bh * NG + ql * span) * per_tok) + w;
    float acc = first[0];
    for (int a = 1; a < span; ++a) acc += first[(size_t)a * per_tok];
    first[0] = acc;
  }
}

cudaError_t launch_coarse_reduce(const AttnParams& p, cudaStream_t s) {
  for (int l = 2; l <= p.L; ++l) {
    if (l >= 3) {
      const size_t total = (size_t)p.B * p.H * (p.N >> (4 * l)) * p.Kl[l] * 2 * p.D;
      int blocks = (int)((total + 255) / 256);
      if (blocks > 148 * 16) blocks = 148 * 16;
      bwd_span_reduce_kernel<<<blocks, 256, 0, s>>>(p, l);
      const cudaError_t e = cudaGetLastError();
      if (e != cudaSuccess) return e;
    }
    bwd_coarse_reduce_kernel<<<dim3(p.N >> (4 * l), p.B * p.H), 2 * p.D, 0, s>>>(p, l);
    const cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

cudaError_t launch_attn_bwd_simt(const AttnParams& p, int dtype, cudaStream_t s) {
  if (dtype == LLSA_BF16)
    return (p.D == 64) ? launch_typed<bf16, 64>(p, s) : launch_typed<bf16, 128>(p, s);
  return (p.D == 64) ? launch_typed<float, 64>(p, s) : launch_typed<float, 128>(p, s);
}

}  // namespace llsa
