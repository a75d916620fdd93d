// Sparse attention forward with hierarchical KV enrichment and KV
// reweighting, bf16 tensor-core kernel (Step 3 of the howistudyai explainer
// of "Trainable Log-linear Sparse Attention for Efficient Diffusion
// Transformers").
//
// One warp owns 4 consecutive 16-token query blocks, one after the other (a
// block is exactly the M = 16 of the warp MMA); a CTA of 4 warps covers the
// 16 blocks under one level-2 token, which share every coarse key.  The
// selected 16-token key blocks of a warp's 4 blocks form one stream of
// contiguous 16-row K/V tiles, gathered by 2D TMA loads (128-byte swizzle, no
// multicast) into a 2-stage ring that runs on across block boundaries, and
// the next block's Q tile is loaded into a second buffer while the current
// block is computed, so set-up latency is paid once per warp, not per block.
// S of the next tile is issued before the softmax and PV of the current one.
// The coarse K/V rows (fp32 pyramid) are converted once per CTA to bf16 tiles
// in shared memory, with ln(w_l) per key folded into the scores.
// S = Q K^T and O += P V run on m16n8k16 bf16 MMAs with fp32 accumulation;
// the softmax is online, in base 2, in fp32 registers.  When asked for
// (p.o_res), the epilogue also writes the bf16 rounding residual of O, from
// which the backward forms Delta without a second walk of the keys; a second
// instantiation (kSelect) selects I(1) in its prologue.

#include <math.h>
#include <string.h>

#include "keyset.cuh"
#include "mma_tiles.cuh"
#include "select_core.cuh"

namespace llsa {

namespace {

constexpr int kFwdWarps = 4;  // warps per CTA
constexpr int kBPW = 4;       // consecutive query blocks per warp (same coarse keys)
#ifndef LLSA_FWD_STAGES
#define LLSA_FWD_STAGES 2
#endif
constexpr int kStages = LLSA_FWD_STAGES;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

// Probabilities are taken relative to a reference max m_ref per row that is
// raised when a score exceeds it by more than kRescaleLog2; the output
// accumulators are rescaled only when some row of the warp needs it.
// Threshold 0: the reference is the exact running max, so the largest
// probability of a row is exactly 1 and its bf16 rounding is exact; a lagging
// reference (up to 2^8) let that rounding error through on rows with few keys.
constexpr float kRescaleLog2 = 0.0f;

struct SoftmaxState {
  float m[2];  // reference max of rows g and g+8 (base-2 scaled scores)
  float l[2];  // this thread's partial row sums, relative to m
};

// Online-softmax update of a 16x16 score tile held in two m16n8 accumulators
// (s[nt][0..1]: row g, keys 8nt+2t, 8nt+2t+1; s[nt][2..3]: row g+8), then
// P (bf16 A fragment) and rescaling of the output accumulators when needed.
template <int NT>
__device__ __forceinline__ void softmax_tile(float (&s)[2][4], const float (&lw)[2][2], float sc2,
                                             SoftmaxState& st, float (&o)[NT][4],
                                             uint32_t (&pa)[4]) {
  // pairs of columns run as packed f32x2 operations (bit-identical to scalar)
  float x[2][4];
  const uint64_t sc2x2 = f2_make(sc2, sc2);
#pragma unroll
  for (int nt = 0; nt < 2; ++nt) {
    const uint64_t lwp = f2_make(lw[nt][0], lw[nt][1]);
    const float2 a = f2_split(f2_fma(f2_make(s[nt][0], s[nt][1]), sc2x2, lwp));
    const float2 b = f2_split(f2_fma(f2_make(s[nt][2], s[nt][3]), sc2x2, lwp));
    x[nt][0] = a.x;
    x[nt][1] = a.y;
    x[nt][2] = b.x;
    x[nt][3] = b.y;
  }
  // common path: no max at all, only a check that no score exceeds the
  // reference by more than the threshold (false while the reference is -inf
  // only if the tile is fully masked too)
  bool hi = false;
#pragma unroll
  for (int nt = 0; nt < 2; ++nt)
    hi |= (x[nt][0] > st.m[0] + kRescaleLog2) | (x[nt][1] > st.m[0] + kRescaleLog2) |
          (x[nt][2] > st.m[1] + kRescaleLog2) | (x[nt][3] > st.m[1] + kRescaleLog2);
  if (__any_sync(0xffffffffu, hi)) {
    float mx0 = fmaxf(fmaxf(x[0][0], x[0][1]), fmaxf(x[1][0], x[1][1]));
    float mx1 = fmaxf(fmaxf(x[0][2], x[0][3]), fmaxf(x[1][2], x[1][3]));
    mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 1));
    mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 2));
    mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 1));
    mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 2));
    const bool up0 = mx0 > st.m[0] + kRescaleLog2;
    const bool up1 = mx1 > st.m[1] + kRescaleLog2;
    const float c0 = up0 ? ex2_approx(st.m[0] - mx0) : 1.f;  // 2^-inf = 0 for a first max
    const float c1 = up1 ? ex2_approx(st.m[1] - mx1) : 1.f;
    if (up0) st.m[0] = mx0;
    if (up1) st.m[1] = mx1;
    st.l[0] *= c0;
    st.l[1] *= c1;
    const uint64_t cc0 = f2_make(c0, c0), cc1 = f2_make(c1, c1);
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      const float2 a = f2_split(f2_mul(f2_make(o[nt][0], o[nt][1]), cc0));
      const float2 b = f2_split(f2_mul(f2_make(o[nt][2], o[nt][3]), cc1));
      o[nt][0] = a.x;
      o[nt][1] = a.y;
      o[nt][2] = b.x;
      o[nt][3] = b.y;
    }
  }
  // a row whose every score so far is -inf keeps m = -inf and gets p = 0
  const float b0 = (st.m[0] == -INFINITY) ? 0.f : st.m[0];
  const float b1 = (st.m[1] == -INFINITY) ? 0.f : st.m[1];
  float p[2][4];
  const uint64_t bb0 = f2_make(b0, b0), bb1 = f2_make(b1, b1);
#pragma unroll
  for (int nt = 0; nt < 2; ++nt) {
    const float2 a = f2_split(f2_sub(f2_make(x[nt][0], x[nt][1]), bb0));
    const float2 b = f2_split(f2_sub(f2_make(x[nt][2], x[nt][3]), bb1));
    p[nt][0] = ex2_approx(a.x);
    p[nt][1] = ex2_approx(a.y);
    p[nt][2] = ex2_approx(b.x);
    p[nt][3] = ex2_approx(b.y);
  }
  // l[0] += (p00 + p01) + (p10 + p11), l[1] likewise with p02.., as pairs
  const uint64_t u = f2_add(f2_make(p[0][0], p[0][2]), f2_make(p[0][1], p[0][3]));
  const uint64_t v = f2_add(f2_make(p[1][0], p[1][2]), f2_make(p[1][1], p[1][3]));
  const float2 lsum = f2_split(f2_add(f2_make(st.l[0], st.l[1]), f2_add(u, v)));
  st.l[0] = lsum.x;
  st.l[1] = lsum.y;
  pa[0] = pack_bf16(p[0][0], p[0][1]);
  pa[1] = pack_bf16(p[0][2], p[0][3]);
  pa[2] = pack_bf16(p[1][0], p[1][1]);
  pa[3] = pack_bf16(p[1][2], p[1][3]);
}

// kSelect: the CTA first selects I(1) for its 16 query blocks (the level-1
// step of the hierarchical Top-K, whose 16 sibling queries are exactly this
// CTA's blocks), writes those rows to p.idx[1] and reads them back below.
template <int D, bool kSelect>
__global__ void __launch_bounds__(kFwdWarps * 32)
attn_fwd_mma_kernel(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
                    const __grid_constant__ CUtensorMap tv, AttnParams p, SelectParams sp, int nct) {
  constexpr int TILE = 32 * D;  // bytes of a 16-row bf16 tile
  constexpr int NT = D / 8;
  constexpr int HALVES = D / 64;
  static_assert(kFwdWarps * kBPW == kSelQ, "a CTA's query blocks are one selection group");
  extern __shared__ unsigned char smem_raw[];
  unsigned char* sm = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  if constexpr (kSelect) {
    // the scratch is reused below, partly as TMA destinations
    select_group<D>(sp, blockIdx.y, blockIdx.x, reinterpret_cast<float*>(sm));
    fence_proxy_async_smem();
    __syncthreads();
  }
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, t = lane & 3;
  const int bh = blockIdx.y;
  const int n1 = p.N >> 4;
  const int wb0 = (blockIdx.x * kFwdWarps + warp) * kBPW;  // this warp's first block
  const int K = p.K;

  // per warp: 2 Q buffers | kStages x (K | V); then coarse K, coarse V, ...
  unsigned char* wbase = sm + (size_t)warp * TILE * (2 + 2 * kStages);
  unsigned char* ck = sm + (size_t)kFwdWarps * TILE * (2 + 2 * kStages);
  unsigned char* cv = ck + (size_t)nct * TILE;
  float* clw = reinterpret_cast<float*>(cv + (size_t)nct * TILE);
  uint64_t* bars = reinterpret_cast<uint64_t*>(clw + nct * 16);  // per warp: 2 Q, kStages ring
  int* clist = reinterpret_cast<int*>(bars + kFwdWarps * (2 + kStages));
  __shared__ int s_nc;
  __shared__ int flist_all[kFwdWarps][kBPW][32];  // used fine blocks of each block, ascending
  __shared__ int foff_all[kFwdWarps][kBPW + 1];   // stream offset of each block's tiles

  const uint32_t w0 = smem_u32(wbase);
  auto qbuf = [&](int i) { return w0 + (uint32_t)(i & 1) * TILE; };
  auto stage_k = [&](int st) { return w0 + (uint32_t)(2 + 2 * st) * TILE; };
  auto stage_v = [&](int st) { return w0 + (uint32_t)(3 + 2 * st) * TILE; };
  const uint32_t bar0 = smem_u32(bars + warp * (2 + kStages));
  auto qbar = [&](int i) { return bar0 + 8u * (i & 1); };
  auto bar_of = [&](int st) { return bar0 + 8u * (2 + st); };

  int flags = 0;
  // ---- fine lists of this warp's blocks
  int (*flist)[32] = flist_all[warp];
  int* foff = foff_all[warp];
  int nblk = 0;  // active blocks of this warp
  {
    int off = 0;
#pragma unroll
    for (int i = 0; i < kBPW; ++i) {
      const int b = wb0 + i;
      const bool on = (b < n1) && lane < K;
      const int32_t* src = p.idx[1] + ((size_t)bh * n1 + b) * K + lane;
      // rows this CTA has just written: read them from L2, never through the
      // read-only path
      const int v = on ? (kSelect ? __ldcg(src) : *src) : -1;
      const bool used = warp_row_used(v, lane, n1, on, flags);
      const unsigned m = __ballot_sync(0xffffffffu, used);
      if (used) flist[i][__popc(m & ((1u << lane) - 1u))] = v;
      if (lane == 0) foff[i] = off;
      off += __popc(m);
      if (b < n1) nblk = i + 1;
    }
    if (lane == 0) foff[kBPW] = off;
  }
  // ---- coarse keys shared by the CTA (warp 0 builds the list)
  if (warp == 0) {
    int n = 0;
    const int b0 = blockIdx.x * kFwdWarps * kBPW;
    for (int l = 2; l <= p.L; ++l) {
      const int nl = p.N >> (4 * l);
      const int a = b0 >> (4 * (l - 1));
      const int Kl = p.Kl[l];
      const int c = (lane < Kl) ? p.idx[l][((size_t)bh * nl + a) * Kl + lane] : -1;
      const bool u = warp_row_used(c, lane, nl, lane < Kl, flags);
      const unsigned m = __ballot_sync(0xffffffffu, u);
      if (u) clist[n + __popc(m & ((1u << lane) - 1u))] = (l << 24) | c;
      n += __popc(m);
    }
    if (lane == 0) s_nc = n;
  }
  if (lane == 0) {
    for (int i = 0; i < 2 + kStages; ++i) mbar_init(bar0 + 8u * i, 1);
    fence_mbar_init();
  }
  __syncwarp();
  const size_t rowbase = (size_t)bh * p.N;
  const int T = foff[kBPW];  // tiles in this warp's stream
  // stream item j -> (block, fine index)
  auto issue_item = [&](int j) {
    if (lane == 0) {
      int i = 0;
      while (j >= foff[i + 1]) ++i;
      const int blk = flist[i][j - foff[i]];
      const int st = j % kStages;
      mbar_arrive_expect_tx(bar_of(st), 2u * TILE);
      const int y = (int)(rowbase + (size_t)blk * 16);
#pragma unroll
      for (int h = 0; h < HALVES; ++h) {
        tma_load_2d(stage_k(st) + h * 2048, &tk, 64 * h, y, bar_of(st));
        tma_load_2d(stage_v(st) + h * 2048, &tv, 64 * h, y, bar_of(st));
      }
    }
  };
  auto issue_q = [&](int i) {
    if (lane == 0) {
      mbar_arrive_expect_tx(qbar(i), TILE);
      const int y = (int)(rowbase + (size_t)(wb0 + i) * 16);
#pragma unroll
      for (int h = 0; h < HALVES; ++h) tma_load_2d(qbuf(i) + h * 2048, &tq, 64 * h, y, qbar(i));
    }
  };
  for (int i = 0; i < nblk && i < 2; ++i) issue_q(i);
  for (int j = 0; j < T && j < kStages; ++j) issue_item(j);

  __syncthreads();  // coarse list and every warp's barriers ready
  const int nc = s_nc;
  const int ncpad = (nc + 15) >> 4;
  // coarse rows: fp32 pyramid -> bf16 swizzled tiles; padded keys are zero
  // rows with weight -inf
  for (int e = threadIdx.x; e < ncpad * 16 * (D / 8); e += blockDim.x) {
    const int key = e / (D / 8), j = e % (D / 8);
    uint4 kq = make_uint4(0, 0, 0, 0), vq = make_uint4(0, 0, 0, 0);
    if (key < nc) {
      const int l = clist[key] >> 24, c = clist[key] & 0xffffff;
      const size_t off = ((size_t)bh * (p.N >> (4 * l)) + c) * D + 8 * j;
      const float4* ks = reinterpret_cast<const float4*>(p.pk[l] + off);
      const float4* vs = reinterpret_cast<const float4*>(p.pv[l] + off);
      const float4 k0 = ks[0], k1 = ks[1], v0 = vs[0], v1 = vs[1];
      kq = make_uint4(pack_bf16(k0.x, k0.y), pack_bf16(k0.z, k0.w), pack_bf16(k1.x, k1.y), pack_bf16(k1.z, k1.w));
      vq = make_uint4(pack_bf16(v0.x, v0.y), pack_bf16(v0.z, v0.w), pack_bf16(v1.x, v1.y), pack_bf16(v1.z, v1.w));
    }
    const size_t dst = (size_t)(key >> 4) * TILE + swz(key & 15, j);
    *reinterpret_cast<uint4*>(ck + dst) = kq;
    *reinterpret_cast<uint4*>(cv + dst) = vq;
  }
  for (int e = threadIdx.x; e < ncpad * 16; e += blockDim.x)
    clw[e] = (e < nc) ? p.logw[clist[e] >> 24] * kLog2e : -INFINITY;
  __syncthreads();  // coarse tiles written

  const float sc2 = p.scale * kLog2e;
  const float zero_lw[2][2] = {{0.f, 0.f}, {0.f, 0.f}};
  bool ok = true;
  int j = 0;  // next stream item
  for (int i = 0; i < nblk && ok; ++i) {
    const int b = wb0 + i;
    ok = mbar_wait_bounded(qbar(i), (uint32_t)((i >> 1) & 1));
    if (!ok) break;
    uint32_t qa[D / 16][4];
    load_a_frags<D>(qbuf(i), lane, qa);
    __syncwarp();
    fence_proxy_async_smem();
    if (i + 2 < nblk) issue_q(i + 2);  // this Q buffer is free again

    float o[NT][4];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) o[nt][0] = o[nt][1] = o[nt][2] = o[nt][3] = 0.f;
    SoftmaxState st;
    st.m[0] = st.m[1] = -INFINITY;
    st.l[0] = st.l[1] = 0.f;
    const int jend = foff[i + 1];
    float s_cur[2][4];
    if (j < jend) {
      ok = mbar_wait_bounded(bar_of(j % kStages), (uint32_t)((j / kStages) & 1));
      if (!ok) break;
      qk_tile<D>(qa, stage_k(j % kStages), lane, s_cur);
    }
    for (; j < jend; ++j) {
      const int sidx = j % kStages;
      float s_nx[2][4];
      if (j + 1 < jend) {
        const int nidx = (j + 1) % kStages;
        ok = mbar_wait_bounded(bar_of(nidx), (uint32_t)(((j + 1) / kStages) & 1));
        if (!ok) break;
        qk_tile<D>(qa, stage_k(nidx), lane, s_nx);
      }
      uint32_t pa[4];
      softmax_tile<NT>(s_cur, zero_lw, sc2, st, o, pa);
      pv_tile<D>(pa, stage_v(sidx), lane, o);
      __syncwarp();
      fence_proxy_async_smem();
      if (j + kStages < T) issue_item(j + kStages);
      if (j + 1 < jend) {
#pragma unroll
        for (int a2 = 0; a2 < 2; ++a2)
#pragma unroll
          for (int e = 0; e < 4; ++e) s_cur[a2][e] = s_nx[a2][e];
      }
    }
    if (!ok) break;
    for (int ct = 0; ct < ncpad; ++ct) {
      float s[2][4];
      uint32_t pa[4];
      qk_tile<D>(qa, smem_u32(ck) + ct * TILE, lane, s);
      float lw[2][2];
#pragma unroll
      for (int nt = 0; nt < 2; ++nt) {
        lw[nt][0] = clw[ct * 16 + 8 * nt + 2 * t];
        lw[nt][1] = clw[ct * 16 + 8 * nt + 2 * t + 1];
      }
      softmax_tile<NT>(s, lw, sc2, st, o, pa);
      pv_tile<D>(pa, smem_u32(cv) + ct * TILE, lane, o);
    }
    // ---- epilogue: O = acc / l, LSE = ln(sum) = (m + log2 l) ln 2
    float l0 = st.l[0], l1 = st.l[1];
    l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
    l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
    l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
    l1 += __shfl_xor_sync(0xffffffffu, l1, 2);
    const float i0 = l0 > 0.f ? 1.f / l0 : 0.f;
    const float i1 = l1 > 0.f ? 1.f / l1 : 0.f;
    bf16* O = static_cast<bf16*>(p.out);
    bf16* R = static_cast<bf16*>(p.o_res);
    const size_t tok0 = rowbase + (size_t)b * 16 + g;
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      const float a0 = o[nt][0] * i0, a1 = o[nt][1] * i0;  // row g
      const float c0 = o[nt][2] * i1, c1 = o[nt][3] * i1;  // row g+8
      const uint32_t h0 = pack_bf16(a0, a1), h1 = pack_bf16(c0, c1);
      *reinterpret_cast<uint32_t*>(O + tok0 * D + 8 * nt + 2 * t) = h0;
      *reinterpret_cast<uint32_t*>(O + (tok0 + 8) * D + 8 * nt + 2 * t) = h1;
      if (R != nullptr) {  // what the bf16 rounding of O left out, itself in bf16
        *reinterpret_cast<uint32_t*>(R + tok0 * D + 8 * nt + 2 * t) =
            pack_bf16(a0 - bf16x2_lo(h0), a1 - bf16x2_hi(h0));
        *reinterpret_cast<uint32_t*>(R + (tok0 + 8) * D + 8 * nt + 2 * t) =
            pack_bf16(c0 - bf16x2_lo(h1), c1 - bf16x2_hi(h1));
      }
    }
    if (t == 0) {
      p.lse[tok0] = l0 > 0.f ? (st.m[0] + log2f(l0)) * kLn2 : -INFINITY;
      p.lse[tok0 + 8] = l1 > 0.f ? (st.m[1] + log2f(l1)) * kLn2 : -INFINITY;
    }
  }
  if (!ok) {
    // give the copies already in flight a bounded chance to land, then stop
    for (int q = j; q < T && q < j + kStages; ++q)
      mbar_wait_bounded(bar_of(q % kStages), (uint32_t)((q / kStages) & 1));
    flags |= LLSA_DEV_TIMEOUT;
  }
  flags = __reduce_or_sync(0xffffffffu, flags);
  if (lane == 0) report_status(p.status, flags);
}

template <int D, bool kSelect>
cudaError_t launch_typed(const AttnParams& p, const SelectParams& sp, const CUtensorMap* maps, cudaStream_t s) {
  constexpr int TILE = 32 * D;
  const int nct = (p.Kc + 15) / 16;
  size_t smem = 1024 + (size_t)kFwdWarps * TILE * (2 + 2 * kStages) + 2 * (size_t)nct * TILE +
                nct * 16 * sizeof(float) + kFwdWarps * (2 + kStages) * 8 + nct * 16 * sizeof(int);
  if (kSelect && smem < 1024 + select_scratch_bytes<D>()) smem = 1024 + select_scratch_bytes<D>();
  auto kern = attn_fwd_mma_kernel<D, kSelect>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout, (int)cudaSharedmemCarveoutMaxShared);
  if (e != cudaSuccess) return e;
  const int n1 = p.N / kBlock;
  const int per_cta = kFwdWarps * kBPW;
  dim3 grid((n1 + per_cta - 1) / per_cta, p.B * p.H);
  kern<<<grid, kFwdWarps * 32, smem, s>>>(maps[0], maps[1], maps[2], p, sp, nct);
  return cudaGetLastError();
}

}  // namespace

// maps: Q, K, V as 2D [B*H*N rows, D cols] bf16, box 16 x 64, 128-byte swizzle.
cudaError_t launch_attn_fwd_mma(const AttnParams& p, const CUtensorMap* maps, cudaStream_t s) {
  SelectParams none;
  memset(&none, 0, sizeof(none));
  return (p.D == 64) ? launch_typed<64, false>(p, none, maps, s) : launch_typed<128, false>(p, none, maps, s);
}

// The same forward with the level-1 selection in its prologue: sp describes
// level 1 (parent I(2), out I(1) == p.idx[1]); its query groups are the CTAs.
cudaError_t launch_attn_fwd_mma_select(const AttnParams& p, const SelectParams& sp, const CUtensorMap* maps,
                                       cudaStream_t s) {
  return (p.D == 64) ? launch_typed<64, true>(p, sp, maps, s) : launch_typed<128, true>(p, sp, maps, s);
}

}  // namespace llsa
