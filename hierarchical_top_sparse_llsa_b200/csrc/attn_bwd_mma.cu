// Backward of the enriched sparse attention, bf16 tensor-core kernels (the
// key-major backward of Step 4 of the howistudyai explainer of "Trainable
// Log-linear Sparse Attention for Efficient Diffusion Transformers";
// Building Blocks: Sparse Index Transpose).
//
// Pass 1, query-major (bwd_q_mma_kernel): one warp per 16-token query block,
// 8 sibling blocks per CTA (they share every coarse key).  Selected K/V tiles
// arrive by 2D TMA loads into a 2-stage per-warp ring.  Without the residual
// of O the key list is walked twice:
//   sweep 1: S = Q K^T, dP = dO V^T, P = w e^{S - LSE}, Delta_i = sum_j P dP
//            (from unrounded terms: O is stored rounded);
//   sweep 2: dS = P (dP - Delta), dQ += dS K.
// With it (kResid), Delta_i = dO_i . (O_i + R_i) comes first and the list is
// walked once, as sweep 2.
// In the sums over queries (dK, dV and the coarse partials) P and dS enter
// their MMAs as a bf16 hi + lo pair (about 16 mantissa bits): those sums
// cancel strongly on image-like inputs, and single bf16 rounding left some
// small dK entries 3x (dV 1.5x) outside a 2e-2 relative band.  dQ, a sum
// over keys, takes the same pair: a single bf16 dS stayed within 0.45 of the
// band on image-like inputs but left a few elements 1.13x outside it with
// the paper's level weights (16^l) on random inputs.
// Coarse keys then give dQ their share and, per CTA, the partials
// sum_i dS_ij q_i and sum_i P_ij dO_i over the 8 blocks' queries: the warps
// exchange P and dS (bf16 hi + lo) through shared memory and each warp sums
// the 8 blocks for its own output columns with MMAs in warp order, so no
// atomics are used.
//
// Pass 3, key-major (bwd_kv_mma_kernel): persistent single-warp CTAs take
// 16-token key blocks from a work counter and walk each block's row of the
// level-1 key-major lists (query blocks, ascending).  With the key block as
// the MMA's M: S^T = K Q^T, dP^T = V dO^T, dV += P^T dO, dK += dS^T Q.  The
// next row's K/V, coarse gradient rows and first Q/dO tiles are loaded
// before the current row's epilogue, which adds every coarse gradient
// divided by 16^l.
// (Pass 2, the per-level coarse reduce, is shared with the fp32 path.)

#include <math.h>

#include <algorithm>

#include "keyset.cuh"
#include "mma_tiles.cuh"

namespace llsa {

// tcgen05 key-major pass (attn_bwd_tc.cu): bf16, D = 64; maps as below
bool bwd_kv_tc_supported(const AttnParams& p);
cudaError_t launch_bwd_kv_tc(const AttnParams& p, const CUtensorMap* maps, cudaStream_t s);

namespace {

constexpr int kQWarps = 8;   // query blocks per CTA in pass 1 (one partial group)
constexpr int kRing = 2;    // K/V ring stages per warp in pass 1
#ifndef LLSA_KV_RING
#define LLSA_KV_RING 2
#endif
constexpr int kRingKV = LLSA_KV_RING;  // Q/dO ring stages in pass 3
constexpr float kLog2e = 1.4426950408889634f;

// P = exp2(S * sc2 + lw - lse2) on a 16x16 tile (rows g, g+8 of the query
// side); rows with lse = -inf get P = 0.  Pairs of columns run as packed
// f32x2 operations (bit-identical to the scalar fma).
__device__ __forceinline__ void probs_rows(const float (&s)[2][4], const float (&lw)[2][2], float sc2,
                                           float lse_g, float lse_g8, float (&P)[2][4]) {
  const float n0 = (lse_g == -INFINITY) ? -INFINITY : -lse_g;
  const float n1 = (lse_g8 == -INFINITY) ? -INFINITY : -lse_g8;
  const uint64_t sc = f2_make(sc2, sc2);
#pragma unroll
  for (int nt = 0; nt < 2; ++nt) {
    const float2 a = f2_split(f2_fma(f2_make(s[nt][0], s[nt][1]), sc, f2_make(lw[nt][0] + n0, lw[nt][1] + n0)));
    const float2 b = f2_split(f2_fma(f2_make(s[nt][2], s[nt][3]), sc, f2_make(lw[nt][0] + n1, lw[nt][1] + n1)));
    P[nt][0] = ex2_approx(a.x);
    P[nt][1] = ex2_approx(a.y);
    P[nt][2] = ex2_approx(b.x);
    P[nt][3] = ex2_approx(b.y);
  }
}

// dS = P (dP - Delta) in place of P, rows g (delta_g) and g+8 (delta_g8)
__device__ __forceinline__ void ds_rows(float (&P)[2][4], const float (&dp)[2][4], float delta_g,
                                        float delta_g8) {
  const uint64_t d0 = f2_make(delta_g, delta_g), d1 = f2_make(delta_g8, delta_g8);
#pragma unroll
  for (int nt = 0; nt < 2; ++nt) {
    const float2 a = f2_split(f2_mul(f2_make(P[nt][0], P[nt][1]), f2_sub(f2_make(dp[nt][0], dp[nt][1]), d0)));
    const float2 b = f2_split(f2_mul(f2_make(P[nt][2], P[nt][3]), f2_sub(f2_make(dp[nt][2], dp[nt][3]), d1)));
    P[nt][0] = a.x;
    P[nt][1] = a.y;
    P[nt][2] = b.x;
    P[nt][3] = b.y;
  }
}

// kResid: Delta_i = dO_i . (O_i + R_i) from the forward's bf16 rounding
// residual R of O (together about 16 mantissa bits beyond bf16), read at the
// start, so the key list is walked once instead of twice.
template <int D, bool kResid>
__global__ void __launch_bounds__(kQWarps * 32)
bwd_q_mma_kernel(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
                 const __grid_constant__ CUtensorMap tv, const __grid_constant__ CUtensorMap tdo,
                 AttnParams p, int nct) {
  constexpr int TILE = 32 * D;
  constexpr int NT = D / 8;
  constexpr int HALVES = D / 64;
  extern __shared__ unsigned char smem_raw[];
  unsigned char* sm = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, t = lane & 3;
  const int bh = blockIdx.y;
  const int grp = blockIdx.x;
  if (grp == 0 && bh == 0 && threadIdx.x == 0) *p.work = 0;  // pass 3's work counter
  const int n1 = p.N >> 4;
  const int b = grp * kQWarps + warp;
  const bool active = b < n1;
  const int K = p.K;

  // per warp: Q | dO | kRing x (K | V) tiles
  unsigned char* wbase = sm + (size_t)warp * TILE * (2 + 2 * kRing);
  unsigned char* ck = sm + (size_t)kQWarps * TILE * (2 + 2 * kRing);
  unsigned char* cv = ck + (size_t)nct * TILE;
  float* clw = reinterpret_cast<float*>(cv + (size_t)nct * TILE);
  uint64_t* bars = reinterpret_cast<uint64_t*>(clw + nct * 16);
  int* clist = reinterpret_cast<int*>(bars + kQWarps * (1 + kRing));
  int* cslot = clist + nct * 16;
  __shared__ int s_nc;
  __shared__ int flist_all[kQWarps][32];
  int* flist = flist_all[warp];

  const uint32_t w0 = smem_u32(wbase);
  const uint32_t qt = w0, dot = w0 + TILE;
  const uint32_t bar0 = smem_u32(bars + warp * (1 + kRing));
  auto ring_k = [&](int st) { return w0 + (uint32_t)(2 + 2 * st) * TILE; };
  auto ring_v = [&](int st) { return w0 + (uint32_t)(3 + 2 * st) * TILE; };
  auto bar_of = [&](int st) { return bar0 + 8u * (1 + st); };

  int flags = 0;
  const bool on_row = active && lane < K;
  const int my_blk = on_row ? p.idx[1][((size_t)bh * n1 + b) * K + lane] : -1;
  const bool used = warp_row_used(my_blk, lane, n1, on_row, flags);
  const unsigned fmask = __ballot_sync(0xffffffffu, used);
  const int nf = __popc(fmask);
  if (used) flist[__popc(fmask & ((1u << lane) - 1u))] = my_blk;
  __syncwarp();

  if (warp == 0) {
    int n = 0;
    const int b0 = grp * kQWarps;
    for (int l = 2; l <= p.L; ++l) {
      const int nl = p.N >> (4 * l);
      const int a = b0 >> (4 * (l - 1));
      const int Kl = p.Kl[l];
      const int c = (lane < Kl) ? p.idx[l][((size_t)bh * nl + a) * Kl + lane] : -1;
      const bool u = warp_row_used(c, lane, nl, lane < Kl, flags);
      const unsigned m = __ballot_sync(0xffffffffu, u);
      if (u) {
        const int pos = n + __popc(m & ((1u << lane) - 1u));
        clist[pos] = (l << 24) | c;
        cslot[pos] = lane;
      }
      n += __popc(m);
    }
    if (lane == 0) s_nc = n;
  }
  if (lane == 0) {
    for (int i = 0; i <= kRing; ++i) mbar_init(bar0 + 8u * i, 1);
    fence_mbar_init();
  }
  __syncthreads();
  const int nc = s_nc;
  const int ncpad = (nc + 15) >> 4;
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

  const size_t rowbase = (size_t)bh * p.N;
  const int ntiles = kResid ? nf : 2 * nf;  // without the residual the fine key list is walked twice
  auto issue = [&](int r) {
    if (lane == 0) {
      const int blk = flist[r % nf];
      const int st = r % kRing;
      mbar_arrive_expect_tx(bar_of(st), 2u * TILE);
      const int y = (int)(rowbase + (size_t)blk * 16);
#pragma unroll
      for (int h = 0; h < HALVES; ++h) {
        tma_load_2d(ring_k(st) + h * 2048, &tk, 64 * h, y, bar_of(st));
        tma_load_2d(ring_v(st) + h * 2048, &tv, 64 * h, y, bar_of(st));
      }
    }
  };
  if (active) {
    if (lane == 0) {
      mbar_arrive_expect_tx(bar0, 2u * TILE);
      const int y = (int)(rowbase + (size_t)b * 16);
#pragma unroll
      for (int h = 0; h < HALVES; ++h) {
        tma_load_2d(qt + h * 2048, &tq, 64 * h, y, bar0);
        tma_load_2d(dot + h * 2048, &tdo, 64 * h, y, bar0);
      }
    }
    for (int r = 0; r < ntiles && r < kRing; ++r) issue(r);
  }
  __syncthreads();  // coarse tiles written

  bool ok = true;
  float lse_g = 0.f, lse_g8 = 0.f, delta_g = 0.f, delta_g8 = 0.f;
  float dq[NT][4];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) dq[nt][0] = dq[nt][1] = dq[nt][2] = dq[nt][3] = 0.f;
  const float sc2 = p.scale * kLog2e;
  const float zero_lw[2][2] = {{0.f, 0.f}, {0.f, 0.f}};
  if (active) {
    ok = __all_sync(0xffffffffu, mbar_wait_bounded(bar0, 0));  // warp-uniform before the shuffles
    const size_t tok0 = rowbase + (size_t)b * 16 + g;
    lse_g = p.lse_in[tok0] * kLog2e;
    lse_g8 = p.lse_in[tok0 + 8] * kLog2e;
    if constexpr (kResid) {
      if (ok) {
        // dO from this warp's tile (swizzled), O and its residual from memory;
        // lane (g, t) sums columns 8nt + 2t, +1 of rows g and g+8
        const bf16* Og = static_cast<const bf16*>(p.o);
        const bf16* Rg = static_cast<const bf16*>(p.o_res);
        float a0 = 0.f, a1 = 0.f;
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
          uint32_t d0, d1;
          asm volatile("ld.shared.u32 %0, [%1];" : "=r"(d0) : "r"(dot + swz(g, nt) + 4 * t));
          asm volatile("ld.shared.u32 %0, [%1];" : "=r"(d1) : "r"(dot + swz(g + 8, nt) + 4 * t));
          const uint32_t o0 = *reinterpret_cast<const uint32_t*>(Og + tok0 * D + 8 * nt + 2 * t);
          const uint32_t o1 = *reinterpret_cast<const uint32_t*>(Og + (tok0 + 8) * D + 8 * nt + 2 * t);
          const uint32_t r0 = *reinterpret_cast<const uint32_t*>(Rg + tok0 * D + 8 * nt + 2 * t);
          const uint32_t r1 = *reinterpret_cast<const uint32_t*>(Rg + (tok0 + 8) * D + 8 * nt + 2 * t);
          a0 = fmaf(bf16x2_lo(d0), bf16x2_lo(o0) + bf16x2_lo(r0), a0);
          a0 = fmaf(bf16x2_hi(d0), bf16x2_hi(o0) + bf16x2_hi(r0), a0);
          a1 = fmaf(bf16x2_lo(d1), bf16x2_lo(o1) + bf16x2_lo(r1), a1);
          a1 = fmaf(bf16x2_hi(d1), bf16x2_hi(o1) + bf16x2_hi(r1), a1);
        }
        a0 += __shfl_xor_sync(0xffffffffu, a0, 1);
        a0 += __shfl_xor_sync(0xffffffffu, a0, 2);
        a1 += __shfl_xor_sync(0xffffffffu, a1, 1);
        a1 += __shfl_xor_sync(0xffffffffu, a1, 2);
        delta_g = a0;
        delta_g8 = a1;
      }
    }
    // Both sweeps walk the ring tiles 0..2nf-1 with one software pipeline:
    // S and dP of tile r+1 are issued before the elementwise work of tile r.
    float dp0 = 0.f, dp1 = 0.f;
    float s_cur[2][4], d_cur[2][4];
    int r = 0;
    if (ntiles > 0 && ok) {
      ok = mbar_wait_bounded(bar_of(0), 0);
      if (ok) {
        qk_tile_ss<D>(qt, ring_k(0), lane, s_cur);
        qk_tile_ss<D>(dot, ring_v(0), lane, d_cur);
      }
    }
    for (; r < ntiles && ok; ++r) {
      const int st = r % kRing;
      float s_nx[2][4], d_nx[2][4];
      if (r + 1 < ntiles) {
        const int ns = (r + 1) % kRing;
        ok = mbar_wait_bounded(bar_of(ns), (uint32_t)(((r + 1) / kRing) & 1));
        if (!ok) break;
        qk_tile_ss<D>(qt, ring_k(ns), lane, s_nx);
        qk_tile_ss<D>(dot, ring_v(ns), lane, d_nx);
      }
      float P[2][4];
      probs_rows(s_cur, zero_lw, sc2, lse_g, lse_g8, P);
      if (!kResid && r < nf) {  // sweep 1: Delta
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
          dp0 += P[nt][0] * d_cur[nt][0] + P[nt][1] * d_cur[nt][1];
          dp1 += P[nt][2] * d_cur[nt][2] + P[nt][3] * d_cur[nt][3];
        }
        if (r == nf - 1) {
          // the coarse keys close sweep 1 (their tiles are resident)
          for (int ct = 0; ct < ncpad; ++ct) {
            float s[2][4], dpv[2][4], Pc[2][4], lw[2][2];
#pragma unroll
            for (int nt = 0; nt < 2; ++nt) {
              lw[nt][0] = clw[ct * 16 + 8 * nt + 2 * t];
              lw[nt][1] = clw[ct * 16 + 8 * nt + 2 * t + 1];
            }
            qk_tile_ss<D>(qt, smem_u32(ck) + ct * TILE, lane, s);
            qk_tile_ss<D>(dot, smem_u32(cv) + ct * TILE, lane, dpv);
            probs_rows(s, lw, sc2, lse_g, lse_g8, Pc);
#pragma unroll
            for (int nt = 0; nt < 2; ++nt) {
              dp0 += Pc[nt][0] * dpv[nt][0] + Pc[nt][1] * dpv[nt][1];
              dp1 += Pc[nt][2] * dpv[nt][2] + Pc[nt][3] * dpv[nt][3];
            }
          }
          dp0 += __shfl_xor_sync(0xffffffffu, dp0, 1);
          dp0 += __shfl_xor_sync(0xffffffffu, dp0, 2);
          dp1 += __shfl_xor_sync(0xffffffffu, dp1, 1);
          dp1 += __shfl_xor_sync(0xffffffffu, dp1, 2);
          delta_g = dp0;
          delta_g8 = dp1;
        }
      } else {  // sweep 2: dQ += dS K
        ds_rows(P, d_cur, delta_g, delta_g8);
        uint32_t dsh[4], dsl[4];
        split_frag(P, dsh, dsl);
        pv_tile2<D>(dsh, dsl, ring_k(st), lane, dq);
      }
      __syncwarp();
      fence_proxy_async_smem();
      if (r + kRing < ntiles) issue(r + kRing);
      if (r + 1 < ntiles) {
#pragma unroll
        for (int a2 = 0; a2 < 2; ++a2)
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            s_cur[a2][e] = s_nx[a2][e];
            d_cur[a2][e] = d_nx[a2][e];
          }
      }
    }
    if (!kResid && nf == 0 && ok) {  // no fine keys: Delta from the coarse keys alone
      for (int ct = 0; ct < ncpad; ++ct) {
        float s[2][4], dpv[2][4], Pc[2][4], lw[2][2];
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
          lw[nt][0] = clw[ct * 16 + 8 * nt + 2 * t];
          lw[nt][1] = clw[ct * 16 + 8 * nt + 2 * t + 1];
        }
        qk_tile_ss<D>(qt, smem_u32(ck) + ct * TILE, lane, s);
        qk_tile_ss<D>(dot, smem_u32(cv) + ct * TILE, lane, dpv);
        probs_rows(s, lw, sc2, lse_g, lse_g8, Pc);
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
          dp0 += Pc[nt][0] * dpv[nt][0] + Pc[nt][1] * dpv[nt][1];
          dp1 += Pc[nt][2] * dpv[nt][2] + Pc[nt][3] * dpv[nt][3];
        }
      }
      dp0 += __shfl_xor_sync(0xffffffffu, dp0, 1);
      dp0 += __shfl_xor_sync(0xffffffffu, dp0, 2);
      dp1 += __shfl_xor_sync(0xffffffffu, dp1, 1);
      dp1 += __shfl_xor_sync(0xffffffffu, dp1, 2);
      delta_g = dp0;
      delta_g8 = dp1;
    }
    if (t == 0) {
      p.delta[tok0] = delta_g;
      p.delta[tok0 + 8] = delta_g8;
    }
    if (!ok) {
      for (int q = r; q < ntiles && q < r + kRing; ++q)
        mbar_wait_bounded(bar_of(q % kRing), (uint32_t)((q / kRing) & 1));
      flags |= LLSA_DEV_TIMEOUT;
    }
  }

  // Coarse keys: this block's dQ share, then the CTA's partials
  //   part_dk[key] = scale * sum_i dS_i,key q_i,  part_dv[key] = sum_i P_i,key dO_i
  // over the 8 blocks' 128 queries.  Each warp leaves P and dS (bf16 hi + lo,
  // rows = its queries, columns = the 16 coarse keys) in shared memory; after
  // one barrier, warp w' owns D/32 output n-tiles of one of the two partials
  // and sums the 8 blocks in warp order with MMAs (the 16 queries of a block
  // are the contraction), so no fp32 staging or cross-warp add is needed.
  constexpr int XROW = 48;          // bytes per row of a 16 x 16 bf16 exchange matrix (conflict-free)
  constexpr int XMAT = 16 * XROW;   // one matrix
  constexpr int NTW = D / 32;       // output n-tiles per warp
  const int NG = n1 / kQWarps;
  auto xbuf = [&](int w) { return smem_u32(sm + (size_t)w * TILE * (2 + 2 * kRing) + 2 * TILE); };
  for (int ct = 0; ct < ncpad; ++ct) {
    uint32_t xw = xbuf(warp);  // [dS hi | dS lo | P hi | P lo], reuses this warp's ring
    if (active && ok) {
      float s[2][4], dpv[2][4], P[2][4], dS[2][4], lw[2][2];
#pragma unroll
      for (int nt = 0; nt < 2; ++nt) {
        lw[nt][0] = clw[ct * 16 + 8 * nt + 2 * t];
        lw[nt][1] = clw[ct * 16 + 8 * nt + 2 * t + 1];
      }
      qk_tile_ss<D>(qt, smem_u32(ck) + ct * TILE, lane, s);
      qk_tile_ss<D>(dot, smem_u32(cv) + ct * TILE, lane, dpv);
      probs_rows(s, lw, sc2, lse_g, lse_g8, P);
#pragma unroll
      for (int nt = 0; nt < 2; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) dS[nt][e] = P[nt][e] * (dpv[nt][e] - ((e < 2) ? delta_g : delta_g8));
      uint32_t frag[4][4];  // dS hi, dS lo, P hi, P lo (A-fragment order)
      split_frag(dS, frag[0], frag[1]);
      split_frag(P, frag[2], frag[3]);
      pv_tile2<D>(frag[0], frag[1], smem_u32(ck) + ct * TILE, lane, dq);
      // fragment register i holds rows g (i even) / g+8 (i odd), columns 8(i>>1) + 2t, +1
#pragma unroll
      for (int m = 0; m < 4; ++m)
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int row = g + 8 * (i & 1), col = 8 * (i >> 1) + 2 * t;
          asm volatile("st.shared.u32 [%0], %1;" ::"r"(xw + m * XMAT + row * XROW + col * 2), "r"(frag[m][i])
                       : "memory");
        }
    } else {
      for (int e = lane; e < 4 * XMAT / 4; e += 32)
        asm volatile("st.shared.u32 [%0], %1;" ::"r"(xw + 4 * e), "r"(0u) : "memory");
    }
    __syncthreads();
    {
      const int kv = warp >> 2;           // 0: dK partial (dS, Q), 1: dV partial (P, dO)
      const int j0 = NTW * (warp & 3);    // first output n-tile
      float acc[NTW][4];
#pragma unroll
      for (int j = 0; j < NTW; ++j) acc[j][0] = acc[j][1] = acc[j][2] = acc[j][3] = 0.f;
      const int mi = lane >> 3;
      // A = X^T (keys x queries) from X (queries x keys, row-major): transposed loads
      const int xr = (mi >> 1) * 8 + (lane & 7), xc = (mi & 1) * 8;
      const int vrow = (mi & 1) * 8 + (lane & 7), vc = mi >> 1;
      for (int w = 0; w < kQWarps; ++w) {
        const uint32_t xs = xbuf(w) + (2 * kv) * XMAT + xr * XROW + xc * 2;
        uint32_t ah[4], al[4];
        ldsm_x4_t(xs, ah[0], ah[1], ah[2], ah[3]);
        ldsm_x4_t(xs + XMAT, al[0], al[1], al[2], al[3]);
        const uint32_t tile = smem_u32(sm + (size_t)w * TILE * (2 + 2 * kRing)) + kv * TILE;  // Q_w or dO_w
#pragma unroll
        for (int jj = 0; jj < NTW; jj += 2) {
          const int nn = (j0 + jj) >> 1;
          uint32_t b0, b1, b2, b3;
          ldsm_x4_t(tile + swz(vrow, 2 * nn + vc), b0, b1, b2, b3);
          mma_bf16(acc[jj], ah, b0, b1);
          mma_bf16(acc[jj + 1], ah, b2, b3);
          mma_bf16(acc[jj], al, b0, b1);
          mma_bf16(acc[jj + 1], al, b2, b3);
        }
      }
      const float f = (kv == 0) ? p.scale : 1.f;
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        const int ck_idx = ct * 16 + g + 8 * half;
        if (ck_idx < nc) {
          const int l = clist[ck_idx] >> 24;
          float* part = p.part[l] + ((((size_t)bh * NG + grp) * p.Kl[l] + cslot[ck_idx]) * 2 + kv) * D;
#pragma unroll
          for (int j = 0; j < NTW; ++j)
            *reinterpret_cast<float2*>(part + 8 * (j0 + j) + 2 * t) =
                make_float2(acc[j][2 * half] * f, acc[j][2 * half + 1] * f);
        }
      }
    }
    __syncthreads();  // the exchange matrices are rewritten by the next coarse tile
  }

  if (active) {
    bf16* dQ = static_cast<bf16*>(p.dq);
    const size_t tok0 = rowbase + (size_t)b * 16 + g;
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      *reinterpret_cast<uint32_t*>(dQ + tok0 * D + 8 * nt + 2 * t) =
          pack_bf16(dq[nt][0] * p.scale, dq[nt][1] * p.scale);
      *reinterpret_cast<uint32_t*>(dQ + (tok0 + 8) * D + 8 * nt + 2 * t) =
          pack_bf16(dq[nt][2] * p.scale, dq[nt][3] * p.scale);
    }
  }
  flags = __reduce_or_sync(0xffffffffu, flags);
  if (lane == 0) report_status(p.status, flags);
}

template <int D>
__global__ void __launch_bounds__(32)
bwd_kv_mma_kernel(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
                  const __grid_constant__ CUtensorMap tv, const __grid_constant__ CUtensorMap tdo,
                  AttnParams p) {
  constexpr int TILE = 32 * D;
  constexpr int NT = D / 8;
  constexpr int HALVES = D / 64;
  constexpr int SIDE = 128;       // LSE[16] and Delta[16] of a stage's query block (fp32)
  constexpr int CROW = 2 * D * 4;  // one coarse gradient row dK(l) | dV(l), fp32
  // K_c | V_c | kRingKV x (Q | dO) tiles (each 1024-byte aligned for the
  // 128-byte swizzle), kRingKV side buffers, two sets of L-1 coarse rows
  extern __shared__ unsigned char smem_raw[];
  unsigned char* sm = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  __shared__ __align__(8) uint64_t bars[1 + kRingKV];  // [0]: K/V + coarse rows; then the ring
  const int lane = threadIdx.x;
  const int g = lane >> 2, t = lane & 3;
  const int n1 = p.N >> 4;
  const int items = p.B * p.H * n1;
  const int K = p.K, L = p.L;

  const uint32_t w0 = smem_u32(sm);
  const uint32_t kt = w0, vt = w0 + TILE;
  auto ring_q = [&](int st) { return w0 + (uint32_t)(2 + 2 * st) * TILE; };
  auto ring_do = [&](int st) { return w0 + (uint32_t)(3 + 2 * st) * TILE; };
  unsigned char* sideb = sm + (2 + 2 * kRingKV) * TILE;
  const uint32_t side0 = smem_u32(sideb);
  unsigned char* cgb = sideb + kRingKV * SIDE;
  const uint32_t kvbar = smem_u32(&bars[0]);
  auto bar_of = [&](uint32_t pos) { return smem_u32(&bars[1 + pos % kRingKV]); };
  auto par_of = [&](uint32_t pos) { return (pos / kRingKV) & 1u; };
  if (lane == 0) {
    for (int i = 0; i <= kRingKV; ++i) mbar_init(smem_u32(&bars[i]), 1);
    fence_mbar_init();
  }
  __syncwarp();

  // One key block's row of the level-1 key-major lists.  colw holds
  // col[beg + 32 * win + lane], a window of the row's query blocks.
  struct Row {
    int item, bh, c, beg, nq, colw, win;
  };
  auto row_bounds = [&](int item, Row& R) {
    R.item = item;
    R.bh = 0, R.c = 0, R.beg = 0, R.nq = 0, R.colw = 0, R.win = -1;
    if (item < items) {
      R.bh = item / n1;
      R.c = item - R.bh * n1;
      const int32_t* rp = p.row_ptr[1] + (size_t)R.bh * (n1 + 1);
      R.beg = rp[R.c];
      R.nq = rp[R.c + 1] - R.beg;
    }
  };
  auto row_window = [&](Row& R, int win) {
    R.win = win;
    const int j = 32 * win + lane;
    R.colw = (j < R.nq) ? p.col[1][(size_t)R.bh * n1 * K + R.beg + j] : 0;
  };
  // ring position pos <- tile r of row R (all lanes call; lane 0 issues)
  auto issue = [&](Row& R, int r, uint32_t pos) {
    if ((r >> 5) != R.win) row_window(R, r >> 5);
    const int qb = __shfl_sync(0xffffffffu, R.colw, r & 31);
    if (lane == 0) {
      const uint32_t st = pos % kRingKV;
      const uint32_t bar = bar_of(pos);
      mbar_arrive_expect_tx(bar, 2u * TILE + SIDE);
      const size_t row0 = (size_t)R.bh * p.N + (size_t)qb * 16;
      const int y = (int)row0;
#pragma unroll
      for (int h = 0; h < HALVES; ++h) {
        tma_load_2d(ring_q(st) + h * 2048, &tq, 64 * h, y, bar);
        tma_load_2d(ring_do(st) + h * 2048, &tdo, 64 * h, y, bar);
      }
      bulk_load(side0 + st * SIDE, p.lse_in + row0, 64, bar);
      bulk_load(side0 + st * SIDE + 64, p.delta + row0, 64, bar);
    }
  };
  // K_c, V_c (if the row is not empty) and the coarse gradient rows of key
  // block c into coarse buffer `par`
  auto issue_kv = [&](const Row& R, int par) {
    if (lane == 0) {
      const uint32_t bytes = (R.nq > 0 ? 2u * TILE : 0u) + (uint32_t)(L - 1) * CROW;
      mbar_arrive_expect_tx(kvbar, bytes);
      if (R.nq > 0) {
        const int y = (int)((size_t)R.bh * p.N + (size_t)R.c * 16);
#pragma unroll
        for (int h = 0; h < HALVES; ++h) {
          tma_load_2d(kt + h * 2048, &tk, 64 * h, y, kvbar);
          tma_load_2d(vt + h * 2048, &tv, 64 * h, y, kvbar);
        }
      }
      for (int l = 2; l <= L; ++l) {
        const size_t tc = (size_t)R.bh * (p.N >> (4 * l)) + (R.c >> (4 * (l - 1)));
        bulk_load(smem_u32(cgb + (size_t)(par * (L - 1) + (l - 2)) * CROW), p.coarse[l] + tc * 2 * D, CROW,
                  kvbar);
      }
    }
  };

  // work items are key blocks, taken in order from a counter that pass 1 zeroed
  int nxt_l0 = (lane == 0) ? atomicAdd(p.work, 1) : 0;
  Row cur;
  row_bounds(__shfl_sync(0xffffffffu, nxt_l0, 0), cur);
  nxt_l0 = (lane == 0) ? atomicAdd(p.work, 1) : 0;
  uint32_t pos = 0;     // ring position of cur's first tile
  uint32_t issued = 0;  // ring positions issued so far
  uint32_t kvph = 0;
  int par = 0;
  bool kv_pending = false;
  if (cur.item < items) {
    issue_kv(cur, par);
    kv_pending = true;
    for (int r = 0; r < cur.nq && r < kRingKV; ++r) issue(cur, r, issued++);
  }
  const float sc2 = p.scale * kLog2e;
  bool ok = true;
  while (cur.item < items && ok) {
    Row nxt;
    row_bounds(__shfl_sync(0xffffffffu, nxt_l0, 0), nxt);  // loads stay in flight
    nxt_l0 = (lane == 0) ? atomicAdd(p.work, 1) : 0;         // likewise
    ok = mbar_wait_bounded(kvbar, kvph);
    if (!ok) break;
    kv_pending = false;
    kvph ^= 1u;

    float dk[NT][4], dv[NT][4];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      dk[nt][0] = dk[nt][1] = dk[nt][2] = dk[nt][3] = 0.f;
      dv[nt][0] = dv[nt][1] = dv[nt][2] = dv[nt][3] = 0.f;
    }
    const int nq = cur.nq;
    // software pipeline: S^T and dP^T of query block r+1 are issued before
    // the elementwise step and the dV/dK products of block r
    float s_cur[2][4], d_cur[2][4];
    if (nq > 0) {
      ok = mbar_wait_bounded(bar_of(pos), par_of(pos));
      if (!ok) break;
      qk_tile_ss<D>(kt, ring_q(pos % kRingKV), lane, s_cur);
      qk_tile_ss<D>(vt, ring_do(pos % kRingKV), lane, d_cur);
    }
    if (nxt.item < items) row_window(nxt, 0);  // its query blocks, for the first issues below
    for (int r = 0; r < nq; ++r) {
      const uint32_t pr = pos + r;
      float s_nx[2][4], d_nx[2][4];
      if (r + 1 < nq) {
        ok = mbar_wait_bounded(bar_of(pr + 1), par_of(pr + 1));
        if (!ok) break;
        qk_tile_ss<D>(kt, ring_q((pr + 1) % kRingKV), lane, s_nx);
        qk_tile_ss<D>(vt, ring_do((pr + 1) % kRingKV), lane, d_nx);
      }
      // LSE and Delta of the queries in this thread's columns 8nt + 2t + j;
      // pairs of columns run as packed f32x2 operations.  A query without
      // keys (LSE = -inf) gets exponent -inf, so P = 0.
      const float* side = reinterpret_cast<const float*>(sideb + (pr % kRingKV) * SIDE);
      float P[2][4], dS[2][4];
#pragma unroll
      for (int nt = 0; nt < 2; ++nt) {
        const float2 lse = *reinterpret_cast<const float2*>(side + 8 * nt + 2 * t);
        const float2 del = *reinterpret_cast<const float2*>(side + 16 + 8 * nt + 2 * t);
        const float a0 = lse.x * kLog2e, a1 = lse.y * kLog2e;
        const uint64_t nl = f2_make(a0 == -INFINITY ? -INFINITY : -a0, a1 == -INFINITY ? -INFINITY : -a1);
        const uint64_t dl = f2_make(del.x, del.y);
#pragma unroll
        for (int h = 0; h < 2; ++h) {  // h = 0: row g (e = 0, 1); h = 1: row g + 8 (e = 2, 3)
          const float2 x =
              f2_split(f2_fma(f2_make(s_cur[nt][2 * h], s_cur[nt][2 * h + 1]), f2_make(sc2, sc2), nl));
          P[nt][2 * h] = ex2_approx(x.x);
          P[nt][2 * h + 1] = ex2_approx(x.y);
          const float2 ds = f2_split(f2_mul(f2_make(P[nt][2 * h], P[nt][2 * h + 1]),
                                            f2_sub(f2_make(d_cur[nt][2 * h], d_cur[nt][2 * h + 1]), dl)));
          dS[nt][2 * h] = ds.x;
          dS[nt][2 * h + 1] = ds.y;
        }
      }
      uint32_t ph[4], pl[4], dsh[4], dsl[4];
      split_frag(P, ph, pl);
      split_frag(dS, dsh, dsl);
      pv_tile2<D>(ph, pl, ring_do(pr % kRingKV), lane, dv);
      pv_tile2<D>(dsh, dsl, ring_q(pr % kRingKV), lane, dk);
      __syncwarp();
      fence_proxy_async_smem();
      if (r + kRingKV < nq) issue(cur, r + kRingKV, issued++);
      if (r + 1 < nq) {
#pragma unroll
        for (int a = 0; a < 2; ++a)
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            s_cur[a][e] = s_nx[a][e];
            d_cur[a][e] = d_nx[a][e];
          }
      }
    }
    if (!ok) break;
    pos += nq;
    // the next row's loads go out before this row's epilogue
    __syncwarp();
    fence_proxy_async_smem();
    if (nxt.item < items) {
      issue_kv(nxt, par ^ 1);
      kv_pending = true;
      for (int r = 0; r < nxt.nq && r < kRingKV; ++r) issue(nxt, r, issued++);
    }
    // epilogue: dK = scale * acc + sum_l coarse dK(l)[t >> 4l] / 16^l (likewise dV)
    bf16* dK = static_cast<bf16*>(p.dk);
    bf16* dV = static_cast<bf16*>(p.dv);
    const size_t rowbase = (size_t)cur.bh * p.N;
#pragma unroll
    for (int half = 0; half < 2; ++half) {
      const size_t tok = (size_t)cur.c * 16 + g + 8 * half;
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        const int d = 8 * nt + 2 * t;
        float k0 = dk[nt][2 * half] * p.scale, k1 = dk[nt][2 * half + 1] * p.scale;
        float v0 = dv[nt][2 * half], v1 = dv[nt][2 * half + 1];
        for (int l = 2; l <= L; ++l) {
          const float inv = 1.0f / (float)(1u << (4 * l));
          const float* cg = reinterpret_cast<const float*>(cgb + (size_t)(par * (L - 1) + (l - 2)) * CROW);
          const float2 gk = *reinterpret_cast<const float2*>(cg + d);
          const float2 gv = *reinterpret_cast<const float2*>(cg + D + d);
          k0 += gk.x * inv;
          k1 += gk.y * inv;
          v0 += gv.x * inv;
          v1 += gv.y * inv;
        }
        *reinterpret_cast<uint32_t*>(dK + (rowbase + tok) * D + d) = pack_bf16(k0, k1);
        *reinterpret_cast<uint32_t*>(dV + (rowbase + tok) * D + d) = pack_bf16(v0, v1);
      }
    }
    cur = nxt;
    par ^= 1;
  }
  if (!ok) {
    // let every copy still in flight land before the CTA exits
    if (kv_pending) mbar_wait_bounded(kvbar, kvph);
    for (uint32_t q = pos; q < issued; ++q) mbar_wait_bounded(bar_of(q), par_of(q));
    if (lane == 0) report_status(p.status, LLSA_DEV_TIMEOUT);
  }
}

template <int D>
cudaError_t launch_typed(const AttnParams& p, const CUtensorMap* maps, cudaStream_t s, bool tc_kv) {
  constexpr int TILE = 32 * D;
  const int BH = p.B * p.H;
  const int n1 = p.N / kBlock;
  const int nct = (p.Kc + 15) / 16;
  // pass 1
  const size_t smem1 = 1024 + (size_t)kQWarps * TILE * (2 + 2 * kRing) + 2 * (size_t)nct * TILE +
                       nct * 16 * sizeof(float) + kQWarps * (1 + kRing) * 8 + 2 * nct * 16 * sizeof(int);
  auto kern1 = (p.o_res != nullptr) ? bwd_q_mma_kernel<D, true> : bwd_q_mma_kernel<D, false>;
  cudaError_t e = cudaFuncSetAttribute(kern1, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem1);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(kern1, cudaFuncAttributePreferredSharedMemoryCarveout, (int)cudaSharedmemCarveoutMaxShared);
  if (e != cudaSuccess) return e;
  kern1<<<dim3((n1 + kQWarps - 1) / kQWarps, BH), kQWarps * 32, smem1, s>>>(maps[0], maps[1], maps[2], maps[3], p,
                                                                            nct);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  // pass 2
  e = launch_coarse_reduce(p, s);
  if (e != cudaSuccess) return e;
  // pass 3 on tcgen05 (D = 64) when asked for
  if (tc_kv && bwd_kv_tc_supported(p)) return launch_bwd_kv_tc(p, maps, s);
  // pass 3: persistent single-warp CTAs, as many as fit at once
  const size_t smem3 = 1024 + (size_t)2 * TILE * (1 + kRingKV) + kRingKV * 128 +
                       (size_t)2 * (p.L - 1) * 2 * D * sizeof(float);
  e = cudaFuncSetAttribute(bwd_kv_mma_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem3);
  if (e != cudaSuccess) return e;
  // the occupancy query below assumes the carveout preference: ask for all of it
  e = cudaFuncSetAttribute(bwd_kv_mma_kernel<D>, cudaFuncAttributePreferredSharedMemoryCarveout, (int)cudaSharedmemCarveoutMaxShared);
  if (e != cudaSuccess) return e;
  int dev = 0, nsm = 0, per_sm = 0;
  e = cudaGetDevice(&dev);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev);
  if (e == cudaSuccess) e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, bwd_kv_mma_kernel<D>, 32, smem3);
  if (e != cudaSuccess) return e;
  const long items = (long)BH * n1;
  const int grid3 = (int)std::min<long>(items, (long)nsm * std::max(per_sm, 1));
  bwd_kv_mma_kernel<D><<<grid3, 32, smem3, s>>>(maps[0], maps[1], maps[2], maps[3], p);
  return cudaGetLastError();
}

}  // namespace

// maps: Q, K, V, dO as 2D [B*H*N rows, D cols] bf16 tile maps (16 x 64, 128B swizzle).
cudaError_t launch_attn_bwd_mma(const AttnParams& p, const CUtensorMap* maps, cudaStream_t s, bool tc_kv) {
  return (p.D == 64) ? launch_typed<64>(p, maps, s, tc_kv) : launch_typed<128>(p, maps, s, tc_kv);
}

}  // namespace llsa
