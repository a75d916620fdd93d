// Warp-level tile products shared by the bf16 attention kernels.  A "tile"
// is 16 rows x D bf16 in shared memory as written by a 2D TMA load with
// 128-byte swizzle (see swz()); fragments follow the m16n8k16 layouts.
#pragma once

#include "sm100_ptx.cuh"

namespace llsa {

// A fragments of a 16 x D tile (rows = M, columns = K of the MMA).
template <int D>
__device__ __forceinline__ void load_a_frags(uint32_t tile, int lane, uint32_t (&a)[D / 16][4]) {
  const int mi = lane >> 3;
  const int row = (mi & 1) * 8 + (lane & 7);
#pragma unroll
  for (int kk = 0; kk < D / 16; ++kk)
    ldsm_x4(tile + swz(row, 2 * kk + (mi >> 1)), a[kk][0], a[kk][1], a[kk][2], a[kk][3]);
}

// S (16 x 16) = A (16 x D, A fragments) . T^T for a 16-row tile T at `kt`
// (shared address): rows of T are the 16 output columns.
template <int D>
__device__ __forceinline__ void qk_tile(const uint32_t (&qa)[D / 16][4], uint32_t kt, int lane,
                                        float (&s)[2][4]) {
  const int mi = lane >> 3;
  const int krow = (mi >> 1) * 8 + (lane & 7);
  const int kc = mi & 1;
#pragma unroll
  for (int nt = 0; nt < 2; ++nt)
#pragma unroll
    for (int e = 0; e < 4; ++e) s[nt][e] = 0.f;
#pragma unroll
  for (int kk = 0; kk < D / 16; ++kk) {
    uint32_t b0, b1, b2, b3;
    ldsm_x4(kt + swz(krow, 2 * kk + kc), b0, b1, b2, b3);
    mma_bf16(s[0], qa[kk], b0, b1);
    mma_bf16(s[1], qa[kk], b2, b3);
  }
}

// The same with the A operand read from a 16-row tile `at` in shared memory
// (fragments loaded per k-step instead of held in registers).
template <int D>
__device__ __forceinline__ void qk_tile_ss(uint32_t at, uint32_t kt, int lane, float (&s)[2][4]) {
  const int mi = lane >> 3;
  const int arow = (mi & 1) * 8 + (lane & 7);
  const int ac = mi >> 1;
  const int krow = (mi >> 1) * 8 + (lane & 7);
  const int kc = mi & 1;
#pragma unroll
  for (int nt = 0; nt < 2; ++nt)
#pragma unroll
    for (int e = 0; e < 4; ++e) s[nt][e] = 0.f;
#pragma unroll
  for (int kk = 0; kk < D / 16; ++kk) {
    uint32_t a[4], b0, b1, b2, b3;
    ldsm_x4(at + swz(arow, 2 * kk + ac), a[0], a[1], a[2], a[3]);
    ldsm_x4(kt + swz(krow, 2 * kk + kc), b0, b1, b2, b3);
    mma_bf16(s[0], a, b0, b1);
    mma_bf16(s[1], a, b2, b3);
  }
}

// O (16 x D) += P (16 x 16, A fragment) . T (16 x D tile at vt): rows of T
// are the contraction index.
template <int D>
__device__ __forceinline__ void pv_tile(const uint32_t (&pa)[4], uint32_t vt, int lane,
                                        float (&o)[D / 8][4]) {
  const int mi = lane >> 3;
  const int vrow = (mi & 1) * 8 + (lane & 7);
  const int vc = mi >> 1;
#pragma unroll
  for (int nn = 0; nn < D / 16; ++nn) {
    uint32_t b0, b1, b2, b3;
    ldsm_x4_t(vt + swz(vrow, 2 * nn + vc), b0, b1, b2, b3);
    mma_bf16(o[2 * nn], pa, b0, b1);
    mma_bf16(o[2 * nn + 1], pa, b2, b3);
  }
}

// O (16 x D) += (Ph + Pl) . T: a 16x16 fp32 matrix split into two bf16
// parts (hi = round(x), lo = round(x - hi)) so that the product keeps about
// 16 mantissa bits of x; the B fragments of T are loaded once for both.
template <int D>
__device__ __forceinline__ void pv_tile2(const uint32_t (&ph)[4], const uint32_t (&pl)[4], uint32_t vt,
                                         int lane, float (&o)[D / 8][4]) {
  const int mi = lane >> 3;
  const int vrow = (mi & 1) * 8 + (lane & 7);
  const int vc = mi >> 1;
#pragma unroll
  for (int nn = 0; nn < D / 16; ++nn) {
    uint32_t b0, b1, b2, b3;
    ldsm_x4_t(vt + swz(vrow, 2 * nn + vc), b0, b1, b2, b3);
    mma_bf16(o[2 * nn], ph, b0, b1);
    mma_bf16(o[2 * nn + 1], ph, b2, b3);
    mma_bf16(o[2 * nn], pl, b0, b1);
    mma_bf16(o[2 * nn + 1], pl, b2, b3);
  }
}

// hi/lo bf16 split of an accumulator-layout 16x16 tile into A fragments.
__device__ __forceinline__ void split_frag(const float (&x)[2][4], uint32_t (&hi)[4], uint32_t (&lo)[4]) {
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int nt = i >> 1, e = (i & 1) * 2;  // a0: nt0 e0/1, a1: nt0 e2/3, a2: nt1 e0/1, a3: nt1 e2/3
    const __nv_bfloat162 h = __floats2bfloat162_rn(x[nt][e], x[nt][e + 1]);
    const float2 hf = __bfloat1622float2(h);
    hi[i] = *reinterpret_cast<const uint32_t*>(&h);
    lo[i] = pack_bf16(x[nt][e] - hf.x, x[nt][e + 1] - hf.y);
  }
}

}  // namespace llsa
