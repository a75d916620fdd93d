// Hierarchical Top-K selection of one group of sibling query tokens: the
// shared body of the per-level selection kernel and of the forward kernel
// that selects level 1 in its prologue.
//
// Selection runs level by level, coarsest first.  A CTA owns the 16 sibling query
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

#pragma once

#include "llsa_internal.cuh"
#include "sm100_ptx.cuh"

namespace llsa {

constexpr int kSelQ = 16;        // sibling query tokens per CTA
constexpr int kSelWarps = 4;
constexpr int kSelThreads = kSelWarps * 32;
constexpr int kSelChunk = 128;   // candidates scored per pass
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

// Shared-memory scratch that select_group needs (16-byte aligned).
template <int D>
constexpr size_t select_scratch_bytes() {
  return (size_t)(D * kSelQ + D * (kSelChunk + 4)) * sizeof(float) + kSelChunk * sizeof(int);
}

// The selection of one group of kSelQ query tokens (group grp of head bh):
// all kSelThreads threads of the CTA call it; `scratch` is
// select_scratch_bytes<D>() of shared memory that it may overwrite.  Rows of
// p.out are written by the CTA's own threads, so they may be read back by the
// CTA after a __syncthreads().
template <int D>
__device__ __forceinline__ void select_group(const SelectParams& p, int bh, int grp, float* scratch) {
  constexpr int QLD = kSelQ;            // queries per CTA, row stride of qsT
  constexpr int CLD = kSelChunk + 4;    // row stride of ksT (floats)
  float* qsT = scratch;                            // [D][16] queries, transposed
  float* ksT = qsT + D * QLD;                     // [D][CLD] candidates, transposed
  float* sc = ksT;                                // [16][kSelChunk] scores of a chunk (over ksT)
  int* cid = reinterpret_cast<int*>(ksT + D * CLD);  // [kSelChunk]
  __shared__ int parents[kMaxK];
  __shared__ int n_par;

  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  const int n = p.n;
  const int K = p.K;
  const bool top = (p.parent == nullptr);

  if (warp == 0) {
    int m = 0;
    if (!top) {
      const int np = n / kBlock;
      int f = 0;
      const int Kp = p.Kp;  // the parent row's width
      const int c = (lane < Kp) ? p.parent[((size_t)bh * np + grp) * Kp + lane] : -1;
      const bool u = warp_row_used(c, lane, np, lane < Kp, f);
      const unsigned msk = __ballot_sync(0xffffffffu, u);
      if (u) parents[__popc(msk & ((1u << lane) - 1u))] = c;
      m = __popc(msk);
    }
    if (lane == 0) n_par = m;
  }
  // the 16 query rows, transposed
  const float* qbase = p.ql + ((size_t)bh * n + (size_t)grp * kSelQ) * D;
  for (int e = tid; e < kSelQ * (D / 4); e += kSelThreads) {
    const int r = e % kSelQ, c4 = e / kSelQ;  // lanes walk the rows: conflict-free stores
    float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
    if (grp * kSelQ + r < n) v = *reinterpret_cast<const float4*>(qbase + (size_t)r * D + c4 * 4);
    qsT[(4 * c4 + 0) * QLD + r] = v.x;
    qsT[(4 * c4 + 1) * QLD + r] = v.y;
    qsT[(4 * c4 + 2) * QLD + r] = v.z;
    qsT[(4 * c4 + 3) * QLD + r] = v.w;
  }
  __syncthreads();
  const int C = top ? n : n_par * kBlock;
  // this thread's 4 x 4 block of (query, candidate) scores
  const int qg = tid >> 5;        // queries 4qg .. 4qg+3
  const int cg = tid & 31;        // candidates 4cg .. 4cg+3 of a chunk

  uint64_t run[kSelQ / kSelWarps];  // per warp query: lane r < K holds its r-th best
#pragma unroll
  for (int i = 0; i < kSelQ / kSelWarps; ++i) run[i] = 0;
  const float* kbase = p.kl + (size_t)bh * n * D;
  for (int c0 = 0; c0 < C; c0 += kSelChunk) {
    const int cn = min(kSelChunk, C - c0);
    __syncthreads();
    // all of this thread's row loads are issued before any is stored, so
    // their latencies overlap
    constexpr int kStageIters = kSelChunk * (D / 4) / kSelThreads;
    float4 kv4[kStageIters];
#pragma unroll
    for (int it = 0; it < kStageIters; ++it) {
      const int e = tid + it * kSelThreads;
      const int r = e % kSelChunk, c4 = e / kSelChunk;
      kv4[it] = make_float4(0.f, 0.f, 0.f, 0.f);
      if (r < cn) {
        const int j = c0 + r;
        const int c = top ? j : parents[j / kBlock] * kBlock + (j % kBlock);
        kv4[it] = *reinterpret_cast<const float4*>(kbase + (size_t)c * D + c4 * 4);
        if (c4 == 0) cid[r] = c;
      }
    }
#pragma unroll
    for (int it = 0; it < kStageIters; ++it) {
      const int e = tid + it * kSelThreads;
      const int r = e % kSelChunk, c4 = e / kSelChunk;
      ksT[(4 * c4 + 0) * CLD + r] = kv4[it].x;
      ksT[(4 * c4 + 1) * CLD + r] = kv4[it].y;
      ksT[(4 * c4 + 2) * CLD + r] = kv4[it].z;
      ksT[(4 * c4 + 3) * CLD + r] = kv4[it].w;
    }
    __syncthreads();
    // scores: d = 0..D-1 in order, one rounding per multiply and per add;
    // acc[a][h] holds candidates 4cg + 2h, 4cg + 2h + 1 of query 4qg + a
    uint64_t acc[4][2];
#pragma unroll
    for (int d = 0; d < D; ++d) {
      const float4 qv = *reinterpret_cast<const float4*>(qsT + d * QLD + 4 * qg);
      const float4 kv = *reinterpret_cast<const float4*>(ksT + d * CLD + 4 * cg);
      const uint64_t k01 = f2_make(kv.x, kv.y), k23 = f2_make(kv.z, kv.w);
      const float qq[4] = {qv.x, qv.y, qv.z, qv.w};
#pragma unroll
      for (int a = 0; a < 4; ++a) {
        const uint64_t q2 = f2_make(qq[a], qq[a]);
        const uint64_t m01 = f2_mul(q2, k01), m23 = f2_mul(q2, k23);
        acc[a][0] = (d == 0) ? m01 : f2_add(acc[a][0], m01);
        acc[a][1] = (d == 0) ? m23 : f2_add(acc[a][1], m23);
      }
    }
    __syncthreads();  // every thread is done with ksT, which the scores overwrite
#pragma unroll
    for (int a = 0; a < 4; ++a) {
      const float2 lo = f2_split(acc[a][0]), hi = f2_split(acc[a][1]);
      const float4 o = make_float4(lo.x, lo.y, hi.x, hi.y);
      *reinterpret_cast<float4*>(sc + (4 * qg + a) * kSelChunk + 4 * cg) = o;
    }
    __syncthreads();
    // Top-K merge: the warp's queries advance together, so their K rounds of
    // warp-wide maxima are independent chains
    constexpr int QW = kSelQ / kSelWarps;
    uint64_t item[QW][kSelItems + 1];
#pragma unroll
    for (int qi = 0; qi < QW; ++qi) {
      const int ql = warp * QW + qi;
#pragma unroll
      for (int it = 0; it < kSelItems; ++it) {
        const int j = lane + 32 * it;
        item[qi][it] = (j < cn) ? pack_key(sc[ql * kSelChunk + j], cid[j]) : 0;
      }
      item[qi][kSelItems] = (lane < K) ? run[qi] : 0;
    }
    uint64_t next[QW];
#pragma unroll
    for (int qi = 0; qi < QW; ++qi) next[qi] = 0;
    for (int r = 0; r < K; ++r) {
#pragma unroll
      for (int qi = 0; qi < QW; ++qi) {
        uint64_t mine = 0;
        int arg = 0;
#pragma unroll
        for (int it = 0; it <= kSelItems; ++it)
          if (item[qi][it] > mine) {
            mine = item[qi][it];
            arg = it;
          }
        const uint64_t best = warp_max_u64(mine);  // 0: no candidates left
        if (best != 0 && mine == best) {
#pragma unroll
          for (int it = 0; it <= kSelItems; ++it)
            if (it == arg) item[qi][it] = 0;
        }
        if (lane == r) next[qi] = best;
      }
    }
#pragma unroll
    for (int qi = 0; qi < QW; ++qi) run[qi] = next[qi];
  }
  // ascending index order; the kept entries are lanes 0..cnt-1
#pragma unroll
  for (int qi = 0; qi < kSelQ / kSelWarps; ++qi) {
    const int q = grp * kSelQ + warp * (kSelQ / kSelWarps) + qi;
    const bool valid = (lane < K) && (run[qi] != 0);
    const int id = valid ? (int)(~(uint32_t)run[qi]) : 0x7fffffff;
    int pos = 0;
    for (int r = 0; r < K; ++r) {
      const int other = __shfl_sync(0xffffffffu, id, r);
      pos += (other < id) ? 1 : 0;
    }
    if (q < n && lane < K) {
      int32_t* orow = p.out + ((size_t)bh * n + q) * K;
      if (valid) orow[pos] = id;
      else orow[lane] = -1;  // unfilled rounds are the last K - cnt lanes
    }
  }
}

}  // namespace llsa
