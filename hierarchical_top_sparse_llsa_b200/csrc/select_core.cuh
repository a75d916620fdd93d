// Hierarchical Top-K selection of one group of sibling query tokens: the
// shared body of the per-level selection kernel and of the forward kernel
// that selects level 1 in its prologue.
//
// Selection runs level by level, coarsest first.  A CTA owns the 16 sibling
// query tokens under one parent (level l < L), or 16 consecutive query tokens
// at the top level, so they share one candidate list: the children of the
// keys their parent kept, or every top-level key.  The query rows and the
// candidate K(l) rows (in chunks of 128) are copied into shared memory by
// coalesced 16-byte asynchronous copies, row-major with rows padded to D + 4
// floats.  Thread (warp w, lane c) scores queries 4w..4w+3 against
// candidates c, c+32, c+64, c+96 of the chunk: the four candidate rows of a
// quarter warp sit in distinct banks, the query rows are broadcast, and the
// 16 scores are exactly the items the lane holds for those queries in the
// Top-K below, so they never leave registers.
//
// Score: fp32, d = 0..D-1 left to right, one rounding per multiply and per
// add (no contraction into FMA), so scores are reproducible bit for bit and
// the selected indices are exact.  The products and sums run as packed pairs
// (sm_100 mul/add .f32x2: each half rounded exactly as the scalar .rn op),
// two candidates per instruction.
// Top-K: each (score, index) pair is packed into one 64-bit key that orders
// by score (with -0 == +0) and then by lower index.  Each lane sorts its four
// keys of a query (and the one it holds of the best K of earlier chunks)
// descending; K rounds of a warp-wide maximum of the lanes' heads (two
// redux.sync on 32-bit halves) pick the winners, the winning lane dropping
// its head.  Rows are then sorted ascending by index.

#pragma once

#include "llsa_internal.cuh"
#include "sm100_ptx.cuh"

namespace llsa {

constexpr int kSelQ = 16;        // sibling query tokens per CTA
constexpr int kSelWarps = 4;
constexpr int kSelThreads = kSelWarps * 32;
constexpr int kSelChunk = 128;   // candidates scored per pass

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

// Row stride (floats) of the staged query and candidate rows: rows 4 banks
// apart, so the 16-byte reads of 8 consecutive rows by a quarter warp fall in
// distinct banks.
template <int D>
__host__ __device__ constexpr int sel_row_stride() { return D + 4; }

// Shared-memory scratch that select_group needs (16-byte aligned).
template <int D>
__host__ __device__ constexpr size_t select_scratch_bytes() {
  return (size_t)(kSelQ + kSelChunk) * sel_row_stride<D>() * sizeof(float);
}

// 16-byte asynchronous global -> shared copy (zero-filled when !valid; the
// source address is then not read).
__device__ __forceinline__ void cp_async16(void* dst, const void* src, bool valid) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_u32(dst)), "l"(src),
               "r"(valid ? 16 : 0)
               : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() {
  asm volatile("cp.async.commit_group;\ncp.async.wait_group 0;" ::: "memory");
}

// u64 compare-exchange: afterwards a >= b.
__device__ __forceinline__ void cx_desc(uint64_t& a, uint64_t& b) {
  const uint64_t hi = a > b ? a : b, lo = a > b ? b : a;
  a = hi;
  b = lo;
}

// The selection of one group of kSelQ query tokens (group grp of head bh):
// all kSelThreads threads of the CTA call it; `scratch` is
// select_scratch_bytes<D>() of shared memory that it may overwrite.  Rows of
// p.out are written by the CTA's own threads, so they may be read back by the
// CTA after a __syncthreads().
template <int D>
__device__ __forceinline__ void select_group(const SelectParams& p, int bh, int grp, float* scratch) {
  constexpr int RS = sel_row_stride<D>();
  constexpr int CH = D / 4;  // 16-byte chunks per row
  float* qs = scratch;                 // [16][RS] queries
  float* ks = qs + kSelQ * RS;         // [kSelChunk][RS] candidates
  __shared__ int parents[kMaxK];
  __shared__ int n_par;

  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  const int n = p.n;
  const int K = p.K;
  const bool top = (p.parent == nullptr);

  // the 16 query rows (zero past n), in flight while the parent row is read
  const float* qbase = p.ql + ((size_t)bh * n + (size_t)grp * kSelQ) * D;
  for (int e = tid; e < kSelQ * CH; e += kSelThreads) {
    const int r = e / CH, c = e % CH;
    const bool ok = grp * kSelQ + r < n;
    cp_async16(qs + r * RS + 4 * c, ok ? qbase + (size_t)r * D + 4 * c : qbase, ok);
  }
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
  __syncthreads();
  const int C = top ? n : n_par * kBlock;
  auto cand = [&](int j) { return top ? j : parents[j / kBlock] * kBlock + (j % kBlock); };

  constexpr int QW = kSelQ / kSelWarps;  // queries of this warp: 4 * warp + a
  uint64_t run[QW];                      // lane r < K holds the r-th best so far
#pragma unroll
  for (int a = 0; a < QW; ++a) run[a] = 0;
  const float* kbase = p.kl + (size_t)bh * n * D;
  for (int c0 = 0; c0 < C; c0 += kSelChunk) {
    const int cn = min(kSelChunk, C - c0);
    if (c0 > 0) __syncthreads();  // every thread is done with the previous chunk's rows
    // candidate rows: consecutive lanes copy consecutive 16-byte chunks
    for (int e = tid; e < kSelChunk * CH; e += kSelThreads) {
      const int r = e / CH, c = e % CH;
      const bool ok = r < cn;
      const float* src = ok ? kbase + (size_t)cand(c0 + r) * D + 4 * c : kbase;
      cp_async16(ks + r * RS + 4 * c, src, ok);
    }
    cp_async_wait_all();
    __syncthreads();
    // scores: d = 0..D-1 in order, one rounding per multiply and per add;
    // acc[a][h] holds candidates lane + 64h and lane + 64h + 32 of query 4w + a
    uint64_t acc[QW][2];
    const float* qrow = qs + (size_t)(QW * warp) * RS;
    const float* krow = ks + (size_t)lane * RS;
#pragma unroll 4
    for (int d4 = 0; d4 < D; d4 += 4) {
      float4 qv[QW], kv[4];
#pragma unroll
      for (int a = 0; a < QW; ++a) qv[a] = *reinterpret_cast<const float4*>(qrow + a * RS + d4);
#pragma unroll
      for (int i = 0; i < 4; ++i) kv[i] = *reinterpret_cast<const float4*>(krow + 32 * i * RS + d4);
#pragma unroll
      for (int dd = 0; dd < 4; ++dd) {
        const float k0 = (&kv[0].x)[dd], k1 = (&kv[1].x)[dd], k2 = (&kv[2].x)[dd], k3 = (&kv[3].x)[dd];
        const uint64_t k01 = f2_make(k0, k1), k23 = f2_make(k2, k3);
#pragma unroll
        for (int a = 0; a < QW; ++a) {
          const float qq = (&qv[a].x)[dd];
          const uint64_t q2 = f2_make(qq, qq);
          const uint64_t m01 = f2_mul(q2, k01), m23 = f2_mul(q2, k23);
          acc[a][0] = (d4 + dd == 0) ? m01 : f2_add(acc[a][0], m01);
          acc[a][1] = (d4 + dd == 0) ? m23 : f2_add(acc[a][1], m23);
        }
      }
    }
    // this lane's keys of each query, sorted descending, merged with its
    // entry of the running list; K rounds of the warp-wide maximum
    int cid[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) cid[i] = (lane + 32 * i < cn) ? cand(c0 + lane + 32 * i) : -1;
    uint64_t item[QW][5];
#pragma unroll
    for (int a = 0; a < QW; ++a) {
      const float2 s01 = f2_split(acc[a][0]), s23 = f2_split(acc[a][1]);
      const float sc[4] = {s01.x, s01.y, s23.x, s23.y};
#pragma unroll
      for (int i = 0; i < 4; ++i) item[a][i] = (cid[i] >= 0) ? pack_key(sc[i], cid[i]) : 0;
      cx_desc(item[a][0], item[a][1]);
      cx_desc(item[a][2], item[a][3]);
      cx_desc(item[a][0], item[a][2]);
      cx_desc(item[a][1], item[a][3]);
      cx_desc(item[a][1], item[a][2]);
      item[a][4] = (lane < K) ? run[a] : 0;
      cx_desc(item[a][3], item[a][4]);
      cx_desc(item[a][2], item[a][3]);
      cx_desc(item[a][1], item[a][2]);
      cx_desc(item[a][0], item[a][1]);
    }
    uint64_t next[QW];
#pragma unroll
    for (int a = 0; a < QW; ++a) next[a] = 0;
    for (int r = 0; r < K; ++r) {
#pragma unroll
      for (int a = 0; a < QW; ++a) {
        const uint64_t best = warp_max_u64(item[a][0]);  // 0: no candidates left
        if (best != 0 && item[a][0] == best) {
          item[a][0] = item[a][1];
          item[a][1] = item[a][2];
          item[a][2] = item[a][3];
          item[a][3] = item[a][4];
          item[a][4] = 0;
        }
        if (lane == r) next[a] = best;
      }
    }
#pragma unroll
    for (int a = 0; a < QW; ++a) run[a] = next[a];
  }
  // ascending index order; the kept entries are lanes 0..cnt-1
#pragma unroll
  for (int a = 0; a < QW; ++a) {
    const int q = grp * kSelQ + QW * warp + a;
    const bool valid = (lane < K) && (run[a] != 0);
    const int id = valid ? (int)(~(uint32_t)run[a]) : 0x7fffffff;
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
