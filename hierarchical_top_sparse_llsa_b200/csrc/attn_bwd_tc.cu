// Key-major backward pass (dK, dV) of the enriched sparse attention on the
// 5th-generation tensor cores (tcgen05), bf16, D = 64 (Step 4 of the
// howistudyai explainer of "Trainable Log-linear Sparse Attention for
// Efficient Diffusion Transformers"; Building Blocks: Sparse Index
// Transpose).
//
// Persistent CTAs of 4 warps take 16-token key blocks c from a work counter.
// The query blocks in c's row of the level-1 key-major lists are processed
// in groups of 8 (128 query rows, the M of one MMA); their Q and dO tiles
// arrive by 2D TMA loads (128-byte swizzle, no multicast) into one of two
// stages, the slots past the row's end as zero-filled out-of-range boxes.
// Per group:
//   S  = Q_g K_c^T, dP = dO_g V_c^T   (M 128, N 16, K 64) into tensor memory;
//   128 threads, one per query row, read their S and dP rows (tcgen05.ld),
//   form P = w e^{S - LSE} and dS = P (dP - Delta) and write
//   B = [P_hi | P_lo | dS_hi | dS_lo]  (the bf16 hi + lo split of each, one
//   128-byte row per query) to shared memory;
//   C += [dO_g^T ; Q_g^T] B            (M 128 = two 64-row halves, N 64,
//   K 128) accumulated in tensor memory over the row's groups.
// dV^T is the sum of C's (dO^T, P_hi) and (dO^T, P_lo) quadrants, dK^T that
// of its (Q^T, dS_hi) and (Q^T, dS_lo) quadrants; the other two quadrants
// are computed and discarded (one MMA instead of four of a quarter size).
// Both operands of the last MMA are MN-major: the Q/dO tiles as loaded and
// the B rows as written.  The epilogue adds each coarse gradient / 16^l and
// stores dK, dV.  The next key block's K/V, coarse rows and first group are
// loaded while the current one finishes.  No atomics touch the results; the
// sums run in a fixed order, so results are identical from run to run.

#include <math.h>

#include <algorithm>

#include "llsa_internal.cuh"
#include "sm100_ptx.cuh"
#include "tcgen05.cuh"

namespace llsa {

namespace {

constexpr int kD = 64;
constexpr int kTile = 32 * kD;          // one 16-row bf16 tile (2 KB)
constexpr int kGroup = 8;               // query blocks per group (128 rows)
constexpr int kThreads = 128;           // one per query row
constexpr uint32_t kTmemCols = 128;     // S 0..15, dP 16..31, C 32..95
constexpr float kLog2e = 1.4426950408889634f;

// shared memory (bytes from a 1024-aligned base)
constexpr int kStageBytes = 2 * kGroup * kTile;            // dO_g | Q_g (16 KB each)
constexpr int kOffStage = 0;                               // 2 stages
constexpr int kOffK = kOffStage + 2 * kStageBytes;         // K_c
constexpr int kOffV = kOffK + kTile;                       // V_c
constexpr int kOffB = kOffV + kTile;                       // 128 rows x 128 B
constexpr int kOffSide = kOffB + kGroup * kTile;           // 2 x (LSE[128], Delta[128])
constexpr int kOffCoarse = kOffSide + 2 * 2 * 128 * 4;     // 2 x (L-1) rows of 2D fp32
constexpr int kCoarseRow = 2 * kD * 4;

struct BwdTcShared {
  uint64_t bar_ld[2];  // a stage's Q/dO tiles and LSE/Delta
  uint64_t bar_kv;     // K_c, V_c and the coarse rows
  uint64_t bar_s;      // S and dP of a group are in tensor memory
  uint64_t bar_c;      // C accumulation of a group has finished
  uint32_t tmem_base;
  int item;            // broadcast of the next work item
};

struct Row {
  int item, bh, c, beg, nq;
};

__device__ __forceinline__ uint32_t b_row_chunk(int r, int j) {
  return (uint32_t)((r >> 3) * 1024 + (r & 7) * 128 + ((j ^ (r & 7)) << 4));
}

__global__ void __launch_bounds__(kThreads)
bwd_kv_tc_kernel(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
                 const __grid_constant__ CUtensorMap tv, const __grid_constant__ CUtensorMap tdo,
                 AttnParams p, int total_rows) {
  extern __shared__ unsigned char smem_raw[];
  unsigned char* sm = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  __shared__ BwdTcShared S;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int n1 = p.N >> 4;
  const int items = p.B * p.H * n1;
  const int K = p.K, L = p.L;
  const uint32_t base = smem_u32(sm);
  const uint32_t b_ld0 = smem_u32(&S.bar_ld[0]), b_kv = smem_u32(&S.bar_kv);
  const uint32_t b_s = smem_u32(&S.bar_s), b_c = smem_u32(&S.bar_c);

  if (warp == 0) {
    tmem_alloc(smem_u32(&S.tmem_base), kTmemCols);
    tmem_relinquish();
  }
  if (tid == 0) {
    mbar_init(b_ld0, 1);
    mbar_init(b_ld0 + 8, 1);
    mbar_init(b_kv, 1);
    mbar_init(b_s, 1);
    mbar_init(b_c, 1);
    fence_mbar_init();
    S.item = atomicAdd(p.work, 1);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t taddr = S.tmem_base;
  const uint32_t t_s = taddr, t_c = taddr + 32;
  const uint32_t t_row = (uint32_t)(warp * 32) << 16;  // this warp's TMEM lanes
  const uint32_t idesc1 = idesc_bf16_f32(128, 16, 0);
  const uint32_t idesc3 = idesc_bf16_f32(128, 64, 1, 1);
  const float sc2 = p.scale * kLog2e;

  auto row_of = [&](int item) {
    Row R;
    R.item = item;
    R.bh = 0, R.c = 0, R.beg = 0, R.nq = 0;
    if (item < items) {
      R.bh = item / n1;
      R.c = item - R.bh * n1;
      const int32_t* rp = p.row_ptr[1] + (size_t)R.bh * (n1 + 1);
      R.beg = rp[R.c];
      R.nq = rp[R.c + 1] - R.beg;
    }
    return R;
  };
  // (warp 1, all lanes) group g of row R into stage st: lane 8k + s issues
  // copy k of slot s (dO tile, Q tile, LSE, Delta); slots past the row's end
  // get zero-filled boxes from outside the tensor, so every product stays finite
  auto issue_group = [&](const Row& R, int g, int st) {
    const uint32_t bar = b_ld0 + 8u * st;
    const int nslot = min(kGroup, R.nq - kGroup * g);
    const int s = lane & 7, kind = lane >> 3;
    const bool valid = s < nslot;
    const int qb = valid ? p.col[1][(size_t)R.bh * n1 * K + R.beg + kGroup * g + s] : 0;
    if (lane == 0) mbar_arrive_expect_tx(bar, 2u * kGroup * kTile + 128u * (uint32_t)nslot);
    __syncwarp();
    const uint32_t sb = base + kOffStage + (uint32_t)st * kStageBytes;  // dO_g | Q_g
    const uint32_t side = base + kOffSide + (uint32_t)st * 1024;          // LSE[128] | Delta[128]
    const size_t row0 = (size_t)R.bh * p.N + (size_t)qb * 16;
    const int y = valid ? (int)row0 : total_rows;
    if (kind == 0) tma_load_2d(sb + s * kTile, &tdo, 0, y, bar);
    else if (kind == 1) tma_load_2d(sb + (kGroup + s) * kTile, &tq, 0, y, bar);
    else if (valid) bulk_load(side + (kind - 2) * 512 + s * 64, (kind == 2 ? p.lse_in : p.delta) + row0, 64, bar);
  };
  // (warp 1, all lanes) K_c, V_c (non-empty rows) and the coarse rows into set `par`
  auto issue_kv = [&](const Row& R, int par) {
    if (lane == 0) mbar_arrive_expect_tx(b_kv, (R.nq > 0 ? 2u * kTile : 0u) + (uint32_t)(L - 1) * kCoarseRow);
    __syncwarp();
    const int y = (int)((size_t)R.bh * p.N + (size_t)R.c * 16);
    if (lane == 0 && R.nq > 0) tma_load_2d(base + kOffK, &tk, 0, y, b_kv);
    if (lane == 1 && R.nq > 0) tma_load_2d(base + kOffV, &tv, 0, y, b_kv);
    const int l = lane;  // lanes 2..L: level l
    if (l >= 2 && l <= L) {
      const size_t tc = (size_t)R.bh * (p.N >> (4 * l)) + (R.c >> (4 * (l - 1)));
      bulk_load(base + kOffCoarse + (uint32_t)(par * (L - 1) + (l - 2)) * kCoarseRow, p.coarse[l] + tc * 2 * kD,
                kCoarseRow, b_kv);
    }
  };

  // A bounded wait that gives up only records it; the block stops together
  // at its next barrier (__syncthreads_or), so control flow stays uniform.
  bool fail = false;
  auto wait = [&](uint32_t bar, uint32_t parity) {
    const bool w = mbar_wait_bounded(bar, parity);
    fail |= !w;
    return w;
  };

  Row cur = row_of(S.item);
  int stage = 0, par = 0;
  uint32_t ldph = 0, kvph = 0, sph = 0, cph = 0;
  bool ld_pend[2] = {false, false};
  bool kv_pend = false, s_pend = false, c_pend = false;
  if (warp == 1 && cur.item < items) {
    issue_kv(cur, par);
    if (cur.nq > 0) issue_group(cur, 0, stage);
  }
  if (cur.item < items) {
    kv_pend = true;
    ld_pend[stage] = cur.nq > 0;
  }
  __syncthreads();  // everyone has read S.item
  int nxt_l0 = (tid == 0) ? atomicAdd(p.work, 1) : 0;
  bool stop = false;
  while (cur.item < items) {
    if (tid == 0) S.item = nxt_l0;
    if (__syncthreads_or(fail)) { stop = true; break; }
    const Row nxt = row_of(S.item);  // S.item is next written after the barriers below
    nxt_l0 = (tid == 0) ? atomicAdd(p.work, 1) : 0;  // the item after nxt, in flight
    const int ng = (cur.nq + kGroup - 1) / kGroup;
    if (wait(b_kv, kvph)) {
      kvph ^= 1u;
      kv_pend = false;
    }
    // every thread has waited on this phase of b_kv before warp 1 arms the
    // next one (a waiter two phases behind would wait for the wrong phase)
    if (__syncthreads_or(fail)) { stop = true; break; }
    const int nxt_stage = (stage + ng) & 1;
    if (ng == 0) {  // nothing of this row in flight: the next row's loads go out now
      if (warp == 1 && nxt.item < items) {
        issue_kv(nxt, par ^ 1);
        if (nxt.nq > 0) issue_group(nxt, 0, nxt_stage);
      }
      if (nxt.item < items) {
        kv_pend = true;
        ld_pend[nxt_stage] = nxt.nq > 0;
      }
    }
    for (int g = 0; g < ng; ++g) {
      const int st = (stage + g) & 1;
      if (wait(b_ld0 + 8u * st, (ldph >> st) & 1u)) {
        ldph ^= 1u << st;
        ld_pend[st] = false;
      }
      const uint32_t sb = base + kOffStage + (uint32_t)st * kStageBytes;
      // S = Q_g K_c^T, dP = dO_g V_c^T
      if (tid == 0) {
        tc_fence_after();
#pragma unroll
        for (int ks = 0; ks < kD / 16; ++ks)
          tc_mma_f16(t_s, smem_desc_sw128(sb + kGroup * kTile + ks * 32, 16, 1024),
                     smem_desc_sw128(base + kOffK + ks * 32, 16, 1024), idesc1, ks > 0);
#pragma unroll
        for (int ks = 0; ks < kD / 16; ++ks)
          tc_mma_f16(t_s + 16, smem_desc_sw128(sb + ks * 32, 16, 1024),
                     smem_desc_sw128(base + kOffV + ks * 32, 16, 1024), idesc1, ks > 0);
        tc_commit(b_s);
      }
      s_pend = true;
      if (wait(b_s, sph)) {
        sph ^= 1u;
        s_pend = false;
      }
      if (g > 0 && wait(b_c, cph)) {  // the previous group's accumulation finished before S was written
        cph ^= 1u;
        c_pend = false;
      }
      tc_fence_after();
      // loads for what follows: this row's next group, or the next row
      if (warp == 1) {
        if (g + 1 < ng) {
          issue_group(cur, g + 1, st ^ 1);
        } else if (nxt.item < items) {
          issue_kv(nxt, par ^ 1);
          if (nxt.nq > 0) issue_group(nxt, 0, st ^ 1);
        }
      }
      if (g + 1 < ng) {
        ld_pend[st ^ 1] = true;
      } else if (nxt.item < items) {
        kv_pend = true;
        ld_pend[st ^ 1] = nxt.nq > 0;
      }
      // P and dS of this thread's query row -> B row (bf16 hi, lo)
      {
        const int r = tid;
        const int nslot = min(kGroup, cur.nq - kGroup * g);
        const bool valid = (r >> 4) < nslot;
        float x[32];
        tmem_ld32(t_s + t_row, x);
        tmem_wait_ld();
        const float* side = reinterpret_cast<const float*>(sm + kOffSide + st * 1024);
        float nl = -INFINITY, del = 0.f;
        if (valid) {
          const float l2 = side[r] * kLog2e;
          nl = (l2 == -INFINITY) ? -INFINITY : -l2;
          del = side[128 + r];
        }
        uint32_t hp[8], lp[8], hd[8], ld[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const float p0 = ex2_approx(fmaf(x[2 * j], sc2, nl));
          const float p1 = ex2_approx(fmaf(x[2 * j + 1], sc2, nl));
          const float d0 = p0 * (x[16 + 2 * j] - del);
          const float d1 = p1 * (x[16 + 2 * j + 1] - del);
          const __nv_bfloat162 ph2 = __floats2bfloat162_rn(p0, p1);
          const __nv_bfloat162 dh2 = __floats2bfloat162_rn(d0, d1);
          const float2 phf = __bfloat1622float2(ph2), dhf = __bfloat1622float2(dh2);
          hp[j] = *reinterpret_cast<const uint32_t*>(&ph2);
          hd[j] = *reinterpret_cast<const uint32_t*>(&dh2);
          lp[j] = pack_bf16(p0 - phf.x, p1 - phf.y);
          ld[j] = pack_bf16(d0 - dhf.x, d1 - dhf.y);
        }
        unsigned char* brow = sm + kOffB;
        *reinterpret_cast<uint4*>(brow + b_row_chunk(r, 0)) = make_uint4(hp[0], hp[1], hp[2], hp[3]);
        *reinterpret_cast<uint4*>(brow + b_row_chunk(r, 1)) = make_uint4(hp[4], hp[5], hp[6], hp[7]);
        *reinterpret_cast<uint4*>(brow + b_row_chunk(r, 2)) = make_uint4(lp[0], lp[1], lp[2], lp[3]);
        *reinterpret_cast<uint4*>(brow + b_row_chunk(r, 3)) = make_uint4(lp[4], lp[5], lp[6], lp[7]);
        *reinterpret_cast<uint4*>(brow + b_row_chunk(r, 4)) = make_uint4(hd[0], hd[1], hd[2], hd[3]);
        *reinterpret_cast<uint4*>(brow + b_row_chunk(r, 5)) = make_uint4(hd[4], hd[5], hd[6], hd[7]);
        *reinterpret_cast<uint4*>(brow + b_row_chunk(r, 6)) = make_uint4(ld[0], ld[1], ld[2], ld[3]);
        *reinterpret_cast<uint4*>(brow + b_row_chunk(r, 7)) = make_uint4(ld[4], ld[5], ld[6], ld[7]);
      }
      fence_proxy_async_smem();
      tc_fence_before();
      if (__syncthreads_or(fail)) { stop = true; break; }
      // C += [dO_g^T ; Q_g^T] B: A is MN-major (the two 64-row halves are the
      // dO_g and Q_g tiles, 16 KB apart), B is MN-major (one row per query)
      if (tid == 0) {
        tc_fence_after();
#pragma unroll
        for (int ks = 0; ks < kGroup; ++ks)
          tc_mma_f16(t_c, smem_desc_sw128(sb + ks * 2048, kGroup * kTile, 1024),
                     smem_desc_sw128(base + kOffB + ks * 2048, 16, 1024), idesc3, (g > 0 || ks > 0));
        tc_commit(b_c);
      }
      c_pend = true;
    }
    if (stop) break;
    if (ng > 0 && wait(b_c, cph)) {
      cph ^= 1u;
      c_pend = false;
    }
    tc_fence_after();
    // epilogue: warps 0-1 hold dV^T rows (d = lane + 32 (warp & 1)), warps 2-3
    // dK^T rows; columns: key of the hi part, then of the lo part
    {
      const int kv = (warp < 2) ? 1 : 0;
      const int d = (warp & 1) * 32 + lane;
      float acc[32];
      if (ng > 0) {
        tmem_ld32(t_c + t_row + (kv ? 0u : 32u), acc);
        tmem_wait_ld();
      } else {
#pragma unroll
        for (int j = 0; j < 32; ++j) acc[j] = 0.f;
      }
      float cg = 0.f;
      for (int l = 2; l <= L; ++l) {
        const float* crow = reinterpret_cast<const float*>(sm + kOffCoarse + (par * (L - 1) + (l - 2)) * kCoarseRow);
        cg += crow[kv * kD + d] * (1.0f / (float)(1u << (4 * l)));
      }
      const float f = kv ? 1.f : p.scale;
      bf16* out = static_cast<bf16*>(kv ? p.dv : p.dk) + ((size_t)cur.bh * p.N + (size_t)cur.c * 16) * kD + d;
#pragma unroll
      for (int key = 0; key < 16; ++key) out[(size_t)key * kD] = __float2bfloat16_rn((acc[key] + acc[16 + key]) * f + cg);
    }
    fence_proxy_async_smem();  // the coarse rows read above are reloaded by bulk copies
    tc_fence_before();
    if (__syncthreads_or(fail)) { stop = true; break; }  // coarse set `par` and C are reused
    tc_fence_after();
    stage = nxt_stage;
    par ^= 1;
    cur = nxt;
  }
  if (stop) {
    // let every copy and MMA still in flight finish before the CTA exits
    if (kv_pend) mbar_wait_bounded(b_kv, kvph);
    for (int st = 0; st < 2; ++st)
      if (ld_pend[st]) mbar_wait_bounded(b_ld0 + 8u * st, (ldph >> st) & 1u);
    if (s_pend) mbar_wait_bounded(b_s, sph);
    if (c_pend) mbar_wait_bounded(b_c, cph);
    if (tid == 0) report_status(p.status, LLSA_DEV_TIMEOUT);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(taddr, kTmemCols);
  }
}

}  // namespace

bool bwd_kv_tc_supported(const AttnParams& p) { return p.D == kD; }

// maps: Q, K, V, dO as 2D [B*H*N rows, 64 cols] bf16, box 16 x 64, 128-byte swizzle.
cudaError_t launch_bwd_kv_tc(const AttnParams& p, const CUtensorMap* maps, cudaStream_t s) {
  const size_t smem = 1024 + kOffCoarse + (size_t)2 * (p.L - 1) * kCoarseRow;
  cudaError_t e = cudaFuncSetAttribute(bwd_kv_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  // the occupancy query below assumes the carveout preference: ask for all of it
  e = cudaFuncSetAttribute(bwd_kv_tc_kernel, cudaFuncAttributePreferredSharedMemoryCarveout, (int)cudaSharedmemCarveoutMaxShared);
  if (e != cudaSuccess) return e;
  int dev = 0, nsm = 0, smem_sm = 0, reserved = 0;
  e = cudaGetDevice(&dev);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&smem_sm, cudaDevAttrMaxSharedMemoryPerMultiprocessor, dev);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&reserved, cudaDevAttrReservedSharedMemoryPerBlock, dev);
  if (e != cudaSuccess) return e;
  const long items = (long)p.B * p.H * (p.N / kBlock);
  // CTAs per SM: what shared memory holds, at most 4 (4 x 128 tensor-memory
  // columns fill the 512 of an SM)
  const int per_sm = (int)((size_t)smem_sm / (smem + sizeof(BwdTcShared) + 64 + (size_t)reserved));
  const int per = std::min(std::max(per_sm, 1), 4);
  const int grid = (int)std::min<long>(items, (long)nsm * per);
  const int total_rows = p.B * p.H * p.N;
  bwd_kv_tc_kernel<<<grid, kThreads, smem, s>>>(maps[0], maps[1], maps[2], maps[3], p, total_rows);
  return cudaGetLastError();
}

}  // namespace llsa
