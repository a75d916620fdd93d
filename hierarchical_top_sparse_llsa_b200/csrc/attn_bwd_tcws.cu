// Key-major backward pass (dK, dV) on the 5th-generation tensor cores,
// warp-specialised, bf16, D = 64 (Step 4 of the howistudyai explainer of
// "Trainable Log-linear Sparse Attention for Efficient Diffusion
// Transformers"; Building Blocks: Sparse Index Transpose).
//
// The arithmetic is that of attn_bwd_tc.cu: the query blocks in a key block
// c's row of the level-1 key-major lists go in groups of 8 (128 query rows);
//   S = Q_g K_c^T, dP = dO_g V_c^T       (M 128, N 16, K 64)  -> tensor memory
//   P, dS -> B = [P_hi | P_lo | dS_hi | dS_lo]  (one 128-byte row per query)
//   C += [dO_g^T ; Q_g^T] B               (M 128, N 64, K 128) -> tensor memory
// and dV^T, dK^T are sums of C's quadrants.  Here each step runs on its own
// warps, linked by mbarrier rings, so that they overlap:
//   warp 4     producer: takes key blocks from the work counter and gathers,
//              by TMA, the groups' Q/dO tiles and LSE/Delta into 4 stages and
//              each row's K_c/V_c and coarse gradient rows into 2 row slots;
//   warp 5     MMA issuer (one thread): S/dP of group n into one of 2 tensor
//              memory buffers, then the C update of group n-1, so the tensor
//              core computes S of the next group while the softmax warps
//              work on the current one;
//   warps 0-3  softmax: one thread per query row turns S, dP into B, written
//              to one of 2 shared-memory buffers;
//   warps 6-9  epilogue: per key block, read C from one of 2 tensor-memory
//              accumulators, add the coarse gradients / 16^l, store dK, dV.
// Every wait is bounded; a wait that gives up raises a shared abort flag that
// ends every role's loop, and the CTA lets its copies and MMAs finish before
// it frees its tensor memory.  Results do not depend on timing: each key
// block's sums run in the same order whichever CTA takes it.

#include <math.h>

#include <algorithm>

#include "llsa_internal.cuh"
#include "sm100_ptx.cuh"
#include "tcgen05.cuh"

namespace llsa {

namespace {

constexpr int kD = 64;
constexpr int kTile = 32 * kD;        // one 16-row bf16 tile (2 KB)
constexpr int kGroup = 8;             // query blocks per group (128 rows)
constexpr int kStages = 4;            // Q/dO stages
constexpr int kWarps = 10;
constexpr int kThreads = kWarps * 32;
constexpr int kProducerWarp = 4;
constexpr int kMmaWarp = 5;
constexpr int kEpiWarp0 = 6;          // warps 6..9: TMEM lane quadrants 2, 3, 0, 1
constexpr uint32_t kTmemCols = 256;   // S/dP 2 x 32 columns, C 2 x 64 columns
constexpr float kLog2e = 1.4426950408889634f;
constexpr uint32_t kPolls = 1u << 22;  // per wait; each poll may suspend briefly

// shared memory (bytes from a 1024-aligned base)
constexpr int kStageBytes = 2 * kGroup * kTile;             // dO_g | Q_g (16 KB each)
constexpr int kOffStage = 0;                                // 4 stages
constexpr int kOffKV = kOffStage + kStages * kStageBytes;   // 2 x (K_c | V_c)
constexpr int kOffB = kOffKV + 2 * 2 * kTile;               // 2 x (128 rows x 128 B)
constexpr int kOffSide = kOffB + 2 * kGroup * kTile;        // 4 x (LSE[128] | Delta[128])
constexpr int kOffCoarse = kOffSide + kStages * 1024;       // 2 x (L-1) rows of 2D fp32
constexpr int kCoarseRow = 2 * kD * 4;

struct GroupDesc {
  int done;               // no more groups
  int rslot, kvslot, cslot;
  int nslot;              // valid query blocks in the group
  int first, last;        // first / last group of its key block
};

struct RowDesc {
  int done;               // no more key blocks
  int bh, c, nq, cslot;
};

struct WsShared {
  uint64_t stage_full[kStages], stage_empty[kStages];
  uint64_t row_full[2], coarse_empty[2], kv_empty[2];
  uint64_t s_full[2], s_empty[2], b_full[2], b_empty[2];
  uint64_t c_full[2], c_empty[2];
  uint64_t drain;
  uint32_t tmem_base;
  int abort;
  GroupDesc gd[kStages];
  RowDesc rd[2];
};

__device__ __forceinline__ uint32_t b_row_chunk(int r, int j) {
  return (uint32_t)((r >> 3) * 1024 + (r & 7) * 128 + ((j ^ (r & 7)) << 4));
}

// Wait for phase `parity` of `bar`; gives up (and raises the shared abort
// flag) after kPolls polls, or as soon as another role has given up.
__device__ __forceinline__ bool ws_wait(uint32_t bar, uint32_t parity, volatile int* abort) {
  for (uint32_t i = 0; i < kPolls; ++i) {
    if (mbar_try_wait(bar, parity)) return true;
    if (*abort) return false;
  }
  *abort = 1;
  return false;
}

__global__ void __launch_bounds__(kThreads, 1)
bwd_kv_tcws_kernel(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
                   const __grid_constant__ CUtensorMap tv, const __grid_constant__ CUtensorMap tdo,
                   AttnParams p, int total_rows) {
  extern __shared__ unsigned char smem_raw[];
  unsigned char* sm = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  __shared__ WsShared S;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int n1 = p.N >> 4;
  const int items = p.B * p.H * n1;
  const int K = p.K, L = p.L;
  const uint32_t base = smem_u32(sm);
  volatile int* abort = &S.abort;
  auto B_ = [](uint64_t& b) { return smem_u32(&b); };

  if (warp == 0) {
    tmem_alloc(smem_u32(&S.tmem_base), kTmemCols);
    tmem_relinquish();
  }
  if (tid == 32) {
    for (int i = 0; i < kStages; ++i) {
      mbar_init(B_(S.stage_full[i]), 1);
      mbar_init(B_(S.stage_empty[i]), 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(B_(S.row_full[i]), 1);
      mbar_init(B_(S.coarse_empty[i]), 128);
      mbar_init(B_(S.kv_empty[i]), 1);
      mbar_init(B_(S.s_full[i]), 1);
      mbar_init(B_(S.s_empty[i]), 128);
      mbar_init(B_(S.b_full[i]), 128);
      mbar_init(B_(S.b_empty[i]), 1);
      mbar_init(B_(S.c_full[i]), 1);
      mbar_init(B_(S.c_empty[i]), 128);
    }
    mbar_init(B_(S.drain), 1);
    S.abort = 0;
    fence_mbar_init();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t taddr = S.tmem_base;
  // softmax and epilogue warps run warp-collective tensor-memory loads: a
  // wait's outcome is made the same on every lane of the warp
  auto wwait = [&](uint32_t bar, uint32_t parity) {
    const bool w = ws_wait(bar, parity, abort);
    return __all_sync(0xffffffffu, w) != 0;
  };

  // producer bookkeeping for the exit drain: parity of the last copy phase
  // armed on each barrier, or -1 when none is pending there
  int st_pend[kStages] = {-1, -1, -1, -1}, row_pend[2] = {-1, -1};
  if (warp == kProducerWarp) {
    // ---------------------------------------------------------- producer
    // Key blocks come in batches of 8 from the work counter; the next batch
    // (counter, row bounds) is fetched while the current one is issued, and a
    // batch's query-block lists are loaded in one go when they are short.
    constexpr int kBatch = 8, kColRegs = 4;  // up to 128 list entries preloaded
    auto fetch = [&](int& it0, int& cnt, int& bh_l, int& c_l, int& beg_l, int& nq_l) {
      int v = 0;
      if (lane == 0) v = atomicAdd(p.work, kBatch);
      it0 = __shfl_sync(0xffffffffu, v, 0);
      cnt = max(0, min(kBatch, items - it0));
      const int it = it0 + lane;
      bh_l = 0, c_l = 0, beg_l = 0, nq_l = 0;
      if (lane < cnt) {
        bh_l = it / n1;
        c_l = it - bh_l * n1;
        const int32_t* rp = p.row_ptr[1] + (size_t)bh_l * (n1 + 1);
        beg_l = rp[c_l];
        nq_l = rp[c_l + 1] - beg_l;
      }
    };
    // the producer's waits are on "empty" barriers (no data to observe): lane
    // 0 waits and the warp follows its outcome, so the warp stays converged
    auto pwait = [&](uint32_t bar, uint32_t parity) {
      bool w = true;
      if (lane == 0) w = ws_wait(bar, parity, abort);
      return __shfl_sync(0xffffffffu, (int)w, 0) != 0;
    };
    int it0, cnt, bh_l, c_l, beg_l, nq_l;
    fetch(it0, cnt, bh_l, c_l, beg_l, nq_l);
    int n = 0, m = 0, ne = 0;  // groups, rows, non-empty rows issued
    bool ok = true;
    while (ok) {
      // the next batch is fetched now and used after this one
      int it0n, cntn, bh_n, c_n, beg_n, nq_n;
      if (cnt > 0) fetch(it0n, cntn, bh_n, c_n, beg_n, nq_n);
      // this batch's lists: one contiguous range when its rows share a head
      const int bh0 = __shfl_sync(0xffffffffu, bh_l, 0);
      const int beg0 = __shfl_sync(0xffffffffu, beg_l, 0);
      const bool same_head = __all_sync(0xffffffffu, lane >= cnt || bh_l == bh0);
      const int last = max(cnt - 1, 0);
      const int end0 = __shfl_sync(0xffffffffu, beg_l + nq_l, last);
      const bool pre = cnt > 0 && same_head && end0 - beg0 <= 32 * kColRegs;
      int colr[kColRegs];
#pragma unroll
      for (int k = 0; k < kColRegs; ++k) {
        const int e = beg0 + 32 * k + lane;
        colr[k] = (pre && e < end0) ? p.col[1][(size_t)bh0 * n1 * K + e] : 0;
      }
      for (int j = 0; j < cnt && ok; ++j) {
        const int bh = __shfl_sync(0xffffffffu, bh_l, j), c = __shfl_sync(0xffffffffu, c_l, j);
        const int beg = __shfl_sync(0xffffffffu, beg_l, j), nq = __shfl_sync(0xffffffffu, nq_l, j);
        const int rs = m & 1;
        if (m >= 2 && !pwait(B_(S.coarse_empty[rs]), ((m >> 1) - 1) & 1)) { ok = false; break; }
        const int kvs = ne & 1;
        if (nq > 0 && ne >= 2 && !pwait(B_(S.kv_empty[kvs]), ((ne >> 1) - 1) & 1)) { ok = false; break; }
        if (lane == 0) {
          S.rd[rs].done = 0;
          S.rd[rs].bh = bh;
          S.rd[rs].c = c;
          S.rd[rs].nq = nq;
          S.rd[rs].cslot = kvs;
          mbar_arrive_expect_tx(B_(S.row_full[rs]), (nq > 0 ? 2u * kTile : 0u) + (uint32_t)(L - 1) * kCoarseRow);
        }
        __syncwarp();
        {
          const int y = (int)((size_t)bh * p.N + (size_t)c * 16);
          const uint32_t kvb = base + kOffKV + (uint32_t)kvs * 2 * kTile;
          if (lane == 0 && nq > 0) tma_load_2d(kvb, &tk, 0, y, B_(S.row_full[rs]));
          if (lane == 1 && nq > 0) tma_load_2d(kvb + kTile, &tv, 0, y, B_(S.row_full[rs]));
          const int l = lane;
          if (l >= 2 && l <= L) {
            const size_t tc = (size_t)bh * (p.N >> (4 * l)) + (c >> (4 * (l - 1)));
            bulk_load(base + kOffCoarse + (uint32_t)(rs * (L - 1) + (l - 2)) * kCoarseRow, p.coarse[l] + tc * 2 * kD,
                      kCoarseRow, B_(S.row_full[rs]));
          }
        }
        row_pend[rs] = (m >> 1) & 1;
        const int ng = (nq + kGroup - 1) / kGroup;
        for (int g = 0; g < ng; ++g) {
          const int st = n % kStages;
          if (n >= kStages && !pwait(B_(S.stage_empty[st]), ((n / kStages) - 1) & 1)) { ok = false; break; }
          const int nslot = min(kGroup, nq - kGroup * g);
          if (lane == 0) {
            GroupDesc& d = S.gd[st];
            d.done = 0;
            d.rslot = rs | (((m >> 1) & 1) << 1);  // slot, and the parity of this row's row_full phase
            d.kvslot = kvs;
            d.cslot = kvs;
            d.nslot = nslot;
            d.first = (g == 0);
            d.last = (g == ng - 1);
            mbar_arrive_expect_tx(B_(S.stage_full[st]), 2u * kGroup * kTile + 128u * (uint32_t)nslot);
          }
          __syncwarp();
          // lane 8k + s: copy k of slot s (dO tile, Q tile, LSE, Delta); slots
          // past the row's end get zero-filled boxes from outside the tensor
          const int sl = lane & 7, kind = lane >> 3;
          const bool valid = sl < nslot;
          const int e = beg + kGroup * g + sl;  // list entry of this slot
          int qb = 0;
          if (pre) {
            const int r = e - beg0;
            int v = __shfl_sync(0xffffffffu, colr[0], r & 31);
#pragma unroll
            for (int k = 1; k < kColRegs; ++k) {
              const int w = __shfl_sync(0xffffffffu, colr[k], r & 31);
              if ((r >> 5) == k) v = w;
            }
            qb = valid ? v : 0;
          } else if (valid) {
            qb = p.col[1][(size_t)bh * n1 * K + e];
          }
          const size_t row0 = (size_t)bh * p.N + (size_t)qb * 16;
          const int y = valid ? (int)row0 : total_rows;
          const uint32_t sb = base + kOffStage + (uint32_t)st * kStageBytes;
          const uint32_t side = base + kOffSide + (uint32_t)st * 1024;
          const uint32_t fb = B_(S.stage_full[st]);
          if (kind == 0) tma_load_2d(sb + sl * kTile, &tdo, 0, y, fb);
          else if (kind == 1) tma_load_2d(sb + (kGroup + sl) * kTile, &tq, 0, y, fb);
          else if (valid) bulk_load(side + (kind - 2) * 512 + sl * 64, (kind == 2 ? p.lse_in : p.delta) + row0, 64, fb);
          st_pend[st] = (n / kStages) & 1;
          ++n;
        }
        if (!ok) break;
        ++m;
        if (nq > 0) ++ne;
      }
      if (!ok) break;
      if (cnt == 0) {  // end markers on both rings
        const int rs = m & 1;
        if (m >= 2 && !pwait(B_(S.coarse_empty[rs]), ((m >> 1) - 1) & 1)) break;
        if (lane == 0) {
          S.rd[rs].done = 1;
          mbar_arrive(B_(S.row_full[rs]));
        }
        row_pend[rs] = -1;
        const int st = n % kStages;
        if (n >= kStages && !pwait(B_(S.stage_empty[st]), ((n / kStages) - 1) & 1)) break;
        if (lane == 0) {
          S.gd[st].done = 1;
          mbar_arrive(B_(S.stage_full[st]));
        }
        st_pend[st] = -1;
        break;
      }
      it0 = it0n, cnt = cntn, bh_l = bh_n, c_l = c_n, beg_l = beg_n, nq_l = nq_n;
    }
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------- MMA issuer
    if (lane == 0) {
      const uint32_t idesc1 = idesc_bf16_f32(128, 16, 0);
      const uint32_t idesc3 = idesc_bf16_f32(128, 64, 1, 1);
      uint32_t uc[2] = {0u, 0u};  // key blocks accumulated so far in each C buffer
      auto issue_c = [&](const GroupDesc& d, int n) {
        const int b = n & 1, st = n % kStages;
        if (!ws_wait(B_(S.b_full[b]), (n >> 1) & 1, abort)) return false;
        if (d.first && uc[d.cslot] >= 1 && !ws_wait(B_(S.c_empty[d.cslot]), (uc[d.cslot] - 1) & 1, abort))
          return false;
        tc_fence_after();
        const uint32_t sb = base + kOffStage + (uint32_t)st * kStageBytes;
        const uint32_t bb = base + kOffB + (uint32_t)b * kGroup * kTile;
        const uint32_t tcb = taddr + 64 + 64 * d.cslot;
#pragma unroll
        for (int ks = 0; ks < kGroup; ++ks)
          tc_mma_f16(tcb, smem_desc_sw128(sb + ks * 2048, kGroup * kTile, 1024),
                     smem_desc_sw128(bb + ks * 2048, 16, 1024), idesc3, (!d.first || ks > 0));
        tc_commit(B_(S.b_empty[b]));
        tc_commit(B_(S.stage_empty[st]));
        if (d.last) {
          tc_commit(B_(S.c_full[d.cslot]));
          ++uc[d.cslot];
        }
        return true;
      };
      GroupDesc prev;
      int prev_n = -1;
      int n = 0;
      for (;;) {
        const int st = n % kStages, b = n & 1;
        // The C update of a key block's last group is normally issued behind
        // the next group's S; if that group is not there yet, issue it now: the
        // producer may be holding the next key block until the epilogue has
        // released a row slot, which needs this key block's C.
        if (prev_n >= 0 && prev.last && !mbar_try_wait(B_(S.stage_full[st]), (n / kStages) & 1)) {
          if (!issue_c(prev, prev_n)) break;
          prev_n = -1;
        }
        if (!ws_wait(B_(S.stage_full[st]), (n / kStages) & 1, abort)) break;
        const GroupDesc d = S.gd[st];
        if (d.done) break;
        if (n >= 2 && !ws_wait(B_(S.s_empty[b]), ((n >> 1) - 1) & 1, abort)) break;
        if (d.first && !ws_wait(B_(S.row_full[d.rslot & 1]), (d.rslot >> 1) & 1, abort)) break;
        tc_fence_after();
        const uint32_t sb = base + kOffStage + (uint32_t)st * kStageBytes;
        const uint32_t kvb = base + kOffKV + (uint32_t)d.kvslot * 2 * kTile;
        const uint32_t tsb = taddr + 32 * b;
#pragma unroll
        for (int ks = 0; ks < kD / 16; ++ks)
          tc_mma_f16(tsb, smem_desc_sw128(sb + kGroup * kTile + ks * 32, 16, 1024),
                     smem_desc_sw128(kvb + ks * 32, 16, 1024), idesc1, ks > 0);
#pragma unroll
        for (int ks = 0; ks < kD / 16; ++ks)
          tc_mma_f16(tsb + 16, smem_desc_sw128(sb + ks * 32, 16, 1024),
                     smem_desc_sw128(kvb + kTile + ks * 32, 16, 1024), idesc1, ks > 0);
        tc_commit(B_(S.s_full[b]));
        if (d.last) tc_commit(B_(S.kv_empty[d.kvslot]));
        // the C update of the previous group runs behind this group's S and dP
        if (prev_n >= 0 && !issue_c(prev, prev_n)) break;
        prev = d;
        prev_n = n;
        ++n;
      }
      if (prev_n >= 0 && !*abort) issue_c(prev, prev_n);
      tc_commit(B_(S.drain));  // arrives once every MMA issued above has finished
      mbar_wait_bounded(B_(S.drain), 0);
    }
  } else if (warp < 4) {
    // ---------------------------------------------------------- softmax
    const int r = tid;  // query row of the group, tensor-memory lane r
    const uint32_t t_row = (uint32_t)(warp * 32) << 16;
    const float sc2 = p.scale * kLog2e;
    int n = 0;
    for (;;) {
      const int st = n % kStages, b = n & 1;
      if (!wwait(B_(S.stage_full[st]), (n / kStages) & 1)) break;
      const int done = S.gd[st].done, nslot = S.gd[st].nslot;
      if (done) break;
      if (!wwait(B_(S.s_full[b]), (n >> 1) & 1)) break;
      tc_fence_after();
      float x[32];
      tmem_ld32(taddr + t_row + 32 * b, x);
      tmem_wait_ld();
      tc_fence_before();
      mbar_arrive(B_(S.s_empty[b]));
      const bool valid = (r >> 4) < nslot;
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
      if (n >= 2 && !wwait(B_(S.b_empty[b]), ((n >> 1) - 1) & 1)) break;
      unsigned char* brow = sm + kOffB + b * kGroup * kTile;
      *reinterpret_cast<uint4*>(brow + b_row_chunk(r, 0)) = make_uint4(hp[0], hp[1], hp[2], hp[3]);
      *reinterpret_cast<uint4*>(brow + b_row_chunk(r, 1)) = make_uint4(hp[4], hp[5], hp[6], hp[7]);
      *reinterpret_cast<uint4*>(brow + b_row_chunk(r, 2)) = make_uint4(lp[0], lp[1], lp[2], lp[3]);
      *reinterpret_cast<uint4*>(brow + b_row_chunk(r, 3)) = make_uint4(lp[4], lp[5], lp[6], lp[7]);
      *reinterpret_cast<uint4*>(brow + b_row_chunk(r, 4)) = make_uint4(hd[0], hd[1], hd[2], hd[3]);
      *reinterpret_cast<uint4*>(brow + b_row_chunk(r, 5)) = make_uint4(hd[4], hd[5], hd[6], hd[7]);
      *reinterpret_cast<uint4*>(brow + b_row_chunk(r, 6)) = make_uint4(ld[0], ld[1], ld[2], ld[3]);
      *reinterpret_cast<uint4*>(brow + b_row_chunk(r, 7)) = make_uint4(ld[4], ld[5], ld[6], ld[7]);
      fence_proxy_async_smem();
      mbar_arrive(B_(S.b_full[b]));
      ++n;
    }
  } else if (warp >= kEpiWarp0) {
    // --------------------------------------------------------- epilogue
    const int q = warp & 3;          // tensor-memory lanes 32q .. 32q+31
    const int kv = (q < 2) ? 1 : 0;  // lanes 0-63: dV^T rows, 64-127: dK^T rows
    const int d = (q & 1) * 32 + lane;
    const uint32_t t_row = (uint32_t)(q * 32) << 16;
    uint32_t cu[2] = {0u, 0u};  // key blocks read so far from each C buffer
    int m = 0;
    for (;;) {
      const int rs = m & 1;
      if (!wwait(B_(S.row_full[rs]), (m >> 1) & 1)) break;
      const int done = S.rd[rs].done, bh = S.rd[rs].bh, c = S.rd[rs].c, nq = S.rd[rs].nq, cs = S.rd[rs].cslot;
      if (done) break;
      float acc[32];
      if (nq > 0) {
        if (!wwait(B_(S.c_full[cs]), cu[cs] & 1u)) break;
        tc_fence_after();
        tmem_ld32(taddr + t_row + 64 + 64 * cs + (kv ? 0u : 32u), acc);
        tmem_wait_ld();
        tc_fence_before();
        mbar_arrive(B_(S.c_empty[cs]));
        ++cu[cs];
      } else {
#pragma unroll
        for (int j = 0; j < 32; ++j) acc[j] = 0.f;
      }
      float cg = 0.f;
      for (int l = 2; l <= L; ++l) {
        const float* crow = reinterpret_cast<const float*>(sm + kOffCoarse + (rs * (L - 1) + (l - 2)) * kCoarseRow);
        cg += crow[kv * kD + d] * (1.0f / (float)(1u << (4 * l)));
      }
      const float f = kv ? 1.f : p.scale;
      bf16* out = static_cast<bf16*>(kv ? p.dv : p.dk) + ((size_t)bh * p.N + (size_t)c * 16) * kD + d;
#pragma unroll
      for (int key = 0; key < 16; ++key) out[(size_t)key * kD] = __float2bfloat16_rn((acc[key] + acc[16 + key]) * f + cg);
      fence_proxy_async_smem();  // the coarse rows read above are reloaded by bulk copies
      mbar_arrive(B_(S.coarse_empty[rs]));
      ++m;
    }
  }

  // every role has left its loop; after an abort, let the copies still in
  // flight land (their last armed phases; end markers complete at once)
  __syncthreads();
  if (warp == kProducerWarp && lane == 0 && *abort) {
    for (int st = 0; st < kStages; ++st)
      if (st_pend[st] >= 0) mbar_wait_bounded(B_(S.stage_full[st]), (uint32_t)st_pend[st]);
    for (int rs = 0; rs < 2; ++rs)
      if (row_pend[rs] >= 0) mbar_wait_bounded(B_(S.row_full[rs]), (uint32_t)row_pend[rs]);
  }
  if (tid == 0 && *abort) report_status(p.status, LLSA_DEV_TIMEOUT);
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(taddr, kTmemCols);
  }
}

}  // namespace

// maps: Q, K, V, dO as 2D [B*H*N rows, 64 cols] bf16, box 16 x 64, 128-byte swizzle.
cudaError_t launch_bwd_kv_tcws(const AttnParams& p, const CUtensorMap* maps, cudaStream_t s) {
  const size_t smem = 1024 + kOffCoarse + (size_t)2 * (p.L - 1) * kCoarseRow;
  cudaError_t e = cudaFuncSetAttribute(bwd_kv_tcws_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(bwd_kv_tcws_kernel, cudaFuncAttributePreferredSharedMemoryCarveout,
                           (int)cudaSharedmemCarveoutMaxShared);
  if (e != cudaSuccess) return e;
  int dev = 0, nsm = 0;
  e = cudaGetDevice(&dev);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return e;
  const long items = (long)p.B * p.H * (p.N / kBlock);
  const int grid = (int)std::min<long>(items, (long)nsm);  // one CTA per SM (shared memory)
  const int total_rows = p.B * p.H * p.N;
  bwd_kv_tcws_kernel<<<grid, kThreads, smem, s>>>(maps[0], maps[1], maps[2], maps[3], p, total_rows);
  return cudaGetLastError();
}

}  // namespace llsa
