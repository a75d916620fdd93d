// The QKV projection with the hierarchical compression in its epilogue: the
// step before the path ("Input (Q, K, V) -> Hierarchical Compression -> ..."
// in the pipeline overview of the howistudyai explainer of "Trainable
// Log-linear Sparse Attention for Efficient Diffusion Transformers"), with
// Step 1's level-1 and level-2 means formed while the projected tile is still
// on chip, so the pool's second read of Q, K and V is gone.
//
// [Q | K | V] = X W^T, X bf16 [B*N, C] (tokens in Z-order), W bf16 [3*H*D, C]
// (a linear layer's weight: output feature t*H*D + h*D + d is tensor t, head
// h, channel d), in tiles of 256 tokens x 128 features on the 5th-generation
// tensor cores.  One persistent CTA per SM walks the tiles (features fastest,
// so the tiles that share an X tile run together and find it in L2), with
// its warps specialised:
//   warp 0 (one thread)  TMA loads of the X (256 x 64) and W (128 x 64)
//                        k-slices into a 3-stage ring (K-major, 128-byte
//                        swizzle);
//   warp 1               allocates the 512 TMEM columns; one thread issues,
//                        per 16-wide k step, two M = 128, N = 128 MMAs (the
//                        two 128-token halves) into one of two 256-column
//                        fp32 accumulators, so the next tile's MMAs run while
//                        the epilogue drains the previous one;
//   warps 2-5            the epilogue: each thread reads its token row of the
//                        accumulator (tcgen05.ld; warp w owns TMEM lanes
//                        32 (w % 4) .. +31), rounds it to bf16 and stages it
//                        in shared memory (16-byte chunks XOR-ed with the row,
//                        conflict-free), releases the accumulator, writes the
//                        tile to Q, K or V [B, H, N, D] in coalesced 16-byte
//                        stores, and sums level 1 (16 level-1 tokens) and
//                        level 2 (one level-2 token) from the staged bf16
//                        values exactly as the pool kernel sums them (left to
//                        right, fp32, one rounding per addition, then x 1/16),
//                        so the pyramid equals llsa_pool's on these Q, K, V
//                        bit for bit.  Levels >= 3 come from the pool's
//                        level-up pass.
// A tile never straddles a batch (N % 256 == 0) nor a tensor (H*D % 128 == 0).
// Every wait is bounded; a time-out is reported as LLSA_DEV_TIMEOUT.

#include <cuda.h>

#include "llsa_internal.cuh"
#include "sm100_ptx.cuh"
#include "tcgen05.cuh"

namespace llsa {

namespace {

constexpr int kTokTile = 256;   // tokens per tile (two MMA halves of 128)
constexpr int kFeatTile = 128;  // output features per tile (the MMA's N)
constexpr int kKStep = 64;      // k elements per stage (one 128-byte swizzle row)
constexpr int kStages = 3;
constexpr int kXBytes = kTokTile * kKStep * 2;   // 32 KB
constexpr int kWBytes = kFeatTile * kKStep * 2;  // 16 KB
constexpr int kStageBytes = kXBytes + kWBytes;
constexpr int kAccCols = 2 * kFeatTile;          // one accumulator: two halves
constexpr int kTmemCols = 2 * kAccCols;          // two accumulators
constexpr int kStageOff = kStages * kStageBytes;  // the epilogue's bf16 tile
constexpr int kM1Off = kStageOff + kTokTile * 256;  // level-1 means [16][128] fp32
constexpr int kThreads = 192;
constexpr int kEpiThreads = 128;

struct QkvParams {
  void* out[3];        // Q, K, V bf16 [B, H, N, D]
  float* lvl[3][3];    // pyramid levels 1 and 2 per tensor (V level 1: none)
  int32_t* status;
  int N, H, D, L, C;
  int n_feat_tiles, n_tiles;
};

// byte offset of 16-byte chunk c (0..15) of staged token row r (256 bytes)
__device__ __forceinline__ uint32_t stage_off(int r, int c) { return (uint32_t)(r * 256 + ((c ^ (r & 15)) << 4)); }

__device__ __forceinline__ void epi_bar() { asm volatile("bar.sync 1, 128;" ::: "memory"); }

__global__ void __launch_bounds__(kThreads, 1)
qkv_pool_kernel(const __grid_constant__ CUtensorMap tx, const __grid_constant__ CUtensorMap tw, QkvParams p) {
  extern __shared__ unsigned char smem_raw[];
  unsigned char* sm = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  __shared__ __align__(8) uint64_t full[kStages], empty[kStages], acc_full[2], acc_empty[2];
  __shared__ uint32_t tmem_slot;
  __shared__ int abort_flag, epi_abort;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int HD = p.H * p.D;
  const int nk = p.C / kKStep;
  const uint32_t s0 = smem_u32(sm);
  // this CTA's tiles: blockIdx.x, blockIdx.x + gridDim.x, ...
  const int my_tiles = blockIdx.x < p.n_tiles ? (p.n_tiles - 1 - blockIdx.x) / gridDim.x + 1 : 0;

  if (tid == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(smem_u32(&full[s]), 1);
      mbar_init(smem_u32(&empty[s]), 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(smem_u32(&acc_full[a]), 1);
      mbar_init(smem_u32(&acc_empty[a]), 4);  // one arrival per epilogue warp
    }
    fence_mbar_init();
    abort_flag = 0;
    epi_abort = 0;
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(&tmem_slot), kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      // producer: k-slices of every tile, in order
      int q = 0;  // running stage count
      bool ok = true;
      for (int i = 0; i < my_tiles && ok; ++i) {
        const int tile = blockIdx.x + i * gridDim.x;
        const int F0 = (tile % p.n_feat_tiles) * kFeatTile, m0 = (tile / p.n_feat_tiles) * kTokTile;
        for (int kb = 0; kb < nk; ++kb, ++q) {
          const int s = q % kStages;
          if (q >= kStages) {
            ok = mbar_wait_bounded(smem_u32(&empty[s]), (uint32_t)((q / kStages - 1) & 1));
            if (!ok) break;
          }
          const uint32_t bar = smem_u32(&full[s]);
          const uint32_t xs = s0 + (uint32_t)s * kStageBytes;
          mbar_arrive_expect_tx(bar, kStageBytes);
          tma_load_2d(xs, &tx, kb * kKStep, m0, bar);
          tma_load_2d(xs + kXBytes, &tw, kb * kKStep, F0, bar);
        }
      }
      if (!ok) atomicExch(&abort_flag, 1);
      // every copy issued lands before the CTA goes on (the last ones at most
      // kStages phases back, so their parities are unambiguous)
      for (int j = (q > kStages ? q - kStages : 0); j < q; ++j)
        mbar_wait_bounded(smem_u32(&full[j % kStages]), (uint32_t)((j / kStages) & 1));
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // MMA issue
      const uint32_t idesc = idesc_bf16_f32(128, kFeatTile, 0, 0);
      int q = 0;
      int commits0 = 0, commits1 = 0;  // acc_full commits per accumulator
      bool ok = true;
      for (int i = 0; i < my_tiles && ok; ++i) {
        const int a = i & 1;
        if (i >= 2) {  // the epilogue has read accumulator a (tile i - 2)
          ok = mbar_wait_bounded(smem_u32(&acc_empty[a]), (uint32_t)((i / 2 - 1) & 1));
          if (!ok) break;
          tc_fence_after();
        }
        const uint32_t acc = tbase + (uint32_t)a * kAccCols;
        for (int kb = 0; kb < nk; ++kb, ++q) {
          const int s = q % kStages;
          ok = mbar_wait_bounded(smem_u32(&full[s]), (uint32_t)((q / kStages) & 1));
          if (!ok) break;
          tc_fence_after();
          const uint32_t xs = s0 + (uint32_t)s * kStageBytes, ws = xs + kXBytes;
#pragma unroll
          for (int kk = 0; kk < kKStep / 16; ++kk) {
            const uint64_t bdesc = smem_desc_sw128(ws + kk * 32, 16, 1024);
#pragma unroll
            for (int h = 0; h < 2; ++h)
              tc_mma_f16(acc + (uint32_t)h * kFeatTile,
                         smem_desc_sw128(xs + (uint32_t)h * (kXBytes / 2) + kk * 32, 16, 1024), bdesc, idesc,
                         (kb > 0 || kk > 0) ? 1u : 0u);
          }
          tc_commit(smem_u32(&empty[s]));
        }
        tc_commit(smem_u32(&acc_full[a]));  // also when aborted
        if (a == 0) ++commits0;
        else ++commits1;
      }
      if (!ok) atomicExch(&abort_flag, 1);
      // every MMA issued has finished before TMEM is freed (immediate when
      // the epilogue has consumed both accumulators)
      if (commits0 > 0) mbar_wait_bounded(smem_u32(&acc_full[0]), (uint32_t)((commits0 - 1) & 1));
      if (commits1 > 0) mbar_wait_bounded(smem_u32(&acc_full[1]), (uint32_t)((commits1 - 1) & 1));
    }
  } else {
    // epilogue warps 2..5: TMEM lane quarter eq = warp % 4
    const int et = tid - 64;  // 0..127
    const int eq = warp & 3;
    float* m1 = reinterpret_cast<float*>(sm + kM1Off);
    for (int i = 0; i < my_tiles; ++i) {
      const int a = i & 1;
      const int tile = blockIdx.x + i * gridDim.x;
      const int F0 = (tile % p.n_feat_tiles) * kFeatTile, m0 = (tile / p.n_feat_tiles) * kTokTile;
      // the warp decides as one (tcgen05.ld needs the whole warp); a warp that
      // gave up still meets the others at the barrier below, where all four
      // leave together
      const bool got = __all_sync(0xffffffffu, mbar_wait_bounded(smem_u32(&acc_full[a]), (uint32_t)((i / 2) & 1)));
      if (!got) epi_abort = 1;
      if (got) {
        tc_fence_after();
        const uint32_t acc = tbase + (uint32_t)a * kAccCols + ((uint32_t)(32 * eq) << 16);
#pragma unroll 1
        for (int h = 0; h < 2; ++h) {
          const int r = 128 * h + 32 * eq + lane;  // staged row of this thread
#pragma unroll 1
          for (int c0 = 0; c0 < kFeatTile; c0 += 32) {
            float v[32];
            tmem_ld32(acc + (uint32_t)(h * kFeatTile + c0), v);
            tmem_wait_ld();
#pragma unroll
            for (int qq = 0; qq < 4; ++qq) {
              uint4 u;
              u.x = pack_bf16(v[8 * qq + 0], v[8 * qq + 1]);
              u.y = pack_bf16(v[8 * qq + 2], v[8 * qq + 3]);
              u.z = pack_bf16(v[8 * qq + 4], v[8 * qq + 5]);
              u.w = pack_bf16(v[8 * qq + 6], v[8 * qq + 7]);
              *reinterpret_cast<uint4*>(sm + kStageOff + stage_off(r, c0 / 8 + qq)) = u;
            }
          }
        }
        // accumulator a is read: the MMA thread may overwrite it (tile i + 2)
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&acc_empty[a]));
      }
      epi_bar();  // the whole tile is staged (or some warp gave up)
      if (epi_abort != 0) break;

      const int t = F0 / HD;       // tensor: 0 Q, 1 K, 2 V
      const int f0 = F0 - t * HD;  // first feature within the tensor
      // this tensor's output and pyramid levels, selected without a run-time
      // index into the parameters (which would copy them to local memory)
      void* const out_t = t == 0 ? p.out[0] : (t == 1 ? p.out[1] : p.out[2]);
      float* const o1 = t == 0 ? p.lvl[0][1] : (t == 1 ? p.lvl[1][1] : p.lvl[2][1]);
      float* const o2 = t == 0 ? p.lvl[0][2] : (t == 1 ? p.lvl[1][2] : p.lvl[2][2]);
      const int b = m0 / p.N, n0 = m0 - b * p.N;
      const int D = p.D, CPR = D / 8;  // 16-byte chunks per head row
      // Q, K or V: each head of the tile is 256 contiguous rows of D elements
      bf16* out = static_cast<bf16*>(out_t);
      for (int hh = 0; hh < kFeatTile / D; ++hh) {
        const int head = (f0 + hh * D) / D;
        uint4* dst = reinterpret_cast<uint4*>(out + (((size_t)b * p.H + head) * p.N + n0) * D);
        for (int e = et; e < kTokTile * CPR; e += kEpiThreads) {
          const int r = e / CPR, c = e % CPR;
          dst[e] = *reinterpret_cast<const uint4*>(sm + kStageOff + stage_off(r, hh * CPR + c));
        }
      }
      // level 1: token t1 of the tile, 8 features per task, rows left to right
      for (int e = et; e < 16 * 16; e += kEpiThreads) {
        const int t1 = e / 16, cv = e % 16;
        float sum[8];
        {
          const uint4 u = *reinterpret_cast<const uint4*>(sm + kStageOff + stage_off(16 * t1, cv));
          const uint32_t w4[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            sum[2 * k] = bf16x2_lo(w4[k]);
            sum[2 * k + 1] = bf16x2_hi(w4[k]);
          }
        }
#pragma unroll
        for (int j = 1; j < 16; ++j) {
          const uint4 u = *reinterpret_cast<const uint4*>(sm + kStageOff + stage_off(16 * t1 + j, cv));
          const uint32_t w4[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            sum[2 * k] = __fadd_rn(sum[2 * k], bf16x2_lo(w4[k]));
            sum[2 * k + 1] = __fadd_rn(sum[2 * k + 1], bf16x2_hi(w4[k]));
          }
        }
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          sum[k] = __fmul_rn(sum[k], 0.0625f);
          m1[t1 * kFeatTile + cv * 8 + k] = sum[k];
        }
        if (o1 != nullptr) {
          const int f = f0 + cv * 8, head = f / D, d = f % D;
          float* dst = o1 + (((size_t)b * p.H + head) * (p.N / 16) + n0 / 16 + t1) * D + d;
          *reinterpret_cast<float4*>(dst) = make_float4(sum[0], sum[1], sum[2], sum[3]);
          *reinterpret_cast<float4*>(dst + 4) = make_float4(sum[4], sum[5], sum[6], sum[7]);
        }
      }
      epi_bar();  // level-1 means complete; the staged tile is no longer read
      if (p.L >= 2) {
        // level 2: the tile's one level-2 token, one feature per thread
        const int f = f0 + et, head = f / D, d = f % D;
        float s2 = m1[et];
#pragma unroll
        for (int t1 = 1; t1 < 16; ++t1) s2 = __fadd_rn(s2, m1[t1 * kFeatTile + et]);
        o2[(((size_t)b * p.H + head) * (p.N / 256) + n0 / 256) * D + d] = __fmul_rn(s2, 0.0625f);
      }
      epi_bar();  // m1 is rewritten by the next tile
    }
    if (epi_abort != 0 && et == 0) atomicExch(&abort_flag, 1);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) tmem_dealloc(tbase, kTmemCols);
  if (tid == 0 && abort_flag != 0) report_status(p.status, LLSA_DEV_TIMEOUT);
}

}  // namespace

size_t qkv_pool_smem() { return 1024 + (size_t)kM1Off + 16 * kFeatTile * sizeof(float); }

// maps: X as [B*N rows, C] with 256-row boxes, W as [3*H*D rows, C] with
// 128-row boxes, both 64 columns wide with 128-byte swizzle.
cudaError_t launch_qkv_pool(const CUtensorMap* maps, void* const out[3], float* const lvl[3][3], int32_t* status,
                            int B, int N, int H, int D, int L, int C, cudaStream_t s) {
  QkvParams p;
  for (int t = 0; t < 3; ++t) {
    p.out[t] = out[t];
    for (int l = 0; l < 3; ++l) p.lvl[t][l] = lvl[t][l];
  }
  p.status = status;
  p.N = N;
  p.H = H;
  p.D = D;
  p.L = L;
  p.C = C;
  p.n_feat_tiles = 3 * H * D / kFeatTile;
  const long long tiles = (long long)p.n_feat_tiles * ((long long)B * N / kTokTile);
  if (tiles > 0x7fffffffLL) return cudaErrorInvalidValue;
  p.n_tiles = (int)tiles;
  const size_t smem = qkv_pool_smem();
  cudaError_t e = cudaFuncSetAttribute(qkv_pool_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  int dev = 0, sms = 0;
  e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return e;
  const int grid = p.n_tiles < sms ? p.n_tiles : sms;
  qkv_pool_kernel<<<grid, kThreads, smem, s>>>(maps[0], maps[1], p);
  return cudaGetLastError();
}

}  // namespace llsa
