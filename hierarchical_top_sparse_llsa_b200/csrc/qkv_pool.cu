// The QKV projection with the hierarchical compression in its epilogue: the
// step before the path ("Input (Q, K, V) -> Hierarchical Compression -> ..."
// in the pipeline overview of the howistudyai explainer of "Trainable
// Log-linear Sparse Attention for Efficient Diffusion Transformers"), with
// Step 1's level-1 and level-2 means formed while the projected tile is still
// on chip, so the pool's second read of Q, K and V is gone.
//
// [Q | K | V] = X W^T, X bf16 [B*N, C] (tokens in Z-order), W bf16 [3*H*D, C]
// (a linear layer's weight: output feature t*H*D + h*D + d is tensor t, head
// h, channel d).  One CTA computes a tile of 256 tokens x 128 features on the
// 5th-generation tensor cores:
//   warp 0 (one thread)  TMA loads of X (256 x 64) and W (128 x 64) k-slices
//                        into a 2-stage ring (K-major, 128-byte swizzle);
//   warp 1 (one thread)  per 16-wide k step, two M = 128, N = 128 MMAs (the
//                        two 128-token halves) into 256 TMEM columns (fp32);
//   all four warps       the epilogue: each thread reads its token row of the
//                        accumulator (tcgen05.ld), rounds it to bf16 and
//                        stages it in shared memory (16-byte chunks XOR-ed
//                        with the row, conflict-free); the tile is written to
//                        Q, K or V [B, H, N, D] in coalesced 16-byte stores;
//                        then level 1 (16 level-1 tokens) and level 2 (one
//                        level-2 token) are summed from the staged bf16 values
//                        exactly as the pool kernel sums them (left to right,
//                        fp32, one rounding per addition, then x 1/16), so the
//                        pyramid equals llsa_pool's on these Q, K, V bit for
//                        bit.  Levels >= 3 come from the pool's level-up pass.
// Two CTAs fit on an SM (96 KB of shared memory and 256 TMEM columns each),
// so one CTA's epilogue runs while the other's MMAs do: measured at 256x256
// pixels with C = 1024, 0.41 ms against 0.56 ms for one CTA per SM with a
// 4-stage ring.
// A tile never straddles a batch (N % 256 == 0) nor a tensor (H*D % 128 == 0).
// Every wait is bounded; a time-out is reported as LLSA_DEV_TIMEOUT.

#include <cuda.h>

#include "llsa_internal.cuh"
#include "sm100_ptx.cuh"
#include "tcgen05.cuh"

namespace llsa {

namespace {

constexpr int kTokTile = 256;   // tokens per CTA (two MMA halves of 128)
constexpr int kFeatTile = 128;  // output features per CTA (the MMA's N)
constexpr int kKStep = 64;      // k elements per stage (one 128-byte swizzle row)
constexpr int kStages = 2;
constexpr int kXBytes = kTokTile * kKStep * 2;   // 32 KB
constexpr int kWBytes = kFeatTile * kKStep * 2;  // 16 KB
constexpr int kStageBytes = kXBytes + kWBytes;
constexpr int kTmemCols = 2 * kFeatTile;

struct QkvParams {
  void* out[3];        // Q, K, V bf16 [B, H, N, D]
  float* lvl[3][3];    // pyramid levels 1 and 2 per tensor (V level 1: none)
  int32_t* status;
  int N, H, D, L, C;
};

// byte offset of 16-byte chunk c (0..15) of staged token row r (256 bytes)
__device__ __forceinline__ uint32_t stage_off(int r, int c) { return (uint32_t)(r * 256 + ((c ^ (r & 15)) << 4)); }

__global__ void __launch_bounds__(128, 2)
qkv_pool_kernel(const __grid_constant__ CUtensorMap tx, const __grid_constant__ CUtensorMap tw, QkvParams p) {
  extern __shared__ unsigned char smem_raw[];
  unsigned char* sm = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  __shared__ __align__(8) uint64_t full[kStages], empty[kStages], acc_full;
  __shared__ uint32_t tmem_slot;
  __shared__ int abort_flag;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int HD = p.H * p.D;
  const int F0 = blockIdx.x * kFeatTile;  // first output feature
  const int m0 = blockIdx.y * kTokTile;   // first token row of X
  const int nk = p.C / kKStep;
  const uint32_t s0 = smem_u32(sm);

  if (tid == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(smem_u32(&full[s]), 1);
      mbar_init(smem_u32(&empty[s]), 1);
    }
    mbar_init(smem_u32(&acc_full), 1);
    fence_mbar_init();
    abort_flag = 0;
  }
  if (warp == 0) {
    tmem_alloc(smem_u32(&tmem_slot), kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = tmem_slot;

  if (warp == 0 && lane == 0) {
    // producer
    int kb = 0;
    bool ok = true;
    for (; kb < nk; ++kb) {
      const int s = kb % kStages;
      if (kb >= kStages) {
        ok = mbar_wait_bounded(smem_u32(&empty[s]), (uint32_t)((kb / kStages - 1) & 1));
        if (!ok) break;
      }
      const uint32_t bar = smem_u32(&full[s]);
      const uint32_t xs = s0 + (uint32_t)s * kStageBytes;
      mbar_arrive_expect_tx(bar, kStageBytes);
      tma_load_2d(xs, &tx, kb * kKStep, m0, bar);
      tma_load_2d(xs + kXBytes, &tw, kb * kKStep, F0, bar);
    }
    if (!ok) atomicExch(&abort_flag, 1);
    // every copy issued lands before the CTA goes on (the last ones at most
    // kStages phases back, so their parities are unambiguous)
    for (int j = (kb > kStages ? kb - kStages : 0); j < kb; ++j)
      mbar_wait_bounded(smem_u32(&full[j % kStages]), (uint32_t)((j / kStages) & 1));
  } else if (warp == 1 && lane == 0) {
    // MMA issue
    const uint32_t idesc = idesc_bf16_f32(128, kFeatTile, 0, 0);
    bool ok = true;
    for (int kb = 0; kb < nk; ++kb) {
      const int s = kb % kStages;
      ok = mbar_wait_bounded(smem_u32(&full[s]), (uint32_t)((kb / kStages) & 1));
      if (!ok) break;
      tc_fence_after();
      const uint32_t xs = s0 + (uint32_t)s * kStageBytes, ws = xs + kXBytes;
#pragma unroll
      for (int kk = 0; kk < kKStep / 16; ++kk) {
        const uint64_t bdesc = smem_desc_sw128(ws + kk * 32, 16, 1024);
#pragma unroll
        for (int h = 0; h < 2; ++h)
          tc_mma_f16(tbase + (uint32_t)h * kFeatTile, smem_desc_sw128(xs + (uint32_t)h * (kXBytes / 2) + kk * 32, 16, 1024),
                     bdesc, idesc, (kb > 0 || kk > 0) ? 1u : 0u);
      }
      tc_commit(smem_u32(&empty[s]));
    }
    if (!ok) atomicExch(&abort_flag, 1);
    tc_commit(smem_u32(&acc_full));  // also when aborted: the issued MMAs finish before TMEM is freed
  }
  __syncwarp();

  // epilogue: the accumulator, staged as bf16 over the (now idle) ring
  const bool acc_ok = mbar_wait_bounded(smem_u32(&acc_full), 0);
  tc_fence_after();
  __syncthreads();
  const bool ok = acc_ok && abort_flag == 0;
  if (ok) {
#pragma unroll 1
    for (int h = 0; h < 2; ++h) {
      const int r = 128 * h + 32 * warp + lane;  // staged row of this thread
#pragma unroll 1
      for (int c0 = 0; c0 < kFeatTile; c0 += 32) {
        float v[32];
        tmem_ld32(tbase + ((uint32_t)(32 * warp) << 16) + (uint32_t)(h * kFeatTile + c0), v);
        tmem_wait_ld();
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          uint4 u;
          u.x = pack_bf16(v[8 * q + 0], v[8 * q + 1]);
          u.y = pack_bf16(v[8 * q + 2], v[8 * q + 3]);
          u.z = pack_bf16(v[8 * q + 4], v[8 * q + 5]);
          u.w = pack_bf16(v[8 * q + 6], v[8 * q + 7]);
          *reinterpret_cast<uint4*>(sm + stage_off(r, c0 / 8 + q)) = u;
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tbase, kTmemCols);
  if (!ok) {
    if (tid == 0) report_status(p.status, LLSA_DEV_TIMEOUT);
    return;
  }

  const int t = F0 / HD;            // tensor: 0 Q, 1 K, 2 V
  const int f0 = F0 - t * HD;       // first feature within the tensor
  const int b = m0 / p.N, n0 = m0 - b * p.N;
  const int D = p.D, CPR = D / 8;   // 16-byte chunks per head row
  // Q, K or V: each head of the tile is 256 contiguous rows of D elements
  bf16* out = static_cast<bf16*>(p.out[t]);
  for (int hh = 0; hh < kFeatTile / D; ++hh) {
    const int head = (f0 + hh * D) / D;
    uint4* dst = reinterpret_cast<uint4*>(out + (((size_t)b * p.H + head) * p.N + n0) * D);
    for (int e = tid; e < kTokTile * CPR; e += 128) {
      const int r = e / CPR, c = e % CPR;
      dst[e] = *reinterpret_cast<const uint4*>(sm + stage_off(r, hh * CPR + c));
    }
  }
  // level 1: token t1 of the tile, 8 features per task, rows left to right
  float* m1 = reinterpret_cast<float*>(sm + kTokTile * 256);  // [16][128]
  float* o1 = p.lvl[t][1];
  for (int e = tid; e < 16 * 16; e += 128) {
    const int t1 = e / 16, cv = e % 16;
    float acc[8];
    {
      const uint4 u = *reinterpret_cast<const uint4*>(sm + stage_off(16 * t1, cv));
      const uint32_t w4[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        acc[2 * i] = bf16x2_lo(w4[i]);
        acc[2 * i + 1] = bf16x2_hi(w4[i]);
      }
    }
#pragma unroll
    for (int j = 1; j < 16; ++j) {
      const uint4 u = *reinterpret_cast<const uint4*>(sm + stage_off(16 * t1 + j, cv));
      const uint32_t w4[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        acc[2 * i] = __fadd_rn(acc[2 * i], bf16x2_lo(w4[i]));
        acc[2 * i + 1] = __fadd_rn(acc[2 * i + 1], bf16x2_hi(w4[i]));
      }
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      acc[i] = __fmul_rn(acc[i], 0.0625f);
      m1[t1 * kFeatTile + cv * 8 + i] = acc[i];
    }
    if (o1 != nullptr) {
      const int f = f0 + cv * 8, head = f / D, d = f % D;
      float* dst = o1 + (((size_t)b * p.H + head) * (p.N / 16) + n0 / 16 + t1) * D + d;
      *reinterpret_cast<float4*>(dst) = make_float4(acc[0], acc[1], acc[2], acc[3]);
      *reinterpret_cast<float4*>(dst + 4) = make_float4(acc[4], acc[5], acc[6], acc[7]);
    }
  }
  if (p.L < 2) return;
  __syncthreads();
  // level 2: the tile's one level-2 token, one feature per thread
  {
    const int f = f0 + tid, head = f / D, d = f % D;
    float a = m1[tid];
#pragma unroll
    for (int t1 = 1; t1 < 16; ++t1) a = __fadd_rn(a, m1[t1 * kFeatTile + tid]);
    p.lvl[t][2][(((size_t)b * p.H + head) * (p.N / 256) + n0 / 256) * D + d] = __fmul_rn(a, 0.0625f);
  }
}

}  // namespace

size_t qkv_pool_smem() { return 1024 + (size_t)kStages * kStageBytes; }

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
  const size_t smem = qkv_pool_smem();
  cudaError_t e = cudaFuncSetAttribute(qkv_pool_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const dim3 grid((unsigned)(3 * H * D / kFeatTile), (unsigned)((long long)B * N / kTokTile));
  qkv_pool_kernel<<<grid, 128, smem, s>>>(maps[0], maps[1], p);
  return cudaGetLastError();
}

}  // namespace llsa
