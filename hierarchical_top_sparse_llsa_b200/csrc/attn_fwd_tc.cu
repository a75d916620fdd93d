// Sparse attention forward with hierarchical KV enrichment and KV
// reweighting on the 5th-generation tensor cores (tcgen05), bf16, D = 64
// (Step 3 of the howistudyai explainer of "Trainable Log-linear Sparse
// Attention for Efficient Diffusion Transformers").
//
// A CTA holds 8 sibling 16-token query blocks: 128 query rows, the M of one
// tcgen05 MMA.  Siblings select overlapping key blocks, so the CTA sorts and
// de-duplicates their selections into a union U and walks U in chunks of 4 key
// blocks (64 keys): each chunk's K and V tiles arrive by 2D TMA loads
// (128-byte swizzle, no multicast) into a double buffer, then
//   S = Q K_chunk^T        (M 128, N <= 64, K 64) into tensor memory,
//   P = 2^(S*scale - m)    by 256 threads, two per query row, with the
//                          key blocks its own query block did not select
//                          masked out; P is written as bf16 to shared memory,
//   O += P V_chunk         (M 128, N 64, K <= 64) accumulated in tensor memory.
// The MMAs are issued by one thread and complete on mbarriers; the softmax
// works on half rows in registers (no shuffles), against the running row
// maximum; when it grows, the row of O is rescaled in tensor memory.  The coarse keys, shared by all 8 blocks,
// follow as padded chunks converted from the fp32 pyramid.  Key blocks a row
// did not select cost MMA work but no exponentials; the union keeps that
// waste near |U| / K per block instead of every candidate.

#include <math.h>

#include "keyset.cuh"
#include "sm100_ptx.cuh"
#include "tcgen05.cuh"

namespace llsa {

namespace {

constexpr int kTcBlocks = 8;      // query blocks per CTA (128 rows)
constexpr int kTcWarps = 8;
constexpr int kTcThreads = kTcWarps * 32;  // two threads per query row (32 columns each)
constexpr int kChunkBlocks = 4;   // key blocks per chunk (64 keys)
constexpr int kTcD = 64;
constexpr int kTile = 32 * kTcD;  // bytes of a 16-row bf16 tile (2 KB)
constexpr int kMaxUnion = kTcBlocks * kMaxK;  // 256
constexpr uint32_t kTmemCols = 128;           // S: columns 0..63, O: 64..127
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
// Threshold 0: the reference is the exact running max, so the largest
// probability of a row is exactly 1 and its bf16 rounding is exact; a lagging
// reference (up to 2^8) let that rounding error through on rows with few keys.
constexpr float kRescaleLog2 = 0.0f;

// shared-memory layout (bytes from a 1024-aligned base)
constexpr int kOffQ = 0;                                        // 8 tiles
constexpr int kOffK = kOffQ + kTcBlocks * kTile;                // 2 x 4 tiles
constexpr int kOffV = kOffK + 2 * kChunkBlocks * kTile;         // 2 x 4 tiles
constexpr int kOffP = kOffV + 2 * kChunkBlocks * kTile;         // 128 rows x 128 B
constexpr int kTileBytes = kOffP + kTcBlocks * kTile;           // 64 KB

struct TcShared {
  uint64_t bar_q, bar_s, bar_pv, bar_kv[2];
  uint32_t tmem_base;
  int nu, nc;
  int ent[kTcBlocks * kMaxK];         // selections, 0x7fffffff when unused
  int ulist[kMaxUnion];               // sorted union of the selections
  uint32_t mask[kTcBlocks][kMaxUnion / 32];  // block b selected union entry u
  int clist[kMaxL * kMaxK];           // coarse keys: level << 24 | token
  float clw[kMaxL * kMaxK + 64];      // their log2 weights (-inf for pads)
  float red[2][128];                  // per row and column half: max, then sum
};

template <int E>
__global__ void __launch_bounds__(kTcThreads)
attn_fwd_tc_kernel(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
                   const __grid_constant__ CUtensorMap tv, AttnParams p) {
  extern __shared__ unsigned char smem_raw[];
  unsigned char* sm = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  TcShared& S = *reinterpret_cast<TcShared*>(sm + kTileBytes);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int bh = blockIdx.y;
  const int n1 = p.N >> 4;
  const int b0 = blockIdx.x * kTcBlocks;
  const int K = p.K;
  const size_t rowbase = (size_t)bh * p.N;
  int flags = 0;

  // ---- selections of the 8 blocks (one per warp), coarse list (warp 0)
  for (int i = 0; i < kTcBlocks / kTcWarps; ++i) {
    const int bi = warp * (kTcBlocks / kTcWarps) + i;
    const int b = b0 + bi;
    const bool on = (b < n1) && lane < K;
    const int v = on ? p.idx[1][((size_t)bh * n1 + b) * K + lane] : -1;
    const bool used = warp_row_used(v, lane, n1, on, flags);
    if (lane < K) S.ent[bi * K + lane] = used ? v : 0x7fffffff;
  }
  for (int e = tid; e < kTcBlocks * (kMaxUnion / 32); e += kTcThreads) (&S.mask[0][0])[e] = 0u;
  if (warp == 0) {
    int n = 0;
    for (int l = 2; l <= p.L; ++l) {
      const int nl = p.N >> (4 * l);
      const int a = b0 >> (4 * (l - 1));
      const int Kl = p.Kl[l];
      const int c = (lane < Kl) ? p.idx[l][((size_t)bh * nl + a) * Kl + lane] : -1;
      const bool u = warp_row_used(c, lane, nl, lane < Kl, flags);
      const unsigned m = __ballot_sync(0xffffffffu, u);
      if (u) S.clist[n + __popc(m & ((1u << lane) - 1u))] = (l << 24) | c;
      n += __popc(m);
    }
    if (lane == 0) S.nc = n;
  }
  if (warp == 1) {  // tensor memory for S and O
    tmem_alloc(smem_u32(&S.tmem_base), kTmemCols);
    tmem_relinquish();
  }
  if (tid == 0) {
    mbar_init(smem_u32(&S.bar_q), 1);
    mbar_init(smem_u32(&S.bar_s), 1);
    mbar_init(smem_u32(&S.bar_pv), 1);
    mbar_init(smem_u32(&S.bar_kv[0]), 1);
    mbar_init(smem_u32(&S.bar_kv[1]), 1);
    fence_mbar_init();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) {
    const int u = warp_sorted_union<E>(S.ent, kTcBlocks * K, S.ulist, lane);
    if (lane == 0) S.nu = u;
  }
  __syncthreads();
  const int nu = S.nu;
  // membership: entry (block bi, slot s) sits at union position u
  for (int e = tid; e < kTcBlocks * K; e += kTcThreads) {
    const int v = S.ent[e];
    if (v != 0x7fffffff) {
      const int u = sorted_find(S.ulist, nu, v);
      atomicOr(&S.mask[e / K][u >> 5], 1u << (u & 31));
    }
  }

  const int nc = S.nc;
  const int nfc = (nu + kChunkBlocks - 1) / kChunkBlocks;  // fine chunks
  const int ncc = (nc + 63) / 64;                          // coarse chunks
  const int nch = nfc + ncc;
  const uint32_t base = smem_u32(sm);
  const uint32_t taddr = S.tmem_base;
  const uint32_t t_s = taddr, t_o = taddr + 64;
  const uint32_t bq = smem_u32(&S.bar_q), bs = smem_u32(&S.bar_s), bpv = smem_u32(&S.bar_pv);
  const uint32_t bkv0 = smem_u32(&S.bar_kv[0]);
  auto kbuf = [&](int buf) { return base + kOffK + (uint32_t)buf * kChunkBlocks * kTile; };
  auto vbuf = [&](int buf) { return base + kOffV + (uint32_t)buf * kChunkBlocks * kTile; };
  auto chunk_blocks = [&](int c) { return c < nfc ? min(kChunkBlocks, nu - c * kChunkBlocks) : 4; };
  auto issue_fine = [&](int c) {  // thread 0 only
    const int buf = c & 1, nb = chunk_blocks(c);
    mbar_arrive_expect_tx(bkv0 + 8u * buf, 2u * nb * kTile);
    for (int i = 0; i < nb; ++i) {
      const int y = (int)(rowbase + (size_t)S.ulist[c * kChunkBlocks + i] * 16);
      tma_load_2d(kbuf(buf) + i * kTile, &tk, 0, y, bkv0 + 8u * buf);
      tma_load_2d(vbuf(buf) + i * kTile, &tv, 0, y, bkv0 + 8u * buf);
    }
  };
  if (tid == 0) {
    int nq = 0;
    for (int bi = 0; bi < kTcBlocks; ++bi) nq += (b0 + bi < n1) ? 1 : 0;
    mbar_arrive_expect_tx(bq, nq * kTile);
    for (int bi = 0; bi < nq; ++bi)
      tma_load_2d(base + kOffQ + bi * kTile, &tq, 0, (int)(rowbase + (size_t)(b0 + bi) * 16), bq);
    for (int c = 0; c < nfc && c < 2; ++c) issue_fine(c);
  }
  for (int e = tid; e < ncc * 64; e += kTcThreads)
    S.clw[e] = (e < nc) ? p.logw[S.clist[e] >> 24] * kLog2e : -INFINITY;
  __syncthreads();  // membership masks and coarse weights complete

  // this thread's query row and column half: warp w may only touch TMEM
  // lanes 32 (w % 4) .. +31
  const int quarter = warp & 3, half = warp >> 2;
  const int r = quarter * 32 + lane;       // TMEM lane r, P row r
  const int qb = r >> 4;                   // its query block within the CTA
  const uint32_t t_row = (uint32_t)(quarter * 32) << 16;
  const int col0 = 32 * half;              // this thread's 32 of the 64 chunk columns
  const float sc2 = p.scale * kLog2e;
  float m_ref = -INFINITY, lsum = 0.f;     // lsum: this half's part of the row sum
  bool ok = mbar_wait_bounded(bq, 0);
  const uint32_t idesc_pv = idesc_bf16_f32(128, 64, 1);

  for (int c = 0; c < nch; ++c) {
    const int buf = c & 1;
    const int nb = chunk_blocks(c);
    // (A) the chunk's K and V tiles
    if (c >= nfc) {
      // coarse keys 64(c - nfc) .. +63: fp32 pyramid rows -> bf16 swizzled tiles
      const int k0 = (c - nfc) * 64;
      unsigned char* kd = sm + kOffK + buf * kChunkBlocks * kTile;
      unsigned char* vd = sm + kOffV + buf * kChunkBlocks * kTile;
      for (int e = tid; e < 64 * 8; e += kTcThreads) {
        const int key = e >> 3, j = e & 7;
        uint4 kq = make_uint4(0, 0, 0, 0), vq = make_uint4(0, 0, 0, 0);
        if (k0 + key < nc) {
          const int l = S.clist[k0 + key] >> 24, tok = S.clist[k0 + key] & 0xffffff;
          const size_t off = ((size_t)bh * (p.N >> (4 * l)) + tok) * kTcD + 8 * j;
          const float4* ks = reinterpret_cast<const float4*>(p.pk[l] + off);
          const float4* vs = reinterpret_cast<const float4*>(p.pv[l] + off);
          const float4 a0 = ks[0], a1 = ks[1], v0 = vs[0], v1 = vs[1];
          kq = make_uint4(pack_bf16(a0.x, a0.y), pack_bf16(a0.z, a0.w), pack_bf16(a1.x, a1.y), pack_bf16(a1.z, a1.w));
          vq = make_uint4(pack_bf16(v0.x, v0.y), pack_bf16(v0.z, v0.w), pack_bf16(v1.x, v1.y), pack_bf16(v1.z, v1.w));
        }
        const int dst = (key >> 4) * kTile + (int)swz(key & 15, j);
        *reinterpret_cast<uint4*>(kd + dst) = kq;
        *reinterpret_cast<uint4*>(vd + dst) = vq;
      }
      fence_proxy_async_smem();
      __syncthreads();
    } else if (ok) {
      ok = mbar_wait_bounded(bkv0 + 8u * buf, (uint32_t)((c >> 1) & 1));
    }
    // (B) S = Q K^T into tensor memory
    if (tid == 0 && ok) {
      tc_fence_after();
      const uint32_t idesc_s = idesc_bf16_f32(128, 16 * nb, 0);
#pragma unroll
      for (int ks = 0; ks < kTcD / 16; ++ks)
        tc_mma_f16(t_s, smem_desc_sw128(base + kOffQ + ks * 32, 16, 1024),
                   smem_desc_sw128(kbuf(buf) + ks * 32, 16, 1024), idesc_s, ks > 0);
      tc_commit(bs);
    }
    if (ok) ok = mbar_wait_bounded(bs, (uint32_t)(c & 1));
    tc_fence_after();
    float x[32];
    tmem_ld32(t_s + t_row + col0, x);
    tmem_wait_ld();
    // (C) the previous PV has finished: O is stable, P and the other buffer are free
    if (c > 0 && ok) ok = mbar_wait_bounded(bpv, (uint32_t)((c - 1) & 1));
    tc_fence_after();
    // (D) prefetch the next fine chunk into the buffer just freed
    if (tid == 0 && ok && c + 1 < nfc && c + 1 >= 2) issue_fine(c + 1);
    // (E) scores -> probabilities of this half row
    if (c < nfc) {
      const int u0 = c * kChunkBlocks;
      const uint32_t bits = (S.mask[qb][u0 >> 5] >> (u0 & 31)) & 0xFu;
#pragma unroll
      for (int i = 0; i < 2; ++i) {
        const int blk = 2 * half + i;  // key block of the chunk for columns 16i..16i+15
        const bool sel = (blk < nb) && ((bits >> blk) & 1u);
#pragma unroll
        for (int j = 0; j < 16; ++j) x[16 * i + j] = sel ? x[16 * i + j] * sc2 : -INFINITY;
      }
    } else {
      const int k0 = (c - nfc) * 64 + col0;
#pragma unroll
      for (int j = 0; j < 32; ++j) x[j] = fmaf(x[j], sc2, S.clw[k0 + j]);
    }
    bool hi = false;
#pragma unroll
    for (int j = 0; j < 32; ++j) hi |= x[j] > m_ref + kRescaleLog2;
    if (__syncthreads_or(hi)) {  // raise the running max of some rows
      float mx = -INFINITY;
#pragma unroll
      for (int j = 0; j < 32; ++j) mx = fmaxf(mx, x[j]);
      S.red[half][r] = mx;
      __syncthreads();
      mx = fmaxf(S.red[0][r], S.red[1][r]);
      const bool up = mx > m_ref + kRescaleLog2;
      const float corr = up ? ex2_approx(m_ref - mx) : 1.f;  // 2^-inf = 0 for a first max
      if (up) m_ref = mx;
      lsum *= corr;
      if (c > 0) {  // rescale this half row of O in tensor memory (whole warp)
        float o[32];
        tmem_ld32(t_o + t_row + col0, o);
        tmem_wait_ld();
#pragma unroll
        for (int j = 0; j < 32; ++j) o[j] *= corr;
        tmem_st32(t_o + t_row + col0, o);
        tmem_wait_st();
      }
      __syncthreads();  // S.red reused below
    }
    const float mb = (m_ref == -INFINITY) ? 0.f : m_ref;
    unsigned char* prow = sm + kOffP + r * 128;
#pragma unroll
    for (int jj = 0; jj < 4; ++jj) {
      float pv[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        pv[e] = ex2_approx(x[8 * jj + e] - mb);
        lsum += pv[e];
      }
      const uint4 pk = make_uint4(pack_bf16(pv[0], pv[1]), pack_bf16(pv[2], pv[3]),
                                  pack_bf16(pv[4], pv[5]), pack_bf16(pv[6], pv[7]));
      *reinterpret_cast<uint4*>(prow + (((4 * half + jj) ^ (r & 7)) << 4)) = pk;
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    // (F) O += P V
    if (tid == 0 && ok) {
      tc_fence_after();
      for (int ks = 0; ks < nb; ++ks)
        tc_mma_f16(t_o, smem_desc_sw128(base + kOffP + ks * 32, 16, 1024),
                   smem_desc_sw128(vbuf(buf) + ks * kTile, 8192, 1024), idesc_pv, (c > 0 || ks > 0));
      tc_commit(bpv);
    }
  }
  if (nch > 0 && ok) ok = mbar_wait_bounded(bpv, (uint32_t)((nch - 1) & 1));
  tc_fence_after();

  // ---- epilogue: O = acc / l, LSE = ln(sum) = (m + log2 l) ln 2
  S.red[half][r] = lsum;
  __syncthreads();
  const float ltot = S.red[0][r] + S.red[1][r];
  float o[32];
  tmem_ld32(t_o + t_row + col0, o);
  tmem_wait_ld();
  const int b = b0 + qb;
  if (b < n1) {
    const bool has = ltot > 0.f && nch > 0;
    const float inv = has ? 1.f / ltot : 0.f;
    const size_t tok = rowbase + (size_t)b0 * 16 + r;
    bf16* O = static_cast<bf16*>(p.out) + tok * kTcD + col0;
#pragma unroll
    for (int jj = 0; jj < 4; ++jj) {
      uint4 pk = make_uint4(0, 0, 0, 0);
      if (has)
        pk = make_uint4(pack_bf16(o[8 * jj] * inv, o[8 * jj + 1] * inv), pack_bf16(o[8 * jj + 2] * inv, o[8 * jj + 3] * inv),
                        pack_bf16(o[8 * jj + 4] * inv, o[8 * jj + 5] * inv), pack_bf16(o[8 * jj + 6] * inv, o[8 * jj + 7] * inv));
      reinterpret_cast<uint4*>(O)[jj] = pk;
    }
    if (half == 0) p.lse[tok] = has ? (m_ref + log2f(ltot)) * kLn2 : -INFINITY;
  }
  if (!ok) flags |= LLSA_DEV_TIMEOUT;
  flags = __reduce_or_sync(0xffffffffu, flags);
  if (lane == 0) report_status(p.status, flags);
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(taddr, kTmemCols);
  }
}

}  // namespace

// maps: Q, K, V as 2D [B*H*N rows, 64 cols] bf16, box 16 x 64, 128-byte swizzle.
cudaError_t launch_attn_fwd_tc(const AttnParams& p, const CUtensorMap* maps, cudaStream_t s) {
  const size_t smem = 1024 + kTileBytes + sizeof(TcShared);
  const int ent = kTcBlocks * p.K;
  auto kern = (ent <= 32)   ? attn_fwd_tc_kernel<1>
              : (ent <= 64) ? attn_fwd_tc_kernel<2>
              : (ent <= 128) ? attn_fwd_tc_kernel<4>
                             : attn_fwd_tc_kernel<8>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const int n1 = p.N / kBlock;
  dim3 grid((n1 + kTcBlocks - 1) / kTcBlocks, p.B * p.H);
  kern<<<grid, kTcThreads, smem, s>>>(maps[0], maps[1], maps[2], p);
  return cudaGetLastError();
}

}  // namespace llsa
