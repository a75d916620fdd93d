// Sparse attention forward with hierarchical KV enrichment and KV
// reweighting on the 5th-generation tensor cores (tcgen05), bf16, D = 64 or
// 128 (Step 3 of the howistudyai explainer of "Trainable Log-linear Sparse
// Attention for Efficient Diffusion Transformers": attention of each query
// block over the fine tokens of its selected blocks plus the pooled tokens
// selected at the coarser levels, each coarse key weighted).
//
// A CTA owns 8 sibling 16-token query blocks: 128 query rows, the M of one
// tcgen05 MMA, so every MMA uses the full datapath.  Siblings select
// overlapping key blocks; the CTA walks the sorted union U of their
// selections (about 2.7 key blocks per query block at the 256x256-pixel
// size instead of 8 gathered per block) in chunks of 4 key blocks, and each
// row masks the blocks its own query block did not select.  The coarse keys
// (identical for all 8 blocks: they share every coarse ancestor) come first,
// as chunks converted from the fp32 pyramid in the prologue.
//
//   warp 0      TMA loads: Q once, then the K and V tiles of each union chunk
//               into a ring of stages (2D tiles of 16 rows, 128-byte swizzle,
//               no multicast);
//   warp 1      one thread issues the MMAs (and the warp owns tensor memory):
//                 S_c  = Q K_c^T            (M 128, N 16..64, K = D) into one
//                                           of two S buffers in TMEM,
//                 O   += P_c [V_c | 1]      (A = P from TMEM, M 128,
//                                           N = D + 16, K 16 per key block);
//               the 16 extra columns multiply P by ones, so the tensor core
//               also accumulates l = sum of the bf16 probabilities actually
//               used for O (numerator and denominator agree exactly);
//   warps 2-5   softmax, one thread per query row: read S_c from TMEM, mask,
//               scale, keep the exact running maximum m of the row (when it
//               rises, O and l are rescaled in TMEM), write P_c = 2^(s - m)
//               as bf16 into TMEM; at the end the epilogue
//               (O / l, LSE, and optionally the bf16 residual of O) is staged
//               through shared memory and leaves by TMA stores.
// S_{c+1} runs on the tensor core while the softmax works on chunk c, and
// PV_c overlaps the softmax of chunk c+1.  Every wait is bounded; on a
// time-out the kernel reports LLSA_DEV_TIMEOUT, drains its copies and
// returns.

#include <math.h>

#include "keyset.cuh"
#include "sm100_ptx.cuh"
#include "tcgen05.cuh"

namespace llsa {

namespace {

constexpr int kQB = 8;          // query blocks per CTA (128 rows)
constexpr int kCT = 4;          // key tiles (blocks of 16 keys) per chunk
constexpr int kSub = 2048;      // a 16-row x 64-column bf16 sub-tile (128-byte swizzle)
constexpr int kThreads = 192;   // 6 warps
constexpr int kMaxU = kQB * kMaxK;                // 256
constexpr int kMaxCoarse = (kMaxL - 1) * kMaxK;   // 160
constexpr int kMaxCoarseChunks = (kMaxCoarse + 63) / 64;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
// The reference of the probabilities is the exact running maximum, so the
// largest probability of a row is exactly 1 and its bf16 rounding is exact.
// A reference allowed to lag (up to 2^8, as some FlashAttention kernels do)
// let the rounding of the dominant probability through: with the paper's
// level weights on caller indices a few O elements left the 2e-2 band.

template <int D>
struct Cfg {
  static constexpr int H = D / 64;                        // 64-column halves
  static constexpr int kStages = (D == 64) ? 3 : 2;
  static constexpr int kQBytes = kQB * H * kSub;          // [half][8 tiles]
  static constexpr int kKChunk = H * kCT * kSub;          // [half][4 tiles]
  // D = 64: [4 tiles] (the ones block is one shared region);
  // D = 128: [half 0: 4 tiles][half 1: 4 tiles][ones: 4 tiles]
  static constexpr int kVChunk = (D == 64 ? 1 : 3) * kCT * kSub;
  static constexpr int kOCols = D + 16;
  static constexpr uint32_t kTmemCols = (D == 64) ? 256 : 512;
  static constexpr uint32_t kColS = 0;    // two S buffers of 64 columns
  static constexpr uint32_t kColP = 128;  // P: 64 bf16 per row = 32 columns
  static constexpr uint32_t kColO = 160;  // O and l: D + 16 columns
  static_assert(kStages * kKChunk >= kQBytes, "the residual is staged in the K ring");
};

struct FwdShared {
  uint64_t bar_q, bar_full[3], bar_empty[3], bar_s[2], bar_p, bar_pv, bar_done;
  uint32_t tmem_base;
  int nu, nc;
  int ent[kQB * kMaxK];     // the 8 blocks' selections, 0x7fffffff when unused
  int ulist[kMaxU];         // sorted union of the selections
  uint32_t umask[kMaxU];    // bit b: query block b selected union entry u
  int clist[kMaxCoarse];    // coarse keys: level << 24 | token
  float clw[kMaxCoarseChunks * 64];  // their log2 weights, -inf for pads
};

// Shared-memory offsets (bytes from a 1024-aligned base).
template <int D>
struct Layout {
  uint32_t q, k, v, ck, cv, ones, end;
  __host__ __device__ Layout(int ncc) {
    using C = Cfg<D>;
    q = 0;
    k = q + C::kQBytes;
    v = k + C::kStages * C::kKChunk;
    ck = v + C::kStages * C::kVChunk;
    cv = ck + ncc * C::kKChunk;
    ones = cv + ncc * C::kVChunk;
    end = ones + (D == 64 ? kSub : 0);
  }
};

// Byte offset of 16-byte chunk jj (0..7) of row r in a 128-byte-swizzled
// region whose rows are 128 bytes (the TMA layout of every tile here).
__device__ __forceinline__ uint32_t sw128(int r, int jj) {
  return (uint32_t)(r * 128 + ((jj ^ (r & 7)) << 4));
}

template <int D, int E>
__global__ void __launch_bounds__(kThreads)
attn_fwd_tc_kernel(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
                   const __grid_constant__ CUtensorMap tv, const __grid_constant__ CUtensorMap to,
                   const __grid_constant__ CUtensorMap tr, AttnParams p, int ncc_max) {
  using C = Cfg<D>;
  extern __shared__ unsigned char smem_raw[];
  unsigned char* sm = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  const Layout<D> lay(ncc_max);
  FwdShared& S = *reinterpret_cast<FwdShared*>(sm + lay.end);
  const uint32_t base = smem_u32(sm);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int bh = blockIdx.y;
  const int n1 = p.N >> 4;
  const int b0 = blockIdx.x * kQB;
  const int K = p.K;
  const size_t rowbase = (size_t)bh * p.N;
  int flags = 0;
  bool ok = true;

  // ---------------------------------------------------------------- prologue
  if (warp == 0) {  // the 8 blocks' fine selections (the library's entry rule)
    for (int bi = 0; bi < kQB; ++bi) {
      const int b = b0 + bi;
      const bool on = (b < n1) && lane < K;
      const int v = on ? p.idx[1][((size_t)bh * n1 + b) * K + lane] : -1;
      const bool used = warp_row_used(v, lane, n1, on, flags);
      if (lane < K) S.ent[bi * K + lane] = used ? v : 0x7fffffff;
    }
  } else if (warp == 1) {
    tmem_alloc(smem_u32(&S.tmem_base), C::kTmemCols);
    tmem_relinquish();
  } else if (warp == 2) {  // coarse keys of levels 2..L, shared by the 8 blocks
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
  } else if (tid == 96) {
    mbar_init(smem_u32(&S.bar_q), 1);
    for (int i = 0; i < 3; ++i) {
      mbar_init(smem_u32(&S.bar_full[i]), 1);
      mbar_init(smem_u32(&S.bar_empty[i]), 1);
    }
    mbar_init(smem_u32(&S.bar_s[0]), 1);
    mbar_init(smem_u32(&S.bar_s[1]), 1);
    mbar_init(smem_u32(&S.bar_p), 128);
    mbar_init(smem_u32(&S.bar_pv), 1);
    mbar_init(smem_u32(&S.bar_done), 1);
    fence_mbar_init();
  }
  for (int e = tid; e < kMaxU; e += kThreads) S.umask[e] = 0u;
  tc_fence_before();
  __syncthreads();
  tc_fence_after();

  const int nc = S.nc;
  const int nct = (nc + 15) >> 4;          // coarse key tiles
  const int ncc = (nct + kCT - 1) / kCT;   // coarse chunks
  int issued = 0;                          // fine chunks whose loads warp 0 has issued
  int nu = 0;
  auto kslot = [&](int s) { return base + lay.k + (uint32_t)s * C::kKChunk; };
  auto vslot = [&](int s) { return base + lay.v + (uint32_t)s * C::kVChunk; };
  auto issue_chunk = [&](int f) {  // one thread of warp 0
    const int slot = f % C::kStages;
    const int t0 = f * kCT, nt = min(kCT, nu - t0);
    const uint32_t bar = smem_u32(&S.bar_full[slot]);
    mbar_arrive_expect_tx(bar, (uint32_t)nt * 2u * C::H * kSub);
    for (int t = 0; t < nt; ++t) {
      const int y = (int)(rowbase + (size_t)S.ulist[t0 + t] * 16);
#pragma unroll
      for (int h = 0; h < C::H; ++h) {
        tma_load_2d(kslot(slot) + (uint32_t)(h * kCT + t) * kSub, &tk, 64 * h, y, bar);
        tma_load_2d(vslot(slot) + (uint32_t)(h * kCT + t) * kSub, &tv, 64 * h, y, bar);
      }
    }
  };

  if (warp == 0) {
    const int cnt = kQB * K;
    nu = warp_sorted_union<E>(S.ent, cnt, S.ulist, lane);
    __syncwarp();
    for (int e = lane; e < cnt; e += 32) {
      const int v = S.ent[e];
      if (v != 0x7fffffff) atomicOr(&S.umask[sorted_find(S.ulist, nu, v)], 1u << (e / K));
    }
    if (lane == 0) {
      S.nu = nu;
      int nq = 0;
      for (int bi = 0; bi < kQB; ++bi) nq += (b0 + bi < n1) ? 1 : 0;
      const uint32_t bq = smem_u32(&S.bar_q);
      mbar_arrive_expect_tx(bq, (uint32_t)nq * C::H * kSub);
      for (int bi = 0; bi < nq; ++bi)
#pragma unroll
        for (int h = 0; h < C::H; ++h)
          tma_load_2d(base + lay.q + (uint32_t)(h * kQB + bi) * kSub, &tq, 64 * h,
                      (int)(rowbase + (size_t)(b0 + bi) * 16), bq);
      const int nfc = (nu + kCT - 1) / kCT;
      for (; issued < nfc && issued < C::kStages; ++issued) issue_chunk(issued);
    }
  } else {
    // coarse K/V rows: fp32 pyramid -> bf16 swizzled tiles (zero rows past nc)
    const int t1 = tid - 32;
    for (int e = t1; e < nct * 16 * (D / 8); e += kThreads - 32) {
      const int key = e / (D / 8), j = e % (D / 8);
      const int tile = key >> 4, row = key & 15, cc = tile / kCT, t = tile % kCT, h = j >> 3;
      uint4 kq = make_uint4(0, 0, 0, 0), vq = make_uint4(0, 0, 0, 0);
      if (key < nc) {
        const int l = S.clist[key] >> 24, c = S.clist[key] & 0xffffff;
        const size_t off = ((size_t)bh * (p.N >> (4 * l)) + c) * D + 8 * j;
        const float4* ks = reinterpret_cast<const float4*>(p.pk[l] + off);
        const float4* vs = reinterpret_cast<const float4*>(p.pv[l] + off);
        const float4 a0 = ks[0], a1 = ks[1], v0 = vs[0], v1 = vs[1];
        kq = make_uint4(pack_bf16(a0.x, a0.y), pack_bf16(a0.z, a0.w), pack_bf16(a1.x, a1.y), pack_bf16(a1.z, a1.w));
        vq = make_uint4(pack_bf16(v0.x, v0.y), pack_bf16(v0.z, v0.w), pack_bf16(v1.x, v1.y), pack_bf16(v1.z, v1.w));
      }
      const uint32_t in_chunk = (uint32_t)(h * kCT + t) * kSub + sw128(row, j & 7);
      *reinterpret_cast<uint4*>(sm + lay.ck + (uint32_t)cc * C::kKChunk + in_chunk) = kq;
      *reinterpret_cast<uint4*>(sm + lay.cv + (uint32_t)cc * C::kVChunk + in_chunk) = vq;
    }
    // the ones that make the PV MMA also sum P
    const uint4 one4 = make_uint4(0x3f803f80u, 0x3f803f80u, 0x3f803f80u, 0x3f803f80u);
    if (D == 64) {
      for (int e = t1; e < kSub / 16; e += kThreads - 32)
        reinterpret_cast<uint4*>(sm + lay.ones)[e] = one4;
    } else {
      const int nchunks = C::kStages + ncc_max;
      for (int e = t1; e < nchunks * (kCT * kSub / 16); e += kThreads - 32) {
        const int ch = e / (kCT * kSub / 16), w = e % (kCT * kSub / 16);
        const uint32_t cb = ch < C::kStages ? lay.v + (uint32_t)ch * C::kVChunk
                                            : lay.cv + (uint32_t)(ch - C::kStages) * C::kVChunk;
        reinterpret_cast<uint4*>(sm + cb + 2 * kCT * kSub)[w] = one4;
      }
    }
    for (int e = t1; e < ncc * 64; e += kThreads - 32)
      S.clw[e] = (e < nc) ? p.logw[S.clist[e] >> 24] * kLog2e : -INFINITY;
  }
  fence_proxy_async_smem();  // generic writes above -> MMA operand reads
  __syncthreads();
  nu = S.nu;
  const int nfc = (nu + kCT - 1) / kCT;  // fine chunks
  const int nch = ncc + nfc;
  const uint32_t tbase = S.tmem_base;

  // chunk c: coarse for c < ncc, else fine chunk c - ncc
  auto chunk_tiles = [&](int c) { return c < ncc ? min(kCT, nct - c * kCT) : min(kCT, nu - (c - ncc) * kCT); };

  if (warp == 0) {
    // ------------------------------------------------------------ loader
    if (lane == 0) {
      for (; issued < nfc && ok; ++issued) {
        const int slot = issued % C::kStages;
        ok = mbar_wait_bounded(smem_u32(&S.bar_empty[slot]), (uint32_t)((issued / C::kStages - 1) & 1));
        if (ok) issue_chunk(issued);
      }
      // no copy may still be landing when the CTA exits: wait for the last
      // chunk of every stage (done long ago on the normal path) and for Q
      for (int s = 0; s < C::kStages && s < issued; ++s) {
        const int last = s + ((issued - 1 - s) / C::kStages) * C::kStages;
        if (!mbar_wait_bounded(smem_u32(&S.bar_full[s]), (uint32_t)((last / C::kStages) & 1))) ok = false;
      }
      if (!mbar_wait_bounded(smem_u32(&S.bar_q), 0)) ok = false;
    }
  } else if (warp == 1) {
    // --------------------------------------------------------- MMA issuer
    if (lane == 0) {
      ok = mbar_wait_bounded(smem_u32(&S.bar_q), 0);
      const uint32_t idesc_pv = idesc_bf16_f32(128, C::kOCols, 1, 0);
      for (int c = 0; c <= nch && ok; ++c) {
        if (c < nch) {
          const int nt = chunk_tiles(c);
          uint32_t kaddr;
          if (c < ncc) {
            kaddr = base + lay.ck + (uint32_t)c * C::kKChunk;
          } else {
            const int f = c - ncc;
            ok = mbar_wait_bounded(smem_u32(&S.bar_full[f % C::kStages]), (uint32_t)((f / C::kStages) & 1));
            if (!ok) break;
            kaddr = kslot(f % C::kStages);
          }
          tc_fence_after();
          const uint32_t idesc_s = idesc_bf16_f32(128, 16 * nt, 0, 0);
#pragma unroll
          for (int ks = 0; ks < D / 16; ++ks) {
            const int h = ks >> 2, kk = ks & 3;
            tc_mma_f16(tbase + C::kColS + (uint32_t)(c & 1) * 64,
                       smem_desc_sw128(base + lay.q + (uint32_t)(h * kQB) * kSub + kk * 32, 16, 1024),
                       smem_desc_sw128(kaddr + (uint32_t)(h * kCT) * kSub + kk * 32, 16, 1024), idesc_s, ks > 0);
          }
          tc_commit(smem_u32(&S.bar_s[c & 1]));
        }
        if (c >= 1) {
          const int cp = c - 1, nt = chunk_tiles(cp);
          const uint32_t vaddr = cp < ncc ? base + lay.cv + (uint32_t)cp * C::kVChunk
                                          : vslot((cp - ncc) % C::kStages);
          ok = mbar_wait_bounded(smem_u32(&S.bar_p), (uint32_t)(cp & 1));
          if (!ok) break;
          tc_fence_after();
          for (int t = 0; t < nt; ++t) {
            const uint32_t vt = vaddr + (uint32_t)t * kSub;
            const uint64_t bdesc = (D == 64) ? smem_desc_sw128(vt, base + lay.ones - vt, 1024)
                                             : smem_desc_sw128(vt, kCT * kSub, 1024);
            tc_mma_f16_ts(tbase + C::kColO, tbase + C::kColP + (uint32_t)t * 8, bdesc, idesc_pv,
                          (cp > 0 || t > 0) ? 1u : 0u);
          }
          tc_commit(smem_u32(&S.bar_pv));
          if (cp >= ncc) tc_commit(smem_u32(&S.bar_empty[(cp - ncc) % C::kStages]));
        }
      }
      // every MMA of this CTA has completed before tensor memory is freed
      tc_commit(smem_u32(&S.bar_done));
      if (!mbar_wait_bounded(smem_u32(&S.bar_done), 0)) ok = false;
    }
  } else {
    // ----------------------------------------------- softmax and epilogue
    const int q4 = warp & 3;                      // TMEM lane quarter of this warp
    const int r = q4 * 32 + lane;                 // query row = TMEM lane
    const int qb = r >> 4;                        // its query block in the CTA
    const uint32_t lane_off = (uint32_t)(q4 * 32) << 16;
    const float sc2 = p.scale * kLog2e;
    float m_ref = -INFINITY;
    for (int c = 0; c < nch && ok; ++c) {
      const bool coarse = c < ncc;
      const int nt = chunk_tiles(c);
      const int f = c - ncc;
      ok = mbar_wait_bounded(smem_u32(&S.bar_s[c & 1]), (uint32_t)((c >> 1) & 1));
      if (!ok) break;
      tc_fence_after();
      float x[64];
      bool live[kCT];  // some row of this warp takes key tile t
      uint32_t sel[kCT];
#pragma unroll
      for (int t = 0; t < kCT; ++t) {
        const uint32_t bits = (!coarse && t < nt) ? S.umask[f * kCT + t] : 0u;
        sel[t] = (bits >> qb) & 1u;
        live[t] = t < nt && (coarse || ((bits >> (2 * q4)) & 3u) != 0u);
        if (live[t]) tmem_ld16(tbase + lane_off + C::kColS + (uint32_t)(c & 1) * 64 + 16 * t, x + 16 * t);
      }
      tmem_wait_ld();
      float mx = -INFINITY;
#pragma unroll
      for (int t = 0; t < kCT; ++t) {
        if (live[t]) {
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            const float lw = coarse ? S.clw[c * 64 + 16 * t + j] : (sel[t] ? 0.f : -INFINITY);
            x[16 * t + j] = fmaf(x[16 * t + j], sc2, lw);
            mx = fmaxf(mx, x[16 * t + j]);
          }
        }
      }
      // P of the previous chunk has been read (and O is final up to it)
      if (c > 0) {
        ok = mbar_wait_bounded(smem_u32(&S.bar_pv), (uint32_t)((c - 1) & 1));
        if (!ok) break;
      }
      tc_fence_after();
      const bool need = (m_ref != -INFINITY) && (mx > m_ref);
      if (m_ref == -INFINITY) m_ref = mx;  // O of this row is still exactly zero
      if (__any_sync(0xffffffffu, need)) {  // the maximum rose: rescale O (and l) in TMEM
        const float corr = need ? ex2_approx(m_ref - mx) : 1.f;
        if (need) m_ref = mx;
        const uint64_t cc = f2_make(corr, corr);
#pragma unroll 1
        for (int cb = 0; cb < C::kOCols; cb += 16) {
          float o[16];
          tmem_ld16(tbase + lane_off + C::kColO + cb, o);
          tmem_wait_ld();
#pragma unroll
          for (int j = 0; j < 16; j += 2) {
            const float2 v = f2_split(f2_mul(f2_make(o[j], o[j + 1]), cc));
            o[j] = v.x;
            o[j + 1] = v.y;
          }
          tmem_st16(tbase + lane_off + C::kColO + cb, o);
        }
      }
      const float mb = (m_ref == -INFINITY) ? 0.f : m_ref;
      uint32_t pk[32];
#pragma unroll
      for (int t = 0; t < kCT; ++t) {
        if (live[t]) {
#pragma unroll
          for (int j = 0; j < 8; ++j)
            pk[8 * t + j] = pack_bf16(ex2_approx(x[16 * t + 2 * j] - mb), ex2_approx(x[16 * t + 2 * j + 1] - mb));
        } else {
#pragma unroll
          for (int j = 0; j < 8; ++j) pk[8 * t + j] = 0u;
        }
      }
      tmem_st32u(tbase + lane_off + C::kColP, pk);
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(smem_u32(&S.bar_p));
    }
    if (nch > 0 && ok) ok = mbar_wait_bounded(smem_u32(&S.bar_pv), (uint32_t)((nch - 1) & 1));
    tc_fence_after();

    // ---- epilogue: O = acc / l, LSE = (m + log2 l) ln 2, residual of O
    float lsum = 0.f;
    if (nch > 0) {
      float lv[16];
      tmem_ld16(tbase + lane_off + C::kColO + D, lv);
      tmem_wait_ld();
      lsum = lv[0];
    }
    const bool has = ok && nch > 0 && lsum > 0.f;
    const float inv = has ? 1.f / lsum : 0.f;
    const int b = b0 + qb;
    const size_t tok = rowbase + (size_t)b0 * 16 + r;
    const bool full_cta = (b0 + kQB <= n1);
    bf16* Og = static_cast<bf16*>(p.out);
    bf16* Rg = static_cast<bf16*>(p.o_res);
#pragma unroll 1
    for (int h = 0; h < C::H; ++h) {
      float o[64];
      if (nch > 0) {
#pragma unroll
        for (int q = 0; q < 4; ++q) tmem_ld16(tbase + lane_off + C::kColO + 64 * h + 16 * q, o + 16 * q);
        tmem_wait_ld();
      }
#pragma unroll
      for (int jj = 0; jj < 8; ++jj) {
        float a[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) a[e] = has ? o[8 * jj + e] * inv : 0.f;
        const uint4 ov = make_uint4(pack_bf16(a[0], a[1]), pack_bf16(a[2], a[3]), pack_bf16(a[4], a[5]),
                                    pack_bf16(a[6], a[7]));
        const uint4 rv = make_uint4(pack_bf16(a[0] - bf16x2_lo(ov.x), a[1] - bf16x2_hi(ov.x)),
                                    pack_bf16(a[2] - bf16x2_lo(ov.y), a[3] - bf16x2_hi(ov.y)),
                                    pack_bf16(a[4] - bf16x2_lo(ov.z), a[5] - bf16x2_hi(ov.z)),
                                    pack_bf16(a[6] - bf16x2_lo(ov.w), a[7] - bf16x2_hi(ov.w)));
        if (full_cta) {  // staged (Q region and K ring are free now) for the TMA stores
          const uint32_t off = (uint32_t)(h * kQB) * kSub + sw128(r, jj);
          *reinterpret_cast<uint4*>(sm + lay.q + off) = ov;
          if (Rg != nullptr) *reinterpret_cast<uint4*>(sm + lay.k + off) = rv;
        } else if (b < n1) {
          reinterpret_cast<uint4*>(Og + tok * D + 64 * h)[jj] = ov;
          if (Rg != nullptr) reinterpret_cast<uint4*>(Rg + tok * D + 64 * h)[jj] = rv;
        }
      }
    }
    if (b < n1) p.lse[tok] = has ? (m_ref + log2f(lsum)) * kLn2 : -INFINITY;
    if (full_cta) {
      fence_proxy_async_smem();
      asm volatile("bar.sync 1, 128;" ::: "memory");  // the 4 softmax warps
      if (warp == 2 && lane == 0) {
        const int y = (int)(rowbase + (size_t)b0 * 16);
        for (int h = 0; h < C::H; ++h) {
          tma_store_2d(&to, 64 * h, y, base + lay.q + (uint32_t)(h * kQB) * kSub);
          if (Rg != nullptr) tma_store_2d(&tr, 64 * h, y, base + lay.k + (uint32_t)(h * kQB) * kSub);
        }
        bulk_commit_group();
        bulk_wait_all();
      }
    }
  }

  if (!ok) flags |= LLSA_DEV_TIMEOUT;
  flags = __reduce_or_sync(0xffffffffu, flags);
  if (lane == 0) report_status(p.status, flags);
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tbase, C::kTmemCols);
  }
}

template <int D>
size_t smem_bytes(int ncc) {
  return 1024 + Layout<D>(ncc).end + sizeof(FwdShared);
}

template <int D>
cudaError_t launch_typed(const AttnParams& p, const CUtensorMap* maps, cudaStream_t s) {
  const int ncc = ((p.Kc + 15) / 16 + kCT - 1) / kCT;
  const size_t smem = smem_bytes<D>(ncc);
  const int ent = kQB * p.K;
  auto kern = (ent <= 32)    ? attn_fwd_tc_kernel<D, 1>
              : (ent <= 64)  ? attn_fwd_tc_kernel<D, 2>
              : (ent <= 128) ? attn_fwd_tc_kernel<D, 4>
                             : attn_fwd_tc_kernel<D, 8>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout, (int)cudaSharedmemCarveoutMaxShared);
  if (e != cudaSuccess) return e;
  const int n1 = p.N / kBlock;
  dim3 grid((n1 + kQB - 1) / kQB, p.B * p.H);
  kern<<<grid, kThreads, smem, s>>>(maps[0], maps[1], maps[2], maps[3], maps[4], p, ncc);
  return cudaGetLastError();
}

}  // namespace

// Shared memory the tcgen05 forward needs for this problem (host check: the
// caller uses the warp-MMA forward when it exceeds the per-CTA limit).
size_t attn_fwd_tc_smem(const AttnParams& p) {
  const int ncc = ((p.Kc + 15) / 16 + kCT - 1) / kCT;
  return p.D == 64 ? smem_bytes<64>(ncc) : smem_bytes<128>(ncc);
}

// maps: Q, K, V as 2D [B*H*N rows, D cols] bf16, box 16 x 64, 128-byte
// swizzle; O and its residual (maps 3, 4) the same with box 128 x 64 (stores).
cudaError_t launch_attn_fwd_tc(const AttnParams& p, const CUtensorMap* maps, cudaStream_t s) {
  return (p.D == 64) ? launch_typed<64>(p, maps, s) : launch_typed<128>(p, maps, s);
}

}  // namespace llsa
