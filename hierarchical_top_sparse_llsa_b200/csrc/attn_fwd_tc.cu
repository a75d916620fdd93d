// Sparse attention forward with hierarchical KV enrichment and KV
// reweighting on the 5th-generation tensor cores (tcgen05), bf16, D = 64 or
// 128 (Step 3 of the howistudyai explainer of "Trainable Log-linear Sparse
// Attention for Efficient Diffusion Transformers": attention of each query
// block over the fine tokens of its selected blocks plus the pooled tokens
// selected at the coarser levels, each coarse key weighted).
//
// Work unit: a group of 8 sibling 16-token query blocks = 128 query rows, the
// M of one tcgen05 MMA.  Siblings select overlapping key blocks; a group
// walks the sorted union U of their selections (about 2.7 key blocks per
// query block at the 256x256-pixel size instead of 8 gathered per block) in
// chunks of 8 key blocks (4 at D = 128), each row masking the blocks its own
// query block did not select.  The coarse keys (the same for all 8 blocks: they share every
// coarse ancestor) come first, converted from the fp32 pyramid.
//
// The kernel is persistent (one CTA per SM walks groups g = CTA, CTA + grid,
// ...) and warp-specialised, so the set-up of group g+1 and the epilogue of
// group g-1 overlap the arithmetic of group g:
//   warp 12     fine prep: reads the 8 index rows and builds the union and the
//               membership masks, into the group buffer g % 2;
//   warp 15     coarse prep: builds the coarse list, converts the coarse K/V
//               tiles and TMA-loads Q;
//   warp 14     TMA loads of the K and V tiles of each union chunk into a
//               ring of stages (2D tiles of 16 rows, 128-byte swizzle, no
//               multicast);
//   warp 13     one thread issues the MMAs (the warp owns tensor memory):
//                 S_c = Q K_c^T       (M 128, N 16..128, K = D) into one of
//                                     two S buffers in TMEM,
//                 O  += P_c V_c       (A = P read from TMEM, M 128, N = D,
//                                     K 16 per key block) into the O buffer
//                                     g % 2;
//   warps 0-7   softmax, two threads per query row (each one half of the
//               chunk's columns; the row maximum is combined through shared
//               memory), so two softmax warps share each SM sub-partition and
//               hide each other's TMEM-load latency: read S_c from TMEM, mask,
//               scale, keep the exact running maximum of the row (when it
//               rises, the O row is rescaled in TMEM), write P_c = 2^(s - m)
//               as bf16 into TMEM and add it to the row sum l in fp32;
//   warps 8-11  epilogue, one thread per query row: O / l, LSE and optionally
//               the bf16 residual of O, each row stored as 16-byte chunks.
// S_{c+1} runs on the tensor core while the softmax works on chunk c, and
// PV_c overlaps the softmax of chunk c+1.  Every wait is bounded; on a time-out the kernel
// reports LLSA_DEV_TIMEOUT, drains its copies and returns.

#include <math.h>

#include "keyset.cuh"
#include "sm100_ptx.cuh"
#include "tcgen05.cuh"

namespace llsa {

namespace {

constexpr int kQB = 8;          // query blocks per group (128 rows)
constexpr int kSub = 2048;      // a 16-row x 64-column bf16 sub-tile (128-byte swizzle)
// 16 warps in 4 warpgroups.  Warpgroups 0 and 1: softmax, two threads per
// query row (warps w and w + 4 share the TMEM lane quarter w % 4 and take one
// half of each chunk's columns each).  Warpgroup 2: epilogue, one thread per
// query row.  Warpgroup 3: fine prep, MMA issue, K/V loads, coarse prep.
constexpr int kThreads = 512;
constexpr int kWarpEpi0 = 8, kWarpFine = 12, kWarpMma = 13, kWarpLoad = 14, kWarpCoarse = 15;
constexpr int kSoftmaxWarps = 8, kEpiWarps = 4;
// Registers per thread: the launch gives every thread kRegLaunch; then the
// control warpgroup and the epilogue give some back (setmaxnreg.dec) and the
// softmax warpgroups take them (setmaxnreg.inc).  The shares must not exceed
// what the CTA was launched with, or the increase would wait forever; the
// host checks the compiled count before every launch.
constexpr int kRegLaunch = 128, kRegSoftmax = 160, kRegEpi = 88, kRegCtl = 104;
static_assert(256 * kRegSoftmax + 128 * kRegEpi + 128 * kRegCtl <= kThreads * kRegLaunch, "register split");
constexpr int kMaxU = kQB * kMaxK;                // 256
constexpr int kMaxCoarse = (kMaxL - 1) * kMaxK;   // 160
constexpr int kMaxClw = 256;                     // coarse columns, chunk-padded
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
// The reference of the probabilities is the exact running maximum, so the
// largest probability of a row is exactly 1 and its bf16 rounding is exact.
// A reference allowed to lag (up to 2^8, as some FlashAttention kernels do)
// let the rounding of the dominant probability through: with the paper's
// level weights on caller indices a few O elements left the 2e-2 band.

template <int D>
struct Cfg {
  static constexpr int H = D / 64;                 // 64-column halves
  static constexpr int kCT = (D == 64) ? 8 : 4;    // key tiles (blocks of 16 keys) per chunk
  static constexpr int kKeys = 16 * kCT;           // keys per chunk: the N of S = Q K^T
  static constexpr int kStages = (D == 64) ? 3 : 2;
  static constexpr int kQBytes = kQB * H * kSub;   // [half][8 tiles]
  static constexpr int kChunk = H * kCT * kSub;    // K or V chunk: [half][kCT tiles]
  static constexpr uint32_t kTmemCols = 512;
  static constexpr uint32_t kColS = 0;                      // two S buffers of kKeys columns
  static constexpr uint32_t kColP = 2 * kKeys;              // P: kKeys bf16 per row
  static constexpr uint32_t kColO = kColP + kKeys / 2;      // two O buffers of D columns
  static_assert(kColO + 2 * D <= kTmemCols, "tensor memory");
  static_assert(kMaxClw >= ((kMaxCoarse + kKeys - 1) / kKeys) * kKeys, "coarse weights");
};

struct GroupDesc {
  int bh, b0, nu, nc;
  int ulist[kMaxU];                  // sorted union of the 8 blocks' selections
  uint32_t umask[kMaxU];             // bit b: query block b selected union entry u
  float clw[kMaxClw];                // log2 weights of the coarse keys, -inf for pads
};

struct FwdShared {
  uint64_t desc_full[2], desc_empty[2], coarse_empty;
  uint64_t ring_full[3], ring_empty[3];
  uint64_t s_full[2], p_full, pv, o_full[2], ml_full[2], o_empty[2], done;
  uint32_t tmem_base;
  float red[2][2][128];    // row maxima of the two column halves, by chunk parity
  // softmax -> epilogue, by O buffer: row maxima, the two halves' row sums,
  // and the group's chunk count
  float ml_m[2][128];
  float ml_l[2][2][128];
  int ml_nch[2];
  GroupDesc g[2];
  int ent[kQB * kMaxK];    // fine prep scratch: the selections, 0x7fffffff when unused
  int clist[kMaxCoarse];   // coarse prep scratch: coarse keys, level << 24 | token
};

// Shared-memory offsets (bytes from a 1024-aligned base); nctm = coarse key
// tiles of the largest coarse list.
template <int D>
struct Layout {
  uint32_t q, k, v, ck, cv, end;
  __host__ __device__ explicit Layout(int nctm) {
    using C = Cfg<D>;
    q = 0;                                   // two Q buffers
    k = q + 2 * C::kQBytes;
    v = k + C::kStages * C::kChunk;
    ck = v + C::kStages * C::kChunk;         // coarse K: [half][tile]
    cv = ck + nctm * C::H * kSub;            // coarse V: [half][tile]
    end = cv + nctm * C::H * kSub;
  }
};

// Byte offset of 16-byte chunk jj (0..7) of row r in a 128-byte-swizzled
// region of 128-byte rows (the TMA layout of every tile here).
__device__ __forceinline__ uint32_t sw128(int r, int jj) {
  return (uint32_t)(r * 128 + ((jj ^ (r & 7)) << 4));
}

template <int D, int E>
__global__ void __launch_bounds__(kThreads, 1)
attn_fwd_tc_kernel(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
                   const __grid_constant__ CUtensorMap tv, AttnParams p, int nctm) {
  using C = Cfg<D>;
  constexpr int kCT = C::kCT;
  extern __shared__ unsigned char smem_raw[];
  unsigned char* sm = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  const Layout<D> lay(nctm);
  FwdShared& S = *reinterpret_cast<FwdShared*>(sm + lay.end);
  const uint32_t base = smem_u32(sm);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int n1 = p.N >> 4;
  const int ngx = (n1 + kQB - 1) / kQB;        // groups per (b, h)
  const int ngroups = p.B * p.H * ngx;
  const int K = p.K;
  int flags = 0;
  bool ok = true;

  if (warp == kWarpMma) {
    tmem_alloc(smem_u32(&S.tmem_base), C::kTmemCols);
    tmem_relinquish();
  } else if (tid == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(smem_u32(&S.desc_full[i]), 2);                       // fine and coarse prep
      mbar_init(smem_u32(&S.desc_empty[i]), 1 + kSoftmaxWarps);      // MMA commit + softmax warps
      mbar_init(smem_u32(&S.s_full[i]), 1);
      mbar_init(smem_u32(&S.o_full[i]), 1);
      mbar_init(smem_u32(&S.ml_full[i]), kSoftmaxWarps);
      mbar_init(smem_u32(&S.o_empty[i]), kEpiWarps);
    }
    for (int i = 0; i < 3; ++i) {
      mbar_init(smem_u32(&S.ring_full[i]), 1);
      mbar_init(smem_u32(&S.ring_empty[i]), 1);
    }
    mbar_init(smem_u32(&S.coarse_empty), 1);
    mbar_init(smem_u32(&S.p_full), 32 * kSoftmaxWarps);
    mbar_init(smem_u32(&S.pv), 1);
    mbar_init(smem_u32(&S.done), 1);
    fence_mbar_init();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = S.tmem_base;
  auto qbuf = [&](int b) { return base + lay.q + (uint32_t)b * C::kQBytes; };
  auto kslot = [&](int s) { return base + lay.k + (uint32_t)s * C::kChunk; };
  auto vslot = [&](int s) { return base + lay.v + (uint32_t)s * C::kChunk; };
  auto counts = [&](const GroupDesc& gd, int& nct, int& ncc, int& nfc) {
    nct = (gd.nc + 15) >> 4;
    ncc = (nct + kCT - 1) / kCT;
    nfc = (gd.nu + kCT - 1) / kCT;
  };

  // roles by warpgroup; each warpgroup sets its register share first, so the
  // code of each role is compiled against that share
  if (warp >= kWarpFine) {
  asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegCtl));
  if (warp == kWarpFine) {
    // ------------------------------------------------------------ fine prep
    for (int gi = 0; ok; ++gi) {
      const int G = blockIdx.x + gi * gridDim.x;
      if (G >= ngroups) break;
      const int b = gi & 1;
      GroupDesc& gd = S.g[b];
      const int bh = G / ngx, b0 = (G % ngx) * kQB;
      // the 8 blocks' fine selections under the library's entry rule: rows of
      // K entries side by side across the warp, every load issued first (the
      // group buffer is not touched before it is free)
      const int rpi = 32 / K;                  // rows per pass
      const int npass = (kQB + rpi - 1) / rpi;
      int v[kQB];
#pragma unroll
      for (int i = 0; i < kQB; ++i) {
        const int bi = i * rpi + lane / K, slot = lane % K;
        const bool on = i < npass && lane < rpi * K && bi < kQB && b0 + bi < n1;
        v[i] = on ? p.idx[1][((size_t)bh * n1 + b0 + bi) * K + slot] : -1;
      }
      if (gi >= 2) ok = __all_sync(0xffffffffu, mbar_wait_bounded(smem_u32(&S.desc_empty[b]), (uint32_t)(((gi >> 1) - 1) & 1)));
      if (!ok) break;
      for (int e = lane; e < kMaxU; e += 32) gd.umask[e] = 0u;
#pragma unroll
      for (int i = 0; i < kQB; ++i) {
        if (i < npass) {
          const int bi = i * rpi + lane / K, slot = lane % K;
          const bool on = lane < rpi * K && bi < kQB && b0 + bi < n1;
          const bool used = warp_row_used(v[i], slot, n1, on, flags, K);
          if (lane < rpi * K && bi < kQB) S.ent[bi * K + slot] = used ? v[i] : 0x7fffffff;
        }
      }
      __syncwarp();
      const int nu = warp_sorted_union<E>(S.ent, kQB * K, gd.ulist, lane);
      __syncwarp();
      for (int e = lane; e < kQB * K; e += 32) {
        const int x = S.ent[e];
        if (x != 0x7fffffff) atomicOr(&gd.umask[sorted_find(gd.ulist, nu, x)], 1u << (e / K));
      }
      if (lane == 0) {
        gd.bh = bh;
        gd.b0 = b0;
        gd.nu = nu;
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&S.desc_full[b]));
    }
  } else if (warp == kWarpCoarse) {
    // ---------------------------------------------------------- coarse prep
    int last_group[2] = {-1, -1};
    for (int gi = 0; ok; ++gi) {
      const int G = blockIdx.x + gi * gridDim.x;
      if (G >= ngroups) break;
      const int b = gi & 1;
      GroupDesc& gd = S.g[b];
      const int bh = G / ngx, b0 = (G % ngx) * kQB;
      // coarse keys of levels 2..L, shared by the 8 blocks (loads first)
      int cv[kMaxL + 1];
#pragma unroll
      for (int l = 2; l <= kMaxL; ++l) {
        cv[l] = -1;
        if (l <= p.L && lane < p.Kl[l]) {
          const int nl = p.N >> (4 * l);
          cv[l] = p.idx[l][((size_t)bh * nl + (b0 >> (4 * (l - 1)))) * p.Kl[l] + lane];
        }
      }
      int nc = 0;
#pragma unroll
      for (int l = 2; l <= kMaxL; ++l) {
        if (l <= p.L) {
          const int nl = p.N >> (4 * l);
          const bool u = warp_row_used(cv[l], lane, nl, lane < p.Kl[l], flags);
          const unsigned m = __ballot_sync(0xffffffffu, u);
          if (u) S.clist[nc + __popc(m & ((1u << lane) - 1u))] = (l << 24) | cv[l];
          nc += __popc(m);
        }
      }
      __syncwarp();
      const int nct = (nc + 15) >> 4;
      if (gi >= 2) ok = __all_sync(0xffffffffu, mbar_wait_bounded(smem_u32(&S.desc_empty[b]), (uint32_t)(((gi >> 1) - 1) & 1)));
      if (!ok) break;
      for (int e = lane; e < ((nct + kCT - 1) / kCT) * C::kKeys; e += 32)
        gd.clw[e] = (e < nc) ? p.logw[S.clist[e] >> 24] * kLog2e : -INFINITY;
      // the coarse tiles (one buffer): free once the previous group's coarse PVs ran
      if (gi >= 1) ok = __all_sync(0xffffffffu, mbar_wait_bounded(smem_u32(&S.coarse_empty), (uint32_t)((gi - 1) & 1)));
      if (!ok) break;
      for (int e = lane; e < nct * 16 * (D / 8); e += 32) {
        const int key = e / (D / 8), j = e % (D / 8);
        const int tile = key >> 4, row = key & 15, h = j >> 3;
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
        const uint32_t off = (uint32_t)(h * nctm + tile) * kSub + sw128(row, j & 7);
        *reinterpret_cast<uint4*>(sm + lay.ck + off) = kq;
        *reinterpret_cast<uint4*>(sm + lay.cv + off) = vq;
      }
      fence_proxy_async_smem();  // generic writes -> MMA operand reads
      if (lane == 0) gd.nc = nc;
      __syncwarp();
      if (lane == 0) {
        int nq = 0;
        for (int bi = 0; bi < kQB; ++bi) nq += (b0 + bi < n1) ? 1 : 0;
        const uint32_t bar = smem_u32(&S.desc_full[b]);
        mbar_arrive_expect_tx(bar, (uint32_t)nq * C::H * kSub);
        const size_t rowbase = (size_t)bh * p.N;
        for (int bi = 0; bi < nq; ++bi)
#pragma unroll
          for (int h = 0; h < C::H; ++h)
            tma_load_2d(qbuf(b) + (uint32_t)(h * kQB + bi) * kSub, &tq, 64 * h,
                        (int)(rowbase + (size_t)(b0 + bi) * 16), bar);
      }
      last_group[b] = gi;
    }
    // no Q copy may still be landing when the CTA exits
    if (lane == 0)
      for (int b = 0; b < 2; ++b)
        if (last_group[b] >= 0 && !mbar_wait_bounded(smem_u32(&S.desc_full[b]), (uint32_t)((last_group[b] >> 1) & 1)))
          ok = false;
  } else if (warp == kWarpLoad) {
    // ---------------------------------------------------------- K/V loader
    if (lane == 0) {
      int fg = 0;  // fine chunks issued so far (all groups)
      for (int gi = 0; ok; ++gi) {
        const int G = blockIdx.x + gi * gridDim.x;
        if (G >= ngroups) break;
        const int b = gi & 1;
        const GroupDesc& gd = S.g[b];
        ok = mbar_wait_bounded(smem_u32(&S.desc_full[b]), (uint32_t)((gi >> 1) & 1));
        if (!ok) break;
        const int nu = gd.nu;
        const size_t rowbase = (size_t)gd.bh * p.N;
        for (int t0 = 0; t0 < nu && ok; t0 += kCT, ++fg) {
          const int slot = fg % C::kStages;
          if (fg >= C::kStages)
            ok = mbar_wait_bounded(smem_u32(&S.ring_empty[slot]), (uint32_t)((fg / C::kStages - 1) & 1));
          if (!ok) break;
          const int nt = min(kCT, nu - t0);
          const uint32_t bar = smem_u32(&S.ring_full[slot]);
          mbar_arrive_expect_tx(bar, (uint32_t)nt * 2u * C::H * kSub);
          for (int t = 0; t < nt; ++t) {
            const int y = (int)(rowbase + (size_t)gd.ulist[t0 + t] * 16);
#pragma unroll
            for (int h = 0; h < C::H; ++h) {
              tma_load_2d(kslot(slot) + (uint32_t)(h * kCT + t) * kSub, &tk, 64 * h, y, bar);
              tma_load_2d(vslot(slot) + (uint32_t)(h * kCT + t) * kSub, &tv, 64 * h, y, bar);
            }
          }
        }
      }
      // no copy may still be landing when the CTA exits
      for (int s = 0; s < C::kStages && s < fg; ++s) {
        const int last = s + ((fg - 1 - s) / C::kStages) * C::kStages;
        if (!mbar_wait_bounded(smem_u32(&S.ring_full[s]), (uint32_t)((last / C::kStages) & 1))) ok = false;
      }
    }
  } else if (warp == kWarpMma) {
    // --------------------------------------------------------- MMA issuer
    if (lane == 0) {
      int cg = 0, fg = 0;  // chunks and fine chunks of the groups before this one
      const uint32_t idesc_pv = idesc_bf16_f32(128, D, 1, 0);
      for (int gi = 0; ok; ++gi) {
        const int G = blockIdx.x + gi * gridDim.x;
        if (G >= ngroups) break;
        const int b = gi & 1, ob = gi & 1;
        const GroupDesc& gd = S.g[b];
        ok = mbar_wait_bounded(smem_u32(&S.desc_full[b]), (uint32_t)((gi >> 1) & 1));
        if (ok && gi >= 2) ok = mbar_wait_bounded(smem_u32(&S.o_empty[ob]), (uint32_t)(((gi >> 1) - 1) & 1));
        if (!ok) break;
        tc_fence_after();
        int nct, ncc, nfc;
        counts(gd, nct, ncc, nfc);
        const int nu = gd.nu;
        const int nch = ncc + nfc;
        if (ncc == 0) tc_commit(smem_u32(&S.coarse_empty));  // one phase per group
        if (nch == 0) tc_commit(smem_u32(&S.desc_empty[b]));
        auto tiles = [&](int cl) { return cl < ncc ? min(kCT, nct - cl * kCT) : min(kCT, nu - (cl - ncc) * kCT); };
        for (int cl = 0; cl <= nch && ok; ++cl) {
          if (cl < nch) {
            const int c = cg + cl, nt = tiles(cl);
            uint32_t kaddr, hstride;
            if (cl < ncc) {
              kaddr = base + lay.ck + (uint32_t)(cl * kCT) * kSub;
              hstride = (uint32_t)nctm * kSub;
            } else {
              const int f = fg + cl - ncc;
              ok = mbar_wait_bounded(smem_u32(&S.ring_full[f % C::kStages]), (uint32_t)((f / C::kStages) & 1));
              if (!ok) break;
              kaddr = kslot(f % C::kStages);
              hstride = kCT * kSub;
            }
            tc_fence_after();
            const uint32_t idesc_s = idesc_bf16_f32(128, 16 * nt, 0, 0);
#pragma unroll
            for (int ks = 0; ks < D / 16; ++ks) {
              const int h = ks >> 2, kk = ks & 3;
              tc_mma_f16(tbase + C::kColS + (uint32_t)(c & 1) * C::kKeys,
                         smem_desc_sw128(qbuf(b) + (uint32_t)(h * kQB) * kSub + kk * 32, 16, 1024),
                         smem_desc_sw128(kaddr + h * hstride + kk * 32, 16, 1024), idesc_s, ks > 0);
            }
            tc_commit(smem_u32(&S.s_full[c & 1]));
            if (cl == nch - 1) tc_commit(smem_u32(&S.desc_empty[b]));  // Q of this group is no longer read
          }
          if (cl >= 1) {
            const int cp = cl - 1, c = cg + cp, nt = tiles(cp);
            uint32_t vaddr, hstride;
            if (cp < ncc) {
              vaddr = base + lay.cv + (uint32_t)(cp * kCT) * kSub;
              hstride = (uint32_t)nctm * kSub;
            } else {
              vaddr = vslot((fg + cp - ncc) % C::kStages);
              hstride = kCT * kSub;
            }
            ok = mbar_wait_bounded(smem_u32(&S.p_full), (uint32_t)(c & 1));
            if (!ok) break;
            tc_fence_after();
            for (int t = 0; t < nt; ++t)
              tc_mma_f16_ts(tbase + C::kColO + (uint32_t)ob * D, tbase + C::kColP + (uint32_t)t * 8,
                            smem_desc_sw128(vaddr + (uint32_t)t * kSub, hstride, 1024), idesc_pv,
                            (cp > 0 || t > 0) ? 1u : 0u);
            tc_commit(smem_u32(&S.pv));
            if (cp == ncc - 1) tc_commit(smem_u32(&S.coarse_empty));
            if (cp >= ncc) tc_commit(smem_u32(&S.ring_empty[(fg + cp - ncc) % C::kStages]));
          }
        }
        tc_commit(smem_u32(&S.o_full[ob]));  // O of this group is final (one phase per group)
        cg += nch;
        fg += nfc;
      }
      // every MMA of this CTA has completed before tensor memory is freed
      tc_commit(smem_u32(&S.done));
      if (!mbar_wait_bounded(smem_u32(&S.done), 0)) ok = false;
    }
  }
  } else if (warp < kSoftmaxWarps) {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kRegSoftmax));
    // --------------------------------------------------------------- softmax
    constexpr int kHT = kCT / 2;                  // key tiles of each column half
    const int q4 = warp & 3;                      // TMEM lane quarter of this warp
    const int hs = warp >> 2;                     // column half of this thread
    const int r = q4 * 32 + lane;                 // query row = TMEM lane
    const int qb = r >> 4;                        // its query block in the group
    const uint32_t lane_off = (uint32_t)(q4 * 32) << 16;
    const float sc2 = p.scale * kLog2e;
    const uint64_t sc2x2 = f2_make(sc2, sc2);
    // the two warps of one lane quarter meet on named barrier 1 + q4
    auto pair_bar = [&]() { asm volatile("bar.sync %0, 64;" ::"r"(1 + q4) : "memory"); };
    int cg = 0;
    for (int gi = 0; ok; ++gi) {
      const int G = blockIdx.x + gi * gridDim.x;
      if (G >= ngroups) break;
      const int b = gi & 1, ob = gi & 1;
      const GroupDesc& gd = S.g[b];
      ok = __all_sync(0xffffffffu, mbar_wait_bounded(smem_u32(&S.desc_full[b]), (uint32_t)((gi >> 1) & 1)));
      if (!ok) break;
      int nct, ncc, nfc;
      counts(gd, nct, ncc, nfc);
      const int nch = ncc + nfc, nu = gd.nu;
      float m_ref = -INFINITY, lsum = 0.f;
      for (int cl = 0; cl < nch && ok; ++cl) {
        const int c = cg + cl;
        const bool coarse = cl < ncc;
        const int nt = coarse ? min(kCT, nct - cl * kCT) : min(kCT, nu - (cl - ncc) * kCT);
        const int u0 = (cl - ncc) * kCT;
        ok = __all_sync(0xffffffffu, mbar_wait_bounded(smem_u32(&S.s_full[c & 1]), (uint32_t)((c >> 1) & 1)));
        if (!ok) break;
        tc_fence_after();
        // this thread's tiles: t = hs * kHT + i
        bool live[kHT];  // some row of this warp takes the key tile
        uint64_t lwt[kHT];
        const uint32_t srow = tbase + lane_off + C::kColS + (uint32_t)(c & 1) * C::kKeys + 16 * hs * kHT;
        float x[16 * kHT];
#pragma unroll
        for (int i2 = 0; i2 < kHT; ++i2) {
          const int t = hs * kHT + i2;
          const uint32_t bits = (!coarse && t < nt) ? gd.umask[u0 + t] : 0u;
          live[i2] = t < nt && (coarse || ((bits >> (2 * q4)) & 3u) != 0u);
          const float lwf = ((bits >> qb) & 1u) ? 0.f : -INFINITY;
          lwt[i2] = f2_make(lwf, lwf);
          if (live[i2]) tmem_ld16(srow + 16 * i2, &x[16 * i2]);
        }
        tmem_wait_ld();
        // x = s * scale * log2(e) + log2(w), in pairs; -inf where the row's
        // block did not select the key block (or past the coarse keys); the
        // maximum as a tree, not one dependent chain
        const float* clw = gd.clw + cl * C::kKeys + 16 * hs * kHT;
        float tmax[kHT];
#pragma unroll
        for (int i2 = 0; i2 < kHT; ++i2) {
          tmax[i2] = -INFINITY;
          if (live[i2]) {
            float m2[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
            for (int j = 0; j < 16; j += 2) {
              const uint64_t lw = coarse ? f2_make(clw[16 * i2 + j], clw[16 * i2 + j + 1]) : lwt[i2];
              const float2 v2 = f2_split(f2_fma(f2_make(x[16 * i2 + j], x[16 * i2 + j + 1]), sc2x2, lw));
              x[16 * i2 + j] = v2.x;
              x[16 * i2 + j + 1] = v2.y;
              m2[(j >> 1) & 3] = fmaxf(m2[(j >> 1) & 3], fmaxf(v2.x, v2.y));
            }
            tmax[i2] = fmaxf(fmaxf(m2[0], m2[1]), fmaxf(m2[2], m2[3]));
          }
        }
#pragma unroll
        for (int w = 1; w < kHT; w <<= 1)
#pragma unroll
          for (int t = 0; t + w < kHT; t += 2 * w) tmax[t] = fmaxf(tmax[t], tmax[t + w]);
        // the row maximum over both halves
        S.red[c & 1][hs][r] = tmax[0];
        pair_bar();
        const float mx = fmaxf(S.red[c & 1][0][r], S.red[c & 1][1][r]);
        // the exact running maximum; probabilities against it before waiting
        // for the tensor core (only the stores below need PV of chunk c - 1)
        const bool need = (m_ref != -INFINITY) && (mx > m_ref);
        const float corr = need ? ex2_approx(m_ref - mx) : 1.f;
        m_ref = fmaxf(m_ref, mx);  // a row still at -inf has O exactly zero: nothing to rescale
        const float mb = (m_ref == -INFINITY) ? 0.f : m_ref;
        const uint64_t mb2 = f2_make(mb, mb);
        // PV of the previous chunk has read P, and O is final up to it
        if (c > 0) {
          ok = __all_sync(0xffffffffu, mbar_wait_bounded(smem_u32(&S.pv), (uint32_t)((c - 1) & 1)));
          if (!ok) break;
        }
        tc_fence_after();
        if (__any_sync(0xffffffffu, need)) {  // the maximum rose: rescale this half of the O row
          const uint64_t cc = f2_make(corr, corr);
#pragma unroll
          for (int cb = 0; cb < D / 2; cb += 16) {
            const uint32_t ta = tbase + lane_off + C::kColO + (uint32_t)ob * D + hs * (D / 2) + cb;
            float o[16];
            tmem_ld16(ta, o);
            tmem_wait_ld();
#pragma unroll
            for (int j = 0; j < 16; j += 2) {
              const float2 vv = f2_split(f2_mul(f2_make(o[j], o[j + 1]), cc));
              o[j] = vv.x;
              o[j + 1] = vv.y;
            }
            tmem_st16(ta, o);
          }
        }
        uint64_t acc[2] = {f2_make(0.f, 0.f), f2_make(0.f, 0.f)};
#pragma unroll
        for (int i2 = 0; i2 < kHT; i2 += 2) {
          uint32_t pk[16];
#pragma unroll
          for (int i3 = 0; i3 < 2; ++i3) {
            if (live[i2 + i3]) {
#pragma unroll
              for (int j = 0; j < 8; ++j) {
                const float2 d2 = f2_split(f2_sub(f2_make(x[16 * (i2 + i3) + 2 * j], x[16 * (i2 + i3) + 2 * j + 1]), mb2));
                const float p0 = ex2_approx(d2.x), p1 = ex2_approx(d2.y);
                pk[8 * i3 + j] = pack_bf16(p0, p1);
                acc[j & 1] = f2_add(acc[j & 1], f2_make(p0, p1));
              }
            } else {
#pragma unroll
              for (int j = 0; j < 8; ++j) pk[8 * i3 + j] = 0u;
            }
          }
          tmem_st16u(tbase + lane_off + C::kColP + (uint32_t)((hs * kHT + i2) * 8), pk);
        }
        const float2 a2 = f2_split(f2_add(acc[0], acc[1]));
        lsum = lsum * corr + (a2.x + a2.y);
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(smem_u32(&S.p_full));
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&S.desc_empty[b]));  // masks and weights no longer read
      if (!ok) break;
      // hand the row's maximum and sums to the epilogue (its buffer was read)
      if (gi >= 2) ok = __all_sync(0xffffffffu, mbar_wait_bounded(smem_u32(&S.o_empty[ob]), (uint32_t)(((gi >> 1) - 1) & 1)));
      if (!ok) break;
      if (hs == 0) S.ml_m[ob][r] = m_ref;
      S.ml_l[ob][hs][r] = lsum;
      if (warp == 0 && lane == 0) S.ml_nch[ob] = nch;
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&S.ml_full[ob]));
      cg += nch;
    }
  } else {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegEpi));
    // -------------------------------------------------------------- epilogue
    // one thread per query row: O = acc / l, LSE = (m + log2 l) ln 2 and the
    // residual of O, the row written as whole 16-byte chunks
    const int q4 = warp & 3;
    const int r = q4 * 32 + lane;
    const int qb = r >> 4;
    const uint32_t lane_off = (uint32_t)(q4 * 32) << 16;
    bf16* Og = static_cast<bf16*>(p.out);
    bf16* Rg = static_cast<bf16*>(p.o_res);
    for (int gi = 0; ok; ++gi) {
      const int G = blockIdx.x + gi * gridDim.x;
      if (G >= ngroups) break;
      const int ob = gi & 1;
      const int bh = G / ngx, b0 = (G % ngx) * kQB;
      ok = __all_sync(0xffffffffu, mbar_wait_bounded(smem_u32(&S.ml_full[ob]), (uint32_t)((gi >> 1) & 1)));
      if (ok) ok = __all_sync(0xffffffffu, mbar_wait_bounded(smem_u32(&S.o_full[ob]), (uint32_t)((gi >> 1) & 1)));
      if (!ok) break;
      tc_fence_after();
      const int nch = S.ml_nch[ob];
      const float m = S.ml_m[ob][r];
      const float ltot = S.ml_l[ob][0][r] + S.ml_l[ob][1][r];
      const bool has = nch > 0 && ltot > 0.f;
      const float inv = has ? 1.f / ltot : 0.f;
      const size_t tok = (size_t)bh * p.N + (size_t)b0 * 16 + r;
      const bool valid = b0 + qb < n1;
#pragma unroll 1
      for (int cb = 0; cb < D; cb += 32) {
        float o[32];
        if (nch > 0) {
          tmem_ld16(tbase + lane_off + C::kColO + (uint32_t)ob * D + cb, o);
          tmem_ld16(tbase + lane_off + C::kColO + (uint32_t)ob * D + cb + 16, o + 16);
          tmem_wait_ld();
        }
        if (valid) {
          uint4* orow = reinterpret_cast<uint4*>(Og + tok * D + cb);
          uint4* rrow = Rg != nullptr ? reinterpret_cast<uint4*>(Rg + tok * D + cb) : nullptr;
#pragma unroll
          for (int jj = 0; jj < 4; ++jj) {
            float a[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) a[e] = has ? o[8 * jj + e] * inv : 0.f;
            const uint4 w = make_uint4(pack_bf16(a[0], a[1]), pack_bf16(a[2], a[3]), pack_bf16(a[4], a[5]),
                                       pack_bf16(a[6], a[7]));
            orow[jj] = w;
            if (rrow != nullptr)  // what the bf16 rounding of O left out, itself in bf16
              rrow[jj] = make_uint4(pack_bf16(a[0] - bf16x2_lo(w.x), a[1] - bf16x2_hi(w.x)),
                                    pack_bf16(a[2] - bf16x2_lo(w.y), a[3] - bf16x2_hi(w.y)),
                                    pack_bf16(a[4] - bf16x2_lo(w.z), a[5] - bf16x2_hi(w.z)),
                                    pack_bf16(a[6] - bf16x2_lo(w.w), a[7] - bf16x2_hi(w.w)));
          }
        }
      }
      if (valid) p.lse[tok] = has ? (m + log2f(ltot)) * kLn2 : -INFINITY;
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&S.o_empty[ob]));
    }
  }

  if (!ok) flags |= LLSA_DEV_TIMEOUT;
  flags = __reduce_or_sync(0xffffffffu, flags);
  if (lane == 0) report_status(p.status, flags);
  tc_fence_before();
  __syncthreads();
  if (warp == kWarpMma) {
    tc_fence_after();
    tmem_dealloc(tbase, C::kTmemCols);
  }
}

template <int D>
size_t smem_bytes(int nctm) {
  return 1024 + Layout<D>(nctm).end + sizeof(FwdShared);
}

constexpr size_t kOneCtaSmem = 120 * 1024;

int num_sms() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return 148;
  return n > 0 ? n : 148;
}

template <int D>
cudaError_t launch_typed(const AttnParams& p, const CUtensorMap* maps, cudaStream_t s) {
  const int nctm = (p.Kc + 15) / 16;
  // at least half of an SM's shared memory, so no second CTA (which would
  // wait for the first one's tensor memory) shares an SM with a persistent one
  const size_t smem = smem_bytes<D>(nctm) > kOneCtaSmem ? smem_bytes<D>(nctm) : kOneCtaSmem;
  const int ent = kQB * p.K;
  auto kern = (ent <= 32)    ? attn_fwd_tc_kernel<D, 1>
              : (ent <= 64)  ? attn_fwd_tc_kernel<D, 2>
              : (ent <= 128) ? attn_fwd_tc_kernel<D, 4>
                             : attn_fwd_tc_kernel<D, 8>;
  // the register split inside the kernel assumes kRegLaunch registers per
  // thread at launch; with fewer, setmaxnreg.inc would wait forever
  cudaFuncAttributes fa;
  cudaError_t e = cudaFuncGetAttributes(&fa, kern);
  if (e != cudaSuccess) return e;
  if (fa.numRegs != kRegLaunch) return cudaErrorInvalidConfiguration;
  e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout, (int)cudaSharedmemCarveoutMaxShared);
  if (e != cudaSuccess) return e;
  const int n1 = p.N / kBlock;
  const long long groups = (long long)p.B * p.H * ((n1 + kQB - 1) / kQB);
  const int grid = (int)(groups < num_sms() ? groups : num_sms());
  kern<<<grid, kThreads, smem, s>>>(maps[0], maps[1], maps[2], p, nctm);
  return cudaGetLastError();
}

}  // namespace

// Shared memory the tcgen05 forward needs for this problem (host check: the
// caller uses the warp-MMA forward when it exceeds the per-CTA limit).
size_t attn_fwd_tc_smem(const AttnParams& p) {
  const int nctm = (p.Kc + 15) / 16;
  return p.D == 64 ? smem_bytes<64>(nctm) : smem_bytes<128>(nctm);
}

// maps: Q, K, V as 2D [B*H*N rows, D cols] bf16, box 16 x 64, 128-byte swizzle.
cudaError_t launch_attn_fwd_tc(const AttnParams& p, const CUtensorMap* maps, cudaStream_t s) {
  return (p.D == 64) ? launch_typed<64>(p, maps, s) : launch_typed<128>(p, maps, s);
}

}  // namespace llsa
