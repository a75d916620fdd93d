// Host side of the C ABI declared in include/llsa.h: argument checks, the
// backward workspace layout and kernel dispatch.  No allocation, no state.

#include <cuda.h>
#include <math.h>
#include <string.h>

#include <mutex>

#include "llsa_internal.cuh"

namespace llsa {
cudaError_t launch_attn_fwd_simt(const AttnParams& p, int dtype, cudaStream_t s);
cudaError_t launch_attn_bwd_simt(const AttnParams& p, int dtype, cudaStream_t s);
cudaError_t launch_attn_fwd_mma(const AttnParams& p, const CUtensorMap* maps, cudaStream_t s);
cudaError_t launch_attn_fwd_mma_select(const AttnParams& p, const SelectParams& sp, const CUtensorMap* maps,
                                       cudaStream_t s);
cudaError_t launch_attn_fwd_tc(const AttnParams& p, const CUtensorMap* maps, cudaStream_t s);
size_t attn_fwd_tc_smem(const AttnParams& p);
cudaError_t launch_attn_bwd_mma(const AttnParams& p, const CUtensorMap* maps, cudaStream_t s, bool tc_kv);
cudaError_t launch_qkv_pool(const CUtensorMap* maps, void* const out[3], float* const lvl[3][3], int32_t* status,
                            int B, int N, int H, int D, int L, int C, cudaStream_t s);
}  // namespace llsa

using namespace llsa;

namespace {

// K_l, the width of I(l): topk_l[l], or topk where that is 0.
inline int k_level(const llsa_desc* d, int l) { return d->topk_l[l] > 0 ? d->topk_l[l] : d->topk; }

inline int check_desc(const llsa_desc* d) {
  if (d == nullptr) return LLSA_ERR_INVALID_ARG;
  if (d->B < 1 || d->H < 1 || d->N < kBlock || d->D < 1 || d->L < 1 || d->topk < 1)
    return LLSA_ERR_INVALID_ARG;
  if ((d->flags & ~(LLSA_FLAG_FWD_TCGEN05 | LLSA_FLAG_BWD_TCGEN05 | LLSA_FLAG_FWD_MMA_SYNC)) != 0)
    return LLSA_ERR_INVALID_ARG;
  if ((d->flags & LLSA_FLAG_FWD_TCGEN05) && (d->flags & LLSA_FLAG_FWD_MMA_SYNC)) return LLSA_ERR_INVALID_ARG;
  if (d->dtype != LLSA_F32 && d->dtype != LLSA_BF16) return LLSA_ERR_INVALID_ARG;
  if (d->D != 64 && d->D != 128) return LLSA_ERR_UNSUPPORTED;
  if (d->L > kMaxL || d->topk > kMaxK) return LLSA_ERR_UNSUPPORTED;
  for (int l = 1; l <= d->L; ++l) {
    if (d->topk_l[l] < 0) return LLSA_ERR_INVALID_ARG;
    if (d->topk_l[l] > kMaxK) return LLSA_ERR_UNSUPPORTED;
  }
  const long long span = 1LL << (4 * d->L);
  if (d->N % span != 0) return LLSA_ERR_INVALID_ARG;
  if ((long long)d->B * d->H > 65535) return LLSA_ERR_UNSUPPORTED;  // grid.y
  for (int l = 1; l <= d->L; ++l)  // CSR offsets are int32
    if ((long long)(d->N >> (4 * l)) * k_level(d, l) > 0x7fffffffLL) return LLSA_ERR_UNSUPPORTED;
  if (!(d->sm_scale >= 0.f) || isinf(d->sm_scale)) return LLSA_ERR_INVALID_ARG;
  for (int l = 2; l <= d->L; ++l)
    if (!(d->level_w[l] >= 0.f) || isinf(d->level_w[l])) return LLSA_ERR_INVALID_ARG;
  return LLSA_OK;
}

inline int n_level(const llsa_desc* d, int l) { return d->N >> (4 * l); }


// Lc, the top level whose tokens are keys: coarse levels 2..Lc join the fine
// keys (enrichment depth enrich_levels; 0 = all L levels, < 0 = none).
inline int key_top(const llsa_desc* d) {
  if (d->enrich_levels == 0) return d->L;
  if (d->enrich_levels < 0) return 1;
  return d->enrich_levels >= d->L - 1 ? d->L : 1 + d->enrich_levels;
}

inline float scale_of(const llsa_desc* d) {
  return d->sm_scale > 0.f ? d->sm_scale : 1.0f / sqrtf((float)d->D);
}

struct WsLayout {
  size_t delta = 0;
  size_t part[kMaxL + 1] = {};
  size_t coarse[kMaxL + 1] = {};
  size_t work = 0;
  size_t total = 0;
};

inline WsLayout ws_layout(const llsa_desc* d) {
  WsLayout w;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off += (bytes + 255) & ~(size_t)255;
    return o;
  };
  const size_t BH = (size_t)d->B * d->H;
  w.delta = take(BH * d->N * sizeof(float));
  const int Lc = key_top(d);
  for (int l = 2; l <= Lc; ++l)
    w.part[l] = take(BH * (size_t)(d->N >> 7) * k_level(d, l) * 2 * d->D * sizeof(float));
  for (int l = 2; l <= Lc; ++l)
    w.coarse[l] = take(BH * (size_t)n_level(d, l) * 2 * d->D * sizeof(float));
  w.work = take(sizeof(int32_t));
  w.total = off;
  return w;
}

// Transpose workspace: per level, BH * nchunk * N_l int32 counts.
struct TrWsLayout {
  size_t off[kMaxL + 1];
  size_t total;
};

inline TrWsLayout tr_ws_layout(const llsa_desc* d) {
  TrWsLayout w;
  memset(&w, 0, sizeof(w));
  size_t off = 0;
  const size_t BH = (size_t)d->B * d->H;
  for (int l = 1; l <= key_top(d); ++l) {
    const int n = n_level(d, l);
    int nchunk = 0, rows = 0;
    transpose_chunking(n, &nchunk, &rows);
    w.off[l] = off;
    off += (BH * nchunk * n * sizeof(int32_t) + 255) & ~(size_t)255;
  }
  w.total = off;
  return w;
}

inline int launch_status(cudaError_t e) { return e == cudaSuccess ? LLSA_OK : LLSA_ERR_LAUNCH; }

// cuTensorMapEncodeTiled, fetched from the driver once (no link-time libcuda).
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_tiled() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(f);
  });
  return fn;
}

// A bf16 [rows, D] row-major tensor seen by TMA as tiles of 16 rows x 64
// columns (128 bytes) with 128-byte swizzle.
int make_row_tile_map(CUtensorMap* map, const void* base, uint64_t rows, int D) {
  EncodeTiledFn fn = encode_tiled();
  if (fn == nullptr) return LLSA_ERR_LAUNCH;
  if ((reinterpret_cast<uintptr_t>(base) & 15) != 0) return LLSA_ERR_INVALID_ARG;
  const cuuint64_t dims[2] = {(cuuint64_t)D, (cuuint64_t)rows};
  const cuuint64_t strides[1] = {(cuuint64_t)D * 2};
  const cuuint32_t box[2] = {64, 16};
  const cuuint32_t estride[2] = {1, 1};
  const CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims,
                        strides, box, estride, CU_TENSOR_MAP_INTERLEAVE_NONE,
                        CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? LLSA_OK : LLSA_ERR_LAUNCH;
}

// A bf16 [rows, cols] row-major matrix seen by TMA as boxes of box_rows rows
// x 64 columns (128 bytes) with 128-byte swizzle.
int make_kslice_map(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols, uint32_t box_rows) {
  EncodeTiledFn fn = encode_tiled();
  if (fn == nullptr) return LLSA_ERR_LAUNCH;
  if ((reinterpret_cast<uintptr_t>(base) & 15) != 0) return LLSA_ERR_INVALID_ARG;
  const cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  const cuuint64_t strides[1] = {(cuuint64_t)cols * 2};
  const cuuint32_t box[2] = {64, box_rows};
  const cuuint32_t estride[2] = {1, 1};
  const CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims,
                        strides, box, estride, CU_TENSOR_MAP_INTERLEAVE_NONE,
                        CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? LLSA_OK : LLSA_ERR_LAUNCH;
}

void fill_attn_common(AttnParams& p, const llsa_desc* d, const void* q, const void* k,
                      const void* v, const llsa_pyramid* pyr, const llsa_indices* idx) {
  memset(&p, 0, sizeof(p));
  p.q = q;
  p.k = k;
  p.v = v;
  const int Lc = key_top(d);
  for (int l = 1; l <= Lc; ++l) p.idx[l] = idx->idx[l];
  for (int l = 2; l <= Lc; ++l) {
    p.pk[l] = pyr->k[l];
    p.pv[l] = pyr->v[l];
    const float w = d->level_w[l] > 0.f ? d->level_w[l] : 1.0f;
    p.logw[l] = logf(w);
  }
  p.B = d->B;
  p.H = d->H;
  p.N = d->N;
  p.D = d->D;
  p.L = Lc;  // the kernels see only the levels whose tokens are keys
  p.K = k_level(d, 1);
  p.Kc = 0;
  for (int l = 1; l <= Lc; ++l) {
    p.Kl[l] = k_level(d, l);
    if (l >= 2) p.Kc += p.Kl[l];
  }
  p.scale = scale_of(d);
}

bool coarse_kv_present(const llsa_desc* d, const llsa_pyramid* pyr) {
  for (int l = 2; l <= key_top(d); ++l)
    if (pyr->k[l] == nullptr || pyr->v[l] == nullptr) return false;
  return true;
}

bool indices_present(const llsa_desc* d, const llsa_indices* idx, int top) {
  for (int l = 1; l <= top; ++l)
    if (idx->idx[l] == nullptr) return false;
  return true;
}

// The selection launch of level l.
SelectParams select_params(const llsa_desc* d, const llsa_pyramid* pyr, const llsa_indices* out, int l) {
  SelectParams p;
  p.ql = pyr->q[l];
  p.kl = pyr->k[l];
  p.parent = (l == d->L) ? nullptr : out->idx[l + 1];
  p.out = out->idx[l];
  p.n = n_level(d, l);
  p.K = k_level(d, l);
  p.Kp = (l == d->L) ? 0 : k_level(d, l + 1);
  return p;
}

int check_select_args(const llsa_desc* d, const llsa_pyramid* pyr, const llsa_indices* out) {
  if (pyr == nullptr || out == nullptr || !indices_present(d, out, d->L)) return LLSA_ERR_INVALID_ARG;
  for (int l = 1; l <= d->L; ++l)
    if (pyr->q[l] == nullptr || pyr->k[l] == nullptr) return LLSA_ERR_INVALID_ARG;
  return LLSA_OK;
}

enum class FwdPath { kSimt, kTc, kMma };

struct FwdPlan {
  AttnParams p;
  CUtensorMap maps[3];  // Q, K, V
  FwdPath path;
};

// Shared memory per CTA that kernels may use (B200: 227 KB).
constexpr size_t kMaxSmemPerCta = 227 * 1024;

// Every check of the forward (and its tensor maps), before anything launches.
// o_res: the residual of O to write (bf16 only), or NULL.
int plan_fwd(const llsa_desc* desc, const void* q, const void* k, const void* v, const llsa_pyramid* pyr,
             const llsa_indices* idx, void* o, void* o_res, float* lse, int32_t* dev_status, FwdPlan& f) {
  if (q == nullptr || k == nullptr || v == nullptr || o == nullptr || lse == nullptr ||
      idx == nullptr || pyr == nullptr)
    return LLSA_ERR_INVALID_ARG;
  if (!indices_present(desc, idx, key_top(desc)) || !coarse_kv_present(desc, pyr)) return LLSA_ERR_INVALID_ARG;
  fill_attn_common(f.p, desc, q, k, v, pyr, idx);
  f.p.out = o;
  f.p.lse = lse;
  f.p.status = dev_status;
  if (desc->dtype == LLSA_F32) {
    f.path = FwdPath::kSimt;
    return LLSA_OK;
  }
  // bf16: tensor-core kernels with TMA gathers
  if (((uintptr_t)o & 15) != 0) return LLSA_ERR_INVALID_ARG;
  const uint64_t rows = (uint64_t)desc->B * desc->H * desc->N;
  if (rows > 0x7fffffffULL) return LLSA_ERR_UNSUPPORTED;  // TMA row coordinates are int32
  const void* srcs[3] = {q, k, v};
  for (int i = 0; i < 3; ++i) {
    const int st = make_row_tile_map(&f.maps[i], srcs[i], rows, desc->D);
    if (st != LLSA_OK) return st;
  }
  // Default: the faster of the two bf16 forwards as measured on B200 at the
  // synthetic workloads -- tcgen05 at D = 128 (1.30 vs 2.24 ms at 512x512
  // pixels, K = 8), the warp-MMA kernel at D = 64 (0.31 vs 0.55 ms at 256x256
  // pixels).  The flags force either; tcgen05 also needs its coarse keys to
  // fit in a CTA's shared memory.
  const bool tc_fits = attn_fwd_tc_smem(f.p) <= kMaxSmemPerCta;
  bool tc = desc->D == 128;
  if (desc->flags & LLSA_FLAG_FWD_TCGEN05) tc = true;
  if (desc->flags & LLSA_FLAG_FWD_MMA_SYNC) tc = false;
  f.path = (tc && tc_fits) ? FwdPath::kTc : FwdPath::kMma;
  f.p.o_res = o_res;
  return LLSA_OK;
}

int launch_fwd(const FwdPlan& f, cudaStream_t s) {
  switch (f.path) {
    case FwdPath::kSimt: return launch_status(launch_attn_fwd_simt(f.p, LLSA_F32, s));
    case FwdPath::kTc: return launch_status(launch_attn_fwd_tc(f.p, f.maps, s));
    default: return launch_status(launch_attn_fwd_mma(f.p, f.maps, s));
  }
}

int attn_bwd_impl(const llsa_desc* desc, const void* q, const void* k, const void* v, const llsa_pyramid* pyr,
                  const void* o, const void* o_res, const float* lse, const void* dout,
                  const llsa_indices* idx, const llsa_csr* csr, void* dq, void* dk, void* dv, void* ws,
                  size_t ws_bytes, int32_t* dev_status, void* stream);

}  // namespace

extern "C" {

int llsa_version(void) { return 200; }  // 0.2.0: llsa_desc gained enrich_levels and topk_l

int llsa_reorder(int B, int H, int img_h, int img_w, int D, int dtype, const void* src, void* dst,
                 int to_zorder, void* stream) {
  if (B < 1 || H < 1 || img_h < 1 || img_w < 1 || src == nullptr || dst == nullptr) return LLSA_ERR_INVALID_ARG;
  if (dtype != LLSA_F32 && dtype != LLSA_BF16) return LLSA_ERR_INVALID_ARG;
  if (D != 64 && D != 128) return LLSA_ERR_UNSUPPORTED;
  if (img_h != img_w || img_h < 4 || (img_h & (img_h - 1)) != 0 || img_h > (1 << 15)) return LLSA_ERR_UNSUPPORTED;
  if ((((uintptr_t)src | (uintptr_t)dst) & 15) != 0) return LLSA_ERR_INVALID_ARG;
  const long long N = (long long)img_h * img_w;
  const long long rows = (long long)B * H * N;
  const int row_bytes = D * (dtype == LLSA_BF16 ? 2 : 4);
  const uintptr_t bytes = (uintptr_t)(rows * row_bytes);
  const uintptr_t a = (uintptr_t)src, b = (uintptr_t)dst;
  if (a < b + bytes && b < a + bytes) return LLSA_ERR_INVALID_ARG;  // overlapping buffers
  if (N > 0x7fffffffLL) return LLSA_ERR_UNSUPPORTED;
  int side_log2 = 0;
  while ((1 << side_log2) < img_w) ++side_log2;
  return launch_status(launch_reorder(src, dst, rows, (int)N, side_log2, row_bytes, to_zorder != 0,
                                      (cudaStream_t)stream));
}

const char* llsa_status_string(int status) {
  switch (status) {
    case LLSA_OK: return "ok";
    case LLSA_ERR_INVALID_ARG: return "invalid argument";
    case LLSA_ERR_UNSUPPORTED: return "unsupported configuration";
    case LLSA_ERR_LAUNCH: return "kernel launch failed";
    case LLSA_ERR_WORKSPACE: return "workspace too small";
    default: return "unknown status";
  }
}

int llsa_pool(const llsa_desc* desc, const void* q, const void* k, const void* v,
              const llsa_pyramid* out, void* stream) {
  int st = check_desc(desc);
  if (st != LLSA_OK) return st;
  if (q == nullptr || k == nullptr || v == nullptr || out == nullptr) return LLSA_ERR_INVALID_ARG;
  PoolParams p;
  memset(&p, 0, sizeof(p));
  p.x[0] = q;
  p.x[1] = k;
  p.x[2] = v;
  for (int l = 1; l <= desc->L; ++l) {
    if (out->q[l] == nullptr || out->k[l] == nullptr) return LLSA_ERR_INVALID_ARG;
    if (l >= 2 && out->v[l] == nullptr) return LLSA_ERR_INVALID_ARG;
    p.lvl[0][l] = out->q[l];
    p.lvl[1][l] = out->k[l];
    p.lvl[2][l] = (l >= 2) ? out->v[l] : nullptr;
  }
  p.BH = desc->B * desc->H;
  p.N = desc->N;
  p.D = desc->D;
  p.L = desc->L;
  return launch_status(launch_pool(p, desc->dtype, (cudaStream_t)stream));
}

int llsa_qkv_pool(const llsa_desc* desc, const void* x, const void* w, int C, void* q, void* k, void* v,
                  const llsa_pyramid* out, int32_t* dev_status, void* stream) {
  int st = check_desc(desc);
  if (st != LLSA_OK) return st;
  if (x == nullptr || w == nullptr || q == nullptr || k == nullptr || v == nullptr || out == nullptr)
    return LLSA_ERR_INVALID_ARG;
  if (C < 64 || C % 64 != 0) return LLSA_ERR_INVALID_ARG;
  if (desc->dtype != LLSA_BF16 || (desc->H * desc->D) % 128 != 0 || desc->N % 256 != 0)
    return LLSA_ERR_UNSUPPORTED;
  const void* ptrs[5] = {x, w, q, k, v};
  for (const void* ptr : ptrs)
    if ((reinterpret_cast<uintptr_t>(ptr) & 15) != 0) return LLSA_ERR_INVALID_ARG;
  for (int l = 1; l <= desc->L; ++l) {
    if (out->q[l] == nullptr || out->k[l] == nullptr) return LLSA_ERR_INVALID_ARG;
    if (l >= 2 && out->v[l] == nullptr) return LLSA_ERR_INVALID_ARG;
  }
  const long long tokens = (long long)desc->B * desc->N;
  const int HD = desc->H * desc->D;
  CUtensorMap maps[2];
  st = make_kslice_map(&maps[0], x, (uint64_t)tokens, (uint64_t)C, 256);
  if (st != LLSA_OK) return st;
  st = make_kslice_map(&maps[1], w, (uint64_t)3 * HD, (uint64_t)C, 128);
  if (st != LLSA_OK) return st;
  void* const o[3] = {q, k, v};
  float* const lvl[3][3] = {{nullptr, out->q[1], desc->L >= 2 ? out->q[2] : nullptr},
                            {nullptr, out->k[1], desc->L >= 2 ? out->k[2] : nullptr},
                            {nullptr, nullptr, desc->L >= 2 ? out->v[2] : nullptr}};
  cudaError_t e = launch_qkv_pool(maps, o, lvl, dev_status, desc->B, desc->N, desc->H, desc->D, desc->L, C,
                                  (cudaStream_t)stream);
  if (e != cudaSuccess) return LLSA_ERR_LAUNCH;
  if (desc->L >= 3) {
    PoolParams p;
    memset(&p, 0, sizeof(p));
    for (int l = 1; l <= desc->L; ++l) {
      p.lvl[0][l] = out->q[l];
      p.lvl[1][l] = out->k[l];
      p.lvl[2][l] = (l >= 2) ? out->v[l] : nullptr;
    }
    p.BH = desc->B * desc->H;
    p.N = desc->N;
    p.D = desc->D;
    p.L = desc->L;
    e = launch_pool_up(p, (cudaStream_t)stream);
  }
  return launch_status(e);
}

int llsa_select(const llsa_desc* desc, const llsa_pyramid* pyr, const llsa_indices* out,
                void* stream) {
  int st = check_desc(desc);
  if (st != LLSA_OK) return st;
  st = check_select_args(desc, pyr, out);
  if (st != LLSA_OK) return st;
  const int BH = desc->B * desc->H;
  for (int l = desc->L; l >= 1; --l) {
    st = launch_status(launch_select_level(select_params(desc, pyr, out, l), BH, desc->D, (cudaStream_t)stream));
    if (st != LLSA_OK) return st;
  }
  return LLSA_OK;
}

int llsa_attn_fwd(const llsa_desc* desc, const void* q, const void* k, const void* v,
                  const llsa_pyramid* pyr, const llsa_indices* idx, void* o, float* lse,
                  int32_t* dev_status, void* stream) {
  int st = check_desc(desc);
  if (st != LLSA_OK) return st;
  FwdPlan f;
  st = plan_fwd(desc, q, k, v, pyr, idx, o, nullptr, lse, dev_status, f);
  if (st != LLSA_OK) return st;
  return launch_fwd(f, (cudaStream_t)stream);
}

int llsa_select_attn_fwd(const llsa_desc* desc, const void* q, const void* k, const void* v,
                         const llsa_pyramid* pyr, const llsa_indices* idx, void* o, float* lse,
                         int32_t* dev_status, void* stream) {
  int st = check_desc(desc);
  if (st != LLSA_OK) return st;
  st = check_select_args(desc, pyr, idx);
  if (st != LLSA_OK) return st;
  FwdPlan f;
  st = plan_fwd(desc, q, k, v, pyr, idx, o, nullptr, lse, dev_status, f);
  if (st != LLSA_OK) return st;
  const cudaStream_t s = (cudaStream_t)stream;
  const int BH = desc->B * desc->H;
  for (int l = desc->L; l >= 2; --l) {
    st = launch_status(launch_select_level(select_params(desc, pyr, idx, l), BH, desc->D, s));
    if (st != LLSA_OK) return st;
  }
  const SelectParams s1 = select_params(desc, pyr, idx, 1);
  if (f.path == FwdPath::kMma)  // level 1 selected in the forward's prologue
    return launch_status(launch_attn_fwd_mma_select(f.p, s1, f.maps, s));
  st = launch_status(launch_select_level(s1, BH, desc->D, s));
  if (st != LLSA_OK) return st;
  return launch_fwd(f, s);
}

size_t llsa_transpose_workspace_bytes(const llsa_desc* desc) {
  if (check_desc(desc) != LLSA_OK) return 0;
  return tr_ws_layout(desc).total;
}

int llsa_index_transpose(const llsa_desc* desc, const llsa_indices* idx, const llsa_csr* out,
                         void* ws, size_t ws_bytes, int32_t* dev_status, void* stream) {
  int st = check_desc(desc);
  if (st != LLSA_OK) return st;
  if (idx == nullptr || out == nullptr || ws == nullptr || !indices_present(desc, idx, key_top(desc)))
    return LLSA_ERR_INVALID_ARG;
  if (((uintptr_t)ws & 255) != 0) return LLSA_ERR_INVALID_ARG;
  const TrWsLayout w = tr_ws_layout(desc);
  if (ws_bytes < w.total) return LLSA_ERR_WORKSPACE;
  TransposeParams p;
  memset(&p, 0, sizeof(p));
  p.BH = desc->B * desc->H;
  p.status = dev_status;
  p.nlev = key_top(desc);
  int cta = 0, tile = 0, scan = 0;
  for (int l = 1; l <= p.nlev; ++l) {
    if (out->row_ptr[l] == nullptr || out->col[l] == nullptr) return LLSA_ERR_INVALID_ARG;
    TransposeLevel& t = p.lv[l - 1];
    t.idx = idx->idx[l];
    t.row_ptr = out->row_ptr[l];
    t.col = out->col[l];
    t.cnt = reinterpret_cast<int32_t*>(static_cast<char*>(ws) + w.off[l]);
    t.n = n_level(desc, l);
    t.K = k_level(desc, l);
    transpose_chunking(t.n, &t.nchunk, &t.rows);
    t.cta_begin = cta;
    t.tile_begin = tile;
    t.scan_begin = scan;
    cta += p.BH * t.nchunk;
    tile += p.BH * transpose_prefix_tiles(t.n);
    scan += p.BH;
  }
  return launch_status(launch_transpose(p, (cudaStream_t)stream));
}

size_t llsa_bwd_workspace_bytes(const llsa_desc* desc) {
  if (check_desc(desc) != LLSA_OK) return 0;
  return ws_layout(desc).total;
}

int llsa_attn_bwd(const llsa_desc* desc, const void* q, const void* k, const void* v,
                  const llsa_pyramid* pyr, const void* o, const float* lse, const void* dout,
                  const llsa_indices* idx, const llsa_csr* csr, void* dq, void* dk, void* dv,
                  void* ws, size_t ws_bytes, int32_t* dev_status, void* stream) {
  return attn_bwd_impl(desc, q, k, v, pyr, o, nullptr, lse, dout, idx, csr, dq, dk, dv, ws, ws_bytes, dev_status,
                       stream);
}

int llsa_attn_bwd_res(const llsa_desc* desc, const void* q, const void* k, const void* v,
                      const llsa_pyramid* pyr, const void* o, const void* o_res, const float* lse,
                      const void* dout, const llsa_indices* idx, const llsa_csr* csr, void* dq, void* dk,
                      void* dv, void* ws, size_t ws_bytes, int32_t* dev_status, void* stream) {
  if (desc != nullptr && desc->dtype == LLSA_BF16 && o_res == nullptr) return LLSA_ERR_INVALID_ARG;
  return attn_bwd_impl(desc, q, k, v, pyr, o, o_res, lse, dout, idx, csr, dq, dk, dv, ws, ws_bytes, dev_status,
                       stream);
}

int llsa_attn_fwd_res(const llsa_desc* desc, const void* q, const void* k, const void* v,
                      const llsa_pyramid* pyr, const llsa_indices* idx, void* o, void* o_res, float* lse,
                      int32_t* dev_status, void* stream) {
  int st = check_desc(desc);
  if (st != LLSA_OK) return st;
  if (desc->dtype == LLSA_BF16) {  // fp32: O is not rounded, o_res is not used
    if (o_res == nullptr || ((uintptr_t)o_res & 15) != 0) return LLSA_ERR_INVALID_ARG;
  }
  FwdPlan f;
  st = plan_fwd(desc, q, k, v, pyr, idx, o, desc->dtype == LLSA_BF16 ? o_res : nullptr, lse, dev_status, f);
  if (st != LLSA_OK) return st;
  return launch_fwd(f, (cudaStream_t)stream);
}

}  // extern "C"

namespace {

int attn_bwd_impl(const llsa_desc* desc, const void* q, const void* k, const void* v, const llsa_pyramid* pyr,
                  const void* o, const void* o_res, const float* lse, const void* dout,
                  const llsa_indices* idx, const llsa_csr* csr, void* dq, void* dk, void* dv, void* ws,
                  size_t ws_bytes, int32_t* dev_status, void* stream) {
  int st = check_desc(desc);
  if (st != LLSA_OK) return st;
  if (q == nullptr || k == nullptr || v == nullptr || o == nullptr || lse == nullptr ||
      dout == nullptr || idx == nullptr || csr == nullptr || pyr == nullptr || dq == nullptr ||
      dk == nullptr || dv == nullptr || ws == nullptr)
    return LLSA_ERR_INVALID_ARG;
  if (((uintptr_t)ws & 255) != 0) return LLSA_ERR_INVALID_ARG;
  const int p_top = key_top(desc);
  if (!indices_present(desc, idx, p_top) || !coarse_kv_present(desc, pyr)) return LLSA_ERR_INVALID_ARG;
  for (int l = 1; l <= p_top; ++l)
    if (csr->row_ptr[l] == nullptr || csr->col[l] == nullptr) return LLSA_ERR_INVALID_ARG;
  const WsLayout w = ws_layout(desc);
  if (ws_bytes < w.total) return LLSA_ERR_WORKSPACE;
  AttnParams p;
  fill_attn_common(p, desc, q, k, v, pyr, idx);
  p.o = o;
  p.lse_in = lse;
  p.dout = dout;
  for (int l = 1; l <= p_top; ++l) {
    p.row_ptr[l] = csr->row_ptr[l];
    p.col[l] = csr->col[l];
  }
  char* base = static_cast<char*>(ws);
  p.delta = reinterpret_cast<float*>(base + w.delta);
  for (int l = 2; l <= p_top; ++l) {
    p.part[l] = reinterpret_cast<float*>(base + w.part[l]);
    p.coarse[l] = reinterpret_cast<float*>(base + w.coarse[l]);
  }
  p.work = reinterpret_cast<int32_t*>(base + w.work);
  p.dq = dq;
  p.dk = dk;
  p.dv = dv;
  p.status = dev_status;
  if (desc->dtype == LLSA_F32)  // O is stored unrounded: a residual is not used
    return launch_status(launch_attn_bwd_simt(p, desc->dtype, (cudaStream_t)stream));
  // bf16: tensor-core kernels with TMA gathers
  if ((((uintptr_t)dq | (uintptr_t)dk | (uintptr_t)dv | (uintptr_t)lse | (uintptr_t)o_res) & 15) != 0)
    return LLSA_ERR_INVALID_ARG;  // 16-byte stores and bulk copies
  p.o_res = const_cast<void*>(o_res);
  const uint64_t rows = (uint64_t)desc->B * desc->H * desc->N;
  if (rows > 0x7fffffffULL) return LLSA_ERR_UNSUPPORTED;  // TMA row coordinates are int32
  CUtensorMap maps[4];
  const void* srcs[4] = {q, k, v, dout};
  for (int i = 0; i < 4; ++i) {
    st = make_row_tile_map(&maps[i], srcs[i], rows, desc->D);
    if (st != LLSA_OK) return st;
  }
  const bool tc_kv = (desc->flags & LLSA_FLAG_BWD_TCGEN05) != 0;
  return launch_status(launch_attn_bwd_mma(p, maps, (cudaStream_t)stream, tc_kv));
}

}  // namespace
