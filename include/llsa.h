/*
 * llsa.h - C ABI of the B200 (sm_100a) Log-linear Sparse Attention library.
 *
 * The method is "Trainable Log-linear Sparse Attention for Efficient Diffusion
 * Transformers" (arXiv 2512.16615).  Each entry point below cites the section
 * of the howistudyai explainer of that paper which defines its operation.
 *
 * Conventions for every call
 * --------------------------
 *  - Tokens: N fine tokens per (batch, head) in Z-order (Step 5: Index
 *    Reordering for Images), so 16 consecutive tokens are a 4x4 pixel tile.
 *  - Levels: level 0 is the fine tokens; level l (1 <= l <= L) has
 *    N_l = N / 16^l tokens, each the mean of 16 level-(l-1) tokens.  A level-1
 *    token is a 16-token query/key block.  N must be a multiple of 16^L.
 *  - Layout: every tensor is contiguous [B, H, tokens, D], D innermost.
 *    Q, K, V, O, dO, dQ, dK, dV hold `dtype` elements; pyramids are fp32.
 *  - Index lists I(l): int32 [B, H, N_l, K_l] (K_l = topk_l[l], else topk).
 *    Row q lists the level-l key tokens kept for level-l query token q,
 *    ascending, padded with -1 at the tail.  Kernels that read index lists use an entry iff it lies in
 *    [0, N_l) and is larger than every entry used before it in the row; any
 *    other entry is skipped and reported through `dev_status` (never a fault).
 *  - Memory: the caller allocates and owns every buffer (device memory unless
 *    stated otherwise).  The library allocates nothing and keeps no state
 *    between calls.  Calls are asynchronous on `stream` (a cudaStream_t; NULL
 *    is the legacy default stream); buffers must stay valid until the work on
 *    the stream has finished.
 *  - Host errors: the return value.  Arguments are checked before any launch;
 *    on an error nothing is enqueued.
 *  - Device errors: a bit set OR-ed into *dev_status (a device int32 the
 *    caller zeroes and reads after synchronising), if dev_status is not NULL.
 *  - Versions: llsa_version() changes whenever a struct layout below does;
 *    bindings that mirror the structs should check it.
 */
#ifndef LLSA_H_
#define LLSA_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define LLSA_API __attribute__((visibility("default")))
#else
#define LLSA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

#define LLSA_MAX_LEVELS 6 /* L <= 6 */
#define LLSA_MAX_TOPK 32  /* topk <= 32 */
#define LLSA_BLOCK 16     /* tokens per block and pooling factor per level */

/* element types of Q, K, V, O, dO, dQ, dK, dV */
enum { LLSA_F32 = 0, LLSA_BF16 = 1 };

/* host status (return values) */
enum {
  LLSA_OK = 0,
  LLSA_ERR_INVALID_ARG = 1, /* NULL pointer, bad shape, N not a multiple of 16^L, ... */
  LLSA_ERR_UNSUPPORTED = 2, /* D not in {64, 128}, topk or a K_l > 32, L > 6, ... */
  LLSA_ERR_LAUNCH = 3,      /* a kernel launch failed (cudaGetLastError) */
  LLSA_ERR_WORKSPACE = 4    /* workspace smaller than the matching *_workspace_bytes() */
};

/* descriptor flags */
enum {
  /* bf16: run the forward (llsa_attn_fwd, llsa_attn_fwd_res, the forward of
   * llsa_select_attn_fwd) on the tcgen05 kernel: a persistent kernel whose
   * groups of 8 sibling query blocks (128 rows, one MMA) walk the union of
   * their selected key blocks with S and O in tensor memory.  Without a
   * forward flag the library picks the faster kernel for the head dim, as
   * measured on B200: tcgen05 at D = 128, the warp-MMA kernel at D = 64.
   * Excludes LLSA_FLAG_FWD_MMA_SYNC. */
  LLSA_FLAG_FWD_TCGEN05 = 1,
  /* bf16, D = 64: run the key-major pass of llsa_attn_bwd (dK, dV) on the
   * tcgen05 kernel (8 query blocks of a key block per 128-row MMA, dK and dV
   * accumulated in tensor memory) instead of the warp-MMA kernel. */
  LLSA_FLAG_BWD_TCGEN05 = 2,
  /* bf16: run the forward on the warp-level mma.sync kernel (one warp per 4
   * query blocks, registers as accumulators, each block against exactly its
   * own key blocks).  Both kernels compute the same result within bf16
   * rounding.  The library also takes this kernel when the coarse keys of one
   * CTA need more shared memory than the tcgen05 kernel has (the sum of K_l
   * over levels 2..Lc above 128 at D = 128). */
  LLSA_FLAG_FWD_MMA_SYNC = 4
};

/* device status bits (OR-ed into *dev_status) */
enum {
  LLSA_DEV_BAD_INDEX = 1,    /* an index entry outside [-1, N_l) was skipped */
  LLSA_DEV_NONCANONICAL = 2, /* a duplicate, unsorted entry or a pad before a valid entry */
  LLSA_DEV_TIMEOUT = 4       /* a bounded wait inside a kernel gave up */
};

/* Problem description (plain data, passed by pointer, read before launch). */
typedef struct {
  int B, H, N, D; /* batch, heads, fine tokens, head dim (64 or 128) */
  int L;          /* number of pooled levels, 1 <= L <= LLSA_MAX_LEVELS */
  int topk;       /* K, kept keys per level, 1 <= K <= LLSA_MAX_TOPK (see topk_l) */
  int dtype;      /* LLSA_F32 or LLSA_BF16 */
  int flags;      /* LLSA_FLAG_* bits; other bits must be 0 */
  float sm_scale; /* softmax scale; 0 selects 1/sqrt(D) */
  /* level_w[l], l = 2..L: weight of the coarse keys of level l (KV
   * Reweighting; the paper's setting is 16^l).  0 selects 1.  Entries 0, 1 and
   * above L are ignored. */
  float level_w[LLSA_MAX_LEVELS + 1];
  /* Enrichment depth Le (Hierarchical KV Enrichment): the coarse levels whose
   * pooled tokens join the keys are 2..Lc with Lc = min(L, 1 + Le).  0 selects
   * all of them (Lc = L); a negative value selects none (Lc = 1: fine keys
   * only).  Selection (llsa_select) always walks all L levels; the attention
   * calls and llsa_index_transpose use levels 1..Lc only, and the I(l), CSR
   * and pyramid entries of levels above Lc may be NULL there. */
  int enrich_levels;
  /* topk_l[l], l = 1..L: K_l, the keys kept at level l (a Top-K per level;
   * level l keeps K_l of the 16 * K_{l+1} children of its parent's keys).
   * 0 selects topk; entries 0 and above L are ignored.  I(l) rows and the
   * level-l CSR then have width K_l. */
  int topk_l[LLSA_MAX_LEVELS + 1];
} llsa_desc;

/* fp32 pyramid, [B, H, N_l, D] per level; entry 0 is unused. */
typedef struct {
  float* q[LLSA_MAX_LEVELS + 1]; /* levels 1..L */
  float* k[LLSA_MAX_LEVELS + 1]; /* levels 1..L */
  float* v[LLSA_MAX_LEVELS + 1]; /* levels 2..L (level-1 pooled V is never a key) */
} llsa_pyramid;

/* I(l), int32 [B, H, N_l, K_l] for l = 1..L; entry 0 is unused. */
typedef struct {
  int32_t* idx[LLSA_MAX_LEVELS + 1];
} llsa_indices;

/* Key-major lists per level l = 1..L: row_ptr int32 [B, H, N_l + 1] and
 * col int32 [B, H, N_l * K_l].  Row c of (b, h) is
 * col[row_ptr[c] .. row_ptr[c+1]), the level-l query tokens that kept key c,
 * ascending; offsets restart at 0 for every (b, h); col past row_ptr[N_l] is -1. */
typedef struct {
  int32_t* row_ptr[LLSA_MAX_LEVELS + 1];
  int32_t* col[LLSA_MAX_LEVELS + 1];
} llsa_csr;

/*
 * llsa_pool - hierarchical compression (Step 1; Building Blocks:
 * Hierarchical Compression).
 *   Q(l)[t] = mean of Q(l-1)[16t .. 16t+15] for l = 1..L, likewise K; V for
 *   l = 2..L (V(1) is formed internally).  Sums run left to right in fp32 with
 *   one rounding per addition and are then multiplied by 1/16, so the result
 *   is reproducible bit for bit.
 *   q, k, v: [B, H, N, D] of desc->dtype.  out: pyramid levels as listed in
 *   llsa_pyramid (all required).
 */
LLSA_API int llsa_pool(const llsa_desc* desc, const void* q, const void* k, const void* v,
              const llsa_pyramid* out, void* stream);

/*
 * llsa_qkv_pool - the QKV projection with the hierarchical compression in
 * its epilogue: the step before the path ("Input (Q, K, V) -> Hierarchical
 * Compression -> ..." in the pipeline overview; Step 1, Building Blocks:
 * Hierarchical Compression), fused so that Q, K and V are not read back.
 *   [Q | K | V] = X W^T on the tensor cores (bf16 inputs, fp32 accumulation,
 *   each output rounded once to bf16).  x: bf16 [B, N, C] row-major, tokens
 *   in Z-order; w: bf16 [3*H*D, C] row-major (a linear layer's weight: output
 *   feature t*H*D + h*D + d is tensor t = 0 Q, 1 K, 2 V, head h, channel d).
 *   q, k, v: written, bf16 [B, H, N, D] as the other calls take them.  out:
 *   the pyramid, written exactly as llsa_pool would write it from these q, k,
 *   v (bit for bit); every level listed in llsa_pyramid is required.
 *   Requires dtype LLSA_BF16, H*D a multiple of 128 and N a multiple of 256
 *   (else LLSA_ERR_UNSUPPORTED); C a positive multiple of 64 and every
 *   pointer 16-byte aligned (else LLSA_ERR_INVALID_ARG).  dev_status (may be
 *   NULL): LLSA_DEV_TIMEOUT if a bounded wait of the kernel gave up.
 */
LLSA_API int llsa_qkv_pool(const llsa_desc* desc, const void* x, const void* w, int C, void* q, void* k,
                           void* v, const llsa_pyramid* out, int32_t* dev_status, void* stream);

/*
 * llsa_select - hierarchical Top-K selection (Step 2; Building Blocks:
 * Hierarchical Top-K Selection).
 *   Level L: every level-L query token scores every level-L key token.
 *   Level l < L: query token q scores only the 16 children of each key kept
 *   by its parent q/16 in I(l+1).  Score = Q(l)[q] . K(l)[c], unscaled, in
 *   fp32 summed over d = 0..D-1 left to right with one rounding per multiply
 *   and per add (no FMA).  The min(K_l, #candidates) best scores are kept;
 *   equal scores (IEEE ==) go to the lower key index.  Rows are stored
 *   ascending with -1 padding.
 *   pyr: q[l], k[l] for l = 1..L (from llsa_pool).  out: I(1..L), written.
 */
LLSA_API int llsa_select(const llsa_desc* desc, const llsa_pyramid* pyr, const llsa_indices* out,
                void* stream);

/*
 * llsa_attn_fwd - sparse attention with hierarchical KV enrichment and KV
 * reweighting (Step 3; Building Blocks: Hierarchical KV Enrichment, KV
 * Reweighting).
 *   For query i of block b (i / 16 == b) the keys are the 16 fine tokens of
 *   every block in I(1)[b] (weight 1) and, for l = 2..Lc (Lc as enrich_levels
 *   gives it; L by default), the pooled tokens
 *   K(l)[c], V(l)[c] for c in I(l)[b / 16^(l-1)] (weight level_w[l]):
 *     s_ij = sm_scale * q_i . k_j
 *     O_i  = sum_j w_j e^{s_ij} v_j / sum_j w_j e^{s_ij}
 *     lse_i = ln sum_j w_j e^{s_ij}          (natural log)
 *   A query without keys gets O_i = 0 and lse_i = -inf.
 *   idx may be any caller-made index lists (no hierarchy consistency needed).
 *   idx: I(1..Lc).  pyr: k[l], v[l] for l = 2..Lc.  o: [B, H, N, D] dtype.
 *   lse: fp32 [B, H, N].
 *   dev_status: may be NULL.
 */
LLSA_API int llsa_attn_fwd(const llsa_desc* desc, const void* q, const void* k, const void* v,
                  const llsa_pyramid* pyr, const llsa_indices* idx, void* o, float* lse,
                  int32_t* dev_status, void* stream);

/*
 * llsa_select_attn_fwd - llsa_select followed by llsa_attn_fwd, with the
 * level-1 step of the selection done inside the forward kernel (each of its
 * CTAs owns the 16 sibling query blocks of one level-2 token, which is
 * exactly one level-1 selection group), so I(1) is not read back from memory
 * by a separate launch.  The paper's kernels run the two steps separately;
 * the fusion is this library's.
 *   Arguments as the two calls take them: pyr holds q[l], k[l] for l = 1..L
 *   and k[l], v[l] for l = 2..Lc; idx: I(1..L), all written (as llsa_select
 *   writes them; the backward needs them).  Results are identical to the two
 *   calls made one after the other.  The fusion is done by the warp-MMA
 *   forward (the D = 64 default, or LLSA_FLAG_FWD_MMA_SYNC); with the tcgen05
 *   forward and in fp32 the level-1 selection runs as its own launch before
 *   the forward.
 */
LLSA_API int llsa_select_attn_fwd(const llsa_desc* desc, const void* q, const void* k, const void* v,
                                  const llsa_pyramid* pyr, const llsa_indices* idx, void* o, float* lse,
                                  int32_t* dev_status, void* stream);

/*
 * llsa_attn_fwd_res - llsa_attn_fwd that also writes the rounding residual
 * of O, for a backward that takes it (llsa_attn_bwd_res).  The paper's
 * kernels have no counterpart: this is a speed option of this library.
 *   o_res: [B, H, N, D] bf16, 16-byte aligned, written with
 *   bf16(O_fp32 - float(o)) element by element, where O_fp32 is the kernel's
 *   fp32 output before rounding; o + o_res then holds O to about 16 mantissa
 *   bits.  o and lse are identical to llsa_attn_fwd's.
 *   dtype LLSA_F32: O is stored unrounded, o_res is not used (may be NULL).
 */
LLSA_API int llsa_attn_fwd_res(const llsa_desc* desc, const void* q, const void* k, const void* v,
                               const llsa_pyramid* pyr, const llsa_indices* idx, void* o, void* o_res,
                               float* lse, int32_t* dev_status, void* stream);

/*
 * llsa_transpose_workspace_bytes - device scratch size that
 * llsa_index_transpose needs for desc (0 on an invalid desc): per level,
 * B*H*nchunk*N_l int32 counts with nchunk <= 128 row chunks.
 */
LLSA_API size_t llsa_transpose_workspace_bytes(const llsa_desc* desc);

/*
 * llsa_index_transpose - sparse index transpose (Step 4; Building Blocks:
 * Sparse Index Transpose).
 *   For each level l = 1..Lc and (b, h): count the query tokens that kept each
 *   key token, prefix-sum the counts into row_ptr, and list the query tokens
 *   of each key in ascending order in col.  No dense mask is formed; the
 *   result is deterministic and uses no global atomics.
 *   idx: I(1..Lc), entries screened as the conventions above state.
 *   out: CSR of levels 1..Lc, written: row_ptr[l] int32 [B, H, N_l + 1],
 *   col[l] int32 [B, H, N_l * K] (slots past row_ptr[N_l] set to -1).
 *   ws: device scratch of at least llsa_transpose_workspace_bytes(desc)
 *   bytes, 256-byte aligned, not read before it is written (a smaller or
 *   missing one gives LLSA_ERR_WORKSPACE / LLSA_ERR_INVALID_ARG before any
 *   launch).  dev_status: may be NULL.
 */
LLSA_API int llsa_index_transpose(const llsa_desc* desc, const llsa_indices* idx, const llsa_csr* out,
                         void* ws, size_t ws_bytes, int32_t* dev_status, void* stream);

/*
 * llsa_bwd_workspace_bytes - device scratch size that llsa_attn_bwd needs
 * for desc (0 on an invalid desc).
 */
LLSA_API size_t llsa_bwd_workspace_bytes(const llsa_desc* desc);

/*
 * llsa_attn_bwd - gradients of llsa_attn_fwd with the indices held fixed
 * (Step 4: the key-major backward that the sparse index transpose serves).
 *   With P_ij = w_j e^{s_ij - lse_i} and Delta_i = dO_i . O_i:
 *     dS_ij = P_ij (dO_i . v_j - Delta_i)
 *     dQ_i  = sm_scale * sum_j dS_ij k_j
 *     dk_j  = sm_scale * sum_i dS_ij q_i ,  dv_j = sum_i P_ij dO_i
 *   A fine key's gradient goes to its token; a level-l coarse key's gradient
 *   is spread to each of its 16^l fine tokens divided by 16^l (the mean's
 *   derivative).  Selection passes no gradient.  Sums run in a fixed order
 *   without global atomics, so results are identical from run to run.
 *   o, lse: the outputs of llsa_attn_fwd (o must be valid but is not read:
 *   Delta_i = sum_j P_ij (dO_i . v_j) is recomputed from unrounded terms, as O
 *   itself is stored rounded to dtype).  dout: dO.  csr: llsa_index_transpose
 *   of the same idx (levels 1..Lc).  dq, dk, dv: [B, H, N, D] dtype, written.
 *   ws: device scratch of at least llsa_bwd_workspace_bytes(desc) bytes,
 *   256-byte aligned.  dev_status: may be NULL.
 */
LLSA_API int llsa_attn_bwd(const llsa_desc* desc, const void* q, const void* k, const void* v,
                  const llsa_pyramid* pyr, const void* o, const float* lse, const void* dout,
                  const llsa_indices* idx, const llsa_csr* csr, void* dq, void* dk, void* dv,
                  void* ws, size_t ws_bytes, int32_t* dev_status, void* stream);

/*
 * llsa_attn_bwd_res - llsa_attn_bwd with Delta_i = dO_i . (o_i + o_res_i)
 * (fp32 sums) from the residual that llsa_attn_fwd_res wrote, instead of
 * Delta_i = sum_j P_ij (dO_i . v_j) over the key set: the query-major pass
 * then walks each key list once instead of twice.  Within the same error bar
 * as llsa_attn_bwd, not bit-identical to it.
 *   o_res: bf16 [B, H, N, D], 16-byte aligned (NULL with bf16 gives
 *   LLSA_ERR_INVALID_ARG).  dtype LLSA_F32: o_res is not used (may be NULL;
 *   O itself is unrounded) and the call equals llsa_attn_bwd.
 *   Other arguments as llsa_attn_bwd.
 */
LLSA_API int llsa_attn_bwd_res(const llsa_desc* desc, const void* q, const void* k, const void* v,
                               const llsa_pyramid* pyr, const void* o, const void* o_res, const float* lse,
                               const void* dout, const llsa_indices* idx, const llsa_csr* csr, void* dq,
                               void* dk, void* dv, void* ws, size_t ws_bytes, int32_t* dev_status,
                               void* stream);

/*
 * llsa_attn_bwd_noalloc - llsa_attn_bwd for callers that cannot allocate.
 *   The paper has no counterpart: this is a convenience of this library.
 *   Some callers cannot provide the backward's scratch buffer because they
 *   cannot call cudaMalloc there (a plugin host without an allocator, a
 *   runtime whose device memory is fixed at start-up, a latency-critical loop
 *   where cudaMalloc may block).  This entry point takes the same arguments as
 *   llsa_attn_bwd minus ws/ws_bytes and allocates nothing: its scratch is a
 *   fixed device array of LLSA_NOALLOC_SCRATCH_BYTES inside the library, held
 *   by every GPU that loads the library until the process exits.
 *   - Sizes: if llsa_bwd_workspace_bytes(desc) exceeds
 *     LLSA_NOALLOC_SCRATCH_BYTES the call returns LLSA_ERR_WORKSPACE and
 *     enqueues nothing (use llsa_attn_bwd with your own workspace instead).
 *   - Set-up: the first call on a device looks up the array's device address
 *     (cudaGetSymbolAddress, with that device current) and caches it with
 *     the device's CUDA context; make that first call before any stream
 *     capture.  The first call under a new context of the device (after
 *     cudaDeviceReset, for instance) looks it up again.
 *   - Sharing: every call uses the same array, which keeps the last call's
 *     contents (nothing in it needs to start at zero).  Calls whose work
 *     overlaps on the GPU race on it and give wrong results: serialise them.
 */
#define LLSA_NOALLOC_SCRATCH_BYTES ((size_t)16 << 20)
LLSA_API int llsa_attn_bwd_noalloc(const llsa_desc* desc, const void* q, const void* k,
                                   const void* v, const llsa_pyramid* pyr, const void* o,
                                   const float* lse, const void* dout, const llsa_indices* idx,
                                   const llsa_csr* csr, void* dq, void* dk, void* dv,
                                   int32_t* dev_status, void* stream);

/*
 * llsa_reorder - raster <-> Z-order permutation of the token axis (Step 5:
 * Index Reordering for Images), for callers whose tokens are in raster order
 * (token y * img_w + x for pixel (x, y)).  Z-order token t holds the pixel
 * whose x is made of the even bits of t and whose y of the odd bits, so 16
 * consecutive tokens form a 4x4 tile (the layout every other call expects).
 *   B, H: batch and heads; img_h == img_w, a power of two >= 4 (N = img_h *
 *   img_w tokens; other shapes give LLSA_ERR_UNSUPPORTED); D in {64, 128};
 *   dtype: LLSA_F32 or LLSA_BF16.
 *   src, dst: [B, H, N, D] device tensors of dtype, 16-byte aligned, not
 *   overlapping (overlap gives LLSA_ERR_INVALID_ARG).
 *   to_zorder: nonzero for raster -> Z-order, 0 for Z-order -> raster.
 */
LLSA_API int llsa_reorder(int B, int H, int img_h, int img_w, int D, int dtype, const void* src, void* dst,
                          int to_zorder, void* stream);

/*
 * llsa_selftest_wait_timeout - a check of the kernels' bounded waits.
 *   The paper has no counterpart: this is a test hook of this library.  The
 *   attention kernels wait on mbarriers for their copies and tensor-core
 *   results; every such wait gives up after a time limit (1 s of the GPU's
 *   global timer), reports LLSA_DEV_TIMEOUT in *dev_status and lets the
 *   kernel return, so a lost arrival never holds the GPU.  This call
 *   launches one kernel that runs the same wait on a barrier nothing arrives
 *   on, with a limit of limit_us microseconds, so a caller can see the
 *   time-out reported without any fault.
 *   dev_status: device int32 (required); LLSA_DEV_TIMEOUT is OR-ed into it.
 *   limit_us: 1 .. 2,000,000 (else LLSA_ERR_INVALID_ARG, nothing enqueued).
 */
LLSA_API int llsa_selftest_wait_timeout(int32_t* dev_status, unsigned limit_us, void* stream);

/* Static text for a host status code. */
LLSA_API const char* llsa_status_string(int status);

/* Library version, major * 10000 + minor * 100 + patch. */
LLSA_API int llsa_version(void);

#ifdef __cplusplus
}
#endif

#endif /* LLSA_H_ */
