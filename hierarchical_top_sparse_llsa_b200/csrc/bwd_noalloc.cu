// llsa_attn_bwd_noalloc: the sparse-attention backward with its scratch
// memory taken from a fixed array inside the library instead of from the
// caller.
//
// Who needs it: callers that cannot hand the backward a workspace, because
// they cannot call cudaMalloc at that point -- a plugin host that gives
// kernels no allocator and no workspace, a runtime whose device memory is
// fixed when it starts, or a latency-critical loop that must not call
// cudaMalloc, which can block and synchronise the device.  Such callers
// still pass every input and output buffer; only the scratch comes from here.
//
// The scratch is one file-scope device array of LLSA_NOALLOC_SCRATCH_BYTES
// (16 MiB).  Every GPU that loads this library holds it until the process
// exits.  Host code cannot use the array's name as a device address (in host
// code it names a host-side stand-in), so its device address is looked up
// with cudaGetSymbolAddress, with the device current, on the first call made
// on that device, and cached together with the CUDA context it belongs to.
// A later call under another context of the same device (after
// cudaDeviceReset, say, which reloads the library's module at a possibly
// different address) looks the address up again.
//
// All calls share the one array and it keeps whatever the last call wrote.
// Nothing in it has to start at zero: the backward kernels zero their own
// partial sums and write every other scratch word before reading it.  Two
// calls whose work overlaps on the GPU (for instance on two streams) race
// on the array and give wrong results; serialise them.

#include <cuda.h>

#include <mutex>

#include "llsa_internal.cuh"

namespace {

constexpr size_t kScratchBytes = LLSA_NOALLOC_SCRATCH_BYTES;
static __device__ __align__(256) unsigned char g_bwd_scratch[kScratchBytes];

constexpr int kMaxDevices = 64;
struct CachedAddress {
  CUcontext ctx;
  void* addr;
};
std::mutex g_mutex;
CachedAddress g_scratch[kMaxDevices] = {};

// cuCtxGetCurrent from the driver (no link-time libcuda), fetched once.
typedef CUresult (*CtxGetCurrentFn)(CUcontext*);
CtxGetCurrentFn ctx_get_current() {
  static CtxGetCurrentFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<CtxGetCurrentFn>(f);
  });
  return fn;
}

// Device address of the scratch array on the current device, looked up on
// the first call under each context of the device.
int scratch_on_current_device(void** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return LLSA_ERR_LAUNCH;
  CtxGetCurrentFn get_ctx = ctx_get_current();
  if (get_ctx == nullptr) return LLSA_ERR_LAUNCH;
  std::lock_guard<std::mutex> lock(g_mutex);
  CUcontext ctx = nullptr;
  if (get_ctx(&ctx) != CUDA_SUCCESS) return LLSA_ERR_LAUNCH;
  CachedAddress& c = g_scratch[dev];
  if (ctx == nullptr || ctx != c.ctx || c.addr == nullptr) {
    void* p = nullptr;  // the lookup also makes the device's context current
    const cudaError_t e = cudaGetSymbolAddress(&p, g_bwd_scratch);
    if (e != cudaSuccess || p == nullptr) return LLSA_ERR_LAUNCH;
    if (get_ctx(&ctx) != CUDA_SUCCESS || ctx == nullptr) return LLSA_ERR_LAUNCH;
    c.ctx = ctx;
    c.addr = p;
  }
  *out = c.addr;
  return LLSA_OK;
}

}  // namespace

extern "C" int llsa_attn_bwd_noalloc(const llsa_desc* desc, const void* q, const void* k,
                                     const void* v, const llsa_pyramid* pyr, const void* o,
                                     const float* lse, const void* dout, const llsa_indices* idx,
                                     const llsa_csr* csr, void* dq, void* dk, void* dv,
                                     int32_t* dev_status, void* stream) {
  const size_t need = llsa_bwd_workspace_bytes(desc);
  if (need == 0)  // the descriptor is invalid: let the backward report exactly why
    return llsa_attn_bwd(desc, q, k, v, pyr, o, lse, dout, idx, csr, dq, dk, dv, nullptr, 0,
                         dev_status, stream);
  if (need > kScratchBytes) return LLSA_ERR_WORKSPACE;
  void* ws = nullptr;
  const int st = scratch_on_current_device(&ws);
  if (st != LLSA_OK) return st;
  return llsa_attn_bwd(desc, q, k, v, pyr, o, lse, dout, idx, csr, dq, dk, dv, ws, kScratchBytes,
                       dev_status, stream);
}
