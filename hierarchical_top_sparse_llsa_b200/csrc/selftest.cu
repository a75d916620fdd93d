// llsa_selftest_wait_timeout: one launch whose only work is a bounded wait on
// an mbarrier that nothing ever arrives on.  The attention kernels wait on
// mbarriers for their TMA copies and tensor-core results; each of those waits
// is bounded by the global timer and, when it runs out, the kernel reports
// LLSA_DEV_TIMEOUT in the caller's status word and returns instead of holding
// the GPU.  A correct launch never gets there, so this entry point lets a
// test drive the same wait helper to expiry, with no copy in flight and no
// fault, and check that the status arrives and the stream stays usable.

#include "llsa_internal.cuh"
#include "sm100_ptx.cuh"

namespace {

__global__ void wait_timeout_kernel(int32_t* status, unsigned long long limit_ns) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    llsa::mbar_init(llsa::smem_u32(&bar), 1);  // one arrival completes phase 0; none comes
    llsa::fence_mbar_init();
  }
  __syncthreads();
  const bool done = llsa::mbar_wait_bounded(llsa::smem_u32(&bar), 0, limit_ns);
  if (!done && threadIdx.x == 0) llsa::report_status(status, LLSA_DEV_TIMEOUT);
}

}  // namespace

extern "C" int llsa_selftest_wait_timeout(int32_t* dev_status, unsigned limit_us, void* stream) {
  if (dev_status == nullptr || limit_us < 1 || limit_us > 2000000u) return LLSA_ERR_INVALID_ARG;
  wait_timeout_kernel<<<1, 32, 0, (cudaStream_t)stream>>>(dev_status, 1000ull * limit_us);
  return cudaGetLastError() == cudaSuccess ? LLSA_OK : LLSA_ERR_LAUNCH;
}
