// Raster <-> Z-order permutation of the token axis (Step 5 of the
// howistudyai explainer of "Trainable Log-linear Sparse Attention for
// Efficient Diffusion Transformers": Index Reordering for Images), for
// callers that hold raster-order tokens.  The Z-order index of pixel (x, y)
// interleaves their bits, x on the even bits and y on the odd ones, so that
// every 16 consecutive tokens are a 4x4 tile.
//
// A pure copy bound by HBM bandwidth: one thread per 16-byte chunk of a
// token row, 4 chunks in flight per thread; writes are contiguous, reads are
// whole token rows (128 or 256 bytes) from the permuted position.

#include "llsa_internal.cuh"

namespace llsa {

namespace {

constexpr int kReorderThreads = 256;
constexpr int kReorderUnroll = 4;

// the low 16 bits of v moved to the even bit positions (bit b -> bit 2b)
__device__ __forceinline__ uint32_t spread_bits(uint32_t v) {
  v &= 0x0000ffffu;
  v = (v | (v << 8)) & 0x00ff00ffu;
  v = (v | (v << 4)) & 0x0f0f0f0fu;
  v = (v | (v << 2)) & 0x33333333u;
  v = (v | (v << 1)) & 0x55555555u;
  return v;
}

// the even bits of v packed into the low 16 bits (bit 2b -> bit b)
__device__ __forceinline__ uint32_t gather_bits(uint32_t v) {
  v &= 0x55555555u;
  v = (v | (v >> 1)) & 0x33333333u;
  v = (v | (v >> 2)) & 0x0f0f0f0fu;
  v = (v | (v >> 4)) & 0x00ff00ffu;
  v = (v | (v >> 8)) & 0x0000ffffu;
  return v;
}

__global__ void __launch_bounds__(kReorderThreads)
reorder_kernel(const uint4* __restrict__ src, uint4* __restrict__ dst, long long rows, int N, int side_log2,
               int chunks, int to_zorder) {
  const long long total = rows * chunks;
  const long long stride = (long long)gridDim.x * kReorderThreads * kReorderUnroll;
  for (long long e0 = (long long)blockIdx.x * kReorderThreads * kReorderUnroll + threadIdx.x; e0 < total;
       e0 += stride) {
    uint4 v[kReorderUnroll];
#pragma unroll
    for (int u = 0; u < kReorderUnroll; ++u) {
      const long long e = e0 + (long long)u * kReorderThreads;
      if (e < total) {
        const long long row = e / chunks;
        const int j = (int)(e - row * chunks);
        const long long bh = row / N;
        const uint32_t t = (uint32_t)(row - bh * N);  // destination token
        uint32_t s;                                   // its source token
        if (to_zorder) {  // t is a Z-order token: take its pixel's raster row
          const uint32_t x = gather_bits(t), y = gather_bits(t >> 1);
          s = (y << side_log2) | x;
        } else {          // t = y * side + x: take the pixel's Z-order row
          const uint32_t x = t & ((1u << side_log2) - 1u), y = t >> side_log2;
          s = spread_bits(x) | (spread_bits(y) << 1);
        }
        v[u] = src[((long long)bh * N + s) * chunks + j];
      }
    }
#pragma unroll
    for (int u = 0; u < kReorderUnroll; ++u) {
      const long long e = e0 + (long long)u * kReorderThreads;
      if (e < total) dst[e] = v[u];
    }
  }
}

}  // namespace

cudaError_t launch_reorder(const void* src, void* dst, long long rows, int N, int side_log2, int row_bytes,
                           int to_zorder, cudaStream_t s) {
  const int chunks = row_bytes / 16;
  const long long total = rows * chunks;
  long long blocks = (total + (long long)kReorderThreads * kReorderUnroll - 1) / ((long long)kReorderThreads * kReorderUnroll);
  if (blocks > 148LL * 64) blocks = 148LL * 64;  // grid-stride beyond that
  if (blocks < 1) blocks = 1;
  reorder_kernel<<<(int)blocks, kReorderThreads, 0, s>>>(static_cast<const uint4*>(src), static_cast<uint4*>(dst), rows,
                                                         N, side_log2, chunks, to_zorder);
  return cudaGetLastError();
}

}  // namespace llsa
