// Orders every output row: real entries (index >= 0) by score descending,
// then index ascending, with -0 and +0 equal, followed by the -1 / -inf
// padding.  This is the order of the selection keys in si_common.cuh, rebuilt
// from the (index, score) pairs, so the order is exactly the one the top-k
// selection used ("StreamIndex: Memory-Bounded Compressed Sparse Attention via
// Streaming Top-k", Abstract: the top-k are selected per query; the sorted,
// lower-index-first order is this library's reading).
//
// The selection emits each query's K best keys unsorted; sorting here keeps
// the bitonic network off the fused kernel's critical path.  One CTA per row
// at a time (grid-stride), a bitonic sort of the row's keys in shared memory,
// many CTAs per SM.
#include "si_kernels.h"

namespace si {

constexpr int kSortThreads = 128;

__global__ void __launch_bounds__(kSortThreads)
    k_sort_rows(int32_t* __restrict__ idx, float* __restrict__ score, int64_t rows, int K, int n2) {
  extern __shared__ __align__(16) uint64_t keys[];  // [n2]
  const int tid = threadIdx.x;
  for (int64_t row = blockIdx.x; row < rows; row += gridDim.x) {
    int32_t* ri = idx + row * K;
    float* rs = score + row * K;
    for (int r = tid; r < n2; r += kSortThreads) {
      uint64_t k = 0ull;
      if (r < K) {
        const int j = ri[r];
        if (j >= 0) k = make_key(rs[r], j);
      }
      keys[r] = k;
    }
    __syncthreads();
    for (int size = 2; size <= n2; size <<= 1) {
      for (int s = size >> 1; s > 0; s >>= 1) {
        for (int i = tid; i < (n2 >> 1); i += kSortThreads) {
          const int lo = ((i & ~(s - 1)) << 1) | (i & (s - 1));
          const int hi = lo + s;
          const bool dir = (lo & size) == 0;  // lower index keeps the max
          const uint64_t x = keys[lo], y = keys[hi];
          if ((x < y) == dir) {
            keys[lo] = y;
            keys[hi] = x;
          }
        }
        __syncthreads();
      }
    }
    for (int r = tid; r < K; r += kSortThreads) {
      const uint64_t k = keys[r];
      ri[r] = k ? key_index(k) : -1;
      rs[r] = k ? key_score(k) : __int_as_float(0xFF800000);
    }
    __syncthreads();
  }
}

cudaError_t launch_sort_rows(int32_t* idx, float* score, int64_t rows, int K, int sms,
                             cudaStream_t stream) {
  if (rows <= 0) return cudaSuccess;
  const int n2 = pow2ceil(K < 2 ? 2 : K);
  const size_t smem = sizeof(uint64_t) * n2;
  cudaError_t e =
      cudaFuncSetAttribute(k_sort_rows, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const int64_t want = (int64_t)sms * 16;
  const int grid = (int)(rows < want ? rows : want);
  k_sort_rows<<<grid, kSortThreads, smem, stream>>>(idx, score, rows, K, n2);
  return cudaGetLastError();
}

}  // namespace si
