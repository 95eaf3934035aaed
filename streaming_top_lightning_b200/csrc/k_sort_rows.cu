// Orders every output row: real entries (index >= 0) by score descending,
// then index ascending, with -0 and +0 equal, followed by the -1 / -inf
// padding.  This is the order of the selection keys in si_common.cuh, rebuilt
// from the (index, score) pairs, so the order is exactly the one the top-k
// selection used ("StreamIndex: Memory-Bounded Compressed Sparse Attention via
// Streaming Top-k", Abstract: the top-k are selected per query; the sorted,
// lower-index-first order is this library's reading).
//
// The selection emits each query's K best keys unsorted; sorting here keeps
// the bitonic network off the fused kernel's critical path.  One CTA of 128
// threads sorts one row at a time (grid-stride over rows).  Each thread holds
// EPT consecutive keys (blocked layout, element e = tid*EPT + r) in registers:
// distances below EPT pair registers of one thread, distances below 32*EPT
// pair lanes of one warp (xor shuffles), and only the two largest distances
// go through shared memory.
#include "si_kernels.h"

namespace si {

constexpr int kSortThreads = 128;

template <int EPT, int S>
SI_DEV void sort_stage_reg(uint64_t (&v)[EPT], int e0, int size) {
#pragma unroll
  for (int r = 0; r < EPT; ++r) {
    if ((r & S) == 0) {
      const bool dir = ((e0 + r) & size) == 0;  // lower index keeps the max
      const uint64_t a = v[r], b = v[r | S];
      const bool gt = a > b;
      const uint64_t mx = gt ? a : b, mn = gt ? b : a;
      v[r] = dir ? mx : mn;
      v[r | S] = dir ? mn : mx;
    }
  }
}

template <int EPT>
SI_DEV void sort_stage_pair(uint64_t (&v)[EPT], const uint64_t (&y)[EPT], int e0, int size,
                            bool lower) {
#pragma unroll
  for (int r = 0; r < EPT; ++r) {
    const bool dir = ((e0 + r) & size) == 0;
    const bool gt = v[r] > y[r];
    v[r] = ((lower == dir) == gt) ? v[r] : y[r];
  }
}

template <int EPT>
__global__ void __launch_bounds__(kSortThreads)
    k_sort_rows(int32_t* __restrict__ idx, float* __restrict__ score, int64_t rows, int K) {
  constexpr int N2 = kSortThreads * EPT;
  __shared__ uint64_t xs[N2];  // exchange buffer for the cross-warp distances
  const int tid = threadIdx.x;
  const int e0 = tid * EPT;
  for (int64_t row = blockIdx.x; row < rows; row += gridDim.x) {
    int32_t* ri = idx + row * K;
    float* rs = score + row * K;
    uint64_t v[EPT];
#pragma unroll
    for (int r = 0; r < EPT; ++r) {
      const int e = e0 + r;
      uint64_t k = 0ull;
      if (e < K) {
        const int j = ri[e];
        if (j >= 0) k = make_key(rs[e], j);
      }
      v[r] = k;
    }
#pragma unroll 1
    for (int size = 2; size <= N2; size <<= 1) {
#pragma unroll 1
      for (int s = size >> 1; s > 0; s >>= 1) {
        if (s < EPT) {
          if (s == 8) {
            if constexpr (EPT > 8) sort_stage_reg<EPT, 8>(v, e0, size);
          } else if (s == 4) {
            if constexpr (EPT > 4) sort_stage_reg<EPT, 4>(v, e0, size);
          } else if (s == 2) {
            if constexpr (EPT > 2) sort_stage_reg<EPT, 2>(v, e0, size);
          } else {
            if constexpr (EPT > 1) sort_stage_reg<EPT, 1>(v, e0, size);
          }
        } else {
          const int ts = s / EPT;  // partner thread is tid ^ ts
          uint64_t y[EPT];
          if (ts < 32) {
#pragma unroll
            for (int r = 0; r < EPT; ++r) y[r] = __shfl_xor_sync(0xFFFFFFFFu, v[r], ts);
          } else {
#pragma unroll
            for (int r = 0; r < EPT; ++r) xs[e0 + r] = v[r];
            __syncthreads();
            const int p0 = (tid ^ ts) * EPT;
#pragma unroll
            for (int r = 0; r < EPT; ++r) y[r] = xs[p0 + r];
            __syncthreads();
          }
          sort_stage_pair<EPT>(v, y, e0, size, (tid & ts) == 0);
        }
      }
    }
#pragma unroll
    for (int r = 0; r < EPT; ++r) {
      const int e = e0 + r;
      if (e < K) {
        const uint64_t k = v[r];
        ri[e] = k ? key_index(k) : -1;
        rs[e] = k ? key_score(k) : __int_as_float(0xFF800000);
      }
    }
  }
}

template <int EPT>
static cudaError_t launch_sort_t(int32_t* idx, float* score, int64_t rows, int K, int sms,
                                 cudaStream_t stream) {
  const int64_t want = (int64_t)sms * 16;
  const int grid = (int)(rows < want ? rows : want);
  k_sort_rows<EPT><<<grid, kSortThreads, 0, stream>>>(idx, score, rows, K);
  return cudaGetLastError();
}

cudaError_t launch_sort_rows(int32_t* idx, float* score, int64_t rows, int K, int sms,
                             cudaStream_t stream) {
  if (rows <= 0) return cudaSuccess;
  const int n2 = pow2ceil(K < kSortThreads ? kSortThreads : K);
  switch (n2 / kSortThreads) {
    case 1: return launch_sort_t<1>(idx, score, rows, K, sms, stream);
    case 2: return launch_sort_t<2>(idx, score, rows, K, sms, stream);
    case 4: return launch_sort_t<4>(idx, score, rows, K, sms, stream);
    case 8: return launch_sort_t<8>(idx, score, rows, K, sms, stream);
    case 16: return launch_sort_t<16>(idx, score, rows, K, sms, stream);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace si
