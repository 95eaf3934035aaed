// Partition-merge of per-chunk partial top-k lists.
//
// "StreamIndex: Memory-Bounded Compressed Sparse Attention via Streaming
// Top-k", Abstract: a chunked partition-merge top-k driver keeps the indexer
// from ever holding the full score tensor.  When a query's visible keys span
// several key chunks, each chunk's unit leaves a sorted partial list of K keys
// in scratch; this kernel folds them into the final answer.  Under the strict
// total order of the 64-bit keys, the top K of a union equals the top K of the
// per-part top Ks, so the result is exactly the top K over all chunks.
//
// One CTA per query.  The running list and the next partial list sit in shared
// memory; each fold is a merge path over 256 threads (8 outputs each) that
// rebuilds only the positions at or after the first one the partial list
// takes, staged through registers so it can run in place.
#include "si_select.cuh"
#include "si_kernels.h"

namespace si {

constexpr int kMergeThreads = 256;

__global__ void __launch_bounds__(kMergeThreads)
    k_merge(const uint64_t* __restrict__ partial, SelParams sp, UnitGrid ug) {
  extern __shared__ __align__(16) uint8_t smem[];
  const int K = sp.K, QT = sp.QT;
  int cta = blockIdx.x;
  const int qi = cta % QT;
  cta /= QT;
  const int gl = cta % sp.n_tiles;
  const int b = cta / sp.n_tiles;
  const int g = sp.g_lo + gl;
  const int t = g * QT + qi;
  if (t >= sp.S) return;
  const int nch = tile_chunks(ug, g);
  if (nch <= 1) return;

  uint64_t* L = reinterpret_cast<uint64_t*>(smem);
  uint64_t* C = L + K;
  __shared__ int s_f;
  const int tid = threadIdx.x;
  const uint64_t* base = partial + (((int64_t)b * sp.n_tiles + gl) * sp.nch_max) * QT * K;
  auto list = [&](int c) { return base + ((int64_t)c * QT + qi) * K; };

  for (int r = tid; r < K; r += kMergeThreads) L[r] = list(0)[r];
  for (int c = 1; c < nch; ++c) {
    const uint64_t* src = list(c);
    for (int r = tid; r < K; r += kMergeThreads) C[r] = src[r];
    __syncthreads();
    if (tid == 0) {
      const uint64_t c0 = C[0];
      int lo = 0, hi = K;
      if (c0 == 0ull) {
        lo = K;  // empty partial list: nothing to fold
      } else {
        while (lo < hi) {
          const int mid = (lo + hi) >> 1;
          if (L[mid] > c0) lo = mid + 1;
          else hi = mid;
        }
      }
      s_f = lo;
    }
    __syncthreads();
    const int f = s_f;
    uint64_t* A = L + f;
    const int na = K - f;
    const int n = K;
    constexpr int R = kMergeR, P = kMergeThreads * R;
    for (int ph = (na + P - 1) / P - 1; ph >= 0; --ph) {
      const int d = ph * P + tid * R;
      uint64_t v[R];
      if (d < na) {
        int l2 = d - n > 0 ? d - n : 0;
        int h2 = d < na ? d : na;
        while (l2 < h2) {
          const int mid = (l2 + h2) >> 1;
          if (A[mid] > C[d - 1 - mid]) l2 = mid + 1;
          else h2 = mid;
        }
        int ia = l2, ib = d - l2;
#pragma unroll
        for (int r = 0; r < R; ++r) {
          if (d + r < na) {
            const bool take_a = (ib >= n) || (ia < na && A[ia] > C[ib]);
            v[r] = take_a ? A[ia] : C[ib];
            ia += take_a ? 1 : 0;
            ib += take_a ? 0 : 1;
          }
        }
      }
      __syncthreads();
      if (d < na) {
#pragma unroll
        for (int r = 0; r < R; ++r)
          if (d + r < na) A[d + r] = v[r];
      }
      __syncthreads();
    }
  }
  __syncthreads();
  const int64_t o = ((int64_t)b * sp.S + t) * K;
  for (int r = tid; r < K; r += kMergeThreads) {
    const uint64_t k = L[r];
    sp.out_idx[o + r] = k ? key_index(k) : -1;
    sp.out_score[o + r] = k ? key_score(k) : __int_as_float(0xFF800000);
  }
}

cudaError_t launch_merge(const uint64_t* partial, const SelParams& sp, const UnitGrid& ug,
                         cudaStream_t stream) {
  const size_t smem = sizeof(uint64_t) * 2 * sp.K;
  cudaError_t e =
      cudaFuncSetAttribute(k_merge, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const int grid = ug.B * sp.n_tiles * sp.QT;
  k_merge<<<grid, kMergeThreads, smem, stream>>>(partial, sp, ug);
  return cudaGetLastError();
}

}  // namespace si
