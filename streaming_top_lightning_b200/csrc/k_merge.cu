// Partition-merge of per-chunk partial top-k lists.
//
// "StreamIndex: Memory-Bounded Compressed Sparse Attention via Streaming
// Top-k", Abstract: a chunked partition-merge top-k driver keeps the indexer
// from ever holding the full score tensor.  Each (query tile, key chunk) unit
// leaves, per query, a 0-padded partial list of at most L candidate keys in
// scratch, a superset of that chunk's K best.  This kernel folds a query's
// lists and takes the exact K best.  Under the strict total order of the
// 64-bit keys, the top K of a union equals the top K of the union of any
// per-part supersets of the per-part top Ks, so the result is exactly the top
// K over all chunks.
//
// One warp per query, with the same candidate pool, threshold and radix
// select as the score kernel's selection (si_select.cuh).  For K <= 512 the
// warp also sorts its row in registers; larger rows are written unsorted and
// ordered by the row-sort kernel.
#include <algorithm>

#include "si_kernels.h"

namespace si {

constexpr int kMergeWarps = 4;

// Append the keys of one partial list that beat theta.  Eight keys per lane
// (256 per warp) are loaded before any is appended, so their global-memory
// latencies overlap.
SI_DEV void pool_take_list(const uint64_t* keys, int n, uint64_t* pool, int cap, int K, int& np,
                           uint64_t& theta, uint32_t* hist, int lane) {
  const uint32_t lt_mask = (1u << lane) - 1u;
  for (int r0 = 0; r0 < n; r0 += 256) {
    uint64_t k[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int r = r0 + u * 32 + lane;
      k[u] = r < n ? __ldg(keys + r) : 0ull;
    }
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      if (np + 32 > cap) {
        __syncwarp();
        if (!pool_prune(pool, &np, K, &theta, lane) || np + 32 > cap) {
          theta = pool_shrink(pool, np, K, hist, lane);
          np = K;
        }
      }
      const bool tk = k[u] > theta;  // 0 (padding) never beats theta
      const uint32_t mk = __ballot_sync(0xFFFFFFFFu, tk);
      if (tk) pool[np + __popc(mk & lt_mask)] = k[u];
      np += __popc(mk);
    }
  }
  __syncwarp();
}

__global__ void __launch_bounds__(kMergeWarps * 32)
    k_merge(const uint64_t* __restrict__ partial, SelParams sp, UnitGrid ug, int cap) {
  extern __shared__ __align__(16) uint8_t smem[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int K = sp.K, QT = sp.QT;
  uint32_t* hist = reinterpret_cast<uint32_t*>(smem) + warp * 256;
  uint64_t* pool = reinterpret_cast<uint64_t*>(smem + sizeof(uint32_t) * kMergeWarps * 256) +
                   (size_t)warp * cap;
  const int64_t qid = (int64_t)blockIdx.x * kMergeWarps + warp;
  if (qid >= (int64_t)sp.B * sp.n_tiles * QT) return;
  const int qi = (int)(qid % QT);
  const int gl = (int)((qid / QT) % sp.n_tiles);
  const int b = (int)(qid / ((int64_t)QT * sp.n_tiles));
  const int g = sp.g_lo + gl;
  const int t = g * QT + qi;
  if (t >= sp.S) return;
  const int nch = tile_chunks(ug, g);
  const int L = sp.L;
  const uint64_t* base = partial + (((int64_t)b * sp.n_tiles + gl) * sp.nch_max) * QT * L;
  int np = 0;
  uint64_t theta = 0ull;
  for (int c = 0; c < nch; ++c)
    pool_take_list(base + ((int64_t)c * QT + qi) * L, L, pool, cap, K, np, theta, hist, lane);
  // exact K best, sorted here for K <= 512 (else by the row-sort kernel)
  const int64_t o = ((int64_t)b * sp.S + t) * K;
  finish_row(pool, np, K, hist, sp.out_idx + o, sp.out_score + o, lane);
}

bool merge_sorts_rows(int K) { return rows_sorted_in_warp(K); }

cudaError_t launch_merge(const uint64_t* partial, const SelParams& sp, const UnitGrid& ug,
                         cudaStream_t stream) {
  // pool room: twice K keeps radix selects rare, and at least one step of
  // 64 keys beyond K
  const int K = sp.K;
  const int cap = ((std::max(K + 64, 2 * K) + 31) / 32) * 32;
  const size_t smem = sizeof(uint32_t) * kMergeWarps * 256 + sizeof(uint64_t) * kMergeWarps * cap;
  cudaError_t e =
      cudaFuncSetAttribute(k_merge, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const int64_t queries = (int64_t)ug.B * sp.n_tiles * sp.QT;
  const int grid = (int)((queries + kMergeWarps - 1) / kMergeWarps);
  k_merge<<<grid, kMergeWarps * 32, smem, stream>>>(partial, sp, ug, cap);
  return cudaGetLastError();
}

}  // namespace si
