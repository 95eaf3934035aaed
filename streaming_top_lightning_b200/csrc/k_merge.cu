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
SI_DEV void pool_take_keys(const uint64_t* keys, int n, uint64_t* pool, int cap, int K, int& np,
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

// Bitonic sort of 32*R keys held by one warp, blocked layout: lane l holds
// elements l*R .. l*R+R-1 in v[0..R).  Distances below R pair registers of one
// lane; larger ones pair lanes through xor-shuffles.  The lower index of each
// pair keeps the max where (index & size) == 0, so the result is descending.
template <int R, int S>
SI_DEV void bsort_reg(uint64_t (&v)[R], int lane, int size) {
#pragma unroll
  for (int r = 0; r < R; ++r) {
    if ((r & S) == 0) {
      const bool dir = ((lane * R + r) & size) == 0;
      const uint64_t a = v[r], b = v[r | S];
      const bool gt = a > b;
      const uint64_t mx = gt ? a : b, mn = gt ? b : a;
      v[r] = dir ? mx : mn;
      v[r | S] = dir ? mn : mx;
    }
  }
}

template <int R>
SI_DEV void warp_sort_blocked(uint64_t (&v)[R], int lane) {
#pragma unroll 1
  for (int size = 2; size <= 32 * R; size <<= 1) {
#pragma unroll 1
    for (int s = size >> 1; s > 0; s >>= 1) {
      if (s >= R) {
        const int lm = s / R;
        const bool lower = (lane & lm) == 0;
#pragma unroll
        for (int r = 0; r < R; ++r) {
          const bool dir = ((lane * R + r) & size) == 0;
          const uint64_t y = __shfl_xor_sync(0xFFFFFFFFu, v[r], lm);
          const bool gt = v[r] > y;
          v[r] = ((lower == dir) == gt) ? v[r] : y;
        }
      } else if (s == 8) {
        if constexpr (R > 8) bsort_reg<R, 8>(v, lane, size);
      } else if (s == 4) {
        if constexpr (R > 4) bsort_reg<R, 4>(v, lane, size);
      } else if (s == 2) {
        if constexpr (R > 2) bsort_reg<R, 2>(v, lane, size);
      } else {
        if constexpr (R > 1) bsort_reg<R, 1>(v, lane, size);
      }
    }
  }
}

// Sort the n (<= 32*R) selected keys in pool[0, n) and write the row.  The
// pool is unsorted, so reading it lane-interleaved (conflict-free) and
// treating that as the blocked layout loses nothing.
template <int R>
SI_DEV void sort_and_write(const uint64_t* pool, int n, int K, int32_t* oi, float* os, int lane) {
  uint64_t v[R];
#pragma unroll
  for (int r = 0; r < R; ++r) {
    const int i = 32 * r + lane;
    v[r] = i < n ? pool[i] : 0ull;
  }
  warp_sort_blocked<R>(v, lane);
#pragma unroll
  for (int r = 0; r < R; ++r) {
    const int e = lane * R + r;
    if (e < K) {
      const uint64_t k = v[r];
      oi[e] = k ? key_index(k) : -1;
      os[e] = k ? key_score(k) : __int_as_float(0xFF800000);
    }
  }
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
    pool_take_keys(base + ((int64_t)c * QT + qi) * L, L, pool, cap, K, np, theta, hist, lane);
  // exact K best: prune while far above K, then the radix select
  __syncwarp();
  if (np > K) {
    uint64_t th;
    while (np > K + K / 4 + 64 && pool_prune(pool, &np, K, &th, lane)) {
    }
    pool_shrink(pool, np, K, hist, lane);
    np = K;
  }
  const int n = np;
  const int64_t o = ((int64_t)b * sp.S + t) * K;
  __syncwarp();
  // K <= 512: sort here, in registers; larger K: unsorted rows, ordered by
  // the row-sort kernel afterwards
  const int n2 = pow2ceil(K < 32 ? 32 : K);
  switch (n2) {
    case 32: return sort_and_write<1>(pool, n, K, sp.out_idx + o, sp.out_score + o, lane);
    case 64: return sort_and_write<2>(pool, n, K, sp.out_idx + o, sp.out_score + o, lane);
    case 128: return sort_and_write<4>(pool, n, K, sp.out_idx + o, sp.out_score + o, lane);
    case 256: return sort_and_write<8>(pool, n, K, sp.out_idx + o, sp.out_score + o, lane);
    case 512: return sort_and_write<16>(pool, n, K, sp.out_idx + o, sp.out_score + o, lane);
    default: break;
  }
  for (int r = lane; r < K; r += 32) {
    const bool real = r < n;
    const uint64_t k = real ? pool[r] : 0ull;
    sp.out_idx[o + r] = real ? key_index(k) : -1;
    sp.out_score[o + r] = real ? key_score(k) : __int_as_float(0xFF800000);
  }
}

bool merge_sorts_rows(int K) { return K <= 512; }

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
