// Top-k on a given fp32 score tensor [B,S,T], with the causal visibility rule.
//
// This is the selection stage of the indexer step on its own ("StreamIndex:
// Memory-Bounded Compressed Sparse Attention via Streaming Top-k", Abstract:
// the top-k are selected per query).  It runs the very same streaming
// selection device code as the fused score kernel; only the producer of the
// score strips differs: here four loader warps copy them from global memory.
// The result is bit-exact (indices and score bit patterns) against a plain
// sort of the visible scores.
#include "si_select.cuh"
#include "si_kernels.h"

namespace si {

constexpr int kLoadThreads = 128;
constexpr int kTopkThreads = kLoadThreads + kSelWarps * 32;

struct TopkScoresSmem {
  uint32_t unit;
  uint32_t go[2];  // per strip slot: a slot's flag is rewritten only two barriers later
  uint32_t abort;
};

__global__ void __launch_bounds__(kTopkThreads, 1)
    k_topk_scores(const float* __restrict__ X, SelParams sp, UnitGrid ug, int* counter,
                  uint32_t* err, uint64_t timeout_ns) {
  extern __shared__ __align__(1024) uint8_t smem[];
  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  const int QT = sp.QT, CS = sp.CS;

  // carve shared memory: selection state, strips, metadata, barriers
  SelSmem sm;
  uint8_t* p = smem;
  sel_state_carve(p, QT, sp.cap, sm);
  p += sel_state_bytes(QT, sp.cap);
  float* strip = reinterpret_cast<float*>(p);
  p += sizeof(float) * 2 * QT * CS;
  StripMeta* meta = reinterpret_cast<StripMeta*>(p);
  p += sizeof(StripMeta) * 2;
  uint64_t* bars = reinterpret_cast<uint64_t*>(p);
  p += sizeof(uint64_t) * 4;
  TopkScoresSmem* misc = reinterpret_cast<TopkScoresSmem*>(p);

  const uint32_t full_bar = smem_u32(bars), empty_bar = smem_u32(bars + 2);
  if (tid == 0) {
    mbar_init(full_bar, kLoadThreads);
    mbar_init(full_bar + 8, kLoadThreads);
    mbar_init(empty_bar, kSelWarps * 32);
    mbar_init(empty_bar + 8, kSelWarps * 32);
    misc->abort = 0u;
    mbar_fence_init();
  }
  for (int i = tid; i < QT; i += kTopkThreads) {
    sm.npool[i] = 0;
    sm.theta[i] = 0ull;
  }
  __syncthreads();

  Ctl ctl{err, &misc->abort, timeout_ns, nullptr};
  sm.strip = strip;
  sm.meta = meta;
  sm.full_bar = full_bar;
  sm.empty_bar = empty_bar;
  sm.nslot = 2;

  if (warp >= kLoadThreads / 32) {
    select_loop(sp, sm, ctl, warp - kLoadThreads / 32, lane);
  } else {
    uint32_t it = 0;
    bool more = true;
    while (more) {
      // thread 0 takes the next unit; the loader group agrees on it
      if (tid == 0) misc->unit = (uint32_t)(atomicAdd(counter, 1) - ug.id_base);
      named_bar_sync(1, kLoadThreads);
      const int id = (int)misc->unit;
      named_bar_sync(1, kLoadThreads);
      int b, g, c;
      if (!unit_decode(ug, id, b, g, c)) break;
      const int vmax = tile_vmax_b(ug, b, g);
      const int kbeg = c * ug.C;
      const int kend = min(kbeg + ug.C, vmax);
      for (int j0 = kbeg;; j0 += CS) {
        const int nk = max(0, min(CS, kend - j0));
        const int last = (j0 + CS >= kend) ? 1 : 0;
        const int slot = it & 1;
        const uint32_t ph = (it >> 1) & 1u;
        if (tid == 0) misc->go[slot] = mbar_wait(empty_bar + 8 * slot, ph ^ 1u, ctl) ? 1u : 0u;
        named_bar_sync(1, kLoadThreads);
        if (!misc->go[slot]) {
          more = false;
          break;
        }
        float* st = strip + (size_t)slot * QT * CS;
        for (int qi = 0; qi < QT; ++qi) {
          const int t = g * QT + qi;
          if (t >= sp.S) break;
          const int lim =
              min(nk, row_visible(sp.vis, b, sp.S, sp.t0, sp.tstride, t, sp.T, sp.m) - j0);
          const float* src = X + ((int64_t)b * sp.S + t) * sp.T + j0;
          for (int q = tid; q < lim; q += kLoadThreads) st[(size_t)qi * CS + q] = __ldg(src + q);
        }
        if (tid == 0) meta[slot] = StripMeta{1, b, g, c, j0, nk, last, 0u};
        mbar_arrive(full_bar + 8 * slot);
        ++it;
        if (last) break;
      }
    }
    // no more units: tell the selection warps to stop
    const int slot = it & 1;
    const uint32_t ph = (it >> 1) & 1u;
    if (tid == 0) misc->go[slot] = mbar_wait(empty_bar + 8 * slot, ph ^ 1u, ctl) ? 1u : 0u;
    named_bar_sync(1, kLoadThreads);
    if (misc->go[slot]) {
      if (tid == 0) meta[slot].valid = 0;
      mbar_arrive(full_bar + 8 * slot);
    }
  }
  __syncthreads();
}

size_t topk_scores_smem_bytes(int QT, int cap, int CS) {
  return sel_state_bytes(QT, cap) + sizeof(float) * 2 * QT * CS + sizeof(StripMeta) * 2 +
         sizeof(uint64_t) * 4 + sizeof(TopkScoresSmem) + 64;
}

cudaError_t launch_topk_scores(const float* X, const SelParams& sp, const UnitGrid& ug,
                               int* counter, uint32_t* err, uint64_t timeout_ns, int grid,
                               cudaStream_t stream) {
  const size_t smem = topk_scores_smem_bytes(sp.QT, sp.cap, sp.CS);
  cudaError_t e = cudaFuncSetAttribute(k_topk_scores, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)smem);
  if (e != cudaSuccess) return e;
  k_topk_scores<<<grid, kTopkThreads, smem, stream>>>(X, sp, ug, counter, err, timeout_ns);
  return cudaGetLastError();
}

}  // namespace si
