// Streaming per-query top-k selection, shared by the score kernel (scores
// arrive from the tensor-core epilogue) and the selection-only kernel (scores
// arrive from global memory).
//
// "StreamIndex: Memory-Bounded Compressed Sparse Attention via Streaming
// Top-k", Abstract: the top-k keys are selected per query by a chunked
// partition-merge driver that never holds the full score tensor.  Here each
// query owns a running list of its best K keys so far (sorted, 64-bit keys
// from si_common.cuh, 0 = empty) in shared memory.  Scores are consumed in
// strips of up to CS keys: a key enters a warp-private candidate buffer only if
// it beats the list's current K-th entry; full buffers are bitonic-sorted by
// the warp and merged into the list in place (merge path, back to front).  A
// unit (a tile of QT queries x one key chunk) ends by writing each list out,
// either as the final answer or as a partial list for the merge kernel.
#pragma once

#include "si_common.cuh"

namespace si {

constexpr int kSelWarps = 4;    // selection warps per CTA
constexpr int kCandCap = 256;   // candidate buffer entries per selection warp
constexpr int kMergeR = 8;      // outputs per lane per merge phase

// What a filled strip slot carries from its producer to the selection warps.
struct StripMeta {
  int valid;   // 0: no more work, selection warps exit
  int b, g, c; // batch, query tile, key chunk of the unit
  int j0;      // first key of the strip
  int nkeys;   // keys in the strip (<= CS)
  int last;    // 1 if this is the unit's last strip
  int direct;  // 1: the unit covers every visible key, write the final answer
};

struct SelParams {
  int B, S, T, m, K, QT, CS;
  int g_lo, n_tiles;   // query tiles [g_lo, g_lo + n_tiles) in this launch
  int nch_max;         // chunk slots per query tile in the partial scratch
  int32_t* out_idx;    // [B,S,K]
  float* out_score;    // [B,S,K]
  uint64_t* partial;   // [B, n_tiles, nch_max, QT, K] sorted keys
};

struct SelSmem {
  uint64_t* lists;     // [QT][K]
  uint64_t* cand;      // [kSelWarps][kCandCap]
  float* strip;        // [2][QT][CS]
  StripMeta* meta;     // [2]
  uint32_t full_bar;   // 2 mbarriers, 8 bytes apart
  uint32_t empty_bar;  // 2 mbarriers, 8 bytes apart
};

SI_DEV int visible_keys(int t, int T, int m) {
  int v = (t + 1) / m;
  return v < T ? v : T;
}

// Bitonic sort of a[0, n2) into descending order by one warp (n2 a power of 2).
SI_DEV void warp_sort_desc(uint64_t* a, int n2, int lane) {
  for (int size = 2; size <= n2; size <<= 1) {
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      for (int i = lane; i < (n2 >> 1); i += 32) {
        const int lo = ((i & ~(stride - 1)) << 1) | (i & (stride - 1));
        const int hi = lo + stride;
        const bool up = (lo & size) == 0;
        const uint64_t x = a[lo], y = a[hi];
        if ((x < y) == up) {
          a[lo] = y;
          a[hi] = x;
        }
      }
      __syncwarp();
    }
  }
}

// L[0, K) sorted descending; C[0, n) sorted descending, n >= 1, all keys
// distinct.  Replaces L by the K largest keys of L and C, in place.
// Positions before the first one C[0] would take are unchanged.  The rest is
// rebuilt by merge path in phases from the back: a phase reads only list
// entries at or below its own output range, and no later phase reads that
// range, so staging each phase's outputs in registers makes it safe in place.
SI_DEV void warp_merge_into(uint64_t* L, int K, const uint64_t* C, int n, int lane) {
  const uint64_t c0 = C[0];
  int lo = 0, hi = K;
  while (lo < hi) {
    const int mid = (lo + hi) >> 1;
    if (L[mid] > c0) lo = mid + 1;
    else hi = mid;
  }
  const int f = lo;
  if (f >= K) return;
  uint64_t* A = L + f;
  const int na = K - f;  // also the number of outputs rebuilt
  constexpr int P = 32 * kMergeR;
  for (int ph = (na + P - 1) / P - 1; ph >= 0; --ph) {
    const int d = ph * P + lane * kMergeR;
    uint64_t v[kMergeR];
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
      for (int r = 0; r < kMergeR; ++r) {
        if (d + r < na) {
          const bool take_a = (ib >= n) || (ia < na && A[ia] > C[ib]);
          v[r] = take_a ? A[ia] : C[ib];
          ia += take_a ? 1 : 0;
          ib += take_a ? 0 : 1;
        }
      }
    }
    __syncwarp();
    if (d < na) {
#pragma unroll
      for (int r = 0; r < kMergeR; ++r)
        if (d + r < na) A[d + r] = v[r];
    }
    __syncwarp();
  }
}

SI_DEV void warp_flush(uint64_t* L, int K, uint64_t* cb, int n, int lane) {
  __syncwarp();
  int n2 = 2;
  while (n2 < n) n2 <<= 1;
  for (int i = n + lane; i < n2; i += 32) cb[i] = 0ull;
  __syncwarp();
  warp_sort_desc(cb, n2, lane);
  warp_merge_into(L, K, cb, n, lane);
  __syncwarp();
}

// Consume one strip of scores for one query: keys j0 + p, p < nkeys; only
// keys j < V are visible.
SI_DEV void warp_take_strip(const float* st, int j0, int nkeys, int V, uint64_t* L, int K,
                            uint64_t* cb, int lane) {
  int lim = V - j0;
  if (lim > nkeys) lim = nkeys;
  if (lim <= 0) return;
  uint64_t theta = L[K - 1];
  int nc = 0;
  const uint32_t lt_mask = (1u << lane) - 1u;
  for (int p0 = 0; p0 < lim; p0 += 32) {
    const int p = p0 + lane;
    uint64_t key = 0ull;
    bool take = false;
    if (p < lim) {
      key = make_key(st[p], j0 + p);
      take = key > theta;
    }
    uint32_t mask = __ballot_sync(0xFFFFFFFFu, take);
    if (mask == 0u) continue;
    int cnt = __popc(mask);
    if (nc + cnt > kCandCap) {
      warp_flush(L, K, cb, nc, lane);
      nc = 0;
      theta = L[K - 1];
      take = take && key > theta;
      mask = __ballot_sync(0xFFFFFFFFu, take);
      cnt = __popc(mask);
    }
    if (take) cb[nc + __popc(mask & lt_mask)] = key;
    nc += cnt;
  }
  if (nc > 0) warp_flush(L, K, cb, nc, lane);
}

// Write one query's list out and clear it for the next unit.
SI_DEV void warp_emit(const SelParams& p, const StripMeta& md, int qi, uint64_t* L, int lane) {
  const int t = md.g * p.QT + qi;
  if (md.direct) {
    const int64_t base = ((int64_t)md.b * p.S + t) * p.K;
    for (int r = lane; r < p.K; r += 32) {
      const uint64_t k = L[r];
      p.out_idx[base + r] = k ? key_index(k) : -1;
      p.out_score[base + r] = k ? key_score(k) : __int_as_float(0xFF800000);
      L[r] = 0ull;
    }
  } else {
    const int64_t slot =
        (((int64_t)md.b * p.n_tiles + (md.g - p.g_lo)) * p.nch_max + md.c) * p.QT + qi;
    uint64_t* dst = p.partial + slot * p.K;
    for (int r = lane; r < p.K; r += 32) {
      dst[r] = L[r];
      L[r] = 0ull;
    }
  }
  __syncwarp();
}

// The selection warps' loop: take filled strips in order until a strip says
// there is no more work (or the CTA aborts).
SI_DEV void select_loop(const SelParams& p, const SelSmem& sm, const Ctl& ctl, int sw, int lane) {
  uint64_t* cb = sm.cand + sw * kCandCap;
  for (uint32_t it = 0;; ++it) {
    const int slot = it & 1;
    const uint32_t ph = (it >> 1) & 1u;
    if (!mbar_wait_warp(sm.full_bar + 8 * slot, ph, ctl)) return;
    const StripMeta md = sm.meta[slot];  // ordered after the acquiring wait
    if (!md.valid) return;
    const float* st = sm.strip + (size_t)slot * p.QT * p.CS;
    for (int qi = sw; qi < p.QT; qi += kSelWarps) {
      const int t = md.g * p.QT + qi;
      if (t >= p.S) continue;
      uint64_t* L = sm.lists + (size_t)qi * p.K;
      warp_take_strip(st + (size_t)qi * p.CS, md.j0, md.nkeys, visible_keys(t, p.T, p.m), L, p.K,
                      cb, lane);
      if (md.last) warp_emit(p, md, qi, L, lane);
    }
    __syncwarp();
    mbar_arrive(sm.empty_bar + 8 * slot);
  }
}

// ------------------------------------------------------------------ units
// A launch covers query tiles [g_lo, g_lo + n_tiles) of every batch.  Key
// chunk c of tile g holds keys [c*C, min((c+1)*C, Vmax(g))), where Vmax(g) is
// the visible count of the tile's last query.  Units are numbered chunk-major;
// inside a chunk, tiles run from the largest (most keys) down, batch fastest.
struct UnitGrid {
  int B, S, T, m, QT, C, g_lo, n_tiles;
  int id_base;  // value of the shared unit counter when this launch starts
};

SI_DEV int tile_vmax(const UnitGrid& u, int g) {
  int t = g * u.QT + u.QT - 1;
  if (t > u.S - 1) t = u.S - 1;
  return visible_keys(t, u.T, u.m);
}

// Number of chunks of tile g (at least 1, so tiles with no visible key still
// emit their padding).
SI_DEV int tile_chunks(const UnitGrid& u, int g) {
  const int v = tile_vmax(u, g);
  return v <= 0 ? 1 : (v + u.C - 1) / u.C;
}

// Decode unit id -> (b, g, c); returns false past the end.
SI_DEV bool unit_decode(const UnitGrid& u, int id, int& b, int& g, int& c) {
  if (id < 0) return false;
  const int g_hi = u.g_lo + u.n_tiles;  // exclusive
  for (int cc = 0;; ++cc) {
    // tiles with more than cc chunks form a suffix [g_first, g_hi)
    int lo = u.g_lo, hi = g_hi;
    while (lo < hi) {
      const int mid = (lo + hi) >> 1;
      if (tile_chunks(u, mid) > cc) hi = mid;
      else lo = mid + 1;
    }
    const int cnt = (g_hi - lo) * u.B;
    if (cnt == 0) return false;
    if (id < cnt) {
      g = g_hi - 1 - id / u.B;
      b = id % u.B;
      c = cc;
      return true;
    }
    id -= cnt;
  }
}

}  // namespace si
