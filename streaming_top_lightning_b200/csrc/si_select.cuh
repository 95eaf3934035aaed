// Streaming per-query top-k selection, shared by the score kernel (scores
// arrive from the tensor-core epilogue) and the selection-only kernel (scores
// arrive from global memory).
//
// "StreamIndex: Memory-Bounded Compressed Sparse Attention via Streaming
// Top-k", Abstract: the top-k keys are selected per query by a chunked
// partition-merge driver that never holds the full score tensor.  Here each
// query owns an unsorted candidate pool (64-bit keys from si_common.cuh) in
// shared memory and a threshold theta, the K-th best key seen so far (0 until
// K keys have been seen).  Scores arrive in strips of up to CS keys; a key
// enters the pool only if it beats theta.  When the pool is full, a warp radix
// select finds the exact K-th largest pool key, which becomes theta, and the
// pool is compacted to the K keys at or above it.  A unit (a tile of QT
// queries x one key chunk) ends by pruning its pool to at most L candidates,
// written to scratch as the unit's partial list.  With one key chunk the
// bucket-sort kernel (k_finish.cu) turns each list into the sorted row; with
// several, the merge kernel (k_merge.cu) takes the exact top K over a query's
// lists and the row sort (k_sort_rows.cu) orders rows longer than 512.
// Every pass reads the pool with consecutive lanes on consecutive keys, so no
// access has bank conflicts.
#pragma once

#include "si_common.cuh"

namespace si {

constexpr int kSelWarps = 4;  // selection warps per CTA

// What a filled strip slot carries from its producer to the selection warps.
struct StripMeta {
  int valid;   // 0: no more work, selection warps exit
  int b, g, c; // batch, query tile, key chunk of the unit
  int j0;      // first key of the strip
  int nkeys;   // keys in the strip (<= CS)
  int last;    // 1 if this is the unit's last strip
  uint32_t seq;  // the producer's running unit number
};

struct SelParams {
  int B, S, T, m, K, QT, CS;
  int cap;             // pool entries per query (>= K + 64)
  int L;               // length of a partial list (> K), see partial_len()
  int g_lo, n_tiles;   // query tiles [g_lo, g_lo + n_tiles) in this launch
  int nch_max;         // chunk slots per query tile in the partial scratch
  int32_t* out_idx;    // [B,S,K]
  float* out_score;    // [B,S,K]
  uint64_t* partial;   // [B, n_tiles, nch_max, QT, L] candidate keys, 0-padded
  int final_rows;      // 1: every tile is one unit, whose pools are final: the selection
                       // warps write the exact top-K rows themselves (no partial lists)
  int t0;              // sequence position of query row 0 (0 for a whole prefill)
  int tstride;         // positions of consecutive query rows differ by this (1 but in a
                       // group-representative scan)
  const int* vis;      // [B*S] visible keys of each query row, replacing the position
                       // rule when set (non-decreasing along a batch's rows)
};

// A unit leaves at most this many candidates per query (a superset of its K
// best): enough slack above K that pruning rarely has to fall back to the
// exact select.
__host__ __device__ constexpr int partial_len(int K) { return ((K + K / 4 + 64 + 31) / 32) * 32; }

struct SelSmem {
  uint64_t* pool;      // [QT][cap] candidate keys
  uint64_t* theta;     // [QT] current threshold
  int* npool;          // [QT] keys in each pool
  uint32_t* hist;      // [kSelWarps][8][32] digit counters of each selection warp
  float* strip;        // [nslot][QT][CS] scores
  StripMeta* meta;     // [nslot]
  uint32_t full_bar;   // nslot mbarriers, 8 bytes apart
  uint32_t empty_bar;  // nslot mbarriers, 8 bytes apart
  int nslot;           // strip slots in the ring (2..8)
};

SI_DEV int visible_keys(int t, int T, int m) {
  int v = (t + 1) / m;
  return v < T ? v : T;
}

// Keys query row t of batch b sees: the given count, or min(T, (pos+1)/m) at
// its position pos = t0 + t*tstride.
SI_DEV int row_visible(const int* vis, int b, int S, int t0, int tstride, int t, int T, int m) {
  if (vis) return vis[(int64_t)b * S + t];
  return visible_keys(t0 + t * tstride, T, m);
}

__host__ __device__ constexpr int pow2ceil(int x) {
  int p = 1;
  while (p < x) p <<= 1;
  return p;
}

// ------------------------------------------------------------------ radix select
// Compacts pool[0, np) (np > K, distinct keys) in place to its K largest keys
// and returns the smallest of them.  MSD radix select on 5-bit digits,
// starting at the highest bit where the pool keys differ.  Each lane counts
// the digits of its own keys (every 32nd key) in eight registers of four byte
// counters (digit d in byte d%4 of register d/4), with predicated adds and no
// memory traffic; the counters then go to shared memory as hist[d/4][lane],
// one transposed pass sums lane v's digit v over all lanes, and a suffix sum
// across lanes names the digit bucket that holds the K-th largest key.  It
// stops once a whole bucket is taken; one last pass keeps every key whose
// high bits reach the prefix.  hist: this warp's 8 x 32 words.
// Requires np <= 255 * 32 (byte counters).
static __device__ __noinline__ uint64_t pool_shrink(uint64_t* pool, int np, int K, uint32_t* hist,
                                             int lane) {
  uint64_t all_and = ~0ull, any_or = 0ull;
  {
    int i = lane;
    for (; i + 96 < np; i += 128) {
      const uint64_t k0 = pool[i], k1 = pool[i + 32], k2 = pool[i + 64], k3 = pool[i + 96];
      all_and &= k0 & k1 & k2 & k3;
      any_or |= k0 | k1 | k2 | k3;
    }
    for (; i < np; i += 32) {
      const uint64_t k = pool[i];
      all_and &= k;
      any_or |= k;
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    all_and &= __shfl_xor_sync(0xFFFFFFFFu, all_and, o);
    any_or |= __shfl_xor_sync(0xFFFFFFFFu, any_or, o);
  }
  const uint64_t diff = all_and ^ any_or;  // nonzero: keys are distinct, np >= 2
  int top = 63 - __clzll((long long)diff);
  // bits above `top` are common to every key; there are none when top is 63
  uint64_t prefix = (top >= 63) ? 0ull : (all_and & ~((2ull << top) - 1ull));
  uint32_t need = (uint32_t)K;
  int lo_bit = 0;
  for (;;) {
    const int width = top + 1 < 5 ? top + 1 : 5;
    lo_bit = top - width + 1;
    const uint64_t hi_mask = (top >= 63) ? 0ull : ~((2ull << top) - 1ull);
    const uint32_t dmask = (1u << width) - 1u;
    uint32_t c[8] = {0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u};
    for (int i = lane; i < np; i += 32) {
      const uint64_t k = pool[i];
      const uint32_t d = (uint32_t)(k >> lo_bit) & dmask;
      const uint32_t inc = ((k & hi_mask) == prefix) ? (1u << ((d & 3u) * 8u)) : 0u;
      const uint32_t row = d >> 2;
#pragma unroll
      for (int r = 0; r < 8; ++r) c[r] += (row == (uint32_t)r) ? inc : 0u;
    }
#pragma unroll
    for (int r = 0; r < 8; ++r) hist[r * 32 + lane] = c[r];
    __syncwarp();
    uint32_t cnt = 0;
    if ((uint32_t)lane <= dmask) {
      const uint32_t* row = hist + (lane >> 2) * 32;
      const uint32_t sh = (lane & 3) * 8;
#pragma unroll 8
      for (int l = 0; l < 32; ++l) cnt += (row[(l + lane) & 31] >> sh) & 255u;
    }
    __syncwarp();
    uint32_t suf = cnt;  // keys with digit >= lane
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t y = __shfl_down_sync(0xFFFFFFFFu, suf, o);
      if (lane + o < 32) suf += y;
    }
    const uint32_t above = suf - cnt;
    const uint32_t here = __ballot_sync(0xFFFFFFFFu, cnt > 0u && above < need && need <= suf);
    const int dstar = __ffs(here) - 1;
    const uint32_t a = __shfl_sync(0xFFFFFFFFu, above, dstar);
    const uint32_t cb = __shfl_sync(0xFFFFFFFFu, cnt, dstar);
    prefix |= (uint64_t)dstar << lo_bit;
    need -= a;
    if (cb == need || lo_bit == 0) break;
    top = lo_bit - 1;
  }
  const uint64_t pre_hi = prefix >> lo_bit;
  uint64_t mn = ~0ull;
  int w = 0;
  const uint32_t lt_mask = (1u << lane) - 1u;
  // in place, forward: a block's keys are all read before any is written, and
  // the write position w + rank never passes the read position
  for (int i0 = 0; i0 < np; i0 += 64) {
    const int i = i0 + lane;
    const uint64_t ka = i < np ? pool[i] : 0ull;
    const uint64_t kb = i + 32 < np ? pool[i + 32] : 0ull;
    const bool ta = i < np && (ka >> lo_bit) >= pre_hi;
    const bool tb = i + 32 < np && (kb >> lo_bit) >= pre_hi;
    const uint32_t ma = __ballot_sync(0xFFFFFFFFu, ta);
    const uint32_t mb = __ballot_sync(0xFFFFFFFFu, tb);
    if (ta) {
      pool[w + __popc(ma & lt_mask)] = ka;
      mn = ka < mn ? ka : mn;
    }
    w += __popc(ma);
    if (tb) {
      pool[w + __popc(mb & lt_mask)] = kb;
      mn = kb < mn ? kb : mn;
    }
    w += __popc(mb);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const uint64_t y = __shfl_xor_sync(0xFFFFFFFFu, mn, o);
    mn = y < mn ? y : mn;
  }
  __syncwarp();
  return mn;
}

// ------------------------------------------------------------------ pruning
// Cheap mid-stream shrink.  pool[0, np) holds np > K distinct keys.  Each
// lane samples one key (evenly spread over the pool, which is in arrival
// order), the warp sorts the 32 samples (bitonic, one key per lane, xor
// shuffles) and takes as pivot the sample whose rank predicts about
// target = K + K/8 + 32 pool keys at or above it.  The keys at or above the
// pivot are counted; if fewer than K, a lower sample is tried.  The pool is
// then compacted to the c >= K keys at or above the pivot, and the pivot
// becomes the new threshold: it is a pool key with at least K keys at or
// above it, so no key below it can be among the K best.  Returns false (pool
// unchanged) if even the lowest sample leaves fewer than K keys.
static __device__ __noinline__ bool pool_prune(uint64_t* pool, int* np_io, int K, uint64_t* theta_out,
                                        int lane) {
  const int np = *np_io;
  uint64_t v = pool[(int)(((long long)(2 * lane + 1) * np) >> 6)];
#pragma unroll
  for (int size = 2; size <= 32; size <<= 1) {
#pragma unroll
    for (int s = size >> 1; s > 0; s >>= 1) {
      const bool dir = (lane & size) == 0;  // lower lane keeps the max
      const bool lower = (lane & s) == 0;
      const uint64_t y = __shfl_xor_sync(0xFFFFFFFFu, v, s);
      const bool gt = v > y;
      v = ((lower == dir) == gt) ? v : y;
    }
  }
  // v is now the sample of rank `lane` (0 = largest)
  const long long target = (long long)K + K / 8 + 32;
  int r = (int)((32ll * target + np - 1) / np) - 1;
  if (r < 0) r = 0;
  for (; r < 32; r += 2) {
    const uint64_t pivot = __shfl_sync(0xFFFFFFFFu, v, r);
    // both passes take four 32-key groups per iteration, so their loads and
    // ballots overlap
    int c = 0;
    for (int i0 = 0; i0 < np; i0 += 128) {
      uint64_t k[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int i = i0 + 32 * u + lane;
        k[u] = i < np ? pool[i] : 0ull;
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) c += (i0 + 32 * u + lane < np && k[u] >= pivot) ? 1 : 0;
    }
    c = __reduce_add_sync(0xFFFFFFFFu, c);
    if (c >= K) {
      if (c >= np) return false;  // nothing to drop
      int w = 0;
      const uint32_t lt_mask = (1u << lane) - 1u;
      for (int i0 = 0; i0 < np; i0 += 128) {
        uint64_t k[4];
        uint32_t m[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int i = i0 + 32 * u + lane;
          k[u] = i < np ? pool[i] : 0ull;
        }
#pragma unroll
        for (int u = 0; u < 4; ++u)
          m[u] = __ballot_sync(0xFFFFFFFFu, i0 + 32 * u + lane < np && k[u] >= pivot);
        // forward, in place: the block's keys are all read before any is
        // written, and a write position never passes its read position
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          if (m[u] & (1u << lane)) pool[w + __popc(m[u] & lt_mask)] = k[u];
          w += __popc(m[u]);
        }
      }
      __syncwarp();
      *np_io = w;
      *theta_out = pivot;
      return true;
    }
  }
  return false;
}

// ------------------------------------------------------------------ strips
// Consume one strip of scores for one query: keys j0 + p, p < nkeys; only
// keys j < V are visible.  Keys whose score is at least theta's join the pool
// (only those can beat theta; the few extra keys of equal score are
// harmless); a full pool is pruned, which raises theta.
// The strip is taken in chunks of eight 64-key steps, lane l reading keys
// p0 + l and p0 + 32 + l of each step.  A chunk's loads, compares and ballots
// are all issued before any key is stored, and the steps' pool offsets are
// uniform prefix sums of the ballot counts, so the chunk's latencies overlap
// instead of chaining step after step.  When the pool cannot take the next
// step, the steps that fit are stored, the pool is pruned and the rest of the
// chunk is compared again with the new threshold.
SI_DEV void pool_take_strip(const float* st, int j0, int nkeys, int V, uint64_t* pool, int cap,
                            int K, int* np_p, uint64_t* th_p, uint32_t* hist, int lane,
                            const Ctl& ctl) {
  int lim = V - j0;
  if (lim > nkeys) lim = nkeys;
  if (lim <= 0) return;
  if (lane == 0) role_count(ctl, R_SEL_KEYS, (unsigned long long)lim);
  uint64_t theta = *th_p;
  int np = *np_p;
  // theta 0 takes every key (-inf >= -inf too)
  float thf = theta ? key_score(theta) : __int_as_float(0xFF800000);
  const uint32_t lt_mask = (1u << lane) - 1u;
  constexpr int kSteps = 8;
  for (int c0 = 0; c0 < lim; c0 += 64 * kSteps) {
    // slots past the visible keys read as NaN, which compares false with any
    // threshold (scores are never NaN), so the ballots need no range test
    const float nan = __int_as_float(0x7FC00000);
    float xa[kSteps], xb[kSteps];
#pragma unroll
    for (int u = 0; u < kSteps; ++u) {
      const int pa = c0 + 64 * u + lane;
      xa[u] = pa < lim ? st[pa] : nan;
      xb[u] = pa + 32 < lim ? st[pa + 32] : nan;
    }
    const int nsteps = min(kSteps, (lim - c0 + 63) >> 6);
    int s0 = 0;
    while (s0 < nsteps) {
      uint32_t ma[kSteps], mb[kSteps];
#pragma unroll
      for (int u = 0; u < kSteps; ++u) {
        ma[u] = __ballot_sync(0xFFFFFFFFu, u >= s0 && xa[u] >= thf);
        mb[u] = __ballot_sync(0xFFFFFFFFu, u >= s0 && xb[u] >= thf);
      }
      // the steps [s0, s1) that fit the pool
      int s1 = s0, add = 0;
#pragma unroll
      for (int u = 0; u < kSteps; ++u) {
        const int c = __popc(ma[u]) + __popc(mb[u]);
        if (u >= s0 && u == s1 && u < nsteps && np + add + c <= cap) {
          add += c;
          s1 = u + 1;
        }
      }
      int base = np;
#pragma unroll
      for (int u = 0; u < kSteps; ++u) {
        if (u >= s0 && u < s1) {
          const int pa = c0 + 64 * u + lane;
          const int na = __popc(ma[u]);
          if (ma[u] & (1u << lane)) pool[base + __popc(ma[u] & lt_mask)] = make_key(xa[u], j0 + pa);
          if (mb[u] & (1u << lane))
            pool[base + na + __popc(mb[u] & lt_mask)] = make_key(xb[u], j0 + pa + 32);
          base += na + __popc(mb[u]);
        }
      }
      np += add;
      if (lane == 0) role_count(ctl, R_SEL_APPENDS, (unsigned long long)add);
      s0 = s1;
      if (s0 < nsteps) {
        // the pool cannot take step s0: raise theta, then compare the rest again
        const long long t_p = role_t0();
        __syncwarp();
        if (lane == 0) role_count(ctl, R_SEL_PRUNES, 1);
        if (!pool_prune(pool, &np, K, &theta, lane) || np + 64 > cap) {
          if (lane == 0) role_count(ctl, R_SEL_SHRINKS, 1);
          theta = pool_shrink(pool, np, K, hist, lane);
          np = K;
        }
        thf = key_score(theta);
        if (lane == 0) role_add(ctl, R_SEL_PRUNE_CYC, t_p);
      }
    }
  }
  __syncwarp();
  if (lane == 0) {
    *np_p = np;
    *th_p = theta;
  }
  __syncwarp();
}

// End of a unit: prune the pool until it fits a partial list of L keys (a
// superset of the K best; the exact selection happens in the merge kernel).
// Returns the number of keys left in pool[0, n).
SI_DEV int pool_trim(uint64_t* pool, int np, int K, int L, uint32_t* hist, int lane) {
  __syncwarp();
  uint64_t th;
  while (np > L) {
    if (!pool_prune(pool, &np, K, &th, lane)) {
      pool_shrink(pool, np, K, hist, lane);
      np = K;
    }
  }
  __syncwarp();
  return np;
}

// Write one query's candidates out as its partial list for (tile, chunk).
SI_DEV void warp_emit(const SelParams& p, const StripMeta& md, int qi, const uint64_t* keys,
                      int n, int lane) {
  const int64_t slot =
      (((int64_t)md.b * p.n_tiles + (md.g - p.g_lo)) * p.nch_max + md.c) * p.QT + qi;
  uint64_t* dst = p.partial + slot * p.L;
  for (int r = lane; r < p.L; r += 32) dst[r] = r < n ? keys[r] : 0ull;
  __syncwarp();
}

// ------------------------------------------------------------------ row sort
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

// Sort the n (<= 32*R) keys in pool[0, n) and write the first K of them as an
// output row (index, score), padded with -1 / -inf.  The pool is unsorted, so
// reading it lane-interleaved (conflict-free) and treating that as the
// blocked layout loses nothing.
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

// Final output row from a pool that holds a superset of the row's K best keys
// (np of them): the exact K best (prune, then the radix select), sorted in
// registers for K <= 512; larger rows are written unsorted and ordered by the
// row-sort kernel afterwards.
static __device__ __noinline__ void finish_row(uint64_t* pool, int np, int K, uint32_t* hist,
                                               int32_t* oi, float* os, int lane) {
  __syncwarp();
  if (np > K) {
    uint64_t th;
    while (np > K + K / 4 + 64 && pool_prune(pool, &np, K, &th, lane)) {
    }
    if (np > K) pool_shrink(pool, np, K, hist, lane);
    np = K;
  }
  __syncwarp();
  switch (pow2ceil(K < 32 ? 32 : K)) {
    case 32: sort_and_write<1>(pool, np, K, oi, os, lane); break;
    case 64: sort_and_write<2>(pool, np, K, oi, os, lane); break;
    case 128: sort_and_write<4>(pool, np, K, oi, os, lane); break;
    case 256: sort_and_write<8>(pool, np, K, oi, os, lane); break;
    case 512: sort_and_write<16>(pool, np, K, oi, os, lane); break;
    default:
      for (int r = lane; r < K; r += 32) {
        const bool real = r < np;
        const uint64_t k = real ? pool[r] : 0ull;
        oi[r] = real ? key_index(k) : -1;
        os[r] = real ? key_score(k) : __int_as_float(0xFF800000);
      }
  }
  __syncwarp();
}

// True when finish_row() leaves the row sorted (else the row-sort kernel runs).
__host__ __device__ constexpr bool rows_sorted_in_warp(int K) { return K <= 512; }

// The selection warps' loop: take filled strips in order until a strip says
// there is no more work (or the CTA aborts).  Query qi belongs to selection
// warp qi % kSelWarps for the whole kernel, so its pool, threshold and count
// are only ever touched by that warp.  At a unit's last strip the warp either
// writes the exact output row itself (final_rows: the unit covers all of the
// query's keys) or leaves a pruned partial list for the merge kernel.
SI_DEV void select_loop(const SelParams& p, const SelSmem& sm, const Ctl& ctl, int sw, int lane) {
  uint32_t* hist = sm.hist + sw * 256;
  const long long t_role = role_t0();
  for (uint32_t it = 0;; ++it) {
    const int slot = (int)(it % (uint32_t)sm.nslot);
    const uint32_t ph = (it / (uint32_t)sm.nslot) & 1u;
    if (!mbar_wait_warp(sm.full_bar + 8 * slot, ph, ctl, R_SEL_WAIT_STRIP)) break;
    const StripMeta md = sm.meta[slot];  // ordered after the acquiring wait
    if (!md.valid) break;
    if (lane == 0) role_count(ctl, R_SEL_STRIPS, 1);
    const float* st = sm.strip + (size_t)slot * p.QT * p.CS;
    for (int qi = sw; qi < p.QT; qi += kSelWarps) {
      const int t = md.g * p.QT + qi;
      if (t >= p.S) continue;
      uint64_t* pool = sm.pool + (size_t)qi * p.cap;
      const long long t_in = role_t0();
      pool_take_strip(st + (size_t)qi * p.CS, md.j0, md.nkeys,
                      row_visible(p.vis, md.b, p.S, p.t0, p.tstride, t, p.T, p.m), pool, p.cap,
                      p.K, &sm.npool[qi], &sm.theta[qi], hist, lane, ctl);
      if (lane == 0) role_add(ctl, R_SEL_INTAKE, t_in);
      if (md.last) {
        const long long t_end = role_t0();
        if (p.final_rows) {
          const int64_t o = ((int64_t)md.b * p.S + t) * p.K;
          finish_row(pool, sm.npool[qi], p.K, hist, p.out_idx + o, p.out_score + o, lane);
        } else {
          const int n = pool_trim(pool, sm.npool[qi], p.K, p.L, hist, lane);
          warp_emit(p, md, qi, pool, n, lane);
        }
        if (lane == 0) {
          sm.npool[qi] = 0;
          sm.theta[qi] = 0ull;
          role_add(ctl, R_SEL_UNIT_END, t_end);
        }
        __syncwarp();
      }
    }
    __syncwarp();
    mbar_arrive(sm.empty_bar + 8 * slot);
  }
  if (lane == 0) role_add(ctl, R_SEL_TOTAL, t_role);
}

// Shared-memory bytes of the selection state for QT queries (pools,
// thresholds, counts, digit counters), 16-byte aligned.
__host__ __device__ constexpr size_t sel_state_bytes(int QT, int cap) {
  return ((sizeof(uint64_t) * (size_t)QT * cap + sizeof(uint64_t) * QT + sizeof(int) * QT +
           sizeof(uint32_t) * kSelWarps * 256) + 15) & ~(size_t)15;
}

// Carve the selection state out of shared memory at p (16-byte aligned).
SI_DEV void sel_state_carve(uint8_t* p, int QT, int cap, SelSmem& sm) {
  sm.pool = reinterpret_cast<uint64_t*>(p);
  sm.theta = sm.pool + (size_t)QT * cap;
  sm.npool = reinterpret_cast<int*>(sm.theta + QT);
  sm.hist = reinterpret_cast<uint32_t*>(sm.npool + QT);
}

// ------------------------------------------------------------------ units
// A launch covers query tiles [g_lo, g_lo + n_tiles) of every batch.  Key
// chunk c of tile g holds keys [c*C, min((c+1)*C, Vmax(g))), where Vmax(g) is
// the visible count of the tile's last query.  Units are numbered chunk-major;
// inside a chunk, tiles run from the largest (most keys) down, batch fastest.
// With tile_units, a unit is a whole tile (all its chunks, in order), tiles
// again from the largest down.
struct UnitGrid {
  int B, S, T, m, QT, C, g_lo, n_tiles;
  int id_base;     // value of the shared unit counter when this launch starts
  int tile_units;  // 1: a unit is a whole query tile, its key chunks handled in
                   // order inside it (the tile is loaded once); 0: one unit
                   // per (tile, chunk)
  int t0;          // sequence position of query row 0, the same in every batch
  int tstride;     // position step between query rows
  const int* vis;  // per-row visible counts (see SelParams::vis); tile units only
};

// Visible keys of tile g's last query (the tile's most), by the position rule.
SI_DEV int tile_vmax(const UnitGrid& u, int g) {
  int t = g * u.QT + u.QT - 1;
  if (t > u.S - 1) t = u.S - 1;
  return visible_keys(u.t0 + t * u.tstride, u.T, u.m);
}

// The same for batch b, from the per-row counts when given.
SI_DEV int tile_vmax_b(const UnitGrid& u, int b, int g) {
  if (!u.vis) return tile_vmax(u, g);
  int t = g * u.QT + u.QT - 1;
  if (t > u.S - 1) t = u.S - 1;
  return u.vis[(int64_t)b * u.S + t];
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
  if (u.tile_units) {
    if (id >= u.B * u.n_tiles) return false;
    g = g_hi - 1 - id / u.B;
    b = id % u.B;
    c = 0;
    return true;
  }
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
