// Exact, sorted top-k rows from a query's few candidate lists (one per key
// chunk; a single list when one chunk spans all of the query's keys).
//
// "StreamIndex: Memory-Bounded Compressed Sparse Attention via Streaming
// Top-k", Abstract: the top-k keys are selected per query by a chunked
// partition-merge driver.  The fused kernel leaves per query and key chunk
// one pruned list of at most L candidate keys (a superset of that chunk's K
// best, zero-padded); when a query's lists together hold at most
// kFinishMaxKeys keys, this kernel turns them into the output row in one
// pass (longer sets go to the merge kernel).
//
// One CTA per query, a bucket (counting) sort instead of a comparison
// network.  The candidates' 32-bit score images (the high word of the
// selection keys of si_common.cuh) are mapped monotonically onto NB buckets
// spanning [min, max]: bucket(k) never decreases when the key grows.  A
// histogram (shared-memory atomics), an in-place suffix sum and a scatter
// group the candidates by bucket, highest bucket first; a candidate's final
// position is then its bucket's start plus the number of larger keys in its
// own bucket, counted by direct comparison of the full 64-bit keys (so ties
// in score are ordered by index exactly as the selection orders them).  Only
// buckets that start below K are ranked.  Buckets are small for any spread
// of scores; when one holds more than kMaxBucket keys (many equal scores),
// the row takes the radix select and a shared-memory bitonic sort instead
// (one warp).
#include <algorithm>

#include "si_kernels.h"

namespace si {

constexpr int kMaxBucket = 64;  // larger buckets take the comparison-sort fallback

SI_DEV uint32_t key_ord(uint64_t k) { return (uint32_t)(k >> 32); }

// The score behind an order image (a zero score comes back as +0).
SI_DEV float ord_score(uint32_t o) {
  return __uint_as_float((o & 0x80000000u) ? (o & 0x7FFFFFFFu) : ~o);
}

// Monotone bucket of a score: floor((s - smin) * scale), clamped to [0, nb).
// Subtracting a constant, multiplying by a positive constant (both rounded)
// and truncating never decrease, so neither does the bucket; the buckets are
// linear in the score, so a row's candidates spread over them whatever the
// sign of its scores.  scale == 0 (an infinite or degenerate range) puts
// every key in bucket 0.
SI_DEV int bucket_of(uint32_t ord, float smin, float scale, int nb) {
  if (scale == 0.0f) return 0;
  const int b = (int)((ord_score(ord) - smin) * scale);
  return b < nb - 1 ? b : nb - 1;
}

// Descending bitonic sort of n2 (a power of two) keys in shared memory by one
// warp; used only for rows whose scores tie heavily.
SI_DEV void smem_bitonic_desc(uint64_t* a, int n2, int lane) {
  for (int size = 2; size <= n2; size <<= 1) {
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      for (int i = lane; i < n2 / 2; i += 32) {
        const int lo = 2 * stride * (i / stride) + (i % stride);
        const int hi = lo + stride;
        const bool desc = (lo & size) == 0;
        const uint64_t x = a[lo], y = a[hi];
        if (desc ? (x < y) : (x > y)) {
          a[lo] = y;
          a[hi] = x;
        }
      }
      __syncwarp();
    }
  }
}

struct FinishRed {
  uint32_t n[32], omin[32], omax[32], tot[32], mx[32];
};

// One CTA per query.  Shared memory: raw[nl*L] (the query's nl lists as
// read, one after another), tmp[cap] (bucket-ordered candidates), bins[nb]
// (counts, then bucket starts, then bucket ends), and a small block for
// cross-warp reductions.  Only the lists the fused kernel wrote for the
// query's tile are read: its tile_chunks(), each L keys (L / 2 16-byte words).
__global__ void __launch_bounds__(256)
    k_finish_rows(const uint64_t* __restrict__ partial, SelParams sp, UnitGrid ug, int raw_cap,
                  int tmp_cap, int nb) {
  extern __shared__ __align__(16) uint8_t smem[];
  const int tid = threadIdx.x, nthr = blockDim.x, warp = tid >> 5, lane = tid & 31;
  const int nw = nthr >> 5;
  const int K = sp.K, QT = sp.QT;
  uint64_t* raw = reinterpret_cast<uint64_t*>(smem);
  uint64_t* tmp = raw + raw_cap;
  uint32_t* bins = reinterpret_cast<uint32_t*>(tmp + tmp_cap);
  uint16_t* rawb = reinterpret_cast<uint16_t*>(bins + nb);  // bucket of raw[i]
  uint16_t* tmpb = rawb + raw_cap;                          // bucket of tmp[i]
  FinishRed* red = reinterpret_cast<FinishRed*>(tmpb + tmp_cap);
  const uint32_t qid = blockIdx.x;  // < B*S < 2^31
  const uint32_t tq = qid / (uint32_t)QT;
  const int qi = (int)(qid - tq * (uint32_t)QT);
  const int b = (int)(tq / (uint32_t)sp.n_tiles);
  const int gl = (int)(tq - (uint32_t)b * (uint32_t)sp.n_tiles);
  const int t = (sp.g_lo + gl) * QT + qi;
  if (t >= sp.S) return;
  const int nl = sp.nch_max == 1 ? 1 : min(tile_chunks(ug, sp.g_lo + gl), sp.nch_max);
  const int L = nl * sp.L;  // candidates read (nl lists), at most raw_cap
  if (L > raw_cap) return;  // the host sizes raw_cap for every tile; never taken
  // list c of the query: partial[b][gl][c][qi][0 .. sp.L)
  const uint64_t* src = partial + (((int64_t)b * sp.n_tiles + gl) * sp.nch_max * QT + qi) * sp.L;
  const int64_t list_stride4 = (int64_t)QT * sp.L / 2;  // 16-byte words between lists
  const int l4 = sp.L / 2;                                // 16-byte words of one list
  int32_t* oi = sp.out_idx + ((int64_t)b * sp.S + t) * K;
  float* os = sp.out_score + ((int64_t)b * sp.S + t) * K;

  // pass 1: the lists into shared memory (16-byte loads, all issued before
  // any is used), the count of real candidates (non-zero keys) and the range
  // of their score images
  uint32_t n = 0, omin = 0xFFFFFFFFu, omax = 0u;
  {
    const uint4* s4 = reinterpret_cast<const uint4*>(src);  // sp.L is a multiple of 32
    uint4* r4 = reinterpret_cast<uint4*>(raw);
    const int n4 = L / 2;
    for (int i0 = 0; i0 < n4; i0 += 4 * nthr) {
      uint4 v[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int i = i0 + u * nthr + tid;
        const int c = i / l4;
        v[u] = i < n4 ? __ldg(s4 + c * list_stride4 + (i - c * l4)) : make_uint4(0u, 0u, 0u, 0u);
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int i = i0 + u * nthr + tid;
        if (i < n4) r4[i] = v[u];
        // keys: (x | y<<32) and (z | w<<32); a key is real iff non-zero
        if (v[u].x | v[u].y) {
          ++n;
          omin = min(omin, v[u].y);
          omax = max(omax, v[u].y);
        }
        if (v[u].z | v[u].w) {
          ++n;
          omin = min(omin, v[u].w);
          omax = max(omax, v[u].w);
        }
      }
    }
  }
  n = __reduce_add_sync(0xFFFFFFFFu, n);
  omin = __reduce_min_sync(0xFFFFFFFFu, omin);
  omax = __reduce_max_sync(0xFFFFFFFFu, omax);
  if (lane == 0) {
    red->n[warp] = n;
    red->omin[warp] = omin;
    red->omax[warp] = omax;
  }
  for (int i = tid; i < nb / 4; i += nthr) reinterpret_cast<uint4*>(bins)[i] = make_uint4(0u, 0u, 0u, 0u);
  __syncthreads();
  n = 0;
  omin = 0xFFFFFFFFu;
  omax = 0u;
  for (int w = 0; w < nw; ++w) {
    n += red->n[w];
    omin = min(omin, red->omin[w]);
    omax = max(omax, red->omax[w]);
  }
  const int nreal = (int)n;
  const int nout = nreal < K ? nreal : K;
  const float smin = ord_score(omin);
  float scale = omax > omin ? (float)(nb - 1) / (ord_score(omax) - smin) : 0.0f;
  if (!(scale <= 3.0e38f)) scale = 0.0f;  // infinite range (0) or a tiny one (inf)
  bool fallback = (nreal > 1 && omax == omin);
  if (nreal > 1 && !fallback) {
    // pass 2: histogram (each key's bucket kept for the scatter)
    for (int i = tid; i < L; i += nthr) {
      const uint64_t k = raw[i];
      if (k) {
        const int bk = bucket_of(key_ord(k), smin, scale, nb);
        rawb[i] = (uint16_t)bk;
        atomicAdd(&bins[bk], 1u);
      }
    }
    __syncthreads();
    // exclusive suffix sum in place: bins[b] = keys in buckets above b.  Warp
    // w owns the C = nb/nw buckets [w*C, w*C + C), read in rows of 128: lane l
    // holds buckets 4l..4l+3 of the row (16-byte accesses, no bank conflicts);
    // higher warps hold higher buckets.
    const int C = nb / nw;
    uint4* wb = reinterpret_cast<uint4*>(bins + warp * C);
    uint32_t tot = 0, mx = 0;
    for (int i = lane; i < C / 4; i += 32) {
      const uint4 c = wb[i];
      tot += c.x + c.y + c.z + c.w;
      mx = max(mx, max(max(c.x, c.y), max(c.z, c.w)));
    }
    tot = __reduce_add_sync(0xFFFFFFFFu, tot);
    mx = __reduce_max_sync(0xFFFFFFFFu, mx);
    if (lane == 0) {
      red->tot[warp] = tot;
      red->mx[warp] = mx;
    }
    __syncthreads();
    uint32_t carry = 0;  // keys in the buckets above the current row
    mx = 0;
    for (int w = 0; w < nw; ++w) {
      if (w > warp) carry += red->tot[w];
      mx = max(mx, red->mx[w]);
    }
    if (mx > (uint32_t)kMaxBucket) {
      fallback = true;
    } else {
      for (int r0 = C / 4 - 32; r0 >= 0; r0 -= 32) {
        const uint4 c = wb[r0 + lane];
        const uint32_t own = c.x + c.y + c.z + c.w;
        uint32_t suf = own;  // keys in this row's buckets from this lane's first up
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const uint32_t y = __shfl_down_sync(0xFFFFFFFFu, suf, o);
          if (lane + o < 32) suf += y;
        }
        const uint32_t base = carry + suf - own;  // above this lane's four buckets
        wb[r0 + lane] = make_uint4(base + c.y + c.z + c.w, base + c.z + c.w, base + c.w, base);
        carry += __shfl_sync(0xFFFFFFFFu, suf, 0);
      }
      __syncthreads();
      // pass 3: scatter by bucket (bins[] becomes each bucket's end)
      for (int i = tid; i < L; i += nthr) {
        const uint64_t k = raw[i];
        if (k) {
          const int bk = rawb[i];
          const uint32_t pos = atomicAdd(&bins[bk], 1u);
          tmp[pos] = k;
          tmpb[pos] = (uint16_t)bk;
        }
      }
      __syncthreads();
      // pass 4: exact position = bucket start + larger keys in the bucket
      for (int p = tid; p < nreal; p += nthr) {
        const uint64_t k = tmp[p];
        const int bk = tmpb[p];
        const int s = bk == nb - 1 ? 0 : (int)bins[bk + 1];
        if (s >= K) continue;
        const int e = (int)bins[bk];
        int r = s;
        for (int x = s; x < e; ++x) r += tmp[x] > k ? 1 : 0;
        if (r < K) {
          oi[r] = key_index(k);
          os[r] = key_score(k);
        }
      }
    }
  } else if (nreal == 1) {
    for (int i = tid; i < L; i += nthr) {
      const uint64_t k = raw[i];
      if (k) {
        oi[0] = key_index(k);
        os[0] = key_score(k);
      }
    }
  }
  if (fallback && warp == 0) {
    // many equal scores: gather, exact K best by radix select, then sort
    const uint32_t lt_mask = (1u << lane) - 1u;
    int w = 0;
    for (int i0 = 0; i0 < L; i0 += 32) {
      const int i = i0 + lane;
      const uint64_t k = i < L ? raw[i] : 0ull;
      const uint32_t mk = __ballot_sync(0xFFFFFFFFu, k != 0ull);
      if (k) tmp[w + __popc(mk & lt_mask)] = k;
      w += __popc(mk);
    }
    __syncwarp();
    int m = nreal;
    if (m > K) {
      pool_shrink(tmp, m, K, bins, lane);
      m = K;
    }
    const int n2 = pow2ceil(m);
    for (int i = m + lane; i < n2; i += 32) tmp[i] = 0ull;
    __syncwarp();
    smem_bitonic_desc(tmp, n2, lane);
    for (int r = lane; r < m; r += 32) {
      oi[r] = key_index(tmp[r]);
      os[r] = key_score(tmp[r]);
    }
  }
  // padding after the real entries
  for (int r = nout + tid; r < K; r += nthr) {
    oi[r] = -1;
    os[r] = __int_as_float(0xFF800000);
  }
}

// Launch shape: a CTA per query, 128 threads for short lists and 256 for
// long ones; buckets: twice the candidate count rounded up to a power of
// two, within [1024, 8192], so that the crowded buckets near the K-th score
// stay short; room for the gathered candidates: all of them, and a power of
// two at least K for the fallback sort.
struct FinishShape {
  int threads, nb, raw_cap, tmp_cap;
  size_t smem;
};

static FinishShape finish_shape(int K, int L, int nch) {
  FinishShape f;
  f.raw_cap = L * nch;
  f.threads = f.raw_cap > 1024 ? 256 : 128;
  f.nb = std::min(8192, std::max(1024, 2 * (int)pow2ceil(f.raw_cap)));
  f.tmp_cap = std::max(f.raw_cap, (int)pow2ceil(K));
  f.smem = (sizeof(uint64_t) + sizeof(uint16_t)) * ((size_t)f.raw_cap + f.tmp_cap) +
           sizeof(uint32_t) * f.nb + sizeof(FinishRed) + 16;
  return f;
}

// One list always; two (a decode step's chunks) when they fit.  More lists go
// to the merge kernel: a CTA per query costs more than a warp per query once
// the lists are long and the queries many (S = 32,768, eight chunks of 1,024
// keys, top-512: 1.8 ms here against 0.4 ms in the merge kernel).
bool finish_takes(int L, int nch) { return nch <= 2 && (int64_t)L * nch <= kFinishMaxKeys; }

cudaError_t launch_finish_rows(const uint64_t* partial, const SelParams& sp, const UnitGrid& ug,
                               cudaStream_t stream) {
  if (!finish_takes(sp.L, sp.nch_max)) return cudaErrorInvalidValue;
  const FinishShape f = finish_shape(sp.K, sp.L, sp.nch_max);
  cudaError_t e = cudaFuncSetAttribute(k_finish_rows, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)f.smem);
  if (e != cudaSuccess) return e;
  const int64_t queries = (int64_t)sp.B * sp.n_tiles * sp.QT;
  k_finish_rows<<<(unsigned)queries, f.threads, f.smem, stream>>>(partial, sp, ug, f.raw_cap,
                                                                   f.tmp_cap, f.nb);
  return cudaGetLastError();
}

}  // namespace si
