// Query-group candidate scan: the helpers around the two indexer launches.
//
// The PIVOT news page (query-group indexing for DeepSeek sparse attention):
// nearby queries select nearly the same keys, so a group of queries can share
// one scan of the keys instead of one per query.  Reading used here: the
// queries of a batch form groups of G consecutive positions; the group's last
// position (it sees the most keys) scans all its visible keys with the fused
// indexer and keeps its C best; every query of the group then ranks only those
// candidates it can see, again with the fused indexer, now over a key set of C
// rows per group.  Between the two indexer launches:
//   k_pivot_reps   copies each group's last query row (q and w) into a
//                  compact [B, S/G] problem;
//   k_pivot_cands  sorts each group's candidates by key index, gathers their
//                  key rows into a [B*S/G, C] key set (zero rows past the
//                  candidates) and counts, for each query of the group, the
//                  candidates it can see (a prefix of the sorted list);
// and after the second launch
//   k_pivot_remap  maps each selected candidate position back to its key.
#include "si_kernels.h"

namespace si {

__global__ void __launch_bounds__(128)
    k_pivot_reps(const uint16_t* __restrict__ q, const float* __restrict__ w, PivotParams p,
                 uint16_t* __restrict__ qr, float* __restrict__ wr) {
  const int bg = blockIdx.x;  // b * ng + g
  const int b = bg / p.ng, g = bg - b * p.ng;
  const int64_t row = (int64_t)b * p.S + (int64_t)g * p.G + p.G - 1;
  const int n16 = p.H * p.D / 8;  // 16-byte words of a query row
  const uint4* src = reinterpret_cast<const uint4*>(q + row * p.H * p.D);
  uint4* dst = reinterpret_cast<uint4*>(qr + (int64_t)bg * p.H * p.D);
  for (int i = threadIdx.x; i < n16; i += blockDim.x) dst[i] = __ldg(src + i);
  for (int h = threadIdx.x; h < p.H; h += blockDim.x) wr[(int64_t)bg * p.H + h] = __ldg(w + row * p.H + h);
}

// One CTA per group: bitonic sort of the (at most 2048) candidate indices in
// shared memory, the sorted list, the gathered key rows and the per-query
// visible counts.
__global__ void __launch_bounds__(256)
    k_pivot_cands(const int32_t* __restrict__ rep_idx, const uint16_t* __restrict__ kc,
                  PivotParams p, int32_t* __restrict__ cand, uint16_t* __restrict__ kcg,
                  int* __restrict__ vis) {
  __shared__ int s[2048];
  __shared__ int nvalid;
  const int bg = blockIdx.x;
  const int b = bg / p.ng, g = bg - b * p.ng;
  const int tid = threadIdx.x;
  int n2 = 1;
  while (n2 < p.C) n2 <<= 1;
  if (tid == 0) nvalid = 0;
  __syncthreads();
  int cnt = 0;
  for (int i = tid; i < n2; i += blockDim.x) {
    const int j = i < p.C ? __ldg(rep_idx + (int64_t)bg * p.C + i) : -1;
    const bool ok = j >= 0 && j < p.T;
    s[i] = ok ? j : 0x7FFFFFFF;
    cnt += ok ? 1 : 0;
  }
  atomicAdd(&nvalid, cnt);
  __syncthreads();
  for (int size = 2; size <= n2; size <<= 1) {
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      for (int i = tid; i < n2 / 2; i += blockDim.x) {
        const int lo = 2 * stride * (i / stride) + (i % stride);
        const int hi = lo + stride;
        const bool up = (lo & size) == 0;
        const int x = s[lo], y = s[hi];
        if (up ? (x > y) : (x < y)) {
          s[lo] = y;
          s[hi] = x;
        }
      }
      __syncthreads();
    }
  }
  const int nv = nvalid;
  for (int i = tid; i < p.C; i += blockDim.x) cand[(int64_t)bg * p.C + i] = i < nv ? s[i] : -1;
  // key rows: 16-byte words, zero past the candidates
  const int w16 = p.D / 8;
  for (int e = tid; e < p.C * w16; e += blockDim.x) {
    const int c = e / w16, x = e - c * w16;
    uint4 v = make_uint4(0u, 0u, 0u, 0u);
    if (c < nv) v = __ldg(reinterpret_cast<const uint4*>(kc + ((int64_t)b * p.T + s[c]) * p.D) + x);
    reinterpret_cast<uint4*>(kcg + ((int64_t)bg * p.C + c) * p.D)[x] = v;
  }
  // query i of the group (position g*G + i) sees the candidates below its
  // visible count: the first lower_bound(V) of the sorted list
  for (int i = tid; i < p.G; i += blockDim.x) {
    const int t = g * p.G + i;
    int V = (t + 1) / p.m;
    if (V > p.T) V = p.T;
    int lo = 0, hi = nv;
    while (lo < hi) {
      const int mid = (lo + hi) >> 1;
      if (s[mid] < V) lo = mid + 1;
      else hi = mid;
    }
    vis[(int64_t)b * p.S + t] = lo;
  }
}

__global__ void k_pivot_remap(int32_t* __restrict__ out_idx, const int32_t* __restrict__ cand,
                              PivotParams p, int K) {
  const int64_t n = (int64_t)p.B * p.S * K;
  for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < n;
       e += (int64_t)gridDim.x * blockDim.x) {
    const int c = out_idx[e];
    if (c < 0) continue;
    const int64_t row = e / K;              // b*S + t
    const int64_t bg = row / p.G;           // b*ng + g  (S is a multiple of G)
    out_idx[e] = (c < p.C) ? __ldg(cand + bg * p.C + c) : -1;
  }
}

cudaError_t launch_pivot_reps(const uint16_t* q, const float* w, const PivotParams& p,
                              uint16_t* qr, float* wr, cudaStream_t stream) {
  k_pivot_reps<<<p.B * p.ng, 128, 0, stream>>>(q, w, p, qr, wr);
  return cudaGetLastError();
}

cudaError_t launch_pivot_cands(const int32_t* rep_idx, const uint16_t* kc, const PivotParams& p,
                               int32_t* cand, uint16_t* kcg, int* vis, cudaStream_t stream) {
  k_pivot_cands<<<p.B * p.ng, 256, 0, stream>>>(rep_idx, kc, p, cand, kcg, vis);
  return cudaGetLastError();
}

cudaError_t launch_pivot_remap(int32_t* out_idx, const int32_t* cand, const PivotParams& p, int K,
                               int sms, cudaStream_t stream) {
  const int64_t n = (int64_t)p.B * p.S * K;
  int64_t blocks = (n + 255) / 256;
  if (blocks > (int64_t)sms * 8) blocks = (int64_t)sms * 8;
  if (blocks < 1) blocks = 1;
  k_pivot_remap<<<(unsigned)blocks, 256, 0, stream>>>(out_idx, cand, p, K);
  return cudaGetLastError();
}

}  // namespace si
