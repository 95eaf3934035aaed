// Sparse attention over the entries the indexer selected.
//
// "StreamIndex: Memory-Bounded Compressed Sparse Attention via Streaming
// Top-k", Abstract: the indexer keeps the top-k compressed keys per query and
// a sparse attention kernel reads only those.  The abstract gives no formula;
// this kernel computes multi-query attention over the listed entries, every
// query head sharing one key row and one value row per entry:
//
//   J = { idx[b,t,r] : 0 <= idx < T }                (padding -1 skipped)
//   o[b,t,h,:] = sum_{j in J} softmax_j(scale * qa[b,t,h,:] . ka[b,j,:]) * va[b,j,:]
//   (o = 0 when J is empty)
//
// Shapes: 128 query heads of dim 128 (qa [B,S,128,128] bf16), ka/va [B,T,128]
// bf16, idx [B,S,k] int32 (k <= 2048), o [B,S,128,128] fp32.
//
// Design (one persistent CTA per SM, queries b*S+t taken in a fixed stride):
// per query the heads are the MMA's M = 128 rows, so one query is one
// tcgen05 tile row.  The listed entries are taken 128 at a time ("a tile"):
//   loader warps 0-3   gather the tile's key and value rows (one entry per
//                      thread, 16-byte cp.async into the 128-byte swizzled
//                      layout; unlisted slots are zero-filled) into one of two
//                      stages, and load the query's [128 x 128] block by TMA;
//   MMA warp 12        S = Q K^T (M=128 heads, N=128 entries, K=128) into one
//                      of two TMEM score buffers, then O += P V (M=128 heads,
//                      N=128 dims, K=128 entries) with V read MN-major from
//                      the same stage, one tile behind, so S of the next tile
//                      overlaps the softmax of this one;
//   softmax warps 4-11 two per TMEM lane quadrant, so one head per thread in
//                      each of two warps that split the tile's 128 columns:
//                      both take the running max over all columns, each the
//                      exponentials P = 2^(s - max) of its 64 (in bf16, into
//                      shared memory: the A operand of P V), the rescale of its
//                      half of O in TMEM when the max grows, its share of the
//                      row sum (added across the pair at the query's end), and
//                      O / sum of its half to global memory.
// Tiles whose 128 slots list no valid entry are skipped; a query that lists
// none writes zeros.  Every wait is bounded; a CTA that gives up records the
// error word and leaves.
#include "si_kernels.h"

namespace si {
namespace {

constexpr int kAttnH = 128;      // query heads (MMA M)
constexpr int kAttnD = 128;      // head dim
constexpr int kAttnTile = 128;   // listed entries per tile (MMA N of Q K^T, K of P V)
constexpr int kAttnThreads = 416;
constexpr int kLoadThreads = 128;
constexpr int kSoftWarp0 = 4;   // softmax warps 4-11: two per TMEM lane quadrant
constexpr int kSoftWarps = 8;
constexpr int kMmaWarp = 12;
constexpr uint32_t kTileBytes = kAttnTile * kAttnD * 2;  // 32 KB: one K, V, Q or P block
constexpr uint32_t kHalf = kTileBytes / 2;               // one 64-column half: [128 x 128 B]

struct AttnMeta {
  int valid;     // 0: no more items
  int query;     // b*S + t
  int qb;        // Q buffer of the query
  int first, last, empty;
  uint32_t mask[4];  // listed slots of the tile (bit e%32 of word e/32)
};

struct AttnCtl {
  uint64_t kv_full[2], kv_empty[2], q_full[2], q_empty[2];
  uint64_t s_full[2], s_empty[2], p_full, o_done;
  AttnMeta meta[2];
  uint32_t lmask[16][4];  // the loader's masks of the current query's tiles
  uint64_t xch[4];        // per lane quadrant: the two softmax warps' row sums are in
  float xsum[2][128];     // [column half][head]: a softmax warp's share of a row's sum
  uint32_t tmem_base;
  uint32_t abort;
};

// Byte offset of 16-byte chunk c (0..15) of row r in a [128 x 256 B] block
// stored as two 64-column halves, each 128 rows of 128 B with the 128-byte
// swizzle (chunk position XOR row % 8).
SI_DEV uint32_t sw_off(int r, int c) {
  return (uint32_t)((c >> 3) * kHalf + r * 128 + (((c & 7) ^ (r & 7)) << 4));
}

SI_DEV void cp_async16(uint32_t dst, const void* src, uint32_t src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src),
               "r"(src_bytes)
               : "memory");
}
SI_DEV void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
SI_DEV void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}
SI_DEV void fence_proxy_async() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

// Shared-memory descriptor, 128-byte swizzle, with an explicit leading byte
// offset: for an MN-major operand it is the distance between 64-element
// blocks along N; the stride byte offset (1024) is the distance between
// 8-row groups along K.
SI_DEV uint64_t sdesc_sw128_lbo(uint32_t saddr, uint32_t lbo_bytes) {
  return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)((lbo_bytes >> 4) & 0x3FFFu) << 16) |
         ((uint64_t)64u << 32) | ((uint64_t)1u << 46) | ((uint64_t)2u << 61);
}

SI_DEV void tmem_st32(uint32_t taddr, const float (&v)[32]) {
  const uint32_t* r = reinterpret_cast<const uint32_t*>(v);
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
      "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
      "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
      "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]),
      "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]),
      "r"(r[29]), "r"(r[30]), "r"(r[31])
      : "memory");
}
SI_DEV void tmem_st_wait() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

SI_DEV void fence32(float (&v)[32]) {
  asm volatile(""
               : "+f"(v[0]), "+f"(v[1]), "+f"(v[2]), "+f"(v[3]), "+f"(v[4]), "+f"(v[5]),
                 "+f"(v[6]), "+f"(v[7]), "+f"(v[8]), "+f"(v[9]), "+f"(v[10]), "+f"(v[11]),
                 "+f"(v[12]), "+f"(v[13]), "+f"(v[14]), "+f"(v[15]), "+f"(v[16]), "+f"(v[17]),
                 "+f"(v[18]), "+f"(v[19]), "+f"(v[20]), "+f"(v[21]), "+f"(v[22]), "+f"(v[23]),
                 "+f"(v[24]), "+f"(v[25]), "+f"(v[26]), "+f"(v[27]), "+f"(v[28]), "+f"(v[29]),
                 "+f"(v[30]), "+f"(v[31]));
}

// Named barrier over n threads that also returns, to every one of them,
// whether any passed pred = true (so all leave a loop together).
SI_DEV bool named_bar_or(uint32_t id, uint32_t n, bool pred) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "barrier.cta.red.or.pred q, %2, %3, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"((uint32_t)pred), "r"(id), "r"(n)
      : "memory");
  return r != 0u;
}

SI_DEV uint32_t pack_bf16(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

}  // namespace

__global__ void __launch_bounds__(kAttnThreads, 1)
    k_sparse_attn(const __grid_constant__ CUtensorMap tm_q, const AttnParams p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  // [Q0 | Q1 | K0 | V0 | K1 | V1 | P | ctl], each block 32 KB
  const uint32_t base = smem_u32(smem);
  const uint32_t q_s = base, kv_s = base + 2 * kTileBytes, p_s = base + 6 * kTileBytes;
  AttnCtl* cs = reinterpret_cast<AttnCtl*>(smem + 7 * kTileBytes);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int64_t nq = (int64_t)p.B * p.S;

  if (tid == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(smem_u32(&cs->kv_full[i]), kLoadThreads);
      mbar_init(smem_u32(&cs->kv_empty[i]), 1 + kSoftWarps);  // the MMA side, each softmax warp
      mbar_init(smem_u32(&cs->q_full[i]), 1);
      mbar_init(smem_u32(&cs->q_empty[i]), 1);
      mbar_init(smem_u32(&cs->s_full[i]), 1);
      mbar_init(smem_u32(&cs->s_empty[i]), kSoftWarps * 32);
    }
    mbar_init(smem_u32(&cs->p_full), kSoftWarps * 32);
    for (int i = 0; i < 4; ++i) mbar_init(smem_u32(&cs->xch[i]), 64);
    mbar_init(smem_u32(&cs->o_done), 1);
    cs->abort = 0u;
    mbar_fence_init();
  }
  if (warp == kMmaWarp) {
    tmem_alloc(smem_u32(&cs->tmem_base), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = cs->tmem_base;
  Ctl ctl{p.err, &cs->abort, p.timeout_ns, nullptr};
  const int ntiles = (p.k + kAttnTile - 1) / kAttnTile;

  if (warp < kSoftWarp0) {
    // ------------------------------------------------------------ loaders
    // Each item's rows are signalled as soon as they land (a loader that
    // signalled one item late would wait on a stage that only the MMA of the
    // item it holds back can free).  A failed wait sets the CTA's abort flag,
    // which every loader reads after the per-query barrier, so all of them
    // leave together and the named barriers stay matched.
    uint32_t it = 0, qn = 0;
    for (int64_t qid = blockIdx.x; qid < nq; qid += gridDim.x, ++qn) {
      const int b = (int)(qid / p.S);
      const int32_t* irow = p.idx + qid * p.k;
      // which of the query's tiles list any entry
      for (int ti = 0; ti < ntiles; ++ti) {
        const int e = ti * kAttnTile + tid;
        const int j = e < p.k ? __ldg(irow + e) : -1;
        const uint32_t m = __ballot_sync(0xFFFFFFFFu, j >= 0 && j < p.T);
        if (lane == 0) cs->lmask[ti][warp] = m;
      }
      named_bar_sync(1, kLoadThreads);
      int last_ti = -1;
      for (int ti = 0; ti < ntiles; ++ti)
        if (cs->lmask[ti][0] | cs->lmask[ti][1] | cs->lmask[ti][2] | cs->lmask[ti][3]) last_ti = ti;
      // the query block, by TMA
      const int qb = (int)(qn & 1u);
      bool ok = true;
      if (tid == 0) {
        if (!mbar_wait(smem_u32(&cs->q_empty[qb]), ((qn >> 1) & 1u) ^ 1u, ctl)) {
          ok = false;
        } else {
          const uint32_t bar = smem_u32(&cs->q_full[qb]);
          mbar_arrive_expect_tx(bar, kTileBytes);
          const int row = (int)(qid * kAttnH);
          tma_load_2d(q_s + qb * kTileBytes, &tm_q, bar, 0, row, policy_evict_first());
          tma_load_2d(q_s + qb * kTileBytes + kHalf, &tm_q, bar, 64, row, policy_evict_first());
        }
      }
      bool first = true;
      for (int ti = 0; ok && ti <= (last_ti < 0 ? 0 : last_ti); ++ti) {
        const bool empty = last_ti < 0;
        if (!empty && !(cs->lmask[ti][0] | cs->lmask[ti][1] | cs->lmask[ti][2] | cs->lmask[ti][3]))
          continue;
        const int s = (int)(it & 1u);
        if (!mbar_wait(smem_u32(&cs->kv_empty[s]), ((it >> 1) & 1u) ^ 1u, ctl)) {
          ok = false;
          break;
        }
        if (tid == 0) {
          AttnMeta& md = cs->meta[s];
          md.valid = 1;
          md.query = (int)qid;
          md.qb = qb;
          md.first = first ? 1 : 0;
          md.last = (empty || ti == last_ti) ? 1 : 0;
          md.empty = empty ? 1 : 0;
          for (int w = 0; w < 4; ++w) md.mask[w] = empty ? 0u : cs->lmask[ti][w];
        }
        if (!empty) {
          // entry e of the tile: its key row and value row, 16 chunks each
          const int e = ti * kAttnTile + tid;
          const int j = e < p.k ? __ldg(irow + e) : -1;
          const bool listed = j >= 0 && j < p.T;
          const int64_t row = (int64_t)b * p.T + (listed ? j : 0);
          const uint16_t* kr = p.ka + row * kAttnD;
          const uint16_t* vr = p.va + row * kAttnD;
          const uint32_t kdst = kv_s + s * 2 * kTileBytes, vdst = kdst + kTileBytes;
#pragma unroll
          for (int c = 0; c < 16; ++c) {
            cp_async16(kdst + sw_off(tid, c), kr + c * 8, listed ? 16u : 0u);
            cp_async16(vdst + sw_off(tid, c), vr + c * 8, listed ? 16u : 0u);
          }
          cp_async_commit();
          cp_async_wait<0>();
          fence_proxy_async();  // the rows are read by the tensor cores (async proxy)
        }
        mbar_arrive(smem_u32(&cs->kv_full[s]));
        first = false;
        ++it;
      }
      // lmask is rewritten by the next query; every loader leaves together
      if (named_bar_or(1, kLoadThreads, *ctl.abort != 0u)) break;
    }
    // end marker
    if (!*ctl.abort) {
      const int s = (int)(it & 1u);
      if (mbar_wait(smem_u32(&cs->kv_empty[s]), ((it >> 1) & 1u) ^ 1u, ctl)) {
        if (tid == 0) cs->meta[s].valid = 0;
        mbar_arrive(smem_u32(&cs->kv_full[s]));
      }
    }
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc_s = idesc_make(1, 1, kAttnH, kAttnTile);
      // P V: B (the value rows) is MN-major: bit 16 transposes B
      constexpr uint32_t idesc_o = idesc_make(1, 1, kAttnH, kAttnD) | (1u << 16);
      uint32_t it = 0, n1 = 0, n2 = 0, qn = 0;
      bool pend = false;
      int pend_s = 0, pend_first = 0;
      for (;;) {
        const int s = (int)(it & 1u);
        if (!mbar_wait(smem_u32(&cs->kv_full[s]), (it >> 1) & 1u, ctl)) break;
        const AttnMeta md = cs->meta[s];
        if (md.valid && md.first) ++qn;
        const int qb = md.qb;
        if (md.valid && !md.empty) {
          if (md.first && !mbar_wait(smem_u32(&cs->q_full[qb]), ((qn - 1) >> 1) & 1u, ctl)) break;
          const int sb = (int)(n1 & 1u);
          if (!mbar_wait(smem_u32(&cs->s_empty[sb]), ((n1 >> 1) & 1u) ^ 1u, ctl)) break;
          tc_fence_after();
          const uint32_t qa = q_s + qb * kTileBytes, ka = kv_s + s * 2 * kTileBytes;
#pragma unroll
          for (int kk = 0; kk < kAttnD / 16; ++kk) {
            const uint32_t off = (kk >> 2) * kHalf + (kk & 3) * 32;
            umma_bf16(tmem + sb * kAttnTile, sdesc_sw128(qa + off), sdesc_sw128(ka + off), idesc_s,
                      kk > 0 ? 1u : 0u);
          }
          umma_commit(smem_u32(&cs->s_full[sb]));
          ++n1;
          if (md.last) umma_commit(smem_u32(&cs->q_empty[qb]));
        } else if (md.valid && md.first && md.last) {
          // a query that lists nothing: its block was still loaded
          if (!mbar_wait(smem_u32(&cs->q_full[qb]), ((qn - 1) >> 1) & 1u, ctl)) break;
          mbar_arrive(smem_u32(&cs->q_empty[qb]));
        }
        if (pend) {
          // O += P V of the previous tile
          if (!mbar_wait(smem_u32(&cs->p_full), n2 & 1u, ctl)) break;
          tc_fence_after();
          const uint32_t va = kv_s + pend_s * 2 * kTileBytes + kTileBytes;
#pragma unroll
          for (int kk = 0; kk < kAttnTile / 16; ++kk) {
            const uint32_t aoff = (kk >> 2) * kHalf + (kk & 3) * 32;
            umma_bf16(tmem + 2 * kAttnTile, sdesc_sw128(p_s + aoff),
                      sdesc_sw128_lbo(va + kk * 2048, kHalf), idesc_o,
                      (kk > 0 || !pend_first) ? 1u : 0u);
          }
          umma_commit(smem_u32(&cs->o_done));
          umma_commit(smem_u32(&cs->kv_empty[pend_s]));
          ++n2;
          pend = false;
        }
        if (!md.valid) break;
        if (md.empty) {
          mbar_arrive(smem_u32(&cs->kv_empty[s]));
        } else {
          pend = true;
          pend_s = s;
          pend_first = md.first;
        }
        ++it;
      }
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ softmax
    const int quad = warp & 3;
    const int st = quad * 32 + lane;          // the head, and the TMEM lane
    const int half = (warp - kSoftWarp0) >> 2;  // columns [64*half, 64*half + 64) of S, P and O
    const uint32_t lane_base = tmem + ((uint32_t)(quad * 32) << 16);
    const uint32_t o_col = lane_base + 2 * kAttnTile;
    const float sl2 = p.scale_log2;
    const float ninf = __int_as_float(0xFF800000);
    uint32_t it = 0, n1 = 0, n2i = 0, n2w = 0, nx = 0;
    float m = ninf, l = 0.0f;  // l: this warp's half of the row sum
    bool any = false;  // the current query has had a tile
    for (;;) {
      const int s = (int)(it & 1u);
      if (!mbar_wait_warp(smem_u32(&cs->kv_full[s]), (it >> 1) & 1u, ctl)) break;
      const AttnMeta md = cs->meta[s];
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&cs->kv_empty[s]));
      if (!md.valid) break;
      if (md.first) {
        m = ninf;
        l = 0.0f;
        any = false;
      }
      bool stop = false;
      if (!md.empty) {
        const int sb = (int)(n1 & 1u);
        if (!mbar_wait_warp(smem_u32(&cs->s_full[sb]), (n1 >> 1) & 1u, ctl)) break;
        tc_fence_after();
        const uint32_t s_col = lane_base + sb * kAttnTile;
        float v[32];
        // pass 1: the tile's largest listed score (scale >= 0, so the largest
        // raw dot product scales to the largest logit), four chains, and no
        // per-slot test on a fully listed group of 32.  Both warps of a lane
        // quadrant take all 128 columns here, so each has the row maximum
        // without an exchange; the exponentials below are split by column half.
        float mx4[4] = {ninf, ninf, ninf, ninf};
#pragma unroll 1
        for (int c = 0; c < 4; ++c) {
          tmem_ld32(s_col + c * 32, v);
          tmem_ld_wait();
          fence32(v);
          const uint32_t mk = md.mask[c];
          if (mk == 0xFFFFFFFFu) {
#pragma unroll
            for (int e = 0; e < 32; ++e) mx4[e & 3] = fmaxf(mx4[e & 3], v[e]);
          } else {
#pragma unroll
            for (int e = 0; e < 32; ++e)
              if ((mk >> e) & 1u) mx4[e & 3] = fmaxf(mx4[e & 3], v[e]);
          }
        }
        const float mxr = fmaxf(fmaxf(mx4[0], mx4[1]), fmaxf(mx4[2], mx4[3]));
        const float m_new = fmaxf(m, mxr * sl2);
        // P and O belong to the previous tile's P V until it completes
        if (n2i > n2w) {
          if (!mbar_wait_warp(smem_u32(&cs->o_done), n2w & 1u, ctl)) break;
          ++n2w;
          tc_fence_after();
        }
        // the rescale reads and writes TMEM with warp-collective loads and
        // stores, so a warp does it when any of its heads' maximum grew (a
        // factor of 1 for the others)
        if (any && __any_sync(0xFFFFFFFFu, m_new > m)) {
          const float a = m_new > m ? exp2f(m - m_new) : 1.0f;
          l *= a;
#pragma unroll 1
          for (int c = 2 * half; c < 2 * half + 2; ++c) {
            tmem_ld32(o_col + c * 32, v);
            tmem_ld_wait();
            fence32(v);
#pragma unroll
            for (int e = 0; e < 32; ++e) v[e] *= a;
            tmem_st32(o_col + c * 32, v);
          }
          tmem_st_wait();
        }
        m = m_new;
        // pass 2: P = 2^(s*scale*log2(e) - m) on listed slots, 0 elsewhere
        float l4[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll 1
        for (int c = 2 * half; c < 2 * half + 2; ++c) {
          tmem_ld32(s_col + c * 32, v);
          tmem_ld_wait();
          fence32(v);
          const uint32_t mk = md.mask[c];
          if (mk == 0xFFFFFFFFu) {
#pragma unroll
            for (int e = 0; e < 32; ++e) {
              v[e] = exp2f(fmaf(v[e], sl2, -m));
              l4[e & 3] += v[e];
            }
          } else {
#pragma unroll
            for (int e = 0; e < 32; ++e) {
              v[e] = ((mk >> e) & 1u) ? exp2f(fmaf(v[e], sl2, -m)) : 0.0f;
              l4[e & 3] += v[e];
            }
          }
          // entries 32c .. 32c+31 are chunks 4c .. 4c+3 of the head's P row
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            uint4 w;
            w.x = pack_bf16(v[8 * q + 0], v[8 * q + 1]);
            w.y = pack_bf16(v[8 * q + 2], v[8 * q + 3]);
            w.z = pack_bf16(v[8 * q + 4], v[8 * q + 5]);
            w.w = pack_bf16(v[8 * q + 6], v[8 * q + 7]);
            const uint32_t dst = p_s + sw_off(st, 4 * c + q);
            asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(dst), "r"(w.x),
                         "r"(w.y), "r"(w.z), "r"(w.w)
                         : "memory");
          }
        }
        l += (l4[0] + l4[1]) + (l4[2] + l4[3]);
        tc_fence_before();
        mbar_arrive(smem_u32(&cs->s_empty[sb]));
        ++n1;
        fence_proxy_async();
        mbar_arrive(smem_u32(&cs->p_full));
        ++n2i;
        any = true;
      }
      if (md.last) {
        float* orow = p.out + ((int64_t)md.query * kAttnH + st) * kAttnD;
        if (any) {
          // the row sum: this warp's half plus its partner's (the buffer is
          // rewritten only after the partner's next P, so once per query is safe)
          cs->xsum[half][st] = l;
          mbar_arrive(smem_u32(&cs->xch[quad]));
          if (!mbar_wait_warp(smem_u32(&cs->xch[quad]), nx & 1u, ctl)) stop = true;
          ++nx;
          const float lt = stop ? 1.0f : l + cs->xsum[half ^ 1][st];
          if (!stop && !mbar_wait_warp(smem_u32(&cs->o_done), n2w & 1u, ctl)) stop = true;
          if (!stop) {
            ++n2w;
            tc_fence_after();
            const float inv = 1.0f / lt;
            float v[32];
#pragma unroll 1
            for (int c = 2 * half; c < 2 * half + 2; ++c) {
              tmem_ld32(o_col + c * 32, v);
              tmem_ld_wait();
              fence32(v);
#pragma unroll
              for (int e = 0; e < 32; e += 4)
                *reinterpret_cast<float4*>(orow + c * 32 + e) =
                    make_float4(v[e] * inv, v[e + 1] * inv, v[e + 2] * inv, v[e + 3] * inv);
            }
            tc_fence_before();
          }
        } else {
          for (int c = 64 * half; c < 64 * half + 64; c += 4)
            *reinterpret_cast<float4*>(orow + c) = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
        }
      }
      if (stop) break;
      ++it;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

size_t sparse_attn_smem_bytes() { return 7 * (size_t)kTileBytes + sizeof(AttnCtl) + 1024; }

cudaError_t launch_sparse_attn(const CUtensorMap& tm_q, const AttnParams& p, int grid,
                               cudaStream_t stream) {
  const size_t smem = sparse_attn_smem_bytes();
  cudaError_t e = cudaFuncSetAttribute(k_sparse_attn, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)smem);
  if (e != cudaSuccess) return e;
  k_sparse_attn<<<grid, kAttnThreads, smem, stream>>>(tm_q, p);
  return cudaGetLastError();
}

}  // namespace si
