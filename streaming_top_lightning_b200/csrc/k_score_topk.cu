// Fused lightning-indexer score + streaming top-k on 5th-generation tensor cores.
//
// "StreamIndex: Memory-Bounded Compressed Sparse Attention via Streaming
// Top-k", Abstract: a lightning indexer scores the compressed keys, the top-k
// are selected per query, and the [B,S,H_I,T] fp32 score tensor is never
// materialised.  Score read as I[t,j] = sum_h w[t,h] * max(0, q[t,h,:].kc[j,:]),
// key j visible to t iff (j+1)*m - 1 <= t.
//
// Orientation: compressed keys on the MMA M dimension (128 TMEM lanes), the
// QT = 256/H_I queries of a query tile times their H_I heads on N = 256.  So
// D[j, (t,h)] = kc[j] . q[t,h] lands in TMEM with one key per lane, and each
// epilogue thread reduces the heads of its own key without any cross-lane
// traffic: one max and half a packed FMA per accumulator element.
//
// Warp roles (448 threads, one CTA per SM, persistent):
//   warp 0      TMA producer and unit scheduler: takes (tile, chunk) units from
//               a global counter one unit ahead (starting the next unit's query
//               tile towards L2), loads the query tile once per unit and streams
//               128-key tiles of kc through an NST-stage mbarrier ring;
//   warp 1      allocates 512 TMEM columns and issues tcgen05.mma (one thread)
//               into two 256-column accumulators used alternately;
//   warps 2-9   epilogue: warp w reads TMEM lane quadrant w%4 (32 keys) and
//               column half (w-2)/4 (128 columns: QT/2 queries); tcgen05.ld,
//               ReLU, w-weighted head sum (x s_k for FP8) in several
//               independent packed-FMA chains per query, scores into a
//               shared-memory strip; never to global memory;
//   warps 10-13 streaming selection (si_select.cuh) on the strips.
// So every SM sub-partition runs two epilogue warps and one selection warp.
// Every wait is bounded (si_common.cuh); on expiry the CTA drains its own
// asynchronous copies and MMAs, frees TMEM and exits with an error word set.
#include <algorithm>

#include "si_kernels.h"

namespace si {

constexpr int kThreads = 448;
constexpr int kRing = 4;        // unit ring depth
constexpr int kN = 256;         // largest MMA N: query-tile rows (QT * H)
constexpr int kM = 128;         // MMA M: keys per tile
constexpr int kEpiWarp0 = 2;    // first epilogue warp
constexpr int kEpiWarps = 8;    // two per TMEM lane quadrant, one per column half
constexpr int kEpiThreads = kEpiWarps * 32;
constexpr int kSelWarp0 = kEpiWarp0 + kEpiWarps;  // first selection warp
constexpr int kMaxSlots = 4;    // score-strip ring slots at most
static_assert(kThreads == (kSelWarp0 + kSelWarps) * 32, "warp roles");

struct UnitInfo {
  int valid, b, g, c, kbeg, kend, ntiles;
};

struct ScoreCtlSmem {
  uint64_t full[8], empty[8];
  uint64_t acc_full[2], acc_empty[2];
  uint64_t q_full, q_empty;
  uint64_t unit_full[kRing], unit_empty[kRing];
  uint64_t strip_full[kMaxSlots], strip_empty[kMaxSlots];
  uint64_t drain;
  UnitInfo ring[kRing];
  StripMeta meta[kMaxSlots];
  uint32_t tmem_base;
  uint32_t abort;
};

template <bool FP8, int D, int NQ>
struct OperandGeom {
  static constexpr int kEsz = FP8 ? 1 : 2;
  static constexpr int kRowBytes = D * kEsz;                      // bytes of one row
  static constexpr int kSw = kRowBytes >= 128 ? 128 : kRowBytes;  // swizzle span
  static constexpr int kKBlocks = kRowBytes / kSw;                // K-blocks per row
  static constexpr int kKSteps = kRowBytes / 32;                  // MMA instructions per tile
  static constexpr int kQBytes = NQ * kRowBytes;
  static constexpr int kKcBytes = kM * kRowBytes;
  static constexpr int kKbBytes = kM * kSw;       // one K-block of a key tile: a ring slot
  static constexpr int kPerBlock = kSw / 32;      // MMA instructions per K-block
};

template <int SW>
SI_DEV uint64_t sdesc(uint32_t saddr) {
  // K-major, swizzled: 8-row groups SW*8 bytes apart.  Layout code: 128B -> 2,
  // 64B -> 4 (see the descriptor field notes in si_common.cuh).
  constexpr uint64_t kLayout = SW == 128 ? 2u : 4u;
  return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)1u << 16) |
         ((uint64_t)((SW * 8) >> 4) << 32) | ((uint64_t)1u << 46) | (kLayout << 61);
}

SI_DEV void tmem_ld_fence(float (&v)[32]) {
  asm volatile(""
               : "+f"(v[0]), "+f"(v[1]), "+f"(v[2]), "+f"(v[3]), "+f"(v[4]), "+f"(v[5]),
                 "+f"(v[6]), "+f"(v[7]), "+f"(v[8]), "+f"(v[9]), "+f"(v[10]), "+f"(v[11]),
                 "+f"(v[12]), "+f"(v[13]), "+f"(v[14]), "+f"(v[15]), "+f"(v[16]), "+f"(v[17]),
                 "+f"(v[18]), "+f"(v[19]), "+f"(v[20]), "+f"(v[21]), "+f"(v[22]), "+f"(v[23]),
                 "+f"(v[24]), "+f"(v[25]), "+f"(v[26]), "+f"(v[27]), "+f"(v[28]), "+f"(v[29]),
                 "+f"(v[30]), "+f"(v[31]));
}

// Independent packed accumulators per query of an epilogue warp: enough
// chains to cover the FMA latency, at most 8 float2 in all.  COLS is the
// warp's column count (its share of the MMA N).
template <int H, int COLS>
struct EpiGeom {
  static constexpr int kQH = COLS / H;                 // queries of the warp's columns
  static constexpr int kNA = kQH >= 8 ? 1 : 8 / kQH;   // chains per query
  static_assert(kQH * kNA <= 32 && (H / 2) % kNA == 0, "accumulator split");
};

// Weighted ReLU head sum of one 32-column chunk of this warp's columns into
// the packed accumulators.  Local column c = ch*32 + e is query c / H of the
// warp and head c % H; head pair (c % H)/2 feeds chain ((c % H)/2) % kNA.
// wsrc: the warp's weights, contiguous -- global memory for bf16 (read as
// float4 through the read-only path; the same 16 bytes in every lane, one L1
// wavefront), the shared-memory copy for FP8.
template <bool FP8, int H, int COLS>
SI_DEV void epi_chunk(int ch, const float (&v)[32], const float* wsrc,
                      float2 (&acc)[EpiGeom<H, COLS>::kQH][EpiGeom<H, COLS>::kNA]) {
  constexpr int NA = EpiGeom<H, COLS>::kNA;
#pragma unroll
  for (int e = 0; e < 32; e += 4) {
    const int col = ch * 32 + e;
    const int ql = col / H;
    const int a0 = ((col % H) >> 1) % NA, a1 = (((col + 2) % H) >> 1) % NA;
    const float4 wv = FP8 ? *reinterpret_cast<const float4*>(wsrc + col)
                          : __ldg(reinterpret_cast<const float4*>(wsrc + col));
    const float2 r0 = make_float2(fmaxf(v[e], 0.0f), fmaxf(v[e + 1], 0.0f));
    const float2 r1 = make_float2(fmaxf(v[e + 2], 0.0f), fmaxf(v[e + 3], 0.0f));
    acc[ql][a0] = __ffma2_rn(make_float2(wv.x, wv.y), r0, acc[ql][a0]);
    acc[ql][a1] = __ffma2_rn(make_float2(wv.z, wv.w), r1, acc[ql][a1]);
  }
}

template <bool FP8, int D, int H, int NQ>
__global__ void __launch_bounds__(kThreads, 1)
    k_score_topk(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_kc,
                 const ScoreParams p) {
  using G = OperandGeom<FP8, D, NQ>;
  constexpr int QT = NQ / H;
  constexpr int COLS = NQ / 2;  // accumulator columns per epilogue warp (a column half)
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  // 1024-byte alignment for the swizzled operand tiles
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  const SelParams& sp = p.sel;
  const int CS = sp.CS, NST = p.nst, NSL = p.nslot;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  uint8_t* q_s = smem;
  uint8_t* kc_s = q_s + G::kQBytes;
  float* strip = reinterpret_cast<float*>(kc_s + (size_t)NST * G::kKbBytes);
  uint8_t* sel_base = reinterpret_cast<uint8_t*>(strip + (size_t)NSL * QT * CS);
  SelSmem sm;
  sel_state_carve(sel_base, QT, sp.cap, sm);
  // FP8 only, [kEpiWarps][COLS]: each epilogue warp's copy of its columns'
  // weights folded with the query row scales
  float* w_s = reinterpret_cast<float*>(sel_base + sel_state_bytes(QT, sp.cap));
  ScoreCtlSmem* cs = reinterpret_cast<ScoreCtlSmem*>(w_s + (FP8 ? kEpiWarps * COLS : 0));

  const uint32_t q_addr = smem_u32(q_s), kc_addr = smem_u32(kc_s);
  if (tid == 0) {
    for (int s = 0; s < NST; ++s) {
      mbar_init(smem_u32(&cs->full[s]), 1);
      mbar_init(smem_u32(&cs->empty[s]), 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(smem_u32(&cs->acc_full[i]), 1);
      mbar_init(smem_u32(&cs->acc_empty[i]), kEpiThreads);
    }
    for (int i = 0; i < NSL; ++i) {
      // a strip of CS >= 128 keys is written by every epilogue thread; a
      // shorter one by the two warps (one per column half) of each of its
      // CS/32 lane quadrants
      mbar_init(smem_u32(&cs->strip_full[i]), CS >= kM ? kEpiThreads : 2 * CS);
      mbar_init(smem_u32(&cs->strip_empty[i]), kSelWarps * 32);  // every selection lane
    }
    mbar_init(smem_u32(&cs->q_full), 1);
    mbar_init(smem_u32(&cs->q_empty), 1);
    for (int i = 0; i < kRing; ++i) {
      mbar_init(smem_u32(&cs->unit_full[i]), 1);
      mbar_init(smem_u32(&cs->unit_empty[i]), 1 + kEpiWarps);
    }
    mbar_init(smem_u32(&cs->drain), 1);
    cs->abort = 0u;
    mbar_fence_init();
  }
  if (tid < QT) {
    sm.npool[tid] = 0;
    sm.theta[tid] = 0ull;
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(&cs->tmem_base), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = cs->tmem_base;
  Ctl ctl{p.err, &cs->abort, p.timeout_ns, p.role};

  if (warp == 0) {
    // ---------------------------------------------------------- producer
    if (lane == 0) {
      const long long t_role = role_t0();
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_kc);
      const uint64_t pol_q = policy_evict_first();
      const uint64_t pol_k = policy_evict_last();
      uint32_t ring_it = 0, kstage = 0, q_it = 0;
      bool q_issued = false;
      bool skipped = false;  // debug: one key tile deliberately never loaded
      int skipped_stage = -1;
      // Units are taken and published one ahead: the next unit's descriptor is
      // in the ring before this unit's first key tile is loaded, so the MMA
      // and epilogue warps never wait for it, and its query tile is on its way
      // to L2 while this one streams.  A CTA stops at its first failed decode
      // (which it publishes as the end marker), so the counter still advances
      // by exactly (units + grid) per launch.  The ring has room: its
      // consumers release an entry when they start that unit, and they are at
      // most one unit behind the one being loaded.
      // publish(): 1 = a unit, 0 = the end marker, -1 = abort
      auto publish = [&](int id, UnitInfo& u) -> int {
        int b = 0, g = 0, c = 0;
        const bool ok = unit_decode(p.ug, id, b, g, c);
        const int r = ring_it % kRing;
        if (!mbar_wait(smem_u32(&cs->unit_empty[r]), ((ring_it / kRing) & 1u) ^ 1u, ctl,
                       R_PROD_WAIT_UNIT))
          return -1;
        u = UnitInfo{0, 0, 0, 0, 0, 0, 0};
        if (ok) {
          const int vmax = tile_vmax_b(p.ug, b, g);
          u.valid = 1;
          u.b = b;
          u.g = g;
          u.c = c;
          u.kbeg = c * p.ug.C;
          u.kend = p.ug.tile_units ? vmax : min(u.kbeg + p.ug.C, vmax);
          u.ntiles = u.kend > u.kbeg ? (u.kend - u.kbeg + kM - 1) / kM : 0;
        }
        cs->ring[r] = u;
        mbar_arrive(smem_u32(&cs->unit_full[r]));
        ++ring_it;
        return ok ? 1 : 0;
      };
      UnitInfo u;
      int st = publish(atomicAdd(p.counter, 1) - p.ug.id_base, u);
      while (st > 0) {
        UnitInfo nxt;
        const int st2 = publish(atomicAdd(p.counter, 1) - p.ug.id_base, nxt);
        if (st2 < 0) break;
        if (st2 > 0 && nxt.ntiles > 0 && (nxt.b != u.b || nxt.g != u.g)) {
          const int qrow2 = (nxt.b * sp.S + nxt.g * QT) * H;
#pragma unroll
          for (int kb = 0; kb < G::kKBlocks; ++kb)
            tma_prefetch_l2_2d(&tm_q, kb * (G::kSw / G::kEsz), qrow2);
        }
        if (u.ntiles > 0) {
          // query tile: rows (b*S + g*QT)*H .. +NQ of q viewed as [B*S*H, D]
          if (!mbar_wait(smem_u32(&cs->q_empty), (q_it & 1u) ^ 1u, ctl, R_PROD_WAIT_Q)) break;
          const uint32_t qb = smem_u32(&cs->q_full);
          mbar_arrive_expect_tx(qb, G::kQBytes);
          const int qrow = (u.b * sp.S + u.g * QT) * H;
#pragma unroll
          for (int kb = 0; kb < G::kKBlocks; ++kb)
            tma_load_2d(q_addr + kb * (NQ * G::kSw), &tm_q, qb, kb * (G::kSw / G::kEsz), qrow,
                        pol_q);
          q_issued = true;
          ++q_it;
          // key tiles, one K-block (kM keys x kSw bytes) per ring slot
          bool stop = false;
          for (int i = 0; i < u.ntiles && !stop; ++i) {
            const int krow = u.b * sp.T + u.kbeg + i * kM;
            for (int kb = 0; kb < G::kKBlocks; ++kb) {
              const int s = kstage % NST;
              if (!mbar_wait(smem_u32(&cs->empty[s]), ((kstage / NST) & 1u) ^ 1u, ctl,
                             R_PROD_WAIT_KC)) {
                stop = true;
                break;
              }
              const uint32_t fb = smem_u32(&cs->full[s]);
              mbar_arrive_expect_tx(fb, G::kKbBytes);
              if ((p.debug_flags & 1) && !skipped) {
                skipped = true;  // the consumer's wait on this slot must expire
                skipped_stage = s;
              } else {
                tma_load_2d(kc_addr + s * G::kKbBytes, &tm_kc, fb, kb * (G::kSw / G::kEsz), krow,
                            pol_k);
              }
              ++kstage;
            }
          }
          if (stop) break;
        }
        u = nxt;
        st = st2;
      }
      // drain: wait (bounded, regardless of abort) for every copy this thread
      // issued to land before the CTA may exit
      Ctl drain_ctl{p.err, nullptr, p.timeout_ns, nullptr};
      uint32_t dummy = 0;
      drain_ctl.abort = &dummy;
      for (uint32_t n = (kstage > (uint32_t)NST ? kstage - NST : 0); n < kstage; ++n) {
        const int s = n % NST;
        if (s == skipped_stage) continue;
        mbar_wait(smem_u32(&cs->full[s]), (n / NST) & 1u, drain_ctl);
      }
      if (q_issued) mbar_wait(smem_u32(&cs->q_full), (q_it - 1) & 1u, drain_ctl);
      role_add(ctl, R_PROD_TOTAL, t_role);
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------- MMA issuer
    if (lane == 0) {
      const long long t_role = role_t0();
      constexpr uint32_t idesc = FP8 ? idesc_make(0, 0, kM, NQ) : idesc_make(1, 1, kM, NQ);
      uint32_t ring_it = 0, kstage = 0, acc_it = 0, q_it = 0;
      for (;;) {
        const int r = ring_it % kRing;
        if (!mbar_wait(smem_u32(&cs->unit_full[r]), (ring_it / kRing) & 1u, ctl, R_MMA_WAIT_UNIT))
          break;
        const UnitInfo u = cs->ring[r];  // ordered after the acquiring wait
        mbar_arrive(smem_u32(&cs->unit_empty[r]));
        ++ring_it;
        if (!u.valid) break;
        role_count(ctl, R_UNITS, 1);
        role_count(ctl, R_TILES, (unsigned long long)u.ntiles);
        if (u.ntiles == 0) continue;
        if (!mbar_wait(smem_u32(&cs->q_full), q_it & 1u, ctl, R_MMA_WAIT_Q)) break;
        tc_fence_after();
        bool stop = false;
        for (int i = 0; i < u.ntiles && !stop; ++i) {
          const int ab = acc_it & 1;
          if (!mbar_wait(smem_u32(&cs->acc_empty[ab]), ((acc_it >> 1) & 1u) ^ 1u, ctl,
                         R_MMA_WAIT_ACC)) {
            stop = true;
            break;
          }
          const uint32_t d_tmem = tmem + ab * NQ;
          // the tile's K-blocks, one ring slot each; a slot is released as
          // soon as its MMAs have read it
#pragma unroll
          for (int kb = 0; kb < G::kKBlocks; ++kb) {
            const int s = kstage % NST;
            if (!mbar_wait(smem_u32(&cs->full[s]), (kstage / NST) & 1u, ctl, R_MMA_WAIT_KC)) {
              stop = true;
              break;
            }
            tc_fence_after();
            const uint32_t a0 = kc_addr + s * G::kKbBytes;
#pragma unroll
            for (int kin = 0; kin < G::kPerBlock; ++kin) {
              const uint64_t ad = sdesc<G::kSw>(a0 + kin * 32);
              const uint64_t bd = sdesc<G::kSw>(q_addr + kb * (NQ * G::kSw) + kin * 32);
              const uint32_t acc = (kb > 0 || kin > 0) ? 1u : 0u;
              if (FP8) umma_f8(d_tmem, ad, bd, idesc, acc);
              else umma_bf16(d_tmem, ad, bd, idesc, acc);
            }
            umma_commit(smem_u32(&cs->empty[s]));
            ++kstage;
          }
          if (stop) break;
          umma_commit(smem_u32(&cs->acc_full[ab]));
          ++acc_it;
        }
        if (stop) break;
        umma_commit(smem_u32(&cs->q_empty));
        ++q_it;
      }
      // drain: all MMAs issued by this thread complete before TMEM is freed
      umma_commit(smem_u32(&cs->drain));
      uint32_t dummy = 0;
      Ctl drain_ctl{p.err, &dummy, p.timeout_ns, nullptr};
      mbar_wait(smem_u32(&cs->drain), 0u, drain_ctl);
      role_add(ctl, R_MMA_TOTAL, t_role);
    }
  } else if (warp < kSelWarp0) {
    // ---------------------------------------------------------- epilogue
    using EG = EpiGeom<H, COLS>;
    constexpr int QH = EG::kQH, NA = EG::kNA, NCH = COLS / 32;
    static_assert(NCH % 2 == 0, "epilogue chunk schedule");
    const int ew = warp - kEpiWarp0;  // 0 .. kEpiWarps-1
    const int quad = warp & 3;        // TMEM lane quadrant this warp may access
    const int cb = ew >> 2;           // column block: queries [cb*QH, cb*QH + QH)
    const int kl = quad * 32 + lane;  // key within the tile
    // strips shorter than a tile (CS = 32 or 64): a tile fills SUB strips and
    // this warp's 32 keys belong to strip `sub` of them; its meta is written
    // by the column-0 warp of the strip's first quadrant
    const int SUB = CS >= kM ? 1 : kM / CS;
    const int sub = CS >= kM ? 0 : (quad * 32) / CS;
    const bool meta_writer = CS >= kM ? ew == 0 : (cb == 0 && quad == sub * (CS / 32));
    uint32_t ring_it = 0, acc_it = 0, strip_it = 0;
    const long long t_role = role_t0();
    for (;;) {
      const int r = ring_it % kRing;
      if (!mbar_wait_warp(smem_u32(&cs->unit_full[r]), (ring_it / kRing) & 1u, ctl,
                          R_EPI_WAIT_UNIT))
        break;
      const UnitInfo u = cs->ring[r];  // ordered after the acquiring wait
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&cs->unit_empty[r]));
      ++ring_it;
      if (!u.valid) {
        // no more work: pass the end marker to the selection warps (strips
        // shorter than a tile: through the slot of the tile's first strip,
        // written by that strip's warps)
        const int slot = (int)(strip_it % (uint32_t)NSL);
        if (CS >= kM || sub == 0) {
          if (mbar_wait_warp(smem_u32(&cs->strip_empty[slot]), ((strip_it / NSL) & 1u) ^ 1u,
                             ctl)) {
            if (meta_writer && lane == 0) cs->meta[slot].valid = 0;
            mbar_arrive(smem_u32(&cs->strip_full[slot]));
          }
        }
        break;
      }
      // the unit's weights.  bf16: read in place from global memory (the
      // warp's columns are contiguous in w); every lane reads the same 16
      // bytes, which costs the L1 one wavefront where a shared-memory
      // broadcast of 16 bytes costs four.  Rows past S of a last, partial
      // tile are the next batch's rows, whose scores are never used, except
      // in the last batch, whose tile reads the zero-padded copy the host
      // made in the workspace instead of reading past the end of w.  FP8: a
      // copy in shared memory of the weights folded with the query row
      // scales (positive, so relu(s*x) = s*relu(x)), zero past S.
      const int64_t wrow = (int64_t)u.b * sp.S + (int64_t)u.g * QT;
      const bool tail = u.b == sp.B - 1 && (u.g + 1) * QT > sp.S;
      const float* wsrc = (tail ? p.w_tail : p.w + wrow * H) + cb * COLS;
      if (FP8) {
        float* wq = w_s + ew * COLS;
        for (int i = lane; i < COLS; i += 32) {
          const int col = cb * COLS + i;  // column of the query tile's N columns
          float wv = 0.0f;
          if (u.g * QT + col / H < sp.S) wv = p.w[wrow * H + col] * p.s_q[wrow * H + col];
          wq[i] = wv;
        }
        __syncwarp();
        wsrc = wq;
      }
      int pos = 0, j_strip = u.kbeg;
      const int sp_chunk = p.ug.C;  // keys per chunk (a multiple of 128)
      int chunk_next = u.kbeg + sp_chunk;  // end of the current key chunk
      int chunk_idx = u.kbeg / sp_chunk;
      bool stop = false;
      for (int i = 0; i < u.ntiles || (i == 0 && u.ntiles == 0); ++i) {
        const uint32_t sit = strip_it + (uint32_t)sub;  // this warp's strip
        const int slot = (int)(sit % (uint32_t)NSL);
        if (pos == 0) {
          if (!mbar_wait_warp(smem_u32(&cs->strip_empty[slot]), ((sit / NSL) & 1u) ^ 1u, ctl,
                              R_EPI_WAIT_STRIP)) {
            stop = true;
            break;
          }
        }
        if (u.ntiles > 0) {
          const int ab = acc_it & 1;
          if (!mbar_wait_warp(smem_u32(&cs->acc_full[ab]), (acc_it >> 1) & 1u, ctl, R_EPI_WAIT_ACC)) {
            stop = true;
            break;
          }
          tc_fence_after();
          const uint32_t taddr = tmem + ((uint32_t)(quad * 32) << 16) + ab * NQ + cb * COLS;
          float2 acc[QH][NA];
#pragma unroll
          for (int ql = 0; ql < QH; ++ql)
#pragma unroll
            for (int a = 0; a < NA; ++a) acc[ql][a] = make_float2(0.0f, 0.0f);
          // 32 columns per TMEM load, two loads in flight: chunk c + 2 is read
          // while chunk c is summed
          float va[32], vb[32];
          tmem_ld32(taddr, va);
          tmem_ld32(taddr + 32, vb);
          tmem_ld_wait();
          tmem_ld_fence(va);
          tmem_ld_fence(vb);
#pragma unroll
          for (int c = 0; c < NCH; c += 2) {
            if (c + 2 >= NCH) {
              // every column of this accumulator is in registers: release it
              tc_fence_before();
              mbar_arrive(smem_u32(&cs->acc_empty[ab]));
            }
            epi_chunk<FP8, H, COLS>(c, va, wsrc, acc);
            if (c + 2 < NCH) tmem_ld32(taddr + (c + 2) * 32, va);
            epi_chunk<FP8, H, COLS>(c + 1, vb, wsrc, acc);
            if (c + 2 < NCH) {
              tmem_ld32(taddr + (c + 3) * 32, vb);
              tmem_ld_wait();
              tmem_ld_fence(va);
              tmem_ld_fence(vb);
            }
          }
          ++acc_it;
          float skj = 1.0f;
          if (FP8) {
            const int j = u.kbeg + i * kM + kl;
            skj = j < sp.T ? p.s_k[(int64_t)u.b * sp.T + j] : 0.0f;
          }
          float* st = strip + (size_t)slot * QT * CS + (size_t)cb * QH * CS + pos + kl - sub * CS;
#pragma unroll
          for (int ql = 0; ql < QH; ++ql) {
            float s = 0.0f;
#pragma unroll
            for (int a = 0; a < NA; ++a) s += acc[ql][a].x + acc[ql][a].y;
            if (FP8) s *= skj;
            st[(size_t)ql * CS] = s;
          }
        }
        pos += kM;
        // a strip ends when full, at the end of a key chunk (the selection
        // then leaves that chunk's partial list) or at the unit's last tile
        const int jt_end = u.kbeg + (i + 1) * kM;
        const bool last = (i + 1 >= u.ntiles);
        const bool chunk_end = last || jt_end == chunk_next;
        if (CS < kM) {
          // every tile ends its SUB strips; only the last can end the chunk
          if (meta_writer && lane == 0) {
            const int j0 = u.kbeg + i * kM + sub * CS;
            const int nk = max(0, min(CS, min(chunk_next, u.kend) - j0));
            cs->meta[slot] = StripMeta{1,  u.b, u.g, chunk_idx, j0, nk,
                                       (chunk_end && sub == SUB - 1) ? 1 : 0, 0u};
          }
          mbar_arrive(smem_u32(&cs->strip_full[slot]));
          strip_it += (uint32_t)SUB;
          pos = 0;
          j_strip = jt_end;
          if (chunk_end) {
            chunk_next += sp_chunk;
            ++chunk_idx;
          }
        } else if (pos >= CS || chunk_end) {
          if (meta_writer && lane == 0) {
            const int nk = max(0, min(CS, min(chunk_next, u.kend) - j_strip));
            cs->meta[slot] =
                StripMeta{1, u.b, u.g, chunk_idx, j_strip, nk, chunk_end ? 1 : 0, 0u};
          }
          mbar_arrive(smem_u32(&cs->strip_full[slot]));
          ++strip_it;
          pos = 0;
          j_strip = jt_end;
          if (chunk_end) {
            chunk_next += sp_chunk;
            ++chunk_idx;
          }
        }
      }
      if (stop) break;
    }
    if (lane == 0) role_add(ctl, R_EPI_TOTAL, t_role);
  } else {
    // ---------------------------------------------------------- selection
    sm.strip = strip;
    sm.meta = cs->meta;
    sm.full_bar = smem_u32(&cs->strip_full[0]);
    sm.empty_bar = smem_u32(&cs->strip_empty[0]);
    sm.nslot = NSL;
    select_loop(sp, sm, ctl, warp - kSelWarp0, lane);
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

template <bool FP8, int D, int H, int NQ>
static cudaError_t launch_t(const CUtensorMap& tm_q, const CUtensorMap& tm_kc,
                            const ScoreParams& p, int grid, size_t smem, cudaStream_t stream) {
  auto kern = k_score_topk<FP8, D, H, NQ>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  kern<<<grid, kThreads, smem, stream>>>(tm_q, tm_kc, p);
  return cudaGetLastError();
}

template <bool FP8, int D, int NQ>
static cudaError_t launch_h(int H, const CUtensorMap& tm_q, const CUtensorMap& tm_kc,
                            const ScoreParams& p, int grid, size_t smem, cudaStream_t stream) {
  switch (H) {
    case 8: return launch_t<FP8, D, 8, NQ>(tm_q, tm_kc, p, grid, smem, stream);
    case 16: return launch_t<FP8, D, 16, NQ>(tm_q, tm_kc, p, grid, smem, stream);
    case 32: return launch_t<FP8, D, 32, NQ>(tm_q, tm_kc, p, grid, smem, stream);
    case 64: return launch_t<FP8, D, 64, NQ>(tm_q, tm_kc, p, grid, smem, stream);
    default: return cudaErrorInvalidValue;
  }
}

template <bool FP8, int D>
static cudaError_t launch_n(int H, int nq, const CUtensorMap& tm_q, const CUtensorMap& tm_kc,
                            const ScoreParams& p, int grid, size_t smem, cudaStream_t stream) {
  if (nq == 256) return launch_h<FP8, D, 256>(H, tm_q, tm_kc, p, grid, smem, stream);
  if (nq == 128) return launch_h<FP8, D, 128>(H, tm_q, tm_kc, p, grid, smem, stream);
  return cudaErrorInvalidValue;
}

cudaError_t launch_score_topk(bool fp8, int D, int H, int nq, const CUtensorMap& tm_q,
                              const CUtensorMap& tm_kc, const ScoreParams& p, int grid,
                              size_t smem, cudaStream_t stream) {
  if (fp8) {
    if (D == 128) return launch_n<true, 128>(H, nq, tm_q, tm_kc, p, grid, smem, stream);
    if (D == 64) return launch_n<true, 64>(H, nq, tm_q, tm_kc, p, grid, smem, stream);
  } else {
    if (D == 128) return launch_n<false, 128>(H, nq, tm_q, tm_kc, p, grid, smem, stream);
    if (D == 64) return launch_n<false, 64>(H, nq, tm_q, tm_kc, p, grid, smem, stream);
  }
  return cudaErrorInvalidValue;
}

// Largest score strip (keys per query) for QT queries per tile.
static int strip_max(int QT);

// Shared-memory plan for one MMA width NQ: the query tile (NQ rows), NST
// key-tile ring slots of one K-block each (kM keys x one swizzle span: a
// whole key tile when a row fits one span, half of one for bf16 at d_I =
// 128), a ring of NSL score strips of CS keys per query (cs_req and nsl_req >
// 0 fix them; CS of 32 or 64 keys, a tile's lane quadrants handed over in
// strips of their own, only when asked for, with NSL a multiple of the
// tile's 128/CS strips), the selection pools (cap keys per query), the FP8 weight copy
// and the small control block.  Candidates are ranked lexicographically: a
// pool of at least 1.5K keys first, then strips of 512 keys, then enough ring
// slots (below), then a third strip slot, then the larger pool up to 4K keys
// (a prune's cost per accepted key falls as cap / (cap - 1.2K)), then more
// strip slots, then more ring slots.  Measured with S = 262,144 and
// top-2048, the 512-key strip with one key tile in the ring beats a deeper
// ring with 128-key strips, and a third strip slot (it absorbs the
// selection's uneven pace: a prune holds one query's warp for several
// strips' worth of MMA time) beats the 256 pool keys it costs by 3%.
static ScorePlan plan_score_n(bool fp8, int D, int H, int K, int max_smem, int NQ, int cs_req,
                              int nsl_req) {
  ScorePlan best{};
  best.ok = false;
  const int esz = fp8 ? 1 : 2;
  const int QT = NQ / H;
  const int row_bytes = D * esz;
  const int sw = row_bytes >= 128 ? 128 : row_bytes;
  const int kblocks = row_bytes / sw;                  // ring slots per key tile
  const size_t q_bytes = (size_t)NQ * row_bytes;
  const size_t slot_bytes = (size_t)kM * sw;
  const size_t fixed = 1024 /* alignment slack */ + q_bytes +
                       (fp8 ? sizeof(float) * kEpiWarps * (NQ / 2) : 0) /* FP8 weight copy */ +
                       sizeof(ScoreCtlSmem);
  const int cap_min = ((K + 64 + 31) / 32) * 32;
  const int cap_max = std::max(cap_min, 4 * K);
  const int cs_max = strip_max(QT);
  // ring slots wanted: a full-width tile's MMA (1024 cycles at the dense
  // rate) hides the next tile's loads from L2 with two tiles in the ring; a
  // half-width tile's takes half as long and wants three
  const int min_slots = (NQ == kN ? 2 : 3) * kblocks;
  long best_score[7] = {-1, -1, -1, -1, -1, -1, -1};
  for (int nst = kblocks; nst <= 8; ++nst) {
    // strips shorter than a tile (32 or 64 keys) only when asked for
    for (int cs = (cs_req > 0 && cs_req < kM) ? cs_req : kM; cs <= cs_max; cs <<= 1) {
      if (cs_req > 0 && cs != cs_req) continue;
      for (int nsl = 2; nsl <= kMaxSlots; ++nsl) {
        if (nsl_req > 0 && nsl != nsl_req) continue;
        if (cs < kM && nsl % (kM / cs) != 0) continue;  // a tile's strips: whole slot groups
        const size_t used = fixed + nst * slot_bytes + sizeof(float) * (size_t)nsl * QT * cs;
        if (used + sel_state_bytes(QT, cap_min) > (size_t)max_smem) continue;
        int cap = cap_min;
        while (cap + 32 <= cap_max && used + sel_state_bytes(QT, cap + 32) <= (size_t)max_smem)
          cap += 32;
        const long sc[7] = {std::min(cap, (3 * K) / 2), std::min(cs, 512),
                            std::min(nst, min_slots), std::min(nsl, 3),
                            std::min(cap, 4 * K), nsl, nst};
        bool better = false;
        for (int i = 0; i < 7; ++i) {
          if (sc[i] != best_score[i]) {
            better = sc[i] > best_score[i];
            break;
          }
        }
        if (better) {
          for (int i = 0; i < 7; ++i) best_score[i] = sc[i];
          best.QT = QT;
          best.nq = NQ;
          best.CS = cs;
          best.nst = nst;
          best.nslot = nsl;
          best.cap = cap;
          best.smem = used + sel_state_bytes(QT, cap);
          best.ok = true;
        }
      }
    }
  }
  return best;
}

static int strip_max(int QT) { return std::min(1024, std::max(128, 4096 / QT)); }

// The full-width tile (N = 256: 256/H_I queries) is used when its pools can
// hold 1.5K keys per query: its MMA reads each key tile from shared memory
// for twice the columns of the half-width tile (N = 128), whose operand
// traffic and key-tile stream from L2 cap it well below the dense rate.  For
// larger top-k the half-width tile halves the queries per tile and so
// doubles each query's pool, which keeps pruning rare.  When every batch has
// no more queries than a half-width tile holds (a decode step), the
// half-width tile does the same work with half the MMA and epilogue columns.
ScorePlan plan_score(bool fp8, int D, int H, int K, int max_smem, int cs_req, int nsl_req,
                     int rows) {
  ScorePlan half = plan_score_n(fp8, D, H, K, max_smem, kN / 2, cs_req, nsl_req);
  if (half.ok && rows > 0 && rows <= half.QT) return half;
  const ScorePlan full = plan_score_n(fp8, D, H, K, max_smem, kN, cs_req, nsl_req);
  if (full.ok && full.cap >= (3 * K) / 2) return full;
  if (half.ok && (!full.ok || half.cap > full.cap)) return half;
  if (full.ok) return full;
  half.ok = false;
  half.err = (cs_req > strip_max(kN / H) && cs_req > strip_max(kN / 2 / H)) ? 2 : 1;
  return half;
}

}  // namespace si
