// Device-side building blocks shared by the indexer kernels (sm_100a only).
//
// * the total order used for selection: score descending, then key index
//   ascending, with -0 and +0 equal ("StreamIndex: Memory-Bounded Compressed
//   Sparse Attention via Streaming Top-k", Abstract: the top-k keys per query),
//   packed into one 64-bit key so that a larger key is a better entry;
// * bounded mbarrier waits that give up after a time limit, record an error
//   word and raise a CTA-wide abort flag instead of spinning forever;
// * thin inline-PTX wrappers for TMA, mbarrier and tcgen05 (TMEM, UMMA).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#define SI_DEV __device__ __forceinline__

// Device error word bits (read back by si_get_last_device_error).
#define SI_DEVERR_TIMEOUT 1u
#define SI_DEVERR_BAD_STATE 2u

namespace si {

// ------------------------------------------------------------------ keys
// Order-preserving map of an fp32 score to uint32 (larger score -> larger
// value), with -0 folded into +0 so the two compare equal.
SI_DEV uint32_t score_ord(float s) {
  uint32_t u = __float_as_uint(s);
  if ((u & 0x7FFFFFFFu) == 0u) u = 0u;
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// key = ord(score) << 32 | (0x7FFFFFFF - j) << 1 | (score is -0).
// Distinct j give distinct keys; a larger key ranks first.  The low bit only
// remembers the sign of a zero score so the output keeps the exact bits; it
// never decides an order because the index field above it differs.  Key 0 is
// "empty" and ranks below every real entry.
SI_DEV uint64_t make_key(float s, int j) {
  uint32_t negz = (__float_as_uint(s) == 0x80000000u) ? 1u : 0u;
  return ((uint64_t)score_ord(s) << 32) | ((uint32_t)(0x7FFFFFFF - j) << 1) | negz;
}

SI_DEV float key_score(uint64_t k) {
  uint32_t o = (uint32_t)(k >> 32);
  uint32_t u = (o & 0x80000000u) ? (o & 0x7FFFFFFFu) : ~o;
  if (k & 1ull) u = 0x80000000u;
  return __uint_as_float(u);
}

SI_DEV int key_index(uint64_t k) { return 0x7FFFFFFF - (int)((uint32_t)k >> 1); }

// ------------------------------------------------------------------ control
// Per-CTA role counters of a profiling build (compiled with SI_ROLE_CLOCKS):
// cycles each role spends in total, waiting on each barrier and in each
// selection phase, and event counts.  They cost nothing in the normal build.
enum RoleSlot {
  R_PROD_TOTAL = 0, R_PROD_WAIT_KC, R_PROD_WAIT_Q, R_PROD_WAIT_UNIT,
  R_MMA_TOTAL, R_MMA_WAIT_KC, R_MMA_WAIT_ACC, R_MMA_WAIT_Q, R_MMA_WAIT_UNIT,
  R_EPI_TOTAL, R_EPI_WAIT_UNIT, R_EPI_WAIT_STRIP, R_EPI_WAIT_ACC,
  R_SEL_TOTAL, R_SEL_WAIT_STRIP, R_SEL_INTAKE, R_SEL_UNIT_END, R_SEL_PRUNE_CYC,
  R_SEL_PRUNES, R_SEL_SHRINKS, R_SEL_APPENDS, R_SEL_STRIPS, R_SEL_END_WAIT,
  R_UNITS, R_TILES, R_SEL_KEYS, kRoleSlots = 32
};

struct Ctl {
  uint32_t* err;             // global error word
  volatile uint32_t* abort;  // CTA-wide abort flag in shared memory
  uint64_t timeout_ns;       // limit for any single wait
  unsigned long long* role;  // [grid][kRoleSlots] counters (profiling build), else null
};

SI_DEV long long role_t0() {
#ifdef SI_ROLE_CLOCKS
  return clock64();
#else
  return 0;
#endif
}
// Add the cycles since t0 to a role counter (lane 0 of a warp, or a single thread).
SI_DEV void role_add(const Ctl& c, int slot, long long t0) {
#ifdef SI_ROLE_CLOCKS
  if (slot >= 0 && c.role)
    atomicAdd(&c.role[blockIdx.x * kRoleSlots + slot], (unsigned long long)(clock64() - t0));
#else
  (void)c, (void)slot, (void)t0;
#endif
}
SI_DEV void role_count(const Ctl& c, int slot, unsigned long long v) {
#ifdef SI_ROLE_CLOCKS
  if (c.role) atomicAdd(&c.role[blockIdx.x * kRoleSlots + slot], v);
#else
  (void)c, (void)slot, (void)v;
#endif
}

SI_DEV uint64_t globaltimer() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

SI_DEV void raise_abort(const Ctl& c, uint32_t bits) {
  atomicOr(c.err, bits);
  *c.abort = 1u;
}

SI_DEV uint32_t smem_u32(const void* p) { return (uint32_t)__cvta_generic_to_shared(p); }

// ------------------------------------------------------------------ mbarrier
SI_DEV void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}
SI_DEV void mbar_fence_init() { asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory"); }
SI_DEV void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}
SI_DEV void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
               : "memory");
}
// try_wait with a suspend-time hint: a thread whose phase is not complete
// may sleep (up to ~20 us, or until the phase completes) instead of spinning,
// leaving issue slots to the warps that share its scheduler.
SI_DEV bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity), "r"(20000u)
      : "memory");
  return ok != 0u;
}

// Wait for the phase with the given parity to complete.  Returns false if the
// CTA is aborting or the wait exceeded the time limit (then it raises abort).
// A profiling build adds the wait's cycles to role counter `slot` (if >= 0).
SI_DEV bool mbar_wait_(uint32_t bar, uint32_t parity, const Ctl& c);
SI_DEV bool mbar_wait(uint32_t bar, uint32_t parity, const Ctl& c, int slot = -1) {
#ifdef SI_ROLE_CLOCKS
  const long long t = role_t0();
  const bool r = mbar_wait_(bar, parity, c);
  role_add(c, slot, t);
  return r;
#else
  (void)slot;
  return mbar_wait_(bar, parity, c);
#endif
}
SI_DEV bool mbar_wait_(uint32_t bar, uint32_t parity, const Ctl& c) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer();
  uint32_t n = 0;
  while (!mbar_try_wait(bar, parity)) {
    if ((++n & 15u) == 0u) {
      if (*c.abort) return false;
      if (globaltimer() - t0 > c.timeout_ns) {
        raise_abort(c, SI_DEVERR_TIMEOUT);
        return false;
      }
    }
  }
  return true;
}

// Warp-collective form: every lane returns the same answer, so the warp can
// go on to warp-synchronous code (shuffles, __syncwarp) without diverging.
// Each lane performs its own acquiring try_wait before it returns true.
SI_DEV bool mbar_wait_warp_(uint32_t bar, uint32_t parity, const Ctl& c);
SI_DEV bool mbar_wait_warp(uint32_t bar, uint32_t parity, const Ctl& c, int slot = -1) {
#ifdef SI_ROLE_CLOCKS
  const long long t = role_t0();
  const bool r = mbar_wait_warp_(bar, parity, c);
  if ((threadIdx.x & 31u) == 0u) role_add(c, slot, t);
  return r;
#else
  (void)slot;
  return mbar_wait_warp_(bar, parity, c);
#endif
}
SI_DEV bool mbar_wait_warp_(uint32_t bar, uint32_t parity, const Ctl& c) {
  const uint32_t lane = threadIdx.x & 31u;
  uint64_t t0 = 0;
  for (uint32_t n = 0;; ++n) {
    const bool ok = mbar_try_wait(bar, parity);
    if (__all_sync(0xFFFFFFFFu, ok)) return true;
    if ((n & 15u) == 15u) {
      int stop = 0;
      if (lane == 0) {
        if (t0 == 0) t0 = globaltimer();
        if (*c.abort) {
          stop = 1;
        } else if (globaltimer() - t0 > c.timeout_ns) {
          raise_abort(c, SI_DEVERR_TIMEOUT);
          stop = 1;
        }
      }
      if (__shfl_sync(0xFFFFFFFFu, stop, 0)) return false;
    }
  }
}

// Named barrier among a subset of warps (ids 1..15; 0 is __syncthreads).
SI_DEV void named_bar_sync(uint32_t id, uint32_t nthreads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

// ------------------------------------------------------------------ TMA
SI_DEV void tma_load_2d(uint32_t dst, const CUtensorMap* map, uint32_t bar, int c0, int c1,
                        uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      ".L2::cache_hint [%0], [%1, {%3, %4}], [%2], %5;" ::"r"(dst),
      "l"(map), "r"(bar), "r"(c0), "r"(c1), "l"(policy)
      : "memory");
}
// Start moving one tile towards L2 (no shared-memory destination, no
// completion to wait for).
SI_DEV void tma_prefetch_l2_2d(const CUtensorMap* map, int c0, int c1) {
  asm volatile("cp.async.bulk.prefetch.tensor.2d.L2.global.tile [%0, {%1, %2}];" ::"l"(map),
               "r"(c0), "r"(c1)
               : "memory");
}
SI_DEV void tma_prefetch_desc(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(map) : "memory");
}
SI_DEV uint64_t policy_evict_first() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
  return p;
}
SI_DEV uint64_t policy_evict_last() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(p));
  return p;
}

// ------------------------------------------------------------------ tcgen05
SI_DEV void tmem_alloc(uint32_t dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_smem),
               "r"(ncols)
               : "memory");
}
SI_DEV void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
SI_DEV void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}
SI_DEV void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
SI_DEV void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// D[tmem] (+)= A[smem] * B[smem]^T, both K-major, cta_group::1.
SI_DEV void umma_bf16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                      uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}
SI_DEV void umma_f8(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                    uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// Arrive once on an mbarrier when all previously issued tcgen05 ops complete.
SI_DEV void umma_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   bar)
               : "memory");
}

// 32 lanes x 32 bits, 32 consecutive columns per thread.
SI_DEV void tmem_ld32(uint32_t taddr, float (&v)[32]) {
  uint32_t* r = reinterpret_cast<uint32_t*>(v);
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
        "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
        "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr)
      : "memory");
}
SI_DEV void tmem_ld_wait() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// Shared-memory matrix descriptor for a K-major operand tile stored with the
// 128-byte swizzle: rows of 128 bytes, 8-row groups 1024 bytes apart.
// Fields: start address >> 4 (bits 0-13), leading byte offset >> 4 = 1
// (bits 16-29, unused by this layout), stride byte offset >> 4 = 64 (bits
// 32-45), descriptor version 1 (bits 46-47), swizzle mode 2 = 128B (bits 61-63).
SI_DEV uint64_t sdesc_sw128(uint32_t saddr) {
  return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)1u << 16) | ((uint64_t)64u << 32) |
         ((uint64_t)1u << 46) | ((uint64_t)2u << 61);
}

// Instruction descriptor: dense, D = f32, A/B K-major, M and N given.
// a_fmt/b_fmt: kind::f16 -> 1 = bf16; kind::f8f6f4 -> 0 = e4m3.
__host__ __device__ constexpr uint32_t idesc_make(uint32_t a_fmt, uint32_t b_fmt, uint32_t M,
                                                  uint32_t N) {
  return (1u << 4) | (a_fmt << 7) | (b_fmt << 10) | ((N >> 3) << 17) | ((M >> 4) << 24);
}

}  // namespace si
