// The C ABI (include/streamindex.h): argument checks, workspace plan, tensor
// maps and the chunked partition-merge driver loop.
//
// Driver ("StreamIndex: Memory-Bounded Compressed Sparse Attention via
// Streaming Top-k", Abstract: a chunked partition-merge top-k driver that never
// materialises the full score tensor).  Keys are split into chunks of
// key_chunk keys; each (query tile, key chunk) unit leaves a sorted partial
// list; the merge kernel folds them.  To keep the scratch bounded
// independently of S, query tiles are processed in blocks sized so that one
// block's partial lists fit the scratch budget: one score launch and one merge
// launch per block; a row-sort launch orders the whole output at the end.
// With key_chunk = 0 a single chunk covers each query's keys.
#include <cudaTypedefs.h>

#include <algorithm>
#include <mutex>

#include "streamindex.h"
#include "si_kernels.h"

namespace si {

__device__ uint32_t g_err_word;

#ifdef SI_ROLE_CLOCKS
// role counters of the profiling build: [CTA][kRoleSlots]
constexpr int kRoleCtas = 1024;
__device__ unsigned long long g_role_cycles[kRoleCtas * kRoleSlots];
#endif

namespace {

struct DevInfo {
  bool init = false;
  bool ok = false;
  int sms = 0;
  int max_smem = 0;
  uint32_t* err = nullptr;
  unsigned long long* role = nullptr;  // profiling build: role counters
};

std::mutex g_mu;
DevInfo g_dev[64];
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;

int dev_info(DevInfo** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return SI_ERR_CUDA;
  std::lock_guard<std::mutex> lk(g_mu);
  DevInfo& d = g_dev[dev];
  if (!d.init) {
    int major = 0, minor = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&d.max_smem, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) !=
            cudaSuccess)
      return SI_ERR_CUDA;
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_err_word) != cudaSuccess) return SI_ERR_CUDA;
    d.err = static_cast<uint32_t*>(p);
#ifdef SI_ROLE_CLOCKS
    void* r = nullptr;
    if (cudaGetSymbolAddress(&r, g_role_cycles) != cudaSuccess) return SI_ERR_CUDA;
    d.role = static_cast<unsigned long long*>(r);
#endif
    d.ok = (major == 10 && minor == 0);
    d.init = true;
  }
  if (!g_encode) {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) !=
            cudaSuccess ||
        q != cudaDriverEntryPointSuccess || !fn)
      return SI_ERR_CUDA;
    g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  }
  if (!d.ok) return SI_ERR_UNSUPPORTED;
  *out = &d;
  return SI_OK;
}

// Shared memory and SM count to plan with: the current device's, or the
// sm_100 limits (227 KB of opt-in shared memory per CTA, 148 SMs) on a host
// with no usable device.  Used by the plan query only.
void plan_limits(int* max_smem, int* sms) {
  DevInfo* dev = nullptr;
  if (dev_info(&dev) == SI_OK) {
    *max_smem = dev->max_smem;
    *sms = dev->sms;
  } else {
    *max_smem = 227 * 1024;
    *sms = 148;
  }
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Keys a query at sequence position t sees: min(T, (t+1)/m).
int visible_host(int t, int T, int m) {
  const int v = (int)(((int64_t)t + 1) / m);
  return v < T ? v : T;
}
size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

// 2-D row-major [rows, cols] tensor map with a {box_inner, box_rows} box and
// the given swizzle; out-of-range rows read as zero.
int make_map(CUtensorMap* m, const void* base, CUtensorMapDataType dt, uint64_t rows,
             uint64_t cols, uint32_t esz, uint32_t box_inner, uint32_t box_rows,
             CUtensorMapSwizzle sw) {
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols * esz};
  cuuint32_t box[2] = {box_inner, box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = g_encode(m, dt, 2, const_cast<void*>(base), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? SI_OK : SI_ERR_CUDA;
}

struct Opts {
  int key_chunk, scratch_mb, grid_ctas, timeout_ms, debug_flags, row_finish, key_tile,
      strip_slots;
  cudaEvent_t ev_begin, ev_end;
  cudaEvent_t* ev_list;  // [2i], [2i+1] around query block i's score launch
  int ev_count;
  int plan_heads, plan_dim, plan_fp8;  // si_topk_scores: the fused kernel's plan
};

int read_opts(const si_options* o, Opts* out) {
  Opts d{0, 512, 0, 2000, 0, 0, 0, 0, nullptr, nullptr, nullptr, 0, 0, 0, 0};
  if (o) {
    d.ev_list = reinterpret_cast<cudaEvent_t*>(o->score_event_list);
    d.ev_count = o->score_event_list ? o->score_event_count : 0;
    d.plan_heads = o->plan_heads;
    d.plan_dim = o->plan_dim;
    d.plan_fp8 = o->plan_fp8;
    d.row_finish = o->row_finish;
    d.key_tile = o->key_tile;
    d.strip_slots = o->strip_slots;
    d.ev_begin = static_cast<cudaEvent_t>(o->score_events[0]);
    d.ev_end = static_cast<cudaEvent_t>(o->score_events[1]);
    d.key_chunk = o->key_chunk;
    d.scratch_mb = o->scratch_mb > 0 ? o->scratch_mb : 512;
    d.grid_ctas = o->grid_ctas;
    d.timeout_ms = o->timeout_ms > 0 ? o->timeout_ms : 2000;
    d.debug_flags = o->debug_flags;
  }
  if (d.key_chunk < 0 || (d.key_chunk % 128) != 0 || d.grid_ctas < 0 || d.scratch_mb > (1 << 20) ||
      d.row_finish < 0 || d.row_finish > 2 ||
      !(d.key_tile == 0 || d.key_tile == 32 || d.key_tile == 64 || d.key_tile == 128 ||
        d.key_tile == 256 || d.key_tile == 512 || d.key_tile == 1024) ||
      d.strip_slots < 0 || d.strip_slots == 1 || d.strip_slots > 4 || d.ev_count < 0 ||
      // strips shorter than a 128-key tile: each tile fills 128/key_tile
      // strips, each in a slot of its own
      (d.key_tile == 32 && d.strip_slots != 0 && d.strip_slots != 4) ||
      (d.key_tile == 64 && d.strip_slots == 3) ||
      !(d.plan_heads == 0 || d.plan_heads == 8 || d.plan_heads == 16 || d.plan_heads == 32 ||
        d.plan_heads == 64) ||
      (d.plan_heads > 0 && !(d.plan_dim == 64 || d.plan_dim == 128)) || d.plan_fp8 < 0 ||
      d.plan_fp8 > 1)
    return SI_ERR_OPTIONS;
  *out = d;
  return SI_OK;
}

// The plan of one problem: tiles, chunks and query blocks.  With several key
// chunks every (tile, chunk) unit leaves an L-key partial list per query; the
// query tiles of one launch block share a scratch of B * tb * nch_max * QT * L
// keys, sized to the scratch budget, so the scratch does not grow with S.
// With one chunk per tile (final_rows) the selection warps write the output
// rows themselves: no partial lists, one launch block, no merge.
struct Plan {
  int QT, G, T, C, nch_max, L, tb, n_blocks, final_rows;
  size_t counters_bytes, tail_bytes, partial_bytes;
  // unit counter | padded copy of the last query tile's weights | partial lists
  size_t ws_bytes() const { return align256(counters_bytes) + align256(tail_bytes) + partial_bytes; }
};

Plan make_plan(int B, int S, int T, int K, int QT, int H, const Opts& o) {
  Plan p{};
  p.QT = QT;
  p.T = T;
  p.G = (S + QT - 1) / QT;
  const int tround = ((T > 0 ? T : 1) + 127) / 128 * 128;
  p.C = o.key_chunk > 0 ? o.key_chunk : tround;
  p.nch_max = T > 0 ? (T + p.C - 1) / p.C : 1;
  if (p.nch_max < 1) p.nch_max = 1;
  p.L = partial_len(K);
  // rows finished in the fused kernel only on request: its four selection
  // warps per SM finish rows far slower than the bucket-sort kernel, which
  // spreads that work over the whole GPU (the choice for 0)
  p.final_rows = (p.nch_max == 1 && o.row_finish == 1) ? 1 : 0;
  if (p.final_rows) {
    p.tb = p.G;
    p.partial_bytes = 0;
    p.n_blocks = 1;
  } else {
    const size_t per_tile = (size_t)B * p.nch_max * QT * p.L * sizeof(uint64_t);
    const size_t budget = (size_t)o.scratch_mb << 20;
    size_t tb = budget / per_tile;
    if (tb < 1) tb = 1;
    if (tb > (size_t)p.G) tb = p.G;
    p.tb = (int)tb;
    p.partial_bytes = per_tile * p.tb;
    p.n_blocks = (p.G + p.tb - 1) / p.tb;
  }
  p.counters_bytes = sizeof(int);  // one unit counter shared by every launch
  p.tail_bytes = (size_t)QT * H * sizeof(float);  // one query tile's weights (0: none)
  return p;
}

// The rows of a query block: the bucket-sort kernel when a query's candidate
// lists (one per key chunk) hold at most kFinishMaxKeys keys together, else
// the merge kernel over the chunks.
cudaError_t finish_launch(const uint64_t* partial, const SelParams& sp, const UnitGrid& ug,
                          cudaStream_t stream) {
  if (finish_takes(sp.L, sp.nch_max)) return launch_finish_rows(partial, sp, ug, stream);
  return launch_merge(partial, sp, ug, stream);
}

// True when no row-sort pass is needed after the finishing launches.
bool rows_come_sorted(const Plan& pl, int K) {
  return rows_sorted_in_warp(K) || (!pl.final_rows && finish_takes(pl.L, pl.nch_max));
}

// The selection's invariant: a pool has room for K keys plus one 64-key
// step (appends are checked step by step, and a prune or an exact select
// leaves at most cap - 64 keys), strips are whole warps of keys, and a partial
// list holds at least K keys.  Checked before every launch that runs the
// streaming selection.
bool sel_params_ok(const SelParams& sp) {
  return sp.cap >= ((sp.K + 64 + 31) / 32) * 32 && sp.CS >= 32 && sp.CS % 32 == 0 &&
         sp.L >= sp.K;
}

// Kernel launches of one call: a score launch per query block, a finishing
// launch after each unless the fused kernel finishes the rows, and the row
// sort when the rows do not come out sorted.
int plan_launches(const Plan& pl, int K) {
  return pl.n_blocks * (pl.final_rows ? 1 : 2) + (rows_come_sorted(pl, K) ? 0 : 1);
}

int plan_status(const ScorePlan& sp) {
  if (sp.ok) return SI_OK;
  return sp.err == 2 ? SI_ERR_OPTIONS : SI_ERR_TOPK;
}

// The queries and keys of one call.  Prefill: S queries per batch at
// positions 0 .. S-1, T = S/m keys, t0 = 0.  Decode: S queries per batch at
// positions t0 .. t0+S-1, against T keys.
struct Problem {
  int B, S, T, t0, m;
  bool decode;
  int tstride = 1;           // position step between query rows
  const int* vis = nullptr;  // [B*S] visible keys per row (device), replacing the rule
};

int check_common(int B, int S, int m, int topk) {
  if (B < 1 || S < 1 || m < 1 || S % m != 0) return SI_ERR_DIM;
  if (topk < 1 || topk > SI_MAX_TOPK) return SI_ERR_TOPK;
  return SI_OK;
}

// Sizes of a prefill (S % m == 0, T = S/m, t0 = 0) or decode call.
int check_problem(const Problem& pb, int H, int D, int topk) {
  if (pb.decode) {
    if (pb.B < 1 || pb.S < 1 || pb.T < 1 || pb.t0 < 0 || pb.m < 1 || pb.tstride < 1 ||
        (int64_t)pb.t0 + (int64_t)(pb.S - 1) * pb.tstride + 1 > 0x7FFFFFFF)
      return SI_ERR_DIM;
    if (topk < 1 || topk > SI_MAX_TOPK) return SI_ERR_TOPK;
  } else {
    int rc = check_common(pb.B, pb.S, pb.m, topk);
    if (rc) return rc;
  }
  if (!(H == 8 || H == 16 || H == 32 || H == 64) || !(D == 64 || D == 128)) return SI_ERR_DIM;
  if ((int64_t)pb.B * pb.S * H >= ((int64_t)1 << 31)) return SI_ERR_DIM;
  if ((int64_t)pb.B * pb.T >= ((int64_t)1 << 31)) return SI_ERR_DIM;
  return SI_OK;
}

Problem prefill(int B, int S, int m) { return Problem{B, S, m > 0 ? S / m : 0, 0, m, false}; }

// Pointers first, then sizes, then alignment.
int check_indexer(const void* q, const void* w, const void* kc, const Problem& pb, int H, int D,
                  int topk, const void* oi, const void* os) {
  if (!q || !w || !kc || !oi || !os) return SI_ERR_NULL;
  int rc = check_problem(pb, H, D, topk);
  if (rc) return rc;
  if (!aligned16(q) || !aligned16(w) || !aligned16(kc) || !aligned16(oi) || !aligned16(os))
    return SI_ERR_ALIGN;
  return SI_OK;
}

// Default key chunk of a decode call (0: one chunk per query tile).  With
// fewer query tiles than SMs a tile's keys are split into chunks, so that
// (tile, chunk) units fill the GPU; the chunk count minimises the rounds of
// units times the chunk length, charging each chunk about 256 keys' worth of
// fixed cost (its query-tile load and its partial list).
int decode_key_chunk(const Problem& pb, int QT, int sms) {
  const int64_t tiles = (int64_t)pb.B * ((pb.S + QT - 1) / QT);
  if (pb.vis) return 0;  // per-row counts: tile units, one chunk
  const int vmax = visible_host(pb.t0 + (pb.S - 1) * pb.tstride, pb.T, pb.m);
  if (vmax <= 128 || tiles >= sms) return 0;
  int best_c = 0;
  int64_t best_cost = -1;
  for (int nch = 1; nch <= 64; ++nch) {
    const int c = ((vmax + nch - 1) / nch + 127) / 128 * 128;
    const int64_t n = (vmax + c - 1) / c;
    const int64_t rounds = (tiles * n + sms - 1) / sms;
    const int64_t cost = rounds * (c + 256);
    if (best_cost < 0 || cost < best_cost) {
      best_cost = cost;
      best_c = n == 1 ? 0 : c;
    }
  }
  return best_c;
}

Plan plan_for(const Problem& pb, int K, int QT, int H, const Opts& o, int sms) {
  Opts oc = o;
  if (pb.decode && oc.key_chunk == 0) oc.key_chunk = decode_key_chunk(pb, QT, sms);
  return make_plan(pb.B, pb.S, pb.T, K, QT, H, oc);
}

int run_indexer(bool fp8, const void* q, const float* s_q, const float* w, const void* kc,
                const float* s_k, const Problem& pb, int H, int D, int K, int32_t* out_idx,
                float* out_score, const si_options* opt, void* ws, size_t ws_bytes,
                cudaStream_t stream) {
  const int B = pb.B, S = pb.S, m = pb.m;
  int rc = check_indexer(q, w, kc, pb, H, D, K, out_idx, out_score);
  if (rc) return rc;
  if (fp8 && (!s_q || !s_k)) return SI_ERR_NULL;
  Opts o;
  if ((rc = read_opts(opt, &o))) return rc;
  DevInfo* dev;
  if ((rc = dev_info(&dev))) return rc;
  const ScorePlan sp_plan =
      plan_score(fp8, D, H, K, dev->max_smem, o.key_tile, o.strip_slots, pb.S);
  if ((rc = plan_status(sp_plan))) return rc;  // pools of this topk do not fit, or key_tile
  const Plan pl = plan_for(pb, K, sp_plan.QT, H, o, dev->sms);
  if (!ws || ws_bytes < pl.ws_bytes()) return SI_ERR_WORKSPACE;
  if (!aligned16(ws)) return SI_ERR_ALIGN;

  int* counters = static_cast<int*>(ws);
  float* w_tail = reinterpret_cast<float*>(static_cast<char*>(ws) + align256(pl.counters_bytes));
  uint64_t* partial = reinterpret_cast<uint64_t*>(reinterpret_cast<char*>(w_tail) +
                                                  align256(pl.tail_bytes));
  if (cudaMemsetAsync(counters, 0, pl.counters_bytes, stream) != cudaSuccess) return SI_ERR_CUDA;
  // the last batch's last query tile, when S is not a multiple of its
  // queries, gets a zero-padded copy of its rows of w to read (bf16 path)
  if (!fp8 && S % pl.QT != 0) {
    const int valid = S % pl.QT;
    const int64_t row0 = (int64_t)(B - 1) * S + (int64_t)(pl.G - 1) * pl.QT;
    if (cudaMemsetAsync(w_tail, 0, (size_t)pl.QT * H * sizeof(float), stream) != cudaSuccess ||
        cudaMemcpyAsync(w_tail, w + row0 * H, (size_t)valid * H * sizeof(float),
                        cudaMemcpyDeviceToDevice, stream) != cudaSuccess)
      return SI_ERR_CUDA;
  }

  const int esz = fp8 ? 1 : 2;
  const int row_bytes = D * esz;
  const int sw_bytes = row_bytes >= 128 ? 128 : row_bytes;
  const CUtensorMapSwizzle sw =
      sw_bytes == 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B;
  const CUtensorMapDataType dt =
      fp8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  CUtensorMap tm_q, tm_kc;
  const int T = pl.T;
  if ((rc = make_map(&tm_q, q, dt, (uint64_t)B * S * H, D, esz, sw_bytes / esz, sp_plan.nq, sw)))
    return rc;
  if ((rc = make_map(&tm_kc, kc, dt, (uint64_t)B * (T > 0 ? T : 1), D, esz, sw_bytes / esz, 128,
                     sw)))
    return rc;

  // Every CTA takes units until one decode fails, so a launch advances the
  // shared counter by exactly (its units + its grid).
  int id_base = 0;
  for (int blk = 0; blk < pl.n_blocks; ++blk) {
    const int g_lo = blk * pl.tb;
    const int n_tiles = pl.G - g_lo < pl.tb ? pl.G - g_lo : pl.tb;
    // a prefill's tiles outnumber the SMs: a unit is a whole tile (loaded
    // once, its chunks in order); a decode step's few tiles are split into
    // (tile, chunk) units that spread over the SMs
    UnitGrid ug{B,        S,       T,         m,        pl.QT,    pl.C,    g_lo,
                n_tiles,  id_base, (pb.decode && !pb.vis) ? 0 : 1, pb.t0, pb.tstride, pb.vis};
    ScoreParams p{};
    p.sel = SelParams{B,      S,         T,           m,       K,         pl.QT,
                      sp_plan.CS, sp_plan.cap, pl.L, g_lo, n_tiles, pl.nch_max,
                      out_idx, out_score, partial, pl.final_rows, pb.t0, pb.tstride, pb.vis};
    p.ug = ug;
    p.w = w;
    p.w_tail = w_tail;
    p.s_q = s_q;
    p.s_k = s_k;
    p.counter = counters;
    p.err = dev->err;
    p.timeout_ns = (uint64_t)o.timeout_ms * 1000000ull;
    p.nst = sp_plan.nst;
    p.nslot = sp_plan.nslot;
    p.debug_flags = o.debug_flags;
    p.role = dev->role;
    if (!sel_params_ok(p.sel)) return SI_ERR_TOPK;
    const int units = host_count_units(ug);
    int grid = o.grid_ctas > 0 ? o.grid_ctas : dev->sms;
    if (grid > units) grid = units;
    if (grid < 1) grid = 1;
    if (blk == 0 && o.ev_begin && cudaEventRecord(o.ev_begin, stream) != cudaSuccess)
      return SI_ERR_CUDA;
    const bool blk_ev = o.ev_list && 2 * blk + 1 < o.ev_count;
    if (blk_ev && cudaEventRecord(o.ev_list[2 * blk], stream) != cudaSuccess) return SI_ERR_CUDA;
    if (launch_score_topk(fp8, D, H, sp_plan.nq, tm_q, tm_kc, p, grid, sp_plan.smem,
                          stream) !=
        cudaSuccess)
      return SI_ERR_CUDA;
    if (blk_ev && cudaEventRecord(o.ev_list[2 * blk + 1], stream) != cudaSuccess)
      return SI_ERR_CUDA;
    if (blk + 1 == pl.n_blocks && o.ev_end && cudaEventRecord(o.ev_end, stream) != cudaSuccess)
      return SI_ERR_CUDA;
    id_base += units + grid;
    if (!pl.final_rows && finish_launch(partial, p.sel, ug, stream) != cudaSuccess)
      return SI_ERR_CUDA;
  }
  // rows of more than 512 keys are written unsorted; order them
  if (!rows_come_sorted(pl, K) &&
      launch_sort_rows(out_idx, out_score, (int64_t)B * S, K, dev->sms, stream) != cudaSuccess)
    return SI_ERR_CUDA;
  return SI_OK;
}

int workspace_for(const Problem& pb, int H, int D, int K, const si_options* opt, size_t* bytes) {
  int rc = check_problem(pb, H, D, K);
  if (rc) return rc;
  Opts o;
  if ((rc = read_opts(opt, &o))) return rc;
  int max_smem = 0, sms = 0;
  plan_limits(&max_smem, &sms);
  // the larger need of the two query-tile widths the score plan may choose
  const Plan full = plan_for(pb, K, 256 / H, H, o, sms);
  const Plan half = plan_for(pb, K, 128 / H, H, o, sms);
  *bytes = std::max(full.ws_bytes(), half.ws_bytes());
  return SI_OK;
}

// ------------------------------------------------------------ fixed scratch
// Device scratch for si_indexer_topk_noalloc: a file-scope array, so the call
// needs no allocation.  Every GPU that loads the library holds it until exit.
constexpr size_t kNoAllocScratchBytes = SI_NOALLOC_SCRATCH_BYTES;
static __device__ __align__(256) uint8_t g_noalloc_scratch[kNoAllocScratchBytes];

std::mutex g_noalloc_mu;
void* g_noalloc_ptr[64] = {};

// Device address of the fixed scratch on the current device.  In host code
// the array's name is only a host-side stand-in, so the address is looked up
// once per device (with that device current) and cached.
int noalloc_scratch(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return SI_ERR_CUDA;
  std::lock_guard<std::mutex> lk(g_noalloc_mu);
  if (!g_noalloc_ptr[dev]) {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_noalloc_scratch) != cudaSuccess || !ptr) return SI_ERR_CUDA;
    g_noalloc_ptr[dev] = ptr;
  }
  *out = g_noalloc_ptr[dev];
  return SI_OK;
}

}  // namespace

// ------------------------------------------------------------ unit counting
static int host_tile_vmax(const UnitGrid& u, int g) {
  int t = g * u.QT + u.QT - 1;
  if (t > u.S - 1) t = u.S - 1;
  return visible_host(u.t0 + t * u.tstride, u.T, u.m);
}

int host_tile_chunks(const UnitGrid& u, int g) {
  const int v = host_tile_vmax(u, g);
  return v <= 0 ? 1 : (v + u.C - 1) / u.C;
}

int host_count_units(const UnitGrid& u) {
  if (u.tile_units) return u.B * u.n_tiles;
  int64_t n = 0;
  for (int g = u.g_lo; g < u.g_lo + u.n_tiles; ++g) n += host_tile_chunks(u, g);
  n *= u.B;
  return n > 0x7FFFFFFF ? 0x7FFFFFFF : (int)n;
}

}  // namespace si

using namespace si;

// The plan of a prefill or decode call, as si_plan_info.
static int plan_info(const Problem& pb, int H, int D, int topk, int fp8, const si_options* opt,
              si_plan_info* out) {
  if (!out) return SI_ERR_NULL;
  int rc = check_problem(pb, H, D, topk);
  if (rc) return rc;
  if (fp8 < 0 || fp8 > 1) return SI_ERR_OPTIONS;
  Opts o;
  if ((rc = read_opts(opt, &o))) return rc;
  int max_smem = 0, sms = 0;
  plan_limits(&max_smem, &sms);
  const ScorePlan sp =
      plan_score(fp8 != 0, D, H, topk, max_smem, o.key_tile, o.strip_slots, pb.S);
  if ((rc = plan_status(sp))) return rc;
  const Plan pl = plan_for(pb, topk, sp.QT, H, o, sms);
  si_plan_info r{};
  r.queries_per_tile = sp.QT;
  r.mma_n = sp.nq;
  r.key_tile = sp.CS;
  r.stages = sp.nst;
  r.strip_slots = sp.nslot;
  r.pool_keys = sp.cap;
  r.partial_len = pl.L;
  r.key_chunks = pl.nch_max;
  r.query_blocks = pl.n_blocks;
  r.launches = plan_launches(pl, topk);
  r.workspace_bytes = pl.ws_bytes();
  r.smem_bytes = sp.smem;
  *out = r;
  return SI_OK;
}

extern "C" {

int si_version(void) { return 100; }

const char* si_status_string(int s) {
  switch (s) {
    case SI_OK: return "ok";
    case SI_ERR_NULL: return "a required pointer is NULL";
    case SI_ERR_DIM: return "a dimension is out of range";
    case SI_ERR_TOPK: return "topk out of range (1..2048)";
    case SI_ERR_ALIGN: return "a pointer is not 16-byte aligned";
    case SI_ERR_WORKSPACE: return "workspace too small";
    case SI_ERR_CUDA: return "a CUDA call or kernel launch failed";
    case SI_ERR_DEVICE_TIMEOUT: return "a kernel gave up on a bounded wait";
    case SI_ERR_OPTIONS: return "an option is out of range";
    case SI_ERR_UNSUPPORTED: return "no sm_100 device";
    default: return "unknown status";
  }
}

int si_indexer_topk_workspace_size(int B, int S, int H_I, int d_I, int m, int topk,
                                   const si_options* opt, size_t* bytes) {
  if (!bytes) return SI_ERR_NULL;
  return workspace_for(prefill(B, S, m), H_I, d_I, topk, opt, bytes);
}

int si_indexer_topk_plan(int B, int S, int H_I, int d_I, int m, int topk, int fp8,
                         const si_options* opt, si_plan_info* out) {
  return plan_info(prefill(B, S, m), H_I, d_I, topk, fp8, opt, out);
}

int si_indexer_topk_ex(const void* q, const float* w, const void* kc, int B, int S, int H_I,
                       int d_I, int m, int topk, int32_t* out_idx, float* out_score,
                       const si_options* opt, void* workspace, size_t ws_bytes, void* stream) {
  return run_indexer(false, q, nullptr, w, kc, nullptr, prefill(B, S, m), H_I, d_I, topk, out_idx,
                     out_score, opt, workspace, ws_bytes, static_cast<cudaStream_t>(stream));
}

int si_indexer_topk(const void* q, const float* w, const void* kc, int B, int S, int H_I, int d_I,
                    int m, int topk, int32_t* out_idx, float* out_score, void* stream) {
  size_t bytes = 0;
  int rc = si_indexer_topk_workspace_size(B, S, H_I, d_I, m, topk, nullptr, &bytes);
  if (rc) return rc;
  rc = check_indexer(q, w, kc, prefill(B, S, m), H_I, d_I, topk, out_idx, out_score);
  if (rc) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  void* ws = nullptr;
  if (cudaMallocAsync(&ws, bytes, st) != cudaSuccess) return SI_ERR_CUDA;
  rc = si_indexer_topk_ex(q, w, kc, B, S, H_I, d_I, m, topk, out_idx, out_score, nullptr, ws,
                          bytes, stream);
  if (cudaFreeAsync(ws, st) != cudaSuccess && rc == SI_OK) rc = SI_ERR_CUDA;
  return rc;
}

int si_indexer_topk_fp8(const void* q8, const float* s_q, const float* w, const void* k8,
                        const float* s_k, int B, int S, int H_I, int d_I, int m, int topk,
                        int32_t* out_idx, float* out_score, const si_options* opt,
                        void* workspace, size_t ws_bytes, void* stream) {
  return run_indexer(true, q8, s_q, w, k8, s_k, prefill(B, S, m), H_I, d_I, topk, out_idx,
                     out_score, opt,
                     workspace, ws_bytes, static_cast<cudaStream_t>(stream));
}

int si_quantize_fp8_rows(const void* x, int64_t rows, int cols, void* x8, float* scale,
                         void* stream) {
  if (!x || !x8 || !scale) return SI_ERR_NULL;
  if (rows < 0 || cols < 8 || cols > 4096 || cols % 8 != 0) return SI_ERR_DIM;
  if (!aligned16(x) || !aligned16(x8) || !aligned16(scale)) return SI_ERR_ALIGN;
  DevInfo* dev;
  int rc = dev_info(&dev);
  if (rc) return rc;
  return launch_quantize_fp8(static_cast<const uint16_t*>(x), rows, cols,
                             static_cast<uint8_t*>(x8), scale,
                             static_cast<cudaStream_t>(stream)) == cudaSuccess
             ? SI_OK
             : SI_ERR_CUDA;
}

int si_topk_scores(const float* scores, int B, int S, int T, int m, int topk, int32_t* out_idx,
                   float* out_score, const si_options* opt, void* stream) {
  if (!scores || !out_idx || !out_score) return SI_ERR_NULL;
  if (B < 1 || S < 1 || T < 1 || m < 1) return SI_ERR_DIM;
  if (topk < 1 || topk > SI_MAX_TOPK) return SI_ERR_TOPK;
  if ((int64_t)B * S * T >= ((int64_t)1 << 40)) return SI_ERR_DIM;
  if (!aligned16(scores) || !aligned16(out_idx) || !aligned16(out_score)) return SI_ERR_ALIGN;
  Opts o;
  int rc = read_opts(opt, &o);
  if (rc) return rc;
  DevInfo* dev;
  if ((rc = dev_info(&dev))) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  int QT = 4, CS = 1024;
  int cap = ((std::max(topk + 64, 2 * topk) + 31) / 32) * 32;
  if (o.plan_heads > 0) {
    // the fused kernel's selection plan for that shape: same queries per
    // tile, strip length and pool room, hence the same selection steps
    const ScorePlan fp = plan_score(o.plan_fp8 != 0, o.plan_dim, o.plan_heads, topk,
                                    dev->max_smem, o.key_tile, o.strip_slots, 0);
    if ((rc = plan_status(fp))) return rc;
    QT = fp.QT;
    CS = fp.CS;
    cap = fp.cap;
  }
  if (topk_scores_smem_bytes(QT, cap, CS) > (size_t)dev->max_smem) return SI_ERR_TOPK;
  // the selection-only path sees T keys per row; m still sets visibility
  const Plan pl = make_plan(B, S, T, topk, QT, 0, o);
  const size_t bytes = pl.ws_bytes();
  void* ws = nullptr;
  if (cudaMallocAsync(&ws, bytes, st) != cudaSuccess) return SI_ERR_CUDA;
  int* counters = static_cast<int*>(ws);
  uint64_t* partial =
      reinterpret_cast<uint64_t*>(static_cast<char*>(ws) + align256(pl.counters_bytes));
  rc = SI_OK;
  if (cudaMemsetAsync(counters, 0, pl.counters_bytes, st) != cudaSuccess) rc = SI_ERR_CUDA;
  int id_base = 0;
  for (int blk = 0; rc == SI_OK && blk < pl.n_blocks; ++blk) {
    const int g_lo = blk * pl.tb;
    const int n_tiles = pl.G - g_lo < pl.tb ? pl.G - g_lo : pl.tb;
    UnitGrid ug{B, S, T, m, QT, pl.C, g_lo, n_tiles, id_base, 0, 0, 1, nullptr};
    SelParams sp{B,    S,       T,          m,       topk,    QT,     CS,
                 cap,  pl.L,    g_lo,       n_tiles, pl.nch_max, out_idx, out_score,
                 partial, pl.final_rows, 0, 1, nullptr};
    const int units = host_count_units(ug);
    int grid = o.grid_ctas > 0 ? o.grid_ctas : dev->sms;
    if (grid > units) grid = units;
    if (grid < 1) grid = 1;
    if (!sel_params_ok(sp)) {
      rc = SI_ERR_TOPK;
      break;
    }
    if (launch_topk_scores(scores, sp, ug, counters, dev->err,
                           (uint64_t)o.timeout_ms * 1000000ull, grid, st) != cudaSuccess)
      rc = SI_ERR_CUDA;
    else if (!pl.final_rows && finish_launch(partial, sp, ug, st) != cudaSuccess)
      rc = SI_ERR_CUDA;
    id_base += units + grid;
  }
  if (rc == SI_OK && !rows_come_sorted(pl, topk) &&
      launch_sort_rows(out_idx, out_score, (int64_t)B * S, topk, dev->sms, st) != cudaSuccess)
    rc = SI_ERR_CUDA;
  if (cudaFreeAsync(ws, st) != cudaSuccess && rc == SI_OK) rc = SI_ERR_CUDA;
  return rc;
}

int si_role_cycles(uint64_t* out, int n_words, int reset) {
#ifdef SI_ROLE_CLOCKS
  if (!out && n_words > 0) return SI_ERR_NULL;
  if (n_words < 0) return SI_ERR_DIM;
  DevInfo* dev;
  int rc = dev_info(&dev);
  if (rc) return rc;
  const size_t n = std::min((size_t)n_words, (size_t)kRoleCtas * kRoleSlots);
  if (cudaDeviceSynchronize() != cudaSuccess) return SI_ERR_CUDA;
  if (n && cudaMemcpyFromSymbol(out, g_role_cycles, n * sizeof(uint64_t)) != cudaSuccess)
    return SI_ERR_CUDA;
  if (reset && cudaMemset(dev->role, 0, sizeof(g_role_cycles)) != cudaSuccess) return SI_ERR_CUDA;
  return SI_OK;
#else
  (void)out, (void)n_words, (void)reset;
  return SI_ERR_UNSUPPORTED;
#endif
}

int si_get_last_device_error(void* stream) {
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return SI_ERR_CUDA;
  uint32_t v = 0;
  if (cudaMemcpyFromSymbol(&v, g_err_word, sizeof v) != cudaSuccess) return SI_ERR_CUDA;
  const uint32_t zero = 0;
  if (cudaMemcpyToSymbol(g_err_word, &zero, sizeof zero) != cudaSuccess) return SI_ERR_CUDA;
  if (v & SI_DEVERR_TIMEOUT) return SI_ERR_DEVICE_TIMEOUT;
  return v ? SI_ERR_CUDA : SI_OK;
}

int si_indexer_topk_noalloc(const void* q, const float* w, const void* kc, int B, int S, int H_I,
                            int d_I, int m, int topk, int32_t* out_idx, float* out_score,
                            void* stream) {
  // query blocks sized to the fixed scratch (its last MiB left for the
  // counter); this size check comes first, so NULL tensors may query it
  si_options opt{};
  opt.scratch_mb = (int)(kNoAllocScratchBytes >> 20) - 1;
  size_t need = 0;
  int rc = workspace_for(prefill(B, S, m), H_I, d_I, topk, &opt, &need);
  if (rc) return rc;
  if (need > kNoAllocScratchBytes) return SI_ERR_WORKSPACE;  // one query tile does not fit
  if ((rc = check_indexer(q, w, kc, prefill(B, S, m), H_I, d_I, topk, out_idx, out_score)))
    return rc;
  void* ws = nullptr;
  if ((rc = noalloc_scratch(&ws))) return rc;
  return run_indexer(false, q, nullptr, w, kc, nullptr, prefill(B, S, m), H_I, d_I, topk, out_idx,
                     out_score, &opt, ws, kNoAllocScratchBytes, static_cast<cudaStream_t>(stream));
}

// ------------------------------------------------------------ sparse attention
int si_sparse_attention(const void* qa, const void* ka, const void* va, const int32_t* idx, int B,
                        int S, int T, int H_a, int d_a, int topk, float scale, float* out,
                        const si_options* opt, void* stream) {
  if (!qa || !ka || !va || !idx || !out) return SI_ERR_NULL;
  if (B < 1 || S < 1 || T < 1 || H_a != 128 || d_a != 128) return SI_ERR_DIM;
  if ((int64_t)B * S * H_a >= ((int64_t)1 << 31)) return SI_ERR_DIM;
  if (topk < 1 || topk > SI_MAX_TOPK) return SI_ERR_TOPK;
  if (!(scale >= 0.0f) || scale == INFINITY) return SI_ERR_OPTIONS;  // NaN fails the first test
  if (!aligned16(qa) || !aligned16(ka) || !aligned16(va) || !aligned16(out) ||
      (reinterpret_cast<uintptr_t>(idx) & 3u))
    return SI_ERR_ALIGN;
  Opts o;
  int rc = read_opts(opt, &o);
  if (rc) return rc;
  DevInfo* dev;
  if ((rc = dev_info(&dev))) return rc;
  if (sparse_attn_smem_bytes() > (size_t)dev->max_smem) return SI_ERR_UNSUPPORTED;
  CUtensorMap tm_q;
  if ((rc = make_map(&tm_q, qa, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, (uint64_t)B * S * H_a, d_a, 2,
                     64, 128, CU_TENSOR_MAP_SWIZZLE_128B)))
    return rc;
  AttnParams p{};
  p.ka = static_cast<const uint16_t*>(ka);
  p.va = static_cast<const uint16_t*>(va);
  p.idx = idx;
  p.out = out;
  p.B = B;
  p.S = S;
  p.T = T;
  p.k = topk;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.err = dev->err;
  p.timeout_ns = (uint64_t)o.timeout_ms * 1000000ull;
  const int64_t queries = (int64_t)B * S;
  int grid = o.grid_ctas > 0 ? o.grid_ctas : dev->sms;
  if (grid > queries) grid = (int)queries;
  return launch_sparse_attn(tm_q, p, grid, static_cast<cudaStream_t>(stream)) == cudaSuccess
             ? SI_OK
             : SI_ERR_CUDA;
}

// ------------------------------------------------------------ query-group scan
// Workspace of si_indexer_pivot: the group representatives' q and w, their
// top-C rows, the sorted candidates, the gathered key rows, the per-query
// visible counts, then one indexer workspace shared by the two launches.
struct PivotLayout {
  size_t qr, wr, ridx, rsc, cand, kcg, vis, iws, total;
};

static int pivot_layout(const Problem& full, int H, int D, int K, int G, int C,
                        const si_options* opt, PivotLayout* L, Problem* rep, Problem* rs) {
  int rc = check_problem(full, H, D, K);
  if (rc) return rc;
  if (G < 1 || full.S % G != 0 || C < K || C > SI_MAX_TOPK) return SI_ERR_OPTIONS;
  const int ng = full.S / G;
  const int64_t groups = (int64_t)full.B * ng;
  if (groups * C >= ((int64_t)1 << 31)) return SI_ERR_DIM;
  *rep = Problem{full.B, ng, full.T, G - 1, full.m, true, G, nullptr};
  *rs = Problem{(int)groups, G, C, 0, 1, true, 1, nullptr};
  size_t w1 = 0, w2 = 0;
  si_options o{};
  if (opt) o = *opt;
  o.key_chunk = 0;
  if ((rc = workspace_for(*rep, H, D, C, &o, &w1))) return rc;
  if ((rc = workspace_for(*rs, H, D, K, &o, &w2))) return rc;
  size_t at = 0;
  auto take = [&](size_t bytes) {
    const size_t r = at;
    at += align256(bytes);
    return r;
  };
  L->qr = take((size_t)groups * H * D * 2);
  L->wr = take((size_t)groups * H * 4);
  L->ridx = take((size_t)groups * C * 4);
  L->rsc = take((size_t)groups * C * 4);
  L->cand = take((size_t)groups * C * 4);
  L->kcg = take((size_t)groups * C * D * 2);
  L->vis = take((size_t)full.B * full.S * 4);
  L->iws = take(std::max(w1, w2));
  L->total = at;
  return SI_OK;
}

int si_indexer_pivot_workspace_size(int B, int S, int H_I, int d_I, int m, int topk, int G, int C,
                                    const si_options* opt, size_t* bytes) {
  if (!bytes) return SI_ERR_NULL;
  PivotLayout L;
  Problem rep, rs;
  const int rc = pivot_layout(prefill(B, S, m), H_I, d_I, topk, G, C, opt, &L, &rep, &rs);
  if (rc == SI_OK) *bytes = L.total;
  return rc;
}

int si_indexer_pivot(const void* q, const float* w, const void* kc, int B, int S, int H_I,
                     int d_I, int m, int topk, int G, int C, int32_t* out_idx, float* out_score,
                     const si_options* opt, void* workspace, size_t ws_bytes, void* stream) {
  const Problem full = prefill(B, S, m);
  int rc = check_indexer(q, w, kc, full, H_I, d_I, topk, out_idx, out_score);
  if (rc) return rc;
  PivotLayout L;
  Problem rep, rs;
  if ((rc = pivot_layout(full, H_I, d_I, topk, G, C, opt, &L, &rep, &rs))) return rc;
  if (!workspace || ws_bytes < L.total) return SI_ERR_WORKSPACE;
  if (!aligned16(workspace)) return SI_ERR_ALIGN;
  DevInfo* dev;
  if ((rc = dev_info(&dev))) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  char* ws = static_cast<char*>(workspace);
  uint16_t* qr = reinterpret_cast<uint16_t*>(ws + L.qr);
  float* wr = reinterpret_cast<float*>(ws + L.wr);
  int32_t* ridx = reinterpret_cast<int32_t*>(ws + L.ridx);
  float* rsc = reinterpret_cast<float*>(ws + L.rsc);
  int32_t* cand = reinterpret_cast<int32_t*>(ws + L.cand);
  uint16_t* kcg = reinterpret_cast<uint16_t*>(ws + L.kcg);
  int* vis = reinterpret_cast<int*>(ws + L.vis);
  void* iws = ws + L.iws;
  const size_t iws_bytes = L.total - L.iws;
  const PivotParams pp{B, S, S / m, H_I, d_I, m, G, C, S / G};
  si_options o{};
  if (opt) o = *opt;
  o.key_chunk = 0;
  o.score_event_list = nullptr;
  o.score_event_count = 0;
  o.score_events[0] = o.score_events[1] = nullptr;
  // 1. each group's last query scans its visible keys and keeps C
  if (launch_pivot_reps(static_cast<const uint16_t*>(q), w, pp, qr, wr, st) != cudaSuccess)
    return SI_ERR_CUDA;
  if ((rc = run_indexer(false, qr, nullptr, wr, kc, nullptr, rep, H_I, d_I, C, ridx, rsc, &o, iws,
                        iws_bytes, st)))
    return rc;
  // 2. the candidates sorted by key, their key rows, each query's visible count
  if (launch_pivot_cands(ridx, static_cast<const uint16_t*>(kc), pp, cand, kcg, vis, st) !=
      cudaSuccess)
    return SI_ERR_CUDA;
  // 3. every query ranks the candidates it sees (q and w viewed as [B*S/G, G, ...])
  rs.vis = vis;
  if ((rc = run_indexer(false, q, nullptr, w, kcg, nullptr, rs, H_I, d_I, topk, out_idx,
                        out_score, &o, iws, iws_bytes, st)))
    return rc;
  // 4. candidate positions back to key indices
  return launch_pivot_remap(out_idx, cand, pp, topk, dev->sms, st) == cudaSuccess ? SI_OK
                                                                                  : SI_ERR_CUDA;
}

// ------------------------------------------------------------ decode
int si_indexer_decode_workspace_size(int B, int S_q, int t0, int T, int H_I, int d_I, int m,
                                     int topk, const si_options* opt, size_t* bytes) {
  if (!bytes) return SI_ERR_NULL;
  return workspace_for(Problem{B, S_q, T, t0, m, true}, H_I, d_I, topk, opt, bytes);
}

int si_indexer_decode_plan(int B, int S_q, int t0, int T, int H_I, int d_I, int m, int topk,
                           const si_options* opt, si_plan_info* out) {
  return plan_info(Problem{B, S_q, T, t0, m, true}, H_I, d_I, topk, 0, opt, out);
}

int si_indexer_decode(const void* q, const float* w, const void* kc, int B, int S_q, int t0, int T,
                      int H_I, int d_I, int m, int topk, int32_t* out_idx, float* out_score,
                      const si_options* opt, void* workspace, size_t ws_bytes, void* stream) {
  return run_indexer(false, q, nullptr, w, kc, nullptr, Problem{B, S_q, T, t0, m, true}, H_I, d_I,
                     topk, out_idx, out_score, opt, workspace, ws_bytes,
                     static_cast<cudaStream_t>(stream));
}

}  // extern "C"
