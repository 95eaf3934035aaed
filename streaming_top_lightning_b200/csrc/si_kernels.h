// Internal launch interface between the C ABI (api.cu) and the kernels.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "si_select.cuh"

namespace si {

// Parameters of the fused score + select kernel.
struct ScoreParams {
  SelParams sel;
  UnitGrid ug;
  const float* w;      // [B*S, H] fp32 head weights
  const float* w_tail; // bf16: [QT, H] copy of the last batch's last query tile's
                       // rows of w, zero past S (read instead of w by that tile)
  const float* s_q;    // FP8 only: [B*S, H] query row scales
  const float* s_k;    // FP8 only: [B*T] key row scales
  int* counter;        // shared unit counter; this launch's ids start at ug.id_base
  uint32_t* err;       // device error word
  uint64_t timeout_ns; // limit of any single wait
  int nst;             // key-tile pipeline stages
  int nslot;           // strip ring slots
  int debug_flags;     // bit 0: skip the first key-tile load (timeout test)
  unsigned long long* role;  // role counters of a profiling build, else null
};

// Parameters of the sparse attention kernel (128 heads of dim 128).
struct AttnParams {
  const uint16_t* ka;  // [B*T, 128] bf16 key rows
  const uint16_t* va;  // [B*T, 128] bf16 value rows
  const int32_t* idx;  // [B*S, k] listed entries (-1: none)
  float* out;          // [B*S, 128, 128] fp32
  int B, S, T, k;
  float scale_log2;    // softmax scale times log2(e)
  uint32_t* err;       // device error word
  uint64_t timeout_ns; // limit of any single wait
};
size_t sparse_attn_smem_bytes();
cudaError_t launch_sparse_attn(const CUtensorMap& tm_q, const AttnParams& p, int grid,
                               cudaStream_t stream);

// Sizes of a query-group candidate scan (k_pivot.cu): groups of G queries,
// ng = S/G per batch, C candidates per group.
struct PivotParams {
  int B, S, T, H, D, m, G, C, ng;
};
cudaError_t launch_pivot_reps(const uint16_t* q, const float* w, const PivotParams& p,
                              uint16_t* qr, float* wr, cudaStream_t stream);
cudaError_t launch_pivot_cands(const int32_t* rep_idx, const uint16_t* kc, const PivotParams& p,
                               int32_t* cand, uint16_t* kcg, int* vis, cudaStream_t stream);
cudaError_t launch_pivot_remap(int32_t* out_idx, const int32_t* cand, const PivotParams& p, int K,
                               int sms, cudaStream_t stream);

// Shared-memory plan of the fused kernel for one problem shape.
struct ScorePlan {
  int QT;        // queries per tile (nq / H)
  int nq;        // MMA N: query-tile rows (QT * H), 256 or 128
  int CS;        // keys per score strip
  int nst;       // pipeline stages
  int nslot;     // strip ring slots
  int cap;       // selection pool entries per query
  size_t smem;   // dynamic shared memory bytes
  bool ok;
  int err;       // when !ok: 1 = the pools of this topk do not fit, 2 = cs_req
                 // above the largest strip either tile width allows
};

// cs_req: keys per score strip (128 .. 1024), nsl_req: strip ring slots
// (2 .. 4); 0 = the planner's choice.
// rows: queries per batch when known and small (0: many), see k_score_topk.cu
ScorePlan plan_score(bool fp8, int D, int H, int K, int max_smem, int cs_req, int nsl_req,
                     int rows);

cudaError_t launch_score_topk(bool fp8, int D, int H, int nq, const CUtensorMap& tm_q,
                              const CUtensorMap& tm_kc, const ScoreParams& p, int grid,
                              size_t smem, cudaStream_t stream);

size_t topk_scores_smem_bytes(int QT, int cap, int CS);
cudaError_t launch_topk_scores(const float* X, const SelParams& sp, const UnitGrid& ug,
                               int* counter, uint32_t* err, uint64_t timeout_ns, int grid,
                               cudaStream_t stream);

cudaError_t launch_merge(const uint64_t* partial, const SelParams& sp, const UnitGrid& ug,
                         cudaStream_t stream);

// True when the merge kernel already writes sorted rows (small K).
bool merge_sorts_rows(int K);

// Exact sorted rows from a single candidate list per query (one key chunk);
// every row comes out sorted, whatever K.
// The finishing kernel takes a query's one or two lists when they hold at
// most this many keys together (its shared memory, and the fallback select's
// byte counters: at most 255 * 32 keys); other sets go through the merge kernel.
constexpr int kFinishMaxKeys = 8160;
bool finish_takes(int L, int nch);
cudaError_t launch_finish_rows(const uint64_t* partial, const SelParams& sp, const UnitGrid& ug,
                               cudaStream_t stream);

// Sorts each of the rows [rows, K] of (idx, score) in place into the output
// order (score descending, index ascending, padding last).
cudaError_t launch_sort_rows(int32_t* idx, float* score, int64_t rows, int K, int sms,
                             cudaStream_t stream);

cudaError_t launch_quantize_fp8(const uint16_t* x, int64_t rows, int cols, uint8_t* x8,
                                float* scale, cudaStream_t stream);

// Number of units (query tile x key chunk x batch) in a launch.
int host_count_units(const UnitGrid& u);
int host_tile_chunks(const UnitGrid& u, int g);

}  // namespace si
