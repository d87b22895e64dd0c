// Parameters and launchers of the DoSA support kernels (dsa_dosa.cu).
#pragma once

#include <cuda_runtime.h>
#include <cstdint>

#include "dsa_kernels.cuh"

namespace dsa {

struct SeedPrepParams {
  const int32_t* seed_idx;  // [n_seed]
  int n_seed;
  int64_t q_offset;
  const uint16_t* k;        // [T_k][128]
  uint32_t* seed_bits;      // [ceil(T_k / 32)], zeroed by the caller
  uint16_t* k_seed;         // [n_seed][128]
  uint32_t* err;
};

struct PlanParams {
  const uint16_t* q;       // [T_q][H][128]
  const float* w;          // [T_q][H]
  const uint16_t* k_seed;  // [n_seed][128]
  int n_seed;
  int64_t T_q;
  const float* tau;        // [T_q] topk-th seed score per row
  uint16_t* plan_q;        // [T_q][kPlanRows][128]
  float* plan_s;           // [T_q][kPlanScalars]
  const uint32_t* skip;    // optional: when *skip != 0 the launch does nothing
};

struct CompactParams {
  int64_t T_q;
  int64_t q_offset;
  int topk;
  const uint32_t* bitmask;  // [T_q][mask_words]
  int64_t mask_words;
  const int32_t* surv_count;
  int cap_row;              // survivor ids per row
  int32_t* surv_ids;        // [T_q][cap_row]
  int32_t* refine_len;      // [T_q]
  int32_t* row_flags;       // [T_q]
  const uint64_t* seed_rec; // [T_q][rec_stride] sorted seed records
  int rec_stride;
  uint64_t* init_thr;       // [T_q]
  const uint32_t* err;
  const uint32_t* skip;     // optional: when *skip != 0 the launch does nothing
  // the shared stream's keys of each group of four rows, left out of the
  // rows' own lists (null: no shared stream)
  const uint32_t* group_mask;  // [T_q / 4][mask_words]
  const int32_t* group_len;    // [T_q / 4]
};

// The shared refine stream of each group of four consecutive rows ("DoSA"
// notes, annotation WFZZA9CL, step 3): keys kept by at least two of the four
// rows and visible to all four are scored once for the group.
struct ShareParams {
  int64_t T_q;              // rows of this launch (groups of 4 from row 0)
  int64_t q_offset;         // position of row 0
  const uint32_t* bitmask;  // [T_q][mask_words] survivor bits
  int64_t mask_words;
  const int32_t* surv_count;  // [T_q]
  int cap_row;
  uint32_t* group_mask;     // [T_q / 4][mask_words] (words of the group's common range)
  int32_t* group_ids;       // [T_q / 4][cap_row] ascending shared key ids
  int32_t* group_len;       // [T_q / 4]
  const uint32_t* err;
  const uint32_t* skip;
};

// Row states of the pruned path (row_flags): every non-zero state is
// recomputed by the dense recovery pass.
enum : int32_t {
  kRowRefined = 0,    // screened; survivors refined exactly
  kRowOverflow = 1,   // screened; survivors exceeded the row's list
  kRowBypassed = 2,   // not screened: the probe sent the chunk to the dense path
  kRowBadSeed = 3,    // the seed list failed validation
};

// Probe decision: after the first rows of a chunk went through the pruned
// path, estimate the pruned cost of the chunk relative to the dense cost and
// set *bypass when pruning would not pay.
struct DecideParams {
  int64_t probe_rows;
  int64_t T_q;
  int64_t q_offset;
  int n_seed;
  const int32_t* surv_count;  // [T_q]
  int32_t* row_flags;         // [T_q]
  int32_t* refine_len;        // [T_q]
  uint32_t* bypass;           // control word
};

// Counters of dsa_stats, summed on the device.
struct StatsParams {
  int64_t T_q;
  int64_t q_offset;
  int n_seed;
  int topk;
  CandLayout lay;            // refine candidate layout
  const int32_t* surv_count;
  const int32_t* refine_len;
  const int32_t* row_flags;
  const int32_t* meta;       // refine candidate meta, [unit][kMetaInts]
  const int32_t* seq_ubeg;   // refine units per row
  const int32_t* seq_ucnt;
  // shared refine stream (null when absent): group lengths, meta, units per group
  const int32_t* group_len;
  const int32_t* meta2;
  const int32_t* gs_ubeg;
  const int32_t* gs_ucnt;
  unsigned long long* out;   // [8]
};

// Seeds from historical selection frequency (dsa_history.cu).
struct HistoryParams {
  const int32_t* prev;  // [n_rows][topk] earlier Top-k lists, -1 padding
  int64_t n_rows;
  int topk;
  int64_t n_keys;       // keys 0..n_keys-1 are eligible
  int n_seed;
  int num_sms;
  uint32_t* counts;     // [n_keys], zeroed by the caller
  uint32_t* hist;       // [65536], zeroed by the caller (left zeroed)
  uint32_t* ctl;        // [4] control words, zeroed by the caller
  uint32_t* tile_gt;    // [ceil(n_keys / 1024)]
  uint32_t* tile_eq;    // [ceil(n_keys / 1024)]
  int32_t* seeds;       // [n_seed] out, ascending
};

cudaError_t launch_seed_prep(const SeedPrepParams& p, cudaStream_t st);
cudaError_t launch_keynorm(const uint16_t* k, int64_t T_k, float* knorm, cudaStream_t st);
cudaError_t launch_plan(int H, const PlanParams& p, cudaStream_t st);
cudaError_t launch_compact(const CompactParams& p, cudaStream_t st);
cudaError_t launch_share(const ShareParams& p, cudaStream_t st);
cudaError_t launch_decide(const DecideParams& p, cudaStream_t st);
cudaError_t launch_stats(const StatsParams& p, cudaStream_t st);
cudaError_t launch_history_seeds(const HistoryParams& p, cudaStream_t st);

}  // namespace dsa
