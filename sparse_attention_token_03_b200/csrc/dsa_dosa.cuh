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
};

cudaError_t launch_seed_prep(const SeedPrepParams& p, cudaStream_t st);
cudaError_t launch_keynorm(const uint16_t* k, int64_t T_k, float* knorm, cudaStream_t st);
cudaError_t launch_plan(int H, const PlanParams& p, cudaStream_t st);
cudaError_t launch_compact(const CompactParams& p, cudaStream_t st);
cudaError_t launch_stats(const int32_t* surv_count, const int32_t* refine_len, const int32_t* row_flags,
                         int64_t T_q, unsigned long long* out, cudaStream_t st);

}  // namespace dsa
