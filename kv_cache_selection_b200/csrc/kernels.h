// Internal launchers of libstatekv (not part of the C ABI).
#pragma once

#include <cuda_runtime.h>

#include "common.cuh"

namespace skv {

constexpr int kDtypeBF16 = 0;
constexpr int kDtypeF32 = 1;

cudaError_t launch_attn_simt(const AttnArgs& a, int dtype, int d, int S, cudaStream_t st);
cudaError_t launch_score_simt(const ScoreArgs& a, int dtype, int d, int S, cudaStream_t st);
cudaError_t launch_select(const SelectArgs& a, int S, cudaStream_t st);
cudaError_t launch_gather(const GatherArgs& a, int n_sm, cudaStream_t st);

// Message for statekv_last_error(NULL) (errors of calls without a handle).
void set_free_error(const char* msg);

}  // namespace skv
