// hmean.h -- launchers of the forward through the horizon mean: ctx_mean [B, H]
// from x [B * N_H, H] and the routing's expert_idx (1 <= N_H <= 32).
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

namespace moe {

cudaError_t launch_hmean_fwd_tf32(const float* x, const float* W, const float* bias, const int32_t* expert_idx,
                                  int64_t B, int N_H, int E, int H, float* out, uint32_t* dev_flags, int num_sms,
                                  cudaStream_t s);
cudaError_t launch_hmean_fwd_ffma(const float* x, const float* W, const float* bias, const int32_t* expert_idx,
                                  int64_t B, int N_H, int E, int H, float* out, cudaStream_t s);
// The dynamic shared-memory limit of the tcgen05 kernel, set once per device.
cudaError_t hmean_set_smem_limits();

}  // namespace moe
