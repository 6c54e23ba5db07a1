// gdpa_ops.h -- host-side launch interfaces of the operations beside GDPA
// proper: the rotary temporal embedding and SumKronLinear.  Included by
// gdpa_internal.h; kept apart so that changes here leave the attention
// kernels' sources untouched.
#pragma once
#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "sm100.cuh"

namespace gdpa {

// debug_flags bit 2: the forward turns Q and K inside the attention kernel
// (warps 2-3, in shared memory) instead of in a streaming pass first.
constexpr int kDebugFusedRotary = 4;
inline bool rotary_streamed(const void* rope_q, int debug_flags) {
  return rope_q != nullptr && !(debug_flags & kDebugFusedRotary);
}

// Rotary temporal embedding table: angles t theta_i + tau_t phi_i per token.
struct RotaryArgs {
  // theta_i / pi as hi + lo, and phi_i / pi: angles in half-turns
  float theta_hi[64], theta_lo[64], phi_pi[64];
  double time_scale;
  int D, B;
  int64_t total;
};
cudaError_t launch_rotary_table(const RotaryArgs& r, const int32_t* offsets,
                                const int64_t* time, uint32_t* table, cudaStream_t stream);
// y = x turned by the table's angles (or back, when inverse), bf16 [total][H][D].
struct RotaryJob {
  const void* x;
  void* y;
  const uint32_t* table;
  int64_t total;
};
struct RotaryApplyArgs {
  RotaryJob job[2];  // an unused job has total 0
  int H, D;
  int inverse;
};
cudaError_t launch_rotary_apply(const RotaryApplyArgs& a, int sms, cudaStream_t stream);

// SumKronLinear forward (maps: A [kT][S] boxes 64 x 128, X [B][S][D] boxes
// 64 x 64 x 1, W [kD][D] boxes 64 x kSumKronWRows, bf16).
constexpr int kSumKronWRows = 16;
struct SumKronLaunch {
  DeviceStatus* status;
  __nv_bfloat16* y;
  int B, S, T, D, k;
  int debug_flags;
  uint64_t timeout_ns;
};
cudaError_t launch_sumkron(const SumKronLaunch& L, const CUtensorMap& ta, const CUtensorMap& tx,
                           const CUtensorMap& tw, int sms, cudaStream_t s);

}  // namespace gdpa
