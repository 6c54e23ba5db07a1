// gdpa_ops.h -- host-side launch interfaces of the operations beside GDPA
// proper: the rotary temporal embedding, SumKronLinear and the batched GEMM
// its backward runs on.  Included by gdpa_internal.h; kept apart so that
// changes here leave the attention kernels' sources untouched.
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

// Batched bf16 GEMM on tcgen05 (the SumKronLinear backward's contractions):
// per grid batch z and output tile, C = sum over reduction batches rb of
// A(rb, z) B(rb, z), fp32 accumulate.  Each operand comes from a 3-D tensor
// map (128-byte swizzle) and is either K-major (map dims {K, rows, batch},
// boxes 64 x 128) or MN-major (map dims {M or N, K rows, batch}, boxes
// 64 x KC); see GemmOperand for how a box's coordinates follow from the tile,
// the K chunk, rb and z.
struct GemmOperand {
  int mn_major;   // 0: K-major, 1: MN-major
  int z_rows;     // row coordinate added per grid batch (K-major rows, or MN-major K rows)
  int batch_of;   // the map's batch coordinate: 0 none, 1 the reduction batch, 2 the grid batch
};
struct GemmLaunch {
  int M, N;        // output extent per grid batch
  int Z;           // grid batches
  int n_rb;        // reduction batches
  int nkc;         // K chunks per reduction batch
  int kc;          // K rows per chunk: 64, or 32 (both operands MN-major)
  int splits;      // CTAs sharing one tile's reduction batches
  GemmOperand a, b;
  // Output: fp32 partial sums [split][z][M][N] (f32_out), or bf16 at
  //   z * sZ + (m / mT) * sMb + (m % mT) * sMt + (n / nD) * sNr + n % nD
  int f32_out;
  void* out;
  int mT, nD;
  int64_t sZ, sMb, sMt, sNr;
  DeviceStatus* status;
  uint64_t timeout_ns;
};
cudaError_t launch_gemm(const GemmLaunch& g, const CUtensorMap& ta, const CUtensorMap& tb,
                        int sms, cudaStream_t s);
// out[i] = bf16(sum over s < splits of part[s * count + i]), i < count (count % 8 == 0).
cudaError_t launch_sum_splits(const float* part, int splits, int64_t count, __nv_bfloat16* out,
                              int sms, cudaStream_t s);

}  // namespace gdpa
