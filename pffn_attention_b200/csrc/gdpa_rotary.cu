// gdpa_rotary.cu -- rotation table of the rotary temporal embedding.
//
// Kunlun paper review §2.2: RoPE extended from positions to time gaps; the gap
// between adjacent events is log-scaled by tau_scale, and each angle mixes a
// position frequency theta_i with a time frequency phi_i.  Per token t of a
// sample (0-based) with gap dt_t to the previous event (0 for the first,
// negative gaps clamped to 0):
//   tau_t = ln(1 + dt_t / tau_scale),  alpha_{t,i} = t theta_i + tau_t phi_i,
// and the table holds (cos alpha, sin alpha) as an fp16 pair per (t, i).  The
// forward and backward kernels turn Q and K with it in shared memory.
//
// One CTA per sample; each thread takes (token, pair) elements of the sample.
// The angle is formed and reduced modulo 2 pi in fp64, so its fp32 cosine and
// sine lose nothing to the size of t theta_i.
#include <cuda_fp16.h>

#include "gdpa_internal.h"

namespace gdpa {
namespace {

constexpr int kRotThreads = 256;
constexpr double kTwoPi = 6.283185307179586;

__global__ void __launch_bounds__(kRotThreads)
    gdpa_rotary_table_kernel(const __grid_constant__ RotaryArgs r,
                             const int32_t* __restrict__ offsets,
                             const int64_t* __restrict__ time, uint32_t* __restrict__ table) {
  const int b = blockIdx.x;
  // offsets are trusted to be a valid jagged shape; clamp so a bad one cannot
  // write outside the table
  const int64_t s = offsets[b] > 0 ? (int64_t)offsets[b] : 0;
  const int64_t e = offsets[b + 1] < r.total ? (int64_t)offsets[b + 1] : r.total;
  const int half = r.D / 2;
  const int64_t n = (e - s) * half;
  for (int64_t idx = threadIdx.x; idx < n; idx += kRotThreads) {
    const int64_t t = idx / half;
    const int i = (int)(idx - t * half);
    const int64_t tok = s + t;
    double tau = 0.0;
    if (t > 0) {
      const int64_t dt = time[tok] - time[tok - 1];
      if (dt > 0) tau = log1p((double)dt / r.time_scale);
    }
    double ang = (double)t * (double)r.theta[i] + tau * (double)r.phi[i];
    ang -= kTwoPi * rint(ang / kTwoPi);
    float sn, cs;
    sincosf((float)ang, &sn, &cs);
    const __half2 h = __floats2half2_rn(cs, sn);  // .x = cos, .y = sin
    table[tok * half + i] = *reinterpret_cast<const uint32_t*>(&h);
  }
}

}  // namespace

cudaError_t launch_rotary_table(const RotaryArgs& r, const int32_t* offsets,
                                const int64_t* time, uint32_t* table, cudaStream_t stream) {
  if (r.B <= 0 || r.total <= 0) return cudaSuccess;
  gdpa_rotary_table_kernel<<<r.B, kRotThreads, 0, stream>>>(r, offsets, time, table);
  return cudaGetLastError();
}

}  // namespace gdpa
