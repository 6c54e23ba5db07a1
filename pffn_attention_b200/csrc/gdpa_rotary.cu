// gdpa_rotary.cu -- rotary temporal embedding: the rotation table, and the
// streaming pass that turns Q and K (or back-turns dQ and dK) with it.
//
// Kunlun paper review §2.2: RoPE extended from positions to time gaps; the gap
// between adjacent events is log-scaled by tau_scale, and each angle mixes a
// position frequency theta_i with a time frequency phi_i.  Per token t of a
// sample (0-based) with gap dt_t to the previous event (0 for the first,
// negative gaps clamped to 0):
//   tau_t = ln(1 + dt_t / tau_scale),  alpha_{t,i} = t theta_i + tau_t phi_i,
// and the table holds (cos alpha, sin alpha) as an fp16 pair per (t, i).
//
// Table: a warp per run of 16 tokens (the first one's sample found by binary
// search over the offsets), a lane per pair; tau_t is taken once per token
// (fp32 log1p).
// Angles are handled in half-turns (alpha / pi) in fp32 without rounding the
// large part: theta_i / pi comes as a float pair hi + lo (from fp64 on the
// host), t * hi is split exactly into a rounded product and its remainder
// (one fma), the rounded product is reduced modulo 2 (exact in fp32), and the
// small parts t * lo, the remainder and tau_t * phi_i / pi are added after.
// sincospif then gives the cosine and sine; positions below 2^24 are exact.
//
// Turn: HBM-bound streaming over [total][H][D] bf16.  One warp per token, a
// lane per 16-byte chunk (four pairs) of the token's H * D / 8; the table
// chunk serves all H heads from L1.  Up to two tensors per launch (Q and K,
// or dQ and dK).
#include <cuda_fp16.h>

#include "gdpa_internal.h"

namespace gdpa {
namespace {

constexpr int kRotThreads = 256;
constexpr int kRunTokens = 16;  // table: consecutive tokens per warp

__global__ void __launch_bounds__(kRotThreads)
    gdpa_rotary_table_kernel(const __grid_constant__ RotaryArgs r,
                             const int32_t* __restrict__ offsets,
                             const int64_t* __restrict__ time, uint32_t* __restrict__ table) {
  // per-lane frequency reads from the parameter space would serialise (one
  // address per lane); shared memory serves them in one pass
  __shared__ float th_hi[64], th_lo[64], ph[64];
  if (threadIdx.x < 64) {
    th_hi[threadIdx.x] = r.theta_hi[threadIdx.x];
    th_lo[threadIdx.x] = r.theta_lo[threadIdx.x];
    ph[threadIdx.x] = r.phi_pi[threadIdx.x];
  }
  __syncthreads();
  const int lane = threadIdx.x & 31;
  const int half = r.D / 2;
  const float inv_scale = (float)(1.0 / r.time_scale);
  // a warp takes kRunTokens consecutive tokens: one binary search for the
  // first one's sample (the last b with offsets[b] <= tok; offsets are
  // trusted to be a valid jagged shape), then a forward walk
  const int64_t tok0 = ((int64_t)blockIdx.x * (kRotThreads / 32) + (threadIdx.x >> 5)) * kRunTokens;
  if (tok0 >= r.total) return;
  int b = 0, hi_b = r.B - 1;
  while (b < hi_b) {
    const int mid = (b + hi_b + 1) >> 1;
    if (offsets[mid] <= tok0) b = mid; else hi_b = mid - 1;
  }
  int64_t next = offsets[b + 1];
  const int64_t tok1 = tok0 + kRunTokens < r.total ? tok0 + kRunTokens : r.total;
  for (int64_t tok = tok0; tok < tok1; ++tok) {
    while (tok >= next && b + 1 < r.B) next = offsets[++b + 1];  // skips empty samples
    const int64_t t = tok - offsets[b];
    float tau = 0.f;
    if (t > 0) {
      const int64_t dt = time[tok] - time[tok - 1];
      if (dt > 0) tau = log1pf((float)dt * inv_scale);
    }
    const float tf = (float)t;
    for (int i = lane; i < half; i += 32) {
      const float thi = th_hi[i];
      float hi = tf * thi;
      const float rem = fmaf(tf, thi, -hi);  // t * theta_hi - hi, exactly
      hi -= 2.0f * rintf(0.5f * hi);         // exact: whole turns removed
      const float ang = hi + (rem + fmaf(tf, th_lo[i], tau * ph[i]));
      float sn, cs;
      sincospif(ang, &sn, &cs);
      const __half2 h = __floats2half2_rn(cs, sn);  // .x = cos, .y = sin
      table[tok * half + i] = *reinterpret_cast<const uint32_t*>(&h);
    }
  }
}

// x = (x0, x1) bf16 pair turned by +angle (or -angle when inverse).
__device__ __forceinline__ uint32_t turn(uint32_t x, uint32_t cs, bool inverse) {
  const float x0 = __uint_as_float(x << 16), x1 = __uint_as_float(x & 0xffff0000u);
  float2 f = __half22float2(*reinterpret_cast<const __half2*>(&cs));
  if (inverse) f.y = -f.y;
  const float y0 = fmaf(x0, f.x, -x1 * f.y), y1 = fmaf(x0, f.y, x1 * f.x);
  const uint32_t lo = __bfloat16_as_ushort(__float2bfloat16_rn(y0));
  const uint32_t hi = __bfloat16_as_ushort(__float2bfloat16_rn(y1));
  return lo | (hi << 16);
}

__global__ void __launch_bounds__(kRotThreads)
    gdpa_rotary_apply_kernel(const __grid_constant__ RotaryApplyArgs a) {
  const int CH = a.D / 8;       // chunks per head (a power of two)
  const int HC = a.H * CH;      // chunks per token
  const int warps = kRotThreads / 32;
  const int lane = threadIdx.x & 31;
  const int64_t nwarps = (int64_t)gridDim.x * warps;
  const int64_t ntok = a.job[0].total + a.job[1].total;
  for (int64_t w = (int64_t)blockIdx.x * warps + (threadIdx.x >> 5); w < ntok; w += nwarps) {
    const bool second = w >= a.job[0].total;
    const RotaryJob& j = a.job[second ? 1 : 0];
    const int64_t tok = second ? w - a.job[0].total : w;
    const uint4* xr = reinterpret_cast<const uint4*>(j.x) + tok * HC;
    const uint4* tr = reinterpret_cast<const uint4*>(j.table + tok * (a.D / 2));
    uint4* yr = reinterpret_cast<uint4*>(j.y) + tok * HC;
    for (int idx = lane; idx < HC; idx += 32) {
      const uint4 x = xr[idx];  // plain load: y may alias x
      const uint4 cs = __ldg(tr + (idx & (CH - 1)));
      uint4 y;
      y.x = turn(x.x, cs.x, a.inverse);
      y.y = turn(x.y, cs.y, a.inverse);
      y.z = turn(x.z, cs.z, a.inverse);
      y.w = turn(x.w, cs.w, a.inverse);
      yr[idx] = y;
    }
  }
}

}  // namespace

cudaError_t launch_rotary_table(const RotaryArgs& r, const int32_t* offsets,
                                const int64_t* time, uint32_t* table, cudaStream_t stream) {
  if (r.B <= 0 || r.total <= 0) return cudaSuccess;
  const int64_t per_block = (int64_t)(kRotThreads / 32) * kRunTokens;
  const int64_t grid = (r.total + per_block - 1) / per_block;
  gdpa_rotary_table_kernel<<<(unsigned)grid, kRotThreads, 0, stream>>>(r, offsets, time, table);
  return cudaGetLastError();
}

cudaError_t launch_rotary_apply(const RotaryApplyArgs& a, int sms, cudaStream_t stream) {
  const int64_t ntok = a.job[0].total + a.job[1].total;
  if (ntok <= 0) return cudaSuccess;
  // one warp per token; enough resident warps to cover HBM latency (8 blocks
  // of 256 threads per SM)
  const int64_t want = (ntok + kRotThreads / 32 - 1) / (kRotThreads / 32);
  const int grid = (int)(want < (int64_t)sms * 8 ? want : (int64_t)sms * 8);
  gdpa_rotary_apply_kernel<<<grid, kRotThreads, 0, stream>>>(a);
  return cudaGetLastError();
}

}  // namespace gdpa
