// gdpa_schedule.cu -- jagged tile schedule (longest-processing-time order).
//
// The GDPA kernel's "tile scheduling" over "jagged sequences" (Kunlun paper
// review §2.3 "GDPA", last paragraph) is left undefined by the pages; this is
// the schedule the kernels here use:
//   ntile_b = ceil(Lq_b / BM); each tile m (first row m0 = m*BM) may see keys
//   [max(0, m0 - wl), min(Lk_b, m0 + BM + wr)) rounded out to key blocks of BN;
//   cost_b = sum over tiles of (1 + key blocks);
//   order  = samples by descending cost, ties by ascending index;
//   tile_start[p] = query tiles of order[0..p).
// One CTA: costs into shared memory as 64-bit keys (inverted cost, index) so
// an ascending bitonic sort yields the order with unique keys, then a block
// scan of the tile counts.  The kernel also clears the workspace status.
#include "gdpa_internal.h"

namespace gdpa {
namespace {

constexpr int kSchedThreads = 1024;

__device__ __forceinline__ unsigned long long sample_cost(int Lq, int Lk, int BM, int BN, int wl,
                                                          int wr) {
  const long long ntile = (Lq + BM - 1) / BM;
  if (wl < 0 && wr < 0) {
    const long long nkv = Lk > 0 ? (Lk + BN - 1) / BN : 0;
    return (unsigned long long)(ntile * (1 + nkv));
  }
  unsigned long long cost = 0;
  for (long long m = 0; m < ntile; ++m) {
    const long long m0 = m * BM;
    const long long lo = wl >= 0 ? (m0 - wl > 0 ? m0 - wl : 0) : 0;
    long long hi = Lk;
    if (wr >= 0 && m0 + BM + wr < hi) hi = m0 + BM + wr;
    long long nb = 0;
    if (hi > lo) nb = (hi + BN - 1) / BN - lo / BN;
    cost += 1 + (unsigned long long)nb;
  }
  return cost;
}

// Sample b's rows.  With check set, a sample whose lengths exceed the
// declared maxima, whose offsets decrease, or whose rows reach past the
// tensors (offsets beyond total_q / total_kv) gets zero lengths and true is
// returned: the kernels then skip it instead of reading or writing outside
// the caller's buffers.  Without check, only a negative length is clamped.
__device__ __forceinline__ bool sample_lengths(const int32_t* __restrict__ q_offsets,
                                               const int32_t* __restrict__ kv_offsets, int b,
                                               bool check, int max_q, int max_kv,
                                               int64_t total_q, int64_t total_kv, int& q0,
                                               int& Lq, int& k0, int& Lk) {
  q0 = q_offsets[b];
  k0 = kv_offsets[b];
  Lq = q_offsets[b + 1] - q0;
  Lk = kv_offsets[b + 1] - k0;
  bool bad = Lq < 0 || Lk < 0;
  if (check)
    bad = bad || Lq > max_q || Lk > max_kv || q0 < 0 || k0 < 0 ||
          (int64_t)q0 + Lq > total_q || (int64_t)k0 + Lk > total_kv;
  if (bad) {
    Lq = 0;
    Lk = 0;
  }
  return bad;
}

__global__ void __launch_bounds__(kSchedThreads)
    gdpa_schedule_kernel(const int32_t* __restrict__ q_offsets,
                         const int32_t* __restrict__ kv_offsets, int B, int BM, int BN, int wl,
                         int wr, int32_t* __restrict__ tile_start, int32_t* __restrict__ order,
                         int4* __restrict__ info, int max_q, int max_kv, int64_t total_q,
                         int64_t total_kv, DeviceStatus* status) {
  extern __shared__ unsigned long long keys[];
  __shared__ long long warp_tot[kSchedThreads / 32];
  const int tid = threadIdx.x;
  if (status && tid == 0) {
    status->code = 0;
    status->where = 0;
    status->count = 0;
  }
  __syncthreads();
  int n = 1;
  while (n < B) n <<= 1;
  for (int i = tid; i < n; i += kSchedThreads) {
    unsigned long long key = ~0ull;
    if (i < B) {
      int q0, Lq, k0, Lk;
      sample_lengths(q_offsets, kv_offsets, i, info != nullptr, max_q, max_kv, total_q, total_kv,
                     q0, Lq, k0, Lk);
      unsigned long long c = sample_cost(Lq, Lk, BM, BN, wl, wr);
      if (c > 0xFFFFFFFFull) c = 0xFFFFFFFFull;
      key = ((0xFFFFFFFFull - c) << 32) | (unsigned long long)(unsigned)i;
    }
    keys[i] = key;
  }
  __syncthreads();
  for (int k = 2; k <= n; k <<= 1) {
    for (int j = k >> 1; j > 0; j >>= 1) {
      for (int i = tid; i < n; i += kSchedThreads) {
        const int ixj = i ^ j;
        if (ixj > i) {
          const unsigned long long x = keys[i], y = keys[ixj];
          const bool ascending = (i & k) == 0;
          if ((x > y) == ascending) {
            keys[i] = y;
            keys[ixj] = x;
          }
        }
      }
      __syncthreads();
    }
  }
  // order, then an exclusive scan of the tile counts in that order
  const int chunk = (B + kSchedThreads - 1) / kSchedThreads;
  const int beg = min(B, tid * chunk), end = min(B, beg + chunk);
  long long local = 0;
  for (int p = beg; p < end; ++p) {
    const int b = (int)(keys[p] & 0xFFFFFFFFull);
    order[p] = b;
    int q0, Lq, k0, Lk;
    const bool bad = sample_lengths(q_offsets, kv_offsets, b, info != nullptr, max_q, max_kv,
                                    total_q, total_kv, q0, Lq, k0, Lk);
    local += (Lq + BM - 1) / BM;
    if (info) {
      // a sample outside the declared bounds is reported and skipped
      if (bad && status) record_error(status, 6, b);
      info[p] = make_int4(q0, Lq, k0, Lk);
    }
  }
  // block-wide exclusive scan of `local`
  const int lane = tid & 31, warp = tid >> 5;
  long long incl = local;
  for (int off = 1; off < 32; off <<= 1) {
    const long long v = __shfl_up_sync(0xffffffffu, incl, off);
    if (lane >= off) incl += v;
  }
  if (lane == 31) warp_tot[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    long long w = warp_tot[lane];
    long long wi = w;
    for (int off = 1; off < 32; off <<= 1) {
      const long long v = __shfl_up_sync(0xffffffffu, wi, off);
      if (lane >= off) wi += v;
    }
    warp_tot[lane] = wi - w;  // exclusive prefix of warp totals
  }
  __syncthreads();
  long long run = warp_tot[warp] + incl - local;
  for (int p = beg; p < end; ++p) {
    tile_start[p] = (int32_t)run;
    int q0, Lq, k0, Lk;
    sample_lengths(q_offsets, kv_offsets, order[p], info != nullptr, max_q, max_kv, total_q,
                   total_kv, q0, Lq, k0, Lk);
    run += (Lq + BM - 1) / BM;
  }
  if (end == B && beg < end) tile_start[B] = (int32_t)run;
  if (B == 0 && tid == 0) tile_start[0] = 0;
}

// Grouped forward: per launch group (one CTA each), the entries (problem,
// sample) of every problem in the group, sorted by the same cost (each
// problem's own band), longest first, ties by ascending entry; info[i] is the
// sorted entry's sample descriptor and eprob[i] its problem.  Problem tables in
// shared memory.  The caller clears the workspace status beforehand.
__global__ void __launch_bounds__(kSchedThreads)
    gdpa_group_schedule_kernel(const GroupSchedJob* __restrict__ jobs, int BM,
                               DeviceStatus* status) {
  extern __shared__ unsigned long long keys[];
  __shared__ GroupSchedProblem sp[kMaxGroupProblems];
  const int tid = threadIdx.x;
  const GroupSchedJob job = jobs[blockIdx.x];
  const GroupSchedProblem* __restrict__ probs = job.probs;
  const int n_probs = job.n_probs, n_entries = job.n_entries, BN = job.block_n;
  int4* __restrict__ info = job.info;
  int32_t* __restrict__ eprob = job.eprob;
  for (int i = tid; i < n_probs; i += kSchedThreads) sp[i] = probs[i];
  __syncthreads();
  auto problem_of = [&](int e) {  // last problem whose first entry is <= e
    int lo = 0, hi = n_probs - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (sp[mid].ebase <= e) lo = mid; else hi = mid - 1;
    }
    return lo;
  };
  int n = 1;
  while (n < n_entries) n <<= 1;
  for (int i = tid; i < n; i += kSchedThreads) {
    unsigned long long key = ~0ull;
    if (i < n_entries) {
      const GroupSchedProblem& P = sp[problem_of(i)];
      const int b = i - P.ebase;
      int q0, Lq, k0, Lk;
      sample_lengths(P.q_offsets, P.kv_offsets, b, true, P.max_q, P.max_kv, P.total_q,
                     P.total_kv, q0, Lq, k0, Lk);
      unsigned long long c = sample_cost(Lq, Lk, BM, BN, P.wl, P.wr);
      if (c > 0xFFFFFFFFull) c = 0xFFFFFFFFull;
      key = ((0xFFFFFFFFull - c) << 32) | (unsigned long long)(unsigned)i;
    }
    keys[i] = key;
  }
  __syncthreads();
  for (int k = 2; k <= n; k <<= 1) {
    for (int j = k >> 1; j > 0; j >>= 1) {
      for (int i = tid; i < n; i += kSchedThreads) {
        const int ixj = i ^ j;
        if (ixj > i) {
          const unsigned long long x = keys[i], y = keys[ixj];
          const bool ascending = (i & k) == 0;
          if ((x > y) == ascending) {
            keys[i] = y;
            keys[ixj] = x;
          }
        }
      }
      __syncthreads();
    }
  }
  for (int pos = tid; pos < n_entries; pos += kSchedThreads) {
    const int e = (int)(keys[pos] & 0xFFFFFFFFull);
    const int p = problem_of(e);
    const GroupSchedProblem& P = sp[p];
    const int b = e - P.ebase;
    int q0, Lq, k0, Lk;
    // a sample outside its problem's declared bounds is reported and skipped
    const bool bad = sample_lengths(P.q_offsets, P.kv_offsets, b, true, P.max_q, P.max_kv,
                                    P.total_q, P.total_kv, q0, Lq, k0, Lk);
    if (bad && status) record_error(status, 6, e);
    info[pos] = make_int4(q0, Lq, k0, Lk);
    eprob[pos] = p;
  }
}

}  // namespace

cudaError_t launch_group_schedule(const GroupSchedJob* jobs, int n_jobs, int max_entries,
                                  int block_m, DeviceStatus* status, cudaStream_t stream) {
  if (n_jobs < 1 || max_entries > kMaxSortBatch) return cudaErrorInvalidValue;
  int n = 1;
  while (n < max_entries) n <<= 1;
  const size_t smem = (size_t)n * sizeof(unsigned long long);
  cudaError_t e = cudaFuncSetAttribute(gdpa_group_schedule_kernel,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)(kMaxSortBatch * sizeof(unsigned long long)));
  if (e != cudaSuccess) return e;
  gdpa_group_schedule_kernel<<<n_jobs, kSchedThreads, smem, stream>>>(jobs, block_m, status);
  return cudaGetLastError();
}

cudaError_t launch_schedule(const int32_t* q_offsets, const int32_t* kv_offsets, int B,
                            int block_m, int block_n, int wl, int wr, int32_t* tile_start,
                            int32_t* order, int4* info, int max_q, int max_kv, int64_t total_q,
                            int64_t total_kv, DeviceStatus* status, cudaStream_t stream) {
  int n = 1;
  while (n < B) n <<= 1;
  const size_t smem = (size_t)n * sizeof(unsigned long long);
  cudaError_t e = cudaFuncSetAttribute(gdpa_schedule_kernel,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)(kMaxSortBatch * sizeof(unsigned long long)));
  if (e != cudaSuccess) return e;
  gdpa_schedule_kernel<<<1, kSchedThreads, smem, stream>>>(q_offsets, kv_offsets, B, block_m,
                                                           block_n, wl, wr, tile_start, order,
                                                           info, max_q, max_kv, total_q, total_kv,
                                                           status);
  return cudaGetLastError();
}

}  // namespace gdpa
