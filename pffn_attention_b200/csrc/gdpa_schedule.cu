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
// scan of the tile counts (kept in shared memory by sample from the first
// pass).  Compare-exchange stages whose partners lie within one warp run on
// shuffles in registers, so only the wider stages pass through shared memory
// with a block barrier.  The kernel also clears the workspace status, and lets
// the attention kernel that follows it start its set-up at once (that kernel
// waits for this one's results before it reads them).
#include <atomic>

#include "gdpa_internal.h"
#include "gdpa_pdl.cuh"

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

// One compare-exchange of element i with element i ^ j (j < 32: the partner
// is lane ^ j of the same warp) in the bitonic merge of width k: the lower
// index keeps the smaller key where the merge ascends ((i & k) == 0).
__device__ __forceinline__ unsigned long long shfl_cmpx(unsigned long long x, int i, int j,
                                                        int k) {
  const unsigned long long y = __shfl_xor_sync(0xffffffffu, x, j);
  const bool keep_min = ((i & j) == 0) == ((i & k) == 0);
  return keep_min ? (x < y ? x : y) : (x < y ? y : x);
}

// Ascending bitonic sort of keys[0, n) (n a power of two) by the whole block;
// element i = r * kSchedThreads + tid belongs to thread tid (lane i % 32).
// Returns after a block barrier.
__device__ void block_bitonic_sort(unsigned long long* keys, int n) {
  const int tid = threadIdx.x;
  const int per = (n + kSchedThreads - 1) / kSchedThreads;
  // merges of width <= 32 stay inside a warp
  for (int r = 0; r < per; ++r) {
    const int i = r * kSchedThreads + tid;
    unsigned long long x = i < n ? keys[i] : ~0ull;
    for (int k = 2; k <= 32 && k <= n; k <<= 1)
      for (int j = k >> 1; j > 0; j >>= 1) x = shfl_cmpx(x, i, j, k);
    if (i < n) keys[i] = x;
  }
  __syncthreads();
  for (int k = 64; k <= n; k <<= 1) {
    for (int j = k >> 1; j >= 32; j >>= 1) {
      for (int i = tid; i < n; i += kSchedThreads) {
        const int ixj = i ^ j;
        if (ixj > i) {
          const unsigned long long x = keys[i], y = keys[ixj];
          if ((x > y) == ((i & k) == 0)) {
            keys[i] = y;
            keys[ixj] = x;
          }
        }
      }
      __syncthreads();
    }
    for (int r = 0; r < per; ++r) {
      const int i = r * kSchedThreads + tid;
      unsigned long long x = i < n ? keys[i] : ~0ull;
      for (int j = 16; j > 0; j >>= 1) x = shfl_cmpx(x, i, j, k);
      if (i < n) keys[i] = x;
    }
    __syncthreads();
  }
}

__global__ void __launch_bounds__(kSchedThreads)
    gdpa_schedule_kernel(const int32_t* __restrict__ q_offsets,
                         const int32_t* __restrict__ kv_offsets, int B, int BM, int BN, int wl,
                         int wr, int32_t* __restrict__ tile_start, int32_t* __restrict__ order,
                         int4* __restrict__ info, int max_q, int max_kv, int64_t total_q,
                         int64_t total_kv, DeviceStatus* status) {
  extern __shared__ unsigned long long keys[];  // n keys, then tiles[B]
  __shared__ long long warp_tot[kSchedThreads / 32];
  const int tid = threadIdx.x;
  griddep_launch_dependents();
  if (status && tid == 0) {
    status->code = 0;
    status->where = 0;
    status->count = 0;
  }
  int n = 1;
  while (n < B) n <<= 1;
  int32_t* tiles = reinterpret_cast<int32_t*>(keys + n);  // query tiles by sample index
  const bool check = info != nullptr;
  for (int i = tid; i < n; i += kSchedThreads) {
    unsigned long long key = ~0ull;
    if (i < B) {
      int q0, Lq, k0, Lk;
      sample_lengths(q_offsets, kv_offsets, i, check, max_q, max_kv, total_q, total_kv, q0, Lq,
                     k0, Lk);
      unsigned long long c = sample_cost(Lq, Lk, BM, BN, wl, wr);
      if (c > 0xFFFFFFFFull) c = 0xFFFFFFFFull;
      key = ((0xFFFFFFFFull - c) << 32) | (unsigned long long)(unsigned)i;
      tiles[i] = (Lq + BM - 1) / BM;
    }
    keys[i] = key;
  }
  __syncthreads();
  block_bitonic_sort(keys, n);
  // the order and each sorted sample's descriptor (independent loads per thread)
#pragma unroll 4
  for (int p = tid; p < B; p += kSchedThreads) {
    const int b = (int)(keys[p] & 0xFFFFFFFFull);
    order[p] = b;
    if (info) {
      int q0, Lq, k0, Lk;
      const bool bad = sample_lengths(q_offsets, kv_offsets, b, true, max_q, max_kv, total_q,
                                      total_kv, q0, Lq, k0, Lk);
      // a sample outside the declared bounds is reported and skipped
      if (bad && status) record_error(status, 6, b);
      info[p] = make_int4(q0, Lq, k0, Lk);
    }
  }
  // exclusive scan of the tile counts in sorted order, contiguous chunks
  const int chunk = (B + kSchedThreads - 1) / kSchedThreads;
  const int beg = min(B, tid * chunk), end = min(B, beg + chunk);
  long long local = 0;
  for (int p = beg; p < end; ++p) local += tiles[keys[p] & 0xFFFFFFFFull];
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
    run += tiles[keys[p] & 0xFFFFFFFFull];
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
  griddep_launch_dependents();
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
  block_bitonic_sort(keys, n);
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
  if (B < 0 || B > kMaxSortBatch) return cudaErrorInvalidValue;
  int n = 1;
  while (n < B) n <<= 1;
  const size_t smem = (size_t)n * sizeof(unsigned long long) + (size_t)B * sizeof(int32_t);
  // the shared-memory attribute, once per device
  static std::atomic<uint64_t> ready{0};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const uint64_t dev_bit = dev >= 0 && dev < 64 ? 1ull << dev : 0;
  if (!(ready.load(std::memory_order_acquire) & dev_bit)) {
    e = cudaFuncSetAttribute(gdpa_schedule_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)(kMaxSortBatch * (sizeof(unsigned long long) + sizeof(int32_t))));
    if (e != cudaSuccess) return e;
    ready.fetch_or(dev_bit, std::memory_order_acq_rel);
  }
  gdpa_schedule_kernel<<<1, kSchedThreads, smem, stream>>>(q_offsets, kv_offsets, B, block_m,
                                                           block_n, wl, wr, tile_start, order,
                                                           info, max_q, max_kv, total_q, total_kv,
                                                           status);
  return cudaGetLastError();
}

}  // namespace gdpa
