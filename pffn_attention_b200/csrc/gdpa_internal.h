// gdpa_internal.h -- argument blocks shared by the host launcher and the kernels.
#pragma once
#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "sm100.cuh"

namespace gdpa {

constexpr int kBlockM = 128;        // query rows per tile (UMMA M)
constexpr int kMaxSortBatch = 16384;  // batch limit of the single-CTA LPT sort

// Workspace layout (all offsets 256-byte aligned):
//   [0, 256)                  DeviceStatus
//   [256, ...)                order[B]      int32   (LPT sample order)
//   then                      tile_start[B+1] int32
//   then                      info[B]       int4    {q0, Lq, k0, Lk} of order[p]
//   backward only, then       delta[H][total_q] fp32 (softmax rowsum(dO * O))
//   backward only, then       dQ scratch: grid x slot_rows x D fp32
//   rotary (streamed), then   turned Q [total_q][H][D], turned K [total_kv][H][D] bf16
struct WorkspaceLayout {
  size_t order, tile_start, info, delta, dq_scratch, rope_q, rope_k, total;
  int dq_slot_rows;
  int grid;
};

constexpr size_t ws_align256(size_t x) { return (x + 255) & ~size_t(255); }
// Bytes of the part every call's workspace starts with: the status block, the
// sample order, the tile prefix and the per-sample descriptors for B samples.
// This is the whole of a forward's workspace without rotary copies.
constexpr size_t schedule_ws_bytes(int B) {
  return 256 + ws_align256((size_t)(B > 1 ? B : 1) * 4) + ws_align256((size_t)(B + 1) * 4) +
         ws_align256((size_t)(B > 1 ? B : 1) * 16);
}

// One forward problem's own data: every field a kernel role reads per unit.
// A single-problem call carries it inline (FwdArgs::p0); a grouped call keeps
// one per problem in device memory (FwdArgs::probs).
struct FwdProblem {
  const float* bias;        // [H][total_kv] or nullptr
  __nv_bfloat16* o;         // [total_q][H][D]
  float* lse;               // [H][total_q] or nullptr
  int64_t total_q, total_kv;
  int H;
  int phi;
  int bias_kind;
  int wl, wr;
  float scale;
  uint64_t head_mask;       // heads computed (bit h); ~0 = all
};

struct FwdArgs {
  const int4* info;         // per sorted entry {q0, Lq, k0, Lk}
  DeviceStatus* status;
  int H;                    // head stride of the unit index (the group's largest H)
  int n_units;              // entries * H
  int phi;                  // activation class of the launch (1 = softmax, else element-wise)
  int debug_flags;
  uint64_t timeout_ns;
  uint64_t head_mask;       // single problem: heads computed (bit h), ~0 = all
  // Grouped launch: problem of sorted entry e is eprob[e]; units are
  // (entry, head) with head stride H (the group's largest), units a problem
  // lacks are skipped; per-problem data and Q/K/V/O maps in device memory.
  // All nullptr for a single problem (p0 and the kernel's map parameters).
  const int32_t* eprob;
  const FwdProblem* probs;
  const CUtensorMap* maps;  // [problem][Q, K, V, O]
  FwdProblem p0;
  // rotary temporal embedding (single problem): per-token (cos, sin) fp16
  // pairs, [total_q][D/2] and [total_kv][D/2]; nullptr = no rotation
  const uint32_t* rope_q;
  const uint32_t* rope_kv;
};

struct BwdArgs {
  const int32_t* q_offsets;
  const int32_t* kv_offsets;
  const int32_t* order;
  const int4* info;         // per sorted sample {q0, Lq, k0, Lk}
  const float* bias;        // [H][total_kv] or nullptr
  const float* lse;         // [H][total_q] (softmax)
  const float* delta;       // [H][total_q] (softmax)
  __nv_bfloat16* dq;        // [total_q][H][D]
  __nv_bfloat16* dk;        // [total_kv][H][D]
  __nv_bfloat16* dv;        // [total_kv][H][D]
  float* dbias;             // [H][total_kv], zeroed by the launcher, or nullptr
  float* dq_scratch;        // grid x slot_rows x D
  DeviceStatus* status;
  int64_t total_q, total_kv;
  int B, H;
  int n_units;
  int max_q, max_kv;
  int dq_slot_rows;
  float scale;
  int phi;
  int bias_kind;
  int wl, wr;
  int debug_flags;
  uint64_t timeout_ns;
  uint64_t head_mask;       // heads this launch computes (bit h), ~0 = all
  // rotary temporal embedding: per-token (cos, sin) fp16 pairs [total][D/2];
  // the kernel ran on turned Q and K, and turns dQ and dK back as it writes
  // them.  nullptr = no rotation.
  const uint32_t* rope_q;
  const uint32_t* rope_kv;
};

// Per problem of a grouped forward launch, for its schedule: the problem's
// entries are ebase .. ebase + B - 1 of the group's entry list.
struct GroupSchedProblem {
  const int32_t* q_offsets;
  const int32_t* kv_offsets;
  int64_t total_q, total_kv;
  int B, ebase;
  int wl, wr;
  int max_q, max_kv;
};
constexpr int kMaxGroupProblems = 256;  // per launch group

// One launch group's schedule job (the schedule kernel runs one CTA per group).
struct GroupSchedJob {
  const GroupSchedProblem* probs;
  int n_probs, n_entries, block_n;
  int4* info;
  int32_t* eprob;
};

// Launchers (defined next to their kernels).
cudaError_t launch_schedule(const int32_t* q_offsets, const int32_t* kv_offsets, int B,
                            int block_m, int block_n, int wl, int wr, int32_t* tile_start,
                            int32_t* order, int4* info, int max_q, int max_kv, int64_t total_q,
                            int64_t total_kv, DeviceStatus* status, cudaStream_t stream);
cudaError_t launch_group_schedule(const GroupSchedJob* jobs, int n_jobs, int max_entries,
                                  int block_m, DeviceStatus* status, cudaStream_t stream);
cudaError_t launch_forward(const FwdArgs& a, int D, int block_n, const CUtensorMap& tq,
                           const CUtensorMap& tk, const CUtensorMap& tv, const CUtensorMap& to,
                           int sms, cudaStream_t stream);
int forward_block_n(int D, int phi, int max_kv, int debug_flags);
cudaError_t launch_bwd_preprocess(const __nv_bfloat16* o, const __nv_bfloat16* dout,
                                  float* delta, int64_t total_q, int H, int D,
                                  cudaStream_t stream);
cudaError_t launch_backward(const BwdArgs& a, int D, const CUtensorMap& tq,
                            const CUtensorMap& tk, const CUtensorMap& tv,
                            const CUtensorMap& tdo, int grid, cudaStream_t stream);

// A CTA's walk over (sample, head) units: unit u = p * H + h of the sorted
// sample list, boustrophedon over the grid (even rounds left to right, odd
// rounds right to left).  The next unit's descriptor is loaded one unit ahead
// so its latency hides behind the current unit.
struct GdpaUnit {
  int h, q0, Lq, k0, Lk;
  int prob;  // problem of a grouped launch (0 for a single problem)
};

// GROUPED: units of several problems (per-entry problem index, per-problem
// head counts and masks); otherwise one problem with an optional head mask.
template <bool GROUPED>
struct UnitStreamT {
  const int4* info;
  const int32_t* eprob;      // problem of each sorted entry (GROUPED)
  const FwdProblem* probs;   // per-problem heads and head masks (GROUPED)
  int H, n_units, round, u;
  uint64_t mask;  // heads to walk (bit h); ~0 = all (single problem)
  int4 nxt;
  int nprob;      // problem of the unit next() returns
  __device__ __forceinline__ static int index(int round, int cta, int grid) {
    return round * grid + ((round & 1) ? (grid - 1 - cta) : cta);
  }
  __device__ __forceinline__ static bool head_on(uint64_t m, int h) {
    return m == ~0ull || (h < 64 && ((m >> h) & 1ull));
  }
  // first unit at or after `round` this walk computes
  __device__ __forceinline__ void settle() {
    for (;;) {
      u = index(round, blockIdx.x, gridDim.x);
      if (u >= n_units) break;
      if constexpr (GROUPED) {
        const int h = u % H;
        nprob = __ldg(eprob + u / H);
        if (h < probs[nprob].H && head_on(probs[nprob].head_mask, h)) break;
      } else {
        if (mask == ~0ull || head_on(mask, u % H)) break;
      }
      ++round;
    }
    nxt = u < n_units ? __ldg(info + u / H) : make_int4(0, 0, 0, 0);
  }
  __device__ __forceinline__ UnitStreamT(const int4* info_, int H_, int n_units_,
                                         uint64_t mask_ = ~0ull, const int32_t* eprob_ = nullptr,
                                         const FwdProblem* probs_ = nullptr)
      : info(info_), eprob(eprob_), probs(probs_), H(H_), n_units(n_units_), round(0),
        mask(mask_), nprob(0) {
    settle();
  }
  // The unit the next call of next() returns, without advancing.
  __device__ __forceinline__ bool peek(GdpaUnit& t) const {
    if (u >= n_units) return false;
    t.h = u % H;
    t.q0 = nxt.x;
    t.Lq = nxt.y;
    t.k0 = nxt.z;
    t.Lk = nxt.w;
    t.prob = GROUPED ? nprob : 0;
    return true;
  }
  __device__ __forceinline__ bool next(GdpaUnit& t) {
    if (!peek(t)) return false;
    ++round;
    settle();
    return true;
  }
};
using UnitStream = UnitStreamT<false>;

}  // namespace gdpa

#include "gdpa_ops.h"
