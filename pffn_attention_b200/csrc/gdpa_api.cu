// gdpa_api.cu -- the C ABI (include/gdpa.h): argument checks, workspace layout,
// TMA descriptor encoding, and the launch sequence.  No allocation, no sync
// (except gdpa_get_device_status).
#include <cudaTypedefs.h>

#include <cmath>
#include <cstring>
#include <mutex>
#include <vector>
#include <algorithm>

#include "gdpa.h"
#include "gdpa_internal.h"

using namespace gdpa;

namespace {

constexpr int kMaxDevices = 64;

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// Number of SMs of the current device, and whether it is an sm_100 part.
bool device_info(int* sms) {
  static int cache[kMaxDevices];
  static int major_cache[kMaxDevices];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return false;
  if (cache[dev] == 0) {
    int n = 0, major = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
      return false;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess)
      return false;
    major_cache[dev] = major;
    cache[dev] = n;
  }
  *sms = cache[dev];
  return major_cache[dev] == 10;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

gdpa_status_t check_params(const gdpa_params_t* p) {
  if (!p) return GDPA_ERR_INVALID_ARG;
  if (p->B < 0 || p->H <= 0 || p->total_q < 0 || p->total_kv < 0) return GDPA_ERR_INVALID_ARG;
  if (p->total_q >= (int64_t(1) << 31) || p->total_kv >= (int64_t(1) << 31))
    return GDPA_ERR_INVALID_ARG;
  if (p->max_seqlen_q < 0 || p->max_seqlen_kv < 0) return GDPA_ERR_INVALID_ARG;
  if (p->window_left < -1 || p->window_right < -1) return GDPA_ERR_INVALID_ARG;
  if (!std::isfinite(p->scale)) return GDPA_ERR_INVALID_ARG;
  if (p->wait_timeout_us < 0) return GDPA_ERR_INVALID_ARG;
  if (p->D != 32 && p->D != 64 && p->D != 128) return GDPA_ERR_UNSUPPORTED;
  if (p->phi < 0 || p->phi > 3) return GDPA_ERR_UNSUPPORTED;
  if (p->head_phi) {
    if (p->H > 64) return GDPA_ERR_UNSUPPORTED;
    for (int h = 0; h < p->H; ++h)
      if (p->head_phi[h] < 0 || p->head_phi[h] > 3) return GDPA_ERR_UNSUPPORTED;
  }
  if (p->bias_kind < 0 || p->bias_kind > 2) return GDPA_ERR_UNSUPPORTED;
  if (p->B > kMaxSortBatch) return GDPA_ERR_UNSUPPORTED;
  if ((int64_t)p->H * p->B >= (int64_t(1) << 31)) return GDPA_ERR_UNSUPPORTED;
  // rotation tables: both or neither, 16-byte aligned (one 16-byte load per
  // four pairs)
  if ((p->rope_q == nullptr) != (p->rope_kv == nullptr)) return GDPA_ERR_INVALID_ARG;
  if (p->rope_q && (!aligned16(p->rope_q) || !aligned16(p->rope_kv))) return GDPA_ERR_INVALID_ARG;
  return GDPA_OK;
}

// Heads whose activation is phi (bit h), ~0 for all heads when every head
// uses p->phi, 0 when none does.
uint64_t phi_heads(const gdpa_params_t* p, int phi) {
  if (!p->head_phi) return p->phi == phi ? ~0ull : 0ull;
  uint64_t m = 0;
  for (int h = 0; h < p->H; ++h)
    if (p->head_phi[h] == phi) m |= 1ull << h;
  return m;
}

bool any_softmax(const gdpa_params_t* p) { return phi_heads(p, GDPA_PHI_SOFTMAX) != 0; }

int eff_max_q(const gdpa_params_t* p) {
  return p->max_seqlen_q > 0 ? p->max_seqlen_q : (int)p->total_q;
}
int eff_max_kv(const gdpa_params_t* p) {
  return p->max_seqlen_kv > 0 ? p->max_seqlen_kv : (int)p->total_kv;
}

int backward_grid(const gdpa_params_t* p, int sms) {
  const int64_t units = (int64_t)p->B * p->H;
  return (int)std::max<int64_t>(1, std::min<int64_t>(units, sms));
}

WorkspaceLayout make_layout(const gdpa_params_t* p, int backward, int sms) {
  WorkspaceLayout L{};
  size_t off = sizeof(DeviceStatus);
  L.order = off;
  off += align256((size_t)std::max(p->B, 1) * 4);
  L.tile_start = off;
  off += align256((size_t)(p->B + 1) * 4);
  L.info = off;
  off += align256((size_t)std::max(p->B, 1) * 16);
  off = schedule_ws_bytes(p->B);  // the same end, by the rule that also sizes the no-alloc array
  if (backward) {
    L.delta = off;
    if (any_softmax(p)) off += align256((size_t)p->H * (size_t)p->total_q * 4);
    L.grid = backward_grid(p, sms);
    L.dq_slot_rows = (std::min(eff_max_q(p), (int)p->total_q) + kBlockM - 1) / kBlockM * kBlockM;
    L.dq_scratch = off;
    off += align256((size_t)L.grid * (size_t)L.dq_slot_rows * (size_t)p->D * 4);
  }
  // rotary: the turned Q and K the attention kernels read (the backward's
  // input turn, and the forward's unless it turns them in the kernel)
  if (p->rope_q && (backward || rotary_streamed(p->rope_q, p->debug_flags))) {
    L.rope_q = off;
    off += align256((size_t)p->total_q * (size_t)p->H * (size_t)p->D * 2);
    L.rope_k = off;
    off += align256((size_t)p->total_kv * (size_t)p->H * (size_t)p->D * 2);
  }
  L.total = off;
  return L;
}

// One streaming launch: Q and K turned by their tables into rq, rk (inverse:
// turned back), bf16 [total][H][D].
cudaError_t turn_qk(const gdpa_params_t* p, const void* q, const void* k, void* rq, void* rk,
                    int inverse, int sms, cudaStream_t s) {
  RotaryApplyArgs r{};
  r.H = p->H;
  r.D = p->D;
  r.inverse = inverse;
  r.job[0] = RotaryJob{q, rq, static_cast<const uint32_t*>(p->rope_q), p->total_q};
  r.job[1] = RotaryJob{k, rk, static_cast<const uint32_t*>(p->rope_kv), p->total_kv};
  return launch_rotary_apply(r, sms, s);
}

// [rows][H][D] bf16 tensor, boxes of box_rows rows x one head x panel columns.
bool make_map(CUtensorMap* m, const void* base, int64_t rows, int H, int D, int box_rows) {
  auto enc = encode_fn();
  if (!enc) return false;
  const int panel = D >= 64 ? 64 : 32;
  cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)H, (cuuint64_t)rows};
  cuuint64_t strides[2] = {(cuuint64_t)D * 2, (cuuint64_t)H * D * 2};
  cuuint32_t box[3] = {(cuuint32_t)panel, 1u, (cuuint32_t)box_rows};
  cuuint32_t estr[3] = {1u, 1u, 1u};
  const CUtensorMapSwizzle sw =
      panel == 64 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B;
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides,
                   box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// O [rows][H][D] bf16 for the forward's TMA stores: boxes of 32 rows x one
// head x 32 columns (64 bytes, 64-byte swizzle, the epilogue's staging
// layout).
bool make_map_o(CUtensorMap* m, void* base, int64_t rows, int H, int D) {
  auto enc = encode_fn();
  if (!enc) return false;
  cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)H, (cuuint64_t)rows};
  cuuint64_t strides[2] = {(cuuint64_t)D * 2, (cuuint64_t)H * D * 2};
  cuuint32_t box[3] = {32u, 1u, 32u};
  cuuint32_t estr[3] = {1u, 1u, 1u};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, base, dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B,
                   CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// Row-major bf16 tensor of up to three dims (innermost first), 128-byte
// swizzled boxes whose inner extent is 64 elements.
bool make_map_3d(CUtensorMap* m, const void* base, const cuuint64_t (&dims)[3],
                 const cuuint64_t (&strides)[2], const cuuint32_t (&box)[3]) {
  auto enc = encode_fn();
  if (!enc) return false;
  cuuint32_t estr[3] = {1u, 1u, 1u};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base),
                   const_cast<cuuint64_t*>(dims), const_cast<cuuint64_t*>(strides),
                   const_cast<cuuint32_t*>(box), estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                   CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// Everything gdpa_backward checks about one problem's arguments (the
// workspace aside) before any launch.
gdpa_status_t check_backward_args(const gdpa_params_t* p, const void* q, const void* k,
                                  const void* v, const void* o, const void* dout,
                                  const float* lse, const int32_t* q_offsets,
                                  const int32_t* kv_offsets, const float* bias, const void* dq,
                                  const void* dk, const void* dv, const float* dbias) {
  gdpa_status_t st = check_params(p);
  if (st != GDPA_OK) return st;
  if (!q_offsets || !kv_offsets) return GDPA_ERR_INVALID_ARG;
  // a bias gradient needs a bias; it is fp32 [H][total_kv]
  if (dbias && p->bias_kind == GDPA_BIAS_NONE) return GDPA_ERR_INVALID_ARG;
  if (dbias && (reinterpret_cast<uintptr_t>(dbias) & 3u)) return GDPA_ERR_INVALID_ARG;
  const bool softmax = any_softmax(p);
  if (p->total_q > 0 && (!q || !dout || !dq || (softmax && (!o || !lse))))
    return GDPA_ERR_INVALID_ARG;
  if (p->total_kv > 0 && (!k || !v || !dk || !dv)) return GDPA_ERR_INVALID_ARG;
  if ((p->bias_kind != GDPA_BIAS_NONE) != (bias != nullptr)) return GDPA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(dout) ||
      !aligned16(dq) || !aligned16(dk) || !aligned16(dv))
    return GDPA_ERR_INVALID_ARG;
  if (bias && (reinterpret_cast<uintptr_t>(bias) & 3u)) return GDPA_ERR_INVALID_ARG;
  if (lse && (reinterpret_cast<uintptr_t>(lse) & 3u)) return GDPA_ERR_INVALID_ARG;
  return GDPA_OK;
}

// The grouped backward's status: the first error (in problem order) of the
// problems' own status blocks at base + table[i].
__global__ void gdpa_gather_status_kernel(DeviceStatus* dst, const uint8_t* base,
                                          const uint64_t* table, int n) {
  int count = 0;
  for (int i = 0; i < n; ++i) {
    const DeviceStatus* src = reinterpret_cast<const DeviceStatus*>(base + table[i]);
    if (src->code != 0 && dst->code == 0) {
      dst->code = src->code;
      dst->where = src->where;
    }
    count += src->count;
  }
  dst->count = count;
}

cudaError_t launch_gather_status(DeviceStatus* dst, const uint8_t* base, const uint64_t* table,
                                 int n, cudaStream_t s) {
  gdpa_gather_status_kernel<<<1, 1, 0, s>>>(dst, base, table, n);
  return cudaGetLastError();
}

gdpa_status_t check_sumkron(const gdpa_sumkron_params_t* p) {
  if (!p) return GDPA_ERR_INVALID_ARG;
  if (p->B < 0 || p->S <= 0 || p->T <= 0 || p->D <= 0 || p->k <= 0 || p->wait_timeout_us < 0)
    return GDPA_ERR_INVALID_ARG;
  if (p->T != 32 && p->T != 64) return GDPA_ERR_UNSUPPORTED;
  if (p->D != 128 && p->D != 256 && p->D != 384) return GDPA_ERR_UNSUPPORTED;
  if (p->S % 64 || p->S > 256 || ((int64_t)p->k * p->T) % 128) return GDPA_ERR_UNSUPPORTED;
  if ((int64_t)p->k * p->D >= (int64_t(1) << 31) || (int64_t)p->B * p->S >= (int64_t(1) << 31))
    return GDPA_ERR_UNSUPPORTED;
  return GDPA_OK;
}

// Everything gdpa_forward checks about one problem before any launch.
gdpa_status_t check_forward_args(const gdpa_params_t* p, const void* q, const void* k,
                                 const void* v, const int32_t* q_offsets,
                                 const int32_t* kv_offsets, const float* bias, const void* o,
                                 const float* lse) {
  gdpa_status_t st = check_params(p);
  if (st != GDPA_OK) return st;
  if (!q_offsets || !kv_offsets) return GDPA_ERR_INVALID_ARG;
  if (p->total_q > 0 && (!q || !o)) return GDPA_ERR_INVALID_ARG;
  if (p->total_kv > 0 && (!k || !v)) return GDPA_ERR_INVALID_ARG;
  if ((p->bias_kind != GDPA_BIAS_NONE) != (bias != nullptr)) return GDPA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o)) return GDPA_ERR_INVALID_ARG;
  if (bias && (reinterpret_cast<uintptr_t>(bias) & 3u)) return GDPA_ERR_INVALID_ARG;
  if (lse && (reinterpret_cast<uintptr_t>(lse) & 3u)) return GDPA_ERR_INVALID_ARG;
  return GDPA_OK;
}

uint64_t timeout_ns(const gdpa_params_t* p) {
  const int us = p->wait_timeout_us > 0 ? p->wait_timeout_us : 2000000;
  return (uint64_t)us * 1000ull;
}


// ---- grouped forward
// One activation's heads of one caller problem.
struct VProblem {
  int src;          // index into the caller's problems
  int phi;
  uint64_t heads;
};

// Problems that share a launch: head dim, key-block size, softmax or not.
struct LaunchGroup {
  int D, block_n;
  bool softmax;
  std::vector<VProblem> vp;
  int entries = 0, hmax = 0;
  size_t off_probs = 0, off_maps = 0, off_sched = 0, off_info = 0, off_eprob = 0;
};

// Workspace of a grouped call: status block and the tables the host fills
// (schedule jobs; per group: problem table, tensor maps, schedule table) as
// one contiguous range copied in one transfer (the status copied as zeros),
// then per group the sorted entries and their problems, which the schedule
// kernel writes.
struct GroupedLayout {
  size_t off_jobs = 0, tables_end = 0, total = 0;
  // per caller problem with rotary tables: its turned Q and K copies (0 = none)
  std::vector<size_t> rope_q, rope_k;
};

// Validates every problem, forms the launch groups and lays out the workspace.
// Nothing touches the device.
gdpa_status_t plan_grouped(const gdpa_forward_problem_t* probs, int n,
                           std::vector<LaunchGroup>& groups, GroupedLayout& lay) {
  if (!probs || n < 1) return GDPA_ERR_INVALID_ARG;
  groups.clear();
  for (int i = 0; i < n; ++i) {
    const gdpa_forward_problem_t& f = probs[i];
    const gdpa_params_t* p = &f.params;
    gdpa_status_t st = check_forward_args(p, f.q, f.k, f.v, f.q_offsets, f.kv_offsets, f.bias,
                                          f.o, f.lse);
    if (st != GDPA_OK) return st;
    if (p->rope_q && (p->debug_flags & kDebugFusedRotary))
      return GDPA_ERR_UNSUPPORTED;  // grouped calls turn Q and K in a streaming pass
    const int block_n = forward_block_n(p->D, p->phi, eff_max_kv(p), p->debug_flags);
    for (int phi = 0; phi <= 3; ++phi) {
      const uint64_t heads = phi_heads(p, phi);
      if (!heads) continue;
      const bool sm = phi == GDPA_PHI_SOFTMAX;
      LaunchGroup* g = nullptr;
      for (LaunchGroup& x : groups)
        if (x.D == p->D && x.block_n == block_n && x.softmax == sm) g = &x;
      if (!g) {
        groups.push_back(LaunchGroup{});
        g = &groups.back();
        g->D = p->D;
        g->block_n = block_n;
        g->softmax = sm;
      }
      g->vp.push_back(VProblem{i, phi, heads});
    }
  }
  size_t total = align256(sizeof(DeviceStatus));
  lay.off_jobs = total;
  total = align256(total + groups.size() * sizeof(GroupSchedJob));
  for (LaunchGroup& g : groups) {
    if ((int)g.vp.size() > kMaxGroupProblems) return GDPA_ERR_UNSUPPORTED;
    int64_t entries = 0;
    for (const VProblem& v : g.vp) {
      entries += probs[v.src].params.B;
      g.hmax = std::max(g.hmax, probs[v.src].params.H);
    }
    if (entries > kMaxSortBatch) return GDPA_ERR_UNSUPPORTED;
    if (entries * (int64_t)g.hmax >= (int64_t(1) << 31)) return GDPA_ERR_UNSUPPORTED;
    g.entries = (int)entries;
    const size_t nv = g.vp.size();
    g.off_probs = total;
    g.off_maps = align256(g.off_probs + nv * sizeof(FwdProblem));
    g.off_sched = align256(g.off_maps + 4 * nv * sizeof(CUtensorMap));
    total = align256(g.off_sched + nv * sizeof(GroupSchedProblem));
  }
  lay.tables_end = total;
  for (LaunchGroup& g : groups) {
    g.off_info = total;
    g.off_eprob = align256(g.off_info + (size_t)g.entries * sizeof(int4));
    total = align256(g.off_eprob + (size_t)g.entries * sizeof(int32_t));
  }
  // rotary: turned copies of each such problem's Q and K
  lay.rope_q.assign(n, 0);
  lay.rope_k.assign(n, 0);
  for (int i = 0; i < n; ++i) {
    const gdpa_params_t* p = &probs[i].params;
    if (!p->rope_q) continue;
    lay.rope_q[i] = total;
    total = align256(total + (size_t)p->total_q * p->H * p->D * 2);
    lay.rope_k[i] = total;
    total = align256(total + (size_t)p->total_kv * p->H * p->D * 2);
  }
  lay.total = total;
  return GDPA_OK;
}

}  // namespace

// ---------------------------------------------------------------- SumKronLinear backward
// For Y_b = sum_r A_r X_b W_r and the upstream gradient dY (Kunlun paper review
// §2.4; the reading of the map is the forward's):
//   Z_b   = [A_1; ...; A_k] X_b                   (k T x D, recomputed)
//   U_b   = dY_b [W_1^T ... W_k^T], stored as [r][t][d]      (k T x D)
//   dX_b  = sum_r A_r^T U_b[r] = [A_1; ...; A_k]^T U_b         (S x D)
//   dA_r  = sum_b U_b[r] X_b^T                                  (T x S)
//   dW_r  = sum_b Z_b[r]^T dY_b                                 (D x D)
// five batched GEMMs (gdpa_gemm.cu); dA and dW sum over the samples, split
// across CTAs into fp32 partials that a last pass adds up.
namespace {

int sk_splits_a(int B) { return std::max(1, std::min(B, 64)); }
int sk_splits_w(int B) { return std::max(1, std::min(B, 8)); }

struct SkBwdLayout {
  size_t z, u, pa, pw, end;
};
SkBwdLayout sk_bwd_layout(const gdpa_sumkron_params_t* p) {
  SkBwdLayout L{};
  const size_t kT = (size_t)p->k * p->T;
  size_t off = align256(sizeof(DeviceStatus));
  L.z = off;
  off = align256(off + (size_t)p->B * kT * p->D * 2);
  L.u = off;
  off = align256(off + (size_t)p->B * kT * p->D * 2);
  L.pa = off;
  off = align256(off + (size_t)sk_splits_a(p->B) * kT * p->S * 4);
  L.pw = off;
  off = align256(off + (size_t)sk_splits_w(p->B) * p->k * p->D * p->D * 4);
  L.end = off;
  return L;
}

// bf16 [dim2][dim1][dim0] (dim0 contiguous), boxes box0 x box1 x 1, 128-byte swizzle
bool sk_map(CUtensorMap* m, const void* base, cuuint64_t d0, cuuint64_t d1, cuuint64_t d2,
            cuuint32_t box0, cuuint32_t box1) {
  return make_map_3d(m, base, {d0, d1, d2}, {d0 * 2, d0 * d1 * 2}, {box0, box1, 1u});
}

}  // namespace

extern "C" {

int gdpa_version(void) { return 100; }

const char* gdpa_status_string(gdpa_status_t s) {
  switch (s) {
    case GDPA_OK: return "ok";
    case GDPA_ERR_INVALID_ARG: return "invalid argument";
    case GDPA_ERR_UNSUPPORTED: return "unsupported configuration or device";
    case GDPA_ERR_WORKSPACE: return "workspace missing or too small";
    case GDPA_ERR_CUDA: return "CUDA error";
    case GDPA_ERR_TIMEOUT: return "device wait timed out";
    case GDPA_ERR_DEVICE_CHECK: return "sample beyond the declared maximum length or the tensors";
  }
  return "unknown status";
}

size_t gdpa_workspace_size(const gdpa_params_t* p, int backward) {
  if (check_params(p) != GDPA_OK) return 0;
  int sms = 0;
  if (!device_info(&sms)) sms = 148;
  return make_layout(p, backward, sms).total;
}

gdpa_status_t gdpa_forward_tile_shape(const gdpa_params_t* p, int* block_m, int* block_n) {
  gdpa_status_t st = check_params(p);
  if (st != GDPA_OK) return st;
  if (!block_m || !block_n) return GDPA_ERR_INVALID_ARG;
  *block_m = kBlockM;
  *block_n = forward_block_n(p->D, p->phi, eff_max_kv(p), p->debug_flags);
  return GDPA_OK;
}

gdpa_status_t gdpa_tile_schedule(const gdpa_params_t* p, int block_m, int block_n,
                                 const int32_t* q_offsets, const int32_t* kv_offsets,
                                 int32_t* tile_start, int32_t* order, gdpa_stream_t stream) {
  gdpa_status_t st = check_params(p);
  if (st != GDPA_OK) return st;
  if (!q_offsets || !kv_offsets || !tile_start || (!order && p->B > 0)) return GDPA_ERR_INVALID_ARG;
  if (block_m < 16 || block_m > 256 || block_m % 16 || block_n < 16 || block_n > 256 ||
      block_n % 16)
    return GDPA_ERR_INVALID_ARG;
  int sms = 0;
  if (!device_info(&sms)) return GDPA_ERR_UNSUPPORTED;
  cudaError_t e = launch_schedule(q_offsets, kv_offsets, p->B, block_m, block_n, p->window_left,
                                  p->window_right, tile_start, order, nullptr, 0, 0, p->total_q,
                                  p->total_kv, nullptr, (cudaStream_t)stream);
  return e == cudaSuccess ? GDPA_OK : GDPA_ERR_CUDA;
}

gdpa_status_t gdpa_forward(const gdpa_params_t* p, const void* q, const void* k, const void* v,
                           const int32_t* q_offsets, const int32_t* kv_offsets,
                           const float* bias, void* o, float* lse, void* workspace,
                           size_t workspace_bytes, gdpa_stream_t stream) {
  gdpa_status_t st = check_forward_args(p, q, k, v, q_offsets, kv_offsets, bias, o, lse);
  if (st != GDPA_OK) return st;
  if (!aligned16(workspace)) return GDPA_ERR_INVALID_ARG;
  int sms = 0;
  if (!device_info(&sms)) return GDPA_ERR_UNSUPPORTED;
  const WorkspaceLayout L = make_layout(p, 0, sms);
  if (!workspace || workspace_bytes < L.total) return GDPA_ERR_WORKSPACE;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  DeviceStatus* status = reinterpret_cast<DeviceStatus*>(ws);
  int32_t* order = reinterpret_cast<int32_t*>(ws + L.order);
  int32_t* tile_start = reinterpret_cast<int32_t*>(ws + L.tile_start);
  int4* info = reinterpret_cast<int4*>(ws + L.info);
  const int block_n = forward_block_n(p->D, p->phi, eff_max_kv(p), p->debug_flags);
  cudaStream_t s = (cudaStream_t)stream;

  cudaError_t e = launch_schedule(q_offsets, kv_offsets, p->B, kBlockM, block_n,
                                  p->window_left, p->window_right, tile_start, order, info,
                                  eff_max_q(p), eff_max_kv(p), p->total_q, p->total_kv, status, s);
  if (e != cudaSuccess) return GDPA_ERR_CUDA;
  if (p->B == 0 || p->total_q == 0) return GDPA_OK;

  const bool streamed = rotary_streamed(p->rope_q, p->debug_flags);
  if (streamed) {  // the kernel reads turned copies of Q and K
    void* rq = ws + L.rope_q;
    void* rk = ws + L.rope_k;
    e = turn_qk(p, q, k, rq, rk, 0, sms, s);
    if (e != cudaSuccess) return GDPA_ERR_CUDA;
    q = rq;
    k = rk;
  }
  CUtensorMap tq, tk, tv, to;
  if (!make_map(&tq, q, p->total_q, p->H, p->D, kBlockM)) return GDPA_ERR_CUDA;
  if (!make_map_o(&to, const_cast<void*>(o), p->total_q, p->H, p->D)) return GDPA_ERR_CUDA;
  if (p->total_kv > 0) {
    if (!make_map(&tk, k, p->total_kv, p->H, p->D, block_n)) return GDPA_ERR_CUDA;
    if (!make_map(&tv, v, p->total_kv, p->H, p->D, block_n)) return GDPA_ERR_CUDA;
  } else {
    tk = tq;  // never dereferenced: no sample has a key
    tv = tq;
  }
  FwdArgs a{};
  a.info = info;
  a.status = status;
  a.H = p->H;
  a.n_units = p->B * p->H;
  a.debug_flags = p->debug_flags;
  a.timeout_ns = timeout_ns(p);
  a.p0.bias = bias;
  a.p0.o = static_cast<__nv_bfloat16*>(o);
  a.p0.total_q = p->total_q;
  a.p0.total_kv = p->total_kv;
  a.p0.H = p->H;
  a.p0.bias_kind = p->bias_kind;
  a.p0.wl = p->window_left;
  a.p0.wr = p->window_right;
  a.p0.scale = p->scale;
  if (p->rope_q && !streamed) {  // turned inside the attention kernel
    a.rope_q = static_cast<const uint32_t*>(p->rope_q);
    a.rope_kv = static_cast<const uint32_t*>(p->rope_kv);
  }
  // one launch per activation present (a per-head activation vector groups
  // the heads; each launch walks only its own heads' units)
  for (int phi = 0; phi <= 3; ++phi) {
    const uint64_t heads = phi_heads(p, phi);
    if (!heads) continue;
    a.phi = phi;
    a.head_mask = heads;
    a.p0.phi = phi;
    a.p0.head_mask = heads;
    a.p0.lse = phi == GDPA_PHI_SOFTMAX ? lse : nullptr;
    e = launch_forward(a, p->D, block_n, tq, tk, tv, to, sms, s);
    if (e != cudaSuccess) return GDPA_ERR_CUDA;
  }
  return GDPA_OK;
}

size_t gdpa_backward_grouped_workspace_size(const gdpa_backward_problem_t* problems,
                                            int n_problems) {
  if (!problems || n_problems <= 0 || n_problems > 4096) return 0;
  size_t off = align256(sizeof(DeviceStatus)) + align256((size_t)n_problems * 8);
  for (int i = 0; i < n_problems; ++i) {
    const size_t w = gdpa_workspace_size(&problems[i].params, 1);
    if (w == 0) return 0;
    off += align256(w);
  }
  return off;
}

gdpa_status_t gdpa_backward_grouped(const gdpa_backward_problem_t* problems, int n_problems,
                                    void* workspace, size_t workspace_bytes,
                                    gdpa_stream_t stream) {
  if (!problems || n_problems <= 0 || n_problems > 4096) return GDPA_ERR_INVALID_ARG;
  for (int i = 0; i < n_problems; ++i) {
    const gdpa_backward_problem_t& b = problems[i];
    const gdpa_status_t st =
        check_backward_args(&b.params, b.q, b.k, b.v, b.o, b.dout, b.lse, b.q_offsets,
                            b.kv_offsets, b.bias, b.dq, b.dk, b.dv, b.dbias);
    if (st != GDPA_OK) return st;
  }
  if (!workspace || !aligned16(workspace)) return workspace ? GDPA_ERR_INVALID_ARG
                                                           : GDPA_ERR_WORKSPACE;
  const size_t need = gdpa_backward_grouped_workspace_size(problems, n_problems);
  if (need == 0) return GDPA_ERR_INVALID_ARG;
  if (workspace_bytes < need) return GDPA_ERR_WORKSPACE;
  cudaStream_t s = (cudaStream_t)stream;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  std::vector<uint64_t> offs(n_problems);
  size_t off = align256(sizeof(DeviceStatus)) + align256((size_t)n_problems * 8);
  for (int i = 0; i < n_problems; ++i) {
    offs[i] = off;
    off += align256(gdpa_workspace_size(&problems[i].params, 1));
  }
  // the table is staged before cudaMemcpyAsync returns (pageable host memory)
  uint64_t* table = reinterpret_cast<uint64_t*>(ws + align256(sizeof(DeviceStatus)));
  if (cudaMemsetAsync(ws, 0, sizeof(DeviceStatus), s) != cudaSuccess ||
      cudaMemcpyAsync(table, offs.data(), offs.size() * 8, cudaMemcpyHostToDevice, s) !=
          cudaSuccess)
    return GDPA_ERR_CUDA;
  for (int i = 0; i < n_problems; ++i) {
    const gdpa_backward_problem_t& b = problems[i];
    const size_t w = gdpa_workspace_size(&b.params, 1);
    const gdpa_status_t st =
        gdpa_backward(&b.params, b.q, b.k, b.v, b.o, b.dout, b.lse, b.q_offsets, b.kv_offsets,
                      b.bias, b.dq, b.dk, b.dv, b.dbias, ws + offs[i], w, stream);
    if (st != GDPA_OK) return st;
  }
  return launch_gather_status(reinterpret_cast<DeviceStatus*>(ws), ws, table, n_problems, s) ==
                 cudaSuccess
             ? GDPA_OK
             : GDPA_ERR_CUDA;
}

gdpa_status_t gdpa_backward(const gdpa_params_t* p, const void* q, const void* k, const void* v,
                            const void* o, const void* dout, const float* lse,
                            const int32_t* q_offsets, const int32_t* kv_offsets,
                            const float* bias, void* dq, void* dk, void* dv, float* dbias,
                            void* workspace, size_t workspace_bytes, gdpa_stream_t stream) {
  gdpa_status_t st = check_backward_args(p, q, k, v, o, dout, lse, q_offsets, kv_offsets, bias,
                                         dq, dk, dv, dbias);
  if (st != GDPA_OK) return st;
  if (!aligned16(workspace)) return GDPA_ERR_INVALID_ARG;
  const bool softmax = any_softmax(p);
  int sms = 0;
  if (!device_info(&sms)) return GDPA_ERR_UNSUPPORTED;
  const WorkspaceLayout L = make_layout(p, 1, sms);
  if (!workspace || workspace_bytes < L.total) return GDPA_ERR_WORKSPACE;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  DeviceStatus* status = reinterpret_cast<DeviceStatus*>(ws);
  int32_t* order = reinterpret_cast<int32_t*>(ws + L.order);
  int32_t* tile_start = reinterpret_cast<int32_t*>(ws + L.tile_start);
  int4* info = reinterpret_cast<int4*>(ws + L.info);
  float* delta = reinterpret_cast<float*>(ws + L.delta);
  float* scratch = reinterpret_cast<float*>(ws + L.dq_scratch);
  cudaStream_t s = (cudaStream_t)stream;

  cudaError_t e = launch_schedule(q_offsets, kv_offsets, p->B, kBlockM, 128, p->window_left,
                                  p->window_right, tile_start, order, info, eff_max_q(p),
                                  eff_max_kv(p), p->total_q, p->total_kv, status, s);
  if (e != cudaSuccess) return GDPA_ERR_CUDA;
  if (dbias && p->total_kv > 0) {
    // the kernel adds each key's two column-half sums into it
    e = cudaMemsetAsync(dbias, 0, sizeof(float) * (size_t)p->H * (size_t)p->total_kv, s);
    if (e != cudaSuccess) return GDPA_ERR_CUDA;
  }
  if (p->B == 0 || (p->total_q == 0 && p->total_kv == 0)) return GDPA_OK;
  if (p->rope_q) {  // the attention gradient is taken at the turned Q and K
    void* rq = ws + L.rope_q;
    void* rk = ws + L.rope_k;
    e = turn_qk(p, q, k, rq, rk, 0, sms, s);
    if (e != cudaSuccess) return GDPA_ERR_CUDA;
    q = rq;
    k = rk;
  }
  if (softmax && p->total_q > 0) {
    e = launch_bwd_preprocess(static_cast<const __nv_bfloat16*>(o),
                              static_cast<const __nv_bfloat16*>(dout), delta, p->total_q, p->H,
                              p->D, s);
    if (e != cudaSuccess) return GDPA_ERR_CUDA;
  }
  CUtensorMap tq, tdo, tk, tv;
  if (p->total_q > 0) {
    if (!make_map(&tq, q, p->total_q, p->H, p->D, kBlockM)) return GDPA_ERR_CUDA;
    if (!make_map(&tdo, dout, p->total_q, p->H, p->D, kBlockM)) return GDPA_ERR_CUDA;
  }
  if (p->total_kv > 0) {
    if (!make_map(&tk, k, p->total_kv, p->H, p->D, 128)) return GDPA_ERR_CUDA;
    if (!make_map(&tv, v, p->total_kv, p->H, p->D, 128)) return GDPA_ERR_CUDA;
  }
  if (p->total_q == 0) {  // no query: only zero dK/dV rows are written; maps unused
    tq = tk;
    tdo = tk;
  }
  if (p->total_kv == 0) {  // no key: only zero dQ rows are written; maps unused
    tk = tq;
    tv = tq;
  }
  BwdArgs a{};
  a.q_offsets = q_offsets;
  a.kv_offsets = kv_offsets;
  a.order = order;
  a.info = info;
  a.bias = bias;
  a.lse = lse;
  a.delta = delta;
  a.dq = static_cast<__nv_bfloat16*>(dq);
  a.dk = static_cast<__nv_bfloat16*>(dk);
  a.dv = static_cast<__nv_bfloat16*>(dv);
  a.dbias = dbias;
  a.dq_scratch = scratch;
  a.status = status;
  a.total_q = p->total_q;
  a.total_kv = p->total_kv;
  a.B = p->B;
  a.H = p->H;
  a.n_units = p->B * p->H;
  a.max_q = eff_max_q(p);
  a.max_kv = eff_max_kv(p);
  a.dq_slot_rows = L.dq_slot_rows;
  a.scale = p->scale;
  a.phi = p->phi;
  a.bias_kind = p->bias_kind;
  a.wl = p->window_left;
  a.wr = p->window_right;
  a.debug_flags = p->debug_flags;
  a.timeout_ns = timeout_ns(p);
  // dQ = R^T dQ', dK = R^T dK' (the turn is orthogonal): in the kernel's epilogue
  a.rope_q = static_cast<const uint32_t*>(p->rope_q);
  a.rope_kv = static_cast<const uint32_t*>(p->rope_kv);
  for (int phi = 0; phi <= 3; ++phi) {
    const uint64_t heads = phi_heads(p, phi);
    if (!heads) continue;
    a.phi = phi;
    a.head_mask = heads;
    e = launch_backward(a, p->D, tq, tk, tv, tdo, L.grid, s);
    if (e != cudaSuccess) return GDPA_ERR_CUDA;
  }
  return GDPA_OK;
}

size_t gdpa_forward_grouped_workspace_size(const gdpa_forward_problem_t* problems,
                                           int n_problems) {
  std::vector<LaunchGroup> groups;
  GroupedLayout lay;
  if (plan_grouped(problems, n_problems, groups, lay) != GDPA_OK) return 0;
  return lay.total;
}

gdpa_status_t gdpa_forward_grouped(const gdpa_forward_problem_t* problems, int n_problems,
                                   void* workspace, size_t workspace_bytes,
                                   gdpa_stream_t stream) {
  std::vector<LaunchGroup> groups;
  GroupedLayout lay;
  gdpa_status_t st = plan_grouped(problems, n_problems, groups, lay);
  if (st != GDPA_OK) return st;
  // tensor maps in the workspace must be 64-byte aligned
  if (reinterpret_cast<uintptr_t>(workspace) & 63u) return GDPA_ERR_INVALID_ARG;
  if (!workspace || workspace_bytes < lay.total) return GDPA_ERR_WORKSPACE;
  int sms = 0;
  if (!device_info(&sms)) return GDPA_ERR_UNSUPPORTED;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  DeviceStatus* status = reinterpret_cast<DeviceStatus*>(ws);
  cudaStream_t s = (cudaStream_t)stream;

  // rotary problems: Q and K turned into workspace copies first (one streaming
  // launch each); their tensor maps below read the copies
  std::vector<const void*> qsrc(n_problems), ksrc(n_problems);
  for (int i = 0; i < n_problems; ++i) {
    const gdpa_params_t* p = &problems[i].params;
    qsrc[i] = problems[i].q;
    ksrc[i] = problems[i].k;
    if (!p->rope_q) continue;
    void* rq = ws + lay.rope_q[i];
    void* rk = ws + lay.rope_k[i];
    if (turn_qk(p, problems[i].q, problems[i].k, rq, rk, 0, sms, s) != cudaSuccess)
      return GDPA_ERR_CUDA;
    qsrc[i] = rq;
    ksrc[i] = rk;
  }

  // the cleared status and every table staged on the host, copied in one transfer
  std::vector<uint8_t> host(lay.tables_end, 0);
  auto at = [&](size_t off) { return host.data() + off; };
  GroupSchedJob* jobs = reinterpret_cast<GroupSchedJob*>(at(lay.off_jobs));
  std::vector<int> q_map(groups.size(), -1);
  std::vector<uint64_t> timeouts(groups.size(), 0);
  int max_entries = 1;
  for (size_t gi = 0; gi < groups.size(); ++gi) {
    const LaunchGroup& g = groups[gi];
    const size_t nv = g.vp.size();
    FwdProblem* fp = reinterpret_cast<FwdProblem*>(at(g.off_probs));
    CUtensorMap* maps = reinterpret_cast<CUtensorMap*>(at(g.off_maps));
    GroupSchedProblem* sp = reinterpret_cast<GroupSchedProblem*>(at(g.off_sched));
    int ebase = 0;
    for (size_t j = 0; j < nv; ++j) {
      const VProblem& vp = g.vp[j];
      const gdpa_forward_problem_t& f = problems[vp.src];
      const gdpa_params_t* p = &f.params;
      fp[j].bias = f.bias;
      fp[j].o = static_cast<__nv_bfloat16*>(f.o);
      fp[j].lse = vp.phi == GDPA_PHI_SOFTMAX ? f.lse : nullptr;
      fp[j].total_q = p->total_q;
      fp[j].total_kv = p->total_kv;
      fp[j].H = p->H;
      fp[j].phi = vp.phi;
      fp[j].bias_kind = p->bias_kind;
      fp[j].wl = p->window_left;
      fp[j].wr = p->window_right;
      fp[j].scale = p->scale;
      fp[j].head_mask = vp.heads;
      // encoded into an aligned local object, then copied into the staging bytes
      CUtensorMap m;
      if (p->total_q > 0) {
        if (!make_map(&m, qsrc[vp.src], p->total_q, p->H, p->D, kBlockM)) return GDPA_ERR_CUDA;
        std::memcpy(&maps[4 * j], &m, sizeof(m));
        if (!make_map_o(&m, f.o, p->total_q, p->H, p->D)) return GDPA_ERR_CUDA;
        std::memcpy(&maps[4 * j + 3], &m, sizeof(m));
        if (q_map[gi] < 0) q_map[gi] = (int)j;
      }
      if (p->total_kv > 0) {
        if (!make_map(&m, ksrc[vp.src], p->total_kv, p->H, p->D, g.block_n)) return GDPA_ERR_CUDA;
        std::memcpy(&maps[4 * j + 1], &m, sizeof(m));
        if (!make_map(&m, f.v, p->total_kv, p->H, p->D, g.block_n)) return GDPA_ERR_CUDA;
        std::memcpy(&maps[4 * j + 2], &m, sizeof(m));
      }
      sp[j].q_offsets = f.q_offsets;
      sp[j].kv_offsets = f.kv_offsets;
      sp[j].B = p->B;
      sp[j].ebase = ebase;
      sp[j].wl = p->window_left;
      sp[j].wr = p->window_right;
      sp[j].max_q = eff_max_q(p);
      sp[j].max_kv = eff_max_kv(p);
      sp[j].total_q = p->total_q;
      sp[j].total_kv = p->total_kv;
      ebase += p->B;
      timeouts[gi] = std::max(timeouts[gi], timeout_ns(p));
    }
    // maps of empty tensors are never read; keep every slot a valid map
    if (q_map[gi] >= 0)
      for (size_t j = 0; j < nv; ++j)
        for (int w = 0; w < 4; ++w)
          if (problems[g.vp[j].src].params.total_q == 0 ||
              ((w == 1 || w == 2) && problems[g.vp[j].src].params.total_kv == 0))
            std::memcpy(&maps[4 * j + w], &maps[4 * q_map[gi]], sizeof(CUtensorMap));
    jobs[gi].probs = reinterpret_cast<const GroupSchedProblem*>(ws + g.off_sched);
    jobs[gi].n_probs = (int)nv;
    jobs[gi].n_entries = g.entries;
    jobs[gi].block_n = g.block_n;
    jobs[gi].info = reinterpret_cast<int4*>(ws + g.off_info);
    jobs[gi].eprob = reinterpret_cast<int32_t*>(ws + g.off_eprob);
    max_entries = std::max(max_entries, g.entries);
  }
  if (cudaMemcpyAsync(ws, host.data(), host.size(), cudaMemcpyHostToDevice, s) !=
      cudaSuccess)
    return GDPA_ERR_CUDA;
  cudaError_t e = launch_group_schedule(reinterpret_cast<const GroupSchedJob*>(ws + lay.off_jobs),
                                        (int)groups.size(), max_entries, kBlockM, status, s);
  if (e != cudaSuccess) return GDPA_ERR_CUDA;
  for (size_t gi = 0; gi < groups.size(); ++gi) {
    const LaunchGroup& g = groups[gi];
    if (g.entries == 0 || q_map[gi] < 0) continue;  // no query row in the group
    FwdArgs a{};
    a.info = reinterpret_cast<const int4*>(ws + g.off_info);
    a.status = status;
    a.H = g.hmax;
    a.n_units = g.entries * g.hmax;
    a.phi = g.softmax ? GDPA_PHI_SOFTMAX : GDPA_PHI_SILU;  // launch class only
    a.debug_flags = 0;
    a.timeout_ns = timeouts[gi];
    a.head_mask = ~0ull;
    a.eprob = reinterpret_cast<const int32_t*>(ws + g.off_eprob);
    a.probs = reinterpret_cast<const FwdProblem*>(ws + g.off_probs);
    a.maps = reinterpret_cast<const CUtensorMap*>(ws + g.off_maps);
    CUtensorMap m0;  // kernel parameters, unused when grouped
    std::memcpy(&m0, at(g.off_maps) + 4 * q_map[gi] * sizeof(CUtensorMap), sizeof(m0));
    e = launch_forward(a, g.D, g.block_n, m0, m0, m0, m0, sms, s);
    if (e != cudaSuccess) return GDPA_ERR_CUDA;
  }
  return GDPA_OK;
}

size_t gdpa_rotary_table_bytes(int D, int64_t total) {
  if ((D != 32 && D != 64 && D != 128) || total < 0) return 0;
  return (size_t)total * (size_t)(D / 2) * 4u;
}

gdpa_status_t gdpa_rotary_table(const gdpa_rotary_params_t* r, int B, int64_t total,
                                const int32_t* offsets, const int64_t* time, void* table,
                                gdpa_stream_t stream) {
  if (!r) return GDPA_ERR_INVALID_ARG;
  if (r->D != 32 && r->D != 64 && r->D != 128) return GDPA_ERR_UNSUPPORTED;
  if (!(r->time_scale > 0.f) || !std::isfinite(r->time_scale)) return GDPA_ERR_INVALID_ARG;
  if (B < 0 || B > kMaxSortBatch || total < 0 || total >= (int64_t(1) << 31))
    return GDPA_ERR_INVALID_ARG;
  if (B == 0 || total == 0) return GDPA_OK;
  if (!offsets || !time || !table || !aligned16(table)) return GDPA_ERR_INVALID_ARG;
  RotaryArgs a{};
  a.D = r->D;
  a.B = B;
  a.total = total;
  a.time_scale = r->time_scale;
  const double pi = 3.141592653589793;
  for (int i = 0; i < r->D / 2; ++i) {
    // the default frequencies in fp64; given ones exactly as the caller's floats
    const double th = r->theta ? (double)r->theta[i] : std::pow(10000.0, -2.0 * i / r->D);
    const double ph = r->phi ? (double)r->phi[i] : th;
    if (!std::isfinite(th) || !std::isfinite(ph)) return GDPA_ERR_INVALID_ARG;
    a.theta_hi[i] = (float)(th / pi);
    a.theta_lo[i] = (float)(th / pi - (double)a.theta_hi[i]);
    a.phi_pi[i] = (float)(ph / pi);
  }
  cudaError_t e = launch_rotary_table(a, offsets, time, static_cast<uint32_t*>(table),
                                      (cudaStream_t)stream);
  return e == cudaSuccess ? GDPA_OK : GDPA_ERR_CUDA;
}

gdpa_status_t gdpa_rotary_apply(int64_t total, int H, int D, const void* x, const void* table,
                                void* y, int inverse, gdpa_stream_t stream) {
  if (D != 32 && D != 64 && D != 128) return GDPA_ERR_UNSUPPORTED;
  if (total < 0 || total >= (int64_t(1) << 31) || H <= 0) return GDPA_ERR_INVALID_ARG;
  if (total == 0) return GDPA_OK;
  if (!x || !table || !y || !aligned16(x) || !aligned16(table) || !aligned16(y))
    return GDPA_ERR_INVALID_ARG;
  int sms = 0;
  if (!device_info(&sms)) return GDPA_ERR_UNSUPPORTED;
  RotaryApplyArgs r{};
  r.H = H;
  r.D = D;
  r.inverse = inverse ? 1 : 0;
  r.job[0] = RotaryJob{x, y, static_cast<const uint32_t*>(table), total};
  cudaError_t e = launch_rotary_apply(r, sms, (cudaStream_t)stream);
  return e == cudaSuccess ? GDPA_OK : GDPA_ERR_CUDA;
}

size_t gdpa_sumkron_workspace_size(const gdpa_sumkron_params_t* p) {
  return check_sumkron(p) == GDPA_OK ? sizeof(DeviceStatus) : 0;
}

gdpa_status_t gdpa_sumkron_forward(const gdpa_sumkron_params_t* p, const void* x, const void* a,
                                   const void* w, void* y, void* workspace,
                                   size_t workspace_bytes, gdpa_stream_t stream) {
  gdpa_status_t st = check_sumkron(p);
  if (st != GDPA_OK) return st;
  if (p->B > 0 && (!x || !y)) return GDPA_ERR_INVALID_ARG;
  if (!a || !w || !aligned16(x) || !aligned16(a) || !aligned16(w) || !aligned16(y) ||
      !aligned16(workspace))
    return GDPA_ERR_INVALID_ARG;
  if (!workspace || workspace_bytes < sizeof(DeviceStatus)) return GDPA_ERR_WORKSPACE;
  int sms = 0;
  if (!device_info(&sms)) return GDPA_ERR_UNSUPPORTED;
  cudaStream_t s = (cudaStream_t)stream;
  if (cudaMemsetAsync(workspace, 0, sizeof(DeviceStatus), s) != cudaSuccess) return GDPA_ERR_CUDA;
  if (p->B == 0) return GDPA_OK;
  const cuuint64_t S = p->S, D = p->D, kT = (cuuint64_t)p->k * p->T,
                   kD = (cuuint64_t)p->k * p->D;
  CUtensorMap ta, tx, tw;
  if (!make_map_3d(&ta, a, {S, kT, 1}, {S * 2, S * kT * 2}, {64u, 128u, 1u}) ||
      !make_map_3d(&tx, x, {D, S, (cuuint64_t)p->B}, {D * 2, S * D * 2}, {64u, 64u, 1u}) ||
      !make_map_3d(&tw, w, {D, kD, 1}, {D * 2, kD * D * 2}, {64u, (cuuint32_t)kSumKronWRows, 1u}))
    return GDPA_ERR_CUDA;
  SumKronLaunch L{};
  L.status = static_cast<DeviceStatus*>(workspace);
  L.y = static_cast<__nv_bfloat16*>(y);
  L.B = p->B;
  L.S = p->S;
  L.T = p->T;
  L.D = p->D;
  L.k = p->k;
  L.debug_flags = p->debug_flags;
  L.timeout_ns = (uint64_t)(p->wait_timeout_us > 0 ? p->wait_timeout_us : 2000000) * 1000ull;
  return launch_sumkron(L, ta, tx, tw, sms, s) == cudaSuccess ? GDPA_OK : GDPA_ERR_CUDA;
}


size_t gdpa_sumkron_backward_workspace_size(const gdpa_sumkron_params_t* p) {
  return check_sumkron(p) == GDPA_OK ? sk_bwd_layout(p).end : 0;
}

gdpa_status_t gdpa_sumkron_backward(const gdpa_sumkron_params_t* p, const void* x, const void* a,
                                    const void* w, const void* dy, void* dx, void* da, void* dw,
                                    void* workspace, size_t workspace_bytes,
                                    gdpa_stream_t stream) {
  gdpa_status_t st = check_sumkron(p);
  if (st != GDPA_OK) return st;
  if (p->B > 0 && (!x || !dy || !dx)) return GDPA_ERR_INVALID_ARG;
  if (!a || !w || !da || !dw || !aligned16(x) || !aligned16(a) || !aligned16(w) ||
      !aligned16(dy) || !aligned16(dx) || !aligned16(da) || !aligned16(dw) ||
      !aligned16(workspace))
    return GDPA_ERR_INVALID_ARG;
  const SkBwdLayout L = sk_bwd_layout(p);
  if (!workspace || workspace_bytes < L.end) return GDPA_ERR_WORKSPACE;
  int sms = 0;
  if (!device_info(&sms)) return GDPA_ERR_UNSUPPORTED;
  cudaStream_t s = (cudaStream_t)stream;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  if (cudaMemsetAsync(ws, 0, sizeof(DeviceStatus), s) != cudaSuccess) return GDPA_ERR_CUDA;
  const int B = p->B, S = p->S, T = p->T, D = p->D, k = p->k, kT = k * T;
  if (B == 0) {  // no sample: the parameter gradients are zero
    if (cudaMemsetAsync(da, 0, (size_t)kT * S * 2, s) != cudaSuccess ||
        cudaMemsetAsync(dw, 0, (size_t)k * D * D * 2, s) != cudaSuccess)
      return GDPA_ERR_CUDA;
    return GDPA_OK;
  }
  void* z = ws + L.z;
  void* u = ws + L.u;
  float* pa = reinterpret_cast<float*>(ws + L.pa);
  float* pw = reinterpret_cast<float*>(ws + L.pw);
  const cuuint32_t bT = (cuuint32_t)T;
  CUtensorMap m_ak, m_xmn, m_dyk, m_wk, m_amn, m_umn, m_uk, m_xk, m_zmn, m_dymn;
  if (!sk_map(&m_ak, a, S, kT, 1, 64, 128) ||                    // A [kT][S], K-major (K = s)
      !sk_map(&m_xmn, x, D, S, B, 64, 64) ||                     // X [B][S][D], MN-major (K = s)
      !sk_map(&m_dyk, dy, D, (cuuint64_t)B * T, 1, 64, 128) ||   // dY [B T][D], K-major (K = e)
      !sk_map(&m_wk, w, D, (cuuint64_t)k * D, 1, 64, 128) ||     // W [k D][D], K-major (K = e)
      !sk_map(&m_amn, a, S, kT, 1, 64, 64) ||                    // A, MN-major (M = s, K = r t)
      !sk_map(&m_umn, u, D, kT, B, 64, 64) ||                    // U [B][kT][D], MN-major
      !sk_map(&m_uk, u, D, kT, B, 64, 128) ||                    // U, K-major (K = d)
      !sk_map(&m_xk, x, D, S, B, 64, 128) ||                     // X, K-major (K = d)
      !sk_map(&m_zmn, z, D, kT, B, 64, bT) ||                    // Z [B][kT][D], MN-major (K = t)
      !sk_map(&m_dymn, dy, D, T, B, 64, bT))                     // dY [B][T][D], MN-major (K = t)
    return GDPA_ERR_CUDA;
  GemmLaunch g{};
  g.status = reinterpret_cast<DeviceStatus*>(ws);
  g.timeout_ns = (uint64_t)(p->wait_timeout_us > 0 ? p->wait_timeout_us : 2000000) * 1000ull;
  auto run = [&](const CUtensorMap& ta, const CUtensorMap& tb) {
    return launch_gemm(g, ta, tb, sms, s) == cudaSuccess;
  };
  // Z_b = A X_b: M = kT, N = D, K = S; per sample
  g.M = kT; g.N = D; g.Z = B; g.n_rb = 1; g.nkc = S / 64; g.kc = 64; g.splits = 1;
  g.a = GemmOperand{0, 0, 0};
  g.b = GemmOperand{1, 0, 2};
  g.f32_out = 0; g.out = z; g.mT = kT; g.nD = D;
  g.sZ = (int64_t)kT * D; g.sMb = 0; g.sMt = D; g.sNr = 0;
  if (!run(m_ak, m_xmn)) return GDPA_ERR_CUDA;
  // U = dY [W_1 ... W_k]^T: M = B T rows (b, t), N = k D columns (r, d), K = D;
  // row (b, t), column (r, d) stored at U[b][r][t][d]
  g.M = B * T; g.N = k * D; g.Z = 1; g.n_rb = 1; g.nkc = D / 64; g.kc = 64; g.splits = 1;
  g.a = GemmOperand{0, 0, 0};
  g.b = GemmOperand{0, 0, 0};
  g.f32_out = 0; g.out = u; g.mT = T; g.nD = D;
  g.sZ = 0; g.sMb = (int64_t)kT * D; g.sMt = D; g.sNr = (int64_t)T * D;
  if (!run(m_dyk, m_wk)) return GDPA_ERR_CUDA;
  // dX_b = A^T U_b: M = S, N = D, K = kT; per sample
  g.M = S; g.N = D; g.Z = B; g.n_rb = 1; g.nkc = kT / 64; g.kc = 64; g.splits = 1;
  g.a = GemmOperand{1, 0, 0};
  g.b = GemmOperand{1, 0, 2};
  g.f32_out = 0; g.out = dx; g.mT = S; g.nD = D;
  g.sZ = (int64_t)S * D; g.sMb = 0; g.sMt = D; g.sNr = 0;
  if (!run(m_amn, m_umn)) return GDPA_ERR_CUDA;
  // dA = sum_b U_b X_b^T: M = kT, N = S, K = D per sample, samples split
  const int spa = sk_splits_a(B);
  g.M = kT; g.N = S; g.Z = 1; g.n_rb = B; g.nkc = D / 64; g.kc = 64; g.splits = spa;
  g.a = GemmOperand{0, 0, 1};
  g.b = GemmOperand{0, 0, 1};
  g.f32_out = 1; g.out = pa;
  if (!run(m_uk, m_xk)) return GDPA_ERR_CUDA;
  if (launch_sum_splits(pa, spa, (int64_t)kT * S, static_cast<__nv_bfloat16*>(da), sms, s) !=
      cudaSuccess)
    return GDPA_ERR_CUDA;
  // dW_r = sum_b Z_b[r]^T dY_b: M = N = D, K = T per sample, per r, samples split
  const int spw = sk_splits_w(B);
  g.M = D; g.N = D; g.Z = k; g.n_rb = B; g.nkc = 1; g.kc = T; g.splits = spw;
  g.a = GemmOperand{1, T, 1};
  g.b = GemmOperand{1, 0, 1};
  g.f32_out = 1; g.out = pw;
  if (!run(m_zmn, m_dymn)) return GDPA_ERR_CUDA;
  if (launch_sum_splits(pw, spw, (int64_t)k * D * D, static_cast<__nv_bfloat16*>(dw), sms, s) !=
      cudaSuccess)
    return GDPA_ERR_CUDA;
  return GDPA_OK;
}

gdpa_status_t gdpa_get_device_status(const void* workspace, gdpa_stream_t stream) {
  if (!workspace || !aligned16(workspace)) return GDPA_ERR_INVALID_ARG;
  if (cudaStreamSynchronize((cudaStream_t)stream) != cudaSuccess) return GDPA_ERR_CUDA;
  DeviceStatus st;
  if (cudaMemcpy(&st, workspace, sizeof(st), cudaMemcpyDeviceToHost) != cudaSuccess)
    return GDPA_ERR_CUDA;
  return (gdpa_status_t)st.code;
}

}  // extern "C"
