// gdpa_bwd.cu -- fused GDPA backward for sm_100a, and its delta preprocess.
//
// Gradient of O = phi(scale * Q K^T + beta) V (Kunlun paper review §2.3
// "GDPA", Fig. 2; the fused kernel avoids materialising large intermediates in
// the backward pass).  Per visible pair (i, j):
//   s = scale q_i.k_j + beta_j,  p = phi(s)
//   dV_j += p dO_i,  dP = dO_i . V_j
//   dS = p (dP - delta_i) with delta_i = dO_i . O_i   (softmax, p = exp(s - LSE_i))
//      = dP * (sigma(s) + s sigma(s)(1 - sigma(s)))   (SiLU)
//      = dP                                           (identity)
//   dK_j += scale dS q_i,  dQ_i += scale dS k_j
//
// One persistent CTA per SM walks (sample, head) units longest first.  Within
// a unit the key blocks (128 keys) are the outer loop and the query tiles that
// can see the block (128 queries) the inner loop, so dK and dV accumulate in
// TMEM across all of the sample's queries and are written once.  dQ for a
// (key block, query tile) pair is produced in TMEM and summed over key blocks
// in a per-CTA fp32 scratch slot; the thread that writes a scratch element is
// the thread that reads it back, so no atomics or fences are needed, and the
// slot (rows = max query length) stays in L2.
//
// TMEM (512 columns): [0,128) S^T, later dQ; [128,256) dP^T, then P^T (bf16,
// the A operand of the dV MMA); then dK, dV.
// Shared memory: K, V of the key block; a 2-stage ring of Q, dO tiles; dS^T
// (bf16, 64-query panels, 128-byte swizzle) for the dK and dQ MMAs.
//
// Warp roles (384 threads): 0 TMA producer, 1 MMA issuer, 2 TMEM allocator,
// 3 LSE/delta loader, 4-11 two warpgroups that split each tile's 128 query
// columns (and the D columns of dQ, dK, dV) between them.
#include <climits>

#include "gdpa_internal.h"

namespace gdpa {
namespace {

constexpr int kBwdThreads = 384;
constexpr int kRegsLaunch = 168;   // 65536 / 384 rounded down to a multiple of 8
constexpr int kRegsControl = 88;   // warpgroup 0
constexpr int kRegsPhi = 208;      // warpgroups 1 and 2
static_assert(128 * kRegsControl + 256 * kRegsPhi <= kBwdThreads * kRegsLaunch,
              "register split exceeds the launch's registers");
constexpr float kLog2eB = 1.4426950408889634f;
constexpr float kInvSqrt2Pi = 0.3989422804014327f;  // 1 / sqrt(2 pi)
constexpr float kInvSqrt2 = 0.7071067811865476f;    // Phi(x) = (1 + erf(x / sqrt 2)) / 2

template <int D_>
struct BwdCfg {
  static constexpr int D = D_;
  static constexpr int BM = kBlockM;   // queries per tile
  static constexpr int BN = 128;       // keys per block
  static constexpr int PANEL_ELEMS = D >= 64 ? 64 : 32;
  static constexpr int PANEL_BYTES = PANEL_ELEMS * 2;
  static constexpr int NPANEL = D / PANEL_ELEMS;
  static constexpr uint32_t LAYOUT = D >= 64 ? LAYOUT_SW128 : LAYOUT_SW64;
  static constexpr int KV_BYTES = BN * D * 2;
  static constexpr int QT_BYTES = BM * D * 2;
  static constexpr int PT_BYTES = BN * BM * 2;
  static constexpr int NQ = 2;         // Q/dO ring stages
  static constexpr int OFF_K = 0;
  static constexpr int OFF_V = OFF_K + KV_BYTES;
  static constexpr int OFF_Q = OFF_V + KV_BYTES;                 // [NQ] Q tiles
  static constexpr int OFF_DO = OFF_Q + NQ * QT_BYTES;           // [NQ] dO tiles
  static constexpr int OFF_DST = OFF_DO + NQ * QT_BYTES;
  static constexpr int OFF_ROW = OFF_DST + PT_BYTES;   // float [2][2][BM]: LSE*log2e, delta
  static constexpr int OFF_BAR = OFF_ROW + 2 * 2 * BM * 4;
  static constexpr int B_KVFULL = 0, B_KVEMPTY = 1, B_QFULL = 2, B_QEMPTY = 4, B_SFULL = 6,
                       B_PFULL = 7, B_DQFULL = 8, B_DQEMPTY = 9, B_DKVFULL = 10,
                       B_DKVEMPTY = 11, B_RFULL = 12, B_REMPTY = 14, NBARS = 16;
  static constexpr int OFF_MISC = OFF_BAR + NBARS * 8;
  static constexpr int SMEM_BYTES = OFF_MISC + 16;
  static constexpr int SMEM_ALLOC = SMEM_BYTES;  // base is 1024-aligned (checked at entry)
  static constexpr int T_S = 0, T_DP = 128, T_PT = 128, T_DK = 256, T_DV = 256 + D;
  static constexpr int TMEM_COLS = 512;
  static_assert(SMEM_ALLOC <= 232448, "shared memory budget");
};

using BUnit = GdpaUnit;

// Key blocks [kb0, kb1) query tile m0 may see (same rule as the forward).
__device__ __forceinline__ void bwd_kv_range(int m0, int Lk, int wl, int wr, int& kb0, int& kb1) {
  int lo = wl >= 0 ? max(0, m0 - wl) : 0;
  int hi = wr >= 0 ? min(Lk, m0 + kBlockM + wr) : Lk;
  if (hi <= lo) {
    kb0 = kb1 = 0;
  } else {
    kb0 = lo / 128;
    kb1 = (hi + 127) / 128;
  }
}

template <class C>
struct BSmem {
  uint32_t base;
  uint8_t* ptr;
  __device__ uint32_t k() const { return base + C::OFF_K; }
  __device__ uint32_t v() const { return base + C::OFF_V; }
  __device__ uint32_t q(int s) const { return base + C::OFF_Q + s * C::QT_BYTES; }
  __device__ uint32_t dout(int s) const { return base + C::OFF_DO + s * C::QT_BYTES; }
  __device__ uint32_t dst() const { return base + C::OFF_DST; }
  __device__ float* lse2(int s) const {
    return reinterpret_cast<float*>(ptr + C::OFF_ROW) + s * 2 * C::BM;
  }
  __device__ float* delta(int s) const { return lse2(s) + C::BM; }
  __device__ uint32_t bar(int i) const { return base + C::OFF_BAR + i * 8; }
  __device__ uint32_t* tmem_slot() const { return reinterpret_cast<uint32_t*>(ptr + C::OFF_MISC); }
  __device__ volatile int* abort_flag() const {
    return reinterpret_cast<volatile int*>(ptr + C::OFF_MISC + 4);
  }
};

// Iterate the (key block, query tile) pairs of a unit in the order every role
// uses.  f(kb, mt, first_tile_of_block, last_tile_of_block) for pairs;
// g(kb) for blocks that no tile sees.
template <class F, class G>
__device__ __forceinline__ bool for_each_pair(const BUnit& t, int wl, int wr, F&& f, G&& g) {
  const int ntile = (t.Lq + kBlockM - 1) / kBlockM;
  const int nkb = (t.Lk + 127) / 128;
  for (int kb = 0; kb < nkb; ++kb) {
    int first = -1, last = -1;
    for (int mt = 0; mt < ntile; ++mt) {
      int a0, a1;
      bwd_kv_range(mt * kBlockM, t.Lk, wl, wr, a0, a1);
      if (kb >= a0 && kb < a1) {
        if (first < 0) first = mt;
        last = mt;
      }
    }
    if (first < 0) {
      if (!g(kb)) return false;
      continue;
    }
    for (int mt = first; mt <= last; ++mt) {
      int a0, a1;
      bwd_kv_range(mt * kBlockM, t.Lk, wl, wr, a0, a1);
      if (kb < a0 || kb >= a1) continue;
      if (!f(kb, mt, mt == first, mt == last)) return false;
    }
  }
  return true;
}

// ------------------------------------------------------------------ producer
template <class C>
__device__ void bwd_producer(const BwdArgs& a, const BSmem<C>& sm, const CUtensorMap* tq,
                             const CUtensorMap* tk, const CUtensorMap* tv,
                             const CUtensorMap* tdo) {
  volatile int* abort = sm.abort_flag();
  const uint64_t pol_stream = l2_policy_evict_first();
  const uint64_t pol_keep = l2_policy_evict_last();
  uint32_t kvi = 0, qi = 0;
  bool dropped = false;
  UnitStream units(a.info, a.H, a.n_units, a.head_mask);
  BUnit t;
  while (units.next(t)) {
    bool ok = for_each_pair(
        t, a.wl, a.wr,
        [&](int kb, int mt, bool first, bool) -> bool {
          if (first) {
            if (!mbar_wait(sm.bar(C::B_KVEMPTY), (kvi & 1) ^ 1, abort, a.status, a.timeout_ns,
                           0x1000 + C::B_KVEMPTY))
              return false;
            mbar_arrive_expect_tx(sm.bar(C::B_KVFULL), 2 * C::KV_BYTES);
            for (int p = 0; p < C::NPANEL; ++p) {
              tma_load_3d(sm.k() + p * C::BN * C::PANEL_BYTES, tk, sm.bar(C::B_KVFULL),
                          p * C::PANEL_ELEMS, t.h, t.k0 + kb * C::BN, pol_keep);
              tma_load_3d(sm.v() + p * C::BN * C::PANEL_BYTES, tv, sm.bar(C::B_KVFULL),
                          p * C::PANEL_ELEMS, t.h, t.k0 + kb * C::BN, pol_keep);
            }
            ++kvi;
            // warm L2 with the key block that follows (this unit's next block or
            // the next unit's first), whose load waits for this block's release
            const int nkb = (t.Lk + C::BN - 1) / C::BN;
            BUnit nt = t;
            int nb = kb + 1;
            if (nb >= nkb) {
              nb = 0;
              if (!units.peek(nt)) nt.Lk = 0;
            }
            if (nb * C::BN < nt.Lk) {
              for (int p = 0; p < C::NPANEL; ++p) {
                tma_prefetch_l2_3d(tk, p * C::PANEL_ELEMS, nt.h, nt.k0 + nb * C::BN, pol_keep);
                tma_prefetch_l2_3d(tv, p * C::PANEL_ELEMS, nt.h, nt.k0 + nb * C::BN, pol_keep);
              }
            }
          }
          const int qs = qi % C::NQ;
          if (!mbar_wait(sm.bar(C::B_QEMPTY + qs), ((qi / C::NQ) & 1) ^ 1, abort, a.status,
                         a.timeout_ns, 0x1000 + C::B_QEMPTY + qs))
            return false;
          if ((a.debug_flags & 1) && !dropped && blockIdx.x == 0) {
            dropped = true;  // test hook: this Q/dO tile is never loaded
            ++qi;
            return true;
          }
          mbar_arrive_expect_tx(sm.bar(C::B_QFULL + qs), 2 * C::QT_BYTES);
          for (int p = 0; p < C::NPANEL; ++p) {
            tma_load_3d(sm.q(qs) + p * C::BM * C::PANEL_BYTES, tq, sm.bar(C::B_QFULL + qs),
                        p * C::PANEL_ELEMS, t.h, t.q0 + mt * kBlockM, pol_stream);
            tma_load_3d(sm.dout(qs) + p * C::BM * C::PANEL_BYTES, tdo, sm.bar(C::B_QFULL + qs),
                        p * C::PANEL_ELEMS, t.h, t.q0 + mt * kBlockM, pol_stream);
          }
          ++qi;
          return true;
        },
        [&](int) { return true; });
    if (!ok) return;
  }
}

// ------------------------------------------------------------------ MMA issuer
template <class C>
__device__ void bwd_mma(const BwdArgs& a, const BSmem<C>& sm, uint32_t tmem) {
  volatile int* abort = sm.abort_flag();
  constexpr uint32_t id_st = make_idesc_bf16(128, kBlockM, 0, 0);  // S^T, dP^T
  constexpr uint32_t id_kv = make_idesc_bf16(128, C::D, 0, 1);     // dV, dK
  constexpr uint32_t id_dq = make_idesc_bf16(kBlockM, C::D, 1, 1);  // dQ
  constexpr uint32_t SBO = 8 * C::PANEL_BYTES;
  uint32_t kvi = 0, qi = 0, pi = 0, dqi = 0, bi = 0;
  UnitStream units(a.info, a.H, a.n_units, a.head_mask);
  BUnit t;
  while (units.next(t)) {
    bool ok = for_each_pair(
        t, a.wl, a.wr,
        [&](int kb, int mt, bool first, bool last) -> bool {
          (void)kb;
          (void)mt;
          if (first) {
            if (!mbar_wait(sm.bar(C::B_KVFULL), kvi & 1, abort, a.status, a.timeout_ns,
                           0x1100 + C::B_KVFULL))
              return false;
          }
          const int qs = qi % C::NQ;
          if (!mbar_wait(sm.bar(C::B_QFULL + qs), (qi / C::NQ) & 1, abort, a.status,
                         a.timeout_ns, 0x1100 + C::B_QFULL + qs))
            return false;
          // S^T and dP^T regions are free once the previous dQ has been read
          if (!mbar_wait(sm.bar(C::B_DQEMPTY), (dqi & 1) ^ 1, abort, a.status, a.timeout_ns,
                         0x1100 + C::B_DQEMPTY))
            return false;
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < C::D / 16; ++kk) {
            const int p = kk * 16 / C::PANEL_ELEMS;
            const int w = (kk * 16 % C::PANEL_ELEMS) * 2;
            const uint64_t dk_ = make_smem_desc(sm.k() + p * C::BN * C::PANEL_BYTES + w, 16, SBO,
                                                C::LAYOUT);
            const uint64_t dq_ = make_smem_desc(sm.q(qs) + p * C::BM * C::PANEL_BYTES + w, 16,
                                                SBO, C::LAYOUT);
            mma_bf16_ss(tmem + C::T_S, dk_, dq_, id_st, kk > 0 ? 1u : 0u);
          }
#pragma unroll
          for (int kk = 0; kk < C::D / 16; ++kk) {
            const int p = kk * 16 / C::PANEL_ELEMS;
            const int w = (kk * 16 % C::PANEL_ELEMS) * 2;
            const uint64_t dv_ = make_smem_desc(sm.v() + p * C::BN * C::PANEL_BYTES + w, 16, SBO,
                                                C::LAYOUT);
            const uint64_t do_ = make_smem_desc(sm.dout(qs) + p * C::BM * C::PANEL_BYTES + w,
                                                16, SBO, C::LAYOUT);
            mma_bf16_ss(tmem + C::T_DP, dv_, do_, id_st, kk > 0 ? 1u : 0u);
          }
          mma_commit(sm.bar(C::B_SFULL));
          // P^T, dS^T written by the phi warpgroups
          if (!mbar_wait(sm.bar(C::B_PFULL), pi & 1, abort, a.status, a.timeout_ns,
                         0x1100 + C::B_PFULL))
            return false;
          ++pi;
          if (first && !mbar_wait(sm.bar(C::B_DKVEMPTY), (bi & 1) ^ 1, abort, a.status,
                                  a.timeout_ns, 0x1100 + C::B_DKVEMPTY))
            return false;
          tc_fence_after();
          // dV += P^T dO (P^T from TMEM) ; dK += dS^T Q   (K = 128 queries)
#pragma unroll
          for (int kk = 0; kk < kBlockM / 16; ++kk) {
            const uint32_t a_off = (kk * 16 / 64) * (128 * 128) + (kk * 16 % 64) * 2;
            const uint64_t sa = make_smem_desc(sm.dst() + a_off, 16, 1024, LAYOUT_SW128);
            const uint64_t ob = make_smem_desc(sm.dout(qs) + kk * 16 * C::PANEL_BYTES,
                                               C::BM * C::PANEL_BYTES, SBO, C::LAYOUT);
            const uint64_t qb = make_smem_desc(sm.q(qs) + kk * 16 * C::PANEL_BYTES,
                                               C::BM * C::PANEL_BYTES, SBO, C::LAYOUT);
            const uint32_t acc = (!first || kk > 0) ? 1u : 0u;
            // queries 16kk..16kk+15 of P^T: warpgroup kk/4's columns, 8 per step
            mma_bf16_ts(tmem + C::T_DV, tmem + C::T_PT + (kk / 4) * 64 + (kk % 4) * 8, ob, id_kv,
                        acc);
            mma_bf16_ss(tmem + C::T_DK, sa, qb, id_kv, acc);
          }
          mma_commit(sm.bar(C::B_QEMPTY + qs));
          ++qi;
          // dQ = dS K   (M = 128 queries from dS^T, MN-major; K = 128 keys)
#pragma unroll
          for (int kk = 0; kk < C::BN / 16; ++kk) {
            const uint64_t sa = make_smem_desc(sm.dst() + kk * 16 * 128, 128 * 128, 1024,
                                               LAYOUT_SW128);
            const uint64_t kb_ = make_smem_desc(sm.k() + kk * 16 * C::PANEL_BYTES,
                                                C::BN * C::PANEL_BYTES, SBO, C::LAYOUT);
            mma_bf16_ss(tmem + C::T_S, sa, kb_, id_dq, kk > 0 ? 1u : 0u);
          }
          mma_commit(sm.bar(C::B_DQFULL));
          ++dqi;
          if (last) {
            mma_commit(sm.bar(C::B_DKVFULL));
            mma_commit(sm.bar(C::B_KVEMPTY));
            ++kvi;
            ++bi;
          }
          return true;
        },
        [&](int) { return true; });
    if (!ok) return;
  }
}

// ------------------------------------------------------------------ LSE / delta loader
template <class C>
__device__ void bwd_rows(const BwdArgs& a, const BSmem<C>& sm) {
  volatile int* abort = sm.abort_flag();
  const int lane = threadIdx.x & 31;
  uint32_t ri = 0;
  UnitStream units(a.info, a.H, a.n_units, a.head_mask);
  BUnit t;
  while (units.next(t)) {
    bool ok = for_each_pair(
        t, a.wl, a.wr,
        [&](int, int mt, bool, bool) -> bool {
          const int s = ri & 1;
          bool w = mbar_wait(sm.bar(C::B_REMPTY + s), ((ri >> 1) & 1) ^ 1, abort, a.status,
                             a.timeout_ns, 0x1300 + C::B_REMPTY + s);
          if (!__all_sync(0xffffffffu, w)) return false;
          float* l2 = sm.lse2(s);
          float* dl = sm.delta(s);
          for (int c = lane; c < C::BM; c += 32) {
            const int i = mt * kBlockM + c;
            float x = 0.f, d = 0.f;
            if (i < t.Lq) {
              const int64_t idx = (int64_t)t.h * a.total_q + t.q0 + i;
              x = a.lse[idx] * kLog2eB;
              d = a.delta[idx];
            }
            l2[c] = x;
            dl[c] = d;
          }
          mbar_arrive(sm.bar(C::B_RFULL + s));
          ++ri;
          return true;
        },
        [&](int) { return true; });
    if (!ok) return;
  }
}

// Read NCOL (16 or 32 multiple) fp32 columns of this thread's TMEM lane.
template <int NCOL>
__device__ __forceinline__ void tmem_row(uint32_t taddr, float (&out)[NCOL]) {
  if constexpr (NCOL % 32 == 0) {
#pragma unroll
    for (int c = 0; c < NCOL / 32; ++c) {
      uint32_t r[32];
      tmem_ld32(taddr + c * 32, r);
      tmem_wait_ld();
#pragma unroll
      for (int e = 0; e < 32; ++e) out[c * 32 + e] = __uint_as_float(r[e]);
    }
  } else {
    static_assert(NCOL == 16, "16 or a multiple of 32 columns");
    uint32_t r[16];
    tmem_ld16(taddr, r);
    tmem_wait_ld();
#pragma unroll
    for (int e = 0; e < 16; ++e) out[e] = __uint_as_float(r[e]);
  }
}

// ------------------------------------------------------------------ phi warpgroups
template <class C, int PHI>
__device__ void bwd_phi(const BwdArgs& a, const BSmem<C>& sm, uint32_t tmem) {
  volatile int* abort = sm.abort_flag();
  const int g = ((threadIdx.x >> 5) - 4) >> 2;    // warpgroup 0 or 1
  const int wq = (threadIdx.x >> 5) & 3;          // TMEM lane quarter
  const int lane = threadIdx.x & 31;
  const int r = wq * 32 + lane;                   // key row (S^T) or query row (dQ)
  const uint32_t tl = (uint32_t)(wq * 32) << 16;
  const int ctid = threadIdx.x - 128;             // 0..255 among the phi threads
  constexpr int HALF_D = C::D / 2;
  constexpr bool SOFTMAX = PHI == 1;
  const float sc = SOFTMAX ? a.scale * kLog2eB : a.scale;
  const uint64_t pol_keep = l2_policy_evict_last();
  uint32_t si = 0, dqi = 0, bi = 0, ri = 0;

#define BWD_WAIT(bar_, par_, where_)                                                     \
  do {                                                                                 \
    bool ok_ = mbar_wait(sm.bar(bar_), (par_), abort, a.status, a.timeout_ns, where_);  \
    if (!__all_sync(0xffffffffu, ok_)) return false;                                   \
  } while (0)

  int64_t pre_idx = -1;  // bias element fetched ahead (pre_val), or -1
  float pre_val = 0.f;
  UnitStream units(a.info, a.H, a.n_units, a.head_mask);
  BUnit t;
  while (units.next(t)) {
    // dQ rows of query tiles that no key block reaches are zero
    {
      const int ntile = (t.Lq + kBlockM - 1) / kBlockM;
      for (int mt = 0; mt < ntile; ++mt) {
        int a0, a1;
        bwd_kv_range(mt * kBlockM, t.Lk, a.wl, a.wr, a0, a1);
        if (a1 > a0) continue;
        const int rows = min(kBlockM, t.Lq - mt * kBlockM);
        for (int idx = ctid; idx < rows * (C::D / 8); idx += 256) {
          const int rr = idx / (C::D / 8), cc = (idx % (C::D / 8)) * 8;
          *reinterpret_cast<uint4*>(a.dq + ((int64_t)(t.q0 + mt * kBlockM + rr) * a.H + t.h) *
                                                 C::D + cc) = make_uint4(0, 0, 0, 0);
        }
      }
    }
    float beta = 0.f;
    float graw = 0.f;  // this key's raw bias (gate) value
    float dsum = 0.f;  // this key's sum of dS over this warpgroup's query columns
    bool ok = for_each_pair(
        t, a.wl, a.wr,
        [&](int kb, int mt, bool first, bool last) -> bool {
          const int key = kb * C::BN + r;   // this thread's key (S^T row)
          if (first) dsum = 0.f;
          if (first && a.bias_kind != 0) {
            // this key block's raw bias, fetched one key block ahead
            float gv = 0.f;
            const int64_t gi = key < t.Lk ? (int64_t)t.h * a.total_kv + t.k0 + key : -1;
            if (gi >= 0) gv = gi == pre_idx ? pre_val : a.bias[gi];
            beta = 0.f;
            if (gi >= 0) beta = a.bias_kind == 2 ? fminf(gv, 0.f) - log1pf(__expf(-fabsf(gv))) : gv;
            graw = gv;
            if (SOFTMAX) beta *= kLog2eB;
            // the next key block of this unit, else the next unit's first
            pre_idx = -1;
            if ((kb + 1) * C::BN < t.Lk) {
              if ((kb + 1) * C::BN + r < t.Lk) pre_idx = gi + C::BN;
            } else {
              BUnit nt;
              if (units.peek(nt) && r < nt.Lk) pre_idx = (int64_t)nt.h * a.total_kv + nt.k0 + r;
            }
            if (pre_idx >= 0) pre_val = a.bias[pre_idx];
          }
          const int m0 = mt * kBlockM;
          const int rs = ri & 1;
          if (SOFTMAX) BWD_WAIT(C::B_RFULL + rs, (ri >> 1) & 1, 0x1400 + C::B_RFULL + rs);
          BWD_WAIT(C::B_SFULL, si & 1, 0x1400 + C::B_SFULL);
          ++si;
          tc_fence_after();
          const float* l2 = sm.lse2(rs);
          const float* dl = sm.delta(rs);
          // visible queries of this key: i in [qlo, qhi]
          int qlo = 0, qhi = t.Lq - 1;
          if (a.wr >= 0) qlo = max(qlo, key - a.wr);
          if (a.wl >= 0) qhi = min(qhi, key + a.wl);
          if (key >= t.Lk) qhi = -1;
#pragma unroll
          for (int ch = 0; ch < 2; ++ch) {
            const int c0 = g * 64 + ch * 32;   // first query column of this chunk
            float s[32], dp[32];
            {
              uint32_t r1[32], r2[32];
              tmem_ld32(tmem + tl + C::T_S + c0, r1);
              tmem_ld32(tmem + tl + C::T_DP + c0, r2);
              tmem_wait_ld();
#pragma unroll
              for (int e = 0; e < 32; ++e) {
                s[e] = __uint_as_float(r1[e]);
                dp[e] = __uint_as_float(r2[e]);
              }
            }
#pragma unroll
            for (int e = 0; e < 32; ++e) {
              const int i = m0 + c0 + e;
              const bool vis = i >= qlo && i <= qhi;
              const float x = fmaf(s[e], sc, beta);
              float p, ds;
              if (PHI == 1) {
                p = ex2_approx(x - l2[c0 + e]);
                ds = p * (dp[e] - dl[c0 + e]);
              } else if (PHI == 0) {
                const float hx = 0.5f * x;
                const float th = tanh_approx(hx);
                const float sg = fmaf(0.5f, th, 0.5f);       // sigmoid(x)
                p = x * sg;
                ds = dp[e] * fmaf(x * sg, 1.f - sg, sg);      // sg + x sg (1 - sg)
              } else if (PHI == 3) {
                // gelu(x) = x Phi(x); gelu'(x) = Phi(x) + x phi(x), phi the
                // standard normal density exp(-x^2 / 2) / sqrt(2 pi)
                const float cdf = fmaf(0.5f, erff(x * kInvSqrt2), 0.5f);
                p = x * cdf;
                ds = dp[e] * fmaf(x, kInvSqrt2Pi * __expf(-0.5f * x * x), cdf);
              } else {
                p = x;
                ds = dp[e];
              }
              s[e] = vis ? p : 0.f;
              dp[e] = vis ? ds : 0.f;
              dsum += dp[e];
            }
            // P^T row -> TMEM, two bf16 per column, into this warpgroup's own dP^T
            // columns that have already been read: queries 64g+32ch.. at column
            // T_PT + 64g + 16ch
            {
              uint32_t pk[16];
#pragma unroll
              for (int e = 0; e < 16; ++e) pk[e] = pack_bf16x2(s[2 * e], s[2 * e + 1]);
              tmem_st16(tmem + tl + C::T_PT + g * 64 + ch * 16, pk);
            }
            // dS^T row -> panel g (queries 64g .. 64g+63), 128-byte swizzle
#pragma unroll
            for (int q8 = 0; q8 < 4; ++q8) {
              const int cir = ch * 4 + q8;    // 16-byte chunk within the 128-byte row
              const uint32_t off = g * (128 * 128) + r * 128 + ((cir ^ (r & 7)) << 4);
              st_shared_v4(sm.dst() + off, pack_bf16x2(dp[q8 * 8 + 0], dp[q8 * 8 + 1]),
                           pack_bf16x2(dp[q8 * 8 + 2], dp[q8 * 8 + 3]),
                           pack_bf16x2(dp[q8 * 8 + 4], dp[q8 * 8 + 5]),
                           pack_bf16x2(dp[q8 * 8 + 6], dp[q8 * 8 + 7]));
            }
          }
          tmem_wait_st();
          fence_proxy_async_smem();
          tc_fence_before();
          if (SOFTMAX) {
            mbar_arrive(sm.bar(C::B_REMPTY + rs));
          }
          ++ri;
          mbar_arrive(sm.bar(C::B_PFULL));
          // dQ of this pair: thread = query row, columns [g*D/2, (g+1)*D/2).
          // Partial dQ across key blocks lives in this CTA's scratch slot laid out
          // thread-major ([tile][half g][16-byte chunk][row]) so each warp access
          // is 512 contiguous bytes.  Only this thread reads what it wrote; the
          // slot stays in L2 (evict-last) and is discarded after its last read.
          // The earlier blocks' partial is fetched now, while the dV, dK and dQ
          // MMAs run, so its latency is off the path.
          int b0, b1;
          bwd_kv_range(m0, t.Lk, a.wl, a.wr, b0, b1);
          const bool dq_first = kb == b0, dq_last = kb == b1 - 1;
          constexpr int NCH4 = HALF_D / 4;
          float4* scr4 = reinterpret_cast<float4*>(a.dq_scratch) +
                         ((((int64_t)blockIdx.x * (a.dq_slot_rows / kBlockM) + mt) * 2 + g) *
                          NCH4) * kBlockM + r;
          float4 part[NCH4];
          if (!dq_first) {
#pragma unroll
            for (int c = 0; c < NCH4; ++c)
              part[c] = ld_global_v4_hint(reinterpret_cast<const float*>(scr4 + c * kBlockM),
                                          pol_keep);
          }
          BWD_WAIT(C::B_DQFULL, dqi & 1, 0x1400 + C::B_DQFULL);
          ++dqi;
          tc_fence_after();
          {
            // 32 columns (8 float4 of the partial) at a time; the last chunk's TMEM
            // read releases the dQ columns.  The final rows (bf16) are staged in
            // this warp's own dS^T rows (free once the dQ MMA completed), then
            // written as whole row segments.
            constexpr int CW = HALF_D < 32 ? HALF_D : 32;
            constexpr int NCHUNK = HALF_D / CW;
            constexpr int CPR = HALF_D * 2 / 16;          // 16-byte chunks per half row
            constexpr int SWM = (CPR >= 8 ? 8 : CPR) - 1;
            const uint32_t stage = sm.dst() + g * (128 * 128) + wq * 32 * 128;
#pragma unroll
            for (int ck = 0; ck < NCHUNK; ++ck) {
              float v[CW];
              tmem_row<CW>(tmem + tl + C::T_S + g * HALF_D + ck * CW, v);
              if (ck == NCHUNK - 1) {
                tc_fence_before();
                mbar_arrive(sm.bar(C::B_DQEMPTY));
              }
              if (!dq_first) {
#pragma unroll
                for (int c = 0; c < CW / 4; ++c) {
                  const float4 pc = part[ck * (CW / 4) + c];
                  v[4 * c] += pc.x;
                  v[4 * c + 1] += pc.y;
                  v[4 * c + 2] += pc.z;
                  v[4 * c + 3] += pc.w;
                }
              }
              if (!dq_last) {
#pragma unroll
                for (int c = 0; c < CW / 4; ++c)
                  st_global_v4_hint(reinterpret_cast<float*>(scr4 + (ck * (CW / 4) + c) * kBlockM),
                                    make_float4(v[4 * c], v[4 * c + 1], v[4 * c + 2], v[4 * c + 3]),
                                    pol_keep);
              } else {
#pragma unroll
                for (int c8 = 0; c8 < CW / 8; ++c8) {
                  const int c = ck * (CW / 8) + c8;
                  st_shared_v4(stage + lane * 128 + ((c ^ (lane & SWM)) << 4),
                               pack_bf16x2(v[8 * c8 + 0] * a.scale, v[8 * c8 + 1] * a.scale),
                               pack_bf16x2(v[8 * c8 + 2] * a.scale, v[8 * c8 + 3] * a.scale),
                               pack_bf16x2(v[8 * c8 + 4] * a.scale, v[8 * c8 + 5] * a.scale),
                               pack_bf16x2(v[8 * c8 + 6] * a.scale, v[8 * c8 + 7] * a.scale));
                }
              }
            }
            if (dq_last) {
              __syncwarp();  // the warp's rows are staged and its partial was read
              if (!dq_first && (lane & 7) == 0) {
#pragma unroll
                for (int c = 0; c < NCH4; ++c) discard_l2_line(scr4 + c * kBlockM);
              }
#pragma unroll 1
              for (int it = 0; it < CPR; ++it) {
                const int lin = it * 32 + lane;
                const int jr = lin / CPR, c = lin % CPR;   // row of this warp, chunk
                const uint4 vv = ld_shared_v4(stage + jr * 128 + ((c ^ (jr & SWM)) << 4));
                const int grow = m0 + wq * 32 + jr;
                if (grow < t.Lq)
                  *reinterpret_cast<uint4*>(a.dq + ((int64_t)(t.q0 + grow) * a.H + t.h) * C::D +
                                            g * HALF_D + c * 8) = vv;
              }
              __syncwarp();
            }
          }
          if (last) {
            // dK, dV of this key block: thread = key row, columns [g*D/2, (g+1)*D/2)
            if (a.dbias && key < t.Lk) {
              // d beta_j = sum_i dS_ij; for the gate beta = log sigma(G), whose
              // derivative is 1 - sigma(G) = 1 / (1 + e^G).  The two warpgroups'
              // halves meet in a zeroed element: either order gives the same sum.
              const float fac = a.bias_kind == 2 ? 1.f / (1.f + __expf(graw)) : 1.f;
              atomicAdd(a.dbias + (int64_t)t.h * a.total_kv + t.k0 + key, dsum * fac);
            }
            BWD_WAIT(C::B_DKVFULL, bi & 1, 0x1400 + C::B_DKVFULL);
            ++bi;
            tc_fence_after();
            float dkv[HALF_D], dvv[HALF_D];
            tmem_row<HALF_D>(tmem + tl + C::T_DK + g * HALF_D, dkv);
            tmem_row<HALF_D>(tmem + tl + C::T_DV + g * HALF_D, dvv);
            tc_fence_before();
            mbar_arrive(sm.bar(C::B_DKVEMPTY));
            // Each half row goes through this warp's own dS^T rows (free: every MMA
            // that read dS^T has completed), then out as whole row segments, so a
            // warp's store covers full 128-byte lines instead of one 16-byte piece
            // of 32 rows 2 KB apart.
            constexpr int CPR = HALF_D * 2 / 16;          // 16-byte chunks per half row
            constexpr int SWM = (CPR >= 8 ? 8 : CPR) - 1;
            const uint32_t stage = sm.dst() + g * (128 * 128) + wq * 32 * 128;
            const int wkey = kb * C::BN + wq * 32;        // first key of this warp
#pragma unroll
            for (int tsel = 0; tsel < 2; ++tsel) {
              const float mul = tsel == 0 ? a.scale : 1.f;
#pragma unroll
              for (int c = 0; c < CPR; ++c) {
                const float* v8 = (tsel == 0 ? dkv : dvv) + 8 * c;
                st_shared_v4(stage + lane * 128 + ((c ^ (lane & SWM)) << 4),
                             pack_bf16x2(v8[0] * mul, v8[1] * mul), pack_bf16x2(v8[2] * mul, v8[3] * mul),
                             pack_bf16x2(v8[4] * mul, v8[5] * mul), pack_bf16x2(v8[6] * mul, v8[7] * mul));
              }
              __syncwarp();
              __nv_bfloat16* dst = tsel == 0 ? a.dk : a.dv;
#pragma unroll 1
              for (int it = 0; it < CPR; ++it) {
                const int lin = it * 32 + lane;
                const int j = lin / CPR, c = lin % CPR;   // row of this warp, chunk
                const uint4 v = ld_shared_v4(stage + j * 128 + ((c ^ (j & SWM)) << 4));
                if (wkey + j < t.Lk)
                  *reinterpret_cast<uint4*>(dst + ((int64_t)(t.k0 + wkey + j) * a.H + t.h) * C::D +
                                            g * HALF_D + c * 8) = v;
              }
              __syncwarp();
            }
          }

          return true;
        },
        [&](int kb) -> bool {
          // no query sees this key block: its dK, dV rows are zero
          const int key = kb * C::BN + r;
          if (key < t.Lk) {
            const int64_t row = ((int64_t)(t.k0 + key) * a.H + t.h) * C::D + g * HALF_D;
#pragma unroll
            for (int e = 0; e < HALF_D; e += 8) {
              *reinterpret_cast<uint4*>(a.dk + row + e) = make_uint4(0, 0, 0, 0);
              *reinterpret_cast<uint4*>(a.dv + row + e) = make_uint4(0, 0, 0, 0);
            }
          }
          return true;
        });
    if (!ok) return;
  }
#undef BWD_WAIT
}

template <int D, int PHI>
__global__ void __launch_bounds__(kBwdThreads, 1)
    gdpa_bwd_kernel(const __grid_constant__ BwdArgs a, const __grid_constant__ CUtensorMap tq,
                    const __grid_constant__ CUtensorMap tk, const __grid_constant__ CUtensorMap tv,
                    const __grid_constant__ CUtensorMap tdo) {
  using C = BwdCfg<D>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  BSmem<C> sm;
  sm.base = smem_u32(smem_raw);
  sm.ptr = smem_raw;
  if (sm.base & 1023u) {  // swizzled TMA tiles need 1024-byte alignment
    if (threadIdx.x == 0) record_error(a.status, 2, 0x7001);
    return;
  }
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    mbar_init(sm.bar(C::B_KVFULL), 1);
    mbar_init(sm.bar(C::B_KVEMPTY), 1);
    for (int i = 0; i < C::NQ; ++i) {
      mbar_init(sm.bar(C::B_QFULL + i), 1);
      mbar_init(sm.bar(C::B_QEMPTY + i), 1);
    }
    mbar_init(sm.bar(C::B_SFULL), 1);
    mbar_init(sm.bar(C::B_PFULL), 256);
    mbar_init(sm.bar(C::B_DQFULL), 1);
    mbar_init(sm.bar(C::B_DQEMPTY), 256);
    mbar_init(sm.bar(C::B_DKVFULL), 1);
    mbar_init(sm.bar(C::B_DKVEMPTY), 256);
    for (int i = 0; i < 2; ++i) {
      mbar_init(sm.bar(C::B_RFULL + i), 32);
      mbar_init(sm.bar(C::B_REMPTY + i), 256);
    }
    *sm.abort_flag() = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tq);
    tma_prefetch_desc(&tk);
    tma_prefetch_desc(&tv);
    tma_prefetch_desc(&tdo);
  }
  if (warp == 2) {
    tmem_alloc(smem_u32(sm.tmem_slot()), C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *sm.tmem_slot();

  // Registers: the launch gives 384 x 168; warpgroup 0 (producer, MMA issuer,
  // allocator, row loader) needs few, the two phi warpgroups take the rest:
  // 128 x 88 + 256 x 208 = 64512.  Each budget is set inside its own
  // branch so the compiler allocates each role's code against it.
  if (warp < 4) {
    setmaxnreg_dec<kRegsControl>();
    if (warp == 0) {
      if (lane == 0) bwd_producer<C>(a, sm, &tq, &tk, &tv, &tdo);
    } else if (warp == 1) {
      if (lane == 0) bwd_mma<C>(a, sm, tmem);
    } else if (warp == 3) {
      if (PHI == 1) bwd_rows<C>(a, sm);
    }
  } else {
    setmaxnreg_inc<kRegsPhi>();
    bwd_phi<C, PHI>(a, sm, tmem);
  }
  __syncwarp();
  tc_fence_before();
  __syncthreads();
  if (*sm.abort_flag()) {
    if (threadIdx.x == 0) {
      const uint64_t t0 = globaltimer_ns();
      while (globaltimer_ns() - t0 < 2000000ull) __nanosleep(1000);
    }
    __syncthreads();
  }
  if (warp == 2) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

// delta[h][q] = sum_d dO[q,h,d] O[q,h,d] (fp32), D/8 threads per (q, h) row,
// 16 bytes of each operand per thread; rows are contiguous so reads coalesce.
template <int D>
__global__ void __launch_bounds__(256)
    gdpa_bwd_delta_kernel(const __nv_bfloat16* __restrict__ o,
                          const __nv_bfloat16* __restrict__ dout, float* __restrict__ delta,
                          int64_t total_q, int H) {
  constexpr int TPR = D / 8;  // threads per row
  const int64_t gt = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  const int64_t row = gt / TPR;
  const int part = (int)(gt % TPR);
  const int64_t nrows = total_q * H;
  float acc = 0.f;
  if (row < nrows) {
    const uint4 x = *reinterpret_cast<const uint4*>(o + row * D + part * 8);
    const uint4 y = *reinterpret_cast<const uint4*>(dout + row * D + part * 8);
    const __nv_bfloat162* xa = reinterpret_cast<const __nv_bfloat162*>(&x);
    const __nv_bfloat162* ya = reinterpret_cast<const __nv_bfloat162*>(&y);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float2 xf = __bfloat1622float2(xa[e]);
      const float2 yf = __bfloat1622float2(ya[e]);
      acc = fmaf(xf.x, yf.x, acc);
      acc = fmaf(xf.y, yf.y, acc);
    }
  }
#pragma unroll
  for (int off = TPR / 2; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
  if (row < nrows && part == 0) {
    const int64_t q = row / H;
    const int h = (int)(row - q * H);
    delta[(int64_t)h * total_q + q] = acc;
  }
}

template <int D, int PHI>
cudaError_t launch_bwd_one(const BwdArgs& a, const CUtensorMap& tq, const CUtensorMap& tk,
                           const CUtensorMap& tv, const CUtensorMap& tdo, int grid,
                           cudaStream_t stream) {
  using C = BwdCfg<D>;
  auto kern = gdpa_bwd_kernel<D, PHI>;
  // The phi warpgroups raise their register budget with setmaxnreg, which
  // waits until the block's launch registers cover it: never launch a build
  // whose per-thread count would leave that wait unsatisfiable.
  cudaFuncAttributes fa;
  cudaError_t e = cudaFuncGetAttributes(&fa, kern);
  if (e != cudaSuccess) return e;
  if (fa.numRegs * kBwdThreads < 128 * kRegsControl + 256 * kRegsPhi) return cudaErrorInvalidValue;
  e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_ALLOC);
  if (e != cudaSuccess) return e;
  kern<<<grid, kBwdThreads, C::SMEM_ALLOC, stream>>>(a, tq, tk, tv, tdo);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_bwd_preprocess(const __nv_bfloat16* o, const __nv_bfloat16* dout,
                                  float* delta, int64_t total_q, int H, int D,
                                  cudaStream_t stream) {
  const int64_t threads = total_q * H * (D / 8);
  if (threads == 0) return cudaSuccess;
  const int64_t blocks = (threads + 255) / 256;
  if (D == 128)
    gdpa_bwd_delta_kernel<128><<<(unsigned)blocks, 256, 0, stream>>>(o, dout, delta, total_q, H);
  else if (D == 64)
    gdpa_bwd_delta_kernel<64><<<(unsigned)blocks, 256, 0, stream>>>(o, dout, delta, total_q, H);
  else
    gdpa_bwd_delta_kernel<32><<<(unsigned)blocks, 256, 0, stream>>>(o, dout, delta, total_q, H);
  return cudaGetLastError();
}

cudaError_t launch_backward(const BwdArgs& a, int D, const CUtensorMap& tq, const CUtensorMap& tk,
                            const CUtensorMap& tv, const CUtensorMap& tdo, int grid,
                            cudaStream_t stream) {
#define GDPA_BWD_CASE(D_)                                                      \
  if (D == D_) {                                                               \
    if (a.phi == 1) return launch_bwd_one<D_, 1>(a, tq, tk, tv, tdo, grid, stream); \
    if (a.phi == 0) return launch_bwd_one<D_, 0>(a, tq, tk, tv, tdo, grid, stream); \
    if (a.phi == 3) return launch_bwd_one<D_, 3>(a, tq, tk, tv, tdo, grid, stream); \
    return launch_bwd_one<D_, 2>(a, tq, tk, tv, tdo, grid, stream);             \
  }
  GDPA_BWD_CASE(32)
  GDPA_BWD_CASE(64)
  GDPA_BWD_CASE(128)
#undef GDPA_BWD_CASE
  return cudaErrorInvalidValue;
}

}  // namespace gdpa
