// gdpa_bwd.cu -- fused GDPA backward for sm_100a, and its delta preprocess.
//
// Gradient of O = phi(scale * Q K^T + beta) V (Kunlun paper review §2.3
// "GDPA", Fig. 2; the fused kernel avoids materialising large intermediates in
// the backward pass).  Per visible pair (i, j):
//   s = scale q_i.k_j + beta_j,  p = phi(s)
//   dV_j += p dO_i,  dP = dO_i . V_j
//   dS = p (dP - delta_i) with delta_i = dO_i . O_i   (softmax, p = exp(s - LSE_i))
//      = dP * (sigma(s) + s sigma(s)(1 - sigma(s)))   (SiLU)
//      = dP * (Phi(s) + s phi(s))                     (GELU)
//      = dP                                           (identity)
//   dK_j += scale dS q_i,  dQ_i += scale dS k_j
//
// One persistent CTA per SM walks (sample, head) units longest first.  Within
// a unit the key blocks (128 keys) are the outer loop and the query tiles
// (128 queries) that can see a block the inner loop, so dK and dV accumulate
// in TMEM across all of the sample's queries and are written once.  A block's
// tiles are visited in alternating directions from block to block, so the
// tiles a block reads last are the ones the next block reads first (they are
// still in L2).
//
// The five products of a (key block, query tile) pair n are software
// pipelined across pairs, in this issue order:
//   S^T(n+1) = K Q^T | dK += dS^T(n) Q | dQ(n) = dS(n) K | dP^T(n+1) = V dO^T |
//   dV += P^T(n+1) dO
// so the tensor core computes dK(n), dQ(n) and dP^T(n+1) while the compute
// warpgroups turn S^T(n+1) into P^T(n+1), and dV(n+1) and S^T(n+2) while they
// turn dP^T(n+1) into dS(n+1); a reducer warpgroup drains dQ(n) from the
// columns dP^T(n+1) reuses.  dK and dV take their A operand (dS^T, P^T)
// straight from TMEM.  tcgen05.mma instructions of one thread execute in
// issue order, which the TMEM reuse below relies on (an MMA that overwrites
// columns is issued after every MMA that reads them).
//
// TMEM (512 columns): [0,128) S^T, then P^T (bf16 pairs) and, for an
// element-wise phi, phi'(S)^T (fp16 pairs) over it; [128,256) dP^T, then dS^T (bf16 pairs) over
// it, then dQ (fp32, D columns); then dK, dV.
// Shared memory: K, V of the key block; 2-stage rings of Q and dO tiles; dS
// (bf16, the MN-major A operand of dQ), which also stages the dK, dV rows at
// the end of a key block; LSE / delta rows of two tiles.
//
// With the rotary temporal embedding the kernel reads turned Q and K and turns
// dQ and dK back (the transpose of each token's turn) in its epilogue, so no
// pass over the gradients follows it.
//
// Warp roles (512 threads): 0 TMA producer, 1 MMA issuer, 2 TMEM allocator and
// LSE / delta loader, 3 idle; warpgroups 1-2 compute P and dS (a thread owns
// one key, each warpgroup half of the tile's 128 query columns); warpgroup 3
// drains dQ from TMEM (summing it over key blocks in a per-CTA fp32 scratch
// slot) and writes dK, dV at the end of each key block.
#include <climits>

#include <cuda_fp16.h>

#include "gdpa_internal.h"

namespace gdpa {
namespace {

constexpr int kBwdThreads = 512;
constexpr int kRegsLaunch = 128;   // 65536 / 512
#ifndef GDPA_BWD_RC
#define GDPA_BWD_RC 80
#define GDPA_BWD_RP 120
#define GDPA_BWD_RR 192
#endif
constexpr int kRegsControl = GDPA_BWD_RC;  // warpgroup 0
constexpr int kRegsCompute = GDPA_BWD_RP;  // warpgroups 1 and 2
constexpr int kRegsReduce = GDPA_BWD_RR;   // warpgroup 3
static_assert(128 * kRegsControl + 256 * kRegsCompute + 128 * kRegsReduce <=
                  kBwdThreads * kRegsLaunch,
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
  static constexpr int DS_BYTES = BN * BM * 2;
  static constexpr int OFF_K = 0;
  static constexpr int OFF_V = OFF_K + KV_BYTES;
  static constexpr int OFF_Q = OFF_V + KV_BYTES;       // [2] Q tiles
  static constexpr int OFF_DO = OFF_Q + 2 * QT_BYTES;  // [2] dO tiles
  static constexpr int OFF_DS = OFF_DO + 2 * QT_BYTES;
  static constexpr int OFF_ROW = OFF_DS + DS_BYTES;    // float [2][2][BM]: LSE*log2e, delta
  static constexpr int OFF_BAR = OFF_ROW + 2 * 2 * BM * 4;
  static constexpr int B_KVFULL = 0, B_KVEMPTY = 1, B_QFULL = 2, B_QEMPTY = 4, B_DOFULL = 6,
                       B_DOEMPTY = 8, B_SFULL = 10, B_PFULL = 11, B_DPFULL = 12, B_DSFULL = 13,
                       B_DQFULL = 14, B_DQEMPTY = 15, B_DSFREE = 16, B_DKVFULL = 17,
                       B_DKVEMPTY = 18, B_RFULL = 19, B_REMPTY = 21, B_PREAD = 23, NBARS = 24;
  static constexpr int OFF_MISC = OFF_BAR + NBARS * 8;
  static constexpr int SMEM_BYTES = OFF_MISC + 16;
  static constexpr int SMEM_ALLOC = SMEM_BYTES;  // base is 1024-aligned (checked at entry)
  static constexpr int T_S = 0, T_DP = 128, T_DK = 256, T_DV = 256 + D;
  static constexpr int TMEM_COLS = 512;
  static_assert(T_DV + D <= TMEM_COLS, "TMEM");
  static_assert(SMEM_ALLOC <= 232448, "shared memory budget");
  static_assert(OFF_Q % 1024 == 0 && OFF_DO % 1024 == 0 && OFF_DS % 1024 == 0, "align");
};

using BUnit = GdpaUnit;

// Key blocks [kb0, kb1) query tile m0 may see.
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
  __device__ uint32_t ds() const { return base + C::OFF_DS; }
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

// One (key block, query tile) pair of a unit's walk.
struct BPair {
  int kb, mt;
  int idx, n;             // position within the key block's tiles, and their count
  bool dq_first, dq_last; // the first / last key block that reaches tile mt
};

// The pairs of a unit in the order every role uses: key blocks ascending; the
// tiles a block can see (a contiguous range) ascending for even blocks and
// descending for odd ones.  f(pair) for each pair, g(kb) for key blocks no
// tile sees.  Either returning false stops the walk.
template <class F, class G>
__device__ __forceinline__ bool for_each_pair(const BUnit& t, int wl, int wr, F&& f, G&& g) {
  const int ntile = (t.Lq + kBlockM - 1) / kBlockM;
  const int nkb = (t.Lk + 127) / 128;
  for (int kb = 0; kb < nkb; ++kb) {
    int lo = -1, hi = -1;
    for (int mt = 0; mt < ntile; ++mt) {
      int a0, a1;
      bwd_kv_range(mt * kBlockM, t.Lk, wl, wr, a0, a1);
      if (kb >= a0 && kb < a1) {
        if (lo < 0) lo = mt;
        hi = mt;
      }
    }
    if (lo < 0) {
      if (!g(kb)) return false;
      continue;
    }
    BPair x;
    x.kb = kb;
    x.n = hi - lo + 1;
    for (int i = 0; i < x.n; ++i) {
      x.idx = i;
      x.mt = (kb & 1) ? hi - i : lo + i;
      int a0, a1;
      bwd_kv_range(x.mt * kBlockM, t.Lk, wl, wr, a0, a1);
      x.dq_first = kb == a0;
      x.dq_last = kb == a1 - 1;
      if (!f(x)) return false;
    }
  }
  return true;
}

// ------------------------------------------------------------------ producer
// Per pair: its Q tile and its dO tile into their 2-stage rings; at a key
// block's first pair, after those, the block's K and V (their buffer frees
// once the previous block's last dQ MMA completes).
template <class C>
__device__ void bwd_producer(const BwdArgs& a, const BSmem<C>& sm, const CUtensorMap* tq,
                             const CUtensorMap* tk, const CUtensorMap* tv,
                             const CUtensorMap* tdo) {
  volatile int* abort = sm.abort_flag();
  const uint64_t pol_stream = l2_policy_evict_first();
  const uint64_t pol_keep = l2_policy_evict_last();
  uint32_t gb = 0, gp = 0;
  bool dropped = false;
  UnitStream units(a.info, a.H, a.n_units, a.head_mask);
  BUnit t;
  while (units.next(t)) {
    bool ok = for_each_pair(
        t, a.wl, a.wr,
        [&](const BPair& x) -> bool {
          const int s = gp & 1;
          const uint32_t par = ((gp >> 1) & 1) ^ 1;
          // a tile another key block reads later stays in L2
          const uint64_t pol = x.dq_last ? pol_stream : pol_keep;
          const int row = t.q0 + x.mt * kBlockM;
          if (!mbar_wait(sm.bar(C::B_QEMPTY + s), par, abort, a.status, a.timeout_ns,
                         0x1000 + C::B_QEMPTY + s))
            return false;
          if ((a.debug_flags & 1) && !dropped && blockIdx.x == 0) {
            dropped = true;  // test hook: this Q tile is never loaded
          } else {
            mbar_arrive_expect_tx(sm.bar(C::B_QFULL + s), C::QT_BYTES);
            for (int p = 0; p < C::NPANEL; ++p)
              tma_load_3d(sm.q(s) + p * C::BM * C::PANEL_BYTES, tq, sm.bar(C::B_QFULL + s),
                          p * C::PANEL_ELEMS, t.h, row, pol);
          }
          if (!mbar_wait(sm.bar(C::B_DOEMPTY + s), par, abort, a.status, a.timeout_ns,
                         0x1000 + C::B_DOEMPTY + s))
            return false;
          mbar_arrive_expect_tx(sm.bar(C::B_DOFULL + s), C::QT_BYTES);
          for (int p = 0; p < C::NPANEL; ++p)
            tma_load_3d(sm.dout(s) + p * C::BM * C::PANEL_BYTES, tdo, sm.bar(C::B_DOFULL + s),
                        p * C::PANEL_ELEMS, t.h, row, pol);
          ++gp;
          if (x.idx == 0) {
            if (!mbar_wait(sm.bar(C::B_KVEMPTY), (gb & 1) ^ 1, abort, a.status, a.timeout_ns,
                           0x1000 + C::B_KVEMPTY))
              return false;
            mbar_arrive_expect_tx(sm.bar(C::B_KVFULL), 2 * C::KV_BYTES);
            for (int p = 0; p < C::NPANEL; ++p) {
              tma_load_3d(sm.k() + p * C::BN * C::PANEL_BYTES, tk, sm.bar(C::B_KVFULL),
                          p * C::PANEL_ELEMS, t.h, t.k0 + x.kb * C::BN, pol_keep);
              tma_load_3d(sm.v() + p * C::BN * C::PANEL_BYTES, tv, sm.bar(C::B_KVFULL),
                          p * C::PANEL_ELEMS, t.h, t.k0 + x.kb * C::BN, pol_keep);
            }
            ++gb;
            // warm L2 with the key block that follows (this unit's next block or
            // the next unit's first), whose load waits for this block's release
            const int nkb = (t.Lk + C::BN - 1) / C::BN;
            BUnit nt = t;
            int nb = x.kb + 1;
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

#define MMA_WAIT(bar_, par_)                                                             \
  do {                                                                                   \
    if (!mbar_wait(sm.bar(bar_), (par_), abort, a.status, a.timeout_ns, 0x1100 + (bar_))) \
      return false;                                                                      \
  } while (0)

  // Base descriptors; every operand tile lies at a fixed offset from one of
  // them and the start-address field (address >> 4, 14 bits) cannot overflow
  // below 256 KB of shared memory, so a descriptor is base + (offset >> 4).
  const uint64_t d_k = make_smem_desc(sm.k(), 16, SBO, C::LAYOUT);              // K-major
  const uint64_t d_v = make_smem_desc(sm.v(), 16, SBO, C::LAYOUT);
  const uint64_t d_q = make_smem_desc(sm.q(0), 16, SBO, C::LAYOUT);
  const uint64_t d_do = make_smem_desc(sm.dout(0), 16, SBO, C::LAYOUT);
  const uint64_t m_q = make_smem_desc(sm.q(0), C::BM * C::PANEL_BYTES, SBO, C::LAYOUT);  // MN-major
  const uint64_t m_do = make_smem_desc(sm.dout(0), C::BM * C::PANEL_BYTES, SBO, C::LAYOUT);
  const uint64_t m_k = make_smem_desc(sm.k(), C::BN * C::PANEL_BYTES, SBO, C::LAYOUT);
  const uint64_t m_ds = make_smem_desc(sm.ds(), 128 * 128, 1024, LAYOUT_SW128);
  // K-major operand step kk (16 elements of D) within a tile of `rows` rows
  auto kstep = [](int kk, int rows) -> uint32_t {
    return (uint32_t)(((kk * 16 / C::PANEL_ELEMS) * rows * C::PANEL_BYTES +
                       (kk * 16 % C::PANEL_ELEMS) * 2) >> 4);
  };

  // S^T = K Q^T (M = 128 keys, N = 128 queries, K = D)
  auto issue_s = [&](uint32_t p) -> bool {
    const int s = p & 1;
    MMA_WAIT(C::B_QFULL + s, (p >> 1) & 1);
    // the previous pair's P^T (and phi') have been read back by the compute
    // warpgroups; dV of that pair, the other reader, was issued before this
    if (p > 0) MMA_WAIT(C::B_PREAD, (p - 1) & 1);
    tc_fence_after();
    const uint32_t so = (uint32_t)(s * C::QT_BYTES) >> 4;
#pragma unroll
    for (int kk = 0; kk < C::D / 16; ++kk)
      mma_bf16_ss(tmem + C::T_S, desc_add(d_k, kstep(kk, C::BN)),
                  desc_add(d_q, so + kstep(kk, C::BM)), id_st, kk > 0 ? 1u : 0u);
    mma_commit(sm.bar(C::B_SFULL));
    return true;
  };
  // dP^T = V dO^T into the dP^T / dQ columns, once the previous dQ was drained
  auto issue_dp = [&](uint32_t p) -> bool {
    const int s = p & 1;
    MMA_WAIT(C::B_DOFULL + s, (p >> 1) & 1);
    if (p > 0) MMA_WAIT(C::B_DQEMPTY, (p - 1) & 1);
    tc_fence_after();
    const uint32_t so = (uint32_t)(s * C::QT_BYTES) >> 4;
#pragma unroll
    for (int kk = 0; kk < C::D / 16; ++kk)
      mma_bf16_ss(tmem + C::T_DP, desc_add(d_v, kstep(kk, C::BN)),
                  desc_add(d_do, so + kstep(kk, C::BM)), id_st, kk > 0 ? 1u : 0u);
    mma_commit(sm.bar(C::B_DPFULL));
    return true;
  };
  // dV += P^T dO (P^T from TMEM: queries 16kk.. are warpgroup kk/4's columns)
  auto issue_dv = [&](uint32_t p, bool first) -> bool {
    const int s = p & 1;
    MMA_WAIT(C::B_PFULL, p & 1);
    tc_fence_after();
    const uint32_t so = (uint32_t)(s * C::QT_BYTES) >> 4;
#pragma unroll
    for (int kk = 0; kk < kBlockM / 16; ++kk)
      mma_bf16_ts(tmem + C::T_DV, tmem + C::T_S + (kk / 4) * 64 + (kk % 4) * 8,
                  desc_add(m_do, so + ((kk * 16 * C::PANEL_BYTES) >> 4)), id_kv,
                  (!first || kk > 0) ? 1u : 0u);
    mma_commit(sm.bar(C::B_DOEMPTY + s));
    return true;
  };
  // dK += dS^T Q (dS^T from TMEM), then dQ = dS K (dS from shared memory)
  auto issue_dk_dq = [&](uint32_t p, bool first) -> bool {
    const int s = p & 1;
    MMA_WAIT(C::B_DSFULL, p & 1);
    tc_fence_after();
    const uint32_t so = (uint32_t)(s * C::QT_BYTES) >> 4;
#pragma unroll
    for (int kk = 0; kk < kBlockM / 16; ++kk)
      mma_bf16_ts(tmem + C::T_DK, tmem + C::T_DP + (kk / 4) * 64 + (kk % 4) * 8,
                  desc_add(m_q, so + ((kk * 16 * C::PANEL_BYTES) >> 4)), id_kv,
                  (!first || kk > 0) ? 1u : 0u);
    mma_commit(sm.bar(C::B_QEMPTY + s));
#pragma unroll
    for (int kk = 0; kk < C::BN / 16; ++kk)
      mma_bf16_ss(tmem + C::T_DP, desc_add(m_ds, (kk * 16 * 128) >> 4),
                  desc_add(m_k, (kk * 16 * C::PANEL_BYTES) >> 4), id_dq, kk > 0 ? 1u : 0u);
    mma_commit(sm.bar(C::B_DQFULL));
    return true;
  };

  uint32_t gp = 0, gb = 0;
  UnitStream units(a.info, a.H, a.n_units, a.head_mask);
  BUnit t;
  uint32_t bp0 = 0;  // global index of the current key block's first pair
  while (units.next(t)) {
    bool ok = for_each_pair(
        t, a.wl, a.wr,
        [&](const BPair& x) -> bool {
          // pair x is pair gp; the pipeline is driven from the block's pairs in
          // order: at pair i the products S(i+1), dK(i), dQ(i), dP(i+1), dV(i+1)
          const uint32_t p = gp;
          if (x.idx == 0) {
            bp0 = p;
            MMA_WAIT(C::B_KVFULL, gb & 1);
            if (!issue_s(p)) return false;
            if (!issue_dp(p)) return false;
            // dK, dV of the previous block have been read out
            if (gb > 0) MMA_WAIT(C::B_DKVEMPTY, (gb - 1) & 1);
            if (!issue_dv(p, true)) return false;
          }
          if (x.idx + 1 < x.n) {
            if (!issue_s(p + 1)) return false;
            if (!issue_dk_dq(p, p == bp0)) return false;
            if (!issue_dp(p + 1)) return false;
            if (!issue_dv(p + 1, false)) return false;
          } else {
            if (!issue_dk_dq(p, p == bp0)) return false;
            mma_commit(sm.bar(C::B_DKVFULL));
            mma_commit(sm.bar(C::B_KVEMPTY));
            ++gb;
          }
          ++gp;
          return true;
        },
        [&](int) { return true; });
    if (!ok) return;
  }
#undef MMA_WAIT
}

// ------------------------------------------------------------------ LSE / delta loader
template <class C>
__device__ void bwd_rows(const BwdArgs& a, const BSmem<C>& sm) {
  volatile int* abort = sm.abort_flag();
  const int lane = threadIdx.x & 31;
  uint32_t gp = 0;
  UnitStream units(a.info, a.H, a.n_units, a.head_mask);
  BUnit t;
  while (units.next(t)) {
    bool ok = for_each_pair(
        t, a.wl, a.wr,
        [&](const BPair& x) -> bool {
          const int s = gp & 1;
          bool w = mbar_wait(sm.bar(C::B_REMPTY + s), ((gp >> 1) & 1) ^ 1, abort, a.status,
                             a.timeout_ns, 0x1300 + C::B_REMPTY + s);
          if (!__all_sync(0xffffffffu, w)) return false;
          float* l2 = sm.lse2(s);
          float* dl = sm.delta(s);
          for (int c = lane; c < C::BM; c += 32) {
            const int i = x.mt * kBlockM + c;
            float lv = 0.f, d = 0.f;
            if (i < t.Lq) {
              const int64_t idx = (int64_t)t.h * a.total_q + t.q0 + i;
              lv = a.lse[idx] * kLog2eB;
              d = a.delta[idx];
            }
            l2[c] = lv;
            dl[c] = d;
          }
          mbar_arrive(sm.bar(C::B_RFULL + s));
          ++gp;
          return true;
        },
        [&](int) { return true; });
    if (!ok) return;
  }
}

// ------------------------------------------------------------------ compute warpgroups
// N consecutive fp32 TMEM columns of this thread's lane (N = 16 or a multiple
// of 32), loaded without waiting.
template <int N>
__device__ __forceinline__ void tmem_cols(uint32_t taddr, float* v) {
  if constexpr (N % 32 == 0) {
#pragma unroll
    for (int c = 0; c < N / 32; ++c) tmem_ld32f(taddr + c * 32, v + c * 32);
  } else {
    static_assert(N == 16, "16 or a multiple of 32 columns");
    uint32_t r[16];
    tmem_ld16(taddr, r);
    tmem_wait_ld();
#pragma unroll
    for (int e = 0; e < 16; ++e) v[e] = __uint_as_float(r[e]);
  }
}

// Thread = key r of the block (its TMEM lane); warpgroup g takes query columns
// [64g, 64g + 64) of each tile.  P phase: P^T = phi(S^T), bf16, over the first
// 32 of this warpgroup's S^T columns (the A operand of dV); for an
// element-wise phi, phi'(x) (fp16, which holds its range [-0.2, 1.2] to 2^-11)
// over the next 32.  dS phase: dS^T from
// dP^T and from P (softmax) or phi' read back from TMEM, into the dP^T columns
// (the A operand of dK) and the dS panel (the A operand of dQ).  The arrive on
// PREAD tells the issuer those S^T columns may take the next tile's S^T.
template <class C, int PHI>
__device__ void bwd_compute(const BwdArgs& a, const BSmem<C>& sm, uint32_t tmem) {
  volatile int* abort = sm.abort_flag();
  const int g = ((threadIdx.x >> 5) - 4) >> 2;    // warpgroup 0 or 1
  const int wq = (threadIdx.x >> 5) & 3;          // TMEM lane quarter
  const int lane = threadIdx.x & 31;
  const int r = wq * 32 + lane;                   // key row of the block
  const uint32_t tl = (uint32_t)(wq * 32) << 16;
  constexpr bool SOFTMAX = PHI == 1;
  const float sc = SOFTMAX ? a.scale * kLog2eB : a.scale;

#define CMP_WAIT(bar_, par_)                                                                 \
  do {                                                                                       \
    bool ok_ = mbar_wait(sm.bar(bar_), (par_), abort, a.status, a.timeout_ns, 0x1400 + (bar_)); \
    if (!__all_sync(0xffffffffu, ok_)) return false;                                         \
  } while (0)

  int64_t pre_idx = -1;  // bias element fetched ahead (pre_val), or -1
  float pre_val = 0.f;
  uint32_t gp = 0, gbc = 0;  // pairs, key blocks
  float beta = 0.f, graw = 0.f, dsum = 0.f;
  UnitStream units(a.info, a.H, a.n_units, a.head_mask);
  BUnit t;
  while (units.next(t)) {
    bool ok = for_each_pair(
        t, a.wl, a.wr,
        [&](const BPair& x) -> bool {
          const uint32_t p = gp;
          const int key = x.kb * C::BN + r;
          if (x.idx == 0) {
            dsum = 0.f;
            if (a.bias_kind != 0) {
              // this key block's raw bias, fetched one key block ahead
              float gv = 0.f;
              const int64_t gi = key < t.Lk ? (int64_t)t.h * a.total_kv + t.k0 + key : -1;
              if (gi >= 0) gv = gi == pre_idx ? pre_val : a.bias[gi];
              beta = 0.f;
              if (gi >= 0)
                beta = a.bias_kind == 2 ? fminf(gv, 0.f) - log1pf(__expf(-fabsf(gv))) : gv;
              graw = gv;
              if (SOFTMAX) beta *= kLog2eB;
              pre_idx = -1;
              if ((x.kb + 1) * C::BN < t.Lk) {
                if ((x.kb + 1) * C::BN + r < t.Lk) pre_idx = gi + C::BN;
              } else {
                BUnit nt;
                if (units.peek(nt) && r < nt.Lk) pre_idx = (int64_t)nt.h * a.total_kv + nt.k0 + r;
              }
              if (pre_idx >= 0) pre_val = a.bias[pre_idx];
            }
          }
          const int m0 = x.mt * kBlockM;
          const int rs = p & 1;
          // visible queries of this key: i in [qlo, qhi]
          int qlo = 0, qhi = t.Lq - 1;
          if (a.wr >= 0) qlo = max(qlo, key - a.wr);
          if (a.wl >= 0) qhi = min(qhi, key + a.wl);
          if (key >= t.Lk) qhi = -1;
          const int c0 = g * 64;                   // first query column of this warpgroup

          // ---- P phase
          if (SOFTMAX) CMP_WAIT(C::B_RFULL + rs, (p >> 1) & 1);
          CMP_WAIT(C::B_SFULL, p & 1);
          tc_fence_after();
          const float* l2 = sm.lse2(rs) + c0;
          const uint64_t sc2 = f2_pack(sc, sc);
          const uint64_t beta2 = f2_pack(beta, beta);
          const uint64_t half2 = f2_pack(0.5f, 0.5f);
          const uint64_t one2 = f2_pack(1.f, 1.f);
          uint32_t kk0[16];  // phi' of chunk 0, written once chunk 1's S^T is read
#pragma unroll
          for (int ch = 0; ch < 2; ++ch) {
            float sr[32];
            tmem_ld32f(tmem + tl + C::T_S + c0 + ch * 32, sr);
            tmem_wait_ld();
            // queries [i0, i0 + 32) of this chunk; when every one is visible to
            // every key of the warp, no column needs its mask
            const int i0 = m0 + c0 + ch * 32;
            const bool full = __all_sync(0xffffffffu, i0 >= qlo && i0 + 31 <= qhi);
            uint32_t pk[16], kk[16];
            float4 lv4 = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
            for (int e2 = 0; e2 < 16; ++e2) {
              const int e = 2 * e2;
              const uint64_t x2 = f2_fma(f2_pack(sr[e], sr[e + 1]), sc2, beta2);
              float p0, p1, k0 = 0.f, k1 = 0.f;
              if (PHI == 1) {
                if ((e2 & 1) == 0) lv4 = *reinterpret_cast<const float4*>(l2 + ch * 32 + e);
                float d0, d1;
                f2_unpack(f2_sub(x2, (e2 & 1) ? f2_pack(lv4.z, lv4.w) : f2_pack(lv4.x, lv4.y)),
                          d0, d1);
                p0 = ex2_approx(d0);
                p1 = ex2_approx(d1);
              } else if (PHI == 0) {
                // sigmoid(x) = 1/2 + tanh(x/2)/2; silu = x sigmoid(x);
                // silu'(x) = sigmoid(x) + silu(x) (1 - sigmoid(x))
                float h0, h1;
                f2_unpack(f2_mul(x2, half2), h0, h1);
                const uint64_t sg2 = f2_fma(half2, f2_pack(tanh_approx(h0), tanh_approx(h1)), half2);
                const uint64_t p2 = f2_mul(x2, sg2);
                f2_unpack(p2, p0, p1);
                f2_unpack(f2_fma(p2, f2_sub(one2, sg2), sg2), k0, k1);
              } else if (PHI == 3) {
                // gelu(x) = x Phi(x); gelu'(x) = Phi(x) + x phi(x), phi the
                // standard normal density exp(-x^2 / 2) / sqrt(2 pi)
                float xs[2], pp[2], dd[2];
                f2_unpack(x2, xs[0], xs[1]);
#pragma unroll
                for (int u = 0; u < 2; ++u) {
                  const float cdf = fmaf(0.5f, erff(xs[u] * kInvSqrt2), 0.5f);
                  pp[u] = xs[u] * cdf;
                  dd[u] = fmaf(xs[u], kInvSqrt2Pi * __expf(-0.5f * xs[u] * xs[u]), cdf);
                }
                p0 = pp[0];
                p1 = pp[1];
                k0 = dd[0];
                k1 = dd[1];
              } else {
                f2_unpack(x2, p0, p1);
                k0 = 1.f;
                k1 = 1.f;
              }
              if (!full) {
                const int i = i0 + e;
                const bool v0 = i >= qlo && i <= qhi, v1 = i + 1 >= qlo && i + 1 <= qhi;
                p0 = v0 ? p0 : 0.f;
                p1 = v1 ? p1 : 0.f;
                k0 = v0 ? k0 : 0.f;
                k1 = v1 ? k1 : 0.f;
              }
              pk[e2] = pack_bf16x2(p0, p1);
              if (!SOFTMAX) kk[e2] = pack_f16x2(k0, k1);  // phi' in [-0.2, 1.2]: fp16
            }
            // P^T chunk -> the first 32 S^T columns of this warpgroup (read in
            // chunk 0); phi' -> the last 32, once chunk 1 has read them
            tmem_st16(tmem + tl + C::T_S + c0 + ch * 16, pk);
            if (!SOFTMAX) {
              if (ch == 0) {
#pragma unroll
                for (int e = 0; e < 16; ++e) kk0[e] = kk[e];
              } else {
                tmem_st16(tmem + tl + C::T_S + c0 + 32, kk0);
                tmem_st16(tmem + tl + C::T_S + c0 + 48, kk);
              }
            }
          }
          tmem_wait_st();
          tc_fence_before();
          mbar_arrive(sm.bar(C::B_PFULL));

          // ---- dS phase
          CMP_WAIT(C::B_DPFULL, p & 1);
          // dQ(n-1), the last reader of the previous dS, completed before dP(n)
          // was issued; at a key block's first pair the reducer must also be done
          // staging the previous block's dK, dV in the panel
          if (x.idx == 0 && gbc > 0) CMP_WAIT(C::B_DSFREE, (gbc - 1) & 1);
          tc_fence_after();
          const float* dl = sm.delta(rs) + c0;
          uint64_t dsum2 = f2_pack(0.f, 0.f);
#pragma unroll
          for (int ch = 0; ch < 2; ++ch) {
            float dr[32];
            uint32_t kv[16];  // P (softmax) or phi', bf16 pairs
            tmem_ld32f(tmem + tl + C::T_DP + c0 + ch * 32, dr);
            tmem_ld16(tmem + tl + C::T_S + c0 + (SOFTMAX ? 0 : 32) + ch * 16, kv);
            tmem_wait_ld();
            if (ch == 1) {  // P / phi' read: the S^T columns may take the next S^T
              tc_fence_before();
              mbar_arrive(sm.bar(C::B_PREAD));
            }
            uint32_t pk[16];
            float4 dv4 = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
            for (int e2 = 0; e2 < 16; ++e2) {
              const int e = 2 * e2;
              const uint64_t dp2 = f2_pack(dr[e], dr[e + 1]);
              const uint64_t k2 = SOFTMAX ? f2_pack(__uint_as_float(kv[e2] << 16),
                                                    __uint_as_float(kv[e2] & 0xffff0000u))
                                          : unpack_f16x2(kv[e2]);
              uint64_t ds2;
              if (SOFTMAX) {
                if ((e2 & 1) == 0) dv4 = *reinterpret_cast<const float4*>(dl + ch * 32 + e);
                ds2 = f2_mul(k2, f2_sub(dp2, (e2 & 1) ? f2_pack(dv4.z, dv4.w)
                                                       : f2_pack(dv4.x, dv4.y)));
              } else {
                ds2 = f2_mul(k2, dp2);
              }
              dsum2 = f2_add(dsum2, ds2);
              float d0, d1;
              f2_unpack(ds2, d0, d1);
              pk[e2] = pack_bf16x2(d0, d1);
            }
            tmem_st16(tmem + tl + C::T_DP + c0 + ch * 16, pk);
            // dS^T row r -> panel g (queries 64g .. 64g+63), 128-byte swizzle
#pragma unroll
            for (int q8 = 0; q8 < 4; ++q8) {
              const int cir = ch * 4 + q8;    // 16-byte chunk within the 128-byte row
              st_shared_v4(sm.ds() + g * (128 * 128) + r * 128 + ((cir ^ (r & 7)) << 4),
                           pk[q8 * 4 + 0], pk[q8 * 4 + 1], pk[q8 * 4 + 2], pk[q8 * 4 + 3]);
            }
          }
          {
            float s0, s1;
            f2_unpack(dsum2, s0, s1);
            dsum += s0 + s1;
          }
          tmem_wait_st();
          fence_proxy_async_smem();
          tc_fence_before();
          mbar_arrive(sm.bar(C::B_DSFULL));
          if (SOFTMAX) mbar_arrive(sm.bar(C::B_REMPTY + rs));
          ++gp;

          if (x.idx + 1 == x.n) {
            ++gbc;
            if (a.dbias && key < t.Lk) {
              // d beta_j = sum_i dS_ij; for the gate beta = log sigma(G), whose
              // derivative is 1 - sigma(G) = 1 / (1 + e^G).  The two warpgroups'
              // halves meet in a zeroed element: either order gives the same sum.
              const float fac = a.bias_kind == 2 ? 1.f / (1.f + __expf(graw)) : 1.f;
              atomicAdd(a.dbias + (int64_t)t.h * a.total_kv + t.k0 + key, dsum * fac);
            }
          }
          return true;
        },
        [&](int) { return true; });
    if (!ok) return;
  }
#undef CMP_WAIT
}

// (x0, x1) turned back by the angle whose (cos, sin) is the fp16 pair cs (the
// transpose of the forward turn of a rotary pair).
__device__ __forceinline__ void unturn_pair(float& x0, float& x1, uint32_t cs) {
  const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&cs));
  const float y0 = fmaf(x0, f.x, x1 * f.y);
  x1 = fmaf(x1, f.x, -x0 * f.y);
  x0 = y0;
}
// 32 consecutive values (16 rotary pairs from pair p0) of a row turned back by
// the token's table row.
__device__ __forceinline__ void unturn32(float* v, const uint32_t* row, int p0) {
  const uint4* t = reinterpret_cast<const uint4*>(row + p0);
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const uint4 cs = __ldg(t + q);
    unturn_pair(v[8 * q + 0], v[8 * q + 1], cs.x);
    unturn_pair(v[8 * q + 2], v[8 * q + 3], cs.y);
    unturn_pair(v[8 * q + 4], v[8 * q + 5], cs.z);
    unturn_pair(v[8 * q + 6], v[8 * q + 7], cs.w);
  }
}

// ------------------------------------------------------------------ reducer warpgroup
// Thread = query row r of the tile for dQ, key row r of the block for dK/dV.
// dQ of a pair is summed over the key blocks that reach its tile in this CTA's
// fp32 scratch slot, laid out thread-major ([tile][16-byte chunk][row]) so a
// warp's access is 512 contiguous bytes; only the thread that wrote an element
// reads it back, so no atomics or fences are needed.  The row goes in halves of
// HW columns: the earlier blocks' partial of a half is fetched before the TMEM
// read it joins, so the columns are released (DQ_EMPTY) after the second
// half's read without waiting on a global load.  Final dQ rows go straight to
// global memory (a thread writes its own row); dK and dV rows are staged in
// this warp's quarter of the dS panel (free once the block's last dQ MMA has
// completed) and written as whole rows.  With the rotary embedding, final dQ
// rows and dK rows are turned back (by the transpose of their token's turn)
// as they are written.
template <class C>
__device__ void bwd_reduce(const BwdArgs& a, const BSmem<C>& sm, uint32_t tmem) {
  volatile int* abort = sm.abort_flag();
  const int wq = (threadIdx.x >> 5) & 3;
  const int lane = threadIdx.x & 31;
  const int r = wq * 32 + lane;
  const uint32_t tl = (uint32_t)(wq * 32) << 16;
  const int rtid = threadIdx.x - 384;   // 0..127
  const uint64_t pol_keep = l2_policy_evict_last();
  constexpr int RB = C::D * 2;                    // bytes of one staged bf16 row
  constexpr int CPR = RB / 16;                    // 16-byte chunks per row
  constexpr int SWM = (CPR >= 8 ? 8 : CPR) - 1;
  constexpr int NCH = C::D / 32;                  // 32-column chunks of a row
  constexpr int HW = C::D >= 64 ? 64 : 32;        // columns per half of a dQ row
  constexpr int NHALF = C::D / HW;
  const uint32_t stage = sm.ds() + wq * 32 * RB;  // this warp's 32 staged rows
  const int slot_tiles = a.dq_slot_rows / kBlockM;

#define RED_WAIT(bar_, par_)                                                                 \
  do {                                                                                       \
    bool ok_ = mbar_wait(sm.bar(bar_), (par_), abort, a.status, a.timeout_ns, 0x1500 + (bar_)); \
    if (!__all_sync(0xffffffffu, ok_)) return false;                                         \
  } while (0)

  // Stage 32 fp32 values (times mul) as bf16 chunk `ck` of this thread's row.
  auto stage_chunk = [&](int ck, const float* v, float mul) {
#pragma unroll
    for (int c8 = 0; c8 < 4; ++c8) {
      const int c = ck * 4 + c8;
      st_shared_v4(stage + lane * RB + ((c ^ (lane & SWM)) << 4),
                   pack_bf16x2(v[8 * c8 + 0] * mul, v[8 * c8 + 1] * mul),
                   pack_bf16x2(v[8 * c8 + 2] * mul, v[8 * c8 + 3] * mul),
                   pack_bf16x2(v[8 * c8 + 4] * mul, v[8 * c8 + 5] * mul),
                   pack_bf16x2(v[8 * c8 + 6] * mul, v[8 * c8 + 7] * mul));
    }
  };
  // Write the warp's 32 staged rows (rows row0 + j below `limit`) to dst.
  auto flush_rows = [&](__nv_bfloat16* dst, int64_t row0, int limit) {
    __syncwarp();
#pragma unroll 1
    for (int it = 0; it < CPR; ++it) {
      const int lin = it * 32 + lane;
      const int j = lin / CPR, c = lin % CPR;
      const uint4 vv = ld_shared_v4(stage + j * RB + ((c ^ (j & SWM)) << 4));
      if (j < limit)
        *reinterpret_cast<uint4*>(dst + ((row0 + j) * a.H) * C::D + c * 8) = vv;
    }
    __syncwarp();
  };

  uint32_t gp = 0, gb = 0;
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
        for (int idx = rtid; idx < rows * (C::D / 8); idx += 128) {
          const int rr = idx / (C::D / 8), cc = (idx % (C::D / 8)) * 8;
          *reinterpret_cast<uint4*>(a.dq + ((int64_t)(t.q0 + mt * kBlockM + rr) * a.H + t.h) *
                                                 C::D + cc) = make_uint4(0, 0, 0, 0);
        }
      }
    }
    bool ok = for_each_pair(
        t, a.wl, a.wr,
        [&](const BPair& x) -> bool {
          const uint32_t p = gp;
          const int m0 = x.mt * kBlockM;
          float4* scr4 = reinterpret_cast<float4*>(a.dq_scratch) +
                         (((int64_t)blockIdx.x * slot_tiles + x.mt) * (C::D / 4)) * kBlockM + r;
          const bool row_ok = m0 + r < t.Lq;
          __nv_bfloat16* dq_row = a.dq + ((int64_t)(t.q0 + m0 + r) * a.H + t.h) * C::D;
          float4 part[HW / 4];
          if (!x.dq_first) {
#pragma unroll
            for (int c = 0; c < HW / 4; ++c)
              part[c] = ld_global_v4_hint(reinterpret_cast<const float*>(scr4 + c * kBlockM),
                                          pol_keep);
          }
          RED_WAIT(C::B_DQFULL, p & 1);
          tc_fence_after();
#pragma unroll
          for (int h = 0; h < NHALF; ++h) {
            float v[HW];
#pragma unroll
            for (int ck = 0; ck < HW / 32; ++ck)
              tmem_ld32f(tmem + tl + C::T_DP + h * HW + ck * 32, v + ck * 32);
            tmem_wait_ld();
            if (h == NHALF - 1) {  // dQ read out: the dP^T columns are free
              tc_fence_before();
              mbar_arrive(sm.bar(C::B_DQEMPTY));
            }
            if (!x.dq_first) {
#pragma unroll
              for (int c = 0; c < HW / 4; ++c) add4_ordered(v + 4 * c, part[c]);
              if (h + 1 < NHALF) {  // the next half's partial, before its TMEM read
#pragma unroll
                for (int c = 0; c < HW / 4; ++c)
                  part[c] = ld_global_v4_hint(
                      reinterpret_cast<const float*>(scr4 + ((h + 1) * (HW / 4) + c) * kBlockM),
                      pol_keep);
              }
            }
            if (!x.dq_last) {
#pragma unroll
              for (int c = 0; c < HW / 4; ++c)
                st_global_v4_hint(reinterpret_cast<float*>(scr4 + (h * (HW / 4) + c) * kBlockM),
                                  make_float4(v[4 * c], v[4 * c + 1], v[4 * c + 2], v[4 * c + 3]),
                                  pol_keep);
            } else if (row_ok) {
              if (a.rope_q) {
#pragma unroll
                for (int c = 0; c < HW; c += 32)
                  unturn32(v + c, a.rope_q + (t.q0 + m0 + r) * (int64_t)(C::D / 2),
                           (h * HW + c) / 2);
              }
#pragma unroll
              for (int c8 = 0; c8 < HW / 8; ++c8)
                *reinterpret_cast<uint4*>(dq_row + h * HW + c8 * 8) = make_uint4(
                    pack_bf16x2(v[8 * c8 + 0] * a.scale, v[8 * c8 + 1] * a.scale),
                    pack_bf16x2(v[8 * c8 + 2] * a.scale, v[8 * c8 + 3] * a.scale),
                    pack_bf16x2(v[8 * c8 + 4] * a.scale, v[8 * c8 + 5] * a.scale),
                    pack_bf16x2(v[8 * c8 + 6] * a.scale, v[8 * c8 + 7] * a.scale));
            }
          }
          if (x.dq_last && !x.dq_first && (lane & 7) == 0) {
#pragma unroll 1
            for (int c = 0; c < C::D / 4; ++c) discard_l2_line(scr4 + c * kBlockM);
          }
          if (x.idx + 1 == x.n) {
            // dK, dV of this key block: thread = key row
            RED_WAIT(C::B_DKVFULL, gb & 1);
            tc_fence_after();
            const int wkey = x.kb * C::BN + wq * 32;   // first key of this warp
            // dK (times scale) staged and written, then dV; the accumulators are
            // released once dV has left TMEM
#pragma unroll
            for (int ck = 0; ck < NCH; ++ck) {
              float kr[32];
              tmem_ld32f(tmem + tl + C::T_DK + ck * 32, kr);
              tmem_wait_ld();
              if (a.rope_kv && wkey + lane < t.Lk)
                unturn32(kr, a.rope_kv + (t.k0 + wkey + lane) * (int64_t)(C::D / 2), ck * 16);
              stage_chunk(ck, kr, a.scale);
            }
            flush_rows(a.dk + (int64_t)t.h * C::D, (int64_t)t.k0 + wkey, t.Lk - wkey);
#pragma unroll
            for (int ck = 0; ck < NCH; ++ck) {
              float vr[32];
              tmem_ld32f(tmem + tl + C::T_DV + ck * 32, vr);
              tmem_wait_ld();
              stage_chunk(ck, vr, 1.f);
            }
            tc_fence_before();
            mbar_arrive(sm.bar(C::B_DKVEMPTY));
            flush_rows(a.dv + (int64_t)t.h * C::D, (int64_t)t.k0 + wkey, t.Lk - wkey);
            ++gb;
            // the dS panel may take the next key block's dS
            mbar_arrive(sm.bar(C::B_DSFREE));
          }
          ++gp;
          return true;
        },
        [&](int kb) -> bool {
          // no query sees this key block: its dK, dV rows are zero
          const int key = kb * C::BN + r;
          if (key < t.Lk) {
            const int64_t row = ((int64_t)(t.k0 + key) * a.H + t.h) * C::D;
#pragma unroll
            for (int e = 0; e < C::D; e += 8) {
              *reinterpret_cast<uint4*>(a.dk + row + e) = make_uint4(0, 0, 0, 0);
              *reinterpret_cast<uint4*>(a.dv + row + e) = make_uint4(0, 0, 0, 0);
            }
          }
          return true;
        });
    if (!ok) return;
  }
#undef RED_WAIT
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
    for (int i = 0; i < 2; ++i) {
      mbar_init(sm.bar(C::B_QFULL + i), 1);
      mbar_init(sm.bar(C::B_QEMPTY + i), 1);
      mbar_init(sm.bar(C::B_DOFULL + i), 1);
      mbar_init(sm.bar(C::B_DOEMPTY + i), 1);
      mbar_init(sm.bar(C::B_RFULL + i), 32);
      mbar_init(sm.bar(C::B_REMPTY + i), 256);
    }
    mbar_init(sm.bar(C::B_SFULL), 1);
    mbar_init(sm.bar(C::B_PFULL), 256);
    mbar_init(sm.bar(C::B_DPFULL), 1);
    mbar_init(sm.bar(C::B_DSFULL), 256);
    mbar_init(sm.bar(C::B_DQFULL), 1);
    mbar_init(sm.bar(C::B_DQEMPTY), 128);
    mbar_init(sm.bar(C::B_DSFREE), 128);
    mbar_init(sm.bar(C::B_DKVFULL), 1);
    mbar_init(sm.bar(C::B_DKVEMPTY), 128);
    mbar_init(sm.bar(C::B_PREAD), 256);
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

  // Registers: the launch gives 512 x 128; warpgroup 0 (producer, MMA issuer,
  // allocator, row loader) and the compute warpgroups release some to the
  // reducer, which holds half an fp32 dQ row and its partial: 128 x 80 +
  // 256 x 120 + 128 x 192 = 65536.  Each budget is set inside its own branch so
  // the compiler allocates each role's code against it.
  if (warp < 4) {
    setmaxnreg_to<kRegsControl, kRegsLaunch>();
    if (warp == 0) {
      if (lane == 0) bwd_producer<C>(a, sm, &tq, &tk, &tv, &tdo);
    } else if (warp == 1) {
      if (lane == 0) bwd_mma<C>(a, sm, tmem);
    } else if (warp == 2) {
      if (PHI == 1) bwd_rows<C>(a, sm);
    }
  } else if (warp < 12) {
    setmaxnreg_to<kRegsCompute, kRegsLaunch>();
    bwd_compute<C, PHI>(a, sm, tmem);
  } else {
    setmaxnreg_to<kRegsReduce, kRegsLaunch>();
    bwd_reduce<C>(a, sm, tmem);
  }
  __syncwarp();
  tc_fence_before();
  __syncthreads();
  if (*sm.abort_flag()) {
    // a role gave up: let copies and MMAs already in flight land before the
    // shared memory and TMEM they target are released
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
  // The compute warpgroups raise their register budget with setmaxnreg, which
  // waits until the block's launch registers cover it: never launch a build
  // whose per-thread count would leave that wait unsatisfiable.
  cudaFuncAttributes fa;
  cudaError_t e = cudaFuncGetAttributes(&fa, kern);
  if (e != cudaSuccess) return e;
  if (fa.numRegs * kBwdThreads < 128 * kRegsControl + 256 * kRegsCompute + 128 * kRegsReduce)
    return cudaErrorInvalidValue;
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
