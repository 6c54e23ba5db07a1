// gdpa_fwd.cu -- fused GDPA forward for sm_100a.
//
// Computes, per sample b and head h, O = phi(scale * Q K^T + beta) V with S and
// phi(S) kept on chip (Kunlun paper review §2.3 "GDPA", Fig. 2: QK^T / tau, then
// the activation, then Attn x V, fused block-wise; Kunlun Breakdown, "The Core
// Architecture and Mechanics": one FlashAttention-style kernel).  phi is SiLU or
// identity (element-wise) or a row softmax with running max and sum (Kunlun
// reproduction notes, "Core equations": softmax(QK^T/sqrt(d) + log sigma(G))).
//
// One persistent CTA per SM walks (sample, head) units in longest-first order.
// For each 128-row query tile of the unit it walks the key blocks the tile can
// see (all of them, or the band of the sliding window, Kunlun paper review
// §2.5), so padding rows and invisible key blocks are never loaded.
//
// Warp roles (256 threads):
//   warp 0     TMA producer: Q tile (2 buffers), K and V blocks (ring of stages)
//   warp 1     MMA issuer (one thread): S = Q K^T into TMEM (2 buffers),
//              O += P V into TMEM
//   warp 2     TMEM allocator
//   warp 3     bias warp: beta for each key block (log sigma(G) for the gate)
//   warps 4-7  phi / epilogue warpgroup: one thread per query row; reads S
//              from TMEM, applies the mask and phi, writes P (bf16) to shared
//              memory for the PV MMA, rescales O when the running max moves,
//              and writes O (bf16) and LSE at the end of the tile.
// Every wait is bounded; on expiry the kernel records GDPA_ERR_TIMEOUT in the
// workspace status, all roles leave their loops, TMEM is freed and the kernel
// returns.
#include <algorithm>
#include <cfloat>
#include <climits>

#include "gdpa_internal.h"

namespace gdpa {
namespace {

template <int D_, int BN_>
struct FwdCfg {
  static constexpr int D = D_;
  static constexpr int BN = BN_;
  static constexpr int BM = kBlockM;
  // Q/K/V panels: 64 bf16 (128 B) wide with 128-byte swizzle, or 32 wide
  // (64 B, 64-byte swizzle) when D = 32.  P panels are always 64 keys wide.
  static constexpr int PANEL_ELEMS = D >= 64 ? 64 : 32;
  static constexpr int PANEL_BYTES = PANEL_ELEMS * 2;
  static constexpr int NPANEL = D / PANEL_ELEMS;
  static constexpr uint32_t LAYOUT = D >= 64 ? LAYOUT_SW128 : LAYOUT_SW64;
  static constexpr int Q_BYTES = BM * D * 2;
  static constexpr int KV_BYTES = BN * D * 2;
  static constexpr int P_BYTES = BM * BN * 2;
  static constexpr int NQ = 2;
  // K/V ring: 2 stages of 64 KB for D = 128 with 128-key blocks, else 3-4
  static constexpr int NKV = (D == 128 && BN == 128) ? 2 : (D * BN <= 64 * 64 ? 4 : 3);
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = OFF_Q + NQ * Q_BYTES;
  static constexpr int OFF_V = OFF_K + NKV * KV_BYTES;
  static constexpr int OFF_P = OFF_V + NKV * KV_BYTES;
  static constexpr int OFF_STAGE = OFF_P + P_BYTES;        // O staging when D > BN
  static constexpr int STAGE_BYTES = D > BN ? BM * D * 2 : 0;
  static constexpr int OFF_BIAS = OFF_STAGE + STAGE_BYTES;   // float [2][BN]
  static constexpr int OFF_BAR = OFF_BIAS + 2 * BN * 4;     // uint64 barriers
  // barrier indices
  static constexpr int B_QFULL = 0;
  static constexpr int B_QEMPTY = B_QFULL + NQ;
  static constexpr int B_KVFULL = B_QEMPTY + NQ;
  static constexpr int B_KVEMPTY = B_KVFULL + NKV;
  static constexpr int B_SFULL = B_KVEMPTY + NKV;
  static constexpr int B_SEMPTY = B_SFULL + 2;
  static constexpr int B_PFULL = B_SEMPTY + 2;
  static constexpr int B_PVDONE = B_PFULL + 1;
  static constexpr int B_OFULL = B_PVDONE + 1;
  static constexpr int B_OEMPTY = B_OFULL + 1;
  static constexpr int B_BFULL = B_OEMPTY + 1;   // 2 bias buffers
  static constexpr int B_BEMPTY = B_BFULL + 2;
  static constexpr int NBARS = B_BEMPTY + 2;
  static constexpr int OFF_MISC = OFF_BAR + NBARS * 8;      // tmem addr, abort flag
  static constexpr int SMEM_BYTES = OFF_MISC + 16;
  static constexpr int SMEM_ALLOC = SMEM_BYTES;  // base is 1024-aligned (checked at entry)
  // TMEM: S buffers at columns [0, BN) and [BN, 2BN); O at [2BN, 2BN + D).
  static constexpr int TMEM_S0 = 0;
  static constexpr int TMEM_O = 2 * BN;
  static constexpr int TMEM_COLS = (2 * BN + D) <= 256 ? 256 : 512;
  static_assert(SMEM_ALLOC <= 232448, "shared memory budget");
  static_assert(Q_BYTES % 1024 == 0 && KV_BYTES % 1024 == 0 && P_BYTES % 1024 == 0, "align");
};

constexpr int kThreads = 256;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr float kRescaleThreshold = 8.0f;  // log2 units: P stays below 2^8

using Unit = GdpaUnit;

// Key-block range [kb0, kb1) a tile starting at local row m0 may touch.
template <int BN>
__device__ __forceinline__ void kv_range(int m0, int Lk, int wl, int wr, int& kb0, int& kb1) {
  int lo = wl >= 0 ? max(0, m0 - wl) : 0;
  int hi = wr >= 0 ? min(Lk, m0 + kBlockM + wr) : Lk;
  if (hi <= lo) {
    kb0 = kb1 = 0;
  } else {
    kb0 = lo / BN;
    kb1 = (hi + BN - 1) / BN;
  }
}

// K/V stay in shared memory for all query tiles of a unit when there is no
// band (every tile sees every key block), the unit has more than one tile,
// and its key blocks fit in the K/V ring.  Otherwise each tile streams the
// blocks it can see.
template <class C>
__device__ __forceinline__ bool kv_resident(const FwdArgs& a, const Unit& t, int& nkb) {
  nkb = (t.Lk + C::BN - 1) / C::BN;
  return a.wl < 0 && a.wr < 0 && t.Lq > kBlockM && nkb > 0 && nkb <= C::NKV;
}

template <class C>
struct Smem {
  uint32_t base;  // shared address of the 1024-aligned base
  uint8_t* ptr;
  __device__ uint32_t q(int s) const { return base + C::OFF_Q + s * C::Q_BYTES; }
  __device__ uint32_t k(int s) const { return base + C::OFF_K + s * C::KV_BYTES; }
  __device__ uint32_t v(int s) const { return base + C::OFF_V + s * C::KV_BYTES; }
  __device__ uint32_t p() const { return base + C::OFF_P; }
  // O staging of warp w, row j (0..31), 16-byte chunk cc, chunks XOR-swizzled by
  // row.  With D <= BN it lies in the P rows 32w..32w+31 of each 64-key panel
  // (only warp w writes those); otherwise in a separate region.
  __device__ uint32_t stage(int w, int j, int cc) const {
    constexpr int ROWB = C::D * 2;
    constexpr int SW = (ROWB / 16) >= 8 ? 7 : 3;
    const uint32_t b = j * ROWB + ((cc ^ (j & SW)) << 4);
    if constexpr (C::D <= C::BN) {
      return base + C::OFF_P + (b >> 12) * (kBlockM * 128) + w * 32 * 128 + (b & 4095);
    } else {
      return base + C::OFF_STAGE + w * 32 * ROWB + b;
    }
  }
  __device__ float* bias(int s) const {
    return reinterpret_cast<float*>(ptr + C::OFF_BIAS) + s * C::BN;
  }
  __device__ uint32_t bar(int i) const { return base + C::OFF_BAR + i * 8; }
  __device__ uint32_t* tmem_slot() const { return reinterpret_cast<uint32_t*>(ptr + C::OFF_MISC); }
  __device__ volatile int* abort_flag() const {
    return reinterpret_cast<volatile int*>(ptr + C::OFF_MISC + 4);
  }
};

// ------------------------------------------------------------------ producer
template <class C>
__device__ void role_producer(const FwdArgs& a, const Smem<C>& sm, const CUtensorMap* tq,
                              const CUtensorMap* tk, const CUtensorMap* tv) {
  volatile int* abort = sm.abort_flag();
  const uint64_t pol_stream = l2_policy_evict_first();
  const uint64_t pol_keep = l2_policy_evict_last();
  uint32_t qi = 0, kvi = 0;
  bool dropped = false;
  UnitStream units(a.info, a.H, a.n_units);
  Unit t;
  while (units.next(t)) {
    const int ntile = (t.Lq + kBlockM - 1) / kBlockM;
    int nkb;
    const bool resident = kv_resident<C>(a, t, nkb);
    auto load_kv = [&](int j) -> bool {
      const int ks = kvi % C::NKV;
      if (!mbar_wait(sm.bar(C::B_KVEMPTY + ks), ((kvi / C::NKV) & 1) ^ 1, abort, a.status,
                     a.timeout_ns, 0x000 + C::B_KVEMPTY + ks))
        return false;
      mbar_arrive_expect_tx(sm.bar(C::B_KVFULL + ks), 2 * C::KV_BYTES);
      for (int pnl = 0; pnl < C::NPANEL; ++pnl) {
        tma_load_3d(sm.k(ks) + pnl * C::BN * C::PANEL_BYTES, tk, sm.bar(C::B_KVFULL + ks),
                    pnl * C::PANEL_ELEMS, t.h, t.k0 + j * C::BN, pol_keep);
        tma_load_3d(sm.v(ks) + pnl * C::BN * C::PANEL_BYTES, tv, sm.bar(C::B_KVFULL + ks),
                    pnl * C::PANEL_ELEMS, t.h, t.k0 + j * C::BN, pol_keep);
      }
      ++kvi;
      return true;
    };
    for (int mt = 0; mt < ntile; ++mt) {
      const int m0 = mt * kBlockM;
      int kb0, kb1;
      kv_range<C::BN>(m0, t.Lk, a.wl, a.wr, kb0, kb1);
      if (kb1 <= kb0) continue;
      const int qs = qi % C::NQ;
      if (!mbar_wait(sm.bar(C::B_QEMPTY + qs), ((qi / C::NQ) & 1) ^ 1, abort, a.status,
                     a.timeout_ns, 0x000 + C::B_QEMPTY + qs))
        return;
      if ((a.debug_flags & 1) && !dropped && blockIdx.x == 0) {
        dropped = true;  // test hook: this Q tile is never loaded
      } else {
        mbar_arrive_expect_tx(sm.bar(C::B_QFULL + qs), C::Q_BYTES);
        for (int pnl = 0; pnl < C::NPANEL; ++pnl)
          tma_load_3d(sm.q(qs) + pnl * kBlockM * C::PANEL_BYTES, tq, sm.bar(C::B_QFULL + qs),
                      pnl * C::PANEL_ELEMS, t.h, t.q0 + m0, pol_stream);
      }
      ++qi;
      if (resident && mt > 0) continue;  // the unit's blocks are already in the ring
      for (int j = kb0; j < kb1; ++j)
        if (!load_kv(j)) return;
    }
  }
}

// ------------------------------------------------------------------ MMA issuer
// The issuer keeps one PV behind: S of the next key block (of this tile, or of
// the next tile or unit) is issued before the PV of the current one, so the
// phi warpgroup finds its next S ready when it finishes a block or a tile.
template <class C>
__device__ void role_mma(const FwdArgs& a, const Smem<C>& sm, uint32_t tmem) {
  volatile int* abort = sm.abort_flag();
  constexpr uint32_t idesc_s = make_idesc_bf16(kBlockM, C::BN, 0, 0);
  constexpr uint32_t idesc_o = make_idesc_bf16(kBlockM, C::D, 0, 1);
  constexpr uint32_t SBO_QK = 8 * C::PANEL_BYTES;
  uint32_t qi = 0, kvi = 0, si = 0, pvi = 0, ti = 0;

  struct PendingPV {
    bool valid;
    bool first;         // first key block of its tile (overwrites O)
    bool last;          // last key block of its tile (O complete afterwards)
    int ks;             // K/V stage holding V
    bool release_kv;    // streamed block: free its stage after this PV
    uint32_t unit_kvi;  // resident unit ending with this PV: free its stages
    int unit_nkb;       //   (0 when not)
  } pend = {false, false, false, 0, false, 0u, 0};

  auto issue_pending = [&]() -> bool {
    if (!pend.valid) return true;
    if (!mbar_wait(sm.bar(C::B_PFULL), pvi & 1, abort, a.status, a.timeout_ns,
                   0x100 + C::B_PFULL))
      return false;
    if (pend.first && !mbar_wait(sm.bar(C::B_OEMPTY), (ti & 1) ^ 1, abort, a.status,
                                 a.timeout_ns, 0x100 + C::B_OEMPTY))
      return false;
    tc_fence_after();
#pragma unroll
    for (int kk = 0; kk < C::BN / 16; ++kk) {
      // A = P [128 x BN] K-major, 64-key panels with 128-byte swizzle
      const uint32_t pa = sm.p() + (kk * 16 / 64) * (kBlockM * 128) + (kk * 16 % 64) * 2;
      const uint64_t adesc = make_smem_desc(pa, 16, 1024, LAYOUT_SW128);
      // B = V [BN keys x D], N (= D) contiguous: MN-major; 16 keys per step
      const uint32_t vb = sm.v(pend.ks) + kk * 16 * C::PANEL_BYTES;
      const uint64_t bdesc = make_smem_desc(vb, C::BN * C::PANEL_BYTES, SBO_QK, C::LAYOUT);
      mma_bf16_ss(tmem + C::TMEM_O, adesc, bdesc, idesc_o, (!pend.first || kk > 0) ? 1u : 0u);
    }
    if (pend.release_kv) mma_commit(sm.bar(C::B_KVEMPTY + pend.ks));
    mma_commit(sm.bar(C::B_PVDONE));
    ++pvi;
    if (pend.last) {
      mma_commit(sm.bar(C::B_OFULL));
      ++ti;
    }
    for (int idx = 0; idx < pend.unit_nkb; ++idx)
      mma_commit(sm.bar(C::B_KVEMPTY + (pend.unit_kvi + idx) % C::NKV));
    pend.valid = false;
    return true;
  };

  UnitStream units(a.info, a.H, a.n_units);
  Unit t;
  while (units.next(t)) {
    const int ntile = (t.Lq + kBlockM - 1) / kBlockM;
    int nkb;
    const bool resident = kv_resident<C>(a, t, nkb);
    const uint32_t unit_kvi = kvi;  // first ring index of a resident unit
    for (int mt = 0; mt < ntile; ++mt) {
      int kb0, kb1;
      kv_range<C::BN>(mt * kBlockM, t.Lk, a.wl, a.wr, kb0, kb1);
      const int nkv = kb1 - kb0;
      if (nkv <= 0) continue;
      const int qs = qi % C::NQ;
      if (!mbar_wait(sm.bar(C::B_QFULL + qs), (qi / C::NQ) & 1, abort, a.status, a.timeout_ns,
                     0x100 + C::B_QFULL + qs))
        return;
      if (resident) kvi = unit_kvi;  // every tile walks the same resident stages
      for (int idx = 0; idx < nkv; ++idx) {
        const int ks = kvi % C::NKV;
        // a resident unit frees its stages with its last PV; the next unit's
        // first load may need them, so that PV is not deferred past this wait
        if (pend.valid && pend.unit_nkb > 0 && !issue_pending()) return;
        if ((!resident || mt == 0) &&
            !mbar_wait(sm.bar(C::B_KVFULL + ks), (kvi / C::NKV) & 1, abort, a.status,
                       a.timeout_ns, 0x100 + C::B_KVFULL + ks))
          return;
        const int sb = si & 1;
        if (!mbar_wait(sm.bar(C::B_SEMPTY + sb), ((si >> 1) & 1) ^ 1, abort, a.status,
                       a.timeout_ns, 0x100 + C::B_SEMPTY + sb))
          return;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < C::D / 16; ++kk) {
          const int pnl = kk * 16 / C::PANEL_ELEMS;
          const int within = (kk * 16 % C::PANEL_ELEMS) * 2;
          const uint64_t adesc = make_smem_desc(
              sm.q(qs) + pnl * kBlockM * C::PANEL_BYTES + within, 16, SBO_QK, C::LAYOUT);
          const uint64_t bdesc = make_smem_desc(
              sm.k(ks) + pnl * C::BN * C::PANEL_BYTES + within, 16, SBO_QK, C::LAYOUT);
          mma_bf16_ss(tmem + C::TMEM_S0 + sb * C::BN, adesc, bdesc, idesc_s, kk > 0 ? 1u : 0u);
        }
        mma_commit(sm.bar(C::B_SFULL + sb));
        ++si;
        if (idx == nkv - 1) {
          mma_commit(sm.bar(C::B_QEMPTY + qs));
          ++qi;
        }
        ++kvi;
        // the previous block's PV, now that this block's S is on its way
        if (!issue_pending()) return;
        const bool last_of_unit = resident && mt == ntile - 1 && idx == nkv - 1;
        pend = {true, idx == 0, idx == nkv - 1, ks, !resident,
                last_of_unit ? unit_kvi : 0u, last_of_unit ? nkb : 0};
      }
    }
    if (resident) kvi = unit_kvi + nkb;
  }
  issue_pending();
}

// ------------------------------------------------------------------ bias warp
template <class C>
__device__ void role_bias(const FwdArgs& a, const Smem<C>& sm, bool softmax) {
  volatile int* abort = sm.abort_flag();
  const int lane = threadIdx.x & 31;
  uint32_t bi = 0;
  UnitStream units(a.info, a.H, a.n_units);
  Unit t;
  while (units.next(t)) {
    const int ntile = (t.Lq + kBlockM - 1) / kBlockM;
    for (int mt = 0; mt < ntile; ++mt) {
      int kb0, kb1;
      kv_range<C::BN>(mt * kBlockM, t.Lk, a.wl, a.wr, kb0, kb1);
      for (int j = kb0; j < kb1; ++j) {
        const int bs = bi & 1;
        bool ok = mbar_wait(sm.bar(C::B_BEMPTY + bs), ((bi >> 1) & 1) ^ 1, abort, a.status,
                            a.timeout_ns, 0x300 + C::B_BEMPTY + bs);
        if (!__all_sync(0xffffffffu, ok)) return;
        float* dst = sm.bias(bs);
        const float* src = a.bias + (int64_t)t.h * a.total_kv + t.k0;
        for (int c = lane; c < C::BN; c += 32) {
          const int key = j * C::BN + c;
          float beta = 0.f;
          if (key < t.Lk) {
            const float g = src[key];
            if (a.bias_kind == 2) {
              // log sigma(g) = min(g, 0) - log(1 + exp(-|g|))
              beta = fminf(g, 0.f) - log1pf(__expf(-fabsf(g)));
            } else {
              beta = g;
            }
          }
          dst[c] = softmax ? beta * kLog2e : beta;
        }
        mbar_arrive(sm.bar(C::B_BFULL + bs));  // one arrival per lane, after its writes
        ++bi;
      }
    }
  }
}

// ------------------------------------------------------------------ phi warpgroup
template <class C, bool SOFTMAX>
__device__ void role_phi(const FwdArgs& a, const Smem<C>& sm, uint32_t tmem) {
  volatile int* abort = sm.abort_flag();
  const int wq = (threadIdx.x >> 5) & 3;  // TMEM lane quarter of this warp
  const int lane = threadIdx.x & 31;
  const int r = wq * 32 + lane;             // row of the tile owned by this thread
  const uint32_t tl = (uint32_t)(wq * 32) << 16;
  const bool has_bias = a.bias_kind != 0;
  const bool identity = a.phi == 2;
  const float sc = SOFTMAX ? a.scale * kLog2e : a.scale;
  uint32_t si = 0, pvi = 0, ti = 0, bi = 0;

#define PHI_WAIT(bar_, par_, where_)                                                   \
  do {                                                                               \
    bool ok_ = mbar_wait(sm.bar(bar_), (par_), abort, a.status, a.timeout_ns, where_); \
    if (!__all_sync(0xffffffffu, ok_)) return;                                       \
  } while (0)

  UnitStream units(a.info, a.H, a.n_units);
  Unit t;
  while (units.next(t)) {
    const int ntile = (t.Lq + kBlockM - 1) / kBlockM;
    for (int mt = 0; mt < ntile; ++mt) {
      const int m0 = mt * kBlockM;
      const int row = m0 + r;
      const bool row_ok = row < t.Lq;
      int kb0, kb1;
      kv_range<C::BN>(m0, t.Lk, a.wl, a.wr, kb0, kb1);
      const int nkv = kb1 - kb0;
      if (nkv <= 0) {
        if (row_ok) {
          __nv_bfloat16* orow = a.o + ((int64_t)(t.q0 + row) * a.H + t.h) * C::D;
          uint4 z = make_uint4(0, 0, 0, 0);
          for (int c = 0; c < C::D; c += 8) *reinterpret_cast<uint4*>(orow + c) = z;
          if (SOFTMAX && a.lse) a.lse[(int64_t)t.h * a.total_q + t.q0 + row] = -INFINITY;
        }
        continue;
      }
      // visible keys of this row: [lo, hi]
      const int lo = a.wl >= 0 ? row - a.wl : INT_MIN;
      const int hi = min(t.Lk - 1, a.wr >= 0 ? row + a.wr : INT_MAX);
      float m_run = -INFINITY, l_run = 0.f;
      for (int idx = 0; idx < nkv; ++idx) {
        const int kbase = (kb0 + idx) * C::BN;
        const int bs = bi & 1;
        if (has_bias) PHI_WAIT(C::B_BFULL + bs, (bi >> 1) & 1, 0x400 + C::B_BFULL + bs);
        const int sb = si & 1;
        PHI_WAIT(C::B_SFULL + sb, (si >> 1) & 1, 0x400 + C::B_SFULL + sb);
        tc_fence_after();
        uint32_t sv[C::BN];  // S row, then P (fp32 bits), in place
#pragma unroll
        for (int c = 0; c < C::BN / 32; ++c)
          tmem_ld32p(tmem + tl + C::TMEM_S0 + sb * C::BN + c * 32, sv + c * 32);
        tmem_wait_ld();
        tc_fence_before();
        mbar_arrive(sm.bar(C::B_SEMPTY + sb));
        ++si;
        const float2* bias2 = reinterpret_cast<const float2*>(sm.bias(bs));
        // visible columns of this block: [clo, chi] (no shift of an unbounded side)
        const int clo = a.wl >= 0 ? lo - kbase : INT_MIN;
        const int chi = hi - kbase;  // hi <= Lk - 1 always
        const bool full = clo <= 0 && chi >= C::BN - 1;
        const uint64_t sc2 = f2_pack(sc, sc);
        // scores x = scale * s + beta, two columns per packed instruction
#pragma unroll
        for (int c = 0; c < C::BN; c += 2) {
          uint64_t x2 = f2_pack(__uint_as_float(sv[c]), __uint_as_float(sv[c + 1]));
          if (has_bias) {
            const float2 b = bias2[c >> 1];
            x2 = f2_fma(x2, sc2, f2_pack(b.x, b.y));
          } else {
            x2 = f2_mul(x2, sc2);
          }
          float x0, x1;
          f2_unpack(x2, x0, x1);
          sv[c] = __float_as_uint(x0);
          sv[c + 1] = __float_as_uint(x1);
        }
        if (!full) {  // band edges and the ragged last key block
          const float fill = SOFTMAX ? -INFINITY : 0.f;
#pragma unroll
          for (int c = 0; c < C::BN; ++c)
            if (c < clo || c > chi) sv[c] = __float_as_uint(fill);
        }
        if (!SOFTMAX) {
          if (!identity) {
            const uint64_t half2 = f2_pack(0.5f, 0.5f);
#pragma unroll
            for (int c = 0; c < C::BN; c += 2) {
              // silu(x) = h + h tanh(h), h = x / 2
              const uint64_t h2 =
                  f2_mul(f2_pack(__uint_as_float(sv[c]), __uint_as_float(sv[c + 1])), half2);
              float h0, h1;
              f2_unpack(h2, h0, h1);
              const uint64_t p2 = f2_fma(h2, f2_pack(tanh_approx(h0), tanh_approx(h1)), h2);
              float p0, p1;
              f2_unpack(p2, p0, p1);
              sv[c] = __float_as_uint(p0);
              sv[c + 1] = __float_as_uint(p1);
            }
            if (!full) {  // silu(0) = 0 already; keep masked columns exactly zero
#pragma unroll
              for (int c = 0; c < C::BN; ++c)
                if (c < clo || c > chi) sv[c] = 0u;
            }
          }
        }
        if (has_bias) {
          tc_fence_before();
          mbar_arrive(sm.bar(C::B_BEMPTY + bs));
          ++bi;
        }
        bool need_rescale = false;
        float factor = 1.f;
        if (SOFTMAX) {
          // 4 independent partial maxima over 3-input max: no BN-long chain
          float pm[4];
#pragma unroll
          for (int k = 0; k < 4; ++k) pm[k] = -INFINITY;
#pragma unroll
          for (int c = 0; c < C::BN; c += 2)
            pm[(c >> 1) & 3] = fmax3(pm[(c >> 1) & 3], __uint_as_float(sv[c]),
                                     __uint_as_float(sv[c + 1]));
          const float bm = fmax3(fmaxf(pm[0], pm[1]), pm[2], pm[3]);
          if (idx == 0) {
            m_run = bm;
          } else if (bm > m_run + kRescaleThreshold) {
            factor = (m_run == -INFINITY) ? 0.f : ex2_approx(m_run - bm);
            need_rescale = true;
            l_run *= factor;
            m_run = bm;
          }
          const float m_use = (m_run == -INFINITY) ? 0.f : m_run;
          const uint64_t neg_m2 = f2_pack(-m_use, -m_use);
          uint64_t ps2[2] = {0ull, 0ull};  // packed partial sums
#pragma unroll
          for (int c = 0; c < C::BN; c += 2) {
            const uint64_t d2 =
                f2_add(f2_pack(__uint_as_float(sv[c]), __uint_as_float(sv[c + 1])), neg_m2);
            float d0, d1;
            f2_unpack(d2, d0, d1);
            const float p0 = ex2_approx(d0), p1 = ex2_approx(d1);
            sv[c] = __float_as_uint(p0);
            sv[c + 1] = __float_as_uint(p1);
            ps2[(c >> 1) & 1] = f2_add(ps2[(c >> 1) & 1], f2_pack(p0, p1));
          }
          float s0, s1, s2, s3;
          f2_unpack(ps2[0], s0, s1);
          f2_unpack(ps2[1], s2, s3);
          l_run += (s0 + s1) + (s2 + s3);
        }
        // the previous PV must be done before P is overwritten or O rescaled
        if (idx > 0) PHI_WAIT(C::B_PVDONE, (pvi - 1) & 1, 0x400 + C::B_PVDONE);
        if (SOFTMAX && __any_sync(0xffffffffu, need_rescale)) {
          tc_fence_after();
#pragma unroll
          for (int c = 0; c < C::D / 16; ++c) {
            uint32_t raw[16];
            tmem_ld16(tmem + tl + C::TMEM_O + c * 16, raw);
            tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 16; ++e)
              raw[e] = __float_as_uint(__uint_as_float(raw[e]) * factor);
            tmem_st16(tmem + tl + C::TMEM_O + c * 16, raw);
          }
          tmem_wait_st();
        }
        // P row -> shared memory, 64-key panels, 128-byte swizzle (K-major A operand)
#pragma unroll
        for (int ch = 0; ch < C::BN / 8; ++ch) {
          const int pnl = ch / 8, cir = ch % 8;
          const uint32_t addr =
              sm.p() + pnl * (kBlockM * 128) + r * 128 + ((cir ^ (r & 7)) << 4);
          const uint32_t* q8 = sv + ch * 8;
          st_shared_v4(addr, pack_bf16x2(__uint_as_float(q8[0]), __uint_as_float(q8[1])),
                       pack_bf16x2(__uint_as_float(q8[2]), __uint_as_float(q8[3])),
                       pack_bf16x2(__uint_as_float(q8[4]), __uint_as_float(q8[5])),
                       pack_bf16x2(__uint_as_float(q8[6]), __uint_as_float(q8[7])));
        }
        fence_proxy_async_smem();
        tc_fence_before();
        mbar_arrive(sm.bar(C::B_PFULL));
        ++pvi;
      }
      // epilogue: O row from TMEM -> bf16 -> this warp's staging rows in shared
      // memory -> whole rows to global memory (coalesced); the staging area of
      // warp wq lies inside the P rows that only this warp writes
      PHI_WAIT(C::B_OFULL, ti & 1, 0x400 + C::B_OFULL);
      tc_fence_after();
      float inv = 1.f;
      if (SOFTMAX) inv = l_run > 0.f ? 1.f / l_run : 0.f;
#pragma unroll 1  // keeps the epilogue's registers out of the way of the hot loop
      for (int c = 0; c < C::D / 32; ++c) {
        uint32_t raw[32];
        tmem_ld32(tmem + tl + C::TMEM_O + c * 32, raw);
        tmem_wait_ld();
#pragma unroll
        for (int e = 0; e < 32; e += 8) {
          const int cc = (c * 32 + e) / 8;  // 16-byte chunk of the row
          st_shared_v4(sm.stage(wq, lane, cc),
                       pack_bf16x2(__uint_as_float(raw[e + 0]) * inv, __uint_as_float(raw[e + 1]) * inv),
                       pack_bf16x2(__uint_as_float(raw[e + 2]) * inv, __uint_as_float(raw[e + 3]) * inv),
                       pack_bf16x2(__uint_as_float(raw[e + 4]) * inv, __uint_as_float(raw[e + 5]) * inv),
                       pack_bf16x2(__uint_as_float(raw[e + 6]) * inv, __uint_as_float(raw[e + 7]) * inv));
        }
      }
      __syncwarp();
      {
        constexpr int NCH = C::D / 8;  // 16-byte chunks per row
#pragma unroll 1
        for (int it = 0; it < NCH; ++it) {
          const int lin = it * 32 + lane;
          const int j = lin / NCH, cc = lin % NCH;  // row of this warp, chunk
          const int grow = m0 + wq * 32 + j;
          const uint4 v = ld_shared_v4(sm.stage(wq, j, cc));
          if (grow < t.Lq)
            *reinterpret_cast<uint4*>(a.o + ((int64_t)(t.q0 + grow) * a.H + t.h) * C::D +
                                      cc * 8) = v;
        }
      }
      __syncwarp();
      tc_fence_before();
      mbar_arrive(sm.bar(C::B_OEMPTY));
      ++ti;
      if (SOFTMAX && row_ok && a.lse) {
        a.lse[(int64_t)t.h * a.total_q + t.q0 + row] =
            l_run > 0.f ? (m_run + __log2f(l_run)) * kLn2 : -INFINITY;
      }
    }
  }
#undef PHI_WAIT
}

template <int D, int BN, bool SOFTMAX>
__global__ void __launch_bounds__(kThreads, 1)
    gdpa_fwd_kernel(const __grid_constant__ FwdArgs a, const __grid_constant__ CUtensorMap tq,
                    const __grid_constant__ CUtensorMap tk, const __grid_constant__ CUtensorMap tv) {
  using C = FwdCfg<D, BN>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  Smem<C> sm;
  sm.base = smem_u32(smem_raw);
  sm.ptr = smem_raw;
  if (sm.base & 1023u) {  // swizzled TMA tiles need 1024-byte alignment
    if (threadIdx.x == 0) record_error(a.status, 2, 0x7000);
    return;
  }
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int i = 0; i < C::NQ; ++i) {
      mbar_init(sm.bar(C::B_QFULL + i), 1);
      mbar_init(sm.bar(C::B_QEMPTY + i), 1);
    }
    for (int i = 0; i < C::NKV; ++i) {
      mbar_init(sm.bar(C::B_KVFULL + i), 1);
      mbar_init(sm.bar(C::B_KVEMPTY + i), 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(sm.bar(C::B_SFULL + i), 1);
      mbar_init(sm.bar(C::B_SEMPTY + i), 128);
      mbar_init(sm.bar(C::B_BFULL + i), 32);
      mbar_init(sm.bar(C::B_BEMPTY + i), 128);
    }
    mbar_init(sm.bar(C::B_PFULL), 128);
    mbar_init(sm.bar(C::B_PVDONE), 1);
    mbar_init(sm.bar(C::B_OFULL), 1);
    mbar_init(sm.bar(C::B_OEMPTY), 128);
    *sm.abort_flag() = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tq);
    tma_prefetch_desc(&tk);
    tma_prefetch_desc(&tv);
  }
  if (warp == 2) {
    tmem_alloc(smem_u32(sm.tmem_slot()), C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *sm.tmem_slot();

  if (warp == 0) {
    if (lane == 0) role_producer<C>(a, sm, &tq, &tk, &tv);
  } else if (warp == 1) {
    if (lane == 0) role_mma<C>(a, sm, tmem);
  } else if (warp == 3) {
    if (a.bias_kind != 0) role_bias<C>(a, sm, SOFTMAX);
  } else if (warp >= 4) {
    role_phi<C, SOFTMAX>(a, sm, tmem);
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

template <int D, int BN, bool SOFTMAX>
cudaError_t launch_one(const FwdArgs& a, const CUtensorMap& tq, const CUtensorMap& tk,
                       const CUtensorMap& tv, int sms, cudaStream_t stream) {
  using C = FwdCfg<D, BN>;
  auto kern = gdpa_fwd_kernel<D, BN, SOFTMAX>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       C::SMEM_ALLOC);
  if (e != cudaSuccess) return e;
  int per_sm = 0;
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kThreads, C::SMEM_ALLOC);
  if (e != cudaSuccess) return e;
  if (per_sm < 1) return cudaErrorInvalidConfiguration;
  // persistent: exactly the CTAs that are resident at once
  const int grid = std::max(1, std::min(a.n_units, per_sm * sms));
  kern<<<grid, kThreads, C::SMEM_ALLOC, stream>>>(a, tq, tk, tv);
  return cudaGetLastError();
}

}  // namespace

int forward_block_n(int D, int phi, int max_kv, int debug_flags) {
  (void)D;
  (void)phi;
  return (max_kv <= 64 && !(debug_flags & 2)) ? 64 : 128;
}

cudaError_t launch_forward(const FwdArgs& a, int D, int block_n, const CUtensorMap& tq,
                           const CUtensorMap& tk, const CUtensorMap& tv, int sms,
                           cudaStream_t stream) {
  const bool sm = a.phi == 1;
#define GDPA_FWD_CASE(D_, BN_)                                                       \
  if (D == D_ && block_n == BN_)                                                     \
    return sm ? launch_one<D_, BN_, true>(a, tq, tk, tv, sms, stream)                 \
              : launch_one<D_, BN_, false>(a, tq, tk, tv, sms, stream);
  GDPA_FWD_CASE(32, 64)
  GDPA_FWD_CASE(32, 128)
  GDPA_FWD_CASE(64, 64)
  GDPA_FWD_CASE(64, 128)
  GDPA_FWD_CASE(128, 64)
  GDPA_FWD_CASE(128, 128)
#undef GDPA_FWD_CASE
  return cudaErrorInvalidValue;
}

}  // namespace gdpa
