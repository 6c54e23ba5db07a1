// gdpa_fwd.cu -- fused GDPA forward for sm_100a.
//
// Computes, per sample b and head h, O = phi(scale * Q K^T + beta) V with S and
// phi(S) kept on chip (Kunlun paper review §2.3 "GDPA", Fig. 2: QK^T / tau, then
// the activation, then Attn x V, fused block-wise; Kunlun Breakdown, "The Core
// Architecture and Mechanics": one FlashAttention-style kernel).  phi is SiLU or
// identity (element-wise) or a row softmax with running max and sum (Kunlun
// reproduction notes, "Core equations": softmax(QK^T/sqrt(d) + log sigma(G))).
//
// One persistent CTA per SM walks (sample, head) units in longest-first order
// and, within a unit, its 128-row query tiles.  Tiles alternate between two
// slots, each with its own phi warpgroup, epilogue warpgroup and TMEM (S of
// one 128-key block and the O accumulator: 2 x 256 columns), so one slot's
// MMAs run while the other slot's phi warpgroup works, and a tile's O is
// written out while the slot's next tile is under way.  P (bf16) goes back
// into TMEM over the S columns it came from and is the A operand of the PV
// MMA.  Q tiles come through a ring of stages; K/V blocks through one ring
// shared by both slots; a unit without a band whose blocks fit in the ring
// loads them once for all its tiles.  A tile only loads the key blocks it can
// see (all of them, or the band of the sliding window, Kunlun paper review
// §2.5).  128-key blocks keep the MMA count low: a tcgen05.mma of 128 x N x 16
// costs about the same for N = 64 and N = 128.
//
// Warp roles (640 threads):
//   warp 0       TMA producer: Q tiles, K/V blocks (tile order); publishes
//                each tile's record to the other roles
//   warps 1, 3   MMA issuers (one thread each) of slot 0 and slot 1:
//                S = Q K^T into the slot's S columns, O += P V
//   warp 2       TMEM allocator; bias warp: beta of each key block (log
//                sigma(G)) for both slots
//   (rotary: warp 1 issues for both slots, warps 2-3 turn Q and K)
//   warps 4-7    phi warpgroup of slot 0, warps 8-11 of slot 1: one thread
//                per query row; reads S from TMEM, applies the mask and phi,
//                writes P to TMEM, rescales O when the running max moves,
//                writes LSE at the end of the tile
//   warps 12-15  epilogue warpgroup of slot 0, warps 16-19 of slot 1: O of
//                each tile from TMEM, times 1/l, to bf16 in global memory
// Every wait is bounded; on expiry the kernel records GDPA_ERR_TIMEOUT in the
// workspace status, all roles leave their loops, TMEM is freed and the kernel
// returns.
#include <algorithm>
#include <atomic>
#include <cfloat>
#include <climits>

#include <cuda_fp16.h>

#include "gdpa_internal.h"
#include "gdpa_pdl.cuh"

namespace gdpa {
namespace {

constexpr int kThreads = 640;
constexpr int kRegsLaunch = 96;    // 65536 / 640 rounded down to a multiple of 8
#ifndef GDPA_FWD_RC
#define GDPA_FWD_RC 96
#endif
#ifndef GDPA_FWD_RP
#define GDPA_FWD_RP 104
#endif
#ifndef GDPA_FWD_RE
#define GDPA_FWD_RE 88
#endif
constexpr int kRegsControl = GDPA_FWD_RC;  // warpgroup 0: producer, MMA issuer, allocator, bias
constexpr int kRegsPhi = GDPA_FWD_RP;      // warpgroups 1-2: phi of slot 0 / 1
constexpr int kRegsEpi = GDPA_FWD_RE;      // warpgroups 3-4: O epilogue of slot 0 / 1
static_assert(128 * kRegsControl + 256 * kRegsPhi + 256 * kRegsEpi <= kThreads * kRegsLaunch,
              "register split exceeds the launch's registers");
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr float kInvSqrt2 = 0.7071067811865476f;  // Phi(x) = (1 + erf(x / sqrt 2)) / 2
constexpr float kRescaleThreshold = 8.0f;  // log2 units: P stays below 2^8

#ifndef GDPA_FWD_NQ
#define GDPA_FWD_NQ 8
#endif

template <int D_, int BN_, bool GROUPED_, bool ROPE_ = false>
struct FwdCfg {
  static constexpr int D = D_;
  static constexpr int BN = BN_;
  static constexpr bool GROUPED = GROUPED_;  // units of several problems
  static constexpr bool ROPE = ROPE_;        // Q and K turned by the rotation tables
  // one MMA issuer per slot (warps 1 and 3), or one for both when warps 2-3
  // turn Q and K (rotary)
  static constexpr bool DUAL = !ROPE_;
  // per-slot issuers with 64-key blocks send S in two halves so that phi of
  // block i + 1 starts after half an S (see role_mma_slot); with 128-key
  // blocks the two N = 64 halves cost more tensor time than the overlap
  // returns (measured), so S goes whole after the previous PV
  static constexpr bool SPLIT = DUAL && BN_ == 64;
  // phi of odd blocks takes the key chunks in descending order and writes P
  // over the upper half of the S columns (what a split S needs; the one-issuer
  // kernels with 64-key blocks do the same, so both compute the same values)
  static constexpr bool ALT = BN_ == 64;
  static constexpr int BM = kBlockM;
  // Q/K/V panels: 64 bf16 (128 B) wide with 128-byte swizzle, or 32 wide
  // (64 B, 64-byte swizzle) when D = 32.
  static constexpr int PANEL_ELEMS = D >= 64 ? 64 : 32;
  static constexpr int PANEL_BYTES = PANEL_ELEMS * 2;
  static constexpr int NPANEL = D / PANEL_ELEMS;
  static constexpr uint32_t LAYOUT = D >= 64 ? LAYOUT_SW128 : LAYOUT_SW64;
  static constexpr int Q_BYTES = BM * D * 2;
  static constexpr int KV_BYTES = BN * D * 2;  // one K (or V) block
  // Q tiles come through a ring of NQ stages, so the producer loads a few tiles
  // ahead of the MMAs (one load's latency no longer sits in every tile's
  // chain): 8 stages for D <= 64, 2 (one per slot) for D = 128, where shared
  // memory is full.  (With short K/V, Q is nearly all a tile reads; 4, 6 and
  // 8 stages measured within 1% of each other on the PFFN workload.)
  static constexpr int NQ = D >= 128 ? 2 : GDPA_FWD_NQ;
  // K/V ring: 128 KB of stages for D = 128 (2 of 128 keys or 4 of 64), 64 KB
  // for smaller D, at most 8
  static constexpr int KV_RING = (D >= 128 ? 64 : 32) * 1024;
  static constexpr int NKV = KV_RING / KV_BYTES > 8 ? 8 : KV_RING / KV_BYTES;
  static constexpr int STAGE_WARP = 32 * 64;   // O staging: 32 rows x 64 B per epilogue warp
  static constexpr int OFF_Q = 0;                                // [NQ]
  static constexpr int OFF_K = OFF_Q + NQ * Q_BYTES;             // [NKV]
  static constexpr int OFF_V = OFF_K + NKV * KV_BYTES;           // [NKV]
  static constexpr int OFF_STAGE = OFF_V + NKV * KV_BYTES;       // [8 epilogue warps]
  static constexpr int OFF_INV = OFF_STAGE + 8 * STAGE_WARP;     // float [2 slots][2][BM]
  static constexpr int OFF_BIAS = OFF_INV + 2 * 2 * BM * 4;      // float [2 slots][2][BN]
  static constexpr int OFF_KVCNT = OFF_BIAS + 2 * 2 * BN * 4;    // int [4][8]
  // tile records, producer -> other roles: a ring of NT (even, so a ring
  // entry always holds tiles of the same slot)
  static constexpr int NT = 16;
  static constexpr int OFF_TREC = OFF_KVCNT + 4 * 8 * 4;         // FTile [NT]
  static constexpr int OFF_BAR = OFF_TREC + NT * 64;
  // barrier indices (Q ring stage i: [i]; per slot s: [s]; bias buffers of
  // slot s: [2s + b])
  static constexpr int B_QFULL = 0;
  static constexpr int B_QEMPTY = B_QFULL + NQ;
  static constexpr int B_KVFULL = B_QEMPTY + NQ;
  // K/V stage i released by MMA issuer j: [2i + j] (one issuer: j = 0 only)
  static constexpr int B_KVEMPTY = B_KVFULL + NKV;
  // S of a key block in halves (per-slot issuers): SFULL the half phi takes
  // first, SFULLB the other (one issuer: SFULL the whole block)
  static constexpr int B_SFULL = B_KVEMPTY + 2 * NKV;
  static constexpr int B_SFULLB = B_SFULL + 2;
  static constexpr int B_PFULL = B_SFULLB + 2;
  static constexpr int B_PVDONE = B_PFULL + 2;
  static constexpr int B_OFULL = B_PVDONE + 2;
  static constexpr int B_OEMPTY = B_OFULL + 2;
  static constexpr int B_BFULL = B_OEMPTY + 2;
  static constexpr int B_BEMPTY = B_BFULL + 4;
  // rotary: Q of slot s, K of ring stage i turned and ready for the MMA
  static constexpr int B_QROT = B_BEMPTY + 4;
  static constexpr int B_KROT = B_QROT + 2;
  // softmax row scales 1/l of a tile, phi -> epilogue (slot s, buffer b: [2s + b])
  static constexpr int B_LFULL = B_KROT + NKV;
  static constexpr int B_LEMPTY = B_LFULL + 4;
  // tile record ring entry i written / read by all its readers
  static constexpr int B_TFULL = B_LEMPTY + 4;
  static constexpr int B_TEMPTY = B_TFULL + NT;
  static constexpr int NBARS = B_TEMPTY + NT;
  static constexpr int OFF_MISC = OFF_BAR + NBARS * 8;  // tmem addr, abort flag
  static constexpr int SMEM_BYTES = OFF_MISC + 16;
  static constexpr int SMEM_ALLOC = SMEM_BYTES;  // base is 1024-aligned (checked at entry)
  // TMEM: slot s at column 256 s: S (then P over its first BN / 2 columns)
  // at +0, O at +BN.
  static constexpr int TMEM_SLOT = 256;
  static constexpr int TMEM_O = BN;
  static constexpr int TMEM_COLS = 512;
  static_assert(BN + D <= TMEM_SLOT, "TMEM slot");
  static_assert(NKV >= 2 && NKV <= 8, "K/V ring");
  static_assert(NQ >= 2 && NQ <= 8, "Q ring");
  static_assert(SMEM_ALLOC <= 232448, "shared memory budget");
  static_assert(Q_BYTES % 1024 == 0 && KV_BYTES % 1024 == 0, "align");
};

using Unit = GdpaUnit;

// A unit's problem: the table's in a grouped launch, else the inline one of a
// single-problem call (read from the kernel parameters).  Returned by value
// so only the fields a caller uses are loaded.
template <class C>
__device__ __forceinline__ FwdProblem fwd_problem(const FwdArgs& a, int p) {
  if constexpr (C::GROUPED) return a.probs[p];
  return a.p0;
}

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

// One query tile of the CTA's walk (64 bytes: the record the producer
// publishes to the other roles in shared memory).
struct __align__(16) FTile {
  int h, q0, Lq, k0;
  int Lk, m0, kb0, kb1;  // first local row; visible key blocks [kb0, kb1)
  int ntile;             // query tiles of the unit
  int prob;              // its problem (grouped launch; 0 otherwise)
  int slot;              // 0 or 1: tiles alternate between the two slots
  int resident;          // the unit's blocks are loaded once, at its first tile
  int unit_first;        // first tile of its unit
  int end;               // no tile: the walk is over
  uint32_t kv0;          // K/V ring index of block kb0 (the tile's blocks are consecutive)
  uint32_t qi;           // Q ring index: tiles with visible keys before this one
};
static_assert(sizeof(FTile) == 64, "tile record");

// The CTA's tiles in the order every role uses.  Units come from UnitStream
// (longest first, boustrophedon over the grid); K/V ring indices advance by
// the unit's block count at a resident unit's first tile and by the visible
// block count at every tile of a streamed unit.
template <class C>
struct TileWalk {
  const FwdArgs* args;
  UnitStreamT<C::GROUPED> units;
  Unit t;
  int wl, wr, ntile, mt, nkb;
  uint32_t g, kvi, unit_kv0, nq;
  bool resident, in_unit;
  __device__ explicit TileWalk(const FwdArgs& a)
      : args(&a), units(a.info, a.H, a.n_units, a.head_mask, a.eprob, a.probs), t{},
        wl(a.p0.wl), wr(a.p0.wr), ntile(0), mt(0), nkb(0), g(0), kvi(0), unit_kv0(0), nq(0),
        resident(false), in_unit(false) {}
  __device__ bool next(FTile& x) {
    for (;;) {
      if (!in_unit) {
        if (!units.next(t)) return false;
        if constexpr (C::GROUPED) {  // the band of this unit's problem
          wl = args->probs[t.prob].wl;
          wr = args->probs[t.prob].wr;
        }
        ntile = (t.Lq + kBlockM - 1) / kBlockM;
        nkb = (t.Lk + C::BN - 1) / C::BN;
        resident = wl < 0 && wr < 0 && nkb > 0 && nkb <= C::NKV;
        unit_kv0 = kvi;
        if (resident && ntile > 0) kvi += nkb;
        mt = 0;
        in_unit = true;
      }
      if (mt >= ntile) {
        in_unit = false;
        continue;
      }
      x.h = t.h;
      x.q0 = t.q0;
      x.Lq = t.Lq;
      x.k0 = t.k0;
      x.Lk = t.Lk;
      x.m0 = mt * kBlockM;
      kv_range<C::BN>(x.m0, t.Lk, wl, wr, x.kb0, x.kb1);
      x.ntile = ntile;
      x.resident = resident ? 1 : 0;
      x.unit_first = mt == 0 ? 1 : 0;
      x.end = 0;
      if (resident) {
        x.kv0 = unit_kv0 + x.kb0;
      } else {
        x.kv0 = kvi;
        if (x.kb1 > x.kb0) kvi += x.kb1 - x.kb0;
      }
      x.slot = (int)(g & 1);
      x.prob = t.prob;
      x.qi = nq;
      if (x.kb1 > x.kb0) ++nq;  // only tiles with keys load a Q tile
      ++g;
      ++mt;
      return true;
    }
  }
};

template <class C>
struct Smem {
  uint32_t base;  // shared address of the 1024-aligned base
  uint8_t* ptr;
  __device__ uint32_t q(int st) const { return base + C::OFF_Q + st * C::Q_BYTES; }
  __device__ uint32_t k(int st) const { return base + C::OFF_K + st * C::KV_BYTES; }
  __device__ uint32_t v(int st) const { return base + C::OFF_V + st * C::KV_BYTES; }
  // O staging of epilogue warp ew (0..7), row j (0..31), 16-byte chunk c of a
  // 64-byte row segment, chunks XOR-swizzled by row
  __device__ uint32_t stage(int ew, int j, int c) const {
    return base + C::OFF_STAGE + ew * C::STAGE_WARP + j * 64 + ((c ^ ((j >> 1) & 3)) << 4);
  }
  // softmax row scales 1/l of slot s, buffer b
  __device__ float* inv(int s, int b) const {
    return reinterpret_cast<float*>(ptr + C::OFF_INV) + (s * 2 + b) * C::BM;
  }
  __device__ float* bias(int s, int b) const {
    return reinterpret_cast<float*>(ptr + C::OFF_BIAS) + (s * 2 + b) * C::BN;
  }
  // issuer-private per stage: [0] ring index (+1) its count was set for,
  // [1] PVs still to read it
  __device__ int* kv_count(int i) const {
    return reinterpret_cast<int*>(ptr + C::OFF_KVCNT) + i * 8;
  }
  // per stage: the ring index the producer is loading into it
  __device__ volatile int* kv_tag() const {
    return reinterpret_cast<volatile int*>(ptr + C::OFF_KVCNT) + 2 * 8;
  }
  // per Q ring stage: the Q ring index the producer is loading into it
  __device__ volatile int* q_tag() const {
    return reinterpret_cast<volatile int*>(ptr + C::OFF_KVCNT) + 3 * 8;
  }
  __device__ uint32_t trec(int i) const { return base + C::OFF_TREC + i * 64; }
  __device__ uint32_t bar(int i) const { return base + C::OFF_BAR + i * 8; }
  __device__ uint32_t* tmem_slot() const { return reinterpret_cast<uint32_t*>(ptr + C::OFF_MISC); }
  __device__ volatile int* abort_flag() const {
    return reinterpret_cast<volatile int*>(ptr + C::OFF_MISC + 4);
  }
};

// Readers of tile record i (ring entry i % NT, of slot i % 2): the MMA
// issuer(s) (each reads every record), the slot's phi and epilogue warps, and
// the side warps (the bias warp, or both rotary warps; each reads every
// record).
template <class C>
__device__ __forceinline__ int trec_readers(const FwdArgs& a) {
  const int side = C::ROPE ? 2 : ((C::GROUPED || a.p0.bias_kind != 0) ? 1 : 0);
  return (C::DUAL ? 2 : 1) + 4 + 4 + side;
}

// Reader of the producer's tile records: records first, first + step, ... (a
// reader of one slot steps by 2).  Each record is copied out and released at
// once: by the calling thread, or, for a warp reading together (WARP), by
// lane 0 after the whole warp has copied it.
template <class C, bool WARP>
struct TileRing {
  uint32_t i;
  int step;
  __device__ TileRing(int first, int step_) : i((uint32_t)first), step(step_) {}
  __device__ __forceinline__ void take(const Smem<C>& sm, FTile& x) {
    const int e = (int)(i % C::NT);
    uint4* d = reinterpret_cast<uint4*>(&x);
#pragma unroll
    for (int k = 0; k < 4; ++k) d[k] = ld_shared_v4(sm.trec(e) + 16 * k);
    if (WARP) __syncwarp();
    if (!WARP || (threadIdx.x & 31) == 0) mbar_arrive(sm.bar(C::B_TEMPTY + e));
    i += (uint32_t)step;
  }
  // Blocking (bounded) read of the next record; false at the end of the walk
  // or when the wait gave up.
  __device__ bool next(const FwdArgs& a, const Smem<C>& sm, FTile& x) {
    const int e = (int)(i % C::NT);
    bool ok = mbar_wait(sm.bar(C::B_TFULL + e), (i / C::NT) & 1, sm.abort_flag(), a.status,
                        a.timeout_ns, 0x700 + e);
    if (WARP) ok = __all_sync(0xffffffffu, ok);
    if (!ok) return false;
    take(sm, x);
    return !x.end;
  }
  // Non-blocking: the next record, if the producer has written it.
  __device__ bool poll(const Smem<C>& sm, FTile& x) {
    const int e = (int)(i % C::NT);
    if (!mbar_test_wait(sm.bar(C::B_TFULL + e), (i / C::NT) & 1)) return false;
    take(sm, x);
    return true;
  }
};

// ------------------------------------------------------------------ producer
// Q of each tile into its slot's buffer; K/V blocks into the ring in ring-index
// order (a resident unit's blocks at its first tile, a streamed tile's visible
// blocks at the tile).  While a unit's blocks load, the next unit's first
// blocks are prefetched into L2.
template <class C>
__device__ void role_producer(const FwdArgs& a, const Smem<C>& sm, const CUtensorMap* tq,
                              const CUtensorMap* tk, const CUtensorMap* tv) {
  volatile int* abort = sm.abort_flag();
  const uint64_t pol_stream = l2_policy_evict_first();
  const uint64_t pol_keep = l2_policy_evict_last();
  bool dropped = false;
  TileWalk<C> walk(a);
  FTile x{};
  // a grouped launch keeps each problem's Q, K, V maps in device memory
  auto map_of = [&](int prob, int which) -> const CUtensorMap* {
    if constexpr (C::GROUPED) return a.maps + 4 * prob + which;
    return which == 0 ? tq : which == 1 ? tk : tv;
  };
  auto load_kv = [&](uint32_t ring, int kb) -> bool {
    const int st = (int)(ring % C::NKV);
    for (int j = 0; j < (C::DUAL ? 2 : 1); ++j)
      if (!mbar_wait(sm.bar(C::B_KVEMPTY + 2 * st + j), ((ring / C::NKV) & 1) ^ 1, abort,
                     a.status, a.timeout_ns, 0x000 + C::B_KVEMPTY + 2 * st + j))
        return false;
    sm.kv_tag()[st] = (int)ring;  // published by the arrive below (release)
    mbar_arrive_expect_tx(sm.bar(C::B_KVFULL + st), 2 * C::KV_BYTES);
    const CUtensorMap* mk = map_of(x.prob, 1);
    const CUtensorMap* mv = map_of(x.prob, 2);
    for (int pnl = 0; pnl < C::NPANEL; ++pnl) {
      tma_load_3d(sm.k(st) + pnl * C::BN * C::PANEL_BYTES, mk, sm.bar(C::B_KVFULL + st),
                  pnl * C::PANEL_ELEMS, x.h, x.k0 + kb * C::BN, pol_keep);
      tma_load_3d(sm.v(st) + pnl * C::BN * C::PANEL_BYTES, mv, sm.bar(C::B_KVFULL + st),
                  pnl * C::PANEL_ELEMS, x.h, x.k0 + kb * C::BN, pol_keep);
    }
    return true;
  };
  // publish tile record g to the other roles (the ring entry is free once
  // every reader of its previous record has copied it)
  uint32_t g = 0;
  auto publish = [&](const FTile& t) -> bool {
    const int e = (int)(g % C::NT);
    if (!mbar_wait(sm.bar(C::B_TEMPTY + e), ((g / C::NT) & 1) ^ 1, abort, a.status,
                   a.timeout_ns, 0x000 + C::B_TEMPTY + e))
      return false;
    const uint4* src = reinterpret_cast<const uint4*>(&t);
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const uint4 v = src[k];
      st_shared_v4(sm.trec(e) + 16 * k, v.x, v.y, v.z, v.w);
    }
    mbar_arrive(sm.bar(C::B_TFULL + e));  // release: the record is visible to the waiters
    ++g;
    return true;
  };
  while (walk.next(x)) {
    if (!publish(x)) return;
    if (x.kb1 <= x.kb0) continue;  // no visible keys: the epilogue warpgroup writes zeros
    const int qs = (int)(x.qi % C::NQ);
    if (!mbar_wait(sm.bar(C::B_QEMPTY + qs), ((x.qi / C::NQ) & 1) ^ 1, abort, a.status,
                   a.timeout_ns, 0x000 + C::B_QEMPTY + qs))
      return;
    sm.q_tag()[qs] = (int)x.qi;  // published by the arrive below (release)
    if ((a.debug_flags & 1) && !dropped && blockIdx.x == 0) {
      dropped = true;  // test hook: this Q tile is never loaded
    } else {
      mbar_arrive_expect_tx(sm.bar(C::B_QFULL + qs), C::Q_BYTES);
      const CUtensorMap* mq = map_of(x.prob, 0);
      for (int pnl = 0; pnl < C::NPANEL; ++pnl)
        tma_load_3d(sm.q(qs) + pnl * kBlockM * C::PANEL_BYTES, mq, sm.bar(C::B_QFULL + qs),
                    pnl * C::PANEL_ELEMS, x.h, x.q0 + x.m0, pol_stream);
    }
    if (x.resident && !x.unit_first) continue;  // the unit's blocks are in the ring
    if (x.unit_first) {
      // warm L2 with the next unit's first blocks (its loads wait for ring stages)
      Unit nt;
      if (walk.units.peek(nt)) {
        const int nb = min((nt.Lk + C::BN - 1) / C::BN, 2);
        const CUtensorMap* mk = map_of(nt.prob, 1);
        const CUtensorMap* mv = map_of(nt.prob, 2);
        for (int j = 0; j < nb; ++j)
          for (int pnl = 0; pnl < C::NPANEL; ++pnl) {
            tma_prefetch_l2_3d(mk, pnl * C::PANEL_ELEMS, nt.h, nt.k0 + j * C::BN, pol_keep);
            tma_prefetch_l2_3d(mv, pnl * C::PANEL_ELEMS, nt.h, nt.k0 + j * C::BN, pol_keep);
          }
      }
    }
    for (int kb = x.kb0; kb < x.kb1; ++kb)
      if (!load_kv(x.kv0 + (uint32_t)(kb - x.kb0), kb)) return;
  }
  // one end record per slot
  FTile last{};
  last.end = 1;
  if (publish(last)) publish(last);
}

// ------------------------------------------------------------------ MMA issuers
// One issuer for both slots (the rotary kernels, whose warps 2-3 turn Q and
// K).  Per slot: S of block i goes once the slot's previous PV has completed
// (P lives in the S columns); PV of block i goes once the phi warpgroup has
// written P (and, for the tile's first block, the epilogue has read the
// previous O).  The issuer polls both slots without blocking and issues
// whatever is ready, so one slot's MMAs run while the other slot's phi works.
//
// A K/V stage is released when every PV that reads it has been issued: its
// use count (tiles of a resident unit, or 1) is set at its first use and
// counted down at each PV; the commit after the last covers all earlier MMAs.
template <class C>
__device__ void role_mma(const FwdArgs& a, const Smem<C>& sm, uint32_t tmem) {
  volatile int* abort = sm.abort_flag();
  constexpr uint32_t idesc_s = make_idesc_bf16(kBlockM, C::BN, 0, 0);
  constexpr uint32_t idesc_o = make_idesc_bf16(kBlockM, C::D, 0, 1);
  constexpr uint32_t SBO = 8 * C::PANEL_BYTES;
  // Base descriptors of Q slot 0, K and V stage 0.  Every operand tile the
  // issuer names lies at a fixed offset from one of them, and the start
  // address field (address >> 4, 14 bits) cannot overflow below 256 KB of
  // shared memory, so an operand's descriptor is base + (offset >> 4).
  const uint64_t qdesc0 = make_smem_desc(sm.q(0), 16, SBO, C::LAYOUT);
  const uint64_t kdesc0 = make_smem_desc(sm.k(0), 16, SBO, C::LAYOUT);
  const uint64_t vdesc0 = make_smem_desc(sm.v(0), C::BN * C::PANEL_BYTES, SBO, C::LAYOUT);
  int* kv_ring = sm.kv_count(0);  // ring index a stage's count was set for (+1)
  int* kv_left = sm.kv_count(1);  // PVs still to read the stage
  for (int i = 0; i < C::NKV; ++i) {
    kv_ring[i] = 0;
    kv_left[i] = 0;
  }

  struct Slot {
    uint32_t qi;          // Q ring index of the tile
    uint32_t kv0;         // ring index of the tile's first block
    int nkv, ntile;       // blocks of the tile; tiles of its unit
    int resident;
    bool have, done;      // a tile in hand; the slot's walk is over
    int ns, npv;          // S and PV issued for the tile
    uint32_t pc, tq;      // PV and non-empty tile counts of the slot
  };
  Slot sl[2];
  // each slot's tiles from the producer's records (every other record); tiles
  // without visible keys are skipped.  Polled, never waited on: the producer
  // may itself wait for a Q stage that only the other slot's S MMA frees.
  TileRing<C, false> ring0(0, 2), ring1(1, 2);
  auto fetch = [&](Slot& z, TileRing<C, false>& rg) -> bool {
    FTile x;
    while (!z.have && !z.done && rg.poll(sm, x)) {
      if (x.end) {
        z.done = true;
      } else if (x.kb1 > x.kb0) {
        z.have = true;
        z.qi = x.qi;
        z.kv0 = x.kv0;
        z.nkv = x.kb1 - x.kb0;
        z.ntile = x.ntile;
        z.resident = x.resident;
        z.ns = z.npv = 0;
        return true;
      }
    }
    return false;
  };
  for (int s = 0; s < 2; ++s) {
    sl[s].pc = sl[s].tq = 0;
    sl[s].have = sl[s].done = false;
  }

  uint64_t idle_since = 0;
  uint32_t idle_polls = 0;
  while (!(sl[0].done && sl[1].done)) {
    bool progress = false;
#pragma unroll
    for (int s = 0; s < 2; ++s) {
      Slot& z = sl[s];
      if (!z.have && !fetch(z, s == 0 ? ring0 : ring1)) continue;
      const uint32_t tslot = tmem + s * C::TMEM_SLOT;
      // ---- S = Q K^T of block ns
      if (z.ns < z.nkv && z.ns == z.npv) {
        const uint32_t ring = z.kv0 + (uint32_t)z.ns;
        const int st = (int)(ring % C::NKV);
        // Q and K are ready once loaded, or once turned when rotary (the
        // turning warps arrive per slot, in the slot's tile order).  Like a K/V
        // stage, a Q stage's full barrier identifies this tile's phase only
        // once the producer has started loading it.
        constexpr int KREADY = C::ROPE ? C::B_KROT : C::B_KVFULL;
        const int qst = (int)(z.qi % C::NQ);
        bool ok = z.ns > 0 ||
                  (C::ROPE ? mbar_test_wait(sm.bar(C::B_QROT + s), z.tq & 1)
                           : (sm.q_tag()[qst] == (int)z.qi &&
                              mbar_test_wait(sm.bar(C::B_QFULL + qst), (z.qi / C::NQ) & 1)));
        // The other slot may be far ahead or behind in the ring: the stage's
        // full barrier identifies this ring index's phase only once the
        // producer has started loading it (the previous content's phase done).
        ok = ok && sm.kv_tag()[st] == (int)ring;
        ok = ok && mbar_test_wait(sm.bar(KREADY + st), (ring / C::NKV) & 1);
        ok = ok && (z.pc == 0 || mbar_test_wait(sm.bar(C::B_PVDONE + s), (z.pc - 1) & 1));
        if (ok) {
          tc_fence_after();
          const uint64_t qd = qdesc0 + (uint64_t)((qst * C::Q_BYTES) >> 4);
          const uint64_t kd = kdesc0 + (uint64_t)((st * C::KV_BYTES) >> 4);
#pragma unroll
          for (int kk = 0; kk < C::D / 16; ++kk) {
            // K-major operands: 32 bytes per 16 elements within a 64-element
            // panel, then the next panel (offsets added to the start address field)
            const int pnl = kk * 16 / C::PANEL_ELEMS;
            const int within = (kk * 16 % C::PANEL_ELEMS) * 2;
            mma_bf16_ss(tslot, desc_add(qd, (pnl * kBlockM * C::PANEL_BYTES + within) >> 4),
                        desc_add(kd, (pnl * C::BN * C::PANEL_BYTES + within) >> 4), idesc_s,
                        kk > 0 ? 1u : 0u);
          }
          mma_commit(sm.bar(C::B_SFULL + s));
          if (z.ns == z.nkv - 1) mma_commit(sm.bar(C::B_QEMPTY + qst));
          ++z.ns;
          progress = true;
        }
      }
      // ---- O += P V of block npv
      if (z.npv < z.ns) {
        bool ok = mbar_test_wait(sm.bar(C::B_PFULL + s), z.pc & 1);
        ok = ok && (z.npv > 0 || mbar_test_wait(sm.bar(C::B_OEMPTY + s), (z.tq & 1) ^ 1));
        if (ok) {
          const uint32_t ring = z.kv0 + (uint32_t)z.npv;
          const int st = (int)(ring % C::NKV);
          tc_fence_after();
          const uint64_t vd = vdesc0 + (uint64_t)((st * C::KV_BYTES) >> 4);
#pragma unroll
          for (int kk = 0; kk < C::BN / 16; ++kk) {
            // A = P [128 x BN] from TMEM (bf16 pairs, 8 columns per 16 keys,
            // over the lower half of the S columns; the upper half for odd
            // blocks of the slot with 64-key blocks);
            // B = V [BN keys x D], N (= D) contiguous: MN-major, 16 keys per step
            mma_bf16_ts(tslot + C::TMEM_O,
                        tslot + ((C::ALT && (z.pc & 1)) ? C::BN / 2 : 0) + kk * 8,
                        desc_add(vd, (kk * 16 * C::PANEL_BYTES) >> 4), idesc_o,
                        (z.npv > 0 || kk > 0) ? 1u : 0u);
          }
          mma_commit(sm.bar(C::B_PVDONE + s));
          if (kv_ring[st] != (int)ring + 1) {
            kv_ring[st] = (int)ring + 1;
            kv_left[st] = z.resident ? z.ntile : 1;
          }
          if (--kv_left[st] == 0) mma_commit(sm.bar(C::B_KVEMPTY + 2 * st));
          ++z.npv;
          ++z.pc;
          if (z.npv == z.nkv) {
            mma_commit(sm.bar(C::B_OFULL + s));
            ++z.tq;
            z.have = false;
          }
          progress = true;
        }
      }
    }
    if (progress) {
      idle_since = 0;
      idle_polls = 0;
    } else if ((++idle_polls & 255u) == 0) {
      // nothing has been ready for a while: give up (bounded) if nothing moves.
      // The poll itself does not sleep: a sleeping issuer notices a finished
      // phi block or MMA only when it wakes, which stalls both slots.
      const uint64_t now = globaltimer_ns();
      if (idle_since == 0) idle_since = now;
      if (*abort) return;
      if (now - idle_since > a.timeout_ns) {
        *abort = 1;
        record_error(a.status, 5, 0x100);
        return;
      }
    }
  }
}

// One slot's MMA issuer (warp 1 for slot 0, warp 3 for slot 1).  S of a key
// block goes in two halves of BN/2 keys: phi writes block i's P over one half
// of the S columns (the lower half for even i, the upper for odd i) and reads
// the other half first in block i + 1.  So once block i's phi is done, the
// issuer sends S of block i + 1 into the half without P, then block i's PV,
// then the other half of S over block i's P (one thread's tcgen05.mma
// execute in issue order, so that half is written after the PV has read P):
// phi of block i + 1 starts after half an S, not after PV + S.  The issuer
// waits on its own slot's barriers only, so neither slot's MMAs wait for the
// other slot's events.
//
// Each issuer reads every tile record, to release K/V stages: a stage use
// (one ring index) is released by both issuers, each with a commit on its own
// barrier after its last PV that reads it, or, when none of its tiles reads
// it, as soon as the producer has taken the stage for it (a commit, which
// still follows the issuer's earlier MMAs).  A resident unit's stages are
// read by all its tiles, which alternate slots from the slot of its first
// tile.
template <class C>
__device__ void role_mma_slot(const FwdArgs& a, const Smem<C>& sm, uint32_t tmem, int s) {
  volatile int* abort = sm.abort_flag();
  constexpr uint32_t idesc_s = make_idesc_bf16(kBlockM, C::BN, 0, 0);
  constexpr uint32_t idesc_h = make_idesc_bf16(kBlockM, C::BN / 2, 0, 0);
  constexpr uint32_t idesc_o = make_idesc_bf16(kBlockM, C::D, 0, 1);
  constexpr uint32_t SBO = 8 * C::PANEL_BYTES;
  const uint64_t qdesc0 = make_smem_desc(sm.q(0), 16, SBO, C::LAYOUT);
  const uint64_t kdesc0 = make_smem_desc(sm.k(0), 16, SBO, C::LAYOUT);
  const uint64_t vdesc0 = make_smem_desc(sm.v(0), C::BN * C::PANEL_BYTES, SBO, C::LAYOUT);
  int* kv_left = sm.kv_count(s);  // this issuer's PVs still to read each stage
  for (int i = 0; i < C::NKV; ++i) kv_left[i] = 0;
  const uint32_t tslot = tmem + s * C::TMEM_SLOT;
  uint32_t pc = 0, tq = 0;  // PVs and tiles of the slot

#define MMA_WAIT(bar_, par_, where_)                                                    \
  do {                                                                                \
    if (!mbar_wait(sm.bar(bar_), (par_), abort, a.status, a.timeout_ns, where_)) return; \
  } while (0)
  // a stage's full barrier identifies this use's phase only once the producer
  // has started loading it (its tag names the use)
  auto wait_tag = [&](volatile int* tag, int want, int where) -> bool {
    if (*tag == want) return true;
    const uint64_t t0 = globaltimer_ns();
    while (*tag != want) {
      if (*abort) return false;
      if (globaltimer_ns() - t0 > a.timeout_ns) {
        *abort = 1;
        record_error(a.status, 5, where);
        return false;
      }
      __nanosleep(32);
    }
    return true;
  };

  // S = Q K^T into the slot's columns: all BN keys (h < 0), or half h (keys
  // [h BN/2, (h+1) BN/2) into columns [h BN/2, (h+1) BN/2))
  auto issue_s = [&](int qst, int st, int h) {
    const int h0 = h < 0 ? 0 : h;
    const uint64_t qd = qdesc0 + (uint64_t)((qst * C::Q_BYTES) >> 4);
    const uint64_t kd =
        kdesc0 + (uint64_t)((st * C::KV_BYTES + h0 * (C::BN / 2) * C::PANEL_BYTES) >> 4);
#pragma unroll
    for (int kk = 0; kk < C::D / 16; ++kk) {
      const int pnl = kk * 16 / C::PANEL_ELEMS;
      const int within = (kk * 16 % C::PANEL_ELEMS) * 2;
      mma_bf16_ss(tslot + h0 * (C::BN / 2),
                  desc_add(qd, (pnl * kBlockM * C::PANEL_BYTES + within) >> 4),
                  desc_add(kd, (pnl * C::BN * C::PANEL_BYTES + within) >> 4),
                  h < 0 ? idesc_s : idesc_h, kk > 0 ? 1u : 0u);
    }
  };
  // the block whose PV is still to be issued
  struct PendPV {
    bool valid, first, last, resident;
    int st, podd;  // its K/V stage; its P over the upper half of the S columns
    uint32_t use;  // its K/V ring index
  } pend{};
  // O += P V of that block (its P complete), then its releases
  auto issue_pv = [&](const PendPV& b) -> bool {
    if (b.first && !mbar_wait(sm.bar(C::B_OEMPTY + s), (tq & 1) ^ 1, abort, a.status,
                              a.timeout_ns, 0x100 + C::B_OEMPTY + s))
      return false;
    tc_fence_after();
    const uint64_t vd = vdesc0 + (uint64_t)((b.st * C::KV_BYTES) >> 4);
    const uint32_t pcol = tslot + (b.podd ? C::BN / 2 : 0);
#pragma unroll
    for (int kk = 0; kk < C::BN / 16; ++kk)
      mma_bf16_ts(tslot + C::TMEM_O, pcol + kk * 8,
                  desc_add(vd, (kk * 16 * C::PANEL_BYTES) >> 4), idesc_o,
                  (!b.first || kk > 0) ? 1u : 0u);
    mma_commit(sm.bar(C::B_PVDONE + s));
    if (!b.resident || --kv_left[b.st] == 0) mma_commit(sm.bar(C::B_KVEMPTY + 2 * b.st + s));
    if (b.last) {
      mma_commit(sm.bar(C::B_OFULL + s));
      ++tq;
    }
    return true;
  };
  // Waiting for K/V ring index u while the pending PV holds its stage: the
  // producer loads indices in order and cannot reach u past a reuse of that
  // stage (an index at least NKV beyond the pending one) before the PV has
  // released it, so issue the PV first.
  auto clear_for = [&](uint32_t u) -> bool {
    if (!pend.valid || (int)(u - pend.use) < C::NKV) return true;
    if (!mbar_wait(sm.bar(C::B_PFULL + s), (pc - 1) & 1, abort, a.status, a.timeout_ns,
                   0x100 + C::B_PFULL + s))
      return false;
    pend.valid = false;
    return issue_pv(pend);
  };

  TileRing<C, false> ring(0, 1);
  FTile x{};
  while (ring.next(a, sm, x)) {
    const int nb = x.kb1 - x.kb0;
    if (nb <= 0) continue;
    const bool mine = x.slot == s;
    if (!x.resident || x.unit_first) {
      // K/V stage uses that start at this tile: how many of this issuer's PVs
      // read each (a streamed tile's uses, possibly more than the ring's
      // stages, are each read by the tile's own PV, released right after it)
      const int n_mine = x.resident ? (x.ntile + (x.slot == s ? 1 : 0)) / 2 : (mine ? 1 : 0);
      for (int j = 0; j < nb && (x.resident || !mine); ++j) {
        const int st = (int)((x.kv0 + (uint32_t)j) % C::NKV);
        // the pending PV's count or release of this stage comes first
        if (!clear_for(x.kv0 + (uint32_t)j)) return;
        if (n_mine == 0) {
          // not before the producer has taken the stage for this use: a
          // release ahead of its wait would complete the phase it waits on
          // for the next use
          if (!wait_tag(sm.kv_tag() + st, (int)(x.kv0 + (uint32_t)j), 0x190 + st)) return;
          mma_commit(sm.bar(C::B_KVEMPTY + 2 * st + s));
        } else {
          kv_left[st] = n_mine;
        }
      }
    }
    if (!mine) continue;
    const int qst = (int)(x.qi % C::NQ);
    for (int idx = 0; idx < nb; ++idx) {
      const uint32_t ring_i = x.kv0 + (uint32_t)idx;
      const int st = (int)(ring_i % C::NKV);
      if (idx == 0) {
        if (!wait_tag(sm.q_tag() + qst, (int)x.qi, 0x180 + qst)) return;
        MMA_WAIT(C::B_QFULL + qst, (x.qi / C::NQ) & 1, 0x100 + C::B_QFULL + qst);
      }
      if (!clear_for(ring_i)) return;
      if (!wait_tag(sm.kv_tag() + st, (int)ring_i, 0x190 + st)) return;
      MMA_WAIT(C::B_KVFULL + st, (ring_i / C::NKV) & 1, 0x100 + C::B_KVFULL + st);
      if constexpr (!C::SPLIT) {
        // ---- S whole over the previous block's P: issued after that block's
        // PV by this thread, so it executes after the PV has read P (no wait
        // for the PV's completion); then PV once phi is done
        tc_fence_after();
        issue_s(qst, st, -1);
        mma_commit(sm.bar(C::B_SFULL + s));
        if (idx == nb - 1) mma_commit(sm.bar(C::B_QEMPTY + qst));
        MMA_WAIT(C::B_PFULL + s, pc & 1, 0x100 + C::B_PFULL + s);
        PendPV b{true, idx == 0, idx == nb - 1, x.resident != 0, st, 0, ring_i};
        if (!issue_pv(b)) return;
        ++pc;
        continue;
      }
      // ---- S of block pc, the half phi takes first: into the columns the
      // previous block's phi has read and not written (its P is over the
      // other half)
      if (pend.valid) MMA_WAIT(C::B_PFULL + s, (pc - 1) & 1, 0x100 + C::B_PFULL + s);
      tc_fence_after();
      const int first_half = (int)(pc & 1);  // odd blocks take the upper keys first
      issue_s(qst, st, first_half);
      mma_commit(sm.bar(C::B_SFULL + s));
      // ---- O += P V of the previous block
      if (pend.valid && !issue_pv(pend)) return;
      // ---- the other half of S, over the previous block's P: issued after
      // that block's PV, and one thread's tcgen05.mma execute in issue order
      issue_s(qst, st, first_half ^ 1);
      mma_commit(sm.bar(C::B_SFULLB + s));
      if (idx == nb - 1) mma_commit(sm.bar(C::B_QEMPTY + qst));
      pend.valid = true;
      pend.st = st;
      pend.first = idx == 0;
      pend.last = idx == nb - 1;
      pend.resident = x.resident != 0;
      pend.podd = (int)(pc & 1);
      pend.use = ring_i;
      ++pc;
    }
  }
  if (pend.valid) {
    MMA_WAIT(C::B_PFULL + s, (pc - 1) & 1, 0x100 + C::B_PFULL + s);
    issue_pv(pend);
  }
#undef MMA_WAIT
}

// ------------------------------------------------------------------ bias warp
// beta of each key block a tile sees, into its slot's 2-buffer ring, in tile
// order over both slots.
template <class C>
__device__ void role_bias(const FwdArgs& a, const Smem<C>& sm, bool softmax) {
  volatile int* abort = sm.abort_flag();
  const int lane = threadIdx.x & 31;
  uint32_t bcs[2] = {0u, 0u};
  TileRing<C, true> ring(0, 1);
  FTile x{};
  while (ring.next(a, sm, x)) {
    const FwdProblem P = fwd_problem<C>(a, x.prob);
    if (P.bias_kind == 0) continue;  // the phi warpgroup adds no bias for this tile
    const int s = x.slot;
    for (int j = x.kb0; j < x.kb1; ++j) {
      uint32_t& bc = bcs[s];
      const int bb = bc & 1;
      bool ok = mbar_wait(sm.bar(C::B_BEMPTY + 2 * s + bb), ((bc >> 1) & 1) ^ 1, abort, a.status,
                          a.timeout_ns, 0x300 + C::B_BEMPTY + 2 * s + bb);
      if (!__all_sync(0xffffffffu, ok)) return;
      float* dst = sm.bias(s, bb);
      const float* src = P.bias + (int64_t)x.h * P.total_kv + x.k0;
      for (int c = lane; c < C::BN; c += 32) {
        const int key = j * C::BN + c;
        float beta = 0.f;
        if (key < x.Lk) {
          const float g = src[key];
          if (P.bias_kind == 2) {
            // log sigma(g) = min(g, 0) - log(1 + exp(-|g|))
            beta = fminf(g, 0.f) - log1pf(__expf(-fabsf(g)));
          } else {
            beta = g;
          }
        }
        dst[c] = softmax ? beta * kLog2e : beta;
      }
      mbar_arrive(sm.bar(C::B_BFULL + 2 * s + bb));  // one arrival per lane, after its writes
      ++bc;
    }
  }
}

// ------------------------------------------------------------------ rotation warps
// Pair (x0, x1) of bf16 values turned by the angle whose (cos, sin) is the
// fp16 pair cs.
__device__ __forceinline__ uint32_t rotate_pair(uint32_t x, uint32_t cs) {
  const float x0 = __uint_as_float(x << 16), x1 = __uint_as_float(x & 0xffff0000u);
  const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&cs));
  return pack_bf16x2(fmaf(x0, f.x, -x1 * f.y), fmaf(x0, f.y, x1 * f.x));
}

// Rows [r0, min(r1, nvalid)) of a swizzled tile of `rows` rows turned in place
// by the table rows of tokens tok0 + row.  A lane takes 16-byte chunks (four
// pairs), two at a time (four spill under the control warps' register budget).
template <class C>
__device__ __forceinline__ void rotate_tile(uint32_t tile, int rows, int r0, int r1, int nvalid,
                                            const uint32_t* __restrict__ tab, int64_t tok0,
                                            int lane) {
  constexpr int CH = C::D / 8;              // chunks per row
  constexpr int CPP = C::PANEL_BYTES / 16;  // chunks per panel row
  const int n = (min(r1, nvalid) - r0) * CH;
  auto addr_of = [&](int it, int& row, int& ch) {
    row = r0 + it / CH;
    ch = it % CH;
    const int pnl = ch / CPP, cw = ch % CPP;
    const int swz = C::PANEL_BYTES == 128 ? (row & 7) : ((row >> 1) & 3);
    return tile + (uint32_t)(pnl * rows * C::PANEL_BYTES + row * C::PANEL_BYTES + ((cw ^ swz) << 4));
  };
  for (int base = 0; base < n; base += 64) {
    uint4 cs[2], x[2];
    uint32_t ad[2];
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const int it = base + u * 32 + lane;
      if (it < n) {
        int row, ch;
        ad[u] = addr_of(it, row, ch);
        cs[u] = __ldg(reinterpret_cast<const uint4*>(tab + (tok0 + row) * (C::D / 2) + ch * 4));
        x[u] = ld_shared_v4(ad[u]);
      }
    }
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      if (base + u * 32 + lane < n)
        st_shared_v4(ad[u], rotate_pair(x[u].x, cs[u].x), rotate_pair(x[u].y, cs[u].y),
                     rotate_pair(x[u].z, cs[u].z), rotate_pair(x[u].w, cs[u].w));
    }
  }
}

// Rotary temporal embedding (Kunlun paper review §2.2): warps 2 and 3 turn
// each Q tile, and each K block as it is loaded, in shared memory between the
// TMA load and the S MMA, in the producer's order; each warp takes half the
// rows.  The issuer waits for the turned tiles.  With a bias the same warps
// also write beta (both slots, in tile order, one block after its K block, so
// every wait depends only on work already done).
template <class C>
__device__ void role_rotary(const FwdArgs& a, const Smem<C>& sm, bool softmax) {
  volatile int* abort = sm.abort_flag();
  const int w = (threadIdx.x >> 5) - 2;  // 0 or 1
  const int lane = threadIdx.x & 31;
  const bool has_bias = a.p0.bias_kind != 0;
  uint32_t bc[2] = {0u, 0u};
  TileRing<C, true> ring(0, 1);
  FTile x{};
#define ROT_WAIT(bar_, par_, where_)                                                   \
  do {                                                                               \
    bool ok_ = mbar_wait(sm.bar(bar_), (par_), abort, a.status, a.timeout_ns, where_); \
    if (!__all_sync(0xffffffffu, ok_)) return;                                       \
  } while (0)
  while (ring.next(a, sm, x)) {
    if (x.kb1 <= x.kb0) continue;  // nothing loaded: the epilogue warpgroup writes zeros
    const int s = x.slot;
    // tiles are turned in load order, so this wait identifies the tile's phase
    const int qs = (int)(x.qi % C::NQ);
    ROT_WAIT(C::B_QFULL + qs, (x.qi / C::NQ) & 1, 0x500 + C::B_QFULL + qs);
    rotate_tile<C>(sm.q(qs), kBlockM, w * (kBlockM / 2), (w + 1) * (kBlockM / 2), x.Lq - x.m0,
                   a.rope_q, (int64_t)x.q0 + x.m0, lane);
    fence_proxy_async_smem();  // the MMA reads the turned tile through the async proxy
    mbar_arrive(sm.bar(C::B_QROT + s));
    const bool loads = !(x.resident && !x.unit_first);
    for (int kb = x.kb0; kb < x.kb1; ++kb) {
      if (loads) {
        const uint32_t ring = x.kv0 + (uint32_t)(kb - x.kb0);
        const int st = (int)(ring % C::NKV);
        ROT_WAIT(C::B_KVFULL + st, (ring / C::NKV) & 1, 0x500 + C::B_KVFULL + st);
        rotate_tile<C>(sm.k(st), C::BN, w * (C::BN / 2), (w + 1) * (C::BN / 2),
                       x.Lk - kb * C::BN, a.rope_kv, (int64_t)x.k0 + kb * C::BN, lane);
        fence_proxy_async_smem();
        mbar_arrive(sm.bar(C::B_KROT + st));
      }
      if (has_bias) {
        const int bb = bc[s] & 1;
        ROT_WAIT(C::B_BEMPTY + 2 * s + bb, ((bc[s] >> 1) & 1) ^ 1, 0x500 + C::B_BEMPTY + 2 * s + bb);
        float* dst = sm.bias(s, bb);
        const float* src = a.p0.bias + (int64_t)x.h * a.p0.total_kv + x.k0;
        for (int c = w * 32 + lane; c < C::BN; c += 64) {
          const int key = kb * C::BN + c;
          float beta = 0.f;
          if (key < x.Lk) {
            const float g = src[key];
            beta = a.p0.bias_kind == 2 ? fminf(g, 0.f) - log1pf(__expf(-fabsf(g))) : g;
          }
          dst[c] = softmax ? beta * kLog2e : beta;
        }
        mbar_arrive(sm.bar(C::B_BFULL + 2 * s + bb));
        ++bc[s];
      }
    }
  }
#undef ROT_WAIT
}

// ------------------------------------------------------------------ phi warpgroups
// One warpgroup per slot; thread r owns row r of the slot's tiles.  Per key
// block: x = scale s + beta from the S columns, P = phi(x) written back over
// them as bf16 pairs (softmax: the block's row maximum first, O rescaled when
// it grows).  At the end of a softmax tile the row's 1/l goes to the slot's
// epilogue warpgroup through shared memory, and the LSE row is written here.
template <class C, bool SOFTMAX>
__device__ void role_phi(const FwdArgs& a, const Smem<C>& sm, uint32_t tmem, int s) {
  volatile int* abort = sm.abort_flag();
  const int warp = threadIdx.x >> 5;
  const int wq = warp & 3;                  // TMEM lane quarter of this warp
  const int lane = threadIdx.x & 31;
  const int r = wq * 32 + lane;             // row of the tile owned by this thread
  const uint32_t tslot = tmem + ((uint32_t)(wq * 32) << 16) + s * C::TMEM_SLOT;
  uint32_t nsb = 0, bc = 0, lt = 0;  // S blocks, bias blocks, softmax tiles of the slot

#define PHI_WAIT(bar_, par_, where_)                                                   \
  do {                                                                               \
    bool ok_ = mbar_wait(sm.bar(bar_), (par_), abort, a.status, a.timeout_ns, where_); \
    if (!__all_sync(0xffffffffu, ok_)) return;                                       \
  } while (0)

  TileRing<C, true> ring(s, 2);
  FTile x{};
  while (ring.next(a, sm, x)) {
    const int nkv = x.kb1 - x.kb0;
    if (nkv <= 0) continue;  // no visible keys: the epilogue warpgroup writes the tile
    // this tile's problem: scale, activation, bias and band
    const FwdProblem P = fwd_problem<C>(a, x.prob);
    const int wl = P.wl, wr = P.wr;
    const bool has_bias = P.bias_kind != 0;
    const bool identity = P.phi == 2;
    const bool gelu = P.phi == 3;
    const float sc = SOFTMAX ? P.scale * kLog2e : P.scale;
    const int row = x.m0 + r;
    // visible keys of this row: [lo, hi]
    const int lo = wl >= 0 ? row - wl : INT_MIN;
    const int hi = min(x.Lk - 1, wr >= 0 ? row + wr : INT_MAX);
    float m_run = -INFINITY, l_run = 0.f;
    for (int idx = 0; idx < nkv; ++idx) {
      const int kbase = (x.kb0 + idx) * C::BN;
      const int bb = bc & 1;
      if (has_bias) PHI_WAIT(C::B_BFULL + 2 * s + bb, (bc >> 1) & 1, 0x400 + C::B_BFULL + 2 * s + bb);
      PHI_WAIT(C::B_SFULL + s, nsb & 1, 0x400 + C::B_SFULL + s);
      tc_fence_after();
      const float2* bias2 = reinterpret_cast<const float2*>(sm.bias(s, bb));
      // visible columns of this block: [clo, chi] (no shift of an unbounded side)
      const int clo = wl >= 0 ? lo - kbase : INT_MIN;
      const int chi = hi - kbase;  // hi <= Lk - 1 always
      const bool full = clo <= 0 && chi >= C::BN - 1;
      const uint64_t sc2 = f2_pack(sc, sc);
      // scores of 32 columns starting at c0: x = scale * s + beta (masked
      // columns: -inf for softmax, 0 otherwise), two columns per instruction
      auto scores = [&](int c0, uint32_t (&v)[32]) {
        tmem_ld32(tslot + c0, v);
        tmem_wait_ld();
#pragma unroll
        for (int e = 0; e < 32; e += 2) {
          uint64_t x2 = f2_pack(__uint_as_float(v[e]), __uint_as_float(v[e + 1]));
          if (has_bias) {
            const float2 bv = bias2[(c0 + e) >> 1];
            x2 = f2_fma(x2, sc2, f2_pack(bv.x, bv.y));
          } else {
            x2 = f2_mul(x2, sc2);
          }
          float x0, x1;
          f2_unpack(x2, x0, x1);
          v[e] = __float_as_uint(x0);
          v[e + 1] = __float_as_uint(x1);
        }
        if (!full) {  // band edges and the ragged last key block
          const float fill = SOFTMAX ? -INFINITY : 0.f;
#pragma unroll
          for (int e = 0; e < 32; ++e)
            if (c0 + e < clo || c0 + e > chi) v[e] = __float_as_uint(fill);
        }
      };
      // Softmax in one pass: a chunk's P is taken against the running row
      // maximum m_run while the chunk's maximum stays within kRescaleThreshold
      // of it (so P <= 2^threshold).  A chunk that goes beyond moves m_run up
      // to its maximum and scales by 2^(m_old - m_new) what was taken against
      // the old value: the block's P chunks already in TMEM, the block's
      // partial sums and l, and O (at the end of the block).
      bool need_rescale = false;  // this row's O needs `factor` (not the tile's first block)
      float factor = 1.f;
      const uint64_t half2 = f2_pack(0.5f, 0.5f);
      uint64_t ps2[2] = {0ull, 0ull};  // packed partial sums (softmax)
      // P = phi(x), 32 columns at a time, written back as bf16 pairs over one
      // half of the S columns.  Blocks take the chunks in ascending order and
      // write chunk ci's pairs to columns [16 ci, 16 ci + 16), except odd
      // blocks of the slot with 64-key blocks (ALT), which take them in
      // descending order and write them to BN/2 + [16 ci, 16 ci + 16).  Either
      // way a chunk's pairs land on S columns of chunks already read.  With a
      // split S (per-slot issuers, 64-key blocks) S comes in two halves: the
      // one read first, then (SFULLB) the other.
      constexpr int NCH = C::BN / 32;
      const bool odd = C::ALT && (nsb & 1) != 0;
      const int pbase = odd ? C::BN / 2 : 0;
#pragma unroll 1
      for (int k = 0; k < NCH; ++k) {
        const int ci = odd ? NCH - 1 - k : k;
        const int c0 = ci * 32;
        if (C::SPLIT && k == NCH / 2) {
          PHI_WAIT(C::B_SFULLB + s, nsb & 1, 0x400 + C::B_SFULLB + s);
          tc_fence_after();
        }
        uint32_t v[32];
        scores(c0, v);
        if (SOFTMAX) {
          float pm[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
          for (int e = 0; e < 32; e += 2)
            pm[(e >> 1) & 3] = fmax3(pm[(e >> 1) & 3], __uint_as_float(v[e]),
                                     __uint_as_float(v[e + 1]));
          const float cm = fmax3(fmaxf(pm[0], pm[1]), pm[2], pm[3]);
          const bool grow = cm > m_run + kRescaleThreshold;
          if (__any_sync(0xffffffffu, grow)) {
            float f = 1.f;
            if (grow) {
              f = (m_run == -INFINITY) ? 0.f : ex2_approx(m_run - cm);
              m_run = cm;
              l_run *= f;
              factor *= f;
              need_rescale = idx > 0;
              const uint64_t f2 = f2_pack(f, f);
              ps2[0] = f2_mul(ps2[0], f2);
              ps2[1] = f2_mul(ps2[1], f2);
            }
            // the block's P pairs already written (k chunks)
            tmem_wait_st();
            const int wlo = odd ? C::BN / 2 + 16 * (NCH - k) : 0;
            const int whi = odd ? C::BN : 16 * k;
#pragma unroll 1
            for (int c = wlo; c < whi; c += 16) {
              uint32_t pr[16];
              tmem_ld16(tslot + c, pr);
              tmem_wait_ld();
#pragma unroll
              for (int e = 0; e < 16; ++e)
                pr[e] = pack_bf16x2(__uint_as_float(pr[e] << 16) * f,
                                    __uint_as_float(pr[e] & 0xffff0000u) * f);
              tmem_st16(tslot + c, pr);
            }
          }
          const float m_use = (m_run == -INFINITY) ? 0.f : m_run;
          const uint64_t neg_m2 = f2_pack(-m_use, -m_use);
#pragma unroll
          for (int e = 0; e < 32; e += 2) {
            const uint64_t d2 =
                f2_add(f2_pack(__uint_as_float(v[e]), __uint_as_float(v[e + 1])), neg_m2);
            float d0, d1;
            f2_unpack(d2, d0, d1);
            const float p0 = ex2_approx(d0), p1 = ex2_approx(d1);
            v[e] = __float_as_uint(p0);
            v[e + 1] = __float_as_uint(p1);
            ps2[(e >> 1) & 1] = f2_add(ps2[(e >> 1) & 1], f2_pack(p0, p1));
          }
        } else if (gelu) {
#pragma unroll
          for (int e = 0; e < 32; ++e) {
            // gelu(x) = x Phi(x), Phi from erf (masked columns: gelu(0) = 0)
            const float x = __uint_as_float(v[e]);
            v[e] = __float_as_uint(x * fmaf(0.5f, erff(x * kInvSqrt2), 0.5f));
          }
        } else if (!identity) {
#pragma unroll
          for (int e = 0; e < 32; e += 2) {
            // silu(x) = h + h tanh(h), h = x / 2 (masked columns: silu(0) = 0)
            const uint64_t h2 =
                f2_mul(f2_pack(__uint_as_float(v[e]), __uint_as_float(v[e + 1])), half2);
            float h0, h1;
            f2_unpack(h2, h0, h1);
            const uint64_t p2 = f2_fma(h2, f2_pack(tanh_approx(h0), tanh_approx(h1)), h2);
            float p0, p1;
            f2_unpack(p2, p0, p1);
            v[e] = __float_as_uint(p0);
            v[e + 1] = __float_as_uint(p1);
          }
        }
        uint32_t pk[16];
#pragma unroll
        for (int e = 0; e < 16; ++e)
          pk[e] = pack_bf16x2(__uint_as_float(v[2 * e]), __uint_as_float(v[2 * e + 1]));
        tmem_st16(tslot + pbase + ci * 16, pk);
      }
      if (has_bias) {
        mbar_arrive(sm.bar(C::B_BEMPTY + 2 * s + bb));
        ++bc;
      }
      if (SOFTMAX) {
        float s0, s1, s2, s3;
        f2_unpack(ps2[0], s0, s1);
        f2_unpack(ps2[1], s2, s3);
        l_run += (s0 + s1) + (s2 + s3);
      }
      if (SOFTMAX && idx > 0 && __any_sync(0xffffffffu, need_rescale)) {
        // O must hold every earlier PV of the tile before it is rescaled: the
        // commit of the previous block's PV covers all of them
        PHI_WAIT(C::B_PVDONE + s, (nsb - 1) & 1, 0x400 + C::B_PVDONE + s);
        tc_fence_after();
#pragma unroll 1
        for (int c = 0; c < C::D; c += 16) {
          uint32_t raw[16];
          tmem_ld16(tslot + C::TMEM_O + c, raw);
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 16; ++e) raw[e] = __float_as_uint(__uint_as_float(raw[e]) * factor);
          tmem_st16(tslot + C::TMEM_O + c, raw);
        }
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(sm.bar(C::B_PFULL + s));
      ++nsb;
    }
    if (SOFTMAX) {
      // 1/l of the row to the epilogue; the LSE row from here
      const int b = lt & 1;
      PHI_WAIT(C::B_LEMPTY + 2 * s + b, ((lt >> 1) & 1) ^ 1, 0x400 + C::B_LEMPTY + 2 * s + b);
      sm.inv(s, b)[r] = l_run > 0.f ? 1.f / l_run : 0.f;
      mbar_arrive(sm.bar(C::B_LFULL + 2 * s + b));
      ++lt;
      if (row < x.Lq && P.lse)
        P.lse[(int64_t)x.h * P.total_q + x.q0 + row] =
            l_run > 0.f ? (m_run + __log2f(l_run)) * kLn2 : -INFINITY;
    }
  }
#undef PHI_WAIT
}

// ------------------------------------------------------------------ epilogue warpgroups
// One warpgroup per slot: O of each tile from TMEM (released to the next
// tile's PV as soon as it is read), times 1/l for softmax, to bf16 in the
// warp's staging box in shared memory (32 rows x 32 columns, 64-byte
// swizzle), 32 columns per pass; a box whose 32 rows all lie in the sample
// goes out as one TMA store (the async proxy: no load-store unit traffic,
// which the other roles' shared-memory and barrier operations share), a
// ragged one as plain stores of its valid rows.  Tiles without visible keys
// get O = 0 (and LSE = -inf) here.  Each warp handles its 32 rows on its own.
template <class C, bool SOFTMAX>
__device__ void role_epilogue(const FwdArgs& a, const Smem<C>& sm, uint32_t tmem, int s,
                              const CUtensorMap* to) {
  volatile int* abort = sm.abort_flag();
  const int warp = threadIdx.x >> 5;
  const int wq = warp & 3;                  // TMEM lane quarter of this warp
  const int ew = warp - 12;                 // epilogue warp index: its staging slice
  const int lane = threadIdx.x & 31;
  const int r = wq * 32 + lane;
  const uint32_t tO = tmem + ((uint32_t)(wq * 32) << 16) + s * C::TMEM_SLOT + C::TMEM_O;
  uint32_t tq = 0, lt = 0;  // tiles with keys; softmax tiles (1/l buffers)

#define EPI_WAIT(bar_, par_, where_)                                                   \
  do {                                                                               \
    bool ok_ = mbar_wait(sm.bar(bar_), (par_), abort, a.status, a.timeout_ns, where_); \
    if (!__all_sync(0xffffffffu, ok_)) return;                                       \
  } while (0)

  TileRing<C, true> ring(s, 2);
  FTile x{};
  while (ring.next(a, sm, x)) {
    const FwdProblem P = fwd_problem<C>(a, x.prob);
    __nv_bfloat16* const out = P.o;
    const int Hp = P.H;
    const int row = x.m0 + r;
    if (x.kb1 <= x.kb0) {
      if (row < x.Lq) {
        __nv_bfloat16* orow = out + ((int64_t)(x.q0 + row) * Hp + x.h) * C::D;
        const uint4 z = make_uint4(0, 0, 0, 0);
        for (int c = 0; c < C::D; c += 8) *reinterpret_cast<uint4*>(orow + c) = z;
        if (SOFTMAX && P.lse) P.lse[(int64_t)x.h * P.total_q + x.q0 + row] = -INFINITY;
      }
      continue;
    }
    float inv = 1.f;
    if (SOFTMAX) {
      const int b = lt & 1;
      EPI_WAIT(C::B_LFULL + 2 * s + b, (lt >> 1) & 1, 0x600 + C::B_LFULL + 2 * s + b);
      inv = sm.inv(s, b)[r];
      mbar_arrive(sm.bar(C::B_LEMPTY + 2 * s + b));
      ++lt;
    }
    EPI_WAIT(C::B_OFULL + s, tq & 1, 0x600 + C::B_OFULL + s);
    tc_fence_after();
    const CUtensorMap* omap = C::GROUPED ? a.maps + 4 * x.prob + 3 : to;
    const int r0 = x.m0 + wq * 32;          // this warp's first row in the sample
    const bool boxed = r0 + 32 <= x.Lq;     // all 32 rows in the sample
    constexpr int NPASS = C::D / 32;
#pragma unroll 1
    for (int ps = 0; ps < NPASS; ++ps) {
      if (lane == 0) bulk_wait_read_all();  // the previous box has left the staging rows
      __syncwarp();
#pragma unroll
      for (int hf = 0; hf < 2; ++hf) {  // 16 columns per TMEM load
        uint32_t raw[16];
        tmem_ld16(tO + ps * 32 + hf * 16, raw);
        tmem_wait_ld();
        if (ps == NPASS - 1 && hf == 1) {  // O fully read: the slot's next tile may overwrite it
          tc_fence_before();
          mbar_arrive(sm.bar(C::B_OEMPTY + s));
        }
#pragma unroll
        for (int e = 0; e < 16; e += 8)
          st_shared_v4(sm.stage(ew, lane, hf * 2 + (e >> 3)),
                       pack_bf16x2(__uint_as_float(raw[e + 0]) * inv, __uint_as_float(raw[e + 1]) * inv),
                       pack_bf16x2(__uint_as_float(raw[e + 2]) * inv, __uint_as_float(raw[e + 3]) * inv),
                       pack_bf16x2(__uint_as_float(raw[e + 4]) * inv, __uint_as_float(raw[e + 5]) * inv),
                       pack_bf16x2(__uint_as_float(raw[e + 6]) * inv, __uint_as_float(raw[e + 7]) * inv));
      }
      if (boxed) {
        fence_proxy_async_smem();  // the staged rows, visible to the TMA engine
        __syncwarp();
        if (lane == 0) {
          tma_store_3d(omap, sm.stage(ew, 0, 0), ps * 32, x.h, x.q0 + r0);
          bulk_commit_group();
        }
      } else {
        __syncwarp();
#pragma unroll
        for (int it = 0; it < 4; ++it) {
          const int j = it * 8 + (lane >> 2), cc = lane & 3;  // row of this warp, chunk
          const uint4 v = ld_shared_v4(sm.stage(ew, j, cc));
          if (r0 + j < x.Lq)
            *reinterpret_cast<uint4*>(out + ((int64_t)(x.q0 + r0 + j) * Hp + x.h) * C::D +
                                      ps * 32 + cc * 8) = v;
        }
        __syncwarp();
      }
    }
    ++tq;
  }
  if (lane == 0) bulk_wait_all();  // every box written before the CTA ends
#undef EPI_WAIT
}

template <int D, int BN, bool SOFTMAX, bool GROUPED, bool ROPE>
__global__ void __launch_bounds__(kThreads, 1)
    gdpa_fwd_kernel(const __grid_constant__ FwdArgs a, const __grid_constant__ CUtensorMap tq,
                    const __grid_constant__ CUtensorMap tk, const __grid_constant__ CUtensorMap tv,
                    const __grid_constant__ CUtensorMap to) {
  using C = FwdCfg<D, BN, GROUPED, ROPE>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  Smem<C> sm;
  sm.base = smem_u32(smem_raw);
  sm.ptr = smem_raw;
  if (sm.base & 1023u) {  // swizzled TMA tiles need 1024-byte alignment
    griddep_wait();
    if (threadIdx.x == 0) record_error(a.status, 2, 0x7000);
    return;
  }
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int i = 0; i < C::NQ; ++i) {
      mbar_init(sm.bar(C::B_QFULL + i), 1);
      mbar_init(sm.bar(C::B_QEMPTY + i), 1);
      sm.q_tag()[i] = -1;
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(sm.bar(C::B_SFULL + s), 1);
      mbar_init(sm.bar(C::B_SFULLB + s), 1);
      mbar_init(sm.bar(C::B_PFULL + s), 128);
      mbar_init(sm.bar(C::B_PVDONE + s), 1);
      mbar_init(sm.bar(C::B_OFULL + s), 1);
      mbar_init(sm.bar(C::B_OEMPTY + s), 128);
    }
    for (int i = 0; i < C::NKV; ++i) {
      mbar_init(sm.bar(C::B_KVFULL + i), 1);
      mbar_init(sm.bar(C::B_KVEMPTY + 2 * i), 1);
      mbar_init(sm.bar(C::B_KVEMPTY + 2 * i + 1), 1);
    }
    for (int i = 0; i < 4; ++i) {
      mbar_init(sm.bar(C::B_BFULL + i), C::ROPE ? 64 : 32);  // rotary: both warps write beta
      mbar_init(sm.bar(C::B_BEMPTY + i), 128);
      mbar_init(sm.bar(C::B_LFULL + i), 128);
      mbar_init(sm.bar(C::B_LEMPTY + i), 128);
    }
    for (int i = 0; i < C::NT; ++i) {
      mbar_init(sm.bar(C::B_TFULL + i), 1);
      mbar_init(sm.bar(C::B_TEMPTY + i), trec_readers<C>(a));
    }
    if (C::ROPE) {
      for (int s = 0; s < 2; ++s) mbar_init(sm.bar(C::B_QROT + s), 64);
      for (int i = 0; i < C::NKV; ++i) mbar_init(sm.bar(C::B_KROT + i), 64);
    }
    for (int i = 0; i < 8; ++i) sm.kv_tag()[i] = -1;
    *sm.abort_flag() = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tq);
    tma_prefetch_desc(&tk);
    tma_prefetch_desc(&tv);
    tma_prefetch_desc(&to);
  }
  if (warp == 2) {
    tmem_alloc(smem_u32(sm.tmem_slot()), C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *sm.tmem_slot();
  // The set-up above touches only this CTA's own state, so it may overlap the
  // schedule kernel before it; everything below reads that kernel's results.
  griddep_wait();

  // Registers: the phi warpgroups take the most, the epilogue warpgroups the
  // fewest; each budget is set inside its own branch.
  if (warp < 4) {
    setmaxnreg_to<kRegsControl, kRegsLaunch>();
    if (warp == 0) {
      if (lane == 0) role_producer<C>(a, sm, &tq, &tk, &tv);
    } else if constexpr (C::ROPE) {
      if (warp == 1) {
        if (lane == 0) role_mma<C>(a, sm, tmem);
      } else {
        role_rotary<C>(a, sm, SOFTMAX);
      }
    } else if (warp == 1 || warp == 3) {
      if (lane == 0) role_mma_slot<C>(a, sm, tmem, warp >> 1);
    } else {
      // a grouped launch may mix problems with and without a bias
      if (C::GROUPED || a.p0.bias_kind != 0) role_bias<C>(a, sm, SOFTMAX);
    }
  } else if (warp < 12) {
    setmaxnreg_to<kRegsPhi, kRegsLaunch>();
    role_phi<C, SOFTMAX>(a, sm, tmem, (warp - 4) >> 2);
  } else {
    setmaxnreg_to<kRegsEpi, kRegsLaunch>();
    role_epilogue<C, SOFTMAX>(a, sm, tmem, (warp - 12) >> 2, &to);
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

template <int D, int BN, bool SOFTMAX, bool GROUPED, bool ROPE = false>
cudaError_t launch_one(const FwdArgs& a, const CUtensorMap& tq, const CUtensorMap& tk,
                       const CUtensorMap& tv, const CUtensorMap& to, int sms,
                       cudaStream_t stream) {
  using C = FwdCfg<D, BN, GROUPED, ROPE>;
  auto kern = gdpa_fwd_kernel<D, BN, SOFTMAX, GROUPED, ROPE>;
  // The per-build checks and the shared-memory attribute, once per device.
  static std::atomic<uint64_t> ready{0};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const uint64_t dev_bit = dev >= 0 && dev < 64 ? 1ull << dev : 0;
  if (!(ready.load(std::memory_order_acquire) & dev_bit)) {
    // when the roles' register budgets differ, the raising side's setmaxnreg
    // waits until the block's launch registers cover it: never launch a build
    // whose per-thread count would leave that wait unsatisfiable
    cudaFuncAttributes fa;
    e = cudaFuncGetAttributes(&fa, kern);
    if (e != cudaSuccess) return e;
    constexpr bool kSplit =
        kRegsControl != kRegsLaunch || kRegsPhi != kRegsLaunch || kRegsEpi != kRegsLaunch;
    if (kSplit && fa.numRegs * kThreads < 128 * kRegsControl + 256 * kRegsPhi + 256 * kRegsEpi)
      return cudaErrorInvalidValue;
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_ALLOC);
    if (e != cudaSuccess) return e;
    int per_sm = 0;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kThreads, C::SMEM_ALLOC);
    if (e != cudaSuccess) return e;
    // the kernel allocates all 512 TMEM columns: exactly one CTA per SM
    if (per_sm != 1) return cudaErrorInvalidConfiguration;
    ready.fetch_or(dev_bit, std::memory_order_acq_rel);
  }
  const int grid = std::max(1, std::min(a.n_units, sms));
  // programmatic stream serialization: the CTAs start their set-up while the
  // schedule kernel before them finishes (the kernel waits before reading it)
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = C::SMEM_ALLOC;
  cfg.stream = stream;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  e = cudaLaunchKernelEx(&cfg, kern, a, tq, tk, tv, to);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace

int forward_block_n(int D, int phi, int max_kv, int debug_flags) {
  (void)D;
  (void)phi;
  (void)debug_flags;
  return max_kv <= 64 ? 64 : 128;
}

cudaError_t launch_forward(const FwdArgs& a, int D, int block_n, const CUtensorMap& tq,
                           const CUtensorMap& tk, const CUtensorMap& tv, const CUtensorMap& to,
                           int sms, cudaStream_t stream) {
  const bool sm = a.phi == 1;
  const bool grouped = a.probs != nullptr;
  const bool rope = a.rope_q != nullptr;
  if (grouped && rope) return cudaErrorInvalidValue;
#define GDPA_FWD_CASE(D_, BN_)                                                         \
  if (D == D_ && block_n == BN_) {                                                     \
    if (grouped)                                                                       \
      return sm ? launch_one<D_, BN_, true, true>(a, tq, tk, tv, to, sms, stream)          \
                : launch_one<D_, BN_, false, true>(a, tq, tk, tv, to, sms, stream);        \
    if (rope)                                                                          \
      return sm ? launch_one<D_, BN_, true, false, true>(a, tq, tk, tv, to, sms, stream)   \
                : launch_one<D_, BN_, false, false, true>(a, tq, tk, tv, to, sms, stream); \
    return sm ? launch_one<D_, BN_, true, false>(a, tq, tk, tv, to, sms, stream)           \
              : launch_one<D_, BN_, false, false>(a, tq, tk, tv, to, sms, stream);         \
  }
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
