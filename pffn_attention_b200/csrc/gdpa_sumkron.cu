// gdpa_sumkron.cu -- fused SumKronLinear forward for sm_100a.
//
// Kunlun paper review §2.4 (HSP and SumKronLinear): the second stage of
// Hierarchical Seed Pooling maps the seed summaries X [B, S, D] to Y [B, T, D]
// with a rank-k sum of Kronecker products,
//     Y_b = sum_r A_r X_b W_r,   A_r [T x S], W_r [D x D],
// (k (S T + D^2) parameters).  Computed as two contractions per sample:
//     Z_b = A X_b           A = [A_1; ...; A_k]  (k T x S),  Z_b (k T x D)
//     Y_b = sum_r Z_b[r] W_r = [Z_b[1] ... Z_b[k]] [W_1; ...; W_k]
// The second one has only T rows per sample, so a CTA takes G = 128 / T
// samples at once: its rows (sample, t) fill one 128-row MMA tile.  Z never
// leaves the SM: each 128 x 64 block of Z_b (stage 1, tcgen05 into TMEM) is
// read back by the drain warps, rounded to bf16 and written into the shared
// A operand of stage 2, whose fp32 Y accumulator (128 x D) stays in TMEM for
// the whole group.
//
// Loop of a group, per M tile mt of A (R = 128 / T values of r) and 64-wide
// chunk dc of d:
//   stage 1  for each of the G samples: Z (128 x 64) = A[mt] (128 x S) X_b[:, dc]
//            (TMEM, two buffers), drained into A2[r_local] rows (sample, t)
//   stage 2  for each r of the tile: Y (128 x D) += A2[r_local] (128 x 64) W_r[dc rows]
//
// Shared memory: the 128-row tile of A stays resident for all samples and d
// chunks of its tile (S <= 256); X comes in 64 x 64 chunks, W in 16-row chunks
// through the deepest ring the rest of shared memory allows.
//
// Warp roles (224 threads): warp 0 TMA producer of A tiles and X chunks;
// warp 6 TMA producer of W chunks, so that W for the next stage 2
// streams in while stage 1 runs and the stage-1 ring never waits behind it;
// warp 1 TMEM allocator and MMA issuer (one thread); warps 2-5 drain Z and
// write the group's Y (one TMEM lane each: row (sample, t)).  Every wait is
// bounded; on expiry the kernel records GDPA_ERR_TIMEOUT in the workspace
// status and returns after its copies land.
#include <algorithm>

#include "gdpa_internal.h"

namespace gdpa {
namespace {

constexpr int kSkThreads = 224;

template <int D_, int T_>
struct SkCfg {
  static constexpr int D = D_;
  static constexpr int T = T_;
  static constexpr int G = 128 / T;       // samples per group
  static constexpr int R = 128 / T;       // values of r per 128-row tile of A
  static constexpr int NDC = D / 64;      // 64-wide chunks of d
  static constexpr int MAX_S = 256;
  static constexpr int A_PANEL = 128 * 64 * 2;   // A tile: 128 rows, 64 seeds per panel
  static constexpr int A_BYTES = MAX_S / 64 * A_PANEL;  // resident M tile of A (S <= 256)
  static constexpr int X_BYTES = 64 * 64 * 2;    // X chunk: 64 seeds x 64 d
  static constexpr int NX = 4;                   // stage-1 operand ring
  static constexpr int W_ROWS = kSumKronWRows;   // one K step of stage 2 (the W map's box)
  static constexpr int W_BYTES = W_ROWS * D * 2; // W chunk: 16 rows x D (NDC panels)
  static constexpr int A2_SUB = 128 * 64 * 2;    // one r: 128 rows x 64 K
  static constexpr int BUDGET = 227 * 1024 - 1024;  // dynamic shared memory, less barriers
  static constexpr int NW_FIT = (BUDGET - A_BYTES - NX * X_BYTES - R * A2_SUB) / W_BYTES;
  static constexpr int NW = NW_FIT > 8 ? 8 : NW_FIT;  // stage-2 operand ring
  static constexpr int OFF_A = 0;
  static constexpr int OFF_X = OFF_A + A_BYTES;
  static constexpr int OFF_W = OFF_X + NX * X_BYTES;
  static constexpr int OFF_A2 = OFF_W + NW * W_BYTES;
  static constexpr int OFF_BAR = OFF_A2 + R * A2_SUB;
  // barriers
  static constexpr int B_AFULL = 0, B_AEMPTY = 1;
  static constexpr int B_XFULL = 2, B_XEMPTY = B_XFULL + NX;
  static constexpr int B_WFULL = B_XEMPTY + NX, B_WEMPTY = B_WFULL + NW;
  static constexpr int B_ZFULL = B_WEMPTY + NW, B_ZEMPTY = B_ZFULL + 2;
  static constexpr int B_A2FULL = B_ZEMPTY + 2, B_A2EMPTY = B_A2FULL + 1;
  static constexpr int B_YFULL = B_A2EMPTY + 1, B_YEMPTY = B_YFULL + 1;
  static constexpr int NBARS = B_YEMPTY + 1;
  static constexpr int OFF_MISC = OFF_BAR + NBARS * 8;
  static constexpr int SMEM = OFF_MISC + 16;
  // TMEM: Y at columns [0, D), Z buffers at 384 and 448
  static constexpr int TM_Z = 384;
  static_assert(D % 64 == 0 && D <= 384, "D");
  static_assert(T == 32 || T == 64, "T");
  static_assert(SMEM <= 232448, "shared memory");
  static_assert(W_BYTES % 1024 == 0 && NW >= 2, "W ring");
};

struct SkArgs {
  DeviceStatus* status;
  __nv_bfloat16* y;
  int B, S, k;
  int n_groups;
  int debug_flags;
  uint64_t timeout_ns;
};

template <class C>
struct SkSmem {
  uint32_t base;
  uint8_t* ptr;
  __device__ uint32_t a(int panel) const { return base + C::OFF_A + panel * C::A_PANEL; }
  __device__ uint32_t x(int st) const { return base + C::OFF_X + st * C::X_BYTES; }
  __device__ uint32_t w(int st) const { return base + C::OFF_W + st * C::W_BYTES; }
  __device__ uint32_t a2(int rl) const { return base + C::OFF_A2 + rl * C::A2_SUB; }
  __device__ uint32_t bar(int i) const { return base + C::OFF_BAR + i * 8; }
  __device__ uint32_t* tmem_slot() const { return reinterpret_cast<uint32_t*>(ptr + C::OFF_MISC); }
  __device__ volatile int* abort_flag() const {
    return reinterpret_cast<volatile int*>(ptr + C::OFF_MISC + 4);
  }
};

#define SK_WAIT(bar_, par_, where_)                                                        \
  (mbar_wait(sm.bar(bar_), (par_), sm.abort_flag(), a.status, a.timeout_ns, (where_)))

// ------------------------------------------------------------------ producer
template <class C>
__device__ void sk_producer_xa(const SkArgs& a, const SkSmem<C>& sm, const CUtensorMap* ta,
                               const CUtensorMap* tx) {
  const uint64_t keep = l2_policy_evict_last();     // A: read by every CTA
  const uint64_t stream = l2_policy_evict_first();  // X: once per M tile of A
  const int MT = a.k * C::T / 128, NKC = a.S / 64;
  uint32_t xc = 0, ac = 0;
  for (int g = blockIdx.x; g < a.n_groups; g += gridDim.x)
    for (int mt = 0; mt < MT; ++mt, ++ac) {
      // the M tile of A, resident for every sample and d chunk of this tile
      if (!SK_WAIT(C::B_AEMPTY, (ac & 1) ^ 1, 0x020)) return;
      mbar_arrive_expect_tx(sm.bar(C::B_AFULL), NKC * C::A_PANEL);
      for (int kc = 0; kc < NKC; ++kc)
        tma_load_3d(sm.a(kc), ta, sm.bar(C::B_AFULL), kc * 64, mt * 128, 0, keep);
      for (int dc = 0; dc < C::NDC; ++dc)
        for (int bl = 0; bl < C::G; ++bl)
          for (int kc = 0; kc < NKC; ++kc, ++xc) {
            const int st = xc % C::NX;
            if (!SK_WAIT(C::B_XEMPTY + st, ((xc / C::NX) & 1) ^ 1, 0x000 + st)) return;
            // test hook: CTA 0's second X chunk is never loaded
            if ((a.debug_flags & 1) && blockIdx.x == 0 && xc == 1) continue;
            mbar_arrive_expect_tx(sm.bar(C::B_XFULL + st), C::X_BYTES);
            // samples past B read as zeros (their Y rows are not stored)
            tma_load_3d(sm.x(st), tx, sm.bar(C::B_XFULL + st), dc * 64, kc * 64,
                        g * C::G + bl, stream);
          }
    }
}

template <class C>
__device__ void sk_producer_w(const SkArgs& a, const SkSmem<C>& sm, const CUtensorMap* tw) {
  const uint64_t keep = l2_policy_evict_last();  // W: read by every CTA
  const int MT = a.k * C::T / 128;
  uint32_t wc = 0;
  for (int g = blockIdx.x; g < a.n_groups; g += gridDim.x) {
    for (int mt = 0; mt < MT; ++mt)
      for (int dc = 0; dc < C::NDC; ++dc) {
        for (int rl = 0; rl < C::R; ++rl)
          for (int h = 0; h < 64 / C::W_ROWS; ++h, ++wc) {
            const int st = wc % C::NW;
            if (!SK_WAIT(C::B_WEMPTY + st, ((wc / C::NW) & 1) ^ 1, 0x010 + st)) return;
            mbar_arrive_expect_tx(sm.bar(C::B_WFULL + st), C::W_BYTES);
            const int row = (mt * C::R + rl) * C::D + dc * 64 + h * C::W_ROWS;
            for (int p = 0; p < C::NDC; ++p)
              tma_load_3d(sm.w(st) + p * C::W_ROWS * 128, tw, sm.bar(C::B_WFULL + st), p * 64,
                          row, 0, keep);
          }
      }
  }
}

// ------------------------------------------------------------------ MMA issuer
template <class C>
__device__ void sk_mma(const SkArgs& a, const SkSmem<C>& sm, uint32_t tmem) {
  // stage 1: A chunk K-major (128 rows x 64 seeds, one 128-byte panel); X chunk
  // MN-major (64 seeds x 64 d: one panel, 16 seed rows per step)
  constexpr uint32_t id1 = make_idesc_bf16(128, 64, 0, 1);
  // stage 2: A2 K-major; W chunk MN-major, NDC panels of 64 columns, panel
  // stride 32 rows x 128 bytes; N split into MMAs of at most 256
  constexpr int N0 = C::D > 256 ? 256 : C::D;
  constexpr int N1 = C::D - N0;
  constexpr uint32_t id2a = make_idesc_bf16(128, N0, 0, 1);
  constexpr uint32_t id2b = make_idesc_bf16(128, N1 > 0 ? N1 : 16, 0, 1);
  const uint64_t adesc0 = make_smem_desc(sm.a(0), 16, 1024, LAYOUT_SW128);  // panel 0
  const uint64_t xdesc0 = make_smem_desc(sm.x(0), 64 * 128, 1024, LAYOUT_SW128);
  const uint64_t wdesc0 = make_smem_desc(sm.w(0), C::W_ROWS * 128, 1024, LAYOUT_SW128);
  const uint64_t a2desc0 = make_smem_desc(sm.a2(0), 16, 1024, LAYOUT_SW128);
  const int MT = a.k * C::T / 128, NKC = a.S / 64;
  uint32_t xc = 0, wc = 0, zc = 0, a2c = 0, gc = 0, ac = 0;
  for (int g = blockIdx.x; g < a.n_groups; g += gridDim.x, ++gc) {
    bool first = true;  // first stage-2 MMA of the group overwrites Y
    for (int mt = 0; mt < MT; ++mt, ++ac) {
      if (!SK_WAIT(C::B_AFULL, ac & 1, 0x140)) return;
      for (int dc = 0; dc < C::NDC; ++dc) {
        for (int bl = 0; bl < C::G; ++bl, ++zc) {
          const int zb = zc & 1;
          if (!SK_WAIT(C::B_ZEMPTY + zb, ((zc >> 1) & 1) ^ 1, 0x100 + zb)) return;
          tc_fence_after();
          const uint32_t zt = tmem + C::TM_Z + zb * 64;
          for (int kc = 0; kc < NKC; ++kc, ++xc) {
            const int st = xc % C::NX;
            if (!SK_WAIT(C::B_XFULL + st, (xc / C::NX) & 1, 0x110 + st)) return;
            tc_fence_after();
            const uint64_t ad = adesc0 + (uint64_t)((kc * C::A_PANEL) >> 4);
            const uint64_t xd = xdesc0 + (uint64_t)((st * C::X_BYTES) >> 4);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)  // 16 seeds: 32 bytes along A, 16 rows along X
              mma_bf16_ss(zt, desc_add(ad, (kk * 32) >> 4), desc_add(xd, (kk * 16 * 128) >> 4),
                          id1, (kc > 0 || kk > 0) ? 1u : 0u);
            mma_commit(sm.bar(C::B_XEMPTY + st));
          }
          mma_commit(sm.bar(C::B_ZFULL + zb));
          // the tile's last stage-1 MMA: A may be replaced once it completes
          if (dc == C::NDC - 1 && bl == C::G - 1) mma_commit(sm.bar(C::B_AEMPTY));
        }
        if (!SK_WAIT(C::B_A2FULL, a2c & 1, 0x120)) return;
        if (first && !SK_WAIT(C::B_YEMPTY, (gc & 1) ^ 1, 0x121)) return;
        tc_fence_after();
        for (int rl = 0; rl < C::R; ++rl)
          for (int h = 0; h < 64 / C::W_ROWS; ++h, ++wc) {
            const int st = wc % C::NW;
            if (!SK_WAIT(C::B_WFULL + st, (wc / C::NW) & 1, 0x130 + st)) return;
            tc_fence_after();
            const uint64_t wd = wdesc0 + (uint64_t)((st * C::W_BYTES) >> 4);
            const uint64_t a2d = a2desc0 + (uint64_t)((rl * C::A2_SUB) >> 4);
#pragma unroll
            for (int kk = 0; kk < C::W_ROWS / 16; ++kk) {
              // K step of 16: A2 columns h*32 + kk*16 (bytes 2x), W rows kk*16
              const uint64_t ak = desc_add(a2d, ((h * C::W_ROWS + kk * 16) * 2) >> 4);
              const uint64_t wk = desc_add(wd, (kk * 16 * 128) >> 4);
              const uint32_t acc = first ? 0u : 1u;
              mma_bf16_ss(tmem, ak, wk, id2a, acc);
              if (N1 > 0)
                mma_bf16_ss(tmem + N0, ak, desc_add(wk, (4 * C::W_ROWS * 128) >> 4), id2b, acc);
              first = false;
            }
            mma_commit(sm.bar(C::B_WEMPTY + st));
          }
        mma_commit(sm.bar(C::B_A2EMPTY));
        ++a2c;
      }
    }
    mma_commit(sm.bar(C::B_YFULL));
  }
}

// ------------------------------------------------------------------ drain / epilogue
template <class C>
__device__ void sk_drain(const SkArgs& a, const SkSmem<C>& sm, uint32_t tmem) {
  const int q = (threadIdx.x >> 5) & 3;      // TMEM lane quarter (warps 2..5 -> 2,3,0,1)
  const int lane = threadIdx.x & 31;
  const int L = q * 32 + lane;               // TMEM lane = row of Z tile / of A2 and Y
  const uint32_t lane_off = (uint32_t)(q * 32) << 16;
  const int rl = L / C::T, t = L % C::T;     // stage-1 row: (r within the tile, t)
  const int MT = a.k * C::T / 128;
  uint32_t zc = 0, a2c = 0, gc = 0;
#define DR_WAIT(bar_, par_, where_)                                                    \
  do {                                                                               \
    bool ok_ = SK_WAIT(bar_, par_, where_);                                          \
    if (!__all_sync(0xffffffffu, ok_)) return;                                       \
  } while (0)
  for (int g = blockIdx.x; g < a.n_groups; g += gridDim.x, ++gc) {
    for (int mt = 0; mt < MT; ++mt)
      for (int dc = 0; dc < C::NDC; ++dc, ++a2c) {
        DR_WAIT(C::B_A2EMPTY, (a2c & 1) ^ 1, 0x200);  // stage 2 of the last step read A2
        for (int bl = 0; bl < C::G; ++bl, ++zc) {
          const int zb = zc & 1;
          DR_WAIT(C::B_ZFULL + zb, (zc >> 1) & 1, 0x210 + zb);
          tc_fence_after();
          uint32_t v[64];
          tmem_ld32p(tmem + lane_off + C::TM_Z + zb * 64, v);
          tmem_ld32p(tmem + lane_off + C::TM_Z + zb * 64 + 32, v + 32);
          tmem_wait_ld();
          tc_fence_before();
          mbar_arrive(sm.bar(C::B_ZEMPTY + zb));
          // A2[rl] row (sample bl, t), 64 K values = 8 chunks of 16 bytes, swizzled
          const int row = bl * C::T + t;
          const uint32_t rbase = sm.a2(rl) + row * 128;
#pragma unroll
          for (int c = 0; c < 8; ++c)
            st_shared_v4(rbase + ((c ^ (row & 7)) << 4),
                         pack_bf16x2(__uint_as_float(v[8 * c + 0]), __uint_as_float(v[8 * c + 1])),
                         pack_bf16x2(__uint_as_float(v[8 * c + 2]), __uint_as_float(v[8 * c + 3])),
                         pack_bf16x2(__uint_as_float(v[8 * c + 4]), __uint_as_float(v[8 * c + 5])),
                         pack_bf16x2(__uint_as_float(v[8 * c + 6]), __uint_as_float(v[8 * c + 7])));
        }
        fence_proxy_async_smem();  // the MMA reads A2 through the async proxy
        mbar_arrive(sm.bar(C::B_A2FULL));
      }
    // the group's Y: lane L is row (sample L / T, t = L % T)
    DR_WAIT(C::B_YFULL, gc & 1, 0x220);
    tc_fence_after();
    const int b = g * C::G + L / C::T;
    __nv_bfloat16* yrow = a.y + ((int64_t)b * C::T + L % C::T) * C::D;
#pragma unroll 1
    for (int c0 = 0; c0 < C::D; c0 += 32) {
      uint32_t v[32];
      tmem_ld32(tmem + lane_off + c0, v);
      tmem_wait_ld();
      if (b < a.B) {
#pragma unroll
        for (int e = 0; e < 32; e += 8)
          *reinterpret_cast<uint4*>(yrow + c0 + e) =
              make_uint4(pack_bf16x2(__uint_as_float(v[e + 0]), __uint_as_float(v[e + 1])),
                         pack_bf16x2(__uint_as_float(v[e + 2]), __uint_as_float(v[e + 3])),
                         pack_bf16x2(__uint_as_float(v[e + 4]), __uint_as_float(v[e + 5])),
                         pack_bf16x2(__uint_as_float(v[e + 6]), __uint_as_float(v[e + 7])));
      }
    }
    tc_fence_before();
    mbar_arrive(sm.bar(C::B_YEMPTY));
  }
#undef DR_WAIT
}

template <int D, int T>
__global__ void __launch_bounds__(kSkThreads, 1)
    gdpa_sumkron_kernel(const __grid_constant__ SkArgs a, const __grid_constant__ CUtensorMap ta,
                        const __grid_constant__ CUtensorMap tx,
                        const __grid_constant__ CUtensorMap tw) {
  using C = SkCfg<D, T>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  SkSmem<C> sm;
  sm.base = smem_u32(smem_raw);
  sm.ptr = smem_raw;
  if (sm.base & 1023u) {
    if (threadIdx.x == 0) record_error(a.status, 2, 0x7000);
    return;
  }
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    mbar_init(sm.bar(C::B_AFULL), 1);
    mbar_init(sm.bar(C::B_AEMPTY), 1);
    for (int i = 0; i < C::NX; ++i) {
      mbar_init(sm.bar(C::B_XFULL + i), 1);
      mbar_init(sm.bar(C::B_XEMPTY + i), 1);
    }
    for (int i = 0; i < C::NW; ++i) {
      mbar_init(sm.bar(C::B_WFULL + i), 1);
      mbar_init(sm.bar(C::B_WEMPTY + i), 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(sm.bar(C::B_ZFULL + i), 1);
      mbar_init(sm.bar(C::B_ZEMPTY + i), 128);
    }
    mbar_init(sm.bar(C::B_A2FULL), 128);
    mbar_init(sm.bar(C::B_A2EMPTY), 1);
    mbar_init(sm.bar(C::B_YFULL), 1);
    mbar_init(sm.bar(C::B_YEMPTY), 128);
    *sm.abort_flag() = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&ta);
    tma_prefetch_desc(&tx);
    tma_prefetch_desc(&tw);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(sm.tmem_slot()), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *sm.tmem_slot();
  if (warp == 0) {
    if (lane == 0) sk_producer_xa<C>(a, sm, &ta, &tx);
  } else if (warp == 6) {
    if (lane == 0) sk_producer_w<C>(a, sm, &tw);
  } else if (warp == 1) {
    if (lane == 0) sk_mma<C>(a, sm, tmem);
  } else {
    sk_drain<C>(a, sm, tmem);
  }
  __syncwarp();
  tc_fence_before();
  __syncthreads();
  if (*sm.abort_flag()) {
    // a role gave up: let copies and MMAs already in flight land first
    if (threadIdx.x == 0) {
      const uint64_t t0 = globaltimer_ns();
      while (globaltimer_ns() - t0 < 2000000ull) __nanosleep(1000);
    }
    __syncthreads();
  }
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}
#undef SK_WAIT

template <int D, int T>
cudaError_t sk_launch(const SkArgs& a, const CUtensorMap& ta, const CUtensorMap& tx,
                      const CUtensorMap& tw, int sms, cudaStream_t s) {
  using C = SkCfg<D, T>;
  auto kern = gdpa_sumkron_kernel<D, T>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
  if (e != cudaSuccess) return e;
  int per_sm = 0;
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kSkThreads, C::SMEM);
  if (e != cudaSuccess) return e;
  if (per_sm != 1) return cudaErrorInvalidConfiguration;  // all 512 TMEM columns
  const int grid = std::max(1, std::min(a.n_groups, sms));
  kern<<<grid, kSkThreads, C::SMEM, s>>>(a, ta, tx, tw);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_sumkron(const SumKronLaunch& L, const CUtensorMap& ta, const CUtensorMap& tx,
                           const CUtensorMap& tw, int sms, cudaStream_t s) {
  SkArgs a{};
  a.status = L.status;
  a.y = L.y;
  a.B = L.B;
  a.S = L.S;
  a.k = L.k;
  a.debug_flags = L.debug_flags;
  a.n_groups = (L.B + (128 / L.T) - 1) / (128 / L.T);
  a.timeout_ns = L.timeout_ns;
  if (a.n_groups == 0) return cudaSuccess;
#define SK_CASE(D_, T_) \
  if (L.D == D_ && L.T == T_) return sk_launch<D_, T_>(a, ta, tx, tw, sms, s);
  SK_CASE(128, 32)
  SK_CASE(256, 32)
  SK_CASE(384, 32)
  SK_CASE(128, 64)
  SK_CASE(256, 64)
  SK_CASE(384, 64)
#undef SK_CASE
  return cudaErrorInvalidValue;
}

}  // namespace gdpa
