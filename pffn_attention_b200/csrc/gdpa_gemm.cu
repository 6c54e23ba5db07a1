// gdpa_gemm.cu -- batched bf16 GEMM on tcgen05, for the SumKronLinear
// backward (Kunlun paper review §2.4: its gradients are plain contractions;
// see gdpa_api.cu for which products they are).
//
// Persistent CTAs walk work units (output tile 128 x 128, split of the
// reduction batches, grid batch).  Per unit the K loop runs over the unit's
// reduction batches and, within each, over the batch's K chunks; A and B
// chunks come through a ring of shared memory stages by TMA (the ring runs on
// across units), the MMAs accumulate into one of two TMEM accumulators (128
// columns each), and the epilogue writes a unit's tile, as fp32 partial sums
// or as bf16 at the caller's layout, while the MMAs of the next unit go into
// the other accumulator.  Rows or columns past the operands' extents load as
// zeros, and output rows or columns past M, N are not written.
//
// Warp roles (256 threads): warp 0 TMA producer (one thread); warp 1 MMA
// issuer (one thread); warp 2 TMEM allocator; warps 4-7 epilogue, one TMEM
// lane (output row) per thread.  Every wait is bounded; on expiry the kernel
// records GDPA_ERR_TIMEOUT in the status block and returns after its copies
// land.
#include <algorithm>

#include "gdpa_internal.h"

namespace gdpa {
namespace {

constexpr int kGemmThreads = 256;
constexpr int kGemmStages = 4;
constexpr int kGemmTile = 128;

template <int KC>
struct GemmCfg {
  static constexpr int OP_BYTES = kGemmTile * KC * 2;  // one operand tile of a stage
  static constexpr int OFF_A = 0;
  static constexpr int OFF_B = OFF_A + kGemmStages * OP_BYTES;
  static constexpr int OFF_BAR = OFF_B + kGemmStages * OP_BYTES;
  // ring stages; accumulator a full (MMAs done) / empty (epilogue read it)
  static constexpr int B_FULL = 0, B_EMPTY = kGemmStages, B_ACCFULL = 2 * kGemmStages,
                       B_ACCEMPTY = 2 * kGemmStages + 2;
  static constexpr int NBARS = 2 * kGemmStages + 4;
  static constexpr int OFF_MISC = OFF_BAR + NBARS * 8;  // tmem addr, abort flag
  static constexpr int SMEM = OFF_MISC + 16;
  static_assert(OP_BYTES % 1024 == 0, "swizzle atoms");
};

// Coordinates of the box (or of panel p of an MN-major tile) for output tile
// t (along M for A, N for B), K chunk j of reduction batch rb, grid batch z.
__device__ __forceinline__ void operand_coords(const GemmOperand& o, int kc, int t, int p, int j,
                                               int rb, int z, int& c0, int& c1, int& c2) {
  if (o.mn_major) {
    c0 = t * kGemmTile + p * 64;
    c1 = j * kc + o.z_rows * z;
  } else {
    c0 = j * 64;
    c1 = t * kGemmTile + o.z_rows * z;
  }
  c2 = o.batch_of == 1 ? rb : (o.batch_of == 2 ? z : 0);
}

template <int KC>
__global__ void __launch_bounds__(kGemmThreads)
    gdpa_gemm_kernel(const __grid_constant__ GemmLaunch g, const __grid_constant__ CUtensorMap ta,
                     const __grid_constant__ CUtensorMap tb) {
  using C = GemmCfg<KC>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const uint32_t base = smem_u32(smem_raw);
  if (base & 1023u) {
    if (threadIdx.x == 0) record_error(g.status, 2, 0x7200);
    return;
  }
  auto bar = [&](int i) { return base + C::OFF_BAR + i * 8; };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem_raw + C::OFF_MISC);
  volatile int* abort = reinterpret_cast<volatile int*>(smem_raw + C::OFF_MISC + 4);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  const int mtiles = (g.M + kGemmTile - 1) / kGemmTile;
  const int ntiles = (g.N + kGemmTile - 1) / kGemmTile;
  const int tiles = mtiles * ntiles;
  const int64_t units = (int64_t)tiles * g.splits * g.Z;
  // unit u: tile u % tiles, split (u / tiles) % splits, grid batch u / (tiles splits)
  auto unit_of = [&](int64_t u, int& tm, int& tn, int& split, int& z, int& rb0, int& steps) {
    const int t = (int)(u % tiles);
    tm = t % mtiles;
    tn = t / mtiles;
    split = (int)((u / tiles) % g.splits);
    z = (int)(u / ((int64_t)tiles * g.splits));
    rb0 = (int)((int64_t)g.n_rb * split / g.splits);
    const int rb1 = (int)((int64_t)g.n_rb * (split + 1) / g.splits);
    steps = (rb1 - rb0) * g.nkc;
  };

  if (threadIdx.x == 0) {
    for (int i = 0; i < kGemmStages; ++i) {
      mbar_init(bar(C::B_FULL + i), 1);
      mbar_init(bar(C::B_EMPTY + i), 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(bar(C::B_ACCFULL + i), 1);
      mbar_init(bar(C::B_ACCEMPTY + i), 128);
    }
    *abort = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&ta);
    tma_prefetch_desc(&tb);
  }
  if (warp == 2) {
    tmem_alloc(smem_u32(tmem_slot), 256);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      // ---- producer: A and B chunks of every step of every unit into the ring
      const uint64_t pol = l2_policy_evict_last();
      uint32_t i = 0;  // ring steps so far
      bool ok = true;
      for (int64_t u = blockIdx.x; u < units && ok; u += gridDim.x) {
        int tm, tn, split, z, rb0, steps;
        unit_of(u, tm, tn, split, z, rb0, steps);
        for (int j = 0; j < steps; ++j, ++i) {
          const int st = (int)(i % kGemmStages);
          ok = mbar_wait(bar(C::B_EMPTY + st), ((i / kGemmStages) & 1) ^ 1, abort, g.status,
                         g.timeout_ns, 0x7000 + st);
          if (!ok) break;
          mbar_arrive_expect_tx(bar(C::B_FULL + st), 2 * C::OP_BYTES);
          const int rb = rb0 + j / g.nkc, kc = j % g.nkc;
          const uint32_t sa = base + C::OFF_A + st * C::OP_BYTES;
          const uint32_t sb = base + C::OFF_B + st * C::OP_BYTES;
          int c0, c1, c2;
          for (int p = 0; p < (g.a.mn_major ? 2 : 1); ++p) {
            operand_coords(g.a, KC, tm, p, kc, rb, z, c0, c1, c2);
            tma_load_3d(sa + p * (C::OP_BYTES / 2), &ta, bar(C::B_FULL + st), c0, c1, c2, pol);
          }
          for (int p = 0; p < (g.b.mn_major ? 2 : 1); ++p) {
            operand_coords(g.b, KC, tn, p, kc, rb, z, c0, c1, c2);
            tma_load_3d(sb + p * (C::OP_BYTES / 2), &tb, bar(C::B_FULL + st), c0, c1, c2, pol);
          }
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ---- MMA issuer: KC / 16 MMAs of K = 16 per step into the unit's accumulator
      const uint32_t idesc = make_idesc_bf16(kGemmTile, kGemmTile, g.a.mn_major, g.b.mn_major);
      // K-major tile: 128 rows x 128 bytes (one swizzle panel), 16 elements =
      // 32 bytes per K step; MN-major tile: two panels of 64 M (or N) x KC
      // rows, 16 rows = 2 KB per K step
      const uint32_t lbo = g.a.mn_major ? KC * 128 : 16;
      const uint32_t lbo_b = g.b.mn_major ? KC * 128 : 16;
      const uint32_t ka = g.a.mn_major ? (16 * 128) >> 4 : 32 >> 4;
      const uint32_t kb = g.b.mn_major ? (16 * 128) >> 4 : 32 >> 4;
      uint32_t i = 0, n = 0;  // ring steps; units with steps (accumulator uses)
      bool ok = true;
      for (int64_t u = blockIdx.x; u < units && ok; u += gridDim.x) {
        int tm, tn, split, z, rb0, steps;
        unit_of(u, tm, tn, split, z, rb0, steps);
        if (steps == 0) continue;
        const int acc = (int)(n & 1);
        // the epilogue has read this accumulator's previous unit
        ok = mbar_wait(bar(C::B_ACCEMPTY + acc), ((n >> 1) & 1) ^ 1, abort, g.status,
                       g.timeout_ns, 0x7140 + acc);
        if (!ok) break;
        tc_fence_after();
        const uint32_t tacc = tmem + acc * kGemmTile;
        for (int j = 0; j < steps; ++j, ++i) {
          const int st = (int)(i % kGemmStages);
          ok = mbar_wait(bar(C::B_FULL + st), (i / kGemmStages) & 1, abort, g.status,
                         g.timeout_ns, 0x7100 + st);
          if (!ok) break;
          tc_fence_after();
          const uint64_t da = make_smem_desc(base + C::OFF_A + st * C::OP_BYTES, lbo, 1024,
                                             LAYOUT_SW128);
          const uint64_t db = make_smem_desc(base + C::OFF_B + st * C::OP_BYTES, lbo_b, 1024,
                                             LAYOUT_SW128);
#pragma unroll
          for (int kk = 0; kk < KC / 16; ++kk)
            mma_bf16_ss(tacc, desc_add(da, kk * ka), desc_add(db, kk * kb), idesc,
                        (j > 0 || kk > 0) ? 1u : 0u);
          mma_commit(bar(C::B_EMPTY + st));
        }
        if (!ok) break;
        mma_commit(bar(C::B_ACCFULL + acc));  // after every MMA of the unit
        ++n;
      }
    }
  } else if (warp >= 4) {
    // ---- epilogue: thread = output row of each unit
    const int wq = warp & 3;
    uint32_t n = 0;
    bool ok = true;
    for (int64_t u = blockIdx.x; u < units && ok; u += gridDim.x) {
      int tm, tn, split, z, rb0, steps;
      unit_of(u, tm, tn, split, z, rb0, steps);
      const int m = tm * kGemmTile + wq * 32 + lane;
      const int acc = (int)(n & 1);
      if (steps > 0) {
        ok = mbar_wait(bar(C::B_ACCFULL + acc), (n >> 1) & 1, abort, g.status, g.timeout_ns,
                       0x7180 + acc);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
        tc_fence_after();
      }
      const uint32_t trow = tmem + ((uint32_t)(wq * 32) << 16) + acc * kGemmTile;
#pragma unroll 1
      for (int c0 = 0; c0 < kGemmTile; c0 += 32) {
        const int n0 = tn * kGemmTile + c0;
        if (n0 >= g.N) break;
        float v[32];
        if (steps > 0) {
          tmem_ld32f(trow + c0, v);
          tmem_wait_ld();
        } else {
#pragma unroll
          for (int e = 0; e < 32; ++e) v[e] = 0.f;
        }
        if (m >= g.M) continue;
        if (g.f32_out) {
          float* o = static_cast<float*>(g.out) +
                     (((int64_t)split * g.Z + z) * g.M + m) * (int64_t)g.N + n0;
#pragma unroll
          for (int e = 0; e < 32; e += 4)
            *reinterpret_cast<float4*>(o + e) = make_float4(v[e], v[e + 1], v[e + 2], v[e + 3]);
        } else {
          __nv_bfloat16* o = static_cast<__nv_bfloat16*>(g.out) + z * g.sZ +
                             (m / g.mT) * g.sMb + (m % g.mT) * g.sMt + (n0 / g.nD) * g.sNr +
                             n0 % g.nD;
#pragma unroll
          for (int e = 0; e < 32; e += 8)
            *reinterpret_cast<uint4*>(o + e) =
                make_uint4(pack_bf16x2(v[e], v[e + 1]), pack_bf16x2(v[e + 2], v[e + 3]),
                           pack_bf16x2(v[e + 4], v[e + 5]), pack_bf16x2(v[e + 6], v[e + 7]));
        }
      }
      if (steps > 0) {  // the accumulator may take a later unit
        tc_fence_before();
        mbar_arrive(bar(C::B_ACCEMPTY + acc));
        ++n;
      }
    }
  }
  __syncwarp();
  tc_fence_before();
  __syncthreads();
  if (*abort) {
    // a role gave up: let copies and MMAs already in flight land first
    if (threadIdx.x == 0) {
      const uint64_t t0 = globaltimer_ns();
      while (globaltimer_ns() - t0 < 2000000ull) __nanosleep(1000);
    }
    __syncthreads();
  }
  if (warp == 2) {
    tc_fence_after();
    tmem_dealloc(tmem, 256);
  }
}

__global__ void __launch_bounds__(256)
    gdpa_sum_splits_kernel(const float* __restrict__ part, int splits, int64_t count,
                           __nv_bfloat16* __restrict__ out) {
  const int64_t n8 = count / 8;
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n8;
       i += (int64_t)gridDim.x * blockDim.x) {
    float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    for (int s = 0; s < splits; ++s) {
      const float4* p = reinterpret_cast<const float4*>(part + s * count + i * 8);
      const float4 x = p[0], y = p[1];
      acc[0] += x.x; acc[1] += x.y; acc[2] += x.z; acc[3] += x.w;
      acc[4] += y.x; acc[5] += y.y; acc[6] += y.z; acc[7] += y.w;
    }
    reinterpret_cast<uint4*>(out)[i] =
        make_uint4(pack_bf16x2(acc[0], acc[1]), pack_bf16x2(acc[2], acc[3]),
                   pack_bf16x2(acc[4], acc[5]), pack_bf16x2(acc[6], acc[7]));
  }
}

template <int KC>
cudaError_t launch_kc(const GemmLaunch& g, const CUtensorMap& ta, const CUtensorMap& tb,
                      int sms, cudaStream_t s) {
  using C = GemmCfg<KC>;
  auto kern = gdpa_gemm_kernel<KC>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
  if (e != cudaSuccess) return e;
  const int64_t units = (int64_t)((g.M + kGemmTile - 1) / kGemmTile) *
                       ((g.N + kGemmTile - 1) / kGemmTile) * g.splits * g.Z;
  int per_sm = 0;
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kGemmThreads, C::SMEM);
  if (e != cudaSuccess) return e;
  per_sm = std::max(1, std::min(per_sm, 2));  // two 256-column TMEM allocations per SM
  const int grid = (int)std::min<int64_t>(units, (int64_t)sms * per_sm);
  kern<<<grid, kGemmThreads, C::SMEM, s>>>(g, ta, tb);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_gemm(const GemmLaunch& g, const CUtensorMap& ta, const CUtensorMap& tb,
                        int sms, cudaStream_t s) {
  if (g.M <= 0 || g.N <= 0 || g.Z <= 0 || g.splits <= 0 || g.n_rb < 0 || g.nkc <= 0)
    return cudaErrorInvalidValue;
  if (sms <= 0) return cudaErrorInvalidValue;
  if (g.kc == 64) return launch_kc<64>(g, ta, tb, sms, s);
  if (g.kc == 32 && g.a.mn_major && g.b.mn_major) return launch_kc<32>(g, ta, tb, sms, s);
  return cudaErrorInvalidValue;
}

cudaError_t launch_sum_splits(const float* part, int splits, int64_t count, __nv_bfloat16* out,
                              int sms, cudaStream_t s) {
  if (count <= 0) return cudaSuccess;
  if (count % 8) return cudaErrorInvalidValue;
  const int64_t n8 = count / 8;
  const int blocks = (int)std::min<int64_t>((n8 + 255) / 256, (int64_t)sms * 8);
  gdpa_sum_splits_kernel<<<blocks, 256, 0, s>>>(part, splits, count, out);
  return cudaGetLastError();
}

}  // namespace gdpa
