// Projection GEMM on the sm_100a tensor cores: C = A · Bᵀ with A [M, K] and
// B [N, K] bf16 (both K-major, rows contiguous), fp32 accumulation in tensor
// memory, and an epilogue that writes column ranges of C to up to three
// outputs (each bf16 or fp32, with an optional per-column bias).
//
// Page "SAMBA混合注意力状态空间模型", section 数学框架 / Mamba层: the
// selective parameters are linear maps of the layer input, B_t = Linear_B(x_t),
// C_t = Linear_C(x_t), Δ_t = τ_Δ(Linear_Δ(x_t)); the layers around the two
// mixers (the Mamba input and output projections, the attention's Q/K/V and
// output projections) are linear maps of the same kind.  One GEMM with a
// column-split epilogue produces such a map's outputs directly in the layouts
// the mixers read: for instance x and z of the Mamba input projection in one
// pass, or Δ-low-rank, B and C of the selective-parameter projection.
//
// Design: persistent CTAs, one per SM, walking the 128 x BN tiles of C
// (BN = 256, 128 when N < 256, 64 when M <= 128) with the N tile fastest;
// K in steps of 64 (128-byte
// rows, 128-byte swizzle).  Warp 4 streams A and B tiles into a STG-deep
// shared-memory ring with TMA, continuously across tiles; warp 5 issues the
// tcgen05.mma (kind::f16, M = 128, N = BN, K = 16 per instruction) into one of
// two BN-column accumulators in tensor memory, alternating per tile; warps
// 0-3 (one TMEM lane quarter each, thread = row) read a finished accumulator
// back and write the outputs while the next tile accumulates into the other,
// so the epilogue runs under the next tile's main loop.  Every wait is
// bounded.
#include "common.cuh"
#include "host.hpp"
#include "pdl.cuh"

namespace samba {

struct GemmOut {
  void* ptr;          // row-major [M, col1 - col0] (leading dimension ld, in elements)
  const float* bias;  // [col1 - col0] or null
  int64_t ld;
  int col0, col1;     // columns [col0, col1) of C
  int dtype;          // SAMBA_BF16 or SAMBA_F32
};

struct GemmParams {
  int64_t M, N, K;
  GemmOut out[3];
  int nout;
};

template <int BN, int STG>
struct GemmCfg {
  static constexpr int BM = 128, BK = 64;
  static constexpr int A_BYTES = BM * BK * 2, B_BYTES = BN * BK * 2, STAGE = A_BYTES + B_BYTES;
  static constexpr int BAR_OFF = STG * STAGE;
  static constexpr int SMEM = BAR_OFF + 256 + 1024;  // barriers + alignment slack
  static constexpr uint32_t TMEM_COLS = 2 * BN;      // two accumulators
  static constexpr int THREADS = 192;
};

template <int BN, int STG>
__global__ void __launch_bounds__(192, 1)
    gemm_kernel(const __grid_constant__ CUtensorMap map_a, const __grid_constant__ CUtensorMap map_b,
                const GemmParams p) {
  using Cfg = GemmCfg<BN, STG>;
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + Cfg::BAR_OFF);
  uint64_t* empty = full + STG;
  uint64_t* acc_full = empty + STG;   // [2] an accumulator holds a finished tile
  uint64_t* acc_empty = acc_full + 2; // [2] the epilogue has read it (4 warps)
  uint64_t* done = acc_empty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(done + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  static_assert((2 * STG + 5) * 8 + 8 <= 256, "barrier block");
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int ktiles = static_cast<int>((p.K + Cfg::BK - 1) / Cfg::BK);
  const int64_t n_tiles_n = (p.N + BN - 1) / BN;
  const int64_t n_tiles = n_tiles_n * ((p.M + Cfg::BM - 1) / Cfg::BM);

  if (threadIdx.x == 0) {
    for (int s = 0; s < STG; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&acc_full[a], 1);
      mbar_init(&acc_empty[a], 4);
    }
    mbar_init(done, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 5) {
    tmem_alloc(tmem_slot, Cfg::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 4) {
    // ================================================================ TMA
    if (lane == 0) {
      tma_prefetch_desc(&map_a);
      tma_prefetch_desc(&map_b);
      uint32_t it = 0;  // k-steps issued so far, over all tiles of this CTA
      bool ok = true;
      for (int64_t tile = blockIdx.x; tile < n_tiles && ok; tile += gridDim.x) {
        const int64_t n0 = (tile % n_tiles_n) * BN, m0 = (tile / n_tiles_n) * Cfg::BM;
        for (int i = 0; i < ktiles; ++i, ++it) {
          const int s = it % STG;
          if (it >= STG && !mbar_wait(&empty[s], ((it / STG) - 1) & 1, abort_flag)) { ok = false; break; }
          unsigned char* st = smem + s * Cfg::STAGE;
          mbar_arrive_expect_tx(&full[s], Cfg::STAGE);
          tma_load_2d(st, &map_a, &full[s], i * Cfg::BK, static_cast<int>(m0));
          tma_load_2d(st + Cfg::A_BYTES, &map_b, &full[s], i * Cfg::BK, static_cast<int>(n0));
        }
      }
      // copies still in flight complete before the CTA can exit
      volatile int never = 0;
      for (uint32_t i = (it > STG ? it - STG : 0); i < it; ++i) mbar_wait(&full[i % STG], (i / STG) & 1, &never);
    }
  } else if (warp == 5) {
    // ================================================================ MMA
    constexpr uint32_t IDESC = idesc_bf16_f32(Cfg::BM, BN, 0, 0);
    const uint32_t base = smem_u32(smem);
    const uint64_t d_a0 = smem_desc(base, 16, 1024, 2);
    const uint32_t hi = static_cast<uint32_t>(d_a0 >> 32), lo0 = static_cast<uint32_t>(d_a0);
    constexpr uint32_t kStageDesc = Cfg::STAGE >> 4, kBDesc = Cfg::A_BYTES >> 4;
    auto desc64 = [&](uint32_t lo) { return (static_cast<uint64_t>(hi) << 32) | lo; };
    auto wait = [&](uint64_t* bar, uint32_t parity) {
      return __all_sync(0xffffffffu, mbar_wait(bar, parity, abort_flag));
    };
    bool ok = true;
    uint32_t it = 0, lt = 0;
    for (int64_t tile = blockIdx.x; tile < n_tiles && ok; tile += gridDim.x, ++lt) {
      const uint32_t acc = lt & 1;
      // the accumulator's previous tile (two tiles back) must have been read out
      if (lt >= 2 && !(ok = wait(&acc_empty[acc], ((lt >> 1) - 1) & 1))) break;
      tc_fence_after();
      const uint32_t d_tmem = tmem + acc * BN;
      for (int i = 0; i < ktiles; ++i, ++it) {
        const int s = it % STG;
        ok = wait(&full[s], (it / STG) & 1);
        if (!ok) break;
        tc_fence_after();
        const uint32_t la = lo0 + s * kStageDesc, lb = la + kBDesc;
#pragma unroll
        for (int k = 0; k < Cfg::BK / 16; ++k)  // 16 K-elements = 32 bytes = 2 descriptor units
          umma_ss_w(d_tmem, desc64(la + 2 * k), desc64(lb + 2 * k), IDESC, (i > 0 || k > 0) ? 1u : 0u);
        tc_commit_w(&empty[s]);
      }
      if (!ok) break;
      tc_commit_w(&acc_full[acc]);  // every MMA of this tile has completed
    }
    tc_commit_w(done);
    volatile int never = 0;
    mbar_wait(done, 0, &never);
  } else {
    // ============================================================ epilogue
    const int row_local = warp * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>(warp * 32) << 16;
    uint32_t lt = 0;
    bool ok = true;
    for (int64_t tile = blockIdx.x; tile < n_tiles && ok; tile += gridDim.x, ++lt) {
      const int64_t n0 = (tile % n_tiles_n) * BN, m0 = (tile / n_tiles_n) * Cfg::BM;
      const int64_t row = m0 + row_local;
      const uint32_t acc = lt & 1;
      ok = __all_sync(0xffffffffu, mbar_wait(&acc_full[acc], (lt >> 1) & 1, abort_flag));
      if (!ok) break;
      tc_fence_after();
      const uint32_t t_row = tmem + lane_off + acc * BN;
#pragma unroll 1
      for (int c0 = 0; c0 < BN; c0 += 32) {
        uint32_t r[32];
        tmem_ld32(t_row + c0, r);  // warp-collective: every lane, whatever its row
        tc_wait_ld();
        if (row >= p.M || !SAMBA_CHECK(row >= 0 && n0 + c0 < p.N)) continue;
#pragma unroll
        for (int j = 0; j < 32; j += 8) {
          const int64_t col = n0 + c0 + j;  // 8 consecutive columns
#pragma unroll
          for (int o = 0; o < 3; ++o) {
            if (o >= p.nout) break;
            const GemmOut& out = p.out[o];
            if (col + 8 <= out.col0 || col >= out.col1) continue;
            const bool whole = col >= out.col0 && col + 8 <= out.col1 && col + 8 <= p.N;
            float v[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) {
              v[e] = __uint_as_float(r[j + e]);
              const int64_t cc = col + e - out.col0;
              if (out.bias && cc >= 0 && cc < out.col1 - out.col0) v[e] += out.bias[cc];
            }
            const int64_t base_idx = row * out.ld + (col - out.col0);
            if (out.dtype == SAMBA_BF16) {
              __nv_bfloat16* dst = reinterpret_cast<__nv_bfloat16*>(out.ptr) + base_idx;
              if (whole && (reinterpret_cast<uintptr_t>(dst) & 15u) == 0) {
                uint4 pk;
                pk.x = (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(v[0])) |
                       ((uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(v[1])) << 16);
                pk.y = (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(v[2])) |
                       ((uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(v[3])) << 16);
                pk.z = (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(v[4])) |
                       ((uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(v[5])) << 16);
                pk.w = (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(v[6])) |
                       ((uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(v[7])) << 16);
                *reinterpret_cast<uint4*>(dst) = pk;
              } else {
                for (int e = 0; e < 8; ++e) {
                  const int64_t cc = col + e;
                  if (cc >= out.col0 && cc < out.col1 && cc < p.N) dst[e] = __float2bfloat16_rn(v[e]);
                }
              }
            } else {
              float* dst = reinterpret_cast<float*>(out.ptr) + base_idx;
              if (whole && (reinterpret_cast<uintptr_t>(dst) & 15u) == 0) {
                reinterpret_cast<float4*>(dst)[0] = make_float4(v[0], v[1], v[2], v[3]);
                reinterpret_cast<float4*>(dst)[1] = make_float4(v[4], v[5], v[6], v[7]);
              } else {
                for (int e = 0; e < 8; ++e) {
                  const int64_t cc = col + e;
                  if (cc >= out.col0 && cc < out.col1 && cc < p.N) dst[e] = v[e];
                }
              }
            }
          }
        }
      }
      // this accumulator may take the tile after next
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acc_empty[acc]);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 5) {
    tc_fence_after();
    tmem_dealloc(tmem, Cfg::TMEM_COLS);
  }
}

// ------------------------------------------------------------ skinny GEMM
// C = A · Bᵀ for at most 32 rows of A (a decode step's activations, one row
// per sequence).  The operands trade places so that the weight fills the
// 128-row side of the MMA: D[n, m] = sum_k B[n, k] A[m, k] with M = 128 rows
// of B and N = MP = 16 or 32 rows of A (rows of A past M read as zeros).
// The problem's nblk × kb k-steps (128-row blocks of B × 64-wide K steps)
// are dealt to the CTAs in equal contiguous ranges, so every SM streams an
// equal share of the weight; a range may end inside one block and go on in
// the next.  A CTA whose range covers a block's whole K writes the outputs
// from its accumulator.  Otherwise each epilogue warp adds its 32 rows'
// partial sums into an fp32 accumulator in the workspace and then counts its
// k-steps on the (block, warp) counter; the warp whose count completes the
// block reads the sums back, writes the outputs and returns the accumulator
// rows and the counter to zero, so the workspace is zero again after every
// call.  Roles: warp 4 loads (TMA), warp 5 issues tcgen05.mma into one of two
// MP-column accumulators (alternating per range piece), warps 0-3 drain.  It
// is launched as a programmatic dependent of the kernel before it (pdl.cuh):
// the first stages' weight tiles are requested before the wait for that
// kernel, A's tiles and every global write after it.
#ifndef SAMBA_SKINNY_MIN_KSTEPS
#define SAMBA_SKINNY_MIN_KSTEPS 4  // fixed by measurement (serving loop: 1, 2, 4, 8 -> 266, 258, 254, 254 us per step)
#endif

struct SkinnyParams {
  int64_t M, N, K;
  GemmOut out[3];
  int nout;
  int kb;            // k-steps per block
  int64_t T;         // nblk * kb
  float* acc;        // [nblk * 128][MP] fp32, zero between calls
  uint32_t* cnt;     // [nblk][4], zero between calls
};

template <int MP, int STG>
struct SkinnyCfg {
  static constexpr int BN = 128, BK = 64;
  static constexpr int B_BYTES = BN * BK * 2, A_BYTES = MP * BK * 2, STAGE = B_BYTES + A_BYTES;
  static_assert(STAGE % 1024 == 0, "stages stay 1024-byte aligned for the 128-byte swizzle");
  static constexpr int BAR_OFF = STG * STAGE;
  static constexpr int SMEM = BAR_OFF + 256 + 1024;
  static constexpr uint32_t TMEM_COLS = 2 * MP < 32 ? 32 : 2 * MP;
  static constexpr int THREADS = 192;
};

template <int MP>
__device__ __forceinline__ void skinny_store(const SkinnyParams& p, int64_t n, const float (&v)[MP]) {
  if (n >= p.N || !SAMBA_CHECK(n >= 0 && p.M <= MP)) return;
#pragma unroll
  for (int o = 0; o < 3; ++o) {
    if (o >= p.nout) break;
    const GemmOut& out = p.out[o];
    if (n < out.col0 || n >= out.col1) continue;
    const int64_t cc = n - out.col0;
    const float b = out.bias ? out.bias[cc] : 0.f;
#pragma unroll
    for (int m = 0; m < MP; ++m) {
      if (m >= p.M) break;
      const int64_t idx = m * out.ld + cc;
      if (out.dtype == SAMBA_BF16) reinterpret_cast<__nv_bfloat16*>(out.ptr)[idx] = __float2bfloat16_rn(v[m] + b);
      else reinterpret_cast<float*>(out.ptr)[idx] = v[m] + b;
    }
  }
}

template <int MP, int STG>
__global__ void __launch_bounds__(192, 1)
    skinny_gemm_kernel(const __grid_constant__ CUtensorMap map_a, const __grid_constant__ CUtensorMap map_b,
                       const SkinnyParams p) {
  using Cfg = SkinnyCfg<MP, STG>;
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + Cfg::BAR_OFF);
  uint64_t* empty = full + STG;
  uint64_t* acc_full = empty + STG;
  uint64_t* acc_empty = acc_full + 2;
  uint64_t* done = acc_empty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(done + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  static_assert((2 * STG + 5) * 8 + 8 <= 256, "barrier block");
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int kb = p.kb;
  // this CTA's k-steps [g0, g1) of the nblk * kb
  const int64_t g0 = p.T * blockIdx.x / gridDim.x, g1 = p.T * (blockIdx.x + 1) / gridDim.x;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STG; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&acc_full[a], 1);
      mbar_init(&acc_empty[a], 4);
    }
    mbar_init(done, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 5) {
    tmem_alloc(tmem_slot, Cfg::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  pdl_launch_dependents();
  if (warp == 4) {
    // ================================================================ TMA
    if (lane == 0) {
      tma_prefetch_desc(&map_a);
      tma_prefetch_desc(&map_b);
      // The weight tiles of the first stages go out before the wait for the
      // kernel that writes A (no kernel writes the weight); A's tiles after.
      const int pre = static_cast<int>(g1 - g0 < STG ? g1 - g0 : STG);
      for (int i = 0; i < pre; ++i) {
        const int64_t g = g0 + i, nb = g / kb;
        const int kk = static_cast<int>(g - nb * kb);
        mbar_arrive_expect_tx(&full[i], Cfg::STAGE);
        tma_load_2d(smem + i * Cfg::STAGE, &map_b, &full[i], kk * Cfg::BK, static_cast<int>(nb * Cfg::BN));
      }
      pdl_wait();
      for (int i = 0; i < pre; ++i) {
        const int64_t g = g0 + i, nb = g / kb;
        const int kk = static_cast<int>(g - nb * kb);
        tma_load_2d(smem + i * Cfg::STAGE + Cfg::B_BYTES, &map_a, &full[i], kk * Cfg::BK, 0);
      }
      uint32_t it = static_cast<uint32_t>(pre);
      bool ok = true;
      for (int64_t g = g0 + pre; g < g1 && ok; ++g, ++it) {
        const int64_t nb = g / kb;
        const int kk = static_cast<int>(g - nb * kb);
        const int s = it % STG;
        if (it >= STG && !mbar_wait(&empty[s], ((it / STG) - 1) & 1, abort_flag)) { ok = false; break; }
        unsigned char* st = smem + s * Cfg::STAGE;
        mbar_arrive_expect_tx(&full[s], Cfg::STAGE);
        tma_load_2d(st, &map_b, &full[s], kk * Cfg::BK, static_cast<int>(nb * Cfg::BN));
        tma_load_2d(st + Cfg::B_BYTES, &map_a, &full[s], kk * Cfg::BK, 0);
      }
      volatile int never = 0;
      for (uint32_t i = (it > STG ? it - STG : 0); i < it; ++i) mbar_wait(&full[i % STG], (i / STG) & 1, &never);
    }
  } else if (warp == 5) {
    // ================================================================ MMA
    constexpr uint32_t IDESC = idesc_bf16_f32(128, MP, 0, 0);
    const uint32_t base = smem_u32(smem);
    const uint64_t d0 = smem_desc(base, 16, 1024, 2);
    const uint32_t hi = static_cast<uint32_t>(d0 >> 32), lo0 = static_cast<uint32_t>(d0);
    constexpr uint32_t kStageDesc = Cfg::STAGE >> 4, kADesc = Cfg::B_BYTES >> 4;
    auto desc64 = [&](uint32_t lo) { return (static_cast<uint64_t>(hi) << 32) | lo; };
    auto wait = [&](uint64_t* bar, uint32_t parity) {
      return __all_sync(0xffffffffu, mbar_wait(bar, parity, abort_flag));
    };
    bool ok = true;
    uint32_t it = 0, j = 0;
    for (int64_t g = g0; g < g1 && ok; ++j) {
      const int64_t nb = g / kb;
      const int64_t end = (nb + 1) * kb < g1 ? (nb + 1) * kb : g1;
      const uint32_t acc = j & 1;
      if (j >= 2 && !(ok = wait(&acc_empty[acc], ((j >> 1) - 1) & 1))) break;
      tc_fence_after();
      const uint32_t d_tmem = tmem + acc * MP;
      for (int64_t i = g; i < end; ++i, ++it) {
        const int s = it % STG;
        ok = wait(&full[s], (it / STG) & 1);
        if (!ok) break;
        tc_fence_after();
        const uint32_t lb = lo0 + s * kStageDesc, la = lb + kADesc;
#pragma unroll
        for (int k = 0; k < Cfg::BK / 16; ++k)
          umma_ss_w(d_tmem, desc64(lb + 2 * k), desc64(la + 2 * k), IDESC, (i > g || k > 0) ? 1u : 0u);
        tc_commit_w(&empty[s]);
      }
      if (!ok) break;
      tc_commit_w(&acc_full[acc]);
      g = end;
    }
    tc_commit_w(done);
    volatile int never = 0;
    mbar_wait(done, 0, &never);
  } else {
    // ============================================================ epilogue
    pdl_wait();  // the outputs and the workspace may still be in use before it
    const uint32_t lane_off = static_cast<uint32_t>(warp * 32) << 16;
    bool ok = true;
    uint32_t j = 0;
    for (int64_t g = g0; g < g1 && ok; ++j) {
      const int64_t nb = g / kb;
      const int64_t end = (nb + 1) * kb < g1 ? (nb + 1) * kb : g1;
      const int nk = static_cast<int>(end - g);
      g = end;
      const uint32_t acc = j & 1;
      ok = __all_sync(0xffffffffu, mbar_wait(&acc_full[acc], (j >> 1) & 1, abort_flag));
      if (!ok) break;
      tc_fence_after();
      uint32_t r[MP];
      {
        uint32_t r16[16];
        tmem_ld16(tmem + lane_off + acc * MP, r16);
        tc_wait_ld();
#pragma unroll
        for (int e = 0; e < 16; ++e) r[e] = r16[e];
        if constexpr (MP == 32) {
          tmem_ld16(tmem + lane_off + acc * MP + 16, r16);
          tc_wait_ld();
#pragma unroll
          for (int e = 0; e < 16; ++e) r[16 + e] = r16[e];
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acc_empty[acc]);
      const int64_t n = nb * Cfg::BN + warp * 32 + lane;
      float v[MP];
#pragma unroll
      for (int e = 0; e < MP; ++e) v[e] = __uint_as_float(r[e]);
      if (nk == kb) {  // the block's whole K in this range
        skinny_store<MP>(p, n, v);
        continue;
      }
      if (!SAMBA_CHECK(nb * 4 + warp < p.T / kb * 4)) continue;  // the workspace holds nblk blocks
      float4* row = reinterpret_cast<float4*>(p.acc + n * MP);
#pragma unroll
      for (int q = 0; q < MP / 4; ++q) atomicAdd(row + q, make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]));
      __threadfence();
      __syncwarp();
      uint32_t* counter = p.cnt + nb * 4 + warp;
      uint32_t before = 0;
      if (lane == 0) before = atomicAdd(counter, static_cast<uint32_t>(nk));
      before = __shfl_sync(0xffffffffu, before, 0);
      if (before + nk == static_cast<uint32_t>(kb)) {  // every range of this block has added its sums
        __threadfence();
#pragma unroll
        for (int q = 0; q < MP / 4; ++q) {
          const float4 t = __ldcg(row + q);
          v[4 * q] = t.x;
          v[4 * q + 1] = t.y;
          v[4 * q + 2] = t.z;
          v[4 * q + 3] = t.w;
          __stcg(row + q, make_float4(0.f, 0.f, 0.f, 0.f));
        }
        skinny_store<MP>(p, n, v);
        if (lane == 0) *counter = 0;
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 5) {
    tc_fence_after();
    tmem_dealloc(tmem, Cfg::TMEM_COLS);
  }
}

static int skinny_mp(int64_t M) { return M <= 16 ? 16 : 32; }

size_t gemm_workspace_size(int64_t M, int64_t N) {
  if (M < 1 || M > 32 || N < 1) return 0;
  const int64_t nblk = (N + 127) / 128;
  const size_t acc = static_cast<size_t>(nblk) * 128 * skinny_mp(M) * 4;
  return (acc + static_cast<size_t>(nblk) * 4 * 4 + 255) / 256 * 256;
}

template <int MP>
static int launch_skinny_t(const samba_gemm_args& a, cudaStream_t stream) {
  constexpr int STG = 8;
  using Cfg = SkinnyCfg<MP, STG>;
  auto kern = skinny_gemm_kernel<MP, STG>;
  static PerDeviceOnce attr;
  const int arc = once_per_device(attr, [&] {
    return cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg::SMEM) == cudaSuccess
               ? SAMBA_OK
               : fail(SAMBA_ERR_CUDA, "gemm: cannot set shared memory size");
  });
  if (arc != SAMBA_OK) return arc;
  CUtensorMap ma, mb;
  const uint32_t box_a[2] = {(uint32_t)Cfg::BK, (uint32_t)MP};
  const uint32_t box_b[2] = {(uint32_t)Cfg::BK, (uint32_t)Cfg::BN};
  const uint64_t da[2] = {(uint64_t)a.K, (uint64_t)a.M}, sa[1] = {(uint64_t)a.lda * 2};
  const uint64_t db[2] = {(uint64_t)a.K, (uint64_t)a.N}, sb[1] = {(uint64_t)a.ldb * 2};
  int rc = encode_tiled(&ma, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, a.A, da, sa, box_a, CU_TENSOR_MAP_SWIZZLE_128B,
                        "gemm A");
  if (rc) return rc;
  rc = encode_tiled(&mb, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, a.B, db, sb, box_b, CU_TENSOR_MAP_SWIZZLE_128B, "gemm B");
  if (rc) return rc;
  SkinnyParams p;
  p.M = a.M;
  p.N = a.N;
  p.K = a.K;
  p.nout = a.nout;
  for (int o = 0; o < a.nout; ++o) {
    p.out[o].ptr = a.out[o].ptr;
    p.out[o].bias = a.out[o].bias;
    p.out[o].ld = a.out[o].ld;
    p.out[o].col0 = static_cast<int>(a.out[o].col0);
    p.out[o].col1 = static_cast<int>(a.out[o].col1);
    p.out[o].dtype = a.out[o].dtype;
  }
  const int64_t nblk = (a.N + Cfg::BN - 1) / Cfg::BN;
  p.kb = static_cast<int>((a.K + Cfg::BK - 1) / Cfg::BK);
  p.T = nblk * p.kb;
  p.acc = reinterpret_cast<float*>(a.workspace);
  p.cnt = reinterpret_cast<uint32_t*>(reinterpret_cast<unsigned char*>(a.workspace) +
                                      static_cast<size_t>(nblk) * Cfg::BN * MP * 4);
  // At least SAMBA_SKINNY_MIN_KSTEPS k-steps per CTA (a block's whole K when
  // it has fewer): fewer partial sums meet in the workspace for small weights.
  const int64_t min_ks = std::min<int64_t>(p.kb, SAMBA_SKINNY_MIN_KSTEPS);
  const unsigned grid = (unsigned)std::min<int64_t>((p.T + min_ks - 1) / min_ks, sm_count());
  const cudaError_t e = launch_pdl(kern, dim3(grid), dim3(Cfg::THREADS), Cfg::SMEM, stream, ma, mb, p);
  if (e != cudaSuccess) return fail(SAMBA_ERR_CUDA, "samba_gemm: launch failed: %s", cudaGetErrorString(e));
  return check_launch("samba_gemm");
}

int take_status_gemm(cudaStream_t s) { return take_status_word(s); }

template <int BN>
static int launch_gemm_t(const samba_gemm_args& a, cudaStream_t stream) {
  constexpr int STG = BN == 256 ? 4 : (BN == 128 ? 6 : 8);
  using Cfg = GemmCfg<BN, STG>;
  auto kern = gemm_kernel<BN, STG>;
  static PerDeviceOnce attr;
  const int arc = once_per_device(attr, [&] {
    return cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg::SMEM) == cudaSuccess
               ? SAMBA_OK
               : fail(SAMBA_ERR_CUDA, "gemm: cannot set shared memory size");
  });
  if (arc != SAMBA_OK) return arc;
  CUtensorMap ma, mb;
  const uint32_t box_a[2] = {(uint32_t)Cfg::BK, (uint32_t)Cfg::BM};
  const uint32_t box_b[2] = {(uint32_t)Cfg::BK, (uint32_t)BN};
  const uint64_t da[2] = {(uint64_t)a.K, (uint64_t)a.M}, sa[1] = {(uint64_t)a.lda * 2};
  const uint64_t db[2] = {(uint64_t)a.K, (uint64_t)a.N}, sb[1] = {(uint64_t)a.ldb * 2};
  int rc = encode_tiled(&ma, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, a.A, da, sa, box_a, CU_TENSOR_MAP_SWIZZLE_128B,
                        "gemm A");
  if (rc) return rc;
  rc = encode_tiled(&mb, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, a.B, db, sb, box_b, CU_TENSOR_MAP_SWIZZLE_128B, "gemm B");
  if (rc) return rc;
  GemmParams p;
  p.M = a.M;
  p.N = a.N;
  p.K = a.K;
  p.nout = a.nout;
  for (int o = 0; o < a.nout; ++o) {
    p.out[o].ptr = a.out[o].ptr;
    p.out[o].bias = a.out[o].bias;
    p.out[o].ld = a.out[o].ld;
    p.out[o].col0 = static_cast<int>(a.out[o].col0);
    p.out[o].col1 = static_cast<int>(a.out[o].col1);
    p.out[o].dtype = a.out[o].dtype;
  }
  const int64_t tiles = ((a.N + BN - 1) / BN) * ((a.M + Cfg::BM - 1) / Cfg::BM);
  const unsigned grid = (unsigned)std::min<int64_t>(tiles, sm_count());
  kern<<<grid, Cfg::THREADS, Cfg::SMEM, stream>>>(ma, mb, p);
  return check_launch("samba_gemm");
}

// Up to 32 rows with a workspace: the split-K kernel above.  Otherwise tile
// width 256 columns for large problems and, with at most one 128-row block
// (decode-sized M without a workspace), 64 columns, so that the weight matrix
// is streamed by as many SMs as the tiles allow.
int launch_gemm(const samba_gemm_args& a, cudaStream_t s) {
  if (a.M <= 32 && a.workspace && a.workspace_bytes >= gemm_workspace_size(a.M, a.N))
    return a.M <= 16 ? launch_skinny_t<16>(a, s) : launch_skinny_t<32>(a, s);
  if (a.M <= 128) return launch_gemm_t<64>(a, s);
  return a.N >= 256 ? launch_gemm_t<256>(a, s) : launch_gemm_t<128>(a, s);
}

}  // namespace samba
