// Banded sliding-window attention prefill on the sm_100a tensor cores.
//
// Page "SAMBA混合注意力状态空间模型", section 滑动窗口注意力: attention with
// softmax(Q Kᵀ/√d_k + M) V where the window mask M keeps the last W keys of
// every query (read here as the causal band 0 <= i - j < W); hackernoon page
// §2.1.2 "Sliding Window Attention (SWA) Layer" slides a window of 2048.
//
// Design (one CTA per SM, persistent over work units):
//   * A work unit is (batch b, kv head g, 2·TOK consecutive query tokens).
//     The GROUP = Hq/Hkv query heads that share kv head g are stacked into the
//     128 rows of one tile: row r = token (r / GROUP), head (r % GROUP), with
//     TOK = 128 / GROUP tokens.  Two such Q tiles (A: the first TOK tokens,
//     B: the next TOK) are processed ping-pong, so every K/V tile that is
//     loaded serves 256 query rows.
//   * Key tiles of 128 keys are aligned to the top of the unit and walk
//     down the band: tile m holds keys [top - 128(m+1), top - 128m) with
//     top = first token + 2·TOK, so ceil((W + 2·TOK - 1) / 128) tiles cover
//     the band of both Q tiles; tiles outside the band are never loaded.
//     Only tiles crossing the diagonal, the window's lower edge or key 0 are
//     masked element by element.
//   * Warp 8 issues TMA (Q once per unit, K and V per tile into a STG-deep
//     ring).  Warp 9 owns tensor memory and one thread of it issues every
//     tcgen05.mma: S = Q·Kᵀ (bf16, fp32 accumulate into TMEM) and
//     O += P·V with P read straight from TMEM.  Warps 0-3 and 4-7 are the
//     softmax warpgroups of Q tiles A and B: each thread owns one row, reads
//     its S row from TMEM, keeps the running max and sum in fp32, writes P
//     back to TMEM as bf16, and rescales O in TMEM only when the running max
//     grows by more than 2^8 (the result does not depend on the reference
//     max; the threshold only bounds P <= 256).
//   * TMEM columns: S_A 0-127, S_B 128-255, P_A 256-319, P_B 320-383,
//     O_A 384-447, O_B 448-511 (fp32, one row per lane).
#include "common.cuh"

namespace samba {

struct SwaParams {
  __nv_bfloat16* o;
  float* lse;
  int64_t L, W;
  int Hq, Hkv, B;
  float scale_log2;  // softmax scale × log2(e)
  int units_per_head;
  int total_units;
};

template <int HD, int GROUP, int STG>
struct SwaCfg {
  static constexpr int TOK = 128 / GROUP;
  static constexpr int ROW_BYTES = HD * 2;                 // one K-major row (= swizzle span)
  static constexpr int TILE_BYTES = 128 * ROW_BYTES;       // 128 rows
  static constexpr int Q_OFF = 0;                          // Q_A, Q_B
  static constexpr int K_OFF = 2 * TILE_BYTES;
  static constexpr int V_OFF = K_OFF + STG * TILE_BYTES;
  static constexpr int BAR_OFF = V_OFF + STG * TILE_BYTES;
  static constexpr int SMEM = BAR_OFF + 256 + 1024;        // + alignment slack
  static constexpr uint32_t SWZ = HD == 64 ? 2u : (HD == 32 ? 4u : 6u);  // descriptor swizzle code
  static constexpr uint32_t ATOM = 8 * ROW_BYTES;          // 8-row swizzle atom
  static constexpr int THREADS = 320;
  static constexpr uint32_t TMEM_COLS = 512;
  static constexpr uint32_t COL_S = 0, COL_P = 256, COL_O = 384;
};

// Warp roles: 0-3 softmax of Q tile A, 4-7 softmax of Q tile B (warp % 4 is
// the TMEM lane quarter a warp may access), 8 TMA producer, 9 MMA issuer.
constexpr int kWarpTma = 8, kWarpMma = 9;

// Barrier indices inside the barrier block.
enum : int {
  BQ_FULL = 0, BQ_EMPTY, BS_A, BS_B, BP_A, BP_B, BO_A, BO_B, BOE_A, BOE_B, BMMA_DONE, B_STAGE0
};

__device__ __forceinline__ float ex2f(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Every SWA_POLY-th pair of probabilities is evaluated on the FMA pipe
// (0: never); the rest use the MUFU ex2.  Build-time, fixed by measurement.
#ifndef SWA_POLY
#define SWA_POLY 4
#endif

// 2^x for a pair of arguments on the FMA pipe, accurate to ~1e-4 relative
// (ample for probabilities that are rounded to bf16): x = j + f with
// j = rint(x) by magic-number rounding, 2^f by a degree-3 polynomial fitted
// on [-1/2, 1/2] for relative error with p(0) = 1 (fit made for this
// library), and j added to the exponent bits.  x is clamped below at -125,
// so masked scores (-inf) give 2^-125 instead of 0, which no sum can notice.
__device__ __forceinline__ f2 ex2_poly3x2(f2 x) {
  float2 xv = up2(x);
  xv.x = fmaxf(xv.x, -125.f);
  xv.y = fmaxf(xv.y, -125.f);
  const f2 xc = pk2(xv.x, xv.y);
  const f2 magic = pk2(12582912.f, 12582912.f);  // 1.5 * 2^23
  const f2 t = add2(xc, magic);
  const f2 f = sub2(xc, sub2(t, magic));
  f2 p = pk2(0x1.c2a212p-5f, 0x1.c2a212p-5f);
  p = fma2(p, f, pk2(0x1.f00c4ep-3f, 0x1.f00c4ep-3f));
  p = fma2(p, f, pk2(0x1.62f5fap-1f, 0x1.62f5fap-1f));
  p = fma2(p, f, pk2(1.f, 1.f));
  const float2 tv = up2(t), pv = up2(p);
  return pk2(__int_as_float(__float_as_int(pv.x) + (__float_as_int(tv.x) << 23)),
             __int_as_float(__float_as_int(pv.y) + (__float_as_int(tv.y) << 23)));
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

// unit index -> (b, g, first query token)
__device__ __forceinline__ void unit_coords(int u, const SwaParams& p, int tok2, int& b, int& g, int64_t& i0) {
  const int per_b = p.Hkv * p.units_per_head;
  b = u / per_b;
  const int r = u - b * per_b;
  g = r / p.units_per_head;
  i0 = static_cast<int64_t>(r - g * p.units_per_head) * tok2;
}

// number of key tiles of a unit (tiles lying entirely before key 0 are skipped)
__device__ __forceinline__ int unit_tiles(int64_t top, int64_t W, int tok2) {
  const int64_t n_band = (W + tok2 - 1 + 127) / 128;
  const int64_t n_pos = (top + 127) / 128;
  return static_cast<int>(n_band < n_pos ? n_band : n_pos);
}

template <int HD, int GROUP, int STG>
__global__ void __launch_bounds__(320, 1)
    swa_fwd_kernel(const __grid_constant__ CUtensorMap map_q, const __grid_constant__ CUtensorMap map_k,
                   const __grid_constant__ CUtensorMap map_v, const SwaParams p) {
  using Cfg = SwaCfg<HD, GROUP, STG>;
  constexpr int TOK = Cfg::TOK;
  constexpr int TOK2 = 2 * TOK;
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Cfg::BAR_OFF);
  uint64_t* kfull = bars + B_STAGE0;
  uint64_t* vfull = kfull + STG;
  uint64_t* kvempty = vfull + STG;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(kvempty + STG);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    mbar_init(&bars[BQ_FULL], 1);
    mbar_init(&bars[BQ_EMPTY], 1);
    mbar_init(&bars[BS_A], 1);
    mbar_init(&bars[BS_B], 1);
    mbar_init(&bars[BP_A], 128);
    mbar_init(&bars[BP_B], 128);
    mbar_init(&bars[BO_A], 1);
    mbar_init(&bars[BO_B], 1);
    mbar_init(&bars[BOE_A], 128);
    mbar_init(&bars[BOE_B], 128);
    mbar_init(&bars[BMMA_DONE], 1);
    for (int s = 0; s < STG; ++s) {
      mbar_init(&kfull[s], 1);
      mbar_init(&vfull[s], 1);
      mbar_init(&kvempty[s], 1);
    }
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == kWarpMma) {
    tmem_alloc(tmem_slot, Cfg::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == kWarpTma) {
    // ================================================================ TMA
    if (lane == 0) {
      tma_prefetch_desc(&map_q);
      tma_prefetch_desc(&map_k);
      tma_prefetch_desc(&map_v);
      uint32_t it = 0, nu = 0;
      bool ok = true;
      for (int u = blockIdx.x; u < p.total_units && ok; u += gridDim.x, ++nu) {
        int b, g;
        int64_t i0;
        unit_coords(u, p, TOK2, b, g, i0);
        const int64_t top = i0 + TOK2;
        const int nt = unit_tiles(top, p.W, TOK2);
        if (nu > 0 && !mbar_wait(&bars[BQ_EMPTY], (nu - 1) & 1, abort_flag)) { ok = false; break; }
        mbar_arrive_expect_tx(&bars[BQ_FULL], 2 * Cfg::TILE_BYTES);
        tma_load_4d(smem + Cfg::Q_OFF, &map_q, &bars[BQ_FULL], 0, g * GROUP, (int)i0, b);
        tma_load_4d(smem + Cfg::Q_OFF + Cfg::TILE_BYTES, &map_q, &bars[BQ_FULL], 0, g * GROUP, (int)(i0 + TOK), b);
        for (int m = 0; m < nt; ++m, ++it) {
          const int s = it % STG;
          if (it >= STG && !mbar_wait(&kvempty[s], ((it / STG) - 1) & 1, abort_flag)) { ok = false; break; }
          const int k0 = (int)(top - 128 * (m + 1));
          mbar_arrive_expect_tx(&kfull[s], Cfg::TILE_BYTES);
          tma_load_4d(smem + Cfg::K_OFF + s * Cfg::TILE_BYTES, &map_k, &kfull[s], 0, g, k0, b);
          mbar_arrive_expect_tx(&vfull[s], Cfg::TILE_BYTES);
          tma_load_4d(smem + Cfg::V_OFF + s * Cfg::TILE_BYTES, &map_v, &vfull[s], 0, g, k0, b);
        }
      }
      // Drain copies that may still be in flight (after an abort only).
      if (!ok) {
        volatile int never = 0;
        for (uint32_t i = (it > STG ? it - STG : 0); i < it; ++i) {
          mbar_wait(&kfull[i % STG], (i / STG) & 1, &never);
          mbar_wait(&vfull[i % STG], (i / STG) & 1, &never);
        }
      }
    }
  } else if (warp == kWarpMma) {
    // ================================================================ MMA
    if (lane == 0) {
      constexpr uint32_t IDESC_S = idesc_bf16_f32(128, 128, 0, 0);
      constexpr uint32_t IDESC_O = idesc_bf16_f32(128, HD, 0, 1);
      const uint32_t q_base = smem_u32(smem + Cfg::Q_OFF);
      const uint32_t k_base = smem_u32(smem + Cfg::K_OFF);
      const uint32_t v_base = smem_u32(smem + Cfg::V_OFF);
      const uint32_t tS[2] = {tmem + Cfg::COL_S, tmem + Cfg::COL_S + 128};
      const uint32_t tP[2] = {tmem + Cfg::COL_P, tmem + Cfg::COL_P + 64};
      const uint32_t tO[2] = {tmem + Cfg::COL_O, tmem + Cfg::COL_O + 64};
      uint32_t it = 0, tcount = 0, nu = 0;
      bool ok = true;

      auto issue_s = [&](int x, uint32_t stage) {
        const uint32_t qa = q_base + x * Cfg::TILE_BYTES;
        const uint32_t ka = k_base + stage * Cfg::TILE_BYTES;
#pragma unroll
        for (int k = 0; k < HD / 16; ++k) {
          const uint64_t da = smem_desc(qa + 32 * k, 16, Cfg::ATOM, Cfg::SWZ);
          const uint64_t db = smem_desc(ka + 32 * k, 16, Cfg::ATOM, Cfg::SWZ);
          umma_ss(tS[x], da, db, IDESC_S, k > 0 ? 1u : 0u);
        }
      };
      auto issue_pv = [&](int x, uint32_t stage, bool first) {
        const uint32_t va = v_base + stage * Cfg::TILE_BYTES;
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          // 16 keys per step = two 8-row atoms of V
          const uint64_t db = smem_desc(va + k * 2 * Cfg::ATOM, 4096, Cfg::ATOM, Cfg::SWZ);
          umma_ts(tO[x], tP[x] + 8 * k, db, IDESC_O, (first && k == 0) ? 0u : 1u);
        }
      };

      for (int u = blockIdx.x; u < p.total_units && ok; u += gridDim.x, ++nu) {
        int b, g;
        int64_t i0;
        unit_coords(u, p, TOK2, b, g, i0);
        const int nt = unit_tiles(i0 + TOK2, p.W, TOK2);
        if (!mbar_wait(&bars[BQ_FULL], nu & 1, abort_flag)) { ok = false; break; }
        uint32_t s0 = it % STG;
        if (!mbar_wait(&kfull[s0], (it / STG) & 1, abort_flag)) { ok = false; break; }
        tc_fence_after();
        issue_s(0, s0);
        tc_commit(&bars[BS_A]);
        issue_s(1, s0);
        tc_commit(&bars[BS_B]);
        for (int jt = 0; jt < nt; ++jt, ++it, ++tcount) {
          const uint32_t s = it % STG;
          const uint32_t sn = (it + 1) % STG;
          // ---- tile A: O_A += P_A V, then S_A of the next tile
          if (!mbar_wait(&vfull[s], (it / STG) & 1, abort_flag)) { ok = false; break; }
          if (!mbar_wait(&bars[BP_A], tcount & 1, abort_flag)) { ok = false; break; }
          if (jt == 0 && nu > 0 && !mbar_wait(&bars[BOE_A], (nu - 1) & 1, abort_flag)) { ok = false; break; }
          tc_fence_after();
          issue_pv(0, s, jt == 0);
          tc_commit(&bars[BO_A]);
          if (jt + 1 < nt) {
            if (!mbar_wait(&kfull[sn], ((it + 1) / STG) & 1, abort_flag)) { ok = false; break; }
            tc_fence_after();
            issue_s(0, sn);
            tc_commit(&bars[BS_A]);
          }
          // ---- tile B
          if (!mbar_wait(&bars[BP_B], tcount & 1, abort_flag)) { ok = false; break; }
          if (jt == 0 && nu > 0 && !mbar_wait(&bars[BOE_B], (nu - 1) & 1, abort_flag)) { ok = false; break; }
          tc_fence_after();
          issue_pv(1, s, jt == 0);
          tc_commit(&bars[BO_B]);
          tc_commit(&kvempty[s]);
          if (jt + 1 < nt) {
            issue_s(1, sn);
            tc_commit(&bars[BS_B]);
          }
        }
        if (!ok) break;
        tc_commit(&bars[BQ_EMPTY]);  // every MMA reading this unit's Q has been issued
      }
      // Wait until every MMA issued by this thread has finished before the
      // tensor memory can be released.
      tc_commit(&bars[BMMA_DONE]);
      volatile int never = 0;
      mbar_wait(&bars[BMMA_DONE], 0, &never);
    }
  } else {
    // ============================================================ softmax
    const int x = (warp >= 4) ? 1 : 0;        // Q tile A or B
    const int wq = warp & 3;                  // TMEM lane quarter
    const int r = wq * 32 + lane;             // row of the tile
    const int tok = r / GROUP, hh = r % GROUP;
    const uint32_t lane_off = static_cast<uint32_t>(wq * 32) << 16;
    const uint32_t tS = tmem + lane_off + Cfg::COL_S + 128 * x;
    const uint32_t tP = tmem + lane_off + Cfg::COL_P + 64 * x;
    const uint32_t tO = tmem + lane_off + Cfg::COL_O + 64 * x;
    uint64_t* bar_s = &bars[BS_A + x];
    uint64_t* bar_p = &bars[BP_A + x];
    uint64_t* bar_o = &bars[BO_A + x];
    uint64_t* bar_oe = &bars[BOE_A + x];
    const float sl = p.scale_log2;
    uint32_t tcount = 0;
    bool ok = true;

    for (int u = blockIdx.x; u < p.total_units && ok; u += gridDim.x) {
      int b, g;
      int64_t i0;
      unit_coords(u, p, TOK2, b, g, i0);
      const int64_t top = i0 + TOK2;
      const int nt = unit_tiles(top, p.W, TOK2);
      const int64_t irow = i0 + TOK * x + tok;           // absolute query token of this row
      const int64_t first_tok = i0 + TOK * x, last_tok = first_tok + TOK - 1;
      float m_run = -INFINITY, l_run = 0.f;

      for (int jt = 0; jt < nt; ++jt, ++tcount) {
        const int64_t k0 = top - 128 * (jt + 1);
        const bool need_mask = (k0 + 127 > first_tok) || (k0 < last_tok - p.W + 1) || (k0 < 0);
        const bool okw = mbar_wait(bar_s, tcount & 1, abort_flag);
        if (!__all_sync(0xffffffffu, okw)) { ok = false; break; }
        tc_fence_after();
        // The whole 128-column row in four loads, one wait.
        uint32_t sr[128];
        tmem_ld32(tS, *reinterpret_cast<uint32_t(*)[32]>(&sr[0]));
        tmem_ld32(tS + 32, *reinterpret_cast<uint32_t(*)[32]>(&sr[32]));
        tmem_ld32(tS + 64, *reinterpret_cast<uint32_t(*)[32]>(&sr[64]));
        tmem_ld32(tS + 96, *reinterpret_cast<uint32_t(*)[32]>(&sr[96]));
        tc_wait_ld();
        float* s = reinterpret_cast<float*>(sr);
        if (need_mask) {
          // visible: 0 <= irow - (k0 + c) < W and k0 + c >= 0, i.e. c in [lo, hi]
          const int64_t lo64 = k0 < 0 ? -k0 : 0;
          const int64_t lw = irow - p.W + 1 - k0;
          const int lo = (int)(lo64 > lw ? lo64 : lw);
          const int hi = (int)(irow - k0);
#pragma unroll
          for (int c = 0; c < 128; ++c)
            if (c < lo || c > hi) s[c] = -INFINITY;
        }
        // Row max over 8 independent partial maxima (short dependency chains).
        float m8[8];
#pragma unroll
        for (int q = 0; q < 8; ++q) m8[q] = s[q];
#pragma unroll
        for (int c = 8; c < 128; ++c) m8[c & 7] = fmaxf(m8[c & 7], s[c]);
        const float mx = fmaxf(fmaxf(fmaxf(m8[0], m8[1]), fmaxf(m8[2], m8[3])),
                               fmaxf(fmaxf(m8[4], m8[5]), fmaxf(m8[6], m8[7])));
        const float m_tile = mx * sl;  // scale > 0
        float factor = 1.f;
        bool rescale = false;
        if (m_tile > m_run + 8.f) {  // also true when m_run = -inf and the tile has a visible key
          factor = ex2f(m_run - m_tile);  // 0 when m_run = -inf
          m_run = m_tile;
          rescale = true;
        }
        const float m_use = (m_run == -INFINITY) ? 0.f : m_run;
        // p = 2^(s·scale·log2e - m) in packed pairs; every SWA_POLY-th pair on
        // the FMA pipe, the rest on MUFU; four partial sums.
        uint32_t pk[64];
        const f2 sl2 = pk2(sl, sl), nm2 = pk2(-m_use, -m_use);
        f2 acc4[4] = {pk2(0.f, 0.f), pk2(0.f, 0.f), pk2(0.f, 0.f), pk2(0.f, 0.f)};
#pragma unroll
        for (int c = 0; c < 64; ++c) {
          const f2 xx = fma2(pk2(s[2 * c], s[2 * c + 1]), sl2, nm2);
          f2 pv;
          if (SWA_POLY > 0 && (c % (SWA_POLY > 0 ? SWA_POLY : 1)) == SWA_POLY - 1) {
            pv = ex2_poly3x2(xx);
          } else {
            const float2 xv = up2(xx);
            pv = pk2(ex2f(xv.x), ex2f(xv.y));
          }
          acc4[c & 3] = add2(acc4[c & 3], pv);
          const float2 pp = up2(pv);
          pk[c] = pack_bf16(pp.x, pp.y);
        }
        const float2 r01 = up2(add2(add2(acc4[0], acc4[1]), add2(acc4[2], acc4[3])));
        const float rs = r01.x + r01.y;
        l_run = l_run * factor + rs;
        // P_X and O_X are still read by the previous PV: wait for it.
        if (jt > 0) {
          const bool oko = mbar_wait(bar_o, (tcount - 1) & 1, abort_flag);
          if (!__all_sync(0xffffffffu, oko)) { ok = false; break; }
          tc_fence_after();
          if (rescale) {
            uint32_t o[16];
#pragma unroll
            for (int q = 0; q < HD / 16; ++q) {
              tmem_ld16(tO + 16 * q, o);
              tc_wait_ld();
#pragma unroll
              for (int c = 0; c < 16; ++c) o[c] = __float_as_uint(__uint_as_float(o[c]) * factor);
              tmem_st16(tO + 16 * q, o);
            }
          }
        }
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          uint32_t w[16];
#pragma unroll
          for (int c = 0; c < 16; ++c) w[c] = pk[16 * q + c];
          tmem_st16(tP + 16 * q, w);
        }
        tc_wait_st();
        tc_fence_before();
        mbar_arrive(bar_p);
      }
      if (!ok) break;
      // ---- epilogue: O / l  -> bf16 rows
      const bool oko = mbar_wait(bar_o, (tcount - 1) & 1, abort_flag);
      if (!__all_sync(0xffffffffu, oko)) { ok = false; break; }
      tc_fence_after();
      uint32_t o[HD];
#pragma unroll
      for (int q = 0; q < HD / 16; ++q) {
        uint32_t t16[16];
        tmem_ld16(tO + 16 * q, t16);
        tc_wait_ld();
#pragma unroll
        for (int c = 0; c < 16; ++c) o[16 * q + c] = t16[c];
      }
      tc_fence_before();
      mbar_arrive(bar_oe);  // O_X may be overwritten by the next unit
      if (irow < p.L) {
        const float inv = 1.f / l_run;
        const int h = g * GROUP + hh;
        __nv_bfloat16* dst = p.o + ((static_cast<int64_t>(b) * p.L + irow) * p.Hq + h) * HD;
#pragma unroll
        for (int c = 0; c < HD; c += 8) {
          uint4 v;
          v.x = pack_bf16(__uint_as_float(o[c + 0]) * inv, __uint_as_float(o[c + 1]) * inv);
          v.y = pack_bf16(__uint_as_float(o[c + 2]) * inv, __uint_as_float(o[c + 3]) * inv);
          v.z = pack_bf16(__uint_as_float(o[c + 4]) * inv, __uint_as_float(o[c + 5]) * inv);
          v.w = pack_bf16(__uint_as_float(o[c + 6]) * inv, __uint_as_float(o[c + 7]) * inv);
          *reinterpret_cast<uint4*>(dst + c) = v;
        }
        if (p.lse) {
          p.lse[(static_cast<int64_t>(b) * p.Hq + h) * p.L + irow] = (m_run + __log2f(l_run)) * 0.6931471805599453f;
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kWarpMma) {
    tc_fence_after();
    tmem_dealloc(tmem, Cfg::TMEM_COLS);
  }
}

}  // namespace samba

// ------------------------------------------------------------------- launcher
#include <cmath>

#include "host.hpp"

namespace samba {

int take_status_swa(cudaStream_t s) { return take_status_word(s); }

template <int HD, int GROUP>
static int launch_swa_t(const samba_swa_args& a, cudaStream_t stream) {
  constexpr int STG = 3;
  using Cfg = SwaCfg<HD, GROUP, STG>;
  auto kern = swa_fwd_kernel<HD, GROUP, STG>;
  static bool attr_done = false;
  if (!attr_done) {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg::SMEM) != cudaSuccess)
      return fail(SAMBA_ERR_CUDA, "swa: cannot set shared memory size");
    attr_done = true;
  }
  const uint64_t B = a.batch, L = a.seqlen, Hq = a.heads_q, Hkv = a.heads_kv;
  const CUtensorMapSwizzle swz =
      HD == 64 ? CU_TENSOR_MAP_SWIZZLE_128B : (HD == 32 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_32B);
  CUtensorMap mq, mk, mv;
  {
    const uint64_t dq[4] = {(uint64_t)HD, Hq, L, B};
    const uint64_t sq[3] = {HD * 2ull, Hq * HD * 2ull, L * Hq * HD * 2ull};
    const uint32_t bq[4] = {(uint32_t)HD, (uint32_t)GROUP, (uint32_t)Cfg::TOK, 1};
    int rc = encode_tiled(&mq, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, a.q, dq, sq, bq, swz, "swa q");
    if (rc) return rc;
    const uint64_t dk[4] = {(uint64_t)HD, Hkv, L, B};
    const uint64_t sk[3] = {HD * 2ull, Hkv * HD * 2ull, L * Hkv * HD * 2ull};
    const uint32_t bk[4] = {(uint32_t)HD, 1, 128, 1};
    rc = encode_tiled(&mk, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, a.k, dk, sk, bk, swz, "swa k");
    if (rc) return rc;
    rc = encode_tiled(&mv, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, a.v, dk, sk, bk, swz, "swa v");
    if (rc) return rc;
  }
  SwaParams p;
  p.o = reinterpret_cast<__nv_bfloat16*>(a.o);
  p.lse = a.lse;
  p.L = a.seqlen;
  p.W = a.window;
  p.Hq = a.heads_q;
  p.Hkv = a.heads_kv;
  p.B = (int)a.batch;
  const float scale = a.scale > 0.f ? a.scale : 1.0f / std::sqrt((float)HD);
  p.scale_log2 = scale * 1.4426950408889634f;
  p.units_per_head = (int)((a.seqlen + 2 * Cfg::TOK - 1) / (2 * Cfg::TOK));
  const int64_t total = (int64_t)p.units_per_head * a.heads_kv * a.batch;
  if (total > INT32_MAX) return fail(SAMBA_ERR_UNSUPPORTED, "samba_swa_fwd: problem too large");
  p.total_units = (int)total;
  const int grid = (int)std::min<int64_t>(total, sm_count());
  kern<<<grid, Cfg::THREADS, Cfg::SMEM, stream>>>(mq, mk, mv, p);
  return check_launch("samba_swa_fwd");
}

template <int HD>
static int launch_swa_hd(const samba_swa_args& a, cudaStream_t s) {
  switch (a.heads_q / a.heads_kv) {
    case 1: return launch_swa_t<HD, 1>(a, s);
    case 2: return launch_swa_t<HD, 2>(a, s);
    case 4: return launch_swa_t<HD, 4>(a, s);
    case 8: return launch_swa_t<HD, 8>(a, s);
    default: return launch_swa_t<HD, 16>(a, s);
  }
}

int launch_swa(const samba_swa_args& a, cudaStream_t s) {
  switch (a.head_dim) {
    case 16: return launch_swa_hd<16>(a, s);
    case 32: return launch_swa_hd<32>(a, s);
    default: return launch_swa_hd<64>(a, s);
  }
}

}  // namespace samba
