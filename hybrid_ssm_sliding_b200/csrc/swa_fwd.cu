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
//   * Warp 8 issues TMA: Q once per unit into one of two buffers (so the
//     next unit's Q lands while this one is finishing), K and V per key tile
//     into a STG-deep ring.  Warps 9 and 10 issue the tcgen05.mma of Q tiles
//     A and B (warp 9 also owns the tensor memory), each whole warp in
//     lock-step with one elected lane issuing: S = Q·Kᵀ (bf16, fp32
//     accumulate into TMEM) and O += P·V with P read straight from TMEM.
//     Over the flat sequence of key tiles (crossing unit boundaries) each
//     issues S of tile t+1 into the columns of S(t) as soon as its softmax
//     has read them, so Q·Kᵀ runs under the exps.  With one issuing warp per
//     Q tile, neither tile's MMAs wait behind the other tile's softmax, and
//     the softmax of B starts its first tile only once A has written its
//     first P, so that the two softmax warpgroups do not reach their exp
//     loops (the special-function unit) at the same time.
//   * Warps 0-3 and 4-7 are the softmax warpgroups of Q tiles A and B:
//     each thread owns one row, reads its S row from TMEM, keeps the running
//     max and sum in fp32, writes P back to TMEM as bf16 (16 packed pairs at
//     a time), and rescales O in TMEM only when the running max grows by
//     more than 2^8 (the result does not depend on the reference max; the
//     threshold only bounds P <= 256).  The exp2 of the probabilities
//     (special-function unit, with every SWA_POLY-th pair on the FMA pipe)
//     bounds this kernel.
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
  static constexpr int Q_OFF = 0;                          // two buffers of (Q_A, Q_B)
  static constexpr int K_OFF = 4 * TILE_BYTES;
  static constexpr int V_OFF = K_OFF + STG * TILE_BYTES;
  static constexpr int BAR_OFF = V_OFF + STG * TILE_BYTES;
  static constexpr int SMEM = BAR_OFF + 256 + 1024;        // + alignment slack
  static constexpr uint32_t SWZ = HD == 64 ? 2u : (HD == 32 ? 4u : 6u);  // descriptor swizzle code
  static constexpr uint32_t ATOM = 8 * ROW_BYTES;          // 8-row swizzle atom
  static constexpr int THREADS = 352;
  static constexpr uint32_t TMEM_COLS = 512;
  static constexpr uint32_t COL_S = 0, COL_P = 256, COL_O = 384;
};

// Warp roles: 0-3 softmax of Q tile A, 4-7 softmax of Q tile B (warp % 4 is
// the TMEM lane quarter a warp may access; thread i of warp w owns row
// 32 (w % 4) + i of its tile), 8 TMA producer, 9 and 10 MMA issuers of Q
// tiles A and B.
constexpr int kSoftmaxWarps = 8, kWarpTma = 8, kWarpMma = 9, kWarpMmaB = 10;

// Barrier indices inside the barrier block.  Per Q tile X in {A, B}:
// BS_X  S_X of the next key tile is in TMEM          (tcgen05.commit)
// BSF_X the softmax of X has read S_X into registers (one arrival per warp)
// BP_X  P_X is in TMEM                               (one arrival per warp)
// BO_X  O_X += P_X V has completed                   (tcgen05.commit)
// BQ_EMPTY and the K/V stages' empty barriers take one commit from each of
// the two MMA warps (count 2): a buffer is free once both tiles are done.
enum : int {
  BQ_FULL0 = 0, BQ_FULL1, BQ_EMPTY0, BQ_EMPTY1, BS_A, BS_B, BSF_A, BSF_B, BP_A, BP_B, BO_A, BO_B,
  BMMA_DONE, BMMA_DONE_B, B_STAGE0
};

__device__ __forceinline__ float ex2f(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Every SWA_POLY-th pair of probabilities is evaluated on the FMA pipe
// (0: never); the rest use the MUFU ex2.  Build-time, fixed by measurement.
#ifndef SWA_POLY
#define SWA_POLY 8
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

// max(a, b, c) in one instruction (three-input form of sm_100).
__device__ __forceinline__ float fmax3f(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
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


// Position in the flat sequence of key tiles a CTA walks through: work unit
// u (the nu-th unit of this CTA), key tile jt of the unit's nt tiles.
struct TileCursor {
  int u;
  uint32_t nu;
  int jt, nt;
};

__device__ __forceinline__ int tiles_of_unit(int u, const SwaParams& p, int tok2) {
  int b, g;
  int64_t i0;
  unit_coords(u, p, tok2, b, g, i0);
  return unit_tiles(i0 + tok2, p.W, tok2);
}

__device__ __forceinline__ bool cursor_begin(TileCursor& c, const SwaParams& p, int tok2) {
  c.u = blockIdx.x;
  c.nu = 0;
  c.jt = 0;
  if (c.u >= p.total_units) return false;
  c.nt = tiles_of_unit(c.u, p, tok2);
  return true;
}

__device__ __forceinline__ bool cursor_next(TileCursor& c, const SwaParams& p, int tok2) {
  if (++c.jt < c.nt) return true;
  c.u += gridDim.x;
  ++c.nu;
  c.jt = 0;
  if (c.u >= p.total_units) return false;
  c.nt = tiles_of_unit(c.u, p, tok2);
  return true;
}


template <int HD, int GROUP, int STG>
__global__ void __launch_bounds__(352, 1)
    swa_fwd_kernel(const __grid_constant__ CUtensorMap map_q, const __grid_constant__ CUtensorMap map_k,
                   const __grid_constant__ CUtensorMap map_v, const SwaParams p) {
  using Cfg = SwaCfg<HD, GROUP, STG>;
  static_assert((B_STAGE0 + 2 * STG) * 8 + 8 <= 256, "barrier block overflows its 256 bytes");
  static_assert(HD == 16 || HD == 32 || HD == 64, "head dim");
  constexpr int TOK = Cfg::TOK;
  constexpr int TOK2 = 2 * TOK;
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Cfg::BAR_OFF);
  uint64_t* kvfull = bars + B_STAGE0;  // K and V tile of a stage landed
  uint64_t* kvempty = kvfull + STG;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(kvempty + STG);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    mbar_init(&bars[BQ_FULL0], 1);
    mbar_init(&bars[BQ_FULL1], 1);
    mbar_init(&bars[BQ_EMPTY0], 2);
    mbar_init(&bars[BQ_EMPTY1], 2);
    mbar_init(&bars[BS_A], 1);
    mbar_init(&bars[BS_B], 1);
    mbar_init(&bars[BSF_A], kSoftmaxWarps / 2);
    mbar_init(&bars[BSF_B], kSoftmaxWarps / 2);
    mbar_init(&bars[BP_A], kSoftmaxWarps / 2);
    mbar_init(&bars[BP_B], kSoftmaxWarps / 2);
    mbar_init(&bars[BO_A], 1);
    mbar_init(&bars[BO_B], 1);
    mbar_init(&bars[BMMA_DONE], 1);
    mbar_init(&bars[BMMA_DONE + 1], 1);
    for (int s = 0; s < STG; ++s) {
      mbar_init(&kvfull[s], 1);
      mbar_init(&kvempty[s], 2);
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
        // Q of unit nu goes to buffer nu % 2 once unit nu - 2 has issued its last Q·Kᵀ.
        const uint32_t qb = nu & 1;
        if (nu >= 2 && !mbar_wait(&bars[BQ_EMPTY0 + qb], ((nu >> 1) - 1) & 1, abort_flag)) { ok = false; break; }
        unsigned char* qdst = smem + Cfg::Q_OFF + 2 * qb * Cfg::TILE_BYTES;
        mbar_arrive_expect_tx(&bars[BQ_FULL0 + qb], 2 * Cfg::TILE_BYTES);
        tma_load_4d(qdst, &map_q, &bars[BQ_FULL0 + qb], 0, g * GROUP, (int)i0, b);
        tma_load_4d(qdst + Cfg::TILE_BYTES, &map_q, &bars[BQ_FULL0 + qb], 0, g * GROUP, (int)(i0 + TOK), b);
        for (int m = 0; m < nt; ++m, ++it) {
          const int s = it % STG;
          if (it >= STG && !mbar_wait(&kvempty[s], ((it / STG) - 1) & 1, abort_flag)) { ok = false; break; }
          const int k0 = (int)(top - 128 * (m + 1));
          mbar_arrive_expect_tx(&kvfull[s], 2 * Cfg::TILE_BYTES);
          tma_load_4d(smem + Cfg::K_OFF + s * Cfg::TILE_BYTES, &map_k, &kvfull[s], 0, g, k0, b);
          tma_load_4d(smem + Cfg::V_OFF + s * Cfg::TILE_BYTES, &map_v, &kvfull[s], 0, g, k0, b);
        }
      }
      // Drain copies that may still be in flight (after an abort only).
      if (!ok) {
        volatile int never = 0;
        for (uint32_t i = (it > STG ? it - STG : 0); i < it; ++i) mbar_wait(&kvfull[i % STG], (i / STG) & 1, &never);
        for (uint32_t n = (nu > 2 ? nu - 2 : 0); n < nu; ++n) mbar_wait(&bars[BQ_FULL0 + (n & 1)], (n >> 1) & 1, &never);
      }
    }
  } else if (warp == kWarpMma || warp == kWarpMmaB) {
    // ================================================================ MMA
    // One warp per Q tile X: S_X(t+1) as soon as the softmax of X has read
    // S_X(t), then O_X += P_X(t) V(t) once P_X(t) is in TMEM.  The stage of
    // tile t is free when both warps have committed their P·V (count 2).
    const int x = warp - kWarpMma;  // Q tile A (0) or B (1)
    constexpr uint32_t IDESC_S = idesc_bf16_f32(128, 128, 0, 0);
    constexpr uint32_t IDESC_O = idesc_bf16_f32(128, HD, 0, 1);
    const uint32_t q_base = smem_u32(smem + Cfg::Q_OFF);
    const uint32_t k_base = smem_u32(smem + Cfg::K_OFF);
    const uint32_t v_base = smem_u32(smem + Cfg::V_OFF);
    bool ok = true;
    auto wait = [&](uint64_t* bar, uint32_t parity) {
      return __all_sync(0xffffffffu, mbar_wait(bar, parity, abort_flag));
    };
    // Descriptors are built once: the upper halves are constant, and the
    // start-address field of the lower half (address / 16, below 2^14 for
    // any shared-memory address) advances by 2 per 16 K-elements of Q and K
    // and by ROW_BYTES per 16 keys of V without carrying out of its field.
    const uint64_t d_q0 = smem_desc(q_base, 16, Cfg::ATOM, Cfg::SWZ);
    const uint64_t d_k0 = smem_desc(k_base, 16, Cfg::ATOM, Cfg::SWZ);
    const uint64_t d_v0 = smem_desc(v_base, 4096, Cfg::ATOM, Cfg::SWZ);
    const uint32_t hi_qk = static_cast<uint32_t>(d_q0 >> 32), hi_v = static_cast<uint32_t>(d_v0 >> 32);
    const uint32_t lo_q0 = static_cast<uint32_t>(d_q0), lo_k0 = static_cast<uint32_t>(d_k0);
    const uint32_t lo_v0 = static_cast<uint32_t>(d_v0);
    constexpr uint32_t kTileDesc = Cfg::TILE_BYTES >> 4;
    auto desc64 = [](uint32_t lo, uint32_t hi) { return (static_cast<uint64_t>(hi) << 32) | lo; };
    auto issue_s = [&](uint32_t qb, uint32_t stage) {
      const uint32_t lq = lo_q0 + (2 * qb + x) * kTileDesc;
      const uint32_t lk = lo_k0 + stage * kTileDesc;
#pragma unroll
      for (int k = 0; k < HD / 16; ++k)
        umma_ss_w(tmem + Cfg::COL_S + 128 * x, desc64(lq + 2 * k, hi_qk), desc64(lk + 2 * k, hi_qk), IDESC_S,
                  k > 0 ? 1u : 0u);
    };
    auto issue_pv = [&](uint32_t stage, bool first) {
      const uint32_t lv = lo_v0 + stage * kTileDesc;
#pragma unroll
      for (int k = 0; k < 8; ++k)  // 16 keys per step = two 8-row atoms of V
        umma_ts_w(tmem + Cfg::COL_O + 64 * x, tmem + Cfg::COL_P + 64 * x + 8 * k,
                  desc64(lv + k * (Cfg::ROW_BYTES), hi_v), IDESC_O, (first && k == 0) ? 0u : 1u);
    };
    uint64_t* bar_s = &bars[BS_A + x];
    uint64_t* bar_sf = &bars[BSF_A + x];
    uint64_t* bar_p = &bars[BP_A + x];
    uint64_t* bar_o = &bars[BO_A + x];
    TileCursor cs;  // tile t
    bool more = cursor_begin(cs, p, TOK2);
    bool first_cur = true;
    if (more) {
      ok = wait(&bars[BQ_FULL0], 0) && wait(&kvfull[0], 0);
      if (ok) {
        tc_fence_after();
        issue_s(0, 0);
        tc_commit_w(bar_s);
        if (cs.nt == 1) tc_commit_w(&bars[BQ_EMPTY0]);
      }
    }
    for (uint32_t t = 0; more && ok; ++t) {
      TileCursor cn = cs;  // tile t + 1
      const bool has_next = cursor_next(cn, p, TOK2);
      const bool first_next = has_next && cn.jt == 0;
      const uint32_t s = t % STG, sn = (t + 1) % STG;
      const uint32_t qbn = cn.nu & 1;
      auto next_s = [&]() {  // S of tile t + 1, once its K/V (and Q) landed and S(t) was read
        if (first_next && !wait(&bars[BQ_FULL0 + qbn], (cn.nu >> 1) & 1)) return false;
        if (!wait(&kvfull[sn], ((t + 1) / STG) & 1)) return false;
        if (!wait(bar_sf, t & 1)) return false;
        tc_fence_after();
        issue_s(qbn, sn);
        tc_commit_w(bar_s);
        if (cn.jt == cn.nt - 1) tc_commit_w(&bars[BQ_EMPTY0 + qbn]);
        return true;
      };
      auto this_pv = [&]() {  // O += P(t) V(t) once P(t) is in TMEM; then stage s is free
        if (!wait(bar_p, t & 1)) return false;
        tc_fence_after();
        issue_pv(s, first_cur);
        tc_commit_w(bar_o);
        tc_commit_w(&kvempty[s]);
        return true;
      };
      // S(t+1) goes first, so that Q·Kᵀ runs under the softmax of tile t.
      ok = (!has_next || next_s()) && this_pv();
      if (!ok) break;
      first_cur = first_next;
      cs = cn;
      more = has_next;
    }
    // Wait until every MMA issued by this warp has finished before the
    // tensor memory can be released.
    tc_commit_w(&bars[BMMA_DONE + x]);
    volatile int never = 0;
    mbar_wait(&bars[BMMA_DONE + x], 0, &never);
  } else if (warp < kSoftmaxWarps) {
    // ============================================================ softmax
    const int x = warp >> 2;                  // Q tile A or B
    const int wq = warp & 3;                  // TMEM lane quarter
    const int r = wq * 32 + lane;             // row of the tile
    const int tok = r / GROUP, hh = r % GROUP;
    const uint32_t lane_off = static_cast<uint32_t>(wq * 32) << 16;
    const uint32_t tS = tmem + lane_off + Cfg::COL_S + 128 * x;
    const uint32_t tP = tmem + lane_off + Cfg::COL_P + 64 * x;
    const uint32_t tO = tmem + lane_off + Cfg::COL_O + 64 * x;
    uint64_t* bar_s = &bars[BS_A + x];
    uint64_t* bar_sf = &bars[BSF_A + x];
    uint64_t* bar_p = &bars[BP_A + x];
    uint64_t* bar_o = &bars[BO_A + x];
    const float sl = p.scale_log2;
    uint32_t t = 0;  // flat key-tile index
    bool ok = true;
    auto wait = [&](uint64_t* bar, uint32_t parity) {
      return __all_sync(0xffffffffu, mbar_wait(bar, parity, abort_flag));
    };
    // One arrival per warp: the tcgen05 loads and stores before it are
    // warp-collective and complete in every lane, so after the warp has
    // converged one lane signals for all of them.
    auto warp_arrive = [&](uint64_t* bar) {
      __syncwarp();
      if (lane == 0) mbar_arrive(bar);
    };

    // Tile B starts once tile A has written its first P (see the header).
    if (x == 1 && (int)blockIdx.x < p.total_units) ok = wait(&bars[BP_A], 0);
    for (int u = blockIdx.x; u < p.total_units && ok; u += gridDim.x) {
      int b, g;
      int64_t i0;
      unit_coords(u, p, TOK2, b, g, i0);
      const int64_t top = i0 + TOK2;
      const int nt = unit_tiles(top, p.W, TOK2);
      const int64_t irow = i0 + TOK * x + tok;           // absolute query token of this row
      const int64_t first_tok = i0 + TOK * x, last_tok = first_tok + TOK - 1;
      float m_run = -INFINITY, l_run = 0.f;

      for (int jt = 0; jt < nt; ++jt, ++t) {
        const int64_t k0 = top - 128 * (jt + 1);
        const bool need_mask = (k0 + 127 > first_tok) || (k0 < last_tok - p.W + 1) || (k0 < 0);
        if (!wait(bar_s, t & 1)) { ok = false; break; }
        tc_fence_after();
        // The whole 128-column row in four loads, one wait.
        uint32_t sr[128];
        tmem_ld32(tS, *reinterpret_cast<uint32_t(*)[32]>(&sr[0]));
        tmem_ld32(tS + 32, *reinterpret_cast<uint32_t(*)[32]>(&sr[32]));
        tmem_ld32(tS + 64, *reinterpret_cast<uint32_t(*)[32]>(&sr[64]));
        tmem_ld32(tS + 96, *reinterpret_cast<uint32_t(*)[32]>(&sr[96]));
        tc_wait_ld();
        tc_fence_before();
        warp_arrive(bar_sf);  // S_X may now be overwritten by the next tile's Q·Kᵀ
        float* sc = reinterpret_cast<float*>(sr);
        if (need_mask) {
          // visible: 0 <= irow - (k0 + c) < W and k0 + c >= 0, i.e. c in [lo, hi]
          const int64_t lo64 = k0 < 0 ? -k0 : 0;
          const int64_t lw = irow - p.W + 1 - k0;
          const int lo = (int)(lo64 > lw ? lo64 : lw);
          const int hi = (int)(irow - k0);
          // Branch-free: one unsigned compare and one select per column
          // (c - lo wraps to a large value for c < lo).  A row that sees no
          // key of this tile (hi < lo: the tile lies in its future, or below
          // its window) gets an empty interval.
          const int span_i = hi - lo;
          const unsigned span = span_i < 0 ? 0u : static_cast<unsigned>(span_i);
          const int lo_e = span_i < 0 ? (1 << 20) : lo;
#pragma unroll
          for (int c = 0; c < 128; ++c) sc[c] = ((unsigned)(c - lo_e) <= span) ? sc[c] : -INFINITY;
        }
        // Row max: eight chains of three-input maxima, chain q over the
        // columns c = q (mod 8).
        float m8[8];
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          float m = fmax3f(sc[q], sc[q + 8], sc[q + 16]);
#pragma unroll
          for (int c = 24; c < 120; c += 16) m = fmax3f(m, sc[c + q], sc[c + 8 + q]);
          m8[q] = fmaxf(m, sc[120 + q]);
        }
        const float mx = fmaxf(fmax3f(fmax3f(m8[0], m8[1], m8[2]), fmax3f(m8[3], m8[4], m8[5]), m8[6]), m8[7]);
        const float m_tile = mx * sl;  // scale > 0
        float factor = 1.f;
        bool rescale = false;
        if (m_tile > m_run + 8.f) {  // also true when m_run = -inf and the tile has a visible key
          factor = ex2f(m_run - m_tile);  // 0 when m_run = -inf
          m_run = m_tile;
          rescale = true;
        }
        const float m_use = (m_run == -INFINITY) ? 0.f : m_run;
        // P_X and O_X are still read by the previous O += P·V of this unit:
        // wait for it before P is overwritten.  At the first tile of a unit
        // the epilogue of the previous unit has already waited for it.
        if (jt > 0) {
          if (!wait(bar_o, (t - 1) & 1)) { ok = false; break; }
          tc_fence_after();
        }
        // p = 2^(s·scale·log2e - m) in packed pairs; every SWA_POLY-th pair on
        // the FMA pipe, the rest on MUFU; four partial sums; each 16 packed
        // pairs go to TMEM as soon as they are ready.
        const f2 sl2 = pk2(sl, sl), nm2 = pk2(-m_use, -m_use);
        f2 acc4[4] = {pk2(0.f, 0.f), pk2(0.f, 0.f), pk2(0.f, 0.f), pk2(0.f, 0.f)};
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          uint32_t pk[16];
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            const int c = 16 * k + j;
            const f2 xx = fma2(pk2(sc[2 * c], sc[2 * c + 1]), sl2, nm2);
            f2 pv;
            if (SWA_POLY > 0 && (c % (SWA_POLY > 0 ? SWA_POLY : 1)) == SWA_POLY - 1) {
              pv = ex2_poly3x2(xx);
            } else {
              const float2 xv = up2(xx);
              pv = pk2(ex2f(xv.x), ex2f(xv.y));
            }
            acc4[c & 3] = add2(acc4[c & 3], pv);
            const float2 pp = up2(pv);
            pk[j] = pack_bf16(pp.x, pp.y);
          }
          tmem_st16(tP + 16 * k, pk);
        }
        const float2 r01 = up2(add2(add2(acc4[0], acc4[1]), add2(acc4[2], acc4[3])));
        l_run = l_run * factor + (r01.x + r01.y);
        if (jt > 0 && rescale) {
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
        tc_wait_st();
        tc_fence_before();
        warp_arrive(bar_p);  // also tells the MMA warp that O_X has been read, if this starts a unit
      }
      if (!ok) break;
      // ---- epilogue: O / l  -> bf16 rows
      if (!wait(bar_o, (t - 1) & 1)) { ok = false; break; }
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
      if (irow < p.L && SAMBA_CHECK(b < p.B && irow >= 0 && g * GROUP + hh < p.Hq)) {
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

// K/V ring depth (stages of one K and one V tile each); build-time.
#ifndef SWA_STAGES
#define SWA_STAGES 5
#endif

template <int HD, int GROUP>
static int launch_swa_t(const samba_swa_args& a, cudaStream_t stream) {
  constexpr int STG = SWA_STAGES;
  using Cfg = SwaCfg<HD, GROUP, STG>;
  auto kern = swa_fwd_kernel<HD, GROUP, STG>;
  static PerDeviceOnce attr;
  const int arc = once_per_device(attr, [&] {
    return cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg::SMEM) == cudaSuccess
               ? SAMBA_OK
               : fail(SAMBA_ERR_CUDA, "swa: cannot set shared memory size");
  });
  if (arc != SAMBA_OK) return arc;
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
