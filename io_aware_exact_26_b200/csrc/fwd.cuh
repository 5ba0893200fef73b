// Forward exact attention for sm_100a: O = softmax(scale * Q K^T) V and LSE.
//
// Method (page "attention 的显存线性化" §三; page "attn-efficient", online-softmax
// section): Q is cut into 128-row tiles and K/V into 128-key tiles; for each
// query tile the key tiles stream through shared memory, S_ij = Q_i K_j^T is
// formed on chip, a running row max m and exp-sum l are updated, the partial
// output is rescaled by exp(m_old - m_new) when the max grows, and only O and the
// log-sum-exp leave the chip.  S and P never reach HBM.
//
// B200 mapping (one persistent CTA per SM, 608 threads = 19 warps):
//   warps 0-15 softmax: group k = warp / 4 (k = 0..3) owns keys [32k, 32k+32) of
//              every S tile and O columns [k*D/4, (k+1)*D/4); thread = one query
//              row = one TMEM lane (warp w reaches lanes 32*(w%4)..+31).  The four
//              warps that share a row quadrant sit on the same SM sub-partition,
//              so each sub-partition runs four softmax warps, enough to keep its
//              MUFU pipe busy.  The groups exchange partial row maxima through
//              shared memory once per tile (so all take the same rescale
//              decisions) and partial row sums once per query tile.
//   warp 16    TMA producer for Q (double buffered) and the K ring
//   warp 17    MMA issuer: S = Q K^T (SS, both K-major) and O += P V (A = P from
//              TMEM, B = V MN-major), accumulating in TMEM.
//   warp 18    TMA producer for the V ring (its own stream, so a K load never
//              queues behind a V load that waits for a free stage)
// TMEM (512 columns): three 128-column S/P buffers, then O (D columns).  Three
// S buffers let S(j+2) be issued while P(j-1) may still be read by its PV MMA.
// P(j) (bf16) is written over the S buffer: group k's 32 keys go to columns
// 32k..32k+15, inside its own S columns, so no group overwrites scores another
// group still reads.
//
// exp2 with a folded scale: c = scale * log2(e), p = exp2(s*c - m) where m is
// kept in log2 units; LSE = ln(2) * (m + log2 l).  The max used for the
// exponent is allowed to be stale by up to kRescaleTau (log2 units): by shift
// invariance of softmax (page "attn-efficient": subtracting the same number from
// a whole score row leaves the result unchanged) any reference value works as
// long as O and l use the same one; this keeps p <= 2^tau and skips most O
// rescales.  l is the fp32 sum of the p that are rounded to bf16 for the PV MMA.
#pragma once
#include "sm100.cuh"

namespace attn {

constexpr float kRescaleTau = 8.0f;

template <int D>
struct FwdCfg {
  static constexpr int kTile = 128 * D * 2;          // bytes of one 128 x D bf16 tile
  static constexpr int kBox = 128 * 128;             // bytes of one 128 x 64 swizzled box
  static constexpr int KST = 3;                      // K ring stages (== S buffers: S(g) frees stage g % 3)
  static constexpr int VST = (D == 128) ? 2 : 3;     // V ring stages (<= 3, see FwdShared::pv_done)
  static_assert(VST <= 3, "the V producer's waits on pv_done need VST <= 3");
  static constexpr int kGroups = 4;                  // softmax groups of 4 warps
  // Of every 8 score pairs, how many are exponentiated on the FMA pipe instead of
  // MUFU (16 ex2 per SM per clock, so one exp per score costs as much MUFU time as
  // the d = 128 tile's two MMAs).  Measured on B200 with four softmax warps per
  // sub-partition: 0 is fastest or within noise of 1-3 at d = 64 and d = 128, so
  // the issue slots the polynomial takes cost more than the MUFU time it saves.
  static constexpr int kFmaPairs = 0;
  static constexpr int kThreads = 608;
  static constexpr int kTmemCols = 512;
  static constexpr int kOCol = 384;                  // O accumulator column
  static constexpr int kOffQ = 0;                    // 2 tiles
  static constexpr int kOffK = 2 * kTile;
  static constexpr int kOffV = kOffK + KST * kTile;
  static constexpr int kOffSh = kOffV + VST * kTile; // FwdShared
  static constexpr int kLayout = kOffSh + 2560;
  // the d = 128 layout leaves no room for alignment slack under the 227 KB limit;
  // the kernel checks the base alignment at run time
  static constexpr int kSmem = (kLayout + 1024 <= 232448) ? kLayout + 1024 : kLayout;
};

struct FwdParams {
  void* o;
  float* lse;
  int B, Hq, Hkv, N, G;
  int n_qtiles, total_tiles;
  float c;          // scale * log2(e)
  int causal;
};

struct FwdShared {
  // Partial row maxima of tile g: xmax[g & 1][group][row], as bf16 rounded
  // upward (the common maximum is only the exponent's reference point, and any
  // value at or above the true maximum works).  Once every group has finished
  // its last tile of a query tile, the same bytes carry the partial row sums.
  union {
    uint16_t xmax[2][4][128];
    float xsum[4][128];
  } x;
  uint64_t q_full[2], q_empty[2];
  uint64_t k_full[3];        // K(g) landed in stage g % 3 (the stage is free again once S(g) completes)
  uint64_t v_full[3];        // V(g) landed in stage g % VST
  uint64_t s_full[3];        // S(g) complete in buffer g % 3; K stage g % 3 free
  uint64_t p_ready[3];       // P(g) written over buffer g % 3 by both groups
  // PV(g) complete (P(g) consumed, and V(g) read) on pv_done[g % 3].  Every wait
  // on it targets a PV whose successor on the same barrier, PV(g + 3), cannot
  // have completed yet: it needs P(g + 3), or for the V producer (VST <= 3)
  // V(g + 3 - VST), which that producer has not loaded.  So a parity wait never
  // sees the barrier two phases ahead.
  uint64_t pv_done[3];
  uint64_t xbar[2];          // both groups posted their maxima for a tile
  uint64_t ebar;             // every group is done with the maxima of a query tile
  uint64_t sbar;             // every group posted its sum for a query tile
  uint64_t sread;            // every group read the sums (the bytes may be reused)
  uint64_t o_free;
  uint64_t drain;
  uint64_t teardown;         // every warp is done with TMEM
  uint32_t tmem_base;
};
static_assert(sizeof(FwdShared) <= 2560, "FwdShared does not fit its slot");

// Work tile t -> (query tile, batch*head).  Tiles are numbered KV head by KV
// head (the G query heads of a group interleaved), so the CTAs that run at the
// same time read the same K/V and it is fetched from HBM about once; inside a
// group, causal tiles go longest first.
__device__ __forceinline__ void fwd_tile_coords(const FwdParams& p, int t, int& qt, int& bh) {
  const int per_group = p.G * p.n_qtiles;
  const int gk = t / per_group;                  // b * Hkv + kv-head
  const int r = t - gk * per_group;
  const int rq = r / p.G;
  const int hin = r - rq * p.G;
  qt = p.causal ? (p.n_qtiles - 1 - rq) : rq;
  bh = (gk / p.Hkv) * p.Hq + (gk % p.Hkv) * p.G + hin;
}

__device__ __forceinline__ int fwd_n_kv(const FwdParams& p, int qt) {
  int n_kv_all = (p.N + 127) / 128;
  return p.causal ? (qt + 1) : n_kv_all;
}

template <int D>
__global__ void __launch_bounds__(608, 1)
    attn_fwd_kernel(const __grid_constant__ CUtensorMap tmq, const __grid_constant__ CUtensorMap tmk,
                    const __grid_constant__ CUtensorMap tmv, const FwdParams p) {
  using C = FwdCfg<D>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  if (static_cast<int>(smem - smem_raw) + C::kLayout > C::kSmem) {
    // the 128B-swizzled tiles need a 1024-byte aligned base that this launch cannot give
    if (threadIdx.x == 0) record_error(&g_attn_status, 3);
    return;
  }
  FwdShared& sh = *reinterpret_cast<FwdShared*>(smem + C::kOffSh);
  uint8_t* sQ = smem + C::kOffQ;                   // 2 tiles
  uint8_t* sK = smem + C::kOffK;                   // KST tiles
  uint8_t* sV = smem + C::kOffV;                   // VST tiles

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int i = 0; i < 2; ++i) { mbar_init(&sh.q_full[i], 1); mbar_init(&sh.q_empty[i], 1); }
    for (int i = 0; i < C::VST; ++i) mbar_init(&sh.v_full[i], 1);
    for (int i = 0; i < 3; ++i) {
      mbar_init(&sh.pv_done[i], 1);
      mbar_init(&sh.k_full[i], 1);
      mbar_init(&sh.s_full[i], 1);
      mbar_init(&sh.p_ready[i], 16);
    }
    mbar_init(&sh.xbar[0], 16);
    mbar_init(&sh.xbar[1], 16);
    mbar_init(&sh.ebar, 16);
    mbar_init(&sh.sbar, 16);
    mbar_init(&sh.sread, 16);
    mbar_init(&sh.o_free, 16);
    mbar_init(&sh.drain, 1);
    mbar_init(&sh.teardown, 19);
    fence_barrier_init();
  }
  if (warp == 0) { tmem_alloc(&sh.tmem_base, C::kTmemCols); tmem_relinquish(); }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sh.tmem_base;

  if (warp == 16) {
    // ------------------------------------------------------------ TMA producer: Q and K
    if (lane == 0) {
      tma_prefetch_desc(&tmq); tma_prefetch_desc(&tmk);
      int it = 0, tl = 0, nk = 0, nq = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < p.total_tiles && ok; t += gridDim.x, ++tl) {
        int qt, bh;
        fwd_tile_coords(p, t, qt, bh);
        const int n_kv = fwd_n_kv(p, qt);
        const int bkv = (bh / p.Hq) * p.Hkv + (bh % p.Hq) / p.G;
        const int qb = tl & 1;
        if (tl >= 2) ok = mbar_wait(&sh.q_empty[qb], ((tl >> 1) - 1) & 1);
        if (!ok) break;
        mbar_arrive_expect_tx(&sh.q_full[qb], C::kTile);
        for (int c = 0; c < D / 64; ++c)
          tma_load_3d(sQ + qb * C::kTile + c * C::kBox, &tmq, &sh.q_full[qb], c * 64, qt * 128, bh);
        nq = tl + 1;
        for (int s = 0; s < n_kv && ok; ++s) {
          const int g = it + s, st = g % C::KST;
          if (g >= C::KST) ok = mbar_wait(&sh.s_full[st], ((g / C::KST) - 1) & 1);   // S(g - 3) read K
          if (!ok) break;
          mbar_arrive_expect_tx(&sh.k_full[st], C::kTile);
          for (int c = 0; c < D / 64; ++c)
            tma_load_3d(sK + st * C::kTile + c * C::kBox, &tmk, &sh.k_full[st], c * 64, s * 128, bkv);
          nk = g + 1;
        }
        it += n_kv;
      }
      if (!ok) {
        // Let the copies already in flight land before the CTA exits (bounded).
        for (int g = max(0, nk - C::KST); g < nk; ++g) mbar_drain_wait(&sh.k_full[g % C::KST], (g / C::KST) & 1);
        for (int g = max(0, nq - 2); g < nq; ++g) mbar_drain_wait(&sh.q_full[g & 1], (g >> 1) & 1);
      }
    }
  } else if (warp == 18) {
    // ------------------------------------------------------------ TMA producer: V
    if (lane == 0) {
      tma_prefetch_desc(&tmv);
      int it = 0, nv = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < p.total_tiles && ok; t += gridDim.x) {
        int qt, bh;
        fwd_tile_coords(p, t, qt, bh);
        const int n_kv = fwd_n_kv(p, qt);
        const int bkv = (bh / p.Hq) * p.Hkv + (bh % p.Hq) / p.G;
        for (int s = 0; s < n_kv && ok; ++s) {
          const int g = it + s, st = g % C::VST;
          if (g >= C::VST) {                                  // PV(g - VST) read stage st
            const int gp = g - C::VST;
            ok = mbar_wait(&sh.pv_done[gp % 3], (gp / 3) & 1);
          }
          if (!ok) break;
          mbar_arrive_expect_tx(&sh.v_full[st], C::kTile);
          for (int c = 0; c < D / 64; ++c)
            tma_load_3d(sV + st * C::kTile + c * C::kBox, &tmv, &sh.v_full[st], c * 64, s * 128, bkv);
          nv = g + 1;
        }
        it += n_kv;
      }
      if (!ok)
        for (int g = max(0, nv - C::VST); g < nv; ++g) mbar_drain_wait(&sh.v_full[g % C::VST], (g / C::VST) & 1);
    }
  } else if (warp == 17) {
    // ------------------------------------------------------------ MMA issuer
    // The whole warp follows the schedule (so descriptor arithmetic stays
    // warp-uniform); one lane, elected once, issues every MMA and commit, so its
    // final commit covers all of them.
    const bool leader = elect_one();
    constexpr uint32_t idS = idesc_bf16_f32(128, 128, false, false);
    constexpr uint32_t idO = idesc_bf16_f32(128, D, false, true);
    constexpr uint32_t hi = sdesc_hi_sw128(1024);
    const uint32_t q_lo0 = sdesc_lo(smem_u32(sQ), 16);
    const uint32_t k_lo0 = sdesc_lo(smem_u32(sK), 16);
    const uint32_t v_lo0 = sdesc_lo(smem_u32(sV), C::kBox);
    auto wait = [&](uint64_t* bar, uint32_t parity) -> bool {
      return __all_sync(0xffffffffu, mbar_wait(bar, parity));
    };
    int it = 0, tl = 0;
    bool ok = true;
    for (int t = blockIdx.x; t < p.total_tiles && ok; t += gridDim.x, ++tl) {
      int qt, bh;
      fwd_tile_coords(p, t, qt, bh);
      const int n_kv = fwd_n_kv(p, qt);
      const int qb = tl & 1;
      ok = wait(&sh.q_full[qb], (tl >> 1) & 1);
      if (!ok) break;
      tc_fence_after();
      const uint32_t q_lo = q_lo0 + qb * (C::kTile >> 4);
      // S(g) = Q K(g)^T into S buffer g % 3 (the buffer last held P(g - 3))
      auto issue_s = [&](int j) -> bool {
        const int g = it + j, sb = g % 3;
        if (!wait(&sh.k_full[sb], (g / 3) & 1)) return false;
        if (g >= 3 && !wait(&sh.pv_done[sb], ((g - 3) / 3) & 1)) return false;   // P(g - 3) consumed
        tc_fence_after();
        const uint32_t k_lo = k_lo0 + sb * (C::kTile >> 4);
        if (leader) {
#pragma unroll
          for (int k = 0; k < D / 16; ++k) {
            const uint32_t off = ((k >> 2) * C::kBox + (k & 3) * 32) >> 4;
            umma_ss_lo(tmem + sb * 128, q_lo + off, k_lo + off, hi, idS, k > 0);
          }
          umma_commit(&sh.s_full[sb]);
          if (j == n_kv - 1) umma_commit(&sh.q_empty[qb]);
        }
        __syncwarp();
        return true;
      };
      // S runs two tiles ahead of PV, so the softmax groups can load S(j+1) while
      // they exponentiate tile j.
      ok = issue_s(0) && (n_kv < 2 || issue_s(1));
      for (int j = 0; j < n_kv && ok; ++j) {
        if (j + 2 < n_kv && !issue_s(j + 2)) { ok = false; break; }
        // O (+)= P(g) V(g); keys 16kk..16kk+15 of P sit at column 32*(kk/2) + 8*(kk%2)
        const int g = it + j, vst = g % C::VST, sb = g % 3;
        ok = wait(&sh.v_full[vst], (g / C::VST) & 1) && wait(&sh.p_ready[sb], (g / 3) & 1);
        if (ok && j == 0 && tl >= 1) ok = wait(&sh.o_free, (tl - 1) & 1);
        if (!ok) break;
        tc_fence_after();
        const uint32_t v_lo = v_lo0 + vst * (C::kTile >> 4);
        if (leader) {
#pragma unroll
          for (int k = 0; k < 8; ++k)
            umma_ts_lo(tmem + C::kOCol, tmem + sb * 128 + (k >> 1) * 32 + (k & 1) * 8, v_lo + ((k * 2048) >> 4), hi,
                       idO, (j > 0 || k > 0));
          umma_commit(&sh.pv_done[sb]);
        }
        __syncwarp();
      }
      it += n_kv;
    }
    // Drain every MMA this warp issued before TMEM is released.
    if (leader) {
      umma_commit(&sh.drain);
      mbar_wait(&sh.drain, 0);
    }
    __syncwarp();
  } else if (warp < 16) {
    // ------------------------------------------------------------ softmax groups
    const int grp = warp >> 2;                                  // keys [32 grp, 32 grp + 32)
    const int quad = warp & 3;
    const int row = quad * 32 + lane;                           // TMEM lane == tile row
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(quad * 32) << 16);
    constexpr int OQ = D / 4;                                   // O columns per group
    const uint32_t o_base = lane_base + C::kOCol + grp * OQ;
    const float c = p.c;
    const uint64_t c2 = f2pack(c, c);
    int it = 0, tl = 0;
    bool ok = true;
    for (int t = blockIdx.x; t < p.total_tiles && ok; t += gridDim.x, ++tl) {
      int qt, bh;
      fwd_tile_coords(p, t, qt, bh);
      const int n_kv = fwd_n_kv(p, qt);
      const int qrow = qt * 128 + row;
      float m_used = -INFINITY;
      uint64_t lsum = f2pack(0.f, 0.f);                         // two partial sums
      // last visible key of this row within this group's 32 columns of tile j
      auto last_col = [&](int j) -> int {
        const int kbase = j * 128 + grp * 32;
        const int lim = p.N - 1 - kbase;
        return p.causal ? min(lim, qrow - kbase) : lim;
      };
      auto mask16 = [&](uint32_t (&r)[16], int col0, int lim) {
#pragma unroll
        for (int k = 0; k < 16; ++k)
          if (col0 + k > lim) r[k] = 0xff800000u;
      };
      auto max16 = [&](float (&mx4)[4], const uint32_t (&r)[16]) {
#pragma unroll
        for (int k = 0; k < 16; k += 8) {
#pragma unroll
          for (int e = 0; e < 4; ++e)
            mx4[e] = max3f(mx4[e], __uint_as_float(r[k + e]), __uint_as_float(r[k + e + 4]));
        }
      };
      // post this group's partial max of tile j for the other groups
      auto post = [&](int j, const float (&mx4)[4]) -> bool {
        const int g = it + j, xp = g & 1;
        const float pm = fmaxf(fmaxf(mx4[0], mx4[1]), fmaxf(mx4[2], mx4[3]));
        if (j == 0 && tl >= 1) {       // the previous query tile's sums used these bytes
          if (!__all_sync(0xffffffffu, mbar_wait(&sh.sread, (tl - 1) & 1))) return false;
        }
        sh.x.xmax[xp][grp][row] = bf16_bits_round_up(pm);
        __syncwarp();
        if (lane == 0) mbar_arrive(&sh.xbar[xp]);
        return true;
      };
      // tile 0's maximum, before the pipelined loop
      {
        const int g = it, sb = g % 3;
        ok = __all_sync(0xffffffffu, mbar_wait(&sh.s_full[sb], (g / 3) & 1));
        if (!ok) break;
        tc_fence_after();
        const int lim = last_col(0);
        const bool msk = __any_sync(0xffffffffu, lim < 31);
        float mx4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
        uint32_t r0[16], r1[16];
        tmem_ld16(lane_base + sb * 128 + grp * 32, r0);
        tmem_ld16(lane_base + sb * 128 + grp * 32 + 16, r1);
        tmem_wait_ld();
        reg_fence(r0);
        reg_fence(r1);
        if (msk) { mask16(r0, 0, lim); mask16(r1, 16, lim); }
        max16(mx4, r0);
        max16(mx4, r1);
        ok = post(0, mx4);
        if (!ok) break;
      }
      // Tile j: (1) take the common max of tile j; (2) read this group's columns of
      // tile j+1 and post their max at once, so the other groups find it long before
      // they need it and the groups can drift apart by most of a tile (one group's
      // waits then overlap another's exponentials); (3) exponentiate tile j in two
      // chunks of 16 columns, write P; (4) rescale this group's O columns if the max
      // moved, hand P to the MMA warp.  A group posts j+1 only after it has read the
      // maxima of j, and reaches j only once every group has posted j, i.e. has read
      // j-1: so two parity slots suffice.
      for (int j = 0; j < n_kv && ok; ++j) {
        const int g = it + j, sb = g % 3, xp = g & 1;
        ok = __all_sync(0xffffffffu, mbar_wait(&sh.xbar[xp], (g >> 1) & 1));
        if (!ok) break;
        const float m_tile = fmaxf(fmaxf(bf16_bits_to_float(sh.x.xmax[xp][0][row]), bf16_bits_to_float(sh.x.xmax[xp][1][row])),
                                   fmaxf(bf16_bits_to_float(sh.x.xmax[xp][2][row]), bf16_bits_to_float(sh.x.xmax[xp][3][row]))) * c;
        float alpha = 1.f;
        const bool need = (m_used == -INFINITY) || (m_tile > m_used + kRescaleTau);
        if (need) {
          const float m_new = fmaxf(m_used, m_tile);
          alpha = (m_used == -INFINITY) ? 0.f : ex2_approx(m_used - m_new);
          float l0, l1;
          f2unpack(lsum, l0, l1);
          lsum = f2pack(l0 * alpha, l1 * alpha);
          m_used = m_new;
        }
        if (j + 1 < n_kv) {
          const int sbn = (g + 1) % 3;
          ok = __all_sync(0xffffffffu, mbar_wait(&sh.s_full[sbn], ((g + 1) / 3) & 1));
          if (!ok) break;
          tc_fence_after();
          const int limn = last_col(j + 1);
          const bool mskn = __any_sync(0xffffffffu, limn < 31);
          uint32_t rn0[16], rn1[16];
          tmem_ld16(lane_base + sbn * 128 + grp * 32, rn0);
          tmem_ld16(lane_base + sbn * 128 + grp * 32 + 16, rn1);
          tmem_wait_ld();
          reg_fence(rn0);
          reg_fence(rn1);
          if (mskn) { mask16(rn0, 0, limn); mask16(rn1, 16, limn); }
          float mx4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
          max16(mx4, rn0);
          max16(mx4, rn1);
          ok = post(j + 1, mx4);
          if (!ok) break;
        }
        const int lim = last_col(j);
        const bool msk = __any_sync(0xffffffffu, lim < 31);
        const uint64_t nm2 = f2pack(-m_used, -m_used);
        const uint32_t s_col = lane_base + sb * 128 + grp * 32;
#pragma unroll
        for (int cc = 0; cc < 2; ++cc) {
          uint32_t r[16];
          tmem_ld16(s_col + cc * 16, r);
          tmem_wait_ld();
          reg_fence(r);
          if (msk) mask16(r, cc * 16, lim);
          uint32_t pk[8];
#pragma unroll
          for (int k = 0; k < 8; ++k) {
            const uint64_t x = ffma2(f2pack(__uint_as_float(r[2 * k]), __uint_as_float(r[2 * k + 1])), c2, nm2);
            float x0, x1, a, b;
            f2unpack(x, x0, x1);
            if (k >= 8 - C::kFmaPairs) {
              exp2_fma_pair(x0, x1, a, b);
            } else {
              a = ex2_approx(x0);
              b = ex2_approx(x1);
            }
            lsum = fadd2(lsum, f2pack(a, b));
            pk[k] = pack_bf16x2(a, b);
          }
          tmem_st8(s_col + cc * 8, pk);
        }
        // Rescale this group's columns of the running output when its max moved.
        if (__any_sync(0xffffffffu, need && j > 0)) {
          const int gp = g - 1;
          ok = __all_sync(0xffffffffu, mbar_wait(&sh.pv_done[gp % 3], (gp / 3) & 1));
          if (!ok) break;
          tc_fence_after();
          if constexpr (OQ == 32) {
            uint32_t o[32];
            tmem_ld32(o_base, o);
            tmem_wait_ld();
            reg_fence(o);
#pragma unroll
            for (int k = 0; k < 32; ++k) o[k] = __float_as_uint(__uint_as_float(o[k]) * alpha);
            tmem_st32(o_base, o);
          } else {
            uint32_t o[16];
            tmem_ld16(o_base, o);
            tmem_wait_ld();
            reg_fence(o);
#pragma unroll
            for (int k = 0; k < 16; ++k) o[k] = __float_as_uint(__uint_as_float(o[k]) * alpha);
            tmem_st16(o_base, o);
          }
        }
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&sh.p_ready[sb]);
      }
      if (!ok) break;
      // epilogue: combine the partial sums, wait for the last PV, O / l -> bf16, LSE
      const int glast = it + n_kv - 1;
      if (lane == 0) mbar_arrive(&sh.ebar);                    // done reading this tile's maxima
      ok = __all_sync(0xffffffffu, mbar_wait(&sh.ebar, tl & 1));
      if (!ok) break;
      float l0, l1;
      f2unpack(lsum, l0, l1);
      sh.x.xsum[grp][row] = l0 + l1;
      __syncwarp();
      if (lane == 0) mbar_arrive(&sh.sbar);
      ok = __all_sync(0xffffffffu, mbar_wait(&sh.sbar, tl & 1));
      if (!ok) break;
      const float l = (sh.x.xsum[0][row] + sh.x.xsum[1][row]) + (sh.x.xsum[2][row] + sh.x.xsum[3][row]);
      __syncwarp();
      if (lane == 0) mbar_arrive(&sh.sread);
      ok = __all_sync(0xffffffffu, mbar_wait(&sh.pv_done[glast % 3], (glast / 3) & 1));
      if (!ok) break;
      tc_fence_after();
      const float inv_l = 1.f / l;
      const bool live = qrow < p.N;
      __nv_bfloat16* orow = reinterpret_cast<__nv_bfloat16*>(p.o) + (static_cast<size_t>(bh) * p.N + qrow) * D + grp * OQ;
      {
        uint32_t o[OQ];
        if constexpr (OQ == 32) tmem_ld32(o_base, o); else tmem_ld16(o_base, o);
        tmem_wait_ld();
        reg_fence(o);
        uint32_t pk[OQ / 2];
#pragma unroll
        for (int k = 0; k < OQ / 2; ++k)
          pk[k] = pack_bf16x2(__uint_as_float(o[2 * k]) * inv_l, __uint_as_float(o[2 * k + 1]) * inv_l);
        if (live) {
          uint4* dst = reinterpret_cast<uint4*>(orow);
#pragma unroll
          for (int k = 0; k < OQ / 8; ++k) dst[k] = make_uint4(pk[4 * k], pk[4 * k + 1], pk[4 * k + 2], pk[4 * k + 3]);
        }
      }
      if (live && grp == 0) p.lse[static_cast<size_t>(bh) * p.N + qrow] = (m_used + __log2f(l)) * 0.69314718055994531f;
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sh.o_free);
      it += n_kv;
    }
  }

  // Teardown without a shared code path (the warpgroups run under different
  // register budgets): every warp posts, warp 0 releases TMEM once all have.
  tc_fence_before();
  __syncwarp();
  if (lane == 0) mbar_arrive(&sh.teardown);
  if (warp == 0) {
    mbar_wait(&sh.teardown, 0);
    tc_fence_after();
    tmem_dealloc(tmem, C::kTmemCols);
  }
}

}  // namespace attn
