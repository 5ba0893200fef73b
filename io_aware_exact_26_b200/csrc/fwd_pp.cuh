// Forward exact attention for sm_100a, two query tiles per CTA ("ping-pong").
//
// Method (page "attention 的显存线性化" §三; page "attn-efficient", online-softmax
// section): per 128-row query tile, stream 128-key tiles of K/V, form S on chip,
// keep a running row max m and sum l, rescale the partial output when the max
// grows, write only O and the log-sum-exp.  S and P never reach HBM.
//
// Scheduling: CTAs claim work units from a global counter (g_sched) in the
// order pp_unit numbers them, so a CTA that drew short causal units takes more;
// the producer warp claims and passes each unit index to the other warps through
// a small ring in shared memory.
//
// B200 mapping.  A work unit is a pair of query tiles A and B that read the same
// KV head (two heads of a GQA group at one query tile, or two adjacent query
// tiles of one head); each K/V tile is loaded once for both.  Team A (warps 0-7)
// owns tile A, team B (warps 8-15) tile B; the MMA warp interleaves the two
// teams' products, so while one team exponentiates, the tensor cores work on the
// other team's S or PV, and the two teams' MUFU phases alternate.
//   warps 0-7, 8-15  softmax teams; inside a team, group k = (warp % 8) / 4 owns
//                    keys [64k, 64k+64) of each S tile and O columns
//                    [k*DT/2, (k+1)*DT/2); thread = query row = TMEM lane.
//   warp 16          TMA producer: Q_A, Q_B (one buffer per team at d = 128, two
//                    at d = 64), K and V rings (2 stages each), loaded as K(0) V(0)
//                    K(1) V(1) ..., the order in which the MMA warp releases them
//   warp 17          MMA issuer
// TMEM: S_A at 0, S_B at 128 (P written over S as bf16: keys 0-63 in columns
// 0-31, keys 64-127 in 64-95), O_A at 256, O_B at 256 + DT (DT = d, or 128 for
// zero-padded e4m3 tiles at d = 64).
// Per team the loop is S(j) -> softmax(j) -> PV(j) -> S(j+1), one S buffer per
// tile with P written over it.  S(j+1) is issued right behind PV(j): MMAs issued
// by one thread are performed in issue order, so PV(j) has read P(j) before
// S(j+1) writes those columns, and the commit that signals S(j+1) also covers
// PV(j).  PV(j) is issued in two halves: the team signals when each group has written
// its first 32 keys of P (p_half), and the MMAs for keys 0-31 and 64-95 run while the
// team still exponentiates the rest; after p_ready only the other half and S(j+1)
// stand between the team and its next tile (measured +6-7% at d = 128, +3.5% at
// d = 64; a signal per quarter of P measured 13-22% slower).
// Each step a team's two groups exchange partial row maxima of the tile in
// shared memory; the exp2 with folded scale and the lazy rescale threshold are
// described in fwd.cuh.
#pragma once
#include "fwd.cuh"

namespace attn {

// F8 = false: bf16 Q, K, V and P (kind::f16).  F8 = true: e4m3 Q, K, V and P
// (kind::f8f6f4), each tile row of d bytes, with per-tensor descales folded into
// the exponent scale (Q, K) and the output (V).  An e4m3 row of d = 64 is 64 bytes:
// its tiles are padded to the 128-byte swizzle row (DT = 128 columns), the TMA
// filling columns 64-127 with zeros, so S = Q K^T is unchanged, O's padding columns
// stay 0 and only the first d columns are written out.
template <int D, bool F8 = false>
struct PpCfg {
  static constexpr int ES = F8 ? 1 : 2;                 // bytes per element
  static constexpr int DT = (F8 && D * ES < 128) ? 128 / ES : D;   // tile columns (padded)
  static constexpr int kTile = 128 * DT * ES;
  static constexpr int kBox = 128 * 128;                // one TMA box: 128 rows x 128 bytes
  static constexpr int NB = DT * ES / 128;              // boxes per tile
  static constexpr int KS = DT * ES / 32;               // S = Q K^T: 32-byte K steps
  static constexpr int PVK = F8 ? 32 : 16;              // keys per P V instruction
  static_assert(NB >= 1, "a tile row must fill one 128-byte swizzle row");
  static constexpr int KST = 2;
  static constexpr int VST = 2;
  static constexpr int kThreads = 576;
  // Of every 8 score pairs, how many are exponentiated on the FMA pipe instead of
  // MUFU (16 ex2 per SM per clock).  At d = 64 a tile's two products take 512
  // tensor-core cycles (bf16; fewer with e4m3) against 1024 MUFU cycles for its
  // exponentials, and moving 2 pairs in 8 to the FMA pipe measured +8% to +21%
  // (N = 1024 to 4096).  At d = 128, once PV is issued in halves and the exponent
  // pass is on the critical path, 1 pair in 8 measured +1.0% to +1.7% (2 or 3: less).
  static constexpr int kFmaPairs = D == 64 ? 2 : 1;
  static constexpr int kTmemCols = 512;
  static constexpr int kS0 = 0, kS1 = 128, kO0 = 256, kO1 = 256 + DT;
  // Q buffers per team: two at d = 64, so the next unit's Q loads while the current
  // unit still reads its own (short units, e.g. N = 1024, would wait for it); one
  // at d = 128, where shared memory has no room and units are longer.
  static constexpr int QST = (kTile <= 16384) ? 2 : 1;
  static constexpr int kOffQ = 0;                       // Q slots [team][QST]
  static constexpr int kOffK = 2 * QST * kTile;
  static constexpr int kOffV = kOffK + KST * kTile;
  static constexpr int kOffSh = kOffV + VST * kTile;
  static constexpr int kLayout = kOffSh + 8192;
  static constexpr int kSmem = kLayout + 1024;
  static_assert(kSmem <= 232448, "shared memory layout exceeds 227 KB");
};

struct PpShared {
  float xmax[2][2][2][128];   // [team][parity][group][row] partial row maxima of a step
  float xsum[2][2][128];      // [team][group][row] partial row sums of a unit
  uint64_t q_full[2][2], q_empty[2][2];   // [team][Q slot]
  uint64_t k_full[2], k_empty[2], v_full[2], v_empty[2];
  uint64_t s_full[2];         // per team: S of its current step complete
  uint64_t p_ready[2];        // per team: P written by its 8 warps
  uint64_t p_half[2];         // per team: the first half of each group's P columns written
  uint64_t pv_done[2];        // per team: PV of its step complete
  uint64_t xbar[2][2];        // [team][parity]: both groups posted their maxima
  uint64_t sbar[2];           // per team: both groups posted their sums
  uint64_t o_free[2];         // per team: O read out by the epilogue
  UnitRing ring;              // unit indices for the MMA warp and the 16 softmax warps
  uint64_t drain;
  uint64_t teardown;
  uint32_t tmem_base;
};
static_assert(sizeof(PpShared) <= 8192, "PpShared does not fit its slot");


struct PpUnit {
  int bh0, qt0, a0, n0;       // tile A: key tiles [a0, a0 + n0)
  int bh1, qt1, a1, n1;       // tile B (n1 = 0: no tile B)
  int u0, u1;                 // union of the two key ranges, [u0, u1]
  int bkv;
  __device__ __forceinline__ int n(int x) const { return x ? n1 : n0; }
  __device__ __forceinline__ int a(int x) const { return x ? a1 : a0; }
  __device__ __forceinline__ int qt(int x) const { return x ? qt1 : qt0; }
  __device__ __forceinline__ int bh(int x) const { return x ? bh1 : bh0; }
};

// Unit u -> two query tiles of one KV head.  The tiles of a KV head group are
// listed query-tile-major (last tile first when key ranges grow with the tile,
// as under causal masking: longest first), the G heads inside; consecutive list
// entries are paired.  The unit streams the union of the two tiles' key ranges;
// each team works on its own range inside it.
// Units are claimed group after group, so the CTAs running at one time share the
// K/V of a few heads in L2.  The last `tail_groups` groups are interleaved instead
// (their units longest first across all of them): otherwise a CTA that claims a
// long unit of the last group near the end finishes long after the others
// (measured 7-13% idle at the end with 16-32 heads).
__device__ __forceinline__ PpUnit pp_unit(const FwdParams& p, int u) {
  const int per_group = p.G * p.n_qtiles;
  const int upg = (per_group + 1) >> 1;
  const int ngroups = p.B * p.Hkv;
  const int head = (ngroups - p.tail_groups) * upg;     // units before the interleaved tail
  int gk, m;
  if (u < head) {
    gk = u / upg;
    m = u - gk * upg;
  } else {
    const int v = u - head;
    m = v / p.tail_groups;
    gk = ngroups - p.tail_groups + (v - m * p.tail_groups);
  }
  PpUnit r;
  r.bkv = gk;
  auto tile = [&](int l, int& bh, int& qt, int& a, int& n) {
    if (l < per_group) {
      const int rq = l / p.G;
      const int h = l - rq * p.G;
      qt = p.desc ? (p.n_qtiles - 1 - rq) : rq;
      bh = (gk / p.Hkv) * p.Hq + (gk % p.Hkv) * p.G + h;
      fwd_kv_range(p, qt, a, n);
    } else {
      bh = 0; qt = 0; a = 0; n = 0;
    }
  };
  tile(2 * m, r.bh0, r.qt0, r.a0, r.n0);
  tile(2 * m + 1, r.bh1, r.qt1, r.a1, r.n1);
  r.u0 = r.n1 > 0 ? min(r.a0, r.a1) : r.a0;
  r.u1 = r.n1 > 0 ? max(r.a0 + r.n0, r.a1 + r.n1) - 1 : r.a0 + r.n0 - 1;
  return r;
}

__device__ __forceinline__ int pp_units(const FwdParams& p) {
  return p.B * p.Hkv * ((p.G * p.n_qtiles + 1) >> 1);
}

template <int D, bool F8 = false>
__global__ void __launch_bounds__(576, 1)
    attn_fwd_pp_kernel(const __grid_constant__ CUtensorMap tmq, const __grid_constant__ CUtensorMap tmk,
                       const __grid_constant__ CUtensorMap tmv, const FwdParams p) {
  using C = PpCfg<D, F8>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  PpShared& sh = *reinterpret_cast<PpShared*>(smem + C::kOffSh);
  uint8_t* sQ = smem + C::kOffQ;
  uint8_t* sK = smem + C::kOffK;
  uint8_t* sV = smem + C::kOffV;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_units = pp_units(p);

  if (threadIdx.x == 0) {
    for (int i = 0; i < 2; ++i) {
      for (int q = 0; q < C::QST; ++q) {
        mbar_init(&sh.q_full[i][q], 1);
        mbar_init(&sh.q_empty[i][q], 1);
      }
      mbar_init(&sh.k_full[i], 1);
      mbar_init(&sh.k_empty[i], 1);
      mbar_init(&sh.v_full[i], 1);
      mbar_init(&sh.v_empty[i], 1);
      mbar_init(&sh.s_full[i], 1);
      mbar_init(&sh.p_ready[i], 8);
      mbar_init(&sh.p_half[i], 8);
      mbar_init(&sh.pv_done[i], 1);
      mbar_init(&sh.xbar[i][0], 8);
      mbar_init(&sh.xbar[i][1], 8);
      mbar_init(&sh.sbar[i], 8);
      mbar_init(&sh.o_free[i], 8);
    }
    unit_ring_init(sh.ring, 17);
    mbar_init(&sh.drain, 1);
    mbar_init(&sh.teardown, 18);
    fence_barrier_init();
  }
  if (warp == 0) { tmem_alloc(&sh.tmem_base, C::kTmemCols); tmem_relinquish(); }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sh.tmem_base;

  if (warp == 16) {
    // ------------------------------------------------------------ TMA producer: Q_A, Q_B, K, V
    if (lane == 0) {
      tma_prefetch_desc(&tmq); tma_prefetch_desc(&tmk); tma_prefetch_desc(&tmv);
      int kc = 0, uq0 = 0, uq1 = 0;
      int nk = 0;
      bool ok = true;
      // A unit is claimed only when the producer is ready to load it: claiming
      // ahead leaves units reserved by busy CTAs at the tail (measured slower).
      int u = 0;
      for (int k = 0; ok; ++k) {
        u = unit_ring_claim(sh.ring, k, p.sched_slot, p.sched_gen, n_units);
        if (u < 0) break;
        const PpUnit w = pp_unit(p, u);
        auto load_q = [&](int x, int uq) -> bool {     // Q of team x, its uq-th unit
          const int qs = uq % C::QST;
          if (uq >= C::QST && !mbar_wait(&sh.q_empty[x][qs], ((uq / C::QST) - 1) & 1)) return false;
          mbar_arrive_expect_tx(&sh.q_full[x][qs], C::kTile);
          in_range(w.qt(x), p.n_qtiles);
          in_range(w.bh(x), static_cast<long long>(p.B) * p.Hq);
          for (int c = 0; c < C::NB; ++c)
            tma_load_3d(sQ + (x * C::QST + qs) * C::kTile + c * C::kBox, &tmq, &sh.q_full[x][qs], c * 128 / C::ES,
                        w.qt(x) * 128, w.bh(x));
          return true;
        };
        ok = load_q(0, uq0++);
        if (ok && w.n1 > 0) ok = load_q(1, uq1++);
        for (int j = w.u0; j <= w.u1 && ok; ++j, ++kc) {
          const int st = kc & 1;
          if (kc >= 2) ok = mbar_wait(&sh.k_empty[st], ((kc >> 1) - 1) & 1);
          if (!ok) break;
          mbar_arrive_expect_tx(&sh.k_full[st], C::kTile);
          in_range(j, p.n_qtiles);
          in_range(w.bkv, static_cast<long long>(p.B) * p.Hkv);
          for (int c = 0; c < C::NB; ++c)
            tma_load_3d(sK + st * C::kTile + c * C::kBox, &tmk, &sh.k_full[st], c * 128 / C::ES, j * 128, w.bkv);
          if (kc >= 2) ok = mbar_wait(&sh.v_empty[st], ((kc >> 1) - 1) & 1);
          if (!ok) { nk = kc + 1; break; }
          mbar_arrive_expect_tx(&sh.v_full[st], C::kTile);
          for (int c = 0; c < C::NB; ++c)
            tma_load_3d(sV + st * C::kTile + c * C::kBox, &tmv, &sh.v_full[st], c * 128 / C::ES, j * 128, w.bkv);
          nk = kc + 1;
        }
      }
      if (u == -2) ok = false;
      if (!ok)
        for (int g = max(0, nk - 2); g < nk; ++g) {
          mbar_drain_wait(&sh.k_full[g & 1], (g >> 1) & 1);
          mbar_drain_wait(&sh.v_full[g & 1], (g >> 1) & 1);
        }
    }
  } else if (warp == 17) {
    // ------------------------------------------------------------ MMA issuer
    // Per step j: PV_A(j), S_A(j+1), PV_B(j), S_B(j+1).  S_X(j+1) waits for PV_X(j)
    // (the P it overwrites); meanwhile the tensor cores run the other team's work.
    // PV_X(j) goes out in two halves, on p_half and on p_ready.
    const bool leader = elect_one();
    constexpr uint32_t idS = F8 ? idesc_e4m3_f32(128, 128, false, false) : idesc_bf16_f32(128, 128, false, false);
    constexpr uint32_t idO = F8 ? idesc_e4m3_f32(128, C::DT, false, true) : idesc_bf16_f32(128, D, false, true);
    constexpr uint32_t hi = sdesc_hi_sw128(1024);
    const uint32_t q_lo0 = sdesc_lo(smem_u32(sQ), 16);
    const uint32_t k_lo0 = sdesc_lo(smem_u32(sK), 16);
    const uint32_t v_lo0 = sdesc_lo(smem_u32(sV), C::kBox);
    auto wait = [&](uint64_t* bar, uint32_t parity) -> bool {
      return __all_sync(0xffffffffu, mbar_wait(bar, parity));
    };
    int kc = 0, vc = 0;
    int gs0 = 0, gs1 = 0;        // steps issued per team
    int uu0 = 0, uu1 = 0;        // units per team
    bool ok = true;
    // S_X = Q_X K^T for team x from K stage st
    auto issue_s = [&](int x, int qs, int st, bool last) {
      if (leader) {
        const uint32_t q_lo = q_lo0 + (x * C::QST + qs) * (C::kTile >> 4);
        const uint32_t k_lo = k_lo0 + st * (C::kTile >> 4);
#pragma unroll
        for (int k = 0; k < C::KS; ++k) {
          const uint32_t off = ((k >> 2) * C::kBox + (k & 3) * 32) >> 4;
          if constexpr (F8)
            umma_ss_f8_lo(tmem + (x ? C::kS1 : C::kS0), q_lo + off, k_lo + off, hi, idS, k > 0);
          else
            umma_ss_lo(tmem + (x ? C::kS1 : C::kS0), q_lo + off, k_lo + off, hi, idS, k > 0);
        }
        umma_commit(&sh.s_full[x]);
        if (last) umma_commit(&sh.q_empty[x][qs]);
      }
      __syncwarp();
    };
    // O_X (+)= P_X V for team x from V stage st
    auto issue_pv = [&](int x, int st, bool first, int half) {
      if (leader) {
        const uint32_t v_lo = v_lo0 + st * (C::kTile >> 4);
        const uint32_t sbase = tmem + (x ? C::kS1 : C::kS0);
        // P of keys [k * PVK, (k + 1) * PVK) sits in 8 TMEM columns: keys 0-63 from column
        // 0, keys 64-127 from column 64 (bf16: 2 per column, e4m3: 4 per column)
        if constexpr (F8) {
#pragma unroll
          for (int kk = 0; kk < 2; ++kk) {
            const int k = kk * 2 + half;     // half 0: keys 0-31 and 64-95
            umma_ts_f8_lo(tmem + (x ? C::kO1 : C::kO0), sbase + (k >> 1) * 64 + (k & 1) * 8,
                          v_lo + ((k * C::PVK * 128) >> 4), hi, idO, !(first && k == 0));
          }
        } else {
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const int k = (kk >> 1) * 4 + half * 2 + (kk & 1);   // half 0: keys 0-31 and 64-95
            umma_ts_lo(tmem + (x ? C::kO1 : C::kO0), sbase + (k >> 2) * 64 + (k & 3) * 8,
                       v_lo + ((k * C::PVK * 128) >> 4), hi, idO, !(first && k == 0));
          }
        }
        if (half) umma_commit(&sh.pv_done[x]);
      }
      __syncwarp();
    };
    for (int k = 0; ok; ++k) {
      const int u = unit_ring_take(sh.ring, k, lane, ok);
      if (u < 0) break;
      const PpUnit w = pp_unit(p, u);
      // Team x works on key tiles [a_x, l_x] inside the unit's union [u0, u1]; its S for
      // the first of them is issued as soon as that K tile is in (K(u0) here, later ones
      // from the step before).
      {
        const int st = kc & 1;
        ok = wait(&sh.k_full[st], (kc >> 1) & 1);
#pragma unroll
        for (int x = 0; x < 2; ++x) {
          const int uux = x ? uu1 : uu0;
          if (!ok || w.n(x) == 0 || w.a(x) != w.u0) continue;
          ok = wait(&sh.q_full[x][uux % C::QST], (uux / C::QST) & 1);
          if (!ok) continue;
          tc_fence_after();
          issue_s(x, uux % C::QST, st, w.n(x) == 1);
        }
        if (!ok) break;
        if (leader) umma_commit(&sh.k_empty[st]);
        __syncwarp();
        ++kc;
      }
      for (int j = w.u0; j <= w.u1 && ok; ++j, ++vc) {
        const int vst = vc & 1;
        ok = wait(&sh.v_full[vst], (vc >> 1) & 1);
        const bool next_k = j + 1 <= w.u1;
        bool k_ready = false;
#pragma unroll
        for (int x = 0; x < 2; ++x) {
          const int gsx = x ? gs1 : gs0, uux = x ? uu1 : uu0, nx = w.n(x), ax = w.a(x);
          if (!ok || nx == 0) continue;
          const int lx = ax + nx - 1;
          if (ax <= j && j <= lx) {
            const int g = gsx + (j - ax);
            ok = wait(&sh.p_half[x], g & 1);
            if (ok && j == ax && uux >= 1) ok = wait(&sh.o_free[x], (uux - 1) & 1);
            if (!ok) continue;
            tc_fence_after();
            issue_pv(x, vst, j == ax, 0);
            ok = wait(&sh.p_ready[x], g & 1);
            if (!ok) continue;
            tc_fence_after();
            issue_pv(x, vst, j == ax, 1);
            if (j + 1 <= lx) {
              if (!k_ready) {
                ok = wait(&sh.k_full[kc & 1], (kc >> 1) & 1);
                k_ready = true;
              }
              if (!ok) continue;
              tc_fence_after();
              issue_s(x, uux % C::QST, kc & 1, j + 1 == lx);   // in issue order behind PV_X(j)
            }
          } else if (j + 1 == ax) {          // team x starts at the next key tile
            if (!k_ready) {
              ok = wait(&sh.k_full[kc & 1], (kc >> 1) & 1);
              k_ready = true;
            }
            if (ok) ok = wait(&sh.q_full[x][uux % C::QST], (uux / C::QST) & 1);
            if (!ok) continue;
            tc_fence_after();
            issue_s(x, uux % C::QST, kc & 1, nx == 1);
          }
        }
        if (!ok) break;
        if (leader) {
          umma_commit(&sh.v_empty[vst]);
          if (next_k) umma_commit(&sh.k_empty[kc & 1]);
        }
        __syncwarp();
        if (next_k) ++kc;
      }
      gs0 += w.n0; ++uu0;
      if (w.n1 > 0) { gs1 += w.n1; ++uu1; }
    }
    if (leader) {
      umma_commit(&sh.drain);
      mbar_wait(&sh.drain, 0);
    }
    __syncwarp();
  } else if (warp < 16) {
    // ------------------------------------------------------------ softmax teams
    const int x = warp >> 3;                                    // team
    const int grp = (warp >> 2) & 1;                            // keys [64 grp, 64 grp + 64)
    const int quad = warp & 3;
    const int row = quad * 32 + lane;
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(quad * 32) << 16);
    const uint32_t s_base = lane_base + (x ? C::kS1 : C::kS0) + grp * 64;
    constexpr int OH = C::DT / 2;                               // O columns per group (padded)
    const uint32_t o_base = lane_base + (x ? C::kO1 : C::kO0) + grp * OH;
    const float c = p.c;
    const uint64_t c2 = f2pack(c, c);
    int gs = 0, uu = 0;
    bool ok = true;
    // -inf outside the visible columns [lo, lim].  (A causal-only variant testing one
    // bound per element measured slower: the second code path in the hot loop cost
    // more than the compares it saved.)
    auto mask16 = [&](uint32_t (&r)[16], int col0, int lo, int lim) {
#pragma unroll
      for (int k = 0; k < 16; ++k)
        if (col0 + k < lo || col0 + k > lim) r[k] = 0xff800000u;
    };
    for (int k = 0; ok; ++k) {
      const int u = unit_ring_take(sh.ring, k, lane, ok);
      if (u < 0) break;
      const PpUnit w = pp_unit(p, u);
      const int n = w.n(x), a = w.a(x);
      if (n == 0) continue;
      const int qrow = w.qt(x) * 128 + row;
      const int bh = w.bh(x);
      float m_used = -INFINITY;
      uint64_t lsum = f2pack(0.f, 0.f);
      for (int j = 0; j < n && ok; ++j) {
        const int g = gs + j, xp = g & 1;
        ok = __all_sync(0xffffffffu, mbar_wait(&sh.s_full[x], g & 1));
        if (!ok) break;
        tc_fence_after();
        const int kbase = (a + j) * 128 + grp * 64;
        const int lo = qrow - p.wl - kbase;                          // first visible column
        const int lim = min(p.N - 1, qrow + p.wr) - kbase;           // last visible column
        const bool msk = __any_sync(0xffffffffu, lo > 0 || lim < 63);
        // pass 1: this group's partial row max of the 64 columns
        float mx4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
        {
          uint32_t r0[16], r1[16], r2[16], r3[16];
          tmem_ld16(s_base, r0);
          tmem_ld16(s_base + 16, r1);
          tmem_ld16(s_base + 32, r2);
          tmem_ld16(s_base + 48, r3);
          tmem_wait_ld();
          reg_fence(r0);
          reg_fence(r1);
          reg_fence(r2);
          reg_fence(r3);
          if (msk) {
            // Masked columns become -inf here and go back to TMEM, so the exponent pass
            // below reads them already masked and needs no test of its own.
            mask16(r0, 0, lo, lim);
            mask16(r1, 16, lo, lim);
            mask16(r2, 32, lo, lim);
            mask16(r3, 48, lo, lim);
            tmem_st16(s_base, r0);
            tmem_st16(s_base + 16, r1);
            tmem_st16(s_base + 32, r2);
            tmem_st16(s_base + 48, r3);
            tmem_wait_st();
          }
#pragma unroll
          for (int k = 0; k < 16; k += 8) {
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              mx4[e] = max3f(mx4[e], __uint_as_float(r0[k + e]), __uint_as_float(r0[k + e + 4]));
              mx4[e] = max3f(mx4[e], __uint_as_float(r1[k + e]), __uint_as_float(r1[k + e + 4]));
              mx4[e] = max3f(mx4[e], __uint_as_float(r2[k + e]), __uint_as_float(r2[k + e + 4]));
              mx4[e] = max3f(mx4[e], __uint_as_float(r3[k + e]), __uint_as_float(r3[k + e + 4]));
            }
          }
        }
        sh.xmax[x][xp][grp][row] = fmaxf(fmaxf(mx4[0], mx4[1]), fmaxf(mx4[2], mx4[3]));
        __syncwarp();
        if (lane == 0) mbar_arrive(&sh.xbar[x][xp]);
        ok = __all_sync(0xffffffffu, mbar_wait(&sh.xbar[x][xp], (g >> 1) & 1));
        if (!ok) break;
        // tile max in log2 units; a row whose keys in this tile are all masked keeps -inf
        const float mx = fmaxf(sh.xmax[x][xp][0][row], sh.xmax[x][xp][1][row]);
        const float m_tile = mx == -INFINITY ? -INFINITY : mx * c;
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
        // Rescale this group's O columns if the max moved.  The commit that signalled
        // S_X(j) also covers PV_X(j-1), so O already holds every step before j; the
        // wait below is then immediate.
        if (__any_sync(0xffffffffu, need && j > 0)) {
          ok = __all_sync(0xffffffffu, mbar_wait(&sh.pv_done[x], (g - 1) & 1));
          if (!ok) break;
          tc_fence_after();
#pragma unroll 1
          for (int q4 = 0; q4 < OH / 16; ++q4) {
            uint32_t o[16];
            tmem_ld16(o_base + q4 * 16, o);
            tmem_wait_ld();
            reg_fence(o);
#pragma unroll
            for (int k = 0; k < 16; ++k) o[k] = __float_as_uint(__uint_as_float(o[k]) * alpha);
            tmem_st16(o_base + q4 * 16, o);
          }
        }
        // pass 2: exponentiate, P (bf16) over the columns already read.  Masked columns
        // hold -inf (written back by pass 1), and c > 0 (the host floors it at 1e-30), so
        // their exponent argument is -inf and p = 0; the base is 0 while the row has seen
        // no visible key.
        const float mb = m_used == -INFINITY ? 0.f : m_used;
        const uint64_t nm2 = f2pack(-mb, -mb);
#pragma unroll
        for (int cc = 0; cc < 4; ++cc) {
          uint32_t r[16];
          tmem_ld16(s_base + cc * 16, r);
          tmem_wait_ld();
          reg_fence(r);
          uint32_t pk[8];
#pragma unroll
          for (int k = 0; k < 8; ++k) {
            const uint64_t xx = ffma2(f2pack(__uint_as_float(r[2 * k]), __uint_as_float(r[2 * k + 1])), c2, nm2);
            float x0, x1;
            f2unpack(xx, x0, x1);
            float a, b;
            if (k >= 8 - C::kFmaPairs) {
              exp2_fma_pair(x0, x1, a, b);
            } else {
              a = ex2_approx(x0);
              b = ex2_approx(x1);
            }
            lsum = fadd2(lsum, f2pack(a, b));
            if constexpr (F8) {
              // four e4m3 per column, lowest key in the low byte; p <= 2^tau = 256 < 448
              const uint32_t two = pack_e4m3x2(a, b);
              pk[k >> 1] = (k & 1) ? (pk[k >> 1] | (two << 16)) : two;
            } else {
              pk[k] = pack_bf16x2(a, b);
            }
          }
          if (cc == 2) {
            // chunks 0 and 1 were stored a chunk ago: signal that half of P is in
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&sh.p_half[x]);
          }
          if constexpr (F8) {
            const uint32_t (&p4)[4] = *reinterpret_cast<const uint32_t (*)[4]>(pk);
            tmem_st4(s_base + cc * 4, p4);
          } else {
            tmem_st8(s_base + cc * 8, pk);
          }
        }
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&sh.p_ready[x]);
      }
      if (!ok) break;
      // epilogue: combine the two groups' sums, wait for the last PV, O / l, LSE
      const int glast = gs + n - 1;
      float l0, l1;
      f2unpack(lsum, l0, l1);
      sh.xsum[x][grp][row] = l0 + l1;
      __syncwarp();
      if (lane == 0) mbar_arrive(&sh.sbar[x]);
      ok = __all_sync(0xffffffffu, mbar_wait(&sh.sbar[x], uu & 1));
      if (!ok) break;
      const float l = sh.xsum[x][0][row] + sh.xsum[x][1][row];
      ok = __all_sync(0xffffffffu, mbar_wait(&sh.pv_done[x], glast & 1));
      if (!ok) break;
      tc_fence_after();
      const float inv_l = p.oscale / l;      // oscale: V's descale (1 for bf16)
      const bool live = qrow < p.N && in_range(bh, static_cast<long long>(p.B) * p.Hq);
      __nv_bfloat16* orow = reinterpret_cast<__nv_bfloat16*>(p.o) + (static_cast<size_t>(bh) * p.N + qrow) * D + grp * OH;
      const bool cols = grp * OH < D;       // padded tiles: the second group's columns are padding
      if constexpr (OH == 64) {
        // 128 bytes of the row per group, in two halves of 32 columns.  Each half is
        // exchanged among groups of 4 lanes before it is stored, so one store instruction
        // writes 64 contiguous bytes of each of 8 rows instead of 16 bytes of each of 32:
        // stores scattered over 32 rows bounded this epilogue (measured at d = 128: +5-9%
        // forward at N = 1024, +3% at N = 4096, +0.7% at N = 32768).
        const int row0 = w.qt(x) * 128 + quad * 32 + (lane & ~3);
        const bool hl = in_range(bh, static_cast<long long>(p.B) * p.Hq) && cols;
        __nv_bfloat16* obase = reinterpret_cast<__nv_bfloat16*>(p.o) + static_cast<size_t>(bh) * p.N * D + grp * OH +
                               (lane & 3) * 8;
#pragma unroll 1
        for (int hh = 0; hh < 2; ++hh) {
          uint32_t o[2][16];
          tmem_ld16(o_base + hh * 32, o[0]);
          tmem_ld16(o_base + hh * 32 + 16, o[1]);
          tmem_wait_ld();
          reg_fence(o[0]);
          reg_fence(o[1]);
          uint32_t ch[4][4];            // 16-byte chunk k of this half row: its columns 8k .. 8k+7
#pragma unroll
          for (int k = 0; k < 16; ++k)
            ch[k >> 2][k & 3] = pack_bf16x2(__uint_as_float(o[k >> 3][2 * (k & 7)]) * inv_l,
                                            __uint_as_float(o[k >> 3][2 * (k & 7) + 1]) * inv_l);
          transpose_row_chunks<4>(ch, lane);
          if (hl) {
#pragma unroll
            for (int t = 0; t < 4; ++t)
              if (row0 + t < p.N)
                *reinterpret_cast<uint4*>(obase + static_cast<size_t>(row0 + t) * D + hh * 32) =
                    make_uint4(ch[t][0], ch[t][1], ch[t][2], ch[t][3]);
          }
        }
      } else {
        // 64 bytes of the row per group, 16 columns at a time, stored by the row's own
        // thread (the exchange measured no gain at d = 64)
#pragma unroll 1
        for (int q4 = 0; q4 < OH / 16; ++q4) {
          uint32_t o[16];
          tmem_ld16(o_base + q4 * 16, o);
          tmem_wait_ld();
          reg_fence(o);
          uint32_t pk[8];
#pragma unroll
          for (int k = 0; k < 8; ++k)
            pk[k] = pack_bf16x2(__uint_as_float(o[2 * k]) * inv_l, __uint_as_float(o[2 * k + 1]) * inv_l);
          if (live && cols) {
            uint4* dst = reinterpret_cast<uint4*>(orow + q4 * 16);
            dst[0] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
            dst[1] = make_uint4(pk[4], pk[5], pk[6], pk[7]);
          }
        }
      }
      if (live && grp == 0) p.lse[static_cast<size_t>(bh) * p.N + qrow] = (m_used + __log2f(l)) * 0.69314718055994531f;
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sh.o_free[x]);
      gs += n;
      ++uu;
    }
  }

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
