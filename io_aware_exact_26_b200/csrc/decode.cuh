// Split-KV decoding ("FlashDecoding") for sm_100a: Nq new query rows against Nk
// cached keys, with Nq small (1 .. a few hundred) and Nk long.
//
// Method (page "attention 的显存线性化", reading list: FlashDecoding; page
// "attn-efficient", online-softmax section): the keys of each (batch, kv-head) are
// cut into S contiguous splits; each split runs the tiled online softmax of the
// forward over its key tiles and leaves a partial (O_s normalised by its own sum,
// LSE_s).  A merge kernel combines the partials of a query row with the same
// rescale the online softmax uses: with m = max_s LSE_s and w_s = exp(LSE_s - m),
//     O = sum_s w_s O_s / sum_s w_s,   LSE = m + ln sum_s w_s.
// With S = 1 the kernel writes O and LSE itself and no merge runs.
//
// B200 mapping.  Decoding reads every K/V byte once and does little arithmetic per
// byte, so it is bound by HBM; the design keeps K/V streaming at full rate:
//  - one work unit = (b, kv-head g, query block, key split).  The query block packs
//    the G query heads of the group times R query rows (G*R <= 128) into the 128
//    rows of one tcgen05 tile, so K/V of a group cross HBM once for all its heads;
//  - the producer warp packs the Q block into shared memory itself (rows from G
//    heads are not one TMA box; 128B-swizzled K-major layout, the same the TMA
//    writes) and streams K and V tiles by TMA through 2-stage rings;
//  - the MMA warp keeps S two tiles ahead (two S buffers in TMEM), so the softmax
//    of tile j+1 overlaps P(j)V;
//  - 8 softmax warps as in the forward: two groups of 64 keys per tile, thread =
//    tile row = TMEM lane, partial maxima exchanged in shared memory, lazy rescale;
//  - units are claimed from a per-launch counter (g_sched) by one CTA per SM.
// Causal reading for Nq != Nk: query i sits at position Nk - Nq + i and sees keys
// j <= Nk - Nq + i.
#pragma once
#include "fwd.cuh"

namespace attn {

struct DecParams {
  const __nv_bfloat16* q;   // [B][Hq][Nq][D]
  __nv_bfloat16* o;         // [B][Hq][Nq][D]   (S == 1)
  float* lse;               // [B][Hq][Nq]      (S == 1)
  float* opart;             // [B*Hq*Nq][S][D]  partial O_s, fp32 (S > 1)
  float* lpart;             // [B*Hq*Nq][S]     partial LSE_s, natural log; -inf: no visible key
  int B, Hq, Hkv, G, Nq, Nk;
  int R;        // query rows per head in a block (G * R <= 128)
  int nqb;      // query blocks per (b, kv-head)
  int S;        // key splits
  int T;        // key tiles per split
  int causal;
  float c;      // scale * log2(e), floored (folded_scale)
  int n_units;
  int sched_slot;
  unsigned int sched_gen;
};

struct DecUnit {
  int bg, qb, s;   // b * Hkv + g, query block, split
  int j0, n;       // key tiles [j0, j0 + n); n = 0: no key of the split is visible
};

__device__ __forceinline__ DecUnit dec_unit(const DecParams& p, int u) {
  DecUnit w;
  w.s = u % p.S;
  const int r = u / p.S;
  w.qb = r % p.nqb;
  w.bg = r / p.nqb;
  const int qlast = min(p.Nq - 1, w.qb * p.R + p.R - 1);
  const int kmax = p.causal ? min(p.Nk - 1, p.Nk - p.Nq + qlast) : p.Nk - 1;
  const int ntk = (kmax >> 7) + 1;
  w.j0 = w.s * p.T;
  w.n = max(0, min(w.j0 + p.T, ntk) - w.j0);
  return w;
}

template <int D>
struct DecCfg {
  static constexpr int kTile = 128 * D * 2;
  static constexpr int kBox = 128 * 128;          // one 64-column box: 128 rows x 128 bytes
  static constexpr int QST = 2, KST = 2, VST = 2;
  static constexpr int kThreads = 320;            // 8 softmax warps, producer, MMA
  static constexpr int kS0 = 0, kS1 = 128, kO = 256;
  static constexpr int kTmemCols = 512;
  static constexpr int kOffQ = 0;
  static constexpr int kOffK = QST * kTile;
  static constexpr int kOffV = kOffK + KST * kTile;
  static constexpr int kOffSh = kOffV + VST * kTile;
  static constexpr int kLayout = kOffSh + 4096;
  static constexpr int kSmem = kLayout + 1024;
  static_assert(kSmem <= 232448, "shared memory layout exceeds 227 KB");
};

struct DecShared {
  float xmax[2][2][128];     // [step parity][group][row] partial row maxima
  float xsum[2][128];        // [group][row] partial row sums of a unit
  uint64_t q_full[2], q_empty[2];
  uint64_t k_full[2], k_empty[2], v_full[2], v_empty[2];
  uint64_t s_full[2];        // S of step g complete in buffer g % 2
  uint64_t p_ready[2];       // P of step g written over buffer g % 2 by the 8 softmax warps
  uint64_t pv_done;          // P V of a step complete
  uint64_t xbar[2];          // [step parity]: both groups posted their maxima
  uint64_t sbar;             // both groups posted their sums
  uint64_t o_free;           // O read out by the epilogue
  UnitRing ring;             // unit indices for the MMA warp and the 8 softmax warps
  uint64_t drain;
  uint64_t teardown;
  uint32_t tmem_base;
};
static_assert(sizeof(DecShared) <= 4096, "DecShared does not fit its slot");

template <int D>
__global__ void __launch_bounds__(320, 1)
    attn_decode_kernel(const __grid_constant__ CUtensorMap tmk, const __grid_constant__ CUtensorMap tmv,
                       const DecParams p) {
  using C = DecCfg<D>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  DecShared& sh = *reinterpret_cast<DecShared*>(smem + C::kOffSh);
  uint8_t* sQ = smem + C::kOffQ;
  uint8_t* sK = smem + C::kOffK;
  uint8_t* sV = smem + C::kOffV;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(&sh.q_full[i], 1);
      mbar_init(&sh.q_empty[i], 1);
      mbar_init(&sh.k_full[i], 1);
      mbar_init(&sh.k_empty[i], 1);
      mbar_init(&sh.v_full[i], 1);
      mbar_init(&sh.v_empty[i], 1);
      mbar_init(&sh.s_full[i], 1);
      mbar_init(&sh.p_ready[i], 8);
      mbar_init(&sh.xbar[i], 8);
    }
    mbar_init(&sh.pv_done, 1);
    mbar_init(&sh.sbar, 8);
    mbar_init(&sh.o_free, 8);
    unit_ring_init(sh.ring, 9);
    mbar_init(&sh.drain, 1);
    mbar_init(&sh.teardown, 10);
    fence_barrier_init();
  }
  if (warp == 0) { tmem_alloc(&sh.tmem_base, C::kTmemCols); tmem_relinquish(); }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sh.tmem_base;

  if (warp == 8) {
    // ------------------------------------------------------------ producer: Q block (whole warp), K, V (lane 0)
    if (lane == 0) { tma_prefetch_desc(&tmk); tma_prefetch_desc(&tmv); }
    int kc = 0, uq = 0, nk = 0;
    bool ok = true;
    int u = 0;
    for (int k = 0; ok; ++k) {
      if (lane == 0) u = unit_ring_claim(sh.ring, k, p.sched_slot, p.sched_gen, p.n_units);
      u = __shfl_sync(0xffffffffu, u, 0);
      if (u < 0) break;
      const DecUnit w = dec_unit(p, u);
      if (w.n == 0) continue;
      // Q block: tile row t = h * R + i holds query qb * R + i of head g * G + h; the rest is zero
      const int qs = uq & 1;
      if (uq >= 2) ok = __all_sync(0xffffffffu, mbar_wait(&sh.q_empty[qs], ((uq >> 1) - 1) & 1));
      if (!ok) break;
      {
        constexpr int CPR = D / 8;                    // 16-byte chunks per row
        const int b = w.bg / p.Hkv, g = w.bg - b * p.Hkv;
        uint8_t* dst0 = sQ + qs * C::kTile;
#pragma unroll 4
        for (int ci = lane; ci < 128 * CPR; ci += 32) {
          const int t = ci / CPR, c8 = ci - t * CPR;
          const int h = t / p.R, i = t - h * p.R;
          const int qi = w.qb * p.R + i;
          uint4 val = make_uint4(0u, 0u, 0u, 0u);
          const size_t qoff = ((static_cast<size_t>(b) * p.Hq + g * p.G + h) * p.Nq + qi) * D + c8 * 8;
          if (h < p.G && qi < p.Nq && in_range(static_cast<long long>(qoff), static_cast<long long>(p.B) * p.Hq * p.Nq * D))
            val = *reinterpret_cast<const uint4*>(p.q + qoff);
          // 128B swizzle: 16-byte chunk cc of row t lands at chunk cc ^ (t & 7) of the row
          const int box = c8 >> 3, cc = c8 & 7;
          *reinterpret_cast<uint4*>(dst0 + box * C::kBox + t * 128 + ((cc ^ (t & 7)) << 4)) = val;
        }
        fence_proxy_async_smem();                     // generic-proxy writes -> tensor-core reads
        __syncwarp();
        if (lane == 0) mbar_arrive(&sh.q_full[qs]);
        ++uq;
      }
      if (lane == 0) {
        for (int j = 0; j < w.n && ok; ++j, ++kc) {
          const int st = kc & 1;
          if (kc >= 2) ok = mbar_wait(&sh.k_empty[st], ((kc >> 1) - 1) & 1);
          if (!ok) break;
          mbar_arrive_expect_tx(&sh.k_full[st], C::kTile);
          in_range(w.j0 + j, (p.Nk + 127) / 128);
          in_range(w.bg, static_cast<long long>(p.B) * p.Hkv);
          for (int c = 0; c < D / 64; ++c)
            tma_load_3d(sK + st * C::kTile + c * C::kBox, &tmk, &sh.k_full[st], c * 64, (w.j0 + j) * 128, w.bg);
          if (kc >= 2) ok = mbar_wait(&sh.v_empty[st], ((kc >> 1) - 1) & 1);
          if (!ok) { nk = kc + 1; break; }
          mbar_arrive_expect_tx(&sh.v_full[st], C::kTile);
          for (int c = 0; c < D / 64; ++c)
            tma_load_3d(sV + st * C::kTile + c * C::kBox, &tmv, &sh.v_full[st], c * 64, (w.j0 + j) * 128, w.bg);
          nk = kc + 1;
        }
      }
      ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
    }
    if (u == -2) ok = false;
    if (!ok && lane == 0)
      for (int g = max(0, nk - 2); g < nk; ++g) {
        mbar_drain_wait(&sh.k_full[g & 1], (g >> 1) & 1);
        mbar_drain_wait(&sh.v_full[g & 1], (g >> 1) & 1);
      }
    __syncwarp();
  } else if (warp == 9) {
    // ------------------------------------------------------------ MMA issuer
    // Per unit: S(0), S(1); then per step j: PV(j), S(j + 2) into the buffer PV(j) just
    // read (MMAs of one thread run in issue order, so PV(j) reads P(j) first).
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
    int kc = 0, vc = 0, gs = 0, uq = 0;
    bool ok = true;
    auto issue_s = [&](int g, int qs) -> bool {     // S(g) = Q K(kc)^T into buffer g % 2
      const int st = kc & 1;
      if (!wait(&sh.k_full[st], (kc >> 1) & 1)) return false;
      tc_fence_after();
      if (leader) {
        const uint32_t q_lo = q_lo0 + qs * (C::kTile >> 4);
        const uint32_t k_lo = k_lo0 + st * (C::kTile >> 4);
#pragma unroll
        for (int k = 0; k < D / 16; ++k) {
          const uint32_t off = ((k >> 2) * C::kBox + (k & 3) * 32) >> 4;
          umma_ss_lo(tmem + ((g & 1) ? C::kS1 : C::kS0), q_lo + off, k_lo + off, hi, idS, k > 0);
        }
        umma_commit(&sh.s_full[g & 1]);
        umma_commit(&sh.k_empty[st]);
      }
      __syncwarp();
      ++kc;
      return true;
    };
    for (int k = 0; ok; ++k) {
      const int u = unit_ring_take(sh.ring, k, lane, ok);
      if (u < 0) break;
      const DecUnit w = dec_unit(p, u);
      if (w.n == 0) continue;
      const int qs = uq & 1;
      ok = wait(&sh.q_full[qs], (uq >> 1) & 1);
      for (int t = 0; t < 2 && t < w.n && ok; ++t) {
        ok = issue_s(gs + t, qs);
        if (ok && t == w.n - 1 && leader) umma_commit(&sh.q_empty[qs]);
        __syncwarp();
      }
      for (int j = 0; j < w.n && ok; ++j, ++vc) {
        const int g = gs + j, vst = vc & 1;
        ok = wait(&sh.v_full[vst], (vc >> 1) & 1);
        if (ok) ok = wait(&sh.p_ready[g & 1], (g >> 1) & 1);
        if (ok && j == 0 && uq >= 1) ok = wait(&sh.o_free, (uq - 1) & 1);
        if (!ok) break;
        tc_fence_after();
        if (leader) {
          const uint32_t v_lo = v_lo0 + vst * (C::kTile >> 4);
          const uint32_t sbase = tmem + ((g & 1) ? C::kS1 : C::kS0);
#pragma unroll
          for (int k = 0; k < 8; ++k)
            umma_ts_lo(tmem + C::kO, sbase + (k >> 2) * 64 + (k & 3) * 8, v_lo + ((k * 2048) >> 4), hi, idO,
                       !(j == 0 && k == 0));
          umma_commit(&sh.pv_done);
          umma_commit(&sh.v_empty[vst]);
        }
        __syncwarp();
        if (j + 2 < w.n) {
          ok = issue_s(g + 2, qs);
          if (ok && j + 2 == w.n - 1 && leader) umma_commit(&sh.q_empty[qs]);
          __syncwarp();
        }
      }
      gs += w.n;
      ++uq;
    }
    if (leader) {
      umma_commit(&sh.drain);
      mbar_wait(&sh.drain, 0);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ softmax warps 0-7
    const int grp = warp >> 2;                                  // keys [64 grp, 64 grp + 64)
    const int quad = warp & 3;
    const int row = quad * 32 + lane;                           // tile row = TMEM lane
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(quad * 32) << 16);
    constexpr int OH = D / 2;
    const uint32_t o_base = lane_base + C::kO + grp * OH;
    const float c = p.c;
    const uint64_t c2 = f2pack(c, c);
    const int h = row / p.R, i = row - h * p.R;
    int gs = 0, uq = 0;
    bool ok = true;
    auto mask16 = [&](uint32_t (&r)[16], int col0, int lim) {
#pragma unroll
      for (int k = 0; k < 16; ++k)
        if (col0 + k > lim) r[k] = 0xff800000u;
    };
    for (int k = 0; ok; ++k) {
      const int u = unit_ring_take(sh.ring, k, lane, ok);
      if (u < 0) break;
      const DecUnit w = dec_unit(p, u);
      const int qi = w.qb * p.R + i;
      const bool valid = h < p.G && qi < p.Nq && in_range(w.bg, static_cast<long long>(p.B) * p.Hkv) &&
                         in_range(w.s, p.S);
      const int b = w.bg / p.Hkv, g = w.bg - b * p.Hkv;
      const size_t qrow = (static_cast<size_t>(b) * p.Hq + g * p.G + h) * p.Nq + qi;   // global query row
      if (w.n == 0) {                  // no visible key in this split: an empty partial
        if (valid) {
          float* dst = p.opart + (qrow * p.S + w.s) * D + grp * OH;
          for (int x = 0; x < OH; x += 4) *reinterpret_cast<float4*>(dst + x) = make_float4(0.f, 0.f, 0.f, 0.f);
          if (grp == 0) p.lpart[qrow * p.S + w.s] = -INFINITY;
        }
        continue;
      }
      const int lastk = (p.causal && valid) ? min(p.Nk - 1, p.Nk - p.Nq + qi) : p.Nk - 1;
      float m_used = -INFINITY;
      uint64_t lsum = f2pack(0.f, 0.f);
      for (int j = 0; j < w.n && ok; ++j) {
        const int g2 = gs + j, xp = g2 & 1;
        const uint32_t s_base = lane_base + ((g2 & 1) ? C::kS1 : C::kS0) + grp * 64;
        ok = __all_sync(0xffffffffu, mbar_wait(&sh.s_full[g2 & 1], (g2 >> 1) & 1));
        if (!ok) break;
        tc_fence_after();
        const int lim = lastk - ((w.j0 + j) * 128 + grp * 64);     // last visible column
        const bool msk = __any_sync(0xffffffffu, lim < 63);
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
          if (msk) { mask16(r0, 0, lim); mask16(r1, 16, lim); mask16(r2, 32, lim); mask16(r3, 48, lim); }
#pragma unroll
          for (int kk = 0; kk < 16; kk += 8) {
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              mx4[e] = max3f(mx4[e], __uint_as_float(r0[kk + e]), __uint_as_float(r0[kk + e + 4]));
              mx4[e] = max3f(mx4[e], __uint_as_float(r1[kk + e]), __uint_as_float(r1[kk + e + 4]));
              mx4[e] = max3f(mx4[e], __uint_as_float(r2[kk + e]), __uint_as_float(r2[kk + e + 4]));
              mx4[e] = max3f(mx4[e], __uint_as_float(r3[kk + e]), __uint_as_float(r3[kk + e + 4]));
            }
          }
        }
        sh.xmax[xp][grp][row] = fmaxf(fmaxf(mx4[0], mx4[1]), fmaxf(mx4[2], mx4[3]));
        __syncwarp();
        if (lane == 0) mbar_arrive(&sh.xbar[xp]);
        ok = __all_sync(0xffffffffu, mbar_wait(&sh.xbar[xp], (g2 >> 1) & 1));
        if (!ok) break;
        const float mx = fmaxf(sh.xmax[xp][0][row], sh.xmax[xp][1][row]);
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
        // S(j) was issued before PV(j - 1) (and after PV(j - 2), which its commit covers):
        // wait for PV(j - 1) before rescaling O
        if (__any_sync(0xffffffffu, need && j > 0)) {
          ok = __all_sync(0xffffffffu, mbar_wait(&sh.pv_done, (g2 - 1) & 1));
          if (!ok) break;
          tc_fence_after();
#pragma unroll 1
          for (int q4 = 0; q4 < OH / 16; ++q4) {
            uint32_t o[16];
            tmem_ld16(o_base + q4 * 16, o);
            tmem_wait_ld();
            reg_fence(o);
#pragma unroll
            for (int kk = 0; kk < 16; ++kk) o[kk] = __float_as_uint(__uint_as_float(o[kk]) * alpha);
            tmem_st16(o_base + q4 * 16, o);
          }
        }
        const float mb = m_used == -INFINITY ? 0.f : m_used;
        const uint64_t nm2 = f2pack(-mb, -mb);
#pragma unroll
        for (int cc = 0; cc < 4; ++cc) {
          uint32_t r[16];
          tmem_ld16(s_base + cc * 16, r);
          tmem_wait_ld();
          reg_fence(r);
          if (msk) mask16(r, cc * 16, lim);
          uint32_t pk[8];
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            const uint64_t xx =
                ffma2(f2pack(__uint_as_float(r[2 * kk]), __uint_as_float(r[2 * kk + 1])), c2, nm2);
            float x0, x1;
            f2unpack(xx, x0, x1);
            // at d = 64 a 32 KB K/V tile takes about as long to stream as its 16384
            // exponentials take on MUFU: 2 pairs in 8 go to the FMA pipe, as in the forward
            float a0, a1;
            if (D == 64 && kk >= 6) {
              exp2_fma_pair(x0, x1, a0, a1);
            } else {
              a0 = ex2_approx(x0);
              a1 = ex2_approx(x1);
            }
            lsum = fadd2(lsum, f2pack(a0, a1));
            pk[kk] = pack_bf16x2(a0, a1);
          }
          tmem_st8(s_base + cc * 8, pk);
        }
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&sh.p_ready[g2 & 1]);
      }
      if (!ok) break;
      // epilogue: the two groups' sums, the last PV, O / l and the LSE of this split
      const int glast = gs + w.n - 1;
      float l0, l1;
      f2unpack(lsum, l0, l1);
      sh.xsum[grp][row] = l0 + l1;
      __syncwarp();
      if (lane == 0) mbar_arrive(&sh.sbar);
      ok = __all_sync(0xffffffffu, mbar_wait(&sh.sbar, uq & 1));
      if (!ok) break;
      const float l = sh.xsum[0][row] + sh.xsum[1][row];
      // pv_done completes once per step.  S(glast) covered PV(glast - 2) only, so the
      // phases of PV(glast - 1) and PV(glast) are waited for in turn (a parity wait
      // can only tell apart the phase in progress and the one before it).
      if (glast >= 1) ok = __all_sync(0xffffffffu, mbar_wait(&sh.pv_done, (glast - 1) & 1));
      if (ok) ok = __all_sync(0xffffffffu, mbar_wait(&sh.pv_done, glast & 1));
      if (!ok) break;
      tc_fence_after();
      const float inv_l = l > 0.f ? 1.f / l : 0.f;
      const float lse_s = l > 0.f ? (m_used + __log2f(l)) * 0.69314718055994531f : -INFINITY;
#pragma unroll 1
      for (int q4 = 0; q4 < OH / 16; ++q4) {
        uint32_t o[16];
        tmem_ld16(o_base + q4 * 16, o);
        tmem_wait_ld();
        reg_fence(o);
        if (!valid) continue;
        if (p.S == 1) {
          uint32_t pk[8];
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            pk[kk] = pack_bf16x2(__uint_as_float(o[2 * kk]) * inv_l, __uint_as_float(o[2 * kk + 1]) * inv_l);
          uint4* dst = reinterpret_cast<uint4*>(p.o + qrow * D + grp * OH + q4 * 16);
          dst[0] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
          dst[1] = make_uint4(pk[4], pk[5], pk[6], pk[7]);
        } else {
          float4* dst = reinterpret_cast<float4*>(p.opart + (qrow * p.S + w.s) * D + grp * OH + q4 * 16);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            dst[kk] = make_float4(__uint_as_float(o[4 * kk]) * inv_l, __uint_as_float(o[4 * kk + 1]) * inv_l,
                                  __uint_as_float(o[4 * kk + 2]) * inv_l, __uint_as_float(o[4 * kk + 3]) * inv_l);
        }
      }
      if (valid && grp == 0) {
        if (p.S == 1) p.lse[qrow] = lse_s;
        else p.lpart[qrow * p.S + w.s] = lse_s;
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sh.o_free);
      gs += w.n;
      ++uq;
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

// Merge of the S partials of every query row: one warp per row, D / 32 columns per lane.
template <int D>
__global__ void __launch_bounds__(256) attn_decode_merge_kernel(const float* __restrict__ opart,
                                                                const float* __restrict__ lpart,
                                                                __nv_bfloat16* __restrict__ o,
                                                                float* __restrict__ lse, long long rows, int S) {
  constexpr int PER = D / 32;
  const int lane = threadIdx.x & 31;
  const long long w0 = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const long long nw = (static_cast<long long>(gridDim.x) * blockDim.x) >> 5;
  for (long long r = w0; r < rows; r += nw) {
    const float* lp = lpart + r * S;
    float m = -INFINITY;
    for (int s = 0; s < S; ++s) m = fmaxf(m, lp[s]);
    float acc[PER];
#pragma unroll
    for (int x = 0; x < PER; ++x) acc[x] = 0.f;
    float wsum = 0.f;
    for (int s = 0; s < S; ++s) {
      const float ls = lp[s];
      const float w = ls == -INFINITY ? 0.f : ex2_approx((ls - m) * 1.4426950408889634f);
      wsum += w;
      const float* src = opart + (r * S + s) * D + lane * PER;
#pragma unroll
      for (int x = 0; x < PER; ++x) acc[x] = fmaf(w, src[x], acc[x]);
    }
    const float inv = 1.f / wsum;
    __nv_bfloat16* dst = o + r * D + lane * PER;
#pragma unroll
    for (int x = 0; x < PER; x += 2)
      *reinterpret_cast<uint32_t*>(dst + x) = pack_bf16x2(acc[x] * inv, acc[x + 1] * inv);
    if (lane == 0) lse[r] = m + __logf(wsum);
  }
}

}  // namespace attn

namespace attn {

// Merge of one partial result into a running one, for attention whose keys arrive in
// blocks (the ring of sequence shards across GPUs): with m = max(lse_acc, lse_part),
// a = exp(lse_acc - m), b = exp(lse_part - m):
//     o_acc <- (a o_acc + b o_part) / (a + b),   lse_acc <- m + ln(a + b)
// (page "attn-efficient", online-softmax section: the same rescale as the tiled
// loop, applied to whole blocks).  lse_acc = -inf marks an empty accumulator.
// o_acc is fp32 so that repeated merges round only once, when `out` (bf16) is given.
template <int D>
__global__ void __launch_bounds__(256) attn_merge_kernel(float* __restrict__ o_acc, float* __restrict__ lse_acc,
                                                         const __nv_bfloat16* __restrict__ o_part,
                                                         const float* __restrict__ lse_part,
                                                         __nv_bfloat16* __restrict__ out, long long rows) {
  constexpr int PER = D / 32;
  const int lane = threadIdx.x & 31;
  const long long w0 = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const long long nw = (static_cast<long long>(gridDim.x) * blockDim.x) >> 5;
  for (long long r = w0; r < rows; r += nw) {
    const float la = lse_acc[r], lb = lse_part[r];
    const float m = fmaxf(la, lb);
    const float a = la == -INFINITY ? 0.f : ex2_approx((la - m) * 1.4426950408889634f);
    const float b = lb == -INFINITY ? 0.f : ex2_approx((lb - m) * 1.4426950408889634f);
    const float inv = a + b > 0.f ? 1.f / (a + b) : 0.f;
    float* acc = o_acc + r * D + lane * PER;
    const __nv_bfloat16* part = o_part + r * D + lane * PER;
    float res[PER];
#pragma unroll
    for (int x = 0; x < PER; ++x) {
      const float prev = a > 0.f ? acc[x] : 0.f;     // an empty accumulator may hold anything
      res[x] = (a * prev + b * __bfloat162float(part[x])) * inv;
      acc[x] = res[x];
    }
    if (out) {
#pragma unroll
      for (int x = 0; x < PER; x += 2)
        *reinterpret_cast<uint32_t*>(out + r * D + lane * PER + x) = pack_bf16x2(res[x], res[x + 1]);
    }
    if (lane == 0) lse_acc[r] = a + b > 0.f ? m + __logf(a + b) : -INFINITY;
  }
}

// acc[i] += part[i] for i < n (fp32 accumulator, bf16 part), 8 elements per thread and
// iteration: one 16-byte load of the part, two of the accumulator.  n is a multiple of 8
// and both pointers are 16-byte aligned (checked on the host).
__global__ void __launch_bounds__(256) attn_accumulate_kernel(float* __restrict__ acc,
                                                              const __nv_bfloat16* __restrict__ part, long long n8) {
  const long long stride = static_cast<long long>(gridDim.x) * blockDim.x;
  for (long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; i < n8; i += stride) {
    const uint4 pv = reinterpret_cast<const uint4*>(part)[i];
    float4* a = reinterpret_cast<float4*>(acc) + 2 * i;
    float4 lo = a[0], hi = a[1];
    const uint32_t w[4] = {pv.x, pv.y, pv.z, pv.w};
    float f[8];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      f[2 * k] = __uint_as_float(w[k] << 16);             // bf16 -> fp32: the high half of the word
      f[2 * k + 1] = __uint_as_float(w[k] & 0xffff0000u);
    }
    lo.x += f[0]; lo.y += f[1]; lo.z += f[2]; lo.w += f[3];
    hi.x += f[4]; hi.y += f[5]; hi.z += f[6]; hi.w += f[7];
    a[0] = lo;
    a[1] = hi;
  }
}

}  // namespace attn
