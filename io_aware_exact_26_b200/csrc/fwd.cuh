// Forward exact attention for sm_100a: O = softmax(scale * Q K^T) V and LSE.
//
// Method (page "attention 的显存线性化" §三; page "attn-efficient", online-softmax
// section): Q is cut into 128-row tiles and K/V into 128-key tiles; for each
// query tile the key tiles stream through shared memory, S_ij = Q_i K_j^T is
// formed on chip, a running row max m and exp-sum l are updated, the partial
// output is rescaled by exp(m_old - m_new) when the max grows, and only O and the
// log-sum-exp leave the chip.  S and P never reach HBM.
//
// B200 mapping (one persistent CTA per SM, 192 threads):
//   warps 0-3  softmax warpgroup: thread = one query row = one TMEM lane.
//              tcgen05.ld the S row, row max / exp2 / row sum in registers,
//              P written back to TMEM as bf16 (aliasing S), O rescale, epilogue.
//   warp 4     TMA producer: Q tile (double buffered), K ring, V ring.
//   warp 5     MMA issuer (one thread): S = Q K^T (SS, both K-major) and
//              O += P V (A = P from TMEM, B = V MN-major), accumulating in TMEM.
// TMEM (512 columns): three 128-column S/P buffers, then O (D columns).  Three
// S buffers let S(j+1) be issued while P(j-1) may still be read by its PV MMA.
//
// exp2 with a folded scale: c = scale * log2(e), p = exp2(s*c - m) where m is
// kept in log2 units; LSE = ln(2) * (m + log2 l).  The max used for the
// exponent is allowed to be stale by up to kRescaleTau (log2 units): by shift
// invariance of softmax (page "attn-efficient": subtracting the same number from
// a whole score row leaves the result unchanged) any reference value works as
// long as O and l use the same one; this keeps p <= 2^tau and skips most O
// rescales.  Two row sums are kept: l of the bf16-rounded p that the PV MMA
// consumes (O is normalised by it, so a constant V comes out exactly), and the
// fp32 sum of the unrounded p, from which the LSE is formed.
#pragma once
#include "sm100.cuh"

namespace attn {

constexpr float kRescaleTau = 8.0f;

template <int D>
struct FwdCfg {
  static constexpr int BM = 128, BN = 128;
  static constexpr int kTile = 128 * D * 2;          // bytes of one 128 x D bf16 tile
  static constexpr int kBox = 128 * 128;             // bytes of one 128 x 64 swizzled box
  static constexpr int KST = (D == 128) ? 3 : 4;     // K ring stages
  static constexpr int VST = (D == 128) ? 2 : 4;     // V ring stages
  static constexpr int kSmem = (2 + KST + VST) * kTile + 1024;
  static constexpr int kThreads = 192;
  static constexpr int kTmemCols = 512;
  static constexpr int kOCol = 384;                  // O accumulator column
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
  uint64_t q_full[2], q_empty[2];
  uint64_t k_full[4], k_empty[4];
  uint64_t v_full[4], v_empty[4];
  uint64_t s_full[3], p_ready[3], pv_done[3];
  uint64_t o_free;
  uint64_t drain;
  uint32_t tmem_base;
};

// Work tile t -> (query tile, batch*head).  Causal: longest rows first.
__device__ __forceinline__ void fwd_tile_coords(const FwdParams& p, int t, int& qt, int& bh) {
  int BH = p.B * p.Hq;
  int r = t / BH;
  bh = t - r * BH;
  qt = p.causal ? (p.n_qtiles - 1 - r) : r;
}

__device__ __forceinline__ int fwd_n_kv(const FwdParams& p, int qt) {
  int n_kv_all = (p.N + 127) / 128;
  return p.causal ? (qt + 1) : n_kv_all;
}

template <int D>
__global__ void __launch_bounds__(192, 1)
    attn_fwd_kernel(const __grid_constant__ CUtensorMap tmq, const __grid_constant__ CUtensorMap tmk,
                    const __grid_constant__ CUtensorMap tmv, const FwdParams p) {
  using C = FwdCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  __shared__ FwdShared sh;
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem;                              // 2 tiles
  uint8_t* sK = smem + 2 * C::kTile;               // KST tiles
  uint8_t* sV = sK + C::KST * C::kTile;            // VST tiles

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int i = 0; i < 2; ++i) { mbar_init(&sh.q_full[i], 1); mbar_init(&sh.q_empty[i], 1); }
    for (int i = 0; i < C::KST; ++i) { mbar_init(&sh.k_full[i], 1); mbar_init(&sh.k_empty[i], 1); }
    for (int i = 0; i < C::VST; ++i) { mbar_init(&sh.v_full[i], 1); mbar_init(&sh.v_empty[i], 1); }
    for (int i = 0; i < 3; ++i) {
      mbar_init(&sh.s_full[i], 1);
      mbar_init(&sh.p_ready[i], 4);
      mbar_init(&sh.pv_done[i], 1);
    }
    mbar_init(&sh.o_free, 4);
    mbar_init(&sh.drain, 1);
    fence_barrier_init();
  }
  if (warp == 0) { tmem_alloc(&sh.tmem_base, C::kTmemCols); tmem_relinquish(); }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sh.tmem_base;

  if (warp == 4) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      tma_prefetch_desc(&tmq); tma_prefetch_desc(&tmk); tma_prefetch_desc(&tmv);
      int it = 0, tl = 0, nk = 0, nv = 0, nq = 0;
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
        // loads in the order the MMA warp consumes them: K0, K1, V0, K2, V1, ...
        for (int s = 0; s <= n_kv && ok; ++s) {
          if (s < n_kv) {
            const int g = it + s, st = g % C::KST;
            if (g >= C::KST) ok = mbar_wait(&sh.k_empty[st], ((g / C::KST) - 1) & 1);
            if (!ok) break;
            mbar_arrive_expect_tx(&sh.k_full[st], C::kTile);
            for (int c = 0; c < D / 64; ++c)
              tma_load_3d(sK + st * C::kTile + c * C::kBox, &tmk, &sh.k_full[st], c * 64, s * 128, bkv);
            nk = g + 1;
          }
          if (s >= 1) {
            const int g = it + s - 1, st = g % C::VST;
            if (g >= C::VST) ok = mbar_wait(&sh.v_empty[st], ((g / C::VST) - 1) & 1);
            if (!ok) break;
            mbar_arrive_expect_tx(&sh.v_full[st], C::kTile);
            for (int c = 0; c < D / 64; ++c)
              tma_load_3d(sV + st * C::kTile + c * C::kBox, &tmv, &sh.v_full[st], c * 64, (s - 1) * 128, bkv);
            nv = g + 1;
          }
        }
        it += n_kv;
      }
      if (!ok) {
        // Let the copies already in flight land before the CTA exits (bounded).
        for (int g = max(0, nk - C::KST); g < nk; ++g) mbar_drain_wait(&sh.k_full[g % C::KST], (g / C::KST) & 1);
        for (int g = max(0, nv - C::VST); g < nv; ++g) mbar_drain_wait(&sh.v_full[g % C::VST], (g / C::VST) & 1);
        for (int g = max(0, nq - 2); g < nq; ++g) mbar_drain_wait(&sh.q_full[g & 1], (g >> 1) & 1);
      }
    }
  } else if (warp == 5) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idS = idesc_bf16_f32(128, 128, false, false);
      constexpr uint32_t idO = idesc_bf16_f32(128, D, false, true);
      int it = 0, tl = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < p.total_tiles && ok; t += gridDim.x, ++tl) {
        int qt, bh;
        fwd_tile_coords(p, t, qt, bh);
        const int n_kv = fwd_n_kv(p, qt);
        const int qb = tl & 1;
        ok = mbar_wait(&sh.q_full[qb], (tl >> 1) & 1);
        if (!ok) break;
        tc_fence_after();
        const uint32_t q_addr = smem_u32(sQ + qb * C::kTile);
        for (int s = 0; s <= n_kv && ok; ++s) {
          if (s < n_kv) {
            // S(g) = Q K(g)^T into S buffer g % 3
            const int g = it + s, kst = g % C::KST, sb = g % 3;
            ok = mbar_wait(&sh.k_full[kst], (g / C::KST) & 1);
            if (ok && g >= 3) ok = mbar_wait(&sh.pv_done[sb], ((g / 3) - 1) & 1);
            if (!ok) break;
            tc_fence_after();
            const uint32_t k_addr = smem_u32(sK + kst * C::kTile);
#pragma unroll
            for (int k = 0; k < D / 16; ++k) {
              const uint32_t off = (k >> 2) * C::kBox + (k & 3) * 32;
              umma_ss(tmem + sb * 128, sdesc_sw128(q_addr + off, 16, 1024),
                      sdesc_sw128(k_addr + off, 16, 1024), idS, k > 0);
            }
            umma_commit(&sh.s_full[sb]);
            umma_commit(&sh.k_empty[kst]);
            if (s == n_kv - 1) umma_commit(&sh.q_empty[qb]);
          }
          if (s >= 1) {
            // O (+)= P(g) V(g)
            const int g = it + s - 1, vst = g % C::VST, sb = g % 3;
            ok = mbar_wait(&sh.v_full[vst], (g / C::VST) & 1);
            if (ok) ok = mbar_wait(&sh.p_ready[sb], (g / 3) & 1);
            if (ok && s == 1 && tl >= 1) ok = mbar_wait(&sh.o_free, (tl - 1) & 1);
            if (!ok) break;
            tc_fence_after();
            const uint32_t v_addr = smem_u32(sV + vst * C::kTile);
#pragma unroll
            for (int k = 0; k < 8; ++k)
              umma_ts(tmem + C::kOCol, tmem + sb * 128 + k * 8,
                      sdesc_sw128(v_addr + k * 2048, C::kBox, 1024), idO, (s > 1 || k > 0));
            umma_commit(&sh.pv_done[sb]);
            umma_commit(&sh.v_empty[vst]);
          }
        }
        it += n_kv;
      }
      // Drain every MMA this thread issued before TMEM is released.
      umma_commit(&sh.drain);
      mbar_wait(&sh.drain, 0);
    }
  } else {
    // ------------------------------------------------------------ softmax warpgroup
    const int row = warp * 32 + lane;                       // TMEM lane == tile row
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(warp * 32) << 16);
    const float c = p.c;
    int it = 0, tl = 0;
    bool ok = true;
    for (int t = blockIdx.x; t < p.total_tiles && ok; t += gridDim.x, ++tl) {
      int qt, bh;
      fwd_tile_coords(p, t, qt, bh);
      const int n_kv = fwd_n_kv(p, qt);
      const int qrow = qt * 128 + row;
      float m_used = -INFINITY, l = 0.f, l_exact = 0.f;
      for (int j = 0; j < n_kv && ok; ++j) {
        const int g = it + j, sb = g % 3;
        ok = __all_sync(0xffffffffu, mbar_wait(&sh.s_full[sb], (g / 3) & 1));
        if (!ok) break;
        tc_fence_after();
        uint32_t r[128];
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4)
          tmem_ld32(lane_base + sb * 128 + q4 * 32, *reinterpret_cast<uint32_t(*)[32]>(&r[q4 * 32]));
        tmem_wait_ld();
        // masking: causal diagonal tile and the ragged key tail
        const int kbase = j * 128;
        int lim = p.N - 1 - kbase;
        if (p.causal) lim = min(lim, qrow - kbase);
        if (lim < 127) {
#pragma unroll
          for (int k = 0; k < 128; ++k)
            if (k > lim) r[k] = __float_as_uint(-INFINITY);
        }
        // row max with 8 independent chains (one warp per SMSP: no other warp hides latency)
        float mx8[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) mx8[k] = __uint_as_float(r[k]);
#pragma unroll
        for (int k = 8; k < 128; ++k) mx8[k & 7] = fmaxf(mx8[k & 7], __uint_as_float(r[k]));
#pragma unroll
        for (int k = 0; k < 4; ++k) mx8[k] = fmaxf(mx8[k], mx8[k + 4]);
        const float mx = fmaxf(fmaxf(mx8[0], mx8[1]), fmaxf(mx8[2], mx8[3]));
        const float m_tile = mx * c;
        float alpha = 1.f;
        const bool need = (m_used == -INFINITY) || (m_tile > m_used + kRescaleTau);
        if (need) {
          const float m_new = fmaxf(m_used, m_tile);
          alpha = (m_used == -INFINITY) ? 0.f : ex2_approx(m_used - m_new);
          l *= alpha;
          l_exact *= alpha;
          m_used = m_new;
        }
        const float neg_m = -m_used;
        float lr[4] = {0.f, 0.f, 0.f, 0.f}, le[4] = {0.f, 0.f, 0.f, 0.f};   // independent partial sums
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4) {
          uint32_t pk[16];
#pragma unroll
          for (int k = 0; k < 16; ++k) {
            const float a = ex2_approx(fmaf(__uint_as_float(r[q4 * 32 + 2 * k]), c, neg_m));
            const float b = ex2_approx(fmaf(__uint_as_float(r[q4 * 32 + 2 * k + 1]), c, neg_m));
            __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
            lr[k & 3] += __low2float(h) + __high2float(h);
            le[k & 3] += a + b;
            pk[k] = *reinterpret_cast<uint32_t*>(&h);
          }
          tmem_st16(lane_base + sb * 128 + q4 * 16, pk);
        }
        l += (lr[0] + lr[1]) + (lr[2] + lr[3]);
        l_exact += (le[0] + le[1]) + (le[2] + le[3]);
        // Rescale the running output when this warp's max moved (rare after the first tiles).
        if (__any_sync(0xffffffffu, need && j > 0)) {
          const int gp = g - 1;
          ok = __all_sync(0xffffffffu, mbar_wait(&sh.pv_done[gp % 3], (gp / 3) & 1));
          if (!ok) break;
          tc_fence_after();
#pragma unroll
          for (int q4 = 0; q4 < D / 32; ++q4) {
            uint32_t o[32];
            tmem_ld32(lane_base + C::kOCol + q4 * 32, o);
            tmem_wait_ld();
#pragma unroll
            for (int k = 0; k < 32; ++k) o[k] = __float_as_uint(__uint_as_float(o[k]) * alpha);
            tmem_st32(lane_base + C::kOCol + q4 * 32, o);
          }
        }
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&sh.p_ready[sb]);
      }
      if (!ok) break;
      // epilogue: wait for the last PV, O / l -> bf16, LSE
      const int glast = it + n_kv - 1;
      ok = __all_sync(0xffffffffu, mbar_wait(&sh.pv_done[glast % 3], (glast / 3) & 1));
      if (!ok) break;
      tc_fence_after();
      const float inv_l = 1.f / l;
      const bool live = qrow < p.N;
      __nv_bfloat16* orow = reinterpret_cast<__nv_bfloat16*>(p.o) + (static_cast<size_t>(bh) * p.N + qrow) * D;
#pragma unroll
      for (int q4 = 0; q4 < D / 32; ++q4) {
        uint32_t o[32];
        tmem_ld32(lane_base + C::kOCol + q4 * 32, o);
        tmem_wait_ld();
        uint32_t pk[16];
#pragma unroll
        for (int k = 0; k < 16; ++k)
          pk[k] = pack_bf16x2(__uint_as_float(o[2 * k]) * inv_l, __uint_as_float(o[2 * k + 1]) * inv_l);
        if (live) {
          uint4* dst = reinterpret_cast<uint4*>(orow + q4 * 32);
#pragma unroll
          for (int k = 0; k < 4; ++k) dst[k] = make_uint4(pk[4 * k], pk[4 * k + 1], pk[4 * k + 2], pk[4 * k + 3]);
        }
      }
      if (live) p.lse[static_cast<size_t>(bh) * p.N + qrow] = (m_used + __log2f(l_exact)) * 0.69314718055994531f;
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sh.o_free);
      it += n_kv;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, C::kTmemCols);
  }
}

}  // namespace attn
