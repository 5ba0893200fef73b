// Backward exact attention for sm_100a: dQ, dK, dV of sum(O * dO).
//
// Recompute instead of store (page "attention 的显存线性化" §五; page
// "attn-efficient", recompute paragraph): the forward keeps only O and the
// log-sum-exp; every S/P tile is rebuilt on chip from Q, K and the saved LSE.
// Gradient formulas (chain rule through the row softmax; the pages state none):
// with D_i = sum_k dO_ik O_ik,
//   P = exp(scale Q K^T - LSE),  dV = P^T dO,  dP = dO V^T,
//   dS = P * (dP - D),  dQ = scale dS K,  dK = scale dS^T Q.
//
// Kernels
//   bwd_prep : one row per D/8 lanes: D_i and LSE in log2 units, both stored negated.
//   bwd_kv   : persistent; one work item = (b, kv-head, 128-key tile j).  K_j, V_j
//              stay in shared memory while the item walks its G q-heads and the
//              query tiles that see tile j; dK_j and dV_j accumulate in TMEM and are
//              written once.
//   bwd_q    : persistent; one work item = (b, q-head, 128-query tile i).  Q_i, dO_i
//              stay in shared memory while the item walks the key tiles tile i sees;
//              dQ_i accumulates in TMEM and is written once.
// Splitting dQ from dK/dV costs a second recompute of S and dP (7 instead of 5
// tile contractions per query/key tile pair) but removes every cross-CTA
// reduction: no atomics, no ordering, no fp32 scratch for dQ, and each output is
// summed by one CTA in a fixed order, so results are bitwise reproducible.
//
// Every tcgen05.mma here has M = 128 and N >= 128 where the head dim allows it
// (an M = 128, N = 64 MMA takes as long as N = 128 on this part).
#pragma once
#include "sm100.cuh"

namespace attn {

// Untiled bulk copy global -> shared (both 16-byte aligned, size a multiple of 16).
__device__ __forceinline__ void bulk_load(void* smem_dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                   smem_u32(smem_dst)),
               "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(smem_u32(bar))
               : "memory");
}

struct BwdLayout {
  // workspace carve-up (byte offsets, each 256-byte aligned): -lse2 and -D per row
  size_t nlse2_off, ndd_off, total;
};

__host__ __device__ inline BwdLayout bwd_layout(long long BHq, int N) {
  const long long npad = (N + 127) / 128 * 128;
  auto up = [](size_t x) { return (x + 255) / 256 * 256; };
  BwdLayout L;
  L.nlse2_off = 0;
  L.ndd_off = up(L.nlse2_off + BHq * npad * 4);
  L.total = up(L.ndd_off + BHq * npad * 4);
  return L;
}

inline size_t bwd_workspace_bytes(int B, int Hq, int Hkv, int N, int d) {
  (void)Hkv;
  (void)d;
  return bwd_layout(static_cast<long long>(B) * Hq, N).total;
}

// ------------------------------------------------------------------ preprocess
// D_i = sum_k dO_ik O_ik (fp32) and lse2_i = LSE_i * log2(e), both stored negated (the
// dS warps add them with packed f32x2 FMAs and adds, which take no negated operand);
// padded rows get 0.
// Each row is read with 16-byte loads by D/8 lanes, so one warp covers 256/D rows.
template <int D>
__global__ void __launch_bounds__(256) attn_bwd_prep_kernel(const __nv_bfloat16* __restrict__ o,
                                                            const __nv_bfloat16* __restrict__ dO,
                                                            const float* __restrict__ lse, float* nlse2,
                                                            float* ndd, long long BHq, int N) {
  constexpr int LPR = D / 8;             // lanes per row
  constexpr int RPW = 32 / LPR;          // rows per warp pass
  const int npad = (N + 127) / 128 * 128;
  const long long rows = BHq * npad;
  const int lane = threadIdx.x & 31;
  const int sub = lane / LPR, part = lane % LPR;
  const long long warp0 = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const long long nwarps = (static_cast<long long>(gridDim.x) * blockDim.x) >> 5;
  for (long long r0 = warp0 * RPW; r0 < rows; r0 += nwarps * RPW) {
    const long long r = r0 + sub;
    float acc = 0.f, l2 = 0.f;
    bool live = false;
    long long bh = 0;
    int n = 0;
    if (r < rows) {
      bh = r / npad;
      n = static_cast<int>(r - bh * npad);
      live = n < N;
    }
    if (live) {
      const size_t base = (static_cast<size_t>(bh) * N + n) * D + part * 8;
      const uint4 a = *reinterpret_cast<const uint4*>(o + base);
      const uint4 b = *reinterpret_cast<const uint4*>(dO + base);
      const __nv_bfloat162* pa = reinterpret_cast<const __nv_bfloat162*>(&a);
      const __nv_bfloat162* pb = reinterpret_cast<const __nv_bfloat162*>(&b);
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const float2 fa = __bfloat1622float2(pa[k]), fb = __bfloat1622float2(pb[k]);
        acc = fmaf(fa.x, fb.x, acc);
        acc = fmaf(fa.y, fb.y, acc);
      }
      l2 = lse[static_cast<size_t>(bh) * N + n] * 1.4426950408889634f;
    }
#pragma unroll
    for (int off = LPR / 2; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
    if (part == 0 && r < rows) {
      ndd[r] = -acc;
      nlse2[r] = -l2;
    }
  }
}

struct BwdParams {
  __nv_bfloat16* dq;
  __nv_bfloat16* dk;
  __nv_bfloat16* dv;
  const float* nlse2;   // -LSE * log2(e) per row (padded to whole tiles)
  const float* ndd;     // -D per row
  int B, Hq, Hkv, N, G;
  int nt;           // number of 128-row tiles along N
  int npair;        // (nt + 1) / 2: key-tile pairs per KV head (causal dK/dV units)
  int total_items;
  int wl, wr;       // window: query i sees keys i - wl .. i + wr (0 <= wl, wr <= N)
  int pair;         // causal (wl = N, wr = 0): dK/dV units are pairs of key tiles
  int desc;         // dQ items list query tiles last-first (key ranges grow with the tile)
  float c;          // scale * log2(e)
  float scale;
};

// Exps of one 16-column slice of a score tile held by this thread, two columns per
// packed f32x2 instruction: p = 2^(s c + nl) with nl = -lse2 (the column's or the
// row's).  Masked columns (only on band-edge / ragged tiles) get s = -inf first; c > 0
// (the host floors it at 1e-30), so p = 0 (or 2^-126.5 on the FMA-pipe path); the exp
// loop itself has no branch.  pf2[k] holds columns 2k and 2k+1.  One pair in four
// goes to the FMA pipe, one in two at d = 64 (measured: +2-3% there, no change at
// d = 128 for none, one or two in four).
template <int D>
__device__ __forceinline__ void bwd_exp16(uint32_t (&sr)[16], const uint64_t (&nl)[8], uint64_t c2, bool masked,
                                          int col0, int lo, int hi, uint64_t* pf2) {
  if (masked) {
#pragma unroll
    for (int k = 0; k < 16; ++k)
      if (col0 + k < lo || col0 + k > hi) sr[k] = 0xff800000u;
  }
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    const uint64_t x = ffma2(f2pack(__uint_as_float(sr[2 * k]), __uint_as_float(sr[2 * k + 1])), c2, nl[k]);
    float x0, x1, y0, y1;
    f2unpack(x, x0, x1);
    if (D == 64 ? (k & 1) == 1 : (k & 3) == 3) {
      exp2_fma_pair(x0, x1, y0, y1);
    } else {
      y0 = ex2_approx(x0);
      y1 = ex2_approx(x1);
    }
    pf2[k] = f2pack(y0, y1);
  }
}

// ================================================================== bwd_kv
template <int D>
struct KvCfg {
  static constexpr int kTile = 128 * D * 2;
  static constexpr int kBox = 128 * 128;
  static constexpr int kGroups = 2;                      // dS warpgroups: kCols queries of every step each
  static constexpr int kCols = 128 / kGroups;
  static constexpr int kDsWarps = 4 * kGroups;
  static constexpr int kWarpLoad = kDsWarps, kWarpMma = kDsWarps + 1;
  static constexpr int kThreads = 32 * (kDsWarps + 2);   // dS warps, TMA, MMA
  // TMEM columns: S^T (lane = key, column = query), P^T as bf16 over it (warpgroup g
  // packs its kCols queries into the first kCols / 2 of the columns it read, so it
  // overwrites only columns it has read); dP^T with dS^T as bf16 over it (same
  // placement); dV and dK accumulators (D columns each).  At d = 64 the accumulators
  // leave 128 columns free for a second S^T buffer (step g uses buffer g % 2), so S^T of
  // the next step is computed while the exponentials of this one run; at d = 128 there
  // is one buffer and S^T(g+1) follows dV(g), which reads P^T(g) from it.
  static constexpr int SB = (D == 64) ? 2 : 1;           // S^T buffers
  static constexpr int kS = 0, kDP = 128, kDV = 256, kDK = 256 + D, kS1 = 256 + 2 * D;
  static_assert(SB == 1 || kS1 + 128 <= 512, "second S^T buffer must fit in TMEM");
  static constexpr int kTmemCols = 512;
  static constexpr int kOffK = 0, kOffV = kTile;
  static constexpr int kOffQ = 2 * kTile;                // 2 stages
  static constexpr int kOffDO = 4 * kTile;               // 2 stages
  static constexpr int kOffVec = 6 * kTile;              // per stage: -lse2[128], -D[128]
  static constexpr int kOffBar = kOffVec + 2048;
  static constexpr int kLayout = kOffBar + 256;
  static constexpr int kSmem = kLayout + 1024;
  static_assert(kSmem <= 232448, "shared memory layout exceeds 227 KB");
};

struct KvShared {
  uint64_t kv_full, kv_empty;
  uint64_t qdo_full[2], qdo_empty[2];
  uint64_t s_full[2], dp_full;  // S^T of the step (in buffer step % SB) / dP^T in TMEM
  // P^T (bf16) written back by both dS warpgroups, one barrier per S^T buffer (step g
  // uses p_ready[g % SB]).  With two buffers S^T(g+1) is ready before dV(g) is issued,
  // so a fast warp can finish the exponentials of step g+1 before a slow one has
  // arrived for step g; on a single barrier that early arrival would complete step g's
  // phase with one of its warps' P^T columns still unwritten.  Per buffer, a warp's
  // next arrival on the same barrier is two steps later, after S^T(g+2), which is
  // issued behind dV(g).
  uint64_t p_ready[2];
  uint64_t ds_ready;            // dS^T (bf16) written back by both dS warpgroups
  uint64_t p_half;              // one S^T buffer: the first half of each warpgroup's P^T written
  uint64_t k_done;              // dK MMA of the step complete (the item's last one ends it)
  uint64_t acc_free;            // dV / dK of the previous item read out
  uint64_t drain;
  uint32_t tmem_base;
};
static_assert(sizeof(KvShared) <= 256, "KvShared does not fit its slot");

// Work units of the dK/dV kernel, numbered KV head by KV head, so the CTAs running at
// the same time stream the Q/dO of the same few head groups.
//  - In general unit t is key tile j = t mod nt, one item, walking its query tiles
//    from the last one down.
//  - Causal: unit t is the pair of key tiles (pr, nt-1-pr), two items (one for the
//    middle tile when nt is odd). Together they see nt+1 query tiles whatever pr is,
//    so units cost the same and the CTAs that start them together stay in step.
//    The first item walks its query tiles from the last one down, the second from
//    its diagonal tile up: at step T of a unit the CTAs of one head group read
//    query tile nt-1-T or T-1, so each Q/dO tile reaches L2 from HBM about twice
//    per group instead of once per key tile.
__device__ __forceinline__ int kv_halves(const BwdParams& p, int t) {
  if (!p.pair) return 1;
  const int pr = t % p.npair;
  return 2 * pr + 1 == p.nt ? 1 : 2;
}
__device__ __forceinline__ void kv_item(const BwdParams& p, int t, int hf, int& bhkv, int& j, bool& up) {
  if (!p.pair) {
    bhkv = t / p.nt;
    j = t - bhkv * p.nt;
    up = false;
    return;
  }
  bhkv = t / p.npair;
  const int pr = t - bhkv * p.npair;
  j = hf ? p.nt - 1 - pr : pr;
  up = hf != 0;
}
// Query tiles [i0, i1] that see key tile j: queries i with key - wr <= i <= key + wl.
__device__ __forceinline__ void kv_q_range(const BwdParams& p, int j, int& i0, int& i1) {
  const int k0 = j * 128, k1 = min(p.N - 1, k0 + 127);
  i0 = max(0, k0 - p.wr) >> 7;
  i1 = min(p.N - 1, k1 + p.wl) >> 7;
}
// s-th query tile an item visits, s in [0, i1 - i0]
__device__ __forceinline__ int kv_q_tile(int i0, int i1, bool up, int s) { return up ? i0 + s : i1 - s; }

// TMEM column of the k-th 16-element slice of a packed bf16 operand written by
// warpgroups of `cols` fp32 columns each (see the TMEM plans of the configs).
__device__ __forceinline__ constexpr uint32_t packed_col(int k, int cols) {
  return static_cast<uint32_t>(cols * (k / (cols / 16)) + (k % (cols / 16)) * 8);
}

template <int D>
__global__ void __launch_bounds__(KvCfg<D>::kThreads, 1)
    attn_bwd_kv_kernel(const __grid_constant__ CUtensorMap tmq, const __grid_constant__ CUtensorMap tmk,
                       const __grid_constant__ CUtensorMap tmv, const __grid_constant__ CUtensorMap tmdo,
                       const BwdParams p) {
  using C = KvCfg<D>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  KvShared& sh = *reinterpret_cast<KvShared*>(smem + C::kOffBar);
  uint8_t* sK = smem + C::kOffK;
  uint8_t* sV = smem + C::kOffV;
  uint8_t* sQ = smem + C::kOffQ;
  uint8_t* sDO = smem + C::kOffDO;
  float* sVec = reinterpret_cast<float*>(smem + C::kOffVec);   // [stage][-lse2 128 | -D 128]

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    mbar_init(&sh.kv_full, 1);
    mbar_init(&sh.kv_empty, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&sh.qdo_full[i], 1);
      mbar_init(&sh.qdo_empty[i], 1);
    }
    mbar_init(&sh.s_full[0], 1);
    mbar_init(&sh.s_full[1], 1);
    mbar_init(&sh.dp_full, 1);
    mbar_init(&sh.p_ready[0], C::kDsWarps);
    mbar_init(&sh.p_ready[1], C::kDsWarps);
    mbar_init(&sh.p_half, C::kDsWarps);
    mbar_init(&sh.ds_ready, C::kDsWarps);
    mbar_init(&sh.k_done, 1);
    mbar_init(&sh.acc_free, C::kDsWarps);
    mbar_init(&sh.drain, 1);
    fence_barrier_init();
  }
  if (warp == 0) { tmem_alloc(&sh.tmem_base, C::kTmemCols); tmem_relinquish(); }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sh.tmem_base;

  if (warp == C::kWarpLoad) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      tma_prefetch_desc(&tmq); tma_prefetch_desc(&tmk); tma_prefetch_desc(&tmv); tma_prefetch_desc(&tmdo);
      const uint64_t pol_reuse = l2_policy_evict_last(), pol_once = l2_policy_evict_first();
      int gs = 0, it = 0, nq = 0, nkv = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < p.total_items && ok; t += gridDim.x)
      for (int hf = 0; hf < kv_halves(p, t) && ok; ++hf, ++it) {
        int bhkv, j;
        bool up;
        kv_item(p, t, hf, bhkv, j, up);
        if (it >= 1) ok = mbar_wait(&sh.kv_empty, (it - 1) & 1);
        if (!ok) break;
        mbar_arrive_expect_tx(&sh.kv_full, 2 * C::kTile);
        in_range(j, p.nt);
        in_range(bhkv, static_cast<long long>(p.B) * p.Hkv);
        for (int c = 0; c < D / 64; ++c) {                  // K_j, V_j: read by this item only
          tma_load_3d_hint(sK + c * C::kBox, &tmk, &sh.kv_full, c * 64, j * 128, bhkv, pol_once);
          tma_load_3d_hint(sV + c * C::kBox, &tmv, &sh.kv_full, c * 64, j * 128, bhkv, pol_once);
        }
        nkv = it + 1;
        const int b = bhkv / p.Hkv, hk = bhkv - b * p.Hkv;
        // Query tiles in the item's order, the G heads of the group inside.
        int i0, i1;
        kv_q_range(p, j, i0, i1);
        for (int s = 0; s <= i1 - i0 && ok; ++s) {
          const int i = kv_q_tile(i0, i1, up, s);
          for (int h = 0; h < p.G; ++h, ++gs) {
            const int bhq = b * p.Hq + hk * p.G + h;
            const int st = gs & 1;
            if (gs >= 2) ok = mbar_wait(&sh.qdo_empty[st], ((gs >> 1) - 1) & 1);
            if (!ok) break;
            mbar_arrive_expect_tx(&sh.qdo_full[st], 2 * C::kTile + 1024);
            for (int c = 0; c < D / 64; ++c) {              // Q_i, dO_i: read by every key tile's item
              tma_load_3d_hint(sQ + st * C::kTile + c * C::kBox, &tmq, &sh.qdo_full[st], c * 64, i * 128, bhq,
                               pol_reuse);
              tma_load_3d_hint(sDO + st * C::kTile + c * C::kBox, &tmdo, &sh.qdo_full[st], c * 64, i * 128, bhq,
                               pol_reuse);
            }
            size_t vrow = static_cast<size_t>(bhq) * (p.nt * 128) + i * 128;
            in_range(i, p.nt);
            if (!in_range(bhq, static_cast<long long>(p.B) * p.Hq)) vrow = 0;   // keep the bulk copy inside
            bulk_load(sVec + st * 256, p.nlse2 + vrow, 512, &sh.qdo_full[st]);
            bulk_load(sVec + st * 256 + 128, p.ndd + vrow, 512, &sh.qdo_full[st]);
            nq = gs + 1;
          }
        }
      }
      if (!ok) {
        if (nkv >= 1) mbar_drain_wait(&sh.kv_full, (nkv - 1) & 1);
        for (int g = max(0, nq - 2); g < nq; ++g) mbar_drain_wait(&sh.qdo_full[g & 1], (g >> 1) & 1);
      }
    }
  } else if (warp == C::kWarpMma) {
    // ------------------------------------------------------------ MMA issuer
    // Order per step g:  dV(g) S^T(g+1) dK(g) dP^T(g+1) with one S^T buffer (d = 128),
    // S^T(g+1) dV(g) dK(g) dP^T(g+1) with two (d = 64).  The exps of step g+1 (phase A)
    // run under dK(g) and dP^T(g+1); dS of step g (phase B) under dV(g) and S^T(g+1).
    // The whole warp follows the schedule (descriptor arithmetic stays warp-uniform);
    // one lane, elected once, issues every MMA and commit.
    const bool leader = elect_one();
    constexpr uint32_t idST = idesc_bf16_f32(128, 128, false, false);   // S^T, dP^T
    constexpr uint32_t idKV = idesc_bf16_f32(128, D, false, true);      // dV, dK
    constexpr uint32_t hi = sdesc_hi_sw128(1024);
    const uint32_t k_lo = sdesc_lo(smem_u32(sK), 16), v_lo = sdesc_lo(smem_u32(sV), 16);
    const uint32_t q_lo0 = sdesc_lo(smem_u32(sQ), 16), do_lo0 = sdesc_lo(smem_u32(sDO), 16);
    const uint32_t q_mn0 = sdesc_lo(smem_u32(sQ), C::kBox), do_mn0 = sdesc_lo(smem_u32(sDO), C::kBox);
    auto wait = [&](uint64_t* bar, uint32_t parity) -> bool {
      return __all_sync(0xffffffffu, mbar_wait(bar, parity));
    };
    int gs = 0, it = 0;
    bool ok = true;
    auto issue_st = [&](int g) -> bool {   // S^T(g) = K Q(g)^T into buffer g % SB
      const int st = g & 1, sb = g % C::SB;
      if (!wait(&sh.qdo_full[st], (g >> 1) & 1)) return false;
      // S^T(g) overwrites P^T(g - SB): issued behind dV(g - SB) by this thread, which the
      // tensor cores perform first (MMAs of one thread run in issue order).
      tc_fence_after();
      if (leader) {
        const uint32_t q_lo = q_lo0 + st * (C::kTile >> 4);
#pragma unroll
        for (int k = 0; k < D / 16; ++k) {
          const uint32_t off = ((k >> 2) * C::kBox + (k & 3) * 32) >> 4;
          umma_ss_lo(tmem + (sb ? C::kS1 : C::kS), k_lo + off, q_lo + off, hi, idST, k > 0);
        }
        umma_commit(&sh.s_full[sb]);
      }
      __syncwarp();
      return true;
    };
    auto issue_dp = [&](int g) -> bool {   // dP^T(g) = V dO(g)^T
      const int st = g & 1;
      // dP^T(g) overwrites dS^T(g-1): issued behind dK(g-1), performed after it.
      tc_fence_after();
      if (leader) {
        const uint32_t do_lo = do_lo0 + st * (C::kTile >> 4);
#pragma unroll
        for (int k = 0; k < D / 16; ++k) {
          const uint32_t off = ((k >> 2) * C::kBox + (k & 3) * 32) >> 4;
          umma_ss_lo(tmem + C::kDP, v_lo + off, do_lo + off, hi, idST, k > 0);
        }
        umma_commit(&sh.dp_full);
      }
      __syncwarp();
      return true;
    };
    for (int t = blockIdx.x; t < p.total_items && ok; t += gridDim.x)
    for (int hf = 0; hf < kv_halves(p, t) && ok; ++hf, ++it) {
      int bhkv, j;
      bool up;
      kv_item(p, t, hf, bhkv, j, up);
      ok = wait(&sh.kv_full, it & 1);
      if (!ok) break;
      int i0, i1;
      kv_q_range(p, j, i0, i1);
      const int n_steps = p.G * (i1 - i0 + 1);
      ok = issue_st(gs) && issue_dp(gs);
      for (int u = 0; u < n_steps && ok; ++u, ++gs) {
        const int st = gs & 1;
        // Two S^T buffers: S^T(g+1) goes first, into the buffer dV(g-1) has finished
        // with, and runs under the exponentials of step g.
        if (C::SB == 2 && u + 1 < n_steps && !issue_st(gs + 1)) { ok = false; break; }
        // dV += P^T dO  (A = P^T in TMEM, K = queries; B = dO MN-major).  With one S^T
        // buffer dV is on the chain P^T(g) -> dV(g) -> S^T(g+1) -> exponentials of g+1, so
        // it goes out in two halves: queries 0-31 and 64-95 as soon as each warpgroup has
        // written its first 32 (p_half), under the rest of the exponentials, and the other
        // half on p_ready (measured +6% on the long causal backward; with two buffers, at
        // d = 64, the split measured 1% slower and is not used).
        if constexpr (C::SB == 1) {
          ok = wait(&sh.p_half, gs & 1);
          if (ok && u == 0 && it >= 1) ok = wait(&sh.acc_free, (it - 1) & 1);
          if (!ok) break;
#pragma unroll 1
          for (int half = 0; half < 2 && ok; ++half) {
            if (half == 1) ok = wait(&sh.p_ready[gs % C::SB], (gs / C::SB) & 1);
            if (!ok) break;
            tc_fence_after();
            if (leader) {
              const uint32_t do_mn = do_mn0 + st * (C::kTile >> 4);
#pragma unroll
              for (int kk = 0; kk < 4; ++kk) {
                const int k = (kk >> 1) * 4 + half * 2 + (kk & 1);
                umma_ts_lo(tmem + C::kDV, tmem + C::kS + packed_col(k, C::kCols), do_mn + ((k * 2048) >> 4), hi,
                           idKV, !(u == 0 && k == 0));
              }
            }
            __syncwarp();
          }
          if (!ok) break;
        } else {
          ok = wait(&sh.p_ready[gs % C::SB], (gs / C::SB) & 1);
          if (ok && u == 0 && it >= 1) ok = wait(&sh.acc_free, (it - 1) & 1);
          if (!ok) break;
          tc_fence_after();
          if (leader) {
            const uint32_t do_mn = do_mn0 + st * (C::kTile >> 4);
            const uint32_t pcol = (gs % C::SB) ? C::kS1 : C::kS;
#pragma unroll
            for (int k = 0; k < 8; ++k)
              umma_ts_lo(tmem + C::kDV, tmem + pcol + packed_col(k, C::kCols), do_mn + ((k * 2048) >> 4), hi,
                         idKV, !(u == 0 && k == 0));
          }
          __syncwarp();
        }
        if (C::SB == 1 && u + 1 < n_steps && !issue_st(gs + 1)) { ok = false; break; }
        // dK += dS^T Q  (A = dS^T in TMEM; B = Q MN-major)
        ok = wait(&sh.ds_ready, gs & 1);
        if (!ok) break;
        tc_fence_after();
        if (leader) {
          const uint32_t q_mn = q_mn0 + st * (C::kTile >> 4);
#pragma unroll
          for (int k = 0; k < 8; ++k)
            umma_ts_lo(tmem + C::kDK, tmem + C::kDP + packed_col(k, C::kCols), q_mn + ((k * 2048) >> 4), hi,
                       idKV, !(u == 0 && k == 0));
          umma_commit(&sh.k_done);
          umma_commit(&sh.qdo_empty[st]);
        }
        __syncwarp();
        if (u + 1 < n_steps && !issue_dp(gs + 1)) { ok = false; break; }
      }
      if (!ok) break;
      if (leader) umma_commit(&sh.kv_empty);
      __syncwarp();
    }
    if (leader) {
      umma_commit(&sh.drain);
      mbar_wait(&sh.drain, 0);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ dS warpgroups (rows = keys)
    // warpgroup hb (warps 4hb .. 4hb+3): queries kCols*hb .. kCols*hb + kCols-1 of
    // every step; in the item's epilogue the first half of the warpgroups writes dV,
    // the second half dK.
    constexpr int CW = C::kCols;
    const int hb = warp >> 2;
    const int r = (warp & 3) * 32 + lane;
    const uint32_t lane_base = tmem + (static_cast<uint32_t>((warp & 3) * 32) << 16);
    const uint64_t c2 = f2pack(p.c, p.c);
    int gs = 0;
    bool ok = true;
    for (int t = blockIdx.x; t < p.total_items && ok; t += gridDim.x)
    for (int hf = 0; hf < kv_halves(p, t) && ok; ++hf) {
      int bhkv, j;
      bool up;
      kv_item(p, t, hf, bhkv, j, up);
      const int key = j * 128 + r;
      const bool key_live = key < p.N;
      int i0, i1;
      kv_q_range(p, j, i0, i1);
      for (int s = 0; s <= i1 - i0 && ok; ++s) {
        const int i = kv_q_tile(i0, i1, up, s);
        for (int h = 0; h < p.G && ok; ++h, ++gs) {
          const int st = gs & 1;
          const float* sNlse = sVec + st * 256 + CW * hb;
          const float* sNdd = sNlse + 128;
          // visible query columns (relative to this warpgroup's CW) for this key row:
          // queries key - wr .. key + wl
          const int qbase = i * 128 + CW * hb;
          const int hi = key_live ? (min(p.N - 1, key + p.wl) - qbase) : -1;
          const int lo = key - p.wr - qbase;
          const bool masked = !__all_sync(0xffffffffu, lo <= 0 && hi >= CW - 1);
          ok = __all_sync(0xffffffffu, mbar_wait(&sh.qdo_full[st], (gs >> 1) & 1));
          if (ok) ok = __all_sync(0xffffffffu, mbar_wait(&sh.s_full[gs % C::SB], (gs / C::SB) & 1));
          if (!ok) break;
          tc_fence_after();
          // ---- phase A: P^T = exp2(S^T c - lse2); bf16 into TMEM, fp32 pairs kept for phase B
          const uint32_t sbuf = (gs % C::SB) ? C::kS1 : C::kS;
          uint64_t pf2[CW / 2];
#pragma unroll
          for (int q16 = 0; q16 < CW / 16; ++q16) {
            uint32_t sr[16];
            tmem_ld16(lane_base + sbuf + CW * hb + q16 * 16, sr);
            uint64_t nl[8];
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              const ulonglong2 a = reinterpret_cast<const ulonglong2*>(sNlse + q16 * 16)[k];
              nl[2 * k] = a.x;
              nl[2 * k + 1] = a.y;
            }
            tmem_wait_ld();
            reg_fence(sr);
            bwd_exp16<D>(sr, nl, c2, masked, q16 * 16, lo, hi, pf2 + q16 * 8);
            uint32_t pk[8];
#pragma unroll
            for (int k = 0; k < 8; ++k) pk[k] = pack_bf16x2_2(pf2[q16 * 8 + k]);
            if (C::SB == 1 && q16 == 2) {
              // chunks 0 and 1 were stored a chunk ago: the first half of dV can start
              tmem_wait_st();
              tc_fence_before();
              __syncwarp();
              if (lane == 0) mbar_arrive(&sh.p_half);
            }
            tmem_st8(lane_base + sbuf + CW * hb + q16 * 8, pk);
          }
          tmem_wait_st();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&sh.p_ready[gs % C::SB]);
          // ---- phase B: dS^T = P^T (dP^T - D); bf16 into TMEM over dP^T
          ok = __all_sync(0xffffffffu, mbar_wait(&sh.dp_full, gs & 1));
          if (!ok) break;
          tc_fence_after();
#pragma unroll
          for (int q16 = 0; q16 < CW / 16; ++q16) {
            uint32_t dr[16];
            tmem_ld16(lane_base + C::kDP + CW * hb + q16 * 16, dr);
            uint64_t nd[8];
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              const ulonglong2 b = reinterpret_cast<const ulonglong2*>(sNdd + q16 * 16)[k];
              nd[2 * k] = b.x;
              nd[2 * k + 1] = b.y;
            }
            tmem_wait_ld();
            reg_fence(dr);
            uint32_t dk[8];
#pragma unroll
            for (int k = 0; k < 8; ++k)
              dk[k] = pack_bf16x2_2(fmul2(pf2[q16 * 8 + k],
                                          fadd2(f2pack(__uint_as_float(dr[2 * k]), __uint_as_float(dr[2 * k + 1])), nd[k])));
            tmem_st8(lane_base + C::kDP + CW * hb + q16 * 8, dk);
          }
          tmem_wait_st();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&sh.ds_ready);
        }
      }
      if (!ok) break;
      // epilogue of the item (TMEM lane = key): the first half of the warpgroups writes
      // dV, the second half scale * dK, each warpgroup every (kGroups / 2)-th 32 columns
      ok = __all_sync(0xffffffffu, mbar_wait(&sh.k_done, (gs - 1) & 1));
      if (!ok) break;
      tc_fence_after();
      constexpr int kHalf = C::kGroups / 2;
      const bool is_dv = hb < kHalf;
      const bool head_live = in_range(bhkv, static_cast<long long>(p.B) * p.Hkv);
      const float mul = is_dv ? 1.f : p.scale;
      // d = 128: rows of 256 bytes, stored whole after a 4-lane chunk exchange (lane 4g + i
      // writes 16 bytes of keys row0 + t, t = 0..3), so each store instruction covers 64
      // contiguous bytes of 8 keys instead of 16 bytes of 32 (measured: +5-10% backward at
      // N = 1024-4096, +0.7% at N = 32768).  d = 64: each thread stores its own row (the
      // exchange measured slower there).
      const int row0 = j * 128 + (warp & 3) * 32 + (lane & ~3);
      __nv_bfloat16* dst = (is_dv ? p.dv : p.dk) + static_cast<size_t>(bhkv) * p.N * D + (lane & 3) * 8;
      const uint32_t col = is_dv ? C::kDV : C::kDK;
#pragma unroll 1
      for (int q4 = hb % kHalf; q4 < D / 32; q4 += kHalf) {
        uint32_t x[32];
        tmem_ld32(lane_base + col + q4 * 32, x);
        tmem_wait_ld();
        reg_fence(x);
        if constexpr (D == 128) {
          uint32_t ch[4][4];
#pragma unroll
          for (int k = 0; k < 4; ++k)
#pragma unroll
            for (int e = 0; e < 4; ++e)
              ch[k][e] = pack_bf16x2(__uint_as_float(x[8 * k + 2 * e]) * mul, __uint_as_float(x[8 * k + 2 * e + 1]) * mul);
          transpose_row_chunks<4>(ch, lane);
          if (head_live) {
#pragma unroll
            for (int t = 0; t < 4; ++t)
              if (row0 + t < p.N)
                *reinterpret_cast<uint4*>(dst + static_cast<size_t>(row0 + t) * D + q4 * 32) =
                    make_uint4(ch[t][0], ch[t][1], ch[t][2], ch[t][3]);
          }
        } else if (head_live && key < p.N) {
          uint4* own = reinterpret_cast<uint4*>((is_dv ? p.dv : p.dk) + (static_cast<size_t>(bhkv) * p.N + key) * D + q4 * 32);
#pragma unroll
          for (int k = 0; k < 4; ++k)
            own[k] = make_uint4(
                pack_bf16x2(__uint_as_float(x[8 * k]) * mul, __uint_as_float(x[8 * k + 1]) * mul),
                pack_bf16x2(__uint_as_float(x[8 * k + 2]) * mul, __uint_as_float(x[8 * k + 3]) * mul),
                pack_bf16x2(__uint_as_float(x[8 * k + 4]) * mul, __uint_as_float(x[8 * k + 5]) * mul),
                pack_bf16x2(__uint_as_float(x[8 * k + 6]) * mul, __uint_as_float(x[8 * k + 7]) * mul));
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sh.acc_free);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, C::kTmemCols);
  }
}

// ================================================================== bwd_q
template <int D>
struct QCfg {
  static constexpr int kTile = 128 * D * 2;
  static constexpr int kBox = 128 * 128;
  static constexpr int kGroups = 2;                      // dS warpgroups: kCols keys of every step each
  static constexpr int kCols = 128 / kGroups;
  static constexpr int kDsWarps = 4 * kGroups;
  static constexpr int kWarpLoad = kDsWarps, kWarpMma = kDsWarps + 1, kWarpV = kDsWarps + 2;
  static constexpr int kThreads = 32 * (kDsWarps + 3);   // dS warps, K/Q/dO TMA, MMA, V TMA
  static constexpr int KST = 3;                          // K ring stages (a K tile is held until dQ(j) is done)
  static constexpr int VST = 2;                          // V ring stages
  // TMEM columns: two S buffers (lane = query, column = key) with dS as bf16 over
  // them (warpgroup g packs its kCols keys into the first kCols / 2 of the columns
  // it read), dP, and the dQ accumulator.
  static constexpr int kS0 = 0, kS1 = 128, kDP = 256, kDQ = 384;
  static constexpr int kTmemCols = 512;
  static constexpr int kOffQ = 0, kOffDO = kTile;
  static constexpr int kOffK = 2 * kTile;                // KST stages
  static constexpr int kOffV = kOffK + KST * kTile;      // VST stages
  static constexpr int kOffBar = kOffV + VST * kTile;
  static constexpr int kLayout = kOffBar + 256;
  static constexpr int kSmem = kLayout + 1024;
  static_assert(KST <= 4 && VST <= 4, "ring barriers hold 4 stages");
  static_assert(kSmem <= 232448, "shared memory layout exceeds 227 KB");
};

struct QShared {
  uint64_t qdo_full, qdo_empty;
  uint64_t k_full[4], k_empty[4], v_full[4], v_empty[4];
  uint64_t s_full[2];           // S(j) in buffer j % 2
  uint64_t dp_full;             // dP(j)
  uint64_t dp_free;             // dP(j) read by both warpgroups
  uint64_t ds_ready;            // dS(j) (bf16) written over S buffer j % 2
  uint64_t q_done[2];           // dQ MMA of step j complete (S buffer j % 2 free)
  uint64_t acc_free;            // dQ of the previous item read out
  uint64_t drain;
  uint32_t tmem_base;
};
static_assert(sizeof(QShared) <= 256, "QShared does not fit its slot");

// Work units of the dQ kernel, numbered KV head by KV head (the G query heads of a
// group interleaved), so CTAs running at the same time share K/V in L2.
//  - In general unit t is one query tile (longest rows first within a group when
//    key ranges grow with the tile).
//  - Causal: unit t is the pair of query tiles (nt-1-pr, pr), two items (one for
//    the middle tile when nt is odd), which together see nt+1 key tiles whatever pr
//    is, so units cost the same and a static round-robin over them stays balanced.
__device__ __forceinline__ int q_halves(const BwdParams& p, int t) {
  if (!p.pair) return 1;
  const int pr = (t / p.G) % p.npair;
  return 2 * pr + 1 == p.nt ? 1 : 2;
}
__device__ __forceinline__ void q_item(const BwdParams& p, int t, int hf, int& bhq, int& i) {
  const int units = p.G * (p.pair ? p.npair : p.nt);   // per (b, kv-head)
  const int gk = t / units;                             // b * Hkv + kv-head
  const int r = t - gk * units;
  const int rq = r / p.G;
  const int hin = r - rq * p.G;
  if (p.pair)
    i = hf ? rq : p.nt - 1 - rq;
  else
    i = p.desc ? (p.nt - 1 - rq) : rq;
  bhq = (gk / p.Hkv) * p.Hq + (gk % p.Hkv) * p.G + hin;
}
// Key tiles [j0, j0 + n) that query tile i sees: keys i - wl .. i + wr.
__device__ __forceinline__ void q_kv_range(const BwdParams& p, int i, int& j0, int& n) {
  const int r0 = i * 128, r1 = min(p.N - 1, r0 + 127);
  j0 = max(0, r0 - p.wl) >> 7;
  n = (min(p.N - 1, r1 + p.wr) >> 7) - j0 + 1;
}

template <int D>
__global__ void __launch_bounds__(QCfg<D>::kThreads, 1)
    attn_bwd_q_kernel(const __grid_constant__ CUtensorMap tmq, const __grid_constant__ CUtensorMap tmk,
                      const __grid_constant__ CUtensorMap tmv, const __grid_constant__ CUtensorMap tmdo,
                      const BwdParams p) {
  using C = QCfg<D>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  QShared& sh = *reinterpret_cast<QShared*>(smem + C::kOffBar);
  uint8_t* sQ = smem + C::kOffQ;
  uint8_t* sDO = smem + C::kOffDO;
  uint8_t* sK = smem + C::kOffK;
  uint8_t* sV = smem + C::kOffV;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    mbar_init(&sh.qdo_full, 1);
    mbar_init(&sh.qdo_empty, 1);
    for (int i = 0; i < 4; ++i) {
      mbar_init(&sh.k_full[i], 1);
      mbar_init(&sh.k_empty[i], 1);
      mbar_init(&sh.v_full[i], 1);
      mbar_init(&sh.v_empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&sh.s_full[i], 1);
      mbar_init(&sh.q_done[i], 1);
    }
    mbar_init(&sh.dp_full, 1);
    mbar_init(&sh.dp_free, C::kDsWarps);
    mbar_init(&sh.ds_ready, C::kDsWarps);
    mbar_init(&sh.acc_free, C::kDsWarps);
    mbar_init(&sh.drain, 1);
    fence_barrier_init();
  }
  if (warp == 0) { tmem_alloc(&sh.tmem_base, C::kTmemCols); tmem_relinquish(); }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sh.tmem_base;

  if (warp == C::kWarpLoad) {
    // ------------------------------------------------------------ TMA producer: Q, dO and K
    if (lane == 0) {
      tma_prefetch_desc(&tmq); tma_prefetch_desc(&tmk); tma_prefetch_desc(&tmdo);
      int gj = 0, it = 0, nk = 0, nqd = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < p.total_items && ok; t += gridDim.x)
      for (int hf = 0; hf < q_halves(p, t) && ok; ++hf, ++it) {
        int bhq, i;
        q_item(p, t, hf, bhq, i);
        const int bkv = (bhq / p.Hq) * p.Hkv + (bhq % p.Hq) / p.G;
        int j0, n_kv;
        q_kv_range(p, i, j0, n_kv);
        if (it >= 1) ok = mbar_wait(&sh.qdo_empty, (it - 1) & 1);
        if (!ok) break;
        mbar_arrive_expect_tx(&sh.qdo_full, 2 * C::kTile);
        in_range(i, p.nt);
        in_range(bhq, static_cast<long long>(p.B) * p.Hq);
        for (int c = 0; c < D / 64; ++c) {
          tma_load_3d(sQ + c * C::kBox, &tmq, &sh.qdo_full, c * 64, i * 128, bhq);
          tma_load_3d(sDO + c * C::kBox, &tmdo, &sh.qdo_full, c * 64, i * 128, bhq);
        }
        nqd = it + 1;
        for (int j = 0; j < n_kv && ok; ++j) {
          const int g = gj + j, st = g % C::KST;
          if (g >= C::KST) ok = mbar_wait(&sh.k_empty[st], ((g / C::KST) - 1) & 1);
          if (!ok) break;
          mbar_arrive_expect_tx(&sh.k_full[st], C::kTile);
          in_range(j0 + j, p.nt);
          in_range(bkv, static_cast<long long>(p.B) * p.Hkv);
          for (int c = 0; c < D / 64; ++c)
            tma_load_3d(sK + st * C::kTile + c * C::kBox, &tmk, &sh.k_full[st], c * 64, (j0 + j) * 128, bkv);
          nk = g + 1;
        }
        gj += n_kv;
      }
      if (!ok) {
        if (nqd >= 1) mbar_drain_wait(&sh.qdo_full, (nqd - 1) & 1);
        for (int g = max(0, nk - C::KST); g < nk; ++g) mbar_drain_wait(&sh.k_full[g % C::KST], (g / C::KST) & 1);
      }
    }
  } else if (warp == C::kWarpV) {
    // ------------------------------------------------------------ TMA producer: V
    if (lane == 0) {
      tma_prefetch_desc(&tmv);
      int gj = 0, nv = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < p.total_items && ok; t += gridDim.x)
      for (int hf = 0; hf < q_halves(p, t) && ok; ++hf) {
        int bhq, i;
        q_item(p, t, hf, bhq, i);
        const int bkv = (bhq / p.Hq) * p.Hkv + (bhq % p.Hq) / p.G;
        int j0, n_kv;
        q_kv_range(p, i, j0, n_kv);
        for (int j = 0; j < n_kv && ok; ++j) {
          const int g = gj + j, st = g % C::VST;
          if (g >= C::VST) ok = mbar_wait(&sh.v_empty[st], ((g / C::VST) - 1) & 1);
          if (!ok) break;
          mbar_arrive_expect_tx(&sh.v_full[st], C::kTile);
          for (int c = 0; c < D / 64; ++c)
            tma_load_3d(sV + st * C::kTile + c * C::kBox, &tmv, &sh.v_full[st], c * 64, (j0 + j) * 128, bkv);
          nv = g + 1;
        }
        gj += n_kv;
      }
      if (!ok)
        for (int g = max(0, nv - C::VST); g < nv; ++g) mbar_drain_wait(&sh.v_full[g % C::VST], (g / C::VST) & 1);
    }
  } else if (warp == C::kWarpMma) {
    // ------------------------------------------------------------ MMA issuer
    // Order per step j:  S(j+1)  [dS(j)] dQ(j)  dP(j+1).  The warpgroups' exps of step
    // j+1 run under dQ(j) and dP(j+1); dS of step j needs dP(j).  The whole warp
    // follows the schedule; one lane, elected once, issues every MMA and commit.
    const bool leader = elect_one();
    constexpr uint32_t idS = idesc_bf16_f32(128, 128, false, false);   // S, dP
    constexpr uint32_t idQ = idesc_bf16_f32(128, D, false, true);      // dQ += dS K
    constexpr uint32_t hi = sdesc_hi_sw128(1024);
    const uint32_t q_lo = sdesc_lo(smem_u32(sQ), 16), do_lo = sdesc_lo(smem_u32(sDO), 16);
    const uint32_t k_lo0 = sdesc_lo(smem_u32(sK), 16), v_lo0 = sdesc_lo(smem_u32(sV), 16);
    const uint32_t k_mn0 = sdesc_lo(smem_u32(sK), C::kBox);
    auto wait = [&](uint64_t* bar, uint32_t parity) -> bool {
      return __all_sync(0xffffffffu, mbar_wait(bar, parity));
    };
    int gj = 0, it = 0;
    bool ok = true;
    auto issue_s = [&](int g) -> bool {     // S(g) = Q K(g)^T into buffer g % 2
      const int st = g % C::KST, sb = g & 1;
      if (!wait(&sh.k_full[st], (g / C::KST) & 1)) return false;
      // S(g) overwrites dS(g-2): issued behind dQ(g-2), performed after it.
      tc_fence_after();
      if (leader) {
        const uint32_t k_lo = k_lo0 + st * (C::kTile >> 4);
#pragma unroll
        for (int k = 0; k < D / 16; ++k) {
          const uint32_t off = ((k >> 2) * C::kBox + (k & 3) * 32) >> 4;
          umma_ss_lo(tmem + (sb ? C::kS1 : C::kS0), q_lo + off, k_lo + off, hi, idS, k > 0);
        }
        umma_commit(&sh.s_full[sb]);
      }
      __syncwarp();
      return true;
    };
    auto issue_dp = [&](int g) -> bool {    // dP(g) = dO V(g)^T
      const int st = g % C::VST;
      if (!wait(&sh.v_full[st], (g / C::VST) & 1)) return false;
      if (g >= 1 && !wait(&sh.dp_free, (g - 1) & 1)) return false;       // dP(g-1) read
      tc_fence_after();
      if (leader) {
        const uint32_t v_lo = v_lo0 + st * (C::kTile >> 4);
#pragma unroll
        for (int k = 0; k < D / 16; ++k) {
          const uint32_t off = ((k >> 2) * C::kBox + (k & 3) * 32) >> 4;
          umma_ss_lo(tmem + C::kDP, do_lo + off, v_lo + off, hi, idS, k > 0);
        }
        umma_commit(&sh.dp_full);
        umma_commit(&sh.v_empty[st]);
      }
      __syncwarp();
      return true;
    };
    for (int t = blockIdx.x; t < p.total_items && ok; t += gridDim.x)
    for (int hf = 0; hf < q_halves(p, t) && ok; ++hf, ++it) {
      int bhq, i;
      q_item(p, t, hf, bhq, i);
      int j0, n_kv;
      q_kv_range(p, i, j0, n_kv);
      ok = wait(&sh.qdo_full, it & 1);
      if (!ok) break;
      ok = issue_s(gj) && issue_dp(gj);
      for (int u = 0; u < n_kv && ok; ++u) {
        const int g = gj + u, st = g % C::KST, sb = g & 1;
        if (u + 1 < n_kv && !issue_s(g + 1)) { ok = false; break; }
        // dQ += dS K  (A = dS in TMEM, M = queries, K = keys; B = K MN-major)
        ok = wait(&sh.ds_ready, g & 1);
        if (ok && u == 0 && it >= 1) ok = wait(&sh.acc_free, (it - 1) & 1);
        if (!ok) break;
        tc_fence_after();
        if (leader) {
          const uint32_t k_mn = k_mn0 + st * (C::kTile >> 4);
          const uint32_t sbase = tmem + (sb ? C::kS1 : C::kS0);
#pragma unroll
          for (int k = 0; k < 8; ++k)
            umma_ts_lo(tmem + C::kDQ, sbase + packed_col(k, C::kCols), k_mn + ((k * 2048) >> 4), hi, idQ,
                       !(u == 0 && k == 0));
          umma_commit(&sh.q_done[sb]);
          umma_commit(&sh.k_empty[st]);
          if (u + 1 == n_kv) umma_commit(&sh.qdo_empty);     // the item's last reads of Q and dO are issued
        }
        __syncwarp();
        if (u + 1 < n_kv && !issue_dp(g + 1)) { ok = false; break; }
      }
      if (!ok) break;
      gj += n_kv;
    }
    if (leader) {
      umma_commit(&sh.drain);
      mbar_wait(&sh.drain, 0);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ dS warpgroups (rows = queries)
    // warpgroup hb (warps 4hb .. 4hb+3): keys kCols*hb .. kCols*hb + kCols-1 of every
    // step.  The row's LSE and D are this thread's own, held in registers for the item.
    constexpr int CW = C::kCols;
    const int hb = warp >> 2;
    const int r = (warp & 3) * 32 + lane;
    const uint32_t lane_base = tmem + (static_cast<uint32_t>((warp & 3) * 32) << 16);
    const uint64_t c2 = f2pack(p.c, p.c);
    int gj = 0;
    bool ok = true;
    for (int t = blockIdx.x; t < p.total_items && ok; t += gridDim.x)
    for (int hf = 0; hf < q_halves(p, t) && ok; ++hf) {
      int bhq, i;
      q_item(p, t, hf, bhq, i);
      int j0, n_kv;
      q_kv_range(p, i, j0, n_kv);
      const int qrow = i * 128 + r;
      size_t vrow = static_cast<size_t>(bhq) * (p.nt * 128) + qrow;
      if (!in_range(static_cast<long long>(vrow), static_cast<long long>(p.B) * p.Hq * p.nt * 128)) vrow = 0;
      const float nl2 = p.nlse2[vrow], nd = p.ndd[vrow];
      uint64_t nl[8];
#pragma unroll
      for (int k = 0; k < 8; ++k) nl[k] = f2pack(nl2, nl2);
      const uint64_t nd2 = f2pack(nd, nd);
      for (int u = 0; u < n_kv && ok; ++u) {
        const int g = gj + u, sb = g & 1;
        const uint32_t sbase = lane_base + (sb ? C::kS1 : C::kS0) + CW * hb;
        // visible key columns (relative to this warpgroup's CW) for this query row:
        // keys qrow - wl .. qrow + wr
        const int kbase = (j0 + u) * 128 + CW * hb;
        const int hi = min(p.N - 1, qrow + p.wr) - kbase;
        const int lo = qrow - p.wl - kbase;
        const bool masked = !__all_sync(0xffffffffu, lo <= 0 && hi >= CW - 1);
        ok = __all_sync(0xffffffffu, mbar_wait(&sh.s_full[sb], (g >> 1) & 1));
        if (!ok) break;
        tc_fence_after();
        // phase A: P = exp2(S c - lse2) for this warpgroup's CW keys
        uint64_t pf2[CW / 2];
#pragma unroll
        for (int q16 = 0; q16 < CW / 16; ++q16) {
          uint32_t sr[16];
          tmem_ld16(sbase + q16 * 16, sr);
          tmem_wait_ld();
          reg_fence(sr);
          bwd_exp16<D>(sr, nl, c2, masked, q16 * 16, lo, hi, pf2 + q16 * 8);
        }
        // phase B: dS = P (dP - D) -> bf16 over the S buffer
        ok = __all_sync(0xffffffffu, mbar_wait(&sh.dp_full, g & 1));
        if (!ok) break;
        tc_fence_after();
#pragma unroll
        for (int q16 = 0; q16 < CW / 16; ++q16) {
          uint32_t dr[16];
          tmem_ld16(lane_base + C::kDP + CW * hb + q16 * 16, dr);
          tmem_wait_ld();
          reg_fence(dr);
          uint32_t dk[8];
#pragma unroll
          for (int k = 0; k < 8; ++k)
            dk[k] = pack_bf16x2_2(fmul2(pf2[q16 * 8 + k],
                                        fadd2(f2pack(__uint_as_float(dr[2 * k]), __uint_as_float(dr[2 * k + 1])), nd2)));
          tmem_st8(sbase + q16 * 8, dk);
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&sh.dp_free);
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&sh.ds_ready);
      }
      if (!ok) break;
      // epilogue: dQ (TMEM lane = query row), scaled, bf16; the warpgroups split the columns
      const int glast = gj + n_kv - 1;
      ok = __all_sync(0xffffffffu, mbar_wait(&sh.q_done[glast & 1], (glast >> 1) & 1));
      if (!ok) break;
      tc_fence_after();
      const bool head_live = in_range(bhq, static_cast<long long>(p.B) * p.Hq);
      // rows stored as for dK and dV (exchanged among 4 lanes at d = 128)
      const int row0 = i * 128 + (warp & 3) * 32 + (lane & ~3);
      __nv_bfloat16* dst = p.dq + static_cast<size_t>(bhq) * p.N * D + (lane & 3) * 8;
#pragma unroll 1
      for (int q4 = hb; q4 < D / 32; q4 += C::kGroups) {
        uint32_t x[32];
        tmem_ld32(lane_base + C::kDQ + q4 * 32, x);
        tmem_wait_ld();
        reg_fence(x);
        if constexpr (D == 128) {
          uint32_t ch[4][4];
#pragma unroll
          for (int k = 0; k < 4; ++k)
#pragma unroll
            for (int e = 0; e < 4; ++e)
              ch[k][e] = pack_bf16x2(__uint_as_float(x[8 * k + 2 * e]) * p.scale,
                                     __uint_as_float(x[8 * k + 2 * e + 1]) * p.scale);
          transpose_row_chunks<4>(ch, lane);
          if (head_live) {
#pragma unroll
            for (int t = 0; t < 4; ++t)
              if (row0 + t < p.N)
                *reinterpret_cast<uint4*>(dst + static_cast<size_t>(row0 + t) * D + q4 * 32) =
                    make_uint4(ch[t][0], ch[t][1], ch[t][2], ch[t][3]);
          }
        } else if (head_live && qrow < p.N) {
          uint4* own = reinterpret_cast<uint4*>(p.dq + (static_cast<size_t>(bhq) * p.N + qrow) * D + q4 * 32);
#pragma unroll
          for (int k = 0; k < 4; ++k)
            own[k] = make_uint4(
                pack_bf16x2(__uint_as_float(x[8 * k]) * p.scale, __uint_as_float(x[8 * k + 1]) * p.scale),
                pack_bf16x2(__uint_as_float(x[8 * k + 2]) * p.scale, __uint_as_float(x[8 * k + 3]) * p.scale),
                pack_bf16x2(__uint_as_float(x[8 * k + 4]) * p.scale, __uint_as_float(x[8 * k + 5]) * p.scale),
                pack_bf16x2(__uint_as_float(x[8 * k + 6]) * p.scale, __uint_as_float(x[8 * k + 7]) * p.scale));
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sh.acc_free);
      gj += n_kv;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, C::kTmemCols);
  }
}

int launch_bwd(const void* q, const void* k, const void* v, const void* o, const float* lse, const void* dO,
               void* dq, void* dk, void* dv, int B, int Hq, int Hkv, int N, int d, float scale, int wl, int wr,
               void* workspace, cudaStream_t stream, int sms);

}  // namespace attn
