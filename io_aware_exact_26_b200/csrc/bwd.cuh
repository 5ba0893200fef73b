// Backward exact attention for sm_100a: dQ, dK, dV of sum(O * dO).
//
// Recompute instead of store (page "attention 的显存线性化" §五; page
// "attn-efficient", recompute paragraph): the forward keeps only O and the
// log-sum-exp; here every S/P tile is rebuilt on chip from Q, K and the saved
// LSE.  Gradient formulas (chain rule through the row softmax; the pages state
// none): with D_i = sum_k dO_ik O_ik,
//   P = exp(scale Q K^T - LSE),  dV = P^T dO,  dP = dO V^T,
//   dS = P * (dP - D),  dQ = scale dS K,  dK = scale dS^T Q.
//
// Kernels
//   bwd_prep   : one warp per query row: D_i and LSE in log2 units; zeroes the
//                dQ ordering tickets.
//   bwd_main   : persistent, one work item = (b, kv-head, 128-key tile j); K_j, V_j
//                stay in shared memory while the item walks its G q-heads and
//                the query tiles that see tile j (i >= j when causal).
//   bwd_dq     : sums the dQ chains in a fixed order, scales, rounds to bf16.
// Roles in bwd_main (320 threads):
//   warps 0-3  "dS" warpgroup, thread = key row = TMEM lane: reads S^T and dP^T
//              from TMEM, forms P^T (bf16, back into TMEM over S^T) and dS^T
//              (bf16, 128B-swizzled shared memory).
//   warps 4-7  dQ warpgroup, thread = head-dim column of dQ^T: moves the dQ^T tile
//              out of TMEM and adds it into the fp32 accumulator in a fixed order
//              (tickets), one coalesced line per query row and warp; the last
//              contributor writes bf16 dq.  At the end of an item it writes dK
//              (scaled) and dV from TMEM (thread = key row there).
//   warp 8     TMA producer: K_j, V_j per item; Q_i, dO_i per step (2 stages).
//   warp 9     MMA issuer: S^T = K Q^T, dP^T = V dO^T, dV += P^T dO,
//              dK += dS^T Q, dQ^T = K^T dS^T.
// The dS^T tile in shared memory is the K-major A operand of dK and, read as
// MN-major, the B operand of dQ^T; the K tile is the A operand of S^T (K-major)
// and, read MN-major, of dQ^T.
//
// Determinism: dK and dV of an item are accumulated in TMEM by one CTA in a
// fixed loop order.  dQ of query tile i collects one partial per key tile; the
// partials are added in a fixed order of key tiles (position below) enforced by
// per-(tile, warp) tickets, so the fp32 sums are bitwise reproducible.
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

__device__ __forceinline__ void red_add_f32(float* p, float v) {
  asm volatile("red.global.add.f32 [%0], %1;" ::"l"(p), "f"(v) : "memory");
}

__device__ __forceinline__ int ld_acquire(const int* p) {
  int v;
  asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ void st_release(int* p, int v) {
  asm volatile("st.release.gpu.global.b32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

struct BwdLayout {
  // workspace carve-up (byte offsets, each 256-byte aligned)
  size_t lse2_off, dd_off, acc_off, ticket_off, total;
};

// Number of independent fixed-order dQ accumulation chains per query tile.  The
// key tiles contributing to a query tile are dealt round-robin (by their position
// in the order) to kChains fp32 accumulators; within a chain the adds happen in a
// fixed order, and the chains are summed in a fixed order at the end.  Consecutive
// contributors of one chain are kChains steps apart, which hides the hand-off.
constexpr int kChains = 4;

__host__ __device__ inline BwdLayout bwd_layout(long long BHq, int N, int d) {
  const long long npad = (N + 127) / 128 * 128;
  const long long nq = npad / 128;
  auto up = [](size_t x) { return (x + 255) / 256 * 256; };
  BwdLayout L;
  L.lse2_off = 0;
  L.dd_off = up(L.lse2_off + BHq * npad * 4);
  L.acc_off = up(L.dd_off + BHq * npad * 4);
  L.ticket_off = up(L.acc_off + static_cast<size_t>(kChains) * BHq * npad * d * 4);
  L.total = up(L.ticket_off + BHq * nq * kChains * 4 * 4);
  return L;
}

inline size_t bwd_workspace_bytes(int B, int Hq, int Hkv, int N, int d) {
  (void)Hkv;
  return bwd_layout(static_cast<long long>(B) * Hq, N, d).total;
}

// ------------------------------------------------------------------ preprocess
// D_i = sum_k dO_ik O_ik (fp32) and lse2_i = LSE_i * log2(e); padded rows get 0.
// Each row is read with 16-byte loads by D/8 lanes, so one warp covers 256/D rows.
template <int D>
__global__ void __launch_bounds__(256) attn_bwd_prep_kernel(const __nv_bfloat16* __restrict__ o,
                                                            const __nv_bfloat16* __restrict__ dO,
                                                            const float* __restrict__ lse, float* lse2,
                                                            float* dd, int* tickets, long long BHq, int N,
                                                            long long n_tickets) {
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
      dd[r] = acc;
      lse2[r] = l2;
    }
  }
  const long long tid = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  for (long long t = tid; t < n_tickets; t += static_cast<long long>(gridDim.x) * blockDim.x) tickets[t] = 0;
}

// ------------------------------------------------------------------ main kernel
struct BwdParams {
  __nv_bfloat16* dq;
  __nv_bfloat16* dk;
  __nv_bfloat16* dv;
  const float* lse2;
  const float* dd;
  float* acc;
  int* tickets;
  int B, Hq, Hkv, N, G;
  long long BHq;
  int nt;           // number of 128-row tiles along N
  int total_items;
  int order;        // 0 = causal, 1 = linear (non-causal), 2 = cyclic (non-causal)
  float c;          // scale * log2(e)
  float scale;
};

template <int D>
struct BwdCfg {
  static constexpr int kTile = 128 * D * 2;
  static constexpr int kBox = 128 * 128;
  static constexpr int kThreads = 320;
  // TMEM columns
  static constexpr int kS = 0, kDP = 128;
  // dQ^T (128 lanes = head dim, 128 columns = queries) aliases dP^T when D == 128
  static constexpr int kDQ = (D == 128) ? 128 : 256;
  static constexpr int kDV = (D == 128) ? 256 : 384;
  static constexpr int kDK = (D == 128) ? 384 : 448;
  static constexpr int kTmemCols = 512;
  // shared memory (offsets from the 1024-aligned base)
  static constexpr int kOffK = 0;
  static constexpr int kOffV = kTile;
  static constexpr int kOffQ = 2 * kTile;                // 2 stages of Q
  static constexpr int kOffDO = 4 * kTile;               // 2 stages of dO
  static constexpr int kOffDS = 6 * kTile;               // dS^T, 128 x 128 bf16
  static constexpr int kOffVec = kOffDS + 32768;         // per stage: lse2[128], dd[128]
  static constexpr int kOffBar = kOffVec + 2048;         // BwdShared
  static constexpr int kLayout = kOffBar + 256;
  // request what the layout needs plus alignment slack, capped at the opt-in maximum
  static constexpr int kSmem = (kLayout + 1024 <= 232448) ? kLayout + 1024 : 232448;
};

struct BwdShared {
  uint64_t kv_full, kv_empty;
  uint64_t qdo_full[2], qdo_empty[2];
  uint64_t st_full, ds_ready, step_done, dq_full, dq_free, acc_free;
  uint64_t drain;
  uint32_t tmem_base;
};

// item t -> (bh_kv, key tile j)
__device__ __forceinline__ void bwd_item(const BwdParams& p, int t, int& bhkv, int& j) {
  bhkv = t / p.nt;
  const int r = t - bhkv * p.nt;
  j = (p.order == 2) ? r : (p.nt - 1 - r);
}

__device__ __forceinline__ int bwd_steps_per_head(const BwdParams& p, int j) {
  return p.order == 0 ? (p.nt - j) : p.nt;
}

// step s of a head -> query tile i and this key tile's place in the dQ order of tile
// i: global position `gpos` among the tile's contributors, its chain (gpos mod
// kChains) and its position inside that chain (gpos / kChains).
__device__ __forceinline__ void bwd_step(const BwdParams& p, int j, int s, int& i, int& chain, int& pos) {
  int gpos;
  if (p.order == 0) {
    i = j + s; gpos = i - j;
  } else if (p.order == 1) {
    i = s; gpos = p.nt - 1 - j;
  } else {
    i = (j + s) % p.nt; gpos = (i - j + p.nt) % p.nt;
  }
  chain = gpos % kChains;
  pos = gpos / kChains;
}

template <int D>
__global__ void __launch_bounds__(320, 1)
    attn_bwd_main_kernel(const __grid_constant__ CUtensorMap tmq, const __grid_constant__ CUtensorMap tmk,
                         const __grid_constant__ CUtensorMap tmv, const __grid_constant__ CUtensorMap tmdo,
                         const BwdParams p) {
  using C = BwdCfg<D>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  if (static_cast<int>(smem - smem_raw) + C::kLayout > C::kSmem) {
    // the 128B-swizzled tiles need a 1024-byte aligned base that this launch cannot give
    if (threadIdx.x == 0) record_error(&g_attn_status, 3);
    return;
  }
  BwdShared& sh = *reinterpret_cast<BwdShared*>(smem + C::kOffBar);
  uint8_t* sK = smem + C::kOffK;
  uint8_t* sV = smem + C::kOffV;
  uint8_t* sQ = smem + C::kOffQ;
  uint8_t* sDO = smem + C::kOffDO;
  uint8_t* sDS = smem + C::kOffDS;
  float* sVec = reinterpret_cast<float*>(smem + C::kOffVec);   // [stage][lse2 128 | dd 128]

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    mbar_init(&sh.kv_full, 1);
    mbar_init(&sh.kv_empty, 1);
    for (int i = 0; i < 2; ++i) { mbar_init(&sh.qdo_full[i], 1); mbar_init(&sh.qdo_empty[i], 1); }
    mbar_init(&sh.st_full, 1);
    mbar_init(&sh.ds_ready, 4);
    mbar_init(&sh.step_done, 1);
    mbar_init(&sh.dq_full, 1);
    mbar_init(&sh.dq_free, 4);
    mbar_init(&sh.acc_free, 4);
    mbar_init(&sh.drain, 1);
    fence_barrier_init();
  }
  if (warp == 0) { tmem_alloc(&sh.tmem_base, C::kTmemCols); tmem_relinquish(); }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sh.tmem_base;

  if (warp == 8) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      tma_prefetch_desc(&tmq); tma_prefetch_desc(&tmk); tma_prefetch_desc(&tmv); tma_prefetch_desc(&tmdo);
      int gs = 0, it = 0, nq = 0, nkv = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < p.total_items && ok; t += gridDim.x, ++it) {
        int bhkv, j;
        bwd_item(p, t, bhkv, j);
        if (it >= 1) ok = mbar_wait(&sh.kv_empty, (it - 1) & 1);
        if (!ok) break;
        mbar_arrive_expect_tx(&sh.kv_full, 2 * C::kTile);
        for (int c = 0; c < D / 64; ++c) {
          tma_load_3d(sK + c * C::kBox, &tmk, &sh.kv_full, c * 64, j * 128, bhkv);
          tma_load_3d(sV + c * C::kBox, &tmv, &sh.kv_full, c * 64, j * 128, bhkv);
        }
        nkv = it + 1;
        const int b = bhkv / p.Hkv, hk = bhkv - b * p.Hkv;
        const int steps = bwd_steps_per_head(p, j);
        for (int h = 0; h < p.G && ok; ++h) {
          const int bhq = b * p.Hq + hk * p.G + h;
          for (int s = 0; s < steps; ++s, ++gs) {
            int i, chain, pos;
            bwd_step(p, j, s, i, chain, pos);
            const int st = gs & 1;
            if (gs >= 2) ok = mbar_wait(&sh.qdo_empty[st], ((gs >> 1) - 1) & 1);
            if (!ok) break;
            mbar_arrive_expect_tx(&sh.qdo_full[st], 2 * C::kTile + 1024);
            for (int c = 0; c < D / 64; ++c) {
              tma_load_3d(sQ + st * C::kTile + c * C::kBox, &tmq, &sh.qdo_full[st], c * 64, i * 128, bhq);
              tma_load_3d(sDO + st * C::kTile + c * C::kBox, &tmdo, &sh.qdo_full[st], c * 64, i * 128, bhq);
            }
            const size_t vrow = static_cast<size_t>(bhq) * (p.nt * 128) + i * 128;
            bulk_load(sVec + st * 256, p.lse2 + vrow, 512, &sh.qdo_full[st]);
            bulk_load(sVec + st * 256 + 128, p.dd + vrow, 512, &sh.qdo_full[st]);
            nq = gs + 1;
          }
        }
      }
      if (!ok) {
        if (nkv >= 1) mbar_drain_wait(&sh.kv_full, (nkv - 1) & 1);
        for (int g = max(0, nq - 2); g < nq; ++g) mbar_drain_wait(&sh.qdo_full[g & 1], (g >> 1) & 1);
      }
    }
  } else if (warp == 9) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idST = idesc_bf16_f32(128, 128, false, false);
      constexpr uint32_t idKV = idesc_bf16_f32(128, D, false, true);   // dV, dK
      constexpr uint32_t idQ = idesc_bf16_f32(128, 128, true, true);   // dQ^T
      int gs = 0, it = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < p.total_items && ok; t += gridDim.x, ++it) {
        int bhkv, j;
        bwd_item(p, t, bhkv, j);
        ok = mbar_wait(&sh.kv_full, it & 1);
        if (!ok) break;
        const uint32_t k_addr = smem_u32(sK), v_addr = smem_u32(sV), ds_addr = smem_u32(sDS);
        const int steps = bwd_steps_per_head(p, j);
        bool first = true;
        for (int h = 0; h < p.G && ok; ++h) {
          for (int s = 0; s < steps; ++s, ++gs) {
            const int st = gs & 1;
            ok = mbar_wait(&sh.qdo_full[st], (gs >> 1) & 1);
            if (ok && gs >= 1) ok = mbar_wait(&sh.step_done, (gs - 1) & 1);
            if (ok && D == 128 && gs >= 1) ok = mbar_wait(&sh.dq_free, (gs - 1) & 1);  // dQ aliases dP^T
            if (!ok) break;
            tc_fence_after();
            const uint32_t q_addr = smem_u32(sQ + st * C::kTile), do_addr = smem_u32(sDO + st * C::kTile);
            // S^T = K Q^T and dP^T = V dO^T  (M = keys, N = queries, K = head dim)
#pragma unroll
            for (int k = 0; k < D / 16; ++k) {
              const uint32_t off = (k >> 2) * C::kBox + (k & 3) * 32;
              umma_ss(tmem + C::kS, sdesc_sw128(k_addr + off, 16, 1024), sdesc_sw128(q_addr + off, 16, 1024), idST,
                      k > 0);
            }
#pragma unroll
            for (int k = 0; k < D / 16; ++k) {
              const uint32_t off = (k >> 2) * C::kBox + (k & 3) * 32;
              umma_ss(tmem + C::kDP, sdesc_sw128(v_addr + off, 16, 1024), sdesc_sw128(do_addr + off, 16, 1024),
                      idST, k > 0);
            }
            umma_commit(&sh.st_full);
            ok = mbar_wait(&sh.ds_ready, gs & 1);
            if (ok && first && it >= 1) ok = mbar_wait(&sh.acc_free, (it - 1) & 1);
            if (!ok) break;
            tc_fence_after();
            // dV += P^T dO  (A = P^T from TMEM, B = dO MN-major; K = queries)
#pragma unroll
            for (int k = 0; k < 8; ++k)
              umma_ts(tmem + C::kDV, tmem + C::kS + k * 8, sdesc_sw128(do_addr + k * 2048, C::kBox, 1024), idKV,
                      !(first && k == 0));
            // dK += dS^T Q  (A = dS^T K-major smem, B = Q MN-major)
#pragma unroll
            for (int k = 0; k < 8; ++k) {
              const uint32_t off = (k >> 2) * C::kBox + (k & 3) * 32;
              umma_ss(tmem + C::kDK, sdesc_sw128(ds_addr + off, 16, 1024),
                      sdesc_sw128(q_addr + k * 2048, C::kBox, 1024), idKV, !(first && k == 0));
            }
            // dQ^T = K^T dS^T  (M = head dim, N = queries, K = keys; A = K read MN-major,
            // B = dS^T read MN-major).  For D = 64 the A operand spans 128 rows: rows 64-127
            // read the next smem tile and land in TMEM lanes 64-127, which nobody reads.
            if (D != 128 && gs >= 1) {
              ok = mbar_wait(&sh.dq_free, (gs - 1) & 1);
              if (!ok) break;
              tc_fence_after();
            }
#pragma unroll
            for (int k = 0; k < 8; ++k)
              umma_ss(tmem + C::kDQ, sdesc_sw128(k_addr + k * 2048, C::kBox, 1024),
                      sdesc_sw128(ds_addr + k * 2048, C::kBox, 1024), idQ, k > 0);
            umma_commit(&sh.dq_full);
            umma_commit(&sh.qdo_empty[st]);
            umma_commit(&sh.step_done);
            first = false;
          }
        }
        if (!ok) break;
        umma_commit(&sh.kv_empty);
      }
      umma_commit(&sh.drain);
      mbar_wait(&sh.drain, 0);
    }
  } else if (warp < 4) {
    // ------------------------------------------------------------ dS warpgroup (rows = keys)
    const int r = warp * 32 + lane;
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(warp * 32) << 16);
    const float c = p.c;
    int gs = 0;
    bool ok = true;
    for (int t = blockIdx.x; t < p.total_items && ok; t += gridDim.x) {
      int bhkv, j;
      bwd_item(p, t, bhkv, j);
      const int b = bhkv / p.Hkv, hk = bhkv - b * p.Hkv;
      const int steps = bwd_steps_per_head(p, j);
      const int key = j * 128 + r;
      for (int h = 0; h < p.G && ok; ++h) {
        const int bhq = b * p.Hq + hk * p.G + h;
        for (int s = 0; s < steps; ++s, ++gs) {
          int i, chain, pos;
          bwd_step(p, j, s, i, chain, pos);
          (void)bhq; (void)pos; (void)chain;
          const int st = gs & 1;
          const float* sLse = sVec + st * 256;
          const float* sDd = sLse + 128;
          ok = __all_sync(0xffffffffu, mbar_wait(&sh.qdo_full[st], (gs >> 1) & 1));
          if (ok) ok = __all_sync(0xffffffffu, mbar_wait(&sh.st_full, gs & 1));
          if (ok && gs >= 1) ok = __all_sync(0xffffffffu, mbar_wait(&sh.step_done, (gs - 1) & 1));
          if (!ok) break;
          tc_fence_after();
          // visible queries of this key row: causal needs query >= key; both need < N
          const int qbase = i * 128;
          const int qmax = p.N - 1 - qbase;                           // last valid column
          const int qmin = (p.order == 0) ? (key - qbase) : 0;        // first causal column
          const bool key_live = key < p.N;
          // most tiles are fully visible: skip the per-element mask there (warp-uniform choice)
          const bool full = __all_sync(0xffffffffu, key_live && qmin <= 0 && qmax >= 127);
#pragma unroll 1
          for (int q4 = 0; q4 < 4; ++q4) {
            uint32_t sr[32], dr[32];
            tmem_ld32(lane_base + C::kS + q4 * 32, sr);
            tmem_ld32(lane_base + C::kDP + q4 * 32, dr);
            // this chunk's 32 values of lse2 and D: same address in every thread (broadcast)
            float lv[32], dv[32];
#pragma unroll
            for (int k = 0; k < 8; ++k) {
              const float4 a = reinterpret_cast<const float4*>(sLse + q4 * 32)[k];
              const float4 b = reinterpret_cast<const float4*>(sDd + q4 * 32)[k];
              lv[4 * k] = a.x; lv[4 * k + 1] = a.y; lv[4 * k + 2] = a.z; lv[4 * k + 3] = a.w;
              dv[4 * k] = b.x; dv[4 * k + 1] = b.y; dv[4 * k + 2] = b.z; dv[4 * k + 3] = b.w;
            }
            tmem_wait_ld();
            uint32_t pk[16], dk[16];
            if (full) {
#pragma unroll
              for (int k = 0; k < 16; ++k) {
                const float p0 = ex2_approx(fmaf(__uint_as_float(sr[2 * k]), c, -lv[2 * k]));
                const float p1 = ex2_approx(fmaf(__uint_as_float(sr[2 * k + 1]), c, -lv[2 * k + 1]));
                pk[k] = pack_bf16x2(p0, p1);
                dk[k] = pack_bf16x2(p0 * (__uint_as_float(dr[2 * k]) - dv[2 * k]),
                                    p1 * (__uint_as_float(dr[2 * k + 1]) - dv[2 * k + 1]));
              }
            } else {
#pragma unroll
              for (int k = 0; k < 16; ++k) {
                float pv[2], dv2[2];
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                  const int col = q4 * 32 + 2 * k + e;
                  const bool vis = key_live && col >= qmin && col <= qmax;
                  const float pe = vis ? ex2_approx(fmaf(__uint_as_float(sr[2 * k + e]), c, -lv[2 * k + e])) : 0.f;
                  pv[e] = pe;
                  dv2[e] = pe * (__uint_as_float(dr[2 * k + e]) - dv[2 * k + e]);
                }
                pk[k] = pack_bf16x2(pv[0], pv[1]);
                dk[k] = pack_bf16x2(dv2[0], dv2[1]);
              }
            }
            tmem_st16(lane_base + C::kS + q4 * 16, pk);
            // dS^T row r, queries [32 q4, 32 q4 + 32): 4 chunks of 16 bytes, 128B swizzle
            uint8_t* rowp = sDS + (q4 >> 1) * C::kBox + r * 128;
#pragma unroll
            for (int ch = 0; ch < 4; ++ch) {
              const int chunk = (q4 & 1) * 4 + ch;
              *reinterpret_cast<uint4*>(rowp + ((chunk ^ (r & 7)) << 4)) =
                  make_uint4(dk[4 * ch], dk[4 * ch + 1], dk[4 * ch + 2], dk[4 * ch + 3]);
            }
          }
          fence_proxy_async_smem();
          tmem_wait_st();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&sh.ds_ready);
        }
      }
    }
  } else {
    // ------------------------------------------------------------ dQ / epilogue warpgroup
    // dQ^T lives in TMEM with lane = head-dim index, column = query row, so a warp's
    // accumulator accesses for one query row are 32 consecutive floats (one line).
    const int wq = warp - 4;
    const int r = wq * 32 + lane;               // key row (epilogue) / head-dim index (dQ)
    const bool dd_live = r < D;                 // D = 64: warps 6-7 carry no dQ columns
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(wq * 32) << 16);
    int gs = 0, it = 0;
    bool ok = true;
    for (int t = blockIdx.x; t < p.total_items && ok; t += gridDim.x, ++it) {
      int bhkv, j;
      bwd_item(p, t, bhkv, j);
      const int b = bhkv / p.Hkv, hk = bhkv - b * p.Hkv;
      const int steps = bwd_steps_per_head(p, j);
      for (int h = 0; h < p.G && ok; ++h) {
        const int bhq = b * p.Hq + hk * p.G + h;
        for (int s = 0; s < steps; ++s, ++gs) {
          int i, chain, pos;
          bwd_step(p, j, s, i, chain, pos);
          ok = __all_sync(0xffffffffu, mbar_wait(&sh.dq_full, gs & 1));
          if (!ok) break;
          tc_fence_after();
          float part[128];
#pragma unroll
          for (int q4 = 0; q4 < 4; ++q4) {
            uint32_t x[32];
            tmem_ld32(lane_base + C::kDQ + q4 * 32, x);
            tmem_wait_ld();
#pragma unroll
            for (int k = 0; k < 32; ++k) part[q4 * 32 + k] = __uint_as_float(x[k]);
          }
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&sh.dq_free);
          if (!dd_live) continue;
          // wait for this warp's turn in its chain on query tile i
          int* ticket = p.tickets + ((static_cast<size_t>(bhq) * p.nt + i) * kChains + chain) * 4 + wq;
          bool turn = true;
          if (pos > 0) {
            if (lane == 0) {
              turn = false;
              const uint64_t t0 = globaltimer_ns();
              for (uint32_t spin = 0;; ++spin) {
                if (ld_acquire(ticket) == pos) { turn = true; break; }
                if ((spin & 15) == 15) {
                  if (status_set()) break;
                  if (globaltimer_ns() - t0 > kWaitTimeoutNs) {
                    record_error(&g_attn_status, 2);
                    break;
                  }
                  __nanosleep(32);
                }
              }
            }
            turn = __shfl_sync(0xffffffffu, turn, 0);
          }
          if (!turn) { ok = false; break; }
          // one coalesced 128-byte line per query row and warp; the chain's first
          // contributor stores, the others add with fire-and-forget reductions
          const int nrows = min(128, p.N - i * 128);
          float* accp = p.acc + ((static_cast<size_t>(chain) * p.BHq + bhq) * (p.nt * 128) + i * 128) * D + r;
          if (pos == 0) {
#pragma unroll
            for (int q = 0; q < 128; ++q)
              if (q < nrows) accp[static_cast<size_t>(q) * D] = part[q];
          } else {
#pragma unroll
            for (int q = 0; q < 128; ++q)
              if (q < nrows) red_add_f32(accp + static_cast<size_t>(q) * D, part[q]);
          }
          __threadfence();
          __syncwarp();
          if (lane == 0) st_release(ticket, pos + 1);
        }
      }
      if (!ok) break;
      // epilogue of the item: dV and scale * dK rows (TMEM lane = key)
      ok = __all_sync(0xffffffffu, mbar_wait(&sh.step_done, (gs - 1) & 1));
      if (!ok) break;
      tc_fence_after();
      const int key = j * 128 + r;
      const bool live = key < p.N;
      const size_t krow = (static_cast<size_t>(bhkv) * p.N + key) * D;
#pragma unroll
      for (int which = 0; which < 2; ++which) {
        const float mul = which == 0 ? 1.f : p.scale;
        __nv_bfloat16* dst = (which == 0 ? p.dv : p.dk) + krow;
        const uint32_t col = which == 0 ? C::kDV : C::kDK;
#pragma unroll
        for (int q4 = 0; q4 < D / 32; ++q4) {
          uint32_t x[32];
          tmem_ld32(lane_base + col + q4 * 32, x);
          tmem_wait_ld();
          if (live) {
#pragma unroll
            for (int k = 0; k < 4; ++k)
              reinterpret_cast<uint4*>(dst + q4 * 32)[k] = make_uint4(
                  pack_bf16x2(__uint_as_float(x[8 * k]) * mul, __uint_as_float(x[8 * k + 1]) * mul),
                  pack_bf16x2(__uint_as_float(x[8 * k + 2]) * mul, __uint_as_float(x[8 * k + 3]) * mul),
                  pack_bf16x2(__uint_as_float(x[8 * k + 4]) * mul, __uint_as_float(x[8 * k + 5]) * mul),
                  pack_bf16x2(__uint_as_float(x[8 * k + 6]) * mul, __uint_as_float(x[8 * k + 7]) * mul));
          }
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

// ------------------------------------------------------------------ dQ convert
// dq = bf16(scale * sum_c acc[c]) with the chains summed in order c = 0, 1, ...;
// chain c holds a contribution for query tile i only if the tile has more than c
// contributors (i + 1 of them when causal, nt otherwise).
template <int D>
__global__ void __launch_bounds__(256) attn_bwd_dq_kernel(const float* __restrict__ acc, __nv_bfloat16* dq,
                                                          long long BHq, int N, int nt, int causal, float scale) {
  const long long npad = static_cast<long long>(nt) * 128;
  const long long vecs = BHq * N * (D / 8);
  const long long stride = static_cast<long long>(gridDim.x) * blockDim.x;
  for (long long x = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; x < vecs; x += stride) {
    const long long row = x / (D / 8);
    const int c8 = static_cast<int>(x - row * (D / 8)) * 8;
    const long long bh = row / N;
    const int n = static_cast<int>(row - bh * N);
    const int contributors = causal ? (n / 128 + 1) : nt;
    const int nch = contributors < kChains ? contributors : kChains;
    float v[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    for (int c = 0; c < nch; ++c) {
      const float4* src = reinterpret_cast<const float4*>(acc + ((c * BHq + bh) * npad + n) * D + c8);
      const float4 a = src[0], b = src[1];
      v[0] += a.x; v[1] += a.y; v[2] += a.z; v[3] += a.w;
      v[4] += b.x; v[5] += b.y; v[6] += b.z; v[7] += b.w;
    }
    *reinterpret_cast<uint4*>(dq + row * D + c8) =
        make_uint4(pack_bf16x2(v[0] * scale, v[1] * scale), pack_bf16x2(v[2] * scale, v[3] * scale),
                   pack_bf16x2(v[4] * scale, v[5] * scale), pack_bf16x2(v[6] * scale, v[7] * scale));
  }
}

int launch_bwd(const void* q, const void* k, const void* v, const void* o, const float* lse, const void* dO,
               void* dq, void* dk, void* dv, int B, int Hq, int Hkv, int N, int d, float scale, int causal,
               void* workspace, cudaStream_t stream, int sms);

}  // namespace attn
