// Forward exact attention for sm_100a: definitions shared by the forward kernel
// (fwd_pp.cuh).
//
// exp2 with a folded scale: c = scale * log2(e), p = exp2(s*c - m) where m is
// kept in log2 units; LSE = ln(2) * (m + log2 l).  The max used for the
// exponent is allowed to be stale by up to kRescaleTau (log2 units): by shift
// invariance of softmax (page "attn-efficient": subtracting the same number from
// a whole score row leaves the result unchanged) any reference value works as
// long as O and l use the same one; this keeps p <= 2^tau and skips most O
// rescales.  l is the fp32 sum of the unrounded p; P is rounded to bf16 for the
// PV MMA.
#pragma once
#include "sm100.cuh"

namespace attn {

constexpr float kRescaleTau = 8.0f;

// Folded scale c = scale * log2(e), floored at 1e-30 so that a masked score (-inf)
// times c stays -inf (with c = 0 it would be NaN).  The floor changes nothing else:
// for any c <= 1e-30 every finite exponent argument s*c - m rounds to the same
// fp32 value as with the exact c (|s| is far below 1e20 for bf16 inputs of this
// size), so scale = 0 still gives uniform attention over the visible keys.
__host__ __device__ inline float folded_scale(float scale) {
  const float c = scale * 1.4426950408889634f;
  return c > 1e-30f ? c : 1e-30f;
}

// Visibility of key j from query i: i - wl <= j <= i + wr.  wl = wr = N is full
// attention, (N, 0) causal, (w - 1, 0) a causal sliding window of w keys (page
// "attn-efficient", sliding-window row of the family table).
struct FwdParams {
  void* o;
  float* lse;
  int B, Hq, Hkv, N, G;
  int n_qtiles;
  float c;          // scale * log2(e) (with the Q and K descales for e4m3 inputs)
  float oscale;     // output multiplier: V's descale for e4m3 inputs, else 1
  int wl, wr;       // window: 0 <= wl, wr <= N
  int desc;         // list query tiles last-first (their key ranges grow with the tile)
  int tail_groups;  // number of last KV groups whose units are interleaved (1 <= . <= B * Hkv)
  int sched_slot;   // g_sched slot this launch claims work units from
  unsigned int sched_gen;   // the launch's generation in that slot
};

// Key tiles [j0, j0 + n) that query tile qt sees (n >= 1 for a tile with a row < N).
__device__ __forceinline__ void fwd_kv_range(const FwdParams& p, int qt, int& j0, int& n) {
  const int r0 = qt * 128, r1 = min(p.N - 1, r0 + 127);
  const int k0 = max(0, r0 - p.wl), k1 = min(p.N - 1, r1 + p.wr);
  j0 = k0 >> 7;
  n = (k1 >> 7) - j0 + 1;
}

}  // namespace attn
