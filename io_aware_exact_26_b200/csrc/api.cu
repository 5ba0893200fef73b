// Host side of libattn_b200.so: the extern "C" entry points declared in
// include/attn.h.  Validates arguments, encodes the TMA tensor maps, picks the
// kernel instance and launches it on the caller's stream.  No synchronisation on
// the launch path; the only allocation is attn_bwd's stream-ordered workspace when
// the caller passes none.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <atomic>
#include <climits>
#include <cmath>
#include <cstdint>
#include <mutex>

#include "attn.h"
#include "fwd.cuh"
#include "fwd_pp.cuh"
#include "bwd.cuh"
#include "decode.cuh"

namespace {


PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    cudaDriverEntryPointQueryResult q;
    void* p = nullptr;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// 3-D view [heads][rows][d] of a bf16 (elem = 2) or 8-bit (elem = 1) tensor; box =
// 128 bytes of columns x box_rows rows, 128B swizzle.
bool make_map(CUtensorMap* m, const void* ptr, int d, int rows, long long heads, int box_rows, int elem = 2) {
  auto enc = encode_fn();
  if (!enc) return false;
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(rows),
                        static_cast<cuuint64_t>(heads)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(d) * elem, static_cast<cuuint64_t>(d) * elem * rows};
  cuuint32_t box[3] = {static_cast<cuuint32_t>(128 / elem), static_cast<cuuint32_t>(box_rows), 1};
  cuuint32_t es[3] = {1, 1, 1};
  return enc(m, elem == 2 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_UINT8, 3,
             const_cast<void*>(ptr), dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
             CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

struct DeviceInfo {
  int sms = 0;
  int major = 0;
  bool fwd64 = false, fwd128 = false;
};

int device_info(DeviceInfo** out) {
  static DeviceInfo infos[64];
  static std::mutex mu;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 1;
  std::lock_guard<std::mutex> lock(mu);
  DeviceInfo& di = infos[dev];
  if (di.sms == 0) {
    cudaDeviceProp prop;
    if (cudaGetDeviceProperties(&prop, dev) != cudaSuccess) return 1;
    di.major = prop.major;
    di.sms = prop.multiProcessorCount;
  }
  *out = &di;
  return di.major == 10 ? 0 : 1;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int check_common(int B, int Hq, int Hkv, int N, int d, float scale, int causal) {
  if (d != 64 && d != 128) return ATTN_ERR_UNSUPPORTED;
  if (B < 1 || Hq < 1 || Hkv < 1 || N < 1) return ATTN_ERR_INVALID_ARG;
  if (Hq % Hkv != 0) return ATTN_ERR_INVALID_ARG;
  if (!std::isfinite(scale) || scale < 0.f) return ATTN_ERR_INVALID_ARG;
  if (causal != 0 && causal != 1) return ATTN_ERR_INVALID_ARG;
  const long long tiles = static_cast<long long>(B) * Hq * ((N + 127) / 128);
  if (tiles > INT_MAX / 2) return ATTN_ERR_INVALID_ARG;
  if (static_cast<long long>(N) * d * 2 * 2 >= (1ll << 40)) return ATTN_ERR_INVALID_ARG;
  return ATTN_OK;
}


// Band of visible keys as the kernels take it: query i sees keys i - wl .. i + wr,
// each side at most N (= no limit).  A negative window side means no limit.
struct Band {
  int wl, wr;
};
Band band_of_causal(int N, int causal) { return {N, causal ? 0 : N}; }
Band band_of_window(int N, int left, int right) {
  return {(left < 0 || left > N) ? N : left, (right < 0 || right > N) ? N : right};
}

// Work-unit counter slot and generation for the next dynamically scheduled launch:
// slots rotate over attn::kSchedSlots, the generation counts launches (never 0), so
// a launch can tell when a later one has taken its slot over.
struct SchedTicket {
  int slot;
  unsigned int gen;
};
SchedTicket next_sched_ticket() {
  static std::atomic<unsigned> n{0};
  const unsigned v = n.fetch_add(1, std::memory_order_relaxed);
  return {static_cast<int>(v % attn::kSchedSlots), v + 1u == 0u ? 1u : v + 1u};
}

// Forward: two query tiles per CTA (fwd_pp.cuh); F8: e4m3 inputs with descales
// (qk_descale multiplies the scores, o_scale the output).
template <int D, bool F8 = false>
int launch_fwd_pp(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq, int Hkv,
               int N, float scale, Band band, cudaStream_t stream, const DeviceInfo& di, float qk_descale = 1.f,
               float o_scale = 1.f) {
  using C = attn::PpCfg<D, F8>;
  static std::once_flag attr_once[64];
  static bool attr_ok[64];
  int dev = 0;
  cudaGetDevice(&dev);
  std::call_once(attr_once[dev], [&] {
    attr_ok[dev] = cudaFuncSetAttribute(attn::attn_fwd_pp_kernel<D, F8>,
                                        cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmem) == cudaSuccess;
  });
  if (!attr_ok[dev]) return ATTN_ERR_LAUNCH;
  CUtensorMap tq, tk, tv;
  if (!make_map(&tq, q, D, N, static_cast<long long>(B) * Hq, 128, C::ES) ||
      !make_map(&tk, k, D, N, static_cast<long long>(B) * Hkv, 128, C::ES) ||
      !make_map(&tv, v, D, N, static_cast<long long>(B) * Hkv, 128, C::ES))
    return ATTN_ERR_LAUNCH;
  attn::FwdParams p;
  p.o = o;
  p.lse = lse;
  p.B = B;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.N = N;
  p.G = Hq / Hkv;
  p.n_qtiles = (N + 127) / 128;
  p.c = attn::folded_scale(scale * qk_descale);
  p.oscale = o_scale;
  p.wl = band.wl;
  p.wr = band.wr;
  p.desc = band.wr <= band.wl;
  const int upg = (p.G * p.n_qtiles + 1) / 2;
  const int units = B * Hkv * upg;
  const int grid = units < di.sms ? units : di.sms;
  // interleave the last groups that hold about two units per CTA
  int tail = (2 * grid + upg - 1) / upg;
  p.tail_groups = tail < 1 ? 1 : (tail > B * Hkv ? B * Hkv : tail);
  const SchedTicket ticket = next_sched_ticket();
  p.sched_slot = ticket.slot;
  p.sched_gen = ticket.gen;
  attn::sched_reset_kernel<<<1, 32, 0, stream>>>(ticket.slot, ticket.gen);
  attn::attn_fwd_pp_kernel<D, F8><<<grid, C::kThreads, C::kSmem, stream>>>(tq, tk, tv, p);
  return cudaPeekAtLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_LAUNCH;
}

// Split-KV decoding (decode.cuh): how the keys of each (b, kv-head, query block) are
// split.  The work is bound by HBM; units are claimed dynamically, so a few per SM
// keep the tail short while each unit still streams several key tiles.
struct DecodePlan {
  int G, R, nqb, nkt, S, T;
  long long units;
};

DecodePlan decode_plan(int B, int Hq, int Hkv, int Nq, int Nk, int sms) {
  DecodePlan pl;
  pl.G = Hq / Hkv;
  pl.R = Nq < 128 / pl.G ? Nq : 128 / pl.G;
  pl.nqb = (Nq + pl.R - 1) / pl.R;
  pl.nkt = (Nk + 127) / 128;
  const long long pairs = static_cast<long long>(B) * Hkv * pl.nqb;
  const long long target = 8LL * sms;                       // units to aim for
  long long T = (pl.nkt * pairs + target - 1) / target;     // key tiles per split
  if (T < 4) T = 4;
  if (T > pl.nkt) T = pl.nkt;
  pl.S = static_cast<int>((pl.nkt + T - 1) / T);
  pl.T = (pl.nkt + pl.S - 1) / pl.S;                        // equal splits (the last may be shorter)
  pl.units = pairs * pl.S;
  return pl;
}

// Workspace of the split partials: O_s fp32 [rows][S][d], then LSE_s fp32 [rows][S].
struct DecodeWs {
  size_t o_off, l_off, total;
};
DecodeWs decode_ws(long long rows, int S, int d) {
  DecodeWs w;
  auto up = [](size_t x) { return (x + 255) / 256 * 256; };
  w.o_off = 0;
  if (S <= 1) {
    w.l_off = 0;
    w.total = 0;
    return w;
  }
  w.l_off = up(static_cast<size_t>(rows) * S * d * 4);
  w.total = up(w.l_off + static_cast<size_t>(rows) * S * 4);
  return w;
}

template <int D>
int launch_decode(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq, int Hkv,
                  int Nq, int Nk, float scale, int causal, const DecodePlan& pl, void* ws, cudaStream_t stream,
                  const DeviceInfo& di) {
  using C = attn::DecCfg<D>;
  static std::once_flag attr_once[64];
  static bool attr_ok[64];
  int dev = 0;
  cudaGetDevice(&dev);
  std::call_once(attr_once[dev], [&] {
    attr_ok[dev] = cudaFuncSetAttribute(attn::attn_decode_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                        C::kSmem) == cudaSuccess;
  });
  if (!attr_ok[dev]) return ATTN_ERR_LAUNCH;
  CUtensorMap tk, tv;
  if (!make_map(&tk, k, D, Nk, static_cast<long long>(B) * Hkv, 128) ||
      !make_map(&tv, v, D, Nk, static_cast<long long>(B) * Hkv, 128))
    return ATTN_ERR_LAUNCH;
  const long long rows = static_cast<long long>(B) * Hq * Nq;
  const DecodeWs W = decode_ws(rows, pl.S, D);
  attn::DecParams p;
  p.q = static_cast<const __nv_bfloat16*>(q);
  p.o = static_cast<__nv_bfloat16*>(o);
  p.lse = lse;
  p.opart = pl.S > 1 ? reinterpret_cast<float*>(static_cast<char*>(ws) + W.o_off) : nullptr;
  p.lpart = pl.S > 1 ? reinterpret_cast<float*>(static_cast<char*>(ws) + W.l_off) : nullptr;
  p.B = B;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.G = pl.G;
  p.Nq = Nq;
  p.Nk = Nk;
  p.R = pl.R;
  p.nqb = pl.nqb;
  p.S = pl.S;
  p.T = pl.T;
  p.causal = causal;
  p.c = attn::folded_scale(scale);
  p.n_units = static_cast<int>(pl.units);
  const SchedTicket ticket = next_sched_ticket();
  p.sched_slot = ticket.slot;
  p.sched_gen = ticket.gen;
  const int grid = pl.units < di.sms ? static_cast<int>(pl.units) : di.sms;
  attn::sched_reset_kernel<<<1, 32, 0, stream>>>(ticket.slot, ticket.gen);
  attn::attn_decode_kernel<D><<<grid, C::kThreads, C::kSmem, stream>>>(tk, tv, p);
  if (cudaPeekAtLastError() != cudaSuccess) return ATTN_ERR_LAUNCH;
  if (pl.S > 1) {
    long long blocks = (rows * 32 + 255) / 256;
    const long long cap = static_cast<long long>(di.sms) * 16;
    if (blocks > cap) blocks = cap;
    attn::attn_decode_merge_kernel<D><<<static_cast<int>(blocks), 256, 0, stream>>>(
        p.opart, p.lpart, static_cast<__nv_bfloat16*>(o), lse, rows, pl.S);
    if (cudaPeekAtLastError() != cudaSuccess) return ATTN_ERR_LAUNCH;
  }
  return ATTN_OK;
}

int check_decode(int B, int Hq, int Hkv, int Nq, int Nk, int d, float scale, int causal) {
  if (d != 64 && d != 128) return ATTN_ERR_UNSUPPORTED;
  if (B < 1 || Hq < 1 || Hkv < 1 || Nq < 1 || Nk < 1) return ATTN_ERR_INVALID_ARG;
  if (Hq % Hkv != 0 || Hq / Hkv > 128) return ATTN_ERR_INVALID_ARG;
  if (!std::isfinite(scale) || scale < 0.f) return ATTN_ERR_INVALID_ARG;
  if (causal != 0 && causal != 1) return ATTN_ERR_INVALID_ARG;
  if (causal && Nq > Nk) return ATTN_ERR_INVALID_ARG;
  const long long rows = static_cast<long long>(B) * Hq * Nq;
  if (rows * d >= (1ll << 40) || static_cast<long long>(Nk) * d * 2 >= (1ll << 40)) return ATTN_ERR_INVALID_ARG;
  // work units (b, kv-head, query block, key split) must stay below 2^31: blocks <= Nq, splits <= key tiles
  if (static_cast<long long>(B) * Hkv * Nq * ((Nk + 127) / 128) >= (1ll << 31)) return ATTN_ERR_INVALID_ARG;
  return ATTN_OK;
}

}  // namespace

namespace attn {

template <int D>
static int launch_bwd_d(const void* q, const void* k, const void* v, const void* o, const float* lse,
                        const void* dO, void* dq, void* dk, void* dv, int B, int Hq, int Hkv, int N, float scale,
                        int wl, int wr, void* workspace, cudaStream_t stream, int sms) {
  static std::once_flag attr_once[64];
  static bool attr_ok[64];
  int dev = 0;
  cudaGetDevice(&dev);
  std::call_once(attr_once[dev], [&] {
    attr_ok[dev] = cudaFuncSetAttribute(attn_bwd_kv_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                        KvCfg<D>::kSmem) == cudaSuccess &&
                   cudaFuncSetAttribute(attn_bwd_q_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                        QCfg<D>::kSmem) == cudaSuccess;
  });
  if (!attr_ok[dev]) return ATTN_ERR_LAUNCH;
  const long long BHq = static_cast<long long>(B) * Hq;
  const BwdLayout L = bwd_layout(BHq, N);
  char* ws = static_cast<char*>(workspace);
  float* nlse2 = reinterpret_cast<float*>(ws + L.nlse2_off);
  float* ndd = reinterpret_cast<float*>(ws + L.ndd_off);
  const int nt = (N + 127) / 128;
  {
    const long long rows = BHq * nt * 128;
    long long blocks = (rows * (D / 8) + 255) / 256;
    const long long cap = static_cast<long long>(sms) * 16;
    if (blocks > cap) blocks = cap;
    attn_bwd_prep_kernel<D><<<static_cast<int>(blocks), 256, 0, stream>>>(
        static_cast<const __nv_bfloat16*>(o), static_cast<const __nv_bfloat16*>(dO), lse, nlse2, ndd, BHq, N);
    if (cudaPeekAtLastError() != cudaSuccess) return ATTN_ERR_LAUNCH;
  }
  CUtensorMap tq, tk, tv, tdo;
  if (!make_map(&tq, q, D, N, BHq, 128) || !make_map(&tk, k, D, N, static_cast<long long>(B) * Hkv, 128) ||
      !make_map(&tv, v, D, N, static_cast<long long>(B) * Hkv, 128) || !make_map(&tdo, dO, D, N, BHq, 128))
    return ATTN_ERR_LAUNCH;
  BwdParams p;
  p.dq = static_cast<__nv_bfloat16*>(dq);
  p.dk = static_cast<__nv_bfloat16*>(dk);
  p.dv = static_cast<__nv_bfloat16*>(dv);
  p.nlse2 = nlse2;
  p.ndd = ndd;
  p.B = B;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.N = N;
  p.G = Hq / Hkv;
  p.nt = nt;
  p.wl = wl;
  p.wr = wr;
  p.pair = wr == 0 && wl >= N - 1;     // causal: every key tile sees all later query tiles
  p.desc = wr <= wl;
  p.c = folded_scale(scale);
  p.scale = scale;
  // dK, dV: one item per (b, kv-head, key tile); causal: units of two key tiles
  p.npair = (nt + 1) / 2;
  p.total_items = B * Hkv * (p.pair ? p.npair : nt);
  int grid = p.total_items < sms ? p.total_items : sms;
  attn_bwd_kv_kernel<D><<<grid, KvCfg<D>::kThreads, KvCfg<D>::kSmem, stream>>>(tq, tk, tv, tdo, p);
  if (cudaPeekAtLastError() != cudaSuccess) return ATTN_ERR_LAUNCH;
  // dQ: one item per (b, q-head, query tile); causal: units of two query tiles
  p.total_items = B * Hq * (p.pair ? p.npair : nt);
  grid = p.total_items < sms ? p.total_items : sms;
  attn_bwd_q_kernel<D><<<grid, QCfg<D>::kThreads, QCfg<D>::kSmem, stream>>>(tq, tk, tv, tdo, p);
  return cudaPeekAtLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_LAUNCH;
}

int launch_bwd(const void* q, const void* k, const void* v, const void* o, const float* lse, const void* dO,
               void* dq, void* dk, void* dv, int B, int Hq, int Hkv, int N, int d, float scale, int wl, int wr,
               void* workspace, cudaStream_t stream, int sms) {
  if (d == 64)
    return launch_bwd_d<64>(q, k, v, o, lse, dO, dq, dk, dv, B, Hq, Hkv, N, scale, wl, wr, workspace, stream, sms);
  return launch_bwd_d<128>(q, k, v, o, lse, dO, dq, dk, dv, B, Hq, Hkv, N, scale, wl, wr, workspace, stream, sms);
}

}  // namespace attn

// ---------------------------------------------------------------------------
// Scratch for attn_bwd_noalloc: a fixed device array that this library owns, so
// callers that cannot allocate device memory can still run the backward.  Every
// GPU that loads the library holds these bytes until the process exits.
static constexpr size_t kNoAllocScratchBytes = static_cast<size_t>(64) << 20;   // 64 MiB
static __device__ __align__(256) unsigned char g_bwd_scratch[kNoAllocScratchBytes];

// Device address of g_bwd_scratch on the current device, looked up with that device
// current and cached once the lookup succeeds.  In host code the array's name is
// only a host-side stand-in, so kernels must be given this address instead.
// Returns nullptr if the lookup failed (e.g. tried during a stream capture); a
// later call tries again.
static void* noalloc_scratch_on_current_device() {
  static std::atomic<void*> addr[64];
  static std::mutex mu;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  void* a = addr[dev].load(std::memory_order_acquire);
  if (a) return a;
  std::lock_guard<std::mutex> lock(mu);
  a = addr[dev].load(std::memory_order_relaxed);
  if (!a) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_bwd_scratch) == cudaSuccess && p) {
      a = p;
      addr[dev].store(p, std::memory_order_release);
    } else {
      (void)cudaGetLastError();
    }
  }
  return a;
}

extern "C" {

static int fwd_impl(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq, int Hkv,
                    int N, int d, float scale, int causal, Band band, void* stream) {
  int st = check_common(B, Hq, Hkv, N, d, scale, causal);
  if (st != ATTN_OK) return st;
  if (!q || !k || !v || !o || !lse) return ATTN_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse))
    return ATTN_ERR_ALIGNMENT;
  DeviceInfo* di = nullptr;
  if (device_info(&di) != 0) return ATTN_ERR_UNSUPPORTED;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (d == 64) return launch_fwd_pp<64>(q, k, v, o, lse, B, Hq, Hkv, N, scale, band, s, *di);
  return launch_fwd_pp<128>(q, k, v, o, lse, B, Hq, Hkv, N, scale, band, s, *di);
}

int attn_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq, int Hkv, int N,
             int d, float scale, int causal, void* stream) {
  return fwd_impl(q, k, v, o, lse, B, Hq, Hkv, N, d, scale, causal, band_of_causal(N, causal), stream);
}

int attn_fwd_window(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq, int Hkv,
                    int N, int d, float scale, int window_left, int window_right, void* stream) {
  return fwd_impl(q, k, v, o, lse, B, Hq, Hkv, N, d, scale, 0, band_of_window(N, window_left, window_right),
                  stream);
}

int attn_fwd_fp8(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq, int Hkv, int N,
                 int d, float scale, float q_descale, float k_descale, float v_descale, int causal, void* stream) {
  int st = check_common(B, Hq, Hkv, N, d, scale, causal);
  if (st != ATTN_OK) return st;
  for (float x : {q_descale, k_descale, v_descale})
    if (!std::isfinite(x) || !(x > 0.f)) return ATTN_ERR_INVALID_ARG;
  if (!std::isfinite(scale * q_descale * k_descale)) return ATTN_ERR_INVALID_ARG;
  if (!q || !k || !v || !o || !lse) return ATTN_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse))
    return ATTN_ERR_ALIGNMENT;
  DeviceInfo* di = nullptr;
  if (device_info(&di) != 0) return ATTN_ERR_UNSUPPORTED;
  if (d == 64)
    return launch_fwd_pp<64, true>(q, k, v, o, lse, B, Hq, Hkv, N, scale, band_of_causal(N, causal),
                                   static_cast<cudaStream_t>(stream), *di, q_descale * k_descale, v_descale);
  return launch_fwd_pp<128, true>(q, k, v, o, lse, B, Hq, Hkv, N, scale, band_of_causal(N, causal),
                                  static_cast<cudaStream_t>(stream), *di, q_descale * k_descale, v_descale);
}

size_t attn_bwd_workspace_size(int B, int Hq, int Hkv, int N, int d, int causal) {
  if (check_common(B, Hq, Hkv, N, d, 1.f, causal) != ATTN_OK) return 0;
  return attn::bwd_workspace_bytes(B, Hq, Hkv, N, d);
}

static int bwd_impl(const void* q, const void* k, const void* v, const void* o, const float* lse, const void* dO,
                    void* dq, void* dk, void* dv, int B, int Hq, int Hkv, int N, int d, float scale, int causal,
                    Band band, void* workspace, size_t workspace_bytes, void* stream) {
  int st = check_common(B, Hq, Hkv, N, d, scale, causal);
  if (st != ATTN_OK) return st;
  if (!q || !k || !v || !o || !lse || !dO || !dq || !dk || !dv) return ATTN_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse) || !aligned16(dO) ||
      !aligned16(dq) || !aligned16(dk) || !aligned16(dv))
    return ATTN_ERR_ALIGNMENT;
  const size_t need = attn::bwd_workspace_bytes(B, Hq, Hkv, N, d);
  if (workspace && workspace_bytes < need) return ATTN_ERR_WORKSPACE;
  if (workspace && !aligned16(workspace)) return ATTN_ERR_ALIGNMENT;
  DeviceInfo* di = nullptr;
  if (device_info(&di) != 0) return ATTN_ERR_UNSUPPORTED;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  // No caller workspace: a stream-ordered allocation, freed on the same stream right
  // behind the kernels that use it (the memory returns to the device's pool once they end).
  void* ws = workspace;
  if (!ws) {
    if (cudaMallocAsync(&ws, need, s) != cudaSuccess) {
      (void)cudaGetLastError();
      return ATTN_ERR_ALLOC;
    }
  }
  const int st2 = attn::launch_bwd(q, k, v, o, lse, dO, dq, dk, dv, B, Hq, Hkv, N, d, scale, band.wl, band.wr,
                                   ws, s, di->sms);
  if (!workspace && cudaFreeAsync(ws, s) != cudaSuccess) {
    (void)cudaGetLastError();
    return st2 != ATTN_OK ? st2 : ATTN_ERR_ALLOC;
  }
  return st2;
}

int attn_bwd(const void* q, const void* k, const void* v, const void* o, const float* lse, const void* dO,
             void* dq, void* dk, void* dv, int B, int Hq, int Hkv, int N, int d, float scale, int causal,
             void* workspace, size_t workspace_bytes, void* stream) {
  return bwd_impl(q, k, v, o, lse, dO, dq, dk, dv, B, Hq, Hkv, N, d, scale, causal, band_of_causal(N, causal),
                  workspace, workspace_bytes, stream);
}

int attn_bwd_window(const void* q, const void* k, const void* v, const void* o, const float* lse,
                    const void* dO, void* dq, void* dk, void* dv, int B, int Hq, int Hkv, int N, int d,
                    float scale, int window_left, int window_right, void* workspace, size_t workspace_bytes,
                    void* stream) {
  return bwd_impl(q, k, v, o, lse, dO, dq, dk, dv, B, Hq, Hkv, N, d, scale, 0,
                  band_of_window(N, window_left, window_right), workspace, workspace_bytes, stream);
}

size_t attn_decode_workspace_size(int B, int Hq, int Hkv, int Nq, int Nk, int d, int causal) {
  if (check_decode(B, Hq, Hkv, Nq, Nk, d, 1.f, causal) != ATTN_OK) return 0;
  DeviceInfo* di = nullptr;
  if (device_info(&di) != 0) return 0;
  const DecodePlan pl = decode_plan(B, Hq, Hkv, Nq, Nk, di->sms);
  return decode_ws(static_cast<long long>(B) * Hq * Nq, pl.S, d).total;
}

int attn_decode(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq, int Hkv, int Nq,
                int Nk, int d, float scale, int causal, void* workspace, size_t workspace_bytes, void* stream) {
  int st = check_decode(B, Hq, Hkv, Nq, Nk, d, scale, causal);
  if (st != ATTN_OK) return st;
  if (!q || !k || !v || !o || !lse) return ATTN_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse))
    return ATTN_ERR_ALIGNMENT;
  if (workspace && !aligned16(workspace)) return ATTN_ERR_ALIGNMENT;
  DeviceInfo* di = nullptr;
  if (device_info(&di) != 0) return ATTN_ERR_UNSUPPORTED;
  const DecodePlan pl = decode_plan(B, Hq, Hkv, Nq, Nk, di->sms);
  const size_t need = decode_ws(static_cast<long long>(B) * Hq * Nq, pl.S, d).total;
  if (workspace && workspace_bytes < need) return ATTN_ERR_WORKSPACE;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  void* ws = workspace;
  if (!ws && need > 0) {
    if (cudaMallocAsync(&ws, need, s) != cudaSuccess) {
      (void)cudaGetLastError();
      return ATTN_ERR_ALLOC;
    }
  }
  const int st2 = d == 64 ? launch_decode<64>(q, k, v, o, lse, B, Hq, Hkv, Nq, Nk, scale, causal, pl, ws, s, *di)
                          : launch_decode<128>(q, k, v, o, lse, B, Hq, Hkv, Nq, Nk, scale, causal, pl, ws, s, *di);
  if (!workspace && need > 0 && cudaFreeAsync(ws, s) != cudaSuccess) {
    (void)cudaGetLastError();
    return st2 != ATTN_OK ? st2 : ATTN_ERR_ALLOC;
  }
  return st2;
}

int attn_decode_splits(int B, int Hq, int Hkv, int Nq, int Nk, int d, int causal) {
  if (check_decode(B, Hq, Hkv, Nq, Nk, d, 1.f, causal) != ATTN_OK) return 0;
  DeviceInfo* di = nullptr;
  if (device_info(&di) != 0) return 0;
  return decode_plan(B, Hq, Hkv, Nq, Nk, di->sms).S;
}

int attn_merge(float* o_acc, float* lse_acc, const void* o_part, const float* lse_part, long long rows, int d,
               void* out, void* stream) {
  if (d != 64 && d != 128) return ATTN_ERR_UNSUPPORTED;
  if (rows < 1 || rows * d >= (1ll << 40)) return ATTN_ERR_INVALID_ARG;
  if (!o_acc || !lse_acc || !o_part || !lse_part) return ATTN_ERR_INVALID_ARG;
  if (!aligned16(o_acc) || !aligned16(lse_acc) || !aligned16(o_part) || !aligned16(lse_part) ||
      (out && !aligned16(out)))
    return ATTN_ERR_ALIGNMENT;
  DeviceInfo* di = nullptr;
  if (device_info(&di) != 0) return ATTN_ERR_UNSUPPORTED;
  long long blocks = (rows * 32 + 255) / 256;
  const long long cap = static_cast<long long>(di->sms) * 16;
  if (blocks > cap) blocks = cap;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  auto* po = static_cast<const __nv_bfloat16*>(o_part);
  auto* pout = static_cast<__nv_bfloat16*>(out);
  if (d == 64)
    attn::attn_merge_kernel<64><<<static_cast<int>(blocks), 256, 0, s>>>(o_acc, lse_acc, po, lse_part, pout, rows);
  else
    attn::attn_merge_kernel<128><<<static_cast<int>(blocks), 256, 0, s>>>(o_acc, lse_acc, po, lse_part, pout, rows);
  return cudaPeekAtLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_LAUNCH;
}

int attn_accumulate(float* acc, const void* part, long long n, void* stream) {
  if (!acc || !part || n < 8 || n % 8 != 0 || n >= (1ll << 40)) return ATTN_ERR_INVALID_ARG;
  if (!aligned16(acc) || !aligned16(part)) return ATTN_ERR_ALIGNMENT;
  DeviceInfo* di = nullptr;
  if (device_info(&di) != 0) return ATTN_ERR_UNSUPPORTED;
  const long long n8 = n / 8;
  long long blocks = (n8 + 255) / 256;
  const long long cap = static_cast<long long>(di->sms) * 8;
  if (blocks > cap) blocks = cap;
  attn::attn_accumulate_kernel<<<static_cast<int>(blocks), 256, 0, static_cast<cudaStream_t>(stream)>>>(
      acc, static_cast<const __nv_bfloat16*>(part), n8);
  return cudaPeekAtLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_LAUNCH;
}

int attn_bwd_noalloc(const void* q, const void* k, const void* v, const void* o, const float* lse,
                     const void* dO, void* dq, void* dk, void* dv, int B, int Hq, int Hkv, int N, int d,
                     float scale, int causal, void* stream) {
  int st = check_common(B, Hq, Hkv, N, d, scale, causal);
  if (st != ATTN_OK) return st;
  if (attn::bwd_workspace_bytes(B, Hq, Hkv, N, d) > kNoAllocScratchBytes) return ATTN_ERR_WORKSPACE;
  DeviceInfo* di = nullptr;
  if (device_info(&di) != 0) return ATTN_ERR_UNSUPPORTED;
  void* scratch = noalloc_scratch_on_current_device();
  if (!scratch) return ATTN_ERR_LAUNCH;
  return attn_bwd(q, k, v, o, lse, dO, dq, dk, dv, B, Hq, Hkv, N, d, scale, causal, scratch,
                  kNoAllocScratchBytes, stream);
}

}  // extern "C"

namespace {
// Waits on an mbarrier that nothing arrives on, with the kernels' bounded-wait
// code and a short limit: the wait gives up, records the timeout in the error
// word and the kernel returns.
__global__ void selftest_timeout_kernel(unsigned long long limit_ns) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    attn::mbar_init(&bar, 1);
    attn::fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) (void)attn::mbar_wait_for(&bar, 0, limit_ns);
}
// Hands the index check a value outside its range; nothing is accessed with it.
__global__ void selftest_bounds_kernel() {
  if (threadIdx.x == 0) (void)attn::in_range(5, 3);
}
// Runs the work-unit claim on the self-test slot as launch generation `gen`: one
// producer posts `count` claims (of n = 3 units) into a ring, the warp takes them
// and writes them to out[0 .. count).
__global__ void selftest_sched_kernel(int* out, unsigned int gen, int count) {
  __shared__ attn::UnitRing ring;
  const int lane = threadIdx.x;
  if (lane == 0) {
    attn::unit_ring_init(ring, 1);
    attn::fence_barrier_init();
  }
  __syncwarp();
  if (lane == 0)
    for (int k = 0; k < count; ++k) (void)attn::unit_ring_claim(ring, k, attn::kSchedSelftestSlot, gen, 3);
  __syncwarp();
  for (int k = 0; k < count; ++k) {
    bool ok = true;
    const int u = attn::unit_ring_take(ring, k, lane, ok);
    if (lane == 0) out[k] = ok ? u : -2;
  }
}
}  // namespace

extern "C" {

int attn_selftest_sched(int* out, void* stream) {
  if (out == nullptr) return ATTN_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(out) % alignof(int) != 0) return ATTN_ERR_ALIGNMENT;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  // generation 7 claims units 0, 1, 2 and then none; after generation 8 takes the
  // slot over, generation 7 gets nothing (and records the conflict) and its stray
  // increment makes generation 8 start at 1
  attn::sched_reset_kernel<<<1, 32, 0, s>>>(attn::kSchedSelftestSlot, 7u);
  selftest_sched_kernel<<<1, 32, 0, s>>>(out, 7u, 4);
  attn::sched_reset_kernel<<<1, 32, 0, s>>>(attn::kSchedSelftestSlot, 8u);
  selftest_sched_kernel<<<1, 32, 0, s>>>(out + 4, 7u, 1);
  selftest_sched_kernel<<<1, 32, 0, s>>>(out + 5, 8u, 1);
  return cudaPeekAtLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_LAUNCH;
}

int attn_selftest_timeout(long long limit_ns, void* stream) {
  if (limit_ns <= 0 || limit_ns > 1000000000LL) return ATTN_ERR_INVALID_ARG;
  selftest_timeout_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(static_cast<unsigned long long>(limit_ns));
  return cudaPeekAtLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_LAUNCH;
}

int attn_get_device_status(void* stream) {
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return ATTN_ERR_LAUNCH;
  int v = 0, zero = 0;
  if (cudaMemcpyFromSymbol(&v, attn::g_attn_status, sizeof(int)) != cudaSuccess) return ATTN_ERR_LAUNCH;
  if (v != 0 && cudaMemcpyToSymbol(attn::g_attn_status, &zero, sizeof(int)) != cudaSuccess)
    return ATTN_ERR_LAUNCH;
  return v == 0 ? ATTN_OK : v == 2 ? ATTN_ERR_DEVICE_BOUNDS : v == 3 ? ATTN_ERR_SCHED_CONFLICT
                                                                       : ATTN_ERR_DEVICE_TIMEOUT;
}

int attn_checks_enabled(void) { return attn::kChecks ? 1 : 0; }

int attn_selftest_bounds(void* stream) {
  selftest_bounds_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>();
  return cudaPeekAtLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_LAUNCH;
}

const char* attn_status_string(int status) {
  switch (status) {
    case ATTN_OK: return "ok";
    case ATTN_ERR_INVALID_ARG: return "invalid argument";
    case ATTN_ERR_UNSUPPORTED: return "unsupported (head dim must be 64 or 128; device must be sm_100)";
    case ATTN_ERR_ALIGNMENT: return "pointer not 16-byte aligned";
    case ATTN_ERR_LAUNCH: return "CUDA launch or attribute error";
    case ATTN_ERR_DEVICE_TIMEOUT: return "a bounded device-side wait expired";
    case ATTN_ERR_WORKSPACE: return "backward workspace too small";
    case ATTN_ERR_ALLOC: return "stream-ordered allocation of the library's workspace failed";
    case ATTN_ERR_DEVICE_BOUNDS: return "a device-side index check failed (checking build)";
    case ATTN_ERR_SCHED_CONFLICT:
      return "a launch's work counter was taken over by a later launch (over 128 in flight); both outputs are incomplete";
    default: return "unknown status";
  }
}

}  // extern "C"
