// Issue-rate probe for the tensor-core instruction shapes the attention kernels use.
//
// One CTA per SM allocates all of tensor memory, fills 96 KB of shared memory with
// zeros and has one elected thread issue `reps` groups of 8 tcgen05.mma (M = 128,
// K = 16, bf16 in, fp32 accumulate; 8 instructions = one K = 128 contraction) back to
// back, then waits (bounded) for their commit.  The elapsed SM cycles divided by the
// instruction count is the steady-state cost of one instruction of that shape:
//   SS: A and B from shared memory (128B-swizzled, K-major), as S = Q K^T;
//   TS: A from tensor memory, B from shared memory, as O += P V;
// and two sequences as the kernels issue them: the dK/dV step (8 TS, 8 SS, 8 TS, 8 SS)
// and the forward tile (8 SS, 8 TS).  A second kernel measures tcgen05.ld bandwidth.
// The values are zeros: no result is read, only time.
#include "sm100.cuh"

using namespace attn;

namespace {

constexpr int kSmemBytes = 200 * 1024;   // one CTA per SM, so each may allocate all 512 columns

// mode: 0 SS N=128, 1 SS N=64, 2 TS N=128, 3 TS N=64, 4 SS N=256,
//       5 dK/dV step sequence, 6 forward tile sequence
__global__ void __launch_bounds__(128, 1) mma_rate_kernel(int mode, int reps, unsigned long long* out) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;            // 128 rows x 128 bf16: two 16 KB boxes of 64 columns
  uint8_t* sB = smem + 32768;    // up to 256 rows x 128 bf16
  __shared__ uint64_t bar;
  __shared__ uint32_t tbase;
  for (int i = threadIdx.x; i < (32768 + 65536) / 16; i += blockDim.x)
    reinterpret_cast<uint4*>(smem)[i] = make_uint4(0, 0, 0, 0);
  fence_proxy_async_smem();
  const int warp = threadIdx.x >> 5;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_barrier_init();
  }
  if (warp == 0) {
    tmem_alloc(&tbase, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tbase;
  if (warp == 0) {
    const bool leader = elect_one();
    const uint32_t hi = sdesc_hi_sw128(1024);
    const uint32_t a_lo = sdesc_lo(smem_u32(sA), 16), b_lo = sdesc_lo(smem_u32(sB), 16);
    // accumulators in columns 0-255, the tensor-memory A operand in columns 256-351
    auto group = [&](bool ts, int n, uint32_t dcol) {
      const uint32_t id = idesc_bf16_f32(128, n, false, false);
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        const uint32_t off = ((k >> 2) * 16384 + (k & 3) * 32) >> 4;
        if (ts)
          umma_ts_lo(tmem + dcol, tmem + 256 + (k >> 2) * 64 + (k & 3) * 8, b_lo + off, hi, id, 1);
        else
          umma_ss_lo(tmem + dcol, a_lo + off, b_lo + off, hi, id, 1);
      }
    };
    const long long t0 = clock64();
    if (leader) {
      for (int r = 0; r < reps; ++r) {
        switch (mode) {
          case 0: group(false, 128, 0); break;
          case 1: group(false, 64, 0); break;
          case 2: group(true, 128, 0); break;
          case 3: group(true, 64, 0); break;
          case 4: group(false, 256, 0); break;
          case 5: group(true, 128, 0); group(false, 128, 128); group(true, 128, 0); group(false, 128, 128); break;
          default: group(false, 128, 0); group(true, 128, 128); break;
        }
      }
      umma_commit(&bar);
    }
    __syncwarp();
    const bool ok = mbar_wait(&bar, 0);
    const long long t1 = clock64();
    if (leader) {
      out[blockIdx.x * 2] = static_cast<unsigned long long>(t1 - t0);
      out[blockIdx.x * 2 + 1] = ok ? 1ull : 0ull;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// Every warp loads 64 columns (4 x 16) of its lane quarter per iteration and waits;
// with `store`, it also writes 16 columns back.  Cycles per warp.
__global__ void __launch_bounds__(512, 1) tmem_ld_rate_kernel(int reps, int store, unsigned long long* out) {
  __shared__ uint32_t tbase;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (warp == 0) {
    tmem_alloc(&tbase, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tbase;
  const uint32_t base = tmem + (static_cast<uint32_t>((warp & 3) * 32) << 16) + (warp >> 2) * 64;
  uint32_t acc = 0;
  const long long t0 = clock64();
  for (int r = 0; r < reps; ++r) {
    uint32_t a[16], b[16], c[16], d[16];
    tmem_ld16(base, a);
    tmem_ld16(base + 16, b);
    tmem_ld16(base + 32, c);
    tmem_ld16(base + 48, d);
    tmem_wait_ld();
    reg_fence(a);
    reg_fence(b);
    reg_fence(c);
    reg_fence(d);
#pragma unroll
    for (int i = 0; i < 16; ++i) acc ^= a[i] ^ b[i] ^ c[i] ^ d[i];
    if (store) {
      tmem_st16(base, a);
      tmem_wait_st();
    }
  }
  const long long t1 = clock64();
  if (lane == 0) out[blockIdx.x * 16 + warp] = static_cast<unsigned long long>(t1 - t0) + (acc == 0x9e3779b9u);
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

int finish(unsigned long long* d, unsigned long long* host, size_t n) {
  cudaError_t e = cudaDeviceSynchronize();
  if (e == cudaSuccess) e = cudaMemcpy(host, d, n * sizeof(unsigned long long), cudaMemcpyDeviceToHost);
  cudaFree(d);
  return e == cudaSuccess ? 0 : -3;
}

}  // namespace

extern "C" {

// host_out: 2 * grid values (cycles, completed flag) per CTA.
int probe_mma_rate(int mode, int reps, int grid, unsigned long long* host_out) {
  if (mode < 0 || mode > 6 || reps < 1 || grid < 1 || grid > 1024 || host_out == nullptr) return -1;
  if (cudaFuncSetAttribute(mma_rate_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes) != cudaSuccess)
    return -2;
  unsigned long long* d = nullptr;
  if (cudaMalloc(&d, 2 * grid * sizeof(unsigned long long)) != cudaSuccess) return -2;
  mma_rate_kernel<<<grid, 128, kSmemBytes>>>(mode, reps, d);
  return finish(d, host_out, 2 * static_cast<size_t>(grid));
}

// host_out: 16 * grid values (cycles per warp slot; unused slots 0).
int probe_tmem_ld_rate(int reps, int warps, int store, int grid, unsigned long long* host_out) {
  if (warps < 1 || warps > 16 || reps < 1 || grid < 1 || grid > 1024 || host_out == nullptr) return -1;
  if (cudaFuncSetAttribute(tmem_ld_rate_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, 150 * 1024) !=
      cudaSuccess)
    return -2;
  unsigned long long* d = nullptr;
  if (cudaMalloc(&d, 16 * grid * sizeof(unsigned long long)) != cudaSuccess) return -2;
  if (cudaMemset(d, 0, 16 * grid * sizeof(unsigned long long)) != cudaSuccess) {
    cudaFree(d);
    return -2;
  }
  tmem_ld_rate_kernel<<<grid, warps * 32, 150 * 1024>>>(reps, store, d);
  return finish(d, host_out, 16 * static_cast<size_t>(grid));
}

}  // extern "C"
