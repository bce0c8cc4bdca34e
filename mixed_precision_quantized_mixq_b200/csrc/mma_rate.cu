// Tensor-core rate loop: the dense tcgen05.mma throughput of this device,
// measured with the same instruction forms the layer's GEMMs use, so that the
// tensor-bound GEMMs can be reported against a peak taken on the same chip in
// the same run (rather than a nominal figure or another data type's rate).
//
// Every CTA (one per SM: its shared-memory request leaves room for no second
// CTA) keeps one A tile (128 rows x 128 bytes) and one B tile (256 rows x 128
// bytes) resident in shared memory in the 128-byte swizzled K-major layout,
// filled with a hashed byte pattern (operand values change the power drawn,
// so they are not zeros), and one elected thread issues `iters` rounds of four
// back-to-back MMAs, M = 128, N = 256, one 32-byte K slice each, into one
// tensor-memory accumulator.  One commit at the end; the CTA waits for it
// (bounded) and frees its tensor memory.
//   kind 0: kind::i8, s8 x s8 -> s32, K = 32 per MMA
//   kind 1: kind::f16, f16 x f16 -> f32, K = 16 per MMA
#include <cuda_fp16.h>

#include <atomic>

#include "internal.h"
#include "ptx.cuh"
#include "tma_host.h"

namespace mixq {
namespace {

constexpr int kRThreads = 128;
constexpr int kRABytes = 128 * 128;
constexpr int kRBBytes = 256 * 128;
// about half the shared memory of an SM: one CTA per SM
constexpr int kRSmem = 120 * 1024;
constexpr int kRCols = 256;

template <int KIND>
__global__ void __launch_bounds__(kRThreads, 1)
    mma_rate_kernel(int iters, int32_t *status, uint64_t limit_ns) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t *A = smem;
  uint8_t *B = smem + kRABytes;
  uint64_t *bar = reinterpret_cast<uint64_t *>(smem + kRABytes + kRBBytes);
  uint32_t *holder = reinterpret_cast<uint32_t *>(bar + 1);
  const int warp = threadIdx.x >> 5;

  uint32_t *words = reinterpret_cast<uint32_t *>(smem);
  for (int i = threadIdx.x; i < (kRABytes + kRBBytes) / 4; i += kRThreads) {
    uint32_t h = (static_cast<uint32_t>(i) + 7919u * blockIdx.x) * 2654435761u;
    h ^= h >> 15;
    h *= 2246822519u;
    h ^= h >> 13;
    // fp16: finite values of magnitude below 0.5 with random signs
    words[i] = KIND == 0 ? h : ((h & 0x37FF37FFu) | (h & 0x80008000u));
  }
  fence_proxy_async_smem();
  if (threadIdx.x == 0) {
    mbar_init(bar, 1);
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(holder, kRCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t d = *holder;

  if (threadIdx.x == 0) {
    const uint64_t ad = sw128_kmajor_desc(smem_u32(A));
    const uint64_t bd = sw128_kmajor_desc(smem_u32(B));
    const uint32_t id = KIND == 0 ? idesc_s8_s32(128, 256) : idesc_f16_f32(128, 256);
#pragma unroll 1
    for (int i = 0; i < iters; ++i) {
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const uint32_t acc = (i | k) != 0 ? 1u : 0u;
        if (KIND == 0)
          mma_i8(d, ad + 2 * k, bd + 2 * k, id, acc);
        else
          mma_f16(d, ad + 2 * k, bd + 2 * k, id, acc);
      }
    }
    mma_commit(bar);
  }
  __syncwarp();
  // every MMA completes on its own (nothing it waits for): a wait that runs out
  // is reported, then waited out again before the accumulator is freed
  if (!mbar_wait(bar, 0, limit_ns)) {
    if (threadIdx.x == 0) record_error(status, kErrTimeout);
    mbar_wait(bar, 0, limit_ns);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(d, kRCols);
  }
}

}  // namespace

double mma_rate_ops_per_launch(int kind, int iters, int num_sms) {
  const double k = kind == 0 ? 32.0 : 16.0;
  return static_cast<double>(num_sms) * iters * 4.0 * 2.0 * 128.0 * 256.0 * k;
}

cudaError_t launch_mma_rate(int kind, int iters, int num_sms, int32_t *status,
                            uint64_t wait_limit_ns, cudaStream_t stream) {
  static std::atomic<uint64_t> done_i8{0}, done_f16{0};
  cudaError_t e = kind == 0 ? ensure_smem(mma_rate_kernel<0>, kRSmem, done_i8)
                            : ensure_smem(mma_rate_kernel<1>, kRSmem, done_f16);
  if (e != cudaSuccess) return e;
  if (kind == 0)
    mma_rate_kernel<0><<<num_sms, kRThreads, kRSmem, stream>>>(iters, status, wait_limit_ns);
  else
    mma_rate_kernel<1><<<num_sms, kRThreads, kRSmem, stream>>>(iters, status, wait_limit_ns);
  return cudaGetLastError();
}

}  // namespace mixq
