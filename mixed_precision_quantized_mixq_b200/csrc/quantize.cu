// Fused activation pass of the MixQ layer: per-token amax over outlier and
// non-outlier channels, the amax > threshold outlier test, the order-preserved
// gather of outlier channels into X_out, INT8 quantization of the rest, and a
// matrix-wide detection bitmap (MixQ article "一键部署LLM混合精度推理…",
// MixQ的解决方案: the amax of quantization doubles as the outlier test;
// Fig. 10 equivalent transformation; Fig. 11 order-preserved outlier matrix).
//
// HBM-bound: one read of X (16-byte vector loads, the second pass over a row
// hits L1), one write of Xq (8-byte stores), K_out_pad fp16 per token of
// X_out.  One CTA walks token rows with a grid stride; the outlier channel
// mask lives in shared memory as a bitset built once per CTA.
#include <cuda_fp16.h>

#include "internal.h"
#include "ptx.cuh"

namespace mixq {
namespace {

constexpr int kQThreads = 256;
constexpr int kQWarps = kQThreads / 32;

__global__ void reset_detect_kernel(uint32_t *__restrict__ bitmap, int words,
                                    int32_t *__restrict__ flags) {
  for (int w = threadIdx.x; w < words; w += blockDim.x) bitmap[w] = 0u;
  if (threadIdx.x < 4) flags[threadIdx.x] = 0;
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

__device__ __forceinline__ int warp_sum(int v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// clamp(rint(x * inv), -127, 127): one IEEE fp32 multiply, round half to even.
__device__ __forceinline__ uint32_t code8(float x, float inv) {
  int q = __float2int_rn(__fmul_rn(x, inv));
  q = max(-127, min(127, q));
  return static_cast<uint32_t>(q) & 0xFFu;
}

__global__ void __launch_bounds__(kQThreads) quantize_act_kernel(
    const __half *__restrict__ X, int M, int K, int ldx, const int32_t *__restrict__ idx,
    int K_out, int K_out_pad, float T, int8_t *__restrict__ Xq, float *__restrict__ s_x,
    __half *__restrict__ X_out, uint32_t *__restrict__ bitmap, int32_t *__restrict__ flags,
    int32_t *__restrict__ status) {
  extern __shared__ uint32_t qsm[];
  const int words = K >> 5;  // K % 128 == 0
  uint32_t *s_mask = qsm;                                    // outlier channel bitset
  uint32_t *s_det = qsm + words;                             // channels with |x| > T
  int32_t *s_idx = reinterpret_cast<int32_t *>(qsm + 2 * words);  // validated idx copy
  __shared__ float s_red[2][kQWarps];
  __shared__ int s_bad, s_last, s_cnt[kQWarps];

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  for (int w = tid; w < words; w += kQThreads) {
    s_mask[w] = 0u;
    s_det[w] = 0u;
  }
  if (tid == 0) s_bad = 0;
  __syncthreads();
  for (int j = tid; j < K_out; j += kQThreads) {
    int c = idx[j];
    const bool ok = c >= 0 && c < K && (j == 0 || idx[j - 1] < c);
    if (!ok) {
      s_bad = 1;
      c = -1;
    }
    s_idx[j] = c;
    if (c >= 0) atomicOr(&s_mask[c >> 5], 1u << (c & 31));
  }
  __syncthreads();
  if (s_bad && tid == 0 && blockIdx.x == 0) record_error(status, kErrInvalidArg);

  const int nvec = K >> 3;  // 8 fp16 per 16-byte vector
  int mixed_rows = 0;
  for (int m = blockIdx.x; m < M; m += gridDim.x) {
    const uint4 *xr = reinterpret_cast<const uint4 *>(X + static_cast<size_t>(m) * ldx);
    float aI = 0.f, aN = 0.f;
    for (int v = tid; v < nvec; v += kQThreads) {
      const uint4 raw = __ldg(xr + v);
      const int k0 = v << 3;
      const uint32_t mb = (s_mask[k0 >> 5] >> (k0 & 31)) & 0xFFu;
      const __half2 *h = reinterpret_cast<const __half2 *>(&raw);
      uint32_t det = 0;
#pragma unroll
      for (int e2 = 0; e2 < 4; ++e2) {
        const float2 f = __half22float2(h[e2]);
        const float a0 = fabsf(f.x), a1 = fabsf(f.y);
        if ((mb >> (2 * e2)) & 1u) aI = fmaxf(aI, a0); else aN = fmaxf(aN, a0);
        if ((mb >> (2 * e2 + 1)) & 1u) aI = fmaxf(aI, a1); else aN = fmaxf(aN, a1);
        det |= (a0 > T ? 1u : 0u) << (2 * e2);
        det |= (a1 > T ? 1u : 0u) << (2 * e2 + 1);
      }
      if (det) atomicOr(&s_det[k0 >> 5], det << (k0 & 31));
    }
    aI = warp_max(aI);
    aN = warp_max(aN);
    if (lane == 0) {
      s_red[0][warp] = aI;
      s_red[1][warp] = aN;
    }
    __syncthreads();
    float rI = s_red[0][0], rN = s_red[1][0];
#pragma unroll
    for (int w = 1; w < kQWarps; ++w) {
      rI = fmaxf(rI, s_red[0][w]);
      rN = fmaxf(rN, s_red[1][w]);
    }
    __syncthreads();  // s_red is rewritten by the next row

    const float amax = fmaxf(rI, rN);
    const bool mixed = K_out > 0 && amax > T;
    const float a = mixed ? rN : amax;
    const float inv = a > 0.f ? __fdiv_rn(127.f, a) : 0.f;
    if (tid == 0) {
      s_x[m] = __fdiv_rn(a, 127.f);
      mixed_rows += mixed ? 1 : 0;
    }

    uint2 *qr = reinterpret_cast<uint2 *>(Xq + static_cast<size_t>(m) * K);
    for (int v = tid; v < nvec; v += kQThreads) {
      const uint4 raw = __ldg(xr + v);
      const int k0 = v << 3;
      const uint32_t mb = mixed ? (s_mask[k0 >> 5] >> (k0 & 31)) & 0xFFu : 0u;
      const __half2 *h = reinterpret_cast<const __half2 *>(&raw);
      uint32_t lo = 0, hi = 0;
#pragma unroll
      for (int e2 = 0; e2 < 4; ++e2) {
        const float2 f = __half22float2(h[e2]);
        const uint32_t q0 = ((mb >> (2 * e2)) & 1u) ? 0u : code8(f.x, inv);
        const uint32_t q1 = ((mb >> (2 * e2 + 1)) & 1u) ? 0u : code8(f.y, inv);
        const uint32_t pair = q0 | (q1 << 8);
        if (e2 < 2) lo |= pair << (16 * e2);
        else hi |= pair << (16 * (e2 - 2));
      }
      qr[v] = make_uint2(lo, hi);
    }
    if (K_out_pad > 0) {
      const __half *xh = X + static_cast<size_t>(m) * ldx;
      __half *orow = X_out + static_cast<size_t>(m) * K_out_pad;
      for (int j = tid; j < K_out_pad; j += kQThreads) {
        __half v = __ushort_as_half(0);
        if (mixed && j < K_out) {
          const int c = s_idx[j];
          if (c >= 0) v = xh[c];
        }
        orow[j] = v;
      }
    }
  }

  // Publish this CTA's share of the matrix-wide outputs.
  __syncthreads();
  for (int w = tid; w < words; w += kQThreads) {
    const uint32_t d = s_det[w];
    if (d) atomicOr(&bitmap[w], d);
  }
  if (tid == 0 && mixed_rows) atomicAdd(reinterpret_cast<int *>(&flags[0]), mixed_rows);
  __threadfence();
  __syncthreads();
  if (tid == 0) {
    const int prev = atomicAdd(reinterpret_cast<int *>(&flags[2]), 1);
    s_last = prev == static_cast<int>(gridDim.x) - 1;
  }
  __syncthreads();
  if (!s_last) return;
  // Last CTA: every CTA's bitmap bits are in; count detections outside idx.
  __threadfence();
  int cnt = 0;
  for (int w = tid; w < words; w += kQThreads) cnt += __popc(__ldcg(&bitmap[w]) & ~s_mask[w]);
  cnt = warp_sum(cnt);
  if (lane == 0) s_cnt[warp] = cnt;
  __syncthreads();
  if (tid == 0) {
    int total = 0;
    for (int w = 0; w < kQWarps; ++w) total += s_cnt[w];
    flags[1] = total;
    flags[2] = 0;
  }
}

}  // namespace

cudaError_t launch_quantize_act(const void *X, int M, int K, int ldx, const int32_t *idx,
                                int K_out, float threshold, int8_t *Xq, float *s_x, void *X_out,
                                uint32_t *bitmap, int32_t *flags, int32_t *status,
                                cudaStream_t stream, int num_sms) {
  const int words = K / 32;
  reset_detect_kernel<<<1, 256, 0, stream>>>(bitmap, words, flags);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess || M == 0) return e;
  const size_t smem = sizeof(uint32_t) * 2 * words + sizeof(int32_t) * K_out;
  static bool configured = false;
  if (!configured) {
    e = cudaFuncSetAttribute(quantize_act_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             200 * 1024);
    if (e != cudaSuccess) return e;
    configured = true;
  }
  const int grid = M < num_sms * 8 ? M : num_sms * 8;
  quantize_act_kernel<<<grid, kQThreads, smem, stream>>>(
      static_cast<const __half *>(X), M, K, ldx, idx, K_out, k_out_pad(K_out), threshold, Xq,
      s_x, static_cast<__half *>(X_out), bitmap, flags, status);
  return cudaGetLastError();
}

}  // namespace mixq
