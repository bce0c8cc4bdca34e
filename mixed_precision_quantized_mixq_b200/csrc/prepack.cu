// Offline weight prepack for the MixQ layer.
//
// 8-bit (MixQ article "一键部署LLM混合精度推理…", 研究背景 Fig. 5): per output
// channel symmetric INT8, a = max |W[n,:]| over all K, code = clamp(rint(w *
// 127/a), -127, 127), s_w = a/127; outlier weight columns W[:, idx] gathered
// in idx order (Fig. 11).
//
// 4-bit (QServe W4A8KV4 reading notes, 渐进量化 + group-wise; MixLLM page,
// "MixLLM: Ein neuer Ansatz"): the INT8 codes are quantized again per group of
// 128 along K with an integer scale s2 and zero z2 chosen so that the
// effective weight (q - z2) * s2 always fits int8; the GEMM mainloop rebuilds
// it with one integer multiply-add per four codes.
//
// 4-bit reading B (MixLLM page, "MixLLM: Ein neuer Ansatz": asymmetric
// group-wise 4-bit weights dequantized in two steps onto INT8 tensor cores):
// no INT8 level; each row and group of 128 along K gets a real fp16 scale s and
// an integer zero z over a range widened to hold 0, q = clamp(rint(w/s) + z,
// 0, 15), so that q - z is an INT8 operand and s multiplies the group's INT32
// partial sum.  The codes share the 4-bit layout below; the group pairs hold
// (s, z) instead of (s2, z2).
//
// Both code layouts are reordered for the GEMM (QServe notes, "compute-aware
// weight reordering": the layout is chosen so the kernel's loads need no
// address arithmetic): the weights are cut into tiles of 128 output channels
// x 128 K, stored tile after tile (channel tile major, K tile minor), each
// tile one contiguous block that a single bulk copy moves into shared memory
// exactly as the tensor core (W8) or the expansion warps (W4) read it.
//   W8 tile (16 KB): row r at r*128; the 16-byte chunk holding K offsets
//     16j..16j+15 sits at chunk position j ^ (r & 7) (the 128-byte swizzle of
//     a K-major tcgen05 operand).
//   W4 tile (8 KB): row r at r*64; the 16-byte chunk c (K offsets 32c..32c+31)
//     sits at chunk position c ^ ((r >> 1) & 3) (conflict-free row reads);
//     inside a chunk, byte 4w+i holds the code of K offset 32c+8w+i in its low
//     nibble and that of 32c+8w+4+i in its high nibble, so a 32-bit word
//     splits into two words of four consecutive codes with one mask and one
//     shift.
#include <cuda_fp16.h>

#include "internal.h"
#include "ptx.cuh"

namespace mixq {
namespace {

constexpr int kPThreads = 256;
constexpr int kPWarps = kPThreads / 32;

// Byte offset of W8 code (n, k) in the tiled layout (k a multiple of 8 gives
// the start of 8 consecutive codes inside one 16-byte chunk).
__host__ __device__ __forceinline__ size_t w8_offset(int n, int k, int KB) {
  const size_t tile = static_cast<size_t>(n >> 7) * KB + (k >> 7);
  const int r = n & 127;
  return (tile * 128 + r) * 128 + ((((k & 127) >> 4) ^ (r & 7)) << 4) + (k & 15);
}

// Byte offset of 4-bit chunk c (K offsets 32c..32c+31 of K tile kb) of row n.
__host__ __device__ __forceinline__ size_t w4_chunk_offset(int n, int kb, int c, int KB) {
  const size_t tile = static_cast<size_t>(n >> 7) * KB + kb;
  const int r = n & 127;
  return (tile * 128 + r) * 64 + ((c ^ ((r >> 1) & 3)) << 4);
}

__device__ __forceinline__ float warp_max_f(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

__device__ __forceinline__ int warp_min_i(int v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = min(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

__device__ __forceinline__ int warp_max_i(int v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = max(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

template <bool kW4>
__global__ void __launch_bounds__(kPThreads) prepack_kernel(
    const __half *__restrict__ W, int N, int K, const int32_t *__restrict__ idx, int K_out,
    int K_out_pad, void *__restrict__ Wq, float *__restrict__ s_w, __half2 *__restrict__ grp,
    __half *__restrict__ W_out, int32_t *__restrict__ status) {
  extern __shared__ int8_t psm[];  // kW4: the row's INT8 codes, then its 4-bit codes
  __shared__ float s_red[kPWarps];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int nvec = K >> 3;
  for (int n = blockIdx.x; n < N; n += gridDim.x) {
    const uint4 *wr = reinterpret_cast<const uint4 *>(W + static_cast<size_t>(n) * K);
    float a = 0.f;
    for (int v = tid; v < nvec; v += kPThreads) {
      const uint4 raw = __ldg(wr + v);
      const __half2 *h = reinterpret_cast<const __half2 *>(&raw);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 f = __half22float2(h[e]);
        a = fmaxf(a, fmaxf(fabsf(f.x), fabsf(f.y)));
      }
    }
    a = warp_max_f(a);
    if (lane == 0) s_red[warp] = a;
    __syncthreads();
    a = s_red[0];
#pragma unroll
    for (int w = 1; w < kPWarps; ++w) a = fmaxf(a, s_red[w]);
    __syncthreads();
    const float inv = a > 0.f ? __fdiv_rn(127.f, a) : 0.f;
    if (tid == 0) s_w[n] = __fdiv_rn(a, 127.f);

    for (int v = tid; v < nvec; v += kPThreads) {
      const uint4 raw = __ldg(wr + v);
      const __half2 *h = reinterpret_cast<const __half2 *>(&raw);
      uint32_t word[2] = {0u, 0u};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 f = __half22float2(h[e]);
        int q0 = max(-127, min(127, __float2int_rn(__fmul_rn(f.x, inv))));
        int q1 = max(-127, min(127, __float2int_rn(__fmul_rn(f.y, inv))));
        const uint32_t pair = (static_cast<uint32_t>(q0) & 0xFFu) |
                              ((static_cast<uint32_t>(q1) & 0xFFu) << 8);
        word[e >> 1] |= pair << (16 * (e & 1));
      }
      if (kW4) {
        reinterpret_cast<uint2 *>(psm)[v] = make_uint2(word[0], word[1]);
      } else {
        *reinterpret_cast<uint2 *>(static_cast<int8_t *>(Wq) + w8_offset(n, v * 8, K / 128)) =
            make_uint2(word[0], word[1]);
      }
    }
    if (K_out_pad > 0) {
      const __half *wh = W + static_cast<size_t>(n) * K;
      for (int j = tid; j < K_out_pad; j += kPThreads) {
        __half v = __ushort_as_half(0);
        if (j < K_out) {
          const int c = idx[j];
          const bool ok = c >= 0 && c < K && (j == 0 || idx[j - 1] < c);
          if (ok) v = wh[c];
          else record_error(status, kErrInvalidArg);
        }
        W_out[static_cast<size_t>(n) * K_out_pad + j] = v;
      }
    }
    if (kW4) {
      __syncthreads();
      // Level 2: one warp per group of 128 codes, four codes per lane.
      const int groups = K / kGroup;
      for (int g = warp; g < groups; g += kPWarps) {
        int8_t *c = psm + g * kGroup + lane * 4;
        int v[4], lo = 127, hi = -127;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          v[i] = c[i];
          lo = min(lo, v[i]);
          hi = max(hi, v[i]);
        }
        lo = warp_min_i(lo);
        hi = warp_max_i(hi);
        const int s2 = max(1, (hi - lo + 14) / 15);
        const int z2 = max(0, min(15, __float2int_rn(__fdiv_rn(-static_cast<float>(lo),
                                                                static_cast<float>(s2)))));
        const int qlo = max(0, z2 - 128 / s2);
        const int qhi = min(15, z2 + 127 / s2);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int r = __float2int_rn(__fdiv_rn(static_cast<float>(v[i]), static_cast<float>(s2)));
          c[i] = static_cast<int8_t>(max(qlo, min(qhi, r + z2)));
        }
        if (lane == 0)
          grp[static_cast<size_t>(g) * N + n] =
              __halves2half2(__int2half_rn(s2), __int2half_rn(z2));
      }
      __syncthreads();
      // Pack: one 32-bit word (8 codes, k = 8wi .. 8wi+7) per thread and step.
      uint8_t *dst = static_cast<uint8_t *>(Wq);
      for (int wi = tid; wi < K / 8; wi += kPThreads) {
        const int8_t *src = psm + wi * 8;
        uint32_t word = 0;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const uint32_t byte = (static_cast<uint32_t>(src[i]) & 0xFu) |
                                ((static_cast<uint32_t>(src[i + 4]) & 0xFu) << 4);
          word |= byte << (8 * i);
        }
        const int kb = wi >> 4, c = (wi >> 2) & 3, w = wi & 3;
        *reinterpret_cast<uint32_t *>(dst + w4_chunk_offset(n, kb, c, K / 128) + 4 * w) = word;
      }
      __syncthreads();
    }
  }
}

__device__ __forceinline__ float warp_min_f(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fminf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// Reading-B prepack: one CTA per weight row (grid-stride), one warp per group
// of 128 K (four consecutive weights per lane), then the common 4-bit packing.
// Every decision is taken in fp32 with single IEEE operations in a fixed order:
//   lo = min(0, min w), hi = max(0, max w)
//   s  = fp16_rn(fp32(hi - lo) / 15)
//   z  = s > 0 ? clamp(rint(-lo / s), 0, 15) : 0
//   q  = s > 0 ? clamp(rint(w / s) + z, 0, 15) : 0
__global__ void __launch_bounds__(kPThreads) prepack_w4b_kernel(
    const __half *__restrict__ W, int N, int K, const int32_t *__restrict__ idx, int K_out,
    int K_out_pad, uint8_t *__restrict__ Wq, __half2 *__restrict__ grp,
    __half *__restrict__ W_out, int32_t *__restrict__ status) {
  extern __shared__ int8_t psm[];  // the row's 4-bit codes, one per byte
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int groups = K / kGroup;
  for (int n = blockIdx.x; n < N; n += gridDim.x) {
    const __half *wr = W + static_cast<size_t>(n) * K;
    for (int g = warp; g < groups; g += kPWarps) {
      const uint2 raw = __ldg(reinterpret_cast<const uint2 *>(wr + g * kGroup) + lane);
      const float2 f01 = __half22float2(*reinterpret_cast<const __half2 *>(&raw.x));
      const float2 f23 = __half22float2(*reinterpret_cast<const __half2 *>(&raw.y));
      const float v[4] = {f01.x, f01.y, f23.x, f23.y};
      float lo = fminf(fminf(v[0], v[1]), fminf(v[2], v[3]));
      float hi = fmaxf(fmaxf(v[0], v[1]), fmaxf(v[2], v[3]));
      lo = fminf(warp_min_f(lo), 0.f);
      hi = fmaxf(warp_max_f(hi), 0.f);
      float range = __fsub_rn(hi, lo);
      if (range <= 0.f) range = 0.f;  // +0 whatever the signs of zero min/max chose
      const __half s16 = __float2half_rn(__fdiv_rn(range, 15.f));
      const float s = __half2float(s16);
      const int z = s > 0.f ? max(0, min(15, __float2int_rn(__fdiv_rn(-lo, s)))) : 0;
      int8_t *c = psm + g * kGroup + lane * 4;
#pragma unroll
      for (int i = 0; i < 4; ++i)
        c[i] = static_cast<int8_t>(
            s > 0.f ? max(0, min(15, __float2int_rn(__fdiv_rn(v[i], s)) + z)) : 0);
      if (lane == 0) grp[static_cast<size_t>(g) * N + n] = __halves2half2(s16, __int2half_rn(z));
    }
    if (K_out_pad > 0) {
      for (int j = tid; j < K_out_pad; j += kPThreads) {
        __half v = __ushort_as_half(0);
        if (j < K_out) {
          const int c = idx[j];
          const bool ok = c >= 0 && c < K && (j == 0 || idx[j - 1] < c);
          if (ok) v = wr[c];
          else record_error(status, kErrInvalidArg);
        }
        W_out[static_cast<size_t>(n) * K_out_pad + j] = v;
      }
    }
    __syncthreads();
    for (int wi = tid; wi < K / 8; wi += kPThreads) {
      const int8_t *src = psm + wi * 8;
      uint32_t word = 0;
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const uint32_t byte = (static_cast<uint32_t>(src[i]) & 0xFu) |
                              ((static_cast<uint32_t>(src[i + 4]) & 0xFu) << 4);
        word |= byte << (8 * i);
      }
      const int kb = wi >> 4, c = (wi >> 2) & 3, w = wi & 3;
      *reinterpret_cast<uint32_t *>(Wq + w4_chunk_offset(n, kb, c, K / 128) + 4 * w) = word;
    }
    __syncthreads();
  }
}

__global__ void unpack_w4_kernel(int N, int K, const uint8_t *__restrict__ Wq4,
                                 const __half2 *__restrict__ grp, uint8_t *__restrict__ q,
                                 uint8_t *__restrict__ s2, uint8_t *__restrict__ z2) {
  const size_t total = static_cast<size_t>(N) * K;
  const int groups = K / kGroup;
  for (size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; i < total;
       i += static_cast<size_t>(gridDim.x) * blockDim.x) {
    const int n = static_cast<int>(i / K), k = static_cast<int>(i % K);
    const int g = k / kGroup, r = k % kGroup;
    const int c = r >> 5, w = (r >> 3) & 3, e = r & 7;
    const uint8_t byte = Wq4[w4_chunk_offset(n, g, c, groups) + 4 * w + (e & 3)];
    q[i] = (e & 4) ? (byte >> 4) : (byte & 0xF);
    if (r == 0) {
      const float2 sz = __half22float2(grp[static_cast<size_t>(g) * N + n]);
      s2[static_cast<size_t>(n) * groups + g] = static_cast<uint8_t>(sz.x);
      z2[static_cast<size_t>(n) * groups + g] = static_cast<uint8_t>(sz.y);
    }
  }
}

// Outlier weight columns alone, in idx order (MixQ Fig. 11), for an outlier
// set that changed after the prepack: W_out[n][j] = W[n][idx[j]] for j < K_out,
// +0.0 up to K_out_pad.  The INT8/4-bit codes do not depend on idx (the weight
// range covers every column), so only these columns are rebuilt.
__global__ void __launch_bounds__(256) extract_outlier_kernel(
    const __half *__restrict__ W, int N, int K, const int32_t *__restrict__ idx, int K_out,
    int K_out_pad, __half *__restrict__ W_out, int32_t *__restrict__ status) {
  for (int n = blockIdx.x; n < N; n += gridDim.x) {
    const __half *wh = W + static_cast<size_t>(n) * K;
    for (int j = threadIdx.x; j < K_out_pad; j += blockDim.x) {
      __half v = __ushort_as_half(0);
      if (j < K_out) {
        const int c = idx[j];
        const bool ok = c >= 0 && c < K && (j == 0 || idx[j - 1] < c);
        if (ok) v = wh[c];
        else record_error(status, kErrInvalidArg);
      }
      W_out[static_cast<size_t>(n) * K_out_pad + j] = v;
    }
  }
}

__global__ void unpack_w8_kernel(int N, int K, const int8_t *__restrict__ Wq,
                                 int8_t *__restrict__ out) {
  const size_t total = static_cast<size_t>(N) * K;
  for (size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; i < total;
       i += static_cast<size_t>(gridDim.x) * blockDim.x) {
    const int n = static_cast<int>(i / K), k = static_cast<int>(i % K);
    out[i] = Wq[w8_offset(n, k, K / 128)];
  }
}

}  // namespace

cudaError_t launch_prepack(int mode, const void *W, int N, int K, const int32_t *idx, int K_out,
                           void *Wq, float *s_w, void *grp, void *W_out, int32_t *status,
                           cudaStream_t stream) {
  if (N == 0) return cudaSuccess;
  const int grid = N < 4096 ? N : 4096;
  if (mode == 0) {
    prepack_kernel<false><<<grid, kPThreads, 0, stream>>>(
        static_cast<const __half *>(W), N, K, idx, K_out, k_out_pad(K_out), Wq, s_w, nullptr,
        static_cast<__half *>(W_out), status);
  } else if (mode == 2) {
    const size_t smem = static_cast<size_t>(K);
    cudaError_t e = cudaFuncSetAttribute(prepack_w4b_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem < 48 * 1024 ? 48 * 1024 : smem));
    if (e != cudaSuccess) return e;
    prepack_w4b_kernel<<<grid, kPThreads, smem, stream>>>(
        static_cast<const __half *>(W), N, K, idx, K_out, k_out_pad(K_out),
        static_cast<uint8_t *>(Wq), static_cast<__half2 *>(grp), static_cast<__half *>(W_out),
        status);
  } else {
    const size_t smem = static_cast<size_t>(K);
    cudaError_t e = cudaFuncSetAttribute(prepack_kernel<true>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem < 48 * 1024 ? 48 * 1024 : smem));
    if (e != cudaSuccess) return e;
    prepack_kernel<true><<<grid, kPThreads, smem, stream>>>(
        static_cast<const __half *>(W), N, K, idx, K_out, k_out_pad(K_out), Wq, s_w,
        static_cast<__half2 *>(grp), static_cast<__half *>(W_out), status);
  }
  return cudaGetLastError();
}

cudaError_t launch_extract_outliers(const void *W, int N, int K, const int32_t *idx, int K_out,
                                    void *W_out, int32_t *status, cudaStream_t stream) {
  const int kp = k_out_pad(K_out);
  if (N == 0 || kp == 0) return cudaSuccess;
  const int grid = N < 8192 ? N : 8192;
  extract_outlier_kernel<<<grid, 256, 0, stream>>>(static_cast<const __half *>(W), N, K, idx,
                                                   K_out, kp, static_cast<__half *>(W_out),
                                                   status);
  return cudaGetLastError();
}

cudaError_t launch_unpack_w4(int N, int K, const void *Wq4, const void *grp, uint8_t *q,
                             uint8_t *s2, uint8_t *z2, cudaStream_t stream) {
  if (N == 0) return cudaSuccess;
  unpack_w4_kernel<<<1024, 256, 0, stream>>>(N, K, static_cast<const uint8_t *>(Wq4),
                                             static_cast<const __half2 *>(grp), q, s2, z2);
  return cudaGetLastError();
}

}  // namespace mixq

namespace mixq {
cudaError_t launch_unpack_w8(int N, int K, const void *Wq, int8_t *out, cudaStream_t stream) {
  if (N == 0) return cudaSuccess;
  unpack_w8_kernel<<<1024, 256, 0, stream>>>(N, K, static_cast<const int8_t *>(Wq), out);
  return cudaGetLastError();
}
}  // namespace mixq
