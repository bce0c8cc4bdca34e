// Fused activation pass of the MixQ layer: per-token amax over outlier and
// non-outlier channels, the amax > threshold outlier test, the order-preserved
// gather of outlier channels into X_out, INT8 quantization of the rest, and a
// matrix-wide detection bitmap (MixQ article "一键部署LLM混合精度推理…",
// MixQ的解决方案: the amax of quantization doubles as the outlier test;
// Fig. 10 equivalent transformation; Fig. 11 order-preserved outlier matrix).
//
// HBM-bound: X is read once with 16-byte vector loads and kept in registers
// (VPT vectors per thread), Xq is written with 8-byte stores, the outlier
// channels of a mixed token are scattered straight from registers into X_out
// (a channel's column is its rank in the sorted outlier list, from a prefix
// count over the outlier bitset kept in shared memory).  A group of 256
// threads owns one token at a time; a CTA holds G such groups.
//
// Matrix-wide outputs (bitmap, flags):
//   - one thread-block cluster covers all tokens (decode-sized M): CTAs keep
//     their detection words and counts in shared memory and the cluster
//     combines them through distributed shared memory; plain stores, no
//     atomics and no reset pass;
//   - otherwise: a 1-block reset kernel zeroes bitmap/flags, CTAs OR/add into
//     them with atomics, and the last CTA to finish (ticket in flags[2])
//     counts the detections outside the outlier list.
// All kernels use programmatic dependent launch: they wait for the preceding
// grid before touching X, the outputs or the status word (the main pass reads
// the outlier list and builds its bitset before that wait).
#include <cuda_fp16.h>

#include <atomic>
#include <mutex>

#include "internal.h"
#include "ptx.cuh"

// Scratch of mixq_quantize_act_static, in the library's own device memory:
// word 0 is the ticket of the multi-CTA pass (whatever the shape, the pass
// needs no more); the rest of the 256 bytes is unused.  Every device that
// loads the library holds one copy until the process exits.
constexpr int kStaticScratchWords = 64;
static __device__ __align__(256) int32_t g_quantize_scratch[kStaticScratchWords];

namespace mixq {
namespace {

constexpr int kRowThreads = 256;  // threads per token group, bandwidth-bound shapes
constexpr int kMaxClusterCtas = 16;  // non-portable cluster size (opted in per kernel)

__global__ void reset_detect_kernel(uint32_t *__restrict__ bitmap, int words,
                                    int32_t *__restrict__ flags) {
  griddep_wait();
  for (int w = threadIdx.x; w < words; w += blockDim.x) bitmap[w] = 0u;
  if (threadIdx.x < 4) flags[threadIdx.x] = 0;
  __syncthreads();
  if (threadIdx.x == 0) griddep_launch_dependents();
}

// Reset pass of the variant whose CTA ticket lives in the library's static
// scratch (mixq_quantize_act_static): the two flag words and the ticket.
__global__ void reset_detect_static_kernel(uint32_t *__restrict__ bitmap, int words,
                                           int32_t *__restrict__ flags,
                                           int32_t *__restrict__ ticket) {
  griddep_wait();
  for (int w = threadIdx.x; w < words; w += blockDim.x) bitmap[w] = 0u;
  if (threadIdx.x < 2) flags[threadIdx.x] = 0;
  if (threadIdx.x == 0) *ticket = 0;
  __syncthreads();
  if (threadIdx.x == 0) griddep_launch_dependents();
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

__device__ __forceinline__ float warp_sum_f(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = __fadd_rn(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

__device__ __forceinline__ int warp_sum(int v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

__device__ __forceinline__ __half2 u32_as_half2(uint32_t w) {
  __half2 h;
  memcpy(&h, &w, sizeof h);
  return h;
}

// clamp(rint(x * inv), -127, 127): one IEEE fp32 multiply, round half to even.
__device__ __forceinline__ uint32_t code8(float x, float inv) {
  int q = __float2int_rn(__fmul_rn(x, inv));
  q = max(-127, min(127, q));
  return static_cast<uint32_t>(q) & 0xFFu;
}

struct QArgs {
  const __half *X;
  int M, K, ldx;
  const __half *gamma;  // RMS-normalisation gain [K] (NORM variants)
  float eps;
  __half *Xn;           // optional normalised tokens [M][ldxn] (NORM variants)
  int ldxn;
  const int32_t *idx;
  int K_out, K_out_pad;
  float T;
  int8_t *Xq;
  float *s_x;
  __half *X_out;
  uint32_t *bitmap;
  int32_t *flags;
  int32_t *status;
  int cluster_mode;  // one cluster covers the whole grid
  int32_t *ticket;   // STATIC_TICKET variants: the CTA ticket in the library's scratch
};

// RT threads per token group (256 for bandwidth-bound shapes; 512 or 1024
// for decode-sized M, where each group handles one token and the time is the
// latency of one token's pass), G groups per CTA, VPT 16-byte vectors per
// thread.  NORM: the token is first RMS-normalised in registers
// (x / sqrt(mean x^2 + eps) * gamma, rounded to fp16 as the normalisation's
// output would be), so the pass reads X once for both operations.
template <int VPT, int G, int RT, bool NORM, bool STATIC_TICKET = false>
__global__ void __launch_bounds__(RT *G) quantize_act_kernel(const QArgs a) {
  constexpr int kRowWarps = RT / 32;
  extern __shared__ uint32_t qsm[];
  const int words = a.K >> 5;  // K % 128 == 0
  uint32_t *s_mask = qsm;               // outlier channel bitset
  uint32_t *s_det = qsm + words;        // channels with |x| > T seen by this CTA
  uint32_t *s_rank = qsm + 2 * words;   // outlier channels in words before w
  // the group's X_out row of a mixed token, written out with 16-byte stores
  // (the padding columns stay zero: they are cleared once and never written)
  __half *s_xo = reinterpret_cast<__half *>(qsm + 3 * words) + (threadIdx.x / RT) * a.K_out_pad;
  __shared__ float s_red[G][2][kRowWarps];
  __shared__ int s_bad, s_last, s_part[2], s_cnt[G * kRowWarps];
  __shared__ uint32_t s_mixed_total;  // cluster mode: rank 0 accumulates every CTA's count
  // Lane masks of an 8-channel vector by its outlier bits b (bit e = channel
  // e is in idx): s_keep[b] word p keeps the magnitude bits (0x7FFF) of the
  // non-outlier halves of pair p, s_bkeep[b] keeps their code bytes.
  __shared__ uint4 s_keep[256];
  __shared__ uint2 s_bkeep[256];

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int g = tid / RT, gt = tid % RT, gw = gt >> 5;
  const int nvec = a.K >> 3;  // 8 fp16 per 16-byte vector
  const int row_stride = gridDim.x * G;

  // The outlier list does not come from the preceding kernel: its bitset and
  // rank prefix are built before waiting for that kernel, so under
  // programmatic dependent launch this part overlaps the preceding kernel.
  if (tid == 0) griddep_launch_dependents();
  int c_first = -1, c_prev = -1;
  if (tid < a.K_out) {
    c_first = a.idx[tid];
    c_prev = tid > 0 ? a.idx[tid - 1] : -1;
  }
  for (int w = tid; w < words; w += blockDim.x) {
    s_mask[w] = 0u;
    s_det[w] = 0u;
  }
  for (int j = tid % RT; j < a.K_out_pad; j += RT) s_xo[j] = __ushort_as_half(0);
  for (int b = tid; b < 256; b += blockDim.x) {
    uint32_t hk[4], bk[2] = {0u, 0u};
#pragma unroll
    for (int p = 0; p < 4; ++p)
      hk[p] = (((b >> (2 * p)) & 1) ? 0u : 0x7FFFu) | (((b >> (2 * p + 1)) & 1) ? 0u : 0x7FFF0000u);
#pragma unroll
    for (int e = 0; e < 8; ++e)
      if (!((b >> e) & 1)) bk[e >> 2] |= 0xFFu << (8 * (e & 3));
    s_keep[b] = make_uint4(hk[0], hk[1], hk[2], hk[3]);
    s_bkeep[b] = make_uint2(bk[0], bk[1]);
  }
  if (tid == 0) {
    s_bad = 0;
    s_mixed_total = 0u;
  }
  __syncthreads();
  // cluster mode: signal that this CTA's accumulators are initialised; the
  // matching wait comes before any CTA adds into rank 0's
  if (a.cluster_mode) cluster_arrive_relaxed();
  for (int j = tid; j < a.K_out; j += blockDim.x) {
    const int c = j == tid ? c_first : a.idx[j];
    const int cp = j == tid ? c_prev : a.idx[j - 1];
    const bool ok = c >= 0 && c < a.K && (j == 0 || cp < c);
    if (!ok) s_bad = 1;
    else atomicOr(&s_mask[c >> 5], 1u << (c & 31));
  }
  __syncthreads();
  if (warp == 0) {  // exclusive prefix count of outlier channels per bitset word
    const int per = (words + 31) / 32;
    const int w0 = lane * per;
    int local = 0;
    for (int w = w0; w < w0 + per && w < words; ++w) local += __popc(s_mask[w]);
    int incl = local;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int t = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += t;
    }
    int run = incl - local;
    for (int w = w0; w < w0 + per && w < words; ++w) {
      s_rank[w] = static_cast<uint32_t>(run);
      run += __popc(s_mask[w]);
    }
  }
  __syncthreads();
  const __half t_half = __float2half_rd(a.T);  // |x| > T  <=>  |x| > t_half for fp16 |x|
  griddep_wait();
  if (tid == 0 && s_bad) record_error(a.status, kErrInvalidArg);
  int m = blockIdx.x * G + g;
  uint4 v[VPT];
#pragma unroll
  for (int i = 0; i < VPT; ++i) {
    const int vi = gt + i * RT;
    v[i] = (m < a.M && vi < nvec)
               ? __ldg(reinterpret_cast<const uint4 *>(a.X + static_cast<size_t>(m) * a.ldx) + vi)
               : make_uint4(0u, 0u, 0u, 0u);
  }

  // The group's next token is loaded while this one is processed (when the
  // two rows fit in registers).  Only the 256-thread grid-stride shapes give
  // a group a second token; the wide decode shapes launch a group per token.
  constexpr bool kPrefetch = VPT <= 8 && G * RT == kRowThreads;
  constexpr int kVn = kPrefetch ? VPT : 1;
  auto load_row = [&](int row, uint4 *dst, int count) {
#pragma unroll
    for (int i = 0; i < count; ++i) {
      const int vi = gt + i * RT;
      dst[i] = (row < a.M && vi < nvec)
                   ? __ldg(reinterpret_cast<const uint4 *>(a.X + static_cast<size_t>(row) * a.ldx) +
                           vi)
                   : make_uint4(0u, 0u, 0u, 0u);
    }
  };
  int mixed_rows = 0;
  uint32_t det_acc[VPT];  // detection bits of the thread's vectors over its tokens
#pragma unroll
  for (int i = 0; i < VPT; ++i) det_acc[i] = 0u;
  for (; m < a.M; m += row_stride) {
    uint4 vn[kVn];
    if (kPrefetch) load_row(m + row_stride, vn, kVn);
    if (NORM) {
      // mean square of the token (fp32, sequential per thread, then a
      // shuffle tree, then the warps in order), one IEEE sqrt, and per
      // element one IEEE division and one multiply, rounded to fp16.  The
      // gain vectors are loaded here (cached after the first token) so their
      // latency overlaps the reduction, without holding registers across tokens.
      uint4 gv[VPT];
#pragma unroll
      for (int i = 0; i < VPT; ++i) {
        const int vi = gt + i * RT;
        gv[i] = vi < nvec ? __ldg(reinterpret_cast<const uint4 *>(a.gamma) + vi)
                          : make_uint4(0u, 0u, 0u, 0u);
      }
      float ss = 0.f;
#pragma unroll
      for (int i = 0; i < VPT; ++i) {
        const __half2 *h = reinterpret_cast<const __half2 *>(&v[i]);
#pragma unroll
        for (int e2 = 0; e2 < 4; ++e2) {
          const float2 f = __half22float2(h[e2]);
          ss = __fadd_rn(ss, __fmul_rn(f.x, f.x));
          ss = __fadd_rn(ss, __fmul_rn(f.y, f.y));
        }
      }
      ss = warp_sum_f(ss);
      if (lane == 0) s_red[g][0][gw] = ss;
      named_barrier(1 + g, RT);
      float tot = 0.f;
#pragma unroll
      for (int w = 0; w < kRowWarps; ++w) tot = __fadd_rn(tot, s_red[g][0][w]);
      named_barrier(1 + g, RT);  // s_red is rewritten by the amax below
      const float den = __fsqrt_rn(__fadd_rn(__fdiv_rn(tot, static_cast<float>(a.K)), a.eps));
      __half *xn_row = a.Xn ? a.Xn + static_cast<size_t>(m) * a.ldxn : nullptr;
#pragma unroll
      for (int i = 0; i < VPT; ++i) {
        const int vi = gt + i * RT;
        __half2 *h = reinterpret_cast<__half2 *>(&v[i]);
        const __half2 *gh = reinterpret_cast<const __half2 *>(&gv[i]);
#pragma unroll
        for (int e2 = 0; e2 < 4; ++e2) {
          const float2 f = __half22float2(h[e2]);
          const float2 gf = __half22float2(gh[e2]);
          const float y0 = den > 0.f ? __fmul_rn(__fdiv_rn(f.x, den), gf.x) : 0.f;
          const float y1 = den > 0.f ? __fmul_rn(__fdiv_rn(f.y, den), gf.y) : 0.f;
          h[e2] = __floats2half2_rn(y0, y1);
        }
        if (xn_row && vi < nvec) reinterpret_cast<uint4 *>(xn_row)[vi] = v[i];
      }
    }
    // |x| over all channels and over the non-outlier ones, in fp16 (abs and
    // max are exact there, and max skips NaN like fmaxf), two lanes at a time;
    // the detection bits only for vectors whose largest |x| is above T
    // (|x| > T for an fp16 |x| exactly when |x| > T rounded down to fp16)
    __half2 mA = __float2half2_rn(0.f), mN = mA;
#pragma unroll
    for (int i = 0; i < VPT; ++i) {
      const int vi = gt + i * RT;
      const int k0 = vi << 3;
      const uint32_t mb = vi < nvec ? (s_mask[k0 >> 5] >> (k0 & 31)) & 0xFFu : 0u;
      const uint4 kp = s_keep[mb];
      const uint32_t hw[4] = {v[i].x, v[i].y, v[i].z, v[i].w};
      const uint32_t kw[4] = {kp.x, kp.y, kp.z, kp.w};
      __half2 vm = __float2half2_rn(0.f);
#pragma unroll
      for (int e2 = 0; e2 < 4; ++e2) {
        vm = __hmax2(vm, u32_as_half2(hw[e2] & 0x7FFF7FFFu));
        mN = __hmax2(mN, u32_as_half2(hw[e2] & kw[e2]));
      }
      mA = __hmax2(mA, vm);
      if (__hgt(__hmax(__low2half(vm), __high2half(vm)), t_half)) {
        uint32_t det = 0;
#pragma unroll
        for (int e2 = 0; e2 < 4; ++e2) {
          const __half2 ab = u32_as_half2(hw[e2] & 0x7FFF7FFFu);
          det |= (__hgt(__low2half(ab), t_half) ? 1u : 0u) << (2 * e2);
          det |= (__hgt(__high2half(ab), t_half) ? 1u : 0u) << (2 * e2 + 1);
        }
        det_acc[i] |= det;
      }
    }
    float aA = fmaxf(__low2float(mA), __high2float(mA));
    float aN = fmaxf(__low2float(mN), __high2float(mN));
    aA = warp_max(aA);
    aN = warp_max(aN);
    if (lane == 0) {
      s_red[g][0][gw] = aA;
      s_red[g][1][gw] = aN;
    }
    named_barrier(1 + g, RT);
    float rA = s_red[g][0][0], rN = s_red[g][1][0];
#pragma unroll
    for (int w = 1; w < kRowWarps; ++w) {
      rA = fmaxf(rA, s_red[g][0][w]);
      rN = fmaxf(rN, s_red[g][1][w]);
    }
    named_barrier(1 + g, RT);  // s_red is rewritten by the group's next token

    const float amax = rA;
    const bool mixed = a.K_out > 0 && amax > a.T;
    const float am = mixed ? rN : amax;
    const float inv = am > 0.f ? __fdiv_rn(127.f, am) : 0.f;
    if (gt == 0) {
      a.s_x[m] = __fdiv_rn(am, 127.f);
      mixed_rows += mixed ? 1 : 0;
    }

    uint2 *qr = reinterpret_cast<uint2 *>(a.Xq + static_cast<size_t>(m) * a.K);
    __half *orow = a.X_out + static_cast<size_t>(m) * a.K_out_pad;
#pragma unroll
    for (int i = 0; i < VPT; ++i) {
      const int vi = gt + i * RT;
      if (vi >= nvec) continue;
      const int k0 = vi << 3;
      const uint32_t word = s_mask[k0 >> 5];
      const uint32_t mb = mixed ? (word >> (k0 & 31)) & 0xFFu : 0u;
      const __half2 *h = reinterpret_cast<const __half2 *>(&v[i]);
      uint32_t q[8];
#pragma unroll
      for (int e2 = 0; e2 < 4; ++e2) {
        const float2 f = __half22float2(h[e2]);
        q[2 * e2] = code8(f.x, inv);
        q[2 * e2 + 1] = code8(f.y, inv);
      }
      // low bytes packed in channel order; the outlier channels of a mixed
      // token are zero
      const uint2 bk = s_bkeep[mb];
      const uint32_t lo =
          __byte_perm(__byte_perm(q[0], q[1], 0x0040u), __byte_perm(q[2], q[3], 0x0040u), 0x5410u) &
          bk.x;
      const uint32_t hi =
          __byte_perm(__byte_perm(q[4], q[5], 0x0040u), __byte_perm(q[6], q[7], 0x0040u), 0x5410u) &
          bk.y;
      qr[vi] = make_uint2(lo, hi);
      if (mb) {  // outlier channels of a mixed token -> their X_out columns
        const int base = static_cast<int>(s_rank[k0 >> 5]) +
                         __popc(word & ((1u << (k0 & 31)) - 1u));
        const unsigned short *hs = reinterpret_cast<const unsigned short *>(&v[i]);
        int j = base;
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          if ((mb >> e) & 1u) {
            s_xo[j] = __ushort_as_half(hs[e]);
            ++j;
          }
        }
      }
    }
    // the token's X_out row: its outlier channels (mixed) or zeros
    if (mixed) named_barrier(1 + g, RT);  // the group's columns are in s_xo
    for (int j = gt; j < a.K_out_pad / 8; j += RT)
      reinterpret_cast<uint4 *>(orow)[j] =
          mixed ? reinterpret_cast<const uint4 *>(s_xo)[j] : make_uint4(0u, 0u, 0u, 0u);
    if (kPrefetch) {
#pragma unroll
      for (int i = 0; i < kVn; ++i) v[i] = vn[i];
    } else {
      load_row(m + row_stride, v, VPT);
    }
  }

  // ------------------------------------------- matrix-wide bitmap and flags
#pragma unroll
  for (int i = 0; i < VPT; ++i) {
    const int k0 = (gt + i * RT) << 3;
    if (det_acc[i]) atomicOr(&s_det[k0 >> 5], det_acc[i] << (k0 & 31));
  }
  if (lane == 0) s_cnt[warp] = 0;
  __syncwarp();
  if (gt == 0) s_cnt[warp] = mixed_rows;
  __syncthreads();
  if (tid == 0) {
    int t = 0;
    for (int w = 0; w < G * kRowWarps; ++w) t += s_cnt[w];
    s_part[1] = t;  // mixed tokens seen by this CTA
  }
  __syncthreads();

  if (a.cluster_mode) {
    // Every CTA ORs its detection words and adds its mixed-token count into
    // CTA rank 0's shared memory; after one cluster barrier rank 0 owns the
    // matrix-wide result and no CTA reads another's memory again.
    const uint32_t rank = cluster_ctarank();
    cluster_wait();  // rank 0's accumulators are initialised
    if (rank != 0) {
      for (int w = tid; w < words; w += blockDim.x) {
        const uint32_t d = s_det[w];
        if (d) red_or_dsmem(mapa_shared(smem_u32(&s_det[w]), 0u), d);
      }
    }
    if (tid == 0)
      red_add_dsmem(mapa_shared(smem_u32(&s_mixed_total), 0u), static_cast<uint32_t>(s_part[1]));
    cluster_sync_all();  // every CTA's contributions have landed in rank 0
    if (rank != 0) return;
    int outside = 0;
    for (int w = tid; w < words; w += blockDim.x) {
      const uint32_t bits = s_det[w];
      a.bitmap[w] = bits;
      outside += __popc(bits & ~s_mask[w]);
    }
    outside = warp_sum(outside);
    if (lane == 0) s_cnt[warp] = outside;
    __syncthreads();
    if (tid == 0) {
      int t = 0;
      for (int w = 0; w < G * kRowWarps; ++w) t += s_cnt[w];
      a.flags[0] = static_cast<int32_t>(s_mixed_total);
      a.flags[1] = t;
      if (!STATIC_TICKET) {
        a.flags[2] = 0;
        a.flags[3] = 0;
      }
    }
    return;
  }

  for (int w = tid; w < words; w += blockDim.x) {
    const uint32_t d = s_det[w];
    if (d) atomicOr(&a.bitmap[w], d);
  }
  if (tid == 0 && s_part[1]) atomicAdd(reinterpret_cast<int *>(&a.flags[0]), s_part[1]);
  __threadfence();
  __syncthreads();
  int32_t *const ticket = STATIC_TICKET ? a.ticket : &a.flags[2];
  if (tid == 0) {
    const int prev = atomicAdd(reinterpret_cast<int *>(ticket), 1);
    s_last = prev == static_cast<int>(gridDim.x) - 1;
  }
  __syncthreads();
  if (!s_last) return;
  // Last CTA: every CTA's bitmap bits are in; count detections outside idx.
  __threadfence();
  int cnt = 0;
  for (int w = tid; w < words; w += blockDim.x) cnt += __popc(__ldcg(&a.bitmap[w]) & ~s_mask[w]);
  cnt = warp_sum(cnt);
  if (lane == 0) s_cnt[warp] = cnt;
  __syncthreads();
  if (tid == 0) {
    int total = 0;
    for (int w = 0; w < G * kRowWarps; ++w) total += s_cnt[w];
    a.flags[1] = total;
    *ticket = 0;
  }
}

template <int VPT, int G, int RT, bool STATIC_TICKET = false>
cudaError_t launch_variant(const QArgs &a, int grid, int cluster, cudaStream_t stream) {
  void (*kernel)(const QArgs);
  if constexpr (STATIC_TICKET)
    kernel = quantize_act_kernel<VPT, G, RT, false, true>;
  else
    kernel = a.gamma ? quantize_act_kernel<VPT, G, RT, true> : quantize_act_kernel<VPT, G, RT, false>;
  // outlier bitset, detection words, rank prefix; one X_out row per group
  const size_t smem = sizeof(uint32_t) * 3 * (a.K / 32) + sizeof(__half) * G * a.K_out_pad;
  cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem < 48 * 1024 ? 48 * 1024 : smem));
  if (e == cudaSuccess && cluster > 8)
    e = cudaFuncSetAttribute(kernel, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(grid, 1, 1);
  cfg.blockDim = dim3(RT * G, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  attr[1].id = cudaLaunchAttributeClusterDimension;
  attr[1].val.clusterDim.x = cluster;
  attr[1].val.clusterDim.y = 1;
  attr[1].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  return cudaLaunchKernelEx(&cfg, kernel, a);
}

// Device address of g_quantize_scratch on the current device, looked up once
// per device (the host-side name is only a stand-in for the device symbol).
cudaError_t static_scratch(int32_t **out) {
  static std::atomic<int32_t *> ptr[64];
  static std::mutex mu;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  int32_t *p = ptr[dev].load(std::memory_order_acquire);
  if (!p) {
    std::lock_guard<std::mutex> lock(mu);
    p = ptr[dev].load(std::memory_order_acquire);
    if (!p) {
      void *q = nullptr;
      e = cudaGetSymbolAddress(&q, g_quantize_scratch);
      if (e != cudaSuccess) return e;
      p = static_cast<int32_t *>(q);
      ptr[dev].store(p, std::memory_order_release);
    }
  }
  *out = p;
  return cudaSuccess;
}

}  // namespace

int quantize_max_k() { return 16 * kRowThreads * 8; }

cudaError_t launch_quantize_act_static(const void *X, int M, int K, int ldx, const int32_t *idx,
                                       int K_out, float threshold, int8_t *Xq, float *s_x,
                                       void *X_out, uint32_t *bitmap, int32_t *flags,
                                       int32_t *status, cudaStream_t stream, int num_sms) {
  int32_t *ticket = nullptr;
  cudaError_t e = static_scratch(&ticket);
  if (e != cudaSuccess) return e;
  QArgs a{};
  a.X = static_cast<const __half *>(X);
  a.M = M;
  a.K = K;
  a.ldx = ldx;
  a.idx = idx;
  a.K_out = K_out;
  a.K_out_pad = k_out_pad(K_out);
  a.T = threshold;
  a.Xq = Xq;
  a.s_x = s_x;
  a.X_out = static_cast<__half *>(X_out);
  a.bitmap = bitmap;
  a.flags = flags;
  a.status = status;
  a.ticket = ticket;
  const int nvec = K / 8;
  // the launch shapes of mixq_quantize_act, with the ticket in the scratch
  if (M > 0 && M <= 64) {
    if (nvec <= 512 && (M + 1) / 2 <= kMaxClusterCtas) {
      a.cluster_mode = 1;
      return launch_variant<1, 2, 512, true>(a, (M + 1) / 2, (M + 1) / 2, stream);
    }
    if (nvec <= 512 && (M + 3) / 4 <= kMaxClusterCtas) {
      a.cluster_mode = 1;
      return launch_variant<2, 4, 256, true>(a, (M + 3) / 4, (M + 3) / 4, stream);
    }
    if (nvec > 512 && nvec <= 2048 && M <= kMaxClusterCtas) {
      a.cluster_mode = 1;
      return launch_variant<2, 1, 1024, true>(a, M, M, stream);
    }
    if (nvec > 512 && nvec <= 1536 && (M + 1) / 2 <= kMaxClusterCtas) {
      a.cluster_mode = 1;
      return launch_variant<3, 2, 512, true>(a, (M + 1) / 2, (M + 1) / 2, stream);
    }
  }
  const int vpt_need = (nvec + kRowThreads - 1) / kRowThreads;
  const int vpt = vpt_need <= 1 ? 1 : vpt_need <= 2 ? 2 : vpt_need <= 4 ? 4 : vpt_need <= 8 ? 8 : 16;
  {
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3(1, 1, 1);
    cfg.blockDim = dim3(256, 1, 1);
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, reset_detect_static_kernel, bitmap, K / 32, flags, ticket);
    if (e != cudaSuccess || M == 0) return e;
  }
  a.cluster_mode = 0;
  if (M <= 64 && nvec <= 512) return launch_variant<1, 2, 512, true>(a, (M + 1) / 2, 1, stream);
  if (M <= 64 && nvec <= 2048) return launch_variant<2, 1, 1024, true>(a, M, 1, stream);
  const int grid = M < num_sms * 8 ? M : num_sms * 8;
  switch (vpt) {
    case 1: return launch_variant<1, 1, kRowThreads, true>(a, grid, 1, stream);
    case 2: return launch_variant<2, 1, kRowThreads, true>(a, grid, 1, stream);
    case 4: return launch_variant<4, 1, kRowThreads, true>(a, grid, 1, stream);
    case 8: return launch_variant<8, 1, kRowThreads, true>(a, grid, 1, stream);
    default: return launch_variant<16, 1, kRowThreads, true>(a, grid, 1, stream);
  }
}

cudaError_t launch_quantize_act(const void *X, int M, int K, int ldx, const int32_t *idx,
                                int K_out, float threshold, int8_t *Xq, float *s_x, void *X_out,
                                uint32_t *bitmap, int32_t *flags, int32_t *status,
                                cudaStream_t stream, int num_sms, const void *gamma, float eps,
                                void *Xn, int ldxn) {
  QArgs a{};
  a.X = static_cast<const __half *>(X);
  a.M = M;
  a.K = K;
  a.ldx = ldx;
  a.gamma = static_cast<const __half *>(gamma);
  a.eps = eps;
  a.Xn = static_cast<__half *>(Xn);
  a.ldxn = ldxn;
  a.idx = idx;
  a.K_out = K_out;
  a.K_out_pad = k_out_pad(K_out);
  a.T = threshold;
  a.Xq = Xq;
  a.s_x = s_x;
  a.X_out = static_cast<__half *>(X_out);
  a.bitmap = bitmap;
  a.flags = flags;
  a.status = status;
  const int nvec = K / 8;
  if (M > 0 && M <= 64) {
    // Decode-sized M: one token per group and wide groups (the kernel's time
    // is one token's latency chain, measured: a second token per group adds
    // 2-4 us), all groups in one cluster when that takes at most 16 CTAs (no
    // reset pass, no atomics).
    // K <= 4096: 2 x 512 threads per CTA up to 32 tokens, 4 x 256 up to 64
    if (nvec <= 512 && (M + 1) / 2 <= kMaxClusterCtas) {
      a.cluster_mode = 1;
      return launch_variant<1, 2, 512>(a, (M + 1) / 2, (M + 1) / 2, stream);
    }
    if (nvec <= 512 && (M + 3) / 4 <= kMaxClusterCtas) {
      a.cluster_mode = 1;
      return launch_variant<2, 4, 256>(a, (M + 3) / 4, (M + 3) / 4, stream);
    }
    // K <= 16384: 1024 threads per token up to 16 tokens; K <= 12288: 2 x 512
    // up to 32 (with four 256-thread tokens per CTA, 16 CTAs streaming 64
    // tokens of K = 11008 measured slower than 64 CTAs and the reset pass)
    if (nvec > 512 && nvec <= 2048 && M <= kMaxClusterCtas) {
      a.cluster_mode = 1;
      return launch_variant<2, 1, 1024>(a, M, M, stream);
    }
    if (nvec > 512 && nvec <= 1536 && (M + 1) / 2 <= kMaxClusterCtas) {
      a.cluster_mode = 1;
      return launch_variant<3, 2, 512>(a, (M + 1) / 2, (M + 1) / 2, stream);
    }
  }
  // Otherwise one token per 256-thread CTA at a time (grid-stride over tokens)
  // and VPT vectors per thread.
  const int vpt_need = (nvec + kRowThreads - 1) / kRowThreads;
  const int vpt = vpt_need <= 1 ? 1 : vpt_need <= 2 ? 2 : vpt_need <= 4 ? 4 : vpt_need <= 8 ? 8 : 16;
  // Reset pass (waits for the preceding grid itself), then the main pass.
  {
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3(1, 1, 1);
    cfg.blockDim = dim3(256, 1, 1);
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cudaError_t e = cudaLaunchKernelEx(&cfg, reset_detect_kernel, bitmap, K / 32, flags);
    if (e != cudaSuccess || M == 0) return e;
  }
  a.cluster_mode = 0;
  if (M <= 64 && nvec <= 512) return launch_variant<1, 2, 512>(a, (M + 1) / 2, 1, stream);
  if (M <= 64 && nvec <= 2048) return launch_variant<2, 1, 1024>(a, M, 1, stream);
  const int grid = M < num_sms * 8 ? M : num_sms * 8;
  switch (vpt) {
    case 1: return launch_variant<1, 1, kRowThreads>(a, grid, 1, stream);
    case 2: return launch_variant<2, 1, kRowThreads>(a, grid, 1, stream);
    case 4: return launch_variant<4, 1, kRowThreads>(a, grid, 1, stream);
    case 8: return launch_variant<8, 1, kRowThreads>(a, grid, 1, stream);
    default: return launch_variant<16, 1, kRowThreads>(a, grid, 1, stream);
  }
}

}  // namespace mixq
