// Mixed-precision GEMM of the MixQ layer on sm_100a tensor cores.
//
//   acc[m,n] = sum_k Xq[m,k] Wq[n,k]          tcgen05.mma kind::i8  -> INT32 in TMEM
//   o[m,n]   = sum_j X_out[m,j] W_out[n,j]    tcgen05.mma kind::f16 -> FP32 in TMEM
//   Y[m,n]   = fp16((float(acc) * s_x[m]) * s_w[n] + o)     epilogue in registers
//
// (MixQ article "一键部署LLM混合精度推理…": 研究背景 Fig. 5 two products summed;
// MixQ的解决方案 Fig. 12 dequantize/scale/add of the low-precision result in
// registers.)  The W4 variant rebuilds INT8 weights from 4-bit group codes
// inside the mainloop (QServe reading notes, 渐进量化 / 寄存器压力和并行性:
// weight dequantization in the mainloop, four codes per register operation,
// no intermediate overflows; MixLLM page: two-stage dequantization onto INT8
// tensor cores).
//
// One CTA computes one 128 x BN output tile over a K range:
//   warp 0 lane 0   TMA producer: A (Xq or X_out) and B (Wq, W_out, or packed
//                   4-bit codes + group constants) tiles into a ring of
//                   shared-memory stages (128-byte swizzle, K-major)
//   warp 1 lane 0   MMA issuer: 4 tcgen05.mma per stage (32 bytes of K each),
//                   tcgen05.commit frees the stage
//   warps 4..7      (W4 only) expansion: packed codes -> INT8 operand tile
//   warps 0..3      epilogue: tcgen05.ld of the accumulators, scale, add, store
// When K is split over a thread-block cluster (decode-sized M), each CTA of
// the cluster owns a K range, writes its INT32 partial tile to its own shared
// memory, and the cluster reduces through distributed shared memory (integer
// sums, so the split is exact and order-free); CTA rank 0 also runs the FP16
// outlier slice.  No global workspace, no atomics.
//
// Every wait on an mbarrier is bounded in wall time; a wait that runs out
// records MIXQ_ERR_TIMEOUT in *status and the CTA winds down without hanging.
#include <cuda_fp16.h>

#include <atomic>
#include <mutex>

#include "internal.h"
#include "ptx.cuh"

namespace mixq {
namespace {

template <int BN, bool W4>
struct Cfg {
  static constexpr int kA = kTileM * kBlockK;             // A stage: 128 rows x 128 B
  static constexpr int kB = BN * kBlockK;                 // B stage: BN rows x 128 B
  static constexpr int kP = W4 ? BN * (kBlockK / 2) : 0;  // packed 4-bit codes
  static constexpr int kG = W4 ? ((BN * 4 + 1023) / 1024) * 1024 : 0;  // (s2,z2) per row
  static constexpr int kStage = kA + kB + kP + kG;
  static constexpr int kStages = W4 ? (BN == 256 ? 3 : 5) : (BN == 256 ? 4 : 6);
  static constexpr int kThreads = W4 ? 256 : 128;
  static constexpr int kTmemCols = 2 * BN;  // INT32 acc [0,BN), FP32 outlier acc [BN,2BN)
  static constexpr int kBarBytes = 1024;
  static constexpr int kSmem = kStages * kStage + kBarBytes + 1024;  // + alignment slack
  // cluster reduction buffers (reuse the stage ring after the mainloop)
  static constexpr int kCW = 128;
  static constexpr int kPitch = kCW + 4;  // words; +4 keeps 16-byte rows off one bank group
  static_assert(2 * kTileM * kPitch * 4 <= kStages * kStage, "reduction buffers do not fit");
  static_assert(kSmem <= 232448, "shared memory budget");
};

struct KParams {
  int M, N, K, K_out_pad;
  const float *s_x;
  const float *s_w;
  const int32_t *flags;
  void *Y;
  int ldy;
  int32_t *status;
  uint64_t wait_limit_ns;
  int debug_stall;
  int b_streamed;  // B tiles are read by one CTA only: evict them from L2 first
};

__device__ __forceinline__ void fail(int *s_err, int32_t *status) {
  atomicOr(s_err, 1);
  record_error(status, kErrTimeout);
}

// 4 codes (one byte each, low nibbles of w) -> 4 signed INT8 weights:
// byte = (q*s2 + 128 - z2*s2) ^ 0x80 == (q - z2)*s2 as two's complement.
// Each byte's value q*s2 + 128 - z2*s2 = (q - z2)*s2 + 128 lies in [0, 255], so
// the 32-bit multiply-add never carries or borrows between bytes.
__device__ __forceinline__ uint32_t expand4(uint32_t nibbles, uint32_t s2, uint32_t c) {
  return (nibbles * s2 + c) ^ 0x80808080u;
}

template <int BN, bool W4, bool RAW>
__global__ void __launch_bounds__(Cfg<BN, W4>::kThreads, 1)
    mixq_gemm_kernel(const __grid_constant__ CUtensorMap tm_a,   // Xq   [M][K] int8
                     const __grid_constant__ CUtensorMap tm_b,   // Wq [N][K] int8 | Wq4 [N][K/2]
                     const __grid_constant__ CUtensorMap tm_g,   // grp [K/128][N] (s2,z2)
                     const __grid_constant__ CUtensorMap tm_xo,  // X_out [M][K_out_pad] fp16
                     const __grid_constant__ CUtensorMap tm_wo,  // W_out [N][K_out_pad] fp16
                     const KParams p) {
  using C = Cfg<BN, W4>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t *ring = smem;
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + C::kStages * C::kStage);
  uint64_t *full = bars;
  uint64_t *empty = bars + C::kStages;
  uint64_t *ready = bars + 2 * C::kStages;
  uint64_t *accum_full = bars + 3 * C::kStages;
  uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(accum_full + 1);
  int *s_misc = reinterpret_cast<int *>(tmem_holder + 1);  // err, any_out, consumed, issued

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int m0 = blockIdx.x * kTileM;
  const int n0 = blockIdx.y * BN;
  const int S = gridDim.z;
  const int rank = blockIdx.z;
  const int KB = p.K / kBlockK;
  const int kb_begin = static_cast<int>(static_cast<long long>(rank) * KB / S);
  const int kb_end = static_cast<int>(static_cast<long long>(rank + 1) * KB / S);

  if (threadIdx.x == 0) {
    for (int i = 0; i < C::kStages; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
      if (W4) mbar_init(&ready[i], 128);
    }
    mbar_init(accum_full, 1);
    fence_mbar_init();
    int any_out = 0;
    if (!RAW && p.K_out_pad > 0) any_out = p.flags ? (p.flags[0] > 0) : 1;
    s_misc[0] = 0;
    s_misc[1] = any_out;
    s_misc[2] = 0;
    s_misc[3] = 0;
    tma_prefetch_desc(&tm_a);
    tma_prefetch_desc(&tm_b);
    if (W4) tma_prefetch_desc(&tm_g);
    if (any_out && rank == 0) {
      tma_prefetch_desc(&tm_xo);
      tma_prefetch_desc(&tm_wo);
    }
  }
  if (warp == 1) {
    tmem_alloc(tmem_holder, C::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;
  const int any_out = s_misc[1];
  const bool do_out = any_out && rank == 0;
  const int n_out = do_out ? p.K_out_pad / kOutBlockK : 0;
  const int njobs = n_out + (kb_end - kb_begin);
  int *s_err = &s_misc[0];

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0 && !p.debug_stall) {
      const uint64_t pol_a = policy_evict_last();
      const uint64_t pol_b = p.b_streamed ? policy_evict_first() : policy_evict_last();
      int issued = 0;
      for (int j = 0; j < njobs; ++j) {
        const int s = j % C::kStages;
        const uint32_t ph = (j / C::kStages) & 1;
        if (!mbar_wait(&empty[s], ph ^ 1, p.wait_limit_ns)) {
          fail(s_err, p.status);
          break;
        }
        uint8_t *sA = ring + s * C::kStage;
        uint8_t *sB = sA + C::kA;
        uint8_t *sP = sB + C::kB;
        uint8_t *sG = sP + C::kP;
        if (j < n_out) {
          mbar_arrive_expect_tx(&full[s], C::kA + C::kB);
          tma_load_2d(sA, &tm_xo, &full[s], j * kOutBlockK, m0, pol_a);
          tma_load_2d(sB, &tm_wo, &full[s], j * kOutBlockK, n0, pol_b);
        } else {
          const int kb = kb_begin + (j - n_out);
          if (!W4) {
            mbar_arrive_expect_tx(&full[s], C::kA + C::kB);
            tma_load_2d(sA, &tm_a, &full[s], kb * kBlockK, m0, pol_a);
            tma_load_2d(sB, &tm_b, &full[s], kb * kBlockK, n0, pol_b);
          } else {
            mbar_arrive_expect_tx(&full[s], C::kA + C::kP + BN * 4);
            tma_load_2d(sA, &tm_a, &full[s], kb * kBlockK, m0, pol_a);
            tma_load_2d(sP, &tm_b, &full[s], kb * (kBlockK / 2), n0, pol_b);
            tma_load_2d(sG, &tm_g, &full[s], n0, kb, pol_b);
          }
        }
        issued = j + 1;
      }
      s_misc[3] = issued;
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t kIdI8 = idesc_s8_s32(kTileM, BN);
      constexpr uint32_t kIdF16 = idesc_f16_f32(kTileM, BN);
      const uint32_t t_i32 = tmem_base;
      const uint32_t t_f32 = tmem_base + BN;
      int consumed = 0;
      for (int j = 0; j < njobs; ++j) {
        const int s = j % C::kStages;
        const uint32_t ph = (j / C::kStages) & 1;
        if (!mbar_wait(W4 ? &ready[s] : &full[s], ph, p.wait_limit_ns)) {
          fail(s_err, p.status);
          break;
        }
        tc_fence_after();
        const uint32_t a_addr = smem_u32(ring + s * C::kStage);
        const uint64_t ad = sw128_kmajor_desc(a_addr);
        const uint64_t bd = sw128_kmajor_desc(a_addr + C::kA);
        if (j < n_out) {
#pragma unroll
          for (int k = 0; k < 4; ++k)
            mma_f16(t_f32, ad + 2 * k, bd + 2 * k, kIdF16, (j > 0 || k > 0) ? 1u : 0u);
        } else {
#pragma unroll
          for (int k = 0; k < 4; ++k)
            mma_i8(t_i32, ad + 2 * k, bd + 2 * k, kIdI8, (j > n_out || k > 0) ? 1u : 0u);
        }
        mma_commit(&empty[s]);
        consumed = j + 1;
      }
      mma_commit(accum_full);
      s_misc[2] = consumed;
    }
  } else if (W4 && warp >= 4) {
    // ------------------------------------------- 4-bit -> INT8 expansion
    const int et = threadIdx.x - 128;
    for (int j = 0; j < njobs; ++j) {
      const int s = j % C::kStages;
      const uint32_t ph = (j / C::kStages) & 1;
      if (!mbar_wait(&full[s], ph, p.wait_limit_ns)) {
        fail(s_err, p.status);
        break;
      }
      if (j >= n_out) {
        uint8_t *sB = ring + s * C::kStage + C::kA;
        const uint8_t *sP = sB + C::kB;
        const uint32_t *sG = reinterpret_cast<const uint32_t *>(sP + C::kP);
#pragma unroll 2
        for (int t = et; t < BN * 4; t += 128) {
          const int row = t >> 2, c = t & 3;
          const uint4 pk = *reinterpret_cast<const uint4 *>(sP + row * 64 + c * 16);
          const uint32_t g = sG[row];
          const uint32_t s2 = static_cast<uint32_t>(__half2float(__ushort_as_half(
              static_cast<unsigned short>(g & 0xFFFFu))));
          const uint32_t z2 = static_cast<uint32_t>(__half2float(__ushort_as_half(
              static_cast<unsigned short>(g >> 16))));
          const uint32_t cst = (128u - z2 * s2) * 0x01010101u;
          uint4 o0, o1;
          o0.x = expand4(pk.x & 0x0F0F0F0Fu, s2, cst);
          o0.y = expand4((pk.x >> 4) & 0x0F0F0F0Fu, s2, cst);
          o0.z = expand4(pk.y & 0x0F0F0F0Fu, s2, cst);
          o0.w = expand4((pk.y >> 4) & 0x0F0F0F0Fu, s2, cst);
          o1.x = expand4(pk.z & 0x0F0F0F0Fu, s2, cst);
          o1.y = expand4((pk.z >> 4) & 0x0F0F0F0Fu, s2, cst);
          o1.z = expand4(pk.w & 0x0F0F0F0Fu, s2, cst);
          o1.w = expand4((pk.w >> 4) & 0x0F0F0F0Fu, s2, cst);
          const int sw = row & 7;
          *reinterpret_cast<uint4 *>(sB + row * 128 + (((2 * c) ^ sw) << 4)) = o0;
          *reinterpret_cast<uint4 *>(sB + row * 128 + (((2 * c + 1) ^ sw) << 4)) = o1;
        }
        fence_proxy_async_smem();
      }
      mbar_arrive(&ready[s]);
    }
  }
  __syncwarp();

  // ---------------------------------------------------------------- epilogue
  if (warp < 4) {
    if (!mbar_wait(accum_full, 0, p.wait_limit_ns)) fail(s_err, p.status);
    tc_fence_after();
  }
  __syncthreads();
  const bool failed = *s_err != 0;
  const uint32_t lane_base = static_cast<uint32_t>(warp * 32) << 16;

  if (S == 1) {
    if (warp < 4 && !failed) {
      const int row = warp * 32 + lane;
      const int m = m0 + row;
      const float sx = (!RAW && m < p.M) ? p.s_x[m] : 0.f;
#pragma unroll 1
      for (int c = 0; c < BN / 32; ++c) {
        const int n = n0 + c * 32;
        if (n >= p.N) break;
        uint32_t acc[32], o[32];
        tmem_ld32(tmem_base + lane_base + c * 32, acc);
        if (do_out) tmem_ld32(tmem_base + lane_base + BN + c * 32, o);
        tmem_ld_wait();
        if (m < p.M) {
          if (RAW) {
            int4 *dst = reinterpret_cast<int4 *>(static_cast<int32_t *>(p.Y) +
                                                 static_cast<size_t>(m) * p.ldy + n);
#pragma unroll
            for (int i = 0; i < 8; ++i)
              dst[i] = make_int4(static_cast<int>(acc[4 * i]), static_cast<int>(acc[4 * i + 1]),
                                 static_cast<int>(acc[4 * i + 2]),
                                 static_cast<int>(acc[4 * i + 3]));
          } else {
            const float4 *sw4 = reinterpret_cast<const float4 *>(p.s_w + n);
            uint32_t h[16];
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              const float4 w = __ldg(sw4 + i);
              const float wv[4] = {w.x, w.y, w.z, w.w};
              float y[4];
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                const int q = 4 * i + e;
                float v = __fmul_rn(__fmul_rn(static_cast<float>(static_cast<int>(acc[q])), sx),
                                    wv[e]);
                if (do_out) v = __fadd_rn(v, __uint_as_float(o[q]));
                y[e] = v;
              }
              const __half2 h0 = __floats2half2_rn(y[0], y[1]);
              const __half2 h1 = __floats2half2_rn(y[2], y[3]);
              h[2 * i] = *reinterpret_cast<const uint32_t *>(&h0);
              h[2 * i + 1] = *reinterpret_cast<const uint32_t *>(&h1);
            }
            uint4 *dst = reinterpret_cast<uint4 *>(static_cast<__half *>(p.Y) +
                                                   static_cast<size_t>(m) * p.ldy + n);
#pragma unroll
            for (int i = 0; i < 4; ++i)
              dst[i] = make_uint4(h[4 * i], h[4 * i + 1], h[4 * i + 2], h[4 * i + 3]);
          }
        }
      }
    }
  } else {
    // ------------------------------------ K split: reduce across the cluster
    int32_t *pbuf = reinterpret_cast<int32_t *>(ring);
    float *obuf = reinterpret_cast<float *>(ring + kTileM * C::kPitch * 4);
    const int rows_valid = min(kTileM, p.M - m0);
    const uint32_t my_rank = cluster_ctarank();
    // this CTA reduces columns [c_begin, c_end) of each 128-column chunk
    const int c_begin = static_cast<int>(my_rank) * (C::kCW / 4) / S * 4;
    const int c_end = (static_cast<int>(my_rank) + 1) * (C::kCW / 4) / S * 4;
    const int c4n = (c_end - c_begin) / 4;
#pragma unroll 1
    for (int r = 0; r < BN / C::kCW; ++r) {
      if (warp < 4 && !failed) {
        const int row = warp * 32 + lane;
#pragma unroll 1
        for (int c = 0; c < C::kCW / 32; ++c) {
          uint32_t acc[32], o[32];
          const uint32_t col = r * C::kCW + c * 32;
          tmem_ld32(tmem_base + lane_base + col, acc);
          if (do_out) tmem_ld32(tmem_base + lane_base + BN + col, o);
          tmem_ld_wait();
          if (row < rows_valid) {
            int4 *pd = reinterpret_cast<int4 *>(pbuf + row * C::kPitch + c * 32);
#pragma unroll
            for (int i = 0; i < 8; ++i)
              pd[i] = make_int4(static_cast<int>(acc[4 * i]), static_cast<int>(acc[4 * i + 1]),
                                static_cast<int>(acc[4 * i + 2]),
                                static_cast<int>(acc[4 * i + 3]));
            if (do_out) {
              int4 *od = reinterpret_cast<int4 *>(obuf + row * C::kPitch + c * 32);
#pragma unroll
              for (int i = 0; i < 8; ++i)
                od[i] = make_int4(static_cast<int>(o[4 * i]), static_cast<int>(o[4 * i + 1]),
                                  static_cast<int>(o[4 * i + 2]),
                                  static_cast<int>(o[4 * i + 3]));
            }
          }
        }
      }
      cluster_sync_all();
      if (!failed) {
#pragma unroll 1
        for (int e = threadIdx.x; e < rows_valid * c4n; e += blockDim.x) {
          const int row = e / c4n, c4 = e % c4n;
          const int col = c_begin + c4 * 4;
          const int n = n0 + r * C::kCW + col;
          if (n >= p.N) continue;
          const int m = m0 + row;
          const uint32_t off = smem_u32(pbuf + row * C::kPitch + col);
          int4 sum = make_int4(0, 0, 0, 0);
          for (int q = 0; q < S; ++q) {
            const int4 v = ld_dsmem_v4(mapa_shared(off, static_cast<uint32_t>(q)));
            sum.x += v.x;
            sum.y += v.y;
            sum.z += v.z;
            sum.w += v.w;
          }
          if (RAW) {
            *reinterpret_cast<int4 *>(static_cast<int32_t *>(p.Y) + static_cast<size_t>(m) * p.ldy +
                                      n) = sum;
          } else {
            float ov[4] = {0.f, 0.f, 0.f, 0.f};
            if (any_out) {
              const int4 oi = ld_dsmem_v4(mapa_shared(smem_u32(obuf + row * C::kPitch + col), 0u));
              ov[0] = __int_as_float(oi.x);
              ov[1] = __int_as_float(oi.y);
              ov[2] = __int_as_float(oi.z);
              ov[3] = __int_as_float(oi.w);
            }
            const float sx = p.s_x[m];
            const float4 w = __ldg(reinterpret_cast<const float4 *>(p.s_w + n));
            const int si[4] = {sum.x, sum.y, sum.z, sum.w};
            const float wv[4] = {w.x, w.y, w.z, w.w};
            float y[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              float v = __fmul_rn(__fmul_rn(static_cast<float>(si[i]), sx), wv[i]);
              if (any_out) v = __fadd_rn(v, ov[i]);
              y[i] = v;
            }
            const __half2 h0 = __floats2half2_rn(y[0], y[1]);
            const __half2 h1 = __floats2half2_rn(y[2], y[3]);
            *reinterpret_cast<uint2 *>(static_cast<__half *>(p.Y) + static_cast<size_t>(m) * p.ldy +
                                       n) =
                make_uint2(*reinterpret_cast<const uint32_t *>(&h0),
                           *reinterpret_cast<const uint32_t *>(&h1));
          }
        }
      }
      cluster_sync_all();
    }
  }

  // ---------------------------------------------------------------- teardown
  tc_fence_before();
  __syncthreads();
  if (failed && threadIdx.x == 0) {
    // Let any tile copy still in flight land before the CTA's shared memory
    // is released: wait (bounded) for every load issued but never consumed.
    for (int j = s_misc[2]; j < s_misc[3]; ++j)
      mbar_wait(&full[j % C::kStages], (j / C::kStages) & 1, p.wait_limit_ns);
  }
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, C::kTmemCols);
  }
}

// ------------------------------------------------------------------ host side
using EncodeTiledFn = CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                   const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                   const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// Row-major 2-D tensor [outer][inner] of `elem` bytes per element.
bool make_map(CUtensorMap *map, CUtensorMapDataType dt, int elem, const void *base,
              uint64_t inner, uint64_t outer, uint64_t row_bytes, uint32_t box_inner,
              uint32_t box_outer, CUtensorMapSwizzle sw) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {row_bytes};
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t estr[2] = {1, 1};
  (void)elem;
  return fn(map, dt, 2, const_cast<void *>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// cudaFuncSetAttribute once per (kernel, device).
template <typename K>
cudaError_t ensure_smem(K kernel, int bytes, std::atomic<uint64_t> &done_mask) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const uint64_t bit = 1ull << (dev & 63);
  if (done_mask.load(std::memory_order_acquire) & bit) return cudaSuccess;
  e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e == cudaSuccess) done_mask.fetch_or(bit, std::memory_order_acq_rel);
  return e;
}

template <int BN, bool W4, bool RAW>
cudaError_t launch_variant(const GemmArgs &a, const GemmPlan &plan, cudaStream_t stream,
                           const char **why) {
  using C = Cfg<BN, W4>;
  static std::atomic<uint64_t> smem_done{0};
  auto kernel = mixq_gemm_kernel<BN, W4, RAW>;
  cudaError_t e = ensure_smem(kernel, C::kSmem, smem_done);
  if (e != cudaSuccess) return e;

  const int kp = k_out_pad(a.K_out);
  alignas(64) CUtensorMap tm_a, tm_b, tm_g, tm_xo, tm_wo;
  memset(&tm_g, 0, sizeof tm_g);
  memset(&tm_xo, 0, sizeof tm_xo);
  memset(&tm_wo, 0, sizeof tm_wo);
  bool ok = make_map(&tm_a, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, a.Xq, a.K, a.M, a.K, kBlockK,
                     kTileM, CU_TENSOR_MAP_SWIZZLE_128B);
  if (!W4) {
    ok = ok && make_map(&tm_b, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, a.Wq, a.K, a.N, a.K, kBlockK,
                        BN, CU_TENSOR_MAP_SWIZZLE_128B);
  } else {
    ok = ok && make_map(&tm_b, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, a.Wq, a.K / 2, a.N, a.K / 2,
                        kBlockK / 2, BN, CU_TENSOR_MAP_SWIZZLE_NONE);
    ok = ok && make_map(&tm_g, CU_TENSOR_MAP_DATA_TYPE_UINT32, 4, a.grp, a.N, a.K / kGroup,
                        static_cast<uint64_t>(a.N) * 4, BN, 1, CU_TENSOR_MAP_SWIZZLE_NONE);
  }
  if (!RAW && kp > 0) {
    ok = ok && make_map(&tm_xo, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, a.X_out, kp, a.M,
                        static_cast<uint64_t>(kp) * 2, kOutBlockK, kTileM,
                        CU_TENSOR_MAP_SWIZZLE_128B);
    ok = ok && make_map(&tm_wo, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, a.W_out, kp, a.N,
                        static_cast<uint64_t>(kp) * 2, kOutBlockK, BN,
                        CU_TENSOR_MAP_SWIZZLE_128B);
  }
  if (!ok) {
    *why = "cuTensorMapEncodeTiled failed (or the driver entry point is unavailable)";
    return cudaErrorInvalidValue;
  }

  KParams kp_{};
  kp_.M = a.M;
  kp_.N = a.N;
  kp_.K = a.K;
  kp_.K_out_pad = RAW ? 0 : kp;
  kp_.s_x = a.s_x;
  kp_.s_w = a.s_w;
  kp_.flags = a.flags;
  kp_.Y = a.Y;
  kp_.ldy = a.ldy;
  kp_.status = a.status;
  kp_.wait_limit_ns = a.wait_limit_ns;
  kp_.debug_stall = a.debug_stall;
  kp_.b_streamed = (a.M + kTileM - 1) / kTileM == 1;

  const int m_tiles = (a.M + kTileM - 1) / kTileM;
  const int n_tiles = (a.N + BN - 1) / BN;
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(m_tiles, n_tiles, plan.split);
  cfg.blockDim = dim3(C::kThreads, 1, 1);
  cfg.dynamicSmemBytes = C::kSmem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 1;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = plan.split;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, tm_a, tm_b, tm_g, tm_xo, tm_wo, kp_);
}

}  // namespace

GemmPlan plan_gemm(int mode, int M, int N, int K, int num_sms) {
  // Time model (microseconds).  Compute: waves of CTAs (one per SM), each
  // running its K range at one 128 x BN x 128 INT8 MMA stage per
  // 0.28 us * BN/256, plus a fixed prologue/epilogue and the cluster
  // reduction when K is split.  Memory: the bytes that must come from HBM at
  // least once (weights, activations, output) at the smaller of the HBM
  // rate and what the active SMs can pull (~60 GB/s each).  The plan with
  // the smaller max(compute, memory) wins; ties keep fewer CTAs.
  GemmPlan best{256, 1, 0};
  double best_cost = 1e300;
  const int m_tiles = (M + kTileM - 1) / kTileM;
  const int KB = K / kBlockK;
  const double w_bytes = (mode == 1 ? 0.5 + 4.0 / kGroup : 1.0) * static_cast<double>(N) * K;
  const double unique_bytes = w_bytes + static_cast<double>(M) * K + 2.0 * M * N;
  const int bns[2] = {256, 128};
  for (int bn : bns) {
    const int n_tiles = (N + bn - 1) / bn;
    for (int s = 1; s <= 8 && s <= KB; ++s) {
      const long long ctas = static_cast<long long>(m_tiles) * n_tiles * s;
      const long long waves = (ctas + num_sms - 1) / num_sms;
      const int kb_per = (KB + s - 1) / s;
      const double fixed = 1.0 + (s > 1 ? 0.3 + 0.05 * s : 0.0);
      const double compute = waves * (kb_per * 0.28 * (bn / 256.0) + fixed);
      const double active = static_cast<double>(ctas < num_sms ? ctas : num_sms);
      const double bw = active * 60e3 < 6.5e6 ? active * 60e3 : 6.5e6;  // bytes per us
      const double memory = unique_bytes / bw + fixed;
      const double cost = compute > memory ? compute : memory;
      if (cost < best_cost * (1 - 1e-6)) {
        best_cost = cost;
        best = GemmPlan{bn, s, static_cast<int>(ctas)};
      }
    }
  }
  return best;
}

cudaError_t launch_gemm(const GemmArgs &a, const GemmPlan &plan, cudaStream_t stream,
                        const char **why) {
  const bool w4 = a.mode == 1;
  const bool raw = a.epi == Epi::kRawI32;
  if (plan.bn == 256) {
    if (w4) return raw ? launch_variant<256, true, true>(a, plan, stream, why)
                       : launch_variant<256, true, false>(a, plan, stream, why);
    return raw ? launch_variant<256, false, true>(a, plan, stream, why)
               : launch_variant<256, false, false>(a, plan, stream, why);
  }
  if (w4) return raw ? launch_variant<128, true, true>(a, plan, stream, why)
                     : launch_variant<128, true, false>(a, plan, stream, why);
  return raw ? launch_variant<128, false, true>(a, plan, stream, why)
             : launch_variant<128, false, false>(a, plan, stream, why);
}

}  // namespace mixq
