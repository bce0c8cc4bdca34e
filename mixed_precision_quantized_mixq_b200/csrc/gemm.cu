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
#include "tma_host.h"

namespace mixq {
namespace {

// Shared-memory plan (all offsets multiples of 1 KB):
//   ring  = [A slots: stages x a_stride][B stages: stages x kBStage]
//   then    barriers (1 KB), s_w of the tile (1 KB), s_x of the tile (512 B).
// An A slot holds the Xq (or X_out) tile of one stage: a_stride = 16 KB (128
// rows) normally.  With SM ("small M", at most 64 tokens) a slot holds only
// the token rows (M rounded up to 8, 128 bytes each); the MMA still reads 128
// rows, and rows past the slot run into the next slots or the B stages --
// rows of D that are never stored.  That keeps a decode-sized CTA near
// 100 KB, so one CTA of the next kernel fits beside it on the SM (two CTAs'
// TMEM, 2 x 2 x 128 columns, fit too) and, launched early by programmatic
// dependent launch, streams its weights while this kernel finishes.
// A B stage holds the INT8 weight tile (or the W_out tile), and for W4 the
// packed 4-bit codes and their group constants.
template <int BN, bool W4, bool SM>
struct Cfg {
  static constexpr int kMaxStages = 8;
  static constexpr int kB = BN * kBlockK;                  // INT8 / fp16 B tile
  static constexpr int kP = W4 ? BN * (kBlockK / 2) : 0;   // packed 4-bit codes
  static constexpr int kG = W4 ? ((BN * 4 + 1023) / 1024) * 1024 : 0;  // (s2,z2) per row
  static constexpr int kBStage = kB + kP + kG;
  // full-size (not SM) stage count; SM stage counts are chosen at launch
  static constexpr int kStages = W4 ? (BN == 256 ? 3 : 5) : (BN == 256 ? 4 : 6);
  static constexpr int kExpandThreads = W4 ? (SM ? 128 : 256) : 0;  // warps 4..
  static constexpr int kThreads = 128 + kExpandThreads;
  static constexpr int kMinBlocks = SM ? 2 : 1;
  static constexpr int kTmemCols = 2 * BN;  // INT32 acc [0,BN), FP32 outlier acc [BN,2BN)
  static constexpr int kExtra = 1024 + 1024 + 512;  // barriers, s_w, s_x
  // weight bytes of one 128-row tile of one K block, and of one weight row
  static constexpr int kSubW = W4 ? 128 * (kBlockK / 2) : 128 * kBlockK;
  static constexpr int kRowW = W4 ? kBlockK / 2 : kBlockK;
  static constexpr int kSubRows = BN < 128 ? BN : 128;  // rows per bulk copy
  static_assert(BN == 32 || BN == 64 || BN == 128 || BN == 256, "tile width");
  static_assert(BN >= 128 || SM, "narrow tiles are small-M only");
  // cluster reduction buffers (reuse the ring after the mainloop)
  static constexpr int kCW = BN < 128 ? BN : 128;  // columns per reduction round
  static constexpr int kPitch = kCW + 4;  // words; +4 keeps 16-byte rows off one bank group
  static constexpr int kRedRows = SM ? 64 : 128;
  static constexpr int kRedBytes = 2 * kRedRows * kPitch * 4;
  __host__ __device__ static constexpr int ring_bytes(int stages, int a_stride) {
    return stages * (a_stride + kBStage);
  }
  __host__ __device__ static constexpr int smem_bytes(int stages, int a_stride) {
    return ring_bytes(stages, a_stride) + kExtra + 1024;  // + alignment slack
  }
};

struct KParams {
  int M, N, K, K_out_pad;
  int a_rows;            // rows of the A / X_out TMA box (M rounded up to 8, at most 128)
  int a_stride;          // bytes of one A slot
  int stages;            // pipeline depth
  const uint8_t *wq;     // tiled weight codes (W8: 16 KB tiles, W4: 8 KB tiles)
  const uint8_t *grp;    // W4 group constants [K/128][N] (s2, z2) fp16 pairs
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

// Whether the FP16 outlier slice runs: some token is mixed (flags[0] > 0), or
// the caller passed no flags.  Read after griddep_wait().
__device__ __forceinline__ int outliers_present(const KParams &p, bool raw) {
  if (raw || p.K_out_pad == 0) return 0;
  return p.flags ? (*reinterpret_cast<const volatile int32_t *>(p.flags) > 0) : 1;
}

template <int BN, bool W4, bool SM, bool RAW>
__global__ void __launch_bounds__(Cfg<BN, W4, SM>::kThreads, Cfg<BN, W4, SM>::kMinBlocks)
    mixq_gemm_kernel(const __grid_constant__ CUtensorMap tm_a,   // Xq   [M][K] int8
                     const __grid_constant__ CUtensorMap tm_xo,  // X_out [M][K_out_pad] fp16
                     const __grid_constant__ CUtensorMap tm_wo,  // W_out [N][K_out_pad] fp16
                     const __grid_constant__ CUtensorMap tm_y,   // Y [M][ldy] fp16 (store)
                     const KParams p) {
  using C = Cfg<BN, W4, SM>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const int stages = p.stages;
  uint8_t *ring = smem;
  uint8_t *b_region = ring + stages * p.a_stride;
  auto a_slot = [&](int s) { return ring + s * p.a_stride; };
  auto b_slot = [&](int s) { return b_region + s * C::kBStage; };
  uint8_t *extra = ring + C::ring_bytes(stages, p.a_stride);
  uint64_t *bars = reinterpret_cast<uint64_t *>(extra);
  uint64_t *full = bars;
  uint64_t *empty = bars + C::kMaxStages;
  uint64_t *ready = bars + 2 * C::kMaxStages;
  uint64_t *accum_full = bars + 3 * C::kMaxStages;
  uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(accum_full + 1);
  int *s_misc = reinterpret_cast<int *>(tmem_holder + 1);  // err, -, consumed, issued
  float *s_sw = reinterpret_cast<float *>(extra + 1024);   // [BN]
  float *s_sx = reinterpret_cast<float *>(extra + 2048);   // [128]

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int m0 = blockIdx.x * kTileM;
  const int n0 = blockIdx.y * BN;
  const int S = gridDim.z;
  const int rank = blockIdx.z;
  const int KB = p.K / kBlockK;
  const int kb_begin = static_cast<int>(static_cast<long long>(rank) * KB / S);
  const int kb_end = static_cast<int>(static_cast<long long>(rank + 1) * KB / S);
  const int n_i8 = kb_end - kb_begin;                   // INT8 jobs come first
  // weight rows of the tile come in n_sub slices of kSubRows rows (a slice of
  // one 128-row weight tile when BN < 128; for BN = 256 the second slice is
  // absent in the last column tile when N % 256 == 128)
  const int n_sub = BN < 128 ? 1 : min(BN, p.N - n0) / 128;
  const uint32_t a_bytes = static_cast<uint32_t>(p.a_rows) * kBlockK;
  const uint32_t b_bytes = static_cast<uint32_t>(n_sub) * C::kSubRows * (C::kRowW + (W4 ? 4 : 0));
  const int pre = n_i8 < stages ? n_i8 : stages;        // stages whose weights go out early

  // address of the weight slice h of K block kb, and of its group constants
  auto w_src = [&](int kb, int h) {
    const int nrow = n0 + h * 128;
    const size_t tile = static_cast<size_t>(nrow / 128) * KB + kb;
    return p.wq + tile * C::kSubW + (nrow % 128) * C::kRowW;
  };
  auto g_src = [&](int kb, int h) {
    return p.grp + (static_cast<size_t>(kb) * p.N + n0 + h * 128) * 4;
  };
  // weights of INT8 job j (K block kb_begin + j) into stage s: one bulk copy
  // per weight slice (plus its group constants for W4)
  auto issue_b = [&](int j, int s, uint64_t pol_b) {
    const int kb = kb_begin + j;
    uint8_t *sB = b_slot(s);
    uint8_t *dstW = W4 ? sB + C::kB : sB;
    uint8_t *dstG = sB + C::kB + C::kP;
    for (int h = 0; h < n_sub; ++h) {
      bulk_load(dstW + h * 128 * C::kRowW, w_src(kb, h), C::kSubRows * C::kRowW, &full[s], pol_b);
      if (W4) bulk_load(dstG + h * 128 * 4, g_src(kb, h), C::kSubRows * 4, &full[s], pol_b);
    }
  };

  if (threadIdx.x == 0) {
    for (int i = 0; i < stages; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
      if (W4) mbar_init(&ready[i], C::kExpandThreads);
    }
    mbar_init(accum_full, 1);
    fence_mbar_init();
    s_misc[0] = 0;
    s_misc[1] = 0;
    s_misc[2] = 0;
    s_misc[3] = 0;
    // The weights do not depend on the preceding kernel: start streaming them
    // first, before the rest of the set-up and before waiting for that kernel.
    if (!p.debug_stall) {
      const uint64_t pol_b = p.b_streamed ? policy_evict_first() : policy_evict_last();
      for (int j = 0; j < pre; ++j) {
        mbar_arrive_expect_tx(&full[j], a_bytes + b_bytes);
        issue_b(j, j, pol_b);
      }
    }
    tma_prefetch_desc(&tm_a);
    if (!RAW && p.K_out_pad > 0 && rank == 0) {
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
  if (threadIdx.x == 0) griddep_launch_dependents();
  const uint32_t tmem_base = *tmem_holder;
  int *s_err = &s_misc[0];

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0 && !p.debug_stall) {
      const uint64_t pol_a = policy_evict_last();
      const uint64_t pol_b = p.b_streamed ? policy_evict_first() : policy_evict_last();
      griddep_wait();
      // the token tiles of the early stages go out before the flags word is
      // read: queued behind the weight stream, that read takes microseconds
      for (int j = 0; j < pre; ++j)
        tma_load_2d(a_slot(j), &tm_a, &full[j], (kb_begin + j) * kBlockK, m0, pol_a);
      const int n_out = (outliers_present(p, RAW) && rank == 0) ? p.K_out_pad / kOutBlockK : 0;
      const int njobs = n_i8 + n_out;
      int issued = pre;
      int s = pre == stages ? 0 : pre;
      uint32_t ph = pre == stages ? 1u : 0u;
      for (int j = pre; j < njobs; ++j) {
        if (j > pre && ++s == stages) {
          s = 0;
          ph ^= 1u;
        }
        if (!mbar_wait(&empty[s], ph ^ 1, p.wait_limit_ns)) {
          fail(s_err, p.status);
          break;
        }
        if (j < n_i8) {
          mbar_arrive_expect_tx(&full[s], a_bytes + b_bytes);
          tma_load_2d(a_slot(s), &tm_a, &full[s], (kb_begin + j) * kBlockK, m0, pol_a);
          issue_b(j, s, pol_b);
        } else {
          const int o = j - n_i8;
          mbar_arrive_expect_tx(&full[s], a_bytes + C::kB);
          tma_load_2d(a_slot(s), &tm_xo, &full[s], o * kOutBlockK, m0, pol_a);
          tma_load_2d(b_slot(s), &tm_wo, &full[s], o * kOutBlockK, n0, pol_b);
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
      // This thread's per-job path bounds a decode-sized CTA (its MMAs are
      // short): the ring position advances incrementally, and a stage's
      // descriptors are those of stage 0 plus a fixed start-address offset.
      const uint64_t ad0 = sw128_kmajor_desc(smem_u32(a_slot(0)));
      const uint64_t bd0 = sw128_kmajor_desc(smem_u32(b_slot(0)));
      const uint64_t a_step = static_cast<uint64_t>(p.a_stride >> 4);
      constexpr uint64_t b_step = static_cast<uint64_t>(C::kBStage >> 4);
      uint64_t *const gate = W4 ? ready : full;
      griddep_wait();
      // the INT8 jobs first: the flags word (is there an outlier slice) is
      // read once they are issued, off the path of the first MMAs
      int njobs = p.debug_stall ? 1 : n_i8;
      bool counted = p.debug_stall != 0;
      int s = 0, j = 0;
      uint32_t ph = 0;
      uint64_t ad = ad0, bd = bd0;
      for (;; ++j) {
        if (j == njobs) {
          if (counted) break;
          counted = true;
          njobs += (outliers_present(p, RAW) && rank == 0) ? p.K_out_pad / kOutBlockK : 0;
          if (j == njobs) break;
        }
        if (!mbar_try_wait(&gate[s], ph) && !mbar_wait(&gate[s], ph, p.wait_limit_ns)) {
          fail(s_err, p.status);
          break;
        }
        tc_fence_after();
        if (j < n_i8) {
#pragma unroll
          for (int k = 0; k < 4; ++k)
            mma_i8(t_i32, ad + 2 * k, bd + 2 * k, kIdI8, (j > 0 || k > 0) ? 1u : 0u);
        } else {
#pragma unroll
          for (int k = 0; k < 4; ++k)
            mma_f16(t_f32, ad + 2 * k, bd + 2 * k, kIdF16, (j > n_i8 || k > 0) ? 1u : 0u);
        }
        mma_commit(&empty[s]);
        if (++s == stages) {
          s = 0;
          ph ^= 1u;
          ad = ad0;
          bd = bd0;
        } else {
          ad += a_step;
          bd += b_step;
        }
      }
      mma_commit(accum_full);
      s_misc[2] = j;
    }
  } else if ((warp == 2 || warp == 3) && !RAW) {
    // ------------------------------------ token scales of the tile, early
    // per-channel weight scales first (they do not depend on the preceding
    // kernel), then the token scales; both during the mainloop, off the
    // set-up path (a global read there delays every role by its latency)
    for (int i = threadIdx.x - 64; i < BN; i += 64) s_sw[i] = n0 + i < p.N ? p.s_w[n0 + i] : 0.f;
    griddep_wait();
    for (int i = threadIdx.x - 64; i < kTileM; i += 64)
      s_sx[i] = m0 + i < p.M ? p.s_x[m0 + i] : 0.f;
  } else if (W4 && warp >= 4) {
    // ------------------------------------------- 4-bit -> INT8 expansion
    // Thread -> one weight row, so the row's (s2, z2) constants are decoded
    // once per K block.
    constexpr int kCpt = W4 ? BN * 4 / C::kExpandThreads : 1;  // 16-byte chunks per thread
    const int et = threadIdx.x - 128;
    const int row = et % BN;
    const int c0 = W4 ? (et / BN) * kCpt : 0;
    // the INT8 jobs need nothing from the preceding kernel; the flags word is
    // read (after waiting for that kernel) once they are done
    int njobs = p.debug_stall ? 0 : n_i8;
    bool counted = p.debug_stall != 0;
    for (int j = 0;; ++j) {
      if (j == njobs) {
        if (counted) break;
        counted = true;
        griddep_wait();
        njobs += (outliers_present(p, RAW) && rank == 0) ? p.K_out_pad / kOutBlockK : 0;
        if (j == njobs) break;
      }
      const int s = j % stages;
      const uint32_t ph = (j / stages) & 1;
      if (!mbar_wait(&full[s], ph, p.wait_limit_ns)) {
        fail(s_err, p.status);
        break;
      }
      if (j < n_i8) {
        uint8_t *sB = b_slot(s);
        const uint8_t *sP = sB + C::kB;
        const uint32_t g = reinterpret_cast<const uint32_t *>(sP + C::kP)[row];
        const uint32_t s2 = static_cast<uint32_t>(__half2float(__ushort_as_half(
            static_cast<unsigned short>(g & 0xFFFFu))));
        const uint32_t z2 = static_cast<uint32_t>(__half2float(__ushort_as_half(
            static_cast<unsigned short>(g >> 16))));
        const uint32_t cst = (128u - z2 * s2) * 0x01010101u;
        const int psw = (row >> 1) & 3, osw = row & 7;
        uint4 pk[kCpt];
#pragma unroll
        for (int i = 0; i < kCpt; ++i)
          pk[i] = *reinterpret_cast<const uint4 *>(sP + row * 64 + (((c0 + i) ^ psw) << 4));
#pragma unroll
        for (int i = 0; i < kCpt; ++i) {
          const int c = c0 + i;
          uint4 o0, o1;
          o0.x = expand4(pk[i].x & 0x0F0F0F0Fu, s2, cst);
          o0.y = expand4((pk[i].x >> 4) & 0x0F0F0F0Fu, s2, cst);
          o0.z = expand4(pk[i].y & 0x0F0F0F0Fu, s2, cst);
          o0.w = expand4((pk[i].y >> 4) & 0x0F0F0F0Fu, s2, cst);
          o1.x = expand4(pk[i].z & 0x0F0F0F0Fu, s2, cst);
          o1.y = expand4((pk[i].z >> 4) & 0x0F0F0F0Fu, s2, cst);
          o1.z = expand4(pk[i].w & 0x0F0F0F0Fu, s2, cst);
          o1.w = expand4((pk[i].w >> 4) & 0x0F0F0F0Fu, s2, cst);
          *reinterpret_cast<uint4 *>(sB + row * 128 + (((2 * c) ^ osw) << 4)) = o0;
          *reinterpret_cast<uint4 *>(sB + row * 128 + (((2 * c + 1) ^ osw) << 4)) = o1;
        }
        fence_proxy_async_smem();
      }
      mbar_arrive(&ready[s]);
    }
  }
  __syncwarp();

  // ---------------------------------------------------------------- epilogue
  griddep_wait();
  const int any_out = outliers_present(p, RAW);
  const bool do_out = any_out && rank == 0;
  if (warp < 4) {
    if (!mbar_wait_sleep(accum_full, 0, p.wait_limit_ns)) fail(s_err, p.status);
    tc_fence_after();
  }
  __syncthreads();
  const bool failed = *s_err != 0;
  const uint32_t lane_base = static_cast<uint32_t>(warp * 32) << 16;

  if (S == 1 && !RAW && BN >= 64) {
    // Stage the fp16 tile in shared memory in the 128-byte swizzled layout of
    // a TMA store (64-column sub-tiles of a_rows rows; a thread's 16-byte
    // pieces of one row land on 8 different bank groups), then one thread
    // writes it out with coalesced bulk tensor stores.
    uint8_t *stage_y = ring;  // the ring is free: every MMA has completed
    const int box_rows = p.a_rows;
    if (warp < 4 && !failed) {
      const int row = warp * 32 + lane;
      const float sx = s_sx[row];
#pragma unroll 1
      for (int c = 0; c < BN / 32; ++c) {
        if (n0 + c * 32 >= p.N) break;
        uint32_t acc[32], o[32];
        tmem_ld32(tmem_base + lane_base + c * 32, acc);
        if (do_out) tmem_ld32(tmem_base + lane_base + BN + c * 32, o);
        tmem_ld_wait();
        if (row < box_rows) {
          const float4 *sw4 = reinterpret_cast<const float4 *>(s_sw + c * 32);
          uint32_t h[16];
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const float4 w = sw4[i];
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
          uint8_t *rowp = stage_y + (c >> 1) * box_rows * 128 + row * 128;
          const int j0 = (c & 1) * 4;
#pragma unroll
          for (int q = 0; q < 4; ++q)
            *reinterpret_cast<uint4 *>(rowp + (((j0 + q) ^ (row & 7)) << 4)) =
                make_uint4(h[4 * q], h[4 * q + 1], h[4 * q + 2], h[4 * q + 3]);
        }
      }
      fence_proxy_async_smem();
    }
    if (warp < 4) named_barrier(1, 128);
    if (threadIdx.x == 0 && !failed) {
      const int cols = min(BN, p.N - n0);
      for (int t = 0; t < cols / 64; ++t)
        tma_store_2d(&tm_y, stage_y + t * box_rows * 128, n0 + t * 64, m0);
      bulk_commit_group();
      bulk_wait_all();
    }
  } else if (S == 1) {
    if (warp < 4 && !failed) {
      const int row = warp * 32 + lane;
      const int m = m0 + row;
      const float sx = RAW ? 0.f : s_sx[row];
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
            const float4 *sw4 = reinterpret_cast<const float4 *>(s_sw + c * 32);
            uint32_t h[16];
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              const float4 w = sw4[i];
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
    float *obuf = reinterpret_cast<float *>(ring + C::kRedRows * C::kPitch * 4);
    const int rows_valid = min(C::kRedRows, p.M - m0);
    const uint32_t my_rank = cluster_ctarank();
    // this CTA reduces columns [c_begin, c_end) of each 128-column chunk
    const int c_begin = static_cast<int>(my_rank) * (C::kCW / 4) / S * 4;
    const int c_end = (static_cast<int>(my_rank) + 1) * (C::kCW / 4) / S * 4;
    const int c4n = (c_end - c_begin) / 4;
#pragma unroll 1
    for (int r = 0; r < BN / C::kCW; ++r) {
      // only the warps whose TMEM lanes hold token rows read the accumulators
      if (warp < 4 && warp * 32 < rows_valid && !failed) {
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
          // issue every peer's load before summing, so their latencies overlap
          int4 part[C::kMaxStages];
#pragma unroll
          for (int q = 0; q < 8; ++q)
            if (q < S) part[q] = ld_dsmem_v4(mapa_shared(off, static_cast<uint32_t>(q)));
          int4 oi = make_int4(0, 0, 0, 0);
          if (!RAW && any_out)
            oi = ld_dsmem_v4(mapa_shared(smem_u32(obuf + row * C::kPitch + col), 0u));
          int4 sum = make_int4(0, 0, 0, 0);
#pragma unroll
          for (int q = 0; q < 8; ++q) {
            if (q < S) {
              sum.x += part[q].x;
              sum.y += part[q].y;
              sum.z += part[q].z;
              sum.w += part[q].w;
            }
          }
          if (RAW) {
            *reinterpret_cast<int4 *>(static_cast<int32_t *>(p.Y) + static_cast<size_t>(m) * p.ldy +
                                      n) = sum;
          } else {
            const float ov[4] = {__int_as_float(oi.x), __int_as_float(oi.y), __int_as_float(oi.z),
                                 __int_as_float(oi.w)};
            const float sx = s_sx[row];
            const float4 w = *reinterpret_cast<const float4 *>(s_sw + r * C::kCW + col);
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
      mbar_wait(&full[j % stages], (j / stages) & 1, p.wait_limit_ns);
  }
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, C::kTmemCols);
  }
}

// ------------------------------------------------------------------ host side
// Pipeline geometry of a launch: stage count, A slot size, dynamic smem.
// Full-size variants use 128-row A slots and a fixed depth; the small-M
// variant sizes its A slots to the token rows and takes as many stages as fit
// in half an SM's shared memory (so a CTA of the next kernel fits beside it).
struct Geometry {
  int stages, a_stride, smem;
};

template <int BN, bool W4, bool SM>
Geometry geometry(int M, int split) {
  using C = Cfg<BN, W4, SM>;
  Geometry g{};
  if (!SM) {
    g.stages = C::kStages;
    g.a_stride = kTileM * kBlockK;
  } else {
    const int a_rows = M >= kTileM ? kTileM : (M + 7) / 8 * 8;  // = the TMA box rows
    g.a_stride = a_rows * kBlockK;
    const int budget = 233472 / 2 - 1024 - C::kExtra - 1024;  // half an SM, minus reserve
    g.stages = budget / (g.a_stride + C::kBStage);
    if (g.stages > C::kMaxStages) g.stages = C::kMaxStages;
    while (split > 1 && g.stages < C::kMaxStages &&
           C::ring_bytes(g.stages, g.a_stride) < C::kRedBytes)
      ++g.stages;
  }
  g.smem = C::smem_bytes(g.stages, g.a_stride);
  return g;
}

template <int BN, bool W4, bool SM>
constexpr int max_smem() {
  using C = Cfg<BN, W4, SM>;
  return SM ? 233472 / 2 - 1024 : C::smem_bytes(C::kStages, kTileM * kBlockK);
}

template <int BN, bool W4, bool SM, bool RAW>
cudaError_t launch_variant(const GemmArgs &a, const GemmPlan &plan, cudaStream_t stream,
                           const char **why) {
  using C = Cfg<BN, W4, SM>;
  static_assert(max_smem<BN, W4, SM>() <= 232448, "shared memory budget");
  static std::atomic<uint64_t> smem_done{0};
  auto kernel = mixq_gemm_kernel<BN, W4, SM, RAW>;
  cudaError_t e = ensure_smem(kernel, max_smem<BN, W4, SM>(), smem_done);
  if (e != cudaSuccess) return e;
  if (plan.split > 1 && a.M > C::kRedRows && (a.M + kTileM - 1) / kTileM * kTileM > C::kRedRows &&
      C::kRedRows < kTileM) {
    *why = "a K split of this variant reduces at most 64 rows per tile";
    return cudaErrorInvalidValue;
  }
  const Geometry geo = geometry<BN, W4, SM>(a.M, plan.split);
  if (geo.smem > max_smem<BN, W4, SM>() || geo.stages < 2 ||
      (plan.split > 1 && C::ring_bytes(geo.stages, geo.a_stride) < C::kRedBytes)) {
    *why = "no pipeline geometry fits the shared-memory budget";
    return cudaErrorInvalidValue;
  }

  const int kp = k_out_pad(a.K_out);
  const int a_rows = a.M >= kTileM ? kTileM : (a.M + 7) / 8 * 8;
  alignas(64) CUtensorMap tm_a, tm_xo, tm_wo, tm_y;
  memset(&tm_xo, 0, sizeof tm_xo);
  memset(&tm_wo, 0, sizeof tm_wo);
  memset(&tm_y, 0, sizeof tm_y);
  bool ok = make_map(&tm_a, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, a.Xq, a.K, a.M, a.K, kBlockK,
                     a_rows, CU_TENSOR_MAP_SWIZZLE_128B);
  if (a.epi != Epi::kRawI32 && kp > 0) {
    ok = ok && make_map(&tm_xo, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, a.X_out, kp, a.M,
                        static_cast<uint64_t>(kp) * 2, kOutBlockK, a_rows,
                        CU_TENSOR_MAP_SWIZZLE_128B);
    ok = ok && make_map(&tm_wo, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, a.W_out, kp, a.N,
                        static_cast<uint64_t>(kp) * 2, kOutBlockK, BN,
                        CU_TENSOR_MAP_SWIZZLE_128B);
  }
  if (a.epi != Epi::kRawI32 && BN >= 64)
    ok = ok && make_map(&tm_y, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, a.Y, a.N, a.M,
                        static_cast<uint64_t>(a.ldy) * 2, 64, a_rows,
                        CU_TENSOR_MAP_SWIZZLE_128B);
  if (!ok) {
    *why = "cuTensorMapEncodeTiled failed (or the driver entry point is unavailable)";
    return cudaErrorInvalidValue;
  }

  KParams kp_{};
  kp_.M = a.M;
  kp_.N = a.N;
  kp_.K = a.K;
  kp_.K_out_pad = RAW ? 0 : kp;
  kp_.a_rows = a_rows;
  kp_.a_stride = geo.a_stride;
  kp_.stages = geo.stages;
  kp_.wq = static_cast<const uint8_t *>(a.Wq);
  kp_.grp = static_cast<const uint8_t *>(a.grp);
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
  cfg.dynamicSmemBytes = geo.smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 1;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = plan.split;
  // programmatic dependent launch: the CTAs may start (and stream weights)
  // while the preceding kernel in the stream finishes; they wait for it with
  // griddepcontrol.wait before touching its outputs
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  return cudaLaunchKernelEx(&cfg, kernel, tm_a, tm_xo, tm_wo, tm_y, kp_);
}

template <int BN, bool W4, bool SM>
int max_active_clusters_variant(int split) {
  using C = Cfg<BN, W4, SM>;
  static std::atomic<uint64_t> smem_done{0};
  auto kernel = mixq_gemm_kernel<BN, W4, SM, false>;
  if (ensure_smem(kernel, max_smem<BN, W4, SM>(), smem_done) != cudaSuccess) return -1;
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(1, 1, split);
  cfg.blockDim = dim3(C::kThreads, 1, 1);
  cfg.dynamicSmemBytes = geometry<BN, W4, SM>(SM ? 16 : 4096, split).smem;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 1;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = split;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int n = -1;
  if (cudaOccupancyMaxActiveClusters(&n, kernel, &cfg) != cudaSuccess) return -1;
  return n;
}

}  // namespace

int gemm_max_active_clusters(int mode, int bn, int split, int small_m) {
  if (small_m) {
    if (bn == 32) return mode == 1 ? max_active_clusters_variant<32, true, true>(split)
                                   : max_active_clusters_variant<32, false, true>(split);
    if (bn == 64) return mode == 1 ? max_active_clusters_variant<64, true, true>(split)
                                   : max_active_clusters_variant<64, false, true>(split);
    if (bn != 128) return -1;
    return mode == 1 ? max_active_clusters_variant<128, true, true>(split)
                     : max_active_clusters_variant<128, false, true>(split);
  }
  if (bn == 256) return mode == 1 ? max_active_clusters_variant<256, true, false>(split)
                                  : max_active_clusters_variant<256, false, false>(split);
  return mode == 1 ? max_active_clusters_variant<128, true, false>(split)
                   : max_active_clusters_variant<128, false, false>(split);
}

int decode_split(int n_tiles, int KB, int num_sms) {
  // Decode-sized M is latency bound: each CTA works through its K blocks one
  // pipeline round trip at a time, so the time falls with the K blocks per
  // CTA until the fixed per-CTA cost (set-up, first load, cluster reduction)
  // dominates.  Measured on 4096/11008-wide Llama shapes (W8 and W4, M 1..64):
  // best at about 10 K blocks per CTA once at least ~0.8 CTA per SM stream,
  // and no more than two CTAs per SM (the decode variants fit two).  Smallest
  // K split (cluster size) that meets both, else the largest that fits.
  int best = 1;
  for (int s = 1; s <= 8 && s <= KB; ++s) {
    const int ctas = n_tiles * s;
    if (ctas > 2 * num_sms) break;
    best = s;
    if (ctas * 5 >= num_sms * 4 && (KB + s - 1) / s <= 11) break;
  }
  return best;
}

GemmPlan plan_gemm(int mode, int M, int N, int K, int num_sms) {
  // W4: expanded weights in tensor memory at every M (measured against the
  // smem operand on the Llama shapes: 1.4x at M = 16, 1.13x at M = 512, up to
  // 1.24x at M = 512 with N = 28672, 0-5 % at M = 2048 and 8192 with 256-token
  // tiles).  The W4 branches of the smem x smem kernel remain for the
  // narrow-tile debug launches.
  if (mode == 1) return plan_gemm_w4ts(M, N, K, num_sms);
  const int n128 = (N + 127) / 128;
  if (M <= 64) {
    const int split = decode_split(n128, K / kBlockK, num_sms);
    return GemmPlan{128, split, n128 * split, 1};
  }
  // M >= 256: the persistent CTA-pair kernel (256 x 256 tiles, two SMs per
  // tile; measured 1.3-1.5x the 128 x 128 kernel on the Llama prefill and 70B
  // shapes, M = 512..8192, even where its tiles leave pairs idle).
  const int pairs = num_sms / 2;
  const int tiles256 = (M + 255) / 256 * ((N + 255) / 256);
  if (M >= 256) {
    GemmPlan g{256, 1, 2 * (tiles256 < pairs ? tiles256 : pairs), 0, 0, 1};
    return g;
  }
  // 64 < M < 256: two 128 x 128 CTAs per SM (about 100 KB each), so one CTA's
  // epilogue overlaps the other's mainloop and the grid packs into waves
  // twice as finely.
  return GemmPlan{128, 1, (M + kTileM - 1) / kTileM * n128, 1};
}

cudaError_t launch_gemm(const GemmArgs &a, const GemmPlan &plan, cudaStream_t stream,
                        const char **why) {
  if (a.mode == 1 && plan.pair) return launch_gemm_pair_w4(a, stream, why);
  if (a.mode == 1 && plan.ts) return launch_gemm_w4ts(a, plan, stream, why);
  if (a.mode == 0 && plan.pair) return launch_gemm_pair(a, stream, why);
  const bool w4 = a.mode == 1;
  const bool raw = a.epi == Epi::kRawI32;
#define MIXQ_DISPATCH(BN_, SM_)                                                      \
  if (w4) return raw ? launch_variant<BN_, true, SM_, true>(a, plan, stream, why)   \
                     : launch_variant<BN_, true, SM_, false>(a, plan, stream, why); \
  return raw ? launch_variant<BN_, false, SM_, true>(a, plan, stream, why)          \
             : launch_variant<BN_, false, SM_, false>(a, plan, stream, why);
  if (plan.small_m) {
    if (plan.bn == 32) { MIXQ_DISPATCH(32, true) }
    if (plan.bn == 64) { MIXQ_DISPATCH(64, true) }
    MIXQ_DISPATCH(128, true)
  }
  if (plan.bn == 256) { MIXQ_DISPATCH(256, false) }
  MIXQ_DISPATCH(128, false)
#undef MIXQ_DISPATCH
}

}  // namespace mixq
