// W4A8 GEMM of the MixQ layer for 4-bit weights of reading B (sm_100a): a real
// fp16 scale s and an integer zero point z per weight row and group of 128 K.
//
//   P[n,m,g] = sum_{k in g} (q[n,k] - z[n,g]) Xq[m,k]   tcgen05.mma kind::i8,
//                                                         exact INT32 per group
//   acc[n,m] = sum_g s[n,g] * float(P[n,m,g])           fp32, groups in K order
//                                                         (K split: per CTA, then
//                                                         the CTAs in rank order)
//   o[n,m]   = sum_j W_out[n,j] X_out[m,j]              tcgen05.mma kind::f16
//   Y[m,n]   = fp16(acc * s_x[m] + o)
//
// (MixLLM page, "MixLLM: Ein neuer Ansatz": 8-bit activations, asymmetric
// group-wise 4-bit weights, a two-step dequantization that keeps the products
// on INT8 tensor cores, and a fast integer-to-float conversion of the results;
// MixQ article "一键部署LLM混合精度推理…", 研究背景 Fig. 5 and MixQ的解决方案
// Fig. 12 for the FP16 outlier product added in the epilogue.)
//
// Step one of the dequantization is the expansion of reading A's kernel with
// the group scale fixed at 1: each byte (q + 128 - z) ^ 0x80 is the INT8
// operand q - z in [-15, 15], four codes per 32-bit add.  Step two needs one
// INT32 result per group, so the accumulator cannot run over all of K in
// tensor memory: every group's four MMAs write a fresh INT32 partial tile (two
// tiles, used in turn), and four drain warps convert each partial to fp32 and
// accumulate s * P in registers while the tensor core fills the other tile.
// The conversion adds the integer to the bit pattern of 1.5 * 2^23 and
// subtracts that float: the floats in [2^23, 2^24) are exactly the integers,
// so the result is exact for |P| < 2^22 (here |P| <= 128 * 127 * 15).
//
// One CTA (384 threads) computes a 128-weight-row x BT-token tile over a K
// range: one CTA per SM with 512 TMEM columns and BT = 16..64, or, for at most
// 16 tokens, two per SM with 256 columns and half the shared memory each (the
// decode variant: a K split of its few tiles over clusters then keeps about a
// CTA per SM streaming weights):
//   warp 0 lane 0   producer: packed codes + (s, z) pairs by bulk copy, token
//                   tiles by TMA (128-byte swizzle), outlier stages (W_out and
//                   X_out tiles, 64-byte swizzle)
//   warp 1 lane 0   MMA issuer: per group 4 TS MMAs into partial tile g % 2 and
//                   a commit; 2 SS MMAs per outlier stage
//   warps 2..3      token scales into shared memory
//   warps 4..7      expansion: thread = weight row = TMEM lane, into a ring of
//                   TMEM A stages
//   warps 8..11     drain: thread = weight row, BT fp32 sums in registers;
//                   then the epilogue
// K split over a thread-block cluster when the tiles leave SMs idle: every CTA
// stores its fp32 sums token-major in shared memory and the cluster reduces
// them through distributed shared memory in rank order (deterministic).
// Every mbarrier wait is bounded; a wait that runs out records
// MIXQ_ERR_TIMEOUT in *status and the CTA winds down.
#include <cuda_fp16.h>

#include <atomic>

#include "gemm_w4b.h"
#include "ptx.cuh"
#include "tma_host.h"

namespace mixq {
namespace {

constexpr int kBThreads = 384;   // warps 0-3 roles, 4-7 expansion, 8-11 drain
constexpr int kBMaxStages = 12;
constexpr int kBPacked = 128 * (kBlockK / 2);  // 8 KB of codes per 128 x 128 block
constexpr int kBGrp = 128 * 4;                  // (s, z) fp16 pair per row
constexpr int kBOutK = 32;                      // fp16 K per outlier stage (64 bytes)
constexpr int kBWOut = 128 * kBOutK * 2;        // W_out tile of an outlier stage
constexpr int kBMaxTokens = 64;                 // tokens per tile (MMA N) at most
constexpr int kBExtra = 1024 + 4 * kBMaxTokens;  // barriers, s_x[BT]
constexpr int kBPitch = 128 + 4;                 // floats per token row of a partial tile
constexpr int kBSmallMaxTokens = 16;             // tokens per tile of the two-CTA variant

// One CTA per SM (512 TMEM columns, all of shared memory), or -- SM2, decode-
// sized M -- two per SM with half of each, so that a K split of the few
// output tiles still has one CTA per SM beside it (and a CTA of the next
// kernel can start there).  TMEM: INT32 partial tile b at column kPartCol b,
// the FP32 outlier accumulator at kF32Col, the A ring from kACol.
template <bool SM2>
struct BCfg {
  static constexpr int kMinBlocks = SM2 ? 2 : 1;
  static constexpr int kSmemMax = SM2 ? 233472 / 2 - 1024 : 232448;
  static constexpr int kTmemCols = SM2 ? 256 : 512;
  static constexpr int kPartCol = SM2 ? 32 : 64;
  static constexpr int kF32Col = SM2 ? 64 : 128;
  static constexpr int kACol = SM2 ? 128 : 256;
  static constexpr int kMaxTokens = SM2 ? kBSmallMaxTokens : kBMaxTokens;
};

// Stage layout as in reading A's kernel: [codes: kbpj x 8 KB][pairs: kbpj x
// 512 B] padded to 1 KB (= w_slot), then the token tiles [kbpj][BT x 128 B].
struct BParams {
  int M, N, K, K_out_pad;
  int kbpj;         // K blocks (= groups) per job (1 or 2)
  int stages;       // shared-memory ring depth (>= a_stages)
  int stage_bytes;  // w_slot + kbpj * BT * 128
  int w_slot;       // bytes before the token tiles
  int a_stages;     // TMEM A ring depth (32 * kbpj columns each)
  const uint8_t *wq;   // tiled 4-bit codes: [N/128][K/128] tiles of 128 rows x 64 bytes
  const uint8_t *grp;  // [K/128][N] (s, z) fp16 pairs
  const float *s_x;
  const int32_t *flags;
  __half *Y;  // [M][ldy]
  int ldy;
  int32_t *status;
  uint64_t wait_limit_ns;
  int w_streamed;  // weights are read by one CTA only: evict them from L2 first
};

__device__ __forceinline__ void b_fail(int *s_err, int32_t *status) {
  atomicOr(s_err, 1);
  record_error(status, kErrTimeout);
}

__device__ __forceinline__ bool b_warp_wait(uint64_t *bar, uint32_t parity, uint64_t limit_ns) {
  return __all_sync(0xFFFFFFFFu, mbar_wait(bar, parity, limit_ns));
}

__device__ __forceinline__ int b_outliers_present(const BParams &p) {
  if (p.K_out_pad == 0) return 0;
  return p.flags ? (*reinterpret_cast<const volatile int32_t *>(p.flags) > 0) : 1;
}

// Exact int32 -> fp32 for |v| < 2^22 with one integer add and one float
// subtraction (see the file comment).
__device__ __forceinline__ float b_exact_i2f(uint32_t v) {
  return __fsub_rn(__uint_as_float(v + 0x4B400000u), 12582912.0f);
}

// The group scale s of a packed (s, z) pair (s in the low half).
__device__ __forceinline__ float b_pair_scale(uint32_t pair) {
  return __half2float(__ushort_as_half(static_cast<unsigned short>(pair & 0xFFFFu)));
}

// 4 chunks (K 0..127 of a block) of one weight row's code bytes -> 32 words of
// INT8 weights q - z, word t holding K 4t .. 4t+3.  Chunk c word w: low
// nibbles = K 32c+8w+0..3, high nibbles = K 32c+8w+4..7.  Each byte
// q + 128 - z lies in [113, 143]: the add never carries between bytes.
__device__ __forceinline__ void b_expand_block(const uint8_t *codes, const uint8_t *pairs,
                                               int row, int psw, uint32_t (&wv)[32]) {
  uint4 pk[4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
    pk[i] = *reinterpret_cast<const uint4 *>(codes + row * 64 + ((i ^ psw) << 4));
  const uint32_t pr = reinterpret_cast<const uint32_t *>(pairs)[row];
  const uint32_t z = static_cast<uint32_t>(
      __half2float(__ushort_as_half(static_cast<unsigned short>(pr >> 16))));
  const uint32_t cst = (128u - z) * 0x01010101u;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const uint32_t q4[4] = {pk[i].x, pk[i].y, pk[i].z, pk[i].w};
#pragma unroll
    for (int w = 0; w < 4; ++w) {
      wv[8 * i + 2 * w] = ((q4[w] & 0x0F0F0F0Fu) + cst) ^ 0x80808080u;
      wv[8 * i + 2 * w + 1] = (((q4[w] >> 4) & 0x0F0F0F0Fu) + cst) ^ 0x80808080u;
    }
  }
}

struct BRing {
  int slot = 0;
  uint32_t phase = 0;
  __device__ __forceinline__ void advance(int n) {
    if (++slot == n) {
      slot = 0;
      phase ^= 1u;
    }
  }
};

template <int NCH, bool SM2>
__global__ void __launch_bounds__(kBThreads, BCfg<SM2>::kMinBlocks)
    mixq_w4b_kernel(const __grid_constant__ CUtensorMap tm_a,   // Xq [M][K] int8, box {128, BT}
                    const __grid_constant__ CUtensorMap tm_xo,  // X_out [M][K_out_pad], box {32, BT}
                    const __grid_constant__ CUtensorMap tm_wo,  // W_out [N][K_out_pad], box {32, 128}
                    const __grid_constant__ CUtensorMap tm_y,   // Y [M][ldy] fp16, box {64, BT}
                    const BParams p) {
  using C = BCfg<SM2>;
  constexpr int BT = 16 * NCH;
  static_assert(BT <= C::kMaxTokens && BT <= C::kPartCol, "token tile of the variant");
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const int stages = p.stages;
  const int kbpj = SM2 ? 1 : p.kbpj;  // SM2: one K block per job (register budget)
  auto stage = [&](int s) { return smem + s * p.stage_bytes; };
  uint8_t *extra = smem + stages * p.stage_bytes;
  uint64_t *bars = reinterpret_cast<uint64_t *>(extra);
  uint64_t *wfull = bars;                     // codes + pairs (or W_out) landed
  uint64_t *tfull = bars + kBMaxStages;       // token tile(s) (Xq or X_out) landed
  uint64_t *empty = bars + 2 * kBMaxStages;   // 4 expansion-warp arrivals + MMA commit
  uint64_t *afull = bars + 3 * kBMaxStages;   // TMEM A stage written (4 warp arrivals)
  uint64_t *part_full = bars + 4 * kBMaxStages;  // [2] partial tile written (MMA commit)
  uint64_t *part_empty = part_full + 2;          // [2] partial tile read (4 drain warps)
  uint64_t *accum_full = part_empty + 2;
  uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(accum_full + 1);
  int *s_misc = reinterpret_cast<int *>(tmem_holder + 1);  // err, weights issued, tokens issued
  float *s_sx = reinterpret_cast<float *>(extra + 1024);   // [BT]

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int m0 = blockIdx.x * BT;
  const int n0 = blockIdx.y * 128;
  const int S = gridDim.z;
  const int rank = blockIdx.z;
  const int KB = p.K / kBlockK;
  const int kb_begin = static_cast<int>(static_cast<long long>(rank) * KB / S);
  const int kb_end = static_cast<int>(static_cast<long long>(rank + 1) * KB / S);
  const int n_grp = kb_end - kb_begin;                      // groups of this CTA
  const int n_i8 = (n_grp + kbpj - 1) / kbpj;               // INT8 jobs, then outlier jobs
  const int pre = n_i8 < stages ? n_i8 : stages;
  const uint32_t tok_bytes = static_cast<uint32_t>(BT) * kBlockK;
  const size_t wtile0 = static_cast<size_t>(n0 / 128) * KB;
  auto job_kb = [&](int j) { return kb_begin + j * kbpj; };
  auto job_nkb = [&](int j) { return min(kbpj, kb_end - job_kb(j)); };
  auto issue_w = [&](int j, int s, uint64_t pol) {
    const int kb = job_kb(j), nkb = job_nkb(j);
    mbar_arrive_expect_tx(&wfull[s], nkb * (kBPacked + kBGrp));
    bulk_load(stage(s), p.wq + (wtile0 + kb) * kBPacked, nkb * kBPacked, &wfull[s], pol);
    for (int kk = 0; kk < nkb; ++kk)
      bulk_load(stage(s) + kbpj * kBPacked + kk * kBGrp,
                p.grp + (static_cast<size_t>(kb + kk) * p.N + n0) * 4, kBGrp, &wfull[s], pol);
  };
  auto issue_t = [&](int j, int s, uint64_t pol) {
    const int kb = job_kb(j), nkb = job_nkb(j);
    mbar_arrive_expect_tx(&tfull[s], nkb * tok_bytes);
    for (int kk = 0; kk < nkb; ++kk)
      tma_load_2d(stage(s) + p.w_slot + kk * tok_bytes, &tm_a, &tfull[s], (kb + kk) * kBlockK, m0,
                  pol);
  };

  if (threadIdx.x == 0) {
    for (int i = 0; i < stages; ++i) {
      mbar_init(&wfull[i], 1);
      mbar_init(&tfull[i], 1);
      mbar_init(&empty[i], 4 + 1);
    }
    for (int a = 0; a < p.a_stages; ++a) mbar_init(&afull[a], 4);
    for (int b = 0; b < 2; ++b) {
      mbar_init(&part_full[b], 1);
      mbar_init(&part_empty[b], 4);
    }
    mbar_init(accum_full, 1);
    fence_mbar_init();
    s_misc[0] = 0;
    // the weights do not depend on the preceding kernel: stream them first
    const uint64_t pol_w = p.w_streamed ? policy_evict_first() : policy_evict_last();
    for (int j = 0; j < pre; ++j) issue_w(j, j, pol_w);
    s_misc[1] = pre;
    s_misc[2] = 0;
    tma_prefetch_desc(&tm_a);
    if (p.K_out_pad > 0 && rank == 0) {
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
  const uint32_t t_part = tmem_base;
  const uint32_t t_f32 = tmem_base + C::kF32Col;
  const uint32_t t_a = tmem_base + C::kACol;
  const uint32_t a_cols = 32u * kbpj;
  int *s_err = &s_misc[0];
  float acc[BT];  // drain warps: fp32 sums of the thread's weight row
#pragma unroll
  for (int i = 0; i < BT; ++i) acc[i] = 0.f;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      const uint64_t pol_a = policy_evict_last();
      const uint64_t pol_w = p.w_streamed ? policy_evict_first() : policy_evict_last();
      griddep_wait();
      // the token tiles of the early stages go out before the flags word is
      // read: queued behind the weight stream, that read takes microseconds
      for (int j = 0; j < pre; ++j) issue_t(j, j, pol_a);
      s_misc[2] = pre;
      const int n_out = (b_outliers_present(p) && rank == 0) ? p.K_out_pad / kBOutK : 0;
      const int njobs = n_i8 + n_out;
      BRing r;
      r.slot = pre == stages ? 0 : pre;
      r.phase = pre == stages ? 1u : 0u;
      for (int j = pre; j < njobs; ++j) {
        const int s = r.slot;
        if (!mbar_wait(&empty[s], r.phase ^ 1, p.wait_limit_ns)) {
          b_fail(s_err, p.status);
          break;
        }
        if (j < n_i8) {
          issue_w(j, s, pol_w);
          s_misc[1] = j + 1;
          issue_t(j, s, pol_a);
        } else {
          const int o = j - n_i8;
          mbar_arrive_expect_tx(&wfull[s], kBWOut);
          tma_load_2d(stage(s), &tm_wo, &wfull[s], o * kBOutK, n0, pol_w);
          s_misc[1] = j + 1;
          mbar_arrive_expect_tx(&tfull[s], static_cast<uint32_t>(BT) * kBOutK * 2);
          tma_load_2d(stage(s) + p.w_slot, &tm_xo, &tfull[s], o * kBOutK, m0, pol_a);
        }
        s_misc[2] = j + 1;
        r.advance(stages);
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------- MMA issuer
    if (lane == 0) {
      const uint32_t id_i8 = idesc_s8_s32(128, BT);
      const uint32_t id_f16 = idesc_f16_f32(128, BT);
      griddep_wait();
      // the INT8 jobs first: the flags word (is there an outlier slice) is
      // read once they are issued, off the path of the first MMAs
      int njobs = n_i8;
      bool counted = false;
      BRing r, ra;
      int gi = 0;  // group of this CTA's K range
      bool ok = true;
      for (int j = 0; ok; ++j) {
        if (j == njobs) {
          if (counted) break;
          counted = true;
          njobs += (b_outliers_present(p) && rank == 0) ? p.K_out_pad / kBOutK : 0;
          if (j == njobs) break;
        }
        const int s = r.slot;
        if (j < n_i8) {
          if (!mbar_wait(&tfull[s], r.phase, p.wait_limit_ns) ||
              !mbar_wait(&afull[ra.slot], ra.phase, p.wait_limit_ns)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t ta = t_a + ra.slot * a_cols;
          const uint64_t bd = sw128_kmajor_desc(smem_u32(stage(s) + p.w_slot));
          const int nkb = job_nkb(j);
          for (int kk = 0; kk < nkb; ++kk, ++gi) {
            const int b = gi & 1;
            // use u = gi / 2 of partial tile b: the drain must have read use u - 1
            if (gi >= 2) {
              if (!mbar_wait(&part_empty[b], ((gi >> 1) - 1) & 1, p.wait_limit_ns)) {
                ok = false;
                break;
              }
              tc_fence_after();
            }
            const uint64_t bdk = bd + static_cast<uint64_t>(kk * tok_bytes >> 4);
#pragma unroll
            for (int k = 0; k < 4; ++k)
              mma_i8_ts(t_part + b * C::kPartCol, ta + kk * 32 + k * 8, bdk + 2 * k, id_i8,
                        k > 0 ? 1u : 0u);
            mma_commit(&part_full[b]);
          }
          if (!ok) break;
          ra.advance(p.a_stages);
        } else {
          if (!mbar_wait(&wfull[s], r.phase, p.wait_limit_ns) ||
              !mbar_wait(&tfull[s], r.phase, p.wait_limit_ns)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t ad = sw64_kmajor_desc(smem_u32(stage(s)));
          const uint64_t bd = sw64_kmajor_desc(smem_u32(stage(s) + p.w_slot));
#pragma unroll
          for (int k = 0; k < 2; ++k)
            mma_f16(t_f32, ad + 2 * k, bd + 2 * k, id_f16, (j > n_i8 || k > 0) ? 1u : 0u);
        }
        // frees the shared-memory stage and, for INT8 jobs, the TMEM A stage
        mma_commit(&empty[s]);
        r.advance(stages);
      }
      if (!ok) b_fail(s_err, p.status);
      mma_commit(accum_full);
    }
  } else if (warp == 2 || warp == 3) {
    // ------------------------------------------------ token scales, early
    griddep_wait();
    for (int i = threadIdx.x - 64; i < BT; i += 64) s_sx[i] = m0 + i < p.M ? p.s_x[m0 + i] : 0.f;
  } else if (warp < 8) {
    // ------------------------------------------- 4-bit -> INT8 expansion
    const int row = (warp & 3) * 32 + lane;
    const uint32_t lane_addr = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const int psw = (row >> 1) & 3;
    bool ok = true;
    BRing r, ra, rf;
    for (int j = 0; j < n_i8; ++j) {
      const int s = r.slot;
      if (!b_warp_wait(&wfull[s], r.phase, p.wait_limit_ns)) {
        ok = false;
        break;
      }
      const uint8_t *sp = stage(s);
      const int nkb = job_nkb(j);
      uint32_t wv0[32], wv1[32];
      b_expand_block(sp, sp + kbpj * kBPacked, row, psw, wv0);
      if (nkb == 2) b_expand_block(sp + kBPacked, sp + kbpj * kBPacked + kBGrp, row, psw, wv1);
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[s]);
      r.advance(stages);
      if (j >= p.a_stages) {
        // A stage j % a_stages was last read by job j - a_stages, whose commit
        // completes that job's phase of empty[] (stages >= a_stages keeps the
        // phase unambiguous)
        if (!b_warp_wait(&empty[rf.slot], rf.phase, p.wait_limit_ns)) {
          ok = false;
          break;
        }
        rf.advance(stages);
      }
      tc_fence_after();
      const uint32_t ta = t_a + lane_addr + ra.slot * a_cols;
      tmem_st32(ta, wv0);
      if (nkb == 2) tmem_st32(ta + 32, wv1);
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&afull[ra.slot]);
      ra.advance(p.a_stages);
    }
    if (ok) {
      griddep_wait();
      const int n_out = (b_outliers_present(p) && rank == 0) ? p.K_out_pad / kBOutK : 0;
      for (int j = n_i8; j < n_i8 + n_out; ++j) {
        // outlier stages: release each stage only once its tiles are there
        if (!b_warp_wait(&wfull[r.slot], r.phase, p.wait_limit_ns)) {
          ok = false;
          break;
        }
        if (lane == 0) mbar_arrive(&empty[r.slot]);
        r.advance(stages);
      }
    }
    if (!ok) b_fail(s_err, p.status);
  } else {
    // ------------------------------------------------ drain: s * float(P)
    const int row = (warp & 3) * 32 + lane;
    const uint32_t lane_addr = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const uint32_t *pairs = reinterpret_cast<const uint32_t *>(p.grp) + n0 + row;
    // the scales do not depend on the preceding kernel; two groups are loaded ahead
    float s_cur = b_pair_scale(__ldg(pairs + static_cast<size_t>(kb_begin) * p.N));
    float s_nxt = n_grp > 1 ? b_pair_scale(__ldg(pairs + static_cast<size_t>(kb_begin + 1) * p.N))
                            : 0.f;
    bool ok = true;
    for (int gi = 0; gi < n_grp; ++gi) {
      const float s_g = s_cur;
      s_cur = s_nxt;
      if (gi + 2 < n_grp)
        s_nxt = b_pair_scale(__ldg(pairs + static_cast<size_t>(kb_begin + gi + 2) * p.N));
      const int b = gi & 1;
      if (!b_warp_wait(&part_full[b], (gi >> 1) & 1, p.wait_limit_ns)) {
        ok = false;
        break;
      }
      tc_fence_after();
      uint32_t v[NCH][16];
#pragma unroll
      for (int c = 0; c < NCH; ++c) tmem_ld16(t_part + b * C::kPartCol + lane_addr + c * 16, v[c]);
      tmem_ld_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&part_empty[b]);
#pragma unroll
      for (int c = 0; c < NCH; ++c)
#pragma unroll
        for (int i = 0; i < 16; ++i)
          acc[c * 16 + i] = __fmaf_rn(s_g, b_exact_i2f(v[c][i]), acc[c * 16 + i]);
    }
    if (!ok) b_fail(s_err, p.status);
  }
  __syncwarp();

  // ---------------------------------------------------------------- epilogue
  griddep_wait();
  const int any_out = b_outliers_present(p);
  const bool do_out = any_out && rank == 0;
  if (!mbar_wait_sleep(accum_full, 0, p.wait_limit_ns)) b_fail(s_err, p.status);
  tc_fence_after();
  __syncthreads();
  const bool failed = *s_err != 0;
  const bool drain = warp >= 8;
  const int row = (warp & 3) * 32 + lane;  // weight row n0 + row = TMEM lane
  const uint32_t lane_addr = static_cast<uint32_t>((warp & 3) * 32) << 16;

  if (S == 1) {
    // fp16 tile staged in shared memory as two 64-column TMA-store boxes in the
    // 128-byte swizzle (box t holds weight rows 64t..64t+63 as columns)
    uint8_t *stage_y = smem;  // the ring is free: every MMA has completed
    if (drain && !failed) {
      uint8_t *box = stage_y + (row >> 6) * BT * 128;
      const int chunk = (row & 63) >> 3, within = (row & 7) * 2;
#pragma unroll
      for (int c = 0; c < NCH; ++c) {
        uint32_t o[16];
        if (do_out) {
          tmem_ld16(t_f32 + lane_addr + c * 16, o);
          tmem_ld_wait();
        }
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const int m = c * 16 + i;
          float y = __fmul_rn(acc[m], s_sx[m]);
          if (do_out) y = __fadd_rn(y, __uint_as_float(o[i]));
          *reinterpret_cast<__half *>(box + m * 128 + ((chunk ^ (m & 7)) << 4) + within) =
              __float2half_rn(y);
        }
      }
      fence_proxy_async_smem();
    }
    __syncthreads();
    if (threadIdx.x == 0 && !failed) {
      tma_store_2d(&tm_y, stage_y, n0, m0);
      tma_store_2d(&tm_y, stage_y + BT * 128, n0 + 64, m0);
      bulk_commit_group();
      bulk_wait_all();
    }
  } else {
    // ------------------------------------ K split: reduce across the cluster
    float *pbuf = reinterpret_cast<float *>(smem);
    float *obuf = pbuf + BT * kBPitch;
    const int rows_valid = min(BT, p.M - m0);
    if (drain && !failed) {
#pragma unroll
      for (int c = 0; c < NCH; ++c) {
        uint32_t o[16];
        if (do_out) {
          tmem_ld16(t_f32 + lane_addr + c * 16, o);
          tmem_ld_wait();
        }
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const int m = c * 16 + i;
          if (m < rows_valid) {
            pbuf[m * kBPitch + row] = acc[m];
            if (do_out) obuf[m * kBPitch + row] = __uint_as_float(o[i]);
          }
        }
      }
    }
    cluster_sync_all();
    if (!failed) {
      // this CTA reduces weight rows [c_begin, c_end) of the tile, ranks in order
      const int my_rank = static_cast<int>(cluster_ctarank());
      const int c_begin = my_rank * 32 / S * 4;
      const int c_end = (my_rank + 1) * 32 / S * 4;
      const int c4n = (c_end - c_begin) / 4;
#pragma unroll 1
      for (int e = threadIdx.x; e < rows_valid * c4n; e += kBThreads) {
        const int m = e / c4n;
        const int col = c_begin + (e % c4n) * 4;
        const uint32_t off = smem_u32(pbuf + m * kBPitch + col);
        int4 part[8];
#pragma unroll
        for (int q = 0; q < 8; ++q)
          if (q < S) part[q] = ld_dsmem_v4(mapa_shared(off, static_cast<uint32_t>(q)));
        int4 oi = make_int4(0, 0, 0, 0);
        if (any_out) oi = ld_dsmem_v4(mapa_shared(smem_u32(obuf + m * kBPitch + col), 0u));
        float sum[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          if (q < S) {
            sum[0] = __fadd_rn(sum[0], __int_as_float(part[q].x));
            sum[1] = __fadd_rn(sum[1], __int_as_float(part[q].y));
            sum[2] = __fadd_rn(sum[2], __int_as_float(part[q].z));
            sum[3] = __fadd_rn(sum[3], __int_as_float(part[q].w));
          }
        }
        const float ov[4] = {__int_as_float(oi.x), __int_as_float(oi.y), __int_as_float(oi.z),
                             __int_as_float(oi.w)};
        const float sx = s_sx[m];
        float y[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          float v = __fmul_rn(sum[i], sx);
          if (any_out) v = __fadd_rn(v, ov[i]);
          y[i] = v;
        }
        const __half2 h0 = __floats2half2_rn(y[0], y[1]);
        const __half2 h1 = __floats2half2_rn(y[2], y[3]);
        *reinterpret_cast<uint2 *>(p.Y + static_cast<size_t>(m0 + m) * p.ldy + n0 + col) =
            make_uint2(*reinterpret_cast<const uint32_t *>(&h0),
                       *reinterpret_cast<const uint32_t *>(&h1));
      }
    }
    cluster_sync_all();
  }

  // ---------------------------------------------------------------- teardown
  tc_fence_before();
  __syncthreads();
  if (failed && threadIdx.x == 0) {
    // let every copy still in flight land before the shared memory is released
    const int wi = s_misc[1], ti = s_misc[2];
    for (int j = wi > stages ? wi - stages : 0; j < wi; ++j)
      mbar_wait(&wfull[j % stages], (j / stages) & 1, p.wait_limit_ns);
    for (int j = ti > stages ? ti - stages : 0; j < ti; ++j)
      mbar_wait(&tfull[j % stages], (j / stages) & 1, p.wait_limit_ns);
  }
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, C::kTmemCols);
  }
}

// ------------------------------------------------------------------ host side
struct BGeometry {
  int bt, kbpj, w_slot, stages, stage_bytes, a_stages, smem;
};

int b_tokens(int M) {
  const int bt = M >= kBMaxTokens ? kBMaxTokens : (M + 15) / 16 * 16;
  return bt < 16 ? 16 : bt;
}

template <bool SM2>
BGeometry b_geometry(int M) {
  using C = BCfg<SM2>;
  BGeometry g{};
  g.bt = b_tokens(M);
  // two K blocks per job unless that leaves fewer than three stages; the
  // two-CTA variant takes one (its expansion threads have 80 registers)
  for (int kbpj = SM2 ? 1 : 2; kbpj >= 1; --kbpj) {
    g.kbpj = kbpj;
    g.w_slot = (kbpj * (kBPacked + kBGrp) + 1023) / 1024 * 1024;
    g.stage_bytes = g.w_slot + kbpj * g.bt * kBlockK;
    g.stages = (C::kSmemMax - 1024 - kBExtra) / g.stage_bytes;
    if (g.stages > kBMaxStages) g.stages = kBMaxStages;
    if (g.stages >= 3) break;
  }
  g.a_stages = (C::kTmemCols - C::kACol) / (32 * g.kbpj);
  if (g.a_stages > g.stages) g.a_stages = g.stages;
  g.smem = g.stages * g.stage_bytes + kBExtra + 1024;
  return g;
}

template <int NCH, bool SM2>
cudaError_t launch_b_variant(const GemmArgs &a, const GemmPlan &plan, const BGeometry &geo,
                             cudaStream_t stream, const char **why) {
  using C = BCfg<SM2>;
  static std::atomic<uint64_t> smem_done{0};
  auto kernel = mixq_w4b_kernel<NCH, SM2>;
  cudaError_t e = ensure_smem(kernel, C::kSmemMax, smem_done);
  if (e != cudaSuccess) return e;
  const int red_bytes = 2 * geo.bt * kBPitch * 4;
  if (geo.bt != 16 * NCH || geo.stages < 2 || geo.stages < geo.a_stages ||
      geo.a_stages > kBMaxStages || geo.smem > C::kSmemMax || geo.w_slot < kBWOut ||
      plan.split < 1 || plan.split > 8 || plan.split > a.K / kBlockK ||
      (plan.split > 1 && geo.stages * geo.stage_bytes < red_bytes) ||
      (plan.split == 1 && geo.stages * geo.stage_bytes < 2 * geo.bt * 128)) {
    *why = "no pipeline geometry fits the shared-memory budget";
    return cudaErrorInvalidValue;
  }
  const int kp = k_out_pad(a.K_out);
  alignas(64) CUtensorMap tm_a, tm_xo, tm_wo, tm_y;
  memset(&tm_xo, 0, sizeof tm_xo);
  memset(&tm_wo, 0, sizeof tm_wo);
  bool ok = make_map(&tm_a, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, a.Xq, a.K, a.M, a.K, kBlockK,
                     geo.bt, CU_TENSOR_MAP_SWIZZLE_128B);
  if (kp > 0) {
    ok = ok && make_map(&tm_xo, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, a.X_out, kp, a.M,
                        static_cast<uint64_t>(kp) * 2, kBOutK, geo.bt, CU_TENSOR_MAP_SWIZZLE_64B);
    ok = ok && make_map(&tm_wo, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, a.W_out, kp, a.N,
                        static_cast<uint64_t>(kp) * 2, kBOutK, 128, CU_TENSOR_MAP_SWIZZLE_64B);
  }
  ok = ok && make_map(&tm_y, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, a.Y, a.N, a.M,
                      static_cast<uint64_t>(a.ldy) * 2, 64, geo.bt, CU_TENSOR_MAP_SWIZZLE_128B);
  if (!ok) {
    *why = "cuTensorMapEncodeTiled failed (or the driver entry point is unavailable)";
    return cudaErrorInvalidValue;
  }

  BParams bp{};
  bp.M = a.M;
  bp.N = a.N;
  bp.K = a.K;
  bp.K_out_pad = kp;
  bp.kbpj = geo.kbpj;
  bp.stages = geo.stages;
  bp.stage_bytes = geo.stage_bytes;
  bp.w_slot = geo.w_slot;
  bp.a_stages = geo.a_stages;
  bp.wq = static_cast<const uint8_t *>(a.Wq);
  bp.grp = static_cast<const uint8_t *>(a.grp);
  bp.s_x = a.s_x;
  bp.flags = a.flags;
  bp.Y = static_cast<__half *>(a.Y);
  bp.ldy = a.ldy;
  bp.status = a.status;
  bp.wait_limit_ns = a.wait_limit_ns;
  const int m_tiles = (a.M + geo.bt - 1) / geo.bt;
  bp.w_streamed = m_tiles == 1;

  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(m_tiles, a.N / 128, plan.split);
  cfg.blockDim = dim3(kBThreads, 1, 1);
  cfg.dynamicSmemBytes = geo.smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 1;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = plan.split;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  return cudaLaunchKernelEx(&cfg, kernel, tm_a, tm_xo, tm_wo, tm_y, bp);
}

}  // namespace

GemmPlan plan_gemm_w4b(int M, int N, int K, int num_sms) {
  const int KB = K / kBlockK;
  const int bt = b_tokens(M);
  const int tiles = (M + bt - 1) / bt * (N / 128);
  if (M <= kBSmallMaxTokens) {
    // decode-sized M: the two-CTA variant, K split as for the other decode
    // kernels (about 10 K blocks per CTA once ~0.8 CTA per SM stream, at
    // most two CTAs per SM)
    const int split = decode_split(tiles, KB, num_sms);
    return GemmPlan{128, split, tiles * split, 1, 0};
  }
  // One CTA per SM.  While the output tiles leave SMs idle, split K over a
  // cluster: the smallest split giving at least 0.8 CTA per SM with at most
  // 11 K blocks per CTA, else the largest that still fits one wave.
  int best = 1;
  for (int s = 1; s <= 8 && s <= KB; ++s) {
    if (s > 1 && tiles * s > num_sms) break;
    best = s;
    if (tiles * s * 5 >= num_sms * 4 && (KB + s - 1) / s <= 11) break;
  }
  return GemmPlan{128, best, tiles * best, 0, 0};
}

cudaError_t launch_gemm_w4b(const GemmArgs &a, const GemmPlan &plan, cudaStream_t stream,
                            const char **why) {
  if (a.epi != Epi::kMixed) {
    *why = "the reading-B GEMM has no raw accumulator output";
    return cudaErrorInvalidValue;
  }
  if (plan.small_m) {
    if (a.M > kBSmallMaxTokens) {
      *why = "the two-CTA reading-B variant takes at most 16 tokens";
      return cudaErrorInvalidValue;
    }
    return launch_b_variant<1, true>(a, plan, b_geometry<true>(a.M), stream, why);
  }
  const BGeometry geo = b_geometry<false>(a.M);
  switch (geo.bt / 16) {
    case 1:
      return launch_b_variant<1, false>(a, plan, geo, stream, why);
    case 2:
      return launch_b_variant<2, false>(a, plan, geo, stream, why);
    case 3:
      return launch_b_variant<3, false>(a, plan, geo, stream, why);
    default:
      return launch_b_variant<4, false>(a, plan, geo, stream, why);
  }
}

}  // namespace mixq
