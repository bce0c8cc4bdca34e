// W4A8 GEMM of the MixQ layer for large M on CTA pairs (sm_100a, tcgen05
// cta_group::2), persistent, with the 4-bit weights expanded into tensor
// memory.
//
//   w8[n,k]  = (q[n,k] - z2[n,g]) * s2[n,g]             expansion warps, into TMEM
//   acc[n,m] = sum_k w8[n,k] Xq[m,k]                    tcgen05.mma kind::i8,
//                                                       A = weights (TMEM),
//                                                       B = tokens (smem)
//   c[n,m]   = (float(acc) * s_x[m]) * s_w[n]           epilogue warps, in TMEM
//   y[n,m]   = c + sum_j W_out[n,j] X_out[m,j]          tcgen05.mma kind::f16
//   Y[m,n]   = fp16(y)
//
// (QServe reading notes, 渐进量化 and 寄存器压力和并行性: 4-bit group codes
// expanded back to INT8 inside the mainloop, four codes per 32-bit operation,
// no intermediate overflow, every product on INT8 tensor cores; MixQ article
// "一键部署LLM混合精度推理…", 研究背景 Fig. 5 and MixQ的解决方案 Fig. 12: the FP16
// outlier product added to the dequantized, scaled INT32 result.)
//
// A pair computes a 256-weight-row x 256-token tile with MMAs of M = 256,
// N = 256: each CTA expands its own 128 weight rows into its own tensor memory
// (A) and loads its own 128 of the 256 token rows (B); the MMA reads B from
// both CTAs.  Per SM that is 8.5 KB of codes and group constants plus 16 KB of
// tokens per 128 x 256 x 128 MACs.  TMEM per CTA: one 256-column accumulator
// and a ring of four 64-column A stages (one job of two K blocks each).  The
// A ring is what hides the expansion's latency (codes -> registers -> TMEM ->
// the leader's barrier, across the pair), so it takes the columns a second
// accumulator would: the next tile's MMAs start once the epilogue has drained
// the accumulator.  N = 256 also keeps an MMA (128 cycles of tensor work per
// SM) longer than the issuing thread's cost per tcgen05 instruction.
//   warp 0 lane 0   producer (both CTAs): per job its codes and group
//                   constants (bulk copies, local barrier) and its token tiles
//                   (TMA, cta_group::2 form, leader's barrier)
//   warp 1          TMEM allocation (collective); lane 0 of the leader issues
//                   every MMA of the pair
//   warps 2..9      epilogue: warp w reads TMEM lanes 32(w%4).. (weight rows),
//                   half of the 256 token columns each
//   warps 10..17    expansion: thread = weight row = TMEM lane; warps 10..13
//                   take the even jobs, 14..17 the odd ones, both K blocks
//                   each (a TMEM store completes behind the MMAs in flight,
//                   so two groups keep two jobs' stores in flight)
// Outlier jobs (64 channels each) carry a W_out tile (A) and an X_out tile (B),
// both by TMA to the leader's barrier; the outlier product accumulates onto
// the accumulator after the epilogue has converted it in place to FP32, as in
// the 8-bit pair kernel.  Every mbarrier wait is bounded; a wait that runs out
// records MIXQ_ERR_TIMEOUT in *status and the pair winds down together.
#include <cuda_fp16.h>

#include <atomic>

#include "internal.h"
#include "ptx.cuh"
#include "tma_host.h"

namespace mixq {
namespace {

constexpr int kQThreads = 576;  // 0 producer, 1 MMA/TMEM, 2..9 epilogue, 10..17 expansion
constexpr int kQEpiWarps = 8;
constexpr int kQExpWarps = 8;
constexpr int kQGroupWarps = 4;  // expansion warps per job (two groups take alternate jobs)
constexpr int kQBT = 256;                     // tokens per pair tile (MMA N)
constexpr int kQHalf = kQBT / 2;              // token rows per CTA
constexpr int kQCodes = 128 * (kBlockK / 2);  // 8 KB of codes per 128 x 128 block
constexpr int kQGrp = 128 * 4;                // (s2, z2) fp16 pair per row and block
constexpr int kQKbJob = 2;                    // K blocks per INT8 job
constexpr int kQWSlot = kQKbJob * (kQCodes + kQGrp);  // 17 KB: codes, then constants
constexpr int kQTok = kQHalf * kBlockK;               // 16 KB token tile of one K block
constexpr int kQStage = kQWSlot + kQKbJob * kQTok;    // 49 KB
constexpr int kQStages = 4;
constexpr int kQOutTile = 128 * 128;  // W_out tile of an outlier job (64 fp16 x 128 rows)
constexpr int kQExtra = 1024 + 2 * kQBT * 4;  // barriers, s_x of two tiles
constexpr int kQTmemCols = 512;
constexpr int kQACol = kQBT;  // A ring after the accumulator
constexpr int kQAStages = 4;  // 64 columns each
static_assert(kQACol + kQAStages * 32 * kQKbJob <= kQTmemCols, "tensor memory");
// job n uses shared-memory slot n % 4 and (INT8 jobs) A stage n % 4, and is
// expanded by group n % 2: every slot and stage belongs to one group, whose
// barrier phases it therefore sees one by one
static_assert(kQAStages == kQStages && kQStages % 2 == 0, "slot and stage share the job index");
static_assert(kQWSlot % 1024 == 0 && kQStage % 1024 == 0, "swizzle atoms stay aligned");
static_assert(kQOutTile <= kQWSlot, "outlier W_out tile fits the weight slot");

struct QParams {
  int M, N, K, K_out_pad;
  int m_tiles, n_tiles, pairs;
  const uint8_t *wq;   // tiled 4-bit codes: [N/128][K/128] tiles of 128 rows x 64 bytes
  const uint8_t *grp;  // [K/128][N] (s2, z2) fp16 pairs
  const float *s_x;
  const float *s_w;
  const int32_t *flags;
  void *Y;  // fp16 [M][ldy] or int32 [M][ldy] (raw)
  int ldy;
  int32_t *status;
  uint64_t wait_limit_ns;
};

__device__ __forceinline__ void q_fail(int *s_err, int32_t *status) {
  atomicOr(s_err, 1);
  record_error(status, kErrTimeout);
}

__device__ __forceinline__ bool q_warp_wait(uint64_t *bar, uint32_t parity, uint64_t limit_ns) {
  return __all_sync(0xFFFFFFFFu, mbar_wait_sleep(bar, parity, limit_ns));
}

__device__ __forceinline__ int q_outliers(const QParams &p, bool raw) {
  if (raw || p.K_out_pad == 0) return 0;
  return p.flags ? (*reinterpret_cast<const volatile int32_t *>(p.flags) > 0) : 1;
}

// 4 codes (one byte each, low nibbles of w) -> 4 INT8 weights (q - z2) * s2,
// as the byte (q * s2 + 128 - z2 * s2) ^ 0x80; each byte's value lies in
// [0, 255], so the 32-bit multiply-add never carries between bytes.
__device__ __forceinline__ uint32_t q_expand4(uint32_t nibbles, uint32_t s2, uint32_t c) {
  return (nibbles * s2 + c) ^ 0x80808080u;
}

// One weight row's 64 code bytes of a prepacked 128 x 128 block -> 32 words of
// INT8 weights (word t = K 4t .. 4t+3).  Chunk c (16 bytes) sits at position
// c ^ ((row >> 1) & 3); its word w holds K 32c+8w+0..3 in the low nibbles and
// 32c+8w+4..7 in the high ones.
__device__ __forceinline__ void q_expand_block(const uint8_t *codes, const uint8_t *consts,
                                               int row, uint32_t (&wv)[32]) {
  const int psw = (row >> 1) & 3;
  uint4 pk[4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
    pk[i] = *reinterpret_cast<const uint4 *>(codes + row * 64 + ((i ^ psw) << 4));
  const uint32_t g = reinterpret_cast<const uint32_t *>(consts)[row];
  const uint32_t s2 = static_cast<uint32_t>(
      __half2float(__ushort_as_half(static_cast<unsigned short>(g & 0xFFFFu))));
  const uint32_t z2 = static_cast<uint32_t>(
      __half2float(__ushort_as_half(static_cast<unsigned short>(g >> 16))));
  const uint32_t cst = (128u - z2 * s2) * 0x01010101u;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const uint32_t q4[4] = {pk[i].x, pk[i].y, pk[i].z, pk[i].w};
#pragma unroll
    for (int w = 0; w < 4; ++w) {
      wv[8 * i + 2 * w] = q_expand4(q4[w] & 0x0F0F0F0Fu, s2, cst);
      wv[8 * i + 2 * w + 1] = q_expand4((q4[w] >> 4) & 0x0F0F0F0Fu, s2, cst);
    }
  }
}

// Job order of a pair (producer, MMA issuer and expansion warps walk it the
// same way): per tile iteration its INT8 jobs (two K blocks each), then, with
// outliers, its outlier jobs (one 64-channel chunk each).  f(kind, iter, job,
// n) returns false to stop.
template <typename F>
__device__ __forceinline__ void q_for_each_job(int iters, int jobs8, int kb8, int chunks_o,
                                               F &&f) {
  for (int it = 0; it < iters; ++it) {
    for (int j = 0; j < jobs8; ++j)
      if (!f(0, it, j, min(kQKbJob, kb8 - j * kQKbJob))) return;
    for (int c = 0; c < chunks_o; ++c)
      if (!f(1, it, c, 1)) return;
  }
}

template <bool RAW>
__global__ void __launch_bounds__(kQThreads, 1)
    mixq_pair_w4_kernel(const __grid_constant__ CUtensorMap tm_a,   // Xq [M][K], box {128, 96}
                        const __grid_constant__ CUtensorMap tm_xo,  // X_out [M][Kp], box {64, 96}
                        const __grid_constant__ CUtensorMap tm_wo,  // W_out [N][Kp], box {64, 128}
                        const QParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  auto stage = [&](int s) { return smem + s * kQStage; };
  uint8_t *extra = smem + kQStages * kQStage;
  uint64_t *bars = reinterpret_cast<uint64_t *>(extra);
  uint64_t *wfull = bars;                   // local: codes + constants landed
  uint64_t *tfull = wfull + kQStages;       // leader: both CTAs' B (and outlier A) tiles
  uint64_t *sempty = tfull + kQStages;      // local: codes read (8) + MMAs done (1)
  uint64_t *afull = sempty + kQStages;      // leader: both CTAs' A stage written (16)
  uint64_t *aempty = afull + kQAStages;     // [2] both: the MMAs have read the A stage
  uint64_t *acc_full = aempty + kQAStages;  // both: INT8 product of the tile done
  uint64_t *conv_done = acc_full + 1;       // leader (16): converted in place
  uint64_t *out_full = conv_done + 1;       // both: outlier product added
  uint64_t *tmem_empty = out_full + 1;      // leader (16): accumulator drained
  uint64_t *drain = tmem_empty + 1;
  uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(drain + 1);
  int *s_misc = reinterpret_cast<int *>(tmem_holder + 1);  // err, issued, consumed
  float *s_sx = reinterpret_cast<float *>(extra + 1024);   // [2][256]

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const int pair = blockIdx.x >> 1;
  const int tiles = p.m_tiles * p.n_tiles;
  const int iters = pair < tiles ? (tiles - pair + p.pairs - 1) / p.pairs : 0;
  const int KB = p.K / kBlockK;
  const int jobs8 = (KB + kQKbJob - 1) / kQKbJob;
  auto tile_of = [&](int it, int &tm, int &tn) {
    const int t = pair + it * p.pairs;
    tm = t % p.m_tiles;
    tn = t / p.m_tiles;
  };
  const uint32_t tfull_l = mapa_shared(smem_u32(tfull), 0u);
  const uint32_t afull_l = mapa_shared(smem_u32(afull), 0u);
  const uint32_t conv_l = mapa_shared(smem_u32(conv_done), 0u);
  const uint32_t tmem_empty_l = mapa_shared(smem_u32(tmem_empty), 0u);

  if (threadIdx.x == 0) {
    for (int i = 0; i < kQStages; ++i) {
      mbar_init(&wfull[i], 1);
      mbar_init(&tfull[i], 1);
      mbar_init(&sempty[i], kQGroupWarps + 1);
    }
    for (int a = 0; a < kQAStages; ++a) {
      mbar_init(&afull[a], 2 * kQGroupWarps);
      mbar_init(&aempty[a], 1);
    }
    mbar_init(acc_full, 1);
    mbar_init(conv_done, 2 * kQEpiWarps);
    mbar_init(out_full, 1);
    mbar_init(tmem_empty, 2 * kQEpiWarps);
    mbar_init(drain, 1);
    fence_mbar_init();
    s_misc[0] = 0;
    s_misc[1] = 0;
    s_misc[2] = 0;
    tma_prefetch_desc(&tm_a);
    if (!RAW && p.K_out_pad > 0) {
      tma_prefetch_desc(&tm_xo);
      tma_prefetch_desc(&tm_wo);
    }
  }
  if (warp == 1) {
    tmem_alloc_pair(tmem_holder, kQTmemCols);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();
  tc_fence_after();
  if (threadIdx.x == 0) griddep_launch_dependents();
  const uint32_t tmem_base = *tmem_holder;
  const uint32_t t_a = tmem_base + kQACol;
  int *s_err = &s_misc[0];

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0 && iters > 0) {
      const uint64_t pol = policy_evict_last();
      // the codes of this CTA's 128 weight rows, or none past the last row
      auto issue_codes = [&](int s, int tn, int j, int nkb) {
        const int nrow = 256 * tn + 128 * static_cast<int>(rank);
        if (nrow >= p.N) {
          mbar_arrive(&wfull[s]);  // nothing to load; rows past N are not stored
          return;
        }
        const int kb = j * kQKbJob;
        mbar_arrive_expect_tx(&wfull[s], nkb * (kQCodes + kQGrp));
        bulk_load(stage(s), p.wq + (static_cast<size_t>(nrow / 128) * KB + kb) * kQCodes,
                  nkb * kQCodes, &wfull[s], pol);
        for (int kk = 0; kk < nkb; ++kk)
          bulk_load(stage(s) + kQKbJob * kQCodes + kk * kQGrp,
                    p.grp + (static_cast<size_t>(kb + kk) * p.N + nrow) * 4, kQGrp, &wfull[s],
                    pol);
      };
      const int pre = min(kQStages, jobs8);
      int tm0, tn0;
      tile_of(0, tm0, tn0);
      // weights do not depend on the preceding kernel: the first stages' codes
      // go out before waiting for it
      for (int j = 0; j < pre; ++j)
        issue_codes(j, tn0, j, min(kQKbJob, KB - j * kQKbJob));
      griddep_wait();
      const int chunks_o = q_outliers(p, RAW) ? p.K_out_pad / 64 : 0;
      int slot = 0, n = 0;
      uint32_t phase = 0;
      q_for_each_job(iters, jobs8, KB, chunks_o, [&](int kind, int it, int j, int nkb) {
        int tm, tn;
        tile_of(it, tm, tn);
        const int row_t = kQBT * tm + kQHalf * static_cast<int>(rank);
        const uint32_t bar = tfull_l + 8u * slot;
        uint8_t *tok = stage(slot) + kQWSlot;
        if (n >= pre) {
          if (!mbar_wait_sleep(&sempty[slot], phase ^ 1, p.wait_limit_ns)) {
            q_fail(s_err, p.status);
            return false;
          }
        }
        if (kind == 0) {
          if (n >= pre) issue_codes(slot, tn, j, nkb);
          if (rank == 0) mbar_arrive_expect_tx(&tfull[slot], 2u * kQTok * nkb);
          for (int kk = 0; kk < nkb; ++kk)
            tma_load_2d_pair(tok + kk * kQTok, &tm_a, bar, (j * kQKbJob + kk) * kBlockK, row_t,
                             pol);
        } else {
          // outlier chunk j: W_out rows of this CTA (A) and its X_out rows (B);
          // no codes, so the stage's expansion-side arrivals come from here
          if (rank == 0) mbar_arrive_expect_tx(&tfull[slot], 2u * (kQOutTile + kQTok));
          tma_load_2d_pair(stage(slot), &tm_wo, bar, j * 64,
                           256 * tn + 128 * static_cast<int>(rank), pol);
          tma_load_2d_pair(tok, &tm_xo, bar, j * 64, row_t, pol);
          mbar_arrive(&wfull[slot]);  // every use of a slot completes one phase
          mbar_arrive_cnt(&sempty[slot], kQGroupWarps);
        }
        ++n;
        if (++slot == kQStages) {
          slot = 0;
          phase ^= 1u;
        }
        return true;
      });
      s_misc[1] = n;
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------- MMA issuer
    if (lane == 0 && rank == 0 && iters > 0) {
      constexpr uint32_t kIdI8 = idesc_s8_s32(256, kQBT);
      constexpr uint32_t kIdF16 = idesc_f16_f32(256, kQBT);
      const uint64_t bd0 = sw128_kmajor_desc(smem_u32(stage(0) + kQWSlot));
      const uint64_t od0 = sw128_kmajor_desc(smem_u32(stage(0)));
      constexpr uint64_t kStageD = kQStage >> 4, kTokD = kQTok >> 4;
      griddep_wait();
      const int chunks_o = q_outliers(p, RAW) ? p.K_out_pad / 64 : 0;
      int slot = 0, n = 0;
      uint32_t phase = 0, aph = 0;  // aph: phase bit of each A stage (INT8 uses only)
      bool ok = true;
      q_for_each_job(iters, jobs8, KB, chunks_o, [&](int kind, int it, int j, int nkb) {
        const uint32_t use = static_cast<uint32_t>(it);
        const int as = slot;
        if (kind == 0 && j == 0 && it >= 1) {
          // the previous tile's accumulator has been drained by both CTAs
          if (!mbar_wait_sleep(tmem_empty, (use - 1) & 1, p.wait_limit_ns)) return ok = false;
          tc_fence_after();
        }
        if (kind == 1 && j == 0) {
          if (!mbar_wait_sleep(conv_done, use & 1, p.wait_limit_ns)) return ok = false;
          tc_fence_after();
        }
        if (!mbar_try_wait(&tfull[slot], phase) && !mbar_wait(&tfull[slot], phase, p.wait_limit_ns))
          return ok = false;
        const uint32_t d = tmem_base;
        if (kind == 0) {
          const uint32_t ap = (aph >> as) & 1u;
          if (!mbar_try_wait(&afull[as], ap) && !mbar_wait(&afull[as], ap, p.wait_limit_ns))
            return ok = false;
          tc_fence_after();
          const uint64_t bd = bd0 + slot * kStageD;
          const uint32_t ta = t_a + static_cast<uint32_t>(as * 32 * kQKbJob);
          for (int kk = 0; kk < nkb; ++kk) {
#pragma unroll
            for (int k = 0; k < 4; ++k)
              mma_i8_pair_ts(d, ta + kk * 32 + k * 8, bd + kk * kTokD + 2 * k, kIdI8,
                             (j > 0 || kk > 0 || k > 0) ? 1u : 0u);
          }
          mma_commit_pair(&aempty[as], 3);
          aph ^= 1u << as;
        } else {
          tc_fence_after();
          const uint64_t ad = od0 + slot * kStageD, bd = bd0 + slot * kStageD;
#pragma unroll
          for (int k = 0; k < 4; ++k) mma_f16_pair(d, ad + 2 * k, bd + 2 * k, kIdF16, 1u);
        }
        mma_commit_pair(&sempty[slot], 3);
        if (kind == 0 && j == jobs8 - 1) mma_commit_pair(acc_full, 3);
        if (kind == 1 && j == chunks_o - 1) mma_commit_pair(out_full, 3);
        ++n;
        if (++slot == kQStages) {
          slot = 0;
          phase ^= 1u;
        }
        return true;
      });
      s_misc[2] = n;
      if (!ok) {
        q_fail(s_err, p.status);
        mma_commit_pair(drain, 1);
        mbar_wait(drain, 0, p.wait_limit_ns);
      }
    }
  } else if (warp >= 10) {
    // ------------------------------------------- 4-bit -> INT8 expansion
    // Two groups of four warps take alternate jobs (storing to TMEM waits
    // behind the MMAs in flight, so a group keeps one job's store in flight
    // while the other expands the next job); a warp expands both K blocks of
    // its job for its 32 weight rows.
    const int row = (warp & 3) * 32 + lane;  // weight row of this CTA's 128 = TMEM lane
    const int grp = (warp - 10) >> 2;        // jobs n with n % 2 == grp
    const uint32_t lane_addr = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const uint32_t afull_w = afull_l;
    int slot = 0, n = 0;
    uint32_t phase = 0, aph = 0;  // aph: phase bit of each A stage (INT8 uses only)
    bool ok = true;
    if (iters > 0) {
      griddep_wait();
      const int chunks_o = q_outliers(p, RAW) ? p.K_out_pad / 64 : 0;
      q_for_each_job(iters, jobs8, KB, chunks_o, [&](int kind, int it, int j, int nkb) {
        (void)it;
        (void)j;
        if ((n & 1) == grp) {
          // an outlier job's stage carries no codes, but its phase of wfull is
          // waited for all the same: a group that skipped it could run two
          // phases ahead of the barrier, where a parity wait cannot tell them apart
          if (!q_warp_wait(&wfull[slot], phase, p.wait_limit_ns)) return ok = false;
          if (kind == 0) {
            const int as = slot;
            const uint8_t *sp = stage(slot);
            uint32_t wv0[32], wv1[32];
            q_expand_block(sp, sp + kQKbJob * kQCodes, row, wv0);
            if (nkb > 1) q_expand_block(sp + kQCodes, sp + kQKbJob * kQCodes + kQGrp, row, wv1);
            __syncwarp();
            if (lane == 0) mbar_arrive(&sempty[slot]);  // codes read
            // A stage `as` was last read by the MMAs of this group's job kQAStages jobs ago
            if (!q_warp_wait(&aempty[as], ((aph >> as) & 1u) ^ 1u, p.wait_limit_ns))
              return ok = false;
            tc_fence_after();
            const uint32_t ta = t_a + lane_addr + static_cast<uint32_t>(as * 32 * kQKbJob);
            tmem_st32(ta, wv0);
            if (nkb > 1) tmem_st32(ta + 32, wv1);
            tmem_st_wait();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_cluster(afull_w + 8u * as);
            aph ^= 1u << as;
          }
        }
        ++n;
        if (++slot == kQStages) {
          slot = 0;
          phase ^= 1u;
        }
        return true;
      });
    }
    if (!ok) q_fail(s_err, p.status);
  } else if (warp >= 2) {
    // ------------------------------------------------------------ epilogue
    const int g = warp & 3;
    const int h = (warp - 2) >> 2;           // token half of the 256 columns
    const int row = g * 32 + lane;           // weight row of this CTA = TMEM lane
    const int et = threadIdx.x - 64;         // 0..255
    const uint32_t lane_addr = static_cast<uint32_t>(g * 32) << 16;
    griddep_wait();
    const int chunks_o = q_outliers(p, RAW) ? p.K_out_pad / 64 : 0;
    bool ok = true;
    for (int it = 0; it < iters; ++it) {
      int tm, tn;
      tile_of(it, tm, tn);
      const int b = it & 1;  // s_x buffer
      const uint32_t ph = static_cast<uint32_t>(it) & 1;
      const int n = 256 * tn + 128 * static_cast<int>(rank) + row;
      const int m_base = kQBT * tm;
      float sw = 0.f;
      if (!RAW) {
        sw = n < p.N ? __ldg(p.s_w + n) : 0.f;
        if (et < kQBT) s_sx[b * kQBT + et] = m_base + et < p.M ? __ldg(p.s_x + m_base + et) : 0.f;
        named_barrier(1, 32 * kQEpiWarps);
      }
      if (!ok) continue;
      if (!q_warp_wait(acc_full, ph, p.wait_limit_ns)) {
        ok = false;
        continue;
      }
      tc_fence_after();
      const uint32_t d = tmem_base + lane_addr;
      const float *sx = s_sx + b * kQBT;
      if (!RAW && chunks_o > 0) {
#pragma unroll 1
        for (int c = 0; c < kQHalf / 32; ++c) {
          const int col = kQHalf * h + 32 * c;
          uint32_t v[32];
          tmem_ld32(d + col, v);
          tmem_ld_wait();
#pragma unroll
          for (int e = 0; e < 32; ++e)
            v[e] = __float_as_uint(
                __fmul_rn(__fmul_rn(static_cast<float>(static_cast<int>(v[e])), sx[col + e]), sw));
          tmem_st32(d + col, v);
        }
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive_cluster(conv_l);
        if (!q_warp_wait(out_full, ph, p.wait_limit_ns)) {
          ok = false;
          continue;
        }
        tc_fence_after();
      }
      // two 32-token chunks per TMEM round trip; the accumulator is released
      // after the last load, so the next tile's MMAs overlap the last stores
#pragma unroll 1
      for (int c = 0; c < kQHalf / 32; c += 2) {
        const int col = kQHalf * h + 32 * c;
        uint32_t v[2][32];
        tmem_ld32(d + col, v[0]);
        tmem_ld32(d + col + 32, v[1]);
        tmem_ld_wait();
        if (c + 2 == kQHalf / 32) {
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive_cluster(tmem_empty_l);
        }
        if (n >= p.N) continue;
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          const int m0c = m_base + col + 32 * hh;
          const int mcount = min(32, p.M - m0c);
          if (mcount <= 0) break;
          const size_t off0 = static_cast<size_t>(m0c) * p.ldy + n;
          if (RAW) {
            int32_t *yp = static_cast<int32_t *>(p.Y) + off0;
#pragma unroll
            for (int e = 0; e < 32; ++e)
              if (e < mcount) yp[static_cast<size_t>(e) * p.ldy] = static_cast<int32_t>(v[hh][e]);
          } else {
            __half *yp = static_cast<__half *>(p.Y) + off0;
#pragma unroll
            for (int e = 0; e < 32; ++e) {
              if (e >= mcount) break;
              const float y =
                  chunks_o > 0 ? __uint_as_float(v[hh][e])
                               : __fmul_rn(__fmul_rn(static_cast<float>(static_cast<int>(v[hh][e])),
                                                     sx[col + 32 * hh + e]),
                                           sw);
              yp[static_cast<size_t>(e) * p.ldy] = __float2half_rn(y);
            }
          }
        }
      }
    }
    if (!ok) q_fail(s_err, p.status);
  }
  __syncwarp();

  // ---------------------------------------------------------------- teardown
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();
  if (*s_err != 0 && threadIdx.x == 0) {
    // let copies still in flight land before the pair's shared memory is freed
    const int issued = s_misc[1];
    const int done = rank == 0 ? s_misc[2] : 0;
    for (int j = done; j < issued; ++j) {
      mbar_wait(&wfull[j % kQStages], (j / kQStages) & 1, p.wait_limit_ns);
      if (rank == 0) mbar_wait(&tfull[j % kQStages], (j / kQStages) & 1, p.wait_limit_ns);
    }
  }
  cluster_sync_all();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, kQTmemCols);
  }
}

// ------------------------------------------------------------------ host side
constexpr int q_smem() { return kQStages * kQStage + kQExtra + 1024; }
static_assert(q_smem() <= 232448, "shared memory per CTA");

template <bool RAW>
int q_max_pairs() {
  static std::atomic<int> cached[64];
  static std::atomic<uint64_t> smem_done{0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return -1;
  const int c = cached[dev].load();
  if (c > 0) return c;
  auto kernel = mixq_pair_w4_kernel<RAW>;
  if (ensure_smem(kernel, q_smem(), smem_done) != cudaSuccess) return -1;
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(2, 1, 1);
  cfg.blockDim = dim3(kQThreads, 1, 1);
  cfg.dynamicSmemBytes = q_smem();
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int n = -1;
  if (cudaOccupancyMaxActiveClusters(&n, kernel, &cfg) != cudaSuccess || n <= 0) {
    cudaGetLastError();
    return -1;
  }
  cached[dev].store(n);
  return n;
}

template <bool RAW>
cudaError_t q_launch(const GemmArgs &a, cudaStream_t stream, const char **why) {
  static std::atomic<uint64_t> smem_done{0};
  auto kernel = mixq_pair_w4_kernel<RAW>;
  cudaError_t e = ensure_smem(kernel, q_smem(), smem_done);
  if (e != cudaSuccess) return e;
  const int max_pairs = q_max_pairs<RAW>();
  if (max_pairs <= 0) {
    *why = "no cluster of two CTAs of the 4-bit pair kernel fits on this device";
    return cudaErrorInvalidConfiguration;
  }
  const int kp = RAW ? 0 : k_out_pad(a.K_out);
  alignas(64) CUtensorMap tm_a, tm_xo, tm_wo;
  memset(&tm_xo, 0, sizeof tm_xo);
  memset(&tm_wo, 0, sizeof tm_wo);
  bool ok = make_map(&tm_a, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, a.Xq, a.K, a.M, a.K, kBlockK,
                     kQHalf, CU_TENSOR_MAP_SWIZZLE_128B);
  if (kp > 0) {
    ok = ok && make_map(&tm_xo, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, a.X_out, kp, a.M,
                        static_cast<uint64_t>(kp) * 2, 64, kQHalf, CU_TENSOR_MAP_SWIZZLE_128B);
    ok = ok && make_map(&tm_wo, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, a.W_out, kp, a.N,
                        static_cast<uint64_t>(kp) * 2, 64, 128, CU_TENSOR_MAP_SWIZZLE_128B);
  }
  if (!ok) {
    *why = "cuTensorMapEncodeTiled failed (or the driver entry point is unavailable)";
    return cudaErrorInvalidValue;
  }
  QParams qp{};
  qp.M = a.M;
  qp.N = a.N;
  qp.K = a.K;
  qp.K_out_pad = kp;
  qp.m_tiles = (a.M + kQBT - 1) / kQBT;
  qp.n_tiles = (a.N + 255) / 256;
  const int tiles = qp.m_tiles * qp.n_tiles;
  qp.pairs = tiles < max_pairs ? tiles : max_pairs;
  qp.wq = static_cast<const uint8_t *>(a.Wq);
  qp.grp = static_cast<const uint8_t *>(a.grp);
  qp.s_x = a.s_x;
  qp.s_w = a.s_w;
  qp.flags = a.flags;
  qp.Y = a.Y;
  qp.ldy = a.ldy;
  qp.status = a.status;
  qp.wait_limit_ns = a.wait_limit_ns;

  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(2 * qp.pairs, 1, 1);
  cfg.blockDim = dim3(kQThreads, 1, 1);
  cfg.dynamicSmemBytes = q_smem();
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  return cudaLaunchKernelEx(&cfg, kernel, tm_a, tm_xo, tm_wo, qp);
}

}  // namespace

cudaError_t launch_gemm_pair_w4(const GemmArgs &a, cudaStream_t stream, const char **why) {
  if (a.mode != 1) {
    *why = "the 4-bit CTA-pair kernel takes progressive 4-bit weights";
    return cudaErrorInvalidValue;
  }
  return a.epi == Epi::kRawI32 ? q_launch<true>(a, stream, why) : q_launch<false>(a, stream, why);
}

}  // namespace mixq
