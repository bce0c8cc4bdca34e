// W8A8 GEMM of the MixQ layer for large M on CTA pairs (sm_100a, tcgen05
// cta_group::2), persistent.
//
//   acc[m,n] = sum_k Xq[m,k] Wq[n,k]                  tcgen05.mma kind::i8
//   c[m,n]   = (float(acc) * s_x[m]) * s_w[n]         epilogue warps, in TMEM
//   y[m,n]   = c + sum_j X_out[m,j] W_out[n,j]        tcgen05.mma kind::f16,
//                                                     accumulated onto c
//   Y[m,n]   = fp16(y)
//
// (MixQ article "一键部署LLM混合精度推理…": 研究背景 Fig. 5, the low-bit
// product plus the FP16 outlier product; MixQ的解决方案 Fig. 12, dequantize,
// scale and add of the INT32 result next to the tensor core, here in tensor
// memory.)
//
// Why pairs: at large M the operand tiles come from L2, and what the tensor
// core can use is bounded by the bytes each SM can bring into shared memory
// per MAC.  A CTA pair computes a 256-token x 256-weight-row tile with MMAs of
// M = 256: each CTA loads only its own 128 token rows (A) and its own 128 of
// the 256 weight rows (B), and the MMA reads B from both CTAs.  Per SM that is
// 32 KB per 128 x 256 x 128 MACs, a third less than a one-CTA 128 x 256 tile
// and half a 128 x 128 one.
//
// Per pair (cluster of 2 CTAs, one per SM), persistent over tiles
// pair, pair + P, ... (P = pairs resident at once):
//   warp 0 lane 0   producer (both CTAs): per job (two K blocks), its CTA's A
//                   and B tiles by TMA into a ring of 64 KB shared-memory
//                   stages; the loads signal the leader CTA's `full` barrier
//                   (cta_group::2 form)
//   warp 1          TMEM allocation (both CTAs, collective, 512 columns);
//                   lane 0 of the leader issues every MMA of the pair
//   warps 2..9      epilogue (both CTAs): warp w reads TMEM lanes 32(w%4)..,
//                   half of the 256 columns each
// The MMA issuer is the pair's critical thread: a job of two K blocks (eight
// MMAs) costs it one wait and one commit, and waiting warps sleep in their
// barrier waits rather than spin beside it.
// TMEM holds two 256-column accumulators used by alternate tiles, so one
// tile's epilogue runs beside the next tile's mainloop.  With outliers, the
// epilogue first converts the INT32 accumulator in place to the scaled FP32
// value c, the leader then accumulates the FP16 outlier product onto it (those
// MMAs are issued a few K blocks into the next tile, after the conversion),
// and the epilogue reads y back.  Jobs (a K block of the INT8 product, or 64
// outlier channels of the FP16 one) flow through the ring in the order both
// the producer and the MMA issuer derive from the same rule.
//
// Every mbarrier wait is bounded; a wait that runs out records
// MIXQ_ERR_TIMEOUT in *status and the CTA winds down (the pair still meets at
// its cluster barriers and frees its tensor memory together).
#include <cuda_fp16.h>

#include <atomic>
#include <mutex>

#include "internal.h"
#include "ptx.cuh"
#include "tma_host.h"

namespace mixq {
namespace {

constexpr int kPrThreads = 320;  // warp 0 producer, warp 1 MMA/TMEM, warps 2..9 epilogue
constexpr int kPrEpiWarps = 8;
constexpr int kPrMaxStages = 3;
constexpr int kPrTile = 128 * kBlockK;   // 128 rows x 128 bytes (one K block of A or B)
constexpr int kPrKbJob = 2;              // K blocks (or 64-channel outlier chunks) per job
constexpr int kPrStage = 2 * kPrKbJob * kPrTile;  // [A: 2 K blocks][B: 2 K blocks]
constexpr int kPrExtra = 1024 + 2 * 256 * 4;  // barriers, s_w of two tiles
constexpr int kPrTmemCols = 512;
constexpr int kPrLag = 2;  // jobs of the next tile before a tile's outlier jobs

struct PrParams {
  int M, N, K, K_out_pad;
  int m_tiles, n_tiles, pairs;  // 256 x 256 tiles; resident pairs (grid = 2 * pairs)
  int stages;
  const float *s_x;
  const float *s_w;
  const int32_t *flags;
  void *Y;  // fp16 [M][ldy] or int32 [M][ldy] (raw)
  int ldy;
  int32_t *status;
  uint64_t wait_limit_ns;
};

__device__ __forceinline__ void pr_fail(int *s_err, int32_t *status) {
  atomicOr(s_err, 1);
  record_error(status, kErrTimeout);
}

__device__ __forceinline__ bool pr_warp_wait(uint64_t *bar, uint32_t parity, uint64_t limit_ns) {
  return __all_sync(0xFFFFFFFFu, mbar_wait_sleep(bar, parity, limit_ns));
}

__device__ __forceinline__ int pr_outliers(const PrParams &p, bool raw) {
  if (raw || p.K_out_pad == 0) return 0;
  return p.flags ? (*reinterpret_cast<const volatile int32_t *>(p.flags) > 0) : 1;
}

// The job order of a pair, the same for its producers and its MMA issuer.
// A job is up to kPrKbJob K blocks of the INT8 product of one tile (or up to
// kPrKbJob 64-channel chunks of its outlier product), one shared-memory
// stage.  Tile iteration i contributes its INT8 jobs; when outliers are
// present, the outlier jobs of iteration i - 1 come after the first kPrLag
// INT8 jobs of iteration i (so the epilogue's in-place conversion of i - 1 has
// time to finish), and those of the last iteration come at the end.
// f(kind, iter, job, n_kb) returns false to stop.
template <typename F>
__device__ __forceinline__ void pr_for_each_job(int iters, int jobs8, int jobs_o, int kb8,
                                                int chunks_o, F &&f) {
  const int lag = jobs8 < kPrLag ? jobs8 : kPrLag;
  auto outl = [&](int it) {
    for (int j = 0; j < jobs_o; ++j)
      if (!f(1, it, j, min(kPrKbJob, chunks_o - j * kPrKbJob))) return false;
    return true;
  };
  for (int it = 0; it < iters; ++it) {
    for (int j = 0; j < jobs8; ++j) {
      if (it > 0 && j == lag && !outl(it - 1)) return;
      if (!f(0, it, j, min(kPrKbJob, kb8 - j * kPrKbJob))) return;
    }
    if (it > 0 && lag == jobs8 && !outl(it - 1)) return;
  }
  if (iters > 0) outl(iters - 1);
}

template <bool RAW>
__global__ void __launch_bounds__(kPrThreads, 1)
    mixq_pair_w8_kernel(const __grid_constant__ CUtensorMap tm_a,   // Xq [M][K], box {128, 128}
                        const __grid_constant__ CUtensorMap tm_w,   // Wq tiles as [N*K/128][128]
                        const __grid_constant__ CUtensorMap tm_xo,  // X_out [M][K_out_pad], {64, 128}
                        const __grid_constant__ CUtensorMap tm_wo,  // W_out [N][K_out_pad], {64, 128}
                        const PrParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const int stages = p.stages;
  auto a_slot = [&](int s) { return smem + s * kPrStage; };
  auto b_slot = [&](int s) { return smem + s * kPrStage + kPrKbJob * kPrTile; };
  uint8_t *extra = smem + stages * kPrStage;
  uint64_t *bars = reinterpret_cast<uint64_t *>(extra);
  uint64_t *full = bars;                      // leader: both CTAs' tiles of a stage landed
  uint64_t *empty = bars + kPrMaxStages;      // both: the MMAs have read the stage
  uint64_t *acc_full = empty + kPrMaxStages;  // [2] both: INT8 product of a tile done
  uint64_t *conv_done = acc_full + 2;         // [2] leader: both CTAs converted in place
  uint64_t *out_full = conv_done + 2;         // [2] both: outlier product added
  uint64_t *tmem_empty = out_full + 2;        // [2] leader: both CTAs drained the buffer
  uint64_t *drain = tmem_empty + 2;           // leader: wind-down commit
  uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(drain + 1);
  int *s_misc = reinterpret_cast<int *>(tmem_holder + 1);  // err, issued, consumed
  float *s_sw = reinterpret_cast<float *>(extra + 1024);   // [2][256]

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();  // 0 = leader
  const int pair = blockIdx.x >> 1;
  const int tiles = p.m_tiles * p.n_tiles;
  const int iters = pair < tiles ? (tiles - pair + p.pairs - 1) / p.pairs : 0;
  const int KB = p.K / kBlockK;
  const int jobs8 = (KB + kPrKbJob - 1) / kPrKbJob;
  auto tile_of = [&](int it, int &tm, int &tn) {
    const int t = pair + it * p.pairs;
    tm = t % p.m_tiles;
    tn = t / p.m_tiles;
  };
  // leader's barriers as shared::cluster addresses
  const uint32_t full_l = mapa_shared(smem_u32(full), 0u);
  const uint32_t conv_l = mapa_shared(smem_u32(conv_done), 0u);
  const uint32_t tmem_empty_l = mapa_shared(smem_u32(tmem_empty), 0u);

  if (threadIdx.x == 0) {
    for (int i = 0; i < stages; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&conv_done[b], 2 * kPrEpiWarps);
      mbar_init(&out_full[b], 1);
      mbar_init(&tmem_empty[b], 2 * kPrEpiWarps);
    }
    mbar_init(drain, 1);
    fence_mbar_init();
    s_misc[0] = 0;
    s_misc[1] = 0;
    s_misc[2] = 0;
    tma_prefetch_desc(&tm_a);
    tma_prefetch_desc(&tm_w);
    if (!RAW && p.K_out_pad > 0) {
      tma_prefetch_desc(&tm_xo);
      tma_prefetch_desc(&tm_wo);
    }
  }
  if (warp == 1) {
    tmem_alloc_pair(tmem_holder, kPrTmemCols);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  __syncthreads();
  // the peer's loads and arrivals target the leader's barriers: both CTAs'
  // barriers are initialised before either starts
  cluster_sync_all();
  tc_fence_after();
  if (threadIdx.x == 0) griddep_launch_dependents();
  const uint32_t tmem_base = *tmem_holder;
  int *s_err = &s_misc[0];

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0 && iters > 0) {
      const uint64_t pol = policy_evict_last();
      const int pre = min(stages, jobs8);
      int tm0, tn0;
      tile_of(0, tm0, tn0);
      // weights do not depend on the preceding kernel: the first stages' weight
      // tiles go out before waiting for it (the first jobs are always INT8 jobs
      // of the first tile)
      const int wrow0 = (2 * tn0 + static_cast<int>(rank)) * KB;
      for (int j = 0; j < pre; ++j) {
        const int nkb = min(kPrKbJob, KB - j * kPrKbJob);
        if (rank == 0) mbar_arrive_expect_tx(&full[j], 2u * 2u * kPrTile * nkb);
        for (int kb = 0; kb < nkb; ++kb)
          tma_load_2d_pair(b_slot(j) + kb * kPrTile, &tm_w, full_l + 8u * j, 0,
                           (wrow0 + j * kPrKbJob + kb) * 128, pol);
      }
      griddep_wait();
      const int chunks_o = pr_outliers(p, RAW) ? p.K_out_pad / 64 : 0;
      const int jobs_o = (chunks_o + kPrKbJob - 1) / kPrKbJob;
      int slot = 0, n = 0;
      uint32_t phase = 0;
      pr_for_each_job(iters, jobs8, jobs_o, KB, chunks_o, [&](int kind, int it, int j, int nkb) {
        int tm, tn;
        tile_of(it, tm, tn);
        const int row_a = 256 * tm + 128 * static_cast<int>(rank);
        const int row_b = 256 * tn + 128 * static_cast<int>(rank);
        const uint32_t bar = full_l + 8u * slot;
        if (n < pre) {
          for (int kb = 0; kb < nkb; ++kb)
            tma_load_2d_pair(a_slot(slot) + kb * kPrTile, &tm_a, bar,
                             (j * kPrKbJob + kb) * kBlockK, row_a, pol);
        } else {
          if (!mbar_wait_sleep(&empty[slot], phase ^ 1, p.wait_limit_ns)) {
            pr_fail(s_err, p.status);
            return false;
          }
          if (rank == 0) mbar_arrive_expect_tx(&full[slot], 2u * 2u * kPrTile * nkb);
          for (int kb = 0; kb < nkb; ++kb) {
            const int c = j * kPrKbJob + kb;  // K block, or 64-channel outlier chunk
            if (kind == 0) {
              tma_load_2d_pair(a_slot(slot) + kb * kPrTile, &tm_a, bar, c * kBlockK, row_a, pol);
              tma_load_2d_pair(b_slot(slot) + kb * kPrTile, &tm_w, bar, 0,
                               ((2 * tn + static_cast<int>(rank)) * KB + c) * 128, pol);
            } else {
              tma_load_2d_pair(a_slot(slot) + kb * kPrTile, &tm_xo, bar, c * 64, row_a, pol);
              tma_load_2d_pair(b_slot(slot) + kb * kPrTile, &tm_wo, bar, c * 64, row_b, pol);
            }
          }
        }
        ++n;
        if (++slot == stages) {
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
      constexpr uint32_t kIdI8 = idesc_s8_s32(256, 256);
      constexpr uint32_t kIdF16 = idesc_f16_f32(256, 256);
      // descriptors of stage 0; a stage or a K block further is a fixed offset
      // of the start-address field (shared-memory addresses >> 4)
      const uint64_t ad0 = sw128_kmajor_desc(smem_u32(a_slot(0)));
      const uint64_t bd0 = sw128_kmajor_desc(smem_u32(b_slot(0)));
      constexpr uint64_t kStageD = kPrStage >> 4, kTileD = kPrTile >> 4;
      griddep_wait();
      const int chunks_o = pr_outliers(p, RAW) ? p.K_out_pad / 64 : 0;
      const int jobs_o = (chunks_o + kPrKbJob - 1) / kPrKbJob;
      int slot = 0, n = 0;
      uint32_t phase = 0;
      bool ok = true;
      pr_for_each_job(iters, jobs8, jobs_o, KB, chunks_o, [&](int kind, int it, int j, int nkb) {
        const int b = it & 1;
        const uint32_t use = static_cast<uint32_t>(it >> 1);
        if (kind == 0 && j == 0 && it >= 2) {
          // the accumulator buffer's previous tile has been drained by both CTAs
          if (!mbar_wait_sleep(&tmem_empty[b], (use - 1) & 1, p.wait_limit_ns)) return ok = false;
          tc_fence_after();
        }
        if (kind == 1 && j == 0) {
          // both CTAs have converted the tile's accumulator to FP32 in place
          if (!mbar_wait_sleep(&conv_done[b], use & 1, p.wait_limit_ns)) return ok = false;
          tc_fence_after();
        }
        if (!mbar_try_wait(&full[slot], phase) && !mbar_wait(&full[slot], phase, p.wait_limit_ns))
          return ok = false;
        tc_fence_after();
        const uint32_t d = tmem_base + 256u * b;
        const uint64_t ad = ad0 + slot * kStageD, bd = bd0 + slot * kStageD;
        if (kind == 0) {
          for (int kb = 0; kb < nkb; ++kb) {
#pragma unroll
            for (int k = 0; k < 4; ++k)
              mma_i8_pair(d, ad + kb * kTileD + 2 * k, bd + kb * kTileD + 2 * k, kIdI8,
                          (j > 0 || kb > 0 || k > 0) ? 1u : 0u);
          }
        } else {
          for (int kb = 0; kb < nkb; ++kb) {
#pragma unroll
            for (int k = 0; k < 4; ++k)
              mma_f16_pair(d, ad + kb * kTileD + 2 * k, bd + kb * kTileD + 2 * k, kIdF16, 1u);
          }
        }
        mma_commit_pair(&empty[slot], 3);
        if (kind == 0 && j == jobs8 - 1) mma_commit_pair(&acc_full[b], 3);
        if (kind == 1 && j == jobs_o - 1) mma_commit_pair(&out_full[b], 3);
        ++n;
        if (++slot == stages) {
          slot = 0;
          phase ^= 1u;
        }
        return true;
      });
      s_misc[2] = n;
      if (!ok) {
        pr_fail(s_err, p.status);
        // every MMA issued so far completes before the pair winds down
        mma_commit_pair(drain, 1);
        mbar_wait(drain, 0, p.wait_limit_ns);
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int g = warp & 3;           // TMEM lane group
    const int h = (warp - 2) >> 2;    // column half of the 256-column tile
    const int row = g * 32 + lane;    // token row of this CTA's 128 = TMEM lane
    const int et = threadIdx.x - 64;  // 0..255 among the epilogue threads
    const uint32_t lane_addr = static_cast<uint32_t>(g * 32) << 16;
    griddep_wait();
    const int JO = pr_outliers(p, RAW) ? p.K_out_pad / 64 : 0;
    bool ok = true;
    // every epilogue warp runs every iteration (the named barrier below counts
    // all of them); after a failed wait a warp only skips the work
    for (int it = 0; it < iters; ++it) {
      int tm, tn;
      tile_of(it, tm, tn);
      const int b = it & 1;
      const uint32_t ph = static_cast<uint32_t>(it >> 1) & 1;
      const int m = 256 * tm + 128 * static_cast<int>(rank) + row;
      const int n_base = 256 * tn;
      float sx = 0.f;
      if (!RAW) {
        sx = m < p.M ? __ldg(p.s_x + m) : 0.f;
        // weight scales of the tile into shared memory (one per epilogue thread);
        // buffer b was last read two tiles ago, before the previous barrier
        s_sw[b * 256 + et] = n_base + et < p.N ? __ldg(p.s_w + n_base + et) : 0.f;
        named_barrier(1, 32 * kPrEpiWarps);
      }
      if (!ok) continue;
      if (!pr_warp_wait(&acc_full[b], ph, p.wait_limit_ns)) {
        ok = false;
        continue;
      }
      tc_fence_after();
      const uint32_t d = tmem_base + 256u * b + lane_addr;
      const float *sw = s_sw + b * 256;
      if (!RAW && JO > 0) {
        // c = (float(acc) * s_x) * s_w, written back in place as FP32
#pragma unroll 1
        for (int c = 0; c < 4; ++c) {
          const int col = 128 * h + 32 * c;
          uint32_t v[32];
          tmem_ld32(d + col, v);
          tmem_ld_wait();
#pragma unroll
          for (int e = 0; e < 32; ++e)
            v[e] = __float_as_uint(
                __fmul_rn(__fmul_rn(static_cast<float>(static_cast<int>(v[e])), sx), sw[col + e]));
          tmem_st32(d + col, v);
        }
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive_cluster(conv_l + 8u * b);
        if (!pr_warp_wait(&out_full[b], ph, p.wait_limit_ns)) {
          ok = false;
          continue;
        }
        tc_fence_after();
      }
#pragma unroll 1
      for (int c = 0; c < 4; ++c) {
        const int col = 128 * h + 32 * c;
        uint32_t v[32];
        tmem_ld32(d + col, v);
        tmem_ld_wait();
        if (m >= p.M || n_base + col >= p.N) continue;
        if (RAW) {
          int4 *dst = reinterpret_cast<int4 *>(static_cast<int32_t *>(p.Y) +
                                               static_cast<size_t>(m) * p.ldy + n_base + col);
#pragma unroll
          for (int i = 0; i < 8; ++i)
            dst[i] = make_int4(static_cast<int>(v[4 * i]), static_cast<int>(v[4 * i + 1]),
                               static_cast<int>(v[4 * i + 2]), static_cast<int>(v[4 * i + 3]));
        } else {
          uint32_t hv[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            float y0, y1;
            if (JO > 0) {
              y0 = __uint_as_float(v[2 * i]);
              y1 = __uint_as_float(v[2 * i + 1]);
            } else {
              y0 = __fmul_rn(__fmul_rn(static_cast<float>(static_cast<int>(v[2 * i])), sx),
                             sw[col + 2 * i]);
              y1 = __fmul_rn(__fmul_rn(static_cast<float>(static_cast<int>(v[2 * i + 1])), sx),
                             sw[col + 2 * i + 1]);
            }
            const __half2 hh = __floats2half2_rn(y0, y1);
            hv[i] = *reinterpret_cast<const uint32_t *>(&hh);
          }
          uint4 *dst = reinterpret_cast<uint4 *>(static_cast<__half *>(p.Y) +
                                                 static_cast<size_t>(m) * p.ldy + n_base + col);
#pragma unroll
          for (int i = 0; i < 4; ++i)
            dst[i] = make_uint4(hv[4 * i], hv[4 * i + 1], hv[4 * i + 2], hv[4 * i + 3]);
        }
      }
      // this warp has read its part of the buffer: the next tile may reuse it
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(tmem_empty_l + 8u * b);
    }
    if (!ok) pr_fail(s_err, p.status);
  }
  __syncwarp();

  // ---------------------------------------------------------------- teardown
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();  // both CTAs have stopped issuing loads and MMAs
  if (*s_err != 0 && threadIdx.x == 0 && rank == 0) {
    // let tiles still in flight land before the pair's shared memory is freed
    const int issued = s_misc[1], consumed = s_misc[2];
    for (int j = consumed; j < issued; ++j)
      mbar_wait(&full[j % stages], (j / stages) & 1, p.wait_limit_ns);
  }
  cluster_sync_all();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, kPrTmemCols);
  }
}

// ------------------------------------------------------------------ host side
constexpr int pr_smem(int stages) { return stages * kPrStage + kPrExtra + 1024; }
static_assert(pr_smem(kPrMaxStages) <= 232448, "shared memory per CTA");
static_assert(kPrMaxStages * 8 * 2 + 9 * 8 + 16 <= 1024, "barrier region");

template <bool RAW>
int pr_max_pairs() {
  // resident clusters of two CTAs (one per SM), per device
  static std::atomic<int> cached[64];
  static std::atomic<uint64_t> smem_done{0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return -1;
  const int c = cached[dev].load();
  if (c > 0) return c;
  auto kernel = mixq_pair_w8_kernel<RAW>;
  if (ensure_smem(kernel, pr_smem(kPrMaxStages), smem_done) != cudaSuccess) return -1;
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(2, 1, 1);
  cfg.blockDim = dim3(kPrThreads, 1, 1);
  cfg.dynamicSmemBytes = pr_smem(kPrMaxStages);
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
cudaError_t pr_launch(const GemmArgs &a, cudaStream_t stream, const char **why) {
  static std::atomic<uint64_t> smem_done{0};
  auto kernel = mixq_pair_w8_kernel<RAW>;
  cudaError_t e = ensure_smem(kernel, pr_smem(kPrMaxStages), smem_done);
  if (e != cudaSuccess) return e;
  const int max_pairs = pr_max_pairs<RAW>();
  if (max_pairs <= 0) {
    *why = "no cluster of two CTAs of the pair kernel fits on this device";
    return cudaErrorInvalidConfiguration;
  }
  const int kp = RAW ? 0 : k_out_pad(a.K_out);
  alignas(64) CUtensorMap tm_a, tm_w, tm_xo, tm_wo;
  memset(&tm_xo, 0, sizeof tm_xo);
  memset(&tm_wo, 0, sizeof tm_wo);
  // the prepacked weight tiles are already in the swizzled operand layout:
  // viewed as rows of 128 bytes, one box is one 16 KB tile, copied as is
  const uint64_t w_rows = static_cast<uint64_t>(a.N) * (a.K / kBlockK);
  bool ok = make_map(&tm_a, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, a.Xq, a.K, a.M, a.K, kBlockK, 128,
                     CU_TENSOR_MAP_SWIZZLE_128B);
  ok = ok && make_map(&tm_w, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, a.Wq, kBlockK, w_rows, kBlockK,
                      kBlockK, 128, CU_TENSOR_MAP_SWIZZLE_NONE);
  if (kp > 0) {
    ok = ok && make_map(&tm_xo, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, a.X_out, kp, a.M,
                        static_cast<uint64_t>(kp) * 2, 64, 128, CU_TENSOR_MAP_SWIZZLE_128B);
    ok = ok && make_map(&tm_wo, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, a.W_out, kp, a.N,
                        static_cast<uint64_t>(kp) * 2, 64, 128, CU_TENSOR_MAP_SWIZZLE_128B);
  }
  if (!ok) {
    *why = "cuTensorMapEncodeTiled failed (or the driver entry point is unavailable)";
    return cudaErrorInvalidValue;
  }
  PrParams pp{};
  pp.M = a.M;
  pp.N = a.N;
  pp.K = a.K;
  pp.K_out_pad = kp;
  pp.m_tiles = (a.M + 255) / 256;
  pp.n_tiles = (a.N + 255) / 256;
  const int tiles = pp.m_tiles * pp.n_tiles;
  pp.pairs = tiles < max_pairs ? tiles : max_pairs;
  pp.stages = kPrMaxStages;
  pp.s_x = a.s_x;
  pp.s_w = a.s_w;
  pp.flags = a.flags;
  pp.Y = a.Y;
  pp.ldy = a.ldy;
  pp.status = a.status;
  pp.wait_limit_ns = a.wait_limit_ns;

  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(2 * pp.pairs, 1, 1);
  cfg.blockDim = dim3(kPrThreads, 1, 1);
  cfg.dynamicSmemBytes = pr_smem(pp.stages);
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
  return cudaLaunchKernelEx(&cfg, kernel, tm_a, tm_w, tm_xo, tm_wo, pp);
}

}  // namespace

int pair_max_active(int raw) { return raw ? pr_max_pairs<true>() : pr_max_pairs<false>(); }

cudaError_t launch_gemm_pair(const GemmArgs &a, cudaStream_t stream, const char **why) {
  if (a.mode != 0) {
    *why = "the CTA-pair kernel takes 8-bit weights";
    return cudaErrorInvalidValue;
  }
  return a.epi == Epi::kRawI32 ? pr_launch<true>(a, stream, why) : pr_launch<false>(a, stream, why);
}

}  // namespace mixq
