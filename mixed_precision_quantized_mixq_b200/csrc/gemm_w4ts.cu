// W4A8 GEMM of the MixQ layer with the expanded INT8 weights held in tensor
// memory (sm_100a).
//
//   acc[n,m] = sum_k Wq[n,k] Xq[m,k]        tcgen05.mma kind::i8, A = weights
//                                           from TMEM, B = tokens from smem
//   o[n,m]   = sum_j W_out[n,j] X_out[m,j]  tcgen05.mma kind::f16, both smem
//   Y[m,n]   = fp16((float(acc) * s_x[m]) * s_w[n] + o)
//
// (MixQ article "一键部署LLM混合精度推理…": 研究背景 Fig. 5 the two products
// summed, MixQ的解决方案 Fig. 12 dequantize/scale/add in registers; QServe
// reading notes, 渐进量化 and 寄存器压力和并行性: 4-bit group codes expanded to
// INT8 inside the mainloop, four codes per 32-bit operation, no intermediate
// overflow; MixLLM page: two-stage dequantization feeding INT8 tensor cores.)
//
// Why weights are the A operand: expanding 4-bit codes to INT8 is register
// work.  Written back to shared memory (as the B operand of a smem x smem
// MMA) the expanded tile costs a store and an MMA read of shared memory on
// top of the packed-code read -- three passes through the 128 B/clk shared
// memory port per weight byte, which caps a 128 x 256 tile below the INT8
// tensor-core rate.  tcgen05.mma takes A from tensor memory instead: the
// expansion threads store each weight row straight from registers into its
// TMEM lane (tcgen05.st), and shared memory only carries the packed codes and
// the token tile.  The output tile is therefore transposed in TMEM: lane =
// weight row n (128 per CTA), column = token m (the MMA's N, 16..128).
//
// One CTA computes the 128-weight-row x BT-token output tile over a K range:
//   warp 0 lane 0   producer: packed codes + group constants (1-D bulk copies
//                   of the prepacked 8 KB tiles) and the token tile (TMA,
//                   128-byte swizzle) into a ring of shared-memory stages;
//                   outlier stages carry a 32-column W_out tile and the
//                   matching X_out tile (64-byte swizzle)
//   warp 1 lane 0   MMA issuer: 4 TS MMAs per INT8 stage (32 K each), 2 SS
//                   MMAs per outlier stage (16 K each)
//   warps 4..7      expansion: thread = weight row = TMEM lane; 64 bytes of
//                   codes -> 32 words of INT8 -> one tcgen05.st per K block
//                   into a ring of TMEM A stages
//   warps 2..3      scales of the tile into shared memory
//   all 8 warps     epilogue (warps w and w+4 share TMEM lanes 32(w%4).. and
//                   split the token columns)
// Stages of packed weights are released as soon as the expansion threads have
// read them (the MMA reads only the token tile from shared memory), so the
// weight stream runs ahead of the tensor cores by the whole ring.
//
// K split over a thread-block cluster (decode-sized M): every CTA of the
// cluster owns a K range, stores its INT32 partial tile to its own shared
// memory token-major, and the cluster reduces through distributed shared
// memory (integer sums: exact and order-free).  CTA rank 0 runs the outlier
// slice.  Every mbarrier wait is bounded; a wait that runs out records
// MIXQ_ERR_TIMEOUT in *status and the CTA winds down.
#include <cuda_fp16.h>

#include <atomic>

#include "internal.h"
#include "ptx.cuh"
#include "tma_host.h"

namespace mixq {
namespace {

constexpr int kTsThreads = 256;  // warps 0-3: roles; 4-7: expansion
constexpr int kTsMaxStages = 12;
constexpr int kTsPacked = 128 * (kBlockK / 2);        // 8 KB of codes per 128 x 128 block
constexpr int kTsGrp = 128 * 4;                        // (s2, z2) fp16 pair per row
constexpr int kTsOutK = 32;                            // fp16 K per outlier stage (64 bytes)
constexpr int kTsWOut = 128 * kTsOutK * 2;             // W_out tile of an outlier stage
constexpr int kTsExtra = 1024 + 512 + 1024;            // barriers, s_w[128], s_x[256]
constexpr int kTsPitch = 128 + 4;                      // words per token row of a partial tile

// SM = two CTAs per SM (half the shared memory, 256 TMEM columns each): the
// decode variant, which also lets a CTA of the next kernel start beside it.
// Otherwise one CTA per SM with 512 TMEM columns and the deepest ring.
template <bool SM>
struct TsCfg {
  static constexpr int kMinBlocks = SM ? 2 : 1;
  static constexpr int kSmemMax = SM ? 233472 / 2 - 1024 : 232448;
  static constexpr int kTmemCols = SM ? 256 : 512;
  static constexpr int kACol = SM ? 128 : 256;  // first column of the TMEM A ring
};

// A job is `kbpj` (1 or 2) K blocks of 128: one wait and one commit per job,
// so two blocks per job halve the fixed per-stage cost of the MMA issuer
// (about 0.4 us per job, measured) where shared memory allows.
// Stage layout: [codes: kbpj x 8 KB][constants: kbpj x 512 B] padded to 1 KB
// (= w_slot), then the token tiles [kbpj][bt rows x 128 B].  An outlier stage
// holds a 32-column W_out tile at 0 and the X_out tile at w_slot.
struct TsParams {
  int M, N, K, K_out_pad;
  int bt;           // tokens per tile = MMA N (multiple of 16, at most 256)
  int kbpj;         // K blocks per job (1 or 2)
  int stages;       // shared-memory ring depth (>= a_stages)
  int stage_bytes;  // w_slot + kbpj * bt * 128
  int w_slot;       // bytes before the token tiles
  int a_stages;     // TMEM A ring depth (32 * kbpj columns each)
  int f32_col;      // TMEM column of the FP32 outlier accumulator
  const uint8_t *wq;   // tiled 4-bit codes: [N/128][K/128] tiles of 128 rows x 64 bytes
  const uint8_t *grp;  // [K/128][N] (s2, z2) fp16 pairs
  const float *s_x;
  const float *s_w;
  const int32_t *flags;
  void *Y;  // fp16 [M][ldy], or int32 [M][ldy] for the raw variant
  int ldy;
  int32_t *status;
  uint64_t wait_limit_ns;
  int w_streamed;  // weights are read by one CTA only: evict them from L2 first
};

__device__ __forceinline__ void ts_fail(int *s_err, int32_t *status) {
  atomicOr(s_err, 1);
  record_error(status, kErrTimeout);
}

// 4 codes (one per byte, low nibbles) -> 4 signed INT8 weights
// (q - z2) * s2 = ((q * s2 + 128 - z2 * s2) ^ 0x80) as two's complement; each
// byte's value (q - z2) * s2 + 128 lies in [0, 255], so the 32-bit multiply-add
// never carries between bytes.
__device__ __forceinline__ uint32_t ts_expand4(uint32_t nibbles, uint32_t s2, uint32_t c) {
  return (nibbles * s2 + c) ^ 0x80808080u;
}

__device__ __forceinline__ int ts_outliers_present(const TsParams &p, bool raw) {
  if (raw || p.K_out_pad == 0) return 0;
  return p.flags ? (*reinterpret_cast<const volatile int32_t *>(p.flags) > 0) : 1;
}

// Warp-uniform bounded wait: every lane waits, the warp proceeds only if all
// lanes saw the phase complete (the TMEM stores that follow are warp-wide).
__device__ __forceinline__ bool warp_wait(uint64_t *bar, uint32_t parity, uint64_t limit_ns) {
  return __all_sync(0xFFFFFFFFu, mbar_wait(bar, parity, limit_ns));
}

// NCH 16-byte chunks (starting at chunk c0) of one weight row's 64 code bytes
// in a prepacked 128 x 128 block -> 8 * NCH words of INT8 weights, word t
// holding K 32*c0 + 4t .. 4t+3.  Chunk c word w: low nibbles = K 32c+8w+0..3,
// high nibbles = K 32c+8w+4..7.
template <int NCH>
__device__ __forceinline__ void expand_chunks(const uint8_t *codes, const uint8_t *consts, int row,
                                              int psw, int c0, uint32_t (&wv)[8 * NCH]) {
  uint4 pk[NCH];
#pragma unroll
  for (int i = 0; i < NCH; ++i)
    pk[i] = *reinterpret_cast<const uint4 *>(codes + row * 64 + (((c0 + i) ^ psw) << 4));
  const uint32_t g = reinterpret_cast<const uint32_t *>(consts)[row];
  const uint32_t s2 = static_cast<uint32_t>(
      __half2float(__ushort_as_half(static_cast<unsigned short>(g & 0xFFFFu))));
  const uint32_t z2 = static_cast<uint32_t>(
      __half2float(__ushort_as_half(static_cast<unsigned short>(g >> 16))));
  const uint32_t cst = (128u - z2 * s2) * 0x01010101u;
#pragma unroll
  for (int i = 0; i < NCH; ++i) {
    const uint32_t q4[4] = {pk[i].x, pk[i].y, pk[i].z, pk[i].w};
#pragma unroll
    for (int w = 0; w < 4; ++w) {
      wv[8 * i + 2 * w] = ts_expand4(q4[w] & 0x0F0F0F0Fu, s2, cst);
      wv[8 * i + 2 * w + 1] = ts_expand4((q4[w] >> 4) & 0x0F0F0F0Fu, s2, cst);
    }
  }
}

// Position in a ring of `n` slots, advanced one job at a time.
struct RingPos {
  int slot = 0;
  uint32_t phase = 0;
  __device__ __forceinline__ void advance(int n) {
    if (++slot == n) {
      slot = 0;
      phase ^= 1u;
    }
  }
};

template <bool SM, bool RAW>
__global__ void __launch_bounds__(kTsThreads, TsCfg<SM>::kMinBlocks)
    mixq_w4ts_kernel(const __grid_constant__ CUtensorMap tm_a,   // Xq [M][K] int8, box {128, bt}
                     const __grid_constant__ CUtensorMap tm_xo,  // X_out [M][K_out_pad], box {32, bt}
                     const __grid_constant__ CUtensorMap tm_wo,  // W_out [N][K_out_pad], box {32, 128}
                     const __grid_constant__ CUtensorMap tm_y,   // Y [M][ldy] fp16, box {64, bt}
                     const TsParams p) {
  using C = TsCfg<SM>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const int stages = p.stages;
  const int kbpj = p.kbpj;
  auto stage = [&](int s) { return smem + s * p.stage_bytes; };
  uint8_t *extra = smem + stages * p.stage_bytes;
  uint64_t *bars = reinterpret_cast<uint64_t *>(extra);
  uint64_t *wfull = bars;                      // weights (codes or W_out) landed
  uint64_t *tfull = bars + kTsMaxStages;       // token tile(s) (Xq or X_out) landed
  uint64_t *empty = bars + 2 * kTsMaxStages;   // 4 expansion-warp arrivals + MMA commit
  uint64_t *afull = bars + 3 * kTsMaxStages;   // TMEM A stage written (4 warp arrivals)
  uint64_t *accum_full = bars + 4 * kTsMaxStages;
  uint64_t *i8_done = accum_full + 1;
  uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(i8_done + 1);
  int *s_misc = reinterpret_cast<int *>(tmem_holder + 1);  // err, weights issued, tokens issued
  float *s_sw = reinterpret_cast<float *>(extra + 1024);   // [128]
  float *s_sx = reinterpret_cast<float *>(extra + 1536);   // [bt], bt <= 256

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int bt = p.bt;
  const int m0 = blockIdx.x * bt;
  const int n0 = blockIdx.y * 128;
  const int S = gridDim.z;
  const int rank = blockIdx.z;
  const int KB = p.K / kBlockK;
  const int kb_begin = static_cast<int>(static_cast<long long>(rank) * KB / S);
  const int kb_end = static_cast<int>(static_cast<long long>(rank + 1) * KB / S);
  const int n_i8 = (kb_end - kb_begin + kbpj - 1) / kbpj;  // INT8 jobs, then outlier jobs
  const int pre = n_i8 < stages ? n_i8 : stages;
  const uint32_t tok_bytes = static_cast<uint32_t>(bt) * kBlockK;
  const size_t wtile0 = static_cast<size_t>(n0 / 128) * KB;
  auto job_kb = [&](int j) { return kb_begin + j * kbpj; };
  auto job_nkb = [&](int j) { return min(kbpj, kb_end - job_kb(j)); };
  // codes of a job's K blocks are adjacent 8 KB tiles: one bulk copy; the
  // constants are [K/128][N]: one 512-byte copy per block
  auto issue_w = [&](int j, int s, uint64_t pol) {
    const int kb = job_kb(j), nkb = job_nkb(j);
    mbar_arrive_expect_tx(&wfull[s], nkb * (kTsPacked + kTsGrp));
    bulk_load(stage(s), p.wq + (wtile0 + kb) * kTsPacked, nkb * kTsPacked, &wfull[s], pol);
    for (int kk = 0; kk < nkb; ++kk)
      bulk_load(stage(s) + kbpj * kTsPacked + kk * kTsGrp,
                p.grp + (static_cast<size_t>(kb + kk) * p.N + n0) * 4, kTsGrp, &wfull[s], pol);
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
      mbar_init(&empty[i], 4 + 1);  // one arrival per expansion warp + the MMA commit
    }
    for (int a = 0; a < p.a_stages; ++a) mbar_init(&afull[a], 4);  // one per expansion warp
    mbar_init(accum_full, 1);
    mbar_init(i8_done, 1);
    fence_mbar_init();
    s_misc[0] = 0;
    // The weights do not depend on the preceding kernel: start streaming them
    // before anything else, and before waiting for that kernel.
    const uint64_t pol_w = p.w_streamed ? policy_evict_first() : policy_evict_last();
    for (int j = 0; j < pre; ++j) issue_w(j, j, pol_w);
    s_misc[1] = pre;
    s_misc[2] = 0;
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
  const uint32_t t_i32 = tmem_base;
  const uint32_t t_f32 = tmem_base + p.f32_col;
  const uint32_t t_a = tmem_base + C::kACol;
  const uint32_t a_cols = 32u * kbpj;  // TMEM columns of one A stage
  // the FP32 accumulator may share columns with the A ring (bt = 128 in the
  // two-CTA variant): the outlier MMAs then start once every INT8 MMA is done
  const bool f32_aliases_a = p.f32_col >= C::kACol;
  int *s_err = &s_misc[0];

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
      const int n_out = (ts_outliers_present(p, RAW) && rank == 0) ? p.K_out_pad / kTsOutK : 0;
      const int njobs = n_i8 + n_out;
      RingPos r;  // position of job j (no division in the loop)
      r.slot = pre == stages ? 0 : pre;
      r.phase = pre == stages ? 1u : 0u;
      for (int j = pre; j < njobs; ++j) {
        const int s = r.slot;
        if (!mbar_wait(&empty[s], r.phase ^ 1, p.wait_limit_ns)) {
          ts_fail(s_err, p.status);
          break;
        }
        if (j < n_i8) {
          issue_w(j, s, pol_w);
          s_misc[1] = j + 1;
          issue_t(j, s, pol_a);
        } else {
          const int o = j - n_i8;
          mbar_arrive_expect_tx(&wfull[s], kTsWOut);
          tma_load_2d(stage(s), &tm_wo, &wfull[s], o * kTsOutK, n0, pol_w);
          s_misc[1] = j + 1;
          mbar_arrive_expect_tx(&tfull[s], static_cast<uint32_t>(bt) * kTsOutK * 2);
          tma_load_2d(stage(s) + p.w_slot, &tm_xo, &tfull[s], o * kTsOutK, m0, pol_a);
        }
        s_misc[2] = j + 1;
        r.advance(stages);
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------- MMA issuer
    if (lane == 0) {
      const uint32_t id_i8 = idesc_s8_s32(128, bt);
      const uint32_t id_f16 = idesc_f16_f32(128, bt);
      // token-tile descriptor of stage 0; stage s adds a fixed start-address offset
      const uint64_t bd0 = sw128_kmajor_desc(smem_u32(stage(0) + p.w_slot));
      const uint64_t st_step = static_cast<uint64_t>(p.stage_bytes >> 4);
      griddep_wait();
      // the INT8 jobs first: the flags word (is there an outlier slice) is
      // read once they are issued, off the path of the first MMAs
      int njobs = n_i8;
      bool counted = false;
      RingPos r, ra;
      for (int j = 0;; ++j) {
        if (j == njobs) {
          if (counted) break;
          counted = true;
          njobs += (ts_outliers_present(p, RAW) && rank == 0) ? p.K_out_pad / kTsOutK : 0;
          if (j == njobs) break;
        }
        const int s = r.slot;
        if (j < n_i8) {
          if (!mbar_wait(&tfull[s], r.phase, p.wait_limit_ns) ||
              !mbar_wait(&afull[ra.slot], ra.phase, p.wait_limit_ns)) {
            ts_fail(s_err, p.status);
            break;
          }
          tc_fence_after();
          const uint32_t ta = t_a + ra.slot * a_cols;
          const uint64_t bd = bd0 + static_cast<uint64_t>(s) * st_step;
          const int nkb = job_nkb(j);
          for (int kk = 0; kk < nkb; ++kk) {
            const uint64_t bdk = bd + static_cast<uint64_t>(kk * tok_bytes >> 4);
#pragma unroll
            for (int k = 0; k < 4; ++k)
              mma_i8_ts(t_i32, ta + kk * 32 + k * 8, bdk + 2 * k, id_i8,
                        (j > 0 || kk > 0 || k > 0) ? 1u : 0u);
          }
          ra.advance(p.a_stages);
        } else {
          if (j == n_i8 && f32_aliases_a && n_i8 > 0) {
            mma_commit(i8_done);
            if (!mbar_wait(i8_done, 0, p.wait_limit_ns)) {
              ts_fail(s_err, p.status);
              break;
            }
            tc_fence_after();
          }
          if (!mbar_wait(&wfull[s], r.phase, p.wait_limit_ns) ||
              !mbar_wait(&tfull[s], r.phase, p.wait_limit_ns)) {
            ts_fail(s_err, p.status);
            break;
          }
          tc_fence_after();
          const uint64_t ad = sw64_kmajor_desc(smem_u32(stage(s)));
          const uint64_t bd = sw64_kmajor_desc(smem_u32(stage(s) + p.w_slot));
#pragma unroll
          for (int k = 0; k < 2; ++k)
            mma_f16(t_f32, ad + 2 * k, bd + 2 * k, id_f16, (j > n_i8 || k > 0) ? 1u : 0u);
        }
        // one commit per job: frees the shared-memory stage and, for INT8
        // jobs, the TMEM A stage the MMAs read
        mma_commit(&empty[s]);
        r.advance(stages);
      }
      mma_commit(accum_full);
    }
  } else if ((warp == 2 || warp == 3) && !RAW) {
    // ------------------------------------ token scales of the tile, early
    // weight scales (independent of the preceding kernel), then token
    // scales, during the mainloop rather than on the set-up path
    for (int i = threadIdx.x - 64; i < 128; i += 64) s_sw[i] = p.s_w[n0 + i];
    griddep_wait();
    for (int i = threadIdx.x - 64; i < bt; i += 64) s_sx[i] = m0 + i < p.M ? p.s_x[m0 + i] : 0.f;
  } else if (warp >= 4) {
    // ------------------------------------------- 4-bit -> INT8 expansion
    // Warp w covers TMEM lanes 32(w%4).. = the tile's weight rows; a thread
    // owns one row.  (Eight warps splitting each job measured slower.)
    const int row = (warp & 3) * 32 + lane;  // weight row of the tile = TMEM lane
    const uint32_t lane_addr = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const int psw = (row >> 1) & 3;          // chunk swizzle of the prepacked tile
    bool ok = true;
    RingPos r, ra;
    RingPos rf;  // job j - a_stages: its commit frees the A stage job j writes
    for (int j = 0; j < n_i8; ++j) {
      const int s = r.slot;
      if (!warp_wait(&wfull[s], r.phase, p.wait_limit_ns)) {
        ok = false;
        break;
      }
      // expand both K blocks of the job first (independent work for the
      // scheduler), release the codes, and only then wait for the A stage
      const uint8_t *sp = stage(s);
      const int nkb = job_nkb(j);
      uint32_t wv0[32], wv1[32];
      expand_chunks<4>(sp, sp + kbpj * kTsPacked, row, psw, 0, wv0);
      if (nkb == 2) expand_chunks<4>(sp + kTsPacked, sp + kbpj * kTsPacked + kTsGrp, row, psw, 0, wv1);
      // the codes are consumed: the stage's weight half is free (one arrival
      // per warp)
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[s]);
      r.advance(stages);
      if (j >= p.a_stages) {
        // A stage j % a_stages was last read by job j - a_stages, whose commit
        // completes that job's phase of empty[].  (stages >= a_stages keeps the
        // phase unambiguous: this warp's arrival for that slot's next use comes
        // only after the producer refilled it, i.e. after that phase.)
        if (!warp_wait(&empty[rf.slot], rf.phase, p.wait_limit_ns)) {
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
      const int n_out = (ts_outliers_present(p, RAW) && rank == 0) ? p.K_out_pad / kTsOutK : 0;
      for (int j = n_i8; j < n_i8 + n_out; ++j) {
        // outlier stages: only release the stage once its tiles are there (an
        // arrival for a later use of the slot must not land early)
        if (!warp_wait(&wfull[r.slot], r.phase, p.wait_limit_ns)) {
          ok = false;
          break;
        }
        if (lane == 0) mbar_arrive(&empty[r.slot]);
        r.advance(stages);
      }
    }
    if (!ok) ts_fail(s_err, p.status);
  }
  __syncwarp();

  // ---------------------------------------------------------------- epilogue
  griddep_wait();
  const int any_out = ts_outliers_present(p, RAW);
  const bool do_out = any_out && rank == 0;
  if (!mbar_wait_sleep(accum_full, 0, p.wait_limit_ns)) ts_fail(s_err, p.status);
  tc_fence_after();
  __syncthreads();
  const bool failed = *s_err != 0;
  const int row = (warp & 3) * 32 + lane;  // weight row n0 + row = TMEM lane
  const uint32_t lane_addr = static_cast<uint32_t>((warp & 3) * 32) << 16;
  const int nchunks = bt / 16;
  // warps w and w+4 share TMEM lanes and split the 16-token chunks
  const int c_first = warp >> 2;
  constexpr int kCStep = 2;

  if (S == 1 && !RAW) {
    // fp16 tile staged in shared memory as two 64-column TMA-store boxes in the
    // 128-byte swizzle (box t holds weight rows 64t..64t+63 as columns), then
    // written by coalesced bulk tensor stores
    uint8_t *stage_y = smem;  // the ring is free: every MMA has completed
    if (!failed) {
      const float sw = s_sw[row];
      uint8_t *box = stage_y + (row >> 6) * bt * 128;
      const int chunk = (row & 63) >> 3, within = (row & 7) * 2;
#pragma unroll 1
      for (int c = c_first; c < nchunks; c += kCStep) {
        uint32_t acc[16], o[16];
        tmem_ld16(t_i32 + lane_addr + c * 16, acc);
        if (do_out) tmem_ld16(t_f32 + lane_addr + c * 16, o);
        tmem_ld_wait();
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const int m = c * 16 + i;
          float v = __fmul_rn(__fmul_rn(static_cast<float>(static_cast<int>(acc[i])), s_sx[m]), sw);
          if (do_out) v = __fadd_rn(v, __uint_as_float(o[i]));
          *reinterpret_cast<__half *>(box + m * 128 + ((chunk ^ (m & 7)) << 4) + within) =
              __float2half_rn(v);
        }
      }
      fence_proxy_async_smem();
    }
    __syncthreads();
    if (threadIdx.x == 0 && !failed) {
      tma_store_2d(&tm_y, stage_y, n0, m0);
      tma_store_2d(&tm_y, stage_y + bt * 128, n0 + 64, m0);
      bulk_commit_group();
      bulk_wait_all();
    }
  } else if (S == 1) {
    if (!failed) {
#pragma unroll 1
      for (int c = c_first; c < nchunks; c += kCStep) {
        uint32_t acc[16];
        tmem_ld16(t_i32 + lane_addr + c * 16, acc);
        tmem_ld_wait();
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const int m = m0 + c * 16 + i;
          if (m < p.M)
            static_cast<int32_t *>(p.Y)[static_cast<size_t>(m) * p.ldy + n0 + row] =
                static_cast<int32_t>(acc[i]);
        }
      }
    }
  } else {
    // ------------------------------------ K split: reduce across the cluster
    int32_t *pbuf = reinterpret_cast<int32_t *>(smem);
    float *obuf = reinterpret_cast<float *>(smem + bt * kTsPitch * 4);
    const int rows_valid = min(bt, p.M - m0);  // tokens of this tile
    if (!failed) {
#pragma unroll 1
      for (int c = c_first; c < nchunks; c += kCStep) {
        uint32_t acc[16], o[16];
        tmem_ld16(t_i32 + lane_addr + c * 16, acc);
        if (do_out) tmem_ld16(t_f32 + lane_addr + c * 16, o);
        tmem_ld_wait();
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const int m = c * 16 + i;
          if (m < rows_valid) {
            pbuf[m * kTsPitch + row] = static_cast<int32_t>(acc[i]);
            if (do_out) obuf[m * kTsPitch + row] = __uint_as_float(o[i]);
          }
        }
      }
    }
    cluster_sync_all();
    if (!failed) {
      // this CTA reduces weight rows [c_begin, c_end) of the tile
      const int my_rank = static_cast<int>(cluster_ctarank());
      const int c_begin = my_rank * 32 / S * 4;
      const int c_end = (my_rank + 1) * 32 / S * 4;
      const int c4n = (c_end - c_begin) / 4;
#pragma unroll 1
      for (int e = threadIdx.x; e < rows_valid * c4n; e += kTsThreads) {
        const int m = e / c4n;
        const int col = c_begin + (e % c4n) * 4;
        const uint32_t off = smem_u32(pbuf + m * kTsPitch + col);
        int4 part[8];
#pragma unroll
        for (int q = 0; q < 8; ++q)
          if (q < S) part[q] = ld_dsmem_v4(mapa_shared(off, static_cast<uint32_t>(q)));
        int4 oi = make_int4(0, 0, 0, 0);
        if (!RAW && any_out) oi = ld_dsmem_v4(mapa_shared(smem_u32(obuf + m * kTsPitch + col), 0u));
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
        const size_t yoff = static_cast<size_t>(m0 + m) * p.ldy + n0 + col;
        if (RAW) {
          *reinterpret_cast<int4 *>(static_cast<int32_t *>(p.Y) + yoff) = sum;
        } else {
          const int si[4] = {sum.x, sum.y, sum.z, sum.w};
          const float ov[4] = {__int_as_float(oi.x), __int_as_float(oi.y), __int_as_float(oi.z),
                               __int_as_float(oi.w)};
          const float sx = s_sx[m];
          float y[4];
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            float v = __fmul_rn(__fmul_rn(static_cast<float>(si[i]), sx), s_sw[col + i]);
            if (any_out) v = __fadd_rn(v, ov[i]);
            y[i] = v;
          }
          const __half2 h0 = __floats2half2_rn(y[0], y[1]);
          const __half2 h1 = __floats2half2_rn(y[2], y[3]);
          *reinterpret_cast<uint2 *>(static_cast<__half *>(p.Y) + yoff) =
              make_uint2(*reinterpret_cast<const uint32_t *>(&h0),
                         *reinterpret_cast<const uint32_t *>(&h1));
        }
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
struct TsGeometry {
  int bt, kbpj, w_slot, stages, stage_bytes, a_stages, smem, f32_col;
};

template <bool SM>
TsGeometry ts_geometry(int M) {
  using C = TsCfg<SM>;
  TsGeometry g{};
  // the one-CTA variant takes 256 tokens per tile above M = 1024 (MMA N = 256:
  // each 8.5 KB stage of codes feeds twice the tokens of a 128-token tile)
  g.bt = SM ? (M >= 128 ? 128 : (M + 15) / 16 * 16) : (M > 1024 ? 256 : 128);
  if (g.bt < 16) g.bt = 16;
  // two K blocks per job unless that leaves fewer than three stages
  for (int kbpj = 2; kbpj >= 1; --kbpj) {
    g.kbpj = kbpj;
    g.w_slot = (kbpj * (kTsPacked + kTsGrp) + 1023) / 1024 * 1024;
    g.stage_bytes = g.w_slot + kbpj * g.bt * kBlockK;
    g.stages = (C::kSmemMax - 1024 - kTsExtra) / g.stage_bytes;
    if (g.stages > kTsMaxStages) g.stages = kTsMaxStages;
    if (g.stages >= 3) break;
  }
  g.a_stages = (C::kTmemCols - C::kACol) / (32 * g.kbpj);
  if (g.a_stages > g.stages) g.a_stages = g.stages;
  g.smem = g.stages * g.stage_bytes + kTsExtra + 1024;
  g.f32_col = 2 * g.bt <= C::kACol ? g.bt : C::kACol;
  return g;
}

template <bool SM, bool RAW>
cudaError_t launch_ts_variant(const GemmArgs &a, const GemmPlan &plan, const TsGeometry &geo,
                              cudaStream_t stream, const char **why) {
  using C = TsCfg<SM>;
  static_assert(C::kSmemMax <= 232448, "shared memory budget");
  static std::atomic<uint64_t> smem_done{0};
  auto kernel = mixq_w4ts_kernel<SM, RAW>;
  cudaError_t e = ensure_smem(kernel, C::kSmemMax, smem_done);
  if (e != cudaSuccess) return e;
  const int red_bytes = 2 * geo.bt * kTsPitch * 4;
  if (geo.stages < 2 || geo.stages < geo.a_stages || geo.a_stages > kTsMaxStages ||
      geo.smem > C::kSmemMax || (plan.split > 1 && geo.stages * geo.stage_bytes < red_bytes)) {
    *why = "no pipeline geometry fits the shared-memory budget";
    return cudaErrorInvalidValue;
  }
  const int kp = k_out_pad(a.K_out);
  alignas(64) CUtensorMap tm_a, tm_xo, tm_wo, tm_y;
  memset(&tm_xo, 0, sizeof tm_xo);
  memset(&tm_wo, 0, sizeof tm_wo);
  memset(&tm_y, 0, sizeof tm_y);
  bool ok = make_map(&tm_a, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, a.Xq, a.K, a.M, a.K, kBlockK,
                     geo.bt, CU_TENSOR_MAP_SWIZZLE_128B);
  if (!RAW && kp > 0) {
    ok = ok && make_map(&tm_xo, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, a.X_out, kp, a.M,
                        static_cast<uint64_t>(kp) * 2, kTsOutK, geo.bt, CU_TENSOR_MAP_SWIZZLE_64B);
    ok = ok && make_map(&tm_wo, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, a.W_out, kp, a.N,
                        static_cast<uint64_t>(kp) * 2, kTsOutK, 128, CU_TENSOR_MAP_SWIZZLE_64B);
  }
  if (!RAW)
    ok = ok && make_map(&tm_y, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, a.Y, a.N, a.M,
                        static_cast<uint64_t>(a.ldy) * 2, 64, geo.bt, CU_TENSOR_MAP_SWIZZLE_128B);
  if (!ok) {
    *why = "cuTensorMapEncodeTiled failed (or the driver entry point is unavailable)";
    return cudaErrorInvalidValue;
  }

  TsParams kp_{};
  kp_.M = a.M;
  kp_.N = a.N;
  kp_.K = a.K;
  kp_.K_out_pad = RAW ? 0 : kp;
  kp_.bt = geo.bt;
  kp_.kbpj = geo.kbpj;
  kp_.stages = geo.stages;
  kp_.stage_bytes = geo.stage_bytes;
  kp_.w_slot = geo.w_slot;
  kp_.a_stages = geo.a_stages;
  kp_.f32_col = geo.f32_col;
  kp_.wq = static_cast<const uint8_t *>(a.Wq);
  kp_.grp = static_cast<const uint8_t *>(a.grp);
  kp_.s_x = a.s_x;
  kp_.s_w = a.s_w;
  kp_.flags = a.flags;
  kp_.Y = a.Y;
  kp_.ldy = a.ldy;
  kp_.status = a.status;
  kp_.wait_limit_ns = a.wait_limit_ns;
  const int m_tiles = (a.M + geo.bt - 1) / geo.bt;
  kp_.w_streamed = m_tiles == 1;

  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(m_tiles, a.N / 128, plan.split);
  cfg.blockDim = dim3(kTsThreads, 1, 1);
  cfg.dynamicSmemBytes = geo.smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 1;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = plan.split;
  // programmatic dependent launch: weights stream (and expand) while the
  // preceding kernel finishes; its outputs are read after griddepcontrol.wait
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  return cudaLaunchKernelEx(&cfg, kernel, tm_a, tm_xo, tm_wo, tm_y, kp_);
}

}  // namespace

GemmPlan plan_gemm_w4ts(int M, int N, int K, int num_sms) {
  const int KB = K / kBlockK;
  const int n_tiles = N / 128;
  if (M <= 64) {
    const int split = decode_split(n_tiles, KB, num_sms);
    return GemmPlan{128, split, n_tiles * split, 1, 1};
  }
  if (M >= 2048) {
    // the persistent CTA-pair kernel (gemm_pair_w4.cu): 256 weight rows x 256
    // tokens per pair of SMs (measured 2 % ahead of the one-CTA 256-token
    // variant at M = 8192, even at 2048; behind it with fewer tiles)
    const int pairs = num_sms / 2;
    const int tiles = (M + 255) / 256 * ((N + 255) / 256);
    GemmPlan g{256, 1, 2 * (tiles < pairs ? tiles : pairs), 0, 0, 1};
    return g;
  }
  if (M > 1024) {
    // one CTA per SM with 256-token tiles: half the code bytes per MAC of a
    // 128-token tile
    return GemmPlan{128, 1, (M + 255) / 256 * n_tiles, 0, 1};
  }
  const int m_tiles = (M + 127) / 128;
  const int ctas = m_tiles * n_tiles;
  if (M >= 256 && ctas * 5 < num_sms * 4) {
    // too few 128-token tiles to occupy the SMs: 256-token tiles without a K
    // split (measured 1.5x the split 128-token plan at 512 x 4096 x 4096)
    return GemmPlan{128, 1, (M + 255) / 256 * n_tiles, 0, 1};
  }
  if (ctas * 5 < num_sms * 4) {
    // too few 128 x 128 tiles to occupy the SMs: split K over a cluster (the
    // one-CTA variant holds the reduction buffers of 128 tokens)
    int s = 1;
    while (s < 8 && s < KB && ctas * (s + 1) <= num_sms + num_sms / 4 && ctas * s * 5 < num_sms * 4)
      ++s;
    return GemmPlan{128, s, ctas * s, 0, 1};
  }
  // two CTAs per SM: one CTA's epilogue and pipeline fill overlap the other's
  // mainloop (measured 1.6x the one-CTA variant at 2048 x 11008 x 4096)
  return GemmPlan{128, 1, ctas, 1, 1};
}

cudaError_t launch_gemm_w4ts(const GemmArgs &a, const GemmPlan &plan, cudaStream_t stream,
                             const char **why) {
  const bool raw = a.epi == Epi::kRawI32;
  if (plan.small_m) {
    const TsGeometry geo = ts_geometry<true>(a.M);
    return raw ? launch_ts_variant<true, true>(a, plan, geo, stream, why)
               : launch_ts_variant<true, false>(a, plan, geo, stream, why);
  }
  const TsGeometry geo = ts_geometry<false>(a.M);
  return raw ? launch_ts_variant<false, true>(a, plan, geo, stream, why)
             : launch_ts_variant<false, false>(a, plan, geo, stream, why);
}

}  // namespace mixq
