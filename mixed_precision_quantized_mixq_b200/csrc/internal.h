// Internal host-side interfaces between the C ABI layer (abi.cu) and the
// kernel launchers.  Launchers assume validated arguments and return the
// cudaError_t of their launch.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace mixq {

constexpr int kGroup = 128;     // 4-bit group size along K
constexpr int kBlockK = 128;    // K per pipeline stage (bytes of INT8)
constexpr int kOutBlockK = 64;  // fp16 K per outlier stage (128 bytes)
constexpr int kTileM = 128;     // output tile rows (tcgen05 M)

inline int k_out_pad(int k_out) { return (k_out + 63) / 64 * 64; }

// ---------------------------------------------------------------- quantize
int quantize_max_k();  // largest K the quantize kernel holds in registers
// gamma != nullptr: RMS-normalise each token first (eps; optional Xn output).
cudaError_t launch_quantize_act(const void *X, int M, int K, int ldx, const int32_t *idx,
                                int K_out, float threshold, int8_t *Xq, float *s_x, void *X_out,
                                uint32_t *bitmap, int32_t *flags, int32_t *status,
                                cudaStream_t stream, int num_sms, const void *gamma = nullptr,
                                float eps = 0.f, void *Xn = nullptr, int ldxn = 0);

// The same pass with its CTA ticket in the library's static device scratch
// (flags holds the two output words only); no gamma.
cudaError_t launch_quantize_act_static(const void *X, int M, int K, int ldx, const int32_t *idx,
                                       int K_out, float threshold, int8_t *Xq, float *s_x,
                                       void *X_out, uint32_t *bitmap, int32_t *flags,
                                       int32_t *status, cudaStream_t stream, int num_sms);

// ----------------------------------------------------------------- prepack
cudaError_t launch_prepack(int mode, const void *W, int N, int K, const int32_t *idx, int K_out,
                           void *Wq, float *s_w, void *grp, void *W_out, int32_t *status,
                           cudaStream_t stream);
cudaError_t launch_extract_outliers(const void *W, int N, int K, const int32_t *idx, int K_out,
                                    void *W_out, int32_t *status, cudaStream_t stream);
cudaError_t launch_unpack_w8(int N, int K, const void *Wq, int8_t *out, cudaStream_t stream);
cudaError_t launch_unpack_w4(int N, int K, const void *Wq4, const void *grp, uint8_t *q,
                             uint8_t *s2, uint8_t *z2, cudaStream_t stream);

// -------------------------------------------------------------------- gemm
struct GemmPlan {
  int bn;       // output tile width in weight rows (32..256; always 128 for W4)
  int split;    // K split = cluster size along z (1..8)
  int ctas;     // total CTAs launched
  int small_m;  // two-CTA-per-SM kernel variant (half the shared memory and TMEM)
  int ts;       // W4 through the tensor-memory-operand kernel (gemm_w4ts.cu)
  int pair;     // W8 through the persistent CTA-pair kernel (gemm_pair.cu)
};

GemmPlan plan_gemm(int mode, int M, int N, int K, int num_sms);
// Clusters of `split` CTAs of the smem x smem kernel the current device runs at
// once (-1 on error); a diagnostic for the debug entry point.
int gemm_max_active_clusters(int mode, int bn, int split, int small_m);

enum class Epi { kMixed = 0, kRawI32 = 1 };

struct GemmArgs {
  int mode;  // 0 = W8, 1 = W4G128
  int M, N, K, K_out;
  const int8_t *Xq;
  const float *s_x;
  const void *X_out;
  const void *Wq;
  const void *grp;
  const float *s_w;
  const void *W_out;
  const int32_t *flags;
  void *Y;  // fp16 [M][ldy] or int32 [M][ldy] (raw mode)
  int ldy;
  Epi epi;
  int32_t *status;
  uint64_t wait_limit_ns;
  int debug_stall;  // producer issues nothing (timeout test)
};

// W8 runs the smem x smem kernel (gemm.cu); W4 runs the kernel that keeps the
// expanded weights in tensor memory (gemm_w4ts.cu, plan.ts = 1), except the
// narrow-tile debug launches.
cudaError_t launch_gemm(const GemmArgs &a, const GemmPlan &plan, cudaStream_t stream,
                        const char **why);
GemmPlan plan_gemm_w4ts(int M, int N, int K, int num_sms);
// K split of a decode-sized (M <= 64) launch of n_tiles 128-channel tiles.
int decode_split(int n_tiles, int KB, int num_sms);
cudaError_t launch_gemm_w4ts(const GemmArgs &a, const GemmPlan &plan, cudaStream_t stream,
                             const char **why);

// Tensor-core rate loop (mma_rate.cu): kind 0 = kind::i8, 1 = kind::f16.
double mma_rate_ops_per_launch(int kind, int iters, int num_sms);
cudaError_t launch_mma_rate(int kind, int iters, int num_sms, int32_t *status,
                            uint64_t wait_limit_ns, cudaStream_t stream);

// W8 at large M on CTA pairs (gemm_pair.cu): persistent, 256 x 256 tiles,
// tcgen05 cta_group::2.  pair_max_active: resident pairs (-1 on error).
cudaError_t launch_gemm_pair(const GemmArgs &a, cudaStream_t stream, const char **why);
int pair_max_active(int raw);
// W4 (progressive 4-bit) at large M on CTA pairs (gemm_pair_w4.cu): persistent,
// 256-weight-row x 192-token tiles, weights expanded into tensor memory.
cudaError_t launch_gemm_pair_w4(const GemmArgs &a, cudaStream_t stream, const char **why);

// Device properties cached per device.
int device_sm_count(int dev);
int device_cc_major(int dev);
size_t device_max_smem_optin(int dev);

}  // namespace mixq
