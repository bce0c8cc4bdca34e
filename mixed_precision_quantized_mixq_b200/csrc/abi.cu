// extern "C" boundary of libmixq.so (declared and documented in include/mixq.h):
// argument validation that the host can do, device checks, dispatch to the
// kernel launchers, and the thread-local error text.
#include <cuda_runtime.h>

#include <atomic>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <string>

#include "../../include/mixq.h"
#include "gemm_w4b.h"
#include "internal.h"

namespace {

thread_local std::string g_last_error = "no error";

mixq_status fail(mixq_status s, const char *fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof buf, fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return s;
}

mixq_status ok() { return MIXQ_OK; }

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

constexpr uint64_t kDefaultWaitNs = 2000000000ull;  // 2 s per pipeline wait

// Device checks: a current device with compute capability 10.x.
mixq_status check_device(int *sms) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    cudaGetLastError();
    return fail(MIXQ_ERR_NO_DEVICE, "no CUDA device is available");
  }
  if (mixq::device_cc_major(dev) != 10)
    return fail(MIXQ_ERR_NO_DEVICE, "device %d is not an sm_100 (Blackwell B200-class) GPU", dev);
  if (sms) *sms = mixq::device_sm_count(dev);
  return MIXQ_OK;
}

mixq_status from_cuda(cudaError_t e, const char *what, const char *why = nullptr) {
  if (e == cudaSuccess) return MIXQ_OK;
  return fail(MIXQ_ERR_CUDA, "%s: %s%s%s", what, cudaGetErrorString(e), why ? " -- " : "",
              why ? why : "");
}

mixq_status check_shape(int M, int N, int K, int K_out) {
  if (M < 0) return fail(MIXQ_ERR_UNSUPPORTED_SHAPE, "M = %d must be >= 0", M);
  if (N <= 0 || N % 128) return fail(MIXQ_ERR_UNSUPPORTED_SHAPE, "N = %d must be a positive multiple of 128", N);
  if (K <= 0 || K % 128) return fail(MIXQ_ERR_UNSUPPORTED_SHAPE, "K = %d must be a positive multiple of 128", K);
  if (K_out < 0 || K_out > K)
    return fail(MIXQ_ERR_UNSUPPORTED_SHAPE, "K_out = %d must lie in [0, K = %d]", K_out, K);
  return MIXQ_OK;
}

}  // namespace

namespace mixq {

namespace {
struct DevAttr {
  std::atomic<int> sms{0};
  std::atomic<int> major{-1};
  std::atomic<long long> smem{0};
};
DevAttr g_attr[64];

void fill_attr(int dev) {
  if (dev < 0 || dev >= 64) return;
  if (g_attr[dev].major.load() >= 0) return;
  int sms = 0, major = 0, smem = 0;
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
  cudaDeviceGetAttribute(&smem, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
  g_attr[dev].sms = sms;
  g_attr[dev].smem = smem;
  g_attr[dev].major = major;
}
}  // namespace

int device_sm_count(int dev) {
  fill_attr(dev);
  return dev >= 0 && dev < 64 ? g_attr[dev].sms.load() : 0;
}
int device_cc_major(int dev) {
  fill_attr(dev);
  return dev >= 0 && dev < 64 ? g_attr[dev].major.load() : 0;
}
size_t device_max_smem_optin(int dev) {
  fill_attr(dev);
  return dev >= 0 && dev < 64 ? static_cast<size_t>(g_attr[dev].smem.load()) : 0;
}

}  // namespace mixq

extern "C" {

const char *mixq_last_error(void) { return g_last_error.c_str(); }

int mixq_version(void) { return 100; }

static bool valid_mode(int mode) {
  return mode == MIXQ_W8 || mode == MIXQ_W4G128 || mode == MIXQ_W4G128_F16S;
}

mixq_status mixq_prepack_size(int mode, int N, int K, int K_out, size_t *wq_bytes,
                              size_t *grp_bytes, size_t *wout_bytes) {
  if (!valid_mode(mode)) return fail(MIXQ_ERR_INVALID_ARG, "mode = %d", mode);
  mixq_status s = check_shape(0, N, K, K_out);
  if (s != MIXQ_OK) return s;
  const size_t n = static_cast<size_t>(N), k = static_cast<size_t>(K);
  if (wq_bytes) *wq_bytes = mode == MIXQ_W8 ? n * k : n * k / 2;
  if (grp_bytes) *grp_bytes = mode == MIXQ_W8 ? 0 : 4 * n * (k / 128);
  if (wout_bytes) *wout_bytes = 2 * n * static_cast<size_t>(mixq::k_out_pad(K_out));
  return ok();
}

mixq_status mixq_prepack_weights(int mode, const void *W, int N, int K, const int32_t *idx,
                                 int K_out, void *Wq, float *s_w, void *grp, void *W_out,
                                 int32_t *status, void *stream) {
  if (!valid_mode(mode)) return fail(MIXQ_ERR_INVALID_ARG, "mode = %d", mode);
  mixq_status s = check_shape(0, N, K, K_out);
  if (s != MIXQ_OK) return s;
  if (!W || !Wq) return fail(MIXQ_ERR_INVALID_ARG, "W and Wq must be non-null");
  if (mode != MIXQ_W4G128_F16S && !s_w) return fail(MIXQ_ERR_INVALID_ARG, "s_w must be non-null");
  if (mode != MIXQ_W8 && !grp) return fail(MIXQ_ERR_INVALID_ARG, "grp must be non-null for 4-bit weights");
  if (K_out > 0 && (!idx || !W_out))
    return fail(MIXQ_ERR_INVALID_ARG, "idx and W_out must be non-null when K_out > 0");
  if (!aligned16(W) || !aligned16(Wq) || (s_w && !aligned16(s_w)) || (grp && !aligned16(grp)) ||
      (W_out && !aligned16(W_out)))
    return fail(MIXQ_ERR_MISALIGNED, "matrix pointers must be 16-byte aligned");
  s = check_device(nullptr);
  if (s != MIXQ_OK) return s;
  return from_cuda(mixq::launch_prepack(mode, W, N, K, idx, K_out, Wq, s_w, grp, W_out, status,
                                        static_cast<cudaStream_t>(stream)),
                   "prepack launch");
}

mixq_status mixq_extract_outlier_weights(const void *W, int N, int K, const int32_t *idx,
                                         int K_out, void *W_out, int32_t *status,
                                         void *stream) {
  mixq_status s = check_shape(0, N, K, K_out);
  if (s != MIXQ_OK) return s;
  if (K_out == 0) return ok();
  if (!W || !idx || !W_out) return fail(MIXQ_ERR_INVALID_ARG, "W, idx and W_out must be non-null");
  if (!aligned16(W) || !aligned16(W_out))
    return fail(MIXQ_ERR_MISALIGNED, "W and W_out must be 16-byte aligned");
  s = check_device(nullptr);
  if (s != MIXQ_OK) return s;
  return from_cuda(mixq::launch_extract_outliers(W, N, K, idx, K_out, W_out, status,
                                                 static_cast<cudaStream_t>(stream)),
                   "outlier extraction launch");
}

mixq_status mixq_merge_outliers(const uint32_t *detect_bitmap, int K, const int32_t *idx,
                                int K_out, int32_t *idx_new, int *K_out_new) {
  if (K <= 0 || K % 32 || K_out < 0 || K_out > K || !detect_bitmap || !idx_new || !K_out_new ||
      (K_out > 0 && !idx))
    return fail(MIXQ_ERR_INVALID_ARG, "merge: bad K, K_out or null pointer");
  // sorted union of idx and the detected channels: one pass over the channels
  int j = 0, n = 0;
  for (int c = 0; c < K; ++c) {
    bool in_idx = false;
    if (j < K_out && idx[j] == c) {
      in_idx = true;
      ++j;
    } else if (j < K_out && (idx[j] < c || idx[j] >= K || (j > 0 && idx[j] <= idx[j - 1]))) {
      return fail(MIXQ_ERR_INVALID_ARG, "merge: idx must be sorted, unique, inside [0, K)");
    }
    const bool detected = (detect_bitmap[c >> 5] >> (c & 31)) & 1u;
    if (in_idx || detected) idx_new[n++] = c;
  }
  if (j != K_out) return fail(MIXQ_ERR_INVALID_ARG, "merge: idx must be sorted, unique, inside [0, K)");
  *K_out_new = n;
  return ok();
}

static mixq_status quantize_common(const void *X, int M, int K, int ldx, const int32_t *idx,
                                   int K_out, float threshold, int8_t *Xq, float *s_x,
                                   void *X_out, uint32_t *detect_bitmap, int32_t *flags,
                                   int32_t *status, void *stream, const void *gamma, float eps,
                                   void *Xn, int ldxn) {
  mixq_status s = check_shape(M, 128, K, K_out);
  if (s != MIXQ_OK) return s;
  if (K > mixq::quantize_max_k())
    return fail(MIXQ_ERR_UNSUPPORTED_SHAPE, "K = %d exceeds %d for mixq_quantize_act", K,
                mixq::quantize_max_k());
  if (ldx < K || ldx % 8) return fail(MIXQ_ERR_INVALID_ARG, "ldx = %d must be >= K and a multiple of 8", ldx);
  if (!(threshold >= 0.f) || threshold != threshold)
    return fail(MIXQ_ERR_INVALID_ARG, "threshold must be a finite value >= 0");
  if (!detect_bitmap || !flags) return fail(MIXQ_ERR_INVALID_ARG, "detect_bitmap and flags must be non-null");
  if (M > 0 && (!X || !Xq || !s_x)) return fail(MIXQ_ERR_INVALID_ARG, "X, Xq and s_x must be non-null");
  if (K_out > 0 && !idx) return fail(MIXQ_ERR_INVALID_ARG, "idx must be non-null when K_out > 0");
  if (K_out > 0 && M > 0 && !X_out) return fail(MIXQ_ERR_INVALID_ARG, "X_out must be non-null when K_out > 0");
  if (Xn && (ldxn < K || ldxn % 8))
    return fail(MIXQ_ERR_INVALID_ARG, "ldxn = %d must be >= K and a multiple of 8", ldxn);
  if ((X && !aligned16(X)) || (Xq && !aligned16(Xq)) || (X_out && !aligned16(X_out)) ||
      !aligned16(detect_bitmap) || !aligned16(flags) || (gamma && !aligned16(gamma)) ||
      (Xn && !aligned16(Xn)))
    return fail(MIXQ_ERR_MISALIGNED, "matrix pointers must be 16-byte aligned");
  int sms = 0;
  s = check_device(&sms);
  if (s != MIXQ_OK) return s;
  return from_cuda(mixq::launch_quantize_act(X, M, K, ldx, idx, K_out, threshold, Xq, s_x, X_out,
                                             detect_bitmap, flags, status,
                                             static_cast<cudaStream_t>(stream), sms, gamma, eps,
                                             Xn, ldxn),
                   "quantize launch");
}

mixq_status mixq_quantize_act(const void *X, int M, int K, int ldx, const int32_t *idx, int K_out,
                              float threshold, int8_t *Xq, float *s_x, void *X_out,
                              uint32_t *detect_bitmap, int32_t *flags, int32_t *status,
                              void *stream) {
  return quantize_common(X, M, K, ldx, idx, K_out, threshold, Xq, s_x, X_out, detect_bitmap,
                         flags, status, stream, nullptr, 0.f, nullptr, 0);
}

mixq_status mixq_rmsnorm_quantize_act(const void *X, int M, int K, int ldx, const void *gamma,
                                      float eps, void *Xn, int ldxn, const int32_t *idx,
                                      int K_out, float threshold, int8_t *Xq, float *s_x,
                                      void *X_out, uint32_t *detect_bitmap, int32_t *flags,
                                      int32_t *status, void *stream) {
  if (!gamma) return fail(MIXQ_ERR_INVALID_ARG, "gamma must be non-null");
  if (!(eps >= 0.f) || eps != eps || eps > 3.0e38f)
    return fail(MIXQ_ERR_INVALID_ARG, "eps must be a finite value >= 0");
  return quantize_common(X, M, K, ldx, idx, K_out, threshold, Xq, s_x, X_out, detect_bitmap,
                         flags, status, stream, gamma, eps, Xn, ldxn);
}

mixq_status mixq_quantize_act_static(const void *X, int M, int K, int ldx, const int32_t *idx,
                                     int K_out, float threshold, int8_t *Xq, float *s_x,
                                     void *X_out, uint32_t *detect_bitmap, int32_t *flags,
                                     int32_t *status, void *stream) {
  mixq_status s = check_shape(M, 128, K, K_out);
  if (s != MIXQ_OK) return s;
  if (K > mixq::quantize_max_k())
    return fail(MIXQ_ERR_UNSUPPORTED_SHAPE, "K = %d exceeds %d for mixq_quantize_act_static", K,
                mixq::quantize_max_k());
  if (ldx < K || ldx % 8) return fail(MIXQ_ERR_INVALID_ARG, "ldx = %d must be >= K and a multiple of 8", ldx);
  if (!(threshold >= 0.f) || threshold != threshold)
    return fail(MIXQ_ERR_INVALID_ARG, "threshold must be a finite value >= 0");
  if (!detect_bitmap || !flags) return fail(MIXQ_ERR_INVALID_ARG, "detect_bitmap and flags must be non-null");
  if (M > 0 && (!X || !Xq || !s_x)) return fail(MIXQ_ERR_INVALID_ARG, "X, Xq and s_x must be non-null");
  if (K_out > 0 && !idx) return fail(MIXQ_ERR_INVALID_ARG, "idx must be non-null when K_out > 0");
  if (K_out > 0 && M > 0 && !X_out) return fail(MIXQ_ERR_INVALID_ARG, "X_out must be non-null when K_out > 0");
  if ((X && !aligned16(X)) || (Xq && !aligned16(Xq)) || (X_out && !aligned16(X_out)) ||
      !aligned16(detect_bitmap) || (reinterpret_cast<uintptr_t>(flags) & 3u))
    return fail(MIXQ_ERR_MISALIGNED,
                "matrix pointers must be 16-byte aligned and flags 4-byte aligned");
  int sms = 0;
  s = check_device(&sms);
  if (s != MIXQ_OK) return s;
  return from_cuda(mixq::launch_quantize_act_static(X, M, K, ldx, idx, K_out, threshold, Xq, s_x,
                                                    X_out, detect_bitmap, flags, status,
                                                    static_cast<cudaStream_t>(stream), sms),
                   "quantize (static scratch) launch");
}

static mixq_status gemm_common(int mode, int M, int N, int K, int K_out, const int8_t *Xq,
                               const float *s_x, const void *X_out, const void *Wq,
                               const void *grp, const float *s_w, const void *W_out,
                               const int32_t *flags, void *Y, int ldy, int32_t *status,
                               void *stream) {
  mixq_status s = check_shape(M, N, K, K_out);
  if (s != MIXQ_OK) return s;
  if (ldy < N || ldy % 8) return fail(MIXQ_ERR_INVALID_ARG, "ldy = %d must be >= N and a multiple of 8", ldy);
  if (M == 0) return check_device(nullptr);
  if (!Xq || !s_x || !Wq || !Y || (mode != MIXQ_W4G128_F16S && !s_w))
    return fail(MIXQ_ERR_INVALID_ARG, "Xq, s_x, Wq, s_w and Y must be non-null");
  if (mode != MIXQ_W8 && !grp) return fail(MIXQ_ERR_INVALID_ARG, "grp must be non-null");
  if (K_out > 0 && (!X_out || !W_out))
    return fail(MIXQ_ERR_INVALID_ARG, "X_out and W_out must be non-null when K_out > 0");
  if (!aligned16(Xq) || !aligned16(Wq) || !aligned16(Y) || (s_w && !aligned16(s_w)) ||
      (grp && !aligned16(grp)) || (X_out && !aligned16(X_out)) || (W_out && !aligned16(W_out)))
    return fail(MIXQ_ERR_MISALIGNED, "matrix pointers must be 16-byte aligned");
  int sms = 0;
  s = check_device(&sms);
  if (s != MIXQ_OK) return s;
  mixq::GemmArgs a{};
  a.mode = mode;
  a.M = M;
  a.N = N;
  a.K = K;
  a.K_out = K_out;
  a.Xq = Xq;
  a.s_x = s_x;
  a.X_out = X_out;
  a.Wq = Wq;
  a.grp = grp;
  a.s_w = s_w;
  a.W_out = W_out;
  a.flags = flags;
  a.Y = Y;
  a.ldy = ldy;
  a.epi = mixq::Epi::kMixed;
  a.status = status;
  a.wait_limit_ns = kDefaultWaitNs;
  const char *why = nullptr;
  if (mode == MIXQ_W4G128_F16S) {
    const mixq::GemmPlan plan = mixq::plan_gemm_w4b(M, N, K, sms);
    const cudaError_t e = mixq::launch_gemm_w4b(a, plan, static_cast<cudaStream_t>(stream), &why);
    return from_cuda(e, "gemm launch", why);
  }
  const mixq::GemmPlan plan = mixq::plan_gemm(mode, M, N, K, sms);
  const cudaError_t e = mixq::launch_gemm(a, plan, static_cast<cudaStream_t>(stream), &why);
  return from_cuda(e, "gemm launch", why);
}

mixq_status mixq_gemm_w8a8o16(int M, int N, int K, int K_out, const int8_t *Xq, const float *s_x,
                              const void *X_out, const void *Wq, const float *s_w,
                              const void *W_out, const int32_t *flags, void *Y, int ldy,
                              int32_t *status, void *stream) {
  return gemm_common(MIXQ_W8, M, N, K, K_out, Xq, s_x, X_out, Wq, nullptr, s_w, W_out, flags, Y,
                     ldy, status, stream);
}

mixq_status mixq_gemm_w4a8o16(int M, int N, int K, int K_out, const int8_t *Xq, const float *s_x,
                              const void *X_out, const void *Wq4, const void *grp,
                              const float *s_w, const void *W_out, const int32_t *flags, void *Y,
                              int ldy, int32_t *status, void *stream) {
  return gemm_common(MIXQ_W4G128, M, N, K, K_out, Xq, s_x, X_out, Wq4, grp, s_w, W_out, flags, Y,
                     ldy, status, stream);
}

mixq_status mixq_gemm_w4a8o16_f16s(int M, int N, int K, int K_out, const int8_t *Xq,
                                   const float *s_x, const void *X_out, const void *Wq4,
                                   const void *grp, const void *W_out, const int32_t *flags,
                                   void *Y, int ldy, int32_t *status, void *stream) {
  return gemm_common(MIXQ_W4G128_F16S, M, N, K, K_out, Xq, s_x, X_out, Wq4, grp, nullptr, W_out,
                     flags, Y, ldy, status, stream);
}

size_t mixq_gemm_workspace_size(int M, int N, int K) {
  (void)M;
  (void)N;
  (void)K;
  return 0;
}

mixq_status mixq_gemm_plan(int mode, int M, int N, int K, int num_sms, int *bn, int *split,
                           int *ctas) {
  if (!valid_mode(mode)) return fail(MIXQ_ERR_INVALID_ARG, "mode = %d", mode);
  mixq_status s = check_shape(M, N, K, 0);
  if (s != MIXQ_OK) return s;
  if (num_sms <= 0) {
    s = check_device(&num_sms);
    if (s != MIXQ_OK) return s;
  }
  const mixq::GemmPlan p = mode == MIXQ_W4G128_F16S ? mixq::plan_gemm_w4b(M, N, K, num_sms)
                                                   : mixq::plan_gemm(mode, M, N, K, num_sms);
  if (bn) *bn = p.bn;
  if (split) *split = p.split;
  if (ctas) *ctas = p.ctas;
  return ok();
}

mixq_status mixq_debug_max_active_clusters(int mode, int bn, int split, int small_m,
                                           int *clusters) {
  if ((mode != MIXQ_W8 && mode != MIXQ_W4G128) ||
      (bn != 32 && bn != 64 && bn != 128 && bn != 256) || split < 1 || split > 8 || !clusters ||
      (small_m && bn == 256) || (!small_m && bn < 128))
    return fail(MIXQ_ERR_INVALID_ARG, "bad mode/bn/split/small_m/pointer");
  mixq_status s = check_device(nullptr);
  if (s != MIXQ_OK) return s;
  *clusters = mixq::gemm_max_active_clusters(mode, bn, split, small_m);
  if (*clusters < 0) return fail(MIXQ_ERR_CUDA, "cudaOccupancyMaxActiveClusters failed");
  return ok();
}

mixq_status mixq_debug_gemm_i32(int mode, int M, int N, int K, const int8_t *Xq, const void *Wq,
                                const void *grp, int32_t *acc, int ldacc, int bn, int split,
                                int32_t *status, void *stream) {
  if (mode != MIXQ_W8 && mode != MIXQ_W4G128) return fail(MIXQ_ERR_INVALID_ARG, "mode = %d", mode);
  mixq_status s = check_shape(M, N, K, 0);
  if (s != MIXQ_OK) return s;
  if (ldacc < N || ldacc % 4) return fail(MIXQ_ERR_INVALID_ARG, "ldacc = %d must be >= N and a multiple of 4", ldacc);
  if (bn != 0 && bn != 32 && bn != 64 && bn != 128 && bn != 256 && bn != 512)
    return fail(MIXQ_ERR_INVALID_ARG, "bn = %d", bn);
  if (bn == 512 && split > 1)
    return fail(MIXQ_ERR_INVALID_ARG, "bn = 512 (the CTA-pair kernels) takes no K split");
  if ((bn == 32 || bn == 64) && M > 64)
    return fail(MIXQ_ERR_INVALID_ARG, "bn = %d needs M <= 64", bn);
  if (split < 0 || split > 8)
    return fail(MIXQ_ERR_INVALID_ARG, "split = %d", split);
  if (split > K / 128) return fail(MIXQ_ERR_UNSUPPORTED_SHAPE, "split %d exceeds K/128", split);
  if (mode == MIXQ_W4G128 && bn == 128 && split > 1 && M > 64)
    return fail(MIXQ_ERR_UNSUPPORTED_SHAPE,
                "W4 two-CTA variant (bn = 128) splits K only for M <= 64");
  if (mode == MIXQ_W4G128 && bn == 256 && split > 1 && M > 1024)
    return fail(MIXQ_ERR_UNSUPPORTED_SHAPE,
                "W4 one-CTA variant (bn = 256) splits K only for M <= 1024");
  if (M == 0) return check_device(nullptr);
  if (!Xq || !Wq || !acc || (mode == MIXQ_W4G128 && !grp))
    return fail(MIXQ_ERR_INVALID_ARG, "null pointer");
  if (!aligned16(Xq) || !aligned16(Wq) || !aligned16(acc) || (grp && !aligned16(grp)))
    return fail(MIXQ_ERR_MISALIGNED, "matrix pointers must be 16-byte aligned");
  int sms = 0;
  s = check_device(&sms);
  if (s != MIXQ_OK) return s;
  mixq::GemmPlan plan = mixq::plan_gemm(mode, M, N, K, sms);
  if (split) plan.split = split;
  if (bn == 512) {
    plan.pair = 1;
  } else if (bn != 0 || split != 0) {
    plan.pair = 0;
  }
  if (plan.pair) {
    // the CTA-pair kernel
  } else if (mode == MIXQ_W4G128 && (bn == 128 || bn == 256 || (bn == 0 && plan.ts))) {
    // tensor-memory-operand kernel: bn = 128 the two-CTA-per-SM variant,
    // 256 the one-CTA variant, 0 the planner's choice
    if (bn == 128) plan.small_m = 1;
    if (bn == 256) plan.small_m = 0;
    plan.bn = 128;
    plan.ts = 1;
  } else {
    plan.ts = 0;
    if (bn) plan.bn = bn;
    // two-CTA-per-SM variant for bn <= 128, except a K split with more rows
    // than its reduction buffers hold (64)
    if (bn || split) plan.small_m = (plan.bn <= 128 && (M <= 64 || plan.split == 1)) ? 1 : 0;
  }
  mixq::GemmArgs a{};
  a.mode = mode;
  a.M = M;
  a.N = N;
  a.K = K;
  a.Xq = Xq;
  a.Wq = Wq;
  a.grp = grp;
  a.Y = acc;
  a.ldy = ldacc;
  a.epi = mixq::Epi::kRawI32;
  a.status = status;
  a.wait_limit_ns = kDefaultWaitNs;
  const char *why = nullptr;
  const cudaError_t e = mixq::launch_gemm(a, plan, static_cast<cudaStream_t>(stream), &why);
  return from_cuda(e, "debug gemm launch", why);
}

mixq_status mixq_debug_unpack_w8(int N, int K, const void *Wq, int8_t *out, void *stream) {
  mixq_status s = check_shape(0, N, K, 0);
  if (s != MIXQ_OK) return s;
  if (!Wq || !out) return fail(MIXQ_ERR_INVALID_ARG, "null pointer");
  s = check_device(nullptr);
  if (s != MIXQ_OK) return s;
  return from_cuda(mixq::launch_unpack_w8(N, K, Wq, out, static_cast<cudaStream_t>(stream)),
                   "unpack launch");
}

mixq_status mixq_debug_unpack_w4(int N, int K, const void *Wq4, const void *grp, uint8_t *q,
                                 uint8_t *s2, uint8_t *z2, int32_t *status, void *stream) {
  (void)status;
  mixq_status s = check_shape(0, N, K, 0);
  if (s != MIXQ_OK) return s;
  if (!Wq4 || !grp || !q || !s2 || !z2) return fail(MIXQ_ERR_INVALID_ARG, "null pointer");
  s = check_device(nullptr);
  if (s != MIXQ_OK) return s;
  return from_cuda(mixq::launch_unpack_w4(N, K, Wq4, grp, q, s2, z2,
                                          static_cast<cudaStream_t>(stream)),
                   "unpack launch");
}

mixq_status mixq_debug_gemm_stall(int M, int N, int K, const int8_t *Xq, const void *Wq,
                                  const float *s_x, const float *s_w, void *Y, int ldy,
                                  uint64_t wait_limit_ns, int32_t *status, void *stream) {
  mixq_status s = check_shape(M, N, K, 0);
  if (s != MIXQ_OK) return s;
  if (M == 0 || !Xq || !Wq || !s_x || !s_w || !Y || !status)
    return fail(MIXQ_ERR_INVALID_ARG, "null pointer or M == 0");
  if (ldy < N || ldy % 8) return fail(MIXQ_ERR_INVALID_ARG, "ldy");
  if (wait_limit_ns == 0 || wait_limit_ns > kDefaultWaitNs)
    return fail(MIXQ_ERR_INVALID_ARG, "wait_limit_ns must lie in (0, 2 s]");
  int sms = 0;
  s = check_device(&sms);
  if (s != MIXQ_OK) return s;
  mixq::GemmArgs a{};
  a.mode = MIXQ_W8;
  a.M = M;
  a.N = N;
  a.K = K;
  a.Xq = Xq;
  a.Wq = Wq;
  a.s_x = s_x;
  a.s_w = s_w;
  a.Y = Y;
  a.ldy = ldy;
  a.epi = mixq::Epi::kMixed;
  a.status = status;
  a.wait_limit_ns = wait_limit_ns;
  a.debug_stall = 1;
  mixq::GemmPlan plan = mixq::plan_gemm(MIXQ_W8, M, N, K, sms);
  plan.split = 1;
  plan.bn = 128;
  plan.small_m = M <= 64 ? 1 : 0;
  const char *why = nullptr;
  const cudaError_t e = mixq::launch_gemm(a, plan, static_cast<cudaStream_t>(stream), &why);
  return from_cuda(e, "stall gemm launch", why);
}

mixq_status mixq_debug_mma_rate(int kind, int iters, double *ops, int32_t *status, void *stream) {
  if (kind != 0 && kind != 1) return fail(MIXQ_ERR_INVALID_ARG, "kind = %d must be 0 or 1", kind);
  if (iters < 1 || iters > (1 << 20))
    return fail(MIXQ_ERR_INVALID_ARG, "iters = %d must lie in [1, 1048576]", iters);
  if (!ops) return fail(MIXQ_ERR_INVALID_ARG, "ops must be non-null");
  int sms = 0;
  mixq_status s = check_device(&sms);
  if (s != MIXQ_OK) return s;
  *ops = mixq::mma_rate_ops_per_launch(kind, iters, sms);
  return from_cuda(mixq::launch_mma_rate(kind, iters, sms, status, kDefaultWaitNs,
                                         static_cast<cudaStream_t>(stream)),
                   "mma rate launch");
}

}  // extern "C"
