/*
 * mixq.h -- C ABI of libmixq.so, the B200 (sm_100a) outlier-decomposed
 * mixed-precision quantized linear layer.
 *
 * The layer (MixQ article "一键部署LLM混合精度推理，端到端吞吐比AWQ最大提升6倍！",
 * 研究背景 Fig. 5 and MixQ的解决方案 Figs. 10-12) splits Y = X W^T into
 *   Y = diag(s_x) (Xq Wq^T) diag(s_w) + X_out W_out^T
 * where Xq/Wq are INT8 codes of the dense part, and X_out/W_out hold the few
 * fixed outlier channels, concatenated in their original order, in FP16.  The
 * W4A8 variant (QServe W4A8KV4 reading notes, 渐进量化 / 寄存器压力和并行性;
 * MixLLM page, "MixLLM: Ein neuer Ansatz") stores Wq as 4-bit group codes and
 * expands them back to INT8 inside the GEMM mainloop, so every product still
 * runs on INT8 tensor cores.
 *
 * Conventions for every call:
 *   - All matrix pointers are DEVICE pointers owned by the caller; the library
 *     allocates no device memory, keeps no state between calls (beyond cached
 *     device attributes and a thread-local error string) and needs no
 *     workspace.  Matrix pointers must be 16-byte aligned.
 *   - fp16 data is IEEE binary16, passed as void*.  Matrices are row-major.
 *   - Every call is asynchronous on `stream` (a cudaStream_t passed as void*;
 *     NULL = the legacy default stream).  Errors a host can see (bad sizes,
 *     null or misaligned pointers, no device) return synchronously as a
 *     mixq_status and leave the stream untouched.  Errors only the device can
 *     see (an invalid outlier list, a wait that ran out of time) are written
 *     to `*status` (a device int32 the caller zeroes; the first error wins;
 *     may be NULL to ignore them); read it after synchronizing the stream.
 *   - mixq_last_error() returns a thread-local description of the last
 *     non-OK status returned on the calling thread.
 *   - Calls that share output buffers must not overlap on the GPU.
 *   - Kernels are launched with programmatic dependent launch: a call's
 *     kernels may begin while the preceding kernel on the stream finishes, and
 *     wait for it before reading its outputs.  The gemm calls start streaming
 *     the prepacked weights (Wq, grp) before that wait, and the activation
 *     passes read the outlier list idx before it, so those buffers must not be
 *     written by the kernel immediately preceding the call.
 *
 * Shape rules (MIXQ_ERR_UNSUPPORTED_SHAPE otherwise): K % 128 == 0, K > 0,
 * N % 128 == 0, N > 0, M >= 0, 0 <= K_out <= K.  K_out_pad is K_out rounded up
 * to a multiple of 64; the padding columns of X_out / W_out are zero-filled by
 * the library.
 */
#ifndef MIXQ_H
#define MIXQ_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum mixq_status {
  MIXQ_OK = 0,
  MIXQ_ERR_INVALID_ARG = 1,      /* null pointer, bad leading dimension, bad mode, bad idx */
  MIXQ_ERR_UNSUPPORTED_SHAPE = 2,/* violates the shape rules above */
  MIXQ_ERR_MISALIGNED = 3,       /* a matrix pointer or row pitch is not 16-byte aligned */
  MIXQ_ERR_CUDA = 4,             /* a CUDA runtime/driver call failed (see mixq_last_error) */
  MIXQ_ERR_TIMEOUT = 5,          /* device only: a pipeline wait ran out of time */
  MIXQ_ERR_NO_DEVICE = 6         /* no usable sm_100 device is current */
} mixq_status;

/* Weight formats.  MIXQ_W4G128 is the progressive 4-bit format (integer
 * group scale s2 over per-row INT8 codes, reading A); MIXQ_W4G128_F16S is
 * the 4-bit format with a real fp16 scale and an integer zero per group
 * (MixLLM page, "MixLLM: Ein neuer Ansatz", reading B). */
enum { MIXQ_W8 = 0, MIXQ_W4G128 = 1, MIXQ_W4G128_F16S = 2 };

/* Thread-local text for the last non-OK status returned on this thread. */
const char *mixq_last_error(void);

/* ABI version (major*100 + minor). */
int mixq_version(void);

/*
 * Sizes of the prepacked weight buffers for mode, N, K, K_out (host only).
 *   *wq_bytes   MIXQ_W8: N*K (int8 codes, tiled, see mixq_prepack_weights).
 *               MIXQ_W4G128, MIXQ_W4G128_F16S: N*K/2 (two 4-bit codes per
 *               byte, tiled).
 *   *grp_bytes  4-bit formats: 4*N*(K/128) (one fp16 pair per group,
 *               group-major [K/128][N]); MIXQ_W8: 0.
 *   *wout_bytes 2*N*K_out_pad (fp16 [N][K_out_pad]).
 * Any output pointer may be NULL.
 */
mixq_status mixq_prepack_size(int mode, int N, int K, int K_out, size_t *wq_bytes,
                              size_t *grp_bytes, size_t *wout_bytes);

/*
 * Offline weight prepack (MixQ Fig. 5: weights in low bits; Fig. 11: outlier
 * columns extracted in original order; QServe 渐进量化 + group-wise: 4-bit level).
 *   W      fp16 [N][K]           input weights (read only)
 *   idx    int32 [K_out]          outlier channels, sorted ascending, unique,
 *                                 inside [0, K) (checked on the device)
 *   Wq     codes in a tiled layout made for the GEMM's bulk copies (QServe
 *          notes, compute-aware weight reordering): tiles of 128 output
 *          channels x 128 K, tile (n/128, k/128) at tile index
 *          (n/128)*(K/128) + k/128, each tile contiguous.
 *          MIXQ_W8: code = clamp(rint(W * 127/a), -127, 127) with a =
 *          max_k |W[n,k]| over all K; 16 KB tiles, row r = n%128 at r*128, the
 *          16-byte chunk of K offsets 16j..16j+15 at chunk position j^(r%8).
 *          MIXQ_W4G128: 4-bit level-2 codes q; 8 KB tiles, row r at r*64, the
 *          16-byte chunk c (K offsets 32c..32c+31) at chunk position
 *          c^((r/2)%4); inside it byte 4w+i holds q at K offset 32c+8w+i in
 *          its low nibble and q at 32c+8w+4+i in its high nibble.
 *          MIXQ_W4G128_F16S: its 4-bit codes q in the same layout.
 *          mixq_debug_unpack_w8 / _w4 return the logical codes.
 *   s_w    fp32 [N]               a / 127 (MIXQ_W4G128_F16S: unused, may be NULL)
 *   grp    4-bit formats only (else NULL): one fp16 pair per row and group of
 *          128 K, at [g][n].
 *          MIXQ_W4G128: (s2, z2) with s2 = max(1, ceil((hi-lo)/15)),
 *          z2 = clamp(rint(-lo/s2), 0, 15) over the group's INT8 codes, and
 *          q = clamp(rint(w8/s2)+z2, qlo, qhi) so the effective weight
 *          (q - z2)*s2 always fits int8.
 *          MIXQ_W4G128_F16S (MixLLM page, "MixLLM: Ein neuer Ansatz": 4-bit
 *          asymmetric group-wise weights, two-step dequantization): (s, z)
 *          straight from the fp16 weights, with lo = min(0, min W) and
 *          hi = max(0, max W) over the group, s = fp16(fp32(hi - lo) / 15),
 *          z = clamp(rint(-lo/s), 0, 15), q = clamp(rint(W/s) + z, 0, 15), all
 *          in fp32; s == 0 (an all-zero group, or a range below the fp16
 *          range) gives z = q = 0.  The effective weight is s*(q - z).
 *   W_out  fp16 [N][K_out_pad]    W[:, idx[j]] for j < K_out, zero after; may be
 *                                 NULL when K_out == 0.
 */
mixq_status mixq_prepack_weights(int mode, const void *W, int N, int K, const int32_t *idx,
                                 int K_out, void *Wq, float *s_w, void *grp, void *W_out,
                                 int32_t *status, void *stream);

/*
 * Fused amax + threshold test + outlier gather + INT8 quantization of the
 * activations (MixQ MixQ的解决方案: the amax taken for quantization shows
 * whether outliers exist; Fig. 10 equivalent transformation; Fig. 11 order-
 * preserved outlier matrix).  Per token m:
 *   aI = max_{k in idx} |x|, aN = max_{k not in idx} |x|
 *   mixed = K_out > 0 && max(aI, aN) > threshold        (strictly greater)
 *   a = mixed ? aN : max(aI, aN),  s_x[m] = a / 127
 *   Xq[m,k] = (mixed && k in idx) ? 0 : clamp(rint(x * 127/a), -127, 127)
 *   X_out[m,j] = (mixed && j < K_out) ? X[m, idx[j]] : 0
 *   X              fp16 [M][ldx], ldx >= K, ldx % 8 == 0 (read only)
 *   Xq             int8 [M][K]
 *   s_x            fp32 [M]
 *   X_out          fp16 [M][K_out_pad] (may be NULL when K_out == 0)
 *   detect_bitmap  uint32 [ceil(K/32)]: bit k%32 of word k/32 is set iff some
 *                  token has |X[m,k]| > threshold (written, not accumulated)
 *   flags          int32 [4]: [0] = number of mixed tokens, [1] = number of
 *                  detected channels that are not in idx, [2] and [3] are used
 *                  by the call and read 0 when it completes.  gemm calls read
 *                  flags[0] on the device to skip the FP16 slice when no
 *                  token is mixed.
 * K must not exceed 32768 (a token's row is held in registers).
 * When one thread-block cluster of at most 16 CTAs covers the matrix the call
 * is one kernel: M <= 64 with K <= 4096 (2 tokens per CTA up to M = 32, 4
 * above), M <= 16 with K <= 16384 (1 token per CTA), M <= 32 with K <= 12288
 * (2 tokens per CTA); otherwise it is a 1-block reset of bitmap/flags
 * followed by the main pass.
 */
mixq_status mixq_quantize_act(const void *X, int M, int K, int ldx, const int32_t *idx, int K_out,
                              float threshold, int8_t *Xq, float *s_x, void *X_out,
                              uint32_t *detect_bitmap, int32_t *flags, int32_t *status,
                              void *stream);

/*
 * mixq_quantize_act for callers that cannot allocate device memory.  It has
 * no counterpart in the pages; it exists for callers that hold only the
 * layer's own input and output buffers and cannot add a scratch buffer: a
 * plugin of an inference runtime that is handed fixed, pre-planned buffers,
 * code whose device memory belongs to another allocator (a framework's
 * caching allocator or a static arena) that it may not call from here, or a
 * hot path on which a cudaMalloc, which can synchronize the device, is not
 * acceptable.  mixq_quantize_act asks the caller for two extra flag words
 * (flags[2], flags[3]) that its multi-CTA pass uses as a completion ticket;
 * this entry keeps that ticket in a 256-byte array inside the library
 * instead, and calls no cudaMalloc, cudaFree or other allocating routine.
 *   Arguments, outputs and shape limits are those of mixq_quantize_act,
 *   except flags, which is int32 [2] here ([0] mixed tokens, [1] detected
 *   channels outside idx; 4-byte aligned).  The scratch needs one word
 *   whatever the shape, so no shape exceeds it; K > 32768 is rejected with
 *   MIXQ_ERR_UNSUPPORTED_SHAPE, as by mixq_quantize_act.
 *   Scratch: int32 [64] (256 bytes) per device, held by every device that
 *   loads the library until the process exits.  The first call on a device
 *   looks up the array's device address (cudaGetSymbolAddress, with that
 *   device current), which can load the library's kernels on it: make that
 *   first call before any stream capture.  Every call shares the array and
 *   it keeps the last call's contents; each call clears the ticket before
 *   using it.  Calls that overlap on the GPU (two streams, or two host
 *   threads on one device) race on the array: serialise them.
 */
mixq_status mixq_quantize_act_static(const void *X, int M, int K, int ldx, const int32_t *idx,
                                     int K_out, float threshold, int8_t *Xq, float *s_x,
                                     void *X_out, uint32_t *detect_bitmap, int32_t *flags,
                                     int32_t *status, void *stream);

/*
 * The activation pass with the preceding RMS normalisation absorbed (MixQ
 * article, MixQ的解决方案: the quantization amax can be taken inside the
 * operation before the layer).  Per token, in fp32 with IEEE division and
 * square root:
 *   Xn[m,k] = fp16( X[m,k] / sqrt(mean_k X[m,k]^2 + eps) * gamma[k] )
 * then exactly mixq_quantize_act on Xn (same outputs, same launches).  X is
 * read once and Xn never has to go through HBM; it is written only when
 * Xn != NULL (ldxn >= K, multiple of 8).  A row whose mean square plus eps is
 * 0 normalises to zeros.
 *   gamma fp16 [K] (16-byte aligned, non-null), eps finite >= 0; the other
 *   arguments as mixq_quantize_act.  Errors: MIXQ_ERR_INVALID_ARG for a null
 *   gamma or a bad eps/ldxn, otherwise as mixq_quantize_act.
 */
mixq_status mixq_rmsnorm_quantize_act(const void *X, int M, int K, int ldx, const void *gamma,
                                      float eps, void *Xn, int ldxn, const int32_t *idx,
                                      int K_out, float threshold, int8_t *Xq, float *s_x,
                                      void *X_out, uint32_t *detect_bitmap, int32_t *flags,
                                      int32_t *status, void *stream);

/*
 * Outlier set kept across decode steps (MixQ article, MixQ的解决方案 Fig. 9:
 * outliers recur in the same channels, so the set is found once and reused).
 * When a step reports detections outside the set (flags[1] > 0), the set
 * grows by those channels and the outlier weight columns are rebuilt; the
 * INT8 / 4-bit codes stay as they are (the weight range covers all columns).
 *
 * mixq_merge_outliers (host memory only, no GPU): idx_new = sorted union of
 * idx (sorted, unique, in [0, K)) and the channels whose bit is set in
 * detect_bitmap [K/32] (bit k%32 of word k/32).  idx_new has room for K
 * entries; *K_out_new receives the count.  MIXQ_ERR_INVALID_ARG for a bad K,
 * an unsorted idx or a null pointer.
 */
mixq_status mixq_merge_outliers(const uint32_t *detect_bitmap, int K, const int32_t *idx,
                                int K_out, int32_t *idx_new, int *K_out_new);

/*
 * mixq_extract_outlier_weights (device): W_out [N][K_out_pad] fp16 =
 * W[:, idx[j]] for j < K_out in idx order, +0.0 up to K_out_pad (the W_out
 * of mixq_prepack_weights for a new idx).  W fp16 [N][K] (the full-precision
 * weights), idx device int32 [K_out] sorted, unique, in [0, K) (else
 * MIXQ_ERR_INVALID_ARG in *status).  Pointers 16-byte aligned.
 */
mixq_status mixq_extract_outlier_weights(const void *W, int N, int K, const int32_t *idx,
                                         int K_out, void *W_out, int32_t *status, void *stream);

/*
 * Mixed-precision GEMM, 8-bit weights (MixQ Fig. 5 decomposition; Fig. 12
 * fused dequantize, scale and add of the INT32 result in registers):
 *   acc[m,n] = sum_k Xq[m,k] Wq[n,k]                     (exact INT32, tcgen05 kind::i8)
 *   o[m,n]   = sum_j X_out[m,j] W_out[n,j]               (fp32, tcgen05 kind::f16;
 *                                                         skipped if flags[0] == 0)
 *   Y[m,n]   = fp16((float(acc) * s_x[m]) * s_w[n] + o)
 *   Xq int8 [M][K], s_x fp32 [M], X_out fp16 [M][K_out_pad] (NULL if K_out == 0),
 *   Wq/s_w/W_out from mixq_prepack_weights(MIXQ_W8), flags int32 [4] from
 *   mixq_quantize_act (NULL means "some token may be mixed"),
 *   Y fp16 [M][ldy], ldy >= N, ldy % 8 == 0.
 */
mixq_status mixq_gemm_w8a8o16(int M, int N, int K, int K_out, const int8_t *Xq, const float *s_x,
                              const void *X_out, const void *Wq, const float *s_w,
                              const void *W_out, const int32_t *flags, void *Y, int ldy,
                              int32_t *status, void *stream);

/*
 * Same layer with 4-bit group-wise weights (QServe 渐进量化 / 寄存器压力和并行性,
 * MixLLM two-stage dequantization): inside the mainloop every 4-bit code is
 * expanded back to the INT8 weight (q - z2)*s2, four codes per 32-bit
 * register operation, and multiplied on INT8 tensor cores.  The expanded
 * weights go from registers into tensor memory and are the MMA's A operand
 * (tokens are B), so each CTA owns 128 output channels x up to 256 tokens.
 *   Wq4/grp/s_w/W_out from mixq_prepack_weights(MIXQ_W4G128); the rest as
 *   mixq_gemm_w8a8o16.
 */
mixq_status mixq_gemm_w4a8o16(int M, int N, int K, int K_out, const int8_t *Xq, const float *s_x,
                              const void *X_out, const void *Wq4, const void *grp,
                              const float *s_w, const void *W_out, const int32_t *flags, void *Y,
                              int ldy, int32_t *status, void *stream);

/*
 * Same layer with MIXQ_W4G128_F16S weights (MixLLM page, "MixLLM: Ein neuer
 * Ansatz": two-step dequantization and a fast integer-to-float conversion):
 *   P[m,n,g] = sum_{k in g} Xq[m,k] (q[n,k] - z[n,g])  (exact INT32 per group
 *              of 128 K; q - z is the INT8 operand of tcgen05 kind::i8)
 *   acc[m,n] = sum_g s[n,g] * float(P[m,n,g])          (fp32 fused multiply-adds)
 *   Y[m,n]   = fp16(acc * s_x[m] + o[m,n])             (o as mixq_gemm_w8a8o16)
 *   Wq4/grp/W_out from mixq_prepack_weights(MIXQ_W4G128_F16S); the rest as
 *   mixq_gemm_w8a8o16.  Order of the fp32 sum: without a K split (see
 *   mixq_gemm_plan) the groups in K order; with a K split over S CTAs each CTA
 *   sums the groups of its K range in K order and the S partial sums are then
 *   added in rank order (rank 0 first).
 */
mixq_status mixq_gemm_w4a8o16_f16s(int M, int N, int K, int K_out, const int8_t *Xq,
                                   const float *s_x, const void *X_out, const void *Wq4,
                                   const void *grp, const void *W_out, const int32_t *flags,
                                   void *Y, int ldy, int32_t *status, void *stream);

/*
 * Device workspace the gemm calls need for a shape, in bytes (host only): always
 * 0.  K-split partial sums are reduced through the distributed shared memory of
 * a thread-block cluster, so no call takes a workspace argument.
 */
size_t mixq_gemm_workspace_size(int M, int N, int K);

/*
 * The launch plan the gemm calls use for a shape (host only, no GPU needed):
 * output tile width *bn in output channels (MIXQ_W8 at M >= 256: 256, the
 * persistent CTA-pair kernel, 256-token x 256-channel tiles on two SMs each,
 * *ctas = 2 x the pairs it starts; MIXQ_W4G128 at M >= 2048: 256, its 4-bit
 * pair kernel, 256 weight rows x 256 tokens per pair with the weights expanded
 * into tensor memory; otherwise 128: MIXQ_W8 tiles are 128 tokens high, two
 * CTAs per SM, token-sized A slots when M <= 64; MIXQ_W4G128 tiles hold all
 * tokens when M <= 64, 128 tokens up to M = 1024 (256 from M = 256 when
 * 128-token tiles would leave SMs idle), 256 tokens above; MIXQ_W4G128_F16S
 * tiles hold all tokens when M <= 64 (two CTAs per SM when M <= 16, else one)
 * and 64 tokens above, one CTA per SM), the K-split factor *split (thread-block
 * cluster size along K, 1..8; used at M <= 64, and for 4-bit tiles too few
 * to fill the SMs) and the number of CTAs *ctas.  num_sms <= 0 means "query
 * the current device".
 */
mixq_status mixq_gemm_plan(int mode, int M, int N, int K, int num_sms, int *bn, int *split,
                           int *ctas);

/*
 * Test-only: the gemm mainloop alone, raw INT32 accumulators out
 * (acc int32 [M][ldacc], ldacc % 4 == 0).  mode MIXQ_W8 uses Wq; MIXQ_W4G128
 * uses Wq4 + grp.  bn/split override the plan when > 0.  MIXQ_W8: bn 32 and
 * 64 need M <= 64; with M <= 64 and bn <= 128 the small-M variant runs.
 * MIXQ_W4G128: bn 128 = the tensor-memory-operand kernel's two-CTA-per-SM
 * variant (a K split only with M <= 64, else MIXQ_ERR_UNSUPPORTED_SHAPE),
 * 256 = its one-CTA-per-SM variant (256-token tiles above M = 1024, where it
 * splits no K), 32/64 = the shared-memory-operand
 * kernel with narrow tiles (M <= 64); 0 = the plan.  bn 512 (no K split):
 * the persistent CTA-pair kernel of the mode at any M.
 */
mixq_status mixq_debug_gemm_i32(int mode, int M, int N, int K, const int8_t *Xq, const void *Wq,
                                const void *grp, int32_t *acc, int ldacc, int bn, int split,
                                int32_t *status, void *stream);

/* Test-only: how many thread-block clusters of the gemm kernel (mode, tile
 * width bn, K-split cluster size split, small_m = the M <= 64 variant that
 * fits two CTAs per SM, bn 32/64/128; bn 32/64 exist only as small_m) the
 * current device runs at once. */
mixq_status mixq_debug_max_active_clusters(int mode, int bn, int split, int small_m,
                                           int *clusters);

/* Test-only: logical INT8 codes back from the tiled W8 layout: out int8 [N][K]. */
mixq_status mixq_debug_unpack_w8(int N, int K, const void *Wq, int8_t *out, void *stream);

/* Test-only: logical 4-bit codes back from the packed layout:
 * q uint8 [N][K], s2/z2 uint8 [N][K/128] (the grp pair converted to integers;
 * for MIXQ_W4G128_F16S weights z2 = z, and the real scale is read from grp). */
mixq_status mixq_debug_unpack_w4(int N, int K, const void *Wq4, const void *grp, uint8_t *q,
                                 uint8_t *s2, uint8_t *z2, int32_t *status, void *stream);

/*
 * Test-only: the W8 gemm kernel with its TMA producer told to issue nothing
 * and every pipeline wait limited to wait_limit_ns.  The kernel must return
 * on its own and write MIXQ_ERR_TIMEOUT to *status; used to check that a
 * stalled pipeline ends with an error instead of hanging the GPU.
 */
mixq_status mixq_debug_gemm_stall(int M, int N, int K, const int8_t *Xq, const void *Wq,
                                  const float *s_x, const float *s_w, void *Y, int ldy,
                                  uint64_t wait_limit_ns, int32_t *status, void *stream);

/*
 * Diagnostic: the dense tensor-core rate of this device, measured with the
 * instruction forms the gemm calls use (no page counterpart; it gives the
 * tensor-bound GEMMs a peak taken on the same chip in the same run).  One CTA
 * per SM keeps an A tile (128 x 128 bytes) and a B tile (256 x 128 bytes) in
 * shared memory, filled with a hashed byte pattern, and one thread issues
 * `iters` rounds of four back-to-back tcgen05.mma, M = 128, N = 256, into one
 * tensor-memory accumulator, then waits for them (bounded; a wait that runs
 * out writes MIXQ_ERR_TIMEOUT to *status).
 *   kind 0: kind::i8 (s8 x s8 -> s32, K = 32 per MMA)
 *   kind 1: kind::f16 (f16 x f16 -> f32, K = 16 per MMA)
 *   iters in [1, 1048576]; *ops (host, non-null) receives the operations one
 *   launch performs (2 * 128 * 256 * K per MMA, all SMs).  Time the launch
 *   with events on `stream`; its outputs are discarded.
 */
mixq_status mixq_debug_mma_rate(int kind, int iters, double *ops, int32_t *status, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* MIXQ_H */
