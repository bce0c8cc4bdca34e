// Internal interface of the GEMM for 4-bit weights of reading B (a real fp16
// scale and an integer zero point per row and group of 128 K; per-group INT32
// partial sums scaled and accumulated in fp32).  Used by the C ABI layer.
#pragma once

#include "internal.h"

namespace mixq {

// Launch shape of the reading-B GEMM: K split `split` (cluster size along z,
// 1..8) and the CTAs launched.  bn is always 128 and small_m / ts are 0.
GemmPlan plan_gemm_w4b(int M, int N, int K, int num_sms);

// a.mode is ignored; a.grp holds the (s, z) fp16 pairs [K/128][N]; a.s_w is
// unused; a.epi must be Epi::kMixed.
cudaError_t launch_gemm_w4b(const GemmArgs &a, const GemmPlan &plan, cudaStream_t stream,
                            const char **why);

}  // namespace mixq
