// Gate arithmetic shared by the standalone gate kernel and the GEMM epilogue.
//
// "Anthology of the SOTA, theory-128", section "The account": the decay is
// exp(-exp(A) softplus(a + dt_bias)) and the write strength is a sigmoid.
// FP32 with CUDA's accurate expf / log1pf.  softplus(x) is evaluated as
// max(x, 0) + log1p(exp(-|x|)), which needs no threshold.
#pragma once

namespace gdn {

__device__ __forceinline__ float gate_log_alpha(float a, float A_log, float dt_bias) {
  const float x = __fadd_rn(a, dt_bias);
  const float sp = __fadd_rn(fmaxf(x, 0.0f), log1pf(expf(-fabsf(x))));
  return -__fmul_rn(expf(A_log), sp);
}

__device__ __forceinline__ float gate_beta(float b) {
  return __fdiv_rn(1.0f, __fadd_rn(1.0f, expf(-b)));
}

}  // namespace gdn
