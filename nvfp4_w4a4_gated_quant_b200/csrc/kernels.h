// Internal launchers of the sm_100a kernels (host side, no validation: the
// C-ABI entry points in api.cu check every argument before calling these).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/gdn.h"

namespace gdn {

int launch_quantize(const void* x, int x_dtype, int64_t rows, int64_t cols, int64_t ld, int mode, const float* g_enc_in,
                    uint8_t* codes, uint8_t* scales, int tiled, int64_t row_off, float* g_out, unsigned* amax_ws,
                    cudaStream_t stream);

// max |x| over the tensor folded into *amax (atomic max on the FP32 bits;
// *amax >= 0 on entry, not reset); and *g_enc = 2688 / *amax.
int launch_amax_update(const void* x, int x_dtype, int64_t rows, int64_t cols, int64_t ld, float* amax,
                       cudaStream_t stream);
int launch_encode_scale(const float* amax, float* g_enc, cudaStream_t stream);

// The short causal convolution (+ SiLU) and the gated output RMSNorm.
int launch_short_conv(const uint16_t* x, int64_t B, int64_t T, int64_t C, int64_t ld_x, const float* w,
                      const uint16_t* state_in, uint16_t* y, int64_t ld_y, uint16_t* state_out, cudaStream_t stream);
int launch_gated_rmsnorm(const uint16_t* o, const uint16_t* g, int64_t M, int H, int dv, const float* gamma,
                         uint16_t* y, float* amax, cudaStream_t stream);

int launch_gates(const float* a, const float* b, int64_t M, int H, const float* A_log, const float* dt_bias,
                 float* log_alpha, float* beta, cudaStream_t stream);

// `ctas` CTAs, each issuing iters x 4 FP4 MMAs of 128 x 256 x 64 back to back.
int launch_fp4_mma_ceiling(int64_t iters, int ctas, cudaStream_t stream);

int launch_gemm_nvfp4(const gdn_nvfp4_t* A, const float* g_a, const gdn_nvfp4_t* B, int64_t M, int64_t N,
                      int64_t K, const gdn_epilogue_segment_t* segs, int n_segs, cudaStream_t stream);

// NVFP4 quantization of the scan's bf16 o with a given encode scale: codes
// [B*T, H*dv/2], TILED scales (K = H*dv), decode scale 1 / g_enc.
struct OQuant {
  uint8_t* codes;
  uint8_t* scales;
  const float* g_enc;   // device scalar
  float* g_out;         // device scalar, written: 1 / g_enc
};

// oq: when given, o (bf16) is also quantized -- inside the tensor-core scan's
// epilogue, or by a separate given-scale pass when another kernel runs.
// ws / ws_bytes: scratch for the segmented tensor-core path (long sequences
// on few chains); without it (or too small) every sequence runs in one piece.
int launch_delta_rule(const uint16_t* q, const uint16_t* k, const uint16_t* v, int64_t ld_q, int64_t ld_k,
                      int64_t ld_v, const float* log_alpha, const float* beta, const float* S0, int64_t B,
                      int64_t T, int H, int dk, int dv, int flags, void* o, float* S_T, unsigned* o_amax,
                      cudaStream_t stream, const OQuant* oq = nullptr, void* ws = nullptr, size_t ws_bytes = 0);
// Scratch bytes the tensor-core path can use to cut long sequences into
// segments (0 when it would not), for the current device.
size_t delta_rule_tc_workspace(int64_t B, int64_t T, int H, int dk, int dv);

// The token-by-token recurrence (state in registers; decode and short
// continuations).
int launch_delta_rule_step(const uint16_t* q, const uint16_t* k, const uint16_t* v, int64_t ld_q, int64_t ld_k,
                           int64_t ld_v, const float* log_alpha, const float* beta, const float* S_in, float* S_out,
                           int64_t B, int64_t T, int H, int dk, int dv, int flags, void* o, cudaStream_t stream);

// The tcgen05 scan (d_k = 128, d_v % 64 == 0, T < 2^31: its tensor maps take
// 32-bit token coordinates); launch_delta_rule dispatches to it unless
// GDN_DR_MMA_SYNC is set.
bool delta_rule_tc_supported(int dk, int dv, int64_t T);
int launch_delta_rule_tc(const uint16_t* q, const uint16_t* k, const uint16_t* v, int64_t ld_q, int64_t ld_k,
                         int64_t ld_v, const float* log_alpha, const float* beta, const float* S0, int64_t B,
                         int64_t T, int H, int dk, int dv, int flags, void* o, float* S_T, unsigned* o_amax,
                         cudaStream_t stream, const OQuant* oq = nullptr, void* ws = nullptr, size_t ws_bytes = 0);

}  // namespace gdn
