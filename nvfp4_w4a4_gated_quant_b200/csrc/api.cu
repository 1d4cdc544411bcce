// C-ABI entry points: argument checks, workspace arithmetic, status plumbing.
// Every check runs on the host before anything is enqueued.
#include <stdarg.h>
#include <stdio.h>
#include <string.h>

#include <mutex>

#include "common.cuh"
#include "kernels.h"
#include "tmap.cuh"

namespace gdn {

namespace {
__device__ int g_status_word = GDN_OK;

// Waits on an mbarrier that nothing ever arrives on, with the same bounded
// poll-and-back-off loop the pipelined kernels use, then reports
// GDN_ERR_TIMEOUT through the device status word and returns.
__global__ void bounded_wait_selftest_kernel(uint32_t poll_limit, int* status) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    bool done = false;
    for (uint32_t i = 0; i < poll_limit && !done; ++i) {
      done = mbar_try_wait(&bar, 0);
      if (!done) __nanosleep(32);
    }
    if (!done) report_status(status, GDN_ERR_TIMEOUT);
  }
}

thread_local char t_last_error[256] = "no error";

constexpr int kMaxDevices = 64;
int* g_status_ptr[kMaxDevices];
int g_num_sms[kMaxDevices];
std::mutex g_dev_mu;

int current_device() {
  int d = 0;
  if (cudaGetDevice(&d) != cudaSuccess) return -1;
  return d;
}
}  // namespace

PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  });
  return fn;
}


int record_cuda_error(cudaError_t err) {
  snprintf(t_last_error, sizeof(t_last_error), "%s: %s", cudaGetErrorName(err), cudaGetErrorString(err));
  return GDN_ERR_CUDA;
}

void set_error_text(const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(t_last_error, sizeof(t_last_error), fmt, ap);
  va_end(ap);
}

int* device_status_word() {
  const int d = current_device();
  if (d < 0 || d >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lk(g_dev_mu);
  if (!g_status_ptr[d]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_status_word) != cudaSuccess) return nullptr;
    g_status_ptr[d] = static_cast<int*>(p);
  }
  return g_status_ptr[d];
}

int num_sms() {
  const int d = current_device();
  if (d < 0 || d >= kMaxDevices) return 148;
  std::lock_guard<std::mutex> lk(g_dev_mu);
  if (!g_num_sms[d]) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, d) != cudaSuccess || n <= 0) n = 148;
    g_num_sms[d] = n;
  }
  return g_num_sms[d];
}

}  // namespace gdn

using namespace gdn;

namespace {
constexpr size_t kQuantWs = 256;



cudaStream_t as_stream(gdn_stream_t s) { return reinterpret_cast<cudaStream_t>(s); }

int check_quant_args(const void* x, int x_dtype, int64_t rows, int64_t cols, int64_t ld_x, int mode, const float* g_enc_in,
                     const uint8_t* codes, const uint8_t* scales, int sf_layout, int64_t sf_row_offset,
                     const float* g_out, const void* ws, size_t ws_bytes) {
  if (rows < 0 || cols <= 0 || ld_x < cols || !g_out) return GDN_ERR_INVALID_ARG;
  if (x_dtype != GDN_DTYPE_BF16 && x_dtype != GDN_DTYPE_F32) return GDN_ERR_INVALID_ARG;
  const int64_t per16 = x_dtype == GDN_DTYPE_F32 ? 4 : 8;  // elements per 16 bytes
  if (mode != GDN_QUANT_DYNAMIC && mode != GDN_QUANT_GIVEN_SCALE && mode != GDN_QUANT_GIVEN_AMAX)
    return GDN_ERR_INVALID_ARG;
  if (sf_layout != GDN_SF_TILED && sf_layout != GDN_SF_LINEAR) return GDN_ERR_INVALID_ARG;
  if (sf_row_offset < 0 || (sf_layout == GDN_SF_LINEAR && sf_row_offset != 0)) return GDN_ERR_INVALID_ARG;
  if (mode != GDN_QUANT_DYNAMIC && !g_enc_in) return GDN_ERR_INVALID_ARG;
  if (mode == GDN_QUANT_DYNAMIC && (!ws || ws_bytes < kQuantWs)) return GDN_ERR_WORKSPACE;
  if (cols % 16 != 0 || (sf_layout == GDN_SF_TILED && cols % 64 != 0)) return GDN_ERR_UNSUPPORTED_SHAPE;
  if (rows > 0 && (!x || !codes || !scales)) return GDN_ERR_INVALID_ARG;
  if (rows > 0 && (!aligned(x, 16) || ld_x % per16 != 0 || !aligned(codes, 8))) return GDN_ERR_ALIGNMENT;
  if (ws && !aligned(ws, 16)) return GDN_ERR_ALIGNMENT;
  if (!aligned(g_out, 4) || (g_enc_in && !aligned(g_enc_in, 4))) return GDN_ERR_ALIGNMENT;
  return GDN_OK;
}
}  // namespace

extern "C" {

const char* gdn_status_string(int status) {
  switch (status) {
    case GDN_OK: return "ok";
    case GDN_ERR_INVALID_ARG: return "invalid argument";
    case GDN_ERR_UNSUPPORTED_SHAPE: return "unsupported shape";
    case GDN_ERR_ALIGNMENT: return "pointer or stride alignment";
    case GDN_ERR_CUDA: return "CUDA error";
    case GDN_ERR_TIMEOUT: return "device-side wait timed out";
    case GDN_ERR_WORKSPACE: return "workspace missing or too small";
    case GDN_ERR_RANGE: return "a scan operand left the FP16 range";
    default: return "unknown status";
  }
}

const char* gdn_last_error(void) { return t_last_error; }

const char* gdn_version(void) { return "0.1.0"; }

int gdn_stream_check(gdn_stream_t stream) {
  cudaError_t e = cudaStreamSynchronize(as_stream(stream));
  if (e != cudaSuccess) return record_cuda_error(e);
  int* p = device_status_word();
  if (!p) return record_cuda_error(cudaErrorInvalidDevice);
  int word = GDN_OK;
  e = cudaMemcpy(&word, p, sizeof(int), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return record_cuda_error(e);
  if (word != GDN_OK) {
    const int zero = GDN_OK;
    e = cudaMemcpy(p, &zero, sizeof(int), cudaMemcpyHostToDevice);
    if (e != cudaSuccess) return record_cuda_error(e);
  }
  return word;
}

int gdn_fp4_mma_ceiling(int64_t iters, int* ctas, gdn_stream_t stream) {
  if (iters <= 0 || iters > ((int64_t)1 << 32) || !ctas) return GDN_ERR_INVALID_ARG;
  *ctas = num_sms();
  return launch_fp4_mma_ceiling(iters, *ctas, as_stream(stream));
}

int gdn_selftest_bounded_wait(uint32_t poll_limit, gdn_stream_t stream) {
  if (poll_limit == 0 || poll_limit > (1u << 26)) return GDN_ERR_INVALID_ARG;
  int* status = device_status_word();
  if (!status) return record_cuda_error(cudaErrorInvalidDevice);
  gdn::bounded_wait_selftest_kernel<<<1, 32, 0, as_stream(stream)>>>(poll_limit, status);
  return check_launch();
}

size_t gdn_quantize_workspace_size(void) { return kQuantWs; }

size_t gdn_scales_tiled_bytes(int64_t rows, int64_t cols) {
  if (rows < 0 || cols < 0) return 0;
  return (size_t)(cdiv(rows, 128) * 128) * (size_t)(cdiv(cols, 64) * 4);
}

int gdn_quantize_nvfp4(const void* x, int x_dtype, int64_t rows, int64_t cols, int64_t ld_x, int mode,
                       const float* g_enc_in, uint8_t* codes, uint8_t* scales, int sf_layout, int64_t sf_row_offset,
                       float* g_out, void* ws, size_t ws_bytes, gdn_stream_t stream) {
  int st = check_quant_args(x, x_dtype, rows, cols, ld_x, mode, g_enc_in, codes, scales, sf_layout, sf_row_offset, g_out, ws,
                            ws_bytes);
  if (st) return st;
  return launch_quantize(x, x_dtype, rows, cols, ld_x, mode, g_enc_in, codes, scales,
                         sf_layout == GDN_SF_TILED ? 1 : 0, sf_row_offset, g_out, static_cast<unsigned*>(ws),
                         as_stream(stream));
}

int gdn_amax_update(const void* x, int x_dtype, int64_t rows, int64_t cols, int64_t ld_x, float* amax,
                    gdn_stream_t stream) {
  if (rows < 0 || cols <= 0 || ld_x < cols || !amax) return GDN_ERR_INVALID_ARG;
  if (x_dtype != GDN_DTYPE_BF16 && x_dtype != GDN_DTYPE_F32) return GDN_ERR_INVALID_ARG;
  if (cols % 16 != 0) return GDN_ERR_UNSUPPORTED_SHAPE;
  const int64_t per16 = x_dtype == GDN_DTYPE_F32 ? 4 : 8;
  if (rows > 0 && (!x || !aligned(x, 16) || ld_x % per16 != 0)) return x ? GDN_ERR_ALIGNMENT : GDN_ERR_INVALID_ARG;
  if (!aligned(amax, 4)) return GDN_ERR_ALIGNMENT;
  return launch_amax_update(x, x_dtype, rows, cols, ld_x, amax, as_stream(stream));
}

int gdn_encode_scale_from_amax(const float* amax, float* g_enc, gdn_stream_t stream) {
  if (!amax || !g_enc) return GDN_ERR_INVALID_ARG;
  if (!aligned(amax, 4) || !aligned(g_enc, 4)) return GDN_ERR_ALIGNMENT;
  return launch_encode_scale(amax, g_enc, as_stream(stream));
}

int gdn_short_conv(const void* x, int64_t B, int64_t T, int64_t C, int64_t ld_x, const float* w, const void* state_in,
                   void* y, int64_t ld_y, void* state_out, gdn_stream_t stream) {
  if (B < 0 || T < 0 || C <= 0 || ld_x < C || ld_y < C || !w) return GDN_ERR_INVALID_ARG;
  if (C % 8 != 0 || B > 65535 || T > (int64_t)65535 * 64) return GDN_ERR_UNSUPPORTED_SHAPE;
  if (B > 0 && T > 0) {
    if (!x || !y) return GDN_ERR_INVALID_ARG;
    if (x == y) return GDN_ERR_INVALID_ARG;   // the window reads earlier inputs: no in-place call
    if (!aligned(x, 16) || !aligned(y, 16) || ld_x % 8 || ld_y % 8) return GDN_ERR_ALIGNMENT;
  }
  if (!aligned(w, 16) || (state_in && !aligned(state_in, 16)) || (state_out && !aligned(state_out, 16)))
    return GDN_ERR_ALIGNMENT;
  return launch_short_conv(static_cast<const uint16_t*>(x), B, T, C, ld_x, w, static_cast<const uint16_t*>(state_in),
                           static_cast<uint16_t*>(y), ld_y, static_cast<uint16_t*>(state_out), as_stream(stream));
}

int gdn_gated_rmsnorm(const void* o, const void* g, int64_t M, int H, int dv, const float* gamma, void* y,
                      float* amax, gdn_stream_t stream) {
  if (M < 0 || H <= 0) return GDN_ERR_INVALID_ARG;
  if (dv != 32 && dv != 64 && dv != 128) return GDN_ERR_UNSUPPORTED_SHAPE;
  if (M > 0 && (!o || !g || !gamma || !y)) return GDN_ERR_INVALID_ARG;
  if ((o && !aligned(o, 16)) || (g && !aligned(g, 16)) || (y && !aligned(y, 16)) || (amax && !aligned(amax, 4)))
    return GDN_ERR_ALIGNMENT;
  return launch_gated_rmsnorm(static_cast<const uint16_t*>(o), static_cast<const uint16_t*>(g), M, H, dv, gamma,
                              static_cast<uint16_t*>(y), amax, as_stream(stream));
}

int gdn_gemm_nvfp4(const gdn_nvfp4_t* A, const float* g_a, const gdn_nvfp4_t* B, int64_t M, int64_t N, int64_t K,
                   const gdn_epilogue_segment_t* segs, int n_segs, gdn_stream_t stream) {
  if (!A || !B || !g_a || !segs) return GDN_ERR_INVALID_ARG;
  if (M < 0 || N < 0 || K <= 0) return GDN_ERR_INVALID_ARG;
  if (n_segs < 1 || n_segs > GDN_MAX_SEGMENTS) return GDN_ERR_INVALID_ARG;
  if (K % 64 != 0) return GDN_ERR_UNSUPPORTED_SHAPE;
  if (M > (1 << 30) || N > (1 << 30) || K > (1 << 24)) return GDN_ERR_UNSUPPORTED_SHAPE;
  int64_t expect = 0;
  for (int i = 0; i < n_segs; ++i) {
    const gdn_epilogue_segment_t& s = segs[i];
    if (s.n_begin != expect || s.n_end <= s.n_begin || !s.g_b || !s.out || s.ld_out <= 0) return GDN_ERR_INVALID_ARG;
    if (s.kind < GDN_EPI_STORE_BF16 || s.kind > GDN_EPI_BETA) return GDN_ERR_INVALID_ARG;
    if (s.kind == GDN_EPI_LOG_ALPHA && (!s.A_log || !s.dt_bias)) return GDN_ERR_INVALID_ARG;
    if (s.ld_out < s.n_end - s.n_begin) return GDN_ERR_INVALID_ARG;
    if (!aligned(s.out, s.kind == GDN_EPI_STORE_BF16 ? 2 : 4)) return GDN_ERR_ALIGNMENT;
    expect = s.n_end;
  }
  if (expect != N) return GDN_ERR_INVALID_ARG;
  if (M > 0 && N > 0) {
    if (!A->codes || !A->scales || !B->codes || !B->scales) return GDN_ERR_INVALID_ARG;
    if (!aligned(A->codes, 16) || !aligned(B->codes, 16) || !aligned(A->scales, 16) || !aligned(B->scales, 16))
      return GDN_ERR_ALIGNMENT;
  }
  return launch_gemm_nvfp4(A, g_a, B, M, N, K, segs, n_segs, as_stream(stream));
}

int gdn_gates(const float* a, const float* b, int64_t M, int H, const float* A_log, const float* dt_bias,
              float* log_alpha, float* beta, gdn_stream_t stream) {
  if (M < 0 || H <= 0) return GDN_ERR_INVALID_ARG;
  if (M > 0 && (!a || !b || !A_log || !dt_bias || !log_alpha || !beta)) return GDN_ERR_INVALID_ARG;
  return launch_gates(a, b, M, H, A_log, dt_bias, log_alpha, beta, as_stream(stream));
}

size_t gdn_delta_rule_workspace_size(int64_t B, int64_t T, int H, int dk, int dv) {
  if (B <= 0 || T <= 0 || H <= 0) return 0;
  return delta_rule_tc_workspace(B, T, H, dk, dv);
}

int gdn_delta_rule_fwd(const void* q, const void* k, const void* v, int64_t ld_q, int64_t ld_k, int64_t ld_v,
                       const float* log_alpha, const float* beta, const float* S0, int64_t B, int64_t T, int H, int dk,
                       int dv, int flags, void* o, float* S_T, void* ws, size_t ws_bytes, gdn_stream_t stream) {
  if (B < 0 || T < 0 || H <= 0) return GDN_ERR_INVALID_ARG;
  if (flags & ~(GDN_DR_L2NORM_QK | GDN_DR_O_FP32 | GDN_DR_MMA_SYNC)) return GDN_ERR_INVALID_ARG;
  if ((dk != 32 && dk != 64 && dk != 128) || (dv != 32 && dv != 64 && dv != 128)) return GDN_ERR_UNSUPPORTED_SHAPE;
  if (B * (int64_t)H > (1 << 30) || T > (int64_t)1 << 40) return GDN_ERR_UNSUPPORTED_SHAPE;
  if (ld_q < (int64_t)H * dk || ld_k < (int64_t)H * dk || ld_v < (int64_t)H * dv) return GDN_ERR_INVALID_ARG;
  if (B > 0 && T > 0) {
    if (!q || !k || !v || !log_alpha || !beta || !o) return GDN_ERR_INVALID_ARG;
    if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || ld_q % 8 || ld_k % 8 || ld_v % 8)
      return GDN_ERR_ALIGNMENT;
    if (!aligned(o, (flags & GDN_DR_O_FP32) ? 8 : 4) || !aligned(log_alpha, 4) || !aligned(beta, 4))
      return GDN_ERR_ALIGNMENT;
  }
  if ((S0 && !aligned(S0, 4)) || (S_T && !aligned(S_T, 4))) return GDN_ERR_ALIGNMENT;
  if (ws && !aligned(ws, 256)) return GDN_ERR_ALIGNMENT;
  return launch_delta_rule(static_cast<const uint16_t*>(q), static_cast<const uint16_t*>(k),
                           static_cast<const uint16_t*>(v), ld_q, ld_k, ld_v, log_alpha, beta, S0, B, T, H, dk, dv,
                           flags, o, S_T, nullptr, as_stream(stream), nullptr, ws, ws ? ws_bytes : 0);
}

int gdn_delta_rule_step(const void* q, const void* k, const void* v, int64_t ld_q, int64_t ld_k, int64_t ld_v,
                        const float* log_alpha, const float* beta, const float* S_in, float* S_out, int64_t B,
                        int64_t T, int H, int dk, int dv, int flags, void* o, gdn_stream_t stream) {
  if (B < 0 || T < 0 || H <= 0) return GDN_ERR_INVALID_ARG;
  if (flags & ~(GDN_DR_L2NORM_QK | GDN_DR_O_FP32 | GDN_DR_DECAYED_READ)) return GDN_ERR_INVALID_ARG;
  if ((dk != 32 && dk != 64 && dk != 128) || (dv != 32 && dv != 64 && dv != 128)) return GDN_ERR_UNSUPPORTED_SHAPE;
  if (B * (int64_t)H > (1 << 28) || T > (int64_t)1 << 40) return GDN_ERR_UNSUPPORTED_SHAPE;
  if (ld_q < (int64_t)H * dk || ld_k < (int64_t)H * dk || ld_v < (int64_t)H * dv) return GDN_ERR_INVALID_ARG;
  if (B == 0) return GDN_OK;
  if (!S_out) return GDN_ERR_INVALID_ARG;
  if (T > 0) {
    if (!q || !k || !v || !log_alpha || !beta || !o) return GDN_ERR_INVALID_ARG;
    if (!aligned(q, 2) || !aligned(k, 2) || !aligned(v, 2)) return GDN_ERR_ALIGNMENT;
    if (!aligned(o, (flags & GDN_DR_O_FP32) ? 4 : 2) || !aligned(log_alpha, 4) || !aligned(beta, 4))
      return GDN_ERR_ALIGNMENT;
  }
  if ((S_in && !aligned(S_in, 4)) || !aligned(S_out, 4)) return GDN_ERR_ALIGNMENT;
  return launch_delta_rule_step(static_cast<const uint16_t*>(q), static_cast<const uint16_t*>(k),
                                static_cast<const uint16_t*>(v), ld_q, ld_k, ld_v, log_alpha, beta, S_in, S_out, B,
                                T, H, dk, dv, flags, o, as_stream(stream));
}

}  // extern "C"
