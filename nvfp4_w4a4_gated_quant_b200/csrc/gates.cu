// Standalone gate kernel: log(alpha) and beta from the gate pre-activations.
// Elementwise and HBM-bound (16 bytes in, 8 bytes out per (token, head)).
#include "common.cuh"
#include "gate_math.cuh"
#include "kernels.h"

namespace gdn {
namespace {

__global__ void gates_kernel(const float* __restrict__ a, const float* __restrict__ b, int64_t n, int H,
                             const float* __restrict__ A_log, const float* __restrict__ dt_bias,
                             float* __restrict__ log_alpha, float* __restrict__ beta) {
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x) {
    const int h = (int)(i % H);
    log_alpha[i] = gate_log_alpha(a[i], A_log[h], dt_bias[h]);
    beta[i] = gate_beta(b[i]);
  }
}

}  // namespace

int launch_gates(const float* a, const float* b, int64_t M, int H, const float* A_log, const float* dt_bias,
                 float* log_alpha, float* beta, cudaStream_t stream) {
  const int64_t n = M * H;
  if (n == 0) return GDN_OK;
  const int threads = 256;
  const int64_t blocks = std::min<int64_t>(cdiv(n, threads), (int64_t)num_sms() * 32);
  gates_kernel<<<(unsigned)blocks, threads, 0, stream>>>(a, b, n, H, A_log, dt_bias, log_alpha, beta);
  return check_launch();
}

}  // namespace gdn
