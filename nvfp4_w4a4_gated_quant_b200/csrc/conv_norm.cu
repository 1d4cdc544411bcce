// The rest of a Gated DeltaNet block around the recurrence: a short causal
// depthwise convolution with SiLU over the q | k | v channels, and the output
// RMSNorm gated by SiLU of a sixth projection.  The pages name "the
// convolution" only as an alternative explanation and define neither; both
// follow the Gated DeltaNet block's outside specification (Yang, Kautz and
// Hatamizadeh, "Gated Delta Networks: Improving Mamba2 with Delta Rule",
// ICLR 2025):
//   y_t[c] = SiLU( sum_{j=0..3} w[c][j] x_{t-3+j}[c] )   (tokens before the
//            first from a carried state, else zero)
//   out    = o / sqrt(mean_dv(o^2) + 1e-6) * gamma * SiLU(g)   per (token, head)
// Both are HBM-bound elementwise passes: FP32 arithmetic on bf16 storage,
// 16-byte vectors, one thread per eight channels (convolution) or one warp
// per (token, head) row (norm).
#include "common.cuh"
#include "kernels.h"

namespace gdn {
namespace {

constexpr int CW = 4;          // kernel width
constexpr int CONV_TOK = 64;   // tokens one thread walks
constexpr int CONV_THREADS = 128;

__device__ __forceinline__ float silu_f(float x) { return __fdiv_rn(x, 1.0f + expf(-x)); }

__device__ __forceinline__ void unpack8(const uint4& u, float* f) {
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    f[2 * i] = bf16_bits_to_f32(w[i] & 0xFFFFu);
    f[2 * i + 1] = bf16_bits_to_f32(w[i] >> 16);
  }
}
__device__ __forceinline__ uint4 pack8(const float* f) {
  return make_uint4(pack_bf16x2(f[0], f[1]), pack_bf16x2(f[2], f[3]), pack_bf16x2(f[4], f[5]),
                    pack_bf16x2(f[6], f[7]));
}

// grid (channel vectors / CONV_THREADS, token blocks, batch): a thread keeps
// the three previous inputs of its eight channels in registers while it walks
// CONV_TOK tokens, reading each input row once.
__global__ void __launch_bounds__(CONV_THREADS) short_conv_kernel(const uint16_t* __restrict__ x, int64_t T, int64_t C,
                                                                  int64_t ld_x, const float* __restrict__ w,
                                                                  const uint16_t* __restrict__ state_in,
                                                                  uint16_t* __restrict__ y, int64_t ld_y,
                                                                  uint16_t* __restrict__ state_out) {
  const int64_t cv = (int64_t)blockIdx.x * CONV_THREADS + threadIdx.x;
  if (cv * 8 >= C) return;
  const int64_t c0 = cv * 8;
  const int64_t b = blockIdx.z;
  const int64_t t_begin = (int64_t)blockIdx.y * CONV_TOK;
  const int64_t t_end = t_begin + CONV_TOK < T ? t_begin + CONV_TOK : T;
  float wk[8][CW];
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    const float4 w4 = *reinterpret_cast<const float4*>(w + (c0 + e) * CW);
    wk[e][0] = w4.x; wk[e][1] = w4.y; wk[e][2] = w4.z; wk[e][3] = w4.w;
  }
  float win[3][8];
#pragma unroll
  for (int i = 0; i < 3; ++i) {
    const int64_t t = t_begin - 3 + i;
    if (t >= 0) {
      unpack8(*reinterpret_cast<const uint4*>(x + (b * T + t) * ld_x + c0), win[i]);
    } else if (state_in) {
      unpack8(*reinterpret_cast<const uint4*>(state_in + (b * 3 + (t + 3)) * C + c0), win[i]);
    } else {
#pragma unroll
      for (int e = 0; e < 8; ++e) win[i][e] = 0.0f;
    }
  }
  for (int64_t t = t_begin; t < t_end; ++t) {
    float cur[8], out[8];
    unpack8(*reinterpret_cast<const uint4*>(x + (b * T + t) * ld_x + c0), cur);
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      float acc = wk[e][0] * win[0][e];
      acc = fmaf(wk[e][1], win[1][e], acc);
      acc = fmaf(wk[e][2], win[2][e], acc);
      acc = fmaf(wk[e][3], cur[e], acc);
      out[e] = silu_f(acc);
      win[0][e] = win[1][e];
      win[1][e] = win[2][e];
      win[2][e] = cur[e];
    }
    *reinterpret_cast<uint4*>(y + (b * T + t) * ld_y + c0) = pack8(out);
  }
  // the last three inputs (carried state included) for the next call
  if (state_out && t_end == T) {
#pragma unroll
    for (int i = 0; i < 3; ++i)
      *reinterpret_cast<uint4*>(state_out + (b * 3 + i) * C + c0) = pack8(win[i]);
  }
}

// One warp per (token, head) row of DV values, DV / 32 per lane.
template <int DV>
__global__ void __launch_bounds__(256) gated_rmsnorm_kernel(const uint16_t* __restrict__ o,
                                                            const uint16_t* __restrict__ g, int64_t rows,
                                                            const float* __restrict__ gamma,
                                                            uint16_t* __restrict__ y, unsigned* __restrict__ amax) {
  constexpr int E = DV / 32;
  const int lane = threadIdx.x & 31;
  const int64_t row = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
  uint32_t am = 0;
  if (row < rows) {
    const int64_t off = row * DV + lane * E;
    float ov[E], gv[E];
#pragma unroll
    for (int i = 0; i < E; ++i) {
      ov[i] = bf16_bits_to_f32(o[off + i]);
      gv[i] = bf16_bits_to_f32(g[off + i]);
    }
    float ss = 0.0f;
#pragma unroll
    for (int i = 0; i < E; ++i) ss = fmaf(ov[i], ov[i], ss);
#pragma unroll
    for (int d = 16; d > 0; d >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, d);
    const float r = __fdiv_rn(1.0f, __fsqrt_rn(__fdiv_rn(ss, (float)DV) + 1e-6f));
#pragma unroll
    for (int i = 0; i < E; ++i) {
      const float v = ov[i] * r * gamma[lane * E + i] * silu_f(gv[i]);
      const uint32_t bits = f32_to_bf16_bits(v);
      y[off + i] = (uint16_t)bits;
      am = max(am, (bits & 0x7FFFu) << 16);   // bf16 |value| as FP32 bits
    }
  }
  if (amax) {
#pragma unroll
    for (int d = 16; d > 0; d >>= 1) am = max(am, __shfl_xor_sync(0xffffffffu, am, d));
    if (lane == 0 && am) atomicMax(amax, am);
  }
}

}  // namespace

int launch_short_conv(const uint16_t* x, int64_t B, int64_t T, int64_t C, int64_t ld_x, const float* w,
                      const uint16_t* state_in, uint16_t* y, int64_t ld_y, uint16_t* state_out, cudaStream_t stream) {
  if (B == 0) return GDN_OK;
  if (T == 0) {
    // no tokens: the carried state is unchanged
    if (!state_out) return GDN_OK;
    cudaError_t e = state_in ? cudaMemcpyAsync(state_out, state_in, (size_t)B * 3 * C * 2, cudaMemcpyDeviceToDevice,
                                               stream)
                             : cudaMemsetAsync(state_out, 0, (size_t)B * 3 * C * 2, stream);
    return e == cudaSuccess ? GDN_OK : record_cuda_error(e);
  }
  const int64_t vecs = C / 8;
  dim3 grid((unsigned)cdiv(vecs, CONV_THREADS), (unsigned)cdiv(T, CONV_TOK), (unsigned)B);
  short_conv_kernel<<<grid, CONV_THREADS, 0, stream>>>(x, T, C, ld_x, w, state_in, y, ld_y, state_out);
  return check_launch();
}

int launch_gated_rmsnorm(const uint16_t* o, const uint16_t* g, int64_t M, int H, int dv, const float* gamma,
                         uint16_t* y, float* amax, cudaStream_t stream) {
  const int64_t rows = M * H;
  if (rows == 0) return GDN_OK;
  unsigned* am = reinterpret_cast<unsigned*>(amax);
  const unsigned blocks = (unsigned)cdiv(rows, 8);
  switch (dv) {
    case 32: gated_rmsnorm_kernel<32><<<blocks, 256, 0, stream>>>(o, g, rows, gamma, y, am); break;
    case 64: gated_rmsnorm_kernel<64><<<blocks, 256, 0, stream>>>(o, g, rows, gamma, y, am); break;
    default: gated_rmsnorm_kernel<128><<<blocks, 256, 0, stream>>>(o, g, rows, gamma, y, am); break;
  }
  return check_launch();
}

}  // namespace gdn
