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
// 16-byte vectors with several rows in flight per thread, one thread per
// eight channels (convolution, its rows staged by cp.async) or DV/8 lanes per
// (token, head) row (norm).  SiLU(u) = u sigmoid(u) with
// sigmoid(u) = 1/2 + tanh(u/2)/2 on the SFU's tanh.approx (relative error
// ~2^-11, below the bf16 rounding of the stored result), so the passes stay
// memory-bound.
#include <algorithm>

#include "common.cuh"
#include "kernels.h"

namespace gdn {
namespace {

constexpr int CW = 4;          // kernel width
constexpr int CONV_TOK = 64;   // tokens one thread walks
constexpr int CONV_THREADS = 256;
constexpr int CONV_NR = 8;     // input rows per group; two groups staged
constexpr size_t CONV_SMEM = (size_t)2 * CONV_NR * CONV_THREADS * 16;

__device__ __forceinline__ float tanh_approx(float x) {
  float y;
  asm("tanh.approx.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ float silu_f(float x) { return x * fmaf(0.5f, tanh_approx(0.5f * x), 0.5f); }

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

__device__ __forceinline__ void cp_async16(void* dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(dst)), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// grid (channel octets / CONV_THREADS, token blocks, batch): a thread keeps
// the three previous inputs of its eight channels in registers while it walks
// CONV_TOK tokens, reading each input row once.  Its rows arrive by cp.async
// (16 bytes each) into its own slots of a shared-memory stage, CONV_NR rows a
// group, the next group in flight while this one is computed: the bytes in
// flight sit in shared memory, not in registers.
__global__ void __launch_bounds__(CONV_THREADS) short_conv_kernel(const uint16_t* __restrict__ x, int64_t T, int64_t C,
                                                                  int64_t ld_x, const float* __restrict__ w,
                                                                  const uint16_t* __restrict__ state_in,
                                                                  uint16_t* __restrict__ y, int64_t ld_y,
                                                                  uint16_t* __restrict__ state_out) {
  extern __shared__ uint4 conv_stage[];   // [2][CONV_NR][CONV_THREADS]
  const int64_t cv = (int64_t)blockIdx.x * CONV_THREADS + threadIdx.x;
  if (cv * 8 >= C) return;
  const int64_t c0 = cv * 8;
  const int64_t b = blockIdx.z;
  const int64_t t_begin = (int64_t)blockIdx.y * CONV_TOK;
  const int64_t t_end = t_begin + CONV_TOK < T ? t_begin + CONV_TOK : T;
  auto slot = [&](int buf, int u) { return &conv_stage[(buf * CONV_NR + u) * CONV_THREADS + threadIdx.x]; };
  // rows t .. t+n-1 into stage buf (one commit group)
  auto issue = [&](int64_t t, int buf, int64_t n) {
    for (int u = 0; u < n; ++u) cp_async16(slot(buf, u), x + (b * T + t + u) * ld_x + c0);
    cp_async_commit();
  };
  issue(t_begin, 0, t_end - t_begin < CONV_NR ? t_end - t_begin : CONV_NR);
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
  int g = 0;
  for (int64_t t = t_begin; t < t_end; t += CONV_NR, ++g) {
    const int64_t n = t_end - t < CONV_NR ? t_end - t : CONV_NR;
    if (t + CONV_NR < t_end) {
      const int64_t rest = t_end - t - CONV_NR;
      issue(t + CONV_NR, (g + 1) & 1, rest < CONV_NR ? rest : CONV_NR);
      cp_async_wait<1>();
    } else {
      cp_async_wait<0>();
    }
    for (int u = 0; u < n; ++u) {
      float cur[8], out[8];
      unpack8(*slot(g & 1, u), cur);
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
      *reinterpret_cast<uint4*>(y + (b * T + t + u) * ld_y + c0) = pack8(out);
    }
  }
  // the last three inputs (carried state included) for the next call
  if (state_out && t_end == T) {
#pragma unroll
    for (int i = 0; i < 3; ++i) *reinterpret_cast<uint4*>(state_out + (b * 3 + i) * C + c0) = pack8(win[i]);
  }
}

// A (token, head) row of DV bf16 values is DV/8 lanes x 16 bytes, so one
// warp-wide load covers 32/(DV/8) rows; each warp keeps NORM_NR such loads
// of o and of g in flight and walks the rows grid-stride.
constexpr int NORM_NR = 4;
constexpr int NORM_WARPS = 8;

template <int DV>
__global__ void __launch_bounds__(NORM_WARPS * 32) gated_rmsnorm_kernel(const uint16_t* __restrict__ o,
                                                                        const uint16_t* __restrict__ g, int64_t rows,
                                                                        const float* __restrict__ gamma,
                                                                        uint16_t* __restrict__ y,
                                                                        unsigned* __restrict__ amax) {
  constexpr int LPR = DV / 8;        // lanes per row
  constexpr int RPL = 32 / LPR;      // rows per warp-wide load
  constexpr int RPW = RPL * NORM_NR; // rows per warp step
  const int lane = threadIdx.x & 31;
  const int sub = lane / LPR, li = lane % LPR;
  float gm[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) gm[i] = gamma[li * 8 + i];
  uint32_t am = 0;
  const int64_t stride = (int64_t)gridDim.x * NORM_WARPS * RPW;
  for (int64_t base = ((int64_t)blockIdx.x * NORM_WARPS + (threadIdx.x >> 5)) * RPW; base < rows; base += stride) {
    uint4 ou[NORM_NR], gu[NORM_NR];
#pragma unroll
    for (int u = 0; u < NORM_NR; ++u) {
      const int64_t r = base + u * RPL + sub;
      if (r < rows) {
        ou[u] = *reinterpret_cast<const uint4*>(o + r * DV + li * 8);
        gu[u] = *reinterpret_cast<const uint4*>(g + r * DV + li * 8);
      } else {
        ou[u] = gu[u] = make_uint4(0u, 0u, 0u, 0u);
      }
    }
#pragma unroll
    for (int u = 0; u < NORM_NR; ++u) {
      float ov[8], gv[8];
      unpack8(ou[u], ov);
      unpack8(gu[u], gv);
      float ss = 0.0f;
#pragma unroll
      for (int i = 0; i < 8; ++i) ss = fmaf(ov[i], ov[i], ss);
#pragma unroll
      for (int d = LPR / 2; d > 0; d >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, d);   // within the row's lanes
      const float rr = __fdiv_rn(1.0f, __fsqrt_rn(__fdiv_rn(ss, (float)DV) + 1e-6f));
      float out[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) out[i] = ov[i] * rr * gm[i] * silu_f(gv[i]);
      const uint4 pk = pack8(out);
      const int64_t r = base + u * RPL + sub;
      if (r < rows) {
        *reinterpret_cast<uint4*>(y + r * DV + li * 8) = pk;
        const uint32_t w[4] = {pk.x, pk.y, pk.z, pk.w};
#pragma unroll
        for (int i = 0; i < 4; ++i)   // bf16 |value| as FP32 bits
          am = max(am, max((w[i] & 0x7FFFu) << 16, (w[i] >> 16 & 0x7FFFu) << 16));
      }
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
  // 64 KB of stage per block: three blocks per SM (80 registers) need the
  // largest shared-memory carveout, which the driver may not pick by itself
  cudaError_t e = cudaFuncSetAttribute(short_conv_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)CONV_SMEM);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(short_conv_kernel, cudaFuncAttributePreferredSharedMemoryCarveout,
                             (int)cudaSharedmemCarveoutMaxShared);
  if (e != cudaSuccess) return record_cuda_error(e);
  short_conv_kernel<<<grid, CONV_THREADS, CONV_SMEM, stream>>>(x, T, C, ld_x, w, state_in, y, ld_y, state_out);
  return check_launch();
}

int launch_gated_rmsnorm(const uint16_t* o, const uint16_t* g, int64_t M, int H, int dv, const float* gamma,
                         uint16_t* y, float* amax, cudaStream_t stream) {
  const int64_t rows = M * H;
  if (rows == 0) return GDN_OK;
  unsigned* am = reinterpret_cast<unsigned*>(amax);
  const int64_t rows_per_block = (int64_t)NORM_WARPS * NORM_NR * (32 / (dv / 8));
  const unsigned blocks = (unsigned)std::min<int64_t>(cdiv(rows, rows_per_block), (int64_t)num_sms() * 8);
  switch (dv) {
    case 32: gated_rmsnorm_kernel<32><<<blocks, NORM_WARPS * 32, 0, stream>>>(o, g, rows, gamma, y, am); break;
    case 64: gated_rmsnorm_kernel<64><<<blocks, NORM_WARPS * 32, 0, stream>>>(o, g, rows, gamma, y, am); break;
    default: gated_rmsnorm_kernel<128><<<blocks, NORM_WARPS * 32, 0, stream>>>(o, g, rows, gamma, y, am); break;
  }
  return check_launch();
}

}  // namespace gdn
