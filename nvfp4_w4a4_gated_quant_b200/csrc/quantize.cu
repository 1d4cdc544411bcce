// NVFP4 activation quantizer: per-tensor amax, E4M3 block scales, E2M1 codes.
//
// Method: "Why Gated DeltaNet Survives 4-Bit Quantization", section "Why the
// 'Fragile' Recurrence is Actually Robust" -- NVFP4 scales every 16-element
// block separately.  Two HBM-bound passes:
//   amax_kernel   max |x| over the tensor (bf16 bit patterns, one atomicMax
//                 per CTA on the FP32 bits of the result), four rows per step;
//   quant_kernel  one thread per 16-element block and row: two 16-byte loads,
//                 the block scale, eight packed code bytes and one scale byte;
//                 two rows per step.
// CTA widths are chosen so the threads tile a row with the fewest left idle.
// The FP32 operation order is fixed (see gdn.h); divisions and products use
// the round-to-nearest intrinsics so no contraction or approximation changes
// a code.  E4M3 and E2M1 rounding use the hardware cvt.rn.satfinite forms.
#include <float.h>
#include <stdint.h>

#include "common.cuh"
#include "kernels.h"
#include "quant_math.cuh"

namespace gdn {
namespace {

__device__ __forceinline__ uint4 ld_vec(const void* p) { return *reinterpret_cast<const uint4*>(p); }

template <typename In, typename E>
__global__ void amax_kernel(const E* __restrict__ x, int64_t rows, int64_t vpr, int64_t ld,
                            unsigned* __restrict__ amax_bits) {
  uint32_t m = 0;
  // four rows per step: four independent 16-byte loads in flight per thread
  const int64_t gy = gridDim.y;
  for (int64_t r = blockIdx.y; r < rows; r += 4 * gy) {
    for (int64_t c = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; c < vpr; c += (int64_t)gridDim.x * blockDim.x) {
      uint4 v[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int64_t rr = r + u * gy;
        v[u] = rr < rows ? ld_vec(x + rr * ld + c * In::kPerVec) : make_uint4(0u, 0u, 0u, 0u);
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) m = max(m, In::absmax_bits(v[u]));
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = max(m, __shfl_xor_sync(0xffffffffu, m, o));
  __shared__ uint32_t red[32];
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = m;
  __syncthreads();
  if (threadIdx.x < 32) {
    m = threadIdx.x < (blockDim.x >> 5) ? red[threadIdx.x] : 0u;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = max(m, __shfl_xor_sync(0xffffffffu, m, o));
    if (threadIdx.x == 0 && m) atomicMax(amax_bits, m);  // FP32 bits of |x| order like the values
  }
}

template <typename In, typename E>
__global__ void quant_kernel(const E* __restrict__ x, int64_t rows, int64_t cols, int64_t ld,
                             int mode, const float* __restrict__ g_enc_in,
                             const unsigned* __restrict__ amax_bits, uint8_t* __restrict__ codes,
                             uint8_t* __restrict__ scales, int tiled, int64_t row_off,
                             float* __restrict__ g_out) {
  const float g_enc = mode == GDN_QUANT_DYNAMIC      ? encode_scale_from_amax(__uint_as_float(*amax_bits))
                      : mode == GDN_QUANT_GIVEN_AMAX ? encode_scale_from_amax(*g_enc_in)
                                                     : *g_enc_in;
  if (blockIdx.x == 0 && blockIdx.y == 0 && threadIdx.x == 0) *g_out = __fdiv_rn(1.0f, g_enc);
  const int64_t bpr = cols >> 4;  // 16-element blocks per row
  const int64_t kc = cols >> 6;   // 64-element scale chunks per row (TILED)
  // Two rows per step so that each thread has two blocks' loads in flight.
  constexpr int RU = 2;
  const int64_t gy = gridDim.y;
  for (int64_t r = blockIdx.y; r < rows; r += RU * gy) {
    for (int64_t j = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; j < bpr; j += (int64_t)gridDim.x * blockDim.x) {
      constexpr int NV = 16 / In::kPerVec;
      uint4 v[RU][NV];
#pragma unroll
      for (int u = 0; u < RU; ++u) {
        const int64_t rr = r + u * gy;
        if (rr < rows) {
#pragma unroll
          for (int i = 0; i < NV; ++i) v[u][i] = ld_vec(x + rr * ld + j * 16 + i * In::kPerVec);
        }
      }
#pragma unroll
      for (int u = 0; u < RU; ++u) {
        const int64_t rr = r + u * gy;
        if (rr < rows)
          quant_block<In>(v[u], g_enc, codes + rr * (cols >> 1) + j * 8,
                          tiled ? scales + scale_offset(rr + row_off, j, kc) : scales + rr * bpr + j);
      }
    }
  }
}

// Threads per CTA for rows of n items: the width among a few warp multiples
// that leaves the fewest idle threads at the end of a row (the layer's rows
// have 640 vectors and 320 blocks; 256-wide CTAs would idle 17% and 37%).
int threads_for_row(int64_t n) {
  const int cands[] = {256, 192, 160, 128, 96, 64};
  int best = 256;
  int64_t best_waste = INT64_MAX;
  for (int t : cands) {
    const int64_t waste = cdiv(n, t) * t - n;
    if (waste < best_waste) best = t, best_waste = waste;
  }
  return best;
}

void grid_for_rows(int64_t rows, int64_t per_row_items, int threads, dim3& grid) {
  const int64_t gx = std::min<int64_t>(cdiv(per_row_items, threads), 1024);
  const int64_t want = (int64_t)num_sms() * 16;  // CTAs in flight
  int64_t gy = std::max<int64_t>(1, want / std::max<int64_t>(gx, 1));
  gy = std::min<int64_t>(gy, std::max<int64_t>(rows, 1));
  gy = std::min<int64_t>(gy, 65535);
  grid = dim3((unsigned)std::max<int64_t>(gx, 1), (unsigned)gy, 1);
}

// The amax pass runs exactly one resident wave (SMs x CTAs that fit per SM
// at this width): several waves left part of the machine idle at the end of
// the pass (32768 x 5120 bf16, amax + quant: 171 -> 161 us).  The quant pass
// keeps several waves: one wave made it slower (84 -> 107 us).
template <typename K>
void grid_one_wave(K kernel, int64_t rows, int64_t per_row_items, int threads, dim3& grid) {
  int per_sm = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, threads, 0) != cudaSuccess || per_sm < 1) {
    cudaGetLastError();
    per_sm = 1;
  }
  const int64_t gx = std::min<int64_t>(cdiv(per_row_items, threads), 1024);
  int64_t gy = std::max<int64_t>(1, (int64_t)num_sms() * per_sm / std::max<int64_t>(gx, 1));
  gy = std::min<int64_t>(gy, std::max<int64_t>(rows, 1));
  gy = std::min<int64_t>(gy, 65535);
  grid = dim3((unsigned)std::max<int64_t>(gx, 1), (unsigned)gy, 1);
}

template <typename In, typename E>
int launch_quantize_t(const E* x, int64_t rows, int64_t cols, int64_t ld, int mode, const float* g_enc_in,
                    uint8_t* codes, uint8_t* scales, int tiled, int64_t row_off, float* g_out, unsigned* amax_ws,
                    cudaStream_t stream) {
  if (mode == GDN_QUANT_DYNAMIC) {
    cudaError_t e = cudaMemsetAsync(amax_ws, 0, sizeof(unsigned), stream);
    if (e != cudaSuccess) return record_cuda_error(e);
    if (rows > 0) {
      const int at = threads_for_row(cols / In::kPerVec);
      dim3 grid;
      grid_one_wave(amax_kernel<In, E>, rows, cols / In::kPerVec, at, grid);
      amax_kernel<In, E><<<grid, at, 0, stream>>>(x, rows, cols / In::kPerVec, ld, amax_ws);
      int st = check_launch();
      if (st) return st;
    }
  }
  const int threads = threads_for_row(cols / 16);
  dim3 grid;
  grid_for_rows(rows, cols / 16, threads, grid);
  quant_kernel<In, E><<<grid, threads, 0, stream>>>(x, rows, cols, ld, mode, g_enc_in, amax_ws, codes, scales, tiled,
                                             row_off, g_out);
  return check_launch();
}

// *g_enc = 2688 / *amax (the per-tensor encode scale of a calibrated amax).
__global__ void encode_scale_kernel(const float* __restrict__ amax, float* __restrict__ g_enc) {
  *g_enc = encode_scale_from_amax(*amax);
}

template <typename In, typename E>
int launch_amax_update_t(const E* x, int64_t rows, int64_t cols, int64_t ld, unsigned* amax_bits,
                         cudaStream_t stream) {
  if (rows == 0) return GDN_OK;
  const int at = threads_for_row(cols / In::kPerVec);
  dim3 grid;
  grid_one_wave(amax_kernel<In, E>, rows, cols / In::kPerVec, at, grid);
  amax_kernel<In, E><<<grid, at, 0, stream>>>(x, rows, cols / In::kPerVec, ld, amax_bits);
  return check_launch();
}

}  // namespace

int launch_amax_update(const void* x, int x_dtype, int64_t rows, int64_t cols, int64_t ld, float* amax,
                       cudaStream_t stream) {
  unsigned* bits = reinterpret_cast<unsigned*>(amax);
  if (x_dtype == GDN_DTYPE_F32)
    return launch_amax_update_t<F32In>(static_cast<const float*>(x), rows, cols, ld, bits, stream);
  return launch_amax_update_t<Bf16In>(static_cast<const uint16_t*>(x), rows, cols, ld, bits, stream);
}

int launch_encode_scale(const float* amax, float* g_enc, cudaStream_t stream) {
  encode_scale_kernel<<<1, 1, 0, stream>>>(amax, g_enc);
  return check_launch();
}

int launch_quantize(const void* x, int x_dtype, int64_t rows, int64_t cols, int64_t ld, int mode,
                    const float* g_enc_in, uint8_t* codes, uint8_t* scales, int tiled, int64_t row_off, float* g_out,
                    unsigned* amax_ws, cudaStream_t stream) {
  if (x_dtype == GDN_DTYPE_F32)
    return launch_quantize_t<F32In>(static_cast<const float*>(x), rows, cols, ld, mode, g_enc_in, codes, scales,
                                    tiled, row_off, g_out, amax_ws, stream);
  return launch_quantize_t<Bf16In>(static_cast<const uint16_t*>(x), rows, cols, ld, mode, g_enc_in, codes, scales,
                                   tiled, row_off, g_out, amax_ws, stream);
}

}  // namespace gdn
