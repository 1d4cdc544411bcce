// Gated delta rule, token by token (decode and short continuations).
//
// Method: "Anthology of the SOTA, theory-128", section "The account" -- the
// state update S_t = alpha_t S_{t-1} + beta_t k_t (v_t - S_{t-1}^T k_t)^T and
// the read o_t = S_t^T q_t, over L2-normalised q and k.  With
// GDN_DR_DECAYED_READ the correction reads alpha_t S_{t-1} instead (the other
// common reading of the same update).
//
// One CTA per (batch, head) chain and block of 32 state columns (small CTAs,
// many per SM, so one CTA's state loads overlap another's arithmetic and
// stores).  The CTA's d_k x 32 block of the state is copied into shared
// memory by cp.async (16-byte pieces when the state is 16-byte aligned),
// updated there for every token of the call and copied back once, so the
// state is read from HBM once and written once, whatever T is; it holds no
// registers while it is in flight, which lets about twelve CTAs share an SM.
// Thread (part, j) owns column j of rows part, part + 4, ... (one warp per
// part, 32 adjacent columns: conflict-free).  Per token, warp 0 stages the
// normalised k and q in shared memory; the threads form r_j = S[:, j] . k
// (FP32 partial sums over their rows, then the four parts summed as
// (p0 + p1) + (p2 + p3)), u_j = beta (v_j - r_j), S[:, j] = alpha S[:, j] +
// k u_j and o_j = S[:, j] . q.  Columns are independent, so no state crosses
// columns.  HBM-bound at decode sizes: 2 d_k d_v 4 bytes of state per chain
// and call, plus the token's q, k, v, gates and o.
#include <atomic>

#include "common.cuh"
#include "kernels.h"

namespace gdn {
namespace {

constexpr int PARTS = 4;   // threads (warps) per state column
constexpr int COLS = 32;   // state columns per CTA

__device__ __forceinline__ void cp_async(uint32_t dst, const void* src, bool v16) {
  if (v16)
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
  else
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(dst), "l"(src) : "memory");
}

template <int DK, bool O_F32>
__global__ void __launch_bounds__(PARTS * COLS) delta_rule_step_kernel(
    const uint16_t* __restrict__ q, const uint16_t* __restrict__ k, const uint16_t* __restrict__ v, int64_t ld_q,
    int64_t ld_k, int64_t ld_v, const float* __restrict__ log_alpha, const float* __restrict__ beta,
    const float* S_in, float* S_out, int64_t T, int H, int dv, int l2norm, int decayed_read, void* __restrict__ o,
    int v16) {
  constexpr int R = DK / PARTS;   // state rows per thread: i = PARTS * e + part
  __shared__ __align__(16) float Ss[DK][COLS];
  __shared__ float kq[2][DK];
  __shared__ float red[PARTS][COLS];
  const int ncb = dv / COLS;
  const int64_t chain = blockIdx.x / ncb;
  const int64_t b = chain / H;
  const int h = (int)(chain % H);
  const int tid = threadIdx.x;
  const int part = tid / COLS, jc = tid % COLS;   // warp = part, lane = column in the block
  const int j = (int)(blockIdx.x % ncb) * COLS + jc;
  const int lane = tid & 31;
  const int64_t sbase = chain * DK * dv + (int64_t)(blockIdx.x % ncb) * COLS;

  // the state block into shared memory (or zeros)
  if (S_in) {
    if (v16) {
#pragma unroll
      for (int i = tid; i < DK * COLS / 4; i += PARTS * COLS) {
        const int row = i / (COLS / 4), c4 = (i % (COLS / 4)) * 4;
        cp_async(smem_u32(&Ss[row][c4]), S_in + sbase + (int64_t)row * dv + c4, true);
      }
    } else {
#pragma unroll 4
      for (int i = tid; i < DK * COLS; i += PARTS * COLS)
        cp_async(smem_u32(&Ss[i / COLS][i % COLS]), S_in + sbase + (int64_t)(i / COLS) * dv + i % COLS, false);
    }
    asm volatile("cp.async.commit_group;" ::: "memory");
  } else {
    for (int i = tid; i < DK * COLS; i += PARTS * COLS) Ss[i / COLS][i % COLS] = 0.0f;
  }

  for (int64_t t = 0; t < T; ++t) {
    const int64_t tok = b * T + t;
    __syncthreads();   // the previous token's k, q and reductions have been read
    if (tid < 32) {
      constexpr int PER = DK / 32;
      float kr[PER], qr[PER];
      float kk = 0.0f, qq = 0.0f;
#pragma unroll
      for (int e = 0; e < PER; ++e) {
        const int i = lane + 32 * e;
        kr[e] = bf16_bits_to_f32(k[tok * ld_k + (int64_t)h * DK + i]);
        qr[e] = bf16_bits_to_f32(q[tok * ld_q + (int64_t)h * DK + i]);
        kk = fmaf(kr[e], kr[e], kk);
        qq = fmaf(qr[e], qr[e], qq);
      }
      float ik = 1.0f, iq = 1.0f;
      if (l2norm) {
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) {
          kk += __shfl_xor_sync(0xffffffffu, kk, off);
          qq += __shfl_xor_sync(0xffffffffu, qq, off);
        }
        ik = __fdiv_rn(1.0f, __fsqrt_rn(kk + 1e-6f));
        iq = __fdiv_rn(1.0f, __fsqrt_rn(qq + 1e-6f));
      }
#pragma unroll
      for (int e = 0; e < PER; ++e) {
        kq[0][lane + 32 * e] = kr[e] * ik;
        kq[1][lane + 32 * e] = qr[e] * iq;
      }
    }
    const int64_t gi = tok * H + h;
    const float a = expf(log_alpha[gi]);
    const float bt = beta[gi];
    const float vj = bf16_bits_to_f32(v[tok * ld_v + (int64_t)h * dv + j]);
    if (t == 0 && S_in) asm volatile("cp.async.wait_group 0;" ::: "memory");
    __syncthreads();
    // r_j = S[:, j] . k: this thread's rows, then the column's four parts
    float r = 0.0f;
#pragma unroll
    for (int e = 0; e < R; ++e) r = fmaf(Ss[PARTS * e + part][jc], kq[0][PARTS * e + part], r);
    red[part][jc] = r;
    __syncthreads();
    r = (red[0][jc] + red[1][jc]) + (red[2][jc] + red[3][jc]);
    if (decayed_read) r *= a;
    const float u = bt * (vj - r);
    float y = 0.0f;
#pragma unroll
    for (int e = 0; e < R; ++e) {
      const int i = PARTS * e + part;
      const float sv = fmaf(a, Ss[i][jc], kq[0][i] * u);
      Ss[i][jc] = sv;
      y = fmaf(sv, kq[1][i], y);
    }
    __syncthreads();   // every part has read red for r
    red[part][jc] = y;
    __syncthreads();
    if (part == 0) {
      y = (red[0][jc] + red[1][jc]) + (red[2][jc] + red[3][jc]);
      const int64_t oi = gi * dv + j;
      if (O_F32)
        static_cast<float*>(o)[oi] = y;
      else
        static_cast<uint16_t*>(o)[oi] = (uint16_t)f32_to_bf16_bits(y);
    }
  }

  if (T == 0 && S_in) asm volatile("cp.async.wait_group 0;" ::: "memory");
  __syncthreads();
  if (v16) {
#pragma unroll
    for (int i = tid; i < DK * COLS / 4; i += PARTS * COLS) {
      const int row = i / (COLS / 4), c4 = (i % (COLS / 4)) * 4;
      *reinterpret_cast<float4*>(S_out + sbase + (int64_t)row * dv + c4) =
          *reinterpret_cast<const float4*>(&Ss[row][c4]);
    }
  } else {
    for (int i = tid; i < DK * COLS; i += PARTS * COLS)
      S_out[sbase + (int64_t)(i / COLS) * dv + i % COLS] = Ss[i / COLS][i % COLS];
  }
}

// About twelve 18 KB CTAs share an SM only with the largest shared-memory
// carveout, which the driver may not pick for so small a block by itself;
// asked for once per kernel and device.
template <typename K>
void prefer_shared(K kernel, std::atomic<uint64_t>& done) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return;
  const uint64_t bit = 1ull << dev;
  if (done.load(std::memory_order_relaxed) & bit) return;
  if (cudaFuncSetAttribute(kernel, cudaFuncAttributePreferredSharedMemoryCarveout,
                           (int)cudaSharedmemCarveoutMaxShared) == cudaSuccess)
    done.fetch_or(bit, std::memory_order_relaxed);
  else
    cudaGetLastError();
}

template <int DK>
void launch_dk(bool o_f32, dim3 grid, int dv, cudaStream_t stream, const uint16_t* q, const uint16_t* k,
               const uint16_t* v, int64_t ld_q, int64_t ld_k, int64_t ld_v, const float* log_alpha,
               const float* beta, const float* S_in, float* S_out, int64_t T, int H, int l2norm, int decayed,
               void* o, int v16) {
  static std::atomic<uint64_t> done_f32{0}, done_bf16{0};
  if (o_f32)
    prefer_shared(delta_rule_step_kernel<DK, true>, done_f32);
  else
    prefer_shared(delta_rule_step_kernel<DK, false>, done_bf16);
  if (o_f32)
    delta_rule_step_kernel<DK, true><<<grid, PARTS * COLS, 0, stream>>>(q, k, v, ld_q, ld_k, ld_v, log_alpha, beta, S_in,
                                                              S_out, T, H, dv, l2norm, decayed, o, v16);
  else
    delta_rule_step_kernel<DK, false><<<grid, PARTS * COLS, 0, stream>>>(q, k, v, ld_q, ld_k, ld_v, log_alpha, beta, S_in,
                                                               S_out, T, H, dv, l2norm, decayed, o, v16);
}

}  // namespace

int launch_delta_rule_step(const uint16_t* q, const uint16_t* k, const uint16_t* v, int64_t ld_q, int64_t ld_k,
                           int64_t ld_v, const float* log_alpha, const float* beta, const float* S_in, float* S_out,
                           int64_t B, int64_t T, int H, int dk, int dv, int flags, void* o, cudaStream_t stream) {
  const int64_t chains = B * H;
  if (chains == 0) return GDN_OK;
  const dim3 grid((unsigned)(chains * (dv / COLS)));
  const bool o_f32 = (flags & GDN_DR_O_FP32) != 0;
  const int l2 = (flags & GDN_DR_L2NORM_QK) ? 1 : 0;
  const int dec = (flags & GDN_DR_DECAYED_READ) ? 1 : 0;
  // 16-byte state pieces when both state buffers allow them
  const int v16 = (!S_in || reinterpret_cast<uintptr_t>(S_in) % 16 == 0) && reinterpret_cast<uintptr_t>(S_out) % 16 == 0;
  switch (dk) {
    case 32:
      launch_dk<32>(o_f32, grid, dv, stream, q, k, v, ld_q, ld_k, ld_v, log_alpha, beta, S_in, S_out, T, H, l2, dec,
                    o, v16);
      break;
    case 64:
      launch_dk<64>(o_f32, grid, dv, stream, q, k, v, ld_q, ld_k, ld_v, log_alpha, beta, S_in, S_out, T, H, l2, dec,
                    o, v16);
      break;
    default:
      launch_dk<128>(o_f32, grid, dv, stream, q, k, v, ld_q, ld_k, ld_v, log_alpha, beta, S_in, S_out, T, H, l2, dec,
                     o, v16);
      break;
  }
  return check_launch();
}

}  // namespace gdn
