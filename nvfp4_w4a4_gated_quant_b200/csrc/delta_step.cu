// Gated delta rule, token by token (decode and short continuations).
//
// Method: "Anthology of the SOTA, theory-128", section "The account" -- the
// state update S_t = alpha_t S_{t-1} + beta_t k_t (v_t - S_{t-1}^T k_t)^T and
// the read o_t = S_t^T q_t, over L2-normalised q and k.  With
// GDN_DR_DECAYED_READ the correction reads alpha_t S_{t-1} instead (the other
// common reading of the same update).
//
// One CTA per (batch, head) chain and block of 32 state columns (small CTAs,
// several per SM, so one CTA's state loads overlap another's arithmetic and
// stores), four adjacent threads per column j of the d_k x d_v state, each
// holding every fourth row of it in registers for the whole call, so the
// state is read from HBM once and written once, whatever T is.  Per token,
// warp 0 of each CTA stages the normalised k and q in shared memory; the
// threads then form r_j = S[:, j] . k (FP32 partial sums, combined across the
// column's four lanes by shuffles), u_j = beta (v_j - r_j),
// S[:, j] = alpha S[:, j] + k u_j and o_j = S[:, j] . q.  Columns are
// independent, so no state crosses columns.  HBM-bound at decode sizes:
// 2 d_k d_v 4 bytes of state per chain and call, plus the token's q, k, v,
// gates and o.
#include "common.cuh"
#include "kernels.h"

namespace gdn {
namespace {

constexpr int PARTS = 4;   // threads per state column
constexpr int COLS = 32;   // state columns per CTA

template <int DK, bool O_F32>
__global__ void __launch_bounds__(PARTS * COLS) delta_rule_step_kernel(
    const uint16_t* __restrict__ q, const uint16_t* __restrict__ k, const uint16_t* __restrict__ v, int64_t ld_q,
    int64_t ld_k, int64_t ld_v, const float* __restrict__ log_alpha, const float* __restrict__ beta,
    const float* S_in, float* S_out, int64_t T, int H, int dv, int l2norm, int decayed_read, void* __restrict__ o) {
  constexpr int R = DK / PARTS;   // state rows per thread: i = PARTS * e + part
  __shared__ float kq[2][DK];
  const int ncb = dv / COLS;             // column blocks per chain
  const int64_t chain = blockIdx.x / ncb;
  const int64_t b = chain / H;
  const int h = (int)(chain % H);
  const int j = (int)(blockIdx.x % ncb) * COLS + threadIdx.x / PARTS;   // column of the state
  const int part = threadIdx.x % PARTS;
  const int lane = threadIdx.x & 31;

  float s[R];
  const int64_t sbase = chain * DK * dv + j;
#pragma unroll
  for (int e = 0; e < R; ++e) s[e] = S_in ? S_in[sbase + (int64_t)(PARTS * e + part) * dv] : 0.0f;

  for (int64_t t = 0; t < T; ++t) {
    const int64_t tok = b * T + t;
    __syncthreads();   // the previous token's k and q have been read
    if (threadIdx.x < 32) {
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
    __syncthreads();
    const int64_t gi = tok * H + h;
    const float a = expf(log_alpha[gi]);
    const float bt = beta[gi];
    // r_j = S[:, j] . k: this thread's rows, then the column's PARTS threads
    // (adjacent lanes of one warp)
    float r = 0.0f;
#pragma unroll
    for (int e = 0; e < R; ++e) r = fmaf(s[e], kq[0][PARTS * e + part], r);
#pragma unroll
    for (int off = 1; off < PARTS; off <<= 1) r += __shfl_xor_sync(0xffffffffu, r, off);
    if (decayed_read) r *= a;
    const float u = bt * (bf16_bits_to_f32(v[tok * ld_v + (int64_t)h * dv + j]) - r);
    float y = 0.0f;
#pragma unroll
    for (int e = 0; e < R; ++e) {
      s[e] = fmaf(a, s[e], kq[0][PARTS * e + part] * u);
      y = fmaf(s[e], kq[1][PARTS * e + part], y);
    }
#pragma unroll
    for (int off = 1; off < PARTS; off <<= 1) y += __shfl_xor_sync(0xffffffffu, y, off);
    if (part == 0) {
      const int64_t oi = gi * dv + j;
      if (O_F32)
        static_cast<float*>(o)[oi] = y;
      else
        static_cast<uint16_t*>(o)[oi] = (uint16_t)f32_to_bf16_bits(y);
    }
  }

#pragma unroll
  for (int e = 0; e < R; ++e) S_out[sbase + (int64_t)(PARTS * e + part) * dv] = s[e];
}

template <int DK>
void launch_dk(bool o_f32, dim3 grid, int dv, cudaStream_t stream, const uint16_t* q, const uint16_t* k,
               const uint16_t* v, int64_t ld_q, int64_t ld_k, int64_t ld_v, const float* log_alpha,
               const float* beta, const float* S_in, float* S_out, int64_t T, int H, int l2norm, int decayed,
               void* o) {
  if (o_f32)
    delta_rule_step_kernel<DK, true><<<grid, PARTS * COLS, 0, stream>>>(q, k, v, ld_q, ld_k, ld_v, log_alpha, beta, S_in,
                                                              S_out, T, H, dv, l2norm, decayed, o);
  else
    delta_rule_step_kernel<DK, false><<<grid, PARTS * COLS, 0, stream>>>(q, k, v, ld_q, ld_k, ld_v, log_alpha, beta, S_in,
                                                               S_out, T, H, dv, l2norm, decayed, o);
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
  switch (dk) {
    case 32:
      launch_dk<32>(o_f32, grid, dv, stream, q, k, v, ld_q, ld_k, ld_v, log_alpha, beta, S_in, S_out, T, H, l2, dec, o);
      break;
    case 64:
      launch_dk<64>(o_f32, grid, dv, stream, q, k, v, ld_q, ld_k, ld_v, log_alpha, beta, S_in, S_out, T, H, l2, dec, o);
      break;
    default:
      launch_dk<128>(o_f32, grid, dv, stream, q, k, v, ld_q, ld_k, ld_v, log_alpha, beta, S_in, S_out, T, H, l2, dec,
                     o);
      break;
  }
  return check_launch();
}

}  // namespace gdn
