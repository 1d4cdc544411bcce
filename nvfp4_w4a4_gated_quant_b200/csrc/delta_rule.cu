// Chunked gated delta rule forward (sm_100a).
//
// Recurrence ("Anthology of the SOTA, theory-128", section "The account"):
//   S_t = alpha_t S_{t-1} + beta_t k_t (v_t - S_{t-1}^T k_t)^T,   o_t = S_t^T q_t
// over L2-normalised q, k.  With u_t = beta_t (v_t - S_{t-1}^T k_t) and, inside
// a chunk of C = 64 tokens entered with state S, G_t = sum_{s<=t} log alpha_s:
//   L_ts = beta_t e^{G_{t-1}-G_s} k_t.k_s (s < t),   X = (I + L)^{-1}
//   U    = X diag(beta) V - X diag(beta e^{G_{t-1}}) K S          (= U~ - W S)
//   O    = diag(e^{G_t}) Q S + (Gamma o Q K^T) U,  Gamma_ts = e^{G_t-G_s} (s <= t)
//   S'   = e^{G_C} S + (diag(e^{G_C-G_s}) K)^T U
// Every exponent is <= 0, so nothing overflows whatever the decay.
//
// One CTA of 8 warps walks one (batch, head, d_v slice) chain chunk by chunk.
// The columns of S evolve independently (column j only sees v[:, j]), so a
// head's d_v is split into slices of DVS columns across CTAs when there are
// too few (batch, head) chains to fill the SMs.  Per chunk:
//   P0  gates: inclusive scan of log alpha (FP32), per-token decay factors;
//       q, k L2-normalised in FP32 and stored FP16; beta*v as FP16.
//   P1  K K^T and Q K^T on mma.sync m16n8k16 (FP16 in, FP32 accumulate) with
//       the decay / beta factors applied in FP32 -> L and Gamma o QK^T (FP16).
//   P2  X = (I + L)^{-1}: 16x16 diagonal blocks by forward substitution,
//       off-diagonal blocks by X_ij = -sum_k (X_ii L_ik) X_kj on mma.sync.
//   P3  W = X diag(beta e^{G_{t-1}}) K and U~ = X (beta o V) on mma.sync.
//   P4  the state-dependent part: U = U~ - W S and Q S (S as FP16), then
//       O = e^{G_t} Q S + A U and S' = e^{G_C} S + Kd^T U, S kept in FP32
//       registers across chunks.
// The next chunk's raw q / k / v / gates are prefetched with cp.async while
// the current chunk computes.  Supported: d_k in {32, 64, 128}, d_v slices of
// DVS in {16, 32, 64, 128} columns.
#include <cuda_fp16.h>

#include "common.cuh"
#include "kernels.h"

namespace gdn {
namespace {

constexpr int C = 64;        // chunk length
constexpr int NT = 256;      // 8 warps
constexpr int LDX = C + 8;   // FP16 row stride of 64-wide tiles
constexpr float kLog2e = 1.4426950408889634f;

template <int DK, int DVS>
struct Smem {
  static constexpr int LDH = DK + 8;   // FP16 row stride of d_k-wide tiles (halves)
  static constexpr int LDR = DK + 8;   // bf16 staging row stride (halves)
  static constexpr int LDV = DVS + 8;
  // raw bf16 staging of the next chunk
  uint16_t qr[C * LDR];
  uint16_t kr[C * LDR];
  uint16_t vr[C * LDV];
  float lar[C];
  float ber[C];
  // FP16 operands of the current chunk
  __half qh[C * LDH];     // q_hat
  __half kh[C * LDH];     // k_hat
  __half kd[C * LDH];     // e^{G_C - G_s} k_hat_s
  __half vh[C * LDV];     // beta o v, later U (the new values)
  __half lh[C * LDX];     // L
  __half ah[C * LDX];     // Gamma o Q K^T
  __half xh[C * LDX];     // X = (I + L)^{-1}
  __half xw[C * LDX];     // X diag(beta e^{G_{t-1}})
  __half wh[C * LDH];     // -W
  __half sh[DK * LDV];    // S as FP16
  // per-token factors
  float g2[C];            // G_t * log2(e)
  float g2m1[C];          // G_{t-1} * log2(e)
  float be[C];
  float d1[C];            // beta_t e^{G_{t-1}}
  float eg[C];            // e^{G_t}
  float dk[C];            // e^{G_C - G_t}
  float warp_tot;
};

// ---------------------------------------------------------------- helpers
__device__ __forceinline__ void mma16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
__device__ __forceinline__ void ldsm4(uint32_t (&r)[4], const void* p) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(smem_u32(p)));
}
__device__ __forceinline__ void ldsm4t(uint32_t (&r)[4], const void* p) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(smem_u32(p)));
}
__device__ __forceinline__ void ldsm2t(uint32_t& r0, uint32_t& r1, const void* p) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x2.trans.shared.b16 {%0,%1}, [%2];"
               : "=r"(r0), "=r"(r1)
               : "r"(smem_u32(p)));
}

// A fragment (16 x 16) of a row-major [m][k] tile at (m0, k0).
__device__ __forceinline__ void frag_a(uint32_t (&a)[4], const __half* base, int ld, int m0, int k0, int lane) {
  const int i = lane >> 3;
  ldsm4(a, base + (m0 + (lane & 7) + (i & 1) * 8) * ld + k0 + (i >> 1) * 8);
}
// A fragment of A = T^T where T is stored row-major [k][m].
__device__ __forceinline__ void frag_a_t(uint32_t (&a)[4], const __half* base, int ld, int m0, int k0, int lane) {
  const int i = lane >> 3;
  ldsm4t(a, base + (k0 + (lane & 7) + (i >> 1) * 8) * ld + m0 + (i & 1) * 8);
}
// B fragments of two adjacent n-tiles (n0, n0+8) for B[k][n] stored [n][k].
__device__ __forceinline__ void frag_b_nk(uint32_t (&b)[4], const __half* base, int ld, int k0, int n0, int lane) {
  const int i = lane >> 3;
  ldsm4(b, base + (n0 + (lane & 7) + (i >> 1) * 8) * ld + k0 + (i & 1) * 8);
}
// B fragments of two adjacent n-tiles for B[k][n] stored row-major [k][n].
__device__ __forceinline__ void frag_b_kn(uint32_t (&b)[4], const __half* base, int ld, int k0, int n0, int lane) {
  const int i = lane >> 3;
  ldsm4t(b, base + (k0 + (lane & 7) + (i & 1) * 8) * ld + n0 + (i >> 1) * 8);
}
// B fragment of one n-tile for B[k][n] stored row-major [k][n].
__device__ __forceinline__ void frag_b_kn1(uint32_t& b0, uint32_t& b1, const __half* base, int ld, int k0, int n0,
                                           int lane) {
  const int i = (lane >> 3) & 1;
  ldsm2t(b0, b1, base + (k0 + (lane & 7) + i * 8) * ld + n0);
}

__device__ __forceinline__ uint32_t pack_h2(float lo, float hi) {
  __half2 h = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}
__device__ __forceinline__ void st_h2(__half* p, float lo, float hi) {
  *reinterpret_cast<__half2*>(p) = __floats2half2_rn(lo, hi);
}
// The C fragments of two adjacent n-tiles (16 x 16) as an A fragment.
__device__ __forceinline__ void c_to_a(uint32_t (&a)[4], const float (&c0)[4], const float (&c1)[4]) {
  a[0] = pack_h2(c0[0], c0[1]);
  a[1] = pack_h2(c0[2], c0[3]);
  a[2] = pack_h2(c1[0], c1[1]);
  a[3] = pack_h2(c1[2], c1[3]);
}

__device__ __forceinline__ void cp_async16(void* dst, const void* src, bool valid) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_u32(dst)), "l"(src),
               "r"(valid ? 16 : 0)
               : "memory");
}
__device__ __forceinline__ void cp_async4(void* dst, const void* src, bool valid) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;" ::"r"(smem_u32(dst)), "l"(src), "r"(valid ? 4 : 0)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_group 0;" ::: "memory"); }

struct Args {
  const uint16_t* q;
  const uint16_t* k;
  const uint16_t* v;
  int64_t ld_q, ld_k, ld_v;
  const float* log_alpha;
  const float* beta;
  const float* S0;
  int64_t T;
  int H, dv, nsplit;
  int l2norm;
  void* o;
  float* S_T;
  unsigned* o_amax;   // optional: FP32 bits of max |stored o| (atomicMax), for the next quantizer
  int* status;        // device status word (GDN_ERR_RANGE when an output is not finite)
};

template <int DK, int DVS>
__device__ __forceinline__ void issue_chunk_loads(Smem<DK, DVS>& sm, const Args& a, int64_t bt0, int h, int dv_off,
                                                  int valid, int tid) {
  constexpr int LDV = Smem<DK, DVS>::LDV;
  constexpr int LDR = Smem<DK, DVS>::LDR;
  constexpr int QV = DK / 8;  // 16-byte vectors per q / k row
  for (int i = tid; i < C * QV; i += NT) {
    const int r = i / QV, c = i % QV;
    const bool ok = r < valid;
    const int64_t tok = bt0 + (ok ? r : 0);
    cp_async16(&sm.qr[r * LDR + c * 8], a.q + tok * a.ld_q + (int64_t)h * DK + c * 8, ok);
    cp_async16(&sm.kr[r * LDR + c * 8], a.k + tok * a.ld_k + (int64_t)h * DK + c * 8, ok);
  }
  constexpr int VV = DVS / 8;
  for (int i = tid; i < C * VV; i += NT) {
    const int r = i / VV, c = i % VV;
    const bool ok = r < valid;
    const int64_t tok = bt0 + (ok ? r : 0);
    cp_async16(&sm.vr[r * LDV + c * 8], a.v + tok * a.ld_v + (int64_t)h * a.dv + dv_off + c * 8, ok);
  }
  if (tid < C) {
    const bool ok = tid < valid;
    const int64_t tok = bt0 + (ok ? tid : 0);
    cp_async4(&sm.lar[tid], a.log_alpha + tok * a.H + h, ok);
    cp_async4(&sm.ber[tid], a.beta + tok * a.H + h, ok);
  }
  cp_async_commit();
}

template <int DK, int DVS, bool O_F32>
__global__ void __launch_bounds__(NT, 1) delta_rule_kernel(const __grid_constant__ Args a) {
  constexpr int LDV = Smem<DK, DVS>::LDV;
  constexpr int LDH = Smem<DK, DVS>::LDH;
  constexpr int LDR = Smem<DK, DVS>::LDR;
  constexpr int SW = DK / 16;         // warps that own 16 state rows each
  constexpr int KH = DK / 32;         // 16-wide d_k column pairs per warp half (W)
  constexpr int NVT = DVS / 8;        // n-tiles of the d_v slice
  constexpr int NVH = NVT / 2;        // n-tiles per warp half
  static_assert(DVS >= 16 && DVS % 16 == 0, "d_v slice must be a multiple of 16");
  extern __shared__ __align__(16) uint8_t smem_raw[];
  Smem<DK, DVS>& sm = *reinterpret_cast<Smem<DK, DVS>*>(smem_raw);

  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  const int g = lane >> 2, c4 = lane & 3;
  const int mrow = warp & 3;   // chunk rows 16*mrow .. +15
  const int nhalf = warp >> 2;

  const int chain = blockIdx.x / a.nsplit;
  const int split = blockIdx.x % a.nsplit;
  const int b = chain / a.H, h = chain % a.H;
  const int dv_off = split * DVS;
  const int64_t T = a.T;
  const int64_t tok0 = (int64_t)b * T;

  // Warps 0 .. SW-1 own state rows 16*warp .. +15 (d_k), all DVS columns, FP32.
  const bool s_owner = warp < SW;
  float S[NVT][4];
#pragma unroll
  for (int j = 0; j < NVT; ++j)
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int r = 16 * warp + g + (e >> 1) * 8, col = 8 * j + 2 * c4 + (e & 1);
      S[j][e] = (a.S0 && s_owner) ? a.S0[((int64_t)chain * DK + r) * a.dv + dv_off + col] : 0.0f;
    }

  uint32_t amax_bits = 0;   // FP32 bits of the largest |o| this thread stored
  const int64_t nchunks = (T + C - 1) / C;
  if (nchunks > 0) issue_chunk_loads<DK, DVS>(sm, a, tok0, h, dv_off, (int)(T < C ? T : C), tid);

  for (int64_t ch = 0; ch < nchunks; ++ch) {
    const int64_t t0 = ch * C;
    const int valid = (int)(T - t0 < C ? T - t0 : C);
    cp_async_wait_all();
    __syncthreads();

    // ---------------------------------------------------- P0: gates, norms
    // q, k rows: four threads per row (DK/4 columns each), FP32 norms.
    constexpr int QC = DK / 4;
    const int pr = tid >> 2, pq = tid & 3;
    float qv[QC], kv[QC];
    float nq, nk;
    {
      const uint4* qsrc = reinterpret_cast<const uint4*>(&sm.qr[pr * LDR + pq * QC]);
      const uint4* ksrc = reinterpret_cast<const uint4*>(&sm.kr[pr * LDR + pq * QC]);
      float qs = 0.f, ks = 0.f;
#pragma unroll
      for (int i = 0; i < QC / 8; ++i) {
        const uint4 uq = qsrc[i], uk = ksrc[i];
        const uint32_t wq[4] = {uq.x, uq.y, uq.z, uq.w}, wk[4] = {uk.x, uk.y, uk.z, uk.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          qv[i * 8 + 2 * e] = bf16_bits_to_f32(wq[e] & 0xFFFFu);
          qv[i * 8 + 2 * e + 1] = bf16_bits_to_f32(wq[e] >> 16);
          kv[i * 8 + 2 * e] = bf16_bits_to_f32(wk[e] & 0xFFFFu);
          kv[i * 8 + 2 * e + 1] = bf16_bits_to_f32(wk[e] >> 16);
        }
      }
#pragma unroll
      for (int i = 0; i < QC; ++i) {
        qs = fmaf(qv[i], qv[i], qs);
        ks = fmaf(kv[i], kv[i], ks);
      }
      qs += __shfl_xor_sync(0xffffffffu, qs, 1);
      ks += __shfl_xor_sync(0xffffffffu, ks, 1);
      qs += __shfl_xor_sync(0xffffffffu, qs, 2);
      ks += __shfl_xor_sync(0xffffffffu, ks, 2);
      nq = a.l2norm ? 1.0f / sqrtf(qs + 1e-6f) : 1.0f;
      nk = a.l2norm ? 1.0f / sqrtf(ks + 1e-6f) : 1.0f;
    }
    // gates: warp 0, two tokens per lane, one inclusive scan of pair sums
    if (warp == 0) {
      const float la0 = sm.lar[2 * lane], la1 = sm.lar[2 * lane + 1];
      const float pair = la0 + la1;
      float x = pair;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const float y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
      }
      const float ex = x - pair;                       // G before token 2*lane
      const float G0 = ex + la0, G1 = x;
      const float GC = __shfl_sync(0xffffffffu, x, 31);
      const float b0 = sm.ber[2 * lane], b1 = sm.ber[2 * lane + 1];
      const float Gs[2] = {G0, G1}, Gm[2] = {ex, G0}, bs[2] = {b0, b1};
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int t = 2 * lane + e;
        sm.g2[t] = Gs[e] * kLog2e;
        sm.g2m1[t] = Gm[e] * kLog2e;
        sm.be[t] = bs[e];
        sm.d1[t] = bs[e] * exp2f(Gm[e] * kLog2e);
        sm.eg[t] = exp2f(Gs[e] * kLog2e);
        sm.dk[t] = exp2f((GC - Gs[e]) * kLog2e);
      }
      if (lane == 31) sm.warp_tot = GC * kLog2e;
    }
    __syncthreads();
    const float g2C = sm.warp_tot;
    {
      const float dkr = sm.dk[pr] * nk;
      uint4* qd = reinterpret_cast<uint4*>(&sm.qh[pr * LDH + pq * QC]);
      uint4* kd = reinterpret_cast<uint4*>(&sm.kh[pr * LDH + pq * QC]);
      uint4* dd = reinterpret_cast<uint4*>(&sm.kd[pr * LDH + pq * QC]);
#pragma unroll
      for (int i = 0; i < QC / 8; ++i) {
        qd[i] = make_uint4(pack_h2(qv[8 * i] * nq, qv[8 * i + 1] * nq), pack_h2(qv[8 * i + 2] * nq, qv[8 * i + 3] * nq),
                           pack_h2(qv[8 * i + 4] * nq, qv[8 * i + 5] * nq), pack_h2(qv[8 * i + 6] * nq, qv[8 * i + 7] * nq));
        kd[i] = make_uint4(pack_h2(kv[8 * i] * nk, kv[8 * i + 1] * nk), pack_h2(kv[8 * i + 2] * nk, kv[8 * i + 3] * nk),
                           pack_h2(kv[8 * i + 4] * nk, kv[8 * i + 5] * nk), pack_h2(kv[8 * i + 6] * nk, kv[8 * i + 7] * nk));
        dd[i] = make_uint4(pack_h2(kv[8 * i] * dkr, kv[8 * i + 1] * dkr), pack_h2(kv[8 * i + 2] * dkr, kv[8 * i + 3] * dkr),
                           pack_h2(kv[8 * i + 4] * dkr, kv[8 * i + 5] * dkr), pack_h2(kv[8 * i + 6] * dkr, kv[8 * i + 7] * dkr));
      }
    }
    // beta o v as FP16, 8 columns per thread step
    for (int i = tid; i < C * DVS / 8; i += NT) {
      const int r = i / (DVS / 8), cc = (i % (DVS / 8)) * 8;
      const uint4 w = *reinterpret_cast<const uint4*>(&sm.vr[r * LDV + cc]);
      const float bt = sm.be[r];
      *reinterpret_cast<uint4*>(&sm.vh[r * LDV + cc]) =
          make_uint4(pack_h2(bf16_bits_to_f32(w.x & 0xFFFFu) * bt, bf16_bits_to_f32(w.x >> 16) * bt),
                     pack_h2(bf16_bits_to_f32(w.y & 0xFFFFu) * bt, bf16_bits_to_f32(w.y >> 16) * bt),
                     pack_h2(bf16_bits_to_f32(w.z & 0xFFFFu) * bt, bf16_bits_to_f32(w.z >> 16) * bt),
                     pack_h2(bf16_bits_to_f32(w.w & 0xFFFFu) * bt, bf16_bits_to_f32(w.w >> 16) * bt));
    }
    __syncthreads();
    // staging is free: prefetch the next chunk
    if (ch + 1 < nchunks)
      issue_chunk_loads<DK, DVS>(sm, a, tok0 + t0 + C, h, dv_off, (int)(T - t0 - C < C ? T - t0 - C : C), tid);

    // ---------------------------------------------------- P1: K K^T -> L
    // The ten lower-triangular 16x16 blocks (i, j <= i), one or two per warp.
#pragma unroll 1
    for (int task = warp; task < 10; task += 8) {
      const int bi = task < 1 ? 0 : task < 3 ? 1 : task < 6 ? 2 : 3;
      const int bj = task - bi * (bi + 1) / 2;
      float acc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
      float acc2[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll
      for (int kk = 0; kk < DK / 16; kk += 2) {   // two k-chains in flight
        uint32_t af[4], bf[4], af2[4], bf2[4];
        frag_a(af, sm.kh, LDH, 16 * bi, 16 * kk, lane);
        frag_b_nk(bf, sm.kh, LDH, 16 * kk, 16 * bj, lane);
        frag_a(af2, sm.kh, LDH, 16 * bi, 16 * kk + 16, lane);
        frag_b_nk(bf2, sm.kh, LDH, 16 * kk + 16, 16 * bj, lane);
        mma16816(acc[0], af, bf[0], bf[1]);
        mma16816(acc[1], af, bf[2], bf[3]);
        mma16816(acc2[0], af2, bf2[0], bf2[1]);
        mma16816(acc2[1], af2, bf2[2], bf2[3]);
      }
#pragma unroll
      for (int n = 0; n < 2; ++n)
#pragma unroll
        for (int e = 0; e < 4; ++e) acc[n][e] += acc2[n][e];
#pragma unroll
      for (int n = 0; n < 2; ++n)
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          const int t = 16 * bi + g + hh * 8;
          const int s0 = 16 * bj + 8 * n + 2 * c4;
          const float bt = sm.be[t], gm = sm.g2m1[t];
          const float v0 = (s0 < t) ? bt * exp2f(gm - sm.g2[s0]) * acc[n][2 * hh] : 0.f;
          const float v1 = (s0 + 1 < t) ? bt * exp2f(gm - sm.g2[s0 + 1]) * acc[n][2 * hh + 1] : 0.f;
          st_h2(&sm.lh[t * LDX + s0], v0, v1);
        }
    }
    __syncthreads();

    // ------------------------------- P2: X = (I+L)^-1 (warps 0-3) || Q K^T (warps 4-7)
    if (warp < 4) {
      if (lane < 16) {
        // diagonal block `warp`, column j = lane, forward substitution in FP32
        const int base = 16 * warp;
        const int j = lane;
        float lrow[16][16];
#pragma unroll
        for (int t = 1; t < 16; ++t)
#pragma unroll
          for (int s2 = 0; s2 < t; ++s2) lrow[t][s2] = __half2float(sm.lh[(base + t) * LDX + base + s2]);
        float x[16];
#pragma unroll
        for (int t = 0; t < 16; ++t) {
          float acc = (t == j) ? 1.0f : 0.0f;
#pragma unroll
          for (int s2 = 0; s2 < t; ++s2) acc -= lrow[t][s2] * x[s2];
          x[t] = (t < j) ? 0.0f : acc;
        }
#pragma unroll
        for (int t = 0; t < 16; ++t) sm.xh[(base + t) * LDX + base + j] = __float2half_rn(x[t]);
      }
      asm volatile("bar.sync 1, 128;" ::: "memory");
      // off-diagonal blocks, one level (distance) at a time; warp i owns block
      // row i and keeps P_ik = X_ii L_ik in registers.
      uint32_t P[3][4];
#pragma unroll 1
      for (int d = 1; d < 4; ++d) {
        if (warp >= d) {
          const int i = warp, jb = warp - d;
          {
            float p0[4] = {0.f, 0.f, 0.f, 0.f}, p1[4] = {0.f, 0.f, 0.f, 0.f};
            uint32_t af[4], bf[4];
            frag_a(af, sm.xh, LDX, 16 * i, 16 * i, lane);
            frag_b_kn(bf, sm.lh, LDX, 16 * i, 16 * (i - d), lane);
            mma16816(p0, af, bf[0], bf[1]);
            mma16816(p1, af, bf[2], bf[3]);
            c_to_a(P[d - 1], p0, p1);
          }
          float z0[4] = {0.f, 0.f, 0.f, 0.f}, z1[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
          for (int dd = 1; dd <= 3; ++dd) {
            if (dd <= d) {
              const int kb = i - dd;
              uint32_t bf[4];
              frag_b_kn(bf, sm.xh, LDX, 16 * kb, 16 * jb, lane);
              mma16816(z0, P[dd - 1], bf[0], bf[1]);
              mma16816(z1, P[dd - 1], bf[2], bf[3]);
            }
          }
          const int r0 = 16 * i + g;
          const int cc = 16 * jb + 2 * c4;
          st_h2(&sm.xh[r0 * LDX + cc], -z0[0], -z0[1]);
          st_h2(&sm.xh[(r0 + 8) * LDX + cc], -z0[2], -z0[3]);
          st_h2(&sm.xh[r0 * LDX + cc + 8], -z1[0], -z1[1]);
          st_h2(&sm.xh[(r0 + 8) * LDX + cc + 8], -z1[2], -z1[3]);
        }
        asm volatile("bar.sync 1, 128;" ::: "memory");
      }
    } else {
      // Gamma o Q K^T: the ten lower blocks over warps 4-7
#pragma unroll 1
      for (int task = warp - 4; task < 10; task += 4) {
        const int bi = task < 1 ? 0 : task < 3 ? 1 : task < 6 ? 2 : 3;
        const int bj = task - bi * (bi + 1) / 2;
        float acc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
        float acc2[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll
        for (int kk = 0; kk < DK / 16; kk += 2) {
          uint32_t af[4], bf[4], af2[4], bf2[4];
          frag_a(af, sm.qh, LDH, 16 * bi, 16 * kk, lane);
          frag_b_nk(bf, sm.kh, LDH, 16 * kk, 16 * bj, lane);
          frag_a(af2, sm.qh, LDH, 16 * bi, 16 * kk + 16, lane);
          frag_b_nk(bf2, sm.kh, LDH, 16 * kk + 16, 16 * bj, lane);
          mma16816(acc[0], af, bf[0], bf[1]);
          mma16816(acc[1], af, bf[2], bf[3]);
          mma16816(acc2[0], af2, bf2[0], bf2[1]);
          mma16816(acc2[1], af2, bf2[2], bf2[3]);
        }
#pragma unroll
        for (int n = 0; n < 2; ++n)
#pragma unroll
          for (int e = 0; e < 4; ++e) acc[n][e] += acc2[n][e];
#pragma unroll
        for (int n = 0; n < 2; ++n)
#pragma unroll
          for (int hh = 0; hh < 2; ++hh) {
            const int t = 16 * bi + g + hh * 8;
            const int s0 = 16 * bj + 8 * n + 2 * c4;
            const float gt = sm.g2[t];
            const float v0 = (s0 <= t) ? exp2f(gt - sm.g2[s0]) * acc[n][2 * hh] : 0.f;
            const float v1 = (s0 + 1 <= t) ? exp2f(gt - sm.g2[s0 + 1]) * acc[n][2 * hh + 1] : 0.f;
            st_h2(&sm.ah[t * LDX + s0], v0, v1);
          }
      }
    }
    __syncthreads();
    // X diag(d1): lower blocks only
    for (int i = tid; i < C * C / 2; i += NT) {
      const int r = i / (C / 2), cc = (i % (C / 2)) * 2;
      if ((cc >> 4) <= (r >> 4)) {
        const __half2 xv = *reinterpret_cast<const __half2*>(&sm.xh[r * LDX + cc]);
        const float2 xf = __half22float2(xv);
        st_h2(&sm.xw[r * LDX + cc], xf.x * sm.d1[cc], xf.y * sm.d1[cc + 1]);
      }
    }
    __syncthreads();

    // ---------------------------------------------------- P3: W, U~
    float U[NVH][4];
    {
      // -W = -(Xw K_hat): rows 16*mrow, d_k columns nhalf*DK/2 .. +DK/2-1
      float w[2 * KH][4];
#pragma unroll
      for (int j = 0; j < 2 * KH; ++j)
#pragma unroll
        for (int e = 0; e < 4; ++e) w[j][e] = 0.f;
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) {
        if (kk <= mrow) {
          uint32_t af[4];
          frag_a(af, sm.xw, LDX, 16 * mrow, 16 * kk, lane);
#pragma unroll
          for (int jj = 0; jj < KH; ++jj) {
            uint32_t bf[4];
            frag_b_kn(bf, sm.kh, LDH, 16 * kk, nhalf * (DK / 2) + 16 * jj, lane);
            mma16816(w[2 * jj], af, bf[0], bf[1]);
            mma16816(w[2 * jj + 1], af, bf[2], bf[3]);
          }
        }
      }
#pragma unroll
      for (int j = 0; j < 2 * KH; ++j) {
        const int r0 = 16 * mrow + g, cc = nhalf * (DK / 2) + 8 * j + 2 * c4;
        st_h2(&sm.wh[r0 * LDH + cc], -w[j][0], -w[j][1]);
        st_h2(&sm.wh[(r0 + 8) * LDH + cc], -w[j][2], -w[j][3]);
      }
      // U~ = X (beta o V): rows 16*mrow, slice n-tiles nhalf*NVH .. +NVH-1
#pragma unroll
      for (int j = 0; j < NVH; ++j)
#pragma unroll
        for (int e = 0; e < 4; ++e) U[j][e] = 0.f;
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) {
        if (kk <= mrow) {
          uint32_t af[4];
          frag_a(af, sm.xh, LDX, 16 * mrow, 16 * kk, lane);
#pragma unroll
          for (int j = 0; j < NVH; ++j) {
            uint32_t b0, b1;
            frag_b_kn1(b0, b1, sm.vh, LDV, 16 * kk, 8 * (nhalf * NVH + j), lane);
            mma16816(U[j], af, b0, b1);
          }
        }
      }
    }
    // S -> FP16 (rows 16*warp)
    if (s_owner) {
#pragma unroll
      for (int j = 0; j < NVT; ++j) {
        const int r0 = 16 * warp + g, cc = 8 * j + 2 * c4;
        st_h2(&sm.sh[r0 * LDV + cc], S[j][0], S[j][1]);
        st_h2(&sm.sh[(r0 + 8) * LDV + cc], S[j][2], S[j][3]);
      }
    }
    __syncthreads();

    // ---------------------------------------------------- P4: state part
    float OQ[NVH][4];
    {
#pragma unroll
      for (int j = 0; j < NVH; ++j)
#pragma unroll
        for (int e = 0; e < 4; ++e) OQ[j][e] = 0.f;
      constexpr int NP = (NVH % 2 != 0) ? 4 : 1;
      float Up[NP][NVH][4], OQp[NP][NVH][4];
#pragma unroll
      for (int q = 0; q < NP; ++q)
#pragma unroll
        for (int j = 0; j < NVH; ++j)
#pragma unroll
          for (int e = 0; e < 4; ++e) Up[q][j][e] = OQp[q][j][e] = 0.f;
#pragma unroll
      for (int kk = 0; kk < DK / 16; ++kk) {
        uint32_t aw[4], aq[4];
        frag_a(aw, sm.wh, LDH, 16 * mrow, 16 * kk, lane);
        frag_a(aq, sm.qh, LDH, 16 * mrow, 16 * kk, lane);
        if constexpr (NVH % 2 == 0) {
#pragma unroll
          for (int j = 0; j < NVH; j += 2) {
            uint32_t bf[4];
            frag_b_kn(bf, sm.sh, LDV, 16 * kk, 8 * (nhalf * NVH + j), lane);
            mma16816(U[j], aw, bf[0], bf[1]);
            mma16816(OQ[j], aq, bf[0], bf[1]);
            mma16816(U[j + 1], aw, bf[2], bf[3]);
            mma16816(OQ[j + 1], aq, bf[2], bf[3]);
          }
        } else {
          // one n-tile per warp: the k-loop is the only parallelism, so four
          // partial sums keep four MMA chains in flight
#pragma unroll
          for (int j = 0; j < NVH; ++j) {
            uint32_t b0, b1;
            frag_b_kn1(b0, b1, sm.sh, LDV, 16 * kk, 8 * (nhalf * NVH + j), lane);
            mma16816(Up[kk & 3][j], aw, b0, b1);
            mma16816(OQp[kk & 3][j], aq, b0, b1);
          }
        }
      }
      if constexpr (NVH % 2 != 0) {
#pragma unroll
        for (int j = 0; j < NVH; ++j)
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            U[j][e] += (Up[0][j][e] + Up[1][j][e]) + (Up[2][j][e] + Up[3][j][e]);
            OQ[j][e] = (OQp[0][j][e] + OQp[1][j][e]) + (OQp[2][j][e] + OQp[3][j][e]);
          }
      }
    }
    // U (the new values) -> FP16, replacing beta o v
#pragma unroll
    for (int j = 0; j < NVH; ++j) {
      const int r0 = 16 * mrow + g, cc = 8 * (nhalf * NVH + j) + 2 * c4;
      st_h2(&sm.vh[r0 * LDV + cc], U[j][0], U[j][1]);
      st_h2(&sm.vh[(r0 + 8) * LDV + cc], U[j][2], U[j][3]);
    }
    __syncthreads();
    {
      // O = e^{G_t} Q S + A U
      const float e0 = sm.eg[16 * mrow + g], e1 = sm.eg[16 * mrow + g + 8];
#pragma unroll
      for (int j = 0; j < NVH; ++j) {
        OQ[j][0] *= e0;
        OQ[j][1] *= e0;
        OQ[j][2] *= e1;
        OQ[j][3] *= e1;
      }
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) {
        if (kk <= mrow) {
          uint32_t af[4];
          frag_a(af, sm.ah, LDX, 16 * mrow, 16 * kk, lane);
          if constexpr (NVH % 2 == 0) {
#pragma unroll
            for (int j = 0; j < NVH; j += 2) {
              uint32_t bf[4];
              frag_b_kn(bf, sm.vh, LDV, 16 * kk, 8 * (nhalf * NVH + j), lane);
              mma16816(OQ[j], af, bf[0], bf[1]);
              mma16816(OQ[j + 1], af, bf[2], bf[3]);
            }
          } else {
#pragma unroll
            for (int j = 0; j < NVH; ++j) {
              uint32_t b0, b1;
              frag_b_kn1(b0, b1, sm.vh, LDV, 16 * kk, 8 * (nhalf * NVH + j), lane);
              mma16816(OQ[j], af, b0, b1);
            }
          }
        }
      }
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        const int t = 16 * mrow + g + hh * 8;
        if (t < valid) {
          const int64_t orow = ((tok0 + t0 + t) * a.H + h) * (int64_t)a.dv + dv_off;
#pragma unroll
          for (int j = 0; j < NVH; ++j) {
            const int cc = 8 * (nhalf * NVH + j) + 2 * c4;
            if (O_F32) {
              *reinterpret_cast<float2*>(reinterpret_cast<float*>(a.o) + orow + cc) =
                  make_float2(OQ[j][2 * hh], OQ[j][2 * hh + 1]);
              amax_bits = max(amax_bits, max(__float_as_uint(OQ[j][2 * hh]) & 0x7FFFFFFFu,
                                             __float_as_uint(OQ[j][2 * hh + 1]) & 0x7FFFFFFFu));
            } else {
              const uint32_t b0 = f32_to_bf16_bits(OQ[j][2 * hh]), b1 = f32_to_bf16_bits(OQ[j][2 * hh + 1]);
              *reinterpret_cast<uint32_t*>(reinterpret_cast<uint16_t*>(a.o) + orow + cc) = b0 | (b1 << 16);
              amax_bits = max(amax_bits, max(b0 & 0x7FFFu, b1 & 0x7FFFu) << 16);
            }
          }
        }
      }
    }
    if (s_owner) {
      // S' = e^{G_C} S + Kd^T U   (rows 16*warp of d_k)
      const float eC = exp2f(g2C);
#pragma unroll
      for (int j = 0; j < NVT; ++j)
#pragma unroll
        for (int e = 0; e < 4; ++e) S[j][e] *= eC;
      if constexpr (NVT <= 4) {
        // few n-tiles: two k-chains in flight, summed into S at the end
        float S2[NVT][4];
#pragma unroll
        for (int j = 0; j < NVT; ++j)
#pragma unroll
          for (int e = 0; e < 4; ++e) S2[j][e] = 0.f;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          uint32_t af[4];
          frag_a_t(af, sm.kd, LDH, 16 * warp, 16 * kk, lane);
#pragma unroll
          for (int j = 0; j < NVT; j += 2) {
            uint32_t bf[4];
            frag_b_kn(bf, sm.vh, LDV, 16 * kk, 8 * j, lane);
            if (kk & 1) {
              mma16816(S2[j], af, bf[0], bf[1]);
              mma16816(S2[j + 1], af, bf[2], bf[3]);
            } else {
              mma16816(S[j], af, bf[0], bf[1]);
              mma16816(S[j + 1], af, bf[2], bf[3]);
            }
          }
        }
#pragma unroll
        for (int j = 0; j < NVT; ++j)
#pragma unroll
          for (int e = 0; e < 4; ++e) S[j][e] += S2[j][e];
      } else {
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          uint32_t af[4];
          frag_a_t(af, sm.kd, LDH, 16 * warp, 16 * kk, lane);
#pragma unroll
          for (int j = 0; j < NVT; j += 2) {
            uint32_t bf[4];
            frag_b_kn(bf, sm.vh, LDV, 16 * kk, 8 * j, lane);
            mma16816(S[j], af, bf[0], bf[1]);
            mma16816(S[j + 1], af, bf[2], bf[3]);
          }
        }
      }
    }
    __syncthreads();
  }

  // An FP16 operand that overflowed (|x| >= 65520 rounds to infinity) reaches
  // o or the FP32 state as inf or NaN: report it instead of returning it silently.
  {
    bool bad = amax_bits >= 0x7F800000u;
    if (s_owner) {
#pragma unroll
      for (int j = 0; j < NVT; ++j)
#pragma unroll
        for (int e = 0; e < 4; ++e) bad |= !isfinite(S[j][e]);
    }
    if (bad) report_status(a.status, GDN_ERR_RANGE);
  }
  if (a.o_amax) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) amax_bits = max(amax_bits, __shfl_xor_sync(0xffffffffu, amax_bits, o));
    if (lane == 0 && amax_bits) atomicMax(a.o_amax, amax_bits);
  }
  if (a.S_T && s_owner) {
#pragma unroll
    for (int j = 0; j < NVT; ++j)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int r = 16 * warp + g + (e >> 1) * 8, col = 8 * j + 2 * c4 + (e & 1);
        a.S_T[((int64_t)chain * DK + r) * a.dv + dv_off + col] = S[j][e];
      }
  }
}

template <int DK, int DVS, bool O_F32>
int launch_dvs(const Args& a, int64_t chains, cudaStream_t stream) {
  const size_t smem = sizeof(Smem<DK, DVS>);
  cudaError_t e =
      cudaFuncSetAttribute(delta_rule_kernel<DK, DVS, O_F32>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return record_cuda_error(e);
  delta_rule_kernel<DK, DVS, O_F32><<<(unsigned)(chains * a.nsplit), NT, smem, stream>>>(a);
  return check_launch();
}

template <int DK, bool O_F32>
int launch_dk(const Args& a, int dvs, int64_t chains, cudaStream_t stream) {
  switch (dvs) {
    case 16: return launch_dvs<DK, 16, O_F32>(a, chains, stream);
    case 32: return launch_dvs<DK, 32, O_F32>(a, chains, stream);
    case 64: return launch_dvs<DK, 64, O_F32>(a, chains, stream);
    default: return launch_dvs<DK, 128, O_F32>(a, chains, stream);
  }
}

}  // namespace

int launch_delta_rule(const uint16_t* q, const uint16_t* k, const uint16_t* v, int64_t ld_q, int64_t ld_k,
                      int64_t ld_v, const float* log_alpha, const float* beta, const float* S0, int64_t B,
                      int64_t T, int H, int dk, int dv, int flags, void* o, float* S_T, unsigned* o_amax,
                      cudaStream_t stream, const OQuant* oq, void* ws, size_t ws_bytes) {
  const int64_t chains = B * H;
  if (chains == 0) return GDN_OK;
  if (oq && (flags & GDN_DR_O_FP32)) return GDN_ERR_UNSUPPORTED_SHAPE;   // o is quantized from its bf16 values
  // the tensor-core kernel stores o and S_T in 16-byte vectors
  if (!(flags & GDN_DR_MMA_SYNC) && delta_rule_tc_supported(dk, dv, T) && aligned(o, 16) && (!S_T || aligned(S_T, 16)))
    return launch_delta_rule_tc(q, k, v, ld_q, ld_k, ld_v, log_alpha, beta, S0, B, T, H, dk, dv, flags, o, S_T,
                                o_amax, stream, oq, ws, ws_bytes);
  if (oq) {
    int st = launch_delta_rule(q, k, v, ld_q, ld_k, ld_v, log_alpha, beta, S0, B, T, H, dk, dv, flags, o, S_T, o_amax,
                               stream, nullptr);
    if (st) return st;
    const int64_t HV = (int64_t)H * dv;
    return launch_quantize(o, GDN_DTYPE_BF16, B * T, HV, HV, GDN_QUANT_GIVEN_SCALE, oq->g_enc, oq->codes, oq->scales,
                           1, 0, oq->g_out, nullptr, stream);
  }
  // Split d_v so that the CTAs cover the SMs (one CTA per SM).
  const int sms = num_sms();
  int dvs = dv;
  while (dvs > 16 && chains * (dv / dvs) * 2 <= sms) dvs /= 2;
  Args a{};
  a.q = q;
  a.k = k;
  a.v = v;
  a.ld_q = ld_q;
  a.ld_k = ld_k;
  a.ld_v = ld_v;
  a.log_alpha = log_alpha;
  a.beta = beta;
  a.S0 = S0;
  a.T = T;
  a.H = H;
  a.dv = dv;
  a.nsplit = dv / dvs;
  a.l2norm = (flags & GDN_DR_L2NORM_QK) ? 1 : 0;
  a.o = o;
  a.S_T = S_T;
  a.o_amax = o_amax;
  a.status = device_status_word();
  const bool f32 = (flags & GDN_DR_O_FP32) != 0;
  switch (dk) {
    case 32: return f32 ? launch_dk<32, true>(a, dvs, chains, stream) : launch_dk<32, false>(a, dvs, chains, stream);
    case 64: return f32 ? launch_dk<64, true>(a, dvs, chains, stream) : launch_dk<64, false>(a, dvs, chains, stream);
    default:
      return f32 ? launch_dk<128, true>(a, dvs, chains, stream) : launch_dk<128, false>(a, dvs, chains, stream);
  }
}

}  // namespace gdn
