// Chunked gated delta rule forward on the 5th-generation tensor cores
// (sm_100a), for d_k = 128 and d_v slices of 64 or 128 columns.
//
// Recurrence ("Anthology of the SOTA, theory-128", section "The account"):
//   S_t = alpha_t S_{t-1} + beta_t k_t (v_t - S_{t-1}^T k_t)^T,   o_t = S_t^T q_t
// over L2-normalised q, k, in the chunk form (C = 64 tokens, entered with
// state S, G_t = sum_{s<=t} log alpha_s inside the chunk, G_{-1} = 0):
//   L_ts = beta_t e^{G_{t-1}-G_s} k_t.k_s (s < t),   X = (I + L)^{-1}
//   W    = X diag(beta_s e^{G_{s-1}}) K,   U~ = X diag(beta) V,   U = U~ - W S
//   O    = diag(e^{G_t}) Q S + A U,        A_ts = e^{G_t-G_s} q_t.k_s (s <= t)
//   S'   = e^{G_C} S + K^T diag(e^{G_C-G_s}) U
// Every exponent is <= 0, so nothing overflows whatever the decay.
//
// One CTA (8 warps) walks one (batch, head, d_v slice) chain.  Every product
// of the chunk runs as tcgen05.mma.kind::f16 (FP16 operands from shared
// memory in 128-byte swizzled layouts, FP32 accumulators in TMEM), stacked so
// that each MMA has M = 128:
//   MMA-a  [K; Q] K^T           -> K K^T (rows 0..63) and Q K^T (64..127)
//   MMA-b  [Xw; X] K, [Xw; X] V -> W (rows 0..63 of the first), U~ (rows
//                                  64..127 of the second; V already beta-scaled)
//   MMA-1  [Q; W] S_h           -> Q S (rows 0..63) and W S (64..127)
//   MMA-2  [A; *] U             -> A U (rows 0..63; the other rows unused)
//   MMA-3  S += K^T U'          (U' = diag(e^{G_C-G_s}) U; S lives in TMEM)
// The state stays FP32 in TMEM for the whole sequence; its FP16 copy S_h is
// the B operand of MMA-1.  The 64 x 64 unit-lower-triangular inverse runs on
// mma.sync in warps 0-3 (diagonal blocks by right-looking substitution, then
// the off-diagonal blocks level by level) while warps 4-7 turn the state into
// S_h and apply the chunk's decay to it.
//
// Pipeline: the chunk inputs are double-buffered.  Chunk ch+1's q and k land
// by TMA (3-D tensor maps, so rows past the end of a sequence read as zeros)
// directly in the [K; Q] rows of the other buffer, and its v in the other
// beta-V tile; while the tensor cores run chunk ch's MMA-b, MMA-1 and MMA-2/3,
// the CTA normalises those q and k rows in place, scales v by beta and scans
// the gates.  The state update of chunk ch is waited for only at the top of
// chunk ch+1.  o leaves by TMA stores through shared memory.
//
// TMEM (512 columns): RA = K K^T | Q K^T, later A U;  RB = [Xw; X] K, later
// [Q; W] S_h;  R2 = [Xw; X] V;  RS = the state.
// Every wait is bounded: a wait that runs out records GDN_ERR_TIMEOUT and the
// CTA leaves the chunk loop.
#include <cuda_fp16.h>

#include <cstring>

#include "common.cuh"
#include "quant_math.cuh"
#include "kernels.h"
#include "tmap.cuh"

namespace gdn {
namespace {

constexpr int C = 64;
constexpr int DK = 128;
constexpr int NT = 256;
constexpr float kLog2e = 1.4426950408889634f;

// Shared-memory map (byte offsets from a 1024-aligned base).  The chunk
// inputs are double-buffered (buffer ch & 1): chunk ch+1's q, k, v land by TMA
// and are normalised / beta-scaled in place while chunk ch computes.
template <int DVS>
struct Map {
  static constexpr uint32_t T3_ATOM = 192 * 128;             // one 64-column atom of [K; Q; W]
  static constexpr uint32_t T3_BYTES = 2 * T3_ATOM;
  static constexpr uint32_t T3 = 0;                          // 2 x [K; Q; W]: 192 rows x 128 fp16, K-major
  static constexpr uint32_t P = T3 + 2 * T3_BYTES;           // [A; Xw; X]: 192 rows x 64 fp16 (L in X's place)
  static constexpr uint32_t VB_BYTES = 64 * 2 * DVS;
  static constexpr uint32_t VB = P + 192 * 128;              // 2 x (v, beta v, then U): 64 tokens x DVS, N-major
  static constexpr uint32_t UP = VB + 2 * VB_BYTES;          // U' = diag(e^{G_C-G_s}) U
  static constexpr uint32_t SH = UP + VB_BYTES;              // S_h: 128 (d_k) x DVS, N-major
  static constexpr uint32_t OS = SH + 128 * 2 * DVS;         // o staging: 32 x 64 bf16 boxes, 4 KiB each
  static constexpr uint32_t LD32 = OS + (DVS / 64) * 2 * 4096;   // FP32 diagonal 16 x 16 blocks of L
  static constexpr uint32_t F = LD32 + 4 * 16 * 16 * 4;      // 2 x per-token factors
  static constexpr uint32_t F_BYTES = 6 * C * 4 + 16;
  static constexpr uint32_t G2 = 0, G2M1 = C * 4, BE = 2 * C * 4, D1 = 3 * C * 4, EG = 4 * C * 4, DKF = 5 * C * 4,
                            GC2 = 6 * C * 4;                 // offsets inside one factor block
  static constexpr uint32_t MISC = F + 2 * F_BYTES;          // mbarriers, tmem ptr, flags
  static constexpr uint32_t LD_BYTES = 4 * 64 * 128 + 64 * 2 * DVS;   // one chunk's TMA bytes
  static constexpr uint32_t BYTES = MISC + 64;
};
static_assert(Map<128>::P % 1024 == 0 && Map<128>::VB % 1024 == 0 && Map<128>::UP % 1024 == 0 &&
                  Map<128>::SH % 1024 == 0 && Map<128>::OS % 1024 == 0 && Map<64>::OS % 1024 == 0,
              "swizzled tiles need 1024-byte alignment");
static_assert(Map<128>::BYTES + 1024 <= 232448, "shared memory budget");

constexpr uint32_t RA = 0, RB = 128, R2 = 256, RS = 384;

// Byte offset of element (r, c), c < 64, in a 128-byte-swizzled fp16 atom
// whose rows are 128 bytes: the 16-byte chunk index is XORed with r mod 8
// (the TMA / tensor-core 128B swizzle on a 1024-aligned atom).
__device__ __forceinline__ uint32_t swz(int r, int c) {
  return (uint32_t)(r * 128 + ((((c >> 3) ^ r) & 7) << 4) + (c & 7) * 2);
}

// Shared-memory matrix descriptor, 128-byte swizzle.  K-major operands use
// only SBO (1024: eight 128-byte rows); N/M-major ones use LBO as the stride
// between 64-element atoms along N/M and SBO between 8-row groups along K.
__device__ __forceinline__ uint64_t sdesc(uint32_t saddr, uint32_t lbo) {
  uint64_t d = (uint64_t)((saddr >> 4) & 0x3FFFu);
  d |= (uint64_t)((lbo >> 4) & 0x3FFFu) << 16;
  d |= (uint64_t)(1024 >> 4) << 32;
  d |= (uint64_t)1 << 46;
  d |= (uint64_t)2 << 61;
  return d;
}
// Instruction descriptor of kind::f16: FP16 A and B, FP32 accumulator.
__host__ __device__ constexpr uint32_t idesc_f16(int M, int N, int a_mn_major, int b_mn_major) {
  return (1u << 4) | ((uint32_t)a_mn_major << 15) | ((uint32_t)b_mn_major << 16) | ((uint32_t)(N >> 3) << 17) |
         ((uint32_t)(M >> 4) << 24);
}
// Warp-collective issue: every lane of the warp executes this with the same
// (warp-uniform) operands and one elected lane issues the MMA, so the
// descriptors stay in uniform registers instead of being moved there per
// instruction from one diverged thread.
__device__ __forceinline__ void mma_f16_warp(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                             uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p, e;\n\t"
      "elect.sync _|e, 0xffffffff;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}
__device__ __forceinline__ void fence_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

// 2^x on the SFU (ex2.approx, relative error ~2^-22); every argument here is
// <= 0, and results below 2^-126 flush to zero.
__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ void tma_load_3d(uint32_t dst, const void* tmap, uint32_t bar, int32_t c0, int32_t c1,
                                            int32_t c2) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4, %5}], [%2];" ::
          "r"(dst),
      "l"(tmap), "r"(bar), "r"(c0), "r"(c1), "r"(c2)
      : "memory");
}
__device__ __forceinline__ void tma_store_3d(const void* tmap, uint32_t src, int32_t c0, int32_t c1, int32_t c2) {
  asm volatile("cp.async.bulk.tensor.3d.global.shared::cta.bulk_group [%0, {%2, %3, %4}], [%1];" ::"l"(tmap), "r"(src),
               "r"(c0), "r"(c1), "r"(c2)
               : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_read0() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait0() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

__device__ __forceinline__ void mma16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
__device__ __forceinline__ void ldsm4(uint32_t (&r)[4], uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}
__device__ __forceinline__ void ldsm4t(uint32_t (&r)[4], uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}
// A fragment (16 x 16) at (m0, k0) of a swizzled 64-column tile.
__device__ __forceinline__ void frag_a(uint32_t (&a)[4], uint32_t base, int m0, int k0, int lane) {
  const int i = lane >> 3;
  ldsm4(a, base + swz(m0 + (lane & 7) + (i & 1) * 8, k0 + (i >> 1) * 8));
}
// B fragments of two adjacent n-tiles for B[k][n] stored row-major [k][n].
__device__ __forceinline__ void frag_b_kn(uint32_t (&b)[4], uint32_t base, int k0, int n0, int lane) {
  const int i = lane >> 3;
  ldsm4t(b, base + swz(k0 + (lane & 7) + (i & 1) * 8, n0 + (i >> 1) * 8));
}
__device__ __forceinline__ uint32_t pack_h2(float lo, float hi) {
  __half2 h = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}
__device__ __forceinline__ void c_to_a(uint32_t (&a)[4], const float (&c0)[4], const float (&c1)[4]) {
  a[0] = pack_h2(c0[0], c0[1]);
  a[1] = pack_h2(c0[2], c0[3]);
  a[2] = pack_h2(c1[0], c1[1]);
  a[3] = pack_h2(c1[2], c1[3]);
}
__device__ __forceinline__ void st_s32(uint32_t addr, uint32_t v) {
  asm volatile("st.shared.b32 [%0], %1;" ::"r"(addr), "r"(v) : "memory");
}
__device__ __forceinline__ void st_s128(uint32_t addr, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
  asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c), "r"(d) : "memory");
}
__device__ __forceinline__ uint4 ld_s128(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "r"(addr));
  return v;
}
// Eight consecutive FP32 values -> one 16-byte chunk of FP16.
__device__ __forceinline__ void st_chunk_h(uint32_t addr, const float* v) {
  st_s128(addr, pack_h2(v[0], v[1]), pack_h2(v[2], v[3]), pack_h2(v[4], v[5]), pack_h2(v[6], v[7]));
}
// One 16-byte chunk of bf16 -> eight FP32 values.
__device__ __forceinline__ void unpack_bf16x8(const uint4& u, float* f) {
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    f[2 * e] = bf16_bits_to_f32(w[e] & 0xFFFFu);
    f[2 * e + 1] = bf16_bits_to_f32(w[e] >> 16);
  }
}


struct Args {
  const float* log_alpha;
  const float* beta;
  const float* S0;
  int64_t T;
  int H, dv, nsplit;
  int l2norm;
  void* o;
  float* S_T;
  unsigned* o_amax;
  int* status;
  // fused NVFP4 quantization of the bf16 o (codes == nullptr: off)
  uint8_t* oq_codes;
  uint8_t* oq_scales;
  const float* oq_g_enc;
  float* oq_g_out;
};
struct Maps {
  CUtensorMap q, k, v, o;   // 3-D: (feature, token, batch); o only for bf16 output
};

// The chunk's q (rows 64..127) and k (rows 0..63) straight into buffer p of
// [K; Q; W] and its v into buffer p of VB, by TMA from one thread; rows past
// the end of the sequence arrive as zeros.
template <int DVS>
__device__ __forceinline__ void issue_chunk_loads(uint32_t sb, const Maps& m, const Args& a, int b, int h,
                                                  int dv_off, int64_t t0, int p) {
  using M = Map<DVS>;
  const uint32_t bar = sb + M::MISC + 8;
  mbar_arrive_expect_tx(reinterpret_cast<uint64_t*>(__cvta_shared_to_generic(bar)), M::LD_BYTES);
  const uint32_t t3 = sb + M::T3 + (uint32_t)p * M::T3_BYTES;
#pragma unroll
  for (int at = 0; at < 2; ++at) {
    tma_load_3d(t3 + at * M::T3_ATOM, &m.k, bar, h * DK + 64 * at, (int32_t)t0, b);
    tma_load_3d(t3 + at * M::T3_ATOM + 64 * 128, &m.q, bar, h * DK + 64 * at, (int32_t)t0, b);
  }
  const uint32_t vb = sb + M::VB + (uint32_t)p * M::VB_BYTES;
#pragma unroll
  for (int at = 0; at < DVS / 64; ++at)
    tma_load_3d(vb + at * 8192, &m.v, bar, h * a.dv + dv_off + 64 * at, (int32_t)t0, b);
}

// In place: bf16 rows of [K; Q] buffer p -> L2-normalised FP16 (rows r0 ..
// r0+63; four threads per row, 32 columns each).
template <int DVS>
__device__ __forceinline__ void normalize_rows(uint32_t t3, int r0, int tid, int l2norm) {
  using M = Map<DVS>;
  constexpr int QC = DK / 4;
  const int pr = tid >> 2, pq = tid & 3;
  float v[QC];
  uint32_t off[QC / 8];
#pragma unroll
  for (int i = 0; i < QC / 8; ++i) {
    const int col = pq * QC + 8 * i;
    off[i] = t3 + (uint32_t)(col >> 6) * M::T3_ATOM + swz(r0 + pr, col & 63);
    unpack_bf16x8(ld_s128(off[i]), &v[8 * i]);
  }
  float s0 = 0.f, s1 = 0.f;
#pragma unroll
  for (int i = 0; i < QC; i += 2) {
    s0 = fmaf(v[i], v[i], s0);
    s1 = fmaf(v[i + 1], v[i + 1], s1);
  }
  float ss = s0 + s1;
  ss += __shfl_xor_sync(0xffffffffu, ss, 1);
  ss += __shfl_xor_sync(0xffffffffu, ss, 2);
  const float n = l2norm ? rsqrtf(ss + 1e-6f) : 1.0f;
#pragma unroll
  for (int i = 0; i < QC; ++i) v[i] *= n;
#pragma unroll
  for (int i = 0; i < QC / 8; ++i) st_chunk_h(off[i], &v[8 * i]);
}

// Every thread waits (bounded) for the phase of `bar` with the given parity,
// then the CTA synchronises; returns false on every thread when the wait ran
// out.  (Every thread polling measured ~1% faster on the layer shape than
// thread 0 polling while the others sit in the barrier.)
__device__ __forceinline__ bool cta_wait(uint64_t* bar, uint32_t parity, volatile int* abort_flag, int* status) {
  if (!mbar_wait(bar, parity, status)) *abort_flag = 1;
  __syncthreads();
  tc_fence_after();
  return *abort_flag == 0;
}

// The raw gates of chunk t0 (warp 7: two tokens per lane; zero past the end
// of the sequence), fetched well before they are needed.
__device__ __forceinline__ void fetch_gates(const Args& a, int64_t tok0, int h, int64_t t0, int lane, float (&la)[2],
                                            float (&bs)[2]) {
#pragma unroll
  for (int e = 0; e < 2; ++e) {
    const int64_t t = t0 + 2 * lane + e;
    const bool ok = t < a.T;
    la[e] = ok ? __ldg(a.log_alpha + (tok0 + t) * a.H + h) : 0.0f;
    bs[e] = ok ? __ldg(a.beta + (tok0 + t) * a.H + h) : 0.0f;
  }
}

// Warp 7: the chunk's gate factors into factor block f from the fetched raw
// gates (an inclusive scan of log alpha, two tokens per lane).
template <int DVS>
__device__ __forceinline__ void scan_gates(float* f, const float (&la)[2], const float (&bs)[2], int lane) {
  using M = Map<DVS>;
  const float pair = la[0] + la[1];
  float x = pair;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const float y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  const float ex = x - pair;
  const float G0 = ex + la[0], G1 = x;
  const float GC = __shfl_sync(0xffffffffu, x, 31);
  const float Gs[2] = {G0, G1}, Gm[2] = {ex, G0};
#pragma unroll
  for (int e = 0; e < 2; ++e) {
    const int t = 2 * lane + e;
    f[M::G2 / 4 + t] = Gs[e] * kLog2e;
    f[M::G2M1 / 4 + t] = Gm[e] * kLog2e;
    f[M::D1 / 4 + t] = bs[e] * ex2(Gm[e] * kLog2e);
    f[M::EG / 4 + t] = ex2(Gs[e] * kLog2e);
    f[M::DKF / 4 + t] = ex2((GC - Gs[e]) * kLog2e);
  }
  if (lane == 31) f[M::GC2 / 4] = GC * kLog2e;
}

// beta o v in place in VB buffer vb, with beta from factor block f (the rows
// past the end of the sequence hold zeros and get beta 0).
template <int DVS>
__device__ __forceinline__ void scale_v(uint32_t vb, const float* f, int tid) {
  using M = Map<DVS>;
  for (int i = tid; i < C * DVS / 8; i += NT) {
    const uint32_t off = (uint32_t)i * 16;
    const int r = (i >> 3) & 63;             // token row of this 16-byte chunk
    const float bt = f[M::BE / 4 + r];
    float x[8];
    unpack_bf16x8(ld_s128(vb + off), x);
#pragma unroll
    for (int e = 0; e < 8; ++e) x[e] *= bt;
    st_chunk_h(vb + off, x);
  }
}

// MMA-a of the chunk in [K; Q; W] buffer t3: [K; Q] K^T into TMEM column d
// (64 columns: K K^T in lanes 0..63, Q K^T in lanes 64..127); one warp.
template <int DVS>
__device__ __forceinline__ void issue_mma_a(uint32_t tmem_d, uint32_t t3, uint64_t* bar) {
  using M = Map<DVS>;
  constexpr uint32_t id = idesc_f16(128, 64, 0, 0);
#pragma unroll
  for (int j = 0; j < DK / 16; ++j) {
    const uint64_t d = sdesc(t3 + (j >> 2) * M::T3_ATOM + (j & 3) * 32, 16);
    mma_f16_warp(tmem_d, d, d, id, j > 0 ? 1u : 0u);
  }
  tc_commit_warp(bar);
}

// Every thread waits (bounded) for a chunk's TMA loads; a wait that runs out
// raises the abort flag, which the CTA reads after its next barrier.
__device__ __forceinline__ void wait_loads(uint64_t* bar, uint32_t parity, volatile int* abort_flag, int* status) {
  if (!mbar_wait(bar, parity, status)) *abort_flag = 1;
}

template <int DVS, bool O_F32>
__global__ void __launch_bounds__(NT, 1)
    delta_rule_tc_kernel(const __grid_constant__ Args a, const __grid_constant__ Maps maps) {
  using M = Map<DVS>;
  constexpr int HALF = DVS / 2;          // columns of the d_v slice per warp of a TMEM quarter
  extern __shared__ uint8_t smem_raw[];
  // 1024-aligned base in the shared window (every tile address below is a
  // 32-bit shared-space address)
  const uint32_t sraw = smem_u32(smem_raw);
  const uint32_t sb = (sraw + 1023u) & ~1023u;
  uint8_t* smem = smem_raw + (sb - sraw);
  uint64_t* bar_mma = reinterpret_cast<uint64_t*>(smem + M::MISC);
  uint64_t* bar_ld = reinterpret_cast<uint64_t*>(smem + M::MISC + 8);
  uint64_t* bar_3 = reinterpret_cast<uint64_t*>(smem + M::MISC + 16);   // MMA-3 (state update) done
  uint32_t* tmem_ptr = reinterpret_cast<uint32_t*>(smem + M::MISC + 24);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + M::MISC + 28);
  uint64_t* bar_a = reinterpret_cast<uint64_t*>(smem + M::MISC + 32);   // MMA-a (K K^T, Q K^T) done
  uint64_t* bar_b2 = reinterpret_cast<uint64_t*>(smem + M::MISC + 40);  // MMA-b2 (U~) done

  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  const int quarter = warp & 3, colhalf = warp >> 2;

  const int chain = blockIdx.x / a.nsplit;
  const int split = blockIdx.x % a.nsplit;
  const int b = chain / a.H, h = chain % a.H;
  const int dv_off = split * DVS;
  const int64_t T = a.T;
  const int64_t tok0 = (int64_t)b * T;

  if (tid == 0) {
    mbar_init(bar_mma, 1);
    mbar_init(bar_ld, 1);
    mbar_init(bar_3, 1);
    mbar_init(bar_a, 1);
    mbar_init(bar_b2, 1);
    *abort_flag = 0;
    fence_mbar_init();
    prefetch_tmap(&maps.q);
    prefetch_tmap(&maps.k);
    prefetch_tmap(&maps.v);
    if (!O_F32) prefetch_tmap(&maps.o);
  }
  if (warp == 0) {
    tmem_alloc(tmem_ptr, 512);
    tmem_relinquish();
  }
  // [A; Xw; X] starts zero: the strictly upper blocks of Xw are never written
  // afterwards (those of X are rewritten with zeros every chunk).
  for (int i = tid; i < 192 * 128 / 16; i += NT) st_s128(sb + M::P + i * 16, 0u, 0u, 0u, 0u);
  fence_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_ptr;
  const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;

  // S (FP32, TMEM RS): lane r = d_k row, column n = d_v column of the slice.
  {
    const int r = quarter * 32 + lane;
#pragma unroll
    for (int c0 = 0; c0 < HALF; c0 += 16) {
      uint32_t v[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const int col = colhalf * HALF + c0 + i;
        v[i] = __float_as_uint(a.S0 ? a.S0[((int64_t)chain * DK + r) * a.dv + dv_off + col] : 0.0f);
      }
      tmem_st_32x32b_x16(tmem + lane_off + RS + colhalf * HALF + c0, v);
    }
    tc_wait_st();
  }

  // o: warps of quarters 0 and 1 write 64 columns each (the second column
  // half only when the slice has 128 columns)
  const bool o_worker = quarter < 2 && (DVS == 128 || colhalf == 0);
  const int o_col0 = (DVS == 128) ? colhalf * 64 : 0;
  const uint32_t o_stage = sb + M::OS + (uint32_t)((DVS == 128 ? colhalf * 2 : 0) + quarter) * 4096;

  uint32_t amax_bits = 0;
  uint32_t mma_phase = 0;
  const float oq_genc = a.oq_codes ? *a.oq_g_enc : 1.0f;
  if (a.oq_codes && blockIdx.x == 0 && tid == 0) *a.oq_g_out = __fdiv_rn(1.0f, oq_genc);
  const int64_t nchunks = (T + C - 1) / C;

  // chunk loads issued and waited for (uniform across the CTA); chunk i's
  // load completes phase i of bar_ld
  int64_t lds_issued = 0, lds_waited = 0;
  // chunk 0's inputs, prepared before the loop
  if (nchunks > 0) {
    if (tid == 64) issue_chunk_loads<DVS>(sb, maps, a, b, h, dv_off, 0, 0);
    lds_issued = 1;
    wait_loads(bar_ld, 0, abort_flag, a.status);
    lds_waited = 1;
    normalize_rows<DVS>(sb + M::T3, 0, tid, a.l2norm);
    normalize_rows<DVS>(sb + M::T3, 64, tid, a.l2norm);
    float* f0 = reinterpret_cast<float*>(smem + M::F);
    if (warp == 7) {
      float la[2], bs[2];
      fetch_gates(a, tok0, h, 0, lane, la, bs);
      f0[M::BE / 4 + 2 * lane] = bs[0];
      f0[M::BE / 4 + 2 * lane + 1] = bs[1];
      scan_gates<DVS>(f0, la, bs, lane);
    }
    fence_async_smem();      // the normalised rows, for MMA-a
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
      tc_fence_after();
      issue_mma_a<DVS>(tmem + R2, sb + M::T3, bar_a);
    }
    scale_v<DVS>(sb + M::VB, f0, tid);
    fence_async_smem();
  }
  float nla[2] = {0.f, 0.f}, nbs[2] = {0.f, 0.f};   // warp 7: the next chunk's raw gates
  tc_fence_before();

#pragma unroll 1
  for (int64_t ch = 0; ch < nchunks; ++ch) {
    const int64_t t0 = ch * C;
    const int valid = (int)(T - t0 < C ? T - t0 : C);
    const int p = (int)(ch & 1), pn = p ^ 1;
    const bool has_next = ch + 1 < nchunks;
    const uint32_t t3 = sb + M::T3 + (uint32_t)p * M::T3_BYTES;
    const uint32_t t3n = sb + M::T3 + (uint32_t)pn * M::T3_BYTES;
    const uint32_t vb = sb + M::VB + (uint32_t)p * M::VB_BYTES;
    const float* fb = reinterpret_cast<const float*>(smem + M::F + (uint32_t)p * M::F_BYTES);
    const float* g2 = fb + M::G2 / 4;
    const float* g2m1 = fb + M::G2M1 / 4;
    const float* be = fb + M::BE / 4;
    const float* d1 = fb + M::D1 / 4;
    const float* eg = fb + M::EG / 4;
    const float* dkf = fb + M::DKF / 4;

    // The previous chunk's state update (MMA-3) has finished: its operands in
    // buffer pn are free for the next chunk's loads and its state is final.
    if (ch > 0 && !mbar_wait(bar_3, (uint32_t)(ch - 1) & 1, a.status)) *abort_flag = 1;
    __syncthreads();
    tc_fence_after();
    if (*abort_flag) break;
    // MMA-a: chunk 0's was issued in the prologue
    if (warp == 0 && ch > 0) issue_mma_a<DVS>(tmem + R2, t3, bar_a);
    if (has_next) {
      if (tid == 64) issue_chunk_loads<DVS>(sb, maps, a, b, h, dv_off, t0 + C, pn);
      if (warp == 7) fetch_gates(a, tok0, h, t0 + C, lane, nla, nbs);
      lds_issued = ch + 2;
    }
    float* fn = reinterpret_cast<float*>(smem + M::F + (uint32_t)pn * M::F_BYTES);

    if (!cta_wait(bar_a, (uint32_t)ch & 1, abort_flag, a.status)) break;

    // ------------------------------------------ P1: L and A from R2 (MMA-a)
    const uint32_t Xb = sb + M::P + 128 * 128;    // X, and L before it
    const uint32_t Xwb = sb + M::P + 64 * 128;
    {
      uint32_t r[32];
      tmem_ld_32x32b_x32(tmem + lane_off + R2 + colhalf * 32, r);
      tc_wait_ld();
      const int s0 = colhalf * 32;
      float v[32];
      if (quarter < 2) {
        const int t = quarter * 32 + lane;
        const float bt = be[t], gm = g2m1[t];
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const int s = s0 + i;
          v[i] = (s < t) ? bt * ex2(fminf(gm - g2[s], 0.0f)) * __uint_as_float(r[i]) : 0.0f;
        }
        // L (strictly lower; zeros elsewhere) in X's place
#pragma unroll
        for (int c = 0; c < 4; ++c) st_chunk_h(Xb + swz(t, s0 + 8 * c), &v[8 * c]);
        // row t of its diagonal block in FP32 for the substitution
        const int blk = t >> 4;
        if ((blk >> 1) == colhalf) {
          // the block's 16 columns are the first or second half of this
          // thread's 32
          const uint32_t dst = sb + M::LD32 + (uint32_t)(blk * 256 + (t & 15) * 16) * 4;
          if (blk & 1) {
#pragma unroll
            for (int c = 0; c < 4; ++c)
              st_s128(dst + c * 16, __float_as_uint(v[16 + 4 * c]), __float_as_uint(v[17 + 4 * c]),
                      __float_as_uint(v[18 + 4 * c]), __float_as_uint(v[19 + 4 * c]));
          } else {
#pragma unroll
            for (int c = 0; c < 4; ++c)
              st_s128(dst + c * 16, __float_as_uint(v[4 * c]), __float_as_uint(v[1 + 4 * c]),
                      __float_as_uint(v[2 + 4 * c]), __float_as_uint(v[3 + 4 * c]));
          }
        }
      } else {
        const int t = (quarter - 2) * 32 + lane;
        const float gt = g2[t];
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const int s = s0 + i;
          v[i] = (s <= t) ? ex2(fminf(gt - g2[s], 0.0f)) * __uint_as_float(r[i]) : 0.0f;
        }
#pragma unroll
        for (int c = 0; c < 4; ++c) st_chunk_h(sb + M::P + swz(t, s0 + 8 * c), &v[8 * c]);
      }
    }
    fence_async_smem();
    tc_fence_before();
    __syncthreads();

    // ---------------- P2: X = (I + L)^{-1} and Xw = X diag(d1) (warps 0-3)
    //                  || S -> S_h, S *= e^{G_C} (warps 4-7)
    if (warp < 4) {
      // P_ik = X_ii L_ik needs L_ik before X_ik overwrites it: warp i reads
      // only its own block row of L, and only before writing that row
      if (lane < 16) {
        // diagonal block `warp`, column j = lane: right-looking substitution
        // over the block's 16 rows in FP32
        const int base = 16 * warp;
        const int j = lane;
        const float4* lb4 = reinterpret_cast<const float4*>(smem + M::LD32 + warp * 1024);
        // left-looking: x_t = [t == j] - sum_{s<t} L_ts x_s, x_t = 0 for t < j;
        // row t of L read as four 16-byte vectors, four partial sums
        float acc[16];
#pragma unroll
        for (int t = 0; t < 16; ++t) {
          float l[16];
#pragma unroll
          for (int c = 0; c < (t + 3) / 4; ++c) {
            const float4 v4 = lb4[t * 4 + c];   // ordinary loads: free to issue early
            l[4 * c] = v4.x; l[4 * c + 1] = v4.y; l[4 * c + 2] = v4.z; l[4 * c + 3] = v4.w;
          }
          float p0 = (t == j) ? 1.0f : 0.0f, p1 = 0.0f, p2 = 0.0f, p3 = 0.0f;
#pragma unroll
          for (int s2 = 0; s2 < t; ++s2) {
            if ((s2 & 3) == 0) p0 = fmaf(-l[s2], acc[s2], p0);
            if ((s2 & 3) == 1) p1 = fmaf(-l[s2], acc[s2], p1);
            if ((s2 & 3) == 2) p2 = fmaf(-l[s2], acc[s2], p2);
            if ((s2 & 3) == 3) p3 = fmaf(-l[s2], acc[s2], p3);
          }
          acc[t] = (t < j) ? 0.0f : (p0 + p1) + (p2 + p3);
        }
        const float dj = d1[base + j];
        __syncwarp(0x0000ffffu);
        // P_ik below reads this block row's L, and the diagonal block holds no
        // L entries the other lanes still need (they come from the FP32 copy)
#pragma unroll
        for (int t = 0; t < 16; ++t) {
          const __half hx = __float2half_rn(acc[t]);
          const __half hw = __float2half_rn(acc[t] * dj);
          asm volatile("st.shared.b16 [%0], %1;" ::"r"(Xb + swz(base + t, base + j)), "h"(__half_as_ushort(hx))
                       : "memory");
          asm volatile("st.shared.b16 [%0], %1;" ::"r"(Xwb + swz(base + t, base + j)), "h"(__half_as_ushort(hw))
                       : "memory");
        }
      }
      asm volatile("bar.sync 1, 128;" ::: "memory");
      // off-diagonal blocks: warp i owns block row i; P_ik = X_ii L_ik for
      // every k < i is formed first, then block X_ij (i - j = d) at level d:
      // X_ij = -sum_{k=j}^{i-1} P_ik X_kj, every X_kj from an earlier level
      uint32_t Pk[3][4];
      const int g = lane >> 2, c4 = lane & 3;
      {
        uint32_t af[4];
        frag_a(af, Xb, 16 * warp, 16 * warp, lane);
#pragma unroll
        for (int dd = 1; dd <= 3; ++dd) {
          if (dd <= warp) {
            float p0[4] = {0.f, 0.f, 0.f, 0.f}, p1[4] = {0.f, 0.f, 0.f, 0.f};
            uint32_t bf[4];
            frag_b_kn(bf, Xb, 16 * warp, 16 * (warp - dd), lane);   // still L_ik
            mma16816(p0, af, bf[0], bf[1]);
            mma16816(p1, af, bf[2], bf[3]);
            c_to_a(Pk[dd - 1], p0, p1);
          }
        }
      }
      __syncwarp();
#pragma unroll
      for (int d = 1; d < 4; ++d) {
        if (warp >= d) {
          const int i = warp, jb = warp - d;
          float z0[4] = {0.f, 0.f, 0.f, 0.f}, z1[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
          for (int dd = 1; dd <= 3; ++dd) {
            if (dd <= d) {
              uint32_t bf[4];
              frag_b_kn(bf, Xb, 16 * (i - dd), 16 * jb, lane);
              mma16816(z0, Pk[dd - 1], bf[0], bf[1]);
              mma16816(z1, Pk[dd - 1], bf[2], bf[3]);
            }
          }
          const int r0 = 16 * i + g, cc = 16 * jb + 2 * c4;
          const float da = d1[cc], db = d1[cc + 1], dc = d1[cc + 8], dd2 = d1[cc + 9];
          st_s32(Xb + swz(r0, cc), pack_h2(-z0[0], -z0[1]));
          st_s32(Xb + swz(r0 + 8, cc), pack_h2(-z0[2], -z0[3]));
          st_s32(Xb + swz(r0, cc + 8), pack_h2(-z1[0], -z1[1]));
          st_s32(Xb + swz(r0 + 8, cc + 8), pack_h2(-z1[2], -z1[3]));
          st_s32(Xwb + swz(r0, cc), pack_h2(-z0[0] * da, -z0[1] * db));
          st_s32(Xwb + swz(r0 + 8, cc), pack_h2(-z0[2] * da, -z0[3] * db));
          st_s32(Xwb + swz(r0, cc + 8), pack_h2(-z1[0] * dc, -z1[1] * dd2));
          st_s32(Xwb + swz(r0 + 8, cc + 8), pack_h2(-z1[2] * dc, -z1[3] * dd2));
        }
        asm volatile("bar.sync 1, 128;" ::: "memory");
      }
    } else {
      // S (lanes = d_k rows of this quarter, all DVS columns) -> S_h; S *= e^{G_C}
      const int rr = quarter * 32 + lane;
      const float eC = ex2(fb[M::GC2 / 4]);   // published by the barriers above
#pragma unroll
      for (int n0 = 0; n0 < DVS; n0 += 32) {
        uint32_t r[32];
        tmem_ld_32x32b_x32(tmem + lane_off + RS + n0, r);
        tc_wait_ld();
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const int col = n0 + 8 * c;
          float f[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) f[e] = __uint_as_float(r[8 * c + e]);
          st_chunk_h(sb + M::SH + (uint32_t)(col >> 6) * (128 * 128) + swz(rr, col & 63), f);
        }
        uint32_t lo[16], hi[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          lo[e] = __float_as_uint(__uint_as_float(r[e]) * eC);
          hi[e] = __float_as_uint(__uint_as_float(r[16 + e]) * eC);
        }
        tmem_st_32x32b_x16(tmem + lane_off + RS + n0, lo);
        tmem_st_32x32b_x16(tmem + lane_off + RS + n0 + 16, hi);
      }
      tc_wait_st();
      if (warp == 7 && has_next) {     // the next chunk's beta, for scale_v after the barrier
        fn[M::BE / 4 + 2 * lane] = nbs[0];
        fn[M::BE / 4 + 2 * lane + 1] = nbs[1];
      }
    }
    fence_async_smem();
    tc_fence_before();
    __syncthreads();

    // ------------------------------------------ MMA-b: [Xw; X] K -> RB (warp 0), [Xw; X] V -> R2 (warp 1)
    // Two issuing warps: the halves write different TMEM columns, and each
    // MMA costs its issuing thread about 80 cycles.
    if (warp == 0) {
      tc_fence_after();
      constexpr uint32_t idk = idesc_f16(128, DK, 0, 1);
#pragma unroll
      for (int j = 0; j < C / 16; ++j)
        mma_f16_warp(tmem + RB, sdesc(sb + M::P + 64 * 128 + j * 32, 16), sdesc(t3 + j * 2048, M::T3_ATOM), idk,
                     j > 0 ? 1u : 0u);
      tc_commit_warp(bar_mma);
    } else if (warp == 1) {
      tc_fence_after();
      constexpr uint32_t idv = idesc_f16(128, DVS, 0, 1);
#pragma unroll
      for (int j = 0; j < C / 16; ++j)
        mma_f16_warp(tmem + R2, sdesc(sb + M::P + 64 * 128 + j * 32, 16), sdesc(vb + j * 2048, 64 * 128), idv,
                     j > 0 ? 1u : 0u);
      tc_commit_warp(bar_b2);
    }
    // while the tensor cores work: the next chunk's q rows, normalised in place
    if (has_next) {
      wait_loads(bar_ld, (uint32_t)(ch + 1) & 1, abort_flag, a.status);
      lds_waited = ch + 2;
      normalize_rows<DVS>(t3n, 64, tid, a.l2norm);
    }
    if (!cta_wait(bar_mma, mma_phase++ & 1, abort_flag, a.status)) break;

    // ------------------------------------------ P3: W -> [K; Q; W] rows 128..191
    if (quarter < 2) {
      const int t = quarter * 32 + lane;
      const int d0 = colhalf * (DK / 2);
      uint32_t r0[32], r1[32];
      tmem_ld_32x32b_x32(tmem + lane_off + RB + d0, r0);
      tmem_ld_32x32b_x32(tmem + lane_off + RB + d0 + 32, r1);
      tc_wait_ld();
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        const int col = d0 + 8 * c;
        float f[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) f[e] = __uint_as_float(c < 4 ? r0[8 * c + e] : r1[8 * (c - 4) + e]);
        st_chunk_h(t3 + (uint32_t)(col >> 6) * M::T3_ATOM + swz(128 + t, col & 63), f);
      }
    }
    fence_async_smem();
    tc_fence_before();
    __syncthreads();

    // ------------------------------------------ MMA-1: [Q; W] S_h -> RB
    if (warp == 0) {
      tc_fence_after();
      constexpr uint32_t id = idesc_f16(128, DVS, 0, 1);
#pragma unroll
      for (int j = 0; j < DK / 16; ++j)
        mma_f16_warp(tmem + RB, sdesc(t3 + 64 * 128 + (j >> 2) * M::T3_ATOM + (j & 3) * 32, 16),
                sdesc(sb + M::SH + j * 2048, 128 * 128), id, j > 0 ? 1u : 0u);
      tc_commit_warp(bar_mma);
    }
    // the next chunk's k rows and (warp 7) its gate factors
    if (has_next) {
      normalize_rows<DVS>(t3n, 0, tid, a.l2norm);
      if (warp == 7) scan_gates<DVS>(fn, nla, nbs, lane);
    }
    // MMA-1, and U~ (issued by warp 1: MMA-1's commit does not cover it)
    if (!mbar_wait(bar_b2, (uint32_t)ch & 1, a.status)) *abort_flag = 1;
    if (!cta_wait(bar_mma, mma_phase++ & 1, abort_flag, a.status)) break;

    // ------------------------------------------ P4: U = U~ - W S -> U, U'
    if (quarter >= 2) {
      const int t = (quarter - 2) * 32 + lane;
      const float dkt = dkf[t];
#pragma unroll
      for (int c0 = 0; c0 < HALF; c0 += 32) {
        const int n0 = colhalf * HALF + c0;
        uint32_t ru[32], rw[32];
        tmem_ld_32x32b_x32(tmem + lane_off + R2 + n0, ru);
        tmem_ld_32x32b_x32(tmem + lane_off + RB + n0, rw);
        tc_wait_ld();
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const int col = n0 + 8 * c;
          float f[8], fd[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            f[e] = __uint_as_float(ru[8 * c + e]) - __uint_as_float(rw[8 * c + e]);
            fd[e] = f[e] * dkt;
          }
          const uint32_t off = (uint32_t)(col >> 6) * (64 * 128) + swz(t, col & 63);
          st_chunk_h(vb + off, f);
          st_chunk_h(sb + M::UP + off, fd);
        }
      }
    }
    fence_async_smem();
    tc_fence_before();
    __syncthreads();

    // ------------------------------------------ MMA-2: [A; *] U -> RA (warp 0);  MMA-3: S += K^T U' (warp 1)
    if (warp == 0) {
      tc_fence_after();
      constexpr uint32_t id2 = idesc_f16(128, DVS, 0, 1);
#pragma unroll
      for (int j = 0; j < C / 16; ++j)
        mma_f16_warp(tmem + RA, sdesc(sb + M::P + j * 32, 16), sdesc(vb + j * 2048, 64 * 128), id2, j > 0 ? 1u : 0u);
      tc_commit_warp(bar_mma);
    } else if (warp == 1) {
      tc_fence_after();
      constexpr uint32_t id3 = idesc_f16(128, DVS, 1, 1);
#pragma unroll
      for (int j = 0; j < C / 16; ++j)
        mma_f16_warp(tmem + RS, sdesc(t3 + j * 2048, M::T3_ATOM), sdesc(sb + M::UP + j * 2048, 64 * 128), id3, 1u);
      tc_commit_warp(bar_3);
    }
    // the next chunk's beta v
    if (has_next) scale_v<DVS>(sb + M::VB + (uint32_t)pn * M::VB_BYTES, fn, tid);
    // the previous chunk's o staging must be read out before P5 rewrites it
    if (!O_F32 && o_worker && lane == 0) bulk_wait_read0();
    if (!cta_wait(bar_mma, mma_phase++ & 1, abort_flag, a.status)) break;

    // ------------------------------------------ P5: O = e^{G_t} Q S + A U
    if (o_worker) {
      const int t = quarter * 32 + lane;
      const float et = eg[t];
      uint32_t rq0[32], ra0[32];
      if (O_F32) {
#pragma unroll
        for (int c0 = 0; c0 < 64; c0 += 32) {
          const int n0 = o_col0 + c0;
          tmem_ld_32x32b_x32(tmem + lane_off + RB + n0, rq0);
          tmem_ld_32x32b_x32(tmem + lane_off + RA + n0, ra0);
          tc_wait_ld();
          if (t < valid) {
            float4* dst = reinterpret_cast<float4*>(reinterpret_cast<float*>(a.o) +
                                                    ((tok0 + t0 + t) * a.H + h) * (int64_t)a.dv + dv_off + n0);
#pragma unroll
            for (int c = 0; c < 8; ++c) {
              float y[4];
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                y[e] = fmaf(et, __uint_as_float(rq0[4 * c + e]), __uint_as_float(ra0[4 * c + e]));
                amax_bits = max(amax_bits, __float_as_uint(y[e]) & 0x7FFFFFFFu);
              }
              dst[c] = make_float4(y[0], y[1], y[2], y[3]);
            }
          }
        }
      } else {
        // bf16 row of 64 columns -> swizzled 32 x 64 staging box -> TMA store
        uint32_t rq1[32], ra1[32];
        tmem_ld_32x32b_x32(tmem + lane_off + RB + o_col0, rq0);
        tmem_ld_32x32b_x32(tmem + lane_off + RA + o_col0, ra0);
        tmem_ld_32x32b_x32(tmem + lane_off + RB + o_col0 + 32, rq1);
        tmem_ld_32x32b_x32(tmem + lane_off + RA + o_col0 + 32, ra1);
        tc_wait_ld();
        float am = 0.0f;
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          uint32_t w[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int i = (8 * c + 2 * e) & 31;
            const uint32_t* rq = c < 4 ? rq0 : rq1;
            const uint32_t* ra = c < 4 ? ra0 : ra1;
            const float y0 = fmaf(et, __uint_as_float(rq[i]), __uint_as_float(ra[i]));
            const float y1 = fmaf(et, __uint_as_float(rq[i + 1]), __uint_as_float(ra[i + 1]));
            am = fmaxf(am, fmaxf(fabsf(y0), fabsf(y1)));
            w[e] = pack_bf16x2(y0, y1);
          }
          st_s128(o_stage + swz(lane, 8 * c), w[0], w[1], w[2], w[3]);
        }
        // bf16 rounding is monotone: the largest stored |o| is the rounded max
        if (t < valid) amax_bits = max(amax_bits, f32_to_bf16_bits(am) << 16);
        fence_async_smem();
        __syncwarp();
        if (lane == 0) {
          tma_store_3d(&maps.o, o_stage, h * a.dv + dv_off + o_col0, (int32_t)(t0 + quarter * 32), b);
          bulk_commit();
        }
        if (a.oq_codes && t < valid) {
          // this row's 64 staged bf16 values -> four NVFP4 blocks (codes and
          // tiled scales of the output projection's activation, K = H*dv)
          const int64_t row = tok0 + t0 + t;
          const int64_t HV = (int64_t)a.H * a.dv;
          const int64_t kcol = (int64_t)h * a.dv + dv_off + o_col0;
          uint8_t* cp = a.oq_codes + row * (HV >> 1) + (kcol >> 1);
          uint8_t* sp = a.oq_scales + (row >> 7) * (HV >> 6) * 512 + (kcol >> 6) * 512 + (row & 31) * 16 +
                        ((row & 127) >> 5) * 4;
#pragma unroll
          for (int qb = 0; qb < 4; ++qb) {
            const uint4 blk[2] = {ld_s128(o_stage + swz(lane, 16 * qb)), ld_s128(o_stage + swz(lane, 16 * qb + 8))};
            quant_block<Bf16In>(blk, oq_genc, cp + 8 * qb, sp + qb);
          }
        }
      }
    }
    fence_async_smem();       // the next chunk's inputs, written in place above
    tc_fence_before();
  }

  if (!O_F32 && o_worker && lane == 0) bulk_wait0();
  if (tid == 0 && nchunks > 0 && !mbar_wait(bar_3, (uint32_t)(nchunks - 1) & 1, a.status)) *abort_flag = 1;
  __syncthreads();
  tc_fence_after();
  if (a.o_amax) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) amax_bits = max(amax_bits, __shfl_xor_sync(0xffffffffu, amax_bits, o));
    if (lane == 0 && amax_bits) atomicMax(a.o_amax, amax_bits);
  }
  if (a.S_T && *abort_flag == 0) {
    const int r = quarter * 32 + lane;
#pragma unroll
    for (int c0 = 0; c0 < HALF; c0 += 32) {
      const int n0 = colhalf * HALF + c0;
      uint32_t v[32];
      tmem_ld_32x32b_x32(tmem + lane_off + RS + n0, v);
      tc_wait_ld();
      float4* dst = reinterpret_cast<float4*>(a.S_T + ((int64_t)chain * DK + r) * a.dv + dv_off + n0);
#pragma unroll
      for (int c = 0; c < 8; ++c)
        dst[c] = make_float4(__uint_as_float(v[4 * c]), __uint_as_float(v[4 * c + 1]), __uint_as_float(v[4 * c + 2]),
                             __uint_as_float(v[4 * c + 3]));
    }
  }
  // a chunk load still in flight after an abort lands before the CTA exits
  if (tid == 0 && lds_issued > lds_waited) {
    for (uint32_t i = 0; i < kWaitLimit && !mbar_try_wait(bar_ld, (uint32_t)lds_waited & 1); ++i) __nanosleep(32);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// 3-D tensor map over a bf16 tensor addressed (feature, token, batch) with a
// token stride of ld elements: boxes of 64 features x `rows` tokens, 128-byte
// swizzle.
bool make_map_3d(CUtensorMap* map, const void* base, int64_t features, int64_t T, int64_t B, int64_t ld,
                 uint32_t rows) {
  auto encode = tensor_map_encoder();
  if (!encode) return false;
  cuuint64_t dims[3] = {(cuuint64_t)features, (cuuint64_t)T, (cuuint64_t)B};
  cuuint64_t strides[2] = {(cuuint64_t)(ld * 2), (cuuint64_t)(ld * 2 * T)};
  cuuint32_t box[3] = {64, rows, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  return encode(map, CU_TENSOR_MAP_DATA_TYPE_UINT16, 3, const_cast<void*>(base), dims, strides, box, estr,
                CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int DVS, bool O_F32>
int launch_dvs(const Args& a, const Maps& m, int64_t chains, cudaStream_t stream) {
  const size_t smem = Map<DVS>::BYTES + 1024;
  cudaError_t e =
      cudaFuncSetAttribute(delta_rule_tc_kernel<DVS, O_F32>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return record_cuda_error(e);
  delta_rule_tc_kernel<DVS, O_F32><<<(unsigned)(chains * a.nsplit), NT, smem, stream>>>(a, m);
  return check_launch();
}

}  // namespace

bool delta_rule_tc_supported(int dk, int dv, int64_t T) { return dk == DK && dv % 64 == 0 && T < ((int64_t)1 << 31); }

int launch_delta_rule_tc(const uint16_t* q, const uint16_t* k, const uint16_t* v, int64_t ld_q, int64_t ld_k,
                         int64_t ld_v, const float* log_alpha, const float* beta, const float* S0, int64_t B,
                         int64_t T, int H, int dk, int dv, int flags, void* o, float* S_T, unsigned* o_amax,
                         cudaStream_t stream, const OQuant* oq) {
  const int64_t chains = B * H;
  if (chains == 0) return GDN_OK;
  if (!delta_rule_tc_supported(dk, dv, T)) return GDN_ERR_UNSUPPORTED_SHAPE;
  if (oq && (flags & GDN_DR_O_FP32)) return GDN_ERR_UNSUPPORTED_SHAPE;
  // d_v slices of 128 columns unless the chains leave more than half the SMs idle
  const int sms = num_sms();
  int dvs = (dv % 128 == 0) ? 128 : 64;
  if (dvs == 128 && chains * (dv / 128) * 2 <= sms) dvs = 64;
  const bool f32 = (flags & GDN_DR_O_FP32) != 0;
  Maps m;
  memset(&m, 0, sizeof(m));
  const int64_t Tm = T > 0 ? T : 1;
  if (!make_map_3d(&m.q, q, (int64_t)H * dk, Tm, B, ld_q, 64) || !make_map_3d(&m.k, k, (int64_t)H * dk, Tm, B, ld_k, 64) ||
      !make_map_3d(&m.v, v, (int64_t)H * dv, Tm, B, ld_v, 64) ||
      (!f32 && !make_map_3d(&m.o, o, (int64_t)H * dv, Tm, B, (int64_t)H * dv, 32)))
    return record_cuda_error(cudaErrorInvalidValue);
  Args a{};
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
  if (oq) {
    a.oq_codes = oq->codes;
    a.oq_scales = oq->scales;
    a.oq_g_enc = oq->g_enc;
    a.oq_g_out = oq->g_out;
  }
  if (dvs == 128) return f32 ? launch_dvs<128, true>(a, m, chains, stream) : launch_dvs<128, false>(a, m, chains, stream);
  return f32 ? launch_dvs<64, true>(a, m, chains, stream) : launch_dvs<64, false>(a, m, chains, stream);
}

}  // namespace gdn
