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
// S_h and apply the chunk's decay to it.  q, k, v arrive by TMA (3-D tensor
// maps, so the rows past the end of a sequence read as zeros) into 128-byte
// swizzled staging, one chunk ahead; o leaves by TMA through shared memory.
//
// TMEM (512 columns): RA = K K^T | Q K^T, later A U;  RB = [Xw; X] K, later
// [Q; W] S_h;  R2 = [Xw; X] V;  RS = the state.
// Every wait is bounded: a wait that runs out records GDN_ERR_TIMEOUT and the
// CTA leaves the chunk loop.
#include <cuda_fp16.h>

#include <cstring>

#include "common.cuh"
#include "kernels.h"
#include "tmap.cuh"

namespace gdn {
namespace {

constexpr int C = 64;
constexpr int DK = 128;
constexpr int NT = 256;
constexpr float kLog2e = 1.4426950408889634f;

// Shared-memory map (byte offsets from a 1024-aligned base).
template <int DVS>
struct Map {
  static constexpr uint32_t T3_ATOM = 192 * 128;             // one 64-column atom of [K; Q; W]
  static constexpr uint32_t T3 = 0;                          // [K; Q; W]: 192 rows x 128 fp16, K-major
  static constexpr uint32_t P = T3 + 2 * T3_ATOM;            // [A; Xw; X]: 192 rows x 64 fp16
  static constexpr uint32_t L = P + 192 * 128;               // L: 64 x 64 fp16
  static constexpr uint32_t BV = L + 64 * 128;               // beta V, later U: 64 tokens x DVS, N-major
  static constexpr uint32_t UP = BV + 64 * 2 * DVS;          // U' = diag(e^{G_C-G_s}) U; o staging
  static constexpr uint32_t SH = UP + 64 * 2 * DVS;          // S_h: 128 (d_k) x DVS, N-major
  static constexpr uint32_t QS = SH + 128 * 2 * DVS;         // raw bf16 q: 2 atoms of 64 rows x 128 B
  static constexpr uint32_t KS = QS + 2 * 64 * 128;          // raw bf16 k
  static constexpr uint32_t VS = KS + 2 * 64 * 128;          // raw bf16 v: DVS / 64 atoms
  static constexpr uint32_t LD_BYTES = 4 * 64 * 128 + 64 * 2 * DVS;   // one chunk's TMA bytes
  static constexpr uint32_t LAR = VS + 64 * 2 * DVS;         // raw log alpha, beta
  static constexpr uint32_t BER = LAR + C * 4;
  static constexpr uint32_t G2 = BER + C * 4;                // G_t log2 e
  static constexpr uint32_t G2M1 = G2 + C * 4;               // G_{t-1} log2 e
  static constexpr uint32_t BE = G2M1 + C * 4;               // beta_t
  static constexpr uint32_t D1 = BE + C * 4;                 // beta_t e^{G_{t-1}}
  static constexpr uint32_t EG = D1 + C * 4;                 // e^{G_t}
  static constexpr uint32_t DKF = EG + C * 4;                // e^{G_C - G_t}
  static constexpr uint32_t MISC = DKF + C * 4;              // mbarriers, tmem ptr, flags, G_C
  static constexpr uint32_t BYTES = MISC + 64;
};

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
__device__ __forceinline__ void mma_f16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                        uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
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
__device__ __forceinline__ float2 unpack_h2(uint32_t w) {
  return __half22float2(*reinterpret_cast<const __half2*>(&w));
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

__device__ __forceinline__ void cp_async4(uint32_t dst, const void* src, bool valid) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;" ::"r"(dst), "l"(src), "r"(valid ? 4 : 0) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_group 0;" ::: "memory"); }

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
};
struct Maps {
  CUtensorMap q, k, v, o;   // 3-D: (feature, token, batch); o only for bf16 output
};

// The chunk's q, k, v tiles by TMA (thread 0) and its gates by cp.async
// (warp 1); rows past the end of the sequence arrive as zeros.
template <int DVS>
__device__ __forceinline__ void issue_chunk_loads(uint32_t sb, const Maps& m, const Args& a, int b, int h,
                                                  int dv_off, int64_t t0, int tid, int warp, int lane) {
  using M = Map<DVS>;
  if (tid == 0) {
    const uint32_t bar = sb + M::MISC + 8;
    mbar_arrive_expect_tx(reinterpret_cast<uint64_t*>(__cvta_shared_to_generic(bar)), M::LD_BYTES);
#pragma unroll
    for (int at = 0; at < 2; ++at) {
      tma_load_3d(sb + M::QS + at * 8192, &m.q, bar, h * DK + 64 * at, (int32_t)t0, b);
      tma_load_3d(sb + M::KS + at * 8192, &m.k, bar, h * DK + 64 * at, (int32_t)t0, b);
    }
#pragma unroll
    for (int at = 0; at < DVS / 64; ++at)
      tma_load_3d(sb + M::VS + at * 8192, &m.v, bar, h * a.dv + dv_off + 64 * at, (int32_t)t0, b);
  }
  if (warp == 1) {
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const int t = 2 * lane + e;
      const bool ok = t0 + t < a.T;
      const int64_t tok = (int64_t)b * a.T + (ok ? t0 + t : 0);
      cp_async4(sb + M::LAR + t * 4, a.log_alpha + tok * a.H + h, ok);
      cp_async4(sb + M::BER + t * 4, a.beta + tok * a.H + h, ok);
    }
    cp_async_commit();
  }
}

// Thread 0 waits (bounded) for the phase of `bar` with the given parity, then
// the CTA synchronises; returns false on every thread when the wait ran out.
__device__ __forceinline__ bool cta_wait(uint64_t* bar, uint32_t parity, volatile int* abort_flag, int* status) {
  if (threadIdx.x == 0) {
    if (!mbar_wait(bar, parity, status)) *abort_flag = 1;
  }
  __syncthreads();
  tc_fence_after();
  return *abort_flag == 0;
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
  const float* g2 = reinterpret_cast<const float*>(smem + M::G2);
  const float* g2m1 = reinterpret_cast<const float*>(smem + M::G2M1);
  const float* be = reinterpret_cast<const float*>(smem + M::BE);
  const float* d1 = reinterpret_cast<const float*>(smem + M::D1);
  const float* eg = reinterpret_cast<const float*>(smem + M::EG);
  const float* dkf = reinterpret_cast<const float*>(smem + M::DKF);
  uint64_t* bar_mma = reinterpret_cast<uint64_t*>(smem + M::MISC);
  uint64_t* bar_ld = reinterpret_cast<uint64_t*>(smem + M::MISC + 8);
  uint32_t* tmem_ptr = reinterpret_cast<uint32_t*>(smem + M::MISC + 16);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + M::MISC + 20);
  float* gC2 = reinterpret_cast<float*>(smem + M::MISC + 24);

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
  // [A; Xw; X] starts zero: the strictly upper blocks of Xw and X are never
  // written afterwards.
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
  const uint32_t o_stage = sb + M::UP + (uint32_t)((DVS == 128 ? colhalf * 2 : 0) + quarter) * 4096;

  uint32_t amax_bits = 0;
  uint32_t mma_phase = 0, ld_phase = 0;
  const int64_t nchunks = (T + C - 1) / C;
  if (nchunks > 0) issue_chunk_loads<DVS>(sb, maps, a, b, h, dv_off, 0, tid, warp, lane);
  tc_fence_before();

#pragma unroll 1
  for (int64_t ch = 0; ch < nchunks; ++ch) {
    const int64_t t0 = ch * C;
    const int valid = (int)(T - t0 < C ? T - t0 : C);
    cp_async_wait_all();
    if (!O_F32 && o_worker && lane == 0) bulk_wait_read0();   // o staging (UP) is rewritten in P4
    if (!cta_wait(bar_ld, ld_phase & 1, abort_flag, a.status)) break;
    ++ld_phase;

    // ------------------------------------------ P0: norms, gates
    {
      constexpr int QC = DK / 4;          // 32 columns per thread, 4 threads per row
      const int pr = tid >> 2, pq = tid & 3;
      float qv[QC], kv[QC];
#pragma unroll
      for (int i = 0; i < QC / 8; ++i) {
        const int col = pq * QC + 8 * i;
        const uint32_t off = (uint32_t)(col >> 6) * 8192 + swz(pr, col & 63);
        unpack_bf16x8(ld_s128(sb + M::QS + off), &qv[8 * i]);
        unpack_bf16x8(ld_s128(sb + M::KS + off), &kv[8 * i]);
      }
      float qs0 = 0.f, qs1 = 0.f, ks0 = 0.f, ks1 = 0.f;
#pragma unroll
      for (int i = 0; i < QC; i += 2) {
        qs0 = fmaf(qv[i], qv[i], qs0);
        qs1 = fmaf(qv[i + 1], qv[i + 1], qs1);
        ks0 = fmaf(kv[i], kv[i], ks0);
        ks1 = fmaf(kv[i + 1], kv[i + 1], ks1);
      }
      float qs = qs0 + qs1, ks = ks0 + ks1;
      qs += __shfl_xor_sync(0xffffffffu, qs, 1);
      ks += __shfl_xor_sync(0xffffffffu, ks, 1);
      qs += __shfl_xor_sync(0xffffffffu, qs, 2);
      ks += __shfl_xor_sync(0xffffffffu, ks, 2);
      const float nq = a.l2norm ? rsqrtf(qs + 1e-6f) : 1.0f;
      const float nk = a.l2norm ? rsqrtf(ks + 1e-6f) : 1.0f;
#pragma unroll
      for (int i = 0; i < QC; ++i) {
        qv[i] *= nq;
        kv[i] *= nk;
      }
      // K rows 0..63 and Q rows 64..127 of [K; Q; W]
#pragma unroll
      for (int i = 0; i < QC / 8; ++i) {
        const int col = pq * QC + 8 * i;
        const uint32_t atom = (uint32_t)(col >> 6) * M::T3_ATOM;
        st_chunk_h(sb + M::T3 + atom + swz(pr, col & 63), &kv[8 * i]);
        st_chunk_h(sb + M::T3 + atom + swz(64 + pr, col & 63), &qv[8 * i]);
      }
    }
    // gates: warp 7, two tokens per lane, one inclusive scan of pair sums
    if (warp == 7) {
      const float* lar = reinterpret_cast<const float*>(smem + M::LAR);
      const float* ber = reinterpret_cast<const float*>(smem + M::BER);
      float* w_g2 = reinterpret_cast<float*>(smem + M::G2);
      float* w_g2m1 = reinterpret_cast<float*>(smem + M::G2M1);
      float* w_be = reinterpret_cast<float*>(smem + M::BE);
      float* w_d1 = reinterpret_cast<float*>(smem + M::D1);
      float* w_eg = reinterpret_cast<float*>(smem + M::EG);
      float* w_dkf = reinterpret_cast<float*>(smem + M::DKF);
      const float la0 = lar[2 * lane], la1 = lar[2 * lane + 1];
      const float pair = la0 + la1;
      float x = pair;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const float y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
      }
      const float ex = x - pair;
      const float G0 = ex + la0, G1 = x;
      const float GC = __shfl_sync(0xffffffffu, x, 31);
      const float b0 = ber[2 * lane], b1 = ber[2 * lane + 1];
      const float Gs[2] = {G0, G1}, Gm[2] = {ex, G0}, bs[2] = {b0, b1};
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int t = 2 * lane + e;
        w_g2[t] = Gs[e] * kLog2e;
        w_g2m1[t] = Gm[e] * kLog2e;
        w_be[t] = bs[e];
        w_d1[t] = bs[e] * ex2(Gm[e] * kLog2e);
        w_eg[t] = ex2(Gs[e] * kLog2e);
        w_dkf[t] = ex2((GC - Gs[e]) * kLog2e);
      }
      if (lane == 31) *gC2 = GC * kLog2e;
    }
    __syncthreads();
    // beta o V: the staging and the operand share the N-major swizzled layout
    for (int i = tid; i < C * DVS / 8; i += NT) {
      const uint32_t off = (uint32_t)i * 16;
      const int r = (i >> 3) & 63;           // token row of this 16-byte chunk
      float f[8];
      unpack_bf16x8(ld_s128(sb + M::VS + off), f);
      const float bt = be[r];
#pragma unroll
      for (int e = 0; e < 8; ++e) f[e] *= bt;
      st_chunk_h(sb + M::BV + off, f);
    }
    fence_async_smem();
    __syncthreads();

    // ------------------------------------------ MMA-a: [K; Q] K^T -> RA
    if (tid == 0) {
      tc_fence_after();
      constexpr uint32_t id = idesc_f16(128, 64, 0, 0);
#pragma unroll
      for (int j = 0; j < DK / 16; ++j) {
        const uint64_t d = sdesc(sb + M::T3 + (j >> 2) * M::T3_ATOM + (j & 3) * 32, 16);
        mma_f16(tmem + RA, d, d, id, j > 0 ? 1u : 0u);
      }
      tc_commit(bar_mma);
    }
    // staging consumed: prefetch the next chunk
    if (ch + 1 < nchunks) issue_chunk_loads<DVS>(sb, maps, a, b, h, dv_off, t0 + C, tid, warp, lane);
    if (!cta_wait(bar_mma, mma_phase++ & 1, abort_flag, a.status)) break;

    // ------------------------------------------ P1: L and A from RA
    {
      uint32_t r[32];
      tmem_ld_32x32b_x32(tmem + lane_off + RA + colhalf * 32, r);
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
#pragma unroll
        for (int c = 0; c < 4; ++c) st_chunk_h(sb + M::L + swz(t, s0 + 8 * c), &v[8 * c]);
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
    const uint32_t Xb = sb + M::P + 128 * 128;
    const uint32_t Xwb = sb + M::P + 64 * 128;
    const uint32_t Lb = sb + M::L;
    if (warp < 4) {
      if (lane < 16) {
        // diagonal block `warp`, column j = lane: right-looking substitution
        // over the block's 16 rows in FP32
        const int base = 16 * warp;
        const int j = lane;
        uint32_t lw[16][8];            // row t of the block: 16 fp16 as 8 half2
#pragma unroll
        for (int t = 1; t < 16; ++t) {
          const uint4 u0 = ld_s128(Lb + swz(base + t, base));
          const uint4 u1 = ld_s128(Lb + swz(base + t, base + 8));
          lw[t][0] = u0.x; lw[t][1] = u0.y; lw[t][2] = u0.z; lw[t][3] = u0.w;
          lw[t][4] = u1.x; lw[t][5] = u1.y; lw[t][6] = u1.z; lw[t][7] = u1.w;
        }
        float acc[16];
#pragma unroll
        for (int t = 0; t < 16; ++t) acc[t] = (t == j) ? 1.0f : 0.0f;
#pragma unroll
        for (int s2 = 0; s2 < 16; ++s2) {
          const float xs = (s2 < j) ? 0.0f : acc[s2];
          acc[s2] = xs;
#pragma unroll
          for (int t = s2 + 1; t < 16; ++t) {
            const float2 lp = unpack_h2(lw[t][s2 >> 1]);
            acc[t] = fmaf(-((s2 & 1) ? lp.y : lp.x), xs, acc[t]);
          }
        }
        const float dj = d1[base + j];
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
      // off-diagonal blocks, one level (distance) at a time; warp i owns block
      // row i and keeps P_ik = X_ii L_ik in registers
      uint32_t Pk[3][4];
      const int g = lane >> 2, c4 = lane & 3;
#pragma unroll 1
      for (int d = 1; d < 4; ++d) {
        if (warp >= d) {
          const int i = warp, jb = warp - d;
          {
            float p0[4] = {0.f, 0.f, 0.f, 0.f}, p1[4] = {0.f, 0.f, 0.f, 0.f};
            uint32_t af[4], bf[4];
            frag_a(af, Xb, 16 * i, 16 * i, lane);
            frag_b_kn(bf, Lb, 16 * i, 16 * (i - d), lane);
            mma16816(p0, af, bf[0], bf[1]);
            mma16816(p1, af, bf[2], bf[3]);
            c_to_a(Pk[d - 1], p0, p1);
          }
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
      const float eC = ex2(*gC2);
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
    }
    fence_async_smem();
    tc_fence_before();
    __syncthreads();

    // ------------------------------------------ MMA-b: [Xw; X] K -> RB, [Xw; X] V -> R2
    if (tid == 0) {
      tc_fence_after();
      constexpr uint32_t idk = idesc_f16(128, DK, 0, 1);
      constexpr uint32_t idv = idesc_f16(128, DVS, 0, 1);
#pragma unroll
      for (int j = 0; j < C / 16; ++j) {
        const uint64_t ad = sdesc(sb + M::P + 64 * 128 + j * 32, 16);
        mma_f16(tmem + RB, ad, sdesc(sb + M::T3 + j * 2048, M::T3_ATOM), idk, j > 0 ? 1u : 0u);
        mma_f16(tmem + R2, ad, sdesc(sb + M::BV + j * 2048, 64 * 128), idv, j > 0 ? 1u : 0u);
      }
      tc_commit(bar_mma);
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
        st_chunk_h(sb + M::T3 + (uint32_t)(col >> 6) * M::T3_ATOM + swz(128 + t, col & 63), f);
      }
    }
    fence_async_smem();
    tc_fence_before();
    __syncthreads();

    // ------------------------------------------ MMA-1: [Q; W] S_h -> RB
    if (tid == 0) {
      tc_fence_after();
      constexpr uint32_t id = idesc_f16(128, DVS, 0, 1);
#pragma unroll
      for (int j = 0; j < DK / 16; ++j)
        mma_f16(tmem + RB, sdesc(sb + M::T3 + 64 * 128 + (j >> 2) * M::T3_ATOM + (j & 3) * 32, 16),
                sdesc(sb + M::SH + j * 2048, 128 * 128), id, j > 0 ? 1u : 0u);
      tc_commit(bar_mma);
    }
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
          st_chunk_h(sb + M::BV + off, f);
          st_chunk_h(sb + M::UP + off, fd);
        }
      }
    }
    fence_async_smem();
    tc_fence_before();
    __syncthreads();

    // ------------------------------------------ MMA-2: [A; *] U -> RA;  MMA-3: S += K^T U'
    if (tid == 0) {
      tc_fence_after();
      constexpr uint32_t id2 = idesc_f16(128, DVS, 0, 1);
      constexpr uint32_t id3 = idesc_f16(128, DVS, 1, 1);
#pragma unroll
      for (int j = 0; j < C / 16; ++j) {
        const uint64_t ub = sdesc(sb + M::BV + j * 2048, 64 * 128);
        mma_f16(tmem + RA, sdesc(sb + M::P + j * 32, 16), ub, id2, j > 0 ? 1u : 0u);
        mma_f16(tmem + RS, sdesc(sb + M::T3 + j * 2048, M::T3_ATOM), sdesc(sb + M::UP + j * 2048, 64 * 128), id3,
                1u);
      }
      tc_commit(bar_mma);
    }
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
#pragma unroll
        for (int c0 = 0; c0 < 64; c0 += 32) {
          const int n0 = o_col0 + c0;
          tmem_ld_32x32b_x32(tmem + lane_off + RB + n0, rq0);
          tmem_ld_32x32b_x32(tmem + lane_off + RA + n0, ra0);
          tc_wait_ld();
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            uint32_t w[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const float y0 = fmaf(et, __uint_as_float(rq0[8 * c + 2 * e]), __uint_as_float(ra0[8 * c + 2 * e]));
              const float y1 =
                  fmaf(et, __uint_as_float(rq0[8 * c + 2 * e + 1]), __uint_as_float(ra0[8 * c + 2 * e + 1]));
              const uint32_t b0 = f32_to_bf16_bits(y0), b1 = f32_to_bf16_bits(y1);
              if (t < valid) amax_bits = max(amax_bits, max(b0 & 0x7FFFu, b1 & 0x7FFFu) << 16);
              w[e] = b0 | (b1 << 16);
            }
            st_s128(o_stage + swz(lane, c0 + 8 * c), w[0], w[1], w[2], w[3]);
          }
        }
        fence_async_smem();
        __syncwarp();
        if (lane == 0) {
          tma_store_3d(&maps.o, o_stage, h * a.dv + dv_off + o_col0, (int32_t)(t0 + quarter * 32), b);
          bulk_commit();
        }
      }
    }
    tc_fence_before();
  }

  cp_async_wait_all();
  if (!O_F32 && o_worker && lane == 0) bulk_wait0();
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
  if (tid == 0 && *abort_flag) {
    for (uint32_t i = 0; i < kWaitLimit && !mbar_try_wait(bar_ld, ld_phase & 1); ++i) __nanosleep(32);
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
                         cudaStream_t stream) {
  const int64_t chains = B * H;
  if (chains == 0) return GDN_OK;
  if (!delta_rule_tc_supported(dk, dv, T)) return GDN_ERR_UNSUPPORTED_SHAPE;
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
  if (dvs == 128) return f32 ? launch_dvs<128, true>(a, m, chains, stream) : launch_dvs<128, false>(a, m, chains, stream);
  return f32 ? launch_dvs<64, true>(a, m, chains, stream) : launch_dvs<64, false>(a, m, chains, stream);
}

}  // namespace gdn
