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
// One CTA (12 warps) walks one (batch, head, d_v slice) chain; the layout of
// the work is described above the kernel.  Every product of the chunk runs as
// tcgen05.mma.kind::f16 (FP16 operands from shared memory in 128-byte swizzled
// layouts, FP32 accumulators in TMEM), stacked so that each MMA has M = 128:
//   MMA-a  [K; Q] K^T            -> K K^T (rows 0..63) and Q K^T (64..127)
//   MMA-b  [Xw; X] K, [Xw; X] bV -> W (rows 0..63 of the first), U~ (rows
//                                   64..127 of the second)
//   MMA-1  [Q'; W] S_h           -> Q' S (rows 0..63) and W S (64..127),
//                                   Q' = diag(e^{G_t}) Q
//   MMA-2  [A; *] U              -> adds A U to rows 0..63 (o = Q' S + A U)
//   MMA-3  S += K'^T U           (K' = diag(e^{G_C-G_s}) K; S lives in TMEM)
// The state stays FP32 in TMEM for the whole sequence; its FP16 copy S_h is
// the B operand of MMA-1.  The 64 x 64 unit-lower-triangular inverse runs on
// mma.sync (diagonal 16 x 16 blocks by substitution in FP32, then the
// off-diagonal blocks level by level).
#include <cuda_fp16.h>

#include <algorithm>
#include <cstring>

#include "common.cuh"
#include "quant_math.cuh"
#include "kernels.h"
#include "tmap.cuh"

namespace gdn {
namespace {

constexpr int C = 64;
constexpr int DK = 128;
constexpr float kLog2e = 1.4426950408889634f;
constexpr uint32_t kImgBytes = 128 * 128;   // one chunk's [Xw; X]: 128 rows of 64 FP16

// Per-token factors of one chunk (float offsets into a factor block): G_t and
// G_{t-1} times log2(e), beta_t, beta_t e^{G_{t-1}}, e^{G_t}, e^{G_C - G_t}, and
// G_C times log2(e).
struct Fac {
  static constexpr uint32_t G2 = 0, G2M1 = C, BE = 2 * C, D1 = 3 * C, EG = 4 * C, DKF = 5 * C, GC2 = 6 * C;
  static constexpr uint32_t BYTES = 6 * C * 4 + 32;
};

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

// Untiled bulk copy global -> shared (16-byte aligned, size % 16 == 0),
// completing on the mbarrier at shared address bar.
__device__ __forceinline__ void bulk_load_s(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
               "l"(src), "r"(bytes), "r"(bar)
               : "memory");
}
__device__ __forceinline__ void tma_load_3d(uint32_t dst, const void* tmap, uint32_t bar, int32_t c0, int32_t c1,
                                            int32_t c2) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4, %5}], [%2];" ::
          "r"(dst),
      "l"(tmap), "r"(bar), "r"(c0), "r"(c1), "r"(c2)
      : "memory");
}
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
  // segments: every sequence is cut into nseg pieces of T_seg tokens (the
  // last one shorter), one CTA per (batch, segment, head, d_v slice); S0 and
  // S_T are per (batch, segment, head) unless st_last_only, when S_T is the
  // last segment's final state per (batch, head).  nseg = 1, T_seg = T: one
  // piece per sequence.
  int nseg;
  int64_t T_seg;
  int st_last_only;
  // state columns per row of S0 / S_T (dv, or more when some slices carry
  // other columns), and the number of leading slices whose v is taken as
  // zero and whose initial state is the identity (they propagate the
  // segment's state-transition matrix instead of its state)
  int dv_state;
  int zero_splits;
  void* o;              // may be null: no o (nor its amax or NVFP4 codes)
  float* S_T;
  unsigned* o_amax;
  int* status;
  // [Xw; X] images of every chunk, precomputed by chunk_inverse_kernel
  // (kernels instantiated with XPRE), indexed ((b * nch_T + chunk) * H + h);
  // nch_T = chunks per sequence
  const uint8_t* xinv;
  int64_t nch_T;
  // fused NVFP4 quantization of the bf16 o (codes == nullptr: off)
  uint8_t* oq_codes;
  uint8_t* oq_scales;
  const float* oq_g_enc;
  float* oq_g_out;
};
struct Maps {
  CUtensorMap q, k, v;      // 3-D: (feature, token, batch)
};

// The raw gates of chunk t0 (warp 7: two tokens per lane; zero past the end
// of the segment, `len` tokens), fetched well before they are needed.
__device__ __forceinline__ void fetch_gates(const Args& a, int64_t tok0, int h, int64_t t0, int64_t len, int lane,
                                            float (&la)[2], float (&bs)[2]) {
#pragma unroll
  for (int e = 0; e < 2; ++e) {
    const int64_t t = t0 + 2 * lane + e;
    const bool ok = t < len;
    la[e] = ok ? __ldg(a.log_alpha + (tok0 + t) * a.H + h) : 0.0f;
    bs[e] = ok ? __ldg(a.beta + (tok0 + t) * a.H + h) : 0.0f;
  }
}

// Warp 7: the chunk's gate factors into factor block f from the fetched raw
// gates (an inclusive scan of log alpha, two tokens per lane).
__device__ __forceinline__ void scan_gates(float* f, const float (&la)[2], const float (&bs)[2], int lane) {
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
    f[Fac::G2 + t] = Gs[e] * kLog2e;
    f[Fac::G2M1 + t] = Gm[e] * kLog2e;
    f[Fac::D1 + t] = bs[e] * ex2(Gm[e] * kLog2e);
    f[Fac::EG + t] = ex2(Gs[e] * kLog2e);
    f[Fac::DKF + t] = ex2((GC - Gs[e]) * kLog2e);
  }
  if (lane == 31) f[Fac::GC2] = GC * kLog2e;
}

// ===========================================================================
// Pipelined scan: the state-independent work of a chunk overlaps the state
// update of the previous one.
//
// Only three products of the chunk form touch the state: W S and Q' S (one
// stacked MMA), A U and the update S += K'^T U.  Everything else -- the
// normalisation, the gates, K K^T and Q K^T, L and A, the 64 x 64 inverse,
// W = Xw K and U~ = X beta V -- depends on the chunk's inputs alone.  So the
// CTA (12 warps) splits into two warp groups:
//   prep group  (warps 0-7): chunk c+1's normalisation, gates, MMA-a, L / A,
//               inverse (warps 0-3) with Q' = diag(e^{G_t}) Q (warps 4-7) beside
//               it, MMA-b, W;
//   state group (warps 8-11): chunk c's S -> S_h, MMA-1 PO = [Q'; W] S_h,
//               U = U~ - W S, MMA-2 PO += [A; *] U and MMA-3 S += K'^T U with
//               K' = diag(e^{G_C - G_s}) K, then o = the Q' S + A U rows of PO.
// The chunk tiles ([K; Q; W], [A; Xw; X], beta V / U) are double-buffered:
// chunk c+2's q, k, v are loaded by TMA into chunk c's buffers as soon as its
// MMA-2 and MMA-3 have completed.  The prep work runs on twice the warps of
// the state work: it is latency-bound, and two warps per scheduler hide
// about half of the shared-memory and dependent-FMA latency one warp cannot.
//
// TMEM: PS = the state (FP32, d_k lanes x d_v), PO = [Q' S + A U; W S],
// PP = prep scratch (K K^T | Q K^T, then W = [Xw; X] K), PU = [*; U~].
//
// Every FP16 operand is range-checked: a value of magnitude >= 65520 (which
// rounds to infinity in FP16) records GDN_ERR_RANGE in the status word.
// Every wait is bounded; a wait that runs out (or sees the other group give
// up) makes both groups leave their loops through uniform barrier votes.
constexpr uint32_t PS = 0, PO = 128, PP = 256, PU = 384;
constexpr int NTP = 384;                    // threads of the pipelined kernel
constexpr int NPG = 256, NSG = 128;         // prep group, state group
constexpr float kHalfOverflow = 65520.0f;   // smallest magnitude that rounds to +-inf in FP16

template <int DVS>
struct PMap {
  static constexpr uint32_t T3_ATOM = 192 * 128;             // one 64-column atom of [K; Q; W]
  static constexpr uint32_t T3_BYTES = 2 * T3_ATOM;          // 192 rows x 128 fp16, K-major
  static constexpr uint32_t P_BYTES = 192 * 128;             // [A; Xw; X]: 192 rows x 64 fp16 (L in X's place)
  static constexpr uint32_t VB_BYTES = 64 * 2 * DVS;         // beta v, then U: 64 tokens x DVS, N-major
  static constexpr uint32_t STAGE = T3_BYTES + P_BYTES + VB_BYTES;
  static constexpr uint32_t SH = 2 * STAGE;                  // S_h: 128 (d_k) x DVS fp16, N-major
  static constexpr uint32_t LD32 = SH + 128 * 2 * DVS;       // FP32 diagonal 16 x 16 blocks of L
  static constexpr uint32_t F = LD32 + 4 * 16 * 16 * 4;      // 2 x per-token factors
  static constexpr uint32_t F_BYTES = Fac::BYTES;
  static constexpr uint32_t MISC = F + 2 * F_BYTES;          // mbarriers, tmem ptr, flags, counters
  static constexpr uint32_t LD_KQ = 2 * 64 * 128 * 2;        // one chunk's k and q bytes
  static constexpr uint32_t LD_V = 64 * 2 * DVS;              // one chunk's v bytes
  static constexpr uint32_t BYTES = MISC + 128;
  static constexpr uint32_t t3(int s) { return (uint32_t)s * STAGE; }
  static constexpr uint32_t pt(int s) { return (uint32_t)s * STAGE + T3_BYTES; }
  static constexpr uint32_t vb(int s) { return (uint32_t)s * STAGE + T3_BYTES + P_BYTES; }
};
static_assert(PMap<128>::STAGE % 1024 == 0 && PMap<64>::STAGE % 1024 == 0 && PMap<128>::SH % 1024 == 0 &&
                  PMap<64>::SH % 1024 == 0,
              "swizzled tiles need 1024-byte alignment");
static_assert(PMap<128>::BYTES + 1024 <= 232448, "shared memory budget");

__device__ __forceinline__ void named_bar(int id, int n) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory");
}
// Barrier over `n` threads that also returns the OR of every thread's `p`
// (the same value on every thread: a uniform decision).
__device__ __forceinline__ bool bar_vote_or(int id, int n, bool p) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred pi, po;\n\t"
      "setp.ne.u32 pi, %1, 0;\n\t"
      "bar.red.or.pred po, %2, %3, pi;\n\t"
      "selp.u32 %0, 1, 0, po;\n\t}"
      : "=r"(r)
      : "r"((uint32_t)p), "r"(id), "r"(n)
      : "memory");
  return r != 0;
}
// Bounded wait that also gives up when the abort flag is raised.
__device__ __forceinline__ bool mbar_wait_ab(uint64_t* bar, uint32_t parity, volatile int* abort_flag,
                                             int* status) {
  for (uint32_t i = 0; i < kWaitLimit; ++i) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((i & 255u) == 255u && *abort_flag) return false;
    if (i > 64) __nanosleep(32);
  }
  report_status(status, GDN_ERR_TIMEOUT);
  return false;
}
// Every thread of an n-thread group waits, then the group votes: true on
// every thread when all waits completed and nobody has given up.
__device__ __forceinline__ bool grp_wait(uint64_t* bar, uint32_t parity, volatile int* abort_flag, int* status,
                                         int bar_id, int n) {
  bool bad = !mbar_wait_ab(bar, parity, abort_flag, status);
  bad = bar_vote_or(bar_id, n, bad || *abort_flag != 0);
  if (bad) *abort_flag = 1;
  return !bad;
}
__device__ __forceinline__ bool grp_ok(volatile int* abort_flag, int bar_id, int n) {
  return !bar_vote_or(bar_id, n, *abort_flag != 0);
}

// Largest magnitude of eight values, as a tree (short dependency chains).
__device__ __forceinline__ float absmax8(const float* v) {
  const float a = fmaxf(fabsf(v[0]), fabsf(v[1])), b = fmaxf(fabsf(v[2]), fabsf(v[3]));
  const float c = fmaxf(fabsf(v[4]), fabsf(v[5])), d = fmaxf(fabsf(v[6]), fabsf(v[7]));
  return fmaxf(fmaxf(a, b), fmaxf(c, d));
}
// Eight FP32 values -> one 16-byte chunk of FP16, tracking the largest magnitude.
__device__ __forceinline__ void st_chunk_hc(uint32_t addr, const float* v, float& hmax) {
  hmax = fmaxf(hmax, absmax8(v));
  st_chunk_h(addr, v);
}
// One 16-byte chunk of FP16 -> eight FP32 values.
__device__ __forceinline__ void unpack_h8(const uint4& u, float* f) {
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const float2 p = __half22float2(*reinterpret_cast<const __half2*>(&w[e]));
    f[2 * e] = p.x;
    f[2 * e + 1] = p.y;
  }
}
// In place: the eight FP16 values at `addr` times `e` (e <= 1: stays in range).
__device__ __forceinline__ void scale_chunk_h(uint32_t addr, float e) {
  float f[8];
  unpack_h8(ld_s128(addr), f);
#pragma unroll
  for (int i = 0; i < 8; ++i) f[i] *= e;
  st_chunk_h(addr, f);
}

// The q and k rows of chunk t0 into stage s, and (separately) its v rows
// (with XPRE also the chunk's precomputed [Xw; X]); rows past the end of the
// sequence arrive as zeros.  One thread each; the stage's load barrier
// completes once both halves have landed.
template <int DVS>
__device__ __forceinline__ void pipe_load_kq(uint32_t sb, uint64_t* bar, const Maps& m, int b, int h, int64_t t0,
                                             int s) {
  using M = PMap<DVS>;
  mbar_arrive_expect_tx(bar, M::LD_KQ);
  const uint32_t bar_s = smem_u32(bar);
  const uint32_t t3 = sb + M::t3(s);
#pragma unroll
  for (int at = 0; at < 2; ++at) {
    tma_load_3d(t3 + at * M::T3_ATOM, &m.k, bar_s, h * DK + 64 * at, (int32_t)t0, b);
    tma_load_3d(t3 + at * M::T3_ATOM + 64 * 128, &m.q, bar_s, h * DK + 64 * at, (int32_t)t0, b);
  }
}
template <int DVS, bool XPRE>
__device__ __forceinline__ void pipe_load_v(uint32_t sb, uint64_t* bar, const Maps& m, const Args& a, int b, int h,
                                            int dv_off, int64_t t0, int s) {
  using M = PMap<DVS>;
  mbar_arrive_expect_tx(bar, M::LD_V + (XPRE ? kImgBytes : 0u));
  const uint32_t bar_s = smem_u32(bar);
  const uint32_t vb = sb + M::vb(s);
#pragma unroll
  for (int at = 0; at < DVS / 64; ++at)
    tma_load_3d(vb + at * 8192, &m.v, bar_s, h * a.dv + dv_off + 64 * at, (int32_t)t0, b);
  // the chunk's precomputed [Xw; X] into rows 64..191 of [A; Xw; X]
  if (XPRE)
    bulk_load_s(sb + M::pt(s) + 64 * 128, a.xinv + (((int64_t)b * a.nch_T + t0 / C) * a.H + h) * kImgBytes,
                kImgBytes, bar_s);
}

// In place: the bf16 rows r0 .. r0 + nthreads/4 - 1 of a tile of 64-column
// atoms ATOM bytes apart -> L2-normalised FP16 (four threads per row, 32
// columns each).  Thread pq of a row takes the 16-byte chunks pq and pq + 4
// of both 64-column atoms, in an order that puts the eight threads of two
// adjacent rows on eight distinct swizzled bank groups (the plain column
// order hit every bank group twice).
template <uint32_t ATOM>
__device__ __forceinline__ void normalize_rows(uint32_t t3, int r0, int tid, int l2norm, float& hmax) {
  constexpr int QC = DK / 4;
  const int pr = tid >> 2, pq = tid & 3;
  float v[QC];
  uint32_t off[QC / 8];
#pragma unroll
  for (int i = 0; i < QC / 8; ++i) {
    const int L = pq + 4 * ((i & 1) ^ (pr & 1));   // eight distinct bank groups per two rows
    off[i] = t3 + (uint32_t)(i >> 1) * ATOM + swz(r0 + pr, 8 * L);
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
  for (int i = 0; i < QC / 8; ++i) st_chunk_hc(off[i], &v[8 * i], hmax);
}

// One row t of L (quarters 0 and 1 of the K K^T accumulator: rows t < 64),
// columns s0 = 32 colhalf .. s0 + 31 in r:
//   L_ts = beta_t e^{G_{t-1} - G_s} k_t.k_s  (s < t),  0 otherwise,
// stored as FP16 in X's place (the inverse overwrites it), the row's chunks of
// Xw zeroed (the inverse writes only Xw's lower blocks, and the rows may hold
// other data), and the row's piece of its diagonal 16 x 16 block kept in FP32
// at ld32 (4 blocks of 16 x 16).
__device__ __forceinline__ void build_l_row(const uint32_t (&r)[32], int t, int colhalf, uint32_t Xb, uint32_t Xwb,
                                            uint32_t ld32, const float* be, const float* g2m1, const float* g2,
                                            float& hmax) {
  const int s0 = colhalf * 32;
  const float bt = be[t], gm = g2m1[t];
  float v[32];
#pragma unroll
  for (int i = 0; i < 32; ++i) {
    const int s2 = s0 + i;
    v[i] = (s2 < t) ? bt * ex2(fminf(gm - g2[s2], 0.0f)) * __uint_as_float(r[i]) : 0.0f;
  }
#pragma unroll
  for (int cc = 0; cc < 4; ++cc) {
    st_chunk_hc(Xb + swz(t, s0 + 8 * cc), &v[8 * cc], hmax);
    st_s128(Xwb + swz(t, s0 + 8 * cc), 0u, 0u, 0u, 0u);
  }
  const int blk = t >> 4;
  if ((blk >> 1) == colhalf) {
    // the diagonal block's 16 columns are the first or second half of these 32
    const uint32_t dst = ld32 + (uint32_t)(blk * 256 + (t & 15) * 16) * 4;
    if (blk & 1) {
#pragma unroll
      for (int cc = 0; cc < 4; ++cc)
        st_s128(dst + cc * 16, __float_as_uint(v[16 + 4 * cc]), __float_as_uint(v[17 + 4 * cc]),
                __float_as_uint(v[18 + 4 * cc]), __float_as_uint(v[19 + 4 * cc]));
    } else {
#pragma unroll
      for (int cc = 0; cc < 4; ++cc)
        st_s128(dst + cc * 16, __float_as_uint(v[4 * cc]), __float_as_uint(v[1 + 4 * cc]),
                __float_as_uint(v[2 + 4 * cc]), __float_as_uint(v[3 + 4 * cc]));
    }
  }
}

// X = (I + L)^{-1} and Xw = X diag(d1) (d1_s = beta_s e^{G_{s-1}}), both
// FP16 in 128-byte-swizzled 64 x 64 tiles, from L in X's place and its FP32
// diagonal blocks at ld32.  Four warps (warp = 0..3, 128 threads meeting at
// named barrier bar_id): the diagonal 16 x 16 blocks by substitution in FP32,
// then the off-diagonal blocks level by level on mma.sync,
//   X_ij = -X_ii sum_{i > k >= j} L_ik X_kj.
__device__ __forceinline__ void chunk_inverse(const float4* ld32, uint32_t Xb, uint32_t Xwb, const float* d1,
                                              int warp, int lane, float& hmax, int bar_id) {
  {
    // every lane solves column j = lane % 16 (the two half-warps the
    // same column): lanes 0-15 store X, lanes 16-31 store Xw
    const int base = 16 * warp;
    const int j = lane & 15;
    const bool wside = lane >= 16;
    const float4* lb4 = ld32 + warp * 64;
    float acc[16];
#pragma unroll
    for (int t = 0; t < 16; ++t) {
      float l[16];
#pragma unroll
      for (int cc = 0; cc < (t + 3) / 4; ++cc) {
        const float4 v4 = lb4[t * 4 + cc];
        l[4 * cc] = v4.x; l[4 * cc + 1] = v4.y; l[4 * cc + 2] = v4.z; l[4 * cc + 3] = v4.w;
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
    const float dj = wside ? d1[base + j] : 1.0f;
    const uint32_t dst = wside ? Xwb : Xb;
    __syncwarp();
    float am = 0.0f;
#pragma unroll
    for (int t = 0; t < 16; ++t) {
      const float x = acc[t] * dj;
      am = fmaxf(am, fabsf(x));
      const __half hx = __float2half_rn(x);
      asm volatile("st.shared.b16 [%0], %1;" ::"r"(dst + swz(base + t, base + j)), "h"(__half_as_ushort(hx))
                   : "memory");
    }
    hmax = fmaxf(hmax, am);
  }
  named_bar(bar_id, 128);
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
      hmax = fmaxf(hmax, fmaxf(fmaxf(fmaxf(fabsf(z0[0]), fabsf(z0[1])), fmaxf(fabsf(z0[2]), fabsf(z0[3]))),
                               fmaxf(fmaxf(fabsf(z1[0]), fabsf(z1[1])), fmaxf(fabsf(z1[2]), fabsf(z1[3])))));
      st_s32(Xb + swz(r0, cc), pack_h2(-z0[0], -z0[1]));
      st_s32(Xb + swz(r0 + 8, cc), pack_h2(-z0[2], -z0[3]));
      st_s32(Xb + swz(r0, cc + 8), pack_h2(-z1[0], -z1[1]));
      st_s32(Xb + swz(r0 + 8, cc + 8), pack_h2(-z1[2], -z1[3]));
      st_s32(Xwb + swz(r0, cc), pack_h2(-z0[0] * da, -z0[1] * db));
      st_s32(Xwb + swz(r0 + 8, cc), pack_h2(-z0[2] * da, -z0[3] * db));
      st_s32(Xwb + swz(r0, cc + 8), pack_h2(-z1[0] * dc, -z1[1] * dd2));
      st_s32(Xwb + swz(r0 + 8, cc + 8), pack_h2(-z1[2] * dc, -z1[3] * dd2));
    }
    named_bar(bar_id, 128);
  }
}

template <int DVS, bool O_F32, bool XPRE>
__global__ void __launch_bounds__(NTP, 1)
    delta_rule_pipe_kernel(const __grid_constant__ Args a, const __grid_constant__ Maps maps) {
  using M = PMap<DVS>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t sraw = smem_u32(smem_raw);
  const uint32_t sb = (sraw + 1023u) & ~1023u;
  uint8_t* smem = smem_raw + (sb - sraw);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + M::MISC);
  uint64_t* bar_ld = bars;          // [2] chunk loads of stage s
  uint64_t* bar_prep = bars + 2;    // [2] stage s prepared (prep -> state)
  uint64_t* bar_a = bars + 4;       // MMA-a done
  uint64_t* bar_b = bars + 5;       // MMA-b done
  uint64_t* bar_u = bars + 6;       // U~ read out of PU (state -> prep), two arrivals
  uint64_t* bar_1 = bars + 7;       // MMA-1 done
  uint64_t* bar_23 = bars + 8;      // MMA-2 and MMA-3 done
  uint64_t* bar_fin = bars + 9;     // [2] everything an issuing warp started has completed
  uint32_t* tmem_ptr = reinterpret_cast<uint32_t*>(smem + M::MISC + 96);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + M::MISC + 100);
  int* consumed = reinterpret_cast<int*>(smem + M::MISC + 104);     // [2] chunk loads waited for, per stage

  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  const int chain = blockIdx.x / a.nsplit;   // (batch, segment, head)
  const int split = blockIdx.x % a.nsplit;
  const int h = chain % a.H;
  const int b = (chain / a.H) / a.nseg, p = (chain / a.H) % a.nseg;
  const bool zero_v = split < a.zero_splits;
  const int dv_off = zero_v ? 0 : (split - a.zero_splits) * DVS;     // the v / o columns of this slice
  const int st_off = split * DVS;                                    // its S0 / S_T columns
  const int64_t T = a.T;
  const int64_t seg0 = (int64_t)p * a.T_seg;                         // the segment's first token
  const int64_t len = T - seg0 < a.T_seg ? T - seg0 : a.T_seg;
  const int64_t tok0 = (int64_t)b * T + seg0;
  const int64_t nchunks = (len + C - 1) / C;
  constexpr int LD_ISSUER = NTP - 32;   // warp 11, lane 0: issues every chunk load
  constexpr int BAR_PG = 1, BAR_SG = 2, BAR_INV = 3;

  if (tid == 0) {
    mbar_init(&bar_ld[0], 2);       // k and q, then v
    mbar_init(&bar_ld[1], 2);
    mbar_init(&bar_prep[0], 1);
    mbar_init(&bar_prep[1], 1);
    mbar_init(bar_a, 1);
    mbar_init(bar_b, 1);
    mbar_init(bar_u, 2);
    mbar_init(bar_1, 1);
    mbar_init(bar_23, 1);
    mbar_init(&bar_fin[0], 1);
    mbar_init(&bar_fin[1], 1);
    *abort_flag = 0;
    consumed[0] = consumed[1] = 0;
    fence_mbar_init();
  }
  if (tid == LD_ISSUER) {
    prefetch_tmap(&maps.q);
    prefetch_tmap(&maps.k);
    prefetch_tmap(&maps.v);
  }
  if (warp == 0) {
    tmem_alloc(tmem_ptr, 512);
    tmem_relinquish();
  }
  // [A; Xw; X] of both stages start zero (every row is rewritten each chunk)
  for (int i = tid; i < 2 * (int)(M::P_BYTES / 16); i += NTP) {
    const int s = i / (int)(M::P_BYTES / 16), j = i % (int)(M::P_BYTES / 16);
    st_s128(sb + M::pt(s) + (uint32_t)j * 16, 0u, 0u, 0u, 0u);
  }
  fence_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_ptr;
  const int quarter = warp & 3;     // the TMEM lane quarter this warp may access
  const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
  // LD_ISSUER only: chunks whose k, q (kq*) and v (v*) loads were issued to
  // stages 0 and 1
  int kq0 = 0, kq1 = 0, v0 = 0, v1 = 0;
  if (tid == LD_ISSUER) {
    if (nchunks > 0) {
      pipe_load_kq<DVS>(sb, &bar_ld[0], maps, b, h, seg0, 0);
      pipe_load_v<DVS, XPRE>(sb, &bar_ld[0], maps, a, b, h, dv_off, seg0, 0);
      kq0 = v0 = 1;
    }
    if (nchunks > 1) {
      pipe_load_kq<DVS>(sb, &bar_ld[1], maps, b, h, seg0 + C, 1);
      pipe_load_v<DVS, XPRE>(sb, &bar_ld[1], maps, a, b, h, dv_off, seg0 + C, 1);
      kq1 = v1 = 1;
    }
  }
  float hmax = 0.0f;                // largest magnitude this thread converted to FP16

  if (warp < 8) {
    // ======================================================== prep group
    const int colhalf = warp >> 2;
    float nla[2] = {0.f, 0.f}, nbs[2] = {0.f, 0.f};
    if (warp == 7 && nchunks > 0) fetch_gates(a, tok0, h, 0, len, lane, nla, nbs);
    int64_t c = 0;
#pragma unroll 1
    for (; c < nchunks; ++c) {
      const int s = (int)(c & 1);
      const uint32_t ph = (uint32_t)(c >> 1) & 1u;
      const uint32_t t3 = sb + M::t3(s), pb = sb + M::pt(s), vb = sb + M::vb(s);
      float* fb = reinterpret_cast<float*>(smem + M::F + (uint32_t)s * M::F_BYTES);
      const float* g2 = fb + Fac::G2;
      const float* g2m1 = fb + Fac::G2M1;
      const float* be = fb + Fac::BE;
      const float* eg = fb + Fac::EG;
      // the gate factors of chunk c (raw gates fetched one chunk ahead)
      if (warp == 7) {
        const float la[2] = {nla[0], nla[1]}, bs[2] = {nbs[0], nbs[1]};
        if (c + 1 < nchunks) fetch_gates(a, tok0, h, (c + 1) * C, len, lane, nla, nbs);
        fb[Fac::BE + 2 * lane] = bs[0];
        fb[Fac::BE + 2 * lane + 1] = bs[1];
        scan_gates(fb, la, bs, lane);
      }
      if (!grp_wait(&bar_ld[s], ph, abort_flag, a.status, BAR_PG, NPG)) break;
      // q, k rows normalised in place (k rows 0..63, q rows 64..127)
      normalize_rows<M::T3_ATOM>(t3, 0, tid, a.l2norm, hmax);
      normalize_rows<M::T3_ATOM>(t3, 64, tid, a.l2norm, hmax);
      named_bar(BAR_PG, NPG);     // the factor block, for beta
      // beta v in place
      for (int i = tid; i < C * DVS / 8; i += NPG) {
        const uint32_t off = (uint32_t)i * 16;
        const float bt = zero_v ? 0.0f : be[(i >> 3) & 63];
        float x[8];
        unpack_bf16x8(ld_s128(vb + off), x);
#pragma unroll
        for (int e = 0; e < 8; ++e) x[e] *= bt;
        st_chunk_hc(vb + off, x, hmax);
      }
      fence_async_smem();
      named_bar(BAR_PG, NPG);
      // MMA-a: [K; Q] K^T -> PP (K K^T in lanes 0..63, Q K^T in lanes 64..127)
      if (warp == 0) {
        tc_fence_after();
        constexpr uint32_t id = idesc_f16(128, 64, 0, 0);
#pragma unroll
        for (int j = 0; j < DK / 16; ++j) {
          const uint64_t d = sdesc(t3 + (j >> 2) * M::T3_ATOM + (j & 3) * 32, 16);
          mma_f16_warp(tmem + PP, d, d, id, j > 0 ? 1u : 0u);
        }
        tc_commit_warp(bar_a);
      }
      if (!grp_wait(bar_a, (uint32_t)c & 1u, abort_flag, a.status, BAR_PG, NPG)) break;
      tc_fence_after();

      // ---- L (quarters 0, 1; in X's place, plus FP32 diagonal blocks) and A (quarters 2, 3)
      const uint32_t Xb = pb + 128 * 128, Xwb = pb + 64 * 128;
      // Q' = diag(e^{G_t}) Q in place, 128 threads j (MMA-a has finished
      // reading Q); the two threads of a row walk their atoms half a row
      // apart, so four rows' eight chunks fall on distinct bank groups
      auto q_prime = [&](int j) {
        const int row = j >> 1, c0 = (j & 1) * 64;
        const float e = eg[row];
#pragma unroll
        for (int cc = 0; cc < 64; cc += 8) {
          const int col = c0 + ((cc + 32 * (j & 1)) & 63);
          scale_chunk_h(t3 + (uint32_t)(col >> 6) * M::T3_ATOM + swz(64 + row, col & 63), e);
        }
      };
      if (!XPRE || quarter >= 2) {
        uint32_t r[32];
        tmem_ld_32x32b_x32(tmem + lane_off + PP + colhalf * 32, r);
        tc_wait_ld();
        if (quarter < 2) {
          build_l_row(r, quarter * 32 + lane, colhalf, Xb, Xwb, sb + M::LD32, be, g2m1, g2, hmax);
        } else {
          const int t = (quarter - 2) * 32 + lane;
          const float gt = g2[t];
          const int s0 = colhalf * 32;
          float v[32];
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            const int s2 = s0 + i;
            v[i] = (s2 <= t) ? ex2(fminf(gt - g2[s2], 0.0f)) * __uint_as_float(r[i]) : 0.0f;
          }
#pragma unroll
          for (int cc = 0; cc < 4; ++cc) st_chunk_hc(pb + swz(t, s0 + 8 * cc), &v[8 * cc], hmax);
        }
      } else {
        // X and Xw came with the chunk's loads: quarters 0, 1 take Q' beside A
        q_prime((((warp >> 2) << 1) | (warp & 1)) * 32 + lane);
      }
      if (!XPRE) {
        named_bar(BAR_PG, NPG);
        if (warp < 4) {
          // ---- X = (I + L)^{-1} and Xw = X diag(beta_s e^{G_{s-1}}) (warps 0-3)
          chunk_inverse(reinterpret_cast<const float4*>(smem + M::LD32), Xb, Xwb, fb + Fac::D1, warp, lane, hmax,
                        BAR_INV);
        } else {
          q_prime(tid - 128);   // beside the inverse (warps 4-7)
        }
      }
      fence_async_smem();
      tc_fence_before();
      // the state group has read chunk c-1's U~ out of PU
      if (c > 0) {
        if (!grp_wait(bar_u, (uint32_t)(c - 1) & 1u, abort_flag, a.status, BAR_PG, NPG)) break;
      } else if (!grp_ok(abort_flag, BAR_PG, NPG)) {
        break;
      }
      // MMA-b: [Xw; X] K -> PP (W in lanes 0..63), [Xw; X] beta V -> PU (U~ in lanes 64..127)
      if (warp == 0) {
        tc_fence_after();
        constexpr uint32_t idk = idesc_f16(128, DK, 0, 1);
        constexpr uint32_t idv = idesc_f16(128, DVS, 0, 1);
#pragma unroll
        for (int j = 0; j < C / 16; ++j)
          mma_f16_warp(tmem + PP, sdesc(pb + 64 * 128 + j * 32, 16), sdesc(t3 + j * 2048, M::T3_ATOM), idk,
                       j > 0 ? 1u : 0u);
#pragma unroll
        for (int j = 0; j < C / 16; ++j)
          mma_f16_warp(tmem + PU, sdesc(pb + 64 * 128 + j * 32, 16), sdesc(vb + j * 2048, 64 * 128), idv,
                       j > 0 ? 1u : 0u);
        tc_commit_warp(bar_b);
      }
      if (!grp_wait(bar_b, (uint32_t)c & 1u, abort_flag, a.status, BAR_PG, NPG)) break;
      tc_fence_after();
      // ---- W -> [K; Q; W] rows 128..191 (quarters 0, 1: 64 columns per warp)
      if (quarter < 2) {
        const int t = quarter * 32 + lane;
        const int d0 = colhalf * (DK / 2);
#pragma unroll
        for (int c0 = 0; c0 < DK / 2; c0 += 32) {
          uint32_t r[32];
          tmem_ld_32x32b_x32(tmem + lane_off + PP + d0 + c0, r);
          tc_wait_ld();
#pragma unroll
          for (int cc = 0; cc < 4; ++cc) {
            const int col = d0 + c0 + 8 * cc;
            float f[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) f[e] = __uint_as_float(r[8 * cc + e]);
            st_chunk_hc(t3 + (uint32_t)(col >> 6) * M::T3_ATOM + swz(128 + t, col & 63), f, hmax);
          }
        }
      }
      fence_async_smem();
      tc_fence_before();
      named_bar(BAR_PG, NPG);
      if (tid == 0) mbar_arrive(&bar_prep[s]);
    }
    if (tid == 0) {
      consumed[0] = (int)((c + 1) / 2);
      consumed[1] = (int)(c / 2);
    }
    // every MMA this group issued has completed before TMEM is freed
    if (warp == 0) {
      tc_commit_warp(&bar_fin[0]);
      mbar_wait(&bar_fin[0], 0, a.status);
    }
  } else {
    // ======================================================= state group
    const int gt = tid - NPG;
    // S (FP32, TMEM PS): lane r = d_k row, column n = d_v column of the slice
    {
      const int r = quarter * 32 + lane;
#pragma unroll
      for (int c0 = 0; c0 < DVS; c0 += 16) {
        uint32_t v[16];
#pragma unroll
        for (int i = 0; i < 16; ++i)
          v[i] = __float_as_uint(zero_v ? (r == st_off + c0 + i ? 1.0f : 0.0f)
                                 : a.S0 ? a.S0[((int64_t)chain * DK + r) * a.dv_state + st_off + c0 + i] : 0.0f);
        tmem_st_32x32b_x16(tmem + lane_off + PS + c0, v);
      }
      tc_wait_st();
    }
    uint32_t amax_bits = 0;
    const float oq_genc = a.oq_codes ? *a.oq_g_enc : 1.0f;
    if (a.oq_codes && blockIdx.x == 0 && gt == 0) *a.oq_g_out = __fdiv_rn(1.0f, oq_genc);
    int64_t c = 0;
#pragma unroll 1
    for (; c < nchunks; ++c) {
      const int s = (int)(c & 1);
      const uint32_t ph = (uint32_t)(c >> 1) & 1u;
      const int64_t t0 = c * C;
      const int valid = (int)(len - t0 < C ? len - t0 : C);
      const uint32_t t3 = sb + M::t3(s), pb = sb + M::pt(s), vb = sb + M::vb(s);
      const float* fb = reinterpret_cast<const float*>(smem + M::F + (uint32_t)s * M::F_BYTES);
      tc_fence_before();
      if (!grp_wait(&bar_prep[s], ph, abort_flag, a.status, BAR_SG, NSG)) break;
      tc_fence_after();
      // ---- S -> S_h (FP16, shared);  S *= e^{G_C} (TMEM)
      {
        const int rr = quarter * 32 + lane;
        const float eC = ex2(fb[Fac::GC2]);
#pragma unroll
        for (int n0 = 0; n0 < DVS; n0 += 32) {
          uint32_t r[32];
          tmem_ld_32x32b_x32(tmem + lane_off + PS + n0, r);
          tc_wait_ld();
#pragma unroll
          for (int cc = 0; cc < 4; ++cc) {
            const int col = n0 + 8 * cc;
            float f[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) f[e] = __uint_as_float(r[8 * cc + e]);
            st_chunk_hc(sb + M::SH + (uint32_t)(col >> 6) * (128 * 128) + swz(rr, col & 63), f, hmax);
          }
          uint32_t lo[16], hi[16];
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            lo[e] = __float_as_uint(__uint_as_float(r[e]) * eC);
            hi[e] = __float_as_uint(__uint_as_float(r[16 + e]) * eC);
          }
          tmem_st_32x32b_x16(tmem + lane_off + PS + n0, lo);
          tmem_st_32x32b_x16(tmem + lane_off + PS + n0 + 16, hi);
        }
        tc_wait_st();
      }
      fence_async_smem();
      tc_fence_before();
      named_bar(BAR_SG, NSG);
      // ---- MMA-1: [Q'; W] S_h -> PO
      if (warp == 8) {
        tc_fence_after();
        constexpr uint32_t id = idesc_f16(128, DVS, 0, 1);
#pragma unroll
        for (int j = 0; j < DK / 16; ++j)
          mma_f16_warp(tmem + PO, sdesc(t3 + 64 * 128 + (j >> 2) * M::T3_ATOM + (j & 3) * 32, 16),
                       sdesc(sb + M::SH + j * 2048, 128 * 128), id, j > 0 ? 1u : 0u);
        tc_commit_warp(bar_1);
      }
      // while it runs: K' = diag(e^{G_C - G_s}) K, for MMA-3, into the X / Xw
      // rows of [A; Xw; X] (MMA-b is done with them): its two 64-column halves
      // as rows 64..127 and 128..191, so the [K; Q; W] tile is free for chunk
      // c+2's k and q as soon as MMA-1 completes
      {
        const float* dkf = fb + Fac::DKF;
        const int row = gt >> 1, half = gt & 1;     // halves half a row apart: distinct bank groups
        const float e = dkf[row];
#pragma unroll
        for (int c8 = 0; c8 < 64; c8 += 8) {
          const int cc = (c8 + 32 * half) & 63;
          float f[8];
          unpack_h8(ld_s128(t3 + (uint32_t)half * M::T3_ATOM + swz(row, cc)), f);
#pragma unroll
          for (int i = 0; i < 8; ++i) f[i] *= e;
          st_chunk_h(pb + swz(64 + 64 * half + row, cc), f);
        }
      }
      fence_async_smem();
      if (!grp_wait(bar_1, (uint32_t)c & 1u, abort_flag, a.status, BAR_SG, NSG)) break;
      tc_fence_after();
      // the [K; Q; W] tile of stage s is free: chunk c+2's k and q
      if (tid == LD_ISSUER && c + 2 < nchunks) {
        pipe_load_kq<DVS>(sb, &bar_ld[s], maps, b, h, seg0 + t0 + 2 * C, s);
        if (s == 0) ++kq0; else ++kq1;
      }
      // ---- U = U~ - W S -> beta-V tile (quarters 2, 3: token rows in lanes 64..127)
      if (quarter >= 2) {
        const int t = (quarter - 2) * 32 + lane;
#pragma unroll
        for (int n0 = 0; n0 < DVS; n0 += 32) {
          uint32_t ru[32], rw[32];
          tmem_ld_32x32b_x32(tmem + lane_off + PU + n0, ru);
          tmem_ld_32x32b_x32(tmem + lane_off + PO + n0, rw);
          tc_wait_ld();
#pragma unroll
          for (int cc = 0; cc < 4; ++cc) {
            const int col = n0 + 8 * cc;
            float f[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) f[e] = __uint_as_float(ru[8 * cc + e]) - __uint_as_float(rw[8 * cc + e]);
            st_chunk_hc(vb + (uint32_t)(col >> 6) * (64 * 128) + swz(t, col & 63), f, hmax);
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar_u);     // PU may take the next chunk's U~
      }
      fence_async_smem();
      tc_fence_before();
      named_bar(BAR_SG, NSG);
      // ---- MMA-2: PO += [A; *] U (rows 0..63: Q'S + AU = o);  MMA-3: S += K'^T U
      if (warp == 8) {
        tc_fence_after();
        constexpr uint32_t id2 = idesc_f16(128, DVS, 0, 1);
        constexpr uint32_t id3 = idesc_f16(128, DVS, 1, 1);
#pragma unroll
        for (int j = 0; j < C / 16; ++j)
          mma_f16_warp(tmem + PO, sdesc(pb + j * 32, 16), sdesc(vb + j * 2048, 64 * 128), id2, 1u);
#pragma unroll
        for (int j = 0; j < C / 16; ++j)
          mma_f16_warp(tmem + PS, sdesc(pb + 64 * 128 + j * 2048, 64 * 128), sdesc(vb + j * 2048, 64 * 128), id3,
                       1u);
        tc_commit_warp(bar_23);
      }
      if (!grp_wait(bar_23, (uint32_t)c & 1u, abort_flag, a.status, BAR_SG, NSG)) break;
      tc_fence_after();
      // the beta-V tile of stage s is free: chunk c+2's v
      if (tid == LD_ISSUER && c + 2 < nchunks) {
        pipe_load_v<DVS, XPRE>(sb, &bar_ld[s], maps, a, b, h, dv_off, seg0 + t0 + 2 * C, s);
        if (s == 0) ++v0; else ++v1;
      }
      // ---- o rows (quarters 0, 1: token rows in lanes 0..63), 32 columns at a time
      if (quarter < 2 && a.o) {
        const int t = quarter * 32 + lane;
        const int64_t row = tok0 + t0 + t;
#pragma unroll 1
        for (int c0 = 0; c0 < DVS; c0 += 32) {
          uint32_t r[32];
          tmem_ld_32x32b_x32(tmem + lane_off + PO + c0, r);
          tc_wait_ld();
          if (O_F32) {
            if (t < valid) {
              float4* dst = reinterpret_cast<float4*>(reinterpret_cast<float*>(a.o) +
                                                      (row * a.H + h) * (int64_t)a.dv + dv_off + c0);
#pragma unroll
              for (int cc = 0; cc < 8; ++cc) {
                float y[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                  y[e] = __uint_as_float(r[4 * cc + e]);
                  amax_bits = max(amax_bits, __float_as_uint(y[e]) & 0x7FFFFFFFu);
                }
                dst[cc] = make_float4(y[0], y[1], y[2], y[3]);
              }
            }
          } else {
            uint4 w4[4];
            float am = 0.0f;
#pragma unroll
            for (int cc = 0; cc < 4; ++cc) {
              uint32_t w[4];
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                const float y0 = __uint_as_float(r[8 * cc + 2 * e]), y1 = __uint_as_float(r[8 * cc + 2 * e + 1]);
                am = fmaxf(am, fmaxf(fabsf(y0), fabsf(y1)));
                w[e] = pack_bf16x2(y0, y1);
              }
              w4[cc] = make_uint4(w[0], w[1], w[2], w[3]);
            }
            if (t < valid) {
              // bf16 rounding is monotone: the largest stored |o| is the rounded max
              amax_bits = max(amax_bits, f32_to_bf16_bits(am) << 16);
              uint4* dst = reinterpret_cast<uint4*>(reinterpret_cast<uint16_t*>(a.o) +
                                                    (row * a.H + h) * (int64_t)a.dv + dv_off + c0);
#pragma unroll
              for (int cc = 0; cc < 4; ++cc) dst[cc] = w4[cc];
              if (a.oq_codes) {
                // these 32 bf16 values -> two NVFP4 blocks (codes and tiled
                // scales of the output projection's activation, K = H*dv)
                const int64_t HV = (int64_t)a.H * a.dv;
                const int64_t kcol = (int64_t)h * a.dv + dv_off + c0;
                uint8_t* cp = a.oq_codes + row * (HV >> 1) + (kcol >> 1);
                uint8_t* sp = a.oq_scales + (row >> 7) * (HV >> 6) * 512 + (kcol >> 6) * 512 + (row & 31) * 16 +
                              ((row & 127) >> 5) * 4 + ((kcol >> 4) & 3);
#pragma unroll
                for (int qb = 0; qb < 2; ++qb) {
                  const uint4 blk[2] = {w4[2 * qb], w4[2 * qb + 1]};
                  quant_block<Bf16In>(blk, oq_genc, cp + 8 * qb, sp + qb);
                }
              }
            }
          }
        }
      }
    }
    // the final state
    if (c == nchunks && a.S_T && *abort_flag == 0 && (!a.st_last_only || p == a.nseg - 1)) {
      const int r = quarter * 32 + lane;
      const int64_t srow = a.st_last_only ? (int64_t)b * a.H + h : chain;
#pragma unroll
      for (int n0 = 0; n0 < DVS; n0 += 32) {
        uint32_t v[32];
        tmem_ld_32x32b_x32(tmem + lane_off + PS + n0, v);
        tc_wait_ld();
        float4* dst = reinterpret_cast<float4*>(a.S_T + (srow * DK + r) * a.dv_state + st_off + n0);
#pragma unroll
        for (int cc = 0; cc < 8; ++cc)
          dst[cc] = make_float4(__uint_as_float(v[4 * cc]), __uint_as_float(v[4 * cc + 1]),
                                __uint_as_float(v[4 * cc + 2]), __uint_as_float(v[4 * cc + 3]));
      }
    }
    if (a.o_amax) {
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) amax_bits = max(amax_bits, __shfl_xor_sync(0xffffffffu, amax_bits, o));
      if (lane == 0 && amax_bits) atomicMax(a.o_amax, amax_bits);
    }
    if (warp == 8) {
      tc_commit_warp(&bar_fin[1]);
      mbar_wait(&bar_fin[1], 0, a.status);
    }
  }

  // an FP16 operand out of range
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) hmax = fmaxf(hmax, __shfl_xor_sync(0xffffffffu, hmax, o));
  if (lane == 0 && hmax >= kHalfOverflow) report_status(a.status, GDN_ERR_RANGE);
  tc_fence_before();
  __syncthreads();
  // chunk loads still in flight after an early exit land before the CTA exits
  if (tid == LD_ISSUER) {
    // a stage whose k and q went out without its v: complete the phase
    if (v0 < kq0) pipe_load_v<DVS, XPRE>(sb, &bar_ld[0], maps, a, b, h, dv_off, seg0 + (int64_t)(2 * (kq0 - 1)) * C, 0);
    if (v1 < kq1)
      pipe_load_v<DVS, XPRE>(sb, &bar_ld[1], maps, a, b, h, dv_off, seg0 + (int64_t)(2 * (kq1 - 1) + 1) * C, 1);
    for (int k = consumed[0]; k < kq0; ++k) mbar_wait(&bar_ld[0], (uint32_t)k & 1u, a.status);
    for (int k = consumed[1]; k < kq1; ++k) mbar_wait(&bar_ld[1], (uint32_t)k & 1u, a.status);
  }
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ===========================================================================
// Inverse pre-pass: X and Xw of every chunk of every (batch, head) chain,
// ahead of the scan.
//
// Nothing in X = (I + L)^{-1} or Xw = X diag(beta_s e^{G_{s-1}}) depends on
// the state: L is built from the chunk's normalised keys and its gates alone.
// So one wide pass computes them for all chunks at once, with every SM busy
// and several CTAs per SM, and writes each
// chunk's pair as the 16 KB shared-memory image that the scan's MMA-b reads
// ([Xw; X]: 128 rows of 64 FP16, 128-byte swizzled).  The scan (XPRE) then
// loads the image with one bulk copy beside the chunk's v instead of building
// L and inverting on its critical path.  The arithmetic is the scan's own
// (the same normalisation, K K^T on the same tensor-core MMA, the same L rows
// and inverse), so the image holds the values the scan would compute.
//
// One CTA of four warps per chunk-head idx = (b * nch_T + chunk) * H + h (the
// launch gives each CTA one; the loop also walks a grid-stride range, loading
// the next chunk's k as soon as the MMA has read this one): TMA load of the
// chunk's 64 k rows, normalisation in place, K K^T into TMEM by one tcgen05
// MMA group (M = 128: the A operand's rows 64..127 are whatever follows the k
// tile in shared memory; their products land in TMEM lanes that are never
// read), the L rows (warps 0, 1: lanes 0..63), the inverse (warps 0-3), the
// image to global memory.
constexpr int NTI = 128;
struct IMap {
  static constexpr uint32_t KT = 0;                  // k: two 64-column atoms of 64 rows
  static constexpr uint32_t K_ATOM = 64 * 128;
  static constexpr uint32_t IMG = 2 * K_ATOM;        // [Xw; X]
  static constexpr uint32_t LD32 = IMG + kImgBytes;  // FP32 diagonal blocks of L
  static constexpr uint32_t F = LD32 + 4 * 16 * 16 * 4;
  static constexpr uint32_t MISC = F + (Fac::BYTES + 15) / 16 * 16;
  static constexpr uint32_t BYTES = MISC + 64;
};
static_assert(IMap::IMG % 1024 == 0, "swizzled tiles need 1024-byte alignment");

__global__ void __launch_bounds__(NTI, 6) chunk_inverse_kernel(const __grid_constant__ Args a,
                                                            const __grid_constant__ Maps maps, uint8_t* img,
                                                            int64_t B) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t sraw = smem_u32(smem_raw);
  const uint32_t sb = (sraw + 1023u) & ~1023u;
  uint8_t* smem = smem_raw + (sb - sraw);
  uint64_t* bar_ld = reinterpret_cast<uint64_t*>(smem + IMap::MISC);
  uint64_t* bar_mma = bar_ld + 1;
  uint64_t* bar_fin = bar_ld + 2;
  uint32_t* tmem_ptr = reinterpret_cast<uint32_t*>(smem + IMap::MISC + 24);
  float* fb = reinterpret_cast<float*>(smem + IMap::F);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int64_t nch = a.nch_T, total = B * nch * a.H;
  const uint32_t kt = sb + IMap::KT, Xwb = sb + IMap::IMG, Xb = Xwb + 64 * 128;
  if (tid == 0) {
    mbar_init(bar_ld, 1);
    mbar_init(bar_mma, 1);
    mbar_init(bar_fin, 1);
    fence_mbar_init();
    prefetch_tmap(&maps.k);
  }
  if (warp == 0) {
    tmem_alloc(tmem_ptr, 64);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_ptr;
  // tid 0: the k rows of chunk-head idx
  auto load = [&](int64_t idx) {
    const int h = (int)(idx % a.H);
    const int64_t g = (idx / a.H) % nch;
    const int b = (int)(idx / (a.H * nch));
    mbar_arrive_expect_tx(bar_ld, 2 * IMap::K_ATOM);
#pragma unroll
    for (int at = 0; at < 2; ++at)
      tma_load_3d(kt + at * IMap::K_ATOM, &maps.k, smem_u32(bar_ld), h * DK + 64 * at, (int32_t)(g * C), b);
  };
  int issued = 0, landed = 0;   // tid 0: k loads issued / waited for
  if (tid == 0 && (int64_t)blockIdx.x < total) {
    load(blockIdx.x);
    issued = 1;
  }
  float hmax = 0.0f;
  uint32_t it = 0;
  // warp 3: the raw gates of chunk-head idx (zero past the end of the
  // sequence), fetched one chunk-head ahead
  float nla[2] = {0.f, 0.f}, nbs[2] = {0.f, 0.f};
  auto fetch = [&](int64_t idx) {
    const int h = (int)(idx % a.H);
    const int64_t g = (idx / a.H) % nch;
    const int b = (int)(idx / (a.H * nch));
    fetch_gates(a, (int64_t)b * a.T, h, g * C, a.T, lane, nla, nbs);
  };
  if (warp == 3 && (int64_t)blockIdx.x < total) fetch(blockIdx.x);
#pragma unroll 1
  for (int64_t idx = blockIdx.x; idx < total; idx += gridDim.x, ++it) {
    if (warp == 3) {
      // the chunk's gate factors
      const float la[2] = {nla[0], nla[1]}, bs[2] = {nbs[0], nbs[1]};
      if (idx + gridDim.x < total) fetch(idx + gridDim.x);
      fb[Fac::BE + 2 * lane] = bs[0];
      fb[Fac::BE + 2 * lane + 1] = bs[1];
      scan_gates(fb, la, bs, lane);
    }
    bool bad = !mbar_wait(bar_ld, it & 1u, a.status);
    if (__syncthreads_or(bad)) break;
    if (tid == 0) landed = issued;
    normalize_rows<IMap::K_ATOM>(kt, 0, tid, a.l2norm, hmax);
    normalize_rows<IMap::K_ATOM>(kt, 32, tid, a.l2norm, hmax);
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    // K K^T -> TMEM (lanes 0..63, 64 columns)
    if (warp == 0) {
      tc_fence_after();
      constexpr uint32_t id = idesc_f16(128, 64, 0, 0);
#pragma unroll
      for (int j = 0; j < DK / 16; ++j) {
        const uint64_t d = sdesc(kt + (j >> 2) * IMap::K_ATOM + (j & 3) * 32, 16);
        mma_f16_warp(tmem, d, d, id, j > 0 ? 1u : 0u);
      }
      tc_commit_warp(bar_mma);
    }
    bad = !mbar_wait(bar_mma, it & 1u, a.status);
    if (__syncthreads_or(bad)) break;
    tc_fence_after();
    // the k tile is free: the next chunk-head's k
    if (tid == 0 && idx + gridDim.x < total) {
      load(idx + gridDim.x);
      ++issued;
    }
    if (warp < 2) {
#pragma unroll
      for (int ch = 0; ch < 2; ++ch) {
        uint32_t r[32];
        tmem_ld_32x32b_x32(tmem + ((uint32_t)(warp * 32) << 16) + ch * 32, r);
        tc_wait_ld();
        build_l_row(r, warp * 32 + lane, ch, Xb, Xwb, sb + IMap::LD32, fb + Fac::BE, fb + Fac::G2M1, fb + Fac::G2,
                    hmax);
      }
    }
    tc_fence_before();
    __syncthreads();
    chunk_inverse(reinterpret_cast<const float4*>(smem + IMap::LD32), Xb, Xwb, fb + Fac::D1, warp, lane, hmax, 1);
    // the image out (the inverse ends at a barrier of all four warps)
    uint4* dst = reinterpret_cast<uint4*>(img + idx * (int64_t)kImgBytes);
#pragma unroll
    for (int i = tid; i < (int)(kImgBytes / 16); i += NTI) dst[i] = ld_s128(Xwb + (uint32_t)i * 16);
  }
  // after an early exit: a k load still in flight lands before the CTA exits
  if (tid == 0 && issued > landed)
    for (uint32_t i = 0; i < kWaitLimit && !mbar_try_wait(bar_ld, (uint32_t)landed & 1u); ++i) __nanosleep(32);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) hmax = fmaxf(hmax, __shfl_xor_sync(0xffffffffu, hmax, o));
  if (lane == 0 && hmax >= kHalfOverflow) report_status(a.status, GDN_ERR_RANGE);
  // every MMA this CTA issued has completed before TMEM is freed
  if (warp == 0) {
    tc_commit_warp(bar_fin);
    mbar_wait(bar_fin, 0, a.status);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 64);
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

template <int DVS, bool O_F32, bool XPRE>
int launch_dvs(const Args& a, const Maps& m, int64_t units, cudaStream_t stream) {
  const size_t smem = PMap<DVS>::BYTES + 1024;
  cudaError_t e = cudaFuncSetAttribute(delta_rule_pipe_kernel<DVS, O_F32, XPRE>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return record_cuda_error(e);
  delta_rule_pipe_kernel<DVS, O_F32, XPRE><<<(unsigned)(units * a.nsplit), NTP, smem, stream>>>(a, m);
  return check_launch();
}

// XPRE (the precomputed inverse) runs with 128-column slices only: the
// segmented path, the one that uses it.
int launch_args(const Args& a, const Maps& m, int64_t units, int dvs, bool f32, cudaStream_t stream) {
  if (a.xinv) {
    if (dvs != 128) return GDN_ERR_UNSUPPORTED_SHAPE;
    return f32 ? launch_dvs<128, true, true>(a, m, units, stream) : launch_dvs<128, false, true>(a, m, units, stream);
  }
  if (dvs == 128)
    return f32 ? launch_dvs<128, true, false>(a, m, units, stream) : launch_dvs<128, false, false>(a, m, units, stream);
  return f32 ? launch_dvs<64, true, false>(a, m, units, stream) : launch_dvs<64, false, false>(a, m, units, stream);
}

// The pre-pass asks for the largest shared-memory carveout: with the default
// the driver may size the SM's shared memory for one 40 KB CTA and leave the
// rest to L1, while the pass needs several CTAs per SM to hide its latency.
cudaError_t inverse_attributes(int smem) {
  cudaError_t e = cudaFuncSetAttribute(chunk_inverse_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  return cudaFuncSetAttribute(chunk_inverse_kernel, cudaFuncAttributePreferredSharedMemoryCarveout,
                              (int)cudaSharedmemCarveoutMaxShared);
}

int launch_inverse(const Args& a, const Maps& m, uint8_t* img, int64_t B, cudaStream_t stream) {
  const int64_t total = B * a.nch_T * a.H;
  if (total == 0) return GDN_OK;
  const int smem = (int)IMap::BYTES + 1024;
  cudaError_t e = inverse_attributes(smem);
  if (e != cudaSuccess) return record_cuda_error(e);
  // one CTA per chunk-head (as many resident per SM as fit: 80 registers,
  // 40 KB of shared memory); measured faster than a persistent grid sized
  // by the occupancy query
  // (the kernel walks a grid-stride range, so a grid capped below 2^31
  // still covers any count)
  chunk_inverse_kernel<<<(unsigned)std::min<int64_t>(total, (int64_t)1 << 30), NTI, smem, stream>>>(a, m, img, B);
  return check_launch();
}

// ---------------------------------------------------------------------------
// Segments: sequences cut into pieces that run in parallel.
//
// The chunk map of the recurrence is affine in the state: a segment takes its
// entry state S to M S + B, where B is the segment's final state when it
// starts from zero and M (d_k x d_k) is what the same steps do to the
// identity with v taken as zero (the write term is the only one that does
// not scale with S).  So with few (batch, head) chains and long sequences --
// too few CTAs to cover the SMs, each walking a long chain of chunks -- the
// sequence is cut into P segments:
//   phase A  segments 0 .. P-2 run from [I | 0] (the identity block with
//            v = 0, then the real v from a zero state): final [M_p | B_p];
//   phase B  S_0 = S0, S_{p+1} = M_p S_p + B_p (FP32, P-1 small products);
//   phase C  every segment runs again from its entry state S_p, writing o
//            and, for the last one, S_T.
// Phase A costs (d_k + d_v) / d_v times the state work of P-1 segments and
// phase C one pass, but both run on P times as many CTAs.

// E[b, p, h] = S_p for p = 0 .. nseg-1, S_0 = S0 (or 0), S_{p+1} = M_p S_p +
// B_p with [M_p | B_p] = MB[b, p, h] ([d_k, d_k + dv]).  One CTA of 256
// threads per (batch, head, 16 state columns): thread t owns column t % 16 of
// rows t / 16 + 16 i (i < 8); S_p's sixteen columns stay in shared memory, and
// M_p with the CTA's 16 columns of B_p is staged there by cp.async,
// double-buffered (p + 1's load while M_p S_p is formed), rows of M padded to
// 132 floats so that the two rows a warp reads fall on distinct banks.  Each
// element sums B_p then k = 0 .. d_k-1 in order.
constexpr int CMB_LD = DK + 4;
constexpr size_t CMB_SMEM = (size_t)(2 * DK * CMB_LD + 2 * DK * 16 + DK * 16) * 4;
__device__ __forceinline__ void cp_async16(void* dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(dst)), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}
__global__ void __launch_bounds__(256) segment_combine_kernel(const float* __restrict__ MB,
                                                              const float* __restrict__ S0, float* __restrict__ E,
                                                              int H, int dv, int nseg) {
  extern __shared__ float cmb[];
  float* Mb = cmb;                      // [2][DK][CMB_LD]
  float* Bb = Mb + 2 * DK * CMB_LD;     // [2][DK][16]: this CTA's 16 columns of B_p
  float* Ss = Bb + 2 * DK * 16;         // [DK][16]
  const int ncb = dv / 16;
  const int cb = blockIdx.x % ncb, bh = blockIdx.x / ncb;
  const int b = bh / H, h = bh % H;
  const int tid = threadIdx.x, c = tid & 15, rg = tid >> 4;
  const int col = cb * 16 + c;
  const int ld = DK + dv;
  auto mb = [&](int p) { return MB + (((int64_t)b * (nseg - 1) + p) * H + h) * DK * ld; };
  auto stage = [&](int p) {
    const float* src = mb(p);
    float* dst = Mb + (p & 1) * DK * CMB_LD;
    for (int i = tid; i < DK * DK / 4; i += 256) {
      const int r = i >> 5, k4 = (i & 31) * 4;
      cp_async16(dst + r * CMB_LD + k4, src + (int64_t)r * ld + k4);
    }
    float* bdst = Bb + (p & 1) * DK * 16;
    for (int i = tid; i < DK * 4; i += 256) {
      const int r = i >> 2, c4 = (i & 3) * 4;
      cp_async16(bdst + r * 16 + c4, src + (int64_t)r * ld + DK + cb * 16 + c4);
    }
    cp_async_commit();
  };
  if (nseg > 1) stage(0);
  float st[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) st[i] = S0 ? S0[(((int64_t)b * H + h) * DK + rg + 16 * i) * dv + col] : 0.0f;
  for (int p = 0;; ++p) {
#pragma unroll
    for (int i = 0; i < 8; ++i) E[((((int64_t)b * nseg + p) * H + h) * DK + rg + 16 * i) * dv + col] = st[i];
    if (p + 1 == nseg) break;
#pragma unroll
    for (int i = 0; i < 8; ++i) Ss[(rg + 16 * i) * 16 + c] = st[i];
    if (p + 2 < nseg) {
      stage(p + 1);
      cp_async_wait<1>();
    } else {
      cp_async_wait<0>();
    }
    __syncthreads();
    const float* M = Mb + (p & 1) * DK * CMB_LD;
    const float* Bp = Bb + (p & 1) * DK * 16;
    float acc[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[i] = Bp[(rg + 16 * i) * 16 + c];
#pragma unroll 2
    for (int k = 0; k < DK; k += 4) {
      float s4[4];
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) s4[kk] = Ss[(k + kk) * 16 + c];
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const float4 m = *reinterpret_cast<const float4*>(M + (rg + 16 * i) * CMB_LD + k);
        acc[i] = fmaf(m.x, s4[0], acc[i]);
        acc[i] = fmaf(m.y, s4[1], acc[i]);
        acc[i] = fmaf(m.z, s4[2], acc[i]);
        acc[i] = fmaf(m.w, s4[3], acc[i]);
      }
    }
    __syncthreads();   // Ss and this M buffer are rewritten next
#pragma unroll
    for (int i = 0; i < 8; ++i) st[i] = acc[i];
  }
}

struct SegPlan {
  int P = 1;
  int64_t T_seg = 0;
};

// The segment count that minimises the chunk steps on the critical path --
// waves of CTAs x (chunks per CTA + the pipeline's fill and drain, about four
// chunk steps), plus one step per sequential product of phase B -- if it
// beats one piece per sequence by a clear margin; d_v a multiple of 128 (the
// identity block is one 128-column slice).
SegPlan plan_segments(int64_t B, int64_t T, int H, int dv, int sms) {
  SegPlan best;
  if (dv % 128 != 0 || T <= 0 || B * H <= 0) return best;
  constexpr int64_t kFill = 4;
  const int64_t chains = B * H, nch = (T + C - 1) / C, sl = dv / 128;
  int64_t plain_split = sl;
  if (chains * sl * 2 <= sms) plain_split = 2 * sl;
  double best_cost = 0.75 * (double)cdiv(chains * plain_split, sms) * (double)(nch + kFill);
  for (int P = 2; P <= 64; ++P) {
    const int64_t tc = cdiv(nch, P);
    if ((P - 1) * tc >= nch) break;   // the last segment would be empty
    const double cost =
        (double)(cdiv(chains * (P - 1) * (1 + sl), sms) + cdiv(chains * P * sl, sms)) * (double)(tc + kFill) + (P - 1);
    if (cost < best_cost) {
      best_cost = cost;
      best.P = P;
      best.T_seg = tc * C;
    }
  }
  return best;
}

size_t seg_bytes_mb(int64_t B, int H, int dv, int P) { return (size_t)(B * (P - 1) * H) * DK * (DK + dv) * 4; }
size_t seg_bytes_e(int64_t B, int H, int dv, int P) { return (size_t)(B * P * H) * DK * dv * 4; }
size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

}  // namespace

bool delta_rule_tc_supported(int dk, int dv, int64_t T) { return dk == DK && dv % 64 == 0 && T < ((int64_t)1 << 31); }

namespace {
// Workspace of the segmented path: [M_p | B_p] and the entry states, then the
// [Xw; X] image of every chunk (the inverse pre-pass).  Both passes of the
// segmented path walk every chunk, so the pre-pass saves one of the two
// inversions of each chunk; in one piece per sequence the scan inverts each
// chunk once, beside the state update, and a pre-pass would cost more than it
// takes off the critical path (measured at B = 4, T = 8192, H = 32).
size_t seg_bytes(int64_t B, int H, int dv, int P) {
  return P > 1 ? align256(align256(seg_bytes_mb(B, H, dv, P)) + seg_bytes_e(B, H, dv, P)) : 0;
}
size_t img_bytes(int64_t B, int64_t T, int H) { return (size_t)(B * ((T + C - 1) / C) * H) * kImgBytes; }
}  // namespace

size_t delta_rule_tc_workspace(int64_t B, int64_t T, int H, int dk, int dv) {
  if (!delta_rule_tc_supported(dk, dv, T) || T <= 0) return 0;
  const SegPlan pl = plan_segments(B, T, H, dv, num_sms());
  return pl.P > 1 ? seg_bytes(B, H, dv, pl.P) + img_bytes(B, T, H) : 0;
}

int launch_delta_rule_tc(const uint16_t* q, const uint16_t* k, const uint16_t* v, int64_t ld_q, int64_t ld_k,
                         int64_t ld_v, const float* log_alpha, const float* beta, const float* S0, int64_t B,
                         int64_t T, int H, int dk, int dv, int flags, void* o, float* S_T, unsigned* o_amax,
                         cudaStream_t stream, const OQuant* oq, void* ws, size_t ws_bytes) {
  const int64_t chains = B * H;
  if (chains == 0) return GDN_OK;
  if (!delta_rule_tc_supported(dk, dv, T)) return GDN_ERR_UNSUPPORTED_SHAPE;
  if (oq && (flags & GDN_DR_O_FP32)) return GDN_ERR_UNSUPPORTED_SHAPE;
  const int sms = num_sms();
  const bool f32 = (flags & GDN_DR_O_FP32) != 0;
  Maps m;
  memset(&m, 0, sizeof(m));
  const int64_t Tm = T > 0 ? T : 1;
  if (!make_map_3d(&m.q, q, (int64_t)H * dk, Tm, B, ld_q, 64) || !make_map_3d(&m.k, k, (int64_t)H * dk, Tm, B, ld_k, 64) ||
      !make_map_3d(&m.v, v, (int64_t)H * dv, Tm, B, ld_v, 64))
    return record_cuda_error(cudaErrorInvalidValue);
  Args a{};
  a.log_alpha = log_alpha;
  a.beta = beta;
  a.S0 = S0;
  a.T = T;
  a.H = H;
  a.dv = dv;
  a.l2norm = (flags & GDN_DR_L2NORM_QK) ? 1 : 0;
  a.nseg = 1;
  a.T_seg = Tm;
  a.st_last_only = 0;
  a.dv_state = dv;
  a.zero_splits = 0;
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
  const SegPlan pl = plan_segments(B, T, H, dv, sms);
  const size_t need_seg = seg_bytes(B, H, dv, pl.P);
  const bool ws_ok = ws && aligned(ws, 256);
  // the inverse pre-pass, when the sequences are cut into segments and the
  // workspace holds every chunk's image
  if (pl.P > 1 && ws_ok && ws_bytes >= need_seg + img_bytes(B, T, H)) {
    a.nch_T = (T + C - 1) / C;
    uint8_t* img = static_cast<uint8_t*>(ws) + need_seg;
    a.xinv = img;
    const int st = launch_inverse(a, m, img, B, stream);
    if (st) return st;
  }
  if (pl.P > 1 && ws_ok && ws_bytes >= need_seg) {
    float* MB = static_cast<float*>(ws);
    float* E = reinterpret_cast<float*>(static_cast<uint8_t*>(ws) + align256(seg_bytes_mb(B, H, dv, pl.P)));
    // phase A: segments 0 .. P-2 from [I | 0]; the state transition and the
    // zero-start state of each, no o
    Args pa = a;
    pa.nseg = pl.P - 1;
    pa.T_seg = pl.T_seg;
    pa.S0 = nullptr;
    pa.S_T = MB;
    pa.dv_state = DK + dv;
    pa.zero_splits = 1;
    pa.nsplit = 1 + dv / 128;
    pa.o = nullptr;
    pa.o_amax = nullptr;
    pa.oq_codes = nullptr;
    int st = launch_args(pa, m, B * (pl.P - 1) * H, 128, f32, stream);
    if (st) return st;
    // phase B: the entry state of every segment
    cudaError_t ce =
        cudaFuncSetAttribute(segment_combine_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)CMB_SMEM);
    if (ce != cudaSuccess) return record_cuda_error(ce);
    segment_combine_kernel<<<(unsigned)(B * H * (dv / 16)), 256, CMB_SMEM, stream>>>(MB, S0, E, H, dv, pl.P);
    st = check_launch();
    if (st) return st;
    // phase C: every segment from its entry state
    Args pc = a;
    pc.nseg = pl.P;
    pc.T_seg = pl.T_seg;
    pc.S0 = E;
    pc.st_last_only = 1;
    pc.nsplit = dv / 128;
    return launch_args(pc, m, B * pl.P * H, 128, f32, stream);
  }
  // one piece per sequence: d_v slices of 128 columns unless the chains leave
  // more than half the SMs idle
  int dvs = (dv % 128 == 0) ? 128 : 64;
  if (dvs == 128 && chains * (dv / 128) * 2 <= sms) dvs = 64;
  a.nsplit = dv / dvs;
  return launch_args(a, m, chains, dvs, f32, stream);
}

}  // namespace gdn
