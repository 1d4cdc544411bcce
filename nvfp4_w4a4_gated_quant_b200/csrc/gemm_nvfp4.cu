// Block-scaled NVFP4 GEMM on the 5th-generation tensor cores (sm_100a).
//
// Y[m, n] = g_a * g_b(seg(n)) * sum_k e2m1(A[m,k]) sa[m,k/16] e2m1(B[n,k]) sb[n,k/16]
//
// Method: every projection of the W4A4 Gated DeltaNet layer, gate projections
// included ("Why Gated DeltaNet Survives 4-Bit Quantization", section
// "Performance and Efficiency Gains"), with one decode scale per fused column
// segment (section "Critical Lessons for Model Serving": modules scaled
// separately must not share one global scale inside a fused kernel).
//
// Design (one CTA per SM, persistent over 128 x 256 output tiles, N fastest:
// the CTAs in flight share a few 128-row blocks of A and sweep all of B, so
// each A block is read from DRAM once and B stays resident in L2; with M
// fastest the layer's 84 MB activation operand was re-read per column block):
//   warp 0        TMA producer: A tile 128 x 256 fp4 and B tile 256 x 256 fp4
//                 (128-byte rows, 128B swizzle) plus the E4M3 scale blocks
//                 they need (untiled bulk copies of the tensor-core scale
//                 layout) into a 4-stage shared-memory ring.  The scale
//                 copies complete on their own barrier, ahead of the 48 KB of
//                 operand tiles.  No multicast.
//   warps 12..15  scale loaders, one per 32-lane TMEM quarter: as soon as a
//                 stage's scales land they read them from shared memory into
//                 registers, then, once one of five TMEM scale buffers is
//                 free, write them with tcgen05.st, replicated into the four
//                 quarters (the layout the block-scaled MMA reads), while the
//                 operand tiles are still in flight.  Warp stores keep these
//                 copies off the MMA pipe, where tcgen05.cp serialises with
//                 the MMAs.
//   warp 1        TMEM owner and MMA issuer:
//                 tcgen05.mma.kind::mxf4nvf4.block_scale.block16 (M=128,
//                 N=256, K=64) into a 128 x 256 FP32 accumulator in TMEM;
//                 tcgen05.commit frees smem stages, scale buffers and tiles.
//                 (The MMA's shared-memory operand reads plus the TMA writes
//                 come close to the SM's shared-memory bandwidth; the widest
//                 N tile re-reads A the least.)
//   warps 4..11   epilogue: tcgen05.ld of 32-column slices with the
//                 per-segment scale (g_a * g_b, precomputed into a
//                 shared-memory segment table at kernel start).  When a
//                 warp's 128 columns lie in one bf16 segment they are packed
//                 to bf16 in registers, the accumulator is released at once
//                 and the stores overlap the next tile's MMAs; other tiles
//                 (segment edges, gates, FP32 outputs) take the per-column
//                 path and release after their last load.
// TMEM: accumulator at columns 0..255, scale buffers at 256 + 48b.
// Every mbarrier wait is bounded; a wait that runs out records
// GDN_ERR_TIMEOUT, raises a CTA-wide abort flag and every role drains out.
#include <cstring>


#include "common.cuh"
#include "gate_math.cuh"
#include "kernels.h"
#include "tmap.cuh"

namespace gdn {
namespace {

constexpr int BM = 128;
constexpr int BN = 256;
constexpr int BK = 256;                 // fp4 elements per stage (128 bytes per row)
constexpr int KSTEP = 64;               // K of one MMA
#ifndef GDN_GEMM_TMA_STORE
#define GDN_GEMM_TMA_STORE 1
#endif
#ifndef GDN_GEMM_STAGES
#define GDN_GEMM_STAGES (GDN_GEMM_TMA_STORE ? 3 : 4)
#endif
constexpr int STAGES = GDN_GEMM_STAGES;
constexpr bool TMA_STORE = GDN_GEMM_TMA_STORE != 0;
constexpr int A_BYTES = BM * BK / 2;    // 16 KiB
constexpr int B_BYTES = BN * BK / 2;    // 32 KiB
constexpr int NUM_THREADS = 512;
constexpr int EPI_WARP0 = 4;
constexpr int NUM_EPI_WARPS = 8;
constexpr int SF_WARP0 = 12;            // warps 12..15: scale loaders
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t ACC_COL = 0;         // one accumulator of BN FP32 columns
constexpr int SF_NBUF = 5;
constexpr uint32_t SF_COL = BN;         // five buffers of 48 columns:
constexpr uint32_t SF_BUF = 48;         //   +0: A, 4 k-steps x 4; +16: B, 4 k-steps x 8
constexpr uint32_t SFB_OFF = 16;
constexpr uint32_t SFB_PER_K = BN / 32;
static_assert(SF_COL + SF_NBUF * SF_BUF <= TMEM_COLS, "TMEM budget");

struct SegSmem {
  int n_begin, n_end, kind;
  int tma;                // bf16 segment with an output tensor map
  float alpha;            // g_a * g_b of the segment
  int64_t ld_out;
  void* out;
  const float* A_log;
  const float* dt_bias;
};

constexpr int SFA_BYTES = (BK / KSTEP) * 512;      // 2 KiB
constexpr int SFB_BYTES = 2 * (BK / KSTEP) * 512;  // two 128-row scale blocks, 4 KiB

// Epilogue staging for TMA stores: one 32-row x 64-column bf16 box (4 KiB,
// 128-byte swizzle) per epilogue warp.
constexpr int STG_BYTES = 32 * 64 * 2;
constexpr int STAGING_BYTES = TMA_STORE ? NUM_EPI_WARPS * STG_BYTES : 0;

constexpr size_t SMEM_BYTES = 1024 /*alignment slack*/ +
                              (size_t)STAGES * (A_BYTES + B_BYTES + SFA_BYTES + SFB_BYTES) + STAGING_BYTES + 512 +
                              GDN_MAX_SEGMENTS * sizeof(SegSmem);
static_assert(SMEM_BYTES <= 232448, "shared memory budget");

// Output tensor maps of the bf16 segments (TMA-store epilogue).
struct OutMaps {
  CUtensorMap m[GDN_MAX_SEGMENTS];
};

struct Segment {
  int n_begin, n_end, kind, tma;
  const float* g_b;
  void* out;
  int64_t ld_out;
  const float* A_log;
  const float* dt_bias;
};

struct Params {
  int M, N, K;
  int num_m, num_n, num_tiles;
  int kc;                      // K / 64: scale blocks per 128-row block
  const uint8_t* sfa;
  const uint8_t* sfb;
  const float* g_a;
  int n_segs;
  Segment segs[GDN_MAX_SEGMENTS];
  int* status;
};

// K-major operand in 128-byte swizzled rows, 8-row core groups 1024 B apart.
__device__ __forceinline__ uint64_t desc_sw128(uint32_t saddr) {
  uint64_t d = (uint64_t)((saddr >> 4) & 0x3FFFu);
  d |= (uint64_t)1 << 16;                 // leading byte offset (unused when swizzled)
  d |= (uint64_t)(1024 >> 4) << 32;       // stride byte offset
  d |= (uint64_t)1 << 46;                 // descriptor version (sm_100)
  d |= (uint64_t)2 << 61;                 // 128-byte swizzle
  return d;
}
// Instruction descriptor: E2M1 x E2M1, UE4M3 scales, FP32 accumulate,
// both operands K-major, M = 128, N = BN, dense, K = 64.
constexpr uint32_t kIdesc = (1u << 7) | (1u << 10) | ((uint32_t)(BN >> 3) << 17) | ((uint32_t)(BM >> 4) << 24);

__device__ __forceinline__ bool wait_or_abort(uint64_t* bar, uint32_t parity, int* status, volatile int* abort_flag) {
  for (uint32_t i = 0; i < kWaitLimit; ++i) {
    if (mbar_try_wait(bar, parity)) return true;
    if (*abort_flag) return false;
    if (i > 64) __nanosleep(32);
  }
  report_status(status, GDN_ERR_TIMEOUT);
  *abort_flag = 1;
  return false;
}

// Warp-collective wait, used by every role.  Every lane polls the same
// barrier and abort flag with the same counter, so a converged warp leaves
// the loop together and no vote follows.  On 8192 x 12288 x 5120: a vote
// after each wait in the MMA warp cost 6%, lane 0 polling and a shuffle 23%;
// the scale loaders and the epilogue moving from lane-0 polling to this form
// took the kernel from 252-255 to 235 us.
__device__ __forceinline__ bool wait_or_abort_warp(uint64_t* bar, uint32_t parity, int* status,
                                                   volatile int* abort_flag) {
  return wait_or_abort(bar, parity, status, abort_flag);
}

__device__ __forceinline__ int find_segment(const SegSmem* segs, int n_segs, int n) {
  int s = 0;
#pragma unroll 1
  while (s + 1 < n_segs && n >= segs[s].n_end) ++s;
  return s;
}

__device__ __forceinline__ void epilogue_store_one(const SegSmem& sg, int m, int n, float y) {
  const int64_t off = (int64_t)m * sg.ld_out + (n - sg.n_begin);
  switch (sg.kind) {
    case GDN_EPI_STORE_BF16:
      reinterpret_cast<uint16_t*>(sg.out)[off] = (uint16_t)f32_to_bf16_bits(y);
      break;
    case GDN_EPI_STORE_F32:
      reinterpret_cast<float*>(sg.out)[off] = y;
      break;
    case GDN_EPI_LOG_ALPHA: {
      const int j = n - sg.n_begin;
      reinterpret_cast<float*>(sg.out)[off] = gate_log_alpha(y, sg.A_log[j], sg.dt_bias[j]);
      break;
    }
    default:
      reinterpret_cast<float*>(sg.out)[off] = gate_beta(y);
      break;
  }
}

__device__ __forceinline__ void tma_store_2d(const void* tmap, uint32_t src, int32_t c0, int32_t c1) {
  asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%2, %3}], [%1];" ::"l"(tmap), "r"(src),
               "r"(c0), "r"(c1)
               : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_read0() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait0() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }
__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
  asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c), "r"(d) : "memory");
}

__device__ __forceinline__ uint32_t word(const uint4& v, int i) {
  return i == 0 ? v.x : i == 1 ? v.y : i == 2 ? v.z : v.w;
}

__global__ void __launch_bounds__(NUM_THREADS, 1)
gemm_nvfp4_kernel(const __grid_constant__ CUtensorMap tmap_a, const __grid_constant__ CUtensorMap tmap_b,
                  const __grid_constant__ Params p, const __grid_constant__ OutMaps om) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  uint8_t* sA = smem;
  uint8_t* sB = sA + STAGES * A_BYTES;
  uint8_t* sSFA = sB + STAGES * B_BYTES;
  uint8_t* sSFB = sSFA + STAGES * SFA_BYTES;
  uint8_t* staging = sSFB + STAGES * SFB_BYTES;   // 1024-aligned: every stage size is a multiple of 1 KiB
  SegSmem* segs = reinterpret_cast<SegSmem*>(staging + STAGING_BYTES);
  uint64_t* full = reinterpret_cast<uint64_t*>(segs + GDN_MAX_SEGMENTS);
  uint64_t* empty = full + STAGES;
  uint64_t* sf_land = empty + STAGES;      // [STAGES] a stage's scale copies have landed
  uint64_t* sf_full = sf_land + STAGES;    // [SF_NBUF] a TMEM scale buffer is filled
  uint64_t* sf_free = sf_full + SF_NBUF;   // [SF_NBUF] the MMAs that read a buffer are done
  uint64_t* acc_full = sf_free + SF_NBUF;
  uint64_t* acc_empty = acc_full + 1;
  uint32_t* tmem_ptr = reinterpret_cast<uint32_t*>(acc_empty + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_ptr + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
      mbar_init(&sf_land[s], 1);
    }
    for (int b = 0; b < SF_NBUF; ++b) {
      mbar_init(&sf_full[b], 4);
      mbar_init(&sf_free[b], 1);
    }
    mbar_init(acc_full, 1);
    mbar_init(acc_empty, NUM_EPI_WARPS);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (threadIdx.x < p.n_segs) {
    const Segment& g = p.segs[threadIdx.x];
    SegSmem& d = segs[threadIdx.x];
    d.n_begin = g.n_begin;
    d.n_end = g.n_end;
    d.kind = g.kind;
    d.tma = g.tma;
    d.alpha = __fmul_rn(*p.g_a, *g.g_b);
    d.ld_out = g.ld_out;
    d.out = g.out;
    d.A_log = g.A_log;
    d.dt_bias = g.dt_bias;
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tmap_a);
    prefetch_tmap(&tmap_b);
  }
  if (TMA_STORE && warp == EPI_WARP0 && lane < p.n_segs && p.segs[lane].tma) prefetch_tmap(&om.m[lane]);
  if (warp == 1) {
    tmem_alloc(tmem_ptr, TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_ptr;
  const int n_segs = p.n_segs;

  const int num_kb = (p.K + BK - 1) / BK;
  const int ksteps_total = p.K / KSTEP;
  const int sf_blocks_n = (p.N + 127) / 128;

  if (warp == 0) {
    // ------------------------------------------------------- producer
    // The whole warp runs this loop; one elected lane issues each copy.
    uint32_t it = 0;
    uint32_t last_round[STAGES];
    bool issued[STAGES];
    for (int s = 0; s < STAGES; ++s) issued[s] = false, last_round[s] = 0;
    bool ok = true;
    for (int tile = blockIdx.x; ok && tile < p.num_tiles; tile += gridDim.x) {
      const int mb = tile / p.num_n, nb = tile % p.num_n;
      const int b0 = (nb * BN) / 128;                 // first 128-row scale block of B
      const int nh = min(2, sf_blocks_n - b0);
      for (int kb = 0; kb < num_kb; ++kb, ++it) {
        const int s = it % STAGES;
        const uint32_t round = it / STAGES;
        if (!wait_or_abort_warp(&empty[s], (round & 1) ^ 1, p.status, abort_flag)) { ok = false; break; }
        const int nks = min(BK / KSTEP, ksteps_total - kb * (BK / KSTEP));
        mbar_arrive_expect_tx_warp(&full[s], A_BYTES + B_BYTES);
        tma_load_2d_warp(sA + s * A_BYTES, &tmap_a, &full[s], kb * (BK / 2), mb * BM);
        tma_load_2d_warp(sB + s * B_BYTES, &tmap_b, &full[s], kb * (BK / 2), nb * BN);
        // the stage's scales after its operand tiles (248 -> 246 us)
        mbar_arrive_expect_tx_warp(&sf_land[s], (uint32_t)nks * 512u * (1u + (uint32_t)nh));
        bulk_load_warp(sSFA + s * SFA_BYTES, p.sfa + ((int64_t)mb * p.kc + kb * 4) * 512, nks * 512, &sf_land[s]);
        for (int h = 0; h < nh; ++h)
          bulk_load_warp(sSFB + s * SFB_BYTES + h * 2048, p.sfb + ((int64_t)(b0 + h) * p.kc + kb * 4) * 512,
                         nks * 512, &sf_land[s]);
        issued[s] = true;
        last_round[s] = round;
      }
    }
    // Drain: every copy this warp issued lands before the CTA exits.
    for (int s = 0; s < STAGES; ++s)
      if (issued[s]) {
        for (uint32_t i = 0; i < kWaitLimit && !mbar_try_wait(&full[s], last_round[s] & 1); ++i) __nanosleep(32);
        for (uint32_t i = 0; i < kWaitLimit && !mbar_try_wait(&sf_land[s], last_round[s] & 1); ++i) __nanosleep(32);
      }
    __syncwarp();
  } else if (warp >= SF_WARP0) {
    // ------------------------------------------------------- scale loaders
    // Warp w writes TMEM lanes 32*(w%4) .. +31.  For k-step j, column c of
    // the A part holds in lane l the four scales of row (l%32) + 32c: the
    // 16 bytes at (l%32)*16 of the k-step's 512-byte block.  The B part has
    // BN/32 columns; its rows 32c + l of the tile form 32-row group
    // g = nb*BN/32 + c, which sits in scale block g/4 (relative to the first
    // block the tile touches) as word g%4 of the lane's 16 bytes.
    const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
    uint32_t it = 0;
    bool ok = true;
    for (int tile = blockIdx.x; ok && tile < p.num_tiles; tile += gridDim.x) {
      for (int kb = 0; kb < num_kb; ++kb, ++it) {
        const int s = it % STAGES;
        const uint32_t buf = it % SF_NBUF;
        if (!wait_or_abort_warp(&sf_land[s], (it / STAGES) & 1, p.status, abort_flag)) { ok = false; break; }
        const uint4* fa = reinterpret_cast<const uint4*>(sSFA + s * SFA_BYTES) + lane;
        const uint4* fb = reinterpret_cast<const uint4*>(sSFB + s * SFB_BYTES) + lane;
        uint32_t ra[16], rb[16], rc[16];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const uint4 a4 = fa[j * 32];
          ra[4 * j + 0] = a4.x; ra[4 * j + 1] = a4.y; ra[4 * j + 2] = a4.z; ra[4 * j + 3] = a4.w;
        }
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const uint4 x0 = fb[j * 32];          // block 0, k-step j
          const uint4 x1 = fb[128 + j * 32];    // block 1, k-step j
#pragma unroll
          for (int c = 0; c < (int)SFB_PER_K; ++c) {
            const uint32_t v = word(c < 4 ? x0 : x1, c & 3);   // tile starts on a scale block
            const int idx = j * SFB_PER_K + c;
            if (idx < 16) rb[idx] = v; else rc[idx - 16] = v;
          }
        }
        if (!wait_or_abort_warp(&sf_free[buf], ((it / SF_NBUF) & 1) ^ 1, p.status, abort_flag)) { ok = false; break; }
        tc_fence_after();
        const uint32_t col = tmem + lane_base + SF_COL + buf * SF_BUF;
        tmem_st_32x32b_x16(col, ra);
        tmem_st_32x32b_x16(col + SFB_OFF, rb);
        tmem_st_32x32b_x16(col + SFB_OFF + 16, rc);
        tc_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&sf_full[buf]);
      }
    }
  } else if (warp == 1) {
    // --------------------------------------------------------- MMA issuer
    // The whole warp runs this loop (every lane polls the same barriers);
    // one elected lane issues each MMA and commit.
    uint32_t it = 0, tile_iter = 0;
    bool ok = true;
    for (int tile = blockIdx.x; ok && tile < p.num_tiles; tile += gridDim.x, ++tile_iter) {
      if (!wait_or_abort_warp(acc_empty, (tile_iter & 1) ^ 1, p.status, abort_flag)) { ok = false; break; }
      tc_fence_after();
      const uint32_t acc = tmem + ACC_COL;
      for (int kb = 0; kb < num_kb; ++kb, ++it) {
        const int s = it % STAGES;
        const uint32_t buf = it % SF_NBUF;
        if (!wait_or_abort_warp(&full[s], (it / STAGES) & 1, p.status, abort_flag) ||
            !wait_or_abort_warp(&sf_full[buf], (it / SF_NBUF) & 1, p.status, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const int nks = min(BK / KSTEP, ksteps_total - kb * (BK / KSTEP));
        const uint32_t a_s = smem_u32(sA + s * A_BYTES);
        const uint32_t b_s = smem_u32(sB + s * B_BYTES);
        const uint32_t sf = tmem + SF_COL + buf * SF_BUF;
        for (int j = 0; j < nks; ++j)
          tc_mma_nvf4_warp(acc, desc_sw128(a_s + j * 32), desc_sw128(b_s + j * 32), kIdesc, sf + j * 4,
                           sf + SFB_OFF + j * SFB_PER_K, (kb > 0 || j > 0) ? 1u : 0u);
        tc_commit_warp(&empty[s]);
        tc_commit_warp(&sf_free[buf]);
      }
      if (ok) tc_commit_warp(acc_full);
    }
    __syncwarp();
  } else if (warp >= EPI_WARP0) {
    // --------------------------------------------------------- epilogue
    const int ew = warp - EPI_WARP0;
    const int quad = warp & 3;            // TMEM lanes quad*32 .. quad*32+31
    const int half = ew >> 2;             // columns half*128 .. half*128+127
    uint32_t tile_iter = 0;
    for (int tile = blockIdx.x; tile < p.num_tiles; tile += gridDim.x, ++tile_iter) {
      const int mb = tile / p.num_n, nb = tile % p.num_n;
      const int m = mb * BM + quad * 32 + lane;
      const int nw0 = nb * BN + half * 128;   // first column of this warp
      // resolve the segment before waiting: fast path when all 128 columns
      // sit in one bf16 segment with 16-byte aligned rows
      int s0 = 0;
      bool fast = false;
      if (nw0 < p.N) {
        s0 = find_segment(segs, n_segs, nw0);
        const SegSmem& sg = segs[s0];
        if (TMA_STORE)
          fast = sg.tma && nw0 + 127 < sg.n_end && nw0 + 127 < p.N;
        else
          fast = sg.kind == GDN_EPI_STORE_BF16 && nw0 + 127 < sg.n_end && nw0 + 127 < p.N && (sg.ld_out % 8) == 0 &&
                 ((reinterpret_cast<uintptr_t>(sg.out) + (int64_t)(nw0 - sg.n_begin) * 2) % 16) == 0;
      }
      if (!wait_or_abort_warp(acc_full, tile_iter & 1, p.status, abort_flag)) break;
      tc_fence_after();
      const uint32_t tbase = tmem + ((uint32_t)(quad * 32) << 16) + ACC_COL + half * 128;
      if (TMA_STORE && fast) {
        // two 64-column halves: both TMEM loads of a half in flight at once,
        // packed to bf16, staged as a 32 x 64 box and stored by TMA (rows
        // past M are clipped by the tensor map); the accumulator is released
        // once the second half is in registers
        const SegSmem& sg = segs[s0];
        const float alpha = sg.alpha;
        const uint32_t stg = smem_u32(staging + ew * STG_BYTES);
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          uint32_t r0[32], r1[32];
          tmem_ld_32x32b_x32(tbase + hh * 64, r0);
          tmem_ld_32x32b_x32(tbase + hh * 64 + 32, r1);
          tc_wait_ld();
          if (hh == 1) {
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(acc_empty);
          }
          uint32_t pk[32];   // bf16 pairs of the 64 columns
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            pk[e] = pack_bf16x2(__fmul_rn(__uint_as_float(r0[2 * e]), alpha),
                                __fmul_rn(__uint_as_float(r0[2 * e + 1]), alpha));
            pk[16 + e] = pack_bf16x2(__fmul_rn(__uint_as_float(r1[2 * e]), alpha),
                                     __fmul_rn(__uint_as_float(r1[2 * e + 1]), alpha));
          }
          if (lane == 0) bulk_wait_read0();
          __syncwarp();
#pragma unroll
          for (int c = 0; c < 8; ++c)
            st_shared_v4(stg + lane * 128 + ((c ^ (lane & 7)) << 4), pk[4 * c], pk[4 * c + 1], pk[4 * c + 2],
                         pk[4 * c + 3]);
          asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
          __syncwarp();
          if (lane == 0) {
            tma_store_2d(&om.m[s0], stg, nw0 - sg.n_begin + 64 * hh, mb * BM + quad * 32);
            bulk_commit();
          }
        }
      } else if (fast) {
        const SegSmem& sg = segs[s0];
        const float alpha = sg.alpha;
        uint32_t pk[64];
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          uint32_t r[32];
          tmem_ld_32x32b_x32(tbase + c * 32, r);
          tc_wait_ld();
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            const float y0 = __fmul_rn(__uint_as_float(r[2 * e]), alpha);
            const float y1 = __fmul_rn(__uint_as_float(r[2 * e + 1]), alpha);
            pk[c * 16 + e] = f32_to_bf16_bits(y0) | (f32_to_bf16_bits(y1) << 16);
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(acc_empty);
        if (m < p.M) {
          uint4* dst = reinterpret_cast<uint4*>(reinterpret_cast<uint16_t*>(sg.out) + (int64_t)m * sg.ld_out +
                                                (nw0 - sg.n_begin));
#pragma unroll
          for (int v = 0; v < 16; ++v) dst[v] = make_uint4(pk[4 * v], pk[4 * v + 1], pk[4 * v + 2], pk[4 * v + 3]);
        }
      } else {
#pragma unroll 1
        for (int c = 0; c < 4; ++c) {
          uint32_t r[32];
          __syncwarp();
          tmem_ld_32x32b_x32(tbase + c * 32, r);
          tc_wait_ld();
          if (c == 3) {
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(acc_empty);
          }
          const int n0 = nw0 + c * 32;
          if (m >= p.M || n0 >= p.N) continue;
#pragma unroll 1
          for (int i = 0; i < 32; ++i) {
            const int n = n0 + i;
            if (n >= p.N) break;
            const SegSmem& sgi = segs[find_segment(segs, n_segs, n)];
            epilogue_store_one(sgi, m, n, __fmul_rn(__uint_as_float(r[i]), sgi.alpha));
          }
        }
      }
    }
    // the staging buffer stays valid until the last store has read it
    if (TMA_STORE && lane == 0) bulk_wait0();
    __syncwarp();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
}

int make_codes_map(CUtensorMap* map, const uint8_t* codes, int64_t rows, int64_t K, uint32_t box_rows) {
  auto encode = tensor_map_encoder();
  if (!encode) return record_cuda_error(cudaErrorNotSupported);
  cuuint64_t dims[2] = {(cuuint64_t)(K / 2), (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)(K / 2)};
  cuuint32_t box[2] = {(cuuint32_t)(BK / 2), box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = encode(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t*>(codes), dims, strides, box, estr,
                      CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                      CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return record_cuda_error(cudaErrorInvalidValue);
  return GDN_OK;
}

// Tensor map of a bf16 output segment: [M rows, n_end - n_begin columns],
// row stride ld_out, 32 x 64 boxes with the 128-byte swizzle.  Returns false
// (the segment then takes the per-element store path) when the segment does
// not meet TMA's alignment rules.
bool make_out_map(CUtensorMap* map, const gdn_epilogue_segment_t& sg, int64_t M) {
  auto encode = tensor_map_encoder();
  if (!encode || sg.kind != GDN_EPI_STORE_BF16 || sg.n_begin % 8 != 0 || (sg.ld_out * 2) % 16 != 0 ||
      (reinterpret_cast<uintptr_t>(sg.out) % 16) != 0)
    return false;
  cuuint64_t dims[2] = {(cuuint64_t)(sg.n_end - sg.n_begin), (cuuint64_t)M};
  cuuint64_t strides[1] = {(cuuint64_t)(sg.ld_out * 2)};
  cuuint32_t box[2] = {64, 32};
  cuuint32_t estr[2] = {1, 1};
  return encode(map, CU_TENSOR_MAP_DATA_TYPE_UINT16, 2, sg.out, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_NONE,
                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// The FP4 tensor-core ceiling of this GEMM's MMA: M = 128, N = 256, K = 64
// kind::mxf4nvf4 with block-16 scales, issued back to back by one converged
// warp from operand tiles resident in shared memory (E2M1 codes from a
// hash, so the multipliers see ordinary data) and scales resident in TMEM --
// no loads, no scale hand-off, no epilogue.  One CTA per SM; the GEMM's
// achieved rate divided by this rate is its efficiency against what the
// tensor pipe delivers at the clock and power of the moment.
constexpr int CEIL_THREADS = 128;
// more shared memory than two CTAs can hold on one SM: one CTA per SM (each
// allocates all of TMEM)
constexpr size_t CEIL_SMEM = 120 * 1024;
static_assert(CEIL_SMEM >= 1024 + A_BYTES + B_BYTES + 64, "ceiling tiles");

__global__ void __launch_bounds__(CEIL_THREADS, 1) fp4_mma_ceiling_kernel(int64_t iters, int* status) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t sraw = smem_u32(smem_raw);
  const uint32_t sb = (sraw + 1023u) & ~1023u;
  uint8_t* smem = smem_raw + (sb - sraw);
  uint64_t* bar = reinterpret_cast<uint64_t*>(smem + A_BYTES + B_BYTES);
  uint32_t* tmem_ptr = reinterpret_cast<uint32_t*>(smem + A_BYTES + B_BYTES + 8);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  // codes: any nibble is a valid E2M1 value
  for (int i = tid; i < (A_BYTES + B_BYTES) / 4; i += CEIL_THREADS) {
    uint32_t x = (uint32_t)i * 2654435761u + 0x9E3779B9u * (blockIdx.x + 1);
    x ^= x >> 15;
    x *= 0x2C1B3C6Du;
    x ^= x >> 12;
    reinterpret_cast<uint32_t*>(smem)[i] = x;
  }
  if (tid == 0) {
    mbar_init(bar, 1);
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(tmem_ptr, TMEM_COLS);
    tmem_relinquish();
  }
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_ptr;
  {
    // every scale 1.0 (E4M3 0x38) in the 48 columns the MMAs read
    uint32_t one[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) one[i] = 0x38383838u;
    const uint32_t col = tmem + ((uint32_t)(warp * 32) << 16) + SF_COL;
    tmem_st_32x32b_x16(col, one);
    tmem_st_32x32b_x16(col + 16, one);
    tmem_st_32x32b_x16(col + 32, one);
    tc_wait_st();
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    const uint32_t a_s = sb, b_s = sb + A_BYTES;
    const uint32_t acc = tmem + ACC_COL, sf = tmem + SF_COL;
    for (int64_t it = 0; it < iters; ++it)
#pragma unroll
      for (int j = 0; j < BK / KSTEP; ++j)
        tc_mma_nvf4_warp(acc, desc_sw128(a_s + j * 32), desc_sw128(b_s + j * 32), kIdesc, sf + j * 4,
                         sf + SFB_OFF + j * SFB_PER_K, (it > 0 || j > 0) ? 1u : 0u);
    tc_commit_warp(bar);
    mbar_wait(bar, 0, status);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
}

}  // namespace

int launch_fp4_mma_ceiling(int64_t iters, int ctas, cudaStream_t stream) {
  cudaError_t e =
      cudaFuncSetAttribute(fp4_mma_ceiling_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)CEIL_SMEM);
  if (e != cudaSuccess) return record_cuda_error(e);
  fp4_mma_ceiling_kernel<<<ctas, CEIL_THREADS, CEIL_SMEM, stream>>>(iters, device_status_word());
  return check_launch();
}

int launch_gemm_nvfp4(const gdn_nvfp4_t* A, const float* g_a, const gdn_nvfp4_t* B, int64_t M, int64_t N, int64_t K,
                      const gdn_epilogue_segment_t* segs, int n_segs, cudaStream_t stream) {
  if (M == 0 || N == 0) return GDN_OK;
  Params p{};
  p.M = (int)M;
  p.N = (int)N;
  p.K = (int)K;
  p.num_m = (int)cdiv(M, BM);
  p.num_n = (int)cdiv(N, BN);
  p.num_tiles = p.num_m * p.num_n;
  p.kc = (int)(K / 64);
  p.sfa = A->scales;
  p.sfb = B->scales;
  p.g_a = g_a;
  p.n_segs = n_segs;
  for (int i = 0; i < n_segs; ++i) {
    p.segs[i].n_begin = (int)segs[i].n_begin;
    p.segs[i].n_end = (int)segs[i].n_end;
    p.segs[i].kind = segs[i].kind;
    p.segs[i].g_b = segs[i].g_b;
    p.segs[i].out = segs[i].out;
    p.segs[i].ld_out = segs[i].ld_out;
    p.segs[i].A_log = segs[i].A_log;
    p.segs[i].dt_bias = segs[i].dt_bias;
  }
  OutMaps om;
  memset(&om, 0, sizeof(om));
  for (int i = 0; i < n_segs; ++i) p.segs[i].tma = TMA_STORE && make_out_map(&om.m[i], segs[i], M) ? 1 : 0;
  p.status = device_status_word();
  CUtensorMap ta, tb;
  int st = make_codes_map(&ta, A->codes, M, K, BM);
  if (st) return st;
  st = make_codes_map(&tb, B->codes, N, K, BN);
  if (st) return st;
  cudaError_t attr_err =
      cudaFuncSetAttribute(gemm_nvfp4_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SMEM_BYTES);
  if (attr_err != cudaSuccess) return record_cuda_error(attr_err);
  const int grid = (int)std::min<int64_t>(p.num_tiles, num_sms());
  gemm_nvfp4_kernel<<<grid, NUM_THREADS, SMEM_BYTES, stream>>>(ta, tb, p, om);
  return check_launch();
}

}  // namespace gdn
