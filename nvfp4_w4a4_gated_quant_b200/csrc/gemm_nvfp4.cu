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
// Two forms of one persistent, warp-specialised kernel (template PAIR):
//
//   PAIR (the main path, M > 128): clusters of two CTAs on two SMs share a
//   256 x 256 output tile through tcgen05.mma.cta_group::2 (M = 256).  CTA r
//   of the pair holds A rows 128r..128r+127 and B rows 128r..128r+127 of the
//   tile in its own shared memory; the pair's MMA, issued by CTA 0, reads both
//   CTAs' halves and accumulates rows 128r.. into CTA r's TMEM.  Per SM that
//   is 32 KiB of operands per 256-deep k-block instead of 48 KiB for a
//   one-SM 128 x 256 tile (the same 128 x 256 x 256 MMA work): L2 -> SM
//   traffic per FLOP drops by a third, and the smaller stages let the ring
//   hold five of them.  On this GEMM the one-SM form was bound by the L2
//   bandwidth its tile needs (94 B/cycle/SM at the MMA's rate).
//   SINGLE (M <= 128, and the fallback): one CTA, 128 x 256 tiles.
//
// Roles (512 threads, one CTA per SM; tiles walked N-fastest so the CTAs in
// flight share a few row blocks of A and sweep B, which stays in L2):
//   warp 0        TMA producer: this CTA's A and B rows of a 256-deep
//                 k-block (128-byte rows, 128B swizzle) into a shared-memory
//                 ring, plus the E4M3 scale blocks the CTA's TMEM needs
//                 (untiled bulk copies of the tensor-core scale layout: A
//                 for its own 128 rows, B for all 256 tile columns), on
//                 their own barrier ahead of the operand tiles.  No
//                 multicast: each CTA loads its own halves.
//   warp 1        CTA 0: TMEM owner and MMA issuer,
//                 tcgen05.mma.kind::mxf4nvf4.block_scale.block16 (K = 64);
//                 tcgen05.commit frees stages, scale buffers and the
//                 accumulator, multicast to both CTAs of a pair.
//                 CTA 1 of a pair: relays "my half of stage s has landed"
//                 to a barrier of CTA 0 (a remote mbarrier arrive), so that
//                 every CTA's copies complete on its own barriers.
//   warps 12..15  scale loaders, one per 32-lane TMEM quarter: read a
//                 stage's scales from shared memory and, once one of five
//                 TMEM scale buffers is free, write them with tcgen05.st,
//                 replicated into the four quarters (the layout the
//                 block-scaled MMA reads), while the operand tiles are still
//                 in flight; they arrive on CTA 0's buffer barrier.  Warp
//                 stores keep these copies off the MMA pipe, where tcgen05.cp
//                 serialises with the MMAs.
//   warps 4..11   epilogue: tcgen05.ld of 32-column slices of the CTA's
//                 accumulator rows with the per-segment scale (g_a * g_b,
//                 precomputed into a shared-memory segment table).  When a
//                 warp's 128 columns lie in one bf16 segment they are packed
//                 to bf16, staged and stored by TMA, and the accumulator is
//                 released (to CTA 0) as soon as it is in registers; other
//                 tiles (segment edges, gates, FP32 outputs) take the
//                 per-column path.
// TMEM per CTA: accumulator at columns 0..255, scale buffers at 256 + 48b.
// Every mbarrier wait is bounded; a wait that runs out records
// GDN_ERR_TIMEOUT, raises the CTA's abort flag and every role drains out.
// Before a pair exits, the issuing thread waits for its last tensor-core
// operations and both CTAs meet at a cluster barrier, so no CTA leaves while
// its peer's copies, MMAs or arrivals can still reach it.
#include <algorithm>
#include <atomic>
#include <cstring>


#include "common.cuh"
#include "gate_math.cuh"
#include "kernels.h"
#include "tmap.cuh"

namespace gdn {
namespace {

constexpr int BM = 128;                 // accumulator rows per CTA
constexpr int BN = 256;
constexpr int BK = 256;                 // fp4 elements per stage (128 bytes per row)
constexpr int KSTEP = 64;               // K of one MMA
constexpr int A_BYTES = BM * BK / 2;    // 16 KiB
constexpr int B_BYTES = BN * BK / 2;    // 32 KiB: a full 256-row B tile
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
constexpr int STAGING_BYTES = NUM_EPI_WARPS * STG_BYTES;

template <bool PAIR>
struct Shape {
  static constexpr int TM = PAIR ? 2 * BM : BM;              // output rows of a tile
  static constexpr int B_ROWS = PAIR ? BN / 2 : BN;          // B rows one CTA loads
  static constexpr int B_CTA_BYTES = B_ROWS * BK / 2;
  static constexpr int STAGES = PAIR ? 5 : 3;
  static constexpr int STAGE_BYTES = A_BYTES + B_CTA_BYTES + SFA_BYTES + SFB_BYTES;
  static constexpr size_t SMEM = 1024 /*alignment slack*/ + (size_t)STAGES * STAGE_BYTES + STAGING_BYTES + 512 +
                                 GDN_MAX_SEGMENTS * sizeof(SegSmem);
  static_assert(SMEM <= 232448, "shared memory budget");
  static_assert((4 * STAGES + 2 * SF_NBUF + 3) * 8 + 8 <= 512, "barrier area");
};

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
  int num_m, num_n, num_tiles;  // tiles of Shape::TM x BN
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
// both operands K-major, N = BN, dense, K = 64; M = 128 (one CTA) or 256
// (a CTA pair).
constexpr uint32_t idesc_nvf4(int m) {
  return (1u << 7) | (1u << 10) | ((uint32_t)(BN >> 3) << 17) | ((uint32_t)(m >> 4) << 24);
}
constexpr uint32_t kIdesc = idesc_nvf4(BM);

// ---- cluster (CTA pair) primitives
__device__ __forceinline__ uint32_t cluster_ctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
// shared::cluster address of this CTA's shared-memory word `p` as seen in CTA
// `rank` of the cluster (the same offset there)
__device__ __forceinline__ uint32_t cluster_addr(const void* p, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(smem_u32(p)), "r"(rank));
  return r;
}
// Arrive on a barrier of another CTA of the cluster (a shared::cluster
// address).  What it publishes is either tensor-core state the arriving
// thread has already waited for (tcgen05.wait::st / ::ld, then
// tcgen05.fence::before_thread_sync) or copies whose completion it has
// observed on its own barrier; the MMAs that the arrival releases read them
// through the async proxy.
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t caddr) {
  asm volatile("mbarrier.arrive.shared::cluster.b64 _, [%0];" ::"r"(caddr) : "memory");
}
__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// ---- tcgen05 of a CTA pair (every tcgen05 allocation, MMA and commit of
// the pair kernel uses cta_group::2)
__device__ __forceinline__ void tmem_alloc_pair(uint32_t* dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst_smem)),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish_pair() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tc_mma_nvf4_pair_warp(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                                      uint32_t sfa_tmem, uint32_t sfb_tmem, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p, e;\n\t"
      "elect.sync _|e, 0xffffffff;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "@e tcgen05.mma.cta_group::2.kind::mxf4nvf4.block_scale.block16 [%0], %1, %2, %3, [%5], [%6], p;\n\t}" ::"r"(
          d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(sfa_tmem), "r"(sfb_tmem)
      : "memory");
}
// Arrive on the barrier at this offset in every CTA of `mask` once the pair
// MMAs issued so far by this thread have completed.
__device__ __forceinline__ void tc_commit_pair_warp(uint64_t* bar, uint16_t mask) {
  asm volatile(
      "{\n\t.reg .pred e;\n\t"
      "elect.sync _|e, 0xffffffff;\n\t"
      "@e tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;\n\t}" ::"r"(
          smem_u32(bar)),
      "h"(mask)
      : "memory");
}

// Bounded wait (warp-collective: every lane polls the same barrier and
// abort flag with the same counter, so a converged warp leaves the loop
// together and no vote follows).
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

template <bool PAIR>
__global__ void __launch_bounds__(NUM_THREADS, 1)
gemm_nvfp4_kernel(const __grid_constant__ CUtensorMap tmap_a, const __grid_constant__ CUtensorMap tmap_b,
                  const __grid_constant__ Params p, const __grid_constant__ OutMaps om) {
  using S = Shape<PAIR>;
  constexpr int STAGES = S::STAGES;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  uint8_t* sA = smem;
  uint8_t* sB = sA + STAGES * A_BYTES;
  uint8_t* sSFA = sB + STAGES * S::B_CTA_BYTES;
  uint8_t* sSFB = sSFA + STAGES * SFA_BYTES;
  uint8_t* staging = sSFB + STAGES * SFB_BYTES;   // 1024-aligned: every stage size is a multiple of 1 KiB
  SegSmem* segs = reinterpret_cast<SegSmem*>(staging + STAGING_BYTES);
  uint64_t* full = reinterpret_cast<uint64_t*>(segs + GDN_MAX_SEGMENTS);
  uint64_t* empty = full + STAGES;
  uint64_t* pfull = empty + STAGES;        // [STAGES] pair, CTA 0: stage s of both CTAs is ready (see below)
  uint64_t* sf_land = pfull + STAGES;      // [STAGES] a stage's scale copies have landed
  uint64_t* sf_full = sf_land + STAGES;    // [SF_NBUF] a TMEM scale buffer is filled
  uint64_t* sf_free = sf_full + SF_NBUF;   // [SF_NBUF] the MMAs that read a buffer are done
  uint64_t* acc_full = sf_free + SF_NBUF;
  uint64_t* acc_empty = acc_full + 1;
  uint64_t* mma_done = acc_empty + 1;      // the issuer's last tensor-core operations
  uint32_t* tmem_ptr = reinterpret_cast<uint32_t*>(mma_done + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_ptr + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = PAIR ? cluster_ctarank() : 0u;
  const int cid = PAIR ? (int)(blockIdx.x >> 1) : (int)blockIdx.x;   // cluster dims (2, 1, 1)
  const int ncl = PAIR ? (int)(gridDim.x >> 1) : (int)gridDim.x;
  constexpr uint16_t kBoth = 0x3;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      // a pair's MMA warp waits on one barrier per k-block (each check costs
      // the issuing warp ~150 cycles): CTA 0's own operand tiles complete on
      // it (its producer's arrive.expect_tx), plus the peer's relay and the
      // eight scale loaders of both CTAs
      mbar_init(&pfull[s], 10);
      mbar_init(&empty[s], 1);
      mbar_init(&sf_land[s], 1);
    }
    for (int b = 0; b < SF_NBUF; ++b) {
      mbar_init(&sf_full[b], PAIR ? 8 : 4);
      mbar_init(&sf_free[b], 1);
    }
    mbar_init(acc_full, 1);
    mbar_init(acc_empty, PAIR ? 2 * NUM_EPI_WARPS : NUM_EPI_WARPS);
    mbar_init(mma_done, 1);
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
  if (warp == EPI_WARP0 && lane < p.n_segs && p.segs[lane].tma) prefetch_tmap(&om.m[lane]);
  if (warp == 1) {
    if (PAIR) {
      tmem_alloc_pair(tmem_ptr, TMEM_COLS);
      tmem_relinquish_pair();
    } else {
      tmem_alloc(tmem_ptr, TMEM_COLS);
      tmem_relinquish();
    }
  }
  tc_fence_before();
  __syncthreads();
  if (PAIR) cluster_sync_all();    // the peer's barriers are initialised before any remote arrive
  tc_fence_after();
  const uint32_t tmem = *tmem_ptr;
  const int n_segs = p.n_segs;

  const int num_kb = (p.K + BK - 1) / BK;
  const int ksteps_total = p.K / KSTEP;
  const int sf_blocks_n = (p.N + 127) / 128;
  // TMEM scale buffers in use: a pair ties them to the stages (one commit per
  // k-block frees both; a cta_group::2 commit costs the MMA pipe ~9%)
  constexpr int NBUF = PAIR ? STAGES : SF_NBUF;
  static_assert(NBUF <= SF_NBUF, "TMEM scale buffers");

  if (warp == 0) {
    // ------------------------------------------------------- producer
    // The whole warp runs this loop; one elected lane issues each copy.
    uint32_t it = 0;   // k-blocks issued
    // the barrier the operand tiles complete on: CTA 0 of a pair counts them
    // into the MMA warp's one barrier
    uint64_t* opbar = PAIR && rank == 0 ? pfull : full;
    bool ok = true;
    for (int tile = cid; ok && tile < p.num_tiles; tile += ncl) {
      const int mb = tile / p.num_n, nb = tile % p.num_n;
      const int a_row = mb * S::TM + (int)rank * BM;          // this CTA's A rows
      const int b_row = nb * BN + (int)rank * S::B_ROWS;      // this CTA's B rows
      // rows of a pair's second half can lie wholly past M or N: nothing to
      // load (the MMA then reads stale data into rows or columns that the
      // epilogue never stores)
      const bool a_live = a_row < p.M, b_live = b_row < p.N;
      const int b0 = (nb * BN) / 128;                 // first 128-row scale block of B
      const int nh = min(2, sf_blocks_n - b0);
      for (int kb = 0; kb < num_kb; ++kb, ++it) {
        const int s = it % STAGES;
        const uint32_t round = it / STAGES;
        if (!wait_or_abort(&empty[s], (round & 1) ^ 1, p.status, abort_flag)) { ok = false; break; }
        const int nks = min(BK / KSTEP, ksteps_total - kb * (BK / KSTEP));
        mbar_arrive_expect_tx_warp(&opbar[s], (a_live ? A_BYTES : 0) + (b_live ? S::B_CTA_BYTES : 0));
        if (a_live) tma_load_2d_warp(sA + s * A_BYTES, &tmap_a, &opbar[s], kb * (BK / 2), a_row);
        if (b_live) tma_load_2d_warp(sB + s * S::B_CTA_BYTES, &tmap_b, &opbar[s], kb * (BK / 2), b_row);
        // the stage's scales after its operand tiles (248 -> 246 us)
        mbar_arrive_expect_tx_warp(&sf_land[s], (uint32_t)nks * 512u * ((a_live ? 1u : 0u) + (uint32_t)nh));
        if (a_live)
          bulk_load_warp(sSFA + s * SFA_BYTES, p.sfa + ((int64_t)(a_row / 128) * p.kc + kb * 4) * 512, nks * 512,
                         &sf_land[s]);
        for (int h = 0; h < nh; ++h)
          bulk_load_warp(sSFB + s * SFB_BYTES + h * 2048, p.sfb + ((int64_t)(b0 + h) * p.kc + kb * 4) * 512,
                         nks * 512, &sf_land[s]);
      }
    }
    // Drain: every copy this warp issued lands before the CTA exits (the
    // last of the `it` k-blocks that went to stage s is of round
    // (it - 1 - s) / STAGES).
    for (uint32_t s = 0; s < (uint32_t)STAGES && s < it; ++s) {
      const uint32_t last_round = (it - 1 - s) / STAGES;
      for (uint32_t i = 0; i < kWaitLimit && !mbar_try_wait(&opbar[s], last_round & 1); ++i) __nanosleep(32);
      for (uint32_t i = 0; i < kWaitLimit && !mbar_try_wait(&sf_land[s], last_round & 1); ++i) __nanosleep(32);
    }
    __syncwarp();
  } else if (warp >= SF_WARP0) {
    // ------------------------------------------------------- scale loaders
    // Warp w writes TMEM lanes 32*(w%4) .. +31.  For k-step j, column c of
    // the A part holds in lane l the four scales of row (l%32) + 32c: the
    // 16 bytes at (l%32)*16 of the k-step's 512-byte block.  The B part has
    // BN/32 columns; its rows 32c + l of the tile form 32-row group
    // g = nb*BN/32 + c, which sits in scale block g/4 (relative to the first
    // block the tile touches) as word g%4 of the lane's 16 bytes.  In a pair
    // each CTA holds the A scales of its own rows and the B scales of all
    // 256 tile columns: the layout the pair MMA reads from both TMEMs.
    const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
    uint32_t it = 0;
    bool ok = true;
    for (int tile = cid; ok && tile < p.num_tiles; tile += ncl) {
      for (int kb = 0; kb < num_kb; ++kb, ++it) {
        const int s = it % STAGES;
        const uint32_t buf = it % NBUF;
        if (!wait_or_abort(&sf_land[s], (it / STAGES) & 1, p.status, abort_flag)) { ok = false; break; }
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
        if (!wait_or_abort(PAIR ? &empty[buf] : &sf_free[buf], ((it / NBUF) & 1) ^ 1, p.status, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t col = tmem + lane_base + SF_COL + buf * SF_BUF;
        tmem_st_32x32b_x16(col, ra);
        tmem_st_32x32b_x16(col + SFB_OFF, rb);
        tmem_st_32x32b_x16(col + SFB_OFF + 16, rc);
        tc_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          if (PAIR)
            mbar_arrive_cluster(cluster_addr(&pfull[buf], 0));   // buf == stage in a pair
          else
            mbar_arrive(&sf_full[buf]);
        }
      }
    }
  } else if (warp == 1 && PAIR && rank != 0) {
    // ------------------------------------------------ relay (pair, CTA 1)
    uint32_t it = 0;
    bool ok = true;
    for (int tile = cid; ok && tile < p.num_tiles; tile += ncl) {
      for (int kb = 0; kb < num_kb; ++kb, ++it) {
        const int s = it % STAGES;
        if (!wait_or_abort(&full[s], (it / STAGES) & 1, p.status, abort_flag)) { ok = false; break; }
        __syncwarp();
        if (lane == 0) mbar_arrive_cluster(cluster_addr(&pfull[s], 0));
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // --------------------------------------------------------- MMA issuer
    // The whole warp runs this loop (every lane polls the same barriers);
    // one elected lane issues each MMA and commit.
    constexpr uint32_t idesc = idesc_nvf4(S::TM);
    uint32_t it = 0, tile_iter = 0;
    bool ok = true, any = false;
    for (int tile = cid; ok && tile < p.num_tiles; tile += ncl, ++tile_iter) {
      if (!wait_or_abort(acc_empty, (tile_iter & 1) ^ 1, p.status, abort_flag)) { ok = false; break; }
      tc_fence_after();
      const uint32_t acc = tmem + ACC_COL;
      for (int kb = 0; kb < num_kb; ++kb, ++it) {
        const int s = it % STAGES;
        const uint32_t buf = it % NBUF;
        if (PAIR ? !wait_or_abort(&pfull[s], (it / STAGES) & 1, p.status, abort_flag)
                 : (!wait_or_abort(&full[s], (it / STAGES) & 1, p.status, abort_flag) ||
                    !wait_or_abort(&sf_full[buf], (it / NBUF) & 1, p.status, abort_flag))) {
          ok = false;
          break;
        }
        tc_fence_after();
        const int nks = min(BK / KSTEP, ksteps_total - kb * (BK / KSTEP));
        const uint32_t a_s = smem_u32(sA + s * A_BYTES);
        const uint32_t b_s = smem_u32(sB + s * S::B_CTA_BYTES);
        const uint32_t sf = tmem + SF_COL + buf * SF_BUF;
        for (int j = 0; j < nks; ++j) {
          if (PAIR)
            tc_mma_nvf4_pair_warp(acc, desc_sw128(a_s + j * 32), desc_sw128(b_s + j * 32), idesc, sf + j * 4,
                                  sf + SFB_OFF + j * SFB_PER_K, (kb > 0 || j > 0) ? 1u : 0u);
          else
            tc_mma_nvf4_warp(acc, desc_sw128(a_s + j * 32), desc_sw128(b_s + j * 32), idesc, sf + j * 4,
                             sf + SFB_OFF + j * SFB_PER_K, (kb > 0 || j > 0) ? 1u : 0u);
        }
        any = true;
        if (PAIR) {
          tc_commit_pair_warp(&empty[s], kBoth);   // frees the stage and its scale buffer
        } else {
          tc_commit_warp(&empty[s]);
          tc_commit_warp(&sf_free[buf]);
        }
      }
      if (ok) {
        if (PAIR)
          tc_commit_pair_warp(acc_full, kBoth);
        else
          tc_commit_warp(acc_full);
      }
    }
    // every MMA and commit of this thread has completed before TMEM is freed
    // or the pair parts (they read the peer's shared memory and arrive on
    // its barriers)
    if (any) {
      if (PAIR)
        tc_commit_pair_warp(mma_done, 0x1);
      else
        tc_commit_warp(mma_done);
      for (uint32_t i = 0; i < kWaitLimit && !mbar_try_wait(mma_done, 0); ++i) __nanosleep(32);
    }
    __syncwarp();
  } else if (warp >= EPI_WARP0 && warp < EPI_WARP0 + NUM_EPI_WARPS) {
    // --------------------------------------------------------- epilogue
    const int ew = warp - EPI_WARP0;
    const int quad = warp & 3;            // TMEM lanes quad*32 .. quad*32+31
    const int half = ew >> 2;             // columns half*128 .. half*128+127
    uint32_t tile_iter = 0;
    for (int tile = cid; tile < p.num_tiles; tile += ncl, ++tile_iter) {
      const int mb = tile / p.num_n, nb = tile % p.num_n;
      const int mrow = mb * S::TM + (int)rank * BM + quad * 32;   // first row of this warp
      const int m = mrow + lane;
      const int nw0 = nb * BN + half * 128;   // first column of this warp
      // resolve the segment before waiting: fast path when all 128 columns
      // sit in one bf16 segment with an output tensor map
      int s0 = 0;
      bool fast = false;
      if (nw0 < p.N) {
        s0 = find_segment(segs, n_segs, nw0);
        const SegSmem& sg = segs[s0];
        fast = sg.tma && nw0 + 127 < sg.n_end && nw0 + 127 < p.N;
      }
      if (!wait_or_abort(acc_full, tile_iter & 1, p.status, abort_flag)) break;
      tc_fence_after();
      const uint32_t tbase = tmem + ((uint32_t)(quad * 32) << 16) + ACC_COL + half * 128;
      auto release = [&]() {
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          if (PAIR)
            mbar_arrive_cluster(cluster_addr(acc_empty, 0));
          else
            mbar_arrive(acc_empty);
        }
      };
      if (fast) {
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
          if (hh == 1) release();
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
          if (lane == 0 && mrow < p.M) {
            tma_store_2d(&om.m[s0], stg, nw0 - sg.n_begin + 64 * hh, mrow);
            bulk_commit();
          }
        }
      } else {
#pragma unroll 1
        for (int c = 0; c < 4; ++c) {
          uint32_t r[32];
          __syncwarp();
          tmem_ld_32x32b_x32(tbase + c * 32, r);
          tc_wait_ld();
          if (c == 3) release();
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
    if (lane == 0) bulk_wait0();
    __syncwarp();
  }

  tc_fence_before();
  __syncthreads();
  if (PAIR) cluster_sync_all();    // neither CTA leaves while the other can still reach it
  if (warp == 1) {
    tc_fence_after();
    if (PAIR)
      tmem_dealloc_pair(tmem, TMEM_COLS);
    else
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
  const int tid = threadIdx.x, warp = tid >> 5;
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


namespace {

// CTA pairs of the pair kernel that fit on the device at once (a cluster of
// two needs two free SMs of one GPC, so this can be below SMs / 2), per
// device, cached.
constexpr int kMaxDev = 64;
std::atomic<int> g_pair_clusters[kMaxDev];

int pair_clusters() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDev) return num_sms() / 2;
  int n = g_pair_clusters[dev].load(std::memory_order_relaxed);
  if (n > 0) return n;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(2 * (num_sms() / 2)), 1, 1);
  cfg.blockDim = dim3(NUM_THREADS, 1, 1);
  cfg.dynamicSmemBytes = Shape<true>::SMEM;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cudaOccupancyMaxActiveClusters(&n, gemm_nvfp4_kernel<true>, &cfg) != cudaSuccess || n <= 0) {
    (void)cudaGetLastError();
    n = num_sms() / 2;
  }
  n = std::min(n, num_sms() / 2);
  g_pair_clusters[dev].store(n, std::memory_order_relaxed);
  return n;
}

template <bool PAIR>
int launch_gemm_t(const gdn_nvfp4_t* A, const float* g_a, const gdn_nvfp4_t* B, int64_t M, int64_t N, int64_t K,
                  const gdn_epilogue_segment_t* segs, int n_segs, cudaStream_t stream) {
  using S = Shape<PAIR>;
  Params p{};
  p.M = (int)M;
  p.N = (int)N;
  p.K = (int)K;
  p.num_m = (int)cdiv(M, S::TM);
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
  for (int i = 0; i < n_segs; ++i) p.segs[i].tma = make_out_map(&om.m[i], segs[i], M) ? 1 : 0;
  p.status = device_status_word();
  CUtensorMap ta, tb;
  int st = make_codes_map(&ta, A->codes, M, K, BM);
  if (st) return st;
  st = make_codes_map(&tb, B->codes, N, K, S::B_ROWS);
  if (st) return st;
  cudaError_t e = cudaFuncSetAttribute(gemm_nvfp4_kernel<PAIR>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)S::SMEM);
  if (e != cudaSuccess) return record_cuda_error(e);
  if (!PAIR) {
    const int grid = (int)std::min<int64_t>(p.num_tiles, num_sms());
    gemm_nvfp4_kernel<PAIR><<<grid, NUM_THREADS, S::SMEM, stream>>>(ta, tb, p, om);
    return check_launch();
  }
  const int clusters = (int)std::min<int64_t>(p.num_tiles, pair_clusters());
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(2 * clusters), 1, 1);
  cfg.blockDim = dim3(NUM_THREADS, 1, 1);
  cfg.dynamicSmemBytes = S::SMEM;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  e = cudaLaunchKernelEx(&cfg, gemm_nvfp4_kernel<PAIR>, ta, tb, p, om);
  return e == cudaSuccess ? GDN_OK : record_cuda_error(e);
}

}  // namespace

int launch_gemm_nvfp4(const gdn_nvfp4_t* A, const float* g_a, const gdn_nvfp4_t* B, int64_t M, int64_t N, int64_t K,
                      const gdn_epilogue_segment_t* segs, int n_segs, cudaStream_t stream) {
  if (M == 0 || N == 0) return GDN_OK;
  // a pair tile holds 256 rows: for M <= 128 its second CTA would idle
  return M > BM ? launch_gemm_t<true>(A, g_a, B, M, N, K, segs, n_segs, stream)
                : launch_gemm_t<false>(A, g_a, B, M, N, K, segs, n_segs, stream);
}

}  // namespace gdn
