/*
 * gdn.h -- C ABI of the NVFP4 W4A4 Gated DeltaNet layer forward (sm_100a).
 *
 * The method: "Why Gated DeltaNet Survives 4-Bit Quantization: NVFP4 W4A4 for
 * the Recurrent Half of a Hybrid 27B LLM" (franklineh.com research summary)
 * and "Anthology of the SOTA, theory-128" (section "The account").  A Gated
 * DeltaNet layer runs every projection, the gate projections included, with
 * 4-bit NVFP4 weights and activations, and carries a d_k x d_v state per head
 * through the gated delta rule.
 *
 * Conventions shared by every entry point
 *   - Every pointer argument that names tensor data is a DEVICE pointer owned
 *     by the caller.  The library never allocates or frees device memory; a
 *     call that needs scratch space takes a caller-provided workspace whose
 *     size comes from the matching *_workspace_size query.
 *   - Every call enqueues its kernels on the caller's stream (a cudaStream_t
 *     passed as void*; NULL is the legacy default stream) and returns without
 *     synchronising.  Calls hold no state between them, so calls on different
 *     streams may run concurrently as long as their buffers do not overlap.
 *   - Every call returns a gdn_status_t.  Argument checks run on the host
 *     before anything is launched; on a check failure nothing is enqueued.
 *     GDN_ERR_CUDA means a launch failed (gdn_last_error() has the CUDA text).
 *     Device-side waits are bounded: a wait that runs out records
 *     GDN_ERR_TIMEOUT in a device status word that gdn_stream_check() reads.
 *   - bf16 is IEEE bfloat16 storage (uint16 bit patterns).
 *
 * NVFP4 storage produced by gdn_quantize_nvfp4 and consumed by gdn_gemm_nvfp4
 *   codes   uint8 [rows, K/2], row-major, row stride K/2 bytes.  Element 2j of
 *           a row is the low nibble of byte j, element 2j+1 the high nibble.
 *           A nibble is E2M1: bit 3 sign, bits 2..1 exponent (bias 1), bit 0
 *           mantissa; magnitudes 0, .5, 1, 1.5, 2, 3, 4, 6.
 *   scales  one E4M3 (bias 7, finite max 448) byte per 16 consecutive
 *           elements of a row.  Two layouts:
 *             GDN_SF_LINEAR  [rows, K/16] row-major;
 *             GDN_SF_TILED   the tensor-core layout: blocks of 128 rows x 64
 *               elements (4 scales) are 512 contiguous bytes, blocks ordered
 *               row-block major then K-block; the scale of (row r, element
 *               group j) sits at byte
 *                 (r/128)*(K/64)*512 + (j/4)*512 + (r%32)*16 + ((r%128)/32)*4 + j%4.
 *               The buffer holds ceil(rows/128)*128 rows; bytes of padding
 *               rows are never read for any stored output.
 *   g       one FP32 per-tensor DECODE scale: x ~= e2m1 * e4m3 * g.
 */
#ifndef GDN_H_
#define GDN_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  GDN_OK = 0,
  GDN_ERR_INVALID_ARG = 1,       /* null pointer, negative size, bad enum      */
  GDN_ERR_UNSUPPORTED_SHAPE = 2, /* a size outside what the kernels support    */
  GDN_ERR_ALIGNMENT = 3,         /* a pointer or stride breaks an alignment rule */
  GDN_ERR_CUDA = 4,              /* a CUDA runtime / driver call failed         */
  GDN_ERR_TIMEOUT = 5,           /* a bounded device-side wait ran out          */
  GDN_ERR_WORKSPACE = 6,         /* workspace missing or smaller than required  */
  GDN_ERR_RANGE = 7              /* a value left the FP16 range of the scan's
                                    tensor-core operands (|x| >= 65520); the
                                    outputs of that call are not valid          */
} gdn_status_t;

typedef void* gdn_stream_t; /* cudaStream_t */

/* Text for a status code (static storage). */
const char* gdn_status_string(int status);
/* Text of the last CUDA error seen by this thread's calls (static storage). */
const char* gdn_last_error(void);
/* Library version, e.g. "0.1.0". */
const char* gdn_version(void);
/* Synchronise `stream`, then return and clear the device status word
 * (GDN_OK, or GDN_ERR_TIMEOUT when a bounded device wait ran out), or
 * GDN_ERR_CUDA when the synchronisation itself failed. */
int gdn_stream_check(gdn_stream_t stream);
/* Diagnostic: enqueue a one-warp kernel that waits, at most poll_limit polls
 * (1 .. 2^26), on an mbarrier nothing arrives on -- the bounded wait the
 * pipelined kernels use -- and so records GDN_ERR_TIMEOUT in the device
 * status word; gdn_stream_check() then returns and clears it.  Checks the
 * watchdog path without faulting or hanging anything. */
int gdn_selftest_bounded_wait(uint32_t poll_limit, gdn_stream_t stream);

/* Diagnostic: the FP4 tensor-core ceiling of gdn_gemm_nvfp4's MMA.  Enqueues
 * one CTA per SM (*ctas receives the count), each issuing iters x 4
 * tcgen05.mma.kind::mxf4nvf4.block_scale.block16 of M = 128, N = 256, K = 64
 * back to back from operands resident in shared memory and scales resident
 * in TMEM (no loads, no epilogue): 2 * 128 * 256 * 64 * 4 * iters * *ctas
 * FLOP.  Time it with events on `stream`; the achieved rate is the ceiling a
 * GEMM of this shape is measured against.  iters in 1 .. 2^32. */
int gdn_fp4_mma_ceiling(int64_t iters, int* ctas, gdn_stream_t stream);

/* ------------------------------------------------------------------------ *
 * Step 1: quantize activations to NVFP4.
 *
 * Passage: "Why Gated DeltaNet Survives 4-Bit Quantization", section "Why the
 * 'Fragile' Recurrence is Actually Robust" -- NVFP4 block scaling over groups
 * of 16 elements, which keeps an outlier's error inside its own block.
 *
 * Recipe (FP32, round-to-nearest-even, one operation at a time):
 *   DYNAMIC mode:      amax_t = max|x| over the tensor,
 *                      g_enc  = 2688 / amax_t (1 if amax_t == 0; FLT_MAX if
 *                      the quotient overflows);
 *   GIVEN_SCALE mode:  g_enc  = *g_enc_in (device scalar, > 0, finite).
 *   GIVEN_AMAX mode:   amax_t = *g_enc_in (device scalar: the tensor's amax,
 *                      e.g. recorded by the kernel that produced x), then as
 *                      DYNAMIC without the amax pass.
 *   per 16-block:      s = E4M3_satfinite((amax_b / 6) * g_enc);
 *                      code_i = E2M1_satfinite(x_i * (g_enc / s))
 *                      (all codes 0 when s == 0; a negative value that rounds
 *                      to zero keeps its sign bit, code 0x8);
 *   *g_out = 1 / g_enc (the decode scale).
 *
 * x        [rows, cols], element (r, c) at x[r*ld_x + c]; x_dtype
 *          GDN_DTYPE_BF16 (activations) or GDN_DTYPE_F32 (e.g. FP32 master
 *          weights); 16-byte aligned, ld_x * element size % 16 == 0.
 * cols     multiple of 16 (LINEAR) or of 64 (TILED).
 * codes    uint8 [rows, cols/2] (row stride cols/2), 8-byte aligned.
 * scales   LINEAR: uint8 [rows, cols/16].  TILED: the buffer of a larger
 *          matrix whose rows [sf_row_offset, sf_row_offset + rows) this call
 *          fills (lets separately scaled projections share one operand);
 *          sf_row_offset must be 0 for LINEAR.
 * g_out    device float, written with the decode scale.
 * ws       DYNAMIC mode only: gdn_quantize_workspace_size() bytes, 16-byte
 *          aligned (holds the running amax; overwritten).  May be NULL in
 *          the GIVEN_* modes.
 * rows == 0 is valid (only *g_out is written).
 * ------------------------------------------------------------------------ */
enum { GDN_QUANT_DYNAMIC = 0, GDN_QUANT_GIVEN_SCALE = 1, GDN_QUANT_GIVEN_AMAX = 2 };
enum { GDN_DTYPE_BF16 = 0, GDN_DTYPE_F32 = 1 };
enum { GDN_SF_TILED = 0, GDN_SF_LINEAR = 1 };

size_t gdn_quantize_workspace_size(void);
/* Bytes of a TILED scale buffer for a [rows, cols] matrix. */
size_t gdn_scales_tiled_bytes(int64_t rows, int64_t cols);

int gdn_quantize_nvfp4(const void* x, int x_dtype, int64_t rows, int64_t cols, int64_t ld_x,
                       int mode, const float* g_enc_in,
                       uint8_t* codes, uint8_t* scales, int sf_layout,
                       int64_t sf_row_offset, float* g_out,
                       void* ws, size_t ws_bytes, gdn_stream_t stream);

/* ------------------------------------------------------------------------ *
 * Calibration of static activation scales.
 *
 * Passage: "Why Gated DeltaNet Survives 4-Bit Quantization", section
 * "Critical Lessons for Model Serving" -- activation scales are calibrated
 * for each module on its own, and a fused module must keep every module's
 * own scale.  A static scale is the encode scale of the largest |x| a module
 * saw over a calibration set: run gdn_amax_update on every calibration batch
 * of that module's input (one running amax per module), then
 * gdn_encode_scale_from_amax.  gdn_layer_fwd takes the two activation
 * scales of the layer, x_g_enc and o_g_enc (gdn_layer_weights_t).
 *
 * gdn_amax_update: *amax = max(*amax, max |x|) over x [rows, cols] (row
 *   stride ld_x elements; bf16 or FP32; 16-byte aligned, cols % 16 == 0).
 *   *amax is a device FP32, >= 0 on entry (zero it before the first batch);
 *   it is never reset by the call.  rows == 0 leaves it unchanged.
 * gdn_encode_scale_from_amax: *g_enc = 2688 / *amax in FP32 (1 for 0; FLT_MAX
 *   when the quotient overflows), the encode scale step 1 uses; both device.
 * ------------------------------------------------------------------------ */
int gdn_amax_update(const void* x, int x_dtype, int64_t rows, int64_t cols, int64_t ld_x, float* amax,
                    gdn_stream_t stream);
int gdn_encode_scale_from_amax(const float* amax, float* g_enc, gdn_stream_t stream);

/* ------------------------------------------------------------------------ *
 * Step 2: block-scaled FP4 GEMM  Y[m, n] = sum_k A_hat[m, k] * B_hat[n, k].
 *
 * Passage: "Why Gated DeltaNet Survives 4-Bit Quantization", section
 * "Performance and Efficiency Gains" -- all 496 linear layers, gate
 * projections included, run with NVFP4 weights and activations; section
 * "Critical Lessons for Model Serving" -- fusing modules that were scaled
 * separately mixes up their global scales and silently corrupts the gates,
 * so every column segment of a fused projection carries its own B scale.
 *
 * A   [M, K] NVFP4 (codes + TILED scales), decode scale *g_a (device).
 * B   [N, K] NVFP4 (codes + TILED scales); segment s covers rows
 *     [n_begin, n_end) of B and uses decode scale *segs[s].g_b.
 * The FP32 accumulator of column n in segment s is multiplied by
 * (*g_a) * (*g_b) and then:
 *   GDN_EPI_STORE_BF16  out[m*ld_out + (n - n_begin)] = bf16_rne(y)
 *   GDN_EPI_STORE_F32   out[m*ld_out + (n - n_begin)] = y
 *   GDN_EPI_LOG_ALPHA   out[...] = -exp(A_log[j]) * softplus(y + dt_bias[j]),
 *                       j = n - n_begin (FP32; the decay gate of step 3)
 *   GDN_EPI_BETA        out[...] = sigmoid(y) (FP32; the write strength)
 * Segments must be sorted, disjoint and cover [0, N); at most
 * GDN_MAX_SEGMENTS.  Outputs of different segments may share a buffer.
 *
 * Shapes: K % 64 == 0, K >= 64; M, N >= 0 arbitrary (ragged tiles handled).
 * Alignment: codes and scales 16-byte aligned; bf16 outputs 4-byte aligned.
 * ------------------------------------------------------------------------ */
enum {
  GDN_EPI_STORE_BF16 = 0,
  GDN_EPI_STORE_F32 = 1,
  GDN_EPI_LOG_ALPHA = 2,
  GDN_EPI_BETA = 3
};
#define GDN_MAX_SEGMENTS 8

typedef struct {
  const uint8_t* codes;  /* [rows, K/2] */
  const uint8_t* scales; /* TILED layout */
} gdn_nvfp4_t;

typedef struct {
  int64_t n_begin, n_end;
  int kind;
  const float* g_b;      /* device scalar: decode scale of these B rows */
  void* out;
  int64_t ld_out;        /* elements */
  const float* A_log;    /* LOG_ALPHA only: [n_end - n_begin] */
  const float* dt_bias;  /* LOG_ALPHA only: [n_end - n_begin] */
} gdn_epilogue_segment_t;

int gdn_gemm_nvfp4(const gdn_nvfp4_t* A, const float* g_a, const gdn_nvfp4_t* B,
                   int64_t M, int64_t N, int64_t K,
                   const gdn_epilogue_segment_t* segs, int n_segs,
                   gdn_stream_t stream);

/* ------------------------------------------------------------------------ *
 * Step 3: gates, standalone.
 *
 * Passage: "Anthology of the SOTA, theory-128", section "The account" -- the
 * decay is exp(-exp(A) * softplus(a + dt_bias)) and the write strength is a
 * sigmoid.  (The page prints "softplus(a + b)"; the b there is the per-head
 * bias dt_bias.)
 *
 * a, b            FP32 [M, H] row-major (gate pre-activations).
 * A_log, dt_bias  FP32 [H].
 * log_alpha       FP32 [M, H] out: -exp(A_log[h]) * softplus(a + dt_bias[h]).
 * beta            FP32 [M, H] out: 1 / (1 + exp(-b)).
 * FP32 with CUDA's expf / log1pf (not the fast intrinsics).
 * ------------------------------------------------------------------------ */
int gdn_gates(const float* a, const float* b, int64_t M, int H,
              const float* A_log, const float* dt_bias,
              float* log_alpha, float* beta, gdn_stream_t stream);

/* ------------------------------------------------------------------------ *
 * Step 4: gated delta rule forward (chunked; chunk length 64).
 *
 * Passage: "Anthology of the SOTA, theory-128", section "The account" --
 *   S_t = alpha_t S_{t-1} + beta_t k_t (v_t - S_{t-1}^T k_t)^T,  o_t = S_t^T q_t,
 * with q, k L2-normalised per (token, head) over d_k when
 * GDN_DR_L2NORM_QK is set: x_hat = x / sqrt(||x||^2 + 1e-6).
 *
 * q, k   bf16, element (b, t, h, i) at q[(b*T + t)*ld_q + h*dk + i]
 *        (ld_k likewise); v bf16 with ld_v and dv.  16-byte aligned,
 *        ld % 8 == 0.
 * log_alpha, beta  FP32 [B, T, H] contiguous.
 * S0     FP32 [B, H, dk, dv] initial state, or NULL for zeros.
 * o      [B, T, H, dv] contiguous; bf16, or FP32 with GDN_DR_O_FP32.
 * S_T    FP32 [B, H, dk, dv] final state, or NULL.
 * Supported: dk and dv in {32, 64, 128}; any T >= 0 (a ragged last chunk is
 * handled); B*H >= 1.  The chunk contractions run on FP16 tensor-core
 * operands with FP32 accumulation (FP16 keeps three more mantissa bits than
 * bf16, which the 2e-3 tolerance at 32K tokens needs).  Values of beta v, of
 * the state and of the chunk intermediates must stay inside the FP16 range:
 * a value of magnitude >= 65520 rounds to infinity, and the call then records
 * GDN_ERR_RANGE in the device status word (gdn_stream_check() returns it);
 * its o and S_T are not valid.  With the tensor-core kernel every FP16
 * operand is checked where it is converted; with the mma.sync kernel the
 * check is that o and S_T came out finite.
 * Kernels: dk = 128 with dv a multiple of 64 runs on the 5th-generation
 * tensor cores (tcgen05.mma, state kept in TMEM); other shapes, or the flag
 * GDN_DR_MMA_SYNC, run the warp-level mma.sync kernel.  Both compute the same
 * chunk form; they differ in FP32 summation order only.
 * ws     gdn_delta_rule_workspace_size(...) bytes (may be 0 / NULL), 256-byte
 *        aligned, owned by the caller, not read after the call's kernels
 *        end.  The tensor-core path uses it when it cuts long sequences on
 *        few chains into segments (the size is 0 otherwise): (1) the segment
 *        states, then (2) 16 KB per chunk of 64 tokens per (batch, head): the
 *        inverse (I + L)^{-1} of every chunk and its beta-weighted copy,
 *        computed once by a wide pass ahead of both passes over the
 *        segments.  With fewer bytes than (1) + (2) both passes invert each
 *        chunk themselves (the same bits), with fewer than (1) every sequence
 *        runs in one piece.  Unused by the mma.sync kernel.
 * flags  GDN_DR_L2NORM_QK | GDN_DR_O_FP32 | GDN_DR_MMA_SYNC; any other bit
 *        (GDN_DR_DECAYED_READ included: the chunked form implements the
 *        literal read) is GDN_ERR_INVALID_ARG.
 * ------------------------------------------------------------------------ */
enum { GDN_DR_L2NORM_QK = 1, GDN_DR_O_FP32 = 2, GDN_DR_MMA_SYNC = 4 };

size_t gdn_delta_rule_workspace_size(int64_t B, int64_t T, int H, int dk, int dv);

int gdn_delta_rule_fwd(const void* q, const void* k, const void* v,
                       int64_t ld_q, int64_t ld_k, int64_t ld_v,
                       const float* log_alpha, const float* beta,
                       const float* S0, int64_t B, int64_t T, int H, int dk, int dv,
                       int flags, void* o, float* S_T,
                       void* ws, size_t ws_bytes, gdn_stream_t stream);

/* ------------------------------------------------------------------------ *
 * Step 4, token by token (decode): the recurrence itself, without chunking.
 *
 * Passage: as gdn_delta_rule_fwd ("Anthology of the SOTA, theory-128",
 * section "The account").  Each (batch, head) chain keeps its state on chip
 * (shared memory) across the T tokens of the call and walks them in order:
 *   r_t = S_{t-1}^T k_t     (alpha_t S_{t-1}^T k_t with GDN_DR_DECAYED_READ,
 *                            the reading S_t = alpha_t (I - beta_t k_t k_t^T)
 *                            S_{t-1} + beta_t k_t v_t^T),
 *   S_t = alpha_t S_{t-1} + beta_t k_t (v_t - r_t)^T,   o_t = S_t^T q_t.
 * Meant for decode (T = 1) and short continuations after a chunked prefill;
 * the state is read and written once per call (2 dk dv 4 bytes per chain).
 *
 * q, k, v, ld_*    as gdn_delta_rule_fwd (bf16, element (b, t, h, i) at
 *                  q[(b*T + t)*ld_q + h*dk + i]); element-aligned only.
 * log_alpha, beta  FP32 [B, T, H] contiguous.
 * S_in             FP32 [B, H, dk, dv], or NULL for zeros.
 * S_out            FP32 [B, H, dk, dv], required; may be S_in (in place).
 * o                [B, T, H, dv] contiguous; bf16, or FP32 with GDN_DR_O_FP32.
 * flags            GDN_DR_L2NORM_QK | GDN_DR_O_FP32 | GDN_DR_DECAYED_READ.
 * Supported: dk and dv in {32, 64, 128}; T >= 0 (T = 0 copies S_in to
 * S_out); 0 <= B*H <= 2^28.  All FP32 arithmetic; exp via CUDA's expf.
 * ------------------------------------------------------------------------ */
enum { GDN_DR_DECAYED_READ = 8 };

int gdn_delta_rule_step(const void* q, const void* k, const void* v,
                        int64_t ld_q, int64_t ld_k, int64_t ld_v,
                        const float* log_alpha, const float* beta,
                        const float* S_in, float* S_out,
                        int64_t B, int64_t T, int H, int dk, int dv,
                        int flags, void* o, gdn_stream_t stream);

/* ------------------------------------------------------------------------ *
 * The rest of a Gated DeltaNet block: short convolution and gated output norm.
 *
 * The pages name "the convolution" only as an alternative explanation and
 * define neither piece; both follow the outside specification of the Gated
 * DeltaNet block (Yang, Kautz and Hatamizadeh, "Gated Delta Networks:
 * Improving Mamba2 with Delta Rule", ICLR 2025).
 *
 * gdn_short_conv: causal depthwise convolution of width 4 over tokens, then
 *   SiLU, per channel c of x [B, T, C] (bf16, row stride ld_x elements):
 *     y_t[c] = SiLU(sum_{j=0..3} w[c*4 + j] * x_{t-3+j}[c]),   SiLU(u) = u sigmoid(u)
 *   w FP32 [C, 4] (16-byte aligned).  Tokens before t = 0 come from state_in
 *   (bf16 [B, 3, C], the last three inputs of the previous call, oldest
 *   first) or are zero when it is NULL; state_out (bf16 [B, 3, C], may be
 *   NULL) receives this call's last three inputs, carried state included.
 *   y bf16 [B, T, C] with row stride ld_y; must not alias x.  C % 8 == 0,
 *   x, y 16-byte aligned, ld % 8 == 0; B <= 65535, T <= 65535 * 64.  FP32
 *   arithmetic, CUDA's expf.
 * gdn_gated_rmsnorm: per (token m, head h) row of dv values of o and g
 *   (bf16 [M, H*dv], row m*H + h at (m*H + h)*dv):
 *     y = o / sqrt(mean(o^2) + 1e-6) * gamma * SiLU(g)          (bf16 out)
 *   o, g, y 16-byte aligned; gamma FP32 [dv]; dv in {32, 64, 128}.  When
 *   amax is non-NULL, max |y|
 *   (of the stored bf16 values) is folded into *amax (>= 0 on entry), for a
 *   given-amax quantization of y.
 * ------------------------------------------------------------------------ */
int gdn_short_conv(const void* x, int64_t B, int64_t T, int64_t C, int64_t ld_x, const float* w, const void* state_in,
                   void* y, int64_t ld_y, void* state_out, gdn_stream_t stream);
int gdn_gated_rmsnorm(const void* o, const void* g, int64_t M, int H, int dv, const float* gamma, void* y,
                      float* amax, gdn_stream_t stream);

/* ------------------------------------------------------------------------ *
 * The layer: steps 1-4 and the output projection, in one call.
 *
 *   xq = quant(x); [q|k|v|a|b] = gemm(xq, W_qkvab) with gates in the epilogue;
 *   o  = delta_rule(q, k, v, log_alpha, beta; L2-normalised q, k);
 *   y  = gemm(quant(o), W_out)  (bf16 out); quant(x) and quant(o) use their
 *        tensor's own amax, or the static encode scales w->x_g_enc and
 *        w->o_g_enc when they are given (calibrated per module, see
 *        "Calibration of static activation scales").
 * Optional (cfg->conv, cfg->out_gate), from the Gated DeltaNet block's outside
 * specification: q, k, v pass through gdn_short_conv (zero history: each
 * call holds whole sequences) before the scan, and o through
 * gdn_gated_rmsnorm with g = x W_g (a sixth W4A4 projection) before it is
 * quantized for the output projection.  No residual.
 *
 * Weights are pre-quantized by the caller (gdn_quantize_nvfp4, one call per
 * projection so each keeps its own decode scale; q, k, v, a, b share one TILED
 * scale buffer through sf_row_offset).  W_qkvab rows: q [0, H*dk), k [H*dk,
 * 2*H*dk), v [2*H*dk, 2*H*dk + H*dv), a (H rows), b (H rows); K = d_model.
 * W_out: [d_model, H*dv].  With cfg->out_gate, W_qkvab holds H*dv more rows
 * after b: the output gate g (decode scale w->g_g), and w->norm_w is the
 * RMSNorm weight [dv]; with cfg->conv, w->conv_w is the convolution weight
 * FP32 [2*H*dk + H*dv, 4] over the q | k | v channels.
 *
 * x   bf16 [B*T, d_model];  y bf16 [B*T, d_model];  S0 / S_T as in step 4.
 * ws  gdn_layer_workspace_size(cfg) bytes, 256-byte aligned.  After the call
 *     it holds the intermediates at the offsets gdn_layer_workspace_offsets
 *     reports (useful to check each stage).
 * Supported: d_model % 64 == 0, H*dv % 64 == 0, dk and dv in {32, 64, 128}.
 * ------------------------------------------------------------------------ */
typedef struct {
  int64_t B, T, d_model;
  int H, dk, dv;
  int conv;      /* 1: short convolution + SiLU on q, k, v; 0: none */
  int out_gate;  /* 1: gated RMSNorm of o with the g projection; 0: none */
} gdn_layer_cfg_t;

typedef struct {
  gdn_nvfp4_t w_qkvab;   /* [2*H*dk + H*dv + 2*H, d_model] */
  const float* g_q;      /* device decode scales, one per projection */
  const float* g_k;
  const float* g_v;
  const float* g_a;
  const float* g_b;
  gdn_nvfp4_t w_out;     /* [d_model, H*dv] */
  const float* g_out;
  const float* A_log;    /* [H] */
  const float* dt_bias;  /* [H] */
  const float* o_g_enc;  /* NULL: o is quantized with its own amax (dynamic).
                            Else a device FP32 encode scale for o (a static,
                            calibrated activation scale): the scan writes o's
                            NVFP4 codes and scales itself (in its epilogue when
                            the tensor-core scan runs) and no quantizer pass
                            runs; the decode scale is 1 / o_g_enc. */
  const float* x_g_enc;  /* NULL: x is quantized with its own amax (dynamic:
                            an amax pass, then the quantizer).  Else a device
                            FP32 encode scale for x (static, calibrated): one
                            quantizer pass; the decode scale is 1 / x_g_enc. */
  const float* conv_w;   /* cfg->conv: FP32 [2*H*dk + H*dv, 4] */
  const float* g_g;      /* cfg->out_gate: decode scale of the g rows */
  const float* norm_w;   /* cfg->out_gate: RMSNorm weight FP32 [dv] */
} gdn_layer_weights_t;

enum {
  GDN_WS_X_CODES = 0, GDN_WS_X_SCALES, GDN_WS_X_G, GDN_WS_QKV, GDN_WS_LOG_ALPHA,
  GDN_WS_BETA, GDN_WS_O, GDN_WS_O_CODES, GDN_WS_O_SCALES, GDN_WS_O_G,
  GDN_WS_QUANT, GDN_WS_SCAN, GDN_WS_QKV_CONV, GDN_WS_G, GDN_WS_O_GATED, GDN_WS_COUNT
};

size_t gdn_layer_workspace_size(const gdn_layer_cfg_t* cfg);
/* offsets[GDN_WS_COUNT] in bytes from ws: x codes, x scales (TILED), x decode
 * scale, qkv bf16 [B*T, 2*H*dk + H*dv], log_alpha / beta FP32 [B*T, H],
 * o bf16 [B*T, H*dv], o codes / scales / decode scale, quantizer and scan
 * scratch, and (empty unless cfg->conv / cfg->out_gate) the convolved qkv,
 * g bf16 [B*T, H*dv] and the gated o bf16 [B*T, H*dv]. */
int gdn_layer_workspace_offsets(const gdn_layer_cfg_t* cfg, int64_t* offsets);

int gdn_layer_fwd(const gdn_layer_weights_t* w, const gdn_layer_cfg_t* cfg,
                  const void* x, void* y, const float* S0, float* S_T,
                  void* ws, size_t ws_bytes, gdn_stream_t stream);

/* ------------------------------------------------------------------------ *
 * Allocation-free layer forward (no counterpart in the paper).
 *
 * For callers that cannot allocate device memory: plugins that receive only
 * their input and output pointers from a host framework that owns every
 * allocation, and real-time paths whose memory budget is fixed up front.
 * Same computation, arguments and results as gdn_layer_fwd (bit for bit),
 * except that the workspace is a static device array of
 * GDN_LAYER_STATIC_WS_BYTES inside the library (present on every GPU that
 * loads it, until the process exits).
 *   - Sizes: a cfg whose gdn_layer_workspace_size() exceeds the array is
 *     rejected with GDN_ERR_WORKSPACE (gdn_last_error() says by how much);
 *     with d_model 5120, H 32, d 128 that is about 860 tokens per call.
 *   - Set-up: the first call on a device looks up the array's device address
 *     (cudaGetSymbolAddress with that device current); make that first call
 *     before any stream capture.
 *   - Concurrency: every call shares the one array, so calls that overlap on
 *     the GPU (different streams, or threads without ordering) race; order
 *     them on one stream.  The array keeps the last call's intermediates.
 *   - Allocates nothing: no cudaMalloc / cudaFree or allocating routine.
 *   - The looked-up address is cached per device for the life of the
 *     process: do not call this entry point again after cudaDeviceReset()
 *     (or any other teardown of the device's primary context).  The same
 *     holds for the device status word every entry point writes.
 * ------------------------------------------------------------------------ */
#define GDN_LAYER_STATIC_WS_BYTES (32u << 20)

int gdn_layer_fwd_static_ws(const gdn_layer_weights_t* w, const gdn_layer_cfg_t* cfg,
                            const void* x, void* y, const float* S0, float* S_T,
                            gdn_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* GDN_H_ */
