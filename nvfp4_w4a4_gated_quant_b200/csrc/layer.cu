// The W4A4 Gated DeltaNet layer forward: quantize -> fused q/k/v/a/b GEMM with
// the gates in its epilogue -> chunked delta rule -> quantize -> output GEMM.
// Five kernel launches (plus one 4-byte memset per quantization) on the
// caller's stream; every intermediate lives in the caller's workspace.
#include <mutex>

#include "common.cuh"
#include "kernels.h"

using namespace gdn;

namespace {

int64_t align256(int64_t x) { return (x + 255) & ~(int64_t)255; }

bool cfg_ok(const gdn_layer_cfg_t* c) {
  return c && c->B >= 0 && c->T >= 0 && c->d_model > 0 && c->H > 0 && c->dk > 0 && c->dv > 0 &&
         (c->conv == 0 || c->conv == 1) && (c->out_gate == 0 || c->out_gate == 1);
}

int layout(const gdn_layer_cfg_t* c, int64_t* off, int64_t* total) {
  const int64_t M = c->B * c->T;
  const int64_t D = c->d_model;
  const int64_t HV = (int64_t)c->H * c->dv;
  const int64_t NQKV = 2 * (int64_t)c->H * c->dk + HV;
  int64_t sizes[GDN_WS_COUNT];
  sizes[GDN_WS_X_CODES] = M * D / 2;
  sizes[GDN_WS_X_SCALES] = (int64_t)gdn_scales_tiled_bytes(M, D);
  sizes[GDN_WS_X_G] = 4;
  sizes[GDN_WS_QKV] = M * NQKV * 2;
  sizes[GDN_WS_LOG_ALPHA] = M * c->H * 4;
  sizes[GDN_WS_BETA] = M * c->H * 4;
  sizes[GDN_WS_O] = M * HV * 2;
  sizes[GDN_WS_O_CODES] = M * HV / 2;
  sizes[GDN_WS_O_SCALES] = (int64_t)gdn_scales_tiled_bytes(M, HV);
  sizes[GDN_WS_O_G] = 4;
  sizes[GDN_WS_QUANT] = (int64_t)gdn_quantize_workspace_size();
  sizes[GDN_WS_SCAN] = (int64_t)gdn_delta_rule_workspace_size(c->B, c->T, c->H, c->dk, c->dv);
  sizes[GDN_WS_QKV_CONV] = c->conv ? M * NQKV * 2 : 0;
  sizes[GDN_WS_G] = c->out_gate ? M * HV * 2 : 0;
  sizes[GDN_WS_O_GATED] = c->out_gate ? M * HV * 2 : 0;
  int64_t pos = 0;
  for (int i = 0; i < GDN_WS_COUNT; ++i) {
    off[i] = pos;
    pos += align256(sizes[i]);
  }
  *total = pos;
  return GDN_OK;
}

}  // namespace

extern "C" {

size_t gdn_layer_workspace_size(const gdn_layer_cfg_t* cfg) {
  if (!cfg_ok(cfg)) return 0;
  int64_t off[GDN_WS_COUNT], total = 0;
  layout(cfg, off, &total);
  return (size_t)total;
}

int gdn_layer_workspace_offsets(const gdn_layer_cfg_t* cfg, int64_t* offsets) {
  if (!cfg_ok(cfg) || !offsets) return GDN_ERR_INVALID_ARG;
  int64_t total = 0;
  return layout(cfg, offsets, &total);
}

int gdn_layer_fwd(const gdn_layer_weights_t* w, const gdn_layer_cfg_t* cfg, const void* x, void* y, const float* S0,
                  float* S_T, void* ws, size_t ws_bytes, gdn_stream_t stream) {
  if (!w || !cfg_ok(cfg)) return GDN_ERR_INVALID_ARG;
  const int64_t M = cfg->B * cfg->T;
  const int64_t D = cfg->d_model;
  const int H = cfg->H, dk = cfg->dk, dv = cfg->dv;
  const int64_t HK = (int64_t)H * dk, HV = (int64_t)H * dv;
  const int64_t NQKV = 2 * HK + HV;
  if (D % 64 != 0 || HV % 64 != 0) return GDN_ERR_UNSUPPORTED_SHAPE;
  if ((dk != 32 && dk != 64 && dk != 128) || (dv != 32 && dv != 64 && dv != 128)) return GDN_ERR_UNSUPPORTED_SHAPE;
  int64_t off[GDN_WS_COUNT], total = 0;
  layout(cfg, off, &total);
  if (!ws || (int64_t)ws_bytes < total) return GDN_ERR_WORKSPACE;
  if (!aligned(ws, 256)) return GDN_ERR_ALIGNMENT;
  if (!w->g_q || !w->g_k || !w->g_v || !w->g_a || !w->g_b || !w->g_out || !w->A_log || !w->dt_bias)
    return GDN_ERR_INVALID_ARG;
  if ((cfg->conv && !w->conv_w) || (cfg->out_gate && (!w->g_g || !w->norm_w))) return GDN_ERR_INVALID_ARG;
  if (cfg->conv && (NQKV % 8 != 0 || !aligned(w->conv_w, 16))) return GDN_ERR_UNSUPPORTED_SHAPE;
  if (M > 0) {
    if (!x || !y || !w->w_qkvab.codes || !w->w_qkvab.scales || !w->w_out.codes || !w->w_out.scales)
      return GDN_ERR_INVALID_ARG;
    if (!aligned(x, 16) || !aligned(y, 16)) return GDN_ERR_ALIGNMENT;
  }
  uint8_t* base = static_cast<uint8_t*>(ws);
  uint8_t* x_codes = base + off[GDN_WS_X_CODES];
  uint8_t* x_scales = base + off[GDN_WS_X_SCALES];
  float* x_g = reinterpret_cast<float*>(base + off[GDN_WS_X_G]);
  uint16_t* qkv = reinterpret_cast<uint16_t*>(base + off[GDN_WS_QKV]);
  float* log_alpha = reinterpret_cast<float*>(base + off[GDN_WS_LOG_ALPHA]);
  float* beta = reinterpret_cast<float*>(base + off[GDN_WS_BETA]);
  uint16_t* o = reinterpret_cast<uint16_t*>(base + off[GDN_WS_O]);
  uint8_t* o_codes = base + off[GDN_WS_O_CODES];
  uint8_t* o_scales = base + off[GDN_WS_O_SCALES];
  float* o_g = reinterpret_cast<float*>(base + off[GDN_WS_O_G]);
  void* qws = base + off[GDN_WS_QUANT];
  uint16_t* qkv_conv = reinterpret_cast<uint16_t*>(base + off[GDN_WS_QKV_CONV]);
  uint16_t* g = reinterpret_cast<uint16_t*>(base + off[GDN_WS_G]);
  uint16_t* o_gated = reinterpret_cast<uint16_t*>(base + off[GDN_WS_O_GATED]);
  const size_t qws_bytes = gdn_quantize_workspace_size();
  gdn_stream_t s = stream;

  // x: its own amax (two passes), or the calibrated static scale (one pass)
  int st = w->x_g_enc ? gdn_quantize_nvfp4(x, GDN_DTYPE_BF16, M, D, D, GDN_QUANT_GIVEN_SCALE, w->x_g_enc, x_codes,
                                           x_scales, GDN_SF_TILED, 0, x_g, nullptr, 0, s)
                      : gdn_quantize_nvfp4(x, GDN_DTYPE_BF16, M, D, D, GDN_QUANT_DYNAMIC, nullptr, x_codes, x_scales,
                                           GDN_SF_TILED, 0, x_g, qws, qws_bytes, s);
  if (st) return st;

  gdn_nvfp4_t xa{x_codes, x_scales};
  gdn_epilogue_segment_t seg[6] = {};
  seg[0] = {0, HK, GDN_EPI_STORE_BF16, w->g_q, qkv, NQKV, nullptr, nullptr};
  seg[1] = {HK, 2 * HK, GDN_EPI_STORE_BF16, w->g_k, qkv + HK, NQKV, nullptr, nullptr};
  seg[2] = {2 * HK, NQKV, GDN_EPI_STORE_BF16, w->g_v, qkv + 2 * HK, NQKV, nullptr, nullptr};
  seg[3] = {NQKV, NQKV + H, GDN_EPI_LOG_ALPHA, w->g_a, log_alpha, H, w->A_log, w->dt_bias};
  seg[4] = {NQKV + H, NQKV + 2 * H, GDN_EPI_BETA, w->g_b, beta, H, nullptr, nullptr};
  if (cfg->out_gate) seg[5] = {NQKV + 2 * H, NQKV + 2 * H + HV, GDN_EPI_STORE_BF16, w->g_g, g, HV, nullptr, nullptr};
  st = gdn_gemm_nvfp4(&xa, x_g, &w->w_qkvab, M, NQKV + 2 * H + (cfg->out_gate ? HV : 0), D, seg,
                      cfg->out_gate ? 6 : 5, s);
  if (st) return st;

  // the short convolution (+ SiLU) over the q | k | v channels, from zero history
  const uint16_t* qkv_in = qkv;
  if (cfg->conv) {
    st = gdn_short_conv(qkv, cfg->B, cfg->T, NQKV, NQKV, w->conv_w, nullptr, qkv_conv, NQKV, nullptr, s);
    if (st) return st;
    qkv_in = qkv_conv;
  }

  // Dynamic o scale: the scan records max |o| of the bf16 values it stores,
  // so o is quantized in one pass (given-amax mode) instead of amax pass +
  // pass.  Static o scale (w->o_g_enc): the scan writes o's codes and scales
  // itself, and no quantizer pass runs.
  unsigned* o_amax = static_cast<unsigned*>(qws);
  cudaError_t ce = cudaMemsetAsync(o_amax, 0, sizeof(unsigned), reinterpret_cast<cudaStream_t>(s));
  if (ce != cudaSuccess) return record_cuda_error(ce);
  OQuant oq{o_codes, o_scales, w->o_g_enc, o_g};
  const bool fuse_oq = w->o_g_enc && !cfg->out_gate;   // the scan quantizes o itself
  st = launch_delta_rule(qkv_in, qkv_in + HK, qkv_in + 2 * HK, NQKV, NQKV, NQKV, log_alpha, beta, S0, cfg->B, cfg->T,
                         H, dk, dv, GDN_DR_L2NORM_QK, o, S_T, cfg->out_gate ? nullptr : o_amax,
                         reinterpret_cast<cudaStream_t>(s), fuse_oq ? &oq : nullptr, base + off[GDN_WS_SCAN],
                         (size_t)gdn_delta_rule_workspace_size(cfg->B, cfg->T, H, dk, dv));
  if (st) return st;

  // the gated output norm; then o (or the gated o) is quantized for the
  // output projection with its own amax or the static scale
  const uint16_t* o_q = o;
  if (cfg->out_gate) {
    st = gdn_gated_rmsnorm(o, g, M, H, dv, w->norm_w, o_gated, reinterpret_cast<float*>(o_amax), s);
    if (st) return st;
    o_q = o_gated;
  }
  if (!fuse_oq) {
    st = w->o_g_enc ? gdn_quantize_nvfp4(o_q, GDN_DTYPE_BF16, M, HV, HV, GDN_QUANT_GIVEN_SCALE, w->o_g_enc, o_codes,
                                         o_scales, GDN_SF_TILED, 0, o_g, nullptr, 0, s)
                    : gdn_quantize_nvfp4(o_q, GDN_DTYPE_BF16, M, HV, HV, GDN_QUANT_GIVEN_AMAX,
                                         reinterpret_cast<const float*>(o_amax), o_codes, o_scales, GDN_SF_TILED, 0,
                                         o_g, nullptr, 0, s);
    if (st) return st;
  }

  gdn_nvfp4_t oa{o_codes, o_scales};
  gdn_epilogue_segment_t yseg = {0, D, GDN_EPI_STORE_BF16, w->g_out, y, D, nullptr, nullptr};
  return gdn_gemm_nvfp4(&oa, o_g, &w->w_out, M, D, HV, &yseg, 1, s);
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Allocation-free layer forward.
//
// Some callers cannot allocate device memory at all: plugins that are given
// only their input and output pointers by a host framework that owns every
// allocation, and real-time paths whose memory budget is fixed up front.  They
// call gdn_layer_fwd_static_ws, which takes the layer's scratch (the
// intermediates between its kernels) from the file-scope device array below
// instead of a caller workspace.
//
// The array is GDN_LAYER_STATIC_WS_BYTES (32 MiB) and lives on every GPU that
// loads this library until the process exits.  Host code cannot pass the
// array's name to a kernel: in host code the name is only a host-side stand-in
// for the symbol.  The first call on each device therefore looks up the
// array's device address with cudaGetSymbolAddress (with that device
// current) and caches it.
static __device__ __align__(256) uint8_t g_layer_static_ws[GDN_LAYER_STATIC_WS_BYTES];

namespace {
constexpr int kMaxDev = 64;
void* g_static_ws_ptr[kMaxDev];
std::mutex g_static_ws_mu;

int static_ws_address(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return record_cuda_error(e);
  if (dev < 0 || dev >= kMaxDev) return GDN_ERR_INVALID_ARG;
  std::lock_guard<std::mutex> lk(g_static_ws_mu);
  if (!g_static_ws_ptr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_layer_static_ws);
    if (e != cudaSuccess) return record_cuda_error(e);
    g_static_ws_ptr[dev] = p;
  }
  *out = g_static_ws_ptr[dev];
  return GDN_OK;
}
}  // namespace

extern "C" int gdn_layer_fwd_static_ws(const gdn_layer_weights_t* w, const gdn_layer_cfg_t* cfg, const void* x,
                                       void* y, const float* S0, float* S_T, gdn_stream_t stream) {
  if (!w || !cfg_ok(cfg)) return GDN_ERR_INVALID_ARG;
  const size_t need = gdn_layer_workspace_size(cfg);
  if (need > (size_t)GDN_LAYER_STATIC_WS_BYTES) {
    set_error_text("layer workspace of %zu bytes exceeds the %zu-byte static scratch", need,
                   (size_t)GDN_LAYER_STATIC_WS_BYTES);
    return GDN_ERR_WORKSPACE;
  }
  void* ws = nullptr;
  const int st = static_ws_address(&ws);
  if (st) return st;
  // Nothing in the scratch has to start at zero: the quantizer clears its own
  // amax word on the stream before each use, and every other intermediate is
  // written before it is read within the call.
  return gdn_layer_fwd(w, cfg, x, y, S0, S_T, ws, (size_t)GDN_LAYER_STATIC_WS_BYTES, stream);
}
