// C ABI of libdfssm (declared in include/dfssm.h): argument validation and kernel launches.

#include <cstdio>
#include <cstring>

#include "common.cuh"
#include "internal.h"

namespace {

thread_local char g_last_cuda_error[256] = "";

int cuda_fail(cudaError_t e) {
  std::snprintf(g_last_cuda_error, sizeof(g_last_cuda_error), "%s: %s", cudaGetErrorName(e),
                cudaGetErrorString(e));
  return DFSSM_ECUDA;
}

inline bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }
inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

// Linear-decode workspace: [status word, kStatusBytes][quantize -> GEMV hand-off (quant scratch)].
size_t linear_decode_ws(int B, int d_in) { return dfssm::kStatusBytes + dfssm::quant_scratch_bytes(B, d_in); }

struct LayerWs {
  float* zxbcdt;  // [B][d_ip]
  float* xc;      // [B][C]
  float* g;       // [B][E]
  dfssm::QuantScratch qs;
};

size_t chain_ws_bytes(int B, int d_model, int E, int C, int d_ip) {
  const int nmax = d_model > E ? d_model : E;
  return align256(sizeof(float) * (size_t)B * d_ip) + align256(sizeof(float) * (size_t)B * C) +
         align256(sizeof(float) * (size_t)B * E) + dfssm::quant_scratch_bytes(B, nmax);
}

// Layer-decode workspace: [fused-kernel region][per-op chain region].  The fused region comes first so
// that its error word sits at a fixed offset (dfssm_device_status).
size_t layer_ws_bytes(int B, int d_model, int E, int C, int d_ip) {
  return align256(dfssm::fused_decode_workspace_bytes()) + chain_ws_bytes(B, d_model, E, C, d_ip);
}

LayerWs carve_layer_ws(void* base, int B, int d_model, int E, int C, int d_ip) {
  char* p = static_cast<char*>(base) + align256(dfssm::fused_decode_workspace_bytes());
  LayerWs w;
  w.zxbcdt = reinterpret_cast<float*>(p);
  p += align256(sizeof(float) * (size_t)B * d_ip);
  w.xc = reinterpret_cast<float*>(p);
  p += align256(sizeof(float) * (size_t)B * C);
  w.g = reinterpret_cast<float*>(p);
  p += align256(sizeof(float) * (size_t)B * E);
  const int nmax = d_model > E ? d_model : E;
  w.qs = dfssm::carve_quant_scratch(p, B, nmax);
  return w;
}

// Greedy-choice scratch of the head kernel: the 64-bit argmax key and the finished-CTA count.
constexpr size_t kGreedyBytes = 256;

// Generation workspace: [layer-decode region (B = 1, sized as dfssm_workspace_size reports)]
// [hidden f32 d_model][logits f32 V][greedy scratch].
struct GenerateWs {
  size_t layer, hidden, logits, greedy, total;
};
GenerateWs generate_ws(int V, int d_model, int d_inner) {
  GenerateWs g;
  const int C = d_inner + 2048, d_ip = 2 * d_inner + 2048 + 1024;
  g.layer = 0;
  g.hidden = align256(layer_ws_bytes(1, d_model, d_inner, C, d_ip));
  g.logits = g.hidden + align256(sizeof(float) * (size_t)d_model);
  g.greedy = g.logits + align256(sizeof(float) * (size_t)V);
  g.total = g.greedy + kGreedyBytes;
  return g;
}

// Layer-prefill workspace: [zxbcdt f32 M x d_ip][xc f32 M x C][g f32 M x E][SiLU(z) f32 M x E]
// [dt, dA f32 M x nheads x 2][linear-prefill region], with C, d_ip and nheads at their largest supported
// values (2 ngroups d_state <= 2048, nheads <= 1024).
struct PrefillLayerWs {
  size_t zx, xc, g, sz, dtdA, lin, total;
};
PrefillLayerWs prefill_layer_ws(int M, int d_model, int E) {
  PrefillLayerWs w;
  const size_t C = (size_t)E + 2048, d_ip = 2 * (size_t)E + 2048 + 1024;
  w.zx = dfssm::kStatusBytes;  // the status word comes first
  w.xc = w.zx + align256(sizeof(float) * (size_t)M * d_ip);
  w.g = w.xc + align256(sizeof(float) * (size_t)M * C);
  w.sz = w.g + align256(sizeof(float) * (size_t)M * E);
  w.dtdA = w.sz + align256(sizeof(float) * (size_t)M * E);
  w.lin = w.dtdA + align256(sizeof(float) * (size_t)M * 1024 * 2);
  const size_t a = dfssm::prefill_workspace_bytes(M, d_model, (int)d_ip);
  const size_t b = dfssm::prefill_workspace_bytes(M, E, d_model);
  w.total = w.lin + align256(a > b ? a : b);
  return w;
}

int check_head(const int8_t* W, const float* s_row, int V, int d) {
  if (!W || !s_row || V < 1 || d < 16 || d % 16) return DFSSM_EINVAL;
  if (d > 8192) return DFSSM_EUNSUPPORTED;
  if (!aligned(W, 16) || !aligned(s_row, 4)) return DFSSM_EALIGN;
  return DFSSM_OK;
}

int enqueue_embed(const int8_t* W, const float* s_row, int V, int d, const int32_t* token, float* h,
                  int* status, cudaStream_t s) {
  dfssm::EmbedArgs ea{W, s_row, V, d, token, h, status};
  const cudaError_t e = dfssm::launch_embed(ea, s);
  return e == cudaSuccess ? DFSSM_OK : cuda_fail(e);
}

int enqueue_head(const int8_t* W, const float* s_row, int V, int d, const float* h, const float* norm_w,
                 float* logits, int32_t* acc, int32_t* token, void* greedy, cudaStream_t s) {
  dfssm::Int8GemvArgs ia{W, s_row, V, d, h, logits, acc};
  ia.norm_w = norm_w;
  ia.greedy = static_cast<unsigned long long*>(greedy);
  ia.token = token;
  const cudaError_t e = dfssm::launch_int8_gemv(ia, s);
  return e == cudaSuccess ? DFSSM_OK : cuda_fail(e);
}

// Clock budget of one device-side wait of the fused decode kernel (about 1 s at 2 GHz).
constexpr long long kSpinLimitCycles = 2000000000LL;

// The current device is an sm_100 part (asked every call: the answer depends on the calling thread's
// current device, and the two runtime queries cost well under a microsecond).
bool device_ok() {
  int dev = 0, major = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess) {
    cudaGetLastError();
    return false;
  }
  return major == 10;
}

dfssm::GemvArgs gemv_args(const dfssm_linear_t* L, int B, const dfssm::QuantScratch& qs) {
  dfssm::GemvArgs g{};
  g.bits = L->bits;
  g.w_scale = L->w_scale;
  g.lora_a = L->lora_a;
  g.lora_a_scale = L->lora_a_scale;
  g.lora_b_scale = L->lora_b_scale;
  g.rank = L->rank;
  g.d_out = L->d_out;
  g.d_in = L->d_in;
  g.B = B;
  g.in = qs;
  return g;
}

// dfssm_layer_decode; with launch == false only the arguments are checked.
int layer_decode_impl(const dfssm_layer_t* layers, int n_layers, const dfssm_dims_t* dims, float* hidden,
                      float* const* conv_states, float* const* ssm_states, int B, void* workspace,
                      size_t ws_bytes, void* stream, bool launch) {
  if (!layers || !dims || !hidden || !conv_states || !ssm_states) return DFSSM_EINVAL;
  if (n_layers < 1 || B < 1) return DFSSM_EINVAL;
  if (n_layers > DFSSM_MAX_LAYERS || B > DFSSM_MAX_BATCH) return DFSSM_EUNSUPPORTED;
  const int Dm = dims->d_model, H = dims->nheads, P = dims->headdim, N = dims->d_state,
            G = dims->ngroups;
  if (Dm < 32 || Dm % 32 || H < 1 || P < 1 || N < 4 || G < 1 || H % G) return DFSSM_EINVAL;
  const int E = H * P;
  const int C = E + 2 * G * N;
  const int d_ip = 2 * E + 2 * G * N + H;
  if (E % 32 || N % 4 || N > 512 || Dm > 8192 || E > 8192 || 2 * G * N > 2048 || H > 1024)
    return DFSSM_EUNSUPPORTED;
  if (!aligned(hidden, 16)) return DFSSM_EALIGN;
  for (int l = 0; l < n_layers; ++l) {
    const dfssm_layer_t& Ly = layers[l];
    int st = dfssm::check_linear(&Ly.in_proj);
    if (st) return st;
    st = dfssm::check_linear(&Ly.out_proj);
    if (st) return st;
    if (Ly.in_proj.d_out != d_ip || Ly.in_proj.d_in != Dm || Ly.out_proj.d_out != Dm ||
        Ly.out_proj.d_in != E)
      return DFSSM_EINVAL;
    if (!Ly.conv_w || !Ly.conv_b || !Ly.A_log || !Ly.dt_bias || !Ly.D || !Ly.norm_w || !Ly.gnorm_w)
      return DFSSM_EINVAL;
    if (!conv_states[l] || !ssm_states[l]) return DFSSM_EINVAL;
    if (!aligned(Ly.conv_w, 16) || !aligned(ssm_states[l], 16)) return DFSSM_EALIGN;
  }
  if (!workspace || !aligned(workspace, 256) || ws_bytes < layer_ws_bytes(B, Dm, E, C, d_ip))
    return DFSSM_EWORKSPACE;
  if (!device_ok()) return DFSSM_EDEVICE;
  if (!launch) return DFSSM_OK;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (dfssm::fused_decode_supported(*dims, B, layers, n_layers, conv_states)) {
    const cudaError_t fe = dfssm::launch_fused_decode(layers, n_layers, hidden, conv_states, ssm_states,
                                                      workspace, s, kSpinLimitCycles);
    return fe == cudaSuccess ? DFSSM_OK : cuda_fail(fe);
  }
  LayerWs w = carve_layer_ws(workspace, B, Dm, E, C, d_ip);
  cudaError_t e = cudaSuccess;
  for (int l = 0; l < n_layers && e == cudaSuccess; ++l) {
    const dfssm_layer_t& Ly = layers[l];
    // pre-norm + quantize + LoRA-down
    dfssm::QuantArgs qa{};
    qa.x = hidden;
    qa.ldx = Dm;
    qa.norm_w = Ly.norm_w;
    qa.n = Dm;
    qa.B = B;
    qa.lora_b = Ly.in_proj.lora_b;
    qa.lora_b_scale = Ly.in_proj.lora_b_scale;
    qa.rank = Ly.in_proj.rank;
    qa.permute = true;
    qa.out = w.qs;
    e = dfssm::launch_quant(qa, s);
    if (e != cudaSuccess) break;
    // in_proj
    dfssm::GemvArgs ga = gemv_args(&Ly.in_proj, B, w.qs);
    ga.y = w.zxbcdt;
    ga.ldy = d_ip;
    e = dfssm::launch_gemv(ga, s);
    if (e != cudaSuccess) break;
    // conv over x|B|C
    dfssm::ConvArgs ca{conv_states[l], Ly.conv_w, Ly.conv_b, w.zxbcdt + E, d_ip, w.xc, C, B, C};
    e = dfssm::launch_conv(ca, s);
    if (e != cudaSuccess) break;
    // SSM + gate
    dfssm::SsmArgs sa{};
    sa.state = ssm_states[l];
    sa.x = w.xc;
    sa.ldx = C;
    sa.dt_raw = w.zxbcdt + E + C;
    sa.lddt = d_ip;
    sa.A_log = Ly.A_log;
    sa.dt_bias = Ly.dt_bias;
    sa.D = Ly.D;
    sa.Bm = w.xc + E;
    sa.Cm = w.xc + E + G * N;
    sa.ldbc = C;
    sa.y = w.g;
    sa.ldy = E;
    sa.z = w.zxbcdt;
    sa.ldz = d_ip;
    sa.B = B;
    sa.H = H;
    sa.P = P;
    sa.N = N;
    sa.G = G;
    e = dfssm::launch_ssm(sa, s);
    if (e != cudaSuccess) break;
    // gated norm + quantize + LoRA-down
    qa.x = w.g;
    qa.ldx = E;
    qa.norm_w = Ly.gnorm_w;
    qa.n = E;
    qa.lora_b = Ly.out_proj.lora_b;
    qa.lora_b_scale = Ly.out_proj.lora_b_scale;
    qa.rank = Ly.out_proj.rank;
    e = dfssm::launch_quant(qa, s);
    if (e != cudaSuccess) break;
    // out_proj + residual
    ga = gemv_args(&Ly.out_proj, B, w.qs);
    ga.resid = hidden;
    ga.ldr = Dm;
    e = dfssm::launch_gemv(ga, s);
  }
  return e == cudaSuccess ? DFSSM_OK : cuda_fail(e);
}

// Shared checks of the density-field entry points: DFSSM_OK or the status to return.
int check_field(int rows, int N) {
  if (rows < 0 || N < 8 || N % 8) return DFSSM_EINVAL;
  if (N > 256) return DFSSM_EUNSUPPORTED;
  return DFSSM_OK;
}

}  // namespace

// Argument checks of one linear descriptor: d_in a multiple of 32 (above 8192: unsupported), rank 0..16,
// the pointers present and aligned as the header states.
int dfssm::check_linear(const dfssm_linear_t* L) {
  if (!L) return DFSSM_EINVAL;
  if (L->d_out < 1 || L->d_in < 32 || L->d_in % 32 != 0) return DFSSM_EINVAL;
  if (L->d_in > 8192) return DFSSM_EUNSUPPORTED;
  if (L->rank < 0 || L->rank > DFSSM_MAX_RANK) return DFSSM_EINVAL;
  if (!L->bits || !L->w_scale) return DFSSM_EINVAL;
  if (L->rank > 0 && (!L->lora_b || !L->lora_b_scale || !L->lora_a || !L->lora_a_scale))
    return DFSSM_EINVAL;
  if (!aligned(L->bits, 16) || !aligned(L->w_scale, 4)) return DFSSM_EALIGN;
  if (L->rank > 0) {
    if (!aligned(L->lora_b, 4) || !aligned(L->lora_b_scale, 4) || !aligned(L->lora_a_scale, 4))
      return DFSSM_EALIGN;
    if (L->rank == DFSSM_MAX_RANK && !aligned(L->lora_a, 16)) return DFSSM_EALIGN;
  }
  return DFSSM_OK;
}

int dfssm::read_status_word(int* word, cudaStream_t st, int* code) {
  int h = 0;
  cudaError_t e = cudaMemcpyAsync(&h, word, sizeof(int), cudaMemcpyDeviceToHost, st);
  if (e == cudaSuccess) e = cudaStreamSynchronize(st);
  if (e == cudaSuccess) e = cudaMemsetAsync(word, 0, sizeof(int), st);
  if (e == cudaSuccess) e = cudaStreamSynchronize(st);
  *code = h;
  return e == cudaSuccess ? 0 : (int)e;
}

int dfssm::record_cuda_failure(cudaError_t e) { return cuda_fail(e); }

extern "C" {

int dfssm_abi_version(void) { return DFSSM_ABI_VERSION; }

const char* dfssm_status_string(int s) {
  switch (s) {
    case DFSSM_OK: return "ok";
    case DFSSM_EINVAL: return "invalid argument";
    case DFSSM_EALIGN: return "misaligned pointer";
    case DFSSM_EUNSUPPORTED: return "unsupported configuration";
    case DFSSM_ECUDA: return "CUDA error";
    case DFSSM_ETIMEOUT: return "device wait timed out";
    case DFSSM_EDEVICE: return "no usable sm_100 device";
    case DFSSM_EWORKSPACE: return "workspace missing, too small or misaligned";
    default: return "unknown status";
  }
}

const char* dfssm_last_cuda_error(void) { return g_last_cuda_error; }

size_t dfssm_workspace_size(int op, int a, int b, int c) {
  switch (op) {
    case DFSSM_OP_LINEAR_DECODE:
      if (a < 1 || a > DFSSM_MAX_BATCH || b < 32 || b % 32 || b > 8192) return 0;
      return linear_decode_ws(a, b);
    case DFSSM_OP_LINEAR_PREFILL:
      if (a < 1 || b < 128 || b % 128 || c < 1) return 0;
      return dfssm::prefill_workspace_bytes(a, b, c);
    case DFSSM_OP_LAYER_DECODE: {
      if (a < 1 || a > DFSSM_MAX_BATCH || b < 32 || c < 32) return 0;
      // conv channels and in_proj rows depend on d_state/ngroups/nheads; size for the largest
      // supported (2*ngroups*d_state <= 2048, nheads <= 1024).
      const int C = c + 2048, d_ip = 2 * c + 2048 + 1024;
      return layer_ws_bytes(a, b, c, C, d_ip);
    }
    case DFSSM_OP_LM_HEAD:
      if (b < 16 || b % 16 || b > 8192 || c < 1) return 0;
      return dfssm::quant_scratch_bytes(1, b);
    case DFSSM_OP_HEAD_GREEDY:
      if (b < 16 || b % 16 || b > 8192 || c < 1) return 0;
      return kGreedyBytes;
    case DFSSM_OP_GENERATE:
      if (a < 1 || b < 32 || b % 32 || b > 8192 || c < 32) return 0;
      return generate_ws(a, b, c).total;
    case DFSSM_OP_LAYER_PREFILL:
      if (a < 1 || b < 128 || b % 128 || b > 8192 || c < 128 || c % 128 || c > 8192) return 0;
      return prefill_layer_ws(a, b, c).total;
    case DFSSM_OP_LINEAR_MULTI:
    case DFSSM_OP_EMBED:
      return dfssm::kStatusBytes;
    default: return 0;
  }
}

int dfssm_pack_signs(const int8_t* signs, int d_out, int d_in, uint32_t* bits) {
  if (!signs || !bits || d_out < 1 || d_in < 32 || d_in % 32) return DFSSM_EINVAL;
  const int words = d_in / 32;
  for (int o = 0; o < d_out; ++o) {
    for (int w = 0; w < words; ++w) {
      uint32_t v = 0;
      for (int j = 0; j < 32; ++j)
        if (signs[(size_t)o * d_in + 32 * w + j] > 0) v |= (1u << j);
      bits[(size_t)o * words + w] = v;
    }
  }
  return DFSSM_OK;
}

int dfssm_linear_decode(const dfssm_linear_t* lin, const float* x, int B, float* y, void* workspace,
                        size_t ws_bytes, const dfssm_debug_t* dbg, void* stream) {
  int st = dfssm::check_linear(lin);
  if (st) return st;
  if (!x || !y || B < 1) return DFSSM_EINVAL;
  if (B > DFSSM_MAX_BATCH) return DFSSM_EUNSUPPORTED;
  if (!aligned(x, 16) || !aligned(y, 4)) return DFSSM_EALIGN;
  if (!workspace || !aligned(workspace, 256) || ws_bytes < linear_decode_ws(B, lin->d_in))
    return DFSSM_EWORKSPACE;
  if (!device_ok()) return DFSSM_EDEVICE;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (dfssm::stream_supported(lin->d_in, B))
    return dfssm::launch_linear_stream(lin, 1, x, B, &y, dbg, static_cast<int*>(workspace), s);
  dfssm::QuantScratch qs =
      dfssm::carve_quant_scratch(static_cast<char*>(workspace) + dfssm::kStatusBytes, B, lin->d_in);
  dfssm::QuantArgs qa{};
  qa.x = x;
  qa.ldx = lin->d_in;
  qa.norm_w = nullptr;
  qa.n = lin->d_in;
  qa.B = B;
  qa.lora_b = lin->lora_b;
  qa.lora_b_scale = lin->lora_b_scale;
  qa.rank = lin->rank;
  qa.permute = true;
  qa.out = qs;
  if (dbg) {
    qa.dbg_xq = dbg->xq;
    qa.dbg_s = dbg->xscale;
    qa.dbg_t = dbg->lora_t;
  }
  cudaError_t e = dfssm::launch_quant(qa, s);
  if (e != cudaSuccess) return cuda_fail(e);
  dfssm::GemvArgs ga = gemv_args(lin, B, qs);
  ga.y = y;
  ga.ldy = lin->d_out;
  ga.dbg_acc = dbg ? dbg->acc : nullptr;
  e = dfssm::launch_gemv(ga, s);
  if (e != cudaSuccess) return cuda_fail(e);
  return DFSSM_OK;
}

int dfssm_linear_decode_multi(const dfssm_linear_t* lins, int n, const float* x, int B, float* const* ys,
                              void* workspace, size_t ws_bytes, void* stream) {
  if (!lins || !ys || !x || n < 1 || B < 1) return DFSSM_EINVAL;
  if (n > DFSSM_MAX_LAYERS) return DFSSM_EUNSUPPORTED;
  for (int j = 0; j < n; ++j) {
    const int st = dfssm::check_linear(&lins[j]);
    if (st) return st;
    if (lins[j].d_in != lins[0].d_in) return DFSSM_EINVAL;
    if (!ys[j]) return DFSSM_EINVAL;
    if (!aligned(ys[j], 4)) return DFSSM_EALIGN;
  }
  if (!dfssm::stream_supported(lins[0].d_in, B)) return DFSSM_EUNSUPPORTED;
  if (!aligned(x, 16)) return DFSSM_EALIGN;
  if (!workspace || !aligned(workspace, 256) || ws_bytes < dfssm::kStatusBytes) return DFSSM_EWORKSPACE;
  if (!device_ok()) return DFSSM_EDEVICE;
  return dfssm::launch_linear_stream(lins, n, x, B, ys, nullptr, static_cast<int*>(workspace),
                                     static_cast<cudaStream_t>(stream));
}

int dfssm_conv_step(float* conv_state, const float* w, const float* b, const float* x_in, float* x_out,
                    int B, int C, void* stream) {
  if (!conv_state || !w || !b || !x_in || !x_out || B < 1 || C < 1) return DFSSM_EINVAL;
  if (!aligned(w, 16) || !aligned(conv_state, 4)) return DFSSM_EALIGN;
  if (!device_ok()) return DFSSM_EDEVICE;
  dfssm::ConvArgs a{conv_state, w, b, x_in, C, x_out, C, B, C};
  cudaError_t e = dfssm::launch_conv(a, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? DFSSM_OK : cuda_fail(e);
}

int dfssm_state_field_encode(const float* state, int rows, int N, uint32_t* field, float* scale,
                             void* stream) {
  const int st = check_field(rows, N);
  if (st || rows == 0) return st;
  if (!state || !field || !scale) return DFSSM_EINVAL;
  if (!aligned(state, 16) || !aligned(field, 4) || !aligned(scale, 4)) return DFSSM_EALIGN;
  if (!device_ok()) return DFSSM_EDEVICE;
  cudaError_t e = dfssm::launch_field_encode(state, nullptr, field, scale, rows, N,
                                             static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? DFSSM_OK : cuda_fail(e);
}

int dfssm_state_field_decode(const uint32_t* field, const float* scale, int rows, int N, float* state,
                             void* stream) {
  const int st = check_field(rows, N);
  if (st || rows == 0) return st;
  if (!state || !field || !scale) return DFSSM_EINVAL;
  if (!aligned(state, 16) || !aligned(field, 4) || !aligned(scale, 4)) return DFSSM_EALIGN;
  if (!device_ok()) return DFSSM_EDEVICE;
  cudaError_t e = dfssm::launch_field_decode(field, scale, rows, N, state, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? DFSSM_OK : cuda_fail(e);
}

int dfssm_state_field_roundtrip(float* state, int rows, int N, uint32_t* field, float* scale, void* stream) {
  const int st = check_field(rows, N);
  if (st || rows == 0) return st;
  if (!state || (field == nullptr) != (scale == nullptr)) return DFSSM_EINVAL;
  if (!aligned(state, 16) || !aligned(field, 4) || !aligned(scale, 4)) return DFSSM_EALIGN;
  if (!device_ok()) return DFSSM_EDEVICE;
  cudaError_t e = dfssm::launch_field_encode(state, state, field, scale, rows, N,
                                             static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? DFSSM_OK : cuda_fail(e);
}

int dfssm_ssm_step(float* ssm_state, const float* x, const float* dt_raw, const float* A_log,
                   const float* dt_bias, const float* D, const float* Bm, const float* Cm, float* y,
                   int B, int H, int P, int N, int G, void* stream) {
  if (!ssm_state || !x || !dt_raw || !A_log || !dt_bias || !D || !Bm || !Cm || !y) return DFSSM_EINVAL;
  if (B < 1 || H < 1 || P < 1 || N < 4 || G < 1 || H % G) return DFSSM_EINVAL;
  if (N % 4 || N > 512) return DFSSM_EUNSUPPORTED;
  if (!aligned(ssm_state, 16) || !aligned(Bm, 16) || !aligned(Cm, 16)) return DFSSM_EALIGN;
  if (!device_ok()) return DFSSM_EDEVICE;
  dfssm::SsmArgs a{};
  a.state = ssm_state;
  a.x = x;
  a.ldx = H * P;
  a.dt_raw = dt_raw;
  a.lddt = H;
  a.A_log = A_log;
  a.dt_bias = dt_bias;
  a.D = D;
  a.Bm = Bm;
  a.Cm = Cm;
  a.ldbc = G * N;
  a.y = y;
  a.ldy = H * P;
  a.z = nullptr;
  a.B = B;
  a.H = H;
  a.P = P;
  a.N = N;
  a.G = G;
  cudaError_t e = dfssm::launch_ssm(a, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? DFSSM_OK : cuda_fail(e);
}

int dfssm_layer_decode(const dfssm_layer_t* layers, int n_layers, const dfssm_dims_t* dims,
                       float* hidden, float* const* conv_states, float* const* ssm_states, int B,
                       void* workspace, size_t ws_bytes, void* stream) {
  return layer_decode_impl(layers, n_layers, dims, hidden, conv_states, ssm_states, B, workspace,
                           ws_bytes, stream, true);
}

int dfssm_device_status(void* workspace, void* stream) {
  if (workspace && !aligned(workspace, 256)) return DFSSM_EWORKSPACE;
  if (!device_ok()) return DFSSM_EDEVICE;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  int* word = static_cast<int*>(workspace);
  if (!word) {
    const int st = dfssm::noalloc_status_word(&word);
    if (st) return st;
  }
  int code = 0;
  const int e = dfssm::read_status_word(word, s, &code);
  if (e) return cuda_fail(static_cast<cudaError_t>(e));
  if (code == dfssm::kBadTokenCode) return DFSSM_EINVAL;
  return code ? DFSSM_ETIMEOUT : DFSSM_OK;
}

int dfssm_selftest_timeout(void* workspace, size_t ws_bytes, void* stream) {
  if (!workspace || !aligned(workspace, 256) || ws_bytes < dfssm::fused_decode_workspace_bytes())
    return DFSSM_EWORKSPACE;
  if (!device_ok()) return DFSSM_EDEVICE;
  const cudaError_t e =
      dfssm::launch_timeout_selftest(workspace, static_cast<cudaStream_t>(stream), 2000000LL);
  return e == cudaSuccess ? DFSSM_OK : cuda_fail(e);
}

int dfssm_lm_head(const int8_t* W, const float* s_row, int V, int d, const float* x, float* logits,
                  int32_t* acc, void* workspace, size_t ws_bytes, void* stream) {
  if (!W || !s_row || !x || !logits || V < 1 || d < 16 || d % 16) return DFSSM_EINVAL;
  if (d > 8192) return DFSSM_EUNSUPPORTED;
  if (!aligned(W, 16) || !aligned(x, 4)) return DFSSM_EALIGN;
  (void)workspace;  // the kernel quantizes the token itself; the workspace is no longer used
  (void)ws_bytes;
  if (!device_ok()) return DFSSM_EDEVICE;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  dfssm::Int8GemvArgs ia{W, s_row, V, d, x, logits, acc};
  const cudaError_t e = dfssm::launch_int8_gemv(ia, s);
  return e == cudaSuccess ? DFSSM_OK : cuda_fail(e);
}

int dfssm_embed(const int8_t* W, const float* s_row, int V, int d, const int32_t* token, float* h,
                void* workspace, size_t ws_bytes, void* stream) {
  int st = check_head(W, s_row, V, d);
  if (st) return st;
  if (!token || !h) return DFSSM_EINVAL;
  if (!aligned(token, 4) || !aligned(h, 16)) return DFSSM_EALIGN;
  if (!workspace || !aligned(workspace, 256) || ws_bytes < dfssm::kStatusBytes) return DFSSM_EWORKSPACE;
  if (!device_ok()) return DFSSM_EDEVICE;
  return enqueue_embed(W, s_row, V, d, token, h, static_cast<int*>(workspace),
                       static_cast<cudaStream_t>(stream));
}

int dfssm_head_greedy(const int8_t* W, const float* s_row, int V, int d, const float* h,
                      const float* norm_w, float* logits, int32_t* acc, int32_t* token, void* workspace,
                      size_t ws_bytes, void* stream) {
  int st = check_head(W, s_row, V, d);
  if (st) return st;
  if (!h || !logits || !token) return DFSSM_EINVAL;
  if (!aligned(h, 4) || !aligned(token, 4) || (norm_w && !aligned(norm_w, 4))) return DFSSM_EALIGN;
  if (!workspace || !aligned(workspace, 256) || ws_bytes < kGreedyBytes) return DFSSM_EWORKSPACE;
  if (!device_ok()) return DFSSM_EDEVICE;
  return enqueue_head(W, s_row, V, d, h, norm_w, logits, acc, token, workspace,
                      static_cast<cudaStream_t>(stream));
}

int dfssm_generate(const dfssm_layer_t* layers, int n_layers, const dfssm_dims_t* dims,
                   const int8_t* W, const float* s_row, int V, const float* final_norm_w,
                   int32_t* tokens, int n_tokens, float* const* conv_states, float* const* ssm_states,
                   float* hidden_taps, float* logits, void* workspace, size_t ws_bytes, void* stream) {
  if (!dims || !tokens || !final_norm_w || n_tokens < 1) return DFSSM_EINVAL;
  const int Dm = dims->d_model, E = dims->nheads * dims->headdim;
  int st = check_head(W, s_row, V, Dm);
  if (st) return st;
  if (!aligned(tokens, 4) || !aligned(final_norm_w, 4) || (hidden_taps && !aligned(hidden_taps, 4)) ||
      (logits && !aligned(logits, 4)))
    return DFSSM_EALIGN;
  if (Dm < 32 || Dm % 32 || E < 32) return DFSSM_EINVAL;
  const GenerateWs g = generate_ws(V, Dm, E);
  if (!workspace || !aligned(workspace, 256) || ws_bytes < g.total) return DFSSM_EWORKSPACE;
  char* base = static_cast<char*>(workspace);
  float* hidden = reinterpret_cast<float*>(base + g.hidden);
  float* lg = reinterpret_cast<float*>(base + g.logits);
  void* greedy = base + g.greedy;
  st = layer_decode_impl(layers, n_layers, dims, hidden, conv_states, ssm_states, 1, base + g.layer,
                         g.hidden, stream, false);
  if (st) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  for (int t = 0; t < n_tokens; ++t) {
    st = enqueue_embed(W, s_row, V, Dm, tokens + t, hidden, reinterpret_cast<int*>(base + g.layer), s);
    if (st) return st;
    st = layer_decode_impl(layers, n_layers, dims, hidden, conv_states, ssm_states, 1, base + g.layer,
                           g.hidden, stream, true);
    if (st) return st;
    if (hidden_taps) {
      const cudaError_t e = cudaMemcpyAsync(hidden_taps + (size_t)t * Dm, hidden, sizeof(float) * Dm,
                                            cudaMemcpyDeviceToDevice, s);
      if (e != cudaSuccess) return cuda_fail(e);
    }
    st = enqueue_head(W, s_row, V, Dm, hidden, final_norm_w, lg, nullptr, tokens + t + 1, greedy, s);
    if (st) return st;
  }
  if (logits) {
    const cudaError_t e =
        cudaMemcpyAsync(logits, lg, sizeof(float) * (size_t)V, cudaMemcpyDeviceToDevice, s);
    if (e != cudaSuccess) return cuda_fail(e);
  }
  return DFSSM_OK;
}

int dfssm_layer_prefill(const dfssm_layer_t* layers, int n_layers, const dfssm_dims_t* dims,
                        float* hidden, float* const* conv_states, float* const* ssm_states, int M,
                        void* workspace, size_t ws_bytes, void* stream) {
  if (!layers || !dims || !hidden || !conv_states || !ssm_states || n_layers < 1 || M < 1)
    return DFSSM_EINVAL;
  if (n_layers > DFSSM_MAX_LAYERS) return DFSSM_EUNSUPPORTED;
  const int Dm = dims->d_model, H = dims->nheads, P = dims->headdim, N = dims->d_state, G = dims->ngroups;
  if (Dm < 32 || H < 1 || P < 1 || N < 4 || G < 1 || H % G) return DFSSM_EINVAL;
  const int E = H * P;
  const int C = E + 2 * G * N;
  const int d_ip = 2 * E + 2 * G * N + H;
  if (Dm % 128 || E % 128 || Dm > 8192 || E > 8192 || 2 * G * N > 2048 || H > 1024 ||
      !dfssm::scan_supported(H, P, N, G))
    return DFSSM_EUNSUPPORTED;
  if (!aligned(hidden, 16)) return DFSSM_EALIGN;
  for (int l = 0; l < n_layers; ++l) {
    const dfssm_layer_t& Ly = layers[l];
    int st = dfssm::check_linear(&Ly.in_proj);
    if (st) return st;
    st = dfssm::check_linear(&Ly.out_proj);
    if (st) return st;
    if (Ly.in_proj.d_out != d_ip || Ly.in_proj.d_in != Dm || Ly.out_proj.d_out != Dm ||
        Ly.out_proj.d_in != E)
      return DFSSM_EINVAL;
    if (!Ly.conv_w || !Ly.conv_b || !Ly.A_log || !Ly.dt_bias || !Ly.D || !Ly.norm_w || !Ly.gnorm_w)
      return DFSSM_EINVAL;
    if (!conv_states[l] || !ssm_states[l]) return DFSSM_EINVAL;
    if (!aligned(Ly.conv_w, 16) || !aligned(ssm_states[l], 16) || !aligned(Ly.norm_w, 16) ||
        !aligned(Ly.gnorm_w, 16))
      return DFSSM_EALIGN;
  }
  const PrefillLayerWs w = prefill_layer_ws(M, Dm, E);
  if (!workspace || !aligned(workspace, 256) || ws_bytes < w.total) return DFSSM_EWORKSPACE;
  if (!device_ok()) return DFSSM_EDEVICE;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  char* base = static_cast<char*>(workspace);
  float* zx = reinterpret_cast<float*>(base + w.zx);
  float* xc = reinterpret_cast<float*>(base + w.xc);
  float* g = reinterpret_cast<float*>(base + w.g);
  void* lin_ws = base + w.lin;
  const size_t lin_bytes = ws_bytes - w.lin;
  int* status = reinterpret_cast<int*>(base);
  for (int l = 0; l < n_layers; ++l) {
    const dfssm_layer_t& Ly = layers[l];
    int st = dfssm::linear_prefill_impl(&Ly.in_proj, hidden, M, zx, Ly.norm_w, false, lin_ws, lin_bytes,
                                        status, nullptr, stream);
    if (st) return st;
    dfssm::ConvSeqArgs ca{zx, d_ip, E, conv_states[l], Ly.conv_w, Ly.conv_b, xc, M, C};
    cudaError_t e = dfssm::launch_conv_seq(ca, s);
    if (e != cudaSuccess) return cuda_fail(e);
    dfssm::ScanArgs sa{};
    sa.zx = zx;
    sa.ld_zx = d_ip;
    sa.dt_off = E + C;
    sa.xc = xc;
    sa.ld_xc = C;
    sa.b_off = E;
    sa.c_off = E + G * N;
    sa.A_log = Ly.A_log;
    sa.dt_bias = Ly.dt_bias;
    sa.D = Ly.D;
    sa.state = ssm_states[l];
    sa.g = g;
    sa.sz = reinterpret_cast<float*>(base + w.sz);
    sa.dtdA = reinterpret_cast<float*>(base + w.dtdA);
    sa.M = M;
    sa.H = H;
    sa.P = P;
    sa.N = N;
    sa.G = G;
    e = dfssm::launch_ssm_scan(sa, s);
    if (e != cudaSuccess) return cuda_fail(e);
    st = dfssm::linear_prefill_impl(&Ly.out_proj, g, M, hidden, Ly.gnorm_w, true, lin_ws, lin_bytes,
                                    status, nullptr, stream);
    if (st) return st;
  }
  return DFSSM_OK;
}

}  // extern "C"
