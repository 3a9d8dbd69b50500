// DF-SSM CPU oracle — TEST INFRASTRUCTURE ONLY.
//
// A plain, slow, scalar C++ statement of what the DF-SSM decode/prefill hot path computes.  Only the
// test-suite, the package's smoke check and the benchmark's CPU-baseline leg may load this file's
// library; the product path never does.  It shares no code, header, table or helper with the CUDA
// library under bit_quantized_mamba_b200/csrc, and neither side includes or links the other.
//
// Sources (the method is described only in prose; no equations are printed):
//   [ABS]   "Density Field State Space Models: 1-Bit Distillation, Efficient Inference, and Knowledge
//           Organization in Mamba-2" (arXiv 2606.10932), abstract.
//   [TS-2B] gist.science technical summary of the same paper, §2.B "Frozen Scaffold with LoRA Correction".
//   [TS-2C] same summary, §2.C "Optimized Inference Pipeline".
//   [TS-2D] same summary, §2.D "Density Field State Representation".
//   [TS-3]  same summary, §3 "Key Results" (model size and composition).
//   [MAP]   mlsanity.com citation map of the paper, "Builds on": Mamba; "Transformers are SSMs ...
//           Structured State Space Duality" (Mamba-2 / SSD).  The Mamba-2 block itself is only cited,
//           so every Mamba-2 equation below is a READING of that cited architecture.
//
// Arithmetic convention (a reading; the pages fix the stored precision — int8 activations, int32
// accumulation, fp32 state/activations [TS-2C], [TS-3] "Other (FP16/FP32)" — but not the rounding
// sequence):
//   * every fp32 value the method stores is the fp32 rounding of an expression evaluated in fp64;
//   * a single fp32 operation (a*b, a+b, a/b) is written (float)((double)a OP (double)b); for these
//     operations double rounding through fp64 is innocuous (53 >= 2*24+2), so this equals the IEEE
//     fp32 operation;
//   * sums of more than two terms are accumulated in fp64 in index order and rounded once;
//   * transcendental functions (exp, log1p, sqrt) are evaluated in fp64 and rounded once to fp32.
// The library must therefore be built with -ffp-contract=off (no fused multiply-add).
//
// Parity status per function is stated in each header comment ("pinned by" / "parity unpinned").

#include <omp.h>

#include <cmath>
#include <cstdint>
#include <cstdlib>
#include <cstring>
#include <vector>

namespace {

inline float r32(double v) { return (float)v; }

// [TS-2C] "1-bit packed weights": reading (i) — row-major words, d_in/32 words per row, bit j of word
// w is input 32*w+j (least significant bit first); a set bit means +1, a clear bit means -1.
inline int unpack_sign(const uint32_t* bits, int d_in, int o, int i) {
  const uint32_t w = bits[(size_t)o * (size_t)(d_in / 32) + (size_t)(i / 32)];
  return ((w >> (i % 32)) & 1u) ? 1 : -1;
}

// Per-token absmax int8 quantizer (the activation side of the "INT8 tensor cores" scaffold matmul,
// [TS-2C]).  Reading (ii): s = absmax/127 in fp32, q = clamp(rint(v/s), -127, 127) with an fp32
// division and round-half-to-even; an all-zero row gives s = 0 and q = 0.
void quantize_row(const float* v, int n, int8_t* q, float* s_out) {
  float m = 0.0f;
  for (int i = 0; i < n; ++i) {
    const float a = std::fabs(v[i]);
    if (a > m) m = a;
  }
  if (m == 0.0f) {
    for (int i = 0; i < n; ++i) q[i] = 0;
    *s_out = 0.0f;
    return;
  }
  const float s = r32((double)m / 127.0);
  for (int i = 0; i < n; ++i) {
    const float ratio = r32((double)v[i] / (double)s);
    float k = std::nearbyint(ratio);  // default rounding mode: nearest, ties to even
    if (k > 127.0f) k = 127.0f;
    if (k < -127.0f) k = -127.0f;
    q[i] = (int8_t)k;
  }
  *s_out = s;
}

// LoRA down-projection ([TS-2B]: a rank-16 LoRA module W_A (W_B x) with int8 matrices and per-row
// scales, applied to the layer input; [TS-2C]: the linear's input is the per-token int8 activation of the
// INT8 scaffold matmul).  Reading (iii): W_B multiplies the same int8 codes q as the scaffold, with int32
// accumulation, and the intermediate stays fp32 (it is not requantized):
//   t[r]  = sum_i W_B[r,i] * q[i]              (exact integer; |t| <= 127*127*d_in fits int32)
//   tf[r] = fl32(t[r] * sB[r] * s)             (fp64, this order; s the input's quantizer scale)
void lora_down(int d_in, int rank, const int8_t* lora_b, const float* lora_b_scale, const int8_t* q,
               float s, int32_t* t_out, float* tf) {
  for (int r = 0; r < rank; ++r) {
    int64_t t = 0;
    for (int i = 0; i < d_in; ++i) t += (int64_t)lora_b[(size_t)r * d_in + i] * (int64_t)q[i];
    if (t_out) t_out[r] = (int32_t)t;
    tf[r] = r32((double)t * (double)lora_b_scale[r] * (double)s);
  }
}

// Scaffold + LoRA-up on an already-quantized row ([TS-2B], [TS-2C]); reading (iv): per-row scales for
// W_B (rank rows) and W_A (d_out rows).
//   acc[o] = sum_i sign(o,i) * q[i]                       (exact integer; fits int32)
//   y[o]   = fl32(acc[o]*s*sW[o] + sA[o] * sum_r W_A[o,r]*tf[r])
void linear_core(int d_out, int d_in, int rank, const uint32_t* bits, const float* w_scale,
                 const int8_t* lora_a, const float* lora_a_scale, const int8_t* q, float s,
                 const float* tf, int32_t* acc_out, float* y) {
#pragma omp parallel for schedule(static)
  for (int o = 0; o < d_out; ++o) {
    int64_t a = 0;
    for (int i = 0; i < d_in; ++i) a += (int64_t)unpack_sign(bits, d_in, o, i) * (int64_t)q[i];
    if (acc_out) acc_out[o] = (int32_t)a;
    double lora = 0.0;
    for (int r = 0; r < rank; ++r) lora += (double)lora_a[(size_t)o * rank + r] * (double)tf[r];
    const double scaffold = (double)a * (double)s * (double)w_scale[o];
    const double corr = rank > 0 ? (double)lora_a_scale[o] * lora : 0.0;
    y[o] = r32(scaffold + corr);
  }
}

// Mamba-2 RMSNorm (reading: eps = 1e-5, one weight per channel) followed by the per-token quantizer,
// each exactly as defined, one after the other:
//   r   = fl32(1 / sqrt(sum_i h_i^2 / n + eps))     (fp64; the sum in index order, the squares exact)
//   u_i = fl32(fl32(h_i * r) * w_i)                  (the normalized, weighted row, stored fp32)
//   (q, s) = quantize(u)                             (quantize_row above)
// Writes u to u_out and returns r.
float rmsnorm_quantize(const float* h, const float* w, int n, double eps, int8_t* q, float* s_out,
                       float* u_out) {
  double ss = 0.0;
  for (int i = 0; i < n; ++i) ss += (double)h[i] * (double)h[i];
  const float r = r32(1.0 / std::sqrt(ss / (double)n + eps));
  for (int i = 0; i < n; ++i) u_out[i] = r32((double)r32((double)h[i] * (double)r) * (double)w[i]);
  quantize_row(u_out, n, q, s_out);
  return r;
}

inline double silu64(double v) { return v / (1.0 + std::exp(-v)); }

}  // namespace

extern "C" {

int oracle_abi_version(void) { return 6; }

// Host threads the OpenMP loops of this library use (timing of the CPU baseline); returns the previous
// maximum.  No arithmetic.
int oracle_set_threads(int n) {
  const int prev = omp_get_max_threads();
  if (n > 0) omp_set_num_threads(n);
  return prev;
}

// Pinned by: exhaustive byte-pattern round trip against an independent packer, brute force.
int oracle_sign(const uint32_t* bits, int d_in, int o, int i) { return unpack_sign(bits, d_in, o, i); }

// Pinned by: absmax maps to +-127, reconstruction error <= s/2, power-of-two scale invariance, zero row,
// agreement with numpy fp32 division.
void oracle_quantize(const float* x, int B, int n, int8_t* q, float* s) {
  for (int b = 0; b < B; ++b) quantize_row(x + (size_t)b * n, n, q + (size_t)b * n, s + b);
}

// dfssm linear decode: quantize each of the B rows of x, then the scaffold + LoRA linear.
// Pinned by: brute-force +-1 integer matmul, 2*sum_{bit=1} q - sum q identity, bit-flip negation,
// one-hot inputs, rank-0 == scaffold alone, W_A == 0 == scaffold alone, one-hot W_B rows, brute-force
// integer LoRA-down, the real-number epilogue formula.
void oracle_linear_decode(int d_out, int d_in, int rank, const uint32_t* bits, const float* w_scale,
                          const int8_t* lora_b, const float* lora_b_scale, const int8_t* lora_a,
                          const float* lora_a_scale, const float* x, int B, float* y,
                          int32_t* acc, int32_t* t_out, int8_t* xq, float* xscale) {
  std::vector<int8_t> q((size_t)d_in);
  std::vector<float> tf((size_t)(rank > 0 ? rank : 1));
  for (int b = 0; b < B; ++b) {
    float s = 0.0f;
    quantize_row(x + (size_t)b * d_in, d_in, q.data(), &s);
    if (xq) std::memcpy(xq + (size_t)b * d_in, q.data(), (size_t)d_in);
    if (xscale) xscale[b] = s;
    lora_down(d_in, rank, lora_b, lora_b_scale, q.data(), s, t_out ? t_out + (size_t)b * rank : nullptr,
              tf.data());
    linear_core(d_out, d_in, rank, bits, w_scale, lora_a, lora_a_scale, q.data(), s, tf.data(),
                acc ? acc + (size_t)b * d_out : nullptr, y + (size_t)b * d_out);
  }
}

// LoRA down-projection alone (see lora_down): t[r] and tf[r] for codes q with scale s.
void oracle_lora_down(int d_in, int rank, const int8_t* lora_b, const float* lora_b_scale,
                      const int8_t* q, float s, int32_t* t, float* tf) {
  lora_down(d_in, rank, lora_b, lora_b_scale, q, s, t, tf);
}

// Scaffold + LoRA-up on pre-quantized codes q with scale s and LoRA intermediate tf (teacher-forced and
// sampled checks).
void oracle_linear_core(int d_out, int d_in, int rank, const uint32_t* bits, const float* w_scale,
                        const int8_t* lora_a, const float* lora_a_scale, const int8_t* q, float s,
                        const float* tf, int32_t* acc, float* y) {
  linear_core(d_out, d_in, rank, bits, w_scale, lora_a, lora_a_scale, q, s, tf, acc, y);
}

// Sampled rows of the linear: only output rows listed in `rows` are computed (y[k] for rows[k]).
// Used for the full-size prefill and multi-copy checks, where a whole oracle pass is too slow.
void oracle_linear_rows(int d_out, int d_in, int rank, const uint32_t* bits, const float* w_scale,
                        const int8_t* lora_a, const float* lora_a_scale, const int8_t* q, float s,
                        const float* tf, const int* rows, int n_rows, int32_t* acc, float* y) {
  (void)d_out;
  for (int k = 0; k < n_rows; ++k) {
    const int o = rows[k];
    int64_t a = 0;
    for (int i = 0; i < d_in; ++i) a += (int64_t)unpack_sign(bits, d_in, o, i) * (int64_t)q[i];
    double lora = 0.0;
    for (int r = 0; r < rank; ++r) lora += (double)lora_a[(size_t)o * rank + r] * (double)tf[r];
    const double scaffold = (double)a * (double)s * (double)w_scale[o];
    const double corr = rank > 0 ? (double)lora_a_scale[o] * lora : 0.0;
    if (acc) acc[k] = (int32_t)a;
    y[k] = r32(scaffold + corr);
  }
}

// Width-4 stateful shift-register causal convolution, one decode step ([TS-2C] "stateful shift
// register"; width 4 and SiLU from the Mamba-2 block [MAP]).  Readings (vi): the state holds the last
// three inputs, oldest first; w[c][3] multiplies the current input; a bias is present.
//   pre = fl32(b[c] + w[c,0]*st0 + w[c,1]*st1 + w[c,2]*st2 + w[c,3]*x)   (fp64, this order)
//   out = fl32(pre / (1 + exp(-pre)))                                      (SiLU, fp64)
//   state <- (st1, st2, x)
// Pinned by: the stepped register equals the textbook causal 1-D convolution of a whole sequence;
// an impulse reproduces the taps.
void oracle_conv_step(float* conv_state, const float* w, const float* bias, const float* x_in,
                      float* x_out, int B, int C) {
  for (int b = 0; b < B; ++b) {
    for (int c = 0; c < C; ++c) {
      float* st = conv_state + ((size_t)b * C + c) * 3;
      const float xv = x_in[(size_t)b * C + c];
      const float* wc = w + (size_t)c * 4;
      double e = (double)bias[c];
      e += (double)wc[0] * (double)st[0];
      e += (double)wc[1] * (double)st[1];
      e += (double)wc[2] * (double)st[2];
      e += (double)wc[3] * (double)xv;
      const float pre = r32(e);
      x_out[(size_t)b * C + c] = r32(silu64((double)pre));
      st[0] = st[1];
      st[1] = st[2];
      st[2] = xv;
    }
  }
}

// Mamba-2 selective-SSM state update and readout for one decode step ([TS-2C] "SSM recurrence";
// the equations are the cited Mamba-2/SSD layer [MAP], a reading):
//   v   = fl32(dt_raw[h] + dt_bias[h]);  dt = fl32(softplus(v))  with softplus(v) = v for v > 20,
//         else log1p(exp(v))  (reading (vii), no dt clamp)
//   A   = fl32(-exp(A_log[h]));  dA = fl32(exp(fl32(dt*A)))
//   dtx = fl32(dt * x[h,p])
//   S[h,p,n] <- fl32( fl32(dA*S[h,p,n]) + fl32(dtx*B[g,n]) )
//   y[h,p]   =  fl32( sum_n S[h,p,n]*C[g,n] + D[h]*x[h,p] )        (fp64 sum, index order)
// with g = h / (H/G) the head's group.
// Pinned by: the stepped recurrence equals the quadratic (SSD "dual") form of the same model over a
// sequence; constant input gives the geometric closed form; dt -> 0 freezes the state; dA -> 0 makes it
// memoryless.
void oracle_ssm_step(float* ssm_state, const float* x, const float* dt_raw, const float* A_log,
                     const float* dt_bias, const float* D, const float* Bm, const float* Cm, float* y,
                     int B, int H, int P, int N, int G) {
  const int heads_per_group = H / G;
  for (int b = 0; b < B; ++b) {
    for (int h = 0; h < H; ++h) {
      const int g = h / heads_per_group;
      const float v = r32((double)dt_raw[(size_t)b * H + h] + (double)dt_bias[h]);
      const float dt = r32(v > 20.0f ? (double)v : std::log1p(std::exp((double)v)));
      const float A = r32(-std::exp((double)A_log[h]));
      const float dA = r32(std::exp((double)r32((double)dt * (double)A)));
      const float* Bg = Bm + ((size_t)b * G + g) * N;
      const float* Cg = Cm + ((size_t)b * G + g) * N;
      for (int p = 0; p < P; ++p) {
        const float xv = x[(size_t)b * H * P + (size_t)h * P + p];
        const float dtx = r32((double)dt * (double)xv);
        float* S = ssm_state + (((size_t)b * H + h) * P + p) * N;
        double acc = 0.0;
        for (int n = 0; n < N; ++n) {
          const float decayed = r32((double)dA * (double)S[n]);
          const float inject = r32((double)dtx * (double)Bg[n]);
          const float s_new = r32((double)decayed + (double)inject);
          S[n] = s_new;
          acc += (double)s_new * (double)Cg[n];
        }
        y[(size_t)b * H * P + (size_t)h * P + p] = r32(acc + (double)D[h] * (double)xv);
      }
    }
  }
}

// RMSNorm + per-token quantization of B rows (rmsnorm_quantize); also returns the normalized rows
// u [B][n] and the factors r [B].
// Pinned by: r against the correctly rounded fp32 of the real-number factor (exact decimal arithmetic);
// u against the real-number normalization to fp32 accuracy; the codes and scale are the pinned
// quantizer's on u; a constant row gives w*sign(c)/sqrt(1 + eps/c^2); a zero weight zeroes a code.
void oracle_rmsnorm_quantize(const float* h, const float* w, int B, int n, int8_t* q, float* s,
                             float* u, float* r) {
  for (int b = 0; b < B; ++b) {
    const float rb = rmsnorm_quantize(h + (size_t)b * n, w, n, 1e-5, q + (size_t)b * n, s + b,
                                      u + (size_t)b * n);
    if (r) r[b] = rb;
  }
}

// Gate of the Mamba-2 output: g = fl32(y * fl32(SiLU(z))) (reading (ix): gate before the norm).
// Pinned by: SiLU against a library logistic function.
void oracle_gate(const float* y, const float* z, float* g, int n) {
  for (int i = 0; i < n; ++i) {
    const float sz = r32(silu64((double)z[i]));
    g[i] = r32((double)y[i] * (double)sz);
  }
}

// One Mamba-2 layer decode step with the DF-SSM linears, B rows, the layer's residual stream h
// updated in place.  Wiring (reading; the Mamba-2 block [MAP] with the DF-SSM linears [TS-2B]):
//   (q, s)  = rmsnorm_quantize(h, norm_w);  tf = lora_down(q, s)
//   zxbcdt  = in_proj(q, s, tf)                  (reading (v): order z | x | B | C | dt)
//   xc      = conv_step(xBC)                     (SiLU applied to x, B and C channels)
//   y       = ssm_step(xc.x, dt, xc.B, xc.C)
//   g       = gate(y, z);  (q', s') = rmsnorm_quantize(g, gnorm_w);  tf' = lora_down(q', s')
//   h       = fl32(h + out_proj(q', s', tf'))
// Shapes: D = d_model, E = d_inner = H*P, C = E + 2*G*N conv channels, in_proj rows 2E + 2GN + H.
// Pinned by: the whole step written out by hand in float64 from the definitions for one head of 32
// channels with d_state 1 over four tokens (and over a five-token prompt through two layers); a zero
// out_proj scale leaves h unchanged.
void oracle_layer_decode(int B, int Dm, int H, int P, int N, int G, int rank,
                         // in_proj
                         const uint32_t* in_bits, const float* in_ws, const int8_t* in_lb,
                         const float* in_lbs, const int8_t* in_la, const float* in_las,
                         // out_proj
                         const uint32_t* out_bits, const float* out_ws, const int8_t* out_lb,
                         const float* out_lbs, const int8_t* out_la, const float* out_las,
                         const float* conv_w, const float* conv_b, const float* A_log,
                         const float* dt_bias, const float* Dskip, const float* norm_w,
                         const float* gnorm_w, float* h, float* conv_state, float* ssm_state,
                         // optional per-layer taps (may be NULL): zxbcdt [B][d_in_proj], y [B][E]
                         float* tap_zxbcdt, float* tap_y) {
  const int E = H * P;
  const int C = E + 2 * G * N;
  const int d_ip = 2 * E + 2 * G * N + H;
  std::vector<int8_t> q((size_t)(E > Dm ? E : Dm));
  std::vector<float> v((size_t)(E > Dm ? E : Dm));
  std::vector<float> zx((size_t)d_ip), xbc((size_t)C), xc((size_t)C), dt((size_t)H), y((size_t)E),
      g((size_t)E), out((size_t)Dm), tf((size_t)(rank > 0 ? rank : 1));
  for (int b = 0; b < B; ++b) {
    float* hb = h + (size_t)b * Dm;
    float s = 0.0f;
    rmsnorm_quantize(hb, norm_w, Dm, 1e-5, q.data(), &s, v.data());
    lora_down(Dm, rank, in_lb, in_lbs, q.data(), s, nullptr, tf.data());
    linear_core(d_ip, Dm, rank, in_bits, in_ws, in_la, in_las, q.data(), s, tf.data(), nullptr,
                zx.data());
    if (tap_zxbcdt) std::memcpy(tap_zxbcdt + (size_t)b * d_ip, zx.data(), sizeof(float) * d_ip);
    std::memcpy(xbc.data(), zx.data() + E, sizeof(float) * C);
    std::memcpy(dt.data(), zx.data() + E + C, sizeof(float) * H);
    oracle_conv_step(conv_state + (size_t)b * C * 3, conv_w, conv_b, xbc.data(), xc.data(), 1, C);
    oracle_ssm_step(ssm_state + (size_t)b * H * P * N, xc.data(), dt.data(), A_log, dt_bias, Dskip,
                    xc.data() + E, xc.data() + E + G * N, y.data(), 1, H, P, N, G);
    if (tap_y) std::memcpy(tap_y + (size_t)b * E, y.data(), sizeof(float) * E);
    oracle_gate(y.data(), zx.data(), g.data(), E);
    rmsnorm_quantize(g.data(), gnorm_w, E, 1e-5, q.data(), &s, v.data());
    lora_down(E, rank, out_lb, out_lbs, q.data(), s, nullptr, tf.data());
    linear_core(Dm, E, rank, out_bits, out_ws, out_la, out_las, q.data(), s, tf.data(), nullptr,
                out.data());
    for (int i = 0; i < Dm; ++i) hb[i] = r32((double)hb[i] + (double)out[i]);
  }
}

// Int8 per-row-scaled LM head on one token (reading (xii)): quantize x per token, then
//   logits[v] = fl32(acc[v] * s * s_row[v]),  acc[v] = sum_i W[v,i] * q[i].
// [TS-2B] "embedding/LM head matrices are quantized to int8 with per-channel/row scaling".
// Pinned by: brute-force int64 matmul.  Only rows listed in `rows` are computed when rows != NULL.
void oracle_lm_head(const int8_t* W, const float* s_row, int V, int d, const float* x,
                    const int* rows, int n_rows, float* logits, int32_t* acc_out) {
  std::vector<int8_t> q((size_t)d);
  float s = 0.0f;
  quantize_row(x, d, q.data(), &s);
  const int count = rows ? n_rows : V;
#pragma omp parallel for schedule(static)
  for (int k = 0; k < count; ++k) {
    const int vrow = rows ? rows[k] : k;
    int64_t a = 0;
    for (int i = 0; i < d; ++i) a += (int64_t)W[(size_t)vrow * d + i] * (int64_t)q[i];
    if (acc_out) acc_out[k] = (int32_t)a;
    logits[k] = r32((double)a * (double)s * (double)s_row[vrow]);
  }
}


// Token embedding from the int8 embedding matrix ([TS-2B]: "embedding/LM head matrices are quantized
// to int8 with per-channel/row scaling").  Reading: the embedding and the LM head are ONE tied matrix
// W [V][d] with one scale per row ([TS-3]: the embedding/LM-head share is 37% of 278 MB, i.e. a single
// 50288 x 2048 int8 matrix), so
//   e[i] = fl32(W[tok, i] * s_row[tok]).
// Returns 0, or -1 (e left untouched) when tok is outside [0, V).
// Pinned by: power-of-two row scales give the exact products; agreement with an IEEE fp32 multiply;
// the row index selects the row.
int oracle_embed(const int8_t* W, const float* s_row, int V, int d, int tok, float* e) {
  if (tok < 0 || tok >= V) return -1;
  for (int i = 0; i < d; ++i) e[i] = r32((double)W[(size_t)tok * d + i] * (double)s_row[tok]);
  return 0;
}

// Final RMSNorm + int8 LM head on one token (reading: the Mamba-2 language model [MAP] applies an
// RMSNorm with its own weight, eps 1e-5, to the last layer's residual stream before the LM head), the
// same norm-then-quantize as the pre-mixer norm (rmsnorm_quantize):
//   (q, s) = rmsnorm_quantize(h, norm_w);  logits[v] = fl32(acc[v] * s * s_row[v]),
//   acc[v] = sum_i W[v,i] * q[i].
// norm_w == NULL gives the plain LM head (oracle_lm_head).  Only rows listed in `rows` are computed
// when rows != NULL.
// Pinned by: brute-force int64 matmul of the pinned codes; equality with the plain LM head applied to the
// pinned normalized row; a constant row's closed form; a zero norm weight zeroes its codes.
void oracle_final_head(const int8_t* W, const float* s_row, int V, int d, const float* h,
                       const float* norm_w, const int* rows, int n_rows, float* logits,
                       int32_t* acc_out) {
  std::vector<int8_t> q((size_t)d);
  std::vector<float> v((size_t)d);
  float s = 0.0f;
  if (norm_w)
    rmsnorm_quantize(h, norm_w, d, 1e-5, q.data(), &s, v.data());
  else
    quantize_row(h, d, q.data(), &s);
  const int count = rows ? n_rows : V;
#pragma omp parallel for schedule(static)
  for (int k = 0; k < count; ++k) {
    const int vrow = rows ? rows[k] : k;
    int64_t a = 0;
    for (int i = 0; i < d; ++i) a += (int64_t)W[(size_t)vrow * d + i] * (int64_t)q[i];
    if (acc_out) acc_out[k] = (int32_t)a;
    logits[k] = r32((double)a * (double)s * (double)s_row[vrow]);
  }
}

// ---------------------------------------------------------------------------------- density field
//
// [TS-2D]: the SSM hidden state is kept as a K x K binary field per state element with K^2 about
// 4 d_state; normalization, sigma-delta injection (error feedback), binarization, and a popcount readout
// that recovers continuous values, at chunk boundaries.  Reading (F4): a "state element" is one state
// row S[h][p][0..N) (N = d_state values), its field is 4N cells (four per value, so K^2 = 4N), and:
//   normalization   c = max_n |S_n| (fp32); x_n = fl32(S_n / c), x_n = 0 when c = 0;
//                   d_n = fl32(x_n + 1) / 2, a density in [0, 1];
//   injection       the cells j = 4n + k (k = 0..3) in order, each fed its value's density d_n, through
//                   a first-order sigma-delta modulator: v = d + e, b_j = [v >= 1/2], e = v - b_j,
//                   with e = 0 before the first cell of the row;
//   binarization    b_j, stored least significant bit first: cell j is bit j % 32 of word j / 32 (value
//                   n is nibble n % 8 of word n / 8), N / 8 words per row, beside c;
//   readout         p_n = popcount of value n's four cells, S^_n = fl32(c (p_n / 2 - 1)).
// Every density is a multiple of 2^-25 (fl32(x + 1) is a multiple of 2^-24 for |x| <= 1) and |v| < 2,
// so the modulator below runs exactly in fp64.
// Pinned by: a hand-derived row (tests/golden/density_field.txt); the closed form of the first-order
// modulator (ones among the first j + 1 cells = floor(P_j + 1/2), P_j the exact sum of their
// densities); exact round trips of the five levels c {-1, -1/2, 0, 1/2, 1}; the running readout error
// bounded by c / 4; the zero row.
void oracle_field_encode(const float* state, int rows, int N, uint32_t* field, float* scale) {
  const int words = N / 8;
#pragma omp parallel for schedule(static)
  for (int r = 0; r < rows; ++r) {
    const float* S = state + (size_t)r * N;
    uint32_t* F = field + (size_t)r * words;
    float c = 0.0f;
    for (int n = 0; n < N; ++n) {
      const float a = std::fabs(S[n]);
      if (a > c) c = a;
    }
    for (int w = 0; w < words; ++w) F[w] = 0u;
    double e = 0.0;
    for (int n = 0; n < N; ++n) {
      const float x = c > 0.0f ? r32((double)S[n] / (double)c) : 0.0f;
      const float d = r32((double)r32((double)x + 1.0) * 0.5);
      for (int k = 0; k < 4; ++k) {
        const double v = (double)d + e;
        const int b = v >= 0.5 ? 1 : 0;
        e = v - (double)b;
        const int j = 4 * n + k;
        F[j / 32] |= (uint32_t)b << (j % 32);
      }
    }
    scale[r] = c;
  }
}

// The readout of oracle_field_encode's fields: S^_n = fl32(c (popcount(cells of n) / 2 - 1)).
// Pinned with oracle_field_encode (above).
void oracle_field_decode(const uint32_t* field, const float* scale, int rows, int N, float* state) {
  const int words = N / 8;
#pragma omp parallel for schedule(static)
  for (int r = 0; r < rows; ++r) {
    const uint32_t* F = field + (size_t)r * words;
    for (int n = 0; n < N; ++n) {
      int p = 0;
      for (int k = 0; k < 4; ++k) {
        const int j = 4 * n + k;
        p += (int)((F[j / 32] >> (j % 32)) & 1u);
      }
      state[(size_t)r * N + n] = r32((double)scale[r] * ((double)p * 0.5 - 1.0));
    }
  }
}

}  // extern "C"
