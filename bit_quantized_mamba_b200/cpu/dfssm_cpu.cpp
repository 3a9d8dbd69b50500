// Host-CPU engine of the DF-SSM decode step (include/dfssm_cpu.h): the pages' CPU path (gist.science
// technical summary of DF-SSM, §2.C "CPU path": the 1-bit packed weights are expanded to int8 for the
// VNNI dot product, loading 8x less weight data than int8 weights).
//
// Scaffold GEMV: 64 sign bits (two consecutive u32 words of a row; bit k is input 64c + k) become a
// 64-bit mask, `vmovdqu8` with zero-masking turns it into 64 bytes of 0 or 1, and `vpdpbusd` multiplies
// them (as u8) with 64 int8 codes of each token, accumulating four products per 32-bit lane.  The sum
// over the set bits gives the +-1 scaffold sum as acc = 2 sum_{bit=1} q - sum q (exact integers).  The
// expanded bytes serve every token of the call.
//
// Every other step follows the library's definition and rounding sequence: fp32 values are single
// IEEE operations or the fp32 rounding of an fp64 expression, sums of more than two terms are fp64 in
// index order, transcendental functions are fp64 and rounded once.  Built with -ffp-contract=off so
// that no product and sum are fused where the definition rounds them separately.

#include <immintrin.h>
#include <omp.h>

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstdlib>
#include <cstring>
#include <vector>

#include "dfssm_cpu.h"

namespace {

constexpr double kEps = 1e-5;

inline float f32(double v) { return (float)v; }
inline double silu(double v) { return v / (1.0 + std::exp(-v)); }

bool has_vnni() {
  __builtin_cpu_init();
  return __builtin_cpu_supports("avx512f") && __builtin_cpu_supports("avx512bw") &&
         __builtin_cpu_supports("avx512vl") && __builtin_cpu_supports("avx512vnni");
}

// 64-byte aligned scratch that lives for one call.
struct Buf {
  void* p = nullptr;
  explicit Buf(size_t bytes) { p = std::aligned_alloc(64, (bytes + 63) / 64 * 64 + 64); }
  ~Buf() { std::free(p); }
  template <class T>
  T* as() const { return static_cast<T*>(p); }
};

// ---------------------------------------------------------------------------------------- quantizer

// Per-token absmax int8 quantizer: s = fl32(m / 127), q = clamp(rint(fl32(v / s)), +-127) with round
// half to even; an all-zero row gives s = 0, q = 0.  Returns s; writes the code sum.  Sixteen values at a
// time: the IEEE division and the rounding to nearest even are single AVX-512 operations.
__attribute__((target("avx512f,avx512bw,avx512vl"))) float quantize(const float* v, int n, int8_t* q, int* sumq) {
  __m512 vm = _mm512_setzero_ps();
  for (int i = 0; i < n; i += 16) {
    const __mmask16 k = n - i >= 16 ? (__mmask16)0xFFFF : (__mmask16)((1u << (n - i)) - 1u);
    vm = _mm512_max_ps(vm, _mm512_abs_ps(_mm512_maskz_loadu_ps(k, v + i)));
  }
  const float m = _mm512_reduce_max_ps(vm);
  if (m == 0.0f) {
    std::memset(q, 0, (size_t)n);
    *sumq = 0;
    return 0.0f;
  }
  const float s = m / 127.0f;
  const __m512 vs = _mm512_set1_ps(s), hi = _mm512_set1_ps(127.0f), lo = _mm512_set1_ps(-127.0f);
  __m512i vsum = _mm512_setzero_si512();
  for (int i = 0; i < n; i += 16) {
    const __mmask16 k = n - i >= 16 ? (__mmask16)0xFFFF : (__mmask16)((1u << (n - i)) - 1u);
    __m512 t = _mm512_div_ps(_mm512_maskz_loadu_ps(k, v + i), vs);
    t = _mm512_roundscale_ps(t, _MM_FROUND_TO_NEAREST_INT | _MM_FROUND_NO_EXC);
    t = _mm512_min_ps(hi, _mm512_max_ps(lo, t));
    const __m512i c = _mm512_maskz_cvtps_epi32(k, t);
    _mm_mask_storeu_epi8(q + i, k, _mm512_cvtepi32_epi8(c));
    vsum = _mm512_add_epi32(vsum, c);
  }
  *sumq = _mm512_reduce_add_epi32(vsum);
  return s;
}

// RMSNorm (eps 1e-5, weight w), then the quantizer on the normalised row:
//   r = fl32(1 / sqrt(sum h^2 / n + eps)) (the fp64 sum in index order, the squares exact),
//   u = fl32(fl32(h r) w).
__attribute__((target("avx512f,avx512bw,avx512vl"))) float norm_quantize(const float* h, const float* w, int n,
                                                                 float* u, int8_t* q, int* sumq) {
  double ss = 0.0;
  for (int i = 0; i < n; ++i) ss += (double)h[i] * (double)h[i];
  const float r = f32(1.0 / std::sqrt(ss / (double)n + kEps));
  const __m512 vr = _mm512_set1_ps(r);
  for (int i = 0; i < n; i += 16) {
    const __mmask16 k = n - i >= 16 ? (__mmask16)0xFFFF : (__mmask16)((1u << (n - i)) - 1u);
    const __m512 hr = _mm512_mul_ps(_mm512_maskz_loadu_ps(k, h + i), vr);
    _mm512_mask_storeu_ps(u + i, k, _mm512_mul_ps(hr, _mm512_maskz_loadu_ps(k, w + i)));
  }
  return quantize(u, n, q, sumq);
}

// ---------------------------------------------------------------------------------------- linear

// acc[b][o] for rows [o0, o1): BT token slots (codes zero-padded to BT tokens and to whole 64-byte
// chunks), the expanded sign bytes shared by all of them.  With fewer than four tokens each token keeps
// U = 4 / BT partial sums over alternating chunks, so that U vpdpbusd chains run side by side (integer
// sums: the order does not change the result).
template <int BT>
__attribute__((target("avx512f,avx512bw,avx512vnni"))) void scaffold_rows(
    const uint32_t* bits, int d_in, int o0, int o1, const int8_t* qpad, int dpad, const int* sumq, int B,
    int32_t* acc, int d_out) {
  constexpr int U = BT >= 4 ? 1 : 4 / BT;
  const __m512i ones = _mm512_set1_epi8(1);
  const int words = d_in / 32, full = d_in / 64;
  for (int o = o0; o < o1; ++o) {
    const uint32_t* w = bits + (size_t)o * words;
    __m512i a[U][BT];
#pragma GCC unroll 16
    for (int u = 0; u < U; ++u)
#pragma GCC unroll 16
      for (int b = 0; b < BT; ++b) a[u][b] = _mm512_setzero_si512();
    int c = 0;
    for (; c + U <= full; c += U) {
#pragma GCC unroll 4
      for (int u = 0; u < U; ++u) {
        const uint64_t m = (uint64_t)w[2 * (c + u)] | ((uint64_t)w[2 * (c + u) + 1] << 32);
        const __m512i v = _mm512_maskz_mov_epi8((__mmask64)m, ones);
#pragma GCC unroll 16
        for (int b = 0; b < BT; ++b)
          a[u][b] = _mm512_dpbusd_epi32(a[u][b], v, _mm512_load_si512(qpad + (size_t)b * dpad + 64 * (c + u)));
      }
    }
    for (; c < full; ++c) {
      const uint64_t m = (uint64_t)w[2 * c] | ((uint64_t)w[2 * c + 1] << 32);
      const __m512i v = _mm512_maskz_mov_epi8((__mmask64)m, ones);
#pragma GCC unroll 16
      for (int b = 0; b < BT; ++b)
        a[0][b] = _mm512_dpbusd_epi32(a[0][b], v, _mm512_load_si512(qpad + (size_t)b * dpad + 64 * c));
    }
    if (words & 1) {  // d_in % 64 == 32: the last word alone (the codes beyond d_in are zero)
      const uint64_t m = (uint64_t)w[words - 1];
      const __m512i v = _mm512_maskz_mov_epi8((__mmask64)m, ones);
#pragma GCC unroll 16
      for (int b = 0; b < BT; ++b)
        a[0][b] = _mm512_dpbusd_epi32(a[0][b], v, _mm512_load_si512(qpad + (size_t)b * dpad + 64 * full));
    }
    for (int b = 0; b < B; ++b) {
      __m512i t = a[0][b];
#pragma GCC unroll 4
      for (int u = 1; u < U; ++u) t = _mm512_add_epi32(t, a[u][b]);
      acc[(size_t)b * d_out + o] = 2 * _mm512_reduce_add_epi32(t) - sumq[b];
    }
  }
}

// t[r] = sum_i W_B[r,i] q[i] for one token (exact int32): vpdpbusd multiplies unsigned by signed bytes,
// so the codes enter as q + 128 (1..255) and 128 sum_i W_B[r,i] is taken off afterwards.
__attribute__((target("avx512f,avx512bw,avx512vnni"))) void lora_down_vnni(const int8_t* wb, int rank,
                                                                            int d_in, const int8_t* qpad,
                                                                            int32_t* t) {
  const __m512i bias = _mm512_set1_epi8((char)0x80), ones = _mm512_set1_epi8(1);
  const int chunks = (d_in + 63) / 64;
  for (int r = 0; r < rank; ++r) {
    const int8_t* w = wb + (size_t)r * d_in;
    __m512i acc = _mm512_setzero_si512(), wsum = _mm512_setzero_si512();
    for (int c = 0; c < chunks; ++c) {
      const int n = std::min(64, d_in - 64 * c);
      const __mmask64 k = n == 64 ? ~0ull : ((1ull << n) - 1ull);
      const __m512i wv = _mm512_maskz_loadu_epi8(k, w + 64 * c);
      const __m512i qv = _mm512_xor_si512(_mm512_load_si512(qpad + 64 * c), bias);  // q + 128 as u8
      acc = _mm512_dpbusd_epi32(acc, qv, wv);
      wsum = _mm512_dpbusd_epi32(wsum, ones, wv);
    }
    t[r] = _mm512_reduce_add_epi32(acc) - 128 * _mm512_reduce_add_epi32(wsum);
  }
}

using RowsFn = void (*)(const uint32_t*, int, int, int, const int8_t*, int, const int*, int, int32_t*, int);
RowsFn rows_fn(int B) {
  if (B <= 1) return scaffold_rows<1>;
  if (B <= 2) return scaffold_rows<2>;
  if (B <= 4) return scaffold_rows<4>;
  if (B <= 8) return scaffold_rows<8>;
  return scaffold_rows<16>;
}
int slots(int B) { return B <= 1 ? 1 : B <= 2 ? 2 : B <= 4 ? 4 : B <= 8 ? 8 : 16; }

// One linear on B already-quantized tokens: codes q [B][d_in] (natural order), scales s, code sums.
//   t[r] = sum_i W_B[r,i] q[i] (int32), tf[r] = fl32(t sB s) (fp64, this order)
//   y[o] = fl32(acc s sW + sA sum_r W_A[o,r] tf[r])  (fp64, left to right; the LoRA sum in r order)
// out_add: y = fl32(out_add + y) when not null (the residual add), else y is written as is.
void linear(const dfssm_linear_t& L, const int8_t* q, const float* s, const int* sumq, int B, float* y,
            const float* out_add, int32_t* dbg_acc, int32_t* dbg_t) {
  const int d_in = L.d_in, d_out = L.d_out, rank = L.rank;
  const int BT = slots(B);
  const int dpad = (d_in + 63) / 64 * 64;
  Buf qb((size_t)BT * dpad);
  int8_t* qpad = qb.as<int8_t>();
  std::memset(qpad, 0, (size_t)BT * dpad);
  for (int b = 0; b < B; ++b) std::memcpy(qpad + (size_t)b * dpad, q + (size_t)b * d_in, (size_t)d_in);
  int sq[16] = {0};
  for (int b = 0; b < B; ++b) sq[b] = sumq[b];
  // LoRA down-projection (the padded codes past d_in are zero and the masked W_B loads read nothing there)
  std::vector<float> tf((size_t)B * DFSSM_MAX_RANK, 0.0f);
  for (int b = 0; b < B; ++b) {
    int32_t t[DFSSM_MAX_RANK];
    lora_down_vnni(L.lora_b, rank, d_in, qpad + (size_t)b * dpad, t);
    for (int r = 0; r < rank; ++r) {
      if (dbg_t) dbg_t[(size_t)b * rank + r] = t[r];
      tf[(size_t)b * DFSSM_MAX_RANK + r] = f32((double)t[r] * (double)L.lora_b_scale[r] * (double)s[b]);
    }
  }
  // scaffold accumulators, then the epilogue of the same rows, in chunks of 64 rows handed out as threads
  // come free (the cores of a shared host run at uneven speeds)
  Buf ab((size_t)B * d_out * 4);
  int32_t* acc = ab.as<int32_t>();
  const RowsFn fn = rows_fn(B);
  constexpr int kChunk = 64;
  const int chunks = (d_out + kChunk - 1) / kChunk;
#pragma omp parallel for schedule(dynamic, 1)
  for (int ci = 0; ci < chunks; ++ci) {
    const int o0 = ci * kChunk, o1 = std::min(d_out, o0 + kChunk);
    fn(L.bits, d_in, o0, o1, qpad, dpad, sq, B, acc, d_out);
    // epilogue, eight outputs at a time so that their LoRA sums (each in r order) run side by side
    for (int b = 0; b < B; ++b) {
      const float* tb = tf.data() + (size_t)b * DFSSM_MAX_RANK;
      for (int ob = o0; ob < o1; ob += 8) {
        const int no = std::min(8, o1 - ob);
        double lora[8] = {};
        for (int r = 0; r < rank; ++r) {
          const double t = (double)tb[r];
          for (int k = 0; k < no; ++k) lora[k] += (double)L.lora_a[(size_t)(ob + k) * rank + r] * t;
        }
        for (int k = 0; k < no; ++k) {
          const int o = ob + k;
          const size_t i = (size_t)b * d_out + o;
          const int a = acc[i];
          const double scaffold = (double)a * (double)s[b] * (double)L.w_scale[o];
          const double corr = rank > 0 ? (double)L.lora_a_scale[o] * lora[k] : 0.0;
          const float v = f32(scaffold + corr);
          y[i] = out_add ? out_add[i] + v : v;
          if (dbg_acc) dbg_acc[i] = a;
        }
      }
    }
  }
}

int check_linear(const dfssm_linear_t* L) {
  if (!L || L->d_out < 1 || L->d_in < 32 || L->d_in % 32 || L->rank < 0 || L->rank > DFSSM_MAX_RANK)
    return DFSSM_EINVAL;
  if (L->d_in > 8192) return DFSSM_EUNSUPPORTED;
  if (!L->bits || !L->w_scale) return DFSSM_EINVAL;
  if (L->rank > 0 && (!L->lora_b || !L->lora_b_scale || !L->lora_a || !L->lora_a_scale)) return DFSSM_EINVAL;
  return DFSSM_OK;
}

// ---------------------------------------------------------------------------------------- stateful

// Width-4 conv step with SiLU on C channels: fl32(b + w0 s0 + w1 s1 + w2 s2 + w3 x) (fp64, this order),
// then fl32(SiLU), the state shifted by one.
void conv_step(float* st_all, const float* w, const float* bias, const float* x, float* out, int C) {
#pragma omp parallel for schedule(static)
  for (int c = 0; c < C; ++c) {
    float* st = st_all + (size_t)c * 3;
    const float* wc = w + (size_t)c * 4;
    double e = (double)bias[c];
    e += (double)wc[0] * (double)st[0];
    e += (double)wc[1] * (double)st[1];
    e += (double)wc[2] * (double)st[2];
    e += (double)wc[3] * (double)x[c];
    out[c] = f32(silu((double)f32(e)));
    st[0] = st[1];
    st[1] = st[2];
    st[2] = x[c];
  }
}

// 8 R rows of one head (R groups of eight), n in [0, N8) with N8 a multiple of 8: the update as three
// fp32 vector operations per element (no fusion), the readout products fl64(S) fl64(C) (exact) turned
// from row-major 8 x 8 blocks into columns by an 8 x 8 transpose, so that lane k of group j accumulates
// row 8j + k's sum in index order.  The R groups' add chains run side by side.
template <int R>
__attribute__((target("avx512f"))) void ssm_rows8(float* S, int N, int N8, float dA, const float* dtx,
                                                   const float* Bg, const float* Cg, double* acc_out) {
  const __m256 vdA = _mm256_set1_ps(dA);
  __m512d acc[R];
#pragma GCC unroll 2
  for (int j = 0; j < R; ++j) acc[j] = _mm512_setzero_pd();
  const __m512i lo2 = _mm512_setr_epi64(0, 1, 8, 9, 4, 5, 12, 13), hi2 = _mm512_setr_epi64(2, 3, 10, 11, 6, 7, 14, 15);
  const __m512i lo4 = _mm512_setr_epi64(0, 1, 2, 3, 8, 9, 10, 11), hi4 = _mm512_setr_epi64(4, 5, 6, 7, 12, 13, 14, 15);
  for (int n = 0; n < N8; n += 8) {
    const __m256 vb = _mm256_loadu_ps(Bg + n);
    const __m512d vc = _mm512_cvtps_pd(_mm256_loadu_ps(Cg + n));
#pragma GCC unroll 2
    for (int j = 0; j < R; ++j) {
      __m512d r[8];
#pragma GCC unroll 8
      for (int k = 0; k < 8; ++k) {
        float* Sk = S + (size_t)(8 * j + k) * N + n;
        const __m256 upd = _mm256_add_ps(_mm256_mul_ps(vdA, _mm256_loadu_ps(Sk)),
                                         _mm256_mul_ps(_mm256_set1_ps(dtx[8 * j + k]), vb));
        _mm256_storeu_ps(Sk, upd);
        r[k] = _mm512_mul_pd(_mm512_cvtps_pd(upd), vc);
      }
      __m512d a[8], b[8];
#pragma GCC unroll 4
      for (int k = 0; k < 8; k += 2) {
        a[k] = _mm512_unpacklo_pd(r[k], r[k + 1]);      // columns 0, 2, 4, 6 of rows k, k+1
        a[k + 1] = _mm512_unpackhi_pd(r[k], r[k + 1]);  // columns 1, 3, 5, 7
      }
#pragma GCC unroll 2
      for (int k = 0; k < 8; k += 4) {
        b[k] = _mm512_permutex2var_pd(a[k], lo2, a[k + 2]);          // columns 0, 4 of rows k..k+3
        b[k + 2] = _mm512_permutex2var_pd(a[k], hi2, a[k + 2]);      // columns 2, 6
        b[k + 1] = _mm512_permutex2var_pd(a[k + 1], lo2, a[k + 3]);  // columns 1, 5
        b[k + 3] = _mm512_permutex2var_pd(a[k + 1], hi2, a[k + 3]);  // columns 3, 7
      }
      __m512d t = acc[j];
      t = _mm512_add_pd(t, _mm512_permutex2var_pd(b[0], lo4, b[4]));  // column 0
      t = _mm512_add_pd(t, _mm512_permutex2var_pd(b[1], lo4, b[5]));  // column 1
      t = _mm512_add_pd(t, _mm512_permutex2var_pd(b[2], lo4, b[6]));  // column 2
      t = _mm512_add_pd(t, _mm512_permutex2var_pd(b[3], lo4, b[7]));  // column 3
      t = _mm512_add_pd(t, _mm512_permutex2var_pd(b[0], hi4, b[4]));  // column 4
      t = _mm512_add_pd(t, _mm512_permutex2var_pd(b[1], hi4, b[5]));  // column 5
      t = _mm512_add_pd(t, _mm512_permutex2var_pd(b[2], hi4, b[6]));  // column 6
      t = _mm512_add_pd(t, _mm512_permutex2var_pd(b[3], hi4, b[7]));  // column 7
      acc[j] = t;
    }
  }
#pragma GCC unroll 2
  for (int j = 0; j < R; ++j) _mm512_storeu_pd(acc_out + 8 * j, acc[j]);
}

// SSM state update and readout of one token, then the gate:
//   dt = fl32(softplus(fl32(dt_raw + dt_bias))), A = fl32(-exp(A_log)), dA = fl32(exp(fl32(dt A)))
//   S <- fl32(fl32(dA S) + fl32(fl32(dt x) B));  y = fl32(sum_n S C + D x) (fp64, n in order)
//   gate = fl32(y fl32(SiLU(z)))  (y itself is not stored)
// Rows go sixteen (or eight) at a time through ssm_rows8 for the whole multiple of 8 in n; the rest of n,
// and the rows left over when P % 8 != 0, continue each row's sum one term at a time.
void ssm_step(float* S_all, const float* x, const float* dt_raw, const float* A_log, const float* dt_bias,
              const float* Dv, const float* Bm, const float* Cm, const float* z, float* gate, int H, int P,
              int N, int G) {
  const int hpg = H / G, N8 = N / 8 * 8;
#pragma omp parallel for schedule(static)
  for (int h = 0; h < H; ++h) {
    const int g = h / hpg;
    const float v = dt_raw[h] + dt_bias[h];
    const float dt = f32(v > 20.0f ? (double)v : std::log1p(std::exp((double)v)));
    const float A = f32(-std::exp((double)A_log[h]));
    const float dA = f32(std::exp((double)(dt * A)));
    const float* Bg = Bm + (size_t)g * N;
    const float* Cg = Cm + (size_t)g * N;
    for (int p0 = 0; p0 < P; p0 += 16) {
      const int np = std::min(16, P - p0);
      double acc[16] = {};
      float dtx[16];
      for (int k = 0; k < np; ++k) dtx[k] = dt * x[(size_t)h * P + p0 + k];
      float* S0 = S_all + ((size_t)h * P + p0) * N;
      int n0 = 0, nv = 0;  // the first nv rows went through ssm_rows8 for n < n0
      if (N8 > 0 && np == 16) {
        ssm_rows8<2>(S0, N, N8, dA, dtx, Bg, Cg, acc);
        n0 = N8, nv = 16;
      } else if (N8 > 0 && np >= 8) {
        ssm_rows8<1>(S0, N, N8, dA, dtx, Bg, Cg, acc);
        n0 = N8, nv = 8;
      }
      for (int k = 0; k < np; ++k) {
        float* S = S0 + (size_t)k * N;
        double a = acc[k];
        for (int n = k < nv ? n0 : 0; n < N; ++n) {
          S[n] = (dA * S[n]) + (dtx[k] * Bg[n]);
          a += (double)S[n] * (double)Cg[n];
        }
        const size_t idx = (size_t)h * P + p0 + k;
        const float yv = f32(a + (double)Dv[h] * (double)x[idx]);
        gate[idx] = yv * f32(silu((double)z[idx]));
      }
    }
  }
}

// ------------------------------------------------------------------------------------ density field

// One state row of the density-field representation (libdfssm's dfssm_state_field_encode): c = max |S|,
// densities as integers D_n = fl32(fl32(S_n / c) + 1) 2^24 (exact: multiples of 2^-25 times 2^25), and
// the four cells of value n the carries of lo + k D_n past 2^25, k = 1..4, lo = (4 Q_n + 2^24) mod 2^25
// with Q_n the prefix sum of D (only Q mod 2^23 enters, so wrapping 32-bit arithmetic is exact).  The
// divisions and conversions of a row are vectorised; the prefix sum runs in index order.  field and
// readout may each be NULL.
__attribute__((target("avx512f"))) void field_row(const float* S, int N, uint32_t* field, float* scale,
                                                  float* readout) {
  alignas(64) uint32_t D[256];
  float c = 0.0f;
  for (int n = 0; n < N; ++n) c = std::max(c, std::fabs(S[n]));
  const __m512 vc = _mm512_set1_ps(c), one = _mm512_set1_ps(1.0f), k24 = _mm512_set1_ps(16777216.0f);
  for (int n = 0; n < N; n += 16) {
    const __mmask16 m = N - n >= 16 ? (__mmask16)0xFFFF : (__mmask16)((1u << (N - n)) - 1u);
    const __m512 x = c > 0.0f ? _mm512_div_ps(_mm512_maskz_loadu_ps(m, S + n), vc) : _mm512_setzero_ps();
    // fl32(x + 1) 2^24: the sum rounds once, the product by 2^24 is exact, the conversion is exact
    const __m512i d = _mm512_cvtps_epu32(_mm512_mul_ps(_mm512_add_ps(x, one), k24));
    _mm512_mask_storeu_epi32(D + n, m, d);
  }
  uint32_t q = 0;
  for (int w = 0; w < N / 8; ++w) {
    uint32_t word = 0;
    for (int i = 0; i < 8; ++i) {
      const int n = 8 * w + i;
      const uint32_t a1 = ((4u * q + (1u << 24)) & ((1u << 25) - 1u)) + D[n];
      const uint32_t a2 = a1 + D[n], a3 = a2 + D[n], a4 = a3 + D[n];
      const uint32_t t1 = a1 >> 25, t2 = a2 >> 25, t3 = a3 >> 25, t4 = a4 >> 25;
      word |= (8u * t4 - 4u * t3 - 2u * t2 - t1) << (4 * i);
      if (readout) readout[n] = c * ((float)t4 * 0.5f - 1.0f);
      q += D[n];
    }
    if (field) field[w] = word;
  }
  if (scale) *scale = c;
}

bool field_args_ok(int rows, int N) { return rows >= 0 && N >= 8 && N % 8 == 0; }

}  // namespace

extern "C" {

int dfssm_cpu_abi_version(void) { return DFSSM_CPU_ABI_VERSION; }

int dfssm_cpu_available(void) { return has_vnni() ? 1 : 0; }

int dfssm_cpu_set_threads(int n) {
  if (n > 0) omp_set_num_threads(n);
  else omp_set_num_threads(omp_get_num_procs());
  return omp_get_max_threads();
}

int dfssm_cpu_linear_decode(const dfssm_linear_t* lin, const float* x, int B, float* y,
                            const dfssm_debug_t* dbg) {
  const int st = check_linear(lin);
  if (st) return st;
  if (!x || !y || B < 1 || B > DFSSM_MAX_BATCH) return DFSSM_EINVAL;
  if (!has_vnni()) return DFSSM_EUNSUPPORTED;
  const int d_in = lin->d_in;
  std::vector<int8_t> q((size_t)B * d_in);
  std::vector<float> s(B);
  std::vector<int> sq(B);
  for (int b = 0; b < B; ++b) {
    s[b] = quantize(x + (size_t)b * d_in, d_in, q.data() + (size_t)b * d_in, &sq[b]);
    if (dbg && dbg->xscale) dbg->xscale[b] = s[b];
  }
  if (dbg && dbg->xq) std::memcpy(dbg->xq, q.data(), q.size());
  linear(*lin, q.data(), s.data(), sq.data(), B, y, nullptr, dbg ? dbg->acc : nullptr,
         dbg ? dbg->lora_t : nullptr);
  return DFSSM_OK;
}

int dfssm_cpu_state_field_encode(const float* state, int rows, int N, uint32_t* field, float* scale) {
  if (!field_args_ok(rows, N)) return DFSSM_EINVAL;
  if (N > 256) return DFSSM_EUNSUPPORTED;
  if (rows == 0) return DFSSM_OK;
  if (!state || !field || !scale) return DFSSM_EINVAL;
  if (!has_vnni()) return DFSSM_EUNSUPPORTED;
#pragma omp parallel for schedule(static)
  for (int r = 0; r < rows; ++r)
    field_row(state + (size_t)r * N, N, field + (size_t)r * (N / 8), scale + r, nullptr);
  return DFSSM_OK;
}

int dfssm_cpu_state_field_decode(const uint32_t* field, const float* scale, int rows, int N, float* state) {
  if (!field_args_ok(rows, N)) return DFSSM_EINVAL;
  if (N > 256) return DFSSM_EUNSUPPORTED;
  if (rows == 0) return DFSSM_OK;
  if (!state || !field || !scale) return DFSSM_EINVAL;
#pragma omp parallel for schedule(static)
  for (int r = 0; r < rows; ++r) {
    const uint32_t* F = field + (size_t)r * (N / 8);
    const float c = scale[r];
    for (int n = 0; n < N; ++n) {
      const int p = __builtin_popcount((F[n / 8] >> (4 * (n % 8))) & 0xFu);
      state[(size_t)r * N + n] = c * ((float)p * 0.5f - 1.0f);
    }
  }
  return DFSSM_OK;
}

int dfssm_cpu_state_field_roundtrip(float* state, int rows, int N, uint32_t* field, float* scale) {
  if (!field_args_ok(rows, N)) return DFSSM_EINVAL;
  if (N > 256) return DFSSM_EUNSUPPORTED;
  if (rows == 0) return DFSSM_OK;
  if (!state || (field == nullptr) != (scale == nullptr)) return DFSSM_EINVAL;
  if (!has_vnni()) return DFSSM_EUNSUPPORTED;
#pragma omp parallel for schedule(static)
  for (int r = 0; r < rows; ++r) {
    float* S = state + (size_t)r * N;
    alignas(64) float tmp[256];
    field_row(S, N, field ? field + (size_t)r * (N / 8) : nullptr, scale ? scale + r : nullptr, tmp);
    std::memcpy(S, tmp, (size_t)N * 4);
  }
  return DFSSM_OK;
}

int dfssm_cpu_layer_decode(const dfssm_layer_t* layers, int n_layers, const dfssm_dims_t* dims,
                           float* hidden, float* const* conv_states, float* const* ssm_states, int B) {
  if (!layers || !dims || !hidden || !conv_states || !ssm_states || n_layers < 1 || B < 1 ||
      B > DFSSM_MAX_BATCH)
    return DFSSM_EINVAL;
  if (n_layers > DFSSM_MAX_LAYERS) return DFSSM_EUNSUPPORTED;
  const int Dm = dims->d_model, H = dims->nheads, P = dims->headdim, N = dims->d_state, G = dims->ngroups;
  if (Dm < 32 || Dm % 32 || H < 1 || P < 1 || N < 1 || G < 1 || H % G) return DFSSM_EINVAL;
  const int E = H * P, C = E + 2 * G * N, d_ip = 2 * E + 2 * G * N + H;
  if (E % 32) return DFSSM_EINVAL;
  for (int l = 0; l < n_layers; ++l) {
    const dfssm_layer_t& Ly = layers[l];
    int st = check_linear(&Ly.in_proj);
    if (st) return st;
    st = check_linear(&Ly.out_proj);
    if (st) return st;
    if (Ly.in_proj.d_out != d_ip || Ly.in_proj.d_in != Dm || Ly.out_proj.d_out != Dm || Ly.out_proj.d_in != E)
      return DFSSM_EINVAL;
    if (!Ly.conv_w || !Ly.conv_b || !Ly.A_log || !Ly.dt_bias || !Ly.D || !Ly.norm_w || !Ly.gnorm_w ||
        !conv_states[l] || !ssm_states[l])
      return DFSSM_EINVAL;
  }
  if (!has_vnni()) return DFSSM_EUNSUPPORTED;
  const int nmax = std::max(Dm, E);
  std::vector<float> u((size_t)nmax), zx((size_t)B * d_ip), xc((size_t)C), g((size_t)B * E);
  std::vector<int8_t> q((size_t)B * nmax);
  std::vector<float> s(B);
  std::vector<int> sq(B);
  for (int l = 0; l < n_layers; ++l) {
    const dfssm_layer_t& Ly = layers[l];
    // pre-norm + quantize, in_proj
    for (int b = 0; b < B; ++b)
      s[b] = norm_quantize(hidden + (size_t)b * Dm, Ly.norm_w, Dm, u.data(), q.data() + (size_t)b * Dm, &sq[b]);
    linear(Ly.in_proj, q.data(), s.data(), sq.data(), B, zx.data(), nullptr, nullptr, nullptr);
    for (int b = 0; b < B; ++b) {
      const float* zb = zx.data() + (size_t)b * d_ip;
      // conv on x|B|C, SSM step, gate y SiLU(z)
      conv_step(conv_states[l] + (size_t)b * C * 3, Ly.conv_w, Ly.conv_b, zb + E, xc.data(), C);
      ssm_step(ssm_states[l] + (size_t)b * H * P * N, xc.data(), zb + E + C, Ly.A_log, Ly.dt_bias, Ly.D,
               xc.data() + E, xc.data() + E + G * N, zb, g.data() + (size_t)b * E, H, P, N, G);
    }
    // gated norm + quantize, out_proj with the residual add
    for (int b = 0; b < B; ++b)
      s[b] = norm_quantize(g.data() + (size_t)b * E, Ly.gnorm_w, E, u.data(), q.data() + (size_t)b * E, &sq[b]);
    linear(Ly.out_proj, q.data(), s.data(), sq.data(), B, hidden, hidden, nullptr, nullptr);
  }
  return DFSSM_OK;
}

}  // extern "C"
