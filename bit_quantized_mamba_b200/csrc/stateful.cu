// Stateful Mamba-2 decode ops of DF-SSM (gist.science technical summary, §2.C "Stateful Ops: custom CUDA
// kernels handle the stateful shift register (convolution) and SSM recurrence (warp-level reduction)"),
// and the int8 LM-head GEMV (same summary, §2.B: int8 LM head with per-row scaling).
//
// All fp32 values that later feed a quantizer are single correctly rounded operations; the 5-term conv
// sum, the d_state-long SSM readout and every transcendental are evaluated in fp64 and rounded once.

#include "common.cuh"
#include "internal.h"

namespace dfssm {

template <typename Kern, typename... Args>
static cudaError_t launch_pdl(Kern k, dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                              Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, k, args...);
}

// ------------------------------------------------------------------------------------ conv step
// pre = fl32(b + w0*s0 + w1*s1 + w2*s2 + w3*x) in fp64 in this order (each product is exact in fp64);
// out = fl32(SiLU(pre)) in fp64; state <- (s1, s2, x).

__global__ void __launch_bounds__(256) conv_step_kernel(ConvArgs a) {
  const int idx = blockIdx.x * blockDim.x + threadIdx.x;
  const int total = a.B * a.C;
  const int c = idx % a.C;
  float4 w = make_float4(0.f, 0.f, 0.f, 0.f);
  float bias = 0.0f;
  if (idx < total) {
    w = ld_stream_f4(a.w + (size_t)c * 4);
    bias = a.bias[c];
  }
  pdl_launch_dependents();
  pdl_wait();
  if (idx >= total) return;
  const int b = idx / a.C;
  float* st = a.state + (size_t)idx * 3;
  const float s0 = st[0], s1 = st[1], s2 = st[2];
  const float xv = a.x_in[(size_t)b * a.ldx + c];
  a.x_out[(size_t)b * a.ldo + c] = conv_out(w, bias, s0, s1, s2, xv);
  st[0] = s1;
  st[1] = s2;
  st[2] = xv;
}

cudaError_t launch_conv(const ConvArgs& a, cudaStream_t st) {
  const int total = a.B * a.C;
  return launch_pdl(conv_step_kernel, dim3((total + 255) / 256), dim3(256), 0, st, a);
}

// ------------------------------------------------------------------------------------- SSM step
// One warp per (token b, head h, channel p) state row of N fp32 values; each lane owns N/128 float4s.
//   v = fl32(dt_raw + dt_bias); dt = fl32(softplus(v)); A = fl32(-exp(A_log)); dA = fl32(exp(fl32(dt*A)))
//   dtx = fl32(dt*x);  S <- fl32(fl32(dA*S) + fl32(dtx*B));  y = fl32(sum_n S*C + D*x)  (fp64 sum)
// Optional gate: y <- fl32(y * fl32(SiLU(z))).

__global__ void __launch_bounds__(256) ssm_step_kernel(SsmArgs a) {
  const int warp_g = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  const int HP = a.H * a.P;
  const int rows = a.B * HP;
  const bool valid = warp_g < rows;
  const int b = valid ? warp_g / HP : 0;
  const int hp = valid ? warp_g % HP : 0;
  const int h = hp / a.P;
  const int g = h / (a.H / a.G);
  float A_log = 0.f, dt_bias = 0.f, Dh = 0.f;
  if (valid) {
    A_log = a.A_log[h];
    dt_bias = a.dt_bias[h];
    Dh = a.D[h];
  }
  pdl_launch_dependents();
  pdl_wait();
  if (!valid) return;

  const float dt = ssm_dt(a.dt_raw[(size_t)b * a.lddt + h], dt_bias);
  const float dA = ssm_dA(dt, A_log);
  const float xv = a.x[(size_t)b * a.ldx + hp];
  const float dtx = fmul(dt, xv);

  float* S = a.state + (size_t)warp_g * a.N;
  const float* Bg = a.Bm + (size_t)b * a.ldbc + (size_t)g * a.N;
  const float* Cg = a.Cm + (size_t)b * a.ldbc + (size_t)g * a.N;
  double acc = 0.0;
  for (int n4 = lane; n4 < a.N / 4; n4 += 32) {
    float4 s4 = ld_evict_first_f4(S + 4 * n4);
    const float4 b4 = *reinterpret_cast<const float4*>(Bg + 4 * n4);
    const float4 c4 = *reinterpret_cast<const float4*>(Cg + 4 * n4);
    s4.x = ssm_state(dA, s4.x, dtx, b4.x);
    s4.y = ssm_state(dA, s4.y, dtx, b4.y);
    s4.z = ssm_state(dA, s4.z, dtx, b4.z);
    s4.w = ssm_state(dA, s4.w, dtx, b4.w);
    acc = fma((double)s4.x, (double)c4.x, acc);  // products of two fp32 are exact in fp64
    acc = fma((double)s4.y, (double)c4.y, acc);
    acc = fma((double)s4.z, (double)c4.z, acc);
    acc = fma((double)s4.w, (double)c4.w, acc);
    st_f4(S + 4 * n4, s4);
  }
  acc = warp_sum(acc);
  if (lane == 0) {
    float y = __double2float_rn(dadd(acc, dmul((double)Dh, (double)xv)));
    if (a.z) y = fmul(y, silu_f64(a.z[(size_t)b * a.ldz + hp]));
    a.y[(size_t)b * a.ldy + hp] = y;
  }
}

cudaError_t launch_ssm(const SsmArgs& a, cudaStream_t st) {
  const long long threads = (long long)a.B * a.H * a.P * 32;
  return launch_pdl(ssm_step_kernel, dim3((unsigned)((threads + 255) / 256)), dim3(256), 0, st, a);
}

// ------------------------------------------------------------------------------ int8 LM-head GEMV
// logits[v] = fl32(acc[v] * s * s_row[v]) (fp64, this order), acc[v] = sum_i W[v,i] q_i (int32 exact).
// Every CTA quantizes the token itself (per-token absmax int8, the decode quantizer: no separate launch
// and no hand-off); with a final RMSNorm weight the token is first normalized as for the layers'
// pre-norm: r = fl32(1/sqrt(sum x^2 / d + 1e-5)) (fp64) and v = fl32(fl32(x r) w) is quantized.  Each warp owns a
// contiguous, balanced range of rows and streams it as units of 2 KB (four 16-byte chunks per lane of
// one row), always with the next unit's loads in flight while the current one is summed; the first unit
// is requested before the quantizer runs, so its latency is hidden.  The stream rate is set by the
// number of resident threads (1024 per SM), not by the loads per thread.
//
// Greedy choice: every warp keeps the largest (logit, -row) key of its rows and merges it into one
// 64-bit word with atomicMax; the CTA that finishes last (counted with a second word, release/acquire
// through the fences around the count) turns the key into the row index and clears both words.

constexpr int LMH_U = 4;  // chunks per lane per unit (a unit is 32 x 4 x 16 B = 2 KB of one row)
constexpr int LMH_CTAS_PER_SM = 4;  // 1024 streaming threads per SM

// Order-preserving map of a finite fp32 value to u32 (larger value, larger key); -0 maps as +0, so
// equal logits tie and the smaller row wins.
__device__ __forceinline__ unsigned long long greedy_key(float v, int row) {
  unsigned u = __float_as_uint(v == 0.0f ? 0.0f : v);
  u = (u & 0x80000000u) ? ~u : (u | 0x80000000u);
  return ((unsigned long long)u << 32) | (unsigned long long)(0xFFFFFFFFu - (unsigned)row);
}

__global__ void __launch_bounds__(256, LMH_CTAS_PER_SM) int8_gemv_kernel(Int8GemvArgs a) {
  extern __shared__ __align__(16) unsigned char smem[];
  uint4* qsm = reinterpret_cast<uint4*>(smem);
  __shared__ float red[8];
  __shared__ double red_ss[8];
  const int lane = threadIdx.x & 31;
  const int warps_total = gridDim.x * (blockDim.x >> 5);
  const int warp_g = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int chunks = a.d >> 4;
  const int G = (chunks + 32 * LMH_U - 1) / (32 * LMH_U);  // units per row
  const int r0 = (int)((long long)warp_g * a.V / warps_total);
  const int r1 = (int)((long long)(warp_g + 1) * a.V / warps_total);
  const int n_units = (r1 - r0) * G;
  // unit j: row r0 + j / G, chunks g * 128 + lane + 32 u (g = j % G)
  const auto load_unit = [&](int j, uint4 (&x)[LMH_U]) {
    const int row = r0 + j / G, g = j - (j / G) * G;
    const uint4* w = reinterpret_cast<const uint4*>(a.W + (size_t)row * a.d);
#pragma unroll
    for (int u = 0; u < LMH_U; ++u) {
      const int c = g * 32 * LMH_U + lane + 32 * u;
      x[u] = (j < n_units && c < chunks) ? ld_stream_u4(w + c) : make_uint4(0u, 0u, 0u, 0u);
    }
  };
  uint4 cur[LMH_U];
  load_unit(0, cur);  // weights do not depend on the token: in flight during the quantizer
  pdl_launch_dependents();
  pdl_wait();
  const bool norm = a.norm_w != nullptr;
  // quantize the token (8 KB for d = 2048; with a norm weight a first pass sums the squares):
  // thread t takes inputs t + 256 k
  float rn = 1.0f;
  if (norm) {
    double ss = 0.0;
    for (int k0 = 0; k0 * 256 < a.d; k0 += 8) {
      float v[8];
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        const int i = threadIdx.x + 256 * (k0 + k);
        v[k] = i < a.d ? __ldg(a.x + i) : 0.0f;
      }
#pragma unroll
      for (int k = 0; k < 8; ++k) ss = fma((double)v[k], (double)v[k], ss);  // exact squares in fp64
    }
    ss = warp_sum(ss);
    if (lane == 0) red_ss[threadIdx.x >> 5] = ss;
    __syncthreads();
    ss = 0.0;
#pragma unroll
    for (int w = 0; w < 8; ++w) ss += red_ss[w];
    rn = rms_factor(ss, a.d);
  }
  const auto value = [&](int i) {
    if (i >= a.d) return 0.0f;
    const float xv = __ldg(a.x + i);
    return norm ? norm_value(xv, rn, __ldg(a.norm_w + i)) : xv;
  };
  float m = 0.0f;
  for (int k0 = 0; k0 * 256 < a.d; k0 += 8) {
    float v[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) v[k] = value(threadIdx.x + 256 * (k0 + k));
#pragma unroll
    for (int k = 0; k < 8; ++k) m = fmaxf(m, fabsf(v[k]));
  }
  m = warp_max(m);
  if (lane == 0) red[threadIdx.x >> 5] = m;
  __syncthreads();
  m = 0.0f;
#pragma unroll
  for (int w = 0; w < 8; ++w) m = fmaxf(m, red[w]);
  const float s0 = quant_scale(m);
  const float inv_s0 = quant_inv(s0);
  const float s = s0;
  int8_t* qb = reinterpret_cast<int8_t*>(smem);
  for (int k0 = 0; k0 * 256 < a.d; k0 += 8) {
    float vv[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) vv[k] = value(threadIdx.x + 256 * (k0 + k));
    int cd[8];
    quant_codes<8>(vv, s0, inv_s0, cd);
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const int i = threadIdx.x + 256 * (k0 + k);
      if (i < a.d) qb[i] = (int8_t)cd[k];
    }
  }
  __syncthreads();
  int acc = 0;
  unsigned long long best = 0ull;
  for (int j = 0; j < n_units; ++j) {
    uint4 nxt[LMH_U];
    load_unit(j + 1, nxt);
    const int g = j % G;
#pragma unroll
    for (int u = 0; u < LMH_U; ++u) {
      const int c = g * 32 * LMH_U + lane + 32 * u;
      const uint4 q = c < chunks ? qsm[c] : make_uint4(0u, 0u, 0u, 0u);
      acc = dp4a_ss(cur[u].x, q.x, acc);
      acc = dp4a_ss(cur[u].y, q.y, acc);
      acc = dp4a_ss(cur[u].z, q.z, acc);
      acc = dp4a_ss(cur[u].w, q.w, acc);
    }
    if (g == G - 1) {
      const int row = r0 + j / G;
      acc = warp_sum(acc);
      if (lane == 0) {
        const float lg = __double2float_rn(dmul(dmul((double)acc, (double)s), (double)a.s_row[row]));
        a.logits[row] = lg;
        if (a.acc) a.acc[row] = acc;
        const unsigned long long key = greedy_key(lg, row);
        best = key > best ? key : best;
      }
      acc = 0;
    }
#pragma unroll
    for (int u = 0; u < LMH_U; ++u) cur[u] = nxt[u];
  }
  if (a.greedy) {
    if (lane == 0 && n_units > 0) atomicMax(a.greedy, best);
    __syncthreads();
    if (threadIdx.x == 0) {
      __threadfence();
      const unsigned long long done = atomicAdd(a.greedy + 1, 1ull);
      if (done == (unsigned long long)gridDim.x - 1) {
        __threadfence();
        const unsigned long long key = atomicOr(a.greedy, 0ull);
        *a.token = (int32_t)(0xFFFFFFFFu - (unsigned)(key & 0xFFFFFFFFull));
        a.greedy[0] = 0ull;
        a.greedy[1] = 0ull;
      }
    }
  }
}

cudaError_t launch_int8_gemv(const Int8GemvArgs& a, cudaStream_t st) {
  const int blocks = num_sms() * LMH_CTAS_PER_SM;  // all resident: each CTA quantizes x once
  return launch_pdl(int8_gemv_kernel, dim3(blocks), dim3(256), (size_t)a.d, st, a);
}

// ------------------------------------------------------------------------------ embedding lookup
// One CTA; thread t converts 16 consecutive int8 values of the row (d % 16 == 0, rows 16-byte aligned).
__global__ void __launch_bounds__(512) embed_kernel(EmbedArgs a) {
  pdl_launch_dependents();
  pdl_wait();
  const int tok = *a.token;
  const bool ok = tok >= 0 && tok < a.V;
  if (!ok && threadIdx.x == 0) atomicExch(a.status, kBadTokenCode);
  const float sc = ok ? a.s_row[tok] : 0.0f;
  const uint4* row = reinterpret_cast<const uint4*>(a.W + (size_t)(ok ? tok : 0) * a.d);
  float4* h4 = reinterpret_cast<float4*>(a.h);
  for (int c = threadIdx.x; c < (a.d >> 4); c += blockDim.x) {
    const uint4 w = ok ? __ldg(row + c) : make_uint4(0u, 0u, 0u, 0u);
    const uint32_t wv[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      float4 o;
      o.x = fmul((float)(int8_t)(wv[k] & 0xFFu), sc);
      o.y = fmul((float)(int8_t)((wv[k] >> 8) & 0xFFu), sc);
      o.z = fmul((float)(int8_t)((wv[k] >> 16) & 0xFFu), sc);
      o.w = fmul((float)(int8_t)(wv[k] >> 24), sc);
      h4[4 * c + k] = o;
    }
  }
}

cudaError_t launch_embed(const EmbedArgs& a, cudaStream_t st) {
  const int threads = (a.d >> 4) < 512 ? (((a.d >> 4) + 31) & ~31) : 512;
  return launch_pdl(embed_kernel, dim3(1), dim3(threads), 0, st, a);
}

}  // namespace dfssm
