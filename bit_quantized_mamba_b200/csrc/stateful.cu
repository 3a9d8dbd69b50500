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
// One warp per row; each lane streams 16-byte chunks of the row and accumulates 4 dp4a per chunk.

__global__ void __launch_bounds__(256) int8_gemv_kernel(Int8GemvArgs a) {
  extern __shared__ __align__(16) unsigned char smem[];
  uint4* qsm = reinterpret_cast<uint4*>(smem);
  const int lane = threadIdx.x & 31;
  const int warps_total = gridDim.x * (blockDim.x >> 5);
  const int warp_g = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int chunks = a.d >> 4;
  pdl_launch_dependents();
  pdl_wait();
  const uint4* qsrc = reinterpret_cast<const uint4*>(a.in.q);
  for (int i = threadIdx.x; i < chunks; i += blockDim.x) qsm[i] = qsrc[i];
  __syncthreads();
  const float s = a.in.s[0];
  for (int row = warp_g; row < a.V; row += warps_total) {
    const uint4* wrow = reinterpret_cast<const uint4*>(a.W + (size_t)row * a.d);
    int acc = 0;
    for (int c = lane; c < chunks; c += 32) {
      const uint4 w = ld_stream_u4(wrow + c);
      const uint4 q = qsm[c];
      acc = dp4a_ss(w.x, q.x, acc);
      acc = dp4a_ss(w.y, q.y, acc);
      acc = dp4a_ss(w.z, q.z, acc);
      acc = dp4a_ss(w.w, q.w, acc);
    }
    acc = warp_sum(acc);
    if (lane == 0) {
      a.logits[row] =
          __double2float_rn(dmul(dmul((double)acc, (double)s), (double)a.s_row[row]));
      if (a.acc) a.acc[row] = acc;
    }
  }
}

cudaError_t launch_int8_gemv(const Int8GemvArgs& a, cudaStream_t st) {
  const int blocks = num_sms() * 8;
  return launch_pdl(int8_gemv_kernel, dim3(blocks), dim3(256), (size_t)a.d, st, a);
}

}  // namespace dfssm
