// Sequence (prefill) forms of the stateful Mamba-2 ops of a DF-SSM layer (gist.science technical summary,
// §2.C "Stateful Ops": the width-4 shift-register convolution and the SSM recurrence), over the M tokens
// of one prompt at batch 1.  Both reproduce, token after token, exactly the arithmetic of the decode
// step (csrc/stateful.cu and the fused decode kernel), so a prefill of M tokens leaves the conv and SSM
// states where M decode steps would leave them:
//   conv:  out[t][c] = SiLU(fl32(b + w0 x[t-3] + w1 x[t-2] + w2 x[t-1] + w3 x[t]))  (fp64, this order),
//          x[t < 0] taken from the incoming state; the state becomes (x[M-3], x[M-2], x[M-1]).
//   SSM:   S[h,p,n] <- fl32(fl32(dA S) + fl32(dt x B[n])) for t = 0 .. M-1 in order, and
//          y[t][h,p] = fl32(sum_n S C[n] + D x) (fp64 sum), gated: g = fl32(y * fl32(SiLU(z))).
// The scan is the stepped recurrence, not the chunked (SSD dual) reordering of it: every state element
// follows the same rounding sequence as in decode.  Parallelism comes from the 262,144 independent
// (h, p, n) recurrences of the 1.3B shape: one warp per (h, p) row (four state elements per lane), sixteen
// rows of one head per CTA, the tokens' B, C, dt, x and z staged through shared memory sixteen tokens at
// a time, the next chunk's loads in flight while the current one is stepped.

#include "common.cuh"
#include "internal.h"

namespace dfssm {
namespace scan {

constexpr int SW = 16;  // rows (warps) per CTA
constexpr int ST = 16;  // tokens per staged chunk

// ------------------------------------------------------------------------------ causal conv
__global__ void __launch_bounds__(256) conv_seq_kernel(ConvSeqArgs a) {
  const long long idx = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= (long long)a.M * a.C) return;
  const int t = (int)(idx / a.C), c = (int)(idx - (long long)t * a.C);
  float xin[4];
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const int tk = t - 3 + k;
    xin[k] = tk >= 0 ? __ldg(a.zx + (size_t)tk * a.ld_zx + a.x_off + c) : __ldg(a.state + (size_t)c * 3 + (tk + 3));
  }
  const float4 w = __ldg(reinterpret_cast<const float4*>(a.w) + c);
  a.xc[(size_t)t * a.C + c] = conv_out(w, __ldg(a.b + c), xin[0], xin[1], xin[2], xin[3]);
}

// The new shift-register state of each channel; runs after conv_seq_kernel (which reads the old one).
__global__ void __launch_bounds__(256) conv_state_kernel(ConvSeqArgs a) {
  const int c = blockIdx.x * blockDim.x + threadIdx.x;
  if (c >= a.C) return;
  float nv[3];
#pragma unroll
  for (int k = 0; k < 3; ++k) {
    const int tk = a.M - 3 + k;
    nv[k] = tk >= 0 ? a.zx[(size_t)tk * a.ld_zx + a.x_off + c] : a.state[(size_t)c * 3 + (tk + 3)];
  }
#pragma unroll
  for (int k = 0; k < 3; ++k) a.state[(size_t)c * 3 + k] = nv[k];
}

// ------------------------------------------------------------------------------ SSM scan
// NJ float4 chunks of the state row per lane (N <= 128 NJ).  Shared memory per buffer: B and C of ST
// tokens (2 ST N floats), x and z of the CTA's rows (2 ST SW), dt and dA (2 ST); plus two ST x SW
// buffers of gated outputs.
template <int NJ>
__global__ void __launch_bounds__(SW * 32, NJ == 1 ? 2 : 1) ssm_scan_kernel(ScanArgs a) {
  extern __shared__ __align__(16) float smf[];
  const int N = a.N, n4 = N / 4;
  const int buf_floats = 2 * ST * N + 2 * ST * SW + 2 * ST;
  float* gs = smf + 2 * buf_floats;  // [2][ST][SW]
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int row0 = blockIdx.x * SW;  // SW consecutive (h, p) rows of one head (P % SW == 0)
  const int h = row0 / a.P;
  const int grp = h / (a.H / a.G);
  const int E = a.H * a.P;
  const int row = row0 + warp;
  const float Dh = __ldg(a.D + h), dtb = __ldg(a.dt_bias + h), Al = __ldg(a.A_log + h);
  const float* Bsrc = a.xc + a.b_off + (size_t)grp * N;
  const float* Csrc = a.xc + a.c_off + (size_t)grp * N;

  float4 S[NJ];
#pragma unroll
  for (int j = 0; j < NJ; ++j) {
    const int c = lane + 32 * j;
    S[j] = c < n4 ? reinterpret_cast<const float4*>(a.state + (size_t)row * N)[c] : make_float4(0.f, 0.f, 0.f, 0.f);
  }

  // staging of chunk k into registers, then into buffer k & 1
  constexpr int PF = (2 * ST * 32 * NJ + SW * 32 - 1) / (SW * 32);  // B/C float4 per thread (max)
  float4 pbc[PF];
  float px = 0.f, pz = 0.f, pdt = 0.f;
  const auto load_chunk = [&](int t0) {
    const int nT = min(ST, a.M - t0);
#pragma unroll
    for (int k = 0; k < PF; ++k) {
      const int i = tid + k * SW * 32;
      pbc[k] = make_float4(0.f, 0.f, 0.f, 0.f);
      if (i < nT * 2 * n4) {
        const int tt = i / (2 * n4), rem = i - tt * 2 * n4;
        const int which = rem >= n4, c = rem - which * n4;
        const float* src = (which ? Csrc : Bsrc) + (size_t)(t0 + tt) * a.ld_xc;
        pbc[k] = __ldg(reinterpret_cast<const float4*>(src) + c);
      }
    }
    if (tid < ST * SW) {
      const int tt = tid / SW, w = tid - tt * SW;
      if (tt < nT) {
        px = __ldg(a.xc + (size_t)(t0 + tt) * a.ld_xc + row0 + w);
        pz = __ldg(a.zx + (size_t)(t0 + tt) * a.ld_zx + row0 + w);
      }
    }
    if (tid < nT) pdt = __ldg(a.zx + (size_t)(t0 + tid) * a.ld_zx + a.dt_off + h);
  };
  const auto store_chunk = [&](int t0, int b) {
    const int nT = min(ST, a.M - t0);
    float* base = smf + b * buf_floats;
    float* Bs = base;               // [ST][N]
    float* Cs = base + ST * N;      // [ST][N]
    float* xs = base + 2 * ST * N;  // [ST][SW]
    float* zs = xs + ST * SW;       // [ST][SW]
    float* dts = zs + ST * SW;      // [ST]
    float* dAs = dts + ST;          // [ST]
#pragma unroll
    for (int k = 0; k < PF; ++k) {
      const int i = tid + k * SW * 32;
      if (i < nT * 2 * n4) {
        const int tt = i / (2 * n4), rem = i - tt * 2 * n4;
        const int which = rem >= n4, c = rem - which * n4;
        reinterpret_cast<float4*>((which ? Cs : Bs) + (size_t)tt * N)[c] = pbc[k];
      }
    }
    if (tid < ST * SW) {
      xs[tid] = px;
      zs[tid] = pz;
    }
    if (tid < nT) {
      const float dt = ssm_dt(pdt, dtb);
      dts[tid] = dt;
      dAs[tid] = ssm_dA(dt, Al);
    }
  };

  const int n_chunks = (a.M + ST - 1) / ST;
  load_chunk(0);
  store_chunk(0, 0);
  __syncthreads();
  for (int k = 0; k < n_chunks; ++k) {
    const int t0 = k * ST, nT = min(ST, a.M - t0);
    if (k + 1 < n_chunks) load_chunk(t0 + ST);  // in flight while this chunk is stepped
    // the previous chunk's gated outputs, coalesced
    if (k > 0 && tid < ST * SW) {
      const int tt = tid / SW, w = tid - tt * SW;
      a.g[(size_t)(t0 - ST + tt) * E + row0 + w] = gs[((k - 1) & 1) * ST * SW + tid];
    }
    const float* base = smf + (k & 1) * buf_floats;
    const float* Bs = base;
    const float* Cs = base + ST * N;
    const float* xs = base + 2 * ST * N;
    const float* zs = xs + ST * SW;
    const float* dts = zs + ST * SW;
    const float* dAs = dts + ST;
    float* gout = gs + (k & 1) * ST * SW;
    for (int tt = 0; tt < nT; ++tt) {
      const float dt = dts[tt], dA = dAs[tt], xv = xs[tt * SW + warp];
      const float dtx = fmul(dt, xv);
      double acc = 0.0;
#pragma unroll
      for (int j = 0; j < NJ; ++j) {
        const int c = lane + 32 * j;
        if (c < n4) {
          const float4 b4 = reinterpret_cast<const float4*>(Bs + (size_t)tt * N)[c];
          const float4 c4 = reinterpret_cast<const float4*>(Cs + (size_t)tt * N)[c];
          S[j].x = ssm_state(dA, S[j].x, dtx, b4.x);
          S[j].y = ssm_state(dA, S[j].y, dtx, b4.y);
          S[j].z = ssm_state(dA, S[j].z, dtx, b4.z);
          S[j].w = ssm_state(dA, S[j].w, dtx, b4.w);
          acc = fma((double)S[j].x, (double)c4.x, acc);  // products of two fp32 are exact in fp64
          acc = fma((double)S[j].y, (double)c4.y, acc);
          acc = fma((double)S[j].z, (double)c4.z, acc);
          acc = fma((double)S[j].w, (double)c4.w, acc);
        }
      }
      acc = warp_sum(acc);
      if (lane == 0) {
        const float y = __double2float_rn(dadd(acc, dmul((double)Dh, (double)xv)));
        gout[tt * SW + warp] = fmul(y, silu_f64(zs[tt * SW + warp]));
      }
    }
    if (k + 1 < n_chunks) store_chunk(t0 + ST, (k + 1) & 1);  // buffer (k+1)&1 was last read in chunk k-1
    __syncthreads();
  }
  // the last chunk's gated outputs
  {
    const int k = n_chunks - 1, t0 = k * ST, nT = min(ST, a.M - t0);
    if (tid < ST * SW) {
      const int tt = tid / SW, w = tid - tt * SW;
      if (tt < nT) a.g[(size_t)(t0 + tt) * E + row0 + w] = gs[(k & 1) * ST * SW + tid];
    }
  }
#pragma unroll
  for (int j = 0; j < NJ; ++j) {
    const int c = lane + 32 * j;
    if (c < n4) reinterpret_cast<float4*>(a.state + (size_t)row * N)[c] = S[j];
  }
}

template <int NJ>
cudaError_t launch_scan_nj(const ScanArgs& a, cudaStream_t st) {
  const size_t smem = sizeof(float) * (2 * (2 * ST * a.N + 2 * ST * SW + 2 * ST) + 2 * ST * SW);
  static bool attr = false;
  if (!attr) {
    const cudaError_t e = cudaFuncSetAttribute(ssm_scan_kernel<NJ>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                               (int)(sizeof(float) * (2 * (2 * ST * 512 + 2 * ST * SW + 2 * ST) +
                                                                      2 * ST * SW)));
    if (e != cudaSuccess) return e;
    attr = true;
  }
  ssm_scan_kernel<NJ><<<(a.H * a.P) / SW, SW * 32, smem, st>>>(a);
  return cudaGetLastError();
}

}  // namespace scan

cudaError_t launch_conv_seq(const ConvSeqArgs& a, cudaStream_t st) {
  const long long n = (long long)a.M * a.C;
  scan::conv_seq_kernel<<<(unsigned)((n + 255) / 256), 256, 0, st>>>(a);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  scan::conv_state_kernel<<<(a.C + 255) / 256, 256, 0, st>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_ssm_scan(const ScanArgs& a, cudaStream_t st) {
  if (a.N <= 128) return scan::launch_scan_nj<1>(a, st);
  if (a.N <= 256) return scan::launch_scan_nj<2>(a, st);
  return scan::launch_scan_nj<4>(a, st);
}

bool scan_supported(int H, int P, int N, int G) {
  return P % scan::SW == 0 && N % 4 == 0 && N <= 512 && G >= 1 && H % G == 0;
}

}  // namespace dfssm
