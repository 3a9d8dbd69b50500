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
// rows of one head per CTA, the tokens' B, C, dt, x and z staged through shared memory eight tokens at a
// time, the next chunk's loads in flight while the current one is stepped.

#include "common.cuh"
#include "internal.h"

namespace dfssm {
namespace scan {

constexpr int SW = 16;  // rows (warps) per CTA
constexpr int ST = 8;   // tokens per staged chunk
static_assert(ST == 8, "the scan's token butterfly maps 8 tokens onto lane bits 4..2");

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
// Per-token scalars of the scan, all tokens in parallel ahead of the sequential kernel: the gate
// fl32(SiLU(z)) of every (t, h, p) and dt, dA of every (t, h) (fp64 transcendental functions, rounded as
// in decode).  Thread j < E of token t takes z[t][j]; thread E + h takes head h's dt.
__global__ void __launch_bounds__(256) scan_prep_kernel(ScanArgs a) {
  const int E = a.H * a.P;
  const long long idx = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= (long long)a.M * (E + a.H)) return;
  const int t = (int)(idx / (E + a.H)), j = (int)(idx - (long long)t * (E + a.H));
  if (j < E) {
    a.sz[(size_t)t * E + j] = silu_f64(__ldg(a.zx + (size_t)t * a.ld_zx + j));
  } else {
    const int h = j - E;
    const float dt = ssm_dt(__ldg(a.zx + (size_t)t * a.ld_zx + a.dt_off + h), __ldg(a.dt_bias + h));
    reinterpret_cast<float2*>(a.dtdA)[(size_t)t * a.H + h] = make_float2(dt, ssm_dA(dt, __ldg(a.A_log + h)));
  }
}

// NJ float4 chunks of the state row per lane (N <= 128 NJ).  Shared memory per buffer: B and C of ST
// tokens (2 ST N), x and fl32(SiLU(z)) of the CTA's rows (2 ST SW), dt and dA (2 ST); plus two ST x SW
// buffers of gated outputs.
//
// Per token a lane advances its state elements (the fp32 recurrence) and adds their readout products to
// its partial sum.  Each product S C of two fp32 values is split exactly into fl32(S C) + error (one fma)
// and accumulated as an unevaluated pair of fp32 values (hi + lo, with the exact two-sum error of every
// addition folded into lo): about 48 significant bits, like an fp64 accumulation far below the fp32
// rounding of the result, but on the fp32 pipes (converting every state element to fp64 each step would
// saturate the conversion unit).  The ST partial pairs of a chunk are reduced across the warp together by
// a transposed butterfly (ST/2 + ST/4 + ... exchanges instead of five per token), converted to fp64 once
// per token, and the token outputs are finished by ST lane groups in parallel.
__host__ __device__ constexpr int SCAN_BUF_FLOATS(int N) { return 2 * ST * N + 2 * ST * SW + 2 * ST; }

// (hi, lo) += a: the two-sum of hi and a (exact: hi + a = t + e) with e folded into lo.
__device__ __forceinline__ void df_add(float& hi, float& lo, float a) {
  const float t = __fadd_rn(hi, a);
  const float bp = __fsub_rn(t, hi);
  const float e = __fadd_rn(__fsub_rn(hi, __fsub_rn(t, bp)), __fsub_rn(a, bp));
  hi = t;
  lo = __fadd_rn(lo, e);
}
// (hi, lo) += s c with the product split exactly: s c = p + fma(s, c, -p).
__device__ __forceinline__ void df_add_prod(float& hi, float& lo, float s, float c) {
  const float p = __fmul_rn(s, c);
  lo = __fadd_rn(lo, __fmaf_rn(s, c, -p));
  df_add(hi, lo, p);
}

// NFIX > 0 fixes d_state at compile time (then NJ = NFIX / 128 and every index is a constant shift);
// NFIX = 0 reads it from the arguments.
template <int NJ, int NFIX>
__global__ void __launch_bounds__(SW * 32, NJ == 1 ? 2 : 1) ssm_scan_kernel(ScanArgs a) {
  extern __shared__ __align__(16) float smf[];
  const int N = NFIX > 0 ? NFIX : a.N, n4 = N / 4;
  const int buf_floats = SCAN_BUF_FLOATS(N);
  float* gs = smf + 2 * buf_floats;  // [2][ST][SW]
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int row0 = blockIdx.x * SW;  // SW consecutive (h, p) rows of one head (P % SW == 0)
  const int h = row0 / a.P;
  const int grp = h / (a.H / a.G);
  const int E = a.H * a.P;
  const int row = row0 + warp;
  const float Dh = __ldg(a.D + h);
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
  float px = 0.f, pz = 0.f;
  float2 pdt = make_float2(0.f, 0.f);
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
        pz = __ldg(a.sz + (size_t)(t0 + tt) * E + row0 + w);
      }
    }
    if (tid < nT) pdt = __ldg(reinterpret_cast<const float2*>(a.dtdA) + (size_t)(t0 + tid) * a.H + h);
  };
  const auto store_chunk = [&](int t0, int b) {
    const int nT = min(ST, a.M - t0);
    float* base = smf + b * buf_floats;
    float* Bs = base;                                     // [ST][N]
    float* Cs = base + ST * N;                            // [ST][N]
    float* xs = base + 2 * ST * N;                        // [ST][SW]
    float* szs = xs + ST * SW;                            // [ST][SW] fl32(SiLU(z))
    float* dts = szs + ST * SW;                           // [ST]
    float* dAs = dts + ST;                                // [ST]
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
      szs[tid] = pz;
    }
    if (tid < nT) {
      dts[tid] = pdt.x;
      dAs[tid] = pdt.y;
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
    const float* szs = xs + ST * SW;
    const float* dts = szs + ST * SW;
    const float* dAs = dts + ST;
    // 1. the recurrence through the chunk; (ph[tt], pl[tt]) = this lane's share of token tt's readout
    float ph[ST], pl[ST];
#pragma unroll
    for (int tt = 0; tt < ST; ++tt) {
      ph[tt] = 0.0f;
      pl[tt] = 0.0f;
      if (tt < nT) {
        const float dA = dAs[tt];
        const float dtx = fmul(dts[tt], xs[tt * SW + warp]);
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
            df_add_prod(ph[tt], pl[tt], S[j].x, c4.x);
            df_add_prod(ph[tt], pl[tt], S[j].y, c4.y);
            df_add_prod(ph[tt], pl[tt], S[j].z, c4.z);
            df_add_prod(ph[tt], pl[tt], S[j].w, c4.w);
          }
        }
      }
    }
    // 2. transposed butterfly: after the exchanges over lane bits 4, 3, 2 each lane holds one token's
    //    partial pair (token = lane bits 4..2), summed over lane bits 1, 0 at the end
#pragma unroll
    for (int half = ST / 2, off = 16; half >= 1; half >>= 1, off >>= 1) {
      const bool upper = (lane & off) != 0;
#pragma unroll
      for (int i = 0; i < half; ++i) {
        const float send_h = upper ? ph[i] : ph[i + half], send_l = upper ? pl[i] : pl[i + half];
        const float keep_h = upper ? ph[i + half] : ph[i], keep_l = upper ? pl[i + half] : pl[i];
        const float oh = __shfl_xor_sync(0xffffffffu, send_h, off);
        const float ol = __shfl_xor_sync(0xffffffffu, send_l, off);
        ph[i] = keep_h;
        pl[i] = __fadd_rn(keep_l, ol);
        df_add(ph[i], pl[i], oh);
      }
    }
#pragma unroll
    for (int off = 2; off >= 1; off >>= 1) {
      const float oh = __shfl_xor_sync(0xffffffffu, ph[0], off);
      const float ol = __shfl_xor_sync(0xffffffffu, pl[0], off);
      pl[0] = __fadd_rn(pl[0], ol);
      df_add(ph[0], pl[0], oh);
    }
    const double tot = dadd((double)ph[0], (double)pl[0]);
    // 3. token outputs: lane group g = lane / 4 finishes token g
    {
      const int tt = ((lane >> 4) & 1) * 4 + ((lane >> 3) & 1) * 2 + ((lane >> 2) & 1);
      if ((lane & 3) == 0 && tt < nT) {
        const float xv = xs[tt * SW + warp];
        const float y = __double2float_rn(dadd(tot, dmul((double)Dh, (double)xv)));
        gs[(k & 1) * ST * SW + tt * SW + warp] = fmul(y, szs[tt * SW + warp]);
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

// d_state 128 (the model shape): each lane owns eight state elements (two float4 chunks: c and c + 16),
// a warp two (h, p) rows (lanes 0-15 and 16-31), a CTA of eight warps the same sixteen rows of one head
// as above.  Twice the state elements per lane spread the per-token loads, the butterfly and the output
// step over twice the work; the butterfly runs within each half-warp (token = lane bits 3..1).
constexpr int W128 = SW / 2;  // warps per CTA
__global__ void __launch_bounds__(W128 * 32, 2) ssm_scan128_kernel(ScanArgs a) {
  constexpr int N = 128, n4 = 32;
  constexpr int NT = W128 * 32;
  extern __shared__ __align__(16) float smf[];
  constexpr int buf_floats = SCAN_BUF_FLOATS(N);
  float* gs = smf + 2 * buf_floats;  // [2][ST][SW]
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int hl = lane & 15;                // lane within the half-warp
  const int rloc = 2 * warp + (lane >> 4);  // this half-warp's row within the CTA
  const int row0 = blockIdx.x * SW;
  const int h = row0 / a.P;
  const int grp = h / (a.H / a.G);
  const int E = a.H * a.P;
  const int row = row0 + rloc;
  const float Dh = __ldg(a.D + h);
  const float* Bsrc = a.xc + a.b_off + (size_t)grp * N;
  const float* Csrc = a.xc + a.c_off + (size_t)grp * N;

  float4 S[2];
#pragma unroll
  for (int j = 0; j < 2; ++j) S[j] = reinterpret_cast<const float4*>(a.state + (size_t)row * N)[hl + 16 * j];

  constexpr int PF = 2 * ST * n4 / NT;  // B/C float4 per thread per chunk (2)
  float4 pbc[PF];
  float px = 0.f, pz = 0.f;
  float2 pdt = make_float2(0.f, 0.f);
  const auto load_chunk = [&](int t0) {
    const int nT = min(ST, a.M - t0);
#pragma unroll
    for (int k = 0; k < PF; ++k) {
      const int i = tid + k * NT;  // < 2 ST n4
      const int tt = i >> 6, which = (i >> 5) & 1, c = i & 31;
      pbc[k] = tt < nT ? __ldg(reinterpret_cast<const float4*>((which ? Csrc : Bsrc) + (size_t)(t0 + tt) * a.ld_xc) + c)
                       : make_float4(0.f, 0.f, 0.f, 0.f);
    }
    if (tid < ST * SW) {
      const int tt = tid / SW, w = tid - tt * SW;
      if (tt < nT) {
        px = __ldg(a.xc + (size_t)(t0 + tt) * a.ld_xc + row0 + w);
        pz = __ldg(a.sz + (size_t)(t0 + tt) * E + row0 + w);
      }
    }
    if (tid < nT) pdt = __ldg(reinterpret_cast<const float2*>(a.dtdA) + (size_t)(t0 + tid) * a.H + h);
  };
  const auto store_chunk = [&](int t0, int b) {
    const int nT = min(ST, a.M - t0);
    float* base = smf + b * buf_floats;
#pragma unroll
    for (int k = 0; k < PF; ++k) {
      const int i = tid + k * NT;
      const int tt = i >> 6, which = (i >> 5) & 1, c = i & 31;
      reinterpret_cast<float4*>(base + which * ST * N + tt * N)[c] = pbc[k];
    }
    float* xs = base + 2 * ST * N;
    if (tid < ST * SW) {
      xs[tid] = px;
      xs[ST * SW + tid] = pz;
    }
    if (tid < nT) {
      xs[2 * ST * SW + tid] = pdt.x;
      xs[2 * ST * SW + ST + tid] = pdt.y;
    }
  };

  const int n_chunks = (a.M + ST - 1) / ST;
  load_chunk(0);
  store_chunk(0, 0);
  __syncthreads();
  for (int k = 0; k < n_chunks; ++k) {
    const int t0 = k * ST, nT = min(ST, a.M - t0);
    if (k + 1 < n_chunks) load_chunk(t0 + ST);
    if (k > 0 && tid < ST * SW) {
      const int tt = tid / SW, w = tid - tt * SW;
      a.g[(size_t)(t0 - ST + tt) * E + row0 + w] = gs[((k - 1) & 1) * ST * SW + tid];
    }
    const float* base = smf + (k & 1) * buf_floats;
    const float* Bs = base;
    const float* Cs = base + ST * N;
    const float* xs = base + 2 * ST * N;
    const float* szs = xs + ST * SW;
    const float* dts = szs + ST * SW;
    const float* dAs = dts + ST;
    float ph[ST], pl[ST];
#pragma unroll
    for (int tt = 0; tt < ST; ++tt) {
      ph[tt] = 0.0f;
      pl[tt] = 0.0f;
      if (tt < nT) {
        const float dA = dAs[tt];
        const float dtx = fmul(dts[tt], xs[tt * SW + rloc]);
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          const float4 b4 = reinterpret_cast<const float4*>(Bs + tt * N)[hl + 16 * j];
          const float4 c4 = reinterpret_cast<const float4*>(Cs + tt * N)[hl + 16 * j];
          S[j].x = ssm_state(dA, S[j].x, dtx, b4.x);
          S[j].y = ssm_state(dA, S[j].y, dtx, b4.y);
          S[j].z = ssm_state(dA, S[j].z, dtx, b4.z);
          S[j].w = ssm_state(dA, S[j].w, dtx, b4.w);
          df_add_prod(ph[tt], pl[tt], S[j].x, c4.x);
          df_add_prod(ph[tt], pl[tt], S[j].y, c4.y);
          df_add_prod(ph[tt], pl[tt], S[j].z, c4.z);
          df_add_prod(ph[tt], pl[tt], S[j].w, c4.w);
        }
      }
    }
    // transposed butterfly within each half-warp over lane bits 3, 2, 1, then the pair over bit 0
#pragma unroll
    for (int half = ST / 2, off = 8; half >= 1; half >>= 1, off >>= 1) {
      const bool upper = (lane & off) != 0;
#pragma unroll
      for (int i = 0; i < half; ++i) {
        const float send_h = upper ? ph[i] : ph[i + half], send_l = upper ? pl[i] : pl[i + half];
        const float keep_h = upper ? ph[i + half] : ph[i], keep_l = upper ? pl[i + half] : pl[i];
        const float oh = __shfl_xor_sync(0xffffffffu, send_h, off);
        const float ol = __shfl_xor_sync(0xffffffffu, send_l, off);
        ph[i] = keep_h;
        pl[i] = __fadd_rn(keep_l, ol);
        df_add(ph[i], pl[i], oh);
      }
    }
    {
      const float oh = __shfl_xor_sync(0xffffffffu, ph[0], 1);
      const float ol = __shfl_xor_sync(0xffffffffu, pl[0], 1);
      pl[0] = __fadd_rn(pl[0], ol);
      df_add(ph[0], pl[0], oh);
    }
    {
      const int tt = ((lane >> 3) & 1) * 4 + ((lane >> 2) & 1) * 2 + ((lane >> 1) & 1);
      if ((lane & 1) == 0 && tt < nT) {
        const double tot = dadd((double)ph[0], (double)pl[0]);
        const float xv = xs[tt * SW + rloc];
        const float y = __double2float_rn(dadd(tot, dmul((double)Dh, (double)xv)));
        gs[(k & 1) * ST * SW + tt * SW + rloc] = fmul(y, szs[tt * SW + rloc]);
      }
    }
    if (k + 1 < n_chunks) store_chunk(t0 + ST, (k + 1) & 1);
    __syncthreads();
  }
  {
    const int k = n_chunks - 1, t0 = k * ST, nT = min(ST, a.M - t0);
    if (tid < ST * SW) {
      const int tt = tid / SW, w = tid - tt * SW;
      if (tt < nT) a.g[(size_t)(t0 + tt) * E + row0 + w] = gs[(k & 1) * ST * SW + tid];
    }
  }
#pragma unroll
  for (int j = 0; j < 2; ++j) reinterpret_cast<float4*>(a.state + (size_t)row * N)[hl + 16 * j] = S[j];
}

template <int NJ, int NFIX>
cudaError_t launch_scan_nj(const ScanArgs& a, cudaStream_t st) {
  const size_t smem = sizeof(float) * (2 * SCAN_BUF_FLOATS(a.N) + 2 * ST * SW);
  {
    const cudaError_t e = set_max_dynamic_smem(reinterpret_cast<const void*>(ssm_scan_kernel<NJ, NFIX>),
                                               (int)(sizeof(float) * (2 * SCAN_BUF_FLOATS(512) + 2 * ST * SW)));
    if (e != cudaSuccess) return e;
  }
  const long long n_prep = (long long)a.M * (a.H * a.P + a.H);
  scan_prep_kernel<<<(unsigned)((n_prep + 255) / 256), 256, 0, st>>>(a);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  ssm_scan_kernel<NJ, NFIX><<<(a.H * a.P) / SW, SW * 32, smem, st>>>(a);
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
  if (a.N == 128) {
    const size_t smem = sizeof(float) * (2 * scan::SCAN_BUF_FLOATS(128) + 2 * scan::ST * scan::SW);
    const long long n_prep = (long long)a.M * (a.H * a.P + a.H);
    scan::scan_prep_kernel<<<(unsigned)((n_prep + 255) / 256), 256, 0, st>>>(a);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    scan::ssm_scan128_kernel<<<(a.H * a.P) / scan::SW, scan::W128 * 32, smem, st>>>(a);
    return cudaGetLastError();
  }
  if (a.N <= 128) return scan::launch_scan_nj<1, 0>(a, st);
  if (a.N <= 256) return scan::launch_scan_nj<2, 0>(a, st);
  return scan::launch_scan_nj<4, 0>(a, st);
}

bool scan_supported(int H, int P, int N, int G) {
  return P % scan::SW == 0 && N % 4 == 0 && N <= 512 && G >= 1 && H % G == 0;
}

}  // namespace dfssm
