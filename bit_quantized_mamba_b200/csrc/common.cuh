// Internal device helpers shared by the libdfssm kernels (sm_100a only).
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

#include "dfssm.h"

#if defined(__CUDA_ARCH__) && (__CUDA_ARCH__ < 1000)
#error "libdfssm is built for sm_100a only"
#endif

namespace dfssm {

constexpr int kWarp = 32;

// ---------------------------------------------------------------- programmatic dependent launch
// A kernel launched with programmatic stream serialization may start before the previous kernel of the
// stream has finished.  Everything it reads that an earlier kernel may write (activations, states,
// workspace) and everything it writes must come after pdl_wait(); only immutable weights may be
// fetched before it.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// ---------------------------------------------------------------- loads
// Streaming 16-byte load of read-only data that is used once (weights): not allocated in L1.
__device__ __forceinline__ uint4 ld_stream_u4(const void* p) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p));
  return r;
}
__device__ __forceinline__ uint32_t ld_stream_u32(const void* p) {
  uint32_t r;
  asm volatile("ld.global.nc.L1::no_allocate.u32 %0, [%1];" : "=r"(r) : "l"(p));
  return r;
}
__device__ __forceinline__ float4 ld_stream_f4(const void* p) {
  float4 r;
  asm volatile("ld.global.nc.L1::no_allocate.v4.f32 {%0, %1, %2, %3}, [%4];"
               : "=f"(r.x), "=f"(r.y), "=f"(r.z), "=f"(r.w)
               : "l"(p));
  return r;
}
// 16-byte load of data that is read once and then overwritten by this thread (SSM state): no L1.
__device__ __forceinline__ float4 ld_evict_first_f4(const void* p) {
  float4 r;
  asm volatile("ld.global.L1::no_allocate.v4.f32 {%0, %1, %2, %3}, [%4];"
               : "=f"(r.x), "=f"(r.y), "=f"(r.z), "=f"(r.w)
               : "l"(p));
  return r;
}
__device__ __forceinline__ void st_f4(void* p, float4 v) {
  asm volatile("st.global.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(p), "f"(v.x), "f"(v.y), "f"(v.z),
               "f"(v.w)
               : "memory");
}

// ---------------------------------------------------------------- integer dot products
// d = c + sum_j a.u8[j] * b.s8[j]   (a unsigned bytes, b signed bytes)
__device__ __forceinline__ int dp4a_us(uint32_t a, uint32_t b, int c) {
  int d;
  asm("dp4a.u32.s32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}
// d = c + sum_j a.s8[j] * b.s8[j]
__device__ __forceinline__ int dp4a_ss(uint32_t a, uint32_t b, int c) {
  int d;
  asm("dp4a.s32.s32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}

// ---------------------------------------------------------------- exact-rounding float helpers
// Products and sums that feed a quantizer must be single IEEE operations (never contracted to FMA).
__device__ __forceinline__ float fmul(float a, float b) { return __fmul_rn(a, b); }
__device__ __forceinline__ float fadd(float a, float b) { return __fadd_rn(a, b); }
__device__ __forceinline__ double dmul(double a, double b) { return __dmul_rn(a, b); }
__device__ __forceinline__ double dadd(double a, double b) { return __dadd_rn(a, b); }

// SiLU evaluated in fp64 and rounded once: v / (1 + exp(-v)).
__device__ __forceinline__ float silu_f64(float v) {
  const double d = (double)v;
  return __double2float_rn(__ddiv_rn(d, __dadd_rn(1.0, exp(-d))));
}

// Per-token quantizer scale s0 = fl32(m / 127) of a row with absmax m, and the reciprocal the code fast
// path multiplies by.  s0 is the fp32 rounding of the fp64 product m * fl64(1/127): its relative error is
// below 2^-51, and m / 127 is never within 2^-32 (relative) of an fp32 rounding midpoint (m has a 24-bit
// significand, so 127 times a midpoint would need an odd multiple of 127 to equal an even integer), so the
// result is always the IEEE quotient.  The reciprocal is approximate (relative error ~2^-23), which the
// code fast path tolerates (see quant_codes); m == 0 gives s0 = 0 and a zero reciprocal.
__device__ __forceinline__ float quant_scale(float m) {
  return __double2float_rn(__dmul_rn((double)m, 1.0 / 127.0));
}
__device__ __forceinline__ float quant_inv(float s0) {
  if (s0 == 0.0f) return 0.0f;
  if (s0 < 1e-30f) return __frcp_rn(s0);  // subnormal range: no flush to zero
  float r;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(s0));
  return r;
}

// Round-half-to-even of |t| < 2^22 on the fp32 adder: t + 1.5*2^23 rounds t to an integer (ties to even)
// and leaves that integer in the low significand bits.  kf is the rounded value as a float.
__device__ __forceinline__ int round_even_small(float t, float& kf) {
  const float y = __fadd_rn(t, 12582912.0f);
  kf = __fsub_rn(y, 12582912.0f);
  return __float_as_int(y) - 0x4B400000;
}
__device__ __forceinline__ int clamp127(int k) { return min(max(k, -127), 127); }

// Per-token quantization code of v for scale s0 > 0: clamp(rint(fl32(v / s0)), -127, 127), the IEEE
// quotient rounded half to even.
__device__ __forceinline__ int quant_code(float v, float s0) {
  float kf;
  return clamp127(round_even_small(__fdiv_rn(v, s0), kf));
}
// Same code, computed as the rounding of t = v * inv_s0 unless t lies within 1e-3 of a rounding boundary:
// |v/s0| <= 127, and both t (inv_s0 within 2^-22 of 1/s0) and fl32(v/s0) are within 5e-5 of v/s0, so away
// from a boundary they round to the same integer; near one, the IEEE division decides.
__device__ __forceinline__ int quant_code_fast(float v, float s0, float inv_s0) {
  const float t = v * inv_s0;
  float kf;
  const int k = round_even_small(t, kf);
  if (fabsf(t - kf) < 0.499f) return clamp127(k);
  return quant_code(v, s0);
}
// The codes of N values at once, the same as quant_code_fast for each: the product path for all of them
// without branches, then (rarely) the IEEE division for those close to a rounding boundary, behind one
// branch.  inv_s0 = 0 (an all-zero token) gives code 0 everywhere.  No conversion instructions: the
// rounding runs on the fp32 adder (round_even_small).
template <int N>
__device__ __forceinline__ void quant_codes(const float (&v)[N], float s0, float inv_s0, int (&code)[N]) {
  uint32_t near = 0u;
#pragma unroll
  for (int e = 0; e < N; ++e) {
    const float t = v[e] * inv_s0;
    float kf;
    code[e] = clamp127(round_even_small(t, kf));
    near |= (fabsf(t - kf) < 0.499f ? 0u : 1u) << e;
  }
  if (near) {
#pragma unroll
    for (int e = 0; e < N; ++e)
      if ((near >> e) & 1u) code[e] = quant_code(v[e], s0);
  }
}

// Position of natural-order activation index i inside the dp4a-friendly permuted layout: within each
// 32-element block, word k (k = 0..7) holds elements k, k+8, k+16, k+24 in its four bytes.  With that
// layout, (w & (0x01010101 << k)) selects exactly the sign bits that pair with word k.
__device__ __forceinline__ int perm_index(int i) {
  const int j = i & 31;
  return (i & ~31) + ((j & 7) << 2) + (j >> 3);
}

// ---------------------------------------------------------------- scaffold GEMV inner loop

// Shared-memory position of natural activation index i: the dp4a-permuted codes of 128-input segment
// `seg` occupy eight 16-byte chunks, and chunk v of every segment is stored contiguously across the
// NSEG segments (byte (v * NSEG + seg) * 16 + pos % 16), so the lanes that each own one segment read
// consecutive chunks without bank conflicts.
template <int NSEG>
__device__ __forceinline__ int seg_index(int i) {
  const int seg = i >> 7;
  const int pos = perm_index(i) & 127;
  return ((pos >> 4) * NSEG + seg) * 16 + (pos & 15);
}

// Sum over bit=1 positions of q for 128 weights (one uint4 of sign bits) against the permuted codes of
// their segment; chunk v of the segment is qp4[v * NSEG].
template <int NSEG>
__device__ __forceinline__ int bits_dot(uint4 w, const uint4* qp4) {
  int acc8[8];
#pragma unroll
  for (int k = 0; k < 8; ++k) acc8[k] = 0;
  const uint32_t w4[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const uint4 qa = qp4[(2 * j) * NSEG], qb = qp4[(2 * j + 1) * NSEG];
    const uint32_t qp[8] = {qa.x, qa.y, qa.z, qa.w, qb.x, qb.y, qb.z, qb.w};
#pragma unroll
    for (int k = 0; k < 8; ++k) acc8[k] = dp4a_us(w4[j] & (0x01010101u << k), qp[k], acc8[k]);
  }
  int S = 0;
#pragma unroll
  for (int k = 0; k < 8; ++k) S += acc8[k] >> k;
  return S;
}

// ---------------------------------------------------------------- the method's arithmetic
// These few functions fix the rounding sequence of every fp32 value the decode path stores; all
// kernels (the per-op kernels and the fused decode kernel) use them, so both paths agree bit for bit.

// Exact fp64 value of a 32-bit integer without the (slow) integer-to-double conversion unit:
// 2^52 + 2^31 + w read as a double, minus 2^52 + 2^31.
__device__ __forceinline__ double int_to_f64(int w) {
  return __hiloint2double(0x43300000, w ^ (int)0x80000000) - 4503601774854144.0;
}

// Linear output for one (token, row): fl32(acc*s*sW + sA * sum_r W_A[r]*tf[r]), fp64 in this order.
// Operands already in fp64 (exact images of the fp32 values); wa holds W_A[row][0..15] as 16 bytes
// (entries >= rank ignored).  Integers reach fp64 through int_to_f64, not the conversion unit.
// N independent (token, row) outputs are evaluated with their dependency chains interleaved; RK is the
// rank when known at compile time, or -1 (then `rank` is used).
template <int N, int RK>
__device__ __forceinline__ void linear_out_n(const int (&acc)[N], const double (&s)[N], const double (&sW)[N],
                                             const double (&sA)[N], const uint4 (&wa)[N],
                                             const double* const (&tf)[N], int rank, float (&out)[N]) {
  const int rk = RK >= 0 ? RK : rank;
  double lora[N];
#pragma unroll
  for (int n = 0; n < N; ++n) lora[n] = 0.0;
#pragma unroll
  for (int r = 0; r < DFSSM_MAX_RANK; ++r) {
    if (r < rk) {
#pragma unroll
      for (int n = 0; n < N; ++n) {
        const uint32_t w = r < 4 ? wa[n].x : r < 8 ? wa[n].y : r < 12 ? wa[n].z : wa[n].w;
        // W_A[r] tf[r] is exact in fp64 (8-bit by 24-bit), so the fused multiply-add rounds exactly as
        // the separate product and sum do
        lora[n] = fma(int_to_f64((int)(int8_t)(w >> (8 * (r & 3)))), tf[n][r], lora[n]);
      }
    }
  }
#pragma unroll
  for (int n = 0; n < N; ++n) {
    const double scaffold = dmul(dmul(int_to_f64(acc[n]), s[n]), sW[n]);
    const double corr = rk > 0 ? dmul(sA[n], lora[n]) : 0.0;
    out[n] = __double2float_rn(dadd(scaffold, corr));
  }
}
__device__ __forceinline__ float linear_out_d(int acc, double s, double sW, double sA, uint4 wa,
                                              const double* tf, int rank) {
  const int a[1] = {acc};
  const double sv[1] = {s}, w[1] = {sW}, av[1] = {sA};
  const uint4 wv[1] = {wa};
  const double* const t[1] = {tf};
  float o[1];
  linear_out_n<1, -1>(a, sv, w, av, wv, t, rank, o);
  return o[0];
}
// Same with fp32 operands.
__device__ __forceinline__ float linear_out(int acc, float s, float sW, float sA, uint4 wa, const float* tf,
                                            int rank) {
  double tfd[DFSSM_MAX_RANK];
#pragma unroll
  for (int r = 0; r < DFSSM_MAX_RANK; ++r) tfd[r] = r < rank ? (double)tf[r] : 0.0;
  return linear_out_d(acc, (double)s, (double)sW, (double)sA, wa, tfd, rank);
}
// Same, W_A row in 16-byte-aligned memory (shared memory or registers).
__device__ __forceinline__ float linear_out(int acc, float s, float sW, float sA, const int8_t* wa,
                                            const float* tf, int rank) {
  return linear_out(acc, s, sW, sA, *reinterpret_cast<const uint4*>(wa), tf, rank);
}

// LoRA intermediate tf = fl32(t * sB * s) (fp64, this order): t = sum_i W_B[r,i] q_i is the exact int32
// LoRA-down of the int8 codes q, s the codes' quantizer scale.
__device__ __forceinline__ float lora_tf(int t, float sB, float s) {
  return __double2float_rn(dmul(dmul(int_to_f64(t), (double)sB), (double)s));
}

// RMSNorm (eps 1e-5, a weight per channel), then the quantizer on the normalized row:
//   r = fl32(1 / sqrt(ss / n + 1e-5))   (fp64; ss the fp64 sum of the exact squares of the row)
//   u = fl32(fl32(h * r) * w)
// The reciprocal square root is CUDA's fp64 rsqrt (at most 1 ulp from the real value) rounded once to
// fp32: it gives the fp32 value of the IEEE sqrt-then-divide sequence except when the real value lies
// within about 2 fp64 ulps of an fp32 rounding boundary, the same class of last-bit difference as the
// order of the fp64 sum of squares.
__device__ __forceinline__ float rms_factor(double ss, int n) {
  return __double2float_rn(rsqrt(__dadd_rn(__ddiv_rn(ss, (double)n), 1e-5)));
}
__device__ __forceinline__ float norm_value(float h, float r, float w) { return fmul(fmul(h, r), w); }

// Conv pre-activation fl32(b + w0*s0 + w1*s1 + w2*s2 + w3*x) (fp64, this order), then SiLU.  Each
// product of two fp32 values is exact in fp64, so each fused multiply-add rounds exactly as the separate
// product and sum do.
__device__ __forceinline__ float conv_out(float4 w, float bias, float s0, float s1, float s2, float x) {
  double e = (double)bias;
  e = fma((double)w.x, (double)s0, e);
  e = fma((double)w.y, (double)s1, e);
  e = fma((double)w.z, (double)s2, e);
  e = fma((double)w.w, (double)x, e);
  return silu_f64(__double2float_rn(e));
}

// dt = fl32(softplus(fl32(dt_raw + dt_bias))), softplus(v) = v for v > 20 else log1p(exp(v)) (fp64).
__device__ __forceinline__ float ssm_dt(float dt_raw, float dt_bias) {
  const float v = fadd(dt_raw, dt_bias);
  return v > 20.0f ? v : __double2float_rn(log1p(exp((double)v)));
}
// dA = fl32(exp(fl32(dt * fl32(-exp(A_log))))) (fp64 transcendental functions).
__device__ __forceinline__ float ssm_dA(float dt, float A_log) {
  const float A = __double2float_rn(-exp((double)A_log));
  return __double2float_rn(exp((double)fmul(dt, A)));
}
// One state element: fl32(fl32(dA*S) + fl32(dtx*B)).
__device__ __forceinline__ float ssm_state(float dA, float S, float dtx, float Bn) {
  return fadd(fmul(dA, S), fmul(dtx, Bn));
}

// ---------------------------------------------------------------- block reductions
template <typename T>
__device__ __forceinline__ T warp_sum(T v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

}  // namespace dfssm
