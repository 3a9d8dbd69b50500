// Fused persistent decode of a DF-SSM Mamba-2 stack: one cooperative launch carries one token through
// every layer (gist.science technical summary of DF-SSM, §2.C: batch-1 decode of the 1-bit scaffold with
// int8 LoRA, the conv shift register and the SSM recurrence; the pages capture the 48-layer forward as a
// CUDA graph — here the whole forward is one kernel, so no launch sits between layers).
//
// One CTA per SM owns a fixed slice of every layer:
//   * ~E/NC SSM rows (h,p): their SSM state rows, the matching z and x rows of in_proj, the conv
//     channels of those x rows;
//   * ~320/NC of the rows every CTA needs (B, C and dt rows of in_proj): the CTA computes their outputs
//     to the end — B and C through their conv channel and SiLU, dt through softplus and the decay dA —
//     and publishes the final values;
//   * ~d_model/NC rows of out_proj and the matching entries of the residual stream (kept in registers
//     from layer to layer).
// The weights and states of a CTA's slice are loaded into registers and shared memory at the start of
// the layer (and prefetched into L2 one layer ahead), before the CTA waits on anything, so the HBM stream
// overlaps the dependency chain.
//
// Cross-CTA hand-offs (three per layer: the residual stream h, the B/C/dt values, the gated SSM output g)
// carry their synchronisation in the data: every exchanged fp32 value travels as one 64-bit word
// {value, tag} written with a single relaxed store, the tag naming the layer that produced it.  A reader
// polls exactly the words it needs until their tags match, so a hand-off costs one trip through L2 — no
// counter, no release fence, no second read of the data.  Single buffers suffice: a CTA can only produce
// layer l+1's words after every CTA has consumed layer l's (each hand-off needs the previous one from all
// CTAs).  The tags are cleared before every launch.
//
// Every CTA quantizes the whole h (and g) itself, so it also computes the LoRA down-projection
// t = W_B q of the codes itself (exact int32 dp4a against W_B staged in shared memory).  A poll that runs
// past its clock budget records DFSSM_ETIMEOUT in the workspace status word; the CTA (and every other
// CTA, which sees the abort word) then waits for its own copies in flight and returns.
//
// All arithmetic goes through the functions in common.cuh, so the results are those of the per-op path.

#include "common.cuh"
#include "internal.h"

namespace dfssm {
namespace fused {

constexpr int DM = 2048, E = 4096, H = 64, P = 64, N = 128, R = 16;
constexpr int SH0 = 2 * E;              // first in_proj row every CTA needs (B rows, then C, then dt)
constexpr int NSH = 2 * N + H;          // 320 such rows
constexpr int NT = 512, NW = NT / 32;   // NW == R: warp r computes LoRA row r
constexpr int MAX_IN = 64, MAX_OUT = 16, MAX_SSM = 32;
static_assert((DM & (DM - 1)) == 0 && (E & (E - 1)) == 0, "norm lengths are powers of two");
constexpr int MIN_CTAS = 137, MAX_CTAS = 256;  // >= 137: <= 15 out_proj rows, <= 3 shared rows per CTA
static_assert(NW == R, "one warp per LoRA row");
constexpr int kCopyThread = 64;         // warp 2: the layer's out-set copy (end of the previous layer)
constexpr int kPrefetchThread = 224;    // warp 7: the next layer's L2 prefetches (phase B)
constexpr int kAheadCopyThread = 256;   // warp 8: the next layer's in-set and state copies (phase B)
constexpr int kBcWarp = NW - 1;         // warp 15: LoRA intermediates and the shared rows' epilogues
constexpr int kBcBase = kBcWarp * 32;
constexpr int kZxBase = 320;            // threads kZxBase + j: epilogues of the CTA's z and x rows j

struct LayerPtrs {
  const uint32_t* in_bits;
  const float* in_ws;
  const int8_t* in_lb;
  const float* in_lbs;
  const int8_t* in_la;
  const float* in_las;
  const uint32_t* out_bits;
  const float* out_ws;
  const int8_t* out_lb;
  const float* out_lbs;
  const int8_t* out_la;
  const float* out_las;
  const float* conv_w;
  const float* conv_b;
  const float* A_log;
  const float* dt_bias;
  const float* D;
  const float* norm_w;
  const float* gnorm_w;
  float* conv_state;
  float* ssm_state;
};

struct Params {
  LayerPtrs L[DFSSM_MAX_LAYERS];
  int n_layers;
  float* hidden;
  int* err;
  int* status;
  unsigned long long* hx;   // [DM]   tagged residual stream
  unsigned long long* gx;   // [E]    tagged gated SSM output
  unsigned long long* bcx;  // [2N + 2H] tagged B, C (after conv + SiLU), then (dt, dA) per head
  long long spin_limit;
};

// ------------------------------------------------------------------------------ phase trace
// Built only with -DDFSSM_TRACE_DECODE (bit_quantized_mamba_b200/trace_decode.py): thread 0 of CTAs 0 and
// kTraceCta2 stamps the global timer (ns) at eleven points of every layer, read by
// dfssm_decode_trace_ptr().  The default build has no stamps.
#ifdef DFSSM_TRACE_DECODE
constexpr int kTraceCta2 = 74;  // a CTA on the other die
constexpr int kTracePoints = 12;
__device__ unsigned long long g_decode_trace[2 * 64 * kTracePoints];
__device__ __forceinline__ unsigned long long trace_now() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}
#define DTR(k)                                                                                          \
  do {                                                                                                  \
    if (threadIdx.x == 0 && (blockIdx.x == 0 || blockIdx.x == kTraceCta2) && l < 64)                    \
      g_decode_trace[((blockIdx.x == 0 ? 0 : 1) * 64 + l) * kTracePoints + (k)] = trace_now();          \
  } while (0)
#else
#define DTR(k) \
  do {         \
  } while (0)
#endif

// ------------------------------------------------------------------------------ workspace layout
// [status word 128 B][abort word 128 B][hx DM x 8 B][gx E x 8 B][bcx (2N + 2H) x 8 B]
// Everything from the abort word on is cleared before every launch (tag 0 = not yet written); the
// status word is sticky: a timed-out wait stores kTimeoutMagic there, and only dfssm_device_status
// clears it.
constexpr size_t OFF_STATUS = 0;
constexpr size_t OFF_ERR = 128;
constexpr size_t OFF_HX = 256;
constexpr size_t OFF_GX = OFF_HX + DM * 8;
constexpr size_t OFF_BCX = OFF_GX + E * 8;
constexpr size_t WS_BYTES = OFF_BCX + (2 * N + 2 * H) * 8;
constexpr size_t CLEAR_OFF = OFF_ERR, CLEAR_BYTES = WS_BYTES - OFF_ERR;
// dynamic shared memory, filled by bulk copies:
//   in-set  [2] (layers of each parity): W_B of in_proj [R][DM] + the pre-norm weight [DM] (one layer ahead)
//   out-set     W_B of out_proj [R][E] + the gated-norm weight [E] (issued at the start of the layer)
//   state   [2] the CTA's SSM state rows (one layer ahead)
constexpr int IN_SET = R * DM + DM * 4;
constexpr int OUT_SET = R * E + E * 4;
constexpr int ST_BYTES = MAX_SSM * N * 4;
constexpr int OFF_OUT_SET = 2 * IN_SET;
constexpr int OFF_STATE = OFF_OUT_SET + OUT_SET;
constexpr int DYN_BYTES = OFF_STATE + 2 * ST_BYTES;

constexpr int kTimeoutMagic = kDeviceTimeout;

// ------------------------------------------------------------------------------ tagged exchange

__device__ __forceinline__ int ld_relaxed(const int* p) {
  int v;
  asm volatile("ld.relaxed.gpu.global.s32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ void st_tagged(unsigned long long* p, float v, uint32_t tag) {
  const unsigned long long w = ((unsigned long long)tag << 32) | (unsigned long long)__float_as_uint(v);
  asm volatile("st.relaxed.gpu.global.u64 [%0], %1;" ::"l"(p), "l"(w) : "memory");
}
// Two consecutive tagged words (16-byte aligned); each 64-bit word is read as one single-copy-atomic unit.
__device__ __forceinline__ ulonglong2 ld_tagged2(const unsigned long long* p) {
  ulonglong2 r;
  asm volatile("ld.relaxed.gpu.global.v2.u64 {%0, %1}, [%2];" : "=l"(r.x), "=l"(r.y) : "l"(p) : "memory");
  return r;
}
__device__ __forceinline__ bool tag_is(unsigned long long w, uint32_t tag) { return (uint32_t)(w >> 32) == tag; }
__device__ __forceinline__ float tag_val(unsigned long long w) { return __uint_as_float((uint32_t)w); }

// This thread's NP pairs of tagged words at base + off[k] (16-byte aligned) until all carry `tag`;
// values to v[2k], v[2k+1].  Bounded: false when the clock budget ran out (the abort and status words are
// then set) or another CTA already aborted.
template <int NP>
__device__ bool poll_pairs(const unsigned long long* base, const int (&off)[NP], uint32_t tag, float (&v)[2 * NP],
                           int* err, int* status, long long limit) {
  uint32_t pending = (1u << NP) - 1u;
  long long t0 = 0;
  unsigned it = 0;
  while (true) {
    ulonglong2 r[NP];
#pragma unroll
    for (int k = 0; k < NP; ++k)
      if ((pending >> k) & 1u) r[k] = ld_tagged2(base + off[k]);
#pragma unroll
    for (int k = 0; k < NP; ++k) {
      if (((pending >> k) & 1u) && tag_is(r[k].x, tag) && tag_is(r[k].y, tag)) {
        v[2 * k] = tag_val(r[k].x);
        v[2 * k + 1] = tag_val(r[k].y);
        pending &= ~(1u << k);
      }
    }
    if (pending == 0u) return true;
    if (it == 0) t0 = clock64();
    if ((++it & 7u) == 0) {
      if (ld_relaxed(err) != 0) return false;
      if (clock64() - t0 > limit) {
        atomicExch(err, 1);
        atomicExch(status, kTimeoutMagic);
        return false;
      }
    }
  }
}

// Named CTA barrier `id` over n threads: bar_arrive signals (and publishes this thread's earlier shared-
// memory writes) without waiting; bar_sync waits until all n have arrived.
__device__ __forceinline__ void bar_sync(int id, int n) { asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory"); }
__device__ __forceinline__ void bar_arrive(int id, int n) { asm volatile("bar.arrive %0, %1;" ::"r"(id), "r"(n) : "memory"); }

// ------------------------------------------------------------------------------ asynchronous copies

__device__ __forceinline__ void prefetch_l2(const void* p, unsigned bytes) {
  if (bytes >= 16)
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(p), "r"(bytes & ~15u) : "memory");
}

// One prefetch per 128-byte line of [p, p + bytes) (the first line is aligned down inside the array).
__device__ __forceinline__ void prefetch_lines(const void* p, unsigned bytes) {
  const char* a = reinterpret_cast<const char*>(reinterpret_cast<uintptr_t>(p) & ~uintptr_t(127));
  const char* e = reinterpret_cast<const char*>(p) + bytes;
  for (; a < e; a += 128) asm volatile("prefetch.global.L2 [%0];" ::"l"(a) : "memory");
}

// Asynchronous global -> shared copies, committed in groups; a thread waits for its own groups
// (cp_async_wait<N>: all but the N most recent are complete), and a CTA barrier then publishes them.
__device__ __forceinline__ void cp_async4(void* dst, const void* src) {
  const unsigned d = (unsigned)__cvta_generic_to_shared(dst);
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(d), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async16(void* dst, const void* src) {
  const unsigned d = (unsigned)__cvta_generic_to_shared(dst);
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(d), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// Bulk asynchronous copies (one instruction per contiguous range) with mbarrier completion.
__device__ __forceinline__ uint32_t smem_u32(const void* q) { return (uint32_t)__cvta_generic_to_shared(q); }
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred q;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 q, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}
// Bounded wait for the phase with the given parity; false when the clock budget ran out.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, long long limit) {
  if (mbar_try_wait(bar, parity)) return true;
  const long long t0 = clock64();
  while (!mbar_try_wait(bar, parity))
    if (clock64() - t0 > limit) return false;
  return true;
}
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

// ------------------------------------------------------------------------------ block helpers

// LoRA down-projection of the K natural-order codes qn against W_B [R][K], split by inputs: warp w takes
// inputs [w K/16, (w+1) K/16) for all R rows (each lane K/512 consecutive codes, read once) and leaves
// its R partial sums in red_t[w][0..R); t[r] = sum_w red_t[w][r] (exact int32).
template <int K>
__device__ __forceinline__ void lora_slice(const int8_t* wb, const int8_t* qn, int warp, int lane,
                                           int (*red_t)[R]) {
  constexpr int WPL = K / (16 * 32 * 4);  // 4-byte words per lane
  static_assert(WPL == 1 || WPL == 2, "K is 2048 or 4096");
  const int i0 = warp * (K / 16) + lane * 4 * WPL;
  uint32_t q[WPL];
  if constexpr (WPL == 1) {
    q[0] = *reinterpret_cast<const uint32_t*>(qn + i0);
  } else {
    const uint2 v = *reinterpret_cast<const uint2*>(qn + i0);
    q[0] = v.x;
    q[1] = v.y;
  }
  int part[R];
#pragma unroll
  for (int r = 0; r < R; ++r) {
    if constexpr (WPL == 1) {
      part[r] = dp4a_ss(*reinterpret_cast<const uint32_t*>(wb + r * K + i0), q[0], 0);
    } else {
      const uint2 w = *reinterpret_cast<const uint2*>(wb + r * K + i0);
      part[r] = dp4a_ss(w.y, q[1], dp4a_ss(w.x, q[0], 0));
    }
  }
#pragma unroll
  for (int r = 0; r < R; ++r) {
    const int t = __reduce_add_sync(0xffffffffu, part[r]);
    if (lane == r) red_t[warp][r] = t;
  }
}
__device__ __forceinline__ int lora_t_sum(const int (*red_t)[R], int r) {
  int t = 0;
#pragma unroll
  for (int w = 0; w < NW; ++w) t += red_t[w][r];
  return t;
}

// Block-wide fp64 sum of the threads' v (every thread gets the same value: the sixteen per-warp sums are
// added in one fixed tree order), and the OR over the block of `flag` (through *any_flag, zero before
// the call).  Contains one CTA barrier.
__device__ __forceinline__ double block_sum_d(double v, int lane, int warp, double* red_d, bool flag,
                                              int* any_flag, bool& any) {
  v = warp_sum(v);
  if (lane == 0) red_d[warp] = v;
  if (flag) *any_flag = 1;
  __syncthreads();
  double a[NW / 2];
#pragma unroll
  for (int q = 0; q < NW / 2; ++q) {
    const double2 d = reinterpret_cast<const double2*>(red_d)[q];
    a[q] = d.x + d.y;
  }
#pragma unroll
  for (int w = NW / 4; w > 0; w >>= 1)
#pragma unroll
    for (int q = 0; q < w; ++q) a[q] = a[2 * q] + a[2 * q + 1];
  any = *any_flag != 0;
  return a[0];
}
// rms_factor for a row of length n = 2^k, with ss / n formed as the (exact) product by 2^-k, which equals
// the IEEE quotient.
__device__ __forceinline__ float rms_factor_pow2(double ss, int n) {
  return __double2float_rn(rsqrt(__dadd_rn(__dmul_rn(ss, 1.0 / (double)n), 1e-5)));
}
// Block-wide absmax of the threads' non-negative m (one redux per warp; the bit patterns of non-negative
// floats order like the floats).  Contains one CTA barrier.
__device__ __forceinline__ float block_absmax(float m, int lane, int warp, unsigned* red_u) {
  const unsigned mw = __reduce_max_sync(0xffffffffu, __float_as_uint(m));
  if (lane == 0) red_u[warp] = mw;
  __syncthreads();
  unsigned mb = 0u;
#pragma unroll
  for (int q = 0; q < NW / 4; ++q) {
    const uint4 u = reinterpret_cast<const uint4*>(red_u)[q];
    mb = max(max(mb, u.x), max(u.y, max(u.z, u.w)));
  }
  return __uint_as_float(mb);
}
// Sum of the sixteen per-warp partial sums.
__device__ __forceinline__ int block_sum16(const int* red_i) {
  int t = 0;
#pragma unroll
  for (int q = 0; q < NW / 4; ++q) {
    const int4 u = reinterpret_cast<const int4*>(red_i)[q];
    t += (u.x + u.y) + (u.z + u.w);
  }
  return t;
}

// Sum over bit=1 positions of q for 128 weights (one uint4 of sign bits) against the eight 16-byte chunks
// of their segment's dp4a-permuted codes held in registers (as bits_dot).
__device__ __forceinline__ int bits_dot_reg(uint4 w, const uint4 (&q)[8]) {
  int acc8[8];
#pragma unroll
  for (int k = 0; k < 8; ++k) acc8[k] = 0;
  const uint32_t w4[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const uint32_t qp[8] = {q[2 * j].x, q[2 * j].y, q[2 * j].z, q[2 * j].w,
                            q[2 * j + 1].x, q[2 * j + 1].y, q[2 * j + 1].z, q[2 * j + 1].w};
#pragma unroll
    for (int k = 0; k < 8; ++k) acc8[k] = dp4a_us(w4[j] & (0x01010101u << k), qp[k], acc8[k]);
  }
  int S = 0;
#pragma unroll
  for (int k = 0; k < 8; ++k) S += acc8[k] >> k;
  return S;
}

// RMSNorm of the NV values this thread holds of a row of length n (the row's squares summed over the
// block; the weights w_sm in shared memory), then the quantizer on the normalized row: codes to q_perm
// (dp4a segment layout, NSEG segments) and q_nat, their per-warp sums to red_i.  Element k of the thread is
// row index idx[k] (k even, k + 1 adjacent).  Returns the scale s; `abort_any` is true (for every thread)
// when some thread's wait failed (`failed`).  Contains three CTA barriers.
template <int NV, int NSEG>
__device__ __forceinline__ float norm_quantize(const float (&hv)[NV], const float* w_sm, const int (&idx)[NV],
                                               int n, int lane, int warp, double* red_d, unsigned* red_u,
                                               int* red_i, int* any_flag, int8_t* q_perm, int8_t* q_nat,
                                               bool failed, bool& abort_any) {
  double ss = 0.0;
#pragma unroll
  for (int k = 0; k < NV; ++k) ss += (double)hv[k] * (double)hv[k];  // exact squares in fp64
  const float rn = rms_factor_pow2(block_sum_d(ss, lane, warp, red_d, failed, any_flag, abort_any), n);
  float v[NV];
  float m = 0.0f;
#pragma unroll
  for (int k = 0; k < NV; k += 2) {
    const float2 w = *reinterpret_cast<const float2*>(w_sm + idx[k]);
    v[k] = norm_value(hv[k], rn, w.x);
    v[k + 1] = norm_value(hv[k + 1], rn, w.y);
    m = fmaxf(m, fmaxf(fabsf(v[k]), fabsf(v[k + 1])));
  }
  m = block_absmax(m, lane, warp, red_u);
  const float s0 = quant_scale(m);
  const float inv_s0 = quant_inv(s0);
  int cd[NV];
  quant_codes<NV>(v, s0, inv_s0, cd);
  int sq = 0;
#pragma unroll
  for (int k = 0; k < NV; ++k) {
    q_perm[seg_index<NSEG>(idx[k])] = (int8_t)cd[k];
    q_nat[idx[k]] = (int8_t)cd[k];
    sq += cd[k];
  }
  sq = __reduce_add_sync(0xffffffffu, sq);
  if (lane == 0) red_i[warp] = sq;
  __syncthreads();
  return s0;
}

// ------------------------------------------------------------------------------ the kernel
//
// Per layer (three hand-offs, tags: h entering layer l carries l; B/C/dt and g of layer l carry l + 1):
//   A  h (poll; layer 0 reads the input) -> RMSNorm + quantize, scaffold GEMV of the owned in_proj rows,
//      LoRA-down; the shared rows' epilogues (B/C conv + SiLU, dt softplus + dA) published
//   B  the own z/x rows' epilogues (gate value SiLU(z), x conv); B/C/dt (poll) -> SSM of the owned rows,
//      g = y SiLU(z) published
//   C  g (poll) -> gated RMSNorm + quantize, LoRA-down, out_proj GEMV of the owned rows, residual;
//      the new h published (the last layer writes it to the output instead)

__global__ void __launch_bounds__(NT, 1) decode_kernel(const __grid_constant__ Params p) {
  extern __shared__ __align__(128) int8_t dyn_sm[];
  // every layer's pointers, copied once: the layer loop never indexes the parameter block at run time
  __shared__ LayerPtrs lsm[DFSSM_MAX_LAYERS];
  const auto wb_in = [&](int l) { return dyn_sm + (l & 1) * IN_SET; };
  const auto nw_sm = [&](int l) { return reinterpret_cast<const float*>(dyn_sm + (l & 1) * IN_SET + R * DM); };
  int8_t* const wb_out = dyn_sm + OFF_OUT_SET;
  const float* const gw_sm = reinterpret_cast<const float*>(dyn_sm + OFF_OUT_SET + R * E);
  float* const st_sm = reinterpret_cast<float*>(dyn_sm + OFF_STATE);  // [2][MAX_SSM][N], layer l in l & 1
  __shared__ __align__(16) int8_t q_perm[E];
  __shared__ __align__(16) int8_t q_nat[E];
  __shared__ __align__(16) double red_d[NW];
  __shared__ __align__(16) unsigned red_u[NW];
  __shared__ __align__(16) int red_i[NW];
  __shared__ int any_flag[2];                   // [0] the pre-norm quantizer's, [1] the gated norm's
  __shared__ float lbs_in[R], lbs_o[2][R];      // W_B row scales (out_proj's by layer parity)
  __shared__ __align__(16) int red_t[NW][R];  // LoRA-down partial sums, per warp
  __shared__ double tf_d[R];                    // in_proj LoRA intermediates
  __shared__ float s_in_sm;
  // in_proj rows owned by this CTA (slot order: shared rows, z rows, x rows)
  __shared__ int acc_in[MAX_IN];
  __shared__ float in_sw[MAX_IN], in_sa[MAX_IN];
  __shared__ __align__(16) int8_t in_wa[MAX_IN][R];
  // bulk-copy completion: the in-set of layer l on inbar[l & 1] (once per two layers), the out-set on
  // outbar (once per layer)
  __shared__ uint64_t inbar[2], outbar;
  // SSM state rows of layer l arrive in buffer l & 1, one layer ahead (completes once per two layers)
  __shared__ uint64_t stbar[2];
  __shared__ __align__(16) float Bsm[N];
  __shared__ __align__(16) double Cd[N];
  __shared__ float zsm[MAX_SSM], xsm[MAX_SSM];
  __shared__ float dtv[2], dAv[2], Dv[2];
  // out_proj rows
  __shared__ int acc_out[MAX_OUT];
  __shared__ float o_sw[MAX_OUT], o_sa[MAX_OUT];
  __shared__ __align__(16) int8_t o_wa[MAX_OUT][R];

  const int c = blockIdx.x, NC = gridDim.x;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

  // ---- fixed ownership
  const int rs0 = (int)((long long)c * E / NC), rs1 = (int)((long long)(c + 1) * E / NC);
  const int n_ssm = rs1 - rs0;
  const int sh0 = c * NSH / NC, sh1 = (c + 1) * NSH / NC, n_sh = sh1 - sh0;
  const int ro0 = c * DM / NC, ro1 = (c + 1) * DM / NC, n_out = ro1 - ro0;
  const int n_in = n_sh + 2 * n_ssm;
  const int hA = rs0 / P;                       // first head of this CTA's SSM rows
  const int n_heads = (rs1 - 1) / P - hA + 1;   // one or two heads
  auto in_row = [&](int slot) -> int {
    if (slot < n_sh) return SH0 + sh0 + slot;
    const int j = slot - n_sh;
    return j < n_ssm ? rs0 + j : E + rs0 + (j - n_ssm);
  };
  const int li_in = lane & 15;
  const int slot_in[2] = {warp * 2 + (lane >> 4), 32 + warp * 2 + (lane >> 4)};
  const int slot_out = warp;  // out_proj: one row per warp, 32 lanes x 128 weights
  const int ssm_slot[2] = {warp, NW + warp};
  // this thread's entries of h (k < 4) and of g (k < 8): the pairs 2 tr, 2 tr + 1 of each 1024-block, with
  // the thread index rotated per CTA so that the CTAs' simultaneous reads of a hand-off spread over L2
  const int tr = (tid + 53 * c) & (NT - 1);
  int hidx[4], gidx[8];
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    const int i = 2 * tr + (k & 1) + 1024 * (k >> 1);
    if (k < 4) hidx[k] = i;
    gidx[k] = i;
  }
  const int hoff[2] = {2 * tr, 1024 + 2 * tr};
  const int goff[4] = {2 * tr, 1024 + 2 * tr, 2048 + 2 * tr, 3072 + 2 * tr};
  // the shared row of this thread (warp kBcWarp, lanes < n_sh): B/C (conv channel E + k) or dt (head)
  const int bc_j = tid - kBcBase;
  const bool bc_own = bc_j >= 0 && bc_j < n_sh;
  const int bc_k = sh0 + bc_j;
  float h_own = 0.0f;  // residual stream entry ro0 + tid (tid < n_out), carried from layer to layer

  {
    // LayerPtrs is 21 pointers: thread t copies pointer t % 21 of layer t / 21
    constexpr int NPTR = sizeof(LayerPtrs) / sizeof(void*);
    static_assert(sizeof(LayerPtrs) == NPTR * sizeof(void*), "LayerPtrs holds pointers only");
    const void* const* src = reinterpret_cast<const void* const*>(p.L);
    const void** dst = reinterpret_cast<const void**>(lsm);
    for (int k = tid; k < p.n_layers * NPTR; k += NT) dst[k] = src[k];
    if (tid < 2) any_flag[tid] = 0;
    if (tid == 0) {
      mbar_init(&inbar[0], 1);
      mbar_init(&inbar[1], 1);
      mbar_init(&outbar, 1);
      mbar_init(&stbar[0], 1);
      mbar_init(&stbar[1], 1);
      asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
      // layer 0's SSM state rows and in-set
      mbar_expect_tx(&stbar[0], n_ssm * N * 4);
      bulk_g2s(st_sm, p.L[0].ssm_state + (size_t)rs0 * N, n_ssm * N * 4, &stbar[0]);
      mbar_expect_tx(&inbar[0], IN_SET);
      bulk_g2s(wb_in(0), p.L[0].in_lb, R * DM, &inbar[0]);
      bulk_g2s(wb_in(0) + R * DM, p.L[0].norm_w, DM * 4, &inbar[0]);
    }
    if (tid < n_out) h_own = p.hidden[ro0 + tid];
    __syncthreads();
  }
  // An aborting CTA first waits (bounded) for everything it may still have landing in its shared memory:
  // its own cp.async copies and the bulk copies of layer l.
  // next_issued: the next layer's in-set and state copies (phase B of layer l) were issued.
  const auto drain = [&](int l, bool next_issued) {
    cp_async_wait<0>();
    if (tid == 0) {
      mbar_wait(&inbar[l & 1], (l >> 1) & 1, p.spin_limit);
      mbar_wait(&outbar, l & 1, p.spin_limit);
      mbar_wait(&stbar[l & 1], (l >> 1) & 1, p.spin_limit);
      if (next_issued) {
        mbar_wait(&stbar[(l + 1) & 1], ((l + 1) >> 1) & 1, p.spin_limit);
        mbar_wait(&inbar[(l + 1) & 1], ((l + 1) >> 1) & 1, p.spin_limit);
      }
    }
  };
  const auto fail = [&]() {
    atomicExch(p.err, 1);
    atomicExch(p.status, kTimeoutMagic);
  };
  // What layer ll needs from memory at the start of its dependency chain: its sign bits and row parameters
  // (registers, cp.async into shared memory) and its out-set (bulk copy).  Issued at the end of the
  // previous layer (for layer 0, before the loop), after every read of the buffers it refills.  The
  // layer's in-set and SSM state rows are copied, and the next layer's slice prefetched into L2, during
  // the previous layer's phase B by warps that idle there (issue_ahead).
  uint4 w_in[2], w_out;
  float4 cw = make_float4(0.f, 0.f, 0.f, 0.f);
  float cb = 0.f, cs0 = 0.f, cs1 = 0.f, cs2 = 0.f;
  float bsw = 0.f, bsa = 0.f;
  uint4 bwa = make_uint4(0, 0, 0, 0);
  float4 bcw = make_float4(0.f, 0.f, 0.f, 0.f);
  float bcb = 0.f, bs0 = 0.f, bs1 = 0.f, bs2 = 0.f, dtb = 0.f, A_h = 0.f;
  const auto issue_loads = [&](int ll) {
    const LayerPtrs& Lq = lsm[ll];
    // registers: sign bits
#pragma unroll
    for (int ps = 0; ps < 2; ++ps) {
      const int slot = slot_in[ps];
      w_in[ps] = slot < n_in ? ld_stream_u4(Lq.in_bits + (size_t)in_row(slot) * (DM / 32) + li_in * 4)
                             : make_uint4(0, 0, 0, 0);
    }
    w_out = slot_out < n_out ? ld_stream_u4(Lq.out_bits + (size_t)(ro0 + slot_out) * (E / 32) + lane * 4)
                             : make_uint4(0, 0, 0, 0);
    // own x channels: conv taps, bias, state (thread kZxBase + j handles channel rs0 + j)
    if (tid >= kZxBase && tid - kZxBase < n_ssm) {
      const int ch = rs0 + (tid - kZxBase);
      cw = __ldg(reinterpret_cast<const float4*>(Lq.conv_w) + ch);
      cb = __ldg(Lq.conv_b + ch);
      cs0 = Lq.conv_state[(size_t)ch * 3 + 0];
      cs1 = Lq.conv_state[(size_t)ch * 3 + 1];
      cs2 = Lq.conv_state[(size_t)ch * 3 + 2];
    }
    // the shared row of this thread: its epilogue parameters and its conv channel or head parameters
    if (bc_own) {
      const int row = SH0 + bc_k;
      bsw = __ldg(Lq.in_ws + row);
      bsa = __ldg(Lq.in_las + row);
      bwa = __ldg(reinterpret_cast<const uint4*>(Lq.in_la + (size_t)row * R));
      if (bc_k < 2 * N) {
        const int ch = E + bc_k;
        bcw = __ldg(reinterpret_cast<const float4*>(Lq.conv_w) + ch);
        bcb = __ldg(Lq.conv_b + ch);
        bs0 = Lq.conv_state[(size_t)ch * 3 + 0];
        bs1 = Lq.conv_state[(size_t)ch * 3 + 1];
        bs2 = Lq.conv_state[(size_t)ch * 3 + 2];
      } else {
        dtb = __ldg(Lq.dt_bias + (bc_k - 2 * N));
        A_h = __double2float_rn(-exp((double)__ldg(Lq.A_log + (bc_k - 2 * N))));
      }
    }
    // epilogue parameters of the owned rows into shared memory, asynchronously
    if (tid < n_in) {
      const int row = in_row(tid);
      cp_async4(&in_sw[tid], Lq.in_ws + row);
      cp_async4(&in_sa[tid], Lq.in_las + row);
      cp_async16(in_wa[tid], Lq.in_la + (size_t)row * R);
    }
    if (tid == kCopyThread) {
      // this layer's out-set (its buffer was last read before the previous layer's GEMV barrier); every
      // generic access of the previous layer to it is ordered before the copy by that barrier
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      mbar_expect_tx(&outbar, OUT_SET);
      bulk_g2s(wb_out, Lq.out_lb, R * E, &outbar);
      bulk_g2s(wb_out + R * E, Lq.gnorm_w, E * 4, &outbar);
    }
    if (tid < n_out) {
      const int row = ro0 + tid;
      cp_async4(&o_sw[tid], Lq.out_ws + row);
      cp_async4(&o_sa[tid], Lq.out_las + row);
      cp_async16(o_wa[tid], Lq.out_la + (size_t)row * R);
    }
    if (tid < 2 && hA + tid < H) cp_async4(&Dv[tid], Lq.D + hA + tid);
    if (tid < R) {
      cp_async4(&lbs_in[tid], Lq.in_lbs + tid);
      cp_async4(&lbs_o[ll & 1][tid], Lq.out_lbs + tid);
    }
    cp_async_commit();  // this thread's row parameters (awaited before the quantizer's barriers)
  };
  issue_loads(0);
  // During phase B of layer l (l + 1 < n_layers): the next layer's SSM state rows and in-set into the
  // buffers of its parity (both last read in layer l - 1, before this layer's barriers) and the L2 prefetch
  // of the next layer's slice, by warps that idle while the B/C/dt values are awaited.
  const auto issue_ahead = [&](int l) {
    if (tid == kAheadCopyThread) {
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      const int nb = (l + 1) & 1;
      mbar_expect_tx(&stbar[nb], n_ssm * N * 4);
      bulk_g2s(st_sm + nb * MAX_SSM * N, lsm[l + 1].ssm_state + (size_t)rs0 * N, n_ssm * N * 4, &stbar[nb]);
      mbar_expect_tx(&inbar[nb], IN_SET);
      bulk_g2s(wb_in(l + 1), lsm[l + 1].in_lb, R * DM, &inbar[nb]);
      bulk_g2s(wb_in(l + 1) + R * DM, lsm[l + 1].norm_w, DM * 4, &inbar[nb]);
    }
    if (tid == kPrefetchThread || tid == kPrefetchThread + 1) {
      // this CTA's slice of the next layer, and (spread over CTAs 0..2) the parts every CTA reads.
      // A bulk prefetch stalls its thread, so an otherwise idle warp issues them.
      const LayerPtrs& Nx = lsm[l + 1];
      if (tid == kPrefetchThread) {
        prefetch_l2(Nx.in_bits + (size_t)(SH0 + sh0) * (DM / 32), n_sh * (DM / 8));
        prefetch_l2(Nx.in_bits + (size_t)rs0 * (DM / 32), n_ssm * (DM / 8));
        prefetch_l2(Nx.in_bits + (size_t)(E + rs0) * (DM / 32), n_ssm * (DM / 8));
        prefetch_l2(Nx.out_bits + (size_t)ro0 * (E / 32), n_out * (E / 8));
        prefetch_l2(Nx.ssm_state + (size_t)rs0 * N, n_ssm * N * 4);
        prefetch_l2(Nx.in_la + (size_t)rs0 * R, n_ssm * R);
        prefetch_l2(Nx.in_la + (size_t)(E + rs0) * R, n_ssm * R);
        prefetch_l2(Nx.out_la + (size_t)ro0 * R, n_out * R);
        prefetch_l2(Nx.conv_w + (size_t)rs0 * 4, n_ssm * 16);
      } else {
        prefetch_lines(Nx.in_ws + rs0, n_ssm * 4);
        prefetch_lines(Nx.in_ws + E + rs0, n_ssm * 4);
        prefetch_lines(Nx.in_las + rs0, n_ssm * 4);
        prefetch_lines(Nx.in_las + E + rs0, n_ssm * 4);
        prefetch_lines(Nx.out_ws + ro0, n_out * 4);
        prefetch_lines(Nx.out_las + ro0, n_out * 4);
        prefetch_lines(Nx.conv_b + rs0, n_ssm * 4);
        prefetch_lines(Nx.conv_state + (size_t)rs0 * 3, n_ssm * 12);
        switch (c) {
          case 1: prefetch_l2(Nx.gnorm_w, E * 4); prefetch_l2(Nx.out_lb, R * E); break;
          case 2:
            prefetch_lines(Nx.dt_bias, H * 4);
            prefetch_lines(Nx.A_log, H * 4);
            prefetch_lines(Nx.D, H * 4);
            prefetch_lines(Nx.in_lbs, R * 4);
            prefetch_lines(Nx.out_lbs, R * 4);
            break;
          default: break;
        }
      }
    }
  };
  for (int l = 0; l < p.n_layers; ++l) {
    const LayerPtrs& Lp = lsm[l];
    const bool has_next = l + 1 < p.n_layers;
    const uint32_t tag_h = (uint32_t)l, tag_l = (uint32_t)(l + 1);

    // ---------------------------------------------------------------- phase A: h -> in_proj
    DTR(0);
    float hv[4];
    bool ok = true;
    if (l == 0) {
#pragma unroll
      for (int k = 0; k < 4; k += 2) {
        const float2 v = *reinterpret_cast<const float2*>(p.hidden + hidx[k]);
        hv[k] = v.x;
        hv[k + 1] = v.y;
      }
    } else {
      // every warp has finished the previous layer (the out_proj epilogue and the loads for this layer)
      // before any thread starts polling: spinning loads would otherwise slow those warps down
      __syncthreads();
      ok = poll_pairs<2>(p.hx, hoff, tag_h, hv, p.err, p.status, p.spin_limit);
    }
    DTR(1);
    cp_async_wait<0>();  // this thread's row parameters; the quantizer's barriers publish them
    if (ok && !mbar_wait(&inbar[l & 1], (l >> 1) & 1, p.spin_limit)) {  // in_proj W_B and the norm weight
      fail();
      ok = false;
    }
    bool abort_any = false;
    const float s_in = norm_quantize<4, DM / 128>(hv, nw_sm(l), hidx, DM, lane, warp, red_d, red_u, red_i,
                                                  &any_flag[0], q_perm, q_nat, !ok, abort_any);
    if (abort_any) {
      drain(l, false);
      return;
    }
    DTR(2);
    if (tid == 0) any_flag[1] = 0;  // the gated norm's flag (last read in the previous layer)
    const int sumq = block_sum16(red_i);
    // scaffold GEMV over the owned rows, pass 0 (the shared rows first), then LoRA-down row `warp`
    uint4 qreg[8];  // this lane's segment of the codes, for both passes
#pragma unroll
    for (int v = 0; v < 8; ++v) qreg[v] = reinterpret_cast<const uint4*>(q_perm)[li_in + v * (DM / 128)];
    {
      int S = bits_dot_reg(w_in[0], qreg);
#pragma unroll
      for (int o = 8; o > 0; o >>= 1) S += __shfl_xor_sync(0xffffffffu, S, o);
      if (li_in == 0 && slot_in[0] < n_in) acc_in[slot_in[0]] = 2 * S - sumq;
      lora_slice<DM>(wb_in(l), q_nat, warp, lane, red_t);
    }
    __syncthreads();
    DTR(3);
    const auto pass1 = [&]() {
      int S = bits_dot_reg(w_in[1], qreg);
#pragma unroll
      for (int o = 8; o > 0; o >>= 1) S += __shfl_xor_sync(0xffffffffu, S, o);
      if (li_in == 0 && slot_in[1] < n_in) acc_in[slot_in[1]] = 2 * S - sumq;
    };
    if (warp == kBcWarp) {
      // LoRA intermediates (published to the z/x epilogues through barrier 1 without waiting there),
      // then the shared rows' epilogues, published to every CTA as final values
      if (lane < R) tf_d[lane] = (double)lora_tf(lora_t_sum(red_t, lane), lbs_in[lane], s_in);
      if (lane == R) s_in_sm = s_in;
      if (32 + warp * 2 < n_in) pass1();  // only when a CTA owns more than 62 in_proj rows
      bar_arrive(1, NT);
      __syncwarp();
      if (bc_own) {
        double tfl[R];
#pragma unroll
        for (int r = 0; r < R; ++r) tfl[r] = tf_d[r];
        const float y = linear_out_d(acc_in[bc_j], (double)s_in, (double)bsw, (double)bsa, bwa, tfl, R);
        if (bc_k < 2 * N) {
          st_tagged(p.bcx + bc_k, conv_out(bcw, bcb, bs0, bs1, bs2, y), tag_l);
          float* st = Lp.conv_state + (size_t)(E + bc_k) * 3;
          st[0] = bs1;
          st[1] = bs2;
          st[2] = y;
        } else {
          const float dt = ssm_dt(y, dtb);
          const float dA = __double2float_rn(exp((double)fmul(dt, A_h)));
          const int hh = bc_k - 2 * N;
          st_tagged(p.bcx + 2 * N + 2 * hh, dt, tag_l);
          st_tagged(p.bcx + 2 * N + 2 * hh + 1, dA, tag_l);
        }
      }
    } else {
      // pass 1: the remaining z/x rows
      if (32 + warp * 2 < n_in) pass1();
      bar_sync(1, NT);
    }

    // ---------------------------------------------------------------- phase B: z/x epilogues + SSM
    DTR(4);
    if (tid >= kZxBase && tid - kZxBase < n_ssm) {
      // the owned z rows (gate value SiLU(z) kept) and x rows (conv of the owned x channels)
      const int j = tid - kZxBase;
      const int sz = n_sh + j, sx = n_sh + n_ssm + j;
      double tfl[R];
#pragma unroll
      for (int r = 0; r < R; ++r) tfl[r] = tf_d[r];
      const double sd = (double)s_in_sm;
      const float zr = linear_out_d(acc_in[sz], sd, (double)in_sw[sz], (double)in_sa[sz],
                                    *reinterpret_cast<const uint4*>(in_wa[sz]), tfl, R);
      const float xr = linear_out_d(acc_in[sx], sd, (double)in_sw[sx], (double)in_sa[sx],
                                    *reinterpret_cast<const uint4*>(in_wa[sx]), tfl, R);
      zsm[j] = silu_f64(zr);
      xsm[j] = conv_out(cw, cb, cs0, cs1, cs2, xr);
      float* st = Lp.conv_state + (size_t)(rs0 + j) * 3;
      st[0] = cs1;
      st[1] = cs2;
      st[2] = xr;
    }
    if (has_next) issue_ahead(l);
    // B and C (threads 0..127: one pair each), dt and dA of the CTA's heads (threads 128, 129)
    ok = true;
    if (tid < N) {
      float v[2];
      const int off[1] = {2 * tid};
      ok = poll_pairs<1>(p.bcx, off, tag_l, v, p.err, p.status, p.spin_limit);
      if (ok) {
        const int i = 2 * tid;
        if (i < N) {
          Bsm[i] = v[0];
          Bsm[i + 1] = v[1];
        } else {
          Cd[i - N] = (double)v[0];
          Cd[i + 1 - N] = (double)v[1];
        }
      }
    } else if (tid - N < n_heads) {
      float v[2];
      const int off[1] = {2 * N + 2 * (hA + tid - N)};
      ok = poll_pairs<1>(p.bcx, off, tag_l, v, p.err, p.status, p.spin_limit);
      if (ok) {
        dtv[tid - N] = v[0];
        dAv[tid - N] = v[1];
      }
    }
    if (ok && !mbar_wait(&stbar[l & 1], (l >> 1) & 1, p.spin_limit)) {  // this layer's SSM state rows
      fail();
      ok = false;
    }
    if (__syncthreads_or(!ok)) {
      drain(l, has_next);
      return;
    }
    DTR(5);
    float4 snew[2];
#pragma unroll
    for (int ps = 0; ps < 2; ++ps) {
      const int rr = ssm_slot[ps];
      snew[ps] = make_float4(0.f, 0.f, 0.f, 0.f);
      if (rr < n_ssm) {
        const int hp = rs0 + rr;
        const int hi = hp / P - hA;
        const float dt = dtv[hi], dA = dAv[hi];
        const float xv = xsm[rr];
        const float dtx = fmul(dt, xv);
        const float4 b4 = reinterpret_cast<const float4*>(Bsm)[lane];
        const double2 c01 = reinterpret_cast<const double2*>(Cd)[2 * lane];
        const double2 c23 = reinterpret_cast<const double2*>(Cd)[2 * lane + 1];
        float4 s4 = reinterpret_cast<const float4*>(st_sm + ((l & 1) * MAX_SSM + rr) * N)[lane];
        s4.x = ssm_state(dA, s4.x, dtx, b4.x);
        s4.y = ssm_state(dA, s4.y, dtx, b4.y);
        s4.z = ssm_state(dA, s4.z, dtx, b4.z);
        s4.w = ssm_state(dA, s4.w, dtx, b4.w);
        snew[ps] = s4;
        double acc = (double)s4.x * c01.x;
        acc = fma((double)s4.y, c01.y, acc);
        acc = fma((double)s4.z, c23.x, acc);
        acc = fma((double)s4.w, c23.y, acc);
        acc = warp_sum(acc);
        if (lane == 0) {
          const float y = __double2float_rn(dadd(acc, dmul((double)Dv[hi], (double)xv)));
          st_tagged(p.gx + hp, fmul(y, zsm[rr]), tag_l);
        }
      }
    }
#pragma unroll
    for (int ps = 0; ps < 2; ++ps)
      if (ssm_slot[ps] < n_ssm) st_f4(Lp.ssm_state + (size_t)(rs0 + ssm_slot[ps]) * N + lane * 4, snew[ps]);

    // ---------------------------------------------------------------- phase C: gated norm -> out_proj
    DTR(6);
    float gv[8];
    __syncthreads();  // as before the h poll: no thread spins while others still work on this phase
    ok = poll_pairs<4>(p.gx, goff, tag_l, gv, p.err, p.status, p.spin_limit);
    DTR(7);
    if (ok && !mbar_wait(&outbar, l & 1, p.spin_limit)) {  // out_proj W_B and the gated-norm weight
      fail();
      ok = false;
    }
    const float s_out = norm_quantize<8, E / 128>(gv, gw_sm, gidx, E, lane, warp, red_d, red_u, red_i,
                                                  &any_flag[1], q_perm, q_nat, !ok, abort_any);
    if (abort_any) {
      drain(l, has_next);
      return;
    }
    DTR(8);
    if (tid == 0) any_flag[0] = 0;  // the next layer's pre-norm flag
    {
      // LoRA down of the codes (by input slices); every warp with an out_proj row then takes it
      lora_slice<E>(wb_out, q_nat, warp, lane, red_t);
      if (slot_out < n_out) {
        const int sumq_c = block_sum16(red_i);
        int S = bits_dot<E / 128>(w_out, reinterpret_cast<const uint4*>(q_perm) + lane);
        S = warp_sum(S);
        if (lane == 0) acc_out[slot_out] = 2 * S - sumq_c;
      }
    }
    __syncthreads();
    DTR(9);
    if (warp == 0) {
      // lanes r < R form the LoRA intermediate tf[r]; every epilogue lane takes all sixteen by shuffle
      const double tf_r = lane < R ? (double)lora_tf(lora_t_sum(red_t, lane), lbs_o[l & 1][lane], s_out) : 0.0;
      double tfd[R];
#pragma unroll
      for (int r = 0; r < R; ++r) tfd[r] = __shfl_sync(0xffffffffu, tf_r, r);
      if (tid < n_out) {
        const float y = linear_out_d(acc_out[tid], (double)s_out, (double)o_sw[tid], (double)o_sa[tid],
                                     *reinterpret_cast<const uint4*>(o_wa[tid]), tfd, R);
        h_own = fadd(h_own, y);
        if (has_next) st_tagged(p.hx + ro0 + tid, h_own, tag_l);
        else p.hidden[ro0 + tid] = h_own;
      }
    }
    DTR(10);
    if (has_next) issue_loads(l + 1);
    DTR(11);
  }
}

// Polls a tagged word that nothing writes, with a short budget: exercises the timeout path.
__global__ void timeout_selftest_kernel(const unsigned long long* word, int* err, int* status, long long limit) {
  float v[2];
  const int off[1] = {0};
  poll_pairs<1>(word, off, 1u, v, err, status, limit);
}

}  // namespace fused

size_t fused_decode_workspace_bytes() { return fused::WS_BYTES; }

bool fused_decode_supported(const dfssm_dims_t& d, int B, const dfssm_layer_t* layers, int n,
                            float* const* conv_states) {
  if (B != 1 || d.d_model != fused::DM || d.nheads != fused::H || d.headdim != fused::P ||
      d.d_state != fused::N || d.ngroups != 1)
    return false;
  // vector loads (16 bytes: W_A rows, conv taps; 8 bytes: norm weights) and the bulk copies of W_B
  const auto a16 = [](const void* q) { return (reinterpret_cast<uintptr_t>(q) & 15) == 0; };
  const auto a8 = [](const void* q) { return (reinterpret_cast<uintptr_t>(q) & 7) == 0; };
  for (int l = 0; l < n; ++l) {
    const dfssm_layer_t& L = layers[l];
    if (L.in_proj.rank != fused::R || L.out_proj.rank != fused::R) return false;
    if (!a16(L.in_proj.lora_a) || !a16(L.out_proj.lora_a) || !a16(L.in_proj.lora_b) ||
        !a16(L.out_proj.lora_b) || !a16(L.conv_w) || !a8(L.norm_w) || !a8(L.gnorm_w) ||
        !a16(conv_states[l]))
      return false;
  }
  const int nc = num_sms();
  // ownership limits: in_proj rows per CTA <= 64, out_proj rows <= 16, SSM rows <= 32
  if (nc < fused::MIN_CTAS || nc > fused::MAX_CTAS) return false;
  int coop = 0, dev = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&coop, cudaDevAttrCooperativeLaunch, dev);
  return coop != 0;
}

cudaError_t launch_fused_decode(const dfssm_layer_t* layers, int n_layers, float* hidden,
                                float* const* conv_states, float* const* ssm_states, void* ws,
                                cudaStream_t st, long long spin_limit) {
  static_assert(sizeof(fused::Params) < 32000, "kernel parameter block too large");
  fused::Params p;  // copied into the launch
  for (int l = 0; l < n_layers; ++l) {
    const dfssm_layer_t& Ly = layers[l];
    fused::LayerPtrs& q = p.L[l];
    q.in_bits = Ly.in_proj.bits;
    q.in_ws = Ly.in_proj.w_scale;
    q.in_lb = Ly.in_proj.lora_b;
    q.in_lbs = Ly.in_proj.lora_b_scale;
    q.in_la = Ly.in_proj.lora_a;
    q.in_las = Ly.in_proj.lora_a_scale;
    q.out_bits = Ly.out_proj.bits;
    q.out_ws = Ly.out_proj.w_scale;
    q.out_lb = Ly.out_proj.lora_b;
    q.out_lbs = Ly.out_proj.lora_b_scale;
    q.out_la = Ly.out_proj.lora_a;
    q.out_las = Ly.out_proj.lora_a_scale;
    q.conv_w = Ly.conv_w;
    q.conv_b = Ly.conv_b;
    q.A_log = Ly.A_log;
    q.dt_bias = Ly.dt_bias;
    q.D = Ly.D;
    q.norm_w = Ly.norm_w;
    q.gnorm_w = Ly.gnorm_w;
    q.conv_state = conv_states[l];
    q.ssm_state = ssm_states[l];
  }
  char* base = static_cast<char*>(ws);
  p.n_layers = n_layers;
  p.hidden = hidden;
  p.status = reinterpret_cast<int*>(base + fused::OFF_STATUS);
  p.err = reinterpret_cast<int*>(base + fused::OFF_ERR);
  p.hx = reinterpret_cast<unsigned long long*>(base + fused::OFF_HX);
  p.gx = reinterpret_cast<unsigned long long*>(base + fused::OFF_GX);
  p.bcx = reinterpret_cast<unsigned long long*>(base + fused::OFF_BCX);
  p.spin_limit = spin_limit;
  cudaError_t e = cudaMemsetAsync(base + fused::CLEAR_OFF, 0, fused::CLEAR_BYTES, st);
  if (e != cudaSuccess) return e;
  e = set_max_dynamic_smem(reinterpret_cast<const void*>(fused::decode_kernel), fused::DYN_BYTES);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(num_sms());
  cfg.blockDim = dim3(fused::NT);
  cfg.dynamicSmemBytes = fused::DYN_BYTES;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, fused::decode_kernel, p);
}

cudaError_t launch_timeout_selftest(void* ws, cudaStream_t st, long long spin_limit) {
  char* base = static_cast<char*>(ws);
  int* err = reinterpret_cast<int*>(base + fused::OFF_ERR);
  int* status = reinterpret_cast<int*>(base + fused::OFF_STATUS);
  const unsigned long long* word = reinterpret_cast<const unsigned long long*>(base + fused::OFF_HX);
  cudaError_t e = cudaMemsetAsync(base + fused::CLEAR_OFF, 0, fused::CLEAR_BYTES, st);
  if (e != cudaSuccess) return e;
  fused::timeout_selftest_kernel<<<1, 32, 0, st>>>(word, err, status, spin_limit);
  return cudaGetLastError();
}

#ifdef DFSSM_TRACE_DECODE
extern "C" void* dfssm_decode_trace_ptr() {
  void* q = nullptr;
  return cudaGetSymbolAddress(&q, fused::g_decode_trace) == cudaSuccess ? q : nullptr;
}
#endif

}  // namespace dfssm
