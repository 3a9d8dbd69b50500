// Fused persistent decode of a DF-SSM Mamba-2 stack: one cooperative launch carries one token through
// every layer (gist.science technical summary of DF-SSM, §2.C: batch-1 decode of the 1-bit scaffold with
// int8 LoRA, the conv shift register and the SSM recurrence; the pages capture the 48-layer forward as a
// CUDA graph — here the whole forward is one kernel, so no launch sits between layers).
//
// One CTA per SM owns a fixed slice of every layer:
//   * ~E/NC SSM rows (h,p): their SSM state rows, the matching z and x rows of in_proj, the conv
//     channels of those x rows;
//   * ~320/NC of the rows every CTA needs (B, C and dt rows of in_proj), whose scaffold accumulators it
//     publishes;
//   * ~d_model/NC rows of out_proj and the matching entries of the residual stream.
// The weights and states of a CTA's slice are loaded into registers and shared memory at the start of
// the layer (and prefetched into L2 one layer ahead), before the CTA waits on anything, so the HBM stream
// overlaps the dependency chain.  Cross-CTA hand-offs go through global memory with monotonically
// increasing counters (arrive = CTA barrier + release add; wait = bounded relaxed spin + acquire fence),
// three per layer.  Every CTA quantizes the whole h (and g) itself, so it also computes the LoRA
// down-projection t = W_B q of the codes itself (exact int32 dp4a against W_B staged in shared memory)
// and no hand-off is needed for it.  A wait that runs past its clock budget records DFSSM_ETIMEOUT in the
// workspace status word and the CTA returns.
//
// All arithmetic goes through the functions in common.cuh, so the results are those of the per-op path.

#include "common.cuh"
#include "internal.h"

namespace dfssm {
namespace fused {

constexpr int DM = 2048, E = 4096, H = 64, P = 64, N = 128, R = 16;
constexpr int SH0 = 2 * E;              // first in_proj row every CTA needs (B rows, then C, then dt)
constexpr int NSH = 2 * N + H;          // 320 such rows
constexpr int NT = 512, NW = NT / 32;   // NW == R: warp r computes LoRA row r's partial sums
constexpr int MAX_IN = 64, MAX_OUT = 16, MAX_SSM = 32;
constexpr int MIN_CTAS = 137, MAX_CTAS = 256;  // >= 137: at most 15 out_proj rows per CTA
static_assert(NW == R, "one warp per LoRA row");
constexpr int kPrefetchThread = 32;     // warp 1 issues the next layer's L2 prefetches
constexpr int kCopyThread = 64;         // warp 2 issues the layer's bulk copies (thread 0 polls)
constexpr int kChainWarp = NW - 1;      // warp 15 forms the LoRA intermediate (no out_proj row)
constexpr int kChainBase = kChainWarp * 32;

enum { CTR_H = 0, CTR_BC, CTR_G, N_CTR };
constexpr int CTR_STRIDE = 32;          // one 128-byte line per counter

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
  int* ctr;
  int* err;
  int* status;
  int* sacc;
  float* gbuf;
  long long spin_limit;
};

// ------------------------------------------------------------------------------ workspace layout
// [counters N_CTR x 128 B][abort word 128 B][status word 128 B][sacc 320][gbuf 4096]
// The counters and the abort word are cleared before every launch; the status word is sticky: a timed
// out wait stores kTimeoutMagic there, and only dfssm_device_status clears it.
constexpr size_t OFF_CTR = 0;
constexpr size_t OFF_ERR = OFF_CTR + N_CTR * CTR_STRIDE * 4;
constexpr size_t OFF_STATUS = OFF_ERR + 128;
constexpr size_t CLEAR_BYTES = OFF_STATUS;  // counters + abort word
constexpr size_t OFF_SACC = OFF_STATUS + 128;
constexpr size_t OFF_GBUF = OFF_SACC + ((NSH * 4 + 255) / 256) * 256;
constexpr size_t WS_BYTES = OFF_GBUF + E * 4;
// dynamic shared memory: W_B of in_proj [R][DM] and of out_proj [R][E]
constexpr int WB_BYTES = R * (DM + E);
// dynamic shared memory: W_B of both linears, then the CTA's SSM state rows of two consecutive layers
constexpr int ST_BYTES = MAX_SSM * N * 4;
constexpr int DYN_BYTES = WB_BYTES + 2 * ST_BYTES;

// ------------------------------------------------------------------------------ synchronisation

__device__ __forceinline__ int ld_relaxed(const int* p) {
  int v;
  asm volatile("ld.relaxed.gpu.global.s32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

constexpr int kTimeoutMagic = 0x7E0D1E57;

// All threads of the CTA: returns once *ctr >= target.  Returns false (for every thread) when the
// clock budget ran out (the abort and status words are then set) or another CTA already aborted.
// Thread 0 polls with relaxed loads and finishes with an acquire fence; the CTA barrier then orders
// the other threads' reads after it.
__device__ bool block_wait(const int* ctr, int target, int* err, int* status, long long limit,
                           int* sflag) {
  if (threadIdx.x == 0) {
    int ok = 1;
    if (ld_relaxed(ctr) < target) {
      const long long t0 = clock64();
      unsigned it = 0;
      while (ld_relaxed(ctr) < target) {
        if ((++it & 15u) == 0) {
          if (ld_relaxed(err) != 0) {
            ok = 0;
            break;
          }
          if (clock64() - t0 > limit) {
            atomicExch(err, 1);
            atomicExch(status, kTimeoutMagic);
            ok = 0;
            break;
          }
        }
      }
    }
    if (ok) asm volatile("fence.acq_rel.gpu;" ::: "memory");
    *sflag = ok;
  }
  __syncthreads();
  return *sflag != 0;
}

// All threads of the CTA: count one arrival after every global write the CTA made so far (the CTA
// barrier orders them before thread 0's release).
__device__ __forceinline__ void block_arrive(int* ctr) {
  __syncthreads();
  if (threadIdx.x == 0) asm volatile("red.release.gpu.global.add.s32 [%0], 1;" ::"l"(ctr) : "memory");
}

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

// LoRA down-projection row r = warp: t[r] = sum_i W_B[r,i] q_i over NCH 16-byte chunks, lane taking
// chunks lane, lane + 32, ... of the natural-order codes and of W_B row r (conflict-free in shared memory).
template <int NCH>
__device__ __forceinline__ int lora_row(const int8_t* wb_row, const int8_t* qn, int lane) {
  const uint4* w4 = reinterpret_cast<const uint4*>(wb_row);
  const uint4* q4 = reinterpret_cast<const uint4*>(qn);
  int t = 0;
#pragma unroll
  for (int k = 0; k < NCH / 32; ++k) {
    const uint4 w = w4[lane + 32 * k], q = q4[lane + 32 * k];
    t = dp4a_ss(w.x, q.x, t);
    t = dp4a_ss(w.y, q.y, t);
    t = dp4a_ss(w.z, q.z, t);
    t = dp4a_ss(w.w, q.w, t);
  }
  return __reduce_add_sync(0xffffffffu, t);
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
// Block-wide fp64 sum of the threads' v (every thread gets the same value: the per-warp sums are added
// in warp order).  Contains one CTA barrier.
__device__ __forceinline__ double block_sum_d(double v, int lane, int warp, double* red_d) {
  v = warp_sum(v);
  if (lane == 0) red_d[warp] = v;
  __syncthreads();
  double t = 0.0;
#pragma unroll
  for (int q = 0; q < NW; ++q) t += red_d[q];
  return t;
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

// ------------------------------------------------------------------------------ the kernel
//
// Per layer (three hand-offs):
//   A  wait h    -> RMSNorm+quantize h, LoRA-down from the partials, scaffold GEMV of the owned rows;
//                   the B/C/dt rows' accumulators are published first (arrive B/C)
//   B  wait B/C  -> epilogues (B/C conv, dt, own z gate, own x conv), SSM of the owned rows, g of the
//                   owned rows and their LoRA-down partial sums published (arrive g)
//   C  wait g    -> gated RMSNorm+quantize, out_proj GEMV of the owned rows, residual; the next layer's
//                   (arrive h)
// The first layer reads the input hidden state directly (it is complete before the launch).

__global__ void __launch_bounds__(NT, 1) decode_kernel(const __grid_constant__ Params p) {
  extern __shared__ __align__(16) int8_t wb_sm[];  // W_B of in_proj [R][DM], then of out_proj [R][E]
  // every layer's pointers, copied once: the layer loop never indexes the parameter block at run time
  __shared__ LayerPtrs lsm[DFSSM_MAX_LAYERS];
  int8_t* const wb_in = wb_sm;
  int8_t* const wb_out = wb_sm + R * DM;
  float* const st_sm = reinterpret_cast<float*>(wb_sm + WB_BYTES);  // [2][MAX_SSM][N], layer l in l & 1
  __shared__ __align__(16) int8_t q_perm[E];
  __shared__ __align__(16) int8_t q_nat[E];
  __shared__ __align__(16) double red_d[NW];   // per-warp sums of squares
  __shared__ __align__(16) unsigned red_u[NW];  // per-warp absmax (bit pattern of a non-negative float)
  __shared__ __align__(16) int red_i[NW];       // per-warp code sums
  __shared__ float lbs_o[R];                    // out_proj W_B row scales
  __shared__ int t_sm[R];
  __shared__ int sflag;
  __shared__ float tf[R];
  __shared__ float s_scale;
  // in_proj rows owned by this CTA (slot order: shared rows, z rows, x rows)
  __shared__ int acc_in[MAX_IN];
  __shared__ float in_sw[MAX_IN], in_sa[MAX_IN];
  __shared__ __align__(16) int8_t in_wa[MAX_IN][R];
  // the 320 rows every CTA needs
  __shared__ __align__(16) float sh_sw[NSH];
  __shared__ __align__(16) float sh_sa[NSH];
  __shared__ __align__(16) int8_t sh_wa[NSH][R];
  __shared__ __align__(16) float4 bc_w[2 * N];
  __shared__ __align__(16) float bc_b[2 * N];
  __shared__ __align__(16) float bc_st[2 * N][3];
  // bulk-copy completion: [0] the rows every CTA needs + in_proj W_B, [1] out_proj W_B (once per layer)
  __shared__ uint64_t ldbar[2];
  // SSM state rows of layer l arrive in buffer l & 1, one layer ahead (completes once per two layers)
  __shared__ uint64_t stbar[2];
  __shared__ float bc_new[2 * N];
  __shared__ __align__(16) float Bsm[N];
  __shared__ __align__(16) double Cd[N];
  // SSM rows
  __shared__ float zsm[MAX_SSM], xsm[MAX_SSM];
  __shared__ float dtv[2], dAv[2], Dv[2];
  // out_proj rows
  __shared__ int acc_out[MAX_OUT];
  __shared__ float o_sw[MAX_OUT], o_sa[MAX_OUT], h_old[MAX_OUT];
  __shared__ __align__(16) int8_t o_wa[MAX_OUT][R];

  const int c = blockIdx.x, NC = gridDim.x;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

  // ---- fixed ownership
  const int rs0 = (int)((long long)c * E / NC), rs1 = (int)((long long)(c + 1) * E / NC);
  const int n_ssm = rs1 - rs0;
  const int sh0 = c * NSH / NC, sh1 = (c + 1) * NSH / NC, n_sh = sh1 - sh0;
  const int ro0 = c * DM / NC, ro1 = (c + 1) * DM / NC, n_out = ro1 - ro0;
  const int n_in = n_sh + 2 * n_ssm;
  const int hA = rs0 / P;  // first head of this CTA's SSM rows (at most two heads)
  auto in_row = [&](int slot) -> int {
    if (slot < n_sh) return SH0 + sh0 + slot;
    const int j = slot - n_sh;
    return j < n_ssm ? rs0 + j : E + rs0 + (j - n_ssm);
  };
  const int li_in = lane & 15;
  const int slot_in[2] = {warp * 2 + (lane >> 4), 32 + warp * 2 + (lane >> 4)};
  const int slot_out = warp;  // out_proj: one row per warp, 32 lanes x 128 weights
  const int ssm_slot[2] = {warp, NW + warp};
  const int dt_head = tid - 2 * N;  // threads [256, 320) own the dt rows
  const bool dt_own = tid >= 2 * N && tid < NSH && (dt_head == hA || dt_head == hA + 1);

  {
    // LayerPtrs is 21 pointers: thread t copies pointer t % 21 of layer t / 21
    constexpr int NPTR = sizeof(LayerPtrs) / sizeof(void*);
    static_assert(sizeof(LayerPtrs) == NPTR * sizeof(void*), "LayerPtrs holds pointers only");
    const void* const* src = reinterpret_cast<const void* const*>(p.L);
    const void** dst = reinterpret_cast<const void**>(lsm);
    for (int k = tid; k < p.n_layers * NPTR; k += NT) dst[k] = src[k];
    if (tid == 0) {
      mbar_init(&ldbar[0], 1);
      mbar_init(&ldbar[1], 1);
      mbar_init(&stbar[0], 1);
      mbar_init(&stbar[1], 1);
      asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
      // layer 0's SSM state rows of this CTA
      mbar_expect_tx(&stbar[0], n_ssm * N * 4);
      bulk_g2s(st_sm, p.L[0].ssm_state + (size_t)rs0 * N, n_ssm * N * 4, &stbar[0]);
    }
    __syncthreads();
  }
  // An aborting CTA first waits (bounded) for everything it may still have landing in its shared memory:
  // its own cp.async copies and the bulk copies of layer l (and of layer l + 1's state rows).
  const auto drain = [&](int l, bool has_next) {
    cp_async_wait<0>();
    if (tid == 0) {
      mbar_wait(&ldbar[0], l & 1, p.spin_limit);
      mbar_wait(&ldbar[1], l & 1, p.spin_limit);
      mbar_wait(&stbar[l & 1], (l >> 1) & 1, p.spin_limit);
      if (has_next) mbar_wait(&stbar[(l + 1) & 1], ((l + 1) >> 1) & 1, p.spin_limit);
    }
  };
  for (int l = 0; l < p.n_layers; ++l) {
    const LayerPtrs& Lp = lsm[l];
    const bool has_next = l + 1 < p.n_layers;

    // ---------------------------------------------------------------- loads for the whole layer
    if ((tid == kPrefetchThread || tid == kPrefetchThread + 1) && has_next) {
      // this CTA's slice of the next layer, and (spread over CTAs 0..4) the parts every CTA reads.
      // Issued by warp 1: a bulk prefetch stalls its thread, and thread 0 polls the counters.
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
          case 0: prefetch_l2(Nx.norm_w, DM * 4); break;
          case 1: prefetch_l2(Nx.gnorm_w, E * 4); break;
          case 2:
            prefetch_lines(Nx.in_ws + SH0, NSH * 4);
            prefetch_lines(Nx.in_las + SH0, NSH * 4);
            prefetch_l2(Nx.in_la + (size_t)SH0 * R, NSH * R);
            break;
          case 3:
            prefetch_l2(Nx.conv_w + (size_t)E * 4, 2 * N * 16);
            prefetch_lines(Nx.conv_b + E, 2 * N * 4);
            prefetch_lines(Nx.conv_state + (size_t)E * 3, 2 * N * 12);
            break;
          case 4:
            prefetch_lines(Nx.dt_bias, H * 4);
            prefetch_lines(Nx.A_log, H * 4);
            prefetch_lines(Nx.D, H * 4);
            prefetch_lines(Nx.in_lbs, R * 4);
            prefetch_lines(Nx.out_lbs, R * 4);
            break;
          case 5: prefetch_l2(Nx.in_lb, R * DM); break;
          case 6: prefetch_l2(Nx.out_lb, R * E); break;
          default: break;
        }
      }
    }
    // registers: sign bits, SSM state rows, norm weights, LoRA columns of the owned rows
    uint4 w_in[2], w_out;
#pragma unroll
    for (int ps = 0; ps < 2; ++ps) {
      const int slot = slot_in[ps];
      w_in[ps] = slot < n_in ? ld_stream_u4(Lp.in_bits + (size_t)in_row(slot) * (DM / 32) + li_in * 4)
                             : make_uint4(0, 0, 0, 0);
    }
    w_out = slot_out < n_out ? ld_stream_u4(Lp.out_bits + (size_t)(ro0 + slot_out) * (E / 32) + lane * 4)
                             : make_uint4(0, 0, 0, 0);
    float nw[4], gw[8];
#pragma unroll
    for (int k = 0; k < 4; ++k) nw[k] = __ldg(Lp.norm_w + tid + k * NT);
#pragma unroll
    for (int k = 0; k < 8; ++k) gw[k] = __ldg(Lp.gnorm_w + tid + k * NT);
    float lbs_in = 0.f;
    if (tid >= kChainBase && tid < kChainBase + R) lbs_in = __ldg(Lp.in_lbs + tid - kChainBase);
    // own x channels: conv taps, bias, state (thread NSH + j handles channel rs0 + j)
    float4 cw = make_float4(0.f, 0.f, 0.f, 0.f);
    float cb = 0.f, cs0 = 0.f, cs1 = 0.f, cs2 = 0.f;
    if (tid >= NSH && tid - NSH < n_ssm) {
      const int ch = rs0 + (tid - NSH);
      cw = __ldg(reinterpret_cast<const float4*>(Lp.conv_w) + ch);
      cb = __ldg(Lp.conv_b + ch);
      cs0 = Lp.conv_state[(size_t)ch * 3 + 0];
      cs1 = Lp.conv_state[(size_t)ch * 3 + 1];
      cs2 = Lp.conv_state[(size_t)ch * 3 + 2];
    }
    float dtb = 0.f, A_h = 0.f;
    if (dt_own) {
      dtb = __ldg(Lp.dt_bias + dt_head);
      A_h = __double2float_rn(-exp((double)__ldg(Lp.A_log + dt_head)));
    }
    // epilogue parameters into shared memory, asynchronously
    if (tid < n_in) {
      const int row = in_row(tid);
      cp_async4(&in_sw[tid], Lp.in_ws + row);
      cp_async4(&in_sa[tid], Lp.in_las + row);
      cp_async16(in_wa[tid], Lp.in_la + (size_t)row * R);
    }
    if (tid == kCopyThread) {
      // the contiguous ranges every CTA needs, one bulk copy each; every generic access of the previous
      // layer to these buffers is ordered before them by the barrier that ended that layer.  Issued by a
      // thread other than the poller of the h hand-off, so that polling starts at once.
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      // first in the copy queue: the next layer's SSM state rows of this CTA (their buffer was last
      // read in layer l - 1)
      if (has_next) {
        const int nb = (l + 1) & 1;
        mbar_expect_tx(&stbar[nb], n_ssm * N * 4);
        bulk_g2s(st_sm + nb * MAX_SSM * N, lsm[l + 1].ssm_state + (size_t)rs0 * N, n_ssm * N * 4, &stbar[nb]);
      }
      mbar_expect_tx(&ldbar[0], NSH * 4 * 2 + NSH * R + 2 * N * (16 + 4 + 12) + R * DM);
      bulk_g2s(sh_sw, Lp.in_ws + SH0, NSH * 4, &ldbar[0]);
      bulk_g2s(sh_sa, Lp.in_las + SH0, NSH * 4, &ldbar[0]);
      bulk_g2s(sh_wa, Lp.in_la + (size_t)SH0 * R, NSH * R, &ldbar[0]);
      bulk_g2s(bc_w, Lp.conv_w + (size_t)E * 4, 2 * N * 16, &ldbar[0]);
      bulk_g2s(bc_b, Lp.conv_b + E, 2 * N * 4, &ldbar[0]);
      bulk_g2s(bc_st, Lp.conv_state + (size_t)E * 3, 2 * N * 12, &ldbar[0]);
      bulk_g2s(wb_in, Lp.in_lb, R * DM, &ldbar[0]);
      mbar_expect_tx(&ldbar[1], R * E);
      bulk_g2s(wb_out, Lp.out_lb, R * E, &ldbar[1]);
    }
    if (tid < n_out) {
      const int row = ro0 + tid;
      cp_async4(&o_sw[tid], Lp.out_ws + row);
      cp_async4(&o_sa[tid], Lp.out_las + row);
      cp_async16(o_wa[tid], Lp.out_la + (size_t)row * R);
    }
    if (tid < 2 && hA + tid < H) cp_async4(&Dv[tid], Lp.D + hA + tid);
    if (tid < R) cp_async4(&lbs_o[tid], Lp.out_lbs + tid);
    cp_async_commit();  // this thread's row parameters (awaited after the h wait)

    // ---------------------------------------------------------------- phase A: h -> in_proj
    if (l > 0 && !block_wait(p.ctr + CTR_H * CTR_STRIDE, NC * l, p.err, p.status, p.spin_limit, &sflag)) {
      drain(l, has_next);
      return;
    }
    cp_async_wait<0>();  // this thread's row parameters; the quantizer's barriers publish them
    if (!mbar_wait(&ldbar[0], l & 1, p.spin_limit)) {  // shared rows and in_proj W_B
      atomicExch(p.err, 1);
      atomicExch(p.status, kTimeoutMagic);
      drain(l, has_next);
      return;
    }
    // RMSNorm, then the quantizer on the normalized row: r from the block sum of squares, then the
    // absmax of u = fl32(fl32(h r) w)
    float s0A;
    {
      float hv[4], v[4];
      double ss = 0.0;
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        hv[k] = __ldcg(p.hidden + tid + k * NT);
        ss += (double)hv[k] * (double)hv[k];
      }
      if (tid < n_out) h_old[tid] = __ldcg(p.hidden + ro0 + tid);
      const float rn = rms_factor(block_sum_d(ss, lane, warp, red_d), DM);
      float m = 0.0f;
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        v[k] = norm_value(hv[k], rn, nw[k]);
        m = fmaxf(m, fabsf(v[k]));
      }
      m = block_absmax(m, lane, warp, red_u);
      const float s0 = m == 0.0f ? 0.0f : __fdiv_rn(m, 127.0f);
      const float inv_s0 = m == 0.0f ? 0.0f : __frcp_rn(s0);
      int sq = 0;
      int cd[4];
      quant_codes<4>(v, s0, inv_s0, cd);
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        q_perm[seg_index<DM / 128>(tid + k * NT)] = (int8_t)cd[k];
        q_nat[tid + k * NT] = (int8_t)cd[k];
        sq += cd[k];
      }
      sq = __reduce_add_sync(0xffffffffu, sq);
      if (lane == 0) red_i[warp] = sq;
      __syncthreads();
      s0A = s0;
    }
    const int sumq = block_sum16(red_i);
    // scaffold GEMV over the owned rows; pass 0 holds the rows every CTA needs
    {
      const uint4* qp4 = reinterpret_cast<const uint4*>(q_perm) + li_in;
#pragma unroll
      for (int ps = 0; ps < 2; ++ps) {
        int S = bits_dot<DM / 128>(w_in[ps], qp4);
#pragma unroll
        for (int o = 8; o > 0; o >>= 1) S += __shfl_xor_sync(0xffffffffu, S, o);
        if (li_in == 0 && slot_in[ps] < n_in) {
          acc_in[slot_in[ps]] = 2 * S - sumq;
          if (ps == 0 && slot_in[0] < n_sh) p.sacc[sh0 + slot_in[0]] = 2 * S - sumq;
        }
        if (ps == 0) {
          block_arrive(p.ctr + CTR_BC * CTR_STRIDE);  // its barrier orders the accumulators above
          // LoRA down of the codes: warp r computes t[r]
          const int t = lora_row<DM / 16>(wb_in + warp * DM, q_nat, lane);
          if (lane == 0) t_sm[warp] = t;
        }
      }
    }
    // the LoRA intermediate (off the GEMV's critical path: the epilogue needs it only after the B/C wait)
    __syncthreads();
    if (tid >= kChainBase && tid < kChainBase + R) tf[tid - kChainBase] = lora_tf(t_sm[tid - kChainBase], lbs_in, s0A);
    if (tid == kChainBase + R) s_scale = s0A;

    // ---------------------------------------------------------------- phase B: epilogues + SSM
    if (!block_wait(p.ctr + CTR_BC * CTR_STRIDE, NC * (l + 1), p.err, p.status, p.spin_limit, &sflag)) {
      drain(l, has_next);
      return;
    }
    const float s_in = s_scale;
    if (tid < NSH) {
      // rows every CTA needs: B, C (conv + SiLU) and dt of this CTA's heads
      const float y = linear_out(__ldcg(p.sacc + tid), s_in, sh_sw[tid], sh_sa[tid], sh_wa[tid], tf, R);
      if (tid < 2 * N) {
        bc_new[tid] = y;
        const float xc = conv_out(bc_w[tid], bc_b[tid], bc_st[tid][0], bc_st[tid][1], bc_st[tid][2], y);
        if (tid < N) Bsm[tid] = xc;
        else Cd[tid - N] = (double)xc;
      } else if (dt_own) {
        const float dt = ssm_dt(y, dtb);
        dtv[dt_head - hA] = dt;
        dAv[dt_head - hA] = __double2float_rn(exp((double)fmul(dt, A_h)));
      }
    } else if (tid - NSH < n_ssm) {
      // the owned z rows (gate value SiLU(z) kept) and x rows (conv of the owned x channels)
      const int j = tid - NSH;
      const int sz = n_sh + j, sx = n_sh + n_ssm + j;
      zsm[j] = silu_f64(linear_out(acc_in[sz], s_in, in_sw[sz], in_sa[sz], in_wa[sz], tf, R));
      const float xr = linear_out(acc_in[sx], s_in, in_sw[sx], in_sa[sx], in_wa[sx], tf, R);
      xsm[j] = conv_out(cw, cb, cs0, cs1, cs2, xr);
      float* st = Lp.conv_state + (size_t)(rs0 + j) * 3;
      st[0] = cs1;
      st[1] = cs2;
      st[2] = xr;
    }
    __syncthreads();
    if (!mbar_wait(&stbar[l & 1], (l >> 1) & 1, p.spin_limit)) {  // this layer's SSM state rows
      atomicExch(p.err, 1);
      atomicExch(p.status, kTimeoutMagic);
      drain(l, has_next);
      return;
    }
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
          const float g = fmul(y, zsm[rr]);
          p.gbuf[hp] = g;
        }
      }
    }
    block_arrive(p.ctr + CTR_G * CTR_STRIDE);
#pragma unroll
    for (int ps = 0; ps < 2; ++ps)
      if (ssm_slot[ps] < n_ssm) st_f4(Lp.ssm_state + (size_t)(rs0 + ssm_slot[ps]) * N + lane * 4, snew[ps]);

    // ---------------------------------------------------------------- phase C: gated norm -> out_proj
    if (!block_wait(p.ctr + CTR_G * CTR_STRIDE, NC * (l + 1), p.err, p.status, p.spin_limit, &sflag)) {
      drain(l, has_next);
      return;
    }
    if (!mbar_wait(&ldbar[1], l & 1, p.spin_limit)) {  // out_proj W_B
      atomicExch(p.err, 1);
      atomicExch(p.status, kTimeoutMagic);
      drain(l, has_next);
      return;
    }
    // every CTA has now read the old B/C conv state: the owners of those rows shift it
    for (int j = tid; j < n_sh; j += NT) {
      const int k = sh0 + j;
      if (k < 2 * N) {
        float* st = Lp.conv_state + (size_t)(E + k) * 3;
        st[0] = bc_st[k][1];
        st[1] = bc_st[k][2];
        st[2] = bc_new[k];
      }
    }
    {
      float gv[8], v[8];
      double ss = 0.0;
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        gv[k] = __ldcg(p.gbuf + tid + k * NT);
        ss += (double)gv[k] * (double)gv[k];
      }
      const float rn = rms_factor(block_sum_d(ss, lane, warp, red_d), E);
      float m = 0.0f;
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        v[k] = norm_value(gv[k], rn, gw[k]);
        m = fmaxf(m, fabsf(v[k]));
      }
      m = block_absmax(m, lane, warp, red_u);
      const float s0 = m == 0.0f ? 0.0f : __fdiv_rn(m, 127.0f);
      const float inv_s0 = m == 0.0f ? 0.0f : __frcp_rn(s0);
      int sq = 0;
      int cd[8];
      quant_codes<8>(v, s0, inv_s0, cd);
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        q_perm[seg_index<E / 128>(tid + k * NT)] = (int8_t)cd[k];
        q_nat[tid + k * NT] = (int8_t)cd[k];
        sq += cd[k];
      }
      sq = __reduce_add_sync(0xffffffffu, sq);
      if (lane == 0) red_i[warp] = sq;
      if (tid == 0) s_scale = s0;
      __syncthreads();
      // LoRA down of the codes (warp r: t[r]); every warp with an out_proj row then takes it
      const int t = lora_row<E / 16>(wb_out + warp * E, q_nat, lane);
      if (lane == 0) t_sm[warp] = t;
      if (warp != kChainWarp) {
        const int sumq_c = block_sum16(red_i);
        const uint4* qp4 = reinterpret_cast<const uint4*>(q_perm) + lane;
        int S = bits_dot<E / 128>(w_out, qp4);
        S = warp_sum(S);
        if (lane == 0 && slot_out < n_out) acc_out[slot_out] = 2 * S - sumq_c;
      }
    }
    __syncthreads();
    if (tid < n_out) {
      // each epilogue thread forms the sixteen LoRA intermediates itself (no further barrier)
      double tfd[R];
#pragma unroll
      for (int r = 0; r < R; ++r) tfd[r] = (double)lora_tf(t_sm[r], lbs_o[r], s_scale);
      const float y = linear_out_d(acc_out[tid], (double)s_scale, (double)o_sw[tid], (double)o_sa[tid],
                                   *reinterpret_cast<const uint4*>(o_wa[tid]), tfd, R);
      p.hidden[ro0 + tid] = fadd(h_old[tid], y);
    }
    block_arrive(p.ctr + CTR_H * CTR_STRIDE);
  }
}

// Waits on a counter that nothing increments, with a short budget: exercises the timeout path.
__global__ void timeout_selftest_kernel(int* ctr, int* err, int* status, long long limit) {
  __shared__ int sflag;
  block_wait(ctr, 1, err, status, limit, &sflag);
}

}  // namespace fused

size_t fused_decode_workspace_bytes() { return fused::WS_BYTES; }

bool fused_decode_supported(const dfssm_dims_t& d, int B, const dfssm_layer_t* layers, int n,
                            float* const* conv_states) {
  if (B != 1 || d.d_model != fused::DM || d.nheads != fused::H || d.headdim != fused::P ||
      d.d_state != fused::N || d.ngroups != 1)
    return false;
  // the ranges fetched by bulk copy must start on 16-byte boundaries
  const auto a16 = [](const void* q) { return (reinterpret_cast<uintptr_t>(q) & 15) == 0; };
  for (int l = 0; l < n; ++l) {
    const dfssm_layer_t& L = layers[l];
    if (L.in_proj.rank != fused::R || L.out_proj.rank != fused::R) return false;
    if (!a16(L.in_proj.w_scale) || !a16(L.in_proj.lora_a_scale) || !a16(L.in_proj.lora_a) ||
        !a16(L.in_proj.lora_b) || !a16(L.out_proj.lora_b) || !a16(L.conv_w) || !a16(L.conv_b) ||
        !a16(conv_states[l]))
      return false;
  }
  const int nc = num_sms();
  // ownership limits: in_proj rows per CTA <= 64, out_proj rows <= 16, SSM rows <= 32; partial-sum
  // buffers sized for MAX_CTAS
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
  p.ctr = reinterpret_cast<int*>(base + fused::OFF_CTR);
  p.err = reinterpret_cast<int*>(base + fused::OFF_ERR);
  p.status = reinterpret_cast<int*>(base + fused::OFF_STATUS);
  p.sacc = reinterpret_cast<int*>(base + fused::OFF_SACC);
  p.gbuf = reinterpret_cast<float*>(base + fused::OFF_GBUF);
  p.spin_limit = spin_limit;
  cudaError_t e = cudaMemsetAsync(p.ctr, 0, fused::CLEAR_BYTES, st);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(num_sms());
  cfg.blockDim = dim3(fused::NT);
  // set once (not per launch, so that launches can be captured in a CUDA graph)
  static const cudaError_t attr_set = cudaFuncSetAttribute(
      fused::decode_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, fused::DYN_BYTES);
  if (attr_set != cudaSuccess) return attr_set;
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
  int* ctr = reinterpret_cast<int*>(base + fused::OFF_CTR);
  int* err = reinterpret_cast<int*>(base + fused::OFF_ERR);
  int* status = reinterpret_cast<int*>(base + fused::OFF_STATUS);
  cudaError_t e = cudaMemsetAsync(ctr, 0, fused::CLEAR_BYTES, st);
  if (e != cudaSuccess) return e;
  fused::timeout_selftest_kernel<<<1, 32, 0, st>>>(ctr, err, status, spin_limit);
  return cudaGetLastError();
}

int read_device_error(void* ws, cudaStream_t st, int* code) {
  char* base = static_cast<char*>(ws);
  int* status = reinterpret_cast<int*>(base + fused::OFF_STATUS);
  int h = 0;
  cudaError_t e = cudaMemcpyAsync(&h, status, sizeof(int), cudaMemcpyDeviceToHost, st);
  if (e == cudaSuccess) e = cudaStreamSynchronize(st);
  if (e == cudaSuccess) e = cudaMemsetAsync(status, 0, sizeof(int), st);
  if (e == cudaSuccess) e = cudaStreamSynchronize(st);
  *code = (h == fused::kTimeoutMagic) ? 1 : 0;
  return e == cudaSuccess ? 0 : (int)e;
}

}  // namespace dfssm
