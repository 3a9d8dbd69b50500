// M-token prefill of one DF-SSM linear on the 5th-generation (tcgen05) int8 tensor cores
// (gist.science technical summary of DF-SSM, §2.C: "1-bit packed weights are expanded on-the-fly to int8
// and processed via ... INT8 tensor cores").  At M = 2048 tokens the scaffold matmul is a dense
// contraction, so it runs as an int8 GEMM with int32 accumulation in tensor memory:
//   1. quantize every token (per-token absmax int8 codes, natural order, exactly as in decode) and its
//      LoRA down-projection (fp32, one warp per token);
//   2. expand the packed sign bits once to +-1 int8 rows in the workspace;
//   3. acc[m][n] = sum_k q[m][k] w[n][k] on tcgen05.mma kind::i8 (128x128 tiles, K steps of 128 bytes,
//      TMA loads with 128-byte swizzle into a 4-stage shared-memory ring, a persistent kernel); the
//      epilogue reads the accumulator from tensor memory while the next tile accumulates and forms
//      y[m][n] = fl32(acc s[m] sW[n] + sA[n] sum_r W_A[n][r] tf[m][r]) in fp64 with the decode path's
//      rounding sequence (the rank-16 LoRA-up is 16 multiply-adds per output, far below the scaffold's K).
// The integer accumulators are exact and every output equals the decode definition bit for bit.
//
// Every wait on an mbarrier is bounded: a wait that runs out of budget sets the workspace error word,
// the CTA stops issuing work, waits (bounded) for its copies in flight, frees its tensor memory and
// returns.

#include <cuda.h>
#include <cudaTypedefs.h>

#include <cstdio>
#include <mutex>

#include "common.cuh"
#include "internal.h"

namespace dfssm {
namespace prefill {

constexpr int BM = 128, BN = 128, BK = 128;  // tile; BK bytes = BK int8 elements
constexpr int STAGES = 4;
constexpr int UMMA_K = 32;                   // K of one kind::i8 MMA (bytes)
constexpr int A_BYTES = BM * BK, B_BYTES = BN * BK, STAGE_BYTES = A_BYTES + B_BYTES;
constexpr long long kWaitBudget = 4000000000LL;  // clock cycles per wait (~2 s)

struct EpiArgs {
  const float* s;       // [M] per-token scale
  const float* w_scale; // [N]
  const float* la_scale;// [N]
  int rank;
  float* y;             // [M][N]
  int32_t* acc;         // [M][N] or null
  const float* tf;      // [M][16] LoRA intermediates (zero beyond the rank)
  const int8_t* lora_a; // [N][rank]
  int M, N, K;
  int* err;
  int resid;            // 1: y[m][n] = fl32(y[m][n] + out) (residual add in place), 0: y = out
};

// ------------------------------------------------------------------------------ PTX helpers

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return (uint32_t)__cvta_generic_to_shared(p);
}
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
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}
// Bounded wait for the given phase parity; false when the budget ran out or another role aborted.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, volatile int* abort_flag) {
  const long long t0 = clock64();
  while (!mbar_try_wait(bar, parity)) {
    if (*abort_flag) return false;
    if (clock64() - t0 > kWaitBudget) return false;
  }
  return true;
}
__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, int c0, int c1,
                                            uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], "
      "[%4];" ::"r"(smem_u32(dst)),
      "l"(map), "r"(c0), "r"(c1), "r"(smem_u32(bar))
      : "memory");
}

// K-major operand in 128-byte-swizzled rows of 128 bytes: 8-row groups 1024 bytes apart.
__device__ __forceinline__ uint64_t umma_desc_k_sw128(uint32_t smem_addr) {
  uint64_t d = 0;
  d |= (uint64_t)((smem_addr >> 4) & 0x3FFFu);  // start address (16-byte units)
  d |= (uint64_t)1 << 16;                        // leading byte offset (unused with swizzle)
  d |= (uint64_t)(1024 >> 4) << 32;              // stride byte offset: next 8-row group
  d |= (uint64_t)1 << 46;                        // descriptor version for sm_100
  d |= (uint64_t)2 << 61;                        // 128-byte swizzle
  return d;
}
// kind::i8 instruction descriptor: D s32, A s8, B s8, both K-major, M = BM, N = BN.
constexpr uint32_t kIdesc = (2u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(BN >> 3) << 17) |
                            ((uint32_t)(BM >> 4) << 24);

__device__ __forceinline__ void umma_i8(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc, uint32_t accum) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::i8 [%0], %1, %2, %3, p;\n\t}" ::"r"(tmem_d),
      "l"(adesc), "l"(bdesc), "r"(kIdesc), "r"(accum)
      : "memory");
}
__device__ __forceinline__ void umma_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   smem_u32(bar))
               : "memory");
}
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, "
      "[%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]),
        "=r"(r[15])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// ------------------------------------------------------------------------------ kernels

// w8[n][k] = +1 for a set sign bit, -1 otherwise.  One thread per 32-bit word (32 weights).
__global__ void expand_bits_kernel(const uint32_t* __restrict__ bits, int8_t* __restrict__ w8,
                                   long long words) {
  const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= words) return;
  const uint32_t w = bits[i];
  uint32_t out[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const uint32_t nib = (w >> (4 * j)) & 0xFu;
    uint32_t v = 0;
#pragma unroll
    for (int b = 0; b < 4; ++b) v |= (((nib >> b) & 1u) ? 0x01u : 0xFFu) << (8 * b);
    out[j] = v;
  }
  uint4* dst = reinterpret_cast<uint4*>(w8 + i * 32);
  dst[0] = make_uint4(out[0], out[1], out[2], out[3]);
  dst[1] = make_uint4(out[4], out[5], out[6], out[7]);
}

// Quantization for the prefill: one warp per token.  Codes (natural order) and scale exactly as the
// decode quantizer; the LoRA down-projection t = W_B q on the codes (int32, dp4a) with W_B staged in
// shared memory (zero rows beyond the rank, so every lane runs all sixteen rows without branches), and
// tf = fl32(t sB s) rounded as in the decode path.  Each lane keeps eight 16-byte loads of its token in
// flight.  With a norm weight (a layer's pre-norm or gated norm) the token is first normalized as in
// decode: r = fl32(1/sqrt(sum x^2 / K + 1e-5)) (fp64) and v = fl32(fl32(x r) w) is quantized.
constexpr int QW = 8;  // tokens (warps) per CTA
constexpr int QU = 8;  // float4 loads in flight per lane
__global__ void __launch_bounds__(QW * 32) prefill_quant_kernel(const float* __restrict__ x, int M, int K,
                                                               const int8_t* __restrict__ lora_b,
                                                               const float* __restrict__ lora_b_scale,
                                                               int rank, const float* __restrict__ norm_w,
                                                               int8_t* __restrict__ xq,
                                                               float* __restrict__ s_out,
                                                               float* __restrict__ tf_out,
                                                               int8_t* dbg_xq, float* dbg_s, int32_t* dbg_t) {
  extern __shared__ __align__(16) unsigned char sm[];
  int8_t* wb = reinterpret_cast<int8_t*>(sm);  // [16][K]
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // W_B into shared memory: 16-byte loads when W_B is 16-byte aligned (rank K is a multiple of 16),
  // else eight 4-byte loads in flight per thread
  if ((reinterpret_cast<uintptr_t>(lora_b) & 15) == 0) {
    for (int i0 = threadIdx.x * 16; i0 < DFSSM_MAX_RANK * K; i0 += 8 * QW * 32 * 16) {
      uint4 w[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int i = i0 + u * QW * 32 * 16;
        w[u] = i < rank * K ? __ldg(reinterpret_cast<const uint4*>(lora_b + i)) : make_uint4(0u, 0u, 0u, 0u);
      }
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int i = i0 + u * QW * 32 * 16;
        if (i < DFSSM_MAX_RANK * K) *reinterpret_cast<uint4*>(wb + i) = w[u];
      }
    }
  } else
  for (int i0 = threadIdx.x * 4; i0 < DFSSM_MAX_RANK * K; i0 += 8 * QW * 32 * 4) {
    uint32_t w[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int i = i0 + u * QW * 32 * 4;
      w[u] = i < rank * K ? __ldg(reinterpret_cast<const uint32_t*>(lora_b + i)) : 0u;
    }
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int i = i0 + u * QW * 32 * 4;
      if (i < DFSSM_MAX_RANK * K) *reinterpret_cast<uint32_t*>(wb + i) = w[u];
    }
  }
  __syncthreads();
  const int m = blockIdx.x * QW + warp;
  if (m >= M) return;
  const float4* xr = reinterpret_cast<const float4*>(x + (size_t)m * K);
  const float4* wr = reinterpret_cast<const float4*>(norm_w);
  const int K4 = K / 4;  // a multiple of 32: the bounds tests below are uniform over the warp
  constexpr int UB = QU;  // float4 per lane per batch
  // RMSNorm factor (with a norm weight): a first pass for the sum of squares (exact squares in fp64)
  float rn = 1.0f;
  if (wr) {
    double ss = 0.0;
    for (int i0 = lane; i0 < K4; i0 += 32 * UB) {
      float4 v[UB];
#pragma unroll
      for (int u = 0; u < UB; ++u)
        v[u] = i0 + 32 * u < K4 ? __ldg(xr + i0 + 32 * u) : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
      for (int u = 0; u < UB; ++u) {
        ss = fma((double)v[u].x, (double)v[u].x, ss);
        ss = fma((double)v[u].y, (double)v[u].y, ss);
        ss = fma((double)v[u].z, (double)v[u].z, ss);
        ss = fma((double)v[u].w, (double)v[u].w, ss);
      }
    }
    rn = rms_factor(warp_sum(ss), K);
  }
  // v = fl32(fl32(x r) w) with a norm weight, else x
  const auto scale4 = [&](float4 a, int i) {
    if (!wr) return a;
    const float4 w = __ldg(wr + i);
    return make_float4(norm_value(a.x, rn, w.x), norm_value(a.y, rn, w.y), norm_value(a.z, rn, w.z),
                       norm_value(a.w, rn, w.w));
  };
  float m_abs = 0.0f;
  for (int i0 = lane; i0 < K4; i0 += 32 * UB) {
    float4 v[UB];
#pragma unroll
    for (int u = 0; u < UB; ++u)
      v[u] = i0 + 32 * u < K4 ? __ldg(xr + i0 + 32 * u) : make_float4(0.f, 0.f, 0.f, 0.f);
    if (wr) {
#pragma unroll
      for (int u = 0; u < UB; ++u)
        if (i0 + 32 * u < K4) v[u] = scale4(v[u], i0 + 32 * u);
    }
#pragma unroll
    for (int u = 0; u < UB; ++u)
      m_abs = fmaxf(m_abs, fmaxf(fmaxf(fabsf(v[u].x), fabsf(v[u].y)), fmaxf(fabsf(v[u].z), fabsf(v[u].w))));
  }
  m_abs = warp_max(m_abs);
  const float s0 = quant_scale(m_abs);
  const float inv_s0 = quant_inv(s0);
  const float s_tok = s0;
  int u[DFSSM_MAX_RANK];
#pragma unroll
  for (int r = 0; r < DFSSM_MAX_RANK; ++r) u[r] = 0;
  for (int i0 = lane; i0 < K4; i0 += 32 * UB) {
    float4 v[UB];
#pragma unroll
    for (int q = 0; q < UB; ++q)
      v[q] = i0 + 32 * q < K4 ? __ldg(xr + i0 + 32 * q) : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int q = 0; q < UB; ++q) {
      const int i = i0 + 32 * q;
      if (i < K4) {
        const float4 vs = scale4(v[q], i);
        const float vv[4] = {vs.x, vs.y, vs.z, vs.w};
        int cd[4];
        quant_codes<4>(vv, s0, inv_s0, cd);
        uint32_t packed = 0;
#pragma unroll
        for (int j = 0; j < 4; ++j) packed |= ((uint32_t)cd[j] & 0xFFu) << (8 * j);
        reinterpret_cast<uint32_t*>(xq + (size_t)m * K)[i] = packed;
        if (dbg_xq) reinterpret_cast<uint32_t*>(dbg_xq + (size_t)m * K)[i] = packed;
#pragma unroll
        for (int r = 0; r < DFSSM_MAX_RANK; ++r)
          u[r] = dp4a_ss(reinterpret_cast<const uint32_t*>(wb + (size_t)r * K)[i], packed, u[r]);
      }
    }
  }
#pragma unroll
  for (int r = 0; r < DFSSM_MAX_RANK; ++r) u[r] = __reduce_add_sync(0xffffffffu, u[r]);
  float tf = 0.0f;
  if (lane < DFSSM_MAX_RANK) {
    int tv = 0;
#pragma unroll
    for (int r = 0; r < DFSSM_MAX_RANK; ++r)
      if (r == lane) tv = u[r];
    tf = lane < rank ? lora_tf(tv, __ldg(lora_b_scale + lane), s_tok) : 0.0f;
    tf_out[(size_t)m * DFSSM_MAX_RANK + lane] = tf;
    if (dbg_t && lane < rank) dbg_t[(size_t)m * rank + lane] = tv;
  }
  if (lane == 0) {
    s_out[m] = s_tok;
    if (dbg_s) dbg_s[m] = s_tok;
  }
}

// Persistent tcgen05 GEMM: one CTA per SM walks the 128 x 128 output tiles; warp 0 streams A/B stages
// with TMA, warp 1 issues the int8 MMAs into one of two int32 accumulators, warps 2..9 drain the other
// one (two warps per 32-lane TMEM quadrant, each taking half of the 128 columns) and evaluate the fp64
// epilogue, so a tile's epilogue overlaps the next tile's main loop.  TMEM columns: [0, 256).
constexpr int EPI_WARPS = 8;
constexpr int PNT = 64 + EPI_WARPS * 32;   // 320 threads
constexpr int PTMEM_COLS = 2 * BN;         // two int32 accumulators of BN columns
constexpr int STG_LD = 17;                 // staging row stride (floats): conflict-free both ways
constexpr size_t OFF_BARS = (size_t)STAGES * STAGE_BYTES;
constexpr size_t OFF_COLS = OFF_BARS + 512;
constexpr size_t OFF_WA = OFF_COLS + 2 * BN * 16;  // [2][BN][16] W_A rows as fp64 (zero beyond the rank)
constexpr size_t OFF_STG = OFF_WA + 2 * BN * DFSSM_MAX_RANK * 8;
constexpr size_t PSMEM_BYTES = 1024 + OFF_STG + EPI_WARPS * 32 * STG_LD * 4;

// Bounded wait that ignores the abort flag (used to drain work already issued).
__device__ __forceinline__ void mbar_wait_drain(uint64_t* bar, uint32_t parity) {
  const long long t0 = clock64();
  while (!mbar_try_wait(bar, parity))
    if (clock64() - t0 > kWaitBudget) return;
}

__global__ void __launch_bounds__(PNT, 1)
    gemm_kernel(const __grid_constant__ CUtensorMap map_a, const __grid_constant__ CUtensorMap map_b,
                const EpiArgs ep) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  // aligned by an offset from the array itself, so that every access stays a shared-memory access
  unsigned char* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + OFF_BARS);
  uint64_t* empty = full + STAGES;
  uint64_t* acc_full = empty + STAGES;     // [2] MMA -> epilogue
  uint64_t* acc_empty = acc_full + 2;      // [2] epilogue -> MMA
  uint64_t* mma_done = acc_empty + 2;      // every MMA of this CTA complete
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(mma_done + 1);
  // per-accumulator column parameters of the tile being drained: sW, sA (fp64 images), W_A row
  double* col_sw = reinterpret_cast<double*>(smem + OFF_COLS);  // [2][BN]
  double* col_sa = col_sw + 2 * BN;                             // [2][BN]
  double* col_wa = reinterpret_cast<double*>(smem + OFF_WA);  // [2][BN][16]
  float* stg_all = reinterpret_cast<float*>(smem + OFF_STG);  // [EPI_WARPS][32][STG_LD]
  __shared__ int abort_flag;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int tiles_n = (ep.N + BN - 1) / BN, tiles_m = (ep.M + BM - 1) / BM;
  const int tiles = tiles_n * tiles_m;
  const int kblocks = ep.K / BK;

  if (threadIdx.x == 0) {
    abort_flag = 0;
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], EPI_WARPS);
    }
    mbar_init(mma_done, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(tmem_holder)),
                 "r"(PTMEM_COLS)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
  __syncthreads();
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
  const uint32_t tmem_base = *tmem_holder;

  if (warp == 0 && lane == 0) {
    // ---- TMA producer: each tile's k-blocks through the stage ring
    int it = 0;
    bool ok = true;
    for (int t = blockIdx.x; t < tiles && ok; t += gridDim.x) {
      const int n0 = (t % tiles_n) * BN, m0 = (t / tiles_n) * BM;
      for (int kb = 0; kb < kblocks; ++kb, ++it) {
        const int s = it % STAGES;
        if (it >= STAGES && !mbar_wait(&empty[s], ((it / STAGES) - 1) & 1, &abort_flag)) {
          abort_flag = 1;
          ok = false;
          break;
        }
        unsigned char* a_dst = smem + s * STAGE_BYTES;
        mbar_expect_tx(&full[s], STAGE_BYTES);
        tma_load_2d(a_dst, &map_a, kb * BK, m0, &full[s]);
        tma_load_2d(a_dst + A_BYTES, &map_b, kb * BK, n0, &full[s]);
      }
    }
    // the last copies land before this CTA may exit
    for (int j = (it > STAGES ? it - STAGES : 0); j < it; ++j) mbar_wait_drain(&full[j % STAGES], (j / STAGES) & 1);
  } else if (warp == 1 && lane == 0) {
    // ---- MMA issuer
    int it = 0, local = 0;
    bool ok = true, issued = false;
    for (int t = blockIdx.x; t < tiles && ok; t += gridDim.x, ++local) {
      const int buf = local & 1;
      if (local >= 2 && !mbar_wait(&acc_empty[buf], ((local >> 1) - 1) & 1, &abort_flag)) {
        abort_flag = 1;
        break;
      }
      asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
      const uint32_t d_tmem = tmem_base + (uint32_t)(buf * BN);
      for (int kb = 0; kb < kblocks; ++kb, ++it) {
        const int s = it % STAGES;
        if (!mbar_wait(&full[s], (it / STAGES) & 1, &abort_flag)) {
          abort_flag = 1;
          ok = false;
          break;
        }
        asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
        const uint32_t a_addr = smem_u32(smem + s * STAGE_BYTES);
        const uint32_t b_addr = a_addr + A_BYTES;
#pragma unroll
        for (int kk = 0; kk < BK / UMMA_K; ++kk)
          umma_i8(d_tmem, umma_desc_k_sw128(a_addr + kk * UMMA_K), umma_desc_k_sw128(b_addr + kk * UMMA_K),
                  (kb > 0 || kk > 0) ? 1u : 0u);
        umma_commit(&empty[s]);
        issued = true;
      }
      if (!ok) break;
      umma_commit(&acc_full[buf]);
    }
    // every MMA this thread issued completes before the tensor memory is released
    if (issued) {
      umma_commit(mma_done);
      mbar_wait_drain(mma_done, 0);
    }
  } else if (warp >= 2) {
    // ---- epilogue: warp e = warp - 2 drains TMEM lanes [32 (warp % 4), +32) and column half e / 4
    const int e = warp - 2;
    const int q = warp & 3;
    const int half = e >> 2;
    const int etid = threadIdx.x - 64;  // 0..255
    float* stg = stg_all + (size_t)e * 32 * STG_LD;
    int local = 0;
    for (int t = blockIdx.x; t < tiles; t += gridDim.x, ++local) {
      const int buf = local & 1;
      const int n0 = (t % tiles_n) * BN, m0 = (t / tiles_n) * BM;
      // column parameters of this tile, staged once per tile: sW, sA and the W_A row (zero beyond the
      // rank)
      if (etid < BN) {
        const int n = n0 + etid;
        col_sw[buf * BN + etid] = n < ep.N ? (double)__ldg(ep.w_scale + n) : 0.0;
        col_sa[buf * BN + etid] = (n < ep.N && ep.rank > 0) ? (double)__ldg(ep.la_scale + n) : 0.0;
        double* wd = col_wa + (size_t)(buf * BN + etid) * DFSSM_MAX_RANK;
#pragma unroll
        for (int r = 0; r < DFSSM_MAX_RANK; ++r)
          wd[r] = (n < ep.N && r < ep.rank) ? (double)ep.lora_a[(size_t)n * ep.rank + r] : 0.0;
      }
      asm volatile("bar.sync 1, %0;" ::"n"(EPI_WARPS * 32) : "memory");
      const int row = q * 32 + lane;
      const int m = m0 + row;
      const double sm = m < ep.M ? (double)__ldg(ep.s + m) : 0.0;
      // this row's LoRA intermediates in fp64 (exact images of the fp32 values)
      double tfd[DFSSM_MAX_RANK];
#pragma unroll
      for (int r = 0; r < DFSSM_MAX_RANK; ++r)
        tfd[r] = (m < ep.M && r < ep.rank) ? (double)__ldg(ep.tf + (size_t)m * DFSSM_MAX_RANK + r) : 0.0;
      // every epilogue warp runs every tile iteration (the named barrier above counts on it); after an
      // abort the accumulators are simply not read
      const bool ok = !abort_flag && mbar_wait(&acc_full[buf], (local >> 1) & 1, &abort_flag);
      asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
      if (!ok) {
        abort_flag = 1;
        if (lane == 0) atomicExch(ep.err, 1);
      }
      for (int cc = 0; ok && cc < BN / 2; cc += 16) {
        const int c0 = half * (BN / 2) + cc;
        uint32_t v[16];
        tmem_ld16(tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(buf * BN + c0), v);
        float out[16];
        // y = fl32(acc s sW + sA sum_r W_A tf), fp64, the decode path's rounding sequence (linear_out_n):
        // the LoRA sum runs over r = 0..15 in order; fma(w, tf, lora) equals lora + w tf rounded once
        // because the product of an int8 and an fp32 value is exact in fp64, and the zero weights beyond
        // the rank leave the sum unchanged (it is never -0).
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          const int cidx = buf * BN + c0 + j;
          const double2* w2 = reinterpret_cast<const double2*>(col_wa + (size_t)cidx * DFSSM_MAX_RANK);
          double lora = 0.0;
#pragma unroll
          for (int r2 = 0; r2 < DFSSM_MAX_RANK / 2; ++r2) {
            const double2 w = w2[r2];
            lora = fma(w.x, tfd[2 * r2], lora);
            lora = fma(w.y, tfd[2 * r2 + 1], lora);
          }
          const double scaffold = dmul(dmul(int_to_f64((int)v[j]), sm), col_sw[cidx]);
          const double corr = ep.rank > 0 ? dmul(col_sa[cidx], lora) : 0.0;
          out[j] = __double2float_rn(dadd(scaffold, corr));
        }
        if (ep.acc && m < ep.M) {
#pragma unroll
          for (int j = 0; j < 16; ++j)
            if (n0 + c0 + j < ep.N) ep.acc[(size_t)m * ep.N + n0 + c0 + j] = (int)v[j];
        }
        // through shared memory: lane l holds row l of the chunk; the stores then write two 64-byte row
        // segments per instruction (lanes 0-15 one row, 16-31 the next)
#pragma unroll
        for (int j = 0; j < 16; ++j) stg[lane * STG_LD + j] = out[j];
        __syncwarp();
        const int cj = lane & 15, n = n0 + c0 + cj;
#pragma unroll 4
        for (int k = 0; k < 16; ++k) {
          const int r = 2 * k + (lane >> 4);
          const int mr = m0 + q * 32 + r;
          if (mr < ep.M && n < ep.N) {
            float* dst = ep.y + (size_t)mr * ep.N + n;
            *dst = ep.resid ? fadd(*dst, stg[r * STG_LD + cj]) : stg[r * STG_LD + cj];
          }
        }
        __syncwarp();
      }
      // this warp's reads of the accumulators are complete: release them to the MMA warp
      asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
      __syncwarp();
      if (lane == 0)
        asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(&acc_empty[buf]))
                     : "memory");
    }
  }
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
  __syncthreads();
  if (abort_flag && threadIdx.x == 0) atomicExch(ep.err, 1);
  if (warp == 1) {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(PTMEM_COLS)
                 : "memory");
  }
}

// ------------------------------------------------------------------------------ host side

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// Row-major int8 matrix [rows][K] viewed as a 2-D tensor (K innermost) with box {BK, box_rows}.
bool make_map(CUtensorMap* map, const void* base, int rows, int K, int box_rows) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {(cuuint64_t)K, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)K};
  cuuint32_t box[2] = {(cuuint32_t)BK, (cuuint32_t)box_rows};
  cuuint32_t estr[2] = {1, 1};
  const CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides,
                        box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

inline size_t al256(size_t x) { return (x + 255) & ~size_t(255); }

struct Ws {
  int8_t* xq;
  float* s;
  int32_t* sumq;
  float* tf;
  int8_t* w8;
  int* err;
};

size_t ws_bytes(int M, int K, int N) {
  return al256((size_t)M * K) + al256((size_t)M * 4) * 2 + al256((size_t)M * 16 * 4) +
         al256((size_t)N * K) + 256;
}

Ws carve(void* base, int M, int K, int N) {
  char* p = static_cast<char*>(base);
  Ws w;
  w.xq = reinterpret_cast<int8_t*>(p);
  p += al256((size_t)M * K);
  w.s = reinterpret_cast<float*>(p);
  p += al256((size_t)M * 4);
  w.sumq = reinterpret_cast<int32_t*>(p);
  p += al256((size_t)M * 4);
  w.tf = reinterpret_cast<float*>(p);
  p += al256((size_t)M * 16 * 4);
  w.w8 = reinterpret_cast<int8_t*>(p);
  p += al256((size_t)N * K);
  w.err = reinterpret_cast<int*>(p);
  return w;
}

}  // namespace prefill

bool encode_u8_map_sw128(CUtensorMap* map, const void* base, int rows, int row_bytes, int box_rows) {
  auto fn = prefill::encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {(cuuint64_t)row_bytes, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)row_bytes};
  cuuint32_t box[2] = {128u, (cuuint32_t)box_rows};
  cuuint32_t estr[2] = {1, 1};
  const CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box,
                        estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

size_t prefill_workspace_bytes(int M, int d_in, int d_out) { return prefill::ws_bytes(M, d_in, d_out); }

}  // namespace dfssm

extern "C" int dfssm_linear_prefill(const dfssm_linear_t* lin, const float* x, int M, float* y,
                                    void* workspace, size_t ws_bytes, const dfssm_debug_t* dbg,
                                    void* stream) {
  return dfssm::linear_prefill_impl(lin, x, M, y, nullptr, false, workspace, ws_bytes, dbg, stream);
}

int dfssm::linear_prefill_impl(const dfssm_linear_t* lin, const float* x, int M, float* y,
                               const float* norm_w, bool resid, void* workspace, size_t ws_bytes,
                               const dfssm_debug_t* dbg, void* stream) {
  using namespace dfssm;
  if (!lin || !x || !y || M < 1) return DFSSM_EINVAL;
  if (lin->d_out < 1 || lin->d_in < 128 || lin->d_in % 128 || lin->d_in > 8192) return DFSSM_EINVAL;
  if (lin->rank < 0 || lin->rank > DFSSM_MAX_RANK) return DFSSM_EINVAL;
  if (!lin->bits || !lin->w_scale) return DFSSM_EINVAL;
  if (lin->rank > 0 && (!lin->lora_b || !lin->lora_b_scale || !lin->lora_a || !lin->lora_a_scale))
    return DFSSM_EINVAL;
  if ((reinterpret_cast<uintptr_t>(lin->bits) & 15) || (reinterpret_cast<uintptr_t>(x) & 15) ||
      (reinterpret_cast<uintptr_t>(y) & 15))
    return DFSSM_EALIGN;
  if (lin->rank == DFSSM_MAX_RANK && (reinterpret_cast<uintptr_t>(lin->lora_a) & 15)) return DFSSM_EALIGN;
  if (norm_w && (reinterpret_cast<uintptr_t>(norm_w) & 15)) return DFSSM_EALIGN;
  if (lin->rank > 0 && (reinterpret_cast<uintptr_t>(lin->lora_b) & 3)) return DFSSM_EALIGN;
  const int K = lin->d_in, N = lin->d_out;
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255) ||
      ws_bytes < prefill::ws_bytes(M, K, N))
    return DFSSM_EWORKSPACE;
  int dev = 0, major = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess || major != 10)
    return DFSSM_EDEVICE;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  prefill::Ws w = prefill::carve(workspace, M, K, N);

  // 1. per-token quantization and LoRA down-projection (one warp per token)
  const size_t qsmem = (size_t)DFSSM_MAX_RANK * K;  // W_B padded to sixteen rows
  const cudaError_t ea = set_max_dynamic_smem(reinterpret_cast<const void*>(prefill::prefill_quant_kernel), 16 * 8192);
  if (ea != cudaSuccess) return record_cuda_failure(ea);
  prefill::prefill_quant_kernel<<<(M + prefill::QW - 1) / prefill::QW, prefill::QW * 32, qsmem, st>>>(
      x, M, K, lin->lora_b, lin->lora_b_scale, lin->rank, norm_w, w.xq, w.s, w.tf, dbg ? dbg->xq : nullptr,
      dbg ? dbg->xscale : nullptr, dbg ? dbg->lora_t : nullptr);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return record_cuda_failure(e);
  // 2. +-1 int8 weights
  const long long words = (long long)N * (K / 32);
  prefill::expand_bits_kernel<<<(unsigned)((words + 255) / 256), 256, 0, st>>>(lin->bits, w.w8, words);
  e = cudaGetLastError();
  if (e != cudaSuccess) return record_cuda_failure(e);
  e = cudaMemsetAsync(w.err, 0, sizeof(int), st);
  if (e != cudaSuccess) return record_cuda_failure(e);
  // 3. tcgen05 GEMM + epilogue
  CUtensorMap map_a, map_b;
  if (!prefill::make_map(&map_a, w.xq, M, K, prefill::BM) || !prefill::make_map(&map_b, w.w8, N, K, prefill::BN))
    return DFSSM_EUNSUPPORTED;
  prefill::EpiArgs ep{};
  ep.s = w.s;
  ep.w_scale = lin->w_scale;
  ep.la_scale = lin->lora_a_scale;
  ep.rank = lin->rank;
  ep.tf = w.tf;
  ep.lora_a = lin->lora_a;
  ep.y = y;
  ep.acc = dbg ? dbg->acc : nullptr;
  ep.M = M;
  ep.N = N;
  ep.K = K;
  ep.err = w.err;
  ep.resid = resid ? 1 : 0;
  e = set_max_dynamic_smem(reinterpret_cast<const void*>(prefill::gemm_kernel), (int)prefill::PSMEM_BYTES);
  if (e != cudaSuccess) return record_cuda_failure(e);
  const int tiles = ((N + prefill::BN - 1) / prefill::BN) * ((M + prefill::BM - 1) / prefill::BM);
  const int grid = tiles < num_sms() ? tiles : num_sms();
  prefill::gemm_kernel<<<grid, prefill::PNT, prefill::PSMEM_BYTES, st>>>(map_a, map_b, ep);
  e = cudaGetLastError();
  if (e != cudaSuccess) return record_cuda_failure(e);
  return DFSSM_OK;
}
