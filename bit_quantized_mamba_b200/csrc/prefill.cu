// M-token prefill of one DF-SSM linear on the 5th-generation (tcgen05) int8 tensor cores
// (gist.science technical summary of DF-SSM, §2.C: the packed 1-bit weights are expanded on the fly to
// int8 and multiplied on the INT8 tensor cores).  At M = 2048 tokens the scaffold matmul is a dense
// contraction, so it runs as an int8 GEMM with int32 accumulation in tensor memory:
//   1. quantize every token (per-token absmax int8 codes and scale exactly as in decode), its code sum
//      and its LoRA down-projection; the codes are stored for the GEMM in the bit-sliced order of every
//      32-input block (position 4j + b holds input 8b + j);
//   2. acc[n][m] = sum over set sign bits of q[m] on tcgen05.mma kind::i8: tiles of 128 weight rows (the
//      MMA's M) by 256 tokens (its N), K steps of 128.  The sign bits travel by TMA (2 KB per step) and
//      four expander warps turn them into 0/1 byte masks in shared memory, mask word j of a 32-bit sign
//      word being (w >> j) & 0x01010101 (two operations per four weights) in the codes' order; the
//      codes arrive by TMA with the 128-byte swizzle.  The expanded weights never touch global memory;
//   3. the epilogue reads each accumulator from tensor memory while the next tile accumulates into the
//      other one, forms the scaffold sum 2 acc - sum q and
//      y[m][n] = fl32(scaffold s[m] sW[n] + sA[n] sum_r W_A[n][r] tf[m][r]) in fp64 with the decode
//      path's rounding sequence (one lane per weight row, so a warp's stores of a token cover 32
//      consecutive outputs).
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

constexpr int BM = 128;   // weight rows per tile (the MMA's M)
constexpr int BN = 256;   // tokens per tile (the MMA's N)
constexpr int BK = 128;   // K per stage (bytes = int8 elements)
constexpr int STAGES = 3;
constexpr int UMMA_K = 32;  // K of one kind::i8 MMA (bytes)
// stage: expanded weight masks [BM][BK] (128-byte swizzle), codes [BN][BK] (128-byte swizzle), sign bits
// [BM][BK / 8]
constexpr int A_BYTES = BM * BK, B_BYTES = BN * BK, BITS_BYTES = BM * (BK / 8);
constexpr int STAGE_BYTES = A_BYTES + B_BYTES + BITS_BYTES;
// Token table of one tile of BN tokens, written by the quantizer and bulk-copied whole by the GEMM:
// tf f32 [BN][16] | s f64 [BN] | sum of codes i32 [BN] | exact-LoRA flag i32 [BN]
constexpr int TAB_TF = 0, TAB_S = BN * DFSSM_MAX_RANK * 4, TAB_SQ = TAB_S + BN * 8, TAB_EX = TAB_SQ + BN * 4;
constexpr int TAB_BYTES = TAB_EX + BN * 4;
constexpr long long kWaitBudget = 4000000000LL;  // clock cycles per wait (~2 s)

struct EpiArgs {
  const unsigned char* tab;  // [ceil(M / BN)][TAB_BYTES] token tables (tf, s, sum of codes, exact flag)
  const float* w_scale; // [N]
  const float* la_scale;// [N]
  int rank;
  float* y;             // [M][N]
  int32_t* acc;         // [M][N] or null
  const int8_t* lora_a; // [N][rank]
  int M, N, K;
  int* err;             // status word: kDeviceTimeout after a wait ran out of budget
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

// Bulk copy of `bytes` (a multiple of 16; both addresses 16-byte aligned) from global to shared memory,
// completion counted on `bar`.
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                   smem_u32(dst)),
               "l"(src), "r"(bytes), "r"(smem_u32(bar))
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
// kind::i8 instruction descriptor: D s32, A s8 (0/1 masks), B s8 (codes), both K-major, M = BM, N = BN.
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
// d += A (16 x 4) B (4 x 8) in fp64 on the tensor core (the warp-wide legacy MMA).  Fragments: lane (g, t4)
// = (lane / 4, lane % 4) holds A[g][t4] (a0) and A[g + 8][t4] (a1), B[t4][g] (b), and D[g][2 t4 + {0, 1}]
// (d[0], d[1]) and D[g + 8][2 t4 + {0, 1}] (d[2], d[3]).
__device__ __forceinline__ void dmma_m16n8k4(double (&d)[4], double a0, double a1, double b) {
  asm volatile("mma.sync.aligned.m16n8k4.row.col.f64.f64.f64.f64 {%0, %1, %2, %3}, {%4, %5}, {%6}, {%0, %1, %2, %3};"
               : "+d"(d[0]), "+d"(d[1]), "+d"(d[2]), "+d"(d[3])
               : "d"(a0), "d"(a1), "d"(b));
}
__device__ __forceinline__ void tmem_ld8(uint32_t taddr, uint32_t (&r)[8]) {
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7])
               : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// ------------------------------------------------------------------------------ kernels

// Quantization for the prefill: one warp per token.  Codes and scale exactly as the decode quantizer,
// stored for the GEMM in the bit-sliced order of every 32-input block (byte 4j + b = input 8b + j, gathered
// across the block's eight lanes by shuffles), and their sum; the LoRA down-projection t = W_B q on the codes (int32, dp4a) with W_B staged in
// shared memory (zero rows beyond the rank, so every lane runs all sixteen rows without branches), and
// tf = fl32(t sB s) rounded as in the decode path.  Each lane keeps eight 16-byte loads of its token in
// flight.  With a norm weight (a layer's pre-norm or gated norm) the token is first normalized as in
// decode: r = fl32(1/sqrt(sum x^2 / K + 1e-5)) (fp64) and v = fl32(fl32(x r) w) is quantized.
constexpr int QW = 8;  // tokens (warps) per CTA
static_assert(BN % QW == 0, "the quantizer's CTAs cover whole token tables");
constexpr int QU = 8;  // float4 loads in flight per lane
template <bool XREG>  // XREG: K <= 2048, the token's values stay in registers between the passes
__global__ void __launch_bounds__(QW * 32) prefill_quant_kernel(const float* __restrict__ x, int M, int K,
                                                               const int8_t* __restrict__ lora_b,
                                                               const float* __restrict__ lora_b_scale,
                                                               int rank, const float* __restrict__ norm_w,
                                                               int8_t* __restrict__ xq,
                                                               unsigned char* __restrict__ tab,
                                                               int8_t* dbg_xq, float* dbg_s, int32_t* dbg_t) {
  extern __shared__ __align__(16) unsigned char sm[];
  int8_t* wb = reinterpret_cast<int8_t*>(sm);  // [16][K]
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // W_B into shared memory by asynchronous copies (16 bytes when W_B is 16-byte aligned, else 4), rows
  // past the rank zeroed; awaited just before the codes pass, so the copies overlap the first passes
  {
    const bool a16 = (reinterpret_cast<uintptr_t>(lora_b) & 15) == 0;
    const int step = a16 ? 16 : 4;
    for (int i = threadIdx.x * step; i < DFSSM_MAX_RANK * K; i += QW * 32 * step) {
      const uint32_t d = (uint32_t)__cvta_generic_to_shared(wb + i);
      if (i >= rank * K) {
        if (a16) *reinterpret_cast<uint4*>(wb + i) = make_uint4(0u, 0u, 0u, 0u);
        else *reinterpret_cast<uint32_t*>(wb + i) = 0u;
      } else if (a16) {
        asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(d), "l"(lora_b + i) : "memory");
      } else {
        asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(d), "l"(lora_b + i) : "memory");
      }
    }
    asm volatile("cp.async.commit_group;" ::: "memory");
  }
  const int m = blockIdx.x * QW + warp;
  unsigned char* tb = tab + (size_t)(m / BN) * TAB_BYTES;
  const int mi = m % BN;
  const bool active = m < M;  // warps past M reach the staging barrier, then write zero parameters
  const float4* xr = reinterpret_cast<const float4*>(x + (size_t)(active ? m : 0) * K);
  const float4* wr = reinterpret_cast<const float4*>(norm_w);
  const int K4 = K / 4;  // a multiple of 32: the bounds tests below are uniform over the warp
  constexpr int UB = QU;  // float4 per lane per batch
  constexpr int VR = XREG ? 16 : 1;  // float4 per lane kept in registers (K <= 2048)
  const int V = K4 / 32;
  float4 xv[VR];
  if (XREG && active) {
#pragma unroll
    for (int k = 0; k < VR; ++k) xv[k] = k < V ? __ldg(xr + lane + 32 * k) : make_float4(0.f, 0.f, 0.f, 0.f);
  }
  // RMSNorm factor (with a norm weight): a first pass for the sum of squares (exact squares in fp64, each
  // lane's in increasing index order)
  float rn = 1.0f;
  if (XREG) {
    if (wr && active) {
      double ss = 0.0;
#pragma unroll
      for (int k = 0; k < VR; ++k) {
        ss = fma((double)xv[k].x, (double)xv[k].x, ss);
        ss = fma((double)xv[k].y, (double)xv[k].y, ss);
        ss = fma((double)xv[k].z, (double)xv[k].z, ss);
        ss = fma((double)xv[k].w, (double)xv[k].w, ss);
      }
      rn = rms_factor(warp_sum(ss), K);
    }
  } else if (wr && active) {
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
  if (XREG) {
    if (active) {
#pragma unroll
      for (int k = 0; k < VR; ++k) {
        if (wr && k < V) xv[k] = scale4(xv[k], lane + 32 * k);
        m_abs = fmaxf(m_abs, fmaxf(fmaxf(fabsf(xv[k].x), fabsf(xv[k].y)), fmaxf(fabsf(xv[k].z), fabsf(xv[k].w))));
      }
    }
  } else if (active)
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
  int sq = 0;
  // lane l holds inputs 4l'..4l'+3 of its 32-input block (l' = l & 7); the GEMM word l' of the block is
  // inputs l', 8 + l', 16 + l', 24 + l', i.e. byte (l' & 3) of lanes 2b + (l' >> 2) of the block
  const int lb = lane & ~7, lj = lane & 7;
  const uint32_t bsel = (uint32_t)(lj & 3);
  asm volatile("cp.async.wait_all;" ::: "memory");
  __syncthreads();  // W_B staged
  if (!active) {
    // the last table's tokens past M: zero parameters, trivially exact
    if (lane < DFSSM_MAX_RANK) reinterpret_cast<float*>(tb + TAB_TF)[mi * DFSSM_MAX_RANK + lane] = 0.0f;
    if (lane == 0) {
      reinterpret_cast<double*>(tb + TAB_S)[mi] = 0.0;
      reinterpret_cast<int*>(tb + TAB_SQ)[mi] = 0;
      reinterpret_cast<int*>(tb + TAB_EX)[mi] = 1;
    }
    return;
  }
  // one token group of four values: codes, the bit-sliced gather, the LoRA-down dot products
  const auto codes4 = [&](const float4 vs, int i) {
    const float vv[4] = {vs.x, vs.y, vs.z, vs.w};
    int cd[4];
    quant_codes<4>(vv, s0, inv_s0, cd);
    uint32_t packed = 0;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      packed |= ((uint32_t)cd[j] & 0xFFu) << (8 * j);
      sq += cd[j];
    }
    uint32_t g = 0;
#pragma unroll
    for (int b = 0; b < 4; ++b) {
      const uint32_t v = __shfl_sync(0xffffffffu, packed, lb + 2 * b + (lj >> 2));
      g |= ((v >> (8 * bsel)) & 0xFFu) << (8 * b);
    }
    reinterpret_cast<uint32_t*>(xq + (size_t)m * K)[i] = g;
    if (dbg_xq) reinterpret_cast<uint32_t*>(dbg_xq + (size_t)m * K)[i] = packed;
#pragma unroll
    for (int r = 0; r < DFSSM_MAX_RANK; ++r)
      u[r] = dp4a_ss(reinterpret_cast<const uint32_t*>(wb + (size_t)r * K)[i], packed, u[r]);
  };
  if (XREG) {
#pragma unroll
    for (int k = 0; k < VR; ++k)
      if (k < V) codes4(xv[k], lane + 32 * k);
  } else
  for (int i0 = lane; i0 < K4; i0 += 32 * UB) {
    float4 v[UB];
#pragma unroll
    for (int q = 0; q < UB; ++q)
      v[q] = i0 + 32 * q < K4 ? __ldg(xr + i0 + 32 * q) : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int q = 0; q < UB; ++q) {
      const int i = i0 + 32 * q;
      if (i < K4) codes4(scale4(v[q], i), i);
    }
  }
#pragma unroll
  for (int r = 0; r < DFSSM_MAX_RANK; ++r) u[r] = __reduce_add_sync(0xffffffffu, u[r]);
  sq = __reduce_add_sync(0xffffffffu, sq);
  float tf = 0.0f;
  if (lane < DFSSM_MAX_RANK) {
    int tv = 0;
#pragma unroll
    for (int r = 0; r < DFSSM_MAX_RANK; ++r)
      if (r == lane) tv = u[r];
    tf = lane < rank ? lora_tf(tv, __ldg(lora_b_scale + lane), s_tok) : 0.0f;
    reinterpret_cast<float*>(tb + TAB_TF)[mi * DFSSM_MAX_RANK + lane] = tf;
    if (dbg_t && lane < rank) dbg_t[(size_t)m * rank + lane] = tv;
  }
  // Exactness of the LoRA-up sum of this token (the GEMM epilogue may then take it in any order): with
  // W_A integer (|W_A| <= 2^7) and sixteen terms, every partial sum of W_A tf is a multiple of the last
  // place of the smallest nonzero tf and below 2^11 times the largest |tf|, so when the biased exponents
  // of the nonzero tf (denormals counted as 1) span at most 18, every partial sum fits a 53-bit
  // significand and the fp64 sum is exact whatever the order.
  const uint32_t fb = __float_as_uint(tf) & 0x7FFFFFFFu;
  const int ex = fb ? max((int)(fb >> 23), 1) : 0;
  const int emax = __reduce_max_sync(0xffffffffu, ex);
  const int emin = __reduce_min_sync(0xffffffffu, fb ? ex : 255);
  if (lane == 0) {
    reinterpret_cast<double*>(tb + TAB_S)[mi] = (double)s_tok;
    reinterpret_cast<int*>(tb + TAB_SQ)[mi] = sq;
    reinterpret_cast<int*>(tb + TAB_EX)[mi] = (emax == 0 || emax - emin <= 18) ? 1 : 0;
    if (dbg_s) dbg_s[m] = s_tok;
  }
}

// Persistent tcgen05 GEMM: one CTA per SM walks the (128 weight rows x 256 tokens) output tiles.  Warp 0
// streams each K step's codes and sign bits by TMA; warps 2..5 expand the sign bits into 0/1 byte masks
// (one weight row per thread); warp 1 issues the int8 MMAs into one of two int32 accumulators of 256
// columns; warps 6..13 drain the other one (two warps per 32-lane TMEM quadrant, each taking half of the
// 256 token columns) and evaluate the fp64 epilogue, so a tile's epilogue overlaps the next tile's main
// loop.  TMEM columns: [0, 512).
constexpr int EXP_WARPS = 4;
constexpr int EPI_WARPS = 8;
constexpr int EPI_COLS = BN / (EPI_WARPS / 4);       // token columns per epilogue warp
constexpr int EPI_BASE = 2 + EXP_WARPS;              // first epilogue warp
constexpr int PNT = (EPI_BASE + EPI_WARPS) * 32;     // 448 threads
constexpr int PTMEM_COLS = 2 * BN;                   // two int32 accumulators of BN columns
constexpr size_t OFF_BARS = (size_t)STAGES * STAGE_BYTES;
constexpr size_t OFF_TAB = OFF_BARS + 512;                          // [2][TAB_BYTES] token tables
constexpr size_t OFF_LO = OFF_TAB + 2 * (size_t)TAB_BYTES;          // [EPI_WARPS][32][8] LoRA sums
constexpr size_t PSMEM_BYTES = 1024 + OFF_LO + (size_t)EPI_WARPS * 32 * 8 * 8;

// Bounded wait that ignores the abort flag (used to drain work already issued).
__device__ __forceinline__ void mbar_wait_drain(uint64_t* bar, uint32_t parity) {
  const long long t0 = clock64();
  while (!mbar_try_wait(bar, parity))
    if (clock64() - t0 > kWaitBudget) return;
}

template <bool RESID>  // RESID: y[m][n] = fl32(y[m][n] + out), a residual add in place
__global__ void __launch_bounds__(PNT, 1)
    gemm_kernel(const __grid_constant__ CUtensorMap map_q, const __grid_constant__ CUtensorMap map_bits,
                const EpiArgs ep) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  // aligned by an offset from the array itself, so that every access stays a shared-memory access
  unsigned char* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + OFF_BARS);  // [STAGES] TMA -> expanders, MMA
  uint64_t* aready = full + STAGES;        // [STAGES] expanders -> MMA
  uint64_t* empty = aready + STAGES;       // [STAGES] MMA -> producer
  uint64_t* acc_full = empty + STAGES;     // [2] MMA -> epilogue
  uint64_t* acc_empty = acc_full + 2;      // [2] epilogue -> MMA
  uint64_t* mma_done = acc_empty + 2;      // every MMA of this CTA complete
  uint64_t* tab_full = mma_done + 1;       // [2] token-table copy landed
  uint64_t* tab_empty = tab_full + 2;      // [2] epilogue -> producer
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(tab_empty + 2);
  double* lo_all = reinterpret_cast<double*>(smem + OFF_LO);
  __shared__ int abort_flag;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int tiles_r = (ep.N + BM - 1) / BM, tiles_t = (ep.M + BN - 1) / BN;
  const int tiles = tiles_r * tiles_t;
  const int kblocks = ep.K / BK;

  if (threadIdx.x == 0) {
    abort_flag = 0;
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&aready[s], EXP_WARPS);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], EPI_WARPS);
    }
    mbar_init(mma_done, 1);
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tab_full[b], 1);
      mbar_init(&tab_empty[b], EPI_WARPS);
    }
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
    // ---- TMA producer: each tile's K steps through the stage ring
    int it = 0, pl = 0;
    bool ok = true;
    for (int t = blockIdx.x; t < tiles && ok; t += gridDim.x, ++pl) {
      const int r0 = (t % tiles_r) * BM, n0 = (t / tiles_r) * BN;
      // the tile's token table (one bulk copy) into the slot the epilogue of tile pl - 2 released
      const int sl = pl & 1;
      if (pl >= 2 && !mbar_wait(&tab_empty[sl], ((pl >> 1) - 1) & 1, &abort_flag)) {
        abort_flag = 1;
        ok = false;
        break;
      }
      mbar_expect_tx(&tab_full[sl], TAB_BYTES);
      bulk_g2s(smem + OFF_TAB + (size_t)sl * TAB_BYTES, ep.tab + (size_t)(n0 / BN) * TAB_BYTES, TAB_BYTES,
               &tab_full[sl]);
      for (int kb = 0; kb < kblocks; ++kb, ++it) {
        const int s = it % STAGES;
        if (it >= STAGES && !mbar_wait(&empty[s], ((it / STAGES) - 1) & 1, &abort_flag)) {
          abort_flag = 1;
          ok = false;
          break;
        }
        unsigned char* st = smem + (size_t)s * STAGE_BYTES;
        mbar_expect_tx(&full[s], B_BYTES + BITS_BYTES);
        tma_load_2d(st + A_BYTES, &map_q, kb * BK, n0, &full[s]);                 // codes, 256 tokens
        tma_load_2d(st + A_BYTES + B_BYTES, &map_bits, kb * (BK / 8), r0, &full[s]);  // bits, 128 rows
      }
    }
    // the last copies land before this CTA may exit (a table copy of tile j completes phase j / 2 of its
    // slot; the epilogue may already have consumed it, which leaves the wait satisfied)
    for (int j = (it > STAGES ? it - STAGES : 0); j < it; ++j) mbar_wait_drain(&full[j % STAGES], (j / STAGES) & 1);
    for (int j = (pl > 2 ? pl - 2 : 0); j < pl; ++j) mbar_wait_drain(&tab_full[j & 1], (j >> 1) & 1);
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
        if (!mbar_wait(&full[s], (it / STAGES) & 1, &abort_flag) ||
            !mbar_wait(&aready[s], (it / STAGES) & 1, &abort_flag)) {
          abort_flag = 1;
          ok = false;
          break;
        }
        asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
        const uint32_t a_addr = smem_u32(smem + (size_t)s * STAGE_BYTES);
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
  } else if (warp >= 2 && warp < EPI_BASE) {
    // ---- expanders: thread r owns weight row r of the tile; its 16 bytes of sign bits (128 weights)
    // become 128 mask bytes, 16-byte chunk c holding mask words 4 (c & 1) .. + 3 of sign word c >> 1,
    // stored at chunk position c ^ (r & 7) of the row (the 128-byte swizzle the MMA descriptor reads)
    const int r = threadIdx.x - 64;
    int it = 0;
    for (int t = blockIdx.x; t < tiles; t += gridDim.x) {
      bool ok = true;
      for (int kb = 0; kb < kblocks; ++kb, ++it) {
        const int s = it % STAGES;
        if (!mbar_wait(&full[s], (it / STAGES) & 1, &abort_flag)) {
          abort_flag = 1;
          ok = false;
          break;
        }
        unsigned char* st = smem + (size_t)s * STAGE_BYTES;
        const uint4 wv = reinterpret_cast<const uint4*>(st + A_BYTES + B_BYTES)[r];
        const uint32_t w4[4] = {wv.x, wv.y, wv.z, wv.w};
        unsigned char* arow = st + r * 128;
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          const uint32_t w = w4[c >> 1];
          const int j0 = 4 * (c & 1);
          const uint4 m = make_uint4((w >> j0) & 0x01010101u, (w >> (j0 + 1)) & 0x01010101u,
                                     (w >> (j0 + 2)) & 0x01010101u, (w >> (j0 + 3)) & 0x01010101u);
          *reinterpret_cast<uint4*>(arow + ((c ^ (r & 7)) << 4)) = m;
        }
        // the masks were written by the generic proxy; the tensor core reads them through the async proxy
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        __syncwarp();
        if (lane == 0)
          asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(&aready[s])) : "memory");
      }
      if (!ok) break;
    }
  } else if (warp >= EPI_BASE) {
    // ---- epilogue: warp e drains TMEM lanes [32 (warp % 4), +32) (weight rows) and token half e / 4
    const int e = warp - EPI_BASE;
    const int q = warp & 3;
    const int part = e >> 2;
    const int g = lane >> 2, t4 = lane & 3;        // DMMA fragment coordinates
    double* lo = lo_all + (size_t)e * 32 * 8;      // this warp's LoRA sums, [32 rows][8 tokens], swizzled
    int local = 0;
    bool ok = true;
    for (int t = blockIdx.x; t < tiles; t += gridDim.x, ++local) {
      const int buf = local & 1, sl = local & 1;
      const int r0 = (t % tiles_r) * BM, n0 = (t / tiles_r) * BN;
      // this lane's weight row: sW, sA and the W_A bytes (zero beyond the rank), loads issued first
      const int row = r0 + q * 32 + lane;
      const bool rv = row < ep.N;
      const float fw = rv ? __ldg(ep.w_scale + row) : 0.0f;
      const float fa = (rv && ep.rank > 0) ? __ldg(ep.la_scale + row) : 0.0f;
      uint32_t war[4] = {0u, 0u, 0u, 0u};
      if (rv && ep.rank == DFSSM_MAX_RANK) {
        const uint4 w = __ldg(reinterpret_cast<const uint4*>(ep.lora_a + (size_t)row * DFSSM_MAX_RANK));
        war[0] = w.x;
        war[1] = w.y;
        war[2] = w.z;
        war[3] = w.w;
      } else if (rv) {
#pragma unroll
        for (int r = 0; r < DFSSM_MAX_RANK; ++r)
          if (r < ep.rank)
            war[r >> 2] |= (uint32_t)(uint8_t)ep.lora_a[(size_t)row * ep.rank + r] << (8 * (r & 3));
      }
      const double sw = (double)fw, sa = (double)fa;
      const bool rows_full = r0 + BM <= ep.N;  // every lane of the tile has a row
      // W_A of the warp's 32 rows as DMMA A fragments [m block][k step][row g / g + 8], k = 4 ks + t4,
      // gathered from the rows' lanes
      double afr[2][4][2];
#pragma unroll
      for (int mb = 0; mb < 2; ++mb)
#pragma unroll
        for (int h = 0; h < 2; ++h)
#pragma unroll
          for (int ks = 0; ks < 4; ++ks) {
            const uint32_t w = __shfl_sync(0xffffffffu, war[ks], 16 * mb + 8 * h + g);
            afr[mb][ks][h] = int_to_f64((int)(int8_t)(w >> (8 * t4)));
          }
      // every epilogue warp runs every tile iteration; after an abort the accumulators are not read
      ok = ok && !abort_flag && mbar_wait(&tab_full[sl], (local >> 1) & 1, &abort_flag) &&
           mbar_wait(&acc_full[buf], (local >> 1) & 1, &abort_flag);
      asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
      if (!ok) {
        abort_flag = 1;
        if (lane == 0) atomicExch(ep.err, kDeviceTimeout);
      }
      const unsigned char* tb = smem + OFF_TAB + (size_t)sl * TAB_BYTES;
      const float* tf_t = reinterpret_cast<const float*>(tb + TAB_TF);
      const double* s_t = reinterpret_cast<const double*>(tb + TAB_S);
      const int* sq_t = reinterpret_cast<const int*>(tb + TAB_SQ);
      const int* ex_t = reinterpret_cast<const int*>(tb + TAB_EX);
      const bool lora_on = ep.rank > 0;
      for (int cc = 0; ok && cc < EPI_COLS; cc += 8) {
        const int c0 = part * EPI_COLS + cc;
        uint32_t v[8];
        tmem_ld8(tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(buf * BN + c0), v);
        // y = fl32(a s sW + sA sum_r W_A tf), fp64, the decode path's rounding sequence (linear_out_n), with
        // a = 2 acc - sum q the +-1 scaffold sum.  The LoRA sum of the sixteen products (each exact in
        // fp64) is, for a block of eight tokens whose sums are all exact, taken on the fp64 tensor core
        // (any order gives the exact value, so the sequential fp64 sum's); otherwise by the sequential fma
        // chain over r = 0..15, fma(w, tf, lora) rounding as lora + w tf does.  Zero weights beyond the rank
        // leave either sum unchanged (it is never -0).
        double lora[8];
        if (!lora_on) {
#pragma unroll
          for (int jj = 0; jj < 8; ++jj) lora[jj] = 0.0;
        } else if (__all_sync(0xffffffffu, lane >= 8 || ex_t[c0 + lane] != 0)) {
          double d[2][4];
#pragma unroll
          for (int mb = 0; mb < 2; ++mb)
#pragma unroll
            for (int i = 0; i < 4; ++i) d[mb][i] = 0.0;
#pragma unroll
          for (int ks = 0; ks < 4; ++ks) {
            const double b = (double)tf_t[(c0 + g) * DFSSM_MAX_RANK + 4 * ks + t4];
#pragma unroll
            for (int mb = 0; mb < 2; ++mb) dmma_m16n8k4(d[mb], afr[mb][ks][0], afr[mb][ks][1], b);
          }
          // fragment (row 16 mb + 8 h + g, tokens 2 t4, 2 t4 + 1) -> this lane's row: through a row-major
          // [32][8] buffer whose 16-byte chunks are swizzled by (row / 2) & 3 (conflict-free both ways)
#pragma unroll
          for (int mb = 0; mb < 2; ++mb)
#pragma unroll
            for (int h = 0; h < 2; ++h) {
              const int rw = 16 * mb + 8 * h + g;
              *reinterpret_cast<double2*>(lo + rw * 8 + ((t4 ^ ((rw >> 1) & 3)) << 1)) =
                  make_double2(d[mb][2 * h], d[mb][2 * h + 1]);
            }
          __syncwarp();
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const double2 x = *reinterpret_cast<const double2*>(lo + lane * 8 + ((i ^ ((lane >> 1) & 3)) << 1));
            lora[2 * i] = x.x;
            lora[2 * i + 1] = x.y;
          }
          __syncwarp();
        } else {
#pragma unroll
          for (int jj = 0; jj < 8; ++jj) lora[jj] = 0.0;
#pragma unroll 1
          for (int r = 0; r < ep.rank; ++r) {
            const uint32_t wr = r < 4 ? war[0] : r < 8 ? war[1] : r < 12 ? war[2] : war[3];
            const double w = int_to_f64((int)(int8_t)(wr >> (8 * (r & 3))));
#pragma unroll
            for (int jj = 0; jj < 8; ++jj) lora[jj] = fma(w, (double)tf_t[(c0 + jj) * DFSSM_MAX_RANK + r], lora[jj]);
          }
        }
        float out[8];
        int av[8];
        if (lora_on) {
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            av[j] = 2 * (int)v[j] - sq_t[c0 + j];
            out[j] = __double2float_rn(dadd(dmul(dmul(int_to_f64(av[j]), s_t[c0 + j]), sw), dmul(sa, lora[j])));
          }
        } else {
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            av[j] = 2 * (int)v[j] - sq_t[c0 + j];
            out[j] = __double2float_rn(dadd(dmul(dmul(int_to_f64(av[j]), s_t[c0 + j]), sw), 0.0));
          }
        }
        if (RESID) {
#pragma unroll
          for (int j = 0; j < 8; ++j)
            if (rv && n0 + c0 + j < ep.M) out[j] = fadd(ep.y[(size_t)(n0 + c0 + j) * ep.N + row], out[j]);
        }
        float* yp = ep.y + (size_t)(n0 + c0) * ep.N + row;
        if (rows_full && n0 + c0 + 8 <= ep.M) {
#pragma unroll
          for (int j = 0; j < 8; ++j) yp[(size_t)j * ep.N] = out[j];
        } else {
#pragma unroll
          for (int j = 0; j < 8; ++j)
            if (rv && n0 + c0 + j < ep.M) yp[(size_t)j * ep.N] = out[j];
        }
        if (ep.acc) {
#pragma unroll
          for (int j = 0; j < 8; ++j)
            if (rv && n0 + c0 + j < ep.M) ep.acc[(size_t)(n0 + c0 + j) * ep.N + row] = av[j];
        }
      }
      // this warp's reads of the accumulators and of the token table are complete
      asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
      __syncwarp();
      if (lane == 0) {
        asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(&acc_empty[buf])) : "memory");
        asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(&tab_empty[sl])) : "memory");
      }
    }
  }
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
  __syncthreads();
  if (abort_flag && threadIdx.x == 0) atomicExch(ep.err, kDeviceTimeout);
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

// Packed sign bits [rows][K / 32] u32 viewed as a 2-D byte tensor with box {BK / 8 bytes, BM rows}, no
// swizzle (each row's 16 bytes of a K step land contiguously).
bool make_bits_map(CUtensorMap* map, const void* base, int rows, int K) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {(cuuint64_t)(K / 8), (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)(K / 8)};
  cuuint32_t box[2] = {(cuuint32_t)(BK / 8), (cuuint32_t)BM};
  cuuint32_t estr[2] = {1, 1};
  const CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides,
                        box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

inline size_t al256(size_t x) { return (x + 255) & ~size_t(255); }

struct Ws {
  int* err;
  int8_t* xq;
  unsigned char* tab;
};

// [status word (256 B)][codes M x K][token tables ceil(M / BN) x TAB_BYTES]
size_t ws_bytes(int M, int K, int /*N*/) {
  return kStatusBytes + al256((size_t)M * K) + (size_t)((M + BN - 1) / BN) * TAB_BYTES;
}

Ws carve(void* base, int M, int K) {
  char* p = static_cast<char*>(base);
  Ws w;
  w.err = reinterpret_cast<int*>(p);
  p += kStatusBytes;
  w.xq = reinterpret_cast<int8_t*>(p);
  p += al256((size_t)M * K);
  w.tab = reinterpret_cast<unsigned char*>(p);
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
  return dfssm::linear_prefill_impl(lin, x, M, y, nullptr, false, workspace, ws_bytes, nullptr, dbg, stream);
}

int dfssm::linear_prefill_impl(const dfssm_linear_t* lin, const float* x, int M, float* y,
                               const float* norm_w, bool resid, void* workspace, size_t ws_bytes,
                               int* status, const dfssm_debug_t* dbg, void* stream) {
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
  prefill::Ws w = prefill::carve(workspace, M, K);

  // 1. per-token quantization and LoRA down-projection (one warp per token)
  const size_t qsmem = (size_t)DFSSM_MAX_RANK * K;  // W_B padded to sixteen rows
  const auto qk = K <= 2048 ? prefill::prefill_quant_kernel<true> : prefill::prefill_quant_kernel<false>;
  const cudaError_t ea = set_max_dynamic_smem(reinterpret_cast<const void*>(qk), 16 * 8192);
  if (ea != cudaSuccess) return record_cuda_failure(ea);
  const int m_pad = (M + prefill::BN - 1) / prefill::BN * prefill::BN;  // whole token tables
  qk<<<m_pad / prefill::QW, prefill::QW * 32, qsmem, st>>>(
      x, M, K, lin->lora_b, lin->lora_b_scale, lin->rank, norm_w, w.xq, w.tab, dbg ? dbg->xq : nullptr,
      dbg ? dbg->xscale : nullptr, dbg ? dbg->lora_t : nullptr);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return record_cuda_failure(e);
  // 2. tcgen05 GEMM (sign bits expanded in shared memory) + epilogue
  CUtensorMap map_q, map_bits;
  if (!prefill::make_map(&map_q, w.xq, M, K, prefill::BN) || !prefill::make_bits_map(&map_bits, lin->bits, N, K))
    return DFSSM_EUNSUPPORTED;
  prefill::EpiArgs ep{};
  ep.tab = w.tab;
  ep.w_scale = lin->w_scale;
  ep.la_scale = lin->lora_a_scale;
  ep.rank = lin->rank;
  ep.lora_a = lin->lora_a;
  ep.y = y;
  ep.acc = dbg ? dbg->acc : nullptr;
  ep.M = M;
  ep.N = N;
  ep.K = K;
  ep.err = status ? status : w.err;
  const auto kern = resid ? prefill::gemm_kernel<true> : prefill::gemm_kernel<false>;
  e = set_max_dynamic_smem(reinterpret_cast<const void*>(kern), (int)prefill::PSMEM_BYTES);
  if (e != cudaSuccess) return record_cuda_failure(e);
  const int tiles = ((N + prefill::BM - 1) / prefill::BM) * ((M + prefill::BN - 1) / prefill::BN);
  const int grid = tiles < num_sms() ? tiles : num_sms();
  kern<<<grid, prefill::PNT, prefill::PSMEM_BYTES, st>>>(map_q, map_bits, ep);
  e = cudaGetLastError();
  if (e != cudaSuccess) return record_cuda_failure(e);
  return DFSSM_OK;
}
