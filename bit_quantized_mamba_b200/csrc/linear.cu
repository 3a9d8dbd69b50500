// Decode-time DF-SSM linear: per-token int8 quantization + LoRA-down, then the packed-bit scaffold GEMV
// with the LoRA-up epilogue (gist.science technical summary of DF-SSM, §2.B "Frozen Scaffold with LoRA
// Correction" and §2.C "Optimized Inference Pipeline").
//
// The pages' GPU engine expands the bits to int8 and calls cuBLAS INT8 GEMM.  At batch 1 that is a
// matrix-vector product bound by HBM, so here the bits are streamed once with 16-byte loads and
// expanded in registers: with the activation codes stored in a permuted order (see perm_index), the
// eight sign bits that pair with one activation word are selected by a single AND, and one
// dp4a.u32.s32 accumulates four products:
//     sum_{i: bit=1} q_i  =  sum_k  (sum over bytes of (w & (0x01010101<<k)) * qperm_k) >> k
//     acc                =  2 * sum_{i: bit=1} q_i - sum_i q_i
// which is 2 integer instructions per 4 weights, exact in int32.

#include <atomic>
#include <mutex>
#include <vector>

#include "common.cuh"
#include "internal.h"

namespace dfssm {

// ------------------------------------------------------------------------------------ scratch layout

static inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

size_t quant_scratch_bytes(int B, int n) {
  return align256((size_t)B * n) + align256(sizeof(float) * 16) + align256(sizeof(int32_t) * 16) +
         align256(sizeof(float) * 16 * 16);
}

QuantScratch carve_quant_scratch(void* base, int B, int n) {
  char* p = static_cast<char*>(base);
  QuantScratch s;
  s.q = reinterpret_cast<int8_t*>(p);
  p += align256((size_t)B * n);
  s.s = reinterpret_cast<float*>(p);
  p += align256(sizeof(float) * 16);
  s.sumq = reinterpret_cast<int32_t*>(p);
  p += align256(sizeof(int32_t) * 16);
  s.tf = reinterpret_cast<float*>(p);
  return s;
}

int num_sms() {
  constexpr int kMaxDevices = 64;
  static std::atomic<int> cache[kMaxDevices];  // 0 = not yet queried
  int dev = 0;
  cudaGetDevice(&dev);
  int sms = (dev >= 0 && dev < kMaxDevices) ? cache[dev].load(std::memory_order_relaxed) : 0;
  if (sms == 0) {
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (sms <= 0) sms = 148;
    if (dev >= 0 && dev < kMaxDevices) cache[dev].store(sms, std::memory_order_relaxed);
  }
  return sms;
}

cudaError_t set_max_dynamic_smem(const void* func, int bytes) {
  struct Done {
    const void* func;
    int dev, bytes;
  };
  static std::mutex mu;
  static std::vector<Done> done;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> lock(mu);
  for (const Done& d : done)
    if (d.func == func && d.dev == dev && d.bytes >= bytes) return cudaSuccess;
  e = cudaFuncSetAttribute(func, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e == cudaSuccess) done.push_back(Done{func, dev, bytes});
  return e;
}

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

// ------------------------------------------------------------------------------- quantize kernel
// One CTA per token.  v = x, or with a norm weight the RMSNorm of x: r = fl32(1/sqrt(sum x^2/n + 1e-5))
// (fp64) and v = fl32(fl32(x r) w); then s = fl32(absmax(v)/127), q = clamp(rint(fl32(v/s)), +-127).
// LoRA down on the codes: t[r] = sum_i W_B[r,i] q_i (int32, dp4a), tf[r] = fl32(t[r] sB[r] s).

constexpr int kQuantThreads = 512;

__global__ void __launch_bounds__(kQuantThreads) quant_kernel(QuantArgs a) {
  pdl_launch_dependents();
  pdl_wait();
  extern __shared__ __align__(16) unsigned char smem[];
  float* v = reinterpret_cast<float*>(smem);                       // [n]
  int8_t* qn = reinterpret_cast<int8_t*>(smem + (size_t)a.n * 4);  // [n] natural-order codes
  __shared__ double red_d[kQuantThreads / 32];
  __shared__ float red_f[kQuantThreads / 32];
  __shared__ int red_i[kQuantThreads / 32];
  __shared__ int t_sm[DFSSM_MAX_RANK];
  const int b = blockIdx.x;
  const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
  constexpr int NW = kQuantThreads / 32;
  const float* x = a.x + (size_t)b * a.ldx;

  float r = 1.0f;
  if (a.norm_w) {
    double ss = 0.0;
    for (int i = tid; i < a.n; i += kQuantThreads) {
      const float xv = x[i];
      ss += (double)xv * (double)xv;  // the square of an fp32 value is exact in fp64
    }
    ss = warp_sum(ss);
    if (lane == 0) red_d[wid] = ss;
    __syncthreads();
    ss = 0.0;
    for (int w = 0; w < NW; ++w) ss += red_d[w];
    r = rms_factor(ss, a.n);
  }
  float m = 0.0f;
  for (int i = tid; i < a.n; i += kQuantThreads) {
    const float xv = x[i];
    const float vv = a.norm_w ? norm_value(xv, r, a.norm_w[i]) : xv;
    v[i] = vv;
    m = fmaxf(m, fabsf(vv));
  }
  m = warp_max(m);
  if (lane == 0) red_f[wid] = m;
  __syncthreads();
  m = 0.0f;
  for (int w = 0; w < NW; ++w) m = fmaxf(m, red_f[w]);
  const float s0 = quant_scale(m);
  const float inv_s0 = quant_inv(s0);

  int8_t* qout = a.out.q + (size_t)b * a.n;
  int sq = 0;
  for (int i = tid; i < a.n; i += kQuantThreads) {
    const int c = (m == 0.0f) ? 0 : quant_code_fast(v[i], s0, inv_s0);
    sq += c;
    qn[i] = (int8_t)c;
    qout[a.permute ? perm_index(i) : i] = (int8_t)c;
    if (a.dbg_xq) a.dbg_xq[(size_t)b * a.n + i] = (int8_t)c;
  }
  sq = warp_sum(sq);
  if (lane == 0) red_i[wid] = sq;
  __syncthreads();
  // LoRA down: warp r computes t[r] over 4-byte words of W_B row r and of the codes.
  for (int r = wid; r < a.rank; r += NW) {
    const uint32_t* wb = reinterpret_cast<const uint32_t*>(a.lora_b + (size_t)r * a.n);
    const uint32_t* q4 = reinterpret_cast<const uint32_t*>(qn);
    int part = 0;
    for (int w = lane; w < a.n / 4; w += 32) part = dp4a_ss(ld_stream_u32(wb + w), q4[w], part);
    part = __reduce_add_sync(0xffffffffu, part);
    if (lane == 0) t_sm[r] = part;
  }
  __syncthreads();
  const float s = s0;
  if (tid < DFSSM_MAX_RANK) {
    float tf = 0.0f;
    if (tid < a.rank) {
      tf = lora_tf(t_sm[tid], a.lora_b_scale[tid], s);
      if (a.dbg_t) a.dbg_t[(size_t)b * a.rank + tid] = t_sm[tid];
    }
    a.out.tf[b * DFSSM_MAX_RANK + tid] = tf;
  }
  if (tid == DFSSM_MAX_RANK) {
    int tot = 0;
    for (int w = 0; w < NW; ++w) tot += red_i[w];
    a.out.sumq[b] = tot;
  }
  if (tid == DFSSM_MAX_RANK + 1) {
    a.out.s[b] = s;
    if (a.dbg_s) a.dbg_s[b] = s;
  }
}

cudaError_t launch_quant(const QuantArgs& a, cudaStream_t st) {
  const size_t smem = (size_t)a.n * 5;  // <= 40 KB for n <= 8192
  return launch_pdl(quant_kernel, dim3(a.B), dim3(kQuantThreads), smem, st, a);
}

// ----------------------------------------------------------------------------- scaffold GEMV kernels

constexpr int kGemvThreads = 256;

// LoRA-up epilogue for one (token b, row o).
__device__ __forceinline__ void gemv_epilogue(const GemvArgs& a, int b, int row, int acc, float sW,
                                              float sA, const int8_t* wa, const float* tf,
                                              float s) {
  const float yv = linear_out(acc, s, sW, sA, wa, tf, a.rank);
  if (a.resid) {
    float* h = a.resid + (size_t)b * a.ldr + row;
    *h = fadd(*h, yv);
  } else {
    a.y[(size_t)b * a.ldy + row] = yv;
  }
  if (a.dbg_acc) a.dbg_acc[(size_t)b * a.d_out + row] = acc;
}

// Stage the quantized tokens and the LoRA intermediate tf[b][r] = fl32(t sB s) in shared memory.
__device__ __forceinline__ void gemv_stage(const GemvArgs& a, uint4* qsm, float (*tf)[DFSSM_MAX_RANK],
                                           float* ssm, int* sumq, int nb) {
  const int n16 = nb * a.d_in / 16;
  const uint4* src = reinterpret_cast<const uint4*>(a.in.q);
  for (int i = threadIdx.x; i < n16; i += blockDim.x) qsm[i] = src[i];
  if (threadIdx.x < nb * DFSSM_MAX_RANK) {
    const int b = threadIdx.x / DFSSM_MAX_RANK, r = threadIdx.x % DFSSM_MAX_RANK;
    float v = 0.0f;
    if (r < a.rank) v = a.in.tf[b * DFSSM_MAX_RANK + r];
    tf[b][r] = v;
  }
  if (threadIdx.x < nb) {
    ssm[threadIdx.x] = a.in.s[threadIdx.x];
    sumq[threadIdx.x] = a.in.sumq[threadIdx.x];
  }
}

// Fast path: LPR lanes per row, each lane NSEG 16-byte segments (4 words = 128 weights), BT token slots.
template <int LPR, int NSEG, int BT>
__global__ void __launch_bounds__(kGemvThreads) gemv_kernel(GemvArgs a) {
  constexpr int RPW = 32 / LPR;
  constexpr int RPC = (kGemvThreads / 32) * RPW;
  extern __shared__ __align__(16) unsigned char smem[];
  uint4* qsm = reinterpret_cast<uint4*>(smem);
  __shared__ float tf[BT][DFSSM_MAX_RANK];
  __shared__ float ssc[BT];
  __shared__ int sumq[BT];

  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int li = lane % LPR;
  const int row = blockIdx.x * RPC + warp * RPW + lane / LPR;
  const bool valid = row < a.d_out;
  const int wpr = a.d_in >> 5;

  // Weights first (immutable; may be fetched before the producer of the activations finishes).
  uint4 wv[NSEG];
#pragma unroll
  for (int s = 0; s < NSEG; ++s)
    wv[s] = valid ? ld_stream_u4(a.bits + (size_t)row * wpr + (size_t)(s * LPR + li) * 4)
                  : make_uint4(0, 0, 0, 0);
  float sW = 0.0f, sA = 0.0f;
  alignas(16) int8_t wa[DFSSM_MAX_RANK];
  if (valid) {
    sW = a.w_scale[row];
    if (a.rank > 0) {
      sA = a.lora_a_scale[row];
      if (a.rank == DFSSM_MAX_RANK) {
        *reinterpret_cast<uint4*>(wa) = ld_stream_u4(a.lora_a + (size_t)row * DFSSM_MAX_RANK);
      } else {
        for (int r = 0; r < a.rank; ++r) wa[r] = a.lora_a[(size_t)row * a.rank + r];
      }
    }
  }

  pdl_launch_dependents();
  pdl_wait();
  gemv_stage(a, qsm, tf, ssc, sumq, a.B);
  __syncthreads();

  const int qwords = a.d_in >> 2;  // uint32 words per token in qsm
  const uint32_t* q32 = reinterpret_cast<const uint32_t*>(qsm);
  if constexpr (BT == 1) {
    int acc8[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) acc8[k] = 0;
#pragma unroll
    for (int s = 0; s < NSEG; ++s) {
      const int seg = s * LPR + li;  // 128-weight segment index
      const uint4* qp4 = qsm + seg * 8;
      const uint32_t w4[4] = {wv[s].x, wv[s].y, wv[s].z, wv[s].w};
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const uint4 qa = qp4[2 * j], qb = qp4[2 * j + 1];
        const uint32_t qp[8] = {qa.x, qa.y, qa.z, qa.w, qb.x, qb.y, qb.z, qb.w};
#pragma unroll
        for (int k = 0; k < 8; ++k) acc8[k] = dp4a_us(w4[j] & (0x01010101u << k), qp[k], acc8[k]);
      }
    }
    int S = 0;
#pragma unroll
    for (int k = 0; k < 8; ++k) S += acc8[k] >> k;
#pragma unroll
    for (int o = LPR / 2; o > 0; o >>= 1) S += __shfl_xor_sync(0xffffffffu, S, o);
    if (valid && li == 0) gemv_epilogue(a, 0, row, 2 * S - sumq[0], sW, sA, wa, tf[0], ssc[0]);
  } else {
    int S[BT];
#pragma unroll
    for (int b = 0; b < BT; ++b) S[b] = 0;
#pragma unroll
    for (int s = 0; s < NSEG; ++s) {
      const int seg = s * LPR + li;
      const uint32_t w4[4] = {wv[s].x, wv[s].y, wv[s].z, wv[s].w};
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        uint32_t msk[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) msk[k] = (w4[j] >> k) & 0x01010101u;
#pragma unroll
        for (int b = 0; b < BT; ++b) {
          if (b < a.B) {
            const uint4* qp4 = reinterpret_cast<const uint4*>(q32 + (size_t)b * qwords) + seg * 8;
            const uint4 qa = qp4[2 * j], qb = qp4[2 * j + 1];
            const uint32_t qp[8] = {qa.x, qa.y, qa.z, qa.w, qb.x, qb.y, qb.z, qb.w};
#pragma unroll
            for (int k = 0; k < 8; ++k) S[b] = dp4a_us(msk[k], qp[k], S[b]);
          }
        }
      }
    }
#pragma unroll
    for (int b = 0; b < BT; ++b) {
#pragma unroll
      for (int o = LPR / 2; o > 0; o >>= 1) S[b] += __shfl_xor_sync(0xffffffffu, S[b], o);
    }
    if (valid) {
#pragma unroll
      for (int b = 0; b < BT; ++b)
        if (b < a.B && (b % LPR) == li)
          gemv_epilogue(a, b, row, 2 * S[b] - sumq[b], sW, sA, wa, tf[b], ssc[b]);
    }
  }
}

// Generic path for any d_in % 32 == 0: one warp per row, one 32-bit word per lane-iteration.
template <int BT>
__global__ void __launch_bounds__(kGemvThreads) gemv_generic_kernel(GemvArgs a) {
  constexpr int RPC = kGemvThreads / 32;
  extern __shared__ __align__(16) unsigned char smem[];
  uint4* qsm = reinterpret_cast<uint4*>(smem);
  __shared__ float tf[BT][DFSSM_MAX_RANK];
  __shared__ float ssc[BT];
  __shared__ int sumq[BT];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int row = blockIdx.x * RPC + warp;
  const bool valid = row < a.d_out;
  const int wpr = a.d_in >> 5;
  pdl_launch_dependents();
  pdl_wait();
  gemv_stage(a, qsm, tf, ssc, sumq, a.B);
  __syncthreads();
  const uint32_t* q32 = reinterpret_cast<const uint32_t*>(qsm);
  const int qwords = a.d_in >> 2;
  int S[BT];
#pragma unroll
  for (int b = 0; b < BT; ++b) S[b] = 0;
  if (valid) {
    for (int w = lane; w < wpr; w += 32) {
      const uint32_t bits = ld_stream_u32(a.bits + (size_t)row * wpr + w);
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        const uint32_t msk = (bits >> k) & 0x01010101u;
#pragma unroll
        for (int b = 0; b < BT; ++b)
          if (b < a.B) S[b] = dp4a_us(msk, q32[(size_t)b * qwords + w * 8 + k], S[b]);
      }
    }
  }
#pragma unroll
  for (int b = 0; b < BT; ++b) S[b] = warp_sum(S[b]);
  if (valid && lane == 0) {
    float sW = a.w_scale[row];
    float sA = a.rank > 0 ? a.lora_a_scale[row] : 0.0f;
    alignas(16) int8_t wa[DFSSM_MAX_RANK] = {};
    for (int r = 0; r < a.rank; ++r) wa[r] = a.lora_a[(size_t)row * a.rank + r];
#pragma unroll
    for (int b = 0; b < BT; ++b)
      if (b < a.B) gemv_epilogue(a, b, row, 2 * S[b] - sumq[b], sW, sA, wa, tf[b], ssc[b]);
  }
}

template <int LPR, int NSEG, int BT>
static cudaError_t launch_fast(const GemvArgs& a, cudaStream_t st) {
  constexpr int RPC = (kGemvThreads / 32) * (32 / LPR);
  const size_t smem = (size_t)a.B * a.d_in;
  auto k = gemv_kernel<LPR, NSEG, BT>;
  if (smem > 48 * 1024) {
    // the largest size any call can need, once per device
    const cudaError_t set = set_max_dynamic_smem(reinterpret_cast<const void*>(k), DFSSM_MAX_BATCH * 8192);
    if (set != cudaSuccess) return set;
  }
  return launch_pdl(k, dim3((a.d_out + RPC - 1) / RPC), dim3(kGemvThreads), smem, st, a);
}

template <int BT>
static cudaError_t launch_generic(const GemvArgs& a, cudaStream_t st) {
  constexpr int RPC = kGemvThreads / 32;
  const size_t smem = (size_t)a.B * a.d_in;
  auto k = gemv_generic_kernel<BT>;
  if (smem > 48 * 1024) {
    const cudaError_t set = set_max_dynamic_smem(reinterpret_cast<const void*>(k), DFSSM_MAX_BATCH * 8192);
    if (set != cudaSuccess) return set;
  }
  return launch_pdl(k, dim3((a.d_out + RPC - 1) / RPC), dim3(kGemvThreads), smem, st, a);
}

template <int BT>
static cudaError_t dispatch_bt(const GemvArgs& a, cudaStream_t st) {
  const int words = a.d_in / 32;
  if (words % 4 == 0) {
    const int segs = words / 4;
    switch (segs) {
      case 2: return launch_fast<2, 1, BT>(a, st);
      case 4: return launch_fast<4, 1, BT>(a, st);
      case 8: return launch_fast<8, 1, BT>(a, st);
      case 16: return launch_fast<16, 1, BT>(a, st);
      case 32: return launch_fast<32, 1, BT>(a, st);
      case 64: return launch_fast<32, 2, BT>(a, st);
      default: break;
    }
  }
  return launch_generic<BT>(a, st);
}

cudaError_t launch_gemv(const GemvArgs& a, cudaStream_t st) {
  if (a.B <= 1) return dispatch_bt<1>(a, st);
  if (a.B <= 4) return dispatch_bt<4>(a, st);
  return dispatch_bt<16>(a, st);
}

}  // namespace dfssm
