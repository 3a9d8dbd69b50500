// Streaming decode of DF-SSM linears that share one input (gist.science technical summary of DF-SSM,
// §2.B "Frozen Scaffold with LoRA Correction" and §2.C "Optimized Inference Pipeline": the scaffold
// matmul on 1-bit packed weights with int8 activations and int32 accumulation, plus the int8 LoRA).
//
// At batch <= 16 the scaffold product is a matrix-vector product (ALU-bound beyond a few tokens), so
// one persistent, warp-specialised kernel does everything for any number of linears that read the same x:
//   * the rows of all linears are cut into tiles of packed bits (16 KB; 32 KB at one token slot when the
//     launch has more 16 KB tiles than SMs); each CTA takes a contiguous range of tiles.  A producer warp
//     streams every tile into a ring of shared-memory stages and its rows' W_A
//     and scales into a second ring, with bulk asynchronous copies (cp.async.bulk, completion counted on
//     mbarriers), several tiles ahead, and copies each linear's W_B ahead of that linear's first tile;
//     a bits stage is refilled as soon as the GEMV warps have read it, a parameter stage once its
//     epilogue is done;
//   * sixteen GEMV warps quantize x (per-token absmax int8, codes in the dp4a-permuted,
//     bank-conflict-free segment layout and in natural order; at batch 1 each lane keeps its segment's
//     codes in registers), compute each linear's LoRA-down t = W_B q (exact int32, dp4a) and
//     tf = fl32(t sB s), and turn every stage into int32 accumulators
//     acc = 2 sum_{bit=1} q - sum q (one AND and one dp4a per four weights);
//   * up to six epilogue warps (never more than ring stages) turn each stage's accumulators into
//     y = fl32(acc s sW + sA sum_r W_A tf) (the fp64 epilogue shared by every path) while the GEMV warps
//     already work on the next stages, and release the stage to the producer.
// Template parameters: LPR lanes per row and NSEG 16-byte segments per lane (d_in = 128 LPR NSEG), BT
// token slots (1, 4 or 16), TB tile bytes.
// The linear descriptors are copied into shared memory at the start, so the hot loops never index the
// kernel's parameter block with a run-time index.
// The sign bits are immutable weights, so the producer starts streaming before the kernel waits on the
// preceding kernel of the stream (programmatic dependent launch).
//
// Every mbarrier wait is bounded.  A wait that runs out of budget stores a timeout code in the call's
// status word (the first word of its workspace; read and cleared by dfssm_device_status); the CTA then
// stops computing, still waits (bounded) for every copy it issued, and returns.

#include "common.cuh"
#include "internal.h"

namespace dfssm {
namespace stream {

constexpr int NCW = 16;                  // GEMV warps
constexpr int NEW = 6;                   // epilogue warps
constexpr int PROD_WARP = NCW + NEW;     // producer warp
constexpr int NT = (NCW + NEW + 1) * 32;
// Packed bits per tile (tb): 16 KB, or 32 KB with one token slot when a launch has more tiles than SMs
// (half the per-tile hand-offs per byte; more token slots need the shared memory for their codes).
constexpr int MAX_TR = 256;              // rows per tile (d_in >= 1024)
constexpr int MAX_B = 16;
constexpr int R = DFSSM_MAX_RANK;
constexpr int MAX_NS = 8;                // stages per ring (bits ring and parameter ring alike)
// Permuted codes of one token in shared memory: eight rows of 16-byte chunks (row v holds chunk v of every
// 128-input segment, in segment order) plus one pad chunk per row.  A GEMV lane that owns segment seg reads
// row v at chunk seg (consecutive lanes, consecutive chunks); the pad puts the eight chunks of one segment
// (written together by the quantizer) in eight different bank groups.
__host__ __device__ constexpr int q_row(int segs) { return segs + 1; }        // chunks per row
__host__ __device__ constexpr int q_tok(int segs) { return 8 * q_row(segs); }  // chunks per token
__host__ __device__ constexpr int q_tok_bytes(int din) { return 16 * q_tok(din / 128); }
// Byte offset, within a token, of natural input index i.
template <int SEGS>
__device__ __forceinline__ int q_index(int i) {
  const int seg = i >> 7;
  const int pos = perm_index(i) & 127;
  return ((pos >> 4) * q_row(SEGS) + seg) * 16 + (pos & 15);
}
// Parameter stage of a tile of tr rows for bt token slots: W_A rows (16 B each), sW and sA (4 B each) by
// bulk copy, then the int32 accumulators [bt][tr] and the LoRA intermediates [bt][16] (fp64) written by the
// GEMV warps.  Every offset is a multiple of 16 bytes for tr >= 16.
struct PLayout {
  int sw, sa, acc, tf, bytes;
};
__host__ __device__ constexpr int rows_per_tile(int din, int tb) { return tb / (din / 8); }
__host__ __device__ constexpr PLayout p_layout(int din, int bt, int tb) {
  return PLayout{rows_per_tile(din, tb) * 16, rows_per_tile(din, tb) * 20, rows_per_tile(din, tb) * 24,
                 rows_per_tile(din, tb) * 24 + rows_per_tile(din, tb) * bt * 4,
                 rows_per_tile(din, tb) * 24 + rows_per_tile(din, tb) * bt * 4 + bt * R * 8};
}
constexpr int MAX_LIN = DFSSM_MAX_LAYERS;
constexpr long long kWaitBudget = 2000000000LL;  // clock cycles per wait (~1 s)
constexpr int kTimeoutCode = kDeviceTimeout;

struct Lin {
  const uint32_t* bits;
  const float* w_scale;
  const int8_t* lora_b;
  const float* lora_b_scale;
  const int8_t* lora_a;
  const float* lora_a_scale;
  float* y;        // [B][d_out]
  int d_out;
  int rank;
  int tile0;       // index of this linear's first tile in the global tile list
  int ntiles;
  int ptma;        // set on the device: the per-row parameters may travel with the bits (bulk copy)
};

struct Params {
  // per linear, for the tensor-core path (several token slots): the sign bits as a 2-D tensor
  // [d_out][d_in / 8 bytes], loaded as boxes of 128 bytes x TR rows with the 128-byte swizzle
  CUtensorMap tmap[MAX_LIN];
  Lin lin[MAX_LIN];
  int n_lin;
  int d_in;
  int B;
  const float* x;  // [B][d_in]
  int total_tiles;
  int tile_rows;
  // optional taps (single linear only): codes, scales, LoRA-down t, scaffold accumulators
  int8_t* dbg_xq;
  float* dbg_s;
  int32_t* dbg_t;
  int32_t* dbg_acc;
  int* status;
};

// ------------------------------------------------------------------------------ mbarrier / bulk copy

// acc += A(16 x 32, u8, row-major) * B(32 x 8, s8, column-major), int32 (the warp-wide legacy MMA).
__device__ __forceinline__ void mma_u8s8(int (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k32.row.col.s32.u8.s8.s32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return (uint32_t)__cvta_generic_to_shared(p);
}
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
               : "memory");
}
// One 2-D TMA box (coordinates: byte column c0, row c1) into shared memory, completion on bar.
__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, int c0, int c1, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], "
      "[%4];" ::"r"(smem_u32(dst)),
      "l"(map), "r"(c0), "r"(c1), "r"(smem_u32(bar))
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
// Bounded wait for the completion of the phase with the given parity.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity) {
  if (mbar_try_wait(bar, parity)) return true;
  const long long t0 = clock64();
  while (!mbar_try_wait(bar, parity))
    if (clock64() - t0 > kWaitBudget) return false;
  return true;
}
// Bulk copy of `bytes` (multiple of 16; both addresses 16-byte aligned) from global to shared memory,
// completion counted on `bar`.
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}
// Named barrier over the GEMV warps only.
__device__ __forceinline__ void consumer_sync() {
  asm volatile("bar.sync 1, %0;" ::"n"(NCW * 32) : "memory");
}

// Bounded wait that also gives up once another role has aborted.
__device__ __forceinline__ bool mbar_wait_or_abort(uint64_t* bar, uint32_t parity, volatile int* abort_flag) {
  if (mbar_try_wait(bar, parity)) return true;
  const long long t0 = clock64();
  while (!mbar_try_wait(bar, parity)) {
    if (*abort_flag) return false;
    if (clock64() - t0 > kWaitBudget) return false;
  }
  return true;
}

// One L2 prefetch per 128-byte line of [p, p + bytes), spread over n threads (this one is idx).
__device__ __forceinline__ void prefetch_range(const void* p, size_t bytes, int idx, int n) {
  const uintptr_t a0 = reinterpret_cast<uintptr_t>(p) & ~uintptr_t(127);
  const uintptr_t e = reinterpret_cast<uintptr_t>(p) + bytes;
  for (uintptr_t a = a0 + (uintptr_t)idx * 128; a < e; a += (uintptr_t)n * 128)
    asm volatile("prefetch.global.L2 [%0];" ::"l"(a) : "memory");
}

// Dynamic shared memory: the bits ring, the parameter ring (ns stages each), W_B of the current linear
// when it fits, and the codes in both layouts.  W_B in shared memory is preferred (it takes the LoRA-down
// off global-memory latency) as long as ~96 KB of bits stay in flight; then the largest stage count <= 8.
constexpr size_t kSmemBudget = 214 * 1024;  // 1 KB is kept for aligning the tile ring to 1 KB
// Token stride of the permuted codes: with several token slots (tensor-core path) each token is padded by
// 16 bytes, so that the eight tokens of an MMA column block fall into different shared-memory banks.
__host__ __device__ constexpr int q_tok_stride(int din, int bt) { return q_tok_bytes(din) + (bt > 1 ? 16 : 0); }
__host__ __device__ constexpr size_t base_smem(int din, int bt, int ns, int tb) {
  return (size_t)ns * (tb + p_layout(din, bt, tb).bytes) + (size_t)bt * (q_tok_stride(din, bt) + din);
}
__host__ __device__ constexpr bool fits(int din, int bt, int ns, bool wb, int tb) {
  return base_smem(din, bt, ns, tb) + (wb ? (size_t)R * din : 0) <= kSmemBudget;
}
// W_B stays in shared memory if at least ~96 KB of sign bits remain in flight beside it
__host__ __device__ constexpr bool wb_in_smem(int din, int bt, int tb) {
  return fits(din, bt, tb >= 32768 ? 4 : 6, true, tb);
}
__host__ __device__ constexpr int n_stages(int din, int bt, int tb) {
  return fits(din, bt, 8, wb_in_smem(din, bt, tb), tb)   ? 8
         : fits(din, bt, 7, wb_in_smem(din, bt, tb), tb) ? 7
         : fits(din, bt, 6, wb_in_smem(din, bt, tb), tb) ? 6
         : fits(din, bt, 5, wb_in_smem(din, bt, tb), tb) ? 5
                                                         : 4;
}
__host__ __device__ constexpr size_t smem_bytes(int din, int bt, int tb) {
  return base_smem(din, bt, n_stages(din, bt, tb), tb) + (wb_in_smem(din, bt, tb) ? (size_t)R * din : 0) +
         1024;
}

// Position in the CTA's contiguous tile range: linear j, tile t of that linear.
struct Cursor {
  int j, t;
  __device__ __forceinline__ void start(const Lin* L, int n, int k) {
    j = 0;
    while (j + 1 < n && L[j + 1].tile0 <= k) ++j;
    t = k - L[j].tile0;
  }
  __device__ __forceinline__ void next(const Lin* L) {
    if (++t == L[j].ntiles) {
      ++j;
      t = 0;
    }
  }
};

// W_A row of one output row as 16 bytes (zero beyond rank).
__device__ __forceinline__ uint4 load_wa(const Lin& L, int row) {
  if (L.rank == R) return __ldg(reinterpret_cast<const uint4*>(L.lora_a + (size_t)row * R));
  uint32_t w[4] = {0u, 0u, 0u, 0u};
  for (int r = 0; r < L.rank; ++r)
    w[r >> 2] |= (uint32_t)(uint8_t)L.lora_a[(size_t)row * L.rank + r] << (8 * (r & 3));
  return make_uint4(w[0], w[1], w[2], w[3]);
}

// 128 x (sum over bit=1 positions of q) for 128 weights against BT tokens' permuted codes of one segment:
// token b's chunk v is q0[b * q_tok(SEGS) + v * q_row(SEGS)].
template <int SEGS, int BT>
__device__ __forceinline__ void bits_dot_tokens(uint4 w, const uint4* q0, int B, int (&S)[BT]) {
  constexpr int DIN16 = q_tok(SEGS);  // 16-byte chunks per token, pads included
  const uint32_t w4[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
  for (int b = 0; b < BT; ++b) {
    if (b < B) {
      const uint4* qp4 = q0 + b * DIN16;
      int acc8[8];
#pragma unroll
      for (int k = 0; k < 8; ++k) acc8[k] = 0;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const uint4 qa = qp4[(2 * j) * q_row(SEGS)], qb = qp4[(2 * j + 1) * q_row(SEGS)];
        const uint32_t qp[8] = {qa.x, qa.y, qa.z, qa.w, qb.x, qb.y, qb.z, qb.w};
#pragma unroll
        for (int k = 0; k < 8; ++k) acc8[k] = dp4a_us(w4[j] & (0x01010101u << k), qp[k], acc8[k]);
      }
      // acc8[k] = 2^k X_k exactly; sum_k acc8[k] 2^(7-k) = 128 sum_k X_k (multiply-adds, no shifts)
#pragma unroll
      for (int k = 0; k < 8; ++k) S[b] += acc8[k] * (1 << (7 - k));
    }
  }
}

// Same (128 x the sum) for one token whose eight code chunks of the segment are held in registers.
__device__ __forceinline__ int bits_dot_regs(uint4 w, const uint4 (&q)[8]) {
  const uint32_t w4[4] = {w.x, w.y, w.z, w.w};
  int acc8[8];
#pragma unroll
  for (int k = 0; k < 8; ++k) acc8[k] = 0;
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const uint4 qa = q[2 * j], qb = q[2 * j + 1];
    const uint32_t qp[8] = {qa.x, qa.y, qa.z, qa.w, qb.x, qb.y, qb.z, qb.w};
#pragma unroll
    for (int k = 0; k < 8; ++k) acc8[k] = dp4a_us(w4[j] & (0x01010101u << k), qp[k], acc8[k]);
  }
  int S = 0;
#pragma unroll
  for (int k = 0; k < 8; ++k) S += acc8[k] * (1 << (7 - k));
  return S;
}

// Row sums of P passes held by the LPR lanes of a row group (each lane one partial per pass): after the
// call, lane li holds the full sum of pass pass_of(li).  Each butterfly stage sends the half of the
// passes that the partner keeps, so P passes cost log2(P) extra values instead of P full reductions.
template <int P, int LPR>
__device__ __forceinline__ int pass_of(int li) {
  if constexpr (P == 1) return 0;
  else if constexpr (P == 2) return (li & (LPR / 2)) ? 1 : 0;
  else return ((li & (LPR / 2)) ? 2 : 0) + ((li & (LPR / 4)) ? 1 : 0);
}
template <int P, int LPR>
__device__ __forceinline__ int reduce_passes(const int (&S)[P], int li) {
  static_assert(P == 1 || P == 2 || P == 4, "one, two or four passes");
  static_assert(LPR >= 2 * P, "row group too small");
  int v;
  if constexpr (P == 1) {
    v = S[0];
  } else if constexpr (P == 2) {
    const bool hi = (li & (LPR / 2)) != 0;
    v = (hi ? S[1] : S[0]) + __shfl_xor_sync(0xffffffffu, hi ? S[0] : S[1], LPR / 2);
  } else {
    const bool hi = (li & (LPR / 2)) != 0;
    const int t0 = (hi ? S[2] : S[0]) + __shfl_xor_sync(0xffffffffu, hi ? S[0] : S[2], LPR / 2);
    const int t1 = (hi ? S[3] : S[1]) + __shfl_xor_sync(0xffffffffu, hi ? S[1] : S[3], LPR / 2);
    const bool hi2 = (li & (LPR / 4)) != 0;
    v = (hi2 ? t1 : t0) + __shfl_xor_sync(0xffffffffu, hi2 ? t0 : t1, LPR / 4);
  }
#pragma unroll
  for (int o = LPR / (2 * P); o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// LPR lanes per row, NSEG 16-byte segments per lane (d_in = 128 LPR NSEG >= 1024), BT token slots, TB
// bytes of sign bits per tile.  Warps 0..15 quantize x, compute the LoRA-down at each linear and accumulate
// the scaffold rows of every stage into the accumulator ring; warps 16..21 (the first NEP of them) turn
// accumulators into outputs (fp64 epilogue); warp 22 streams the stages.
template <int LPR, int NSEG, int BT, int TB>
__global__ void __launch_bounds__(NT, 1) stream_kernel(const __grid_constant__ Params p) {
  constexpr int SEGS = LPR * NSEG;
  constexpr int DIN = 128 * SEGS;
  constexpr int ROW16 = DIN / 128;             // 16-byte chunks of packed bits per row
  constexpr int RPW = 32 / LPR;                // rows per warp per pass
  constexpr int RPP = NCW * RPW;               // rows per pass
  constexpr int TILE_BYTES = TB;
  constexpr int TR = rows_per_tile(DIN, TB);  // rows per tile
  constexpr PLayout PL = p_layout(DIN, BT, TB);
  constexpr int PASSES = TR / RPP;
  static_assert(PASSES >= 1 && PASSES * RPP == TR && TR <= MAX_TR, "tile shape");
  constexpr bool WB_SMEM = wb_in_smem(DIN, BT, TB);
  constexpr int NS = n_stages(DIN, BT, TB);
  constexpr int XPT = DIN / (NCW * 32);                    // x values per GEMV thread per token
  constexpr bool XREG = BT * XPT <= 16;                    // keep x in registers between the two passes
  constexpr bool REGQ = BT == 1 && NSEG == 1;              // one token: the lane's codes live in registers
  // several token slots: the scaffold product on the int8 MMA (0/1 sign masks x codes), the tiles loaded by
  // TMA with the 128-byte swizzle; warp w takes rows [16 (w / KS), +16) x segments [SEGW (w % KS), +SEGW)
  constexpr bool MMA = BT > 1;
  constexpr int MB = TR / 16, KS = MMA ? NCW / MB : 1, SEGW = SEGS / KS, NB = (BT + 7) / 8;
  static_assert(!MMA || (MB * KS == NCW && KS * SEGW == SEGS && DIN % 1024 == 0), "MMA tile split");
  constexpr int QTS = q_tok_stride(DIN, BT);
  // Epilogue warps in use.  Warp e takes every NEP-th tile, so it waits on a stage's barriers at most one
  // phase ahead of the last completed one only if NEP <= NS (an mbarrier parity wait cannot tell phase n
  // from phase n - 2).
  constexpr int NEP = NEW < NS ? NEW : NS;

  extern __shared__ __align__(1024) unsigned char smem_raw[];
  // the tile ring starts on a 1 KB boundary (the 128-byte swizzle of the TMA path repeats every 1 KB),
  // reached by an offset from the array itself so that every access stays a shared-memory access
  unsigned char* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  unsigned char* pring = smem + (size_t)NS * TILE_BYTES;                            // [NS][PL.bytes]
  int8_t* wb_sm = reinterpret_cast<int8_t*>(pring + (size_t)NS * PL.bytes);         // [R][DIN] if WB_SMEM
  constexpr int QTB = q_tok_bytes(DIN);                                             // permuted token bytes
  int8_t* q_perm = wb_sm + (WB_SMEM ? R * DIN : 0);                                 // [BT][QTB]
  int8_t* q_nat = q_perm + BT * QTS;                                                // [BT][DIN]
  __shared__ Lin lin_sm[MAX_LIN];
  __shared__ uint64_t bfull[MAX_NS], bempty[MAX_NS], pfull[MAX_NS], pacc[MAX_NS], pempty[MAX_NS], wb_full,
      wb_empty;
  __shared__ float s_tok[MAX_B];
  __shared__ double s_tokd[MAX_B];
  __shared__ double tf_cur[MAX_B][R];
  __shared__ int t_sm[MAX_B][R];
  __shared__ float red_f[NCW][MAX_B];
  __shared__ int red_i[NCW][MAX_B];
  __shared__ int s_sumq[MAX_B];
  __shared__ volatile int abort_flag;
  __shared__ int wb_ok;

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int G = gridDim.x, c = blockIdx.x;
  const int k0 = (int)((long long)c * p.total_tiles / G);
  const int k1 = (int)((long long)(c + 1) * p.total_tiles / G);
  const int ntiles = k1 - k0;
  const int B = p.B;
  // fewer tiles than epilogue warps: every epilogue warp takes a share of every tile instead of whole tiles
  const bool epi_split = ntiles < NEP;

  if (tid < p.n_lin) {
    Lin L = p.lin[tid];
    const auto al16 = [](const void* q) { return (reinterpret_cast<uintptr_t>(q) & 15) == 0; };
    L.ptma = L.rank == R && al16(L.lora_a) && al16(L.w_scale) && al16(L.lora_a_scale);
    lin_sm[tid] = L;
  }
  if (tid == 0) {
    for (int s = 0; s < NS; ++s) {
      mbar_init(&bfull[s], 1);
      mbar_init(&bempty[s], NCW);
      mbar_init(&pfull[s], 1);
      mbar_init(&pacc[s], NCW);
      mbar_init(&pempty[s], epi_split ? NEP : 1);
    }
    mbar_init(&wb_full, 1);
    mbar_init(&wb_empty, 1);
    abort_flag = 0;
    int ok = WB_SMEM ? 1 : 0;
    for (int j = 0; j < p.n_lin; ++j)
      if (p.lin[j].rank > 0 && (reinterpret_cast<uintptr_t>(p.lin[j].lora_b) & 15)) ok = 0;
    wb_ok = ok;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if constexpr (MMA) {
    for (int s2 = 0; s2 < NS; ++s2) {
      int* acc0 = reinterpret_cast<int*>(pring + (size_t)s2 * PL.bytes + PL.acc);
      for (int k = tid; k < TR * BT; k += NT) acc0[k] = 0;
    }
  }
  __syncthreads();
  pdl_launch_dependents();
  const bool use_wb = wb_ok != 0;
  if (ntiles <= 0) return;

  // ------------------------------------------------------------------ producer warp
  // lane l < NS owns stage l of both rings and issues tiles l, l + NS, ... of the range (one warp
  // instruction issues the copies of several stages); lane 31 streams the linears' W_B; the remaining
  // lanes warm L2 with the parameters that do not travel by bulk copy.
  if (warp == PROD_WARP) {
    // the W_B copies (lane 31): the first one goes into the copy queue ahead of every tile
    Cursor wa, wz;
    wa.start(lin_sm, p.n_lin, k0);
    wz.start(lin_sm, p.n_lin, k1 - 1);
    int wj = wa.j, wm = 0;
    bool wok = true;
    const auto issue_wb = [&]() {  // next linear of the range with a LoRA; false when none is left
      while (wj <= wz.j && lin_sm[wj].rank == 0) ++wj;
      if (wj > wz.j) return false;
      if (wm > 0 && !mbar_wait_or_abort(&wb_empty, (wm - 1) & 1, &abort_flag)) {
        wok = false;
        return false;
      }
      const Lin& L = lin_sm[wj];
      mbar_expect_tx(&wb_full, (uint32_t)(L.rank * DIN));
      bulk_g2s(wb_sm, L.lora_b, (uint32_t)(L.rank * DIN), &wb_full);
      ++wm;
      ++wj;
      return true;
    };
    if (use_wb && lane == 31) issue_wb();
    __syncwarp();
    if (lane < NS) {
      const int sl = lane;
      Cursor cu;
      cu.start(lin_sm, p.n_lin, min(k0 + sl, k1 - 1));
      int i = sl;
      bool ok = true;
      for (; i < ntiles; i += NS) {
        if (i > sl)
          for (int q = 0; q < NS; ++q) cu.next(lin_sm);
        const Lin& L = lin_sm[cu.j];
        const uint32_t par = ((i / NS) & 1) ^ 1;
        if ((i >= NS && (!mbar_wait_or_abort(&bempty[sl], par, &abort_flag) ||
                         !mbar_wait_or_abort(&pempty[sl], par, &abort_flag))) || abort_flag) {
          ok = false;
          break;
        }
        const int r0 = cu.t * TR, nr = min(TR, L.d_out - r0), n4 = nr & ~3;
        if constexpr (MMA) {
          // DIN / 1024 boxes of TR rows x 128 bytes (rows past d_out arrive as zeros)
          mbar_expect_tx(&bfull[sl], (uint32_t)(TR * (DIN / 8)));
#pragma unroll
          for (int h = 0; h < DIN / 1024; ++h)
            tma_load_2d(smem + (size_t)sl * TILE_BYTES + h * TR * 128, &p.tmap[cu.j], h * 128, r0, &bfull[sl]);
        } else {
          const uint32_t bits_bytes = (uint32_t)nr * (DIN / 8);
          mbar_expect_tx(&bfull[sl], bits_bytes);
          bulk_g2s(smem + (size_t)sl * TILE_BYTES, L.bits + (size_t)r0 * (DIN / 32), bits_bytes, &bfull[sl]);
        }
        unsigned char* ps = pring + (size_t)sl * PL.bytes;
        mbar_expect_tx(&pfull[sl], L.ptma ? (uint32_t)(nr * 16 + 2 * n4 * 4) : 0u);
        if (L.ptma) {
          bulk_g2s(ps, L.lora_a + (size_t)r0 * R, (uint32_t)(nr * 16), &pfull[sl]);
          if (n4 > 0) {
            bulk_g2s(ps + PL.sw, L.w_scale + r0, (uint32_t)(n4 * 4), &pfull[sl]);
            bulk_g2s(ps + PL.sa, L.lora_a_scale + r0, (uint32_t)(n4 * 4), &pfull[sl]);
          }
        }
      }
      if (!ok) {
        // stop: record the failure and wait (bounded) for this stage's copies still in flight
        atomicExch(p.status, kTimeoutCode);
        abort_flag = 1;
        if (i - NS >= 0) {
          mbar_wait(&bfull[sl], ((i - NS) / NS) & 1);
          mbar_wait(&pfull[sl], ((i - NS) / NS) & 1);
        }
      }
    } else if (lane == 31) {
      if (!use_wb) return;
      // the following linears' W_B, in order; the GEMV warps release the buffer after computing t of
      // the previous one
      while (wok && !abort_flag && issue_wb()) {
      }
      if (!wok) {
        atomicExch(p.status, kTimeoutCode);
        abort_flag = 1;
      }
      if (!wok || abort_flag)
        if (wm > 0) mbar_wait(&wb_full, (wm - 1) & 1);
    } else {
      Cursor a, b;
      a.start(lin_sm, p.n_lin, k0);
      b.start(lin_sm, p.n_lin, k1 - 1);
      const int idx = lane - NS, nl = 31 - NS;
      for (int j = a.j; j <= b.j; ++j) {
        const Lin& L = lin_sm[j];
        const int ra = j == a.j ? a.t * TR : 0;
        const int rb = j == b.j ? min(L.d_out, (b.t + 1) * TR) : L.d_out;
        if (L.rank > 0) prefetch_range(L.lora_b_scale, (size_t)L.rank * 4, idx, nl);
        if (!use_wb && L.rank > 0) prefetch_range(L.lora_b, (size_t)L.rank * DIN, idx, nl);
        if (rb > ra && !L.ptma) {
          prefetch_range(L.w_scale + ra, (size_t)(rb - ra) * 4, idx, nl);
          if (L.rank > 0) {
            prefetch_range(L.lora_a_scale + ra, (size_t)(rb - ra) * 4, idx, nl);
            prefetch_range(L.lora_a + (size_t)ra * L.rank, (size_t)(rb - ra) * L.rank, idx, nl);
          }
        }
      }
    }
    return;
  }

  // ------------------------------------------------------------------ epilogue warps
  // epilogue warp e takes the tiles i = e, e + NEP, ... of the range, whole, so several tiles' fp64
  // epilogues are in flight at once; with fewer tiles than warps each warp takes a share of every tile
  if (warp >= NCW) {
    const int e = warp - NCW;
    if (e >= NEP) return;
    pdl_wait();  // the outputs may still be read or written by the preceding kernel of the stream
    Cursor cu;
    cu.start(lin_sm, p.n_lin, k0);
    bool dead = false;
    for (int i = 0; i < ntiles; ++i, cu.next(lin_sm)) {
      if (!epi_split && i % NEP != e) continue;
      const Lin& L = lin_sm[cu.j];
      const int sp = i % NS;
      const uint32_t par = (i / NS) & 1;
      if (!dead && (!mbar_wait_or_abort(&pacc[sp], par, &abort_flag) ||
                    !mbar_wait_or_abort(&pfull[sp], par, &abort_flag))) {
        dead = true;
        atomicExch(p.status, kTimeoutCode);
        abort_flag = 1;
      }
      if (!dead) {
        const int r0 = cu.t * TR, nr = min(TR, L.d_out - r0), n4 = nr & ~3;
        const unsigned char* ps = pring + (size_t)sp * PL.bytes;
        const uint4* wa_st = reinterpret_cast<const uint4*>(ps);
        const float* sw_st = reinterpret_cast<const float*>(ps + PL.sw);
        const float* sa_st = reinterpret_cast<const float*>(ps + PL.sa);
        int* acc = reinterpret_cast<int*>(const_cast<unsigned char*>(ps) + PL.acc);
        const double* tf = reinterpret_cast<const double*>(ps + PL.tf);
        // the row's parameters: W_A bytes, sW, sA (stage copy, or global memory past the copied rows)
        const auto row_params = [&](int rr, uint4& wa, float& fw, float& fa) {
          const int row = r0 + rr;
          fa = 0.0f;
          wa = make_uint4(0u, 0u, 0u, 0u);
          if (L.ptma) {
            wa = wa_st[rr];
            if (rr < n4) {
              fw = sw_st[rr];
              fa = sa_st[rr];
            } else {
              fw = __ldg(L.w_scale + row);
              fa = __ldg(L.lora_a_scale + row);
            }
          } else {
            fw = __ldg(L.w_scale + row);
            if (L.rank > 0) {
              fa = __ldg(L.lora_a_scale + row);
              wa = load_wa(L, row);
            }
          }
        };
        if constexpr (MMA) {
          // lane = row: sW and sA are converted once per row and shared by every token; four tokens' LoRA
          // chains run interleaved, each W_A entry reaching fp64 once per four tokens, the tf rows read as
          // broadcasts
          const int rstart = (epi_split ? e * 32 : 0) + lane, rstride = epi_split ? NEP * 32 : 32;
          const int rk = L.rank;
          for (int rr = rstart; rr < nr; rr += rstride) {
            uint4 wa;
            float fw, fa;
            row_params(rr, wa, fw, fa);
            const double sw = (double)fw, sa = (double)fa;
            const uint32_t w4[4] = {wa.x, wa.y, wa.z, wa.w};
            const int row = r0 + rr;
            for (int b0 = 0; b0 < B; b0 += 4) {
              double lora[4] = {0.0, 0.0, 0.0, 0.0};
              if (rk == R) {
#pragma unroll 2
                for (int r = 0; r < R; r += 2) {
                  const double w0 = int_to_f64((int)(int8_t)(w4[r >> 2] >> (8 * (r & 3))));
                  const double w1 = int_to_f64((int)(int8_t)(w4[r >> 2] >> (8 * ((r + 1) & 3))));
#pragma unroll
                  for (int k = 0; k < 4; ++k) {
                    const double2 t = *reinterpret_cast<const double2*>(tf + (b0 + k) * R + r);
                    lora[k] = fma(w0, t.x, lora[k]);
                    lora[k] = fma(w1, t.y, lora[k]);
                  }
                }
              } else {
#pragma unroll
                for (int r = 0; r < R; ++r)
                  if (r < rk) {
                    const double w = int_to_f64((int)(int8_t)(w4[r >> 2] >> (8 * (r & 3))));
#pragma unroll
                    for (int k = 0; k < 4; ++k) lora[k] = fma(w, tf[(b0 + k) * R + r], lora[k]);
                  }
              }
#pragma unroll
              for (int k = 0; k < 4; ++k) {
                const int b = b0 + k;  // slots past B (inside BT, a multiple of 4) are read, never stored
                const int a = acc[b * TR + rr];
                acc[b * TR + rr] = 0;  // the next tile of this stage adds into zero
                const double scaffold = dmul(dmul(int_to_f64(a), s_tokd[b]), sw);
                const double corr = rk > 0 ? dmul(sa, lora[k]) : 0.0;
                if (b < B) {
                  L.y[(size_t)b * L.d_out + row] = __double2float_rn(dadd(scaffold, corr));
                  if (p.dbg_acc) p.dbg_acc[(size_t)b * L.d_out + row] = a;
                }
              }
            }
          }
        } else {
        // two (token, row) jobs per lane per step, their fp64 chains interleaved; consecutive lanes take
        // consecutive rows of one token (coalesced outputs, one broadcast tf row)
        const auto fetch = [&](int job, int& a, double& sw, double& sa, uint4& wa, int& row, int& b) {
          b = job / nr;
          const int rr = job - b * nr;
          row = r0 + rr;
          float fw, fa;
          row_params(rr, wa, fw, fa);
          sw = (double)fw;
          sa = (double)fa;
          a = acc[b * TR + rr];
        };
        const int jstride = epi_split ? NEP * 32 : 32;
        for (int job = (epi_split ? e * 32 : 0) + lane; job < nr * B; job += 2 * jstride) {
          int a[2], row[2], b[2];
          double sd[2], sw[2], sa[2];
          uint4 wa[2];
          const bool two = job + jstride < nr * B;
          fetch(job, a[0], sw[0], sa[0], wa[0], row[0], b[0]);
          fetch(two ? job + jstride : job, a[1], sw[1], sa[1], wa[1], row[1], b[1]);
          sd[0] = s_tokd[b[0]];
          sd[1] = s_tokd[b[1]];
          const double* const t2[2] = {tf + b[0] * R, tf + b[1] * R};
          float out[2];
          if (L.rank == R) linear_out_n<2, R>(a, sd, sw, sa, wa, t2, R, out);
          else linear_out_n<2, -1>(a, sd, sw, sa, wa, t2, L.rank, out);
#pragma unroll
          for (int n = 0; n < 2; ++n) {
            if (n == 0 || two) {
              L.y[(size_t)b[n] * L.d_out + row[n]] = out[n];
              if (p.dbg_acc) p.dbg_acc[(size_t)b[n] * L.d_out + row[n]] = a[n];
            }
          }
        }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&pempty[sp]);
    }
    return;
  }

  // ------------------------------------------------------------------ GEMV warps
  pdl_wait();  // x may come from the preceding kernel of the stream
  int sumq[BT];
  if constexpr (BT > 1) {
    // WPT warps per token slot, each over a contiguous slice of the token, 16-byte loads issued in
    // batches before any use: every CTA asks for all of x at once with many loads in flight, instead of
    // token by token.  The token of each slot is rotated by the CTA index, so that the CTAs do not all
    // ask for the same lines of x at the same moment.
    constexpr int WPT = NCW / BT;               // warps per token slot
    constexpr int CH = DIN / 4 / WPT;           // float4 per warp slice
    constexpr int U = CH / 32 < 8 ? CH / 32 : 8;  // loads in flight per lane
    static_assert(CH % (32 * U) == 0, "quantizer slice");
    const int slot = warp / WPT, part = warp % WPT;
    const bool active = slot < B;
    const int b = active ? (slot + c) % B : 0;
    const float4* xs = reinterpret_cast<const float4*>(p.x + (size_t)b * DIN) + part * CH;
    float m = 0.0f;
    if (active) {
#pragma unroll 1
      for (int v0 = lane; v0 < CH; v0 += 32 * U) {
        float4 t[U];
#pragma unroll
        for (int u = 0; u < U; ++u) t[u] = __ldg(xs + v0 + 32 * u);
#pragma unroll
        for (int u = 0; u < U; ++u)
          m = fmaxf(m, fmaxf(fmaxf(fabsf(t[u].x), fabsf(t[u].y)), fmaxf(fabsf(t[u].z), fabsf(t[u].w))));
      }
    }
    m = warp_max(m);
    if (lane == 0) red_f[warp][0] = m;
    consumer_sync();
    m = 0.0f;
#pragma unroll
    for (int j = 0; j < WPT; ++j) m = fmaxf(m, red_f[slot * WPT + j][0]);
    const float s0 = quant_scale(m);
    const float inv_s0 = quant_inv(s0);
    int sq = 0;
    if (active) {
#pragma unroll 1
      for (int v0 = lane; v0 < CH; v0 += 32 * U) {
        float4 t[U];
#pragma unroll
        for (int u = 0; u < U; ++u) t[u] = __ldg(xs + v0 + 32 * u);
        // codes two float4 at a time (one rarely taken branch per eight values)
#pragma unroll
        for (int u2 = 0; u2 < U; u2 += 2) {
          constexpr int G = U < 2 ? U : 2;
          float tv[4 * G];
#pragma unroll
          for (int g = 0; g < G; ++g) {
            tv[4 * g] = t[u2 + g].x;
            tv[4 * g + 1] = t[u2 + g].y;
            tv[4 * g + 2] = t[u2 + g].z;
            tv[4 * g + 3] = t[u2 + g].w;
          }
          int cd[4 * G];
          quant_codes<4 * G>(tv, s0, inv_s0, cd);
#pragma unroll
          for (int g = 0; g < G; ++g) {
            const int v = part * CH + v0 + 32 * (u2 + g);  // float4 index within the token
            uint32_t packed = 0u;
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              q_perm[b * QTS + q_index<SEGS>(4 * v + e)] = (int8_t)cd[4 * g + e];
              packed |= (uint32_t)(cd[4 * g + e] & 0xFF) << (8 * e);
              sq += cd[4 * g + e];
            }
            reinterpret_cast<uint32_t*>(q_nat + b * DIN)[v] = packed;
          }
        }
      }
    }
    sq = warp_sum(sq);
    if (lane == 0) red_i[warp][0] = sq;
    if (active && part == 0 && lane == 0) {
      s_tok[b] = s0;
      s_tokd[b] = (double)s0;
      if (p.dbg_s && c == 0) p.dbg_s[b] = s0;
    }
    consumer_sync();
    if (tid < B) {
      const int sl = ((tid - c) % B + B) % B;  // the slot that quantized token tid
      int t = 0;
#pragma unroll
      for (int j = 0; j < WPT; ++j) t += red_i[sl * WPT + j][0];
      s_sumq[tid] = t;
    }
    consumer_sync();
#pragma unroll
    for (int bb = 0; bb < BT; ++bb) sumq[bb] = bb < B ? s_sumq[bb] : 0;
  } else {
    float xr[XREG ? BT * XPT : 1];
#pragma unroll
    for (int b = 0; b < BT; ++b) {
      float m = 0.0f;
#pragma unroll
      for (int k = 0; k < XPT; ++k) {
        const int i = tid + k * NCW * 32;
        const float v = b < B ? __ldg(p.x + (size_t)b * DIN + i) : 0.0f;
        if (XREG) xr[b * XPT + k] = v;
        m = fmaxf(m, fabsf(v));
      }
      m = warp_max(m);
      if (lane == 0) red_f[warp][b] = m;
    }
    consumer_sync();
#pragma unroll
    for (int b = 0; b < BT; ++b) {
      float m = 0.0f;
#pragma unroll
      for (int w = 0; w < NCW; ++w) m = fmaxf(m, red_f[w][b]);
      const float s0 = quant_scale(m);
      const float inv_s0 = quant_inv(s0);
      int sq = 0;
      if (b < B) {
        float v[XPT];
#pragma unroll
        for (int k = 0; k < XPT; ++k)
          v[k] = XREG ? xr[b * XPT + k] : __ldg(p.x + (size_t)b * DIN + tid + k * NCW * 32);
        int cd[XPT];
        quant_codes<XPT>(v, s0, inv_s0, cd);
#pragma unroll
        for (int k = 0; k < XPT; ++k) {
          const int i = tid + k * NCW * 32;
          q_perm[b * QTS + q_index<SEGS>(i)] = (int8_t)cd[k];
          q_nat[b * DIN + i] = (int8_t)cd[k];
          sq += cd[k];
        }
      }
      sq = warp_sum(sq);
      if (lane == 0) red_i[warp][b] = sq;
      if (tid == b && b < B) {
        s_tok[b] = s0;
        s_tokd[b] = (double)s0;
        if (p.dbg_s && c == 0) p.dbg_s[b] = s0;
      }
    }
    consumer_sync();
#pragma unroll
    for (int b = 0; b < BT; ++b) {
      int sq = 0;
#pragma unroll
      for (int w = 0; w < NCW; ++w) sq += red_i[w][b];
      sumq[b] = sq;
      if (tid == b) s_sumq[b] = sq;
    }
  }

  if (p.dbg_xq && c == 0)  // debug tap: the natural-order codes (published by the last consumer_sync)
    for (int i = tid; i < B * DIN; i += NCW * 32) p.dbg_xq[i] = q_nat[i];
  const int li = lane % LPR, rsub = lane / LPR;
  uint4 qreg[REGQ ? 8 : 1];
  if (REGQ) {
    const uint4* q0 = reinterpret_cast<const uint4*>(q_perm) + li;
#pragma unroll
    for (int v = 0; v < 8; ++v) qreg[v] = q0[v * q_row(SEGS)];
  }
  Cursor cu;
  cu.start(lin_sm, p.n_lin, k0);
  int cur_j = -1, m_wb = 0;
  bool dead = false;
  for (int i = 0; i < ntiles; ++i, cu.next(lin_sm)) {
    const Lin& L = lin_sm[cu.j];
    if (cu.j != cur_j) {
      // LoRA down-projection of this linear for every token: warp r computes t[.][r]
      const float sB = (tid < BT * R && tid % R < L.rank) ? __ldg(L.lora_b_scale + tid % R) : 0.0f;
      if (L.rank > 0 && use_wb && !dead && !mbar_wait_or_abort(&wb_full, m_wb & 1, &abort_flag)) {
        dead = true;
        atomicExch(p.status, kTimeoutCode);
        abort_flag = 1;
      }
      consumer_sync();
      if (!dead) {
        for (int rw = warp; rw < L.rank; rw += NCW) {
          const int r = (rw + c) % L.rank;  // rotated by CTA: the CTAs read different W_B rows at a time
          int part[BT];
#pragma unroll
          for (int b = 0; b < BT; ++b) part[b] = 0;
          if (use_wb) {
            const uint4* w4 = reinterpret_cast<const uint4*>(wb_sm + r * DIN);
#pragma unroll
            for (int ch = lane; ch < DIN / 16; ch += 32) {
              const uint4 w = w4[ch];
              // every token slot, used or not (slots >= B read stale codes and are never stored): no
              // per-token branches in the unrolled loop
#pragma unroll
              for (int b = 0; b < BT; ++b) {
                const uint4 q = reinterpret_cast<const uint4*>(q_nat + b * DIN)[ch];
                part[b] = dp4a_ss(w.x, q.x, part[b]);
                part[b] = dp4a_ss(w.y, q.y, part[b]);
                part[b] = dp4a_ss(w.z, q.z, part[b]);
                part[b] = dp4a_ss(w.w, q.w, part[b]);
              }
            }
          } else {
            // eight words of the W_B row in flight per lane before they are used
            const uint32_t* wb = reinterpret_cast<const uint32_t*>(L.lora_b + (size_t)r * DIN);
#pragma unroll 1
            for (int w0 = lane; w0 < DIN / 4; w0 += 32 * 8) {  // DIN / 4 is a multiple of 256
              uint32_t wv[8];
#pragma unroll
              for (int u = 0; u < 8; ++u) wv[u] = __ldg(wb + w0 + 32 * u);
#pragma unroll
              for (int u = 0; u < 8; ++u)
#pragma unroll
                for (int b = 0; b < BT; ++b)  // every slot, as above
                  part[b] = dp4a_ss(wv[u], reinterpret_cast<const uint32_t*>(q_nat + b * DIN)[w0 + 32 * u], part[b]);
            }
          }
#pragma unroll
          for (int b = 0; b < BT; ++b) {
            part[b] = __reduce_add_sync(0xffffffffu, part[b]);
            if (lane == 0 && b < B) t_sm[b][r] = part[b];
          }
        }
      }
      consumer_sync();
      if (L.rank > 0 && use_wb) {
        if (tid == 0) mbar_arrive(&wb_empty);  // W_B buffer free for the next linear
        ++m_wb;
      }
      if (tid < BT * R) {
        const int b = tid / R, r = tid % R;
        float tf = 0.0f;
        if (b < B && r < L.rank) {
          tf = lora_tf(t_sm[b][r], sB, s_tok[b]);
          if (p.dbg_t && c == 0) p.dbg_t[b * L.rank + r] = t_sm[b][r];
        }
        tf_cur[b][r] = (double)tf;
      }
      consumer_sync();
      cur_j = cu.j;
    }
    const int sb = i % NS, sp = sb;
    if (!dead && !mbar_wait_or_abort(&bfull[sb], (i / NS) & 1, &abort_flag)) {
      dead = true;
      atomicExch(p.status, kTimeoutCode);
      abort_flag = 1;
    }
    if (!dead) {
      const uint4* tile = reinterpret_cast<const uint4*>(smem + (size_t)sb * TILE_BYTES);
      int* acc = reinterpret_cast<int*>(pring + (size_t)sp * PL.bytes + PL.acc);
      const int nr = min(TR, L.d_out - cu.t * TR);
      if constexpr (MMA) {
        // rows ra = 16 mb + g and ra + 8 of the tile, segments seg of this warp's k-slice; A = the 0/1 sign
        // masks of 32 inputs, k-ordered as the permuted codes (k = 4j + b <-> input 8b + j of the 32-input
        // block, so that mask word j is (w >> j) & 0x01010101 and code word j is word j of the block)
        const int mb = warp / KS, ks = warp % KS;
        const int g = lane >> 2, t = lane & 3;
        const int ra = mb * 16 + g, rb = ra + 8;
        const unsigned char* tl = reinterpret_cast<const unsigned char*>(tile);
        int cf[NB][4];
#pragma unroll
        for (int nb = 0; nb < NB; ++nb)
#pragma unroll
          for (int q = 0; q < 4; ++q) cf[nb][q] = 0;
        // this lane's token of each column block (slots past BT read the last slot: in bounds, not stored)
        const int8_t* qtok[NB];
#pragma unroll
        for (int nb = 0; nb < NB; ++nb) qtok[nb] = q_perm + min(nb * 8 + g, BT - 1) * QTS + 4 * t;
#pragma unroll
        for (int sgi = 0; sgi < SEGW; ++sgi) {
          const int seg = ks * SEGW + sgi;
          const int hb = (seg >> 3) * TR * 128, ch = seg & 7;
          const uint4 wa = *reinterpret_cast<const uint4*>(tl + hb + ra * 128 + ((ch ^ (ra & 7)) << 4));
          const uint4 wb = *reinterpret_cast<const uint4*>(tl + hb + rb * 128 + ((ch ^ (rb & 7)) << 4));
          const uint32_t w_a[4] = {wa.x, wa.y, wa.z, wa.w}, w_b[4] = {wb.x, wb.y, wb.z, wb.w};
#pragma unroll
          for (int kb = 0; kb < 4; ++kb) {
            const uint32_t af[4] = {(w_a[kb] >> t) & 0x01010101u, (w_b[kb] >> t) & 0x01010101u,
                                    (w_a[kb] >> (t + 4)) & 0x01010101u, (w_b[kb] >> (t + 4)) & 0x01010101u};
            const int o0 = ((2 * kb) * q_row(SEGS) + seg) * 16, o1 = o0 + q_row(SEGS) * 16;
#pragma unroll
            for (int nb = 0; nb < NB; ++nb)
              mma_u8s8(cf[nb], af, *reinterpret_cast<const uint32_t*>(qtok[nb] + o0),
                       *reinterpret_cast<const uint32_t*>(qtok[nb] + o1));
          }
        }
        // acc = 2 sum_{bit=1} q - sum q, summed over the KS k-slices in shared memory
#pragma unroll
        for (int nb = 0; nb < NB; ++nb) {
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const int row = q < 2 ? ra : rb, tok = nb * 8 + 2 * t + (q & 1);
            if (row < nr && tok < B)
              atomicAdd(acc + tok * TR + row, 2 * cf[nb][q] - (ks == 0 ? s_sumq[tok] : 0));
          }
        }
      } else {
        // one token: every pass's partial sum first, then one transposed reduction over the row group
        // (a few shuffles for all passes instead of a full reduction per pass)
        int Sp[PASSES];
#pragma unroll
        for (int ps = 0; ps < PASSES; ++ps) {
          const int rr = ps * RPP + warp * RPW + rsub;
          const bool valid = rr < nr;
          int Sv = 0;
#pragma unroll
          for (int sg = 0; sg < NSEG; ++sg) {
            const int seg = sg * LPR + li;
            const uint4 w = valid ? tile[rr * ROW16 + seg] : make_uint4(0u, 0u, 0u, 0u);
            if constexpr (REGQ) {
              Sv += bits_dot_regs(w, qreg);
            } else {
              int St[1] = {0};
              bits_dot_tokens<SEGS, 1>(w, reinterpret_cast<const uint4*>(q_perm) + seg, 1, St);
              Sv += St[0];
            }
          }
          Sp[ps] = Sv;
        }
        const int Sr = reduce_passes<PASSES, LPR>(Sp, li);
        const int rr = pass_of<PASSES, LPR>(li) * RPP + warp * RPW + rsub;
        if ((li & (LPR / PASSES - 1)) == 0 && rr < nr) acc[rr] = (Sr >> 6) - sumq[0];  // 2 sum - sum q
      }
      if (tid < BT * R)
        reinterpret_cast<double*>(pring + (size_t)sp * PL.bytes + PL.tf)[tid] = tf_cur[tid / R][tid % R];
    }
    __syncwarp();
    if (lane == 0) {
      mbar_arrive(&bempty[sb]);  // the bits stage may be refilled
      mbar_arrive(&pacc[sp]);    // accumulators and tf of this tile are ready
    }
  }
}


template <int LPR, int NSEG, int BT, int TB>
cudaError_t launch_t(const Params& p, int grid, cudaStream_t st) {
  constexpr int DIN = 128 * LPR * NSEG;
  constexpr size_t smem = smem_bytes(DIN, BT, TB);
  auto k = stream_kernel<LPR, NSEG, BT, TB>;
  const cudaError_t set = set_max_dynamic_smem(reinterpret_cast<const void*>(k), (int)smem);
  if (set != cudaSuccess) return set;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(NT);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, k, p);
}

template <int BT, int TB>
cudaError_t dispatch(const Params& p, int grid, cudaStream_t st) {
  switch (p.d_in / 128) {
    case 8: return launch_t<8, 1, BT, TB>(p, grid, st);
    case 16: return launch_t<16, 1, BT, TB>(p, grid, st);
    case 32: return launch_t<32, 1, BT, TB>(p, grid, st);
    case 64:
      if constexpr (BT <= 4) return launch_t<32, 2, BT, TB>(p, grid, st);
      return cudaErrorInvalidValue;
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace stream

bool stream_supported(int d_in, int B) {
  if (B < 1 || B > stream::MAX_B) return false;
  if (B <= 4) return d_in == 1024 || d_in == 2048 || d_in == 4096 || d_in == 8192;
  return d_in == 1024 || d_in == 2048 || d_in == 4096;  // 16 token slots of codes must fit beside the rings
}

int launch_linear_stream(const dfssm_linear_t* lins, int n, const float* x, int B, float* const* ys,
                         const dfssm_debug_t* dbg, int* status, cudaStream_t st) {
  stream::Params p;
  const int d_in = lins[0].d_in;
  // tile size: 32 KB with one token slot when 16 KB tiles would outnumber the SMs, else 16 KB
  int tiles16 = 0;
  for (int j = 0; j < n; ++j) tiles16 += (lins[j].d_out + stream::rows_per_tile(d_in, 16384) - 1) /
                                         stream::rows_per_tile(d_in, 16384);
  const int tb = (B == 1 && tiles16 > num_sms()) ? 32768 : 16384;
  const int tile_rows = stream::rows_per_tile(d_in, tb);
  int tiles = 0;
  for (int j = 0; j < n; ++j) {
    const dfssm_linear_t& L = lins[j];
    stream::Lin& q = p.lin[j];
    q.bits = L.bits;
    q.w_scale = L.w_scale;
    q.lora_b = L.lora_b;
    q.lora_b_scale = L.lora_b_scale;
    q.lora_a = L.lora_a;
    q.lora_a_scale = L.lora_a_scale;
    q.y = ys[j];
    q.d_out = L.d_out;
    q.rank = L.rank;
    q.tile0 = tiles;
    q.ntiles = (L.d_out + tile_rows - 1) / tile_rows;
    tiles += q.ntiles;
    // the tensor-core path (several token slots) loads the sign bits as swizzled 2-D boxes
    if (B > 1 && !encode_u8_map_sw128(&p.tmap[j], L.bits, L.d_out, d_in / 8, tile_rows))
      return DFSSM_EUNSUPPORTED;
  }
  p.n_lin = n;
  p.d_in = d_in;
  p.B = B;
  p.x = x;
  p.total_tiles = tiles;
  p.tile_rows = tile_rows;
  p.dbg_xq = dbg ? dbg->xq : nullptr;
  p.dbg_s = dbg ? dbg->xscale : nullptr;
  p.dbg_t = dbg ? dbg->lora_t : nullptr;
  p.dbg_acc = dbg ? dbg->acc : nullptr;
  p.status = status;
  const int grid = tiles < num_sms() ? tiles : num_sms();
  const cudaError_t e = B == 1   ? (tb == 32768 ? stream::dispatch<1, 32768>(p, grid, st)
                                                : stream::dispatch<1, 16384>(p, grid, st))
                        : B <= 4 ? stream::dispatch<4, 16384>(p, grid, st)
                                 : stream::dispatch<16, 16384>(p, grid, st);
  if (e != cudaSuccess) return record_cuda_failure(e);
  return DFSSM_OK;
}

}  // namespace dfssm
