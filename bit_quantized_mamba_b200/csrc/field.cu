// Density-field state representation (gist.science technical summary of DF-SSM, §2.D "Density Field
// State Representation": a binary field per state element with K^2 about 4 d_state cells, built by
// normalization, sigma-delta injection with error feedback and binarization, read back by popcount).
//
// One SSM state row S[0..N) becomes 4N cells, four per value, and its absmax c:
//   x_n = fl32(S_n / c) (0 when c = 0), d_n = fl32(x_n + 1) / 2, the cells j = 4n + k fed d_n in order
//   through a first-order sigma-delta modulator (v = d + e, b = [v >= 1/2], e = v - b, e = 0 at the row
//   start); cell j is bit j % 32 of word j / 32; the readout is c (popcount of value n's cells / 2 - 1).
//
// The modulator is a serial recurrence, but its output has a closed form: with P_j the exact sum of the
// densities of cells 0..j, the number of ones among them is floor(P_j + 1/2) (induction on j: each
// density is in [0, 1], so the count rises by at most one per cell and the threshold picks exactly when).
// Every density is a whole multiple of 2^-25 (fl32(x + 1) is a multiple of 2^-24 for |x| <= 1), so with
// densities as integers D_n = d_n 2^25 and Q_n = D_0 + ... + D_{n-1}, the ones among the first k cells of
// value n number floor((4 Q_n + k D_n + 2^24) / 2^25) - floor((4 Q_n + 2^24) / 2^25) = (lo + k D_n) >> 25
// with lo = (4 Q_n + 2^24) mod 2^25.  Only Q_n mod 2^23 enters lo, so the prefix sums run in wrapping
// 32-bit integers, exactly.  A row goes to LPR lanes (16 for N <= 128, two rows per warp; else 32): each
// lane its ceil(N / LPR) consecutive values, one scan over the row's lanes for the Q of its first value;
// no serial chain.  The readout kernel keeps one warp per row.  The state row is read once (and, for the
// round trip, written once), the field and scale written once.

#include <cstdint>
#include <cuda_runtime.h>

#include "dfssm.h"
#include "internal.h"

namespace dfssm {
namespace {

constexpr int kWarps = 8;                    // warps per CTA
constexpr unsigned kFull = 0xffffffffu;
constexpr float kUnits = 33554432.0f;        // 2^25
constexpr uint32_t kHalfUnit = 1u << 24;
constexpr uint32_t kUnitMask = (1u << 25) - 1u;

// Row groups a warp holds at once (the loads of all of them are issued before the first is processed); a
// group is one row, or two for the sixteen-lane split of the encoder.
template <int V>
constexpr int rows_per_warp() { return V <= 4 ? 4 : 2; }

// The values lane `lane` owns: [lane V, lane V + V) clipped to N.  With V % 4 == 0 (and N % 8 == 0) a
// lane's range is whole or empty and 16-byte aligned when the row is.
template <int V>
__device__ __forceinline__ void load_vals(const float* __restrict__ row, int N, int lane, float (&s)[V]) {
  const int v0 = lane * V;
  if constexpr (V % 4 == 0) {
    if (v0 < N) {
#pragma unroll
      for (int i = 0; i < V; i += 4) {
        const float4 t = __ldcs(reinterpret_cast<const float4*>(row + v0 + i));
        s[i] = t.x;
        s[i + 1] = t.y;
        s[i + 2] = t.z;
        s[i + 3] = t.w;
      }
    } else {
#pragma unroll
      for (int i = 0; i < V; ++i) s[i] = 0.0f;
    }
  } else {
#pragma unroll
    for (int i = 0; i < V; ++i) s[i] = v0 + i < N ? __ldcs(row + v0 + i) : 0.0f;
  }
}

template <int V>
__device__ __forceinline__ void store_vals(float* __restrict__ row, int N, int lane, const float (&y)[V]) {
  const int v0 = lane * V;
  if constexpr (V % 4 == 0) {
    if (v0 < N) {
#pragma unroll
      for (int i = 0; i < V; i += 4)
        __stcs(reinterpret_cast<float4*>(row + v0 + i), make_float4(y[i], y[i + 1], y[i + 2], y[i + 3]));
    }
  } else {
#pragma unroll
    for (int i = 0; i < V; ++i)
      if (v0 + i < N) __stcs(row + v0 + i, y[i]);
  }
}

// c (p / 2 - 1): p / 2 - 1 is exact, so this is the correctly rounded product of c and the level.
__device__ __forceinline__ float readout(float c, int p) {
  return __fmul_rn(c, __fadd_rn(__fmul_rn((float)p, 0.5f), -1.0f));
}

// Normalization and injection of one row held by LPR lanes (a whole warp, or one half): returns c (every
// lane of the row), the nibble of each of the lane's values (cell k of the value in bit k) and its
// popcount.  li = the lane's index within the row.
template <int V, int LPR>
__device__ __forceinline__ float encode_row(const float (&s)[V], int N, int li, uint32_t (&nib)[V],
                                            int (&pop)[V]) {
  float m = 0.0f;
#pragma unroll
  for (int i = 0; i < V; ++i) m = fmaxf(m, fabsf(s[i]));
  // non-negative floats order like their bit patterns
  uint32_t mb = __float_as_uint(m);
  if constexpr (LPR == 32) {
    mb = __reduce_max_sync(kFull, mb);
  } else {
#pragma unroll
    for (int o = LPR / 2; o > 0; o >>= 1) mb = max(mb, __shfl_xor_sync(kFull, mb, o));
  }
  const float c = __uint_as_float(mb);
  uint32_t D[V];
  uint32_t own = 0;
  const bool whole = V % 4 == 0 && li * V < N;  // with V % 4 == 0 a lane's range is whole or empty
#pragma unroll
  for (int i = 0; i < V; ++i) {
    const float x = c > 0.0f ? __fdiv_rn(s[i], c) : 0.0f;
    const float d = __fmul_rn(__fadd_rn(x, 1.0f), 0.5f);
    const bool in = V % 4 == 0 ? whole : li * V + i < N;
    D[i] = in ? __float2uint_rn(__fmul_rn(d, kUnits)) : 0u;  // exact: d 2^25 <= 2^25
    own += D[i];
  }
  uint32_t inc = own;  // inclusive scan over the row's lanes, modulo 2^32
#pragma unroll
  for (int o = 1; o < LPR; o <<= 1) {
    const uint32_t t = __shfl_up_sync(kFull, inc, o, LPR);
    if (li >= o) inc += t;
  }
  uint32_t q = inc - own;  // Q of the lane's first value, modulo 2^32
#pragma unroll
  for (int i = 0; i < V; ++i) {
    const uint32_t a1 = ((4u * q + kHalfUnit) & kUnitMask) + D[i];
    const uint32_t a2 = a1 + D[i], a3 = a2 + D[i], a4 = a3 + D[i];  // below 2^28
    const uint32_t t1 = a1 >> 25, t2 = a2 >> 25, t3 = a3 >> 25, t4 = a4 >> 25;
    // bit k is t_{k+1} - t_k (0 or 1), so the nibble is sum_k 2^k (t_{k+1} - t_k) = 8 t4 - 4 t3 - 2 t2 - t1
    nib[i] = 8u * t4 - 4u * t3 - 2u * t2 - t1;
    pop[i] = (int)t4;
    q += D[i];
  }
  return c;
}

// Four bytes holding one nibble each (byte i = nibble i) -> those nibbles in bits 4i..4i+3.
__device__ __forceinline__ uint32_t pack4(uint32_t b) {
  return (b & 0xFu) | ((b >> 4) & 0xF0u) | ((b >> 8) & 0xF00u) | ((b >> 12) & 0xF000u);
}

// Encode rows of `in`; kField: store the field and scale; kReadout: store the readout to `out` (which
// may be `in`: every row is read before it is written, by the same lanes).  LPR lanes per row, so a
// warp holds 32 / LPR rows side by side and R such groups at once.
template <int V, int LPR, bool kField, bool kReadout>
__global__ void __launch_bounds__(kWarps * 32) field_encode_kernel(const float* in, float* out, int rows,
                                                                   int N, uint32_t* field, float* scale) {
  constexpr int RPW = 32 / LPR;
  constexpr int R = rows_per_warp<V>();
  __shared__ __align__(16) uint8_t nbuf[kWarps][256];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int li = lane & (LPR - 1), sub = lane / LPR;  // lane within the row; which of the warp's rows
  uint8_t* const nb = &nbuf[warp][sub * (256 / RPW)];  // N <= 256 / RPW bytes of this row
  const int W = N / 8;
  const long long per_warp = (long long)R * RPW;
  const long long step = (long long)gridDim.x * kWarps * per_warp;
  for (long long r0 = ((long long)blockIdx.x * kWarps + warp) * per_warp; r0 < rows; r0 += step) {
    float s[R][V];
#pragma unroll
    for (int j = 0; j < R; ++j) {
      const long long r = r0 + (long long)j * RPW + sub;
      if (r < rows) {
        load_vals<V>(in + r * N, N, li, s[j]);
      } else {
#pragma unroll
        for (int i = 0; i < V; ++i) s[j][i] = 0.0f;
      }
    }
#pragma unroll
    for (int j = 0; j < R; ++j) {
      const long long rb = r0 + (long long)j * RPW;
      if (rb >= rows) break;  // the same for the whole warp
      const long long r = rb + sub;
      const bool valid = r < rows;  // the second row of a pair may lie past the end
      uint32_t nib[V];
      int pop[V];
      const float c = encode_row<V, LPR>(s[j], N, li, nib, pop);
      if constexpr (kField) {
        if constexpr (V == 8) {  // the lane's eight values are word li
          uint32_t wd = 0;
#pragma unroll
          for (int i = 0; i < 8; ++i) wd |= nib[i] << (4 * i);
          if (valid && li < W) __stcs(field + r * W + li, wd);
        } else if constexpr (V == 4) {  // lanes 2t and 2t + 1 of a row hold the two halves of word t
          const uint32_t half = nib[0] | (nib[1] << 4) | (nib[2] << 8) | (nib[3] << 12);
          const uint32_t up = __shfl_down_sync(kFull, half, 1);
          if (valid && (li & 1) == 0 && (li >> 1) < W) __stcs(field + r * W + (li >> 1), half | (up << 16));
        } else {
#pragma unroll
          for (int i = 0; i < V; ++i)
            if (li * V + i < N) nb[li * V + i] = (uint8_t)nib[i];
          __syncwarp();
          if (valid && li < W) {
            const uint32_t lo = *reinterpret_cast<const uint32_t*>(nb + 8 * li);
            const uint32_t hi = *reinterpret_cast<const uint32_t*>(nb + 8 * li + 4);
            __stcs(field + r * W + li, pack4(lo) | (pack4(hi) << 16));
          }
          __syncwarp();  // nbuf is rewritten for the next row
        }
        if (valid && li == 0) scale[r] = c;
      }
      if constexpr (kReadout) {
        float yv[V];
#pragma unroll
        for (int i = 0; i < V; ++i) yv[i] = readout(c, pop[i]);
        if (valid) store_vals<V>(out + r * N, N, li, yv);
      }
    }
  }
}

template <int V>
__global__ void __launch_bounds__(kWarps * 32) field_decode_kernel(const uint32_t* field, const float* scale,
                                                                   int rows, int N, float* out) {
  constexpr int R = rows_per_warp<V>();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int W = N / 8;
  const long long step = (long long)gridDim.x * kWarps * R;
  for (long long r0 = ((long long)blockIdx.x * kWarps + warp) * R; r0 < rows; r0 += step) {
    uint32_t w[R];
    float c[R];
#pragma unroll
    for (int j = 0; j < R; ++j) {
      const bool ok = r0 + j < rows;
      w[j] = ok && lane < W ? __ldcs(field + (r0 + j) * W + lane) : 0u;
      c[j] = ok ? __ldg(scale + r0 + j) : 0.0f;
    }
#pragma unroll
    for (int j = 0; j < R; ++j) {
      const long long r = r0 + j;
      if (r >= rows) break;  // the same for the whole warp
      float y[V];
#pragma unroll
      for (int i = 0; i < V; ++i) {
        const int v = lane * V + i;                                // < 256, so v / 8 < 32
        const uint32_t word = __shfl_sync(kFull, w[j], v >> 3);
        y[i] = readout(c[j], __popc((word >> (4 * (v & 7))) & 0xFu));
      }
      store_vals<V>(out + r * N, N, lane, y);
    }
  }
}

int grid_for(int rows, int rows_per_cta) {
  const long long need = ((long long)rows + rows_per_cta - 1) / rows_per_cta;
  const long long cap = (long long)num_sms() * 32;
  return (int)(need < cap ? need : cap);
}

template <int V, int LPR>
cudaError_t encode_v(const float* in, float* out, uint32_t* field, float* scale, int rows, int N,
                     cudaStream_t st) {
  const int grid = grid_for(rows, kWarps * rows_per_warp<V>() * (32 / LPR));
  if (field && out)
    field_encode_kernel<V, LPR, true, true><<<grid, kWarps * 32, 0, st>>>(in, out, rows, N, field, scale);
  else if (field)
    field_encode_kernel<V, LPR, true, false><<<grid, kWarps * 32, 0, st>>>(in, nullptr, rows, N, field, scale);
  else
    field_encode_kernel<V, LPR, false, true><<<grid, kWarps * 32, 0, st>>>(in, out, rows, N, nullptr, nullptr);
  return cudaGetLastError();
}

template <int V>
cudaError_t decode_v(const uint32_t* field, const float* scale, int rows, int N, float* out, cudaStream_t st) {
  const int grid = grid_for(rows, kWarps * rows_per_warp<V>());
  field_decode_kernel<V><<<grid, kWarps * 32, 0, st>>>(field, scale, rows, N, out);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_field_encode(const float* in, float* out, uint32_t* field, float* scale, int rows, int N,
                                cudaStream_t st) {
  if (rows == 0) return cudaSuccess;
  if (N <= 128) {  // sixteen lanes per row, two rows per warp
    switch ((N + 15) / 16) {
      case 1: return encode_v<1, 16>(in, out, field, scale, rows, N, st);
      case 2: return encode_v<2, 16>(in, out, field, scale, rows, N, st);
      case 3: return encode_v<3, 16>(in, out, field, scale, rows, N, st);
      case 4: return encode_v<4, 16>(in, out, field, scale, rows, N, st);
      case 5: return encode_v<5, 16>(in, out, field, scale, rows, N, st);
      case 6: return encode_v<6, 16>(in, out, field, scale, rows, N, st);
      case 7: return encode_v<7, 16>(in, out, field, scale, rows, N, st);
      case 8: return encode_v<8, 16>(in, out, field, scale, rows, N, st);
      default: return cudaErrorInvalidValue;
    }
  }
  switch ((N + 31) / 32) {
    case 5: return encode_v<5, 32>(in, out, field, scale, rows, N, st);
    case 6: return encode_v<6, 32>(in, out, field, scale, rows, N, st);
    case 7: return encode_v<7, 32>(in, out, field, scale, rows, N, st);
    case 8: return encode_v<8, 32>(in, out, field, scale, rows, N, st);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_field_decode(const uint32_t* field, const float* scale, int rows, int N, float* out,
                                cudaStream_t st) {
  if (rows == 0) return cudaSuccess;
  switch ((N + 31) / 32) {
    case 1: return decode_v<1>(field, scale, rows, N, out, st);
    case 2: return decode_v<2>(field, scale, rows, N, out, st);
    case 3: return decode_v<3>(field, scale, rows, N, out, st);
    case 4: return decode_v<4>(field, scale, rows, N, out, st);
    case 5: return decode_v<5>(field, scale, rows, N, out, st);
    case 6: return decode_v<6>(field, scale, rows, N, out, st);
    case 7: return decode_v<7>(field, scale, rows, N, out, st);
    case 8: return decode_v<8>(field, scale, rows, N, out, st);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace dfssm
