/*
 * dfssm_cpu.h — C ABI of libdfssm_cpu, the host-CPU (AVX-512 VNNI) engine of the DF-SSM decode step.
 *
 * The pages describe a CPU inference path beside the GPU one (gist.science technical summary of DF-SSM,
 * §2.C "CPU path": a bit-packed kernel expands the 1-bit weights to int8 for the VNNI dot-product
 * instruction, loading 8x less weight data than int8 weights; §3 "Inference Performance": 2.9x on an
 * AVX-512 Xeon).  This engine computes the same definitions as libdfssm (include/dfssm.h) on host memory:
 * the scaffold GEMV turns 64 sign bits at a time into 0/1 bytes in a register (a masked byte move) and
 * multiplies them with the int8 codes by vpdpbusd (u8 x s8 -> s32), so acc = 2 sum_{bit=1} q - sum q
 * is exact; every floating-point step follows libdfssm's rounding sequence (fp32 values rounded once,
 * sums of more than two terms in fp64 in index order, transcendental functions in fp64), so codes,
 * accumulators and outputs are bit-identical to it and to a plain evaluation of the definitions.
 *
 * Conventions:
 *   - All pointers are HOST pointers (the dfssm_linear_t / dfssm_layer_t structs of dfssm.h filled with
 *     host addresses).  The caller owns every buffer; calls are synchronous; no global state besides the
 *     OpenMP thread count.
 *   - Each entry point checks at run time that the CPU supports AVX-512 F/BW/VL and VNNI and returns
 *     DFSSM_EUNSUPPORTED otherwise (dfssm_cpu_available() tells in advance).
 *   - Arguments are validated first; on a negative status nothing was written.
 */
#ifndef DFSSM_CPU_H_
#define DFSSM_CPU_H_

#include "dfssm.h"

#ifdef __cplusplus
extern "C" {
#endif

#define DFSSM_CPU_ABI_VERSION 2

int dfssm_cpu_abi_version(void);

/* 1 when the host CPU has AVX-512 F, BW, VL and VNNI, else 0. */
int dfssm_cpu_available(void);

/* OpenMP threads used by the following calls (n <= 0: all available).  Returns the count in use. */
int dfssm_cpu_set_threads(int n);

/*
 * One linear for B tokens (dfssm_linear_decode's definition):
 *   x host f32 [B][d_in], y host f32 [B][d_out], 1 <= B <= 16; d_in % 32 == 0, d_in <= 8192.
 *   dbg (optional, host pointers): acc [B][d_out], lora_t [B][rank], xq [B][d_in], xscale [B].
 */
int dfssm_cpu_linear_decode(const dfssm_linear_t* lin, const float* x, int B, float* y,
                            const dfssm_debug_t* dbg);

/*
 * One decode step of every layer for B tokens (dfssm_layer_decode's definition): RMSNorm + quantize,
 * in_proj, conv step, SSM step, gate, gated RMSNorm + quantize, out_proj, residual.
 *   hidden host f32 [B][d_model] (in/out), conv_states[l] host f32 [B][C][3], ssm_states[l] host f32
 *   [B][nheads][headdim][d_state] (updated in place).  1 <= B <= 16, 1 <= n_layers <= 64.
 */
int dfssm_cpu_layer_decode(const dfssm_layer_t* layers, int n_layers, const dfssm_dims_t* dims,
                           float* hidden, float* const* conv_states, float* const* ssm_states, int B);

/*
 * Density-field state representation (dfssm_state_field_encode / _decode / _roundtrip's definition,
 * technical summary §2.D "Density Field State Representation"), on host rows [rows][N]:
 *   state host f32 [rows][N], field host u32 [rows][N/8], scale host f32 [rows];
 *   8 <= N, N % 8 == 0 (else DFSSM_EINVAL), N <= 256 (else DFSSM_EUNSUPPORTED); rows == 0 does nothing.
 * The readout needs no AVX-512; encode and round trip return DFSSM_EUNSUPPORTED without it.
 */
int dfssm_cpu_state_field_encode(const float* state, int rows, int N, uint32_t* field, float* scale);
int dfssm_cpu_state_field_decode(const uint32_t* field, const float* scale, int rows, int N, float* state);
int dfssm_cpu_state_field_roundtrip(float* state, int rows, int N, uint32_t* field, float* scale);

#ifdef __cplusplus
}
#endif

#endif  // DFSSM_CPU_H_
