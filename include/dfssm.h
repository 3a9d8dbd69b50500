/*
 * dfssm.h — C ABI of libdfssm, the B200 (sm_100a) implementation of the DF-SSM decode/prefill hot path.
 *
 * DF-SSM ("Density Field State Space Models: 1-Bit Distillation, Efficient Inference, and Knowledge
 * Organization in Mamba-2", arXiv 2606.10932) compresses Mamba-2 so that in_proj and out_proj are a
 * frozen 1-bit sign scaffold with per-output-channel scales, applied to per-token int8 activations with
 * int32 accumulation, plus an int8 rank-16 LoRA correction (gist.science technical summary, §2.B "Frozen
 * Scaffold with LoRA Correction" and §2.C "Optimized Inference Pipeline").  The stateful ops are the
 * width-4 causal-conv shift register and the per-head SSM recurrence (same summary, §2.C).  The Mamba-2
 * block equations are those of the cited Mamba-2/SSD layer (mlsanity citation map, "Builds on").
 *
 * Conventions for every entry point:
 *   - Pointers documented as "device" must point to memory of the current CUDA device.  The caller owns
 *     every buffer, and the library calls no allocating routine.  Scratch comes from a caller-provided
 *     workspace of at least dfssm_workspace_size(...) bytes, 256-byte aligned, zero-filled before its
 *     first use.  The one exception is dfssm_linear_decode_noalloc, which keeps its scratch and status
 *     word in fixed arrays of the library's own device memory.
 *   - Device-side errors (a wait that ran out of its clock budget, an embedding id out of range) are
 *     recorded in a status word at the start of the call's workspace (for dfssm_linear_decode,
 *     dfssm_linear_decode_multi, dfssm_linear_prefill, dfssm_embed, dfssm_layer_decode,
 *     dfssm_layer_prefill and dfssm_generate), read and cleared by dfssm_device_status.
 *   - Every call is asynchronous on `stream` (a cudaStream_t; NULL = legacy default stream).  Inputs
 *     must not be modified, and outputs not read, until the stream reaches the call.  Weights and
 *     parameters must be fully written before the call is enqueued (kernels may read them before they
 *     wait on the preceding kernel of the stream).
 *   - Arguments are validated before anything is launched; on a negative status nothing was enqueued.
 *   - Concurrency: calls that share a workspace must not overlap on the GPU.  The library's only state
 *     outside the caller's buffers is per-device and set once (the kernels' shared-memory attribute and
 *     the SM count, guarded by a mutex) plus the no-alloc entry point's module arrays; so calls on
 *     different streams with different workspaces may run concurrently, from any host threads.  A
 *     cudaDeviceReset invalidates those per-device records: do not use the library after one.
 *   - fp32 values that feed an int8 quantizer are computed as single correctly rounded fp32 operations,
 *     with sums and transcendental functions evaluated in fp64 and rounded once, so that quantization
 *     codes are reproducible by a plain CPU evaluation of the same definitions.
 */
#ifndef DFSSM_H_
#define DFSSM_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define DFSSM_ABI_VERSION 5
#define DFSSM_MAX_RANK 16
#define DFSSM_MAX_BATCH 16
#define DFSSM_MAX_LAYERS 64

typedef enum {
  DFSSM_OK = 0,
  DFSSM_EINVAL = -1,       /* bad size, NULL pointer or inconsistent arguments                      */
  DFSSM_EALIGN = -2,       /* a pointer is not aligned as documented                                */
  DFSSM_EUNSUPPORTED = -3, /* valid, but outside what the library implements (e.g. B > 16)         */
  DFSSM_ECUDA = -4,        /* a CUDA runtime call failed; see dfssm_last_cuda_error()                */
  DFSSM_ETIMEOUT = -5,     /* a device-side wait ran out of its iteration budget                    */
  DFSSM_EDEVICE = -6,      /* no usable sm_100 device                                               */
  DFSSM_EWORKSPACE = -7    /* workspace NULL, too small or misaligned                               */
} dfssm_status;

/*
 * One DF-SSM linear: y = scaffold(x) + LoRA(x) (technical summary §2.B–C).
 *   bits          device u32 [d_out][d_in/32], row-major.  Bit j of word w of row o is the sign of weight
 *                 (o, 32w+j): set = +1, clear = -1 (least significant bit first).  16-byte aligned.
 *   w_scale       device f32 [d_out]   per-output-channel scaffold scale sW
 *   lora_b        device i8  [rank][d_in]   W_B, row-major; 4-byte aligned
 *   lora_b_scale  device f32 [rank]    per-row scale of W_B
 *   lora_a        device i8  [d_out][rank]  W_A, row-major
 *   lora_a_scale  device f32 [d_out]   per-row scale of W_A
 * Constraints: d_in % 32 == 0, d_out >= 1, 0 <= rank <= 16 (otherwise DFSSM_EINVAL); d_in <= 8192
 * (otherwise DFSSM_EUNSUPPORTED).  rank == 0 means no LoRA
 * (lora_* may then be NULL).
 * Computes, for each token b with input x and (q, s) its per-token int8 quantization:
 *   acc[o] = sum_i sign(o,i) q[i]  (int32, exact)
 *   t[r]   = sum_i W_B[r,i] q[i]  (int32, exact)           (LoRA down on the same int8 codes)
 *   tf[r]  = fl32(t[r] sB[r] s)                            (fp64 inside, this order)
 *   y[o]   = fl32(acc[o] s sW[o] + sA[o] sum_r W_A[o,r] tf[r])   (fp64 inside)
 */
typedef struct {
  int32_t d_out, d_in, rank;
  const uint32_t* bits;
  const float* w_scale;
  const int8_t* lora_b;
  const float* lora_b_scale;
  const int8_t* lora_a;
  const float* lora_a_scale;
} dfssm_linear_t;

/* Optional device taps of the intermediates (any member may be NULL). */
typedef struct {
  int32_t* acc;   /* [B][d_out]  scaffold accumulators (int32, exact)                      */
  int32_t* lora_t; /* [B][rank]  LoRA-down accumulators t (int32, exact)                  */
  int8_t* xq;     /* [B][d_in]   quantized activations, natural order                     */
  float* xscale;  /* [B]         per-token scale s                                         */
} dfssm_debug_t;

/* Workspace sizing.  `op` selects the entry point; the remaining arguments are that entry point's
 * sizes as listed; unused ones are ignored.  Returns 0 for invalid sizes. */
enum {
  DFSSM_OP_LINEAR_DECODE = 1,  /* a = B,  b = d_in,  c = d_out                         */
  DFSSM_OP_LINEAR_PREFILL = 2, /* a = M,  b = d_in,  c = d_out                         */
  DFSSM_OP_LAYER_DECODE = 3,   /* a = B,  b = d_model, c = d_inner (nheads*headdim)     */
  DFSSM_OP_LM_HEAD = 4,        /* a = 1,  b = d,     c = V                             */
  DFSSM_OP_HEAD_GREEDY = 5,    /* a = 1,  b = d,     c = V                             */
  DFSSM_OP_GENERATE = 6,       /* a = V,  b = d_model, c = d_inner                     */
  DFSSM_OP_LAYER_PREFILL = 7,  /* a = M,  b = d_model, c = d_inner                     */
  DFSSM_OP_LINEAR_MULTI = 8,   /* (no size arguments): the status word only             */
  DFSSM_OP_EMBED = 9           /* (no size arguments): the status word only             */
};
size_t dfssm_workspace_size(int op, int a, int b, int c);

/*
 * Batch-B decode of one linear (scaffold GEMV + fused int8 LoRA), technical summary §2.B–C.
 *   x   device f32 [B][d_in] (16-byte aligned),  y device f32 [B][d_out]
 *   1 <= B <= 16.  dbg may be NULL.  workspace: dfssm_workspace_size(DFSSM_OP_LINEAR_DECODE, B, d_in, d_out).
 * For d_in in {1024, 2048, 4096} (any B <= 16) and d_in = 8192 with B <= 4 the call is one kernel that
 * quantizes x in every CTA and streams the sign bits through shared memory; only the workspace's status
 * word is used then.  Otherwise a quantize kernel writes the codes into the workspace and a GEMV kernel
 * reads them.
 */
int dfssm_linear_decode(const dfssm_linear_t* lin, const float* x, int B, float* y, void* workspace,
                        size_t ws_bytes, const dfssm_debug_t* dbg, void* stream);

/*
 * Decode of n independent linears that read the same input x, in one launch: y_j = linear_j(x) for
 * j < n, each exactly as dfssm_linear_decode computes it (technical summary §2.B–C; a Mamba-2 layer's
 * projections of one activation, or a stack of layer copies, stream their sign bits back to back).
 *   lins  host array of n descriptors (device pointers inside), all with the same d_in
 *   x     device f32 [B][d_in] (16-byte aligned);  ys host array of n device pointers, ys[j] f32 [B][d_out_j]
 *   1 <= n <= 64; d_in in {1024, 2048, 4096} with 1 <= B <= 16, or d_in = 8192 with 1 <= B <= 4; other
 *   sizes return DFSSM_EUNSUPPORTED.
 *   workspace: dfssm_workspace_size(DFSSM_OP_LINEAR_MULTI, 0, 0, 0) bytes (the status word).
 * The outputs must not overlap each other or x.
 */
int dfssm_linear_decode_multi(const dfssm_linear_t* lins, int n, const float* x, int B, float* const* ys,
                              void* workspace, size_t ws_bytes, void* stream);

/*
 * dfssm_linear_decode for callers that cannot allocate device memory.  The paper has no counterpart: this
 * is a deployment variant of the same computation, with the same arguments and results except that there
 * is no workspace.  It serves code that may only hand the library its inputs and outputs — a plugin whose
 * host process owns every device allocation, or a real-time loop that must not call cudaMalloc because it
 * can block and synchronise the device.
 *   Limits: 1 <= B <= 16 and d_in <= 8192; larger sizes return DFSSM_EUNSUPPORTED before anything runs.
 *   Scratch: a fixed 132,608-byte array in the library's own device memory, held by every device that
 *   loads the library until the process exits.  The call allocates and frees nothing.  Calls in the
 *   streaming kernel's range (d_in in {1024, 2048, 4096}, or d_in = 8192 with B <= 4) run that kernel and
 *   use no scratch.
 *   Set-up: the first call on a device looks up that array's device address (cudaGetSymbolAddress, with
 *   that device current) and caches it; make that first call before any stream capture, and do not use
 *   the library across a cudaDeviceReset of that device.
 *   Sharing: all calls on a device use the same array.  Each call writes everything it reads there, so
 *   nothing needs clearing, but calls that overlap on the GPU (unordered streams) race: order them.
 *   Status: a timed-out wait is recorded in a module status word beside the array, read and cleared by
 *   dfssm_device_status(NULL, stream).
 */
int dfssm_linear_decode_noalloc(const dfssm_linear_t* lin, const float* x, int B, float* y,
                                const dfssm_debug_t* dbg, void* stream);

/*
 * M-token prefill of one linear on int8 tcgen05 tensor cores (technical summary §2.C: the 1-bit weights
 * expanded on the fly to int8 for the INT8 tensor cores; here the expansion happens in shared memory and
 * never reaches global memory).  Same math as dfssm_linear_decode, per row of x.
 *   x device f32 [M][d_in], y device f32 [M][d_out], M >= 1.  d_in % 128 == 0 required.
 *   workspace: dfssm_workspace_size(DFSSM_OP_LINEAR_PREFILL, M, d_in, d_out) bytes (status word first).
 *   dbg->acc, dbg->xq, dbg->xscale and dbg->lora_t are exact, and y is bit-identical to the decode path
 *   (the epilogue evaluates the definition in fp64 with the decode rounding sequence).
 */
int dfssm_linear_prefill(const dfssm_linear_t* lin, const float* x, int M, float* y, void* workspace,
                         size_t ws_bytes, const dfssm_debug_t* dbg, void* stream);

/*
 * Width-4 stateful shift-register causal convolution, one decode step, with SiLU (technical summary §2.C
 * "stateful shift register (convolution)").
 *   conv_state device f32 [B][C][3]  (the last three inputs, oldest first; updated in place)
 *   w device f32 [C][4] (w[c][3] multiplies the current input), b device f32 [C]
 *   x_in device f32 [B][C], x_out device f32 [B][C]   (x_out = SiLU(b + sum_k w[c,k] window_k))
 */
int dfssm_conv_step(float* conv_state, const float* w, const float* b, const float* x_in, float* x_out,
                    int B, int C, void* stream);

/*
 * Mamba-2 SSM state update and readout for one decode step (technical summary §2.C "SSM recurrence").
 *   ssm_state device f32 [B][H][P][N] (updated in place), x device f32 [B][H*P], dt_raw device f32 [B][H],
 *   A_log, dt_bias, D device f32 [H], Bm, Cm device f32 [B][G][N], y device f32 [B][H*P].
 *   dt = softplus(dt_raw + dt_bias); dA = exp(dt * -exp(A_log));
 *   S = dA S + (dt x) B;  y = S . C + D x.      Requires H % G == 0, N % 4 == 0, N <= 512.
 */
int dfssm_ssm_step(float* ssm_state, const float* x, const float* dt_raw, const float* A_log,
                   const float* dt_bias, const float* D, const float* Bm, const float* Cm, float* y,
                   int B, int H, int P, int N, int G, void* stream);

/*
 * Density-field state representation (technical summary §2.D "Density Field State Representation": the
 * SSM hidden state kept as a binary field per state element, K^2 about 4 d_state cells, built by
 * normalization, sigma-delta injection with error feedback and binarization, read back by popcount, at
 * chunk boundaries).  One state row S[0..N) (N = d_state; an SSM state [B][H][P][N] is B*H*P rows) is
 * 4N cells, four per value, plus c = max |S|:
 *   x_n = fl32(S_n / c) (0 when c = 0), d_n = fl32(x_n + 1) / 2;
 *   cells j = 4n + k, in order, fed d_n through v = d + e, b_j = [v >= 1/2], e = v - b_j (e = 0 at the row
 *   start; exact arithmetic: every d_n is a multiple of 2^-25);
 *   readout S^_n = fl32(c (popcount(cells of n) / 2 - 1)), one of {-c, -c/2, 0, c/2, c}.
 *   state device f32 [rows][N] (16-byte aligned), finite values;
 *   field device u32 [rows][N/8]: cell j is bit j % 32 of word j / 32 (value n is nibble n % 8 of word n / 8);
 *   scale device f32 [rows]: c.
 * Requires 8 <= N, N % 8 == 0 (else DFSSM_EINVAL), N <= 256 (else DFSSM_EUNSUPPORTED), rows >= 0; with
 * rows == 0 nothing is read or launched (the pointers may be NULL), otherwise NULL pointers give
 * DFSSM_EINVAL.  The library applies no schedule: the caller calls these at its chunk boundaries.
 */
int dfssm_state_field_encode(const float* state, int rows, int N, uint32_t* field, float* scale,
                             void* stream);
/* The popcount readout of a field into state rows (state written, field and scale read). */
int dfssm_state_field_decode(const uint32_t* field, const float* scale, int rows, int N, float* state,
                             void* stream);
/* Encode and read back in place in one pass: state <- readout(encode(state)); field and scale are
 * stored too when both are non-NULL (both NULL: not stored; one NULL: DFSSM_EINVAL). */
int dfssm_state_field_roundtrip(float* state, int rows, int N, uint32_t* field, float* scale, void* stream);

/* Shape of a DF-SSM Mamba-2 layer.  d_inner = nheads*headdim; conv channels = d_inner + 2*ngroups*d_state;
 * in_proj rows = 2*d_inner + 2*ngroups*d_state + nheads, ordered z | x | B | C | dt. */
typedef struct {
  int32_t d_model, nheads, headdim, d_state, ngroups;
} dfssm_dims_t;

/* Parameters of one layer (all device pointers). */
typedef struct {
  dfssm_linear_t in_proj;   /* d_out = 2*d_inner + 2*ngroups*d_state + nheads, d_in = d_model */
  dfssm_linear_t out_proj;  /* d_out = d_model, d_in = d_inner                               */
  const float* conv_w;      /* [conv channels][4] */
  const float* conv_b;      /* [conv channels]    */
  const float* A_log;       /* [nheads] */
  const float* dt_bias;     /* [nheads] */
  const float* D;           /* [nheads] */
  const float* norm_w;      /* [d_model]  pre-mixer RMSNorm weight, eps 1e-5 */
  const float* gnorm_w;     /* [d_inner]  gated RMSNorm weight, eps 1e-5    */
} dfssm_layer_t;

/*
 * One decode step (one token per sequence) through n_layers DF-SSM Mamba-2 layers.
 *   layers       HOST array [n_layers] (read during the call only)
 *   hidden       device f32 [B][d_model]; the residual stream, updated in place
 *   conv_states  HOST array [n_layers] of device f32 [B][conv channels][3]
 *   ssm_states   HOST array [n_layers] of device f32 [B][nheads][headdim][d_state]
 * Per layer: (q,s) = quant(RMSNorm(h)); zxbcdt = in_proj (LoRA on RMSNorm(h)); x|B|C = SiLU(conv(xBC));
 * y = SSM(x, dt, B, C); g = y*SiLU(z); (q',s') = quant(RMSNorm(g)); h += out_proj.  The RMS factor is
 * folded into the quantizer scale: the codes q are those of v = fl32(h w), s = fl32(s0/rms) with s0 the
 * absmax scale of v, and the LoRA intermediate is tf = fl32(t sB s) with t = W_B q (int32).
 * 1 <= B <= 16, n_layers <= 64.
 * workspace: dfssm_workspace_size(DFSSM_OP_LAYER_DECODE, B, d_model, d_inner).
 */
int dfssm_layer_decode(const dfssm_layer_t* layers, int n_layers, const dfssm_dims_t* dims,
                       float* hidden, float* const* conv_states, float* const* ssm_states, int B,
                       void* workspace, size_t ws_bytes, void* stream);

/*
 * Prefill of an M-token prompt (batch 1) through n_layers layers: for each layer, in order,
 *   (q, s) = quant(RMSNorm(h_t)) and zxbcdt = in_proj for all t  (tcgen05 int8 GEMM, as dfssm_linear_prefill
 *   with the pre-norm folded into the quantizer);  xBC = conv over the sequence, continuing conv_state;
 *   y = the SSM recurrence stepped through t = 0 .. M-1, continuing ssm_state;  g = y SiLU(z);
 *   h_t += out_proj(quant(RMSNorm(g_t)))  (tcgen05 GEMM with the gated norm folded in, residual add in
 *   its epilogue).
 * The conv and SSM steps follow, token after token, exactly the decode step's arithmetic (technical
 * summary §2.C "Stateful Ops"), so afterwards conv_states / ssm_states hold what M calls of
 * dfssm_layer_decode would leave and decoding continues from them; the linears are exact as in decode.
 * The SSM readout sum_n S C is accumulated in about 48 bits (a pair of fp32 values) instead of fp64, so
 * the outputs agree with the decode definition to that precision, not bit for bit.
 *   hidden device f32 [M][d_model] (16-byte aligned), updated in place: the residual stream after the last
 *   layer.  Layers, dims and states as for dfssm_layer_decode with B = 1.  Requires d_model and d_inner
 *   multiples of 128 (<= 8192), headdim a multiple of 16, d_state a multiple of 4 (<= 512).
 *   workspace: dfssm_workspace_size(DFSSM_OP_LAYER_PREFILL, M, d_model, d_inner).
 */
int dfssm_layer_prefill(const dfssm_layer_t* layers, int n_layers, const dfssm_dims_t* dims,
                        float* hidden, float* const* conv_states, float* const* ssm_states, int M,
                        void* workspace, size_t ws_bytes, void* stream);

/*
 * Int8 LM head on one token (technical summary §2.B: int8 LM head with per-row scaling).
 *   W device i8 [V][d] (16-byte aligned, d % 16 == 0), s_row device f32 [V], x device f32 [d],
 *   logits device f32 [V].   logits[v] = fl32(acc[v] s s_row[v]), acc[v] = sum_i W[v,i] q[i], with
 *   (q, s) the per-token absmax int8 quantization of x (as in dfssm_linear_decode).  d <= 8192.
 *   acc (device i32 [V]) may be NULL.  One kernel: every CTA quantizes x itself, so the call needs no
 *   scratch; workspace and ws_bytes are not read (may be NULL / 0; dfssm_workspace_size still reports the
 *   size earlier versions used).
 */
int dfssm_lm_head(const int8_t* W, const float* s_row, int V, int d, const float* x, float* logits,
                  int32_t* acc, void* workspace, size_t ws_bytes, void* stream);

/*
 * Token embedding from the tied int8 embedding / LM-head matrix (technical summary §2.B: the embedding
 * and LM head are int8 with per-row scaling; §3: together they are 37% of the 278 MB model, i.e. one
 * V x d_model matrix, read here as shared by both).
 *   W device i8 [V][d] (16-byte aligned, d % 16 == 0, d <= 8192), s_row device f32 [V],
 *   token device i32 [1] (read on the device when the stream reaches the call), h device f32 [d]
 *   (16-byte aligned).   h[i] = fl32(W[tok, i] * s_row[tok]).
 * A token outside [0, V) writes h = 0 and records a sticky code in the workspace's status word:
 * dfssm_device_status(workspace) then returns DFSSM_EINVAL.  One single-CTA kernel.
 *   workspace: dfssm_workspace_size(DFSSM_OP_EMBED, 0, 0, 0) bytes (the status word).
 */
int dfssm_embed(const int8_t* W, const float* s_row, int V, int d, const int32_t* token, float* h,
                void* workspace, size_t ws_bytes, void* stream);

/*
 * Final RMSNorm + int8 LM head + greedy choice on one token (the Mamba-2 language model's final norm
 * before its LM head, a reading of the cited architecture; the head as in dfssm_lm_head).
 *   h device f32 [d] (the residual stream after the last layer); norm_w device f32 [d] or NULL (then no
 *   norm: the logits are exactly dfssm_lm_head's).  With norm_w the token is normalized first:
 *   r = fl32(1 / sqrt(sum h^2 / d + 1e-5)) (fp64), u = fl32(fl32(h r) w), (q, s) = quant(u), and
 *   logits[v] = fl32(acc[v] s s_row[v]), acc[v] = sum_i W[v,i] q[i].
 *   token device i32 [1] receives the index of the largest logit (the smallest index on ties; -0 and +0
 *   are equal).  logits device f32 [V] (required), acc device i32 [V] or NULL.
 *   workspace: dfssm_workspace_size(DFSSM_OP_HEAD_GREEDY, 1, d, V) bytes, zero-filled before its first
 *   use; each call leaves it zero again.  One kernel.
 */
int dfssm_head_greedy(const int8_t* W, const float* s_row, int V, int d, const float* h,
                      const float* norm_w, float* logits, int32_t* acc, int32_t* token, void* workspace,
                      size_t ws_bytes, void* stream);

/*
 * Greedy generation at batch 1 (technical summary §2.C: the 48-layer decode step, with the int8
 * embedding and LM head of §2.B): for t = 0 .. n_tokens-1
 *   h = embed(tokens[t]);  dfssm_layer_decode(layers, h);  tokens[t+1] = greedy(final_head(h)).
 *   tokens device i32 [n_tokens + 1]: tokens[0] is the first token (set by the caller), the rest are
 *   written.  W, s_row, V as for dfssm_embed; final_norm_w device f32 [d_model].  Layers, dims and
 *   states as for dfssm_layer_decode with B = 1 (the states advance by n_tokens steps).
 *   hidden_taps device f32 [n_tokens][d_model] or NULL: the residual stream after the last layer at each
 *   step.  logits (device f32 [V] or NULL) receives the last step's logits.
 *   workspace: dfssm_workspace_size(DFSSM_OP_GENERATE, V, d_model, d_inner), zero-filled before its first
 *   use.  Three kernels per token (embedding, the layers, the head); the calls are stream-ordered and
 *   can be captured in a CUDA graph.
 */
int dfssm_generate(const dfssm_layer_t* layers, int n_layers, const dfssm_dims_t* dims,
                   const int8_t* W, const float* s_row, int V, const float* final_norm_w,
                   int32_t* tokens, int n_tokens, float* const* conv_states, float* const* ssm_states,
                   float* hidden_taps, float* logits, void* workspace, size_t ws_bytes, void* stream);

/*
 * Device-side failure detection.  The fused decode kernel of dfssm_layer_decode (batch 1, Mamba-2-1.3B
 * shape) hands data between its CTAs through tagged words in the workspace; every wait has a clock
 * budget (about one second).  A wait that runs out makes every CTA of that launch return early (its
 * outputs are then incomplete) and records a sticky code in the workspace's status word; each new launch
 * starts with fresh tags.  The streaming linear kernel (dfssm_linear_decode in its range,
 * dfssm_linear_decode_multi) bounds its shared-memory pipeline waits the same way and records a timeout
 * in the status word of the call's workspace; dfssm_embed records an out-of-range token there.
 * dfssm_device_status synchronises `stream`, reads and clears the status word at the start of
 * `workspace` (NULL: the module status word of dfssm_linear_decode_noalloc), and returns DFSSM_OK,
 * DFSSM_ETIMEOUT, or DFSSM_EINVAL for an out-of-range embedding id.  No device trap or fault is ever
 * raised.
 */
int dfssm_device_status(void* workspace, void* stream);

/* Diagnostic: launch a one-warp kernel that waits, with a budget of about 1 ms, on a workspace word that
 * nothing writes, so that the next dfssm_device_status returns DFSSM_ETIMEOUT.  workspace as
 * for dfssm_layer_decode. */
int dfssm_selftest_timeout(void* workspace, size_t ws_bytes, void* stream);

/* Host helper: pack a +-1 int8 matrix [d_out][d_in] (row-major, host) into the bit layout above
 * (host u32 [d_out][d_in/32]).  Any value > 0 maps to a set bit. */
int dfssm_pack_signs(const int8_t* signs, int d_out, int d_in, uint32_t* bits);

/* Text for a status code (static storage). */
const char* dfssm_status_string(int status);

/* The last CUDA error string recorded by a DFSSM_ECUDA return on this thread (static storage). */
const char* dfssm_last_cuda_error(void);

/* DFSSM_ABI_VERSION of the loaded library. */
int dfssm_abi_version(void);

#ifdef __cplusplus
}
#endif
#endif /* DFSSM_H_ */
