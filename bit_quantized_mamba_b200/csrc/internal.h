// Internal host-side interfaces between the C-ABI layer (api.cu) and the kernel files.
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

namespace dfssm {

// Scratch carved from the caller's workspace for one quantize -> linear hand-off.
struct QuantScratch {
  int8_t* q;     // [B][n] codes (dp4a-permuted or natural order)
  float* s;      // [B] per-token scale
  int32_t* sumq; // [B] sum of the codes of each token
  float* tf;     // [B][16] LoRA intermediate (entries >= rank are 0)
};
size_t quant_scratch_bytes(int B, int n);
QuantScratch carve_quant_scratch(void* base, int B, int n);

struct QuantArgs {
  const float* x;
  int ldx;                 // row stride of x (elements)
  const float* norm_w;     // non-NULL: RMSNorm(eps 1e-5) folded into the scale
  int n;                   // row length
  int B;
  const int8_t* lora_b;    // [rank][n] or NULL
  const float* lora_b_scale;
  int rank;
  bool permute;            // dp4a-permuted layout (scaffold GEMV) or natural (int8 GEMV)
  QuantScratch out;
  int8_t* dbg_xq;          // optional taps
  float* dbg_s;
  int32_t* dbg_t;          // [B][rank] exact LoRA-down t
};
cudaError_t launch_quant(const QuantArgs& a, cudaStream_t st);

struct GemvArgs {
  const uint32_t* bits;
  const float* w_scale;
  const int8_t* lora_a;
  const float* lora_a_scale;
  const float* lora_b_scale;
  int rank, d_out, d_in, B;
  QuantScratch in;
  float* y;
  int ldy;
  float* resid;            // non-NULL: resid = fl32(resid + y) instead of writing y
  int ldr;
  int32_t* dbg_acc;        // [B][d_out] or NULL
};
cudaError_t launch_gemv(const GemvArgs& a, cudaStream_t st);

struct ConvArgs {
  float* state;            // [B][C][3]
  const float* w;          // [C][4]
  const float* bias;       // [C]
  const float* x_in;
  int ldx;
  float* x_out;
  int ldo;
  int B, C;
};
cudaError_t launch_conv(const ConvArgs& a, cudaStream_t st);

struct SsmArgs {
  float* state;            // [B][H][P][N]
  const float* x;          // [B][ldx], head-major H*P
  int ldx;
  const float* dt_raw;     // [B][lddt]
  int lddt;
  const float* A_log;
  const float* dt_bias;
  const float* D;
  const float* Bm;         // [B][ldbc] rows, group g at offset g*N
  const float* Cm;
  int ldbc;
  float* y;                // [B][ldy]
  int ldy;
  const float* z;          // optional gate input [B][ldz]: y is replaced by fl32(y * SiLU(z))
  int ldz;
  int B, H, P, N, G;
};
cudaError_t launch_ssm(const SsmArgs& a, cudaStream_t st);

// Sequence conv of a prompt (B = 1): xc[t][c] for t < M from the in_proj output rows zx[t][x_off + c]
// and the incoming shift-register state [C][3] (oldest first), then the state is advanced by M tokens.
struct ConvSeqArgs {
  const float* zx;
  int ld_zx, x_off;
  float* state;
  const float* w;  // [C][4], 16-byte aligned
  const float* b;
  float* xc;       // [M][C]
  int M, C;
};
cudaError_t launch_conv_seq(const ConvSeqArgs& a, cudaStream_t st);

// Sequence SSM scan of a prompt (B = 1) with the gate: g[t][h*P+p] for t < M; the state [H][P][N]
// advances by M tokens.  z at column 0 and dt_raw at column dt_off of zx rows; x at column 0, B at b_off
// and C at c_off (group g at + g*N) of xc rows.
struct ScanArgs {
  const float* zx;
  int ld_zx, dt_off;
  const float* xc;
  int ld_xc, b_off, c_off;
  const float* A_log;
  const float* dt_bias;
  const float* D;
  float* state;
  float* g;        // [M][H*P]
  float* sz;       // scratch [M][H*P]: fl32(SiLU(z)), written by the scan's first kernel
  float* dtdA;     // scratch [M][H][2]: dt and dA
  int M, H, P, N, G;
};
cudaError_t launch_ssm_scan(const ScanArgs& a, cudaStream_t st);
bool scan_supported(int H, int P, int N, int G);

struct Int8GemvArgs {
  const int8_t* W;
  const float* s_row;
  int V, d;
  const float* x;           // the token, fp32 [d] (quantized by every CTA of the kernel)
  float* logits;
  int32_t* acc;
  const float* norm_w = nullptr;     // final RMSNorm weight [d], folded into the quantizer (optional)
  // greedy choice (optional): the argmax key and the CTA count live in `greedy` (2 x u64, zero
  // before the launch, left zero after it); the last CTA writes the index to *token
  unsigned long long* greedy = nullptr;
  int32_t* token = nullptr;
};
cudaError_t launch_int8_gemv(const Int8GemvArgs& a, cudaStream_t st);

// Codes a kernel leaves in a device status word (the first word of a call's workspace, or the no-alloc
// entry point's module word): a bounded wait ran out of its budget, or an embedding id was out of range.
constexpr int kDeviceTimeout = 0x7E0D1E57;
constexpr int kBadTokenCode = 0x70CE1D;
// Every workspace that carries a status word keeps it in its first kStatusBytes.
constexpr size_t kStatusBytes = 256;

// Embedding row lookup from the tied int8 matrix: h[i] = fl32(W[tok, i] * s_row[tok]), tok = *token.
// An id outside [0, V) writes zeros and sets *status to kBadTokenCode.
struct EmbedArgs {
  const int8_t* W;
  const float* s_row;
  int V, d;
  const int32_t* token;
  float* h;
  int* status;
};
cudaError_t launch_embed(const EmbedArgs& a, cudaStream_t st);

// Density-field state representation of state rows [rows][N] (8 <= N <= 256, N % 8 == 0; rows 16-byte
// aligned): encode to field [rows][N/8] + scale [rows] (either both or neither stored) and/or write the
// popcount readout to `out` (may equal `in`, or be NULL); decode a field back to rows.
cudaError_t launch_field_encode(const float* in, float* out, uint32_t* field, float* scale, int rows, int N,
                                cudaStream_t st);
cudaError_t launch_field_decode(const uint32_t* field, const float* scale, int rows, int N, float* out,
                                cudaStream_t st);

// Streaming multiprocessors of the current device.
int num_sms();
// Sets the dynamic shared-memory limit of a kernel on the current device, once per (kernel, device): the
// attribute is per device, and setting it once (not per launch) keeps launches capturable in a CUDA
// graph.  Thread-safe.  The record is per process: after cudaDeviceReset the library must not be used.
cudaError_t set_max_dynamic_smem(const void* func, int bytes);

}  // namespace dfssm

namespace dfssm {
// Prefill (tcgen05) workspace requirement for M tokens of a d_in -> d_out linear.
size_t prefill_workspace_bytes(int M, int d_in, int d_out);

// Fused persistent decode (one cooperative launch per token through all layers).
size_t fused_decode_workspace_bytes();

// dfssm_linear_prefill with two options for the layer prefill: a norm weight folded into the per-token
// quantizer (norm_w, may be NULL), and a residual epilogue (y[m][n] = fl32(y[m][n] + out)).
// status: the word a timed-out wait is recorded in (NULL: the first word of `workspace`).
int linear_prefill_impl(const dfssm_linear_t* lin, const float* x, int M, float* y, const float* norm_w,
                        bool resid, void* workspace, size_t ws_bytes, int* status, const dfssm_debug_t* dbg,
                        void* stream);
bool fused_decode_supported(const dfssm_dims_t& d, int B, const dfssm_layer_t* layers, int n,
                            float* const* conv_states);
cudaError_t launch_fused_decode(const dfssm_layer_t* layers, int n_layers, float* hidden,
                                float* const* conv_states, float* const* ssm_states, void* ws,
                                cudaStream_t st, long long spin_limit);
// Launches a kernel that waits on a counter nothing increments, with the given clock budget.
cudaError_t launch_timeout_selftest(void* ws, cudaStream_t st, long long spin_limit);
// Streaming decode of n linears that share x (B <= 16 at d_in 1024/2048/4096, B <= 4 at 8192): one
// persistent launch; a wait that runs out of budget stores kDeviceTimeout in *status.
bool stream_supported(int d_in, int B);
int launch_linear_stream(const dfssm_linear_t* lins, int n, const float* x, int B, float* const* ys,
                         const dfssm_debug_t* dbg, int* status, cudaStream_t st);
// Reads and clears a device status word (synchronises st); *code = the word's value.
int read_status_word(int* word, cudaStream_t st, int* code);
// The no-alloc entry point's module status word on the current device.
int noalloc_status_word(int** out);
// A row-major u8 matrix [rows][row_bytes] (row_bytes a multiple of 128) as a TMA tensor map with boxes of
// 128 bytes x box_rows rows and the 128-byte swizzle (16-byte chunk c of row r lands at chunk c ^ (r & 7)).
bool encode_u8_map_sw128(CUtensorMap* map, const void* base, int rows, int row_bytes, int box_rows);
// Argument checks shared by the linear entry points (DFSSM_OK or the status to return).
int check_linear(const dfssm_linear_t* L);
// Records e as the text returned by dfssm_last_cuda_error (this thread) and returns DFSSM_ECUDA.
int record_cuda_failure(cudaError_t e);
}  // namespace dfssm
