// dfssm_linear_decode_noalloc: the batch-B decode of one DF-SSM linear, for callers that can pass the
// library their inputs and outputs but cannot give it any other device memory.
//
// Who cannot allocate: code whose device memory is owned by someone else — a plugin inside a framework or
// an inference server whose host process manages every device allocation and hands the plugin only the
// tensors of the call — and real-time loops in which cudaMalloc is not allowed, because it can block and
// synchronise the device at an unpredictable moment.  dfssm_linear_decode needs a caller workspace for
// the hand-off between its quantize kernel and its GEMV kernel; this entry point keeps that hand-off in a
// fixed array in the library's own device memory instead, and calls no allocating routine.
//
// The array (kScratchBytes, enough for B <= 16 tokens of d_in <= 8192) is a module global: every device
// that loads the library holds it until the process exits.  All calls on a device share it and each call
// overwrites it before reading it (the quantize kernel writes every code, scale, code sum and LoRA
// intermediate that the GEMV kernel then reads), so nothing has to start at zero; two calls that overlap on the GPU
// (different streams, no ordering between them) race on it.
//
// In host code the array's name is only a host-side stand-in, not a device address.  The device address
// is looked up with cudaGetSymbolAddress the first time this entry point runs on a device (with that
// device current) and cached; that first call on each device should therefore come before any stream
// capture, and the library must not be used across a cudaDeviceReset of that device.  A timed-out wait
// of the streaming kernel on this path is recorded in a module status word beside the array (read by
// dfssm_device_status with a NULL workspace).

#include <cstdio>
#include <mutex>

#include "common.cuh"
#include "internal.h"

namespace {

constexpr int kMaxTokens = DFSSM_MAX_BATCH;  // 16
constexpr int kMaxDin = 8192;
// Same layout as the workspace of dfssm_linear_decode: codes [B][d_in], then the per-token scale,
// code sum and LoRA-down sums, each in its own 256-byte-aligned block.
constexpr size_t kScratchBytes = (size_t)kMaxTokens * kMaxDin + 256 + 256 + 1024;

static __device__ __align__(256) unsigned char g_linear_scratch[kScratchBytes];
// This entry point's status word (a timed-out wait of the streaming kernel; read and cleared by
// dfssm_device_status with a NULL workspace).
static __device__ int g_noalloc_status;

constexpr int kMaxDevices = 64;
void* g_scratch_addr[kMaxDevices] = {};
std::mutex g_scratch_mu;

bool aligned_to(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

void* g_status_addr[kMaxDevices] = {};

// Device addresses of g_linear_scratch and g_noalloc_status on the current device (looked up once per
// device; the cache assumes the device's context lives as long as the process: no cudaDeviceReset).
int module_addresses(void** scratch, int** status) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return dfssm::record_cuda_failure(e);
  if (dev < 0 || dev >= kMaxDevices) return DFSSM_EUNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (g_scratch_addr[dev] == nullptr) {
    void* p = nullptr;
    void* q = nullptr;
    e = cudaGetSymbolAddress(&p, g_linear_scratch);
    if (e == cudaSuccess) e = cudaGetSymbolAddress(&q, g_noalloc_status);
    if (e != cudaSuccess) return dfssm::record_cuda_failure(e);
    g_scratch_addr[dev] = p;
    g_status_addr[dev] = q;
  }
  if (scratch) *scratch = g_scratch_addr[dev];
  if (status) *status = static_cast<int*>(g_status_addr[dev]);
  return DFSSM_OK;
}

}  // namespace

int dfssm::noalloc_status_word(int** out) { return module_addresses(nullptr, out); }

extern "C" int dfssm_linear_decode_noalloc(const dfssm_linear_t* lin, const float* x, int B, float* y,
                                           const dfssm_debug_t* dbg, void* stream) {
  int st = dfssm::check_linear(lin);
  if (st) return st;
  if (!x || !y || B < 1) return DFSSM_EINVAL;
  if (B > kMaxTokens) return DFSSM_EUNSUPPORTED;
  if (dfssm::quant_scratch_bytes(B, lin->d_in) > kScratchBytes) return DFSSM_EUNSUPPORTED;
  if (!aligned_to(x, 16) || !aligned_to(y, 4)) return DFSSM_EALIGN;
  int dev = 0, major = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
      major != 10)
    return DFSSM_EDEVICE;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  void* scratch = nullptr;
  int* status = nullptr;
  st = module_addresses(&scratch, &status);
  if (st) return st;
  // in the streaming kernel's range the single kernel needs no scratch (only the status word)
  if (dfssm::stream_supported(lin->d_in, B))
    return dfssm::launch_linear_stream(lin, 1, x, B, &y, dbg, status, s);

  const dfssm::QuantScratch qs = dfssm::carve_quant_scratch(scratch, B, lin->d_in);
  dfssm::QuantArgs qa{};
  qa.x = x;
  qa.ldx = lin->d_in;
  qa.norm_w = nullptr;
  qa.n = lin->d_in;
  qa.B = B;
  qa.lora_b = lin->lora_b;
  qa.lora_b_scale = lin->lora_b_scale;
  qa.rank = lin->rank;
  qa.permute = true;
  qa.out = qs;
  if (dbg) {
    qa.dbg_xq = dbg->xq;
    qa.dbg_s = dbg->xscale;
    qa.dbg_t = dbg->lora_t;
  }
  cudaError_t e = dfssm::launch_quant(qa, s);
  if (e != cudaSuccess) return dfssm::record_cuda_failure(e);
  dfssm::GemvArgs ga{};
  ga.bits = lin->bits;
  ga.w_scale = lin->w_scale;
  ga.lora_a = lin->lora_a;
  ga.lora_a_scale = lin->lora_a_scale;
  ga.lora_b_scale = lin->lora_b_scale;
  ga.rank = lin->rank;
  ga.d_out = lin->d_out;
  ga.d_in = lin->d_in;
  ga.B = B;
  ga.in = qs;
  ga.y = y;
  ga.ldy = lin->d_out;
  ga.dbg_acc = dbg ? dbg->acc : nullptr;
  e = dfssm::launch_gemv(ga, s);
  if (e != cudaSuccess) return dfssm::record_cuda_failure(e);
  return DFSSM_OK;
}
