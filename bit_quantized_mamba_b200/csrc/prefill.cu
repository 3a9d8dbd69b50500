// Prefill of one DF-SSM linear on int8 tcgen05 tensor cores (placeholder until the kernel lands).
#include "common.cuh"
#include "internal.h"

namespace dfssm {
size_t prefill_workspace_bytes(int M, int d_in, int d_out) {
  (void)M; (void)d_in; (void)d_out;
  return 256;
}
}  // namespace dfssm

extern "C" int dfssm_linear_prefill(const dfssm_linear_t* lin, const float* x, int M, float* y,
                                    void* workspace, size_t ws_bytes, const dfssm_debug_t* dbg,
                                    void* stream) {
  (void)lin; (void)x; (void)M; (void)y; (void)workspace; (void)ws_bytes; (void)dbg; (void)stream;
  return DFSSM_EUNSUPPORTED;
}
