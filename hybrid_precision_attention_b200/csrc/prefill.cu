// prefill.cu — hybrid-precision causal prefill (placeholder until the tcgen05 kernel lands).
#include "common.cuh"

namespace hq {
size_t prefill_workspace(int B, int Hq, int Hkv, int L) { return 256; }
hq_status launch_prefill(int, int, int, int, const uint16_t*, const uint16_t*, const uint16_t*, const int32_t*, int, int, int,
                         float, uint16_t*, void*, cudaStream_t) {
  return HQ_ERR_UNSUPPORTED;
}
}  // namespace hq
