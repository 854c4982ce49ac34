// bf16 tcgen05 sparse MQA attention (placeholder until the kernel lands).
#include "internal.h"
namespace dsa {
AttnPlan attn_bf16_plan(int, int, int) { return AttnPlan{256, 8}; }
size_t attn_bf16_workspace(int, int, int) { return 0; }
cudaError_t launch_attn_bf16(const void *, const void *, int, float, const int *, int, const Layout &, void *, float *,
                             void *, size_t, const ErrCtx &, int, cudaStream_t) {
  return cudaErrorNotSupported;
}
}  // namespace dsa
