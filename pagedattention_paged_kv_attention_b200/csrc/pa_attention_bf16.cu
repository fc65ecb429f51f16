// Attention kernels instantiated for bfloat16 queries (bfloat16 or FP8-E4M3 caches).
#include "pa_launch.cuh"

namespace pa {
cudaError_t launch_attention_bf16(const CUtensorMap& tk, const CUtensorMap& tv, const AttnArgs& a, bool fp8_cache,
                                  int D, int G, int grid, cudaStream_t stream) {
  if (fp8_cache) return launch_attention<__nv_bfloat16, __nv_fp8_e4m3>(tk, tv, a, D, G, grid, stream);
  return launch_attention<__nv_bfloat16, __nv_bfloat16>(tk, tv, a, D, G, grid, stream);
}
}  // namespace pa
