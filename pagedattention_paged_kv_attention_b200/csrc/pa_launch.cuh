// pa_launch.cuh -- host-side launch of the attention kernels for one (query dtype, cache dtype) pair.
// Included by the per-dtype translation units so that their template instantiations compile in
// parallel.
#pragma once

#include <cuda_runtime.h>

#include "pa_attention.cuh"
#include "pa_host_util.h"

namespace pa {

template <typename QT, typename KVT, int D, int G, bool BS = false>
cudaError_t launch_attention_one(const CUtensorMap& tk, const CUtensorMap& tv, const AttnArgs& a, int grid,
                                 cudaStream_t stream) {
  constexpr int EB = Elem<KVT>::kBytes;
  constexpr size_t smem = Layout<QT, D, G, EB>::kAllocBytes;
  auto kernel = paged_attention_main<QT, KVT, D, G, BS>;
  // The attribute is per device; setting it on every call costs a few microseconds of host time at
  // most and keeps multi-device processes correct.
  cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  e = pa_host::launch_overlapped(kernel, dim3(grid), dim3(kThreads), smem, stream, tk, tv, a);
  if (e != cudaSuccess) return e;
  if (a.num_partitions > 1) {
    const long rows = static_cast<long>(a.num_heads) * a.num_seqs;
    if (a.num_partitions > kReduceSplitAbove)
      e = pa_host::launch_overlapped(paged_attention_reduce<QT, D, true>, dim3(static_cast<unsigned>(rows)),
                                     dim3(kReduceWarps * 32), 0, stream, a);
    else {
      const dim3 grid(static_cast<unsigned>((rows + kReduceWarps - 1) / kReduceWarps));
      if (a.num_partitions <= 4)
        e = pa_host::launch_overlapped(paged_attention_reduce<QT, D, false, 4>, grid, dim3(kReduceWarps * 32), 0,
                                       stream, a);
      else if (a.num_partitions <= 8)
        e = pa_host::launch_overlapped(paged_attention_reduce<QT, D, false, 8>, grid, dim3(kReduceWarps * 32), 0,
                                       stream, a);
      else
        e = pa_host::launch_overlapped(paged_attention_reduce<QT, D, false, 16>, grid, dim3(kReduceWarps * 32), 0,
                                       stream, a);
    }
  }
  return e;
}

template <typename QT, typename KVT>
cudaError_t launch_attention(const CUtensorMap& tk, const CUtensorMap& tv, const AttnArgs& a, int D, int G,
                             int grid, cudaStream_t stream) {
  if constexpr (sizeof(KVT) == 1) {
    if (D == 128 && a.scale_block_stride != 0) {  // per-block scales
      switch (G) {
        case 1: return launch_attention_one<QT, KVT, 128, 1, true>(tk, tv, a, grid, stream);
        case 2: return launch_attention_one<QT, KVT, 128, 2, true>(tk, tv, a, grid, stream);
        case 4: return launch_attention_one<QT, KVT, 128, 4, true>(tk, tv, a, grid, stream);
        case 8: return launch_attention_one<QT, KVT, 128, 8, true>(tk, tv, a, grid, stream);
      }
    } else if (D == 128) {
      switch (G) {
        case 1: return launch_attention_one<QT, KVT, 128, 1>(tk, tv, a, grid, stream);
        case 2: return launch_attention_one<QT, KVT, 128, 2>(tk, tv, a, grid, stream);
        case 4: return launch_attention_one<QT, KVT, 128, 4>(tk, tv, a, grid, stream);
        case 8: return launch_attention_one<QT, KVT, 128, 8>(tk, tv, a, grid, stream);
      }
    }
  } else {
    if (D == 128) {
      switch (G) {
        case 1: return launch_attention_one<QT, KVT, 128, 1>(tk, tv, a, grid, stream);
        case 2: return launch_attention_one<QT, KVT, 128, 2>(tk, tv, a, grid, stream);
        case 4: return launch_attention_one<QT, KVT, 128, 4>(tk, tv, a, grid, stream);
        case 8: return launch_attention_one<QT, KVT, 128, 8>(tk, tv, a, grid, stream);
      }
    } else if (D == 64) {
      switch (G) {
        case 1: return launch_attention_one<QT, KVT, 64, 1>(tk, tv, a, grid, stream);
        case 2: return launch_attention_one<QT, KVT, 64, 2>(tk, tv, a, grid, stream);
        case 4: return launch_attention_one<QT, KVT, 64, 4>(tk, tv, a, grid, stream);
        case 8: return launch_attention_one<QT, KVT, 64, 8>(tk, tv, a, grid, stream);
      }
    }
  }
  return cudaErrorInvalidValue;
}

// Per-dtype entry points (defined in pa_attention_<dtype>.cu).
cudaError_t launch_attention_bf16(const CUtensorMap& tk, const CUtensorMap& tv, const AttnArgs& a, bool fp8_cache,
                                  int D, int G, int grid, cudaStream_t stream);
cudaError_t launch_attention_f16(const CUtensorMap& tk, const CUtensorMap& tv, const AttnArgs& a, bool fp8_cache,
                                 int D, int G, int grid, cudaStream_t stream);

}  // namespace pa
