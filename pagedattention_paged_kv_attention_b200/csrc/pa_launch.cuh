// pa_launch.cuh -- host-side launch of the attention kernels for one (query dtype, cache dtype) pair.
// Included by the per-dtype translation units so that their template instantiations compile in
// parallel.
#pragma once

#include <cuda_runtime.h>

#include "pa_attention.cuh"

namespace pa {

// Dynamic shared memory of paged_attention_main<.., D, G> with `stages` ring slots (matches the
// kernel's layout: 1024 bytes of alignment slack, the ring, P and alpha buffers, the mbarriers and
// a flag word).
template <int D, int G, int EB>
constexpr size_t attention_smem_bytes(int stages) {
  using S = Shape<D, G, EB>;
  return 1024 + static_cast<size_t>(stages) * S::kStageBytes + kConsumerWarps * kStageTokens * G * 4 +
         kConsumerWarps * G * 4 + 8 + 2 * static_cast<size_t>(stages) * 8 + 16;
}

// Ring depth: as many 64-token stages as fit the per-CTA share of the SM's shared memory (about
// 200 KB for the ring when one CTA runs per SM, half of that when two do), rounded down to a multiple
// of the consumer-warp count. Stage j goes to slot j % depth and to warp j % kConsumerWarps, so with
// depth % kConsumerWarps == 0 every slot is only ever consumed by one warp, which finishes round r of
// the slot before it waits on round r + 1 (an mbarrier parity wait cannot tell round r + 2 from r).
#ifndef PA_RING_BYTES_PER_SM
#define PA_RING_BYTES_PER_SM (200 * 1024)
#endif
template <int D, int G, int EB>
constexpr int attention_stages() {
  constexpr int fit = PA_RING_BYTES_PER_SM / min_ctas_per_sm<G>() / Shape<D, G, EB>::kStageBytes;
  constexpr int capped = fit > kMaxStages ? kMaxStages : fit;
  constexpr int n = capped / kConsumerWarps * kConsumerWarps;
  static_assert(n >= kConsumerWarps, "ring must hold one stage per consumer warp");
  return n;
}

template <typename QT, typename KVT, int D, int G>
cudaError_t launch_attention_one(const CUtensorMap& tk, const CUtensorMap& tv, AttnArgs a, dim3 grid,
                                 cudaStream_t stream) {
  constexpr int EB = Elem<KVT>::kBytes;
  a.num_stages = attention_stages<D, G, EB>();
  const size_t smem = attention_smem_bytes<D, G, EB>(a.num_stages);
  auto kernel = paged_attention_main<QT, KVT, D, G>;
  static size_t configured = 0;  // per instantiation; the attribute only ever grows
  if (smem > configured) {
    cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    configured = smem;
  }
  kernel<<<grid, kThreads, smem, stream>>>(tk, tv, a);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  if (a.num_partitions > 1) {
    paged_attention_reduce<QT, D><<<dim3(a.num_heads, a.num_seqs), D, 0, stream>>>(a);
    e = cudaGetLastError();
  }
  return e;
}

template <typename QT, typename KVT>
cudaError_t launch_attention(const CUtensorMap& tk, const CUtensorMap& tv, const AttnArgs& a, int D, int G,
                             dim3 grid, cudaStream_t stream) {
  if constexpr (sizeof(KVT) == 1) {
    if (D == 128) {
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
                                  int D, int G, dim3 grid, cudaStream_t stream);
cudaError_t launch_attention_f16(const CUtensorMap& tk, const CUtensorMap& tv, const AttnArgs& a, bool fp8_cache,
                                 int D, int G, dim3 grid, cudaStream_t stream);

}  // namespace pa
