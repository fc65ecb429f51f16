// pa_host_util.h -- host helpers shared by the C-ABI translation units: argument checks, sizes and
// the driver's tensor-map encoder (fetched through the runtime, so no libcuda link is needed).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <cstdint>
#include <mutex>
#include <utility>

#include "pagedattn.h"

namespace pa_host {

inline bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }
inline size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }
// ceil(a / b) for a >= 0, b > 0, without forming a + b - 1 (which overflows near INT_MAX).
inline int ceil_div(int a, int b) { return a / b + (a % b != 0); }
inline bool is_16bit(pa_dtype t) { return t == PA_F16 || t == PA_BF16; }
inline bool is_fp8(pa_dtype t) { return t == PA_FP8_E4M3 || t == PA_FP8_E4M3_BLOCK; }
inline bool is_dtype(pa_dtype t) { return t == PA_F16 || t == PA_BF16 || is_fp8(t); }
inline int elem_bytes(pa_dtype t) { return is_fp8(t) ? 1 : 2; }
// Scale index stride per block: 0 for per-kv-head scales, num_kv_heads for per-(block, kv head) ones.
inline int scale_block_stride(pa_dtype t, int num_kv_heads) { return t == PA_FP8_E4M3_BLOCK ? num_kv_heads : 0; }

inline PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// Launch with programmatic stream serialisation: the kernel may be scheduled while the previous kernel
// in the stream is still running. Every kernel launched this way begins with grid_dependency_wait()
// (pa_device.cuh) before any global-memory access, so stream order holds for memory and only the
// launch latency and the shared-memory prologue overlap the previous kernel.
template <typename... Params, typename... Args>
cudaError_t launch_overlapped(void (*kernel)(Params...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                              Args&&... args) {
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// Ordinary launch (full stream serialisation) whose status is the launch's own: unlike <<<>>> followed
// by cudaGetLastError, it neither reports nor clears an earlier error left by the caller's code.
template <typename... Params, typename... Args>
cudaError_t launch_plain(void (*kernel)(Params...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                         Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cfg.attrs = nullptr;
  cfg.numAttrs = 0;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// Every argument check of pa_paged_attention except those on the workspace, with no CUDA call. On
// PA_OK, *workspace_bytes is the workspace the call needs and *empty tells whether the call has
// nothing to do (num_seqs == 0). Defined in pa_api.cu; pa_paged_attention_static runs it before
// comparing that size with its fixed array.
pa_status paged_attention_check(const void* out, const void* query, pa_dtype q_dtype, const void* key_cache,
                                const void* value_cache, pa_dtype kv_dtype, const float* k_scale,
                                const float* v_scale, const int32_t* block_tables, int max_blocks_per_seq,
                                const int32_t* context_lens, int num_seqs, int num_heads, int num_kv_heads,
                                int head_size, int block_size, int num_blocks, int max_context_len, float scale,
                                int partition_size, size_t* workspace_bytes, bool* empty);

}  // namespace pa_host
