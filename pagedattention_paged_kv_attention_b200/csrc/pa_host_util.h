// pa_host_util.h -- host helpers shared by the C-ABI translation units: argument checks, sizes and
// the driver's tensor-map encoder (fetched through the runtime, so no libcuda link is needed).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <cstdint>
#include <mutex>

#include "pagedattn.h"

namespace pa_host {

inline bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }
inline size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }
inline int ceil_div(int a, int b) { return (a + b - 1) / b; }
inline bool is_16bit(pa_dtype t) { return t == PA_F16 || t == PA_BF16; }
inline bool is_dtype(pa_dtype t) { return t == PA_F16 || t == PA_BF16 || t == PA_FP8_E4M3; }
inline int elem_bytes(pa_dtype t) { return t == PA_FP8_E4M3 ? 1 : 2; }

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

}  // namespace pa_host
