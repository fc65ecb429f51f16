// pa_static_workspace.cu -- pa_paged_attention_static: paged attention whose scratch memory is a
// fixed array inside the library instead of a workspace the caller allocates.
//
// Who needs it: callers that cannot call cudaMalloc -- plugins hosted by an engine that owns every
// byte of device memory, and serving loops that must not allocate (or pay cudaMalloc's implicit
// device synchronisation) once they are running. They still pass their inputs and outputs.
//
// The array below is reserved on every GPU that loads this library, for as long as the process
// runs. In host code its name is only a host-side stand-in, never a device address (handing it to a
// kernel would fault, or silently touch the wrong memory on systems where the GPU can reach host
// memory), so the device address is looked up with cudaGetSymbolAddress, once per device, with that
// device current, and passed to the kernels as their workspace.
#include <cuda_runtime.h>

#include <mutex>

#include "pagedattn.h"

namespace {

__device__ __align__(256) unsigned char g_static_workspace[PA_STATIC_WORKSPACE_BYTES];

constexpr int kMaxDevices = 64;
void* g_static_address[kMaxDevices] = {};
std::mutex g_static_mutex;

// Device address of g_static_workspace on the current device; the first call on a device looks it
// up (the one-time set-up), later calls reuse it.
cudaError_t static_workspace_address(void** address) {
  int device = 0;
  cudaError_t e = cudaGetDevice(&device);
  if (e != cudaSuccess) return e;
  if (device < 0 || device >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_static_mutex);
  if (g_static_address[device] == nullptr) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_static_workspace);
    if (e != cudaSuccess) return e;
    g_static_address[device] = p;
  }
  *address = g_static_address[device];
  return cudaSuccess;
}

}  // namespace

extern "C" pa_status pa_paged_attention_static(void* out, const void* query, pa_dtype q_dtype,
                                               const void* key_cache, const void* value_cache, pa_dtype kv_dtype,
                                               const float* k_scale, const float* v_scale,
                                               const int32_t* block_tables, int max_blocks_per_seq,
                                               const int32_t* context_lens, int num_seqs, int num_heads,
                                               int num_kv_heads, int head_size, int block_size, int num_blocks,
                                               int max_context_len, float scale, int partition_size,
                                               unsigned int* device_error_out, pa_stream_t stream) {
  // Host-only size check first: nothing is enqueued for a request that does not fit.
  const size_t need = pa_paged_attention_workspace_size(num_seqs, num_heads, num_kv_heads, head_size,
                                                        max_context_len, partition_size);
  if (need == 0) return PA_ERR_INVALID_ARGUMENT;
  if (need > PA_STATIC_WORKSPACE_BYTES) return PA_ERR_WORKSPACE_TOO_SMALL;
  if (num_seqs == 0) return PA_OK;
  if (device_error_out && reinterpret_cast<uintptr_t>(device_error_out) % alignof(unsigned int) != 0)
    return PA_ERR_INVALID_ARGUMENT;

  void* workspace = nullptr;
  if (static_workspace_address(&workspace) != cudaSuccess) return PA_ERR_CUDA;
  const pa_status status = pa_paged_attention(out, query, q_dtype, key_cache, value_cache, kv_dtype, k_scale, v_scale,
                                              block_tables, max_blocks_per_seq, context_lens, num_seqs, num_heads,
                                              num_kv_heads, head_size, block_size, num_blocks, max_context_len,
                                              scale, partition_size, workspace, PA_STATIC_WORKSPACE_BYTES, stream);
  if (status != PA_OK) return status;
  // The error word starts at zero (the array is zero when the library loads) and is handed out and
  // cleared after every call, so the next call starts from zero again.
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (device_error_out &&
      cudaMemcpyAsync(device_error_out, workspace, sizeof(unsigned int), cudaMemcpyDeviceToDevice, st) != cudaSuccess)
    return PA_ERR_CUDA;
  if (cudaMemsetAsync(workspace, 0, sizeof(unsigned int), st) != cudaSuccess) return PA_ERR_CUDA;
  return PA_OK;
}
