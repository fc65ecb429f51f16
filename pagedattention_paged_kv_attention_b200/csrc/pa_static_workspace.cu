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
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <mutex>

#include "pa_host_util.h"
#include "pagedattn.h"

namespace {

__device__ __align__(256) unsigned char g_static_workspace[PA_STATIC_WORKSPACE_BYTES];

constexpr int kMaxDevices = 64;
struct StaticAddress {
  CUcontext context;  // the context the address was looked up in
  void* address;
};
StaticAddress g_static_address[kMaxDevices] = {};
std::mutex g_static_mutex;

// cuCtxGetCurrent through the runtime's driver entry point (no link against libcuda).
PFN_cuCtxGetCurrent_v4000 context_query() {
  static PFN_cuCtxGetCurrent_v4000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(p);
  });
  return fn;
}

// Device address of g_static_workspace in the current device's current context. The first call on a
// device looks it up (the one-time set-up); later calls reuse it while the same context is current,
// and look it up again when another context has become current on that device.
cudaError_t static_workspace_address(void** address) {
  int device = 0;
  cudaError_t e = cudaGetDevice(&device);
  if (e != cudaSuccess) return e;
  if (device < 0 || device >= kMaxDevices) return cudaErrorInvalidDevice;
  const PFN_cuCtxGetCurrent_v4000 query = context_query();
  if (!query) return cudaErrorDeviceUninitialized;
  CUcontext ctx = nullptr;
  if (query(&ctx) != CUDA_SUCCESS) return cudaErrorDeviceUninitialized;
  std::lock_guard<std::mutex> lock(g_static_mutex);
  StaticAddress& slot = g_static_address[device];
  if (ctx == nullptr || slot.address == nullptr || slot.context != ctx) {
    // The lookup also binds the device's primary context to this thread when none was current yet.
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_static_workspace);
    if (e != cudaSuccess) return e;
    if (query(&ctx) != CUDA_SUCCESS || ctx == nullptr) return cudaErrorDeviceUninitialized;
    slot.context = ctx;
    slot.address = p;
  }
  *address = slot.address;
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
  // Host-only checks first, in the order pa_paged_attention makes them, then the size of the fixed
  // array: nothing is enqueued for a request that is invalid or does not fit.
  size_t need = 0;
  bool empty = false;
  const pa_status checked = pa_host::paged_attention_check(
      out, query, q_dtype, key_cache, value_cache, kv_dtype, k_scale, v_scale, block_tables, max_blocks_per_seq,
      context_lens, num_seqs, num_heads, num_kv_heads, head_size, block_size, num_blocks, max_context_len, scale,
      partition_size, &need, &empty);
  if (checked != PA_OK) return checked;
  if (device_error_out && !pa_host::aligned(device_error_out, alignof(unsigned int))) return PA_ERR_INVALID_ARGUMENT;
  if (empty) return PA_OK;
  if (need > PA_STATIC_WORKSPACE_BYTES) return PA_ERR_WORKSPACE_TOO_SMALL;

  void* workspace = nullptr;
  if (static_workspace_address(&workspace) != cudaSuccess) return PA_ERR_CUDA;
  const pa_status status = pa_paged_attention(out, query, q_dtype, key_cache, value_cache, kv_dtype, k_scale, v_scale,
                                              block_tables, max_blocks_per_seq, context_lens, num_seqs, num_heads,
                                              num_kv_heads, head_size, block_size, num_blocks, max_context_len,
                                              scale, partition_size, workspace, PA_STATIC_WORKSPACE_BYTES, stream);
  // The error word starts at zero (the array is zero when the library loads). Whatever the call's
  // status -- a later launch can fail after an earlier kernel was enqueued -- the word is handed out
  // and cleared, so the next call starts from zero again.
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  bool copied = true;
  if (device_error_out)
    copied = cudaMemcpyAsync(device_error_out, workspace, sizeof(unsigned int), cudaMemcpyDeviceToDevice, st) ==
             cudaSuccess;
  const bool cleared = cudaMemsetAsync(workspace, 0, sizeof(unsigned int), st) == cudaSuccess;
  if (status != PA_OK) return status;
  return copied && cleared ? PA_OK : PA_ERR_CUDA;
}
