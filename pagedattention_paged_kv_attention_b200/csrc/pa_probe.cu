// pa_probe.cu -- read-bandwidth probes (include/pa_probe.h): a sequential stream and a read of exactly
// the K/V rows a paged decode batch needs, both with 16-byte loads and no compute. They give the
// ceilings the decode kernel is measured against (page "PagedAttention 与连续批处理：LLM Serving 的底层
// 架构拆解", section "对 agent 开发者的启示": decode is memory-bound).
#include <cuda_runtime.h>

#include <cstdint>

#include "pa_host_util.h"
#include "pa_probe.h"

namespace {

constexpr int kStreamThreads = 512;
constexpr int kStreamCtasPerSm = 4;
constexpr int kPagedThreads = 256;
constexpr int kUnroll = 4;
constexpr uint32_t kNeverValue = 0x9e3779b9u;  // the fold almost never equals it; a write then is harmless

__device__ __forceinline__ uint4 load_stream(const uint4* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

__device__ __forceinline__ uint32_t fold(uint4 v) { return v.x ^ v.y ^ v.z ^ v.w; }

// Grid-stride over the 16-byte vectors; each thread keeps kUnroll loads in flight.
__device__ __forceinline__ uint32_t read_range(const uint4* base, size_t n16, size_t first, size_t stride) {
  uint32_t acc = 0;
  size_t i = first;
  for (; i + (kUnroll - 1) * stride < n16; i += kUnroll * stride) {
    uint4 v[kUnroll];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) v[u] = load_stream(base + i + u * stride);
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) acc ^= fold(v[u]);
  }
  for (; i < n16; i += stride) acc ^= fold(load_stream(base + i));
  return acc;
}

__global__ void __launch_bounds__(kStreamThreads) stream_read_kernel(const uint4* buf, size_t n16, int repeat,
                                                                      unsigned long long* sink) {
  const size_t first = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  const size_t stride = static_cast<size_t>(gridDim.x) * blockDim.x;
  uint32_t acc = 0;
  for (int r = 0; r < repeat; ++r) acc ^= read_range(buf, n16, first, stride) + static_cast<uint32_t>(r);
  if (acc == kNeverValue) atomicAdd(sink, 1ull);
}

// CTA (j, s): logical block j of sequence s, its valid token rows of K and of V (contiguous runs).
__global__ void __launch_bounds__(kPagedThreads) paged_read_kernel(const uint8_t* key_cache, const uint8_t* value_cache,
                                                                    const int32_t* block_tables, int max_blocks_per_seq,
                                                                    const int32_t* context_lens, int block_size,
                                                                    int num_blocks, size_t token_bytes,
                                                                    unsigned long long* sink) {
  const int j = static_cast<int>(blockIdx.x);
  const int s = static_cast<int>(blockIdx.y);
  const int L = context_lens[s];
  if (L <= 0 || static_cast<long long>(L) > static_cast<long long>(max_blocks_per_seq) * block_size) return;
  const int tok0 = j * block_size;
  if (tok0 >= L) return;
  const int blk = block_tables[static_cast<size_t>(s) * max_blocks_per_seq + j];
  if (blk < 0 || blk >= num_blocks) return;
  const int ntok = min(block_size, L - tok0);
  const size_t n16 = ntok * token_bytes / 16;
  const size_t off = static_cast<size_t>(blk) * block_size * token_bytes;
  uint32_t acc = read_range(reinterpret_cast<const uint4*>(key_cache + off), n16, threadIdx.x, blockDim.x);
  acc ^= read_range(reinterpret_cast<const uint4*>(value_cache + off), n16, threadIdx.x, blockDim.x);
  if (acc == kNeverValue) atomicAdd(sink, 1ull);
}

cudaError_t sm_count(int* sms) {
  int device = 0;
  cudaError_t e = cudaGetDevice(&device);
  if (e != cudaSuccess) return e;
  e = cudaDeviceGetAttribute(sms, cudaDevAttrMultiProcessorCount, device);
  if (e == cudaSuccess && *sms <= 0) e = cudaErrorInvalidDevice;
  return e;
}

}  // namespace

extern "C" pa_status pa_probe_stream_read(const void* buf, size_t bytes, int repeat, unsigned long long* sink,
                                          pa_stream_t stream) {
  if (!buf || !sink || !pa_host::aligned(buf, 16) || !pa_host::aligned(sink, 8) || bytes == 0 || bytes % 16 != 0 ||
      repeat < 1 || repeat > 4096)
    return PA_ERR_INVALID_ARGUMENT;
  int sms = 0;
  if (sm_count(&sms) != cudaSuccess) return PA_ERR_CUDA;
  const cudaError_t e =
      pa_host::launch_plain(stream_read_kernel, dim3(static_cast<unsigned>(sms * kStreamCtasPerSm)),
                            dim3(kStreamThreads), 0, reinterpret_cast<cudaStream_t>(stream),
                            static_cast<const uint4*>(buf), bytes / 16, repeat, sink);
  return e == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

extern "C" pa_status pa_probe_paged_read(const void* key_cache, const void* value_cache, pa_dtype kv_dtype,
                                         const int32_t* block_tables, int max_blocks_per_seq,
                                         const int32_t* context_lens, int num_seqs, int num_kv_heads, int head_size,
                                         int block_size, int num_blocks, unsigned long long* sink,
                                         pa_stream_t stream) {
  if (num_seqs < 0 || num_kv_heads <= 0 || head_size <= 0 || block_size <= 0 || num_blocks <= 0 ||
      max_blocks_per_seq <= 0 || !pa_host::is_dtype(kv_dtype))
    return PA_ERR_INVALID_ARGUMENT;
  if (num_seqs == 0) return PA_OK;
  if (!key_cache || !value_cache || !block_tables || !context_lens || !sink || !pa_host::aligned(key_cache, 16) ||
      !pa_host::aligned(value_cache, 16) || !pa_host::aligned(block_tables, 4) || !pa_host::aligned(context_lens, 4) ||
      !pa_host::aligned(sink, 8))
    return PA_ERR_INVALID_ARGUMENT;
  const size_t token_bytes = static_cast<size_t>(num_kv_heads) * head_size * pa_host::elem_bytes(kv_dtype);
  if (token_bytes % 16 != 0 || num_seqs > 65535) return PA_ERR_UNSUPPORTED;
  const cudaError_t e = pa_host::launch_plain(
      paged_read_kernel, dim3(static_cast<unsigned>(max_blocks_per_seq), static_cast<unsigned>(num_seqs)),
      dim3(kPagedThreads), 0, reinterpret_cast<cudaStream_t>(stream), static_cast<const uint8_t*>(key_cache),
      static_cast<const uint8_t*>(value_cache), block_tables, max_blocks_per_seq, context_lens, block_size,
      num_blocks, token_bytes, sink);
  return e == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}
