// pa_api.cu -- the C ABI of libpagedattn.so (declared and documented in include/pagedattn.h).
//
// Host side only: argument validation (before any CUDA call), launch planning (partition size, grid,
// workspace layout), TMA descriptor encoding and dispatch to the kernels. Nothing here allocates
// device memory; every buffer belongs to the caller (tutorial page "企业官网建设流程全解析", sec. 3.2
// "关键性能优化": the block pool is preallocated at start-up; work is issued asynchronously on CUDA
// streams).
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <mutex>
#include <unordered_set>

#include "pa_cache_ops.cuh"
#include "pa_host_util.h"
#include "pa_launch.cuh"
#include "pagedattn.h"

namespace {

// Automatic partition size. With the kernel's longest-first work order, a sweep on the B200 put the
// best size where each persistent CTA gets about five items if every context were max_context_len
// long (fewer, larger items mean fewer split-K partials to write and merge; the order keeps the tail
// short), and never more than 32 partitions (the merge's cost grows with them): 768 for the 70B-shape
// batch, 512-768 for 7B, 1024 for 8 x 32768 tokens.
constexpr int kPlanSMs = 148;            // B200 SM count; planning is a pure function of the sizes
constexpr int kPlanItemsPerCta = 5;
constexpr int kPlanMaxPartitions = 32;
constexpr int kMinAutoPartition = 256;

using pa_host::aligned;
using pa_host::ceil_div;
using pa_host::elem_bytes;
using pa_host::is_16bit;
using pa_host::is_dtype;
using pa_host::is_fp8;
using pa_host::scale_block_stride;
using pa_host::round_up;
using pa_host::tensor_map_encoder;

// Query heads handled per CTA (the kernel template's G) and CTAs per kv head.
void group_tiling(int group, int* g_tile, int* subgroups) {
  int g = 1;
  while (g < group && g < 8) g *= 2;
  *g_tile = g;
  *subgroups = ceil_div(group, g);
}

int plan_partition(int num_seqs, int num_heads, int num_kv_heads, int max_context_len, int partition_size) {
  if (partition_size < 0) return -1;
  if (partition_size > 0) return (partition_size % pa::kPartitionQuantum == 0) ? partition_size : -1;
  if (num_seqs < 0 || num_heads <= 0 || num_kv_heads <= 0 || num_heads % num_kv_heads || max_context_len < 0)
    return -1;
  int g_tile, subgroups;
  group_tiling(num_heads / num_kv_heads, &g_tile, &subgroups);
  const long long units =
      std::max<long long>(1, static_cast<long long>(num_seqs) * ceil_div(num_kv_heads, pa::kHeadBlock) * subgroups);
  const long long ctx = std::max(1, max_context_len);
  const long long per_cta = static_cast<long long>(kPlanSMs) * kPlanItemsPerCta;
  const long long balance = (units * ctx + per_cta - 1) / per_cta;              // ~5 items per CTA
  const long long merge = (ctx + kPlanMaxPartitions - 1) / kPlanMaxPartitions;  // <= 32 partitions
  long long ps = std::max<long long>({balance, merge, static_cast<long long>(kMinAutoPartition)});
  ps = (ps + pa::kPartitionQuantum - 1) / pa::kPartitionQuantum * pa::kPartitionQuantum;
  // No split beyond the context itself (one partition covers it); stays within int.
  const long long whole = (ctx + pa::kPartitionQuantum - 1) / pa::kPartitionQuantum * pa::kPartitionQuantum;
  ps = std::min<long long>(ps, std::max<long long>(whole, kMinAutoPartition));
  ps = std::min<long long>(ps, 0x7fffffffLL / pa::kPartitionQuantum * pa::kPartitionQuantum);
  return static_cast<int>(ps);
}

struct WorkspaceLayout {
  size_t part_m, part_l, part_o, trace, total;
};

WorkspaceLayout workspace_layout(int num_seqs, int num_heads, int num_kv_heads, int head_size, int partitions) {
  WorkspaceLayout w{};
  w.total = PA_WORKSPACE_HEADER_BYTES;
  if (partitions > 1) {
    const size_t rows = static_cast<size_t>(num_seqs) * num_heads * partitions;
    w.part_m = w.total;
    w.part_l = w.part_m + round_up(rows * 4, 256);
    w.part_o = w.part_l + round_up(rows * 4, 256);
    w.total = w.part_o + round_up(rows * head_size * 4, 256);
  }
#ifdef PA_TRACE
  // Timing records of the trace build (pa::kTraceItemBase words, then 4 per work item) at the end.
  int g_tile, subgroups;
  group_tiling(num_heads / num_kv_heads, &g_tile, &subgroups);
  const size_t items = static_cast<size_t>(partitions) * num_seqs * ceil_div(num_kv_heads, pa::kHeadBlock) * subgroups;
  w.trace = w.total;
  w.total += round_up((pa::kTraceItemBase + 4 * items) * 8, 256);
#else
  (void)num_kv_heads;
#endif
  return w;
}

// 4-D view of a cache; box = one 128-byte chunk of the rows of 8 consecutive tokens for 8 consecutive
// kv heads of one block (heads past the last one read as zeros), written to shared memory with the
// 128-byte swizzle.
bool encode_cache_map(CUtensorMap* map, const void* cache, int elem_bytes, int head_size, int num_kv_heads,
                      int block_size, int num_blocks) {
  auto encode = tensor_map_encoder();
  if (!encode) return false;
  const cuuint64_t e = static_cast<cuuint64_t>(elem_bytes);
  // Dimensions in the order {d, token, kv head, block}: the token dimension (stride Hkv*d) is listed
  // before the head dimension (stride d), so a box lands in shared memory as [head][token][chunk].
  cuuint64_t dims[4] = {static_cast<cuuint64_t>(head_size), static_cast<cuuint64_t>(block_size),
                        static_cast<cuuint64_t>(num_kv_heads), static_cast<cuuint64_t>(num_blocks)};
  cuuint64_t strides[3] = {num_kv_heads * head_size * e, head_size * e, block_size * num_kv_heads * head_size * e};
  cuuint32_t box[4] = {static_cast<cuuint32_t>(128 / elem_bytes), static_cast<cuuint32_t>(pa::kBoxTokens),
                       static_cast<cuuint32_t>(pa::kHeadBlock), 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = encode(map, elem_bytes == 2 ? CU_TENSOR_MAP_DATA_TYPE_UINT16 : CU_TENSOR_MAP_DATA_TYPE_UINT8, 4,
                      const_cast<void*>(cache), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                      CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                      CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

bool supported_block_size(int bs) { return bs == 8 || bs == 16 || bs == 32 || bs == 64; }

// Elements of one token's [num_kv_heads][head_size] row that the cache-write kernels index with int.
constexpr int64_t kMaxRowElems = int64_t(1) << 24;

// The plan of a valid paged-attention call (sizes only; no pointer is dereferenced).
struct AttnPlan {
  bool empty;
  int ps, partitions, g_tile, subgroups, head_blocks;
  unsigned long long items;
  WorkspaceLayout ws;
};

pa_status check_attention(const void* out, const void* query, pa_dtype q_dtype, const void* key_cache,
                          const void* value_cache, pa_dtype kv_dtype, const float* k_scale, const float* v_scale,
                          const int32_t* block_tables, int max_blocks_per_seq, const int32_t* context_lens,
                          int num_seqs, int num_heads, int num_kv_heads, int head_size, int block_size,
                          int num_blocks, int max_context_len, float scale, int partition_size, AttnPlan* plan) {
  *plan = AttnPlan{};
  if (num_seqs < 0 || num_heads <= 0 || num_kv_heads <= 0 || num_heads % num_kv_heads != 0 ||
      head_size <= 0 || block_size <= 0 || num_blocks <= 0 || max_blocks_per_seq <= 0 || max_context_len < 0 ||
      partition_size < 0 || !std::isfinite(scale))
    return PA_ERR_INVALID_ARGUMENT;
  if (!is_dtype(q_dtype) || !is_dtype(kv_dtype) || !is_16bit(q_dtype)) return PA_ERR_INVALID_ARGUMENT;
  if (num_seqs == 0) {
    plan->empty = true;
    return PA_OK;
  }
  if (!out || !query || !key_cache || !value_cache || !block_tables || !context_lens) return PA_ERR_INVALID_ARGUMENT;
  if (!aligned(out, 16) || !aligned(query, 16) || !aligned(key_cache, 16) || !aligned(value_cache, 16) ||
      !aligned(block_tables, 4) || !aligned(context_lens, 4))
    return PA_ERR_INVALID_ARGUMENT;
  const bool fp8 = is_fp8(kv_dtype);
  if (fp8 && (!k_scale || !v_scale || !aligned(k_scale, 4) || !aligned(v_scale, 4))) return PA_ERR_INVALID_ARGUMENT;
  if (!fp8 && kv_dtype != q_dtype) return PA_ERR_UNSUPPORTED;
  if (head_size != 64 && head_size != 128) return PA_ERR_UNSUPPORTED;
  if (fp8 && head_size != 128) return PA_ERR_UNSUPPORTED;
  if (!supported_block_size(block_size)) return PA_ERR_UNSUPPORTED;
  if (num_blocks >= (1 << 27)) return PA_ERR_UNSUPPORTED;  // block ids ride in 28 bits of a stage message
  plan->ps = plan_partition(num_seqs, num_heads, num_kv_heads, max_context_len, partition_size);
  if (plan->ps <= 0) return PA_ERR_INVALID_ARGUMENT;
  plan->partitions = std::max(1, ceil_div(max_context_len, plan->ps));
  group_tiling(num_heads / num_kv_heads, &plan->g_tile, &plan->subgroups);
  plan->head_blocks = ceil_div(num_kv_heads, pa::kHeadBlock);
  plan->items = static_cast<unsigned long long>(plan->partitions) * num_seqs * plan->head_blocks * plan->subgroups;
  if (num_seqs > 65535 || plan->items > 0x7fffffffULL) return PA_ERR_UNSUPPORTED;
  plan->ws = workspace_layout(num_seqs, num_heads, num_kv_heads, head_size, plan->partitions);
  return PA_OK;
}

}  // namespace

namespace pa_host {

pa_status paged_attention_check(const void* out, const void* query, pa_dtype q_dtype, const void* key_cache,
                                const void* value_cache, pa_dtype kv_dtype, const float* k_scale,
                                const float* v_scale, const int32_t* block_tables, int max_blocks_per_seq,
                                const int32_t* context_lens, int num_seqs, int num_heads, int num_kv_heads,
                                int head_size, int block_size, int num_blocks, int max_context_len, float scale,
                                int partition_size, size_t* workspace_bytes, bool* empty) {
  AttnPlan plan;
  const pa_status st = check_attention(out, query, q_dtype, key_cache, value_cache, kv_dtype, k_scale, v_scale,
                                       block_tables, max_blocks_per_seq, context_lens, num_seqs, num_heads,
                                       num_kv_heads, head_size, block_size, num_blocks, max_context_len, scale,
                                       partition_size, &plan);
  *workspace_bytes = plan.ws.total;
  *empty = plan.empty;
  return st;
}

}  // namespace pa_host

extern "C" {

const char* pa_status_string(pa_status status) {
  switch (status) {
    case PA_OK: return "PA_OK";
    case PA_ERR_INVALID_ARGUMENT: return "PA_ERR_INVALID_ARGUMENT: invalid argument (null/misaligned pointer, bad size or mapping)";
    case PA_ERR_UNSUPPORTED: return "PA_ERR_UNSUPPORTED: valid but outside the supported head_size/block_size/dtype set";
    case PA_ERR_WORKSPACE_TOO_SMALL: return "PA_ERR_WORKSPACE_TOO_SMALL: workspace smaller than pa_paged_attention_workspace_size()";
    case PA_ERR_CUDA: return "PA_ERR_CUDA: a CUDA call or kernel launch failed";
    case PA_ERR_OUT_OF_BLOCKS: return "PA_ERR_OUT_OF_BLOCKS: too few free blocks in the pool (state unchanged)";
    case PA_ERR_HOST_MEMORY: return "PA_ERR_HOST_MEMORY: a host memory allocation failed (state unchanged)";
  }
  return "unknown pa_status";
}

int pa_paged_attention_partition_size(int num_seqs, int num_heads, int num_kv_heads, int max_context_len,
                                      int partition_size) {
  return plan_partition(num_seqs, num_heads, num_kv_heads, max_context_len, partition_size);
}

size_t pa_paged_attention_workspace_size(int num_seqs, int num_heads, int num_kv_heads, int head_size,
                                         int max_context_len, int partition_size) {
  if (num_seqs < 0 || num_heads <= 0 || num_kv_heads <= 0 || head_size <= 0 || max_context_len < 0) return 0;
  const int ps = plan_partition(num_seqs, num_heads, num_kv_heads, max_context_len, partition_size);
  if (ps <= 0) return 0;
  const int partitions = std::max(1, ceil_div(max_context_len, ps));
  return workspace_layout(num_seqs, num_heads, num_kv_heads, head_size, partitions).total;
}

pa_status pa_paged_attention(void* out, const void* query, pa_dtype q_dtype, const void* key_cache,
                             const void* value_cache, pa_dtype kv_dtype, const float* k_scale,
                             const float* v_scale, const int32_t* block_tables, int max_blocks_per_seq,
                             const int32_t* context_lens, int num_seqs, int num_heads, int num_kv_heads,
                             int head_size, int block_size, int num_blocks, int max_context_len, float scale,
                             int partition_size, void* workspace, size_t workspace_bytes,
                             pa_stream_t stream) {
  // ---- validation: no CUDA call before every check has passed ----
  AttnPlan plan;
  const pa_status checked = check_attention(out, query, q_dtype, key_cache, value_cache, kv_dtype, k_scale, v_scale,
                                            block_tables, max_blocks_per_seq, context_lens, num_seqs, num_heads,
                                            num_kv_heads, head_size, block_size, num_blocks, max_context_len, scale,
                                            partition_size, &plan);
  if (checked != PA_OK) return checked;
  if (plan.empty) return PA_OK;  // empty batch: nothing is read or written
  if (!workspace || !aligned(workspace, 16)) return PA_ERR_INVALID_ARGUMENT;
  if (workspace_bytes < plan.ws.total) return PA_ERR_WORKSPACE_TOO_SMALL;
  const int ps = plan.ps, partitions = plan.partitions, g_tile = plan.g_tile, subgroups = plan.subgroups;
  const int head_blocks = plan.head_blocks;
  const unsigned long long items = plan.items;
  const bool fp8 = is_fp8(kv_dtype);
  const WorkspaceLayout& ws = plan.ws;

  // ---- launch ----
  CUtensorMap tk, tv;
  const int eb = elem_bytes(kv_dtype);
  if (!encode_cache_map(&tk, key_cache, eb, head_size, num_kv_heads, block_size, num_blocks) ||
      !encode_cache_map(&tv, value_cache, eb, head_size, num_kv_heads, block_size, num_blocks))
    return PA_ERR_CUDA;
  int device = 0, sms = 0;
  if (cudaGetDevice(&device) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, device) != cudaSuccess || sms <= 0)
    return PA_ERR_CUDA;
  uint8_t* wsb = static_cast<uint8_t*>(workspace);
  pa::AttnArgs a{};
  a.out = out;
  a.query = query;
  a.k_scale = k_scale;
  a.v_scale = v_scale;
  a.block_tables = block_tables;
  a.context_lens = context_lens;
  a.part_m = partitions > 1 ? reinterpret_cast<float*>(wsb + ws.part_m) : nullptr;
  a.part_l = partitions > 1 ? reinterpret_cast<float*>(wsb + ws.part_l) : nullptr;
  a.part_o = partitions > 1 ? reinterpret_cast<float*>(wsb + ws.part_o) : nullptr;
  a.header = reinterpret_cast<unsigned int*>(wsb);
  a.max_blocks_per_seq = max_blocks_per_seq;
  a.num_seqs = num_seqs;
  a.num_heads = num_heads;
  a.num_kv_heads = num_kv_heads;
  a.group = num_heads / num_kv_heads;
  a.subgroups = subgroups;
  a.head_blocks = head_blocks;
  a.block_size = block_size;
  a.num_blocks = num_blocks;
  a.partition_size = ps;
  a.num_partitions = partitions;
  a.num_items = static_cast<unsigned int>(items);
  a.scale_log2 = scale * pa::kLog2e;
  a.scale_block_stride = scale_block_stride(kv_dtype, num_kv_heads);
#ifdef PA_TRACE
  a.trace = reinterpret_cast<unsigned long long*>(wsb + ws.trace);
#endif
  const int grid = static_cast<int>(std::min<unsigned long long>(static_cast<unsigned long long>(sms), items));
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t e = q_dtype == PA_BF16 ? pa::launch_attention_bf16(tk, tv, a, fp8, head_size, g_tile, grid, st)
                                     : pa::launch_attention_f16(tk, tv, a, fp8, head_size, g_tile, grid, st);
  return e == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

pa_status pa_reshape_and_cache(const void* key, const void* value, pa_dtype in_dtype, void* key_cache,
                               void* value_cache, pa_dtype kv_dtype, const float* k_scale, const float* v_scale,
                               const int64_t* slot_mapping, int num_tokens, int num_kv_heads, int head_size,
                               int block_size, int num_blocks, pa_stream_t stream) {
  if (num_tokens < 0 || num_kv_heads <= 0 || head_size <= 0 || block_size <= 0 || num_blocks <= 0)
    return PA_ERR_INVALID_ARGUMENT;
  if (!is_dtype(in_dtype) || !is_dtype(kv_dtype) || !is_16bit(in_dtype)) return PA_ERR_INVALID_ARGUMENT;
  if (num_tokens == 0) return PA_OK;  // empty batch: nothing is read, pointers may be null
  if (!key || !value || !key_cache || !value_cache || !slot_mapping) return PA_ERR_INVALID_ARGUMENT;
  if (!aligned(key, 16) || !aligned(value, 16) || !aligned(key_cache, 16) || !aligned(value_cache, 16) ||
      !aligned(slot_mapping, 8))
    return PA_ERR_INVALID_ARGUMENT;
  const bool fp8 = is_fp8(kv_dtype);
  if (fp8 && (!k_scale || !v_scale || !aligned(k_scale, 4) || !aligned(v_scale, 4))) return PA_ERR_INVALID_ARGUMENT;
  if (!fp8 && kv_dtype != in_dtype) return PA_ERR_UNSUPPORTED;
  const int sstride = scale_block_stride(kv_dtype, num_kv_heads);
  if (head_size % 8 != 0 || static_cast<int64_t>(num_kv_heads) * head_size > kMaxRowElems) return PA_ERR_UNSUPPORTED;
  const int row = num_kv_heads * head_size;
  const int threads = static_cast<int>(std::min<size_t>(256, round_up(static_cast<size_t>(ceil_div(row, 8)), 32)));
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const dim3 grid(static_cast<unsigned>(num_tokens));
  const auto launch = [&](auto in_tag, auto cache_tag) {
    using IT = decltype(in_tag);
    using KVT = decltype(cache_tag);
    return pa_host::launch_overlapped(pa::reshape_and_cache_kernel<IT, KVT>, grid, dim3(threads), 0, st,
                                      static_cast<const IT*>(key), static_cast<const IT*>(value),
                                      static_cast<KVT*>(key_cache), static_cast<KVT*>(value_cache), k_scale, v_scale,
                                      slot_mapping, num_kv_heads, head_size, block_size, num_blocks, sstride);
  };
  cudaError_t e;
  if (in_dtype == PA_BF16)
    e = fp8 ? launch(__nv_bfloat16{}, __nv_fp8_e4m3{}) : launch(__nv_bfloat16{}, __nv_bfloat16{});
  else
    e = fp8 ? launch(__half{}, __nv_fp8_e4m3{}) : launch(__half{}, __half{});
  return e == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

pa_status pa_copy_blocks(void* key_cache, void* value_cache, pa_dtype kv_dtype, const int64_t* block_mapping,
                         int num_pairs, int num_kv_heads, int head_size, int block_size, int num_blocks,
                         pa_stream_t stream) {
  if (num_pairs < 0 || num_kv_heads <= 0 || head_size <= 0 || block_size <= 0 || num_blocks <= 0)
    return PA_ERR_INVALID_ARGUMENT;
  if (!is_dtype(kv_dtype)) return PA_ERR_INVALID_ARGUMENT;
  if (!key_cache || !value_cache || (num_pairs > 0 && !block_mapping)) return PA_ERR_INVALID_ARGUMENT;
  if (!aligned(key_cache, 16) || !aligned(value_cache, 16) || (block_mapping && !aligned(block_mapping, 8)))
    return PA_ERR_INVALID_ARGUMENT;
  const int64_t block_bytes = static_cast<int64_t>(block_size) * num_kv_heads * head_size * elem_bytes(kv_dtype);
  if (block_bytes % 16 != 0) return PA_ERR_UNSUPPORTED;
  if (num_pairs == 0) return PA_OK;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const cudaError_t e = pa_host::launch_overlapped(pa::copy_blocks_kernel, dim3(static_cast<unsigned>(num_pairs), 2),
                                                   dim3(256), 0, st, static_cast<uint8_t*>(key_cache),
                                                   static_cast<uint8_t*>(value_cache), block_mapping, block_bytes,
                                                   num_blocks);
  return e == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

pa_status pa_reshape_and_cache_layers(const void* const* keys, const void* const* values, pa_dtype in_dtype,
                                      void* const* key_caches, void* const* value_caches, pa_dtype kv_dtype,
                                      const float* const* k_scales, const float* const* v_scales,
                                      const int64_t* slot_mapping, int num_tokens, int num_layers, int num_kv_heads,
                                      int head_size, int block_size, int num_blocks, pa_stream_t stream) {
  if (num_tokens < 0 || num_layers < 0 || num_kv_heads <= 0 || head_size <= 0 || block_size <= 0 || num_blocks <= 0)
    return PA_ERR_INVALID_ARGUMENT;
  if (!is_dtype(in_dtype) || !is_dtype(kv_dtype) || !is_16bit(in_dtype)) return PA_ERR_INVALID_ARGUMENT;
  if (num_tokens == 0 || num_layers == 0) return PA_OK;  // nothing is read, pointers may be null
  if (!keys || !values || !key_caches || !value_caches || !slot_mapping) return PA_ERR_INVALID_ARGUMENT;
  if (!aligned(keys, 8) || !aligned(values, 8) || !aligned(key_caches, 8) || !aligned(value_caches, 8) ||
      !aligned(slot_mapping, 8))
    return PA_ERR_INVALID_ARGUMENT;
  const bool fp8 = is_fp8(kv_dtype);
  if (fp8 && (!k_scales || !v_scales || !aligned(k_scales, 8) || !aligned(v_scales, 8))) return PA_ERR_INVALID_ARGUMENT;
  if (!fp8 && kv_dtype != in_dtype) return PA_ERR_UNSUPPORTED;
  const int sstride = scale_block_stride(kv_dtype, num_kv_heads);
  if (head_size % 8 != 0 || num_layers > 65535 || static_cast<int64_t>(num_kv_heads) * head_size > kMaxRowElems)
    return PA_ERR_UNSUPPORTED;
  const int row = num_kv_heads * head_size;
  const int threads = static_cast<int>(std::min<size_t>(256, round_up(static_cast<size_t>(ceil_div(row, 8)), 32)));
  const dim3 grid(static_cast<unsigned>(num_tokens), static_cast<unsigned>(num_layers));
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const float* const* ks = fp8 ? k_scales : nullptr;
  const float* const* vs = fp8 ? v_scales : nullptr;
  const auto launch = [&](auto in_tag, auto cache_tag) {
    using IT = decltype(in_tag);
    using KVT = decltype(cache_tag);
    return pa_host::launch_plain(pa::reshape_and_cache_layers_kernel<IT, KVT>, grid, dim3(threads), 0, st, keys,
                                 values, key_caches, value_caches, ks, vs, slot_mapping, num_kv_heads, head_size,
                                 block_size, num_blocks, sstride);
  };
  cudaError_t e;
  if (in_dtype == PA_BF16)
    e = fp8 ? launch(__nv_bfloat16{}, __nv_fp8_e4m3{}) : launch(__nv_bfloat16{}, __nv_bfloat16{});
  else
    e = fp8 ? launch(__half{}, __nv_fp8_e4m3{}) : launch(__half{}, __half{});
  return e == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

pa_status pa_copy_blocks_layers(void* const* key_caches, void* const* value_caches, int num_layers, pa_dtype kv_dtype,
                                const int64_t* block_mapping, int num_pairs, int num_kv_heads, int head_size,
                                int block_size, int num_blocks, pa_stream_t stream) {
  if (num_pairs < 0 || num_layers < 0 || num_kv_heads <= 0 || head_size <= 0 || block_size <= 0 || num_blocks <= 0)
    return PA_ERR_INVALID_ARGUMENT;
  if (!is_dtype(kv_dtype)) return PA_ERR_INVALID_ARGUMENT;
  if (!key_caches || !value_caches || (num_pairs > 0 && !block_mapping)) return PA_ERR_INVALID_ARGUMENT;
  if (!aligned(key_caches, 8) || !aligned(value_caches, 8) || (block_mapping && !aligned(block_mapping, 8)))
    return PA_ERR_INVALID_ARGUMENT;
  const int64_t block_bytes = static_cast<int64_t>(block_size) * num_kv_heads * head_size * elem_bytes(kv_dtype);
  if (block_bytes % 16 != 0 || num_layers > 65535) return PA_ERR_UNSUPPORTED;
  if (num_pairs == 0 || num_layers == 0) return PA_OK;
  const cudaError_t e = pa_host::launch_plain(
      pa::copy_blocks_layers_kernel, dim3(static_cast<unsigned>(num_pairs), 2, static_cast<unsigned>(num_layers)),
      dim3(256), 0, reinterpret_cast<cudaStream_t>(stream), key_caches, value_caches, block_mapping, block_bytes,
      num_blocks);
  return e == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

namespace {
// Device-reachable address of a pointer (device memory, managed memory, or pinned/registered host
// memory); nullptr for pageable host memory or an unknown pointer.
void* device_reachable(const void* p) {
  cudaPointerAttributes attr;
  if (cudaPointerGetAttributes(&attr, p) != cudaSuccess) {
    cudaGetLastError();  // clear the sticky-free error of an unknown pointer
    return nullptr;
  }
  if (attr.type == cudaMemoryTypeDevice || attr.type == cudaMemoryTypeManaged) return const_cast<void*>(p);
  if (attr.type == cudaMemoryTypeHost) return attr.devicePointer;
  return nullptr;
}
}  // namespace

pa_status pa_swap_blocks(void* dst_key_cache, void* dst_value_cache, const void* src_key_cache,
                         const void* src_value_cache, pa_dtype kv_dtype, const int64_t* block_mapping, int num_pairs,
                         int num_kv_heads, int head_size, int block_size, int src_num_blocks, int dst_num_blocks,
                         pa_stream_t stream) {
  if (num_pairs < 0 || num_kv_heads <= 0 || head_size <= 0 || block_size <= 0 || src_num_blocks <= 0 ||
      dst_num_blocks <= 0 || !is_dtype(kv_dtype))
    return PA_ERR_INVALID_ARGUMENT;
  if (!dst_key_cache || !dst_value_cache || !src_key_cache || !src_value_cache || (num_pairs > 0 && !block_mapping))
    return PA_ERR_INVALID_ARGUMENT;
  if (!aligned(dst_key_cache, 16) || !aligned(dst_value_cache, 16) || !aligned(src_key_cache, 16) ||
      !aligned(src_value_cache, 16) || (block_mapping && !aligned(block_mapping, 8)))
    return PA_ERR_INVALID_ARGUMENT;
  const int64_t block_bytes = static_cast<int64_t>(block_size) * num_kv_heads * head_size * elem_bytes(kv_dtype);
  if (block_bytes % 16 != 0) return PA_ERR_UNSUPPORTED;
  if (num_pairs == 0) return PA_OK;
  // Every pool and the mapping must be reachable from the GPU; pageable host memory is refused here
  // (a kernel touching it would fault).
  void* dk = device_reachable(dst_key_cache);
  void* dv = device_reachable(dst_value_cache);
  void* sk = device_reachable(src_key_cache);
  void* sv = device_reachable(src_value_cache);
  void* bm = device_reachable(block_mapping);
  if (!dk || !dv || !sk || !sv || !bm) return PA_ERR_INVALID_ARGUMENT;
  const cudaError_t e = pa_host::launch_plain(
      pa::swap_blocks_kernel, dim3(static_cast<unsigned>(num_pairs), 2), dim3(256), 0,
      reinterpret_cast<cudaStream_t>(stream), static_cast<uint8_t*>(dk), static_cast<uint8_t*>(dv),
      static_cast<const uint8_t*>(sk), static_cast<const uint8_t*>(sv), static_cast<const int64_t*>(bm), block_bytes,
      src_num_blocks, dst_num_blocks);
  return e == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

pa_status pa_copy_blocks_check(const int64_t* host_block_mapping, int num_pairs, int num_blocks) {
  if (num_pairs < 0 || num_blocks <= 0 || (num_pairs > 0 && !host_block_mapping)) return PA_ERR_INVALID_ARGUMENT;
  std::unordered_set<int64_t> srcs, dsts;
  for (int p = 0; p < num_pairs; ++p) {
    const int64_t s = host_block_mapping[2 * p], d = host_block_mapping[2 * p + 1];
    if (s < 0 || s >= num_blocks || d < 0 || d >= num_blocks) return PA_ERR_INVALID_ARGUMENT;
    srcs.insert(s);
    if (!dsts.insert(d).second) return PA_ERR_INVALID_ARGUMENT;
  }
  for (int64_t d : dsts)
    if (srcs.count(d)) return PA_ERR_INVALID_ARGUMENT;
  return PA_OK;
}

pa_status pa_selftest_wait_timeout(unsigned int* device_error_word, unsigned long long limit_ns, pa_stream_t stream) {
  if (!device_error_word || !aligned(device_error_word, 4) || limit_ns == 0 || limit_ns > 10000000000ull)
    return PA_ERR_INVALID_ARGUMENT;
  const cudaError_t e = pa_host::launch_plain(pa::selftest_wait_kernel, dim3(1), dim3(32), 0,
                                              reinterpret_cast<cudaStream_t>(stream), device_error_word, limit_ns);
  return e == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

pa_status pa_get_device_error(const void* workspace, unsigned int* err_out, pa_stream_t stream) {
  if (!workspace || !err_out || !aligned(workspace, 16)) return PA_ERR_INVALID_ARGUMENT;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  unsigned int value = 0;
  if (cudaMemcpyAsync(&value, workspace, sizeof(value), cudaMemcpyDeviceToHost, st) != cudaSuccess)
    return PA_ERR_CUDA;
  if (cudaStreamSynchronize(st) != cudaSuccess) return PA_ERR_CUDA;
  *err_out = value;
  return PA_OK;
}

pa_status pa_clear_device_error(void* workspace, pa_stream_t stream) {
  if (!workspace || !aligned(workspace, 16)) return PA_ERR_INVALID_ARGUMENT;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  // The error word only: the header's other words are the kernels' own (work and finished-CTA counters).
  return cudaMemsetAsync(workspace, 0, sizeof(unsigned int), st) == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

}  // extern "C"
