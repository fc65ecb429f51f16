// pa_prefill.cu -- C ABI of the causal paged prefill attention (include/pagedattn.h): validation before
// any CUDA call, TMA descriptors for the query and the two caches, and the launch of
// pa::pf::paged_prefill_kernel (pa_prefill.cuh).
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>

#include "pa_host_util.h"
#include "pa_prefill.cuh"
#include "pagedattn.h"

namespace {

using pa_host::aligned;
using pa_host::ceil_div;
using pa_host::is_16bit;
using pa_host::is_dtype;

constexpr float kLog2e = 1.4426950408889634f;

// Query [T][H][d] as {d, H, T}; box = one 128-byte chunk x the G heads of a kv head x tile_tokens
// tokens, so a box lands as 128 rows (token-major, head-minor) of 128 bytes, 128-byte swizzled.
bool encode_query_map(CUtensorMap* map, const void* query, int head_size, int num_heads, int num_q_tokens, int group,
                      int tile_tokens) {
  auto encode = pa_host::tensor_map_encoder();
  if (!encode) return false;
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(head_size), static_cast<cuuint64_t>(num_heads),
                        static_cast<cuuint64_t>(num_q_tokens)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(head_size) * 2, static_cast<cuuint64_t>(num_heads) * head_size * 2};
  cuuint32_t box[3] = {64, static_cast<cuuint32_t>(group), static_cast<cuuint32_t>(tile_tokens)};
  cuuint32_t estr[3] = {1, 1, 1};
  return encode(map, CU_TENSOR_MAP_DATA_TYPE_UINT16, 3, const_cast<void*>(query), dims, strides, box, estr,
                CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Cache [NB][bs][Hkv][d] as {d, token, kv head, block}; box = one 128-byte chunk of the bs token rows
// of one kv head of one block (64 columns of a 16-bit cache, 128 of an E4M3 one).
bool encode_block_map(CUtensorMap* map, const void* cache, int elem_bytes, int head_size, int num_kv_heads,
                      int block_size, int num_blocks) {
  auto encode = pa_host::tensor_map_encoder();
  if (!encode) return false;
  const cuuint64_t e = static_cast<cuuint64_t>(elem_bytes);
  cuuint64_t dims[4] = {static_cast<cuuint64_t>(head_size), static_cast<cuuint64_t>(block_size),
                        static_cast<cuuint64_t>(num_kv_heads), static_cast<cuuint64_t>(num_blocks)};
  cuuint64_t strides[3] = {num_kv_heads * head_size * e, head_size * e, block_size * num_kv_heads * head_size * e};
  cuuint32_t box[4] = {static_cast<cuuint32_t>(128 / elem_bytes), static_cast<cuuint32_t>(block_size), 1, 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  return encode(map, elem_bytes == 2 ? CU_TENSOR_MAP_DATA_TYPE_UINT16 : CU_TENSOR_MAP_DATA_TYPE_UINT8, 4,
                const_cast<void*>(cache), dims, strides, box, estr,
                CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <typename T, int D, int KVB = 2, bool BS = false>
cudaError_t launch_prefill(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                           const pa::pf::PrefillArgs& a, dim3 grid, cudaStream_t st) {
  auto kernel = pa::pf::paged_prefill_kernel<T, D, KVB, BS>;
  const int smem = static_cast<int>(pa::pf::Layout<D>::kBytes);
  cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  return pa_host::launch_plain(kernel, grid, dim3(pa::pf::kThreads), static_cast<size_t>(smem), st, tq, tk, tv, a);
}

}  // namespace

extern "C" pa_status pa_paged_prefill(void* out, const void* query, pa_dtype q_dtype, const void* key_cache,
                                      const void* value_cache, pa_dtype kv_dtype, const float* k_scale,
                                      const float* v_scale, const int32_t* block_tables,
                                      int max_blocks_per_seq, const int32_t* context_lens, const int32_t* q_start,
                                      int num_seqs, int num_q_tokens, int num_heads, int num_kv_heads,
                                      int head_size, int block_size, int num_blocks, int max_q_len, float scale,
                                      void* workspace, size_t workspace_bytes, pa_stream_t stream) {
  if (num_seqs < 0 || num_q_tokens < 0 || num_heads <= 0 || num_kv_heads <= 0 || num_heads % num_kv_heads != 0 ||
      head_size <= 0 || block_size <= 0 || num_blocks <= 0 || max_blocks_per_seq <= 0 || max_q_len < 0 ||
      !std::isfinite(scale) || !(scale > 0.f))
    return PA_ERR_INVALID_ARGUMENT;
  if (!is_dtype(q_dtype) || !is_dtype(kv_dtype) || !is_16bit(q_dtype)) return PA_ERR_INVALID_ARGUMENT;
  if (num_seqs == 0 || num_q_tokens == 0 || max_q_len == 0) return PA_OK;  // nothing to compute
  if (!out || !query || !key_cache || !value_cache || !block_tables || !context_lens || !q_start || !workspace)
    return PA_ERR_INVALID_ARGUMENT;
  if (!aligned(out, 16) || !aligned(query, 16) || !aligned(key_cache, 16) || !aligned(value_cache, 16) ||
      !aligned(workspace, 16) || !aligned(block_tables, 4) || !aligned(context_lens, 4) || !aligned(q_start, 4))
    return PA_ERR_INVALID_ARGUMENT;
  if (workspace_bytes < PA_WORKSPACE_HEADER_BYTES) return PA_ERR_WORKSPACE_TOO_SMALL;
  const int group = num_heads / num_kv_heads;
  const bool fp8 = pa_host::is_fp8(kv_dtype);
  if (fp8 && (!k_scale || !v_scale || !aligned(k_scale, 4) || !aligned(v_scale, 4))) return PA_ERR_INVALID_ARGUMENT;
  if (!fp8 && kv_dtype != q_dtype) return PA_ERR_UNSUPPORTED;
  if (fp8 && head_size != 128) return PA_ERR_UNSUPPORTED;
  if (head_size != 64 && head_size != 128) return PA_ERR_UNSUPPORTED;
  if (block_size != 8 && block_size != 16 && block_size != 32 && block_size != 64 && block_size != 128)
    return PA_ERR_UNSUPPORTED;
  if (group > pa::pf::kRows || pa::pf::kRows % group != 0) return PA_ERR_UNSUPPORTED;
  const int tile_tokens = pa::pf::kRows / group;
  const int q_pairs = ceil_div(max_q_len, tile_tokens * pa::pf::kTiles);
  if (num_seqs > 65535 || num_kv_heads > 65535) return PA_ERR_UNSUPPORTED;

  CUtensorMap tq, tk, tv;
  if (!encode_query_map(&tq, query, head_size, num_heads, num_q_tokens, group, tile_tokens) ||
      !encode_block_map(&tk, key_cache, pa_host::elem_bytes(kv_dtype), head_size, num_kv_heads, block_size,
                        num_blocks) ||
      !encode_block_map(&tv, value_cache, pa_host::elem_bytes(kv_dtype), head_size, num_kv_heads, block_size,
                        num_blocks))
    return PA_ERR_CUDA;
  pa::pf::PrefillArgs a{};
  a.out = out;
  a.k_scale = fp8 ? k_scale : nullptr;
  a.v_scale = fp8 ? v_scale : nullptr;
  a.scale_block_stride = pa_host::scale_block_stride(kv_dtype, num_kv_heads);
  a.block_tables = block_tables;
  a.context_lens = context_lens;
  a.q_start = q_start;
  a.error_word = static_cast<unsigned int*>(workspace);
  a.max_blocks_per_seq = max_blocks_per_seq;
  a.num_seqs = num_seqs;
  a.num_q_tokens = num_q_tokens;
  a.num_heads = num_heads;
  a.num_kv_heads = num_kv_heads;
  a.group = group;
  a.tile_tokens = tile_tokens;
  a.block_size = block_size;
  a.num_blocks = num_blocks;
  a.num_pairs = q_pairs;
  a.scale_log2 = scale * kLog2e;
  const dim3 grid(static_cast<unsigned>(q_pairs), static_cast<unsigned>(num_kv_heads),
                  static_cast<unsigned>(num_seqs));
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t e;
  const bool per_block = kv_dtype == PA_FP8_E4M3_BLOCK;
  if (q_dtype == PA_BF16) {
    if (fp8)
      e = per_block ? launch_prefill<__nv_bfloat16, 128, 1, true>(tq, tk, tv, a, grid, st)
                    : launch_prefill<__nv_bfloat16, 128, 1, false>(tq, tk, tv, a, grid, st);
    else
      e = head_size == 128 ? launch_prefill<__nv_bfloat16, 128>(tq, tk, tv, a, grid, st)
                           : launch_prefill<__nv_bfloat16, 64>(tq, tk, tv, a, grid, st);
  } else {
    if (fp8)
      e = per_block ? launch_prefill<__half, 128, 1, true>(tq, tk, tv, a, grid, st)
                    : launch_prefill<__half, 128, 1, false>(tq, tk, tv, a, grid, st);
    else
      e = head_size == 128 ? launch_prefill<__half, 128>(tq, tk, tv, a, grid, st)
                           : launch_prefill<__half, 64>(tq, tk, tv, a, grid, st);
  }
  return e == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}
