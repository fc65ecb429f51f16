// pa_cache_ops.cuh -- writing new tokens into their slots and copy-on-write of whole blocks.
//
// reshape_and_cache: page "vLLM的诞生背景：大模型推理的痛点与PagedAttention的破局", section
// "PagedAttention的破局思路" -- a sequence's KV grows into blocks allocated on demand; token i goes to
// slot slot_mapping[i] = block * block_size + offset. FP8 caches (tutorial page "企业官网建设流程全解析",
// sec. 3.2 "关键性能优化", FP8 storage of blocks) store E4M3(x / scale[kv head]).
// copy_blocks: same page, section "PagedAttention的局限性" -- copy-on-write of shared blocks.
// Both are pure data movement (plus the FP8 encode): 16-byte vector loads and stores, no staging.
#pragma once

#include "pa_device.cuh"

namespace pa {

// One CTA per token; thread i handles 8 consecutive elements of the token's [Hkv][D] row.
template <typename IT, typename KVT>
__device__ __forceinline__ void reshape_and_cache_token(const IT* __restrict__ key, const IT* __restrict__ value,
                                                        KVT* __restrict__ key_cache, KVT* __restrict__ value_cache,
                                                        const float* __restrict__ k_scale,
                                                        const float* __restrict__ v_scale,
                                                        const int64_t* __restrict__ slot_mapping, int num_kv_heads,
                                                        int head_size, int block_size, int num_blocks,
                                                        int scale_stride) {
  const int64_t token = blockIdx.x;
  const int64_t slot = slot_mapping[token];
  if (slot < 0 || slot >= static_cast<int64_t>(num_blocks) * block_size) return;
  const int64_t blk = slot / block_size;
  const int64_t off = slot - blk * block_size;
  const int row = num_kv_heads * head_size;  // elements per token
  const IT* ksrc = key + token * row;
  const IT* vsrc = value + token * row;
  const int64_t dst_base = (blk * block_size + off) * row;
  for (int e = threadIdx.x * 8; e < row; e += blockDim.x * 8) {
    const uint4 kin = *reinterpret_cast<const uint4*>(ksrc + e);
    const uint4 vin = *reinterpret_cast<const uint4*>(vsrc + e);
    if constexpr (sizeof(KVT) == sizeof(IT)) {
      *reinterpret_cast<uint4*>(key_cache + dst_base + e) = kin;
      *reinterpret_cast<uint4*>(value_cache + dst_base + e) = vin;
    } else {
      // E4M3: code = cvt.rn.satfinite(x / scale), the division correctly rounded (IEEE); the scale is
      // the kv head's, or with per-block scales (scale_stride = num_kv_heads) the slot's block's.
      const int h = e / head_size;
      const float ks = k_scale[blk * scale_stride + h], vs = v_scale[blk * scale_stride + h];
      const IT* kx = reinterpret_cast<const IT*>(&kin);
      const IT* vx = reinterpret_cast<const IT*>(&vin);
      uint32_t kout[2], vout[2];
#pragma unroll
      for (int w = 0; w < 2; ++w) {
        uint32_t kw = 0, vw = 0;
#pragma unroll
        for (int k = 0; k < 2; ++k) {
          const int i = w * 4 + k * 2;
          const float2 kf = make_float2(__fdiv_rn(to_f32(kx[i]), ks), __fdiv_rn(to_f32(kx[i + 1]), ks));
          const float2 vf = make_float2(__fdiv_rn(to_f32(vx[i]), vs), __fdiv_rn(to_f32(vx[i + 1]), vs));
          const uint32_t kc = __nv_cvt_float2_to_fp8x2(kf, __NV_SATFINITE, __NV_E4M3);
          const uint32_t vc = __nv_cvt_float2_to_fp8x2(vf, __NV_SATFINITE, __NV_E4M3);
          kw |= (kc & 0xffffu) << (16 * k);
          vw |= (vc & 0xffffu) << (16 * k);
        }
        kout[w] = kw;
        vout[w] = vw;
      }
      *reinterpret_cast<uint2*>(key_cache + dst_base + e) = make_uint2(kout[0], kout[1]);
      *reinterpret_cast<uint2*>(value_cache + dst_base + e) = make_uint2(vout[0], vout[1]);
    }
  }
}

template <typename IT, typename KVT>
__global__ void __launch_bounds__(256)
reshape_and_cache_kernel(const IT* __restrict__ key, const IT* __restrict__ value, KVT* __restrict__ key_cache,
                         KVT* __restrict__ value_cache, const float* __restrict__ k_scale,
                         const float* __restrict__ v_scale, const int64_t* __restrict__ slot_mapping,
                         int num_kv_heads, int head_size, int block_size, int num_blocks, int scale_stride) {
  grid_dependency_wait();
  grid_dependents_launch();
  reshape_and_cache_token<IT, KVT>(key, value, key_cache, value_cache, k_scale, v_scale, slot_mapping, num_kv_heads,
                                   head_size, block_size, num_blocks, scale_stride);
}

// All layers in one launch: grid (tokens, layers); per-layer pointers come from device arrays.
template <typename IT, typename KVT>
__global__ void __launch_bounds__(256)
reshape_and_cache_layers_kernel(const void* const* __restrict__ keys, const void* const* __restrict__ values,
                                void* const* __restrict__ key_caches, void* const* __restrict__ value_caches,
                                const float* const* __restrict__ k_scales, const float* const* __restrict__ v_scales,
                                const int64_t* __restrict__ slot_mapping, int num_kv_heads, int head_size,
                                int block_size, int num_blocks, int scale_stride) {
  const int layer = blockIdx.y;
  reshape_and_cache_token<IT, KVT>(static_cast<const IT*>(keys[layer]), static_cast<const IT*>(values[layer]),
                                   static_cast<KVT*>(key_caches[layer]), static_cast<KVT*>(value_caches[layer]),
                                   k_scales ? k_scales[layer] : nullptr, v_scales ? v_scales[layer] : nullptr,
                                   slot_mapping, num_kv_heads, head_size, block_size, num_blocks, scale_stride);
}

// One CTA per (pair, key|value): copy one contiguous block of `block_bytes` (a multiple of 16).
__global__ void __launch_bounds__(256)
copy_blocks_kernel(uint8_t* __restrict__ key_cache, uint8_t* __restrict__ value_cache,
                   const int64_t* __restrict__ block_mapping, int64_t block_bytes, int num_blocks) {
  grid_dependency_wait();
  grid_dependents_launch();
  const int pair = blockIdx.x;
  const int64_t src = block_mapping[2 * pair];
  const int64_t dst = block_mapping[2 * pair + 1];
  if (src < 0 || src >= num_blocks || dst < 0 || dst >= num_blocks) return;
  uint8_t* base = blockIdx.y == 0 ? key_cache : value_cache;
  const uint4* s = reinterpret_cast<const uint4*>(base + src * block_bytes);
  uint4* d = reinterpret_cast<uint4*>(base + dst * block_bytes);
  const int64_t n = block_bytes / 16;
  for (int64_t i = threadIdx.x; i < n; i += blockDim.x) d[i] = s[i];
}

// Copy-on-write over all layers in one launch: grid (pairs, key|value, layers).
__global__ void __launch_bounds__(256)
copy_blocks_layers_kernel(void* const* __restrict__ key_caches, void* const* __restrict__ value_caches,
                          const int64_t* __restrict__ block_mapping, int64_t block_bytes, int num_blocks) {
  const int pair = blockIdx.x;
  const int64_t src = block_mapping[2 * pair];
  const int64_t dst = block_mapping[2 * pair + 1];
  if (src < 0 || src >= num_blocks || dst < 0 || dst >= num_blocks) return;
  uint8_t* base = static_cast<uint8_t*>(blockIdx.y == 0 ? key_caches[blockIdx.z] : value_caches[blockIdx.z]);
  const uint4* s = reinterpret_cast<const uint4*>(base + src * block_bytes);
  uint4* d = reinterpret_cast<uint4*>(base + dst * block_bytes);
  const int64_t n = block_bytes / 16;
  for (int64_t i = threadIdx.x; i < n; i += blockDim.x) d[i] = s[i];
}

// Swapping blocks between two pools that may live in different memories (device, or pinned host
// memory reached through its unified address): one CTA per (pair, key|value), 16-byte vectors. Page
// "PagedAttention 与连续批处理：LLM Serving 的底层架构拆解", section "PagedAttention：把显存做成虚拟内存":
// pages of inactive sequences go to CPU memory and come back when needed.
__global__ void __launch_bounds__(256)
swap_blocks_kernel(uint8_t* __restrict__ dst_key, uint8_t* __restrict__ dst_value, const uint8_t* __restrict__ src_key,
                   const uint8_t* __restrict__ src_value, const int64_t* __restrict__ block_mapping,
                   int64_t block_bytes, int src_num_blocks, int dst_num_blocks) {
  const int pair = blockIdx.x;
  const int64_t src = block_mapping[2 * pair];
  const int64_t dst = block_mapping[2 * pair + 1];
  if (src < 0 || src >= src_num_blocks || dst < 0 || dst >= dst_num_blocks) return;
  const uint4* s = reinterpret_cast<const uint4*>((blockIdx.y == 0 ? src_key : src_value) + src * block_bytes);
  uint4* d = reinterpret_cast<uint4*>((blockIdx.y == 0 ? dst_key : dst_value) + dst * block_bytes);
  const int64_t n = block_bytes / 16;
  for (int64_t i = threadIdx.x; i < n; i += blockDim.x) d[i] = s[i];
}

// Self-test of the bounded wait used by every pipeline wait: an mbarrier that nothing ever arrives on
// is waited for with a short limit; the wait must give up, set PA_DEVERR_TIMEOUT and return.
__global__ void selftest_wait_kernel(unsigned int* error_word, unsigned long long limit_ns) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) mbar_wait(&bar, 0u, error_word, limit_ns);
}

}  // namespace pa
