/*
 * pagedattn.h -- C ABI of libpagedattn.so: paged KV-cache decode attention on NVIDIA B200 (sm_100a).
 *
 * The operations follow three web pages on PagedAttention, cited by title and section:
 *  [T] "企业官网建设流程全解析" (the body is a PagedAttention tutorial; the title is unrelated):
 *      sec. 2.1 "基本数据结构设计" -- KV stored in fixed-size blocks (16 tokens by default), a block table
 *      mapping logical to physical blocks; sec. 2.2 "分块注意力计算过程" -- Attention(Q,K,V) =
 *      softmax(QK^T/sqrt(d))V computed over the blocks; sec. 2.3 "显存共享机制" -- blocks shared by
 *      reference count; sec. 3.2 "关键性能优化" -- preallocated block pool, asynchronous copies on CUDA
 *      streams, FP8 storage of blocks.
 *  [V] "vLLM的诞生背景：大模型推理的痛点与PagedAttention的破局": "PagedAttention的破局思路" -- blocks are
 *      allocated on demand as a sequence grows; "PagedAttention的局限性" -- copy-on-write of shared
 *      blocks, extra indexing cost of scattered blocks, block-size tuning.
 *  [C] "PagedAttention 与连续批处理：LLM Serving 的底层架构拆解": "PagedAttention：把显存做成虚拟内存" --
 *      attention finds each page through the page table; "对 agent 开发者的启示" -- decode is
 *      memory-bound.
 *
 * Conventions for every entry point
 *  - Ownership: the caller allocates every buffer (the block pool is preallocated, [T] sec. 3.2). The
 *    library calls no allocator, keeps no per-call state and never frees caller memory; its one fixed
 *    device array (PA_STATIC_WORKSPACE_BYTES) serves pa_paged_attention_static only.
 *  - Pointers are DEVICE pointers unless a parameter says "host". Every device pointer must be 16-byte
 *    aligned. Tensors are dense, row-major, in the layouts given below.
 *  - Asynchrony: each call validates its arguments on the host, enqueues its kernels on `stream` and
 *    returns without synchronising ([T] sec. 3.2). A NULL stream is the legacy default stream. The
 *    kernels of pa_copy_blocks, pa_reshape_and_cache and pa_paged_attention(_static) are launched with
 *    programmatic stream serialisation: one may be scheduled while the previous kernel in the stream
 *    finishes, but it waits for that kernel's completion and memory before its first global access,
 *    so every memory effect keeps stream order.
 *  - Errors: invalid arguments are reported before anything is enqueued (nothing runs, no CUDA call is
 *    made). Launch failures return PA_ERR_CUDA. The library never aborts, never throws across the ABI
 *    and its kernels never trap; contract violations that only the device can see (a block id
 *    outside the pool, a context length past the table or past max_context_len) are recorded in the
 *    workspace's error word (see pa_get_device_error) and the affected output rows are set to NaN.
 *
 * Cache layout (shared by all calls): key_cache and value_cache are
 *   [num_blocks][block_size][num_kv_heads][head_size]
 * so element (blk, off, h, i) lives at ((blk*block_size + off)*num_kv_heads + h)*head_size + i.
 * Token t of sequence s is stored in physical block block_tables[s][t / block_size] at offset
 * t % block_size ([T] sec. 2.1; [V] "PagedAttention的破局思路").
 *
 * Supported set (decode attention): head_size in {64, 128}; block_size in {8, 16, 32, 64};
 * num_heads % num_kv_heads == 0; num_seqs <= 65535; num_blocks < 2^27; query/output dtype PA_F16 or PA_BF16; cache dtype
 * equal to the query dtype, or PA_FP8_E4M3 / PA_FP8_E4M3_BLOCK with head_size 128. Anything else returns
 * PA_ERR_UNSUPPORTED.
 */
#ifndef PAGEDATTN_H_
#define PAGEDATTN_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define PA_API __attribute__((visibility("default")))
#else
#define PA_API
#endif

struct CUstream_st;                     /* cudaStream_t is `struct CUstream_st *` */
typedef struct CUstream_st* pa_stream_t;

typedef enum pa_status {
  PA_OK = 0,
  PA_ERR_INVALID_ARGUMENT = 1,          /* null/misaligned pointer, negative size, bad mapping, ... */
  PA_ERR_UNSUPPORTED = 2,               /* valid but outside the supported set above */
  PA_ERR_WORKSPACE_TOO_SMALL = 3,       /* workspace_bytes < pa_paged_attention_workspace_size(...) */
  PA_ERR_CUDA = 4,                      /* a CUDA runtime/driver call or a launch failed */
  PA_ERR_OUT_OF_BLOCKS = 5,             /* block manager: the pool has too few free blocks (no change) */
  PA_ERR_HOST_MEMORY = 6                /* block manager: a host allocation failed (no change) */
} pa_status;

typedef enum pa_dtype {
  PA_F16 = 0,                           /* IEEE binary16 */
  PA_BF16 = 1,                          /* bfloat16 */
  PA_FP8_E4M3 = 2,                      /* OCP FP8 E4M3 (bias 7, max 448, no infinities); k_scale and
                                           v_scale hold one fp32 scale per kv head: [num_kv_heads] */
  PA_FP8_E4M3_BLOCK = 3                 /* the same E4M3 codes with one scale per (block, kv head):
                                           k_scale, v_scale are [num_blocks][num_kv_heads] (tutorial
                                           page "企业官网建设流程全解析", sec. 3.2: blocks are stored in
                                           FP8 one by one, so each carries its own scale). Copying a
                                           block (copy_blocks, swap_blocks) does not copy its scales:
                                           the caller keeps them with the block. */
} pa_dtype;

/* Bits of the device error word (pa_get_device_error). */
#define PA_DEVERR_BLOCK_ID    0x1u      /* a needed block-table entry was outside [0, num_blocks) */
#define PA_DEVERR_CONTEXT_LEN 0x2u      /* context_lens[s] < 0, > max_blocks_per_seq*block_size or
                                           > max_context_len */
#define PA_DEVERR_TIMEOUT     0x4u      /* a pipeline wait inside a kernel gave up (should not happen) */

/* Bytes of the workspace header that holds the device error word (the workspace's first bytes). */
#define PA_WORKSPACE_HEADER_BYTES 256

/*
 * Tokens per context partition that pa_paged_attention will use for these sizes.
 * partition_size > 0 requests that size (it must be a multiple of 64); 0 lets the library choose from
 * num_seqs, num_heads/num_kv_heads and max_context_len (the choice depends on nothing else).
 * Returns the partition size, or -1 if the request is invalid. Host only; makes no CUDA call.
 */
PA_API int pa_paged_attention_partition_size(int num_seqs, int num_heads, int num_kv_heads,
                                      int max_context_len, int partition_size);

/*
 * Workspace bytes pa_paged_attention needs for these sizes (same partition_size rule as above):
 * PA_WORKSPACE_HEADER_BYTES for the error word plus, when the context is split into P > 1
 * partitions, fp32 partial results num_seqs*num_heads*P*(head_size + 2)*4 bytes.
 * Returns 0 if the arguments are invalid. Host only; makes no CUDA call.
 */
PA_API size_t pa_paged_attention_workspace_size(int num_seqs, int num_heads, int num_kv_heads, int head_size,
                                         int max_context_len, int partition_size);

/*
 * Paged decode attention ([T] sec. 2.2 formula, normalised over the whole context; [C]
 * "PagedAttention：把显存做成虚拟内存" for the page-table walk). For each sequence s and query head h,
 * with G = num_heads / num_kv_heads and kv head h / G:
 *     out[s][h][:] = sum_t softmax_t(scale * q[s][h] . k_t) * v_t,   t = 0 .. context_lens[s]-1,
 * where k_t / v_t are read from block block_tables[s][t / block_size] at offset t % block_size.
 * FP8 caches dequantise as code * k_scale[kv head] (resp. v_scale). A context of length 0 gives 0.
 *
 *  out            [num_seqs][num_heads][head_size], q_dtype; written.
 *  query          [num_seqs][num_heads][head_size], q_dtype (PA_F16 or PA_BF16).
 *  key_cache,
 *  value_cache    [num_blocks][block_size][num_kv_heads][head_size], kv_dtype; read only.
 *  k_scale,
 *  v_scale        [num_kv_heads] fp32 dequantisation scales; required for PA_FP8_E4M3, else ignored.
 *  block_tables   [num_seqs][max_blocks_per_seq] int32 physical block ids; only the first
 *                 min(ceil(context_lens[s]/block_size), max_blocks_per_seq) entries of row s are
 *                 read, so the rest may hold anything (the kernel prefetches ids a window at a time,
 *                 clamped to that count).
 *  context_lens   [num_seqs] int32.
 *  max_context_len host int, >= every context_lens[s]; sizes the launch (partitions).
 *  scale          the softmax scale (1/sqrt(head_size) in the pages' formula).
 *  partition_size 0 = library's choice, else a multiple of 64 (tokens per split-K partition).
 *  workspace      device scratch of workspace_bytes >= pa_paged_attention_workspace_size(...); its
 *                 first PA_WORKSPACE_HEADER_BYTES hold the error word, which the caller zeroes once
 *                 (e.g. with cudaMemset or pa_clear_device_error) and the kernels only OR into.
 * Calls that share a workspace must be ordered on one stream. num_seqs == 0 is a no-op (pointers
 * may then be NULL).
 */
PA_API pa_status pa_paged_attention(void* out, const void* query, pa_dtype q_dtype,
                             const void* key_cache, const void* value_cache, pa_dtype kv_dtype,
                             const float* k_scale, const float* v_scale,
                             const int32_t* block_tables, int max_blocks_per_seq,
                             const int32_t* context_lens, int num_seqs, int num_heads,
                             int num_kv_heads, int head_size, int block_size, int num_blocks,
                             int max_context_len, float scale, int partition_size,
                             void* workspace, size_t workspace_bytes, pa_stream_t stream);

/*
 * Paged attention without a caller-allocated workspace. The pages have no counterpart: this entry
 * point exists for callers that cannot call cudaMalloc -- a plugin hosted by an engine that owns all
 * device memory, or a serving loop that must not allocate (nor pay cudaMalloc's implicit device
 * synchronisation) once it runs. It computes exactly what pa_paged_attention computes, with the same
 * arguments and rules, except that its scratch memory is a fixed array inside the library:
 *  - size: PA_STATIC_WORKSPACE_BYTES, reserved on every GPU that loads the library until the process
 *    exits; a call whose pa_paged_attention_workspace_size(...) exceeds it returns
 *    PA_ERR_WORKSPACE_TOO_SMALL without enqueuing anything;
 *  - set-up: the first call on each device looks up the array's device address on that device (it
 *    must be the current device); make that first call before any stream capture. The address is
 *    kept per device together with the context it was found in, and looked up again when another
 *    context is current; after cudaDeviceReset the module is loaded anew and the array may move, so
 *    do not keep using this entry point across a device reset;
 *  - checks: every argument check of pa_paged_attention (except those on the workspace) runs first,
 *    with the same results; only then is the request's size compared with the array;
 *  - sharing: every call on a device uses the same array, which keeps the last call's contents; calls
 *    that overlap on the GPU (different streams without ordering) race and give undefined results;
 *  - errors: the device error word lives in the array; when device_error_out (a DEVICE pointer to
 *    one unsigned int, or NULL) is given, the call copies the word there on `stream` after its
 *    kernels, then clears it for the next call.
 * It allocates nothing: no cudaMalloc, no cudaFree, no allocating library call.
 */
#define PA_STATIC_WORKSPACE_BYTES (32u << 20)
PA_API pa_status pa_paged_attention_static(void* out, const void* query, pa_dtype q_dtype,
                                    const void* key_cache, const void* value_cache, pa_dtype kv_dtype,
                                    const float* k_scale, const float* v_scale,
                                    const int32_t* block_tables, int max_blocks_per_seq,
                                    const int32_t* context_lens, int num_seqs, int num_heads,
                                    int num_kv_heads, int head_size, int block_size, int num_blocks,
                                    int max_context_len, float scale, int partition_size,
                                    unsigned int* device_error_out, pa_stream_t stream);

/*
 * Causal paged prefill attention: a chunk of new query tokens per sequence attends to its prefix in
 * the paged cache (page "PagedAttention 与连续批处理：LLM Serving 的底层架构拆解": prefill is the
 * compute-bound phase, section "对 agent 开发者的启示", and a token attends to the tokens before it,
 * section "PagedAttention：把显存做成虚拟内存"; formula of the tutorial page "企业官网建设流程全解析",
 * sec. 2.2). Sequence s owns query rows q_start[s] .. q_start[s+1]-1 (n_s rows); its cache holds
 * context_lens[s] = L_s >= n_s tokens INCLUDING the chunk's own keys and values (write them with
 * pa_reshape_and_cache first), and the chunk is the last n_s of them. For query j of the chunk at
 * position p = L_s - n_s + j and every head h (kv head h / (num_heads / num_kv_heads)):
 *     out[q_start[s] + j][h][:] = softmax_t<=p(scale * q . k_t) . v_t       (fp32 accumulation)
 * Runs on the tcgen05 tensor cores: 128 query rows (128/G tokens x G grouped heads) per CTA.
 *
 *  out, query     [num_q_tokens][num_heads][head_size], q_dtype (PA_F16 / PA_BF16); 16-byte aligned.
 *  key_cache,
 *  value_cache    [num_blocks][block_size][num_kv_heads][head_size]; kv_dtype == q_dtype, or E4M3
 *                 (PA_FP8_E4M3 / PA_FP8_E4M3_BLOCK, head_size 128; the tutorial page, sec. 3.2, stores
 *                 blocks in FP8) dequantised as code * scale as in pa_paged_attention.
 *  k_scale,
 *  v_scale        fp32 scales as in pa_paged_attention ([num_kv_heads], or [num_blocks][num_kv_heads] for
 *                 PA_FP8_E4M3_BLOCK); required for the FP8 formats, else ignored. The FP8 path runs the
 *                 tensor cores on f16: E4M3 values are exact in f16; a bf16 query is rounded to f16
 *                 (magnitudes past 65504 overflow); per-block scales multiply the f16 values (one
 *                 rounding of code * scale), per-kv-head scales are applied in fp32.
 *  block_tables   [num_seqs][max_blocks_per_seq] int32; context_lens [num_seqs] int32;
 *  q_start        [num_seqs + 1] int32, non-decreasing, q_start[0] = 0, q_start[num_seqs] = num_q_tokens.
 *  max_q_len      >= max_s n_s (sizes the grid; tiles past a sequence's chunk exit at once).
 *  workspace      >= PA_WORKSPACE_HEADER_BYTES, zeroed once; its first word is the device error word
 *                 (read with pa_get_device_error).
 * scale must be positive and finite. Supported: head_size 64 or 128; block_size 8, 16, 32, 64 or 128;
 * num_heads / num_kv_heads dividing 128. A chunk outside its context (n_s > L_s, or L_s beyond the block table) sets
 * PA_DEVERR_CONTEXT_LEN and NaNs its rows; a block id outside the pool sets PA_DEVERR_BLOCK_ID.
 */
PA_API pa_status pa_paged_prefill(void* out, const void* query, pa_dtype q_dtype, const void* key_cache,
                                  const void* value_cache, pa_dtype kv_dtype, const float* k_scale,
                                  const float* v_scale, const int32_t* block_tables,
                                  int max_blocks_per_seq, const int32_t* context_lens, const int32_t* q_start,
                                  int num_seqs, int num_q_tokens, int num_heads, int num_kv_heads, int head_size,
                                  int block_size, int num_blocks, int max_q_len, float scale, void* workspace,
                                  size_t workspace_bytes, pa_stream_t stream);

/*
 * Write new tokens into their physical slots ([V] "PagedAttention的破局思路": blocks are filled as the
 * sequence grows). For token i with slot = slot_mapping[i] in [0, num_blocks*block_size):
 *     key_cache[slot / block_size][slot % block_size][h][:] = key[i][h][:]   (same for value)
 * slot < 0 marks padding and is skipped; slots past the pool are skipped too. For an FP8 cache each
 * element stores the E4M3 code of (float)x / scale (IEEE division, round to nearest even, magnitudes
 * beyond 448 saturate, any NaN becomes the canonical NaN code 0x7F), where scale is k_scale[h]
 * (PA_FP8_E4M3) or k_scale[slot / block_size][h] (PA_FP8_E4M3_BLOCK); v_scale likewise for values.
 *
 *  key, value     [num_tokens][num_kv_heads][head_size], in_dtype (PA_F16 or PA_BF16); read only.
 *  key_cache,
 *  value_cache    as above, kv_dtype = in_dtype, PA_FP8_E4M3 or PA_FP8_E4M3_BLOCK; written at the
 *                 given slots only.
 *  k_scale,
 *  v_scale        fp32, required for the FP8 formats: [num_kv_heads] for PA_FP8_E4M3,
 *                 [num_blocks][num_kv_heads] for PA_FP8_E4M3_BLOCK (read only; the caller chooses each
 *                 block's scale before writing into it).
 *  slot_mapping   [num_tokens] int64.
 * Supported: head_size a multiple of 8 and num_kv_heads * head_size <= 2^24 (else PA_ERR_UNSUPPORTED).
 * Two tokens mapped to the same slot race (the result is one of them). num_tokens == 0 is a no-op
 * (pointers may then be null).
 */
PA_API pa_status pa_reshape_and_cache(const void* key, const void* value, pa_dtype in_dtype,
                               void* key_cache, void* value_cache, pa_dtype kv_dtype,
                               const float* k_scale, const float* v_scale,
                               const int64_t* slot_mapping, int num_tokens, int num_kv_heads,
                               int head_size, int block_size, int num_blocks, pa_stream_t stream);

/*
 * Copy-on-write of shared blocks ([V] "PagedAttention的局限性"; sharing by reference count in [T]
 * sec. 2.3): for each pair p, copy the whole key block and the whole value block
 * block_mapping[p][0] -> block_mapping[p][1].
 *
 *  block_mapping  [num_pairs][2] int64 (src, dst), device. Pairs with an id outside [0, num_blocks)
 *                 are skipped. Destinations must be distinct and must not be a source of any pair
 *                 (otherwise the copies race); pa_copy_blocks_check verifies this on a host copy.
 */
PA_API pa_status pa_copy_blocks(void* key_cache, void* value_cache, pa_dtype kv_dtype,
                         const int64_t* block_mapping, int num_pairs, int num_kv_heads,
                         int head_size, int block_size, int num_blocks, pa_stream_t stream);

/*
 * reshape_and_cache for every layer of a model in one launch. The same slot_mapping applies to all
 * layers; layer l reads keys[l]/values[l] ([num_tokens][num_kv_heads][head_size], in_dtype) and writes
 * key_caches[l]/value_caches[l] (scales k_scales[l]/v_scales[l] for FP8). The pointer arrays are
 * DEVICE arrays of num_layers device pointers, each 16-byte aligned; the library cannot inspect them
 * (an invalid entry is the caller's error). Same semantics per layer as pa_reshape_and_cache.
 */
PA_API pa_status pa_reshape_and_cache_layers(const void* const* keys, const void* const* values, pa_dtype in_dtype,
                                             void* const* key_caches, void* const* value_caches, pa_dtype kv_dtype,
                                             const float* const* k_scales, const float* const* v_scales,
                                             const int64_t* slot_mapping, int num_tokens, int num_layers,
                                             int num_kv_heads, int head_size, int block_size, int num_blocks,
                                             pa_stream_t stream);

/*
 * copy_blocks for every layer in one launch: the same (src, dst) mapping applied to key_caches[l] and
 * value_caches[l] for l < num_layers (DEVICE arrays of device pointers, as above). Same semantics per
 * layer as pa_copy_blocks.
 */
PA_API pa_status pa_copy_blocks_layers(void* const* key_caches, void* const* value_caches, int num_layers,
                                       pa_dtype kv_dtype, const int64_t* block_mapping, int num_pairs,
                                       int num_kv_heads, int head_size, int block_size, int num_blocks,
                                       pa_stream_t stream);

/*
 * Swap whole blocks between two pools ([C] "PagedAttention：把显存做成虚拟内存": pages of inactive
 * sequences are moved to CPU memory and brought back when needed). For each pair p, the key block and
 * the value block block_mapping[p][0] of the source pool are copied to block block_mapping[p][1] of the
 * destination pool; both pools have the cache layout above with the same block shape.
 *  dst_*, src_*   pool base pointers; each may be device memory or PINNED host memory (cudaHostAlloc /
 *                 cudaHostRegister / torch pin_memory), reached by the kernel through its unified
 *                 address. Pageable host memory is refused with PA_ERR_INVALID_ARGUMENT.
 *  block_mapping  [num_pairs][2] int64 (src, dst), device or pinned host memory. Pairs with an id outside
 *                 its pool are skipped. Destinations must be distinct (otherwise the copies race).
 *  src_num_blocks, dst_num_blocks  pool sizes in blocks.
 * One launch moves every pair (no per-block copy calls). Asynchronous on `stream`.
 */
PA_API pa_status pa_swap_blocks(void* dst_key_cache, void* dst_value_cache, const void* src_key_cache,
                                const void* src_value_cache, pa_dtype kv_dtype, const int64_t* block_mapping,
                                int num_pairs, int num_kv_heads, int head_size, int block_size,
                                int src_num_blocks, int dst_num_blocks, pa_stream_t stream);

/*
 * Host-side check of a copy_blocks mapping (host pointer, [num_pairs][2] int64): every id in
 * [0, num_blocks), destinations distinct, no destination also a source. PA_OK or
 * PA_ERR_INVALID_ARGUMENT. Makes no CUDA call.
 */
PA_API pa_status pa_copy_blocks_check(const int64_t* host_block_mapping, int num_pairs, int num_blocks);

/*
 * Read the device error word of a workspace into *err_out (host pointer). Synchronises `stream`.
 * Returns PA_ERR_CUDA if the copy or the synchronisation fails.
 */
PA_API pa_status pa_get_device_error(const void* workspace, unsigned int* err_out, pa_stream_t stream);

/* Zero the device error word of a workspace (enqueued on `stream`, asynchronous). Only that word: the
 * rest of the header holds the kernels' own counters, which they leave at zero after every call. */
PA_API pa_status pa_clear_device_error(void* workspace, pa_stream_t stream);

/*
 * Self-test of failure detection (no counterpart on the pages): every wait inside these kernels is
 * bounded, and on expiry sets PA_DEVERR_TIMEOUT and lets the kernel finish instead of hanging. This call
 * launches a one-warp kernel that waits, with the bounded-wait routine the kernels use, on an mbarrier
 * that nothing ever arrives on; after limit_ns nanoseconds (1 ns .. 10 s) it ORs PA_DEVERR_TIMEOUT into
 * *device_error_word (a DEVICE pointer) and returns. Asynchronous on `stream`; the context stays usable.
 */
PA_API pa_status pa_selftest_wait_timeout(unsigned int* device_error_word, unsigned long long limit_ns,
                                          pa_stream_t stream);

/* Static description of a status code. Never NULL. */
PA_API const char* pa_status_string(pa_status status);

#ifdef __cplusplus
}
#endif

#endif /* PAGEDATTN_H_ */
