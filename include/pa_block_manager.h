/*
 * pa_block_manager.h -- host-side manager of the paged KV pool: which physical block holds which
 * logical block of which sequence. It produces the block tables, context lengths and slot mappings
 * that the device calls in pagedattn.h consume, and the (src, dst) pairs for pa_copy_blocks and
 * pa_swap_blocks.
 *
 * The scheme it follows:
 *  - The pool of num_blocks blocks exists from the start (tutorial page "企业官网建设流程全解析",
 *    sec. 3.2 "关键性能优化": pools are preallocated). Blocks are taken only when a token needs one
 *    (page "vLLM的诞生背景：大模型推理的痛点与PagedAttention的破局", section "PagedAttention的破局思路").
 *  - Each sequence has a block table from logical to physical blocks (tutorial sec. 2.1).
 *  - Blocks are shared by reference count (tutorial sec. 2.3 "显存共享机制"): pa_bm_fork shares every
 *    block of a parent (within a request, e.g. beam search); pa_bm_add_sequence with a prefix shares
 *    the parent's full blocks of the common prefix (between requests). Only whole blocks are shared:
 *    a prefix is shared up to the last block boundary it covers (page "PagedAttention 与连续批处理：
 *    LLM Serving 的底层架构拆解", section "对 agent 开发者的启示").
 *  - A token written into a block whose count is above one goes to a fresh copy of that block
 *    (copy-on-write; "vLLM的诞生背景" page, section "PagedAttention的局限性"). The (old, new) pair is
 *    returned; the caller runs pa_copy_blocks on it BEFORE writing the new tokens.
 *  - A finished sequence's blocks are released; a block is free again when its count is zero
 *    ("PagedAttention 与连续批处理" page, section "连续批处理：让 GPU 永远有活干").
 *  - Inactive sequences can be moved to a host pool and back ("PagedAttention 与连续批处理" page,
 *    section "PagedAttention：把显存做成虚拟内存"). Each block of the swapped sequence gets its own host
 *    block; a block still shared with a resident sequence stays on the device for it. A sequence that
 *    comes back holds private blocks.
 *
 * Allocation policy (fixed, so two runs with the same calls make the same decisions): free blocks
 * are a stack that starts as 0, 1, 2, ... from the top; a released block goes back on top. Within
 * one call, sequences are served in the order given and a released table is walked front to back.
 *
 * Every call either completes or returns an error and leaves the manager unchanged; that includes a
 * failed host allocation, which returns PA_ERR_HOST_MEMORY (no C++ exception crosses the ABI). A call
 * performs its allocations before its first change. Sequence ids are
 * any int64 >= 0 chosen by the caller; PA_BM_NO_SEQUENCE (-1) means "none". All arrays are HOST
 * memory owned by the caller (pinned memory works and lets the outputs go straight to the device).
 * A manager may be used from several threads: calls are serialised by a lock inside it.
 */
#ifndef PA_BLOCK_MANAGER_H_
#define PA_BLOCK_MANAGER_H_

#include "pagedattn.h"

#ifdef __cplusplus
extern "C" {
#endif

typedef struct pa_block_manager pa_block_manager;

#define PA_BM_NO_SEQUENCE ((int64_t)-1)

/* A manager of num_blocks device blocks of block_size tokens and num_host_blocks host blocks (0: no
 * swapping). PA_ERR_INVALID_ARGUMENT for non-positive sizes or a null out. */
PA_API pa_status pa_bm_create(int num_blocks, int block_size, int num_host_blocks, pa_block_manager** out);

/* Frees the manager (null is ignored). */
PA_API void pa_bm_destroy(pa_block_manager* bm);

/*
 * A new sequence of num_tokens prompt tokens. With prefix_seq != PA_BM_NO_SEQUENCE, its first
 * prefix_tokens tokens are those of resident sequence prefix_seq, and the full blocks among them are
 * shared. The slots of the tokens that must still be written (token shared_blocks*block_size up to
 * num_tokens-1, in order) go to slots_out[0 .. *num_slots_out); slots_capacity must be >= num_tokens.
 * Errors: unknown prefix or duplicate id, prefix_tokens > num_tokens -> INVALID_ARGUMENT; too few
 * free blocks -> OUT_OF_BLOCKS.
 */
PA_API pa_status pa_bm_add_sequence(pa_block_manager* bm, int64_t seq_id, int64_t num_tokens, int64_t prefix_seq,
                                    int64_t prefix_tokens, int64_t* slots_out, int64_t slots_capacity,
                                    int64_t* num_slots_out);

/* child becomes a copy of resident sequence parent that shares all of its blocks. */
PA_API pa_status pa_bm_fork(pa_block_manager* bm, int64_t parent, int64_t child);

/*
 * One new token for each of the n resident sequences seq_ids[0..n) (distinct). slot_mapping_out[i]
 * receives the slot of sequence i's token (block * block_size + offset); cow_pairs_out ([n][2] int64,
 * (src, dst)) receives the copy-on-write pairs, *num_cow_out of them. OUT_OF_BLOCKS when the pool
 * cannot serve all n (nothing changes).
 */
PA_API pa_status pa_bm_append_slots(pa_block_manager* bm, const int64_t* seq_ids, int n, int64_t* slot_mapping_out,
                                    int64_t* cow_pairs_out, int* num_cow_out);

/*
 * Rows of block tables for the n resident sequences seq_ids[0..n): tables_out is [n][max_blocks]
 * int32 (entries past a sequence's blocks are `pad`), context_lens_out is [n] int32.
 * INVALID_ARGUMENT if a sequence has more than max_blocks blocks or is not resident.
 */
PA_API pa_status pa_bm_block_tables(pa_block_manager* bm, const int64_t* seq_ids, int n, int32_t* tables_out,
                                    int max_blocks, int32_t pad, int32_t* context_lens_out);

/*
 * One decode step's plan: pa_bm_append_slots followed by pa_bm_block_tables for the same sequences,
 * as one all-or-nothing call (the tables include the new tokens).
 */
PA_API pa_status pa_bm_plan_decode(pa_block_manager* bm, const int64_t* seq_ids, int n, int64_t* slot_mapping_out,
                                   int64_t* cow_pairs_out, int* num_cow_out, int32_t* tables_out, int max_blocks,
                                   int32_t pad, int32_t* context_lens_out);

/* Releases a sequence, resident or swapped out. */
PA_API pa_status pa_bm_free_sequence(pa_block_manager* bm, int64_t seq_id);

/*
 * Moves a resident sequence to the host pool: mapping_out ([capacity][2] int64) receives one
 * (device block, host block) pair per table entry, in table order, for pa_swap_blocks. capacity must
 * be >= the sequence's block count. OUT_OF_BLOCKS when the host pool is short.
 */
PA_API pa_status pa_bm_swap_out(pa_block_manager* bm, int64_t seq_id, int64_t* mapping_out, int capacity,
                                int* num_pairs_out);

/* Brings a swapped sequence back: (host block, device block) pairs, as above. */
PA_API pa_status pa_bm_swap_in(pa_block_manager* bm, int64_t seq_id, int64_t* mapping_out, int capacity,
                               int* num_pairs_out);

/* Free device and host blocks (either pointer may be null). */
PA_API pa_status pa_bm_num_free_blocks(pa_block_manager* bm, int* device_out, int* host_out);

/* A sequence's token count, block count and state (1 = swapped out); INVALID_ARGUMENT if unknown. */
PA_API pa_status pa_bm_sequence_info(pa_block_manager* bm, int64_t seq_id, int64_t* num_tokens_out,
                                     int* num_blocks_out, int* swapped_out);

/* Reference count of a device block. */
PA_API pa_status pa_bm_ref_count(pa_block_manager* bm, int block, int* count_out);

#ifdef __cplusplus
}
#endif

#endif  /* PA_BLOCK_MANAGER_H_ */
