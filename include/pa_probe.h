/*
 * pa_probe.h -- read-bandwidth probes of libpagedattn.so: the practical ceilings that the decode
 * attention kernel is measured against. The pages have no counterpart; they only say that decode is
 * memory-bound (page "PagedAttention 与连续批处理：LLM Serving 的底层架构拆解", section "对 agent
 * 开发者的启示"), which makes a read ceiling the yardstick.
 *
 * Each probe reads its bytes with 16-byte vector loads that bypass L1 and does no other work: it folds
 * the loaded words into a register and writes one word to *sink (a DEVICE pointer) only if the fold
 * hits a fixed value, so the loads cannot be removed and nothing else is written. Same conventions as
 * pagedattn.h: device pointers, validation before any CUDA call, asynchronous on `stream`, launch
 * failures return PA_ERR_CUDA. Both grids are sized from the device's SM count.
 */
#ifndef PA_PROBE_H_
#define PA_PROBE_H_

#include "pagedattn.h"

#ifdef __cplusplus
extern "C" {
#endif

/*
 * Sequential read of `bytes` bytes of `buf`, `repeat` times over. buf 16-byte aligned, bytes a positive
 * multiple of 16, 1 <= repeat <= 4096. With a buffer far larger than L2 and repeat = 1 this is the
 * HBM read ceiling; with a buffer well under L2 and a large repeat, the L2 read ceiling.
 */
PA_API pa_status pa_probe_stream_read(const void* buf, size_t bytes, int repeat, unsigned long long* sink,
                                      pa_stream_t stream);

/*
 * Reads exactly the K and V rows of every valid token of a paged decode batch, once, through the block
 * table: for each sequence s and logical block j < ceil(context_lens[s] / block_size), the first
 * min(block_size, context_lens[s] - j*block_size) token rows ([num_kv_heads][head_size], contiguous
 * in the cache layout of pagedattn.h) of block block_tables[s][j] in key_cache and value_cache. These
 * are the bytes decode attention must read, fetched with plain loads and no compute: the ceiling of the
 * batch's own access pattern. Block ids outside [0, num_blocks) and lengths past the table are skipped.
 * Arguments as in pa_paged_attention; kv_dtype any of pa_dtype; num_seqs <= 65535.
 */
PA_API pa_status pa_probe_paged_read(const void* key_cache, const void* value_cache, pa_dtype kv_dtype,
                                     const int32_t* block_tables, int max_blocks_per_seq,
                                     const int32_t* context_lens, int num_seqs, int num_kv_heads, int head_size,
                                     int block_size, int num_blocks, unsigned long long* sink,
                                     pa_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* PA_PROBE_H_ */
