// pa_attention.cuh -- paged decode attention kernels for sm_100a.
//
// What is computed (tutorial page "企业官网建设流程全解析", sec. 2.2 "分块注意力计算过程": the formula
// softmax(QK^T/sqrt(d))V, normalised over the whole context -- NOT that section's per-block loop, whose
// per-block softmaxes are summed without renormalisation): for sequence s and query head h,
//   out[s][h] = sum_t exp(z_t - m) v_t / sum_t exp(z_t - m),  z_t = scale * q[s][h] . k_t,
// where token t is found through the block table (sec. 2.1 "基本数据结构设计"; page "PagedAttention 与
// 连续批处理：LLM Serving 的底层架构拆解", section "PagedAttention：把显存做成虚拟内存").
//
// Design (B200). Decode reads every K/V byte once; the kernel is shaped so that HBM sees long
// contiguous reads and stays busy:
//  * A work item is (context partition, sequence, block of 8 kv heads [, query-head subgroup]).
//    Because a cache block is laid out [token][kv head][d], the 8 heads of one token are contiguous,
//    and for an 8-kv-head cache a whole block is one contiguous run.
//  * Persistent CTAs, one per SM, take items from an atomic counter in the workspace header in
//    partition-major order (every sequence's first partition before any second one); the last CTA to
//    finish resets the counter.
//  * Warp 0 is the producer. Per item it bulk-copies the query rows of the 8 heads into shared memory;
//    then, for each 8-token stage, it reads one block-table entry (prefetched a window at a time) and
//    issues 4-D TMA tile loads {128-byte chunk, 8 tokens, 8 kv heads, 1 block} of K and V (128-byte
//    swizzle; the tensor map lists the token dimension before the head dimension, so each head's 8
//    token rows form one swizzle atom) into a shared-memory ring whose slots are guarded by mbarriers,
//    with a small message (item, valid tokens, first/last stage). The page-table walk is a TMA
//    coordinate.
//  * Warps 1..8 are consumers; warp w owns kv head w of the block for the whole item and keeps an fp32
//    online-softmax state (running max m, running sum l, accumulator acc[G][d]) for the G query heads
//    of that kv head (grouped-query heads are batched: each K/V element is read once for all G heads).
//    Two ways to compute, chosen at compile time:
//    - Tensor cores (G >= 2): Q[G x d] K^T and P V are contractions over d and over the stage's
//      tokens, done with warp-level mma.sync tiles (m16n8k16 for S = Q K^T with the query rows held as
//      A fragments, m16n8k8 for O += P V). 16-bit K^T and V come from the swizzled tiles through
//      ldmatrix (V transposed); FP8 pairs are read into the fragment layout and widened to f16 pairs
//      by one hardware conversion (exact). The score fragment becomes the P fragment in registers;
//      the softmax statistics are per query head (one quad of lanes per head).
//    - CUDA cores (G == 1): NS >= 8 lanes cooperate on one token (each holds 1/NS of
//      d and the G query rows in registers, pre-scaled by scale*log2(e)); a butterfly reduce-scatter
//      leaves each lane with the full score of one head; p goes through a per-warp shared buffer; for
//      PV, D/8 lanes cover one V row and every lane accumulates all G heads; packed f32x2 FMAs.
//    Either way: online softmax with alpha = 2^(m_old - m_new), p = 2^(z - m_new), fp32 statistics
//    and accumulators. At the end of an item each warp writes its heads' normalised output, or
//    (m, l, acc/l) partials that the reduce kernel merges across partitions (log-sum-exp merge).
// Arithmetic order depends only on logical token positions, never on physical block ids or on which
// CTA handled an item, so outputs are bitwise invariant to block placement and deterministic.
#pragma once

#include <type_traits>

#include "pa_device.cuh"

namespace pa {

constexpr int kHeadBlock = 8;            // kv heads per work item (one consumer warp each)
constexpr int kConsumerWarps = kHeadBlock;
constexpr int kBoxTokens = 8;            // tokens per TMA box (block_size >= 8); one swizzle atom
constexpr int kMaxStages = 8;            // ring depth cap (the depth itself is per variant, see Layout)
constexpr int kSmemBudget = 216 * 1024;  // ring + query + small tables (the order table and slack come on top; 227 KB per CTA)
constexpr int kQueryBuffers = 1;         // consumers copy the query into registers at an item's first stage
constexpr int kIdWindow = 4;             // block ids prefetched per item: 32 * kIdWindow stages
constexpr int kThreads = (kConsumerWarps + 1) * 32;
constexpr int kPartitionQuantum = 64;    // partition sizes are multiples of this
constexpr int kOrderMaxSeqs = 1024;      // batches up to this size take their items longest first
#ifndef PA_ORDER_MAX_ROUNDS
#define PA_ORDER_MAX_ROUNDS 128
#endif
constexpr int kOrderMaxRounds = PA_ORDER_MAX_ROUNDS;  // ... and the context splits into at most this many partitions
constexpr int kRemBins = 128;            // partial partitions are ordered by size in this many bins
constexpr int kClaimAhead = 6;           // the next item is claimed when this many stages remain to issue
constexpr float kLog2e = 1.4426950408889634f;

// Workspace header words: error bits, work counter, finished-CTA counter.
constexpr int kWsError = 0;
constexpr int kWsWork = 1;
constexpr int kWsDone = 2;

// Stage message flags.
constexpr int kMsgFirst = 1;
constexpr int kMsgBlkShift = 4;  // StageMsg.flags: bits 0-3 flags, bits 4-31 box 0's block id
constexpr int kMsgLast = 2;
constexpr int kMsgBadBlock = 4;

struct AttnArgs {
  void* out;                    // [S][H][D] query dtype
  const void* query;            // [S][H][D]
  const float* k_scale;         // [Hkv] (FP8 only)
  const float* v_scale;
  const int32_t* block_tables;  // [S][max_blocks_per_seq]
  const int32_t* context_lens;  // [S]
  float* part_m;                // [S][H][P]
  float* part_l;                // [S][H][P]
  float* part_o;                // [S][H][P][D]
  unsigned int* header;         // workspace header: [0] error bits, [1] work counter, [2] done counter
  int max_blocks_per_seq;
  int num_seqs;
  int num_heads;
  int num_kv_heads;
  int head_blocks;              // ceil(num_kv_heads / kHeadBlock)
  int group;                    // num_heads / num_kv_heads
  int subgroups;                // query-head subgroups per kv head (ceil(group / G))
  int block_size;
  int num_blocks;
  int partition_size;           // tokens per partition, multiple of kPartitionQuantum
  int num_partitions;
  unsigned int num_items;       // num_partitions * num_seqs * head_blocks * subgroups
  float scale_log2;             // softmax scale * log2(e)
  int scale_block_stride;       // FP8 scales: 0 = per kv head, num_kv_heads = per (block, kv head)
  unsigned long long* trace;    // timing records, written only by builds with PA_TRACE defined (else null)
};

// Timing records of a PA_TRACE build (%globaltimer, ns), in 64-bit words: [0] ~(first start of a
// split-K reduce CTA), [1] last end of one; CTA c at kTraceCtaBase + 4c: start, end, items, SM id;
// item i at kTraceItemBase + 4i: producer start, consumer finish, CTA, tokens.
constexpr int kTraceMaxCtas = 1024;
constexpr int kTraceCtaBase = 8;
constexpr int kTraceItemBase = kTraceCtaBase + 4 * kTraceMaxCtas;

__host__ __device__ constexpr int ilog2(int x) { return x <= 1 ? 0 : 1 + ilog2(x / 2); }
__host__ __device__ constexpr int cmin(int a, int b) { return a < b ? a : b; }
__host__ __device__ constexpr int cmax(int a, int b) { return a > b ? a : b; }

template <int D, int G, int EB>
struct Shape {
  static constexpr int kRowBytes = D * EB;
  static constexpr int kChunks = kRowBytes / 128;        // 128-byte swizzle chunks per row
  static constexpr int kChunkElems = 128 / EB;
  static constexpr int kPieceBytes = 8 * EB;             // one piece = 8 elements
  static constexpr int kPiecesPerRow = D / 8;
  // QK mapping: NS lanes per token, NS >= 8 so that a phase reads distinct units of one row.
  static constexpr int kNS = cmin(D / 8, cmax(8, 2 * G));
  static constexpr int kLog2NS = ilog2(kNS);
  static constexpr int kLog2G = ilog2(G);
  static constexpr int kTPI = 32 / kNS;                  // tokens per QK step
  static constexpr int kNPL = kPiecesPerRow / kNS;       // pieces per lane
  // A stage is kGroups boxes of 8 tokens: 8 for 16-bit caches, 16 for FP8 (same bytes per stage).
  static constexpr int kGroups = (EB == 1) ? 2 : 1;
  static constexpr int kTS = kBoxTokens * kGroups;      // tokens per stage
  static constexpr int kIters = kTS / kTPI;
  static constexpr int kTsShift = kLog2NS;               // token-slot lane bits sit above the ds bits
  // PV mapping: LPT lanes per token.
  static constexpr int kLPT = D / 8;
  static constexpr int kLog2LPT = ilog2(kLPT);
  static constexpr int kTPV = 32 / kLPT;
  // One stage: [K|V][chunk][group][head][8 tokens][128 B]; tile row r = group*64 + head*8 + token%8.
  static constexpr int kBoxBytes = kBoxTokens * kHeadBlock * 128;
  static constexpr int kChunkBytes = kGroups * kBoxBytes;
  static constexpr int kTileBytes = kChunks * kChunkBytes;
  static constexpr int kStageBytes = 2 * kTileBytes;
  // Tensor-core path: at least two query heads per kv head. FP8 caches enter the tensor cores as
  // f16 (every E4M3 value is exact in f16), with f16 query fragments.
  static constexpr bool kMma = G >= 2;
  static constexpr int kKSteps = D / 16;                 // m16n8k16 steps over d
  static constexpr int kNBlocks = D / 8;                 // n8 blocks of the output row
  static_assert(kRowBytes == 128 || kRowBytes == 256, "row must be 128 or 256 bytes");
  static_assert(kNS >= 8 && G <= kNS, "lane mapping");
  static_assert(kNPL >= 1 && kNPL * kNS == kPiecesPerRow, "pieces must split evenly");
  static_assert(kIters >= 1, "stage shorter than one QK step");
};

struct StageMsg {
  int item;    // CTA-local item sequence number, -1 = no more work
  int ntok;    // valid tokens in the stage
  int flags;   // kMsgFirst | kMsgLast | kMsgBadBlock
  int blk1;    // physical blocks of the stage's two 8-token boxes, for per-block scales (0 when a box
};             // is not loaded); box 0's is carried in flags >> kMsgBlkShift

struct ItemInfo {
  int s, part, kvh0, h_sub, heads, write_final, pad0, pad1;  // h_sub: first query-head offset in a group
};

// Work order of one launch, built by every CTA from the context lengths (the same table in each):
// first the full partitions round by round (round r = partition r of every sequence that has more
// than r full partitions, sequences with more full partitions first), then each sequence's last,
// partial partition (or the single item of an empty or invalid context), largest first. Tickets map
// one to one onto real items, and the smallest items come last.
struct OrderTable {
  uint16_t full[kOrderMaxSeqs];          // sequences by full-partition count, descending
  uint16_t part[kOrderMaxSeqs];          // sequences with a partial item, by its size, descending
  int round_start[kOrderMaxRounds + 1];  // round r's first index into `full`-ordered items
  int nf_cursor[kOrderMaxRounds + 1];    // counting-sort cursors by full-partition count
  int rem_cursor[kRemBins];              // counting-sort cursors by partial size
  int ok, full_items, part_items, pad;
};

// Shared-memory layout (byte offsets from the 1024-aligned base).
template <typename QT, int D, int G, int EB>
struct Layout {
  using S = Shape<D, G, EB>;
  // Query rows [8 kv heads][G][kQRow]: each row padded by 32 bytes, so that the fragment loads of the
  // G rows at an item's start fall in different banks (rows 256 bytes apart would share them).
  static constexpr int kQRow = D + 32 / int(sizeof(QT));
  static constexpr int kQueryOne = kHeadBlock * G * kQRow * int(sizeof(QT));
  static constexpr int kSmall = kConsumerWarps * S::kTS * G * 4 + kConsumerWarps * G * 4 + 1024;
  // Ring depth: as many stages as the budget leaves after the query buffers and small tables.
  static constexpr int kStages = cmin(kMaxStages, (kSmemBudget - kQueryBuffers * kQueryOne - kSmall) / S::kStageBytes);
  static_assert(kStages >= 2, "ring too shallow");
  static constexpr int kRing = 0;
  static constexpr int kRingBytes = kStages * S::kStageBytes;
  static constexpr int kQuery = kRingBytes;
  static constexpr int kPbuf = kQuery + kQueryBuffers * kQueryOne;             // [W][TS][G] f32
  static constexpr int kAbuf = kPbuf + kConsumerWarps * S::kTS * G * 4;      // [W][G] f32
  static constexpr int kMsgs = (kAbuf + kConsumerWarps * G * 4 + 15) / 16 * 16;
  static constexpr int kInfo = kMsgs + kStages * int(sizeof(StageMsg));
  static constexpr int kBars = (kInfo + kQueryBuffers * int(sizeof(ItemInfo)) + 7) / 8 * 8;
  // full[kStages], empty[kStages], qfull[NQ], qempty[NQ]
  static constexpr int kNumBars = 2 * kStages + 2 * kQueryBuffers;
  static constexpr int kOrder = (kBars + kNumBars * 8 + 15) / 16 * 16;
  static constexpr int kEnd = kOrder + int(sizeof(OrderTable));
  static constexpr int kAllocBytes = kEnd + 1024;  // alignment slack
  static_assert(kAllocBytes <= 227 * 1024, "shared memory layout too large");
};

// Tile row of token t (within the stage) of kv head `head`: boxes of 8 tokens, each [head][token].
__device__ __forceinline__ int tile_row(int head, int t) { return (t >> 3) * (kHeadBlock * kBoxTokens) + head * kBoxTokens + (t & 7); }

// Byte offset of piece `pc` (8 elements) of tile row r inside a [chunk][rows][128 B] tile written by
// TMA with the 128-byte swizzle (16-byte unit u of row r lives at unit u ^ (r & 7) = u ^ (token % 8)).
template <class S>
__device__ __forceinline__ uint32_t piece_offset(int r, int pc) {
  const int byte = pc * S::kPieceBytes;
  const int c = byte >> 7;
  const int b = byte & 127;
  return static_cast<uint32_t>(c * S::kChunkBytes + r * 128 + ((((b >> 4) ^ (r & 7)) << 4) | (b & 15)));
}

// Piece read by a lane in QK step j. FP8 rows with 8 lanes per token alternate halves by token
// parity so that two tokens sharing a half-warp phase hit disjoint banks.
template <class S, int EB>
__device__ __forceinline__ int qk_piece(int j, int ds, int tslot) {
  if constexpr (EB == 1 && S::kNS == 8 && S::kNPL == 2) return ds + 8 * (j ^ (tslot & 1));
  return ds + S::kNS * j;
}

template <int G, int NS_LOG2>
__device__ __forceinline__ float reduce_scatter(float (&v)[G], int lane) {
  // Halving exchange over the ds lane bits (the low NS_LOG2 bits), high bit first: after log2(G)
  // halvings each lane holds one head's partial sum; the remaining bits finish a full reduction.
  constexpr int kLog2G = ilog2(G);
#pragma unroll
  for (int step = 0; step < NS_LOG2; ++step) {
    const int mask = 1 << (NS_LOG2 - 1 - step);
    if (step < kLog2G) {
      const int half = (G >> step) >> 1;
      const bool upper = (lane & mask) != 0;
#pragma unroll
      for (int i = 0; i < G / 2; ++i) {
        if (i < half) {
          const float send = upper ? v[i] : v[i + half];
          const float keep = upper ? v[i + half] : v[i];
          v[i] = keep + __shfl_xor_sync(0xffffffffu, send, mask);
        }
      }
    } else {
      v[0] += __shfl_xor_sync(0xffffffffu, v[0], mask);
    }
  }
  return v[0];
}

__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Item index -> (partition, sequence, head block, query-head subgroup). Partition-major.
struct ItemCoord {
  int part, s, hb, sub;
};
__device__ __forceinline__ ItemCoord decode_item(unsigned int idx, const AttnArgs& a) {
  const unsigned int per_seq = static_cast<unsigned int>(a.head_blocks) * a.subgroups;
  const unsigned int per_part = static_cast<unsigned int>(a.num_seqs) * per_seq;
  ItemCoord c;
  c.part = static_cast<int>(idx / per_part);
  unsigned int r = idx - static_cast<unsigned int>(c.part) * per_part;
  c.s = static_cast<int>(r / per_seq);
  r -= static_cast<unsigned int>(c.s) * per_seq;
  c.hb = static_cast<int>(r / a.subgroups);
  c.sub = static_cast<int>(r - static_cast<unsigned int>(c.hb) * a.subgroups);
  return c;
}

__device__ __forceinline__ bool context_len_invalid(int L, const AttnArgs& a) {
  return L < 0 || L > a.max_blocks_per_seq * a.block_size || L > a.num_partitions * a.partition_size;
}

// How a sequence enters the work order: its full partitions, whether it has one more item (a partial
// last partition, or the single item of an empty or invalid context), and that item's size bin.
struct SeqClass {
  int nf, pr, bin;
};
__device__ __forceinline__ SeqClass classify_seq(int L, const AttnArgs& a) {
  const bool valid = L > 0 && !context_len_invalid(L, a);
  const int ps = a.partition_size;
  SeqClass c;
  c.nf = valid ? L / ps : 0;
  const int rem = valid ? L % ps : 0;
  c.pr = (!valid || rem != 0) ? 1 : 0;
  c.bin = static_cast<int>((static_cast<long long>(rem) * kRemBins) / ps);
  return c;
}

// Exclusive scan of v[0..n) (n <= 32 * 5) by one warp, in place; returns the total.
__device__ __forceinline__ int warp_exclusive_scan(int* v, int n, int lane) {
  constexpr int kPer = 5;
  int local[kPer];
  int sum = 0;
#pragma unroll
  for (int i = 0; i < kPer; ++i) {
    const int idx = lane * kPer + i;
    local[i] = idx < n ? v[idx] : 0;
    sum += local[i];
  }
  int incl = sum;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  const int total = __shfl_sync(0xffffffffu, incl, 31);
  int run = incl - sum;
  __syncwarp();
#pragma unroll
  for (int i = 0; i < kPer; ++i) {
    const int idx = lane * kPer + i;
    if (idx < n) v[idx] = run;
    run += local[i];
  }
  __syncwarp();
  return total;
}

// Builds the work order (one warp). Counting sorts with ranks taken in sequence order (match_any),
// so every CTA builds the same table. Leaves ok = 0 when the batch is too large for the table.
__device__ __noinline__ static void build_order(OrderTable* ot, const AttnArgs& a, int lane) {
  const int S = a.num_seqs, P = a.num_partitions;
  if (S > kOrderMaxSeqs || P > kOrderMaxRounds) {
    if (lane == 0) ot->ok = 0;
    __syncwarp();
    return;
  }
  // Histograms, highest count first: index P - nf and kRemBins - 1 - bin.
  for (int i = lane; i <= P; i += 32) ot->nf_cursor[i] = 0;
  for (int i = lane; i < kRemBins; i += 32) ot->rem_cursor[i] = 0;
  __syncwarp();
  for (int s = lane; s < S; s += 32) {
    const SeqClass c = classify_seq(__ldg(a.context_lens + s), a);
    atomicAdd(&ot->nf_cursor[P - c.nf], 1);
    if (c.pr) atomicAdd(&ot->rem_cursor[kRemBins - 1 - c.bin], 1);
  }
  __syncwarp();
  // Round r holds the sequences with more than r full partitions: nf_cursor (after the scan) at index
  // P - r is how many sequences have more than r of them.
  const int part_items = warp_exclusive_scan(ot->rem_cursor, kRemBins, lane);
  warp_exclusive_scan(ot->nf_cursor, P + 1, lane);
  for (int r = lane; r < P; r += 32) ot->round_start[r] = ot->nf_cursor[P - r];  // sequences in round r
  __syncwarp();
  const int full_items = warp_exclusive_scan(ot->round_start, P, lane);
  if (lane == 0) {
    ot->round_start[P] = full_items;
    ot->full_items = full_items;
    ot->part_items = part_items;
    ot->ok = 1;
  }
  __syncwarp();
  // Scatter in sequence order: lanes with the same key take consecutive places, by lane.
  const unsigned lt = (1u << lane) - 1u;
  for (int s0 = 0; s0 < S; s0 += 32) {
    const int s = s0 + lane;
    const bool in = s < S;
    const SeqClass c = classify_seq(in ? __ldg(a.context_lens + s) : 0, a);
    const int kf = in ? P - c.nf : -1;
    const unsigned peers_f = __match_any_sync(0xffffffffu, kf);
    const int base_f = in ? ot->nf_cursor[kf] : 0;
    const int kr = (in && c.pr) ? kRemBins - 1 - c.bin : -1;
    const unsigned peers_r = __match_any_sync(0xffffffffu, kr);
    const int base_r = kr >= 0 ? ot->rem_cursor[kr] : 0;
    __syncwarp();
    if (in) {
      ot->full[base_f + __popc(peers_f & lt)] = static_cast<uint16_t>(s);
      if ((peers_f & lt) == 0) ot->nf_cursor[kf] = base_f + __popc(peers_f);
    }
    if (kr >= 0) {
      ot->part[base_r + __popc(peers_r & lt)] = static_cast<uint16_t>(s);
      if ((peers_r & lt) == 0) ot->rem_cursor[kr] = base_r + __popc(peers_r);
    }
    __syncwarp();
  }
}

// Ticket -> item under the work order. part = -1 marks a sequence's last item, whose partition index
// follows from its length (partial partition, or 0 for an empty or invalid context).
__device__ __forceinline__ ItemCoord decode_ordered(unsigned int t, const AttnArgs& a, const OrderTable* ot) {
  const unsigned int per = static_cast<unsigned int>(a.head_blocks) * a.subgroups;
  const unsigned int q = t / per, r = t - q * per;
  ItemCoord c;
  c.hb = static_cast<int>(r / a.subgroups);
  c.sub = static_cast<int>(r - static_cast<unsigned int>(c.hb) * a.subgroups);
  if (q < static_cast<unsigned int>(ot->full_items)) {
    int lo = 0, hi = a.num_partitions - 1;  // the last round whose start is <= q
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (static_cast<unsigned int>(ot->round_start[mid]) <= q) lo = mid; else hi = mid - 1;
    }
    c.part = lo;
    c.s = ot->full[q - ot->round_start[lo]];
  } else {
    c.part = -1;
    c.s = ot->part[q - ot->full_items];
  }
  return c;
}

// BS: FP8 cache with per-(block, kv head) scales (args.scale_block_stride != 0); a separate
// instantiation so that the per-head FP8 path carries none of its work.
template <typename QT, typename KVT, int D, int G, bool BS>
__global__ void __launch_bounds__(kThreads, 1)
paged_attention_main(const __grid_constant__ CUtensorMap tmap_k, const __grid_constant__ CUtensorMap tmap_v,
                     const AttnArgs args) {
  constexpr int EB = Elem<KVT>::kBytes;
  using S = Shape<D, G, EB>;
  using Lay = Layout<QT, D, G, EB>;
  using Piece = typename Elem<KVT>::Piece;
  using MmaT = typename std::conditional<EB == 2, KVT, __half>::type;  // tensor-core input type
  constexpr int kStages = Lay::kStages;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  unsigned int* err = args.header + kWsError;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  StageMsg* msgs = reinterpret_cast<StageMsg*>(smem + Lay::kMsgs);
  ItemInfo* infos = reinterpret_cast<ItemInfo*>(smem + Lay::kInfo);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Lay::kBars);
  uint64_t* full = bars;
  uint64_t* empty = bars + kStages;
  uint64_t* qfull = bars + 2 * kStages;
  uint64_t* qempty = qfull + kQueryBuffers;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kStages; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], kConsumerWarps);
    }
    for (int i = 0; i < kQueryBuffers; ++i) {
      mbar_init(&qfull[i], 1);
      mbar_init(&qempty[i], kConsumerWarps);
    }
    fence_mbar_init();
  }
  // Everything above touched shared memory only; from here on the previous kernel's writes (the new
  // tokens in the cache, a reset workspace) must be visible.
  grid_dependency_wait();
  grid_dependents_launch();
#ifdef PA_TRACE
  if (threadIdx.x == 0 && blockIdx.x < kTraceMaxCtas) {
    unsigned int smid;
    asm volatile("mov.u32 %0, %%smid;" : "=r"(smid));
    args.trace[kTraceCtaBase + 4 * blockIdx.x] = global_timer_ns();
    args.trace[kTraceCtaBase + 4 * blockIdx.x + 3] = smid;
  }
#endif
  OrderTable* order = reinterpret_cast<OrderTable*>(smem + Lay::kOrder);
  if (warp == 0) build_order(order, args, lane);
  __syncthreads();

  if (warp == 0) {
    // =============================== producer warp ===============================
    if (lane == 0) {
      tma_prefetch_desc(&tmap_k);
      tma_prefetch_desc(&tmap_v);
    }
    const int bs = args.block_size;
    const int boxes_per_part = args.partition_size / kBoxTokens;
    // K/V are read once per item: let L2 evict them first, keeping partial results, queries and
    // block tables resident.
    const uint64_t kv_policy = l2_policy_evict_first();
    bool aborted = false;
    int local = 0;   // CTA-local item sequence number
    int issued = 0;  // stages issued so far (ring position)

    // The next item is claimed late -- when kClaimAhead stages of the current one remain to be issued --
    // so that a CTA holds at most a few stages of unstarted work while others may run dry; its context
    // length and a window of its block ids (one id per lane per 32 boxes) are loaded while those stages
    // issue. Only the table entries the context needs (the first ceil(L / block_size), at most the
    // table's width) are ever read; the rest of the window holds 0 and is never used.
    const bool ordered = order->ok != 0;
    const unsigned int num_tickets = ordered
        ? static_cast<unsigned int>(order->full_items + order->part_items) * args.head_blocks * args.subgroups
        : args.num_items;
    unsigned int cur_idx = 0, nxt_idx = 0;
    ItemCoord cur_c{}, nxt_c{};
    int cur_L = 0, nxt_L = 0;
    int cur_ids[kIdWindow], nxt_ids[kIdWindow];
    bool have_next = false;
#define PA_PREPARE(IDX, C, LV, IDS)                                                                    \
  do {                                                                                                 \
    if ((IDX) < num_tickets) {                                                                         \
      C = ordered ? decode_ordered((IDX), args, order) : decode_item((IDX), args);                     \
      LV = __ldg(args.context_lens + C.s);                                                             \
      if (C.part < 0) C.part = (LV > 0 && !context_len_invalid(LV, args)) ? (LV - 1) / args.partition_size : 0; \
      const int need_ = LV <= 0 ? 0 : cmin(args.max_blocks_per_seq, LV / bs + (LV % bs != 0));         \
      const int32_t* row_ = args.block_tables + static_cast<size_t>(C.s) * args.max_blocks_per_seq;    \
      _Pragma("unroll") for (int j_ = 0; j_ < kIdWindow; ++j_) {                                       \
        const int entry_ = ((C.part * boxes_per_part + j_ * 32 + lane) * kBoxTokens) / bs;             \
        IDS[j_] = entry_ < need_ ? __ldg(row_ + entry_) : 0;                                           \
      }                                                                                                \
    }                                                                                                  \
  } while (0)
// Claiming the next item takes three steps spread over consecutive stages of the current one, so that
// no step waits on the one before it: (1) the ticket's atomic, (2) the ticket's decode and the context
// length's load, (3) the block-id window's loads. Each step is a no-op once done.
#define PA_CLAIM_STEP()                                                                                \
  do {                                                                                                 \
    if (claim_step == 0) {                                                                             \
      if (lane == 0) pend_t = atomicAdd(args.header + kWsWork, 1u);                                    \
    } else if (claim_step == 1) {                                                                      \
      nxt_idx = __shfl_sync(0xffffffffu, pend_t, 0);                                                   \
      if (nxt_idx < num_tickets) {                                                                     \
        nxt_c = ordered ? decode_ordered(nxt_idx, args, order) : decode_item(nxt_idx, args);           \
        nxt_L = __ldg(args.context_lens + nxt_c.s);                                                    \
      }                                                                                                \
    } else if (claim_step == 2) {                                                                      \
      if (nxt_idx < num_tickets) {                                                                     \
        if (nxt_c.part < 0)                                                                            \
          nxt_c.part = (nxt_L > 0 && !context_len_invalid(nxt_L, args)) ? (nxt_L - 1) / args.partition_size : 0; \
        const int need_ = nxt_L <= 0 ? 0 : cmin(args.max_blocks_per_seq, nxt_L / bs + (nxt_L % bs != 0)); \
        const int32_t* row_ = args.block_tables + static_cast<size_t>(nxt_c.s) * args.max_blocks_per_seq; \
        _Pragma("unroll") for (int j_ = 0; j_ < kIdWindow; ++j_) {                                     \
          const int entry_ = ((nxt_c.part * boxes_per_part + j_ * 32 + lane) * kBoxTokens) / bs;       \
          nxt_ids[j_] = entry_ < need_ ? __ldg(row_ + entry_) : 0;                                     \
        }                                                                                              \
      }                                                                                                \
      have_next = true;                                                                                \
    }                                                                                                  \
    if (claim_step < 3) ++claim_step;                                                                  \
  } while (0)
    unsigned int pend_t = 0;
    int claim_step = 0;

    {
      unsigned int t0 = 0;
      if (lane == 0) t0 = atomicAdd(args.header + kWsWork, 1u);
      cur_idx = __shfl_sync(0xffffffffu, t0, 0);
      PA_PREPARE(cur_idx, cur_c, cur_L, cur_ids);
    }
    while (!aborted && cur_idx < num_tickets) {
      have_next = false;
      claim_step = 0;
      const ItemCoord c = cur_c;
      const int L = cur_L;
      const bool bad_len = context_len_invalid(L, args);
      const int n_parts = bad_len ? 1 : (L + args.partition_size - 1) / args.partition_size;
      const int kvh0 = c.hb * kHeadBlock;
      const int kv_here = cmin(kHeadBlock, args.num_kv_heads - kvh0);
      const int h_sub = c.sub * G;                       // first query head of the subgroup in a group
      const int heads = cmin(G, args.group - h_sub);     // query heads per kv head in this item
      if (c.part < cmax(n_parts, 1)) {
        if (L == 0 || bad_len) {
          // Empty context -> zeros; a context the launch cannot cover -> NaN and an error bit.
          if (bad_len && lane == 0) atomicOr(err, PA_DEVERR_CONTEXT_LEN);
          const float fill = bad_len ? __int_as_float(0x7fc00000) : 0.0f;
          for (int i = lane; i < kv_here * heads * D; i += 32) {
            const int kv = i / (heads * D), g = (i / D) % heads, e = i % D;
            const size_t h = static_cast<size_t>(kvh0 + kv) * args.group + h_sub + g;
            static_cast<QT*>(args.out)[(static_cast<size_t>(c.s) * args.num_heads + h) * D + e] = QT(fill);
          }
        } else {
          const int tok_begin = c.part * args.partition_size;
          const int tok_end = cmin(L, tok_begin + args.partition_size);
          const int n_stages = (tok_end - tok_begin + S::kTS - 1) / S::kTS;
          const int qb = local % kQueryBuffers;
          // Query rows of the item's heads, and the item description.
          bool ok = true;
          if (lane == 0) ok = mbar_wait(&qempty[qb], (static_cast<uint32_t>(local / kQueryBuffers) & 1u) ^ 1u, err);
          if (!__shfl_sync(0xffffffffu, ok, 0)) {
            aborted = true;
            break;
          }
          const uint32_t row_bytes = static_cast<uint32_t>(heads * D * sizeof(QT));
          if (lane == 0) {
            ItemInfo inf;
            inf.s = c.s;
            inf.part = c.part;
            inf.kvh0 = kvh0;
            inf.h_sub = h_sub;
            inf.heads = heads;
            inf.write_final = n_parts <= 1;
            inf.pad0 = static_cast<int>(cur_idx);
            inf.pad1 = 0;
#ifdef PA_TRACE
            unsigned long long* rec = args.trace + kTraceItemBase + 4ull * cur_idx;
            rec[0] = global_timer_ns();
            rec[2] = blockIdx.x;
            rec[3] = static_cast<unsigned long long>(tok_end - tok_begin);
#endif
            infos[qb] = inf;
            mbar_arrive_expect_tx(&qfull[qb], row_bytes * kv_here);
          }
          __syncwarp();
          // One bulk copy per query row (row r = kv * heads + g), into its padded slot.
          for (int r = lane; r < kv_here * heads; r += 32) {
            const int kv = r / heads, g = r - kv * heads;
            const QT* qsrc = static_cast<const QT*>(args.query) +
                             (static_cast<size_t>(c.s) * args.num_heads + (kvh0 + kv) * args.group + h_sub + g) * D;
            bulk_copy_g2s(smem + Lay::kQuery + qb * Lay::kQueryOne + (kv * G + g) * Lay::kQRow * sizeof(QT), qsrc,
                          static_cast<uint32_t>(D * sizeof(QT)), &qfull[qb]);
          }

          const int32_t* row = args.block_tables + static_cast<size_t>(c.s) * args.max_blocks_per_seq;
          // TMA ops of one stage are spread over lanes: lane = (box * 2 + kv) * kChunks + chunk.
          const int op_box = lane / (2 * S::kChunks);
          const int op_kv = (lane / S::kChunks) & 1;
          const int op_ch = lane % S::kChunks;
          const int claim_at = cmax(0, n_stages - kClaimAhead);
          for (int k = 0; k < n_stages; ++k) {
            if (k >= claim_at) PA_CLAIM_STEP();
            const int t0 = tok_begin + k * S::kTS;
            const int ntok = cmin(S::kTS, tok_end - t0);
            const int nbox = (ntok + kBoxTokens - 1) / kBoxTokens;
            // Block id of this lane's box: item-relative box rel sits in window register rel >> 5 of
            // lane rel & 31.
            const int rel = k * S::kGroups + (op_box < S::kGroups ? op_box : 0);
            int blk = 0;
#pragma unroll
            for (int j = 0; j < kIdWindow; ++j) {
              const int v = __shfl_sync(0xffffffffu, cur_ids[j], rel & 31);
              if ((rel >> 5) == j) blk = v;
            }
            const bool mine = op_box < nbox;  // this lane issues a TMA op for this stage
            if (rel >= kIdWindow * 32 && mine) blk = __ldg(row + (t0 + op_box * kBoxTokens) / bs);  // beyond the window
            bool bad = mine && (blk < 0 || blk >= args.num_blocks);
            if (bad) blk = args.num_blocks;  // out-of-range coordinate: TMA fills the box with zeros
            bad = __any_sync(0xffffffffu, bad);
            const int slot = issued % kStages;
            bool ok2 = true;
            if (lane == 0) ok2 = mbar_wait(&empty[slot], (static_cast<uint32_t>(issued / kStages) & 1u) ^ 1u, err);
            if (!__shfl_sync(0xffffffffu, ok2, 0)) {
              aborted = true;
              break;
            }
            // Block of box 0 and box 1 (their lanes' ids) for per-block scales; unloaded or invalid
            // boxes report block 0, a valid index whose scales meet only zero weights or NaN rows.
            int blk0 = 0, blk1 = 0;
            if constexpr (BS) {
              const int safe_blk = (mine && blk < args.num_blocks) ? blk : 0;
              blk0 = __shfl_sync(0xffffffffu, safe_blk, 0);
              blk1 = __shfl_sync(0xffffffffu, safe_blk, (2 * S::kChunks) & 31);
            }
            if (lane == 0) {
              StageMsg m;
              m.item = local;
              m.ntok = ntok;
              m.flags = (k == 0 ? kMsgFirst : 0) | (k == n_stages - 1 ? kMsgLast : 0) | (bad ? kMsgBadBlock : 0);
              m.flags |= blk0 << kMsgBlkShift;
              m.blk1 = S::kGroups > 1 ? blk1 : blk0;
              msgs[slot] = m;
              if (bad) atomicOr(err, PA_DEVERR_BLOCK_ID);
              mbar_arrive_expect_tx(&full[slot], static_cast<uint32_t>(nbox * 2 * S::kChunks * S::kBoxBytes));
            }
            __syncwarp();
            if (mine && lane < 2 * S::kChunks * S::kGroups) {
              uint8_t* dst = smem + Lay::kRing + slot * S::kStageBytes + op_kv * S::kTileBytes + op_ch * S::kChunkBytes +
                             op_box * S::kBoxBytes;
              tma_load_4d_hint(dst, op_kv ? &tmap_v : &tmap_k, &full[slot], op_ch * S::kChunkElems,
                               (t0 + op_box * kBoxTokens) % bs, kvh0, blk, kv_policy);
            }
            ++issued;
          }
          ++local;
        }
      }
      if (aborted) break;
      while (!have_next) PA_CLAIM_STEP();  // items with few stages (or none: empty, invalid, past the context)
      cur_idx = nxt_idx;
      cur_c = nxt_c;
      cur_L = nxt_L;
#pragma unroll
      for (int j = 0; j < kIdWindow; ++j) cur_ids[j] = nxt_ids[j];
    }
#undef PA_CLAIM_STEP
#undef PA_PREPARE
    // No work left: one terminating message.
    if (!aborted) {
      const int slot = issued % kStages;
      bool ok = true;
      if (lane == 0) ok = mbar_wait(&empty[slot], (static_cast<uint32_t>(issued / kStages) & 1u) ^ 1u, err);
      if (__shfl_sync(0xffffffffu, ok, 0) && lane == 0) {
        msgs[slot] = StageMsg{-1, 0, 0, 0};
        mbar_arrive(&full[slot]);
      }
      ++issued;
    }
    // Every issued copy has landed before the CTA may leave (bounded waits).
    if (lane == 0)
      for (int p = cmax(0, issued - kStages); p < issued; ++p)
        mbar_wait(&full[p % kStages], static_cast<uint32_t>(p / kStages) & 1u, err);
    __syncwarp();
  } else {
    // =============================== consumer warps ===============================
    const int cw = warp - 1;  // kv head within the item's head block
    const int ds = lane & (S::kNS - 1);
    const int tslot = lane >> S::kLog2NS;
    const int g_lane = ds >> (S::kLog2NS - S::kLog2G);                 // head owned after reduce-scatter
    const bool primary = (ds & ((S::kNS >> S::kLog2G) - 1)) == 0;      // first of the duplicate lanes
    const int dp = lane & (S::kLPT - 1);
    const int vslot = lane >> S::kLog2LPT;
    float* pw = reinterpret_cast<float*>(smem + Lay::kPbuf) + cw * S::kTS * G;
    float* aw = reinterpret_cast<float*>(smem + Lay::kAbuf) + cw * G;

    float2 qr[G][S::kNPL][4];
    float m_run = -INFINITY, l_run = 0.f;
    float2 acc[G][4];
    uint32_t qa[S::kKSteps][2];   // tensor-core path: query A fragments (rows g = lane/4), a0 and a2
    float o[S::kNBlocks][4];      // tensor-core path: output accumulator fragments
    bool poisoned = false;
    bool active = false;  // this warp's kv head exists in the current item
    float zitem = 0.f;    // per-head FP8: scale_log2 * k_scale of this warp's kv head for the item
    ItemInfo inf{};

    for (int j = 0;; ++j) {
      const int slot = j % kStages;
      if (!__all_sync(0xffffffffu, mbar_wait(&full[slot], static_cast<uint32_t>(j / kStages) & 1u, err))) break;
      const StageMsg m = msgs[slot];
      if (m.item < 0) break;
      if (m.flags & kMsgFirst) {
        // New item: load this head's query rows and reset the state.
        const int qb = m.item % kQueryBuffers;
        if (!__all_sync(0xffffffffu, mbar_wait(&qfull[qb], static_cast<uint32_t>(m.item / kQueryBuffers) & 1u, err)))
          break;
        inf = infos[qb];
        active = inf.kvh0 + cw < args.num_kv_heads;
        float qscale = args.scale_log2;
        if constexpr (EB == 1) {
          if (active && !BS) qscale *= args.k_scale[inf.kvh0 + cw];
        }
        zitem = qscale;
        const QT* qs = reinterpret_cast<const QT*>(smem + Lay::kQuery + qb * Lay::kQueryOne) + cw * G * Lay::kQRow;
        if constexpr (S::kMma) {
          const int g = lane >> 2, t4 = lane & 3;
          const bool row_ok = active && g < inf.heads;
#pragma unroll
          for (int ks = 0; ks < S::kKSteps; ++ks) {
            if constexpr (EB == 2) {
              qa[ks][0] = row_ok ? *reinterpret_cast<const uint32_t*>(qs + g * Lay::kQRow + ks * 16 + 2 * t4) : 0u;
              qa[ks][1] = row_ok ? *reinterpret_cast<const uint32_t*>(qs + g * Lay::kQRow + ks * 16 + 8 + 2 * t4) : 0u;
            } else {
              // FP8 K fragments come from ldmatrix over byte rows (see the stage code): step ks holds
              // d = 16*ks + 4*t4 + {0,1} in b0 and + {2,3} in b1, so the query uses the same order.
              // One 8-byte load per lane (the four values of this step), conflict-free with the padded rows.
              if (row_ok) {
                const uint2 raw = *reinterpret_cast<const uint2*>(qs + g * Lay::kQRow + ks * 16 + 4 * t4);
                const QT* qrow = reinterpret_cast<const QT*>(&raw);
                qa[ks][0] = pack2<__half>(to_f32(qrow[0]), to_f32(qrow[1]));
                qa[ks][1] = pack2<__half>(to_f32(qrow[2]), to_f32(qrow[3]));
              } else {
                qa[ks][0] = qa[ks][1] = 0u;
              }
            }
          }
#pragma unroll
          for (int nb = 0; nb < S::kNBlocks; ++nb) o[nb][0] = o[nb][1] = o[nb][2] = o[nb][3] = 0.f;
        } else
#pragma unroll
        for (int g = 0; g < G; ++g) {
#pragma unroll
          for (int jj = 0; jj < S::kNPL; ++jj) {
            const int pc = qk_piece<S, EB>(jj, ds, tslot);
            if (active && g < inf.heads) {
              const uint4 raw = *reinterpret_cast<const uint4*>(qs + g * Lay::kQRow + pc * 8);
              const QT* e = reinterpret_cast<const QT*>(&raw);
#pragma unroll
              for (int k = 0; k < 4; ++k)
                qr[g][jj][k] = make_float2(to_f32(e[2 * k]) * qscale, to_f32(e[2 * k + 1]) * qscale);
            } else {
#pragma unroll
              for (int k = 0; k < 4; ++k) qr[g][jj][k] = make_float2(0.f, 0.f);
            }
          }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&qempty[qb]);
        m_run = -INFINITY;
        l_run = 0.f;
        poisoned = false;
#pragma unroll
        for (int g = 0; g < G; ++g)
#pragma unroll
          for (int k = 0; k < 4; ++k) acc[g][k] = make_float2(0.f, 0.f);
      }
      poisoned |= (m.flags & kMsgBadBlock) != 0;

      if constexpr (S::kMma) {
       if (active) {
        // ---------------- tensor-core stage ----------------
        constexpr int NG = S::kGroups;
        const int nvalid = m.ntok;
        const uint32_t kbase = smem_u32(smem + Lay::kRing + slot * S::kStageBytes);
        const uint32_t vbase = kbase + S::kTileBytes;
        const int t4 = lane & 3;
        // ldmatrix row addresses: lane i points at token row i % 8 of this head (in box gr), unit i / 8.
        // Two accumulators per box (even and odd k-steps) halve the dependent MMA chain; summed after.
        float sacc[NG][4], sacc2[NG][4];
#pragma unroll
        for (int gr = 0; gr < NG; ++gr) {
          sacc[gr][0] = sacc[gr][1] = sacc[gr][2] = sacc[gr][3] = 0.f;
          sacc2[gr][0] = sacc2[gr][1] = sacc2[gr][2] = sacc2[gr][3] = 0.f;
          const int lrow = tile_row(cw, gr * kBoxTokens + (lane & 7));
          if constexpr (EB == 2) {
#pragma unroll
            for (int q4 = 0; q4 < S::kKSteps / 2; ++q4) {
              uint32_t kb[4];
              ldmatrix_x4(kbase + piece_offset<S>(lrow, q4 * 4 + (lane >> 3)), kb);
              const uint32_t a0[4] = {qa[2 * q4][0], 0u, qa[2 * q4][1], 0u};
              mma_16816<MmaT>(sacc[gr], a0, kb[0], kb[1]);
              const uint32_t a1[4] = {qa[2 * q4 + 1][0], 0u, qa[2 * q4 + 1][1], 0u};
              mma_16816<MmaT>(sacc2[gr], a1, kb[2], kb[3]);
            }
          } else {
            // FP8 rows are 128 bytes (one swizzle chunk, 16-byte unit u = 16 values of d). ldmatrix
            // over the byte rows gives lane (g, t4) the 4 bytes d = 16u + 4*t4 + {0..3} of token g; the
            // low pair becomes b0 and the high pair b1 after widening to f16.
            static_assert(D == 128, "FP8 caches need head_size 128");
            const uint32_t kaddr = kbase + lrow * 128;
#pragma unroll
            for (int q4 = 0; q4 < S::kKSteps / 4; ++q4) {
              uint32_t kb[4];
              ldmatrix_x4(kaddr + (((q4 * 4 + (lane >> 3)) ^ (lane & 7)) << 4), kb);
#pragma unroll
              for (int j4 = 0; j4 < 4; ++j4) {
                const uint32_t b0 = e4m3x2_to_f16x2(static_cast<uint16_t>(kb[j4] & 0xffffu));
                const uint32_t b1 = e4m3x2_to_f16x2(static_cast<uint16_t>(kb[j4] >> 16));
                const uint32_t a[4] = {qa[q4 * 4 + j4][0], 0u, qa[q4 * 4 + j4][1], 0u};
                mma_16816<MmaT>((j4 & 1) ? sacc2[gr] : sacc[gr], a, b0, b1);
              }
            }
          }
#pragma unroll
          for (int i = 0; i < 4; ++i) sacc[gr][i] += sacc2[gr][i];
        }
        // Scores of query head lane/4 for tokens 8*gr + 2*t4 and 8*gr + 2*t4 + 1. FP8 scales: K's scales
        // the scores of its box, V's the weights that enter P V of its box (per-block scales), or the
        // output (per-head scales).
        float zs[NG], vsb[NG];
#pragma unroll
        for (int gr = 0; gr < NG; ++gr) {
          zs[gr] = zitem;
          vsb[gr] = 1.0f;
          if constexpr (BS) {
            {
              const int blk = gr == 0 ? (m.flags >> kMsgBlkShift) : m.blk1;
              const int si = blk * args.scale_block_stride + inf.kvh0 + cw;
              zs[gr] = args.scale_log2 * __ldg(args.k_scale + si);
              vsb[gr] = __ldg(args.v_scale + si);
            }
          }
        }
        float sv[NG][2];
        float cm = -INFINITY;
#pragma unroll
        for (int gr = 0; gr < NG; ++gr) {
          sv[gr][0] = gr * kBoxTokens + 2 * t4 < nvalid ? sacc[gr][0] * zs[gr] : -INFINITY;
          sv[gr][1] = gr * kBoxTokens + 2 * t4 + 1 < nvalid ? sacc[gr][1] * zs[gr] : -INFINITY;
          cm = fmaxf(cm, fmaxf(sv[gr][0], sv[gr][1]));
        }
        cm = fmaxf(cm, __shfl_xor_sync(0xffffffffu, cm, 1));
        cm = fmaxf(cm, __shfl_xor_sync(0xffffffffu, cm, 2));
        const float m_new = fmaxf(m_run, cm);
        const float alpha = fast_exp2(m_run - m_new);
        uint32_t pfrag[NG];
        float psum = 0.f;
#pragma unroll
        for (int gr = 0; gr < NG; ++gr) {
          const float p0 = fast_exp2(sv[gr][0] - m_new), p1 = fast_exp2(sv[gr][1] - m_new);
          pfrag[gr] = pack2<MmaT>(p0, p1);
          // The sum uses the rounded weights that enter P V, so the weights of the output sum to one.
          const float2 pr = unpack2<MmaT>(pfrag[gr]);
          psum += pr.x + pr.y;
          // Per-block V scales ride on the weights of their box (the sum keeps the unscaled ones).
          if constexpr (BS) pfrag[gr] = pack2<MmaT>(pr.x * vsb[gr], pr.y * vsb[gr]);
        }
        l_run = l_run * alpha + psum;
        m_run = m_new;
#pragma unroll
        for (int nb = 0; nb < S::kNBlocks; ++nb) {
          o[nb][0] *= alpha;
          o[nb][1] *= alpha;
        }
        // V rows of tokens past the valid ones may hold anything (even NaN): zero their halves of the
        // B fragments (low half = token 2*t4, high half = token 2*t4 + 1 of each box).
        uint32_t vmask[NG];
#pragma unroll
        for (int gr = 0; gr < NG; ++gr)
          vmask[gr] = (gr * kBoxTokens + 2 * t4 < nvalid ? 0x0000ffffu : 0u) |
                      (gr * kBoxTokens + 2 * t4 + 1 < nvalid ? 0xffff0000u : 0u);
        // A full stage (every stage but an item's last) has no invalid rows: its fragments skip the masks.
        auto pv = [&](auto masked_tag) {
          constexpr bool kMasked = decltype(masked_tag)::value;
          if constexpr (EB == 2) {
            static_assert(NG == 1, "16-bit caches use one box per stage");
            const int lrow = tile_row(cw, lane & 7);
#pragma unroll
            for (int q4 = 0; q4 < S::kNBlocks / 4; ++q4) {
              uint32_t vb[4];
              ldmatrix_x4_trans(vbase + piece_offset<S>(lrow, q4 * 4 + (lane >> 3)), vb);
#pragma unroll
              for (int j4 = 0; j4 < 4; ++j4)
                mma_1688<MmaT>(o[q4 * 4 + j4], pfrag[0], 0u, kMasked ? (vb[j4] & vmask[0]) : vb[j4]);
            }
          } else {
            // ldmatrix.trans over the byte rows of box gr gives lane (g, t4) the bytes
            // [V[2t4][16u+2g], V[2t4][16u+2g+1], V[2t4+1][16u+2g], V[2t4+1][16u+2g+1]]; one byte permute
            // splits them into the even-d fragment (block 2u: d = 16u + 2g) and the odd-d fragment
            // (block 2u + 1: d = 16u + 2g + 1). The two boxes are the two k-halves of an m16n8k16 step.
            static_assert(NG == 2, "FP8 caches use two boxes per stage");
            const uint32_t a[4] = {pfrag[0], 0u, pfrag[1], 0u};
            const uint32_t vaddr0 = vbase + tile_row(cw, lane & 7) * 128;
            const uint32_t vaddr1 = vbase + tile_row(cw, kBoxTokens + (lane & 7)) * 128;
#pragma unroll
            for (int q4 = 0; q4 < S::kNBlocks / 8; ++q4) {
              const uint32_t off = ((q4 * 4 + (lane >> 3)) ^ (lane & 7)) << 4;
              uint32_t vb0[4], vb1[4];
              ldmatrix_x4_trans(vaddr0 + off, vb0);
              ldmatrix_x4_trans(vaddr1 + off, vb1);
#pragma unroll
              for (int j4 = 0; j4 < 4; ++j4) {
                const int u = q4 * 4 + j4;
                uint32_t ev0 = e4m3x2_to_f16x2(static_cast<uint16_t>(__byte_perm(vb0[j4], 0u, 0x4420u)));
                uint32_t ev1 = e4m3x2_to_f16x2(static_cast<uint16_t>(__byte_perm(vb1[j4], 0u, 0x4420u)));
                uint32_t od0 = e4m3x2_to_f16x2(static_cast<uint16_t>(__byte_perm(vb0[j4], 0u, 0x4431u)));
                uint32_t od1 = e4m3x2_to_f16x2(static_cast<uint16_t>(__byte_perm(vb1[j4], 0u, 0x4431u)));
                if constexpr (kMasked) {
                  ev0 &= vmask[0];
                  ev1 &= vmask[1];
                  od0 &= vmask[0];
                  od1 &= vmask[1];
                }
                mma_16816<MmaT>(o[2 * u], a, ev0, ev1);
                mma_16816<MmaT>(o[2 * u + 1], a, od0, od1);
              }
            }
          }
        };
        if (nvalid == S::kTS) pv(std::false_type{}); else pv(std::true_type{});
       }
      } else if (active) {
        const int nvalid = m.ntok;
        const uint8_t* ktile = smem + Lay::kRing + slot * S::kStageBytes;
        const uint8_t* vtile = ktile + S::kTileBytes;
        // Per-block FP8 scales of the stage's two 8-token boxes (K scales the scores, V the weights).
        float ksb[2] = {1.f, 1.f}, vsb2[2] = {1.f, 1.f};
        if constexpr (BS) {
#pragma unroll
          for (int bx = 0; bx < 2; ++bx) {
            const int blk = bx == 0 ? (m.flags >> kMsgBlkShift) : m.blk1;
            const int si = blk * args.scale_block_stride + inf.kvh0 + cw;
            ksb[bx] = __ldg(args.k_scale + si);
            vsb2[bx] = __ldg(args.v_scale + si);
          }
        }
        // ---- scores ----
        float sc[S::kIters];
#pragma unroll
        for (int it = 0; it < S::kIters; ++it) {
          const int t = it * S::kTPI + tslot;
          float2 pacc[G];
#pragma unroll
          for (int g = 0; g < G; ++g) pacc[g] = make_float2(0.f, 0.f);
#pragma unroll
          for (int jj = 0; jj < S::kNPL; ++jj) {
            const int pc = qk_piece<S, EB>(jj, ds, tslot);
            const Piece kp = *reinterpret_cast<const Piece*>(ktile + piece_offset<S>(tile_row(cw, t), pc));
            float2 kf[4];
            Elem<KVT>::to_float(kp, kf);
#pragma unroll
            for (int g = 0; g < G; ++g)
#pragma unroll
              for (int k = 0; k < 4; ++k) pacc[g] = ffma2(qr[g][jj][k], kf[k], pacc[g]);
          }
          float v[G];
#pragma unroll
          for (int g = 0; g < G; ++g) v[g] = pacc[g].x + pacc[g].y;
          float z = reduce_scatter<G, S::kLog2NS>(v, lane);
          if constexpr (BS) z *= ksb[t / kBoxTokens];
          sc[it] = t < nvalid ? z : -INFINITY;
        }
        // ---- online softmax (per head g_lane) ----
        float cm = sc[0];
#pragma unroll
        for (int it = 1; it < S::kIters; ++it) cm = fmaxf(cm, sc[it]);
#pragma unroll
        for (int b = S::kTsShift; b < 5; ++b) cm = fmaxf(cm, __shfl_xor_sync(0xffffffffu, cm, 1 << b));
        const float m_new = fmaxf(m_run, cm);
        const float alpha = fast_exp2(m_run - m_new);
        float lsum = 0.f;
#pragma unroll
        for (int it = 0; it < S::kIters; ++it) {
          const float p = fast_exp2(sc[it] - m_new);
          lsum += p;
          if (primary) pw[(it * S::kTPI + tslot) * G + g_lane] = p;
        }
        l_run = l_run * alpha + lsum;
        m_run = m_new;
        if (primary && tslot == 0) aw[g_lane] = alpha;
        __syncwarp();
        // ---- P V ----
#pragma unroll
        for (int g = 0; g < G; ++g) {
          const float a = aw[g];
#pragma unroll
          for (int k = 0; k < 4; ++k) acc[g][k] = make_float2(acc[g][k].x * a, acc[g][k].y * a);
        }
#pragma unroll
        for (int t0 = 0; t0 < S::kTS; t0 += S::kTPV) {
          const int t = t0 + vslot;
          if (t < nvalid) {
            const Piece vp = *reinterpret_cast<const Piece*>(vtile + piece_offset<S>(tile_row(cw, t), dp));
            float2 vf[4];
            Elem<KVT>::to_float(vp, vf);
            float p[G];
            if constexpr (G >= 4) {
#pragma unroll
              for (int g = 0; g < G; g += 4) {
                const float4 p4 = *reinterpret_cast<const float4*>(pw + t * G + g);
                p[g] = p4.x; p[g + 1] = p4.y; p[g + 2] = p4.z; p[g + 3] = p4.w;
              }
            } else {
#pragma unroll
              for (int g = 0; g < G; ++g) p[g] = pw[t * G + g];
            }
            if constexpr (BS) {
#pragma unroll
              for (int g = 0; g < G; ++g) p[g] *= vsb2[t / kBoxTokens];
            }
#pragma unroll
            for (int g = 0; g < G; ++g) {
              const float2 pp = make_float2(p[g], p[g]);
#pragma unroll
              for (int k = 0; k < 4; ++k) acc[g][k] = ffma2(pp, vf[k], acc[g][k]);
            }
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[slot]);

#ifdef PA_TRACE
      if ((m.flags & kMsgLast) && cw == 0 && lane == 0)
        args.trace[kTraceItemBase + 4ull * static_cast<unsigned int>(inf.pad0) + 1] = global_timer_ns();
#endif
      if constexpr (S::kMma) {
       if ((m.flags & kMsgLast) && active) {
        // ---- end of the item (tensor-core path): row g = lane/4 is query head g ----
        float l_tot = l_run + __shfl_xor_sync(0xffffffffu, l_run, 1);
        l_tot += __shfl_xor_sync(0xffffffffu, l_tot, 2);
        const int g = lane >> 2, t4 = lane & 3;
        if (g < inf.heads) {
          float r = ((EB == 1 && !BS) ? args.v_scale[inf.kvh0 + cw] : 1.0f) / l_tot;
          if (poisoned) r = __int_as_float(0x7fc00000);
          const int h = (inf.kvh0 + cw) * args.group + inf.h_sub + g;
          const size_t rowi = (static_cast<size_t>(inf.s) * args.num_heads + h) * args.num_partitions + inf.part;
          if (inf.write_final) {
            QT* out = static_cast<QT*>(args.out) + (static_cast<size_t>(inf.s) * args.num_heads + h) * D;
            if constexpr (EB == 2) {
#pragma unroll
              for (int nb = 0; nb < S::kNBlocks; ++nb)
                *reinterpret_cast<uint32_t*>(out + nb * 8 + 2 * t4) = pack2<QT>(o[nb][0] * r, o[nb][1] * r);
            } else {
              // Blocks 2u (even d) and 2u + 1 (odd d) together hold d = 16u + 4*t4 + {0, 1, 2, 3}.
#pragma unroll
              for (int u = 0; u < S::kNBlocks / 2; ++u)
                *reinterpret_cast<uint2*>(out + u * 16 + 4 * t4) =
                    pack4<QT>(o[2 * u][0] * r, o[2 * u + 1][0] * r, o[2 * u][1] * r, o[2 * u + 1][1] * r);
            }
          } else {
            float* po = args.part_o + rowi * D;
            if constexpr (EB == 2) {
#pragma unroll
              for (int nb = 0; nb < S::kNBlocks; ++nb)
                *reinterpret_cast<float2*>(po + nb * 8 + 2 * t4) = make_float2(o[nb][0] * r, o[nb][1] * r);
            } else {
#pragma unroll
              for (int u = 0; u < S::kNBlocks / 2; ++u)
                *reinterpret_cast<float4*>(po + u * 16 + 4 * t4) =
                    make_float4(o[2 * u][0] * r, o[2 * u + 1][0] * r, o[2 * u][1] * r, o[2 * u + 1][1] * r);
            }
            if (t4 == 0) {
              args.part_m[rowi] = m_run;
              args.part_l[rowi] = l_tot;
            }
          }
        }
       }
      } else if ((m.flags & kMsgLast) && active) {
        // ---- end of the item: normalise and write this kv head's query heads ----
        float l_tot = l_run;
#pragma unroll
        for (int b = S::kTsShift; b < 5; ++b) l_tot += __shfl_xor_sync(0xffffffffu, l_tot, 1 << b);
#pragma unroll
        for (int b = S::kLog2LPT; b < 5; ++b) {
#pragma unroll
          for (int g = 0; g < G; ++g)
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              acc[g][k].x += __shfl_xor_sync(0xffffffffu, acc[g][k].x, 1 << b);
              acc[g][k].y += __shfl_xor_sync(0xffffffffu, acc[g][k].y, 1 << b);
            }
        }
        // l and m of head g live on the primary lanes with tslot 0 (lane g << (log2 NS - log2 G)).
        const float vscale = (EB == 1 && !BS) ? args.v_scale[inf.kvh0 + cw] : 1.0f;
#pragma unroll
        for (int g = 0; g < G; ++g) {
          const int src = g << (S::kLog2NS - S::kLog2G);
          const float lg = __shfl_sync(0xffffffffu, l_tot, src);
          const float mg = __shfl_sync(0xffffffffu, m_run, src);
          if (g < inf.heads && vslot == 0) {
            float r = vscale / lg;
            if (poisoned) r = __int_as_float(0x7fc00000);
            const int h = (inf.kvh0 + cw) * args.group + inf.h_sub + g;
            if (inf.write_final) {
              QT* out = static_cast<QT*>(args.out) + (static_cast<size_t>(inf.s) * args.num_heads + h) * D + dp * 8;
              *reinterpret_cast<uint2*>(out) = pack4<QT>(acc[g][0].x * r, acc[g][0].y * r, acc[g][1].x * r, acc[g][1].y * r);
              *reinterpret_cast<uint2*>(out + 4) = pack4<QT>(acc[g][2].x * r, acc[g][2].y * r, acc[g][3].x * r, acc[g][3].y * r);
            } else {
              const size_t rowi = (static_cast<size_t>(inf.s) * args.num_heads + h) * args.num_partitions + inf.part;
              float* po = args.part_o + rowi * D + dp * 8;
              *reinterpret_cast<float4*>(po) = make_float4(acc[g][0].x * r, acc[g][0].y * r, acc[g][1].x * r, acc[g][1].y * r);
              *reinterpret_cast<float4*>(po + 4) = make_float4(acc[g][2].x * r, acc[g][2].y * r, acc[g][3].x * r, acc[g][3].y * r);
              if (dp == 0) {
                args.part_m[rowi] = mg;
                args.part_l[rowi] = lg;
              }
            }
          }
        }
      }
    }
  }

  // The last CTA to finish resets the work counter for the next launch on this workspace.
  __syncthreads();
#ifdef PA_TRACE
  if (threadIdx.x == 0 && blockIdx.x < kTraceMaxCtas) args.trace[kTraceCtaBase + 4 * blockIdx.x + 1] = global_timer_ns();
#endif
  if (threadIdx.x == 0) {
    __threadfence();
    const unsigned int done = atomicAdd(args.header + kWsDone, 1u);
    if (done == gridDim.x - 1) {
      atomicExch(args.header + kWsWork, 0u);
      atomicExch(args.header + kWsDone, 0u);
    }
  }
}

// Split-K merge of partitions: out = sum_p w_p o_p / sum_p w_p with w_p = l_p 2^(m_p - max m).
// One warp per (sequence, query head): lanes hold 4 (or 2) consecutive elements of the row and walk
// the partitions; the partition statistics are read once per lane group. Sequences with one
// partition (or an empty or invalid context) were finished by the main kernel.
constexpr int kReduceWarps = 4;
constexpr int kReduceSplitAbove = 16;  // more partitions than this: one CTA per row, its warps split them

// Merges partitions p0 .. p1-1 of one row into (wsum, acc), in partition order: lane i computes the
// weight of partition q + i once (one load of its m and l per warp instead of per lane) and the weights
// reach every lane by shuffle.
template <int D>
__device__ __forceinline__ void merge_range(const AttnArgs& a, size_t base, int p0, int p1, float M, int lane,
                                            float& wsum, float (&acc)[D / 32]) {
  constexpr int kPer = D / 32;
  const float* po = a.part_o + base * D + lane * kPer;
  for (int q = p0; q < p1; q += 32) {
    const int p = q + lane;
    const float w_lane = p < p1 ? a.part_l[base + p] * fast_exp2(a.part_m[base + p] - M) : 0.f;
    const int cnt = min(32, p1 - q);
#pragma unroll 8
    for (int i = 0; i < cnt; ++i) {
      const float w = __shfl_sync(0xffffffffu, w_lane, i);
      wsum += w;
      if constexpr (kPer == 4) {
        const float4 v = *reinterpret_cast<const float4*>(po + static_cast<size_t>(q + i) * D);
        acc[0] += w * v.x; acc[1] += w * v.y; acc[2] += w * v.z; acc[3] += w * v.w;
      } else {
        const float2 v = *reinterpret_cast<const float2*>(po + static_cast<size_t>(q + i) * D);
        acc[0] += w * v.x; acc[1] += w * v.y;
      }
    }
  }
}

// Split-K merge of partitions: out = sum_p w_p o_p / sum_p w_p with w_p = l_p 2^(m_p - max m).
// SPLIT = false: one warp per (sequence, query head), lanes holding 4 (or 2) consecutive elements of the
// row, walking the partitions. SPLIT = true (many partitions): one CTA per row; each of its warps
// merges a quarter of the partitions against their own max, and warp 0 brings the four results to the
// row's max and adds them in warp order. Sequences with one partition (or an empty or invalid context)
// were finished by the main kernel.
// MAXP (SPLIT = false): a bound on the partition count the launch was sized for (4, 8 or 16), so that a
// row's preloaded values take no more registers than it needs and more warps stay resident.
template <typename QT, int D, bool SPLIT, int MAXP = kReduceSplitAbove>
__global__ void __launch_bounds__(kReduceWarps * 32)
paged_attention_reduce(const AttnArgs args) {
  constexpr int kPer = D / 32;  // elements per lane: 4 for d = 128, 2 for d = 64
  grid_dependency_wait();
  grid_dependents_launch();
#ifdef PA_TRACE
  if (threadIdx.x == 0) atomicMax(args.trace, ~global_timer_ns());
  struct TraceEnd {
    unsigned long long* t;
    __device__ ~TraceEnd() {  // thread 0's exit stands for its CTA's
      if (threadIdx.x == 0) atomicMax(t + 1, global_timer_ns());
    }
  } trace_end{args.trace};
#endif
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const long row = SPLIT ? static_cast<long>(blockIdx.x) : static_cast<long>(blockIdx.x) * kReduceWarps + warp;
  if (row >= static_cast<long>(args.num_seqs) * args.num_heads) return;
  const int s = static_cast<int>(row / args.num_heads);
  const int L = args.context_lens[s];
  const int PS = args.partition_size;
  if (L <= 0 || context_len_invalid(L, args)) return;
  const int n_parts = (L + PS - 1) / PS;
  if (n_parts <= 1) return;
  const size_t base = static_cast<size_t>(row) * args.num_partitions;
  float wsum = 0.f;
  float acc[kPer];
#pragma unroll
  for (int k = 0; k < kPer; ++k) acc[k] = 0.f;
  if constexpr (!SPLIT) {
    // At most MAXP partitions: every load of the row (lane p's m and l, and each lane's
    // elements of every partition) is issued before any result is needed, so the row costs one
    // load round trip. Same order and arithmetic as merge_range.
    float m_lane = -INFINITY, l_lane = 0.f;
    if (lane < n_parts) {
      m_lane = args.part_m[base + lane];
      l_lane = args.part_l[base + lane];
    }
    const float* po = args.part_o + base * D + lane * kPer;
    float ov[MAXP][kPer];
#pragma unroll
    for (int p = 0; p < MAXP; ++p) {
      if (p < n_parts) {
        if constexpr (kPer == 4) {
          const float4 v = *reinterpret_cast<const float4*>(po + static_cast<size_t>(p) * D);
          ov[p][0] = v.x; ov[p][1] = v.y; ov[p][2] = v.z; ov[p][3] = v.w;
        } else {
          const float2 v = *reinterpret_cast<const float2*>(po + static_cast<size_t>(p) * D);
          ov[p][0] = v.x; ov[p][1] = v.y;
        }
      }
    }
    float M = m_lane;
#pragma unroll
    for (int b = 16; b > 0; b >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, b));
    const float w_lane = lane < n_parts ? l_lane * fast_exp2(m_lane - M) : 0.f;
#pragma unroll
    for (int p = 0; p < MAXP; ++p) {
      if (p < n_parts) {
        const float w = __shfl_sync(0xffffffffu, w_lane, p);
        wsum += w;
#pragma unroll
        for (int k = 0; k < kPer; ++k) acc[k] += w * ov[p][k];
      }
    }
  } else {
    const int chunk = (n_parts + kReduceWarps - 1) / kReduceWarps;
    const int p0 = min(n_parts, warp * chunk), p1 = min(n_parts, (warp + 1) * chunk);
    float Mw;  // the max this warp's weights are taken against
    if (chunk <= kReduceSplitAbove) {
      // One load round trip, as above, over this warp's partitions and against their own max; the
      // warps' results are brought to the row's max when they are added.
      float m_lane = -INFINITY, l_lane = 0.f;
      if (p0 + lane < p1) {
        m_lane = args.part_m[base + p0 + lane];
        l_lane = args.part_l[base + p0 + lane];
      }
      const float* po = args.part_o + (base + p0) * D + lane * kPer;
      float ov[kReduceSplitAbove][kPer];
#pragma unroll
      for (int p = 0; p < kReduceSplitAbove; ++p) {
        if (p0 + p < p1) {
          if constexpr (kPer == 4) {
            const float4 v = *reinterpret_cast<const float4*>(po + static_cast<size_t>(p) * D);
            ov[p][0] = v.x; ov[p][1] = v.y; ov[p][2] = v.z; ov[p][3] = v.w;
          } else {
            const float2 v = *reinterpret_cast<const float2*>(po + static_cast<size_t>(p) * D);
            ov[p][0] = v.x; ov[p][1] = v.y;
          }
        }
      }
      Mw = m_lane;
#pragma unroll
      for (int b = 16; b > 0; b >>= 1) Mw = fmaxf(Mw, __shfl_xor_sync(0xffffffffu, Mw, b));
      const float w_lane = p0 + lane < p1 ? l_lane * fast_exp2(m_lane - Mw) : 0.f;
#pragma unroll
      for (int p = 0; p < kReduceSplitAbove; ++p) {
        if (p0 + p < p1) {
          const float w = __shfl_sync(0xffffffffu, w_lane, p);
          wsum += w;
#pragma unroll
          for (int k = 0; k < kPer; ++k) acc[k] += w * ov[p][k];
        }
      }
    } else {
      Mw = -INFINITY;
      for (int p = lane; p < n_parts; p += 32) Mw = fmaxf(Mw, args.part_m[base + p]);
#pragma unroll
      for (int b = 16; b > 0; b >>= 1) Mw = fmaxf(Mw, __shfl_xor_sync(0xffffffffu, Mw, b));
      merge_range<D>(args, base, p0, p1, Mw, lane, wsum, acc);
    }
    __shared__ float part_acc[kReduceWarps][D];
    __shared__ float part_wsum[kReduceWarps];
    __shared__ float part_max[kReduceWarps];
#pragma unroll
    for (int k = 0; k < kPer; ++k) part_acc[warp][lane * kPer + k] = acc[k];
    if (lane == 0) {
      part_wsum[warp] = wsum;
      part_max[warp] = Mw;
    }
    __syncthreads();
    if (warp != 0) return;
    float M = part_max[0];
#pragma unroll
    for (int w = 1; w < kReduceWarps; ++w) M = fmaxf(M, part_max[w]);
    wsum = 0.f;
#pragma unroll
    for (int k = 0; k < kPer; ++k) acc[k] = 0.f;
#pragma unroll
    for (int w = 0; w < kReduceWarps; ++w) {
      // A warp without partitions has max -inf and adds nothing (factor 0).
      const float f = part_wsum[w] > 0.f ? fast_exp2(part_max[w] - M) : 0.f;
      wsum += f * part_wsum[w];
#pragma unroll
      for (int k = 0; k < kPer; ++k) acc[k] += f * part_acc[w][lane * kPer + k];
    }
  }
  const float r = 1.0f / wsum;
  QT* out = static_cast<QT*>(args.out) + static_cast<size_t>(row) * D + lane * kPer;
  if constexpr (kPer == 4) {
    *reinterpret_cast<uint2*>(out) = pack4<QT>(acc[0] * r, acc[1] * r, acc[2] * r, acc[3] * r);
  } else {
    *reinterpret_cast<uint32_t*>(out) = pack2<QT>(acc[0] * r, acc[1] * r);
  }
}

}  // namespace pa
