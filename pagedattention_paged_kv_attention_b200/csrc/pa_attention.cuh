// pa_attention.cuh -- paged decode attention kernels for sm_100a.
//
// What is computed (tutorial page "企业官网建设流程全解析", sec. 2.2 "分块注意力计算过程": the formula
// softmax(QK^T/sqrt(d))V, normalised over the whole context -- NOT that section's per-block loop, whose
// per-block softmaxes are summed without renormalisation): for sequence s and query head h,
//   out[s][h] = sum_t exp(z_t - m) v_t / sum_t exp(z_t - m),  z_t = scale * q[s][h] . k_t,
// where token t is found through the block table (sec. 2.1 "基本数据结构设计"; page "PagedAttention 与
// 连续批处理：LLM Serving 的底层架构拆解", section "PagedAttention：把显存做成虚拟内存").
//
// Design (B200): one CTA per (kv head [x head sub-group], sequence, context partition).
//  * Warp 4 is a producer: for each 64-token stage it reads the stage's block ids from the block
//    table and issues one 4-D TMA tile load per (block, 128-byte chunk) for K and for V into a ring of
//    shared-memory stages (128-byte swizzle), completion counted on an mbarrier. The page-table walk
//    is therefore a TMA coordinate, and the bytes in flight per SM are the ring depth.
//  * Warps 0-3 are consumers. Warp w owns stages w, w+4, ... and keeps its own fp32 online-softmax
//    state (running max m, running sum l, accumulator acc[G][d]) for the G query heads that share
//    this kv head (grouped-query heads are batched: each K/V element is read once for all G heads).
//      QK: NS lanes cooperate on one token (each holds 1/NS of d and all G query rows in registers,
//          pre-scaled by scale*log2(e)); a butterfly reduce-scatter leaves each lane with the full
//          score of one head.
//      softmax: stage max per head across lanes, rescale factor alpha = 2^(m_old - m_new),
//          p = 2^(z - m_new) written to a per-warp shared buffer.
//      PV: D/8 lanes cover one V row (8 elements each); every lane accumulates all G heads.
//    Packed f32x2 FMAs are used throughout; inputs are widened to fp32 once per element.
//  * At the end the four warp states are merged through shared memory (log-sum-exp merge). With one
//    partition the CTA writes the normalised output; otherwise it writes (m, l, acc/l) partials and
//    the reduce kernel merges partitions the same way.
// Arithmetic order depends only on logical token positions, never on physical block ids, so outputs
// are bitwise invariant to block placement and deterministic run to run.
#pragma once

#include "pa_device.cuh"

namespace pa {

constexpr int kStageTokens = 64;
constexpr int kConsumerWarps = 4;
constexpr int kThreads = (kConsumerWarps + 1) * 32;
constexpr int kMaxStages = 8;
constexpr float kLog2e = 1.4426950408889634f;

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
  unsigned int* error_word;
  int max_blocks_per_seq;
  int num_seqs;
  int num_heads;
  int num_kv_heads;
  int group;                    // num_heads / num_kv_heads
  int subgroups;                // CTAs per kv head (ceil(group / G))
  int block_size;
  int num_blocks;
  int partition_size;           // tokens per partition, multiple of kStageTokens
  int num_partitions;
  int num_stages;               // ring depth, 2..kMaxStages
  float scale_log2;             // softmax scale * log2(e)
};

__host__ __device__ constexpr int ilog2(int x) { return x <= 1 ? 0 : 1 + ilog2(x / 2); }
__host__ __device__ constexpr int cmin(int a, int b) { return a < b ? a : b; }

template <int D, int G, int EB>
struct Shape {
  static constexpr int kRowBytes = D * EB;
  static constexpr int kChunks = kRowBytes / 128;        // 128-byte swizzle chunks per row
  static constexpr int kChunkElems = 128 / EB;
  static constexpr int kPieceBytes = 8 * EB;             // one piece = 8 elements
  static constexpr int kPiecesPerRow = D / 8;
  // QK mapping: NS lanes per token.
  static constexpr int kNS = cmin(D / 8, G <= 2 ? 4 : 2 * G);
  static constexpr int kLog2NS = ilog2(kNS);
  static constexpr int kLog2G = ilog2(G);
  static constexpr int kTPI = 32 / kNS;                  // tokens per QK step
  static constexpr int kLog2TPI = ilog2(kTPI);
  static constexpr int kNPL = kPiecesPerRow / kNS;       // pieces per lane
  static constexpr int kIters = kStageTokens / kTPI;
  static constexpr bool kDsFastest = kNS >= 8;
  static constexpr int kDsShift = kDsFastest ? 0 : kLog2TPI;
  static constexpr int kTsShift = kDsFastest ? kLog2NS : 0;
  // PV mapping: LPT lanes per token.
  static constexpr int kLPT = D / 8;
  static constexpr int kLog2LPT = ilog2(kLPT);
  static constexpr int kTPV = 32 / kLPT;
  static constexpr int kTileBytes = kStageTokens * kRowBytes;
  static constexpr int kStageBytes = 2 * kTileBytes;
  static_assert(kRowBytes == 128 || kRowBytes == 256, "row must be 128 or 256 bytes");
  static_assert(G <= kNS, "group larger than the lanes of a token");
  static_assert(kNPL >= 1 && kNPL * kNS == kPiecesPerRow, "pieces must split evenly");
};

// Byte offset of piece `pc` (8 elements) of token row `t` inside a [chunk][64 tokens][128 B] tile
// written by TMA with the 128-byte swizzle (16-byte unit u of row t lives at unit u ^ (t & 7)).
template <class S>
__device__ __forceinline__ uint32_t piece_offset(int t, int pc) {
  const int byte = pc * S::kPieceBytes;
  const int c = byte >> 7;
  const int b = byte & 127;
  return static_cast<uint32_t>(c * (kStageTokens * 128) + t * 128 + ((((b >> 4) ^ (t & 7)) << 4) | (b & 15)));
}

// Piece read by a lane in QK step j. FP8 rows with 8 lanes per token alternate halves by token
// parity so that two tokens sharing a half-warp hit disjoint banks.
template <class S, int EB>
__device__ __forceinline__ int qk_piece(int j, int ds, int tslot) {
  if constexpr (EB == 1 && S::kNS == 8 && S::kNPL == 2) return ds + 8 * (j ^ (tslot & 1));
  return ds + S::kNS * j;
}

template <int G, int NS_LOG2, int DS_SHIFT>
__device__ __forceinline__ float reduce_scatter(float (&v)[G], int lane) {
  // Halving exchange over the ds lane bits, high bit first: after log2(G) halvings each lane holds
  // one head's partial sum over its lane pair group; the remaining bits finish a full reduction.
  constexpr int kLog2G = ilog2(G);
#pragma unroll
  for (int step = 0; step < NS_LOG2; ++step) {
    const int bit = NS_LOG2 - 1 - step;
    const int mask = 1 << (bit + DS_SHIFT);
    if (step < kLog2G) {
      const int n = G >> step;
      const int half = n >> 1;
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

// CTAs per SM the kernel is compiled for (registers are not capped below what the G query rows and
// accumulators need).
template <int G>
constexpr int min_ctas_per_sm() { return 1; }

template <typename QT, typename KVT, int D, int G>
__global__ void __launch_bounds__(kThreads, min_ctas_per_sm<G>())
paged_attention_main(const __grid_constant__ CUtensorMap tmap_k, const __grid_constant__ CUtensorMap tmap_v,
                     const AttnArgs args) {
  constexpr int EB = Elem<KVT>::kBytes;
  using S = Shape<D, G, EB>;
  using Piece = typename Elem<KVT>::Piece;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int kvh = blockIdx.x / args.subgroups;
  const int sub = blockIdx.x - kvh * args.subgroups;
  const int h0 = kvh * args.group + sub * G;
  const int heads_here = cmin(G, args.group - sub * G);
  const int s = blockIdx.y;
  const int part = blockIdx.z;
  const int PS = args.partition_size;

  const int L = args.context_lens[s];
  const bool bad_len = L < 0 || L > args.max_blocks_per_seq * args.block_size ||
                       L > args.num_partitions * PS;
  const int n_parts = bad_len ? 1 : (L + PS - 1) / PS;
  if (part >= (n_parts > 0 ? n_parts : 1)) return;  // whole CTA leaves: partition past the context
  const bool write_final = n_parts <= 1;

  if (L == 0 || bad_len) {
    // Empty context -> zeros; a context the launch cannot cover -> NaN and an error bit.
    if (bad_len && threadIdx.x == 0) atomicOr(args.error_word, PA_DEVERR_CONTEXT_LEN);
    const float fill = bad_len ? __int_as_float(0x7fc00000) : 0.0f;
    QT* out = static_cast<QT*>(args.out);
    for (int i = threadIdx.x; i < heads_here * D; i += kThreads) {
      const int g = i / D;
      out[(static_cast<size_t>(s) * args.num_heads + h0 + g) * D + (i - g * D)] = QT(fill);
    }
    return;
  }

  const int tok_begin = part * PS;
  const int tok_end = cmin(L, tok_begin + PS);
  const int n_stages = (tok_end - tok_begin + kStageTokens - 1) / kStageTokens;
  const int NST = args.num_stages;

  // Shared memory: [stage ring][P buffers][alpha buffers][mbarriers][flags], 1024-aligned ring.
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  float* pbuf = reinterpret_cast<float*>(smem + NST * S::kStageBytes);           // [W][64][G]
  float* abuf = pbuf + kConsumerWarps * kStageTokens * G;                         // [W][G]
  uint64_t* full = reinterpret_cast<uint64_t*>(abuf + kConsumerWarps * G + ((kConsumerWarps * G) & 1));
  uint64_t* empty = full + NST;
  int* flags = reinterpret_cast<int*>(empty + NST);                               // [0]: bad block

  if (threadIdx.x == 0) {
    for (int i = 0; i < NST; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
    }
    flags[0] = 0;
    fence_mbar_init();
  }
  __syncthreads();

  if (warp == kConsumerWarps) {
    // ------------------------------- producer warp -------------------------------
    if (lane == 0) {
      tma_prefetch_desc(&tmap_k);
      tma_prefetch_desc(&tmap_v);
    }
    const int bs = args.block_size;
    const int32_t* table = args.block_tables + static_cast<size_t>(s) * args.max_blocks_per_seq;
    auto stage_block_id = [&](int j) -> int {
      const int t0 = tok_begin + j * kStageTokens;
      const int nb = (cmin(kStageTokens, tok_end - t0) + bs - 1) / bs;
      return lane < nb ? __ldg(table + t0 / bs + lane) : 0;
    };
    bool bad_block = false;
    int issued = 0;
    int id_next = n_stages > 0 ? stage_block_id(0) : 0;
    for (int j = 0; j < n_stages; ++j) {
      const int id = id_next;
      if (j + 1 < n_stages) id_next = stage_block_id(j + 1);  // next stage's ids load during the wait
      const int slot = j % NST;
      const uint32_t round = static_cast<uint32_t>(j / NST);
      bool ok = true;
      if (lane == 0) ok = mbar_wait(&empty[slot], (round & 1u) ^ 1u, args.error_word);
      if (!__shfl_sync(0xffffffffu, ok, 0)) break;
      const int t0 = tok_begin + j * kStageTokens;
      const int nb = (cmin(kStageTokens, tok_end - t0) + bs - 1) / bs;
      uint8_t* ktile = smem + slot * S::kStageBytes;
      uint8_t* vtile = ktile + S::kTileBytes;
      if (lane == 0) mbar_arrive_expect_tx(&full[slot], static_cast<uint32_t>(nb * bs * S::kRowBytes * 2));
      for (int i = 0; i < nb; ++i) {
        int blk = __shfl_sync(0xffffffffu, id, i);
        if (lane == 0) {
          if (blk < 0 || blk >= args.num_blocks) {
            bad_block = true;
            blk = args.num_blocks;  // out-of-range coordinate: TMA fills the box with zeros
          }
#pragma unroll
          for (int c = 0; c < S::kChunks; ++c) {
            const int dst = c * (kStageTokens * 128) + i * bs * 128;
            tma_load_4d(ktile + dst, &tmap_k, &full[slot], c * S::kChunkElems, kvh, 0, blk);
            tma_load_4d(vtile + dst, &tmap_v, &full[slot], c * S::kChunkElems, kvh, 0, blk);
          }
        }
      }
      issued = j + 1;
    }
    bad_block = __any_sync(0xffffffffu, bad_block);
    if (bad_block && lane == 0) {
      atomicOr(args.error_word, PA_DEVERR_BLOCK_ID);
      flags[0] = 1;
    }
    // Drain: every issued stage's bytes have landed before the ring memory is reused or the CTA ends.
    if (lane == 0)
      for (int j = (issued > NST ? issued - NST : 0); j < issued; ++j)
        mbar_wait(&full[j % NST], static_cast<uint32_t>(j / NST) & 1u, args.error_word);
    __syncwarp();
    named_barrier(1, kThreads);
    return;
  }

  // ------------------------------- consumer warps -------------------------------
  // QK lane roles.
  const int ds = S::kDsFastest ? (lane & (S::kNS - 1)) : (lane >> S::kLog2TPI);
  const int tslot = S::kDsFastest ? (lane >> S::kLog2NS) : (lane & (S::kTPI - 1));
  const int g_lane = ds >> (S::kLog2NS - S::kLog2G);                 // head owned after reduce-scatter
  const bool primary = (ds & ((S::kNS >> S::kLog2G) - 1)) == 0;      // first of the duplicate lanes
  // PV lane roles.
  const int dp = lane & (S::kLPT - 1);
  const int vslot = lane >> S::kLog2LPT;

  // Query rows in registers, pre-scaled (scale * log2 e, times k_scale for FP8 caches).
  float qscale = args.scale_log2;
  if constexpr (EB == 1) qscale *= args.k_scale[kvh];
  float2 qr[G][S::kNPL][4];
  {
    const QT* q = static_cast<const QT*>(args.query) + (static_cast<size_t>(s) * args.num_heads + h0) * D;
#pragma unroll
    for (int g = 0; g < G; ++g) {
#pragma unroll
      for (int j = 0; j < S::kNPL; ++j) {
        const int pc = qk_piece<S, EB>(j, ds, tslot);
        if (g < heads_here) {
          const uint4 raw = __ldg(reinterpret_cast<const uint4*>(q + static_cast<size_t>(g) * D + pc * 8));
          const QT* e = reinterpret_cast<const QT*>(&raw);
#pragma unroll
          for (int k = 0; k < 4; ++k)
            qr[g][j][k] = make_float2(to_f32(e[2 * k]) * qscale, to_f32(e[2 * k + 1]) * qscale);
        } else {
#pragma unroll
          for (int k = 0; k < 4; ++k) qr[g][j][k] = make_float2(0.f, 0.f);
        }
      }
    }
  }

  float m_run = -INFINITY;  // running max of head g_lane (log2 domain)
  float l_run = 0.f;        // this lane's share of the running sum of head g_lane
  float2 acc[G][4];
#pragma unroll
  for (int g = 0; g < G; ++g)
#pragma unroll
    for (int k = 0; k < 4; ++k) acc[g][k] = make_float2(0.f, 0.f);

  float* pw = pbuf + warp * kStageTokens * G;
  float* aw = abuf + warp * G;

  for (int j = warp; j < n_stages; j += kConsumerWarps) {
    const int slot = j % NST;
    if (!__all_sync(0xffffffffu, mbar_wait(&full[slot], static_cast<uint32_t>(j / NST) & 1u, args.error_word))) break;
    const int nvalid = cmin(kStageTokens, tok_end - (tok_begin + j * kStageTokens));
    const uint8_t* ktile = smem + slot * S::kStageBytes;
    const uint8_t* vtile = ktile + S::kTileBytes;

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
        const Piece kp = *reinterpret_cast<const Piece*>(ktile + piece_offset<S>(t, pc));
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
      const float z = reduce_scatter<G, S::kLog2NS, S::kDsShift>(v, lane);
      sc[it] = t < nvalid ? z : -INFINITY;
    }

    // ---- online softmax (per head g_lane) ----
    float cmax = sc[0];
#pragma unroll
    for (int it = 1; it < S::kIters; ++it) cmax = fmaxf(cmax, sc[it]);
#pragma unroll
    for (int b = 0; b < 5 - S::kLog2NS; ++b) cmax = fmaxf(cmax, __shfl_xor_sync(0xffffffffu, cmax, 1 << (b + S::kTsShift)));
    const float m_new = fmaxf(m_run, cmax);
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
    for (int t0 = 0; t0 < nvalid; t0 += S::kTPV) {
      const int t = t0 + vslot;
      if (t < nvalid) {
        const Piece vp = *reinterpret_cast<const Piece*>(vtile + piece_offset<S>(t, dp));
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
#pragma unroll
        for (int g = 0; g < G; ++g) {
          const float2 pp = make_float2(p[g], p[g]);
#pragma unroll
          for (int k = 0; k < 4; ++k) acc[g][k] = ffma2(pp, vf[k], acc[g][k]);
        }
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[slot]);
  }

  // ---- per-warp totals ----
#pragma unroll
  for (int b = 0; b < 5 - S::kLog2NS; ++b) l_run += __shfl_xor_sync(0xffffffffu, l_run, 1 << (b + S::kTsShift));
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

  named_barrier(1, kThreads);  // producer has drained: the ring memory is free for the merge

  float* ma = reinterpret_cast<float*>(smem);              // [W][G][D]
  float* mm = ma + kConsumerWarps * G * D;                 // [W][G]
  float* ml = mm + kConsumerWarps * G;                     // [W][G]
  if (vslot == 0) {
#pragma unroll
    for (int g = 0; g < G; ++g) {
      float* dst = ma + (warp * G + g) * D + dp * 8;
      *reinterpret_cast<float4*>(dst) = make_float4(acc[g][0].x, acc[g][0].y, acc[g][1].x, acc[g][1].y);
      *reinterpret_cast<float4*>(dst + 4) = make_float4(acc[g][2].x, acc[g][2].y, acc[g][3].x, acc[g][3].y);
    }
  }
  if (primary && tslot == 0) {
    mm[warp * G + g_lane] = m_run;
    ml[warp * G + g_lane] = l_run;
  }
  named_barrier(2, kConsumerWarps * 32);

  const bool poisoned = flags[0] != 0;
  const float vscale = (EB == 1) ? args.v_scale[kvh] : 1.0f;
  for (int idx = threadIdx.x; idx < G * (D / 4); idx += kConsumerWarps * 32) {
    const int g = idx / (D / 4);
    const int d0 = (idx - g * (D / 4)) * 4;
    if (g >= heads_here) continue;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < kConsumerWarps; ++w) M = fmaxf(M, mm[w * G + g]);
    float lsum = 0.f;
    float4 o = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int w = 0; w < kConsumerWarps; ++w) {
      const float e = fast_exp2(mm[w * G + g] - M);
      lsum += e * ml[w * G + g];
      const float4 a = *reinterpret_cast<const float4*>(ma + (w * G + g) * D + d0);
      o.x += e * a.x; o.y += e * a.y; o.z += e * a.z; o.w += e * a.w;
    }
    float r = vscale / lsum;
    if (poisoned) r = __int_as_float(0x7fc00000);
    const int h = h0 + g;
    if (write_final) {
      QT* out = static_cast<QT*>(args.out) + (static_cast<size_t>(s) * args.num_heads + h) * D + d0;
      *reinterpret_cast<uint2*>(out) = pack4<QT>(o.x * r, o.y * r, o.z * r, o.w * r);
    } else {
      const size_t row = (static_cast<size_t>(s) * args.num_heads + h) * args.num_partitions + part;
      *reinterpret_cast<float4*>(args.part_o + row * D + d0) = make_float4(o.x * r, o.y * r, o.z * r, o.w * r);
      if (d0 == 0) {
        args.part_m[row] = M;
        args.part_l[row] = lsum;
      }
    }
  }
}

// Split-K merge of partitions: out = sum_p w_p o_p / sum_p w_p with w_p = l_p 2^(m_p - max m).
// One CTA of D threads per (query head, sequence); sequences with one partition (or an empty or
// invalid context) were finished by the main kernel.
template <typename QT, int D>
__global__ void __launch_bounds__(D)
paged_attention_reduce(const AttnArgs args) {
  const int h = blockIdx.x;
  const int s = blockIdx.y;
  const int i = threadIdx.x;
  const int L = args.context_lens[s];
  const int PS = args.partition_size;
  if (L <= 0 || L > args.max_blocks_per_seq * args.block_size || L > args.num_partitions * PS) return;
  const int n_parts = (L + PS - 1) / PS;
  if (n_parts <= 1) return;
  const size_t base = (static_cast<size_t>(s) * args.num_heads + h) * args.num_partitions;
  float M = -INFINITY;
  for (int p = 0; p < n_parts; ++p) M = fmaxf(M, args.part_m[base + p]);
  float wsum = 0.f, o = 0.f;
  for (int p = 0; p < n_parts; ++p) {
    const float w = args.part_l[base + p] * fast_exp2(args.part_m[base + p] - M);
    wsum += w;
    o += w * args.part_o[(base + p) * D + i];
  }
  QT* out = static_cast<QT*>(args.out) + (static_cast<size_t>(s) * args.num_heads + h) * D;
  out[i] = QT(o / wsum);
}

}  // namespace pa
