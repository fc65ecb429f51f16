// pa_prefill.cuh -- causal paged prefill attention on the sm_100a tensor cores (tcgen05 + TMEM).
//
// A chunk of n_s new query tokens of sequence s (the last n_s of its L_s cached tokens, whose keys
// and values are already in the paged cache) attends causally to its prefix: query j at position
// p = L_s - n_s + j reads keys 0..p (page "PagedAttention 与连续批处理：LLM Serving 的底层架构拆解":
// prefill is the compute-bound phase, section "对 agent 开发者的启示"; a token attends to its prefix,
// section "PagedAttention：把显存做成虚拟内存"; softmax(QK^T * scale) V from the tutorial page
// "企业官网建设流程全解析", sec. 2.2; the block table indirection from sec. 2.1).
//
// One CTA per (pair of 128-row query tiles A and B, kv head, sequence). A tile's 128 rows are 128/G
// query tokens x the G query heads that share the kv head, so grouped heads reuse every K/V tile, and
// the two tiles share the K/V stream. Per 128-key tile j:
//   warp 0        TMA: both query tiles once; K and V boxes of one block x one kv head x 64 columns,
//                 straight from the paged cache through the block table, into a 2-stage ring;
//   warp 1        one thread issues, per tile X, S_X = Q_X K^T (M 128, N 128) into TMEM and
//                 O_X += P_X V (M 128, N d) with P read from TMEM, in the order
//                 S_A(0) S_B(0) | PV_A(j) S_A(j+1) PV_B(j) S_B(j+1) | ..., so that each softmax
//                 warpgroup works on its S while the tensor cores run the other tile's pair;
//   warps 4..7    softmax of tile A, warps 8..11 of tile B: thread r owns row r (TMEM lane r); it reads
//                 its S row, applies the causal mask, computes P = exp2(S * scale * log2e - m) against
//                 a running max m that is raised only when a row's maximum exceeds it by more than 8
//                 (then O and the sum are rescaled in place), and writes P (16-bit pairs) over S for the
//                 PV MMA; at the end it normalises O and stores the row.
// FP8-E4M3 caches (KVB = 1; tutorial page, sec. 3.2 "关键性能优化": blocks stored in FP8) take the same
// path on f16 operands. TMA lands each E4M3 tile (128 keys x 128 one-byte columns) in the upper half of
// its f16 operand slot; warps 2-3 widen it in place (every E4M3 value is exact in f16), each thread
// owning whole rows, so a row is read before it is overwritten. A bf16 query is converted to f16 in
// place once. Per-kv-head scales are exact fp32 factors on the softmax scale (K) and on the output (V);
// per-block scales multiply the widened values (f16, one extra rounding of code x scale).
// Every wait is bounded; a timed-out wait records PA_DEVERR_TIMEOUT and the CTA winds down (waiting,
// bounded, for its own copies and MMAs) before it frees TMEM.
#pragma once

#include <cuda.h>
#include <math.h>

#include "pa_device.cuh"
#include "pa_tcgen05.cuh"

namespace pa {
namespace pf {

constexpr int kRows = 128;      // query rows per tile (M of both MMAs)
constexpr int kTiles = 2;       // query tiles per CTA
constexpr int kKvTile = 128;    // keys per KV tile (N of QK^T, K of PV)
constexpr int kStages = 2;      // K/V ring depth
constexpr int kThreads = 384;   // warp 0 TMA, warp 1 MMA, warps 2-3 idle, warps 4-7 / 8-11 softmax
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kTmemTile = 256;  // per query tile: S (and P over it) in [0, 128), O in [128, 128 + d)
constexpr uint32_t kTmemO = 128;
constexpr float kRescaleThreshold = 8.0f;  // log2 units: P stays below 2^8 between rescales

struct PrefillArgs {
  void* out;                    // [T][H][d]
  const float* k_scale;         // FP8: [Hkv] or [num_blocks][Hkv] (scale_block_stride = Hkv); else null
  const float* v_scale;
  int scale_block_stride;
  const int32_t* block_tables;  // [S][max_blocks_per_seq]
  const int32_t* context_lens;  // [S]
  const int32_t* q_start;       // [S + 1]
  unsigned int* error_word;
  int max_blocks_per_seq, num_seqs, num_q_tokens, num_heads, num_kv_heads, group, tile_tokens, block_size,
      num_blocks, num_pairs;
  float scale_log2;             // scale * log2(e)
};

template <int D>
struct Layout {
  static constexpr int kChunks = D / 64;                        // 128-byte column chunks of a d row
  static constexpr uint32_t kTileChunk = kRows * 128;           // one chunk of a 128-row tile
  static constexpr uint32_t kQ = 0;                             // tile X at kQ + X * kQTile
  static constexpr uint32_t kQTile = kChunks * kTileChunk;
  static constexpr uint32_t kKV = kQ + kTiles * kQTile;
  static constexpr uint32_t kK = 0;                             // inside a stage
  static constexpr uint32_t kV = kChunks * kKvTile * 128;
  static constexpr uint32_t kStage = 2 * kChunks * kKvTile * 128;
  static constexpr uint32_t kBars = kKV + kStages * kStage;
  // Barriers, flags and box scales, alignment slack; at least 120 KB so that one CTA holds an SM (and
  // with it all 512 TMEM columns: a second CTA's allocation would wait for the first to finish).
  static constexpr uint32_t kBytes = (kBars + 1024 + 1024) > 120u * 1024 ? (kBars + 1024 + 1024) : 120u * 1024;
};

struct Bars {
  uint64_t q_full, k_full[kStages], k_empty[kStages], v_full[kStages], v_empty[kStages], s_full[kTiles],
      p_full[kTiles], o_final[kTiles], mma_done;
  uint64_t q_ready, k_load[kStages], v_load[kStages];  // FP8: query in f16, E4M3 tiles landed
  float box_scale[kStages][2][kKvTile / 8];            // per-block FP8: K and V scale of each box
  uint32_t tmem_base;
  int abort;
};

__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// A bounded wait that gives up at once after any role of the CTA has given up.
__device__ __forceinline__ bool wait_or_abort(Bars* b, uint64_t* bar, uint32_t parity, unsigned int* err) {
  if (*reinterpret_cast<volatile int*>(&b->abort)) return false;
  if (mbar_wait(bar, parity, err)) return true;
  *reinterpret_cast<volatile int*>(&b->abort) = 1;
  return false;
}

// The same wait taken by a whole warp, with one outcome for all of its lanes (the warp-wide
// instructions that follow need every lane).
__device__ __forceinline__ bool warp_wait_or_abort(Bars* b, uint64_t* bar, uint32_t parity, unsigned int* err) {
  return __all_sync(0xffffffffu, wait_or_abort(b, bar, parity, err));
}

template <typename T>
__device__ __forceinline__ uint32_t pack_pair(float a, float b);
template <>
__device__ __forceinline__ uint32_t pack_pair<__nv_bfloat16>(float a, float b) {
  __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&h);
}
template <>
__device__ __forceinline__ uint32_t pack_pair<__half>(float a, float b) {
  __half2 h = __floats2half2_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&h);
}
// Widens row r of an E4M3 tile in place: the row's 128 codes (128-byte swizzled row r at `staged`) become
// 128 f16 values in the two 128-byte-swizzled chunks of the f16 tile at `tile` (chunk stride
// kKvTile * 128), multiplied by `scale` when it is not 1. The whole row is read before any write.
__device__ __forceinline__ void widen_row(uint8_t* tile, const uint8_t* staged, int r, __half2 scale, bool scaled) {
  uint4 q[8];
#pragma unroll
  for (int u = 0; u < 8; ++u) q[u] = *reinterpret_cast<const uint4*>(staged + r * 128 + ((u ^ (r & 7)) << 4));
#pragma unroll
  for (int u = 0; u < 8; ++u) {
    const uint32_t w[4] = {q[u].x, q[u].y, q[u].z, q[u].w};
    uint32_t h[8];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      h[2 * k] = e4m3x2_to_f16x2(static_cast<uint16_t>(w[k] & 0xffffu));
      h[2 * k + 1] = e4m3x2_to_f16x2(static_cast<uint16_t>(w[k] >> 16));
    }
    if (scaled) {
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        __half2 x = *reinterpret_cast<__half2*>(&h[k]);
        x = __hmul2(x, scale);
        h[k] = *reinterpret_cast<uint32_t*>(&x);
      }
    }
    // Values 16u .. 16u + 15 are f16 units 2u and 2u + 1 of the row: chunk u / 4, units 2(u % 4) + {0, 1}.
    uint8_t* row = tile + (u >> 2) * (kKvTile * 128) + r * 128;
    *reinterpret_cast<uint4*>(row + (((2 * (u & 3)) ^ (r & 7)) << 4)) = make_uint4(h[0], h[1], h[2], h[3]);
    *reinterpret_cast<uint4*>(row + (((2 * (u & 3) + 1) ^ (r & 7)) << 4)) = make_uint4(h[4], h[5], h[6], h[7]);
  }
}

// KVB: cache element bytes (2: a T cache; 1: E4M3). BS: E4M3 with per-(block, kv head) scales.
template <typename T, int D, int KVB, bool BS>
__global__ void __launch_bounds__(kThreads, 1)
paged_prefill_kernel(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
                     const __grid_constant__ CUtensorMap tv, const PrefillArgs a) {
  using L = Layout<D>;
  constexpr bool kFp8 = KVB == 1;
  using MT = typename std::conditional<kFp8, __half, T>::type;  // tensor-core operand type
  static_assert(!kFp8 || D == 128, "FP8 caches need head_size 128");
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  Bars* b = reinterpret_cast<Bars*>(sm + L::kBars);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int pair = a.num_pairs - 1 - static_cast<int>(blockIdx.x);  // longest prefixes first
  const int kvh = blockIdx.y, s = blockIdx.z;
  const int G = a.group;

  // ---- the tiles' extent; every condition below is uniform over the CTA ----
  const int q0 = a.q_start[s];
  const int n = a.q_start[s + 1] - q0;
  const int ctx = a.context_lens[s];
  const int tok0 = pair * kTiles * a.tile_tokens;  // first token of tile A; tile B follows
  if (n <= 0 || tok0 >= n || q0 < 0) {
    if (pair == 0 && threadIdx.x == 0 && (n < 0 || q0 < 0)) atomicOr(a.error_word, PA_DEVERR_CONTEXT_LEN);
    return;
  }
  if (n > ctx || q0 + n > a.num_q_tokens ||
      static_cast<long long>(ctx) > static_cast<long long>(a.max_blocks_per_seq) * a.block_size) {
    // A chunk must lie inside its context and inside the query array: flag it, NaN the rows.
    if (threadIdx.x == 0) atomicOr(a.error_word, PA_DEVERR_CONTEXT_LEN);
    if (threadIdx.x < kTiles * kRows && q0 + n <= a.num_q_tokens) {
      const int tok = tok0 + static_cast<int>(threadIdx.x) / G;
      if (tok < n) {
        T* o = static_cast<T*>(a.out) +
               (static_cast<size_t>(q0 + tok) * a.num_heads + kvh * G + threadIdx.x % G) * D;
        const float nan = __int_as_float(0x7fc00000);
        for (int i = 0; i < D; i += 2) *reinterpret_cast<uint32_t*>(o + i) = pack_pair<T>(nan, nan);
      }
    }
    return;
  }
  // Per tile: first token, KV tiles needed (0 when the tile lies past the chunk).
  int tile_tok0[kTiles], nkv_t[kTiles];
  int p_max = 0;
#pragma unroll
  for (int x = 0; x < kTiles; ++x) {
    tile_tok0[x] = tok0 + x * a.tile_tokens;
    if (tile_tok0[x] < n) {
      const int pm = ctx - n + min(n, tile_tok0[x] + a.tile_tokens) - 1;  // last key the tile needs
      nkv_t[x] = pm / kKvTile + 1;
      p_max = max(p_max, pm);
    } else {
      nkv_t[x] = 0;
    }
  }
  const int nkv = p_max / kKvTile + 1;  // = nkv_t of the last active tile

  // The TMA warp fetches its tensor maps and the first KV tile's block ids now, so that those loads
  // overlap the set-up below.
  int blk_first = 0;
  if (warp == 0) {
    if (lane == 0) {
      tma_prefetch_desc(&tq);
      tma_prefetch_desc(&tk);
      tma_prefetch_desc(&tv);
    }
    if (lane * a.block_size < min(kKvTile, p_max + 1))
      blk_first = __ldg(a.block_tables + static_cast<size_t>(s) * a.max_blocks_per_seq + lane);
  }

  // ---- set-up: barriers (thread 0), TMEM (warp 1) ----
  if (threadIdx.x == 0) {
    mbar_init(&b->q_full, 1);
    mbar_init(&b->q_ready, 64);
    for (int i = 0; i < kStages; ++i) {
      mbar_init(&b->k_full[i], kFp8 ? 64 : 1);   // FP8: the 64 widening threads arrive
      mbar_init(&b->k_empty[i], 1);
      mbar_init(&b->v_full[i], kFp8 ? 64 : 1);
      mbar_init(&b->v_empty[i], 1);
      mbar_init(&b->k_load[i], 1);
      mbar_init(&b->v_load[i], 1);
    }
    for (int x = 0; x < kTiles; ++x) {
      mbar_init(&b->s_full[x], 1);
      mbar_init(&b->p_full[x], kRows);
      mbar_init(&b->o_final[x], 1);
    }
    mbar_init(&b->mma_done, 1);
    b->abort = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(&b->tmem_base, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = b->tmem_base;
  unsigned int* err = a.error_word;
  if (warp == 0) {
    // ================================ TMA producer ================================
    int issued[2 * kStages] = {0, 0, 0, 0};
    const int bs = a.block_size;
    const int32_t* table = a.block_tables + static_cast<size_t>(s) * a.max_blocks_per_seq;
    if (lane == 0) {
      const int tiles = (nkv_t[1] > 0) ? 2 : 1;
      mbar_arrive_expect_tx(&b->q_full, tiles * L::kQTile);
      for (int x = 0; x < tiles; ++x)
        for (int c = 0; c < L::kChunks; ++c)
          tma_load_3d(sm + L::kQ + x * L::kQTile + c * L::kTileChunk, &tq, &b->q_full, c * 64, kvh * G,
                      q0 + tile_tok0[x]);
    }
    // K and V of a tile go to separate rings: a K slot is freed once both query tiles' S MMAs have
    // read it, long before the PV MMAs release the V slot, so the next K arrives early.
    for (int j = 0; j < nkv; ++j) {
      const int stage = j % kStages;
      const int first = j * kKvTile;
      const int ntok = min(kKvTile, p_max + 1 - first);
      const int nblk = (ntok + bs - 1) / bs;
      int blk = 0;
      bool ok = false;
      if (lane < nblk) {
        blk = j == 0 ? blk_first : table[first / bs + lane];
        ok = blk >= 0 && blk < a.num_blocks;
        if (!ok) atomicOr(err, PA_DEVERR_BLOCK_ID);
      }
      const unsigned okmask = __ballot_sync(0xffffffffu, ok);
      const uint32_t bytes = __popc(okmask) * bs * 128 * (kFp8 ? 1 : L::kChunks);
      uint8_t* st = sm + L::kKV + stage * L::kStage;
      bool go = true;
#pragma unroll
      for (int part = 0; part < 2; ++part) {  // 0: K, 1: V
        uint64_t* full = kFp8 ? (part == 0 ? &b->k_load[stage] : &b->v_load[stage])
                              : (part == 0 ? &b->k_full[stage] : &b->v_full[stage]);
        uint64_t* empty = part == 0 ? &b->k_empty[stage] : &b->v_empty[stage];
        if (j >= kStages && !warp_wait_or_abort(b, empty, ((j / kStages) - 1) & 1, err)) {
          go = false;
          break;
        }
        if constexpr (kFp8 && BS) {
          // Scale of each box for the widening warps: the slot's previous tile has been widened (its
          // MMAs, which waited for that, have released the slot), and the arrive below publishes it.
          if (lane < nblk)
            b->box_scale[stage][part][lane] =
                ok ? __ldg((part == 0 ? a.k_scale : a.v_scale) + static_cast<size_t>(blk) * a.scale_block_stride + kvh)
                   : 0.f;
          __syncwarp();
        }
        if (lane == 0) mbar_arrive_expect_tx(full, bytes);
        __syncwarp();
        if (ok) {
          if constexpr (kFp8) {
            // The E4M3 tile (one 128-byte chunk per row) lands in the upper half of the f16 slot.
            tma_load_4d(st + (part == 0 ? L::kK : L::kV) + (kKvTile * 128) + lane * bs * 128, part == 0 ? &tk : &tv,
                        full, 0, 0, kvh, blk);
          } else {
            for (int c = 0; c < L::kChunks; ++c)
              tma_load_4d(st + (part == 0 ? L::kK : L::kV) + c * (kKvTile * 128) + lane * bs * 128,
                          part == 0 ? &tk : &tv, full, c * 64, 0, kvh, blk);
          }
        }
        ++issued[part * kStages + stage];
      }
      if (!go) break;
    }
    // Wind-down: the last load issued into each slot has landed (immediate unless the CTA aborted).
    for (int part = 0; part < 2; ++part)
      for (int i = 0; i < kStages; ++i)
        if (issued[part * kStages + i] > 0)
          mbar_wait(kFp8 ? (part == 0 ? &b->k_load[i] : &b->v_load[i]) : (part == 0 ? &b->k_full[i] : &b->v_full[i]),
                    (issued[part * kStages + i] - 1) & 1, err);
  } else if (kFp8 && (warp == 2 || warp == 3)) {
    // ================================ E4M3 widening (FP8 caches) ================================
    const int ct = threadIdx.x - 64;  // 0..63
    bool ok = warp_wait_or_abort(b, &b->q_full, 0, err);
    if (ok && std::is_same<T, __nv_bfloat16>::value) {
      // The query tiles to f16, in place (same positions; every value of the bf16 range that f16 holds
      // converts exactly up to f16's precision and range).
      const int tiles = (nkv_t[1] > 0) ? 2 : 1;
      uint4* q = reinterpret_cast<uint4*>(sm + L::kQ);
      for (int i = ct; i < tiles * static_cast<int>(L::kQTile) / 16; i += 64) {
        uint4 v = q[i];
        uint32_t* w = reinterpret_cast<uint32_t*>(&v);
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w[k]));
          const __half2 h = __floats2half2_rn(f.x, f.y);
          w[k] = *reinterpret_cast<const uint32_t*>(&h);
        }
        q[i] = v;
      }
    }
    fence_proxy_async_smem();
    mbar_arrive(&b->q_ready);
    for (int j = 0; ok && j < nkv; ++j) {
      const int stage = j % kStages;
      for (int part = 0; part < 2; ++part) {
        if (!(ok = warp_wait_or_abort(b, part == 0 ? &b->k_load[stage] : &b->v_load[stage], (j / kStages) & 1, err)))
          break;
        uint8_t* tile = sm + L::kKV + stage * L::kStage + (part == 0 ? L::kK : L::kV);
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const int r = ct + 64 * h;
          __half2 sc = __float2half2_rn(1.f);
          if constexpr (BS) {
            if (j * kKvTile + r <= p_max) sc = __float2half2_rn(b->box_scale[stage][part][r / a.block_size]);
          }
          widen_row(tile, tile + kKvTile * 128, r, sc, BS);
        }
        fence_proxy_async_smem();
        mbar_arrive(part == 0 ? &b->k_full[stage] : &b->v_full[stage]);
      }
    }
  } else if (warp == 1) {
    // ================================ MMA issuer ================================
    constexpr uint32_t idesc_s = mma_idesc_f16<MT>(kRows, kKvTile, false);
    constexpr uint32_t idesc_o = mma_idesc_f16<MT>(kRows, D, true);
    auto kv_addr = [&](int j, uint32_t part) { return smem_u32(sm + L::kKV + (j % kStages) * L::kStage + part); };
    auto issue_s = [&](int x, int j) {  // S_x = Q_x K_j^T over d in steps of 16
      const uint32_t q_addr = smem_u32(sm + L::kQ + x * L::kQTile), k_addr = kv_addr(j, L::kK);
#pragma unroll
      for (int k = 0; k < D / 16; ++k) {
        const uint32_t qo = (k >> 2) * L::kTileChunk + (k & 3) * 32;
        const uint32_t ko = (k >> 2) * (kKvTile * 128) + (k & 3) * 32;
        mma_f16_ss(tmem + x * kTmemTile, smem_desc_sw128(q_addr + qo, 16, 1024),
                   smem_desc_sw128(k_addr + ko, 16, 1024), idesc_s, k > 0);
      }
      mma_commit(&b->s_full[x]);
    };
    auto issue_pv = [&](int x, int j) {  // O_x += P_x V_j over keys in steps of 16, P from TMEM
      const uint32_t v_addr = kv_addr(j, L::kV);
#pragma unroll
      for (int k = 0; k < kKvTile / 16; ++k)
        mma_f16_ts(tmem + x * kTmemTile + kTmemO, tmem + x * kTmemTile + 8 * k,
                   smem_desc_sw128(v_addr + k * 16 * 128, kKvTile * 128, 1024), idesc_o, (j > 0 || k > 0) ? 1u : 0u);
    };
    bool ok = warp_wait_or_abort(b, kFp8 ? &b->q_ready : &b->q_full, 0, err) &&
              warp_wait_or_abort(b, &b->k_full[0], 0, err);
    if (ok) {
      tc_fence_after();
      if (lane == 0) {
        for (int x = 0; x < kTiles; ++x)
          if (nkv_t[x] > 0) issue_s(x, 0);
        mma_commit(&b->k_empty[0]);
      }
      __syncwarp();
    }
    for (int j = 0; ok && j < nkv; ++j) {
      if (!(ok = warp_wait_or_abort(b, &b->v_full[j % kStages], (j / kStages) & 1, err))) break;
      if (j == nkv - 1) {
        // Keys past the last one any row needs (not loaded, or past the context) must not reach PV
        // as stale or NaN values: zero those V rows of the last tile before its PV MMAs.
        const int cut = p_max + 1 - j * kKvTile;
        if (cut < kKvTile) {
          uint8_t* vb = sm + L::kKV + (j % kStages) * L::kStage + L::kV;
          const int units = (kKvTile - cut) * 8;
          for (int c = 0; c < L::kChunks; ++c)
            for (int u = lane; u < units; u += 32)
              *reinterpret_cast<uint4*>(vb + c * (kKvTile * 128) + cut * 128 + u * 16) = make_uint4(0, 0, 0, 0);
          fence_proxy_async_smem();
        }
        __syncwarp();
      }
      bool next_k = false;  // K_{j+1} waited for
      for (int x = 0; x < kTiles; ++x) {
        if (j >= nkv_t[x]) continue;
        if (!(ok = warp_wait_or_abort(b, &b->p_full[x], j & 1, err))) break;
        tc_fence_after();
        if (lane == 0) issue_pv(x, j);
        if (j + 1 < nkv_t[x]) {
          if (!next_k && !(ok = warp_wait_or_abort(b, &b->k_full[(j + 1) % kStages], ((j + 1) / kStages) & 1, err)))
            break;
          next_k = true;
          tc_fence_after();
          if (lane == 0) issue_s(x, j + 1);
        } else if (lane == 0) {
          mma_commit(&b->o_final[x]);
        }
        __syncwarp();
      }
      if (!ok) break;
      if (lane == 0) {
        mma_commit(&b->v_empty[j % kStages]);
        if (next_k) mma_commit(&b->k_empty[(j + 1) % kStages]);
      }
      __syncwarp();
    }
    // Wind-down: every MMA issued above has completed before TMEM can be freed.
    if (lane == 0) {
      mma_commit(&b->mma_done);
      mbar_wait(&b->mma_done, 0, err);
    }
    __syncwarp();
  } else if (warp >= 4) {
    // ================================ softmax / epilogue ================================
    const int x = (warp - 4) >> 2;                  // query tile of this warpgroup
    const int r = threadIdx.x - 128 - x * kRows;    // row == TMEM lane
    const int nkv_x = nkv_t[x];
    if (nkv_x > 0) {
      const int tok = tile_tok0[x] + r / G;
      const bool row_valid = tok < n;
      const int pos = ctx - n + min(tok, n - 1);    // rows past the chunk reuse its last position
      const int pos_lane0 = __shfl_sync(0xffffffffu, pos, 0);
      const uint32_t t_s = tmem + x * kTmemTile + (static_cast<uint32_t>(r & ~31) << 16);
      const uint32_t t_o = t_s + kTmemO;
      // Per-kv-head FP8 scales are exact fp32 factors: K's on the softmax scale, V's on the output.
      const float sl2 = (kFp8 && !BS) ? a.scale_log2 * __ldg(a.k_scale + kvh) : a.scale_log2;
      const float out_scale = (kFp8 && !BS) ? __ldg(a.v_scale + kvh) : 1.f;
      float m = -INFINITY, l = 0.f;
      bool ok = true;
      for (int j = 0; j < nkv_x; ++j) {
        if (!(ok = warp_wait_or_abort(b, &b->s_full[x], j & 1, err))) break;
        tc_fence_after();
        const int base = j * kKvTile;
        // The whole S row at once: four loads in flight, then one wait.
        uint32_t v[kKvTile / 32][32];
#pragma unroll
        for (int c = 0; c < kKvTile / 32; ++c) tmem_ld32(t_s + 32 * c, v[c]);
#pragma unroll
        for (int c = 0; c < kKvTile / 32; ++c) tmem_wait_ld(v[c]);
        // Causal mask: keys past this row's position become -inf (then exp2 gives 0). Only chunks that
        // reach past the warp's first row position need it (positions rise with the lane).
        float mxs[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};  // independent chains
#pragma unroll
        for (int c = 0; c < kKvTile / 32; ++c) {
          if (base + 32 * c + 31 > pos_lane0) {
#pragma unroll
            for (int i = 0; i < 32; ++i)
              if (base + 32 * c + i > pos) v[c][i] = __float_as_uint(-INFINITY);
          }
#pragma unroll
          for (int i = 0; i < 32; i += 2)
            mxs[(i >> 1) & 3] = fmax3(mxs[(i >> 1) & 3], __uint_as_float(v[c][i]), __uint_as_float(v[c][i + 1]));
        }
        const float m_cand = fmaxf(fmaxf(mxs[0], mxs[1]), fmaxf(mxs[2], mxs[3])) * sl2;
        if (j == 0) {
          m = m_cand;                               // O is written fresh by the first PV
        } else {
          // S_x(j) was issued after PV_x(j-1), so O holds every earlier tile and may be rescaled.
          const bool raise = m_cand > m + kRescaleThreshold;
          if (__any_sync(0xffffffffu, raise)) {
            const float alpha = raise ? ex2(m - m_cand) : 1.f;
#pragma unroll 1
            for (int c = 0; c < D / 8; ++c) {      // 8 columns at a time: the S row stays in registers
              uint32_t o[8];
              tmem_ld8(t_o + 8 * c, o);
              tmem_wait_ld8(o);
#pragma unroll
              for (int i = 0; i < 8; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
              tmem_st8(t_o + 8 * c, o);
            }
            if (raise) {
              l *= alpha;
              m = m_cand;
            }
          }
        }
        // P = exp2(S * scale * log2e - m), written over S as 16-bit pairs (columns 16c .. 16c+15 were
        // read above); the row sum is kept in fp32.
        float2 ls[4];                               // independent chains
#pragma unroll
        for (int i = 0; i < 4; ++i) ls[i] = make_float2(0.f, 0.f);
        const float2 sl2x2 = make_float2(sl2, sl2), negm = make_float2(-m, -m);
#pragma unroll
        for (int c = 0; c < kKvTile / 32; ++c) {
          uint32_t w[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const float2 xy = __ffma2_rn(make_float2(__uint_as_float(v[c][2 * i]), __uint_as_float(v[c][2 * i + 1])),
                                         sl2x2, negm);
            const float2 p = make_float2(ex2(xy.x), ex2(xy.y));
            w[i] = pack_pair<MT>(p.x, p.y);
            ls[i & 3] = __fadd2_rn(ls[i & 3], p);
          }
          tmem_st16(t_s + 16 * c, w);
        }
        const float2 l2 = __fadd2_rn(__fadd2_rn(ls[0], ls[1]), __fadd2_rn(ls[2], ls[3]));
        const float lsum = l2.x + l2.y;
        l += lsum;
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(&b->p_full[x]);
      }
      if (ok) ok = warp_wait_or_abort(b, &b->o_final[x], 0, err);
      if (ok) {
        tc_fence_after();
        const float inv = out_scale / l;
        T* dst = static_cast<T*>(a.out) + (static_cast<size_t>(q0 + min(tok, n - 1)) * a.num_heads + kvh * G + r % G) * D;
#pragma unroll 1
        for (int c = 0; c < D / 32; ++c) {
          uint32_t v[32];
          tmem_ld32(t_o + 32 * c, v);
          tmem_wait_ld(v);
          if (row_valid) {
#pragma unroll
            for (int i = 0; i < 32; i += 8)
              *reinterpret_cast<uint4*>(dst + 32 * c + i) = make_uint4(
                  pack_pair<T>(__uint_as_float(v[i]) * inv, __uint_as_float(v[i + 1]) * inv),
                  pack_pair<T>(__uint_as_float(v[i + 2]) * inv, __uint_as_float(v[i + 3]) * inv),
                  pack_pair<T>(__uint_as_float(v[i + 4]) * inv, __uint_as_float(v[i + 5]) * inv),
                  pack_pair<T>(__uint_as_float(v[i + 6]) * inv, __uint_as_float(v[i + 7]) * inv));
          }
        }
      }
    }
  }

  // ---- teardown: every role has finished with TMEM ----
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace pf
}  // namespace pa
