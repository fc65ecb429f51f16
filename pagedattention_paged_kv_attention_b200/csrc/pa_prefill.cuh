// pa_prefill.cuh -- causal paged prefill attention on the sm_100a tensor cores (tcgen05 + TMEM).
//
// A chunk of n_s new query tokens of sequence s (the last n_s of its L_s cached tokens, whose keys
// and values are already in the paged cache) attends causally to its prefix: query j at position
// p = L_s - n_s + j reads keys 0..p (page "PagedAttention 与连续批处理：LLM Serving 的底层架构拆解":
// prefill is the compute-bound phase, section "对 agent 开发者的启示"; a token attends to its prefix,
// section "PagedAttention：把显存做成虚拟内存"; softmax(QK^T * scale) V from the tutorial page
// "企业官网建设流程全解析", sec. 2.2; the block table indirection from sec. 2.1).
//
// One CTA per (128-row query tile, kv head, sequence). A tile's 128 rows are 128/G query tokens x the
// G query heads that share the kv head, so grouped heads reuse every K/V tile. Per 128-token KV tile:
//   warp 0      TMA: the query tile once; K and V boxes of one block x one kv head x 64 columns,
//               straight from the paged cache through the block table, into a 2-stage ring;
//   warp 1      one thread issues S = Q K^T (M 128, N 128) into TMEM, then O_tile = P V (M 128, N d)
//               into TMEM, and commits each to an mbarrier; the warp owns the TMEM allocation;
//   warps 4..7  thread r owns row r (TMEM lane r): reads its S row, applies the causal mask, keeps the
//               online-softmax max/sum in fp32, writes P (16-bit, 128-byte swizzled K-major) to shared
//               memory for the PV MMA, and accumulates O_tile into fp32 registers with the rescale;
//               at the end it normalises and stores the row.
// Every wait is bounded; a timed-out wait records PA_DEVERR_TIMEOUT and the CTA winds down (waiting,
// bounded, for its own copies and MMAs) before it frees TMEM.
#pragma once

#include <cuda.h>
#include <math.h>

#include "pa_device.cuh"
#include "pa_tcgen05.cuh"

namespace pa {
namespace pf {

constexpr int kRows = 128;      // query rows per CTA (M of both MMAs)
constexpr int kKvTile = 128;    // keys per KV tile (N of QK^T, K of PV)
constexpr int kStages = 2;      // K/V ring depth
constexpr int kThreads = 256;   // warp 0 TMA, warp 1 MMA, warps 2-3 idle, warps 4-7 softmax
constexpr uint32_t kTmemCols = 256;
constexpr uint32_t kTmemS = 0;    // S: columns [0, 128)
constexpr uint32_t kTmemO = 128;  // O tile: columns [128, 128 + d)

struct PrefillArgs {
  void* out;                    // [T][H][d]
  const int32_t* block_tables;  // [S][max_blocks_per_seq]
  const int32_t* context_lens;  // [S]
  const int32_t* q_start;       // [S + 1]
  unsigned int* error_word;
  int max_blocks_per_seq, num_seqs, num_q_tokens, num_heads, num_kv_heads, group, tile_tokens, block_size,
      num_blocks, num_q_tiles;
  float scale_log2;             // scale * log2(e)
};

template <int D>
struct Layout {
  static constexpr int kChunks = D / 64;                        // 128-byte column chunks of a d row
  static constexpr uint32_t kTileChunk = kRows * 128;           // one chunk of a 128-row tile
  static constexpr uint32_t kQ = 0;
  static constexpr uint32_t kP = kQ + kChunks * kTileChunk;     // P: 128 rows x 128 keys = 2 chunks
  static constexpr uint32_t kKV = kP + 2 * kTileChunk;
  static constexpr uint32_t kK = 0;                             // inside a stage
  static constexpr uint32_t kV = kChunks * kKvTile * 128;
  static constexpr uint32_t kStage = 2 * kChunks * kKvTile * 128;
  static constexpr uint32_t kBars = kKV + kStages * kStage;
  static constexpr uint32_t kBytes = kBars + 256 + 1024;        // barriers and flags, alignment slack
};

struct Bars {
  uint64_t q_full, kv_full[kStages], kv_empty[kStages], s_full, p_full, o_full, o_empty, mma_done;
  uint32_t tmem_base;
  int abort;
};

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
template <typename T>
__device__ __forceinline__ float2 unpack_pair(uint32_t w);
template <>
__device__ __forceinline__ float2 unpack_pair<__nv_bfloat16>(uint32_t w) {
  return __bfloat1622float2(*reinterpret_cast<__nv_bfloat162*>(&w));
}
template <>
__device__ __forceinline__ float2 unpack_pair<__half>(uint32_t w) {
  return __half22float2(*reinterpret_cast<__half2*>(&w));
}

template <typename T, int D>
__global__ void __launch_bounds__(kThreads, 1)
paged_prefill_kernel(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
                     const __grid_constant__ CUtensorMap tv, const PrefillArgs a) {
  using L = Layout<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  Bars* b = reinterpret_cast<Bars*>(sm + L::kBars);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int q_tile = a.num_q_tiles - 1 - static_cast<int>(blockIdx.x);  // longest prefixes first
  const int kvh = blockIdx.y, s = blockIdx.z;
  const int G = a.group;

  // ---- the tile's extent; every condition below is uniform over the CTA ----
  const int q0 = a.q_start[s];
  const int n = a.q_start[s + 1] - q0;
  const int ctx = a.context_lens[s];
  const int tok0 = q_tile * a.tile_tokens;
  if (n <= 0 || tok0 >= n || q0 < 0) {
    if (q_tile == 0 && threadIdx.x == 0 && (n < 0 || q0 < 0)) atomicOr(a.error_word, PA_DEVERR_CONTEXT_LEN);
    return;
  }
  if (n > ctx || q0 + n > a.num_q_tokens ||
      static_cast<long long>(ctx) > static_cast<long long>(a.max_blocks_per_seq) * a.block_size) {
    // A chunk must lie inside its context and inside the query array: flag it, NaN the rows.
    if (threadIdx.x == 0) atomicOr(a.error_word, PA_DEVERR_CONTEXT_LEN);
    if (threadIdx.x < kRows && q0 + n <= a.num_q_tokens) {
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
  const int p_max = ctx - n + min(n, tok0 + a.tile_tokens) - 1;  // last key any row of the tile needs
  const int nkv = p_max / kKvTile + 1;

  // ---- set-up: barriers (thread 0), TMEM (warp 1) ----
  if (threadIdx.x == 0) {
    mbar_init(&b->q_full, 1);
    for (int i = 0; i < kStages; ++i) {
      mbar_init(&b->kv_full[i], 1);
      mbar_init(&b->kv_empty[i], 1);
    }
    mbar_init(&b->s_full, 1);
    mbar_init(&b->p_full, kRows);
    mbar_init(&b->o_full, 1);
    mbar_init(&b->o_empty, kRows);
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
    int issued[kStages] = {0, 0};
    const int bs = a.block_size;
    const int32_t* table = a.block_tables + static_cast<size_t>(s) * a.max_blocks_per_seq;
    if (lane == 0) {
      mbar_arrive_expect_tx(&b->q_full, L::kChunks * L::kTileChunk);
      for (int c = 0; c < L::kChunks; ++c)
        tma_load_3d(sm + L::kQ + c * L::kTileChunk, &tq, &b->q_full, c * 64, kvh * G, q0 + tok0);
    }
    for (int j = 0; j < nkv; ++j) {
      const int stage = j % kStages;
      if (j >= kStages && !warp_wait_or_abort(b, &b->kv_empty[stage], ((j / kStages) - 1) & 1, err)) break;
      const int first = j * kKvTile;
      const int ntok = min(kKvTile, p_max + 1 - first);
      const int nblk = (ntok + bs - 1) / bs;
      int blk = 0;
      bool ok = false;
      if (lane < nblk) {
        blk = table[first / bs + lane];
        ok = blk >= 0 && blk < a.num_blocks;
        if (!ok) atomicOr(err, PA_DEVERR_BLOCK_ID);
      }
      const unsigned okmask = __ballot_sync(0xffffffffu, ok);
      uint8_t* st = sm + L::kKV + stage * L::kStage;
      if (lane == 0) mbar_arrive_expect_tx(&b->kv_full[stage], __popc(okmask) * bs * 128 * L::kChunks * 2);
      __syncwarp();
      if (ok) {
        for (int c = 0; c < L::kChunks; ++c) {
          const uint32_t off = c * (kKvTile * 128) + lane * bs * 128;
          tma_load_4d(st + L::kK + off, &tk, &b->kv_full[stage], c * 64, 0, kvh, blk);
          tma_load_4d(st + L::kV + off, &tv, &b->kv_full[stage], c * 64, 0, kvh, blk);
        }
      }
      ++issued[stage];
    }
    // Wind-down: the last load issued into each stage has landed (immediate unless the CTA aborted).
    for (int i = 0; i < kStages; ++i)
      if (issued[i] > 0) mbar_wait(&b->kv_full[i], (issued[i] - 1) & 1, err);
  } else if (warp == 1) {
    // ================================ MMA issuer ================================
    if (lane == 0) {
      constexpr uint32_t idesc_s = mma_idesc_f16<T>(kRows, kKvTile, false);
      constexpr uint32_t idesc_o = mma_idesc_f16<T>(kRows, D, true);
      const uint32_t q_addr = smem_u32(sm + L::kQ), p_addr = smem_u32(sm + L::kP);
      bool ok = wait_or_abort(b, &b->q_full, 0, err);
      for (int j = 0; ok && j < nkv; ++j) {
        const int stage = j % kStages;
        const uint32_t k_addr = smem_u32(sm + L::kKV + stage * L::kStage + L::kK);
        const uint32_t v_addr = smem_u32(sm + L::kKV + stage * L::kStage + L::kV);
        if (!(ok = wait_or_abort(b, &b->kv_full[stage], (j / kStages) & 1, err))) break;
        tc_fence_after();
#pragma unroll
        for (int k = 0; k < D / 16; ++k) {  // S = Q K^T over d in steps of 16
          const uint32_t qo = (k >> 2) * L::kTileChunk + (k & 3) * 32;
          const uint32_t ko = (k >> 2) * (kKvTile * 128) + (k & 3) * 32;
          mma_f16_ss(tmem + kTmemS, smem_desc_sw128(q_addr + qo, 16, 1024), smem_desc_sw128(k_addr + ko, 16, 1024),
                     idesc_s, k > 0);
        }
        mma_commit(&b->s_full);
        if (!(ok = wait_or_abort(b, &b->p_full, j & 1, err))) break;
        if (j > 0 && !(ok = wait_or_abort(b, &b->o_empty, (j - 1) & 1, err))) break;
        tc_fence_after();
#pragma unroll
        for (int k = 0; k < kKvTile / 16; ++k) {  // O_tile = P V over keys in steps of 16
          const uint32_t po = (k >> 2) * L::kTileChunk + (k & 3) * 32;
          const uint32_t vo = k * 16 * 128;
          mma_f16_ss(tmem + kTmemO, smem_desc_sw128(p_addr + po, 16, 1024),
                     smem_desc_sw128(v_addr + vo, kKvTile * 128, 1024), idesc_o, k > 0);
        }
        mma_commit(&b->o_full);
        mma_commit(&b->kv_empty[stage]);
      }
      // Wind-down: every MMA issued above has completed before TMEM can be freed.
      mma_commit(&b->mma_done);
      mbar_wait(&b->mma_done, 0, err);
    }
    __syncwarp();
  } else if (warp >= 4) {
    // ================================ softmax / epilogue ================================
    const int r = threadIdx.x - 128;                // row == TMEM lane
    const int tok = tok0 + r / G;
    const bool row_valid = tok < n;
    const int pos = ctx - n + min(tok, n - 1);      // rows past the chunk reuse its last position
    const uint32_t t_lane = tmem + (static_cast<uint32_t>(r & ~31) << 16);
    const float sl2 = a.scale_log2;
    float o[D];
#pragma unroll
    for (int i = 0; i < D; ++i) o[i] = 0.f;
    float m = -INFINITY, l = 0.f;
    bool ok = true;
    for (int j = 0; j < nkv; ++j) {
      if (!(ok = warp_wait_or_abort(b, &b->s_full, j & 1, err))) break;
      tc_fence_after();
      const int base = j * kKvTile;
      // Pass 1: the row maximum over the keys this row may see.
      float mx = -INFINITY;
#pragma unroll 1
      for (int c = 0; c < kKvTile / 32; ++c) {
        uint32_t v[32];
        tmem_ld32(t_lane + kTmemS + 32 * c, v);
        tmem_wait_ld(v);
#pragma unroll
        for (int i = 0; i < 32; ++i)
          if (base + 32 * c + i <= pos) mx = fmaxf(mx, __uint_as_float(v[i]));
      }
      const float m_new = fmaxf(m, mx * sl2);
      const float alpha = ex2(m - m_new);           // 0 on the first tile (m = -inf)
      // The last tile holds keys past the tile's last needed key (unloaded or past the context):
      // zero those V rows so that 0 * (stale or NaN) cannot reach the PV product.
      if (j == nkv - 1) {
        const int cut = p_max + 1 - base;
        if (cut < kKvTile) {
          const int stage = j % kStages;
          if (!(ok = warp_wait_or_abort(b, &b->kv_full[stage], (j / kStages) & 1, err))) break;
          uint8_t* vb = sm + L::kKV + stage * L::kStage + L::kV;
          const int units = (kKvTile - cut) * 8;
          for (int c = 0; c < L::kChunks; ++c)
            for (int u = r; u < units; u += kRows)
              *reinterpret_cast<uint4*>(vb + c * (kKvTile * 128) + cut * 128 + u * 16) = make_uint4(0, 0, 0, 0);
        }
      }
      // Pass 2: P = exp2(S * scale * log2e - m), rounded to 16 bits; the sum uses the rounded values.
      float lsum = 0.f;
#pragma unroll 1
      for (int c = 0; c < kKvTile / 32; ++c) {
        uint32_t v[32];
        tmem_ld32(t_lane + kTmemS + 32 * c, v);
        tmem_wait_ld(v);
        uint32_t w[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const int t = base + 32 * c + 2 * i;
          const float p0 = (t <= pos) ? ex2(fmaf(__uint_as_float(v[2 * i]), sl2, -m_new)) : 0.f;
          const float p1 = (t + 1 <= pos) ? ex2(fmaf(__uint_as_float(v[2 * i + 1]), sl2, -m_new)) : 0.f;
          w[i] = pack_pair<T>(p0, p1);
          const float2 back = unpack_pair<T>(w[i]);
          lsum += back.x + back.y;
        }
        uint8_t* prow = sm + L::kP + (c >> 1) * L::kTileChunk + r * 128;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int unit = ((c & 1) * 4 + q) ^ (r & 7);
          *reinterpret_cast<uint4*>(prow + unit * 16) = make_uint4(w[4 * q], w[4 * q + 1], w[4 * q + 2], w[4 * q + 3]);
        }
      }
      l = l * alpha + lsum;
      m = m_new;
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(&b->p_full);
      if (!(ok = warp_wait_or_abort(b, &b->o_full, j & 1, err))) break;
      tc_fence_after();
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        uint32_t v[32];
        tmem_ld32(t_lane + kTmemO + 32 * c, v);
        tmem_wait_ld(v);
#pragma unroll
        for (int i = 0; i < 32; ++i) o[32 * c + i] = fmaf(o[32 * c + i], alpha, __uint_as_float(v[i]));
      }
      tc_fence_before();
      mbar_arrive(&b->o_empty);
    }
    if (ok && row_valid) {
      const float inv = 1.f / l;
      T* dst = static_cast<T*>(a.out) + (static_cast<size_t>(q0 + tok) * a.num_heads + kvh * G + r % G) * D;
#pragma unroll
      for (int i = 0; i < D; i += 8)
        *reinterpret_cast<uint4*>(dst + i) =
            make_uint4(pack_pair<T>(o[i] * inv, o[i + 1] * inv), pack_pair<T>(o[i + 2] * inv, o[i + 3] * inv),
                       pack_pair<T>(o[i + 4] * inv, o[i + 5] * inv), pack_pair<T>(o[i + 6] * inv, o[i + 7] * inv));
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
