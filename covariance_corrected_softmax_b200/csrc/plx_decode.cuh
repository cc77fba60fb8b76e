// plx_decode.cuh -- single-token Parallax decode over a KV cache (sm_100a).
//
// Operator (page 1 "Parallax: Parameterized Local Linear Attention Gives
// Transformers a 'Second Eye'", section 1.3; page 3 "Parallax keeps softmax,
// adds covariance correction branch"): for query head h of batch b,
//
//   out = o_SA - Sigma_KV^T rho
//       = (1 + tbar) * o - u,   o = sum_j a_j v_j,  u = sum_j a_j t_j v_j,
//         t_j = rho . k_j,      tbar = sum_j a_j t_j,  a = softmax(scale q.k)
//
// The expanded form lets one pass over the cache feed both branches (page 3:
// the same KV stream is reused by the softmax and the covariance branch).
//
// Design (B200):
//  * Work is the sequence of key tiles of all (batch, kv-head, head-group)
//    segments.  A persistent grid of CTAs splits the tile sequence into equal
//    contiguous ranges (split-K with perfect balance for any mix of lengths);
//    a segment that crosses a range boundary leaves partial states that the
//    combine kernel merges with the log-sum-exp rule.
//  * One producer warp streams K and V tiles (TK keys x d) of the cache into a
//    multi-stage shared-memory ring with TMA; the cache is read exactly once.
//  * Twelve consumer warps: each half-warp owns KPH keys of a tile, 16 lanes
//    split the head dimension.  s = scale q.k and t = rho.k are partial dot
//    products (packed fp32x2 FMA), reduced by a transpose through shared
//    memory so that each lane ends up with one full score; the online softmax
//    runs on those distributed scores (m, l, z per head) with a few shuffles,
//    and the weights p and p t are broadcast back through shared memory; the
//    two accumulators o and u per head stay in registers.
#pragma once

#include "plx_device.cuh"

namespace plx {

constexpr int kDecConsumerWarps = 12;
constexpr int kDecThreads = (kDecConsumerWarps + 1) * 32;  // + producer warp
constexpr int kDecSmemBudget = 225 * 1024;
// Transpose-reduction scratch per half-warp: 16 rows of 16 partial sums padded
// to 20 floats (conflict-free 16-byte writes), and a 16-float skew between the
// two half-warps of a warp (conflict-free column reads).
constexpr int kDecRedRow = 20;
constexpr int kDecRedRegion = 16 * kDecRedRow + 16;

template <typename T, int D>
struct DecodeTile {
  static constexpr int KPH = sizeof(T) == 2 ? 4 : 2;             // keys per half-warp per tile
  static constexpr int TK = KPH * 2 * kDecConsumerWarps;         // keys per tile
  static constexpr int EPL = D / 16;                             // elements per lane per row
  static constexpr int ROW_BYTES = D * (int)sizeof(T);
  static constexpr int TILE_BYTES = TK * ROW_BYTES;              // one K (or V) tile
  static constexpr int STAGE_BYTES = 2 * TILE_BYTES;
  // room left after the merge scratch of the widest head group (2 heads)
  static constexpr int RING_BUDGET = kDecSmemBudget - 2048 -
                                     kDecConsumerWarps * 2 * (2 * D + 4) * 4 -
                                     (2 * kDecConsumerWarps * (kDecRedRegion + 16)) * 4;
  static constexpr int STAGES_RAW = RING_BUDGET / STAGE_BYTES;
  static constexpr int STAGES = STAGES_RAW > 4 ? 4 : STAGES_RAW;
  static_assert(STAGES >= 2, "decode tile too large for the stage ring");
  static_assert(EPL * sizeof(T) % 8 == 0, "lane slice must be 8-byte aligned");
  static_assert(TK % 16 == 0, "paged loads move 16-row chunks");
};

// Per-slot partial state layout (floats): header, then per head m, l, z, pad,
// o[D], u[D].
constexpr int kPartHeader = 4;  // seg id, head flag, end flag, pad (as int)
template <int D>
__host__ __device__ constexpr int part_head_floats() { return 2 * D + 4; }
template <int D>
__host__ __device__ constexpr int part_floats(int hpw) {
  return kPartHeader + hpw * part_head_floats<D>();
}
constexpr int kWsHeaderFloats = 16;  // [0] = total tiles (int), rest reserved

struct DecodeParams {
  const void* q;         // [B, Hq, D]
  const void* rho;       // [B, Hq, D]
  const int32_t* seqlens;
  void* out;             // [B, Hq, D]
  float* ws;             // workspace (partials)
  int B, Hq, Hkv, G, S_max;
  int nhg;               // head groups per kv head (G / HPW)
  float qscale;          // softmax scale * log2(e)
  int grid;              // number of persistent CTAs
  unsigned* err;         // device error word
  // Paged cache (block_table != nullptr): K and V live in pools
  // [num_pages, page_size, Hkv, D]; position j of batch b is row
  // j % page_size of page block_table[b * max_pages + j / page_size].
  const int32_t* block_table;
  int num_pages, page_size, max_pages;
  // State mode (state != nullptr): instead of out, each (b, h) row's softmax
  // state over this cache -- m (log2 units of the scaled scores), l, z, 0,
  // o[D], u[D], unnormalised -- is written to state[(b * Hq + h) * (2D + 4)].
  float* state;
};

// Tile metadata written by the producer next to each stage.
struct TileMeta {
  int b, hkv, hg, kt;
  int nvalid;            // valid keys in this tile (<= TK)
  int seg;               // global segment id
  int flags;             // bit0: first tile of the segment in this CTA
                         // bit1: last tile of the segment in this CTA
                         // bit2: the segment starts in this CTA (kt == 0 seen)
                         // bit3: the segment ends in this CTA
  int pad;
};

__device__ __forceinline__ int clamp_len(int s, int S_max) {
  return s < 0 ? 0 : (s > S_max ? S_max : s);
}

}  // namespace plx
