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
//    CTA holding its last piece merges with the log-sum-exp rule.
//  * One producer warp streams K and V tiles (TK keys x d) of the cache into a
//    multi-stage shared-memory ring with TMA; the cache is read exactly once.
//    A segment's last, partial tile is fetched in 16-row chunks, so rows past
//    the length are not read from HBM (bf16).
//  * bf16 cache: eight consumer warps, each owning 16 keys of a 128-key tile.
//    The per-key work is moved to the tensor cores so that the stream, not the
//    instruction issue, bounds the kernel: the scores s and t of the group's
//    query heads come from one mma.sync m16n8k16 chain per 8 keys, whose A
//    rows are [q_h; rho_h] and whose B operand is the K tile (ldmatrix from
//    the 128-byte-swizzled TMA layout); the online softmax runs on the
//    accumulator fragments; and o += p v, u += (p t) v come from one
//    m16n8k16 per 16 head dimensions, A = V^T (ldmatrix.trans), B = the eight
//    weight rows [p_h, p_h t] split into bf16 high and low parts (16
//    significant bits; the exact bf16 V needs no conversion).  The fragment
//    layout makes each lane compute exactly the weights its B fragment holds.
//  * fp32 cache (the correctness path): twelve consumer warps; each half-warp
//    owns KPH keys of a tile, 16 lanes split the head dimension.  s and t are
//    partial dot products (packed fp32x2 FMA), reduced by a transpose through
//    shared memory so that each lane ends up with one full score; the online
//    softmax runs on those distributed scores with a few shuffles, and the
//    weights p and p t are broadcast back through shared memory; the two
//    accumulators o and u per head stay in registers.
#pragma once

#include "plx_device.cuh"

namespace plx {

constexpr int kDecSmemBudget = 225 * 1024;
// Transpose-reduction scratch per half-warp (fp32 path): 16 rows of 16 partial
// sums padded to 20 floats (conflict-free 16-byte writes), and a 16-float skew
// between the two half-warps of a warp (conflict-free column reads).
constexpr int kDecRedRow = 20;
constexpr int kDecRedRegion = 16 * kDecRedRow + 16;
constexpr int kDecChunkRows = 16;  // rows of one chunked (tail or paged) load

template <typename T, int D>
struct DecodeTile {
  static constexpr bool MMA = sizeof(T) == 2;                    // tensor-core consumers
  static constexpr int NW = MMA ? 8 : 12;                        // consumer warps
  static constexpr int THREADS = (NW + 1) * 32;                  // + producer warp
  static constexpr int KPH = MMA ? 8 : 2;                        // keys per half-warp per tile
  static constexpr int TK = KPH * 2 * NW;                        // keys per tile
  static constexpr int EPL = D / 16;                             // elements per lane per row (fp32)
  static constexpr int ROW_BYTES = D * (int)sizeof(T);
  static constexpr int TILE_BYTES = TK * ROW_BYTES;              // one K (or V) tile
  static constexpr int STAGE_BYTES = 2 * TILE_BYTES;
  // bf16 tiles arrive as 64-column boxes in the 128-byte swizzle (the layout
  // ldmatrix reads without bank conflicts); fp32 tiles as one box of full rows
  static constexpr int CB = MMA ? D / 64 : 1;                    // column boxes per tile
  static constexpr int BOX_ROW = ROW_BYTES / CB;                 // bytes of a row in one box
  static constexpr int BOX_BYTES = TK * BOX_ROW;                 // one column box of a tile
  static constexpr int MERGE_BYTES = NW * 2 * (2 * D + 4) * 4;   // widest head group (2 heads)
  static constexpr int RED_BYTES = MMA ? 0 : (2 * NW * (kDecRedRegion + 16)) * 4;
  static constexpr int RING_BUDGET = kDecSmemBudget - 2048 - MERGE_BYTES - RED_BYTES;
  static constexpr int STAGES_RAW = RING_BUDGET / STAGE_BYTES;
  static constexpr int STAGES = STAGES_RAW > 4 ? 4 : STAGES_RAW;
  static_assert(STAGES >= 2, "decode tile too large for the stage ring");
  static_assert(EPL * sizeof(T) % 8 == 0, "lane slice must be 8-byte aligned");
  static_assert(TK % kDecChunkRows == 0, "chunked loads move 16-row pieces");
  static_assert(!MMA || BOX_ROW == 128, "swizzled boxes are 128-byte rows");
  static_assert(!MMA || BOX_BYTES % 1024 == 0, "swizzle atoms stay 1024-byte aligned");
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
constexpr int kWsHeaderFloats = 16;  // reserved

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
