// plx_prefill_bwd_tc.cu -- gradients of the Parallax prefill operator for
// bf16 inputs on the 5th-generation tensor cores (tcgen05, fp32 accumulation).
//
// Operator (page 1 "Parallax: Parameterized Local Linear Attention Gives
// Transformers a 'Second Eye'", opening formula and section 1.3; page 3
// "Parallax keeps softmax, adds covariance correction branch"), row i, keys j:
//   a_ij = softmax_j(scale q_i.k_j),  t_ij = rho_i.k_j,  tbar_i = sum_j a t,
//   out_i = sum_j a_ij c_ij v_j,  c_ij = 1 + tbar_i - t_ij.
// The pages print no gradient; with g = dLoss/dout and gv_ij = g_i.v_j:
//   go_i = g_i.o_i = sum_j a gv,   D_i = g_i.out_i + tbar_i go_i
//        = (1 + 2 tbar_i) go_i - sum_j a t gv          (row sums only)
//   dv_j = sum_i a c g_i,   dk_j = sum_i scale ds q_i + dt rho_i,
//   dq_i = scale sum_j ds k_j,   drho_i = sum_j dt k_j,
//   ds_ij = a (c gv + t go - D),   dt_ij = a (go - gv).
// Two kernels, no atomics:
//  rows  one CTA per (batch, query head, 128-row query tile), two passes over
//        the row's 64-key tiles.  Pass 1: S = Q K^T, T = R K^T, GV = G V^T;
//        thread (row, quarter) runs an online softmax over its quarter of
//        every key tile, with sum a, sum a t, sum a gv and sum a t gv; the four
//        quarters merge at the end into the row statistics (lse, tbar, go, D),
//        which go to the workspace.  Pass 2: S, T, GV again; ds and dt, as high and low
//        bf16 parts, are written over S and T in TMEM, and dQ += (scale ds) K,
//        dR += dt K accumulate in TMEM.
//  keys  one CTA per (batch, kv head, 128-key tile), over the query heads of
//        the group and their 64-row query tiles: S^T = K Q^T, T^T = K R^T,
//        GV^T = V G^T with keys in the TMEM lanes; the statistics of each
//        query column come from the rows kernel.  P' = a c, scale ds and dt
//        (high and low bf16 parts) are written over S^T, T^T and GV^T, and
//        dV += P'^T G, dK += (scale ds)^T Q + dt^T R accumulate in TMEM.
// The statistics are recomputed from the inputs in fp32 (not taken from the
// forward pass): ds = a (X - D) cancels where one key dominates a row, and
// would amplify any rounding of the normaliser.
// Per CTA: warp 0 issues the TMA loads, warp 1 (one thread) the MMAs and owns
// the TMEM columns, warps 2-17 do the elementwise work (thread = TMEM lane and
// a quarter of a tile's columns, four warps per lane quadrant) and the
// epilogue.  The products of a step are
// issued once the elementwise warps have stored their operands, and the next
// step's S/T/GV after them, so the tensor core never overwrites a column that
// is still to be read.
#include "plx_launch.h"

namespace plx {

namespace {

// Elementwise warps 2 .. 17: four per TMEM lane quadrant, each thread one
// TMEM lane and a quarter (16 columns) of every tile or step.
constexpr int kBwdEltWarps = 16;
constexpr int kBwdThreads = (2 + kBwdEltWarps) * 32;  // 576
constexpr int kBwdStages = 3;                         // ring depth of the streamed operand
constexpr int kTileM = 128;                           // TMEM lanes: rows (rows kernel) or keys
constexpr int kTileN = 64;                            // keys (rows kernel) or query rows per step

// bf16 [B, L, H, d] tile of `rows` rows and one 64-column block: rows x 128 bytes
// with the 128-byte swizzle (the layout TMA writes for box (64, 1, rows, 1)).
__host__ __device__ constexpr int blk_bytes(int rows) { return rows * 128; }

struct BwdTcParams {
  float *dq, *drho, *dk, *dv;
  float4* stats;  // [B, Hq, L]: lse (log2 units of the scaled scores), tbar, go, D
  int B, L, Hq, Hkv, G, causal;
  int units;      // rows kernel: B Hq ceil(L / 128); keys kernel: B Hkv ceil(L / 128)
  float scale;    // softmax scale
  float qscale;   // scale * log2(e)
  unsigned* err;
};

template <int D>
struct BwdCfg {
  static_assert(D == 64 || D == 128, "head dimension 64 or 128");
  static constexpr int KB = D / 64;                   // 64-column blocks
  static constexpr int BIG = KB * blk_bytes(kTileM);  // one 128-row operand (all blocks)
  static constexpr int SMALL = KB * blk_bytes(kTileN);  // one 64-row operand
  // TMEM columns: two fp32 accumulators of width D, then S, T, GV (64 each).
  static constexpr uint32_t COL_A0 = 0, COL_A1 = D;
  static constexpr uint32_t COL_S = 2 * D, COL_T = COL_S + kTileN, COL_GV = COL_T + kTileN;
  static_assert(COL_GV + kTileN <= 512, "TMEM columns");
  // S/T/GV: bf16 x bf16, both K-major, 128 x 64.  Gradient products: bf16 A
  // from TMEM x bf16 B (MN-major), 128 x D.
  static constexpr uint32_t IDESC_S = umma_idesc_f16kind(kTileM, kTileN, false, false);
  static constexpr uint32_t IDESC_G = umma_idesc_f16kind(kTileM, D, true, false);
};

// Column of the bf16 pairs of columns [16 kk, 16 kk + 16) of a 64-column S/T/GV
// block once the elementwise warps have written their operand over it: the
// thread of quarter kk writes the high bf16 parts of its 16 columns at
// packed_col(kk) and the low parts (value - high, rounded) 16 columns further
// (+kLoCols), so each half of the block holds the high parts of its two
// quarters in its first 16 columns and their low parts in the next 16.  The
// gradient products run once on each part, so the operands keep about 16
// significant bits: the fp32 gradients' own error, not bf16's.
__device__ __forceinline__ uint32_t packed_col(int kk) {
  return (uint32_t)(32 * (kk >> 1) + 8 * (kk & 1));
}
constexpr uint32_t kLoCols = 16;

// High and low bf16 pairs of (a, b): hi + lo = (a, b) to about 2^-17.
__device__ __forceinline__ void split_bf16(float a, float b, uint32_t& hi, uint32_t& lo) {
  hi = float2_to_bf16x2(a, b);
  const float2 h = bf16x2_to_float2(hi);
  lo = float2_to_bf16x2(a - h.x, b - h.y);
}

// K-major operand descriptor for k-step k (16 elements of d) of an operand of
// `rows` rows stored as KB column blocks of rows x 128 bytes.
__device__ __forceinline__ uint64_t kmajor_step(uint64_t desc, int k, int rows) {
  return desc + (uint64_t)(((k >> 2) * blk_bytes(rows) + (k & 3) * 32) >> 4);
}
// MN-major operand (K-dim = the rows of a 64-row tile) for k-step kk (16 rows).
__device__ __forceinline__ uint64_t mnmajor_step(uint64_t desc, int kk) {
  return desc + (uint64_t)((kk * 16 * 128) >> 4);
}


// The k-th unit of this CTA: rounds of gridDim.x units (heaviest first), in CTA
// order in even rounds and in reverse in odd ones, so the heavy and light ends
// of each round even out across the CTAs.  Past the last unit: -1.
__device__ __forceinline__ int cta_unit(int k, int units) {
  const long long g = gridDim.x;
  const long long u = (long long)k * g + ((k & 1) ? g - 1 - blockIdx.x : (long long)blockIdx.x);
  return u < units ? (int)u : -1;
}

// 1-D bulk copy global -> this CTA's shared memory, completing on an mbarrier
// (addresses 16-byte aligned, size a multiple of 16 bytes).
__device__ __forceinline__ void bulk_load_1d(void* dst, const void* src, uint32_t bytes,
                                             uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::
          "r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

// Lets copies already in flight land before the CTA's shared memory is released.
__device__ __forceinline__ void settle_after_abort(volatile int* abort_flag) {
  if (*abort_flag) {
    const uint64_t t0 = globaltimer_ns();
    while (globaltimer_ns() - t0 < 100000) {
    }
  }
}

// ---------------------------------------------------------------------------
// rows kernel: dq, drho and the row statistics
// ---------------------------------------------------------------------------
struct RowsBars {
  uint64_t q_full, q_empty;                              // Q, R, G of the unit
  uint64_t kv_full[kBwdStages], kv_empty[kBwdStages];    // K, V of step t
  uint64_t s_full;                                       // S, T, GV of step t computed
  uint64_t s_done;                                       // elementwise warps done with step t
  uint64_t acc_full, acc_empty;                          // dQ, dR of the unit complete / read
  uint64_t drain;
};

template <int D>
__global__ void __launch_bounds__(kBwdThreads, 1)
    plx_bwd_rows_tc_kernel(const __grid_constant__ CUtensorMap qmap,
                           const __grid_constant__ CUtensorMap rmap,
                           const __grid_constant__ CUtensorMap gmap,
                           const __grid_constant__ CUtensorMap kmap,
                           const __grid_constant__ CUtensorMap vmap, const BwdTcParams p) {
  using C = BwdCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint8_t* sQ = smem;
  uint8_t* sR = smem + C::BIG;
  uint8_t* sG = smem + 2 * C::BIG;
  uint8_t* sKV = smem + 3 * C::BIG;  // stage st: K at st * 2 SMALL, V after it
  float* xch = reinterpret_cast<float*>(sKV + kBwdStages * 2 * C::SMALL);  // [5][4][128]
  RowsBars* bars = reinterpret_cast<RowsBars*>(xch + 5 * 4 * kTileM);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (tid == 0) {
    *abort_flag = 0;
    mbar_init(&bars->q_full, 1);
    mbar_init(&bars->q_empty, 1);
    for (int s = 0; s < kBwdStages; ++s) {
      mbar_init(&bars->kv_full[s], 1);
      mbar_init(&bars->kv_empty[s], 1);
    }
    mbar_init(&bars->s_full, 1);
    mbar_init(&bars->s_done, kBwdEltWarps);
    mbar_init(&bars->acc_full, 1);
    mbar_init(&bars->acc_empty, kBwdEltWarps);
    mbar_init(&bars->drain, 1);
    fence_mbarrier_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *tmem_slot;
  const int nqt = (p.L + kTileM - 1) / kTileM, nkt = (p.L + kTileN - 1) / kTileN;
  // unit u: query tile mt of (b, h), heaviest causal tiles first; n key tiles
  auto unit_of = [&](int u, int& b, int& h, int& mt, int& n) {
    const int bh = p.B * p.Hq;
    mt = nqt - 1 - u / bh;
    const int r = u % bh;
    b = r / p.Hq;
    h = r % p.Hq;
    n = p.causal ? min(nkt, (mt * kTileM + kTileM - 1) / kTileN + 1) : nkt;
  };

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      tma_prefetch_desc(&qmap);
      tma_prefetch_desc(&rmap);
      tma_prefetch_desc(&gmap);
      tma_prefetch_desc(&kmap);
      tma_prefetch_desc(&vmap);
      int t = 0, ku = 0;
      bool ok = true;
      for (int k = 0, u; ok && (u = cta_unit(k, p.units)) >= 0; ++k) {
        int b, h, mt, n;
        unit_of(u, b, h, mt, n);
        const int hk = h / p.G;
        if (ku > 0 && !mbar_wait(&bars->q_empty, (ku - 1) & 1, abort_flag, p.err)) break;
        mbar_arrive_expect_tx(&bars->q_full, 3 * C::BIG);
        for (int kb = 0; kb < C::KB; ++kb) {
          tma_load_4d(sQ + kb * blk_bytes(kTileM), &qmap, &bars->q_full, kb * 64, h, mt * kTileM, b);
          tma_load_4d(sR + kb * blk_bytes(kTileM), &rmap, &bars->q_full, kb * 64, h, mt * kTileM, b);
          tma_load_4d(sG + kb * blk_bytes(kTileM), &gmap, &bars->q_full, kb * 64, h, mt * kTileM, b);
        }
        // two passes over the unit's key tiles
        for (int s2 = 0; ok && s2 < 2 * n; ++s2, ++t) {
          const int j = s2 % n, st = t % kBwdStages;
          if (t >= kBwdStages && !mbar_wait(&bars->kv_empty[st], ((t / kBwdStages) - 1) & 1,
                                            abort_flag, p.err)) {
            ok = false;
            break;
          }
          uint8_t* dst = sKV + st * 2 * C::SMALL;
          mbar_arrive_expect_tx(&bars->kv_full[st], 2 * C::SMALL);
          for (int kb = 0; kb < C::KB; ++kb) {
            tma_load_4d(dst + kb * blk_bytes(kTileN), &kmap, &bars->kv_full[st], kb * 64, hk,
                        j * kTileN, b);
            tma_load_4d(dst + C::SMALL + kb * blk_bytes(kTileN), &vmap, &bars->kv_full[st],
                        kb * 64, hk, j * kTileN, b);
          }
        }
        ++ku;
      }
      settle_after_abort(abort_flag);
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint64_t dq = smem_desc_sw128(smem_u32(sQ), 16, 1024);
      const uint64_t dr = smem_desc_sw128(smem_u32(sR), 16, 1024);
      const uint64_t dg = smem_desc_sw128(smem_u32(sG), 16, 1024);
      int t = 0, ku = 0;
      bool ok = true;
      for (int k = 0, u; ok && (u = cta_unit(k, p.units)) >= 0; ++k) {
        int b, h, mt, n;
        unit_of(u, b, h, mt, n);
        if (!mbar_wait(&bars->q_full, ku & 1, abort_flag, p.err)) break;
        for (int s2 = 0; s2 < 2 * n; ++s2, ++t) {
          const int j = s2 % n, st = t % kBwdStages;
          const bool grad = s2 >= n;  // second pass
          if (!mbar_wait(&bars->kv_full[st], (t / kBwdStages) & 1, abort_flag, p.err)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t k_off = (uint32_t)(st * 2 * C::SMALL);
          const uint64_t dk = smem_desc_sw128(smem_u32(sKV + k_off), 16, 1024);
          const uint64_t dv = smem_desc_sw128(smem_u32(sKV + k_off + C::SMALL), 16, 1024);
#pragma unroll
          for (int k = 0; k < D / 16; ++k)
            umma_ss(tbase + C::COL_S, kmajor_step(dq, k, kTileM), kmajor_step(dk, k, kTileN),
                    C::IDESC_S, k > 0 ? 1u : 0u);
#pragma unroll
          for (int k = 0; k < D / 16; ++k)
            umma_ss(tbase + C::COL_T, kmajor_step(dr, k, kTileM), kmajor_step(dk, k, kTileN),
                    C::IDESC_S, k > 0 ? 1u : 0u);
#pragma unroll
          for (int k = 0; k < D / 16; ++k)
            umma_ss(tbase + C::COL_GV, kmajor_step(dg, k, kTileM), kmajor_step(dv, k, kTileN),
                    C::IDESC_S, k > 0 ? 1u : 0u);
          umma_commit(&bars->s_full);
          // the elementwise warps have read S, T, GV (and, in the second pass,
          // written scale ds and dt over S and T)
          if (!mbar_wait(&bars->s_done, t & 1, abort_flag, p.err)) {
            ok = false;
            break;
          }
          tc_fence_after();
          if (grad) {
            if (j == 0 && ku > 0 && !mbar_wait(&bars->acc_empty, (ku - 1) & 1, abort_flag, p.err)) {
              ok = false;
              break;
            }
            tc_fence_after();
            // K as the MN-major B operand: K-dim = the tile's 64 keys, N = d
            const uint64_t dkm = smem_desc_sw128(smem_u32(sKV + k_off), blk_bytes(kTileN), 1024);
#pragma unroll
            for (int kk = 0; kk < kTileN / 16; ++kk) {
              umma_ts(tbase + C::COL_A0, tbase + C::COL_S + packed_col(kk), mnmajor_step(dkm, kk),
                      C::IDESC_G, (j > 0 || kk > 0) ? 1u : 0u);
              umma_ts(tbase + C::COL_A0, tbase + C::COL_S + packed_col(kk) + kLoCols,
                      mnmajor_step(dkm, kk), C::IDESC_G, 1u);
            }
#pragma unroll
            for (int kk = 0; kk < kTileN / 16; ++kk) {
              umma_ts(tbase + C::COL_A1, tbase + C::COL_T + packed_col(kk), mnmajor_step(dkm, kk),
                      C::IDESC_G, (j > 0 || kk > 0) ? 1u : 0u);
              umma_ts(tbase + C::COL_A1, tbase + C::COL_T + packed_col(kk) + kLoCols,
                      mnmajor_step(dkm, kk), C::IDESC_G, 1u);
            }
          }
          umma_commit(&bars->kv_empty[st]);
        }
        if (!ok) break;
        umma_commit(&bars->q_empty);
        umma_commit(&bars->acc_full);
        ++ku;
      }
      // every MMA has completed before the columns are released
      umma_commit(&bars->drain);
      volatile int never = 0;
      mbar_wait(&bars->drain, 0, &never, p.err);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ elementwise + epilogue
    const int quarter = (warp - 2) >> 2;  // which 16 columns of each tile
    const int qd = warp & 3;              // TMEM lane quadrant
    const int r = qd * 32 + lane;         // row of the query tile
    const uint32_t lane_addr = tbase + ((uint32_t)(qd * 32) << 16);
    const uint32_t my = (uint32_t)(quarter * 16);
    const uint32_t hi_col = packed_col(quarter), lo_col = hi_col + kLoCols;
    const float qs = p.qscale;
    int t = 0, ku = 0;
    for (int k = 0, u; (u = cta_unit(k, p.units)) >= 0; ++k) {
      int b, h, mt, n;
      unit_of(u, b, h, mt, n);
      const int i = mt * kTileM + r;
      const int lim = p.causal ? i : p.L - 1;  // last key the row sees
      // pass 1: online softmax over this quarter of every key tile (log2 units)
      float m = -INFINITY, l = 0.f, st_ = 0.f, sg = 0.f, stg = 0.f;
      for (int j = 0; j < n; ++j, ++t) {
        mbar_wait(&bars->s_full, t & 1, abort_flag, p.err);
        tc_fence_after();
        uint32_t sv[16], tv[16], gv[16];
        tmem_ld2x16_sync(lane_addr + C::COL_S + my, lane_addr + C::COL_T + my, sv, tv);
        tmem_ld16_sync(lane_addr + C::COL_GV + my, gv);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars->s_done);
        const int nvis = max(0, min(16, lim - (j * kTileN + quarter * 16) + 1));
        float x[16];
        float mx = -INFINITY;
#pragma unroll
        for (int c = 0; c < 16; ++c) {
          x[c] = __uint_as_float(sv[c]) * qs;
          if (c < nvis) mx = fmaxf(mx, x[c]);
        }
        if (mx > m) {
          const float f = m == -INFINITY ? 0.f : exp2f(m - mx);
          l *= f;
          st_ *= f;
          sg *= f;
          stg *= f;
          m = mx;
        }
#pragma unroll
        for (int c = 0; c < 16; ++c) {
          const float e = c < nvis ? exp2f(x[c] - m) : 0.f;
          const float tt = __uint_as_float(tv[c]), g_ = __uint_as_float(gv[c]);
          l += e;
          st_ = fmaf(e, tt, st_);
          sg = fmaf(e, g_, sg);
          stg = fmaf(e * tt, g_, stg);
        }
      }
      // merge the four quarters of the row
      {
        float* w = xch + quarter * kTileM + r;
        w[0] = m;
        w[4 * kTileM] = l;
        w[8 * kTileM] = st_;
        w[12 * kTileM] = sg;
        w[16 * kTileM] = stg;
      }
      named_bar_sync(1 + qd, 128);
      float mq[4], M = -INFINITY;
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        mq[q] = xch[q * kTileM + r];
        M = fmaxf(M, mq[q]);
      }
      float L_ = 0.f, st_all = 0.f, sg_all = 0.f, stg_all = 0.f;
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const float f = mq[q] == -INFINITY ? 0.f : exp2f(mq[q] - M);
        const float* o = xch + q * kTileM + r;
        L_ = fmaf(o[4 * kTileM], f, L_);
        st_all = fmaf(o[8 * kTileM], f, st_all);
        sg_all = fmaf(o[12 * kTileM], f, sg_all);
        stg_all = fmaf(o[16 * kTileM], f, stg_all);
      }
      const float inv = 1.f / L_;
      const float lse2 = M + log2f(L_);
      const float tbar = st_all * inv;
      const float go = sg_all * inv;
      const float wsum = stg_all * inv;
      const float Dr = (1.f + 2.f * tbar) * go - wsum;
      if (quarter == 0 && i < p.L)
        p.stats[((size_t)b * p.Hq + h) * p.L + i] = make_float4(lse2, tbar, go, Dr);
      // pass 2: scale ds and dt, rounded to bf16, over S and T
      for (int j = 0; j < n; ++j, ++t) {
        mbar_wait(&bars->s_full, t & 1, abort_flag, p.err);
        tc_fence_after();
        uint32_t sv[16], tv[16], gv[16];
        tmem_ld2x16_sync(lane_addr + C::COL_S + my, lane_addr + C::COL_T + my, sv, tv);
        tmem_ld16_sync(lane_addr + C::COL_GV + my, gv);
        const int nvis = max(0, min(16, lim - (j * kTileN + quarter * 16) + 1));
        uint32_t pds[2][8], pdt[2][8];  // [0]: high parts, [1]: low parts
#pragma unroll
        for (int c = 0; c < 16; c += 2) {
          float ds2[2], dt2[2];
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const float a =
                c + e < nvis ? exp2f(fmaf(__uint_as_float(sv[c + e]), qs, -lse2)) : 0.f;
            const float tt = __uint_as_float(tv[c + e]), g_ = __uint_as_float(gv[c + e]);
            const float cc = 1.f + tbar - tt;
            dt2[e] = a * (go - g_);
            ds2[e] = p.scale * a * fmaf(cc, g_, fmaf(tt, go, -Dr));
          }
          split_bf16(ds2[0], ds2[1], pds[0][c >> 1], pds[1][c >> 1]);
          split_bf16(dt2[0], dt2[1], pdt[0][c >> 1], pdt[1][c >> 1]);
        }
        tmem_st8(lane_addr + C::COL_S + hi_col, pds[0]);
        tmem_st8(lane_addr + C::COL_S + lo_col, pds[1]);
        tmem_st8(lane_addr + C::COL_T + hi_col, pdt[0]);
        tmem_st8(lane_addr + C::COL_T + lo_col, pdt[1]);
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars->s_done);
      }
      // epilogue: dQ, dR of this row (this quarter's columns), fp32
      mbar_wait(&bars->acc_full, ku & 1, abort_flag, p.err);
      tc_fence_after();
      const size_t ro = (((size_t)b * p.L + i) * p.Hq + h) * D;
#pragma unroll 1
      for (int cc = quarter * (D / 4); cc < (quarter + 1) * (D / 4); cc += 16) {
        uint32_t a0[16], a1[16];
        tmem_ld2x16_sync(lane_addr + C::COL_A0 + cc, lane_addr + C::COL_A1 + cc, a0, a1);
        if (i < p.L) {
          float4* d0 = reinterpret_cast<float4*>(p.dq + ro + cc);
          float4* d1 = reinterpret_cast<float4*>(p.drho + ro + cc);
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            d0[q] = make_float4(__uint_as_float(a0[4 * q]), __uint_as_float(a0[4 * q + 1]),
                                __uint_as_float(a0[4 * q + 2]), __uint_as_float(a0[4 * q + 3]));
            d1[q] = make_float4(__uint_as_float(a1[4 * q]), __uint_as_float(a1[4 * q + 1]),
                                __uint_as_float(a1[4 * q + 2]), __uint_as_float(a1[4 * q + 3]));
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->acc_empty);
      ++ku;
    }
  }

  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tbase, 512);
  }
}

// ---------------------------------------------------------------------------
// keys kernel: dk, dv
// ---------------------------------------------------------------------------
struct KeysBars {
  uint64_t kv_full, kv_empty;                            // K, V of the unit
  uint64_t q_full[kBwdStages], q_empty[kBwdStages];      // Q, R, G, statistics of step t
  uint64_t s_full;                                       // S^T, T^T, GV^T of step t computed
  uint64_t s_done;                                       // elementwise warps done with step t
  uint64_t acc_full, acc_empty;                          // dV, dK of the unit complete / read
  uint64_t drain;
};

template <int D>
__global__ void __launch_bounds__(kBwdThreads, 1)
    plx_bwd_keys_tc_kernel(const __grid_constant__ CUtensorMap qmap,
                           const __grid_constant__ CUtensorMap rmap,
                           const __grid_constant__ CUtensorMap gmap,
                           const __grid_constant__ CUtensorMap kmap,
                           const __grid_constant__ CUtensorMap vmap, const BwdTcParams p) {
  using C = BwdCfg<D>;
  constexpr int STAGE = 3 * C::SMALL + kTileN * 16;  // Q, R, G tiles and 64 float4 statistics
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint8_t* sK = smem;
  uint8_t* sV = smem + C::BIG;
  uint8_t* sRing = smem + 2 * C::BIG;  // stage st at st * STAGE: Q, R, G, statistics
  KeysBars* bars = reinterpret_cast<KeysBars*>(sRing + kBwdStages * STAGE);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (tid == 0) {
    *abort_flag = 0;
    mbar_init(&bars->kv_full, 1);
    mbar_init(&bars->kv_empty, 1);
    for (int s = 0; s < kBwdStages; ++s) {
      mbar_init(&bars->q_full[s], 1);
      mbar_init(&bars->q_empty[s], 1);
    }
    mbar_init(&bars->s_full, 1);
    mbar_init(&bars->s_done, kBwdEltWarps);
    mbar_init(&bars->acc_full, 1);
    mbar_init(&bars->acc_empty, kBwdEltWarps);
    mbar_init(&bars->drain, 1);
    fence_mbarrier_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *tmem_slot;
  const int nq = (p.L + kTileN - 1) / kTileN;
  // unit u: key tile kt of (b, hk), the tiles with the most queries first; its
  // steps run over the group's query heads and, for each, the query tiles
  // from q0 (causal: the first that reaches the key tile) to the last
  auto unit_of = [&](int u, int& b, int& hk, int& kt, int& q0) {
    const int bk = p.B * p.Hkv;
    kt = u / bk;
    const int r = u % bk;
    b = r / p.Hkv;
    hk = r % p.Hkv;
    q0 = p.causal ? (kt * kTileM) / kTileN : 0;
  };

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      tma_prefetch_desc(&qmap);
      tma_prefetch_desc(&rmap);
      tma_prefetch_desc(&gmap);
      tma_prefetch_desc(&kmap);
      tma_prefetch_desc(&vmap);
      int t = 0, ku = 0;
      bool ok = true;
      for (int k = 0, u; ok && (u = cta_unit(k, p.units)) >= 0; ++k) {
        int b, hk, kt, q0;
        unit_of(u, b, hk, kt, q0);
        if (ku > 0 && !mbar_wait(&bars->kv_empty, (ku - 1) & 1, abort_flag, p.err)) break;
        mbar_arrive_expect_tx(&bars->kv_full, 2 * C::BIG);
        for (int kb = 0; kb < C::KB; ++kb) {
          tma_load_4d(sK + kb * blk_bytes(kTileM), &kmap, &bars->kv_full, kb * 64, hk,
                      kt * kTileM, b);
          tma_load_4d(sV + kb * blk_bytes(kTileM), &vmap, &bars->kv_full, kb * 64, hk,
                      kt * kTileM, b);
        }
        const int steps = p.G * (nq - q0);
        for (int s2 = 0; s2 < steps; ++s2, ++t) {
          const int h = hk * p.G + s2 / (nq - q0), qt = q0 + s2 % (nq - q0);
          const int st = t % kBwdStages;
          if (t >= kBwdStages && !mbar_wait(&bars->q_empty[st], ((t / kBwdStages) - 1) & 1,
                                            abort_flag, p.err)) {
            ok = false;
            break;
          }
          uint8_t* dst = sRing + st * STAGE;
          const int rows = min(kTileN, p.L - qt * kTileN);  // statistics rows that exist
          mbar_arrive_expect_tx(&bars->q_full[st], 3 * C::SMALL + rows * 16);
          for (int kb = 0; kb < C::KB; ++kb) {
            tma_load_4d(dst + kb * blk_bytes(kTileN), &qmap, &bars->q_full[st], kb * 64, h,
                        qt * kTileN, b);
            tma_load_4d(dst + C::SMALL + kb * blk_bytes(kTileN), &rmap, &bars->q_full[st],
                        kb * 64, h, qt * kTileN, b);
            tma_load_4d(dst + 2 * C::SMALL + kb * blk_bytes(kTileN), &gmap, &bars->q_full[st],
                        kb * 64, h, qt * kTileN, b);
          }
          bulk_load_1d(dst + 3 * C::SMALL,
                       p.stats + ((size_t)b * p.Hq + h) * p.L + (size_t)qt * kTileN,
                       (uint32_t)(rows * 16), &bars->q_full[st]);
        }
        ++ku;
      }
      settle_after_abort(abort_flag);
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint64_t dk = smem_desc_sw128(smem_u32(sK), 16, 1024);
      const uint64_t dv = smem_desc_sw128(smem_u32(sV), 16, 1024);
      int t = 0, ku = 0;
      bool ok = true;
      for (int k = 0, u; ok && (u = cta_unit(k, p.units)) >= 0; ++k) {
        int b, hk, kt, q0;
        unit_of(u, b, hk, kt, q0);
        if (!mbar_wait(&bars->kv_full, ku & 1, abort_flag, p.err)) break;
        const int steps = p.G * (nq - q0);
        for (int s2 = 0; s2 < steps; ++s2, ++t) {
          const int st = t % kBwdStages;
          if (!mbar_wait(&bars->q_full[st], (t / kBwdStages) & 1, abort_flag, p.err)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint8_t* ring = sRing + st * STAGE;
          const uint64_t bq = smem_desc_sw128(smem_u32(ring), 16, 1024);
          const uint64_t br = smem_desc_sw128(smem_u32(ring + C::SMALL), 16, 1024);
          const uint64_t bg = smem_desc_sw128(smem_u32(ring + 2 * C::SMALL), 16, 1024);
#pragma unroll
          for (int k = 0; k < D / 16; ++k)
            umma_ss(tbase + C::COL_S, kmajor_step(dk, k, kTileM), kmajor_step(bq, k, kTileN),
                    C::IDESC_S, k > 0 ? 1u : 0u);
#pragma unroll
          for (int k = 0; k < D / 16; ++k)
            umma_ss(tbase + C::COL_T, kmajor_step(dk, k, kTileM), kmajor_step(br, k, kTileN),
                    C::IDESC_S, k > 0 ? 1u : 0u);
#pragma unroll
          for (int k = 0; k < D / 16; ++k)
            umma_ss(tbase + C::COL_GV, kmajor_step(dv, k, kTileM), kmajor_step(bg, k, kTileN),
                    C::IDESC_S, k > 0 ? 1u : 0u);
          umma_commit(&bars->s_full);
          // the elementwise warps have written P', scale ds and dt over S^T,
          // T^T and GV^T
          if (!mbar_wait(&bars->s_done, t & 1, abort_flag, p.err)) {
            ok = false;
            break;
          }
          if (s2 == 0 && ku > 0 && !mbar_wait(&bars->acc_empty, (ku - 1) & 1, abort_flag, p.err)) {
            ok = false;
            break;
          }
          tc_fence_after();
          // Q, R, G as MN-major B operands: K-dim = the step's 64 query rows, N = d
          const uint64_t mq = smem_desc_sw128(smem_u32(ring), blk_bytes(kTileN), 1024);
          const uint64_t mr = smem_desc_sw128(smem_u32(ring + C::SMALL), blk_bytes(kTileN), 1024);
          const uint64_t mg =
              smem_desc_sw128(smem_u32(ring + 2 * C::SMALL), blk_bytes(kTileN), 1024);
#pragma unroll
          for (int kk = 0; kk < kTileN / 16; ++kk) {
            umma_ts(tbase + C::COL_A0, tbase + C::COL_S + packed_col(kk), mnmajor_step(mg, kk),
                    C::IDESC_G, (s2 > 0 || kk > 0) ? 1u : 0u);
            umma_ts(tbase + C::COL_A0, tbase + C::COL_S + packed_col(kk) + kLoCols,
                    mnmajor_step(mg, kk), C::IDESC_G, 1u);
          }
#pragma unroll
          for (int kk = 0; kk < kTileN / 16; ++kk) {
            umma_ts(tbase + C::COL_A1, tbase + C::COL_T + packed_col(kk), mnmajor_step(mq, kk),
                    C::IDESC_G, (s2 > 0 || kk > 0) ? 1u : 0u);
            umma_ts(tbase + C::COL_A1, tbase + C::COL_T + packed_col(kk) + kLoCols,
                    mnmajor_step(mq, kk), C::IDESC_G, 1u);
          }
#pragma unroll
          for (int kk = 0; kk < kTileN / 16; ++kk) {
            umma_ts(tbase + C::COL_A1, tbase + C::COL_GV + packed_col(kk), mnmajor_step(mr, kk),
                    C::IDESC_G, 1u);
            umma_ts(tbase + C::COL_A1, tbase + C::COL_GV + packed_col(kk) + kLoCols,
                    mnmajor_step(mr, kk), C::IDESC_G, 1u);
          }
          umma_commit(&bars->q_empty[st]);
        }
        if (!ok) break;
        umma_commit(&bars->kv_empty);
        umma_commit(&bars->acc_full);
        ++ku;
      }
      umma_commit(&bars->drain);
      volatile int never = 0;
      mbar_wait(&bars->drain, 0, &never, p.err);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ elementwise + epilogue
    // sixteen warps: four per TMEM lane quadrant, each thread one key and a
    // quarter (16 query columns) of every step, which is one k step of the
    // gradient products
    const int quarter = (warp - 2) >> 2;  // which 16 query columns of each step
    const int qd = warp & 3;              // TMEM lane quadrant
    const int r = qd * 32 + lane;         // key of the key tile
    const uint32_t lane_addr = tbase + ((uint32_t)(qd * 32) << 16);
    const uint32_t my = (uint32_t)(quarter * 16);
    const uint32_t hi_col = packed_col(quarter), lo_col = hi_col + kLoCols;
    const float qs = p.qscale;
    int t = 0, ku = 0;
    for (int k = 0, u; (u = cta_unit(k, p.units)) >= 0; ++k) {
      int b, hk, kt, q0;
      unit_of(u, b, hk, kt, q0);
      const int j = kt * kTileM + r;  // this thread's key
      const int steps = p.G * (nq - q0);
      for (int s2 = 0; s2 < steps; ++s2, ++t) {
        const int qt = q0 + s2 % (nq - q0);
        const int st = t % kBwdStages;
        // the statistics were written by the bulk copy: wait for it as well
        mbar_wait(&bars->q_full[st], (t / kBwdStages) & 1, abort_flag, p.err);
        mbar_wait(&bars->s_full, t & 1, abort_flag, p.err);
        tc_fence_after();
        uint32_t sv[16], tv[16], gv[16];
        tmem_ld2x16_sync(lane_addr + C::COL_S + my, lane_addr + C::COL_T + my, sv, tv);
        tmem_ld16_sync(lane_addr + C::COL_GV + my, gv);
        const float4* stat =
            reinterpret_cast<const float4*>(sRing + st * STAGE + 3 * C::SMALL) + quarter * 16;
        const int i0 = qt * kTileN + quarter * 16;  // first query column of this quarter
        uint32_t pp[2][8], pds[2][8], pdt[2][8];  // [0]: high parts, [1]: low parts
#pragma unroll
        for (int c = 0; c < 16; c += 2) {
          float pv2[2], ds2[2], dt2[2];
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const int i = i0 + c + e;
            const bool vis = i < p.L && j < p.L && (!p.causal || i >= j);
            // lse (log2), tbar, go, D of query i; a query past L has no
            // statistics (its ring slot holds whatever was there), and a zero
            // weight must not meet a non-finite value
            const float4 w = vis ? stat[c + e] : make_float4(0.f, 0.f, 0.f, 0.f);
            const float a = vis ? exp2f(fmaf(__uint_as_float(sv[c + e]), qs, -w.x)) : 0.f;
            const float tt = __uint_as_float(tv[c + e]), g_ = __uint_as_float(gv[c + e]);
            const float cc = 1.f + w.y - tt;
            pv2[e] = a * cc;
            dt2[e] = a * (w.z - g_);
            ds2[e] = p.scale * a * fmaf(cc, g_, fmaf(tt, w.z, -w.w));
          }
          split_bf16(pv2[0], pv2[1], pp[0][c >> 1], pp[1][c >> 1]);
          split_bf16(ds2[0], ds2[1], pds[0][c >> 1], pds[1][c >> 1]);
          split_bf16(dt2[0], dt2[1], pdt[0][c >> 1], pdt[1][c >> 1]);
        }
        tmem_st8(lane_addr + C::COL_S + hi_col, pp[0]);
        tmem_st8(lane_addr + C::COL_S + lo_col, pp[1]);
        tmem_st8(lane_addr + C::COL_T + hi_col, pds[0]);
        tmem_st8(lane_addr + C::COL_T + lo_col, pds[1]);
        tmem_st8(lane_addr + C::COL_GV + hi_col, pdt[0]);
        tmem_st8(lane_addr + C::COL_GV + lo_col, pdt[1]);
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars->s_done);
      }
      // epilogue: dV, dK of this key (this quarter's columns), fp32
      mbar_wait(&bars->acc_full, ku & 1, abort_flag, p.err);
      tc_fence_after();
      const size_t ro = (((size_t)b * p.L + j) * p.Hkv + hk) * D;
#pragma unroll 1
      for (int cc = quarter * (D / 4); cc < (quarter + 1) * (D / 4); cc += 16) {
        uint32_t a0[16], a1[16];
        tmem_ld2x16_sync(lane_addr + C::COL_A0 + cc, lane_addr + C::COL_A1 + cc, a0, a1);
        if (j < p.L) {
          float4* d0 = reinterpret_cast<float4*>(p.dv + ro + cc);
          float4* d1 = reinterpret_cast<float4*>(p.dk + ro + cc);
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            d0[q] = make_float4(__uint_as_float(a0[4 * q]), __uint_as_float(a0[4 * q + 1]),
                                __uint_as_float(a0[4 * q + 2]), __uint_as_float(a0[4 * q + 3]));
            d1[q] = make_float4(__uint_as_float(a1[4 * q]), __uint_as_float(a1[4 * q + 1]),
                                __uint_as_float(a1[4 * q + 2]), __uint_as_float(a1[4 * q + 3]));
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->acc_empty);
      ++ku;
    }
  }

  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tbase, 512);
  }
}

// 4-D map over a [B, L, H, d] bf16 tensor, box (64, 1, rows, 1), 128-byte swizzle.
cudaError_t encode_bwd_map(CUtensorMap* map, const void* base, int B, int L, int H, int D,
                           int rows) {
  EncodeTiledFn enc = tensor_map_encoder();
  if (!enc) return cudaErrorNotSupported;
  cuuint64_t dims[4] = {(cuuint64_t)D, (cuuint64_t)H, (cuuint64_t)L, (cuuint64_t)B};
  cuuint64_t strides[3] = {(cuuint64_t)D * 2, (cuuint64_t)H * D * 2, (cuuint64_t)L * H * D * 2};
  cuuint32_t box[4] = {64, 1, (cuuint32_t)rows, 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims,
                   strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

template <int D>
constexpr int rows_smem_bytes() {
  using C = BwdCfg<D>;
  return 1024 + 3 * C::BIG + kBwdStages * 2 * C::SMALL + 5 * 4 * kTileM * 4 +
         (int)sizeof(RowsBars) + 16;
}
template <int D>
constexpr int keys_smem_bytes() {
  using C = BwdCfg<D>;
  return 1024 + 2 * C::BIG + kBwdStages * (3 * C::SMALL + kTileN * 16) + (int)sizeof(KeysBars) +
         16;
}
static_assert(rows_smem_bytes<128>() <= 227 * 1024 && keys_smem_bytes<128>() <= 227 * 1024,
              "shared memory");

template <int D>
cudaError_t launch_bwd_tc_d(const BwdTcArgs& a, cudaStream_t stream) {
  BwdTcParams p;
  p.dq = a.dq;
  p.drho = a.drho;
  p.dk = a.dk;
  p.dv = a.dv;
  p.stats = static_cast<float4*>(a.workspace);
  p.B = a.B;
  p.L = a.L;
  p.Hq = a.Hq;
  p.Hkv = a.Hkv;
  p.G = a.Hq / a.Hkv;
  p.causal = a.causal;
  p.scale = a.scale;
  p.qscale = a.scale * 1.4426950408889634f;
  p.err = a.err;
  // rows kernel: Q, R, G in 128-row boxes, K, V in 64-row boxes
  CUtensorMap qm, rm, gm, km, vm;
  cudaError_t e = encode_bwd_map(&qm, a.q, a.B, a.L, a.Hq, D, kTileM);
  if (e == cudaSuccess) e = encode_bwd_map(&rm, a.rho, a.B, a.L, a.Hq, D, kTileM);
  if (e == cudaSuccess) e = encode_bwd_map(&gm, a.dout, a.B, a.L, a.Hq, D, kTileM);
  if (e == cudaSuccess) e = encode_bwd_map(&km, a.k, a.B, a.L, a.Hkv, D, kTileN);
  if (e == cudaSuccess) e = encode_bwd_map(&vm, a.v, a.B, a.L, a.Hkv, D, kTileN);
  if (e != cudaSuccess) return e;
  const long long rows_units = (long long)a.B * a.Hq * ((a.L + kTileM - 1) / kTileM);
  const long long keys_units = (long long)a.B * a.Hkv * ((a.L + kTileM - 1) / kTileM);
  if (rows_units > 0x7fffffffll || keys_units > 0x7fffffffll) return cudaErrorInvalidValue;
  p.units = (int)rows_units;
  auto rows = plx_bwd_rows_tc_kernel<D>;
  int smem = rows_smem_bytes<D>();
  e = cudaFuncSetAttribute(rows, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  const unsigned rows_grid = (unsigned)(rows_units < a.num_sms ? rows_units : a.num_sms);
  rows<<<rows_grid, kBwdThreads, smem, stream>>>(qm, rm, gm, km, vm, p);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  // keys kernel: Q, R, G in 64-row boxes, K, V in 128-row boxes
  e = encode_bwd_map(&qm, a.q, a.B, a.L, a.Hq, D, kTileN);
  if (e == cudaSuccess) e = encode_bwd_map(&rm, a.rho, a.B, a.L, a.Hq, D, kTileN);
  if (e == cudaSuccess) e = encode_bwd_map(&gm, a.dout, a.B, a.L, a.Hq, D, kTileN);
  if (e == cudaSuccess) e = encode_bwd_map(&km, a.k, a.B, a.L, a.Hkv, D, kTileM);
  if (e == cudaSuccess) e = encode_bwd_map(&vm, a.v, a.B, a.L, a.Hkv, D, kTileM);
  if (e != cudaSuccess) return e;
  p.units = (int)keys_units;
  auto keys = plx_bwd_keys_tc_kernel<D>;
  smem = keys_smem_bytes<D>();
  e = cudaFuncSetAttribute(keys, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  const unsigned keys_grid = (unsigned)(keys_units < a.num_sms ? keys_units : a.num_sms);
  keys<<<keys_grid, kBwdThreads, smem, stream>>>(qm, rm, gm, km, vm, p);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_prefill_bwd_tc(const BwdTcArgs& a, cudaStream_t stream) {
  if (a.d == 128) return launch_bwd_tc_d<128>(a, stream);
  if (a.d == 64) return launch_bwd_tc_d<64>(a, stream);
  return cudaErrorInvalidValue;
}

}  // namespace plx
