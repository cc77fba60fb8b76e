// plx_prefill_tc.cu -- bf16 Parallax prefill on the 5th-generation tensor cores.
//
// Operator (page 1 "Parallax: Parameterized Local Linear Attention Gives
// Transformers a 'Second Eye'", opening formula and section 1.3; page 3
// "Parallax keeps softmax, adds covariance correction branch"): for query row i
//
//   out_i = o_i - (u_i - tbar_i o_i),  o = sum_j a_j v_j,  u = sum_j a_j t_j v_j,
//   t_j = rho_i . k_j,  tbar = sum_j a_j t_j,  a = softmax_j(scale q_i . k_j)
//
// which is o_SA - Sigma_KV^T rho written so that one pass over the keys and
// values feeds both branches (page 3: the KV stream is reused by both).
//
// Per CTA (persistent; one 128-row query tile per work unit, heaviest causal
// tiles first):
//   warp 0      TMA producer: Q and R tiles once per unit, K and V tiles of 64
//               keys into a 4-stage ring (128-byte swizzled, UMMA-canonical).
//   warp 1      MMA issuer (one thread): S = Q K^T and T = R K^T share the K
//               tile; O += P V and U += (P o T) V share the V tile.
//   warp 2      allocates / frees the 512 TMEM columns.
//   warps 4-7   softmax + epilogue, one thread per query row (= TMEM lane).
// TMEM columns: O [0, d), U [d, 2d), S buffers at 256 + 64 b, T buffers at
// 384 + 64 b (b = tile parity): the tensor core computes S, T of tile j+1 while
// the softmax warps turn S, T of tile j into P = 2^(s - m) and P t, which
// they store back as fp16 over the first 32 columns of the same buffers; those
// are the A operands (from TMEM) of the two PV products.  The softmax warps also
// convert each V tile to fp16 in place, so the PV products are fp16 x fp16 with
// fp32 accumulation: P rounded to bf16 (8 significant bits) is not accurate
// enough once the correction's (1 + tbar) o - u cancellation amplifies it,
// fp16's 11 bits are.  The normalisers l = sum P and z = sum P t are summed
// from the same rounded values the tensor core multiplies.  The running max is
// rescaled lazily (only when it grows by more than 2^8, so P <= 2^8), and P t
// carries a per-row power-of-two scale that grows only if |t| would push it
// past fp16's range; O and U pass through registers only when either changes.
// Range: |v| and |rho . k| must stay below 65504 (fp16); a non-finite result
// is reported through the device error word.
#include "plx_launch.h"

namespace plx {

namespace {

constexpr int kBM = 128;      // query rows per tile = TMEM lanes
constexpr int kBN = 64;       // keys per tile
constexpr int kStages = 4;    // K/V ring depth
constexpr int kThreads = 256;
constexpr float kRescaleThreshold = 8.0f;  // log2 units

template <int D>
struct TcCfg {
  static constexpr int KB = D / 64;              // 64-element (128-byte) column blocks
  static constexpr int Q_BOX = kBM * 128;        // bytes of one Q/R column block
  static constexpr int KV_BOX = kBN * 128;       // bytes of one K/V column block
  static constexpr int Q_BYTES = KB * Q_BOX;
  static constexpr int KV_BYTES = KB * KV_BOX;
  static constexpr int STAGE_BYTES = 2 * KV_BYTES;
  static constexpr int TILE_SMEM = 2 * Q_BYTES + kStages * STAGE_BYTES;
  static constexpr uint32_t COL_O = 0, COL_U = D, COL_S = 256, COL_T = 384;
  // S, T: bf16 Q/R (K-major) x bf16 K (K-major).  PV: fp16 P from TMEM x fp16 V
  // (MN-major; converted in place from bf16 before use).
  static constexpr uint32_t IDESC_ST = umma_idesc_f16kind(kBM, kBN, false, false);
  static constexpr uint32_t IDESC_PV = umma_idesc_f16kind(kBM, D, true, true);
};

struct TcParams {
  int B, L, Hq, Hkv, G, causal, nqt, units;
  float qscale;  // softmax scale * log2(e)
  void* out;     // bf16 or fp32 (kernel template parameter)
  float* lse;
  unsigned* err;
};

struct Unit {
  int b, h, mt, n;  // batch, query head, query tile, key tiles
};

__device__ __forceinline__ Unit unit_of(const TcParams& p, int u) {
  Unit x;
  const int bh = p.B * p.Hq;
  x.mt = p.nqt - 1 - u / bh;  // heaviest (last) query tiles first
  const int r = u % bh;
  x.b = r / p.Hq;
  x.h = r % p.Hq;
  const int nk = (p.L + kBN - 1) / kBN;
  x.n = p.causal ? min(nk, (x.mt * kBM + kBM - 1) / kBN + 1) : nk;
  return x;
}

struct Bars {
  uint64_t q_full, q_empty, drain;
  uint64_t kv_full[kStages], kv_empty[kStages];
  uint64_t s_full[2], p_full[2], o_done[2];
};

template <int D, typename OutT>
__global__ void __launch_bounds__(kThreads, 1)
    plx_prefill_tc_kernel(const __grid_constant__ CUtensorMap qmap,
                          const __grid_constant__ CUtensorMap rmap,
                          const __grid_constant__ CUtensorMap kmap,
                          const __grid_constant__ CUtensorMap vmap, const TcParams p) {
  using C = TcCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint8_t* sQ = smem;
  uint8_t* sR = smem + C::Q_BYTES;
  uint8_t* sKV = smem + 2 * C::Q_BYTES;
  Bars* bars = reinterpret_cast<Bars*>(smem + C::TILE_SMEM);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  if (tid == 0) {
    *abort_flag = 0;
    mbar_init(&bars->q_full, 1);
    mbar_init(&bars->q_empty, 1);
    mbar_init(&bars->drain, 1);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&bars->kv_full[s], 1);
      mbar_init(&bars->kv_empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&bars->s_full[b], 1);
      mbar_init(&bars->p_full[b], kBM);
      mbar_init(&bars->o_done[b], 1);
    }
    fence_mbarrier_init();
  }
  if (warp == 2) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      tma_prefetch_desc(&qmap);
      tma_prefetch_desc(&rmap);
      tma_prefetch_desc(&kmap);
      tma_prefetch_desc(&vmap);
      int g = 0, ku = 0;
      bool ok = true;
      for (int u = blockIdx.x; ok && u < p.units; u += gridDim.x, ++ku) {
        const Unit x = unit_of(p, u);
        const int hk = x.h / p.G;
        if (ku > 0 && !mbar_wait(&bars->q_empty, (ku - 1) & 1, abort_flag, p.err)) break;
        mbar_arrive_expect_tx(&bars->q_full, 2 * C::Q_BYTES);
        for (int kb = 0; kb < C::KB; ++kb) {
          tma_load_4d(sQ + kb * C::Q_BOX, &qmap, &bars->q_full, kb * 64, x.h, x.mt * kBM, x.b);
          tma_load_4d(sR + kb * C::Q_BOX, &rmap, &bars->q_full, kb * 64, x.h, x.mt * kBM, x.b);
        }
        for (int j = 0; j < x.n; ++j) {
          const int t = g + j, st = t % kStages;
          if (t >= kStages &&
              !mbar_wait(&bars->kv_empty[st], ((t / kStages) - 1) & 1, abort_flag, p.err)) {
            ok = false;
            break;
          }
          uint8_t* sK = sKV + st * C::STAGE_BYTES;
          uint8_t* sV = sK + C::KV_BYTES;
          mbar_arrive_expect_tx(&bars->kv_full[st], C::STAGE_BYTES);
          for (int kb = 0; kb < C::KB; ++kb) {
            tma_load_4d(sK + kb * C::KV_BOX, &kmap, &bars->kv_full[st], kb * 64, hk, j * kBN, x.b);
            tma_load_4d(sV + kb * C::KV_BOX, &vmap, &bars->kv_full[st], kb * 64, hk, j * kBN, x.b);
          }
        }
        g += x.n;
      }
      if (*abort_flag) {
        // let copies already in flight land before the CTA's memory is released
        const uint64_t t0 = globaltimer_ns();
        while (globaltimer_ns() - t0 < 100000) {
        }
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t sq = smem_u32(sQ), sr = smem_u32(sR), skv = smem_u32(sKV);
      int g = 0, ku = 0;
      bool ok = true;
      auto issue_pv = [&](int t, bool first) -> bool {
        const int b = t & 1, st = t % kStages;
        if (!mbar_wait(&bars->p_full[b], (t >> 1) & 1, abort_flag, p.err)) return false;
        tc_fence_after();
        const uint32_t sv = skv + st * C::STAGE_BYTES + C::KV_BYTES;
#pragma unroll
        for (int kk = 0; kk < kBN / 16; ++kk) {
          const uint64_t bv = smem_desc_sw128(sv + kk * 16 * 128, C::KV_BOX, 1024);
          umma_ts(tbase + C::COL_O, tbase + C::COL_S + 64 * b + kk * 8, bv, C::IDESC_PV,
                  (first && kk == 0) ? 0u : 1u);
        }
#pragma unroll
        for (int kk = 0; kk < kBN / 16; ++kk) {
          const uint64_t bv = smem_desc_sw128(sv + kk * 16 * 128, C::KV_BOX, 1024);
          umma_ts(tbase + C::COL_U, tbase + C::COL_T + 64 * b + kk * 8, bv, C::IDESC_PV,
                  (first && kk == 0) ? 0u : 1u);
        }
        umma_commit(&bars->o_done[b]);
        umma_commit(&bars->kv_empty[st]);
        return true;
      };
      for (int u = blockIdx.x; ok && u < p.units; u += gridDim.x, ++ku) {
        const Unit x = unit_of(p, u);
        if (!mbar_wait(&bars->q_full, ku & 1, abort_flag, p.err)) break;
        tc_fence_after();
        for (int j = 0; j < x.n; ++j) {
          const int t = g + j, st = t % kStages, b = t & 1;
          if (!mbar_wait(&bars->kv_full[st], (t / kStages) & 1, abort_flag, p.err)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sk = skv + st * C::STAGE_BYTES;
#pragma unroll
          for (int k = 0; k < D / 16; ++k) {
            const uint32_t off = (k >> 2) * C::Q_BOX + (k & 3) * 32;
            const uint32_t koff = (k >> 2) * C::KV_BOX + (k & 3) * 32;
            umma_ss(tbase + C::COL_S + 64 * b, smem_desc_sw128(sq + off, 16, 1024),
                    smem_desc_sw128(sk + koff, 16, 1024), C::IDESC_ST, k > 0 ? 1u : 0u);
          }
#pragma unroll
          for (int k = 0; k < D / 16; ++k) {
            const uint32_t off = (k >> 2) * C::Q_BOX + (k & 3) * 32;
            const uint32_t koff = (k >> 2) * C::KV_BOX + (k & 3) * 32;
            umma_ss(tbase + C::COL_T + 64 * b, smem_desc_sw128(sr + off, 16, 1024),
                    smem_desc_sw128(sk + koff, 16, 1024), C::IDESC_ST, k > 0 ? 1u : 0u);
          }
          umma_commit(&bars->s_full[b]);
          if (j == x.n - 1) umma_commit(&bars->q_empty);
          if (j > 0 && !issue_pv(t - 1, j == 1)) {
            ok = false;
            break;
          }
        }
        if (ok && !issue_pv(g + x.n - 1, x.n == 1)) ok = false;
        g += x.n;
      }
      // Every MMA must have completed before the columns are released.
      umma_commit(&bars->drain);
      volatile int never = 0;
      mbar_wait(&bars->drain, 0, &never, p.err);
    }
    __syncwarp();
  } else if (warp >= 4) {
    // ------------------------------------------------------------ softmax + epilogue
    const int r = tid - 128;                       // row within the tile = TMEM lane
    const uint32_t lane_addr = tbase + ((uint32_t)((warp - 4) * 32) << 16);
    const bool qpos = p.qscale >= 0.f;
    int g = 0;
    bool ok = true, finite = true;
    for (int u = blockIdx.x; ok && u < p.units; u += gridDim.x) {
      const Unit x = unit_of(p, u);
      const int i = x.mt * kBM + r;
      // Running max m (log2 units of the scaled scores); P = 2^(s - m) <= 2^8
      // (lazy rescaling).  l = sum P and z = sum P t * 2^-eu are summed from the
      // rounded fp16 values the tensor core multiplies; l32 = sum P unrounded
      // (for lse).  eu (>= 0) keeps P t * 2^-eu inside fp16's range.
      float m_run = -INFINITY, l = 0.f, z = 0.f, l32 = 0.f;
      int eu = 0;
      for (int j = 0; j < x.n; ++j) {
        const int t = g + j, b = t & 1, st = t % kStages;
        // V of this key tile -> fp16 in place (the PV products run in fp16).
        if (!mbar_wait(&bars->kv_full[st], (t / kStages) & 1, abort_flag, p.err)) {
          ok = false;
          break;
        }
        {
          uint4* vt = reinterpret_cast<uint4*>(sKV + st * C::STAGE_BYTES + C::KV_BYTES);
#pragma unroll
          for (int c = r; c < C::KV_BYTES / 16; c += kBM) {
            uint4 w = vt[c];
            float2 f;
            f = bf16x2_to_float2(w.x);
            w.x = float2_to_f16x2(f.x, f.y);
            f = bf16x2_to_float2(w.y);
            w.y = float2_to_f16x2(f.x, f.y);
            f = bf16x2_to_float2(w.z);
            w.z = float2_to_f16x2(f.x, f.y);
            f = bf16x2_to_float2(w.w);
            w.w = float2_to_f16x2(f.x, f.y);
            vt[c] = w;
          }
          fence_proxy_async_smem();
        }
        if (!mbar_wait(&bars->s_full[b], (t >> 1) & 1, abort_flag, p.err)) {
          ok = false;
          break;
        }
        tc_fence_after();
        uint32_t sv[64], tv[64];
        {
          uint32_t (&s0)[32] = *reinterpret_cast<uint32_t(*)[32]>(&sv[0]);
          uint32_t (&s1)[32] = *reinterpret_cast<uint32_t(*)[32]>(&sv[32]);
          tmem_ld2x32_sync(lane_addr + C::COL_S + 64 * b, lane_addr + C::COL_S + 64 * b + 32, s0,
                           s1);
          uint32_t (&t0)[32] = *reinterpret_cast<uint32_t(*)[32]>(&tv[0]);
          uint32_t (&t1)[32] = *reinterpret_cast<uint32_t(*)[32]>(&tv[32]);
          tmem_ld2x32_sync(lane_addr + C::COL_T + 64 * b, lane_addr + C::COL_T + 64 * b + 32, t0,
                           t1);
        }
        const int key0 = j * kBN;
        const bool need_mask = p.causal ? (key0 + kBN - 1 > i) : (key0 + kBN > p.L);
        const int nvis = need_mask ? max(0, min(kBN, (p.causal ? i : p.L - 1) - key0 + 1)) : kBN;
        // extreme of the raw scores (max if scale >= 0) and max |t| over the
        // visible keys
        float ext = qpos ? -INFINITY : INFINITY, tmax = 0.f;
#pragma unroll
        for (int c = 0; c < 64; ++c) {
          const float v = __uint_as_float(sv[c]);
          if (c < nvis) {
            ext = qpos ? fmaxf(ext, v) : fminf(ext, v);
            tmax = fmaxf(tmax, fabsf(__uint_as_float(tv[c])));
          }
        }
        const float tile_max = (nvis > 0) ? ext * p.qscale : -INFINITY;
        const float m_new = fmaxf(m_run, tile_max);
        const bool resc = (m_run != -INFINITY) && (m_new > m_run + kRescaleThreshold);
        if (m_run == -INFINITY) m_run = m_new;
        // |P t| <= 2^8 |t|: keep |t| 2^-eu below 2^7 (P t 2^-eu below 2^15)
        int eu_new = eu;
        if (tmax * exp2f((float)-eu) >= 128.f) eu_new = max(eu, (int)ceilf(log2f(tmax)) - 6);
        const bool ubump = eu_new > eu;
        if (__any_sync(0xffffffffu, resc || ubump)) {
          if (j > 0 &&
              !mbar_wait(&bars->o_done[(t - 1) & 1], ((t - 1) >> 1) & 1, abort_flag, p.err)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const float alpha = resc ? exp2f(m_run - m_new) : 1.f;
          const float beta = alpha * exp2f((float)(eu - eu_new));
#pragma unroll 1
          for (int cc = 0; cc < 2 * D; cc += 32) {
            const float f = cc < D ? alpha : beta;
            uint32_t w[32];
            tmem_ld32_sync(lane_addr + C::COL_O + cc, w);
#pragma unroll
            for (int e = 0; e < 32; ++e) w[e] = __float_as_uint(__uint_as_float(w[e]) * f);
            tmem_st32(lane_addr + C::COL_O + cc, w);
          }
          tmem_wait_st();
          l *= alpha;
          l32 *= alpha;
          z *= beta;
          if (resc) m_run = m_new;
          eu = eu_new;
        }
        // P = 2^(s - m) as fp16 over the S buffer
        const bool live = m_run != -INFINITY;
        uint32_t pk[32];
#pragma unroll
        for (int c = 0; c < 32; ++c) {
          float p0 = exp2f(fmaf(__uint_as_float(sv[2 * c]), p.qscale, -m_run));
          float p1 = exp2f(fmaf(__uint_as_float(sv[2 * c + 1]), p.qscale, -m_run));
          if (!live || 2 * c >= nvis) p0 = 0.f;
          if (!live || 2 * c + 1 >= nvis) p1 = 0.f;
          sv[2 * c] = __float_as_uint(p0);
          sv[2 * c + 1] = __float_as_uint(p1);
          l32 += p0 + p1;
          pk[c] = float2_to_f16x2(p0, p1);
          const float2 rp = f16x2_to_float2(pk[c]);
          l += rp.x + rp.y;
        }
        tmem_st32(lane_addr + C::COL_S + 64 * b, pk);
        // P t 2^-eu as fp16 over the T buffer
        const float tsc = exp2f((float)-eu);
#pragma unroll
        for (int c = 0; c < 32; ++c) {
          const float q0 = __uint_as_float(sv[2 * c]) * (__uint_as_float(tv[2 * c]) * tsc);
          const float q1 = __uint_as_float(sv[2 * c + 1]) * (__uint_as_float(tv[2 * c + 1]) * tsc);
          pk[c] = float2_to_f16x2(q0, q1);
          const float2 rq = f16x2_to_float2(pk[c]);
          z += rq.x + rq.y;
        }
        tmem_st32(lane_addr + C::COL_T + 64 * b, pk);
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(&bars->p_full[b]);
      }
      if (!ok) break;
      // ---- epilogue: out = ((1 + z/l) o - u) / l, lse = ln(sum exp(scale s))
      const int tl = g + x.n - 1;
      if (!mbar_wait(&bars->o_done[tl & 1], (tl >> 1) & 1, abort_flag, p.err)) break;
      tc_fence_after();
      const float inv = 1.f / l;
      const float usc = exp2f((float)eu);           // undo the P t scaling
      const float c1 = (1.f + z * usc * inv) * inv;
      const float cu = usc * inv;
      OutT* orow = static_cast<OutT*>(p.out) + (((size_t)x.b * p.L + i) * p.Hq + x.h) * D;
#pragma unroll 1
      for (int cc = 0; cc < D; cc += 32) {
        uint32_t ov[32], uv[32];
        tmem_ld2x32_sync(lane_addr + C::COL_O + cc, lane_addr + C::COL_U + cc, ov, uv);
        float a[32];
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          a[e] = __uint_as_float(ov[e]) * c1 - __uint_as_float(uv[e]) * cu;
          finite = finite && isfinite(a[e]);
        }
        if (i < p.L) {
          if constexpr (sizeof(OutT) == 2) {
            uint4* dst = reinterpret_cast<uint4*>(orow + cc);
#pragma unroll
            for (int q = 0; q < 4; ++q)
              dst[q] = make_uint4(float2_to_bf16x2(a[8 * q], a[8 * q + 1]),
                                  float2_to_bf16x2(a[8 * q + 2], a[8 * q + 3]),
                                  float2_to_bf16x2(a[8 * q + 4], a[8 * q + 5]),
                                  float2_to_bf16x2(a[8 * q + 6], a[8 * q + 7]));
          } else {
            float4* dst = reinterpret_cast<float4*>(orow + cc);
#pragma unroll
            for (int q = 0; q < 8; ++q)
              dst[q] = make_float4(a[4 * q], a[4 * q + 1], a[4 * q + 2], a[4 * q + 3]);
          }
        }
      }
      if (p.lse && i < p.L)
        p.lse[((size_t)x.b * p.Hq + x.h) * p.L + i] =
            (m_run + log2f(l32)) * 0.6931471805599453f;
      tc_fence_before();
      g += x.n;
    }
    // Values past the fp16 range of the PV products (or non-finite inputs)
    // leave a non-finite row: report it rather than return it silently.
    if (!finite) record_error(p.err, kDevNonFinite);
  }

  __syncthreads();
  if (warp == 2) {
    tc_fence_after();
    tmem_dealloc(tbase, 512);
  }
}

// 4-D map over a [B, S, H, D] bf16 tensor, box (64, 1, rows, 1), 128-byte swizzle.
cudaError_t encode_sw128(CUtensorMap* map, const void* base, int B, int S, int H, int D,
                         int rows) {
  EncodeTiledFn enc = tensor_map_encoder();
  if (!enc) return cudaErrorNotSupported;
  cuuint64_t dims[4] = {(cuuint64_t)D, (cuuint64_t)H, (cuuint64_t)S, (cuuint64_t)B};
  cuuint64_t strides[3] = {(cuuint64_t)D * 2, (cuuint64_t)H * D * 2, (cuuint64_t)S * H * D * 2};
  cuuint32_t box[4] = {64, 1, (cuuint32_t)rows, 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims,
                   strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

template <int D, typename OutT>
cudaError_t launch_d(const PrefillTcArgs& a, cudaStream_t stream) {
  using C = TcCfg<D>;
  CUtensorMap qm, rm, km, vm;
  cudaError_t e = encode_sw128(&qm, a.q, a.B, a.L, a.Hq, D, kBM);
  if (e == cudaSuccess) e = encode_sw128(&rm, a.rho, a.B, a.L, a.Hq, D, kBM);
  if (e == cudaSuccess) e = encode_sw128(&km, a.k, a.B, a.L, a.Hkv, D, kBN);
  if (e == cudaSuccess) e = encode_sw128(&vm, a.v, a.B, a.L, a.Hkv, D, kBN);
  if (e != cudaSuccess) return e;
  TcParams p;
  p.B = a.B;
  p.L = a.L;
  p.Hq = a.Hq;
  p.Hkv = a.Hkv;
  p.G = a.Hq / a.Hkv;
  p.causal = a.causal;
  p.nqt = (a.L + kBM - 1) / kBM;
  const long long units = (long long)a.B * a.Hq * p.nqt;
  if (units > 0x7fffffff) return cudaErrorInvalidValue;
  p.units = (int)units;
  p.qscale = a.scale * 1.4426950408889634f;
  p.out = a.out;
  p.lse = a.lse;
  p.err = a.err;
  const int smem = 1024 + C::TILE_SMEM + (int)sizeof(Bars) + 16;
  auto kern = plx_prefill_tc_kernel<D, OutT>;
  e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  const int grid = (int)(units < a.num_sms ? units : a.num_sms);
  kern<<<grid, kThreads, smem, stream>>>(qm, rm, km, vm, p);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_prefill_tc(const PrefillTcArgs& a, cudaStream_t stream) {
  if (a.d == 128)
    return a.out_f32 ? launch_d<128, float>(a, stream) : launch_d<128, __nv_bfloat16>(a, stream);
  if (a.d == 64)
    return a.out_f32 ? launch_d<64, float>(a, stream) : launch_d<64, __nv_bfloat16>(a, stream);
  return cudaErrorInvalidValue;
}

}  // namespace plx
