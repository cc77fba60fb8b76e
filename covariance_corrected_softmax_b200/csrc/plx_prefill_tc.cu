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
// Per CTA (persistent; one 128-row query tile per work unit, bands of the
// heaviest causal tiles first, a band's units grouped by KV head):
//   warp 0      TMA producer: Q and R tiles once per unit, K and V tiles of 64
//               keys into a 4-stage ring (128-byte swizzled, UMMA-canonical).
//   warp 1      S/T issuer (one thread): S = Q K^T and T = R K^T of each key
//               tile (sharing the K tile).
//   warps 2, 12 convert each V tile to fp16 in place (half a tile each);
//               warp 2 also allocates and frees the TMEM columns.
//   warp 3      PV issuer (one thread): O += P V and U += (P o T) V of each
//               key tile (sharing the V tile).
//   warps 4-11  softmax + epilogue: two warpgroups; thread (row, half) owns
//               one query row (= TMEM lane) and half of each key tile's
//               columns.  The partners of a row exchange their partial row
//               maxima through shared memory once per tile.
// Two issuing threads in different warps keep the tensor core fed: a thread's
// barrier wait is ordered behind its own MMAs still queued for the tensor core,
// so a single issuer leaves the tensor core idle while it waits.
//
// The PV products are fp16 x fp16 with fp32 accumulation (P rounded to bf16,
// 8 significant bits, is not accurate enough once the correction's
// (1 + tbar) o - u cancellation amplifies it; fp16's 11 bits are), and their B
// operand is V with a 16-column block of fp16 ones appended, so O gains the
// column l = sum P and U the column z = sum P t: the normalisers are summed by
// the tensor core from exactly the fp16 values it multiplies, and the softmax
// warps do no summing at all.  The ones block is one 8 KB array shared by all
// ring stages: each stage's V descriptor gets its own column-block stride so
// that its third (or, for d = 64, second) block lands on it.
//
// TMEM columns (d = 128): O [0, 144), U [160, 304), S [320, 384),
// T [384, 448), P [448, 480), P t [480, 512).  S and T are single-buffered:
// the softmax warps copy them to registers and release them at once, so the
// tensor core computes S, T of tile j+1 while the softmax works on tile j.  P
// and P t are fp16 pairs, the A operands (from TMEM) of the PV products.  The
// running max is rescaled lazily (only when the scores exceed it by more than a
// factor 2^8, so P <= 2^8), and P t carries a per-row power-of-two scale that
// grows only if |t| would push it past fp16's range; O and U (with their l, z
// columns) pass through registers only when either changes, after P and P t
// of the tile are stored.
// Range: V enters the fp16 products as a block floating-point value: the
// converter warp finds the largest |v| of each V tile and scales the tile by
// 2^-E before rounding it to fp16, E being the running maximum, over the
// unit's tiles so far, of floor(log2 max|v|) - 14 (so every scaled value is
// below 2^15).  When E grows, the V columns of O and U are rescaled with the
// other lazy rescales; the epilogue multiplies by 2^E.  The ones block is not
// scaled, so l and z are unaffected.  Any finite bf16 V thus keeps fp16's 11
// significant bits relative to the largest |v| of its tile.  P t carries its
// own power-of-two scale (eu, above).  A non-finite result (inputs whose result
// exceeds fp32, or non-finite inputs) is reported through the device error
// word.
#include "plx_launch.h"

namespace plx {

namespace {

constexpr int kBM = 128;      // query rows per tile = TMEM lanes
constexpr int kBN = 64;       // keys per tile
constexpr int kHalf = kBN / 2;  // key columns per softmax thread
constexpr int kStages = 4;    // K/V ring depth (the shared-memory layout below assumes 4)
constexpr int kSoftWarps = 8;   // two softmax warpgroups
constexpr int kConvWarps = 2;   // V converters: warp 2 and the last warp
constexpr int kThreads = (4 + kSoftWarps + 1) * 32;
constexpr int kConvWarp2 = 4 + kSoftWarps;  // the second converter's warp index
// Lazy rescaling: the running max m moves only when a score exceeds it by more
// than 2^kRescaleBits, so P <= 2^kRescaleBits; |t| 2^-eu is kept below
// 2^kTBits so that |P t 2^-eu| < 2^15 stays inside fp16's range.
constexpr int kRescaleBits = 8;
constexpr int kTBits = 15 - kRescaleBits;
constexpr uint32_t kOnesBytes = 8192;      // 64 keys x 64 fp16 ones, 128-byte rows
// Block exponent E of V (see the header comment): clamped to [kVExpMin,
// kVExpMax] so that 2^-E and 2^E stay normal fp32 numbers.  A tile whose
// largest |v| lies in [2^kVLowBits, 2^(kVHeadroomBits + 1)) is kept as it is
// (E = 0): fp16 holds it and every value down to 2^-8 of the largest with full
// precision, and the conversion needs no multiply.
constexpr int kVExpMin = -100;
constexpr int kVExpMax = 113;
constexpr int kVHeadroomBits = 14;   // scaled |v| < 2^(kVHeadroomBits + 1)
constexpr int kVLowBits = -6;
// Key pairs (of a thread's 16) whose 2^x runs on the FMA pipe (exp2_poly2)
// rather than the special-function unit, which also does the fp16 packing.
// Two of sixteen: measured against none, four and eight of sixteen, the
// fastest on both prefill workloads.
constexpr uint32_t kPolyPairs = 0x8080u;

template <int D>
struct TcCfg {
  static_assert(D == 64 || D == 128, "head dimension 64 or 128");
  static constexpr int KB = D / 64;              // 64-element (128-byte) column blocks
  static constexpr int Q_BOX = kBM * 128;        // bytes of one Q/R column block
  static constexpr int KV_BOX = kBN * 128;       // bytes of one K/V column block (8 KB)
  static constexpr int Q_BYTES = KB * Q_BOX;
  static constexpr int KV_BYTES = KB * KV_BOX;
  static constexpr int STAGE_BYTES = 2 * KV_BYTES;  // TMA bytes per ring stage
  // K/V region (offsets from its start).  V stage st: block 0 at v_box(st, 0),
  // block c at v_box(st, 0) + c * v_lbo(st); block KB is the ones array at
  // ONES (v_box(st, 0) + KB * v_lbo(st) == ONES for every stage).
  static constexpr int ONES = KB == 2 ? 131072 : 65536;
  __host__ __device__ static constexpr int v_lbo(int st) { return 65536 - 8192 * st; }
  __host__ __device__ static constexpr int v_box(int st, int c) {
    return KB == 2 ? (c == 0 ? 16384 * st : 65536 + 8192 * st) : 8192 * st;
  }
  __host__ __device__ static constexpr int k_box(int st, int c) {
    return KB == 2 ? (c == 0 ? 16384 * st + 8192 : 98304 + 8192 * st) : 32768 + 8192 * st;
  }
  static constexpr int KV_REGION = ONES + kOnesBytes;
  static constexpr int TILE_SMEM = 2 * Q_BYTES + KV_REGION;
  // TMEM columns
  static constexpr uint32_t NPV = D + 16;                 // PV product width (V | ones)
  static constexpr uint32_t OU = (NPV + 31) / 32 * 32;    // column stride of O and U
  static constexpr uint32_t COL_O = 0, COL_U = OU;
  static constexpr uint32_t COL_S = 2 * OU, COL_T = COL_S + kBN;
  static constexpr uint32_t COL_P = COL_T + kBN, COL_PT = COL_P + kBN / 2;
  static_assert(COL_PT + kBN / 2 <= 512, "TMEM columns");
  // S, T: bf16 Q/R (K-major) x bf16 K (K-major).  PV: fp16 P from TMEM x fp16
  // [V | 1] (MN-major; V converted in place from bf16 before use).
  static constexpr uint32_t IDESC_ST = umma_idesc_f16kind(kBM, kBN, false, false);
  static constexpr uint32_t IDESC_PV = umma_idesc_f16kind(kBM, NPV, true, true);
};

// The shared-memory layout above places, for every stage, K and V blocks that do
// not overlap each other, the ones array, or another stage's blocks.
template <int D>
constexpr bool layout_ok() {
  using C = TcCfg<D>;
  int lo[4 * kStages + 1] = {}, hi[4 * kStages + 1] = {}, n = 0;
  for (int st = 0; st < kStages; ++st)
    for (int c = 0; c < C::KB; ++c) {
      lo[n] = C::v_box(st, c);
      hi[n++] = C::v_box(st, c) + C::KV_BOX;
      lo[n] = C::k_box(st, c);
      hi[n++] = C::k_box(st, c) + C::KV_BOX;
      if (C::v_box(st, c) != C::v_box(st, 0) + c * C::v_lbo(st)) return false;
    }
  lo[n] = C::ONES;
  hi[n++] = C::ONES + (int)kOnesBytes;
  for (int st = 0; st < kStages; ++st)
    if (C::v_box(st, 0) + C::KB * C::v_lbo(st) != C::ONES) return false;
  for (int a = 0; a < n; ++a) {
    if (lo[a] % 1024 != 0 || hi[a] > C::KV_REGION) return false;
    for (int b = a + 1; b < n; ++b)
      if (lo[a] < hi[b] && lo[b] < hi[a]) return false;
  }
  return true;
}
static_assert(kStages == 4 && layout_ok<64>() && layout_ok<128>(), "K/V shared-memory layout");

struct TcParams {
  int B, L, Hq, Hkv, G, causal, nqt, units;  // varlen: B = sequences, nqt from max_seqlen
  float qscale;  // softmax scale * log2(e)
  void* out;     // bf16 or fp32 (kernel template parameter)
  float* lse;
  unsigned* err;
  const int32_t* cu_seqlens;  // varlen: sequence s is tokens [cu[s], cu[s+1])
  int total;                  // varlen: tokens in the packed tensors
};

// A work unit: query tile mt of query head h of batch (sequence) b, with n key
// tiles to visit.  Fixed shape: tensors [B, L, H, d]; varlen: packed [T, H, d].
struct Unit {
  int b, h, mt, n;
  int len;      // keys (= queries) of the sequence
  int row0;     // TMA row coordinate of the sequence's position 0
  int bc;       // TMA batch coordinate
  int tok0;     // token index of position 0 in out
  size_t lse0;  // lse index of position 0 of this head
  bool bad;     // varlen: inconsistent cu_seqlens or a sequence longer than max_seqlen
};

template <bool VARLEN>
__device__ __forceinline__ Unit unit_of(const TcParams& p, int u);
constexpr int kBand = 8;  // query tiles per band of the fixed-shape unit order

// The units the recomputing instance (SAFE) takes: a bit per unit of this CTA
// (u = blockIdx.x + k gridDim.x), set where the fast instance left the marker.
constexpr int kMaskUnits = 16384;   // units per CTA the mask covers (2 KB)

// Marker a unit of the fast instance leaves in column 0 of its first row when
// its V lies outside the range fp16 holds as it is (a NaN no arithmetic makes).
constexpr uint16_t kMarkBf16 = 0x7FABu;
constexpr uint32_t kMarkF32 = 0x7FABCDEFu;

template <typename OutT>
__device__ __forceinline__ bool is_marked(const void* out, size_t idx) {
  if constexpr (sizeof(OutT) == 2)
    return reinterpret_cast<const volatile uint16_t*>(out)[idx] == kMarkBf16;
  else
    return reinterpret_cast<const volatile uint32_t*>(out)[idx] == kMarkF32;
}

template <bool VARLEN, bool SAFE>
__device__ __forceinline__ Unit unit_at(const TcParams& p, int u, const uint32_t* mask) {
  Unit x = unit_of<VARLEN>(p, u);
  if constexpr (SAFE) {
    const int k = (u - (int)blockIdx.x) / (int)gridDim.x;
    if (!((mask[k >> 5] >> (k & 31)) & 1u)) x.n = 0;
  }
  return x;
}

template <bool VARLEN>
__device__ __forceinline__ Unit unit_of(const TcParams& p, int u) {
  Unit x;
  const int bh = p.B * p.Hq;
  if constexpr (VARLEN) {
    x.mt = p.nqt - 1 - u / bh;  // heaviest (last) query tiles first
    const int r = u % bh;
    x.b = r / p.Hq;
    x.h = r % p.Hq;
  } else {
    // Bands of kBand query tiles, the heaviest (last) band first, which keeps
    // the causal work balanced over the persistent CTAs; within a band the
    // units of one (batch, KV head) are consecutive (the group's query heads
    // side by side), so the CTAs running at one time share a few K/V streams
    // and read them from L2 rather than all B H_kv of them.  The tiles of a
    // group run heaviest first in even groups and lightest first in odd ones,
    // which evens out the work of the CTAs that take every gridDim-th unit.
    const int band = u / (kBand * bh);
    const int top = p.nqt - band * kBand;  // one past the band's heaviest tile
    const int w = min(kBand, top);         // query tiles in the band
    const int r = u - band * kBand * bh;
    const int grp = r / (w * p.G), i = r % (w * p.G);
    const int k = (grp & 1) ? w - 1 - i / p.G : i / p.G;
    x.b = grp / p.Hkv;
    x.h = (grp % p.Hkv) * p.G + i % p.G;
    x.mt = top - 1 - k;
  }
  x.bad = false;
  if constexpr (VARLEN) {
    const int s0 = p.cu_seqlens[x.b], s1 = p.cu_seqlens[x.b + 1];
    const bool ok = 0 <= s0 && s0 <= s1 && s1 <= p.total;
    x.len = ok ? s1 - s0 : 0;
    x.row0 = ok ? s0 : 0;
    x.bc = 0;
    x.tok0 = x.row0;
    x.lse0 = (size_t)x.h * p.total + x.row0;
    const int nq = (x.len + kBM - 1) / kBM;
    x.bad = !ok || nq > p.nqt;
    if (x.mt >= nq) {  // no such query tile in this sequence
      x.n = 0;
      return x;
    }
  } else {
    x.len = p.L;
    x.row0 = 0;
    x.bc = x.b;
    x.tok0 = x.b * p.L;
    x.lse0 = ((size_t)x.b * p.Hq + x.h) * p.L;
  }
  const int nk = (x.len + kBN - 1) / kBN;
  x.n = p.causal ? min(nk, (x.mt * kBM + kBM - 1) / kBN + 1) : nk;
  return x;
}

// Tile t below is the CTA's running key-tile count over all its units.
struct Bars {
  uint64_t q_full, q_empty, drain;  // drain: one arrival per issuer
  uint64_t kv_full[kStages];   // K and V of the stage landed (TMA)
  uint64_t kv_empty[kStages];  // PV of the stage's tile completed
  uint64_t v_ready[kStages];   // V of the stage converted to fp16 (converter warps)
  uint64_t s_full;             // S, T of tile t computed
  uint64_t s_free;             // S, T of tile t copied to registers (softmax warps)
  uint64_t p_full;             // P, P t of tile t stored (softmax warps)
  uint64_t o_done;             // PV of tile t completed
  uint64_t v_reload[2];        // a V column block fetched again (rare: its range changed E)
  uint64_t v_rescaled;         // O, U rescaled for a changed E (softmax warps; rare)
  int2 vtag[kStages][2];       // per column block: (tile number, exponent E it was scaled by)
  int2 vunit[8][2];            // fast instance, per converter: (unit count, V out of range)
};

// Shared memory the two halves of a row exchange through (two slots, used
// alternately, so one named barrier per exchange suffices).
struct Xchg {
  float2 tile[2][2][kBM];   // [slot][half][row]: (partial max, partial max |t|)
};

// Reads the block exponents E the converters scaled tile t's V column blocks
// by (each posted with the tile number in one 8-byte word), waiting (bounded)
// until both are posted.  Returns false on a timeout or an abort.
template <int KB>
__device__ __forceinline__ bool read_vtags(const int2 (*vtag)[2], int t, int (&e)[2],
                                           volatile int* abort_flag, unsigned* err) {
  const int st = t % kStages;
#pragma unroll
  for (int b = 0; b < 2; ++b) {
    e[b] = 0;
    if (b >= KB) continue;
    volatile const unsigned long long* tag =
        reinterpret_cast<volatile const unsigned long long*>(&vtag[st][b]);
    unsigned long long w = *tag;
    if ((int)(uint32_t)w != t) {
      const uint64_t t0 = globaltimer_ns();
      uint64_t limit = 0;
      for (uint32_t spins = 1; (int)(uint32_t)(w = *tag) != t; ++spins) {
        if ((spins & 63u) == 0) {
          if (*abort_flag) return false;
          if (limit == 0) limit = wait_limit_ns(err);
          if (globaltimer_ns() - t0 > limit || spins >= kWaitMaxPolls) {
            record_error(err, kDevTimeoutMbarrier);
            *abort_flag = 1;
            return false;
          }
        }
      }
    }
    e[b] = (int)(uint32_t)(w >> 32);
  }
  return true;
}

// SAFE = false: the fast instance.  V enters the PV products as it is (fp16
// holds |v| in [2^-6, 2^15) with full precision); a unit whose V reaches
// outside that range leaves a marker in its output and is recomputed by the
// SAFE instance, launched right after on the same stream, which takes only the
// marked units and carries V as block floating point (see the header comment).
template <int D, typename OutT, bool VARLEN, bool SAFE>
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
  Xchg* xch = reinterpret_cast<Xchg*>(smem + C::TILE_SMEM);
  Bars* bars = reinterpret_cast<Bars*>(xch + 1);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  uint32_t* umask = reinterpret_cast<uint32_t*>(tmem_slot + 4);  // SAFE: kMaskUnits bits

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  if constexpr (SAFE) {
    // launched as a programmatic dependent of the fast instance: its output
    // (with the markers) is visible once that grid has completed
    grid_dep_wait();
    // find this CTA's marked units; a CTA with none returns at once
    for (int w = tid; w < kMaskUnits / 32; w += kThreads) umask[w] = 0u;
    __syncthreads();
    int any = 0;
    for (int k = tid; k < kMaskUnits; k += kThreads) {
      const long long u = blockIdx.x + (long long)k * gridDim.x;
      if (u >= p.units) break;
      const Unit x = unit_of<VARLEN>(p, (int)u);
      if (x.n > 0 &&
          is_marked<OutT>(p.out, (((size_t)x.tok0 + x.mt * kBM) * p.Hq + x.h) * D)) {
        atomicOr(&umask[k >> 5], 1u << (k & 31));
        any = 1;
      }
    }
    if (!__syncthreads_or(any)) return;
  }

  if (tid == 0) {
    *abort_flag = 0;
    mbar_init(&bars->q_full, 1);
    mbar_init(&bars->q_empty, 1);
    mbar_init(&bars->drain, 2);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&bars->kv_full[s], 1);
      mbar_init(&bars->kv_empty[s], 1);
      mbar_init(&bars->v_ready[s], kConvWarps);
    }
    mbar_init(&bars->s_full, 1);
    mbar_init(&bars->s_free, kSoftWarps);  // one arrival per softmax warp
    mbar_init(&bars->p_full, kSoftWarps);
    mbar_init(&bars->o_done, 1);
    mbar_init(&bars->v_reload[0], 1);
    mbar_init(&bars->v_reload[1], 1);
    mbar_init(&bars->v_rescaled, kSoftWarps);
    for (int s = 0; s < kStages; ++s) bars->vtag[s][0] = bars->vtag[s][1] = make_int2(-1, 0);
    for (int s = 0; s < 8; ++s) bars->vunit[s][0] = bars->vunit[s][1] = make_int2(-1, 0);
    fence_mbarrier_init();
  }
  {
    // the ones block appended to every V tile (fp16 1.0 = 0x3C00)
    uint4* ones = reinterpret_cast<uint4*>(sKV + C::ONES);
    for (int c = tid; c < (int)(kOnesBytes / 16); c += kThreads)
      ones[c] = make_uint4(0x3C003C00u, 0x3C003C00u, 0x3C003C00u, 0x3C003C00u);
    fence_proxy_async_smem();
  }
  if (warp == 2) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *tmem_slot;
  // the recomputing instance may be scheduled as SMs free up; it waits for
  // this grid to complete before it reads anything this grid writes
  if constexpr (!SAFE) grid_dep_launch_dependents();

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      tma_prefetch_desc(&qmap);
      tma_prefetch_desc(&rmap);
      tma_prefetch_desc(&kmap);
      tma_prefetch_desc(&vmap);
      int g = 0, ku = 0;
      bool ok = true;
      // ku counts the units with work (varlen units past a sequence's last
      // query tile have none); every role counts them the same way
      for (int u = blockIdx.x; ok && u < p.units; u += gridDim.x) {
        const Unit x = unit_at<VARLEN, SAFE>(p, u, umask);
        if constexpr (VARLEN) {
          if (!SAFE && x.bad && x.mt == 0) record_error(p.err, kDevBadArgument);
        }
        if (x.n == 0) continue;
        const int hk = x.h / p.G;
        for (int j = 0; j < x.n; ++j) {
          const int t = g + j, st = t % kStages;
          if (t >= kStages &&
              !mbar_wait(&bars->kv_empty[st], ((t / kStages) - 1) & 1, abort_flag, p.err)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&bars->kv_full[st], C::STAGE_BYTES);
          for (int kb = 0; kb < C::KB; ++kb) {
            tma_load_4d(sKV + C::k_box(st, kb), &kmap, &bars->kv_full[st], kb * 64, hk,
                        x.row0 + j * kBN, x.bc);
            tma_load_4d(sKV + C::v_box(st, kb), &vmap, &bars->kv_full[st], kb * 64, hk,
                        x.row0 + j * kBN, x.bc);
          }
          if (j > 0) continue;
          // Q and R of the unit, once its first K/V tile is on its way (that
          // stage frees before the previous unit's last S/T products complete,
          // which is what frees the Q/R buffers)
          if (ku > 0 && !mbar_wait(&bars->q_empty, (ku - 1) & 1, abort_flag, p.err)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&bars->q_full, 2 * C::Q_BYTES);
          for (int kb = 0; kb < C::KB; ++kb) {
            tma_load_4d(sQ + kb * C::Q_BOX, &qmap, &bars->q_full, kb * 64, x.h,
                        x.row0 + x.mt * kBM, x.bc);
            tma_load_4d(sR + kb * C::Q_BOX, &rmap, &bars->q_full, kb * 64, x.h,
                        x.row0 + x.mt * kBM, x.bc);
          }
          if (u + (int)gridDim.x < p.units) {
            // the next unit's Q and R come from L2 when the Q/R buffers free up
            const Unit y = unit_at<VARLEN, SAFE>(p, u + gridDim.x, umask);
            if (y.n > 0) {
              for (int kb = 0; kb < C::KB; ++kb) {
                tma_prefetch_l2_4d(&qmap, kb * 64, y.h, y.row0 + y.mt * kBM, y.bc);
                tma_prefetch_l2_4d(&rmap, kb * 64, y.h, y.row0 + y.mt * kBM, y.bc);
              }
            }
          }
        }
        g += x.n;
        ++ku;
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
    // ------------------------------------------------------------ S/T issuer
    // S/T of tile t once the softmax has copied S/T of t-1 to registers and K
    // of t has landed (and, at a unit's first tile, its Q and R).
    if (lane == 0) {
      // Descriptors are built once; a tile or k-step only moves the start
      // address, i.e. adds (byte offset >> 4) to the low bits.
      const uint64_t dq = smem_desc_sw128(smem_u32(sQ), 16, 1024);
      const uint64_t dr = smem_desc_sw128(smem_u32(sR), 16, 1024);
      const uint64_t dkv = smem_desc_sw128(smem_u32(sKV), 16, 1024);
      int t = 0, ku = 0;
      bool ok = true;
      for (int u = blockIdx.x; ok && u < p.units; u += gridDim.x) {
        const int n = unit_at<VARLEN, SAFE>(p, u, umask).n;
        if (n == 0) continue;
        for (int j = 0; j < n; ++j, ++t) {
          const int st = t % kStages;
          if ((t > 0 && !mbar_wait(&bars->s_free, (t - 1) & 1, abort_flag, p.err)) ||
              (j == 0 && !mbar_wait(&bars->q_full, ku & 1, abort_flag, p.err)) ||
              !mbar_wait(&bars->kv_full[st], (t / kStages) & 1, abort_flag, p.err)) {
            ok = false;
            break;
          }
          tc_fence_after();
          // S and T products alternate, so that the two accumulate chains
          // are in flight together
#pragma unroll
          for (int k = 0; k < D / 16; ++k) {
            const uint32_t off = ((k >> 2) * C::Q_BOX + (k & 3) * 32) >> 4;
            const uint32_t koff = (C::k_box(st, k >> 2) + (k & 3) * 32) >> 4;
            umma_ss(tbase + C::COL_S, dq + off, dkv + koff, C::IDESC_ST, k > 0 ? 1u : 0u);
            umma_ss(tbase + C::COL_T, dr + off, dkv + koff, C::IDESC_ST, k > 0 ? 1u : 0u);
          }
          umma_commit(&bars->s_full);
          if (j == n - 1) umma_commit(&bars->q_empty);  // Q and R of this unit are no longer read
        }
        ++ku;
      }
      // Every MMA must have completed before the columns are released.
      umma_commit(&bars->drain);
      volatile int never = 0;
      mbar_wait(&bars->drain, 0, &never, p.err);
    }
    __syncwarp();
  } else if (warp == 3) {
    // ------------------------------------------------------------ PV issuer
    // PV of tile t once its P is stored and its V converted.  (S/T of t has
    // completed by then, so the stage's K and V are both free after PV.)
    if (lane == 0) {
      uint64_t dv[kStages];
#pragma unroll
      for (int st = 0; st < kStages; ++st)
        dv[st] = smem_desc_sw128(smem_u32(sKV + C::v_box(st, 0)), C::v_lbo(st), 1024);
      int t = 0, rescales = 0;
      int pe[2] = {0, 0};  // block exponents of the previous tile's V
      bool ok = true;
      for (int u = blockIdx.x; ok && u < p.units; u += gridDim.x) {
        const int n = unit_at<VARLEN, SAFE>(p, u, umask).n;
        for (int j = 0; j < n; ++j, ++t) {
          const int st = t % kStages;
          if (!mbar_wait(&bars->p_full, t & 1, abort_flag, p.err) ||
              !mbar_wait(&bars->v_ready[st], (t / kStages) & 1, abort_flag, p.err)) {
            ok = false;
            break;
          }
          if constexpr (SAFE) {
            // a tile whose V needed another block exponent than the previous
            // one waits until the softmax warps have rescaled O and U
            int e[2];
            read_vtags<C::KB>(bars->vtag, t, e, abort_flag, p.err);  // posted before v_ready
            if (j > 0 && (e[0] != pe[0] || e[1] != pe[1])) {
              if (!mbar_wait(&bars->v_rescaled, rescales & 1, abort_flag, p.err)) {
                ok = false;
                break;
              }
              ++rescales;
            }
            pe[0] = e[0];
            pe[1] = e[1];
          }
          tc_fence_after();
          uint64_t bv = dv[0];
#pragma unroll
          for (int s = 1; s < kStages; ++s)
            if (st == s) bv = dv[s];
#pragma unroll
          for (int kk = 0; kk < kBN / 16; ++kk) {
            umma_ts(tbase + C::COL_O, tbase + C::COL_P + 8 * kk,
                    bv + (uint64_t)((kk * 16 * 128) >> 4), C::IDESC_PV,
                    (j == 0 && kk == 0) ? 0u : 1u);
            umma_ts(tbase + C::COL_U, tbase + C::COL_PT + 8 * kk,
                    bv + (uint64_t)((kk * 16 * 128) >> 4), C::IDESC_PV,
                    (j == 0 && kk == 0) ? 0u : 1u);
          }
          umma_commit(&bars->o_done);
          umma_commit(&bars->kv_empty[st]);
        }
      }
      umma_commit(&bars->drain);
      volatile int never = 0;
      mbar_wait(&bars->drain, 0, &never, p.err);
    }
    __syncwarp();
  } else if (warp == 2 || warp == kConvWarp2) {
    // ------------------------------------------------------------ V converters
    // V of each tile -> fp16 in place (the PV products run in fp16), scaled by
    // 2^-E (block floating point).  Converter warp cw owns V column block cw
    // (d = 64: one block, converter 1 only signals) and its own running block
    // exponent E over the unit's tiles.  It converts the block with the current
    // E, eight 16-byte words per thread at a time, while finding its largest
    // |v|.  If the block asks for another E (the unit's first tile outside
    // the range fp16 holds as it is, or a later tile that needs a larger E),
    // the block is fetched again by TMA and converted with the new E: a rare
    // path, taken only by data far outside fp16's range.  The E is posted with
    // the tile number (vtag), then v_ready releases the tile to the PV products.
    constexpr int kBlockWords = C::KV_BOX / 16;       // 16-byte words of one column block
    constexpr int kIters = kBlockWords / (32 * 8);    // 8 words per thread per step
    static_assert(kBlockWords % (32 * 8) == 0, "converter steps");
    const int cw = warp == 2 ? 0 : 1;                 // the column block of this warp
    const bool has_block = cw < C::KB;
    int g = 0, reloads = 0, uc = 0;  // uc: units with work so far
    bool ok = true;
    if (lane == 0) tma_prefetch_desc(&vmap);
    for (int u = blockIdx.x; ok && u < p.units; u += gridDim.x) {
      const Unit x = unit_at<VARLEN, SAFE>(p, u, umask);
      const int n = x.n;
      const int hk = x.h / p.G;
      int ve = 0;       // this block's running exponent in the unit (0: V as it is)
      float umax = 0.f;  // fast instance: the unit's largest |v| in this block
      for (int j = 0; j < n; ++j) {
        const int t = g + j, st = t % kStages;
        if (!mbar_wait(&bars->kv_full[st], (t / kStages) & 1, abort_flag, p.err)) {
          ok = false;
          break;
        }
        uint4* blk = reinterpret_cast<uint4*>(sKV + C::v_box(st, has_block ? cw : 0));
        // converts the block with 2^-e; returns this thread's largest |v|
        auto convert = [&](int e) {
          const float sc = __int_as_float((127 - e) << 23);  // 2^-e, exact
          const float2 sc2 = make_float2(sc, sc);
          float mx = 0.f;
#pragma unroll 1
          for (int h = 0; h < kIters; ++h) {
            uint4 w[8];
#pragma unroll
            for (int q = 0; q < 8; ++q) w[q] = blk[h * 256 + 32 * q + lane];
#pragma unroll
            for (int q = 0; q < 8; ++q) {
              float2 f0 = bf16x2_to_float2(w[q].x), f1 = bf16x2_to_float2(w[q].y);
              float2 f2v = bf16x2_to_float2(w[q].z), f3 = bf16x2_to_float2(w[q].w);
              mx = fmax3(mx, fabsf(f0.x), fabsf(f0.y));
              mx = fmax3(mx, fabsf(f1.x), fabsf(f1.y));
              mx = fmax3(mx, fabsf(f2v.x), fabsf(f2v.y));
              mx = fmax3(mx, fabsf(f3.x), fabsf(f3.y));
              if (e != 0) {
                f0 = __fmul2_rn(f0, sc2);
                f1 = __fmul2_rn(f1, sc2);
                f2v = __fmul2_rn(f2v, sc2);
                f3 = __fmul2_rn(f3, sc2);
              }
              w[q] = make_uint4(float2_to_f16x2(f0.x, f0.y), float2_to_f16x2(f1.x, f1.y),
                                float2_to_f16x2(f2v.x, f2v.y), float2_to_f16x2(f3.x, f3.y));
              blk[h * 256 + 32 * q + lane] = w[q];
            }
          }
          return mx;
        };
        if (!SAFE) {
          // fast instance: V as it is; the unit's largest |v| decides whether
          // the unit is handed to the recomputing instance
          if (has_block) {
            const float mx =
                __uint_as_float(__reduce_max_sync(0xffffffffu, __float_as_uint(convert(0))));
            umax = j == 0 ? mx : fmaxf(umax, mx);
            fence_proxy_async_smem();
            __syncwarp();
          }
          if (j == n - 1 && lane == 0) {
            // out of range: nonzero and below 2^kVLowBits, at least
            // 2^(kVHeadroomBits + 1), or not finite
            const bool oor = has_block && umax > 0.f &&
                             !(umax >= exp2f((float)kVLowBits) &&
                               umax < exp2f((float)(kVHeadroomBits + 1)));
            *reinterpret_cast<volatile unsigned long long*>(&bars->vunit[uc & 7][cw]) =
                (unsigned long long)(uint32_t)uc | ((unsigned long long)(oor ? 1u : 0u) << 32);
          }
        } else if (has_block) {
          const int used = j == 0 ? 0 : ve;
          // warp max (|v| >= 0: its fp32 bits order like the values)
          const float mx =
              __uint_as_float(__reduce_max_sync(0xffffffffu, __float_as_uint(convert(used))));
          // the exponent this block asks for: 0 while its largest |v| lies in
          // [2^kVLowBits, 2^(kVHeadroomBits + 1)); else floor(log2 max) - 14
          // (inf and NaN count as 2^128: their results are reported anyway)
          int e = 0;
          if (mx > 0.f) {
            const int fl = isfinite(mx) ? ((int)((__float_as_uint(mx) >> 23) & 0xff) - 127) : 128;
            if (fl < kVLowBits || fl > kVHeadroomBits)
              e = min(kVExpMax, max(kVExpMin, fl - kVHeadroomBits));
          }
          const int want = j == 0 ? e : max(ve, e);
          if (want != used) {
            // converted with the wrong scale: fetch the block again and redo
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) {
              mbar_arrive_expect_tx(&bars->v_reload[cw], C::KV_BOX);
              tma_load_4d(sKV + C::v_box(st, cw), &vmap, &bars->v_reload[cw], cw * 64, hk,
                          x.row0 + j * kBN, x.bc);
            }
            if (!mbar_wait(&bars->v_reload[cw], reloads & 1, abort_flag, p.err)) {
              ok = false;
              break;
            }
            ++reloads;
            convert(want);
          }
          ve = want;
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0)  // one 8-byte write: (tile, E)
            *reinterpret_cast<volatile unsigned long long*>(&bars->vtag[st][cw]) =
                (unsigned long long)(uint32_t)t | ((unsigned long long)(uint32_t)ve << 32);
        }
        if (lane == 0) mbar_arrive(&bars->v_ready[st]);
      }
      g += n;
      if (n > 0) ++uc;
    }
  } else {
    // ------------------------------------------------------------ softmax + epilogue
    const int si = tid - 128;                      // 0 .. 255
    const int half = si >> 7;                      // which 32 keys of each tile
    const int qd = warp & 3;                       // TMEM lane quadrant
    const int r = qd * 32 + lane;                  // row within the tile = TMEM lane
    const uint32_t lane_addr = tbase + ((uint32_t)(qd * 32) << 16);
    const uint32_t my_cols = (uint32_t)(half * kHalf);  // first S/T column of this half
    const int bar_id = 1 + qd;                     // named barrier of the row's two warps
    const bool qpos = p.qscale >= 0.f;
    int g = 0, xs = 0, uc = 0;  // uc: units with work so far
    bool ok = true, finite = true;
    // A wait of this thread gave up (sticky).  The thread carries on through
    // the same steps (its TMEM and memory accesses stay in bounds; the values
    // no longer matter) and passes the flag to its partner with the partial
    // maxima, as a negative max |t|: both threads of the row leave at the same
    // exchange, so neither is left waiting at the named barrier.
    bool failed = false;
    for (int u = blockIdx.x; ok && u < p.units; u += gridDim.x) {
      const Unit x = unit_at<VARLEN, SAFE>(p, u, umask);
      if (x.n == 0) continue;  // (varlen) no such query tile
      const int i = x.mt * kBM + r;
      // Running max m (log2 units of the scaled scores); P = 2^(s - m) <= 2^8
      // (lazy rescaling).  eu (>= 0) keeps P t 2^-eu in fp16's range.
      float m_run = -INFINITY;
      int eu = 0;
      // block exponents of the V column blocks of O and U (see the converters)
      int ve[2] = {0, 0};
      float tlim = (float)(1 << kTBits), tsc = 1.f;  // 2^(kTBits + eu), 2^-eu
      // Tile t-1's block exponents, checked one tile late (the converters are
      // long done by then): where they changed, PV of t-1 waits until O and U
      // (V columns only) have been brought to the new scale here.
      auto v_check = [&](int tp, int jp) {
        int e[2];
        if (!read_vtags<C::KB>(bars->vtag, tp, e, abort_flag, p.err)) return false;
        if (jp > 0 && (e[0] != ve[0] || e[1] != ve[1])) {
          const uint32_t base = lane_addr + (half == 0 ? C::COL_O : C::COL_U);
          const float f0 = exp2f((float)(ve[0] - e[0])), f1 = exp2f((float)(ve[1] - e[1]));
#pragma unroll 1
          for (int cc = 0; cc < D; cc += 64) {
            const float f = cc < 64 ? f0 : f1;
            uint32_t wa[32], wb[32];
            tmem_ld2x32_sync(base + cc, base + cc + 32, wa, wb);
#pragma unroll
            for (int q = 0; q < 32; ++q) {
              wa[q] = __float_as_uint(__uint_as_float(wa[q]) * f);
              wb[q] = __float_as_uint(__uint_as_float(wb[q]) * f);
            }
            tmem_st32(base + cc, wa);
            tmem_st32(base + cc + 32, wb);
          }
          tmem_wait_st();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&bars->v_rescaled);
        }
        ve[0] = e[0];
        ve[1] = e[1];
        return true;
      };
      for (int j = 0; j < x.n; ++j) {
        const int t = g + j;
        if (SAFE && j > 0 && !v_check(t - 1, j - 1)) failed = true;
        if (!mbar_wait(&bars->s_full, t & 1, abort_flag, p.err)) failed = true;
        tc_fence_after();
        uint32_t sv[kHalf], tv[kHalf];
        tmem_ld2x32_sync(lane_addr + C::COL_S + my_cols, lane_addr + C::COL_T + my_cols, sv, tv);
        // S and T are in registers: the tensor core may overwrite them
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars->s_free);
        const int key0 = j * kBN + half * kHalf;  // first key of this half
        const int lim = p.causal ? i : x.len - 1;  // last visible key of the row
        const int nvis = max(0, min(kHalf, lim - key0 + 1));
        // partial extreme of the raw scores (max if scale >= 0) and max |t|
        float e2[2], t2[2];
#pragma unroll
        for (int q = 0; q < 2; ++q) {
          e2[q] = qpos ? -INFINITY : INFINITY;
          t2[q] = 0.f;
        }
        if (nvis == kHalf) {
#pragma unroll
          for (int c = 0; c < kHalf; c += 2) {
            const float a = __uint_as_float(sv[c]), b = __uint_as_float(sv[c + 1]);
            e2[(c >> 1) & 1] = qpos ? fmax3(e2[(c >> 1) & 1], a, b) : fmin3(e2[(c >> 1) & 1], a, b);
            t2[(c >> 1) & 1] = fmax3(t2[(c >> 1) & 1], fabsf(__uint_as_float(tv[c])),
                                     fabsf(__uint_as_float(tv[c + 1])));
          }
        } else {
#pragma unroll
          for (int c = 0; c < kHalf; ++c) {
            const float v = __uint_as_float(sv[c]);
            if (c < nvis) {
              e2[c & 1] = qpos ? fmaxf(e2[c & 1], v) : fminf(e2[c & 1], v);
              t2[c & 1] = fmaxf(t2[c & 1], fabsf(__uint_as_float(tv[c])));
            }
          }
        }
        const float ext = qpos ? fmaxf(e2[0], e2[1]) : fminf(e2[0], e2[1]);
        float part_max = (nvis > 0) ? ext * p.qscale : -INFINITY;
        float tmax = fmaxf(t2[0], t2[1]);
        // combine with the partner half of the row
        xch->tile[xs & 1][half][r] = make_float2(part_max, failed ? -1.f : tmax);
        named_bar_sync(bar_id, 64);
        {
          const float2 o = xch->tile[xs & 1][half ^ 1][r];
          if (failed || o.y < 0.f) {
            ok = false;
            break;
          }
          part_max = fmaxf(part_max, o.x);
          tmax = fmaxf(tmax, o.y);
        }
        ++xs;
        const float m_new = fmaxf(m_run, part_max);
        const bool resc = (m_run != -INFINITY) && (m_new > m_run + (float)kRescaleBits);
        if (m_run == -INFINITY) m_run = m_new;
        int eu_new = eu;
        if (tmax >= tlim) eu_new = max(eu, (int)ceilf(log2f(tmax)) - (kTBits - 1));
        const bool ubump = eu_new > eu;
        // O and U (with l, z) are rescaled below, after P and P t are stored;
        // P and P t already use the new m and eu.  (The partner warp holds the
        // same rows, so both warps of a row take the branch together.)
        const bool rescale = __any_sync(0xffffffffu, resc || ubump);
        float fr = 1.f;  // this half's factor: half 0 rescales O (and l), half 1 U (and z)
        if (rescale) {
          const float alpha = resc ? exp2f(m_run - m_new) : 1.f;
          fr = half == 0 ? alpha : alpha * exp2f((float)(eu - eu_new));
          if (resc) m_run = m_new;
          if (ubump) {
            eu = eu_new;
            tlim = exp2f((float)(eu + kTBits));
            tsc = exp2f((float)-eu);
          }
        }
        // P = 2^(s - m) as fp16 pairs
        const bool live = m_run != -INFINITY;
        uint32_t pk[kHalf / 2];
        if (live && nvis == kHalf) {
          const float2 qs2 = make_float2(p.qscale, p.qscale), nm2 = make_float2(-m_run, -m_run);
#pragma unroll
          for (int c = 0; c < kHalf / 2; ++c) {
            const float2 xs = __ffma2_rn(
                make_float2(__uint_as_float(sv[2 * c]), __uint_as_float(sv[2 * c + 1])), qs2, nm2);
            const float2 pp = ((kPolyPairs >> c) & 1u)
                                  ? exp2_poly2(xs)
                                  : make_float2(fast_exp2(xs.x), fast_exp2(xs.y));
            sv[2 * c] = __float_as_uint(pp.x);
            sv[2 * c + 1] = __float_as_uint(pp.y);
            pk[c] = float2_to_f16x2(pp.x, pp.y);
          }
        } else {
#pragma unroll
          for (int c = 0; c < kHalf / 2; ++c) {
            float p0 = fast_exp2(fmaf(__uint_as_float(sv[2 * c]), p.qscale, -m_run));
            float p1 = fast_exp2(fmaf(__uint_as_float(sv[2 * c + 1]), p.qscale, -m_run));
            if (!live || 2 * c >= nvis) p0 = 0.f;
            if (!live || 2 * c + 1 >= nvis) p1 = 0.f;
            sv[2 * c] = __float_as_uint(p0);
            sv[2 * c + 1] = __float_as_uint(p1);
            pk[c] = float2_to_f16x2(p0, p1);
          }
        }
        // the P columns (and O, U) are free once the previous tile's PV has completed
        if (j > 0 && !mbar_wait(&bars->o_done, (t - 1) & 1, abort_flag, p.err)) failed = true;
        tc_fence_after();
        tmem_st16(lane_addr + C::COL_P + my_cols / 2, pk);
        // P t 2^-eu as fp16 pairs
        {
          const float2 tsc2 = make_float2(tsc, tsc);
#pragma unroll
          for (int c = 0; c < kHalf / 2; ++c) {
            const float2 q2 = __fmul2_rn(
                make_float2(__uint_as_float(sv[2 * c]), __uint_as_float(sv[2 * c + 1])),
                __fmul2_rn(make_float2(__uint_as_float(tv[2 * c]), __uint_as_float(tv[2 * c + 1])),
                           tsc2));
            pk[c] = float2_to_f16x2(q2.x, q2.y);
          }
        }
        tmem_st16(lane_addr + C::COL_PT + my_cols / 2, pk);
        if (rescale) {
          const uint32_t base = lane_addr + (half == 0 ? C::COL_O : C::COL_U);
#pragma unroll 1
          for (int cc = 0; cc < D; cc += 64) {
            uint32_t wa[32], wb[32];
            tmem_ld2x32_sync(base + cc, base + cc + 32, wa, wb);
#pragma unroll
            for (int e = 0; e < 32; ++e) {
              wa[e] = __float_as_uint(__uint_as_float(wa[e]) * fr);
              wb[e] = __float_as_uint(__uint_as_float(wb[e]) * fr);
            }
            tmem_st32(base + cc, wa);
            tmem_st32(base + cc + 32, wb);
          }
          uint32_t w[16];
          tmem_ld16_sync(base + D, w);
#pragma unroll
          for (int e = 0; e < 16; ++e) w[e] = __float_as_uint(__uint_as_float(w[e]) * fr);
          tmem_st16(base + D, w);
        }
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars->p_full);
      }
      if (!ok) break;
      // ---- epilogue: out = ((1 + z/l) o - u) / l, lse = ln(sum exp(scale s));
      // l and z are the ones-columns of O and U; each half writes half the row.
      const int tl = g + x.n - 1;
      if (SAFE && !v_check(tl, x.n - 1)) failed = true;
      bool oor = false;  // fast instance: this unit's V is out of range (marker)
      if constexpr (!SAFE) {
        // posted by the converters with the unit count once the unit's last V
        // tile was converted (long ago by now)
        for (int c = 0; c < C::KB; ++c) {
          volatile const unsigned long long* tag =
              reinterpret_cast<volatile const unsigned long long*>(&bars->vunit[uc & 7][c]);
          unsigned long long w = *tag;
          const uint64_t t0 = globaltimer_ns();
          for (uint32_t spins = 1; (int)(uint32_t)w != uc; ++spins) {
            if ((spins & 63u) == 0 &&
                (*abort_flag || globaltimer_ns() - t0 > wait_limit_ns(p.err) ||
                 spins >= kWaitMaxPolls)) {
              if (!*abort_flag) record_error(p.err, kDevTimeoutMbarrier);
              *abort_flag = 1;
              break;
            }
            w = *tag;
          }
          if ((int)(uint32_t)w != uc) failed = true;
          oor = oor || (w >> 32) != 0;
        }
        ++uc;
      }
      if (!mbar_wait(&bars->o_done, tl & 1, abort_flag, p.err)) failed = true;
      tc_fence_after();
      uint32_t lw, zw;
      tmem_ld2x1_sync(lane_addr + C::COL_O + D, lane_addr + C::COL_U + D, lw, zw);
      const float l = __uint_as_float(lw), z = __uint_as_float(zw);
      const float inv = 1.f / l;
      const float usc = exp2f((float)eu);           // undo the P t scaling
      const float c1 = (1.f + z * usc * inv) * inv;
      const float cu = usc * inv;
      const float vsc0 = exp2f((float)ve[0]), vsc1 = exp2f((float)ve[1]);
      OutT* orow = static_cast<OutT*>(p.out) + (((size_t)x.tok0 + i) * p.Hq + x.h) * D;
#pragma unroll 1
      for (int cc = half * (D / 2); cc < (half + 1) * (D / 2); cc += 32) {
        uint32_t ov[32], uv[32];
        tmem_ld2x32_sync(lane_addr + C::COL_O + cc, lane_addr + C::COL_U + cc, ov, uv);
        const float vsc = cc < 64 ? vsc0 : vsc1;  // undo the block scaling of V
        const float c1v = c1 * vsc, cuv = cu * vsc;
        float a[32];
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          a[e] = __uint_as_float(ov[e]) * c1v - __uint_as_float(uv[e]) * cuv;
          finite = finite && (oor || isfinite(a[e]));
        }
        if (i < x.len) {
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
      if (half == 0 && p.lse && i < x.len)
        p.lse[x.lse0 + i] = (m_run + log2f(l)) * 0.6931471805599453f;
      if (oor && half == 0 && r == 0) {
        // hand the unit to the recomputing instance (its first row, column 0;
        // the row itself is rewritten there)
        if constexpr (sizeof(OutT) == 2)
          reinterpret_cast<uint16_t*>(orow)[0] = kMarkBf16;
        else
          reinterpret_cast<uint32_t*>(orow)[0] = kMarkF32;
      }
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

template <int D, typename OutT, bool VARLEN>
cudaError_t launch_d(const PrefillTcArgs& a, cudaStream_t stream) {
  using C = TcCfg<D>;
  CUtensorMap qm, rm, km, vm;
  // varlen: the packed [T, H, d] tensors as one batch of T rows
  const int mb = VARLEN ? 1 : a.B, ms = VARLEN ? a.total : a.L;
  cudaError_t e = encode_sw128(&qm, a.q, mb, ms, a.Hq, D, kBM);
  if (e == cudaSuccess) e = encode_sw128(&rm, a.rho, mb, ms, a.Hq, D, kBM);
  if (e == cudaSuccess) e = encode_sw128(&km, a.k, mb, ms, a.Hkv, D, kBN);
  if (e == cudaSuccess) e = encode_sw128(&vm, a.v, mb, ms, a.Hkv, D, kBN);
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
  p.cu_seqlens = a.cu_seqlens;
  p.total = a.total;
  const int smem =
      1024 + C::TILE_SMEM + (int)sizeof(Xchg) + (int)sizeof(Bars) + 16 + kMaskUnits / 8;
  static_assert(1024 + TcCfg<D>::TILE_SMEM + sizeof(Xchg) + sizeof(Bars) + 16 + kMaskUnits / 8 <=
                    227 * 1024,
                "shared memory");
  // the fast instance over every unit ...
  auto fast = plx_prefill_tc_kernel<D, OutT, VARLEN, false>;
  e = cudaFuncSetAttribute(fast, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  const int grid = (int)(units < a.num_sms ? units : a.num_sms);
  fast<<<grid, kThreads, smem, stream>>>(qm, rm, km, vm, p);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  // ... then the recomputing instance over the units it marked (a CTA with no
  // marked unit returns after one read per unit)
  auto safe = plx_prefill_tc_kernel<D, OutT, VARLEN, true>;
  e = cudaFuncSetAttribute(safe, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  long long sgrid = (units + kMaskUnits - 1) / kMaskUnits;
  if (sgrid < grid) sgrid = grid;
  if (sgrid > 0x7fffffffll) return cudaErrorInvalidValue;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)sgrid);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  e = cudaLaunchKernelEx(&cfg, safe, qm, rm, km, vm, p);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace

template <bool VARLEN>
cudaError_t launch_v(const PrefillTcArgs& a, cudaStream_t stream) {
  if (a.d == 128)
    return a.out_f32 ? launch_d<128, float, VARLEN>(a, stream)
                     : launch_d<128, __nv_bfloat16, VARLEN>(a, stream);
  if (a.d == 64)
    return a.out_f32 ? launch_d<64, float, VARLEN>(a, stream)
                     : launch_d<64, __nv_bfloat16, VARLEN>(a, stream);
  return cudaErrorInvalidValue;
}

cudaError_t launch_prefill_tc(const PrefillTcArgs& a, cudaStream_t stream) {
  return a.cu_seqlens ? launch_v<true>(a, stream) : launch_v<false>(a, stream);
}

}  // namespace plx
