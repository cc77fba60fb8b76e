// plx_probe_gemm.cu -- the probe projection rho = W_R x (page 1 "Parallax:
// Parameterized Local Linear Attention Gives Transformers a 'Second Eye'",
// section 1.3: the one extra projection matrix; page 3 "Parallax keeps
// softmax, adds covariance correction branch": rho_i = W_R x_i).
//
// For all tokens at once this is the GEMM rho[M, N] = x[M, K] W_R[N, K]^T
// (M tokens, K = model width, N = H_q d), run on the 5th-generation tensor
// cores for bf16: a 192 KB ring fed by TMA (128-byte swizzle) with a 128 x 64
// x tile and one or two W_R tiles per stage, tcgen05.mma (M = 128, K = 16)
// issued by one thread, and eight epilogue warps that read a unit's sums
// (tcgen05.ld), round them to bf16 and store.  A unit is one 128 x 128 output
// tile or a pair of adjacent ones; a pair's two W_R tiles lie back to back in
// the stage, so one N = 256 product covers both.  Products into the same
// accumulator complete one after the other (each waits for the previous sum),
// and one such chain keeps the tensor core about half busy, so the even and
// odd k steps accumulate into two accumulators (256 columns each) that the
// epilogue adds: two chains in flight.  The epilogue releases TMEM as soon as
// the sums are in registers and stores while the next unit accumulates.
// Four schedules by the number of output tiles:
//   * at least one 256 x 256 tile per pair of SMs: the SM-pair kernel below
//     (tcgen05 cta_group::2), persistent clusters of two CTAs;
//   * pairs of 128 x 128 tiles (four ring stages), persistent CTAs, when
//     their waves cost no more than single tiles' (a pair moves 1.5 times the
//     bytes);
//   * single tiles (six ring stages), persistent CTAs;
//   * fewer tiles than half the SMs (the decode batch, M of a few dozen): a
//     cluster of up to 8 CTAs per tile (the largest whose clusters all fit at
//     once), each summing its share of the k blocks.  With so few tiles the
//     time is the ring's round trips to memory, so spreading the W_R stream
//     over more SMs is what shortens it.  The fp32 partial tiles meet in
//     shared memory; every CTA of the cluster reads all of them (distributed
//     shared memory) for its slice of the rows, adds them in rank order and
//     stores.
// fp32 inputs take a plain CUDA-core kernel (the correctness path).
#include <atomic>

#include "plx_launch.h"

namespace plx {

namespace {

constexpr int kPM = 128, kPN = 128, kPK = 64;  // output tile, k block (128-byte rows)
constexpr int kPRingBytes = 192 * 1024;       // four stages of pairs or six of single tiles
constexpr int kPMaxStages = 6;
constexpr int kPThreads = 384;                 // warps: 0 TMA, 1 MMA, 2 TMEM, 4-11 epilogue
constexpr int kPEpiWarps = 8;                  // two per TMEM lane quadrant
constexpr int kPAccCols = 256;                 // accumulator of the even k steps; the odd ones follow
constexpr int kPTileBytes = kPM * kPK * 2;     // one A (or B) tile, 16 KB
constexpr int kPPartStride = kPN + 4;          // fp32 partial tile row (floats), conflict-free
constexpr uint32_t kPIdesc1 = umma_idesc_f16kind(kPM, kPN, false, false);      // one W_R tile
constexpr uint32_t kPIdesc2 = umma_idesc_f16kind(kPM, 2 * kPN, false, false);  // two, as one N = 256 operand
static_assert(kPM * kPPartStride * 4 <= kPRingBytes, "partial tile fits the ring");
constexpr int kPMaxSplit = 8;  // cluster size (portable limit)

struct ProjBars {
  uint64_t full[kPMaxStages], empty[kPMaxStages];
  uint64_t acc_full, acc_empty;
  uint64_t drain;
};

struct ProjParams {
  void* rho;
  int M, N, K;
  int tiles_n;   // 128-column output tiles
  int pair;      // 1 or 2 N tiles per unit
  int units_n;   // units per 128-row M tile
  int units;
  int kblocks;   // 64-wide k blocks
  int ksplit;    // CTAs per unit (a cluster); 1: persistent CTAs
  int stages;    // ring stages of stage_bytes: an x tile and `pair` W_R tiles
  int stage_bytes;
  unsigned* err;
};

__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}

// every thread of every CTA of the cluster; shared-memory writes before it are
// visible to the cluster's reads after it
__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::
                   : "memory");
}

__device__ __forceinline__ float4 ld_cluster_f4(uint32_t local_addr, uint32_t rank) {
  uint32_t a;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(a) : "r"(local_addr), "r"(rank));
  float4 v;
  asm volatile("ld.shared::cluster.v4.f32 {%0, %1, %2, %3}, [%4];"
               : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
               : "r"(a)
               : "memory");
  return v;
}

__device__ __forceinline__ void unit_coords(const ProjParams& p, int u, int& mb, int& nb,
                                            bool& two) {
  mb = u / p.units_n;
  nb = p.pair * (u % p.units_n);
  two = p.pair == 2 && nb + 1 < p.tiles_n;
}

__global__ void __launch_bounds__(kPThreads, 1)
    plx_probe_gemm_kernel(const __grid_constant__ CUtensorMap xmap,
                          const __grid_constant__ CUtensorMap wmap, const ProjParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  ProjBars* bars = reinterpret_cast<ProjBars*>(smem + kPRingBytes);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  // this CTA's units and k blocks: with ksplit > 1 the grid is one cluster
  // of ksplit CTAs per unit, rank kr summing k blocks [kb0, kb1)
  const int ks = p.ksplit;
  const int kr = ks > 1 ? (int)cluster_rank() : 0;
  const int kb0 = (int)((long long)p.kblocks * kr / ks);
  const int kb1 = (int)((long long)p.kblocks * (kr + 1) / ks);
  const int u_first = blockIdx.x / ks, u_step = gridDim.x / ks;

  // a kernel launched after this one as its programmatic dependent (the
  // attention that reads rho) waits for this grid's completion before it
  // reads anything, so it may be placed on free SMs at once
  grid_dep_launch_dependents();
  if (tid == 0) {
    *abort_flag = 0;
    for (int s = 0; s < p.stages; ++s) {
      mbar_init(&bars->full[s], 1);
      mbar_init(&bars->empty[s], 1);
    }
    mbar_init(&bars->acc_full, 1);
    mbar_init(&bars->acc_empty, kPEpiWarps);  // one arrival per epilogue warp
    mbar_init(&bars->drain, 1);
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
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      tma_prefetch_desc(&xmap);
      tma_prefetch_desc(&wmap);
      int s = 0;            // ring stage
      uint32_t round = 0;   // passes over the ring so far
      bool ok = true;
      for (int u = u_first; ok && u < p.units; u += u_step) {
        int mb, nb;
        bool two;
        unit_coords(p, u, mb, nb, two);
        for (int kb = kb0; kb < kb1; ++kb) {
          if (round > 0 && !mbar_wait(&bars->empty[s], (round - 1) & 1u, abort_flag, p.err)) {
            ok = false;
            break;
          }
          uint8_t* st = smem + s * p.stage_bytes;
          mbar_arrive_expect_tx(&bars->full[s], (two ? 3 : 2) * kPTileBytes);
          tma_load_2d(st, &xmap, &bars->full[s], kb * kPK, mb * kPM);
          tma_load_2d(st + kPTileBytes, &wmap, &bars->full[s], kb * kPK, nb * kPN);
          if (two) tma_load_2d(st + 2 * kPTileBytes, &wmap, &bars->full[s], kb * kPK, (nb + 1) * kPN);
          if (++s == p.stages) {
            s = 0;
            ++round;
          }
        }
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
      const uint64_t d0 = smem_desc_sw128(smem_u32(smem), 16, 1024);
      int s = 0;
      uint32_t round = 0;
      int lt = 0;
      bool ok = true;
      for (int u = u_first; ok && u < p.units; u += u_step, ++lt) {
        int mb, nb;
        bool two;
        unit_coords(p, u, mb, nb, two);
        // the epilogue has taken the previous unit's sums out of TMEM
        if (lt > 0 && !mbar_wait(&bars->acc_empty, (uint32_t)((lt - 1) & 1), abort_flag, p.err)) {
          ok = false;
          break;
        }
        tc_fence_after();
        // a pair's two W_R tiles are contiguous in the stage: one N = 256 operand
        const uint32_t idesc = two ? kPIdesc2 : kPIdesc1;
        for (int kb = kb0; kb < kb1; ++kb) {
          if (!mbar_wait(&bars->full[s], round & 1u, abort_flag, p.err)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sa = (uint32_t)(s * p.stage_bytes) >> 4;
          const uint32_t sb = (uint32_t)(s * p.stage_bytes + kPTileBytes) >> 4;
          // even k steps into the first accumulator, odd ones into the second
#pragma unroll
          for (int k = 0; k < kPK / 16; ++k)
            umma_ss(tbase + (k & 1) * kPAccCols, d0 + sa + 2 * k, d0 + sb + 2 * k, idesc,
                    (kb > kb0 || k > 1) ? 1u : 0u);
          umma_commit(&bars->empty[s]);  // the stage is free once these MMAs complete
          if (++s == p.stages) {
            s = 0;
            ++round;
          }
        }
        if (!ok) break;
        umma_commit(&bars->acc_full);
      }
      // every MMA must have completed before the columns are released
      umma_commit(&bars->drain);
      volatile int never = 0;
      mbar_wait(&bars->drain, 0, &never, p.err);
    }
    __syncwarp();
  } else if (warp >= 4) {
    // ------------------------------------------------------------ epilogue
    const int qd = warp & 3;                     // TMEM lane quadrant (warp id mod 4)
    const int half = (warp - 4) >> 2;            // which half of the unit's columns
    const int r = qd * 32 + lane;                // row of the tile = TMEM lane
    const uint32_t lane_addr = tbase + ((uint32_t)(qd * 32) << 16);
    int lt = 0;
    for (int u = u_first; u < p.units; u += u_step, ++lt) {
      if (!mbar_wait(&bars->acc_full, (uint32_t)(lt & 1), abort_flag, p.err)) break;
      tc_fence_after();
      int mb, nb0;
      bool two;
      unit_coords(p, u, mb, nb0, two);
      const int hcols = two ? kPN : kPN / 2;     // this warp's columns
      const int c0 = half * hcols;               // the first, within the unit
      uint32_t packed[kPN / 2];                  // bf16 pairs of the sums
#pragma unroll
      for (int j = 0; j < kPN / 32; ++j) {
        if (32 * j < hcols) {
          uint32_t a[32], b[32];
          tmem_ld2x32_sync(lane_addr + c0 + 32 * j, lane_addr + kPAccCols + c0 + 32 * j, a, b);
          if (ks > 1) {
            // this CTA's share of the sum, kept in shared memory (the ring is
            // idle: every load was consumed by the products acc_full follows)
            float* part = reinterpret_cast<float*>(smem) + r * kPPartStride + c0 + 32 * j;
#pragma unroll
            for (int q = 0; q < 8; ++q)
              *reinterpret_cast<float4*>(part + 4 * q) = make_float4(
                  __uint_as_float(a[4 * q]) + __uint_as_float(b[4 * q]),
                  __uint_as_float(a[4 * q + 1]) + __uint_as_float(b[4 * q + 1]),
                  __uint_as_float(a[4 * q + 2]) + __uint_as_float(b[4 * q + 2]),
                  __uint_as_float(a[4 * q + 3]) + __uint_as_float(b[4 * q + 3]));
          } else {
#pragma unroll
            for (int q = 0; q < 16; ++q)
              packed[16 * j + q] =
                  float2_to_bf16x2(__uint_as_float(a[2 * q]) + __uint_as_float(b[2 * q]),
                                   __uint_as_float(a[2 * q + 1]) + __uint_as_float(b[2 * q + 1]));
          }
        }
      }
      // the sums are in registers: the next unit may overwrite the accumulators
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->acc_empty);
      const long long row = (long long)mb * kPM + r;
      if (ks == 1 && row < p.M) {
        __nv_bfloat16* dst = static_cast<__nv_bfloat16*>(p.rho) + row * p.N;
#pragma unroll
        for (int g = 0; g < kPN / 8; ++g) {
          const int col = nb0 * kPN + c0 + 8 * g;
          if (8 * g < hcols && col + 8 <= p.N)
            *reinterpret_cast<uint4*>(dst + col) =
                make_uint4(packed[4 * g], packed[4 * g + 1], packed[4 * g + 2], packed[4 * g + 3]);
        }
      }
    }
  }
  __syncthreads();
  if (ks > 1) {
    // every CTA of the cluster reaches both barriers (all waits above are
    // bounded); the second keeps each partial tile alive until all have read it
    cluster_sync();
    if (blockIdx.x / ks < p.units) {
      int mb, nb;
      bool two;
      unit_coords(p, blockIdx.x / ks, mb, nb, two);
      const int rows = min(kPM, p.M - mb * kPM);
      const int items = rows * (kPN / 4);  // float4 groups of the tile
      const int i0 = (int)((long long)items * kr / ks), i1 = (int)((long long)items * (kr + 1) / ks);
      const uint32_t part0 = smem_u32(smem);
      for (int i = i0 + tid; i < i1; i += kPThreads) {
        const int row = i / (kPN / 4), c4 = i % (kPN / 4);
        const uint32_t off = part0 + (uint32_t)(row * kPPartStride + 4 * c4) * 4u;
        // all loads first (independent), then the sum in rank order
        float4 b[kPMaxSplit];
#pragma unroll
        for (int s2 = 0; s2 < kPMaxSplit; ++s2)
          if (s2 < ks) b[s2] = ld_cluster_f4(off, (uint32_t)s2);
        float4 a = b[0];
#pragma unroll
        for (int s2 = 1; s2 < kPMaxSplit; ++s2)
          if (s2 < ks) {
            a.x += b[s2].x;
            a.y += b[s2].y;
            a.z += b[s2].z;
            a.w += b[s2].w;
          }
        const int col = nb * kPN + 4 * c4;
        if (col + 4 <= p.N) {
          uint2 w;
          w.x = float2_to_bf16x2(a.x, a.y);
          w.y = float2_to_bf16x2(a.z, a.w);
          *reinterpret_cast<uint2*>(static_cast<__nv_bfloat16*>(p.rho) +
                                    ((long long)mb * kPM + row) * p.N + col) = w;
        }
      }
    }
    cluster_sync();
  }
  if (warp == 2) {
    tc_fence_after();
    tmem_dealloc(tbase, 512);
  }
}

// ---------------------------------------------------------------------------
// Pairs of SMs (tcgen05 cta_group::2): for many tiles, a cluster of two CTAs
// computes a 256 x 256 output tile with M = 256, N = 256 products issued by
// the even CTA.  Each CTA stages its own 128 rows of x and its own 128 rows of
// W_R (one tile each, 32 KB per k block, six stages), and each SM's tensor
// core multiplies its x rows by both CTAs' W_R rows, so a CTA moves 32 KB
// through shared memory per k block for a 128 x 256 share of the output where
// the one-SM pair of tiles moves 48 KB.  Both CTAs' loads complete on the even
// CTA's stage barrier, the products' completion is signalled to both CTAs'
// barriers, and both CTAs' epilogue warps release the accumulators on the even
// CTA's barrier.
// ---------------------------------------------------------------------------
constexpr uint32_t kPIdescPair = umma_idesc_f16kind(2 * kPM, 2 * kPN, false, false);
constexpr int kPPairStages = kPRingBytes / (2 * kPTileBytes);
static_assert(kPPairStages <= kPMaxStages, "stage barriers");

__device__ __forceinline__ uint32_t cluster_addr(uint32_t local_addr, uint32_t rank) {
  uint32_t a;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(a) : "r"(local_addr), "r"(rank));
  return a;
}
__device__ __forceinline__ void tmem_alloc_pair(uint32_t* smem_dst, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                   smem_u32(smem_dst)),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish_pair() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void umma_ss_pair(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                             uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// arrive on the barrier at this offset in each CTA of `mask` once the products
// issued so far have completed
__device__ __forceinline__ void umma_commit_pair(uint64_t* bar, uint16_t mask) {
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64"
      " [%0], %1;" ::"r"(smem_u32(bar)),
      "h"(mask)
      : "memory");
}
// a tile into this CTA's shared memory, completing on a barrier of either CTA
// of the pair (bar: shared::cluster address)
__device__ __forceinline__ void tma_load_2d_pair(void* dst, const CUtensorMap* map, uint32_t bar,
                                                 int c0, int c1) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4}], [%2];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(c0), "r"(c1)
      : "memory");
}
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t bar) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(bar)
               : "memory");
}

// p.units = ceil(M / 256) ceil(N / 256) (units_n per 256-row M tile); the
// grid is two CTAs (one cluster) per resident unit.
__global__ void __launch_bounds__(kPThreads, 1)
    plx_probe_gemm_pair_kernel(const __grid_constant__ CUtensorMap xmap,
                               const __grid_constant__ CUtensorMap wmap, const ProjParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  ProjBars* bars = reinterpret_cast<ProjBars*>(smem + kPRingBytes);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint32_t rank = cluster_rank();  // 0: issues the products
  const int u_first = blockIdx.x / 2, u_step = gridDim.x / 2;
  constexpr int kStageBytes = 2 * kPTileBytes;  // x rows and W_R rows of this CTA

  grid_dep_launch_dependents();
  if (tid == 0) {
    *abort_flag = 0;
    for (int s = 0; s < kPPairStages; ++s) {
      mbar_init(&bars->full[s], 1);
      mbar_init(&bars->empty[s], 1);
    }
    mbar_init(&bars->acc_full, 1);
    mbar_init(&bars->acc_empty, 2 * kPEpiWarps);  // both CTAs' epilogue warps
    mbar_init(&bars->drain, 1);
    fence_mbarrier_init();
  }
  if (warp == 2) {
    tmem_alloc_pair(tmem_slot, 512);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  cluster_sync();  // barriers of both CTAs initialised, TMEM of both allocated
  tc_fence_after();
  const uint32_t tbase = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer (both CTAs)
    if (lane == 0) {
      tma_prefetch_desc(&xmap);
      tma_prefetch_desc(&wmap);
      const uint32_t full0 = cluster_addr(smem_u32(&bars->full[0]), 0);
      int s = 0;
      uint32_t round = 0;
      bool ok = true;
      for (int u = u_first; ok && u < p.units; u += u_step) {
        const int xrow = (u / p.units_n) * 2 * kPM + (int)rank * kPM;
        const int wrow = (u % p.units_n) * 2 * kPN + (int)rank * kPN;
        for (int kb = 0; kb < p.kblocks; ++kb) {
          if (round > 0 && !mbar_wait(&bars->empty[s], (round - 1) & 1u, abort_flag, p.err)) {
            ok = false;
            break;
          }
          uint8_t* st = smem + s * kStageBytes;
          if (rank == 0) mbar_arrive_expect_tx(&bars->full[s], 2 * kStageBytes);
          tma_load_2d_pair(st, &xmap, full0 + 8u * (uint32_t)s, kb * kPK, xrow);
          tma_load_2d_pair(st + kPTileBytes, &wmap, full0 + 8u * (uint32_t)s, kb * kPK, wrow);
          if (++s == kPPairStages) {
            s = 0;
            ++round;
          }
        }
      }
      if (*abort_flag) {
        const uint64_t t0 = globaltimer_ns();
        while (globaltimer_ns() - t0 < 100000) {
        }
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer (even CTA)
    if (lane == 0 && rank == 0) {
      const uint64_t d0 = smem_desc_sw128(smem_u32(smem), 16, 1024);
      int s = 0;
      uint32_t round = 0;
      int lt = 0;
      bool ok = true;
      for (int u = u_first; ok && u < p.units; u += u_step, ++lt) {
        if (lt > 0 && !mbar_wait(&bars->acc_empty, (uint32_t)((lt - 1) & 1), abort_flag, p.err)) {
          ok = false;
          break;
        }
        tc_fence_after();
        for (int kb = 0; kb < p.kblocks; ++kb) {
          if (!mbar_wait(&bars->full[s], round & 1u, abort_flag, p.err)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sa = (uint32_t)(s * kStageBytes) >> 4;
          const uint32_t sb = (uint32_t)(s * kStageBytes + kPTileBytes) >> 4;
#pragma unroll
          for (int k = 0; k < kPK / 16; ++k)
            umma_ss_pair(tbase + (k & 1) * kPAccCols, d0 + sa + 2 * k, d0 + sb + 2 * k,
                         kPIdescPair, (kb > 0 || k > 1) ? 1u : 0u);
          umma_commit_pair(&bars->empty[s], 0x3);  // both CTAs' stage s is free
          if (++s == kPPairStages) {
            s = 0;
            ++round;
          }
        }
        if (!ok) break;
        umma_commit_pair(&bars->acc_full, 0x3);
      }
      umma_commit_pair(&bars->drain, 0x1);
      volatile int never = 0;
      mbar_wait(&bars->drain, 0, &never, p.err);
    }
    __syncwarp();
  } else if (warp >= 4) {
    // ------------------------------------------------------------ epilogue (both CTAs)
    const int qd = warp & 3;
    const int half = (warp - 4) >> 2;
    const int r = qd * 32 + lane;
    const uint32_t lane_addr = tbase + ((uint32_t)(qd * 32) << 16);
    const uint32_t acc_empty0 = cluster_addr(smem_u32(&bars->acc_empty), 0);
    int lt = 0;
    for (int u = u_first; u < p.units; u += u_step, ++lt) {
      if (!mbar_wait(&bars->acc_full, (uint32_t)(lt & 1), abort_flag, p.err)) break;
      tc_fence_after();
      const int c0 = half * kPN;  // this warp's 128 of the tile's 256 columns
      uint32_t packed[kPN / 2];
#pragma unroll
      for (int j = 0; j < kPN / 16; ++j) {
        uint32_t a[16], b[16];
        tmem_ld2x16_sync(lane_addr + c0 + 16 * j, lane_addr + kPAccCols + c0 + 16 * j, a, b);
#pragma unroll
        for (int q = 0; q < 8; ++q)
          packed[8 * j + q] =
              float2_to_bf16x2(__uint_as_float(a[2 * q]) + __uint_as_float(b[2 * q]),
                               __uint_as_float(a[2 * q + 1]) + __uint_as_float(b[2 * q + 1]));
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(acc_empty0);
      const long long row = (long long)(u / p.units_n) * 2 * kPM + (long long)rank * kPM + r;
      if (row < p.M) {
        __nv_bfloat16* dst = static_cast<__nv_bfloat16*>(p.rho) + row * p.N;
#pragma unroll
        for (int g = 0; g < kPN / 8; ++g) {
          const int col = (u % p.units_n) * 2 * kPN + c0 + 8 * g;
          if (col + 8 <= p.N)
            *reinterpret_cast<uint4*>(dst + col) =
                make_uint4(packed[4 * g], packed[4 * g + 1], packed[4 * g + 2], packed[4 * g + 3]);
        }
      }
    }
  }
  __syncthreads();
  // no product, load or remote arrival of either CTA is still pending
  tc_fence_before();
  cluster_sync();
  if (warp == 2) {
    tc_fence_after();
    tmem_dealloc_pair(tbase, 512);
  }
}

// fp32: one thread per output, 16 x 16 output tiles through shared memory
// (blockIdx.x over the rows, so M is limited only by the grid's x extent).
__global__ void __launch_bounds__(256)
    plx_probe_simt_kernel(const float* x, const float* w, float* rho, int M, int N, int K) {
  __shared__ float xs[16][17], ws[16][17];
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  const long long m = (long long)blockIdx.x * 16 + ty;
  const long long n = (long long)blockIdx.y * 16 + tx;
  float acc = 0.f;
  for (int k0 = 0; k0 < K; k0 += 16) {
    const long long mx = (long long)blockIdx.x * 16 + ty, nw = (long long)blockIdx.y * 16 + ty;
    xs[ty][tx] = (mx < M && k0 + tx < K) ? x[mx * K + k0 + tx] : 0.f;
    ws[ty][tx] = (nw < N && k0 + tx < K) ? w[nw * K + k0 + tx] : 0.f;
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < 16; ++kk) acc = fmaf(xs[ty][kk], ws[tx][kk], acc);
    __syncthreads();
  }
  if (m < M && n < N) rho[m * N + n] = acc;
}

// 2-D map over a [rows, K] bf16 matrix, box (64, 128), 128-byte swizzle.
cudaError_t encode_2d_sw128(CUtensorMap* map, const void* base, long long rows, int K) {
  EncodeTiledFn enc = tensor_map_encoder();
  if (!enc) return cudaErrorNotSupported;
  cuuint64_t dims[2] = {(cuuint64_t)K, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)K * 2};
  cuuint32_t box[2] = {(cuuint32_t)kPK, (cuuint32_t)kPM};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides,
                   box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

// How many clusters of ks CTAs (smem bytes each) of the kernel (0: the one-SM
// kernel, 1: the SM-pair kernel) the device holds at once, queried once per
// device, kernel and size; 0 if unknown.
int max_active_clusters(int kernel, int ks, int smem) {
  static std::atomic<int> cache[16][2][kPMaxSplit + 1];  // 0: not queried, -1: none
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 16) return 0;
  std::atomic<int>& c = cache[dev][kernel][ks];
  int n = c.load(std::memory_order_relaxed);
  if (n == 0) {
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    cfg.gridDim = dim3((unsigned)ks);
    cfg.blockDim = dim3(kPThreads);
    cfg.dynamicSmemBytes = smem;
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = (unsigned)ks;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    const cudaError_t e = kernel ? cudaOccupancyMaxActiveClusters(&n, plx_probe_gemm_pair_kernel, &cfg)
                                 : cudaOccupancyMaxActiveClusters(&n, plx_probe_gemm_kernel, &cfg);
    if (e != cudaSuccess) {
      (void)cudaGetLastError();
      n = 0;
    }
    n = n > 0 ? n : -1;
    c.store(n, std::memory_order_relaxed);
  }
  return n > 0 ? n : 0;
}

}  // namespace

cudaError_t launch_probe_projection(const void* x, const void* w, void* rho, int M, int N, int K,
                                    bool bf16, int num_sms, unsigned* err, cudaStream_t stream) {
  if (M == 0 || N == 0) return cudaSuccess;
  if (!bf16) {
    dim3 grid((M + 15) / 16, (N + 15) / 16);
    plx_probe_simt_kernel<<<grid, 256, 0, stream>>>(static_cast<const float*>(x),
                                                    static_cast<const float*>(w),
                                                    static_cast<float*>(rho), M, N, K);
    return cudaGetLastError();
  }
  CUtensorMap xm, wm;
  cudaError_t e = encode_2d_sw128(&xm, x, M, K);
  if (e == cudaSuccess) e = encode_2d_sw128(&wm, w, N, K);
  if (e != cudaSuccess) return e;
  ProjParams p;
  p.rho = rho;
  p.M = M;
  p.N = N;
  p.K = K;
  const long long mtiles = (M + kPM - 1) / kPM;
  p.tiles_n = (N + kPN - 1) / kPN;
  p.kblocks = (K + kPK - 1) / kPK;
  const long long tiles = mtiles * p.tiles_n;
  const int smem = 1024 + kPRingBytes + (int)sizeof(ProjBars) + 16;
  p.err = err;
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  cfg.blockDim = dim3(kPThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  // SM pairs when every pair has a 256 x 256 tile to work on
  const long long units2 = ((M + 2 * kPM - 1) / (2 * kPM)) * ((N + 2 * kPN - 1) / (2 * kPN));
  if (units2 >= num_sms / 2 && units2 <= 0x7fffffffll) {
    e = cudaFuncSetAttribute(plx_probe_gemm_pair_kernel,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    const int pairs = max_active_clusters(1, 2, smem);
    if (pairs > 0) {
      p.units = (int)units2;
      p.units_n = (N + 2 * kPN - 1) / (2 * kPN);
      p.pair = 2;
      p.ksplit = 2;
      p.stage_bytes = 2 * kPTileBytes;
      p.stages = kPPairStages;
      const long long clusters = units2 < pairs ? units2 : pairs;
      cfg.gridDim = dim3((unsigned)(2 * clusters));
      attr[0].id = cudaLaunchAttributeClusterDimension;
      attr[0].val.clusterDim.x = 2;
      attr[0].val.clusterDim.y = 1;
      attr[0].val.clusterDim.z = 1;
      cfg.attrs = attr;
      cfg.numAttrs = 1;
      return cudaLaunchKernelEx(&cfg, plx_probe_gemm_pair_kernel, xm, wm, p);
    }
  }
  e = cudaFuncSetAttribute(plx_probe_gemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  p.pair = 1;
  p.ksplit = 1;
  // a pair of tiles moves 1.5 times a single tile's bytes through the ring:
  // pairs when their waves cost no more than the single tiles' waves
  const long long pairs = mtiles * ((p.tiles_n + 1) / 2);
  if (3 * ((pairs + num_sms - 1) / num_sms) <= 2 * ((tiles + num_sms - 1) / num_sms) &&
      pairs < tiles) {
    p.pair = 2;
  } else if (2 * tiles <= num_sms) {
    // the largest cluster whose clusters all run at once (a second wave would
    // cost more than the shorter k range saves)
    for (int ks = kPMaxSplit; ks >= 2; --ks)
      if (tiles * ks <= num_sms && ks <= p.kblocks && tiles <= max_active_clusters(0, ks, smem)) {
        p.ksplit = ks;
        break;
      }
  }
  p.units_n = (p.tiles_n + p.pair - 1) / p.pair;
  const long long units = mtiles * p.units_n;
  if (units > 0x7fffffffll) return cudaErrorInvalidValue;
  p.units = (int)units;
  p.stage_bytes = (1 + p.pair) * kPTileBytes;
  p.stages = kPRingBytes / p.stage_bytes;
  if (p.ksplit > 1) {
    // one cluster per tile (units * ksplit <= num_sms here)
    cfg.gridDim = dim3((unsigned)(units * p.ksplit));
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = (unsigned)p.ksplit;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
  } else {
    cfg.gridDim = dim3((unsigned)(units < num_sms ? units : num_sms));
  }
  e = cudaLaunchKernelEx(&cfg, plx_probe_gemm_kernel, xm, wm, p);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace plx
