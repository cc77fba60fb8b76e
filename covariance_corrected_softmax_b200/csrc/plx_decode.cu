// plx_decode.cu -- Parallax decode kernels: persistent split-K main kernel and
// the log-sum-exp combine kernel.  See plx_decode.cuh for the design.
#include "plx_launch.h"

namespace plx {

// ---------------------------------------------------------------------------
// Element helpers: EPL consecutive elements -> EPL/2 float2.
// ---------------------------------------------------------------------------
template <typename T, int EPL>
struct RowLoad;

template <int EPL>
struct RowLoad<__nv_bfloat16, EPL> {
  static_assert(EPL == 4 || EPL == 8, "bf16 lane slice is 8 or 16 bytes");
  __device__ __forceinline__ static void load(const void* p, float2 (&f)[EPL / 2]) {
    if constexpr (EPL == 8) {
      uint4 w = *reinterpret_cast<const uint4*>(p);
      f[0] = bf16x2_to_float2(w.x);
      f[1] = bf16x2_to_float2(w.y);
      f[2] = bf16x2_to_float2(w.z);
      f[3] = bf16x2_to_float2(w.w);
    } else {
      uint2 w = *reinterpret_cast<const uint2*>(p);
      f[0] = bf16x2_to_float2(w.x);
      f[1] = bf16x2_to_float2(w.y);
    }
  }
};

template <int EPL>
struct RowLoad<float, EPL> {
  static_assert(EPL == 4 || EPL == 8, "fp32 lane slice is 16 or 32 bytes");
  __device__ __forceinline__ static void load(const void* p, float2 (&f)[EPL / 2]) {
    const float4* q = reinterpret_cast<const float4*>(p);
#pragma unroll
    for (int i = 0; i < EPL / 4; ++i) {
      float4 w = q[i];
      f[2 * i] = make_float2(w.x, w.y);
      f[2 * i + 1] = make_float2(w.z, w.w);
    }
  }
};

template <typename T>
__device__ __forceinline__ void store_elem(void* out, size_t idx, float x);
template <>
__device__ __forceinline__ void store_elem<__nv_bfloat16>(void* out, size_t idx, float x) {
  reinterpret_cast<__nv_bfloat16*>(out)[idx] = __float2bfloat16_rn(x);
}
template <>
__device__ __forceinline__ void store_elem<float>(void* out, size_t idx, float x) {
  reinterpret_cast<float*>(out)[idx] = x;
}

__device__ __forceinline__ float2 f2(float a) { return make_float2(a, a); }

// exp2 of (x - m) where x may be -inf; m = -inf only when every x is -inf.
__device__ __forceinline__ float exp2_shift(float x, float m) {
  return (m == -INFINITY) ? 0.f : exp2f(x - m);
}

// Combine weight exp2(m - M) of a partial state with running max m into a
// merged state with max M >= m (0 for an empty state).
__device__ __forceinline__ float merge_weight(float m, float M) {
  return (m == -INFINITY) ? 0.f : exp2f(m - M);
}

// ---------------------------------------------------------------------------
// Block-wide search for this CTA's tile range.  Tiles are ordered batch-major;
// batch b holds ceil(len_b / TK) tiles for each of its Hkv * nhg segments.
// ---------------------------------------------------------------------------
__device__ __forceinline__ long long batch_tiles(const int32_t* seqlens, int b, int S_max,
                                                 int TK, int segs_per_b) {
  int len = clamp_len(seqlens[b], S_max);
  return (long long)((len + TK - 1) / TK) * segs_per_b;
}

struct RangeInfo {
  long long total, t0, t1;
  int b0;              // batch holding tile t0 (valid when t0 < t1)
  long long off0;      // t0 minus the first tile of batch b0
};

__device__ void locate_range(const DecodeParams& p, int TK, RangeInfo* info, long long* scan_ws) {
  const int tid = threadIdx.x, nth = blockDim.x;
  const int lane = tid & 31, warp = tid >> 5, nwarps = nth >> 5;
  const int segs_per_b = p.Hkv * p.nhg;
  const int per = (p.B + nth - 1) / nth;
  const int lo = min(p.B, tid * per), hi = min(p.B, lo + per);
  long long local = 0;
  for (int b = lo; b < hi; ++b) local += batch_tiles(p.seqlens, b, p.S_max, TK, segs_per_b);
  // inclusive warp scan
  long long inc = local;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    long long y = __shfl_up_sync(0xffffffffu, inc, o);
    if (lane >= o) inc += y;
  }
  if (lane == 31) scan_ws[warp] = inc;
  __syncthreads();
  if (tid == 0) {
    long long run = 0;
    for (int w = 0; w < nwarps; ++w) {
      long long x = scan_ws[w];
      scan_ws[w] = run;
      run += x;
    }
    scan_ws[nwarps] = run;
  }
  __syncthreads();
  const long long excl = scan_ws[warp] + inc - local;
  const long long total = scan_ws[nwarps];
  const long long t0 = total * blockIdx.x / p.grid;
  const long long t1 = total * (blockIdx.x + 1) / p.grid;
  if (tid == 0) {
    info->total = total;
    info->t0 = t0;
    info->t1 = t1;
    info->b0 = -1;
    info->off0 = 0;
  }
  __syncthreads();
  if (t0 < t1 && excl <= t0 && t0 < excl + local) {
    long long run = excl;
    for (int b = lo; b < hi; ++b) {
      long long c = batch_tiles(p.seqlens, b, p.S_max, TK, segs_per_b);
      if (t0 < run + c) {
        info->b0 = b;
        info->off0 = t0 - run;
        break;
      }
      run += c;
    }
  }
  __syncthreads();
}

// ---------------------------------------------------------------------------
// Warp-level tensor-core helpers (bf16 consumers).
// ---------------------------------------------------------------------------
// Four 8x8 b16 matrices from shared memory; lanes 8j..8j+7 give the row
// addresses of matrix j; register j of lane L holds row L/4, elements
// 2(L%4), 2(L%4)+1 of matrix j (the .trans form: the transposed matrix).
__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr)
               : "memory");
}
__device__ __forceinline__ void ldsm_x4_trans(uint32_t addr, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr)
               : "memory");
}
// c (16x8 fp32) += a (16x16 bf16, row-major) * b (16x8 bf16, column-major).
__device__ __forceinline__ void mma_bf16_16816(float (&c)[4], const uint32_t (&a)[4],
                                               uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, "
      "{%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// Byte offset of 16-byte chunk c (8 bf16 elements) of row `row` in a tile of
// 64-column boxes with the 128-byte swizzle (chunk index XOR row mod 8).
template <int BOX_BYTES>
__device__ __forceinline__ uint32_t swz_off(int row, int c) {
  return (uint32_t)((c >> 3) * BOX_BYTES + row * 128 + (((c & 7) ^ (row & 7)) << 4));
}

// The result of row (b, h), element c, from its merged softmax sums:
// out = (1 + tbar) o - u with tbar = Z/L, o = O/L, u = U/L, or, in state mode,
// the state (m, l, z, 0, o[D], u[D]) itself.
template <typename T, int D, int MODE>
__device__ __forceinline__ void write_result(const DecodeParams& p, int b, int h, int c, float M,
                                             float L, float Z, float O, float U);

// Kernel instances (see the main kernel).
constexpr int kDecContiguous = 0, kDecPaged = 1, kDecState = 2;
constexpr int kDecStateMode = kDecState;

template <typename T, int D, int MODE>
__device__ __forceinline__ void write_result(const DecodeParams& p, int b, int h, int c, float M,
                                             float L, float Z, float O, float U) {
  constexpr int PHF = part_head_floats<D>();
  if constexpr (MODE == kDecStateMode) {
    float* sr = p.state + ((size_t)b * p.Hq + h) * PHF;
    if (c == 0) {
      sr[0] = M;
      sr[1] = L;
      sr[2] = Z;
      sr[3] = 0.f;
    }
    sr[4 + c] = O;
    sr[4 + D + c] = U;
  } else {
    const float inv = 1.f / L;
    const float val = ((1.f + Z * inv) * O - U) * inv;
    store_elem<T>(p.out, ((size_t)b * p.Hq + h) * D + c, val);
  }
}

// ---------------------------------------------------------------------------
// Segment finalisation.  The NW consumer warps' states of a head group (in
// shared memory: [warp][head] m, l, z, pad, o[D], u[D]) are merged with the
// log-sum-exp rule; then
//  * a segment whose tiles all ran in this CTA writes its output (or, in state
//    mode, the row's softmax state);
//  * a piece of a segment split across CTAs goes to one of this CTA's two
//    workspace slots (slot 0: the CTA's first segment, slot 1: its last); a
//    piece that does not end the segment is published with a header
//    (segment, launch tag) written after the data;
//  * the piece that ends a split segment (necessarily the CTA's first
//    segment) is merged with the earlier pieces once the CTA has finished all
//    its tiles (merge_tail below): every CTA holds about the same work, so the
//    CTAs holding those pieces finish at about the same time.
// Called by all consumer threads between two consumer-wide barriers; false if
// the consumer barrier (cbar) gave up.
// ---------------------------------------------------------------------------
template <typename T, int D, int HPW, int MODE, int NW>
__device__ __forceinline__ bool finalize_segment(const DecodeParams& p, const TileMeta& mt, int h0,
                                                 float* part, const float* merge, int tid,
                                                 uint64_t* cbar, uint32_t& cphase,
                                                 volatile int* abort_flag) {
  constexpr int PHF = part_head_floats<D>();
  static_assert(HPW * D <= NW * 32, "one element per consumer thread");
  const bool starts = (mt.flags & 4) != 0, ends = (mt.flags & 8) != 0;
  const int g = tid / D, c = tid % D;  // one (head, column) per thread
  if (tid < HPW * D) {
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < NW; ++w) M = fmaxf(M, merge[(w * HPW + g) * PHF]);
    float L = 0.f, Z = 0.f, O = 0.f, U = 0.f;
#pragma unroll
    for (int w = 0; w < NW; ++w) {
      const float* src = merge + (w * HPW + g) * PHF;
      const float wt = merge_weight(src[0], M);
      L += wt * src[1];
      Z += wt * src[2];
      O += wt * src[4 + c];
      U += wt * src[4 + D + c];
    }
    if (starts && ends) {
      write_result<T, D, MODE>(p, mt.b, h0 + g, c, M, L, Z, O, U);
    } else {
      float* ph = part + kPartHeader + g * PHF;
      if (c == 0) {
        ph[0] = M;
        ph[1] = L;
        ph[2] = Z;
      }
      ph[4 + c] = O;
      ph[4 + D + c] = U;
    }
  }
  if (!ends) {
    // publish: the data above, then the header
    __threadfence();
    if (!warps_sync(cbar, cphase, abort_flag, p.err)) return false;
    if (tid == 0) {
      volatile int* hdr = reinterpret_cast<volatile int*>(part);
      hdr[1] = starts ? 1 : 0;
      hdr[2] = 0;
      hdr[3] = launch_tag();
      __threadfence();
      hdr[0] = mt.seg;
    }
  }
  return true;
}

// The split segment whose last piece this CTA holds (in its slot 0): merge the
// pieces of the CTAs from the one where the segment began, in CTA order, this
// CTA's last, and write the output or state.  The earlier pieces are found by
// their headers, one consumer thread per CTA waiting (bounded) for its piece:
// all CTAs of the grid are resident, one per SM, and a piece never waits for a
// later one.  Called by all consumer threads after the tiles; `slots` is
// shared scratch of at least gridDim.x ints.
template <typename T, int D, int HPW, int MODE, int NW>
__device__ __forceinline__ void merge_tail(const DecodeParams& p, int b, int seg, int h0,
                                           long long seg_t0, long long total, int tid,
                                           volatile int* abort_flag, int* slots, uint64_t* cbar,
                                           uint32_t& cphase) {
  constexpr int PF = part_floats<D>(HPW);
  constexpr int PHF = part_head_floats<D>();
  const float* base = p.ws + kWsHeaderFloats;
  const int tag = launch_tag();
  long long cf = seg_t0 * p.grid / total;
  while (cf > 0 && total * cf / p.grid > seg_t0) --cf;
  while (cf + 1 < p.grid && total * (cf + 1) / p.grid <= seg_t0) ++cf;
  const int npieces = (int)blockIdx.x - (int)cf;  // earlier CTAs
  for (int k = tid; k < npieces; k += NW * 32) {
    const int cta = (int)cf + k;
    int sl = -2;  // a CTA whose tile range is empty holds no piece
    if (total * cta / p.grid != total * (cta + 1) / p.grid) {
      // the piece is in slot 1 of the CTA where the segment began when that CTA
      // finished an earlier segment first, otherwise in slot 0
      sl = -1;
      const uint64_t t0 = globaltimer_ns();
      uint64_t limit = 0;
      for (uint32_t spins = 0; sl < 0; ++spins) {
        for (int s = 0; s < 2 && sl < 0; ++s) {
          const volatile int* hdr =
              reinterpret_cast<const volatile int*>(base + (size_t)(2 * cta + s) * PF);
          if (hdr[0] == seg && hdr[3] == tag) sl = s;
        }
        if (sl < 0 && (spins & 63u) == 63u) {
          if (*abort_flag) break;
          if (limit == 0) limit = wait_limit_ns(p.err);
          if (globaltimer_ns() - t0 > limit || spins >= kWaitMaxPolls) {
            record_error(p.err, kDevTimeoutMbarrier);
            *abort_flag = 1;
            break;
          }
        }
      }
      __threadfence();  // the piece's data, published before its header, is read below
    }
    slots[k] = sl;
  }
  if (!warps_sync(cbar, cphase, abort_flag, p.err)) return;
  if (tid >= HPW * D) return;
  const int g = tid / D, c = tid % D;
  float M = -INFINITY, L = 0.f, Z = 0.f, O = 0.f, U = 0.f;
  auto absorb = [&](float m, float l, float z, float o, float u) {
    const float Mn = fmaxf(M, m);
    const float wa = merge_weight(M, Mn), wb = merge_weight(m, Mn);
    L = L * wa + l * wb;
    Z = Z * wa + z * wb;
    O = O * wa + o * wb;
    U = U * wa + u * wb;
    M = Mn;
  };
  bool failed = false;
  // pieces in CTA order, four loads in flight at a time
  for (int k0 = 0; k0 <= npieces; k0 += 4) {
    float v[4][5];
    bool use[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int k = k0 + q;
      use[q] = false;
      if (k > npieces) continue;
      const int sl = k < npieces ? slots[k] : 0;  // k == npieces: this CTA's own piece
      if (sl == -1) failed = true;
      if (sl < 0) continue;
      const float* ph = base + (size_t)(2 * ((int)cf + k) + sl) * PF + kPartHeader + g * PHF;
      v[q][0] = __ldcg(ph);
      v[q][1] = __ldcg(ph + 1);
      v[q][2] = __ldcg(ph + 2);
      v[q][3] = __ldcg(ph + 4 + c);
      v[q][4] = __ldcg(ph + 4 + D + c);
      use[q] = true;
    }
#pragma unroll
    for (int q = 0; q < 4; ++q)
      if (use[q]) absorb(v[q][0], v[q][1], v[q][2], v[q][3], v[q][4]);
  }
  if (!failed) write_result<T, D, MODE>(p, b, h0 + g, c, M, L, Z, O, U);
}

// ---------------------------------------------------------------------------
// Main decode kernel.
// ---------------------------------------------------------------------------
// MODE: kDecContiguous, kDecPaged (block-table loads), kDecState (contiguous
// loads, softmax states written instead of the output).  Each is a separate
// instance, so the common one carries no code of the others.

// kmap, vmap: TK-row boxes over the contiguous cache (unused when paged).
// kmap_c, vmap_c: 16-row boxes over the contiguous cache (a segment's last,
// partial tile) or over the page pools (paged).
template <typename T, int D, int HPW, int MODE>
__global__ void __launch_bounds__(DecodeTile<T, D>::THREADS, 1)
    plx_decode_splitk_kernel(const __grid_constant__ CUtensorMap kmap,
                             const __grid_constant__ CUtensorMap vmap,
                             const __grid_constant__ CUtensorMap kmap_c,
                             const __grid_constant__ CUtensorMap vmap_c, const DecodeParams p) {
  using Cfg = DecodeTile<T, D>;
  constexpr int NW = Cfg::NW, TK = Cfg::TK, KPH = Cfg::KPH, EPL = Cfg::EPL,
                STAGES = Cfg::STAGES, CB = Cfg::CB;
  constexpr int H2 = EPL / 2;
  constexpr int PF = part_floats<D>(HPW);
  constexpr int PHF = part_head_floats<D>();
  constexpr int CH = kDecChunkRows;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint8_t* ring = smem;
  TileMeta* metas = reinterpret_cast<TileMeta*>(ring + STAGES * Cfg::STAGE_BYTES);
  uint64_t* full = reinterpret_cast<uint64_t*>(metas + STAGES);
  uint64_t* empty = full + STAGES;
  RangeInfo* info = reinterpret_cast<RangeInfo*>(empty + STAGES);
  long long* scan_ws = reinterpret_cast<long long*>(info + 1);   // 16 entries
  volatile int* abort_flag = reinterpret_cast<volatile int*>(scan_ws + 16);
  uint64_t* cbar = reinterpret_cast<uint64_t*>(scan_ws + 18);  // the consumer warps' barrier
  float* merge = reinterpret_cast<float*>(scan_ws + 20);
  float* red_smem = reinterpret_cast<float*>(
      (reinterpret_cast<uintptr_t>(merge + NW * HPW * PHF) + 15) & ~uintptr_t(15));
  float* bc_smem = red_smem + 2 * NW * kDecRedRegion;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  // Launched as a programmatic dependent of the previous kernel on the stream:
  // this CTA may be resident before that kernel has finished (its launch and
  // set-up overlap the other's tail), but it touches no global memory until
  // that kernel has completed and its writes are visible.  The next kernel may
  // likewise be scheduled as soon as SMs free up.
  grid_dep_wait();
  grid_dep_launch_dependents();

  if (tid == 0) {
    *abort_flag = 0;
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], NW);
    }
    mbar_init(cbar, NW);
    fence_mbarrier_init();
  }
  locate_range(p, TK, info, scan_ws);  // contains __syncthreads

  // Batches with an empty context produce zeros (out = 0 for an empty key set),
  // or the empty state (m = -inf, everything else 0).
  for (int b = blockIdx.x; b < p.B; b += p.grid) {
    if (clamp_len(p.seqlens[b], p.S_max) == 0) {
      if constexpr (MODE == kDecState) {
        for (int e = tid; e < p.Hq * PHF; e += blockDim.x)
          p.state[(size_t)b * p.Hq * PHF + e] = (e % PHF == 0) ? -INFINITY : 0.f;
      } else {
        for (int e = tid; e < p.Hq * D; e += blockDim.x)
          store_elem<T>(p.out, (size_t)b * p.Hq * D + e, 0.f);
      }
    }
  }

  const long long t0 = info->t0, t1 = info->t1;
  const int segs_per_b = p.Hkv * p.nhg;

  if (warp == NW) {
    // ------------------------------------------------------------ producer
    // The tile walk (batch-major over (batch, kv-head, head-group) segments,
    // tiles of TK keys, from this CTA's first tile t0) runs in every lane.
    if (t0 < t1) {
      int b = info->b0;
      int len = clamp_len(p.seqlens[b], p.S_max);
      int nt = (len + TK - 1) / TK;
      int seg_local = (int)(info->off0 / nt);
      int kt = (int)(info->off0 % nt);
      bool starts_here = (kt == 0);
      if (lane == 0) {
        tma_prefetch_desc(&kmap_c);
        tma_prefetch_desc(&vmap_c);
        if constexpr (MODE != kDecPaged) {
          tma_prefetch_desc(&kmap);
          tma_prefetch_desc(&vmap);
        }
      }
      for (long long t = t0, i = 0; t < t1; ++t, ++i) {
        const int stage = (int)(i % STAGES);
        if (i >= STAGES) {
          int okw = 1;
          if (lane == 0)
            okw = mbar_wait(&empty[stage], (uint32_t)(((i / STAGES) - 1) & 1), abort_flag, p.err);
          if (!__shfl_sync(0xffffffffu, okw, 0)) break;
        }
        TileMeta m;
        m.b = b;
        m.hkv = seg_local / p.nhg;
        m.hg = seg_local % p.nhg;
        m.kt = kt;
        m.nvalid = min(TK, len - kt * TK);
        m.seg = b * segs_per_b + seg_local;
        m.flags = ((t == t0 || kt == 0) ? 1 : 0) | ((t == t1 - 1 || kt == nt - 1) ? 2 : 0) |
                  (starts_here ? 4 : 0) | ((kt == nt - 1) ? 8 : 0);
        m.pad = 0;
        uint8_t* dst = ring + stage * Cfg::STAGE_BYTES;
        // Paged caches always, and (bf16) a partial last tile, come in 16-row
        // chunks: lane c loads chunk c; chunks past the length are not loaded
        // (the consumers mask their rows).
        const bool chunked = MODE == kDecPaged || (Cfg::MMA && m.nvalid < TK);
        if (!chunked) {
          if (lane == 0) {
            metas[stage] = m;
            mbar_arrive_expect_tx(&full[stage], Cfg::STAGE_BYTES);
#pragma unroll
            for (int cb = 0; cb < CB; ++cb) {
              tma_load_4d(dst + cb * Cfg::BOX_BYTES, &kmap, &full[stage], cb * 64, m.hkv,
                          kt * TK, b);
              tma_load_4d(dst + Cfg::TILE_BYTES + cb * Cfg::BOX_BYTES, &vmap, &full[stage],
                          cb * 64, m.hkv, kt * TK, b);
            }
          }
        } else {
          const int nch = (m.nvalid + CH - 1) / CH;
          const int c = lane;
          int row = -CH, bc = b;
          if (c < nch) {
            const int pos = kt * TK + CH * c;
            if constexpr (MODE == kDecPaged) {
              // a page index outside the pool is reported and read as zeros
              // (out-of-range TMA rows)
              const int page = p.block_table[(size_t)b * p.max_pages + pos / p.page_size];
              bc = 0;
              if (page >= 0 && page < p.num_pages)
                row = page * p.page_size + pos % p.page_size;
              else
                record_error(p.err, kDevBadArgument);
            } else {
              row = pos;
            }
          }
          if (lane == 0) {
            metas[stage] = m;
            mbar_arrive_expect_tx(&full[stage], (uint32_t)(2 * nch * CH * Cfg::ROW_BYTES));
          }
          __syncwarp();
          if (c < nch) {
#pragma unroll
            for (int cb = 0; cb < CB; ++cb) {
              const int off = cb * Cfg::BOX_BYTES + c * CH * Cfg::BOX_ROW;
              tma_load_4d(dst + off, &kmap_c, &full[stage], cb * 64, m.hkv, row, bc);
              tma_load_4d(dst + Cfg::TILE_BYTES + off, &vmap_c, &full[stage], cb * 64, m.hkv,
                          row, bc);
            }
          }
        }
        // advance the walk
        if (++kt == nt) {
          kt = 0;
          starts_here = true;
          if (++seg_local == segs_per_b) {
            seg_local = 0;
            do {
              ++b;
            } while (b < p.B && clamp_len(p.seqlens[b], p.S_max) == 0);
            if (b < p.B) {
              len = clamp_len(p.seqlens[b], p.S_max);
              nt = (len + TK - 1) / TK;
            }
          }
        }
      }
    }
  } else if constexpr (Cfg::MMA) {
    // ------------------------------------------------------------ consumers (bf16)
    // Warp w owns keys [16w, 16w + 16) of every tile.  Lane L = 4g + tq:
    //  score chain: A rows g = q of head hh, g + 8 = rho of head hh; C holds,
    //    for keys 8nb + 2tq + {0, 1} (nb = 0, 1), q.k in c0, c1 and rho.k in
    //    c2, c3;
    //  weights: B row (kind) g of the value product: p (kinds with bit 1
    //    clear) or p t (bit 1 set) of head hh, its bf16 high part (g < 4) or
    //    the bf16 rounding of the remainder (g >= 4); for keys 2tq + {0, 1}
    //    (b0) and 8 + 2tq + {0, 1} (b1): the very keys of the score fragment;
    //  value accumulators acc[mb]: head dims 16mb + g (c0, c1) and + 8 (c2, c3)
    //    of kinds 2tq (head 0) and 2tq + 1 (head 1): tq = 0 the high parts of
    //    o, 1 of u, 2 the low parts of o, 3 of u.
    constexpr int KS = D / 16;
    const int g = lane >> 2, tq = lane & 3;
    const int hh = HPW == 2 ? (g & 1) : 0;
    const bool w_pt = ((g >> 1) & 1) != 0;
    const bool w_lo = g >= 4;
    const bool w_live = HPW == 2 || (g & 1) == 0;  // one head: odd kinds unused
    const int lj = lane >> 3, lr = lane & 7;       // ldmatrix: matrix, row
    const int kw0 = warp * 16;                     // this warp's first key of a tile
    const uint32_t ring_s = smem_u32(ring);
    uint32_t qa[KS][4];
    float acc[KS][4];
    float m_run = -INFINITY, lsum = 0.f, zsum = 0.f;
    int ordinal = 0;        // segments finalised so far by this CTA
    long long seg_t0 = 0;   // first tile (global order) of the current segment
    int tail_seg = -1, tail_b = 0, tail_h0 = 0;  // the split segment ending here
    long long tail_t0 = 0;
    bool done = true;
    uint32_t cphase = 0;  // completed uses of the consumer barrier
#pragma unroll
    for (int ks = 0; ks < KS; ++ks)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        qa[ks][e] = 0u;
        acc[ks][e] = 0.f;
      }

    for (long long t = t0, i = 0; t < t1; ++t, ++i) {
      const int stage = (int)(i % STAGES);
      if (!mbar_wait(&full[stage], (uint32_t)((i / STAGES) & 1), abort_flag, p.err)) {
        done = false;
        break;
      }
      const TileMeta mt = metas[stage];
      const int h0 = mt.hkv * p.G + mt.hg * HPW;  // first query head of the group

      if (mt.flags & 1) {  // first tile of a segment in this CTA: load q, rho; reset
        seg_t0 = t - mt.kt;  // the segment's first tile in the global order
        const size_t row = ((size_t)mt.b * p.Hq + h0 + hh) * (D / 2);
        const uint32_t* q32 = reinterpret_cast<const uint32_t*>(p.q) + row;
        const uint32_t* r32 = reinterpret_cast<const uint32_t*>(p.rho) + row;
#pragma unroll
        for (int ks = 0; ks < KS; ++ks) {
          qa[ks][0] = q32[8 * ks + tq];
          qa[ks][1] = r32[8 * ks + tq];
          qa[ks][2] = q32[8 * ks + 4 + tq];
          qa[ks][3] = r32[8 * ks + 4 + tq];
#pragma unroll
          for (int e = 0; e < 4; ++e) acc[ks][e] = 0.f;
        }
        m_run = -INFINITY;
        lsum = zsum = 0.f;
      }

      const int nv = mt.nvalid - kw0;  // valid keys of this warp in the tile
      if (nv > 0) {
        const uint32_t kbase = ring_s + stage * Cfg::STAGE_BYTES;
        const uint32_t vbase = kbase + Cfg::TILE_BYTES;
        // scores: cs[nb] = [q; rho] x K^T for keys kw0 + 8nb .. + 7
        float cs[2][4];
#pragma unroll
        for (int nb = 0; nb < 2; ++nb) {
          cs[nb][0] = cs[nb][1] = cs[nb][2] = cs[nb][3] = 0.f;
          const int key = kw0 + 8 * nb + lr;
#pragma unroll
          for (int kp = 0; kp < KS / 2; ++kp) {
            uint32_t bk[4];
            ldsm_x4(kbase + swz_off<Cfg::BOX_BYTES>(key, 4 * kp + lj), bk);
            mma_bf16_16816(cs[nb], qa[2 * kp], bk[0], bk[1]);
            mma_bf16_16816(cs[nb], qa[2 * kp + 1], bk[2], bk[3]);
          }
        }
        // this lane's keys: 2tq, 2tq + 1, 8 + 2tq, 9 + 2tq (of the warp's 16)
        float sv[4] = {cs[0][0] * p.qscale, cs[0][1] * p.qscale, cs[1][0] * p.qscale,
                       cs[1][1] * p.qscale};
        float tv[4] = {cs[0][2], cs[0][3], cs[1][2], cs[1][3]};
        const bool tail = nv < 16;
        if (tail) {
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            if (8 * (kk >> 1) + 2 * tq + (kk & 1) >= nv) {
              sv[kk] = -INFINITY;
              tv[kk] = 0.f;  // rows past the length may hold anything
            }
        }
        float mx = fmaxf(fmaxf(sv[0], sv[1]), fmaxf(sv[2], sv[3]));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
        // lazy running max of head hh: moves only when the tile's max exceeds
        // it by more than 2^8, so every weight stays <= 2^8
        float alpha = 1.f;
        if (mx > m_run + 8.f) {
          alpha = (m_run == -INFINITY) ? 0.f : fast_exp2(m_run - mx);
          m_run = mx;
        }
        const float alpha_x = __shfl_xor_sync(0xffffffffu, alpha, 4);  // the other head's
        const float a0 = (HPW == 1 || hh == 0) ? alpha : alpha_x;
        const float a1 = (HPW == 2 && hh == 1) ? alpha : alpha_x;
        if (a0 != 1.f || a1 != 1.f) {
#pragma unroll
          for (int mb = 0; mb < KS; ++mb) {
            acc[mb][0] *= a0;
            acc[mb][1] *= a1;
            acc[mb][2] *= a0;
            acc[mb][3] *= a1;
          }
        }
        lsum *= alpha;
        zsum *= alpha;
        float w[4];
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          const float pp = fast_exp2(sv[kk] - m_run);  // 0 for a masked key
          const float pt = pp * tv[kk];
          lsum += pp;
          zsum += pt;
          w[kk] = w_pt ? pt : pp;
        }
        uint32_t bw[2];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const uint32_t hi = float2_to_bf16x2(w[2 * h], w[2 * h + 1]);
          if (w_lo) {
            const float2 hf = bf16x2_to_float2(hi);
            bw[h] = float2_to_bf16x2(w[2 * h] - hf.x, w[2 * h + 1] - hf.y);
          } else {
            bw[h] = hi;
          }
          if (!w_live) bw[h] = 0u;
        }
        // value products: acc[mb] += V^T[16mb.., keys] x W^T
        uint32_t mk01 = 0xffffffffu, mk23 = 0xffffffffu;
        if (tail) {
          mk01 = (2 * tq < nv ? 0x0000ffffu : 0u) | (2 * tq + 1 < nv ? 0xffff0000u : 0u);
          mk23 = (2 * tq + 8 < nv ? 0x0000ffffu : 0u) | (2 * tq + 9 < nv ? 0xffff0000u : 0u);
        }
        const int vkey = kw0 + 8 * (lj >> 1) + lr;
#pragma unroll
        for (int mb = 0; mb < KS; ++mb) {
          uint32_t av[4];
          ldsm_x4_trans(vbase + swz_off<Cfg::BOX_BYTES>(vkey, 2 * mb + (lj & 1)), av);
          av[0] &= mk01;
          av[1] &= mk01;
          av[2] &= mk23;
          av[3] &= mk23;
          mma_bf16_16816(acc[mb], av, bw[0], bw[1]);
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[stage]);

      if (mt.flags & 2) {
        // ---- this warp's state of the segment, to shared memory
        float ls = lsum, zs = zsum;
        ls += __shfl_xor_sync(0xffffffffu, ls, 1);
        ls += __shfl_xor_sync(0xffffffffu, ls, 2);
        zs += __shfl_xor_sync(0xffffffffu, zs, 1);
        zs += __shfl_xor_sync(0xffffffffu, zs, 2);
        float* dstw = merge + warp * HPW * PHF;
#pragma unroll
        for (int mb = 0; mb < KS; ++mb) {
          float o[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) o[e] = acc[mb][e] + __shfl_xor_sync(0xffffffffu, acc[mb][e], 2);
          if (tq < 2) {  // tq 0: o (high + low parts), tq 1: u
            const int off = 4 + tq * D + 16 * mb + g;
            dstw[off] = o[0];
            dstw[off + 8] = o[2];
            if (HPW == 2) {
              dstw[PHF + off] = o[1];
              dstw[PHF + off + 8] = o[3];
            }
          }
        }
        if (tq == 0 && g < HPW) {
          dstw[g * PHF + 0] = m_run;
          dstw[g * PHF + 1] = ls;
          dstw[g * PHF + 2] = zs;
        }
      }
      if (mt.flags & 2) {
        // slot 0 holds the CTA's first segment, which may have begun in an
        // earlier CTA; slot 1 its last, which may end in a later one
        float* part = p.ws + kWsHeaderFloats + (size_t)(2 * blockIdx.x + (ordinal == 0 ? 0 : 1)) * PF;
        if (!warps_sync(cbar, cphase, abort_flag, p.err) ||
            !finalize_segment<T, D, HPW, MODE, NW>(p, mt, h0, part, merge, tid, cbar, cphase,
                                                   abort_flag) ||
            !warps_sync(cbar, cphase, abort_flag, p.err)) {
          done = false;
          break;
        }
        if ((mt.flags & 8) && !(mt.flags & 4)) {  // this CTA holds a split segment's end
          tail_seg = mt.seg;
          tail_b = mt.b;
          tail_h0 = h0;
          tail_t0 = seg_t0;
        }
        ++ordinal;
      }
    }
    if (done && tail_seg >= 0)
      merge_tail<T, D, HPW, MODE, NW>(p, tail_b, tail_seg, tail_h0, tail_t0, info->total, tid,
                                      abort_flag, reinterpret_cast<int*>(merge), cbar, cphase);
  } else {
    // ------------------------------------------------------------ consumers (fp32)
    const int hw = lane >> 4, sub = lane & 15;
    const int rowbase = (warp * 2 + hw) * KPH;
    // Per key, the half-warp forms 2 HPW partial dot products per lane (s for
    // each head, then t for each head).  They are reduced by a transpose through
    // shared memory: lane v ends up holding the full sum of value v, i.e. of
    // kind v % NT for key v / NT of this half-warp's KPH keys.
    constexpr int NT = 2 * HPW;
    constexpr int NV = KPH * NT;
    static_assert(NV <= 16 && (NV & (NV - 1)) == 0, "one reduced value per lane");
    const int kv = sub / NT, kind = sub % NT;
    const bool is_s = kind < HPW;              // a score lane (else a probe-score lane)
    const int hsrc = lane - (is_s ? 0 : HPW);  // the score lane of the same key and head
    const int hbase = lane & 16;               // first lane of this half-warp
    float* red = red_smem + (warp * 2 + hw) * kDecRedRegion;
    float* bc = bc_smem + (warp * 2 + hw) * 16;
    float2 qf[HPW][H2], rf[HPW][H2], oa[HPW][H2], ua[HPW][H2];
    // running max of this lane's head, and l (score lanes) or z (probe lanes)
    float m_run = -INFINITY, lz = 0.f;
    int ordinal = 0;        // segments finalised so far by this CTA
    long long seg_t0 = 0;   // first tile (global order) of the current segment
    int tail_seg = -1, tail_b = 0, tail_h0 = 0;  // the split segment ending here
    long long tail_t0 = 0;
    bool done = true;
    uint32_t cphase = 0;  // completed uses of the consumer barrier
#pragma unroll
    for (int g = 0; g < HPW; ++g) {
#pragma unroll
      for (int e = 0; e < H2; ++e) {
        qf[g][e] = rf[g][e] = oa[g][e] = ua[g][e] = make_float2(0.f, 0.f);
      }
    }

    for (long long t = t0, i = 0; t < t1; ++t, ++i) {
      const int stage = (int)(i % STAGES);
      if (!mbar_wait(&full[stage], (uint32_t)((i / STAGES) & 1), abort_flag, p.err)) {
        done = false;
        break;
      }
      const TileMeta mt = metas[stage];
      const int h0 = mt.hkv * p.G + mt.hg * HPW;  // first query head of the group

      if (mt.flags & 1) {  // first tile of a segment in this CTA: load q, rho; reset
        seg_t0 = t - mt.kt;  // the segment's first tile in the global order
#pragma unroll
        for (int g = 0; g < HPW; ++g) {
          const size_t base = ((size_t)mt.b * p.Hq + h0 + g) * D + sub * EPL;
          RowLoad<T, EPL>::load(reinterpret_cast<const T*>(p.q) + base, qf[g]);
          RowLoad<T, EPL>::load(reinterpret_cast<const T*>(p.rho) + base, rf[g]);
#pragma unroll
          for (int e = 0; e < H2; ++e) {
            qf[g][e].x *= p.qscale;
            qf[g][e].y *= p.qscale;
            oa[g][e] = ua[g][e] = make_float2(0.f, 0.f);
          }
        }
        m_run = -INFINITY;
        lz = 0.f;
      }

      const uint8_t* kt_base = ring + stage * Cfg::STAGE_BYTES +
                               (size_t)rowbase * Cfg::ROW_BYTES + sub * EPL * sizeof(T);
      const uint8_t* vt_base = kt_base + Cfg::TILE_BYTES;

      // Phase A: partial dot products s = (scale log2e) q.k and t = rho.k
      float vals[NV];
#pragma unroll
      for (int kk = 0; kk < KPH; ++kk) {
        float2 kf[H2];
        RowLoad<T, EPL>::load(kt_base + kk * Cfg::ROW_BYTES, kf);
#pragma unroll
        for (int g = 0; g < HPW; ++g) {
          float2 as = make_float2(0.f, 0.f), at = make_float2(0.f, 0.f);
#pragma unroll
          for (int e = 0; e < H2; ++e) {
            as = __ffma2_rn(qf[g][e], kf[e], as);
            at = __ffma2_rn(rf[g][e], kf[e], at);
          }
          vals[kk * NT + g] = as.x + as.y;
          vals[kk * NT + HPW + g] = at.x + at.y;
        }
      }
      // Phase B: transpose-reduce over the 16 lanes of the half-warp
#pragma unroll
      for (int q4 = 0; q4 < NV; q4 += 4)
        *reinterpret_cast<float4*>(red + sub * kDecRedRow + q4) =
            make_float4(vals[q4], vals[q4 + 1], vals[q4 + 2], vals[q4 + 3]);
      __syncwarp();
      float acc = 0.f;
      if (sub < NV) {
        float a0 = 0.f, a1 = 0.f;
#pragma unroll
        for (int row = 0; row < 16; row += 2) {
          a0 += red[row * kDecRedRow + sub];
          a1 += red[(row + 1) * kDecRedRow + sub];
        }
        acc = a0 + a1;
      }
      // Phase C: online softmax on the distributed values
      const bool valid_k = (sub < NV) && (rowbase + kv) < mt.nvalid;
      float val = acc;
      if (is_s && !valid_k) val = -INFINITY;
      float mx = val;
#pragma unroll
      for (int o = NT; o < NV; o <<= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
      const float smax = __shfl_sync(0xffffffffu, mx, hsrc);   // tile max of this head
      float alpha = 1.f;
      if (smax > m_run) {
        alpha = merge_weight(m_run, smax);
        lz *= alpha;
        m_run = smax;
      }
      const float pv = is_s ? exp2_shift(val, m_run) : 0.f;
      const float ps = __shfl_sync(0xffffffffu, pv, hsrc);
      const float w = is_s ? pv : (valid_k ? ps * val : 0.f);  // p, or p t
      float sw = w;
#pragma unroll
      for (int o = NT; o < NV; o <<= 1) sw += __shfl_xor_sync(0xffffffffu, sw, o);
      lz += sw;
      float al[HPW];
#pragma unroll
      for (int g = 0; g < HPW; ++g) al[g] = __shfl_sync(0xffffffffu, alpha, hbase + g);
      if (sub < NV) bc[sub] = w;
      __syncwarp();
      float pw[KPH][HPW], ptw[KPH][HPW];
#pragma unroll
      for (int kk = 0; kk < KPH; ++kk) {
        if constexpr (NT == 4) {
          const float4 w4 = *reinterpret_cast<const float4*>(bc + kk * NT);
          pw[kk][0] = w4.x;
          pw[kk][1] = w4.y;
          ptw[kk][0] = w4.z;
          ptw[kk][1] = w4.w;
        } else {
          const float2 w2 = *reinterpret_cast<const float2*>(bc + kk * NT);
          pw[kk][0] = w2.x;
          ptw[kk][0] = w2.y;
        }
      }
#pragma unroll
      for (int g = 0; g < HPW; ++g) {
        if (al[g] != 1.f) {
#pragma unroll
          for (int e = 0; e < H2; ++e) {
            oa[g][e] = __fmul2_rn(oa[g][e], f2(al[g]));
            ua[g][e] = __fmul2_rn(ua[g][e], f2(al[g]));
          }
        }
      }
      // Phase D: accumulate o += p v and u += (p t) v
      const bool tail = mt.nvalid < TK;
#pragma unroll
      for (int kk = 0; kk < KPH; ++kk) {
        float2 vf[H2];
        RowLoad<T, EPL>::load(vt_base + kk * Cfg::ROW_BYTES, vf);
        if (tail && rowbase + kk >= mt.nvalid) {  // rows past the length may hold anything
#pragma unroll
          for (int e = 0; e < H2; ++e) vf[e] = make_float2(0.f, 0.f);
        }
#pragma unroll
        for (int g = 0; g < HPW; ++g) {
#pragma unroll
          for (int e = 0; e < H2; ++e) {
            oa[g][e] = __ffma2_rn(f2(pw[kk][g]), vf[e], oa[g][e]);
            ua[g][e] = __ffma2_rn(f2(ptw[kk][g]), vf[e], ua[g][e]);
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[stage]);

      if (mt.flags & 2) {
        // ---- merge the two half-warp states, to shared memory
        float m[HPW], l[HPW], z[HPW];
#pragma unroll
        for (int g = 0; g < HPW; ++g) {
          m[g] = __shfl_sync(0xffffffffu, m_run, hbase + g);
          l[g] = __shfl_sync(0xffffffffu, lz, hbase + g);
          z[g] = __shfl_sync(0xffffffffu, lz, hbase + HPW + g);
        }
#pragma unroll
        for (int g = 0; g < HPW; ++g) {
          const float mo = __shfl_xor_sync(0xffffffffu, m[g], 16);
          const float M = fmaxf(m[g], mo);
          const float w = merge_weight(m[g], M);
          float lw = l[g] * w, zw = z[g] * w;
          lw += __shfl_xor_sync(0xffffffffu, lw, 16);
          zw += __shfl_xor_sync(0xffffffffu, zw, 16);
          m[g] = M;
          l[g] = lw;
          z[g] = zw;
#pragma unroll
          for (int e = 0; e < H2; ++e) {
            float2 ow = __fmul2_rn(oa[g][e], f2(w)), uw = __fmul2_rn(ua[g][e], f2(w));
            ow.x += __shfl_xor_sync(0xffffffffu, ow.x, 16);
            ow.y += __shfl_xor_sync(0xffffffffu, ow.y, 16);
            uw.x += __shfl_xor_sync(0xffffffffu, uw.x, 16);
            uw.y += __shfl_xor_sync(0xffffffffu, uw.y, 16);
            oa[g][e] = ow;
            ua[g][e] = uw;
          }
          if (hw == 0) {
            float* dst = merge + (warp * HPW + g) * PHF;
            if (sub == 0) {
              dst[0] = M;
              dst[1] = lw;
              dst[2] = zw;
            }
#pragma unroll
            for (int e = 0; e < H2; ++e) {
              dst[4 + sub * EPL + 2 * e] = oa[g][e].x;
              dst[4 + sub * EPL + 2 * e + 1] = oa[g][e].y;
              dst[4 + D + sub * EPL + 2 * e] = ua[g][e].x;
              dst[4 + D + sub * EPL + 2 * e + 1] = ua[g][e].y;
            }
          }
        }
        float* part = p.ws + kWsHeaderFloats + (size_t)(2 * blockIdx.x + (ordinal == 0 ? 0 : 1)) * PF;
        if (!warps_sync(cbar, cphase, abort_flag, p.err) ||
            !finalize_segment<T, D, HPW, MODE, NW>(p, mt, h0, part, merge, tid, cbar, cphase,
                                                   abort_flag) ||
            !warps_sync(cbar, cphase, abort_flag, p.err)) {
          done = false;
          break;
        }
        if ((mt.flags & 8) && !(mt.flags & 4)) {  // this CTA holds a split segment's end
          tail_seg = mt.seg;
          tail_b = mt.b;
          tail_h0 = h0;
          tail_t0 = seg_t0;
        }
        ++ordinal;
      }
    }
    if (done && tail_seg >= 0)
      merge_tail<T, D, HPW, MODE, NW>(p, tail_b, tail_seg, tail_h0, tail_t0, info->total, tid,
                                      abort_flag, reinterpret_cast<int*>(merge), cbar, cphase);
  }
}

// ---------------------------------------------------------------------------
// Merge of R softmax states per (b, h) row (R slices of one key set, e.g. the
// context split over ranks) with the log-sum-exp rule, then
// out = ((1 + z/l) o - u) / l (0 for an empty key set).  One block per row,
// one thread per element.
// ---------------------------------------------------------------------------
template <typename T, int D>
__global__ void __launch_bounds__(D)
    plx_merge_states_kernel(const float* states, int R, long long rows, void* out) {
  constexpr int PHF = part_head_floats<D>();
  const int c = threadIdx.x;
  for (long long row = blockIdx.x; row < rows; row += gridDim.x) {
    float M = -INFINITY;
    for (int r = 0; r < R; ++r) M = fmaxf(M, states[((size_t)r * rows + row) * PHF]);
    float L = 0.f, Z = 0.f, O = 0.f, U = 0.f;
    for (int r = 0; r < R; ++r) {
      const float* sr = states + ((size_t)r * rows + row) * PHF;
      const float w = merge_weight(sr[0], M);
      L += w * sr[1];
      Z += w * sr[2];
      O += w * sr[4 + c];
      U += w * sr[4 + D + c];
    }
    float val = 0.f;
    if (L > 0.f) {
      const float inv = 1.f / L;
      val = ((1.f + Z * inv) * O - U) * inv;
    }
    store_elem<T>(out, (size_t)row * D + c, val);
  }
}

cudaError_t launch_merge_states(const float* states, int R, long long rows, void* out, int d,
                                bool bf16, cudaStream_t stream) {
  if (rows == 0) return cudaSuccess;
  const unsigned grid = (unsigned)(rows < 4096 ? rows : 4096);
  if (d == 128) {
    if (bf16) plx_merge_states_kernel<__nv_bfloat16, 128><<<grid, 128, 0, stream>>>(states, R, rows, out);
    else plx_merge_states_kernel<float, 128><<<grid, 128, 0, stream>>>(states, R, rows, out);
  } else if (d == 64) {
    if (bf16) plx_merge_states_kernel<__nv_bfloat16, 64><<<grid, 64, 0, stream>>>(states, R, rows, out);
    else plx_merge_states_kernel<float, 64><<<grid, 64, 0, stream>>>(states, R, rows, out);
  } else {
    return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// Host-side launch helpers (called from plx_abi.cu).
// ---------------------------------------------------------------------------
template <typename T, int D>
constexpr int decode_smem_bytes(int hpw) {
  using Cfg = DecodeTile<T, D>;
  return 1024 + Cfg::STAGES * Cfg::STAGE_BYTES + Cfg::STAGES * (int)sizeof(TileMeta) +
         2 * Cfg::STAGES * 8 + (int)sizeof(RangeInfo) + 20 * 8 +
         Cfg::NW * hpw * part_head_floats<D>() * 4 + 16 +
         (Cfg::MMA ? 0 : (2 * Cfg::NW * kDecRedRegion + 2 * Cfg::NW * 16) * 4);
}
static_assert(decode_smem_bytes<__nv_bfloat16, 128>(2) <= 227 * 1024, "shared memory");
// the merge buffer doubles as the piece-slot scratch of merge_tail (one int per
// CTA of the grid, at most one CTA per SM; 1024 SMs would still fit)
static_assert(DecodeTile<__nv_bfloat16, 64>::NW * part_head_floats<64>() >= 1024 &&
                  DecodeTile<float, 64>::NW * part_head_floats<64>() >= 1024,
              "merge buffer as slot scratch");
static_assert(decode_smem_bytes<__nv_bfloat16, 64>(2) <= 227 * 1024, "shared memory");
static_assert(decode_smem_bytes<float, 128>(2) <= 227 * 1024, "shared memory");
static_assert(decode_smem_bytes<float, 64>(2) <= 227 * 1024, "shared memory");

template <typename T, int D, int HPW>
cudaError_t launch_decode_t(const DecodeMaps& m, const DecodeParams& p, cudaStream_t stream) {
  using Cfg = DecodeTile<T, D>;
  const int smem = decode_smem_bytes<T, D>(HPW);
  auto kern = p.block_table ? plx_decode_splitk_kernel<T, D, HPW, kDecPaged>
               : p.state     ? plx_decode_splitk_kernel<T, D, HPW, kDecState>
                             : plx_decode_splitk_kernel<T, D, HPW, kDecContiguous>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  // programmatic dependent launch: see the start of the kernel
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)p.grid);
  cfg.blockDim = dim3(Cfg::THREADS);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  e = cudaLaunchKernelEx(&cfg, kern, m.k, m.v, m.k_chunk, m.v_chunk, p);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

template <typename T, int D>
cudaError_t launch_decode_d(const DecodeMaps& m, const DecodeParams& p, int hpw,
                            cudaStream_t stream) {
  switch (hpw) {
    case 1: return launch_decode_t<T, D, 1>(m, p, stream);
    case 2: return launch_decode_t<T, D, 2>(m, p, stream);
    default: return cudaErrorInvalidValue;
  }
}

// ---------------------------------------------------------------------------
// KV-cache append: the new token's key and value rows ([B, Hkv, d]) go to
// cache position seqlens[b] - 1 (the lengths already count the new token);
// batches of length 0 are skipped.  One 16-byte word per thread and step; a
// (b, kv-head) row is contiguous in both layouts.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256)
    plx_kv_append_kernel(const uint4* k_new, const uint4* v_new, uint4* k_cache,
                         uint4* v_cache, const int32_t* seqlens, int B, int Hkv,
                         int words_per_row, int S_max) {
  const long long row_words = (long long)Hkv * words_per_row;  // one batch, one position
  const long long n = (long long)B * row_words;
  for (long long w = (long long)blockIdx.x * blockDim.x + threadIdx.x; w < 2 * n;
       w += (long long)gridDim.x * blockDim.x) {
    const bool is_v = w >= n;
    const long long x = is_v ? w - n : w;
    const int b = (int)(x / row_words);
    const long long rem = x - (long long)b * row_words;
    const int len = clamp_len(seqlens[b], S_max);
    if (len == 0) continue;
    uint4* dst = (is_v ? v_cache : k_cache) + ((long long)b * S_max + (len - 1)) * row_words + rem;
    *dst = (is_v ? v_new : k_new)[x];
  }
}

cudaError_t launch_kv_append(const void* k_new, const void* v_new, void* k_cache, void* v_cache,
                             const int32_t* seqlens, int B, int Hkv, int d, int elem_bytes,
                             int S_max, cudaStream_t stream) {
  const int wpr = d * elem_bytes / 16;
  const long long words = 2ll * B * Hkv * wpr;
  if (words == 0) return cudaSuccess;
  long long blocks = (words + 255) / 256;
  if (blocks > 1184) blocks = 1184;  // 8 per SM of a 148-SM part; the loop covers the rest
  plx_kv_append_kernel<<<(unsigned)blocks, 256, 0, stream>>>(
      static_cast<const uint4*>(k_new), static_cast<const uint4*>(v_new),
      static_cast<uint4*>(k_cache), static_cast<uint4*>(v_cache), seqlens, B, Hkv, wpr, S_max);
  return cudaGetLastError();
}

cudaError_t launch_decode(bool bf16, int d, const DecodeMaps& m, const DecodeParams& p, int hpw,
                          cudaStream_t stream) {
  if (bf16) {
    if (d == 64) return launch_decode_d<__nv_bfloat16, 64>(m, p, hpw, stream);
    if (d == 128) return launch_decode_d<__nv_bfloat16, 128>(m, p, hpw, stream);
  } else {
    if (d == 64) return launch_decode_d<float, 64>(m, p, hpw, stream);
    if (d == 128) return launch_decode_d<float, 128>(m, p, hpw, stream);
  }
  return cudaErrorInvalidValue;
}

int decode_tile_keys(bool bf16, int d) {
  (void)d;
  return bf16 ? DecodeTile<__nv_bfloat16, 128>::TK : DecodeTile<float, 128>::TK;
}

int decode_box_cols(bool bf16, int d) { return bf16 ? 64 : d; }

}  // namespace plx
