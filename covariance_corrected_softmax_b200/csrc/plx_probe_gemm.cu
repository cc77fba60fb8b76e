// plx_probe_gemm.cu -- the probe projection rho = W_R x (page 1 "Parallax:
// Parameterized Local Linear Attention Gives Transformers a 'Second Eye'",
// section 1.3: the one extra projection matrix; page 3 "Parallax keeps
// softmax, adds covariance correction branch": rho_i = W_R x_i).
//
// For all tokens at once this is the GEMM rho[M, N] = x[M, K] W_R[N, K]^T
// (M tokens, K = model width, N = H_q d), run on the 5th-generation tensor
// cores for bf16: persistent CTAs over 128 x 128 output tiles (consecutive tiles
// share the x tile, W_R stays in L2), a 6-stage ring of 128 x 64 x and W_R
// tiles fed by TMA (128-byte swizzle), tcgen05.mma (M = 128, N = 128, K = 16)
// issued by one thread into one of two TMEM accumulators, and four epilogue
// warps that read the other accumulator (tcgen05.ld), round to bf16 and store
// while the next tile accumulates.  fp32 inputs take a plain CUDA-core kernel
// (the correctness path).
#include "plx_launch.h"

namespace plx {

namespace {

constexpr int kPM = 128, kPN = 128, kPK = 64;  // output tile, k block (128-byte rows)
constexpr int kPStages = 6;
constexpr int kPThreads = 256;                 // warps: 0 TMA, 1 MMA, 2 TMEM, 4-7 epilogue
constexpr int kPTileBytes = kPM * kPK * 2;     // one A (or B) tile, 16 KB
constexpr int kPStageBytes = 2 * kPTileBytes;
constexpr uint32_t kPIdesc = umma_idesc_f16kind(kPM, kPN, false, false);

struct ProjBars {
  uint64_t full[kPStages], empty[kPStages];
  uint64_t acc_full[2], acc_empty[2];
  uint64_t drain;
};

struct ProjParams {
  void* rho;
  int M, N, K;
  int tiles_n, tiles, kblocks;
  unsigned* err;
};

__global__ void __launch_bounds__(kPThreads, 1)
    plx_probe_gemm_kernel(const __grid_constant__ CUtensorMap xmap,
                          const __grid_constant__ CUtensorMap wmap, const ProjParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  ProjBars* bars = reinterpret_cast<ProjBars*>(smem + kPStages * kPStageBytes);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  if (tid == 0) {
    *abort_flag = 0;
    for (int s = 0; s < kPStages; ++s) {
      mbar_init(&bars->full[s], 1);
      mbar_init(&bars->empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&bars->acc_full[a], 1);
      mbar_init(&bars->acc_empty[a], 4);  // one arrival per epilogue warp
    }
    mbar_init(&bars->drain, 1);
    fence_mbarrier_init();
  }
  if (warp == 2) {
    tmem_alloc(tmem_slot, 256);
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
      long long it = 0;
      bool ok = true;
      for (int u = blockIdx.x; ok && u < p.tiles; u += gridDim.x) {
        const int mb = u / p.tiles_n, nb = u % p.tiles_n;
        for (int kb = 0; kb < p.kblocks; ++kb, ++it) {
          const int s = (int)(it % kPStages);
          if (it >= kPStages &&
              !mbar_wait(&bars->empty[s], (uint32_t)(((it / kPStages) - 1) & 1), abort_flag, p.err)) {
            ok = false;
            break;
          }
          uint8_t* st = smem + s * kPStageBytes;
          mbar_arrive_expect_tx(&bars->full[s], kPStageBytes);
          tma_load_2d(st, &xmap, &bars->full[s], kb * kPK, mb * kPM);
          tma_load_2d(st + kPTileBytes, &wmap, &bars->full[s], kb * kPK, nb * kPN);
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
      long long it = 0;
      int lt = 0;
      bool ok = true;
      for (int u = blockIdx.x; ok && u < p.tiles; u += gridDim.x, ++lt) {
        const int ab = lt & 1;
        if (lt >= 2 &&
            !mbar_wait(&bars->acc_empty[ab], (uint32_t)(((lt >> 1) - 1) & 1), abort_flag, p.err)) {
          ok = false;
          break;
        }
        tc_fence_after();
        for (int kb = 0; kb < p.kblocks; ++kb, ++it) {
          const int s = (int)(it % kPStages);
          if (!mbar_wait(&bars->full[s], (uint32_t)((it / kPStages) & 1), abort_flag, p.err)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sa = (uint32_t)(s * kPStageBytes) >> 4;
          const uint32_t sb = (uint32_t)(s * kPStageBytes + kPTileBytes) >> 4;
#pragma unroll
          for (int k = 0; k < kPK / 16; ++k)
            umma_ss(tbase + ab * kPN, d0 + sa + 2 * k, d0 + sb + 2 * k, kPIdesc,
                    (kb > 0 || k > 0) ? 1u : 0u);
          umma_commit(&bars->empty[s]);  // the stage is free once these MMAs complete
        }
        if (!ok) break;
        umma_commit(&bars->acc_full[ab]);
      }
      // every MMA must have completed before the columns are released
      umma_commit(&bars->drain);
      volatile int never = 0;
      mbar_wait(&bars->drain, 0, &never, p.err);
    }
    __syncwarp();
  } else if (warp >= 4) {
    // ------------------------------------------------------------ epilogue
    const int qd = warp & 3;                     // TMEM lane quadrant
    const int r = qd * 32 + lane;                // row of the tile = TMEM lane
    const uint32_t lane_addr = tbase + ((uint32_t)(qd * 32) << 16);
    int lt = 0;
    for (int u = blockIdx.x; u < p.tiles; u += gridDim.x, ++lt) {
      const int ab = lt & 1;
      if (!mbar_wait(&bars->acc_full[ab], (uint32_t)((lt >> 1) & 1), abort_flag, p.err)) break;
      tc_fence_after();
      const int mb = u / p.tiles_n, nb = u % p.tiles_n;
      const long long row = (long long)mb * kPM + r;
      __nv_bfloat16* dst = static_cast<__nv_bfloat16*>(p.rho) + row * p.N + (size_t)nb * kPN;
#pragma unroll 1
      for (int c = 0; c < kPN; c += 32) {
        uint32_t v[32];
        tmem_ld32_sync(lane_addr + ab * kPN + c, v);
        if (row < p.M) {
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const int col = nb * kPN + c + 8 * q;
            if (col + 8 <= p.N) {
              uint4 w;
              w.x = float2_to_bf16x2(__uint_as_float(v[8 * q]), __uint_as_float(v[8 * q + 1]));
              w.y = float2_to_bf16x2(__uint_as_float(v[8 * q + 2]), __uint_as_float(v[8 * q + 3]));
              w.z = float2_to_bf16x2(__uint_as_float(v[8 * q + 4]), __uint_as_float(v[8 * q + 5]));
              w.w = float2_to_bf16x2(__uint_as_float(v[8 * q + 6]), __uint_as_float(v[8 * q + 7]));
              *reinterpret_cast<uint4*>(dst + c + 8 * q) = w;
            }
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->acc_empty[ab]);
    }
  }
  __syncthreads();
  if (warp == 2) {
    tc_fence_after();
    tmem_dealloc(tbase, 256);
  }
}

// fp32: one thread per output, 16 x 16 output tiles through shared memory.
__global__ void __launch_bounds__(256)
    plx_probe_simt_kernel(const float* x, const float* w, float* rho, int M, int N, int K) {
  __shared__ float xs[16][17], ws[16][17];
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  const long long m = (long long)blockIdx.y * 16 + ty;
  const long long n = (long long)blockIdx.x * 16 + tx;
  float acc = 0.f;
  for (int k0 = 0; k0 < K; k0 += 16) {
    const long long mx = (long long)blockIdx.y * 16 + ty, nw = (long long)blockIdx.x * 16 + ty;
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

}  // namespace

cudaError_t launch_probe_projection(const void* x, const void* w, void* rho, int M, int N, int K,
                                    bool bf16, int num_sms, unsigned* err, cudaStream_t stream) {
  if (M == 0 || N == 0) return cudaSuccess;
  if (!bf16) {
    dim3 grid((N + 15) / 16, (M + 15) / 16);
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
  p.tiles_n = (N + kPN - 1) / kPN;
  const long long tiles = (long long)((M + kPM - 1) / kPM) * p.tiles_n;
  if (tiles > 0x7fffffffll) return cudaErrorInvalidValue;
  p.tiles = (int)tiles;
  p.kblocks = (K + kPK - 1) / kPK;
  p.err = err;
  const int smem = 1024 + kPStages * kPStageBytes + (int)sizeof(ProjBars) + 16;
  e = cudaFuncSetAttribute(plx_probe_gemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  const int grid = (int)(tiles < num_sms ? tiles : num_sms);
  plx_probe_gemm_kernel<<<grid, kPThreads, smem, stream>>>(xm, wm, p);
  return cudaGetLastError();
}

}  // namespace plx
