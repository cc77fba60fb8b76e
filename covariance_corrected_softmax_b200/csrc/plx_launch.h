// plx_launch.h -- host-side declarations shared by the ABI layer and the
// kernel files: launch parameter structs and launchers.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "plx_decode.cuh"

namespace plx {

struct PrefillSimtParams {
  const float* q;    // [B, L, Hq, D]
  const float* rho;  // [B, L, Hq, D]
  const float* k;    // [B, L, Hkv, D]
  const float* v;    // [B, L, Hkv, D]
  float* out;        // [B, L, Hq, D]
  float* lse;        // [B, Hq, L] or null
  int B, L, Hq, Hkv, G, causal;
  float scale;
};

struct PrefillTcArgs {
  const void* q;
  const void* rho;
  const void* k;
  const void* v;
  void* out;
  float* lse;
  int B, L, Hq, Hkv, d, causal;
  int out_f32;  // 1: out is fp32, 0: out is bf16
  float scale;
  unsigned* err;
  int num_sms;
  // varlen (cu_seqlens != nullptr): q, rho, out [total, Hq, d], k, v [total,
  // Hkv, d]; B sequences, L = max_seqlen; lse [Hq, total]
  const int32_t* cu_seqlens = nullptr;
  int total = 0;
};

cudaError_t launch_prefill_simt(const PrefillSimtParams& p, int d, cudaStream_t stream);
// Tensor-core (tcgen05) bf16 prefill; encodes its own TMA descriptors.
cudaError_t launch_prefill_tc(const PrefillTcArgs& a, cudaStream_t stream);
// TMA maps of one decode call: k, v with tile-high boxes over the contiguous
// cache; k_chunk, v_chunk with 16-row boxes over the contiguous cache (a
// segment's partial last tile) or over the page pools (paged caches).  Boxes
// are decode_box_cols() wide; bf16 boxes use the 128-byte swizzle.
struct DecodeMaps {
  CUtensorMap k, v, k_chunk, v_chunk;
};
cudaError_t launch_decode(bool bf16, int d, const DecodeMaps& m, const DecodeParams& p, int hpw,
                          cudaStream_t stream);
int decode_tile_keys(bool bf16, int d);
int decode_box_cols(bool bf16, int d);
// out[row] from R softmax states [R, rows, 2d + 4] (see DecodeParams::state).
cudaError_t launch_merge_states(const float* states, int R, long long rows, void* out, int d,
                                bool bf16, cudaStream_t stream);
// Writes the new token's K and V rows ([B, Hkv, d], elem_bytes per element) at
// cache position seqlens[b] - 1 of every batch with a non-zero length.
cudaError_t launch_kv_append(const void* k_new, const void* v_new, void* k_cache, void* v_cache,
                             const int32_t* seqlens, int B, int Hkv, int d, int elem_bytes,
                             int S_max, cudaStream_t stream);

// rho[M, N] = x[M, K] w[N, K]^T (the probe projection): bf16 on the tensor
// cores (K % 8 == 0, N % 8 == 0, 16-byte aligned rows), fp32 on CUDA cores.
cudaError_t launch_probe_projection(const void* x, const void* w, void* rho, int M, int N, int K,
                                    bool bf16, int num_sms, unsigned* err, cudaStream_t stream);

// Gradients of the prefill operator: dq, drho [B, L, Hq, d], dk, dv
// [B, L, Hkv, d], all fp32; workspace of prefill_bwd_workspace_bytes().  fp32
// inputs run on the CUDA cores, bf16 inputs on the tensor cores (below).
size_t prefill_bwd_workspace_bytes(int B, int L, int Hq);
cudaError_t launch_prefill_bwd(const void* q, const void* rho, const void* k, const void* v,
                               const void* dout, float* dq, float* drho, float* dk, float* dv,
                               void* workspace, int causal, int B, int L, int Hq, int Hkv, int d,
                               bool bf16, float scale, unsigned* err, int num_sms,
                               cudaStream_t stream);

// The same gradients for bf16 inputs on the tensor cores (two tcgen05 kernels;
// d = 64 or 128).  The workspace holds the row statistics the first kernel
// computes for the second.
struct BwdTcArgs {
  const void *q, *rho, *k, *v, *dout;  // bf16
  float *dq, *drho, *dk, *dv;
  void* workspace;  // prefill_bwd_workspace_bytes()
  int B, L, Hq, Hkv, d, causal;
  float scale;
  unsigned* err;
  int num_sms;
};
cudaError_t launch_prefill_bwd_tc(const BwdTcArgs& a, cudaStream_t stream);

// One warp that waits on an mbarrier nothing ever completes, with the
// device's bounded wait: it records kDevTimeoutMbarrier when the limit runs out
// and returns (the failure-detection self-test).
cudaError_t launch_selftest_wait(unsigned* err, cudaStream_t stream);

// TMA descriptor encoder (cuTensorMapEncodeTiled through the runtime's driver
// entry point); null if unavailable.
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn tensor_map_encoder();

// Records a cudaError_t as this thread's plx_last_cuda_error().
void set_last_cuda_error(int e);

}  // namespace plx
