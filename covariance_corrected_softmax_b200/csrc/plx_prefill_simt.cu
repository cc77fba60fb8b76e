// plx_prefill_simt.cu -- Parallax prefill on CUDA cores, fp32 in and out.
//
// The fp32 path of plx_prefill_fwd: fp32 inputs need fp32 products to meet a
// 1e-4 absolute error bound, which the bf16 tensor-core path does not give.
// One warp owns one query row at a time; lanes split the head dimension.  For
// every visible key the warp forms s = scale q.k and t = rho.k (shuffle
// reductions), updates the running max / sum (m, l) and z = sum p t, and
// accumulates o = sum p v and u = sum p t v; the row ends with
// out = ((1 + z/l) o - u) / l and lse = ln(sum exp(s)).
// Operator: page 1 "Parallax: Parameterized Local Linear Attention Gives
// Transformers a 'Second Eye'", section 1.3 (o_PLX = o_SA - Sigma_KV rho), in
// the one-pass form that page 3 "Parallax keeps softmax, adds covariance
// correction branch" alludes to (one KV stream feeds both branches).
#include "plx_launch.h"

namespace plx {


constexpr int kSimtWarps = 8;
constexpr int kSimtRowsPerBlock = 32;

template <int D>
__global__ void __launch_bounds__(kSimtWarps * 32)
    plx_prefill_simt_kernel(const PrefillSimtParams p) {
  constexpr int EPL = D / 32;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int h = blockIdx.y, b = blockIdx.z, hk = h / p.G;
  const float log2e = 1.4426950408889634f;
  for (int r = warp; r < kSimtRowsPerBlock; r += kSimtWarps) {
    const int i = blockIdx.x * kSimtRowsPerBlock + r;
    if (i >= p.L) break;
    const size_t qoff = (((size_t)b * p.L + i) * p.Hq + h) * D + lane * EPL;
    float qv[EPL], rv[EPL], o[EPL], u[EPL];
#pragma unroll
    for (int e = 0; e < EPL; ++e) {
      qv[e] = p.q[qoff + e] * (p.scale * log2e);
      rv[e] = p.rho[qoff + e];
      o[e] = 0.f;
      u[e] = 0.f;
    }
    float m = -INFINITY, l = 0.f, z = 0.f;
    const int nkeys = p.causal ? i + 1 : p.L;
    for (int j = 0; j < nkeys; ++j) {
      const size_t koff = (((size_t)b * p.L + j) * p.Hkv + hk) * D + lane * EPL;
      float kv[EPL], vv[EPL];
      float s = 0.f, t = 0.f;
#pragma unroll
      for (int e = 0; e < EPL; ++e) {
        kv[e] = p.k[koff + e];
        vv[e] = p.v[koff + e];
        s = fmaf(qv[e], kv[e], s);
        t = fmaf(rv[e], kv[e], t);
      }
#pragma unroll
      for (int off = 16; off >= 1; off >>= 1) {
        s += __shfl_xor_sync(0xffffffffu, s, off);
        t += __shfl_xor_sync(0xffffffffu, t, off);
      }
      if (s > m) {
        const float alpha = (m == -INFINITY) ? 0.f : exp2f(m - s);
        l *= alpha;
        z *= alpha;
#pragma unroll
        for (int e = 0; e < EPL; ++e) {
          o[e] *= alpha;
          u[e] *= alpha;
        }
        m = s;
      }
      const float pr = exp2f(s - m);
      const float pt = pr * t;
      l += pr;
      z += pt;
#pragma unroll
      for (int e = 0; e < EPL; ++e) {
        o[e] = fmaf(pr, vv[e], o[e]);
        u[e] = fmaf(pt, vv[e], u[e]);
      }
    }
    const float inv = 1.f / l;
#pragma unroll
    for (int e = 0; e < EPL; ++e) p.out[qoff + e] = ((1.f + z * inv) * o[e] - u[e]) * inv;
    if (p.lse && lane == 0)
      p.lse[((size_t)b * p.Hq + h) * p.L + i] = (m + log2f(l)) * 0.6931471805599453f;
  }
}

cudaError_t launch_prefill_simt(const PrefillSimtParams& p, int d, cudaStream_t stream) {
  dim3 grid((p.L + kSimtRowsPerBlock - 1) / kSimtRowsPerBlock, p.Hq, p.B);
  if (d == 64)
    plx_prefill_simt_kernel<64><<<grid, kSimtWarps * 32, 0, stream>>>(p);
  else if (d == 128)
    plx_prefill_simt_kernel<128><<<grid, kSimtWarps * 32, 0, stream>>>(p);
  else
    return cudaErrorInvalidValue;
  return cudaGetLastError();
}

}  // namespace plx
