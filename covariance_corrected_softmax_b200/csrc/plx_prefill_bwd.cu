// plx_prefill_bwd.cu -- gradients of the Parallax prefill operator for fp32
// inputs (CUDA cores, fp32 arithmetic throughout: the fp32 bar needs fp32
// products).  bf16 inputs go to the tensor-core kernels of
// plx_prefill_bwd_tc.cu.
//
// Operator (page 1 "Parallax: Parameterized Local Linear Attention Gives
// Transformers a 'Second Eye'", opening formula and section 1.3; page 3
// "Parallax keeps softmax, adds covariance correction branch"), row i, keys j:
//   a_j = softmax_j(scale q.k_j),  t_j = rho.k_j,  tbar = sum a t,
//   out = sum_j a_j c_j v_j,  c_j = 1 + tbar - t_j.
// The pages print no gradient; with g = dLoss/dout, o = sum a v:
//   dv_j += a_j c_j g
//   dt_j  = a_j (g.o - g.v_j)
//   ds_j  = a_j (c_j g.v_j + t_j g.o - D),   D = g.out + tbar g.o
//   dq   += scale sum_j ds_j k_j,   drho += sum_j dt_j k_j
//   dk_j += scale ds_j q + dt_j rho
// Everything is recomputed from q, rho, k, v and g in fp32, the softmax
// normaliser included: the products ds_j = a_j (X_j - D) cancel where one key
// dominates a row, and would amplify the fp16 rounding that the tensor-core
// forward's normaliser (and so its lse) carries.  Two kernels:
//   rows:  one warp per query row; a first pass over the row's keys runs an
//          online softmax (running max and sum) and forms tbar, g.o, o and u
//          (so g.out = g.((1 + tbar) o - u) needs no saved output), a second
//          pass accumulates dq and drho; the row's lse, tbar, g.o and D go to
//          the workspace.
//   keys:  one warp per key row of a KV head; it visits every query row of the
//          head group that sees the key and accumulates dk and dv.
// Lanes split the head dimension; dot products are warp sums.
#include "plx_launch.h"

namespace plx {

namespace {

template <typename T>
__device__ __forceinline__ void load_slice(const T* p, float (&f)[4], int n);
template <>
__device__ __forceinline__ void load_slice<float>(const float* p, float (&f)[4], int n) {
  if (n == 4) {
    const float4 w = *reinterpret_cast<const float4*>(p);
    f[0] = w.x; f[1] = w.y; f[2] = w.z; f[3] = w.w;
  } else {
    const float2 w = *reinterpret_cast<const float2*>(p);
    f[0] = w.x; f[1] = w.y; f[2] = f[3] = 0.f;
  }
}

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  return x;
}

__device__ __forceinline__ float dot4(const float (&a)[4], const float (&b)[4]) {
  return fmaf(a[0], b[0], fmaf(a[1], b[1], fmaf(a[2], b[2], a[3] * b[3])));
}

struct BwdParams {
  const void *q, *rho, *k, *v, *g;
  float *dq, *drho, *dk, *dv;
  float4* stats;      // [B, Hq, L]: lse, tbar, g.o, D
  int B, L, Hq, Hkv, G, causal;
  float scale;
};

template <typename T, int D>
__global__ void __launch_bounds__(256) plx_bwd_rows_kernel(const BwdParams p) {
  constexpr int E = D / 32;  // elements per lane
  const long long r = (long long)blockIdx.x * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  const long long rows = (long long)p.B * p.Hq * p.L;
  if (r >= rows) return;
  const int i = (int)(r % p.L);
  const int h = (int)((r / p.L) % p.Hq);
  const int b = (int)(r / ((long long)p.L * p.Hq));
  const int hk = h / p.G;
  const T* Q = static_cast<const T*>(p.q);
  const T* R = static_cast<const T*>(p.rho);
  const T* Gd = static_cast<const T*>(p.g);
  const T* K = static_cast<const T*>(p.k);
  const T* V = static_cast<const T*>(p.v);
  const size_t qo = (((size_t)b * p.L + i) * p.Hq + h) * D + lane * E;
  float q[4], rh[4], g[4];
  load_slice<T>(Q + qo, q, E);
  load_slice<T>(R + qo, rh, E);
  load_slice<T>(Gd + qo, g, E);
  const int n = p.causal ? i + 1 : p.L;
  auto krow = [&](int j) { return (((size_t)b * p.L + j) * p.Hkv + hk) * D + lane * E; };
  // pass 1 (online softmax): lse, tbar, g.o, o, u
  float m = -INFINITY, l = 0.f;
  float tbar = 0.f, go = 0.f, o[4] = {0.f, 0.f, 0.f, 0.f}, u[4] = {0.f, 0.f, 0.f, 0.f};
  for (int j = 0; j < n; ++j) {
    float kk[4], vv[4];
    load_slice<T>(K + krow(j), kk, E);
    load_slice<T>(V + krow(j), vv, E);
    const float s = warp_sum(dot4(q, kk)) * p.scale;
    const float t = warp_sum(dot4(rh, kk));
    const float gv = warp_sum(dot4(g, vv));
    if (s > m) {  // new running max: rescale the sums (all zero at the first key)
      const float c = m == -INFINITY ? 0.f : expf(m - s);
      l *= c;
      tbar *= c;
      go *= c;
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        o[e] *= c;
        u[e] *= c;
      }
      m = s;
    }
    const float a = expf(s - m);
    l += a;
    tbar = fmaf(a, t, tbar);
    go = fmaf(a, gv, go);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      o[e] = fmaf(a, vv[e], o[e]);
      u[e] = fmaf(a * t, vv[e], u[e]);
    }
  }
  const float inv = 1.f / l;
  const float lse = m + logf(l);
  tbar *= inv;
  go *= inv;
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    o[e] *= inv;
    u[e] *= inv;
  }
  float outv[4];
#pragma unroll
  for (int e = 0; e < 4; ++e) outv[e] = (1.f + tbar) * o[e] - u[e];
  const float dsum = warp_sum(dot4(g, outv)) + tbar * go;
  // pass 2: dq, drho
  float dq[4] = {0.f, 0.f, 0.f, 0.f}, dr[4] = {0.f, 0.f, 0.f, 0.f};
  for (int j = 0; j < n; ++j) {
    float kk[4], vv[4];
    load_slice<T>(K + krow(j), kk, E);
    load_slice<T>(V + krow(j), vv, E);
    const float s = warp_sum(dot4(q, kk)) * p.scale;
    const float t = warp_sum(dot4(rh, kk));
    const float gv = warp_sum(dot4(g, vv));
    const float a = expf(s - lse);
    const float dt = a * (go - gv);
    const float ds = a * ((1.f + tbar - t) * gv + t * go - dsum);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      dq[e] = fmaf(p.scale * ds, kk[e], dq[e]);
      dr[e] = fmaf(dt, kk[e], dr[e]);
    }
  }
#pragma unroll
  for (int e = 0; e < E; ++e) {
    p.dq[qo + e] = dq[e];
    p.drho[qo + e] = dr[e];
  }
  if (lane == 0) p.stats[r] = make_float4(lse, tbar, go, dsum);
}

template <typename T, int D>
__global__ void __launch_bounds__(256) plx_bwd_keys_kernel(const BwdParams p) {
  constexpr int E = D / 32;
  const long long w = (long long)blockIdx.x * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  const long long keys = (long long)p.B * p.Hkv * p.L;
  if (w >= keys) return;
  const int j = (int)(w % p.L);
  const int hk = (int)((w / p.L) % p.Hkv);
  const int b = (int)(w / ((long long)p.L * p.Hkv));
  const T* Q = static_cast<const T*>(p.q);
  const T* R = static_cast<const T*>(p.rho);
  const T* Gd = static_cast<const T*>(p.g);
  const size_t ko = (((size_t)b * p.L + j) * p.Hkv + hk) * D + lane * E;
  float kk[4], vv[4];
  load_slice<T>(static_cast<const T*>(p.k) + ko, kk, E);
  load_slice<T>(static_cast<const T*>(p.v) + ko, vv, E);
  float dk[4] = {0.f, 0.f, 0.f, 0.f}, dv[4] = {0.f, 0.f, 0.f, 0.f};
  for (int h = hk * p.G; h < (hk + 1) * p.G; ++h) {
    for (int i = p.causal ? j : 0; i < p.L; ++i) {
      const size_t qo = (((size_t)b * p.L + i) * p.Hq + h) * D + lane * E;
      const long long r = ((long long)b * p.Hq + h) * p.L + i;
      float q[4], rh[4], g[4];
      load_slice<T>(Q + qo, q, E);
      load_slice<T>(R + qo, rh, E);
      load_slice<T>(Gd + qo, g, E);
      const float4 st = p.stats[r];  // lse, tbar, g.o, D
      const float s = warp_sum(dot4(q, kk)) * p.scale;
      const float t = warp_sum(dot4(rh, kk));
      const float gv = warp_sum(dot4(g, vv));
      const float a = expf(s - st.x);
      const float c = 1.f + st.y - t;
      const float dt = a * (st.z - gv);
      const float ds = a * (c * gv + t * st.z - st.w);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        dk[e] = fmaf(p.scale * ds, q[e], fmaf(dt, rh[e], dk[e]));
        dv[e] = fmaf(a * c, g[e], dv[e]);
      }
    }
  }
#pragma unroll
  for (int e = 0; e < E; ++e) {
    p.dk[ko + e] = dk[e];
    p.dv[ko + e] = dv[e];
  }
}

template <typename T, int D>
cudaError_t launch_bwd_t(const BwdParams& p, cudaStream_t stream) {
  const long long rows = (long long)p.B * p.Hq * p.L, keys = (long long)p.B * p.Hkv * p.L;
  plx_bwd_rows_kernel<T, D><<<(unsigned)((rows + 7) / 8), 256, 0, stream>>>(p);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  plx_bwd_keys_kernel<T, D><<<(unsigned)((keys + 7) / 8), 256, 0, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace

size_t prefill_bwd_workspace_bytes(int B, int L, int Hq) {
  return (size_t)B * Hq * L * sizeof(float4);
}

cudaError_t launch_prefill_bwd(const void* q, const void* rho, const void* k, const void* v,
                               const void* dout, float* dq, float* drho, float* dk, float* dv,
                               void* workspace, int causal, int B, int L, int Hq, int Hkv, int d,
                               bool bf16, float scale, unsigned* err, int num_sms,
                               cudaStream_t stream) {
  if (bf16) {
    // bf16: the tensor-core kernels
    BwdTcArgs a;
    a.q = q;
    a.rho = rho;
    a.k = k;
    a.v = v;
    a.dout = dout;
    a.dq = dq;
    a.drho = drho;
    a.dk = dk;
    a.dv = dv;
    a.workspace = workspace;
    a.B = B;
    a.L = L;
    a.Hq = Hq;
    a.Hkv = Hkv;
    a.d = d;
    a.causal = causal;
    a.scale = scale;
    a.err = err;
    a.num_sms = num_sms;
    return launch_prefill_bwd_tc(a, stream);
  }
  BwdParams p;
  p.q = q;
  p.rho = rho;
  p.k = k;
  p.v = v;
  p.g = dout;
  p.dq = dq;
  p.drho = drho;
  p.dk = dk;
  p.dv = dv;
  p.stats = static_cast<float4*>(workspace);
  p.B = B;
  p.L = L;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.G = Hq / Hkv;
  p.causal = causal;
  p.scale = scale;
  if (d == 128) return launch_bwd_t<float, 128>(p, stream);
  if (d == 64) return launch_bwd_t<float, 64>(p, stream);
  return cudaErrorInvalidValue;
}

}  // namespace plx
