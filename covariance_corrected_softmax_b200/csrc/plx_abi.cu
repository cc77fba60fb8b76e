// plx_abi.cu -- the C ABI of libplx (declared in include/plx.h): host-side
// argument checks, TMA descriptor encoding and kernel launches.  No allocation,
// no synchronisation on the launch paths.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstddef>
#include <mutex>

#include "plx.h"
#include "plx_launch.h"


// The device status block (one per device context): the error word, which
// kernels receive the address of, and the limit of their bounded waits.
__device__ plx::DeviceStatus plx_g_status = {0u, 0u, plx::kWaitLimitNs};

namespace {

thread_local int t_last_cuda_error = 0;

constexpr int kMaxDevices = 64;
std::once_flag g_encode_once;
plx::EncodeTiledFn g_encode = nullptr;
int g_sm_count[kMaxDevices] = {0};
unsigned* g_err_ptr[kMaxDevices] = {nullptr};
std::mutex g_dev_mu;

plx_status cuda_fail(cudaError_t e) {
  t_last_cuda_error = static_cast<int>(e);
  return PLX_ERR_CUDA;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Per-device facts: SM count and the device address of the error word.
cudaError_t device_info(int* sms, unsigned** err) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lk(g_dev_mu);
  if (g_sm_count[dev] == 0) {
    int n = 0;
    e = cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
    void* ptr = nullptr;
    e = cudaGetSymbolAddress(&ptr, plx_g_status);
    if (e != cudaSuccess) return e;
    g_err_ptr[dev] = static_cast<unsigned*>(ptr);
    g_sm_count[dev] = n;
  }
  if (sms) *sms = g_sm_count[dev];
  if (err) *err = g_err_ptr[dev];
  return cudaSuccess;
}

cudaError_t get_encoder() {
  std::call_once(g_encode_once, [] {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &fn, 12000,
                                         cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_encode = reinterpret_cast<plx::EncodeTiledFn>(fn);
  });
  return g_encode ? cudaSuccess : cudaErrorNotSupported;
}

// 4-D map over a [B, S, H, D] tensor, box (box_cols, 1, box_rows, 1): bf16
// boxes of 64 columns with the 128-byte swizzle, fp32 boxes of full rows with
// none (plx::decode_box_cols).
cudaError_t encode_rows_map(CUtensorMap* map, const void* base, bool bf16, int B, int S, int H,
                            int D, int box_rows) {
  cudaError_t e = get_encoder();
  if (e != cudaSuccess) return e;
  const cuuint64_t esz = bf16 ? 2 : 4;
  cuuint64_t dims[4] = {(cuuint64_t)D, (cuuint64_t)H, (cuuint64_t)S, (cuuint64_t)B};
  cuuint64_t strides[3] = {D * esz, (cuuint64_t)H * D * esz, (cuuint64_t)S * H * D * esz};
  cuuint32_t box[4] = {(cuuint32_t)plx::decode_box_cols(bf16, D), 1, (cuuint32_t)box_rows, 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = g_encode(map, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32,
                        4, const_cast<void*>(base), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE,
                        bf16 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

// Query heads handled together per pass over a KV head's cache (register
// budget: two heads' q, rho, o and u per lane).
int heads_per_pass(int G) { return (G % 2 == 0) ? 2 : 1; }

size_t decode_ws_bytes_for(int d, int hpw, int grid) {
  const int pf = (d == 64) ? plx::part_floats<64>(hpw) : plx::part_floats<128>(hpw);
  return (size_t)(plx::kWsHeaderFloats + (size_t)2 * grid * pf) * sizeof(float);
}

bool shape_ok(int H_q, int H_kv, int d) {
  return H_q >= 1 && H_kv >= 1 && H_q % H_kv == 0 && (d == 64 || d == 128);
}

}  // namespace

namespace plx {
EncodeTiledFn tensor_map_encoder() { return get_encoder() == cudaSuccess ? g_encode : nullptr; }
void set_last_cuda_error(int e) { t_last_cuda_error = e; }
}  // namespace plx

extern "C" {

const char* plx_status_string(plx_status s) {
  switch (s) {
    case PLX_OK: return "PLX_OK";
    case PLX_ERR_INVALID_ARGUMENT: return "PLX_ERR_INVALID_ARGUMENT";
    case PLX_ERR_UNSUPPORTED: return "PLX_ERR_UNSUPPORTED";
    case PLX_ERR_WORKSPACE_TOO_SMALL: return "PLX_ERR_WORKSPACE_TOO_SMALL";
    case PLX_ERR_CUDA: return "PLX_ERR_CUDA";
  }
  return "PLX_ERR_UNKNOWN";
}

int plx_last_cuda_error(void) { return t_last_cuda_error; }

int plx_version(void) { return 100; }

plx_status plx_device_error(int* code, int clear) {
  if (!code) return PLX_ERR_INVALID_ARGUMENT;
  unsigned v = 0;
  cudaError_t e = cudaDeviceSynchronize();
  if (e != cudaSuccess) return cuda_fail(e);
  e = cudaMemcpyFromSymbol(&v, plx_g_status, sizeof(v), offsetof(plx::DeviceStatus, error));
  if (e != cudaSuccess) return cuda_fail(e);
  if (clear) {
    unsigned z = 0;
    e = cudaMemcpyToSymbol(plx_g_status, &z, sizeof(z), offsetof(plx::DeviceStatus, error));
    if (e != cudaSuccess) return cuda_fail(e);
  }
  *code = static_cast<int>(v);
  return PLX_OK;
}

plx_status plx_set_wait_limit_ns(unsigned long long ns) {
  t_last_cuda_error = 0;
  if (ns == 0) ns = plx::kWaitLimitNs;
  if (ns < 1000ull || ns > 60000000000ull) return PLX_ERR_INVALID_ARGUMENT;
  const unsigned long long v = ns;
  cudaError_t e = cudaDeviceSynchronize();  // no kernel may be mid-wait
  if (e != cudaSuccess) return cuda_fail(e);
  e = cudaMemcpyToSymbol(plx_g_status, &v, sizeof(v), offsetof(plx::DeviceStatus, wait_limit_ns));
  if (e != cudaSuccess) return cuda_fail(e);
  e = cudaDeviceSynchronize();
  return e == cudaSuccess ? PLX_OK : cuda_fail(e);
}

plx_status plx_selftest_wait(void* stream) {
  t_last_cuda_error = 0;
  unsigned* err = nullptr;
  cudaError_t e = device_info(nullptr, &err);
  if (e != cudaSuccess) return cuda_fail(e);
  e = plx::launch_selftest_wait(err, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? PLX_OK : cuda_fail(e);
}

size_t plx_decode_workspace_bytes(int B, int H_q, int H_kv, int d, int S_max) {
  if (B < 0 || S_max < 1 || !shape_ok(H_q, H_kv, d)) return 0;
  int sms = 0;
  if (device_info(&sms, nullptr) != cudaSuccess) return 0;
  return decode_ws_bytes_for(d, heads_per_pass(H_q / H_kv), sms);
}

}  // extern "C"

namespace {

plx_status prefill_impl(const void* q, const void* rho, const void* k, const void* v, void* out,
                        float* lse, int causal, int B, int L, int H_q, int H_kv, int d,
                        plx_dtype dtype, plx_dtype out_dtype, float softmax_scale, void* stream,
                        bool check_only);

// rho[M, N] = x[M, K] w_r[N, K]^T (all checks first; check_only stops there).
constexpr int kMaxProjRows = 0x7FFFFE00;  // 2^31 - 512
plx_status projection_impl(const void* x, const void* w_r, void* rho, int M, int N, int K,
                           plx_dtype dtype, void* stream, bool check_only) {
  t_last_cuda_error = 0;
  if (dtype != PLX_F32 && dtype != PLX_BF16) return PLX_ERR_INVALID_ARGUMENT;
  if (M < 0 || N < 0 || K < 1) return PLX_ERR_INVALID_ARGUMENT;
  if (M == 0 || N == 0) return PLX_OK;
  if (!x || !w_r || !rho || !aligned16(x) || !aligned16(w_r) || !aligned16(rho))
    return PLX_ERR_INVALID_ARGUMENT;
  if (dtype == PLX_BF16 && (K % 8 != 0 || N % 8 != 0)) return PLX_ERR_UNSUPPORTED;
  // tile row coordinates (up to 255 past M or N) are 32-bit; the fp32
  // kernel's grid holds 65535 tiles of 16 columns
  if (dtype == PLX_BF16 && (M > kMaxProjRows || N > kMaxProjRows)) return PLX_ERR_UNSUPPORTED;
  if (dtype == PLX_F32 && N > 65535 * 16) return PLX_ERR_UNSUPPORTED;
  if (check_only) return PLX_OK;
  int sms = 0;
  unsigned* err = nullptr;
  cudaError_t e = device_info(&sms, &err);
  if (e != cudaSuccess) return cuda_fail(e);
  e = plx::launch_probe_projection(x, w_r, rho, M, N, K, dtype == PLX_BF16, sms, err,
                                   static_cast<cudaStream_t>(stream));
  if (e == cudaErrorNotSupported) return PLX_ERR_UNSUPPORTED;
  return e == cudaSuccess ? PLX_OK : cuda_fail(e);
}

// plx_decode, preceded (when k_new is given) by the KV-cache append of
// plx_decode_append.  Every check runs before the first launch.
// Paged caches (block_table != nullptr): k_cache, v_cache are the page pools
// [num_pages, page_size, H_kv, d] and S_max = max_pages * page_size.
struct Paging {
  const int32_t* block_table = nullptr;
  int num_pages = 0, page_size = 0, max_pages = 0;
};

plx_status decode_impl(const void* q, const void* rho, const void* k_new, const void* v_new,
                       const void* k_cache, const void* v_cache, const int32_t* seqlens,
                       void* out, int B, int H_q, int H_kv, int d, int S_max, plx_dtype dtype,
                       float softmax_scale, void* workspace, size_t workspace_bytes,
                       void* stream, const Paging& pg = Paging(), float* state = nullptr,
                       bool check_only = false) {
  t_last_cuda_error = 0;
  if (dtype != PLX_F32 && dtype != PLX_BF16) return PLX_ERR_INVALID_ARGUMENT;
  if (B < 0 || S_max < 1 || !shape_ok(H_q, H_kv, d)) return PLX_ERR_INVALID_ARGUMENT;
  if (!(softmax_scale == softmax_scale) || softmax_scale > 3.0e38f || softmax_scale < -3.0e38f)
    return PLX_ERR_INVALID_ARGUMENT;
  if (B == 0) return PLX_OK;
  if (!q || !rho || !k_cache || !v_cache || !seqlens || !(out || state) || !workspace)
    return PLX_ERR_INVALID_ARGUMENT;
  if (!aligned16(q) || !aligned16(rho) || !aligned16(k_cache) || !aligned16(v_cache) ||
      !aligned16(out) || !aligned16(state) || !aligned16(workspace) ||
      (reinterpret_cast<uintptr_t>(seqlens) & 3u))
    return PLX_ERR_INVALID_ARGUMENT;
  if ((k_new != nullptr) != (v_new != nullptr)) return PLX_ERR_INVALID_ARGUMENT;
  if (k_new && (!aligned16(k_new) || !aligned16(v_new))) return PLX_ERR_INVALID_ARGUMENT;
  // TMA coordinates are 32-bit; cache extents must fit.
  if ((!pg.block_table && (long long)B * S_max > (1ll << 31)) || (long long)B * H_q > (1 << 30))
    return PLX_ERR_UNSUPPORTED;

  const bool bf16 = dtype == PLX_BF16;
  const int G = H_q / H_kv;
  const int hpw = heads_per_pass(G);
  int sms = 0;
  unsigned* err = nullptr;
  cudaError_t e = device_info(&sms, &err);
  if (e != cudaSuccess) return cuda_fail(e);
  const int tk = plx::decode_tile_keys(bf16, d);
  const long long max_tiles = (long long)B * H_kv * (G / hpw) * ((S_max + tk - 1) / tk);
  const int grid = (int)(max_tiles < sms ? max_tiles : sms);
  if (workspace_bytes < decode_ws_bytes_for(d, hpw, sms)) return PLX_ERR_WORKSPACE_TOO_SMALL;
  if (check_only) return PLX_OK;

  plx::DecodeMaps maps;
  if (pg.block_table) {
    // one [num_pages * page_size, H_kv, d] pool, 16-row boxes
    const int rows = pg.num_pages * pg.page_size;
    e = encode_rows_map(&maps.k_chunk, k_cache, bf16, 1, rows, H_kv, d, 16);
    if (e == cudaSuccess) e = encode_rows_map(&maps.v_chunk, v_cache, bf16, 1, rows, H_kv, d, 16);
    maps.k = maps.k_chunk;  // unused by the paged kernel
    maps.v = maps.v_chunk;
  } else {
    e = encode_rows_map(&maps.k, k_cache, bf16, B, S_max, H_kv, d, tk);
    if (e == cudaSuccess) e = encode_rows_map(&maps.v, v_cache, bf16, B, S_max, H_kv, d, tk);
    if (e == cudaSuccess) e = encode_rows_map(&maps.k_chunk, k_cache, bf16, B, S_max, H_kv, d, 16);
    if (e == cudaSuccess) e = encode_rows_map(&maps.v_chunk, v_cache, bf16, B, S_max, H_kv, d, 16);
  }
  if (e != cudaSuccess) return cuda_fail(e);

  const cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (k_new) {
    e = plx::launch_kv_append(k_new, v_new, const_cast<void*>(k_cache), const_cast<void*>(v_cache),
                              seqlens, B, H_kv, d, bf16 ? 2 : 4, S_max, st);
    if (e != cudaSuccess) return cuda_fail(e);
  }

  plx::DecodeParams p;
  p.q = q;
  p.rho = rho;
  p.seqlens = seqlens;
  p.out = out;
  p.ws = static_cast<float*>(workspace);
  p.B = B;
  p.Hq = H_q;
  p.Hkv = H_kv;
  p.G = G;
  p.S_max = S_max;
  p.nhg = G / hpw;
  p.qscale = softmax_scale * 1.4426950408889634f;
  p.grid = grid;
  p.err = err;
  p.block_table = pg.block_table;
  p.num_pages = pg.num_pages;
  p.page_size = pg.page_size;
  p.max_pages = pg.max_pages;
  p.state = state;
  e = plx::launch_decode(bf16, d, maps, p, hpw, st);
  if (e != cudaSuccess) return cuda_fail(e);
  return PLX_OK;
}

}  // namespace

extern "C" {

plx_status plx_decode(const void* q, const void* rho, const void* k_cache, const void* v_cache,
                      const int32_t* seqlens, void* out, int B, int H_q, int H_kv, int d,
                      int S_max, plx_dtype dtype, float softmax_scale, void* workspace,
                      size_t workspace_bytes, void* stream) {
  return decode_impl(q, rho, nullptr, nullptr, k_cache, v_cache, seqlens, out, B, H_q, H_kv, d,
                     S_max, dtype, softmax_scale, workspace, workspace_bytes, stream);
}

plx_status plx_prefill_varlen(const void* q, const void* rho, const void* k, const void* v,
                              void* out, float* lse, const int32_t* cu_seqlens, int num_seqs,
                              int total_tokens, int max_seqlen, int causal, int H_q, int H_kv,
                              int d, plx_dtype dtype, plx_dtype out_dtype, float softmax_scale,
                              void* stream) {
  t_last_cuda_error = 0;
  if (dtype != PLX_F32 && dtype != PLX_BF16) return PLX_ERR_INVALID_ARGUMENT;
  if (out_dtype != dtype && !(dtype == PLX_BF16 && out_dtype == PLX_F32))
    return PLX_ERR_INVALID_ARGUMENT;
  if (num_seqs < 0 || total_tokens < 0 || max_seqlen < 0 || !shape_ok(H_q, H_kv, d) ||
      (causal != 0 && causal != 1))
    return PLX_ERR_INVALID_ARGUMENT;
  if (!(softmax_scale == softmax_scale) || softmax_scale > 3.0e38f || softmax_scale < -3.0e38f)
    return PLX_ERR_INVALID_ARGUMENT;
  if (num_seqs == 0 || total_tokens == 0 || max_seqlen == 0) return PLX_OK;
  if (!q || !rho || !k || !v || !out || !cu_seqlens) return PLX_ERR_INVALID_ARGUMENT;
  if (!aligned16(q) || !aligned16(rho) || !aligned16(k) || !aligned16(v) || !aligned16(out) ||
      (reinterpret_cast<uintptr_t>(lse) & 3u) || (reinterpret_cast<uintptr_t>(cu_seqlens) & 3u))
    return PLX_ERR_INVALID_ARGUMENT;
  if (dtype != PLX_BF16) return PLX_ERR_UNSUPPORTED;  // the tensor-core path is bf16
  if ((long long)num_seqs * H_q * ((max_seqlen + 127) / 128) > 0x7fffffffll ||
      (long long)total_tokens * H_q > (1ll << 40) || H_q > 65535)
    return PLX_ERR_UNSUPPORTED;

  int sms = 0;
  unsigned* err = nullptr;
  cudaError_t e = device_info(&sms, &err);
  if (e != cudaSuccess) return cuda_fail(e);
  plx::PrefillTcArgs a;
  a.q = q;
  a.rho = rho;
  a.k = k;
  a.v = v;
  a.out = out;
  a.lse = lse;
  a.B = num_seqs;
  a.L = max_seqlen;
  a.Hq = H_q;
  a.Hkv = H_kv;
  a.d = d;
  a.causal = causal;
  a.out_f32 = out_dtype == PLX_F32 ? 1 : 0;
  a.scale = softmax_scale;
  a.err = err;
  a.num_sms = sms;
  a.cu_seqlens = cu_seqlens;
  a.total = total_tokens;
  e = plx::launch_prefill_tc(a, static_cast<cudaStream_t>(stream));
  if (e == cudaErrorNotSupported) return PLX_ERR_UNSUPPORTED;
  return e == cudaSuccess ? PLX_OK : cuda_fail(e);
}

plx_status plx_decode_state(const void* q, const void* rho, const void* k_cache,
                            const void* v_cache, const int32_t* seqlens, float* state, int B,
                            int H_q, int H_kv, int d, int S_max, plx_dtype dtype,
                            float softmax_scale, void* workspace, size_t workspace_bytes,
                            void* stream) {
  if (B > 0 && !state) {
    t_last_cuda_error = 0;
    return PLX_ERR_INVALID_ARGUMENT;
  }
  return decode_impl(q, rho, nullptr, nullptr, k_cache, v_cache, seqlens, nullptr, B, H_q, H_kv,
                     d, S_max, dtype, softmax_scale, workspace, workspace_bytes, stream, Paging(),
                     state);
}

plx_status plx_merge_states(const float* states, int R, void* out, int B, int H_q, int d,
                            plx_dtype out_dtype, void* stream) {
  t_last_cuda_error = 0;
  if (out_dtype != PLX_F32 && out_dtype != PLX_BF16) return PLX_ERR_INVALID_ARGUMENT;
  if (R < 1 || B < 0 || H_q < 1 || (d != 64 && d != 128)) return PLX_ERR_INVALID_ARGUMENT;
  if (B == 0) return PLX_OK;
  if (!states || !out || !aligned16(states) || !aligned16(out)) return PLX_ERR_INVALID_ARGUMENT;
  const cudaError_t e = plx::launch_merge_states(states, R, (long long)B * H_q, out, d,
                                                 out_dtype == PLX_BF16,
                                                 static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? PLX_OK : cuda_fail(e);
}

plx_status plx_decode_paged(const void* q, const void* rho, const void* k_pages,
                            const void* v_pages, const int32_t* block_table,
                            const int32_t* seqlens, void* out, int B, int H_q, int H_kv, int d,
                            int num_pages, int page_size, int max_pages_per_seq, plx_dtype dtype,
                            float softmax_scale, void* workspace, size_t workspace_bytes,
                            void* stream) {
  t_last_cuda_error = 0;
  if (page_size < 16 || page_size % 16 != 0 || num_pages < 1 || max_pages_per_seq < 1)
    return PLX_ERR_INVALID_ARGUMENT;
  if ((long long)num_pages * page_size > (1ll << 31) - 1 ||
      (long long)max_pages_per_seq * page_size > (1ll << 31) - 1)
    return PLX_ERR_UNSUPPORTED;
  if (B > 0 && (!block_table || (reinterpret_cast<uintptr_t>(block_table) & 3u)))
    return PLX_ERR_INVALID_ARGUMENT;
  Paging pg;
  pg.block_table = block_table;
  pg.num_pages = num_pages;
  pg.page_size = page_size;
  pg.max_pages = max_pages_per_seq;
  return decode_impl(q, rho, nullptr, nullptr, k_pages, v_pages, seqlens, out, B, H_q, H_kv, d,
                     max_pages_per_seq * page_size, dtype, softmax_scale, workspace,
                     workspace_bytes, stream, pg);
}

plx_status plx_decode_append(const void* q, const void* rho, const void* k_new,
                             const void* v_new, void* k_cache, void* v_cache,
                             const int32_t* seqlens, void* out, int B, int H_q, int H_kv, int d,
                             int S_max, plx_dtype dtype, float softmax_scale, void* workspace,
                             size_t workspace_bytes, void* stream) {
  if (B > 0 && (!k_new || !v_new)) {
    t_last_cuda_error = 0;
    return PLX_ERR_INVALID_ARGUMENT;
  }
  return decode_impl(q, rho, k_new, v_new, k_cache, v_cache, seqlens, out, B, H_q, H_kv, d,
                     S_max, dtype, softmax_scale, workspace, workspace_bytes, stream);
}

plx_status plx_prefill_fwd(const void* q, const void* rho, const void* k, const void* v,
                           void* out, float* lse, int causal, int B, int L, int H_q, int H_kv,
                           int d, plx_dtype dtype, float softmax_scale, void* stream) {
  return plx_prefill_fwd_ex(q, rho, k, v, out, lse, causal, B, L, H_q, H_kv, d, dtype, dtype,
                            softmax_scale, stream);
}

plx_status plx_prefill_fwd_ex(const void* q, const void* rho, const void* k, const void* v,
                              void* out, float* lse, int causal, int B, int L, int H_q, int H_kv,
                              int d, plx_dtype dtype, plx_dtype out_dtype, float softmax_scale,
                              void* stream) {
  return prefill_impl(q, rho, k, v, out, lse, causal, B, L, H_q, H_kv, d, dtype, out_dtype,
                      softmax_scale, stream, false);
}

}  // extern "C"

namespace {

plx_status prefill_impl(const void* q, const void* rho, const void* k, const void* v, void* out,
                        float* lse, int causal, int B, int L, int H_q, int H_kv, int d,
                        plx_dtype dtype, plx_dtype out_dtype, float softmax_scale, void* stream,
                        bool check_only) {
  t_last_cuda_error = 0;
  if (dtype != PLX_F32 && dtype != PLX_BF16) return PLX_ERR_INVALID_ARGUMENT;
  if (out_dtype != dtype && !(dtype == PLX_BF16 && out_dtype == PLX_F32))
    return PLX_ERR_INVALID_ARGUMENT;
  if (B < 0 || L < 0 || !shape_ok(H_q, H_kv, d) || (causal != 0 && causal != 1))
    return PLX_ERR_INVALID_ARGUMENT;
  if (!(softmax_scale == softmax_scale) || softmax_scale > 3.0e38f || softmax_scale < -3.0e38f)
    return PLX_ERR_INVALID_ARGUMENT;
  if (B == 0 || L == 0) return PLX_OK;
  if (!q || !rho || !k || !v || !out) return PLX_ERR_INVALID_ARGUMENT;
  if (!aligned16(q) || !aligned16(rho) || !aligned16(k) || !aligned16(v) || !aligned16(out) ||
      (reinterpret_cast<uintptr_t>(lse) & 3u))
    return PLX_ERR_INVALID_ARGUMENT;
  if ((long long)B * L > (1ll << 31) || B > 65535 || H_q > 65535) return PLX_ERR_UNSUPPORTED;
  if (check_only) return PLX_OK;

  int sms = 0;
  unsigned* err = nullptr;
  cudaError_t e = device_info(&sms, &err);
  if (e != cudaSuccess) return cuda_fail(e);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (dtype == PLX_F32) {
    plx::PrefillSimtParams p;
    p.q = static_cast<const float*>(q);
    p.rho = static_cast<const float*>(rho);
    p.k = static_cast<const float*>(k);
    p.v = static_cast<const float*>(v);
    p.out = static_cast<float*>(out);
    p.lse = lse;
    p.B = B;
    p.L = L;
    p.Hq = H_q;
    p.Hkv = H_kv;
    p.G = H_q / H_kv;
    p.causal = causal;
    p.scale = softmax_scale;
    e = plx::launch_prefill_simt(p, d, st);
    return e == cudaSuccess ? PLX_OK : cuda_fail(e);
  }
  plx::PrefillTcArgs a;
  a.q = q;
  a.rho = rho;
  a.k = k;
  a.v = v;
  a.out = out;
  a.lse = lse;
  a.B = B;
  a.L = L;
  a.Hq = H_q;
  a.Hkv = H_kv;
  a.d = d;
  a.causal = causal;
  a.out_f32 = out_dtype == PLX_F32 ? 1 : 0;
  a.scale = softmax_scale;
  a.err = err;
  a.num_sms = sms;
  e = plx::launch_prefill_tc(a, st);
  if (e == cudaErrorNotSupported) return PLX_ERR_UNSUPPORTED;
  return e == cudaSuccess ? PLX_OK : cuda_fail(e);
}

}  // namespace

extern "C" {

plx_status plx_probe_projection(const void* x, const void* w_r, void* rho, int M, int N, int K,
                                plx_dtype dtype, void* stream) {
  return projection_impl(x, w_r, rho, M, N, K, dtype, stream, false);
}

plx_status plx_prefill_fwd_x(const void* q, const void* x, const void* w_r, const void* k,
                             const void* v, void* rho, void* out, float* lse, int causal, int B,
                             int L, int H_q, int H_kv, int d, int d_model, plx_dtype dtype,
                             float softmax_scale, void* stream) {
  // every argument of both steps is checked before the first launch
  if (B < 0 || L < 0 || !shape_ok(H_q, H_kv, d) || d_model < 1) {
    t_last_cuda_error = 0;
    return PLX_ERR_INVALID_ARGUMENT;
  }
  const long long M = (long long)B * L;
  if (M > 0x7fffffffll || (long long)H_q * d > 0x7fffffffll) {
    t_last_cuda_error = 0;
    return PLX_ERR_UNSUPPORTED;
  }
  plx_status s = projection_impl(x, w_r, rho, (int)M, H_q * d, d_model, dtype, stream, true);
  if (s == PLX_OK)
    s = prefill_impl(q, rho, k, v, out, lse, causal, B, L, H_q, H_kv, d, dtype, dtype,
                     softmax_scale, stream, true);
  if (s != PLX_OK || M == 0) return s;
  s = projection_impl(x, w_r, rho, (int)M, H_q * d, d_model, dtype, stream, false);
  if (s != PLX_OK) return s;
  return prefill_impl(q, rho, k, v, out, lse, causal, B, L, H_q, H_kv, d, dtype, dtype,
                      softmax_scale, stream, false);
}

plx_status plx_decode_x(const void* q, const void* x, const void* w_r, const void* k_cache,
                        const void* v_cache, const int32_t* seqlens, void* rho, void* out, int B,
                        int H_q, int H_kv, int d, int S_max, int d_model, plx_dtype dtype,
                        float softmax_scale, void* workspace, size_t workspace_bytes,
                        void* stream) {
  if (B < 0 || !shape_ok(H_q, H_kv, d) || d_model < 1) {
    t_last_cuda_error = 0;
    return PLX_ERR_INVALID_ARGUMENT;
  }
  plx_status s = projection_impl(x, w_r, rho, B, H_q * d, d_model, dtype, stream, true);
  if (s == PLX_OK)
    s = decode_impl(q, rho, nullptr, nullptr, k_cache, v_cache, seqlens, out, B, H_q, H_kv, d,
                    S_max, dtype, softmax_scale, workspace, workspace_bytes, stream, Paging(),
                    nullptr, true);
  if (s != PLX_OK || B == 0) return s;
  s = projection_impl(x, w_r, rho, B, H_q * d, d_model, dtype, stream, false);
  if (s != PLX_OK) return s;
  return decode_impl(q, rho, nullptr, nullptr, k_cache, v_cache, seqlens, out, B, H_q, H_kv, d,
                     S_max, dtype, softmax_scale, workspace, workspace_bytes, stream);
}

size_t plx_prefill_bwd_workspace_bytes(int B, int L, int H_q) {
  if (B < 0 || L < 0 || H_q < 1) return 0;
  return plx::prefill_bwd_workspace_bytes(B, L, H_q);
}

plx_status plx_prefill_bwd(const void* q, const void* rho, const void* k, const void* v,
                           const void* dout, float* dq, float* drho, float* dk, float* dv,
                           int causal, int B, int L, int H_q, int H_kv, int d, plx_dtype dtype,
                           float softmax_scale, void* workspace, size_t workspace_bytes,
                           void* stream) {
  t_last_cuda_error = 0;
  if (dtype != PLX_F32 && dtype != PLX_BF16) return PLX_ERR_INVALID_ARGUMENT;
  if (B < 0 || L < 0 || !shape_ok(H_q, H_kv, d) || (causal != 0 && causal != 1))
    return PLX_ERR_INVALID_ARGUMENT;
  if (!(softmax_scale == softmax_scale) || softmax_scale > 3.0e38f || softmax_scale < -3.0e38f)
    return PLX_ERR_INVALID_ARGUMENT;
  if (B == 0 || L == 0) return PLX_OK;
  if (!q || !rho || !k || !v || !dout || !dq || !drho || !dk || !dv || !workspace)
    return PLX_ERR_INVALID_ARGUMENT;
  if (!aligned16(q) || !aligned16(rho) || !aligned16(k) || !aligned16(v) || !aligned16(dout) ||
      !aligned16(dq) || !aligned16(drho) || !aligned16(dk) || !aligned16(dv) ||
      !aligned16(workspace))
    return PLX_ERR_INVALID_ARGUMENT;
  if ((long long)B * L * H_q > 0x7fffffffll * 8) return PLX_ERR_UNSUPPORTED;
  if (workspace_bytes < plx::prefill_bwd_workspace_bytes(B, L, H_q))
    return PLX_ERR_WORKSPACE_TOO_SMALL;
  int sms = 0;
  unsigned* err = nullptr;
  cudaError_t e = device_info(&sms, &err);
  if (e != cudaSuccess) return cuda_fail(e);
  e = plx::launch_prefill_bwd(q, rho, k, v, dout, dq, drho, dk, dv, workspace, causal, B, L, H_q,
                              H_kv, d, dtype == PLX_BF16, softmax_scale, err, sms,
                              static_cast<cudaStream_t>(stream));
  if (e == cudaErrorNotSupported) return PLX_ERR_UNSUPPORTED;
  return e == cudaSuccess ? PLX_OK : cuda_fail(e);
}

}  // extern "C"


