// plx_decode_static.cu -- plx_decode_static_ws: decode that allocates nothing.
//
// plx_decode needs a device workspace for the partial softmax states of the
// KV segments it splits across CTAs, and leaves allocating it to the caller.
// Some callers cannot allocate device memory at the point where they decode:
// a serving loop that must not enter the allocator on its per-token path
// (cudaMalloc can synchronise the device and stall for milliseconds), a plugin
// whose host framework owns the whole device memory pool and hands out no
// extra buffers, or a C caller that has no device allocator at hand at all.
// This entry point serves them: it runs the same kernels as plx_decode with
// the workspace taken from a fixed array in the library's device memory.
//
// The array has a fixed size (kStaticScratchBytes, 1 MiB) and exists once per
// GPU that loads the library, for the life of the process.  Every call on a
// device shares it, so calls whose kernels may overlap on the GPU (other
// streams, other host threads) race on it; serialise them.  Nothing in it needs
// clearing between calls: the kernels rewrite every word they later read (each
// CTA invalidates its own partial slots before any other kernel reads them).
#include <cuda_runtime.h>

#include <mutex>

#include "plx.h"
#include "plx_launch.h"

namespace {

constexpr size_t kStaticScratchBytes = size_t(1) << 20;  // 1 MiB

// Workspace plx_decode needs on a device with `sms` multiprocessors: a header
// plus two partial-state slots per CTA of the persistent grid (at most one CTA
// per SM), each slot holding `hpw` heads' (m, l, z, pad, o[d], u[d]).
constexpr size_t static_need(int sms, int d, int hpw) {
  return (size_t)(plx::kWsHeaderFloats + (size_t)2 * sms * (plx::kPartHeader + hpw * (2 * d + 4))) *
         sizeof(float);
}
// B200 (148 SMs) at the widest slot (d = 128, two heads per pass) fits, and so
// does any device with up to 250 SMs.
static_assert(static_need(148, 128, 2) <= kStaticScratchBytes, "B200 must fit");
static_assert(static_need(250, 128, 2) <= kStaticScratchBytes, "250 SMs must fit");
static_assert(static_need(251, 128, 2) > kStaticScratchBytes, "limit stated in plx.h");

// The scratch itself.  In host code this name is only a stand-in for the
// symbol, not a device address: kernels get the address from
// cudaGetSymbolAddress below.
static __device__ __align__(256) unsigned char plx_static_scratch[kStaticScratchBytes];

constexpr int kMaxStaticDevices = 64;
std::mutex g_static_mu;
void* g_static_ptr[kMaxStaticDevices] = {nullptr};

// Device address of the scratch array on the current device, looked up once per
// device (the first call on a device does this set-up).
cudaError_t static_scratch_address(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxStaticDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lk(g_static_mu);
  if (!g_static_ptr[dev]) {
    void* ptr = nullptr;
    e = cudaGetSymbolAddress(&ptr, plx_static_scratch);
    if (e != cudaSuccess) return e;
    g_static_ptr[dev] = ptr;
  }
  *out = g_static_ptr[dev];
  return cudaSuccess;
}

}  // namespace

extern "C" {

PLX_API plx_status plx_decode_static_ws(const void* q, const void* rho, const void* k_cache,
                                        const void* v_cache, const int32_t* seqlens, void* out,
                                        int B, int H_q, int H_kv, int d, int S_max,
                                        plx_dtype dtype, float softmax_scale, void* stream) {
  if (B == 0) {
    // Nothing to do; plx_decode performs the same checks and returns PLX_OK.
    return plx_decode(q, rho, k_cache, v_cache, seqlens, out, B, H_q, H_kv, d, S_max, dtype,
                      softmax_scale, nullptr, 0, stream);
  }
  void* scratch = nullptr;
  const cudaError_t e = static_scratch_address(&scratch);
  if (e != cudaSuccess) {
    plx::set_last_cuda_error(static_cast<int>(e));
    return PLX_ERR_CUDA;
  }
  // The shape decides how many CTAs split the cache and so how much scratch the
  // partial states take; refuse shapes that would not fit the fixed array.
  // (An invalid shape gives 0 here and is rejected by plx_decode's checks.)
  const size_t need = plx_decode_workspace_bytes(B, H_q, H_kv, d, S_max);
  if (need > kStaticScratchBytes) return PLX_ERR_WORKSPACE_TOO_SMALL;
  return plx_decode(q, rho, k_cache, v_cache, seqlens, out, B, H_q, H_kv, d, S_max, dtype,
                    softmax_scale, scratch, kStaticScratchBytes, stream);
}

}  // extern "C"
