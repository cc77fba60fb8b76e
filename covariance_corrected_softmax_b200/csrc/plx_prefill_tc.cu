// plx_prefill_tc.cu -- bf16 Parallax prefill on the tcgen05 tensor cores.
#include "plx_launch.h"

namespace plx {

cudaError_t launch_prefill_tc(const PrefillTcArgs& a, cudaStream_t stream) {
  (void)a;
  (void)stream;
  return cudaErrorNotSupported;
}

}  // namespace plx
