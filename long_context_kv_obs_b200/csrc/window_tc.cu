// Window attention score on the tensor cores (tcgen05) - bf16 caches, head_dim 128.
#include "kernels.cuh"

namespace kvc {

bool window_tc_supported(const WinParams& p, kvc_dtype dt) {
  (void)p;
  (void)dt;
  return false;
}

cudaError_t launch_window_tc(const WinParams& p, cudaStream_t st) {
  (void)p;
  (void)st;
  return cudaErrorNotSupported;
}

}  // namespace kvc
