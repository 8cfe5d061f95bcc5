// kvc_decode_attn_noalloc: decode attention for callers that cannot allocate.
//
// Some callers cannot call cudaMalloc and cannot hand the library a
// workspace: an inference runtime that reserved all device memory up front
// for its own pool, or code that must not trigger the device-wide
// synchronisation cudaMalloc / cudaFree may cause.  This entry point runs the
// same kernels as kvc_decode_attn, with their split-K partial results in a
// fixed array of this library's device memory instead of a caller workspace.
#include <mutex>
#include <stdio.h>

#include "kernels.cuh"

namespace kvc {

// Largest scratch the no-alloc path offers (bytes).  Every GPU that loads the
// library holds this array until the process exits.
constexpr size_t NOALLOC_SCRATCH_BYTES = size_t(8) << 20;

static __device__ __align__(256) unsigned char g_noalloc_scratch[NOALLOC_SCRATCH_BYTES];

kvc_status report(kvc_status s, const char* msg);  // api.cu: records kvc_last_error()

// Device address of g_noalloc_scratch on the current device.  Looked up once
// per device (with that device current) and cached; the host-side name of the
// array is only a stand-in, never a device address.
static kvc_status scratch_address(void** out) {
  static std::mutex mu;
  static void* cache[64] = {nullptr};
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return report(KVC_ERR_CUDA, "no current CUDA device");
  if (dev < 0 || dev >= 64) return report(KVC_ERR_UNSUPPORTED, "device ordinal above 63");
  std::lock_guard<std::mutex> lock(mu);
  if (!cache[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess || !p) {
      char m[160];
      snprintf(m, sizeof(m), "cudaGetSymbolAddress of the no-alloc scratch failed: %s",
               cudaGetErrorString(e));
      return report(KVC_ERR_CUDA, m);
    }
    cache[dev] = p;
  }
  *out = cache[dev];
  return KVC_OK;
}

}  // namespace kvc

extern "C" kvc_status kvc_decode_attn_noalloc(const kvc_model* m, const kvc_decode_args* a,
                                              kvc_stream_t stream) {
  using namespace kvc;
  size_t need = 0;
  kvc_status s = kvc_workspace_size(KVC_OP_DECODE, m, a, &need);
  if (s != KVC_OK) return s;
  if (need > NOALLOC_SCRATCH_BYTES) {
    char msg[200];
    snprintf(msg, sizeof(msg),
             "this decode needs %zu bytes of scratch; the no-alloc entry point has a fixed %zu "
             "(use kvc_decode_attn with a workspace)",
             need, NOALLOC_SCRATCH_BYTES);
    return report(KVC_ERR_WORKSPACE, msg);
  }
  void* scratch = nullptr;
  if ((s = scratch_address(&scratch)) != KVC_OK) return s;
  return kvc_decode_attn(m, a, scratch, NOALLOC_SCRATCH_BYTES, stream);
}
