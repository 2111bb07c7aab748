// Forward scan for callers that cannot allocate device memory.
//
// Some callers have no way to call cudaMalloc when they run the scan: a
// plugin inside an inference engine or framework that owns every device
// allocation and forbids allocating on its execute path, or a real-time loop
// whose rule is "no allocation after start-up".  For them this entry point
// takes no workspace argument.  It runs the same forward kernels as
// ssm_scan_fwd, with their scratch (the look-back flags and carried states,
// and the error word) in one fixed device array that lives in this library.
//
// Costs and limits, for a user of this library:
//  - the array holds kStaticScratchBytes (4 MiB) on every GPU that loads the
//    library, from load until the process exits;
//  - shapes whose scratch would exceed it are rejected (SSM_ERR_UNSUPPORTED,
//    with a message on stderr) before anything is launched;
//  - every call shares the one array, so two calls whose kernels overlap on
//    the GPU (different streams without ordering, or several host threads)
//    race on it; order them on one stream;
//  - the first call on a device looks up the array's device address for
//    that device (cudaGetSymbolAddress, with that device current); make that
//    first call before any stream capture.
#include <mutex>
#include <stdio.h>
#include <string.h>

#include "ssm_common.cuh"
#include "ssm_scan.h"

namespace {

constexpr size_t kStaticScratchBytes = size_t(4) << 20;
constexpr int kMaxDevices = 64;

// The scratch itself.  Host code may not use the symbol as an address: it is
// a host-side stand-in, so the device address is looked up per device below.
__device__ __align__(256) unsigned char g_scan_scratch[kStaticScratchBytes];

struct DeviceScratch {
  std::once_flag once;
  void *ptr = nullptr;
  cudaError_t err = cudaSuccess;
};
DeviceScratch g_scratch[kMaxDevices];

}  // namespace

extern "C" ssm_status ssm_scan_fwd_noalloc(const ssm_shape *shape, const void *u, const void *delta,
                                           const float *A, const void *B, const void *C,
                                           const float *D, const void *z, const float *delta_bias,
                                           int delta_softplus, const float *initial_state, void *y,
                                           float *last_state, ssm_stream_t stream) {
  if (!shape) return SSM_ERR_INVALID_ARG;
  ssm_shape s = *shape;
  // AUTO takes the look-back schedule here: its scratch is bounded by the
  // resident warps, not by the problem size.
  if (s.path == SSM_PATH_AUTO) s.path = SSM_PATH_LOOKBACK;
  if (s.batch * s.dim * s.seqlen == 0)  // nothing that needs scratch
    return ssm_scan_fwd(&s, u, delta, A, B, C, D, z, delta_bias, delta_softplus, initial_state, y,
                        last_state, nullptr, 0, stream);
  const size_t need = ssm_scan_fwd_workspace_bytes(&s);
  if (need == 0) {
    // invalid shape, or no device: let the regular checks give the status
    return ssm_scan_fwd(&s, u, delta, A, B, C, D, z, delta_bias, delta_softplus, initial_state, y,
                        last_state, nullptr, 0, stream);
  }
  if (need > kStaticScratchBytes) {
    fprintf(stderr,
            "ssm_scan_fwd_noalloc: this shape needs %zu bytes of scratch, more than the %zu-byte "
            "static array; use ssm_scan_fwd with a workspace\n",
            need, kStaticScratchBytes);
    return SSM_ERR_UNSUPPORTED;
  }
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return SSM_ERR_CUDA;
  DeviceScratch &ds = g_scratch[dev];
  std::call_once(ds.once, [&ds]() {
    void *p = nullptr;
    ds.err = cudaGetSymbolAddress(&p, g_scan_scratch);
    ds.ptr = ds.err == cudaSuccess ? p : nullptr;
  });
  if (ds.err != cudaSuccess || !ds.ptr) {
    fprintf(stderr, "ssm_scan_fwd_noalloc: cudaGetSymbolAddress failed: %s\n",
            cudaGetErrorString(ds.err));
    return SSM_ERR_CUDA;
  }
  // ssm_scan_fwd clears the error word and the flags on `stream` first, so
  // nothing left in the array by an earlier call is read.
  return ssm_scan_fwd(&s, u, delta, A, B, C, D, z, delta_bias, delta_softplus, initial_state, y,
                      last_state, ds.ptr, kStaticScratchBytes, stream);
}
