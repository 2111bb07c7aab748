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
//  - the array holds kStaticScratchBytes (16 MiB) on every GPU that loads the
//    library, from load until the process exits;
//  - shapes whose scratch would exceed it are rejected (SSM_ERR_UNSUPPORTED,
//    with a message on stderr) before anything is launched;
//  - every call shares the one array, so two calls whose kernels overlap on
//    the GPU (different streams without ordering, or several host threads)
//    race on it; order them on one stream;
//  - every call looks up the array's device address for the current device
//    and context (cudaGetSymbolAddress, a host-side query that allocates
//    nothing); nothing is cached, so a device reset or a new context between
//    calls is harmless, and a lookup that fails (for example because the
//    module cannot be loaded while a stream is being captured) fails only
//    that call.
#include <stdio.h>
#include <string.h>

#include <cmath>
#include <vector>

#include "ssm_common.cuh"
#include "ssm_scan.h"

namespace {

constexpr size_t kStaticScratchBytes = size_t(16) << 20;

// The scratch itself.  Host code may not use the symbol as an address: it is
// a host-side stand-in, so the device address is looked up on every call.
__device__ __align__(256) unsigned char g_scan_scratch[kStaticScratchBytes];

}  // namespace

extern "C" ssm_status ssm_scan_fwd_noalloc(const ssm_shape *shape, const void *u, const void *delta,
                                           const float *A, const void *B, const void *C,
                                           const float *D, const void *z, const float *delta_bias,
                                           int delta_softplus, const float *initial_state, void *y,
                                           float *last_state, ssm_stream_t stream) {
  if (!shape) return SSM_ERR_INVALID_ARG;
  ssm_shape s = *shape;
  // Saved chunk states would sit in the shared array, where no backward call
  // can reach them and the next call overwrites them.
  if (s.flags & SSM_FLAG_SAVE_STATES) {
    fprintf(stderr, "ssm_scan_fwd_noalloc: SSM_FLAG_SAVE_STATES needs a caller-owned workspace; "
                    "use ssm_scan_fwd\n");
    return SSM_ERR_UNSUPPORTED;
  }
  if (s.batch * s.dim * s.seqlen == 0)  // nothing that needs scratch
    return ssm_scan_fwd(&s, u, delta, A, B, C, D, z, delta_bias, delta_softplus, initial_state, y,
                        last_state, nullptr, 0, stream);
  // AUTO keeps the regular choice when its scratch is bounded by the resident
  // warps (the look-back schedules, warp-specialised or not) or needs none
  // (one warp per group); the split-L schedule, whose scratch grows with the
  // problem, is replaced by the look-back one.
  if (s.path == SSM_PATH_AUTO) {
    const int32_t p = ssm_scan_fwd_path(&s);
    if (p == SSM_PATH_SPLIT_L) s.path = SSM_PATH_LOOKBACK;
  }
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
  void *ptr = nullptr;
  const cudaError_t e = cudaGetSymbolAddress(&ptr, g_scan_scratch);
  if (e != cudaSuccess || !ptr) {
    fprintf(stderr, "ssm_scan_fwd_noalloc: cudaGetSymbolAddress failed: %s\n", cudaGetErrorString(e));
    cudaGetLastError();  // the failure belongs to this call only
    return SSM_ERR_CUDA;
  }
  // ssm_scan_fwd clears the error word and the flags on `stream` first, so
  // nothing left in the array by an earlier call is read.
  return ssm_scan_fwd(&s, u, delta, A, B, C, D, z, delta_bias, delta_softplus, initial_state, y,
                      last_state, ptr, kStaticScratchBytes, stream);
}

// Test hook: the no-allocation forward on a small seeded problem, a device
// reset, then the same call on buffers allocated afresh.  The scratch array's
// address is looked up again after the reset, so both calls must give equal
// bits.  0: equal; 1: they differ; negative: the ssm_status of a failed call,
// or SSM_ERR_CUDA for a failed allocation, copy or reset.
extern "C" int32_t ssm_scan_test_noalloc_reset_cycle(void) {
  constexpr int64_t Bt = 2, Dm = 32, Ls = 200, N = 16;
  const int64_t n_act = Bt * Dm * Ls, n_bc = Bt * Ls * N;
  std::vector<float> u(n_act), dl(n_act), z(n_act), Bm(n_bc), Cm(n_bc), A(Dm * N), Dd(Dm), bias(Dm);
  // smooth, deterministic inputs of the layer's ranges (A negative, delta near 0)
  for (int64_t i = 0; i < n_act; ++i) {
    u[i] = (float)std::sin(0.37 * (double)i);
    dl[i] = (float)(0.5 * std::cos(0.11 * (double)i) - 1.0);
    z[i] = (float)std::sin(0.23 * (double)i + 1.0);
  }
  for (int64_t i = 0; i < n_bc; ++i) {
    Bm[i] = (float)std::cos(0.05 * (double)i);
    Cm[i] = (float)std::sin(0.07 * (double)i + 0.5);
  }
  for (int64_t d = 0; d < Dm; ++d) {
    for (int64_t n = 0; n < N; ++n) A[d * N + n] = -(float)(n + 1);
    Dd[d] = 1.f;
    bias[d] = (float)(0.01 * (double)d);
  }
  ssm_shape s;
  memset(&s, 0, sizeof(s));
  s.batch = Bt; s.dim = Dm; s.seqlen = Ls; s.dstate = N;
  s.io_dtype = SSM_F32; s.path = SSM_PATH_AUTO;

  auto run = [&](std::vector<float> &y, std::vector<float> &last) -> int32_t {
    const std::vector<float> *in[8] = {&u, &dl, &A, &Bm, &Cm, &Dd, &z, &bias};
    float *dev[8] = {nullptr}, *dy = nullptr, *dls = nullptr;
    int32_t rc = 0;
    for (int k = 0; k < 8 && rc == 0; ++k) {
      const size_t bytes = in[k]->size() * sizeof(float);
      if (cudaMalloc(&dev[k], bytes) != cudaSuccess ||
          cudaMemcpy(dev[k], in[k]->data(), bytes, cudaMemcpyHostToDevice) != cudaSuccess)
        rc = SSM_ERR_CUDA;
    }
    if (rc == 0 && (cudaMalloc(&dy, n_act * sizeof(float)) != cudaSuccess ||
                    cudaMalloc(&dls, Bt * Dm * N * sizeof(float)) != cudaSuccess))
      rc = SSM_ERR_CUDA;
    if (rc == 0) {
      const ssm_status st = ssm_scan_fwd_noalloc(&s, dev[0], dev[1], dev[2], dev[3], dev[4], dev[5], dev[6],
                                                 dev[7], 1, nullptr, dy, dls, nullptr);
      if (st != SSM_OK) rc = st;
    }
    if (rc == 0 && cudaDeviceSynchronize() != cudaSuccess) rc = SSM_ERR_CUDA;
    if (rc == 0) {
      y.resize(n_act);
      last.resize(Bt * Dm * N);
      if (cudaMemcpy(y.data(), dy, n_act * sizeof(float), cudaMemcpyDeviceToHost) != cudaSuccess ||
          cudaMemcpy(last.data(), dls, last.size() * sizeof(float), cudaMemcpyDeviceToHost) != cudaSuccess)
        rc = SSM_ERR_CUDA;
    }
    for (float *p : dev) cudaFree(p);
    cudaFree(dy);
    cudaFree(dls);
    return rc;
  };

  std::vector<float> y1, l1, y2, l2;
  int32_t rc = run(y1, l1);
  if (rc != 0) return rc;
  if (cudaDeviceReset() != cudaSuccess) return SSM_ERR_CUDA;
  rc = run(y2, l2);
  if (rc != 0) return rc;
  const bool same = memcmp(y1.data(), y2.data(), y1.size() * sizeof(float)) == 0 &&
                    memcmp(l1.data(), l2.data(), l1.size() * sizeof(float)) == 0;
  return same ? 0 : 1;
}
