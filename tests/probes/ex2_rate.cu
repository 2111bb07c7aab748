// Throughput probe of the special-function unit's exp2 (ex2.approx.ftz.f32)
// on the device it runs on: one CTA per SM, 1024 threads, 8 independent
// chains of x <- 2^-x per thread (the chains converge to the fixed point near
// 0.64, so no value overflows).  Each CTA times itself with the SM cycle
// counter; the result is ex2 operations per SM per cycle, the denominator of
// the scan's special-function roofline.  Built and run by the GPU tests only.
#include <cuda_runtime.h>
#include <stdint.h>

__global__ void __launch_bounds__(1024) k_ex2_rate(int iters, float *sink, long long *cycles) {
  float x[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) x[i] = 0.01f * (threadIdx.x + i);
  __syncthreads();
  const long long t0 = clock64();
  for (int it = 0; it < iters; ++it) {
#pragma unroll
    for (int i = 0; i < 8; ++i) asm volatile("ex2.approx.ftz.f32 %0, %1;" : "=f"(x[i]) : "f"(-x[i]));
  }
  __syncthreads();
  const long long t1 = clock64();
  float s = 0.f;
#pragma unroll
  for (int i = 0; i < 8; ++i) s += x[i];
  sink[blockIdx.x * blockDim.x + threadIdx.x] = s;
  if (threadIdx.x == 0) cycles[blockIdx.x] = t1 - t0;
}

// Returns 0 on success; *rate = ex2 per SM per cycle (median over CTAs is
// left to the caller: per-CTA cycle counts are written to cycles_out).
extern "C" int ex2_rate_probe(int iters, int *sms_out, long long *cycles_out, int max_sms) {
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 1;
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 2;
  if (sms > max_sms || iters < 1 || iters > (1 << 20)) return 3;
  float *sink = nullptr;
  long long *cyc = nullptr;
  if (cudaMalloc(&sink, sizeof(float) * (size_t)sms * 1024) != cudaSuccess) return 4;
  if (cudaMalloc(&cyc, sizeof(long long) * (size_t)sms) != cudaSuccess) { cudaFree(sink); return 4; }
  k_ex2_rate<<<sms, 1024>>>(iters, sink, cyc);  // warm-up
  k_ex2_rate<<<sms, 1024>>>(iters, sink, cyc);
  cudaError_t e = cudaDeviceSynchronize();
  if (e == cudaSuccess) e = cudaMemcpy(cycles_out, cyc, sizeof(long long) * sms, cudaMemcpyDeviceToHost);
  cudaFree(sink);
  cudaFree(cyc);
  *sms_out = sms;
  return e == cudaSuccess ? 0 : 5;
}
