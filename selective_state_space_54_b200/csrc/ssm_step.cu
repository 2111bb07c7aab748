// Single-step (recurrent) update of the selective SSM for sm_100a.
//
// For every batch element b and channel d, one new token:
//   Delta = softplus(delta + delta_bias[d])                 (or delta + bias)
//   h_n  <- exp(Delta * A[d,n]) * h_n + Delta * B[b,n] * u   for n < N
//   y    =  (sum_n C[b,n] h_n + D[d] u) * SiLU(z)
// This is the constant-time-per-token inference mode of the recurrence: the
// fixed-size state (D x N per layer) is all that is kept between tokens
// ("Mamba: Linear-Time Sequence Modeling with Selective State Spaces",
// xyznot.com reading guide, the question on KV caches; "O que e um modelo
// Mamba?", ibm.com, on constant inference memory; "Как работает Mamba",
// aivaro.ru, the O(1)-per-step comparison).  The update is the same
// arithmetic as one step of the scan (ssm_fwd.cu), Euler input term
// Delta * B * u, with the same softplus and SiLU.
//
// Design (B200): the step moves 8 bytes of fp32 state per (b, d, n) (read
// and written once) and 8 bytes of token data per (b, d) in bf16, so it is
// bound by HBM: the kernel's job is to keep enough state bytes in flight.
// A lane owns S = 8 consecutive states of a channel (LPC = N / 8 lanes per
// channel), so that per-channel work (softplus, gate, indexing) is shared by
// 8 states.  On the vector path (N % 8 == 0, 16-byte rows) persistent blocks
// walk the batch rows of their channels with the next row's state slices in
// flight while the current one computes (k_step_rows); other shapes take one
// row per block and plain masked loads (k_step).  The state is read and
// written with streaming (evict-first) accesses: it is touched once per token.
// A, B and C are re-read across batch elements or channels and are served
// from L2/L1.
#include <algorithm>
#include <atomic>

#include "ssm_common.cuh"

namespace ssm {

constexpr int kStepThreads = 256;

template <typename T, int S>
__device__ __forceinline__ void load_io(const T *p, bool vec, int n0, int N, float (&o)[S]);

template <int S>
__device__ __forceinline__ void load_io(const uint16_t *p, bool vec, int n0, int N, float (&o)[S]) {
  if (vec) {
#pragma unroll
    for (int q = 0; q < S / 4; ++q) {
      const uint2 v = __ldg(reinterpret_cast<const uint2 *>(p + n0 + 4 * q));
      o[4 * q] = bf16_lo(v.x); o[4 * q + 1] = bf16_hi(v.x);
      o[4 * q + 2] = bf16_lo(v.y); o[4 * q + 3] = bf16_hi(v.y);
    }
  } else {
#pragma unroll
    for (int i = 0; i < S; ++i) o[i] = n0 + i < N ? bf16_to_f(p[n0 + i]) : 0.f;
  }
}
template <int S>
__device__ __forceinline__ void load_io(const float *p, bool vec, int n0, int N, float (&o)[S]) {
  if (vec) {
#pragma unroll
    for (int q = 0; q < S / 4; ++q) {
      const float4 v = __ldg(reinterpret_cast<const float4 *>(p + n0 + 4 * q));
      o[4 * q] = v.x; o[4 * q + 1] = v.y; o[4 * q + 2] = v.z; o[4 * q + 3] = v.w;
    }
  } else {
#pragma unroll
    for (int i = 0; i < S; ++i) o[i] = n0 + i < N ? p[n0 + i] : 0.f;
  }
}

// grid: x over the (channel, lane) slots of one batch row, y over batch rows
template <typename T, int S, int LPC>
__global__ void __launch_bounds__(kStepThreads) k_step(StepParams p) {
  const int64_t slot = (int64_t)blockIdx.x * kStepThreads + threadIdx.x;
  const int j = (int)(slot % LPC);
  int64_t d = slot / LPC;
  const bool live = d < p.dim;
  if (!live) d = p.dim - 1;  // lanes past the row compute on its last channel, store nothing
  const int N = p.N, n0 = S * j;
  const bool grp = n0 < N;   // lanes past the last group of S states hold zeros
  // S-state groups fully inside the row take 16-byte accesses
  const bool vec = p.vec != 0 && n0 + S <= N;
  for (int64_t b = blockIdx.y; b < p.batch; b += gridDim.y) {
    const int64_t ch = b * p.dim + d;
    const float uu = IO<T>::get(static_cast<const T *>(p.u), ch);
    float s = IO<T>::get(static_cast<const T *>(p.delta), ch);
    if (p.bias) s += p.bias[d];
    const float dl = p.softplus ? softplus_fast(s) : s;
    const float du = dl * uu;
    float h[S], a[S], Bv[S], Cv[S];
    float *hp = p.state + ch * N + n0;
    const float *ap = p.A + d * N + n0;
    if (vec) {
#pragma unroll
      for (int q = 0; q < S / 4; ++q) {
        const float4 hv = __ldcs(reinterpret_cast<const float4 *>(hp + 4 * q));
        const float4 av = __ldg(reinterpret_cast<const float4 *>(ap + 4 * q));
        h[4 * q] = hv.x; h[4 * q + 1] = hv.y; h[4 * q + 2] = hv.z; h[4 * q + 3] = hv.w;
        a[4 * q] = av.x; a[4 * q + 1] = av.y; a[4 * q + 2] = av.z; a[4 * q + 3] = av.w;
      }
    } else {
#pragma unroll
      for (int i = 0; i < S; ++i) {
        const bool in = n0 + i < N;
        h[i] = in ? hp[i] : 0.f;
        a[i] = in ? ap[i] : 0.f;
      }
    }
    load_io<S>(static_cast<const T *>(p.B) + b * N, vec, n0, N, Bv);
    load_io<S>(static_cast<const T *>(p.C) + b * N, vec, n0, N, Cv);
    float y0 = 0.f, y1 = 0.f;
#pragma unroll
    for (int i = 0; i < S; i += 2) {
      const float x0 = dl * a[i] * kLog2e, x1 = dl * a[i + 1] * kLog2e;
      const float e0 = ex2(x0), e1 = ex2(x1);
      const float b0 = p.zoh ? du * expm1_over_x(x0, e0) : du;
      const float b1 = p.zoh ? du * expm1_over_x(x1, e1) : du;
      h[i] = fmaf(e0, h[i], b0 * Bv[i]);
      h[i + 1] = fmaf(e1, h[i + 1], b1 * Bv[i + 1]);
      y0 = fmaf(Cv[i], h[i], y0);  // states past N have C = 0 and h = 0
      y1 = fmaf(Cv[i + 1], h[i + 1], y1);
    }
    float yp = y0 + y1;
#pragma unroll
    for (int o = LPC / 2; o > 0; o >>= 1) yp += __shfl_xor_sync(0xffffffffu, yp, o);
    if (live) {
      if (vec) {
#pragma unroll
        for (int q = 0; q < S / 4; ++q)
          __stcs(reinterpret_cast<float4 *>(hp + 4 * q),
                 make_float4(h[4 * q], h[4 * q + 1], h[4 * q + 2], h[4 * q + 3]));
      } else if (grp) {
#pragma unroll
        for (int i = 0; i < S; ++i)
          if (n0 + i < N) hp[i] = h[i];
      }
      if (j == 0) {
        float y = yp + (p.D ? p.D[d] * uu : 0.f);
        if (p.z) y *= silu_fast(IO<T>::get(static_cast<const T *>(p.z), ch));
        IO<T>::store1(static_cast<T *>(p.y), ch, y);
      }
    }
  }
}

template <typename T, int S, int LPC>
static cudaError_t launch_step_k(const StepParams &p, cudaStream_t s) {
  const int64_t slots = p.dim * LPC;
  const int64_t bx = (slots + kStepThreads - 1) / kStepThreads;
  if (bx > 0x7fffffff) return cudaErrorInvalidConfiguration;
  const dim3 grid((unsigned)bx, (unsigned)(p.batch < 65535 ? p.batch : 65535));
  k_step<T, S, LPC><<<grid, kStepThreads, 0, s>>>(p);
  return cudaGetLastError();
}

// ---- vector path: persistent blocks over batch rows ---------------------------
// A block owns kStepThreads / LPC channels (a channel slice) and walks the
// batch rows b = kb, kb + bps, ... of that slice, bps blocks per slice, as
// many as fill the SMs in one wave.  Every lane keeps two row buffers in
// registers: the next row's S states (one 32-byte load where the state is
// 32-byte aligned, two 16-byte ones otherwise) and its u, delta and z are
// loaded before the current row computes, and the state and token lines of
// the row after that are prefetched into L2, so that each lane has a row in
// flight while it computes.  A, D and the bias of the lane's channel are
// loaded once.
// Held to 64 registers for 4 blocks (32 warps) per SM with bf16 token data
// (3 blocks with fp32, whose wider loads spill at 64).  On B200 at the
// Mamba-2.8B decode shape (batch 128, token inputs cycled over 4 slots so
// that they come from DRAM, CUDA graph replay): 18.3 us per step, against
// 20.0 us without the token-line prefetch (the 2-byte token loads then wait
// on DRAM every row), 22.4 us when B and C lines are prefetched as well,
// 19.9 us with B and C staged through a shared-memory ring, and 20.9 us for
// non-persistent blocks of 4 rows loaded up front; a plain device copy of the
// same bytes takes 15.5 us.  Prefetching 3 rows ahead instead of 2 measured
// 3 % slower, both distances 5 %.  With inputs that stay in L2 a third row buffer
// (two rows in flight) measured 20.7 against 18.6 us, rows taken in pairs at
// 3 blocks per SM 19.6 us.
template <typename T>
constexpr int step_blocks_per_sm() { return sizeof(T) == 2 ? 4 : 3; }

// one batch row of a lane's channel: its state slice and token inputs
template <int S>
struct StepRow {
  float h[S];
  float u, s, z;  // s = delta + bias
};

template <typename T, int S, int LPC>
__global__ void __launch_bounds__(kStepThreads, step_blocks_per_sm<T>()) k_step_rows(StepParams p, int bps) {
  static_assert(S == 8, "a lane's 8 states are one 32-byte access");
  const int tid = threadIdx.x;
  const int slice = (int)(blockIdx.x / bps), kb = (int)(blockIdx.x - slice * bps);
  const int64_t slot = (int64_t)slice * kStepThreads + tid;
  const int j = (int)(slot % LPC);
  int64_t d = slot / LPC;
  const bool live = d < p.dim;
  if (!live) d = p.dim - 1;  // lanes past the row compute on its last channel, store nothing
  const int N = p.N, n0 = S * j;
  const bool v32 = (reinterpret_cast<uintptr_t>(p.state) & 31) == 0;
  // per-channel constants, shared by every row
  float a[S];
  {
    const float *ap = p.A + d * N + n0;
#pragma unroll
    for (int q = 0; q < S / 4; ++q) {
      const float4 av = __ldg(reinterpret_cast<const float4 *>(ap + 4 * q));
      a[4 * q] = av.x * kLog2e; a[4 * q + 1] = av.y * kLog2e;
      a[4 * q + 2] = av.z * kLog2e; a[4 * q + 3] = av.w * kLog2e;
    }
  }
  const float bias = p.bias ? p.bias[d] : 0.f;
  const float Dd = p.D ? p.D[d] : 0.f;

  auto load = [&](StepRow<S> &r, int64_t b) {
    const float *hp = p.state + (b * p.dim + d) * N + n0;
    if (v32) {
      asm volatile("ld.global.cs.v8.f32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
                   : "=f"(r.h[0]), "=f"(r.h[1]), "=f"(r.h[2]), "=f"(r.h[3]), "=f"(r.h[4]), "=f"(r.h[5]),
                     "=f"(r.h[6]), "=f"(r.h[7])
                   : "l"(hp));
    } else {
      const float4 h0 = __ldcs(reinterpret_cast<const float4 *>(hp));
      const float4 h1 = __ldcs(reinterpret_cast<const float4 *>(hp + 4));
      r.h[0] = h0.x; r.h[1] = h0.y; r.h[2] = h0.z; r.h[3] = h0.w;
      r.h[4] = h1.x; r.h[5] = h1.y; r.h[6] = h1.z; r.h[7] = h1.w;
    }
    const int64_t ch = b * p.dim + d;
    r.u = IO<T>::get(static_cast<const T *>(p.u), ch);
    r.s = IO<T>::get(static_cast<const T *>(p.delta), ch) + bias;
    r.z = p.z ? IO<T>::get(static_cast<const T *>(p.z), ch) : 0.f;
  };
  // a later row's state lines and u, delta, z lines into L2, one lane per
  // 128-byte line (4 lanes of state; 128 / sizeof(T) channels of token data)
  constexpr int kTokLineLanes = LPC * 128 / (int)sizeof(T);
  auto prefetch = [&](int64_t b) {
    if (b < p.batch && (tid & 3) == 0)
      asm volatile("prefetch.global.L2 [%0];" ::"l"(p.state + (b * p.dim + d) * N + n0));
    if (b < p.batch && tid % kTokLineLanes == 0) {
      const int64_t ch = b * p.dim + d;
      asm volatile("prefetch.global.L2 [%0];" ::"l"(static_cast<const T *>(p.u) + ch));
      asm volatile("prefetch.global.L2 [%0];" ::"l"(static_cast<const T *>(p.delta) + ch));
      if (p.z) asm volatile("prefetch.global.L2 [%0];" ::"l"(static_cast<const T *>(p.z) + ch));
    }
  };
  auto run = [&](const StepRow<S> &r, int64_t b) {
    float Bv[S], Cv[S];
    load_io<S>(static_cast<const T *>(p.B) + b * N, true, n0, N, Bv);
    load_io<S>(static_cast<const T *>(p.C) + b * N, true, n0, N, Cv);
    const float dl = p.softplus ? softplus_fast(r.s) : r.s;
    const float du = dl * r.u;
    float h[S];
#pragma unroll
    for (int i = 0; i < S; ++i) h[i] = r.h[i];
    float y0 = 0.f, y1 = 0.f;
#pragma unroll
    for (int i = 0; i < S; i += 2) {
      const float x0 = dl * a[i], x1 = dl * a[i + 1];  // a holds A * log2(e)
      const float e0 = ex2(x0), e1 = ex2(x1);
      const float b0 = p.zoh ? du * expm1_over_x(x0, e0) : du;
      const float b1 = p.zoh ? du * expm1_over_x(x1, e1) : du;
      h[i] = fmaf(e0, h[i], b0 * Bv[i]);
      h[i + 1] = fmaf(e1, h[i + 1], b1 * Bv[i + 1]);
      y0 = fmaf(Cv[i], h[i], y0);
      y1 = fmaf(Cv[i + 1], h[i + 1], y1);
    }
    float yp = y0 + y1;
#pragma unroll
    for (int o = LPC / 2; o > 0; o >>= 1) yp += __shfl_xor_sync(0xffffffffu, yp, o);
    if (!live) return;
    float *hp = p.state + (b * p.dim + d) * N + n0;
    if (v32) {
      asm volatile("st.global.cs.v8.f32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"l"(hp), "f"(h[0]), "f"(h[1]),
                   "f"(h[2]), "f"(h[3]), "f"(h[4]), "f"(h[5]), "f"(h[6]), "f"(h[7])
                   : "memory");
    } else {
#pragma unroll
      for (int q = 0; q < S / 4; ++q)
        __stcs(reinterpret_cast<float4 *>(hp + 4 * q), make_float4(h[4 * q], h[4 * q + 1], h[4 * q + 2], h[4 * q + 3]));
    }
    if (j == 0) {
      float y = yp + Dd * r.u;
      if (p.z) y *= silu_fast(r.z);
      IO<T>::store1(static_cast<T *>(p.y), b * p.dim + d, y);
    }
  };

  // rows kb, kb + bps, ... through the two buffers; the trip count is the
  // block's own, so every lane of a warp takes part in each row's shuffles
  int64_t b = kb;
  if (b >= p.batch) return;
  StepRow<S> r0, r1;
  load(r0, b);
  for (;;) {
    const int64_t b1 = b + bps, b2 = b1 + bps;
    if (b1 < p.batch) load(r1, b1);
    prefetch(b2);
    run(r0, b);
    if (b1 >= p.batch) break;
    if (b2 < p.batch) load(r0, b2);
    prefetch(b2 + bps);
    run(r1, b1);
    if (b2 >= p.batch) break;
    b = b2;
  }
}

// Resident blocks of k_step_rows<T, S, LPC> on the current device (SMs x
// blocks per SM).  Both are properties of the kernel and the device model, so
// they are looked up once per device ordinal: a decode step is short enough
// that three runtime queries per call showed in its host time.  Failures are
// not cached.
template <typename T, int S, int LPC>
static cudaError_t step_rows_slots(int &slots) {
  constexpr int kDevs = 64;
  static std::atomic<int> cache[kDevs];
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev >= 0 && dev < kDevs && (slots = cache[dev].load(std::memory_order_relaxed)) > 0) return cudaSuccess;
  int sms = 0, occ = 0;
  if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
  if ((e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, k_step_rows<T, S, LPC>, kStepThreads, 0)) !=
      cudaSuccess)
    return e;
  slots = std::max(sms, 1) * std::max(occ, 1);
  if (dev >= 0 && dev < kDevs) cache[dev].store(slots, std::memory_order_relaxed);
  return cudaSuccess;
}

// grid: slices x bps blocks, block kb of a slice taking rows kb, kb + bps, ...
template <typename T, int S, int LPC>
static cudaError_t launch_step_rows(const StepParams &p, cudaStream_t s) {
  const int64_t slices = (p.dim * LPC + kStepThreads - 1) / kStepThreads;
  int slots = 0;
  const cudaError_t e = step_rows_slots<T, S, LPC>(slots);
  if (e != cudaSuccess) return e;
  const int64_t bps = std::max<int64_t>(1, std::min<int64_t>(p.batch, slots / slices));
  if (slices * bps > 0x7fffffff) return launch_step_k<T, S, LPC>(p, s);
  k_step_rows<T, S, LPC><<<(unsigned)(slices * bps), kStepThreads, 0, s>>>(p, (int)bps);
  return cudaGetLastError();
}

template <typename T>
static cudaError_t launch_step_t(const StepParams &p, cudaStream_t s) {
  const int N = p.N;
  if (p.vec && N % 8 == 0) {  // whole 8-state groups: the row-batched vector path
    if (N == 8) return launch_step_rows<T, 8, 1>(p, s);
    if (N == 16) return launch_step_rows<T, 8, 2>(p, s);
    if (N == 32) return launch_step_rows<T, 8, 4>(p, s);
    if (N == 64) return launch_step_rows<T, 8, 8>(p, s);
  }
  if (N <= 4) return launch_step_k<T, 4, 1>(p, s);
  if (N <= 8) return launch_step_k<T, 8, 1>(p, s);
  if (N <= 16) return launch_step_k<T, 8, 2>(p, s);
  if (N <= 32) return launch_step_k<T, 8, 4>(p, s);
  return launch_step_k<T, 8, 8>(p, s);
}

cudaError_t launch_step(int io_dtype, const StepParams &p, cudaStream_t s) {
  return io_dtype == 1 ? launch_step_t<uint16_t>(p, s) : launch_step_t<float>(p, s);
}

}  // namespace ssm
