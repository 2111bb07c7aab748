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
// 8 states.  On the vector path (N % 8 == 0, 16-byte rows) a block takes
// kRows batch rows of its channels and loads all their state slices into
// registers before computing the first, one 32-byte load per row where the
// state is 32-byte aligned (k_step_rows); other shapes take one row per block
// and plain masked loads (k_step).  The state is read and written with
// streaming (evict-first) accesses: it is touched once per token.  A, B and C
// are re-read across batch elements or channels and are served from L2/L1.
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

// ---- vector path: several batch rows per block ------------------------------
// A block owns kStepThreads / LPC channels and kRows batch rows.  Every lane
// first loads its S states of all kRows rows into registers (one 32-byte load
// per row; two 16-byte ones when the state is only 16-byte aligned), loads A,
// D and the bias of its channel once for all rows, and then walks the rows.
// kRows * 32 bytes of state per thread are in flight before the first row
// computes.  Held to 80 registers for 3 blocks (24 warps) per SM: on B200 at
// the Mamba-2.8B decode shape (batch 128) 20.8 us per step, against 22.8 us
// at 2 blocks per SM (128 registers), 30.0 us at 4 (64 registers, spilling)
// and 25.0 us for the same rows fed through a cp.async ring in shared memory.
// 2, 3, 5 or 6 rows per block measured slower than 4.
constexpr int kRows = 4;

template <typename T, int S, int LPC>
__global__ void __launch_bounds__(kStepThreads, 3) k_step_rows(StepParams p) {
  static_assert(S == 8, "a lane's 8 states are one 32-byte access");
  const int tid = threadIdx.x;
  const int64_t slot = (int64_t)blockIdx.x * kStepThreads + tid;
  const int j = (int)(slot % LPC);
  int64_t d = slot / LPC;
  const bool live = d < p.dim;
  if (!live) d = p.dim - 1;  // lanes past the row compute on its last channel, store nothing
  const int N = p.N, n0 = S * j;
  const int64_t b0 = (int64_t)blockIdx.y * kRows;
  const int rows = (int)(p.batch - b0 < kRows ? p.batch - b0 : kRows);
  // every row's state slice into registers up front (rows past the batch read row b0 again)
  const bool v32 = (reinterpret_cast<uintptr_t>(p.state) & 31) == 0;
  float hreg[kRows][S];
#pragma unroll
  for (int r = 0; r < kRows; ++r) {
    const int64_t b = b0 + (r < rows ? r : 0);
    const float *hp = p.state + (b * p.dim + d) * N + n0;
    if (v32) {
      asm volatile("ld.global.cs.v8.f32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
                   : "=f"(hreg[r][0]), "=f"(hreg[r][1]), "=f"(hreg[r][2]), "=f"(hreg[r][3]),
                     "=f"(hreg[r][4]), "=f"(hreg[r][5]), "=f"(hreg[r][6]), "=f"(hreg[r][7])
                   : "l"(hp));
    } else {
      const float4 h0 = __ldcs(reinterpret_cast<const float4 *>(hp));
      const float4 h1 = __ldcs(reinterpret_cast<const float4 *>(hp + 4));
      hreg[r][0] = h0.x; hreg[r][1] = h0.y; hreg[r][2] = h0.z; hreg[r][3] = h0.w;
      hreg[r][4] = h1.x; hreg[r][5] = h1.y; hreg[r][6] = h1.z; hreg[r][7] = h1.w;
    }
  }
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
  // the token inputs of every row
  float uu[kRows], ss[kRows], zz[kRows];
#pragma unroll
  for (int r = 0; r < kRows; ++r) {
    const int64_t ch = (b0 + (r < rows ? r : 0)) * p.dim + d;
    uu[r] = IO<T>::get(static_cast<const T *>(p.u), ch);
    ss[r] = IO<T>::get(static_cast<const T *>(p.delta), ch) + bias;
    zz[r] = p.z ? IO<T>::get(static_cast<const T *>(p.z), ch) : 0.f;
  }
#pragma unroll
  for (int r = 0; r < kRows; ++r) {
    const int64_t b = b0 + (r < rows ? r : 0);
    float Bv[S], Cv[S];
    load_io<S>(static_cast<const T *>(p.B) + b * N, true, n0, N, Bv);
    load_io<S>(static_cast<const T *>(p.C) + b * N, true, n0, N, Cv);
    const float dl = p.softplus ? softplus_fast(ss[r]) : ss[r];
    const float du = dl * uu[r];
    float h[S];
#pragma unroll
    for (int i = 0; i < S; ++i) h[i] = hreg[r][i];
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
    if (live && r < rows) {
      float *hp = p.state + (b * p.dim + d) * N + n0;
      if (v32) {
        asm volatile("st.global.cs.v8.f32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"l"(hp), "f"(h[0]), "f"(h[1]),
                     "f"(h[2]), "f"(h[3]), "f"(h[4]), "f"(h[5]), "f"(h[6]), "f"(h[7])
                     : "memory");
      } else {
#pragma unroll
        for (int q = 0; q < S / 4; ++q)
          __stcs(reinterpret_cast<float4 *>(hp + 4 * q),
                 make_float4(h[4 * q], h[4 * q + 1], h[4 * q + 2], h[4 * q + 3]));
      }
      if (j == 0) {
        float y = yp + Dd * uu[r];
        if (p.z) y *= silu_fast(zz[r]);
        IO<T>::store1(static_cast<T *>(p.y), b * p.dim + d, y);
      }
    }
  }
}

template <typename T, int S, int LPC>
static cudaError_t launch_step_rows(const StepParams &p, cudaStream_t s) {
  const int64_t slots = p.dim * LPC;
  const int64_t bx = (slots + kStepThreads - 1) / kStepThreads;
  const int64_t by = (p.batch + kRows - 1) / kRows;
  if (bx > 0x7fffffff || by > 65535) return launch_step_k<T, S, LPC>(p, s);
  k_step_rows<T, S, LPC><<<dim3((unsigned)bx, (unsigned)by), kStepThreads, 0, s>>>(p);
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
