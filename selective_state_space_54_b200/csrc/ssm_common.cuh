// Internal definitions shared by the forward and backward kernels and the
// C-ABI layer of libssmscan.so.  Not part of the public interface.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace ssm {

// ---- work decomposition ----------------------------------------------------
// A warp owns a group of 32/LPC channels of one batch element (LPC = lanes
// per channel, 2 or 4).  Lane l handles channel c = l / LPC and, of that
// channel's dstate states, the slice n in [j*S, j*S + S) with j = l % LPC and
// S = NP / LPC (NP = dstate padded up to a power of two >= 4).  Time is
// processed in chunks of kT steps; within a chunk each lane walks the
// recurrence sequentially, so every (t, n) element costs one exp2 and four
// fp32 ops and nothing of size (L, N) is stored.
constexpr int kT = 32;           // time steps per chunk
constexpr int kWarps = 4;        // warps per CTA
constexpr int kThreads = kWarps * 32;
constexpr int kRowPad = 4;       // smem row padding (floats) against bank conflicts
constexpr float kLog2e = 1.4426950408889634f;

// Saved-state layout shared by the forward (writer) and the backward (reader):
// the state entering every kCkptSteps-step chunk, laid out
// [batch][channel group of kCkptChannels][chunk][kCkptChannels][NP] fp32, with
// the channel count padded to a multiple of kCkptPad (see ckpt_groups).
constexpr int kCkptSteps = 8;
constexpr int kCkptChannels = 16;
constexpr int kCkptPad = 64;
__host__ __device__ __forceinline__ int64_t ckpt_groups(int64_t dim) {
  return (dim + kCkptPad - 1) / kCkptPad * (kCkptPad / kCkptChannels);
}
__host__ __device__ __forceinline__ int64_t ckpt_chunks(int64_t L) {
  return (L + kCkptSteps - 1) / kCkptSteps;
}
// Offset (in floats) of the saved state of channel d of batch b entering chunk k.
__host__ __device__ __forceinline__ int64_t ckpt_offset(int64_t b, int64_t d, int64_t k, int64_t dim,
                                                        int64_t L, int NP) {
  return (((b * ckpt_groups(dim) + d / kCkptChannels) * ckpt_chunks(L) + k) * kCkptChannels +
          d % kCkptChannels) * NP;
}

// Workspace header: byte 0 holds the device error word.
constexpr size_t kHeaderBytes = 256;
constexpr unsigned kErrWaitTimeout = 1u;

// Upper bound of one inter-warp wait in the look-back schedule, in ns of the
// GPU global timer.  The wait is only ever reached after the producer warp's
// first item, so in practice it never spins.
constexpr unsigned long long kWaitLimitNs = 2000000000ull;

struct FwdParams {
  const void *u, *delta, *z, *B, *C;
  const float *A, *D, *bias, *h0;
  void *y;
  float *last_state;
  int64_t batch, dim, L;
  int N;
  int softplus;
  int zoh;      // exact zero-order-hold input term instead of Euler
  int tok;      // u/delta/z/y laid out [batch][L][dim] (bf16, warp-specialised path)
  int io_vec;   // u/delta/z/y rows 16-byte aligned: vector loads
  int bc_vec;   // B/C chunk blocks 16-byte aligned and N == NP
  int64_t gpb;        // channel groups per batch element
  int64_t n_groups;   // batch * gpb
  int64_t n_chunks;   // ceil(L / kT)
  // look-back schedule
  int64_t n_workers;  // warps
  float *carry;       // [n_workers][32/LPC][NP]
  unsigned *flags;    // [n_workers]
  unsigned *err;      // workspace header
  unsigned long long wait_limit_ns;
  // split-L schedule
  int64_t n_segs, seg_chunks;
  // saved states for the backward (nullable): the state entering every
  // kCkptSteps-step chunk, at ckpt_offset(b, d, chunk, dim, L, NP)
  float *ckpt_out;
  // B and C as fp32 [batch][L][NP] (warp-specialised schedule; k_widen_bc)
  const float *Bf, *Cf;
  float *seg_h;       // [n_groups * n_segs][32/LPC][NP] segment end state from zero
  float *seg_dsum;    // [n_groups * n_segs][32/LPC]     sum of Delta over the segment
  float *seg_carry;   // [n_groups * n_segs][32/LPC][NP] state entering the segment
};

// Single-step (decode) parameters (ssm_step.cu).
struct StepParams {
  const void *u, *delta, *z, *B, *C;   // u/delta/z [batch][dim], B/C [batch][N], io dtype
  const float *A, *D, *bias;
  float *state;                        // [batch][dim][N] fp32, read and written in place
  void *y;                             // [batch][dim] io dtype
  int64_t batch, dim;
  int N;
  int softplus;
  int zoh;                             // exact zero-order-hold input term instead of Euler
  int vec;                             // N % 4 == 0, state/A 16-byte and B/C 4-element aligned
};

// Causal depthwise conv1d parameters (ssm_conv.cu).
struct ConvParams {
  const void *x;                       // [batch][dim][L] io dtype
  const float *w, *bias;               // [dim][K], [dim]
  const float *s0;                     // [batch][dim][K-1] inputs before t = 0, nullable
  void *out;                           // [batch][dim][L] io dtype
  float *s1;                           // [batch][dim][K-1] last K-1 inputs, nullable
  int64_t batch, dim, L;
  int K;
  int silu;
  int vec;                             // 2: 32-byte rows and buffers, 1: 16-byte, 0: neither
};

// Causal depthwise conv1d backward parameters (ssm_conv.cu).
struct ConvBwdParams {
  const void *x, *dout;                // [batch][dim][L] io dtype
  const float *w, *bias, *s0;          // [dim][K], [dim] nullable, [batch][dim][K-1] nullable
  void *dx;                            // [batch][dim][L] io dtype
  float *dw, *dbias, *ds0;             // [dim][K] (zeroed), [dim] (zeroed) nullable, [batch][dim][K-1] nullable
  int64_t batch, dim, L;
  int K;
  int silu;
  int vec;                             // 16-byte aligned rows
};

// Backward parameters (ssm_bwd.cu, ssm_bwd16.cu).
struct BwdParams {
  const void *u, *delta, *z, *B, *C, *dout;
  const float *A, *D, *bias, *h0;
  void *du, *ddelta, *dz;
  float *dA, *dD, *dbias, *dh0;     // final gradients (k_bwd_reduce)
  float *ckpt;                      // saved states, at ckpt_offset(...)
  int ckpt_given;                   // ckpt holds states saved by the forward: skip the checkpoint pass
  void *dB, *dC;                    // [batch][L][N] io dtype (k_bwd_reduce)
  // per-block partial sums, added in a fixed order by k_bwd_reduce
  float *dBC_part;                  // [channel block][batch][L][2 * NP] (dB states, then dC states)
  float *dA_part;                   // [batch][dim][N]
  float *dD_part, *dbias_part;      // [batch][dim] (nullable with D / delta_bias)
  int64_t n_blocks;                 // channel blocks of dBC_part
  int64_t batch, dim, L;
  int N;
  int softplus;
  int zoh;                          // exact zero-order-hold input term (general kernel)
  int tok;                          // u/delta/z/dout/du/ddelta/dz laid out [batch][L][dim] (k_bwd16)
  int io_vec;
  int bc_vec;                       // B/C rows 16-byte aligned and N == NP
  int64_t cpb;                      // CTAs per batch element
  int64_t K;                        // backward chunks
};

// ---- io helpers ---------------------------------------------------------------
// bf16 values travel as raw 16-bit patterns; widening is a shift.
__device__ __forceinline__ float bf16_lo(uint32_t v) { return __uint_as_float(v << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t v) { return __uint_as_float(v & 0xffff0000u); }
__device__ __forceinline__ float bf16_to_f(uint16_t v) { return __uint_as_float((uint32_t)v << 16); }

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 p = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t *>(&p);
}

template <typename T> struct IO;

template <> struct IO<uint16_t> {
  static constexpr int kBytes = 2;
  __device__ __forceinline__ static float get(const uint16_t *p, int64_t i) { return bf16_to_f(p[i]); }
  // 8 consecutive values row[t..t+8), zeros beyond L.
  __device__ __forceinline__ static void load8(const uint16_t *row, int64_t t, int64_t L,
                                               bool vec, float (&o)[8]) {
    if (vec && t + 8 <= L) {
      const uint4 v = __ldg(reinterpret_cast<const uint4 *>(row + t));
      o[0] = bf16_lo(v.x); o[1] = bf16_hi(v.x); o[2] = bf16_lo(v.y); o[3] = bf16_hi(v.y);
      o[4] = bf16_lo(v.z); o[5] = bf16_hi(v.z); o[6] = bf16_lo(v.w); o[7] = bf16_hi(v.w);
    } else {
#pragma unroll
      for (int i = 0; i < 8; ++i) o[i] = (t + i < L) ? bf16_to_f(row[t + i]) : 0.f;
    }
  }
  __device__ __forceinline__ static void store8(uint16_t *row, int64_t t, int64_t L, bool vec,
                                                const float (&v)[8]) {
    if (vec && t + 8 <= L) {
      uint4 o;
      o.x = pack_bf16x2(v[0], v[1]); o.y = pack_bf16x2(v[2], v[3]);
      o.z = pack_bf16x2(v[4], v[5]); o.w = pack_bf16x2(v[6], v[7]);
      *reinterpret_cast<uint4 *>(row + t) = o;
    } else {
#pragma unroll
      for (int i = 0; i < 8; ++i)
        if (t + i < L) {
          __nv_bfloat16 b = __float2bfloat16_rn(v[i]);
          row[t + i] = *reinterpret_cast<uint16_t *>(&b);
        }
    }
  }
  // 4 consecutive values row[t..t+4), those at or past L dropped
  __device__ __forceinline__ static void store4(uint16_t *row, int64_t t, int64_t L, bool vec,
                                                const float (&v)[4]) {
    if (vec && t + 4 <= L) {
      *reinterpret_cast<uint2 *>(row + t) = make_uint2(pack_bf16x2(v[0], v[1]), pack_bf16x2(v[2], v[3]));
    } else {
#pragma unroll
      for (int i = 0; i < 4; ++i)
        if (t + i < L) store1(row, t + i, v[i]);
    }
  }
  __device__ __forceinline__ static void store1(uint16_t *p, int64_t i, float v) {
    __nv_bfloat16 b = __float2bfloat16_rn(v);
    p[i] = *reinterpret_cast<uint16_t *>(&b);
  }
};

template <> struct IO<float> {
  static constexpr int kBytes = 4;
  __device__ __forceinline__ static float get(const float *p, int64_t i) { return p[i]; }
  __device__ __forceinline__ static void load8(const float *row, int64_t t, int64_t L, bool vec,
                                               float (&o)[8]) {
    if (vec && t + 8 <= L) {
      const float4 a = __ldg(reinterpret_cast<const float4 *>(row + t));
      const float4 b = __ldg(reinterpret_cast<const float4 *>(row + t + 4));
      o[0] = a.x; o[1] = a.y; o[2] = a.z; o[3] = a.w; o[4] = b.x; o[5] = b.y; o[6] = b.z; o[7] = b.w;
    } else {
#pragma unroll
      for (int i = 0; i < 8; ++i) o[i] = (t + i < L) ? row[t + i] : 0.f;
    }
  }
  __device__ __forceinline__ static void store8(float *row, int64_t t, int64_t L, bool vec,
                                                const float (&v)[8]) {
    if (vec && t + 8 <= L) {
      *reinterpret_cast<float4 *>(row + t) = make_float4(v[0], v[1], v[2], v[3]);
      *reinterpret_cast<float4 *>(row + t + 4) = make_float4(v[4], v[5], v[6], v[7]);
    } else {
#pragma unroll
      for (int i = 0; i < 8; ++i)
        if (t + i < L) row[t + i] = v[i];
    }
  }
  __device__ __forceinline__ static void store4(float *row, int64_t t, int64_t L, bool vec,
                                                const float (&v)[4]) {
    if (vec && t + 4 <= L) {
      *reinterpret_cast<float4 *>(row + t) = make_float4(v[0], v[1], v[2], v[3]);
    } else {
#pragma unroll
      for (int i = 0; i < 4; ++i)
        if (t + i < L) row[t + i] = v[i];
    }
  }
  __device__ __forceinline__ static void store1(float *p, int64_t i, float v) { p[i] = v; }
};

// ---- packed fp32 pairs (sm_100a f32x2 arithmetic) -----------------------------
// A pair of fp32 values in one 64-bit register pair; the packed add, multiply
// and fused multiply-add issue once for both halves.
typedef unsigned long long f2;

__device__ __forceinline__ f2 pack2(float lo, float hi) {
  f2 r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
__device__ __forceinline__ void unpack2(f2 v, float &lo, float &hi) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ f2 fma2(f2 a, f2 b, f2 c) {
  f2 d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
__device__ __forceinline__ f2 add2(f2 a, f2 b) {
  f2 d;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ f2 mul2(f2 a, f2 b) {
  f2 d;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ f2 splat2(float v) { return pack2(v, v); }

// ---- math helpers -------------------------------------------------------------
// 2^x on the special-function unit (flush-to-zero; 2^-big == 0 exactly).
__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// softplus(s) = log(1 + e^s); s itself above 20 (the difference is < 2e-9 relative).
__device__ __forceinline__ float softplus_f(float s) { return s > 20.f ? s : log1pf(__expf(s)); }

__device__ __forceinline__ float sigmoid_f(float x) { return __fdividef(1.f, 1.f + __expf(-x)); }


__device__ __forceinline__ unsigned long long global_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// ---- softplus without a second special-function op --------------------------
// softplus(s) = max(s, 0) + log1p(x),  x = exp(-|s|) in (0, 1].
// log1p(x) = x * p(x), p a degree-8 polynomial interpolating log1p(x)/x at the
// Chebyshev nodes of [0, 1] (max relative error 2.3e-7 in fp32 evaluation,
// fitted for this library).
__device__ __forceinline__ float softplus_fast(float s) {
  const float x = ex2(-fabsf(s) * kLog2e);
  float p = 5.126102362e-03f;
  p = fmaf(p, x, -2.907406539e-02f);
  p = fmaf(p, x, 7.751608640e-02f);
  p = fmaf(p, x, -1.360224783e-01f);
  p = fmaf(p, x, 1.907688081e-01f);
  p = fmaf(p, x, -2.483539879e-01f);
  p = fmaf(p, x, 3.331812024e-01f);
  p = fmaf(p, x, -4.999944568e-01f);
  p = fmaf(p, x, 9.999999404e-01f);
  return fmaf(x, p, fmaxf(s, 0.f));
}

__device__ __forceinline__ float rcp_approx(float x) {
  float y;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// SiLU(z) = z / (1 + e^-z)
__device__ __forceinline__ float silu_fast(float z) {
  return z * rcp_approx(1.f + ex2(-z * kLog2e));
}

// Exact zero-order hold for diagonal A: Bbar_n / (Delta B_n) = (e^x - 1) / x
// with x = Delta A_n, given x2 = x / ln 2 (the ex2 argument) and a = 2^x2.
// For |x| < 1/2 the Taylor series sum_k x^k / (k+1)!, k <= 7 (remainder below
// 1.1e-8); otherwise (a - 1) / x, where a - 1 loses nothing (|a - 1| > 0.39).
// x = 0 (A_n = 0 or Delta = 0) gives 1: the Euler term, the exact limit.
constexpr float kLn2 = 0.6931471805599453f;
__device__ __forceinline__ float expm1_over_x(float x2, float a) {
  const float x = x2 * kLn2;
  float q = 2.48015873015873e-05f;         // 1/8!
  q = fmaf(q, x, 1.984126984126984e-04f);  // 1/7!
  q = fmaf(q, x, 1.388888888888889e-03f);  // 1/6!
  q = fmaf(q, x, 8.333333333333333e-03f);  // 1/5!
  q = fmaf(q, x, 4.166666666666667e-02f);  // 1/4!
  q = fmaf(q, x, 1.666666666666667e-01f);  // 1/3!
  q = fmaf(q, x, 0.5f);                    // 1/2!
  q = fmaf(q, x, 1.f);
  return fabsf(x) < 0.5f ? q : (a - 1.f) * rcp_approx(x);
}

// Exact zero-order hold, on pairs, with y = x / ln 2 the ex2 argument
// (x = Delta A_n), a = e^x and rA = 1 / A_n:
//   W = Delta (e^x - 1)/x     (the input term is u W B_n)
//   Y = Delta^2 psi(x), psi(x) = (x e^x - (e^x - 1)) / x^2   (its A_n derivative is u Y B_n).
// Above a threshold in |x| Delta cancels: W = (e^x - 1) / A_n and
// Y = (Delta e^x - W) / A_n, with no reciprocal per element (rA is per state);
// below it the Taylor series, sum_k x^k/(k+1)! to x^5 for W (|x| < 1/4,
// remainder below 5e-8) and sum_m x^m (m+1)/(m+2)! to x^7 for psi
// (|x| < 1/2, remainder below 1e-8), with the ln2^k of y folded into the
// coefficients.  Where e^x - 1 or Delta e^x - W cancel, the series is used.
constexpr float kZohW1 = 3.465735903e-01f, kZohW2 = 8.007550232e-02f, kZohW3 = 1.387602717e-02f,
                kZohW4 = 1.923625822e-03f, kZohW5 = 2.222259691e-04f;  // ln2^k / (k+1)!
constexpr float kZohWSmall = 3.606737602e-01f;                           // 0.25 / ln2
constexpr float kZohP0 = 5.000000000e-01f, kZohP1 = 2.310490602e-01f, kZohP2 = 6.005662674e-02f,
                kZohP3 = 1.110082173e-02f, kZohP4 = 1.603021518e-03f, kZohP5 = 1.904794021e-04f,
                kZohP6 = 1.925441299e-05f, kZohP7 = 1.694748200e-06f;  // ln2^m (m+1) / (m+2)!
constexpr float kZohPSmall = 7.213475204e-01f;                           // 0.5 / ln2
__device__ __forceinline__ f2 zoh_select(f2 y, f2 small, f2 big, float lim) {
  float y0, y1, s0, s1, b0, b1;
  unpack2(y, y0, y1);
  unpack2(small, s0, s1);
  unpack2(big, b0, b1);
  return pack2(fabsf(y0) < lim ? s0 : b0, fabsf(y1) < lim ? s1 : b1);
}
__device__ __forceinline__ f2 zoh_w(f2 y, f2 a, f2 dl2, f2 rA) {
  const f2 big = mul2(add2(a, splat2(-1.f)), rA);
  f2 q = fma2(splat2(kZohW5), y, splat2(kZohW4));
  q = fma2(q, y, splat2(kZohW3));
  q = fma2(q, y, splat2(kZohW2));
  q = fma2(q, y, splat2(kZohW1));
  q = fma2(q, y, splat2(1.f));
  return zoh_select(y, mul2(q, dl2), big, kZohWSmall);
}
__device__ __forceinline__ f2 zoh_y(f2 y, f2 a, f2 w, f2 dl2, f2 rA) {
  const f2 big = mul2(fma2(w, splat2(-1.f), mul2(dl2, a)), rA);
  f2 q = fma2(splat2(kZohP7), y, splat2(kZohP6));
  q = fma2(q, y, splat2(kZohP5));
  q = fma2(q, y, splat2(kZohP4));
  q = fma2(q, y, splat2(kZohP3));
  q = fma2(q, y, splat2(kZohP2));
  q = fma2(q, y, splat2(kZohP1));
  q = fma2(q, y, splat2(kZohP0));
  return zoh_select(y, mul2(q, mul2(dl2, dl2)), big, kZohPSmall);
}

__device__ __forceinline__ unsigned ld_acquire(const unsigned *p) {
  unsigned v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

__device__ __forceinline__ void st_release(unsigned *p, unsigned v) {
  asm volatile("st.release.gpu.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

// Lane 0 waits until *flag != 0 or limit_ns passed; the result is broadcast.
// On give-up the error word gets kErrWaitTimeout.  Never traps, never spins
// without bound.
__device__ __forceinline__ bool warp_wait_flag(const unsigned *flag, unsigned *err,
                                               unsigned long long limit_ns) {
  unsigned ok = 0;
  if ((threadIdx.x & 31) == 0) {
    const unsigned long long t0 = global_ns();
    while (true) {
      if (ld_acquire(flag) != 0u) { ok = 1; break; }
      if (global_ns() - t0 > limit_ns) break;
      __nanosleep(256);
    }
    if (!ok) atomicOr(err, kErrWaitTimeout);
  }
  ok = __shfl_sync(0xffffffffu, ok, 0);
  __threadfence();
  return ok != 0;
}

// ---- launchers (defined in ssm_fwd.cu / ssm_bwd.cu) ----------------------------
int fwd_np_for(int64_t N);
cudaError_t fwd_occupancy(int io_dtype, int NP, int LPC, int zoh, int *ctas_per_sm);
cudaError_t fwd_segment_occupancy(int io_dtype, int NP, int LPC, int emit, int *ctas_per_sm);
cudaError_t launch_fwd_lookback(int io_dtype, int NP, int LPC, const FwdParams &p, cudaStream_t s);
cudaError_t launch_fwd_splitl(int io_dtype, int NP, int LPC, const FwdParams &p, cudaStream_t s);
int fwd_ws_chunk();
int fwd_ws_pairs();
cudaError_t fwd_ws_occupancy(int io_dtype, int NP, int LPC, int *ctas_per_sm);
cudaError_t launch_fwd_ws(int io_dtype, int NP, int LPC, const FwdParams &p, cudaStream_t s);
cudaError_t launch_widen_bc(int io_dtype, const void *B, const void *C, float *Bf, float *Cf, int64_t rows,
                            int N, int NP, cudaStream_t s);
size_t bwd_ckpt_floats(int64_t batch, int64_t dim, int64_t L, int NP);
int64_t bwd_blocks(int64_t dim, int NP, int zoh);
cudaError_t launch_bwd(int io_dtype, int NP, BwdParams &p, cudaStream_t s);
cudaError_t launch_step(int io_dtype, const StepParams &p, cudaStream_t s);
cudaError_t launch_conv(int io_dtype, const ConvParams &p, cudaStream_t s);
cudaError_t launch_conv_bwd(int io_dtype, const ConvBwdParams &p, cudaStream_t s);
cudaError_t launch_wait_timeout_probe(unsigned *flag, unsigned *err, unsigned long long limit_ns,
                                      cudaStream_t s);

}  // namespace ssm
