// Causal depthwise 1-D convolution along the sequence, with optional SiLU,
// for sm_100a: the convolution layer the Mamba block applies to x_proj
// before the SSM, followed by its SiLU activation ("O que e um modelo
// Mamba?", ibm.com, the walk-through of the Mamba block: the convolution
// extracts local patterns between neighbouring tokens, its output goes
// through SiLU and becomes the SSM's input).  Per channel d, width K:
//   out_t = act(bias[d] + sum_{k<K} w[d][k] * x_{t-K+1+k}),
// with x_t for t < 0 taken from the caller's initial state (zeros if none).
//
// Design (B200): 2 bytes in and 2 out per (b, d, t) in bf16, a few FMAs:
// bound by HBM.  A warp takes 2048 consecutive steps of one (b, d) row in 8
// passes; a lane takes 8 steps per pass with one 16-byte load and store,
// all 8 loads issued before the first pass computes.  The K-1 steps before a
// lane's chunk come from neighbouring lanes by shuffles, so every input byte
// is read once.  Input and output are streamed with evict-first hints.
#include "ssm_common.cuh"

namespace ssm {

constexpr int kConvThreads = 256;

constexpr int kConvW = 8;                  // steps per lane and pass
// Passes per warp, all loads issued first: 8 in the forward, i.e. 8 16-byte
// loads in flight per lane, with the bf16 kernel held to 64 registers for 4
// CTAs (32 warps) per SM.  Measured on B200 at the Mamba-2.8B shape (bf16,
// width 4): 0.123 ms, against 0.133 ms at 3 CTAs per SM, 0.132 ms with 7
// passes and 0.140 ms with 4; 9, 10, 12 or 16 passes cost registers (fewer
// resident CTAs) and leave a ragged last segment (0.148-0.169 ms).  4 in the
// backward, whose two input streams and register cap leave no room for more
// (8 passes spill or halve the resident CTAs: 0.280 against 0.261 ms).
constexpr int kConvR = 8;
constexpr int kConvSeg = 32 * kConvW * kConvR;  // steps per forward warp
constexpr int kConvBR = 4;
constexpr int kConvBSeg = 32 * kConvW * kConvBR;  // steps per backward warp

// (row, segment, channel) of this warp; 32-bit divisions when the grid's
// warp count fits (the launcher checks), 64-bit otherwise
struct ConvWarp {
  int64_t row, seg, d;
  bool live;
  __device__ __forceinline__ ConvWarp(int64_t segs, int64_t rows, int64_t dim, bool narrow) {
    if (narrow) {
      const unsigned w = (blockIdx.x * (unsigned)kConvThreads + threadIdx.x) >> 5;
      const unsigned r = w / (unsigned)segs;
      live = r < (unsigned)rows;
      row = r;
      seg = w - r * (unsigned)segs;
      d = r % (unsigned)dim;
    } else {
      const int64_t w = ((int64_t)blockIdx.x * kConvThreads + threadIdx.x) >> 5;
      row = w / segs;
      live = row < rows;
      seg = w - row * segs;
      d = row % dim;
    }
  }
};

// raw io vector of 8 values, kept packed until used
template <typename T> struct Raw8;
template <> struct Raw8<uint16_t> {
  uint4 v;
  __device__ __forceinline__ void load(const uint16_t *row, int64_t t, int64_t L, bool vec) {
    if (vec && t + 8 <= L) {
      v = __ldcs(reinterpret_cast<const uint4 *>(row + t));
    } else {
      uint32_t w[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const uint32_t lo = (t + 2 * i < L) ? row[t + 2 * i] : 0u;
        const uint32_t hi = (t + 2 * i + 1 < L) ? row[t + 2 * i + 1] : 0u;
        w[i] = lo | (hi << 16);
      }
      v = make_uint4(w[0], w[1], w[2], w[3]);
    }
  }
  __device__ __forceinline__ void unpack(float (&o)[8]) const {
    o[0] = bf16_lo(v.x); o[1] = bf16_hi(v.x); o[2] = bf16_lo(v.y); o[3] = bf16_hi(v.y);
    o[4] = bf16_lo(v.z); o[5] = bf16_hi(v.z); o[6] = bf16_lo(v.w); o[7] = bf16_hi(v.w);
  }
};
template <> struct Raw8<float> {
  float4 a, b;
  __device__ __forceinline__ void load(const float *row, int64_t t, int64_t L, bool vec) {
    if (vec && t + 8 <= L) {
      a = __ldcs(reinterpret_cast<const float4 *>(row + t));
      b = __ldcs(reinterpret_cast<const float4 *>(row + t + 4));
    } else {
      float o[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) o[i] = (t + i < L) ? row[t + i] : 0.f;
      a = make_float4(o[0], o[1], o[2], o[3]);
      b = make_float4(o[4], o[5], o[6], o[7]);
    }
  }
  __device__ __forceinline__ void unpack(float (&o)[8]) const {
    o[0] = a.x; o[1] = a.y; o[2] = a.z; o[3] = a.w; o[4] = b.x; o[5] = b.y; o[6] = b.z; o[7] = b.w;
  }
};

// A warp takes kConvSeg consecutive steps of one row in kConvR passes of 256;
// all passes' loads are issued before the first is used, so each lane keeps
// kConvR 16-byte loads in flight.  The K-1 steps before a lane's chunk come
// from the previous lane (shuffle up), or for lane 0 from lane 31 of the
// previous pass; only the warp's first pass reads them from memory.
// NARROW: the grid's thread count fits 32 bits (a separate instantiation:
// a run-time choice of the index width measured 5 % slower)
template <typename T, int K, bool NARROW>
__global__ void __launch_bounds__(kConvThreads, (sizeof(T) == 2 && K <= 4) ? 4 : 1) k_conv(ConvParams p) {
  const int lane = threadIdx.x & 31;
  const int64_t L = p.L;
  const ConvWarp cw((L + kConvSeg - 1) / kConvSeg, p.batch * p.dim, p.dim, NARROW);
  if (!cw.live) return;  // whole warps leave together
  const int64_t row = cw.row, seg = cw.seg, d = cw.d;
  const T *xr = static_cast<const T *>(p.x) + row * L;
  T *orow = static_cast<T *>(p.out) + row * L;
  const bool vec = p.vec != 0;
  Raw8<T> raw[kConvR];
#pragma unroll
  for (int r = 0; r < kConvR; ++r) raw[r].load(xr, seg * kConvSeg + r * 32 * kConvW + lane * kConvW, L, vec);
  float w[K];
#pragma unroll
  for (int k = 0; k < K; ++k) w[k] = p.w[d * K + k];
  const float bias = p.bias ? p.bias[d] : 0.f;
  float carry[K > 1 ? K - 1 : 1];  // the K-1 inputs before the pass, as lane 31 of the last pass saw them
#pragma unroll
  for (int r = 0; r < kConvR; ++r) {
    const int64_t t0 = seg * kConvSeg + r * 32 * kConvW + lane * kConvW;
    if (seg * kConvSeg + r * 32 * kConvW >= L) break;  // warp-uniform
    float v[kConvW];
    raw[r].unpack(v);
    float halo[K > 1 ? K - 1 : 1];
#pragma unroll
    for (int i = 0; i < K - 1; ++i) {
      const float up = __shfl_up_sync(0xffffffffu, v[kConvW - (K - 1) + i], 1);
      const float last = __shfl_sync(0xffffffffu, v[kConvW - (K - 1) + i], 31);
      if (lane > 0) {
        halo[i] = up;
      } else if (r > 0) {
        halo[i] = carry[i];
      } else {
        const int64_t t = t0 - (K - 1) + i;  // the warp's first pass: memory or the initial state
        halo[i] = t >= 0 ? IO<T>::get(xr, t) : (p.s0 ? p.s0[row * (K - 1) + (K - 1) + t] : 0.f);
      }
      carry[i] = last;
    }
    float o[kConvW];
#pragma unroll
    for (int i = 0; i < kConvW; ++i) {
      float acc = bias;
#pragma unroll
      for (int k = 0; k < K; ++k) {
        const int idx = i - (K - 1) + k;  // position in [halo | v]
        acc = fmaf(w[k], idx < 0 ? halo[idx + K - 1] : v[idx], acc);
      }
      o[i] = acc;
    }
    if (p.silu) {  // SiLU(a) = a / (1 + e^-a), on pairs
#pragma unroll
      for (int i = 0; i < kConvW; i += 2) {
        const f2 a2 = pack2(o[i], o[i + 1]);
        float e0, e1, d0, d1;
        unpack2(mul2(a2, pack2(-kLog2e, -kLog2e)), e0, e1);
        unpack2(add2(pack2(ex2(e0), ex2(e1)), pack2(1.f, 1.f)), d0, d1);
        unpack2(mul2(a2, pack2(rcp_approx(d0), rcp_approx(d1))), o[i], o[i + 1]);
      }
    }
    if (t0 < L) {
      if (vec && t0 + kConvW <= L) {
        if constexpr (sizeof(T) == 2) {
          uint4 q;
          q.x = pack_bf16x2(o[0], o[1]); q.y = pack_bf16x2(o[2], o[3]);
          q.z = pack_bf16x2(o[4], o[5]); q.w = pack_bf16x2(o[6], o[7]);
          __stcs(reinterpret_cast<uint4 *>(orow + t0), q);
        } else {
          __stcs(reinterpret_cast<float4 *>(orow + t0), make_float4(o[0], o[1], o[2], o[3]));
          __stcs(reinterpret_cast<float4 *>(orow + t0 + 4), make_float4(o[4], o[5], o[6], o[7]));
        }
      } else {
        IO<T>::store8(orow, t0, L, false, o);
      }
    }
    // final state: the last K-1 inputs of the row, written by the lane holding step L-1
    if (K > 1 && p.s1 && t0 <= L - 1 && L - 1 < t0 + kConvW) {
#pragma unroll
      for (int i = 0; i < K - 1; ++i) {
        const int idx = (int)(L - (K - 1) + i - t0);  // position in v, or in halo when negative
        float val = 0.f;                             // (idx >= -(K - 1) always holds here)
#pragma unroll
        for (int m = 0; m < kConvW; ++m)
          if (m == idx) val = v[m];
#pragma unroll
        for (int m = 0; m < K - 1; ++m)
          if (m - (K - 1) == idx) val = halo[m];
        p.s1[row * (K - 1) + i] = val;
      }
    }
  }
}

// ---- backward -------------------------------------------------------------
// Gradients of sum(dout * out): with a_t = bias + sum_k w_k x_{t-K+1+k} and
// out_t = act(a_t), da_t = dout_t act'(a_t); dx_s = sum_k w_k da_{s+K-1-k};
// dw_k = sum_{b,t} da_t x_{t-K+1+k}; dbias = sum_{b,t} da_t; the initial
// state's gradient is dx of the K-1 inputs before t = 0.  Same warp layout as
// the forward: a warp recomputes a and da pass by pass, accumulates its dw and
// dbias partials, and writes dx of the pass before once it has the next pass's
// first K-1 values of da (a shuffle from lane 0).  The warp's last pass takes
// them from the next segment, recomputed by lane 31 from memory.  A backward
// warp takes 4 passes (1024 steps).
template <typename T, int K>
__device__ __forceinline__ float conv_act_grad(float a, float g, bool silu) {
  if (!silu) return g;
  const float sg = rcp_approx(1.f + ex2(-a * kLog2e));
  return g * sg * fmaf(a, 1.f - sg, 1.f);
}

template <typename T, int K>
__global__ void __launch_bounds__(kConvThreads, (sizeof(T) == 2 && K <= 4) ? 4 : 1) k_conv_bwd(ConvBwdParams p) {
  const int lane = threadIdx.x & 31;
  const int64_t L = p.L;
  // 64-bit index math: the 32-bit form gained nothing here and its extra
  // registers spill under the 64-register cap
  const ConvWarp cw((L + kConvBSeg - 1) / kConvBSeg, p.batch * p.dim, p.dim, false);
  if (!cw.live) return;  // whole warps leave together
  const int64_t row = cw.row, seg = cw.seg, d = cw.d;
  const T *xr = static_cast<const T *>(p.x) + row * L;
  const T *gr = static_cast<const T *>(p.dout) + row * L;
  T *dxr = static_cast<T *>(p.dx) + row * L;
  const bool vec = p.vec != 0;
  const bool silu = p.silu != 0;
  Raw8<T> rx[kConvBR], rg[kConvBR];
#pragma unroll
  for (int r = 0; r < kConvBR; ++r) {
    const int64_t t0 = seg * kConvBSeg + r * 32 * kConvW + lane * kConvW;
    rx[r].load(xr, t0, L, vec);
    rg[r].load(gr, t0, L, vec);
  }
  float w[K];
#pragma unroll
  for (int k = 0; k < K; ++k) w[k] = p.w[d * K + k];
  const float bias = p.bias ? p.bias[d] : 0.f;
  // x_t for t < 0: the initial state, else zero
  auto x_before = [&](int64_t t) -> float {
    return p.s0 ? p.s0[row * (K - 1) + (K - 1) + t] : 0.f;
  };
  float dwp[K], dbp = 0.f;
#pragma unroll
  for (int k = 0; k < K; ++k) dwp[k] = 0.f;
  float carry[K > 1 ? K - 1 : 1];  // x before the pass, as lane 31 of the last pass saw it
  float da_prev[kConvW];           // da of the pass before, waiting for its dx
  int64_t t0_prev = 0;
  bool have_prev = false;
  // dx of one pass from its da and the next K-1 values of da after the lane's chunk
  auto emit_dx = [&](const float (&da)[kConvW], const float (&nxt)[K > 1 ? K - 1 : 1], int64_t t0) {
    float o[kConvW];
#pragma unroll
    for (int i = 0; i < kConvW; ++i) {
      float acc = 0.f;
#pragma unroll
      for (int k = 0; k < K; ++k) {
        const int idx = i + (K - 1) - k;  // position of da_{s+K-1-k} in [da | nxt]
        acc = fmaf(w[k], idx < kConvW ? da[idx] : nxt[idx - kConvW], acc);
      }
      o[i] = acc;
    }
    if (t0 < L) IO<T>::store8(dxr, t0, L, vec, o);
  };
#pragma unroll
  for (int r = 0; r < kConvBR; ++r) {
    const int64_t t0 = seg * kConvBSeg + r * 32 * kConvW + lane * kConvW;
    const bool live = seg * kConvBSeg + r * 32 * kConvW < L;  // warp-uniform
    float v[kConvW], gv[kConvW];
    rx[r].unpack(v);
    rg[r].unpack(gv);
    float halo[K > 1 ? K - 1 : 1];
#pragma unroll
    for (int i = 0; i < K - 1; ++i) {
      const float up = __shfl_up_sync(0xffffffffu, v[kConvW - (K - 1) + i], 1);
      const float last = __shfl_sync(0xffffffffu, v[kConvW - (K - 1) + i], 31);
      if (lane > 0) {
        halo[i] = up;
      } else if (r > 0) {
        halo[i] = carry[i];
      } else {
        const int64_t t = t0 - (K - 1) + i;
        halo[i] = t >= 0 ? IO<T>::get(xr, t) : x_before(t);
      }
      carry[i] = last;
    }
    float da[kConvW], pre[kConvW];
#pragma unroll
    for (int i = 0; i < kConvW; ++i) {
      float acc = bias;
#pragma unroll
      for (int k = 0; k < K; ++k) {
        const int idx = i - (K - 1) + k;
        acc = fmaf(w[k], idx < 0 ? halo[idx + K - 1] : v[idx], acc);
      }
      pre[i] = acc;
    }
    // da = dout * SiLU'(a) = g s (1 + a (1 - s)), s = 1 / (1 + e^-a), on pairs
#pragma unroll
    for (int i = 0; i < kConvW; i += 2) {
      if (silu) {
        float e0, e1, s0, s1;
        unpack2(mul2(pack2(pre[i], pre[i + 1]), pack2(-kLog2e, -kLog2e)), e0, e1);
        unpack2(add2(pack2(ex2(e0), ex2(e1)), pack2(1.f, 1.f)), s0, s1);
        const f2 sg = pack2(rcp_approx(s0), rcp_approx(s1));
        const f2 a2 = pack2(pre[i], pre[i + 1]);
        const f2 one_m = fma2(sg, pack2(-1.f, -1.f), pack2(1.f, 1.f));
        const f2 fac = fma2(a2, one_m, pack2(1.f, 1.f));
        unpack2(mul2(mul2(pack2(gv[i], gv[i + 1]), sg), fac), da[i], da[i + 1]);
      } else {
        da[i] = gv[i];
        da[i + 1] = gv[i + 1];
      }
    }
    if (!(t0 + kConvW <= L)) {  // the chunk holding step L-1: no gradient past L
#pragma unroll
      for (int i = 0; i < kConvW; ++i) da[i] = t0 + i < L ? da[i] : 0.f;
    }
#pragma unroll
    for (int i = 0; i < kConvW; ++i) {
      dbp += da[i];
#pragma unroll
      for (int k = 0; k < K; ++k) {
        const int idx = i - (K - 1) + k;
        dwp[k] = fmaf(da[i], idx < 0 ? halo[idx + K - 1] : v[idx], dwp[k]);
      }
    }
    // the next K-1 values of da after each lane's chunk of the pass before: the
    // next lane's first values, or for lane 31 this pass's lane 0
    if (have_prev) {
      float nxt[K > 1 ? K - 1 : 1];
#pragma unroll
      for (int m = 0; m < K - 1; ++m) {
        const float down = __shfl_down_sync(0xffffffffu, da_prev[m], 1);
        const float first = __shfl_sync(0xffffffffu, da[m], 0);
        nxt[m] = lane < 31 ? down : (live ? first : 0.f);
      }
      emit_dx(da_prev, nxt, t0_prev);
    }
    if (!live) { have_prev = false; break; }
#pragma unroll
    for (int i = 0; i < kConvW; ++i) da_prev[i] = da[i];
    t0_prev = t0;
    have_prev = true;
    // initial-state gradient: dx of x_{-(K-1)+j} = sum_k w_k da_{j-k}, j - k >= 0
    if (K > 1 && p.ds0 && seg == 0 && r == 0 && lane == 0) {
#pragma unroll
      for (int j = 0; j < K - 1; ++j) {
        float acc = 0.f;
#pragma unroll
        for (int k = 0; k < K; ++k)
          if (j - k >= 0) acc = fmaf(w[k], da[j - k], acc);
        p.ds0[row * (K - 1) + j] = acc;
      }
    }
  }
  if (have_prev) {  // the last pass: its next values come from the next segment
    float nxt[K > 1 ? K - 1 : 1];
#pragma unroll
    for (int m = 0; m < K - 1; ++m) {
      const float down = __shfl_down_sync(0xffffffffu, da_prev[m], 1);
      nxt[m] = down;
    }
    if (lane == 31) {
#pragma unroll
      for (int m = 0; m < K - 1; ++m) {
        const int64_t t = t0_prev + kConvW + m;  // a step of the next segment
        float acc = bias;
#pragma unroll
        for (int k = 0; k < K; ++k) {
          const int64_t tx = t - (K - 1) + k;
          acc = fmaf(w[k], tx < L ? IO<T>::get(xr, tx) : 0.f, acc);
        }
        nxt[m] = t < L ? conv_act_grad<T, K>(acc, IO<T>::get(gr, t), silu) : 0.f;
      }
    }
    emit_dx(da_prev, nxt, t0_prev);
  }
  // dw and dbias: warp sums, one atomic per warp
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
#pragma unroll
    for (int k = 0; k < K; ++k) dwp[k] += __shfl_xor_sync(0xffffffffu, dwp[k], o);
    dbp += __shfl_xor_sync(0xffffffffu, dbp, o);
  }
  if (lane == 0) {
#pragma unroll
    for (int k = 0; k < K; ++k) atomicAdd(&p.dw[d * K + k], dwp[k]);
    if (p.dbias) atomicAdd(&p.dbias[d], dbp);
  }
}

template <typename T, bool NARROW>
static cudaError_t launch_conv_k(const ConvParams &p, unsigned g, cudaStream_t s) {
  switch (p.K) {
    case 1: k_conv<T, 1, NARROW><<<g, kConvThreads, 0, s>>>(p); break;
    case 2: k_conv<T, 2, NARROW><<<g, kConvThreads, 0, s>>>(p); break;
    case 3: k_conv<T, 3, NARROW><<<g, kConvThreads, 0, s>>>(p); break;
    case 4: k_conv<T, 4, NARROW><<<g, kConvThreads, 0, s>>>(p); break;
    case 5: k_conv<T, 5, NARROW><<<g, kConvThreads, 0, s>>>(p); break;
    case 6: k_conv<T, 6, NARROW><<<g, kConvThreads, 0, s>>>(p); break;
    case 7: k_conv<T, 7, NARROW><<<g, kConvThreads, 0, s>>>(p); break;
    case 8: k_conv<T, 8, NARROW><<<g, kConvThreads, 0, s>>>(p); break;
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

template <typename T>
static cudaError_t launch_conv_t(const ConvParams &p, cudaStream_t s) {
  const int64_t segs = (p.L + kConvSeg - 1) / kConvSeg;
  const int64_t warps = p.batch * p.dim * segs;
  const int64_t blocks = (warps * 32 + kConvThreads - 1) / kConvThreads;
  if (blocks > 0x7fffffff) return cudaErrorInvalidConfiguration;
  const unsigned g = (unsigned)blocks;
  return blocks * kConvThreads <= 0xffffffffll ? launch_conv_k<T, true>(p, g, s) : launch_conv_k<T, false>(p, g, s);
}

cudaError_t launch_conv(int io_dtype, const ConvParams &p, cudaStream_t s) {
  return io_dtype == 1 ? launch_conv_t<uint16_t>(p, s) : launch_conv_t<float>(p, s);
}

template <typename T>
static cudaError_t launch_conv_bwd_t(const ConvBwdParams &p, cudaStream_t s) {
  const int64_t segs = (p.L + kConvBSeg - 1) / kConvBSeg;
  const int64_t warps = p.batch * p.dim * segs;
  const int64_t blocks = (warps * 32 + kConvThreads - 1) / kConvThreads;
  if (blocks > 0x7fffffff) return cudaErrorInvalidConfiguration;
  const unsigned g = (unsigned)blocks;
  switch (p.K) {
    case 1: k_conv_bwd<T, 1><<<g, kConvThreads, 0, s>>>(p); break;
    case 2: k_conv_bwd<T, 2><<<g, kConvThreads, 0, s>>>(p); break;
    case 3: k_conv_bwd<T, 3><<<g, kConvThreads, 0, s>>>(p); break;
    case 4: k_conv_bwd<T, 4><<<g, kConvThreads, 0, s>>>(p); break;
    case 5: k_conv_bwd<T, 5><<<g, kConvThreads, 0, s>>>(p); break;
    case 6: k_conv_bwd<T, 6><<<g, kConvThreads, 0, s>>>(p); break;
    case 7: k_conv_bwd<T, 7><<<g, kConvThreads, 0, s>>>(p); break;
    case 8: k_conv_bwd<T, 8><<<g, kConvThreads, 0, s>>>(p); break;
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

cudaError_t launch_conv_bwd(int io_dtype, const ConvBwdParams &p, cudaStream_t s) {
  return io_dtype == 1 ? launch_conv_bwd_t<uint16_t>(p, s) : launch_conv_bwd_t<float>(p, s);
}

}  // namespace ssm
