// Backward of the selective scan (S6) by recomputation, sm_100a.
//
// Gradients of sum_t dout_t * y_t for the forward in ssm_fwd.cu:
//   dy_t    = dout_t * SiLU(z_t)            dz_t = dout_t * yss_t * SiLU'(z_t)
//   g_tn    = dy_t C_tn + a_{t+1,n} g_{t+1,n}             (dL/dh_tn, reverse scan)
//   dC_tn  += dy_t h_tn                      dB_tn += g_tn Delta_t u_t   (sums over d)
//   dDelta_t = sum_n g_tn (A_n a_tn h_{t-1,n} + B_tn u_t)
//   dA_n   += g_tn Delta_t a_tn h_{t-1,n}    du_t  = dy_t D + Delta_t sum_n g_tn B_tn
//   ddelta_t = dDelta_t * sigmoid(s_t) (softplus) ; ddelta_bias += ddelta_t ; dD += dy_t u_t
// The states are recomputed, never read from the forward ("Mamba: Linear-Time
// Sequence Modeling with Selective State Spaces" reading guide, "Expansao de
// Estado Ciente de Hardware": intermediate states are recomputed in the
// backward pass instead of being stored in HBM).
//
// Schedule: a CTA of 4 warps owns 32 channels of one batch element; warp w
// holds channels 8w..8w+7 with 4 lanes per channel and S = NP/4 states per
// lane.  Phase A walks the sequence forward in 16-step chunks and stores the
// state entering each chunk in the workspace.  Phase B walks the chunks in
// reverse: it recomputes the chunk's 16 states into registers from the
// checkpoint, runs the reverse recurrence over them, and reduces dB/dC over
// the channels (registers -> warp shuffles -> the CTA's 4 warps in shared
// memory -> vector atomics into fp32 accumulators).  A last kernel rounds
// dB/dC to the io dtype.
#include "ssm_common.cuh"

namespace ssm {

constexpr int kTB = 16;       // steps per backward chunk
constexpr int kBW = 4;        // warps per CTA
constexpr int kBCPW = 8;      // channels per warp
constexpr int kBPad = 4;

// 4 consecutive io values
template <typename T> struct Vec4;
template <> struct Vec4<uint16_t> {
  uint2 v;
  __device__ __forceinline__ void load(const uint16_t *row, int64_t t, int64_t L, bool vec) {
    if (vec && t + 4 <= L) {
      v = __ldg(reinterpret_cast<const uint2 *>(row + t));
    } else {
      uint32_t w[2];
#pragma unroll
      for (int i = 0; i < 2; ++i) {
        const uint32_t lo = (t + 2 * i < L) ? row[t + 2 * i] : 0u;
        const uint32_t hi = (t + 2 * i + 1 < L) ? row[t + 2 * i + 1] : 0u;
        w[i] = lo | (hi << 16);
      }
      v = make_uint2(w[0], w[1]);
    }
  }
  __device__ __forceinline__ void unpack(float (&o)[4]) const {
    o[0] = bf16_lo(v.x); o[1] = bf16_hi(v.x); o[2] = bf16_lo(v.y); o[3] = bf16_hi(v.y);
  }
  __device__ __forceinline__ static void store(uint16_t *row, int64_t t, int64_t L, bool vec,
                                               const float (&o)[4]) {
    if (vec && t + 4 <= L) {
      *reinterpret_cast<uint2 *>(row + t) = make_uint2(pack_bf16x2(o[0], o[1]), pack_bf16x2(o[2], o[3]));
    } else {
#pragma unroll
      for (int i = 0; i < 4; ++i)
        if (t + i < L) IO<uint16_t>::store1(row, t + i, o[i]);
    }
  }
};
template <> struct Vec4<float> {
  float4 v;
  __device__ __forceinline__ void load(const float *row, int64_t t, int64_t L, bool vec) {
    if (vec && t + 4 <= L) {
      v = __ldg(reinterpret_cast<const float4 *>(row + t));
    } else {
      v = make_float4(t < L ? row[t] : 0.f, t + 1 < L ? row[t + 1] : 0.f,
                      t + 2 < L ? row[t + 2] : 0.f, t + 3 < L ? row[t + 3] : 0.f);
    }
  }
  __device__ __forceinline__ void unpack(float (&o)[4]) const { o[0] = v.x; o[1] = v.y; o[2] = v.z; o[3] = v.w; }
  __device__ __forceinline__ static void store(float *row, int64_t t, int64_t L, bool vec,
                                               const float (&o)[4]) {
    if (vec && t + 4 <= L) {
      *reinterpret_cast<float4 *>(row + t) = make_float4(o[0], o[1], o[2], o[3]);
    } else {
#pragma unroll
      for (int i = 0; i < 4; ++i)
        if (t + i < L) row[t + i] = o[i];
    }
  }
};

template <int NP>
struct __align__(16) BwdWarpSmem {
  float dl[kBCPW][kTB + kBPad];    // Delta
  float dlu[kBCPW][kTB + kBPad];   // Delta * u
  float sg[kBCPW][kTB + kBPad];    // sigmoid(s): d softplus / ds
  float dy[kBCPW][kTB + kBPad];    // dout * SiLU(z)
  float ys[kBCPW][kTB + kBPad];    // sum_n C h
  float ddl[kBCPW][kTB + kBPad];   // sum_n g (A a h_prev)
  float s1[kBCPW][kTB + kBPad];    // sum_n g B
  float dBC[kTB][2][NP];           // this warp's dB, dC over its 8 channels
};

template <int NP>
struct __align__(16) BwdSmem {
  float Bs[kTB][NP];
  float Cs[kTB][NP];
  BwdWarpSmem<NP> w[kBW];
};

// B and C chunk [t0, t0 + kTB) into smem (fp32, zero padded), by the whole CTA.
template <typename T, int NP>
__device__ __forceinline__ void bwd_stage_bc(BwdSmem<NP> &sm, const T *Bb, const T *Cb, int64_t t0,
                                             int64_t L, int N, bool with_c) {
  for (int e = threadIdx.x; e < kTB * NP; e += kBW * 32) {
    const int t = e / NP, n = e - t * NP;
    const bool in = n < N && t0 + t < L;
    sm.Bs[t][n] = in ? IO<T>::get(Bb, (t0 + t) * N + n) : 0.f;
    if (with_c) sm.Cs[t][n] = in ? IO<T>::get(Cb, (t0 + t) * N + n) : 0.f;
  }
}

// Sum V values over the 8 lanes that share lane%4 (lane bits 2..4): after the
// call lane l holds V/8 sums (V >= 8) at original indices
// i + c2*V/2 + c1*V/4 + c0*V/8, (c2 c1 c0) = lane bits 4, 3, 2.
template <int V>
__device__ __forceinline__ void halve3(float (&v)[V], int lane) {
  static_assert(V >= 8 && V % 8 == 0, "halve3 needs a multiple of 8 values");
#pragma unroll
  for (int lev = 0; lev < 3; ++lev) {
    const int m = 16 >> lev;           // lane mask: 16, 8, 4
    const int half = V >> (lev + 1);   // values kept after this level
    const bool hi = (lane & m) != 0;
#pragma unroll
    for (int i = 0; i < half; ++i) {
      const float keep = hi ? v[i + half] : v[i];
      const float send = hi ? v[i] : v[i + half];
      v[i] = keep + __shfl_xor_sync(0xffffffffu, send, m);
    }
  }
}

template <typename T, int NP>
__global__ void __launch_bounds__(kBW * 32) k_bwd(BwdParams p) {
  constexpr int S = NP / 4;
  extern __shared__ __align__(16) unsigned char smem_raw[];
  BwdSmem<NP> &sm = *reinterpret_cast<BwdSmem<NP> *>(smem_raw);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  BwdWarpSmem<NP> &ws = sm.w[warp];
  const int c = lane >> 2, j = lane & 3, q = j;   // q: this lane's 4 steps of a chunk
  const int64_t cta = blockIdx.x;
  const int64_t b = cta / p.cpb;
  const int64_t d = (cta - b * p.cpb) * (kBW * kBCPW) + warp * kBCPW + c;
  const bool valid = d < p.dim;
  const int64_t L = p.L, K = p.K;
  const int N = p.N;
  const bool io_vec = p.io_vec != 0;
  const int64_t row = (b * p.dim + (valid ? d : 0)) * L;
  const T *u_row = static_cast<const T *>(p.u) + row;
  const T *dr_row = static_cast<const T *>(p.delta) + row;
  const T *z_row = p.z ? static_cast<const T *>(p.z) + row : nullptr;
  const T *do_row = static_cast<const T *>(p.dout) + row;
  T *du_row = static_cast<T *>(p.du) + row;
  T *dd_row = static_cast<T *>(p.ddelta) + row;
  T *dz_row = p.dz ? static_cast<T *>(p.dz) + row : nullptr;
  const T *Bb = static_cast<const T *>(p.B) + b * L * N;
  const T *Cb = static_cast<const T *>(p.C) + b * L * N;
  const float bias = (p.bias && valid) ? p.bias[d] : 0.f;
  const float Dd = (p.D && valid) ? p.D[d] : 0.f;
  float A2[S], An[S];
#pragma unroll
  for (int s = 0; s < S; ++s) {
    const int n = j * S + s;
    An[s] = (valid && n < N) ? p.A[d * N + n] : 0.f;
    A2[s] = An[s] * kLog2e;
  }
  float *ck = p.ckpt + cta * K * (kBW * kBCPW) * NP;
  const int ch = warp * kBCPW + c;   // channel within the CTA

  // per (channel, step) quantities for this lane's 4 steps of chunk k
  auto prepass = [&](int64_t t0, float (&uu)[4], float (&sgs)[4]) {
    Vec4<T> vu, vd;
    if (valid) {
      vu.load(u_row, t0 + 4 * q, L, io_vec);
      vd.load(dr_row, t0 + 4 * q, L, io_vec);
    } else {
      vu.v = {}; vd.v = {};
    }
    float dr[4];
    vu.unpack(uu);
    vd.unpack(dr);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float s = dr[i] + bias;
      float dl = s, sg = 1.f;
      if (p.softplus) {
        dl = softplus_f(s);
        sg = sigmoid_f(s);
      }
      const bool in = valid && t0 + 4 * q + i < L;
      dl = in ? dl : 0.f;
      ws.dl[c][4 * q + i] = dl;
      ws.dlu[c][4 * q + i] = dl * uu[i];
      sgs[i] = sg;
    }
  };

  // ---- phase A: states entering every chunk ----
  float h[S];
#pragma unroll
  for (int s = 0; s < S; ++s) {
    const int n = j * S + s;
    h[s] = (p.h0 && valid && n < N) ? p.h0[(b * p.dim + d) * N + n] : 0.f;
  }
  for (int64_t k = 0; k < K; ++k) {
    const int64_t t0 = k * kTB;
#pragma unroll
    for (int s = 0; s < S; ++s) ck[(k * (kBW * kBCPW) + ch) * NP + j * S + s] = h[s];
    float uu[4], sgs[4];
    prepass(t0, uu, sgs);
    bwd_stage_bc<T, NP>(sm, Bb, Cb, t0, L, N, false);
    __syncthreads();
#pragma unroll 4
    for (int t = 0; t < kTB; ++t) {
      const float dl = ws.dl[c][t], du = ws.dlu[c][t];
#pragma unroll
      for (int s = 0; s < S; ++s) h[s] = fmaf(ex2(dl * A2[s]), h[s], du * sm.Bs[t][j * S + s]);
    }
    __syncthreads();
  }

  // ---- phase B: reverse ----
  float g[S], dA_acc[S];
#pragma unroll
  for (int s = 0; s < S; ++s) { g[s] = 0.f; dA_acc[s] = 0.f; }
  float dD_acc = 0.f, dbias_acc = 0.f;
  for (int64_t k = K - 1; k >= 0; --k) {
    const int64_t t0 = k * kTB;
    float uu[4], sgs[4];
    prepass(t0, uu, sgs);
    Vec4<T> vz, vo;
    if (valid) {
      vo.load(do_row, t0 + 4 * q, L, io_vec);
      if (z_row) vz.load(z_row, t0 + 4 * q, L, io_vec);
    }
    bwd_stage_bc<T, NP>(sm, Bb, Cb, t0, L, N, true);
    __syncthreads();

    // recompute the chunk's states from its checkpoint
    float H[kTB][S], h0c[S];
#pragma unroll
    for (int s = 0; s < S; ++s) h0c[s] = ck[(k * (kBW * kBCPW) + ch) * NP + j * S + s];
#pragma unroll
    for (int t = 0; t < kTB; t += 4) {
      float yp[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float dl = ws.dl[c][t + i], du = ws.dlu[c][t + i];
        float acc = 0.f;
#pragma unroll
        for (int s = 0; s < S; ++s) {
          const float hp = (t + i == 0) ? h0c[s] : H[t + i - 1][s];
          H[t + i][s] = fmaf(ex2(dl * A2[s]), hp, du * sm.Bs[t + i][j * S + s]);
          acc = fmaf(sm.Cs[t + i][j * S + s], H[t + i][s], acc);
        }
        yp[i] = acc;
      }
      // sum over the channel's 4 lanes; lane j keeps step t + j
      const bool hi2 = (j & 2) != 0, hi1 = (j & 1) != 0;
      float ka = hi2 ? yp[2] : yp[0], kb = hi2 ? yp[3] : yp[1];
      ka += __shfl_xor_sync(0xffffffffu, hi2 ? yp[0] : yp[2], 2);
      kb += __shfl_xor_sync(0xffffffffu, hi2 ? yp[1] : yp[3], 2);
      float kk = hi1 ? kb : ka;
      kk += __shfl_xor_sync(0xffffffffu, hi1 ? ka : kb, 1);
      ws.ys[c][t + j] = kk;
    }
    __syncwarp();

    // output-side gradients of this lane's 4 steps
    {
      float zz[4] = {0.f, 0.f, 0.f, 0.f}, oo[4] = {0.f, 0.f, 0.f, 0.f}, dzv[4];
      if (valid) {
        vo.unpack(oo);
        if (z_row) vz.unpack(zz);
      }
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float yss = fmaf(Dd, uu[i], ws.ys[c][4 * q + i]);
        float dy = oo[i];
        if (z_row) {
          const float sz = sigmoid_f(zz[i]);
          dzv[i] = oo[i] * yss * sz * fmaf(zz[i], 1.f - sz, 1.f);
          dy = oo[i] * zz[i] * sz;
        }
        dy = (valid && t0 + 4 * q + i < L) ? dy : 0.f;
        ws.dy[c][4 * q + i] = dy;
        dD_acc = fmaf(dy, uu[i], dD_acc);
      }
      if (z_row && valid) Vec4<T>::store(dz_row, t0 + 4 * q, L, io_vec, dzv);
    }
    __syncwarp();

    // reverse recurrence over the chunk
#pragma unroll
    for (int t = kTB - 1; t >= 0; --t) {
      const float dy = ws.dy[c][t], dl = ws.dl[c][t], du = ws.dlu[c][t];
      float ddl = 0.f, s1 = 0.f;
      float v[2 * S];
#pragma unroll
      for (int s = 0; s < S; ++s) {
        const float Bv = sm.Bs[t][j * S + s], Cv = sm.Cs[t][j * S + s];
        g[s] = fmaf(dy, Cv, g[s]);
        const float a = ex2(dl * A2[s]);
        const float hp = (t == 0) ? h0c[s] : H[t - 1][s];
        const float qv = g[s] * a * hp;
        dA_acc[s] = fmaf(dl, qv, dA_acc[s]);
        ddl = fmaf(An[s], qv, ddl);
        s1 = fmaf(g[s], Bv, s1);
        v[s] = g[s] * du;            // dB contribution
        v[S + s] = dy * H[t][s];     // dC contribution
        g[s] *= a;
      }
      ddl += __shfl_xor_sync(0xffffffffu, ddl, 1);
      s1 += __shfl_xor_sync(0xffffffffu, s1, 1);
      ddl += __shfl_xor_sync(0xffffffffu, ddl, 2);
      s1 += __shfl_xor_sync(0xffffffffu, s1, 2);
      if (j == 0) { ws.ddl[c][t] = ddl; ws.s1[c][t] = s1; }
      // sum the dB/dC contributions over the warp's 8 channels
      if constexpr (2 * S >= 8) {
        halve3<2 * S>(v, lane);
        const int base = ((c >> 2) & 1) * S + ((c >> 1) & 1) * (S / 2) + (c & 1) * (S / 4);
#pragma unroll
        for (int i = 0; i < 2 * S / 8; ++i) {
          const int o = base + i;
          const int which = o >= S ? 1 : 0;
          ws.dBC[t][which][j * S + (o - which * S)] = v[i];
        }
      } else {
#pragma unroll
        for (int i = 0; i < 2 * S; ++i) {
          float x = v[i];
          x += __shfl_xor_sync(0xffffffffu, x, 4);
          x += __shfl_xor_sync(0xffffffffu, x, 8);
          x += __shfl_xor_sync(0xffffffffu, x, 16);
          if (c == 0) ws.dBC[t][i >= S ? 1 : 0][j * S + (i % S)] = x;
        }
      }
    }
    __syncthreads();

    // input-side gradients of this lane's 4 steps
    {
      float duv[4], ddv[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int t = 4 * q + i;
        const float s1 = ws.s1[c][t], dl = ws.dl[c][t];
        duv[i] = fmaf(dl, s1, ws.dy[c][t] * Dd);
        float dd = fmaf(uu[i], s1, ws.ddl[c][t]);
        if (p.softplus) dd *= sgs[i];
        dd = (valid && t0 + t < L) ? dd : 0.f;
        ddv[i] = dd;
        dbias_acc += dd;
      }
      if (valid) {
        Vec4<T>::store(du_row, t0 + 4 * q, L, io_vec, duv);
        Vec4<T>::store(dd_row, t0 + 4 * q, L, io_vec, ddv);
      }
    }
    // dB, dC of the chunk: sum the 4 warps, add to the fp32 accumulators
    for (int e = threadIdx.x * 4; e < kTB * 2 * NP; e += kBW * 32 * 4) {
      const int t = e / (2 * NP), r = e - t * 2 * NP, which = r / NP, n = r - which * NP;
      if (t0 + t >= L) continue;
      float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
      for (int w = 0; w < kBW; ++w) {
        const float4 x = *reinterpret_cast<const float4 *>(&sm.w[w].dBC[t][which][n]);
        acc.x += x.x; acc.y += x.y; acc.z += x.z; acc.w += x.w;
      }
      float *dst = (which ? p.dC_acc : p.dB_acc) + ((b * L + t0 + t) * NP + n);
      atomicAdd(reinterpret_cast<float4 *>(dst), acc);
    }
    __syncthreads();
  }

  // ---- per-channel sums ----
  if (valid) {
#pragma unroll
    for (int s = 0; s < S; ++s) {
      const int n = j * S + s;
      if (n < N) {
        atomicAdd(&p.dA[d * N + n], dA_acc[s]);
        if (p.dh0) p.dh0[(b * p.dim + d) * N + n] = g[s];
      }
    }
  }
  dD_acc += __shfl_xor_sync(0xffffffffu, dD_acc, 1);
  dD_acc += __shfl_xor_sync(0xffffffffu, dD_acc, 2);
  dbias_acc += __shfl_xor_sync(0xffffffffu, dbias_acc, 1);
  dbias_acc += __shfl_xor_sync(0xffffffffu, dbias_acc, 2);
  if (valid && j == 0) {
    if (p.dD) atomicAdd(&p.dD[d], dD_acc);
    if (p.dbias) atomicAdd(&p.dbias[d], dbias_acc);
  }
}

// dB, dC: fp32 accumulators [batch][L][NP] -> io dtype [batch][L][N]
template <typename T, int NP>
__global__ void k_bwd_finalize(BwdParams p) {
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  const int64_t total = p.batch * p.L * p.N;
  if (i >= total) return;
  const int64_t bt = i / p.N;
  const int n = (int)(i - bt * p.N);
  IO<T>::store1(static_cast<T *>(p.dB), i, p.dB_acc[bt * NP + n]);
  IO<T>::store1(static_cast<T *>(p.dC), i, p.dC_acc[bt * NP + n]);
}

// ---- host side ------------------------------------------------------------------
template <class V> struct BTypeTag { using type = V; };
template <int V> struct BIntTag { static constexpr int value = V; };

template <class F>
static cudaError_t bwd_dispatch(int io_dtype, int NP, F &&f) {
  auto by_np = [&](auto tt) -> cudaError_t {
    switch (NP) {
      case 4: return f(tt, BIntTag<4>{});
      case 8: return f(tt, BIntTag<8>{});
      case 16: return f(tt, BIntTag<16>{});
      case 32: return f(tt, BIntTag<32>{});
      case 64: return f(tt, BIntTag<64>{});
      default: return cudaErrorInvalidValue;
    }
  };
  if (io_dtype == 1) return by_np(BTypeTag<uint16_t>{});
  if (io_dtype == 0) return by_np(BTypeTag<float>{});
  return cudaErrorInvalidValue;
}

size_t bwd_ckpt_floats(int64_t batch, int64_t dim, int64_t L, int NP) {
  const int64_t cpb = (dim + kBW * kBCPW - 1) / (kBW * kBCPW);
  const int64_t K = (L + kTB - 1) / kTB;
  return (size_t)(batch * cpb) * (size_t)K * (kBW * kBCPW) * NP;
}

cudaError_t launch_bwd(int io_dtype, int NP, BwdParams &p, cudaStream_t s) {
  p.cpb = (p.dim + kBW * kBCPW - 1) / (kBW * kBCPW);
  p.K = (p.L + kTB - 1) / kTB;
  return bwd_dispatch(io_dtype, NP, [&](auto tt, auto np) -> cudaError_t {
    using T = typename decltype(tt)::type;
    constexpr int kNP = decltype(np)::value;
    const size_t smem = sizeof(BwdSmem<kNP>);
    if (smem > 48 * 1024) {
      cudaError_t e = cudaFuncSetAttribute(k_bwd<T, kNP>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           (int)smem);
      if (e != cudaSuccess) return e;
    }
    const int64_t ctas = p.batch * p.cpb;
    k_bwd<T, kNP><<<(unsigned)ctas, kBW * 32, smem, s>>>(p);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    const int64_t total = p.batch * p.L * p.N;
    k_bwd_finalize<T, kNP><<<(unsigned)((total + 255) / 256), 256, 0, s>>>(p);
    return cudaGetLastError();
  });
}

}  // namespace ssm
