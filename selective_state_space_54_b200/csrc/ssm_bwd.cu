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
// This is the general kernel (every d_state up to 64); d_state 16 takes
// k_bwd16 (ssm_bwd16.cu).  Schedule: a CTA of 4 warps owns 32 channels of one
// batch element; warp w holds channels 8w..8w+7 with 4 lanes per channel and
// S = NP/4 states per lane.  Phase A walks the sequence forward in 16-step
// chunks and stores the state entering each chunk in the workspace (the
// saved-state layout of ssm_common.cuh, every other 8-step entry).  Phase B
// walks the chunks in reverse: it recomputes the chunk's 16 states into
// registers from the checkpoint, runs the reverse recurrence over them, and
// reduces dB/dC over the channels (registers -> the CTA's 4 warps in shared
// memory -> one partial per 32-channel block).  k_bwd_reduce adds the
// partials (dB/dC over channel blocks, dA/dD/ddelta_bias over the batch) in a
// fixed order and rounds dB/dC to the io dtype: no atomics, bitwise
// repeatable.
#include "ssm_common.cuh"

namespace ssm {

constexpr int kTB = 2 * kCkptSteps;  // steps per backward chunk: two saved-state chunks
constexpr int kBW = 4;        // warps per CTA
constexpr int kBCPW = 8;      // channels per warp
constexpr int kBPad = 4;
static_assert(kCkptPad % (kBW * kBCPW) == 0, "saved states cover every padded channel of a CTA");

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
  float dy[kBCPW][kTB + kBPad];    // dout * SiLU(z)
  float ys[kBCPW][kTB + kBPad];    // sum_n C h
  float uu[kBCPW][kTB + kBPad];    // u (0 past L), for the exact-ZOH derivatives
  // per step, channel and lane j: (sum_n g A a h_prev, sum_n g B) partials;
  // step-major so that a warp's stores of one step are contiguous
  float2 pd[kTB][kBCPW][4];
  // dB, dC contributions of a 4-step group: [step][B|C][lane slice j][channel,
  // state] with 8 floats of padding per row so that a quarter warp's stores
  // hit distinct banks
  float part[4][2][4][kBCPW * (NP / 4) + 8];
};

template <int NP>
struct __align__(16) BwdSmem {
  float Bs[kTB][NP];
  float Cs[kTB][NP];
  BwdWarpSmem<NP> w[kBW];
  // per-warp sums of one 4-step group's dB/dC outputs (16-byte vectors)
  ulonglong2 red[kBW][NP / 4 >= 1 ? 4 * 2 * NP / 4 : 1];
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

// One chunk of B and C in flight as raw 16-byte pieces, spread over the CTA
// (vector path: N == NP, 16-byte aligned rows).
template <typename T, int NP>
struct BwdBC {
  static constexpr int EPP = 16 / (int)sizeof(T);
  static constexpr bool kVec = (NP % EPP) == 0;
  static constexpr int NV = kVec ? kTB * NP / EPP : 1;              // pieces per tensor
  static constexpr int PER = (2 * NV + kBW * 32 - 1) / (kBW * 32);  // pieces per thread
  uint4 r[PER];
  __device__ __forceinline__ void load(const T *Bb, const T *Cb, int64_t t0, int64_t L, bool with_c) {
#pragma unroll
    for (int i = 0; i < PER; ++i) {
      const int v = threadIdx.x + i * kBW * 32;
      const int which = v / NV, vv = v - which * NV;
      const int e = vv * EPP, t = e / NP, n = e - t * NP;
      if (v < 2 * NV && t0 + t < L && (which == 0 || with_c))
        r[i] = __ldg(reinterpret_cast<const uint4 *>((which ? Cb : Bb) + (t0 + t) * NP + n));
      else
        r[i] = make_uint4(0, 0, 0, 0);
    }
  }
  __device__ __forceinline__ void stage(float (*Bs)[NP], float (*Cs)[NP]) const {
#pragma unroll
    for (int i = 0; i < PER; ++i) {
      const int v = threadIdx.x + i * kBW * 32;
      if (v >= 2 * NV) continue;
      const int which = v / NV, vv = v - which * NV;
      const int e = vv * EPP, t = e / NP, n = e - t * NP;
      float *dst = which ? &Cs[t][n] : &Bs[t][n];
      if constexpr (sizeof(T) == 2) {
        *reinterpret_cast<float4 *>(dst) = make_float4(bf16_lo(r[i].x), bf16_hi(r[i].x), bf16_lo(r[i].y), bf16_hi(r[i].y));
        *reinterpret_cast<float4 *>(dst + 4) = make_float4(bf16_lo(r[i].z), bf16_hi(r[i].z), bf16_lo(r[i].w), bf16_hi(r[i].w));
      } else {
        *reinterpret_cast<float4 *>(dst) = make_float4(__uint_as_float(r[i].x), __uint_as_float(r[i].y),
                                                       __uint_as_float(r[i].z), __uint_as_float(r[i].w));
      }
    }
  }
};

__device__ __forceinline__ f2 ex2_2(f2 x) {
  float x0, x1;
  unpack2(x, x0, x1);
  return pack2(ex2(x0), ex2(x1));
}

template <typename T, int NP, bool ZOH>
__global__ void __launch_bounds__(kBW * 32, (NP == 8 || NP == 16) ? 4 : (NP == 4 ? 3 : 2)) k_bwd(BwdParams p) {
  constexpr int S = NP / 4;              // states per lane
  constexpr int SP = S >= 2 ? S / 2 : 1; // state pairs per lane (S = 1 pads one)
  extern __shared__ __align__(16) unsigned char smem_raw[];
  BwdSmem<NP> &sm = *reinterpret_cast<BwdSmem<NP> *>(smem_raw);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  BwdWarpSmem<NP> &ws = sm.w[warp];
  const int c = lane >> 2, j = lane & 3, q = j;   // q: this lane's 4 steps of a chunk
  const int64_t cta = blockIdx.x;
  const int64_t b = cta / p.cpb, cb = cta - b * p.cpb;
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
  // this lane's states n = j*S + s, as pairs; S = 1 uses the low half only
  f2 A2[SP], An[SP];
#pragma unroll
  for (int i = 0; i < SP; ++i) {
    float a[2];
#pragma unroll
    for (int h2 = 0; h2 < 2; ++h2) {
      const int s = 2 * i + h2, n = j * S + s;
      a[h2] = (s < S && valid && n < N) ? p.A[d * N + n] : 0.f;
    }
    An[i] = pack2(a[0], a[1]);
    A2[i] = pack2(a[0] * kLog2e, a[1] * kLog2e);
  }
  // exact ZOH: 1 / A_n per state (infinite for A_n = 0, whose x is 0: the series branch)
  f2 rA[ZOH ? SP : 1];
  if constexpr (ZOH) {
#pragma unroll
    for (int i = 0; i < SP; ++i) {
      float a0, a1;
      unpack2(An[i], a0, a1);
      rA[i] = pack2(__frcp_rn(a0), __frcp_rn(a1));
    }
  }
  // saved state entering 16-step chunk k = 8-step saved chunk 2k (padded channels included)
  float *ck = p.ckpt + ckpt_offset(b, d, 0, p.dim, L, NP) + j * S;
  auto ck_at = [&](int64_t k, int i) -> float * { return &ck[2 * k * kCkptChannels * NP + 2 * i]; };
  auto Bpair = [&](int t, int i) -> f2 {
    if constexpr (S >= 2) return *reinterpret_cast<const f2 *>(&sm.Bs[t][j * S + 2 * i]);
    else return pack2(sm.Bs[t][j], 0.f);
  };
  auto Cpair = [&](int t, int i) -> f2 {
    if constexpr (S >= 2) return *reinterpret_cast<const f2 *>(&sm.Cs[t][j * S + 2 * i]);
    else return pack2(sm.Cs[t][j], 0.f);
  };

  // per (channel, step) quantities for this lane's 4 steps of chunk k
  // per (channel, step) quantities for this lane's 4 steps of a chunk, from
  // the chunk's preloaded u and delta
  auto prepass = [&](int64_t t0, const Vec4<T> &vu, const Vec4<T> &vd, float (&uu)[4],
                     float (&sgs)[4]) {
    float dr[4];
    vu.unpack(uu);
    vd.unpack(dr);
    float dl4[4], du4[4];
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
      dl4[i] = dl;
      du4[i] = dl * uu[i];
      sgs[i] = sg;
    }
    *reinterpret_cast<float4 *>(&ws.dl[c][4 * q]) = make_float4(dl4[0], dl4[1], dl4[2], dl4[3]);
    *reinterpret_cast<float4 *>(&ws.dlu[c][4 * q]) = make_float4(du4[0], du4[1], du4[2], du4[3]);
    if (ZOH) {
      float u4[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) u4[i] = (valid && t0 + 4 * q + i < L) ? uu[i] : 0.f;
      *reinterpret_cast<float4 *>(&ws.uu[c][4 * q]) = make_float4(u4[0], u4[1], u4[2], u4[3]);
    }
  };
  // the input term Bbar_n u: Delta u B_n (Euler) or u W B_n, W = Delta (e^x - 1)/x (exact ZOH)
  auto bterm = [&](int t, f2 dl2, f2 du2, f2 x, f2 a, int i, f2 Bv) -> f2 {
    if constexpr (ZOH) {
      const float uv = ws.uu[c][t];
      return mul2(mul2(pack2(uv, uv), zoh_w(x, a, dl2, rA[i])), Bv);
    } else {
      return mul2(du2, Bv);
    }
  };

  // inputs of one chunk, loaded a chunk ahead of their use
  struct ChunkIn {
    Vec4<T> u, d, o, z;
    BwdBC<T, NP> bc;
  };
  const bool bc_vec = p.bc_vec != 0 && BwdBC<T, NP>::kVec;
  auto load_chunk = [&](int64_t k, bool full, ChunkIn &in) {
    const int64_t t0 = k * kTB;
    if (valid) {
      in.u.load(u_row, t0 + 4 * q, L, io_vec);
      in.d.load(dr_row, t0 + 4 * q, L, io_vec);
      if (full) {
        in.o.load(do_row, t0 + 4 * q, L, io_vec);
        if (z_row) in.z.load(z_row, t0 + 4 * q, L, io_vec);
      }
    } else {
      in.u.v = {}; in.d.v = {}; in.o.v = {}; in.z.v = {};
    }
    if (bc_vec) in.bc.load(Bb, Cb, t0, L, full);
  };
  auto stage_chunk = [&](int64_t t0, const ChunkIn &in, bool full) {
    if (bc_vec) in.bc.stage(sm.Bs, sm.Cs);
    else bwd_stage_bc<T, NP>(sm, Bb, Cb, t0, L, N, full);
  };

  // ---- phase A: states entering every chunk ----
  f2 h[SP];
#pragma unroll
  for (int i = 0; i < SP; ++i) {
    float v[2];
#pragma unroll
    for (int h2 = 0; h2 < 2; ++h2) {
      const int s = 2 * i + h2, n = j * S + s;
      v[h2] = (s < S && p.h0 && valid && n < N) ? p.h0[(b * p.dim + d) * N + n] : 0.f;
    }
    h[i] = pack2(v[0], v[1]);
  }
  ChunkIn nxt;
  if (K > 0 && !p.ckpt_given) load_chunk(0, false, nxt);
  for (int64_t k = 0; k < (p.ckpt_given ? 0 : K); ++k) {
    const int64_t t0 = k * kTB;
#pragma unroll
    for (int i = 0; i < SP; ++i) {
      float lo, hi;
      unpack2(h[i], lo, hi);
      float *dst = ck_at(k, i);
      dst[0] = lo;
      if (S >= 2) dst[1] = hi;
    }
    const ChunkIn cur = nxt;
    if (k + 1 < K) load_chunk(k + 1, false, nxt);
    float uu[4], sgs[4];
    prepass(t0, cur.u, cur.d, uu, sgs);
    stage_chunk(t0, cur, false);
    __syncthreads();
#pragma unroll 4
    for (int t = 0; t < kTB; ++t) {
      const f2 dl2 = pack2(ws.dl[c][t], ws.dl[c][t]), du2 = pack2(ws.dlu[c][t], ws.dlu[c][t]);
#pragma unroll
      for (int i = 0; i < SP; ++i) {
        const f2 x = mul2(dl2, A2[i]), a = ex2_2(x);
        h[i] = fma2(a, h[i], bterm(t, dl2, du2, x, a, i, Bpair(t, i)));
      }
    }
    __syncthreads();
  }

  // ---- phase B: reverse ----
  f2 g[SP], dA_acc[SP];
#pragma unroll
  for (int i = 0; i < SP; ++i) { g[i] = pack2(0.f, 0.f); dA_acc[i] = g[i]; }
  float dD_acc = 0.f, dbias_acc = 0.f;
  constexpr int kRedOutputs = 4 * 2 * NP / 4;   // float4 outputs of a 4-step group
  if (K > 0) load_chunk(K - 1, true, nxt);
  for (int64_t k = K - 1; k >= 0; --k) {
    const int64_t t0 = k * kTB;
    const ChunkIn cur = nxt;
    if (k > 0) load_chunk(k - 1, true, nxt);
    float uu[4], sgs[4];
    prepass(t0, cur.u, cur.d, uu, sgs);
    stage_chunk(t0, cur, true);
    __syncthreads();

    // recompute the chunk's states from its checkpoint, keeping only the
    // state entering each 4-step group (the reverse pass recomputes a group's
    // states again right before it needs them)
    f2 H4[kTB / 4][SP];
    {
      f2 hh[SP];
#pragma unroll
      for (int i = 0; i < SP; ++i) {
        const float *src = ck_at(k, i);  // padded channels: saved states may be unwritten
        hh[i] = valid ? pack2(src[0], S >= 2 ? src[1] : 0.f) : pack2(0.f, 0.f);
      }
#pragma unroll
    for (int t = 0; t < kTB; t += 4) {
      float yp[4];
#pragma unroll
      for (int i = 0; i < SP; ++i) H4[t / 4][i] = hh[i];
#pragma unroll
      for (int i4 = 0; i4 < 4; ++i4) {
        const int tt = t + i4;
        const f2 dl2 = pack2(ws.dl[c][tt], ws.dl[c][tt]), du2 = pack2(ws.dlu[c][tt], ws.dlu[c][tt]);
        f2 acc = pack2(0.f, 0.f);
#pragma unroll
        for (int i = 0; i < SP; ++i) {
          const f2 x = mul2(dl2, A2[i]), a = ex2_2(x);
          hh[i] = fma2(a, hh[i], bterm(tt, dl2, du2, x, a, i, Bpair(tt, i)));
          acc = fma2(Cpair(tt, i), hh[i], acc);
        }
        float a0, a1;
        unpack2(acc, a0, a1);
        yp[i4] = a0 + a1;
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
    }
    __syncwarp();

    // output-side gradients of this lane's 4 steps
    {
      float zz[4] = {0.f, 0.f, 0.f, 0.f}, oo[4] = {0.f, 0.f, 0.f, 0.f}, dzv[4], dyv[4];
      if (valid) {
        cur.o.unpack(oo);
        if (z_row) cur.z.unpack(zz);
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
        dyv[i] = dy;
        dD_acc = fmaf(dy, uu[i], dD_acc);
      }
      *reinterpret_cast<float4 *>(&ws.dy[c][4 * q]) = make_float4(dyv[0], dyv[1], dyv[2], dyv[3]);
      if (z_row && valid) Vec4<T>::store(dz_row, t0 + 4 * q, L, io_vec, dzv);
    }
    __syncwarp();

    // reverse recurrence over the chunk, in 4-step groups: each group's states
    // and decays are recomputed from the state entering it, then walked in
    // reverse; after each group the CTA sums its 32 channels' dB/dC
    // contributions and adds them to the fp32 accumulators
#pragma unroll
    for (int grp = kTB / 4 - 1; grp >= 0; --grp) {
      f2 hg[4][SP], ag[4][SP];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int t = 4 * grp + u;
        const float dlv = ws.dl[c][t], duv = ws.dlu[c][t];
        const f2 dl2 = pack2(dlv, dlv), du2 = pack2(duv, duv);
#pragma unroll
        for (int i = 0; i < SP; ++i) {
          const f2 x = mul2(dl2, A2[i]);
          ag[u][i] = ex2_2(x);
          hg[u][i] = fma2(ag[u][i], u == 0 ? H4[grp][i] : hg[u - 1][i],
                          bterm(t, dl2, du2, x, ag[u][i], i, Bpair(t, i)));
        }
      }
#pragma unroll
      for (int u = 3; u >= 0; --u) {
        const int t = 4 * grp + u;
        const float dyv = ws.dy[c][t], dlv = ws.dl[c][t], duv = ws.dlu[c][t];
        const f2 dy2 = pack2(dyv, dyv), dl2 = pack2(dlv, dlv), du2 = pack2(duv, duv);
        f2 ddl2 = pack2(0.f, 0.f), s12 = ddl2;
        f2 u2 = ddl2;
        if constexpr (ZOH) {
          const float uv = ws.uu[c][t];
          u2 = pack2(uv, uv);
        }
        float *pB = &ws.part[u][0][j][c * S];
        float *pC = &ws.part[u][1][j][c * S];
#pragma unroll
        for (int i = 0; i < SP; ++i) {
          g[i] = fma2(dy2, Cpair(t, i), g[i]);
          const f2 hp = u == 0 ? H4[grp][i] : hg[u - 1][i];
          const f2 ga = mul2(g[i], ag[u][i]);
          const f2 qv = mul2(ga, hp);
          dA_acc[i] = fma2(dl2, qv, dA_acc[i]);
          ddl2 = fma2(An[i], qv, ddl2);
          f2 vB;
          if constexpr (ZOH) {
            // h_t = a h_{t-1} + u W B with W = Delta (e^x - 1)/x, x = Delta A: d/dDelta
            // of the input term is a u B, d/dA is u Y B (Y = Delta^2 psi(x)), d/du is W B
            const f2 x = mul2(dl2, A2[i]);
            const f2 W = zoh_w(x, ag[u][i], dl2, rA[i]);
            const f2 gB = mul2(g[i], Bpair(t, i));
            ddl2 = fma2(mul2(ga, Bpair(t, i)), u2, ddl2);
            dA_acc[i] = fma2(mul2(gB, zoh_y(x, ag[u][i], W, dl2, rA[i])), u2, dA_acc[i]);
            s12 = fma2(gB, W, s12);
            vB = mul2(mul2(g[i], u2), W);
          } else {
            s12 = fma2(g[i], Bpair(t, i), s12);
            vB = mul2(g[i], du2);
          }
          const f2 vC = mul2(dy2, hg[u][i]);
          g[i] = ga;
          if constexpr (S >= 2) {
            *reinterpret_cast<f2 *>(pB + 2 * i) = vB;
            *reinterpret_cast<f2 *>(pC + 2 * i) = vC;
          } else {
            float lo, hi;
            unpack2(vB, lo, hi);
            pB[0] = lo;
            unpack2(vC, lo, hi);
            pC[0] = lo;
          }
        }
        float d0, d1, s0, s1v;
        unpack2(ddl2, d0, d1);
        unpack2(s12, s0, s1v);
        ws.pd[t][c][j] = make_float2(d0 + d1, s0 + s1v);
      }
      __syncthreads();
      // dB, dC of this group: sums over the 4 warps x 8 channels, stored as
      // this 32-channel block's partial (16-byte stores when S >= 4)
      if constexpr (S >= 4) {
        // every warp sums its own 8 channels for each output; warp 0 then
        // adds the 4 warps' sums in order and stores them
        for (int o = lane; o < kRedOutputs; o += 32) {
          const int tl = o / (2 * NP / 4), r4 = (o % (2 * NP / 4)) * 4;
          const int which = r4 / NP, n = r4 - which * NP;
          const int jj = n / S, s0 = n - jj * S;
          f2 acc0 = pack2(0.f, 0.f), acc1 = acc0;
#pragma unroll
          for (int cc = 0; cc < kBCPW; ++cc) {
            const float *src = &ws.part[tl][which][jj][cc * S + s0];
            const ulonglong2 x = *reinterpret_cast<const ulonglong2 *>(src);
            acc0 = add2(acc0, x.x);
            acc1 = add2(acc1, x.y);
          }
          sm.red[warp][o] = make_ulonglong2(acc0, acc1);
        }
        __syncthreads();
        if (warp == 0) {
          for (int o = lane; o < kRedOutputs; o += 32) {
            const int tl = o / (2 * NP / 4), r4 = (o % (2 * NP / 4)) * 4;
            const int which = r4 / NP, n = r4 - which * NP;
            const int t = 4 * grp + tl;
            f2 acc0 = pack2(0.f, 0.f), acc1 = acc0;
#pragma unroll
            for (int w = 0; w < kBW; ++w) {
              const ulonglong2 x = sm.red[w][o];
              acc0 = add2(acc0, x.x);
              acc1 = add2(acc1, x.y);
            }
            if (t0 + t < L) {
              float4 acc;
              unpack2(acc0, acc.x, acc.y);
              unpack2(acc1, acc.z, acc.w);
              *reinterpret_cast<float4 *>(p.dBC_part + ((cb * p.batch + b) * L + t0 + t) * 2 * NP +
                                          which * NP + n) = acc;
            }
          }
        }
      } else {
        for (int o = threadIdx.x; o < 4 * 2 * NP; o += kBW * 32) {
          const int tl = o / (2 * NP), r = o % (2 * NP);
          const int which = r / NP, n = r - which * NP;
          const int jj = n / S, s0 = n - jj * S;
          const int t = 4 * grp + tl;
          if (t0 + t < L) {
            float acc = 0.f;
#pragma unroll
            for (int w = 0; w < kBW; ++w)
#pragma unroll
              for (int cc = 0; cc < kBCPW; ++cc) acc += sm.w[w].part[tl][which][jj][cc * S + s0];
            p.dBC_part[((cb * p.batch + b) * L + t0 + t) * 2 * NP + which * NP + n] = acc;
          }
        }
        __syncthreads();  // the next group rewrites part
      }
      // (S >= 4: the barrier between the per-warp sums and warp 0's combine
      // already orders this group's reads of part before the next group's
      // writes, and warp 0's reads of red before the next group's barrier)
    }

    // input-side gradients of this lane's 4 steps
    {
      float duv[4], ddv[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int t = 4 * q + i;
        const float4 pa = *reinterpret_cast<const float4 *>(&ws.pd[t][c][0]);
        const float4 pb = *reinterpret_cast<const float4 *>(&ws.pd[t][c][2]);
        const float ddl = (pa.x + pa.z) + (pb.x + pb.z);
        const float s1 = (pa.y + pa.w) + (pb.y + pb.w);
        const float dl = ws.dl[c][t];
        // Euler: du = Delta sum g B + D dy; exact ZOH: s1 = sum g W B already holds Delta
        duv[i] = fmaf(ZOH ? 1.f : dl, s1, ws.dy[c][t] * Dd);
        // Euler: dDelta = sum g (A a h_prev + B u); exact ZOH: the u term is
        // already inside ddl (sum g a B u)
        float dd = ZOH ? ddl : fmaf(uu[i], s1, ddl);
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
    __syncthreads();
  }

  // ---- per-channel sums ----
  if (valid) {
#pragma unroll
    for (int i = 0; i < SP; ++i) {
      float lo[2], gg[2];
      unpack2(dA_acc[i], lo[0], lo[1]);
      unpack2(g[i], gg[0], gg[1]);
#pragma unroll
      for (int h2 = 0; h2 < 2; ++h2) {
        const int s = 2 * i + h2, n = j * S + s;
        if (s < S && n < N) {
          p.dA_part[(b * p.dim + d) * N + n] = lo[h2];
          if (p.dh0) p.dh0[(b * p.dim + d) * N + n] = gg[h2];
        }
      }
    }
  }
  dD_acc += __shfl_xor_sync(0xffffffffu, dD_acc, 1);
  dD_acc += __shfl_xor_sync(0xffffffffu, dD_acc, 2);
  dbias_acc += __shfl_xor_sync(0xffffffffu, dbias_acc, 1);
  dbias_acc += __shfl_xor_sync(0xffffffffu, dbias_acc, 2);
  if (valid && j == 0) {
    if (p.dD_part) p.dD_part[b * p.dim + d] = dD_acc;
    if (p.dbias_part) p.dbias_part[b * p.dim + d] = dbias_acc;
  }
}

// The partial sums in a fixed order (bitwise repeatable):
//   dB[b][t][n] = sum over channel blocks cb of dBC_part[cb][b][t][n]      (io dtype)
//   dC[b][t][n] = sum over cb of dBC_part[cb][b][t][NP + n]
//   dA[d][n] = sum over b of dA_part[b][d][n];  dD, ddelta_bias likewise.
// One thread per output; the sums run in index order.
template <typename T, int NP>
__global__ void k_bwd_reduce(BwdParams p) {
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  const int64_t n_bc = p.batch * p.L * p.N;
  const int64_t n_a = p.dim * p.N;
  if (i < n_bc) {
    const int64_t bt = i / p.N;
    const int n = (int)(i - bt * p.N);
    const int64_t stride = p.batch * p.L * 2 * NP;
    const float *src = p.dBC_part + bt * 2 * NP + n;
    float sb = 0.f, sc = 0.f;
    for (int64_t cb = 0; cb < p.n_blocks; ++cb) {
      sb += __ldcs(src + cb * stride);
      sc += __ldcs(src + cb * stride + NP);
    }
    IO<T>::store1(static_cast<T *>(p.dB), i, sb);
    IO<T>::store1(static_cast<T *>(p.dC), i, sc);
    return;
  }
  const int64_t ia = i - n_bc;
  if (ia < n_a) {
    float acc = 0.f;
    for (int64_t b = 0; b < p.batch; ++b) acc += p.dA_part[b * n_a + ia];
    p.dA[ia] = acc;
    return;
  }
  const int64_t id = ia - n_a;
  if (id < p.dim) {
    if (p.dD) {
      float acc = 0.f;
      for (int64_t b = 0; b < p.batch; ++b) acc += p.dD_part[b * p.dim + id];
      p.dD[id] = acc;
    }
    if (p.dbias) {
      float acc = 0.f;
      for (int64_t b = 0; b < p.batch; ++b) acc += p.dbias_part[b * p.dim + id];
      p.dbias[id] = acc;
    }
  }
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
  return (size_t)batch * (size_t)ckpt_groups(dim) * (size_t)ckpt_chunks(L) * kCkptChannels * NP;
}

size_t bwd16_smem_bytes(int io_dtype);
int64_t bwd16_blocks(int64_t dim);
cudaError_t launch_bwd16(int io_dtype, BwdParams &p, cudaStream_t s);

// Channel blocks of the dB/dC partials: 64-channel CTAs of k_bwd16 for
// d_state 16 with the Euler term, 32-channel CTAs of k_bwd otherwise.
// d_state 9..16 (padded to 16) takes the d_state-16 kernel, Euler or exact ZOH
bool bwd_uses_bwd16(int NP, int /*zoh*/) { return NP == 16; }

int64_t bwd_blocks(int64_t dim, int NP, int zoh) {
  return bwd_uses_bwd16(NP, zoh) ? bwd16_blocks(dim) : (dim + kBW * kBCPW - 1) / (kBW * kBCPW);
}

cudaError_t launch_bwd(int io_dtype, int NP, BwdParams &p, cudaStream_t s) {
  p.n_blocks = bwd_blocks(p.dim, NP, p.zoh);
  return bwd_dispatch(io_dtype, NP, [&](auto tt, auto np) -> cudaError_t {
    using T = typename decltype(tt)::type;
    constexpr int kNP = decltype(np)::value;
    cudaError_t e;
    auto general = [&](auto kern) -> cudaError_t {
      p.cpb = (p.dim + kBW * kBCPW - 1) / (kBW * kBCPW);
      p.K = (p.L + kTB - 1) / kTB;
      const size_t smem = sizeof(BwdSmem<kNP>);
      if (smem > 48 * 1024) {
        cudaError_t e2 = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e2 != cudaSuccess) return e2;
      }
      kern<<<(unsigned)(p.batch * p.cpb), kBW * 32, smem, s>>>(p);
      return cudaGetLastError();
    };
    if constexpr (kNP == 16) {
      e = launch_bwd16(io_dtype, p, s);  // Euler and exact ZOH
    } else {
      e = p.zoh ? general(k_bwd<T, kNP, true>) : general(k_bwd<T, kNP, false>);
    }
    if (e != cudaSuccess) return e;
    const int64_t total = p.batch * p.L * p.N + p.dim * p.N + p.dim;
    k_bwd_reduce<T, kNP><<<(unsigned)((total + 255) / 256), 256, 0, s>>>(p);
    return cudaGetLastError();
  });
}

}  // namespace ssm
