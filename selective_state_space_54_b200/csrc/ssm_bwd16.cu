// Backward of the selective scan (S6) for d_state 16, the state size of the
// Mamba layers, sm_100a.
//
// The gradients are those of ssm_bwd.cu (the general kernel, which this one
// replaces for d_state 16):
//   dy_t  = dout_t SiLU(z_t)                 dz_t = dout_t yss_t SiLU'(z_t)
//   g_tn  = dy_t C_tn + a_{t+1,n} g_{t+1,n}  (dL/dh_tn, the reverse recurrence)
//   dC_tn = sum_d dy_t h_tn                  dB_tn = sum_d g_tn Delta_t u_t
//   dA_n  = sum_{b,t} g_tn Delta_t a_tn h_{t-1,n}
//   dDelta_t = sum_n g_tn (A_n a_tn h_{t-1,n} + B_tn u_t),  ddelta_t = dDelta_t sigmoid(s_t)
//   du_t  = dy_t D + Delta_t sum_n g_tn B_tn,  dD = sum dy_t u_t,  ddelta_bias = sum ddelta_t
// With the exact zero-order hold the input term Delta_t u_t B_tn becomes
// u_t W_tn B_tn, W = Delta (e^x - 1)/x with x = Delta A_n (reading guide,
// "Metodo"): dB_tn = sum_d g u W, du_t = dy_t D + sum_n g W B, the input
// term's part of dDelta_t is u_t sum_n g a B, and dA_n gains
// sum g u B Delta^2 psi(x), psi(x) = (x e^x - (e^x - 1))/x^2.
// The states are recomputed from the state entering each 8-step chunk, never
// stored for every step ("Mamba: Linear-Time Sequence Modeling with Selective
// State Spaces" reading guide, "Expansao de Estado Ciente de Hardware":
// intermediate states are recomputed in the backward pass instead of being
// read from HBM).
//
// Work split.  A CTA of 4 warps owns 64 channels of one batch element for the
// whole sequence and walks its 8-step chunks in reverse.  Lane (cg, j) of
// warp w holds channels 16w + 2cg and 16w + 2cg + 1 and, of both, the states
// 4j .. 4j+3, as packed fp32 pairs: per step it handles 8 (channel, state)
// elements.  Holding two channels per lane lets the dB/dC sums over the
// channels start in registers (one FMA per element), and holding 4 states
// keeps B and C one 16-byte shared load each per step.
//
// Per chunk: (1) the inputs of the chunk before are copied ahead into a
// shared-memory ring (cp.async); (2) per (channel, step): Delta, Delta u, dy,
// the softplus and gate derivatives, staged in shared memory as (v, v) pairs;
// (3) the chunk's states are recomputed from its saved entry state and the
// state entering each 2-step group is kept in shared memory (first exp2 per
// element); (4) group by group from the last: the group's 2 states and decays
// are recomputed into registers (second exp2), then the reverse recurrence
// runs over them.  Sums over the 4 lanes of a channel (yss, dDelta, du) and
// over the 8 channel pairs of a warp (dB, dC) are butterfly reduce-scatters;
// the 4 warps' dB/dC sums meet in shared memory.
//
// Every cross-channel and cross-step sum is formed in a fixed order and
// written as a per-block partial (dB/dC per 64-channel block, dA/dD/
// ddelta_bias per batch element); k_bwd_reduce adds the partials in a fixed
// order.  No atomics: two runs give bitwise-equal gradients.
#include "ssm_common.cuh"

namespace ssm {

// Warps per CTA (the code takes 1, 2 or 4).  At the Mamba-1.4B training shape
// (512 CTAs of 4 warps, 3 or 4 per SM) 2-warp CTAs even out the warps per SM
// but measured only 1.3 % faster on B200 (1.874 against 1.899 ms) while
// doubling the dB/dC partials, and 1-warp CTAs 1.9 % slower: the kernel is
// bound by its instruction latency, not by the uneven spread.
constexpr int kQW = 4;
static_assert(kQW == 1 || kQW == 2 || kQW == 4, "1, 2 or 4 warps per CTA");
constexpr int kQC = 16 * kQW;      // channels per CTA
constexpr int kQT = kCkptSteps;    // steps per chunk
constexpr int kQThreads = 32 * kQW;
constexpr float kLn2f = 0.6931471805599453f;
static_assert(kQT == 8, "the group loop below covers 8-step chunks as 4 groups of 2");

// Raw inputs of one chunk.  act[0..3] hold u, delta, z, dout of the CTA's 64
// channels and 8 steps, [channel][step] for channel-major inputs and
// [step][channel] for token-major ones (at(ch, t) gives the index); after
// the pre-pass act[0..2] are reused for du, ddelta, dz.
template <typename T>
struct __align__(16) QRaw {
  T act[4][kQC * kQT];
  T B[kQT][16], C[kQT][16];  // [step][state]
};
template <bool TOK>
__device__ __forceinline__ int at(int ch, int t) { return TOK ? t * kQC + ch : ch * kQT + t; }

struct __align__(16) QStage {
  f2 dl2[kQT][kQC];    // (Delta, Delta)
  f2 du2[kQT][kQC];    // (Delta u, Delta u)
  f2 dy2[kQT][kQC];    // (dy, dy)
  float sg[kQT][kQC];  // d Delta / d delta (sigmoid(s), 1 without softplus, 0 past L)
  float fz[kQT][kQC];  // dz = yss * fz
  float uu[kQT][kQC];  // u (0 past L)
  float Bs[kQT][16];
  float Cs[kQT][16];
};

template <typename T>
struct __align__(16) QSmem {
  QRaw<T> raw[2];
  QStage st;
  float hent[4][kQW][2][32][4];  // state entering group 0..3 of the chunk: [group][warp][channel][lane][4]
  float red[kQT][kQW][32];       // per-warp dB/dC sums of each step
};

// The exact-ZOH instantiation also keeps W = Delta (e^x - 1)/x of the current
// 2-step group, formed while the group's states are recomputed and read back
// by the same thread in its reverse pass: [step][channel][state pair][thread].
// 56 KB per CTA with bf16 io, still 4 CTAs per SM.
template <typename T>
struct __align__(16) QSmemZoh {
  QSmem<T> base;
  f2 wz[2][2][2][kQThreads];
};

__device__ __forceinline__ f2 shfl_xor2(f2 v, int m) {
  float lo, hi;
  unpack2(v, lo, hi);
  lo = __shfl_xor_sync(0xffffffffu, lo, m);
  hi = __shfl_xor_sync(0xffffffffu, hi, m);
  return pack2(lo, hi);
}

__device__ __forceinline__ void q_cp16(void *smem, const void *gmem, int src_bytes) {
  const unsigned sa = static_cast<unsigned>(__cvta_generic_to_shared(smem));
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(sa), "l"(gmem), "r"(src_bytes)
               : "memory");
}
__device__ __forceinline__ void q_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void q_wait_all() { asm volatile("cp.async.wait_group 0;" ::: "memory"); }

// Copy the raw inputs of chunk k into `raw`: u and delta (and z, dout when
// FULL) of the CTA's channels, and B (and C) [8][16].  Steps past L are zero
// filled; channels past dim read nothing.  Channel-major rows are 8 steps of
// one channel; token-major rows are 64 channels of one step (dim % 8 == 0, so
// a 16-byte piece of 8 channels is either inside dim or past it).
template <typename T, bool FULL, bool TOK>
__device__ __forceinline__ void q_fetch(const BwdParams &p, QRaw<T> &raw, int64_t b, int64_t cb, int64_t k) {
  constexpr int ES = (int)sizeof(T), EPP = 16 / ES;
  const int tid = threadIdx.x;
  const int64_t L = p.L, t0 = k * kQT;
  const int64_t left = L - t0;  // >= 1
  constexpr int NA = FULL ? 4 : 2;
  auto src_of = [&](int a) -> const T * {
    return static_cast<const T *>(a == 0 ? p.u : a == 1 ? p.delta : a == 2 ? p.z : p.dout);
  };
  if (TOK) {
    constexpr int PPS = kQC / EPP;  // pieces per step row
    for (int v = tid; v < NA * kQT * PPS; v += kQThreads) {
      const int a = v / (kQT * PPS), rest = v - a * (kQT * PPS), t = rest / PPS, q = rest - t * PPS;
      const int64_t d = cb * kQC + q * EPP;
      const T *src = src_of(a);
      const bool in = src && t < left && d < p.dim;
      q_cp16(&raw.act[a][t * kQC + q * EPP], in ? src + ((b * L + t0 + t) * p.dim + d) : static_cast<const T *>(p.u),
             in ? 16 : 0);
    }
  } else if (p.io_vec) {
    constexpr int PPR = kQT / EPP;  // pieces per channel row
    for (int v = tid; v < kQC * NA * PPR; v += kQThreads) {
      const int ch = v / (NA * PPR), rest = v - ch * (NA * PPR), a = rest / PPR, q = rest - a * PPR;
      const int64_t d = cb * kQC + ch;
      const T *src = src_of(a);
      T *dst = &raw.act[a][ch * kQT + q * EPP];
      const int64_t n_in = left - q * EPP;  // steps of this piece inside L
      const int bytes = (d < p.dim && src) ? (n_in >= EPP ? 16 : (n_in > 0 ? (int)n_in * ES : 0)) : 0;
      const T *g = bytes ? src + ((b * p.dim + d) * L + t0 + q * EPP) : static_cast<const T *>(p.u);
      q_cp16(dst, g, bytes);
    }
  } else {
    for (int v = tid; v < kQC * NA * kQT; v += kQThreads) {
      const int ch = v / (NA * kQT), rest = v - ch * (NA * kQT), a = rest / kQT, t = rest - a * kQT;
      const int64_t d = cb * kQC + ch;
      const T *src = src_of(a);
      raw.act[a][ch * kQT + t] = (d < p.dim && src && t < left) ? src[(b * p.dim + d) * L + t0 + t] : T(0);
    }
  }
  // B and C: [8][16] blocks, contiguous in [batch][L][16]
  constexpr int NB = FULL ? 2 : 1;
  if (p.bc_vec) {
    constexpr int PB = kQT * 16 / EPP;  // pieces per tensor
    for (int v = tid; v < NB * PB; v += kQThreads) {
      const int a = v / PB, q = v - a * PB;
      const int t = q * EPP / 16;
      const T *src = a ? static_cast<const T *>(p.C) : static_cast<const T *>(p.B);
      T *dst = (a ? &raw.C[0][0] : &raw.B[0][0]) + q * EPP;
      const bool in = t < left;
      q_cp16(dst, in ? src + (b * L + t0) * 16 + q * EPP : src, in ? 16 : 0);
    }
  } else {
    for (int v = tid; v < NB * kQT * 16; v += kQThreads) {
      const int a = v / (kQT * 16), e = v - a * (kQT * 16), t = e / 16, n = e - t * 16;
      const T *src = a ? static_cast<const T *>(p.C) : static_cast<const T *>(p.B);
      const bool in = t < left && n < p.N;
      (a ? &raw.C[0][0] : &raw.B[0][0])[e] = in ? src[(b * L + t0 + t) * p.N + n] : T(0);
    }
  }
  q_commit();
}

__device__ __forceinline__ float q_f(uint16_t v) { return bf16_to_f(v); }
__device__ __forceinline__ float q_f(float v) { return v; }
__device__ __forceinline__ void q_put(uint16_t &dst, float v) {
  const __nv_bfloat16 h = __float2bfloat16_rn(v);
  dst = *reinterpret_cast<const uint16_t *>(&h);
}
__device__ __forceinline__ void q_put(float &dst, float v) { dst = v; }

// Per (channel, step) quantities of chunk k into the stage.  FULL adds what
// the reverse pass needs (dy, the gate and softplus derivatives, u).  ZOH:
// the (v, v) row du2 holds u instead of Delta u.
// Thread tid takes channel tid / 2 and steps 4 (tid % 2) .. +3.  Returns this
// thread's contribution to dD (sum of dy u).
template <typename T, bool FULL, bool TOK, bool ZOH>
__device__ __forceinline__ float q_prepass(const BwdParams &p, QRaw<T> &raw, QStage &st, int64_t cb,
                                           int64_t k, float bias, float Dd) {
  const int tid = threadIdx.x, pc = tid >> 1, t4 = (tid & 1) * 4;
  const int64_t d = cb * kQC + pc;
  const bool dvalid = d < p.dim;
  const int64_t t0 = k * kQT;
  const bool has_z = p.z != nullptr;
  float dD = 0.f;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int t = t4 + i;
    const bool in = dvalid && t0 + t < p.L;
    const float u = in ? q_f(raw.act[0][at<TOK>(pc, t)]) : 0.f;
    const float s = q_f(raw.act[1][at<TOK>(pc, t)]) + bias;
    float dl = s, sg = 1.f;
    if (p.softplus) {
      // softplus(s) = max(s, 0) + log1p(x), sigmoid(s) = (s >= 0 ? 1 : x) / (1 + x), x = exp(-|s|)
      const float x = ex2(-fabsf(s) * kLog2e);
      dl = softplus_fast(s);
      sg = __fdividef(s >= 0.f ? 1.f : x, 1.f + x);
    }
    dl = in ? dl : 0.f;
    st.dl2[t][pc] = splat2(dl);
    st.du2[t][pc] = splat2(ZOH ? u : dl * u);
    if (FULL) {
      const float o = in ? q_f(raw.act[3][at<TOK>(pc, t)]) : 0.f;
      float dy = o, fz = 0.f;
      if (has_z) {
        const float z = q_f(raw.act[2][at<TOK>(pc, t)]);
        const float sz = __fdividef(1.f, 1.f + ex2(-z * kLog2e));
        dy = o * z * sz;
        fz = o * sz * fmaf(z, 1.f - sz, 1.f);
      }
      st.dy2[t][pc] = splat2(dy);
      st.sg[t][pc] = in ? sg : 0.f;
      st.fz[t][pc] = fz;
      st.uu[t][pc] = u;
      dD = fmaf(dy, u, dD);
    }
  }
  // B (and C) widened to fp32, 4 values per thread
  for (int v = tid; v < (FULL ? 64 : 32); v += kQThreads) {
    const int e = (v & 31) * 4, t = e >> 4, n = e & 15;
    const T *src = (v >> 5) ? &raw.C[t][n] : &raw.B[t][n];
    float *dst = (v >> 5) ? &st.Cs[t][n] : &st.Bs[t][n];
    *reinterpret_cast<float4 *>(dst) = make_float4(q_f(src[0]), q_f(src[1]), q_f(src[2]), q_f(src[3]));
  }
  (void)Dd;
  return dD;
}

// ZOH: the exact zero-order-hold input term u W B, W = Delta (e^x - 1)/x
// (zoh_w / zoh_y, ssm_common.cuh), a separate instantiation
template <typename T, bool TOK, bool ZOH>
__global__ void __launch_bounds__(kQThreads, 16 / kQW) k_bwd16(BwdParams p) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  QSmem<T> &sm = *reinterpret_cast<QSmem<T> *>(smem_raw);  // the ZOH layout starts with it
  f2 (*const wz)[2][2][kQThreads] = reinterpret_cast<QSmemZoh<T> *>(smem_raw)->wz;  // ZOH only
  QStage &st = sm.st;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int cg = lane >> 2, j = lane & 3;
  const int64_t cb = blockIdx.x % p.cpb, b = blockIdx.x / p.cpb;
  const int64_t L = p.L, Dm = p.dim;
  const int64_t K = ckpt_chunks(L);
  const int ch0 = warp * 16 + 2 * cg;  // the lane's first channel within the CTA
  const int64_t d0 = cb * kQC + ch0;
  bool cvalid[2];
  float Dd[2];
#pragma unroll
  for (int c = 0; c < 2; ++c) {
    cvalid[c] = d0 + c < Dm;
    Dd[c] = (p.D && cvalid[c]) ? p.D[d0 + c] : 0.f;
  }
  // A * log2(e) of the lane's states, per channel, as pairs
  f2 A2[2][2];
  f2 rA[2][2];  // exact ZOH only: 1 / A_n (infinite for A_n = 0, whose x is 0)
#pragma unroll
  for (int c = 0; c < 2; ++c)
#pragma unroll
    for (int q = 0; q < 2; ++q) {
      const int n = 4 * j + 2 * q;  // padded states (n >= N) have A = B = C = 0
      const float a0 = (cvalid[c] && n < p.N) ? p.A[(d0 + c) * p.N + n] : 0.f;
      const float a1 = (cvalid[c] && n + 1 < p.N) ? p.A[(d0 + c) * p.N + n + 1] : 0.f;
      A2[c][q] = pack2(a0 * kLog2e, a1 * kLog2e);
      if constexpr (ZOH) rA[c][q] = pack2(__frcp_rn(a0), __frcp_rn(a1));
    }
  // the pre-pass thread's channel
  const int64_t pd = cb * kQC + (tid >> 1);
  const float pbias = (p.bias && pd < Dm) ? p.bias[pd] : 0.f;
  const float pD = (p.D && pd < Dm) ? p.D[pd] : 0.f;

  auto ld_pairs = [&](const f2 (*arr)[kQC], int t, f2 &x0, f2 &x1) {
    const ulonglong2 v = *reinterpret_cast<const ulonglong2 *>(&arr[t][ch0]);
    x0 = v.x;
    x1 = v.y;
  };
  auto ld_state_pairs = [&](const float (*arr)[16], int t, f2 &x0, f2 &x1) {
    const ulonglong2 v = *reinterpret_cast<const ulonglong2 *>(&arr[t][4 * j]);
    x0 = v.x;
    x1 = v.y;
  };
  // the input term of state pair (c, q): Delta u B (Euler; du = Delta u) or
  // u W B (exact ZOH; du = u); xx = Delta A log2(e), a = its exp2
  auto bterm = [&](f2 dl, f2 du, f2 xx, f2 a, int c, int q, f2 Bq) -> f2 {
    if constexpr (ZOH) return mul2(mul2(du, zoh_w(xx, a, dl, rA[c][q])), Bq);
    else return mul2(du, Bq);
  };
  float *ck_base[2];
#pragma unroll
  for (int c = 0; c < 2; ++c) ck_base[c] = p.ckpt + ckpt_offset(b, d0 + c, 0, Dm, L, 16) + 4 * j;
  constexpr int64_t kCkStride = kCkptChannels * 16;  // floats between consecutive chunks

  // ---- phase A: the state entering every chunk, unless the forward saved them ----
  if (!p.ckpt_given) {
    f2 h[2][2];
#pragma unroll
    for (int c = 0; c < 2; ++c)
#pragma unroll
      for (int q = 0; q < 2; ++q) {
        float v0 = 0.f, v1 = 0.f;
        const int n = 4 * j + 2 * q;
        if (p.h0 && cvalid[c]) {
          if (n < p.N) v0 = p.h0[(b * Dm + d0 + c) * p.N + n];
          if (n + 1 < p.N) v1 = p.h0[(b * Dm + d0 + c) * p.N + n + 1];
        }
        h[c][q] = pack2(v0, v1);
      }
    q_fetch<T, false, TOK>(p, sm.raw[0], b, cb, 0);
    for (int64_t k = 0; k < K; ++k) {
      q_wait_all();
      __syncthreads();
      if (k + 1 < K) q_fetch<T, false, TOK>(p, sm.raw[(k + 1) & 1], b, cb, k + 1);
      q_prepass<T, false, TOK, ZOH>(p, sm.raw[k & 1], st, cb, k, pbias, pD);
      __syncthreads();
#pragma unroll
      for (int c = 0; c < 2; ++c)
        *reinterpret_cast<ulonglong2 *>(ck_base[c] + k * kCkStride) = make_ulonglong2(h[c][0], h[c][1]);
#pragma unroll
      for (int t = 0; t < kQT; ++t) {
        f2 dl[2], du[2], B[2];
        ld_pairs(st.dl2, t, dl[0], dl[1]);
        ld_pairs(st.du2, t, du[0], du[1]);
        ld_state_pairs(st.Bs, t, B[0], B[1]);
#pragma unroll
        for (int c = 0; c < 2; ++c)
#pragma unroll
          for (int q = 0; q < 2; ++q) {
            const f2 xx = mul2(dl[c], A2[c][q]);
            float x0, x1;
            unpack2(xx, x0, x1);
            const f2 a = pack2(ex2(x0), ex2(x1));
            h[c][q] = fma2(a, h[c][q], bterm(dl[c], du[c], xx, a, c, q, B[q]));
          }
      }
    }
    q_wait_all();
    __syncthreads();
  }

  // ---- phase B: chunks in reverse ----
  f2 g[2][2], dA[2][2];
#pragma unroll
  for (int c = 0; c < 2; ++c)
#pragma unroll
    for (int q = 0; q < 2; ++q) g[c][q] = dA[c][q] = pack2(0.f, 0.f);
  float dD_acc = 0.f, dbias_acc = 0.f;
  // the (channel, step) of a group this lane finalises: channel ch0 + (j & 1), step t0 + (j >> 1)
  const int my_c = j & 1, my_s = j >> 1;
  const bool hi16 = (lane & 16) != 0, hi8 = (lane & 8) != 0, hi4 = (lane & 4) != 0;
  const int my_out = (hi16 ? 16 : 0) + 4 * j + (hi8 ? 2 : 0) + (hi4 ? 1 : 0);  // dB/dC output of this lane

  q_fetch<T, true, TOK>(p, sm.raw[(K - 1) & 1], b, cb, K - 1);
  for (int64_t k = K - 1; k >= 0; --k) {
    QRaw<T> &raw = sm.raw[k & 1];
    const int64_t t0 = k * kQT;
    q_wait_all();
    __syncthreads();
    if (k > 0) q_fetch<T, true, TOK>(p, sm.raw[(k - 1) & 1], b, cb, k - 1);
    dD_acc += q_prepass<T, true, TOK, ZOH>(p, raw, st, cb, k, pbias, pD);
    __syncthreads();

    // (3) the chunk's states from its entry state; keep the entry of every 2-step group
    {
      f2 h[2][2];
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        const ulonglong2 v = cvalid[c] ? __ldcg(reinterpret_cast<const ulonglong2 *>(ck_base[c] + k * kCkStride))
                                       : make_ulonglong2(0ull, 0ull);
        h[c][0] = v.x;
        h[c][1] = v.y;
      }
#pragma unroll
      for (int t = 0; t < kQT - 2; ++t) {
        if ((t & 1) == 0) {
#pragma unroll
          for (int c = 0; c < 2; ++c)
            *reinterpret_cast<ulonglong2 *>(&sm.hent[t >> 1][warp][c][lane][0]) = make_ulonglong2(h[c][0], h[c][1]);
        }
        f2 dl[2], du[2], B[2];
        ld_pairs(st.dl2, t, dl[0], dl[1]);
        ld_pairs(st.du2, t, du[0], du[1]);
        ld_state_pairs(st.Bs, t, B[0], B[1]);
#pragma unroll
        for (int c = 0; c < 2; ++c)
#pragma unroll
          for (int q = 0; q < 2; ++q) {
            const f2 xx = mul2(dl[c], A2[c][q]);
            float x0, x1;
            unpack2(xx, x0, x1);
            const f2 a = pack2(ex2(x0), ex2(x1));
            h[c][q] = fma2(a, h[c][q], bterm(dl[c], du[c], xx, a, c, q, B[q]));
          }
      }
#pragma unroll
      for (int c = 0; c < 2; ++c)
        *reinterpret_cast<ulonglong2 *>(&sm.hent[3][warp][c][lane][0]) = make_ulonglong2(h[c][0], h[c][1]);
    }

    // (4) groups of 2 steps, last first
#pragma unroll 1
    for (int gi = kQT / 2 - 1; gi >= 0; --gi) {
      const int tg = 2 * gi;
      f2 he[2][2], hs[2][2][2], as[2][2][2];
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        const ulonglong2 v = *reinterpret_cast<const ulonglong2 *>(&sm.hent[gi][warp][c][lane][0]);
        he[c][0] = v.x;
        he[c][1] = v.y;
      }
      float yv[2][2];
#pragma unroll
      for (int s = 0; s < 2; ++s) {
        const int t = tg + s;
        f2 dl[2], du[2], B[2], C[2];
        ld_pairs(st.dl2, t, dl[0], dl[1]);
        ld_pairs(st.du2, t, du[0], du[1]);
        ld_state_pairs(st.Bs, t, B[0], B[1]);
        ld_state_pairs(st.Cs, t, C[0], C[1]);
#pragma unroll
        for (int c = 0; c < 2; ++c) {
#pragma unroll
          for (int q = 0; q < 2; ++q) {
            const f2 xx = mul2(dl[c], A2[c][q]);
            float x0, x1;
            unpack2(xx, x0, x1);
            as[s][c][q] = pack2(ex2(x0), ex2(x1));
            if constexpr (ZOH) {  // W kept for the reverse pass
              const f2 W = zoh_w(xx, as[s][c][q], dl[c], rA[c][q]);
              wz[s][c][q][tid] = W;
              hs[s][c][q] = fma2(as[s][c][q], s ? hs[0][c][q] : he[c][q], mul2(mul2(du[c], W), B[q]));
            } else {
              hs[s][c][q] = fma2(as[s][c][q], s ? hs[0][c][q] : he[c][q],
                                 bterm(dl[c], du[c], xx, as[s][c][q], c, q, B[q]));
            }
          }
          float lo, hi;
          unpack2(fma2(C[1], hs[s][c][1], mul2(C[0], hs[s][c][0])), lo, hi);
          yv[s][c] = lo + hi;
        }
      }
      // C.h summed over the channel's 4 lanes; lane j keeps (channel j & 1, step j >> 1)
      {
        const bool up = (j & 2) != 0;
        float k0 = up ? yv[1][0] : yv[0][0], k1 = up ? yv[1][1] : yv[0][1];
        k0 += __shfl_xor_sync(0xffffffffu, up ? yv[0][0] : yv[1][0], 2);
        k1 += __shfl_xor_sync(0xffffffffu, up ? yv[0][1] : yv[1][1], 2);
        float yss = my_c ? k1 : k0;
        yss += __shfl_xor_sync(0xffffffffu, my_c ? k0 : k1, 1);
        const int t = tg + my_s, ch = ch0 + my_c;
        yss = fmaf(my_c ? Dd[1] : Dd[0], st.uu[t][ch], yss);
        q_put(raw.act[2][at<TOK>(ch, t)], yss * st.fz[t][ch]);
      }
      // the reverse recurrence over the group's 2 steps
      float ddv[2][2], s1v[2][2], s2v[2][2];  // s2v: exact ZOH only
#pragma unroll
      for (int s = 1; s >= 0; --s) {
        const int t = tg + s;
        f2 dl[2], du[2], dy[2], B[2], C[2];
        ld_pairs(st.dl2, t, dl[0], dl[1]);
        ld_pairs(st.du2, t, du[0], du[1]);
        ld_pairs(st.dy2, t, dy[0], dy[1]);
        ld_state_pairs(st.Bs, t, B[0], B[1]);
        ld_state_pairs(st.Cs, t, C[0], C[1]);
        f2 dBp[2], dCp[2];
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          f2 dd, s1, s2;
#pragma unroll
          for (int q = 0; q < 2; ++q) {
            g[c][q] = fma2(dy[c], C[q], g[c][q]);
            dCp[q] = c ? fma2(dy[c], hs[s][c][q], dCp[q]) : mul2(dy[c], hs[s][c][q]);
            if constexpr (ZOH) {
              // input term u W B: its u derivative W B (s1 = sum_n g W B is du's sum,
              // Delta included), its B derivative u W, its A derivative u Y B
              const f2 xx = mul2(dl[c], A2[c][q]);
              const f2 W = wz[s][c][q][tid];  // from the group's recomputation
              const f2 gB = mul2(g[c][q], B[q]);
              s1 = q ? fma2(gB, W, s1) : mul2(gB, W);
              const f2 uW = mul2(du[c], W);
              dBp[q] = c ? fma2(g[c][q], uW, dBp[q]) : mul2(g[c][q], uW);
              dA[c][q] = fma2(mul2(gB, zoh_y(xx, as[s][c][q], W, dl[c], rA[c][q])), du[c], dA[c][q]);
            } else {
              s1 = q ? fma2(g[c][q], B[q], s1) : mul2(g[c][q], B[q]);
              dBp[q] = c ? fma2(g[c][q], du[c], dBp[q]) : mul2(g[c][q], du[c]);
            }
            // g a_t is both dL/dh_{t-1} and the factor of h_{t-1} in dA and dDelta
            g[c][q] = mul2(g[c][q], as[s][c][q]);
            // exact ZOH: the input term's Delta derivative is a u B (s2 = sum_n g a B)
            if constexpr (ZOH) s2 = q ? fma2(g[c][q], B[q], s2) : mul2(g[c][q], B[q]);
            const f2 qv = mul2(g[c][q], s ? hs[0][c][q] : he[c][q]);  // g a_t h_{t-1}
            dA[c][q] = fma2(dl[c], qv, dA[c][q]);
            dd = q ? fma2(A2[c][q], qv, dd) : mul2(A2[c][q], qv);
          }
          float lo, hi;
          unpack2(dd, lo, hi);
          ddv[s][c] = lo + hi;
          unpack2(s1, lo, hi);
          s1v[s][c] = lo + hi;
          if constexpr (ZOH) {
            unpack2(s2, lo, hi);
            s2v[s][c] = lo + hi;
          }
        }
        // dB, dC over the warp's 8 channel pairs: lane keeps output my_out
        f2 k0 = hi16 ? dCp[0] : dBp[0], k1 = hi16 ? dCp[1] : dBp[1];
        k0 = add2(k0, shfl_xor2(hi16 ? dBp[0] : dCp[0], 16));
        k1 = add2(k1, shfl_xor2(hi16 ? dBp[1] : dCp[1], 16));
        f2 kk = hi8 ? k1 : k0;
        kk = add2(kk, shfl_xor2(hi8 ? k0 : k1, 8));
        float lo, hi;
        unpack2(kk, lo, hi);
        float v = hi4 ? hi : lo;
        v += __shfl_xor_sync(0xffffffffu, hi4 ? lo : hi, 4);
        sm.red[t][warp][my_out] = v;
      }
      // dDelta and sum_n g B over the channel's 4 lanes; lane j keeps (channel j & 1, step j >> 1)
      {
        const bool up = (j & 2) != 0;
        float a0 = up ? ddv[1][0] : ddv[0][0], a1 = up ? ddv[1][1] : ddv[0][1];
        float b0 = up ? s1v[1][0] : s1v[0][0], b1 = up ? s1v[1][1] : s1v[0][1];
        a0 += __shfl_xor_sync(0xffffffffu, up ? ddv[0][0] : ddv[1][0], 2);
        a1 += __shfl_xor_sync(0xffffffffu, up ? ddv[0][1] : ddv[1][1], 2);
        b0 += __shfl_xor_sync(0xffffffffu, up ? s1v[0][0] : s1v[1][0], 2);
        b1 += __shfl_xor_sync(0xffffffffu, up ? s1v[0][1] : s1v[1][1], 2);
        float ddsum = my_c ? a1 : a0, s1sum = my_c ? b1 : b0;
        ddsum += __shfl_xor_sync(0xffffffffu, my_c ? a0 : a1, 1);
        s1sum += __shfl_xor_sync(0xffffffffu, my_c ? b0 : b1, 1);
        // exact ZOH: the Delta derivative's input part is u sum_n g a B (s2)
        float s2sum = s1sum;
        if constexpr (ZOH) {
          float e0 = up ? s2v[1][0] : s2v[0][0], e1 = up ? s2v[1][1] : s2v[0][1];
          e0 += __shfl_xor_sync(0xffffffffu, up ? s2v[0][0] : s2v[1][0], 2);
          e1 += __shfl_xor_sync(0xffffffffu, up ? s2v[0][1] : s2v[1][1], 2);
          s2sum = my_c ? e1 : e0;
          s2sum += __shfl_xor_sync(0xffffffffu, my_c ? e0 : e1, 1);
        }
        const int t = tg + my_s, ch = ch0 + my_c;
        float dlv, dlv_hi, dyv, dyv_hi;
        unpack2(st.dl2[t][ch], dlv, dlv_hi);
        unpack2(st.dy2[t][ch], dyv, dyv_hi);
        // du = Delta sum g B + D dy (Euler); sum g W B + D dy (exact ZOH: W holds Delta)
        const float du_v = fmaf(ZOH ? 1.f : dlv, s1sum, dyv * (my_c ? Dd[1] : Dd[0]));
        const float ddl = st.sg[t][ch] * fmaf(st.uu[t][ch], s2sum, kLn2f * ddsum);
        q_put(raw.act[0][at<TOK>(ch, t)], du_v);
        q_put(raw.act[1][at<TOK>(ch, t)], ddl);
        dbias_acc += ddl;
      }
    }
    __syncthreads();
    // dB/dC of the chunk: the warps' sums, one partial per block of kQC channels
#pragma unroll
    for (int r = 0; r < kQT / kQW; ++r) {
      const int t = warp + kQW * r, out = lane;
      if (t0 + t < L) {
        float v = sm.red[t][0][out];
        if constexpr (kQW == 2) v += sm.red[t][1][out];
        if constexpr (kQW == 4) v = (v + sm.red[t][1][out]) + (sm.red[t][2][out] + sm.red[t][3][out]);
        p.dBC_part[((cb * p.batch + b) * L + t0 + t) * 32 + out] = v;
      }
    }
    // du, ddelta, dz rows of the chunk
    if (TOK) {  // [step][64 channels] rows, 16-byte pieces of 8 channels
      constexpr int EPP = 16 / (int)sizeof(T), PPS = kQC / EPP;
      for (int v = tid; v < 3 * kQT * PPS; v += kQThreads) {
        const int a = v / (kQT * PPS), rest = v - a * (kQT * PPS), t = rest / PPS, q = rest - t * PPS;
        const int64_t d = cb * kQC + q * EPP;
        if (t0 + t < L && d < Dm && (a != 2 || p.dz)) {
          T *dst = static_cast<T *>(a == 0 ? p.du : a == 1 ? p.ddelta : p.dz) + (b * L + t0 + t) * Dm + d;
          *reinterpret_cast<uint4 *>(dst) = *reinterpret_cast<const uint4 *>(&raw.act[a][t * kQC + q * EPP]);
        }
      }
    } else {
      const int ch = tid >> 1, half = tid & 1;
      const int64_t d = cb * kQC + ch;
      if (d < Dm) {
#pragma unroll
        for (int a = 0; a < 3; ++a) {
          if ((a & 1) != half || (a == 2 && !p.dz)) continue;
          T *row = static_cast<T *>(a == 0 ? p.du : a == 1 ? p.ddelta : p.dz) + (b * Dm + d) * L + t0;
          const T *src = &raw.act[a][ch * kQT];
          constexpr int ES = (int)sizeof(T), EPP = 16 / ES;
          if (p.io_vec && t0 + kQT <= L) {
#pragma unroll
            for (int q = 0; q < kQT / EPP; ++q)
              *reinterpret_cast<uint4 *>(row + q * EPP) = *reinterpret_cast<const uint4 *>(src + q * EPP);
          } else {
            for (int t = 0; t < kQT && t0 + t < L; ++t) row[t] = src[t];
          }
        }
      }
    }
  }

  // ---- per-channel results ----
  dD_acc += __shfl_xor_sync(0xffffffffu, dD_acc, 1);  // the pre-pass pair of a channel
  if ((tid & 1) == 0 && pd < Dm) {
    if (p.dD_part) p.dD_part[b * Dm + pd] = dD_acc;
  }
  dbias_acc += __shfl_xor_sync(0xffffffffu, dbias_acc, 2);  // lanes j and j ^ 2 share a channel
#pragma unroll
  for (int c = 0; c < 2; ++c) {
    if (!cvalid[c]) continue;
    const int64_t d = d0 + c;
    if ((j & 2) == 0 && my_c == c && p.dbias_part) p.dbias_part[b * Dm + d] = dbias_acc;
    float v[4], w[4];
    unpack2(dA[c][0], v[0], v[1]);
    unpack2(dA[c][1], v[2], v[3]);
    unpack2(g[c][0], w[0], w[1]);
    unpack2(g[c][1], w[2], w[3]);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int n = 4 * j + i;
      if (n < p.N) {
        p.dA_part[(b * Dm + d) * p.N + n] = v[i];
        if (p.dh0) p.dh0[(b * Dm + d) * p.N + n] = w[i];
      }
    }
  }
}

size_t bwd16_smem_bytes(int io_dtype) {
  return io_dtype == 1 ? sizeof(QSmem<uint16_t>) : sizeof(QSmem<float>);
}

int64_t bwd16_blocks(int64_t dim) { return (dim + kQC - 1) / kQC; }

cudaError_t launch_bwd16(int io_dtype, BwdParams &p, cudaStream_t s) {
  p.cpb = bwd16_blocks(p.dim);
  auto go = [&](auto kern, size_t smem) -> cudaError_t {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    kern<<<(unsigned)(p.batch * p.cpb), kQThreads, smem, s>>>(p);
    return cudaGetLastError();
  };
  if (p.tok && p.zoh) return cudaErrorInvalidValue;  // no forward writes that combination
  if (io_dtype == 1) {
    if (p.tok) return go(k_bwd16<uint16_t, true, false>, sizeof(QSmem<uint16_t>));
    return p.zoh ? go(k_bwd16<uint16_t, false, true>, sizeof(QSmemZoh<uint16_t>))
                 : go(k_bwd16<uint16_t, false, false>, sizeof(QSmem<uint16_t>));
  }
  if (io_dtype == 0 && !p.tok)
    return p.zoh ? go(k_bwd16<float, false, true>, sizeof(QSmemZoh<float>))
                 : go(k_bwd16<float, false, false>, sizeof(QSmem<float>));
  return cudaErrorInvalidValue;
}

}  // namespace ssm
