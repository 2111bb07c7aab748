// Forward selective scan (S6) kernels for sm_100a.
//
// What is computed (per batch element b, channel d, state n, step t):
//   Delta_t = softplus(delta_t + delta_bias[d])          reading guide of
//             "Mamba: Linear-Time Sequence Modeling with Selective State
//             Spaces", section "O Mecanismo de Selecao (S6)"
//   a_tn    = exp(Delta_t * A[d,n])                       section "Metodo" (ZOH)
//   h_tn    = a_tn * h_{t-1,n} + Delta_t * B[b,t,n] * u_t Euler input term, as in
//             the selective_scan example of "Как работает Mamba (State Space
//             Model)..." (aivaro.ru), section 3
//   y_t     = (sum_n C[b,t,n] h_tn + D[d] u_t) * SiLU(z_t)  "O que e um modelo
//             Mamba?" (ibm.com), output equation and block walk-through
//
// Design (B200): the path is bound by the special-function unit (one exp2 per
// (t, n) element) and issue slots, not by HBM.  So each lane walks the
// recurrence sequentially in time over a few states of one channel: per
// element one MUFU ex2 and four fp32 ops (Delta*A, Delta*u*B, the state FMA,
// the C contraction FMA), which is the minimum.  The reading guide's "parallel
// associative scan" is used where time has to be split across warps: the
// split-L schedule combines segment end states with the operator
// (a, b) o (a', b') = (a a', a' b + b'), and the look-back schedule hands a
// state across two warps.  Quantities computed once per (channel, step)
// (softplus, Delta*u, the gate) are staged through shared memory so that the
// four lanes of a channel share them; B and C chunks are widened to fp32 in
// shared memory once per warp and read back as broadcasts.  Nothing of size
// (L, N) is ever written to global memory.
#include "ssm_common.cuh"

namespace ssm {

template <int NP>
struct __align__(16) FwdSmem {
  float dl[kCPW][kT + kRowPad];   // Delta
  float dlu[kCPW][kT + kRowPad];  // Delta * u
  float ys[kCPW][kT + kRowPad];   // sum_n C h (reduced over the channel's lanes)
  float Bs[kT][NP];               // B chunk, fp32, zero padded
  float Cs[kT][NP];               // C chunk
};

template <int S>
__device__ __forceinline__ void lds_vec(const float *p, float (&v)[S]) {
  if constexpr (S % 4 == 0) {
#pragma unroll
    for (int i = 0; i < S; i += 4) {
      const float4 x = *reinterpret_cast<const float4 *>(p + i);
      v[i] = x.x; v[i + 1] = x.y; v[i + 2] = x.z; v[i + 3] = x.w;
    }
  } else if constexpr (S == 2) {
    const float2 x = *reinterpret_cast<const float2 *>(p);
    v[0] = x.x; v[1] = x.y;
  } else {
    v[0] = p[0];
  }
}

// The 4 lanes j = 0..3 of a channel each hold partial sums y0..y3 for 4
// consecutive steps; lane j returns the full sum for step j (2 shuffle rounds).
__device__ __forceinline__ float reduce4_transpose(float y0, float y1, float y2, float y3, int j) {
  const bool hi2 = (j & 2) != 0;
  float ka = hi2 ? y2 : y0, kb = hi2 ? y3 : y1;
  const float sa = hi2 ? y0 : y2, sb = hi2 ? y1 : y3;
  ka += __shfl_xor_sync(0xffffffffu, sa, 2);
  kb += __shfl_xor_sync(0xffffffffu, sb, 2);
  const bool hi1 = (j & 1) != 0;
  float k = hi1 ? kb : ka;
  const float s = hi1 ? ka : kb;
  k += __shfl_xor_sync(0xffffffffu, s, 1);
  return k;
}

// B or C chunk [t0, t0 + kT) of one batch element into smem as fp32 [t][n],
// zero for n >= N or t >= L.
template <typename T, int NP>
__device__ __forceinline__ void stage_bc(float (*dst)[NP], const T *src, int64_t t0, int64_t L,
                                         int N, bool vec, int lane) {
  constexpr int EPV = 16 / (int)sizeof(T);
  if constexpr (NP % EPV == 0) {
    if (vec) {  // N == NP and every 16-byte vector lies inside one row
      constexpr int NV = kT * NP / EPV;
#pragma unroll
      for (int v = lane; v < NV; v += 32) {
        const int e = v * EPV, t = e / NP, n = e - t * NP;
        float o[EPV];
        if (t0 + t < L) {
          const T *ps = src + (t0 + t) * NP + n;
          if constexpr (sizeof(T) == 2) {
            const uint4 x = __ldg(reinterpret_cast<const uint4 *>(ps));
            o[0] = bf16_lo(x.x); o[1] = bf16_hi(x.x); o[2] = bf16_lo(x.y); o[3] = bf16_hi(x.y);
            o[4] = bf16_lo(x.z); o[5] = bf16_hi(x.z); o[6] = bf16_lo(x.w); o[7] = bf16_hi(x.w);
          } else {
            const float4 x = __ldg(reinterpret_cast<const float4 *>(ps));
            o[0] = x.x; o[1] = x.y; o[2] = x.z; o[3] = x.w;
          }
        } else {
#pragma unroll
          for (int i = 0; i < EPV; ++i) o[i] = 0.f;
        }
#pragma unroll
        for (int i = 0; i < EPV; i += 4)
          *reinterpret_cast<float4 *>(&dst[t][n + i]) = make_float4(o[i], o[i + 1], o[i + 2], o[i + 3]);
      }
      return;
    }
  }
  for (int e = lane; e < kT * NP; e += 32) {
    const int t = e / NP, n = e - t * NP;
    dst[t][n] = (n < N && t0 + t < L) ? IO<T>::get(src, (t0 + t) * N + n) : 0.f;
  }
}

// Per-lane view of an 8-channel group.
struct Lane {
  int lane, c, j;
  int64_t b, d;
  bool valid;
};

__device__ __forceinline__ Lane lane_of(const FwdParams &p, int64_t g) {
  Lane r;
  r.lane = threadIdx.x & 31;
  r.c = r.lane >> 2;
  r.j = r.lane & 3;
  r.b = g / p.gpb;
  r.d = (g - r.b * p.gpb) * kCPW + r.c;
  r.valid = r.d < p.dim;
  return r;
}

template <int NP>
__device__ __forceinline__ void init_state(const FwdParams &p, const Lane &ln, float (&h)[NP / 4]) {
  constexpr int S = NP / 4;
#pragma unroll
  for (int s = 0; s < S; ++s) {
    const int n = ln.j * S + s;
    h[s] = (p.h0 && ln.valid && n < p.N) ? p.h0[(ln.b * p.dim + ln.d) * p.N + n] : 0.f;
  }
}

template <int NP>
__device__ __forceinline__ void write_last_state(const FwdParams &p, const Lane &ln,
                                                 const float (&h)[NP / 4]) {
  constexpr int S = NP / 4;
  if (!p.last_state || !ln.valid) return;
#pragma unroll
  for (int s = 0; s < S; ++s) {
    const int n = ln.j * S + s;
    if (n < p.N) p.last_state[(ln.b * p.dim + ln.d) * p.N + n] = h[s];
  }
}

// Walk chunks [k0, k1) of group g from state h.  EMIT: write y (output pass);
// otherwise only advance h and sum Delta (split-L pass 1).
template <typename T, int NP, bool EMIT>
__device__ __forceinline__ void run_chunks(const FwdParams &p, FwdSmem<NP> &sm, const Lane &ln,
                                           int64_t k0, int64_t k1, float (&h)[NP / 4], float &dsum) {
  constexpr int S = NP / 4;
  const int c = ln.c, j = ln.j, q = ln.j;  // q: this lane's 8-step quarter of a chunk
  const int64_t L = p.L;
  const int64_t row = (ln.b * p.dim + (ln.valid ? ln.d : 0)) * L;
  const T *u_row = static_cast<const T *>(p.u) + row;
  const T *dr_row = static_cast<const T *>(p.delta) + row;
  const T *z_row = p.z ? static_cast<const T *>(p.z) + row : nullptr;
  T *y_row = static_cast<T *>(p.y) + row;
  const T *Bb = static_cast<const T *>(p.B) + ln.b * L * p.N;
  const T *Cb = static_cast<const T *>(p.C) + ln.b * L * p.N;
  const float bias = (p.bias && ln.valid) ? p.bias[ln.d] : 0.f;
  const float Dd = (p.D && ln.valid) ? p.D[ln.d] : 0.f;
  const bool io_vec = p.io_vec != 0, bc_vec = p.bc_vec != 0;
  float A2[S];
#pragma unroll
  for (int s = 0; s < S; ++s) {
    const int n = j * S + s;
    A2[s] = (ln.valid && n < p.N) ? p.A[ln.d * p.N + n] * kLog2e : 0.f;
  }

  for (int64_t k = k0; k < k1; ++k) {
    const int64_t t0 = k * kT;
    const int64_t tq = t0 + 8 * q;
    // ---- per (channel, step) quantities of this lane's 8 steps ----
    float uu[8], dr[8], zz[8];
    if (ln.valid) {
      IO<T>::load8(u_row, tq, L, io_vec, uu);
      IO<T>::load8(dr_row, tq, L, io_vec, dr);
      if (EMIT && z_row) IO<T>::load8(z_row, tq, L, io_vec, zz);
    } else {
#pragma unroll
      for (int i = 0; i < 8; ++i) { uu[i] = 0.f; dr[i] = 0.f; zz[i] = 0.f; }
    }
    float dlv[8], dluv[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      float dl = 0.f;
      if (ln.valid && tq + i < L) {
        const float s = dr[i] + bias;
        dl = p.softplus ? softplus_f(s) : s;
      }
      dlv[i] = dl;
      dluv[i] = dl * uu[i];
    }
    *reinterpret_cast<float4 *>(&sm.dl[c][8 * q]) = make_float4(dlv[0], dlv[1], dlv[2], dlv[3]);
    *reinterpret_cast<float4 *>(&sm.dl[c][8 * q + 4]) = make_float4(dlv[4], dlv[5], dlv[6], dlv[7]);
    *reinterpret_cast<float4 *>(&sm.dlu[c][8 * q]) = make_float4(dluv[0], dluv[1], dluv[2], dluv[3]);
    *reinterpret_cast<float4 *>(&sm.dlu[c][8 * q + 4]) = make_float4(dluv[4], dluv[5], dluv[6], dluv[7]);
    stage_bc<T, NP>(sm.Bs, Bb, t0, L, p.N, bc_vec, ln.lane);
    if (EMIT) stage_bc<T, NP>(sm.Cs, Cb, t0, L, p.N, bc_vec, ln.lane);
    __syncwarp();

    // ---- the recurrence: kT steps, S states per lane ----
#pragma unroll 2
    for (int tt = 0; tt < kT; tt += 4) {
      const float4 d4 = *reinterpret_cast<const float4 *>(&sm.dl[c][tt]);
      const float4 u4 = *reinterpret_cast<const float4 *>(&sm.dlu[c][tt]);
      const float dls[4] = {d4.x, d4.y, d4.z, d4.w};
      const float dus[4] = {u4.x, u4.y, u4.z, u4.w};
      float yp[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        float Bv[S], Cv[S];
        lds_vec<S>(&sm.Bs[tt + i][j * S], Bv);
        if (EMIT) lds_vec<S>(&sm.Cs[tt + i][j * S], Cv);
        float acc = 0.f;
#pragma unroll
        for (int s = 0; s < S; ++s) {
          const float a = ex2(dls[i] * A2[s]);
          h[s] = fmaf(a, h[s], dus[i] * Bv[s]);
          if (EMIT) acc = fmaf(Cv[s], h[s], acc);
        }
        yp[i] = acc;
        if (!EMIT) dsum += dls[i];
      }
      if (EMIT) sm.ys[c][tt + j] = reduce4_transpose(yp[0], yp[1], yp[2], yp[3], j);
    }

    // ---- epilogue: D skip, gate, store ----
    if (EMIT) {
      __syncwarp();
      if (ln.valid) {
        const float4 a = *reinterpret_cast<const float4 *>(&sm.ys[c][8 * q]);
        const float4 b4 = *reinterpret_cast<const float4 *>(&sm.ys[c][8 * q + 4]);
        const float ys[8] = {a.x, a.y, a.z, a.w, b4.x, b4.y, b4.z, b4.w};
        float o[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          float v = fmaf(Dd, uu[i], ys[i]);
          if (z_row) v *= silu_f(zz[i]);
          o[i] = v;
        }
        IO<T>::store8(y_row, tq, L, io_vec, o);
      }
    }
    __syncwarp();
  }
}

// ---- LOOKBACK: persistent, equal shares of (group, chunk) items ---------------
// Warp w owns items [w*W/P, (w+1)*W/P) of the W = groups*chunks items in
// (group, chunk) order.  Its range holds at most a tail of one group, whole
// groups, and a head of another (the host keeps P <= groups, so a range is
// never inside one group).  The head is done first, from the initial state,
// and its end state published; the tail, which needs the state the previous
// warp published from ITS head, is done last.  The bounded wait therefore
// only spins if the previous warp has not finished its first item by the
// time this warp has finished everything else.
template <typename T, int NP>
__global__ void __launch_bounds__(kThreads) k_fwd_lookback(FwdParams p) {
  constexpr int S = NP / 4;
  extern __shared__ __align__(16) unsigned char smem_raw[];
  const int warp = threadIdx.x >> 5;
  FwdSmem<NP> &sm = reinterpret_cast<FwdSmem<NP> *>(smem_raw)[warp];
  const int64_t w = (int64_t)blockIdx.x * kWarps + warp;
  const int64_t P = p.n_workers;
  if (w >= P) return;
  const int64_t K = p.n_chunks, W = p.n_groups * K;
  const int64_t s0 = w * W / P, e0 = (w + 1) * W / P;
  if (s0 >= e0) return;
  const int64_t g_first = s0 / K, k_first = s0 - g_first * K;
  const int64_t g_last = (e0 - 1) / K, k_end = e0 - g_last * K;
  float h[S];
  float dsum = 0.f;

  // Runs in execution order: [head of g_last] [whole groups] [tail of g_first].
  const bool one = g_first == g_last;
  const int64_t n_head = (!one && k_end < K) ? 1 : 0;
  const int64_t g_lo = k_first > 0 ? g_first + 1 : g_first;
  const int64_t g_hi = k_end < K ? g_last : g_last + 1;
  const int64_t n_full = one ? 0 : (g_hi > g_lo ? g_hi - g_lo : 0);
  const int64_t n_tail = (!one && k_first > 0) ? 1 : 0;
  const int64_t n_runs = one ? 1 : n_head + n_full + n_tail;
  for (int64_t r = 0; r < n_runs; ++r) {
    int64_t g, k0, k1;
    if (one) { g = g_first; k0 = k_first; k1 = k_end; }
    else if (r < n_head) { g = g_last; k0 = 0; k1 = k_end; }
    else if (r < n_head + n_full) { g = g_lo + (r - n_head); k0 = 0; k1 = K; }
    else { g = g_first; k0 = k_first; k1 = K; }
    const Lane ln = lane_of(p, g);
    if (k0 > 0) {  // continue the previous warp's head of this group
      warp_wait_flag(&p.flags[w - 1], p.err, p.wait_limit_ns);
#pragma unroll
      for (int s = 0; s < S; ++s)
        h[s] = __ldcg(&p.carry[((w - 1) * kCPW + ln.c) * NP + ln.j * S + s]);
    } else {
      init_state<NP>(p, ln, h);
    }
    run_chunks<T, NP, true>(p, sm, ln, k0, k1, h, dsum);
    if (k1 < K) {  // publish the head's end state for warp w + 1
#pragma unroll
      for (int s = 0; s < S; ++s) p.carry[(w * kCPW + ln.c) * NP + ln.j * S + s] = h[s];
      __threadfence();
      __syncwarp();
      if (ln.lane == 0) st_release(&p.flags[w], 1u);
    } else {
      write_last_state<NP>(p, ln, h);
    }
  }
}

// ---- SPLIT_L / PER_GROUP: one warp per (group, time segment) --------------------
// Items are ordered segment-major so that warps running together read the
// same B/C time range.  EMIT=false is pass 1 (segment end state from zero and
// the segment's sum of Delta); EMIT=true is the output pass, entering each
// segment with the state the carry kernel computed (or the initial state
// when there is one segment).
template <typename T, int NP, bool EMIT>
__global__ void __launch_bounds__(kThreads) k_fwd_segment(FwdParams p) {
  constexpr int S = NP / 4;
  extern __shared__ __align__(16) unsigned char smem_raw[];
  const int warp = threadIdx.x >> 5;
  FwdSmem<NP> &sm = reinterpret_cast<FwdSmem<NP> *>(smem_raw)[warp];
  const int64_t w = (int64_t)blockIdx.x * kWarps + warp;
  if (w >= p.n_groups * p.n_segs) return;
  const int64_t seg = w / p.n_groups, g = w - seg * p.n_groups;
  const int64_t k0 = seg * p.seg_chunks;
  const int64_t k1 = k0 + p.seg_chunks < p.n_chunks ? k0 + p.seg_chunks : p.n_chunks;
  const int64_t item = g * p.n_segs + seg;
  const Lane ln = lane_of(p, g);
  float h[S];
  float dsum = 0.f;
  if (!EMIT) {
#pragma unroll
    for (int s = 0; s < S; ++s) h[s] = 0.f;
  } else if (p.n_segs > 1) {
#pragma unroll
    for (int s = 0; s < S; ++s) h[s] = p.seg_carry[(item * kCPW + ln.c) * NP + ln.j * S + s];
  } else {
    init_state<NP>(p, ln, h);
  }
  if (k0 < k1) run_chunks<T, NP, EMIT>(p, sm, ln, k0, k1, h, dsum);
  if (!EMIT) {
#pragma unroll
    for (int s = 0; s < S; ++s) p.seg_h[(item * kCPW + ln.c) * NP + ln.j * S + s] = h[s];
    if (ln.j == 0) p.seg_dsum[item * kCPW + ln.c] = dsum;
  } else if (k1 == p.n_chunks) {
    write_last_state<NP>(p, ln, h);
  }
}

// Carry over segments, one thread per (group, channel, state):
//   carry_0 = h0,  carry_{s+1} = exp(A * sum_s Delta) * carry_s + h_end_s
// -- the associative operator of the recurrence applied segment by segment.
template <int NP>
__global__ void k_fwd_carry(FwdParams p) {
  const int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= p.n_groups * kCPW * NP) return;
  const int64_t g = idx / (kCPW * NP);
  const int c = (int)((idx / NP) % kCPW), n = (int)(idx % NP);
  const int64_t b = g / p.gpb, d = (g - b * p.gpb) * kCPW + c;
  const bool valid = d < p.dim && n < p.N;
  const float A2 = valid ? p.A[d * p.N + n] * kLog2e : 0.f;
  float carry = (valid && p.h0) ? p.h0[(b * p.dim + d) * p.N + n] : 0.f;
  for (int64_t s = 0; s < p.n_segs; ++s) {
    const int64_t item = g * p.n_segs + s;
    p.seg_carry[(item * kCPW + c) * NP + n] = carry;
    carry = fmaf(ex2(A2 * p.seg_dsum[item * kCPW + c]), carry, p.seg_h[(item * kCPW + c) * NP + n]);
  }
}

__global__ void k_wait_probe(unsigned *flag, unsigned *err, unsigned long long limit_ns) {
  warp_wait_flag(flag, err, limit_ns);
}

// ---- host side ------------------------------------------------------------------
template <class V> struct TypeTag { using type = V; };
template <int V> struct IntTag { static constexpr int value = V; };

template <class F>
static cudaError_t dispatch(int io_dtype, int NP, F &&f) {
  auto by_np = [&](auto tt) -> cudaError_t {
    switch (NP) {
      case 4: return f(tt, IntTag<4>{});
      case 8: return f(tt, IntTag<8>{});
      case 16: return f(tt, IntTag<16>{});
      case 32: return f(tt, IntTag<32>{});
      case 64: return f(tt, IntTag<64>{});
      default: return cudaErrorInvalidValue;
    }
  };
  if (io_dtype == 1) return by_np(TypeTag<uint16_t>{});
  if (io_dtype == 0) return by_np(TypeTag<float>{});
  return cudaErrorInvalidValue;
}

int fwd_np_for(int64_t N) { return N <= 4 ? 4 : N <= 8 ? 8 : N <= 16 ? 16 : N <= 32 ? 32 : 64; }

template <typename T, int NP>
static size_t fwd_smem_bytes() { return kWarps * sizeof(FwdSmem<NP>); }

template <class K>
static cudaError_t allow_smem(K kernel, size_t bytes) {
  if (bytes <= 48 * 1024) return cudaSuccess;
  return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
}

cudaError_t fwd_occupancy(int io_dtype, int NP, int *ctas_per_sm) {
  return dispatch(io_dtype, NP, [&](auto tt, auto np) -> cudaError_t {
    using T = typename decltype(tt)::type;
    constexpr int kNP = decltype(np)::value;
    const size_t smem = fwd_smem_bytes<T, kNP>();
    cudaError_t e = allow_smem(k_fwd_lookback<T, kNP>, smem);
    if (e != cudaSuccess) return e;
    return cudaOccupancyMaxActiveBlocksPerMultiprocessor(ctas_per_sm, k_fwd_lookback<T, kNP>,
                                                         kThreads, smem);
  });
}

cudaError_t launch_fwd_lookback(int io_dtype, int NP, const FwdParams &p, cudaStream_t s) {
  return dispatch(io_dtype, NP, [&](auto tt, auto np) -> cudaError_t {
    using T = typename decltype(tt)::type;
    constexpr int kNP = decltype(np)::value;
    const size_t smem = fwd_smem_bytes<T, kNP>();
    cudaError_t e = allow_smem(k_fwd_lookback<T, kNP>, smem);
    if (e != cudaSuccess) return e;
    const unsigned grid = (unsigned)((p.n_workers + kWarps - 1) / kWarps);
    k_fwd_lookback<T, kNP><<<grid, kThreads, smem, s>>>(p);
    return cudaGetLastError();
  });
}

cudaError_t launch_fwd_splitl(int io_dtype, int NP, const FwdParams &p, cudaStream_t s) {
  return dispatch(io_dtype, NP, [&](auto tt, auto np) -> cudaError_t {
    using T = typename decltype(tt)::type;
    constexpr int kNP = decltype(np)::value;
    const size_t smem = fwd_smem_bytes<T, kNP>();
    const unsigned grid = (unsigned)((p.n_groups * p.n_segs + kWarps - 1) / kWarps);
    cudaError_t e;
    if (p.n_segs > 1) {
      e = allow_smem(k_fwd_segment<T, kNP, false>, smem);
      if (e != cudaSuccess) return e;
      k_fwd_segment<T, kNP, false><<<grid, kThreads, smem, s>>>(p);
      const int64_t nthreads = p.n_groups * kCPW * kNP;
      k_fwd_carry<kNP><<<(unsigned)((nthreads + 255) / 256), 256, 0, s>>>(p);
    }
    e = allow_smem(k_fwd_segment<T, kNP, true>, smem);
    if (e != cudaSuccess) return e;
    k_fwd_segment<T, kNP, true><<<grid, kThreads, smem, s>>>(p);
    return cudaGetLastError();
  });
}

cudaError_t launch_wait_timeout_probe(unsigned *flag, unsigned *err, unsigned long long limit_ns,
                                      cudaStream_t s) {
  k_wait_probe<<<1, 32, 0, s>>>(flag, err, limit_ns);
  return cudaGetLastError();
}

}  // namespace ssm
