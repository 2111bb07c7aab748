// Causal depthwise 1-D convolution along the sequence, with optional SiLU,
// for sm_100a: the convolution layer the Mamba block applies to x_proj
// before the SSM, followed by its SiLU activation ("O que e um modelo
// Mamba?", ibm.com, the walk-through of the Mamba block: the convolution
// extracts local patterns between neighbouring tokens, its output goes
// through SiLU and becomes the SSM's input).  Per channel d, width K:
//   out_t = act(bias[d] + sum_{k<K} w[d][k] * x_{t-K+1+k}),
// with x_t for t < 0 taken from the caller's initial state (zeros if none).
//
// Design (B200): 2 bytes in and 2 out per (b, d, t) in bf16 and a few
// instructions per element, so HBM sets the pace.  Both kernels give a lane
// 16 consecutive steps of a row and compute them as 8 packed fp32 pairs
// (t, t + 8): the convolution, the activation and, in the backward, the
// dweight sums and dx run as f32x2 operations on aligned register pairs, and
// only the K-1 pairs at a chunk's edge are assembled from two halves.  The K-1
// inputs before a chunk come from the previous lane by one shuffle, so every
// input byte is read once.
#include "ssm_common.cuh"

#include <algorithm>

namespace ssm {

constexpr int kConvThreads = 256;

// ---- shared by forward and backward ----------------------------------------
__device__ __forceinline__ void conv_cp16(uint32_t dst, const void *src, uint32_t bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(bytes) : "memory");
}
__device__ __forceinline__ void conv_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void conv_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// value i of a lane's raw chunk (bf16 pairs per word, or fp32 words)
template <typename T>
__device__ __forceinline__ float raw_at(const uint32_t *w, int i) {
  if constexpr (sizeof(T) == 2)
    return __uint_as_float((i & 1) ? (w[i >> 1] & 0xffff0000u) : (w[i >> 1] << 16));
  else
    return __uint_as_float(w[i]);
}

__device__ __forceinline__ float lo_of(f2 v) {
  float lo, hi;
  unpack2(v, lo, hi);
  return lo;
}
__device__ __forceinline__ float hi_of(f2 v) {
  float lo, hi;
  unpack2(v, lo, hi);
  return hi;
}

// ---- forward --------------------------------------------------------------
// Lane-contiguous forward: a warp takes P passes of 512 steps of one row; lane
// l owns steps 16 l .. 16 l + 15 of each pass, loaded up front with one 32-byte
// load per pass (two 16-byte ones, or elements, where the row allows less),
// computed as 8 packed pairs (t, t + 8) and stored with one 32-byte store.
template <typename T>
struct ConvFwdPass {
  static constexpr int S = 16, H = 8, PASS = 32 * S;
  static constexpr int P = sizeof(T) == 2 ? 4 : 2;  // passes per warp
  static constexpr int SEG = P * PASS;              // steps per warp
  static constexpr int W = S * (int)sizeof(T) / 4;  // 32-bit words of one lane's chunk
};

template <typename T, int W>
__device__ __forceinline__ void conv_load_chunk(uint32_t (&w)[W], const T *src, int64_t rem, int vec) {
  constexpr int S = W * 4 / (int)sizeof(T);
  if (vec == 2 && rem >= S) {
#pragma unroll
    for (int v = 0; v < W / 8; ++v)
      asm volatile("ld.global.cs.v8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
                   : "=r"(w[8 * v]), "=r"(w[8 * v + 1]), "=r"(w[8 * v + 2]), "=r"(w[8 * v + 3]),
                     "=r"(w[8 * v + 4]), "=r"(w[8 * v + 5]), "=r"(w[8 * v + 6]), "=r"(w[8 * v + 7])
                   : "l"(src + v * (32 / (int)sizeof(T))));
  } else if (vec && rem >= S) {
#pragma unroll
    for (int v = 0; v < W / 4; ++v) {
      const uint4 q = __ldcs(reinterpret_cast<const uint4 *>(src) + v);
      w[4 * v] = q.x; w[4 * v + 1] = q.y; w[4 * v + 2] = q.z; w[4 * v + 3] = q.w;
    }
  } else {
#pragma unroll
    for (int i = 0; i < W; ++i) w[i] = 0u;
#pragma unroll
    for (int e = 0; e < S; ++e)
      if (e < rem) {
        if constexpr (sizeof(T) == 2) w[e >> 1] |= (uint32_t)src[e] << (16 * (e & 1));
        else w[e] = __float_as_uint(src[e]);
      }
  }
}

template <typename T, int K, bool SILU>
__global__ void __launch_bounds__(kConvThreads, (sizeof(T) == 2 && K <= 4) ? 4 : 2) k_conv(ConvParams p) {
  using G = ConvFwdPass<T>;
  constexpr int S = G::S, H = G::H, W = G::W, KM = K - 1, KA = K > 1 ? K - 1 : 1;
  const int lane = threadIdx.x & 31;
  const int64_t L = p.L, segs = (L + G::SEG - 1) / G::SEG;
  const int64_t wid = ((int64_t)blockIdx.x * kConvThreads + threadIdx.x) >> 5;
  const int64_t row = wid / segs, seg = wid - row * segs;
  if (row >= p.batch * p.dim) return;  // whole warps leave together
  const int64_t d = row % p.dim;
  const T *xr = static_cast<const T *>(p.x) + row * L;
  T *orow = static_cast<T *>(p.out) + row * L;
  const int64_t tw = seg * G::SEG;
  uint32_t xw[G::P][W];
#pragma unroll
  for (int r = 0; r < G::P; ++r) {
    const int64_t t0 = tw + r * G::PASS + lane * S;
    conv_load_chunk<T, W>(xw[r], xr + t0, L - t0, p.vec);
  }
  f2 w2[K];
#pragma unroll
  for (int k = 0; k < K; ++k) w2[k] = splat2(p.w[d * K + k]);
  const f2 bias2 = splat2(p.bias ? p.bias[d] : 0.f);
  // lane 31's inputs before the next pass reach lane 0 by the shuffle below; before
  // the warp's first pass they come from memory (lane 31 loads them)
  float prevtail[KA];
#pragma unroll
  for (int m = 0; m < KM; ++m) prevtail[m] = (lane == 31 && tw > 0) ? IO<T>::get(xr, tw - KM + m) : 0.f;
#pragma unroll
  for (int r = 0; r < G::P; ++r) {
    if (tw + r * G::PASS >= L) break;  // warp-uniform
    const int64_t t0 = tw + r * G::PASS + lane * S;
    float hal[KA];
#pragma unroll
    for (int m = 0; m < KM; ++m) {
      const float cur = raw_at<T>(xw[r], S - KM + m);
      float h = __shfl_sync(0xffffffffu, lane == 31 ? prevtail[m] : cur, (lane + 31) & 31);
      prevtail[m] = cur;
      if (lane == 0 && tw == 0 && r == 0) h = p.s0 ? p.s0[row * KM + m] : 0.f;
      hal[m] = h;
    }
    auto xp = [&](int m) -> f2 {
      return pack2(m < 0 ? hal[m + KM] : raw_at<T>(xw[r], m), raw_at<T>(xw[r], m + H));
    };
    float lo_o[H], hi_o[H];
#pragma unroll
    for (int q = 0; q < H; ++q) {
      f2 a = bias2;
#pragma unroll
      for (int k = 0; k < K; ++k) a = fma2(w2[k], xp(q - KM + k), a);
      if constexpr (SILU) {  // SiLU(a) = a / (1 + e^-a), on the pair
        float e0, e1, d0, d1;
        unpack2(mul2(a, splat2(-kLog2e)), e0, e1);
        unpack2(add2(pack2(ex2(e0), ex2(e1)), splat2(1.f)), d0, d1);
        a = mul2(a, pack2(rcp_approx(d0), rcp_approx(d1)));
      }
      unpack2(a, lo_o[q], hi_o[q]);
    }
    const int64_t rem = L - t0;
    if (rem > 0) {
      if constexpr (sizeof(T) == 2) {
        if (p.vec == 2 && rem >= S) {  // the lane's 32 bytes: whole sectors
          asm volatile("st.global.cs.v8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"l"(orow + t0),
                       "r"(pack_bf16x2(lo_o[0], lo_o[1])), "r"(pack_bf16x2(lo_o[2], lo_o[3])),
                       "r"(pack_bf16x2(lo_o[4], lo_o[5])), "r"(pack_bf16x2(lo_o[6], lo_o[7])),
                       "r"(pack_bf16x2(hi_o[0], hi_o[1])), "r"(pack_bf16x2(hi_o[2], hi_o[3])),
                       "r"(pack_bf16x2(hi_o[4], hi_o[5])), "r"(pack_bf16x2(hi_o[6], hi_o[7]))
                       : "memory");
        } else {
          IO<T>::store8(orow, t0, L, p.vec != 0, lo_o);
          if (rem > H) IO<T>::store8(orow, t0 + H, L, p.vec != 0, hi_o);
        }
      } else {
        IO<T>::store8(orow, t0, L, p.vec != 0, lo_o);
        if (rem > H) IO<T>::store8(orow, t0 + H, L, p.vec != 0, hi_o);
      }
    }
  }
  // final state: the row's last K-1 inputs, by lane 0 of the warp holding step L-1
  if (KM > 0 && p.s1 && lane == 0 && tw + G::SEG >= L) {
#pragma unroll
    for (int m = 0; m < KM; ++m) {
      const int64_t t = L - KM + m;
      p.s1[row * KM + m] = t >= 0 ? IO<T>::get(xr, t) : (p.s0 ? p.s0[row * KM + KM + t] : 0.f);
    }
  }
}

template <typename T, int K>
static cudaError_t launch_conv_fwd_k(const ConvParams &p, cudaStream_t s) {
  using G = ConvFwdPass<T>;
  const int64_t segs = (p.L + G::SEG - 1) / G::SEG;
  const int64_t warps = p.batch * p.dim * segs;
  const int64_t blocks = (warps * 32 + kConvThreads - 1) / kConvThreads;
  if (blocks > 0x7fffffff) return cudaErrorInvalidConfiguration;
  if (p.silu) k_conv<T, K, true><<<(unsigned)blocks, kConvThreads, 0, s>>>(p);
  else k_conv<T, K, false><<<(unsigned)blocks, kConvThreads, 0, s>>>(p);
  return cudaGetLastError();
}

template <typename T>
static cudaError_t launch_conv_t(const ConvParams &p, cudaStream_t s) {
  switch (p.K) {
    case 1: return launch_conv_fwd_k<T, 1>(p, s);
    case 2: return launch_conv_fwd_k<T, 2>(p, s);
    case 3: return launch_conv_fwd_k<T, 3>(p, s);
    case 4: return launch_conv_fwd_k<T, 4>(p, s);
    case 5: return launch_conv_fwd_k<T, 5>(p, s);
    case 6: return launch_conv_fwd_k<T, 6>(p, s);
    case 7: return launch_conv_fwd_k<T, 7>(p, s);
    case 8: return launch_conv_fwd_k<T, 8>(p, s);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_conv(int io_dtype, const ConvParams &p, cudaStream_t s) {
  return io_dtype == 1 ? launch_conv_t<uint16_t>(p, s) : launch_conv_t<float>(p, s);
}

// ---- backward -------------------------------------------------------------
// Gradients of sum(dout * out): with a_t = bias + sum_k w_k x_{t-K+1+k} and
// out_t = act(a_t), da_t = dout_t act'(a_t); dx_s = sum_k w_k da_{s+K-1-k};
// dw_k = sum_{b,t} da_t x_{t-K+1+k}; dbias = sum_{b,t} da_t; the initial
// state's gradient is dx of the K-1 inputs before t = 0.
//
// Design (B200): 2 bytes in per stream and 2 out per (b, d, t) in bf16, and
// about 20 thread instructions per element, so HBM-bound once the three K-tap
// sums run on packed pairs.  Persistent warps each walk a contiguous range of
// 512-step segments, row after row.  A segment's x and dout reach shared
// memory by cp.async in coalesced 16-byte pieces, two segments in flight
// behind the one computed (a 3-stage ring per warp); lane l's 16 steps sit in
// a chunk padded to an odd number of 16-byte units, so the lanes' 16-byte
// reads hit distinct banks.  A lane takes its 16 steps as 8 packed pairs
// (t, t + 8): the convolution, SiLU', the dweight sums and dx are f32x2
// operations on aligned register pairs, and only the K-1 pairs at each edge
// of the chunk are assembled from two halves.  The K-1 inputs before a chunk
// come from the previous lane by one shuffle (lane 0 from lane 31 of the
// warp's previous segment, the initial state, or memory at the start of the
// range); the K-1 values of da after it from the next lane.  Lane 31 parks
// the second half of its dx in shared memory until the warp's next segment
// supplies those (lane 0's first values), or recomputes them from memory at
// the end of its range.  dweight and dbias are summed per warp and row and
// added with one atomic each when the row changes (the scan's own backward
// uses no float atomics; this one's parameter sums are not bitwise repeatable).
template <typename T>
struct ConvBwdGeo {
  static constexpr int S = 16;                         // steps per lane and segment
  static constexpr int H = S / 2;                      // packed pairs (t, t + H)
  static constexpr int SEG = 32 * S;                   // steps per segment
  static constexpr int CHUNK = S * (int)sizeof(T);     // one lane's steps of one stream, bytes
  static constexpr int UPL = CHUNK / 16;               // 16-byte pieces per lane and stream
  static constexpr int PAD = CHUNK + 16;               // an odd count of 16-byte units
  static constexpr int STREAM = 32 * PAD;              // one stream of one stage
  static constexpr int STAGE = 2 * STREAM;             // x, then dout
  static constexpr int STAGES = 3;                     // the segment computed + two in flight
  static constexpr int WARP_BYTES = STAGES * STAGE + H * 4;  // + lane 31's parked dx half
  static constexpr int WARPS = 4;                      // warps per CTA
  static constexpr int SMEM = WARPS * WARP_BYTES;
};
// CTAs per SM the registers are sized for: 5 (20 warps, 96 registers) for bf16
// up to width 4.  Measured on B200 at the Mamba-2.8B x_proj shape: 0.247 ms,
// against 0.333 ms at 6 CTAs (80 registers, spilling) and 0.255 ms at 4.
// Wider filters hold more edge pairs and take 4.
template <typename T, int K>
constexpr int conv_bwd_min_blocks() { return sizeof(T) == 2 ? (K <= 4 ? 5 : 4) : 2; }

// da = dout * SiLU'(a) = g s (1 + a (1 - s)), s = 1 / (1 + e^-a), on a pair
__device__ __forceinline__ f2 silu_grad2(f2 a, f2 g) {
  float m0, m1, d0, d1;
  unpack2(mul2(a, splat2(-kLog2e)), m0, m1);
  unpack2(add2(pack2(ex2(m0), ex2(m1)), splat2(1.f)), d0, d1);
  const f2 sg = pack2(rcp_approx(d0), rcp_approx(d1));
  const f2 fac = fma2(a, fma2(sg, splat2(-1.f), splat2(1.f)), splat2(1.f));
  return mul2(mul2(g, sg), fac);
}

// the same, one value (the same operations in the same order)
__device__ __forceinline__ float conv_act_grad(float a, float g, bool silu) {
  if (!silu) return g;
  const float sg = rcp_approx(1.f + ex2(a * -kLog2e));
  return g * sg * fmaf(a, fmaf(sg, -1.f, 1.f), 1.f);
}

// SILU: the activation's derivative applied (a separate instantiation: the run-time
// choice cost 0.8 instructions per element and 2 % of the time)
template <typename T, int K, bool SILU>
__global__ void __launch_bounds__(ConvBwdGeo<T>::WARPS * 32, (conv_bwd_min_blocks<T, K>())) k_conv_bwd(ConvBwdParams p) {
  using G = ConvBwdGeo<T>;
  constexpr int S = G::S, H = G::H, KM = K - 1, KA = K > 1 ? K - 1 : 1;
  static_assert(H == 8 && KM <= H, "dx halves are stored 8 at a time; the edge pairs need K - 1 <= 8");
  extern __shared__ __align__(16) unsigned char conv_smem[];
  const int lane = threadIdx.x & 31, wib = threadIdx.x >> 5;
  const int64_t L = p.L, segs = (L + G::SEG - 1) / G::SEG, items = p.batch * p.dim * segs;
  const int64_t nw = (int64_t)gridDim.x * G::WARPS, wg = (int64_t)blockIdx.x * G::WARPS + wib;
  const int64_t i_begin = items * wg / nw, i_end = items * (wg + 1) / nw;
  if (i_begin >= i_end) return;  // whole warps leave together
  unsigned char *ring = conv_smem + wib * G::WARP_BYTES;
  const uint32_t ring_s = (uint32_t)__cvta_generic_to_shared(ring);
  float *park = reinterpret_cast<float *>(ring + G::STAGES * G::STAGE);  // lane 31's dx half
  const bool vec = p.vec != 0;
  const T *x = static_cast<const T *>(p.x);
  const T *dout = static_cast<const T *>(p.dout);
  T *dx = static_cast<T *>(p.dx);

  // Fill cursor: the next segment to fetch, as its first element's index in the
  // [rows][L] arrays and the steps left in its row from there.  Piece q of a
  // segment (16 bytes; lane q % 32 copies it) goes to unit q % UPL of lane
  // q / UPL's padded chunk: coalesced reads.  This lane's pieces are lane + 32 j.
  int64_t row = i_begin / segs;
  const int64_t seg0 = i_begin - row * segs;
  int64_t fbase = row * L + seg0 * G::SEG, frem = L - seg0 * G::SEG;
  // compute cursor, the same for the segment computed
  int64_t cbase = fbase, crem = frem;
  constexpr int EPP = 16 / (int)sizeof(T);                                  // elements per piece
  const int eoff0 = lane * EPP;                                              // element offset in the segment
  const uint32_t soff0 = (lane / G::UPL) * G::PAD + 16 * (lane % G::UPL);  // byte offset in the stage
  auto fill = [&](int st) {
    const uint32_t sb = ring_s + st * G::STAGE;
#pragma unroll
    for (int j = 0; j < G::UPL; ++j) {
      // piece lane + 32 j: 32 j / UPL chunks further on (32 is a multiple of UPL)
      const int eoff = eoff0 + 32 * j * EPP;
      const uint32_t soff = soff0 + (32 * j / G::UPL) * G::PAD;
      const bool in = eoff < frem;
      if (vec) {  // rows 16-byte aligned, L a whole number of pieces: a piece is all in or all out
        conv_cp16(sb + soff, x + fbase + (in ? eoff : 0), in ? 16u : 0u);
        conv_cp16(sb + soff + G::STREAM, dout + fbase + (in ? eoff : 0), in ? 16u : 0u);
      } else {
        const T *xp = x + fbase + eoff, *gp = dout + fbase + eoff;
        uint32_t a[4] = {0u, 0u, 0u, 0u}, b[4] = {0u, 0u, 0u, 0u};
#pragma unroll
        for (int e = 0; e < 16 / (int)sizeof(T); ++e) {
          if (eoff + e < frem) {
            if constexpr (sizeof(T) == 2) {
              a[e >> 1] |= (uint32_t)xp[e] << (16 * (e & 1));
              b[e >> 1] |= (uint32_t)gp[e] << (16 * (e & 1));
            } else {
              a[e] = __float_as_uint(xp[e]);
              b[e] = __float_as_uint(gp[e]);
            }
          }
        }
        unsigned char *dst = ring + st * G::STAGE + soff;
        *reinterpret_cast<uint4 *>(dst) = make_uint4(a[0], a[1], a[2], a[3]);
        *reinterpret_cast<uint4 *>(dst + G::STREAM) = make_uint4(b[0], b[1], b[2], b[3]);
      }
    }
    // on to the following segment (the next row's first when this row ends here)
    fbase += G::SEG;
    frem -= G::SEG;
    if (frem <= 0) {
      fbase += frem;
      frem = L;
    }
  };

  const int n_items = (int)(i_end - i_begin);
#pragma unroll
  for (int j = 0; j < G::STAGES - 1; ++j) {  // the first segments in flight
    if (j < n_items) fill(j);
    conv_commit();
  }

  f2 w2[K], bias2;
  auto load_w = [&]() {  // the filter of the current row's channel
    const int64_t d = row % p.dim;
#pragma unroll
    for (int k = 0; k < K; ++k) w2[k] = splat2(p.w[d * K + k]);
    bias2 = splat2(p.bias ? p.bias[d] : 0.f);
  };
  load_w();
  f2 dwp[K], dbp = splat2(0.f);  // this lane's dweight / dbias partials of the current row, on pairs
#pragma unroll
  for (int k = 0; k < K; ++k) dwp[k] = splat2(0.f);
  // this lane's last K-1 inputs of the previous segment; lane 31's reach lane 0.  At the
  // start of the range lane 31 takes them from memory (the row's previous segment).
  float prevtail[KA];
#pragma unroll
  for (int m = 0; m < KM; ++m)
    prevtail[m] = (lane == 31 && seg0 > 0) ? IO<T>::get(x + cbase, m - KM) : 0.f;
  bool parked = false;  // lane 31: the second half of the previous segment's dx waits in `park`

  int st = 0;
  for (int it = 0; it < n_items; ++it) {
    if (it + G::STAGES - 1 < n_items) fill(st == 0 ? G::STAGES - 1 : st - 1);  // into the stage computed last
    conv_commit();
    conv_wait<G::STAGES - 1>();
    __syncwarp();
    const bool first = crem == L;                 // the row's first segment
    T *dxl = dx + cbase + lane * S;               // this lane's chunk of dx
    const int64_t lrem = crem - lane * S;         // steps of the row from there

    uint32_t xw[G::CHUNK / 4], gw[G::CHUNK / 4];
    const unsigned char *ch = ring + st * G::STAGE + lane * G::PAD;
#pragma unroll
    for (int u = 0; u < G::UPL; ++u) {
      const uint4 vx = *reinterpret_cast<const uint4 *>(ch + 16 * u);
      const uint4 vg = *reinterpret_cast<const uint4 *>(ch + G::STREAM + 16 * u);
      xw[4 * u] = vx.x; xw[4 * u + 1] = vx.y; xw[4 * u + 2] = vx.z; xw[4 * u + 3] = vx.w;
      gw[4 * u] = vg.x; gw[4 * u + 1] = vg.y; gw[4 * u + 2] = vg.z; gw[4 * u + 3] = vg.w;
    }
    // the K-1 inputs before the chunk
    float hal[KA];
#pragma unroll
    for (int m = 0; m < KM; ++m) {
      const float cur = raw_at<T>(xw, S - KM + m);
      float h = __shfl_sync(0xffffffffu, lane == 31 ? prevtail[m] : cur, (lane + 31) & 31);
      prevtail[m] = cur;
      if (lane == 0 && first) h = p.s0 ? p.s0[row * KM + m] : 0.f;
      hal[m] = h;
    }
    // pair m = (x_{t0+m}, x_{t0+m+H}), m >= -(K-1)
    auto xp = [&](int m) -> f2 {
      return pack2(m < 0 ? hal[m + KM] : raw_at<T>(xw, m), raw_at<T>(xw, m + H));
    };

    // da on pairs; dweight and dbias partials
    f2 da[H + KA];
#pragma unroll
    for (int q = 0; q < H; ++q) {
      f2 a = bias2;
#pragma unroll
      for (int k = 0; k < K; ++k) a = fma2(w2[k], xp(q - KM + k), a);
      const f2 g2 = pack2(raw_at<T>(gw, q), raw_at<T>(gw, q + H));
      const f2 dq = SILU ? silu_grad2(a, g2) : g2;  // zero past L (dout is zero-filled there)
      da[q] = dq;
      dbp = add2(dbp, dq);
#pragma unroll
      for (int k = 0; k < K; ++k) dwp[k] = fma2(dq, xp(q - KM + k), dwp[k]);
    }

    // the next lane's first K-1 values of da; lane 31 receives lane 0's, the values
    // after the previous segment's lane-31 chunk
    float nx[KA];
#pragma unroll
    for (int m = 0; m < KM; ++m) nx[m] = __shfl_sync(0xffffffffu, lo_of(da[m]), (lane + 1) & 31);
    if (parked) {  // lane 31, same row, previous segment: finish and store its second dx half
      float v[H];
#pragma unroll
      for (int s = 0; s < H; ++s) v[s] = park[s];
#pragma unroll
      for (int s = 0; s < H; ++s)
#pragma unroll
        for (int k = 0; k < K; ++k)
          if (s + KM - k >= H) v[s] = fmaf(lo_of(w2[k]), nx[s + KM - k - H], v[s]);
      IO<T>::store8(dx + cbase, -H, crem, vec, v);
      parked = false;
    }
#pragma unroll
    for (int m = 0; m < KM; ++m) da[H + m] = pack2(hi_of(da[m]), lane == 31 ? 0.f : nx[m]);

    // dx on pairs: dx_s = sum_k w_k da_{s+K-1-k}
    float lo_o[H], hi_o[H];
#pragma unroll
    for (int s = 0; s < H; ++s) {
      f2 acc = mul2(w2[K - 1], da[s]);
#pragma unroll
      for (int k = 0; k < K - 1; ++k) acc = fma2(w2[k], da[s + KM - k], acc);
      unpack2(acc, lo_o[s], hi_o[s]);
    }
    if (lrem > 0) IO<T>::store8(dxl, 0, lrem, vec, lo_o);
    // lane 31 of a segment the row continues past: the terms from the next segment's
    // first K-1 steps are still missing
    const bool open = KM > 0 && lane == 31 && crem > G::SEG;
    if (open && it + 1 < n_items) {
#pragma unroll
      for (int s = 0; s < H; ++s) park[s] = hi_o[s];
      parked = true;
    } else {
      if (open) {  // the end of the range: those K-1 values of da from memory
        const T *xs = x + cbase, *gs = dout + cbase;  // steps relative to the segment
        float nd[KA];
#pragma unroll
        for (int m = 0; m < KM; ++m) {
          const int t = G::SEG + m;
          float a = lo_of(bias2);
#pragma unroll
          for (int k = 0; k < K; ++k) {
            const int tx = t - KM + k;
            a = fmaf(lo_of(w2[k]), tx < crem ? IO<T>::get(xs, tx) : 0.f, a);
          }
          nd[m] = t < crem ? conv_act_grad(a, IO<T>::get(gs, t), SILU) : 0.f;
        }
#pragma unroll
        for (int s = 0; s < H; ++s)
#pragma unroll
          for (int k = 0; k < K; ++k)
            if (s + KM - k >= H) hi_o[s] = fmaf(lo_of(w2[k]), nd[s + KM - k - H], hi_o[s]);
      }
      if (lrem > H) IO<T>::store8(dxl, H, lrem, vec, hi_o);
    }
    // initial-state gradient: dx of x_{-(K-1)+j} = sum_k w_k da_{j-k}, j - k >= 0
    if (KM > 0 && p.ds0 && first && lane == 0) {
#pragma unroll
      for (int j = 0; j < KM; ++j) {
        float acc = 0.f;
#pragma unroll
        for (int k = 0; k < K; ++k)
          if (j - k >= 0) acc = fmaf(lo_of(w2[k]), lo_of(da[j - k]), acc);
        p.ds0[row * KM + j] = acc;
      }
    }
    __syncwarp();  // every lane is done with stage st before it is refilled
    st = st + 1 == G::STAGES ? 0 : st + 1;
    // the next segment; the finished row's dweight and dbias go out
    cbase += G::SEG;
    crem -= G::SEG;
    const bool row_done = crem <= 0;
    if (row_done) {
      cbase += crem;
      crem = L;
    }
    if (row_done || it + 1 == n_items) {
      float dws[K], dbs = lo_of(dbp) + hi_of(dbp);
#pragma unroll
      for (int k = 0; k < K; ++k) dws[k] = lo_of(dwp[k]) + hi_of(dwp[k]);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
#pragma unroll
        for (int k = 0; k < K; ++k) dws[k] += __shfl_xor_sync(0xffffffffu, dws[k], o);
        dbs += __shfl_xor_sync(0xffffffffu, dbs, o);
      }
      if (lane == 0) {
        const int64_t d = row % p.dim;
#pragma unroll
        for (int k = 0; k < K; ++k) atomicAdd(&p.dw[d * K + k], dws[k]);
        if (p.dbias) atomicAdd(&p.dbias[d], dbs);
      }
#pragma unroll
      for (int k = 0; k < K; ++k) dwp[k] = splat2(0.f);
      dbp = splat2(0.f);
      if (row_done) {
        ++row;
        if (it + 1 < n_items) load_w();
      }
    }
  }
  conv_wait<0>();  // no copy outlives the kernel (the last groups are empty)
}

template <typename T, int K>
static cudaError_t launch_conv_bwd_k(const ConvBwdParams &p, cudaStream_t s) {
  using G = ConvBwdGeo<T>;
  auto kern = p.silu ? k_conv_bwd<T, K, true> : k_conv_bwd<T, K, false>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, G::SMEM);
  if (e != cudaSuccess) return e;
  int dev = 0, sms = 0, occ = 0;
  if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
  if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
  if ((e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, kern, G::WARPS * 32, G::SMEM)) != cudaSuccess)
    return e;
  // persistent: one wave of CTAs, each warp a contiguous range of segments
  const int64_t segs = (p.L + G::SEG - 1) / G::SEG;
  const int64_t items = p.batch * p.dim * segs;
  const int64_t want = (items + G::WARPS - 1) / G::WARPS;
  const int64_t grid = std::max<int64_t>(1, std::min<int64_t>(want, (int64_t)sms * std::max(occ, 1)));
  kern<<<(unsigned)grid, G::WARPS * 32, G::SMEM, s>>>(p);
  return cudaGetLastError();
}

template <typename T>
static cudaError_t launch_conv_bwd_t(const ConvBwdParams &p, cudaStream_t s) {
  switch (p.K) {
    case 1: return launch_conv_bwd_k<T, 1>(p, s);
    case 2: return launch_conv_bwd_k<T, 2>(p, s);
    case 3: return launch_conv_bwd_k<T, 3>(p, s);
    case 4: return launch_conv_bwd_k<T, 4>(p, s);
    case 5: return launch_conv_bwd_k<T, 5>(p, s);
    case 6: return launch_conv_bwd_k<T, 6>(p, s);
    case 7: return launch_conv_bwd_k<T, 7>(p, s);
    case 8: return launch_conv_bwd_k<T, 8>(p, s);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_conv_bwd(int io_dtype, const ConvBwdParams &p, cudaStream_t s) {
  return io_dtype == 1 ? launch_conv_bwd_t<uint16_t>(p, s) : launch_conv_bwd_t<float>(p, s);
}

}  // namespace ssm
