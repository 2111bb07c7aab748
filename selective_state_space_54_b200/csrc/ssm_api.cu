// C ABI of libssmscan.so: argument checks, schedule planning, workspace
// layout and launches.  The public contract is include/ssm_scan.h.
#include <stdio.h>
#include <string.h>

#include <algorithm>
#include <atomic>

#include "ssm_common.cuh"
#include "ssm_scan.h"

using namespace ssm;

namespace {

constexpr int32_t kVersion = 100;  // 0.1.0

size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }
bool aligned(const void *p, size_t a) { return p == nullptr || ((uintptr_t)p % a) == 0; }

int device_sms() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  int sms = 0;
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
  return sms;
}

ssm_status check_shape(const ssm_shape *s) {
  if (!s) return SSM_ERR_INVALID_ARG;
  if (s->batch < 0 || s->dim < 0 || s->seqlen < 0 || s->dstate < 1) return SSM_ERR_INVALID_ARG;
  if (s->dstate > 64) return SSM_ERR_UNSUPPORTED;
  if (s->io_dtype != SSM_F32 && s->io_dtype != SSM_BF16) return SSM_ERR_UNSUPPORTED;
  if (s->path < SSM_PATH_AUTO || s->path > SSM_PATH_LOOKBACK_WS) return SSM_ERR_UNSUPPORTED;
  // the warp-specialised kernel takes 4 lanes per channel for 5..16 states only
  if (s->path == SSM_PATH_LOOKBACK_WS && s->lanes == 4 && (s->dstate < 5 || s->dstate > 16))
    return SSM_ERR_UNSUPPORTED;
  if (s->lanes != 0 && s->lanes != 2 && s->lanes != 4) return SSM_ERR_UNSUPPORTED;
  if (s->flags & ~(SSM_FLAG_ZOH_EXACT | SSM_FLAG_SAVE_STATES | SSM_FLAG_TOKEN_MAJOR))
    return SSM_ERR_INVALID_ARG;
  // token-major activations: bf16, 16-byte channel rows, warp-specialised Euler path
  if ((s->flags & SSM_FLAG_TOKEN_MAJOR) &&
      (s->io_dtype != SSM_BF16 || s->dim % 8 != 0 || (s->flags & SSM_FLAG_ZOH_EXACT) ||
       (s->path != SSM_PATH_AUTO && s->path != SSM_PATH_LOOKBACK_WS) || s->lanes == 4))
    return SSM_ERR_UNSUPPORTED;
  // the exact-ZOH input term is built into the two look-back kernels
  if ((s->flags & SSM_FLAG_ZOH_EXACT) && s->path != SSM_PATH_AUTO && s->path != SSM_PATH_LOOKBACK &&
      s->path != SSM_PATH_LOOKBACK_WS)
    return SSM_ERR_UNSUPPORTED;
  // saved states are written by the warp-specialised kernel
  if ((s->flags & SSM_FLAG_SAVE_STATES) &&
      ((s->path != SSM_PATH_AUTO && s->path != SSM_PATH_LOOKBACK_WS) || s->lanes == 4))
    return SSM_ERR_UNSUPPORTED;
  // index arithmetic is int64; keep every flat index well inside it
  const double elems = (double)s->batch * (double)s->dim * (double)s->seqlen;
  if (elems > 4.0e15 || (double)s->batch * s->seqlen * s->dstate > 4.0e15) return SSM_ERR_UNSUPPORTED;
  return SSM_OK;
}

struct FwdPlan {
  int path = SSM_PATH_AUTO;
  int NP = 4;
  int LPC = 4;                       // lanes per channel
  int64_t gpb = 0, n_groups = 0, K = 0;
  int64_t P = 0;                     // look-back warps
  int64_t n_segs = 1, seg_chunks = 0;
  size_t off_flags = 0, off_carry = 0, off_seg_h = 0, off_seg_dsum = 0, off_seg_carry = 0;
  size_t off_bcf = 0;                // fp32 B and C (warp-specialised schedule)
  size_t ckpt_bytes = 0;             // saved states, right after the header
  size_t total = kHeaderBytes;
};

int64_t groups_for(const ssm_shape *s, int lpc) {
  const int64_t cpw = 32 / lpc;
  return s->batch * ((s->dim + cpw - 1) / cpw);
}

// Schedule choice.  The look-back schedule needs at least one channel group
// per warp slot it uses (P <= groups) and balances work exactly, so it is
// preferred whenever the problem has enough channel groups.  AUTO takes the
// warp-specialised kernel with 16-channel groups (2 lanes per channel) once
// there are 3/4 as many such groups as SM sub-partitions: even with a single
// producer / consumer pair on most sub-partitions it beats every other
// schedule there (measured on B200: 0.137 ms against 0.172 ms with 8-channel
// groups and 0.236 ms for the plain kernel at batch 8, d_inner 1024, L 2048).
// With fewer, the 8-channel-group version (4 lanes per channel) once those
// groups fill the sub-partitions (0.250 against 0.260 and 0.347 ms at batch 4,
// d_inner 1536, L 4096), the plain look-back kernel where the state count has
// no such version.  Long sequences with few channels take the two-pass
// split-L schedule; tiny problems one warp per group.
ssm_status make_fwd_plan(const ssm_shape *s, FwdPlan *pl) {
  ssm_status st = check_shape(s);
  if (st != SSM_OK) return st;
  FwdPlan p;
  p.NP = fwd_np_for(s->dstate);
  p.K = (s->seqlen + kT - 1) / kT;
  if (s->batch * s->dim == 0 || p.K == 0) {
    p.path = s->path == SSM_PATH_AUTO ? SSM_PATH_PER_GROUP : s->path;
    *pl = p;
    return SSM_OK;
  }
  const int sms = device_sms();
  if (sms <= 0) return SSM_ERR_CUDA;
  const int64_t unit = (int64_t)sms * kWarps;   // one warp per SM sub-partition
  const int64_t g2 = groups_for(s, 2), g4 = groups_for(s, 4);
  int path = s->path, lpc = s->lanes;
  const bool save = (s->flags & SSM_FLAG_SAVE_STATES) != 0;
  if (save || (s->flags & SSM_FLAG_TOKEN_MAJOR)) {  // both live in the warp-specialised kernel
    path = SSM_PATH_LOOKBACK_WS;
    lpc = 2;
  }
  if (save) p.ckpt_bytes = sizeof(float) * bwd_ckpt_floats(s->batch, s->dim, s->seqlen, p.NP);
  // the warp-specialised kernel with 4 lanes per channel exists for 8 and 16 padded states
  const bool ws4 = p.NP == 8 || p.NP == 16;
  if (lpc == 0) {
    if (path == SSM_PATH_SPLIT_L || path == SSM_PATH_LOOKBACK_WS) lpc = 2;
    else if (path == SSM_PATH_PER_GROUP) lpc = 4;
    else if (path == SSM_PATH_AUTO && 4 * g2 >= 3 * unit) lpc = 2;  // the warp-specialised kernel
    else if (g2 >= 2 * unit) lpc = 2;
    else if (g4 >= unit || path == SSM_PATH_LOOKBACK) lpc = 4;
    else lpc = p.K >= 64 ? 2 : 4;
  }
  int64_t G = lpc == 2 ? g2 : g4;
  // the exact-ZOH input term is built into the look-back kernels only
  const bool zoh = (s->flags & SSM_FLAG_ZOH_EXACT) != 0;
  if (path == SSM_PATH_AUTO) {
    if (lpc == 2 && 4 * G >= 3 * unit) path = SSM_PATH_LOOKBACK_WS;
    else if (G >= unit) path = (lpc == 2 || ws4) ? SSM_PATH_LOOKBACK_WS : SSM_PATH_LOOKBACK;
    else if (zoh) path = SSM_PATH_LOOKBACK;  // split-L and per-group are Euler only
    else if (p.K >= 64) path = SSM_PATH_SPLIT_L;
    else path = SSM_PATH_PER_GROUP;
  }
  int occ = 0;
  cudaError_t oe = cudaSuccess;
  if (path == SSM_PATH_LOOKBACK_WS) {
    oe = fwd_ws_occupancy(s->io_dtype, p.NP, lpc, &occ);
    // the warp-specialised kernel's shared memory does not fit every dtype and
    // state count (fp32 with 64 states needs more than a CTA may have, which
    // the occupancy query reports as an error): AUTO falls back to the plain
    // look-back kernel; an explicit request, saved states or token-major
    // activations (which need it) are refused
    if (oe != cudaSuccess || occ <= 0) {
      cudaGetLastError();
      oe = cudaSuccess;
      occ = 0;
      if (s->path != SSM_PATH_AUTO || save || (s->flags & SSM_FLAG_TOKEN_MAJOR)) return SSM_ERR_UNSUPPORTED;
      path = SSM_PATH_LOOKBACK;
      if (s->lanes == 0 && g2 < 2 * unit && g4 >= unit) {  // the plain kernel's own lane choice
        lpc = 4;
        G = g4;
      }
    }
  }
  if (path != SSM_PATH_LOOKBACK_WS) oe = fwd_occupancy(s->io_dtype, p.NP, lpc, zoh, &occ);
  if (oe != cudaSuccess || occ <= 0) {
    cudaGetLastError();
    return SSM_ERR_CUDA;
  }
  if (path == SSM_PATH_LOOKBACK_WS) {
    // a CTA holds fwd_ws_pairs() consumer warps (one per sub-partition); the
    // look-back items are (group, fwd_ws_chunk()-step chunk)
    occ = occ * fwd_ws_pairs() / kWarps;
    p.K = (s->seqlen + fwd_ws_chunk() - 1) / fwd_ws_chunk();
  }
  const int64_t slots = unit * occ;             // resident warps
  const int cpw = 32 / lpc;
  p.path = path;
  p.LPC = lpc;
  p.gpb = (s->dim + cpw - 1) / cpw;
  p.n_groups = G;
  if (path == SSM_PATH_LOOKBACK || path == SSM_PATH_LOOKBACK_WS) {
    // P <= groups keeps every warp's range at least one group long;
    // a multiple of `unit` gives every sub-partition the same work.
    int64_t r = G / unit;
    if (r > occ) r = occ;
    p.P = r >= 1 ? r * unit : G;
    if (p.P > slots) p.P = slots;  // all warps co-resident
    p.off_flags = round_up(kHeaderBytes + p.ckpt_bytes, 256);
    p.off_carry = round_up(p.off_flags + sizeof(unsigned) * (size_t)p.P, 256);
    p.total = round_up(p.off_carry + sizeof(float) * (size_t)p.P * cpw * p.NP, 256);
    if (path == SSM_PATH_LOOKBACK_WS) {  // fp32 B and C, [batch][L][NP] each
      p.off_bcf = p.total;
      p.total = round_up(p.off_bcf + 2 * sizeof(float) * (size_t)s->batch * (size_t)s->seqlen * p.NP, 256);
    }
  } else if (path == SSM_PATH_SPLIT_L) {
    // Segments per group.  Both passes launch one warp per (group, segment)
    // item: pass 1 (end states from zero) at its own occupancy, pass 2 (the
    // output pass, more registers) at a lower one.  The count minimises the
    // estimated time  sum over passes of  weight x waves x (segment length +
    // 2 chunks of per-item start-up), so that neither pass ends on a mostly
    // idle partial wave (pass 2, which also forms y, weighted 1.3); segments
    // hold at least 4 chunks, and the search stops at 8 waves of pass 1.
    int o1 = 0, o2 = 0;
    if (fwd_segment_occupancy(s->io_dtype, p.NP, lpc, 0, &o1) != cudaSuccess ||
        fwd_segment_occupancy(s->io_dtype, p.NP, lpc, 1, &o2) != cudaSuccess || o1 <= 0 || o2 <= 0) {
      cudaGetLastError();
      return SSM_ERR_CUDA;
    }
    const int64_t S1 = (int64_t)sms * o1 * kWarps, S2 = (int64_t)sms * o2 * kWarps;
    const int64_t max_segs = p.K / 4 > 1 ? p.K / 4 : 1;
    const int64_t min_segs = p.K >= 2 ? 2 : 1;
    const int64_t last = std::min(max_segs, std::max(min_segs, 8 * S1 / G));
    int64_t best = min_segs;
    double best_cost = 1e300;
    for (int64_t segs = min_segs; segs <= last; ++segs) {
      const int64_t sc = (p.K + segs - 1) / segs, ns = (p.K + sc - 1) / sc, items = G * ns;
      const double cost = (double)(sc + 2) * ((double)((items + S1 - 1) / S1) + 1.3 * (double)((items + S2 - 1) / S2));
      if (cost < best_cost * (1 - 1e-9)) {
        best_cost = cost;
        best = segs;
      }
    }
    p.seg_chunks = (p.K + best - 1) / best;
    p.n_segs = (p.K + p.seg_chunks - 1) / p.seg_chunks;
    const size_t items = (size_t)G * (size_t)p.n_segs;
    p.off_seg_h = kHeaderBytes;
    p.off_seg_dsum = round_up(p.off_seg_h + sizeof(float) * items * cpw * p.NP, 256);
    p.off_seg_carry = round_up(p.off_seg_dsum + sizeof(float) * items * cpw, 256);
    p.total = round_up(p.off_seg_carry + sizeof(float) * items * cpw * p.NP, 256);
  } else {
    p.n_segs = 1;
    p.seg_chunks = p.K;
  }
  *pl = p;
  return SSM_OK;
}

// Test hook (ssm_scan_test_fail_next): the number of upcoming entry-point
// calls that report a launch failure instead of launching.
std::atomic<int32_t> g_fail_next{0};

// Consumes one armed failure: cudaErrorLaunchFailure in place of the call's
// first launch (nothing is launched), else cudaSuccess.
cudaError_t injected_failure() {
  int32_t v = g_fail_next.load();
  while (v > 0 && !g_fail_next.compare_exchange_weak(v, v - 1)) {
  }
  return v > 0 ? cudaErrorLaunchFailure : cudaSuccess;
}

ssm_status cuda_status(cudaError_t e) {
  if (e == cudaSuccess) return SSM_OK;
  fprintf(stderr, "ssm_scan: CUDA error %s\n", cudaGetErrorString(e));
  return SSM_ERR_CUDA;
}

// Backward workspace: header, saved states (when the backward computes its
// own), then the per-block partial sums k_bwd_reduce adds in a fixed order.
struct BwdLayout {
  size_t off_ckpt, off_bc, off_a, off_d, off_bias, total;
};

BwdLayout bwd_layout(const ssm_shape *s) {
  const int NP = fwd_np_for(s->dstate);
  const size_t bd = (size_t)s->batch * (size_t)s->dim;
  BwdLayout l;
  l.off_ckpt = kHeaderBytes;
  l.off_bc = round_up(l.off_ckpt + sizeof(float) * bwd_ckpt_floats(s->batch, s->dim, s->seqlen, NP), 256);
  // dB/dC partials: [channel block][batch][seqlen][2 * NP]
  const size_t blocks = (size_t)bwd_blocks(s->dim, NP, s->flags & SSM_FLAG_ZOH_EXACT);
  l.off_a = round_up(l.off_bc + sizeof(float) * blocks * (size_t)s->batch * (size_t)s->seqlen * 2 * NP, 256);
  l.off_d = round_up(l.off_a + sizeof(float) * bd * (size_t)s->dstate, 256);
  l.off_bias = round_up(l.off_d + sizeof(float) * bd, 256);
  l.total = round_up(l.off_bias + sizeof(float) * bd, 256);
  return l;
}

}  // namespace

extern "C" {

size_t ssm_scan_bwd_workspace_bytes(const ssm_shape *shape) {
  if (check_shape(shape) != SSM_OK) return 0;
  return bwd_layout(shape).total;
}

const char *ssm_status_string(ssm_status s) {
  switch (s) {
    case SSM_OK: return "ok";
    case SSM_ERR_INVALID_ARG: return "invalid argument";
    case SSM_ERR_UNSUPPORTED: return "unsupported shape, dtype or path";
    case SSM_ERR_WORKSPACE: return "workspace missing or too small";
    case SSM_ERR_CUDA: return "CUDA error";
    case SSM_ERR_DEVICE_TIMEOUT: return "device-side wait timed out";
  }
  return "unknown status";
}

int32_t ssm_scan_version(void) { return kVersion; }

size_t ssm_scan_fwd_workspace_bytes(const ssm_shape *shape) {
  FwdPlan p;
  if (make_fwd_plan(shape, &p) != SSM_OK) return 0;
  return p.total;
}

int32_t ssm_scan_fwd_path(const ssm_shape *shape) {
  FwdPlan p;
  if (make_fwd_plan(shape, &p) != SSM_OK) return SSM_PATH_AUTO;
  return p.path;
}

ssm_status ssm_scan_fwd(const ssm_shape *shape, const void *u, const void *delta,
                        const float *A, const void *B, const void *C, const float *D,
                        const void *z, const float *delta_bias, int delta_softplus,
                        const float *initial_state, void *y, float *last_state,
                        void *workspace, size_t ws_bytes, ssm_stream_t stream) {
  ssm_status st = check_shape(shape);
  if (st != SSM_OK) return st;
  const int64_t nch = shape->batch * shape->dim;
  if (nch == 0) return SSM_OK;
  const cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const size_t es = shape->io_dtype == SSM_BF16 ? 2 : 4;
  if (shape->seqlen == 0) {  // nothing to scan: last_state = initial state
    if (!last_state) return SSM_OK;
    if (!aligned(last_state, 4) || !aligned(initial_state, 4)) return SSM_ERR_INVALID_ARG;
    const size_t bytes = sizeof(float) * (size_t)nch * (size_t)shape->dstate;
    return cuda_status(initial_state
                           ? cudaMemcpyAsync(last_state, initial_state, bytes, cudaMemcpyDeviceToDevice, s)
                           : cudaMemsetAsync(last_state, 0, bytes, s));
  }
  if (!u || !delta || !A || !B || !C || !y) return SSM_ERR_INVALID_ARG;
  if (!aligned(u, es) || !aligned(delta, es) || !aligned(B, es) || !aligned(C, es) ||
      !aligned(z, es) || !aligned(y, es) || !aligned(A, 4) || !aligned(D, 4) ||
      !aligned(delta_bias, 4) || !aligned(initial_state, 4) || !aligned(last_state, 4))
    return SSM_ERR_INVALID_ARG;
  FwdPlan pl;
  st = make_fwd_plan(shape, &pl);
  if (st != SSM_OK) return st;
  if (!workspace || ws_bytes < pl.total || !aligned(workspace, 256)) return SSM_ERR_WORKSPACE;

  FwdParams p;
  memset(&p, 0, sizeof(p));
  p.u = u; p.delta = delta; p.z = z; p.B = B; p.C = C;
  p.A = A; p.D = D; p.bias = delta_bias; p.h0 = initial_state;
  p.y = y; p.last_state = last_state;
  p.batch = shape->batch; p.dim = shape->dim; p.L = shape->seqlen; p.N = (int)shape->dstate;
  p.softplus = delta_softplus ? 1 : 0;
  p.zoh = (shape->flags & SSM_FLAG_ZOH_EXACT) ? 1 : 0;
  p.tok = (shape->flags & SSM_FLAG_TOKEN_MAJOR) ? 1 : 0;
  if (p.tok && !(aligned(u, 16) && aligned(delta, 16) && aligned(z, 16) && aligned(y, 16)))
    return SSM_ERR_INVALID_ARG;
  p.io_vec = ((shape->seqlen * es) % 16 == 0) && aligned(u, 16) && aligned(delta, 16) &&
             aligned(z, 16) && aligned(y, 16);
  p.bc_vec = (shape->dstate == pl.NP) && ((shape->dstate * es) % 16 == 0) && aligned(B, 16) &&
             aligned(C, 16);
  p.gpb = pl.gpb; p.n_groups = pl.n_groups; p.n_chunks = pl.K;
  p.n_workers = pl.P;
  char *ws = static_cast<char *>(workspace);
  p.err = reinterpret_cast<unsigned *>(ws);
  p.wait_limit_ns = kWaitLimitNs;
  p.n_segs = pl.n_segs; p.seg_chunks = pl.seg_chunks;
  if (pl.ckpt_bytes) p.ckpt_out = reinterpret_cast<float *>(ws + kHeaderBytes);

  // the error word starts clear on every path, so that ssm_scan_check reads
  // this call's status whatever the workspace held before
  cudaError_t e = injected_failure();
  if (e == cudaSuccess) e = cudaMemsetAsync(ws, 0, kHeaderBytes, s);
  if (e != cudaSuccess) return cuda_status(e);
  if (pl.path == SSM_PATH_LOOKBACK || pl.path == SSM_PATH_LOOKBACK_WS) {
    p.flags = reinterpret_cast<unsigned *>(ws + pl.off_flags);
    p.carry = reinterpret_cast<float *>(ws + pl.off_carry);
    e = cudaMemsetAsync(ws + pl.off_flags, 0, pl.off_carry - pl.off_flags, s);  // flags
    if (e != cudaSuccess) return cuda_status(e);
    if (pl.path == SSM_PATH_LOOKBACK_WS) {
      float *Bf = reinterpret_cast<float *>(ws + pl.off_bcf);
      float *Cf = Bf + (size_t)shape->batch * (size_t)shape->seqlen * pl.NP;
      p.Bf = Bf;
      p.Cf = Cf;
      e = launch_widen_bc(shape->io_dtype, B, C, Bf, Cf, shape->batch * shape->seqlen, (int)shape->dstate, pl.NP, s);
      if (e != cudaSuccess) return cuda_status(e);
    }
    e = pl.path == SSM_PATH_LOOKBACK_WS ? launch_fwd_ws(shape->io_dtype, pl.NP, pl.LPC, p, s)
                                        : launch_fwd_lookback(shape->io_dtype, pl.NP, pl.LPC, p, s);
  } else {
    if (pl.n_segs > 1) {
      p.seg_h = reinterpret_cast<float *>(ws + pl.off_seg_h);
      p.seg_dsum = reinterpret_cast<float *>(ws + pl.off_seg_dsum);
      p.seg_carry = reinterpret_cast<float *>(ws + pl.off_seg_carry);
    }
    e = launch_fwd_splitl(shape->io_dtype, pl.NP, pl.LPC, p, s);
  }
  return cuda_status(e);
}

ssm_status ssm_scan_step(const ssm_shape *shape, const void *u, const void *delta,
                         const float *A, const void *B, const void *C, const float *D,
                         const void *z, const float *delta_bias, int delta_softplus,
                         float *state, void *y, ssm_stream_t stream) {
  ssm_status st = check_shape(shape);
  if (st != SSM_OK) return st;
  if (shape->seqlen != 1) return SSM_ERR_INVALID_ARG;
  const int64_t nch = shape->batch * shape->dim;
  if (nch == 0) return SSM_OK;
  if (!u || !delta || !A || !B || !C || !state || !y) return SSM_ERR_INVALID_ARG;
  const size_t es = shape->io_dtype == SSM_BF16 ? 2 : 4;
  if (!aligned(u, es) || !aligned(delta, es) || !aligned(B, es) || !aligned(C, es) ||
      !aligned(z, es) || !aligned(y, es) || !aligned(A, 4) || !aligned(D, 4) ||
      !aligned(delta_bias, 4) || !aligned(state, 4))
    return SSM_ERR_INVALID_ARG;
  StepParams p;
  memset(&p, 0, sizeof(p));
  p.u = u; p.delta = delta; p.z = z; p.B = B; p.C = C;
  p.A = A; p.D = D; p.bias = delta_bias; p.state = state; p.y = y;
  p.batch = shape->batch; p.dim = shape->dim; p.N = (int)shape->dstate;
  p.softplus = delta_softplus ? 1 : 0;
  p.zoh = (shape->flags & SSM_FLAG_ZOH_EXACT) ? 1 : 0;
  p.vec = shape->dstate % 4 == 0 && aligned(state, 16) && aligned(A, 16) &&
          aligned(B, 4 * es) && aligned(C, 4 * es);
  const cudaError_t inj = injected_failure();
  if (inj != cudaSuccess) return cuda_status(inj);
  return cuda_status(launch_step(shape->io_dtype, p, reinterpret_cast<cudaStream_t>(stream)));
}

ssm_status ssm_causal_conv1d(int64_t batch, int64_t dim, int64_t seqlen, int32_t width,
                             int32_t io_dtype, const void *x, const float *weight,
                             const float *bias, const float *initial_state, int silu, void *out,
                             float *final_state, ssm_stream_t stream) {
  if (batch < 0 || dim < 0 || seqlen < 0 || width < 1) return SSM_ERR_INVALID_ARG;
  if (width > 8) return SSM_ERR_UNSUPPORTED;
  if (io_dtype != SSM_F32 && io_dtype != SSM_BF16) return SSM_ERR_UNSUPPORTED;
  if ((double)batch * (double)dim * (double)seqlen > 4.0e15) return SSM_ERR_UNSUPPORTED;
  const int64_t rows = batch * dim;
  if (rows == 0) return SSM_OK;
  const cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const size_t es = io_dtype == SSM_BF16 ? 2 : 4;
  if (!weight || !aligned(weight, 4) || !aligned(bias, 4) || !aligned(initial_state, 4) ||
      !aligned(final_state, 4))
    return SSM_ERR_INVALID_ARG;
  if (seqlen == 0) {  // nothing to convolve: the state passes through
    if (!final_state || width == 1) return SSM_OK;
    const size_t bytes = sizeof(float) * (size_t)rows * (size_t)(width - 1);
    return cuda_status(initial_state
                           ? cudaMemcpyAsync(final_state, initial_state, bytes, cudaMemcpyDeviceToDevice, s)
                           : cudaMemsetAsync(final_state, 0, bytes, s));
  }
  if (!x || !out || !aligned(x, es) || !aligned(out, es)) return SSM_ERR_INVALID_ARG;
  ConvParams p;
  memset(&p, 0, sizeof(p));
  p.x = x; p.w = weight; p.bias = bias; p.s0 = initial_state; p.out = out; p.s1 = final_state;
  p.batch = batch; p.dim = dim; p.L = seqlen; p.K = width; p.silu = silu ? 1 : 0;
  // 2: rows of whole 32-byte sectors on 32-byte aligned buffers (a lane's 16 steps move
  // in one 32-byte access); 1: 16-byte rows and buffers; 0: element accesses
  const bool row16 = ((seqlen * (int64_t)es) % 16 == 0) && aligned(x, 16) && aligned(out, 16);
  const bool row32 = ((seqlen * (int64_t)es) % 32 == 0) && aligned(x, 32) && aligned(out, 32);
  p.vec = row32 ? 2 : (row16 ? 1 : 0);
  const cudaError_t inj = injected_failure();
  if (inj != cudaSuccess) return cuda_status(inj);
  return cuda_status(launch_conv(io_dtype, p, s));
}

ssm_status ssm_causal_conv1d_bwd(int64_t batch, int64_t dim, int64_t seqlen, int32_t width,
                                 int32_t io_dtype, const void *x, const float *weight,
                                 const float *bias, const float *initial_state, int silu,
                                 const void *dout, void *dx, float *dweight, float *dbias,
                                 float *dinitial_state, ssm_stream_t stream) {
  if (batch < 0 || dim < 0 || seqlen < 0 || width < 1) return SSM_ERR_INVALID_ARG;
  if (width > 8) return SSM_ERR_UNSUPPORTED;
  if (io_dtype != SSM_F32 && io_dtype != SSM_BF16) return SSM_ERR_UNSUPPORTED;
  if ((double)batch * (double)dim * (double)seqlen > 4.0e15) return SSM_ERR_UNSUPPORTED;
  if ((bias == nullptr) != (dbias == nullptr)) return SSM_ERR_INVALID_ARG;
  const cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const size_t es = io_dtype == SSM_BF16 ? 2 : 4;
  if (dim > 0 && (!weight || !dweight)) return SSM_ERR_INVALID_ARG;
  if (!aligned(weight, 4) || !aligned(bias, 4) || !aligned(initial_state, 4) || !aligned(dweight, 4) ||
      !aligned(dbias, 4) || !aligned(dinitial_state, 4))
    return SSM_ERR_INVALID_ARG;
  const int64_t rows = batch * dim;
  // parameter gradients are sums: start from zero (also when there is no step)
  cudaError_t e = cudaSuccess;
  if (dim > 0) e = cudaMemsetAsync(dweight, 0, sizeof(float) * dim * width, s);
  if (e == cudaSuccess && dim > 0 && dbias) e = cudaMemsetAsync(dbias, 0, sizeof(float) * dim, s);
  if (e == cudaSuccess && rows > 0 && dinitial_state && width > 1)
    e = cudaMemsetAsync(dinitial_state, 0, sizeof(float) * rows * (width - 1), s);
  if (e != cudaSuccess || rows == 0 || seqlen == 0) return cuda_status(e);
  if (!x || !dout || !dx || !aligned(x, es) || !aligned(dout, es) || !aligned(dx, es))
    return SSM_ERR_INVALID_ARG;
  ConvBwdParams p;
  memset(&p, 0, sizeof(p));
  p.x = x; p.dout = dout; p.w = weight; p.bias = bias; p.s0 = initial_state;
  p.dx = dx; p.dw = dweight; p.dbias = dbias; p.ds0 = dinitial_state;
  p.batch = batch; p.dim = dim; p.L = seqlen; p.K = width; p.silu = silu ? 1 : 0;
  p.vec = ((seqlen * (int64_t)es) % 16 == 0) && aligned(x, 16) && aligned(dout, 16) && aligned(dx, 16);
  const cudaError_t inj = injected_failure();
  if (inj != cudaSuccess) return cuda_status(inj);
  return cuda_status(launch_conv_bwd(io_dtype, p, s));
}

ssm_status ssm_scan_bwd(const ssm_shape *shape, const void *u, const void *delta,
                        const float *A, const void *B, const void *C, const float *D,
                        const void *z, const float *delta_bias, int delta_softplus,
                        const float *initial_state, const void *dout, const void *fwd_workspace,
                        void *du, void *ddelta,
                        float *dA, void *dB, void *dC, float *dD, void *dz,
                        float *ddelta_bias, float *dinitial_state, void *workspace,
                        size_t ws_bytes, ssm_stream_t stream) {
  ssm_status st = check_shape(shape);
  if (st != SSM_OK) return st;
  // token-major activations: the d_state-16 kernel (dstate 9..16), bf16, Euler, dim % 8 == 0
  if ((shape->flags & SSM_FLAG_TOKEN_MAJOR) &&
      (fwd_np_for(shape->dstate) != 16 || shape->io_dtype != SSM_BF16 ||
       (shape->flags & SSM_FLAG_ZOH_EXACT) || shape->dim % 8 != 0))
    return SSM_ERR_UNSUPPORTED;
  // saved states come from a forward run with the same shape and flag
  if (fwd_workspace && (!(shape->flags & SSM_FLAG_SAVE_STATES) || !aligned(fwd_workspace, 256)))
    return SSM_ERR_INVALID_ARG;
  const cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const int64_t batch = shape->batch, dim = shape->dim, L = shape->seqlen, N = shape->dstate;
  const size_t es = shape->io_dtype == SSM_BF16 ? 2 : 4;
  if ((z == nullptr) != (dz == nullptr) || (D == nullptr) != (dD == nullptr) ||
      (delta_bias == nullptr) != (ddelta_bias == nullptr))
    return SSM_ERR_INVALID_ARG;
  if (batch * dim == 0 || L == 0) {  // no step to differentiate: parameter gradients are zero
    if (dim > 0 && (!dA || !aligned(dA, 4))) return SSM_ERR_INVALID_ARG;
    cudaError_t e = cudaSuccess;
    if (dim > 0) e = cudaMemsetAsync(dA, 0, sizeof(float) * dim * N, s);
    if (e == cudaSuccess && dim > 0 && dD) e = cudaMemsetAsync(dD, 0, sizeof(float) * dim, s);
    if (e == cudaSuccess && dim > 0 && ddelta_bias) e = cudaMemsetAsync(ddelta_bias, 0, sizeof(float) * dim, s);
    if (e == cudaSuccess && batch * dim > 0 && dinitial_state)
      e = cudaMemsetAsync(dinitial_state, 0, sizeof(float) * batch * dim * N, s);
    return cuda_status(e);
  }
  if (!u || !delta || !A || !B || !C || !dout || !du || !ddelta || !dA || !dB || !dC)
    return SSM_ERR_INVALID_ARG;
  if (!aligned(u, es) || !aligned(delta, es) || !aligned(B, es) || !aligned(C, es) ||
      !aligned(z, es) || !aligned(dout, es) || !aligned(du, es) || !aligned(ddelta, es) ||
      !aligned(dB, es) || !aligned(dC, es) || !aligned(dz, es) || !aligned(A, 4) ||
      !aligned(D, 4) || !aligned(delta_bias, 4) || !aligned(initial_state, 4) ||
      !aligned(dA, 4) || !aligned(dD, 4) || !aligned(ddelta_bias, 4) || !aligned(dinitial_state, 4))
    return SSM_ERR_INVALID_ARG;
  const BwdLayout lay = bwd_layout(shape);
  if (!workspace || ws_bytes < lay.total || !aligned(workspace, 256)) return SSM_ERR_WORKSPACE;
  const int NP = fwd_np_for(N);
  char *ws = static_cast<char *>(workspace);

  BwdParams p;
  memset(&p, 0, sizeof(p));
  p.u = u; p.delta = delta; p.z = z; p.B = B; p.C = C; p.dout = dout;
  p.A = A; p.D = D; p.bias = delta_bias; p.h0 = initial_state;
  p.du = du; p.ddelta = ddelta; p.dz = dz;
  p.dA = dA; p.dD = dD; p.dbias = ddelta_bias; p.dh0 = dinitial_state;
  if (fwd_workspace) {  // the forward's saved states, right after its header
    p.ckpt = reinterpret_cast<float *>(const_cast<char *>(static_cast<const char *>(fwd_workspace)) + kHeaderBytes);
    p.ckpt_given = 1;
  } else {
    p.ckpt = reinterpret_cast<float *>(ws + lay.off_ckpt);
  }
  p.dBC_part = reinterpret_cast<float *>(ws + lay.off_bc);
  p.dA_part = reinterpret_cast<float *>(ws + lay.off_a);
  p.dD_part = D ? reinterpret_cast<float *>(ws + lay.off_d) : nullptr;
  p.dbias_part = delta_bias ? reinterpret_cast<float *>(ws + lay.off_bias) : nullptr;
  p.dB = dB; p.dC = dC;
  p.batch = batch; p.dim = dim; p.L = L; p.N = (int)N;
  p.softplus = delta_softplus ? 1 : 0;
  p.zoh = (shape->flags & SSM_FLAG_ZOH_EXACT) ? 1 : 0;
  p.tok = (shape->flags & SSM_FLAG_TOKEN_MAJOR) ? 1 : 0;
  const bool act16 = aligned(u, 16) && aligned(delta, 16) && aligned(z, 16) && aligned(dout, 16) &&
                     aligned(du, 16) && aligned(ddelta, 16) && aligned(dz, 16);
  if (p.tok && !act16) return SSM_ERR_INVALID_ARG;
  p.io_vec = (p.tok || (L * (int64_t)es) % 16 == 0) && act16;
  p.bc_vec = (N == NP) && ((N * (int64_t)es) % 16 == 0) && aligned(B, 16) && aligned(C, 16);
  const cudaError_t inj = injected_failure();
  if (inj != cudaSuccess) return cuda_status(inj);
  return cuda_status(launch_bwd(shape->io_dtype, NP, p, s));
}

void ssm_scan_test_fail_next(int32_t count) { g_fail_next.store(count > 0 ? count : 0); }

ssm_status ssm_scan_check(void *workspace, ssm_stream_t stream) {
  if (!workspace) return SSM_ERR_WORKSPACE;
  const cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return cuda_status(e);
  unsigned word = 0;
  e = cudaMemcpy(&word, workspace, sizeof(word), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return cuda_status(e);
  if (word == 0) return SSM_OK;
  e = cudaMemset(workspace, 0, sizeof(word));
  if (e != cudaSuccess) return cuda_status(e);
  return SSM_ERR_DEVICE_TIMEOUT;
}

ssm_status ssm_scan_test_wait_timeout(void *workspace, size_t ws_bytes, int64_t timeout_us,
                                      ssm_stream_t stream) {
  if (!workspace || ws_bytes < kHeaderBytes || !aligned(workspace, 256)) return SSM_ERR_WORKSPACE;
  if (timeout_us < 1 || timeout_us > 1000000) return SSM_ERR_INVALID_ARG;
  const cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  char *ws = static_cast<char *>(workspace);
  cudaError_t e = cudaMemsetAsync(ws, 0, kHeaderBytes, s);
  if (e != cudaSuccess) return cuda_status(e);
  // the flag at byte 64 of the zeroed header is never set
  e = launch_wait_timeout_probe(reinterpret_cast<unsigned *>(ws + 64),
                                reinterpret_cast<unsigned *>(ws),
                                (unsigned long long)timeout_us * 1000ull, s);
  return cuda_status(e);
}

}  // extern "C"
