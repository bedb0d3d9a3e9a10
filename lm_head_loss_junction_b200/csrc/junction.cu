// Junction kernels: forward (rescale + gather + concat) and backward (do, de
// rows, and the residual-table gradient through the id-grouped row sums).
//
// The junction maps block m's output o_m[t] (width D_m) and the fresh residual
// embedding e_{m+1}[x_t] (width delta = D_{m+1} - D_m) to block m+1's input
//   y_t = [ s_t o_m[t] ; e_{m+1}[x_t] ],  s_t = ||e_{m+1}[x_t]|| / ||o_m[t]||
// ("Visualizing the core idea of Matryoshka LM Suites", bottom panel: the
// junction; "Matryoshka Language Model Suites", agihunt.info summary, junction
// paragraph).  It is pure HBM streaming: one warp per token, 16-byte vectors,
// the row kept in registers between the norm reduction and the store.
#include "common.cuh"
#include "kernels.h"

namespace mls {

namespace {

constexpr float kJunctionEps = 1e-12f;

// Element type traits: 16-byte vectors of 8 bf16 or 4 f32.
template <bool BF16> struct Elt;
template <> struct Elt<true> {
  static constexpr int kPerVec = 8;
  __device__ static void load(const uint4& u, float (&f)[8]) { bf16x8_to_f32(u, f); }
  __device__ static uint4 store(const float (&f)[8]) { return f32_to_bf16x8(f); }
};
template <> struct Elt<false> {
  static constexpr int kPerVec = 4;
  __device__ static void load(const uint4& u, float (&f)[4]) {
    f[0] = __uint_as_float(u.x); f[1] = __uint_as_float(u.y);
    f[2] = __uint_as_float(u.z); f[3] = __uint_as_float(u.w);
  }
  __device__ static uint4 store(const float (&f)[4]) {
    return make_uint4(__float_as_uint(f[0]), __float_as_uint(f[1]), __float_as_uint(f[2]),
                      __float_as_uint(f[3]));
  }
};

template <bool BF16>
__device__ __forceinline__ float sumsq(const uint4& u) {
  constexpr int N = Elt<BF16>::kPerVec;
  float f[N];
  Elt<BF16>::load(u, f);
  float s = 0.f;
#pragma unroll
  for (int i = 0; i < N; ++i) s = fmaf(f[i], f[i], s);
  return s;
}

template <bool BF16>
__device__ __forceinline__ float dotv(const uint4& a, const uint4& b) {
  constexpr int N = Elt<BF16>::kPerVec;
  float fa[N], fb[N];
  Elt<BF16>::load(a, fa);
  Elt<BF16>::load(b, fb);
  float s = 0.f;
#pragma unroll
  for (int i = 0; i < N; ++i) s = fmaf(fa[i], fb[i], s);
  return s;
}

template <bool BF16>
__device__ __forceinline__ uint4 scale_vec(const uint4& u, float s) {
  constexpr int N = Elt<BF16>::kPerVec;
  float f[N];
  Elt<BF16>::load(u, f);
#pragma unroll
  for (int i = 0; i < N; ++i) f[i] *= s;
  return Elt<BF16>::store(f);
}

// a*g - b*o, elementwise
template <bool BF16>
__device__ __forceinline__ uint4 axpby_vec(float a, const uint4& g, float b, const uint4& o) {
  constexpr int N = Elt<BF16>::kPerVec;
  float fg[N], fo[N];
  Elt<BF16>::load(g, fg);
  Elt<BF16>::load(o, fo);
#pragma unroll
  for (int i = 0; i < N; ++i) fg[i] = fmaf(a, fg[i], -b * fo[i]);
  return Elt<BF16>::store(fg);
}

// g + c*e, elementwise
template <bool BF16>
__device__ __forceinline__ uint4 add_scaled_vec(const uint4& g, float c, const uint4& e) {
  constexpr int N = Elt<BF16>::kPerVec;
  float fg[N], fe[N];
  Elt<BF16>::load(g, fg);
  Elt<BF16>::load(e, fe);
#pragma unroll
  for (int i = 0; i < N; ++i) fg[i] = fmaf(c, fe[i], fg[i]);
  return Elt<BF16>::store(fg);
}

// ga*g + c*e, elementwise
template <bool BF16>
__device__ __forceinline__ uint4 lincomb_vec(float ga, const uint4& g, float c, const uint4& e) {
  constexpr int N = Elt<BF16>::kPerVec;
  float fg[N], fe[N];
  Elt<BF16>::load(g, fg);
  Elt<BF16>::load(e, fe);
#pragma unroll
  for (int i = 0; i < N; ++i) fg[i] = fmaf(c, fe[i], ga * fg[i]);
  return Elt<BF16>::store(fg);
}

// Variant bits (see include/mls.h): 1 = no rescale, 2 = zero fill, 4 = stop-gradient.
constexpr uint32_t kNoRescale = 1, kZeroFill = 2, kStopGrad = 4;

// ---------------------------------------------------------------- forward
// One warp per token.  Pass 1 streams the block-output row (kept in registers,
// CAP 16-byte vectors per lane) and the embedding row (copied straight to the
// output: it does not depend on the scale) while accumulating both squared
// norms; pass 2 writes the rescaled block output from registers.  Columns
// beyond CAP*32 vectors are re-read in pass 2.
// Warps warp0, warp0 + nwarps, ... of the launch (or of its share of a launch) take tokens t = warp0 + k nwarps.
template <bool BF16, int CAP>
__device__ __forceinline__ void fwd_rows_body(int64_t warp0, int64_t nwarps, const int32_t* __restrict__ x,
                                              int64_t T, const uint4* __restrict__ o, int d_vec,
                                              const uint4* __restrict__ E, int64_t V, int dl_vec,
                                              uint4* __restrict__ y, float* __restrict__ scale_out,
                                              int32_t* __restrict__ status, uint32_t variant) {
  const int lane = threadIdx.x & 31;
  const bool zero_fill = (variant & kZeroFill) != 0;
  const int dp_vec = d_vec + dl_vec;
  const uint4 zero = make_uint4(0, 0, 0, 0);
  for (int64_t t = warp0; t < T; t += nwarps) {
    const int32_t id = __ldg(x + t);
    const bool bad = (id < 0) || (static_cast<int64_t>(id) >= V);
    const uint4* orow = o + t * d_vec;
    const uint4* erow = E + static_cast<int64_t>(bad ? 0 : id) * dl_vec;
    uint4* yrow = y + t * dp_vec;
    uint4 oc[CAP];
    float so = 0.f, se = 0.f;
#pragma unroll
    for (int j = 0; j < CAP; ++j) {
      const int i = j * 32 + lane;
      if (i < d_vec) oc[j] = __ldcs(orow + i);
    }
    // loads first, then the copies, in groups of 4 vectors per lane
    for (int i0 = lane; i0 < dl_vec; i0 += 4 * 32) {
      uint4 ev[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int i = i0 + u * 32;
        if (i < dl_vec) ev[u] = __ldg(erow + i);
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int i = i0 + u * 32;
        if (i < dl_vec) {
          se += sumsq<BF16>(ev[u]);
          yrow[d_vec + i] = (bad || zero_fill) ? zero : ev[u];
        }
      }
    }
#pragma unroll
    for (int j = 0; j < CAP; ++j) {
      const int i = j * 32 + lane;
      if (i < d_vec) so += sumsq<BF16>(oc[j]);
    }
    for (int i = CAP * 32 + lane; i < d_vec; i += 32) so += sumsq<BF16>(orow[i]);
    so = warp_sum(so);
    se = warp_sum(se);
    float s = (variant & kNoRescale) ? 1.f : sqrtf(se) / fmaxf(sqrtf(so), kJunctionEps);
    if (bad) s = 0.f;
#pragma unroll
    for (int j = 0; j < CAP; ++j) {
      const int i = j * 32 + lane;
      if (i < d_vec) yrow[i] = scale_vec<BF16>(oc[j], s);
    }
    for (int i = CAP * 32 + lane; i < d_vec; i += 32) yrow[i] = scale_vec<BF16>(orow[i], s);
    if (lane == 0) {
      if (scale_out != nullptr) scale_out[t] = s;
      if (bad) set_flag(status, MLS_DEVFLAG_BAD_ID);
    }
  }
}

template <bool BF16, int CAP>
__global__ void __launch_bounds__(256, 2) junction_fwd_kernel(const int32_t* __restrict__ x, int64_t T,
                                                           const uint4* __restrict__ o, int d_vec,
                                                           const uint4* __restrict__ E, int64_t V,
                                                           int dl_vec, uint4* __restrict__ y,
                                                           float* __restrict__ scale_out,
                                                           int32_t* __restrict__ status, uint32_t variant) {
  const int64_t warp0 = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
  fwd_rows_body<BF16, CAP>(warp0, nwarps, x, T, o, d_vec, E, V, dl_vec, y, scale_out, status, variant);
}

// Short rows (at most CAP = 4 vectors of o and ECAP = 6 of e per lane): a
// persistent grid of warps that each walk several tokens and load token
// t + nwarps's id, block-output row and embedding row into registers while
// token t is reduced and stored, so every warp keeps a row's worth of loads in
// flight and the launch has no partial last wave.
template <bool BF16, int CAP, int ECAP>
__device__ __forceinline__ void fwd_pipe_body(int64_t warp0, int64_t nwarps, const int32_t* __restrict__ x,
                                              int64_t T, const uint4* __restrict__ o, int d_vec,
                                              const uint4* __restrict__ E, int64_t V, int dl_vec,
                                              uint4* __restrict__ y, float* __restrict__ scale_out,
                                              int32_t* __restrict__ status, uint32_t variant) {
  const int lane = threadIdx.x & 31;
  const bool zero_fill = (variant & kZeroFill) != 0;
  int64_t t = warp0;
  if (t >= T) return;
  const int dp_vec = d_vec + dl_vec;
  const uint4 zero = make_uint4(0, 0, 0, 0);
  uint4 oc[CAP], ec[ECAP];
  bool bad;
  auto load_token = [&](int64_t tk, uint4 (&ov)[CAP], uint4 (&ev)[ECAP], bool& bd) {
    const int32_t id = __ldg(x + tk);
    bd = (id < 0) || (static_cast<int64_t>(id) >= V);
    const uint4* orow = o + tk * d_vec;
    const uint4* erow = E + static_cast<int64_t>(bd ? 0 : id) * dl_vec;
#pragma unroll
    for (int j = 0; j < CAP; ++j) {
      const int i = j * 32 + lane;
      ov[j] = (i < d_vec) ? __ldcs(orow + i) : zero;
    }
#pragma unroll
    for (int j = 0; j < ECAP; ++j) {
      const int i = j * 32 + lane;
      ev[j] = (i < dl_vec) ? __ldg(erow + i) : zero;
    }
  };
  load_token(t, oc, ec, bad);
  while (true) {
    const int64_t tn = t + nwarps;
    const bool has_next = tn < T;
    uint4 on[CAP], en[ECAP];
    bool badn = false;
    if (has_next) load_token(tn, on, en, badn);
    float so = 0.f, se = 0.f;
#pragma unroll
    for (int j = 0; j < CAP; ++j) so += sumsq<BF16>(oc[j]);
#pragma unroll
    for (int j = 0; j < ECAP; ++j) se += sumsq<BF16>(ec[j]);
    so = warp_sum(so);
    se = warp_sum(se);
    float s = (variant & kNoRescale) ? 1.f : sqrtf(se) / fmaxf(sqrtf(so), kJunctionEps);
    if (bad) s = 0.f;
    uint4* yrow = y + t * dp_vec;
#pragma unroll
    for (int j = 0; j < CAP; ++j) {
      const int i = j * 32 + lane;
      if (i < d_vec) yrow[i] = scale_vec<BF16>(oc[j], s);
    }
#pragma unroll
    for (int j = 0; j < ECAP; ++j) {
      const int i = j * 32 + lane;
      if (i < dl_vec) yrow[d_vec + i] = (bad || zero_fill) ? zero : ec[j];
    }
    if (lane == 0) {
      if (scale_out != nullptr) scale_out[t] = s;
      if (bad) set_flag(status, MLS_DEVFLAG_BAD_ID);
    }
    if (!has_next) break;
    t = tn;
    bad = badn;
#pragma unroll
    for (int j = 0; j < CAP; ++j) oc[j] = on[j];
#pragma unroll
    for (int j = 0; j < ECAP; ++j) ec[j] = en[j];
  }
}

template <bool BF16, int CAP, int ECAP>
__global__ void __launch_bounds__(256, 2) junction_fwd_pipe_kernel(const int32_t* __restrict__ x, int64_t T,
                                                                  const uint4* __restrict__ o, int d_vec,
                                                                  const uint4* __restrict__ E, int64_t V,
                                                                  int dl_vec, uint4* __restrict__ y,
                                                                  float* __restrict__ scale_out,
                                                                  int32_t* __restrict__ status, uint32_t variant) {
  const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
  const int64_t warp0 = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  fwd_pipe_body<BF16, CAP, ECAP>(warp0, nwarps, x, T, o, d_vec, E, V, dl_vec, y, scale_out, status, variant);
}

// Every junction of a suite in one persistent launch.  The launch's blocks are
// divided among the junctions in proportion to their bytes; each junction's
// share runs the prefetching body (short rows: at most PCAP vectors of o and
// PECAP of the embedding per lane) or the whole-row body (RCAP vectors of o
// per lane in registers), so no junction waits for another's tail.
struct MultiFwdJob {
  const uint4* o;
  const uint4* E;
  uint4* y;
  float* scale_out;
  int d_vec, dl_vec;
  int pipe;          // 1: prefetching body, 0: whole-row body
  int blk0;          // first block of this junction's share
};
struct MultiFwdArgs {
  MultiFwdJob j[kMaxExits - 1];
  int njobs;
  int blk_end;       // one past the last job's blocks
  const int32_t* x;
  int64_t T, V;
  int32_t* status;
};

template <int PCAP, int PECAP, int RCAP>
__global__ void __launch_bounds__(256, 2) junction_fwd_multi_kernel(const __grid_constant__ MultiFwdArgs a) {
  const int b = static_cast<int>(blockIdx.x);
  int k = 0;
  while (k + 1 < a.njobs && b >= a.j[k + 1].blk0) ++k;
  const MultiFwdJob& jb = a.j[k];
  const int b1 = (k + 1 < a.njobs) ? a.j[k + 1].blk0 : a.blk_end;
  const int64_t warp0 = (static_cast<int64_t>(b - jb.blk0) * blockDim.x + threadIdx.x) >> 5;
  const int64_t nwarps = (static_cast<int64_t>(b1 - jb.blk0) * blockDim.x) >> 5;
  if (jb.pipe)
    fwd_pipe_body<true, PCAP, PECAP>(warp0, nwarps, a.x, a.T, jb.o, jb.d_vec, jb.E, a.V, jb.dl_vec, jb.y,
                                     jb.scale_out, a.status, 0u);
  else
    fwd_rows_body<true, RCAP>(warp0, nwarps, a.x, a.T, jb.o, jb.d_vec, jb.E, a.V, jb.dl_vec, jb.y, jb.scale_out,
                              a.status, 0u);
}

// ---------------------------------------------------------------- backward
// do = s (g_o - u (u.g_o)),  de = g_e + (u.g_o) e_hat, written as
//   do = s g_o - (s ug / ||o||) o,   de = g_e + (ug / ||e||) e,   ug = o.g_o / ||o||.
// o and g_o stay in registers between the reductions and the do store; the
// embedding row is read again for de (it was just read, so from cache).
// When coef_out is given, c_t = ug/||e|| is stored for the table scatter.
template <bool BF16, int CAP, int MINB>
__global__ void __launch_bounds__(256, MINB) junction_bwd_kernel(
    const int32_t* __restrict__ x, int64_t T, const uint4* __restrict__ o, int d_vec,
    const uint4* __restrict__ E, int64_t V, int dl_vec, const uint4* __restrict__ dy,
    uint4* __restrict__ do_out, uint4* __restrict__ de_out, float* __restrict__ coef_out,
    int32_t* __restrict__ status, uint32_t variant) {
  const int lane = threadIdx.x & 31;
  const int64_t warp0 = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
  const int dp_vec = d_vec + dl_vec;
  const uint4 zero = make_uint4(0, 0, 0, 0);
  for (int64_t t = warp0; t < T; t += nwarps) {
    const int32_t id = __ldg(x + t);
    const bool bad = (id < 0) || (static_cast<int64_t>(id) >= V);
    const uint4* orow = o + t * d_vec;
    const uint4* grow = dy + t * dp_vec;
    const uint4* erow = E + static_cast<int64_t>(bad ? 0 : id) * dl_vec;
    uint4 oc[CAP], gc[CAP];
    float so = 0.f, sog = 0.f, se = 0.f;
#pragma unroll
    for (int j = 0; j < CAP; ++j) {
      const int i = j * 32 + lane;
      if (i < d_vec) {
        oc[j] = __ldcs(orow + i);
        gc[j] = __ldcs(grow + i);
      }
    }
#pragma unroll 4
    for (int i = lane; i < dl_vec; i += 32) se += sumsq<BF16>(__ldg(erow + i));
#pragma unroll
    for (int j = 0; j < CAP; ++j) {
      const int i = j * 32 + lane;
      if (i < d_vec) {
        so += sumsq<BF16>(oc[j]);
        sog += dotv<BF16>(oc[j], gc[j]);
      }
    }
    for (int i = CAP * 32 + lane; i < d_vec; i += 32) {
      const uint4 ov = orow[i], gv = grow[i];
      so += sumsq<BF16>(ov);
      sog += dotv<BF16>(ov, gv);
    }
    so = warp_sum(so);
    sog = warp_sum(sog);
    se = warp_sum(se);
    const float n_o = fmaxf(sqrtf(so), kJunctionEps);
    const float n_e = sqrtf(se);
    const float s = n_e / n_o;
    const float ug = sog / n_o;
    float a = s, b = s * ug / n_o, c = (n_e > 0.f) ? ug / n_e : 0.f;
    if (variant & kNoRescale) { a = 1.f; b = 0.f; c = 0.f; }   // y = [o ; .]
    if (variant & kStopGrad) { a = 0.f; b = 0.f; }              // nothing flows into o
    const float ge = (variant & kZeroFill) ? 0.f : 1.f;         // the fill does not carry g_e
    if (bad) { a = 0.f; b = 0.f; c = 0.f; }
    uint4* drow = do_out + t * d_vec;
#pragma unroll
    for (int j = 0; j < CAP; ++j) {
      const int i = j * 32 + lane;
      if (i < d_vec) drow[i] = axpby_vec<BF16>(a, gc[j], b, oc[j]);
    }
    for (int i = CAP * 32 + lane; i < d_vec; i += 32) drow[i] = axpby_vec<BF16>(a, grow[i], b, orow[i]);
    if (de_out != nullptr) {
      uint4* erow_out = de_out + t * dl_vec;
      for (int i0 = lane; i0 < dl_vec; i0 += 4 * 32) {
        uint4 gv[4], ev[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int i = i0 + u * 32;
          if (i < dl_vec) {
            gv[u] = __ldcs(grow + d_vec + i);
            ev[u] = __ldg(erow + i);
          }
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int i = i0 + u * 32;
          if (i < dl_vec) erow_out[i] = bad ? zero : lincomb_vec<BF16>(ge, gv[u], c, ev[u]);
        }
      }
    }
    if (lane == 0) {
      if (coef_out != nullptr) coef_out[t] = c;
      if (bad) set_flag(status, MLS_DEVFLAG_BAD_ID);
    }
  }
}

// Short block-output rows (at most CAP = 2 vectors per lane): a persistent grid
// of warps that each walk several tokens and load token t + nwarps's id, o row
// and g_o row into registers while token t is reduced and stored; the
// embedding row and g_e stream as in junction_bwd_kernel.
template <bool BF16, int CAP>
__global__ void __launch_bounds__(256, 2) junction_bwd_pipe_kernel(
    const int32_t* __restrict__ x, int64_t T, const uint4* __restrict__ o, int d_vec,
    const uint4* __restrict__ E, int64_t V, int dl_vec, const uint4* __restrict__ dy,
    uint4* __restrict__ do_out, uint4* __restrict__ de_out, float* __restrict__ coef_out,
    int32_t* __restrict__ status, uint32_t variant) {
  const int lane = threadIdx.x & 31;
  const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
  int64_t t = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  if (t >= T) return;
  const int dp_vec = d_vec + dl_vec;
  const uint4 zero = make_uint4(0, 0, 0, 0);
  uint4 oc[CAP], gc[CAP];
  int32_t id;
  auto load_og = [&](int64_t tk, uint4 (&ov)[CAP], uint4 (&gv)[CAP], int32_t& idk) {
    idk = __ldg(x + tk);
    const uint4* orow = o + tk * d_vec;
    const uint4* grow = dy + tk * dp_vec;
#pragma unroll
    for (int j = 0; j < CAP; ++j) {
      const int i = j * 32 + lane;
      ov[j] = (i < d_vec) ? __ldcs(orow + i) : zero;
      gv[j] = (i < d_vec) ? __ldcs(grow + i) : zero;
    }
  };
  load_og(t, oc, gc, id);
  while (true) {
    const int64_t tn = t + nwarps;
    const bool has_next = tn < T;
    uint4 on[CAP], gn[CAP];
    int32_t idn = 0;
    if (has_next) load_og(tn, on, gn, idn);
    const bool bad = (id < 0) || (static_cast<int64_t>(id) >= V);
    const uint4* grow = dy + t * dp_vec;
    const uint4* erow = E + static_cast<int64_t>(bad ? 0 : id) * dl_vec;
    float so = 0.f, sog = 0.f, se = 0.f;
#pragma unroll 4
    for (int i = lane; i < dl_vec; i += 32) se += sumsq<BF16>(__ldg(erow + i));
#pragma unroll
    for (int j = 0; j < CAP; ++j) {
      so += sumsq<BF16>(oc[j]);
      sog += dotv<BF16>(oc[j], gc[j]);
    }
    so = warp_sum(so);
    sog = warp_sum(sog);
    se = warp_sum(se);
    const float n_o = fmaxf(sqrtf(so), kJunctionEps);
    const float n_e = sqrtf(se);
    const float s = n_e / n_o;
    const float ug = sog / n_o;
    float a = s, b = s * ug / n_o, c = (n_e > 0.f) ? ug / n_e : 0.f;
    if (variant & kNoRescale) { a = 1.f; b = 0.f; c = 0.f; }   // y = [o ; .]
    if (variant & kStopGrad) { a = 0.f; b = 0.f; }              // nothing flows into o
    const float ge = (variant & kZeroFill) ? 0.f : 1.f;         // the fill does not carry g_e
    if (bad) { a = 0.f; b = 0.f; c = 0.f; }
    uint4* drow = do_out + t * d_vec;
#pragma unroll
    for (int j = 0; j < CAP; ++j) {
      const int i = j * 32 + lane;
      if (i < d_vec) drow[i] = axpby_vec<BF16>(a, gc[j], b, oc[j]);
    }
    if (de_out != nullptr) {
      uint4* erow_out = de_out + t * dl_vec;
      constexpr int kDeGroup = 4;                      // vectors per lane in flight
      for (int i0 = lane; i0 < dl_vec; i0 += kDeGroup * 32) {
        uint4 gv[kDeGroup], ev[kDeGroup];
#pragma unroll
        for (int u = 0; u < kDeGroup; ++u) {
          const int i = i0 + u * 32;
          if (i < dl_vec) {
            gv[u] = __ldcs(grow + d_vec + i);
            ev[u] = __ldg(erow + i);
          }
        }
#pragma unroll
        for (int u = 0; u < kDeGroup; ++u) {
          const int i = i0 + u * 32;
          if (i < dl_vec) erow_out[i] = bad ? zero : lincomb_vec<BF16>(ge, gv[u], c, ev[u]);
        }
      }
    }
    if (lane == 0) {
      if (coef_out != nullptr) coef_out[t] = c;
      if (bad) set_flag(status, MLS_DEVFLAG_BAD_ID);
    }
    if (!has_next) break;
    t = tn;
    id = idn;
#pragma unroll
    for (int j = 0; j < CAP; ++j) {
      oc[j] = on[j];
      gc[j] = gn[j];
    }
  }
}

// Short rows (at most CAP = 4 vectors of o and ECAP = 5 of the embedding per
// lane): every row of the token (o, g_o, e, g_e) is loaded into registers
// before any reduction, so a token costs one round trip to memory; the
// embedding row is read once.
template <bool BF16, int CAP, int ECAP>
__global__ void __launch_bounds__(256, 2) junction_bwd_rows_kernel(
    const int32_t* __restrict__ x, int64_t T, const uint4* __restrict__ o, int d_vec,
    const uint4* __restrict__ E, int64_t V, int dl_vec, const uint4* __restrict__ dy,
    uint4* __restrict__ do_out, uint4* __restrict__ de_out, float* __restrict__ coef_out,
    int32_t* __restrict__ status, uint32_t variant) {
  const int lane = threadIdx.x & 31;
  const int64_t warp0 = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
  const int dp_vec = d_vec + dl_vec;
  const uint4 zero = make_uint4(0, 0, 0, 0);
  for (int64_t t = warp0; t < T; t += nwarps) {
    const int32_t id = __ldg(x + t);
    const bool bad = (id < 0) || (static_cast<int64_t>(id) >= V);
    const uint4* orow = o + t * d_vec;
    const uint4* grow = dy + t * dp_vec;
    const uint4* erow = E + static_cast<int64_t>(bad ? 0 : id) * dl_vec;
    uint4 oc[CAP], gc[CAP], ec[ECAP], gec[ECAP];
#pragma unroll
    for (int j = 0; j < CAP; ++j) {
      const int i = j * 32 + lane;
      oc[j] = (i < d_vec) ? __ldcs(orow + i) : zero;
      gc[j] = (i < d_vec) ? __ldcs(grow + i) : zero;
    }
#pragma unroll
    for (int j = 0; j < ECAP; ++j) {
      const int i = j * 32 + lane;
      ec[j] = (i < dl_vec) ? __ldg(erow + i) : zero;
      gec[j] = (i < dl_vec) ? __ldcs(grow + d_vec + i) : zero;
    }
    float so = 0.f, sog = 0.f, se = 0.f;
#pragma unroll
    for (int j = 0; j < ECAP; ++j) se += sumsq<BF16>(ec[j]);
#pragma unroll
    for (int j = 0; j < CAP; ++j) {
      so += sumsq<BF16>(oc[j]);
      sog += dotv<BF16>(oc[j], gc[j]);
    }
    so = warp_sum(so);
    sog = warp_sum(sog);
    se = warp_sum(se);
    const float n_o = fmaxf(sqrtf(so), kJunctionEps);
    const float n_e = sqrtf(se);
    const float s = n_e / n_o;
    const float ug = sog / n_o;
    float a = s, b = s * ug / n_o, c = (n_e > 0.f) ? ug / n_e : 0.f;
    if (variant & kNoRescale) { a = 1.f; b = 0.f; c = 0.f; }   // y = [o ; .]
    if (variant & kStopGrad) { a = 0.f; b = 0.f; }              // nothing flows into o
    const float ge = (variant & kZeroFill) ? 0.f : 1.f;         // the fill does not carry g_e
    if (bad) { a = 0.f; b = 0.f; c = 0.f; }
    uint4* drow = do_out + t * d_vec;
#pragma unroll
    for (int j = 0; j < CAP; ++j) {
      const int i = j * 32 + lane;
      if (i < d_vec) drow[i] = axpby_vec<BF16>(a, gc[j], b, oc[j]);
    }
    if (de_out != nullptr) {
      uint4* erow_out = de_out + t * dl_vec;
#pragma unroll
      for (int j = 0; j < ECAP; ++j) {
        const int i = j * 32 + lane;
        if (i < dl_vec) erow_out[i] = bad ? zero : lincomb_vec<BF16>(ge, gec[j], c, ec[j]);
      }
    }
    if (lane == 0) {
      if (coef_out != nullptr) coef_out[t] = c;
      if (bad) set_flag(status, MLS_DEVFLAG_BAD_ID);
    }
  }
}

int pick_cap(int nvec) {
  const int per_lane = (nvec + 31) / 32;
  static const int caps[] = {1, 2, 4, 6, 8, 9, 12, 16};
  for (int c : caps)
    if (per_lane <= c) return c;
  return 16;
}

int grid_for(int64_t T, int warps_per_block) {
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int64_t need = (T + warps_per_block - 1) / warps_per_block;
  const int64_t cap = static_cast<int64_t>(sms) * 8;
  return static_cast<int>(need < cap ? (need > 0 ? need : 1) : cap);
}

template <bool BF16>
cudaError_t launch_fwd_t(const JunctionArgs& a, cudaStream_t st) {
  constexpr int N = Elt<BF16>::kPerVec;
  const int d_vec = static_cast<int>(a.D / N), dl_vec = static_cast<int>(a.delta / N);
  const int cap = pick_cap(d_vec);
  const int ecap = pick_cap(dl_vec);
  auto* o = static_cast<const uint4*>(a.o);
  auto* E = static_cast<const uint4*>(a.E);
  auto* y = static_cast<uint4*>(a.y);
  if (cap <= 4 && ecap <= 6) {
    // short rows: a persistent grid (two 8-warp blocks per SM) of prefetching warps
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int64_t need = (a.T + 7) / 8;
    const int pgrid = static_cast<int>(need < 2 * sms ? (need > 0 ? need : 1) : 2 * sms);
#define MLS_JFP(C, EC) junction_fwd_pipe_kernel<BF16, C, EC><<<pgrid, 256, 0, st>>>(a.x, a.T, o, d_vec, E, a.V, dl_vec, y, a.scale_out, a.status, a.variant)
#define MLS_JFP_E(C)              \
  switch (ecap) {                 \
    case 1: MLS_JFP(C, 1); break; \
    case 2: MLS_JFP(C, 2); break; \
    case 4: MLS_JFP(C, 4); break; \
    default: MLS_JFP(C, 6); break; \
  }
    switch (cap) {
      case 1: MLS_JFP_E(1); break;
      case 2: MLS_JFP_E(2); break;
      default: MLS_JFP_E(4); break;
    }
#undef MLS_JFP_E
#undef MLS_JFP
    note_launches(1);
    return cudaGetLastError();
  }
  const int grid = grid_for(a.T, 8);
#define MLS_JF(C) junction_fwd_kernel<BF16, C><<<grid, 256, 0, st>>>(a.x, a.T, o, d_vec, E, a.V, dl_vec, y, a.scale_out, a.status, a.variant)
  switch (cap) {
    case 1: MLS_JF(1); break;
    case 2: MLS_JF(2); break;
    case 4: MLS_JF(4); break;
    case 6: MLS_JF(6); break;
    case 8: MLS_JF(8); break;
    case 9: MLS_JF(9); break;
    case 12: MLS_JF(12); break;
    default: MLS_JF(16); break;
  }
#undef MLS_JF
  note_launches(1);
  return cudaGetLastError();
}

// The row kernels of one junction backward: do, de rows, and (coef != NULL)
// the per-token coefficients of the table gradient.
template <bool BF16>
cudaError_t launch_bwd_rows_t(const JunctionArgs& a, float* coef, cudaStream_t st) {
  constexpr int N = Elt<BF16>::kPerVec;
  const int d_vec = static_cast<int>(a.D / N), dl_vec = static_cast<int>(a.delta / N);
  const int cap = pick_cap(d_vec);
  const int grid = grid_for(a.T, 8);
  auto* o = static_cast<const uint4*>(a.o);
  auto* E = static_cast<const uint4*>(a.E);
  auto* dy = static_cast<const uint4*>(a.dy);
  auto* dout = static_cast<uint4*>(a.do_out);
  auto* deo = static_cast<uint4*>(a.de_out);
  // Measured on the B200 (fraction of the copy bandwidth, T = 8192 .. 32768):
  //  - rows of <= 2 vectors per lane: the prefetching persistent kernel
  //    (512 -> 1024: 0.71 against 0.50-0.56);
  //  - 4 vectors per lane: whole rows in registers, 2 blocks per SM (the
  //    prefetching form, at 128 registers, was 0.49-0.68 against 0.60-0.80);
  //  - longer rows: 4 blocks per SM with 2 vectors of o and g_o per lane in
  //    registers and the rest re-read from L1 (2304 -> 4352: 0.74-0.84
  //    against 0.60-0.68 with whole rows in registers at 2 blocks per SM).
  if (cap <= 2) {
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int64_t need = (a.T + 7) / 8;
    const int pgrid = static_cast<int>(need < 2 * sms ? (need > 0 ? need : 1) : 2 * sms);
#define MLS_JBP(C) junction_bwd_pipe_kernel<BF16, C><<<pgrid, 256, 0, st>>>(a.x, a.T, o, d_vec, E, a.V, dl_vec, dy, dout, deo, coef, a.status, a.variant)
    if (cap == 1) MLS_JBP(1);
    else MLS_JBP(2);
#undef MLS_JBP
  } else {
#define MLS_JB(C, B) junction_bwd_kernel<BF16, C, B><<<grid, 256, 0, st>>>(a.x, a.T, o, d_vec, E, a.V, dl_vec, dy, dout, deo, coef, a.status, a.variant)
#define MLS_JBR(C, EC) junction_bwd_rows_kernel<BF16, C, EC><<<grid, 256, 0, st>>>(a.x, a.T, o, d_vec, E, a.V, dl_vec, dy, dout, deo, coef, a.status, a.variant)
    const int ecap = (dl_vec + 31) / 32;              // exact: every register row is used
    if (cap == 4 && ecap <= 5) {
      switch (ecap) {
        case 1: MLS_JBR(4, 1); break;
        case 2: MLS_JBR(4, 2); break;
        case 3: MLS_JBR(4, 3); break;
        case 4: MLS_JBR(4, 4); break;
        default: MLS_JBR(4, 5); break;
      }
    } else if (cap == 4) {
      MLS_JB(4, 2);
    } else {
      MLS_JB(2, 4);
    }
#undef MLS_JBR
#undef MLS_JB
  }
  note_launches(1);
  return cudaGetLastError();
}

size_t coef_bytes(int64_t T) { return (static_cast<size_t>(T) * 4 + 255) & ~size_t(255); }

template <bool BF16>
cudaError_t launch_bwd_t(const JunctionArgs& a, cudaStream_t st) {
  float* coef = a.dE != nullptr ? static_cast<float*>(a.workspace) : nullptr;
  cudaError_t err = launch_bwd_rows_t<BF16>(a, coef, st);
  if (err != cudaSuccess || a.dE == nullptr) return err;
  // Table gradient: tokens grouped by id, fixed-order row sums.
  constexpr int N = Elt<BF16>::kPerVec;
  SegIndexDev ix;
  err = build_segindex(a.x, a.T, a.V, static_cast<char*>(a.workspace) + coef_bytes(a.T), &ix, st);
  if (err != cudaSuccess) return err;
  const float ge = (a.variant & kZeroFill) ? 0.f : 1.f;
  return scatter_table_grad(ix, BF16, a.dy, static_cast<int>(a.D / N), static_cast<int>(a.delta / N), coef, ge, a.E,
                            a.dE, a.accumulate_dE != 0, st);
}

}  // namespace

size_t junction_scatter_bytes(int64_t T, int64_t V) { return coef_bytes(T) + segindex_bytes(T, V); }

size_t junction_multi_scatter_bytes(int64_t T, int64_t V, int J) {
  return coef_bytes(T) * static_cast<size_t>(J) + segindex_bytes(T, V);
}

// All junctions of a suite (they share the ids x and T).  bf16: one launch
// whose blocks are split among the junctions; fp32: one launch per junction.
cudaError_t launch_junction_fwd_multi(const JunctionArgs* js, int J, cudaStream_t st) {
  if (!js[0].bf16) {
    for (int k = 0; k < J; ++k) {
      const cudaError_t err = launch_fwd_t<false>(js[k], st);
      if (err != cudaSuccess) return err;
    }
    return cudaSuccess;
  }
  constexpr int N = 8;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int total_blocks = 2 * sms;              // two 8-warp blocks per SM, persistent
  const int64_t T = js[0].T;
  const int64_t need = (T + 7) / 8;              // blocks that give every token a warp
  MultiFwdArgs m{};
  m.njobs = J;
  m.x = js[0].x;
  m.T = T;
  m.V = js[0].V;
  m.status = js[0].status;
  double bytes[kMaxExits - 1], sum = 0.0;
  int rcap = 1;
  for (int k = 0; k < J; ++k) {
    const JunctionArgs& a = js[k];
    MultiFwdJob& jb = m.j[k];
    jb.o = static_cast<const uint4*>(a.o);
    jb.E = static_cast<const uint4*>(a.E);
    jb.y = static_cast<uint4*>(a.y);
    jb.scale_out = a.scale_out;
    jb.d_vec = static_cast<int>(a.D / N);
    jb.dl_vec = static_cast<int>(a.delta / N);
    jb.pipe = (pick_cap(jb.d_vec) <= 4 && pick_cap(jb.dl_vec) <= 6) ? 1 : 0;
    if (!jb.pipe) rcap = pick_cap(jb.d_vec) > rcap ? pick_cap(jb.d_vec) : rcap;
    bytes[k] = static_cast<double>(2 * jb.d_vec + 2 * jb.dl_vec);
    sum += bytes[k];
  }
  int next = 0;
  for (int k = 0; k < J; ++k) {
    int64_t nb = static_cast<int64_t>(total_blocks * bytes[k] / sum + 0.5);
    nb = nb < 1 ? 1 : (nb > need ? need : nb);
    m.j[k].blk0 = next;
    next += static_cast<int>(nb);
  }
  m.blk_end = next;
  if (rcap <= 1) junction_fwd_multi_kernel<4, 6, 1><<<next, 256, 0, st>>>(m);
  else if (rcap <= 9) junction_fwd_multi_kernel<4, 6, 9><<<next, 256, 0, st>>>(m);
  else junction_fwd_multi_kernel<4, 6, 16><<<next, 256, 0, st>>>(m);
  note_launches(1);
  return cudaGetLastError();
}

// The row kernels of every junction, then one id grouping shared by all table
// gradients and one launch set of row-sum passes over all tables.  On the
// side stream: the id grouping (latency-bound, reads only x) beside the row
// kernels, then the heavy rows' sums beside the pass over the other rows.
cudaError_t launch_junction_bwd_multi(const JunctionArgs* js, int J, bool any_table, void* ws, cudaStream_t st) {
  const bool bf16 = js[0].bf16;
  const int64_t T = js[0].T;
  float* coef[kMaxExits - 1] = {};
  SegIndexDev ix;
  SideScope side(st);
  cudaError_t err = cudaSuccess;
  if (any_table) {
    err = build_segindex(js[0].x, T, js[0].V, static_cast<char*>(ws) + coef_bytes(T) * J, &ix, side.stream());
    if (err != cudaSuccess) return err;
  }
  for (int k = 0; k < J; ++k) {
    coef[k] = js[k].dE != nullptr ? reinterpret_cast<float*>(static_cast<char*>(ws) + coef_bytes(T) * k) : nullptr;
    err = bf16 ? launch_bwd_rows_t<true>(js[k], coef[k], st) : launch_bwd_rows_t<false>(js[k], coef[k], st);
    if (err != cudaSuccess) return err;
  }
  err = side.join();
  if (err != cudaSuccess || !any_table) return err;
  const int N = bf16 ? 8 : 4;
  TableGradJob jobs[kMaxExits - 1];
  int n = 0;
  for (int k = 0; k < J; ++k) {
    if (js[k].dE == nullptr) continue;
    jobs[n++] = TableGradJob{js[k].dy, static_cast<int>(js[k].D / N), static_cast<int>(js[k].delta / N), coef[k],
                             1.f, js[k].E, js[k].dE};
  }
  err = side.fork();
  if (err != cudaSuccess) return err;
  err = scatter_table_grads(ix, bf16, n, jobs, js[0].accumulate_dE != 0, st, side.stream());
  if (err != cudaSuccess) return err;
  return side.join();
}

cudaError_t launch_junction_fwd(const JunctionArgs& a, cudaStream_t st) {
  return a.bf16 ? launch_fwd_t<true>(a, st) : launch_fwd_t<false>(a, st);
}

cudaError_t launch_junction_bwd(const JunctionArgs& a, cudaStream_t st) {
  return a.bf16 ? launch_bwd_t<true>(a, st) : launch_bwd_t<false>(a, st);
}

}  // namespace mls
