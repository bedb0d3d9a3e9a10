// Junction kernels: forward (rescale + gather + concat), backward (do, de rows)
// and the deterministic scatter of de into the residual-embedding table.
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

// ---------------------------------------------------------------- forward
// CAP = 16-byte vectors per lane kept in registers; columns beyond
// CAP*32 vectors are re-read in the second pass.
template <bool BF16, int CAP>
__global__ void __launch_bounds__(256) junction_fwd_kernel(const int32_t* __restrict__ x, int64_t T,
                                                           const uint4* __restrict__ o, int d_vec,
                                                           const uint4* __restrict__ E, int64_t V,
                                                           int dl_vec, uint4* __restrict__ y,
                                                           float* __restrict__ scale_out,
                                                           int32_t* __restrict__ status) {
  const int lane = threadIdx.x & 31;
  const int64_t warp0 = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
  const int dp_vec = d_vec + dl_vec;
  for (int64_t t = warp0; t < T; t += nwarps) {
    const int32_t id = __ldg(x + t);
    const bool bad = (id < 0) || (static_cast<int64_t>(id) >= V);
    const uint4* orow = o + t * d_vec;
    const uint4* erow = E + static_cast<int64_t>(bad ? 0 : id) * dl_vec;
    uint4 oc[CAP], ec[CAP];
    float so = 0.f, se = 0.f;
#pragma unroll
    for (int j = 0; j < CAP; ++j) {
      const int i = j * 32 + lane;
      if (i < d_vec) { oc[j] = __ldcs(orow + i); so += sumsq<BF16>(oc[j]); }
      if (i < dl_vec) { ec[j] = __ldg(erow + i); se += sumsq<BF16>(ec[j]); }
    }
    for (int i = CAP * 32 + lane; i < d_vec; i += 32) so += sumsq<BF16>(orow[i]);
    for (int i = CAP * 32 + lane; i < dl_vec; i += 32) se += sumsq<BF16>(__ldg(erow + i));
    so = warp_sum(so);
    se = warp_sum(se);
    float s = sqrtf(se) / fmaxf(sqrtf(so), kJunctionEps);
    if (bad) s = 0.f;
    uint4* yrow = y + t * dp_vec;
    const uint4 zero = make_uint4(0, 0, 0, 0);
#pragma unroll
    for (int j = 0; j < CAP; ++j) {
      const int i = j * 32 + lane;
      if (i < d_vec) yrow[i] = scale_vec<BF16>(oc[j], s);
      if (i < dl_vec) yrow[d_vec + i] = bad ? zero : ec[j];
    }
    for (int i = CAP * 32 + lane; i < d_vec; i += 32) yrow[i] = scale_vec<BF16>(orow[i], s);
    for (int i = CAP * 32 + lane; i < dl_vec; i += 32) yrow[d_vec + i] = bad ? zero : __ldg(erow + i);
    if (lane == 0) {
      if (scale_out != nullptr) scale_out[t] = s;
      if (bad) set_flag(status, MLS_DEVFLAG_BAD_ID);
    }
  }
}

// ---------------------------------------------------------------- backward
// do = s (g_o - u (u.g_o)),  de = g_e + (u.g_o) e_hat, written as
//   do = s g_o - (s ug / ||o||) o,   de = g_e + (ug / ||e||) e,   ug = o.g_o / ||o||.
// When coef_out is given, c_t = ug/||e|| is stored for the table scatter.
template <bool BF16, int CAP>
__global__ void __launch_bounds__(256) junction_bwd_kernel(
    const int32_t* __restrict__ x, int64_t T, const uint4* __restrict__ o, int d_vec,
    const uint4* __restrict__ E, int64_t V, int dl_vec, const uint4* __restrict__ dy,
    uint4* __restrict__ do_out, uint4* __restrict__ de_out, float* __restrict__ coef_out,
    int32_t* __restrict__ status) {
  const int lane = threadIdx.x & 31;
  const int64_t warp0 = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
  const int dp_vec = d_vec + dl_vec;
  for (int64_t t = warp0; t < T; t += nwarps) {
    const int32_t id = __ldg(x + t);
    const bool bad = (id < 0) || (static_cast<int64_t>(id) >= V);
    const uint4* orow = o + t * d_vec;
    const uint4* grow = dy + t * dp_vec;
    const uint4* erow = E + static_cast<int64_t>(bad ? 0 : id) * dl_vec;
    uint4 oc[CAP], gc[CAP], ec[CAP];
    float so = 0.f, sog = 0.f, se = 0.f;
#pragma unroll
    for (int j = 0; j < CAP; ++j) {
      const int i = j * 32 + lane;
      if (i < d_vec) {
        oc[j] = __ldcs(orow + i);
        gc[j] = __ldcs(grow + i);
        so += sumsq<BF16>(oc[j]);
        sog += dotv<BF16>(oc[j], gc[j]);
      }
      if (i < dl_vec) { ec[j] = __ldg(erow + i); se += sumsq<BF16>(ec[j]); }
    }
    for (int i = CAP * 32 + lane; i < d_vec; i += 32) {
      const uint4 ov = orow[i], gv = grow[i];
      so += sumsq<BF16>(ov);
      sog += dotv<BF16>(ov, gv);
    }
    for (int i = CAP * 32 + lane; i < dl_vec; i += 32) se += sumsq<BF16>(__ldg(erow + i));
    so = warp_sum(so);
    sog = warp_sum(sog);
    se = warp_sum(se);
    const float n_o = fmaxf(sqrtf(so), kJunctionEps);
    const float n_e = sqrtf(se);
    const float s = n_e / n_o;
    const float ug = sog / n_o;
    float a = s, b = s * ug / n_o, c = (n_e > 0.f) ? ug / n_e : 0.f;
    if (bad) { a = 0.f; b = 0.f; c = 0.f; }
    uint4* drow = do_out + t * d_vec;
    const uint4 zero = make_uint4(0, 0, 0, 0);
#pragma unroll
    for (int j = 0; j < CAP; ++j) {
      const int i = j * 32 + lane;
      if (i < d_vec) drow[i] = axpby_vec<BF16>(a, gc[j], b, oc[j]);
    }
    for (int i = CAP * 32 + lane; i < d_vec; i += 32) drow[i] = axpby_vec<BF16>(a, grow[i], b, orow[i]);
    if (de_out != nullptr) {
      uint4* erow_out = de_out + t * dl_vec;
#pragma unroll
      for (int j = 0; j < CAP; ++j) {
        const int i = j * 32 + lane;
        if (i < dl_vec) erow_out[i] = bad ? zero : add_scaled_vec<BF16>(__ldcs(grow + d_vec + i), c, ec[j]);
      }
      for (int i = CAP * 32 + lane; i < dl_vec; i += 32)
        erow_out[i] = bad ? zero : add_scaled_vec<BF16>(grow[d_vec + i], c, __ldg(erow + i));
    }
    if (lane == 0) {
      if (coef_out != nullptr) coef_out[t] = c;
      if (bad) set_flag(status, MLS_DEVFLAG_BAD_ID);
    }
  }
}

// ---------------------------------------------------------------- table scatter
// dE[v] (+)= sum_{t: x_t = v} de_t with de_t = g_e,t + c_t E[v]; so the row sum is
//   dE[v] (+)= (sum_t g_e,t) + (sum_t c_t) E[v],
// both sums taken over the tokens of v in ascending t.  Tokens are grouped by
// id with a stable LSD radix sort (8-bit digits), so the order is fixed and
// the result is deterministic.

constexpr int kSortBlock = 1024;  // keys per sort block (one per thread)

__global__ void __launch_bounds__(kSortBlock) sort_hist_kernel(const int32_t* __restrict__ keys,
                                                               const int32_t* __restrict__ x, int64_t n,
                                                               int64_t V, int shift,
                                                               int32_t* __restrict__ hist, int nblk) {
  __shared__ int32_t h[256];
  for (int i = threadIdx.x; i < 256; i += blockDim.x) h[i] = 0;
  __syncthreads();
  const int64_t i = static_cast<int64_t>(blockIdx.x) * kSortBlock + threadIdx.x;
  if (i < n) {
    int32_t k;
    if (keys != nullptr) {
      k = keys[i];
    } else {  // first pass reads ids directly; invalid ids sort last as key V
      const int32_t id = x[i];
      k = (id < 0 || id >= V) ? static_cast<int32_t>(V) : id;
    }
    atomicAdd(&h[(k >> shift) & 255], 1);
  }
  __syncthreads();
  for (int d = threadIdx.x; d < 256; d += blockDim.x) hist[d * nblk + blockIdx.x] = h[d];
}

// Exclusive prefix sum over hist[0..n) in one block (digit-major, block-minor order).
__global__ void __launch_bounds__(1024) sort_scan_kernel(int32_t* __restrict__ hist, int n) {
  __shared__ int32_t part[1024];
  const int tid = threadIdx.x;
  const int per = (n + 1023) / 1024;
  const int lo = min(n, tid * per), hi = min(n, lo + per);
  int32_t s = 0;
  for (int i = lo; i < hi; ++i) s += hist[i];
  part[tid] = s;
  __syncthreads();
  for (int off = 1; off < 1024; off <<= 1) {   // inclusive Hillis-Steele scan
    const int32_t v = (tid >= off) ? part[tid - off] : 0;
    __syncthreads();
    part[tid] += v;
    __syncthreads();
  }
  int32_t run = part[tid] - s;
  for (int i = lo; i < hi; ++i) {
    const int32_t c = hist[i];
    hist[i] = run;
    run += c;
  }
}

__global__ void __launch_bounds__(kSortBlock) sort_scatter_kernel(
    const int32_t* __restrict__ kin, const int32_t* __restrict__ vin, const int32_t* __restrict__ x,
    int64_t n, int64_t V, int shift, const int32_t* __restrict__ hist, int nblk, int32_t* __restrict__ kout,
    int32_t* __restrict__ vout) {
  __shared__ int32_t wcnt[kSortBlock / 32][256];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  for (int i = tid; i < (kSortBlock / 32) * 256; i += blockDim.x) (&wcnt[0][0])[i] = 0;
  __syncthreads();
  const int64_t i = static_cast<int64_t>(blockIdx.x) * kSortBlock + tid;
  const bool valid = i < n;
  int32_t k = 0, v = 0;
  if (valid) {
    if (kin != nullptr) {
      k = kin[i];
      v = vin[i];
    } else {
      const int32_t id = x[i];
      k = (id < 0 || id >= V) ? static_cast<int32_t>(V) : id;
      v = static_cast<int32_t>(i);
    }
  }
  const int d = (k >> shift) & 255;
  const unsigned peers = __match_any_sync(0xffffffffu, valid ? d : 256 + lane);
  const int rank = __popc(peers & ((1u << lane) - 1u));
  if (valid && rank == 0) wcnt[warp][d] = __popc(peers);
  __syncthreads();
  if (tid < 256) {
    int32_t run = 0;
    for (int w = 0; w < kSortBlock / 32; ++w) {
      const int32_t c = wcnt[w][tid];
      wcnt[w][tid] = run;
      run += c;
    }
  }
  __syncthreads();
  if (valid) {
    const int32_t pos = hist[d * nblk + blockIdx.x] + wcnt[warp][d] + rank;
    kout[pos] = k;
    vout[pos] = v;
  }
}

// One warp per (sorted position, column slice of 32 vectors).  Only the first
// position of each id segment does work; it walks the segment in order.
template <bool BF16>
__global__ void __launch_bounds__(256) table_scatter_kernel(
    const int32_t* __restrict__ keys, const int32_t* __restrict__ toks, int64_t n, int64_t V,
    const uint4* __restrict__ dy, int d_vec, int dl_vec, const float* __restrict__ coef,
    const uint4* __restrict__ E, float* __restrict__ dE, int n_slices) {
  constexpr int N = Elt<BF16>::kPerVec;
  const int lane = threadIdx.x & 31;
  const int64_t w = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int64_t pos = w / n_slices;
  const int slice = static_cast<int>(w % n_slices);
  if (pos >= n) return;
  const int32_t key = keys[pos];
  if (key >= V) return;                                   // invalid ids sort last
  if (pos > 0 && keys[pos - 1] == key) return;           // not a segment start
  const int vi = slice * 32 + lane;
  const bool active = vi < dl_vec;
  const int dp_vec = d_vec + dl_vec;
  float acc[N];
#pragma unroll
  for (int k = 0; k < N; ++k) acc[k] = 0.f;
  float csum = 0.f;
  for (int64_t p = pos; p < n && keys[p] == key; ++p) {
    const int64_t t = toks[p];
    csum += coef[t];
    if (active) {
      float g[N];
      Elt<BF16>::load(__ldg(dy + t * dp_vec + d_vec + vi), g);
#pragma unroll
      for (int k = 0; k < N; ++k) acc[k] += g[k];
    }
  }
  if (!active) return;
  float e[N];
  Elt<BF16>::load(__ldg(E + static_cast<int64_t>(key) * dl_vec + vi), e);
  float* out = dE + static_cast<int64_t>(key) * dl_vec * N + static_cast<int64_t>(vi) * N;
#pragma unroll
  for (int k = 0; k < N; ++k) out[k] += fmaf(csum, e[k], acc[k]);
}

int pick_cap(int nvec) {
  const int per_lane = (nvec + 31) / 32;
  if (per_lane <= 1) return 1;
  if (per_lane <= 2) return 2;
  if (per_lane <= 4) return 4;
  if (per_lane <= 8) return 8;
  if (per_lane <= 12) return 12;
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
  const int cap = pick_cap(d_vec > dl_vec ? d_vec : dl_vec);
  const int grid = grid_for(a.T, 8);
  auto* o = static_cast<const uint4*>(a.o);
  auto* E = static_cast<const uint4*>(a.E);
  auto* y = static_cast<uint4*>(a.y);
#define MLS_JF(C) junction_fwd_kernel<BF16, C><<<grid, 256, 0, st>>>(a.x, a.T, o, d_vec, E, a.V, dl_vec, y, a.scale_out, a.status)
  switch (cap) {
    case 1: MLS_JF(1); break;
    case 2: MLS_JF(2); break;
    case 4: MLS_JF(4); break;
    case 8: MLS_JF(8); break;
    case 12: MLS_JF(12); break;
    default: MLS_JF(16); break;
  }
#undef MLS_JF
  note_launches(1);
  return cudaGetLastError();
}

template <bool BF16>
cudaError_t launch_bwd_t(const JunctionArgs& a, cudaStream_t st) {
  constexpr int N = Elt<BF16>::kPerVec;
  const int d_vec = static_cast<int>(a.D / N), dl_vec = static_cast<int>(a.delta / N);
  const int cap = pick_cap(d_vec > dl_vec ? d_vec : dl_vec);
  const int grid = grid_for(a.T, 8);
  auto* o = static_cast<const uint4*>(a.o);
  auto* E = static_cast<const uint4*>(a.E);
  auto* dy = static_cast<const uint4*>(a.dy);
  auto* dout = static_cast<uint4*>(a.do_out);
  auto* deo = static_cast<uint4*>(a.de_out);
  float* coef = nullptr;
  JunctionScatterWs ws{};
  if (a.dE != nullptr) {
    ws = junction_scatter_layout(a.T, a.workspace);
    coef = ws.coef;
  }
#define MLS_JB(C) junction_bwd_kernel<BF16, C><<<grid, 256, 0, st>>>(a.x, a.T, o, d_vec, E, a.V, dl_vec, dy, dout, deo, coef, a.status)
  switch (cap) {
    case 1: MLS_JB(1); break;
    case 2: MLS_JB(2); break;
    case 4: MLS_JB(4); break;
    case 8: MLS_JB(8); break;
    case 12: MLS_JB(12); break;
    default: MLS_JB(16); break;
  }
#undef MLS_JB
  note_launches(1);
  cudaError_t err = cudaGetLastError();
  if (err != cudaSuccess || a.dE == nullptr) return err;

  // Stable radix sort of the ids, then the per-id segment sums.
  const int64_t n = a.T;
  const int nblk = static_cast<int>((n + kSortBlock - 1) / kSortBlock);
  int bits = 1;
  while ((int64_t(1) << bits) <= a.V) ++bits;          // keys live in [0, V]
  const int passes = (bits + 7) / 8;
  const int32_t* kin = nullptr;
  const int32_t* vin = nullptr;
  int32_t* kbuf[2] = {ws.keys0, ws.keys1};
  int32_t* vbuf[2] = {ws.vals0, ws.vals1};
  for (int p = 0; p < passes; ++p) {
    sort_hist_kernel<<<nblk, kSortBlock, 0, st>>>(kin, a.x, n, a.V, 8 * p, ws.hist, nblk);
    sort_scan_kernel<<<1, 1024, 0, st>>>(ws.hist, 256 * nblk);
    sort_scatter_kernel<<<nblk, kSortBlock, 0, st>>>(kin, vin, a.x, n, a.V, 8 * p, ws.hist, nblk,
                                                     kbuf[p & 1], vbuf[p & 1]);
    kin = kbuf[p & 1];
    vin = vbuf[p & 1];
    note_launches(3);
  }
  if (!a.accumulate_dE) {
    err = cudaMemsetAsync(a.dE, 0, static_cast<size_t>(a.V) * a.delta * sizeof(float), st);
    if (err != cudaSuccess) return err;
  }
  const int n_slices = (dl_vec + 31) / 32;
  const int64_t warps = n * n_slices;
  const int64_t blocks = (warps + 7) / 8;
  table_scatter_kernel<BF16><<<static_cast<unsigned>(blocks), 256, 0, st>>>(
      kin, vin, n, a.V, dy, d_vec, dl_vec, coef, E, a.dE, n_slices);
  note_launches(1);
  return cudaGetLastError();
}

}  // namespace

size_t junction_scatter_bytes(int64_t T) {
  const int64_t nblk = (T + kSortBlock - 1) / kSortBlock;
  const size_t t4 = static_cast<size_t>(T) * 4;
  auto up = [](size_t b) { return (b + 255) & ~size_t(255); };
  return up(t4) * 5 + up(static_cast<size_t>(256) * nblk * 4);
}

JunctionScatterWs junction_scatter_layout(int64_t T, void* base) {
  const int64_t nblk = (T + kSortBlock - 1) / kSortBlock;
  const size_t t4 = static_cast<size_t>(T) * 4;
  auto up = [](size_t b) { return (b + 255) & ~size_t(255); };
  char* p = static_cast<char*>(base);
  JunctionScatterWs w;
  w.coef = reinterpret_cast<float*>(p); p += up(t4);
  w.keys0 = reinterpret_cast<int32_t*>(p); p += up(t4);
  w.keys1 = reinterpret_cast<int32_t*>(p); p += up(t4);
  w.vals0 = reinterpret_cast<int32_t*>(p); p += up(t4);
  w.vals1 = reinterpret_cast<int32_t*>(p); p += up(t4);
  w.hist = reinterpret_cast<int32_t*>(p);
  (void)nblk;
  return w;
}

cudaError_t launch_junction_fwd(const JunctionArgs& a, cudaStream_t st) {
  return a.bf16 ? launch_fwd_t<true>(a, st) : launch_fwd_t<false>(a, st);
}

cudaError_t launch_junction_bwd(const JunctionArgs& a, cudaStream_t st) {
  return a.bf16 ? launch_bwd_t<true>(a, st) : launch_bwd_t<false>(a, st);
}

}  // namespace mls
