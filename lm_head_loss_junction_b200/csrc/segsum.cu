// Deterministic row scatters grouped by token id: the residual-table gradient
// of the junction (dE[v] (+)= sum over tokens with x_t = v) and the one-hot
// part of the head gradient (dW^m[v] -= c sum over tokens with y_t = v of h_t).
//
// Tokens are grouped by id with a stable LSD radix sort (8-bit digits), so
// each id's tokens are visited in ascending t and every sum is taken in a
// fixed order: results are bitwise reproducible, with no floating-point
// atomics.  Rows with few tokens are reduced by one warp; rows with many
// (Zipf-frequent ids) by a whole block whose warps split the tokens and are
// combined in warp order.  The ids present are listed (light and heavy) so
// that no warp is spent on absent ids; each row slice is still summed by one
// warp in token order, so the list order does not change any result.
#include <algorithm>
#include <mutex>

#include "common.cuh"
#include "kernels.h"

namespace mls {

// ------------------------------------------------------------------ side stream
namespace {
struct SideSlot {
  cudaStream_t s = nullptr;
  cudaEvent_t fork = nullptr, join = nullptr;
  bool tried = false;
};
constexpr int kMaxSideDevices = 64;
SideSlot g_side[kMaxSideDevices];
std::mutex g_side_mu;
}  // namespace

// Compile with -DMLS_SIDE_STREAM=0 to run the side work on the caller's stream.
#ifndef MLS_SIDE_STREAM
#define MLS_SIDE_STREAM 1
#endif

SideScope::SideScope(cudaStream_t st) : main_(st), side_(st), slot_(nullptr), joined_(true) {
  if (!MLS_SIDE_STREAM) return;
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxSideDevices) {
    (void)cudaGetLastError();
    return;
  }
  g_side_mu.lock();
  SideSlot& sl = g_side[dev];
  if (!sl.tried) {
    sl.tried = true;
    if (cudaStreamCreateWithFlags(&sl.s, cudaStreamNonBlocking) != cudaSuccess ||
        cudaEventCreateWithFlags(&sl.fork, cudaEventDisableTiming) != cudaSuccess ||
        cudaEventCreateWithFlags(&sl.join, cudaEventDisableTiming) != cudaSuccess) {
      (void)cudaGetLastError();
      sl.s = nullptr;
    }
  }
  if (sl.s == nullptr) {
    g_side_mu.unlock();
    return;
  }
  side_ = sl.s;
  slot_ = &sl;
  if (fork() != cudaSuccess) {
    (void)cudaGetLastError();
    side_ = st;
    slot_ = nullptr;
    g_side_mu.unlock();
  }
}

cudaError_t SideScope::fork() {
  if (slot_ == nullptr) return cudaSuccess;
  // (forking again while forked makes the side stream also wait for the
  // caller's work enqueued since the last fork)
  SideSlot& sl = *static_cast<SideSlot*>(slot_);
  cudaError_t err = cudaEventRecord(sl.fork, main_);
  if (err == cudaSuccess) err = cudaStreamWaitEvent(side_, sl.fork, 0);
  if (err == cudaSuccess) joined_ = false;
  return err;
}

cudaError_t SideScope::join() {
  if (slot_ == nullptr || joined_) return cudaSuccess;
  joined_ = true;
  SideSlot& sl = *static_cast<SideSlot*>(slot_);
  cudaError_t err = cudaEventRecord(sl.join, side_);
  if (err == cudaSuccess) err = cudaStreamWaitEvent(main_, sl.join, 0);
  return err;
}

SideScope::~SideScope() {
  (void)join();
  if (slot_ != nullptr) g_side_mu.unlock();
}

namespace {

constexpr int kSortBlock = 1024;     // keys per sort block (one per thread)
constexpr int kHeavy = 32;           // rows with more tokens than this use a block
constexpr int kHeavyWarps = 16;

size_t up256(size_t b) { return (b + 255) & ~size_t(255); }

__device__ __forceinline__ int32_t clamp_key(int32_t id, int64_t V) {
  return (id < 0 || id >= V) ? static_cast<int32_t>(V) : id;   // invalid ids sort last
}

__global__ void __launch_bounds__(kSortBlock) sort_hist_kernel(const int32_t* __restrict__ keys,
                                                               const int32_t* __restrict__ ids, int64_t n,
                                                               int64_t V, int shift, int32_t* __restrict__ hist,
                                                               int nblk) {
  __shared__ int32_t h[256];
  for (int i = threadIdx.x; i < 256; i += blockDim.x) h[i] = 0;
  __syncthreads();
  const int64_t i = static_cast<int64_t>(blockIdx.x) * kSortBlock + threadIdx.x;
  if (i < n) {
    const int32_t k = keys != nullptr ? keys[i] : clamp_key(ids[i], V);
    atomicAdd(&h[(k >> shift) & 255], 1);
  }
  __syncthreads();
  for (int d = threadIdx.x; d < 256; d += blockDim.x) hist[d * nblk + blockIdx.x] = h[d];
}

// Exclusive prefix sum of n ints in place, one block of 1024 threads: chunks
// of 4096 (4 consecutive values per thread, coalesced), warp-shuffle scans,
// and a running carry between chunks.
__global__ void __launch_bounds__(1024) exclusive_scan_kernel(int32_t* data, int n) {
  __shared__ int32_t warp_tot[32];
  __shared__ int32_t carry_s;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  if (tid == 0) carry_s = 0;
  __syncthreads();
  for (int base = 0; base < n; base += 4096) {
    int32_t v[4];
    const int i0 = base + 4 * tid;
#pragma unroll
    for (int k = 0; k < 4; ++k) v[k] = (i0 + k < n) ? data[i0 + k] : 0;
    const int32_t own = v[0] + v[1] + v[2] + v[3];
    int32_t incl = own;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int32_t u = __shfl_up_sync(0xffffffffu, incl, off);
      if (lane >= off) incl += u;
    }
    if (lane == 31) warp_tot[warp] = incl;
    __syncthreads();
    if (warp == 0) {
      int32_t w = warp_tot[lane];
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const int32_t u = __shfl_up_sync(0xffffffffu, w, off);
        if (lane >= off) w += u;
      }
      warp_tot[lane] = w;   // inclusive over warps
    }
    __syncthreads();
    const int32_t carry = carry_s;
    int32_t run = carry + (warp > 0 ? warp_tot[warp - 1] : 0) + incl - own;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      if (i0 + k < n) data[i0 + k] = run;
      run += v[k];
    }
    __syncthreads();
    if (tid == 1023) carry_s = carry + warp_tot[31];
    __syncthreads();
  }
}

__global__ void __launch_bounds__(kSortBlock) sort_scatter_kernel(
    const int32_t* __restrict__ kin, const int32_t* __restrict__ vin, const int32_t* __restrict__ ids, int64_t n,
    int64_t V, int shift, const int32_t* __restrict__ hist, int nblk, int32_t* __restrict__ kout,
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
      k = clamp_key(ids[i], V);
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

// Segment bounds from the sorted keys: offsets[v] = first position of id v,
// ends[v] = one past its last (both 0 for absent ids, preset by a memset).
// Ids with more than kHeavy tokens are appended to the heavy list, the others
// present to the light list; list order does not matter, every row is reduced
// independently in a fixed order.  counts[0] = heavy ids, counts[1] = light ids.
__global__ void segment_bounds_kernel(const int32_t* __restrict__ keys, int64_t n, int64_t V,
                                      int32_t* __restrict__ offsets, int32_t* __restrict__ ends,
                                      int32_t* __restrict__ heavy, int32_t* __restrict__ light,
                                      int32_t* __restrict__ counts) {
  const int64_t p = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (p >= n) return;
  const int32_t k = keys[p];
  if (k >= V) return;                                    // invalid ids sort last
  if (p == 0 || keys[p - 1] != k) {
    offsets[k] = static_cast<int32_t>(p);
    if (p + kHeavy < n && keys[p + kHeavy] == k) heavy[atomicAdd(counts, 1)] = k;
    else light[atomicAdd(counts + 1, 1)] = k;
  }
  if (p == n - 1 || keys[p + 1] != k) ends[k] = static_cast<int32_t>(p + 1);
}

template <bool BF16>
struct Vec8;
template <>
struct Vec8<true> {
  static constexpr int N = 8;
  __device__ static void add(float (&acc)[8], const uint4& u) {
    float f[8];
    bf16x8_to_f32(u, f);
#pragma unroll
    for (int k = 0; k < 8; ++k) acc[k] += f[k];
  }
  __device__ static void load(const uint4& u, float (&f)[8]) { bf16x8_to_f32(u, f); }
};
template <>
struct Vec8<false> {
  static constexpr int N = 4;
  __device__ static void add(float (&acc)[4], const uint4& u) {
    acc[0] += __uint_as_float(u.x); acc[1] += __uint_as_float(u.y);
    acc[2] += __uint_as_float(u.z); acc[3] += __uint_as_float(u.w);
  }
  __device__ static void load(const uint4& u, float (&f)[4]) {
    f[0] = __uint_as_float(u.x); f[1] = __uint_as_float(u.y);
    f[2] = __uint_as_float(u.z); f[3] = __uint_as_float(u.w);
  }
};

// Writes one row slice: out = base + scale*acc + cs*E (table mode) or out -= scale*acc (target mode).
template <bool BF16, bool TABLE>
__device__ __forceinline__ void emit(float* out_row, int vi, const float (&acc)[Vec8<BF16>::N], float cs,
                                     const uint4* E_row, float scale, bool accumulate) {
  constexpr int N = Vec8<BF16>::N;
  float4* o = reinterpret_cast<float4*>(out_row + static_cast<int64_t>(vi) * N);
  float val[N];
  if (TABLE) {
    float e[N];
    Vec8<BF16>::load(__ldg(E_row + vi), e);
#pragma unroll
    for (int k = 0; k < N; ++k) val[k] = fmaf(cs, e[k], scale * acc[k]);
  }
#pragma unroll
  for (int q = 0; q < N / 4; ++q) {
    float4 r;
    if (TABLE) {
      r = make_float4(val[4 * q], val[4 * q + 1], val[4 * q + 2], val[4 * q + 3]);
      if (accumulate) {
        const float4 b = o[q];
        r.x += b.x; r.y += b.y; r.z += b.z; r.w += b.w;
      }
    } else {
      r = o[q];
      r.x = fmaf(-scale, acc[4 * q], r.x);
      r.y = fmaf(-scale, acc[4 * q + 1], r.y);
      r.z = fmaf(-scale, acc[4 * q + 2], r.z);
      r.w = fmaf(-scale, acc[4 * q + 3], r.w);
    }
    o[q] = r;
  }
}

// One row-sum job: the rows of token t are src + t*src_ld + src_off (16-byte
// vectors, n_vec per row); the sums go to out (fp32 rows of n_vec vectors).
// Several jobs that share the id grouping (the exits of the loss, which share
// the targets) run in one launch, one per blockIdx.z.
struct SegJob {
  const uint4* src;
  int64_t src_ld;
  int src_off;
  int n_vec;
  const uint4* E;
  float* out;
  float scale;
  const float* coef;     // table mode: per-token coefficient of E[v]
};
struct SegJobs {
  SegJob j[kMaxExits];
};

// Light rows: warp w of block (x, y, z) takes light ids x*8 + w, x*8 + w + 8*gridDim.x, ...
// and their slice y of 32 vectors (one 16-byte vector per lane) of job z.
template <bool BF16, bool TABLE>
__global__ void __launch_bounds__(256) segsum_light_kernel(const SegIndexDev ix, const SegJobs jobs, int accumulate) {
  constexpr int N = Vec8<BF16>::N;
  const SegJob& jb = jobs.j[blockIdx.z];
  const float* __restrict__ coef = jb.coef;
  const uint4* __restrict__ src = jb.src;
  const int64_t src_ld = jb.src_ld;
  const int src_off = jb.src_off;
  const int n_vec = jb.n_vec;
  if (static_cast<int>(blockIdx.y) * 32 >= n_vec) return;   // this job's rows are narrower
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const int vi = static_cast<int>(blockIdx.y) * 32 + lane;
  const bool active = vi < n_vec;
  const int n_light = *ix.n_light;
  for (int i = static_cast<int>(blockIdx.x) * 8 + warp; i < n_light; i += static_cast<int>(gridDim.x) * 8) {
    const int64_t v = ix.light[i];
    const int32_t off = ix.offsets[v];
    const int32_t cnt = ix.ends[v] - off;
    float cs = 0.f;
    if (TABLE)
      for (int p = 0; p < cnt; ++p) cs += coef[ix.toks[off + p]];
    if (!active) continue;
    float acc[N];
#pragma unroll
    for (int k = 0; k < N; ++k) acc[k] = 0.f;
    // four rows in flight per lane, added in token order
    int p = 0;
    for (; p + 4 <= cnt; p += 4) {
      uint4 u[4];
#pragma unroll
      for (int b = 0; b < 4; ++b) u[b] = __ldg(src + static_cast<int64_t>(ix.toks[off + p + b]) * src_ld + src_off + vi);
#pragma unroll
      for (int b = 0; b < 4; ++b) Vec8<BF16>::add(acc, u[b]);
    }
    for (; p < cnt; ++p) Vec8<BF16>::add(acc, __ldg(src + static_cast<int64_t>(ix.toks[off + p]) * src_ld + src_off + vi));
    float* out_row = jb.out + v * static_cast<int64_t>(n_vec) * N;
    const uint4* E_row = TABLE ? jb.E + v * static_cast<int64_t>(n_vec) : nullptr;
    emit<BF16, TABLE>(out_row, vi, acc, cs, E_row, jb.scale, accumulate != 0);
  }
}

// Overwrite mode of the table gradients, in one pass over every row of every
// table: one warp per (row v, table) task, consecutive tasks covering row v
// of every table; rows of absent ids get zeros (every store 512 contiguous
// bytes), rows of light ids (at most kHeavy tokens) the sum of their tokens'
// rows in token order, 32 vectors (one per lane) at a time (the same order and
// arithmetic as segsum_light_kernel), rows of heavy ids are left to
// segsum_heavy_kernel.  The zero writes of the many absent rows hide the
// latency of the light rows' gathers.
template <bool BF16>
__global__ void __launch_bounds__(256) table_rows_kernel(const __grid_constant__ SegIndexDev ix,
                                                         const __grid_constant__ SegJobs jobs, int njobs,
                                                         int v_begin, int v_end) {
  constexpr int N = Vec8<BF16>::N;
  const int lane = threadIdx.x & 31;
  const unsigned warp0 = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const unsigned nwarps = (gridDim.x * blockDim.x) >> 5;
  const unsigned ntasks = static_cast<unsigned>(v_end - v_begin) * static_cast<unsigned>(njobs);
  for (unsigned task = warp0; task < ntasks; task += nwarps) {
    const unsigned rv = task / static_cast<unsigned>(njobs);
    const int v = v_begin + static_cast<int>(rv);
    const SegJob& jb = jobs.j[task - rv * static_cast<unsigned>(njobs)];
    const int n_vec = jb.n_vec;
    const int32_t end = ix.ends[v];
    float* out_row = jb.out + static_cast<int64_t>(v) * n_vec * N;
    if (end == 0) {                                      // absent id: zeros
      float4* o = reinterpret_cast<float4*>(out_row);
      const int n4 = n_vec * (N / 4);
      for (int k = lane; k < n4; k += 32) o[k] = make_float4(0.f, 0.f, 0.f, 0.f);
      continue;
    }
    const int32_t off = ix.offsets[v];
    const int32_t cnt = end - off;
    if (cnt > kHeavy) continue;                          // heavy id: its own kernel
    float cs = 0.f;
    for (int p = 0; p < cnt; ++p) cs += jb.coef[ix.toks[off + p]];
    const uint4* __restrict__ src = jb.src;
    const uint4* E_row = jb.E + static_cast<int64_t>(v) * n_vec;
    for (int vi = lane; vi < n_vec; vi += 32) {
      float acc[N];
#pragma unroll
      for (int k = 0; k < N; ++k) acc[k] = 0.f;
      int p = 0;
      for (; p + 4 <= cnt; p += 4) {
        uint4 u[4];
#pragma unroll
        for (int b = 0; b < 4; ++b)
          u[b] = __ldg(src + static_cast<int64_t>(ix.toks[off + p + b]) * jb.src_ld + jb.src_off + vi);
#pragma unroll
        for (int b = 0; b < 4; ++b) Vec8<BF16>::add(acc, u[b]);
      }
      for (; p < cnt; ++p)
        Vec8<BF16>::add(acc, __ldg(src + static_cast<int64_t>(ix.toks[off + p]) * jb.src_ld + jb.src_off + vi));
      emit<BF16, true>(out_row, vi, acc, cs, E_row, jb.scale, false);
    }
  }
}

// One block per (heavy row, slice of 32 vectors, job); warps split the row's
// tokens round-robin and are combined in warp order.
template <bool BF16, bool TABLE>
__global__ void __launch_bounds__(kHeavyWarps * 32) segsum_heavy_kernel(const SegIndexDev ix, const SegJobs jobs,
                                                                        int accumulate) {
  constexpr int N = Vec8<BF16>::N;
  __shared__ float part[kHeavyWarps][32 * N];
  __shared__ float cpart[kHeavyWarps];
  const SegJob& jb = jobs.j[blockIdx.z];
  const float* __restrict__ coef = jb.coef;
  const uint4* __restrict__ src = jb.src;
  const int64_t src_ld = jb.src_ld;
  const int src_off = jb.src_off;
  const int n_vec = jb.n_vec;
  if (static_cast<int>(blockIdx.x) >= *ix.n_heavy || static_cast<int>(blockIdx.y) * 32 >= n_vec) return;
  const int64_t v = ix.heavy[blockIdx.x];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int vi = blockIdx.y * 32 + lane;
  const bool active = vi < n_vec;
  const int32_t off = ix.offsets[v];
  const int32_t cnt = ix.ends[v] - off;
  float acc[N];
#pragma unroll
  for (int k = 0; k < N; ++k) acc[k] = 0.f;
  float cs = 0.f;
  // this warp's tokens p = warp, warp + 16, ...; four rows in flight, added in order
  int p = warp;
  for (; p + 3 * kHeavyWarps < cnt; p += 4 * kHeavyWarps) {
    int64_t t[4];
    uint4 u[4];
#pragma unroll
    for (int b = 0; b < 4; ++b) t[b] = ix.toks[off + p + b * kHeavyWarps];
#pragma unroll
    for (int b = 0; b < 4; ++b) u[b] = active ? __ldg(src + t[b] * src_ld + src_off + vi) : make_uint4(0, 0, 0, 0);
#pragma unroll
    for (int b = 0; b < 4; ++b) {
      if (TABLE) cs += coef[t[b]];
      if (active) Vec8<BF16>::add(acc, u[b]);
    }
  }
  for (; p < cnt; p += kHeavyWarps) {
    const int64_t t = ix.toks[off + p];
    if (TABLE) cs += coef[t];
    if (active) Vec8<BF16>::add(acc, __ldg(src + t * src_ld + src_off + vi));
  }
#pragma unroll
  for (int k = 0; k < N; ++k) part[warp][lane * N + k] = acc[k];
  if (lane == 0) cpart[warp] = cs;
  __syncthreads();
  if (warp == 0) {
    float tot[N];
#pragma unroll
    for (int k = 0; k < N; ++k) tot[k] = 0.f;
    float ctot = 0.f;
    for (int w = 0; w < kHeavyWarps; ++w) {
#pragma unroll
      for (int k = 0; k < N; ++k) tot[k] += part[w][lane * N + k];
      ctot += cpart[w];
    }
    if (active) {
      float* out_row = jb.out + v * static_cast<int64_t>(n_vec) * N;
      const uint4* E_row = TABLE ? jb.E + v * static_cast<int64_t>(n_vec) : nullptr;
      emit<BF16, TABLE>(out_row, vi, tot, ctot, E_row, jb.scale, accumulate != 0);
    }
  }
}

// Row sums of every job; the heavy rows go to heavy_st (rows disjoint from the
// others, so they may run beside them on another stream).
template <bool BF16, bool TABLE>
cudaError_t launch_segsum(const SegIndexDev& ix, const SegJobs& jobs, int njobs, int accumulate, cudaStream_t st,
                          cudaStream_t heavy_st) {
  int slices = 0, total_slices = 0;
  for (int z = 0; z < njobs; ++z) {
    const int sz = (jobs.j[z].n_vec + 31) / 32;
    slices = std::max(slices, sz);
    total_slices += sz;
  }
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (TABLE && !accumulate) {
    // every row of every table in one pass: zeros for absent ids, sums for light ones;
    // one warp per (row, table) task (row ranges of at most 2^31 tasks per launch)
    const int64_t rows_per_launch = std::max<int64_t>(1, ((int64_t(1) << 31) - 1) / njobs);
    for (int64_t v0 = 0; v0 < ix.V; v0 += rows_per_launch) {
      const int64_t v1 = std::min<int64_t>(ix.V, v0 + rows_per_launch);
      const int64_t tasks = (v1 - v0) * njobs;
      const int64_t blocks = std::max<int64_t>(1, (tasks + 7) / 8);
      table_rows_kernel<BF16><<<static_cast<unsigned>(blocks), 256, 0, st>>>(ix, jobs, njobs, static_cast<int>(v0),
                                                                             static_cast<int>(v1));
      note_launches(1);
    }
  } else {
    // light rows: about one full wave of 8-warp blocks over (light ids) x (32-vector slices of every job)
    const int64_t want = (static_cast<int64_t>(sms) * 8 + total_slices - 1) / total_slices;
    const int64_t gx = std::max<int64_t>(1, std::min<int64_t>(want, (ix.max_light + 7) / 8));
    segsum_light_kernel<BF16, TABLE>
        <<<dim3(static_cast<unsigned>(gx), static_cast<unsigned>(slices), static_cast<unsigned>(njobs)), 256, 0, st>>>(
            ix, jobs, accumulate);
    note_launches(1);
  }
  dim3 grid(static_cast<unsigned>(ix.max_heavy), static_cast<unsigned>(slices), static_cast<unsigned>(njobs));
  segsum_heavy_kernel<BF16, TABLE><<<grid, kHeavyWarps * 32, 0, heavy_st>>>(ix, jobs, accumulate);
  note_launches(1);
  return cudaGetLastError();
}

}  // namespace

size_t segindex_bytes(int64_t T, int64_t V) {
  const int64_t nblk = (T + kSortBlock - 1) / kSortBlock;
  const size_t t4 = static_cast<size_t>(T) * 4;
  const int64_t max_heavy = T / (kHeavy + 1) + 1;
  const int64_t max_light = T < V ? T : V;
  return up256(t4) * 4 + up256(static_cast<size_t>(256) * nblk * 4) + up256(static_cast<size_t>(V) * 4) * 2 +
         up256(static_cast<size_t>(max_heavy) * 4) + up256(static_cast<size_t>(max_light) * 4) + 256;
}

cudaError_t build_segindex(const int32_t* ids, int64_t T, int64_t V, void* ws, SegIndexDev* out, cudaStream_t st) {
  const int64_t nblk = (T + kSortBlock - 1) / kSortBlock;
  const size_t t4 = static_cast<size_t>(T) * 4;
  char* p = static_cast<char*>(ws);
  int32_t* keys0 = reinterpret_cast<int32_t*>(p); p += up256(t4);
  int32_t* keys1 = reinterpret_cast<int32_t*>(p); p += up256(t4);
  int32_t* vals0 = reinterpret_cast<int32_t*>(p); p += up256(t4);
  int32_t* vals1 = reinterpret_cast<int32_t*>(p); p += up256(t4);
  int32_t* hist = reinterpret_cast<int32_t*>(p); p += up256(static_cast<size_t>(256) * nblk * 4);
  int32_t* offsets = reinterpret_cast<int32_t*>(p); p += up256(static_cast<size_t>(V) * 4);
  int32_t* ends = reinterpret_cast<int32_t*>(p); p += up256(static_cast<size_t>(V) * 4);
  const int64_t max_heavy = T / (kHeavy + 1) + 1;
  const int64_t max_light = T < V ? T : V;
  int32_t* heavy = reinterpret_cast<int32_t*>(p); p += up256(static_cast<size_t>(max_heavy) * 4);
  int32_t* light = reinterpret_cast<int32_t*>(p); p += up256(static_cast<size_t>(max_light) * 4);
  int32_t* counts = reinterpret_cast<int32_t*>(p);        // [0] heavy ids, [1] light ids

  // stable radix sort of the ids carrying token indices
  int bits = 1;
  while ((int64_t(1) << bits) <= V) ++bits;          // keys live in [0, V]
  const int passes = (bits + 7) / 8;
  const int32_t* kin = nullptr;
  const int32_t* vin = nullptr;
  int32_t* kbuf[2] = {keys0, keys1};
  int32_t* vbuf[2] = {vals0, vals1};
  for (int pass = 0; pass < passes; ++pass) {
    sort_hist_kernel<<<static_cast<unsigned>(nblk), kSortBlock, 0, st>>>(kin, ids, T, V, 8 * pass, hist,
                                                                         static_cast<int>(nblk));
    exclusive_scan_kernel<<<1, 1024, 0, st>>>(hist, static_cast<int>(256 * nblk));
    sort_scatter_kernel<<<static_cast<unsigned>(nblk), kSortBlock, 0, st>>>(
        kin, vin, ids, T, V, 8 * pass, hist, static_cast<int>(nblk), kbuf[pass & 1], vbuf[pass & 1]);
    note_launches(3);
    kin = kbuf[pass & 1];
    vin = vbuf[pass & 1];
  }
  // per-id segment bounds in sorted order, and the heavy ids
  cudaError_t err = cudaMemsetAsync(offsets, 0, static_cast<size_t>(V) * 4, st);
  if (err == cudaSuccess) err = cudaMemsetAsync(ends, 0, static_cast<size_t>(V) * 4, st);
  if (err == cudaSuccess) err = cudaMemsetAsync(counts, 0, 8, st);
  if (err != cudaSuccess) return err;
  segment_bounds_kernel<<<static_cast<unsigned>((T + 255) / 256), 256, 0, st>>>(kin, T, V, offsets, ends, heavy,
                                                                                light, counts);
  note_launches(1);
  out->V = V;
  out->ends = ends;
  out->offsets = offsets;
  out->toks = vin;
  out->heavy = heavy;
  out->n_heavy = counts;
  out->max_heavy = max_heavy;
  out->light = light;
  out->n_light = counts + 1;
  out->max_light = max_light;
  return cudaGetLastError();
}

cudaError_t scatter_table_grads(const SegIndexDev& ix, bool bf16, int njobs, const TableGradJob* tj, bool accumulate,
                                cudaStream_t st, cudaStream_t heavy_st) {
  SegJobs jobs{};
  for (int z = 0; z < njobs; ++z)
    jobs.j[z] = SegJob{static_cast<const uint4*>(tj[z].dy), tj[z].d_vec + tj[z].dl_vec, tj[z].d_vec, tj[z].dl_vec,
                       static_cast<const uint4*>(tj[z].E), tj[z].dE, tj[z].ge, tj[z].coef};
  return bf16 ? launch_segsum<true, true>(ix, jobs, njobs, accumulate, st, heavy_st)
              : launch_segsum<false, true>(ix, jobs, njobs, accumulate, st, heavy_st);
}

cudaError_t scatter_table_grad(const SegIndexDev& ix, bool bf16, const void* dy, int d_vec, int dl_vec,
                               const float* coef, float ge, const void* E, float* dE, bool accumulate,
                               cudaStream_t st) {
  const TableGradJob j{dy, d_vec, dl_vec, coef, ge, E, dE};
  return scatter_table_grads(ix, bf16, 1, &j, accumulate, st, st);
}

cudaError_t scatter_target_rows(const SegIndexDev& ix, int njobs, const void* const* h, const int* d_vec,
                                float* const* dW, const float* scale, cudaStream_t st, cudaStream_t heavy_st) {
  SegJobs jobs{};
  for (int z = 0; z < njobs; ++z)
    jobs.j[z] = SegJob{static_cast<const uint4*>(h[z]), d_vec[z], 0, d_vec[z], nullptr, dW[z], scale[z], nullptr};
  return launch_segsum<true, false>(ix, jobs, njobs, 1, st, heavy_st);
}

}  // namespace mls
