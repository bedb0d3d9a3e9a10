// Tensor-core (tcgen05 + TMEM + TMA) path of the multi-exit LM-head loss, bf16.
//
// Forward.  A persistent kernel walks (token tile of 128) x (vocab tile of 256)
// output tiles.  For each tile it computes the logits of every exit, teacher
// (largest exit) first, into two alternating TMEM regions, and an 8-warp
// epilogue turns each 128-column half ("split") into per-row softmax
// statistics without ever writing logits out:
//   teacher: lse_T over the split and p~ = exp(l_T - max_T) kept in registers;
//   student s: lse_s over the split and Abar_s = sum_v p~_v l_s,v / sum_v p~_v.
// A merge kernel combines the per-split partials of every token exactly (log-
// sum-exp merge, teacher-weighted mean of Abar), which gives lse_m and
// S_m = sum_v p_T,v l_m,v; a fixed-order reduction gives the losses.
//
// Backward.  The same mainloop recomputes each tile's logits; the epilogue forms
// the dense part of the logit gradient
//   G'_m = q_m - alpha_d p_T   (students),   G'_T = p_T   (teacher, stop-gradient)
// in fp16 into a workspace, one block of tokens x one chunk of the vocabulary
// at a time, and two tensor-core GEMMs per exit (fp16 operands: G' and fp16
// copies of the chunk's W rows and the block's h rows) produce
//   dh_m = a (G'_m W^m - c_m W^m[y_t])   and   dW^m (+)= a G'_m^T h_m - a c_m sum_{t: y_t = v} h_t,
// a = grad_scale/T, c_m = 1 - alpha_d (students) or 1 (teacher).  The one-hot
// term is applied exactly in fp32 (a row gather in the dh epilogue and an
// id-grouped row sum for dW) instead of being rounded into G'.  fp16 holds
// G' with an 11-bit significand where bf16 holds 8: the rounding of the large
// entries of peaked rows, which dominates the error of dW, is 8x smaller.
//
// Definitions: "Matryoshka Language Model Suites" (agihunt.info summary,
// distillation paragraph), "Is nesting the cheapest way to build a model
// suite?" (section 4, the 0.7/0.3 mix), "Editing the methods of sub-models are
// made of blocks" (Modeling paragraph: one LM head W^m in R^{V x D_m} per exit).
#include <cuda.h>
#include <cuda_fp16.h>
#include <mutex>

#include "kernels.h"
#include "umma.cuh"

// Raster groups.  Grouped GEMMs: tile rows (of 256 on CTA pairs) per group;
// consecutive tiles go down a group's rows before moving to the next column,
// so a wave of CTAs shares the group's A panels and a few B panels in L2.
// Loss tile kernel: 128-token tiles per group; a group's h panels stay in L2
// while the heads stream past them.
#ifndef MLS_DH_GROUP_M
#define MLS_DH_GROUP_M 8
#endif
#ifndef MLS_DW_GROUP_M
#define MLS_DW_GROUP_M 8
#endif
#ifndef MLS_LOSS_GROUP_TT
#define MLS_LOSS_GROUP_TT 16
#endif

namespace mls {

namespace {

constexpr int kBM = 128;          // token rows per tile (UMMA M)
constexpr int kBK = 64;           // K per stage: one 128-byte swizzle row of bf16
constexpr int kUK = 16;           // K per tcgen05.mma (kind::f16)
constexpr int kThreads = 192;     // GEMM: warp 0 TMA, warp 1 MMA, warps 2-5 epilogue
constexpr float kLog2e = 1.4426950408889634f;

// Loss tile kernel geometry.  One tile = 128 tokens x 256 vocabulary columns;
// each exit's logits of the tile are one accumulation "job" in TMEM.  Two
// 256-column TMEM regions alternate between consecutive jobs, so the epilogue
// of one job overlaps the MMAs of the next.  Eight epilogue warps: two per
// TMEM lane quadrant, each owning one 128-column half ("split") of the tile.
constexpr int kLossBN = 256;
constexpr int kSplitCols = 128;
constexpr int kLossStages = 4;        // 48 KB per stage
constexpr int kLossEpiWarps = 8;
constexpr int kLossThreads = 64 + 32 * kLossEpiWarps;

// ------------------------------------------------------------------ shared layouts
struct LossMaps {
  CUtensorMap h[kMaxExits];
  CUtensorMap w[kMaxExits];
};

struct LossArgs {
  int M;
  int T;                       // tokens of this launch (a block of the call's tokens in the backward)
  int V;                       // vocabulary columns of this launch (a chunk in the backward)
  int v0;                      // first vocabulary id of the launch's columns
  int Vtot;                    // the vocabulary size (targets outside [0, Vtot) are invalid)
  int ldS;                     // row stride of stats (the call's token count)
  int kblocks[kMaxExits];      // D_m / kBK
  int n_tt, n_vt, num_tiles;
  int group_tt;                // token tiles per raster group (W streams once per group)
  const int32_t* y;
  float alpha;                 // alpha_d
  int distill;                 // 0: cross-entropy, 1: KL(q_m || p_M), 2: Jensen-Shannon, 3: 1 - sum min(q, p)
  float exit_w[kMaxExits];     // per-exit weights (teacher-gradient backward only)
  float student_wsum;          // sum of the smaller exits' weights
  float* partial;              // forward: [2 n_vt][2M-1][T]
  float* stats;                // forward: target rows written; backward: lse read
  __half* G;                   // backward: fp16 G' [M][T][V] of the launch's tokens and columns
  int32_t* status;
  uint64_t wait_ns;            // limit of every barrier wait (the library default, or a test's)
  int withhold_loads;          // test of the bounded waits: the producer issues no loads
};

// Per-warp staging of one 32-row x 32-column bf16 chunk of G' (rows padded
// to 80 bytes so the 16-byte writes of a warp hit every bank once per pass).
constexpr int kStageRowBytes = 80;

struct __align__(1024) LossSmem {
  static constexpr int kStages = kLossStages;
  uint8_t a[kStages][kBM * kBK * 2];
  uint8_t b[kStages][kLossBN * kBK * 2];
  uint8_t gstage[kLossEpiWarps][32 * kStageRowBytes];
  uint64_t full[kStages];
  uint64_t empty[kStages];
  uint64_t tfull[2];
  uint64_t tempty[2];
  uint64_t drain;
  uint32_t tmem_base;
  int abort;
};

enum LossMode { kModeStats = 0, kModeGrad = 1, kModeAgree = 2, kModeJS = 3 };

// Partial rows per split in agreement mode: beta_s, KL_s (students), max_m, argmax_m.
__host__ __device__ constexpr int agree_rows(int M) { return 4 * M - 2; }

// Partial rows per split of the Jensen-Shannon pass: sum q log(q/mu) and
// sum p log(p/mu) of every student (mu the mixture (q + p)/2).
__host__ __device__ constexpr int js_rows(int M) { return 2 * (M - 1); }

constexpr float kLn2 = 0.6931471805599453f;

// log(1 + e^x), without overflow for large x.
__device__ __forceinline__ float softplus(float x) { return fmaxf(x, 0.f) + __logf(1.f + __expf(-fabsf(x))); }

// Tile i of the launch -> (token tile, vocabulary tile).  Tiles are visited in
// groups of group_tt token tiles x every vocabulary tile, vocabulary tiles
// outer, so the group's h rows stay in L2 while the heads stream past (W is
// read once per token group).
__device__ __forceinline__ void loss_tile_coords(int i, const LossArgs& a, int& tt, int& vt) {
  const int per_group = a.group_tt * a.n_vt;
  const int g = i / per_group;
  const int first = g * a.group_tt;
  const int gt = min(a.group_tt, a.n_tt - first);
  const int r = i - g * per_group;
  vt = r / gt;
  tt = first + r % gt;
}

// All lanes of a warp wait; the warp agrees on the outcome.
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, volatile int* abort, int32_t* status,
                                          uint64_t limit_ns = kWaitLimitNs) {
  const bool ok = mbar_wait(bar, parity, abort, status, limit_ns);
  return __all_sync(0xffffffffu, ok);
}

// Time-bounded wait that ignores the abort flag (used while draining).
__device__ __forceinline__ void drain_wait(uint64_t* bar, uint32_t parity, int32_t* status) {
  int dummy = 0;
  (void)mbar_wait(bar, parity, &dummy, status);
}

// Teacher probabilities are kept in registers as fp16 pairs (11-bit
// significand) for the students of the same tile.  Values below fp16's range
// (under about 6e-8 relative to the split maximum or the normaliser) carry
// negligible weight in the statistics and in G'; the agreement pass, whose
// acceptance sums those tiny values, reads the teacher's logits from TMEM
// instead (see job_slot).
__device__ __forceinline__ uint32_t pack_p2(float lo, float hi) {
  __half2 h = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}

__device__ __forceinline__ float2 unpack_p2(uint32_t u) { return __half22float2(*reinterpret_cast<__half2*>(&u)); }

// G' is stored in fp16 (11-bit significand, 8x finer than bf16's): round to
// nearest, and values beyond the largest finite fp16 (65504, far outside any
// logit gradient of finite logits) saturate instead of becoming infinite.
__device__ __forceinline__ uint32_t pack_g2(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.satfinite.f16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

// acc + w * x on fp16 pairs (the teacher-gradient accumulator).
__device__ __forceinline__ uint32_t hfma_p2(uint32_t w, uint32_t x, uint32_t acc) {
  __half2 r = __hfma2(*reinterpret_cast<__half2*>(&w), *reinterpret_cast<__half2*>(&x),
                      *reinterpret_cast<__half2*>(&acc));
  return *reinterpret_cast<uint32_t*>(&r);
}

// r[i] of this lane's 32 register values, through the lane's own row of
// shared memory (an indexed read of the registers would move the whole array
// to local memory, and a tree of selects needs 16 more live registers).  The
// row holds 16 values; only this lane reads or writes it.
__device__ __forceinline__ float pick32(const float (&r)[32], int i, float4* row) {
  const int h = i >> 4;
#pragma unroll
  for (int u = 0; u < 4; ++u)
    row[u] = h ? make_float4(r[16 + 4 * u], r[17 + 4 * u], r[18 + 4 * u], r[19 + 4 * u])
               : make_float4(r[4 * u], r[4 * u + 1], r[4 * u + 2], r[4 * u + 3]);
  return reinterpret_cast<const float*>(row)[i & 15];
}

// TMEM region and use count of job j (exit M-1-j) of the tile_iter-th tile of a CTA.
// By default consecutive jobs alternate the two regions.  When the epilogue
// needs the teacher's logits at every element of a student's tile (the
// agreement mode, and the reverse-KL distillation), the teacher stays in
// region 0 for the whole tile and the students run one after another in
// region 1.
__device__ __forceinline__ void job_slot(bool hold_teacher, int M, uint32_t tile_iter, int j, uint32_t job,
                                         uint32_t& region, uint32_t& use) {
  if (hold_teacher) {
    region = (j == 0) ? 0u : 1u;
    use = (j == 0) ? tile_iter : tile_iter * static_cast<uint32_t>(M - 1) + static_cast<uint32_t>(j - 1);
  } else {
    region = job & 1u;
    use = job >> 1;
  }
}

// One 32-column chunk of G' (this lane's row: 16 packed fp16 pairs) through the
// warp's staging rows, so that each store instruction writes 8 rows x 64
// contiguous bytes (full sectors).  Rows at or past T are not stored.
__device__ __forceinline__ void store_g_chunk(uint8_t* stage, int lane, const uint32_t (&packed)[16],
                                              __half* G, int row0, int T, int V, int col) {
  uint4* mine = reinterpret_cast<uint4*>(stage + lane * kStageRowBytes);
#pragma unroll
  for (int u = 0; u < 4; ++u)
    mine[u] = make_uint4(packed[4 * u], packed[4 * u + 1], packed[4 * u + 2], packed[4 * u + 3]);
  __syncwarp();
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int piece = i * 32 + lane;
    const int rr = piece >> 2, ch = piece & 3;
    const uint4 v = *reinterpret_cast<const uint4*>(stage + rr * kStageRowBytes + ch * 16);
    if (row0 + rr < T) *reinterpret_cast<uint4*>(G + static_cast<int64_t>(row0 + rr) * V + col + ch * 8) = v;
  }
  __syncwarp();
}

// ------------------------------------------------------------------ loss tile kernel
// DISTILL (0 cross-entropy, 1 reverse KL, 2 Jensen-Shannon, 3 acceptance) is a template
// parameter so that each form gets its own register allocation.  TGRAD (the
// backward without the teacher's stop-gradient) holds the teacher's logits in
// region 0 while the students pass through region 1, accumulates each
// student's contribution to the teacher's logit gradient in registers (fp16
// pairs), and writes the teacher's G' after the last student.
template <int MODE, int DISTILL, bool TGRAD = false>
__global__ void __launch_bounds__(kLossThreads, 1) loss_tile_kernel(const __grid_constant__ LossMaps maps,
                                                                    const LossArgs a) {
  using Smem = LossSmem;
  constexpr int kStages = Smem::kStages;
  extern __shared__ uint8_t smem_raw[];
  Smem& s = *reinterpret_cast<Smem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  volatile int* abort = &s.abort;
  const int M = a.M;
  const int slot = static_cast<int>(blockIdx.x);
  const int nslots = static_cast<int>(gridDim.x);
  constexpr bool rkl = (DISTILL == 1);
  constexpr bool jsd = (DISTILL == 2);
  constexpr bool accd = (DISTILL == 3);
  // The statistics of the Jensen-Shannon form are the cross-entropy ones (it
  // needs the final normalisers, so its divergence has a pass of its own).
  constexpr bool hold =
      (MODE == kModeAgree) || (MODE == kModeJS) || rkl || (MODE == kModeGrad && (jsd || accd || TGRAD));
  static_assert(!TGRAD || MODE == kModeGrad, "teacher gradient: backward only");

  if (threadIdx.x == 0) {
    for (int i = 0; i < kStages; ++i) {
      mbar_init(&s.full[i], 1);
      mbar_init(&s.empty[i], 1);
    }
    for (int r = 0; r < 2; ++r) {
      mbar_init(&s.tfull[r], 1);
      mbar_init(&s.tempty[r], kLossEpiWarps);
    }
    mbar_init(&s.drain, 1);
    s.abort = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    for (int m = 0; m < M; ++m) {
      tma_prefetch_desc(&maps.h[m]);
      tma_prefetch_desc(&maps.w[m]);
    }
  }
  if (warp == 1) {
    tmem_alloc(&s.tmem_base, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = s.tmem_base;
  // an epilogue warp is done with TMEM region r
  auto release_region = [&](uint32_t r) { mbar_arrive(&s.tempty[r]); };

  if (warp == 0) {
    // ---------------------------------------------------------------- TMA producer
    if (lane == 0 && !a.withhold_loads) {
      uint32_t stage = 0, phase = 0, issued = 0;
      bool ok = true;
      for (int tile = slot; tile < a.num_tiles && ok; tile += nslots) {
        int tt, vt;
        loss_tile_coords(tile, a, tt, vt);
        const int row0 = tt * kBM;               // the tile's tokens
        const int v0 = vt * kLossBN;             // the tile's W rows
        for (int j = 0; j < M && ok; ++j) {
          const int m = M - 1 - j;                // teacher first, then students
          for (int kb = 0; kb < a.kblocks[m]; ++kb) {
            if (!mbar_wait(&s.empty[stage], phase ^ 1, abort, a.status, a.wait_ns)) { ok = false; break; }
            mbar_arrive_expect_tx(&s.full[stage], (kBM + kLossBN) * kBK * 2);
            tma_load_2d(&maps.h[m], &s.full[stage], s.a[stage], kb * kBK, row0);
            tma_load_2d(&maps.w[m], &s.full[stage], s.b[stage], kb * kBK, v0);
            ++issued;
            if (++stage == kStages) { stage = 0; phase ^= 1; }
          }
        }
      }
      if (!ok) {
        // Let every load already issued land before the CTA can exit.
        const uint32_t n = issued < kStages ? issued : kStages;
        uint32_t st = stage, ph = phase;
        for (uint32_t i = 0; i < n; ++i) {
          if (st == 0) { st = kStages - 1; ph ^= 1; } else { --st; }
          drain_wait(&s.full[st], ph, a.status);
        }
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16(kBM, kLossBN, false, false);
      uint32_t stage = 0, phase = 0, job = 0, tile_iter = 0;
      bool ok = true;
      for (int tile = slot; tile < a.num_tiles && ok; tile += nslots, ++tile_iter) {
        for (int j = 0; j < M && ok; ++j, ++job) {
          const int m = M - 1 - j;
          uint32_t region, use;
          job_slot(hold, M, tile_iter, j, job, region, use);
          if (!mbar_wait(&s.tempty[region], (use & 1) ^ 1, abort, a.status, a.wait_ns)) { ok = false; break; }
          tc_fence_after();
          const uint32_t d = tmem + region * kLossBN;
          for (int kb = 0; kb < a.kblocks[m]; ++kb) {
            if (!mbar_wait(&s.full[stage], phase, abort, a.status, a.wait_ns)) { ok = false; break; }
            tc_fence_after();
            const uint64_t da = smem_desc_sw128(smem_u32(s.a[stage]), 16, 1024);
            const uint64_t db = smem_desc_sw128(smem_u32(s.b[stage]), 16, 1024);
#pragma unroll
            for (int k = 0; k < kBK / kUK; ++k) {
              // +32 bytes along K inside the 128-byte swizzled row
              umma_bf16(d, da + static_cast<uint64_t>(k * 2), db + static_cast<uint64_t>(k * 2), idesc,
                        (kb | k) != 0);
            }
            umma_commit(&s.empty[stage]);
            if (++stage == kStages) { stage = 0; phase ^= 1; }
          }
          if (ok) umma_commit(&s.tfull[region]);
        }
      }
      // Make sure every MMA issued has finished before TMEM is released.
      umma_commit(&s.drain);
      drain_wait(&s.drain, 0, a.status);
    }
  } else {
    // ---------------------------------------------------------------- epilogue (8 warps)
    const int q = warp & 3;                          // TMEM lane quadrant this warp may access
    const int half = (warp - 2) >> 2;                // which 128-column split of the tile
    const int row = q * 32 + lane;
    float4* tgt_row = reinterpret_cast<float4*>(s.gstage[warp - 2] + lane * kStageRowBytes);
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(q * 32) << 16) + half * kSplitCols;
    const int Q = 2 * M - 1;
    const float al = a.alpha;
    uint32_t job = 0, tile_iter = 0;
    // teacher probabilities of this thread's row and split, packed fp16 pairs
    uint32_t pt[4][16];
    float inv_z = 0.f;
    for (int tile = slot; tile < a.num_tiles; tile += nslots, ++tile_iter) {
      int tt, vt;
      loss_tile_coords(tile, a, tt, vt);
      const int rbase = tt * kBM;                           // first token of the tile
      const int t = rbase + row;
      const bool valid = t < a.T;
      const int c0 = vt * kLossBN + half * kSplitCols;     // first vocabulary column of the split
      const bool live = c0 < a.V;                           // the last tile may be half outside V
      const int split = vt * 2 + half;
      const int yt = valid ? __ldg(a.y + t) : -1;
      const int yl = yt - a.v0 - c0;                        // target column inside this split, if any
      const bool has_tgt = valid && yl >= 0 && yl < kSplitCols;
      const bool bad = valid && (yt < 0 || yt >= a.Vtot);
      bool stop = false;
      for (int j = 0; j < M; ++j, ++job) {
        const int m = M - 1 - j;
        uint32_t region, use;
        job_slot(hold, M, tile_iter, j, job, region, use);
        const uint32_t base = lane_base + region * kLossBN;
        const uint32_t tbase = lane_base;                   // region 0: the teacher, when held
        if (!warp_wait(&s.tfull[region], use & 1, abort, a.status, a.wait_ns)) { stop = true; break; }
        tc_fence_after();
        if (MODE == kModeStats) {
          float lse_part = -INFINITY, abar = 0.f;
          if (live) {
            if (j == 0) {
              // teacher, one pass over TMEM: online split max; p~ = exp(l - max) as fp16 pairs
              // in registers, the pairs of earlier chunks (and their sum) rescaled by the same
              // fp16 factor when a larger maximum appears
              float mx = -INFINITY, z = 0.f;
#pragma unroll
              for (int c = 0; c < 4; ++c) {
                float r[32];
                tmem_ld32(base + c * 32, r);
                float cm = r[0];
#pragma unroll
                for (int k = 1; k < 32; ++k) cm = fmaxf(cm, r[k]);
                if (has_tgt && (yl >> 5) == c) {
                  a.stats[static_cast<int64_t>(M + m) * a.ldS + t] = pick32(r, yl & 31, tgt_row);
                }
                if (cm > mx) {
                  const uint32_t sc2 = pack_p2(exp2f((mx - cm) * kLog2e), 0.f);
                  z *= unpack_p2(sc2).x;
                  const uint32_t scc = __byte_perm(sc2, sc2, 0x1010);
#pragma unroll
                  for (int c2 = 0; c2 < c; ++c2) {
#pragma unroll
                    for (int k = 0; k < 16; ++k) {
                      uint32_t v;
                      asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(v) : "r"(pt[c2][k]), "r"(scc));
                      pt[c2][k] = v;
                    }
                  }
                  mx = cm;
                }
                const float mxs = mx * kLog2e;
#pragma unroll
                for (int k = 0; k < 32; k += 2) {
                  const float e0 = exp2f(fmaf(r[k], kLog2e, -mxs));
                  const float e1 = exp2f(fmaf(r[k + 1], kLog2e, -mxs));
                  z += e0 + e1;
                  pt[c][k / 2] = pack_p2(e0, e1);
                }
              }
              inv_z = 1.f / z;
              lse_part = mx + logf(z);
            } else if (rkl) {
              // student, reverse KL: online max/sum over the split and the
              // student-weighted sum of (l_m - l_T), the teacher read from region 0
              float ms = -INFINITY, zs = 0.f, B = 0.f;
#pragma unroll 1
              for (int c = 0; c < 4; ++c) {
                float r[32], lt[32];
                tmem_ld32(base + c * 32, r);
                tmem_ld32(tbase + c * 32, lt);
                float cm = r[0];
#pragma unroll
                for (int k = 1; k < 32; ++k) cm = fmaxf(cm, r[k]);
                const float mn = fmaxf(ms, cm);
                const float mns = mn * kLog2e;
                float zc = 0.f, bc = 0.f;
#pragma unroll
                for (int k = 0; k < 32; ++k) {
                  const float e = exp2f(fmaf(r[k], kLog2e, -mns));
                  zc += e;
                  bc = fmaf(e, r[k] - lt[k], bc);
                }
                const float rs = exp2f((ms - mn) * kLog2e);
                zs = zs * rs + zc;
                B = B * rs + bc;
                ms = mn;
                if (has_tgt && (yl >> 5) == c) {
                  a.stats[static_cast<int64_t>(M + m) * a.ldS + t] = pick32(r, yl & 31, tgt_row);
                }
              }
              lse_part = ms + logf(zs);
              abar = B / zs;
            } else {
              // student: online max/sum over the split and the teacher-weighted sum of its logits
              float ms = -INFINITY, zs = 0.f, A = 0.f;
#pragma unroll
              for (int c = 0; c < 4; ++c) {
                float r[32];
                tmem_ld32(base + c * 32, r);
                float cm = r[0];
#pragma unroll
                for (int k = 1; k < 32; ++k) cm = fmaxf(cm, r[k]);
                const float mn = fmaxf(ms, cm);
                const float mns = mn * kLog2e;
                float zc = 0.f;
#pragma unroll
                for (int k = 0; k < 32; k += 2) {
                  zc += exp2f(fmaf(r[k], kLog2e, -mns)) + exp2f(fmaf(r[k + 1], kLog2e, -mns));
                  const float2 pp = unpack_p2(pt[c][k / 2]);
                  A = fmaf(pp.x, r[k], A);
                  A = fmaf(pp.y, r[k + 1], A);
                }
                zs = zs * exp2f((ms - mn) * kLog2e) + zc;
                ms = mn;
                if (has_tgt && (yl >> 5) == c) {
                  a.stats[static_cast<int64_t>(M + m) * a.ldS + t] = pick32(r, yl & 31, tgt_row);
                }
              }
              lse_part = ms + logf(zs);
              abar = A * inv_z;
            }
          }
          tc_fence_before();
          __syncwarp();
          if (lane == 0) {
            if (!hold) {
              release_region(region);
            } else {
              if (j > 0) release_region(1);         // this student's region
              if (j == M - 1) release_region(0);    // the teacher's, after the last student
            }
          }
          if (valid) {
            a.partial[(static_cast<int64_t>(split) * Q + m) * a.T + t] = lse_part;
            if (j > 0) a.partial[(static_cast<int64_t>(split) * Q + M + m) * a.T + t] = abar;
          }
        } else if (MODE == kModeAgree) {
          // ---------------- agreement with the largest exit.  The teacher's tile stays in
          // region 0 while each student's tile arrives in region 1: per element
          // p = exp(l_T - lse_T), q = exp(l_m - lse_m); sum min(q, p) and
          // sum p (log p - log q); first maximum of each exit's logits.
          float mxv = -INFINITY, sum_min = 0.f, kl = 0.f;
          int mxi = -1;
          if (live) {
            const float lse = valid ? a.stats[static_cast<int64_t>(m) * a.ldS + t] : 0.f;
            const float lseT = valid ? a.stats[static_cast<int64_t>(M - 1) * a.ldS + t] : 0.f;
#pragma unroll 1
            for (int c = 0; c < 4; ++c) {
              float r[32];
              tmem_ld32(base + c * 32, r);
#pragma unroll
              for (int k = 0; k < 32; ++k)
                if (r[k] > mxv) { mxv = r[k]; mxi = c0 + c * 32 + k; }
              if (j > 0) {
                float lt[32];
                tmem_ld32(tbase + c * 32, lt);
#pragma unroll
                for (int k = 0; k < 32; ++k) {
                  const float la = lt[k] - lseT;            // log p
                  const float lb = r[k] - lse;              // log q
                  const float pv = exp2f(la * kLog2e);
                  const float qv = exp2f(lb * kLog2e);
                  sum_min += fminf(pv, qv);
                  kl = fmaf(pv, la - lb, kl);
                }
              }
            }
          }
          tc_fence_before();
          __syncwarp();
          if (lane == 0) {
            if (j > 0) release_region(1);         // this student's region
            if (j == M - 1) release_region(0);    // the teacher's, after the last student
          }
          if (valid) {
            const int QA = agree_rows(M);
            float* prow = a.partial + static_cast<int64_t>(split) * QA * a.T + t;
            if (j > 0) {
              prow[static_cast<int64_t>(m) * a.T] = sum_min;
              prow[static_cast<int64_t>(M - 1 + m) * a.T] = kl;
            }
            prow[static_cast<int64_t>(2 * (M - 1) + m) * a.T] = mxv;
            prow[static_cast<int64_t>(3 * M - 2 + m) * a.T] = __int_as_float(mxi);
          }
        } else if (MODE == kModeJS) {
          // ---------------- second pass with the final normalisers, Jensen-Shannon or
          // acceptance.  Jensen-Shannon, per element with d = log p - log q:
          //   log(q/mu) = ln 2 - softplus(d),  log(p/mu) = ln 2 - softplus(-d).
          float jq = 0.f, jp = 0.f;
          if (live && j > 0) {
            const float lse = valid ? a.stats[static_cast<int64_t>(m) * a.ldS + t] : 0.f;
            const float lseT = valid ? a.stats[static_cast<int64_t>(M - 1) * a.ldS + t] : 0.f;
#pragma unroll 1
            for (int c = 0; c < 4; ++c) {
              float r[32], lt[32];
              tmem_ld32(base + c * 32, r);
              tmem_ld32(tbase + c * 32, lt);
#pragma unroll
              for (int k = 0; k < 32; ++k) {
                const float lq = r[k] - lse;
                const float lp = lt[k] - lseT;
                if constexpr (accd) {
                  // acceptance: A = sum of q where q < p, B = sum of p where q >= p (beta = A + B)
                  if (lq < lp) jq += exp2f(lq * kLog2e);
                  else jp += exp2f(lp * kLog2e);
                } else {
                  const float d = lp - lq;
                  const float sp = __logf(1.f + __expf(-fabsf(d)));
                  jq = fmaf(exp2f(lq * kLog2e), kLn2 - fmaxf(d, 0.f) - sp, jq);
                  jp = fmaf(exp2f(lp * kLog2e), kLn2 - fmaxf(-d, 0.f) - sp, jp);
                }
              }
            }
          }
          tc_fence_before();
          __syncwarp();
          if (lane == 0) {
            if (j > 0) release_region(1);
            if (j == M - 1) release_region(0);
          }
          if (valid && j > 0) {
            float* prow = a.partial + static_cast<int64_t>(split) * js_rows(M) * a.T + t;
            prow[static_cast<int64_t>(m) * a.T] = jq;
            prow[static_cast<int64_t>(M - 1 + m) * a.T] = jp;
          }
        } else {
          // ---------------- backward: dense part of the logit gradient, bf16
          if (bad && j == 0 && vt == 0 && half == 0 && a.v0 == 0) set_flag(a.status, MLS_DEVFLAG_BAD_ID);
          uint8_t* const stage = s.gstage[warp - 2];
          const int row0 = rbase + q * 32;                   // first token row of this warp
          if (TGRAD && j == 0) {
#pragma unroll
            for (int c = 0; c < 4; ++c)
#pragma unroll
              for (int k = 0; k < 16; ++k) pt[c][k] = 0u;   // the teacher-gradient accumulator
          }
          const float lseT = (hold && valid) ? a.stats[static_cast<int64_t>(M - 1) * a.ldS + t] : 0.f;
          const float lsT = lseT * kLog2e;
          if (live && !(TGRAD && j == 0)) {
            const float lse = valid ? a.stats[static_cast<int64_t>(m) * a.ldS + t] : 0.f;
            const float ls = lse * kLog2e;
            // per-token statistic of the student from the forward pass:
            //   cross-entropy S_m = sum p_T l_m; reverse KL R_m = sum q_m (l_m - l_T), so that
            //   log q - log p - KL(q_m || p_T) = l_m - l_T - R_m;  Jensen-Shannon: K = KL(q_m || mu) / 2
            const float klt = (hold && j > 0 && valid) ? a.stats[static_cast<int64_t>(2 * M + m) * a.ldS + t] : 0.f;
            // Jensen-Shannon with the teacher gradient: K^p = KL(p_T || mu)/2, stored by the forward pass
            const float kpt = (TGRAD && (jsd || accd) && j > 0 && valid)
                                  ? a.stats[static_cast<int64_t>(3 * M - 1 + m) * a.ldS + t]
                                  : 0.f;
            const uint32_t wm2 = TGRAD ? pack_p2(a.exit_w[m], a.exit_w[m]) : 0u;
            // unrolled where a register array is indexed by c (the teacher's
            // packed probabilities, or the teacher-gradient accumulator)
            constexpr int kUnrollC = (hold && !TGRAD) ? 1 : 4;
            // TMEM is read 16 columns at a time when the accumulator is live
            constexpr int kW = TGRAD ? 16 : 32;
#pragma unroll kUnrollC
            for (int c = 0; c < 4; ++c) {
              uint32_t packed[16];
#pragma unroll
              for (int sub = 0; sub < 32 / kW; ++sub) {
              float r[kW];
              tmem_ld<kW>(base + c * 32 + sub * kW, r);
              float lt[kW];
              if (hold && j > 0) {
                tmem_ld<kW>(tbase + c * 32 + sub * kW, lt);
              } else {
#pragma unroll
                for (int k = 0; k < kW; ++k) lt[k] = 0.f;
              }
#pragma unroll
              for (int kk = 0; kk < kW; kk += 2) {
                const int k = sub * kW + kk;       // column inside the 32-column chunk (pair index k / 2)
                const float e0 = exp2f(fmaf(r[kk], kLog2e, -ls));
                const float e1 = exp2f(fmaf(r[kk + 1], kLog2e, -ls));
                float g0, g1;
                if (j == 0) {                      // teacher: G' = p_T
                  if (!hold) pt[c][k / 2] = pack_p2(e0, e1);
                  g0 = e0;
                  g1 = e1;
                } else if (rkl) {                  // student: G' = q ((1 - a) + a (log q - log p - KL))
                  const float d0 = (r[kk] - lt[kk]) - klt;
                  const float d1 = (r[kk + 1] - lt[kk + 1]) - klt;
                  g0 = e0 * fmaf(al, d0, 1.f - al);
                  g1 = e1 * fmaf(al, d1, 1.f - al);
                  if (TGRAD) pt[c][k / 2] = hfma_p2(wm2, pack_p2(e0, e1), pt[c][k / 2]);   // sum_m w_m q_m
                } else if (jsd) {                  // student: G' = q ((1 - a) + a (log(q/mu)/2 - K))
                  // x = log p - log q; log(q/mu) = ln 2 - softplus(x), log(p/mu) = ln 2 - softplus(x) + x
                  const float x0 = (lt[kk] - lseT) - (r[kk] - lse);
                  const float x1 = (lt[kk + 1] - lseT) - (r[kk + 1] - lse);
                  const float sp0 = softplus(x0), sp1 = softplus(x1);
                  const float d0 = fmaf(-0.5f, sp0, 0.5f * kLn2) - klt;
                  const float d1 = fmaf(-0.5f, sp1, 0.5f * kLn2) - klt;
                  g0 = e0 * fmaf(al, d0, 1.f - al);
                  g1 = e1 * fmaf(al, d1, 1.f - al);
                  if (TGRAD)                       // sum_m w_m (log(p/mu_m)/2 - K^p_m)
                    pt[c][k / 2] = hfma_p2(wm2, pack_p2(0.5f * (kLn2 - sp0 + x0) - kpt, 0.5f * (kLn2 - sp1 + x1) - kpt),
                                           pt[c][k / 2]);
                } else if (accd) {                 // student: G' = q ((1 - a) + a (A - [q < p]))
                  const float i0 = (r[kk] - lse < lt[kk] - lseT) ? 1.f : 0.f;
                  const float i1 = (r[kk + 1] - lse < lt[kk + 1] - lseT) ? 1.f : 0.f;
                  g0 = e0 * fmaf(al, klt - i0, 1.f - al);
                  g1 = e1 * fmaf(al, klt - i1, 1.f - al);
                  if (TGRAD)                       // sum_m w_m (B_m - [q_m >= p])
                    pt[c][k / 2] = hfma_p2(wm2, pack_p2(kpt - (1.f - i0), kpt - (1.f - i1)), pt[c][k / 2]);
                } else {                           // student: G' = q - alpha_d p_T
                  float p0, p1;
                  if (hold) {
                    p0 = exp2f(fmaf(lt[kk], kLog2e, -lsT));
                    p1 = exp2f(fmaf(lt[kk + 1], kLog2e, -lsT));
                  } else {
                    const float2 pp = unpack_p2(pt[c][k / 2]);
                    p0 = pp.x;
                    p1 = pp.y;
                  }
                  g0 = fmaf(-al, p0, e0);
                  g1 = fmaf(-al, p1, e1);
                  if (TGRAD)                       // sum_m w_m (l_m - S_m)
                    pt[c][k / 2] = hfma_p2(wm2, pack_p2(r[kk] - klt, r[kk + 1] - klt), pt[c][k / 2]);
                }
                packed[k / 2] = bad ? 0u : pack_g2(g0, g1);
              }
              }
              store_g_chunk(stage, lane, packed, a.G + static_cast<int64_t>(m) * a.T * a.V, row0, a.T, a.V,
                            c0 + c * 32);
            }
          }
          if (TGRAD && j == M - 1 && j > 0 && live) {
            // the teacher's G' with every student's distillation gradient:
            //   cross-entropy:  w_T p - a p sum_m w_m (l_m - S_m)
            //   reverse KL:     (w_T + a sum_m w_m) p - a sum_m w_m q_m
            //   Jensen-Shannon: w_T p + a p sum_m w_m (log(p/mu_m)/2 - K^p_m)
            //   acceptance:     w_T p + a p sum_m w_m (B_m - [q_m >= p])
            const float wT = a.exit_w[M - 1];
            const float cp = rkl ? fmaf(al, a.student_wsum, wT) : wT;
#pragma unroll
            for (int c = 0; c < 4; ++c) {
              uint32_t packed[16];
#pragma unroll
              for (int sub = 0; sub < 2; ++sub) {
                float lt[16];
                tmem_ld16(tbase + c * 32 + sub * 16, lt);
#pragma unroll
                for (int kk = 0; kk < 16; kk += 2) {
                  const int k = sub * 16 + kk;
                  const float p0 = exp2f(fmaf(lt[kk], kLog2e, -lsT));
                  const float p1 = exp2f(fmaf(lt[kk + 1], kLog2e, -lsT));
                  const float2 acc = unpack_p2(pt[c][k / 2]);
                  float g0, g1;
                  if (rkl) {
                    g0 = fmaf(-al, acc.x, cp * p0);
                    g1 = fmaf(-al, acc.y, cp * p1);
                  } else if (jsd || accd) {
                    g0 = p0 * fmaf(al, acc.x, cp);
                    g1 = p1 * fmaf(al, acc.y, cp);
                  } else {
                    g0 = p0 * fmaf(-al, acc.x, cp);
                    g1 = p1 * fmaf(-al, acc.y, cp);
                  }
                  packed[k / 2] = bad ? 0u : pack_g2(g0, g1);
                }
              }
              store_g_chunk(stage, lane, packed, a.G + static_cast<int64_t>(M - 1) * a.T * a.V, row0, a.T, a.V,
                            c0 + c * 32);
            }
          }
          tc_fence_before();
          __syncwarp();
          if (lane == 0) {
            if (!hold) {
              release_region(region);
            } else {
              if (j > 0) release_region(1);
              if (j == M - 1) release_region(0);
            }
          }
        }
      }
      if (stop || *abort) break;
    }
  }

  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ------------------------------------------------------------------ merge kernel
// Per token: combine the per-split partials into lse_m and S_m, write the stats
// rows and the per-token loss terms.  A block covers 32 tokens; each of its
// thread rows merges a contiguous range of splits, and the rows' results are
// combined in row order (deterministic).
constexpr int kLossMergeRows = 32;   // thread rows per 32-token block of the loss merge
constexpr int kMergeRows = 16;       // ... of the agreement and Jensen-Shannon merges

__global__ void __launch_bounds__(32 * kLossMergeRows) loss_merge_kernel(const float* __restrict__ partial, int n_splits,
                                                                     int M, int T, int V, int distill,
                                                                     const int32_t* __restrict__ y,
                                                                     float* __restrict__ stats,
                                                                     float* __restrict__ terms, int32_t* status) {
  constexpr int S = kMaxExits - 1;
  __shared__ float st_mT[kLossMergeRows][32], st_zT[kLossMergeRows][32];
  __shared__ float st_A[kLossMergeRows][S][32], st_ms[kLossMergeRows][S][32], st_zs[kLossMergeRows][S][32];
  const int lane = threadIdx.x, rowi = threadIdx.y;
  const int t = blockIdx.x * 32 + lane;
  const int Q = 2 * M - 1;
  const int per = (n_splits + kLossMergeRows - 1) / kLossMergeRows;
  const int i0 = min(n_splits, rowi * per), i1 = min(n_splits, i0 + per);
  float mT = -INFINITY, zT = 0.f;
  float A[S] = {0.f, 0.f, 0.f}, ms[S] = {-INFINITY, -INFINITY, -INFINITY}, zs[S] = {0.f, 0.f, 0.f};
  if (t < T) {
    // The partials of kB splits are loaded before any of them is merged, so a
    // thread has that many independent loads in flight; padding splits past i1
    // read as empty (-inf, weight 0) and leave every sum unchanged.
    constexpr int kB = 4;
    for (int i = i0; i < i1; i += kB) {
      float lt[kB], lsv[kB][S], abv[kB][S];
#pragma unroll
      for (int u = 0; u < kB; ++u) {
        const bool in = i + u < i1;
        const float* pi = partial + static_cast<int64_t>(in ? i + u : i0) * Q * T + t;
        lt[u] = in ? pi[static_cast<int64_t>(M - 1) * T] : -INFINITY;
#pragma unroll
        for (int s = 0; s < S; ++s) {
          const bool ok = in && s < M - 1;
          lsv[u][s] = ok ? pi[static_cast<int64_t>(s) * T] : -INFINITY;
          abv[u][s] = ok ? pi[static_cast<int64_t>(M + s) * T] : 0.f;
        }
      }
#pragma unroll
      for (int u = 0; u < kB; ++u) {
        const float l = lt[u];
        if (l > mT) {
          const float r = __expf(mT - l);
          zT *= r;
          if (distill != 1) {   // teacher-weighted sums follow the teacher's max
#pragma unroll
            for (int s = 0; s < S; ++s) if (s < M - 1) A[s] *= r;
          }
          mT = l;
        }
        const float w = (l == -INFINITY) ? 0.f : __expf(l - mT);
        zT += w;
#pragma unroll
        for (int s = 0; s < S; ++s) if (s < M - 1) {
          const float ls = lsv[u][s];
          const float ab = abv[u][s];
          if (distill != 1) A[s] = fmaf(w, ab, A[s]);
          if (ls > ms[s]) {
            const float r = __expf(ms[s] - ls);
            zs[s] *= r;
            if (distill == 1) A[s] *= r;          // reverse KL: weights are the student's own
            ms[s] = ls;
          }
          if (ls != -INFINITY) {
            const float ws = __expf(ls - ms[s]);
            zs[s] += ws;
            if (distill == 1) A[s] = fmaf(ws, ab, A[s]);
          }
        }
      }
    }
  }
  st_mT[rowi][lane] = mT;
  st_zT[rowi][lane] = zT;
#pragma unroll
  for (int s = 0; s < S; ++s) {
    st_A[rowi][s][lane] = A[s];
    st_ms[rowi][s][lane] = ms[s];
    st_zs[rowi][s][lane] = zs[s];
  }
  __syncthreads();
  if (rowi != 0 || t >= T) return;
  for (int r = 1; r < kLossMergeRows; ++r) {
    const float m2 = st_mT[r][lane], z2 = st_zT[r][lane];
    const float mm = fmaxf(mT, m2);
    const float r1 = (mT == -INFINITY) ? 0.f : __expf(mT - mm);
    const float r2 = (m2 == -INFINITY) ? 0.f : __expf(m2 - mm);
    zT = zT * r1 + z2 * r2;
#pragma unroll
    for (int s = 0; s < S; ++s) if (s < M - 1) {
      const float n2 = st_ms[r][s][lane], y2 = st_zs[r][s][lane];
      const float mn = fmaxf(ms[s], n2);
      const float q1 = (ms[s] == -INFINITY) ? 0.f : __expf(ms[s] - mn);
      const float q2 = (n2 == -INFINITY) ? 0.f : __expf(n2 - mn);
      if (distill != 1) A[s] = A[s] * r1 + st_A[r][s][lane] * r2;
      else A[s] = A[s] * q1 + st_A[r][s][lane] * q2;
      zs[s] = zs[s] * q1 + y2 * q2;
      ms[s] = mn;
    }
    mT = mm;
  }
  const int yt = y[t];
  const bool bad = yt < 0 || yt >= V;
  const float lseT = mT + logf(zT);
  stats[static_cast<int64_t>(M - 1) * T + t] = lseT;
  if (bad) stats[static_cast<int64_t>(2 * M - 1) * T + t] = 0.f;
  terms[static_cast<int64_t>(M - 1) * T + t] = bad ? 0.f : lseT - stats[static_cast<int64_t>(2 * M - 1) * T + t];
#pragma unroll
  for (int s = 0; s < S; ++s) if (s < M - 1) {
    const float lse = ms[s] + logf(zs[s]);
    // cross-entropy: S = sum p_T l_m (teacher-weighted); reverse KL: R = sum q_m (l_m - l_T).
    // (Jensen-Shannon: S and the cross-entropy term here; its own pass overwrites both.)
    const float Sv = (distill != 1) ? A[s] / zT : A[s] / zs[s];
    const float kd = (distill != 1) ? lse - Sv : Sv - lse + lseT;
    stats[static_cast<int64_t>(s) * T + t] = lse;
    stats[static_cast<int64_t>(2 * M + s) * T + t] = Sv;
    if (bad) stats[static_cast<int64_t>(M + s) * T + t] = 0.f;
    terms[static_cast<int64_t>(s) * T + t] = bad ? 0.f : lse - stats[static_cast<int64_t>(M + s) * T + t];
    terms[static_cast<int64_t>(M + s) * T + t] = bad ? 0.f : kd;
  }
  if (bad) set_flag(status, MLS_DEVFLAG_BAD_ID);
}

// ------------------------------------------------------------------ agreement merge
// Per token: sums over the splits of beta and KL (plain sums: the agreement
// pass uses the final normalisers), the first maximum over the splits in
// vocabulary order, and the top-1 agreement.  Blocks of 32 tokens x 16 thread
// rows.
__global__ void __launch_bounds__(32 * kMergeRows) agree_merge_kernel(const float* __restrict__ partial,
                                                                      int n_splits, int M, int T,
                                                                      float* __restrict__ terms,
                                                                      int32_t* __restrict__ top1) {
  constexpr int S = kMaxExits - 1;
  __shared__ float sh_b[kMergeRows][S][32], sh_k[kMergeRows][S][32];
  __shared__ float sh_mx[kMergeRows][kMaxExits][32];
  __shared__ int sh_ix[kMergeRows][kMaxExits][32];
  const int lane = threadIdx.x, rowi = threadIdx.y;
  const int t = blockIdx.x * 32 + lane;
  const int QA = agree_rows(M);
  const int per = (n_splits + kMergeRows - 1) / kMergeRows;
  const int i0 = min(n_splits, rowi * per), i1 = min(n_splits, i0 + per);
  float b[S] = {0.f, 0.f, 0.f}, kl[S] = {0.f, 0.f, 0.f};
  float mx[kMaxExits] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
  int ix[kMaxExits] = {-1, -1, -1, -1};
  if (t < T) {
    // kB splits' partials are loaded before any is merged (independent loads in
    // flight); padding splits past i1 add zeros and never beat a maximum.
    constexpr int kB = 4;
    for (int i = i0; i < i1; i += kB) {
      float bv[kB][S], kv[kB][S], mv[kB][kMaxExits];
      int iv[kB][kMaxExits];
#pragma unroll
      for (int u = 0; u < kB; ++u) {
        const bool in = i + u < i1;
        const float* pi = partial + static_cast<int64_t>(in ? i + u : i0) * QA * T + t;
#pragma unroll
        for (int s = 0; s < S; ++s) {
          const bool ok = in && s < M - 1;
          bv[u][s] = ok ? pi[static_cast<int64_t>(s) * T] : 0.f;
          kv[u][s] = ok ? pi[static_cast<int64_t>(M - 1 + s) * T] : 0.f;
        }
#pragma unroll
        for (int m = 0; m < kMaxExits; ++m) {
          const bool ok = in && m < M;
          mv[u][m] = ok ? pi[static_cast<int64_t>(2 * (M - 1) + m) * T] : -INFINITY;
          iv[u][m] = ok ? __float_as_int(pi[static_cast<int64_t>(3 * M - 2 + m) * T]) : -1;
        }
      }
#pragma unroll
      for (int u = 0; u < kB; ++u) {
#pragma unroll
        for (int s = 0; s < S; ++s) if (s < M - 1) {
          b[s] += bv[u][s];
          kl[s] += kv[u][s];
        }
#pragma unroll
        for (int m = 0; m < kMaxExits; ++m) if (m < M) {
          if (mv[u][m] > mx[m]) { mx[m] = mv[u][m]; ix[m] = iv[u][m]; }
        }
      }
    }
  }
#pragma unroll
  for (int s = 0; s < S; ++s) { sh_b[rowi][s][lane] = b[s]; sh_k[rowi][s][lane] = kl[s]; }
#pragma unroll
  for (int m = 0; m < kMaxExits; ++m) { sh_mx[rowi][m][lane] = mx[m]; sh_ix[rowi][m][lane] = ix[m]; }
  __syncthreads();
  if (rowi != 0 || t >= T) return;
  for (int r = 1; r < kMergeRows; ++r) {
#pragma unroll
    for (int s = 0; s < S; ++s) if (s < M - 1) { b[s] += sh_b[r][s][lane]; kl[s] += sh_k[r][s][lane]; }
#pragma unroll
    for (int m = 0; m < kMaxExits; ++m) if (m < M)
      if (sh_mx[r][m][lane] > mx[m]) { mx[m] = sh_mx[r][m][lane]; ix[m] = sh_ix[r][m][lane]; }
  }
#pragma unroll
  for (int m = 0; m < kMaxExits; ++m) if (m < M) top1[static_cast<int64_t>(m) * T + t] = ix[m];
#pragma unroll
  for (int s = 0; s < S; ++s) if (s < M - 1) {
    terms[static_cast<int64_t>(s) * T + t] = b[s];
    terms[static_cast<int64_t>(M - 1 + s) * T + t] = kl[s];
    terms[static_cast<int64_t>(2 * (M - 1) + s) * T + t] = (ix[s] == ix[M - 1]) ? 1.f : 0.f;
  }
}

// ------------------------------------------------------------------ Jensen-Shannon merge
// Per token: plain sums over the splits (the pass used the final normalisers) of
// sum q log(q/mu) and sum p log(p/mu); writes K = KL(q || mu)/2 into the
// statistics row the backward pass reads and JS = (KL(q || mu) + KL(p || mu))/2
// as the distillation term.
__global__ void __launch_bounds__(32 * kMergeRows) js_merge_kernel(const float* __restrict__ partial, int n_splits,
                                                                   int M, int T, int V, int kind, int teacher_rows,
                                                                   const int32_t* __restrict__ y,
                                                                   float* __restrict__ stats,
                                                                   float* __restrict__ terms) {
  constexpr int S = kMaxExits - 1;
  __shared__ float sh_q[kMergeRows][S][32], sh_p[kMergeRows][S][32];
  const int lane = threadIdx.x, rowi = threadIdx.y;
  const int t = blockIdx.x * 32 + lane;
  const int QJ = js_rows(M);
  const int per = (n_splits + kMergeRows - 1) / kMergeRows;
  const int i0 = min(n_splits, rowi * per), i1 = min(n_splits, i0 + per);
  float jq[S] = {0.f, 0.f, 0.f}, jp[S] = {0.f, 0.f, 0.f};
  if (t < T) {
#pragma unroll 4
    for (int i = i0; i < i1; ++i) {
      const float* pi = partial + static_cast<int64_t>(i) * QJ * T + t;
#pragma unroll
      for (int s = 0; s < S; ++s) if (s < M - 1) {
        jq[s] += pi[static_cast<int64_t>(s) * T];
        jp[s] += pi[static_cast<int64_t>(M - 1 + s) * T];
      }
    }
  }
#pragma unroll
  for (int s = 0; s < S; ++s) { sh_q[rowi][s][lane] = jq[s]; sh_p[rowi][s][lane] = jp[s]; }
  __syncthreads();
  if (rowi != 0 || t >= T) return;
  for (int r = 1; r < kMergeRows; ++r)
#pragma unroll
    for (int s = 0; s < S; ++s) if (s < M - 1) { jq[s] += sh_q[r][s][lane]; jp[s] += sh_p[r][s][lane]; }
  const int yt = y[t];
  const bool bad = yt < 0 || yt >= V;
#pragma unroll
  for (int s = 0; s < S; ++s) if (s < M - 1) {
    if (kind == 3) {
      // acceptance: A into the statistics row, 1 - beta = 1 - (A + B) as the term, B for the teacher
      stats[static_cast<int64_t>(2 * M + s) * T + t] = jq[s];
      if (teacher_rows) stats[static_cast<int64_t>(3 * M - 1 + s) * T + t] = jp[s];
      terms[static_cast<int64_t>(M + s) * T + t] = bad ? 0.f : 1.f - (jq[s] + jp[s]);
    } else {
      stats[static_cast<int64_t>(2 * M + s) * T + t] = 0.5f * jq[s];
      // with the teacher gradient: KL(p || mu)/2 in rows 3M-1 .. 4M-3
      if (teacher_rows) stats[static_cast<int64_t>(3 * M - 1 + s) * T + t] = 0.5f * jp[s];
      terms[static_cast<int64_t>(M + s) * T + t] = bad ? 0.f : 0.5f * (jq[s] + jp[s]);
    }
  }
}

// ------------------------------------------------------------------ grouped GEMM kernel (dh, dW)
// For every problem p of a group (one per exit; all share M and K):
//   out_p[M x N_p] (+)= alpha * A_p[M x K] B_p[N_p x K]^T
// with bf16 operands in TMA boxes and fp32 accumulation in TMEM (two
// accumulator buffers so the epilogue of one tile overlaps the mainloop of the
// next).  One persistent launch walks the tiles of all problems, so the grid
// stays full across exits of different widths.
//   A_MN: A stored with M contiguous (boxes of 64 M x 64 K), else K contiguous
//   B_MN: B stored with N contiguous, else K contiguous
constexpr int kGemmStages = 4;

struct GemmMaps {
  CUtensorMap a[kMaxExits];
  CUtensorMap b[kMaxExits];
};

struct GemmArgs {
  int nprob;
  int Mdim, Kdim;
  int n_mt, kblocks, group_m;
  int tile_start[kMaxExits + 1];   // prefix of tiles per problem
  int Ndim[kMaxExits];
  int n_nt[kMaxExits];
  void* out[kMaxExits];
  float alpha[kMaxExits];          // output scale of each problem
  int accumulate;
  int32_t* status;
  // Optional exact one-hot term (bf16 output only): row r of problem p also gets
  //   - alpha * onehot_coef[p] * onehot_rows[p][onehot_idx[r], :]  when onehot_idx[r] in [0, onehot_limit)
  const int32_t* onehot_idx;
  const __nv_bfloat16* onehot_rows[kMaxExits];
  float onehot_coef[kMaxExits];
  int onehot_limit;
  // Optional fp32 partial sums (bf16 output only): out_p = alpha acc + addend_p (same layout as out_p)
  // before the one-hot term and the rounding; the earlier vocabulary chunks of dh.
  const float* addend[kMaxExits];
  int f16;                         // 1: A and B hold fp16 (else bf16)
  const float* bscale[kMaxExits];  // optional device factor on alpha: 1/s of a rescaled fp16 copy of B
};

template <int BN>
struct __align__(1024) GemmSmem {
  uint8_t a[kGemmStages][kBM * kBK * 2];
  uint8_t b[kGemmStages][BN * kBK * 2];
  uint64_t full[kGemmStages];
  uint64_t empty[kGemmStages];
  uint64_t tfull[2];
  uint64_t tempty[2];
  uint64_t drain;
  uint32_t tmem_base;
  int abort;
};

// tile index -> (problem, m tile, n tile); m tiles grouped for L2 reuse
__device__ __forceinline__ void gemm_tile(const GemmArgs& g, int i, int& p, int& mt, int& nt) {
  p = 0;
  while (p + 1 < g.nprob && i >= g.tile_start[p + 1]) ++p;
  const int r0 = i - g.tile_start[p];
  const int per_group = g.group_m * g.n_nt[p];
  const int gi = r0 / per_group;
  const int first = gi * g.group_m;
  const int gm = min(g.group_m, g.n_mt - first);
  const int r = r0 - gi * per_group;
  nt = r / gm;
  mt = first + r % gm;
}

template <bool A_MN, bool B_MN, int BN, bool OUT_BF16>
__global__ void __launch_bounds__(kThreads, 1) gemm_kernel(const __grid_constant__ GemmMaps maps,
                                                           const GemmArgs g) {
  extern __shared__ uint8_t smem_raw[];
  using Smem = GemmSmem<BN>;
  Smem& s = *reinterpret_cast<Smem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  volatile int* abort = &s.abort;
  constexpr uint32_t kTmemCols = (2 * BN <= 32) ? 32 : (2 * BN <= 64) ? 64 : (2 * BN <= 128) ? 128 : (2 * BN <= 256) ? 256 : 512;
  const int num_tiles = g.tile_start[g.nprob];

  if (threadIdx.x == 0) {
    for (int i = 0; i < kGemmStages; ++i) {
      mbar_init(&s.full[i], 1);
      mbar_init(&s.empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s.tfull[i], 1);
      mbar_init(&s.tempty[i], 4);
    }
    mbar_init(&s.drain, 1);
    s.abort = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    for (int p = 0; p < g.nprob; ++p) {
      tma_prefetch_desc(&maps.a[p]);
      tma_prefetch_desc(&maps.b[p]);
    }
  }
  if (warp == 1) {
    tmem_alloc(&s.tmem_base, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = s.tmem_base;

  if (warp == 0) {
    if (lane == 0) {
      uint32_t stage = 0, phase = 0, issued = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x) {
        int p, mt, nt;
        gemm_tile(g, tile, p, mt, nt);
        const CUtensorMap* ma = &maps.a[p];
        const CUtensorMap* mb = &maps.b[p];
        for (int kb = 0; kb < g.kblocks; ++kb) {
          if (!mbar_wait(&s.empty[stage], phase ^ 1, abort, g.status)) { ok = false; break; }
          mbar_arrive_expect_tx(&s.full[stage], (kBM + BN) * kBK * 2);
          if (A_MN) {
#pragma unroll
            for (int j = 0; j < kBM / 64; ++j)
              tma_load_2d(ma, &s.full[stage], s.a[stage] + j * (64 * kBK * 2), mt * kBM + j * 64, kb * kBK);
          } else {
            tma_load_2d(ma, &s.full[stage], s.a[stage], kb * kBK, mt * kBM);
          }
          if (B_MN) {
#pragma unroll
            for (int j = 0; j < BN / 64; ++j)
              tma_load_2d(mb, &s.full[stage], s.b[stage] + j * (64 * kBK * 2), nt * BN + j * 64, kb * kBK);
          } else {
            tma_load_2d(mb, &s.full[stage], s.b[stage], kb * kBK, nt * BN);
          }
          ++issued;
          if (++stage == kGemmStages) { stage = 0; phase ^= 1; }
        }
      }
      if (!ok) {
        const uint32_t n = issued < kGemmStages ? issued : kGemmStages;
        uint32_t st = stage, ph = phase;
        for (uint32_t i = 0; i < n; ++i) {
          if (st == 0) { st = kGemmStages - 1; ph ^= 1; } else { --st; }
          drain_wait(&s.full[st], ph, g.status);
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t idesc = g.f16 ? idesc_f16(kBM, BN, A_MN, B_MN) : idesc_bf16(kBM, BN, A_MN, B_MN);
      // K step of one tcgen05.mma: +32 B inside the swizzled row (K-major) or
      // +16 rows of 128 B (MN-major).
      constexpr uint32_t a_step = A_MN ? (kUK * 128) >> 4 : (kUK * 2) >> 4;
      constexpr uint32_t b_step = B_MN ? (kUK * 128) >> 4 : (kUK * 2) >> 4;
      constexpr uint32_t a_lbo = A_MN ? 64 * kBK * 2 : 16;
      constexpr uint32_t b_lbo = B_MN ? 64 * kBK * 2 : 16;
      uint32_t stage = 0, phase = 0, iter = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x, ++iter) {
        const uint32_t buf = iter & 1;
        if (!mbar_wait(&s.tempty[buf], ((iter >> 1) & 1) ^ 1, abort, g.status)) break;
        tc_fence_after();
        const uint32_t d = tmem + buf * BN;
        for (int kb = 0; kb < g.kblocks; ++kb) {
          if (!mbar_wait(&s.full[stage], phase, abort, g.status)) { ok = false; break; }
          tc_fence_after();
          const uint64_t da = smem_desc_sw128(smem_u32(s.a[stage]), a_lbo, 1024);
          const uint64_t db = smem_desc_sw128(smem_u32(s.b[stage]), b_lbo, 1024);
#pragma unroll
          for (int k = 0; k < kBK / kUK; ++k)
            umma_bf16(d, da + static_cast<uint64_t>(k * a_step), db + static_cast<uint64_t>(k * b_step), idesc,
                      (kb | k) != 0);
          umma_commit(&s.empty[stage]);
          if (++stage == kGemmStages) { stage = 0; phase ^= 1; }
        }
        if (ok) umma_commit(&s.tfull[buf]);
      }
      umma_commit(&s.drain);
      drain_wait(&s.drain, 0, g.status);
    }
  } else {
    const int q = warp & 3;
    const int row_in_tile = q * 32 + lane;
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(q * 32) << 16);
    uint32_t iter = 0;
    for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x, ++iter) {
      int p, mt, nt;
      gemm_tile(g, tile, p, mt, nt);
      const uint32_t buf = iter & 1;
      if (!warp_wait(&s.tfull[buf], (iter >> 1) & 1, abort, g.status)) break;
      tc_fence_after();
      const int64_t row = static_cast<int64_t>(mt) * kBM + row_in_tile;
      const bool valid = row < g.Mdim;
      const int Ndim = g.Ndim[p];
      const int64_t col0 = static_cast<int64_t>(nt) * BN;
      int64_t onehot_row = -1;
      if (OUT_BF16 && valid && g.onehot_idx != nullptr) {
        const int32_t k = __ldg(g.onehot_idx + row);
        if (k >= 0 && k < g.onehot_limit) onehot_row = k;
      }
      const float alpha = g.alpha[p] * (g.bscale[p] != nullptr ? *g.bscale[p] : 1.f);
      const float oh_scale = g.alpha[p] * g.onehot_coef[p];
#pragma unroll 1
      for (int c = 0; c < BN / 32; ++c) {
        float r[32];
        tmem_ld32(lane_base + buf * BN + c * 32, r);
        if (c == BN / 32 - 1) {
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&s.tempty[buf]);
        }
        if (!valid || col0 + c * 32 >= Ndim) continue;   // rows past M, columns past a ragged N
        const int64_t off = row * Ndim + col0 + c * 32;
        if (OUT_BF16) {
          uint4* dst = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(g.out[p]) + off);
          const uint4* oh = (onehot_row >= 0)
                                ? reinterpret_cast<const uint4*>(g.onehot_rows[p] + onehot_row * Ndim + col0 + c * 32)
                                : nullptr;
          const float4* ad = (g.addend[p] != nullptr) ? reinterpret_cast<const float4*>(g.addend[p] + off) : nullptr;
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            float f[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) f[e] = r[8 * u + e] * alpha;
            if (ad != nullptr) {
              const float4 a0 = ad[2 * u], a1 = ad[2 * u + 1];
              f[0] += a0.x; f[1] += a0.y; f[2] += a0.z; f[3] += a0.w;
              f[4] += a1.x; f[5] += a1.y; f[6] += a1.z; f[7] += a1.w;
            }
            if (oh != nullptr) {
              float w[8];
              bf16x8_to_f32(__ldg(oh + u), w);
#pragma unroll
              for (int e = 0; e < 8; ++e) f[e] = fmaf(-oh_scale, w[e], f[e]);
            }
            dst[u] = f32_to_bf16x8(f);
          }
        } else {
          float4* dst = reinterpret_cast<float4*>(static_cast<float*>(g.out[p]) + off);
#pragma unroll
          for (int u = 0; u < 8; ++u) {
            float4 v = make_float4(r[4 * u] * alpha, r[4 * u + 1] * alpha, r[4 * u + 2] * alpha,
                                   r[4 * u + 3] * alpha);
            if (g.accumulate) {
              const float4 o = dst[u];
              v.x += o.x; v.y += o.y; v.z += o.z; v.w += o.w;
            }
            dst[u] = v;
          }
        }
      }
    }
  }

  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// ------------------------------------------------------------------ grouped GEMM on CTA pairs
// Same problem as gemm_kernel with 256 x 256 output tiles computed by a pair
// of CTAs (a 2-CTA cluster) with tcgen05.mma.cta_group::2: each CTA loads its
// 128 rows of A and 128 of the 256 rows of B, so every CTA reads half of B per
// MMA and the B traffic through shared memory and L2 halves.  CTA rank 0 (the
// leader) issues the MMAs; each CTA's TMEM holds its 128 rows of the two
// accumulator buffers and its own epilogue drains them.
constexpr int kPairStages = 6;

struct __align__(1024) PairSmem {
  uint8_t a[kPairStages][kBM * kBK * 2];
  uint8_t b[kPairStages][128 * kBK * 2];
  uint64_t full[kPairStages];      // leader: counts both CTAs' TMA bytes
  uint64_t empty[kPairStages];     // each CTA: its stage may be refilled
  uint64_t tfull[2];               // each CTA: accumulator buffer ready
  uint64_t tempty[2];              // leader: both CTAs drained the buffer (8 warps)
  uint64_t drain;
  uint32_t tmem_base;
  int abort;
};

__device__ __forceinline__ void pair_tile(const GemmArgs& g, int i, int& p, int& mt, int& nt) {
  gemm_tile(g, i, p, mt, nt);        // mt indexes 256-row blocks (g.n_mt counts them)
}

template <bool A_MN, bool B_MN, bool OUT_BF16>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
    gemm_pair_kernel(const __grid_constant__ GemmMaps maps, const GemmArgs g) {
  constexpr int BN = 256;
  extern __shared__ uint8_t smem_raw[];
  PairSmem& s = *reinterpret_cast<PairSmem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  volatile int* abort = &s.abort;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  const int cluster = blockIdx.x >> 1, nclusters = gridDim.x >> 1;
  const int num_tiles = g.tile_start[g.nprob];

  if (threadIdx.x == 0) {
    for (int i = 0; i < kPairStages; ++i) {
      mbar_init(&s.full[i], 1);
      mbar_init(&s.empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s.tfull[i], 1);
      mbar_init(&s.tempty[i], 8);
    }
    mbar_init(&s.drain, 1);
    s.abort = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    for (int p = 0; p < g.nprob; ++p) {
      tma_prefetch_desc(&maps.a[p]);
      tma_prefetch_desc(&maps.b[p]);
    }
  }
  if (warp == 1) {
    tmem_alloc_pair(&s.tmem_base, 512);
    tmem_relinquish_pair();
  }
  __syncwarp();
  tc_fence_before();
  cluster_sync_all();        // every barrier of both CTAs exists before any remote arrive
  tc_fence_after();
  const uint32_t tmem = s.tmem_base;

  if (warp == 0) {
    if (lane == 0) {
      uint32_t stage = 0, phase = 0, issued = 0;
      bool ok = true;
      for (int tile = cluster; tile < num_tiles && ok; tile += nclusters) {
        int p, mt, nt;
        pair_tile(g, tile, p, mt, nt);
        const CUtensorMap* ma = &maps.a[p];
        const CUtensorMap* mb = &maps.b[p];
        const int row0 = mt * 2 * kBM + static_cast<int>(rank) * kBM;   // this CTA's 128 rows of A
        const int n0 = nt * BN + static_cast<int>(rank) * 128;           // this CTA's 128 rows of B
        for (int kb = 0; kb < g.kblocks; ++kb) {
          if (!mbar_wait(&s.empty[stage], phase ^ 1, abort, g.status)) { ok = false; break; }
          const uint32_t lfull = mapa_shared(smem_u32(&s.full[stage]), 0);
          if (leader) mbar_arrive_expect_tx(&s.full[stage], 2 * (kBM + 128) * kBK * 2);
          if (A_MN) {
#pragma unroll
            for (int j = 0; j < kBM / 64; ++j)
              tma_load_2d_pair(ma, lfull, s.a[stage] + j * (64 * kBK * 2), row0 + j * 64, kb * kBK);
          } else {
            tma_load_2d_pair(ma, lfull, s.a[stage], kb * kBK, row0);
          }
          if (B_MN) {
#pragma unroll
            for (int j = 0; j < 2; ++j)
              tma_load_2d_pair(mb, lfull, s.b[stage] + j * (64 * kBK * 2), n0 + j * 64, kb * kBK);
          } else {
            tma_load_2d_pair(mb, lfull, s.b[stage], kb * kBK, n0);
          }
          ++issued;
          if (++stage == kPairStages) { stage = 0; phase ^= 1; }
        }
      }
      if (!ok) {
        // The loads of this CTA complete on the leader's barrier; give them time to land.
        const uint64_t t0 = globaltimer_ns();
        while (globaltimer_ns() - t0 < 2000000ull) {
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0 && leader) {
      const uint32_t idesc = g.f16 ? idesc_f16(2 * kBM, BN, A_MN, B_MN) : idesc_bf16(2 * kBM, BN, A_MN, B_MN);
      constexpr uint32_t a_step = A_MN ? (kUK * 128) >> 4 : (kUK * 2) >> 4;
      constexpr uint32_t b_step = B_MN ? (kUK * 128) >> 4 : (kUK * 2) >> 4;
      constexpr uint32_t a_lbo = A_MN ? 64 * kBK * 2 : 16;
      constexpr uint32_t b_lbo = B_MN ? 64 * kBK * 2 : 16;
      uint32_t stage = 0, phase = 0, iter = 0;
      bool ok = true;
      for (int tile = cluster; tile < num_tiles && ok; tile += nclusters, ++iter) {
        const uint32_t buf = iter & 1;
        if (!mbar_wait(&s.tempty[buf], ((iter >> 1) & 1) ^ 1, abort, g.status)) break;
        tc_fence_after();
        const uint32_t d = tmem + buf * BN;
        for (int kb = 0; kb < g.kblocks; ++kb) {
          if (!mbar_wait(&s.full[stage], phase, abort, g.status)) { ok = false; break; }
          tc_fence_after();
          const uint64_t da = smem_desc_sw128(smem_u32(s.a[stage]), a_lbo, 1024);
          const uint64_t db = smem_desc_sw128(smem_u32(s.b[stage]), b_lbo, 1024);
#pragma unroll
          for (int k = 0; k < kBK / kUK; ++k)
            umma_bf16_pair(d, da + static_cast<uint64_t>(k * a_step), db + static_cast<uint64_t>(k * b_step), idesc,
                           (kb | k) != 0);
          const uint32_t e = smem_u32(&s.empty[stage]);
          umma_commit_pair(mapa_shared(e, 0));
          umma_commit_pair(mapa_shared(e, 1));
          if (++stage == kPairStages) { stage = 0; phase ^= 1; }
        }
        if (ok) {
          const uint32_t f = smem_u32(&s.tfull[buf]);
          umma_commit_pair(mapa_shared(f, 0));
          umma_commit_pair(mapa_shared(f, 1));
        }
      }
      umma_commit_pair(mapa_shared(smem_u32(&s.drain), 0));
      drain_wait(&s.drain, 0, g.status);
    }
  } else {
    const int q = warp & 3;
    const int row_in_tile = q * 32 + lane;
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(q * 32) << 16);
    uint32_t iter = 0;
    for (int tile = cluster; tile < num_tiles; tile += nclusters, ++iter) {
      int p, mt, nt;
      pair_tile(g, tile, p, mt, nt);
      const uint32_t buf = iter & 1;
      if (!warp_wait(&s.tfull[buf], (iter >> 1) & 1, abort, g.status)) break;
      tc_fence_after();
      const int64_t row = static_cast<int64_t>(mt) * 2 * kBM + rank * kBM + row_in_tile;
      const bool valid = row < g.Mdim;
      const int Ndim = g.Ndim[p];
      const int64_t col0 = static_cast<int64_t>(nt) * BN;
      int64_t onehot_row = -1;
      if (OUT_BF16 && valid && g.onehot_idx != nullptr) {
        const int32_t k = __ldg(g.onehot_idx + row);
        if (k >= 0 && k < g.onehot_limit) onehot_row = k;
      }
      const float alpha = g.alpha[p] * (g.bscale[p] != nullptr ? *g.bscale[p] : 1.f);
      const float oh_scale = g.alpha[p] * g.onehot_coef[p];
#pragma unroll 1
      for (int c = 0; c < BN / 32; ++c) {
        float r[32];
        tmem_ld32(lane_base + buf * BN + c * 32, r);
        if (c == BN / 32 - 1) {
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive_cluster(mapa_shared(smem_u32(&s.tempty[buf]), 0));
        }
        if (!valid || col0 + c * 32 >= Ndim) continue;
        const int64_t off = row * Ndim + col0 + c * 32;
        if (OUT_BF16) {
          uint4* dst = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(g.out[p]) + off);
          const uint4* oh = (onehot_row >= 0)
                                ? reinterpret_cast<const uint4*>(g.onehot_rows[p] + onehot_row * Ndim + col0 + c * 32)
                                : nullptr;
          const float4* ad = (g.addend[p] != nullptr) ? reinterpret_cast<const float4*>(g.addend[p] + off) : nullptr;
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            float f[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) f[e] = r[8 * u + e] * alpha;
            if (ad != nullptr) {
              const float4 a0 = ad[2 * u], a1 = ad[2 * u + 1];
              f[0] += a0.x; f[1] += a0.y; f[2] += a0.z; f[3] += a0.w;
              f[4] += a1.x; f[5] += a1.y; f[6] += a1.z; f[7] += a1.w;
            }
            if (oh != nullptr) {
              float w[8];
              bf16x8_to_f32(__ldg(oh + u), w);
#pragma unroll
              for (int e = 0; e < 8; ++e) f[e] = fmaf(-oh_scale, w[e], f[e]);
            }
            dst[u] = f32_to_bf16x8(f);
          }
        } else {
          float4* dst = reinterpret_cast<float4*>(static_cast<float*>(g.out[p]) + off);
#pragma unroll
          for (int u = 0; u < 8; ++u) {
            float4 v = make_float4(r[4 * u] * alpha, r[4 * u + 1] * alpha, r[4 * u + 2] * alpha,
                                   r[4 * u + 3] * alpha);
            if (g.accumulate) {
              const float4 o = dst[u];
              v.x += o.x; v.y += o.y; v.z += o.z; v.w += o.w;
            }
            dst[u] = v;
          }
        }
      }
    }
  }

  __syncthreads();
  tc_fence_before();
  cluster_sync_all();        // no CTA leaves while its pair may still touch its memory
  tc_fence_after();
  if (warp == 1) {
    __syncwarp();
    tmem_dealloc_pair(tmem, 512);
  }
}

// ------------------------------------------------------------------ fp16 operand copies
// tcgen05.mma kind::f16 takes A and B in the same format, so the backward
// GEMMs, whose A is the fp16 G', read fp16 copies of the chunk's rows of W and
// the block's rows of h.  The copy is unscaled when the tensor's largest
// magnitude m lies in [2^-10, 2^15): every bf16 value there converts exactly
// (bf16's 8 significant bits fit in fp16's 11), and the few values below
// fp16's normal range keep an absolute error under 3e-8.  Otherwise a second
// pass copies x * s with s a power of two that puts m in [2^13, 2^14), and the
// GEMM epilogue multiplies by 1/s; powers of two change no significand.
struct HalfJob {
  const uint4* src;          // bf16, 8 per vector
  uint4* dst;                // fp16, 8 per vector
  int64_t n_vec;
  unsigned int* maxbits;     // largest |x| as float bits (non-negative floats order as unsigned ints)
  float* inv_scale;          // 1/s, for the GEMM epilogue
};
struct HalfJobs {
  HalfJob j[kMaxExits];
};

__device__ __forceinline__ uint4 bf16x8_to_half8(const uint4& u, float s, float& mx) {
  float f[8];
  bf16x8_to_f32(u, f);
  uint32_t w[4];
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    mx = fmaxf(mx, fmaxf(fabsf(f[2 * k]), fabsf(f[2 * k + 1])));
    __half2 h = __floats2half2_rn(f[2 * k] * s, f[2 * k + 1] * s);   // beyond the range: infinite, as in the input
    w[k] = *reinterpret_cast<uint32_t*>(&h);
  }
  return make_uint4(w[0], w[1], w[2], w[3]);
}

// First pass: the unscaled copy and the largest magnitude (job = blockIdx.y).
__global__ void __launch_bounds__(256) half_copy_kernel(const __grid_constant__ HalfJobs jobs) {
  const HalfJob& jb = jobs.j[blockIdx.y];
  float mx = 0.f;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  for (; i + 3 * stride < jb.n_vec; i += 4 * stride) {
    uint4 u[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) u[k] = __ldg(jb.src + i + k * stride);
#pragma unroll
    for (int k = 0; k < 4; ++k) jb.dst[i + k * stride] = bf16x8_to_half8(u[k], 1.f, mx);
  }
  for (; i < jb.n_vec; i += stride) jb.dst[i] = bf16x8_to_half8(__ldg(jb.src + i), 1.f, mx);
  mx = warp_max(mx);
  if ((threadIdx.x & 31) == 0 && mx > 0.f) atomicMax(jb.maxbits, __float_as_uint(mx));
}

// Second pass: the scale from the largest magnitude, and the scaled copy when
// the unscaled one does not serve.
__global__ void __launch_bounds__(256) half_rescale_kernel(const __grid_constant__ HalfJobs jobs) {
  const HalfJob& jb = jobs.j[blockIdx.y];
  const float mx = __uint_as_float(*jb.maxbits);
  float s = 1.f;
  if (mx <= 3.4e38f && (mx >= 32768.f || (mx > 0.f && mx < 1.f / 1024.f))) {
    int e = 13 - ilogbf(mx);
    e = e < -126 ? -126 : (e > 126 ? 126 : e);
    s = ldexpf(1.f, e);
  }
  if (blockIdx.x == 0 && threadIdx.x == 0) *jb.inv_scale = 1.f / s;
  if (s == 1.f) return;
  float unused = 0.f;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < jb.n_vec; i += stride)
    jb.dst[i] = bf16x8_to_half8(__ldg(jb.src + i), s, unused);
}

// ------------------------------------------------------------------ host side
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn get_encoder() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// 2-D tensor of 16-bit elements [outer][inner] (inner contiguous; bf16 unless
// fp16 is set), 128-byte swizzled boxes.
bool make_map(CUtensorMap* map, const void* base, uint64_t inner, uint64_t outer, uint32_t box_inner,
              uint32_t box_outer, bool fp16 = false) {
  EncodeTiledFn enc = get_encoder();
  if (enc == nullptr) return false;
  const cuuint64_t dims[2] = {inner, outer};
  const cuuint64_t strides[1] = {inner * 2};
  const cuuint32_t box[2] = {box_inner, box_outer};
  const cuuint32_t estr[2] = {1, 1};
  return enc(map, fp16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
             const_cast<void*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int num_sms() {
  int dev = 0, n = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  return n;
}

// Pairs of CTAs (2-CTA clusters) that can be resident at once for kernel fn with
// this block size and shared memory: a persistent grid larger than that would
// leave whole clusters waiting for a second wave.  Falls back to SMs / 2.
template <typename Kernel>
int resident_pairs(Kernel fn, int threads, size_t smem) {
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(static_cast<unsigned>(num_sms()));
  cfg.blockDim = dim3(static_cast<unsigned>(threads));
  cfg.dynamicSmemBytes = smem;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, fn, &cfg) != cudaSuccess || n <= 0) {
    (void)cudaGetLastError();
    n = num_sms() / 2;
  }
  return n;
}

size_t align_up(size_t b) { return (b + 255) & ~size_t(255); }

// ------------------------------------------------------------------ backward chunk plan
// The backward pass writes the dense logit gradient G' (fp16) of every exit
// for one block of tokens x one chunk of the vocabulary at a time into the
// workspace, then consumes it with the two GEMMs.  dW rows of a chunk are
// complete after their chunk (K runs over the block's tokens; token blocks
// after the first add into dW), dh rows of a block after the block's last
// chunk (K runs over the chunk's columns; the chunks before the last leave
// fp32 partial sums in the workspace).  Workspace: [G' chunk: M x Tb x Vc f16]
// [dh partials: Tb x sum(D) f32, only with more than one chunk][targets
// grouped by id][fp16 copy of the block's h rows: Tb x sum(D)][fp16 copy of
// the chunk's W rows: Vc x sum(D)][copy scales].
struct BwdPlan {
  int64_t Tb, Vc;          // tokens per block (last block shorter), columns per chunk (last chunk shorter)
  int64_t nT, nV;
  size_t g_bytes, acc_bytes, seg_bytes, h16_bytes, w16_bytes, aux_bytes;
  size_t total() const { return g_bytes + acc_bytes + seg_bytes + h16_bytes + w16_bytes + aux_bytes; }
};

// The workspace the query returns is the plan for this budget.  At the 3-exit
// main suite (T = 8192) it holds three vocabulary chunks of 16384 in one token
// block; 1 GiB would need five, whose extra dh partials (0.5 GB of fp32
// read-modify-write per extra chunk) measured 0.5 ms per step slower.
constexpr size_t kDefaultBwdBudget = size_t(3) << 29;   // 1.5 GiB

int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }
int64_t round_up(int64_t a, int64_t b) { return ceil_div(a, b) * b; }

int64_t sum_d(const LossProblem& p) {
  int64_t s = 0;
  for (int m = 0; m < p.M; ++m) s += p.D[m];
  return s;
}

BwdPlan plan_shape(const LossProblem& p, int64_t Tb, int64_t Vc) {
  BwdPlan b{};
  b.Tb = Tb;
  b.Vc = Vc;
  b.nT = ceil_div(p.T, Tb);
  b.nV = ceil_div(p.V, Vc);
  const size_t sd = static_cast<size_t>(sum_d(p));
  b.g_bytes = align_up(static_cast<size_t>(p.M) * Tb * Vc * 2);
  b.acc_bytes = b.nV > 1 ? align_up(static_cast<size_t>(Tb) * sd * sizeof(float)) : 0;
  b.seg_bytes = align_up(segindex_bytes(p.T, p.V));
  b.h16_bytes = align_up(static_cast<size_t>(Tb) * sd * 2);
  b.w16_bytes = align_up(static_cast<size_t>(Vc) * sd * 2);
  b.aux_bytes = 256;
  return b;
}

// Bytes the plan moves beyond one pass over G': the dW read-modify-write of
// every token block after the first, the dh partials of every chunk but the
// last, the fp16 copies of W (once per block) and h, and a fixed charge per
// (block, chunk) for its launches' ramps.
double plan_cost(const LossProblem& p, const BwdPlan& b) {
  const double sd = static_cast<double>(sum_d(p));
  const double dw_rmw = static_cast<double>(b.nT - 1) * 8.0 * static_cast<double>(p.V) * sd;
  const double dh_part = static_cast<double>(b.nT) * static_cast<double>(b.nV - 1) * 8.0 * static_cast<double>(b.Tb) * sd;
  const double copies = 4.0 * sd * (static_cast<double>(b.nT) * static_cast<double>(p.V) + static_cast<double>(p.T));
  return dw_rmw + dh_part + copies + 3.0e8 * static_cast<double>(b.nT * b.nV);
}

// The cheapest plan whose workspace fits in `budget` bytes (Tb = 0 when none fits).
BwdPlan choose_plan(const LossProblem& p, size_t budget) {
  BwdPlan best{};
  double best_cost = 0.0;
  for (int64_t nT = 1;; ++nT) {
    const int64_t Tb = nT == 1 ? p.T : round_up(ceil_div(p.T, nT), kBM);
    if (nT > 1 && Tb >= round_up(ceil_div(p.T, nT - 1), kBM)) {   // same block size as fewer blocks
      if (Tb <= kBM) break;
      continue;
    }
    BwdPlan b = plan_shape(p, Tb, p.V);
    if (b.total() > budget) {
      const BwdPlan probe = plan_shape(p, Tb, kLossBN);   // smallest chunk: does any chunk width fit?
      if (probe.total() > budget) {
        if (Tb <= kBM) break;
        continue;
      }
      // widest chunk (a multiple of the tile width) that fits, then equal chunks of at most that width
      const size_t fixed = probe.acc_bytes + probe.seg_bytes + probe.h16_bytes + probe.aux_bytes;
      const size_t per_col = static_cast<size_t>(p.M) * Tb * 2 + static_cast<size_t>(sum_d(p)) * 2;
      int64_t vmax = static_cast<int64_t>((budget - fixed) / per_col) / kLossBN * kLossBN;
      while (vmax > kLossBN && plan_shape(p, Tb, vmax).total() > budget) vmax -= kLossBN;
      if (vmax < kLossBN) vmax = kLossBN;
      const int64_t nV = ceil_div(p.V, vmax);
      b = plan_shape(p, Tb, round_up(ceil_div(p.V, nV), kLossBN));
    }
    const double c = plan_cost(p, b);
    if (best.Tb == 0 || c < best_cost) {
      best = b;
      best_cost = c;
    }
    if (Tb <= kBM) break;
  }
  return best;
}

struct TcWs {
  float* partial;
  float* terms;
};

int loss_n_vt(const LossProblem& p) { return static_cast<int>((p.V + kLossBN - 1) / kLossBN); }

TcWs fwd_layout(const LossProblem& p, void* ws) {
  const size_t part = static_cast<size_t>(2 * loss_n_vt(p)) * (2 * p.M - 1) * p.T * sizeof(float);
  TcWs w;
  w.partial = static_cast<float*>(ws);
  w.terms = reinterpret_cast<float*>(static_cast<char*>(ws) + align_up(part));
  return w;
}

template <int MODE, int DISTILL, bool TGRAD = false>
cudaError_t run_loss_tiles(const LossProblem& p, const LossArgs& a, cudaStream_t st) {
  LossMaps maps;
  for (int m = 0; m < p.M; ++m) {
    if (!make_map(&maps.h[m], p.h[m], p.D[m], p.T, kBK, kBM)) return cudaErrorInvalidValue;
    if (!make_map(&maps.w[m], p.W[m], p.D[m], p.V, kBK, kLossBN)) return cudaErrorInvalidValue;
  }
  const size_t smem = sizeof(LossSmem) + 1024;
  auto fn = loss_tile_kernel<MODE, DISTILL, TGRAD>;
  cudaError_t err = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (err != cudaSuccess) return err;
  const int grid = a.num_tiles < num_sms() ? a.num_tiles : num_sms();
  fn<<<grid, kLossThreads, smem, st>>>(maps, a);
  note_launches(1);
  return cudaGetLastError();
}

LossArgs base_args(const LossProblem& p) {
  LossArgs a{};
  a.M = p.M;
  a.T = static_cast<int>(p.T);
  a.V = static_cast<int>(p.V);
  a.v0 = 0;
  a.Vtot = static_cast<int>(p.V);
  a.ldS = static_cast<int>(p.T);
  for (int m = 0; m < p.M; ++m) a.kblocks[m] = static_cast<int>(p.D[m] / kBK);
  a.n_tt = static_cast<int>((p.T + kBM - 1) / kBM);
  a.n_vt = loss_n_vt(p);
  a.num_tiles = a.n_tt * a.n_vt;
  a.group_tt = MLS_LOSS_GROUP_TT;
  a.y = p.y;
  a.alpha = p.alpha_d;
  a.distill = p.distill;
  for (int m = 0; m < p.M; ++m) a.exit_w[m] = p.exit_w[m];
  a.student_wsum = 0.f;
  for (int m = 0; m + 1 < p.M; ++m) a.student_wsum += p.exit_w[m];
  a.status = p.status;
  a.wait_ns = p.wait_ns != 0 ? p.wait_ns : kWaitLimitNs;
  a.withhold_loads = p.withhold_loads;
  return a;
}

template <bool A_MN, bool B_MN, int BN, bool OUT_BF16>
cudaError_t run_gemm(const GemmMaps& maps, GemmArgs g, int group_rows, cudaStream_t st) {
  // 256-wide N tiles run on CTA pairs (256 x 256 output tiles), narrower ones on single CTAs.
  constexpr bool kPair = (BN == 256);
  const int rows_per_tile = kPair ? 2 * kBM : kBM;
  g.n_mt = (g.Mdim + rows_per_tile - 1) / rows_per_tile;
  g.kblocks = (g.Kdim + kBK - 1) / kBK;
  g.group_m = kPair ? group_rows : 2 * group_rows;
  g.tile_start[0] = 0;
  for (int p = 0; p < g.nprob; ++p) {
    g.n_nt[p] = (g.Ndim[p] + BN - 1) / BN;     // the last N tile may be ragged (zero-filled by TMA)
    g.tile_start[p + 1] = g.tile_start[p] + g.n_mt * g.n_nt[p];
  }
  const int tiles = g.tile_start[g.nprob];
  cudaError_t err;
  if (kPair) {
    const size_t smem = sizeof(PairSmem) + 1024;
    auto fn = gemm_pair_kernel<A_MN, B_MN, OUT_BF16>;
    err = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (err != cudaSuccess) return err;
    const int resident = resident_pairs(fn, kThreads, smem);
    const int pairs = tiles < resident ? tiles : resident;
    fn<<<2 * pairs, kThreads, smem, st>>>(maps, g);
  } else {
    const size_t smem = sizeof(GemmSmem<BN>) + 1024;
    auto fn = gemm_kernel<A_MN, B_MN, BN, OUT_BF16>;
    err = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (err != cudaSuccess) return err;
    const int grid = tiles < num_sms() ? tiles : num_sms();
    fn<<<grid, kThreads, smem, st>>>(maps, g);
  }
  note_launches(1);
  return cudaGetLastError();
}

// N tile of the grouped GEMMs: 256 unless every exit is narrower (widths are
// multiples of 64; a ragged last tile is zero-filled and not stored).
int pick_bn(const LossProblem& p) {
  int64_t dmax = 0;
  for (int m = 0; m < p.M; ++m) dmax = p.D[m] > dmax ? p.D[m] : dmax;
  return dmax >= 256 ? 256 : dmax >= 128 ? 128 : 64;
}

// One (token block, vocabulary chunk) of the backward pass: its tokens [t0, t0 + Tb)
// and columns [v0, v0 + Vc), with G' = [M][Tb][Vc] fp16 and the fp16 copies of
// the chunk's W rows ([Vc][D_m] per exit, exits one after another) and of the
// block's h rows ([Tb][D_m] per exit).
struct BwdChunk {
  int64_t t0, Tb, v0, Vc;
  bool first_v, last_v;    // first / last chunk of the block
  bool first_t;            // first block
  const __half* G;
  float* acc;              // dh partial sums [Tb][sum D] (NULL with a single chunk)
  const __half* w16;
  const float* w16_inv;    // [M]: 1/s of each exit's copy
  const __half* h16;
  const float* h16_inv;    // [M]
};

// dh_m[Tb x D_m] (+)= a G'_m[Tb x Vc] W^m[v0 : v0 + Vc] for every exit in one launch:
// A = G'_m (K = Vc contiguous), B = the fp16 copy of the chunk's rows of W^m
// (N = D_m contiguous).  The last chunk of a block adds the earlier chunks'
// fp32 partials, subtracts the one-hot row a c_m W^m[y_t] exactly (from the
// bf16 W) and writes bf16 dh; the others write (first) or add to (later) the
// fp32 partials.
template <int BN>
cudaError_t run_dh_chunk(const LossProblem& p, const BwdChunk& c, void* const* dh, float alpha, cudaStream_t st) {
  GemmMaps maps;
  GemmArgs g{};
  g.nprob = p.M;
  g.Mdim = static_cast<int>(c.Tb);
  g.Kdim = static_cast<int>(c.Vc);
  g.f16 = 1;
  for (int m = 0; m < p.M; ++m) g.alpha[m] = alpha * p.exit_w[m];
  const bool tgrad = p.teacher_grad != 0 && p.M > 1;
  if (tgrad) g.alpha[p.M - 1] = alpha;             // the teacher's G' already carries w_T
  g.status = p.status;
  g.onehot_idx = p.y + c.t0;
  g.onehot_limit = static_cast<int>(p.V);
  g.accumulate = c.first_v ? 0 : 1;
  int64_t acc_off = 0, w_off = 0;
  for (int m = 0; m < p.M; ++m) {
    const __half* Gm = c.G + static_cast<int64_t>(m) * c.Tb * c.Vc;
    if (!make_map(&maps.a[m], Gm, c.Vc, c.Tb, kBK, kBM, true)) return cudaErrorInvalidValue;
    if (!make_map(&maps.b[m], c.w16 + w_off, p.D[m], c.Vc, 64, kBK, true)) return cudaErrorInvalidValue;
    w_off += c.Vc * p.D[m];
    g.bscale[m] = c.w16_inv + m;
    g.Ndim[m] = static_cast<int>(p.D[m]);
    float* acc_m = c.acc != nullptr ? c.acc + acc_off : nullptr;
    acc_off += c.Tb * p.D[m];
    if (c.last_v) {
      g.out[m] = static_cast<__nv_bfloat16*>(dh[m]) + c.t0 * p.D[m];
      g.onehot_rows[m] = static_cast<const __nv_bfloat16*>(p.W[m]);
      g.onehot_coef[m] = (m == p.M - 1) ? (tgrad ? p.exit_w[m] : 1.f) : 1.f - p.alpha_d;
      g.addend[m] = c.first_v ? nullptr : acc_m;
    } else {
      g.out[m] = acc_m;
    }
  }
  if (c.last_v) return run_gemm<false, true, BN, true>(maps, g, MLS_DH_GROUP_M, st);
  return run_gemm<false, true, BN, false>(maps, g, MLS_DH_GROUP_M, st);
}

// dW^m[v0 : v0 + Vc] (+)= a G'_m^T h_m[t0 : t0 + Tb] for every exit in one launch:
// A = G'^T (M = Vc contiguous), B = the fp16 copy of the block's rows of h_m
// (N = D_m contiguous), K = Tb.  Blocks after the first (and every block with
// accumulate) add.
template <int BN>
cudaError_t run_dw_chunk(const LossProblem& p, const BwdChunk& c, float* const* dW, float alpha, int accumulate,
                         cudaStream_t st) {
  GemmMaps maps;
  GemmArgs g{};
  g.nprob = p.M;
  g.Mdim = static_cast<int>(c.Vc);
  g.Kdim = static_cast<int>(c.Tb);
  g.f16 = 1;
  for (int m = 0; m < p.M; ++m) g.alpha[m] = alpha * p.exit_w[m];
  if (p.teacher_grad != 0 && p.M > 1) g.alpha[p.M - 1] = alpha;   // the teacher's G' already carries w_T
  g.accumulate = (accumulate || !c.first_t) ? 1 : 0;
  g.status = p.status;
  int64_t h_off = 0;
  for (int m = 0; m < p.M; ++m) {
    const __half* Gm = c.G + static_cast<int64_t>(m) * c.Tb * c.Vc;
    if (!make_map(&maps.a[m], Gm, c.Vc, c.Tb, 64, kBK, true)) return cudaErrorInvalidValue;
    if (!make_map(&maps.b[m], c.h16 + h_off, p.D[m], c.Tb, 64, kBK, true)) return cudaErrorInvalidValue;
    h_off += c.Tb * p.D[m];
    g.bscale[m] = c.h16_inv + m;
    g.Ndim[m] = static_cast<int>(p.D[m]);
    g.out[m] = dW[m] + c.v0 * p.D[m];
  }
  return run_gemm<true, true, BN, false>(maps, g, MLS_DW_GROUP_M, st);
}

// G' of one (token block, vocabulary chunk): the tile kernel on the block's
// rows of h, y and stats and the chunk's rows of W.
cudaError_t run_grad_chunk(const LossProblem& p, const BwdChunk& c, const float* stats, cudaStream_t st) {
  LossProblem q = p;
  q.T = c.Tb;
  q.V = c.Vc;
  q.y = p.y + c.t0;
  for (int m = 0; m < p.M; ++m) {
    q.h[m] = static_cast<const __nv_bfloat16*>(p.h[m]) + c.t0 * p.D[m];
    q.W[m] = static_cast<const __nv_bfloat16*>(p.W[m]) + c.v0 * p.D[m];
  }
  LossArgs a = base_args(q);
  a.v0 = static_cast<int>(c.v0);
  a.Vtot = static_cast<int>(p.V);
  a.ldS = static_cast<int>(p.T);
  a.stats = const_cast<float*>(stats) + c.t0;
  a.G = const_cast<__half*>(c.G);
  const bool tgrad = p.teacher_grad != 0 && p.M > 1;
  return tgrad ? (p.distill == 1   ? run_loss_tiles<kModeGrad, 1, true>(q, a, st)
                  : p.distill == 2 ? run_loss_tiles<kModeGrad, 2, true>(q, a, st)
                  : p.distill == 3 ? run_loss_tiles<kModeGrad, 3, true>(q, a, st)
                                   : run_loss_tiles<kModeGrad, 0, true>(q, a, st))
         : p.distill == 1 ? run_loss_tiles<kModeGrad, 1>(q, a, st)
         : p.distill == 2 ? run_loss_tiles<kModeGrad, 2>(q, a, st)
         : p.distill == 3 ? run_loss_tiles<kModeGrad, 3>(q, a, st)
                          : run_loss_tiles<kModeGrad, 0>(q, a, st);
}

// fp16 copies of rows [r0, r0 + n) of every exit's bf16 matrix src[m] ([*][D_m])
// into dst (exits one after another), with their scales in inv[0 .. M).
cudaError_t run_half_copies(const LossProblem& p, const void* const* src, int64_t r0, int64_t n, __half* dst,
                            unsigned int* maxbits, float* inv, cudaStream_t st) {
  cudaError_t err = cudaMemsetAsync(maxbits, 0, sizeof(unsigned int) * p.M, st);
  if (err != cudaSuccess) return err;
  HalfJobs jobs{};
  int64_t off = 0, most = 0;
  for (int m = 0; m < p.M; ++m) {
    const int64_t nv = n * p.D[m] / 8;
    jobs.j[m] = HalfJob{reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(src[m]) + r0 * p.D[m]),
                        reinterpret_cast<uint4*>(dst + off), nv, maxbits + m, inv + m};
    off += n * p.D[m];
    most = nv > most ? nv : most;
  }
  const int64_t want = ceil_div(most, 256 * 4);
  const int64_t cap = 2 * static_cast<int64_t>(num_sms());
  const dim3 grid(static_cast<unsigned>(want < 1 ? 1 : (want < cap ? want : cap)), static_cast<unsigned>(p.M));
  half_copy_kernel<<<grid, 256, 0, st>>>(jobs);
  half_rescale_kernel<<<grid, 256, 0, st>>>(jobs);
  note_launches(2);
  return cudaGetLastError();
}

}  // namespace

bool tensor_map_encoder_available() { return get_encoder() != nullptr; }

size_t loss_tc_fwd_bytes(const LossProblem& p) {
  const size_t part = static_cast<size_t>(2 * loss_n_vt(p)) * (2 * p.M - 1) * p.T * sizeof(float);
  const size_t terms = static_cast<size_t>(2 * p.M - 1) * p.T * sizeof(float);
  return align_up(part) + align_up(terms);
}

size_t agree_tc_bytes(const LossProblem& p) {
  const size_t part = static_cast<size_t>(2 * loss_n_vt(p)) * agree_rows(p.M) * p.T * sizeof(float);
  const size_t terms = static_cast<size_t>(3 * (p.M - 1)) * p.T * sizeof(float);
  const size_t top1 = static_cast<size_t>(p.M) * p.T * sizeof(int32_t);
  return align_up(part) + align_up(terms) + align_up(top1);
}

cudaError_t agree_tc(const LossProblem& p, const float* stats, float* metrics, float* per_token, int32_t* top1,
                     void* ws, cudaStream_t st) {
  const size_t part = static_cast<size_t>(2 * loss_n_vt(p)) * agree_rows(p.M) * p.T * sizeof(float);
  const size_t terms_b = static_cast<size_t>(3 * (p.M - 1)) * p.T * sizeof(float);
  char* base = static_cast<char*>(ws);
  float* partial = reinterpret_cast<float*>(base);
  float* terms = per_token != nullptr ? per_token : reinterpret_cast<float*>(base + align_up(part));
  int32_t* top = top1 != nullptr ? top1 : reinterpret_cast<int32_t*>(base + align_up(part) + align_up(terms_b));
  LossArgs a = base_args(p);
  a.partial = partial;
  a.stats = const_cast<float*>(stats);
  cudaError_t err = run_loss_tiles<kModeAgree, 0>(p, a, st);
  if (err != cudaSuccess) return err;
  const int T = static_cast<int>(p.T);
  agree_merge_kernel<<<(T + 31) / 32, dim3(32, kMergeRows), 0, st>>>(partial, 2 * a.n_vt, p.M, T, terms, top);
  note_launches(1);
  err = cudaGetLastError();
  if (err != cudaSuccess) return err;
  return launch_row_means(terms, 3 * (p.M - 1), p.T, metrics, st);
}

size_t loss_tc_bwd_bytes(const LossProblem& p) {
  const BwdPlan whole = plan_shape(p, p.T, p.V);
  return whole.total() <= kDefaultBwdBudget ? whole.total() : choose_plan(p, kDefaultBwdBudget).total();
}

size_t loss_tc_bwd_min_bytes(const LossProblem& p) {
  // one tile of tokens per block: either the whole vocabulary at once (no dh
  // partials) or one tile of columns per chunk, whichever is smaller
  const int64_t Tb = p.T < kBM ? p.T : kBM;
  const size_t whole_v = plan_shape(p, Tb, p.V).total();
  const size_t one_tile = plan_shape(p, Tb, p.V < kLossBN ? p.V : kLossBN).total();
  return whole_v < one_tile ? whole_v : one_tile;
}

void loss_tc_bwd_plan(const LossProblem& p, size_t ws_bytes, int64_t* Tb, int64_t* Vc) {
  const BwdPlan b = choose_plan(p, ws_bytes);
  *Tb = b.Tb;
  *Vc = b.Vc;
}

cudaError_t loss_tc_fwd(const LossProblem& p, float* losses, float* stats, void* ws, cudaStream_t st) {
  const TcWs w = fwd_layout(p, ws);
  LossArgs a = base_args(p);
  a.partial = w.partial;
  a.stats = stats;
  // the Jensen-Shannon form starts from the cross-entropy statistics
  cudaError_t err = p.distill == 1 ? run_loss_tiles<kModeStats, 1>(p, a, st) : run_loss_tiles<kModeStats, 0>(p, a, st);
  if (err != cudaSuccess) return err;
  const int T = static_cast<int>(p.T);
  loss_merge_kernel<<<(T + 31) / 32, dim3(32, kLossMergeRows), 0, st>>>(w.partial, 2 * a.n_vt, p.M, T,
                                                                     static_cast<int>(p.V), p.distill, p.y, stats,
                                                                     w.terms, p.status);
  note_launches(1);
  err = cudaGetLastError();
  if (err != cudaSuccess) return err;
  if ((p.distill == 2 || p.distill == 3) && p.M > 1) {
    // Jensen-Shannon or acceptance: a second pass over the logits with the final
    // normalisers (its partials, 2(M-1) rows per split, reuse the statistics partial buffer).
    err = p.distill == 3 ? run_loss_tiles<kModeJS, 3>(p, a, st) : run_loss_tiles<kModeJS, 2>(p, a, st);
    if (err != cudaSuccess) return err;
    js_merge_kernel<<<(T + 31) / 32, dim3(32, kMergeRows), 0, st>>>(w.partial, 2 * a.n_vt, p.M, T,
                                                                     static_cast<int>(p.V), p.distill,
                                                                     p.teacher_grad, p.y, stats, w.terms);
    note_launches(1);
    err = cudaGetLastError();
    if (err != cudaSuccess) return err;
  }
  return launch_loss_reduce(w.terms, p, losses, st);
}

cudaError_t loss_tc_bwd(const LossProblem& p, const float* stats, float grad_scale, void* const* dh,
                        float* const* dW, int accumulate, void* ws, size_t ws_bytes, cudaStream_t st) {
  const BwdPlan plan = choose_plan(p, ws_bytes);
  if (plan.Tb == 0) return cudaErrorInvalidValue;       // the caller checked the minimum size
  char* base = static_cast<char*>(ws);
  __half* G = reinterpret_cast<__half*>(base);
  char* q = base + plan.g_bytes;
  float* acc = plan.acc_bytes ? reinterpret_cast<float*>(q) : nullptr;
  q += plan.acc_bytes;
  void* seg_ws = q;
  q += plan.seg_bytes;
  __half* h16 = reinterpret_cast<__half*>(q);
  q += plan.h16_bytes;
  __half* w16 = reinterpret_cast<__half*>(q);
  q += plan.w16_bytes;
  unsigned int* maxbits = reinterpret_cast<unsigned int*>(q);     // [0, M) W, [M, 2M) h
  float* inv = reinterpret_cast<float*>(q + 2 * kMaxExits * sizeof(unsigned int));
  const float alpha = grad_scale / static_cast<float>(p.T);
  const int bn = pick_bn(p);
  cudaError_t err = cudaSuccess;
  // On the side stream, beside the tensor-core kernels on the caller's stream:
  // the tokens grouped by target (for the exact one-hot part of dW; it reads
  // only the targets), the first block's fp16 h rows and the first piece's
  // fp16 W rows (beside the first gradient tile kernel, which reads the bf16
  // originals), and each next piece's W rows once the current piece's dh GEMM
  // is done with the copy (beside its dW GEMM and the next gradient tile
  // kernel).  The next block's h rows are copied on the caller's stream, after
  // the block before has finished with them.
  SegIndexDev ix;
  SideScope side(st);
  err = build_segindex(p.y, p.T, p.V, seg_ws, &ix, side.stream());
  if (err != cudaSuccess) return err;
  err = run_half_copies(p, p.h, 0, plan.Tb <= p.T ? plan.Tb : p.T, h16, maxbits + p.M, inv + p.M, side.stream());
  if (err != cudaSuccess) return err;
  err = run_half_copies(p, p.W, 0, plan.Vc <= p.V ? plan.Vc : p.V, w16, maxbits, inv, side.stream());
  if (err != cudaSuccess) return err;
  for (int64_t t0 = 0; t0 < p.T && err == cudaSuccess; t0 += plan.Tb) {
    const int64_t Tb = t0 + plan.Tb <= p.T ? plan.Tb : p.T - t0;
    if (t0 > 0) {
      err = run_half_copies(p, p.h, t0, Tb, h16, maxbits + p.M, inv + p.M, st);
      if (err != cudaSuccess) break;
    }
    for (int64_t v0 = 0; v0 < p.V && err == cudaSuccess; v0 += plan.Vc) {
      BwdChunk c;
      c.t0 = t0;
      c.Tb = Tb;
      c.v0 = v0;
      c.Vc = v0 + plan.Vc <= p.V ? plan.Vc : p.V - v0;
      c.first_v = v0 == 0;
      c.last_v = v0 + c.Vc >= p.V;
      c.first_t = t0 == 0;
      c.G = G;
      c.acc = acc;
      c.w16 = w16;
      c.w16_inv = inv;
      c.h16 = h16;
      c.h16_inv = inv + p.M;
      err = run_grad_chunk(p, c, stats, st);
      if (err != cudaSuccess) break;
      err = side.join();                      // this piece's fp16 copies are done
      if (err != cudaSuccess) break;
      switch (bn) {
        case 256: err = run_dh_chunk<256>(p, c, dh, alpha, st); break;
        case 128: err = run_dh_chunk<128>(p, c, dh, alpha, st); break;
        default: err = run_dh_chunk<64>(p, c, dh, alpha, st); break;
      }
      if (err != cudaSuccess) break;
      // the next piece's W rows (the next chunk, or the next block's first chunk)
      const bool more = !(c.last_v && t0 + Tb >= p.T);
      if (more) {
        const int64_t nv0 = c.last_v ? 0 : v0 + plan.Vc;
        const int64_t nVc = nv0 + plan.Vc <= p.V ? plan.Vc : p.V - nv0;
        err = side.fork();
        if (err == cudaSuccess) err = run_half_copies(p, p.W, nv0, nVc, w16, maxbits, inv, side.stream());
        if (err != cudaSuccess) break;
      }
      switch (bn) {
        case 256: err = run_dw_chunk<256>(p, c, dW, alpha, accumulate, st); break;
        case 128: err = run_dw_chunk<128>(p, c, dW, alpha, accumulate, st); break;
        default: err = run_dw_chunk<64>(p, c, dW, alpha, accumulate, st); break;
      }
    }
  }
  if (err != cudaSuccess) return err;
  err = side.join();
  if (err != cudaSuccess) return err;
  // one-hot part of dW over every token: (1 - alpha_d) for students, 1 for the
  // teacher; every exit in one launch pair, the heavy rows on the side stream
  // beside the others (disjoint rows of dW)
  int d_vec[kMaxExits];
  float scale[kMaxExits];
  for (int m = 0; m < p.M; ++m) {
    const float cm = (m == p.M - 1) ? 1.f : 1.f - p.alpha_d;
    d_vec[m] = static_cast<int>(p.D[m] / 8);
    scale[m] = alpha * p.exit_w[m] * cm;
  }
  err = side.fork();
  if (err != cudaSuccess) return err;
  err = scatter_target_rows(ix, p.M, p.h, d_vec, dW, scale, st, side.stream());
  if (err != cudaSuccess) return err;
  return side.join();
}

}  // namespace mls
