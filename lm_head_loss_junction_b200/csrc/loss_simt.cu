// fp32 CUDA-core path of the multi-exit loss (used for MLS_F32 inputs, where
// bf16 tensor cores would change the arithmetic), plus the fixed-order loss
// reduction shared with the tensor-core path.
//
// One thread block per token: every thread walks a strided subset of the
// vocabulary, computes the logits of all exits for its entries, and keeps
// online softmax statistics.  The teacher (largest exit) keeps its running
// max m_T and sum z_T; every student also keeps A_s = sum_v exp(l_T,v - m_T)
// l_s,v so that S_s = sum_v p_T,v l_s,v = A_s / z_T.  Partials are merged by a
// fixed tree, so results are deterministic.
#include "common.cuh"
#include "kernels.h"

namespace mls {

namespace {

constexpr int kSimtThreads = 256;

struct SimtDev {
  int M;
  int64_t T, V;
  int64_t D[kMaxExits];
  int64_t Doff[kMaxExits];   // offsets of each exit's row in the staged h row
  const int32_t* y;
  const float* h[kMaxExits];
  const float* W[kMaxExits];
  float alpha_d;
  float exit_w[kMaxExits];
  int distill;               // 0: cross-entropy, 1: KL(q_m || p_M), 2: Jensen-Shannon, 3: 1 - sum min(q, p)
  int teacher_grad;          // 1: no stop-gradient on the largest exit
  int32_t* status;
  float* dh[kMaxExits];
  float* dW[kMaxExits];
  int vec;                   // every width a multiple of 4 and every W row 16-byte aligned: float4 loads
};

__device__ __forceinline__ void merge_max_sum(float& m1, float& z1, float m2, float z2) {
  const float m = fmaxf(m1, m2);
  if (m == -INFINITY) return;
  z1 = z1 * __expf(m1 - m) + z2 * __expf(m2 - m);
  m1 = m;
}

constexpr float kLn2 = 0.6931471805599453f;

// log(1 + e^x), without overflow for large x.
__device__ __forceinline__ float softplus(float x) { return fmaxf(x, 0.f) + log1pf(expf(-fabsf(x))); }

// a[i] of a per-exit register array by selects (an indexed read with a
// run-time i would move the array to local memory).
__device__ __forceinline__ float exit_at(const float (&a)[kMaxExits], int i) {
  float r = a[0];
#pragma unroll
  for (int k = 1; k < kMaxExits; ++k) r = (i == k) ? a[k] : r;
  return r;
}

// One logit: the staged h row (shared memory) against one W row (global
// memory), with four independent partial sums so that the row's loads are not
// serialised behind one chain of dependent FMAs; float4 loads when p.vec.
__device__ __forceinline__ float dot_row(const float* __restrict__ hh, const float* __restrict__ w, int64_t D,
                                         int vec) {
  float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
  int64_t k = 0;
  if (vec) {
    const float4* w4 = reinterpret_cast<const float4*>(w);
    const float4* h4 = reinterpret_cast<const float4*>(hh);
    const int64_t n4 = D >> 2;
#pragma unroll 4
    for (int64_t i = 0; i < n4; ++i) {
      const float4 x = __ldg(w4 + i);
      const float4 y = h4[i];
      a0 = fmaf(y.x, x.x, a0);
      a1 = fmaf(y.y, x.y, a1);
      a2 = fmaf(y.z, x.z, a2);
      a3 = fmaf(y.w, x.w, a3);
    }
    k = n4 << 2;
  } else {
#pragma unroll 1
    for (; k + 4 <= D; k += 4) {
      a0 = fmaf(hh[k], __ldg(w + k), a0);
      a1 = fmaf(hh[k + 1], __ldg(w + k + 1), a1);
      a2 = fmaf(hh[k + 2], __ldg(w + k + 2), a2);
      a3 = fmaf(hh[k + 3], __ldg(w + k + 3), a3);
    }
  }
  for (; k < D; ++k) a0 = fmaf(hh[k], __ldg(w + k), a0);
  return (a0 + a1) + (a2 + a3);
}

// Quantities per thread, in shared memory for the tree merge:
//   [0] m_T  [1] z_T  [2..2+M-2] A_s  then per student (m_s, z_s), then tgt[M]
__global__ void __launch_bounds__(kSimtThreads, 1) simt_stats_kernel(const SimtDev p, float* __restrict__ stats,
                                                                  float* __restrict__ terms) {
  extern __shared__ float sm[];
  __shared__ float lse_sh[kMaxExits];
  const int M = p.M;
  const int S = M - 1;
  const int64_t t = blockIdx.x;
  const int tid = threadIdx.x;
  float* hrow = sm;
  int64_t hsum = 0;
#pragma unroll
  for (int m = 0; m < kMaxExits; ++m) if (m < M) hsum += p.D[m];
  float* red = sm + hsum;  // [Q][kSimtThreads]
#pragma unroll
  for (int m = 0; m < kMaxExits; ++m) if (m < M)
    for (int64_t k = tid; k < p.D[m]; k += kSimtThreads) hrow[p.Doff[m] + k] = p.h[m][t * p.D[m] + k];
  __syncthreads();

  const int32_t yt = p.y[t];
  const bool bad = yt < 0 || yt >= p.V;
  float mT = -INFINITY, zT = 0.f;
  float A[kMaxExits - 1], ms[kMaxExits - 1], zs[kMaxExits - 1], tgt[kMaxExits];
  for (int s = 0; s < kMaxExits - 1; ++s) { A[s] = 0.f; ms[s] = -INFINITY; zs[s] = 0.f; }
  for (int m = 0; m < kMaxExits; ++m) tgt[m] = 0.f;

  for (int64_t v = tid; v < p.V; v += kSimtThreads) {
    float l[kMaxExits];
#pragma unroll
    for (int m = 0; m < kMaxExits; ++m) if (m < M) {
      l[m] = dot_row(hrow + p.Doff[m], p.W[m] + v * p.D[m], p.D[m], p.vec);
    }
    const float lT = exit_at(l, M - 1);
    if (lT > mT) {
      const float r = __expf(mT - lT);
      zT *= r;
      if (p.distill != 1) {
#pragma unroll
        for (int s = 0; s < kMaxExits - 1; ++s) if (s < S) A[s] *= r;
      }
      mT = lT;
    }
    const float pt = __expf(lT - mT);
    zT += pt;
#pragma unroll
    for (int s = 0; s < kMaxExits - 1; ++s) if (s < S) {
      if (p.distill != 1) A[s] = fmaf(pt, l[s], A[s]);
      if (l[s] > ms[s]) {
        const float r = __expf(ms[s] - l[s]);
        zs[s] *= r;
        if (p.distill == 1) A[s] *= r;   // reverse KL: sum q~ (l_m - l_T) follows the student's max
        ms[s] = l[s];
      }
      const float qs = __expf(l[s] - ms[s]);
      zs[s] += qs;
      if (p.distill == 1) A[s] = fmaf(qs, l[s] - lT, A[s]);
    }
    if (v == yt) {
#pragma unroll
      for (int m = 0; m < kMaxExits; ++m) if (m < M) tgt[m] = l[m];
    }
  }

  // stage per-thread partials
  red[0 * kSimtThreads + tid] = mT;
  red[1 * kSimtThreads + tid] = zT;
#pragma unroll
  for (int s = 0; s < kMaxExits - 1; ++s) if (s < S) red[(2 + s) * kSimtThreads + tid] = A[s];
#pragma unroll
  for (int s = 0; s < kMaxExits - 1; ++s) if (s < S) {
    red[(2 + S + 2 * s) * kSimtThreads + tid] = ms[s];
    red[(2 + S + 2 * s + 1) * kSimtThreads + tid] = zs[s];
  }
#pragma unroll
  for (int m = 0; m < kMaxExits; ++m) if (m < M) red[(2 + 3 * S + m) * kSimtThreads + tid] = tgt[m];
  __syncthreads();
  for (int stride = kSimtThreads / 2; stride > 0; stride >>= 1) {
    if (tid < stride) {
      const int o = tid + stride;
      float m1 = red[tid], z1 = red[kSimtThreads + tid];
      const float m2 = red[o], z2 = red[kSimtThreads + o];
      const float mm = fmaxf(m1, m2);
      const float r1 = (m1 == -INFINITY) ? 0.f : __expf(m1 - mm);
      const float r2 = (m2 == -INFINITY) ? 0.f : __expf(m2 - mm);
      red[tid] = mm;
      red[kSimtThreads + tid] = z1 * r1 + z2 * r2;
#pragma unroll
      for (int s = 0; s < kMaxExits - 1; ++s) if (s < S) {
        float* a = red + (2 + s) * kSimtThreads;
        float* msp = red + (2 + S + 2 * s) * kSimtThreads;
        float* zsp = msp + kSimtThreads;
        if (p.distill != 1) {
          a[tid] = a[tid] * r1 + a[o] * r2;
        } else {
          const float sm = fmaxf(msp[tid], msp[o]);
          const float s1 = (msp[tid] == -INFINITY) ? 0.f : __expf(msp[tid] - sm);
          const float s2 = (msp[o] == -INFINITY) ? 0.f : __expf(msp[o] - sm);
          a[tid] = a[tid] * s1 + a[o] * s2;
        }
        float mA = msp[tid], zA = zsp[tid];
        merge_max_sum(mA, zA, msp[o], zsp[o]);
        msp[tid] = mA;
        zsp[tid] = zA;
      }
#pragma unroll
      for (int m = 0; m < kMaxExits; ++m) if (m < M) red[(2 + 3 * S + m) * kSimtThreads + tid] += red[(2 + 3 * S + m) * kSimtThreads + o];
    }
    __syncthreads();
  }
  if (tid == 0) {
    const float lseT = red[0] + logf(red[kSimtThreads]);
#pragma unroll
    for (int m = 0; m < kMaxExits; ++m) if (m < M) {
      float lse;
      if (m == M - 1) {
        lse = lseT;
      } else {
        lse = red[(2 + S + 2 * m) * kSimtThreads] + logf(red[(2 + S + 2 * m + 1) * kSimtThreads]);
      }
      const float tg = red[(2 + 3 * S + m) * kSimtThreads];
      stats[m * p.T + t] = lse;
      stats[(M + m) * p.T + t] = bad ? 0.f : tg;
      terms[m * p.T + t] = bad ? 0.f : lse - tg;
    }
#pragma unroll
    for (int s = 0; s < kMaxExits - 1; ++s) if (s < S) {
      const float zsum = red[(2 + S + 2 * s + 1) * kSimtThreads];
      const float lse = red[(2 + S + 2 * s) * kSimtThreads] + logf(zsum);
      // cross-entropy: S = sum p_T l_m; reverse KL: R = sum q_m (l_m - l_T)
      const float Sv = red[(2 + s) * kSimtThreads] / (p.distill != 1 ? red[kSimtThreads] : zsum);
      stats[(2 * M + s) * p.T + t] = Sv;
      terms[(M + s) * p.T + t] = bad ? 0.f : (p.distill != 1 ? lse - Sv : Sv - lse + lseT);
    }
    if (bad) set_flag(p.status, MLS_DEVFLAG_BAD_ID);
#pragma unroll
    for (int m = 0; m < kMaxExits; ++m) if (m < M) lse_sh[m] = stats[m * p.T + t];
  }
  if ((p.distill != 2 && p.distill != 3) || S == 0) return;
  // Jensen-Shannon or acceptance: second walk over the vocabulary with the final
  // normalisers; Jensen-Shannon sums q log(q/mu) and p log(p/mu) (mu = (q + p)/2),
  // acceptance sums q where q < p (A) and p where q >= p (B).
  __syncthreads();
  float lse[kMaxExits];
#pragma unroll
  for (int m = 0; m < kMaxExits; ++m) if (m < M) lse[m] = lse_sh[m];
  const float lseT = exit_at(lse, M - 1);
  float jq[kMaxExits - 1], jp[kMaxExits - 1];
  for (int s = 0; s < kMaxExits - 1; ++s) { jq[s] = 0.f; jp[s] = 0.f; }
  for (int64_t v = tid; v < p.V; v += kSimtThreads) {
    float l[kMaxExits];
#pragma unroll
    for (int m = 0; m < kMaxExits; ++m) if (m < M) {
      l[m] = dot_row(hrow + p.Doff[m], p.W[m] + v * p.D[m], p.D[m], p.vec);
    }
    const float lp = exit_at(l, M - 1) - lseT;
    const float pv = expf(lp);
#pragma unroll
    for (int s = 0; s < kMaxExits - 1; ++s) if (s < S) {
      const float lq = l[s] - lse[s];
      if (p.distill == 3) {
        if (lq < lp) jq[s] += expf(lq);
        else jp[s] += pv;
      } else {
        const float d = lp - lq;
        jq[s] = fmaf(expf(lq), kLn2 - softplus(d), jq[s]);
        jp[s] = fmaf(pv, kLn2 - softplus(-d), jp[s]);
      }
    }
  }
#pragma unroll
  for (int s = 0; s < kMaxExits - 1; ++s) if (s < S) {
    red[(2 * s) * kSimtThreads + tid] = jq[s];
    red[(2 * s + 1) * kSimtThreads + tid] = jp[s];
  }
  __syncthreads();
  for (int stride = kSimtThreads / 2; stride > 0; stride >>= 1) {
    if (tid < stride)
      for (int r = 0; r < 2 * S; ++r) red[r * kSimtThreads + tid] += red[r * kSimtThreads + tid + stride];
    __syncthreads();
  }
  if (tid == 0) {
#pragma unroll
    for (int s = 0; s < kMaxExits - 1; ++s) if (s < S) {
      const float a = red[(2 * s) * kSimtThreads], b = red[(2 * s + 1) * kSimtThreads];
      if (p.distill == 3) {                 // A, then B for the teacher; the term is 1 - (A + B)
        stats[(2 * M + s) * p.T + t] = a;
        if (p.teacher_grad) stats[(3 * M - 1 + s) * p.T + t] = b;
        terms[(M + s) * p.T + t] = bad ? 0.f : 1.f - (a + b);
      } else {
        stats[(2 * M + s) * p.T + t] = 0.5f * a;
        if (p.teacher_grad) stats[(3 * M - 1 + s) * p.T + t] = 0.5f * b;   // KL(p_T || mu)/2
        terms[(M + s) * p.T + t] = bad ? 0.f : 0.5f * (a + b);
      }
    }
  }
}

// Backward, one block per token: G'_m[t, :] into the workspace, then
// dh_m[t] = alpha * G'_m[t, :] W^m.
__global__ void __launch_bounds__(kSimtThreads, 1) simt_grad_kernel(const SimtDev p, const float* __restrict__ stats,
                                                                 float alpha, float* __restrict__ G) {
  extern __shared__ float sm[];
  const int M = p.M;
  const int64_t t = blockIdx.x;
  const int tid = threadIdx.x;
  float* hrow = sm;
#pragma unroll
  for (int m = 0; m < kMaxExits; ++m) if (m < M)
    for (int64_t k = tid; k < p.D[m]; k += kSimtThreads) hrow[p.Doff[m] + k] = p.h[m][t * p.D[m] + k];
  __syncthreads();
  const int32_t yt = p.y[t];
  const bool bad = yt < 0 || yt >= p.V;
  float lse[kMaxExits], kl[kMaxExits];
#pragma unroll
  for (int m = 0; m < kMaxExits; ++m) if (m < M) lse[m] = stats[m * p.T + t];
  const float lseT = exit_at(lse, M - 1);
  // reverse KL: KL(q_m || p_T) = R - lse_m + lse_T; Jensen-Shannon: K = KL(q_m || mu)/2 as stored
#pragma unroll
  for (int m = 0; m < kMaxExits - 1; ++m) if (m < M - 1)
    kl[m] = (p.distill >= 2) ? stats[(2 * M + m) * p.T + t] : stats[(2 * M + m) * p.T + t] - lse[m] + lseT;
  const float a = p.alpha_d;
  for (int64_t v = tid; v < p.V; v += kSimtThreads) {
    float l[kMaxExits];
#pragma unroll
    for (int m = 0; m < kMaxExits; ++m) if (m < M) {
      l[m] = dot_row(hrow + p.Doff[m], p.W[m] + v * p.D[m], p.D[m], p.vec);
    }
    const float lT = exit_at(l, M - 1);
    const float pT = __expf(lT - lseT);
    const float hot = (v == yt) ? 1.f : 0.f;
#pragma unroll
    for (int m = 0; m < kMaxExits; ++m) if (m < M) {
      float g;
      if (m == M - 1) {
        g = pT - hot;
        if (p.teacher_grad) {
          // distillation gradient of every smaller exit s on the teacher's logits:
          //   cross-entropy -p_T (l_s - S_s);  reverse KL p_T - q_s;
          //   Jensen-Shannon p_T (log(p_T/mu_s)/2 - K^p_s), log(p/mu) = ln 2 - softplus(log q - log p);
          //   acceptance p_T (B_s - [q_s >= p_T])
          float extra = 0.f;
#pragma unroll
          for (int s = 0; s < kMaxExits - 1; ++s) if (s < M - 1) {
            float ts;
            if (p.distill == 1) {
              ts = pT - __expf(l[s] - lse[s]);
            } else if (p.distill == 2) {
              const float lq = l[s] - lse[s], lp = lT - lseT;
              ts = pT * (0.5f * (kLn2 - softplus(lq - lp)) - stats[(3 * M - 1 + s) * p.T + t]);
            } else if (p.distill == 3) {    // acceptance: p_T (B_s - [q_s >= p_T])
              const float lq = l[s] - lse[s], lp = lT - lseT;
              ts = pT * (stats[(3 * M - 1 + s) * p.T + t] - ((lq < lp) ? 0.f : 1.f));
            } else {
              ts = -pT * (l[s] - stats[(2 * M + s) * p.T + t]);
            }
            extra = fmaf(p.exit_w[s], ts, extra);
          }
          G[(static_cast<int64_t>(m) * p.T + t) * p.V + v] = bad ? 0.f : fmaf(a, extra, p.exit_w[m] * g);
          continue;
        }
      } else if (p.distill == 0) {
        g = __expf(l[m] - lse[m]) - a * pT - (1.f - a) * hot;
      } else if (p.distill == 1) {
        const float q = __expf(l[m] - lse[m]);
        const float d = (l[m] - lse[m]) - (lT - lseT) - kl[m];
        g = (1.f - a) * (q - hot) + a * q * d;
      } else if (p.distill == 2) {
        const float q = __expf(l[m] - lse[m]);
        const float d = 0.5f * (kLn2 - softplus((lT - lseT) - (l[m] - lse[m]))) - kl[m];
        g = (1.f - a) * (q - hot) + a * q * d;
      } else {                              // acceptance: q (A - [q < p])
        const float q = __expf(l[m] - lse[m]);
        const float ind = ((l[m] - lse[m]) < (lT - lseT)) ? 1.f : 0.f;
        g = (1.f - a) * (q - hot) + a * q * (kl[m] - ind);
      }
      G[(static_cast<int64_t>(m) * p.T + t) * p.V + v] = bad ? 0.f : p.exit_w[m] * g;
    }
  }
  __syncthreads();
#pragma unroll
  for (int m = 0; m < kMaxExits; ++m) if (m < M) {
    const float* g = G + (static_cast<int64_t>(m) * p.T + t) * p.V;
    const float* __restrict__ Wm = p.W[m];
    const int64_t D = p.D[m];
    for (int64_t k = tid; k < D; k += kSimtThreads) {
      // four partial sums over the vocabulary (independent loads in flight)
      float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
      int64_t v = 0;
      for (; v + 4 <= p.V; v += 4) {
        a0 = fmaf(g[v], __ldg(Wm + v * D + k), a0);
        a1 = fmaf(g[v + 1], __ldg(Wm + (v + 1) * D + k), a1);
        a2 = fmaf(g[v + 2], __ldg(Wm + (v + 2) * D + k), a2);
        a3 = fmaf(g[v + 3], __ldg(Wm + (v + 3) * D + k), a3);
      }
      for (; v < p.V; ++v) a0 = fmaf(g[v], __ldg(Wm + v * D + k), a0);
      p.dh[m][t * D + k] = bad ? 0.f : alpha * ((a0 + a1) + (a2 + a3));
    }
  }
  if (tid == 0 && bad) set_flag(p.status, MLS_DEVFLAG_BAD_ID);
}

// dW^m[v] (+)= alpha * sum_t G'_m[t, v] h_m[t], one block per (v, m).
__global__ void __launch_bounds__(kSimtThreads, 1) simt_dw_kernel(const SimtDev p, float alpha, const float* __restrict__ G,
                                                               int accumulate) {
  const int64_t v = blockIdx.x;
  const int m = blockIdx.y;
  const float* g = G + static_cast<int64_t>(m) * p.T * p.V + v;
  const float* __restrict__ hm = p.h[m];
  const int64_t D = p.D[m], V = p.V;
  for (int64_t k = threadIdx.x; k < D; k += kSimtThreads) {
    // four partial sums over the tokens (independent loads in flight)
    float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
    int64_t t = 0;
    for (; t + 4 <= p.T; t += 4) {
      a0 = fmaf(g[t * V], __ldg(hm + t * D + k), a0);
      a1 = fmaf(g[(t + 1) * V], __ldg(hm + (t + 1) * D + k), a1);
      a2 = fmaf(g[(t + 2) * V], __ldg(hm + (t + 2) * D + k), a2);
      a3 = fmaf(g[(t + 3) * V], __ldg(hm + (t + 3) * D + k), a3);
    }
    for (; t < p.T; ++t) a0 = fmaf(g[t * V], __ldg(hm + t * D + k), a0);
    const float acc = (a0 + a1) + (a2 + a3);
    float* out = p.dW[m] + v * D + k;
    *out = accumulate ? *out + alpha * acc : alpha * acc;
  }
}

// Fixed-order sum of the per-token loss terms; one block.
struct ExitWeights {
  float w[kMaxExits];
};

__global__ void __launch_bounds__(1024) loss_reduce_kernel(const float* __restrict__ terms, int M, int64_t T,
                                                           float alpha_d, ExitWeights ew, float* __restrict__ losses) {
  __shared__ float part[1024];
  __shared__ float tot[2 * kMaxExits];
  const int tid = threadIdx.x;
  const int Q = 2 * M - 1;
  for (int q = 0; q < Q; ++q) {
    float s = 0.f;
    for (int64_t i = tid; i < T; i += 1024) s += terms[q * T + i];
    part[tid] = s;
    __syncthreads();
    for (int stride = 512; stride > 0; stride >>= 1) {
      if (tid < stride) part[tid] += part[tid + stride];
      __syncthreads();
    }
    if (tid == 0) tot[q] = part[0] / static_cast<float>(T);
    __syncthreads();
  }
  if (tid == 0) {
    float L = ew.w[M - 1] * tot[M - 1];
#pragma unroll
    for (int m = 0; m < kMaxExits; ++m) if (m < M) losses[m] = tot[m];
#pragma unroll
    for (int s = 0; s < kMaxExits - 1; ++s) if (s < M - 1) {
      losses[M + s] = tot[M + s];
      L += ew.w[s] * ((1.f - alpha_d) * tot[s] + alpha_d * tot[M + s]);
    }
    losses[2 * M - 1] = L;
  }
}

// Mean over T of each of Q rows, fixed-order reduction; one block per row.
__global__ void __launch_bounds__(1024) row_means_kernel(const float* __restrict__ rows, int64_t T,
                                                         float* __restrict__ out) {
  __shared__ float part[1024];
  const int tid = threadIdx.x;
  const float* r = rows + static_cast<int64_t>(blockIdx.x) * T;
  float s = 0.f;
  for (int64_t i = tid; i < T; i += 1024) s += r[i];
  part[tid] = s;
  __syncthreads();
  for (int stride = 512; stride > 0; stride >>= 1) {
    if (tid < stride) part[tid] += part[tid + stride];
    __syncthreads();
  }
  if (tid == 0) out[blockIdx.x] = part[0] / static_cast<float>(T);
}

// Agreement of every smaller exit with the largest, one block per token, with
// the normalisers from the forward statistics: sum_v min(q_m, p_T),
// sum_v p_T l_m, sum_v p_T l_T and the first maximum of each exit's logits.
__global__ void __launch_bounds__(kSimtThreads, 1) simt_agree_kernel(const SimtDev p, const float* __restrict__ stats,
                                                                  float* __restrict__ terms,
                                                                  int32_t* __restrict__ top1) {
  extern __shared__ float sm[];
  const int M = p.M;
  const int S = M - 1;
  const int64_t t = blockIdx.x;
  const int tid = threadIdx.x;
  float* hrow = sm;
  int64_t hsum = 0;
#pragma unroll
  for (int m = 0; m < kMaxExits; ++m) if (m < M) hsum += p.D[m];
  float* red = sm + hsum;                     // [2S + 1 + M][kSimtThreads] floats
  int* redi = reinterpret_cast<int*>(red + (2 * S + 1 + M) * kSimtThreads);   // [M][kSimtThreads]
#pragma unroll
  for (int m = 0; m < kMaxExits; ++m) if (m < M)
    for (int64_t k = tid; k < p.D[m]; k += kSimtThreads) hrow[p.Doff[m] + k] = p.h[m][t * p.D[m] + k];
  __syncthreads();
  float lse[kMaxExits];
#pragma unroll
  for (int m = 0; m < kMaxExits; ++m) if (m < M) lse[m] = stats[m * p.T + t];
  const float lseT = exit_at(lse, M - 1);
  float beta[kMaxExits - 1] = {0.f, 0.f, 0.f}, sl[kMaxExits - 1] = {0.f, 0.f, 0.f}, st = 0.f;
  float mx[kMaxExits] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
  int ix[kMaxExits] = {-1, -1, -1, -1};
  for (int64_t v = tid; v < p.V; v += kSimtThreads) {
    float l[kMaxExits];
#pragma unroll
    for (int m = 0; m < kMaxExits; ++m) if (m < M) {
      l[m] = dot_row(hrow + p.Doff[m], p.W[m] + v * p.D[m], p.D[m], p.vec);
      if (l[m] > mx[m]) { mx[m] = l[m]; ix[m] = static_cast<int>(v); }
    }
    const float lT = exit_at(l, M - 1);
    const float pT = __expf(lT - lseT);
    st = fmaf(pT, lT, st);
#pragma unroll
    for (int s = 0; s < kMaxExits - 1; ++s) if (s < S) {
      beta[s] += fminf(__expf(l[s] - lse[s]), pT);
      sl[s] = fmaf(pT, l[s], sl[s]);
    }
  }
#pragma unroll
  for (int s = 0; s < kMaxExits - 1; ++s) if (s < S) {
    red[s * kSimtThreads + tid] = beta[s];
    red[(S + s) * kSimtThreads + tid] = sl[s];
  }
  red[2 * S * kSimtThreads + tid] = st;
#pragma unroll
  for (int m = 0; m < kMaxExits; ++m) if (m < M) {
    red[(2 * S + 1 + m) * kSimtThreads + tid] = mx[m];
    redi[m * kSimtThreads + tid] = ix[m];
  }
  __syncthreads();
  for (int stride = kSimtThreads / 2; stride > 0; stride >>= 1) {
    if (tid < stride) {
      const int o = tid + stride;
      for (int q = 0; q < 2 * S + 1; ++q) red[q * kSimtThreads + tid] += red[q * kSimtThreads + o];
#pragma unroll
      for (int m = 0; m < kMaxExits; ++m) if (m < M) {
        float* mv = red + (2 * S + 1 + m) * kSimtThreads;
        int* iv = redi + m * kSimtThreads;
        // larger value wins; on equal values the smaller vocabulary index
        if (mv[o] > mv[tid] || (mv[o] == mv[tid] && iv[o] >= 0 && (iv[tid] < 0 || iv[o] < iv[tid]))) {
          mv[tid] = mv[o];
          iv[tid] = iv[o];
        }
      }
    }
    __syncthreads();
  }
  if (tid == 0) {
#pragma unroll
    for (int m = 0; m < kMaxExits; ++m) if (m < M) top1[m * p.T + t] = redi[m * kSimtThreads];
    const float stT = red[2 * S * kSimtThreads];
#pragma unroll
    for (int s = 0; s < kMaxExits - 1; ++s) if (s < S) {
      terms[s * p.T + t] = red[s * kSimtThreads];
      terms[(S + s) * p.T + t] = (stT - red[(S + s) * kSimtThreads]) + (lse[s] - lseT);
      terms[(2 * S + s) * p.T + t] = (redi[s * kSimtThreads] == redi[(M - 1) * kSimtThreads]) ? 1.f : 0.f;
    }
  }
}

SimtDev make_dev(const LossProblem& p) {
  SimtDev d{};
  d.M = p.M;
  d.T = p.T;
  d.V = p.V;
  int64_t off = 0;
  for (int m = 0; m < p.M; ++m) {
    d.D[m] = p.D[m];
    d.Doff[m] = off;
    off += p.D[m];
    d.h[m] = static_cast<const float*>(p.h[m]);
    d.W[m] = static_cast<const float*>(p.W[m]);
  }
  d.y = p.y;
  d.alpha_d = p.alpha_d;
  d.distill = p.distill;
  d.teacher_grad = (p.teacher_grad != 0 && p.M > 1) ? 1 : 0;
  for (int m = 0; m < kMaxExits; ++m) d.exit_w[m] = p.exit_w[m];
  d.status = p.status;
  d.vec = 1;
  for (int m = 0; m < p.M; ++m)
    if (p.D[m] % 4 != 0 || reinterpret_cast<uintptr_t>(p.W[m]) % 16 != 0) d.vec = 0;
  return d;
}

int64_t sum_d(const LossProblem& p) {
  int64_t s = 0;
  for (int m = 0; m < p.M; ++m) s += p.D[m];
  return s;
}

cudaError_t ensure_smem(const void* fn, size_t bytes) {
  if (bytes <= 48 * 1024) return cudaSuccess;
  return cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(bytes));
}

}  // namespace

size_t loss_simt_fwd_bytes(const LossProblem& p) {
  return static_cast<size_t>(2 * p.M - 1) * p.T * sizeof(float);
}

size_t loss_simt_bwd_bytes(const LossProblem& p) {
  return static_cast<size_t>(p.M) * p.T * p.V * sizeof(float);
}

cudaError_t launch_row_means(const float* rows, int Q, int64_t T, float* out, cudaStream_t st) {
  row_means_kernel<<<Q, 1024, 0, st>>>(rows, T, out);
  note_launches(1);
  return cudaGetLastError();
}

size_t agree_simt_bytes(const LossProblem& p) {
  const size_t terms = static_cast<size_t>(3 * (p.M - 1)) * p.T * sizeof(float);
  const size_t top1 = static_cast<size_t>(p.M) * p.T * sizeof(int32_t);
  return ((terms + 255) & ~size_t(255)) + top1;
}

cudaError_t agree_simt(const LossProblem& p, const float* stats, float* metrics, float* per_token, int32_t* top1,
                       void* ws, cudaStream_t st) {
  const SimtDev d = make_dev(p);
  const size_t terms_b = static_cast<size_t>(3 * (p.M - 1)) * p.T * sizeof(float);
  float* terms = per_token != nullptr ? per_token : static_cast<float*>(ws);
  int32_t* top = top1 != nullptr ? top1
                                 : reinterpret_cast<int32_t*>(static_cast<char*>(ws) + ((terms_b + 255) & ~size_t(255)));
  const int S = p.M - 1;
  const size_t smem = (sum_d(p) + static_cast<size_t>(2 * S + 1 + p.M) * kSimtThreads) * sizeof(float) +
                      static_cast<size_t>(p.M) * kSimtThreads * sizeof(int);
  cudaError_t err = ensure_smem(reinterpret_cast<const void*>(simt_agree_kernel), smem);
  if (err != cudaSuccess) return err;
  simt_agree_kernel<<<static_cast<unsigned>(p.T), kSimtThreads, smem, st>>>(d, stats, terms, top);
  note_launches(1);
  err = cudaGetLastError();
  if (err != cudaSuccess) return err;
  return launch_row_means(terms, 3 * S, p.T, metrics, st);
}

cudaError_t launch_loss_reduce(const float* terms, const LossProblem& p, float* losses, cudaStream_t st) {
  ExitWeights ew;
  for (int m = 0; m < kMaxExits; ++m) ew.w[m] = p.exit_w[m];
  loss_reduce_kernel<<<1, 1024, 0, st>>>(terms, p.M, p.T, p.alpha_d, ew, losses);
  note_launches(1);
  return cudaGetLastError();
}

cudaError_t loss_simt_fwd(const LossProblem& p, float* losses, float* stats, void* ws, cudaStream_t st) {
  const SimtDev d = make_dev(p);
  const int S = p.M - 1;
  const int Q = 2 + S + 2 * S + p.M;   // per-thread quantities merged by the tree
  const size_t smem = (sum_d(p) + static_cast<size_t>(Q) * kSimtThreads) * sizeof(float);
  cudaError_t err = ensure_smem(reinterpret_cast<const void*>(simt_stats_kernel), smem);
  if (err != cudaSuccess) return err;
  float* terms = static_cast<float*>(ws);
  simt_stats_kernel<<<static_cast<unsigned>(p.T), kSimtThreads, smem, st>>>(d, stats, terms);
  note_launches(1);
  err = cudaGetLastError();
  if (err != cudaSuccess) return err;
  return launch_loss_reduce(terms, p, losses, st);
}

cudaError_t loss_simt_bwd(const LossProblem& p, const float* stats, float grad_scale, void* const* dh,
                          float* const* dW, int accumulate, void* ws, cudaStream_t st) {
  SimtDev d = make_dev(p);
  for (int m = 0; m < p.M; ++m) {
    d.dh[m] = static_cast<float*>(dh[m]);
    d.dW[m] = dW[m];
  }
  const float alpha = grad_scale / static_cast<float>(p.T);
  float* G = static_cast<float*>(ws);
  const size_t smem = sum_d(p) * sizeof(float);
  cudaError_t err = ensure_smem(reinterpret_cast<const void*>(simt_grad_kernel), smem);
  if (err != cudaSuccess) return err;
  simt_grad_kernel<<<static_cast<unsigned>(p.T), kSimtThreads, smem, st>>>(d, stats, alpha, G);
  note_launches(1);
  err = cudaGetLastError();
  if (err != cudaSuccess) return err;
  dim3 grid(static_cast<unsigned>(p.V), static_cast<unsigned>(p.M));
  simt_dw_kernel<<<grid, kSimtThreads, 0, st>>>(d, alpha, G, accumulate);
  note_launches(1);
  return cudaGetLastError();
}

}  // namespace mls
