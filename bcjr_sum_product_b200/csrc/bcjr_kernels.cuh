// Device code of the BCJR forward-backward library (sm_100a).
//
// Operation ("BCJR-QAT: A Differentiable Relaxation of Trellis-Coded Weight
// Quantization", Abstract and Technical Summary "Core Mechanism"): for a
// bitshift trellis with 2^L states and D = k*V bits per step, the soft
// codeword w_hat_t = sum_s c(s) p_t(s), the log-partition function logZ, the
// exact vector-Jacobian product, and the T -> 0 Viterbi decode.
//
// Formulation used here (exact rewriting of the forward-backward recursions).
// Let J = 2^(L-D).  The predecessors of a state s are {(s >> D) | (b << (L-D))},
// so alpha_t(s) = psi_t(s) * sigma_{t-1}(s >> D) with the predecessor-group sum
//     sigma_t(j) = sum_b alpha_t(j | b << (L-D)),   j in [0, J),
// and beta_{t-1}(p) depends on p only through p mod J:
//     rho_{t-1}(i) = sum_b psi_t((i << D) | b) * rho_t(((i << D) | b) mod J).
// Both recursions therefore move J values per step, and the posterior is
//     p_t(q) = psi_t(q) * sigma_{t-1}(q >> D) * rho_t(q mod J) / Z.
// Every step is one gather of 2^D members, one log-sum-exp and one add per
// group (the fused "gather, log-sum-exp, addition" of "Key Technical
// Innovations"), done in base-2 log domain so that no temperature can
// underflow a state the posterior needs.  Stored log values are re-centred each
// step by the previous step's maximum; the offsets are accumulated in fp64.
//
// For the VJP (first-order expectation semiring) the forward carries the ratio
// A_t(j) = E[sum_{u<=t} h_u | group j] and the backward
// Bc_t(i) = E[sum_{u>t} h_u | suffix group i], with h_u(s) = g_u . c(s); then
//     G_t(q) = p_t(q) (A_{t-1}(q >> D) + h_t(q) + Bc_t(q mod J) - Hbar + gZ),
//     dl/dw_t = (2/T) sum_q G_t(q) (c(q) - w_t),
//     dl/dc(q) = sum_t [ g_t p_t(q) + (2/T) G_t(q) (w_t - c(q)) ].
//
// Energies are evaluated in scaled units: with sk = sqrt(log2(e)/T),
// w' = sk*w and c' = sk*c, log2 psi_t(s) = -||w'_t - c'(s)||^2.
#pragma once
#include <cfloat>
#include <cuda_runtime.h>
#include <stdint.h>

namespace bcjr {

constexpr int kMaxThreads = 512;
constexpr int kMaxWarps = kMaxThreads / 32;

// First device-side error recorded by a kernel of this library (a status code
// of the C interface, 0 = none); read and cleared by bcjr_get_device_error.
__device__ int g_device_error = 0;
constexpr int kErrTimeout = 4;   // a bounded wait ran out (the L=16 VJP's codeword ring)
constexpr int kErrNumeric = 5;   // a per-step posterior mass left 1 +- 1e-2, or was not finite
__device__ __forceinline__ void record_device_error(int code) { atomicCAS(&g_device_error, 0, code); }
// The posterior of every step sums to 1 (both sweeps are exact rewritings of
// the same marginals); a sum off by more than 1e-2 (rounding keeps it within
// about 1e-4 even at T = 0.01 and 8192 steps) or not finite (NaN or infinite
// inputs) means the sequence's outputs are not usable.
__device__ __forceinline__ void check_posterior_mass(float s) {
  if (!(fabsf(s - 1.f) <= 1e-2f)) record_device_error(kErrNumeric);
}

struct SweepParams {
  const float* w;        // [n_seq][len]
  const float* cs;       // scaled codebook c' [S][V]
  const float* gsoft;    // [n_seq][len] upstream gradient (VJP)
  const float* gZ;       // [n_seq] or null (VJP)
  float* out_soft;       // [n_seq][len] or null
  float* out_logZ;       // [n_seq] or null
  int32_t* out_argmax;   // [n_seq][n] or null
  float* grad_w;         // [n_seq][len] (VJP)
  float* gc_seq;         // [grid][S*V]  per-sequence codebook gradient (VJP)
  double* gc_part;       // [grid][S*V]  per-CTA codebook gradient (VJP)
  float* hist_l;         // [grid][n][J] forward log2 sigma (re-centred)
  float* hist_a;         // [grid][n][J] forward A (VJP)
  double* hist_c;        // [grid][n]    forward accumulated offsets
  float* state_g;        // [grid][4][J] state buffers when they live in global memory
  int64_t n_seq, len;
  int L, n, J, S;
  float sk;              // sqrt(log2(e) / T)
  float two_over_T;
  int state_in_smem;     // 1: state buffers in shared memory, 0: in state_g
};

__device__ __forceinline__ float ex2f(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ float lg2f(float x) {
  float y;
  asm("lg2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
// better of (p, q) pairs: larger p, ties to the lower index
__device__ __forceinline__ void arg_better(float& p, int& q, float p2, int q2) {
  if (p2 > p || (p2 == p && q2 < q)) { p = p2; q = q2; }
}
__device__ __forceinline__ void warp_argmax(float& p, int& q) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    float p2 = __shfl_xor_sync(0xffffffffu, p, o);
    int q2 = __shfl_xor_sync(0xffffffffu, q, o);
    arg_better(p, q, p2, q2);
  }
}

template <int V>
__device__ __forceinline__ void load_cw(const float* __restrict__ cs, int s, float (&c)[V]) {
  if constexpr (V == 1) {
    c[0] = __ldg(cs + s);
  } else if constexpr (V == 2) {
    float2 t = __ldg(reinterpret_cast<const float2*>(cs) + s);
    c[0] = t.x; c[1] = t.y;
  } else {
    float4 t = __ldg(reinterpret_cast<const float4*>(cs) + s);
    c[0] = t.x; c[1] = t.y; c[2] = t.z; c[3] = t.w;
  }
}

enum { MODE_SOFT = 0, MODE_VJP = 1 };

// One CTA per sequence (grid-stride over sequences), forward then backward.
template <int V, int D, int MODE>
__global__ void __launch_bounds__(kMaxThreads) bcjr_sweep_kernel(SweepParams P) {
  constexpr int B = 1 << D;
  constexpr bool VJP = (MODE == MODE_VJP);
  constexpr int NP = V + 1;
  // VJP: three more per-warp partials per step, sum P(i) (A + Bc), sum P(i) Bc, sum P(i)
  constexpr int NPT = NP + (VJP ? 3 : 0);
  const int tid = threadIdx.x, nthr = blockDim.x, lane = tid & 31, warp = tid >> 5;
  const int nwarps = (nthr + 31) >> 5;
  const int J = P.J, n = P.n, HI = P.L - D;
  const int jmask = J - 1;

  extern __shared__ __align__(16) float smem[];
  float* wsc = smem;                                   // n*V scaled weights
  float* gsc = wsc + n * V;                            // n*V scaled upstream gradient (VJP)
  float* wmax = gsc + (VJP ? n * V : 0);               // [2][32]
  float* part = wmax + 64;                             // [2][32][NPT]
  float* apart = part + 2 * 32 * NPT;                  // [2][32] argmax value
  int* aidx = reinterpret_cast<int*>(apart + 64);      // [2][32] argmax index
  float* sbase = reinterpret_cast<float*>(aidx + 64);  // state buffers (if in smem)
  float* lb[2];
  float* ab[2];
  {
    float* base = P.state_in_smem ? sbase : (P.state_g + (size_t)blockIdx.x * 4 * J);
    lb[0] = base; lb[1] = base + J; ab[0] = base + 2 * J; ab[1] = base + 3 * J;
  }
  float* hist_l = P.hist_l + (size_t)blockIdx.x * n * J;
  float* hist_a = VJP ? P.hist_a + (size_t)blockIdx.x * n * J : nullptr;
  double* hist_c = P.hist_c + (size_t)blockIdx.x * n;
  float* gc_seq = VJP ? P.gc_seq + (size_t)blockIdx.x * P.S * V : nullptr;
  double* gc_part = VJP ? P.gc_part + (size_t)blockIdx.x * P.S * V : nullptr;
  const float* __restrict__ cs = P.cs;

  if constexpr (VJP) {
    for (int x = tid; x < P.S * V; x += nthr) { gc_seq[x] = 0.f; gc_part[x] = 0.0; }
  }

  for (int64_t seq = blockIdx.x; seq < P.n_seq; seq += gridDim.x) {
    const float* wq = P.w + seq * P.len;
    for (int x = tid; x < n * V; x += nthr) wsc[x] = wq[x] * P.sk;
    if constexpr (VJP) {
      const float* gq = P.gsoft + seq * P.len;
      for (int x = tid; x < n * V; x += nthr) gsc[x] = gq[x] / P.sk;
    }
    __syncthreads();

    // ------------------------------------------------------------ forward
    float R = 0.f;      // max of the previous step's stored values
    double C = 0.0;     // accumulated offsets: log2 sigma_t = stored + C_t
    for (int t = 0; t < n; ++t) {
      const float* lprev = lb[(t + 1) & 1];
      float* lcur = lb[t & 1];
      const float* aprev = ab[(t + 1) & 1];
      float* acur = ab[t & 1];
      float wt[V], gt[V];
#pragma unroll
      for (int v = 0; v < V; ++v) { wt[v] = wsc[t * V + v]; gt[v] = VJP ? gsc[t * V + v] : 0.f; }
      C += (double)R;
      // A_{t-1} enters relative to its value at group 0 (stored values stay at
      // the size of their spread over groups); the backward subtracts the same
      const float rA = (VJP && t > 0) ? aprev[0] : 0.f;
      float tmax = -INFINITY;
      for (int j = tid; j < J; j += nthr) {
        float x[B], z[B];
        float m = -INFINITY;
#pragma unroll
        for (int b = 0; b < B; ++b) {
          const int s = j | (b << HI);
          float c[V];
          load_cw<V>(cs, s, c);
          float acc = (t == 0) ? 0.f : lprev[s >> D];
#pragma unroll
          for (int v = 0; v < V; ++v) { float d = wt[v] - c[v]; acc = fmaf(-d, d, acc); }
          x[b] = acc;
          m = fmaxf(m, acc);
          if constexpr (VJP) {
            float h = 0.f;
#pragma unroll
            for (int v = 0; v < V; ++v) h = fmaf(gt[v], c[v], h);
            z[b] = ((t == 0) ? 0.f : aprev[s >> D] - rA) + h;
          }
        }
        float sum = 0.f, num = 0.f;
#pragma unroll
        for (int b = 0; b < B; ++b) {
          float u = ex2f(x[b] - m);
          sum += u;
          if constexpr (VJP) num = fmaf(u, z[b], num);
        }
        const float l = m + lg2f(sum) - R;
        lcur[j] = l;
        if (t < n - 1) hist_l[(size_t)t * J + j] = l;
        if constexpr (VJP) {
          const float a = __fdividef(num, sum);
          acur[j] = a;
          if (t < n - 1) hist_a[(size_t)t * J + j] = a;
        }
        tmax = fmaxf(tmax, l);
      }
      tmax = warp_max(tmax);
      if (lane == 0) wmax[(t & 1) * 32 + warp] = tmax;
      if (tid == 0) hist_c[t] = C;
      __syncthreads();
      R = -INFINITY;
      for (int w2 = 0; w2 < nwarps; ++w2) R = fmaxf(R, wmax[(t & 1) * 32 + w2]);
    }
    // log2 Z = log2 sum_j 2^{stored_{n-1}(j)} + C_{n-1};  VJP: Hbar = E[A_{n-1}]
    double l2Z;
    float Hbar = 0.f;
    {
      const float* lfin = lb[(n - 1) & 1];
      const float* afin = ab[(n - 1) & 1];
      float s0 = 0.f, s1 = 0.f;
      for (int j = tid; j < J; j += nthr) {
        const float u = ex2f(lfin[j] - R);
        s0 += u;
        if constexpr (VJP) s1 = fmaf(u, afin[j], s1);
      }
      s0 = warp_sum(s0);
      if constexpr (VJP) s1 = warp_sum(s1);
      if (lane == 0) { part[warp * NP] = s0; part[warp * NP + 1] = s1; }
      __syncthreads();
      float a0 = 0.f, a1 = 0.f;
      for (int w2 = 0; w2 < nwarps; ++w2) { a0 += part[w2 * NP]; a1 += part[w2 * NP + 1]; }
      l2Z = (double)R + log2((double)a0) + C;
      if constexpr (VJP) Hbar = a1 / a0;
      if (MODE == MODE_SOFT && tid == 0 && P.out_logZ) P.out_logZ[seq] = (float)(l2Z * 0.69314718055994530942);
      __syncthreads();
    }
    const float gzq = (VJP && P.gZ) ? P.gZ[seq] : 0.f;
    // G_t(q) = p_t(q) (A_{t-1}(q >> D) + h_t(q) + Bc_t(q mod J) - K_t + gZ) with
    // K_t = sum_j P_t(j) (A_t(j) + Bc_t(j)), P_t(j) the posterior of group j,
    // formed from the same stored values one step earlier (K_{n-1} = Hbar), so
    // that rounding carried along the recursions cancels in G.  Stored Bc_t is
    // relative to rB, the posterior mean of the previous step's stored values.
    float Kt = Hbar, rB = 0.f;

    // ------------------------------------------------------------ backward
    float Rr = 0.f;    // max of previous stored backward values
    double Cr = 0.0;   // accumulated backward offsets: log2 beta_t = stored + Cr_t
    for (int t = n - 1; t >= 0; --t) {
      const float* rcur = lb[t & 1];          // stored log2 rho_t (t < n-1)
      float* rnext = lb[(t + 1) & 1];         // stored log2 rho_{t-1}
      const float* bcur = ab[t & 1];          // Bc_t
      float* bnext = ab[(t + 1) & 1];         // Bc_{t-1}
      float wt[V], gt[V], graw[V];
#pragma unroll
      for (int v = 0; v < V; ++v) {
        wt[v] = wsc[t * V + v];
        gt[v] = VJP ? gsc[t * V + v] : 0.f;
        graw[v] = gt[v] * P.sk;
      }
      const double Csig = (t >= 1) ? hist_c[t - 1] : 0.0;
      const float K = (float)(Csig + Cr - l2Z);
      const bool last = (t == n - 1);
      const float rA = (VJP && t >= 1) ? hist_a[(size_t)(t - 1) * J] : 0.f;   // the forward's reference
      const float hb = Kt + rA - rB - gzq;   // G = p (A + h + (Bc - rB) - hb)
      float np_[NPT];
#pragma unroll
      for (int k2 = 0; k2 < NPT; ++k2) np_[k2] = 0.f;
      float bestp = -1.f;
      int bestq = 0x7fffffff;
      float tmax = -INFINITY;
      for (int i = tid; i < J; i += nthr) {
        const float lsig = (t >= 1) ? hist_l[(size_t)(t - 1) * J + i] : 0.f;
        float asig = 0.f;
        if constexpr (VJP) asig = (t >= 1) ? hist_a[(size_t)(t - 1) * J + i] : 0.f;
        // With more than 32 codeword components per group only the exponents
        // stay live between the two member loops (codewords and suffix values
        // are read again); up to 32 everything stays in registers.
        constexpr bool RELOAD = (B * V > 32);
        constexpr int BL = RELOAD ? 1 : B;
        float y[B], z[BL], cc[BL][V];
#pragma unroll
        for (int b = 0; b < B; ++b) {
          const int q = (i << D) | b;
          float c[V];
          load_cw<V>(cs, q, c);
          const int r = q & jmask;
          float acc = last ? 0.f : rcur[r];
#pragma unroll
          for (int v = 0; v < V; ++v) { float d = wt[v] - c[v]; acc = fmaf(-d, d, acc); }
          y[b] = acc;
          if constexpr (!RELOAD) {
#pragma unroll
            for (int v = 0; v < V; ++v) cc[b][v] = c[v];
            if constexpr (VJP) {
              float h = 0.f;
#pragma unroll
              for (int v = 0; v < V; ++v) h = fmaf(gt[v], c[v], h);
              z[b] = (last ? 0.f : bcur[r] - rB) + h;
            }
          }
        }
        // the posterior directly, p = 2^(log2 sigma + y + K), one ex2 per state
        const float kh = lsig + K;
        float sum = 0.f, num = 0.f;
#pragma unroll
        for (int b = 0; b < B; ++b) {
          const float p = ex2f(y[b] + kh);
          sum += p;
          const int q = (i << D) | b;
          float c[V], zb = 0.f;
          if constexpr (RELOAD) {
            load_cw<V>(cs, q, c);
            if constexpr (VJP) {
              float h = 0.f;
#pragma unroll
              for (int v = 0; v < V; ++v) h = fmaf(gt[v], c[v], h);
              zb = (last ? 0.f : bcur[q & jmask] - rB) + h;
            }
          } else {
#pragma unroll
            for (int v = 0; v < V; ++v) c[v] = cc[b][v];
            if constexpr (VJP) zb = z[b];
          }
          if constexpr (MODE == MODE_SOFT) {
#pragma unroll
            for (int v = 0; v < V; ++v) np_[v] = fmaf(p, c[v], np_[v]);
            np_[V] += p;
            arg_better(bestp, bestq, p, q);
          } else {
            num = fmaf(p, zb, num);
            const float G = p * (asig + zb - hb);
            np_[V] += G;
            float* gq = gc_seq + (size_t)q * V;
#pragma unroll
            for (int v = 0; v < V; ++v) {
              np_[v] = fmaf(G, c[v], np_[v]);
              const float d = wt[v] - c[v];
              float acc = fmaf(graw[v], p, gq[v]);
              gq[v] = fmaf(P.two_over_T / P.sk, G * d, acc);
            }
          }
        }
        if (t >= 1) {
          // log2 rho_{t-1}(i) = lg2 sum p - (log2 sigma + K); a group whose posterior mass
          // underflows gets rho = 0 (-inf) and Bc = 0, moving no posterior by more than that mass
          const float l = lg2f(sum) - kh - Rr;
          rnext[i] = l;
          tmax = fmaxf(tmax, l);
          if constexpr (VJP) {
            const float bn = (sum > 0.f) ? __fdividef(num, sum) : 0.f;
            bnext[i] = bn;
            const float pg = sum;   // posterior of group i at step t-1
            np_[NP] = fmaf(pg, asig + bn, np_[NP]);
            np_[NP + 1] = fmaf(pg, bn, np_[NP + 1]);
            np_[NP + 2] += pg;
          }
        }
      }
      // per-warp partials of this step
#pragma unroll
      for (int k2 = 0; k2 < NPT; ++k2) np_[k2] = warp_sum(np_[k2]);
      tmax = warp_max(tmax);
      if (MODE == MODE_SOFT) warp_argmax(bestp, bestq);
      const int pb = t & 1;
      if (lane == 0) {
#pragma unroll
        for (int k2 = 0; k2 < NPT; ++k2) part[(pb * 32 + warp) * NPT + k2] = np_[k2];
        wmax[pb * 32 + warp] = tmax;
        apart[pb * 32 + warp] = bestp;
        aidx[pb * 32 + warp] = bestq;
      }
      __syncthreads();
      if (tid == 0) {
        float tot[NP];
#pragma unroll
        for (int k2 = 0; k2 < NP; ++k2) {
          float a = 0.f;
          for (int w2 = 0; w2 < nwarps; ++w2) a += part[(pb * 32 + w2) * NPT + k2];
          tot[k2] = a;
        }
        if constexpr (MODE == MODE_SOFT) {
          check_posterior_mass(tot[V]);
          if (P.out_soft) {
            const float inv = 1.f / (tot[V] * P.sk);
#pragma unroll
            for (int v = 0; v < V; ++v) P.out_soft[seq * P.len + t * V + v] = tot[v] * inv;
          }
          if (P.out_argmax) {
            float bp = -1.f;
            int bq = 0x7fffffff;
            for (int w2 = 0; w2 < nwarps; ++w2) arg_better(bp, bq, apart[pb * 32 + w2], aidx[pb * 32 + w2]);
            P.out_argmax[seq * n + t] = bq;
          }
        } else {
#pragma unroll
          for (int v = 0; v < V; ++v)
            P.grad_w[seq * P.len + t * V + v] = P.two_over_T * (tot[v] / P.sk - (wt[v] / P.sk) * tot[V]);
        }
      }
      Cr += (double)Rr;
      Rr = -INFINITY;
      for (int w2 = 0; w2 < nwarps; ++w2) Rr = fmaxf(Rr, wmax[pb * 32 + w2]);
      if constexpr (!VJP) {
        // the same renormalisation as below: dividing out this step's posterior
        // mass keeps the drift of later steps to their own rounding
        float sp_ = 0.f;
        for (int w2 = 0; w2 < nwarps; ++w2) sp_ += part[(pb * 32 + w2) * NPT + V];
        Cr -= (double)lg2f(sp_);
      }
      if constexpr (VJP) {
        float sk_ = 0.f, sb_ = 0.f, sp_ = 0.f;
        for (int w2 = 0; w2 < nwarps; ++w2) {
          const float* r = part + (pb * 32 + w2) * NPT + NP;
          sk_ += r[0]; sb_ += r[1]; sp_ += r[2];
        }
        Kt = sk_ / sp_;
        rB = sb_ / sp_;
        // (step 0 has no predecessor groups, so no mass is summed there)
        if (tid == 0 && t >= 1) check_posterior_mass(sp_);
        // sp_ = sum_q p_t(q): forward and backward carry different rounding
        // relative to the one log Z, so the posterior sum drifts from 1 along
        // the sweep; folding its logarithm into the backward offset
        // renormalises every next step.
        Cr -= (double)lg2f(sp_);
      }
      // the next step overwrites the other parity only; this step's slots are
      // read above before any thread can pass the next barrier
    }
    if constexpr (VJP) {
      __syncthreads();
      for (int x = tid; x < P.S * V; x += nthr) { gc_part[x] += (double)gc_seq[x]; gc_seq[x] = 0.f; }
    }
    __syncthreads();
  }
}

// Final deterministic reduction of the per-CTA codebook gradients.
__global__ void reduce_gc_kernel(const double* __restrict__ part, int nparts, int SV, float* __restrict__ out) {
  int x = blockIdx.x * blockDim.x + threadIdx.x;
  if (x >= SV) return;
  double a = 0.0;
  for (int p = 0; p < nparts; ++p) a += part[(size_t)p * SV + x];
  out[x] = (float)a;
}

// Self-reconstruction loss of a sequence and its upstream gradient:
// g = 2 (w_hat - w_target), loss[q] = sum (w_hat - w_target)^2; blocks of 256
// threads stride over the sequences, each reduced in a fixed order.
__global__ void recon_grad_kernel(const float* __restrict__ soft, const float* __restrict__ target, int64_t n_seq,
                                  int64_t len, float* __restrict__ g, float* __restrict__ loss) {
  __shared__ float part[8];
  for (int64_t q = blockIdx.x; q < n_seq; q += gridDim.x) {
    const float* a = soft + q * len;
    const float* b = target + q * len;
    float* gq = g + q * len;
    float acc = 0.f;
    for (int64_t x = threadIdx.x; x < len; x += blockDim.x) {
      const float d = a[x] - b[x];
      gq[x] = 2.f * d;
      acc = fmaf(d, d, acc);
    }
    acc = warp_sum(acc);
    if ((threadIdx.x & 31) == 0) part[threadIdx.x >> 5] = acc;
    __syncthreads();
    if (threadIdx.x == 0 && loss) {
      float tot = 0.f;
      for (int i = 0; i < (int)(blockDim.x >> 5); ++i) tot += part[i];
      loss[q] = tot;
    }
    __syncthreads();
  }
}

// x <- x - lr * g
__global__ void sgd_kernel(float* __restrict__ x, const float* __restrict__ g, float lr, int64_t n) {
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x)
    x[i] = fmaf(-lr, g[i], x[i]);
}

// c'(s) = sk * c(s)
__global__ void scale_codebook_kernel(const float* __restrict__ c, int SV, float sk, float* __restrict__ cs) {
  int x = blockIdx.x * blockDim.x + threadIdx.x;
  if (x < SV) cs[x] = c[x] * sk;
}

// ------------------------------------------------------------------ Viterbi
struct ViterbiParams {
  const float* w;       // [n_seq][len]
  const float* c;       // [S][V] raw codebook
  int32_t* out_states;  // [n_seq][n]
  float* out_cost;      // [n_seq] or null
  uint8_t* bp;          // [grid][n][J] backpointers (b of the best predecessor)
  float* state_g;       // [grid][2][J] when not in smem
  int64_t n_seq, len;
  int L, n, J, S;
  int state_in_smem;
};

template <int V>
__device__ __forceinline__ float qcost(const float* wt, const float* c) {
  // q = sum over v in order of fl(fl(w - c)^2), no contraction
  float acc = 0.f;
#pragma unroll
  for (int v = 0; v < V; ++v) {
    const float d = __fsub_rn(wt[v], c[v]);
    const float sq = __fmul_rn(d, d);
    acc = (v == 0) ? sq : __fadd_rn(acc, sq);
  }
  return acc;
}

template <int V, int D>
__global__ void __launch_bounds__(kMaxThreads) viterbi_kernel(ViterbiParams P) {
  constexpr int B = 1 << D;
  const int tid = threadIdx.x, nthr = blockDim.x, lane = tid & 31, warp = tid >> 5;
  const int nwarps = (nthr + 31) >> 5;
  const int J = P.J, n = P.n, HI = P.L - D;
  extern __shared__ __align__(16) float smem[];
  float* wsm = smem;                                   // n*V
  float* red = wsm + n * V;                            // [32] values
  int* redi = reinterpret_cast<int*>(red + 32);        // [32] indices
  float* sbase = reinterpret_cast<float*>(redi + 32);
  float* mb[2];
  {
    float* base = P.state_in_smem ? sbase : (P.state_g + (size_t)blockIdx.x * 2 * J);
    mb[0] = base; mb[1] = base + J;
  }
  uint8_t* bp = P.bp + (size_t)blockIdx.x * n * J;

  for (int64_t seq = blockIdx.x; seq < P.n_seq; seq += gridDim.x) {
    const float* wq = P.w + seq * P.len;
    for (int x = tid; x < n * V; x += nthr) wsm[x] = wq[x];
    __syncthreads();
    float bestv = INFINITY;
    int bests = 0x7fffffff;
    for (int t = 0; t < n; ++t) {
      const float* mprev = mb[(t + 1) & 1];
      float* mcur = mb[t & 1];
      const float* wt = wsm + t * V;
      const bool last = (t == n - 1);
      for (int j = tid; j < J; j += nthr) {
        float best = INFINITY;
        int bb = 0;
#pragma unroll 4
        for (int b = 0; b < B; ++b) {
          const int s = j | (b << HI);
          float c[V];
          load_cw<V>(P.c, s, c);   // one vector load per codeword
          const float qv = qcost<V>(wt, c);
          const float dlt = (t == 0) ? qv : __fadd_rn(mprev[s >> D], qv);
          if (dlt < best) { best = dlt; bb = b; }
          if (last) {
            if (dlt < bestv || (dlt == bestv && s < bests)) { bestv = dlt; bests = s; }
          }
        }
        mcur[j] = best;
        if (!last) bp[(size_t)t * J + j] = (uint8_t)bb;
      }
      __syncthreads();
    }
    // block argmin of delta_{n-1}, ties to the lowest state
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      float v2 = __shfl_xor_sync(0xffffffffu, bestv, o);
      int s2 = __shfl_xor_sync(0xffffffffu, bests, o);
      if (v2 < bestv || (v2 == bestv && s2 < bests)) { bestv = v2; bests = s2; }
    }
    if (lane == 0) { red[warp] = bestv; redi[warp] = bests; }
    __syncthreads();
    if (tid == 0) {
      float bv = INFINITY; int bs = 0x7fffffff;
      for (int w2 = 0; w2 < nwarps; ++w2)
        if (red[w2] < bv || (red[w2] == bv && redi[w2] < bs)) { bv = red[w2]; bs = redi[w2]; }
      if (bs == 0x7fffffff) bs = 0;  // all-NaN sequence
      if (P.out_cost) P.out_cost[seq] = bv;
      int s = bs;
      int32_t* out = P.out_states + seq * n;
      for (int t = n - 1; t >= 0; --t) {
        out[t] = s;
        if (t > 0) {
          const int jj = s >> D;
          const int b = bp[(size_t)(t - 1) * J + jj];
          s = jj | (b << HI);
        }
      }
    }
    __syncthreads();
  }
}

}  // namespace bcjr
