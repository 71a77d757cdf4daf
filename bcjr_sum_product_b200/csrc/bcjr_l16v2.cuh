// Specialised sweep for the vector trellis: L = 16 (65536 states), k = 2,
// V = 2 (two weights per step, D = 4 bits per step, 16 branches), on sm_100a.
//
// Same mathematics as bcjr_kernels.cuh and bcjr_l16.cuh ("BCJR-QAT: A
// Differentiable Relaxation of Trellis-Coded Weight Quantization", Abstract
// and Technical Summary "Core Mechanism"): predecessor-group recursions in
// base-2 log domain with negated stored values, the energy of a state being
// the squared distance of the step's two weights to its 2-D codeword.
//
//   state q = (h << 12) | (mid << 4) | lo,  h, lo in [0, 16), mid in [0, 256).
//   The forward group j = q mod 2^12 = (mid << 4) | lo has members h, and its
//   members' predecessor groups are q >> 4 = (h << 8) | mid; the backward
//   group i = q >> 4 = (h << 8) | mid has members lo, whose successor groups
//   are q mod 2^12 = (mid << 4) | lo.
//   512 threads; thread tau takes mid = tau >> 1 and the half e = tau & 1 of
//   the other index: forward groups (mid, lo = 8e .. 8e + 7) and backward
//   groups (h = 8e .. 8e + 7, mid).  Per step a thread reads 16 group values
//   shared by all of its groups (the 16 predecessors (h << 8) | mid forward,
//   the 16 successors (mid << 4) | lo backward), so the 4096-entry vectors
//   live in a small shared-memory ping-pong; the forward history it writes,
//   sigma_{t-1}((h << 8) | mid) for its 8 h, is what the same thread reads in
//   the backward.
//   Two members share the two lanes of the packed f32x2 instructions.  The
//   scaled codebook is staged twice, in the order each direction reads it
//   (pairs of members of one group as one float4 (c0, c0', c1, c1'), float4 x
//   of thread tau at ((group * 8 + pair) * 512 + tau), so a warp reads 512
//   contiguous bytes); both copies stay in L2.
//   The VJP keeps component 0 of the sequence's per-state codebook gradient
//   in tensor memory (the 128 states of a thread's backward groups = its 128
//   columns) and component 1 in a per-CTA global buffer (L2-resident).
#pragma once
#include "bcjr_l16.cuh"

namespace bcjr {
namespace l16v2 {

using l16::f2;
using l16::f2s;
using l16::bfly16_min;
using l16::bfly16_sum;

constexpr int L = 16, D = 4, J = 1 << 12, NT = 512, S = 1 << 16;
constexpr int G = 8;                       // groups per thread per direction
constexpr int CB4 = G * 8 * NT;            // float4 per codebook copy (32768)

struct Params {
  const float* w;        // [n_seq][len], len = 2 n
  const float4* cf;      // forward-order scaled codebook, CB4 float4
  const float4* cb;      // backward-order scaled codebook, CB4 float4
  const float2* cf1;     // component 1 of cf, CB4 float2 (streamed when component 0 is in TMEM)
  const float2* cb1;     // component 1 of cb, CB4 float2
  const float* gsoft;    // [n_seq][len] (VJP)
  const float* gZ;       // [n_seq] or null (VJP)
  float* out_soft;       // [n_seq][len] or null
  float* out_logZ;       // [n_seq] or null
  int32_t* out_argmax;   // [n_seq][n] or null
  float* grad_w;         // [n_seq][len] (VJP)
  double* gc_part;       // [grid][S][2] (VJP)
  float4* gc1;           // [grid][G * 4][NT] float4: component 1 of the sequence's gradient (VJP)
  float* hist_l;         // [grid][n][J]   [mid][h] order
  float* hist_a;         // [grid][n][J]   (VJP)
  double* hist_c;        // [grid][n]
  int64_t n_seq, len;
  int n;
  float sk, two_over_T;
};

// cf[(k * 8 + p) * 512 + tau]: forward group (mid, lo = 8e + k), members h = 2p, 2p + 1;
// cb[(k * 8 + p) * 512 + tau]: backward group (h = 8e + k, mid), members lo = 2p, 2p + 1;
// each float4 = (c0(first), c0(second), c1(first), c1(second)) * sk.
__global__ void make_codebooks(const float* __restrict__ c, float sk, float4* __restrict__ cf,
                               float4* __restrict__ cb, float2* __restrict__ cf1, float2* __restrict__ cb1) {
  const int x = blockIdx.x * blockDim.x + threadIdx.x;
  if (x >= CB4) return;
  const int tau = x & (NT - 1), p = (x >> 9) & 7, k = x >> 12;
  const int mid = tau >> 1, e = tau & 1;
  const int lo = 8 * e + k;
  const int f0 = ((2 * p) << 12) | (mid << 4) | lo, f1 = ((2 * p + 1) << 12) | (mid << 4) | lo;
  cf[x] = make_float4(c[2 * f0] * sk, c[2 * f1] * sk, c[2 * f0 + 1] * sk, c[2 * f1 + 1] * sk);
  cf1[x] = make_float2(c[2 * f0 + 1] * sk, c[2 * f1 + 1] * sk);
  const int h = 8 * e + k;
  const int b0 = (h << 12) | (mid << 4) | (2 * p), b1 = b0 + 1;
  cb[x] = make_float4(c[2 * b0] * sk, c[2 * b1] * sk, c[2 * b0 + 1] * sk, c[2 * b1 + 1] * sk);
  cb1[x] = make_float2(c[2 * b0 + 1] * sk, c[2 * b1 + 1] * sk);
}

// grad_c[q][v] = sum over CTAs of gc_part[cta][q][v]
__global__ void reduce_gc(const double* __restrict__ part, int nparts, float* __restrict__ out) {
  const int x = blockIdx.x * blockDim.x + threadIdx.x;
  if (x >= 2 * S) return;
  double a = 0.0;
  for (int p = 0; p < nparts; ++p) a += part[(size_t)p * 2 * S + x];
  out[x] = (float)a;
}

// Component 0 of this thread's 8 groups x 8 member pairs of a codebook copy
// into its 128 tensor-memory columns (column 16 k + 2 p + lane).
__device__ __forceinline__ void stage_c0(const float4* __restrict__ cp, uint32_t tbase) {
#pragma unroll
  for (int k = 0; k < G; ++k) {
    float v[16];
#pragma unroll
    for (int p = 0; p < 8; ++p) {
      const float4 cw = __ldg(cp + (k * 8 + p) * NT);
      v[2 * p] = cw.x;
      v[2 * p + 1] = cw.y;
    }
    l16::tmem_st16(tbase + 16 * k, v);
  }
  l16::tmem_wait_st();
}

__device__ __forceinline__ float pick8(const float (&v)[16], int e, int i) { return e ? v[8 + i] : v[i]; }

// min over the 16 members held as 8 lane pairs
__device__ __forceinline__ float min16(const float2 (&x)[8]) {
  float a = fminf(fminf(x[0].x, x[0].y), fminf(x[1].x, x[1].y));
  float b = fminf(fminf(x[2].x, x[2].y), fminf(x[3].x, x[3].y));
  float c = fminf(fminf(x[4].x, x[4].y), fminf(x[5].x, x[5].y));
  float d = fminf(fminf(x[6].x, x[6].y), fminf(x[7].x, x[7].y));
  return fminf(fminf(a, b), fminf(c, d));
}

// ------------------------------------------------------------ soft codeword
template <bool ARGMAX>
__global__ void __launch_bounds__(NT, 1) soft_kernel(Params P) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int mid = tid >> 1, e = tid & 1;
  const int n = P.n;

  extern __shared__ __align__(16) float smem[];
  float* lb[2] = {smem, smem + J};                     // negated group vectors (ping-pong)
  float* rec = smem + 2 * J;                           // [2][32][8] per-warp partials
  int* arec = reinterpret_cast<int*>(rec + 2 * 32 * 8);  // [2][32] argmax index
  uint32_t* tslot = reinterpret_cast<uint32_t*>(arec + 64);  // [4]
  float* wsc = reinterpret_cast<float*>(tslot + 4);    // [n][2]: -w'

  float* hist = P.hist_l + (size_t)blockIdx.x * n * J;
  double* hist_c = P.hist_c + (size_t)blockIdx.x * n;
  const float2* __restrict__ cf1 = P.cf1 + tid;
  const float2* __restrict__ cb1 = P.cb1 + tid;
  const float2 neg1 = f2s(-1.f);
  const int hoff = mid * 16 + 8 * e;                   // this thread's 8 entries of a history step

  // tensor memory: component 0 of the codewords of the thread's groups of the
  // current direction (128 columns), component 1 streams from L2
  if (warp == 0) l16::tmem_alloc512(tslot);
  l16::tmem_fence_before();
  __syncthreads();
  l16::tmem_fence_after();
  const uint32_t tbase = tslot[0] + ((uint32_t)(32 * (warp & 3)) << 16) + (uint32_t)(128 * (warp >> 2));

  for (int64_t seq = blockIdx.x; seq < P.n_seq; seq += gridDim.x) {
    const float* wq = P.w + seq * P.len;
    for (int x = tid; x < 2 * n; x += NT) wsc[x] = -wq[x] * P.sk;
    stage_c0(P.cf + tid, tbase);
    __syncthreads();

    // ------------------------------------------------------------ forward
    float Rn = 0.f;
    double C = 0.0;
    for (int t = 0; t < n; ++t) {
      const float* nprev = lb[(t + 1) & 1];
      float* ncur = lb[t & 1];
      const float2 nw0 = f2s(wsc[2 * t]), nw1 = f2s(wsc[2 * t + 1]);
      C -= (double)Rn;
      float np[16];
      if (t == 0) {
#pragma unroll
        for (int h = 0; h < 16; ++h) np[h] = 0.f;
      } else {
#pragma unroll
        for (int h = 0; h < 16; ++h) np[h] = nprev[(h << 8) | mid];
        float4* hd = reinterpret_cast<float4*>(hist + (size_t)(t - 1) * J + hoff);
        hd[0] = make_float4(pick8(np, e, 0), pick8(np, e, 1), pick8(np, e, 2), pick8(np, e, 3));
        hd[1] = make_float4(pick8(np, e, 4), pick8(np, e, 5), pick8(np, e, 6), pick8(np, e, 7));
      }
      float out[G];
      float tmin = INFINITY;
#pragma unroll
      for (int k = 0; k < G; ++k) {
        float2 x[8];
        float c0v[16];
        l16::tmem_ld16(tbase + 16 * k, c0v);
#pragma unroll
        for (int p = 0; p < 8; ++p) {
          const float2 c1 = __ldg(cf1 + (k * 8 + p) * NT);
          const float2 d0 = __fadd2_rn(f2(c0v[2 * p], c0v[2 * p + 1]), nw0), d1 = __fadd2_rn(c1, nw1);
          x[p] = __ffma2_rn(d1, d1, __ffma2_rn(d0, d0, f2(np[2 * p], np[2 * p + 1])));
        }
        const float m = min16(x);
        float2 s = f2s(0.f);
#pragma unroll
        for (int p = 0; p < 8; ++p) {
          const float2 a = __ffma2_rn(x[p], neg1, f2s(m));
          s = __fadd2_rn(s, f2(ex2f(a.x), ex2f(a.y)));
        }
        out[k] = (m - Rn) - lg2f(s.x + s.y);
        tmin = fminf(tmin, out[k]);
      }
      reinterpret_cast<float4*>(ncur + hoff)[0] = make_float4(out[0], out[1], out[2], out[3]);
      reinterpret_cast<float4*>(ncur + hoff)[1] = make_float4(out[4], out[5], out[6], out[7]);
      tmin = -warp_max(-tmin);
      if (lane == 0) rec[((t & 1) * 32 + warp) * 8] = tmin;
      if (tid == 0) hist_c[t] = C;
      __syncthreads();
      Rn = bfly16_min(rec[((t & 1) * 32 + (lane & 15)) * 8]);
    }
    // log2 Z = -Rn + log2 sum_j 2^(Rn - stored_j) + C
    double l2Z;
    {
      const float* nfin = lb[(n - 1) & 1];
      float s0 = 0.f;
      for (int j = tid; j < J; j += NT) s0 += ex2f(Rn - nfin[j]);
      s0 = warp_sum(s0);
      if (lane == 0) rec[warp * 8 + 1] = s0;
      __syncthreads();
      const float a0 = bfly16_sum(rec[(lane & 15) * 8 + 1]);
      l2Z = -(double)Rn + log2((double)a0) + C;
      if (tid == 0 && P.out_logZ) P.out_logZ[seq] = (float)(l2Z * 0.69314718055994530942);
      __syncthreads();
    }

    // ------------------------------------------------------------ backward
    stage_c0(P.cb + tid, tbase);
    float Rrn = 0.f;
    double Cr = 0.0;
    float4 hsa = make_float4(0.f, 0.f, 0.f, 0.f), hsb = hsa;
    if (n >= 2) {
      hsa = reinterpret_cast<const float4*>(hist + (size_t)(n - 2) * J + hoff)[0];
      hsb = reinterpret_cast<const float4*>(hist + (size_t)(n - 2) * J + hoff)[1];
    }
    for (int t = n - 1; t >= 0; --t) {
      const float* ncur = lb[t & 1];
      float* nnext = lb[(t + 1) & 1];
      const float2 nw0 = f2s(wsc[2 * t]), nw1 = f2s(wsc[2 * t + 1]);
      const double Csig = (t >= 1) ? hist_c[t - 1] : 0.0;
      const float K = (float)(Csig + Cr - l2Z);
      const bool last = (t == n - 1);
      const float hs[G] = {hsa.x, hsa.y, hsa.z, hsa.w, hsb.x, hsb.y, hsb.z, hsb.w};
      if (t >= 2) {   // next step's history
        hsa = reinterpret_cast<const float4*>(hist + (size_t)(t - 2) * J + hoff)[0];
        hsb = reinterpret_cast<const float4*>(hist + (size_t)(t - 2) * J + hoff)[1];
      } else {
        hsa = hsb = make_float4(0.f, 0.f, 0.f, 0.f);
      }
      float nr[16];
      if (last) {
#pragma unroll
        for (int lo = 0; lo < 16; ++lo) nr[lo] = 0.f;
      } else {
#pragma unroll
        for (int v4 = 0; v4 < 4; ++v4) {
          const float4 r = reinterpret_cast<const float4*>(ncur + mid * 16)[v4];
          nr[4 * v4] = r.x; nr[4 * v4 + 1] = r.y; nr[4 * v4 + 2] = r.z; nr[4 * v4 + 3] = r.w;
        }
      }
      float2 acc0 = f2s(0.f), acc1 = f2s(0.f), accp = f2s(0.f);
      float bestp = -1.f;
      int bestq = 0x7fffffff;
      float nout[G];
      float tmin = INFINITY;
#pragma unroll
      for (int k = 0; k < G; ++k) {            // group (h = 8e + k, mid), members lo
        float2 y[8], c0[8], c1[8];
        float c0v[16];
        l16::tmem_ld16(tbase + 16 * k, c0v);
#pragma unroll
        for (int p = 0; p < 8; ++p) {
          c0[p] = f2(c0v[2 * p], c0v[2 * p + 1]);
          c1[p] = __ldg(cb1 + (k * 8 + p) * NT);
          const float2 d0 = __fadd2_rn(c0[p], nw0), d1 = __fadd2_rn(c1[p], nw1);
          y[p] = __ffma2_rn(d1, d1, __ffma2_rn(d0, d0, f2(nr[2 * p], nr[2 * p + 1])));
        }
        // the posterior directly, p = 2^(K - n_sigma - y'), one ex2 per state
        const float kh = K - hs[k];
        float2 s = f2s(0.f);
#pragma unroll
        for (int p = 0; p < 8; ++p) {
          const float2 a = __ffma2_rn(y[p], neg1, f2s(kh));
          const float2 pp = f2(ex2f(a.x), ex2f(a.y));
          s = __fadd2_rn(s, pp);
          acc0 = __ffma2_rn(pp, c0[p], acc0);
          acc1 = __ffma2_rn(pp, c1[p], acc1);
          if constexpr (ARGMAX) {
            const int q = ((8 * e + k) << 12) | (mid << 4) | (2 * p);
            arg_better(bestp, bestq, pp.x, q);
            arg_better(bestp, bestq, pp.y, q + 1);
          }
        }
        accp = __fadd2_rn(accp, s);
        // negated log rho_{t-1}; +inf (rho = 0) when the group's posterior mass underflows
        nout[k] = (kh - Rrn) - lg2f(s.x + s.y);
        tmin = fminf(tmin, nout[k]);
      }
      if (t >= 1) {
#pragma unroll
        for (int k = 0; k < G; ++k) nnext[((8 * e + k) << 8) | mid] = nout[k];
      } else {
        tmin = INFINITY;
      }
      const float a0 = warp_sum(acc0.x + acc0.y);
      const float a1 = warp_sum(acc1.x + acc1.y);
      const float a2 = warp_sum(accp.x + accp.y);
      tmin = -warp_max(-tmin);
      if constexpr (ARGMAX) warp_argmax(bestp, bestq);
      const int pb = t & 1;
      if (lane == 0) {
        float* r = rec + (pb * 32 + warp) * 8;
        r[0] = tmin; r[1] = a0; r[2] = a1; r[3] = a2;
        if constexpr (ARGMAX) { r[4] = bestp; arec[pb * 32 + warp] = bestq; }
      }
      __syncthreads();
      if (tid == 0) {
        float s0 = 0.f, s1 = 0.f, s2 = 0.f;
#pragma unroll
        for (int w2 = 0; w2 < NT / 32; ++w2) {
          const float* r = rec + (pb * 32 + w2) * 8;
          s0 += r[1]; s1 += r[2]; s2 += r[3];
        }
        check_posterior_mass(s2);
        if (P.out_soft) {
          const float inv = 1.f / (s2 * P.sk);
          P.out_soft[seq * P.len + 2 * t] = s0 * inv;
          P.out_soft[seq * P.len + 2 * t + 1] = s1 * inv;
        }
        if constexpr (ARGMAX) {
          float bp = -1.f;
          int bq = 0x7fffffff;
#pragma unroll
          for (int w2 = 0; w2 < NT / 32; ++w2) arg_better(bp, bq, rec[(pb * 32 + w2) * 8 + 4], arec[pb * 32 + w2]);
          if (P.out_argmax) P.out_argmax[seq * n + t] = bq;
        }
      }
      Cr -= (double)Rrn;
      Rrn = bfly16_min(rec[(pb * 32 + (lane & 15)) * 8]);
    }
    __syncthreads();
  }

  l16::tmem_fence_before();
  __syncthreads();
  l16::tmem_fence_after();
  if (warp == 0) l16::tmem_dealloc512(tslot[0]);
}

// ------------------------------------------------------------ VJP
// Forward: negated log sigma and the prefix expectation A (both vectors in the
// shared-memory ping-pong; A_{t-1} enters relative to its value at group 0).
// Backward: negated log rho, the suffix expectation Bc (relative to the
// posterior mean of the previous step's stored values), G, dl/dw per step and
// the per-state codebook gradient; the centring constant K_t and the posterior
// sum of every step are formed one step early from the same stored values, and
// the log of the posterior sum renormalises the next step (see bcjr_l16.cuh).
__global__ void __launch_bounds__(NT, 1) vjp_kernel(Params P) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int mid = tid >> 1, e = tid & 1;
  const int n = P.n;

  extern __shared__ __align__(16) float smem[];
  float* lb[2] = {smem, smem + J};                     // negated sigma / rho (ping-pong)
  float* ab[2] = {smem + 2 * J, smem + 3 * J};         // A / Bc (ping-pong)
  // per-warp partials of a step, [2][32][8]:
  //   0: sum P(i) (A + Bc)  1: sum P(i) Bc  2: sum P(i)  3: min stored value
  //   4: sum G (c0' - w0')  5: sum G (c1' - w1')
  float* rec = smem + 4 * J;
  uint32_t* tslot = reinterpret_cast<uint32_t*>(rec + 2 * 32 * 8);  // [4]
  float* wsc = reinterpret_cast<float*>(tslot + 4);    // [n][2]: -w'
  float* gsc = wsc + 2 * n;                            // [n][2]: g / sk

  float* hist_l = P.hist_l + (size_t)blockIdx.x * n * J;
  float* hist_a = P.hist_a + (size_t)blockIdx.x * n * J;
  double* hist_c = P.hist_c + (size_t)blockIdx.x * n;
  float4* gc1 = P.gc1 + (size_t)blockIdx.x * (G * 4 * NT) + tid;
  double* gcp = P.gc_part + (size_t)blockIdx.x * 2 * S;
  const float2* __restrict__ cf1 = P.cf1 + tid;
  const float4* __restrict__ cb = P.cb + tid;
  const float2 neg1 = f2s(-1.f);
  const int hoff = mid * 16 + 8 * e;

  if (warp == 0) l16::tmem_alloc512(tslot);
  l16::tmem_fence_before();
  __syncthreads();
  l16::tmem_fence_after();
  // this thread's 128 columns: component 0 of the gradient of its backward
  // states, column 16 k + lo for group (h = 8e + k, mid)
  const uint32_t tbase = tslot[0] + ((uint32_t)(32 * (warp & 3)) << 16) + (uint32_t)(128 * (warp >> 2));
  for (int x = tid; x < 2 * S; x += NT) gcp[x] = 0.0;

  for (int64_t seq = blockIdx.x; seq < P.n_seq; seq += gridDim.x) {
    const float* wq = P.w + seq * P.len;
    const float* gq = P.gsoft + seq * P.len;
    for (int x = tid; x < 2 * n; x += NT) { wsc[x] = -wq[x] * P.sk; gsc[x] = gq[x] / P.sk; }
    stage_c0(P.cf + tid, tbase);   // the forward's component 0 (the backward's gradient later)
    __syncthreads();

    // ------------------------------------------------------------ forward
    float Rn = 0.f;
    double C = 0.0;
    for (int t = 0; t < n; ++t) {
      const float* nprev = lb[(t + 1) & 1];
      float* ncur = lb[t & 1];
      const float* aprev = ab[(t + 1) & 1];
      float* acur = ab[t & 1];
      const float2 nw0 = f2s(wsc[2 * t]), nw1 = f2s(wsc[2 * t + 1]);
      const float2 g0 = f2s(gsc[2 * t]), g1 = f2s(gsc[2 * t + 1]);
      C -= (double)Rn;
      float np[16], ap[16];
      if (t == 0) {
#pragma unroll
        for (int h = 0; h < 16; ++h) { np[h] = 0.f; ap[h] = 0.f; }
      } else {
#pragma unroll
        for (int h = 0; h < 16; ++h) { np[h] = nprev[(h << 8) | mid]; ap[h] = aprev[(h << 8) | mid]; }
        float4* hd = reinterpret_cast<float4*>(hist_l + (size_t)(t - 1) * J + hoff);
        hd[0] = make_float4(pick8(np, e, 0), pick8(np, e, 1), pick8(np, e, 2), pick8(np, e, 3));
        hd[1] = make_float4(pick8(np, e, 4), pick8(np, e, 5), pick8(np, e, 6), pick8(np, e, 7));
        float4* ad = reinterpret_cast<float4*>(hist_a + (size_t)(t - 1) * J + hoff);
        ad[0] = make_float4(pick8(ap, e, 0), pick8(ap, e, 1), pick8(ap, e, 2), pick8(ap, e, 3));
        ad[1] = make_float4(pick8(ap, e, 4), pick8(ap, e, 5), pick8(ap, e, 6), pick8(ap, e, 7));
        // A_{t-1} relative to its value at group 0; the backward subtracts the same
        const float rA = aprev[0];
#pragma unroll
        for (int h = 0; h < 16; ++h) ap[h] -= rA;
      }
      float tmin = INFINITY;
#pragma unroll 1
      for (int k = 0; k < G; ++k) {
        float2 x[8], z[8];
        float c0v[16];
        l16::tmem_ld16(tbase + 16 * k, c0v);
#pragma unroll
        for (int p = 0; p < 8; ++p) {
          const float2 c0 = f2(c0v[2 * p], c0v[2 * p + 1]), c1 = __ldg(cf1 + (k * 8 + p) * NT);
          const float2 d0 = __fadd2_rn(c0, nw0), d1 = __fadd2_rn(c1, nw1);
          x[p] = __ffma2_rn(d1, d1, __ffma2_rn(d0, d0, f2(np[2 * p], np[2 * p + 1])));
          z[p] = __ffma2_rn(g1, c1, __ffma2_rn(g0, c0, f2(ap[2 * p], ap[2 * p + 1])));
        }
        const float m = min16(x);
        float2 s = f2s(0.f), num = f2s(0.f);
#pragma unroll
        for (int p = 0; p < 8; ++p) {
          const float2 a = __ffma2_rn(x[p], neg1, f2s(m));
          const float2 u = f2(ex2f(a.x), ex2f(a.y));
          s = __fadd2_rn(s, u);
          num = __ffma2_rn(u, z[p], num);
        }
        const float ss = s.x + s.y;
        const float o = (m - Rn) - lg2f(ss);
        ncur[hoff + k] = o;
        acur[hoff + k] = __fdividef(num.x + num.y, ss);
        tmin = fminf(tmin, o);
      }
      tmin = -warp_max(-tmin);
      if (lane == 0) rec[((t & 1) * 32 + warp) * 8 + 3] = tmin;
      if (tid == 0) hist_c[t] = C;
      __syncthreads();
      Rn = bfly16_min(rec[((t & 1) * 32 + (lane & 15)) * 8 + 3]);
    }
    // the backward reads the histories through ordinary loads after barriers
    // log2 Z and Hbar = E[A_{n-1}]
    double l2Z;
    float Hbar;
    {
      const float* nfin = lb[(n - 1) & 1];
      const float* afin = ab[(n - 1) & 1];
      float s0 = 0.f, s1 = 0.f;
      for (int j = tid; j < J; j += NT) {
        const float u = ex2f(Rn - nfin[j]);
        s0 += u;
        s1 = fmaf(u, afin[j], s1);
      }
      s0 = warp_sum(s0);
      s1 = warp_sum(s1);
      if (lane == 0) { rec[warp * 8 + 4] = s0; rec[warp * 8 + 5] = s1; }
      __syncthreads();
      const float a0 = bfly16_sum(rec[(lane & 15) * 8 + 4]);
      const float a1 = bfly16_sum(rec[(lane & 15) * 8 + 5]);
      l2Z = -(double)Rn + log2((double)a0) + C;
      Hbar = a1 / a0;
      __syncthreads();
    }
    const float gzq = P.gZ ? P.gZ[seq] : 0.f;
    const float2 nc2T = f2s(-P.two_over_T / P.sk);

    // this sequence's codebook gradient starts at 0
    {
      float z16[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) z16[i] = 0.f;
#pragma unroll
      for (int k = 0; k < G; ++k) l16::tmem_st16(tbase + 16 * k, z16);
      l16::tmem_wait_st();
#pragma unroll
      for (int x = 0; x < G * 4; ++x) gc1[x * NT] = make_float4(0.f, 0.f, 0.f, 0.f);
    }

    // ------------------------------------------------------------ backward
    float Rrn = 0.f;
    double Cr = 0.0;
    float Kt = Hbar, rB = 0.f;
    for (int t = n - 1; t >= 0; --t) {
      const float* ncur = lb[t & 1];
      float* nnext = lb[(t + 1) & 1];
      const float* bcur = ab[t & 1];
      float* bnext = ab[(t + 1) & 1];
      const float2 nw0 = f2s(wsc[2 * t]), nw1 = f2s(wsc[2 * t + 1]);
      const float2 g0 = f2s(gsc[2 * t]), g1 = f2s(gsc[2 * t + 1]);
      const float2 gr0 = f2s(gsc[2 * t] * P.sk), gr1 = f2s(gsc[2 * t + 1] * P.sk);
      const double Csig = (t >= 1) ? hist_c[t - 1] : 0.0;
      const float K = (float)(Csig + Cr - l2Z);
      const bool last = (t == n - 1);
      // step t-1's sigma and A of this thread's groups (free start: 0 for t = 0)
      const float* hsp = hist_l + (size_t)(t >= 1 ? t - 1 : 0) * J + hoff;
      const float* hap = hist_a + (size_t)(t >= 1 ? t - 1 : 0) * J + hoff;
      const float rA = (t >= 1) ? hist_a[(size_t)(t - 1) * J] : 0.f;   // the forward's reference (group 0)
      const float hbt = Kt + rA - rB - gzq;   // G = p (A + h + (Bc - rB) - hbt)
      float nr[16], bc[16];
      if (last) {
#pragma unroll
        for (int lo = 0; lo < 16; ++lo) { nr[lo] = 0.f; bc[lo] = 0.f; }
      } else {
#pragma unroll
        for (int v4 = 0; v4 < 4; ++v4) {
          const float4 r = reinterpret_cast<const float4*>(ncur + mid * 16)[v4];
          const float4 b = reinterpret_cast<const float4*>(bcur + mid * 16)[v4];
          nr[4 * v4] = r.x; nr[4 * v4 + 1] = r.y; nr[4 * v4 + 2] = r.z; nr[4 * v4 + 3] = r.w;
          bc[4 * v4] = b.x - rB; bc[4 * v4 + 1] = b.y - rB; bc[4 * v4 + 2] = b.z - rB; bc[4 * v4 + 3] = b.w - rB;
        }
      }
      float2 accG0 = f2s(0.f), accG1 = f2s(0.f);
      float accK = 0.f, accB = 0.f, accP = 0.f;
      float tmin = INFINITY;
#pragma unroll 1
      for (int k = 0; k < G; ++k) {            // group (h = 8e + k, mid), members lo
        const float hsk = (t >= 1) ? hsp[k] : 0.f, hak = (t >= 1) ? hap[k] : 0.f;
        float2 y[8];
#pragma unroll
        for (int p = 0; p < 8; ++p) {
          const float4 cw = __ldg(cb + (k * 8 + p) * NT);
          const float2 d0 = __fadd2_rn(f2(cw.x, cw.y), nw0), d1 = __fadd2_rn(f2(cw.z, cw.w), nw1);
          y[p] = __ffma2_rn(d1, d1, __ffma2_rn(d0, d0, f2(nr[2 * p], nr[2 * p + 1])));
        }
        // the posterior directly, p = 2^(K - n_sigma - y'), one ex2 per state
        const float kh = K - hsk;
        const float2 ah = f2s(hak - hbt);             // A - K + gZ
        float2 s = f2s(0.f), num = f2s(0.f);
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {           // members lo = 8 hf .. 8 hf + 7
        float gcb0[8];
        l16::tmem_ld8(tbase + 16 * k + 8 * hf, gcb0);
        float4 g1v[2];
#pragma unroll
        for (int j = 0; j < 2; ++j) g1v[j] = gc1[(k * 4 + 2 * hf + j) * NT];
#pragma unroll
        for (int pl = 0; pl < 4; ++pl) {
          const int p = 4 * hf + pl;
          const float4 cw = __ldg(cb + (k * 8 + p) * NT);
          const float2 c0 = f2(cw.x, cw.y), c1 = f2(cw.z, cw.w);
          const float2 a = __ffma2_rn(y[p], neg1, f2s(kh));
          const float2 pp = f2(ex2f(a.x), ex2f(a.y));
          s = __fadd2_rn(s, pp);
          const float2 z = __ffma2_rn(g1, c1, __ffma2_rn(g0, c0, f2(bc[2 * p], bc[2 * p + 1])));   // Bc + h
          num = __ffma2_rn(pp, z, num);
          const float2 Gp = __fmul2_rn(pp, __fadd2_rn(z, ah));
          const float2 Gd0 = __fmul2_rn(Gp, __fadd2_rn(c0, nw0));   // G (c0' - w0')
          const float2 Gd1 = __fmul2_rn(Gp, __fadd2_rn(c1, nw1));
          accG0 = __fadd2_rn(accG0, Gd0);
          accG1 = __fadd2_rn(accG1, Gd1);
          float2 q0 = f2(gcb0[2 * pl], gcb0[2 * pl + 1]);
          q0 = __ffma2_rn(Gd0, nc2T, __ffma2_rn(gr0, pp, q0));       // + g p + (2/T) G (w - c)
          gcb0[2 * pl] = q0.x;
          gcb0[2 * pl + 1] = q0.y;
          float4& gv = g1v[pl >> 1];
          float2 q1 = (pl & 1) ? f2(gv.z, gv.w) : f2(gv.x, gv.y);
          q1 = __ffma2_rn(Gd1, nc2T, __ffma2_rn(gr1, pp, q1));
          if (pl & 1) { gv.z = q1.x; gv.w = q1.y; } else { gv.x = q1.x; gv.y = q1.y; }
        }
        l16::tmem_st8(tbase + 16 * k + 8 * hf, gcb0);
#pragma unroll
        for (int j = 0; j < 2; ++j) gc1[(k * 4 + 2 * hf + j) * NT] = g1v[j];
        }
        const float ss = s.x + s.y;
        // negated log rho_{t-1} and Bc; a group whose posterior mass underflows gets
        // rho = 0 (+inf) and Bc = 0, moving no posterior by more than that mass
        const float nout = (kh - Rrn) - lg2f(ss);
        const float bout = __fdividef(num.x + num.y, fmaxf(ss, FLT_MIN));   // num = 0 when sum p = 0
        // posterior of the step t-1 group (h, mid): sum over its members of p
        const float pg = ss;
        accK = fmaf(pg, hak + bout, accK);
        accB = fmaf(pg, bout, accB);
        accP += pg;
        if (t >= 1) {
          nnext[((8 * e + k) << 8) | mid] = nout;
          bnext[((8 * e + k) << 8) | mid] = bout;
          tmin = fminf(tmin, nout);
        }
      }
      l16::tmem_wait_st();
      const float a0 = warp_sum(accG0.x + accG0.y);
      const float a1 = warp_sum(accG1.x + accG1.y);
      const float kk = warp_sum(accK);
      const float kb = warp_sum(accB);
      const float kp = warp_sum(accP);
      tmin = -warp_max(-tmin);
      const int pb = t & 1;
      if (lane == 0) {
        float* r = rec + (pb * 32 + warp) * 8;
        *reinterpret_cast<float4*>(r) = make_float4(kk, kb, kp, tmin);
        r[4] = a0;
        r[5] = a1;
      }
      __syncthreads();
      if (tid == 0) {
        float s0 = 0.f, s1 = 0.f;
#pragma unroll
        for (int w2 = 0; w2 < NT / 32; ++w2) { s0 += rec[(pb * 32 + w2) * 8 + 4]; s1 += rec[(pb * 32 + w2) * 8 + 5]; }
        // dl/dw_{t,v} = (2/T) sum_q G (c_v - w_v) = (2/T) sum_q G (c_v' - w_v') / sk
        P.grad_w[seq * P.len + 2 * t] = P.two_over_T * s0 / P.sk;
        P.grad_w[seq * P.len + 2 * t + 1] = P.two_over_T * s1 / P.sk;
      }
      Cr -= (double)Rrn;
      {
        const float4 r = *reinterpret_cast<const float4*>(rec + (pb * 32 + (lane & 15)) * 8);
        const float sp = bfly16_sum(r.z);   // sum_q p_t(q), 1 up to rounding
        Kt = bfly16_sum(r.x) / sp;
        rB = bfly16_sum(r.y) / sp;
        if (tid == 0) check_posterior_mass(sp);
        Rrn = bfly16_min(r.w);
        // renormalise the next step's posterior (the drift of the posterior sum)
        Cr -= (double)lg2f(sp);
      }
    }

    // fold this sequence's codebook gradient into the CTA partial [q][v]
#pragma unroll
    for (int k = 0; k < G; ++k) {
      float gcb0[16];
      l16::tmem_ld16(tbase + 16 * k, gcb0);
      const int qb = ((8 * e + k) << 12) | (mid << 4);
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const float4 v = gc1[(k * 4 + j) * NT];
        double2* d = reinterpret_cast<double2*>(gcp + 2 * (qb + 4 * j));
        double2 x0 = d[0], x1 = d[1], x2 = d[2], x3 = d[3];
        x0.x += (double)gcb0[4 * j];     x0.y += (double)v.x;
        x1.x += (double)gcb0[4 * j + 1]; x1.y += (double)v.y;
        x2.x += (double)gcb0[4 * j + 2]; x2.y += (double)v.z;
        x3.x += (double)gcb0[4 * j + 3]; x3.y += (double)v.w;
        d[0] = x0; d[1] = x1; d[2] = x2; d[3] = x3;
      }
    }
    __syncthreads();
  }

  l16::tmem_fence_before();
  __syncthreads();
  l16::tmem_fence_after();
  if (warp == 0) l16::tmem_dealloc512(tslot[0]);
}

// ------------------------------------------------------------ Viterbi
// The T -> 0 decode in the same layout: per step and forward group
// j = (mid << 4) | lo, mu_t(j) = min_h delta_t((h << 12) | j) with
// delta_t(q) = fl(mu_{t-1}(q >> 4) + cost_t(q)) (delta_0 = cost_0) and
// cost_t(q) = fl(fl(fl(w0 - c0)^2) + fl(fl(w1 - c1)^2)), the lowest h winning
// ties.  All of a thread's 8 groups read the same 16 predecessor values
// mu_{t-1}((h << 8) | mid), once per step.  Component 0 of the raw codewords
// sits in tensor memory (the thread's 128 states = its 128 columns),
// component 1 streams from the forward-order copy in L2.  The 4-bit
// backpointers of a thread's 8 groups form one 32-bit word per step.  A CTA
// decodes a batch of up to TB sequences, then traces them back in parallel
// (one thread per sequence).  The arithmetic is the prescribed fp32 sequence
// in scalar IEEE round-to-nearest operations that are never fused.
struct VParams {
  const float* w;        // [n_seq][len], len = 2 n
  const float4* cf;      // forward-order raw codebook (make_codebooks with scale 1)
  const float2* cf1;     // its component 1
  int32_t* out_states;   // [n_seq][n]
  float* out_cost;       // [n_seq] or null
  uint32_t* bp;          // [grid][TB][n][NT]
  int64_t n_seq, len;
  int n, tb;
};

__global__ void __launch_bounds__(NT, 1) viterbi_kernel(VParams P) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  constexpr int nwarps = NT / 32;
  const int n = P.n, TB = P.tb;
  const int mid = tid >> 1, e = tid & 1;
  extern __shared__ __align__(16) float smem[];
  float* mb[2] = {smem, smem + J};
  float* redv = smem + 2 * J;                          // [32]
  int* redq = reinterpret_cast<int*>(redv + 32);       // [32]
  int* fin = redq + 32;                                // [TB <= 64] final state per sequence of the batch
  uint32_t* tslot = reinterpret_cast<uint32_t*>(fin + 64);  // [4]
  float* wsm = reinterpret_cast<float*>(tslot + 4);    // 2 n: w
  uint32_t* bp = P.bp + (size_t)blockIdx.x * TB * n * NT;

  if (warp == 0) l16::tmem_alloc512(tslot);
  l16::tmem_fence_before();
  __syncthreads();
  l16::tmem_fence_after();
  const uint32_t tbase = tslot[0] + ((uint32_t)(32 * (warp & 3)) << 16) + (uint32_t)(128 * (warp >> 2));
  stage_c0(P.cf + tid, tbase);
  const float2* __restrict__ c1p = P.cf1 + tid;

  const int64_t stride = (int64_t)gridDim.x;
  for (int64_t base = blockIdx.x; base < P.n_seq; base += stride * TB) {
    int nb = 0;
    for (int i = 0; i < TB; ++i, ++nb) {
      const int64_t seq = base + i * stride;
      if (seq >= P.n_seq) break;
      const float* wq = P.w + seq * P.len;
      for (int x = tid; x < 2 * n; x += NT) wsm[x] = wq[x];
      __syncthreads();
      uint32_t* bpi = bp + (size_t)i * n * NT;
      float bestv = INFINITY;
      int bestq = 0x7fffffff;
      for (int t = 0; t < n; ++t) {
        const float* mprev = mb[(t + 1) & 1];
        float* mcur = mb[t & 1];
        const float w0 = wsm[2 * t], w1 = wsm[2 * t + 1];
        const bool last = (t == n - 1);
        float mu[16];
#pragma unroll
        for (int h = 0; h < 16; ++h) mu[h] = (t > 0) ? mprev[(h << 8) | mid] : 0.f;
        float2 c1n[8];
#pragma unroll
        for (int p = 0; p < 8; ++p) c1n[p] = __ldg(c1p + p * NT);
        float mout[G];
        uint32_t word = 0;
#pragma unroll
        for (int k = 0; k < G; ++k) {
          float c0[16];
          l16::tmem_ld16(tbase + 16 * k, c0);
          float2 c1[8];
#pragma unroll
          for (int p = 0; p < 8; ++p) c1[p] = c1n[p];
          if (k + 1 < G) {
#pragma unroll
            for (int p = 0; p < 8; ++p) c1n[p] = __ldg(c1p + ((k + 1) * 8 + p) * NT);
          }
          float b = INFINITY;
          uint32_t bh = 0;
#pragma unroll
          for (int h = 0; h < 16; ++h) {
            const float d0 = __fsub_rn(w0, c0[h]);
            const float d1 = __fsub_rn(w1, (h & 1) ? c1[h >> 1].y : c1[h >> 1].x);
            const float q = __fadd_rn(__fmul_rn(d0, d0), __fmul_rn(d1, d1));
            const float dl = (t > 0) ? __fadd_rn(mu[h], q) : q;
            if (dl < b) { b = dl; bh = (uint32_t)h; }
            if (last) {
              const int qs = (h << 12) | (mid << 4) | (8 * e + k);
              if (dl < bestv || (dl == bestv && qs < bestq)) { bestv = dl; bestq = qs; }
            }
          }
          mout[k] = b;
          word |= bh << (4 * k);
        }
        reinterpret_cast<float4*>(mcur + (mid << 4) + 8 * e)[0] = make_float4(mout[0], mout[1], mout[2], mout[3]);
        reinterpret_cast<float4*>(mcur + (mid << 4) + 8 * e)[1] = make_float4(mout[4], mout[5], mout[6], mout[7]);
        if (!last) bpi[(size_t)t * NT + tid] = word;
        __syncthreads();
      }
      // argmin of delta_{n-1} over all states, lowest state on ties
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        const float v2 = __shfl_xor_sync(0xffffffffu, bestv, o);
        const int q2 = __shfl_xor_sync(0xffffffffu, bestq, o);
        if (v2 < bestv || (v2 == bestv && q2 < bestq)) { bestv = v2; bestq = q2; }
      }
      if (lane == 0) { redv[warp] = bestv; redq[warp] = bestq; }
      __syncthreads();
      if (tid == 0) {
        float bv = INFINITY;
        int bq = 0x7fffffff;
#pragma unroll
        for (int w2 = 0; w2 < nwarps; ++w2)
          if (redv[w2] < bv || (redv[w2] == bv && redq[w2] < bq)) { bv = redv[w2]; bq = redq[w2]; }
        if (bq == 0x7fffffff) bq = 0;  // all-NaN sequence
        fin[i] = bq;
        if (P.out_cost) P.out_cost[seq] = bv;
      }
      __syncthreads();
    }
    // trace the batch back, one thread per sequence: the state at step t is
    // the backpointer's h of group s_{t+1} >> 4 at step t, above that group
    if (tid < nb) {
      const int i = tid;
      const int64_t seq = base + i * stride;
      const uint32_t* bpi = bp + (size_t)i * n * NT;
      int32_t* out = P.out_states + seq * n;
      int st = fin[i];
      for (int t = n - 1; t >= 0; --t) {
        out[t] = st;
        if (t > 0) {
          const int jp = st >> 4;   // group (mid' << 4) | lo' of the predecessors at step t-1
          const int tau = ((jp >> 4) << 1) | ((jp & 15) >> 3);
          const int h = (bpi[(size_t)(t - 1) * NT + tau] >> (4 * (jp & 7))) & 15;
          st = jp | (h << 12);
        }
      }
    }
    __syncthreads();
  }

  l16::tmem_fence_before();
  __syncthreads();
  l16::tmem_fence_after();
  if (warp == 0) l16::tmem_dealloc512(tslot[0]);
}

}  // namespace l16v2
}  // namespace bcjr
