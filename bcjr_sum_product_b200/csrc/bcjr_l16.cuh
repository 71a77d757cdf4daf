// Specialised sweep for the QTIP-scale trellis: L = 16 (65536 states),
// D = 2 bits per step (4 branches), V = 1 (scalar codewords), on sm_100a.
//
// Same mathematics as bcjr_kernels.cuh (predecessor-group recursions in base-2
// log domain; "BCJR-QAT: A Differentiable Relaxation of Trellis-Coded Weight
// Quantization", Abstract and Technical Summary "Core Mechanism"), with a
// layout chosen so that every reduction is thread-local:
//
//   state q = (h << 14) | (mid << 2) | lo,  h, lo in [0, 4), mid in [0, 4096).
//   The forward group j = q mod 2^14 = (mid << 2) | lo has members h = 0..3;
//   the backward group i = q >> 2 = (h << 12) | mid has members lo = 0..3.
//   A thread owns whole blocks (one mid, all 16 (h, lo)), so it forms both
//   kinds of groups from its own 16 codewords.  Per step it reads the four
//   group values (h << 12) | mid and writes the four values (mid << 2) | lo
//   (forward; mirrored in the backward); the 16384-entry group vector is
//   exchanged through shared memory.
//
//   512 threads; thread tau owns blocks mid = tau + 512 k, k = 0..7.
//   The scaled codebook is stored block-major: cs_tm[mid * 16 + 4 h + lo], so
//   a thread's 16 codewords of a block are one 64-byte line; it is the same
//   every step, so the next block's line is always prefetched.
//   VJP: the per-state codebook gradient of the current sequence lives in
//   tensor memory (512 columns x 128 lanes = 65536 fp32 = one per state),
//   warp w holding lanes 32 (w mod 4) .. + 31, columns 128 (w div 4) + 16 k.
#pragma once
#include "bcjr_kernels.cuh"

namespace bcjr {
namespace l16 {

constexpr int L = 16, D = 2, HB = 12;  // HB: bits of mid
constexpr int J = 1 << 14, NMID = 1 << 12, NT = 512, KB = NMID / NT;
constexpr int S = 1 << 16;

struct Params {
  const float* w;        // [n_seq][len]
  const float* cs_tm;    // block-major scaled codebook [4096][16]
  const float* gsoft;    // [n_seq][len] (VJP)
  const float* gZ;       // [n_seq] or null (VJP)
  float* out_soft;       // [n_seq][len] or null
  float* out_logZ;       // [n_seq] or null
  int32_t* out_argmax;   // [n_seq][n] or null
  float* grad_w;         // [n_seq][len] (VJP)
  double* gc_part;       // [grid][65536] block-major (VJP)
  float* hist_l;         // [grid][n][J]
  float* hist_a;         // [grid][n][J] (VJP)
  double* hist_c;        // [grid][n]
  float* bc_g;           // [grid][2][J] (VJP backward ping-pong)
  int64_t n_seq, len;
  int n;
  float sk, two_over_T;
};

// ------------------------------------------------------------ tensor memory
__device__ __forceinline__ uint32_t smem_addr(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ void tmem_alloc512(uint32_t* dst_smem) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], 512;" ::"r"(smem_addr(dst_smem)));
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
}
__device__ __forceinline__ void tmem_dealloc512(uint32_t taddr) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, 512;" ::"r"(taddr));
}
__device__ __forceinline__ void tmem_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tmem_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float (&r)[16]) {
  uint32_t u[16];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(u[0]), "=r"(u[1]), "=r"(u[2]), "=r"(u[3]), "=r"(u[4]), "=r"(u[5]), "=r"(u[6]), "=r"(u[7]), "=r"(u[8]),
        "=r"(u[9]), "=r"(u[10]), "=r"(u[11]), "=r"(u[12]), "=r"(u[13]), "=r"(u[14]), "=r"(u[15])
      : "r"(taddr)
      : "memory");
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < 16; ++i) r[i] = __uint_as_float(u[i]);
}
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const float (&r)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(
          taddr),
      "r"(__float_as_uint(r[0])), "r"(__float_as_uint(r[1])), "r"(__float_as_uint(r[2])), "r"(__float_as_uint(r[3])),
      "r"(__float_as_uint(r[4])), "r"(__float_as_uint(r[5])), "r"(__float_as_uint(r[6])), "r"(__float_as_uint(r[7])),
      "r"(__float_as_uint(r[8])), "r"(__float_as_uint(r[9])), "r"(__float_as_uint(r[10])),
      "r"(__float_as_uint(r[11])), "r"(__float_as_uint(r[12])), "r"(__float_as_uint(r[13])),
      "r"(__float_as_uint(r[14])), "r"(__float_as_uint(r[15]))
      : "memory");
}
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

__device__ __forceinline__ void ld_cb(const float* __restrict__ cs_tm, int mid, float (&c)[16]) {
  const float4* p = reinterpret_cast<const float4*>(cs_tm + (size_t)mid * 16);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    float4 v = __ldg(p + i);
    c[4 * i] = v.x; c[4 * i + 1] = v.y; c[4 * i + 2] = v.z; c[4 * i + 3] = v.w;
  }
}

// c_tm[mid * 16 + 4 h + lo] = sk * c[(h << 14) | (mid << 2) | lo]
__global__ void make_block_codebook(const float* __restrict__ c, float sk, float* __restrict__ cs_tm) {
  int x = blockIdx.x * blockDim.x + threadIdx.x;
  if (x >= S) return;
  const int mid = x >> 4, h = (x >> 2) & 3, lo = x & 3;
  cs_tm[x] = sk * c[(h << 14) | (mid << 2) | lo];
}

// grad_c[q] = sum over CTAs of gc_part[cta][block-major index of q]
__global__ void reduce_block_gc(const double* __restrict__ part, int nparts, float* __restrict__ out) {
  int q = blockIdx.x * blockDim.x + threadIdx.x;
  if (q >= S) return;
  const int h = q >> 14, mid = (q >> 2) & (NMID - 1), lo = q & 3;
  const size_t x = (size_t)mid * 16 + 4 * h + lo;
  double a = 0.0;
  for (int p = 0; p < nparts; ++p) a += part[(size_t)p * S + x];
  out[q] = (float)a;
}

template <int MODE>
__global__ void __launch_bounds__(NT, 1) sweep_kernel(Params P) {
  constexpr bool VJP = (MODE == MODE_VJP);
  constexpr int NP = 2;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  constexpr int nwarps = NT / 32;
  const int n = P.n;

  extern __shared__ __align__(16) float smem[];
  float* sb = smem;                                    // [2][J] state ping-pong (16-byte aligned)
  float* lb[2] = {sb, sb + J};
  float* wmax = sb + 2 * J;                            // [2][32]
  float* part = wmax + 64;                             // [2][32][NP]
  float* apart = part + 2 * 32 * NP;                   // [2][32]
  int* aidx = reinterpret_cast<int*>(apart + 64);      // [2][32]
  uint32_t* tslot = reinterpret_cast<uint32_t*>(aidx + 64);  // [4]
  float* wsc = reinterpret_cast<float*>(tslot + 4);    // n
  float* gsc = wsc + n;                                // n (VJP)

  float* hist_l = P.hist_l + (size_t)blockIdx.x * n * J;
  float* hist_a = VJP ? P.hist_a + (size_t)blockIdx.x * n * J : nullptr;
  double* hist_c = P.hist_c + (size_t)blockIdx.x * n;
  float* bcg[2] = {nullptr, nullptr};
  double* gcp = nullptr;
  if constexpr (VJP) {
    bcg[0] = P.bc_g + (size_t)blockIdx.x * 2 * J;
    bcg[1] = bcg[0] + J;
    gcp = P.gc_part + (size_t)blockIdx.x * S;
  }
  const float* __restrict__ cs_tm = P.cs_tm;

  uint32_t tbase = 0;
  if constexpr (VJP) {
    if (warp == 0) tmem_alloc512(tslot);
    tmem_fence_before();
    __syncthreads();
    tmem_fence_after();
    tbase = tslot[0] + ((uint32_t)(32 * (warp & 3)) << 16) + (uint32_t)(128 * (warp >> 2));
    float z16[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) z16[i] = 0.f;
#pragma unroll
    for (int k = 0; k < KB; ++k) tmem_st16(tbase + 16 * k, z16);
    tmem_wait_st();
    for (int x = tid; x < S; x += NT) gcp[x] = 0.0;
  }

  for (int64_t seq = blockIdx.x; seq < P.n_seq; seq += gridDim.x) {
    const float* wq = P.w + seq * P.len;
    for (int x = tid; x < n; x += NT) wsc[x] = wq[x] * P.sk;
    if constexpr (VJP) {
      const float* gq = P.gsoft + seq * P.len;
      for (int x = tid; x < n; x += NT) gsc[x] = gq[x] / P.sk;
    }
    __syncthreads();

    // ---------------------------------------------------------- forward
    float R = 0.f;
    double C = 0.0;
    float cbn[16];
    ld_cb(cs_tm, tid, cbn);
    for (int t = 0; t < n; ++t) {
      const float* lprev = lb[(t + 1) & 1];
      float* lcur = lb[t & 1];
      const float wt = wsc[t];
      const float gt = VJP ? gsc[t] : 0.f;
      const float* aprev = (VJP && t > 0) ? hist_a + (size_t)(t - 1) * J : nullptr;
      C += (double)R;
      float tmax = -INFINITY;
#pragma unroll
      for (int k = 0; k < KB; ++k) {
        const int mid = tid + NT * k;
        float cb[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) cb[i] = cbn[i];
        ld_cb(cs_tm, (k + 1 < KB) ? mid + NT : tid, cbn);
        float lsp[4], asp[4];
#pragma unroll
        for (int h = 0; h < 4; ++h) {
          lsp[h] = (t == 0) ? 0.f : lprev[(h << HB) | mid];
          if constexpr (VJP) asp[h] = (t == 0) ? 0.f : aprev[(h << HB) | mid];
        }
        float lout[4], aout[4];
#pragma unroll
        for (int lo = 0; lo < 4; ++lo) {
          float x[4];
          float m = -INFINITY;
#pragma unroll
          for (int h = 0; h < 4; ++h) {
            const float d = wt - cb[4 * h + lo];
            x[h] = fmaf(-d, d, lsp[h]);
            m = fmaxf(m, x[h]);
          }
          float s = 0.f, num = 0.f;
#pragma unroll
          for (int h = 0; h < 4; ++h) {
            const float u = ex2f(x[h] - m);
            s += u;
            if constexpr (VJP) num = fmaf(u, fmaf(gt, cb[4 * h + lo], asp[h]), num);
          }
          lout[lo] = m + lg2f(s) - R;
          if constexpr (VJP) aout[lo] = __fdividef(num, s);
          tmax = fmaxf(tmax, lout[lo]);
        }
        const float4 l4 = make_float4(lout[0], lout[1], lout[2], lout[3]);
        reinterpret_cast<float4*>(lcur)[mid] = l4;
        if (t < n - 1) reinterpret_cast<float4*>(hist_l + (size_t)t * J)[mid] = l4;
        if constexpr (VJP)
          reinterpret_cast<float4*>(hist_a + (size_t)t * J)[mid] = make_float4(aout[0], aout[1], aout[2], aout[3]);
      }
      tmax = warp_max(tmax);
      if (lane == 0) wmax[(t & 1) * 32 + warp] = tmax;
      if (tid == 0) hist_c[t] = C;
      __syncthreads();
      R = -INFINITY;
#pragma unroll
      for (int w2 = 0; w2 < nwarps; ++w2) R = fmaxf(R, wmax[(t & 1) * 32 + w2]);
    }

    // logZ, Hbar
    double l2Z;
    float Hbar = 0.f;
    {
      const float* lfin = lb[(n - 1) & 1];
      const float* afin = VJP ? hist_a + (size_t)(n - 1) * J : nullptr;
      float s0 = 0.f, s1 = 0.f;
      for (int j = tid; j < J; j += NT) {
        const float u = ex2f(lfin[j] - R);
        s0 += u;
        if constexpr (VJP) s1 = fmaf(u, afin[j], s1);
      }
      s0 = warp_sum(s0);
      if constexpr (VJP) s1 = warp_sum(s1);
      if (lane == 0) { part[warp * NP] = s0; part[warp * NP + 1] = s1; }
      __syncthreads();
      float a0 = 0.f, a1 = 0.f;
#pragma unroll
      for (int w2 = 0; w2 < nwarps; ++w2) { a0 += part[w2 * NP]; a1 += part[w2 * NP + 1]; }
      l2Z = (double)R + log2((double)a0) + C;
      if constexpr (VJP) Hbar = a1 / a0;
      if (MODE == MODE_SOFT && tid == 0 && P.out_logZ) P.out_logZ[seq] = (float)(l2Z * 0.69314718055994530942);
      __syncthreads();
    }
    const float gzq = (VJP && P.gZ) ? P.gZ[seq] : 0.f;
    const float hb = Hbar - gzq;
    const float c2T = P.two_over_T / P.sk;

    // ---------------------------------------------------------- backward
    float Rr = 0.f;
    double Cr = 0.0;
    ld_cb(cs_tm, tid, cbn);
    for (int t = n - 1; t >= 0; --t) {
      const float* rcur = lb[t & 1];
      float* rnext = lb[(t + 1) & 1];
      const float* bcur = VJP ? bcg[t & 1] : nullptr;
      float* bnext = VJP ? bcg[(t + 1) & 1] : nullptr;
      const float wt = wsc[t];
      const float gt = VJP ? gsc[t] : 0.f;
      const float graw = gt * P.sk;
      const double Csig = (t >= 1) ? hist_c[t - 1] : 0.0;
      const float K = (float)(Csig + Cr - l2Z);
      const bool last = (t == n - 1);
      const float* hl = (t > 0) ? hist_l + (size_t)(t - 1) * J : nullptr;
      const float* ha = (VJP && t > 0) ? hist_a + (size_t)(t - 1) * J : nullptr;
      float acc0 = 0.f, acc1 = 0.f;  // SOFT: sum p c, sum p; VJP: sum G c, sum G
      float bestp = -1.f;
      int bestq = 0x7fffffff;
      float tmax = -INFINITY;
#pragma unroll
      for (int k = 0; k < KB; ++k) {
        const int mid = tid + NT * k;
        float cb[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) cb[i] = cbn[i];
        ld_cb(cs_tm, (k + 1 < KB) ? mid + NT : tid, cbn);
        float r4[4], b4[4];
        if (last) {
#pragma unroll
          for (int lo = 0; lo < 4; ++lo) { r4[lo] = 0.f; b4[lo] = 0.f; }
        } else {
          const float4 rv = reinterpret_cast<const float4*>(rcur)[mid];
          r4[0] = rv.x; r4[1] = rv.y; r4[2] = rv.z; r4[3] = rv.w;
          if constexpr (VJP) {
            const float4 bv = reinterpret_cast<const float4*>(bcur)[mid];
            b4[0] = bv.x; b4[1] = bv.y; b4[2] = bv.z; b4[3] = bv.w;
          }
        }
        float gcb[16];
        if constexpr (VJP) tmem_ld16(tbase + 16 * k, gcb);
#pragma unroll
        for (int h = 0; h < 4; ++h) {
          const int gi = (h << HB) | mid;
          const float lsig = (t >= 1) ? hl[gi] : 0.f;
          float asig = 0.f;
          if constexpr (VJP) asig = (t >= 1) ? ha[gi] : 0.f;
          float y[4], z[4];
          float m = -INFINITY;
#pragma unroll
          for (int lo = 0; lo < 4; ++lo) {
            const float d = wt - cb[4 * h + lo];
            y[lo] = fmaf(-d, d, r4[lo]);
            m = fmaxf(m, y[lo]);
            if constexpr (VJP) z[lo] = fmaf(gt, cb[4 * h + lo], b4[lo]);
          }
          const float gf = ex2f(m + lsig + K);
          float s = 0.f, num = 0.f;
#pragma unroll
          for (int lo = 0; lo < 4; ++lo) {
            const float u = ex2f(y[lo] - m);
            s += u;
            const float p = u * gf;
            if constexpr (MODE == MODE_SOFT) {
              acc0 = fmaf(p, cb[4 * h + lo], acc0);
              acc1 += p;
              const int q = (h << 14) | (mid << 2) | lo;
              arg_better(bestp, bestq, p, q);
            } else {
              num = fmaf(u, z[lo], num);
              const float G = p * (asig + z[lo] - hb);
              acc1 += G;
              acc0 = fmaf(G, cb[4 * h + lo], acc0);
              const float d = wt - cb[4 * h + lo];
              gcb[4 * h + lo] = fmaf(c2T, G * d, fmaf(graw, p, gcb[4 * h + lo]));
            }
          }
          if (t >= 1) {
            const float l = m + lg2f(s) - Rr;
            rnext[gi] = l;
            tmax = fmaxf(tmax, l);
            if constexpr (VJP) bnext[gi] = __fdividef(num, s);
          }
        }
        if constexpr (VJP) tmem_st16(tbase + 16 * k, gcb);
      }
      if constexpr (VJP) tmem_wait_st();
      acc0 = warp_sum(acc0);
      acc1 = warp_sum(acc1);
      tmax = warp_max(tmax);
      if (MODE == MODE_SOFT) warp_argmax(bestp, bestq);
      const int pb = t & 1;
      if (lane == 0) {
        part[(pb * 32 + warp) * NP] = acc0;
        part[(pb * 32 + warp) * NP + 1] = acc1;
        wmax[pb * 32 + warp] = tmax;
        apart[pb * 32 + warp] = bestp;
        aidx[pb * 32 + warp] = bestq;
      }
      __syncthreads();
      if (tid == 0) {
        float a0 = 0.f, a1 = 0.f;
#pragma unroll
        for (int w2 = 0; w2 < nwarps; ++w2) { a0 += part[(pb * 32 + w2) * NP]; a1 += part[(pb * 32 + w2) * NP + 1]; }
        if constexpr (MODE == MODE_SOFT) {
          if (P.out_soft) P.out_soft[seq * P.len + t] = a0 / (a1 * P.sk);
          if (P.out_argmax) {
            float bp = -1.f;
            int bq = 0x7fffffff;
#pragma unroll
            for (int w2 = 0; w2 < nwarps; ++w2) arg_better(bp, bq, apart[pb * 32 + w2], aidx[pb * 32 + w2]);
            P.out_argmax[seq * n + t] = bq;
          }
        } else {
          P.grad_w[seq * P.len + t] = P.two_over_T * (a0 / P.sk - (wt / P.sk) * a1);
        }
      }
      Cr += (double)Rr;
      Rr = -INFINITY;
#pragma unroll
      for (int w2 = 0; w2 < nwarps; ++w2) Rr = fmaxf(Rr, wmax[pb * 32 + w2]);
    }

    if constexpr (VJP) {
      // fold this sequence's codebook gradient into the CTA partial and clear it
      float z16[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) z16[i] = 0.f;
#pragma unroll
      for (int k = 0; k < KB; ++k) {
        const int mid = tid + NT * k;
        float gcb[16];
        tmem_ld16(tbase + 16 * k, gcb);
        double* dst = gcp + (size_t)mid * 16;
#pragma unroll
        for (int i = 0; i < 16; ++i) dst[i] += (double)gcb[i];
        tmem_st16(tbase + 16 * k, z16);
      }
      tmem_wait_st();
    }
    __syncthreads();
  }

  if constexpr (VJP) {
    tmem_fence_before();
    __syncthreads();
    tmem_fence_after();
    if (warp == 0) tmem_dealloc512(tslot[0]);
  }
}

}  // namespace l16
}  // namespace bcjr
