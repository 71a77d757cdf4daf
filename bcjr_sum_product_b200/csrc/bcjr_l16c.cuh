// VJP sweep for the QTIP-scale trellis (L = 16, D = 2, V = 1) on a cluster of
// two CTAs per sequence, sm_100a.
//
// Same mathematics as the single-CTA l16::vjp_kernel (forward: negated log
// sigma and the prefix expectation A; backward: negated log rho, the suffix
// expectation Bc, G, dl/dw and the per-state codebook gradient; "BCJR-QAT: A
// Differentiable Relaxation of Trellis-Coded Weight Quantization", Abstract and
// Technical Summary "Core Mechanism").  What changes is where the data lives.
// One SM's tensor memory (65536 fp32) holds either the whole scaled codebook or
// the whole per-sequence codebook gradient, not both, so the single-CTA kernel
// streams the codewords from L2 during its backward sweep and keeps A / Bc in
// L2.  Splitting the 4096 blocks of a sequence over two CTAs of a cluster (two
// SMs) halves every per-SM quantity:
//
//   CTA r (cluster rank 0 or 1) owns the blocks mid = 2048 r + lm, lm in [0, 2048);
//   thread tau of 512 owns lm = tau + 512 k, k = 0..3.
//   Tensor memory (per thread: one lane, 128 columns): columns 0..63 hold the
//   thread's 64 codewords for the whole launch, columns 64..127 the current
//   sequence's codebook gradient of the same states.
//   Shared memory: the halves of the group vectors this CTA reads, 8192 values
//   each, double-buffered: negated log sigma / rho and A / Bc (128 KB).
//
// Group values cross to the other CTA through distributed shared memory: a
// thread stores each value it produces into the buffer of the CTA that reads
// it (half of the stores are remote), and one cluster barrier (release /
// acquire) per step orders the stores before the next step's loads.
//
//   forward, group j = (mid << 2) | lo: read by the owner of mid' = j mod 4096,
//     the CTA with bit 11 of j set or not; local index ((j >> 12) << 11) | (j & 2047).
//     A thread's block k goes to CTA (k & 1) at ((2 r + (k >> 1)) << 11) + 4 tau + lo.
//   backward, group i = (h << 12) | mid: read by the owner of mid'' = i >> 2,
//     the CTA i >> 13 = h >> 1; local index i & 8191 = ((h & 1) << 12) | (r << 11) | lm.
//
// Per-step scalars (the re-centring minimum, the centring constant K_t, the
// posterior sums, dl/dw_t) are combined from 32 per-warp partials (16 per CTA)
// that every warp stores into both CTAs; both CTAs read them in the same order,
// so they hold the same bits.
#pragma once
#include "bcjr_l16.cuh"

namespace bcjr {
namespace l16c {

using l16::bidx;
using l16::f2;
using l16::f2s;
constexpr int D = l16::D, J = l16::J, NMID = l16::NMID, S = l16::S;
constexpr int NC = 2;                  // CTAs per cluster (one sequence per cluster)
constexpr int NT = 512;                // threads per CTA
constexpr int KB = NMID / (NC * NT);   // blocks per thread: 4
constexpr int JL = J / NC;             // group values read per CTA: 8192
constexpr int NW = NC * NT / 32;       // warps per cluster: 32
static_assert(KB == 4 && NW == 32, "layout above");

struct Params {
  const float* w;        // [n_seq][len]
  const float* cs_tm;    // block-major scaled codebook [4096][16]
  const float* gsoft;    // [n_seq][len]
  const float* gZ;       // [n_seq] or null
  float* grad_w;         // [n_seq][len]
  double* gc_part;       // [clusters][65536] block-major
  float* hist_l;         // [CTAs][n][2048][4]
  float* hist_a;         // [CTAs][n][2048][4]
  double* hist_c;        // [clusters][n]  forward offsets
  float* hist_r;         // [clusters][n]  forward A reference
  int64_t n_seq, len;
  int n;
  float sk, two_over_T;
};

// ------------------------------------------------------------ cluster helpers
__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ uint32_t cluster_id() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%clusterid.x;" : "=r"(r));
  return r;
}
__device__ __forceinline__ uint32_t cluster_count() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%nclusterid.x;" : "=r"(r));
  return r;
}
// Address in the cluster's shared window of the same offset in CTA `rank`.
__device__ __forceinline__ uint32_t map_rank(uint32_t saddr, uint32_t rank) {
  uint32_t d;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(d) : "r"(saddr), "r"(rank));
  return d;
}
__device__ __forceinline__ void st_cluster4(uint32_t addr, float4 v) {
  asm volatile("st.shared::cluster.v4.f32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "f"(v.x), "f"(v.y), "f"(v.z),
               "f"(v.w)
               : "memory");
}
__device__ __forceinline__ void st_cluster(uint32_t addr, float v) {
  asm volatile("st.shared::cluster.f32 [%0], %1;" ::"r"(addr), "f"(v) : "memory");
}
// All threads of both CTAs; stores before it (shared, distributed shared and
// global) are visible to loads after it.
__device__ __forceinline__ void cluster_sync() {
  asm volatile(
      "barrier.cluster.arrive.release.aligned;\n\t"
      "barrier.cluster.wait.acquire.aligned;" ::: "memory");
}
__device__ __forceinline__ float bfly32_min(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fminf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
__device__ __forceinline__ float bfly32_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// Two 16-column tensor-memory loads completed by one wait.
__device__ __forceinline__ void tmem_ld16x2(uint32_t ta, float (&a)[16], uint32_t tb, float (&b)[16]) {
  uint32_t u[16], v[16];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(u[0]), "=r"(u[1]), "=r"(u[2]), "=r"(u[3]), "=r"(u[4]), "=r"(u[5]), "=r"(u[6]), "=r"(u[7]), "=r"(u[8]),
        "=r"(u[9]), "=r"(u[10]), "=r"(u[11]), "=r"(u[12]), "=r"(u[13]), "=r"(u[14]), "=r"(u[15])
      : "r"(ta));
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]), "=r"(v[8]),
        "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15])
      : "r"(tb));
  asm volatile("tcgen05.wait::ld.sync.aligned;"
               : "+r"(u[0]), "+r"(u[1]), "+r"(u[2]), "+r"(u[3]), "+r"(u[4]), "+r"(u[5]), "+r"(u[6]), "+r"(u[7]),
                 "+r"(u[8]), "+r"(u[9]), "+r"(u[10]), "+r"(u[11]), "+r"(u[12]), "+r"(u[13]), "+r"(u[14]), "+r"(u[15]),
                 "+r"(v[0]), "+r"(v[1]), "+r"(v[2]), "+r"(v[3]), "+r"(v[4]), "+r"(v[5]), "+r"(v[6]), "+r"(v[7]),
                 "+r"(v[8]), "+r"(v[9]), "+r"(v[10]), "+r"(v[11]), "+r"(v[12]), "+r"(v[13]), "+r"(v[14]), "+r"(v[15]));
#pragma unroll
  for (int i = 0; i < 16; ++i) { a[i] = __uint_as_float(u[i]); b[i] = __uint_as_float(v[i]); }
}

// Dynamic shared memory of the kernel, in floats (n = steps per sequence).
__host__ __device__ constexpr size_t smem_floats(int n) {
  return (size_t)4 * JL + 2 * NW * 8 + 4 + 2 * (size_t)n;
}

__global__ void __launch_bounds__(NT, 1) vjp_kernel(Params P) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int n = P.n;
  const uint32_t r = cluster_rank(), peer = r ^ 1u;
  const int64_t cid = cluster_id(), ncl = cluster_count();

  extern __shared__ __align__(16) float smem[];
  float* sb = smem;                  // [2][JL] negated log sigma (forward) / rho (backward)
  float* ab = sb + 2 * JL;           // [2][JL] A (forward) / Bc (backward)
  // per-warp partials of both CTAs, [2 parities][32 warps][8]:
  //   0: sum P(i) (A + Bc)   1: sum P(i) Bc   2: sum P(i)   3: min stored value
  //   4: sum G (c' - w') / logZ sum   5: Hbar sum   6: A reference (forward)
  float* rec = ab + 2 * JL;
  uint32_t* tslot = reinterpret_cast<uint32_t*>(rec + 2 * NW * 8);  // [4]
  float* wsc = reinterpret_cast<float*>(tslot + 4);   // n: -w'
  float* gsc = wsc + n;                               // n: g / sk

  // the peer CTA's copies of sb, ab and rec
  const uint32_t sb_peer = map_rank(l16::smem_addr(sb), peer);
  const uint32_t ab_peer = map_rank(l16::smem_addr(ab), peer);
  const uint32_t rec_peer = map_rank(l16::smem_addr(rec), peer);

  float* hist_l = P.hist_l + (size_t)blockIdx.x * n * JL;   // [n][2048 blocks][4]
  float* hist_a = P.hist_a + (size_t)blockIdx.x * n * JL;
  double* gcp = P.gc_part + (size_t)cid * S;
  const float2 neg1 = f2s(-1.f);
  const int lm0 = tid;                         // lm of block 0; block k is lm0 + 512 k
  const int mid0 = (int)(r << 11) + tid;       // mid of block 0

  if (warp == 0) l16::tmem_alloc512(tslot);
  l16::tmem_fence_before();
  __syncthreads();
  l16::tmem_fence_after();
  const uint32_t tbase = tslot[0] + ((uint32_t)(32 * (warp & 3)) << 16) + (uint32_t)(128 * (warp >> 2));
  // codewords into columns 0..63 for the whole launch
#pragma unroll
  for (int k = 0; k < KB; ++k) {
    float c16[16];
    l16::ld_cb(P.cs_tm, mid0 + NT * k, c16);
    l16::tmem_st16(tbase + 16 * k, c16);
  }
  l16::tmem_wait_st();
  // this CTA's half of the cluster partial
  for (int x = tid; x < S / NC; x += NT) gcp[(size_t)r * (S / NC) + x] = 0.0;
  // the peer must be running before its shared memory is written
  cluster_sync();

  // store one partial of this warp into both CTAs' rec
  auto put_rec = [&](int pb, int slot, float v) {
    const int idx = (pb * NW + (int)r * 16 + warp) * 8 + slot;
    rec[idx] = v;
    st_cluster(rec_peer + 4u * (uint32_t)idx, v);
  };
  auto get_rec = [&](int pb, int slot) -> float { return rec[(pb * NW + lane) * 8 + slot]; };

  for (int64_t seq = cid; seq < P.n_seq; seq += ncl) {
    const float* wq = P.w + seq * P.len;
    const float* gq = P.gsoft + seq * P.len;
    for (int x = tid; x < n; x += NT) { wsc[x] = -wq[x] * P.sk; gsc[x] = gq[x] / P.sk; }
    __syncthreads();

    // ------------------------------------------------------------ forward
    float Rn = 0.f;
    double C = 0.0;
    float refA = 0.f;   // stored A of group 0 at the previous step (cluster-uniform)
    for (int t = 0; t < n; ++t) {
      const float* nprev = sb + ((t + 1) & 1) * JL;
      const float* aprev = ab + ((t + 1) & 1) * JL;
      const int cur = (t & 1) * JL;
      const float2 nw2 = f2s(wsc[t]);
      const float2 g2 = f2s(gsc[t]);
      // A_{t-1} enters relative to its value at group 0, so that the stored
      // prefix expectations stay at the size of their spread over groups; the
      // backward subtracts the same reference.
      const float2 nrA = f2s(-refA);
      if (t > 0 && r == 0 && tid == 0) P.hist_r[(size_t)cid * n + t] = refA;
      C -= (double)Rn;
      float tmin = INFINITY;
      float a0out = 0.f;
#pragma unroll
      for (int k = 0; k < KB; ++k) {
        const int lm = lm0 + NT * k;
        float cb[16];
        l16::tmem_ld16(tbase + 16 * k, cb);
        float2 np01, np23, ap01, ap23;
        if (t == 0) {
          np01 = np23 = ap01 = ap23 = f2s(0.f);
        } else {
          np01 = f2(nprev[(0 << 11) | lm], nprev[(1 << 11) | lm]);
          np23 = f2(nprev[(2 << 11) | lm], nprev[(3 << 11) | lm]);
          ap01 = f2(aprev[(0 << 11) | lm], aprev[(1 << 11) | lm]);
          ap23 = f2(aprev[(2 << 11) | lm], aprev[(3 << 11) | lm]);
          // step t-1's values in block-major order [lm][h], as the backward reads them
          reinterpret_cast<float4*>(hist_l + (size_t)(t - 1) * JL)[lm] =
              make_float4(np01.x, np01.y, np23.x, np23.y);
          reinterpret_cast<float4*>(hist_a + (size_t)(t - 1) * JL)[lm] =
              make_float4(ap01.x, ap01.y, ap23.x, ap23.y);
        }
        const float2 as01 = __fadd2_rn(ap01, nrA), as23 = __fadd2_rn(ap23, nrA);
        float out[4], aout[4];
#pragma unroll
        for (int lo = 0; lo < 4; ++lo) {
          const float2 c01 = f2(cb[bidx(0, lo)], cb[bidx(1, lo)]), c23 = f2(cb[bidx(2, lo)], cb[bidx(3, lo)]);
          const float2 d01 = __fadd2_rn(c01, nw2), d23 = __fadd2_rn(c23, nw2);
          const float2 x01 = __ffma2_rn(d01, d01, np01), x23 = __ffma2_rn(d23, d23, np23);
          const float m = fminf(fminf(x01.x, x01.y), fminf(x23.x, x23.y));
          const float2 a01 = __ffma2_rn(x01, neg1, f2s(m)), a23 = __ffma2_rn(x23, neg1, f2s(m));
          const float2 u01 = f2(ex2f(a01.x), ex2f(a01.y)), u23 = f2(ex2f(a23.x), ex2f(a23.y));
          const float2 z01 = __ffma2_rn(g2, c01, as01), z23 = __ffma2_rn(g2, c23, as23);
          const float2 s2 = __fadd2_rn(u01, u23);
          const float2 q2 = __ffma2_rn(u23, z23, __fmul2_rn(u01, z01));
          const float ssum = s2.x + s2.y;
          out[lo] = (m - Rn) - lg2f(ssum);
          aout[lo] = __fdividef(q2.x + q2.y, ssum);
        }
        if (k == 0) a0out = aout[0];
        tmin = fminf(tmin, fminf(fminf(out[0], out[1]), fminf(out[2], out[3])));
        // groups (mid << 2) | lo go to CTA (k & 1), local ((2 r + (k >> 1)) << 11) + 4 tau
        const int dst = cur + (((int)(2 * r) + (k >> 1)) << 11) + 4 * tid;
        const float4 ov = make_float4(out[0], out[1], out[2], out[3]);
        const float4 av = make_float4(aout[0], aout[1], aout[2], aout[3]);
        if ((uint32_t)(k & 1) == r) {
          *reinterpret_cast<float4*>(sb + dst) = ov;
          *reinterpret_cast<float4*>(ab + dst) = av;
        } else {
          st_cluster4(sb_peer + 4u * (uint32_t)dst, ov);
          st_cluster4(ab_peer + 4u * (uint32_t)dst, av);
        }
      }
      tmin = -warp_max(-tmin);
      if (lane == 0) put_rec(t & 1, 3, tmin);
      // the stored A of group 0 (mid 0, lo 0: CTA 0, thread 0, block 0) is the next step's reference
      if (r == 0 && tid == 0) {
        const int idx = ((t & 1) * NW) * 8 + 6;
        rec[idx] = a0out;
        st_cluster(rec_peer + 4u * (uint32_t)idx, a0out);
      }
      if (r == 0 && tid == 0) P.hist_c[(size_t)cid * n + t] = C;
      cluster_sync();
      Rn = bfly32_min(get_rec(t & 1, 3));
      refA = rec[((t & 1) * NW) * 8 + 6];
    }
    // log2 Z and Hbar = E[A_{n-1}] over both halves
    double l2Z;
    float Hbar;
    {
      const float* nfin = sb + ((n - 1) & 1) * JL;
      const float* afin = ab + ((n - 1) & 1) * JL;
      float s0 = 0.f, s1 = 0.f;
      for (int j = tid; j < JL; j += NT) {
        const float u = ex2f(Rn - nfin[j]);
        s0 += u;
        s1 = fmaf(u, afin[j], s1);
      }
      s0 = warp_sum(s0);
      s1 = warp_sum(s1);
      if (lane == 0) { put_rec(n & 1, 4, s0); put_rec(n & 1, 5, s1); }
      cluster_sync();
      const float a0 = bfly32_sum(get_rec(n & 1, 4));
      const float a1 = bfly32_sum(get_rec(n & 1, 5));
      l2Z = -(double)Rn + log2((double)a0) + C;
      Hbar = a1 / a0;
    }
    const float gzq = P.gZ ? P.gZ[seq] : 0.f;
    const float2 nc2T = f2s(-P.two_over_T / P.sk);

    // columns 64..127 accumulate this sequence's codebook gradient
    {
      float z16[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) z16[i] = 0.f;
#pragma unroll
      for (int k = 0; k < KB; ++k) l16::tmem_st16(tbase + 64 + 16 * k, z16);
      l16::tmem_wait_st();
    }

    // ------------------------------------------------------------ backward
    // G_t(q) = p_t(q) (A_{t-1}(q >> 2) + h_t(q) + Bc_t(q mod J) - K_t + gZ) with
    // K_t = sum_j P_t(j) (A_t(j) + Bc_t(j)), P_t(j) the posterior of group j,
    // formed from the same stored values one step earlier (K_{n-1} = Hbar), so
    // that rounding carried along the recursions cancels in G.  Stored Bc_t is
    // relative to rB, the posterior mean of the previous step's stored values.
    float Rrn = 0.f;
    double Cr = 0.0;
    float Kt = Hbar, rB = 0.f;
    auto hist_at = [&](const float* hbuf, int tt, int kk) -> float4 {
      return (tt >= 1) ? reinterpret_cast<const float4*>(hbuf + (size_t)(tt - 1) * JL)[lm0 + NT * kk]
                       : make_float4(0.f, 0.f, 0.f, 0.f);
    };
    float4 hsn = hist_at(hist_l, n - 1, 0), han = hist_at(hist_a, n - 1, 0);
    for (int t = n - 1; t >= 0; --t) {
      const float* ncur = sb + (t & 1) * JL;
      const float* bcur = ab + (t & 1) * JL;
      const int nxt = ((t + 1) & 1) * JL;
      const float2 nw2 = f2s(wsc[t]);
      const float2 g2 = f2s(gsc[t]);
      const float2 gr2 = f2s(gsc[t] * P.sk);
      const double Csig = (t >= 1) ? P.hist_c[(size_t)cid * n + t - 1] : 0.0;
      const float K = (float)(Csig + Cr - l2Z);
      const bool last = (t == n - 1);
      const float rA = (t >= 1) ? P.hist_r[(size_t)cid * n + t] : 0.f;   // the forward's reference
      const float hbt = Kt + rA - rB - gzq;
      float2 accGd = f2s(0.f);   // sum_q G (c' - w')
      float2 accK = f2s(0.f), accB = f2s(0.f), accP = f2s(0.f);
      float tmin = INFINITY;
#pragma unroll
      for (int k = 0; k < KB; ++k) {
        const int lm = lm0 + NT * k;
        float nr[4], bc[4];
        if (last) {
          nr[0] = nr[1] = nr[2] = nr[3] = 0.f;
          bc[0] = bc[1] = bc[2] = bc[3] = 0.f;
        } else {
          const float4 rv = reinterpret_cast<const float4*>(ncur)[lm];
          const float4 bv = reinterpret_cast<const float4*>(bcur)[lm];
          nr[0] = rv.x; nr[1] = rv.y; nr[2] = rv.z; nr[3] = rv.w;
          bc[0] = bv.x - rB; bc[1] = bv.y - rB; bc[2] = bv.z - rB; bc[3] = bv.w - rB;
        }
        const float4 hs4 = hsn, ha4 = han;
        {
          const int nt = (k + 1 < KB) ? t : t - 1, nk = (k + 1 < KB) ? k + 1 : 0;
          hsn = hist_at(hist_l, nt, nk);
          han = hist_at(hist_a, nt, nk);
        }
        float cb[16], gcb[16];
        tmem_ld16x2(tbase + 16 * k, cb, tbase + 64 + 16 * k, gcb);
        float nout[4], bout[4];
#pragma unroll
        for (int g = 0; g < 2; ++g) {          // groups h = 2g, 2g+1 side by side
          const float hs0 = g ? hs4.z : hs4.x, hs1 = g ? hs4.w : hs4.y;
          const float ha0 = g ? ha4.z : ha4.x, ha1 = g ? ha4.w : ha4.y;
          float2 y[4], c2[4];
#pragma unroll
          for (int lo = 0; lo < 4; ++lo) {
            c2[lo] = f2(cb[bidx(2 * g, lo)], cb[bidx(2 * g + 1, lo)]);
            const float2 dd = __fadd2_rn(c2[lo], nw2);
            y[lo] = __ffma2_rn(dd, dd, f2s(nr[lo]));
          }
          // the posterior directly, p = 2^(K - n_sigma - y'), one ex2 per state
          const float2 kh = __fadd2_rn(f2s(K), f2(-hs0, -hs1));
          const float2 ah = f2(ha0 - hbt, ha1 - hbt);   // A - K + gZ
          float2 ssum = f2s(0.f), num = f2s(0.f);
#pragma unroll
          for (int lo = 0; lo < 4; ++lo) {
            const float2 a = __ffma2_rn(y[lo], neg1, kh);
            const float2 pp = f2(ex2f(a.x), ex2f(a.y));
            ssum = __fadd2_rn(ssum, pp);
            const float2 z = __ffma2_rn(g2, c2[lo], f2s(bc[lo]));          // Bc + h
            num = __ffma2_rn(pp, z, num);
            const float2 G = __fmul2_rn(pp, __fadd2_rn(z, ah));
            const float2 Gd = __fmul2_rn(G, __fadd2_rn(c2[lo], nw2));   // G (c' - w')
            accGd = __fadd2_rn(accGd, Gd);
            float2 gc = f2(gcb[bidx(2 * g, lo)], gcb[bidx(2 * g + 1, lo)]);
            gc = __ffma2_rn(Gd, nc2T, __ffma2_rn(gr2, pp, gc));       // + g p + (2/T) G (w - c)
            gcb[bidx(2 * g, lo)] = gc.x;
            gcb[bidx(2 * g + 1, lo)] = gc.y;
          }
          // negated log rho_{t-1} = (K - n_sigma) - lg2 sum p; a group whose posterior mass
          // underflows gets rho = 0 (+inf) and Bc = 0, moving no posterior by more than that mass
          nout[2 * g] = (kh.x - Rrn) - lg2f(ssum.x);
          nout[2 * g + 1] = (kh.y - Rrn) - lg2f(ssum.y);
          bout[2 * g] = (ssum.x > 0.f) ? __fdividef(num.x, ssum.x) : 0.f;
          bout[2 * g + 1] = (ssum.y > 0.f) ? __fdividef(num.y, ssum.y) : 0.f;
          // posterior of the two step t-1 groups, P(i) = sum_lo p
          const float2 pg = ssum, bo = f2(bout[2 * g], bout[2 * g + 1]);
          accK = __ffma2_rn(pg, __fadd2_rn(f2(ha0, ha1), bo), accK);
          accB = __ffma2_rn(pg, bo, accB);
          accP = __fadd2_rn(accP, pg);
        }
        l16::tmem_st16(tbase + 64 + 16 * k, gcb);
        if (t >= 1) {
          // group (h << 12) | mid goes to CTA h >> 1, local ((h & 1) << 12) | (r << 11) | lm
#pragma unroll
          for (int h = 0; h < 4; ++h) {
            const int dst = nxt + ((h & 1) << 12) + (int)(r << 11) + lm;
            if ((uint32_t)(h >> 1) == r) {
              sb[dst] = nout[h];
              ab[dst] = bout[h];
            } else {
              st_cluster(sb_peer + 4u * (uint32_t)dst, nout[h]);
              st_cluster(ab_peer + 4u * (uint32_t)dst, bout[h]);
            }
          }
          tmin = fminf(tmin, fminf(fminf(nout[0], nout[1]), fminf(nout[2], nout[3])));
        }
      }
      l16::tmem_wait_st();
      const float a0 = warp_sum(accGd.x + accGd.y);
      const float kk = warp_sum(accK.x + accK.y);
      const float kb = warp_sum(accB.x + accB.y);
      const float kp = warp_sum(accP.x + accP.y);
      tmin = -warp_max(-tmin);
      const int pb = t & 1;
      if (lane == 0) {
        const int idx = (pb * NW + (int)r * 16 + warp) * 8;
        const float4 v = make_float4(kk, kb, kp, tmin);
        *reinterpret_cast<float4*>(rec + idx) = v;
        rec[idx + 4] = a0;
        st_cluster4(rec_peer + 4u * (uint32_t)idx, v);
        st_cluster(rec_peer + 4u * (uint32_t)(idx + 4), a0);
      }
      cluster_sync();
      if (r == 0 && tid == 0) {
        float s0 = 0.f;
#pragma unroll
        for (int w2 = 0; w2 < NW; ++w2) s0 += rec[(pb * NW + w2) * 8 + 4];
        // dl/dw_t = (2/T) sum_q G (c - w_t) = (2/T) sum_q G (c' - w') / sk
        P.grad_w[seq * P.len + t] = P.two_over_T * s0 / P.sk;
      }
      Cr -= (double)Rrn;
      {
        const float4 rv = *reinterpret_cast<const float4*>(rec + (pb * NW + lane) * 8);
        const float sp = bfly32_sum(rv.z);   // sum_q p_t(q), 1 up to rounding
        Kt = bfly32_sum(rv.x) / sp;
        rB = bfly32_sum(rv.y) / sp;
        if (r == 0 && tid == 0) check_posterior_mass(sp);
        Rrn = bfly32_min(rv.w);
        // Forward and backward carry different rounding relative to the one
        // log Z, so the posterior sum drifts from 1 along the sweep; folding
        // its logarithm into the backward offset renormalises every next step.
        Cr -= (double)lg2f(sp);
      }
    }

    // fold this sequence's codebook gradient into the cluster partial
#pragma unroll
    for (int k = 0; k < KB; ++k) {
      float gcb[16];
      l16::tmem_ld16(tbase + 64 + 16 * k, gcb);
      double* dst = gcp + (size_t)(mid0 + NT * k) * 16;
#pragma unroll
      for (int i = 0; i < 16; ++i) dst[i] += (double)gcb[i];
    }
    // the next sequence's first stores into the peer's rec / group buffers wait
    // until both CTAs have read this sequence's last partials
    cluster_sync();
  }

  // neither CTA leaves while the other may still store into its shared memory
  cluster_sync();
  l16::tmem_fence_before();
  __syncthreads();
  l16::tmem_fence_after();
  if (warp == 0) l16::tmem_dealloc512(tslot[0]);
}

}  // namespace l16c
}  // namespace bcjr
