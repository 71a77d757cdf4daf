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
//   The scaled codebook is stored block-major, cs_tm[mid * 16 + bidx(h, lo)]
//   with bidx(h, lo) = 8 (h >> 1) + 2 lo + (h & 1): a thread's 16 codewords of
//   a block are one 64-byte line (the same every step), the two halves are
//   the h-pairs {0,1} and {2,3}, and within a half the pair (2g, 2g+1) of one
//   bottom digit lo is adjacent, feeding the packed f32x2 instructions in
//   both directions.
//   Tensor memory (512 columns x 128 lanes = 65536 fp32, one per state) holds,
//   for SOFT, the thread's codewords (read back every step without touching
//   L2) and, for VJP, the current sequence's per-state codebook gradient
//   (the VJP's backward then reads the codebook through a shared-memory ring
//   that bulk copies fill, or streams it from L2); warp w uses lanes
//   32 (w mod 4) .. + 31 and columns 128 (w div 4) + 16 k for block k.
#pragma once
#include "bcjr_kernels.cuh"

namespace bcjr {
namespace l16 {

constexpr int L = 16, D = 2, HB = 12;  // HB: bits of mid
constexpr int J = 1 << 14, NMID = 1 << 12, NT = 512, KB = NMID / NT;
constexpr int S = 1 << 16;
static_assert(NT / 32 == 16, "the per-step reductions combine 16 warps");

struct Params {
  const float* w;        // [n_seq][len]
  const float* cs_tm;    // block-major scaled codebook [4096][16]
  const float* cs_rg;    // the same in ring order (make_ring_codebook), VJP with the codeword ring
  const float* gsoft;    // [n_seq][len] (VJP)
  const float* gZ;       // [n_seq] or null (VJP)
  float* out_soft;       // [n_seq][len] or null
  float* out_logZ;       // [n_seq] or null
  int32_t* out_argmax;   // [n_seq][n] or null
  float* grad_w;         // [n_seq][len] (VJP)
  double* gc_part;       // [grid][65536] block-major (VJP)
  float* hist_l;         // [grid][n][J], or the checkpoint layout when ck > 0
  float* hist_a;         // [grid][n][J] (VJP)
  double* hist_c;        // [grid][n]  fp64 offsets of the forward steps
  float* hist_rn;        // [grid][n]  re-centring value of each forward step
  int ck;                // checkpoint segment length K, 0 = full histories
  float* bc_g;           // [grid][2][J] (VJP backward ping-pong)
  int64_t n_seq, len;
  int n;
  float sk, two_over_T;
  int ring_nofill;       // test hook: the ring is never filled, so its bounded waits run out
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
// Tensor-memory loads and stores touch no generic memory, so they carry no
// "memory" clobber (the compiler may move ordinary loads across them); they are
// volatile, which keeps them in program order among themselves, and the
// destination registers of a load are tied to the wait that completes it, so
// no use can be scheduled before the data has arrived.
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float (&r)[16]) {
  uint32_t u[16];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(u[0]), "=r"(u[1]), "=r"(u[2]), "=r"(u[3]), "=r"(u[4]), "=r"(u[5]), "=r"(u[6]), "=r"(u[7]), "=r"(u[8]),
        "=r"(u[9]), "=r"(u[10]), "=r"(u[11]), "=r"(u[12]), "=r"(u[13]), "=r"(u[14]), "=r"(u[15])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;"
               : "+r"(u[0]), "+r"(u[1]), "+r"(u[2]), "+r"(u[3]), "+r"(u[4]), "+r"(u[5]), "+r"(u[6]), "+r"(u[7]),
                 "+r"(u[8]), "+r"(u[9]), "+r"(u[10]), "+r"(u[11]), "+r"(u[12]), "+r"(u[13]), "+r"(u[14]), "+r"(u[15]));
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
      "r"(__float_as_uint(r[14])), "r"(__float_as_uint(r[15])));
}
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;"); }
__device__ __forceinline__ void tmem_ld8(uint32_t taddr, float (&r)[8]) {
  uint32_t u[8];
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
               : "=r"(u[0]), "=r"(u[1]), "=r"(u[2]), "=r"(u[3]), "=r"(u[4]), "=r"(u[5]), "=r"(u[6]), "=r"(u[7])
               : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;"
               : "+r"(u[0]), "+r"(u[1]), "+r"(u[2]), "+r"(u[3]), "+r"(u[4]), "+r"(u[5]), "+r"(u[6]), "+r"(u[7]));
#pragma unroll
  for (int i = 0; i < 8; ++i) r[i] = __uint_as_float(u[i]);
}
__device__ __forceinline__ void tmem_st8(uint32_t taddr, const float (&r)[8]) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"r"(taddr),
               "r"(__float_as_uint(r[0])), "r"(__float_as_uint(r[1])), "r"(__float_as_uint(r[2])),
               "r"(__float_as_uint(r[3])), "r"(__float_as_uint(r[4])), "r"(__float_as_uint(r[5])),
               "r"(__float_as_uint(r[6])), "r"(__float_as_uint(r[7])));
}

__host__ __device__ constexpr int bidx(int h, int lo) { return 8 * (h >> 1) + 2 * lo + (h & 1); }

// Bulk prefetch of `bytes` (a multiple of 16, 16-byte aligned) from global
// memory into L2 by the tensor-memory-access unit: no registers, no shared
// memory, nothing to wait for.
__device__ __forceinline__ void prefetch_l2_bulk(const void* p, uint32_t bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(p), "r"(bytes) : "memory");
}

__device__ __forceinline__ void ld_cb(const float* __restrict__ cs_tm, int mid, float (&c)[16]) {
  const float4* p = reinterpret_cast<const float4*>(cs_tm + (size_t)mid * 16);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    float4 v = __ldg(p + i);
    c[4 * i] = v.x; c[4 * i + 1] = v.y; c[4 * i + 2] = v.z; c[4 * i + 3] = v.w;
  }
}

// The half of block mid holding the h-pair g: 8 codewords, index 2 lo + (h & 1).
__device__ __forceinline__ void ld_cb8(const float* __restrict__ cs_tm, int mid, int g, float (&c)[8]) {
  const float4* p = reinterpret_cast<const float4*>(cs_tm + (size_t)mid * 16 + 8 * g);
  const float4 a = __ldg(p), b = __ldg(p + 1);
  c[0] = a.x; c[1] = a.y; c[2] = a.z; c[3] = a.w; c[4] = b.x; c[5] = b.y; c[6] = b.z; c[7] = b.w;
}

// cs_tm[mid * 16 + bidx(h, lo)] = sk * c[(h << 14) | (mid << 2) | lo]
__global__ void make_block_codebook(const float* __restrict__ c, float sk, float* __restrict__ cs_tm) {
  int x = blockIdx.x * blockDim.x + threadIdx.x;
  if (x >= S) return;
  const int mid = x >> 4, r = x & 15, h = ((r >> 3) << 1) | (r & 1), lo = (r >> 1) & 3;
  cs_tm[x] = sk * c[(h << 14) | (mid << 2) | lo];
}

// ------------------------------------------------------------ codeword ring
// The VJP backward keeps the sequence's codebook gradient in tensor memory, so
// its codewords come from global memory: through a ring of NS shared-memory
// stages, each holding one block k of every thread (32 KB), filled by bulk
// copies (cp.async.bulk, completion counted on the stage's mbarrier).  Every
// warp, after its last read of a stage, adds one to the stage's release counter;
// the sixteenth warp refills the stage with block k + NS.  A warp therefore
// never waits for a producer, only for the copy, which was issued one block
// earlier.  cs_rg orders each block's chunk quad-major,
// cs_rg[((k * 4 + i) * NT + tau) * 4 + e] = cs_tm[(tau + NT k) * 16 + 4 i + e],
// so that a warp's 16-byte shared-memory reads of one quad are consecutive.
__global__ void make_ring_codebook(const float* __restrict__ cs_tm, float* __restrict__ cs_rg) {
  int x = blockIdx.x * blockDim.x + threadIdx.x;
  if (x >= S) return;
  const int e = x & 3, tau = (x >> 2) & (NT - 1), i = (x >> 11) & 3, k = x >> 13;
  cs_rg[x] = cs_tm[(size_t)(tau + NT * k) * 16 + 4 * i + e];
}

constexpr int NS = 2;                                   // ring stages
constexpr int kStageFloats = 4 * NT * 4;                // one block of every thread, 32 KB
constexpr uint32_t kStageBytes = kStageFloats * sizeof(float);
constexpr int kRingCtlWords = 24;                       // 4 mbarriers, 4 + 4 counters, failure flag, padding
constexpr uint64_t kRingWaitNs = 1000000000ull;        // a wait gives up after 1 s

__device__ __forceinline__ void mbar_init(uint64_t* b, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(b)), "r"(count) : "memory");
}
// Bulk copy of one stage; the mbarrier's phase completes when its bytes have landed.
__device__ __forceinline__ void ring_fill(float* stage, const float* src, uint64_t* full) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_addr(full)), "r"(kStageBytes)
               : "memory");
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                   smem_addr(stage)),
               "l"(src), "r"(kStageBytes), "r"(smem_addr(full))
               : "memory");
}
__device__ __forceinline__ bool mbar_try(uint32_t addr, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}"
      : "=r"(ok)
      : "r"(addr), "r"(parity)
      : "memory");
  return ok != 0;
}
__device__ __forceinline__ uint64_t global_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}
// Waits for the phase of parity `parity` to complete; false after kRingWaitNs.
__device__ __forceinline__ bool mbar_wait(uint64_t* b, uint32_t parity) {
  const uint32_t a = smem_addr(b);
  if (mbar_try(a, parity)) return true;
  const uint64_t t0 = global_ns();
  while (!mbar_try(a, parity)) {
    if (global_ns() - t0 > kRingWaitNs) return false;
  }
  return true;
}
__device__ __forceinline__ uint32_t ring_release(uint32_t* cnt) {
  uint32_t old;
  asm volatile("atom.acq_rel.cta.shared::cta.add.u32 %0, [%1], 1;" : "=r"(old) : "r"(smem_addr(cnt)) : "memory");
  return old;
}

// grad_c[q] = sum over CTAs of gc_part[cta][block-major index of q]
__global__ void reduce_block_gc(const double* __restrict__ part, int nparts, float* __restrict__ out) {
  int q = blockIdx.x * blockDim.x + threadIdx.x;
  if (q >= S) return;
  const int h = q >> 14, mid = (q >> 2) & (NMID - 1), lo = q & 3;
  const size_t x = (size_t)mid * 16 + bidx(h, lo);
  double a = 0.0;
  for (int p = 0; p < nparts; ++p) a += part[(size_t)p * S + x];
  out[q] = (float)a;
}

// ------------------------------------------------------------ soft pass, packed
// The soft-codeword pass (forward + backward + posterior + w_hat, optional
// posterior argmax) with the FP32 work in packed f32x2 instructions.  Log
// values are kept negated ("energies", n = -log2), so that each group is
//   x'_h = d_h^2 + n_h,  m' = min_h x'_h,  n_new = m' - log2 sum_h 2^(m' - x'_h) - offset,
// every line an FFMA/FADD without negations.  Pairs (h, h+1) share one f32x2
// lane pair: in the forward they are two members of one group, in the
// backward two groups with the same member.
//
// The forward stores every step's group values n_t(j) in group order [t][j];
// the backward of block mid at step t reads its own four outputs n_t((mid << 2) | lo)
// (one 16-byte vector) and its four inputs n_{t-1}((h << 12) | mid) (four
// scalars that consecutive threads read from consecutive addresses).
//
// Two backward sweeps (template parameter POST):
//  * posterior space (POST): with u_t(q) = alpha_t(q) / sigma_t(q mod J), the
//    forward weight of q within its group, and P_t(j) the posterior mass of
//    forward group j at step t,
//        p_t(q) = u_t(q) P_t(q mod J),   P_{t-1}(i) = sum_lo p_t((i << 2) | lo),
//        log2 u_t(q) = n_t(q mod J) + Rn_t - (d_t(q)^2 + n_{t-1}(q >> 2)),
//    where Rn_t is the re-centring value of forward step t: one ex2 and one
//    multiply per state, linear sums per group, no logarithm; the exchanged
//    values are probabilities (no range problem at any temperature);
//  * log domain: p = 2^(K - n_sigma - y') with the negated log rho exchanged,
//    one ex2 per state plus one lg2 per group.
__device__ __forceinline__ float2 f2(float a, float b) { return make_float2(a, b); }
__device__ __forceinline__ float2 f2s(float a) { return make_float2(a, a); }

// Block-wide combination of the 16 per-warp partials of a step: lane l holds
// warp (l mod 16)'s value and an xor butterfly over 16 lanes combines them.
// Every level pairs lane l with l ^ o and both form the same commutative
// result, so every lane of every warp ends with the same bits.
__device__ __forceinline__ float bfly16_min(float v) {
#pragma unroll
  for (int o = 8; o > 0; o >>= 1) v = fminf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
__device__ __forceinline__ float bfly16_sum(float v) {
#pragma unroll
  for (int o = 8; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// 2^x on the FMA pipe instead of the MUFU unit, for x <= 127 (the split-ex2
// variant of the soft kernel).  Cody and Waite's range reduction x = n + f with
// n = round(x), f in [-1/2, 1/2] (adding and subtracting 1.5 * 2^23 rounds x to
// an integer held in the low mantissa bits), then 2^f by a degree-5 polynomial
// fitted for relative error (ex2_poly.py: 2.0e-7 in fp32, the accuracy of
// ex2.approx), scaled by 2^n through the exponent field.  x is clamped to
// -126, so results that ex2.approx.ftz flushes to 0 come out below 2^-126.
__device__ __forceinline__ float ex2_fma(float x) {
  constexpr float kRound = 12582912.f;   // 1.5 * 2^23
  x = fminf(fmaxf(x, -126.f), 127.f);
  const float t = __fadd_rn(x, kRound);
  const float f = __fsub_rn(x, __fsub_rn(t, kRound));
  float p = fmaf(0.0013266970636323094f, f, 0.009675459936261177f);
  p = fmaf(p, f, 0.05550742521882057f);
  p = fmaf(p, f, 0.24022121727466583f);
  p = fmaf(p, f, 0.6931469440460205f);
  p = fmaf(p, f, 1.0000001192092896f);
  const uint32_t n = (uint32_t)(__float_as_int(t) - 0x4B400000);
  return __uint_as_float(__float_as_uint(p) + (n << 23));
}

// One forward group of the soft pass: x_h = d_h^2 + n_h for the four members
// (h = 0..3 in two lane pairs); returns the negated log2 of sum_h 2^(-x_h)
// re-centred by Rn.  The smallest x contributes 2^0 = 1 exactly, so only the
// three others need an ex2: a min/max network picks them.  With FMA_EX2 one
// of the three runs on the FMA pipe.
template <bool FMA_EX2 = false>
__device__ __forceinline__ float soft_group(float2 x01, float2 x23, float Rn) {
  const float l01 = fminf(x01.x, x01.y), h01 = fmaxf(x01.x, x01.y);
  const float l23 = fminf(x23.x, x23.y), h23 = fmaxf(x23.x, x23.y);
  const float m = fminf(l01, l23), M = fmaxf(l01, l23);
  const float2 a = __ffma2_rn(f2(h01, h23), f2s(-1.f), f2s(m));
  const float e1 = FMA_EX2 ? ex2_fma(m - M) : ex2f(m - M);
  const float s = (1.f + e1) + (ex2f(a.x) + ex2f(a.y));
  return (m - Rn) - lg2f(s);
}

// Forward values kept for the backward sweep, per CTA.  For sequences whose
// full history fits the scratch budget, every step's vector ([n][J]).
// Otherwise (long sequences) checkpoints: the forward keeps the vector of
// every K-th step and all vectors of the last segment; the backward, before it
// enters each earlier segment, recomputes that segment's forward from its
// checkpoint into the segment buffer (about 2 sqrt(n) vectors instead of n,
// for one more forward sweep over all but the last segment).  The recompute
// repeats the stored per-step re-centring values, so its vectors have the same
// bits as the first forward's.
template <bool CKPT>
struct History {
  float* full;   // [n][J] (full histories)
  float* ckpt;   // [S][J]: vector s = the forward values of step s K - 1 (s >= 1)
  float* seg;    // [K][J]: the forward values of steps s0 .. s0 + K - 1
  int K, s0;     // segment length, first step of the segment in seg
  // vector of step tt; with checkpoints tt >= s0 - 1 (below that: the checkpoint
  // of the segment containing tt + 1, an in-bounds vector of another step)
  __device__ __forceinline__ const float* at(int tt) const {
    if constexpr (!CKPT) return full + (size_t)tt * J;
    return (tt >= s0) ? seg + (size_t)(tt - s0) * J : ckpt + (size_t)((tt + 1) / K) * J;
  }
  __device__ __forceinline__ bool resident(int tt) const { return !CKPT || tt >= s0; }
};

// n_{tt-1}((h << 12) | mid) for h = 0..3 (zero for tt = 0: free start)
template <bool CKPT>
__device__ __forceinline__ float4 hist_in(const History<CKPT>& H, int tt, int mid) {
  if (tt < 1) return make_float4(0.f, 0.f, 0.f, 0.f);
  const float* p = H.at(tt - 1) + mid;
  return make_float4(p[0], p[1 << HB], p[2 << HB], p[3 << HB]);
}
// n_tt((mid << 2) | lo) for lo = 0..3
template <bool CKPT>
__device__ __forceinline__ float4 hist_out(const History<CKPT>& H, int tt, int mid) {
  return reinterpret_cast<const float4*>(H.at(tt))[mid];
}
// The backward of step t reads step t - 1's vector; at its start lanes 0..7 of
// one warp ask for step t - 2's (64 KB) so that it is in L2 for the next step.
template <bool CKPT>
__device__ __forceinline__ void prefetch_history(const History<CKPT>& H, int t, int lane) {
  constexpr uint32_t kChunk = J * sizeof(float) / 8;
  if (t >= 2 && lane < 8 && H.resident(t - 2))
    prefetch_l2_bulk(reinterpret_cast<const char*>(H.at(t - 2)) + lane * kChunk, kChunk);
}
// Copies a J-vector with all threads of the CTA (the caller synchronises).
__device__ __forceinline__ void copy_vec(float* dst, const float* src, int tid) {
  for (int j = 4 * tid; j < J; j += 4 * NT)
    *reinterpret_cast<float4*>(dst + j) = *reinterpret_cast<const float4*>(src + j);
}

template <bool ARGMAX, bool POST, bool FMA_EX2, bool CKPT>
__global__ void __launch_bounds__(NT, 1) soft_kernel(Params P) {
  constexpr int NP = 2;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  constexpr int nwarps = NT / 32;
  const int n = P.n;

  extern __shared__ __align__(16) float smem[];
  float* sb = smem;                                    // [2][J] forward values / backward messages
  float* lb[2] = {sb, sb + J};
  float* wmin = sb + 2 * J;                            // [2][32]
  float* part = wmin + 64;                             // [2][32][NP]
  float* apart = part + 2 * 32 * NP;                   // [2][32]
  int* aidx = reinterpret_cast<int*>(apart + 64);      // [2][32]
  uint32_t* tslot = reinterpret_cast<uint32_t*>(aidx + 64);  // [4]
  float* wsc = reinterpret_cast<float*>(tslot + 4);    // n

  // per-CTA history: full [n][J], or checkpoints [S][J], a segment [K][J] and a
  // save slot [J] for the backward message while a segment is recomputed
  History<CKPT> H{};
  float* msave = nullptr;
  int s_last = 0;
  if constexpr (!CKPT) {
    H.full = P.hist_l + (size_t)blockIdx.x * n * J;
  } else {
    const int K = P.ck, S = (n + K - 1) / K;
    float* base = P.hist_l + (size_t)blockIdx.x * (S + K + 1) * J;
    H.ckpt = base;
    H.seg = base + (size_t)S * J;
    msave = base + (size_t)(S + K) * J;
    H.K = K;
    s_last = ((n - 1) / K) * K;
  }
  double* hist_c = P.hist_c + (size_t)blockIdx.x * n;
  float* hist_rn = P.hist_rn + (size_t)blockIdx.x * n;
  const float2 neg1 = f2s(-1.f);

  if (warp == 0) tmem_alloc512(tslot);
  tmem_fence_before();
  __syncthreads();
  tmem_fence_after();
  const uint32_t tbase = tslot[0] + ((uint32_t)(32 * (warp & 3)) << 16) + (uint32_t)(128 * (warp >> 2));
#pragma unroll
  for (int k = 0; k < KB; ++k) {
    float c16[16];
    ld_cb(P.cs_tm, tid + NT * k, c16);
    tmem_st16(tbase + 16 * k, c16);
  }
  tmem_wait_st();

  // One forward step: reads step t-1's vector from shared memory, writes step
  // t's there and to up to two history slots; returns the thread's minimum of
  // the stored values.
  auto forward_step = [&](int t, float Rn, float* dst_a, float* dst_b) -> float {
    const float* nprev = lb[(t + 1) & 1];
    float* ncur = lb[t & 1];
    const float2 nw2 = f2s(wsc[t]);
    float tmin = INFINITY;
#pragma unroll
    for (int k = 0; k < KB; ++k) {
      const int mid = tid + NT * k;
      float cb[16];
      tmem_ld16(tbase + 16 * k, cb);
      float2 np01, np23;
      if (t == 0) {
        np01 = f2s(0.f); np23 = f2s(0.f);
      } else {
        np01 = f2(nprev[(0 << HB) | mid], nprev[(1 << HB) | mid]);
        np23 = f2(nprev[(2 << HB) | mid], nprev[(3 << HB) | mid]);
      }
      float out[4];
#pragma unroll
      for (int lo = 0; lo < 4; ++lo) {
        const float2 d01 = __fadd2_rn(f2(cb[bidx(0, lo)], cb[bidx(1, lo)]), nw2);
        const float2 d23 = __fadd2_rn(f2(cb[bidx(2, lo)], cb[bidx(3, lo)]), nw2);
        out[lo] = soft_group<FMA_EX2>(__ffma2_rn(d01, d01, np01), __ffma2_rn(d23, d23, np23), Rn);
      }
      tmin = fminf(tmin, fminf(fminf(out[0], out[1]), fminf(out[2], out[3])));
      const float4 ov = make_float4(out[0], out[1], out[2], out[3]);
      reinterpret_cast<float4*>(ncur)[mid] = ov;
      if (dst_a) reinterpret_cast<float4*>(dst_a)[mid] = ov;
      if (dst_b) reinterpret_cast<float4*>(dst_b)[mid] = ov;
    }
    return tmin;
  };

  // Before the backward of step t enters the segment below the one in H.seg:
  // the message of step t is saved, that segment's forward recomputed from its
  // checkpoint, and the message restored.
  auto enter_segment = [&](int t) {
    if constexpr (!CKPT) return;
    copy_vec(msave, lb[t & 1], tid);
    H.s0 -= H.K;
    if (H.s0 > 0) copy_vec(lb[(H.s0 + 1) & 1], H.ckpt + (size_t)(H.s0 / H.K) * J, tid);
    __syncthreads();
    for (int tt = H.s0; tt < H.s0 + H.K; ++tt) {
      forward_step(tt, hist_rn[tt], H.seg + (size_t)(tt - H.s0) * J, nullptr);
      __syncthreads();
    }
    copy_vec(lb[t & 1], msave, tid);
    __syncthreads();
  };

  for (int64_t seq = blockIdx.x; seq < P.n_seq; seq += gridDim.x) {
    const float* wq = P.w + seq * P.len;
    for (int x = tid; x < n; x += NT) wsc[x] = -wq[x] * P.sk;   // -w'
    H.s0 = CKPT ? s_last : 0;
    __syncthreads();

    // ------------------------------------------------------------ forward
    float Rn = 0.f;     // min of the previous step's stored (negated) values
    double C = 0.0;     // log2 sigma_t = -stored + C_t
    for (int t = 0; t < n; ++t) {
      C -= (double)Rn;
      float* dst_a = !CKPT ? H.full + (size_t)t * J : (t >= s_last ? H.seg + (size_t)(t - s_last) * J : nullptr);
      float* dst_b = (CKPT && (t + 1) % H.K == 0 && t + 1 < n) ? H.ckpt + (size_t)((t + 1) / H.K) * J : nullptr;
      float tmin = forward_step(t, Rn, dst_a, dst_b);
      tmin = -warp_max(-tmin);
      if (lane == 0) wmin[(t & 1) * 32 + warp] = tmin;
      if (tid == 0) { hist_c[t] = C; hist_rn[t] = Rn; }
      __syncthreads();
      Rn = bfly16_min(wmin[(t & 1) * 32 + (lane & 15)]);
    }
    // log2 Z = -Rn + log2 sum_j 2^(Rn - stored_j) + C; the posterior space
    // backward starts from P_{n-1}(j) = 2^(Rn - stored_j) / sum, written in place
    double l2Z;
    {
      float* nfin = lb[(n - 1) & 1];
      float s0 = 0.f;
      for (int j = tid; j < J; j += NT) s0 += ex2f(Rn - nfin[j]);
      s0 = warp_sum(s0);
      if (lane == 0) part[warp * NP] = s0;
      __syncthreads();
      float a0 = 0.f;
#pragma unroll
      for (int w2 = 0; w2 < nwarps; ++w2) a0 += part[w2 * NP];
      l2Z = -(double)Rn + log2((double)a0) + C;
      if (tid == 0 && P.out_logZ) P.out_logZ[seq] = (float)(l2Z * 0.69314718055994530942);
      if constexpr (POST) {
        const float inv = 1.f / a0;
        for (int j = tid; j < J; j += NT) nfin[j] = ex2f(Rn - nfin[j]) * inv;
      }
      __syncthreads();
    }

    // ------------------------------------------------------------ backward
    if constexpr (POST) {
      // block kk of step tt: its inputs (scalars) and outputs (vector), one block ahead
      float4 hin_n = hist_in(H, n - 1, tid), hout_n = hist_out(H, n - 1, tid);
      for (int t = n - 1; t >= 0; --t) {
        if (CKPT && t == H.s0 - 1) {
          enter_segment(t);
          hin_n = hist_in(H, t, tid);
          hout_n = hist_out(H, t, tid);
        }
        if (warp == 0) prefetch_history(H, t, lane);
        const float* pcur = lb[t & 1];
        float* pnext = lb[(t + 1) & 1];
        const float2 nw2 = f2s(wsc[t]);
        const float rn = hist_rn[t];
        float2 accc = f2s(0.f), accp = f2s(0.f);
        float bestp = -1.f;
        int bestq = 0x7fffffff;
#pragma unroll
        for (int k = 0; k < KB; ++k) {
          const int mid = tid + NT * k;
          float cb[16];
          tmem_ld16(tbase + 16 * k, cb);
          const float4 hi4 = hin_n, ho4 = hout_n;
          if (k + 1 < KB) {
            hin_n = hist_in(H, t, mid + NT);
            hout_n = hist_out(H, t, mid + NT);
          } else if (t >= 1) {
            hin_n = hist_in(H, t - 1, tid);
            hout_n = hist_out(H, t - 1, tid);
          }
          const float4 pv = reinterpret_cast<const float4*>(pcur)[mid];
          const float pl[4] = {pv.x, pv.y, pv.z, pv.w};
          const float nr[4] = {ho4.x + rn, ho4.y + rn, ho4.z + rn, ho4.w + rn};
          float pn[4];
#pragma unroll
          for (int g = 0; g < 2; ++g) {          // groups h = 2g, 2g+1 side by side
            const float2 np2 = g ? f2(hi4.z, hi4.w) : f2(hi4.x, hi4.y);
            float2 ssum = f2s(0.f);
#pragma unroll
            for (int lo = 0; lo < 4; ++lo) {
              const float2 c2 = f2(cb[bidx(2 * g, lo)], cb[bidx(2 * g + 1, lo)]);
              const float2 d = __fadd2_rn(c2, nw2);
              const float2 a = __ffma2_rn(__ffma2_rn(d, d, np2), neg1, f2s(nr[lo]));
              const float2 pp = __fmul2_rn(f2(ex2f(a.x), ex2f(a.y)), f2s(pl[lo]));
              ssum = __fadd2_rn(ssum, pp);
              accc = __ffma2_rn(pp, c2, accc);
              if constexpr (ARGMAX) {
                arg_better(bestp, bestq, pp.x, ((2 * g) << 14) | (mid << 2) | lo);
                arg_better(bestp, bestq, pp.y, ((2 * g + 1) << 14) | (mid << 2) | lo);
              }
            }
            accp = __fadd2_rn(accp, ssum);
            pn[2 * g] = ssum.x;
            pn[2 * g + 1] = ssum.y;
          }
          if (t >= 1) {
#pragma unroll
            for (int h = 0; h < 4; ++h) pnext[(h << HB) | mid] = pn[h];
          }
        }
        float a0 = warp_sum(accc.x + accc.y);
        float a1 = warp_sum(accp.x + accp.y);
        if constexpr (ARGMAX) warp_argmax(bestp, bestq);
        const int pb = t & 1;
        if (lane == 0) {
          part[(pb * 32 + warp) * NP] = a0;
          part[(pb * 32 + warp) * NP + 1] = a1;
          if constexpr (ARGMAX) { apart[pb * 32 + warp] = bestp; aidx[pb * 32 + warp] = bestq; }
        }
        __syncthreads();
        if (warp == 0) {   // the 16 partials combined by a butterfly: no serial tail before the next step
          const float s0 = bfly16_sum(part[(pb * 32 + (lane & 15)) * NP]);
          const float s1 = bfly16_sum(part[(pb * 32 + (lane & 15)) * NP + 1]);
          if (lane == 0) {
            check_posterior_mass(s1);
            if (P.out_soft) P.out_soft[seq * P.len + t] = s0 / (s1 * P.sk);
          }
          if constexpr (ARGMAX) {
            float bp = apart[pb * 32 + (lane & 15)];
            int bq = aidx[pb * 32 + (lane & 15)];
#pragma unroll
            for (int o = 8; o > 0; o >>= 1) {
              const float p2 = __shfl_xor_sync(0xffffffffu, bp, o);
              const int q2 = __shfl_xor_sync(0xffffffffu, bq, o);
              arg_better(bp, bq, p2, q2);
            }
            if (lane == 0 && P.out_argmax) P.out_argmax[seq * n + t] = bq;
          }
        }
      }
    } else {
      float Rrn = 0.f;
      double Cr = 0.0;   // log2 beta_t = -stored + Cr_t
      float4 hsn = hist_in(H, n - 1, tid);
      for (int t = n - 1; t >= 0; --t) {
        if (CKPT && t == H.s0 - 1) {
          enter_segment(t);
          hsn = hist_in(H, t, tid);
        }
        if (warp == 0) prefetch_history(H, t, lane);
        const float* ncur = lb[t & 1];
        float* nnext = lb[(t + 1) & 1];
        const float2 nw2 = f2s(wsc[t]);
        const double Csig = (t >= 1) ? hist_c[t - 1] : 0.0;
        const float K = (float)(Csig + Cr - l2Z);
        const bool last = (t == n - 1);
        float2 accc = f2s(0.f), accp = f2s(0.f);
        float bestp = -1.f;
        int bestq = 0x7fffffff;
        float tmin = INFINITY;
#pragma unroll
        for (int k = 0; k < KB; ++k) {
          const int mid = tid + NT * k;
          float cb[16];
          tmem_ld16(tbase + 16 * k, cb);
          const float hs[4] = {hsn.x, hsn.y, hsn.z, hsn.w};
          if (k + 1 < KB) hsn = hist_in(H, t, mid + NT);
          else if (t >= 1) hsn = hist_in(H, t - 1, tid);
          float nr[4];
          if (last) {
            nr[0] = nr[1] = nr[2] = nr[3] = 0.f;
          } else {
            const float4 rv = reinterpret_cast<const float4*>(ncur)[mid];
            nr[0] = rv.x; nr[1] = rv.y; nr[2] = rv.z; nr[3] = rv.w;
          }
          float nout[4];
#pragma unroll
          for (int g = 0; g < 2; ++g) {          // groups h = 2g, 2g+1 side by side
            float2 y[4];
#pragma unroll
            for (int lo = 0; lo < 4; ++lo) {
              const float2 d = __fadd2_rn(f2(cb[bidx(2 * g, lo)], cb[bidx(2 * g + 1, lo)]), nw2);
              y[lo] = __ffma2_rn(d, d, f2s(nr[lo]));
            }
            // the posterior directly, p = 2^(K - n_sigma - y'), one ex2 per state
            const float2 kh = __fadd2_rn(f2s(K), f2(-hs[2 * g], -hs[2 * g + 1]));
            float2 ssum = f2s(0.f);
#pragma unroll
            for (int lo = 0; lo < 4; ++lo) {
              const float2 a = __ffma2_rn(y[lo], neg1, kh);
              const float2 pp = f2(ex2f(a.x), ex2f(a.y));
              ssum = __fadd2_rn(ssum, pp);
              accc = __ffma2_rn(pp, f2(cb[bidx(2 * g, lo)], cb[bidx(2 * g + 1, lo)]), accc);
              if constexpr (ARGMAX) {
                arg_better(bestp, bestq, pp.x, ((2 * g) << 14) | (mid << 2) | lo);
                arg_better(bestp, bestq, pp.y, ((2 * g + 1) << 14) | (mid << 2) | lo);
              }
            }
            accp = __fadd2_rn(accp, ssum);
            // negated log rho_{t-1} = (K - n_sigma) - lg2 sum p (+inf, i.e. rho = 0, when the
            // group's posterior mass underflows; it then moves no posterior by more than that mass)
            nout[2 * g] = (kh.x - Rrn) - lg2f(ssum.x);
            nout[2 * g + 1] = (kh.y - Rrn) - lg2f(ssum.y);
          }
          if (t >= 1) {
#pragma unroll
            for (int h = 0; h < 4; ++h) nnext[(h << HB) | mid] = nout[h];
            tmin = fminf(tmin, fminf(fminf(nout[0], nout[1]), fminf(nout[2], nout[3])));
          }
        }
        float a0 = warp_sum(accc.x + accc.y);
        float a1 = warp_sum(accp.x + accp.y);
        tmin = -warp_max(-tmin);
        if constexpr (ARGMAX) warp_argmax(bestp, bestq);
        const int pb = t & 1;
        if (lane == 0) {
          part[(pb * 32 + warp) * NP] = a0;
          part[(pb * 32 + warp) * NP + 1] = a1;
          wmin[pb * 32 + warp] = tmin;
          if constexpr (ARGMAX) { apart[pb * 32 + warp] = bestp; aidx[pb * 32 + warp] = bestq; }
        }
        __syncthreads();
        if (warp == 0) {   // the 16 partials combined by a butterfly: no serial tail before the next step
          const float s0 = bfly16_sum(part[(pb * 32 + (lane & 15)) * NP]);
          const float s1 = bfly16_sum(part[(pb * 32 + (lane & 15)) * NP + 1]);
          if (lane == 0) {
            check_posterior_mass(s1);
            if (P.out_soft) P.out_soft[seq * P.len + t] = s0 / (s1 * P.sk);
          }
          if constexpr (ARGMAX) {
            float bp = apart[pb * 32 + (lane & 15)];
            int bq = aidx[pb * 32 + (lane & 15)];
#pragma unroll
            for (int o = 8; o > 0; o >>= 1) {
              const float p2 = __shfl_xor_sync(0xffffffffu, bp, o);
              const int q2 = __shfl_xor_sync(0xffffffffu, bq, o);
              arg_better(bp, bq, p2, q2);
            }
            if (lane == 0 && P.out_argmax) P.out_argmax[seq * n + t] = bq;
          }
        }
        Cr -= (double)Rrn;
        Rrn = bfly16_min(wmin[pb * 32 + (lane & 15)]);
      }
    }
    __syncthreads();
  }

  tmem_fence_before();
  __syncthreads();
  tmem_fence_after();
  if (warp == 0) tmem_dealloc512(tslot[0]);
}

// ------------------------------------------------------------ VJP pass, packed
// Forward (negated log sigma and the prefix expectation A), then backward
// (suffix expectation, G, dl/dw per step and the per-state codebook gradient).
// Tensor memory holds the codewords during the forward and the current
// sequence's codebook gradient during the backward, when the codewords stream
// from L2 (block-major lines, prefetched two units ahead).  The forward's A_t
// ping-pongs in global scratch (L2-resident); the histories go to HBM: the
// forward values in group order [t][j] (as in the soft pass) and A in
// block-major order [mid][h], written by the next forward step from the values
// it has just read, so that the backward loads one 16-byte vector per block
// (the log-domain backward takes the forward values in that order too).
//
// Backward in posterior space (POST): with u_t(q) and P_t(j) as in the soft
// pass and Bc_t the suffix expectation, the exchanged values are P_t(j) and
// W_t(j) = P_t(j) (Bc_t(j) - Q_t) (Q_t a running reference), so that
//     p_t(q) Bc-part = u_t(q) W_t(q mod J),
//     W_{t-1}(i) = sum_lo [ p_t(q) (h_t(q) - rB_t) + u_t(q) W_t(q mod J) ],
//     G_t(q) = p_t(q) (A_{t-1}(q >> 2) - K_t + gZ + h_t(q)) + u_t(q) W_t(q mod J),
// with no logarithm and no division per group.  The log-domain backward
// exchanges the negated log rho and Bc = W / P instead.  Both renormalise the
// posterior mass of every step (its sum drifts from 1 by the rounding of the
// two sweeps).
// RING: the backward's codewords through the shared-memory ring (full
// histories only), else streamed from L2 and prefetched two units ahead.
template <bool POST, bool CKPT, bool RING>
__global__ void __launch_bounds__(NT, 1) vjp_kernel(Params P) {
  static_assert(!(RING && CKPT), "the codeword ring runs with full histories");
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int n = P.n;

  extern __shared__ __align__(16) float smem[];
  float* ring = smem;                                  // RING: [NS][kStageFloats]
  float* sb = smem + (RING ? NS * kStageFloats : 0);   // [2][J] forward values / P or negated log rho
  float* lb[2] = {sb, sb + J};
  // per-warp partials of a step, [2 parities][32][8]:
  //   0: sum P(i) (A + Bc)   1: sum P(i) Bc   2: sum P(i)   3: min stored value
  //   4: sum G c             5: sum G
  float* rec = sb + 2 * J;
  uint32_t* tslot = reinterpret_cast<uint32_t*>(rec + 2 * 32 * 8);  // [4]
  // RING control: stage mbarriers, release counters, fills issued per stage, failure flag
  uint64_t* fullb = reinterpret_cast<uint64_t*>(tslot + 4);
  uint32_t* rcnt = reinterpret_cast<uint32_t*>(fullb + 4);
  uint32_t* rfill = rcnt + 4;
  uint32_t* rfail = rfill + 4;
  float* wsc = reinterpret_cast<float*>(tslot + 4 + (RING ? kRingCtlWords : 0));   // n: -w'
  float* gsc = wsc + n;                                // n: g / sk

  // Per-CTA histories (see History), full or checkpointed.  Full: the forward
  // values [n][J] (group order for the posterior space backward, block-major
  // inputs for the log-domain one) and A [n][J] (block-major inputs).
  // Checkpoints: the forward values and A of every K-th step in group order
  // [S][J] each, one segment of both histories [K][J] each, and save slots for
  // the backward messages [2][J] and the codebook gradient [4][J] while a
  // segment is recomputed.  Block-major input slots of step t live at index
  // t - 1 (full) or t - s0 (segment).
  History<CKPT> H{};
  float *hl_full = nullptr, *ha_full = nullptr, *ck_a = nullptr, *sg_a = nullptr;
  float *msave = nullptr, *gsave = nullptr;
  int s_last = 0;
  if constexpr (!CKPT) {
    hl_full = P.hist_l + (size_t)blockIdx.x * n * J;
    ha_full = P.hist_a + (size_t)blockIdx.x * n * J;
    H.full = hl_full;
  } else {
    const int K = P.ck, S = (n + K - 1) / K;
    float* base = P.hist_l + (size_t)blockIdx.x * (2 * S + 2 * K + 6) * J;
    H.ckpt = base;
    ck_a = base + (size_t)S * J;
    H.seg = base + (size_t)2 * S * J;
    sg_a = H.seg + (size_t)K * J;
    msave = sg_a + (size_t)K * J;
    gsave = msave + (size_t)2 * J;
    H.K = K;
    s_last = ((n - 1) / K) * K;
  }
  double* hist_c = P.hist_c + (size_t)blockIdx.x * n;
  float* hist_rn = P.hist_rn + (size_t)blockIdx.x * n;
  float* bcg[2] = {P.bc_g + (size_t)blockIdx.x * 2 * J, P.bc_g + (size_t)blockIdx.x * 2 * J + J};
  double* gcp = P.gc_part + (size_t)blockIdx.x * S;
  const float* __restrict__ cs_tm = P.cs_tm;
  const float2 neg1 = f2s(-1.f);

  if (warp == 0) tmem_alloc512(tslot);
  if (RING && tid == 0) {
    for (int s2 = 0; s2 < NS; ++s2) {
      mbar_init(&fullb[s2], 1);
      rcnt[s2] = 0;
      rfill[s2] = 0;
    }
    *rfail = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  tmem_fence_before();
  __syncthreads();
  tmem_fence_after();
  const uint32_t tbase = tslot[0] + ((uint32_t)(32 * (warp & 3)) << 16) + (uint32_t)(128 * (warp >> 2));
  for (int x = tid; x < S; x += NT) gcp[x] = 0.0;
  // ring position of the next block the backward reads (the same on every thread)
  uint32_t rstage = 0, rphase = 0;
  bool ring_ok = true;
  auto issue_fill = [&](uint32_t st, int k) {   // stage st <- block k
    if (P.ring_nofill) return;
    ring_fill(ring + st * kStageFloats, P.cs_rg + (size_t)k * kStageFloats, &fullb[st]);
    atomicAdd(&rfill[st], 1u);
  };

  // One forward step: step t-1's forward values (shared memory) and A (global
  // ping-pong) in, step t's out; history slots that are non-null receive step
  // t-1's values in block-major order (in_l, in_a), step t's in group order
  // (out_l) and the checkpoint copies (ck_lt, ck_at).  Returns the thread's
  // minimum of the stored values.
  auto forward_step = [&](int t, float Rn, float* in_l, float* in_a, float* out_l, float* ck_lt, float* ck_at) -> float {
      const float* nprev = lb[(t + 1) & 1];
      float* ncur = lb[t & 1];
      // A_t ping-pongs in global scratch (L2-resident); the history copy is block-major
      const float* aprev = bcg[(t + 1) & 1];
      float* acur = bcg[t & 1];
      const float2 nw2 = f2s(wsc[t]);
      const float2 g2 = f2s(gsc[t]);
      // A_{t-1} enters relative to its value at group 0, so that the stored
      // prefix expectations stay at the size of their spread over groups
      // instead of growing with t; the histories keep the stored values and
      // the backward subtracts the same reference.
      const float2 nrA = f2s((t > 0) ? -aprev[0] : 0.f);
      float tmin = INFINITY;
      float apn[4] = {0.f, 0.f, 0.f, 0.f};
      if (t > 0) {
#pragma unroll
        for (int h = 0; h < 4; ++h) apn[h] = aprev[(h << HB) | tid];
      }
#pragma unroll
      for (int k = 0; k < KB; ++k) {
        const int mid = tid + NT * k;
        float cb[16];
        tmem_ld16(tbase + 16 * k, cb);
        const float2 ap01 = f2(apn[0], apn[1]), ap23 = f2(apn[2], apn[3]);
        const float2 as01 = __fadd2_rn(ap01, nrA), as23 = __fadd2_rn(ap23, nrA);
        if (t > 0 && k + 1 < KB) {
#pragma unroll
          for (int h = 0; h < 4; ++h) apn[h] = aprev[(h << HB) | (mid + NT)];
        }
        float2 np01, np23;
        if (t == 0) {
          np01 = f2s(0.f); np23 = f2s(0.f);
        } else {
          np01 = f2(nprev[(0 << HB) | mid], nprev[(1 << HB) | mid]);
          np23 = f2(nprev[(2 << HB) | mid], nprev[(3 << HB) | mid]);
          // step t-1's values in block-major order [mid][h], as the backward reads them
          // (the posterior space backward takes the forward values in group order instead)
          if (in_l) reinterpret_cast<float4*>(in_l)[mid] = make_float4(np01.x, np01.y, np23.x, np23.y);
          if (in_a) reinterpret_cast<float4*>(in_a)[mid] = make_float4(ap01.x, ap01.y, ap23.x, ap23.y);
        }
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
        tmin = fminf(tmin, fminf(fminf(out[0], out[1]), fminf(out[2], out[3])));
        const float4 ov = make_float4(out[0], out[1], out[2], out[3]);
        const float4 av = make_float4(aout[0], aout[1], aout[2], aout[3]);
        reinterpret_cast<float4*>(ncur)[mid] = ov;
        reinterpret_cast<float4*>(acur)[mid] = av;
        if (out_l) reinterpret_cast<float4*>(out_l)[mid] = ov;
        if (ck_lt) reinterpret_cast<float4*>(ck_lt)[mid] = ov;
        if (ck_at) reinterpret_cast<float4*>(ck_at)[mid] = av;
      }
    return tmin;
  };

  for (int64_t seq = blockIdx.x; seq < P.n_seq; seq += gridDim.x) {
    const float* wq = P.w + seq * P.len;
    const float* gq = P.gsoft + seq * P.len;
    H.s0 = CKPT ? s_last : 0;
    for (int x = tid; x < n; x += NT) { wsc[x] = -wq[x] * P.sk; gsc[x] = gq[x] / P.sk; }
    // codewords into tensor memory for the forward
#pragma unroll
    for (int k = 0; k < KB; ++k) {
      float c16[16];
      ld_cb(cs_tm, tid + NT * k, c16);
      tmem_st16(tbase + 16 * k, c16);
    }
    tmem_wait_st();
    __syncthreads();

    // ------------------------------------------------------------ forward
    float Rn = 0.f;
    double C = 0.0;
    for (int t = 0; t < n; ++t) {
      C -= (double)Rn;
      float *in_l = nullptr, *in_a = nullptr, *out_l = nullptr, *ck_lt = nullptr, *ck_at = nullptr;
      if constexpr (!CKPT) {
        if (t >= 1) { in_l = POST ? nullptr : hl_full + (size_t)(t - 1) * J; in_a = ha_full + (size_t)(t - 1) * J; }
        if (POST) out_l = hl_full + (size_t)t * J;
      } else {
        if (t >= s_last) {
          if (t >= 1) { in_l = POST ? nullptr : H.seg + (size_t)(t - s_last) * J; in_a = sg_a + (size_t)(t - s_last) * J; }
          if (POST) out_l = H.seg + (size_t)(t - s_last) * J;
        }
        if ((t + 1) % H.K == 0 && t + 1 < n) {
          ck_lt = H.ckpt + (size_t)((t + 1) / H.K) * J;
          ck_at = ck_a + (size_t)((t + 1) / H.K) * J;
        }
      }
      float tmin = forward_step(t, Rn, in_l, in_a, out_l, ck_lt, ck_at);
      tmin = -warp_max(-tmin);
      if (lane == 0) rec[((t & 1) * 32 + warp) * 8 + 3] = tmin;
      if (tid == 0) { hist_c[t] = C; hist_rn[t] = Rn; }
      __syncthreads();
      Rn = bfly16_min(rec[((t & 1) * 32 + (lane & 15)) * 8 + 3]);
    }
    // log2 Z and Hbar = E[A_{n-1}]; the posterior space backward starts from
    // P_{n-1}(j) = 2^(Rn - stored_j) / sum, written in place
    double l2Z;
    float Hbar;
    {
      float* nfin = lb[(n - 1) & 1];
      const float* afin = bcg[(n - 1) & 1];
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
      if constexpr (POST) {
        const float inv = 1.f / a0;
        for (int j = tid; j < J; j += NT) nfin[j] = ex2f(Rn - nfin[j]) * inv;
      }
      __syncthreads();
    }
    const float gzq = P.gZ ? P.gZ[seq] : 0.f;
    const float2 nc2T = f2s(-P.two_over_T / P.sk);

    // tensor memory now accumulates this sequence's codebook gradient
    {
      float z16[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) z16[i] = 0.f;
#pragma unroll
      for (int k = 0; k < KB; ++k) tmem_st16(tbase + 16 * k, z16);
      tmem_wait_st();
    }

    // ------------------------------------------------------------ backward
    // Work unit = one h-pair g of one block k: 8 states, 8 codewords, 8 TMEM
    // columns; codewords are prefetched two units ahead, history values one block ahead.
    // K_t = sum_j P_t(j) (A_t(j) + Bc_t(j)) (P_t(j) the posterior of group j) is
    // formed from the same stored values one step earlier (K_{n-1} = Hbar), so
    // that rounding carried along the recursions cancels in G.  Stored Bc_t is
    // relative to rB, the posterior mean of the previous step's stored values.
    float Kt = Hbar, rB = 0.f;
    float cbn[8], cbm[8];
    if constexpr (RING) {
      // blocks 0 .. NS-1 of step n-1; every stage was released in the previous sequence
      if (tid == 0) {
        uint32_t st = rstage;
        for (int i = 0; i < NS; ++i) {
          issue_fill(st, i);
          st = (st + 1 == NS) ? 0 : st + 1;
        }
      }
    } else {
      ld_cb8(cs_tm, tid, 0, cbn);
      ld_cb8(cs_tm, tid, 1, cbm);
    }
    // block-major input slot of step tt (tt >= 1), full or in the segment
    auto in_slot = [&](const float* full, const float* seg, int tt) -> const float* {
      if constexpr (!CKPT) return full + (size_t)(tt - 1) * J;
      return seg + (size_t)(tt - H.s0) * J;
    };
    // block kk of step tt: A of step tt-1 in block-major order (free start: 0 for tt = 0)
    auto hist_a_at = [&](int tt, int kk) -> float4 {
      return (tt >= 1) ? reinterpret_cast<const float4*>(in_slot(ha_full, sg_a, tt))[tid + NT * kk]
                       : make_float4(0.f, 0.f, 0.f, 0.f);
    };
    // forward values of step tt-1 for block kk: four scalars of the group-order
    // history (posterior space) or one vector of the block-major one (log domain)
    auto hist_l_at = [&](int tt, int kk) -> float4 {
      if constexpr (POST) return hist_in(H, tt, tid + NT * kk);
      return (tt >= 1) ? reinterpret_cast<const float4*>(in_slot(hl_full, H.seg, tt))[tid + NT * kk]
                       : make_float4(0.f, 0.f, 0.f, 0.f);
    };
    // Before the backward of step t enters the segment below the one held: the
    // messages of step t and the codebook gradient are saved, the codewords put
    // back into tensor memory, that segment's forward recomputed from its
    // checkpoint, and gradient and messages restored.
    auto enter_segment = [&](int t) {
      if constexpr (!CKPT) return;
      copy_vec(msave, lb[t & 1], tid);
      copy_vec(msave + J, bcg[t & 1], tid);
#pragma unroll
      for (int k = 0; k < KB; ++k) {
        float v16[16];
        tmem_ld16(tbase + 16 * k, v16);
#pragma unroll
        for (int i = 0; i < 16; ++i) gsave[(size_t)(16 * k + i) * NT + tid] = v16[i];
        ld_cb(cs_tm, tid + NT * k, v16);
        tmem_st16(tbase + 16 * k, v16);
      }
      tmem_wait_st();
      H.s0 -= H.K;
      if (H.s0 > 0) {
        copy_vec(lb[(H.s0 + 1) & 1], H.ckpt + (size_t)(H.s0 / H.K) * J, tid);
        copy_vec(bcg[(H.s0 + 1) & 1], ck_a + (size_t)(H.s0 / H.K) * J, tid);
      }
      __syncthreads();
      for (int tt = H.s0; tt < H.s0 + H.K; ++tt) {
        float* sl = H.seg + (size_t)(tt - H.s0) * J;
        float* sa = sg_a + (size_t)(tt - H.s0) * J;
        forward_step(tt, hist_rn[tt], (!POST && tt >= 1) ? sl : nullptr, tt >= 1 ? sa : nullptr, POST ? sl : nullptr,
                     nullptr, nullptr);
        __syncthreads();
      }
#pragma unroll
      for (int k = 0; k < KB; ++k) {
        float v16[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) v16[i] = gsave[(size_t)(16 * k + i) * NT + tid];
        tmem_st16(tbase + 16 * k, v16);
      }
      tmem_wait_st();
      copy_vec(lb[t & 1], msave, tid);
      copy_vec(bcg[t & 1], msave + J, tid);
      __syncthreads();
    };
    float4 hin_n = hist_l_at(n - 1, 0), han = hist_a_at(n - 1, 0);
    float4 hout_n = POST ? hist_out(H, n - 1, tid) : make_float4(0.f, 0.f, 0.f, 0.f);
    float lsp = 0.f;     // log2 of the previous step's posterior mass (POST)
    float Rrn = 0.f;     // log domain: min of the previous step's stored values
    double Cr = 0.0;     // log domain: log2 beta_t = -stored + Cr_t
    for (int t = n - 1; t >= 0; --t) {
      if (CKPT && t == H.s0 - 1) {
        enter_segment(t);
        hin_n = hist_l_at(t, 0);
        han = hist_a_at(t, 0);
        if constexpr (POST) hout_n = hist_out(H, t, tid);
      }
      if (warp == 0) {
        if constexpr (POST) {
          prefetch_history(H, t, lane);
        } else if (t >= 2 && lane < 8 && (!CKPT || t - 1 >= H.s0)) {
          // the next step's block-major forward values (slot t - 2)
          constexpr uint32_t kChunk = J * sizeof(float) / 8;
          prefetch_l2_bulk(reinterpret_cast<const char*>(in_slot(hl_full, H.seg, t - 1)) + lane * kChunk, kChunk);
        }
      }
      const float* ncur = lb[t & 1];
      float* nnext = lb[(t + 1) & 1];
      const float* bcur = bcg[t & 1];
      float* bnext = bcg[(t + 1) & 1];
      const float nwt = wsc[t];
      const float2 nw2 = f2s(nwt);
      const float2 g2 = f2s(gsc[t]);
      const float2 gr2 = f2s(gsc[t] * P.sk);
      const bool last = (t == n - 1);
      const float rA = (t >= 1) ? in_slot(ha_full, sg_a, t)[0] : 0.f;   // the forward's reference
      const float hbt = Kt + rA - rB - gzq;
      // POST: 2^(n_t + Rn_t - x) / (posterior mass); log domain: K = log2 of 1/Z and the offsets
      const float nrs = POST ? hist_rn[t] - lsp : 0.f;
      float K = 0.f;
      if constexpr (!POST) K = (float)(((t >= 1) ? hist_c[t - 1] : 0.0) + Cr - l2Z);
      const float2 nrB2 = f2s(-rB);
      float2 accGd = f2s(0.f);   // sum_q G (c' - w')
      float2 accK = f2s(0.f), accB = f2s(0.f), accP = f2s(0.f);
      float tmin = INFINITY;
      float4 bvn = make_float4(0.f, 0.f, 0.f, 0.f);
      if (!last) bvn = reinterpret_cast<const float4*>(bcur)[tid];
#pragma unroll
      for (int k = 0; k < KB; ++k) {
        const int mid = tid + NT * k;
        if constexpr (RING) {
          if (ring_ok && !mbar_wait(&fullb[rstage], rphase)) {
            record_device_error(kErrTimeout);
            *rfail = 1;
            ring_ok = false;
          }
        }
        const float4* st4 = reinterpret_cast<const float4*>(ring + rstage * kStageFloats);
        float nr[4], bc[4];   // P and W (POST) or negated log rho and Bc
        if (last && !POST) {
          nr[0] = nr[1] = nr[2] = nr[3] = 0.f;
        } else {
          const float4 rv = reinterpret_cast<const float4*>(ncur)[mid];
          nr[0] = rv.x; nr[1] = rv.y; nr[2] = rv.z; nr[3] = rv.w;
        }
        if (last) {
          bc[0] = bc[1] = bc[2] = bc[3] = 0.f;
        } else {
          if constexpr (POST) {
            bc[0] = bvn.x; bc[1] = bvn.y; bc[2] = bvn.z; bc[3] = bvn.w;
          } else {
            bc[0] = bvn.x - rB; bc[1] = bvn.y - rB; bc[2] = bvn.z - rB; bc[3] = bvn.w - rB;
          }
        }
        if (!last && k + 1 < KB) bvn = reinterpret_cast<const float4*>(bcur)[mid + NT];
        const float4 hi4 = hin_n, ha4 = han, ho4 = hout_n;
        if (k + 1 < KB) {
          hin_n = hist_l_at(t, k + 1);
          han = hist_a_at(t, k + 1);
          if constexpr (POST) hout_n = hist_out(H, t, mid + NT);
        } else if (t >= 1) {
          hin_n = hist_l_at(t - 1, 0);
          han = hist_a_at(t - 1, 0);
          if constexpr (POST) hout_n = hist_out(H, t - 1, tid);
        }
        float lnr[4];   // POST: n_t(j) + Rn_t - log2 mass
        if constexpr (POST) {
          lnr[0] = ho4.x + nrs; lnr[1] = ho4.y + nrs; lnr[2] = ho4.z + nrs; lnr[3] = ho4.w + nrs;
        }
        float nout[4], bout[4];
#pragma unroll
        for (int g = 0; g < 2; ++g) {          // groups h = 2g, 2g+1 side by side
          float cb[8];
          if constexpr (RING) {
            const float4 q0 = st4[(2 * g) * NT + tid], q1 = st4[(2 * g + 1) * NT + tid];
            cb[0] = q0.x; cb[1] = q0.y; cb[2] = q0.z; cb[3] = q0.w;
            cb[4] = q1.x; cb[5] = q1.y; cb[6] = q1.z; cb[7] = q1.w;
          } else {
#pragma unroll
            for (int i = 0; i < 8; ++i) { cb[i] = cbn[i]; cbn[i] = cbm[i]; }
            // codewords two units after (k, g): block k+1 (or 0), same g
            const int nk = (k + 1 < KB) ? k + 1 : 0;
            ld_cb8(cs_tm, tid + NT * nk, g, cbm);
          }
          const float hs0 = g ? hi4.z : hi4.x, hs1 = g ? hi4.w : hi4.y;
          const float ha0 = g ? ha4.z : ha4.x, ha1 = g ? ha4.w : ha4.y;
          float gcb[8];
          tmem_ld8(tbase + 16 * k + 8 * g, gcb);
          const float2 ah = f2(ha0 - hbt, ha1 - hbt);   // A - K + gZ (+ rB in POST)
          if constexpr (POST) {
            const float2 np2 = f2(hs0, hs1);
            float2 Pn = f2s(0.f), Wn = f2s(0.f);
#pragma unroll
            for (int lo = 0; lo < 4; ++lo) {
              const float2 c2 = f2(cb[2 * lo], cb[2 * lo + 1]);
              const float2 dd = __fadd2_rn(c2, nw2);
              const float2 a = __ffma2_rn(__ffma2_rn(dd, dd, np2), neg1, f2s(lnr[lo]));
              const float2 u = f2(ex2f(a.x), ex2f(a.y));
              const float2 pp = __fmul2_rn(u, f2s(nr[lo]));           // posterior
              const float2 uw = __fmul2_rn(u, f2s(bc[lo]));           // u W
              const float2 v = __ffma2_rn(pp, __ffma2_rn(g2, c2, nrB2), uw);   // p (h - rB) + u W
              const float2 G = __ffma2_rn(pp, ah, v);
              Pn = __fadd2_rn(Pn, pp);
              Wn = __fadd2_rn(Wn, v);
              const float2 Gd = __fmul2_rn(G, dd);                    // G (c' - w')
              accGd = __fadd2_rn(accGd, Gd);
              float2 gc = f2(gcb[2 * lo], gcb[2 * lo + 1]);
              gc = __ffma2_rn(Gd, nc2T, __ffma2_rn(gr2, pp, gc));    // + g p + (2/T) G (w - c)
              gcb[2 * lo] = gc.x;
              gcb[2 * lo + 1] = gc.y;
            }
            nout[2 * g] = Pn.x; nout[2 * g + 1] = Pn.y;
            bout[2 * g] = Wn.x; bout[2 * g + 1] = Wn.y;
            accK = __ffma2_rn(Pn, f2(ha0, ha1), __fadd2_rn(accK, Wn));
            accB = __fadd2_rn(accB, Wn);
            accP = __fadd2_rn(accP, Pn);
          } else {
            float2 y[4], c2[4];
#pragma unroll
            for (int lo = 0; lo < 4; ++lo) {
              c2[lo] = f2(cb[2 * lo], cb[2 * lo + 1]);
              const float2 dd = __fadd2_rn(c2[lo], nw2);
              y[lo] = __ffma2_rn(dd, dd, f2s(nr[lo]));
            }
            // the posterior directly, p = 2^(K - n_sigma - y'), one ex2 per state
            const float2 kh = __fadd2_rn(f2s(K), f2(-hs0, -hs1));
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
              float2 gc = f2(gcb[2 * lo], gcb[2 * lo + 1]);
              gc = __ffma2_rn(Gd, nc2T, __ffma2_rn(gr2, pp, gc));       // + g p + (2/T) G (w - c)
              gcb[2 * lo] = gc.x;
              gcb[2 * lo + 1] = gc.y;
            }
            // negated log rho_{t-1} = (K - n_sigma) - lg2 sum p; a group whose posterior mass
            // underflows gets rho = 0 (+inf) and Bc = 0, moving no posterior by more than that mass
            nout[2 * g] = (kh.x - Rrn) - lg2f(ssum.x);
            nout[2 * g + 1] = (kh.y - Rrn) - lg2f(ssum.y);
            bout[2 * g] = __fdividef(num.x, fmaxf(ssum.x, FLT_MIN));   // num = 0 when sum p = 0
            bout[2 * g + 1] = __fdividef(num.y, fmaxf(ssum.y, FLT_MIN));
            // posterior of the two step t-1 groups, P(i) = sum_lo p
            const float2 pg = ssum, bo = f2(bout[2 * g], bout[2 * g + 1]);
            accK = __ffma2_rn(pg, __fadd2_rn(f2(ha0, ha1), bo), accK);
            accB = __ffma2_rn(pg, bo, accB);
            accP = __fadd2_rn(accP, pg);
          }
          tmem_st8(tbase + 16 * k + 8 * g, gcb);
        }
        if constexpr (RING) {
          // this warp has read block k's stage; the last of the 16 warps refills it
          // with block k + NS (in this step or the next; none after the last step)
          __syncwarp();
          if (lane == 0) {
            const uint32_t old = ring_release(&rcnt[rstage]);
            if ((old & 15) == 15 && !(t == 0 && k + NS >= KB) && ring_ok) {
              asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
              issue_fill(rstage, (k + NS) % KB);
            }
          }
          if (++rstage == NS) {
            rstage = 0;
            rphase ^= 1;
          }
        }
        if (t >= 1) {
#pragma unroll
          for (int h = 0; h < 4; ++h) {
            nnext[(h << HB) | mid] = nout[h];
            bnext[(h << HB) | mid] = bout[h];
          }
          if constexpr (!POST) tmin = fminf(tmin, fminf(fminf(nout[0], nout[1]), fminf(nout[2], nout[3])));
        }
      }
      tmem_wait_st();
      const float a0 = warp_sum(accGd.x + accGd.y);
      const float kk = warp_sum(accK.x + accK.y);
      const float kb = warp_sum(accB.x + accB.y);
      const float kp = warp_sum(accP.x + accP.y);
      if constexpr (!POST) tmin = -warp_max(-tmin);
      const int pb = t & 1;
      if (lane == 0) {
        float* r = rec + (pb * 32 + warp) * 8;
        *reinterpret_cast<float4*>(r) = make_float4(kk, kb, kp, tmin);
        r[4] = a0;
      }
      __syncthreads();
      if (tid == 0) {
        float s0 = 0.f;
#pragma unroll
        for (int w2 = 0; w2 < NT / 32; ++w2) s0 += rec[(pb * 32 + w2) * 8 + 4];
        // dl/dw_t = (2/T) sum_q G (c - w_t) = (2/T) sum_q G (c' - w') / sk
        P.grad_w[seq * P.len + t] = P.two_over_T * s0 / P.sk;
      }
      {
        const float4 r = *reinterpret_cast<const float4*>(rec + (pb * 32 + (lane & 15)) * 8);
        const float sp = bfly16_sum(r.z);   // sum_q p_t(q), 1 up to rounding
        Kt = bfly16_sum(r.x) / sp;
        rB = bfly16_sum(r.y) / sp;
        if (tid == 0) check_posterior_mass(sp);
        // Forward and backward carry different rounding, so the posterior sum
        // drifts from 1 along the sweep; dividing it out renormalises every
        // next step.
        if constexpr (POST) {
          lsp = lg2f(sp);
        } else {
          Cr -= (double)Rrn;
          Rrn = bfly16_min(r.w);
          Cr -= (double)lg2f(sp);
        }
      }
    }

    // fold this sequence's codebook gradient into the CTA partial
#pragma unroll
    for (int k = 0; k < KB; ++k) {
      const int mid = tid + NT * k;
      float gcb[16];
      tmem_ld16(tbase + 16 * k, gcb);
      double* dst = gcp + (size_t)mid * 16;
#pragma unroll
      for (int i = 0; i < 16; ++i) dst[i] += (double)gcb[i];
    }
    __syncthreads();
  }

  tmem_fence_before();
  __syncthreads();
  tmem_fence_after();
  if (RING && tid == 0 && *rfail) {
    // after a wait that ran out: the copies still in flight land before the CTA exits
    for (int s2 = 0; s2 < NS; ++s2)
      if (rfill[s2] > 0) mbar_wait(&fullb[s2], (rfill[s2] - 1) & 1);
  }
  if (warp == 0) tmem_dealloc512(tslot[0]);
}

// ------------------------------------------------------------ Viterbi
// The T -> 0 decode in the same block layout: per step and forward group
// j = (mid << 2) | lo, mu_t(j) = min_h delta_t((h << 14) | j) with
// delta_t(q) = fl(mu_{t-1}(q >> 2) + fl(fl(w_t - c(q))^2)) (delta_0 = q_0),
// the lowest h winning ties.  The four 2-bit backpointers of a block form one
// byte per step.  A CTA decodes a batch of up to TB sequences, then traces
// them back in parallel (one thread per sequence).  The arithmetic is the
// prescribed fp32 sequence in scalar IEEE round-to-nearest operations that
// are never fused (the packed f32x2 forms gave 1-ulp differences in the
// accumulated cost on this hardware, so they are not used here).
struct VParams {
  const float* w;       // [n_seq][len]
  const float* cb_raw;  // block-major raw codebook [4096][16]
  int32_t* out_states;  // [n_seq][n]
  float* out_cost;      // [n_seq] or null
  uint8_t* bp;          // [grid][TB][n][NMID]
  int64_t n_seq, len;
  int n, tb;
};

__global__ void __launch_bounds__(NT, 1) viterbi_kernel(VParams P) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  constexpr int nwarps = NT / 32;
  const int n = P.n, TB = P.tb;
  extern __shared__ __align__(16) float smem[];
  float* mb[2] = {smem, smem + J};
  float* redv = smem + 2 * J;                          // [32]
  int* redq = reinterpret_cast<int*>(redv + 32);       // [32]
  int* fin = redq + 32;                                // [TB] final state per sequence of the batch
  uint32_t* tslot = reinterpret_cast<uint32_t*>(fin + 64);  // [4]
  float* wsm = reinterpret_cast<float*>(tslot + 4);    // n: w
  uint8_t* bp = P.bp + (size_t)blockIdx.x * TB * n * NMID;

  if (warp == 0) tmem_alloc512(tslot);
  tmem_fence_before();
  __syncthreads();
  tmem_fence_after();
  const uint32_t tbase = tslot[0] + ((uint32_t)(32 * (warp & 3)) << 16) + (uint32_t)(128 * (warp >> 2));
#pragma unroll
  for (int k = 0; k < KB; ++k) {
    float c16[16];
    ld_cb(P.cb_raw, tid + NT * k, c16);
    tmem_st16(tbase + 16 * k, c16);
  }
  tmem_wait_st();

  const int64_t stride = (int64_t)gridDim.x;
  for (int64_t base = blockIdx.x; base < P.n_seq; base += stride * TB) {
    int nb = 0;
    for (int i = 0; i < TB; ++i, ++nb) {
      const int64_t seq = base + i * stride;
      if (seq >= P.n_seq) break;
      const float* wq = P.w + seq * P.len;
      for (int x = tid; x < n; x += NT) wsm[x] = wq[x];
      __syncthreads();
      uint8_t* bpi = bp + (size_t)i * n * NMID;
      float bestv = INFINITY;
      int bestq = 0x7fffffff;
      for (int t = 0; t < n; ++t) {
        const float* mprev = mb[(t + 1) & 1];
        float* mcur = mb[t & 1];
        const float wv = wsm[t];
        const bool last = (t == n - 1);
#pragma unroll
        for (int k = 0; k < KB; ++k) {
          const int mid = tid + NT * k;
          float cb[16];
          tmem_ld16(tbase + 16 * k, cb);
          float2 mp01 = f2s(0.f), mp23 = f2s(0.f);
          if (t > 0) {
            mp01 = f2(mprev[(0 << HB) | mid], mprev[(1 << HB) | mid]);
            mp23 = f2(mprev[(2 << HB) | mid], mprev[(3 << HB) | mid]);
          }
          float mout[4];
          uint32_t byte = 0;
#pragma unroll
          for (int lo = 0; lo < 4; ++lo) {
            // scalar IEEE operations in the prescribed order: q = fl(fl(w - c)^2), delta = fl(mu + q)
            float e[4];
#pragma unroll
            for (int h = 0; h < 4; ++h) {
              const float d = __fsub_rn(wv, cb[bidx(h, lo)]);
              e[h] = __fmul_rn(d, d);
            }
            if (t > 0) {
              e[0] = __fadd_rn(mp01.x, e[0]); e[1] = __fadd_rn(mp01.y, e[1]);
              e[2] = __fadd_rn(mp23.x, e[2]); e[3] = __fadd_rn(mp23.y, e[3]);
            }
            const float2 e01 = f2(e[0], e[1]), e23 = f2(e[2], e[3]);
            float b = e01.x;
            uint32_t bh = 0;
            if (e01.y < b) { b = e01.y; bh = 1; }
            if (e23.x < b) { b = e23.x; bh = 2; }
            if (e23.y < b) { b = e23.y; bh = 3; }
            mout[lo] = b;
            byte |= bh << (2 * lo);
            if (last) {
              const float dv[4] = {e01.x, e01.y, e23.x, e23.y};
#pragma unroll
              for (int h = 0; h < 4; ++h) {
                const int q = (h << 14) | (mid << 2) | lo;
                if (dv[h] < bestv || (dv[h] == bestv && q < bestq)) { bestv = dv[h]; bestq = q; }
              }
            }
          }
          reinterpret_cast<float4*>(mcur)[mid] = make_float4(mout[0], mout[1], mout[2], mout[3]);
          if (!last) bpi[(size_t)t * NMID + mid] = (uint8_t)byte;
        }
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
    // trace the batch back, one thread per sequence
    if (tid < nb) {
      const int i = tid;
      const int64_t seq = base + i * stride;
      const uint8_t* bpi = bp + (size_t)i * n * NMID;
      int32_t* out = P.out_states + seq * n;
      int st = fin[i];
      for (int t = n - 1; t >= 0; --t) {
        out[t] = st;
        if (t > 0) {
          const int jp = st >> 2;   // group of the predecessors at step t-1
          const int h = (bpi[(size_t)(t - 1) * NMID + (jp >> 2)] >> (2 * (jp & 3))) & 3;
          st = jp | (h << 14);
        }
      }
    }
    __syncthreads();
  }

  tmem_fence_before();
  __syncthreads();
  tmem_fence_after();
  if (warp == 0) tmem_dealloc512(tslot[0]);
}

}  // namespace l16
}  // namespace bcjr
