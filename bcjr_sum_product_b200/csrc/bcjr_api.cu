// Host side of the C ABI declared in include/bcjr.h: argument validation,
// stream-ordered scratch allocation, kernel selection and launch.
#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstdlib>
#include <cstring>
#include <atomic>
#include <mutex>

#include <cuda_runtime.h>

#include "bcjr.h"
#include "bcjr_kernels.cuh"
#include "bcjr_l16.cuh"
#include "bcjr_l16c.cuh"
#include "bcjr_l16v2.cuh"

namespace {

using bcjr::SweepParams;
using bcjr::ViterbiParams;

constexpr int kMaxL = 16;
constexpr int kMaxD = 6;
constexpr int64_t kMaxLen = 8192;
constexpr size_t kMaxDynSmem = 227 * 1024;

struct Shape {
  int L, k, V, D, B, J, S, n;
  int64_t n_seq, len;
};

bool fault_alloc() {
  const char* e = std::getenv("BCJR_FAULT_ALLOC");
  return e && e[0] == '1';
}

// Kernels this library has launched in the process (bcjr_launch_count).
std::atomic<uint64_t> g_launch_count{0};
void counted_launch(int n = 1) { g_launch_count.fetch_add((uint64_t)n, std::memory_order_relaxed); }

// Library-private stream-ordered pool per device.  Scratch freed at the end of
// a call stays mapped in the pool (release threshold = unlimited), so the next
// call of the same size reuses it instead of mapping gigabytes again.
constexpr int kMaxPoolDevices = 64;
std::mutex g_pool_mu;
cudaMemPool_t g_pool[kMaxPoolDevices] = {};

int scratch_alloc(void** mem, size_t bytes, cudaStream_t st) {
  if (fault_alloc()) return BCJR_ERR_CUDA;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxPoolDevices) {
    cudaGetLastError();
    return BCJR_ERR_CUDA;
  }
  cudaMemPool_t pool;
  {
    std::lock_guard<std::mutex> lk(g_pool_mu);
    if (g_pool[dev] == nullptr) {
      cudaMemPoolProps props = {};
      props.allocType = cudaMemAllocationTypePinned;
      props.location.type = cudaMemLocationTypeDevice;
      props.location.id = dev;
      cudaMemPool_t p;
      if (cudaMemPoolCreate(&p, &props) != cudaSuccess) {
        cudaGetLastError();
        return BCJR_ERR_CUDA;
      }
      uint64_t thr = UINT64_MAX;
      cudaMemPoolSetAttribute(p, cudaMemPoolAttrReleaseThreshold, &thr);
      g_pool[dev] = p;
    }
    pool = g_pool[dev];
  }
  if (cudaMallocFromPoolAsync(mem, bytes, pool, st) != cudaSuccess) {
    cudaGetLastError();
    return BCJR_ERR_CUDA;
  }
  return BCJR_OK;
}

int check_dev_ptr(const void* p, bool nullable) {
  if (p == nullptr) return nullable ? BCJR_OK : BCJR_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(p) % 4 != 0) return BCJR_ERR_INVALID_ARG;
  cudaPointerAttributes a;
  cudaError_t e = cudaPointerGetAttributes(&a, p);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return BCJR_ERR_INVALID_ARG;
  }
  if (a.type != cudaMemoryTypeDevice && a.type != cudaMemoryTypeManaged) return BCJR_ERR_INVALID_ARG;
  return BCJR_OK;
}

int check_shape(int64_t n_seq, int64_t len, int L, int k, int V, Shape* sh) {
  if (n_seq < 0 || len < 1 || k < 1 || V < 1 || L < 1) return BCJR_ERR_INVALID_ARG;
  if (len % V != 0) return BCJR_ERR_INVALID_ARG;
  if ((int64_t)k * V > L) return BCJR_ERR_INVALID_ARG;
  if (L > kMaxL) return BCJR_ERR_UNSUPPORTED;
  if (V != 1 && V != 2 && V != 4) return BCJR_ERR_UNSUPPORTED;
  if (k * V > kMaxD) return BCJR_ERR_UNSUPPORTED;
  if (len > kMaxLen) return BCJR_ERR_UNSUPPORTED;
  sh->L = L; sh->k = k; sh->V = V; sh->D = k * V; sh->B = 1 << sh->D;
  sh->J = 1 << (L - sh->D); sh->S = 1 << L; sh->n = (int)(len / V);
  sh->n_seq = n_seq; sh->len = len;
  return BCJR_OK;
}

// BCJR_GENERIC_ONLY=1 routes every call to the generic kernels (used by tests
// that compare the specialised kernels against them).
bool generic_only() {
  const char* e = std::getenv("BCJR_GENERIC_ONLY");
  return e && e[0] == '1';
}

int check_T(float T) { return (std::isfinite(T) && T > 0.f) ? BCJR_OK : BCJR_ERR_INVALID_ARG; }

// Carves one stream-ordered allocation into 256-byte aligned pieces.
struct Arena {
  size_t off = 0;
  char* base = nullptr;
  template <class T>
  T* take(size_t count) {
    size_t bytes = (count * sizeof(T) + 255) & ~size_t(255);
    T* p = reinterpret_cast<T*>(base ? base + off : nullptr);
    off += bytes;
    return p;
  }
};

// Generic kernels: about 32 states per thread per step (J groups of B members),
// 32 to 512 threads.  Small trellises then run several small CTAs per SM instead
// of one large CTA whose per-step barrier and reductions outweigh its work.
int threads_for(int J, int B) {
  const long w = (long)J * B / 32;
  const int t = w < 32 ? 32 : (w > bcjr::kMaxThreads ? bcjr::kMaxThreads : (int)w);
  return (t + 31) / 32 * 32;
}

// Resident CTAs of `kernel` over the device (at most n_seq).  A failed query
// clears the CUDA error it leaves, so that it is not reported by a later call.
template <class K>
int grid_for(K kernel, int threads, size_t smem, int64_t n_seq, int* grid) {
  int dev = 0, nsm = 0, per = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
      cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess ||
      cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per, kernel, threads, smem) != cudaSuccess) {
    cudaGetLastError();
    return BCJR_ERR_CUDA;
  }
  if (per < 1) return BCJR_ERR_UNSUPPORTED;
  int64_t g = (int64_t)per * nsm;
  if (g > n_seq) g = n_seq;
  *grid = (int)(g < 1 ? 1 : g);
  return BCJR_OK;
}

// Scratch budget of one call: half of the free device memory, at most 24 GiB.
size_t scratch_budget() {
  size_t free_b = 0, total_b = 0;
  if (cudaMemGetInfo(&free_b, &total_b) != cudaSuccess) {
    cudaGetLastError();
    return (size_t)1 << 30;
  }
  const size_t cap = (size_t)24 << 30;
  return free_b / 2 < cap ? free_b / 2 : cap;
}

// Fewer resident CTAs when their per-CTA scratch (histories grow with the
// sequence length) would exceed the scratch budget.
void cap_grid_by_memory(int* grid, size_t per_cta_bytes) {
  if (per_cta_bytes == 0) return;
  size_t g = scratch_budget() / per_cta_bytes;
  if (g < 1) g = 1;
  if ((size_t)*grid > g) *grid = (int)g;
}

// Segment length of the checkpointed L = 16 histories: 0 (full histories)
// while every resident CTA's full history fits the scratch budget, else
// ceil(sqrt(n)).  BCJR_L16_CKPT=0 keeps full histories (fewer resident CTAs
// instead); BCJR_L16_CKPT=K > 0 forces segments of K steps.
int l16_checkpoint_len(int n, int grid, size_t full_bytes_per_cta) {
  const char* e = std::getenv("BCJR_L16_CKPT");
  if (e && e[0] != '\0') {
    const long v = std::strtol(e, nullptr, 10);
    if (v <= 0) return 0;
    return (int)(v < n ? v : n);
  }
  if ((double)grid * (double)full_bytes_per_cta <= (double)scratch_budget()) return 0;
  int K = (int)std::ceil(std::sqrt((double)n));
  return K < 1 ? 1 : K;
}

// ----------------------------------------------------------------- sweep
using SweepKernel = void (*)(SweepParams);

template <int MODE>
SweepKernel pick_sweep(int V, int D) {
#define BCJR_CASE(VV, DD) \
  if (V == VV && D == DD) return bcjr::bcjr_sweep_kernel<VV, DD, MODE>;
  BCJR_CASE(1, 1) BCJR_CASE(1, 2) BCJR_CASE(1, 3) BCJR_CASE(1, 4) BCJR_CASE(1, 5) BCJR_CASE(1, 6)
  BCJR_CASE(2, 2) BCJR_CASE(2, 4) BCJR_CASE(2, 6)
  BCJR_CASE(4, 4)
#undef BCJR_CASE
  return nullptr;
}

struct SweepArgs {
  const float* w;
  const float* c;
  float T;
  const float* gsoft;
  const float* gZ;
  float* out_soft;
  float* out_logZ;
  int32_t* out_argmax;
  float* grad_w;
  float* grad_c;
};

// Measured alternatives of the L = 16, k = 2, V = 1 kernels, selected per call.
// BCJR_L16_VJP=cluster runs the VJP on clusters of two CTAs (bcjr_l16c.cuh)
// instead of one CTA per sequence; BCJR_L16_VJP=l2 streams the VJP backward's
// codewords from L2 instead of the shared-memory ring (the ring is the default
// wherever it fits: full histories and shared memory).  The backward sweeps run
// in posterior space for the soft codeword and in log domain for the VJP (the
// faster of the two for each); BCJR_L16_BWD=post or =log selects one of them for
// both.  BCJR_L16_RING_TEST_NOFILL=1 (tests only) never fills the ring, so that
// its bounded waits run out and the call reports BCJR_ERR_TIMEOUT.
bool l16_vjp_cluster() {
  const char* e = std::getenv("BCJR_L16_VJP");
  return e && std::strcmp(e, "cluster") == 0;
}
bool l16_vjp_ring() {
  const char* e = std::getenv("BCJR_L16_VJP");
  return !(e && std::strcmp(e, "l2") == 0);
}
bool l16_ring_test_nofill() {
  const char* e = std::getenv("BCJR_L16_RING_TEST_NOFILL");
  return e && std::strcmp(e, "1") == 0;
}
// BCJR_L16_EX2=fma computes one of the three exponentials of each soft-pass
// forward group on the FMA pipe (posterior-space soft kernel only).
bool l16_fma_ex2() {
  const char* e = std::getenv("BCJR_L16_EX2");
  return e && std::strcmp(e, "fma") == 0;
}
bool l16_posterior_backward(bool vjp) {
  const char* e = std::getenv("BCJR_L16_BWD");
  if (e && std::strcmp(e, "post") == 0) return true;
  if (e && std::strcmp(e, "log") == 0) return false;
  return !vjp;
}

// L = 16, D = 2, V = 1 VJP on clusters of two CTAs (bcjr_l16c.cuh).  Returns
// BCJR_ERR_UNSUPPORTED, with nothing launched, when no cluster fits an SM pair.
int run_l16c_vjp(const Shape& sh, const SweepArgs& a, cudaStream_t st) {
  namespace K = bcjr::l16c;
  const size_t smem = sizeof(float) * K::smem_floats(sh.n);
  if (smem > kMaxDynSmem) return BCJR_ERR_UNSUPPORTED;
  if (cudaFuncSetAttribute(K::vjp_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess) {
    cudaGetLastError();
    return BCJR_ERR_UNSUPPORTED;
  }
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = K::NC;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.blockDim = dim3(K::NT, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int dev = 0, nsm = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
    cudaGetLastError();
    return BCJR_ERR_CUDA;
  }
  cfg.gridDim = dim3((unsigned)(K::NC * (nsm / K::NC)), 1, 1);
  int max_clusters = 0;
  if (cudaOccupancyMaxActiveClusters(&max_clusters, K::vjp_kernel, &cfg) != cudaSuccess) {
    cudaGetLastError();
    return BCJR_ERR_UNSUPPORTED;
  }
  if (max_clusters < 1) return BCJR_ERR_UNSUPPORTED;
  int ncl = (int)std::min<int64_t>(max_clusters, sh.n_seq);
  cap_grid_by_memory(&ncl, sizeof(float) * (size_t)K::NC * 2 * sh.n * K::JL +
                               (sizeof(double) + sizeof(float)) * sh.n + sizeof(double) * K::S);
  K::Params P{};
  auto layout = [&](Arena& ar) {
    P.cs_tm = ar.take<float>(K::S);
    P.hist_l = ar.take<float>((size_t)K::NC * ncl * sh.n * K::JL);
    P.hist_a = ar.take<float>((size_t)K::NC * ncl * sh.n * K::JL);
    P.hist_c = ar.take<double>((size_t)ncl * sh.n);
    P.hist_r = ar.take<float>((size_t)ncl * sh.n);
    P.gc_part = ar.take<double>((size_t)ncl * K::S);
  };
  Arena sizing;
  layout(sizing);
  void* mem = nullptr;
  if (int arc = scratch_alloc(&mem, sizing.off, st)) return arc;
  Arena ar;
  ar.base = static_cast<char*>(mem);
  layout(ar);
  P.w = a.w; P.gsoft = a.gsoft; P.gZ = a.gZ; P.grad_w = a.grad_w;
  P.n_seq = sh.n_seq; P.len = sh.len; P.n = sh.n;
  P.sk = (float)std::sqrt(1.4426950408889634 / (double)a.T);
  P.two_over_T = (float)(2.0 / (double)a.T);
  cfg.gridDim = dim3((unsigned)(K::NC * ncl), 1, 1);
  bcjr::l16::make_block_codebook<<<K::S / 256, 256, 0, st>>>(a.c, P.sk, const_cast<float*>(P.cs_tm));
  counted_launch();
  cudaError_t ke = cudaLaunchKernelEx(&cfg, K::vjp_kernel, P);
  if (ke == cudaSuccess) {
    bcjr::l16::reduce_block_gc<<<K::S / 256, 256, 0, st>>>(P.gc_part, ncl, a.grad_c);
    counted_launch(2);
  }
  cudaError_t le = cudaGetLastError();
  cudaError_t fe = cudaFreeAsync(mem, st);
  if (ke != cudaSuccess || le != cudaSuccess || fe != cudaSuccess) return BCJR_ERR_CUDA;
  return BCJR_OK;
}

// L = 16, D = 2, V = 1: the block-layout kernel of bcjr_l16.cuh.
template <int MODE>
int run_l16(const Shape& sh, const SweepArgs& a, cudaStream_t st) {
  namespace K = bcjr::l16;
  constexpr bool VJP = MODE == bcjr::MODE_VJP;
  if (VJP && l16_vjp_cluster()) {
    const int rc = run_l16c_vjp(sh, a, st);
    if (rc != BCJR_ERR_UNSUPPORTED) return rc;
  }
  const bool post = l16_posterior_backward(VJP);
  const bool fma = post && l16_fma_ex2();
  const bool am = a.out_argmax != nullptr;
  auto pick = [&](bool ckpt, bool ring) -> void (*)(K::Params) {
#define BCJR_SOFT(AM, PO, FM) \
  (ckpt ? K::soft_kernel<AM, PO, FM, true> : K::soft_kernel<AM, PO, FM, false>)
    if (VJP) {
      if (ckpt) return post ? K::vjp_kernel<true, true, false> : K::vjp_kernel<false, true, false>;
      if (post) return ring ? K::vjp_kernel<true, false, true> : K::vjp_kernel<true, false, false>;
      return ring ? K::vjp_kernel<false, false, true> : K::vjp_kernel<false, false, false>;
    }
    if (fma) return am ? BCJR_SOFT(true, true, true) : BCJR_SOFT(false, true, true);
    if (post) return am ? BCJR_SOFT(true, true, false) : BCJR_SOFT(false, true, false);
    return am ? BCJR_SOFT(true, false, false) : BCJR_SOFT(false, false, false);
#undef BCJR_SOFT
  };
  // state ping-pong, per-warp partials, TMEM slot, per-step weights (and gradients),
  // and for the VJP with the codeword ring its stages and their control words
  auto smem_for = [&](bool ring) {
    return sizeof(float) * ((size_t)2 * K::J + (VJP ? 2 * 32 * 8 : 64 + 2 * 32 * 2 + 64 + 64) + 4 +
                            (VJP ? 2 : 1) * (size_t)sh.n +
                            (ring ? (size_t)K::NS * K::kStageFloats + K::kRingCtlWords : 0));
  };
  bool ring = VJP && l16_vjp_ring() && smem_for(true) <= kMaxDynSmem;
  size_t smem = smem_for(ring);
  if (smem > kMaxDynSmem) return BCJR_ERR_UNSUPPORTED;
  void (*kern)(K::Params) = pick(false, ring);
  int grid = 0;
  int rc = grid_for(kern, K::NT, smem, sh.n_seq, &grid);
  if (rc != BCJR_OK) return rc;
  // histories: full ([n][J] per CTA, twice for the VJP) or checkpointed (segments of ck steps)
  const size_t full_cta = sizeof(float) * (size_t)sh.n * K::J * (VJP ? 2 : 1);
  const int ck = l16_checkpoint_len(sh.n, grid, full_cta);
  if (ck) {
    ring = false;
    smem = smem_for(false);
    kern = pick(true, false);
    if ((rc = grid_for(kern, K::NT, smem, sh.n_seq, &grid)) != BCJR_OK) return rc;
  }
  const size_t nseg = ck ? (size_t)((sh.n + ck - 1) / ck) : 0;
  const size_t hist_cta_floats =
      ck ? (size_t)K::J * (VJP ? 2 * nseg + 2 * (size_t)ck + 6 : nseg + (size_t)ck + 1) : (size_t)sh.n * K::J;
  cap_grid_by_memory(&grid, sizeof(float) * hist_cta_floats * (ck || !VJP ? 1 : 2) +
                                (sizeof(double) + sizeof(float)) * sh.n +
                                (VJP ? sizeof(float) * 2 * K::J + sizeof(double) * K::S : 0));
  K::Params P{};
  auto layout = [&](Arena& ar) {
    P.cs_tm = ar.take<float>(K::S);
    P.cs_rg = ring ? ar.take<float>(K::S) : nullptr;
    P.hist_l = ar.take<float>((size_t)grid * hist_cta_floats);
    P.hist_a = (VJP && !ck) ? ar.take<float>((size_t)grid * hist_cta_floats) : nullptr;
    P.hist_c = ar.take<double>((size_t)grid * sh.n);
    P.hist_rn = ar.take<float>((size_t)grid * sh.n);
    P.bc_g = VJP ? ar.take<float>((size_t)grid * 2 * K::J) : nullptr;
    P.gc_part = VJP ? ar.take<double>((size_t)grid * K::S) : nullptr;
  };
  Arena sizing;
  layout(sizing);
  void* mem = nullptr;
  if (int arc = scratch_alloc(&mem, sizing.off, st)) return arc;
  Arena ar;
  ar.base = static_cast<char*>(mem);
  layout(ar);
  P.w = a.w; P.gsoft = a.gsoft; P.gZ = a.gZ;
  P.out_soft = a.out_soft; P.out_logZ = a.out_logZ; P.out_argmax = a.out_argmax; P.grad_w = a.grad_w;
  P.n_seq = sh.n_seq; P.len = sh.len; P.n = sh.n; P.ck = ck;
  P.sk = (float)std::sqrt(1.4426950408889634 / (double)a.T);
  P.two_over_T = (float)(2.0 / (double)a.T);
  P.ring_nofill = (ring && l16_ring_test_nofill()) ? 1 : 0;
  K::make_block_codebook<<<K::S / 256, 256, 0, st>>>(a.c, P.sk, const_cast<float*>(P.cs_tm));
  if (ring) K::make_ring_codebook<<<K::S / 256, 256, 0, st>>>(P.cs_tm, const_cast<float*>(P.cs_rg));
  kern<<<grid, K::NT, smem, st>>>(P);
  if (VJP) K::reduce_block_gc<<<K::S / 256, 256, 0, st>>>(P.gc_part, grid, a.grad_c);
  counted_launch(2 + (ring ? 1 : 0) + (VJP ? 1 : 0));
  cudaError_t le = cudaGetLastError();
  cudaError_t fe = cudaFreeAsync(mem, st);
  if (le != cudaSuccess || fe != cudaSuccess) return BCJR_ERR_CUDA;
  return BCJR_OK;
}

bool use_l16(const Shape& sh) { return !generic_only() && sh.L == 16 && sh.D == 2 && sh.V == 1; }
bool use_l16v2(const Shape& sh) { return !generic_only() && sh.L == 16 && sh.D == 4 && sh.V == 2; }

// L = 16, k = 2, V = 2: the kernels of bcjr_l16v2.cuh.
template <int MODE>
int run_l16v2(const Shape& sh, const SweepArgs& a, cudaStream_t st) {
  namespace K = bcjr::l16v2;
  constexpr bool VJP = MODE == bcjr::MODE_VJP;
  void (*kern)(K::Params) = K::vjp_kernel;
  if (!VJP) kern = a.out_argmax ? K::soft_kernel<true> : K::soft_kernel<false>;
  // group vectors (2, or 4 with A / Bc), per-warp partials, argmax indices or
  // TMEM slot, per-step weights (and gradients)
  const size_t smem = sizeof(float) * ((size_t)(VJP ? 4 : 2) * K::J + 2 * 32 * 8 + (VJP ? 4 : 64 + 4) +
                                       (size_t)(VJP ? 4 : 2) * sh.n);
  if (smem > kMaxDynSmem) return BCJR_ERR_UNSUPPORTED;
  int grid = 0;
  int rc = grid_for(kern, K::NT, smem, sh.n_seq, &grid);
  if (rc != BCJR_OK) return rc;
  cap_grid_by_memory(&grid, sizeof(float) * (size_t)sh.n * K::J * (VJP ? 2 : 1) + sizeof(double) * sh.n +
                                (VJP ? sizeof(float4) * K::G * 4 * K::NT + sizeof(double) * 2 * K::S : 0));
  K::Params P{};
  auto layout = [&](Arena& ar) {
    P.cf = ar.take<float4>(K::CB4);
    P.cb = ar.take<float4>(K::CB4);
    P.cf1 = ar.take<float2>(K::CB4);
    P.cb1 = ar.take<float2>(K::CB4);
    P.hist_l = ar.take<float>((size_t)grid * sh.n * K::J);
    P.hist_a = VJP ? ar.take<float>((size_t)grid * sh.n * K::J) : nullptr;
    P.hist_c = ar.take<double>((size_t)grid * sh.n);
    P.gc1 = VJP ? ar.take<float4>((size_t)grid * K::G * 4 * K::NT) : nullptr;
    P.gc_part = VJP ? ar.take<double>((size_t)grid * 2 * K::S) : nullptr;
  };
  Arena sizing;
  layout(sizing);
  void* mem = nullptr;
  if (int arc = scratch_alloc(&mem, sizing.off, st)) return arc;
  Arena ar;
  ar.base = static_cast<char*>(mem);
  layout(ar);
  P.w = a.w; P.gsoft = a.gsoft; P.gZ = a.gZ;
  P.out_soft = a.out_soft; P.out_logZ = a.out_logZ; P.out_argmax = a.out_argmax; P.grad_w = a.grad_w;
  P.n_seq = sh.n_seq; P.len = sh.len; P.n = sh.n;
  P.sk = (float)std::sqrt(1.4426950408889634 / (double)a.T);
  P.two_over_T = (float)(2.0 / (double)a.T);
  K::make_codebooks<<<K::CB4 / 256, 256, 0, st>>>(a.c, P.sk, const_cast<float4*>(P.cf), const_cast<float4*>(P.cb),
                                                  const_cast<float2*>(P.cf1), const_cast<float2*>(P.cb1));
  kern<<<grid, K::NT, smem, st>>>(P);
  if (VJP) K::reduce_gc<<<2 * K::S / 256, 256, 0, st>>>(P.gc_part, grid, a.grad_c);
  counted_launch(VJP ? 3 : 2);
  cudaError_t le = cudaGetLastError();
  cudaError_t fe = cudaFreeAsync(mem, st);
  if (le != cudaSuccess || fe != cudaSuccess) return BCJR_ERR_CUDA;
  return BCJR_OK;
}

template <int MODE>
int run_sweep(const Shape& sh, const SweepArgs& a, cudaStream_t st) {
  constexpr bool VJP = MODE == bcjr::MODE_VJP;
  if (use_l16(sh)) return run_l16<MODE>(sh, a, st);
  if (use_l16v2(sh)) return run_l16v2<MODE>(sh, a, st);
  SweepKernel kern = pick_sweep<MODE>(sh.V, sh.D);
  if (!kern) return BCJR_ERR_UNSUPPORTED;
  const int threads = threads_for(sh.J, sh.B);
  const int NPT = sh.V + 1 + (VJP ? 3 : 0);   // per-warp partials per step
  size_t fixed = sizeof(float) * ((size_t)sh.n * sh.V * (VJP ? 2 : 1) + 64 + 64 * NPT + 64 + 64);
  size_t state_bytes = sizeof(float) * (size_t)sh.J * (VJP ? 4 : 2);
  const bool in_smem = fixed + state_bytes <= kMaxDynSmem;
  const size_t smem = fixed + (in_smem ? state_bytes : 0);
  if (smem > kMaxDynSmem) return BCJR_ERR_UNSUPPORTED;
  int grid = 0;
  int rc = grid_for(kern, threads, smem, sh.n_seq, &grid);
  if (rc != BCJR_OK) return rc;

  const size_t SV = (size_t)sh.S * sh.V;
  cap_grid_by_memory(&grid, sizeof(float) * (size_t)sh.n * sh.J * (VJP ? 2 : 1) + sizeof(double) * sh.n +
                                (in_smem ? 0 : sizeof(float) * 4 * (size_t)sh.J) +
                                (VJP ? (sizeof(float) + sizeof(double)) * SV : 0));
  auto layout = [&](Arena& ar, SweepParams& P) {
    P.cs = ar.take<float>(SV);
    P.hist_l = ar.take<float>((size_t)grid * sh.n * sh.J);
    P.hist_a = VJP ? ar.take<float>((size_t)grid * sh.n * sh.J) : nullptr;
    P.hist_c = ar.take<double>((size_t)grid * sh.n);
    P.state_g = in_smem ? nullptr : ar.take<float>((size_t)grid * 4 * sh.J);
    P.gc_seq = VJP ? ar.take<float>((size_t)grid * SV) : nullptr;
    P.gc_part = VJP ? ar.take<double>((size_t)grid * SV) : nullptr;
  };
  SweepParams P{};
  Arena sizing;
  layout(sizing, P);
  void* mem = nullptr;
  if (int arc = scratch_alloc(&mem, sizing.off, st)) return arc;
  Arena ar;
  ar.base = static_cast<char*>(mem);
  layout(ar, P);
  P.w = a.w; P.gsoft = a.gsoft; P.gZ = a.gZ;
  P.out_soft = a.out_soft; P.out_logZ = a.out_logZ; P.out_argmax = a.out_argmax; P.grad_w = a.grad_w;
  P.n_seq = sh.n_seq; P.len = sh.len; P.L = sh.L; P.n = sh.n; P.J = sh.J; P.S = sh.S;
  P.sk = (float)std::sqrt(1.4426950408889634 / (double)a.T);
  P.two_over_T = (float)(2.0 / (double)a.T);
  P.state_in_smem = in_smem ? 1 : 0;

  const int sv = (int)SV;
  bcjr::scale_codebook_kernel<<<(sv + 255) / 256, 256, 0, st>>>(a.c, sv, P.sk, const_cast<float*>(P.cs));
  kern<<<grid, threads, smem, st>>>(P);
  if (VJP) bcjr::reduce_gc_kernel<<<(sv + 255) / 256, 256, 0, st>>>(P.gc_part, grid, sv, a.grad_c);
  counted_launch(VJP ? 3 : 2);
  cudaError_t le = cudaGetLastError();
  cudaError_t fe = cudaFreeAsync(mem, st);
  if (le != cudaSuccess || fe != cudaSuccess) return BCJR_ERR_CUDA;
  return BCJR_OK;
}

// ----------------------------------------------------------------- Viterbi
using ViterbiKernel = void (*)(ViterbiParams);

ViterbiKernel pick_viterbi(int V, int D) {
#define BCJR_CASE(VV, DD) \
  if (V == VV && D == DD) return bcjr::viterbi_kernel<VV, DD>;
  BCJR_CASE(1, 1) BCJR_CASE(1, 2) BCJR_CASE(1, 3) BCJR_CASE(1, 4) BCJR_CASE(1, 5) BCJR_CASE(1, 6)
  BCJR_CASE(2, 2) BCJR_CASE(2, 4) BCJR_CASE(2, 6)
  BCJR_CASE(4, 4)
#undef BCJR_CASE
  return nullptr;
}

// L = 16, D = 2, V = 1: the block-layout Viterbi of bcjr_l16.cuh.
int run_viterbi_l16(const Shape& sh, const float* w, const float* c, int32_t* out_states, float* out_cost,
                    cudaStream_t st) {
  namespace K = bcjr::l16;
  const size_t smem = sizeof(float) * ((size_t)2 * K::J + 32 + 32 + 64 + 4 + (size_t)sh.n);
  if (smem > kMaxDynSmem) return BCJR_ERR_UNSUPPORTED;
  int grid = 0;
  int rc = grid_for(K::viterbi_kernel, K::NT, smem, sh.n_seq, &grid);
  if (rc != BCJR_OK) return rc;
  // backpointer batch per CTA: up to 16 sequences, within about 2.5 GB in total
  const size_t per_seq = (size_t)sh.n * K::NMID;
  int64_t tb = (int64_t)(2500000000ull / ((size_t)grid * per_seq));
  if (tb > 16) tb = 16;
  if (tb < 1) tb = 1;
  K::VParams P{};
  auto layout = [&](Arena& ar) {
    P.cb_raw = ar.take<float>(K::S);
    P.bp = ar.take<uint8_t>((size_t)grid * tb * per_seq);
  };
  Arena sizing;
  layout(sizing);
  void* mem = nullptr;
  if (int arc = scratch_alloc(&mem, sizing.off, st)) return arc;
  Arena ar;
  ar.base = static_cast<char*>(mem);
  layout(ar);
  P.w = w; P.out_states = out_states; P.out_cost = out_cost;
  P.n_seq = sh.n_seq; P.len = sh.len; P.n = sh.n; P.tb = (int)tb;
  K::make_block_codebook<<<K::S / 256, 256, 0, st>>>(c, 1.0f, const_cast<float*>(P.cb_raw));
  K::viterbi_kernel<<<grid, K::NT, smem, st>>>(P);
  counted_launch(2);
  cudaError_t le = cudaGetLastError();
  cudaError_t fe = cudaFreeAsync(mem, st);
  if (le != cudaSuccess || fe != cudaSuccess) return BCJR_ERR_CUDA;
  return BCJR_OK;
}

// L = 16, D = 4, V = 2: the Viterbi of bcjr_l16v2.cuh.
int run_viterbi_l16v2(const Shape& sh, const float* w, const float* c, int32_t* out_states, float* out_cost,
                      cudaStream_t st) {
  namespace K = bcjr::l16v2;
  const size_t smem = sizeof(float) * ((size_t)2 * K::J + 32 + 32 + 64 + 4 + 2 * (size_t)sh.n);
  if (smem > kMaxDynSmem) return BCJR_ERR_UNSUPPORTED;
  int grid = 0;
  int rc = grid_for(K::viterbi_kernel, K::NT, smem, sh.n_seq, &grid);
  if (rc != BCJR_OK) return rc;
  // backpointer batch per CTA: up to 16 sequences, within about 2.5 GB in total
  const size_t per_seq = (size_t)sh.n * K::NT;   // 32-bit words
  int64_t tb = (int64_t)(2500000000ull / (sizeof(uint32_t) * (size_t)grid * per_seq));
  if (tb > 16) tb = 16;
  if (tb < 1) tb = 1;
  K::VParams P{};
  float4* cf = nullptr;
  float4* cbk = nullptr;
  float2* cf1 = nullptr;
  float2* cb1 = nullptr;
  auto layout = [&](Arena& ar) {
    cf = ar.take<float4>(K::CB4);
    cbk = ar.take<float4>(K::CB4);
    cf1 = ar.take<float2>(K::CB4);
    cb1 = ar.take<float2>(K::CB4);
    P.bp = ar.take<uint32_t>((size_t)grid * tb * per_seq);
  };
  Arena sizing;
  layout(sizing);
  void* mem = nullptr;
  if (int arc = scratch_alloc(&mem, sizing.off, st)) return arc;
  Arena ar;
  ar.base = static_cast<char*>(mem);
  layout(ar);
  P.w = w; P.cf = cf; P.cf1 = cf1; P.out_states = out_states; P.out_cost = out_cost;
  P.n_seq = sh.n_seq; P.len = sh.len; P.n = sh.n; P.tb = (int)tb;
  K::make_codebooks<<<K::CB4 / 256, 256, 0, st>>>(c, 1.0f, cf, cbk, cf1, cb1);   // raw codewords
  K::viterbi_kernel<<<grid, K::NT, smem, st>>>(P);
  counted_launch(2);
  cudaError_t le = cudaGetLastError();
  cudaError_t fe = cudaFreeAsync(mem, st);
  if (le != cudaSuccess || fe != cudaSuccess) return BCJR_ERR_CUDA;
  return BCJR_OK;
}

int run_viterbi(const Shape& sh, const float* w, const float* c, int32_t* out_states, float* out_cost,
                cudaStream_t st) {
  if (sh.L == 16 && sh.D == 2 && sh.V == 1 && !generic_only()) return run_viterbi_l16(sh, w, c, out_states, out_cost, st);
  if (sh.L == 16 && sh.D == 4 && sh.V == 2 && !generic_only())
    return run_viterbi_l16v2(sh, w, c, out_states, out_cost, st);
  ViterbiKernel kern = pick_viterbi(sh.V, sh.D);
  if (!kern) return BCJR_ERR_UNSUPPORTED;
  const int threads = threads_for(sh.J, sh.B);
  size_t fixed = sizeof(float) * ((size_t)sh.n * sh.V + 64);
  size_t state_bytes = sizeof(float) * (size_t)sh.J * 2;
  const bool in_smem = fixed + state_bytes <= kMaxDynSmem;
  const size_t smem = fixed + (in_smem ? state_bytes : 0);
  int grid = 0;
  int rc = grid_for(kern, threads, smem, sh.n_seq, &grid);
  if (rc != BCJR_OK) return rc;
  cap_grid_by_memory(&grid, (size_t)sh.n * sh.J + (in_smem ? 0 : sizeof(float) * 2 * (size_t)sh.J));
  ViterbiParams P{};
  auto layout = [&](Arena& ar) {
    P.bp = ar.take<uint8_t>((size_t)grid * sh.n * sh.J);
    P.state_g = in_smem ? nullptr : ar.take<float>((size_t)grid * 2 * sh.J);
  };
  Arena sizing;
  layout(sizing);
  void* mem = nullptr;
  if (int arc = scratch_alloc(&mem, sizing.off, st)) return arc;
  Arena ar;
  ar.base = static_cast<char*>(mem);
  layout(ar);
  P.w = w; P.c = c; P.out_states = out_states; P.out_cost = out_cost;
  P.n_seq = sh.n_seq; P.len = sh.len; P.L = sh.L; P.n = sh.n; P.J = sh.J; P.S = sh.S;
  P.state_in_smem = in_smem ? 1 : 0;
  kern<<<grid, threads, smem, st>>>(P);
  counted_launch();
  cudaError_t le = cudaGetLastError();
  cudaError_t fe = cudaFreeAsync(mem, st);
  if (le != cudaSuccess || fe != cudaSuccess) return BCJR_ERR_CUDA;
  return BCJR_OK;
}

static_assert(bcjr::kErrTimeout == BCJR_ERR_TIMEOUT && bcjr::kErrNumeric == BCJR_ERR_NUMERIC,
              "device and host status codes agree");

}  // namespace

extern "C" {

int bcjr_soft_codeword(const float* w, int64_t n_seq, int64_t len, int L, int k, int V, const float* codebook,
                       float T, float* out_soft, float* out_logZ, void* stream) {
  Shape sh;
  int rc = check_shape(n_seq, len, L, k, V, &sh);
  if (rc) return rc;
  if ((rc = check_T(T))) return rc;
  if ((rc = check_dev_ptr(codebook, false))) return rc;
  if (n_seq == 0) return BCJR_OK;
  if ((rc = check_dev_ptr(w, false)) || (rc = check_dev_ptr(out_soft, false)) ||
      (rc = check_dev_ptr(out_logZ, true)))
    return rc;
  SweepArgs a{w, codebook, T, nullptr, nullptr, out_soft, out_logZ, nullptr, nullptr, nullptr};
  return run_sweep<bcjr::MODE_SOFT>(sh, a, static_cast<cudaStream_t>(stream));
}

int bcjr_posterior_argmax(const float* w, int64_t n_seq, int64_t len, int L, int k, int V, const float* codebook,
                          float T, int32_t* out_argmax, void* stream) {
  Shape sh;
  int rc = check_shape(n_seq, len, L, k, V, &sh);
  if (rc) return rc;
  if ((rc = check_T(T))) return rc;
  if ((rc = check_dev_ptr(codebook, false))) return rc;
  if (n_seq == 0) return BCJR_OK;
  if ((rc = check_dev_ptr(w, false)) || (rc = check_dev_ptr(out_argmax, false))) return rc;
  SweepArgs a{w, codebook, T, nullptr, nullptr, nullptr, nullptr, out_argmax, nullptr, nullptr};
  return run_sweep<bcjr::MODE_SOFT>(sh, a, static_cast<cudaStream_t>(stream));
}

int bcjr_vjp(const float* w, int64_t n_seq, int64_t len, int L, int k, int V, const float* codebook, float T,
             const float* grad_soft, const float* grad_logZ, float* grad_w, float* grad_codebook, void* stream) {
  Shape sh;
  int rc = check_shape(n_seq, len, L, k, V, &sh);
  if (rc) return rc;
  if ((rc = check_T(T))) return rc;
  if ((rc = check_dev_ptr(codebook, false)) || (rc = check_dev_ptr(grad_codebook, false))) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (n_seq == 0) {
    return cudaMemsetAsync(grad_codebook, 0, sizeof(float) * (size_t)sh.S * sh.V, st) == cudaSuccess
               ? BCJR_OK
               : BCJR_ERR_CUDA;
  }
  if ((rc = check_dev_ptr(w, false)) || (rc = check_dev_ptr(grad_soft, false)) ||
      (rc = check_dev_ptr(grad_logZ, true)) || (rc = check_dev_ptr(grad_w, false)))
    return rc;
  SweepArgs a{w, codebook, T, grad_soft, grad_logZ, nullptr, nullptr, nullptr, grad_w, grad_codebook};
  return run_sweep<bcjr::MODE_VJP>(sh, a, st);
}

int viterbi_decode(const float* w, int64_t n_seq, int64_t len, int L, int k, int V, const float* codebook,
                   int32_t* out_states, float* out_cost, void* stream) {
  Shape sh;
  int rc = check_shape(n_seq, len, L, k, V, &sh);
  if (rc) return rc;
  if ((rc = check_dev_ptr(codebook, false))) return rc;
  if (n_seq == 0) return BCJR_OK;
  if ((rc = check_dev_ptr(w, false)) || (rc = check_dev_ptr(out_states, false)) ||
      (rc = check_dev_ptr(out_cost, true)))
    return rc;
  return run_viterbi(sh, w, codebook, out_states, out_cost, static_cast<cudaStream_t>(stream));
}

int bcjr_qat_step(float* w, const float* w_target, int64_t n_seq, int64_t len, int L, int k, int V, float* codebook,
                  float T, float lr_w, float lr_c, float* out_soft, float* out_loss, float* grad_w,
                  float* grad_codebook, void* stream) {
  Shape sh;
  int rc = check_shape(n_seq, len, L, k, V, &sh);
  if (rc) return rc;
  if ((rc = check_T(T))) return rc;
  if (!std::isfinite(lr_w) || !std::isfinite(lr_c)) return BCJR_ERR_INVALID_ARG;
  if ((rc = check_dev_ptr(codebook, false)) || (rc = check_dev_ptr(grad_codebook, false))) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (n_seq == 0) {
    return cudaMemsetAsync(grad_codebook, 0, sizeof(float) * (size_t)sh.S * sh.V, st) == cudaSuccess
               ? BCJR_OK
               : BCJR_ERR_CUDA;
  }
  if ((rc = check_dev_ptr(w, false)) || (rc = check_dev_ptr(w_target, false)) ||
      (rc = check_dev_ptr(out_soft, false)) || (rc = check_dev_ptr(out_loss, true)) ||
      (rc = check_dev_ptr(grad_w, false)))
    return rc;
  SweepArgs a{w, codebook, T, nullptr, nullptr, out_soft, nullptr, nullptr, nullptr, nullptr};
  if ((rc = run_sweep<bcjr::MODE_SOFT>(sh, a, st))) return rc;
  const int64_t nw = n_seq * len;
  void* g = nullptr;
  if ((rc = scratch_alloc(&g, sizeof(float) * (size_t)nw, st))) return rc;
  bcjr::recon_grad_kernel<<<(unsigned)std::min<int64_t>(n_seq, 148 * 64), 256, 0, st>>>(
      out_soft, w_target, n_seq, len, static_cast<float*>(g), out_loss);
  counted_launch();
  SweepArgs b{w, codebook, T, static_cast<float*>(g), nullptr, nullptr, nullptr, nullptr, grad_w, grad_codebook};
  rc = run_sweep<bcjr::MODE_VJP>(sh, b, st);
  if (rc == BCJR_OK) {
    const int64_t sv = (int64_t)sh.S * sh.V;
    bcjr::sgd_kernel<<<(unsigned)std::min<int64_t>((nw + 255) / 256, 148 * 16), 256, 0, st>>>(w, grad_w, lr_w, nw);
    if (lr_c != 0.f)
      bcjr::sgd_kernel<<<(unsigned)((sv + 255) / 256), 256, 0, st>>>(codebook, grad_codebook, lr_c, sv);
    counted_launch(lr_c != 0.f ? 2 : 1);
    if (cudaGetLastError() != cudaSuccess) rc = BCJR_ERR_CUDA;
  }
  if (cudaFreeAsync(g, st) != cudaSuccess && rc == BCJR_OK) rc = BCJR_ERR_CUDA;
  return rc;
}

uint64_t bcjr_launch_count(void) { return g_launch_count.load(std::memory_order_relaxed); }

int bcjr_get_device_error(void* stream) {
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(st) != cudaSuccess) {
    cudaGetLastError();
    return BCJR_ERR_CUDA;
  }
  int flag = 0, zero = 0;
  if (cudaMemcpyFromSymbol(&flag, bcjr::g_device_error, sizeof(int)) != cudaSuccess) return BCJR_ERR_CUDA;
  if (flag != 0 && cudaMemcpyToSymbol(bcjr::g_device_error, &zero, sizeof(int)) != cudaSuccess) return BCJR_ERR_CUDA;
  return flag;
}

const char* bcjr_strerror(int status) {
  switch (status) {
    case BCJR_OK: return "ok";
    case BCJR_ERR_INVALID_ARG: return "invalid argument";
    case BCJR_ERR_UNSUPPORTED: return "unsupported configuration";
    case BCJR_ERR_CUDA: return "CUDA error";
    case BCJR_ERR_TIMEOUT: return "device-side wait timed out";
    case BCJR_ERR_NUMERIC: return "numerical check failed on the device (posterior mass off)";
    default: return "unknown status";
  }
}

const char* bcjr_version(void) { return "0.1.0"; }

}  // extern "C"

// ----------------------------------------------------------------- no-allocation variant
// bcjr_soft_codeword_noalloc: the soft-codeword sweep with its scratch taken from
// a fixed, file-scope device array instead of cudaMallocAsync.  For callers that
// may not allocate device memory themselves (see include/bcjr.h).
namespace {

static __device__ __align__(256) unsigned char g_noalloc_scratch[BCJR_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_noalloc_mu;
void* g_noalloc_ptr[kMaxDevices] = {};

// Device address of g_noalloc_scratch on the current device, looked up once per
// device (the symbol name is only a host-side handle; it is not a device address).
int noalloc_scratch(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    cudaGetLastError();
    return BCJR_ERR_CUDA;
  }
  std::lock_guard<std::mutex> lk(g_noalloc_mu);
  if (g_noalloc_ptr[dev] == nullptr) {
    void* p = nullptr;
    cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess || p == nullptr) {
      cudaGetLastError();
      return BCJR_ERR_CUDA;
    }
    g_noalloc_ptr[dev] = p;
  }
  *out = g_noalloc_ptr[dev];
  return BCJR_OK;
}

}  // namespace

extern "C" int bcjr_soft_codeword_noalloc(const float* w, int64_t n_seq, int64_t len, int L, int k, int V,
                                          const float* codebook, float T, float* out_soft, float* out_logZ,
                                          void* stream) {
  Shape sh;
  int rc = check_shape(n_seq, len, L, k, V, &sh);
  if (rc) return rc;
  if ((rc = check_T(T))) return rc;
  if ((rc = check_dev_ptr(codebook, false))) return rc;
  if (n_seq == 0) return BCJR_OK;
  if ((rc = check_dev_ptr(w, false)) || (rc = check_dev_ptr(out_soft, false)) ||
      (rc = check_dev_ptr(out_logZ, true)))
    return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  SweepKernel kern = pick_sweep<bcjr::MODE_SOFT>(sh.V, sh.D);
  if (!kern) return BCJR_ERR_UNSUPPORTED;
  const int threads = threads_for(sh.J, sh.B);
  const int NP = sh.V + 1;
  const size_t fixed = sizeof(float) * ((size_t)sh.n * sh.V + 64 + 64 * NP + 64 + 64);
  const size_t state_bytes = sizeof(float) * (size_t)sh.J * 2;
  const bool in_smem = fixed + state_bytes <= kMaxDynSmem;
  const size_t smem = fixed + (in_smem ? state_bytes : 0);
  if (smem > kMaxDynSmem) return BCJR_ERR_UNSUPPORTED;
  int grid = 0;
  if ((rc = grid_for(kern, threads, smem, sh.n_seq, &grid))) return rc;

  const size_t SV = (size_t)sh.S * sh.V;
  SweepParams P{};
  auto layout = [&](Arena& ar, int g) {
    P.cs = ar.take<float>(SV);
    P.hist_l = ar.take<float>((size_t)g * sh.n * sh.J);
    P.hist_a = nullptr;
    P.hist_c = ar.take<double>((size_t)g * sh.n);
    P.state_g = in_smem ? nullptr : ar.take<float>((size_t)g * 4 * sh.J);
    P.gc_seq = nullptr;
    P.gc_part = nullptr;
  };
  // As many CTAs as the fixed array holds histories for: the codebook and each
  // of the three per-CTA arrays take at most 255 bytes of alignment padding.
  {
    const size_t cb = (sizeof(float) * SV + 255) & ~size_t(255);
    const size_t per_cta = sizeof(float) * (size_t)sh.n * sh.J + sizeof(double) * sh.n +
                           (in_smem ? 0 : sizeof(float) * 4 * (size_t)sh.J);
    const size_t cap = BCJR_NOALLOC_SCRATCH_BYTES;
    if (cb + 3 * 256 + per_cta > cap) return BCJR_ERR_UNSUPPORTED;   // one sequence does not fit
    const size_t fit = (cap - cb - 3 * 256) / per_cta;
    if ((size_t)grid > fit) grid = (int)fit;
    Arena sizing;
    layout(sizing, grid);
    while (sizing.off > cap && grid > 1) {   // the padding bound above makes this a no-op
      --grid;
      sizing = Arena{};
      layout(sizing, grid);
    }
    if (sizing.off > cap) return BCJR_ERR_UNSUPPORTED;
  }
  void* base = nullptr;
  if ((rc = noalloc_scratch(&base))) return rc;
  Arena ar;
  ar.base = static_cast<char*>(base);
  layout(ar, grid);
  P.w = w; P.gsoft = nullptr; P.gZ = nullptr;
  P.out_soft = out_soft; P.out_logZ = out_logZ; P.out_argmax = nullptr; P.grad_w = nullptr;
  P.n_seq = sh.n_seq; P.len = sh.len; P.L = sh.L; P.n = sh.n; P.J = sh.J; P.S = sh.S;
  P.sk = (float)std::sqrt(1.4426950408889634 / (double)T);
  P.two_over_T = (float)(2.0 / (double)T);
  P.state_in_smem = in_smem ? 1 : 0;
  const int sv = (int)SV;
  bcjr::scale_codebook_kernel<<<(sv + 255) / 256, 256, 0, st>>>(codebook, sv, P.sk, const_cast<float*>(P.cs));
  kern<<<grid, threads, smem, st>>>(P);
  counted_launch(2);
  return cudaGetLastError() == cudaSuccess ? BCJR_OK : BCJR_ERR_CUDA;
}

