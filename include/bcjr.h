/*
 * bcjr.h -- C ABI of the B200 (sm_100a) BCJR forward-backward library.
 *
 * The operations follow "BCJR-QAT: A Differentiable Relaxation of
 * Trellis-Coded Weight Quantization":
 *   - Abstract: the hard Viterbi argmax of trellis-coded quantisation is
 *     replaced by the BCJR forward-backward sum-product at temperature T; the
 *     result is a soft codeword equal to the Boltzmann expectation over trellis
 *     paths, exactly differentiable, and equal to the hard code as T -> 0; the
 *     computation is the transfer-matrix computation of a 1D Ising-like chain.
 *   - Technical Summary, "Core Mechanism": the soft codeword
 *       w_hat_t(T) = sum_s c(s) p_T(s_t = s | w),
 *     differentiable in the weights and in the trellis parameters (codebook).
 *   - Technical Summary, "Key Technical Innovations": exact gradients through
 *     the forward-backward recursion; a fused kernel of gather, log-sum-exp and
 *     addition.
 *
 * Trellis and energy (the pages leave them open; these are the readings used):
 *   states s in [0, 2^L); D = k*V bits enter per step at the bottom:
 *   succ(p, b) = ((p << D) & (2^L - 1)) | b, b in [0, 2^D);
 *   step t (0 <= t < n, n = len / V) reads weights w[t*V .. t*V+V-1];
 *   E_t(s) = sum_v (w[t*V+v] - c[s][v])^2; a path has weight exp(-sum_t E_t/T);
 *   free start (every state has weight 1 at t = 0) and free end.
 *
 * Conventions for every entry point:
 *   - All array arguments are DEVICE pointers (cudaMalloc'd or managed memory)
 *     to contiguous row-major fp32 / int32 data, 4-byte aligned.  The caller
 *     owns every buffer; the library never frees or retains them.
 *   - `len` counts weights per sequence and must be a positive multiple of V.
 *   - `codebook` is [2^L][V] fp32.
 *   - `stream` is a cudaStream_t passed as void* (NULL = the legacy default
 *     stream).  Calls are asynchronous: they validate their arguments, enqueue
 *     the work on `stream` and return.  Argument errors are returned at once and
 *     enqueue nothing.  The library allocates its own scratch space, stream-
 *     ordered on `stream`, from a library-private memory pool of the current
 *     device and frees it on `stream` before returning; freed scratch stays
 *     mapped in that pool for reuse by later calls (up to the largest call's
 *     size, several GB for L=16, until the process exits).  No data is kept
 *     between calls.
 *   - Supported: 1 <= D = k*V <= L <= 16, D <= 6, V in {1, 2, 4},
 *     len <= 8192; T finite and > 0.  n_seq == 0 is a no-op returning BCJR_OK.
 *   - Errors: null or non-device pointers, len not a positive multiple of V,
 *     k < 1, V < 1, D > L, T not finite or <= 0  -> BCJR_ERR_INVALID_ARG;
 *     L > 16, D > 6, V not in {1,2,4}, len > 8192 -> BCJR_ERR_UNSUPPORTED;
 *     a failed CUDA call (allocation, launch)   -> BCJR_ERR_CUDA.
 *   - NaN or infinite weights make that sequence's outputs NaN; other
 *     sequences are unaffected.  The soft-codeword and VJP kernels also check
 *     that the posterior of every step sums to 1 within 1e-2 and, if not (NaN
 *     or infinite inputs, or a numerical breakdown), record BCJR_ERR_NUMERIC
 *     for bcjr_get_device_error.
 */
#ifndef BCJR_H_
#define BCJR_H_

#include <stdint.h>

#if defined(__GNUC__)
#define BCJR_API __attribute__((visibility("default")))
#else
#define BCJR_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  BCJR_OK = 0,
  BCJR_ERR_INVALID_ARG = 1,
  BCJR_ERR_UNSUPPORTED = 2,
  BCJR_ERR_CUDA = 3,
  BCJR_ERR_TIMEOUT = 4,  /* recorded on the device: a bounded wait ran out */
  BCJR_ERR_NUMERIC = 5   /* recorded on the device: a step's posterior mass was off */
} bcjr_status;

/*
 * Soft codeword and log-partition function (Abstract; "Core Mechanism").
 *   w         [n_seq][len]  weights (input)
 *   codebook  [2^L][V]      codewords c(s) (input)
 *   T                       temperature
 *   out_soft  [n_seq][len]  w_hat: out_soft[q][t*V+v] = sum_s c(s)[v] p_t(s)
 *   out_logZ  [n_seq]       natural log of Z = sum over paths of exp(-E/T);
 *                           may be NULL
 */
BCJR_API int bcjr_soft_codeword(const float* w, int64_t n_seq, int64_t len, int L, int k, int V,
                       const float* codebook, float T, float* out_soft, float* out_logZ, void* stream);

/*
 * Vector-Jacobian product of  l = sum_{q,t,v} grad_soft[q][t*V+v] * w_hat[q][t*V+v]
 *                               + sum_q grad_logZ[q] * logZ[q]
 * with respect to the weights and the codebook ("Core Mechanism": exactly
 * differentiable with respect to the weight pre-image and the trellis
 * parameters; "Key Technical Innovations": exact gradients).
 *   grad_soft     [n_seq][len]  upstream gradient on out_soft (input)
 *   grad_logZ     [n_seq]       upstream gradient on out_logZ, or NULL (= 0)
 *   grad_w        [n_seq][len]  dl/dw (output, overwritten)
 *   grad_codebook [2^L][V]      dl/dc summed over all sequences and steps
 *                               (output, overwritten, not accumulated)
 */
BCJR_API int bcjr_vjp(const float* w, int64_t n_seq, int64_t len, int L, int k, int V, const float* codebook,
             float T, const float* grad_soft, const float* grad_logZ, float* grad_w,
             float* grad_codebook, void* stream);

/*
 * Viterbi decode, the T -> 0 limit of the soft codeword (Abstract: "recovering
 * the hard QTIP code as T -> 0").  Min-sum over paths in fp32 with this exact
 * operation order (no fused multiply-add):
 *   q_t(s) = sum over v, in order, of fl(fl(w - c(s)[v])^2);
 *   delta_0(s) = q_0(s);  delta_t(s) = fl(min_{p -> s} delta_{t-1}(p) + q_t(s)).
 * Ties go to the lowest predecessor and, for the final state, the lowest index.
 *   out_states [n_seq][n] int32   decoded state s_t of every step
 *   out_cost   [n_seq] fp32       delta_{n-1}(s_{n-1}), or NULL
 * T plays no part.
 */
BCJR_API int viterbi_decode(const float* w, int64_t n_seq, int64_t len, int L, int k, int V, const float* codebook,
                   int32_t* out_states, float* out_cost, void* stream);

/*
 * Per-step argmax of the posterior p_T(s_t = s | w) ("Core Mechanism"), ties to
 * the lowest state (compared in fp32).
 *   out_argmax [n_seq][n] int32
 */
BCJR_API int bcjr_posterior_argmax(const float* w, int64_t n_seq, int64_t len, int L, int k, int V,
                          const float* codebook, float T, int32_t* out_argmax, void* stream);

/*
 * bcjr_soft_codeword_noalloc -- bcjr_soft_codeword without any allocation.
 * The paper has no counterpart to this entry point; it is an interface
 * variant for callers that must not allocate device memory: for example a
 * plugin inside an application or framework that owns every device
 * allocation, a service whose device-memory budget is fixed at start-up, or a
 * latency-critical path where an allocation could block or fail under memory
 * pressure.
 *
 * Arguments, layouts and errors are those of bcjr_soft_codeword, and so are
 * the results up to rounding: this entry point always runs the general sweep
 * kernel, also where bcjr_soft_codeword runs a specialised one (L = 16 with
 * k*V = 2 or 4), so the two agree within the soft-codeword and logZ
 * tolerances (1e-5 of max|c| and of max(|logZ|, (L + D(n-1)) ln 2)), not bit
 * for bit.
 * The call makes no cudaMalloc, cudaMallocAsync or cudaFree call and uses no
 * allocating library routine.  Its scratch space is one fixed array of
 * BCJR_NOALLOC_SCRATCH_BYTES (64 MiB) in this library's device memory; every
 * GPU that loads the library reserves it until the process exits.
 *
 * Limit: the array must hold the scaled codebook (2^L * V floats) plus the
 * history of one sequence ((len/V) * 2^(L-D) floats and (len/V) doubles, plus
 * 4 * 2^(L-D) floats when the per-sequence state does not fit in shared
 * memory).  Larger problems return BCJR_ERR_UNSUPPORTED and enqueue nothing.
 * When the array holds fewer histories than the GPU can run at once, fewer
 * sequences run concurrently: slower, same results.
 *
 * Set-up: the first call on each device looks up the array's device address
 * (cudaGetSymbolAddress, with that device current) and keeps it for the rest
 * of the process; make that first call before any stream capture on the
 * device.  A cudaDeviceReset (or any other way of unloading the library's
 * module from the device) makes the kept address stale: do not call this entry
 * point on a device after resetting it.
 *
 * Sharing: all calls on a device use the same array, which keeps whatever the
 * last call left in it (nothing in it needs to start at zero).  Calls whose
 * GPU work overlaps -- issued on different streams, or from several host
 * threads without ordering -- race on the array and corrupt each other's
 * results; order them, e.g. on one stream.
 */
#define BCJR_NOALLOC_SCRATCH_BYTES (64u << 20)
BCJR_API int bcjr_soft_codeword_noalloc(const float* w, int64_t n_seq, int64_t len, int L, int k, int V,
                                        const float* codebook, float T, float* out_soft, float* out_logZ,
                                        void* stream);

/*
 * One step of quantisation-aware training by self-reconstruction (BCJR-QAT,
 * Technical Summary "Core Mechanism": the soft codeword of the latent weights
 * stands in for the quantised weights, and T is annealed from T0 towards a
 * near-zero T_end over the steps, one call per step with its own T).  With
 * w_hat the soft codeword of w at temperature T,
 *   loss[q] = sum_{t,v} (w_hat[q][t*V+v] - w_target[q][t*V+v])^2,
 * the call computes w_hat and the loss, the VJP of sum_q loss[q] (upstream
 * gradient 2 (w_hat - w_target), no gradient on logZ), and then updates in place
 *   w        <- w        - lr_w * dl/dw
 *   codebook <- codebook - lr_c * dl/dc      (only when lr_c != 0)
 *   w             [n_seq][len]  latent weights (input; updated in place)
 *   w_target      [n_seq][len]  target weights (input)
 *   codebook      [2^L][V]      codewords (input; updated in place when lr_c != 0)
 *   out_soft      [n_seq][len]  w_hat before the update (output)
 *   out_loss      [n_seq]       loss per sequence before the update (output, may be NULL)
 *   grad_w        [n_seq][len]  dl/dw (output)
 *   grad_codebook [2^L][V]      dl/dc (output)
 * All device pointers; w, w_target, out_soft and grad_w must not overlap.
 * lr_w and lr_c must be finite (BCJR_ERR_INVALID_ARG otherwise).  Every step
 * runs in the library's kernels on `stream`; the upstream gradient lives in
 * library scratch.
 */
BCJR_API int bcjr_qat_step(float* w, const float* w_target, int64_t n_seq, int64_t len, int L, int k, int V,
                           float* codebook, float T, float lr_w, float lr_c, float* out_soft, float* out_loss,
                           float* grad_w, float* grad_codebook, void* stream);

/*
 * Synchronises `stream` and returns BCJR_OK, or BCJR_ERR_CUDA if the stream
 * holds a CUDA error, or the first device-side error recorded by a kernel of
 * this library since the last call (BCJR_ERR_NUMERIC: a step's posterior mass
 * left 1 +- 1e-2 or was not finite; BCJR_ERR_TIMEOUT: a wait of the L=16 V=1
 * VJP for a bulk copy into its shared-memory codeword ring did not end within
 * 1 s, after which that CTA computes on without the ring and its sequences'
 * outputs are not usable).  The flag is one per device and process, shared by
 * all streams; reading it clears it.
 */
BCJR_API int bcjr_get_device_error(void* stream);

/* Number of kernels this library has launched in this process, on all devices
 * and streams (launches issued, counted on the host; a call that fails before
 * launching adds nothing).  For accounting, e.g. the launches of a timed region. */
BCJR_API uint64_t bcjr_launch_count(void);

/* Static string for a status code. */
BCJR_API const char* bcjr_strerror(int status);

/* Library version, e.g. "0.1.0". */
BCJR_API const char* bcjr_version(void);

#ifdef __cplusplus
}
#endif

#endif /* BCJR_H_ */
