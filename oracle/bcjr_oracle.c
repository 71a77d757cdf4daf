/*
 * CPU oracle for the temperature-T BCJR forward-backward sum-product over a
 * bitshift trellis.  TEST INFRASTRUCTURE ONLY: it is called by the tests,
 * by __graft_entry__.smoke() and by bench.py's cpu_baseline / reference leg,
 * never by the library.  It shares no code with the CUDA path.
 *
 * What it computes follows "BCJR-QAT: A Differentiable Relaxation of
 * Trellis-Coded Weight Quantization":
 *   - Abstract: the Viterbi argmax is replaced by the BCJR forward-backward
 *     sum-product at temperature T; the soft codeword is the Boltzmann
 *     expectation over trellis paths; T -> 0 recovers the hard code.
 *   - Technical Summary, "Core Mechanism": w_hat_t(T) = sum_s c(s) p_T(s_t = s | w),
 *     exactly differentiable in the weights and the trellis parameters (codebook).
 *   - Technical Summary, "Key Technical Innovations": exact gradients through
 *     the forward-backward recursion.
 * Readings where the pages are silent (trellis rule, energy, boundaries):
 *   - state s in [0, 2^L); one step shifts in D = k*V bits at the bottom:
 *     succ(p, b) = ((p << D) & (2^L - 1)) | b, b in [0, 2^D);
 *   - step t consumes weights w[t*V .. t*V+V-1]; energy of state s at step t
 *     is E_t(s) = sum_v (w[t*V+v] - c[s][v])^2, path weight exp(-sum_t E_t/T);
 *   - free start (every state weight 1) and free end.
 *
 * Plain fp64 log-domain recursions, alpha stored in full, one sequence per
 * OpenMP thread.  The Viterbi decode uses the prescribed fp32 arithmetic and
 * must be compiled with -ffp-contract=off.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

typedef struct {
  int L, D, B, V;
  int64_t S, n;
  int32_t* pred; /* [S][B] predecessors of each state, ascending */
} trellis_t;

/* Build predecessor lists by enumerating the successor rule (the definition). */
static int trellis_init(trellis_t* tr, int L, int k, int V, int64_t len) {
  tr->L = L; tr->V = V; tr->D = k * V; tr->B = 1 << tr->D;
  tr->S = (int64_t)1 << L; tr->n = len / V;
  tr->pred = (int32_t*)malloc(sizeof(int32_t) * (size_t)(tr->S * tr->B));
  int32_t* fill = (int32_t*)calloc((size_t)tr->S, sizeof(int32_t));
  if (!tr->pred || !fill) { free(tr->pred); free(fill); return -1; }
  for (int64_t p = 0; p < tr->S; ++p)
    for (int b = 0; b < tr->B; ++b) {
      int64_t s = ((p << tr->D) & (tr->S - 1)) | b;
      if (fill[s] >= tr->B) { free(fill); return -2; }
      tr->pred[s * tr->B + fill[s]++] = (int32_t)p;
    }
  for (int64_t s = 0; s < tr->S; ++s)
    if (fill[s] != tr->B) { free(fill); return -3; }
  free(fill);
  return 0;
}

static int64_t succ(const trellis_t* tr, int64_t p, int b) { return ((p << tr->D) & (tr->S - 1)) | b; }

/* theta_t(s) = -E_t(s)/T for one sequence: [n][S] */
static void log_potentials(const trellis_t* tr, const float* w, const float* c, double T, double* th) {
  for (int64_t t = 0; t < tr->n; ++t)
    for (int64_t s = 0; s < tr->S; ++s) {
      double e = 0.0;
      for (int v = 0; v < tr->V; ++v) {
        double d = (double)w[t * tr->V + v] - (double)c[s * tr->V + v];
        e += d * d;
      }
      th[t * tr->S + s] = -e / T;
    }
}

static double hval(const float* gq, const float* c, int V, int64_t t, int64_t s) {
  double h = 0.0;
  for (int v = 0; v < V; ++v) h += (double)gq[t * V + v] * (double)c[s * V + v];
  return h;
}

static double lse_array(const double* x, int m) {
  double mx = -INFINITY;
  for (int i = 0; i < m; ++i) if (x[i] > mx) mx = x[i];
  if (mx == -INFINITY) return -INFINITY;
  double acc = 0.0;
  for (int i = 0; i < m; ++i) acc += exp(x[i] - mx);
  return mx + log(acc);
}

/* Forward: la[t][s] = log alpha_t(s); alpha_0 = psi_0 (free start),
 * alpha_t(s) = psi_t(s) * sum_{p -> s} alpha_{t-1}(p). */
static void forward(const trellis_t* tr, const double* th, double* la) {
  double buf[256];
  for (int64_t s = 0; s < tr->S; ++s) la[s] = th[s];
  for (int64_t t = 1; t < tr->n; ++t) {
    const double* prev = la + (t - 1) * tr->S;
    double* cur = la + t * tr->S;
    for (int64_t s = 0; s < tr->S; ++s) {
      for (int i = 0; i < tr->B; ++i) buf[i] = prev[tr->pred[s * tr->B + i]];
      cur[s] = th[t * tr->S + s] + lse_array(buf, tr->B);
    }
  }
}

/* One backward step: lb_prev(p) = log sum_{b} psi_{t}(succ(p,b)) beta_{t}(succ(p,b)). */
static void backward_step(const trellis_t* tr, const double* th_t, const double* lb_t, double* lb_prev) {
  double buf[256];
  for (int64_t p = 0; p < tr->S; ++p) {
    for (int b = 0; b < tr->B; ++b) {
      int64_t q = succ(tr, p, b);
      buf[b] = th_t[q] + lb_t[q];
    }
    lb_prev[p] = lse_array(buf, tr->B);
  }
}

typedef struct {
  double* th;   /* [n][S] */
  double* la;   /* [n][S] */
  double* lb;   /* [S] current beta */
  double* lb2;  /* [S] */
  double* A;    /* [n][S] conditional prefix expectation (VJP) */
  double* Bc;   /* [S] */
  double* Bc2;  /* [S] */
} work_t;

static int work_alloc(work_t* wk, const trellis_t* tr, int vjp) {
  size_t nS = (size_t)(tr->n * tr->S);
  memset(wk, 0, sizeof(*wk));
  wk->th = (double*)malloc(sizeof(double) * nS);
  wk->la = (double*)malloc(sizeof(double) * nS);
  wk->lb = (double*)malloc(sizeof(double) * (size_t)tr->S);
  wk->lb2 = (double*)malloc(sizeof(double) * (size_t)tr->S);
  if (vjp) {
    wk->A = (double*)malloc(sizeof(double) * nS);
    wk->Bc = (double*)malloc(sizeof(double) * (size_t)tr->S);
    wk->Bc2 = (double*)malloc(sizeof(double) * (size_t)tr->S);
  }
  if (!wk->th || !wk->la || !wk->lb || !wk->lb2) return -1;
  if (vjp && (!wk->A || !wk->Bc || !wk->Bc2)) return -1;
  return 0;
}

static void work_free(work_t* wk) {
  free(wk->th); free(wk->la); free(wk->lb); free(wk->lb2); free(wk->A); free(wk->Bc); free(wk->Bc2);
}

/*
 * Soft codeword, logZ and (optionally) posteriors / posterior argmax for all
 * sequences.  w: [n_seq][len] fp32, c: [S][V] fp32.
 * out_soft: [n_seq][len] fp64; out_logZ: [n_seq] fp64 (natural log);
 * out_post: NULL or [n_seq][n][S] fp64; out_argmax: NULL or [n_seq][n] int32
 * (lowest state on ties); out_top2: NULL or [n_seq][n][2] fp64 (largest and
 * second-largest posterior).  Returns 0 on success.
 */
int oracle_soft(const float* w, int64_t n_seq, int64_t len, int L, int k, int V, const float* c, double T,
                double* out_soft, double* out_logZ, double* out_post, int32_t* out_argmax, double* out_top2,
                int nthreads) {
  trellis_t tr;
  if (len % V != 0 || len < V || k < 1 || V < 1 || V > 8 || k * V > L || k * V > 8 || L > 20) return -10;
  if (trellis_init(&tr, L, k, V, len) != 0) return -11;
  int err = 0;
#ifdef _OPENMP
  if (nthreads > 0) omp_set_num_threads(nthreads);
#pragma omp parallel reduction(| : err)
#endif
  {
    work_t wk;
    int ok = work_alloc(&wk, &tr, 0) == 0;
    if (!ok) err |= 1;
    {
#ifdef _OPENMP
#pragma omp for schedule(dynamic, 1)
#endif
      for (int64_t q = 0; q < n_seq; ++q) {
        if (!ok) continue;
        const float* wq = w + q * len;
        log_potentials(&tr, wq, c, T, wk.th);
        forward(&tr, wk.th, wk.la);
        double logZ = lse_array(wk.la + (tr.n - 1) * tr.S, (int)tr.S);
        out_logZ[q] = logZ;
        for (int64_t s = 0; s < tr.S; ++s) wk.lb[s] = 0.0; /* beta_{n-1} = 1 (free end) */
        for (int64_t t = tr.n - 1; t >= 0; --t) {
          double ws[8] = {0, 0, 0, 0, 0, 0, 0, 0};
          double best = -1.0, second = -1.0;
          int32_t arg = 0;
          for (int64_t s = 0; s < tr.S; ++s) {
            double p = exp(wk.la[t * tr.S + s] + wk.lb[s] - logZ);
            if (out_post) out_post[(q * tr.n + t) * tr.S + s] = p;
            for (int v = 0; v < V; ++v) ws[v] += p * (double)c[s * V + v];
            if (p > best) { second = best; best = p; arg = (int32_t)s; }
            else if (p > second) second = p;
          }
          for (int v = 0; v < V; ++v) out_soft[q * len + t * V + v] = ws[v];
          if (out_argmax) out_argmax[q * tr.n + t] = arg;
          if (out_top2) { out_top2[(q * tr.n + t) * 2] = best; out_top2[(q * tr.n + t) * 2 + 1] = second; }
          if (t > 0) {
            backward_step(&tr, wk.th + t * tr.S, wk.lb, wk.lb2);
            double* sw = wk.lb; wk.lb = wk.lb2; wk.lb2 = sw;
          }
        }
      }
    }
    work_free(&wk);
  }
  free(tr.pred);
  return err ? -12 : 0;
}

/*
 * Vector-Jacobian product of  l = sum_t g_t . w_hat_t + gZ * logZ  with
 * respect to the weights w and the codebook c (first-order expectation
 * semiring, written with the conditional expectations
 *   A_t(s) = E[ sum_{u<t} h_u(s_u) | s_t = s ]   (prefix, forward sweep)
 *   B_t(s) = E[ sum_{u>t} h_u(s_u) | s_t = s ]   (suffix, backward sweep)
 * where h_u(s) = g_u . c(s)).  With p_t the posterior and Hbar = E[sum_u h_u]:
 *   G_t(s) = dl/dtheta_t(s) = p_t(s) (A_t(s) + h_t(s) + B_t(s) - Hbar + gZ),
 *   dl/dw_t   = sum_s G_t(s) (2/T) (c(s) - w_t),
 *   dl/dc(s)  = sum_t [ g_t p_t(s) + G_t(s) (2/T) (w_t - c(s)) ].
 * grad_w: [n_seq][len] fp64 (per sequence); grad_c: [S][V] fp64 summed over
 * all sequences; gZ: NULL (zero) or [n_seq] fp32; out_logZ/out_soft optional.
 */
int oracle_vjp(const float* w, int64_t n_seq, int64_t len, int L, int k, int V, const float* c, double T,
               const float* g, const float* gZ, double* grad_w, double* grad_c, double* out_logZ,
               double* out_Hbar, int nthreads) {
  trellis_t tr;
  if (len % V != 0 || len < V || k < 1 || V < 1 || V > 8 || k * V > L || k * V > 8 || L > 20) return -10;
  if (trellis_init(&tr, L, k, V, len) != 0) return -11;
  int nth = 1;
#ifdef _OPENMP
  if (nthreads > 0) omp_set_num_threads(nthreads);
  nth = omp_get_max_threads();
#endif
  double* gc_part = (double*)calloc((size_t)nth * (size_t)(tr.S * V), sizeof(double));
  if (!gc_part) { free(tr.pred); return -13; }
  int err = 0;
#ifdef _OPENMP
#pragma omp parallel reduction(| : err)
#endif
  {
    int tid = 0;
#ifdef _OPENMP
    tid = omp_get_thread_num();
#endif
    double* gcp = gc_part + (size_t)tid * (size_t)(tr.S * V);
    work_t wk;
    int ok = work_alloc(&wk, &tr, 1) == 0;
    if (!ok) err |= 1;
    {
      double buf[256], wts[256];
#ifdef _OPENMP
#pragma omp for schedule(dynamic, 1)
#endif
      for (int64_t q = 0; q < n_seq; ++q) {
        if (!ok) continue;
        const float* wq = w + q * len;
        const float* gq = g + q * len;
        double gz = gZ ? (double)gZ[q] : 0.0;
        log_potentials(&tr, wq, c, T, wk.th);
        forward(&tr, wk.th, wk.la);
        /* h_t(s) = g_t . c(s), evaluated on the fly */
#define H(t, s) hval(gq, c, V, (t), (s))
        /* forward conditional prefix expectation A */
        for (int64_t s = 0; s < tr.S; ++s) wk.A[s] = 0.0;
        for (int64_t t = 1; t < tr.n; ++t) {
          for (int64_t s = 0; s < tr.S; ++s) {
            double mx = -INFINITY;
            for (int i = 0; i < tr.B; ++i) {
              int64_t p = tr.pred[s * tr.B + i];
              buf[i] = wk.la[(t - 1) * tr.S + p];
              if (buf[i] > mx) mx = buf[i];
            }
            double num = 0.0, den = 0.0;
            for (int i = 0; i < tr.B; ++i) {
              int64_t p = tr.pred[s * tr.B + i];
              double wt = (mx == -INFINITY) ? 1.0 : exp(buf[i] - mx);
              num += wt * (wk.A[(t - 1) * tr.S + p] + H(t - 1, p));
              den += wt;
            }
            wk.A[t * tr.S + s] = num / den;
          }
        }
        double logZ = lse_array(wk.la + (tr.n - 1) * tr.S, (int)tr.S);
        if (out_logZ) out_logZ[q] = logZ;
        double Hbar = 0.0;
        for (int64_t s = 0; s < tr.S; ++s) {
          double p = exp(wk.la[(tr.n - 1) * tr.S + s] - logZ);
          Hbar += p * (wk.A[(tr.n - 1) * tr.S + s] + H(tr.n - 1, s));
        }
        if (out_Hbar) out_Hbar[q] = Hbar;
        /* backward: beta and the conditional suffix expectation B */
        for (int64_t s = 0; s < tr.S; ++s) { wk.lb[s] = 0.0; wk.Bc[s] = 0.0; }
        for (int64_t t = tr.n - 1; t >= 0; --t) {
          double gw[8] = {0, 0, 0, 0, 0, 0, 0, 0}, sg = 0.0;
          for (int64_t s = 0; s < tr.S; ++s) {
            double p = exp(wk.la[t * tr.S + s] + wk.lb[s] - logZ);
            double ht = H(t, s);
            double G = p * (wk.A[t * tr.S + s] + ht + wk.Bc[s] - Hbar + gz);
            sg += G;
            for (int v = 0; v < V; ++v) {
              double wv = (double)wq[t * V + v], cv = (double)c[s * V + v];
              gw[v] += G * (2.0 / T) * (cv - wv);
              gcp[s * V + v] += (double)gq[t * V + v] * p + G * (2.0 / T) * (wv - cv);
            }
          }
          (void)sg;
          for (int v = 0; v < V; ++v) grad_w[q * len + t * V + v] = gw[v];
          if (t > 0) {
            const double* th_t = wk.th + t * tr.S;
            for (int64_t pp = 0; pp < tr.S; ++pp) {
              double mx = -INFINITY;
              for (int b = 0; b < tr.B; ++b) {
                int64_t qq = succ(&tr, pp, b);
                wts[b] = th_t[qq] + wk.lb[qq];
                if (wts[b] > mx) mx = wts[b];
              }
              double num = 0.0, den = 0.0;
              for (int b = 0; b < tr.B; ++b) {
                int64_t qq = succ(&tr, pp, b);
                double wt = (mx == -INFINITY) ? 1.0 : exp(wts[b] - mx);
                num += wt * (wk.Bc[qq] + H(t, qq));
                den += wt;
              }
              wk.Bc2[pp] = num / den;
              wk.lb2[pp] = (mx == -INFINITY) ? -INFINITY : mx + log(den);
            }
            double* sw = wk.lb; wk.lb = wk.lb2; wk.lb2 = sw;
            sw = wk.Bc; wk.Bc = wk.Bc2; wk.Bc2 = sw;
          }
        }
#undef H
      }
    }
    work_free(&wk);
  }
  /* deterministic reduction of the per-thread codebook gradients */
  for (int64_t i = 0; i < tr.S * V; ++i) {
    double acc = 0.0;
    for (int t = 0; t < nth; ++t) acc += gc_part[(size_t)t * (size_t)(tr.S * V) + i];
    grad_c[i] = acc;
  }
  free(gc_part);
  free(tr.pred);
  return err ? -12 : 0;
}

/*
 * Viterbi decode (the T -> 0 limit): min-sum with the prescribed fp32 order
 *   q_t(s) = fl( sum_v fl( fl(w - c)^2 ) ), components added in order,
 *   delta_0(s) = q_0(s),  delta_t(s) = fl( min_{p -> s} delta_{t-1}(p) + q_t(s) ),
 * ties to the lowest predecessor; the final state is the lowest argmin.
 * out_states: [n_seq][n] int32; out_cost: NULL or [n_seq] fp32.
 */
int oracle_viterbi(const float* w, int64_t n_seq, int64_t len, int L, int k, int V, const float* c,
                   int32_t* out_states, float* out_cost, int nthreads) {
  trellis_t tr;
  if (len % V != 0 || len < V || k < 1 || V < 1 || V > 8 || k * V > L || k * V > 8 || L > 20) return -10;
  if (trellis_init(&tr, L, k, V, len) != 0) return -11;
  int err = 0;
#ifdef _OPENMP
  if (nthreads > 0) omp_set_num_threads(nthreads);
#pragma omp parallel reduction(| : err)
#endif
  {
    float* d0 = (float*)malloc(sizeof(float) * (size_t)tr.S);
    float* d1 = (float*)malloc(sizeof(float) * (size_t)tr.S);
    int32_t* bp = (int32_t*)malloc(sizeof(int32_t) * (size_t)(tr.S * tr.n));
    int ok = d0 && d1 && bp;
    if (!ok) err |= 1;
    {
#ifdef _OPENMP
#pragma omp for schedule(dynamic, 1)
#endif
      for (int64_t q = 0; q < n_seq; ++q) {
        if (!ok) continue;
        const float* wq = w + q * len;
        float* prev = d0; float* cur = d1;
        for (int64_t t = 0; t < tr.n; ++t) {
          for (int64_t s = 0; s < tr.S; ++s) {
            float acc = 0.0f;
            for (int v = 0; v < V; ++v) {
              float d = wq[t * V + v] - c[s * V + v];
              float sq = d * d;
              acc = (v == 0) ? sq : acc + sq;
            }
            if (t == 0) { cur[s] = acc; continue; }
            float best = prev[tr.pred[s * tr.B]];
            int32_t arg = tr.pred[s * tr.B];
            for (int i = 1; i < tr.B; ++i) {
              int32_t p = tr.pred[s * tr.B + i];
              if (prev[p] < best) { best = prev[p]; arg = p; }
            }
            bp[t * tr.S + s] = arg;
            cur[s] = best + acc;
          }
          float* sw = prev; prev = cur; cur = sw;
        }
        int32_t s = 0;
        for (int64_t i = 1; i < tr.S; ++i) if (prev[i] < prev[s]) s = (int32_t)i;
        if (out_cost) out_cost[q] = prev[s];
        for (int64_t t = tr.n - 1; t >= 0; --t) {
          out_states[q * tr.n + t] = s;
          if (t > 0) s = bp[t * tr.S + s];
        }
      }
    }
    free(d0); free(d1); free(bp);
  }
  free(tr.pred);
  return err ? -12 : 0;
}

/* Successor / predecessor tables for tests of the trellis rule itself. */
int oracle_pred_table(int L, int k, int V, int32_t* out_pred) {
  trellis_t tr;
  if (k < 1 || V < 1 || k * V > L || k * V > 8 || L > 20) return -10;
  if (trellis_init(&tr, L, k, V, V) != 0) return -11;
  memcpy(out_pred, tr.pred, sizeof(int32_t) * (size_t)(tr.S * tr.B));
  free(tr.pred);
  return 0;
}
