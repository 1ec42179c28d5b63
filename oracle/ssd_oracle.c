/*
 * ssd_oracle.c -- float64 CPU oracle for the Mamba-2 SSD layer.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path (the CUDA library and
 * its Python binding) may link, load or call this file.  Only the tests, the
 * smoke check in __graft_entry__ and bench.py's CPU-baseline / reference arm
 * use it.  It shares no source, header, table or helper with the CUDA path.
 *
 * What it computes (the plain definition, one independent chain per
 * (batch b, head h, channel p), sequential in time t):
 *
 *   s[n]   <- exp(dt[b,t,h] * A[h]) * s[n] + dt[b,t,h] * B[b,t,g,n] * x[b,t,h,p]
 *   y[t]    = sum_n C[b,t,g,n] * s[n] + D[h] * x[b,t,h,p]         (uses the updated s)
 *   g       = h / (H / G)                                          (contiguous head groups)
 *
 * Sources:
 *  - decay exp(Delta*A) from zero-order hold and the input term Delta*B (the
 *    small-step form of B-bar): "State Space Model" (book.paithon.it), section
 *    "Un sistema che riassume il passato"; "State Space Models (SSM)"
 *    (ultralytics.com glossary), section "Come funzionano gli SSM".
 *  - the linear recurrence h_t = A_t h_{t-1} + b_t with a scalar transition
 *    A_t = a_t I: "State Space Model", sections "Due strade, una meta" and
 *    "Da ricordare".
 *  - output read from the new state, y_t = C h_t: "State Space Models (SSM)",
 *    section "Come funzionano gli SSM".
 *  - the skip term D x: "Puntata 205 -- State Space Models e Mamba"
 *    (aiperbabbani.it), section "Cos'e un SSM, in 30 secondi".
 *  - input-dependent Delta, B, C (selectivity): same page, section
 *    "Mamba (Gu & Dao, dicembre 2023): selective scan".
 *
 * Readings where the pages are silent:
 *  - the initial state is the state before token 0, so token 0 decays it once;
 *  - dt and A are used as given (no softplus or clamp inside);
 *  - inputs stored as bf16 or f32 are widened exactly to double.
 *
 * Build: gcc -O2 -fopenmp -shared -fPIC ssd_oracle.c -o libssd_oracle.so -lm
 * (oracle/build.py does this).  The optional ORACLE_MUTATION macro compiles a
 * deliberately broken variant used only by the tests that show the pins catch
 * plausible mistakes; the default build has no mutation.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#ifndef ORACLE_MUTATION
#define ORACLE_MUTATION 0
#endif

/* Storage dtypes of x, B, C. */
#define ORACLE_F32 0
#define ORACLE_BF16 1

static double widen(const void* base, int64_t i, int dtype) {
  if (dtype == ORACLE_BF16) {
    uint16_t h = ((const uint16_t*)base)[i];
    uint32_t u = ((uint32_t)h) << 16; /* bf16 is the top half of an f32: exact */
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
  }
  return (double)((const float*)base)[i];
}

/*
 * Run the recurrence for a list of chains.
 *
 * Layouts (row-major, contiguous):
 *   x  [batch, seqlen, nheads, headdim]      (io dtype)
 *   dt [batch, seqlen, nheads]               (f32)
 *   A  [nheads], D [nheads] (D may be NULL -> 0)
 *   B, C [batch, seqlen, ngroups, dstate]    (io dtype)
 *   h0 [n_chains, dstate] double, or NULL for zeros
 *   y  [n_chains, seqlen] double  (output)
 *   h1 [n_chains, dstate] double, or NULL  (output: state after the last token)
 * chain_ids[i] = (b * nheads + h) * headdim + p; NULL means all chains in order.
 * Returns 0, or -1 on bad arguments.
 */
int ssd_oracle_scan_f64(const void* x, const float* dt, const float* A, const void* Bm,
                        const void* Cm, const float* D, int io_dtype, const double* h0,
                        double* y, double* h1, int64_t batch, int64_t seqlen, int64_t nheads,
                        int64_t headdim, int64_t dstate, int64_t ngroups,
                        const int64_t* chain_ids, int64_t n_chains, int nthreads) {
  if (!x || !dt || !A || !Bm || !Cm || !y) return -1;
  if (batch <= 0 || seqlen < 0 || nheads <= 0 || headdim <= 0 || dstate <= 0 || ngroups <= 0)
    return -1;
  if (nheads % ngroups != 0) return -1;
  if (io_dtype != ORACLE_F32 && io_dtype != ORACLE_BF16) return -1;
  const int64_t total = batch * nheads * headdim;
  if (!chain_ids) n_chains = total;
  const int64_t heads_per_group = nheads / ngroups;
#ifdef _OPENMP
  if (nthreads > 0) omp_set_num_threads(nthreads);
#else
  (void)nthreads;
#endif
  int bad = 0;
#pragma omp parallel
  {
    double* s = (double*)malloc(sizeof(double) * (size_t)dstate);
#pragma omp for schedule(dynamic, 1)
    for (int64_t i = 0; i < n_chains; ++i) {
      if (!s) { bad = 1; continue; }
      const int64_t id = chain_ids ? chain_ids[i] : i;
      if (id < 0 || id >= total) { bad = 1; continue; }
      const int64_t p = id % headdim;
      const int64_t h = (id / headdim) % nheads;
      const int64_t b = id / (headdim * nheads);
#if ORACLE_MUTATION == 3
      const int64_t g = h % ngroups; /* planted mistake: interleaved group map */
#else
      const int64_t g = h / heads_per_group;
#endif
      for (int64_t n = 0; n < dstate; ++n) s[n] = h0 ? h0[i * dstate + n] : 0.0;
#if ORACLE_MUTATION == 6
      int first = 1;
#endif
      const double a_h = (double)A[h];
      const double d_h = D ? (double)D[h] : 0.0;
      for (int64_t t = 0; t < seqlen; ++t) {
        const int64_t bt = b * seqlen + t;
        const double delta = (double)dt[bt * nheads + h];
        const double xv = widen(x, (bt * nheads + h) * headdim + p, io_dtype);
#if ORACLE_MUTATION == 4
        const double decay = exp(a_h); /* planted mistake: step size left out of the decay */
#else
        const double decay = exp(delta * a_h);
#endif
        const double u = delta * xv;
        const int64_t bc = (bt * ngroups + g) * dstate;
        double acc = 0.0;
#if ORACLE_MUTATION == 2
        for (int64_t n = 0; n < dstate; ++n) acc += widen(Cm, bc + n, io_dtype) * s[n];
#endif
        for (int64_t n = 0; n < dstate; ++n) {
#if ORACLE_MUTATION == 5
          const double bn = widen(Cm, bc + n, io_dtype); /* planted mistake: B and C swapped */
#else
          const double bn = widen(Bm, bc + n, io_dtype);
#endif
#if ORACLE_MUTATION == 6
          /* planted mistake: the initial state enters after the first decay */
          s[n] = (first ? s[n] : decay * s[n]) + u * bn;
#else
          s[n] = decay * s[n] + u * bn;
#endif
        }
#if ORACLE_MUTATION == 6
        first = 0;
#endif
#if ORACLE_MUTATION != 2
        for (int64_t n = 0; n < dstate; ++n) {
#if ORACLE_MUTATION == 5
          acc += widen(Bm, bc + n, io_dtype) * s[n];
#else
          acc += widen(Cm, bc + n, io_dtype) * s[n];
#endif
        }
#endif
#if ORACLE_MUTATION == 1
        y[i * seqlen + t] = acc; /* planted mistake: skip term dropped */
#else
        y[i * seqlen + t] = acc + d_h * xv;
#endif
      }
      if (h1)
        for (int64_t n = 0; n < dstate; ++n) h1[i * dstate + n] = s[n];
    }
    free(s);
  }
  return bad ? -1 : 0;
}

/* Version tag so the Python side can check it loaded this file's build. */
int ssd_oracle_mutation(void) { return ORACLE_MUTATION; }
