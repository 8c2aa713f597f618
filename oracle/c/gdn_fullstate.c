/*
 * Full-state GDN beam tree in plain C, fp64.  TEST INFRASTRUCTURE: the timed
 * CPU baseline and a second, independently written copy of the oracle.  It is
 * built by the package's build step but only the tests, the smoke check and
 * the benchmark's CPU-baseline leg load it.  It shares no code with the CUDA
 * library.
 *
 * Computes, per request r and head h, for every decode step t and every beam b
 * (OneLA, evolve.pub review, section 3.2 / equation 2, FullState semantics):
 *   S      = copy of the parent's state S_{t-1}[parent_t[b]]   (S_0 = S0)
 *   alpha  = exp(g)
 *   delta  = beta * (v - alpha * S k)
 *   S      = alpha * S + delta k^T
 *   o      = S q
 *
 * Flat layouts (row-major), concatenated over steps t = 0..T-1 with
 * W_t = Wsteps[t] beams at step t and W_prev = 1 at the first step:
 *   S0            [R][H][dv][dk]
 *   q, k          [R][W_t][H][dk]
 *   v, o, delta   [R][W_t][H][dv]
 *   g, beta       [R][W_t][H]
 *   parents       [R][W_t]            (int32, each in [0, W_prev))
 * Returns 0 on success, -1 on bad arguments, -2 on an out-of-range parent,
 * -3 when memory for the per-beam states cannot be had.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

int gdn_oracle_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}

int gdn_oracle_beam_decode(int R, int H, int dk, int dv, int T,
                           const int32_t *Wsteps, const double *S0,
                           const double *q, const double *k, const double *v,
                           const double *g, const double *beta,
                           const int32_t *parents, double *o, double *delta,
                           int nthreads) {
  if (R <= 0 || H <= 0 || dk <= 0 || dv <= 0 || T < 0 || !Wsteps || !S0)
    return -1;
  int Wmax = 1;
  for (int t = 0; t < T; ++t) {
    if (Wsteps[t] <= 0) return -1;
    if (Wsteps[t] > Wmax) Wmax = Wsteps[t];
  }
  /* Validate every parent before touching any state. */
  {
    size_t off = 0;
    int Wp = 1;
    for (int t = 0; t < T; ++t) {
      for (size_t i = 0; i < (size_t)R * Wsteps[t]; ++i)
        if (parents[off + i] < 0 || parents[off + i] >= Wp) return -2;
      off += (size_t)R * Wsteps[t];
      Wp = Wsteps[t];
    }
  }
#ifdef _OPENMP
  if (nthreads > 0) omp_set_num_threads(nthreads);
#else
  (void)nthreads;
#endif
  const size_t SS = (size_t)dv * dk;
  double *Sprev = (double *)malloc(sizeof(double) * SS * (size_t)Wmax);
  double *Snext = (double *)malloc(sizeof(double) * SS * (size_t)Wmax);
  if (!Sprev || !Snext) {
    free(Sprev);
    free(Snext);
    return -3;
  }
  for (int r = 0; r < R; ++r) {
    for (int h = 0; h < H; ++h) {
      memcpy(Sprev, S0 + ((size_t)r * H + h) * SS, sizeof(double) * SS);
      size_t offk = 0, offv = 0, offs = 0, offp = 0;
      for (int t = 0; t < T; ++t) {
        const int W = Wsteps[t];
#pragma omp parallel for schedule(static)
        for (int b = 0; b < W; ++b) {
          const size_t row = ((size_t)r * W + b) * H + h;
          const int p = parents[offp + (size_t)r * W + b];
          const double *kb = k + offk + row * dk;
          const double *qb = q + offk + row * dk;
          const double *vb = v + offv + row * dv;
          const double a = exp(g[offs + row]);
          const double be = beta[offs + row];
          double *S = Snext + (size_t)b * SS;
          memcpy(S, Sprev + (size_t)p * SS, sizeof(double) * SS);
          double *db = delta + offv + row * dv;
          double *ob = o + offv + row * dv;
          for (int i = 0; i < dv; ++i) {
            double u = 0.0;
            for (int j = 0; j < dk; ++j) u += S[(size_t)i * dk + j] * kb[j];
            db[i] = be * (vb[i] - a * u);
          }
          for (int i = 0; i < dv; ++i) {
            double acc = 0.0;
            for (int j = 0; j < dk; ++j) {
              double s = a * S[(size_t)i * dk + j] + db[i] * kb[j];
              S[(size_t)i * dk + j] = s;
              acc += s * qb[j];
            }
            ob[i] = acc;
          }
        }
        double *tmp = Sprev;
        Sprev = Snext;
        Snext = tmp;
        offk += (size_t)R * W * H * dk;
        offv += (size_t)R * W * H * dv;
        offs += (size_t)R * W * H;
        offp += (size_t)R * W;
      }
    }
  }
  free(Sprev);
  free(Snext);
  return 0;
}
