/*
 * ssd_oracle.c -- TEST INFRASTRUCTURE, not the product.
 *
 * A plain, slow, fp64 CPU implementation of the scalar-decay selective SSM
 * that the chunked SSD forward pass computes.  Only the tests, the package's
 * smoke check and the bench's CPU-baseline leg may load this library; the CUDA
 * path shares no code with it.
 *
 * Definition followed ("Transformers are SSMs", wikillm.com card, Method):
 *   step 1 (SSMs as matrices, sec. 2-3): h_t = A_t h_{t-1} + B_t x_t, y_t = C_t^T h_t
 *   step 2 (scalar-identity SSMs, sec. 5.1): A_t = a_t I
 *   step 3 (1-SS masks, sec. 3): the token's own input enters undecayed
 *   step 6/7 (Mamba-2 block, discretisation): a_t = exp(dt_t * A_h), the SSM
 *     input is dt_t * x_t, and the skip D_h * x_t uses the unscaled x_t.
 * Per sequence s and head h, with g the head's group and S a P x N state:
 *   S = init[s,h] (or 0)
 *   for each token t of s:  a = exp(dt[t,h] * A[h])
 *                           S[p][n] = a * S[p][n] + dt[t,h] * x[t,h,p] * B[t,g,n]
 *                           y[t,h,p] = sum_n C[t,g,n] * S[p][n] + D[h] * x[t,h,p]
 *   final[s,h] = S
 * The chunked algorithm reaches exactly this result (up to rounding order).
 *
 * Layouts (row-major, contiguous): x, y (T, H, P); dt (T, H); A, D (H);
 * B, C (T, G, N); init, final (nseq, H, P, N).  Sequence s covers tokens
 * [seq_off[s], seq_off[s+1]).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* head -> group: explicit table when given, else contiguous blocks of H/G heads. */
static int64_t group_of(int64_t h, int64_t H, int64_t G, const int32_t* head_group) {
  return head_group ? (int64_t)head_group[h] : h / (H / G);
}

int oracle_ssd_forward(int64_t nseq, const int64_t* seq_off, int64_t H, int64_t P, int64_t N, int64_t G,
                       const int32_t* head_group,
                       const double* x, const double* dt, const double* A, const double* B, const double* C,
                       const double* D, const double* init, double* y, double* final_state, int nthreads) {
  if (nseq < 0 || H <= 0 || P <= 0 || N <= 0 || G <= 0 || (!head_group && H % G)) return 1;
#ifdef _OPENMP
  if (nthreads > 0) omp_set_num_threads(nthreads);
#else
  (void)nthreads;
#endif
  int err = 0;
#pragma omp parallel
  {
    double* S = (double*)malloc(sizeof(double) * (size_t)(P * N));
    if (!S) {
#pragma omp atomic write
      err = 2;
    }
#pragma omp for schedule(dynamic, 1)
    for (int64_t sh = 0; sh < nseq * H; ++sh) {
      if (!S) continue;
      const int64_t s = sh / H, h = sh % H;
      const int64_t g = group_of(h, H, G, head_group);
      if (init)
        memcpy(S, init + (s * H + h) * P * N, sizeof(double) * (size_t)(P * N));
      else
        memset(S, 0, sizeof(double) * (size_t)(P * N));
      const double Dh = D ? D[h] : 0.0;
      for (int64_t t = seq_off[s]; t < seq_off[s + 1]; ++t) {
        const double dtt = dt[t * H + h];
        const double a = exp(dtt * A[h]);
        const double* xt = x + (t * H + h) * P;
        const double* Bt = B + (t * G + g) * N;
        const double* Ct = C + (t * G + g) * N;
        double* yt = y + (t * H + h) * P;
        for (int64_t p = 0; p < P; ++p) {
          const double u = dtt * xt[p];
          double* Sp = S + p * N;
          double acc = 0.0;
          for (int64_t n = 0; n < N; ++n) {
            Sp[n] = a * Sp[n] + u * Bt[n];
            acc += Ct[n] * Sp[n];
          }
          yt[p] = acc + Dh * xt[p];
        }
      }
      if (final_state) memcpy(final_state + (s * H + h) * P * N, S, sizeof(double) * (size_t)(P * N));
    }
    free(S);
  }
  return err;
}

/*
 * One recurrent decode step (the pages' generation mode, Method step 8, sec. 6.3:
 * N^2-per-step inference).  For each batch row b and head h, the state is
 * advanced in place by one token and the token's output is written:
 *   a = exp(dt[b,h] * A[h]);  S = a*S + dt*x[b,h,:] B[b,g,:]^T;  y[b,h,:] = S C[b,g,:] + D[h] x[b,h,:]
 * Layouts: x, y (batch, H, P); dt (batch, H); B, C (batch, G, N); state (batch, H, P, N).
 */
int oracle_ssd_decode_step(int64_t batch, int64_t H, int64_t P, int64_t N, int64_t G,
                           const double* x, const double* dt, const double* A, const double* B, const double* C,
                           const double* D, double* state, double* y) {
  if (batch < 0 || H <= 0 || P <= 0 || N <= 0 || G <= 0 || H % G) return 1;
  for (int64_t b = 0; b < batch; ++b)
    for (int64_t h = 0; h < H; ++h) {
      const int64_t g = h / (H / G);
      const double dtt = dt[b * H + h];
      const double a = exp(dtt * A[h]);
      const double* xt = x + (b * H + h) * P;
      const double* Bt = B + (b * G + g) * N;
      const double* Ct = C + (b * G + g) * N;
      double* S = state + (b * H + h) * P * N;
      for (int64_t p = 0; p < P; ++p) {
        double acc = 0.0;
        for (int64_t n = 0; n < N; ++n) {
          S[p * N + n] = a * S[p * N + n] + dtt * xt[p] * Bt[n];
          acc += Ct[n] * S[p * N + n];
        }
        y[(b * H + h) * P + p] = acc + (D ? D[h] : 0.0) * xt[p];
      }
    }
  return 0;
}
