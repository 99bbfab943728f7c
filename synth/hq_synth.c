/*
 * hq_synth.c -- host side of the synthetic partial-sum generator (see hq_synth_core.h).
 *
 * Builds a per-column scale (LogNormal column std with planted outlier columns, the
 * "consistent structure" of communicated features described on the page
 * "Revolutionizing LLM Inference: The Power of Efficient Low-Bit Communication",
 * section "Leveraging Outliers for Efficient Communication") and fills any
 * sub-block [r0,r1) x [t0,t1) x [h0,h1) of a batch [P][T][H] of bf16 values.
 *
 * Holds none of the compression method's arithmetic.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>

#include "hq_synth_core.h"

/*
 * colscale[h] = exp(sigma * N_h) for every column, then the first n_out entries of a
 * seeded Fisher-Yates permutation of [0, H) are the outlier columns, whose scale is
 * multiplied by out_mult.  outliers[0..n_out) receives those column indices.
 * exp() here runs on the host only; the device generator is handed colscale.
 */
int syn_colscale(uint64_t seed, int H, double sigma, int n_out, double out_mult,
                 double* colscale, int32_t* outliers) {
  if (H <= 0 || n_out < 0 || n_out > H) return 1;
  uint64_t kstd = syn_key(seed, SYN_COLSTD, 0, 0);
  for (int h = 0; h < H; ++h) colscale[h] = exp(sigma * syn_normal(kstd, 2ULL * (uint64_t)h));
  int32_t* perm = (int32_t*)malloc(sizeof(int32_t) * (size_t)H);
  if (!perm) return 2;
  for (int h = 0; h < H; ++h) perm[h] = h;
  uint64_t kperm = syn_key(seed, SYN_PERM, 0, 0);
  for (int i = H - 1; i >= 1; --i) {
    uint64_t j = syn_draw(kperm, (uint64_t)(H - 1 - i)) % (uint64_t)(i + 1);
    int32_t tmp = perm[i];
    perm[i] = perm[j];
    perm[j] = tmp;
  }
  for (int m = 0; m < n_out; ++m) {
    outliers[m] = perm[m];
    colscale[perm[m]] *= out_mult;
  }
  free(perm);
  return 0;
}

/* The per-rank stream keys of one batch. */
void syn_rank_keys(uint64_t seed, int purpose, int batch, int P, uint64_t* keys) {
  for (int r = 0; r < P; ++r)
    keys[r] = syn_key(seed, (uint64_t)purpose, (uint64_t)batch, (uint64_t)r);
}

/*
 * out[(r-r0)][(t-t0)][(h-h0)] = x[r][t][h] of batch (purpose, batch) of a [P][T][H]
 * partial-sum tensor.  Only H (the row length) enters an element's counter, so P and T
 * are not needed; the caller checks that the block lies inside the tensor.
 */
void syn_fill(uint64_t seed, int purpose, int batch, int H, int dist, const double* colscale,
              double spike_p, double spike_mult, int r0, int r1, int t0, int t1, int h0, int h1,
              uint16_t* out) {
  const int nt = t1 - t0, nh = h1 - h0;
  for (int r = r0; r < r1; ++r) {
    const uint64_t key = syn_key(seed, (uint64_t)purpose, (uint64_t)batch, (uint64_t)r);
#pragma omp parallel for schedule(static)
    for (int t = t0; t < t1; ++t) {
      uint16_t* row = out + ((size_t)(r - r0) * nt + (size_t)(t - t0)) * nh;
      for (int h = h0; h < h1; ++h) {
        uint64_t elem = (uint64_t)t * (uint64_t)H + (uint64_t)h;
        row[h - h0] = syn_element(key, elem, dist, colscale ? colscale[h] : 1.0, spike_p, spike_mult);
      }
    }
  }
}

/* Same element, one at a time (sampled checks on full-size tensors). */
uint16_t syn_one(uint64_t seed, int purpose, int batch, int H, int dist, double colscale_h,
                 double spike_p, double spike_mult, int r, int t, int h) {
  uint64_t key = syn_key(seed, (uint64_t)purpose, (uint64_t)batch, (uint64_t)r);
  return syn_element(key, (uint64_t)t * (uint64_t)H + (uint64_t)h, dist, colscale_h, spike_p, spike_mult);
}

/* Test hooks for the series routines (compared with libm in the generator's tests). */
double syn_log_for_test(double x) { return syn_log(x); }
double syn_cos2pi_for_test(double u) { return syn_cos2pi(u); }
