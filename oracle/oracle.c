/*
 * fp64 CPU oracle for the clip-parallel temporal modules of Video-Infinity.
 *
 * TEST INFRASTRUCTURE ONLY.  This is the plain, slow, obviously correct
 * statement of what the three temporal modules compute.  Only the tests, the
 * package's smoke check and the benchmark's CPU-baseline leg may load it; the
 * CUDA library never does, and the two share no code.
 *
 * Source: "Video-Infinity: Distributed Long Video Generation" (write-up on
 * news.43zhubao.com), paragraphs on clip parallelism and on the three
 * temporal modules (attention, conv, GroupNorm).  Where that text is
 * garbled or silent the reading adopted is stated at each function.
 *
 * Data layout of every activation: [P positions][F frames][C channels],
 * row-major, C = heads * d innermost.  Inputs arrive either as fp32 values
 * (dtype 0) or as bf16 bit patterns (dtype 1); both are widened exactly to
 * double, and every sum, exponential and division below is done in double.
 * Parallelism: OpenMP over independent positions (or clips), which changes
 * no arithmetic.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#ifdef _OPENMP
#include <omp.h>
#endif

/* Exact widening of one input element to double (dtype 0: fp32 values,
   1: bf16 bit patterns, 2: doubles, used to feed one module's exact output
   into the next). */
static double in_val(const void* base, int64_t idx, int dtype) {
  if (dtype == 2) return ((const double*)base)[idx];
  if (dtype == 0) return (double)((const float*)base)[idx];
  uint32_t u = (uint32_t)((const uint16_t*)base)[idx] << 16;
  float f;
  memcpy(&f, &u, 4);
  return (double)f;
}

#ifdef _OPENMP
/* The process's default thread count, read before any call changes it. */
static int all_threads(void) {
  static int all = 0;
  if (all == 0) all = omp_get_max_threads();
  return all;
}
#endif

/* nthreads > 0: that many threads for this call; 0: the process default (every
   call sets it, so a one-thread call does not leave the next call on one thread). */
static void set_threads(int nthreads) {
#ifdef _OPENMP
  const int all = all_threads();
  omp_set_num_threads(nthreads > 0 ? nthreads : all);
#else
  (void)nthreads;
#endif
}

int oracle_max_threads(void) {
#ifdef _OPENMP
  return all_threads();
#else
  return 1;
#endif
}

/*
 * Key/value frame list of clip i (dual-domain attention, attention-module
 * paragraph).  The clip owns frames [s, e) with L = F/N, s = i*L, e = s+L.
 * The list is the concatenation, duplicates kept, of
 *   own    : s .. e-1                                   (the clip itself)
 *   C_pre  : s-n_pre .. s-1, only when i > 0            (tail of clip i-1)
 *   C_post : e .. e+n_post-1, only when i < N-1         (head of clip i+1)
 *   C_glob : j*floor(F/n_global) for j < n_global       (uniform samples of
 *            the whole video, the same for every clip)
 * Reading: the pages drop the symbols of the index sets; the sizes 8/8/16 and
 * the stride F/16 are the fixed reading, the ends are absent (not zero keys)
 * and nothing is de-duplicated.  Requires n_pre, n_post <= L.
 * Returns the list length and writes the frames to out (room for
 * L + n_pre + n_post + n_global entries).
 */
int oracle_key_frames(int i, int F, int N, int n_pre, int n_post, int n_global, int* out) {
  const int L = F / N, s = i * L, e = s + L;
  int n = 0;
  for (int f = s; f < e; ++f) out[n++] = f;
  if (i > 0)
    for (int f = s - n_pre; f < s; ++f) out[n++] = f;
  if (i < N - 1)
    for (int f = e; f < e + n_post; ++f) out[n++] = f;
  if (n_global > 0) {
    const int stride = F / n_global;
    for (int j = 0; j < n_global; ++j) out[n++] = j * stride;
  }
  return n;
}

/*
 * Dual-domain temporal attention (attention-module paragraph).
 * For each listed position p, head h and clip i, every query frame f of the
 * clip attends over the clip's key list K_i:
 *   s_j  = (q[p,f,h,:] . k[p,j,h,:]) / sqrt(d)        for j in K_i
 *   o    = sum_j exp(s_j - max s) v[p,j,h,:] / sum_j exp(s_j - max s)
 * No positional bias, no causal mask; the scale is 1/sqrt(d).
 * out: [n_pos][F][C] doubles, positions taken from pos[].
 */
void oracle_dual_attn(const void* q, const void* k, const void* v, int dtype, double* out,
                      int F, int N, int P, int heads, int d, int n_pre, int n_post, int n_global,
                      const int* pos, int n_pos, int nthreads) {
  (void)P;
  set_threads(nthreads);
  const int C = heads * d, L = F / N;
  const int maxk = L + n_pre + n_post + n_global;
  const double scale = 1.0 / sqrt((double)d);
#pragma omp parallel
  {
    int* keys = (int*)malloc(sizeof(int) * (size_t)maxk);
    double* w = (double*)malloc(sizeof(double) * (size_t)maxk);
#pragma omp for schedule(dynamic)
    for (int64_t job = 0; job < (int64_t)n_pos * heads * N; ++job) {
      const int pi = (int)(job / ((int64_t)heads * N));
      const int h = (int)((job / N) % heads);
      const int i = (int)(job % N);
      const int64_t pbase = (int64_t)pos[pi] * F * C;
      const int nk = oracle_key_frames(i, F, N, n_pre, n_post, n_global, keys);
      for (int f = i * L; f < (i + 1) * L; ++f) {
        double m = -INFINITY;
        for (int j = 0; j < nk; ++j) {
          double dot = 0.0;
          for (int c = 0; c < d; ++c)
            dot += in_val(q, pbase + (int64_t)f * C + h * d + c, dtype) *
                   in_val(k, pbase + (int64_t)keys[j] * C + h * d + c, dtype);
          w[j] = dot * scale;
          if (w[j] > m) m = w[j];
        }
        double denom = 0.0;
        for (int j = 0; j < nk; ++j) {
          w[j] = exp(w[j] - m);
          denom += w[j];
        }
        double* o = out + ((int64_t)pi * F + f) * C + h * d;
        for (int c = 0; c < d; ++c) {
          double acc = 0.0;
          for (int j = 0; j < nk; ++j)
            acc += w[j] * in_val(v, pbase + (int64_t)keys[j] * C + h * d + c, dtype);
          o[c] = acc / denom;
        }
      }
    }
    free(keys);
    free(w);
  }
}

/*
 * Temporal convolution with neighbour padding (conv-module paragraph).
 * Clip i (frames [s, e)) is extended by n = floor(k/2) frames on each side:
 * C_pre = the last n frames of clip i-1 and C_post = the first n frames of
 * clip i+1, zeros where there is no neighbour (the video ends).  A valid
 * cross-correlation (PyTorch Conv1d orientation) over the extended clip gives
 * the clip's L output frames:
 *   y[p,f,co] = b[co] + sum_t sum_ci W[co,ci,t] * ext[f - s + t][ci]
 * where ext[u] holds frame s - n + u.  Requires odd k and n <= L.
 * w: [C_out][C_in][k] and b: [C] in `dtype`; x in `x_dtype`;
 * y: [n_pos][F][C] doubles.
 */
void oracle_temporal_conv(const void* x, const void* w, const void* b, int dtype, double* y,
                          int F, int N, int P, int C, int k, const int* pos, int n_pos,
                          int nthreads, int x_dtype) {
  (void)P;
  set_threads(nthreads);
  const int L = F / N, n = k / 2, E = L + 2 * n;
#pragma omp parallel
  {
    double* ext = (double*)malloc(sizeof(double) * (size_t)E * C);
#pragma omp for schedule(dynamic)
    for (int64_t job = 0; job < (int64_t)n_pos * N; ++job) {
      const int pi = (int)(job / N), i = (int)(job % N);
      const int64_t pbase = (int64_t)pos[pi] * F * C;
      const int s = i * L;
      /* Build the padded clip: [C_pre | own frames | C_post]. */
      for (int u = 0; u < E; ++u) {
        const int f = s - n + u;
        const int from_prev = (u < n), from_next = (u >= n + L);
        const int present = (from_prev && i > 0) || (from_next && i < N - 1) ||
                            (!from_prev && !from_next);
        for (int c = 0; c < C; ++c)
          ext[(int64_t)u * C + c] = present ? in_val(x, pbase + (int64_t)f * C + c, x_dtype) : 0.0;
      }
      for (int fl = 0; fl < L; ++fl)
        for (int co = 0; co < C; ++co) {
          double acc = in_val(b, co, dtype);
          for (int t = 0; t < k; ++t)
            for (int ci = 0; ci < C; ++ci)
              acc += in_val(w, ((int64_t)co * C + ci) * k + t, dtype) * ext[(int64_t)(fl + t) * C + ci];
          y[((int64_t)pi * F + s + fl) * C + co] = acc;
        }
    }
    free(ext);
  }
}

/*
 * GroupNorm with global statistics (GroupNorm-module paragraph), in the
 * order the pages give:
 *   1. each clip i computes its group means mu_{i,g} over its frames, all
 *      positions and the C/G channels of group g;
 *   2. the clip means are aggregated into the global mean
 *      mu_g = sum_i n_i mu_{i,g} / sum_i n_i;
 *   3. each clip computes its sum of squared deviations about mu_g;
 *   4. these are aggregated into the global variance
 *      var_g = sum_i SS_{i,g} / n  (biased, divide by the count).
 * Reading of the truncated last sentence: mu_g and var_g serve as the
 * normalisation statistics of every clip,
 *   y = (x - mu_g) / sqrt(var_g + eps) * gamma[c] + beta[c],
 * so the result is the unpartitioned GroupNorm of the whole latent
 * (batch 1; groups are C/G contiguous channels).
 * mean_out/var_out: [groups]; y: [n_pos][F][C] doubles (may be NULL).
 */
void oracle_groupnorm_global(const void* x, const void* gamma, const void* beta, int dtype,
                             double* y, double* mean_out, double* var_out, int F, int N, int P,
                             int C, int groups, double eps, const int* pos, int n_pos,
                             int nthreads) {
  set_threads(nthreads);
  const int L = F / N, cg = C / groups;
  double* clip_mean = (double*)calloc((size_t)N * groups, sizeof(double));
  double* clip_ss = (double*)calloc((size_t)N * groups, sizeof(double));
  const double n_clip = (double)L * P * cg;
  /* Step 1: per-clip group means. */
#pragma omp parallel for schedule(dynamic)
  for (int i = 0; i < N; ++i)
    for (int g = 0; g < groups; ++g) {
      double s = 0.0;
      for (int p = 0; p < P; ++p)
        for (int f = i * L; f < (i + 1) * L; ++f)
          for (int c = g * cg; c < (g + 1) * cg; ++c)
            s += in_val(x, ((int64_t)p * F + f) * C + c, dtype);
      clip_mean[(int64_t)i * groups + g] = s / n_clip;
    }
  /* Step 2: global means. */
  double* mu = (double*)calloc((size_t)groups, sizeof(double));
  for (int g = 0; g < groups; ++g) {
    double s = 0.0;
    for (int i = 0; i < N; ++i) s += n_clip * clip_mean[(int64_t)i * groups + g];
    mu[g] = s / (n_clip * N);
  }
  /* Step 3: per-clip squared deviations about the global mean. */
#pragma omp parallel for schedule(dynamic)
  for (int i = 0; i < N; ++i)
    for (int g = 0; g < groups; ++g) {
      double s = 0.0;
      for (int p = 0; p < P; ++p)
        for (int f = i * L; f < (i + 1) * L; ++f)
          for (int c = g * cg; c < (g + 1) * cg; ++c) {
            const double dv = in_val(x, ((int64_t)p * F + f) * C + c, dtype) - mu[g];
            s += dv * dv;
          }
      clip_ss[(int64_t)i * groups + g] = s;
    }
  /* Step 4: global variance. */
  double* var = (double*)calloc((size_t)groups, sizeof(double));
  for (int g = 0; g < groups; ++g) {
    double s = 0.0;
    for (int i = 0; i < N; ++i) s += clip_ss[(int64_t)i * groups + g];
    var[g] = s / (n_clip * N);
  }
  if (mean_out) memcpy(mean_out, mu, sizeof(double) * groups);
  if (var_out) memcpy(var_out, var, sizeof(double) * groups);
  if (y) {
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < (int64_t)n_pos * F; ++r) {
      const int pi = (int)(r / F), f = (int)(r % F);
      for (int c = 0; c < C; ++c) {
        const int g = c / cg;
        const double xv = in_val(x, ((int64_t)pos[pi] * F + f) * C + c, dtype);
        y[r * C + c] = (xv - mu[g]) / sqrt(var[g] + eps) * in_val(gamma, c, dtype) +
                       in_val(beta, c, dtype);
      }
    }
  }
  free(clip_mean);
  free(clip_ss);
  free(mu);
  free(var);
}
