/*
 * Seeded synthetic inputs for the NVFP4 attention path.
 *
 * This module only draws numbers. It holds none of the attention or
 * quantisation arithmetic; the CPU oracle and the CUDA path both take its
 * output as plain bf16 arrays.
 *
 * Generator: counter based, so every element can be drawn independently and in
 * parallel, with a result that does not depend on the thread count.
 *   splitmix64 (Steele, Lea, Flood, "Fast splittable pseudorandom number
 *   generators", OOPSLA 2014) mixes a 64-bit counter;
 *   uniform  u = ((h >> 11) + 0.5) * 2^-53, in (0, 1);
 *   normal   Box-Muller: sqrt(-2 ln u1) * cos(2 pi u2) with u1, u2 drawn at
 *            counters 2i and 2i+1 of the element's stream;
 *   Student-t(nu) = Z / sqrt(chi2_nu / nu), chi2_nu = sum of nu squared normals.
 * Every value is rounded to bf16 with round-to-nearest-even.
 *
 * Tensor layout: [B][Hx][N][D] row-major (Hx = H for Q, Hkv for K and V).
 * Workload recipes (cfg):
 *   1 gaussian      Q, K, V ~ N(0,1)
 *   2 heavy-tailed  Q, V ~ N(0,1); K = g_c * z + t3, g_c = 20 on round(0.02 D)
 *                   seeded channels per head (else 1), t3 Student-t(3) noise
 *   3 LLM prefill   Q, K ~ t4 / sqrt(2) (unit variance); V ~ N(0,1)
 *   4 video DiT     Q = F + 0.5 z, K = F + 0.5 z' over a T x Y x X latent grid,
 *                   F = sum_{k<3} A sin(2 pi (ft t/T + fy y/Y + fx x/X) + phi),
 *                   f in {0..3}^3 not all zero, phi ~ U[0, 2 pi), A = sqrt(2/3)
 *                   so that F has unit variance; one field per (b, h, channel),
 *                   shared by Q and K; V ~ N(0,1)
 *   5 long context  Q, K, V ~ N(0,1) with round(0.01 N) seeded token positions
 *                   (shared by Q, K, V and all heads) multiplied by 10
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#ifdef _OPENMP
#include <omp.h>
#endif

static inline uint64_t splitmix64(uint64_t x) {
  uint64_t z = x + 0x9E3779B97F4A7C15ULL;
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
  return z ^ (z >> 31);
}

/* Key of an independent stream (a tensor, a parameter set) under a seed. */
static inline uint64_t stream_key(uint64_t seed, uint64_t stream) {
  return splitmix64(seed ^ splitmix64(stream * 0xD1B54A32D192ED03ULL + 0x5EED));
}

static inline double u01(uint64_t key, uint64_t ctr) {
  uint64_t h = splitmix64(key ^ splitmix64(ctr));
  return ((double)(h >> 11) + 0.5) * (1.0 / 9007199254740992.0);
}

static inline double normal_at(uint64_t key, uint64_t i) {
  double u1 = u01(key, 2 * i), u2 = u01(key, 2 * i + 1);
  return sqrt(-2.0 * log(u1)) * cos(6.283185307179586476925 * u2);
}

static inline double student_t_at(uint64_t key, int nu, uint64_t i) {
  uint64_t base = i * (uint64_t)(nu + 1);
  double z = normal_at(key, base), chi2 = 0.0;
  for (int k = 1; k <= nu; ++k) {
    double g = normal_at(key, base + k);
    chi2 += g * g;
  }
  return z / sqrt(chi2 / nu);
}

static inline uint16_t f32_to_bf16_rne(float f) {
  uint32_t u;
  memcpy(&u, &f, 4);
  if ((u & 0x7FFFFFFFu) > 0x7F800000u) return (uint16_t)((u >> 16) | 0x40);
  u += 0x7FFFu + ((u >> 16) & 1u);
  return (uint16_t)(u >> 16);
}

static void set_threads(int nthreads) {
#ifdef _OPENMP
  if (nthreads > 0) omp_set_num_threads(nthreads);
#else
  (void)nthreads;
#endif
}

/* n i.i.d. N(0, scale^2) values of one stream, as bf16. */
void synth_normal_bf16(uint64_t seed, uint64_t stream, int64_t n, float scale,
                       uint16_t* out, int nthreads) {
  set_threads(nthreads);
  uint64_t key = stream_key(seed, stream);
#pragma omp parallel for schedule(static)
  for (int64_t i = 0; i < n; ++i)
    out[i] = f32_to_bf16_rne((float)(scale * normal_at(key, (uint64_t)i)));
}

/* Uniform integers in [0, m) from one stream (row sampling, channel picks). */
void synth_uniform_int(uint64_t seed, uint64_t stream, int64_t n, int64_t m,
                       int64_t* out) {
  uint64_t key = stream_key(seed, stream);
  for (int64_t i = 0; i < n; ++i) {
    int64_t v = (int64_t)(u01(key, (uint64_t)i) * (double)m);
    out[i] = v < m ? v : m - 1;
  }
}

/* k distinct integers of [0, m), in increasing order (partial Fisher-Yates). */
void synth_distinct(uint64_t seed, uint64_t stream, int64_t k, int64_t m,
                    int64_t* out) {
  int64_t* perm = (int64_t*)malloc((size_t)m * sizeof(int64_t));
  uint64_t key = stream_key(seed, stream);
  for (int64_t i = 0; i < m; ++i) perm[i] = i;
  for (int64_t i = 0; i < k; ++i) {
    int64_t j = i + (int64_t)(u01(key, (uint64_t)i) * (double)(m - i));
    if (j >= m) j = m - 1;
    int64_t t = perm[i]; perm[i] = perm[j]; perm[j] = t;
  }
  for (int64_t i = 0; i < k; ++i) out[i] = perm[i];
  free(perm);
  for (int64_t i = 1; i < k; ++i)  /* insertion sort: k is small */
    for (int64_t j = i; j > 0 && out[j - 1] > out[j]; --j) {
      int64_t t = out[j]; out[j] = out[j - 1]; out[j - 1] = t;
    }
}

enum { STREAM_Q = 1, STREAM_K = 2, STREAM_V = 3, STREAM_CHAN = 16,
       STREAM_FIELD = 17, STREAM_TOKENS = 18 };

/*
 * One tensor (which: 0 = Q, 1 = K, 2 = V) of workload cfg, shape
 * [B][Hx][N][D], written as bf16 to out. grid = {T, Y, X} for cfg 4 (must
 * multiply to N), ignored otherwise. Returns 0, or -1 on bad arguments.
 */
int synth_config_tensor(int cfg, int which, int B, int Hx, int N, int D,
                        const int* grid, uint64_t seed, uint16_t* out,
                        int nthreads) {
  if (B <= 0 || Hx <= 0 || N <= 0 || D <= 0 || which < 0 || which > 2) return -1;
  set_threads(nthreads);
  const int64_t per_head = (int64_t)N * D;
  const int64_t total = (int64_t)B * Hx * per_head;
  const uint64_t key = stream_key(seed, (uint64_t)(STREAM_Q + which));

  if (cfg == 1 || (cfg == 2 && which != 1) || (cfg == 3 && which == 2) ||
      (cfg == 4 && which == 2)) {
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < total; ++i)
      out[i] = f32_to_bf16_rne((float)normal_at(key, (uint64_t)i));
    return 0;
  }
  if (cfg == 2) {  /* K: outlier channels plus Student-t(3) noise */
    int nout = (int)lround(0.02 * D);
    if (nout < 1) nout = 1;
    int64_t* chans = (int64_t*)malloc(sizeof(int64_t) * (size_t)B * Hx * nout);
    for (int64_t g = 0; g < (int64_t)B * Hx; ++g)
      synth_distinct(seed, STREAM_CHAN * 1000003ULL + (uint64_t)g, nout, D,
                     chans + g * nout);
    const uint64_t tkey = stream_key(seed, STREAM_K * 7919ULL + 3);
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < total; ++i) {
      int64_t g = i / per_head;
      int d = (int)(i % D);
      double gain = 1.0;
      for (int c = 0; c < nout; ++c)
        if (chans[g * nout + c] == d) gain = 20.0;
      double z = normal_at(key, (uint64_t)i);
      out[i] = f32_to_bf16_rne((float)(gain * z + student_t_at(tkey, 3, (uint64_t)i)));
    }
    free(chans);
    return 0;
  }
  if (cfg == 3) {  /* Q, K: Student-t(4) / sqrt(2) */
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < total; ++i)
      out[i] = f32_to_bf16_rne((float)(student_t_at(key, 4, (uint64_t)i) *
                                       0.70710678118654752440));
    return 0;
  }
  if (cfg == 4) {  /* Q, K: shared smooth field + 0.5 N(0,1) */
    if (!grid || (int64_t)grid[0] * grid[1] * grid[2] != N) return -1;
    const int T = grid[0], Y = grid[1], X = grid[2];
    const int64_t nfield = (int64_t)B * Hx * D;
    /* per (b, h, d): 3 sinusoids x (ft, fy, fx, phi) */
    double* par = (double*)malloc(sizeof(double) * (size_t)nfield * 12);
    const uint64_t fkey = stream_key(seed, STREAM_FIELD);
    for (int64_t f = 0; f < nfield; ++f)
      for (int s = 0; s < 3; ++s) {
        uint64_t ctr = (uint64_t)(f * 3 + s) * 64;
        int ft, fy, fx;
        do {  /* redraw until the frequency vector is not all zero */
          ft = (int)(u01(fkey, ctr++) * 4.0);
          fy = (int)(u01(fkey, ctr++) * 4.0);
          fx = (int)(u01(fkey, ctr++) * 4.0);
        } while (ft == 0 && fy == 0 && fx == 0);
        double* p = par + (f * 3 + s) * 4;
        p[0] = ft; p[1] = fy; p[2] = fx;
        p[3] = 6.283185307179586476925 * u01(fkey, ctr);
      }
    const double A = sqrt(2.0 / 3.0);
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < total; ++i) {
      int64_t g = i / per_head;
      int64_t n = (i / D) % N;
      int d = (int)(i % D);
      int t = (int)(n / ((int64_t)Y * X)), y = (int)((n / X) % Y), x = (int)(n % X);
      const double* p = par + ((g * D + d) * 3) * 4;
      double F = 0.0;
      for (int s = 0; s < 3; ++s, p += 4)
        F += A * sin(6.283185307179586476925 *
                         (p[0] * t / T + p[1] * y / Y + p[2] * x / X) + p[3]);
      out[i] = f32_to_bf16_rne((float)(F + 0.5 * normal_at(key, (uint64_t)i)));
    }
    free(par);
    return 0;
  }
  if (cfg == 5) {  /* N(0,1) with 1% outlier tokens x10 */
    int64_t nout = (int64_t)llround(0.01 * N);
    unsigned char* hot = (unsigned char*)calloc((size_t)N, 1);
    if (nout > 0) {
      int64_t* pos = (int64_t*)malloc(sizeof(int64_t) * (size_t)nout);
      synth_distinct(seed, STREAM_TOKENS, nout, N, pos);
      for (int64_t k = 0; k < nout; ++k) hot[pos[k]] = 1;
      free(pos);
    }
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < total; ++i) {
      int64_t n = (i / D) % N;
      double z = normal_at(key, (uint64_t)i);
      out[i] = f32_to_bf16_rne((float)(hot[n] ? 10.0 * z : z));
    }
    free(hot);
    return 0;
  }
  return -1;
}

/* The outlier token positions of cfg 5 (k = round(0.01 N) of them). */
int64_t synth_outlier_tokens(uint64_t seed, int N, int64_t* out) {
  int64_t nout = (int64_t)llround(0.01 * N);
  if (nout > 0) synth_distinct(seed, STREAM_TOKENS, nout, N, out);
  return nout;
}
