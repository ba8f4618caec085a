/*
 * Seeded synthetic inputs for the routed W4A16 / block-FP8 MoE layer.
 *
 * This file is the ONE input generator that both the CPU oracle (oracle/) and the
 * CUDA path are fed from.  It holds no arithmetic of the layer itself: it only
 * turns (seed, tensor id, flat element index) into numbers with the value
 * distributions of the workloads (signed INT4 nibbles, bf16 N(0,1) activations,
 * fp32 N(0,1) router logits with an optional Zipf-shaped per-expert bias, bf16
 * group scales U[lo,hi], e4m3 weights and activations with fp32 block scales).
 *
 * Counter-based: element i of tensor `tid` under `seed` is a pure function of
 * (seed, tid, i), so any slice (one expert, one token) can be regenerated alone
 * and large tensors are filled in parallel.  The bit generator is the output
 * function of SplitMix64 (G. Steele, D. Lea, C. Flood, "Fast splittable
 * pseudorandom number generators", OOPSLA 2014) applied to the Weyl sequence
 * key + (i+1)*gamma, where key is itself a SplitMix64 mix of (seed, tid).
 * Normals use the Box-Muller transform (G. Box, M. Muller, 1958), cosine branch.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define GOLDEN 0x9E3779B97F4A7C15ULL

static inline uint64_t mix64(uint64_t z) {
  z ^= z >> 30;
  z *= 0xBF58476D1CE4E5B9ULL;
  z ^= z >> 27;
  z *= 0x94D049BB133111EBULL;
  z ^= z >> 31;
  return z;
}

uint64_t synth_key(uint64_t seed, uint64_t tid) {
  return mix64(seed * GOLDEN + mix64(tid + 0x632BE59BD9B4E019ULL));
}

static inline uint64_t draw(uint64_t key, uint64_t i) { return mix64(key + (i + 1) * GOLDEN); }

uint64_t synth_draw(uint64_t seed, uint64_t tid, uint64_t i) { return draw(synth_key(seed, tid), i); }

/* [0,1) from the top 24 bits. */
static inline double unif24(uint64_t d) { return (double)(d >> 40) * (1.0 / 16777216.0); }

static inline double normal_bm(uint64_t d) {
  double u1 = ((double)(d >> 40) + 0.5) * (1.0 / 16777216.0); /* (0,1) */
  double u2 = (double)((d >> 16) & 0xFFFFFFu) * (1.0 / 16777216.0);
  return sqrt(-2.0 * log(u1)) * cos(6.283185307179586476925286766559 * u2);
}

static inline uint32_t f32_bits(float f) {
  uint32_t u;
  memcpy(&u, &f, 4);
  return u;
}

/* float -> bf16, round to nearest even (inputs here are always finite). */
static inline uint16_t bf16_rne(float f) {
  uint32_t u = f32_bits(f);
  u += 0x7FFFu + ((u >> 16) & 1u);
  return (uint16_t)(u >> 16);
}

static inline float bf16_to_f32(uint16_t h) {
  uint32_t u = (uint32_t)h << 16;
  float f;
  memcpy(&f, &u, 4);
  return f;
}

/* float -> OCP E4M3FN (bias 7, no infinities, max 448), round to nearest even,
   saturating finite values to +-448. */
static uint8_t e4m3_rne_sat(float xf) {
  double x = (double)xf;
  if (x != x) return 0x7F;
  uint8_t sign = 0;
  if (x < 0) {
    sign = 0x80;
    x = -x;
  }
  if (x >= 448.0) return sign | 0x7E;
  if (x < 0.015625) { /* below 2^-6: subnormal grid of 2^-9 */
    double m = nearbyint(x * 512.0);
    return sign | (uint8_t)m; /* m==8 is exactly the smallest normal, code 0x08 */
  }
  int ex;
  double f = frexp(x, &ex); /* x = f * 2^ex, f in [0.5,1) */
  int e = ex - 1;           /* x = (2f) * 2^e, 2f in [1,2) */
  double m = nearbyint((2.0 * f - 1.0) * 8.0);
  if (m >= 8.0) {
    m = 0.0;
    e += 1;
  }
  int code = ((e + 7) << 3) | (int)m;
  if (code > 0x7E) code = 0x7E;
  return sign | (uint8_t)code;
}

/* ---------------------------------------------------------------- parallel-for */
typedef void (*range_fn)(void* ctx, uint64_t lo, uint64_t hi);
typedef struct {
  range_fn fn;
  void* ctx;
  uint64_t lo, hi;
} job_t;
static void* job_run(void* a) {
  job_t* j = (job_t*)a;
  j->fn(j->ctx, j->lo, j->hi);
  return NULL;
}
static void parallel_for(range_fn fn, void* ctx, uint64_t n, int nthreads) {
  if (nthreads < 1) nthreads = 1;
  if (nthreads > 256) nthreads = 256;
  if (n < (1u << 16) || nthreads == 1) {
    fn(ctx, 0, n);
    return;
  }
  pthread_t th[256];
  job_t jobs[256];
  uint64_t per = (n + nthreads - 1) / nthreads;
  int used = 0;
  for (int t = 0; t < nthreads; ++t) {
    uint64_t lo = per * t, hi = lo + per < n ? lo + per : n;
    if (lo >= hi) break;
    jobs[t] = (job_t){fn, ctx, lo, hi};
    pthread_create(&th[t], NULL, job_run, &jobs[t]);
    used++;
  }
  for (int t = 0; t < used; ++t) pthread_join(th[t], NULL);
}

/* ---------------------------------------------------------------- fills */
typedef struct {
  uint64_t key, start;
  void* out;
  double lo, hi;
} fill_ctx;

static void k_u32(void* c, uint64_t a, uint64_t b) {
  fill_ctx* x = (fill_ctx*)c;
  uint32_t* o = (uint32_t*)x->out;
  for (uint64_t i = a; i < b; ++i) o[i] = (uint32_t)draw(x->key, x->start + i);
}
/* Raw 32-bit words: eight independent uniform signed INT4 nibbles in [-8,7] each. */
void synth_u32(uint64_t seed, uint64_t tid, uint64_t start, uint64_t n, uint32_t* out, int nthreads) {
  fill_ctx c = {synth_key(seed, tid), start, out, 0, 0};
  parallel_for(k_u32, &c, n, nthreads);
}

static void k_unif_bf16(void* c, uint64_t a, uint64_t b) {
  fill_ctx* x = (fill_ctx*)c;
  uint16_t* o = (uint16_t*)x->out;
  for (uint64_t i = a; i < b; ++i) {
    double u = unif24(draw(x->key, x->start + i));
    o[i] = bf16_rne((float)(x->lo + (x->hi - x->lo) * u));
  }
}
/* bf16(U[lo,hi]): the fp64 value lo+(hi-lo)*u rounded to fp32, then to bf16 (RNE). */
void synth_uniform_bf16(uint64_t seed, uint64_t tid, uint64_t start, uint64_t n, double lo, double hi,
                        uint16_t* out, int nthreads) {
  fill_ctx c = {synth_key(seed, tid), start, out, lo, hi};
  parallel_for(k_unif_bf16, &c, n, nthreads);
}

static void k_unif_f32(void* c, uint64_t a, uint64_t b) {
  fill_ctx* x = (fill_ctx*)c;
  float* o = (float*)x->out;
  for (uint64_t i = a; i < b; ++i) {
    double u = unif24(draw(x->key, x->start + i));
    o[i] = (float)(x->lo + (x->hi - x->lo) * u);
  }
}
void synth_uniform_f32(uint64_t seed, uint64_t tid, uint64_t start, uint64_t n, double lo, double hi,
                       float* out, int nthreads) {
  fill_ctx c = {synth_key(seed, tid), start, out, lo, hi};
  parallel_for(k_unif_f32, &c, n, nthreads);
}

static void k_norm_bf16(void* c, uint64_t a, uint64_t b) {
  fill_ctx* x = (fill_ctx*)c;
  uint16_t* o = (uint16_t*)x->out;
  for (uint64_t i = a; i < b; ++i) o[i] = bf16_rne((float)normal_bm(draw(x->key, x->start + i)));
}
/* bf16(N(0,1)). */
void synth_normal_bf16(uint64_t seed, uint64_t tid, uint64_t start, uint64_t n, uint16_t* out, int nthreads) {
  fill_ctx c = {synth_key(seed, tid), start, out, 0, 0};
  parallel_for(k_norm_bf16, &c, n, nthreads);
}

static void k_norm_f32(void* c, uint64_t a, uint64_t b) {
  fill_ctx* x = (fill_ctx*)c;
  float* o = (float*)x->out;
  for (uint64_t i = a; i < b; ++i) o[i] = (float)normal_bm(draw(x->key, x->start + i));
}
void synth_normal_f32(uint64_t seed, uint64_t tid, uint64_t start, uint64_t n, float* out, int nthreads) {
  fill_ctx c = {synth_key(seed, tid), start, out, 0, 0};
  parallel_for(k_norm_f32, &c, n, nthreads);
}

static void k_norm_e4m3(void* c, uint64_t a, uint64_t b) {
  fill_ctx* x = (fill_ctx*)c;
  uint8_t* o = (uint8_t*)x->out;
  for (uint64_t i = a; i < b; ++i) o[i] = e4m3_rne_sat((float)normal_bm(draw(x->key, x->start + i)));
}
/* e4m3(N(0,1)) with saturation at +-448 (the N(0,1)-clipped e4m3 weights). */
void synth_normal_e4m3(uint64_t seed, uint64_t tid, uint64_t start, uint64_t n, uint8_t* out, int nthreads) {
  fill_ctx c = {synth_key(seed, tid), start, out, 0, 0};
  parallel_for(k_norm_e4m3, &c, n, nthreads);
}

/* Router logits [T,E] fp32: N(0,1) plus an optional per-expert bias
   b_e = -s * ln(r_e), where r is a seeded permutation of the ranks 1..E
   (so that softmax(b) alone is Zipf(s)-shaped over the experts).  zipf_s <= 0: no bias. */
typedef struct {
  uint64_t key;
  uint64_t t0;
  int E;
  const double* bias;
  float* out;
} logit_ctx;
static void k_logits(void* c, uint64_t a, uint64_t b) {
  logit_ctx* x = (logit_ctx*)c;
  for (uint64_t i = a; i < b; ++i) {
    uint64_t gi = x->t0 * (uint64_t)x->E + i;
    double z = normal_bm(draw(x->key, gi));
    if (x->bias) z += x->bias[i % (uint64_t)x->E];
    x->out[i] = (float)z;
  }
}
void synth_zipf_bias(uint64_t seed, uint64_t tid_perm, int E, double s, double* bias_out) {
  int* rank = (int*)malloc(sizeof(int) * (size_t)E);
  for (int i = 0; i < E; ++i) rank[i] = i + 1;
  uint64_t key = synth_key(seed, tid_perm);
  for (int i = E - 1; i >= 1; --i) { /* Fisher-Yates */
    int j = (int)(draw(key, (uint64_t)i) % (uint64_t)(i + 1));
    int t = rank[i];
    rank[i] = rank[j];
    rank[j] = t;
  }
  for (int e = 0; e < E; ++e) bias_out[e] = -s * log((double)rank[e]);
  free(rank);
}
void synth_logits(uint64_t seed, uint64_t tid, uint64_t tid_perm, uint64_t t0, uint64_t T, int E, double zipf_s,
                  float* out, int nthreads) {
  double* bias = NULL;
  if (zipf_s > 0) {
    bias = (double*)malloc(sizeof(double) * (size_t)E);
    synth_zipf_bias(seed, tid_perm, E, zipf_s, bias);
  }
  logit_ctx c = {synth_key(seed, tid), t0, E, bias, out};
  parallel_for(k_logits, &c, T * (uint64_t)E, nthreads);
  free(bias);
}

/* Block-FP8 activations for rows [t0, t0+T) of a [*, H] tensor: z = bf16(N(0,1)); per
   (row, 128-column group) s = max(amax|z|, 1e-10) / 448 (fp32), q = e4m3(z / s) (fp32
   division, RNE, saturating).  q: [T,H] bytes, s: [T,H/128] fp32. */
typedef struct {
  uint64_t key, t0;
  int H;
  uint8_t* q;
  float* s;
} act8_ctx;
static void k_act8(void* c, uint64_t a, uint64_t b) {
  act8_ctx* x = (act8_ctx*)c;
  int G = x->H / 128;
  float z[128];
  for (uint64_t rg = a; rg < b; ++rg) {
    uint64_t r = rg / (uint64_t)G, g = rg % (uint64_t)G;
    float amax = 0.f;
    for (int i = 0; i < 128; ++i) {
      uint64_t gi = (x->t0 + r) * (uint64_t)x->H + g * 128 + (uint64_t)i;
      z[i] = bf16_to_f32(bf16_rne((float)normal_bm(draw(x->key, gi))));
      float m = fabsf(z[i]);
      if (m > amax) amax = m;
    }
    float sc = (amax > 1e-10f ? amax : 1e-10f) / 448.0f;
    x->s[r * (uint64_t)G + g] = sc;
    for (int i = 0; i < 128; ++i) x->q[r * (uint64_t)x->H + g * 128 + (uint64_t)i] = e4m3_rne_sat(z[i] / sc);
  }
}
void synth_act_e4m3(uint64_t seed, uint64_t tid, uint64_t t0, uint64_t T, int H, uint8_t* q, float* s,
                    int nthreads) {
  act8_ctx c = {synth_key(seed, tid), t0, H, q, s};
  parallel_for(k_act8, &c, T * (uint64_t)(H / 128), nthreads);
}
