/*
 * CPU ORACLE for the routed, weight-quantized Mixture-of-Experts layer.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may link, load or call this
 * file: only the tests, the package's smoke check and the benchmark's CPU-baseline leg
 * use it.  It shares no code with the CUDA path (its own bf16/fp16/e4m3/e2m1/e8m0/INT4 decoders,
 * its own routing, sort, GEMM, activation and combine).
 *
 * What it computes is the plain definition of the layer, written out one token at a time
 * (threads only split the token list), with every dot product accumulated in fp64 in
 * ascending K order and no intermediate rounding except where the method itself rounds
 * (the FP8 quantization of the activations in the block-FP8 and W4A8 layers, below).
 *
 * Sources (titles of the pages the method is described on):
 *  - "Chord Rewrites the INT4 MoE Kernel for Kimi K2.x ..." (Chord article), second
 *    paragraph: W4A16 = BF16 inputs, INT4 weights, one BF16 scale per group of 32 weights;
 *    routing shapes of gate, up and down projections; per-expert token counts.
 *  - "Helion Brings Autotuned GEMM Kernels to vLLM ..." (Helion article), section
 *    "Scope: Hopper and quantized formats": Block_FP8 = FP8 with 1x128 activation scaling
 *    and 128x128 weight scaling.
 *  - "[Performance] W4A8 MoE GEMM significantly slower than W4A16 on H200" (Humming issue),
 *    the opening report: W4A8 = MXFP4 weights with FP8 activations quantized in K groups.
 *  - "AWS Details H200 Kernel Optimizations for MoE Inference", section "Three bottlenecks
 *    require different fixes": a fused MoE operator = token routing, data movement and
 *    expert calculations.
 *  The pages print no formula for the router, the activation or the combine; the readings
 *  taken (softmax over the logits, top-k by logit with lower index winning ties, weights
 *  renormalised over the k winners, SiLU(gate)*up with gate = the first I output columns
 *  of w13, fp32 weighted sum in slot order) are the textbook ones and are listed with the
 *  design notes.
 *
 * Parity pins: every function here is pinned by tests/test_oracle_*.py against values
 * fixed independently of this file (hand-packed words, closed forms, a dense
 * every-expert-then-mask formulation, float64 torch matmul on dequantized weights,
 * brute-force sorting, invariants).
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* ------------------------------------------------------------------ number formats */

/* bf16 bit pattern -> value: the top 16 bits of an IEEE binary32. */
double oracle_bf16(uint16_t h) {
  uint32_t u = (uint32_t)h << 16;
  float f;
  memcpy(&f, &u, 4);
  return (double)f;
}

/* IEEE binary16 bit pattern -> value (1 sign, 5 exponent bits bias 15, 10 fraction bits). */
double oracle_f16(uint16_t h) {
  int s = (h >> 15) & 1, e = (h >> 10) & 31, f = h & 1023;
  double v;
  if (e == 0)
    v = ldexp((double)f, -24); /* subnormal: f * 2^-14 / 2^10 */
  else if (e == 31)
    v = f ? NAN : INFINITY;
  else
    v = ldexp(1.0 + f / 1024.0, e - 15);
  return s ? -v : v;
}

/* Signed INT4 nibble j (bits 4j..4j+3) of a packed word, two's complement in [-8, 7]. */
int oracle_int4(uint32_t word, int j) {
  int n = (int)((word >> (4 * j)) & 0xFu);
  return n >= 8 ? n - 16 : n;
}

/* OCP E4M3FN byte -> value: bias 7, 3 mantissa bits, no infinities, S.1111.111 = NaN. */
double oracle_e4m3(uint8_t b) {
  int s = b >> 7, e = (b >> 3) & 15, m = b & 7;
  double v;
  if (e == 15 && m == 7)
    v = NAN;
  else if (e == 0)
    v = ldexp((double)m / 8.0, -6);
  else
    v = ldexp(1.0 + m / 8.0, e - 7);
  return s ? -v : v;
}

/* value -> E4M3FN, round to nearest with ties to the even code, finite values saturate to
   +-448.  Written as a search over all 127 non-negative finite codes so it depends on
   nothing but the decoder above. */
uint8_t oracle_e4m3_encode(float xf) {
  double x = (double)xf;
  if (x != x) return 0x7F;
  uint8_t sign = (x < 0 || (x == 0 && signbit(x))) ? 0x80 : 0;
  double a = fabs(x);
  if (a >= 448.0) return sign | 0x7E;
  int best = 0;
  double bestd = a;
  for (int c = 1; c <= 0x7E; ++c) {
    double d = fabs(oracle_e4m3((uint8_t)c) - a);
    if (d < bestd || (d == bestd && (c & 1) == 0 && (best & 1) == 1)) {
      best = c;
      bestd = d;
    }
  }
  return sign | (uint8_t)best;
}

/* SiLU(g) = g * sigmoid(g) = g / (1 + e^-g). */
double oracle_silu(double g) { return g / (1.0 + exp(-g)); }

/* ------------------------------------------------------------------ routing */

/* Top-k of each row of logits [T,E] by (logit descending, expert index ascending);
   softmax p_e = exp(l_e - max) / sum_e' exp(l_e' - max) over all E experts;
   weight of slot s = p_{id_s} / sum_{s'} p_{id_s'} if renormalize, else p_{id_s}.
   Slot order is rank order.  Weights are returned in fp64 (w64) and rounded to fp32 (w32);
   either may be NULL. */
void oracle_route(const float* logits, int T, int E, int k, int renormalize, int32_t* ids, float* w32,
                  double* w64) {
  char* taken = (char*)malloc((size_t)E);
  double* p = (double*)malloc(sizeof(double) * (size_t)E);
  for (int t = 0; t < T; ++t) {
    const float* l = logits + (size_t)t * E;
    memset(taken, 0, (size_t)E);
    for (int s = 0; s < k; ++s) {
      int best = -1;
      for (int e = 0; e < E; ++e) {
        if (taken[e]) continue;
        if (best < 0 || l[e] > l[best]) best = e; /* strict '>' keeps the lower index on ties */
      }
      taken[best] = 1;
      ids[(size_t)t * k + s] = best;
    }
    double mx = -INFINITY;
    for (int e = 0; e < E; ++e)
      if ((double)l[e] > mx) mx = (double)l[e];
    double Z = 0.0;
    for (int e = 0; e < E; ++e) {
      p[e] = exp((double)l[e] - mx);
      Z += p[e];
    }
    for (int e = 0; e < E; ++e) p[e] /= Z;
    double S = 0.0;
    for (int s = 0; s < k; ++s) S += p[ids[(size_t)t * k + s]];
    for (int s = 0; s < k; ++s) {
      double w = p[ids[(size_t)t * k + s]];
      if (renormalize) w /= S;
      if (w64) w64[(size_t)t * k + s] = w;
      if (w32) w32[(size_t)t * k + s] = (float)w;
    }
  }
  free(taken);
  free(p);
}

/* ------------------------------------------------------------------ alignment */

/* Token-to-expert permutation.  Pairs p = t*k + s (T*k of them) are sorted by
   (expert ascending, p ascending).  Each expert's run is padded to a multiple of `align`
   with the sentinel T*k.  counts[e] = number of pairs routed to e; offsets[0] = 0,
   offsets[e+1] = offsets[e] + ceil(counts[e]/align)*align; sorted_ids[offsets[e] + r] is
   the r-th pair of expert e; inv_pos[p] = the row of pair p in sorted_ids.
   Returns the number of out-of-range ids found (those pairs are left out). */
int oracle_align(const int32_t* ids, int T, int k, int E, int align, int32_t* counts, int32_t* offsets,
                 int32_t* sorted_ids, int32_t* inv_pos) {
  int P = T * k, bad = 0;
  for (int e = 0; e < E; ++e) counts[e] = 0;
  for (int p = 0; p < P; ++p) {
    if (ids[p] < 0 || ids[p] >= E) {
      bad++;
      inv_pos[p] = -1;
      continue;
    }
    counts[ids[p]]++;
  }
  offsets[0] = 0;
  for (int e = 0; e < E; ++e) offsets[e + 1] = offsets[e] + (counts[e] + align - 1) / align * align;
  for (int e = 0; e < E; ++e) {
    int r = 0;
    for (int p = 0; p < P; ++p) /* ascending p: stable */
      if (ids[p] == e) {
        sorted_ids[offsets[e] + r] = p;
        inv_pos[p] = offsets[e] + r;
        r++;
      }
    for (; r < offsets[e + 1] - offsets[e]; ++r) sorted_ids[offsets[e] + r] = P;
  }
  return bad;
}

/* ------------------------------------------------------------------ W4A16 layer */

/* Dequantized W4A16 weight: element (n, kk) of one expert's [N, K] matrix stored as
   q [N, K/8] int32 (nibble j of word w = K index 8w+j) and s [N, K/32] bf16:
   W[n][kk] = int4(q[n][kk/8], kk%8) * bf16(s[n][kk/32]). */
static inline double w4(const int32_t* q, const uint16_t* s, int K, int n, int kk) {
  uint32_t word = (uint32_t)q[(size_t)n * (K / 8) + kk / 8];
  return (double)oracle_int4(word, kk % 8) * oracle_bf16(s[(size_t)n * (K / 32) + kk / 32]);
}

typedef struct {
  const uint16_t* x;
  const int32_t* ids;
  const float* w;
  int T, H, I, E, k;
  const int32_t *w13_q, *w2_q;
  const uint16_t *w13_s, *w2_s;
  const int32_t* tokens;
  int n_tok;
  double* out;   /* [n_tok, H] */
  double* h_out; /* [n_tok, k, I] or NULL */
  double* g_out; /* [n_tok, k, 2I] or NULL */
  int next;
  pthread_mutex_t mu;
} w4_job;

static void w4_token(w4_job* J, int i) {
  int t = J->tokens[i], H = J->H, I = J->I, k = J->k;
  double* xr = (double*)malloc(sizeof(double) * (size_t)H);
  double* g = (double*)malloc(sizeof(double) * 2 * (size_t)I);
  double* h = (double*)malloc(sizeof(double) * (size_t)I);
  double* o = J->out + (size_t)i * H;
  for (int c = 0; c < H; ++c) {
    xr[c] = oracle_bf16(J->x[(size_t)t * H + c]);
    o[c] = 0.0;
  }
  for (int s = 0; s < k; ++s) {
    int e = J->ids[(size_t)t * k + s];
    double ws = (double)J->w[(size_t)t * k + s];
    const int32_t* q13 = J->w13_q + (size_t)e * 2 * I * (H / 8);
    const uint16_t* s13 = J->w13_s + (size_t)e * 2 * I * (H / 32);
    const int32_t* q2 = J->w2_q + (size_t)e * H * (I / 8);
    const uint16_t* s2 = J->w2_s + (size_t)e * H * (I / 32);
    /* gate/up projection: g[n] = sum_c x[c] * W13[n][c], n in [0, 2I) */
    for (int n = 0; n < 2 * I; ++n) {
      double acc = 0.0;
      for (int c = 0; c < H; ++c) acc += xr[c] * w4(q13, s13, H, n, c);
      g[n] = acc;
    }
    if (J->g_out) memcpy(J->g_out + ((size_t)i * k + s) * 2 * I, g, sizeof(double) * 2 * I);
    /* h[j] = SiLU(gate_j) * up_j with gate = columns [0,I), up = columns [I,2I) */
    for (int j = 0; j < I; ++j) h[j] = oracle_silu(g[j]) * g[I + j];
    if (J->h_out) memcpy(J->h_out + ((size_t)i * k + s) * I, h, sizeof(double) * I);
    /* down projection and weighted combine: out[c] += w_s * sum_j h[j] * W2[c][j] */
    for (int c = 0; c < H; ++c) {
      double acc = 0.0;
      for (int j = 0; j < I; ++j) acc += h[j] * w4(q2, s2, I, c, j);
      o[c] += ws * acc;
    }
  }
  free(xr);
  free(g);
  free(h);
}

static void* w4_worker(void* a) {
  w4_job* J = (w4_job*)a;
  for (;;) {
    pthread_mutex_lock(&J->mu);
    int i = J->next++;
    pthread_mutex_unlock(&J->mu);
    if (i >= J->n_tok) break;
    w4_token(J, i);
  }
  return NULL;
}

static void run_pool(void* (*fn)(void*), void* job, int nthreads) {
  if (nthreads < 1) nthreads = 1;
  if (nthreads > 512) nthreads = 512;
  pthread_t th[512];
  for (int i = 0; i < nthreads; ++i) pthread_create(&th[i], NULL, fn, job);
  for (int i = 0; i < nthreads; ++i) pthread_join(th[i], NULL);
}

/* Routed W4A16 MoE layer output (fp64) for the listed tokens:
   out[i][c] = sum_s w[t][s] * sum_j h_s[j] * W2[e_s][c][j],
   h_s[j]    = SiLU(g_s[j]) * g_s[I+j],  g_s[n] = sum_c x[t][c] * W13[e_s][n][c],
   with t = tokens[i], e_s = ids[t][s].  x bf16 [T,H]; ids int32 [T,k]; w fp32 [T,k];
   w13_q int32 [E,2I,H/8]; w13_s bf16 [E,2I,H/32]; w2_q int32 [E,H,I/8]; w2_s bf16 [E,H,I/32].
   h_out ([n_tok,k,I]) and g_out ([n_tok,k,2I]) optionally receive the intermediates. */
void oracle_w4a16_tokens(const uint16_t* x, const int32_t* ids, const float* w, int T, int H, int I, int E, int k,
                         const int32_t* w13_q, const uint16_t* w13_s, const int32_t* w2_q, const uint16_t* w2_s,
                         const int32_t* tokens, int n_tok, double* out, double* h_out, double* g_out,
                         int nthreads) {
  w4_job J = {x, ids, w, T, H, I, E, k, w13_q, w2_q, w13_s, w2_s, tokens, n_tok, out, h_out, g_out, 0, PTHREAD_MUTEX_INITIALIZER};
  run_pool(w4_worker, &J, nthreads);
  pthread_mutex_destroy(&J.mu);
}

/* Grouped W4A16 GEMM without activation: rows [expert_offsets[e], expert_offsets[e+1]) of
   a [M,K] (bf16 if a_is_bf16 else fp16 bit patterns) are multiplied by expert e's
   dequantized weights: out[m][n] = sum_c a[m][c] * W[e][n][c], W stored as w_q [E,N,K/8],
   w_s [E,N,K/32].  Rows outside every expert range are set to 0. */
void oracle_w4a16_gemm(const uint16_t* a, int a_is_bf16, const int32_t* w_q, const uint16_t* w_s,
                       const int32_t* expert_offsets, int M, int K, int N, int E, double* out) {
  double* ar = (double*)malloc(sizeof(double) * (size_t)K);
  for (int m = 0; m < M; ++m) {
    int e = -1;
    for (int j = 0; j < E; ++j)
      if (m >= expert_offsets[j] && m < expert_offsets[j + 1]) e = j;
    if (e < 0) {
      for (int n = 0; n < N; ++n) out[(size_t)m * N + n] = 0.0;
      continue;
    }
    for (int c = 0; c < K; ++c) {
      uint16_t b = a[(size_t)m * K + c];
      ar[c] = a_is_bf16 ? oracle_bf16(b) : oracle_f16(b);
    }
    const int32_t* q = w_q + (size_t)e * N * (K / 8);
    const uint16_t* s = w_s + (size_t)e * N * (K / 32);
    for (int n = 0; n < N; ++n) {
      double acc = 0.0;
      for (int c = 0; c < K; ++c) acc += ar[c] * w4(q, s, K, n, c);
      out[(size_t)m * N + n] = acc;
    }
  }
  free(ar);
}

/* ------------------------------------------------------------------ block-FP8 layer */

/* 1x128 activation quantization (the Helion article's Block_FP8 activation scaling),
   applied to the intermediate activation the same way as to the layer input.  All in
   fp32, as the values are held: s = max(amax, 1e-10) / 448, q[j] = e4m3(h[j] / s).
   Returns s. */
float oracle_fp8_requant(const float* h, uint8_t* q) {
  float amax = 0.f;
  for (int j = 0; j < 128; ++j)
    if (fabsf(h[j]) > amax) amax = fabsf(h[j]);
  float sc = (amax > 1e-10f ? amax : 1e-10f) / 448.0f;
  for (int j = 0; j < 128; ++j) q[j] = oracle_e4m3_encode(h[j] / sc);
  return sc;
}

typedef struct {
  const uint8_t* x;
  const float* xs;
  const int32_t* ids;
  const float* w;
  int T, H, I, E, k;
  const uint8_t *w13, *w2;
  const float *w13_s, *w2_s;
  const int32_t* tokens;
  int n_tok;
  double* out;
  float* hq_out; /* [n_tok, k, I] dequantized requantized h, or NULL */
  int next;
  pthread_mutex_t mu;
} f8_job;

static void f8_token(f8_job* J, int i) {
  int t = J->tokens[i], H = J->H, I = J->I, k = J->k;
  int GH = H / 128, GI = I / 128;
  double* xr = (double*)malloc(sizeof(double) * (size_t)H);
  double* g = (double*)malloc(sizeof(double) * 2 * (size_t)I);
  float* hf = (float*)malloc(sizeof(float) * (size_t)I);
  double* hd = (double*)malloc(sizeof(double) * (size_t)I);
  double* o = J->out + (size_t)i * H;
  /* x[c] = e4m3(xq[t][c]) * xs[t][c/128] (1x128 activation scaling) */
  for (int c = 0; c < H; ++c) {
    xr[c] = oracle_e4m3(J->x[(size_t)t * H + c]) * (double)J->xs[(size_t)t * GH + c / 128];
    o[c] = 0.0;
  }
  for (int s = 0; s < k; ++s) {
    int e = J->ids[(size_t)t * k + s];
    double ws = (double)J->w[(size_t)t * k + s];
    const uint8_t* q13 = J->w13 + (size_t)e * 2 * I * H;
    const float* s13 = J->w13_s + (size_t)e * (2 * I / 128) * GH;
    const uint8_t* q2 = J->w2 + (size_t)e * H * I;
    const float* s2 = J->w2_s + (size_t)e * (H / 128) * GI;
    /* W13[n][c] = e4m3(w13[e][n][c]) * w13_s[e][n/128][c/128] (128x128 weight scaling) */
    for (int n = 0; n < 2 * I; ++n) {
      double acc = 0.0;
      for (int c = 0; c < H; ++c)
        acc += xr[c] * (oracle_e4m3(q13[(size_t)n * H + c]) * (double)s13[(size_t)(n / 128) * GH + c / 128]);
      g[n] = acc;
    }
    /* h = SiLU(gate) * up, kept in fp32 as the intermediate activation */
    for (int j = 0; j < I; ++j) hf[j] = (float)(oracle_silu(g[j]) * g[I + j]);
    /* requantize h group by group (1x128), then use the dequantized values */
    for (int gi = 0; gi < GI; ++gi) {
      uint8_t qc[128];
      float sc = oracle_fp8_requant(hf + gi * 128, qc);
      for (int j = 0; j < 128; ++j) hd[gi * 128 + j] = oracle_e4m3(qc[j]) * (double)sc;
    }
    if (J->hq_out)
      for (int j = 0; j < I; ++j) J->hq_out[((size_t)i * k + s) * I + j] = (float)hd[j];
    for (int c = 0; c < H; ++c) {
      double acc = 0.0;
      for (int j = 0; j < I; ++j)
        acc += hd[j] * (oracle_e4m3(q2[(size_t)c * I + j]) * (double)s2[(size_t)(c / 128) * GI + j / 128]);
      o[c] += ws * acc;
    }
  }
  free(xr);
  free(g);
  free(hf);
  free(hd);
}

static void* f8_worker(void* a) {
  f8_job* J = (f8_job*)a;
  for (;;) {
    pthread_mutex_lock(&J->mu);
    int i = J->next++;
    pthread_mutex_unlock(&J->mu);
    if (i >= J->n_tok) break;
    f8_token(J, i);
  }
  return NULL;
}

/* Routed block-FP8 MoE layer output (fp64) for the listed tokens.  x e4m3 [T,H] with fp32
   scales xs [T,H/128]; w13 e4m3 [E,2I,H] with fp32 scales [E,2I/128,H/128]; w2 e4m3
   [E,H,I] with fp32 scales [E,H/128,I/128].  The SiLU*up activation is requantized to e4m3
   with 1x128 scales before the down projection. */
void oracle_fp8_tokens(const uint8_t* x, const float* xs, const int32_t* ids, const float* w, int T, int H, int I,
                       int E, int k, const uint8_t* w13, const float* w13_s, const uint8_t* w2, const float* w2_s,
                       const int32_t* tokens, int n_tok, double* out, float* hq_out, int nthreads) {
  f8_job J = {x, xs, ids, w, T, H, I, E, k, w13, w2, w13_s, w2_s, tokens, n_tok, out, hq_out, 0, PTHREAD_MUTEX_INITIALIZER};
  run_pool(f8_worker, &J, nthreads);
  pthread_mutex_destroy(&J.mu);
}

/* ------------------------------------------------------------------ W4A8 (MXFP4 x FP8) layer */

/* The W4A8 format of the Humming issue ("[Performance] W4A8 MoE GEMM significantly slower than
   W4A16 on H200", the opening report): weights MXFP4, activations FP8 quantized along K in
   groups (per token, 32 or 128); this oracle takes the 32-group configuration.  MXFP4 is the
   OCP microscaling format: FP4 E2M1 elements sharing one E8M0 power-of-two scale per block of
   32 consecutive K elements.  The pages leave the activation scale's format open; the reading
   taken is the microscaling one for both operands (an E8M0 power-of-two scale per 32 elements,
   FP8 E4M3 elements), chosen as the smallest power of two that keeps the group inside E4M3's
   finite range. */

/* E2M1 code (low 4 bits) -> value: 1 sign bit, 2 exponent bits (bias 1), 1 mantissa bit;
   exponent field 0 is subnormal (0 or 0.5).  Magnitudes 0, 0.5, 1, 1.5, 2, 3, 4, 6. */
double oracle_e2m1(uint8_t c) {
  int s = (c >> 3) & 1, e = (c >> 1) & 3, m = c & 1;
  double v = e == 0 ? 0.5 * m : ldexp(1.0 + 0.5 * m, e - 1);
  return s ? -v : v;
}

/* E8M0 scale code -> 2^(code - 127); code 255 is NaN. */
double oracle_e8m0(uint8_t c) { return c == 255 ? NAN : ldexp(1.0, (int)c - 127); }

/* One group of 32 fp32 values -> E4M3 codes q and the group's E8M0 scale code.
   X = the smallest integer >= -127 with amax <= 448 * 2^X (at most 127); q[j] = e4m3(v[j] / 2^X),
   nearest with ties to even (the division by a power of two is exact).  Returns X + 127. */
uint8_t oracle_mx_quant32(const float* v, uint8_t* q) {
  double amax = 0.0;
  for (int j = 0; j < 32; ++j)
    if (fabs((double)v[j]) > amax) amax = fabs((double)v[j]);
  int X = -127;
  while (X < 127 && amax > ldexp(448.0, X)) ++X;
  for (int j = 0; j < 32; ++j) q[j] = oracle_e4m3_encode((float)ldexp((double)v[j], -X));
  return (uint8_t)(X + 127);
}

/* MXFP4 weight element (n, c) of one expert's [R, K] matrix: codes packed two per byte along K
   (even K index in the low nibble), [R, K/2]; scale codes [K/128, R, 4] (the scale of K block
   32*(4*b + j) of row n at [b][n][j]). */
static inline double mxw(const uint8_t* q, const uint8_t* sf, int R, int K, int n, int c) {
  uint8_t byte = q[(size_t)n * (K / 2) + c / 2];
  uint8_t code = (c & 1) ? (byte >> 4) : (byte & 15);
  return oracle_e2m1(code) * oracle_e8m0(sf[((size_t)(c / 128) * R + n) * 4 + (c / 32) % 4]);
}

typedef struct {
  const uint16_t* x;
  const int32_t* ids;
  const float* w;
  int T, H, I, E, k;
  const uint8_t *w13, *w13_sf, *w2, *w2_sf;
  const int32_t* tokens;
  int n_tok;
  double* out;
  float* hq_out; /* [n_tok, k, I] dequantized requantized h, or NULL */
  int next;
  pthread_mutex_t mu;
} mx_job;

static void mx_token(mx_job* J, int i) {
  int t = J->tokens[i], H = J->H, I = J->I, k = J->k;
  double* xr = (double*)malloc(sizeof(double) * (size_t)H);
  double* g = (double*)malloc(sizeof(double) * 2 * (size_t)I);
  float* hf = (float*)malloc(sizeof(float) * (size_t)I);
  double* hd = (double*)malloc(sizeof(double) * (size_t)I);
  double* o = J->out + (size_t)i * H;
  float v[32];
  uint8_t qc[32];
  /* the bf16 input row quantized group by group (32 along K), then dequantized */
  for (int g0 = 0; g0 < H; g0 += 32) {
    for (int j = 0; j < 32; ++j) v[j] = (float)oracle_bf16(J->x[(size_t)t * H + g0 + j]);
    double sc = oracle_e8m0(oracle_mx_quant32(v, qc));
    for (int j = 0; j < 32; ++j) xr[g0 + j] = oracle_e4m3(qc[j]) * sc;
  }
  for (int c = 0; c < H; ++c) o[c] = 0.0;
  for (int s = 0; s < k; ++s) {
    int e = J->ids[(size_t)t * k + s];
    double ws = (double)J->w[(size_t)t * k + s];
    const uint8_t* q13 = J->w13 + (size_t)e * 2 * I * (H / 2);
    const uint8_t* f13 = J->w13_sf + (size_t)e * (H / 128) * 2 * I * 4;
    const uint8_t* q2 = J->w2 + (size_t)e * H * (I / 2);
    const uint8_t* f2 = J->w2_sf + (size_t)e * (I / 128) * H * 4;
    for (int n = 0; n < 2 * I; ++n) {
      double acc = 0.0;
      for (int c = 0; c < H; ++c) acc += xr[c] * mxw(q13, f13, 2 * I, H, n, c);
      g[n] = acc;
    }
    /* h = SiLU(gate) * up held in fp32, requantized in groups of 32 like the input */
    for (int j = 0; j < I; ++j) hf[j] = (float)(oracle_silu(g[j]) * g[I + j]);
    for (int g0 = 0; g0 < I; g0 += 32) {
      double sc = oracle_e8m0(oracle_mx_quant32(hf + g0, qc));
      for (int j = 0; j < 32; ++j) hd[g0 + j] = oracle_e4m3(qc[j]) * sc;
    }
    if (J->hq_out)
      for (int j = 0; j < I; ++j) J->hq_out[((size_t)i * k + s) * I + j] = (float)hd[j];
    for (int c = 0; c < H; ++c) {
      double acc = 0.0;
      for (int j = 0; j < I; ++j) acc += hd[j] * mxw(q2, f2, H, I, c, j);
      o[c] += ws * acc;
    }
  }
  free(xr);
  free(g);
  free(hf);
  free(hd);
}

static void* mx_worker(void* a) {
  mx_job* J = (mx_job*)a;
  for (;;) {
    pthread_mutex_lock(&J->mu);
    int i = J->next++;
    pthread_mutex_unlock(&J->mu);
    if (i >= J->n_tok) break;
    mx_token(J, i);
  }
  return NULL;
}

/* Routed W4A8 MoE layer output (fp64) for the listed tokens.  x bf16 [T,H]; w13 MXFP4 codes
   [E,2I,H/2] with scale codes [E,H/128,2I,4]; w2 codes [E,H,I/2] with scale codes
   [E,I/128,H,4].  Input and SiLU*up activations are quantized to E4M3 with one E8M0 scale per
   32 along K before each projection. */
void oracle_w4a8_tokens(const uint16_t* x, const int32_t* ids, const float* w, int T, int H, int I, int E, int k,
                        const uint8_t* w13, const uint8_t* w13_sf, const uint8_t* w2, const uint8_t* w2_sf,
                        const int32_t* tokens, int n_tok, double* out, float* hq_out, int nthreads) {
  mx_job J = {x, ids, w, T, H, I, E, k, w13, w13_sf, w2, w2_sf, tokens, n_tok, out, hq_out, 0,
              PTHREAD_MUTEX_INITIALIZER};
  run_pool(mx_worker, &J, nthreads);
  pthread_mutex_destroy(&J.mu);
}
