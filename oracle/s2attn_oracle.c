/*
 * S2-Attn oracle: a plain, slow, fp64 CPU statement of shifted sparse attention,
 * forward and backward, with RoPE and linear position interpolation applied to q and k.
 *
 * TEST INFRASTRUCTURE ONLY. Only the tests, the smoke check and the bench's CPU-baseline
 * leg load this file's library. The CUDA path shares no code, header or table with it.
 *
 * What it computes, step by step, in the order the pages give:
 *   1. RoPE with position interpolation ("LoRA for Long-Context Adaptation",
 *      sections "Why vanilla LoRA under-delivers on long context" and
 *      "Position interpolation: the prerequisite"): the channel pair (2i, 2i+1) of q and
 *      of k at token m is rotated by phi = (m / s) * theta_i, theta_i = base^(-2i/d)
 *      (the RoFormer form; s = L_new / L_orig). v is not rotated.
 *   2. Head split and half-group shift ("LongLoRA and Shifted Sparse Attention (S^2-Attn)",
 *      definition paragraph; "LongLoRA: Efficient 100k Context LLM Fine-Tuning Guide",
 *      "How Shifted Short Attention Works" items 1-2 and "Implementation ... Step 1"):
 *      the second half of the heads sees the sequence rolled by -G/2 with wrap-around,
 *      i.e. rolled row r holds original row (r + G/2) mod N.
 *   3. Group fold: rolled rows are cut into N/G groups of G consecutive rows.
 *   4. Inside each group: scores q.k / sqrt(d), causal mask (key local index <= query
 *      local index), max-subtracted softmax, weighted sum of v (same Step 1 code).
 *   5. The shifted heads' outputs are rolled back by +G/2: the output of rolled row r is
 *      written at original row (r + G/2) mod N.
 * The backward is the analytic gradient of 1-5 (row-wise softmax gradient
 * dS = P * (dP - rowsum(dO * O)), then the transposed rotation of step 1 on dq and dk).
 *
 * Readings taken where the pages are silent: interleaved RoPE
 * pairs; q/k rotated at their original (pre-roll) token index; LSE = natural log of the
 * sum of exp of the scaled scores; GQA query head h uses kv head h / (Hq / Hkv), and the
 * shift of a kv head follows the query heads that use it (Hkv even keeps these aligned).
 *
 * Layouts: q, o, dout, dq [B][N][Hq][d]; k, v, dk, dv [B][N][Hkv][d]; lse [B][Hq][N].
 * Inputs may be bf16 bit patterns, fp32 or fp64; all arithmetic is fp64.
 *
 * Work unit = (b, kv head, group g): it covers the R = Hq / Hkv query heads of the kv
 * head and the G rolled rows of group g. Units are independent; the full functions run
 * them in parallel with OpenMP. Unit outputs are indexed by the rolled local row i in
 * [0, G): row i belongs to original token src(g*G + i).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

enum { S2O_IN_BF16 = 0, S2O_IN_F32 = 1, S2O_IN_F64 = 2 };

typedef struct {
  int B, N, Hq, Hkv, d, G, causal, shift;
  double s, base;
} cfg_t;

static double load(const void* p, int dt, size_t i) {
  if (dt == S2O_IN_BF16) {
    uint32_t u = (uint32_t)((const uint16_t*)p)[i] << 16;
    float f;
    memcpy(&f, &u, 4);
    return (double)f;
  }
  if (dt == S2O_IN_F32) return (double)((const float*)p)[i];
  return ((const double*)p)[i];
}

/* Shape rules of the pages' Step 1 code: H even (half the heads shift), N a multiple of G,
 * G even (shift = G/2). GQA adds Hq % Hkv == 0 and Hkv even. d even for RoPE pairs. */
int s2o_check(int B, int N, int Hq, int Hkv, int d, int G) {
  if (B <= 0 || N <= 0 || Hq <= 0 || Hkv <= 0 || d <= 0 || G <= 0) return 1;
  if (G > N || N % G != 0 || G % 2 != 0) return 1;
  if (Hq % 2 != 0 || Hkv % 2 != 0 || Hq % Hkv != 0) return 1;
  if (d % 2 != 0) return 1;
  return 0;
}

/* Which heads see the rolled sequence (the shift pattern):
 *   0 (default) the second half of the heads ("LongLoRA and Shifted Sparse Attention
 *     (S^2-Attn)", definition; "LongLoRA: Efficient 100k Context LLM Fine-Tuning Guide",
 *     Implementation, Step 1);
 *   1 alternate heads, the odd ones ("LoRA for Long-Context Adaptation", section
 *     "Shifted sparse attention: making training feasible": heads 0, 2, 4, ... unshifted,
 *     heads 1, 3, 5, ... shifted by half a group);
 *   2 no head (plain grouped attention; with G = N the dense attention the guide's
 *     inference path falls back to, "Dual-Mode" paragraph).
 * Query head h follows its kv head h / R, so with GQA the pattern applies to kv heads. */
static int shifted_head(const cfg_t* c, int h) {
  const int R = c->Hq / c->Hkv;
  if (c->shift == 1) return (h / R) % 2 == 1;
  if (c->shift == 2) return 0;
  return h >= c->Hq / 2;
}

/* Rolled row r -> original row. np.roll(x, -G/2)[r] == x[(r + G/2) mod N]. */
static long src_row(const cfg_t* c, long r, int shifted) {
  return shifted ? (r + c->G / 2) % c->N : r;
}

/* Rotate one head vector of token m: y = R(phi) x per channel pair, or R(phi)^T x. */
static void rope(const double* x, double* y, int d, long m, double s, double base, int inverse) {
  for (int i = 0; i < d / 2; i++) {
    double theta = pow(base, -2.0 * (double)i / (double)d);
    double phi = ((double)m / s) * theta;
    double cs = cos(phi), sn = sin(phi);
    if (inverse) sn = -sn;
    double x0 = x[2 * i], x1 = x[2 * i + 1];
    y[2 * i] = x0 * cs - x1 * sn;
    y[2 * i + 1] = x0 * sn + x1 * cs;
  }
}

/* Exported for the RoPE pins: rotate n rows of x [n][d] at positions pos[n]. */
void s2o_rope(const double* x, double* y, int n, const long* pos, int d, double s, double base,
              int inverse) {
  for (int r = 0; r < n; r++) rope(x + (size_t)r * d, y + (size_t)r * d, d, pos[r], s, base, inverse);
}

static double dot(const double* a, const double* b, int d) {
  double acc = 0.0;
  for (int c = 0; c < d; c++) acc += a[c] * b[c];
  return acc;
}

/* Per-unit scratch: rotated keys, values of the group, and per-head row buffers. */
typedef struct {
  double *kr, *vr, *qr, *orow, *lse, *sc, *dor, *dqr, *dkr, *dvr, *Drow, *tmp;
} scratch_t;

static int scratch_alloc(scratch_t* w, int G, int d) {
  size_t gd = (size_t)G * d;
  memset(w, 0, sizeof(*w));
  w->kr = malloc(gd * sizeof(double));
  w->vr = malloc(gd * sizeof(double));
  w->qr = malloc(gd * sizeof(double));
  w->orow = malloc(gd * sizeof(double));
  w->dor = malloc(gd * sizeof(double));
  w->dqr = malloc(gd * sizeof(double));
  w->dkr = malloc(gd * sizeof(double));
  w->dvr = malloc(gd * sizeof(double));
  w->lse = malloc((size_t)G * sizeof(double));
  w->Drow = malloc((size_t)G * sizeof(double));
  w->sc = malloc((size_t)G * sizeof(double));
  w->tmp = malloc((size_t)d * sizeof(double));
  return w->kr && w->vr && w->qr && w->orow && w->dor && w->dqr && w->dkr && w->dvr && w->lse &&
         w->Drow && w->sc && w->tmp;
}

static void scratch_free(scratch_t* w) {
  free(w->kr); free(w->vr); free(w->qr); free(w->orow); free(w->dor); free(w->dqr);
  free(w->dkr); free(w->dvr); free(w->lse); free(w->Drow); free(w->sc); free(w->tmp);
}

/* Load the group's keys (rotated) and values for kv head kvh, in rolled local order. */
static void load_group_kv(const cfg_t* c, const void* k, const void* v, int dt, int b, int kvh,
                          int g, int shifted, scratch_t* w) {
  int d = c->d;
  for (int j = 0; j < c->G; j++) {
    long m = src_row(c, (long)g * c->G + j, shifted);
    size_t base = (((size_t)b * c->N + m) * c->Hkv + kvh) * d;
    for (int e = 0; e < d; e++) w->tmp[e] = load(k, dt, base + e);
    rope(w->tmp, w->kr + (size_t)j * d, d, m, c->s, c->base, 0);
    for (int e = 0; e < d; e++) w->vr[(size_t)j * d + e] = load(v, dt, base + e);
  }
}

/* Forward of one query head over one group: fills w->qr (rotated q rows), w->orow, w->lse. */
static void head_forward(const cfg_t* c, const void* q, int dt, int b, int h, int g, int shifted,
                         scratch_t* w) {
  int d = c->d, G = c->G;
  double inv_sqrt_d = 1.0 / sqrt((double)d);
  for (int i = 0; i < G; i++) {
    long m = src_row(c, (long)g * G + i, shifted);
    size_t base = (((size_t)b * c->N + m) * c->Hq + h) * d;
    for (int e = 0; e < d; e++) w->tmp[e] = load(q, dt, base + e);
    rope(w->tmp, w->qr + (size_t)i * d, d, m, c->s, c->base, 0);
  }
  for (int i = 0; i < G; i++) {
    const double* qi = w->qr + (size_t)i * d;
    int jmax = c->causal ? i : G - 1;
    double mx = -INFINITY;
    for (int j = 0; j <= jmax; j++) {
      w->sc[j] = dot(qi, w->kr + (size_t)j * d, d) * inv_sqrt_d;
      if (w->sc[j] > mx) mx = w->sc[j];
    }
    double sum = 0.0;
    for (int j = 0; j <= jmax; j++) sum += exp(w->sc[j] - mx);
    double lse = mx + log(sum);
    w->lse[i] = lse;
    double* oi = w->orow + (size_t)i * d;
    for (int e = 0; e < d; e++) oi[e] = 0.0;
    for (int j = 0; j <= jmax; j++) {
      double p = exp(w->sc[j] - lse);
      const double* vj = w->vr + (size_t)j * d;
      for (int e = 0; e < d; e++) oi[e] += p * vj[e];
    }
  }
}

static int unit_args_ok(const cfg_t* c, int b, int kvh, int g) {
  return b >= 0 && b < c->B && kvh >= 0 && kvh < c->Hkv && g >= 0 && g < c->N / c->G;
}

/* `causal` carries two fields: bit 0 the causal mask inside a group, bits 4-5 the shift
 * pattern of shifted_head (0 when the caller passes a plain 0 / 1). */
static void fill_cfg(cfg_t* c, int B, int N, int Hq, int Hkv, int d, int G, int causal, double s,
                     double base) {
  c->B = B; c->N = N; c->Hq = Hq; c->Hkv = Hkv; c->d = d; c->G = G; c->causal = causal & 1;
  c->shift = (causal >> 4) & 3;
  c->s = s; c->base = base;
}

/* One unit's forward. o_u [R][G][d], lse_u [R][G], rolled local row order. */
static int fwd_unit(const cfg_t* c, const void* q, const void* k, const void* v, int dt, int b,
                    int kvh, int g, double* o_u, double* lse_u, scratch_t* w) {
  int R = c->Hq / c->Hkv, G = c->G, d = c->d;
  int shifted = shifted_head(c, kvh * R);
  load_group_kv(c, k, v, dt, b, kvh, g, shifted, w);
  for (int r = 0; r < R; r++) {
    head_forward(c, q, dt, b, kvh * R + r, g, shifted, w);
    memcpy(o_u + (size_t)r * G * d, w->orow, (size_t)G * d * sizeof(double));
    memcpy(lse_u + (size_t)r * G, w->lse, (size_t)G * sizeof(double));
  }
  return 0;
}

/* One unit's backward. dq_u [R][G][d], dk_u, dv_u [G][d], rolled local row order.
 * O and LSE are recomputed here by the oracle's own forward. */
static int bwd_unit(const cfg_t* c, const void* q, const void* k, const void* v, const void* dout,
                    int dt, int b, int kvh, int g, double* dq_u, double* dk_u, double* dv_u,
                    scratch_t* w) {
  int R = c->Hq / c->Hkv, G = c->G, d = c->d;
  double inv_sqrt_d = 1.0 / sqrt((double)d);
  int shifted = shifted_head(c, kvh * R);
  load_group_kv(c, k, v, dt, b, kvh, g, shifted, w);
  memset(w->dkr, 0, (size_t)G * d * sizeof(double));
  memset(w->dvr, 0, (size_t)G * d * sizeof(double));
  for (int r = 0; r < R; r++) {
    int h = kvh * R + r;
    head_forward(c, q, dt, b, h, g, shifted, w);
    for (int i = 0; i < G; i++) {
      long m = src_row(c, (long)g * G + i, shifted);
      size_t base = (((size_t)b * c->N + m) * c->Hq + h) * d;
      for (int e = 0; e < d; e++) w->dor[(size_t)i * d + e] = load(dout, dt, base + e);
      w->Drow[i] = dot(w->dor + (size_t)i * d, w->orow + (size_t)i * d, d);
    }
    memset(w->dqr, 0, (size_t)G * d * sizeof(double));
    for (int i = 0; i < G; i++) {
      const double* qi = w->qr + (size_t)i * d;
      const double* doi = w->dor + (size_t)i * d;
      double* dqi = w->dqr + (size_t)i * d;
      int jmax = c->causal ? i : G - 1;
      for (int j = 0; j <= jmax; j++) {
        const double* kj = w->kr + (size_t)j * d;
        const double* vj = w->vr + (size_t)j * d;
        double s = dot(qi, kj, d) * inv_sqrt_d;
        double p = exp(s - w->lse[i]);
        double dp = dot(doi, vj, d);
        double ds = p * (dp - w->Drow[i]);
        double* dkj = w->dkr + (size_t)j * d;
        double* dvj = w->dvr + (size_t)j * d;
        for (int e = 0; e < d; e++) {
          dqi[e] += ds * inv_sqrt_d * kj[e];
          dkj[e] += ds * inv_sqrt_d * qi[e];
          dvj[e] += p * doi[e];
        }
      }
    }
    for (int i = 0; i < G; i++) {
      long m = src_row(c, (long)g * G + i, shifted);
      rope(w->dqr + (size_t)i * d, dq_u + ((size_t)r * G + i) * d, d, m, c->s, c->base, 1);
    }
  }
  for (int j = 0; j < G; j++) {
    long m = src_row(c, (long)g * G + j, shifted);
    rope(w->dkr + (size_t)j * d, dk_u + (size_t)j * d, d, m, c->s, c->base, 1);
    memcpy(dv_u + (size_t)j * d, w->dvr + (size_t)j * d, (size_t)d * sizeof(double));
  }
  return 0;
}

int s2o_fwd_unit(const void* q, const void* k, const void* v, int dt, int B, int N, int Hq,
                 int Hkv, int d, int G, int causal, double s, double base, int b, int kvh, int g,
                 double* o_u, double* lse_u) {
  cfg_t c;
  scratch_t w;
  if (s2o_check(B, N, Hq, Hkv, d, G)) return 1;
  fill_cfg(&c, B, N, Hq, Hkv, d, G, causal, s, base);
  if (!unit_args_ok(&c, b, kvh, g)) return 1;
  if (!scratch_alloc(&w, G, d)) { scratch_free(&w); return 2; }
  fwd_unit(&c, q, k, v, dt, b, kvh, g, o_u, lse_u, &w);
  scratch_free(&w);
  return 0;
}

int s2o_bwd_unit(const void* q, const void* k, const void* v, const void* dout, int dt, int B,
                 int N, int Hq, int Hkv, int d, int G, int causal, double s, double base, int b,
                 int kvh, int g, double* dq_u, double* dk_u, double* dv_u) {
  cfg_t c;
  scratch_t w;
  if (s2o_check(B, N, Hq, Hkv, d, G)) return 1;
  fill_cfg(&c, B, N, Hq, Hkv, d, G, causal, s, base);
  if (!unit_args_ok(&c, b, kvh, g)) return 1;
  if (!scratch_alloc(&w, G, d)) { scratch_free(&w); return 2; }
  bwd_unit(&c, q, k, v, dout, dt, b, kvh, g, dq_u, dk_u, dv_u, &w);
  scratch_free(&w);
  return 0;
}

/* Full forward: o [B][N][Hq][d], lse [B][Hq][N], original token order (rolled back). */
int s2o_fwd(const void* q, const void* k, const void* v, int dt, int B, int N, int Hq, int Hkv,
            int d, int G, int causal, double s, double base, double* o, double* lse) {
  cfg_t c;
  if (s2o_check(B, N, Hq, Hkv, d, G)) return 1;
  fill_cfg(&c, B, N, Hq, Hkv, d, G, causal, s, base);
  int R = Hq / Hkv, ng = N / G;
  long units = (long)B * Hkv * ng;
  int err = 0;
#pragma omp parallel
  {
    scratch_t w;
    double* o_u = malloc((size_t)R * G * d * sizeof(double));
    double* lse_u = malloc((size_t)R * G * sizeof(double));
    int ok = scratch_alloc(&w, G, d) && o_u && lse_u;
    if (!ok) {
#pragma omp atomic write
      err = 2;
    }
#pragma omp for schedule(dynamic, 1)
    for (long u = 0; u < units; u++) {
      if (!ok) continue;
      int b = (int)(u / ((long)Hkv * ng)), kvh = (int)((u / ng) % Hkv), g = (int)(u % ng);
      int shifted = shifted_head(&c, kvh * R);
      fwd_unit(&c, q, k, v, dt, b, kvh, g, o_u, lse_u, &w);
      for (int r = 0; r < R; r++) {
        int h = kvh * R + r;
        for (int i = 0; i < G; i++) {
          long m = src_row(&c, (long)g * G + i, shifted);
          memcpy(o + (((size_t)b * N + m) * Hq + h) * d, o_u + ((size_t)r * G + i) * d,
                 (size_t)d * sizeof(double));
          lse[((size_t)b * Hq + h) * N + m] = lse_u[(size_t)r * G + i];
        }
      }
    }
    scratch_free(&w);
    free(o_u);
    free(lse_u);
  }
  return err;
}

/* Full backward: dq [B][N][Hq][d], dk, dv [B][N][Hkv][d], original token order. */
int s2o_bwd(const void* q, const void* k, const void* v, const void* dout, int dt, int B, int N,
            int Hq, int Hkv, int d, int G, int causal, double s, double base, double* dq,
            double* dk, double* dv) {
  cfg_t c;
  if (s2o_check(B, N, Hq, Hkv, d, G)) return 1;
  fill_cfg(&c, B, N, Hq, Hkv, d, G, causal, s, base);
  int R = Hq / Hkv, ng = N / G;
  long units = (long)B * Hkv * ng;
  int err = 0;
#pragma omp parallel
  {
    scratch_t w;
    double* dq_u = malloc((size_t)R * G * d * sizeof(double));
    double* dk_u = malloc((size_t)G * d * sizeof(double));
    double* dv_u = malloc((size_t)G * d * sizeof(double));
    int ok = scratch_alloc(&w, G, d) && dq_u && dk_u && dv_u;
    if (!ok) {
#pragma omp atomic write
      err = 2;
    }
#pragma omp for schedule(dynamic, 1)
    for (long u = 0; u < units; u++) {
      if (!ok) continue;
      int b = (int)(u / ((long)Hkv * ng)), kvh = (int)((u / ng) % Hkv), g = (int)(u % ng);
      int shifted = shifted_head(&c, kvh * R);
      bwd_unit(&c, q, k, v, dout, dt, b, kvh, g, dq_u, dk_u, dv_u, &w);
      for (int i = 0; i < G; i++) {
        long m = src_row(&c, (long)g * G + i, shifted);
        for (int r = 0; r < R; r++)
          memcpy(dq + (((size_t)b * N + m) * Hq + kvh * R + r) * d, dq_u + ((size_t)r * G + i) * d,
                 (size_t)d * sizeof(double));
        memcpy(dk + (((size_t)b * N + m) * Hkv + kvh) * d, dk_u + (size_t)i * d,
               (size_t)d * sizeof(double));
        memcpy(dv + (((size_t)b * N + m) * Hkv + kvh) * d, dv_u + (size_t)i * d,
               (size_t)d * sizeof(double));
      }
    }
    scratch_free(&w);
    free(dq_u);
    free(dk_u);
    free(dv_u);
  }
  return err;
}

/* ------------------------------------------------------------------------------------
 * Row-sampled evaluation: the same definition evaluated only at chosen rows, so that large
 * shapes can be checked on sampled outputs. Row indices are rolled local rows of group g.
 * ---------------------------------------------------------------------------------- */

/* Softmax statistics and output of one query row i (rotated q row qi) against the group's
 * rotated keys / values: lse and o (length d). sc is a G-length buffer. */
static void row_forward(const cfg_t* c, const double* qi, const double* kr, const double* vr,
                        int i, double* sc, double* o, double* lse_out) {
  int d = c->d, G = c->G;
  double inv_sqrt_d = 1.0 / sqrt((double)d);
  int jmax = c->causal ? i : G - 1;
  double mx = -INFINITY;
  for (int j = 0; j <= jmax; j++) {
    sc[j] = dot(qi, kr + (size_t)j * d, d) * inv_sqrt_d;
    if (sc[j] > mx) mx = sc[j];
  }
  double sum = 0.0;
  for (int j = 0; j <= jmax; j++) sum += exp(sc[j] - mx);
  double lse = mx + log(sum);
  for (int e = 0; e < d; e++) o[e] = 0.0;
  for (int j = 0; j <= jmax; j++) {
    double p = exp(sc[j] - lse);
    for (int e = 0; e < d; e++) o[e] += p * vr[(size_t)j * d + e];
  }
  *lse_out = lse;
}

static void load_q_row(const cfg_t* c, const void* x, int dt, int b, int h, long m, double* tmp,
                       double* out, int rotate) {
  size_t base = (((size_t)b * c->N + m) * c->Hq + h) * c->d;
  for (int e = 0; e < c->d; e++) tmp[e] = load(x, dt, base + e);
  if (rotate)
    rope(tmp, out, c->d, m, c->s, c->base, 0);
  else
    memcpy(out, tmp, (size_t)c->d * sizeof(double));
}

/* Forward at nrows rolled local rows of query head h in group g:
 * o_rows [nrows][d], lse_rows [nrows]. */
int s2o_fwd_rows(const void* q, const void* k, const void* v, int dt, int B, int N, int Hq,
                 int Hkv, int d, int G, int causal, double s, double base, int b, int h, int g,
                 int nrows, const int* rows, double* o_rows, double* lse_rows) {
  cfg_t c;
  scratch_t w;
  if (s2o_check(B, N, Hq, Hkv, d, G)) return 1;
  fill_cfg(&c, B, N, Hq, Hkv, d, G, causal, s, base);
  int R = Hq / Hkv, kvh = h / R;
  if (h < 0 || h >= Hq || !unit_args_ok(&c, b, kvh, g)) return 1;
  for (int t = 0; t < nrows; t++)
    if (rows[t] < 0 || rows[t] >= G) return 1;
  if (!scratch_alloc(&w, G, d)) { scratch_free(&w); return 2; }
  int shifted = shifted_head(&c, h);
  load_group_kv(&c, k, v, dt, b, kvh, g, shifted, &w);
#pragma omp parallel
  {
    double* sc = malloc((size_t)G * sizeof(double));
    double* tmp = malloc((size_t)d * sizeof(double));
    double* qi = malloc((size_t)d * sizeof(double));
#pragma omp for schedule(dynamic, 4)
    for (int t = 0; t < nrows; t++) {
      long m = src_row(&c, (long)g * G + rows[t], shifted);
      load_q_row(&c, q, dt, b, h, m, tmp, qi, 1);
      row_forward(&c, qi, w.kr, w.vr, rows[t], sc, o_rows + (size_t)t * d, lse_rows + t);
    }
    free(sc); free(tmp); free(qi);
  }
  scratch_free(&w);
  return 0;
}

/* Backward of unit (b, kvh, g) at sampled rows: dq at nq query rows for all R heads of the
 * kv head (dq_rows [nq][R][d]) and dk, dv at nk key rows (dk_rows, dv_rows [nk][d]).
 * The per-row statistics lse_i and D_i = <dO_i, O_i> that every gradient needs are
 * computed for all G rows first (the oracle's own forward). */
int s2o_bwd_rows(const void* q, const void* k, const void* v, const void* dout, int dt, int B,
                 int N, int Hq, int Hkv, int d, int G, int causal, double s, double base, int b,
                 int kvh, int g, int nq, const int* qrows, int nk, const int* krows,
                 double* dq_rows, double* dk_rows, double* dv_rows) {
  cfg_t c;
  scratch_t w;
  if (s2o_check(B, N, Hq, Hkv, d, G)) return 1;
  fill_cfg(&c, B, N, Hq, Hkv, d, G, causal, s, base);
  if (!unit_args_ok(&c, b, kvh, g)) return 1;
  for (int t = 0; t < nq; t++)
    if (qrows[t] < 0 || qrows[t] >= G) return 1;
  for (int t = 0; t < nk; t++)
    if (krows[t] < 0 || krows[t] >= G) return 1;
  if (!scratch_alloc(&w, G, d)) { scratch_free(&w); return 2; }
  int R = Hq / Hkv;
  double inv_sqrt_d = 1.0 / sqrt((double)d);
  int shifted = shifted_head(&c, kvh * R);
  load_group_kv(&c, k, v, dt, b, kvh, g, shifted, &w);
  double* dkr = calloc((size_t)(nk > 0 ? nk : 1) * d, sizeof(double));
  double* dvr = calloc((size_t)(nk > 0 ? nk : 1) * d, sizeof(double));
  for (int r = 0; r < R; r++) {
    int h = kvh * R + r;
    /* statistics of every row of the group */
#pragma omp parallel
    {
      double* sc = malloc((size_t)G * sizeof(double));
      double* tmp = malloc((size_t)d * sizeof(double));
      double* orow = malloc((size_t)d * sizeof(double));
#pragma omp for schedule(dynamic, 16)
      for (int i = 0; i < G; i++) {
        long m = src_row(&c, (long)g * G + i, shifted);
        load_q_row(&c, q, dt, b, h, m, tmp, w.qr + (size_t)i * d, 1);
        load_q_row(&c, dout, dt, b, h, m, tmp, w.dor + (size_t)i * d, 0);
        row_forward(&c, w.qr + (size_t)i * d, w.kr, w.vr, i, sc, orow, w.lse + i);
        w.Drow[i] = dot(w.dor + (size_t)i * d, orow, d);
      }
      free(sc); free(tmp); free(orow);
    }
    /* dq at the sampled query rows */
#pragma omp parallel
    {
      double* acc = malloc((size_t)d * sizeof(double));
#pragma omp for schedule(dynamic, 1)
      for (int t = 0; t < nq; t++) {
        int i = qrows[t];
        const double* qi = w.qr + (size_t)i * d;
        const double* doi = w.dor + (size_t)i * d;
        int jmax = c.causal ? i : G - 1;
        for (int e = 0; e < d; e++) acc[e] = 0.0;
        for (int j = 0; j <= jmax; j++) {
          const double* kj = w.kr + (size_t)j * d;
          double p = exp(dot(qi, kj, d) * inv_sqrt_d - w.lse[i]);
          double ds = p * (dot(doi, w.vr + (size_t)j * d, d) - w.Drow[i]);
          for (int e = 0; e < d; e++) acc[e] += ds * inv_sqrt_d * kj[e];
        }
        long m = src_row(&c, (long)g * G + i, shifted);
        rope(acc, dq_rows + ((size_t)t * R + r) * d, d, m, c.s, c.base, 1);
      }
      free(acc);
    }
    /* dk, dv at the sampled key rows (summed over the kv head's query heads) */
#pragma omp parallel for schedule(dynamic, 1)
    for (int t = 0; t < nk; t++) {
      int j = krows[t];
      const double* kj = w.kr + (size_t)j * d;
      const double* vj = w.vr + (size_t)j * d;
      int ibeg = c.causal ? j : 0;
      for (int i = ibeg; i < G; i++) {
        const double* qi = w.qr + (size_t)i * d;
        const double* doi = w.dor + (size_t)i * d;
        double p = exp(dot(qi, kj, d) * inv_sqrt_d - w.lse[i]);
        double ds = p * (dot(doi, vj, d) - w.Drow[i]);
        for (int e = 0; e < d; e++) {
          dkr[(size_t)t * d + e] += ds * inv_sqrt_d * qi[e];
          dvr[(size_t)t * d + e] += p * doi[e];
        }
      }
    }
  }
  for (int t = 0; t < nk; t++) {
    long m = src_row(&c, (long)g * G + krows[t], shifted);
    rope(dkr + (size_t)t * d, dk_rows + (size_t)t * d, d, m, c.s, c.base, 1);
    memcpy(dv_rows + (size_t)t * d, dvr + (size_t)t * d, (size_t)d * sizeof(double));
  }
  free(dkr);
  free(dvr);
  scratch_free(&w);
  return 0;
}

int s2o_max_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}

void s2o_set_threads(int n) {
#ifdef _OPENMP
  if (n > 0) omp_set_num_threads(n);
#else
  (void)n;
#endif
}
