/*
 * moe_oracle.c -- plain, slow CPU oracle for the forward pass of a sparse Mixture-of-Experts
 * layer with block-quantized expert weights.
 *
 * TEST INFRASTRUCTURE ONLY. Nothing in the product path links, loads or calls this file; it
 * exists so that tests, the smoke check and the CPU-baseline leg of the benchmark can check the
 * CUDA library against an independent, obviously-correct restatement of what the layer computes.
 * It shares no code, header, table or constant generator with the CUDA library.
 *
 * What the layer computes (the pages describe the model, not the formats; the quantized block
 * formats are a stated stand-in):
 *   - 512 routed experts per layer, 10 active per token, always-on shared expert(s):
 *     "Strata vs Llama.cpp vs vLLM", chapter "How Strata is designed to work";
 *     Strata DETAILS.md, "How it works" (routers and shared experts live on the GPU).
 *   - expert math is a quantized matrix multiply that dequantizes on the fly:
 *     "Two-Day Port, 8x Faster Prefill: Strata Engine Benchmarked", section
 *     "Where Strata Is Fast: Not Magic, but Logistics" (MMQ paragraph).
 *   - block formats (stand-in): Q2 = 32 weights of 2-bit codes c and one fp16 scale d,
 *     w = d*(c-2); Q3 = 3-bit codes, w = d*(c-4); Q4 (a further stand-in of the same family)
 *     = 4-bit codes, w = d*(c-8).
 *
 * Arithmetic is fp64 throughout (exact products of exactly-decoded inputs, fp64 sums), except
 * where a rounding is part of the definition (the bf16 output of RMSNorm) or where the
 * diagnostic "mirrored" mode is asked for (it rounds x, weights, h and expert outputs to fp16
 * at the points where the GPU path stores fp16 operands, to separate a logic error from
 * precision loss).
 *
 * Bit layout of the packed planes (this library's ABI; the pages do not fix one):
 *   per block of 32 weights along K, the 2-bit plane holds two 32-bit little-endian words;
 *   word q (weights 16q..16q+15) holds weight 16q+2i+h (i=0..7, h=0..1) at bits 16h+2i..16h+2i+1.
 *   Q3 adds a 1-bit plane, one 32-bit little-endian word per block, holding bit 2 of the code of
 *   weight 16q+2i+h at bit 16h+8q+i.  code = low2 | hibit<<2.
 *   Q4 has one 4-bit plane [n][rows][K/2]: per block four 32-bit little-endian words; word q
 *   (weights 8q..8q+7) holds weight 8q+2i+h (i=0..3, h=0..1) at bits 16h+4i..16h+4i+3.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

typedef struct {
  int32_t qtype;          /* 2 (Q2), 3 (Q3) or 4 (Q4) */
  int32_t n_experts, rows, K;
  const uint8_t *codes;   /* [n][rows][K/4]; Q4: [n][rows][K/2] */
  const uint8_t *hibits;  /* [n][rows][K/8], Q3 only */
  const uint16_t *scales; /* [n][rows][K/32], fp16 bit patterns */
} oq_mat;

/* ---------------------------------------------------------------- number formats */

/* exact value of an IEEE binary16 bit pattern */
double oracle_half_to_double(uint16_t h) {
  int s = h >> 15, e = (h >> 10) & 31, m = h & 1023;
  double v;
  if (e == 0) v = ldexp((double)m, -24);
  else if (e == 31) v = m ? NAN : INFINITY;
  else v = ldexp((double)(m + 1024), e - 25);
  return s ? -v : v;
}

/* exact value of a bfloat16 bit pattern (upper half of an IEEE binary32) */
double oracle_bf16_to_double(uint16_t b) {
  uint32_t u = (uint32_t)b << 16;
  float f;
  memcpy(&f, &u, 4);
  return (double)f;
}

/* round to the nearest binary16, ties to even */
uint16_t oracle_double_to_half(double v) {
  uint16_t sign = signbit(v) ? 0x8000 : 0;
  double a = fabs(v);
  if (isnan(v)) return 0x7e00;
  if (a == 0.0) return sign;
  if (a >= 65520.0) return sign | 0x7c00; /* halfway to 2^16 and above round to infinity */
  int e;
  frexp(a, &e);           /* a = f * 2^e, f in [0.5, 1) */
  int E = e - 1;          /* a in [2^E, 2^(E+1)) */
  if (E < -14) E = -14;   /* subnormal range: fixed ulp 2^-24 */
  double r = rint(ldexp(a, 10 - E)); /* significand in units of ulp = 2^(E-10) */
  if (r < 1024.0) return sign | (uint16_t)r; /* subnormal (only when E == -14) */
  if (r >= 2048.0) { r = 1024.0; E += 1; }
  if (E > 15) return sign | 0x7c00;
  return sign | (uint16_t)(((E + 15) << 10) | ((int)r - 1024));
}

/* round to the nearest bfloat16, ties to even */
uint16_t oracle_double_to_bf16(double v) {
  uint16_t sign = signbit(v) ? 0x8000 : 0;
  double a = fabs(v);
  if (isnan(v)) return 0x7fc0;
  if (a == 0.0) return sign;
  int e;
  frexp(a, &e);
  int E = e - 1;
  if (E < -126) E = -126;
  double r = rint(ldexp(a, 7 - E));
  if (r < 128.0) return sign | (uint16_t)r;
  if (r >= 256.0) { r = 128.0; E += 1; }
  if (E > 127) return sign | 0x7f80;
  return sign | (uint16_t)(((E + 127) << 7) | ((int)r - 128));
}

static double round_f16(double v) { return oracle_half_to_double(oracle_double_to_half(v)); }

/* ---------------------------------------------------------------- dequantization */

/* integer code of weight (e, r, k) from the packed planes (layout in the file header); -1 for a
 * block format other than Q2, Q3 or Q4 (nothing is read then) */
int oracle_code(const oq_mat *m, int e, int r, int k) {
  if (m->qtype != 2 && m->qtype != 3 && m->qtype != 4) return -1;
  size_t row = (size_t)e * m->rows + r;
  int b = k >> 5, j = k & 31;
  if (m->qtype == 4) {  /* word j/8 of the block, pair (i, h) = ((j%8)/2, j%2) at bit 16h+4i */
    const uint8_t *w4 = m->codes + row * (size_t)(m->K / 2) + (size_t)b * 16 + (size_t)(j >> 3) * 4;
    int bit = 16 * (j & 1) + 4 * ((j & 7) >> 1);
    return (w4[bit >> 3] >> (bit & 7)) & 15;
  }
  int q = j >> 4, jj = j & 15, h = jj & 1, i = jj >> 1;
  const uint8_t *w = m->codes + row * (size_t)(m->K / 4) + (size_t)b * 8 + (size_t)q * 4;
  int bit = 16 * h + 2 * i;
  int lo = (w[bit >> 3] >> (bit & 7)) & 3;
  if (m->qtype == 2) return lo;
  const uint8_t *hw = m->hibits + row * (size_t)(m->K / 8) + (size_t)b * 4;
  int hb = 16 * h + 8 * q + i;
  int hi = (hw[hb >> 3] >> (hb & 7)) & 1;
  return lo | (hi << 2);
}

/* w = d * (c - q0), q0 = 2 (Q2), 4 (Q3) or 8 (Q4), d the block's fp16 scale */
double oracle_weight(const oq_mat *m, int e, int r, int k) {
  size_t row = (size_t)e * m->rows + r;
  double d = oracle_half_to_double(m->scales[row * (size_t)(m->K / 32) + (k >> 5)]);
  int q0 = (m->qtype == 2) ? 2 : (m->qtype == 3) ? 4 : 8;
  return d * (double)(oracle_code(m, e, r, k) - q0);
}

/* rows row0..row0+nrows-1 of expert e: exact values (fp64) and, optionally, fp16-rounded values */
void oracle_dequant_rows(const oq_mat *m, int e, int row0, int nrows, double *out, uint16_t *out_f16) {
  for (int r = 0; r < nrows; ++r)
    for (int k = 0; k < m->K; ++k) {
      double v = oracle_weight(m, e, row0 + r, k);
      out[(size_t)r * m->K + k] = v;
      if (out_f16) out_f16[(size_t)r * m->K + k] = oracle_double_to_half(v);
    }
}

static void dequant_row(const oq_mat *m, int e, int r, double *out, int mirrored) {
  for (int k = 0; k < m->K; ++k) {
    double v = oracle_weight(m, e, r, k);
    out[k] = mirrored ? round_f16(v) : v;
  }
}

/* ---------------------------------------------------------------- RMSNorm (stack only) */

/* u = bf16( r / sqrt(mean(r^2) + eps) ), no learned gain */
void oracle_rmsnorm_bf16(const float *r, int T, int H, double eps, uint16_t *u) {
  for (int t = 0; t < T; ++t) {
    double ss = 0.0;
    for (int h = 0; h < H; ++h) ss += (double)r[(size_t)t * H + h] * (double)r[(size_t)t * H + h];
    double inv = 1.0 / sqrt(ss / H + eps);
    for (int h = 0; h < H; ++h) u[(size_t)t * H + h] = oracle_double_to_bf16((double)r[(size_t)t * H + h] * inv);
  }
}

/* ---------------------------------------------------------------- router + top-k */

typedef struct { double l; int e; } scored;

/* descending logit; equal logits: lower expert index first */
static int by_logit_desc(const void *pa, const void *pb) {
  const scored *a = (const scored *)pa, *b = (const scored *)pb;
  if (a->l > b->l) return -1;
  if (a->l < b->l) return 1;
  return (a->e > b->e) - (a->e < b->e);
}

/* logits of one token: l_e = sum_h x_h * Wr[e][h] + bias_e */
static void router_logits(const double *x, int H, const float *Wr, const float *bias, int E, double *l) {
  for (int e = 0; e < E; ++e) {
    double s = 0.0;
    const float *wr = Wr + (size_t)e * H;
    for (int h = 0; h < H; ++h) s += x[h] * (double)wr[h];
    l[e] = s + (bias ? (double)bias[e] : 0.0);
  }
}

/* top-k of one token's logits, slots in descending order, weights = softmax over the selected set */
static void topk_one(const double *l, int E, int k, int32_t *idx, double *w, double *gap, scored *buf) {
  for (int e = 0; e < E; ++e) { buf[e].l = l[e]; buf[e].e = e; }
  qsort(buf, (size_t)E, sizeof(scored), by_logit_desc);
  double lmax = buf[0].l, z = 0.0;
  for (int j = 0; j < k; ++j) { idx[j] = buf[j].e; z += exp(buf[j].l - lmax); }
  for (int j = 0; j < k; ++j) w[j] = exp(buf[j].l - lmax) / z;
  if (gap) *gap = (k < E) ? buf[k - 1].l - buf[k].l : INFINITY;
}

/* weights of a given (forced) selection: softmax of the oracle's logits over that set */
static void forced_weights(const double *l, int k, const int32_t *idx, double *w) {
  double lmax = -INFINITY, z = 0.0;
  for (int j = 0; j < k; ++j) lmax = fmax(lmax, l[idx[j]]);
  for (int j = 0; j < k; ++j) z += exp(l[idx[j]] - lmax);
  for (int j = 0; j < k; ++j) w[j] = exp(l[idx[j]] - lmax) / z;
}

void oracle_router_topk(const uint16_t *x, int T, int H, const float *Wr, const float *bias, int E, int k,
                        int32_t *idx, double *w, double *logits_out, double *gap_out, int nthreads) {
#ifdef _OPENMP
  if (nthreads > 0) omp_set_num_threads(nthreads);
#pragma omp parallel for schedule(dynamic, 1)
#endif
  for (int t = 0; t < T; ++t) {
    double *xd = (double *)malloc(sizeof(double) * (size_t)H);
    double *l = (double *)malloc(sizeof(double) * (size_t)E);
    scored *buf = (scored *)malloc(sizeof(scored) * (size_t)E);
    for (int h = 0; h < H; ++h) xd[h] = oracle_bf16_to_double(x[(size_t)t * H + h]);
    router_logits(xd, H, Wr, bias, E, l);
    topk_one(l, E, k, idx + (size_t)t * k, w + (size_t)t * k, gap_out ? gap_out + t : NULL, buf);
    if (logits_out) memcpy(logits_out + (size_t)t * E, l, sizeof(double) * (size_t)E);
    free(xd); free(l); free(buf);
  }
}

/* ---------------------------------------------------------------- permutation */

/* stable counting sort of the T*k (token, slot) pairs by expert:
 *   counts[e]   = number of pairs routed to e
 *   offsets     = exclusive scan of counts (E+1 entries)
 *   row_of[f]   = destination row of pair f = t*k + j
 *   src[row]    = token of the pair stored at `row` (rows of one expert are in token order) */
void oracle_permute(const int32_t *idx, int T, int k, int E, int32_t *counts, int32_t *offsets,
                    int32_t *row_of, int32_t *src) {
  for (int e = 0; e < E; ++e) counts[e] = 0;
  for (int f = 0; f < T * k; ++f) counts[idx[f]]++;
  offsets[0] = 0;
  for (int e = 0; e < E; ++e) offsets[e + 1] = offsets[e] + counts[e];
  int32_t *cursor = (int32_t *)malloc(sizeof(int32_t) * (size_t)(E > 0 ? E : 1));
  for (int e = 0; e < E; ++e) cursor[e] = offsets[e];
  for (int f = 0; f < T * k; ++f) {
    int row = cursor[idx[f]]++;
    row_of[f] = row;
    src[row] = f / k;
  }
  free(cursor);
}

/* ---------------------------------------------------------------- expert FFN */

/* out = W_down[e] (silu(W_gate[e] x) * (W_up[e] x)), one token, fp64; silu(z) = z / (1 + e^-z) */
static void ffn_one(const oq_mat *g, const oq_mat *u, const oq_mat *d, int e, const double *x, int H, int I,
                    double *out, double *hbuf, double *row, int mirrored) {
  for (int i = 0; i < I; ++i) {
    double gs = 0.0, us = 0.0;
    dequant_row(g, e, i, row, mirrored);
    for (int h = 0; h < H; ++h) gs += row[h] * x[h];
    dequant_row(u, e, i, row, mirrored);
    for (int h = 0; h < H; ++h) us += row[h] * x[h];
    double hv = gs / (1.0 + exp(-gs)) * us;
    hbuf[i] = mirrored ? round_f16(hv) : hv;
  }
  for (int n = 0; n < H; ++n) {
    double s = 0.0;
    dequant_row(d, e, n, row, mirrored);
    for (int i = 0; i < I; ++i) s += row[i] * hbuf[i];
    out[n] = mirrored ? round_f16(s) : s;
  }
}

/* one expert applied to rows of an fp64 input matrix (test hook for dense-vs-sparse checks) */
void oracle_expert_ffn_rows(const oq_mat *g, const oq_mat *u, const oq_mat *d, int e, const double *x, int nrows,
                            int H, int I, double *out, int mirrored) {
  double *hbuf = (double *)malloc(sizeof(double) * (size_t)I);
  double *row = (double *)malloc(sizeof(double) * (size_t)(H > I ? H : I));
  for (int r = 0; r < nrows; ++r) ffn_one(g, u, d, e, x + (size_t)r * H, H, I, out + (size_t)r * H, hbuf, row, mirrored);
  free(hbuf); free(row);
}

/* ---------------------------------------------------------------- layer forward */

/* y[t] = sum_j w_{t,j} FFN_{idx_{t,j}}(x_t) + FFN_shared(x_t) + residual[t]
 *   x: bf16 [T,H]; Wr fp32 [E,H]; bias fp32 [E] or NULL; routed: gate/up [E][I][H], down [E][H][I];
 *   shared (NULL if none): one expert, same shapes; residual fp32 [T,H] or NULL.
 *   forced_idx: NULL to route; otherwise the [T,k] selection to use (weights then come from the
 *   oracle's own logits restricted to that selection).
 *   Outputs: y fp64 [T,H]; idx [T,k]; w fp64 [T,k]; gap fp64 [T] (k-th minus (k+1)-th logit). */
void oracle_layer_forward(const uint16_t *x, int T, int H, const float *Wr, const float *bias, int E, int k, int I,
                          const oq_mat *rg, const oq_mat *ru, const oq_mat *rd,
                          const oq_mat *sg, const oq_mat *su, const oq_mat *sd,
                          const float *residual, const int32_t *forced_idx,
                          double *y, int32_t *idx, double *w, double *gap, int mirrored, int nthreads) {
#ifdef _OPENMP
  if (nthreads > 0) omp_set_num_threads(nthreads);
#pragma omp parallel for schedule(dynamic, 1)
#endif
  for (int t = 0; t < T; ++t) {
    double *xd = (double *)malloc(sizeof(double) * (size_t)H);
    double *xe = (double *)malloc(sizeof(double) * (size_t)H);
    double *l = (double *)malloc(sizeof(double) * (size_t)E);
    scored *buf = (scored *)malloc(sizeof(scored) * (size_t)E);
    double *o = (double *)malloc(sizeof(double) * (size_t)H);
    double *hbuf = (double *)malloc(sizeof(double) * (size_t)I);
    double *row = (double *)malloc(sizeof(double) * (size_t)(H > I ? H : I));
    int32_t *ti = idx + (size_t)t * k;
    double *tw = w + (size_t)t * k;
    double *ty = y + (size_t)t * H;

    for (int h = 0; h < H; ++h) xd[h] = oracle_bf16_to_double(x[(size_t)t * H + h]);
    router_logits(xd, H, Wr, bias, E, l);
    if (forced_idx) {
      for (int j = 0; j < k; ++j) ti[j] = forced_idx[(size_t)t * k + j];
      forced_weights(l, k, ti, tw);
      if (gap) gap[t] = NAN;
    } else {
      topk_one(l, E, k, ti, tw, gap ? gap + t : NULL, buf);
    }
    /* the expert inputs: x itself, or fp16(x) in mirrored mode */
    for (int h = 0; h < H; ++h) xe[h] = mirrored ? round_f16(xd[h]) : xd[h];
    for (int h = 0; h < H; ++h) ty[h] = residual ? (double)residual[(size_t)t * H + h] : 0.0;
    for (int j = 0; j < k; ++j) {
      ffn_one(rg, ru, rd, ti[j], xe, H, I, o, hbuf, row, mirrored);
      for (int h = 0; h < H; ++h) ty[h] += tw[j] * o[h];
    }
    if (sg) {
      ffn_one(sg, su, sd, 0, xe, H, I, o, hbuf, row, mirrored);
      for (int h = 0; h < H; ++h) ty[h] += o[h];
    }
    free(xd); free(xe); free(l); free(buf); free(o); free(hbuf); free(row);
  }
}

int oracle_max_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}
