/*
 * CPU oracle for one auto-regressive decode step (see oracle.h).
 *
 * TEST INFRASTRUCTURE ONLY: called by the tests, the smoke check and the
 * benchmark's CPU-baseline leg, never by the GPU path.  It shares no code with
 * the GPU path; the only thing both sides share is the seeded input generator.
 *
 * Plain, single-threaded, fp64.  No blocking, fusion or reordering: each
 * function is the definition of its operation written out in the order a
 * reader would check it by hand.
 */
#include "oracle.h"

#include <math.h>
#include <stdlib.h>
#include <string.h>

/* ---------------------------------------------------------------------------
 * bfloat16: the top 16 bits of an IEEE binary32.  Widening is exact.
 * Narrowing rounds the double directly to the nearest bfloat16 (ties to even),
 * by scaling the value so that the bfloat16 grid becomes the integers and
 * taking rint() (the default rounding mode is round-to-nearest-even).
 * ------------------------------------------------------------------------- */
double ora_bf16_to_double(uint16_t h) {
  union { uint32_t u; float f; } v;
  v.u = (uint32_t)h << 16;
  return (double)v.f;
}

uint16_t ora_double_to_bf16(double x) {
  union { uint32_t u; float f; } v;
  if (isnan(x)) return 0x7FC0;
  if (x == 0.0) return signbit(x) ? 0x8000 : 0x0000;
  int e;
  frexp(x, &e);              /* |x| in [2^(e-1), 2^e) */
  int ulp_exp = e - 1 - 7;   /* 8 significant bits */
  if (ulp_exp < -133) ulp_exp = -133; /* subnormal bfloat16 spacing 2^-133 */
  double r = ldexp(rint(ldexp(x, -ulp_exp)), ulp_exp);
  if (fabs(r) > 3.3895313892515355e38) r = copysign(INFINITY, x); /* beyond the largest bfloat16 */
  v.f = (float)r;            /* exact: r is on the bfloat16 grid */
  return (uint16_t)(v.u >> 16);
}

/* ---------------------------------------------------------------------------
 * RMSNorm (Zhang & Sennrich, 2019):  out_i = x_i / sqrt(mean_j x_j^2 + eps) * g_i
 * ------------------------------------------------------------------------- */
void ora_rmsnorm(const double* x, int n, const uint16_t* gain, double eps, double* out) {
  double ss = 0.0;
  for (int i = 0; i < n; ++i) ss += x[i] * x[i];
  double inv = 1.0 / sqrt(ss / n + eps);
  for (int i = 0; i < n; ++i) out[i] = x[i] * inv * ora_bf16_to_double(gain[i]);
}

/* ---------------------------------------------------------------------------
 * Rotary position embedding (Su et al., RoFormer, 2021), "rotate-half" pairing:
 * the pair (i, i + d/2) is rotated by the angle pos * theta^(-2i/d).
 * ------------------------------------------------------------------------- */
void ora_rope(double* v, int d, int pos, double theta) {
  int half = d / 2;
  for (int i = 0; i < half; ++i) {
    double ang = (double)pos * pow(theta, -2.0 * i / d);
    double c = cos(ang), s = sin(ang);
    double a = v[i], b = v[i + half];
    v[i] = a * c - b * s;
    v[i + half] = b * c + a * s;
  }
}

/* y_r = sum_c W[r][c] x_c, accumulated in column order. */
void ora_gemv(const uint16_t* w, int rows, int cols, const double* x, double* y) {
  for (int r = 0; r < rows; ++r) {
    const uint16_t* row = w + (size_t)r * cols;
    double acc = 0.0;
    for (int c = 0; c < cols; ++c) acc += ora_bf16_to_double(row[c]) * x[c];
    y[r] = acc;
  }
}

/* ---- low-bit weights ---------------------------------------------------------
 * The pages name fp8 and nvfp4 weight streams (per-block scales) without
 * fixing a block shape; the decodes below are the OCP 8-bit and 4-bit
 * floating-point definitions, written out field by field. */
double ora_e4m3_to_double(uint8_t code) {
  const int sign = code >> 7, e = (code >> 3) & 15, m = code & 7;
  if (e == 15 && m == 7) return NAN;
  const double mag = e == 0 ? ldexp((double)m / 8.0, 1 - 7) : ldexp(1.0 + (double)m / 8.0, e - 7);
  return sign ? -mag : mag;
}

double ora_e2m1_to_double(uint8_t nibble) {
  const int sign = (nibble >> 3) & 1, e = (nibble >> 1) & 3, m = nibble & 1;
  const double mag = e == 0 ? (double)m / 2.0 : ldexp(1.0 + (double)m / 2.0, e - 1);
  return sign ? -mag : mag;
}

void ora_gemv_fp8(const uint8_t* w, const float* scale, int rows, int cols, int block, const double* x, double* y) {
  const int nb = (cols + block - 1) / block;
  for (int r = 0; r < rows; ++r) {
    double acc = 0.0;
    for (int c = 0; c < cols; ++c)
      acc += ora_e4m3_to_double(w[(size_t)r * cols + c]) * (double)scale[(size_t)r * nb + c / block] * x[c];
    y[r] = acc;
  }
}

void ora_gemv_nvfp4(const uint8_t* w, const uint8_t* scale, float tensor_scale, int rows, int cols,
                    const double* x, double* y) {
  for (int r = 0; r < rows; ++r) {
    double acc = 0.0;
    for (int c = 0; c < cols; ++c) {
      const uint8_t byte = w[(size_t)r * (cols / 2) + c / 2];
      const double v = ora_e2m1_to_double(c % 2 ? byte >> 4 : byte & 15);
      acc += v * ora_e4m3_to_double(scale[(size_t)r * (cols / 16) + c / 16]) * (double)tensor_scale * x[c];
    }
    y[r] = acc;
  }
}

/* A layer's projection: its fp8 form when the model has one, else bf16. */
static void gemv_w(const ora_desc* d, const uint16_t* w, const ora_fp8* w8, int rows, int cols, const double* x,
                   double* y) {
  if (d->fp8_block > 0)
    ora_gemv_fp8(w8->codes, w8->scale, rows, cols, d->fp8_block, x, y);
  else
    ora_gemv(w, rows, cols, x, y);
}

/* SiLU (Hendrycks & Gimpel; Elfwing et al.): z * sigmoid(z) = z / (1 + e^-z). */
double ora_silu(double z) { return z / (1.0 + exp(-z)); }

/* ---------------------------------------------------------------------------
 * Scaled dot-product attention of one query over n cached positions
 * (Vaswani et al., 2017):  p_t = softmax_t(q . k_t / sqrt(d)),  out = sum_t p_t v_t.
 * k and v are [n][d] bfloat16; probs (optional) receives p.
 * ------------------------------------------------------------------------- */
void ora_attention(const double* q, const uint16_t* k, const uint16_t* v, int n, int d, double* out,
                   double* probs) {
  double* s = (double*)malloc(sizeof(double) * (size_t)(n > 0 ? n : 1));
  double scale = 1.0 / sqrt((double)d);
  double mx = -INFINITY;
  for (int t = 0; t < n; ++t) {
    double dot = 0.0;
    for (int i = 0; i < d; ++i) dot += q[i] * ora_bf16_to_double(k[(size_t)t * d + i]);
    s[t] = dot * scale;
    if (s[t] > mx) mx = s[t];
  }
  double den = 0.0;
  for (int t = 0; t < n; ++t) {
    s[t] = exp(s[t] - mx);
    den += s[t];
  }
  for (int i = 0; i < d; ++i) out[i] = 0.0;
  for (int t = 0; t < n; ++t) {
    double p = s[t] / den;
    if (probs) probs[t] = p;
    for (int i = 0; i < d; ++i) out[i] += p * ora_bf16_to_double(v[(size_t)t * d + i]);
  }
  free(s);
}

/* SwiGLU MLP (Shazeer, 2020):  y = W_down (silu(W_gate x) * (W_up x)). */
void ora_swiglu(const uint16_t* w_gate, const uint16_t* w_up, const uint16_t* w_down, int ffn, int hidden,
                const double* xn, double* y) {
  double* g = (double*)malloc(sizeof(double) * (size_t)ffn);
  double* u = (double*)malloc(sizeof(double) * (size_t)ffn);
  ora_gemv(w_gate, ffn, hidden, xn, g);
  ora_gemv(w_up, ffn, hidden, xn, u);
  for (int i = 0; i < ffn; ++i) g[i] = ora_silu(g[i]) * u[i];
  ora_gemv(w_down, hidden, ffn, g, y);
  free(g);
  free(u);
}

/* ---------------------------------------------------------------------------
 * Top-k routing (Shazeer et al., 2017, sparsely-gated mixture of experts):
 * pick the k largest router logits (a tie goes to the lower expert index),
 * listed from the largest down, and weight them by the softmax over the k
 * picked logits, which equals the full softmax renormalised over the picks.
 * ------------------------------------------------------------------------- */
void ora_topk(const double* logits, int n, int k, int32_t* sel, double* w) {
  unsigned char* taken = (unsigned char*)calloc((size_t)n, 1);
  for (int j = 0; j < k; ++j) {
    int best = -1;
    for (int e = 0; e < n; ++e) {
      if (taken[e]) continue;
      if (best < 0 || logits[e] > logits[best]) best = e; /* strict: equal keeps the lower index */
    }
    taken[best] = 1;
    sel[j] = best;
  }
  double mx = logits[sel[0]];
  double den = 0.0;
  for (int j = 0; j < k; ++j) den += exp(logits[sel[j]] - mx);
  for (int j = 0; j < k; ++j) w[j] = exp(logits[sel[j]] - mx) / den;
  free(taken);
}

/* ---------------------------------------------------------------------------
 * One decoder layer for every sequence of the batch (pre-norm residual block):
 *   h = x + W_o Attn(RoPE(q), cache + RoPE(k), v)      q,k,v = W_{q,k,v} RMSNorm(x)
 *   x' = h + MLP(RMSNorm(h))                             MLP = SwiGLU or top-k MoE
 * Grouped-query attention: query head j reads KV head floor(j / (n_q / n_kv)).
 * The new token sits at cache index seq_lens[b] and is rotated to positions[b].
 * ------------------------------------------------------------------------- */
int ora_layer_forward(const ora_model* m, int layer, double* x, uint16_t* k_cache, uint16_t* v_cache,
                      const int32_t* positions, const int32_t* seq_lens, double* h_attn, double* router_logits,
                      int32_t* sel, double* sel_w) {
  const ora_desc* d = &m->d;
  /* fp8 weights are modelled for the attention projections and the dense MLP only: a MoE model
   * with fp8_block set has no fp8 router or experts to run, so it is refused rather than run in bf16 */
  if (d->fp8_block > 0 && d->n_experts > 0) return -1;
  const ora_layer* W = &m->layers[layer];
  const int H = d->hidden, hd = d->head_dim, nq = d->n_q_heads, nkv = d->n_kv_heads, T = d->max_ctx;
  const int group = nq / nkv;
  double* xn = (double*)malloc(sizeof(double) * (size_t)H);
  double* q = (double*)malloc(sizeof(double) * (size_t)nq * hd);
  double* k = (double*)malloc(sizeof(double) * (size_t)nkv * hd);
  double* v = (double*)malloc(sizeof(double) * (size_t)nkv * hd);
  double* att = (double*)malloc(sizeof(double) * (size_t)nq * hd);
  double* o = (double*)malloc(sizeof(double) * (size_t)H);
  double* tmp = (double*)malloc(sizeof(double) * (size_t)hd);
  int rc = 0;

  for (int b = 0; b < d->batch; ++b) {
    double* xb = x + (size_t)b * H;
    const int S = seq_lens[b], pos = positions[b];
    if (S < 0 || S >= T || pos < 0) { rc = -1; break; }

    /* attention block */
    ora_rmsnorm(xb, H, W->attn_norm, d->rms_eps, xn);
    gemv_w(d, W->wq, &W->wq8, nq * hd, H, xn, q);
    gemv_w(d, W->wk, &W->wk8, nkv * hd, H, xn, k);
    gemv_w(d, W->wv, &W->wv8, nkv * hd, H, xn, v);
    for (int h = 0; h < nq; ++h) {
      if (d->qk_norm) {
        ora_rmsnorm(q + (size_t)h * hd, hd, W->q_norm, d->rms_eps, tmp);
        memcpy(q + (size_t)h * hd, tmp, sizeof(double) * hd);
      }
      ora_rope(q + (size_t)h * hd, hd, pos, d->rope_theta);
    }
    for (int h = 0; h < nkv; ++h) {
      if (d->qk_norm) {
        ora_rmsnorm(k + (size_t)h * hd, hd, W->k_norm, d->rms_eps, tmp);
        memcpy(k + (size_t)h * hd, tmp, sizeof(double) * hd);
      }
      ora_rope(k + (size_t)h * hd, hd, pos, d->rope_theta);
      /* append the new row (bfloat16) at index S */
      size_t base = (((size_t)b * nkv + h) * T + S) * hd;
      for (int i = 0; i < hd; ++i) {
        k_cache[base + i] = ora_double_to_bf16(k[(size_t)h * hd + i]);
        v_cache[base + i] = ora_double_to_bf16(v[(size_t)h * hd + i]);
      }
    }
    for (int h = 0; h < nq; ++h) {
      int kvh = h / group;
      size_t base = (((size_t)b * nkv + kvh) * T) * hd;
      ora_attention(q + (size_t)h * hd, k_cache + base, v_cache + base, S + 1, hd, att + (size_t)h * hd, NULL);
    }
    gemv_w(d, W->wo, &W->wo8, H, nq * hd, att, o);
    for (int i = 0; i < H; ++i) xb[i] += o[i];
    if (h_attn) memcpy(h_attn + (size_t)b * H, xb, sizeof(double) * H);

    /* MLP block */
    ora_rmsnorm(xb, H, W->mlp_norm, d->rms_eps, xn);
    if (d->n_experts == 0) {
      if (d->fp8_block > 0) {  /* SwiGLU as ora_swiglu, on the fp8 matrices */
        double* gu = (double*)malloc(sizeof(double) * 2 * (size_t)d->ffn_dim);
        gemv_w(d, W->w_gate, &W->gate8, d->ffn_dim, H, xn, gu);
        gemv_w(d, W->w_up, &W->up8, d->ffn_dim, H, xn, gu + d->ffn_dim);
        for (int i = 0; i < d->ffn_dim; ++i) gu[i] = ora_silu(gu[i]) * gu[d->ffn_dim + i];
        gemv_w(d, W->w_down, &W->down8, H, d->ffn_dim, gu, o);
        free(gu);
      } else {
        ora_swiglu(W->w_gate, W->w_up, W->w_down, d->ffn_dim, H, xn, o);
      }
      for (int i = 0; i < H; ++i) xb[i] += o[i];
    } else {
      const int E = d->n_experts, K = d->top_k;
      double* r = (double*)malloc(sizeof(double) * (size_t)E);
      int32_t* s = (int32_t*)malloc(sizeof(int32_t) * (size_t)K);
      double* wsel = (double*)malloc(sizeof(double) * (size_t)K);
      double* acc = (double*)calloc((size_t)H, sizeof(double));
      ora_gemv(W->router, E, H, xn, r);
      ora_topk(r, E, K, s, wsel);
      for (int j = 0; j < K; ++j) {
        const uint16_t* g = m->expert(m->expert_ctx, layer, s[j], 0);
        const uint16_t* u = m->expert(m->expert_ctx, layer, s[j], 1);
        const uint16_t* dn = m->expert(m->expert_ctx, layer, s[j], 2);
        ora_swiglu(g, u, dn, d->expert_ffn_dim, H, xn, o);
        for (int i = 0; i < H; ++i) acc[i] += wsel[j] * o[i];
      }
      for (int i = 0; i < H; ++i) xb[i] += acc[i];
      if (router_logits) memcpy(router_logits + (size_t)b * E, r, sizeof(double) * E);
      if (sel) memcpy(sel + (size_t)b * K, s, sizeof(int32_t) * K);
      if (sel_w) memcpy(sel_w + (size_t)b * K, wsel, sizeof(double) * K);
      free(r);
      free(s);
      free(wsel);
      free(acc);
    }
  }
  free(xn); free(q); free(k); free(v); free(att); free(o); free(tmp);
  return rc;
}

void ora_lm_head(const ora_model* m, const double* x, double* logits) {
  const int H = m->d.hidden;
  double* xn = (double*)malloc(sizeof(double) * (size_t)H);
  ora_rmsnorm(x, H, m->final_norm, m->d.rms_eps, xn);
  ora_gemv(m->lm_head, m->d.vocab, H, xn, logits);
  free(xn);
}

/* ---------------------------------------------------------------------------
 * One decode step: embed the tokens, run every layer, final RMSNorm, LM head.
 * ------------------------------------------------------------------------- */
int ora_decode_step(const ora_model* m, uint16_t* k_cache, uint16_t* v_cache, const int32_t* tokens,
                    const int32_t* positions, const int32_t* seq_lens, double* h_attn, double* h_mlp,
                    double* router_logits, int32_t* sel, double* sel_w, double* logits) {
  const ora_desc* d = &m->d;
  const int H = d->hidden, B = d->batch, L = d->n_layers;
  const size_t layer_kv = (size_t)B * d->n_kv_heads * d->max_ctx * d->head_dim;
  double* x = (double*)malloc(sizeof(double) * (size_t)B * H);
  int rc = 0;
  for (int b = 0; b < B; ++b) {
    if (tokens[b] < 0 || tokens[b] >= d->vocab) { free(x); return -1; }
    const uint16_t* row = m->embed + (size_t)tokens[b] * H;
    for (int i = 0; i < H; ++i) x[(size_t)b * H + i] = ora_bf16_to_double(row[i]);
  }
  for (int l = 0; l < L && rc == 0; ++l) {
    const size_t lo = (size_t)l * B;
    rc = ora_layer_forward(m, l, x, k_cache + l * layer_kv, v_cache + l * layer_kv, positions, seq_lens,
                           h_attn ? h_attn + lo * H : NULL,
                           router_logits ? router_logits + lo * d->n_experts : NULL,
                           sel ? sel + lo * d->top_k : NULL, sel_w ? sel_w + lo * d->top_k : NULL);
    if (h_mlp) memcpy(h_mlp + lo * H, x, sizeof(double) * (size_t)B * H);
  }
  if (rc == 0 && logits)
    for (int b = 0; b < B; ++b) ora_lm_head(m, x + (size_t)b * H, logits + (size_t)b * d->vocab);
  free(x);
  return rc;
}
