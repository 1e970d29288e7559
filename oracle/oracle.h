/*
 * CPU oracle for one auto-regressive decode step of a decoder-only transformer.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the
 * benchmark's CPU-baseline leg may call this code; the GPU path never does.
 *
 * It is the "independent mid-state test oracle" of ForgeMegakernel (arXiv
 * 2609.12379, abstract): it derives every intermediate state of the step
 * (hidden state after attention and after the MLP of every layer, the K/V rows
 * appended to the cache, router logits and expert choices, logits) so that a
 * decode kernel can be checked state by state.  The pages name the operations
 * of the step but print no formula for any of them; each function below
 * therefore writes out the standard textbook definition of its operation and
 * says which one.
 *
 * Arithmetic: weights and the KV cache are stored as bfloat16; every other
 * quantity is IEEE double, accumulated sequentially in index order.  A K/V row
 * is rounded to bfloat16 (round to nearest even) when it is appended, and the
 * step then attends over the rounded row, exactly as over any cached row.
 *
 * Layouts (row-major, element counts):
 *   weight matrices           [out][in]            (y = W x)
 *   KV cache of one layer     [B][n_kv][max_ctx][head_dim]
 *   KV cache of the model     [L][B][n_kv][max_ctx][head_dim]
 *   MoE expert gate/up        [expert_ffn][hidden], down [hidden][expert_ffn]
 */
#ifndef MK_ORACLE_H
#define MK_ORACLE_H
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct ora_desc {
  int n_layers, hidden, n_q_heads, n_kv_heads, head_dim, ffn_dim, vocab;
  int n_experts, top_k, expert_ffn_dim; /* n_experts == 0: dense SwiGLU MLP */
  int qk_norm;                          /* per-head RMSNorm of q and k before RoPE */
  int batch, max_ctx;
  double rms_eps, rope_theta;
  int fp8_block; /* > 0: the layers' projections are fp8 (ora_layer.*8) with one scale per row per
                    fp8_block columns; 0: bf16 */
} ora_desc;

/* An fp8 weight matrix: E4M3 codes [out][in] and fp32 scales [out][ceil(in / fp8_block)]. */
typedef struct ora_fp8 {
  const uint8_t* codes;
  const float* scale;
} ora_fp8;

typedef struct ora_layer {
  const uint16_t *attn_norm, *wq, *wk, *wv, *q_norm, *k_norm, *wo, *mlp_norm;
  const uint16_t *w_gate, *w_up, *w_down; /* dense MLP; unused for MoE */
  const uint16_t *router;                 /* [n_experts][hidden]; MoE only */
  /* fp8 forms of wq wk wv wo and of the dense gate / up / down (ora_desc.fp8_block > 0): they then
     replace the bf16 matrices; norms, router, experts, embedding and LM head stay bf16 */
  ora_fp8 wq8, wk8, wv8, wo8, gate8, up8, down8;
} ora_layer;

/* Returns expert weights on demand: which = 0 gate, 1 up, 2 down. */
typedef const uint16_t* (*ora_expert_fn)(void* ctx, int layer, int expert, int which);

typedef struct ora_model {
  ora_desc d;
  const uint16_t *embed, *final_norm, *lm_head; /* lm_head may equal embed (tied) */
  const ora_layer* layers;                      /* [n_layers] */
  ora_expert_fn expert;
  void* expert_ctx;
} ora_model;

/* ---- bfloat16 <-> double --------------------------------------------------- */
double ora_bf16_to_double(uint16_t h);
uint16_t ora_double_to_bf16(double x); /* round to nearest even, directly from double */

/* ---- primitives (exported so that the tests can pin each one) ------------- */
void ora_rmsnorm(const double* x, int n, const uint16_t* gain, double eps, double* out);
void ora_rope(double* v, int head_dim, int pos, double theta);
void ora_gemv(const uint16_t* w, int rows, int cols, const double* x, double* y);
double ora_silu(double z);
void ora_attention(const double* q, const uint16_t* k, const uint16_t* v, int n, int head_dim, double* out,
                   double* probs);
void ora_swiglu(const uint16_t* w_gate, const uint16_t* w_up, const uint16_t* w_down, int ffn, int hidden,
                const double* xn, double* y);
void ora_topk(const double* logits, int n, int k, int32_t* sel, double* w);

/* ---- low-bit weights (fp8 / nvfp4 weight streaming) -------------------------------------------- */
/* The decode step runs wq, wk, wv, wo and the dense gate / up / down in fp8 when ora_desc.fp8_block
 * is set (a MoE model with fp8_block set is refused); nvfp4 is used by ora_gemv_nvfp4 only. */
/* Exact decodes to double.  E4M3 is the OCP 8-bit floating-point format (sign, 4 exponent bits with
 * bias 7, 3 mantissa bits; exponent 0 is subnormal; 0x7F and 0xFF are NaN; no infinities; largest
 * finite 448).  E2M1 is the OCP 4-bit format of the low nibble (sign, 2 exponent bits with bias 1,
 * 1 mantissa bit; magnitudes 0, 0.5, 1, 1.5, 2, 3, 4, 6). */
double ora_e4m3_to_double(uint8_t code);
double ora_e2m1_to_double(uint8_t nibble);
/* fp8 weights with block scales: W[r][c] = e4m3(w[r][c]) * scale[r][c / block] (scale fp32
 * [rows][ceil(cols / block)]); y_r = sum_c W[r][c] x_c in column order. */
void ora_gemv_fp8(const uint8_t* w, const float* scale, int rows, int cols, int block, const double* x, double* y);
/* nvfp4 weights: two E2M1 codes per byte (column 2j in the low nibble, 2j + 1 in the high one),
 * one E4M3 scale per 16 columns (scale [rows][cols / 16]) and one fp32 scale for the whole matrix:
 * W[r][c] = e2m1(code) * e4m3(scale[r][c / 16]) * tensor_scale.  cols is a multiple of 16. */
void ora_gemv_nvfp4(const uint8_t* w, const uint8_t* scale, float tensor_scale, int rows, int cols,
                    const double* x, double* y);

/* ---- one layer and one step ------------------------------------------------ */
/*
 * x: [B][hidden], the layer's input residual on entry and its output on return.
 * k_cache / v_cache: this layer's cache [B][n_kv][max_ctx][head_dim]; the new
 * token's K/V row is written at index seq_lens[b].
 * Optional outputs (NULL to skip): h_attn [B][hidden] residual after the
 * attention block; router_logits [B][n_experts], sel [B][top_k], sel_w [B][top_k].
 * Returns 0, or -1 on an out-of-range position / length.
 */
int ora_layer_forward(const ora_model* m, int layer, double* x, uint16_t* k_cache, uint16_t* v_cache,
                      const int32_t* positions, const int32_t* seq_lens, double* h_attn, double* router_logits,
                      int32_t* sel, double* sel_w);

/*
 * Whole step.  Caches are the model's [L][B][n_kv][max_ctx][head_dim].
 * Optional dumps (NULL to skip): h_attn, h_mlp [L][B][hidden];
 * router_logits [L][B][n_experts]; sel [L][B][top_k]; sel_w [L][B][top_k];
 * logits [B][vocab].
 */
int ora_decode_step(const ora_model* m, uint16_t* k_cache, uint16_t* v_cache, const int32_t* tokens,
                    const int32_t* positions, const int32_t* seq_lens, double* h_attn, double* h_mlp,
                    double* router_logits, int32_t* sel, double* sel_w, double* logits);

/* Final RMSNorm and LM head of one residual row: logits[vocab]. */
void ora_lm_head(const ora_model* m, const double* x, double* logits);

#ifdef __cplusplus
}
#endif
#endif
