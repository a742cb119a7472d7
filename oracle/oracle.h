/*
 * oracle.h -- plain fp64 CPU reference of the hybrid Gated-DeltaNet +
 * full-attention decoder (TEST INFRASTRUCTURE ONLY).
 *
 * Only the test suite, the smoke check and the benchmark's CPU-baseline leg
 * may load this library.  It shares no code, header, table or helper with
 * the CUDA engine; both sides receive the same seeded bf16 weights and token
 * streams as plain bytes.
 *
 * Precision: every activation, state and accumulation is a C double.  Weights
 * are read as bf16 bit patterns and widened exactly.  The attention KV cache
 * holds bf16-rounded values, because the model stores its KV cache in bf16.
 */
#ifndef MK_ORACLE_H
#define MK_ORACLE_H
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define ORC_MAX_LAYERS 64

typedef struct {
  int32_t n_layers;
  int32_t layer_is_attn[ORC_MAX_LAYERS];
  int32_t hidden, vocab, mlp;
  int32_t dn_heads, dn_dk, dn_dv, conv_k;
  int32_t q_heads, kv_heads, head_dim;
  double rope_theta, rms_eps;
  int32_t max_ctx;
} orc_config;

/* One layer's weights; bf16 tensors are uint16 bit patterns, row-major
 * [out][in].  Unused members (attention members of a DeltaNet layer and
 * vice versa) may be NULL. */
typedef struct {
  const uint16_t *attn_norm;                  /* [H]                       */
  const uint16_t *in_proj;                    /* DN [q|k|v|z|b|a][H]       */
  const uint16_t *conv_w;                     /* DN [q|k|v channels][K]    */
  const float *A_log, *dt_bias;               /* DN [heads] (fp32)         */
  const uint16_t *out_norm;                   /* DN [dv]                   */
  const uint16_t *out_proj;                   /* DN [H][heads*dv]          */
  const uint16_t *w_q, *w_k, *w_v, *w_o;      /* attention                 */
  const uint16_t *mlp_norm;                   /* [H]                       */
  const uint16_t *w_gate, *w_up, *w_down;     /* [I][H], [I][H], [H][I]    */
} orc_layer;

typedef struct orc_model orc_model;

/* ---- scalar / vector primitives (exported so the tests can pin them) ---- */
double orc_bf16_to_double(uint16_t b);
uint16_t orc_double_to_bf16(double x);
double orc_sigmoid(double x);
double orc_softplus(double x);
double orc_silu(double x);
void orc_gemv(const uint16_t *W, int rows, int cols, const double *x, double *y);
void orc_quantize_w4(const uint16_t *W, int rows, int cols, uint8_t *codes, float *scales);
void orc_dequantize_w4(const uint8_t *codes, const float *scales, int rows, int cols,
                       double *Wd);
void orc_gemv_w4(const uint8_t *codes, const float *scales, int rows, int cols, const double *x,
                 double *y);
void orc_rmsnorm(const double *x, const uint16_t *w, int n, double eps, double *y);
void orc_l2norm(const double *x, int n, double eps, double *y);
void orc_causal_conv_step(int channels, int K, const uint16_t *w, double *state,
                          const double *u, double *out);
void orc_gated_delta_step(int dk, int dv, double *S, const double *q,
                          const double *k, const double *v, double alpha,
                          double beta, double *o);
void orc_delta_sequence(int dk, int dv, int steps, double *S, const double *q,
                        const double *k, const double *v, const double *alpha,
                        const double *beta, double *o);
void orc_rope(double *x, int hd, int pos, double theta);
void orc_softmax(const double *s, int n, double *p);
void orc_attention_head(const double *q, const double *K, const double *V,
                        int n, int hd, double *o);

/* ---- the model ---- */
orc_model *orc_create(const orc_config *cfg, const orc_layer *layers,
                      const uint16_t *embed, const uint16_t *final_norm);
orc_model *orc_clone(const orc_model *m);
void orc_destroy(orc_model *m);
/* Threads the independent GEMV rows may use (OpenMP; n <= 0: all cores).
 * Only changes how fast the oracle runs, never what it computes. */
void orc_set_threads(int n);
void orc_reset(orc_model *m);
int orc_pos(const orc_model *m);
/* One token through the whole stack at position orc_pos(); logits [V] and
 * hidden [n_layers][H] (residual stream after each layer) may be NULL.
 * Returns 0, or -1 when the KV cache is full or the token is out of range. */
int orc_step(orc_model *m, int token, double *logits, double *hidden);
/* dn [n_dn][heads][dv][dk], conv [n_dn][channels][K-1] */
void orc_get_state(const orc_model *m, double *dn, double *conv);
/* Install a state as if `pos` tokens had been consumed: dn/conv as above
 * (float32), k/v caches [n_attn][kv_heads][pos][hd] bf16. */
int orc_set_state(orc_model *m, int pos, const float *dn, const float *conv,
                  const uint16_t *k_cache, const uint16_t *v_cache);

#ifdef __cplusplus
}
#endif
#endif
