/*
 * oracle.h -- plain, slow CPU oracle for one Llama-style decoder step.
 *
 * TEST INFRASTRUCTURE ONLY.  Only tests/, __graft_entry__.smoke() and bench.py's
 * cpu_baseline / reference arm may load this library.  It shares no code with the
 * CUDA library (no headers, helpers or tables) and neither side includes the other.
 *
 * What it computes follows the pages:
 *   - decoder step: the computation graph of one LLM decode step that MPK lowers into a
 *     task graph ("Compiler des LLM en MegaKernel ...", Part 1 "Compilateur"), with
 *     the 8B decode workload of "Valeur clé de MPK";
 *   - RMSNorm + linear and the gated MLP: Mirage article (iaiol.com), "Case 1:
 *     Normalization + Linear" and "Case 3: Gated MLP";
 *   - attention O = softmax(Q K) V: Mirage article, the attention example (Q [64,1,128],
 *     K [64,128,4096], V [64,4096,128], fp16);
 *   - optional QK-norm: a LayerNorm on every query and key head before attention, Mirage
 *     article, "Case 4.1: Attention with Query-Key Normalization" (Chameleon, ViT-22B).
 * Where the pages are silent (RoPE pairing, scale, GQA grouping, precision), the
 * readings are stated next to each function in oracle.cpp.
 *
 * Precision: activations are fp32 (T = float) or fp64 (T = double, the "f64" mode used
 * to pin the fp32 mode); weights are bf16 widened exactly; every dot product, norm and
 * softmax accumulates in double.  With kv_round = 1 the K/V cache stores bf16-rounded
 * values (round to nearest even), as the configs' bf16 cache requires.
 *
 * All entry points return 0 on success and a negative number on bad arguments.
 */
#ifndef MK_ORACLE_H
#define MK_ORACLE_H
#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct or_config {
  int n_layers, hidden, n_q_heads, n_kv_heads, head_dim, ffn, vocab;
  double rms_eps, rope_theta;
} or_config;

/* Host bf16 bit patterns, canonical [out, in] row-major.  Per-layer arrays have
 * n_layers entries.  The oracle keeps the pointers; the caller keeps the memory alive. */
typedef struct or_weights {
  const uint16_t* embed;      /* [vocab, hidden] */
  const uint16_t* lm_head;    /* [vocab, hidden] */
  const uint16_t* final_norm; /* [hidden] */
  const uint16_t* const* attn_norm; /* [hidden] */
  const uint16_t* const* wq;  /* [n_q_heads*head_dim, hidden] */
  const uint16_t* const* wk;  /* [n_kv_heads*head_dim, hidden] */
  const uint16_t* const* wv;  /* [n_kv_heads*head_dim, hidden] */
  const uint16_t* const* wo;  /* [hidden, n_q_heads*head_dim] */
  const uint16_t* const* mlp_norm; /* [hidden] */
  const uint16_t* const* wg;  /* [ffn, hidden] */
  const uint16_t* const* wu;  /* [ffn, hidden] */
  const uint16_t* const* wd;  /* [hidden, ffn] */
  /* QK-norm (NULL arrays = the model has none): LayerNorm gain and bias of every query head
   * ([n_q_heads*head_dim], head h at h*head_dim) and key head ([n_kv_heads*head_dim]). */
  const uint16_t* const* q_norm_w;
  const uint16_t* const* q_norm_b;
  const uint16_t* const* k_norm_w;
  const uint16_t* const* k_norm_b;
} or_weights;

typedef struct or_state or_state;

/* f64: 0 = fp32 activations, 1 = fp64 activations.  kv_round: 1 = store K/V as bf16. */
or_state* or_create(const or_config* cfg, const or_weights* w, int batch, int max_seq, int f64, int kv_round);
void or_destroy(or_state* s);
void or_set_threads(int n); /* row-parallel worker count (results do not depend on it) */

/* Prefill T tokens per sequence (tokens [batch][T]) from the current positions; writes the
 * last position's logits [batch][vocab] (may be NULL). */
int or_prefill(or_state* s, const int32_t* tokens, int T, float* last_logits);
/* One decode step: token[b] at position pos[b]; logits [batch][vocab]; positions advance. */
int or_decode(or_state* s, const int32_t* tokens, float* logits);
/* Logits as double (fp64 mode keeps full precision); same semantics as or_decode. */
int or_decode_f64(or_state* s, const int32_t* tokens, double* logits);
/* Replace the cache with caller bf16 values in the layout [layer][K|V][seq][kv_head][pos][head_dim]
 * holding `length` positions, and set every position to `length`. */
int or_set_cache(or_state* s, const uint16_t* kv, int length);
/* Copy the cache out as bf16 bits (fp32 values rounded RNE; exact when kv_round = 1),
 * same layout with `length` positions. */
int or_get_cache(const or_state* s, uint16_t* kv, int length);
/* Set each sequence's position (0..max_seq): the next token of sequence b goes to pos[b] and
 * attends to cache entries 0..pos[b].  Entries at or past pos[b] are ignored and overwritten. */
int or_set_positions(or_state* s, const int32_t* pos);
int or_position(const or_state* s, int b);
/* Greedy pick: index of the largest logit, the lowest index among equal values. */
int or_argmax(const float* logits, int n);
/* The query and key vectors (after QK-norm, if any, and RoPE; before the bf16 rounding of the
 * cache) that layer `layer` computed for the last token of each sequence in the last
 * prefill or decode call: q [batch][n_q_heads*head_dim], k [batch][n_kv_heads*head_dim]. */
int or_get_qk(const or_state* s, int layer, double* q, double* k);

/* ---- single operations (the pieces the decoder step is made of), fp64 I/O ---- */
void or_rmsnorm(const double* x, const double* g, int n, double eps, double* y);
/* LayerNorm: y = (x - mean(x)) / sqrt(var(x) + eps) * g + b, var the mean squared deviation. */
void or_layernorm(const double* x, const double* g, const double* b, int n, double eps, double* y);
void or_matvec_bf16(const uint16_t* W, const double* x, int rows, int cols, double* y);
void or_rope(double* v, int head_dim, int pos, double theta);
void or_rope_cos_sin(int head_dim, int pos, double theta, float* cos_out, float* sin_out);
/* One query head over L keys: scores = scale*q.k_j, p = softmax(scores), o = sum p_j v_j.
 * k, v: [L][d] doubles.  probs may be NULL. */
void or_attention_head(const double* q, const double* k, const double* v, int L, int d, double scale, double* o,
                       double* probs);
double or_silu(double z);

/* Standalone decode attention in the Mirage example's form, fp64 brute force:
 * q [BH][d] fp16, k_t [BH][d][L] fp16 (key index fastest), v [BH][L][d] fp16,
 * o [BH][d] = softmax(scale * q K) V.  Returns 0. */
int or_attention_decode_f16(const uint16_t* q, const uint16_t* k_t, const uint16_t* v, int BH, int d, int L,
                            double scale, double* o);

#ifdef __cplusplus
}
#endif
#endif
