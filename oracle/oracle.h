/*
 * oracle.h -- fp64 CPU reference for one batch-1 decode step of a Llama-style
 * decoder with an optional top-k MoE FFN.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test suite, the smoke check and the
 * benchmark's CPU-baseline leg may load this library.  It shares no code,
 * header, table or constant with the CUDA library; the two meet only in the
 * seeded input generator.
 *
 * What it computes: the plain definition of the decoder forward that the
 * megakernel pages speed up (epic-kernel README, "3B model support" -- Llama
 * 3.2 shapes -- and "Mixtral 8x7B MoE for batch-1 inference"; the Hyperkernel
 * teardown, "What a megakernel buys": a megakernel evaluates the same forward
 * pass in one launch).  Weights and KV cache are bf16 bit patterns (uint16);
 * every product and sum is in double.
 *
 * Every building block and the whole step are pinned by the CPU tests to
 * closed forms, brute force, special cases and an independent fp32
 * restatement; none is parity unpinned.
 */
#ifndef ORC_ORACLE_H
#define ORC_ORACLE_H
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct {
    int n_layers, hidden, n_heads, n_kv_heads, head_dim, ffn, vocab;
    int n_experts; /* 0 = dense FFN */
    int top_k;
    int max_seq;   /* KV cache positions per (layer, kv head) */
    double rms_eps, rope_theta;
} orc_shape;

/* Per-layer pointer arrays have n_layers entries; expert weights have
 * n_layers * n_experts entries, layer-major ([l * n_experts + e]). */
typedef struct {
    const uint16_t *embed;      /* [vocab, hidden] */
    const uint16_t *lm_head;    /* [vocab, hidden] */
    const uint16_t *final_norm; /* [hidden] */
    const uint16_t *const *attn_norm, *const *wq, *const *wk, *const *wv, *const *wo, *const *ffn_norm;
    const uint16_t *const *w_gate, *const *w_up, *const *w_down; /* [ffn,hidden],[ffn,hidden],[hidden,ffn] */
    const uint16_t *const *router;                               /* [n_experts, hidden] (MoE only) */
} orc_weights;

/* Building blocks (exposed so the tests can pin each one on its own). */
double orc_bf16_to_double(uint16_t b);
uint16_t orc_bf16_from_double(double v);
void orc_rmsnorm(const double *x, const uint16_t *w, int n, double eps, double *out);
void orc_gemv(const uint16_t *W, int rows, int cols, const double *x, double *y);
void orc_rope(double *v, int n_heads, int head_dim, int pos, double theta);
void orc_softmax(const double *s, int n, double *p);
void orc_attend(const double *q, const uint16_t *K, const uint16_t *V, int n, int head_dim, double *out);
double orc_silu(double z);
void orc_topk(const double *r, int n_experts, int k, int *idx, double *w);
int orc_argmax(const double *v, int n);

/* One decode step at position `pos` for input token `token`.
 * kcache/vcache: bf16 [n_layers][n_kv_heads][max_seq][head_dim]; positions
 * < pos are read, position pos is written (append).
 * logits: [vocab] out.  hidden: [(n_layers+1) * hidden] out or NULL (x after
 * the embedding and after every layer).  router_idx / router_w:
 * [n_layers * top_k] out or NULL (MoE only).  Returns the argmax token
 * (lowest index on ties), or -1 on bad arguments. */
int orc_decode_step(const orc_shape *s, const orc_weights *w, uint16_t *kcache, uint16_t *vcache, int token,
                    int pos, double *logits, double *hidden, int *router_idx, double *router_w);

/* Speculative expert prediction for MoE layer `layer`: the top_k experts
 * (best first) that the layer's router gives the layer's attention input,
 * rmsnorm(x) with the attention norm weights, where x is the residual entering
 * the layer (hidden[layer] of orc_decode_step).  The expert choice that the
 * FFN of the layer makes applies the same router to the residual after
 * attention, normalised with the FFN norm weights; the prediction reads the
 * residual before attention (epic-kernel README, "Speculative expert
 * prediction").  The pages do not give the predictor's form: this is the
 * plainest reading, the layer's own router on the pre-attention normalised
 * residual.  Returns 0, or -1 on bad arguments. */
int orc_predict_experts(const orc_shape *s, const orc_weights *w, int layer, const double *x, int *idx);

int orc_num_threads(void);

#ifdef __cplusplus
}
#endif
#endif
