/*
 * CPU oracle of the H-Spec block-parallel draft step -- TEST INFRASTRUCTURE ONLY.
 *
 * Plain, slow, obviously-correct C++17: every sum is accumulated in double, the
 * Mamba-2 state update is the sequential recurrence taken step by step, and paged
 * attention first copies the context out of the page pool into a contiguous buffer
 * and then runs a dense softmax over it.  Only the test-suite, the package smoke
 * check and the benchmark's CPU-baseline leg may load this library; the product
 * path (libhspec.so) shares no code, header, table or helper with it.
 *
 * Sources of what is computed:
 *  - H-Spec: Parallel Speculative Decoding Without a Drafter-Side KV Cache
 *    (arXiv 2609.24197), Abstract: attention modules reuse the target KVs in place;
 *    Mamba modules are initialised with the projected last-token target hidden
 *    state; Mamba's parallel scan keeps drafting block-parallel.
 *  - evolve.pub review of H-Spec, Summary: the recurrent layers are Mamba-2, the
 *    context storage is O(1), the backbone is a Mamba-attention hybrid.
 *  - Mamba-2 selective state-space recurrence (Dao & Gu, "Transformers are SSMs",
 *    2024), scalar-times-identity A per head, one B/C group:
 *        h_t = exp(dt_t A) h_{t-1} + dt_t x_t B_t^T,   y_t = h_t C_t + D x_t.
 * Readings where the pages are silent are listed in the design notes; each
 * function below states the one it takes.
 *
 * Element types: ORACLE_F32 (float) or ORACLE_BF16 (uint16 bit pattern, decoded
 * exactly).  In a bf16 draft step the oracle rounds (round-to-nearest-even) at the
 * tensors the product stores in bf16, and keeps everything else in double.
 */
#ifndef HSPEC_ORACLE_H
#define HSPEC_ORACLE_H
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

enum { ORACLE_F32 = 0, ORACLE_BF16 = 1 };

/* h0[c][r] = sum_j W_inj[r][j] h_last[c][j], r = (h*P + p)*N + n, i.e. the
 * projection result reshaped row-major to [H][P][N].  W_inj [HPN, d], h_last [C, d]. */
void oracle_inject(int HPN, int d, const void* W_inj, int w_type, const void* h_last, int h_type,
                   int C, double* h0);

/* Sequential Mamba-2 recurrence over the K block positions of each request.
 * x [C,K,H,P] (x_type), dt [C,K,H] f32, A [H] f32, B and Cm [C,K,N] (bc_type),
 * D [H] f32, h0 [C,H,P,N] f32 (may be NULL = zero state).
 * Outputs y [C,K,H,P] and, if hK != NULL, the final state hK [C,H,P,N]. */
void oracle_ssd_scan(int C, int K, int H, int P, int N, const void* x, int x_type, const float* dt,
                     const float* A, const void* B, const void* Cm, int bc_type, const float* D,
                     const float* h0, double* y, double* hK);

/* Block queries attend over the target's paged KV read through the page table,
 * followed by the block's own K keys.  q [C,K,Hq,D]; pools [num_pages,page,Hkv,D];
 * page_table [C,max_pages]; ctx_lens [C]; k_blk, v_blk [C,K,Hkv,D]; out [C,K,Hq,D].
 * Returns 0, or -1 if a needed page id lies outside [0, num_pages) or a
 * context length is negative or longer than the page table. */
int oracle_attn_paged(int C, int K, int Hq, int Hkv, int D, int page, const void* q,
                      const void* k_pool, const void* v_pool, int dtype, int num_pages,
                      const int32_t* page_table, int max_pages, const int32_t* ctx_lens,
                      const void* k_blk, const void* v_blk, int causal_block, double* out);

/* Same attention over an explicitly contiguous context cache k_ctx/v_ctx
 * [C, max_ctx, Hkv, D] (row t of request c = its t-th context token). */
void oracle_attn_contiguous(int C, int K, int Hq, int Hkv, int D, const void* q,
                            const void* k_ctx, const void* v_ctx, int dtype, int max_ctx,
                            const int32_t* ctx_lens, const void* k_blk, const void* v_blk,
                            int causal_block, double* out);

/* Row-wise RMSNorm: out = x / sqrt(mean(x^2) + eps) * w.  x [rows, n] double. */
void oracle_rmsnorm(int rows, int n, const double* x, const float* w, double eps, double* out);

/* Rotate-half rotary embedding of one head vector pair-wise at position pos. */
void oracle_rope(int D, double theta, long pos, const double* v, double* out);

/* Round a double to the nearest bf16 value (ties to even), returned as a double. */
double oracle_bf16_round(double x);
void oracle_bf16_round_array(long n, const double* in, double* out);

/* Logits of rows hn [rows, d] against W_lm [V, d]; per row the argmax (lowest id on
 * ties), the top logit and the runner-up logit. */
void oracle_lm_head_argmax(int rows, int d, int V, const void* hn, int hn_type, const void* W_lm,
                           int w_type, int32_t* argmax, double* top1, double* top2);

/* Greedy verification of K drafts per request (standard speculative decoding, which
 * H-Spec follows -- evolve.pub review of H-Spec, Frequently asked questions).  logits
 * [C, K+1, V] (type ltype) are the target's, row j predicting block position j;
 * drafts [C, K].  Per request: t_j = argmax_v logits[c][j][v] (lowest id on ties, NaN
 * never wins; -1 if the row has no number), accepted a = number of leading j < K with
 * drafts[c][j] == t_j, next_token = t_a, and ctx_lens[c] += a + 1 when ctx_lens is not
 * NULL (the accepted drafts and the target's token enter the context; the K - a
 * rejected positions roll back). */
void oracle_verify_greedy(int C, int K, int V, const void* logits, int ltype, const int32_t* drafts,
                          int32_t* accepted, int32_t* next_token, int32_t* ctx_lens);

typedef struct {
  int d, Hq, Hkv, D, H, P, N, page, d_ff, vocab, n_layers;
  char kinds[16];       /* 'M' or 'A' per layer */
  double rope_theta, eps;
  int dtype;            /* ORACLE_F32 or ORACLE_BF16: weights, activations, KV */
  int use_rope, use_gate, causal_block;
  int mask_token;
} oracle_cfg;

typedef struct {
  /* shared */
  const float* norm;
  /* Mamba-2 layer */
  const void* W_in; const float* dt_bias; const float* A; const float* D; const float* gnorm;
  const void* W_out; const void* W_inj;
  /* attention layer and the target KV it reads */
  const void* W_qkv; const void* W_o;
  const void* k_pool; const void* v_pool; int num_pages; const int32_t* page_table; int max_pages;
  /* SwiGLU sub-layer (d_ff > 0) */
  const float* mlp_norm; const void* W_gate; const void* W_up; const void* W_down;
} oracle_layer;

typedef struct {
  int C, K;
  const int32_t* tokens;   /* [C,K] block tokens (used when vocab > 0) */
  const void* x_in;        /* [C,K,d] direct block input (used when vocab == 0) */
  int x_in_type;           /* element type of x_in (ORACLE_F32 or ORACLE_BF16) */
  const void* h_last;      /* [C,d] target last-token hidden state */
  const int32_t* ctx_lens; /* [C] */
  const float* final_norm; const void* W_lm;   /* [d], [vocab,d]; W_lm is also the embedding */
  /* reduced-vocabulary draft head (draft_vocab > 0): logits over W_lm_draft [draft_vocab,d]
   * and the draft token draft_to_target[argmax] (evolve.pub review of H-Spec, Frequently
   * asked questions: the drafter's vocabulary may be cut to 32k frequent tokens; the
   * target's verification keeps the output exact).  draft_vocab = 0: the full W_lm head. */
  int draft_vocab; const void* W_lm_draft; const int32_t* draft_to_target;
  /* outputs (any may be NULL) */
  double* hidden;          /* [C,K,d] residual stream after the last layer */
  double* layer_out;       /* [n_layers,C,K,d] residual stream after each layer */
  double* final_normed;    /* [C,K,d] final RMSNorm output (rounded like the product stores it) */
  int32_t* draft_tokens;   /* [C,K] */
  double* top1; double* top2;  /* [C,K] */
} oracle_step;

/* One full draft step.  Returns 0, or -1 on a page-table error. */
int oracle_draft_step(const oracle_cfg* cfg, const oracle_layer* layers, oracle_step* io);

#ifdef __cplusplus
}
#endif
#endif
