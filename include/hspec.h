/*
 * hspec.h -- C-ABI of libhspec.so: the block-parallel draft step of the H-Spec
 * hybrid Mamba-attention drafter on NVIDIA B200 (sm_100a).
 *
 * What the library computes (H-Spec: Parallel Speculative Decoding Without a
 * Drafter-Side KV Cache, arXiv 2609.24197, Abstract; evolve.pub review, Summary):
 * a drafter proposes K tokens of a block in parallel.  Its attention layers read the
 * target model's paged KV cache IN PLACE (the drafter keeps no KV cache of its own),
 * and its Mamba-2 layers start from a state projected from the target's last-token
 * hidden state, h0 = reshape(W_inj . h_last).  The Mamba-2 scan over the K block
 * positions is evaluated in parallel chunks (the SSD form of Dao & Gu, 2024):
 *     h_t = exp(dt_t A) h_{t-1} + dt_t x_t (x) B_t,     y_t = C_t . h_t + D x_t.
 *
 * Conventions for every entry point
 *  - Pointers marked "device" are caller-owned CUDA device memory; the library never
 *    frees, copies or keeps them beyond the call (the target KV pool is read in place
 *    and never written).  Host structs are read during the call only.
 *  - Matrices are row-major; weights are [out_features, in_features].
 *  - Element type: hspec_cfg.dtype selects fp32 or bf16 for weights, activations and
 *    the KV pool.  Recurrent state (h0, hK), dt, A, D, norm weights and the SSD
 *    output y are always fp32.
 *  - Every call is asynchronous on `stream` (a cudaStream_t, NULL = legacy default
 *    stream).  The returned status covers host-side validation and launch errors.
 *    Invalid arguments are rejected before anything is launched.  Errors that only
 *    the device can see (a page id outside the pool, a context longer than the page
 *    table, a token id outside the vocabulary) set a device error word; the kernels
 *    skip the offending read (it contributes nothing) and hspec_sync_status() reports
 *    HSPEC_ERR_DEVICE_CHECK.
 *  - No entry point allocates device memory.  Scratch space comes from a
 *    caller-provided workspace whose size the *_workspace_size functions return.
 *  - Thread safety: calls on different streams may run concurrently if their
 *    workspaces differ.
 */
#ifndef HSPEC_H
#define HSPEC_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define HSPEC_API __attribute__((visibility("default")))
#else
#define HSPEC_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef int hspec_status;
#define HSPEC_OK 0
#define HSPEC_ERR_INVALID_ARG 1     /* null pointer, non-positive size, bad flag        */
#define HSPEC_ERR_SHAPE_MISMATCH 2  /* e.g. Hq not a multiple of Hkv, dims inconsistent  */
#define HSPEC_ERR_PAGE_OOB 3        /* page table width / pool size inconsistent (host)  */
#define HSPEC_ERR_UNSUPPORTED 4     /* shape outside what the kernels implement          */
#define HSPEC_ERR_CUDA 5            /* a CUDA runtime call or kernel launch failed        */
#define HSPEC_ERR_DEVICE_CHECK 6    /* a kernel saw a bad page id / ctx length / token   */
#define HSPEC_ERR_WORKSPACE 7       /* workspace missing, too small or misaligned         */

#define HSPEC_DTYPE_F32 0
#define HSPEC_DTYPE_BF16 1

#define HSPEC_FLAG_ROPE 1           /* rotary embedding on q and block keys at ctx_c + j */
#define HSPEC_FLAG_GATE 2           /* Mamba-2 gated RMSNorm y <- norm(y * silu(z)) w_g  */
#define HSPEC_FLAG_CAUSAL_BLOCK 4   /* block query j sees block key i only when i <= j   */
#define HSPEC_FLAG_FUSE_INJECT 8    /* bf16 draft step, d_state 128: the injection GEMM   */
                                    /* adds h0's share of the scan output from its        */
                                    /* accumulator (h0 never stored) after a zero-state   */
                                    /* scan; default: h0 stored and read by the scan      */

#define HSPEC_MAX_LAYERS 16

/* Shapes and options of one drafter.  The attention dims must equal the target's
 * (the drafter reads the target KV as is: evolve.pub review, limitations). */
typedef struct hspec_cfg {
  int d_model;                      /* d: hidden size (= target hidden size)              */
  int n_q_heads;                    /* Hq                                                  */
  int n_kv_heads;                   /* Hkv; GQA group G = Hq / Hkv                         */
  int head_dim;                     /* D (attention), even                                 */
  int n_ssm_heads;                  /* H  (Mamba-2 heads)                                  */
  int ssm_head_dim;                 /* P  (Mamba-2 head dim)                               */
  int d_state;                      /* N  (Mamba-2 state size)                             */
  int page_size;                    /* tokens per KV page (vLLM block size)                */
  int d_ff;                         /* SwiGLU intermediate size, 0 = no MLP sub-layer      */
  int vocab;                        /* LM-head rows, 0 = no head (step returns hidden)     */
  int n_layers;                     /* <= HSPEC_MAX_LAYERS                                 */
  char layer_kinds[HSPEC_MAX_LAYERS];/* 'M' = Mamba-2 layer, 'A' = attention layer         */
  int dtype;                        /* HSPEC_DTYPE_F32 or HSPEC_DTYPE_BF16                 */
  int flags;                        /* HSPEC_FLAG_*                                        */
  float rope_theta;                 /* RoPE base                                           */
  float norm_eps;                   /* RMSNorm epsilon                                     */
  int ssd_chunk;                    /* SSD chunk length Q (0 = whole block in one chunk)   */
  int attn_split_tokens;            /* split-KV partition length in tokens, multiple of 16 (0 = auto):
                                       fp32, tokens per split of a request; bf16, the length of a
                                       chunk of the tile-space partition in units of 64 tokens
                                       (rounded up), where a sequence counts one unit per 64-key
                                       tile plus 4 for its start; at most 2048 chunks -- auto: one
                                       chunk per SM */
  int draft_vocab;                  /* reduced draft head rows (0 = the full vocab head):    */
                                    /* logits over W_lm_draft, draft token = the mapped id  */
  long long wait_limit_ns;          /* a pipeline wait in a tensor-core kernel (an mbarrier
                                       or a tile counter) gives up after this many ns of the
                                       GPU's global timer, skips the rest of its work and
                                       sets bit 8 of the device error word (see
                                       hspec_sync_status); the kernel still waits for its own
                                       copies and MMAs in flight before it exits.  0 = 2 s,
                                       far above any legitimate wait; >= 0 */
} hspec_cfg;

/* Weights of one layer (caller-owned device memory; fields of the other layer kind
 * and of an absent MLP are ignored). */
typedef struct hspec_layer_weights {
  const float* norm;      /* [d]            pre-mixer RMSNorm weight                     */
  const void* W_in;       /* [2HP+2N+H, d]  Mamba-2 in_proj, rows [z | x | B | C | dt]  */
  const float* dt_bias;   /* [H]            dt = softplus(dt_raw + dt_bias)             */
  const float* A;         /* [H]            negative per-head decay rate                */
  const float* D;         /* [H]            skip coefficient                            */
  const float* gnorm;     /* [HP]           gated-RMSNorm weight                        */
  const void* W_out;      /* [d, HP]        Mamba-2 out_proj                            */
  const void* W_inj;      /* [HPN, d]       state injection, rows (h*P + p)*N + n       */
  const void* W_qkv;      /* [(Hq+2Hkv)D, d] attention projections, rows [q | k | v]    */
  const void* W_o;        /* [d, Hq D]      attention output projection                 */
  const float* mlp_norm;  /* [d]            pre-MLP RMSNorm weight                      */
  const void* W_gate;     /* [d_ff, d]                                                  */
  const void* W_up;       /* [d_ff, d]                                                  */
  const void* W_down;     /* [d, d_ff]                                                  */
} hspec_layer_weights;

typedef struct hspec_model_weights {
  hspec_layer_weights layers[HSPEC_MAX_LAYERS];
  const float* final_norm; /* [d]                                                        */
  const void* W_lm;        /* [vocab, d] shared LM head, also the token embedding table  */
  /* reduced-vocabulary draft head (cfg.draft_vocab > 0; H-Spec's evolve.pub review,
   * Frequently asked questions: the drafter's vocabulary may be cut to frequent tokens):
   * row r of W_lm_draft stands for target token draft_to_target[r] (0 <= id < vocab, a
   * bad id sets the device error word and the token is written as -1) */
  const void* W_lm_draft;          /* [draft_vocab, d]                                   */
  const int32_t* draft_to_target;  /* [draft_vocab]                                      */
} hspec_model_weights;

/* The target's paged KV cache, read in place (never written, never copied). */
typedef struct hspec_kv_view {
  const void* k_pool;          /* device [num_pages, page_size, Hkv, D]                  */
  const void* v_pool;          /* device [num_pages, page_size, Hkv, D]                  */
  int num_pages;               /* pages in the pool                                       */
  const int32_t* page_table;   /* device [C, max_pages]; token t of request c lives in
                                  page page_table[c][t / page_size], slot t % page_size   */
  int max_pages;               /* page-table width; ctx_lens[c] <= max_pages * page_size  */
} hspec_kv_view;

/* ------------------------------------------------------------------ kernels
 * Each of the three calls below is one step of the draft step, usable alone. */

/* State injection (H-Spec Abstract: each Mamba layer starts from a projection of the
 * target's hidden state at the last token).
 *   h0[c][h][p][n] = sum_j W_inj[(h*P+p)*N+n][j] * h_last[c][j]
 * W_inj  device [H*P*N, d] (dtype); h_last device [C, d] (dtype);
 * h0     device [C, H, P, N] fp32, written.  C >= 1. */
HSPEC_API hspec_status hspec_inject_state(const hspec_cfg* cfg, const void* W_inj, const void* h_last, int C,
                                float* h0, void* stream);

/* Mamba-2 SSD scan over the K block positions of every request, started from h0
 * (H-Spec Abstract: the parallel scan is what keeps the drafting block-parallel),
 * evaluated in chunks of cfg->ssd_chunk positions:
 *   h_t = exp(dt_t A_h) h_{t-1} + dt_t x_t (x) B_t;  y_t = C_t . h_t + D_h x_t.
 * x  device [C, K, H, P] (dtype);  dt device [C, K, H] fp32 (already positive);
 * A, D device [H] fp32;  B, Cm device [C, K, N] (dtype, one group for all heads);
 * h0 device [C, H, P, N] fp32 (NULL = zero state);
 * y  device [C, K, H, P] fp32, written;  hK device [C, H, P, N] fp32 final state,
 * written when not NULL.  1 <= K <= 64. */
HSPEC_API hspec_status hspec_ssd_block_scan(const hspec_cfg* cfg, const void* x, const float* dt,
                                  const float* A, const void* B, const void* Cm, const float* D,
                                  const float* h0, int C, int K, float* y, float* hK, void* stream);

/* Workspace bytes hspec_attn_paged_block needs for C requests of K block tokens and
 * a page table of width max_pages (the split-KV partials; on the bf16 path a fixed
 * number of partial slots, C * Hkv * ceil(K*G/128) + 256, whatever the width). */
HSPEC_API size_t hspec_attn_workspace_size(const hspec_cfg* cfg, int C, int K, int max_pages);

/* Paged in-place GQA attention of the K block queries (H-Spec Abstract: the drafter's
 * attention reads the target's KV cache where it lies, with no copy).  Query (c, j, h) attends, with scale
 * 1/sqrt(D), over the ctx_lens[c] context tokens of request c read through the page
 * table, followed by the K block keys of request c (all visible unless
 * HSPEC_FLAG_CAUSAL_BLOCK); kv head = h / (Hq/Hkv).  Long contexts are split across
 * CTAs and the partial (max, sum, acc) merged.  bf16: the split follows an even
 * partition over the SMs of all (request, kv head) key tiles of the call, each
 * sequence's start counted as a few tiles of work, so a request's result depends on
 * the batch (its order and the other lengths) up to rounding; calls on the same batch
 * give bit-identical results.
 * q      device [C, K, Hq, D] (dtype);   kv: the target cache;
 * ctx_lens device [C] int32, 0 <= ctx_lens[c] <= kv->max_pages * page_size;
 * k_blk, v_blk device [C, K, Hkv, D] (dtype);
 * out    device [C, K, Hq, D] (dtype), written;
 * workspace device, >= hspec_attn_workspace_size() bytes, 256-byte aligned. */
HSPEC_API hspec_status hspec_attn_paged_block(const hspec_cfg* cfg, const void* q, const hspec_kv_view* kv,
                                    const int32_t* ctx_lens, const void* k_blk, const void* v_blk,
                                    int C, int K, void* out, void* workspace, size_t ws_bytes,
                                    void* stream);

/* Allocation-free variant of hspec_attn_paged_block.  The H-Spec paper has no
 * counterpart to this entry point; it exists for deployment.  Some callers cannot allocate
 * device memory when they call in: a serving engine that handed nearly all HBM to
 * its KV-cache pool at start-up (a cudaMalloc could fail, or would break the
 * engine's memory accounting), or a plain C host program that links only this
 * library and has no device allocator of its own to provide a workspace.  This entry
 * point takes the same inputs and output as hspec_attn_paged_block but keeps its
 * split-KV partials in a static device array of HSPEC_NOALLOC_SCRATCH_BYTES bytes
 * inside the library.
 *  - When the array's memory is taken: the array sits in a module of its own, which
 *    CUDA loads (and so reserves HSPEC_NOALLOC_SCRATCH_BYTES on that device) at the
 *    first call of this entry point on each device under lazy module loading, CUDA's
 *    default, or when the context is created under CUDA_MODULE_LOADING=EAGER.  It
 *    stays reserved until the context is destroyed.  A caller that hands nearly all
 *    HBM to a KV pool should make one small call per device before sizing the pool
 *    (or load modules eagerly); otherwise that first call may find no room and return
 *    HSPEC_ERR_CUDA with an out-of-memory message.
 *  - Calls whose partials need more than HSPEC_NOALLOC_SCRATCH_BYTES (that is,
 *    hspec_attn_workspace_size(cfg, C, K, kv->max_pages) is larger) are rejected
 *    with HSPEC_ERR_WORKSPACE before anything is launched.
 *  - The first call in each CUDA context looks up the array's device address (a
 *    runtime call that maps the module and allocates nothing else); make that first
 *    call before any CUDA stream capture.
 *  - All calls share the one array, which keeps the previous call's contents.
 *    Nothing in it has to start at zero: each call writes every partial it later
 *    reads.  Calls that overlap on the GPU (different streams, or different host
 *    threads on one device) race on the array; serialise them.
 *  - Calls no cudaMalloc, cudaFree or other allocating routine. */
#define HSPEC_NOALLOC_SCRATCH_BYTES ((size_t)64 << 20)
HSPEC_API hspec_status hspec_attn_paged_block_noalloc(const hspec_cfg* cfg, const void* q,
                                                      const hspec_kv_view* kv, const int32_t* ctx_lens,
                                                      const void* k_blk, const void* v_blk, int C, int K,
                                                      void* out, void* stream);

/* ------------------------------------------------------------- draft step */

typedef struct hspec_drafter hspec_drafter;

/* Validates cfg and keeps a host copy of it and of the weight pointers (device
 * memory stays caller-owned and must outlive the drafter).  Allocates no device
 * memory.  *out receives the handle. */
HSPEC_API hspec_status hspec_drafter_create(const hspec_cfg* cfg, const hspec_model_weights* weights,
                                  hspec_drafter** out);
HSPEC_API void hspec_drafter_destroy(hspec_drafter* drafter);

typedef struct hspec_step_in {
  int C;                       /* requests in the batch                                   */
  int K;                       /* block size (tokens drafted in parallel), 1..64          */
  const int32_t* tokens;       /* device [C, K] block tokens, used when vocab > 0         */
  const void* x_in;            /* device [C, K, d] (dtype) block input, used when vocab == 0 */
  const void* h_last;          /* device [C, d] (dtype) target last-token hidden state    */
  const int32_t* ctx_lens;     /* device [C] target context length per request            */
  hspec_kv_view kv[HSPEC_MAX_LAYERS]; /* one target cache per attention layer, in order   */
} hspec_step_in;

typedef struct hspec_step_out {
  int32_t* draft_tokens;       /* device [C, K] argmax token ids (vocab > 0), or NULL     */
  float* hidden;               /* device [C, K, d] fp32 residual stream after the last
                                  layer, or NULL                                          */
  void* final_normed;          /* device [C, K, d] (dtype) final RMSNorm output (the LM-head
                                  input), or NULL                                         */
  float* top_logit;            /* device [C, K] logit of the argmax token, or NULL        */
  float* layer_hidden;         /* device [n_layers, C, K, d] fp32 residual stream after each
                                  layer (for layer-by-layer validation), or NULL          */
} hspec_step_out;

/* Workspace bytes hspec_draft_step needs (activations, h0 of one Mamba layer,
 * split-KV partials, argmax partials). */
HSPEC_API size_t hspec_step_workspace_size(const hspec_cfg* cfg, int C, int K, int max_pages);

/* Workspace bytes of hspec_verify_greedy for C requests of K drafts over cfg->vocab. */
HSPEC_API size_t hspec_verify_workspace_size(const hspec_cfg* cfg, int C, int K);

/* Greedy verification of the drafts against the target's logits (standard
 * speculative-decoding verification, kept by H-Spec -- evolve.pub review, Frequently
 * asked questions).  Row j of request c is the target's prediction for block position j:
 *   t_j = argmax_v logits[c][j][v]   (lowest id on ties; NaN never wins; -1 if none)
 *   accepted[c] = longest prefix j < K with drafts[c][j] == t_j
 *   next_token[c] = t_accepted;  ctx_lens[c] += accepted[c] + 1 when ctx_lens != NULL
 * (the accepted drafts and the target's token enter the context; the rejected
 * positions roll back -- their KV slots lie past the new length).
 * logits device [C, K+1, cfg->vocab] (cfg->dtype); drafts device [C, K] int32;
 * accepted, next_token device [C] int32, written; ctx_lens device [C] int32 or NULL;
 * workspace device, >= hspec_verify_workspace_size() bytes, 256-byte aligned.
 * C >= 1, 1 <= K <= 64, cfg->vocab >= 1. */
HSPEC_API hspec_status hspec_verify_greedy(const hspec_cfg* cfg, const void* logits, const int32_t* drafts, int C,
                                           int K, int32_t* accepted, int32_t* next_token, int32_t* ctx_lens,
                                           void* workspace, size_t ws_bytes, void* stream);

/* One block-parallel draft step (all layers, then the LM-head argmax when vocab > 0):
 * per layer, pre-norm residual blocks
 *   M: x += W_out gnorm(SSD(in_proj(norm(x)); h0 = W_inj h_last) * silu(z))
 *   A: x += W_o attn(rope(q), target KV in place ++ rope(k_blk), v_blk)
 *   MLP (d_ff > 0): x += W_down (silu(W_gate norm(x)) * W_up norm(x))
 * then draft_tokens = argmax(W_lm final_norm(x)) (with draft_vocab > 0:
 * draft_to_target[argmax(W_lm_draft final_norm(x))]).  max_pages of every kv view must
 * be <= the max_pages given to hspec_step_workspace_size. */
HSPEC_API hspec_status hspec_draft_step(hspec_drafter* drafter, const hspec_step_in* in,
                              const hspec_step_out* out, void* workspace, size_t ws_bytes,
                              void* stream);

/* --------------------------------------------------------------- status */

/* Synchronises `stream`, then returns HSPEC_ERR_DEVICE_CHECK if any kernel of this
 * library flagged a bad page id, context length or token id since the last call (and
 * clears the flag), HSPEC_ERR_CUDA on a CUDA error, else HSPEC_OK. */
HSPEC_API hspec_status hspec_sync_status(void* stream);

/* Static description of a status code. */
HSPEC_API const char* hspec_status_string(hspec_status status);

/* Message of the most recent failure in this thread ("" if none). */
HSPEC_API const char* hspec_last_error(void);

/* Kernels this library has launched since load (all threads). */
HSPEC_API unsigned long long hspec_launch_count(void);

/* Kernel timing (tracing aid).  hspec_profile_enable(1) clears the record and makes
 * hspec_draft_step record a CUDA event pair on its stream around each group of
 * kernels it launches (one group per step of the draft step: "in_proj",
 * "attn_paged", "lm_head_argmax", ...); hspec_profile_enable(0) stops recording.
 * Events are created on demand, so do not enable it during CUDA graph capture. */
HSPEC_API hspec_status hspec_profile_enable(int on);

/* Synchronises the recorded events and writes, per kernel group, its name into
 * names[i*32 .. i*32+31] (NUL-terminated), the summed event time in milliseconds
 * into total_ms[i] and the number of recorded occurrences into count[i], for at
 * most max_entries groups.  Returns the number of groups written, or -1 on a CUDA
 * error. */
HSPEC_API int hspec_profile_read(char* names, double* total_ms, int* count, int max_entries);

/* Library version string. */
HSPEC_API const char* hspec_version(void);

#ifdef __cplusplus
}
#endif
#endif /* HSPEC_H */
