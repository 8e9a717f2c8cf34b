// Internal launchers of the libhspec kernels (called by hspec_abi.cu).
// `dtype` is HSPEC_DTYPE_F32 (elements are float) or HSPEC_DTYPE_BF16 (bf16).
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace hspec {

// ------------------------------------------------------------ rows.cu
// x[m][:] = float(table[tokens[m]][:])  (embedding rows of the tied LM head)
void embed_rows(int dtype, const int32_t* tokens, const void* table, int vocab, float* x, int M, int d,
                int* err, cudaStream_t s);
// x[i] = float(in[i])
void rows_to_f32(int dtype, const void* in, float* x, long n, cudaStream_t s);
// out[m][:] = x[m][:] / sqrt(mean(x[m]^2) + eps) * w   (out in dtype)
void rmsnorm_rows(int dtype, const float* x, const float* w, void* out, int M, int n, float eps,
                  cudaStream_t s);
// out[m][:] = gate ? rmsnorm(y[m] * silu(z[m])) * w : y[m]   (z rows at z_stride elements)
void gated_rmsnorm_rows(int dtype, const float* y, const void* z, long z_stride, const float* w,
                        void* out, int M, int n, float eps, bool gate, cudaStream_t s);
// In-place rotate-half RoPE on heads [0, n_heads) of every row m = c*K + j of qkv, at
// position ctx_lens[c] + j.
void rope_rows(int dtype, void* qkv, long row_stride, const int32_t* ctx_lens, int C, int K,
               int n_heads, int D, float theta, cudaStream_t s);
// cs[m][i] = (cos, sin) of the RoPE angle of row m = c*K + j, pair i < D/2, at position
// ctx_lens[c] + j (computed in double, stored as fp32).
void rope_table(float2* cs, const int32_t* ctx_lens, int C, int K, int D, float theta, cudaStream_t s);
// tokens[m] = argmax over parts of (pval, pidx)[m][:] (lowest id on ties); top[m] = its value.
// Per row the max over the partials (lowest id on ties); with `map` (reduced draft
// head) the token is map[id], checked against [0, vocab) (else -1 and kErrTokenOOB).
void argmax_reduce(const float* pval, const int32_t* pidx, int M, int n_parts, int32_t* tokens,
                   float* top, const int32_t* map, int vocab, int* err, cudaStream_t s);

// ------------------------------------------------------------ gemm_simt.cu / gemm_tc.cu
enum GemmEpi : int {
  kEpiStore = 0,      // out (dtype, or fp32 if out_f32) = acc
  kEpiResid = 1,      // x (fp32) += acc
  kEpiSwiGLU = 2,     // out (dtype) = silu(acc(B)) * acc(B2)
  kEpiArgmax = 3,     // (pval, pidx)[m][n_tile] = per-row max / argmax over the tile's columns
  kEpiSsdRead = 4,    // bf16 only, acc = injected state h0: y += decay * (C . h0) (see SsdReadArgs)
  kEpiRope = 5,       // bf16 only: out (bf16) = acc, with rotate-half RoPE on the heads of columns
                      // [0, rope.cols) at each row's position (see RopeArgs)
};

// kEpiRope: in each head of D columns that lies in [0, cols), the pair (i, i + D/2),
// i < D/2, of row m is rotated by the angle whose (cos, sin) is cs[m * D/2 + i] (the
// table rope_table() writes: row m is block position m % K of request m / K) after the
// projection is rounded to bf16 (the stored value), and the result rounded to bf16 again.
struct RopeArgs {
  const float2* cs;
  int D, cols;
};

// kEpiSsdRead (d_state N = 128, even P): the injection GEMM (row m = request c, column
// (h*P + p)*N + n of h0) adds the initial state's share of the SSD output without
// storing h0:
//   y[c*K + t][h*P + p] += exp(sum_{s<=t} dt[c,s,h] A[h]) * sum_n C[c*K + t][n] * h0[c][h][p][n]
// with dt = softplus(dt_raw + dt_bias) (dt_raw, C: dtype rows of the in-projection).
struct SsdReadArgs {
  int K, P, N;
  const void* Cm; long c_rs;       // C [C*K, N] (dtype), row stride
  const void* dt_raw; long dt_rs;  // [C*K, H] (dtype), row stride
  const float* dt_bias;            // [H]
  const float* A;                  // [H]
  float* y; long y_rs;             // [C*K, H*P] fp32, row stride
};

struct GemmArgs {
  int M, N, K;
  const void* A; long lda;     // [M, K] row-major (dtype)
  const void* B; long ldb;     // [N, K] row-major (dtype)
  const void* B2;              // second [N, K] operand (SwiGLU up projection)
  void* out; long ldo;         // output (see epilogue)
  bool out_f32;                // kEpiStore: fp32 output instead of dtype
  float* pval; int32_t* pidx;  // kEpiArgmax partials [M, n_parts]
  int n_parts;
  // Workspace of a cut K loop (optional): when whole tiles would leave SMs idle the K
  // loop is cut (stream-K or split-K); segments that cover part of a tile write fp32
  // partials to `part`, and the last segment of a tile to finish (counter in
  // `tile_cnt`, zero on entry and left zero) sums them in K order and applies the
  // epilogue, so the result does not depend on scheduling.
  float* part; int* tile_cnt; size_t part_bytes; int max_tiles;
  SsdReadArgs ssd;             // kEpiSsdRead
  RopeArgs rope;               // kEpiRope
  unsigned long long wait_ns;  // pipeline waits give up after this long (0: the default)
};
// Workspace bytes (partials) that gemm() needs for this shape when it cuts the K loop
// (stream-K or split-K; 0 for whole tiles); counters: gemm_tile_count().
size_t gemm_kcut_bytes(int dtype, GemmEpi epi, int M, int N, int K);
int gemm_tile_count(int dtype, GemmEpi epi, int M, int N);

// Whether gemm(kEpiRope) can run this shape (bf16, head dim 64 or 128, the K loop
// whole or cut stream-K); otherwise store with kEpiStore and rotate with rope_rows.
bool gemm_rope_fusable(int dtype, int M, int N, int K, int D);

// Column tile width of the argmax partials (n_parts = ceil(N / argmax_tile_n(dtype))).
int argmax_tile_n(int dtype);
// out = epilogue(A . B^T); false (with the message recorded) if it cannot launch.
bool gemm(int dtype, GemmEpi epi, const GemmArgs& g, cudaStream_t s);

// ------------------------------------------------------------ ssd.cu
struct SsdArgs {
  int C, K, H, P, N, Q;        // Q: chunk length
  const void* x; long x_rs;    // dtype, token row stride (head h at column h*P)
  const void* dt; long dt_rs;  // dt (fp32) or, with dt_bias, dt_raw (dtype); head h at column h
  const float* dt_bias;        // NULL: dt given; else dt = softplus(dt_raw + dt_bias)
  const float* A; const float* D;
  const void* B; const void* Cm; long bc_rs;  // dtype, token row stride
  const float* h0;             // [C,H,P,N] or NULL
  float* y; long y_rs;         // fp32, token row stride (head h at column h*P)
  float* hK;                   // [C,H,P,N] or NULL
  unsigned long long wait_ns;  // pipeline waits give up after this long (0: the default)
};
size_t ssd_smem_bytes(int P, int N, int Q);
void ssd_scan(int dtype, const SsdArgs& a, cudaStream_t s);
// Tensor-core state readout (ssd_tc.cu): bf16, h0 given, the block as one chunk,
// K <= 32, d_state 128, 64 <= P <= 128 dividing 128; with or without the final state.
bool ssd_tc_supported(int dtype, const SsdArgs& a);
bool ssd_tc_launch(const SsdArgs& a, cudaStream_t s);

// ------------------------------------------------------------ attn.cu
constexpr int kAttnTcTile = 64;  // keys per tile of the tensor-core attention path
constexpr int kAttnTcRows = 128; // query rows per row block (MMA M) of that path
// chunks of the tensor-core path's tile-space partition: one per SM (auto), or of an
// explicitly requested length, at most this many (which bounds the partial workspace)
constexpr int kAttnMaxChunksAuto = 256;
// On the line that the tensor-core path cuts into chunks, a sequence takes this many
// units for its start (the Q load, the page ids of its first tiles, the partials at its
// end: together about as long as four tiles), then one unit per 64-key tile, so that
// the chunks balance tiles and sequence starts together.
constexpr int kAttnSeqUnits = 6;
constexpr int kAttnMaxChunksExplicit = 2048;
struct AttnArgs {
  int C, K, Hq, Hkv, D;
  const void* q; long q_rs;              // token row stride; head h at column h*D
  const void* k_pool; const void* v_pool; int num_pages; int page_size;
  const int32_t* page_table; int max_pages;
  const int32_t* ctx_lens;
  const void* kb; long kb_rs;            // block keys, kv head g at column g*D
  const void* vb; long vb_rs;
  void* out; long o_rs;                  // dtype, token row stride
  int split_tokens;                      // fp32 path: tokens per split (multiple of 16);
                                         // tensor-core path: chunk length (0 = one per SM)
  int n_splits;                          // fp32 path: splits per (request, kv head) upper bound
  int max_chunks;                        // tensor-core path: chunk bound of the workspace
  bool causal_block;
  bool tile_pieces;                      // tensor-core path: partials are the pieces of the tile-space
                                         // partition (the block's keys end each sequence)
  int sub_splits;                        // partials per split (tensor-core path: one per softmax warpgroup)
  float* ws_acc; float* ws_ml;           // split partials
  // tensor-core path: [1] total work units T, [2] chunk length Z (units), [3] number of
  // chunks, written by the schedule kernel; from [64] the requests' offsets on the line of
  // units (C + 1): kAttnSeqUnits per sequence start, one per 64-key tile
  int* sched;
  int* err;
  unsigned long long wait_ns;            // pipeline waits give up after this long (0: the default)
};
// Split policy (tokens per split, splits per request) and workspace bytes.
int attn_split_tokens(int dtype, int C, int Hkv, int K, int max_ctx, int requested);
int attn_num_splits(int dtype, int K, int max_ctx, int split_tokens);
// Rows of partials (each D fp32 + (m, l)) and workspace bytes.
size_t attn_partial_rows(int dtype, int C, int Hkv, int K, int G, int n_splits, int max_chunks);
size_t attn_ws_bytes(int dtype, int C, int Hkv, int K, int G, int D, int n_splits, int max_chunks);
int attn_sub_splits(int dtype);
bool attn_supported(int dtype, int K, int G, int D, const char** why);
// Checks the pointer / stride requirements of the tensor-core path (bf16).
bool attn_tc_supported(const AttnArgs& a, const char** why);
bool attn_tc_launch(const AttnArgs& a, cudaStream_t s);
// Split kernel + merge; false (message recorded) if it cannot launch.
bool attn_paged(int dtype, const AttnArgs& a, cudaStream_t s);

// ------------------------------------------------------------ verify.cu
// Greedy verification (see verify.cu); workspace of verify_ws_bytes(dtype, C, K, V) bytes.
size_t verify_ws_bytes(int dtype, int C, int K, int V);
void verify_greedy(int dtype, const void* logits, int V, const int32_t* drafts, int C, int K,
                   int32_t* accepted, int32_t* next_token, int32_t* ctx_lens, void* ws, cudaStream_t s);

}  // namespace hspec
