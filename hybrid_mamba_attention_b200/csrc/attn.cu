// Paged in-place GQA attention of the K block queries over the target's KV cache
// followed by the block's own keys (H-Spec Abstract: the drafter's attention reads
// the target's KV cache in place), split-KV across CTAs, then a merge of the partial
// softmax states.
// bf16 runs on the tensor cores (attn_tc.cu); this file holds the exact fp32 split
// kernel, the merge shared by both, and the split policy.
//
// attn_split_kernel (fp32): one CTA per (split, kv head g, request c).  Its R = K*G query
// rows (block position j, query head g*G + i) share every key/value of kv head g,
// so each 16-token tile of K and V is read from HBM once per CTA, translated through
// the page table in place (token t of request c: page page_table[c][t / page],
// slot t % page), staged in shared memory as fp32 and used by all R rows.  Threads
// form groups of TPR lanes per row; a lane holds D/TPR interleaved dims of q and of
// the running output, dot products are reduced across the group with shuffles, and
// the softmax runs online in the exp2 domain.  The CTA writes its partial
// (m, l, unnormalised acc) per row.
//
// attn_merge_kernel: W = 1, 2, 4 or 8 warps per output row (c, j, h) combine the
// partials of that row, o = sum_s 2^(m_s - M) acc_s / sum_s 2^(m_s - M) l_s.  Warp w
// takes the partials s = w (mod W) in one pass over blocks of four (their (m, l) and
// rows loaded together, folded into a running (M, L, o) that is rescaled when a block
// raises the maximum); the W warps' states are then combined in warp order through
// shared memory, so the result does not depend on timing.
#include "../../include/hspec.h"
#include "common.cuh"
#include "kernels.cuh"

namespace hspec {
namespace {

constexpr int kThreads = 256;
constexpr int kTile = 16;

template <typename T, int TPR>
__global__ void __launch_bounds__(kThreads) attn_split_kernel(AttnArgs a, float scale_log2) {
  pdl_wait();  // the previous kernel on the stream is complete from here on
  pdl_trigger();
  extern __shared__ float sm[];
  const int D = a.D, Dp = D + 1;
  float* sK = sm;                           // [kTile][D+1]
  float* sV = sK + kTile * Dp;              // [kTile][D+1]
  const int split = blockIdx.x, g = blockIdx.y, c = blockIdx.z;
  const int G = a.Hq / a.Hkv, R = a.K * G;
  const int ctx = a.ctx_lens[c];
  if (ctx < 0 || ctx > a.max_pages * a.page_size) {
    if (threadIdx.x == 0 && split == 0) flag_error(a.err, kErrCtxOOB);
    return;
  }
  const int T_total = ctx + a.K;
  const int t_begin = split * a.split_tokens;
  if (t_begin >= T_total) return;  // the merge reads only the splits that hold tokens
  const int t_end = min(T_total, t_begin + a.split_tokens);

  const int row = threadIdx.x / TPR, gl = threadIdx.x % TPR;
  const bool active = row < R;
  const int j = active ? row / G : 0;
  const int h = g * G + (active ? row % G : 0);
  constexpr int DPT_MAX = 128 / TPR > 0 ? 128 / TPR : 1;
  const int dpt = D / TPR;
  float qv[DPT_MAX], acc[DPT_MAX];
  const T* q = (const T*)a.q + (size_t)(c * a.K + j) * a.q_rs + (size_t)h * D;
#pragma unroll
  for (int i = 0; i < DPT_MAX; ++i) {
    qv[i] = (active && i < dpt) ? to_f(q[gl + i * TPR]) * scale_log2 : 0.f;
    acc[i] = 0.f;
  }
  float m_run = -INFINITY, l_run = 0.f;

  const T* kp = (const T*)a.k_pool;
  const T* vp = (const T*)a.v_pool;
  const T* kb = (const T*)a.kb;
  const T* vb = (const T*)a.vb;
  const int32_t* table = a.page_table + (size_t)c * a.max_pages;

  for (int t0 = t_begin; t0 < t_end; t0 += kTile) {
    __syncthreads();
    for (int i = threadIdx.x; i < kTile * D; i += kThreads) {
      const int tt = i / D, e = i % D, t = t0 + tt;
      float kvk = 0.f, kvv = 0.f;
      if (t < ctx) {
        const int pg = table[t / a.page_size];
        if (pg >= 0 && pg < a.num_pages) {
          const size_t off = (((size_t)pg * a.page_size + t % a.page_size) * a.Hkv + g) * D + e;
          kvk = to_f(kp[off]);
          kvv = to_f(vp[off]);
        } else if (e == 0) {
          flag_error(a.err, kErrPageOOB);
        }
      } else if (t < t_end) {
        const size_t off = (size_t)(c * a.K + (t - ctx)) * a.kb_rs + (size_t)g * D + e;
        kvk = to_f(kb[off]);
        kvv = to_f(vb[(size_t)(c * a.K + (t - ctx)) * a.vb_rs + (size_t)g * D + e]);
      }
      sK[tt * Dp + e] = kvk;
      sV[tt * Dp + e] = kvv;
    }
    __syncthreads();
    // rows beyond R compute on q = 0 and are never written: every lane of a warp
    // must take part in the group shuffles below.
    float s[kTile];
    float tile_max = -INFINITY;
#pragma unroll
    for (int tt = 0; tt < kTile; ++tt) {
      float part = 0.f;
#pragma unroll
      for (int i = 0; i < DPT_MAX; ++i)
        if (i < dpt) part = fmaf(qv[i], sK[tt * Dp + gl + i * TPR], part);
#pragma unroll
      for (int o = TPR / 2; o > 0; o >>= 1) part += __shfl_xor_sync(0xffffffffu, part, o);
      const int t = t0 + tt;
      bool vis = t < t_end;
      if (a.causal_block && t >= ctx && (t - ctx) > j) vis = false;
      s[tt] = vis ? part : -INFINITY;
      tile_max = fmaxf(tile_max, s[tt]);
    }
    const float m_new = fmaxf(m_run, tile_max);
    if (m_new == -INFINITY) continue;  // nothing visible yet
    const float alpha = exp2f(m_run - m_new);
    float psum = 0.f;
#pragma unroll
    for (int tt = 0; tt < kTile; ++tt) {
      s[tt] = exp2f(s[tt] - m_new);
      psum += s[tt];
    }
    l_run = l_run * alpha + psum;
    m_run = m_new;
#pragma unroll
    for (int i = 0; i < DPT_MAX; ++i) {
      if (i >= dpt) break;
      float v = acc[i] * alpha;
#pragma unroll
      for (int tt = 0; tt < kTile; ++tt) v = fmaf(s[tt], sV[tt * Dp + gl + i * TPR], v);
      acc[i] = v;
    }
  }
  if (!active) return;
  const size_t base = ((((size_t)c * a.Hkv + g) * a.n_splits + split) * R + row);
  float* pacc = a.ws_acc + base * D;
#pragma unroll
  for (int i = 0; i < DPT_MAX; ++i)
    if (i < dpt) pacc[gl + i * TPR] = acc[i];
  if (gl == 0) {
    a.ws_ml[base * 2] = m_run;
    a.ws_ml[base * 2 + 1] = l_run;
  }
}

// Combines the split partials of one output row (request c, block position j, query
// head h): o = sum_q 2^(m_q - M) acc_q / sum_q 2^(m_q - M) l_q, M = max m_q.  W warps
// share a row, warp w taking partials q = w, w + W, ... (with few rows the partial
// loads of a row then spread over W warps); the warps' (M_w, L_w, o_w) are combined in
// warp order, so the result does not depend on timing.  V4: a lane holds elements
// 4 lane .. 4 lane + 3 (float4 loads); else lane + 32 i.
template <typename T, int W, bool V4>
__global__ void __launch_bounds__(256) attn_merge_kernel(AttnArgs a) {
  pdl_wait();  // the previous kernel on the stream is complete from here on
  pdl_trigger();
  constexpr int RPC = 8 / W;  // rows per CTA
  __shared__ float s_acc[W > 1 ? 8 : 1][128];
  __shared__ float s_ml[8][2];
  const int wib = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int wq = wib % W, rl = wib / W;
  const int G = a.Hq / a.Hkv, R = a.K * G;
  const long rows = (long)a.C * a.K * a.Hq;
  const long row_id = (long)blockIdx.x * RPC + rl;
  const bool live = row_id < rows;
  const int rid = live ? (int)row_id : 0;
  const int h = rid % a.Hq;
  const int j = (rid / a.Hq) % a.K;
  const int c = rid / (a.Hq * a.K);
  const int g = h / G, row = j * G + h % G;
  const int ctx = a.ctx_lens[c];
  const bool valid = live && ctx >= 0 && ctx <= a.max_pages * a.page_size;
  // Partials of the row: q = 0 .. ns - 1 at rows base0 + q * stride.
  //   fp32 path: one per split of (c, g).
  //   tensor-core path: the sequence (c, rb, g) holds t_seq tiles from unit s0 of the
  //   line cut into chunks of Z units; its piece p in chunk k0 + p has slot
  //   c * spr + rb * Hkv + g + k0 + p, two halves each, so q = 2 p + half.  Half h of
  //   a piece holds its tiles of parity h: it exists iff the piece has more than h
  //   tiles (a missing partial is never written, and its weight is 0).
  // A partial with l = 0 saw no key and is skipped.
  int ns = 0, s0 = 0, k0 = 0, t_seq = 0, Z = 1;
  size_t base0 = 0, stride = R;
  if (a.tile_pieces) {
    const int* off = a.sched + 64;
    const int n_rb = (R + kAttnTcRows - 1) / kAttnTcRows, spr = a.Hkv * n_rb;
    const int rb = row / kAttnTcRows, rr = row % kAttnTcRows;
    const int r = rb * a.Hkv + g;
    Z = a.sched[2];
    stride = R < kAttnTcRows ? R : kAttnTcRows;
    if (valid) {
      // the sequence's units on the line: kAttnSeqUnits start units, then its tiles
      const int tw = (off[c + 1] - off[c]) / spr;
      t_seq = tw - kAttnSeqUnits;
      s0 = off[c] + r * tw + kAttnSeqUnits;
      k0 = s0 / Z;
      ns = t_seq > 0 ? 2 * ((s0 + t_seq - 1) / Z - k0 + 1) : 0;
    }
    base0 = ((size_t)c * spr + r + k0) * 2 * stride + rr;
  } else {
    ns = valid ? (ctx + a.K + a.split_tokens - 1) / a.split_tokens * a.sub_splits : 0;
    base0 = (((size_t)c * a.Hkv + g) * a.n_splits * a.sub_splits) * R + row;
  }
  auto has = [&](int q) -> bool {
    if (!a.tile_pieces) return true;
    const int p = q >> 1, hh = q & 1;
    const int lo = max(s0, (k0 + p) * Z), hi = min(s0 + t_seq, (k0 + p + 1) * Z);
    return hi - lo > hh;
  };
  auto ml_of = [&](int q) -> float2 { return *(const float2*)(a.ws_ml + (base0 + (size_t)q * stride) * 2); };
  // This warp's partials q = wq + W k, k < nk, in blocks of 4: the (m, l) and the rows
  // of a block are loaded together (one round trip), then folded into the running
  // (M, L, o), rescaled when the block raises the max -- one pass of the softmax merge
  // in a fixed order.  A missing partial is read (in range) but not used.
  const int nk = ns > wq ? (ns - wq + W - 1) / W : 0;
  float M = -INFINITY, L = 0.f;
  float o[4] = {0.f, 0.f, 0.f, 0.f};
  const bool v4_lane = V4 && 4 * lane < a.D;
  for (int k0 = 0; k0 < nk; k0 += 4) {
    float2 ml[4];
    float x[4][4];
    bool use[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int k = k0 + u;
      const int q = wq + W * min(k, nk - 1);
      use[u] = k < nk && has(q);
      ml[u] = ml_of(q);
      const float* accp = a.ws_acc + (base0 + (size_t)q * stride) * a.D;
      if (V4) {
        float4 f = make_float4(0.f, 0.f, 0.f, 0.f);
        if (v4_lane) f = *(const float4*)(accp + 4 * lane);
        x[u][0] = f.x, x[u][1] = f.y, x[u][2] = f.z, x[u][3] = f.w;
      } else {
#pragma unroll
        for (int i = 0; i < 4; ++i) x[u][i] = lane + 32 * i < a.D ? accp[lane + 32 * i] : 0.f;
      }
    }
    float mb = M;
#pragma unroll
    for (int u = 0; u < 4; ++u)
      if (use[u] && ml[u].y > 0.f) mb = fmaxf(mb, ml[u].x);
    if (mb == -INFINITY) continue;  // no partial with keys yet
    const float sc = M == -INFINITY ? 0.f : exp2f(M - mb);
    L *= sc;
#pragma unroll
    for (int i = 0; i < 4; ++i) o[i] *= sc;
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      if (!(use[u] && ml[u].y > 0.f)) continue;
      const float w = exp2f(ml[u].x - mb);
      L = fmaf(w, ml[u].y, L);
#pragma unroll
      for (int i = 0; i < 4; ++i) o[i] = fmaf(w, x[u][i], o[i]);
    }
    M = mb;
  }
  T* out = (T*)a.out + (size_t)(c * a.K + j) * a.o_rs + (size_t)h * a.D;
  auto store = [&](const float* v, float inv) {
    if (V4) {
      if (v4_lane)
#pragma unroll
        for (int i = 0; i < 4; ++i) out[4 * lane + i] = from_f<T>(v[i] * inv);
    } else {
#pragma unroll
      for (int i = 0; i < 4; ++i)
        if (lane + 32 * i < a.D) out[lane + 32 * i] = from_f<T>(v[i] * inv);
    }
  };
  if constexpr (W == 1) {
    if (live) store(o, L > 0.f ? 1.f / L : 0.f);
  } else {
    // the W warps of the row: (M_w, L_w, o_w) through shared memory, combined in order
#pragma unroll
    for (int i = 0; i < 4; ++i) s_acc[wib][V4 ? 4 * lane + i : lane + 32 * i] = o[i];
    if (lane == 0) s_ml[wib][0] = M, s_ml[wib][1] = L;
    __syncthreads();
    if (wq == 0 && live) {
      float Mx = -INFINITY;
#pragma unroll
      for (int w = 0; w < W; ++w)
        if (s_ml[rl * W + w][1] > 0.f) Mx = fmaxf(Mx, s_ml[rl * W + w][0]);
      float Lt = 0.f, ot[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int w = 0; w < W; ++w) {
        const int src = rl * W + w;
        if (!(s_ml[src][1] > 0.f)) continue;
        const float sc = exp2f(s_ml[src][0] - Mx);
        Lt += sc * s_ml[src][1];
#pragma unroll
        for (int i = 0; i < 4; ++i) ot[i] = fmaf(sc, s_acc[src][V4 ? 4 * lane + i : lane + 32 * i], ot[i]);
      }
      store(ot, Lt > 0.f ? 1.f / Lt : 0.f);
    }
  }
}

template <typename T, int TPR>
void launch_split(const AttnArgs& a, cudaStream_t s) {
  const size_t smem = (size_t)2 * kTile * (a.D + 1) * sizeof(float);
  const float scale_log2 = 1.4426950408889634f / sqrtf((float)a.D);
  launch_pdl(attn_split_kernel<T, TPR>, dim3(a.n_splits, a.Hkv, a.C), kThreads, smem, s, a, scale_log2);
  note_launch();
}

template <typename T>
void launch_simt(const AttnArgs& a, cudaStream_t s) {
  const int R = a.K * (a.Hq / a.Hkv);
  int rows_cap = 1;
  while (rows_cap < R) rows_cap <<= 1;
  const int tpr = kThreads / rows_cap;  // lanes per query row (power of two, 1..32)
  switch (tpr >= 32 ? 32 : tpr) {
    case 32: launch_split<T, 32>(a, s); break;
    case 16: launch_split<T, 16>(a, s); break;
    case 8: launch_split<T, 8>(a, s); break;
    case 4: launch_split<T, 4>(a, s); break;
    case 2: launch_split<T, 2>(a, s); break;
    default: launch_split<T, 1>(a, s); break;
  }
}

template <typename T, int W>
void launch_merge_w(const AttnArgs& a, long rows, cudaStream_t s) {
  const int grid = (int)((rows + 8 / W - 1) / (8 / W));
  if (a.D % 4 == 0) launch_pdl(attn_merge_kernel<T, W, true>, grid, 256, 0, s, a);
  else launch_pdl(attn_merge_kernel<T, W, false>, grid, 256, 0, s, a);
  note_launch();
}

template <typename T>
void launch_merge(const AttnArgs& a, cudaStream_t s) {
  // warps per output row: enough warps in all for about 32 per SM
  const long rows = (long)a.C * a.K * a.Hq;
  int W = 1;
  while (W < 8 && rows * W < 148L * 32) W *= 2;
  switch (W) {
    case 1: launch_merge_w<T, 1>(a, rows, s); break;
    case 2: launch_merge_w<T, 2>(a, rows, s); break;
    case 4: launch_merge_w<T, 4>(a, rows, s); break;
    default: launch_merge_w<T, 8>(a, rows, s); break;
  }
}

}  // namespace

bool attn_supported(int dtype, int K, int G, int D, const char** why) {
  if (K < 1 || K > 64) return *why = "K must be in 1..64", false;
  if (dtype == HSPEC_DTYPE_BF16) {
    if (D != 64 && D != 128) return *why = "bf16 attention needs head_dim 64 or 128", false;
    return true;
  }
  // fp32: one CTA holds all R = K*G query rows; a lane holds at most 128/TPR dims
  const int R = K * G;
  int cap = 1;
  while (cap < R) cap <<= 1;
  if (cap > kThreads || D > 128 || D % 2) return *why = "fp32 attention needs K*G <= 256 and head_dim <= 128", false;
  int tpr = kThreads / cap;
  if (tpr > 32) tpr = 32;
  if (D % tpr) return *why = "head_dim not divisible by lanes per row", false;
  return true;
}

int attn_split_tokens(int dtype, int C, int Hkv, int K, int max_ctx, int requested) {
  // tensor-core path: the requested chunk length in tokens (whole 64-token units of the
  // partition's line), or 0
  // for one chunk per SM, chosen on the device from the actual context lengths
  if (dtype == HSPEC_DTYPE_BF16) return requested > 0 ? ((requested + 63) / 64) * 64 : 0;
  if (requested > 0) return requested;
  const long target_ctas = 148L * 16;
  long per = ((long)C * Hkv * (max_ctx + K) + target_ctas - 1) / target_ctas;
  per = ((per + 63) / 64) * 64;
  if (per < 64) per = 64;
  return (int)per;
}

int attn_num_splits(int dtype, int K, int max_ctx, int split_tokens) {
  if (dtype == HSPEC_DTYPE_BF16) return 0;
  return (max_ctx + K + split_tokens - 1) / split_tokens;
}

int attn_sub_splits(int dtype) { return dtype == HSPEC_DTYPE_BF16 ? 2 : 1; }

size_t attn_partial_rows(int dtype, int C, int Hkv, int K, int G, int n_splits, int max_chunks) {
  const int R = K * G;
  if (dtype == HSPEC_DTYPE_BF16) {
    // a slot per (sequence, chunk) piece: at most C * Hkv * n_rb + chunks slots, two
    // halves of a row block each
    const int n_rb = (R + kAttnTcRows - 1) / kAttnTcRows;
    const size_t slots = (size_t)C * Hkv * n_rb + max_chunks;
    return slots * 2 * (R < kAttnTcRows ? R : kAttnTcRows);
  }
  return (size_t)C * Hkv * n_splits * R;
}

size_t attn_ws_bytes(int dtype, int C, int Hkv, int K, int G, int D, int n_splits, int max_chunks) {
  const size_t rows = attn_partial_rows(dtype, C, Hkv, K, G, n_splits, max_chunks);
  // + the schedule words (256 bytes) and the requests' offsets on the line (C + 1)
  return rows * D * sizeof(float) + rows * 2 * sizeof(float) + 256 + (size_t)(C + 1) * sizeof(int);
}

bool attn_paged(int dtype, const AttnArgs& a, cudaStream_t s) {
  if (dtype == HSPEC_DTYPE_BF16) {
    const char* why = "";
    if (!attn_tc_supported(a, &why)) {
      set_error("paged attention: %s", why);
      return false;
    }
    if (!attn_tc_launch(a, s)) return false;
    launch_merge<bf16>(a, s);
  } else {
    launch_simt<float>(a, s);
    launch_merge<float>(a, s);
  }
  return true;
}

}  // namespace hspec
