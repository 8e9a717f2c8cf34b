// Greedy verification of the K drafts of every request against the target's logits:
// standard speculative-decoding verification, which H-Spec keeps (evolve.pub review of
// H-Spec, Frequently asked questions: the target's verification is what makes the
// output exact).  Row j of request c holds the target's logits for block position j
// (K + 1 rows: after the context, and after each draft):
//   t_j = argmax_v logits[c][j][v]           lowest id on ties; NaN never wins
//   a   = longest prefix j < K with drafts[c][j] == t_j
//   next_token = t_a;  ctx_lens[c] += a + 1   (the K - a rejected positions roll back)
//
// The logits are the only large operand (C (K+1) V elements, read once): a partial
// argmax kernel streams them, one CTA per (row, 32 KB chunk), every thread issuing all
// its 16-byte loads before the first compare,
// and a second kernel, one warp per request, reduces each row's chunk partials in
// chunk order and applies the prefix rule.  Both orders are fixed, so the result is
// exact and repeatable (max and lowest-index are order-free anyway).
#include <stdint.h>

#include "../../include/hspec.h"
#include "common.cuh"
#include "kernels.cuh"

namespace hspec {
namespace {

constexpr int kThreads = 256;
constexpr int kLoads = 8;  // 16-byte loads per thread per chunk
// logits per chunk: 16384 bf16 or 8192 fp32 (32 KB)
template <typename T>
constexpr int chunk_of() {
  return kThreads * kLoads * (16 / (int)sizeof(T));
}
int chunk_for(int dtype) { return dtype == HSPEC_DTYPE_BF16 ? chunk_of<bf16>() : chunk_of<float>(); }
constexpr int kNone = 0x7fffffff;  // no number seen (yet): loses against any id

// (value, id) a beats (value, id) b: larger value, or equal value and lower id.
__device__ __forceinline__ bool beats(float va, int ia, float vb, int ib) {
  return va > vb || (va == vb && ia < ib);
}

__device__ __forceinline__ void take(float x, int id, float& best, int& bidx) {
  if (!isnan(x) && beats(x, id, best, bidx)) best = x, bidx = id;
}

// One CTA per (row, 32 KB chunk).  Every thread issues its 8 16-byte loads before the
// first compare; vector i of thread t holds elements v0 + (i kThreads + t) VEC + k (a
// warp's loads are contiguous).  Per thread two passes over the registers: the maximum
// (fmax ignores NaN; two bf16 per instruction), then the lowest id holding it; the
// (value, lowest id) pairs of the threads are then combined.
__device__ __forceinline__ float vmax(const uint4& w, float m, float) {
  return fmaxf(fmaxf(fmaxf(fmaxf(m, __uint_as_float(w.x)), __uint_as_float(w.y)), __uint_as_float(w.z)),
               __uint_as_float(w.w));
}
__device__ __forceinline__ float vmax(const uint4& w, float m, bf16) {
  const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&w);
  const __nv_bfloat162 a = __hmax2(__hmax2(h[0], h[1]), __hmax2(h[2], h[3]));
  return fmaxf(m, fmaxf(__bfloat162float(a.x), __bfloat162float(a.y)));
}

template <typename T>
__global__ void __launch_bounds__(kThreads) verify_partial_kernel(const T* __restrict__ logits, int V,
                                                                  int n_chunks, float* __restrict__ pval,
                                                                  int32_t* __restrict__ pidx) {
  pdl_wait();  // the previous kernel on the stream is complete from here on
  pdl_trigger();
  constexpr int VEC = 16 / sizeof(T), kChunk = chunk_of<T>();
  __shared__ float sv[kThreads / 32];
  __shared__ int si[kThreads / 32];
  const long row = blockIdx.x;  // rows on x (up to 2^31 - 1), chunks on y
  const int v0 = blockIdx.y * kChunk, v1 = min(V, v0 + kChunk);
  const T* lr = logits + row * (long)V;
  float best = -INFINITY;
  int bidx = kNone;
  // rows are 16-byte aligned when V * sizeof(T) is; the last chunk of a row may be short
  const bool vec = ((V * sizeof(T)) % 16 == 0) && ((((uintptr_t)logits) & 15) == 0);
  if (vec && v1 - v0 == kChunk) {
    uint4 w[kLoads];
#pragma unroll
    for (int i = 0; i < kLoads; ++i) w[i] = __ldcs((const uint4*)(lr + v0 + (i * kThreads + threadIdx.x) * VEC));
    float m = -INFINITY;
#pragma unroll
    for (int i = 0; i < kLoads; ++i) m = vmax(w[i], m, T());
#pragma unroll
    for (int i = kLoads - 1; i >= 0; --i) {  // from the top, so the last hit is the lowest id
      const T* e = reinterpret_cast<const T*>(&w[i]);
      const int vb = v0 + (i * kThreads + threadIdx.x) * VEC;
#pragma unroll
      for (int k = VEC - 1; k >= 0; --k)
        if (to_f(e[k]) == m) bidx = vb + k;
    }
    best = m;  // -inf with bidx kNone when every element is NaN
  } else {
    for (int v = v0 + threadIdx.x; v < v1; v += kThreads) take(to_f(lr[v]), v, best, bidx);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const float ov = __shfl_xor_sync(0xffffffffu, best, o);
    const int oi = __shfl_xor_sync(0xffffffffu, bidx, o);
    if (beats(ov, oi, best, bidx)) best = ov, bidx = oi;
  }
  const int wp = threadIdx.x >> 5, l = threadIdx.x & 31;
  if (l == 0) sv[wp] = best, si[wp] = bidx;
  __syncthreads();
  if (threadIdx.x == 0) {
    for (int k = 1; k < kThreads / 32; ++k)
      if (beats(sv[k], si[k], best, bidx)) best = sv[k], bidx = si[k];
    pval[row * n_chunks + blockIdx.y] = best;
    pidx[row * n_chunks + blockIdx.y] = bidx;
  }
}

// One warp per request.  Lane l takes row j = j0 + l (its chunk partials, loaded
// together, reduced in chunk order); a ballot of the draft matches gives the prefix
// that ends in this group of rows, and the lane at its end holds the next token.
__global__ void verify_finish_kernel(const float* __restrict__ pval, const int32_t* __restrict__ pidx,
                                     int n_chunks, const int32_t* __restrict__ drafts, int C, int K,
                                     int32_t* __restrict__ accepted, int32_t* __restrict__ next_token,
                                     int32_t* __restrict__ ctx_lens) {
  pdl_wait();  // the previous kernel on the stream is complete from here on
  pdl_trigger();
  const int c = (blockIdx.x * blockDim.x + threadIdx.x) >> 5, lane = threadIdx.x & 31;
  if (c >= C) return;
  for (int j0 = 0; j0 <= K; j0 += 32) {
    const int j = j0 + lane;
    int t = -1;
    bool match = false;
    if (j <= K) {
      const long row = (long)c * (K + 1) + j;
      float best = -INFINITY;
      int bidx = kNone;
      for (int p = 0; p < n_chunks; ++p) {
        const float v = pval[row * n_chunks + p];
        const int i = pidx[row * n_chunks + p];
        if (beats(v, i, best, bidx)) best = v, bidx = i;
      }
      t = bidx == kNone ? -1 : bidx;
      match = j < K && drafts[(long)c * K + j] == t;
    }
    const unsigned m = __ballot_sync(0xffffffffu, match);
    if (m == 0xffffffffu) continue;  // all 32 drafts of this group accepted
    const int r = __ffs(~m) - 1;     // first row of the group that does not match
    const int nxt = __shfl_sync(0xffffffffu, t, r);
    if (lane == 0) {
      const int a = j0 + r;
      accepted[c] = a;
      next_token[c] = nxt;
      if (ctx_lens) ctx_lens[c] += a + 1;
    }
    return;
  }
}

}  // namespace

size_t verify_ws_bytes(int dtype, int C, int K, int V) {
  const size_t rows = (size_t)C * (K + 1), n_chunks = (size_t)cdiv(V, chunk_for(dtype));
  return rows * n_chunks * (sizeof(float) + sizeof(int32_t));
}

void verify_greedy(int dtype, const void* logits, int V, const int32_t* drafts, int C, int K,
                   int32_t* accepted, int32_t* next_token, int32_t* ctx_lens, void* ws, cudaStream_t s) {
  const int n_chunks = cdiv(V, chunk_for(dtype));
  const long rows = (long)C * (K + 1);
  float* pval = (float*)ws;
  int32_t* pidx = (int32_t*)(pval + rows * n_chunks);
  const dim3 grid((unsigned)rows, n_chunks);
  if (dtype == HSPEC_DTYPE_BF16)
    launch_pdl(verify_partial_kernel<bf16>, grid, kThreads, 0, s, (const bf16*)logits, V, n_chunks, pval, pidx);
  else
    launch_pdl(verify_partial_kernel<float>, grid, kThreads, 0, s, (const float*)logits, V, n_chunks, pval, pidx);
  note_launch();
  launch_pdl(verify_finish_kernel, cdiv(C, 8), 256, 0, s, (const float*)pval, (const int32_t*)pidx, n_chunks,
             drafts, C, K, accepted, next_token, ctx_lens);
  note_launch();
}

}  // namespace hspec
