// Row-wise kernels of the draft step: embedding gather, RMSNorm, the Mamba-2 gated
// RMSNorm, rotary embedding and the final argmax reduction.  All are HBM-bound
// streaming kernels: one CTA per row (or per group of rows), fp32 arithmetic,
// coalesced loads along the row.
#include "common.cuh"
#include "kernels.cuh"
#include "../../include/hspec.h"

namespace hspec {
namespace {

constexpr int kRowThreads = 256;

template <typename T>
__global__ void embed_kernel(const int32_t* __restrict__ tokens, const T* __restrict__ table, int vocab,
                             float* __restrict__ x, int d, int* err) {
  pdl_wait();  // the previous kernel on the stream is complete from here on
  pdl_trigger();
  const int m = blockIdx.x;
  const int tok = tokens[m];
  const bool ok = tok >= 0 && tok < vocab;
  if (!ok && threadIdx.x == 0) flag_error(err, kErrTokenOOB);
  for (int e = threadIdx.x; e < d; e += blockDim.x)
    x[(size_t)m * d + e] = ok ? to_f(table[(size_t)tok * d + e]) : 0.f;
}

template <typename T>
__global__ void to_f32_kernel(const T* __restrict__ in, float* __restrict__ x, long n) {
  pdl_wait();  // the previous kernel on the stream is complete from here on
  pdl_trigger();
  for (long i = blockIdx.x * (long)blockDim.x + threadIdx.x; i < n; i += (long)gridDim.x * blockDim.x)
    x[i] = to_f(in[i]);
}

// RMSNorm of one fp32 row per CTA: out = x * rsqrt(mean(x^2) + eps) * w.
template <typename T>
__global__ void rmsnorm_kernel(const float* __restrict__ x, const float* __restrict__ w,
                               T* __restrict__ out, int n, float eps) {
  pdl_wait();  // the previous kernel on the stream is complete from here on
  pdl_trigger();
  __shared__ float red[32];
  const float* row = x + (size_t)blockIdx.x * n;
  float ss = 0.f;
  for (int i = threadIdx.x; i < n; i += blockDim.x) ss += row[i] * row[i];
  ss = block_sum(ss, red);
  const float inv = 1.f / sqrtf(ss / n + eps);  // correctly rounded: fewer bf16 rounding flips
  T* o = out + (size_t)blockIdx.x * n;
  for (int i = threadIdx.x; i < n; i += blockDim.x) o[i] = from_f<T>(row[i] * inv * w[i]);
}

// Vectorised forms for rows of n <= 4 * kRowThreads * kV4 values, n % 4 == 0: one
// pass over global memory, the row held in registers (float4 loads, 8- or 16-byte
// stores).  Same arithmetic per element as the scalar kernels above.
constexpr int kV4 = 8;

__device__ __forceinline__ void store4(bf16* o, float a, float b, float c, float d) {
  __nv_bfloat162 lo = __floats2bfloat162_rn(a, b), hi = __floats2bfloat162_rn(c, d);
  uint2 u;
  u.x = *reinterpret_cast<uint32_t*>(&lo);
  u.y = *reinterpret_cast<uint32_t*>(&hi);
  *(uint2*)o = u;
}
__device__ __forceinline__ void store4(float* o, float a, float b, float c, float d) {
  *(float4*)o = make_float4(a, b, c, d);
}
__device__ __forceinline__ float4 load4(const bf16* p) {
  const uint2 u = *(const uint2*)p;
  const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u.x));
  const float2 b = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u.y));
  return make_float4(a.x, a.y, b.x, b.y);
}
__device__ __forceinline__ float4 load4(const float* p) { return *(const float4*)p; }

template <typename T>
__global__ void __launch_bounds__(kRowThreads) rmsnorm_v4_kernel(const float* __restrict__ x,
                                                                 const float* __restrict__ w,
                                                                 T* __restrict__ out, int n, float eps) {
  pdl_wait();  // the previous kernel on the stream is complete from here on
  pdl_trigger();
  __shared__ float red[32];
  const int n4 = n / 4;
  const float4* row = (const float4*)(x + (size_t)blockIdx.x * n);
  float4 v[kV4];
  float ss = 0.f;
#pragma unroll
  for (int k = 0; k < kV4; ++k) {
    const int i = threadIdx.x + k * kRowThreads;
    v[k] = i < n4 ? row[i] : make_float4(0.f, 0.f, 0.f, 0.f);
    ss += v[k].x * v[k].x + v[k].y * v[k].y + v[k].z * v[k].z + v[k].w * v[k].w;
  }
  ss = block_sum(ss, red);
  const float inv = 1.f / sqrtf(ss / n + eps);  // correctly rounded: fewer bf16 rounding flips
  T* o = out + (size_t)blockIdx.x * n;
#pragma unroll
  for (int k = 0; k < kV4; ++k) {
    const int i = threadIdx.x + k * kRowThreads;
    if (i < n4) {
      const float4 ww = ((const float4*)w)[i];
      store4(o + 4 * i, v[k].x * inv * ww.x, v[k].y * inv * ww.y, v[k].z * inv * ww.z, v[k].w * inv * ww.w);
    }
  }
}

template <typename T>
__global__ void __launch_bounds__(kRowThreads) gated_rmsnorm_v4_kernel(const float* __restrict__ y,
                                                                       const T* __restrict__ z, long z_stride,
                                                                       const float* __restrict__ w,
                                                                       T* __restrict__ out, int n, float eps) {
  pdl_wait();  // the previous kernel on the stream is complete from here on
  pdl_trigger();
  __shared__ float red[32];
  const int n4 = n / 4;
  const float* yr = y + (size_t)blockIdx.x * n;
  const T* zr = z + (size_t)blockIdx.x * z_stride;
  float4 gv[kV4];
  float ss = 0.f;
#pragma unroll
  for (int k = 0; k < kV4; ++k) {
    const int i = threadIdx.x + k * kRowThreads;
    if (i < n4) {
      const float4 yy = ((const float4*)yr)[i];
      const float4 zz = load4(zr + 4 * i);
      gv[k] = make_float4(yy.x * silu(zz.x), yy.y * silu(zz.y), yy.z * silu(zz.z), yy.w * silu(zz.w));
    } else {
      gv[k] = make_float4(0.f, 0.f, 0.f, 0.f);
    }
    ss += gv[k].x * gv[k].x + gv[k].y * gv[k].y + gv[k].z * gv[k].z + gv[k].w * gv[k].w;
  }
  ss = block_sum(ss, red);
  const float inv = 1.f / sqrtf(ss / n + eps);
  T* o = out + (size_t)blockIdx.x * n;
#pragma unroll
  for (int k = 0; k < kV4; ++k) {
    const int i = threadIdx.x + k * kRowThreads;
    if (i < n4) {
      const float4 ww = ((const float4*)w)[i];
      store4(o + 4 * i, gv[k].x * inv * ww.x, gv[k].y * inv * ww.y, gv[k].z * inv * ww.z, gv[k].w * inv * ww.w);
    }
  }
}

// Rotate-half RoPE in place with one angle per (row, pair i), shared by all heads:
// CTA = row; thread t takes pair i = t % (D/2) of heads t / (D/2), + groups, ....
template <typename T>
__global__ void __launch_bounds__(kRowThreads) rope_rows_kernel(T* __restrict__ qkv, long row_stride,
                                                                const int32_t* __restrict__ ctx_lens, int K,
                                                                int n_heads, int D, double log_theta) {
  pdl_wait();  // the previous kernel on the stream is complete from here on
  pdl_trigger();
  const int half = D / 2, groups = kRowThreads / half;
  const int t = threadIdx.x, i = t % half, hg = t / half;
  if (hg >= groups) return;
  const long m = blockIdx.x;
  const int c = (int)(m / K), j = (int)(m % K);
  const double pos = (double)ctx_lens[c] + j;
  const double ang = pos * exp(-2.0 * i / D * log_theta);
  double sn, cs;
  sincos(ang, &sn, &cs);
  T* row = qkv + m * row_stride;
  for (int h = hg; h < n_heads; h += groups) {
    T* v = row + (long)h * D;
    const double a = to_f(v[i]), b = to_f(v[i + half]);
    v[i] = from_f<T>((float)(a * cs - b * sn));
    v[i + half] = from_f<T>((float)(a * sn + b * cs));
  }
}

// Mamba-2 output gate: g = y * silu(z), then RMSNorm over the H*P features.
template <typename T>
__global__ void gated_rmsnorm_kernel(const float* __restrict__ y, const T* __restrict__ z, long z_stride,
                                     const float* __restrict__ w, T* __restrict__ out, int n, float eps,
                                     bool gate) {
  pdl_wait();  // the previous kernel on the stream is complete from here on
  pdl_trigger();
  __shared__ float red[32];
  const float* yr = y + (size_t)blockIdx.x * n;
  T* o = out + (size_t)blockIdx.x * n;
  if (!gate) {
    for (int i = threadIdx.x; i < n; i += blockDim.x) o[i] = from_f<T>(yr[i]);
    return;
  }
  const T* zr = z + (size_t)blockIdx.x * z_stride;
  float ss = 0.f;
  for (int i = threadIdx.x; i < n; i += blockDim.x) {
    float g = yr[i] * silu(to_f(zr[i]));
    ss += g * g;
  }
  ss = block_sum(ss, red);
  const float inv = 1.f / sqrtf(ss / n + eps);
  for (int i = threadIdx.x; i < n; i += blockDim.x)
    o[i] = from_f<T>(yr[i] * silu(to_f(zr[i])) * inv * w[i]);
}

// Rotate-half RoPE in place.  One thread per (row, head, pair i); the angle
// pos * theta^(-2i/D) is formed and reduced in double so that positions up to
// 10^5 keep full fp32 accuracy in cos/sin.
template <typename T>
__global__ void rope_kernel(T* __restrict__ qkv, long row_stride, const int32_t* __restrict__ ctx_lens,
                            int K, int n_heads, int D, double log_theta, long total) {
  pdl_wait();  // the previous kernel on the stream is complete from here on
  pdl_trigger();
  const long idx = blockIdx.x * (long)blockDim.x + threadIdx.x;
  if (idx >= total) return;
  const int half = D / 2;
  const int i = (int)(idx % half);
  const long rh = idx / half;
  const int h = (int)(rh % n_heads);
  const long m = rh / n_heads;
  const int c = (int)(m / K), j = (int)(m % K);
  const double pos = (double)ctx_lens[c] + j;
  const double ang = pos * exp(-2.0 * i / D * log_theta);
  double sn, cs;
  sincos(ang, &sn, &cs);
  T* v = qkv + m * row_stride + (long)h * D;
  const double a = to_f(v[i]), b = to_f(v[i + half]);
  v[i] = from_f<T>((float)(a * cs - b * sn));
  v[i + half] = from_f<T>((float)(a * sn + b * cs));
}

// cos and sin of the rotate-half RoPE angle of every (row m = c*K + j, pair i < D/2):
// pos * theta^(-2i/D) with pos = ctx_lens[c] + j, formed and evaluated in double (as the
// row kernel above does), stored as fp32 pairs; the attention projection GEMM's
// epilogue reads them.
__global__ void rope_table_kernel(float2* __restrict__ cs, const int32_t* __restrict__ ctx_lens, int K, int half,
                                  double log_theta, long total) {
  pdl_wait();  // the previous kernel on the stream is complete from here on
  pdl_trigger();
  const long idx = blockIdx.x * (long)blockDim.x + threadIdx.x;
  if (idx >= total) return;
  const int i = (int)(idx % half);
  const long m = idx / half;
  const double pos = (double)ctx_lens[m / K] + (double)(m % K);
  const double ang = pos * exp(-2.0 * i / (2 * half) * log_theta);
  double sn, c;
  sincos(ang, &sn, &c);
  cs[idx] = make_float2((float)c, (float)sn);
}

// One warp per row: scans the per-tile partial maxima in column order, keeping
// the first (lowest id) of equal maxima.
__global__ void argmax_reduce_kernel(const float* __restrict__ pval, const int32_t* __restrict__ pidx,
                                     int M, int n_parts, int32_t* __restrict__ tokens,
                                     float* __restrict__ top, const int32_t* __restrict__ map, int vocab,
                                     int* err) {
  pdl_wait();  // the previous kernel on the stream is complete from here on
  pdl_trigger();
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5, lane = threadIdx.x & 31;
  if (warp >= M) return;
  float best = -INFINITY;
  int bidx = 0x7fffffff;
  for (int p = lane; p < n_parts; p += 32) {
    float v = pval[(size_t)warp * n_parts + p];
    int id = pidx[(size_t)warp * n_parts + p];
    if (v > best || (v == best && id < bidx)) best = v, bidx = id;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    float v = __shfl_xor_sync(0xffffffffu, best, o);
    int id = __shfl_xor_sync(0xffffffffu, bidx, o);
    if (v > best || (v == best && id < bidx)) best = v, bidx = id;
  }
  if (lane == 0) {
    int tok = bidx;
    if (map) {  // reduced draft head: row -> target token id
      tok = map[bidx];
      if (tok < 0 || tok >= vocab) {
        flag_error(err, kErrTokenOOB);
        tok = -1;
      }
    }
    tokens[warp] = tok;
    if (top) top[warp] = best;
  }
}

}  // namespace

void embed_rows(int dtype, const int32_t* tokens, const void* table, int vocab, float* x, int M, int d,
                int* err, cudaStream_t s) {
  if (dtype == HSPEC_DTYPE_BF16)
    launch_pdl(embed_kernel<bf16>, M, kRowThreads, 0, s, tokens, (const bf16*)table, vocab, x, d, err);
  else
    launch_pdl(embed_kernel<float>, M, kRowThreads, 0, s, tokens, (const float*)table, vocab, x, d, err);
  note_launch();
}

void rows_to_f32(int dtype, const void* in, float* x, long n, cudaStream_t s) {
  int grid = (int)((n + kRowThreads - 1) / kRowThreads);
  if (grid > 148 * 16) grid = 148 * 16;
  if (dtype == HSPEC_DTYPE_BF16)
    launch_pdl(to_f32_kernel<bf16>, grid, kRowThreads, 0, s, (const bf16*)in, x, n);
  else
    launch_pdl(to_f32_kernel<float>, grid, kRowThreads, 0, s, (const float*)in, x, n);
  note_launch();
}

void rmsnorm_rows(int dtype, const float* x, const float* w, void* out, int M, int n, float eps,
                  cudaStream_t s) {
  const bool v4 = n % 4 == 0 && n <= 4 * kRowThreads * kV4 && !(((uintptr_t)x | (uintptr_t)w | (uintptr_t)out) & 15);
  if (v4) {
    if (dtype == HSPEC_DTYPE_BF16) launch_pdl(rmsnorm_v4_kernel<bf16>, M, kRowThreads, 0, s, x, w, (bf16*)out, n, eps);
    else launch_pdl(rmsnorm_v4_kernel<float>, M, kRowThreads, 0, s, x, w, (float*)out, n, eps);
  } else if (dtype == HSPEC_DTYPE_BF16)
    launch_pdl(rmsnorm_kernel<bf16>, M, kRowThreads, 0, s, x, w, (bf16*)out, n, eps);
  else
    launch_pdl(rmsnorm_kernel<float>, M, kRowThreads, 0, s, x, w, (float*)out, n, eps);
  note_launch();
}

void gated_rmsnorm_rows(int dtype, const float* y, const void* z, long z_stride, const float* w,
                        void* out, int M, int n, float eps, bool gate, cudaStream_t s) {
  const int zb = dtype == HSPEC_DTYPE_BF16 ? 2 : 4;
  const bool v4 = gate && n % 4 == 0 && n <= 4 * kRowThreads * kV4 && (z_stride * zb) % 16 == 0 &&
                  !(((uintptr_t)y | (uintptr_t)w | (uintptr_t)out) & 15) && !(((uintptr_t)z) & 7);
  if (v4) {
    if (dtype == HSPEC_DTYPE_BF16)
      launch_pdl(gated_rmsnorm_v4_kernel<bf16>, M, kRowThreads, 0, s, y, (const bf16*)z, z_stride, w, (bf16*)out, n, eps);
    else
      launch_pdl(gated_rmsnorm_v4_kernel<float>, M, kRowThreads, 0, s, y, (const float*)z, z_stride, w, (float*)out, n,
                                                               eps);
  } else if (dtype == HSPEC_DTYPE_BF16)
    launch_pdl(gated_rmsnorm_kernel<bf16>, M, kRowThreads, 0, s, y, (const bf16*)z, z_stride, w, (bf16*)out, n,
                                                         eps, gate);
  else
    launch_pdl(gated_rmsnorm_kernel<float>, M, kRowThreads, 0, s, y, (const float*)z, z_stride, w, (float*)out,
                                                          n, eps, gate);
  note_launch();
}

void rope_rows(int dtype, void* qkv, long row_stride, const int32_t* ctx_lens, int C, int K,
               int n_heads, int D, float theta, cudaStream_t s) {
  const long total = (long)C * K * n_heads * (D / 2);
  const int grid = (int)((total + kRowThreads - 1) / kRowThreads);
  const double lt = log((double)theta);
  if (D % 2 == 0 && D / 2 <= kRowThreads) {
    if (dtype == HSPEC_DTYPE_BF16)
      launch_pdl(rope_rows_kernel<bf16>, C * K, kRowThreads, 0, s, (bf16*)qkv, row_stride, ctx_lens, K, n_heads, D, lt);
    else
      launch_pdl(rope_rows_kernel<float>, C * K, kRowThreads, 0, s, (float*)qkv, row_stride, ctx_lens, K, n_heads, D, lt);
  } else if (dtype == HSPEC_DTYPE_BF16)
    launch_pdl(rope_kernel<bf16>, grid, kRowThreads, 0, s, (bf16*)qkv, row_stride, ctx_lens, K, n_heads, D, lt,
                                                   total);
  else
    launch_pdl(rope_kernel<float>, grid, kRowThreads, 0, s, (float*)qkv, row_stride, ctx_lens, K, n_heads, D,
                                                    lt, total);
  note_launch();
}

void rope_table(float2* cs, const int32_t* ctx_lens, int C, int K, int D, float theta, cudaStream_t s) {
  const long total = (long)C * K * (D / 2);
  const int grid = (int)((total + kRowThreads - 1) / kRowThreads);
  launch_pdl(rope_table_kernel, grid, kRowThreads, 0, s, cs, ctx_lens, K, D / 2, log((double)theta), total);
  note_launch();
}

void argmax_reduce(const float* pval, const int32_t* pidx, int M, int n_parts, int32_t* tokens,
                   float* top, const int32_t* map, int vocab, int* err, cudaStream_t s) {
  const int warps_per_block = 8;
  launch_pdl(argmax_reduce_kernel, (M + warps_per_block - 1) / warps_per_block, 32 * warps_per_block, 0, s, pval, pidx, M, n_parts, tokens, top, map, vocab, err);
  note_launch();
}

}  // namespace hspec
