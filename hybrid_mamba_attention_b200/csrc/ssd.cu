// Mamba-2 SSD block scan from an injected initial state, in chunks of Q positions
// (H-Spec Abstract: Mamba's parallel scan keeps drafting block-parallel; the chunked
// "state-space dual" evaluation of Dao & Gu, 2024).  One CTA per (head h, request c):
//
//   for each chunk [k0, k0+q):
//     cum_t  = sum_{r=k0..t} dt_r A_h                       (prefix within the chunk)
//     CB_ts  = C_t . B_s                                     (shared by all heads)
//     y_t[p] = exp(cum_t) sum_n C_t[n] S[p][n]               (state entering the chunk)
//            + sum_{s<=t} CB_ts exp(cum_t - cum_s) dt_s x_s[p]  (inside the chunk)
//            + D_h x_t[p]
//     S      <- exp(cum_last) S + sum_s exp(cum_last - cum_s) dt_s x_s (x) B_s
//
// which equals the step-by-step recurrence h_t = exp(dt_t A) h_{t-1} + dt_t x_t (x) B_t,
// y_t = C_t . h_t + D x_t.  The state S [P][N] lives in shared memory in fp32 (padded
// rows so that a warp reading one column across 32 rows hits 32 banks); the chunk
// pass between chunks is the only sequential part.  Everything is fp32 FMA.
#include "../../include/hspec.h"
#include "common.cuh"
#include "kernels.cuh"

namespace hspec {
namespace {

constexpr int kThreads = 256;

struct SsdSmem {
  // offsets in floats
  int S, xs, Bs, Cs, dts, cum, w, CB, total;
};

__host__ __device__ inline SsdSmem ssd_layout(int P, int N, int Q) {
  SsdSmem L;
  const int Np = N + 1, Qp = Q + 1;
  L.S = 0;
  L.xs = L.S + P * Np;
  L.Bs = L.xs + Q * P;
  L.Cs = L.Bs + Q * Np;
  L.dts = L.Cs + Q * Np;
  L.cum = L.dts + Q;
  L.w = L.cum + Q;
  L.CB = L.w + Q;
  L.total = L.CB + Q * Qp;
  return L;
}

template <typename T, typename TDT>
__global__ void __launch_bounds__(kThreads) ssd_chunk_kernel(SsdArgs a) {
  extern __shared__ float sm[];
  const int h = blockIdx.x, c = blockIdx.y;
  const int P = a.P, N = a.N, K = a.K, Q = a.Q, Np = N + 1, Qp = Q + 1;
  const SsdSmem L = ssd_layout(P, N, Q);
  float* S = sm + L.S;
  float* xs = sm + L.xs;
  float* Bs = sm + L.Bs;
  float* Cs = sm + L.Cs;
  float* dts = sm + L.dts;
  float* cum = sm + L.cum;
  float* w = sm + L.w;
  float* CB = sm + L.CB;
  const T* x = (const T*)a.x;
  const T* B = (const T*)a.B;
  const T* Cm = (const T*)a.Cm;
  const TDT* dt = (const TDT*)a.dt;
  const float Ah = a.A[h], Dh = a.D[h];

  // initial state (the injected h0, or zero)
  const float* h0 = a.h0 ? a.h0 + ((size_t)c * a.H + h) * P * N : nullptr;
  for (int i = threadIdx.x; i < P * N; i += kThreads) S[(i / N) * Np + i % N] = h0 ? h0[i] : 0.f;

  for (int k0 = 0; k0 < K; k0 += Q) {
    const int q = min(Q, K - k0);
    __syncthreads();  // previous chunk finished with xs/Bs/Cs/S
    for (int i = threadIdx.x; i < q * P; i += kThreads) {
      const int t = i / P, p = i % P;
      xs[t * P + p] = to_f(x[(size_t)(c * K + k0 + t) * a.x_rs + (size_t)h * P + p]);
    }
    for (int i = threadIdx.x; i < q * N; i += kThreads) {
      const int t = i / N, n = i % N;
      const size_t row = (size_t)(c * K + k0 + t) * a.bc_rs;
      Bs[t * Np + n] = to_f(B[row + n]);
      Cs[t * Np + n] = to_f(Cm[row + n]);
    }
    if (threadIdx.x < q) {
      const int t = threadIdx.x;
      float d = to_f(dt[(size_t)(c * K + k0 + t) * a.dt_rs + h]);
      if (a.dt_bias) d = softplus(d + a.dt_bias[h]);
      dts[t] = d;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
      float run = 0.f;
      for (int t = 0; t < q; ++t) {
        run += dts[t] * Ah;
        cum[t] = run;
      }
      for (int t = 0; t < q; ++t) w[t] = expf(run - cum[t]) * dts[t];  // weight into the chunk-end state
    }
    for (int i = threadIdx.x; i < q * q; i += kThreads) {
      const int t = i / q, s = i % q;
      float acc = 0.f;
      if (s <= t)
        for (int n = 0; n < N; ++n) acc = fmaf(Cs[t * Np + n], Bs[s * Np + n], acc);
      CB[t * Qp + s] = acc;
    }
    __syncthreads();

    // outputs of the chunk: lanes run over p (consecutive), so S[p][n] reads are conflict-free
    for (int i = threadIdx.x; i < q * P; i += kThreads) {
      const int t = i / P, p = i % P;
      const float* Sp = S + p * Np;
      const float* Ct = Cs + t * Np;
      float off = 0.f;
      for (int n = 0; n < N; ++n) off = fmaf(Ct[n], Sp[n], off);
      float acc = expf(cum[t]) * off;
      for (int s = 0; s <= t; ++s) acc = fmaf(CB[t * Qp + s] * expf(cum[t] - cum[s]) * dts[s], xs[s * P + p], acc);
      acc = fmaf(Dh, xs[t * P + p], acc);
      a.y[(size_t)(c * K + k0 + t) * a.y_rs + (size_t)h * P + p] = acc;
    }

    // state pass to the next chunk (or to the final state)
    if (k0 + q < K || a.hK) {
      __syncthreads();  // all reads of S for the outputs are done
      const float decay = expf(cum[q - 1]);
      for (int i = threadIdx.x; i < P * N; i += kThreads) {
        const int p = i / N, n = i % N;
        float v = decay * S[p * Np + n];
        for (int s = 0; s < q; ++s) v = fmaf(w[s] * xs[s * P + p], Bs[s * Np + n], v);
        S[p * Np + n] = v;
      }
    }
  }
  if (a.hK) {
    __syncthreads();
    float* out = a.hK + ((size_t)c * a.H + h) * P * N;
    for (int i = threadIdx.x; i < P * N; i += kThreads) out[i] = S[(i / N) * Np + i % N];
  }
}

template <typename T, typename TDT>
void launch(const SsdArgs& a, cudaStream_t s) {
  const size_t bytes = ssd_smem_bytes(a.P, a.N, a.Q);
  static bool attr_set[64] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 64 && !attr_set[dev]) {
    cudaFuncSetAttribute(ssd_chunk_kernel<T, TDT>, cudaFuncAttributeMaxDynamicSharedMemorySize, 227 * 1024);
    attr_set[dev] = true;
  }
  ssd_chunk_kernel<T, TDT><<<dim3(a.H, a.C), kThreads, bytes, s>>>(a);
  note_launch();
}

}  // namespace

size_t ssd_smem_bytes(int P, int N, int Q) { return (size_t)ssd_layout(P, N, Q).total * sizeof(float); }

void ssd_scan(int dtype, const SsdArgs& a, cudaStream_t s) {
  if (dtype == HSPEC_DTYPE_BF16) {
    if (a.dt_bias) launch<bf16, bf16>(a, s);
    else launch<bf16, float>(a, s);
  } else {
    launch<float, float>(a, s);
  }
}

}  // namespace hspec
