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
// Stateless form (no h0, no final state, one chunk): S is always zero, so it has no
// shared memory and the readout term is skipped -- the in-block terms and D x only
// (the draft step adds the h0 term in the injection GEMM's epilogue).
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

__host__ __device__ inline SsdSmem ssd_layout(int P, int N, int Q, bool stateless = false) {
  SsdSmem L;
  const int Np = N + 1, Qp = Q + 1;
  L.S = 0;
  L.xs = L.S + (stateless ? 0 : P * Np);
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
  pdl_wait();  // the previous kernel on the stream is complete from here on
  pdl_trigger();
  extern __shared__ float sm[];
  const int h = blockIdx.x, c = blockIdx.y;
  const int P = a.P, N = a.N, K = a.K, Q = a.Q, Np = N + 1, Qp = Q + 1;
  const bool stateless = !a.h0 && !a.hK && Q >= K;
  const SsdSmem L = ssd_layout(P, N, Q, stateless);
  float* S = sm + L.S;     // [P][N+1] state entering the chunk
  float* xs = sm + L.xs;   // [Q][P]   x of the chunk (later x * weight into the chunk-end state)
  float* Bs = sm + L.Bs;   // [Q][N+1]
  float* Cs = sm + L.Cs;   // [Q][N+1]
  float* dts = sm + L.dts;
  float* cum = sm + L.cum;
  float* w = sm + L.w;
  float* Lm = sm + L.CB;   // [Q][Q+1]: CB_ts exp(cum_t - cum_s) dt_s for s <= t, else 0
  const T* x = (const T*)a.x;
  const T* B = (const T*)a.B;
  const T* Cm = (const T*)a.Cm;
  const TDT* dt = (const TDT*)a.dt;
  const float Ah = a.A[h], Dh = a.D[h];
  const int tid = threadIdx.x, nq = tid & 3;
  const int n_pb = (P + 3) / 4;

  // initial state (the injected h0, or zero)
  const float* h0 = a.h0 ? a.h0 + ((size_t)c * a.H + h) * P * N : nullptr;
  if (stateless) {
  } else if (h0 && (N % 4) == 0) {
    const float4* h4 = (const float4*)h0;
    for (int i = tid; i < P * N / 4; i += kThreads) {
      const float4 v = h4[i];
      const int e = 4 * i, r = e / N, n = e % N;
      float* d = S + r * Np + n;
      d[0] = v.x, d[1] = v.y, d[2] = v.z, d[3] = v.w;
    }
  } else {
    for (int i = tid; i < P * N; i += kThreads) S[(i / N) * Np + i % N] = h0 ? h0[i] : 0.f;
  }

  for (int k0 = 0; k0 < K; k0 += Q) {
    const int q = min(Q, K - k0);
    const int n_tb = (q + 3) / 4;
    __syncthreads();  // the previous chunk is done with xs / Bs / Cs / S
    for (int i = tid; i < q * P; i += kThreads) {
      const int t = i / P, p = i % P;
      xs[t * P + p] = to_f(x[(size_t)(c * K + k0 + t) * a.x_rs + (size_t)h * P + p]);
    }
    for (int i = tid; i < q * N; i += kThreads) {
      const int t = i / N, n = i % N;
      const size_t row = (size_t)(c * K + k0 + t) * a.bc_rs;
      Bs[t * Np + n] = to_f(B[row + n]);
      Cs[t * Np + n] = to_f(Cm[row + n]);
    }
    if (tid < q) {
      float d = to_f(dt[(size_t)(c * K + k0 + tid) * a.dt_rs + h]);
      if (a.dt_bias) d = softplus(d + a.dt_bias[h]);
      dts[tid] = d;
    }
    __syncthreads();
    if (tid == 0) {
      float run = 0.f;
      for (int t = 0; t < q; ++t) {
        run += dts[t] * Ah;
        cum[t] = run;
      }
      for (int t = 0; t < q; ++t) w[t] = expf(run - cum[t]) * dts[t];  // weight into the chunk-end state
    }
    for (int i = tid; i < q * q; i += kThreads) {
      const int t = i / q, s2 = i % q;
      float acc = 0.f;
      if (s2 <= t)
        for (int n = 0; n < N; ++n) acc = fmaf(Cs[t * Np + n], Bs[s2 * Np + n], acc);
      Lm[t * Qp + s2] = acc;
    }
    __syncthreads();
    for (int i = tid; i < q * q; i += kThreads) {
      const int t = i / q, s2 = i % q;
      Lm[t * Qp + s2] = s2 <= t ? Lm[t * Qp + s2] * expf(cum[t] - cum[s2]) * dts[s2] : 0.f;
    }
    __syncthreads();

    // y for 4x4 (t, p) register blocks; the four lanes of a quad split N (interleaved)
    // every lane runs every iteration (the quad shuffles below need the full warp);
    // quads past the last block compute on clamped indices and write nothing
    for (int base = 0; base < n_tb * n_pb; base += kThreads / 4) {
      const int blk_raw = base + (tid >> 2);
      const bool blk_ok = blk_raw < n_tb * n_pb;
      const int blk = blk_ok ? blk_raw : 0;
      const int tb = blk / n_pb, pb = blk % n_pb;
      float acc[4][4] = {};
      int tr[4], pr[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        tr[i] = min(4 * tb + i, q - 1);
        pr[i] = min(4 * pb + i, P - 1);
      }
      for (int n = stateless ? N : nq; n < N; n += 4) {  // S = 0 in the stateless form
        float cv[4], sv[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          cv[i] = Cs[tr[i] * Np + n];
          sv[i] = S[pr[i] * Np + n];
        }
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
          for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(cv[i], sv[j], acc[i][j]);
      }
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          acc[i][j] += __shfl_xor_sync(0xffffffffu, acc[i][j], 1);
          acc[i][j] += __shfl_xor_sync(0xffffffffu, acc[i][j], 2);
        }
      // lane nq of the quad finishes row t = 4 tb + nq
      float off[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) off[j] = acc[0][j];
#pragma unroll
      for (int i = 1; i < 4; ++i)
        if (nq == i)
#pragma unroll
          for (int j = 0; j < 4; ++j) off[j] = acc[i][j];
      const int t = 4 * tb + nq;
      if (blk_ok && t < q) {
        const float e = expf(cum[t]);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int p = 4 * pb + j;
          if (p >= P) break;
          float v = e * off[j];
          for (int s2 = 0; s2 <= t; ++s2) v = fmaf(Lm[t * Qp + s2], xs[s2 * P + p], v);
          v = fmaf(Dh, xs[t * P + p], v);
          a.y[(size_t)(c * K + k0 + t) * a.y_rs + (size_t)h * P + p] = v;
        }
      }
    }

    // state pass to the next chunk (or to the final state)
    if (k0 + q < K || a.hK) {
      __syncthreads();  // all reads of S and xs for the outputs are done
      const float decay = expf(cum[q - 1]);
      for (int i = tid; i < q * P; i += kThreads) xs[i] *= w[i / P];
      __syncthreads();
      const int n_nb = (N + 3) / 4;
      for (int blk = tid; blk < n_pb * n_nb; blk += kThreads) {
        const int pb = blk / n_nb, nb = blk % n_nb;
        float acc[4][4];
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const int p = min(4 * pb + i, P - 1), n = min(4 * nb + j, N - 1);
            acc[i][j] = decay * S[p * Np + n];
          }
        for (int s2 = 0; s2 < q; ++s2) {
          float xv[4], bv[4];
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            xv[i] = xs[s2 * P + min(4 * pb + i, P - 1)];
            bv[i] = Bs[s2 * Np + min(4 * nb + i, N - 1)];
          }
#pragma unroll
          for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(xv[i], bv[j], acc[i][j]);
        }
        // each thread reads and writes only its own 4x4 block of S
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const int p = 4 * pb + i, n = 4 * nb + j;
            if (p < P && n < N) S[p * Np + n] = acc[i][j];
          }
      }
    }
  }
  if (a.hK) {
    __syncthreads();
    float* out = a.hK + ((size_t)c * a.H + h) * P * N;
    for (int i = tid; i < P * N; i += kThreads) out[i] = S[(i / N) * Np + i % N];
  }
}

template <typename T, typename TDT>
void launch(const SsdArgs& a, cudaStream_t s) {
  const bool stateless = !a.h0 && !a.hK && a.Q >= a.K;
  const size_t bytes = (size_t)ssd_layout(a.P, a.N, a.Q, stateless).total * sizeof(float);
  static bool attr_set[64] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 64 && !attr_set[dev]) {
    cudaFuncSetAttribute(ssd_chunk_kernel<T, TDT>, cudaFuncAttributeMaxDynamicSharedMemorySize, 227 * 1024);
    attr_set[dev] = true;
  }
  launch_pdl(ssd_chunk_kernel<T, TDT>, dim3(a.H, a.C), kThreads, bytes, s, a);
  note_launch();
}

}  // namespace

size_t ssd_smem_bytes(int P, int N, int Q) { return (size_t)ssd_layout(P, N, Q).total * sizeof(float); }

void ssd_scan(int dtype, const SsdArgs& a, cudaStream_t s) {
  // bf16 drafter, one chunk, no final state: the state readout on the tensor cores
  if (ssd_tc_supported(dtype, a) && ssd_tc_launch(a, s)) return;
  if (dtype == HSPEC_DTYPE_BF16) {
    if (a.dt_bias) launch<bf16, bf16>(a, s);
    else launch<bf16, float>(a, s);
  } else {
    launch<float, float>(a, s);
  }
}

}  // namespace hspec
