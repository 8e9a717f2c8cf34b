// fp32 GEMM on the CUDA cores (exact fp32 FMA, no TF32): out = epi(A . B^T) with
// A [M,K], B [N,K] row-major.  It serves the fp32 drafter, whose tolerance (1e-4
// relative) rules out reduced-precision tensor-core inputs.  bf16 drafters use the
// tcgen05 kernel in gemm_tc.cu.
//
// Tiling: 64x64 output tile per CTA, K-slices of 16 staged through shared memory,
// 256 threads each owning a 4x4 register micro-tile.
#include "common.cuh"
#include "kernels.cuh"
#include "../../include/hspec.h"

namespace hspec {
namespace {

constexpr int BM = 64, BN = 64, BK = 16, PAD = 4;

template <int EPI>
__global__ void __launch_bounds__(256) gemm_simt_kernel(GemmArgs g) {
  pdl_wait();  // the previous kernel on the stream is complete from here on
  pdl_trigger();
  __shared__ float As[BK][BM + PAD];
  __shared__ float Bs[BK][BN + PAD];
  __shared__ float B2s[EPI == kEpiSwiGLU ? BK : 1][BN + PAD];
  __shared__ float redv[BM][17];
  __shared__ int redi[BM][17];
  const float* A = (const float*)g.A;
  const float* B = (const float*)g.B;
  const float* B2 = (const float*)g.B2;
  const int tx = threadIdx.x % 16, ty = threadIdx.x / 16;
  const int m0 = blockIdx.y * BM, n0 = blockIdx.x * BN;
  float acc[4][4] = {}, acc2[4][4] = {};

  for (int k0 = 0; k0 < g.K; k0 += BK) {
    for (int i = threadIdx.x; i < BM * BK; i += 256) {
      const int r = i / BK, kk = i % BK;
      const int gm = m0 + r, gn = n0 + r, gk = k0 + kk;
      As[kk][r] = (gm < g.M && gk < g.K) ? A[(size_t)gm * g.lda + gk] : 0.f;
      Bs[kk][r] = (gn < g.N && gk < g.K) ? B[(size_t)gn * g.ldb + gk] : 0.f;
      if (EPI == kEpiSwiGLU) B2s[kk][r] = (gn < g.N && gk < g.K) ? B2[(size_t)gn * g.ldb + gk] : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < BK; ++kk) {
      float a[4], b[4], b2[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        a[i] = As[kk][ty * 4 + i];
        b[i] = Bs[kk][tx * 4 + i];
        if (EPI == kEpiSwiGLU) b2[i] = B2s[kk][tx * 4 + i];
      }
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
          if (EPI == kEpiSwiGLU) acc2[i][j] = fmaf(a[i], b2[j], acc2[i][j]);
        }
    }
    __syncthreads();
  }

  if (EPI == kEpiArgmax) {
    // per row: max over this thread's 4 columns, then over the 16 threads of the row
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      float best = -INFINITY;
      int bidx = 0x7fffffff;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int gn = n0 + tx * 4 + j;
        if (gn < g.N && acc[i][j] > best) best = acc[i][j], bidx = gn;
      }
      redv[ty * 4 + i][tx] = best;
      redi[ty * 4 + i][tx] = bidx;
    }
    __syncthreads();
    if (threadIdx.x < BM) {
      const int r = threadIdx.x, gm = m0 + r;
      float best = -INFINITY;
      int bidx = 0x7fffffff;
      for (int t = 0; t < 16; ++t)
        if (redv[r][t] > best || (redv[r][t] == best && redi[r][t] < bidx)) best = redv[r][t], bidx = redi[r][t];
      if (gm < g.M) {
        g.pval[(size_t)gm * g.n_parts + blockIdx.x] = best;
        g.pidx[(size_t)gm * g.n_parts + blockIdx.x] = bidx;
      }
    }
    return;
  }

#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int gm = m0 + ty * 4 + i;
    if (gm >= g.M) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int gn = n0 + tx * 4 + j;
      if (gn >= g.N) continue;
      float* o = (float*)g.out + (size_t)gm * g.ldo + gn;
      if (EPI == kEpiStore) *o = acc[i][j];
      else if (EPI == kEpiResid) *o += acc[i][j];
      else if (EPI == kEpiSwiGLU) *o = silu(acc[i][j]) * acc2[i][j];
    }
  }
}

}  // namespace

void gemm_simt_f32(GemmEpi epi, const GemmArgs& g, cudaStream_t s) {
  dim3 grid(cdiv(g.N, BN), cdiv(g.M, BM));
  switch (epi) {
    case kEpiStore: launch_pdl(gemm_simt_kernel<kEpiStore>, grid, 256, 0, s, g); break;
    case kEpiResid: launch_pdl(gemm_simt_kernel<kEpiResid>, grid, 256, 0, s, g); break;
    case kEpiSwiGLU: launch_pdl(gemm_simt_kernel<kEpiSwiGLU>, grid, 256, 0, s, g); break;
    case kEpiArgmax: launch_pdl(gemm_simt_kernel<kEpiArgmax>, grid, 256, 0, s, g); break;
  }
  note_launch();
}

}  // namespace hspec
