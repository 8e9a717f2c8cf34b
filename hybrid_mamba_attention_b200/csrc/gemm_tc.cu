// bf16 GEMM on the 5th-generation tensor cores: out = epi(A . B^T), A [M,K] and
// B [N,K] row-major (K-major) bf16, fp32 accumulation in tensor memory.
//
// Persistent kernel, one CTA per SM; the output is cut into 128 x 256 tiles (SwiGLU:
// 128 x 128 outputs from a 128 x (128 gate + 128 up) accumulator), numbered M-tile
// fastest, and CTA b takes tiles b, b + grid, ... so that the CTAs working on one
// weight tile at a time are resident together and the weight is read from HBM once.
// Three roles:
//   warp 0      TMA producer: streams 128x64 A and 256x64 B tiles (128-byte
//               swizzle) through a 4-stage shared-memory ring of mbarriers, on
//               from one output tile to the next;
//   warp 1      allocates 512 TMEM columns (two 256-column accumulators); one lane
//               issues tcgen05.mma (M=128, N=256, K=16, four per 64-wide stage),
//               commits each stage back to the producer and each finished
//               accumulator to the epilogue;
//   warps 2..5  epilogue: tcgen05.ld of their 32-lane quarter of TMEM, then the fused
//               epilogue (store, residual add, SwiGLU, per-row argmax), while the
//               next tile accumulates into the other TMEM buffer.
// Rows/columns beyond M/N are zero-filled by TMA and skipped by the epilogue.
// With fewer output tiles than SMs (few token rows) the K loop is split: work unit
// (tile, split) accumulates its K range, writes the fp32 partial of its rows, and the
// last unit of a tile to finish (an atomic counter per tile) sums the partials in split
// order and runs the fused epilogue.
#include <mutex>
#include <stdint.h>

#include "../../include/hspec.h"
#include "common.cuh"
#include "kernels.cuh"
#include "tc_prims.cuh"

namespace hspec {

void gemm_simt_f32(GemmEpi epi, const GemmArgs& g, cudaStream_t s);

namespace {

constexpr int BM = 128, BN = 256, BK = 64, STAGES = 4;
constexpr int A_BYTES = BM * BK * 2, B_BYTES = BN * BK * 2, STAGE_BYTES = A_BYTES + B_BYTES;
constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + 1024 /*align*/ + 256 /*barriers*/;
constexpr int THREADS = 192;
constexpr uint32_t TMEM_COLS = 512;  // two accumulators of BN columns

// Fused epilogue of 32 consecutive columns (nb = first output column) of row m.
template <int EPI>
__device__ __forceinline__ void epi32(const GemmArgs& g, int m, int nb, float (&v)[32], const float (&u)[32]) {
  if (EPI == kEpiStore && g.out_f32) {
    float* o = (float*)g.out + (size_t)m * g.ldo + nb;
    if (nb + 32 <= g.N && (((uintptr_t)o) & 15) == 0) {
#pragma unroll
      for (int i = 0; i < 32; i += 4) *(float4*)(o + i) = make_float4(v[i], v[i + 1], v[i + 2], v[i + 3]);
    } else {
      for (int i = 0; i < 32; ++i)
        if (nb + i < g.N) o[i] = v[i];
    }
  } else if (EPI == kEpiResid) {
    float* o = (float*)g.out + (size_t)m * g.ldo + nb;
    if (nb + 32 <= g.N && (((uintptr_t)o) & 15) == 0) {
#pragma unroll
      for (int i = 0; i < 32; i += 4) {
        float4 x = *(float4*)(o + i);
        x.x += v[i], x.y += v[i + 1], x.z += v[i + 2], x.w += v[i + 3];
        *(float4*)(o + i) = x;
      }
    } else {
      for (int i = 0; i < 32; ++i)
        if (nb + i < g.N) o[i] += v[i];
    }
  } else {
    if (EPI == kEpiSwiGLU) {
#pragma unroll
      for (int i = 0; i < 32; ++i) v[i] = silu(v[i]) * u[i];
    }
    bf16* o = (bf16*)g.out + (size_t)m * g.ldo + nb;
    if (nb + 32 <= g.N && (((uintptr_t)o) & 15) == 0) {
#pragma unroll
      for (int i = 0; i < 32; i += 8) {
        __align__(16) bf16 t8[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) t8[k] = __float2bfloat16_rn(v[i + k]);
        *(uint4*)(o + i) = *(uint4*)t8;
      }
    } else {
      for (int i = 0; i < 32; ++i)
        if (nb + i < g.N) o[i] = __float2bfloat16_rn(v[i]);
    }
  }
}

template <int EPI>
__global__ void __launch_bounds__(THREADS, 1)
    gemm_tc_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                   const __grid_constant__ CUtensorMap tmB2, GemmArgs g, int splits, int* err) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = tc::smem_u32(smem_raw);
  uint8_t* smem = smem_raw + (((raw + 1023) & ~1023u) - raw);
  uint64_t* full = (uint64_t*)(smem + STAGES * STAGE_BYTES);
  uint64_t* empty = full + STAGES;
  uint64_t* acc_full = empty + STAGES;   // [2] accumulator b holds a finished unit
  uint64_t* acc_empty = acc_full + 2;    // [2] the epilogue has read accumulator b
  uint32_t* tmem_slot = (uint32_t*)(acc_empty + 2);
  volatile int* s_last = (volatile int*)(tmem_slot + 1);  // split-K: this unit finishes its tile
  volatile int* s_fail = s_last + 1;                      // split-K: an epilogue wait gave up

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int ncols_out = (EPI == kEpiSwiGLU) ? BN / 2 : BN;
  const int n_mt = (g.M + BM - 1) / BM;
  const int n_tiles = n_mt * ((g.N + ncols_out - 1) / ncols_out);
  const int num_k = (g.K + BK - 1) / BK;
  const int kps = (num_k + splits - 1) / splits;  // K blocks per split
  const int n_units = n_tiles * splits;           // unit u: tile u / splits, split u % splits

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      tc::mbar_init(&full[s], 1);
      tc::mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      tc::mbar_init(&acc_full[b], 1);
      tc::mbar_init(&acc_empty[b], 4);
    }
    *s_fail = 0;
    tc::fence_mbar_init();
  }
  if (warp == 1) tc::tmem_alloc(tmem_slot, TMEM_COLS);
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0 && lane == 0) {
    // ---------------------------------------------------------- TMA producer
    tc::tma_prefetch_desc(&tmA);
    tc::tma_prefetch_desc(&tmB);
    if (EPI == kEpiSwiGLU) tc::tma_prefetch_desc(&tmB2);
    int it = 0;  // stage-ring position, continued across units
    bool ok = true;
    for (int u = blockIdx.x; u < n_units && ok; u += gridDim.x) {
      const int t = u / splits, sp = u % splits;
      const int m0 = (t % n_mt) * BM, n0 = (t / n_mt) * ncols_out;
      const int k_lo = sp * kps, k_hi = min(num_k, k_lo + kps);
      for (int kt = k_lo; kt < k_hi; ++kt, ++it) {
        const int s = it % STAGES;
        if (!(ok = tc::mbar_wait(&empty[s], ((it / STAGES) & 1) ^ 1, err))) break;
        uint8_t* sa = smem + s * STAGE_BYTES;
        uint8_t* sb = sa + A_BYTES;
        tc::mbar_arrive_expect_tx(&full[s], STAGE_BYTES);
        tc::tma_load_2d(sa, &tmA, &full[s], kt * BK, m0);
        if (EPI == kEpiSwiGLU) {
          tc::tma_load_2d(sb, &tmB, &full[s], kt * BK, n0);
          tc::tma_load_2d(sb + B_BYTES / 2, &tmB2, &full[s], kt * BK, n0);
        } else {
          tc::tma_load_2d(sb, &tmB, &full[s], kt * BK, n0);
        }
      }
    }
  } else if (warp == 1 && lane == 0) {
    // ---------------------------------------------------------- MMA issuer
    constexpr uint32_t idesc = tc::idesc_bf16_f32(BM, BN);
    bool ok = true;
    int it = 0, lt = 0;
    for (int u = blockIdx.x; u < n_units && ok; u += gridDim.x, ++lt) {
      const int sp = u % splits;
      const int k_lo = sp * kps, k_hi = min(num_k, k_lo + kps);
      const int b = lt & 1;
      // accumulator b is free once the epilogue has read the unit two back
      if (!(ok = tc::mbar_wait(&acc_empty[b], ((lt >> 1) & 1) ^ 1, err))) break;
      tc::tc_fence_after();
      const uint32_t d = tmem + (uint32_t)(b * BN);
      for (int kt = k_lo; kt < k_hi; ++kt, ++it) {
        const int s = it % STAGES;
        if (!(ok = tc::mbar_wait(&full[s], (it / STAGES) & 1, err))) break;
        tc::tc_fence_after();
        const uint32_t sa = tc::smem_u32(smem + s * STAGE_BYTES);
        const uint32_t sb = sa + A_BYTES;
#pragma unroll
        for (int k = 0; k < BK / 16; ++k) {
          tc::mma_bf16(d, tc::sdesc_k128(sa + k * 32), tc::sdesc_k128(sb + k * 32), idesc,
                       (kt != k_lo || k != 0) ? 1u : 0u);
        }
        tc::mma_commit(&empty[s]);
      }
      tc::mma_commit(&acc_full[b]);
    }
  } else if (warp >= 2) {
    // ---------------------------------------------------------- epilogue
    const int quarter = warp & 3;  // TMEM lanes this warp may access
    const int row = quarter * 32 + lane;
    int lt = 0;
    for (int u = blockIdx.x; u < n_units; u += gridDim.x, ++lt) {
      const int t = u / splits;
      const int b = lt & 1;
      const int m0 = (t % n_mt) * BM, n0 = (t / n_mt) * ncols_out, ntile = t / n_mt;
      const int m = m0 + row;
      const bool ok = tc::mbar_wait(&acc_full[b], (lt >> 1) & 1, err);
      __syncwarp();
      tc::tc_fence_after();
      const uint32_t taddr = tmem + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(b * BN);
      float v[32], u2[32];
      if (splits > 1) {
        // this split's partial of the unit's rows, then: is this the tile's last split?
        float* pr = g.part + ((size_t)u * BM + row) * BN;
        for (int c = 0; c < BN; c += 32) {
          tc::tmem_ld32(taddr + c, v);
          if (ok && m < g.M)
#pragma unroll
            for (int i = 0; i < 32; i += 4) *(float4*)(pr + c + i) = make_float4(v[i], v[i + 1], v[i + 2], v[i + 3]);
        }
        tc::tc_fence_before();
        __syncwarp();
        if (lane == 0) tc::mbar_arrive(&acc_empty[b]);
        __threadfence();
        // the four epilogue warps pass the same three barriers per unit and leave together
        if (!ok) *s_fail = 1;
        asm volatile("bar.sync 1, 128;" ::: "memory");
        if (threadIdx.x == 64) *s_last = atomicAdd(&g.tile_cnt[t], 1) == splits - 1;
        asm volatile("bar.sync 1, 128;" ::: "memory");
        const bool last = *s_last != 0, all_ok = *s_fail == 0;
        asm volatile("bar.sync 1, 128;" ::: "memory");  // s_last is read before the next unit writes it
        if (!last) {
          if (!all_ok) break;
          continue;
        }
        __threadfence();
        if (all_ok) {
          // the 128 epilogue threads take (valid row, 32-column chunk) items, so that few
          // valid rows still spread over all of them; loads of several splits in flight
          const int rows_v = min(BM, g.M - m0), nch = ncols_out / 32;
          for (int w = threadIdx.x - 64; w < rows_v * nch; w += 128) {
            const int r = w / nch, c = (w % nch) * 32;
            const float* p0 = g.part + ((size_t)(t * splits) * BM + r) * BN + c;
#pragma unroll
            for (int i = 0; i < 32; ++i) v[i] = 0.f, u2[i] = 0.f;
#pragma unroll 4
            for (int q = 0; q < splits; ++q) {  // split order: the same sums whoever finishes last
              const float* pq = p0 + (size_t)q * BM * BN;
#pragma unroll
              for (int i = 0; i < 32; i += 4) {
                const float4 a4 = __ldcg((const float4*)(pq + i));
                v[i] += a4.x, v[i + 1] += a4.y, v[i + 2] += a4.z, v[i + 3] += a4.w;
                if (EPI == kEpiSwiGLU) {
                  const float4 b4 = __ldcg((const float4*)(pq + BN / 2 + i));
                  u2[i] += b4.x, u2[i + 1] += b4.y, u2[i + 2] += b4.z, u2[i + 3] += b4.w;
                }
              }
            }
            epi32<EPI>(g, m0 + r, n0 + c, v, u2);
          }
        }
        if (threadIdx.x == 64) g.tile_cnt[t] = 0;  // ready for the next launch
        if (!all_ok) break;
        continue;
      }
      if (EPI == kEpiArgmax) {
        float best = -INFINITY;
        int bidx = 0x7fffffff;
        for (int c = 0; c < BN; c += 32) {
          tc::tmem_ld32(taddr + c, v);
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            const int n = n0 + c + i;
            if (n < g.N && v[i] > best) best = v[i], bidx = n;
          }
        }
        if (ok && m < g.M) {
          g.pval[(size_t)m * g.n_parts + ntile] = best;
          g.pidx[(size_t)m * g.n_parts + ntile] = bidx;
        }
      } else {
        for (int c = 0; c < ncols_out; c += 32) {
          tc::tmem_ld32(taddr + c, v);
          if (EPI == kEpiSwiGLU) tc::tmem_ld32(taddr + BN / 2 + c, u2);
          if (!ok || m >= g.M) continue;
          epi32<EPI>(g, m, n0 + c, v, u2);
        }
      }
      // accumulator b may take the unit after next
      tc::tc_fence_before();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(&acc_empty[b]);
      if (!ok) break;
    }
  }
  __syncthreads();
  if (warp == 1) {
    tc::tc_fence_after();
    tc::tmem_dealloc(tmem, TMEM_COLS);
  }
}

// ------------------------------------------------------------ tensor maps

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = (EncodeTiledFn)p;
  });
  return fn;
}

// 2-D bf16 map of a row-major [rows, cols] matrix with leading dimension ld
// (elements), box = box_rows x 64 columns, 128-byte swizzle, zero fill.
bool make_map(CUtensorMap* m, const void* base, long rows, long cols, long ld, int box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)ld * 2};
  cuuint32_t box[2] = {(cuuint32_t)BK, (cuuint32_t)box_rows};
  cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int device_sms() {
  static int n_sm[64] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev >= 64) return 148;
  if (!n_sm[dev]) cudaDeviceGetAttribute(&n_sm[dev], cudaDevAttrMultiProcessorCount, dev);
  return n_sm[dev] > 0 ? n_sm[dev] : 148;
}

template <int EPI>
bool launch_tc(const GemmArgs& g, int splits, cudaStream_t s, int* err) {
  static bool attr_set[64] = {};
  static int n_sm[64] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 64 && !attr_set[dev]) {
    if (cudaFuncSetAttribute(gemm_tc_kernel<EPI>, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES) !=
        cudaSuccess) {
      set_error("cudaFuncSetAttribute(gemm_tc_kernel) failed");
      return false;
    }
    cudaDeviceGetAttribute(&n_sm[dev], cudaDevAttrMultiProcessorCount, dev);
    attr_set[dev] = true;
  }
  CUtensorMap ta, tb, tb2;
  const int brows = (EPI == kEpiSwiGLU) ? BN / 2 : BN;
  bool ok = make_map(&ta, g.A, g.M, g.K, g.lda, BM) && make_map(&tb, g.B, g.N, g.K, g.ldb, brows);
  if (EPI == kEpiSwiGLU) ok = ok && make_map(&tb2, g.B2, g.N, g.K, g.ldb, brows);
  else tb2 = tb;
  if (!ok) {
    set_error("cuTensorMapEncodeTiled failed (M=%d N=%d K=%d)", g.M, g.N, g.K);
    return false;
  }
  const int ncols_out = (EPI == kEpiSwiGLU) ? BN / 2 : BN;
  const long n_units = (long)cdiv(g.M, BM) * cdiv(g.N, ncols_out) * splits;
  const int sms = dev < 64 && n_sm[dev] > 0 ? n_sm[dev] : 148;
  const int grid = n_units < sms ? (int)n_units : sms;
  gemm_tc_kernel<EPI><<<grid, THREADS, SMEM_BYTES, s>>>(ta, tb, tb2, g, splits, err);
  note_launch();
  return true;
}

}  // namespace

int* device_error_word();  // hspec_abi.cu

int argmax_tile_n(int dtype) { return dtype == HSPEC_DTYPE_BF16 ? BN : 64; }

int gemm_tile_count(int dtype, GemmEpi epi, int M, int N) {
  if (dtype != HSPEC_DTYPE_BF16) return 0;
  return cdiv(M, BM) * cdiv(N, epi == kEpiSwiGLU ? BN / 2 : BN);
}

// Split K when the output has fewer tiles than SMs: about one unit per SM, at least
// four 64-wide K blocks per split, every split non-empty.
int gemm_split_count(int dtype, GemmEpi epi, int M, int N, int K) {
  if (dtype != HSPEC_DTYPE_BF16 || epi == kEpiArgmax) return 1;
  const int n_tiles = gemm_tile_count(dtype, epi, M, N), num_k = cdiv(K, BK), sms = device_sms();
  if (n_tiles <= 0 || n_tiles * 2 > sms) return 1;
  int sp = sms / n_tiles;
  if (sp > num_k / 4) sp = num_k / 4;
  if (sp < 2) return 1;
  const int kps = cdiv(num_k, sp);
  return cdiv(num_k, kps);
}

size_t gemm_split_bytes(int dtype, GemmEpi epi, int M, int N, int K) {
  const int sp = gemm_split_count(dtype, epi, M, N, K);
  return sp > 1 ? (size_t)gemm_tile_count(dtype, epi, M, N) * sp * BM * BN * sizeof(float) : 0;
}

bool gemm(int dtype, GemmEpi epi, const GemmArgs& g, cudaStream_t s) {
  if (dtype != HSPEC_DTYPE_BF16) {
    gemm_simt_f32(epi, g, s);
    return true;
  }
  // TMA needs 16-byte aligned bases and row strides.
  if ((g.lda % 8) || (g.ldb % 8) || (((uintptr_t)g.A) & 15) || (((uintptr_t)g.B) & 15) ||
      (g.B2 && (((uintptr_t)g.B2) & 15))) {
    set_error("bf16 GEMM operands need 16-byte aligned bases and leading dimensions (lda=%ld ldb=%ld)",
              g.lda, g.ldb);
    return false;
  }
  int* err = device_error_word();
  int splits = 1;
  if (g.part && g.tile_cnt && !(epi == kEpiStore && g.out_f32)) {
    const int sp = gemm_split_count(dtype, epi, g.M, g.N, g.K);
    if (sp > 1 && gemm_split_bytes(dtype, epi, g.M, g.N, g.K) <= g.part_bytes &&
        gemm_tile_count(dtype, epi, g.M, g.N) <= g.max_tiles && !(((uintptr_t)g.part) & 15))
      splits = sp;
  }
  switch (epi) {
    case kEpiStore: return launch_tc<kEpiStore>(g, splits, s, err);
    case kEpiResid: return launch_tc<kEpiResid>(g, splits, s, err);
    case kEpiSwiGLU: return launch_tc<kEpiSwiGLU>(g, splits, s, err);
    case kEpiArgmax: return launch_tc<kEpiArgmax>(g, splits, s, err);
  }
  return false;
}

}  // namespace hspec
