// Paged in-place GQA attention on the 5th-generation tensor cores (bf16, D = 64 or
// 128).  H-Spec (arXiv 2609.24197) Abstract: the drafter's attention modules reuse
// the target KVs in place -- here the K/V pages are streamed by TMA straight out of
// the target's pool through the page table, never copied to a drafter-side cache.
//
// One CTA per (context split, kv head g, request c [, row block]).  The R = K*G
// queries of kv head g (block position j, query head g*G + i) form the rows of a
// 128-row Q tile (rows >= R are zero), so every K/V byte read from HBM feeds all R
// queries.  Warp roles (192 threads):
//   warp 0      TMA producer: per 64-token tile, one 3-D box of 16 tokens x 64 dims
//               of head g per page and column block (128-byte swizzle), K and V into
//               a 4-stage ring; the block's own K keys come as one extra tile from
//               the projection output, loaded by the last context split.
//   warp 1      TMEM owner and single-thread MMA issuer:
//                 S_b  = Q . K_i^T        (M=128, N=64, K=D; S double-buffered in TMEM)
//                 O   += P_b . V_i        (M=128, N=D, K=64; V as an MN-major operand)
//   warps 2..5  softmax, one TMEM lane (query row) per thread: mask, running max in
//               the exp2 domain, P = exp2(s - m) written to shared memory as bf16;
//               O is rescaled in TMEM only when the running max grows by more than
//               8 (2^8 headroom keeps P exact enough in bf16); zeroes V rows past the
//               end of the context in a partial tile; finally writes the split's
//               partial (m, l, unnormalised O) for the merge kernel.
// Synchronisation is by mbarriers (one per ring slot / per double buffer, so that no
// waiter can fall two phases behind); every wait gives up after a time bound and
// sets the device error word.
#include <stdint.h>

#include "../../include/hspec.h"
#include "common.cuh"
#include "kernels.cuh"
#include "tc_prims.cuh"

namespace hspec {

int* device_error_word();

namespace {

constexpr int TT = 64;        // tokens per tile
constexpr int NS = 4;         // K/V ring stages
constexpr int THREADS = 192;
constexpr int ROWS = 128;     // MMA M

template <int D>
struct Lay {
  static constexpr int DB = D / 64;                     // 64-element column blocks
  static constexpr int Q_BLK = ROWS * 128;              // 16 KB per Q column block
  static constexpr int KV_BLK = TT * 128;               // 8 KB per K (or V) column block
  static constexpr int K_BYTES = DB * KV_BLK;
  static constexpr int STAGE = 2 * K_BYTES;             // K then V
  static constexpr int P_BYTES = ROWS * TT * 2;         // 16 KB
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_KV = DB * Q_BLK;
  static constexpr int OFF_P = OFF_KV + NS * STAGE;
  static constexpr int OFF_BAR = OFF_P + 2 * P_BYTES;
  static constexpr int SMEM = OFF_BAR + 256 + 1024;
  static constexpr uint32_t TMEM_COLS = 256;            // S0 [0,64) S1 [64,128) O [128,128+D)
};

struct TcMaps {
  CUtensorMap k, v, kb, vb;
};

template <int D>
__global__ void __launch_bounds__(THREADS, 1)
    attn_tc_kernel(const __grid_constant__ TcMaps maps, AttnArgs a, float scale_log2, int n_rb) {
  using L = Lay<D>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = tc::smem_u32(smem_raw);
  uint8_t* smem = smem_raw + (((raw + 1023) & ~1023u) - raw);
  uint8_t* sQ = smem + L::OFF_Q;
  uint8_t* sKV = smem + L::OFF_KV;
  uint8_t* sP = smem + L::OFF_P;
  uint64_t* kv_full = (uint64_t*)(smem + L::OFF_BAR);
  uint64_t* kv_empty = kv_full + NS;
  uint64_t* s_full = kv_empty + NS;
  uint64_t* p_full = s_full + 2;
  uint64_t* pv_done = p_full + 2;
  uint64_t* q_ready = pv_done + 2;
  uint32_t* tmem_slot = (uint32_t*)(q_ready + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int split = blockIdx.x, g = blockIdx.y;
  const int c = blockIdx.z / n_rb, rb = blockIdx.z % n_rb;
  const int G = a.Hq / a.Hkv, R = a.K * G;
  const int ctx = a.ctx_lens[c];
  if (ctx < 0 || ctx > a.max_pages * a.page_size) {
    if (threadIdx.x == 0 && split == 0 && rb == 0) flag_error(a.err, kErrCtxOOB);
    return;
  }
  const int n_ctx_splits = (ctx + a.split_tokens - 1) / a.split_tokens;
  const int last_split = n_ctx_splits > 0 ? n_ctx_splits - 1 : 0;
  if (split > last_split) return;  // CTA-uniform: nothing of this request here
  const int c_begin = split * a.split_tokens;
  const int c_end = min(ctx, c_begin + a.split_tokens);
  const int n_ctx_tiles = c_end > c_begin ? (c_end - c_begin + TT - 1) / TT : 0;
  const int n_tiles = n_ctx_tiles + (split == last_split ? 1 : 0);
  int* err = a.err;

  if (threadIdx.x == 0) {
    for (int s = 0; s < NS; ++s) {
      tc::mbar_init(&kv_full[s], 1);
      tc::mbar_init(&kv_empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      tc::mbar_init(&s_full[b], 1);
      tc::mbar_init(&p_full[b], 4);
      tc::mbar_init(&pv_done[b], 1);
    }
    tc::mbar_init(q_ready, 4);
    tc::fence_mbar_init();
  }
  if (warp == 1) tc::tmem_alloc(tmem_slot, L::TMEM_COLS);
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t tO = tmem + 128;

  if (warp == 0) {
    if (lane == 0) {
      // ---------------------------------------------------------- TMA producer
      tc::tma_prefetch_desc(&maps.k);
      tc::tma_prefetch_desc(&maps.v);
      tc::tma_prefetch_desc(&maps.kb);
      tc::tma_prefetch_desc(&maps.vb);
      const int32_t* table = a.page_table + (size_t)c * a.max_pages;
      for (int i = 0; i < n_tiles; ++i) {
        const int s = i % NS;
        if (!tc::mbar_wait(&kv_empty[s], ((i / NS) & 1) ^ 1, err)) break;
        uint8_t* kd = sKV + s * L::STAGE;
        uint8_t* vd = kd + L::K_BYTES;
        if (i < n_ctx_tiles) {
          const int t0 = c_begin + i * TT;
          const int groups = (min(TT, c_end - t0) + 15) / 16;
          tc::mbar_arrive_expect_tx(&kv_full[s], (uint32_t)(groups * L::DB * 2048 * 2));
          for (int q16 = 0; q16 < groups; ++q16) {
            const int t = t0 + 16 * q16;
            int pg = table[t / a.page_size];
            if (pg < 0 || pg >= a.num_pages) {
              flag_error(err, kErrPageOOB);
              pg = 0;  // keep the copy in bounds; the request's output is flagged as invalid
            }
            const int z = pg * a.page_size + t % a.page_size;
            for (int bk = 0; bk < L::DB; ++bk) {
              tc::tma_load_3d(kd + bk * L::KV_BLK + q16 * 2048, &maps.k, &kv_full[s], bk * 64, g, z);
              tc::tma_load_3d(vd + bk * L::KV_BLK + q16 * 2048, &maps.v, &kv_full[s], bk * 64, g, z);
            }
          }
        } else {
          tc::mbar_arrive_expect_tx(&kv_full[s], (uint32_t)(L::DB * L::KV_BLK * 2));
          for (int bk = 0; bk < L::DB; ++bk) {
            tc::tma_load_3d(kd + bk * L::KV_BLK, &maps.kb, &kv_full[s], bk * 64, g, c * a.K);
            tc::tma_load_3d(vd + bk * L::KV_BLK, &maps.vb, &kv_full[s], bk * 64, g, c * a.K);
          }
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ---------------------------------------------------------- MMA issuer
      constexpr uint32_t idesc_qk = tc::idesc_bf16_f32(ROWS, TT);
      constexpr uint32_t idesc_pv = tc::idesc_bf16_f32(ROWS, D) | (1u << 16);  // B (= V) MN-major
      bool ok = tc::mbar_wait(q_ready, 0, err);
      auto issue_qk = [&](int i) -> bool {
        const int s = i % NS;
        if (!tc::mbar_wait(&kv_full[s], (i / NS) & 1, err)) return false;
        tc::tc_fence_after();
        const uint32_t q = tc::smem_u32(sQ), k = tc::smem_u32(sKV + s * L::STAGE);
        const uint32_t dS = tmem + (uint32_t)((i & 1) * TT);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk)
          tc::mma_bf16(dS, tc::sdesc_k128(q + (kk / 4) * L::Q_BLK + (kk % 4) * 32),
                       tc::sdesc_k128(k + (kk / 4) * L::KV_BLK + (kk % 4) * 32), idesc_qk, kk > 0);
        tc::mma_commit(&s_full[i & 1]);
        return true;
      };
      if (ok) ok = issue_qk(0);
      if (ok && n_tiles > 1) ok = issue_qk(1);
      for (int i = 0; i < n_tiles && ok; ++i) {
        const int b = i & 1, s = i % NS;
        if (!(ok = tc::mbar_wait(&p_full[b], (i >> 1) & 1, err))) break;
        tc::tc_fence_after();
        const uint32_t p = tc::smem_u32(sP + b * L::P_BYTES);
        const uint32_t v = tc::smem_u32(sKV + s * L::STAGE + L::K_BYTES);
#pragma unroll
        for (int kk = 0; kk < TT / 16; ++kk)
          tc::mma_bf16(tO, tc::sdesc_k128(p + kk * 32), tc::sdesc_mn128(v + kk * 2048, L::KV_BLK), idesc_pv,
                       (i | kk) != 0);
        tc::mma_commit(&kv_empty[s]);
        tc::mma_commit(&pv_done[b]);
        if (i + 2 < n_tiles) ok = issue_qk(i + 2);
      }
    }
  } else {
    // ------------------------------------------------------------ softmax warps
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;
    const int gr = rb * ROWS + row;
    const bool active = gr < R;
    const int jq = active ? gr / G : 0;
    const int hq = g * G + (active ? gr % G : 0);
    const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;

    // Q row -> shared memory (128-byte swizzle, K-major)
    {
      const bf16* qrow = (const bf16*)a.q + (size_t)(c * a.K + jq) * a.q_rs + (size_t)hq * D;
#pragma unroll
      for (int ch = 0; ch < D / 8; ++ch) {
        uint4 v = make_uint4(0, 0, 0, 0);
        if (active) v = *(const uint4*)(qrow + ch * 8);
        *(uint4*)(sQ + (ch / 8) * L::Q_BLK + row * 128 + (((ch % 8) ^ (row & 7)) << 4)) = v;
      }
      tc::fence_proxy_async();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(q_ready);
    }

    float m_used = -INFINITY, l = 0.f;
    bool ok = true;
    for (int i = 0; i < n_tiles && ok; ++i) {
      const int b = i & 1;
      ok = __all_sync(0xffffffffu, tc::mbar_wait(&s_full[b], (i >> 1) & 1, err));
      if (!ok) break;
      tc::tc_fence_after();
      const bool block_tile = i >= n_ctx_tiles;
      const int valid = block_tile ? a.K : min(TT, c_end - (c_begin + i * TT));
      float s[TT];
      {
        float* s0 = s;
        float(&h0)[32] = *reinterpret_cast<float(*)[32]>(s0);
        float(&h1)[32] = *reinterpret_cast<float(*)[32]>(s0 + 32);
        tc::tmem_ld32(tmem + lane_off + (uint32_t)(b * TT), h0);
        tc::tmem_ld32(tmem + lane_off + (uint32_t)(b * TT + 32), h1);
      }
      float mx = -INFINITY;
#pragma unroll
      for (int j = 0; j < TT; ++j) {
        bool vis = j < valid;
        if (block_tile && a.causal_block && j > jq) vis = false;
        s[j] = vis ? s[j] * scale_log2 : -INFINITY;
        mx = fmaxf(mx, s[j]);
      }
      const float m_new = fmaxf(m_used, mx);
      if (m_new > m_used + 8.f) {
        if (i > 0 && m_used != -INFINITY) {
          // O holds earlier tiles: wait for the last P.V, then rescale it in TMEM
          ok = __all_sync(0xffffffffu, tc::mbar_wait(&pv_done[(i - 1) & 1], ((i - 1) >> 1) & 1, err));
          if (!ok) break;
          tc::tc_fence_after();
          const float alpha = exp2f(m_used - m_new);
#pragma unroll
          for (int cb = 0; cb < D / 32; ++cb) {
            float v[32];
            tc::tmem_ld32(tO + lane_off + cb * 32, v);
#pragma unroll
            for (int e = 0; e < 32; ++e) v[e] *= alpha;
            tc::tmem_st32(tO + lane_off + cb * 32, v);
          }
          l *= alpha;
        }
        m_used = m_new;
      }
      float psum = 0.f;
      uint32_t pk[TT / 2];
#pragma unroll
      for (int j = 0; j < TT; j += 2) {
        const float p0 = (s[j] == -INFINITY) ? 0.f : exp2f(s[j] - m_used);
        const float p1 = (s[j + 1] == -INFINITY) ? 0.f : exp2f(s[j + 1] - m_used);
        psum += p0 + p1;
        __nv_bfloat162 h2 = __floats2bfloat162_rn(p0, p1);
        pk[j / 2] = *reinterpret_cast<uint32_t*>(&h2);
      }
      l += psum;
      if (i >= 2) {  // P buffer b was read by the P.V of tile i-2
        ok = __all_sync(0xffffffffu, tc::mbar_wait(&pv_done[b], ((i - 2) >> 1) & 1, err));
        if (!ok) break;
      }
      uint8_t* prow = sP + b * L::P_BYTES + row * 128;
#pragma unroll
      for (int cc = 0; cc < 8; ++cc)
        *(uint4*)(prow + ((cc ^ (row & 7)) << 4)) = make_uint4(pk[4 * cc], pk[4 * cc + 1], pk[4 * cc + 2], pk[4 * cc + 3]);
      if (valid < TT) {
        // V rows past the last valid token may hold stale data: zero them (P is 0 there)
        uint8_t* vbase = sKV + (i % NS) * L::STAGE + L::K_BYTES;
        const int n_chunks = (TT - valid) * L::DB * 8;
        for (int e = threadIdx.x - 64; e < n_chunks; e += 128) {
          const int r2 = valid + e / (L::DB * 8), rest = e % (L::DB * 8);
          const int bk = rest / 8, cc = rest % 8;
          *(uint4*)(vbase + bk * L::KV_BLK + r2 * 128 + ((cc ^ (r2 & 7)) << 4)) = make_uint4(0, 0, 0, 0);
        }
      }
      tc::fence_proxy_async();
      tc::tc_fence_before();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(&p_full[b]);
    }

    // epilogue: the split's partial state for the merge kernel
    if (ok && n_tiles > 0) {
      const int last = n_tiles - 1;
      ok = __all_sync(0xffffffffu, tc::mbar_wait(&pv_done[last & 1], (last >> 1) & 1, err));
      tc::tc_fence_after();
      const size_t base = (((size_t)c * a.Hkv + g) * a.n_splits + split) * R + gr;
#pragma unroll
      for (int cb = 0; cb < D / 32; ++cb) {
        float v[32];
        tc::tmem_ld32(tO + lane_off + cb * 32, v);
        if (ok && active) {
          float* o = a.ws_acc + base * D + cb * 32;
#pragma unroll
          for (int e = 0; e < 32; e += 4) *(float4*)(o + e) = make_float4(v[e], v[e + 1], v[e + 2], v[e + 3]);
        }
      }
      if (ok && active) {
        a.ws_ml[base * 2] = m_used;
        a.ws_ml[base * 2 + 1] = l;
      }
    }
    tc::tc_fence_before();
  }
  __syncthreads();
  if (warp == 1) {
    tc::tc_fence_after();
    tc::tmem_dealloc(tmem, L::TMEM_COLS);
  }
}

// ------------------------------------------------------------------ host side

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn_attn() {
  static EncodeTiledFn fn = nullptr;
  static bool tried = false;
  if (!tried) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = (EncodeTiledFn)p;
    tried = true;
  }
  return fn;
}

// 3-D map [rows][Hkv][D] (x = D elements, y = kv head, z = token row) with box
// 64 x 1 x box_rows, 128-byte swizzle.
bool make_kv_map(CUtensorMap* m, const void* base, long rows, int Hkv, int D, long row_stride_elems,
                 int box_rows) {
  EncodeTiledFn fn = encode_fn_attn();
  if (!fn) return false;
  cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)Hkv, (cuuint64_t)rows};
  cuuint64_t strides[2] = {(cuuint64_t)D * 2, (cuuint64_t)row_stride_elems * 2};
  cuuint32_t box[3] = {64, 1, (cuuint32_t)box_rows};
  cuuint32_t estr[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int D>
bool launch_tc(const AttnArgs& a, cudaStream_t s) {
  static bool attr_set[64] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 64 && !attr_set[dev]) {
    if (cudaFuncSetAttribute(attn_tc_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, Lay<D>::SMEM) !=
        cudaSuccess) {
      set_error("cudaFuncSetAttribute(attn_tc_kernel) failed");
      return false;
    }
    attr_set[dev] = true;
  }
  TcMaps maps;
  const long pool_rows = (long)a.num_pages * a.page_size;
  bool ok = make_kv_map(&maps.k, a.k_pool, pool_rows, a.Hkv, D, (long)a.Hkv * D, 16) &&
            make_kv_map(&maps.v, a.v_pool, pool_rows, a.Hkv, D, (long)a.Hkv * D, 16) &&
            make_kv_map(&maps.kb, a.kb, (long)a.C * a.K, a.Hkv, D, a.kb_rs, TT) &&
            make_kv_map(&maps.vb, a.vb, (long)a.C * a.K, a.Hkv, D, a.vb_rs, TT);
  if (!ok) {
    set_error("cuTensorMapEncodeTiled failed for the attention K/V maps");
    return false;
  }
  const int R = a.K * (a.Hq / a.Hkv);
  const int n_rb = (R + ROWS - 1) / ROWS;
  const float scale_log2 = 1.4426950408889634f / sqrtf((float)D);
  attn_tc_kernel<D><<<dim3(a.n_splits, a.Hkv, a.C * n_rb), THREADS, Lay<D>::SMEM, s>>>(maps, a, scale_log2, n_rb);
  note_launch();
  return true;
}

}  // namespace

bool attn_tc_supported(const AttnArgs& a, const char** why) {
  if (a.D != 64 && a.D != 128) return *why = "head_dim must be 64 or 128", false;
  if (a.page_size % 16) return *why = "page_size must be a multiple of 16", false;
  if (a.K > 64) return *why = "K must be <= 64", false;
  if ((a.q_rs % 8) || (a.kb_rs % 8) || (a.vb_rs % 8))
    return *why = "q / k_blk / v_blk row strides must be multiples of 8 elements", false;
  const uintptr_t any = (uintptr_t)a.q | (uintptr_t)a.kb | (uintptr_t)a.vb | (uintptr_t)a.k_pool | (uintptr_t)a.v_pool;
  if (any & 15) return *why = "q, k_blk, v_blk and the pools must be 16-byte aligned", false;
  if ((long)a.num_pages * a.page_size > 0x7fffffffL) return *why = "pool too large", false;
  return true;
}

bool attn_tc_launch(const AttnArgs& a, cudaStream_t s) {
  return a.D == 128 ? launch_tc<128>(a, s) : launch_tc<64>(a, s);
}

}  // namespace hspec
