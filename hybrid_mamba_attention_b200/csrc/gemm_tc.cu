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
//               epilogue (store, residual add, SwiGLU, per-row argmax, or the readout
//               of the injected SSD state into y), while the next tile accumulates
//               into the other TMEM buffer.
// Rows/columns beyond M/N are zero-filled by TMA and skipped by the epilogue.
// When whole tiles would leave SMs idle the K loop is cut, in one of two ways:
//   stream-K (one row of tiles, M <= 128): the (tile, 64-wide K block) pairs form one
//     line, tile-major, and CTA b takes its equal chunk [b Z, b Z + Z) of it, walked
//     as segments, one per tile it crosses.  Only a chunk's first and last segments
//     can be partial, so chunk k owns partial slots 2k (its first) and 2k + 1 (its
//     last).  With several rows of tiles this would put the CTAs that share a weight
//     tile at different K offsets (the weight then comes from HBM once per CTA
//     instead of once from L2), so there:
//   split-K (fewer tiles than half the SMs): unit (tile, split) covers an equal K
//     range, all units start at their range's first block together; slot = unit.
// A segment covering a whole tile runs the fused epilogue itself; the others write the
// fp32 partial of their rows to their slot and count in (an atomic counter per tile).
// Split-K: the last segment of a tile to finish sums the partials in K order and runs
// the epilogue.  Stream-K: after its own segments every CTA takes an equal share of the
// split tiles' (row, 32-column) sums, each waiting until its tile is complete -- with
// many rows one CTA summing a tile's ~10 partials at one SM's bandwidth was the limit.
// The counters are not reset (each call site of the draft step has its own, zeroed
// once per step).
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

// kEpiRope: rotates columns i0 .. i0 + 31 of a head (v1, i0 < D/2) with their partners
// i + D/2 (v2) in row m, after rounding both to bf16 (the stored projection), by the
// angles of the row's (cos, sin) table.
__device__ __forceinline__ void rope_rotate(const RopeArgs& r, int m, int i0, float (&v1)[32], float (&v2)[32]) {
  const float4* t = (const float4*)(r.cs + (size_t)m * (r.D / 2) + i0);  // 32 (cos, sin) pairs, 16-byte aligned
#pragma unroll
  for (int e = 0; e < 32; e += 2) {
    const float4 q = __ldg(t + e / 2);
    const float a0 = __bfloat162float(__float2bfloat16_rn(v1[e])), b0 = __bfloat162float(__float2bfloat16_rn(v2[e]));
    const float a1 = __bfloat162float(__float2bfloat16_rn(v1[e + 1])),
                b1 = __bfloat162float(__float2bfloat16_rn(v2[e + 1]));
    v1[e] = a0 * q.x - b0 * q.y;
    v2[e] = a0 * q.y + b0 * q.x;
    v1[e + 1] = a1 * q.z - b1 * q.w;
    v2[e + 1] = a1 * q.w + b1 * q.z;
  }
}

// How the K loop is cut: zk > 0 stream-K chunks of zk K blocks; else `splits` equal K
// ranges of kps blocks (splits = 1: whole tiles).
struct KCut {
  int zk, splits, kps;
};

// The CTA's work as segments (tile t, K blocks [k0, k1)): stream-K positions
// [b zk, b zk + zk) of the (tile, K block) line; else units b, b + grid, ... of
// (tile, split) (unit u = t * splits + split).
struct SegWalk {
  int num_k, zk, splits, kps, pos, end;
  __device__ SegWalk(int nk, int n_tiles, KCut cut) : num_k(nk), zk(cut.zk), splits(cut.splits), kps(cut.kps) {
    if (zk == 0) {
      pos = blockIdx.x, end = n_tiles * splits;
    } else {
      pos = blockIdx.x * zk;
      end = min(n_tiles * nk, pos + zk);
    }
  }
  __device__ bool next(int& t, int& k0, int& k1) {
    if (pos >= end) return false;
    if (zk == 0) {
      t = pos / splits;
      k0 = (pos - t * splits) * kps;
      k1 = min(num_k, k0 + kps);
      pos += gridDim.x;
    } else {
      t = pos / num_k;
      k0 = pos - t * num_k;
      k1 = min(num_k, k0 + (end - pos));
      pos += k1 - k0;
    }
    return true;
  }
};

// Waits (bounded by limit_ns) until *cnt >= target; the acquire load orders the reads
// that follow.
__device__ __forceinline__ bool wait_count(const int* cnt, int target, int* err, uint64_t limit_ns) {
  auto ld = [&]() {
    int v;
    asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(cnt) : "memory");
    return v;
  };
  if (ld() >= target) return true;
  const uint64_t t0 = tc::global_ns();
  while (ld() < target) {
    __nanosleep(256);
    if (tc::global_ns() - t0 > limit_ns) {
      flag_error(err, tc::kErrTimeout);
      return false;
    }
  }
  return true;
}

// Partial slot of tile t's segment in chunk k (stream-K): the chunk's first segment if
// the chunk starts inside the tile, else its last.
__device__ __forceinline__ int seg_slot(int t, int k, int zk, int num_k) {
  return 2 * k + ((long)k * zk < (long)t * num_k ? 1 : 0);
}

template <int EPI>
__global__ void __launch_bounds__(THREADS, 1)
    gemm_tc_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                   const __grid_constant__ CUtensorMap tmB2, GemmArgs g, KCut cut, int* err) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = tc::smem_u32(smem_raw);
  uint8_t* smem = smem_raw + (((raw + 1023) & ~1023u) - raw);
  uint64_t* full = (uint64_t*)(smem + STAGES * STAGE_BYTES);
  uint64_t* empty = full + STAGES;
  uint64_t* acc_full = empty + STAGES;   // [2] accumulator b holds a finished unit
  uint64_t* acc_empty = acc_full + 2;    // [2] the epilogue has read accumulator b
  uint64_t* drain = acc_empty + 2;       // every MMA of the issuer has finished
  uint32_t* tmem_slot = (uint32_t*)(drain + 1);
  volatile int* s_last = (volatile int*)(tmem_slot + 1);  // stream-K: this segment finishes its tile
  volatile int* s_fail = s_last + 1;                      // stream-K: an epilogue wait gave up

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int ncols_out = (EPI == kEpiSwiGLU) ? BN / 2 : BN;
  const int n_mt = (g.M + BM - 1) / BM;
  const int n_tiles = n_mt * ((g.N + ncols_out - 1) / ncols_out);
  const int num_k = (g.K + BK - 1) / BK;
  const uint64_t lim = g.wait_ns ? (uint64_t)g.wait_ns : tc::kWaitLimitNs;  // pipeline waits

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      tc::mbar_init(&full[s], 1);
      tc::mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      tc::mbar_init(&acc_full[b], 1);
      tc::mbar_init(&acc_empty[b], 4);
    }
    tc::mbar_init(drain, 1);
    *s_fail = 0;
    tc::fence_mbar_init();
  }
  if (warp == 1) tc::tmem_alloc(tmem_slot, TMEM_COLS);
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // The next kernel may launch now; it waits for this grid before its own dependent
  // accesses.  This grid's roles wait for the previous one before theirs: the producer
  // after requesting its first weight tiles, the epilogue before any global access, the
  // MMA issuer not at all (it only reads shared memory the producer filled).
  pdl_trigger();

  if (warp == 0 && lane == 0) {
    // ---------------------------------------------------------- TMA producer
    tc::tma_prefetch_desc(&tmA);
    tc::tma_prefetch_desc(&tmB);
    if (EPI == kEpiSwiGLU) tc::tma_prefetch_desc(&tmB2);
    auto load_b = [&](uint8_t* sb, uint64_t* bar, int kt, int n0) {
      if (EPI == kEpiSwiGLU) {
        tc::tma_load_2d(sb, &tmB, bar, kt * BK, n0);
        tc::tma_load_2d(sb + B_BYTES / 2, &tmB2, bar, kt * BK, n0);
      } else {
        tc::tma_load_2d(sb, &tmB, bar, kt * BK, n0);
      }
    };
    int it = 0;  // stage-ring position, continued across segments (= stages filled)
    bool ok = true;
    SegWalk wk(num_k, n_tiles, cut);
    int t = 0, k_lo = 0, k_hi = 0;
    bool have = wk.next(t, k_lo, k_hi);
    int kt = k_lo;
    // The weights never depend on the previous kernel: the first STAGES weight tiles
    // are requested before waiting for it (on fresh stages), their activation tiles after.
    int pre_m0[STAGES], pre_kt[STAGES];
    while (have && it < STAGES) {
      uint8_t* sa = smem + it * STAGE_BYTES;
      tc::mbar_arrive_expect_tx(&full[it], STAGE_BYTES);
      load_b(sa + A_BYTES, &full[it], kt, (t / n_mt) * ncols_out);
      pre_m0[it] = (t % n_mt) * BM, pre_kt[it] = kt;
      ++it;
      if (++kt == k_hi && (have = wk.next(t, k_lo, k_hi))) kt = k_lo;
    }
    pdl_wait();  // the previous kernel on the stream is complete from here on
    for (int j = 0; j < it; ++j) tc::tma_load_2d(smem + j * STAGE_BYTES, &tmA, &full[j], pre_kt[j] * BK, pre_m0[j]);
    while (ok && have) {
      const int m0 = (t % n_mt) * BM, n0 = (t / n_mt) * ncols_out;
      for (; kt < k_hi; ++kt, ++it) {
        const int s = it % STAGES;
        if (!(ok = tc::mbar_wait(&empty[s], ((it / STAGES) & 1) ^ 1, err, lim))) break;
        uint8_t* sa = smem + s * STAGE_BYTES;
        tc::mbar_arrive_expect_tx(&full[s], STAGE_BYTES);
        tc::tma_load_2d(sa, &tmA, &full[s], kt * BK, m0);
        load_b(sa + A_BYTES, &full[s], kt, n0);
      }
      if (!ok) break;
      if ((have = wk.next(t, k_lo, k_hi))) kt = k_lo;
    }
    // no copy may land after the CTA has finished: wait (with the full limit) for the
    // last filling of every stage -- already complete unless a wait above gave up
    for (int j = it > STAGES ? it - STAGES : 0; j < it; ++j) tc::mbar_wait(&full[j % STAGES], (j / STAGES) & 1, err);
  } else if (warp == 1 && lane == 0) {
    // ---------------------------------------------------------- MMA issuer
    constexpr uint32_t idesc = tc::idesc_bf16_f32(BM, BN);
    bool ok = true;
    int it = 0, lt = 0;
    SegWalk wk(num_k, n_tiles, cut);
    int t, k_lo, k_hi;
    for (; ok && wk.next(t, k_lo, k_hi); ++lt) {
      const int b = lt & 1;
      // accumulator b is free once the epilogue has read the segment two back
      if (!(ok = tc::mbar_wait(&acc_empty[b], ((lt >> 1) & 1) ^ 1, err, lim))) break;
      tc::tc_fence_after();
      const uint32_t d = tmem + (uint32_t)(b * BN);
      for (int kt = k_lo; kt < k_hi; ++kt, ++it) {
        const int s = it % STAGES;
        if (!(ok = tc::mbar_wait(&full[s], (it / STAGES) & 1, err, lim))) break;
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
    // no MMA may still run (reading shared memory, writing TMEM) after the CTA finished
    tc::mma_commit(drain);
    tc::mbar_wait(drain, 0, err);
  } else if (warp >= 2) {
    // ---------------------------------------------------------- epilogue
    pdl_wait();  // the previous kernel on the stream is complete from here on
    const int quarter = warp & 3;  // TMEM lanes this warp may access
    const int row = quarter * 32 + lane;
    int lt = 0;
    SegWalk wk(num_k, n_tiles, cut);
    int t, k_lo, k_hi;
    // Once a wait of this warp has given up, it waits no more (`dead`) but walks the
    // same segments and passes the same named barriers as the other epilogue warps,
    // storing nothing; the K-cut path leaves all four warps at the same barrier.
    bool dead = false;
    for (; wk.next(t, k_lo, k_hi); ++lt) {
      const int b = lt & 1;
      const int m0 = (t % n_mt) * BM, n0 = (t / n_mt) * ncols_out, ntile = t / n_mt;
      const int m = m0 + row;
      const bool ok = !dead && tc::mbar_wait_warp(&acc_full[b], (lt >> 1) & 1, err, lim);
      dead = !ok;
      tc::tc_fence_after();
      const uint32_t taddr = tmem + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(b * BN);
      float v[32], u2[32];
      if (k_lo != 0 || k_hi != num_k) {
        // this segment's partial of the tile's rows, then: is it the tile's last segment?
        const int zk = cut.zk;
        // the tile's segments q = 0 .. n_seg - 1 in K order and their slots
        const int kf = zk ? (int)((long)t * num_k / zk) : 0;
        const int n_seg = zk ? (int)(((long)t * num_k + num_k - 1) / zk) - kf + 1 : cut.splits;
        auto slot_of = [&](int q) { return zk ? seg_slot(t, kf + q, zk, num_k) : t * cut.splits + q; };
        const int my_slot = zk ? seg_slot(t, blockIdx.x, zk, num_k) : t * cut.splits + k_lo / cut.kps;
        // slot layout [32-column chunk][float4 of the chunk][row]: a warp's stores (32
        // rows, one float4 each) are 512 contiguous bytes
        float4* pr = (float4*)(g.part + (size_t)my_slot * BM * BN) + row;
        for (int c = 0; c < BN; c += 32) {
          tc::tmem_ld32(taddr + c, v);
          if (ok && m < g.M)
#pragma unroll
            for (int i = 0; i < 8; ++i)
              pr[((c / 32) * 8 + i) * BM] = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
        }
        tc::tc_fence_before();
        __syncwarp();
        if (lane == 0) tc::mbar_arrive(&acc_empty[b]);
        __threadfence();
        // the four epilogue warps pass the same barriers per unit and leave together
        if (!ok) *s_fail = 1;
        asm volatile("bar.sync 1, 128;" ::: "memory");
        if (zk) {
          // stream-K: count the segment in; every CTA sums split tiles after its own work
          if (threadIdx.x == 64) atomicAdd(&g.tile_cnt[t], 1);
          const bool all_ok = *s_fail == 0;
          asm volatile("bar.sync 1, 128;" ::: "memory");
          if (!all_ok) break;
          continue;
        }
        if (threadIdx.x == 64) *s_last = atomicAdd(&g.tile_cnt[t], 1) == n_seg - 1;
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
          // valid rows still spread over all of them; loads of several segments in flight
          // rows fastest, so that a warp's loads of one float4 are contiguous
          const int rows_v = min(BM, g.M - m0), nch = ncols_out / 32;
          for (int w = threadIdx.x - 64; w < rows_v * nch; w += 128) {
            const int r = w % rows_v, cc = w / rows_v;
#pragma unroll
            for (int i = 0; i < 32; ++i) v[i] = 0.f, u2[i] = 0.f;
#pragma unroll 4
            for (int q = 0; q < n_seg; ++q) {  // segment order: the same sums whoever finishes last
              const float4* pq = (const float4*)(g.part + (size_t)slot_of(q) * BM * BN) + r;
#pragma unroll
              for (int i = 0; i < 8; ++i) {
                const float4 a4 = __ldcg(pq + (cc * 8 + i) * BM);
                v[4 * i] += a4.x, v[4 * i + 1] += a4.y, v[4 * i + 2] += a4.z, v[4 * i + 3] += a4.w;
                if (EPI == kEpiSwiGLU) {
                  const float4 b4 = __ldcg(pq + ((cc + BN / 64) * 8 + i) * BM);
                  u2[4 * i] += b4.x, u2[4 * i + 1] += b4.y, u2[4 * i + 2] += b4.z, u2[4 * i + 3] += b4.w;
                }
              }
            }
            epi32<EPI>(g, m0 + r, n0 + cc * 32, v, u2);
          }
        }
        if (threadIdx.x == 64) g.tile_cnt[t] = 0;  // ready for the next launch
        if (!all_ok) break;
        continue;
      }
      if (EPI == kEpiSsdRead) {
        // The tile's 256 columns are the two state rows hp0, hp0 + 1 (d_state 128) of
        // one head h of request m: add their readout C_t . h0[hp] times the head's decay
        // to y.  All loads of a round are issued before their use -- dt of 16 positions,
        // C of 4 positions x 32 states (shared by both rows), y as float2 pairs -- so a
        // tile costs a few L2 round trips.  TMEM loads by all lanes; global memory only
        // for valid rows.
        const SsdReadArgs& r = g.ssd;
        const bool live = ok && m < g.M;
        const bf16* cm = (const bf16*)r.Cm;
        const bf16* dtr = (const bf16*)r.dt_raw;
        const int hp0 = n0 / 128, h = hp0 / r.P;
        const float Ah = r.A[h], bias = r.dt_bias ? r.dt_bias[h] : 0.f;
        float cum = 0.f;
        for (int t0 = 0; t0 < r.K; t0 += 16) {
          const int tn = min(16, r.K - t0);
          float e[16], acc0[16], acc1[16];
#pragma unroll
          for (int t = 0; t < 16; ++t) {
            float dt = 0.f;
            if (live && t < tn) dt = __bfloat162float(dtr[((size_t)m * r.K + t0 + t) * r.dt_rs + h]);
            e[t] = dt;
            acc0[t] = 0.f, acc1[t] = 0.f;
          }
#pragma unroll
          for (int t = 0; t < 16; ++t) {
            float dt = e[t];
            if (r.dt_bias) dt = softplus(dt + bias);
            cum += t < tn ? dt * Ah : 0.f;
            e[t] = expf(cum);
          }
          for (int cb = 0; cb < 128; cb += 32) {
            float v1[32];
            tc::tmem_ld32(taddr + cb, v);
            tc::tmem_ld32(taddr + 128 + cb, v1);
            if (!live) continue;
#pragma unroll
            for (int tg = 0; tg < 16; tg += 4) {
              if (tg >= tn) break;
              uint4 w[4][4];
#pragma unroll
              for (int t = 0; t < 4; ++t) {
                const int tt = min(tg + t, tn - 1);
                const uint4* cp = (const uint4*)(cm + ((size_t)m * r.K + t0 + tt) * r.c_rs + cb);
#pragma unroll
                for (int q = 0; q < 4; ++q) w[t][q] = __ldg(cp + q);
              }
#pragma unroll
              for (int t = 0; t < 4; ++t) {
                float a0 = 0.f, a1 = 0.f;
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                  const uint32_t wv[4] = {w[t][q].x, w[t][q].y, w[t][q].z, w[t][q].w};
#pragma unroll
                  for (int k = 0; k < 4; ++k) {
                    const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&wv[k]));
                    a0 = fmaf(f.x, v[q * 8 + 2 * k], a0);
                    a0 = fmaf(f.y, v[q * 8 + 2 * k + 1], a0);
                    a1 = fmaf(f.x, v1[q * 8 + 2 * k], a1);
                    a1 = fmaf(f.y, v1[q * 8 + 2 * k + 1], a1);
                  }
                }
                acc0[tg + t] += a0;
                acc1[tg + t] += a1;
              }
            }
          }
          if (!live) continue;
          float2 yv[16];
#pragma unroll
          for (int t = 0; t < 16; ++t)
            if (t < tn) yv[t] = *(const float2*)(r.y + ((size_t)m * r.K + t0 + t) * r.y_rs + hp0);
#pragma unroll
          for (int t = 0; t < 16; ++t)
            if (t < tn)
              *(float2*)(r.y + ((size_t)m * r.K + t0 + t) * r.y_rs + hp0) =
                  make_float2(fmaf(e[t], acc0[t], yv[t].x), fmaf(e[t], acc1[t], yv[t].y));
        }
      } else if (EPI == kEpiRope) {
        // heads of D columns, aligned with the tile (D divides BN): chunk pairs (i, i + D/2)
        const int D = g.rope.D, half = D / 2;
        for (int h0 = 0; h0 < BN; h0 += D) {
          for (int q = 0; q < half; q += 32) {
            float w2[32];
            tc::tmem_ld32(taddr + h0 + q, v);
            tc::tmem_ld32(taddr + h0 + half + q, w2);
            if (!ok || m >= g.M) continue;
            const int col = n0 + h0 + q;
            if (col < g.rope.cols) rope_rotate(g.rope, m, q, v, w2);
            epi32<EPI>(g, m, col, v, u2);
            epi32<EPI>(g, m, col + half, w2, u2);
          }
        }
      } else if (EPI == kEpiArgmax) {
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
    }
    if (cut.zk && *s_fail == 0) {
      // stream-K (one row of tiles): the sums of the split tiles, spread over the epilogue
      // threads of all CTAs as (tile, row, 32-column chunk) items, rows fastest.  An item
      // waits (bounded) until all segments of its tile are counted in, then adds their
      // partials in K order -- the same sums whichever CTA takes it.  Every CTA reaches
      // this phase only after its own segments, so no wait depends on a waiting CTA.
      // kEpiRope: an item is a pair of chunks (i, i + D/2) of one head, summed and rotated
      // together (cpd chunks per head, hpc pairs per head)
      const int zk = cut.zk, rows_v = min(BM, g.M), nch = ncols_out / 32;
      const int cpd = EPI == kEpiRope ? g.rope.D / 32 : 1, hpc = cpd / 2;
      const int n_it = EPI == kEpiRope ? nch / 2 : nch;  // items per row of a tile
      const long per_tile = (long)rows_v * n_it, n_items = (long)n_tiles * per_tile;
      float v[32], u2[32];
      int waited = -1;
      for (long it = (long)blockIdx.x * 128 + (threadIdx.x - 64); it < n_items; it += (long)gridDim.x * 128) {
        const int t = (int)(it / per_tile), rem = (int)(it - (long)t * per_tile);
        const int r = rem % rows_v, ci = rem / rows_v;
        const int cc = EPI == kEpiRope ? (ci / hpc) * cpd + ci % hpc : ci;  // (first) chunk of the item
        const int kf = (int)((long)t * num_k / zk), n_seg = (int)(((long)t * num_k + num_k - 1) / zk) - kf + 1;
        if (n_seg == 1) continue;
        if (t != waited) {
          if (!wait_count(&g.tile_cnt[t], n_seg, err, lim)) break;
          waited = t;
        }
#pragma unroll
        for (int i = 0; i < 32; ++i) v[i] = 0.f, u2[i] = 0.f;
        // kEpiRope: u2 holds the partner chunk cc + hpc; SwiGLU: the up projection
        const int c2 = EPI == kEpiRope ? cc + hpc : cc + BN / 64;
#pragma unroll 2
        for (int q = 0; q < n_seg; ++q) {
          const float4* pq = (const float4*)(g.part + (size_t)seg_slot(t, kf + q, zk, num_k) * BM * BN) + r;
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const float4 a4 = __ldcg(pq + (cc * 8 + i) * BM);
            v[4 * i] += a4.x, v[4 * i + 1] += a4.y, v[4 * i + 2] += a4.z, v[4 * i + 3] += a4.w;
            if (EPI == kEpiSwiGLU || EPI == kEpiRope) {
              const float4 b4 = __ldcg(pq + (c2 * 8 + i) * BM);
              u2[4 * i] += b4.x, u2[4 * i + 1] += b4.y, u2[4 * i + 2] += b4.z, u2[4 * i + 3] += b4.w;
            }
          }
        }
        if (EPI == kEpiRope) {
          const int col = t * ncols_out + cc * 32;
          if (col < g.rope.cols) rope_rotate(g.rope, r, (cc % cpd) * 32, v, u2);
          epi32<EPI>(g, r, col, v, u2);
          epi32<EPI>(g, r, t * ncols_out + c2 * 32, u2, v);
        } else {
          epi32<EPI>(g, r, t * ncols_out + cc * 32, v, u2);
        }
      }
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
bool launch_tc(const GemmArgs& g, KCut cut, cudaStream_t s, int* err) {
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
  const long n_tiles = (long)cdiv(g.M, BM) * cdiv(g.N, ncols_out);
  // chunks, or (tile, split) units
  const long n_units = cut.zk > 0 ? cdiv(n_tiles * cdiv(g.K, BK), cut.zk) : n_tiles * cut.splits;
  const int sms = dev < 64 && n_sm[dev] > 0 ? n_sm[dev] : 148;
  const int grid = n_units < sms ? (int)n_units : sms;
  launch_pdl(gemm_tc_kernel<EPI>, grid, THREADS, SMEM_BYTES, s, ta, tb, tb2, g, cut, err);
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

// How gemm() cuts the K loop of this shape (see the kernel's header):
//   one row of tiles, and whole tiles would leave more than 8% of the last wave idle
//   (within 8 waves): stream-K, an equal share of the line per SM, chunks of at least
//   4 K blocks;
//   several rows, fewer tiles than half the SMs: about one (tile, split) unit per SM,
//   at least four K blocks per split, every split non-empty;
//   else whole tiles.
KCut gemm_kcut(int dtype, GemmEpi epi, int M, int N, int K) {
  KCut cut{0, 1, cdiv(K, BK)};
  if (dtype != HSPEC_DTYPE_BF16 || epi == kEpiArgmax || epi == kEpiSsdRead) return cut;
  const long n_tiles = gemm_tile_count(dtype, epi, M, N), num_k = cdiv(K, BK), sms = device_sms();
  if (n_tiles <= 0) return cut;
  if (cdiv(M, BM) == 1) {
    if (n_tiles >= 8 * sms) return cut;
    // With 64+ rows the fp32 partials of a cut K loop are large (up to 128 KB per
    // segment); with enough whole tiles to keep HBM busy (each SM streams its weight
    // tiles well above its share of HBM bandwidth) whole tiles are faster: the SwiGLU
    // GEMM at 128 rows and 16384 columns measured 77 -> 66 us.
    if (M >= 64 && n_tiles >= 112) return cut;
    const long waves = cdiv(n_tiles, sms);
    if ((double)n_tiles / (double)(waves * sms) >= 0.92) return cut;
    const long zk = cdiv(n_tiles * num_k, sms);
    if (zk >= 4) cut.zk = (int)zk;
    return cut;
  }
  if (n_tiles * 2 > sms) return cut;
  long sp = sms / n_tiles;
  if (sp > num_k / 4) sp = num_k / 4;
  if (sp < 2) return cut;
  cut.kps = cdiv(num_k, sp);
  cut.splits = cdiv(num_k, cut.kps);
  return cut;
}

// Partial tiles a cut K loop needs: two per stream-K chunk, one per split unit (at most
// one unit per SM), BM x BN fp32 each.
size_t gemm_kcut_bytes(int dtype, GemmEpi epi, int M, int N, int K) {
  const KCut cut = gemm_kcut(dtype, epi, M, N, K);
  if (cut.zk > 0) return (size_t)2 * device_sms() * BM * BN * sizeof(float);
  if (cut.splits > 1) return (size_t)gemm_tile_count(dtype, epi, M, N) * cut.splits * BM * BN * sizeof(float);
  return 0;
}

bool gemm_rope_fusable(int dtype, int M, int N, int K, int D) {
  if (dtype != HSPEC_DTYPE_BF16 || (D != 64 && D != 128)) return false;
  return gemm_kcut(dtype, kEpiRope, M, N, K).splits == 1;  // whole tiles or stream-K
}

bool gemm(int dtype, GemmEpi epi, const GemmArgs& g, cudaStream_t s) {
  if (dtype != HSPEC_DTYPE_BF16) {
    if (epi == kEpiSsdRead || epi == kEpiRope) {
      set_error("the SSD readout and RoPE epilogues are bf16-only");
      return false;
    }
    gemm_simt_f32(epi, g, s);
    return true;
  }
  if (epi == kEpiSsdRead && (g.ssd.N != 128 || g.ssd.P % 2 || g.ssd.c_rs % 8 || g.ssd.y_rs % 2 ||
                             (((uintptr_t)g.ssd.Cm) & 15) || (((uintptr_t)g.ssd.y) & 7))) {
    set_error("SSD readout epilogue: d_state 128, even head dim, 16-byte aligned C rows, 8-byte aligned y");
    return false;
  }
  // TMA needs 16-byte aligned bases and row strides.
  if ((g.lda % 8) || (g.ldb % 8) || (((uintptr_t)g.A) & 15) || (((uintptr_t)g.B) & 15) ||
      (g.B2 && (((uintptr_t)g.B2) & 15))) {
    set_error("bf16 GEMM operands need 16-byte aligned bases and leading dimensions (lda=%ld ldb=%ld)",
              g.lda, g.ldb);
    return false;
  }
  int* err = device_error_word();
  KCut cut{0, 1, cdiv(g.K, BK)};
  if (g.part && g.tile_cnt && !(epi == kEpiStore && g.out_f32)) {
    const KCut c = gemm_kcut(dtype, epi, g.M, g.N, g.K);
    if ((c.zk > 0 || c.splits > 1) && gemm_kcut_bytes(dtype, epi, g.M, g.N, g.K) <= g.part_bytes &&
        gemm_tile_count(dtype, epi, g.M, g.N) <= g.max_tiles && !(((uintptr_t)g.part) & 15))
      cut = c;
  }
  switch (epi) {
    case kEpiStore: return launch_tc<kEpiStore>(g, cut, s, err);
    case kEpiResid: return launch_tc<kEpiResid>(g, cut, s, err);
    case kEpiSwiGLU: return launch_tc<kEpiSwiGLU>(g, cut, s, err);
    case kEpiArgmax: return launch_tc<kEpiArgmax>(g, cut, s, err);
    case kEpiSsdRead: return launch_tc<kEpiSsdRead>(g, cut, s, err);
    case kEpiRope: return launch_tc<kEpiRope>(g, cut, s, err);
  }
  return false;
}

}  // namespace hspec
