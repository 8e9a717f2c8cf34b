// Mamba-2 SSD block scan from an injected state, readout on the 5th-generation tensor
// cores (bf16 drafter, the whole block as one chunk of K <= 32 positions).
// H-Spec (arXiv 2609.24197) Abstract: each Mamba layer starts from the projected
// last-token hidden state and the block is evaluated in parallel; the chunked
// "state-space dual" form of Dao & Gu (2024) gives, for head h and position t,
//
//   y_t[p] = exp(cum_t) sum_n C_t[n] S[p][n]                      (the injected state)
//          + sum_{s<=t} (C_t . B_s) exp(cum_t - cum_s) dt_s x_s[p]  (inside the block)
//          + D_h x_t[p],                    cum_t = sum_{r<=t} dt_r A_h,
//
// and the state after the block,
//
//   hK[p][n] = exp(cum_{K-1}) S[p][n] + sum_s exp(cum_{K-1} - cum_s) dt_s x_s[p] B_s[n],
//
// the same sums as the step-by-step recurrence.  The state S = h0 of one request is
// H*P rows of N fp32 values: 2 MB per request and layer at Llama shapes, the only large
// operand, read once.  Its readout C . S^T is a dense contraction (K x N by N x H*P)
// and runs on tcgen05 as kind::tf32 with M = 128 state rows (heads x P), N = NT = 16 or
// 32 positions, K = 8 per instruction, the accumulator in TMEM.  So that the product is
// as exact as fp32, the state is split into hi = S with its 13 low mantissa bits
// cleared and lo = S - hi (exact in fp32, below 2^-10 |S|): the A operand of the first
// MMA is the state tile as it landed in shared memory, of which the tensor core reads
// the tf32 part -- hi (it drops the low mantissa bits; a GPU test with every low bit
// set checks this) -- and the second MMA reads lo from TMEM.  C is exact in tf32 (it
// comes from bf16); tf32 x tf32 products are exact and accumulate in fp32.
//
// Persistent kernel, one CTA per SM, a static range of (request, 128-row tile) items:
//   warp 0      TMA producer: the fp32 state tile (N / 32 boxes of 128 rows x 128 B,
//               128-byte swizzle) into one of three (NT = 32: two) stages.
//   warp 1      TMEM owner and MMA issuer: per tile N / 8 MMAs of the state's tf32 part
//               (from shared memory) as soon as the C^T operand is in place, then N / 8
//               of lo (from TMEM) once the transform has written it, into one of two
//               TMEM accumulators.
//   warps 2..5  transform group 0 (tiles k even), warps 6..9 group 1 (k odd); per tile,
//               one state row (= TMEM lane) per thread: for a new request the C^T
//               operand (bf16 -> fp32, swizzled) and the B rows, then C . B^T (one dot
//               product per thread); the tile's dt and cumulative decay (a segmented
//               warp scan); lo of the thread's row into the group's TMEM buffer, and
//               with a final state the row of hK; the in-block matrix L[t][s] =
//               (C_t . B_s) exp(cum_t - cum_s) dt_s; then the epilogue
//               y = exp(cum) (C S^T) + L x + D x, with x held in registers: L x + D x
//               while the tile's MMAs run, the readout term once they are done.  The
//               tile's global loads are issued before its waits, and the two groups
//               overlap each other's latencies.
// Every pipeline wait gives up after the call's limit and sets the device error word;
// before the CTA exits, the producer and the MMA issuer wait for their own copies and
// MMAs in flight.
#include <stdint.h>

#include "../../include/hspec.h"
#include "common.cuh"
#include "kernels.cuh"
#include "tc_prims.cuh"

namespace hspec {

int* device_error_word();

namespace {

constexpr int THREADS = 320;  // producer, MMA, 2 transform warpgroups
constexpr int ROWS = 128;    // MMA M: state rows (head, p) per tile
constexpr int NMAX = 128;    // d_state
constexpr int TILE_BYTES = ROWS * NMAX * 4;  // 64 KB
constexpr int HPT_MAX = 2;   // heads per tile (P >= 64)
// TMEM columns: lo of tile k in [128 (k % 2), +128), accumulator of tile k at 256 + NT (k % 2)
constexpr uint32_t TMEM_COLS = 512;

// NT: MMA N = positions per tile (the block, K <= NT, zero past K): 16 or 32.
template <int NT>
struct SsdTcLay {
  static constexpr int NSTAGE = NT == 16 ? 3 : 2;              // state-tile stages
  static constexpr int OFF_A = 0;                               // stages of the state tile
  static constexpr int OFF_B = OFF_A + NSTAGE * TILE_BYTES;     // C^T: [n/32][NT positions][128 B] fp32
  static constexpr int B_BYTES = NMAX / 32 * NT * 128;
  // per transform group g: the B rows, L^T, exp(cum) and D, C . B^T, dt and cum
  static constexpr int OFF_BR = OFF_B + B_BYTES;                // B rows: [2][NT][NMAX] bf16
  static constexpr int BR_BYTES = NT * NMAX * 2;
  static constexpr int OFF_L = OFF_BR + 2 * BR_BYTES;           // L^T: [2][HPT_MAX][NT (s)][NT (t)]
  static constexpr int L_BYTES = HPT_MAX * NT * NT * 4;
  static constexpr int OFF_E = OFF_L + 2 * L_BYTES;             // exp(cum): [2][HPT_MAX][NT], D_h: [2][HPT_MAX]
  static constexpr int E_BYTES = HPT_MAX * (NT + 1) * 4;
  static constexpr int OFF_CB = OFF_E + 2 * E_BYTES;            // C . B^T: [2][NT (s)][NT (t)]
  static constexpr int OFF_DT = OFF_CB + 2 * NT * NT * 4;       // dt, then cum: [2][2][HPT_MAX][NT]
  static constexpr int OFF_BAR = OFF_DT + 4 * HPT_MAX * NT * 4;
  static constexpr int SMEM = OFF_BAR + 256 + 1024;
};

struct SsdTcArgs {
  SsdArgs a;
  int* err;       // device error word
  int hpt;        // heads per tile = 128 / P
  int n_tiles;    // tiles per request = H / hpt
  int n_items;    // C * n_tiles
};

// hi: the value with its 13 low mantissa bits cleared (the tf32 value the tensor core
// reads); lo = v - hi is exact in fp32 and below 2^-10 |v|.
__device__ __forceinline__ uint32_t tf32_hi(uint32_t bits) { return bits & 0xFFFFE000u; }

// Loads issued where they stand (volatile: not moved towards their first use), so
// their latency overlaps the waits that follow.
__device__ __forceinline__ uint16_t ldg_u16(const void* p) {
  uint16_t v;
  asm volatile("ld.global.nc.u16 %0, [%1];" : "=h"(v) : "l"(p));
  return v;
}
__device__ __forceinline__ uint32_t ldg_u32(const void* p) {
  uint32_t v;
  asm volatile("ld.global.nc.u32 %0, [%1];" : "=r"(v) : "l"(p));
  return v;
}

// Instruction descriptor of kind::tf32: fp32 accumulator, tf32 A and B (K-major).
__host__ __device__ constexpr uint32_t idesc_tf32(int M, int N) {
  return (1u << 4) | (2u << 7) | (2u << 10) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

// A from TMEM (row i in lane i, one tf32 per 32-bit column)
__device__ __forceinline__ void mma_tf32_ts(uint32_t tmem_d, uint32_t tmem_a, uint64_t bdesc, uint32_t idesc,
                                            uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::tf32 [%0], [%1], %2, %3, p;\n\t}\n" ::"r"(tmem_d),
      "r"(tmem_a), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

__device__ __forceinline__ void mma_tf32(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                         uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::tf32 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(tmem_d),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// NT fp32 columns of this thread's TMEM lane
__device__ __forceinline__ void tmem_ld_nt(uint32_t taddr, float (&v)[16]) { tc::tmem_ld16(taddr, v); }
__device__ __forceinline__ void tmem_ld_nt(uint32_t taddr, float (&v)[32]) { tc::tmem_ld32(taddr, v); }

// HK: the final state is written (a separate instantiation, so that the draft step's
// scan carries none of its registers).
template <typename TDT, int NT, bool HK>
__global__ void __launch_bounds__(THREADS, 1) ssd_tc_kernel(const __grid_constant__ CUtensorMap h0_map, SsdTcArgs t) {
  using L = SsdTcLay<NT>;
  constexpr int NSTAGE = L::NSTAGE;
  const SsdArgs& a = t.a;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = tc::smem_u32(smem_raw);
  uint8_t* smem = smem_raw + (((raw + 1023) & ~1023u) - raw);
  uint8_t* sA = smem + L::OFF_A;
  uint8_t* sB = smem + L::OFF_B;
  uint8_t* sBR = smem + L::OFF_BR;
  float* sL = (float*)(smem + L::OFF_L);
  float* sE = (float*)(smem + L::OFF_E);
  float* sCB = (float*)(smem + L::OFF_CB);
  float* sDt = (float*)(smem + L::OFF_DT);
  uint64_t* a_full = (uint64_t*)(smem + L::OFF_BAR);  // [NSTAGE]
  uint64_t* a_empty = a_full + NSTAGE;                 // [NSTAGE]
  // [2] tile k: lo in TMEM buffer k % 2 and the C^T operand ready (one barrier per lo
  // buffer: the transform may finish tile k + 1 before the MMA thread has taken tile k,
  // and the phases of one barrier must not run two ahead of its waiter)
  uint64_t* lo_full = a_empty + NSTAGE;
  uint64_t* acc_full = lo_full + 2;                    // [2] MMAs of the accumulator's tile done
  uint64_t* d_free = acc_full + 2;                     // [2] epilogue has read the accumulator
  // [2] tile k: its state tile has landed and the C^T operand is written, so the MMAs
  // of the state's tf32 part may start before lo is ready
  uint64_t* hi_ready = d_free + 2;
  uint64_t* drain = hi_ready + 2;
  uint32_t* tmem_slot = (uint32_t*)(drain + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int P = a.P, N = a.N, K = a.K, hpt = t.hpt;
  const int nblk = N / 32;  // 128-byte column blocks of a state row
  int* err = t.err;
  const int i0 = (int)((long)blockIdx.x * t.n_items / gridDim.x);
  const int i1 = (int)((long)(blockIdx.x + 1) * t.n_items / gridDim.x);
  const uint64_t lim = a.wait_ns ? (uint64_t)a.wait_ns : tc::kWaitLimitNs;  // pipeline waits

  if (threadIdx.x == 0) {
    for (int s = 0; s < NSTAGE; ++s) {
      tc::mbar_init(&a_full[s], 1);
      tc::mbar_init(&a_empty[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      tc::mbar_init(&acc_full[s], 1);
      tc::mbar_init(&d_free[s], 4);
    }
    tc::mbar_init(&lo_full[0], 4);
    tc::mbar_init(&lo_full[1], 4);
    tc::mbar_init(&hi_ready[0], 4);
    tc::mbar_init(&hi_ready[1], 4);
    tc::mbar_init(drain, 1);
    tc::fence_mbar_init();
  }
  if (warp == 1) tc::tmem_alloc(tmem_slot, TMEM_COLS);
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  pdl_wait();  // the previous kernel on the stream is complete from here on
  pdl_trigger();

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      tc::tma_prefetch_desc(&h0_map);
      int filled = 0;
      for (int i = i0; i < i1; ++i, ++filled) {
        const int k = i - i0, st = k % NSTAGE;
        if (!tc::mbar_wait(&a_empty[st], ((k / NSTAGE) & 1) ^ 1, err, lim)) break;
        const int c = i / t.n_tiles, j = i % t.n_tiles;
        const int row0 = (c * a.H + j * hpt) * P;
        tc::mbar_arrive_expect_tx(&a_full[st], (uint32_t)(nblk * ROWS * 128));
        for (int b = 0; b < nblk; ++b)
          tc::tma_load_2d(sA + st * TILE_BYTES + b * ROWS * 128, &h0_map, &a_full[st], b * 32, row0);
      }
      // no copy may land after the CTA has finished: wait (with the full limit) for the
      // last filling of every stage -- already complete unless a wait gave up
      for (int k = filled > NSTAGE ? filled - NSTAGE : 0; k < filled; ++k)
        tc::mbar_wait(&a_full[k % NSTAGE], (k / NSTAGE) & 1, err);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ---------------------------------------------------------- MMA issuer
      const uint32_t idesc = idesc_tf32(ROWS, NT);
      const uint32_t b_base = tc::smem_u32(sB);
      for (int i = i0; i < i1; ++i) {
        const int k = i - i0, st = k % NSTAGE, db = k & 1;
        // accumulator db is free once the epilogue of tile k - 2 has read it
        if (k >= 2 && !tc::mbar_wait(&d_free[db], ((k >> 1) - 1) & 1, err, lim)) break;
        // the state's tf32 part (hi, read from shared memory as it landed) as soon as the
        // C^T operand is there; lo once the transform has written it to TMEM
        if (!tc::mbar_wait(&hi_ready[k & 1], (k >> 1) & 1, err, lim)) break;
        tc::tc_fence_after();
        const uint32_t st_addr = tc::smem_u32(sA + st * TILE_BYTES);
        const uint32_t lo = tmem + (uint32_t)(128 * (k & 1));
        const uint32_t d = tmem + 256u + (uint32_t)(db * NT);
        auto bdesc = [&](int kb) {
          return tc::sdesc_k128(b_base + (uint32_t)((kb >> 2) * NT * 128 + (kb & 3) * 32));
        };
#pragma unroll
        for (int kb = 0; kb < NMAX / 8; ++kb) {
          const uint32_t aoff = (uint32_t)((kb >> 2) * ROWS * 128 + (kb & 3) * 32);
          mma_tf32(d, tc::sdesc_k128(st_addr + aoff), bdesc(kb), idesc, kb > 0);
        }
        if (!tc::mbar_wait(&lo_full[k & 1], (k >> 1) & 1, err, lim)) break;
        tc::tc_fence_after();
#pragma unroll
        for (int kb = 0; kb < NMAX / 8; ++kb) mma_tf32_ts(d, lo + (uint32_t)(kb * 8), bdesc(kb), idesc, 1u);
        tc::mma_commit(&acc_full[db]);
        tc::mma_commit(&a_empty[st]);
      }
      tc::mma_commit(drain);
      tc::mbar_wait(drain, 0, err);
    }
  } else {
    // ------------------------------------------------------------ transform groups
    const int g = (warp - 2) >> 2;              // group: tiles k with k % 2 == g
    const int tid = threadIdx.x - 64 - 128 * g; // 0..127 within the group
    const int quarter = warp & 3;                // TMEM lanes of this warp
    const int row = quarter * 32 + lane;         // the state row (TMEM lane) of this thread
    const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
    const int hl = row / P, p = row % P;
    constexpr bool want_hK = HK;
    const TDT* dtp = (const TDT*)a.dt;
    const bf16* xg = (const bf16*)a.x;
    const bf16* Bg = (const bf16*)a.B;
    const bf16* Cg = (const bf16*)a.Cm;
    uint8_t* gBR = sBR + g * L::BR_BYTES;        // B rows [NT][NMAX] bf16
    float* gL = sL + g * HPT_MAX * NT * NT;      // [head][s][t]
    float* gE = sE + g * HPT_MAX * (NT + 1);
    float* gCB = sCB + g * NT * NT;
    float* gDt = sDt + g * 2 * HPT_MAX * NT;     // dt [head][t], then cum [head][t]
    int c_prev = -1;
    auto gsync = [&]() {
      if (g == 0) asm volatile("bar.sync 1, 128;" ::: "memory");
      else asm volatile("bar.sync 2, 128;" ::: "memory");
    };

    // The group's warps pass the same named barriers in the same order.  A warp whose
    // wait gave up (`failed`, warp-uniform) says so at the group's next barrier, which
    // ORs it over the group, and the whole group leaves the loop there.
    bool failed = false;
    for (int i = i0 + g; i < i1; i += 2) {
      const int k = i - i0, st = k % NSTAGE;
      const int c = i / t.n_tiles, j = i % t.n_tiles;
      const bool new_req = c != c_prev;
      // the tile's global loads first: x of this thread's row at every position (rows
      // past K re-read row K - 1 and count as zero), and (lane hh * NT + tt of the
      // group's first warps) dt of head hh at position tt
      // (NT = 16: the raw bits land one register each and are packed after the tile's
      // waits)
      uint32_t xw[NT / 2] = {};  // bf16 pairs: position 2i in the low half, 2i + 1 in the high half
      uint32_t xraw[NT == 16 ? NT : 1];
      {
        const bf16* xr = xg + (size_t)c * K * a.x_rs + (size_t)(j * hpt) * P + row;
        if constexpr (NT == 16) {
#pragma unroll
          for (int tt = 0; tt < NT; ++tt) xraw[tt] = ldg_u16(xr + (size_t)(tt < K ? tt : K - 1) * a.x_rs);
        } else {
#pragma unroll
          for (int tt = 0; tt < NT; tt += 2)
            xw[tt / 2] = (uint32_t)ldg_u16(xr + (size_t)(tt < K ? tt : K - 1) * a.x_rs) |
                         ((uint32_t)ldg_u16(xr + (size_t)(tt + 1 < K ? tt + 1 : K - 1) * a.x_rs) << 16);
        }
      }
      // x at position s (fp32; the bf16 bits in the upper half of a word)
      auto xval = [&](int s2) {
        return __uint_as_float((s2 & 1) ? (xw[s2 >> 1] & 0xFFFF0000u) : (xw[s2 >> 1] << 16));
      };
      const int dh = tid / NT, dtt = tid % NT;
      const bool dlane = tid < HPT_MAX * NT;
      const bool dlive = dlane && dh < hpt && dtt < K;
      const int dhead = j * hpt + (dh < hpt ? dh : 0);
      uint32_t draw_bits = 0, dA_bits = 0, dD_bits = 0, dbias_bits = 0;
      if (dlive) {
        const TDT* dp = dtp + (size_t)(c * K + dtt) * a.dt_rs + dhead;
        draw_bits = sizeof(TDT) == 2 ? (uint32_t)ldg_u16(dp) : ldg_u32(dp);
        dA_bits = ldg_u32(a.A + dhead);
        dD_bits = ldg_u32(a.D + dhead);
        if (a.dt_bias) dbias_bits = ldg_u32(a.dt_bias + dhead);
      }
      // the state tile has landed; for a new request also the MMAs of the previous tile
      // (the last reader of the C^T operand) are done
      bool ok = !failed && tc::mbar_wait_warp(&a_full[st], (k / NSTAGE) & 1, err, lim);
      if (ok && new_req && k >= 1) ok = tc::mbar_wait_warp(&acc_full[(k - 1) & 1], ((k - 1) >> 1) & 1, err, lim);
      if (g == 0 ? tc::bar_or<1, 128>(!ok) : tc::bar_or<2, 128>(!ok)) break;  // the group's barrier
      tc::tc_fence_after();
      if constexpr (NT == 16) {
#pragma unroll
        for (int tt = 0; tt < NT; tt += 2) xw[tt / 2] = xraw[tt] | (xraw[tt + 1] << 16);
      }
      if (new_req) {
        // C^T operand: row tt (position) of 128-byte column blocks, zero past K
        constexpr int PER = NT * NMAX / 4 / 128;  // float4 entries per thread
        uint2 rw[PER];
#pragma unroll
        for (int q = 0; q < PER; ++q) {
          const int e = tid + 128 * q, tt = e / (NMAX / 4), n4 = (e % (NMAX / 4)) * 4;
          rw[q] = tt < K ? *(const uint2*)(Cg + (size_t)(c * K + tt) * a.bc_rs + n4) : make_uint2(0u, 0u);
        }
#pragma unroll
        for (int q = 0; q < PER; ++q) {
          const int e = tid + 128 * q, tt = e / (NMAX / 4), n4 = (e % (NMAX / 4)) * 4;
          const float2 lo2 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&rw[q].x));
          const float2 hi2 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&rw[q].y));
          const int ch = (n4 & 31) >> 2;
          *(float4*)(sB + (n4 >> 5) * NT * 128 + tt * 128 + ((ch ^ (tt & 7)) << 4)) =
              make_float4(lo2.x, lo2.y, hi2.x, hi2.y);
        }
        // B rows of the request (bf16 as stored; positions < K), for C . B^T and the
        // final state
        for (int e = tid; e < K * (NMAX / 4); e += 128) {
          const int tt = e / (NMAX / 4), n4 = (e % (NMAX / 4)) * 4;
          *(uint2*)(gBR + (tt * NMAX + n4) * 2) = *(const uint2*)(Bg + (size_t)(c * K + tt) * a.bc_rs + n4);
        }
        c_prev = c;
      }
      // the tile's heads: dt, cum = inclusive scan of dt A_h (segmented, NT lanes), exp(cum)
      if (dlane) {
        float d = sizeof(TDT) == 2 ? __bfloat162float(__ushort_as_bfloat16((unsigned short)draw_bits))
                                   : __uint_as_float(draw_bits);
        if (dlive && a.dt_bias) d = softplus(d + __uint_as_float(dbias_bits));
        const float dA = __uint_as_float(dA_bits), dD = __uint_as_float(dD_bits);
        float cum = dlive ? d * dA : 0.f;
#pragma unroll
        for (int o = 1; o < NT; o <<= 1) {
          const float v = __shfl_up_sync(0xffffffffu, cum, o, NT);
          if (dtt >= o) cum += v;
        }
        if (dlive) {
          gDt[dh * NT + dtt] = d;
          gDt[(HPT_MAX + dh) * NT + dtt] = cum;
          gE[dh * (NT + 1) + dtt] = expf(cum);
          if (dtt == 0) gE[dh * (NT + 1) + NT] = dD;
        }
      }
      tc::fence_proxy_async();  // C^T was written by threads; the MMAs read it
      gsync();  // the C^T operand and B rows of a new request, dt and cum are complete
      if (lane == 0) tc::mbar_arrive(&hi_ready[g]);
      // this thread's state row: lo = S - hi into the group's TMEM buffer (free: the
      // group's previous tile finished its MMAs); with a final state also its row of hK
      {
        const uint8_t* rowp = sA + st * TILE_BYTES + row * 128;
        float w[want_hK ? NT : 1], eK = 0.f;
        if constexpr (want_hK) {
          const float cK = gDt[(HPT_MAX + hl) * NT + (K - 1)];
          eK = expf(cK);
#pragma unroll
          for (int s2 = 0; s2 < NT; ++s2)
            w[s2] = s2 < K ? expf(cK - gDt[(HPT_MAX + hl) * NT + s2]) * gDt[hl * NT + s2] * xval(s2) : 0.f;
        }
        float* hKr = want_hK ? a.hK + ((size_t)(c * a.H + j * hpt + hl) * P + p) * N : nullptr;
#pragma unroll
        for (int cb = 0; cb < NMAX / 32; ++cb) {
          uint4 v[8];
#pragma unroll
          for (int ch = 0; ch < 8; ++ch) v[ch] = *(const uint4*)(rowp + cb * ROWS * 128 + ((ch ^ (row & 7)) << 4));
          uint32_t lo[32];
#pragma unroll
          for (int ch = 0; ch < 8; ++ch) {
            lo[4 * ch + 0] = __float_as_uint(__uint_as_float(v[ch].x) - __uint_as_float(tf32_hi(v[ch].x)));
            lo[4 * ch + 1] = __float_as_uint(__uint_as_float(v[ch].y) - __uint_as_float(tf32_hi(v[ch].y)));
            lo[4 * ch + 2] = __float_as_uint(__uint_as_float(v[ch].z) - __uint_as_float(tf32_hi(v[ch].z)));
            lo[4 * ch + 3] = __float_as_uint(__uint_as_float(v[ch].w) - __uint_as_float(tf32_hi(v[ch].w)));
          }
          tc::tmem_st32_nowait(tmem + lane_off + (uint32_t)(128 * g + 32 * cb), lo);
          if constexpr (want_hK) {
            // hK[n] = exp(cum_{K-1}) S[n] + sum_s w_s B_s[n], n in this 32-column block
            float acc[32];
#pragma unroll
            for (int ch = 0; ch < 8; ++ch) {
              acc[4 * ch + 0] = eK * __uint_as_float(v[ch].x);
              acc[4 * ch + 1] = eK * __uint_as_float(v[ch].y);
              acc[4 * ch + 2] = eK * __uint_as_float(v[ch].z);
              acc[4 * ch + 3] = eK * __uint_as_float(v[ch].w);
            }
#pragma unroll
            for (int s2 = 0; s2 < NT; ++s2) {
              if (s2 >= K) break;
              const uint4* br = (const uint4*)(gBR + (s2 * NMAX + cb * 32) * 2);  // 32 bf16, same for all lanes
              const float ws = w[s2];
#pragma unroll
              for (int q = 0; q < 4; ++q) {
                const uint4 b8 = br[q];
                const uint32_t bw[4] = {b8.x, b8.y, b8.z, b8.w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                  const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&bw[e]));
                  acc[8 * q + 2 * e] = fmaf(ws, f.x, acc[8 * q + 2 * e]);
                  acc[8 * q + 2 * e + 1] = fmaf(ws, f.y, acc[8 * q + 2 * e + 1]);
                }
              }
            }
#pragma unroll
            for (int e = 0; e < 32; e += 4)
              *(float4*)(hKr + cb * 32 + e) = make_float4(acc[e], acc[e + 1], acc[e + 2], acc[e + 3]);
          }
        }
        tc::tmem_wait_st();
      }
      if (new_req) {
        // C . B^T of the request, entries s <= t: one dot product of N per thread, entry
        // e = s K + t (a warp shares s, so its B row reads are broadcasts, and its C rows
        // t fall on distinct 16-byte chunks of the swizzle)
        for (int e = tid; e < K * K; e += 128) {
          const int ss = e / K, tt = e - ss * K;
          if (ss > tt) continue;
          float v = 0.f;
#pragma unroll
          for (int cb = 0; cb < NMAX / 32; ++cb) {
#pragma unroll
            for (int ch = 0; ch < 8; ++ch) {
              const float4 cv = *(const float4*)(sB + cb * NT * 128 + tt * 128 + ((ch ^ (tt & 7)) << 4));
              const uint2 bw = *(const uint2*)(gBR + (ss * NMAX + cb * 32 + 4 * ch) * 2);
              const float2 b01 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&bw.x));
              const float2 b23 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&bw.y));
              v = fmaf(cv.x, b01.x, v);
              v = fmaf(cv.y, b01.y, v);
              v = fmaf(cv.z, b23.x, v);
              v = fmaf(cv.w, b23.y, v);
            }
          }
          gCB[ss * NT + tt] = v;  // [s][t]: consecutive threads, consecutive words
        }
      }
      gsync();  // C . B^T complete
      // L^T[s][t] = (C_t . B_s) exp(cum_t - cum_s) dt_s for s <= t, else 0: entry
      // e = (head, s, t) of a HPT_MAX x NT x NT grid (t fastest, so that a warp's reads
      // of C . B^T and writes of L^T fall on consecutive words), loads first
      {
        constexpr int PER = HPT_MAX * NT * NT / 128;
#pragma unroll
        for (int q0 = 0; q0 < PER; q0 += 4) {
          float cb[4], ct[4], cs[4], dts[4];
          bool live[4];
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const int e = tid + 128 * (q0 + q), hh = e / (NT * NT), ss = (e / NT) % NT, tt = e % NT;
            live[q] = hh < hpt && tt < K && ss <= tt;
            cb[q] = gCB[ss * NT + tt];
            ct[q] = gDt[(HPT_MAX + hh) * NT + tt];
            cs[q] = gDt[(HPT_MAX + hh) * NT + ss];
            dts[q] = gDt[hh * NT + ss];
          }
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const int e = tid + 128 * (q0 + q), hh = e / (NT * NT), ss = (e / NT) % NT, tt = e % NT;
            gL[(hh * NT + ss) * NT + tt] = live[q] ? cb[q] * expf(ct[q] - cs[q]) * dts[q] : 0.f;
          }
        }
      }
      // C^T was written by threads and lo by tcgen05.st; the MMA reads them
      tc::fence_proxy_async();
      tc::tc_fence_before();
      gsync();
      if (lane == 0) tc::mbar_arrive(&lo_full[g]);

      // epilogue: y_t = exp(cum_t) (C S^T)_t + sum_{s<=t} L_ts x_s + D_h x_t, the last two
      // terms while the tile's MMAs run, the first once they are done
      const int h = j * hpt + hl;
      const float* LTh = gL + hl * NT * NT;  // [s][t]
      const float* Eh = gE + hl * (NT + 1);
      // (x past K repeats position K - 1: L is zero in the columns s >= K, and the
      // positions t >= K are never stored)
      float acc[NT];
#pragma unroll
      for (int tt = 0; tt < NT; ++tt) acc[tt] = Eh[NT] * xval(tt);
#pragma unroll
      for (int s2 = 0; s2 < NT; ++s2) {
        const float xs = xval(s2);
#pragma unroll
        for (int t4 = (s2 & ~3); t4 < NT; t4 += 4) {
          const float4 l4 = *(const float4*)(LTh + s2 * NT + t4);  // zero above the diagonal and past K
          acc[t4 + 0] = fmaf(l4.x, xs, acc[t4 + 0]);
          acc[t4 + 1] = fmaf(l4.y, xs, acc[t4 + 1]);
          acc[t4 + 2] = fmaf(l4.z, xs, acc[t4 + 2]);
          acc[t4 + 3] = fmaf(l4.w, xs, acc[t4 + 3]);
        }
      }
      ok = tc::mbar_wait_warp(&acc_full[g], (k >> 1) & 1, err, lim);
      if (!ok) {
        failed = true;
        continue;  // the whole warp (the answer is warp-uniform); the group leaves at its next barrier
      }
      tc::tc_fence_after();
      {
        float dv[NT];
        tmem_ld_nt(tmem + lane_off + 256u + (uint32_t)(g * NT), dv);
        tc::tc_fence_before();
        __syncwarp();
        if (lane == 0) tc::mbar_arrive(&d_free[g]);
#pragma unroll
        for (int tt = 0; tt < NT; ++tt) acc[tt] = fmaf(Eh[tt], dv[tt], acc[tt]);
      }
      float* yr = a.y + (size_t)c * K * a.y_rs + (size_t)h * P + p;
#pragma unroll
      for (int tt = 0; tt < NT; ++tt)
        if (tt < K) yr[(size_t)tt * a.y_rs] = acc[tt];
    }
  }
  __syncthreads();
  if (warp == 1) {
    tc::tc_fence_after();
    tc::tmem_dealloc(tmem, TMEM_COLS);
  }
}

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn_ssd() {
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

template <typename TDT, int NT, bool HK>
bool launch_ssd_tc(const SsdArgs& a, cudaStream_t s) {
  static bool attr_set[64] = {};
  static int n_sm[64] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 64 && !attr_set[dev]) {
    if (cudaFuncSetAttribute(ssd_tc_kernel<TDT, NT, HK>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             SsdTcLay<NT>::SMEM) != cudaSuccess)
      return false;
    cudaDeviceGetAttribute(&n_sm[dev], cudaDevAttrMultiProcessorCount, dev);
    attr_set[dev] = true;
  }
  EncodeTiledFn fn = encode_fn_ssd();
  if (!fn) return false;
  CUtensorMap map;
  cuuint64_t dims[2] = {(cuuint64_t)a.N, (cuuint64_t)a.C * a.H * a.P};
  cuuint64_t strides[1] = {(cuuint64_t)a.N * 4};
  cuuint32_t box[2] = {32, ROWS};
  cuuint32_t estr[2] = {1, 1};
  if (fn(&map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<float*>(a.h0), dims, strides, box, estr,
         CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
         CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return false;
  SsdTcArgs t;
  t.a = a;
  t.err = device_error_word();
  t.hpt = ROWS / a.P;
  t.n_tiles = a.H / t.hpt;
  t.n_items = a.C * t.n_tiles;
  const int sms = dev < 64 && n_sm[dev] > 0 ? n_sm[dev] : 148;
  const int grid = t.n_items < sms ? t.n_items : sms;
  launch_pdl(ssd_tc_kernel<TDT, NT, HK>, grid, THREADS, SsdTcLay<NT>::SMEM, s, map, t);
  note_launch();
  return true;
}

template <int NT, bool HK>
bool launch_ssd_tc_dt(const SsdArgs& a, cudaStream_t s) {
  return a.dt_bias ? launch_ssd_tc<bf16, NT, HK>(a, s) : launch_ssd_tc<float, NT, HK>(a, s);
}

}  // namespace

bool ssd_tc_supported(int dtype, const SsdArgs& a) {
  if (dtype != HSPEC_DTYPE_BF16 || !a.h0 || a.Q != a.K) return false;
  if (a.K < 1 || a.K > 32 || a.N != NMAX || a.C < 1) return false;
  if (a.P < ROWS / HPT_MAX || ROWS % a.P || a.H % (ROWS / a.P)) return false;
  if (((uintptr_t)a.h0 & 15) || (long)a.C * a.H * a.P > 0x7fffffffL) return false;
  if (((uintptr_t)a.B & 7) || ((uintptr_t)a.Cm & 7) || (a.bc_rs & 3)) return false;  // 8-byte loads
  if (a.hK && ((uintptr_t)a.hK & 15)) return false;  // float4 stores of the final state
  return true;
}

bool ssd_tc_launch(const SsdArgs& a, cudaStream_t s) {
  if (a.K <= 16) return a.hK ? launch_ssd_tc_dt<16, true>(a, s) : launch_ssd_tc_dt<16, false>(a, s);
  return a.hK ? launch_ssd_tc_dt<32, true>(a, s) : launch_ssd_tc_dt<32, false>(a, s);
}

}  // namespace hspec
