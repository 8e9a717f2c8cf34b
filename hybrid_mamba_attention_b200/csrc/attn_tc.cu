// Paged in-place GQA attention on the 5th-generation tensor cores (bf16, D = 64 or
// 128).  H-Spec (arXiv 2609.24197) Abstract: the drafter's attention modules reuse
// the target KVs in place -- here the K/V pages are streamed by TMA straight out of
// the target's pool through the page table, never copied to a drafter-side cache.
//
// Work units are (request, context split) pairs; a unit expands into one item per
// (row block, kv head g).  A one-CTA schedule kernel lists the units longest first
// (counting sort on the unit's tile count), so that the short units are the last
// ones taken and the SMs finish together.  The persistent kernel (one CTA per SM)
// takes items from an atomic counter, the heads of one unit adjacent so that
// concurrent CTAs read the same pages.  The R = K*G queries of kv head g (block
// position j, query head g*G + i) form the rows of a 128-row Q tile, so every K/V
// byte read from HBM feeds all R queries; with R <= 64 the rows are spread 16 per
// 32-lane TMEM quarter so that all four SM sub-partitions share the softmax work;
// rows without a query are zero.
// Warp roles (320 threads):
//   warp 0      producer: takes the next item, loads its Q tile (TMA) into one of
//               two Q buffers, reads page ids two tiles ahead, and streams its
//               64-token K/V tiles through a 4-stage ring -- per tile one 3-D TMA box
//               of 16 tokens x 64 dims of head g per page and column block (128-byte
//               swizzle), all boxes of a tile issued at once, one lane each -- and
//               writes the tile's description next to it.  The last context split
//               of a request also streams the block's own keys as one more tile.
//   warp 1      TMEM owner and single-thread MMA issuer, driven by readiness rather
//               than by a fixed order: it issues O_w += P_w . V_i (M=128, N=D, K=64)
//               as soon as the P of tile i is in shared memory, and S_b = Q . K_i^T
//               (M=128, N=64, K=D) into S buffer b = i % 4 as soon as tile i has
//               landed and softmax has read S_b's previous tile, so that the S of a
//               group's next tile is ready while it still works on the current one.
//   warps 2..5  softmax warpgroup 0 (tiles i even), warps 6..9 warpgroup 1 (i odd):
//               one TMEM lane (query row) per thread; mask, running max in the exp2
//               domain, P = exp2(s - m) to shared memory as bf16; O_w is rescaled in
//               TMEM only when the running max grows by more than 8.  Each group
//               keeps its own (m, l, O) per item and writes its own partial when its
//               last tile of the item is done -- the half of the split made of the
//               item's even (or odd) tiles, so the arithmetic does not depend on
//               scheduling; the merge kernel combines the halves and the splits.
// Every wait gives up after a time bound and sets the device error word.
#include <stdint.h>

#include "../../include/hspec.h"
#include "common.cuh"
#include "kernels.cuh"
#include "tc_prims.cuh"

namespace hspec {

int* device_error_word();

namespace {

constexpr int TT = kAttnTcTile;  // tokens per tile
constexpr int PPT = TT / 16;     // 16-token pages per tile
constexpr int NS = TT == 64 ? 5 : 10;   // K/V ring stages (160 KB)
constexpr int NSB = TT == 64 ? 4 : 8;   // S buffers in TMEM (half the columns)
constexpr int NPW = 4;           // producer warps
constexpr int THREADS = 32 * (NPW + 2 + 8);  // producers, 2 MMA warps, 2 softmax warpgroups
constexpr int ROWS = 128;     // MMA M
constexpr int kLenBuckets = 256;  // schedule: units sorted by tile count (capped)

struct TileMeta {  // written by the producer before the stage's barrier arrive
  int c, g, split, rb;
  int valid;       // keys in the tile
  int local;       // tile index within the item
  int n_tiles;     // tiles of the item
  int block;       // 1: the block's own keys
  int qslot, qseq; // Q buffer of the item and the item's use count of that buffer
  int end;         // 1: no more work
  int bt;          // block tiles: index among the block's tiles
};

template <int D>
struct Lay {
  static constexpr int DB = D / 64;                     // 64-element column blocks
  static constexpr int Q_BLK = ROWS * 128;              // 16 KB per Q column block
  static constexpr int Q_BYTES = DB * Q_BLK;
  static constexpr int KV_BLK = TT * 128;               // per K column block
  static constexpr int K_BYTES = DB * KV_BLK;           // K: [column block][TT tokens][128 B]
  static constexpr int V_PAGE = DB * 2048;              // V: [page][column block][16 tokens][128 B]
  static constexpr int STAGE = 2 * K_BYTES;             // K then V
  static constexpr int OFF_Q = 0;                       // two Q buffers
  static constexpr int OFF_KV = 2 * Q_BYTES;
  static constexpr int OFF_META = OFF_KV + NS * STAGE;
  static constexpr int OFF_BAR = OFF_META + 64 * NS;
  static constexpr int SMEM = OFF_BAR + 512 + 1024;
  // TMEM columns: S_b [TT b, TT b + TT) for b < NSB (P of the tile, bf16 packed,
  // overwrites its first TT / 2 columns), O_w [256 + 128w, 256 + 128w + D)
  static constexpr uint32_t TMEM_COLS = 512;
  __host__ __device__ static constexpr uint32_t S_COL(int b) { return (uint32_t)(b * TT); }
  __host__ __device__ static constexpr uint32_t O_COL(int w) { return (uint32_t)(256 + w * 128); }
};

struct TcMaps {
  CUtensorMap k, v, kb, vb, q;
};

// TMEM lane (0..127) -> query row of the row block: identity for R > 64; for
// R <= 64, 16 rows per 32-lane quarter (lanes 0..15 of each quarter), else -1.
__device__ __forceinline__ int row_of_lane(int lane128, bool spread) {
  if (!spread) return lane128;
  const int q = lane128 >> 5, l = lane128 & 31;
  return l < 16 ? q * 16 + l : -1;
}

// Tiles (TT-token context tiles, plus the block's own keys, nbt tiles, in a request's
// last split) of unit (ctx, split sp of n).
__host__ __device__ inline int unit_tiles(int ctx, int sp, int n, int split_tokens, int nbt) {
  const int b = sp * split_tokens, e = min(ctx, b + split_tokens);
  return (e > b ? (e - b + TT - 1) / TT : 0) + (sp == n - 1 ? nbt : 0);
}

// One CTA: lists the (request, split) units longest first into `units` and resets the
// work counter; sched[1] = number of units.  Requests with an invalid context length
// get no unit (their output rows are written as zeros by the merge).
__global__ void __launch_bounds__(1024) attn_sched_kernel(const int32_t* ctx_lens, int C, int split_tokens,
                                                          long max_ctx, int nbt, int* sched, int2* units,
                                                          int* err) {
  __shared__ int hist[kLenBuckets];
  for (int b = threadIdx.x; b < kLenBuckets; b += blockDim.x) hist[b] = 0;
  __syncthreads();
  for (int c = threadIdx.x; c < C; c += blockDim.x) {
    const int ctx = ctx_lens[c];
    if (ctx < 0 || ctx > max_ctx) {
      flag_error(err, kErrCtxOOB);
      continue;
    }
    const int n = ctx > 0 ? (ctx + split_tokens - 1) / split_tokens : 1;
    for (int sp = 0; sp < n; ++sp) atomicAdd(&hist[min(unit_tiles(ctx, sp, n, split_tokens, nbt), kLenBuckets - 1)], 1);
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    int run = 0;
    for (int b = kLenBuckets - 1; b >= 0; --b) {
      const int h = hist[b];
      hist[b] = run;
      run += h;
    }
    sched[0] = 0;
    sched[1] = run;
  }
  __syncthreads();
  for (int c = threadIdx.x; c < C; c += blockDim.x) {
    const int ctx = ctx_lens[c];
    if (ctx < 0 || ctx > max_ctx) continue;
    const int n = ctx > 0 ? (ctx + split_tokens - 1) / split_tokens : 1;
    for (int sp = 0; sp < n; ++sp) {
      const int pos = atomicAdd(&hist[min(unit_tiles(ctx, sp, n, split_tokens, nbt), kLenBuckets - 1)], 1);
      units[pos] = make_int2(c, sp);
    }
  }
}

template <int D>
__global__ void __launch_bounds__(THREADS, 1)
    attn_tc_kernel(const __grid_constant__ TcMaps maps, AttnArgs a, float scale_log2, int n_rb, int* sched,
                   const int2* units) {
  using L = Lay<D>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = tc::smem_u32(smem_raw);
  uint8_t* smem = smem_raw + (((raw + 1023) & ~1023u) - raw);
  uint8_t* sQ = smem + L::OFF_Q;
  uint8_t* sKV = smem + L::OFF_KV;
  volatile TileMeta* meta = (volatile TileMeta*)(smem + L::OFF_META);
  uint64_t* kv_full = (uint64_t*)(smem + L::OFF_BAR);  // one arrival per producer warp
  uint64_t* kv_empty = kv_full + NS;
  uint64_t* s_full = kv_empty + NS;   // [NSB] S_b written by Q.K^T
  uint64_t* s_free = s_full + NSB;    // [NSB] P.V of S_b's tile finished (S_b / P free)
  // P of S_b's tile written (one barrier per S buffer: a group's next tile may finish
  // its softmax before the MMA thread has taken this one, and the phases of one
  // barrier must not run two ahead of its waiter)
  uint64_t* p_full = s_free + NSB;    // [NSB]
  uint64_t* pv_done = p_full + NSB;   // [2]   group w's P.V finished (O_w quiescent)
  uint64_t* q_full = pv_done + 2;     // [2]
  uint64_t* q_empty = q_full + 2;     // [2]
  uint64_t* drain = q_empty + 2;      // [2] every MMA of an issuer (and its arrivals) finished
  uint32_t* tmem_slot = (uint32_t*)(drain + 2);
  volatile int* end_tile = (volatile int*)(tmem_slot + 1);
  volatile int* s_item = end_tile + 1;  // [2] next work item, published by producer warp 0
  volatile int* s_stop = s_item + 2;    // a producer warp gave up waiting

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int G = a.Hq / a.Hkv, R = a.K * G;
  const bool spread = R <= 64;
  int* err = a.err;
  constexpr int QK_WARP = NPW, PV_WARP = NPW + 1, SM_WARP0 = NPW + 2;

  if (threadIdx.x == 0) {
    for (int s = 0; s < NS; ++s) {
      tc::mbar_init(&kv_full[s], NPW);
      tc::mbar_init(&kv_empty[s], 1);
    }
    for (int b = 0; b < NSB; ++b) {
      tc::mbar_init(&s_full[b], 1);
      tc::mbar_init(&s_free[b], 1);
      tc::mbar_init(&p_full[b], 4);
    }
    for (int w = 0; w < 2; ++w) {
      tc::mbar_init(&pv_done[w], 1);
      tc::mbar_init(&q_full[w], 1);
      tc::mbar_init(&q_empty[w], 1);
    }
    tc::mbar_init(&drain[0], 1);
    tc::mbar_init(&drain[1], 1);
    *end_tile = 0x7fffffff;
    *s_stop = 0;
    tc::fence_mbar_init();
  }
  if (warp == QK_WARP) tc::tmem_alloc(tmem_slot, L::TMEM_COLS);
  // Q rows without a query are never written by TMA: zero both Q buffers once
  for (int e = threadIdx.x; e < 2 * L::Q_BYTES / 16; e += THREADS) ((uint4*)sQ)[e] = make_uint4(0, 0, 0, 0);
  tc::fence_proxy_async();
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp < NPW) {
    // ------------------------------------------------------------ producers
    // A tile's TMA boxes are spread over the NPW producer warps (the issue of one box
    // takes a warp tens of nanoseconds; in parallel the boxes keep up with HBM):
    // box bx < KB is K page bx / DB, column block bx % DB (16 tokens x 64 dims of head
    // g, 128-byte swizzle); box KB + q is V page q (one 4-D box, both column blocks).
    // Box bx is issued by lane bx / NPW of warp bx % NPW.  All producer warps walk the
    // same tiles; warp 0 takes the work items and loads the Q tiles.
    constexpr int KB = PPT * L::DB, NBX = KB + PPT;
    const int pw = warp;
    const int bx = pw + NPW * lane;
    const bool has_box = bx < NBX;
    const bool k_box = bx < KB;
    const int q16 = k_box ? bx / L::DB : bx - KB;  // page of the tile
    const int bk = k_box ? bx % L::DB : 0;
    if (threadIdx.x == 0) {
      tc::tma_prefetch_desc(&maps.k);
      tc::tma_prefetch_desc(&maps.v);
      tc::tma_prefetch_desc(&maps.kb);
      tc::tma_prefetch_desc(&maps.vb);
      tc::tma_prefetch_desc(&maps.q);
    }
    // Q boxes: with spread rows, one per 32-lane quarter holding 16 / G block positions
    // (16 rows); otherwise one holding 128 / G positions (128 rows)
    const int q_boxes = spread ? (R + 15) / 16 : 1;
    const int q_pos = spread ? 16 / G : ROWS / G;
    const int per_unit = a.Hkv * n_rb;
    const int n_items = sched[1] * per_unit;
    const int nbt = (a.K + TT - 1) / TT;  // tiles of the block's own keys
    const int pshift = (a.page_size & (a.page_size - 1)) == 0 ? __ffs(a.page_size) - 1 : -1;
    int tile_i = 0;
    bool ok = true;
    int it_next = threadIdx.x == 0 ? atomicAdd(sched, 1) : 0;  // the following item, in flight
    // Every producer warp passes the same item barriers: the loop ends only after one,
    // when the work is done or a producer has given up waiting.
    for (int seq = 0;; ++seq) {
      if (threadIdx.x == 0) s_item[seq & 1] = it_next;
      asm volatile("bar.sync 1, %0;" ::"n"(32 * NPW) : "memory");
      const int item = s_item[seq & 1];
      if (item >= n_items || *s_stop) break;
      if (threadIdx.x == 0) it_next = atomicAdd(sched, 1);  // prefetch: used by the next item
      const int u = item / per_unit, g = item % a.Hkv, rb = (item % per_unit) / a.Hkv;
      const int2 cu = units[u];
      const int c = cu.x, split = cu.y;
      const int ctx = a.ctx_lens[c];
      const int n_ctx_splits = ctx > 0 ? (ctx + a.split_tokens - 1) / a.split_tokens : 1;
      const int c_begin = split * a.split_tokens;
      const int c_end = min(ctx, c_begin + a.split_tokens);
      const int n_ctx_tiles = c_end > c_begin ? (c_end - c_begin + TT - 1) / TT : 0;
      const int n_tiles = n_ctx_tiles + (split == n_ctx_splits - 1 ? nbt : 0);
      const int slot = seq & 1;

      // Q tile of the item into Q buffer `slot` once the item two back is done with it
      if (pw == 0) {
        if (lane == 0) ok = tc::mbar_wait(&q_empty[slot], ((seq >> 1) & 1) ^ 1, err);
        ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
        if (ok) {
          uint8_t* qbuf = sQ + slot * L::Q_BYTES;
          if (lane == 0)
            tc::mbar_arrive_expect_tx(&q_full[slot], (uint32_t)(q_boxes * L::DB * q_pos * G * 128));
          __syncwarp();
          if (lane < q_boxes * L::DB) {
            const int qb = lane / L::DB, qk = lane % L::DB;
            const int pos0 = c * a.K + (spread ? qb * q_pos : rb * q_pos);
            tc::tma_load_3d(qbuf + qk * L::Q_BLK + qb * 32 * 128, &maps.q, &q_full[slot], qk * 64, g * G, pos0);
          }
          __syncwarp();
        }
      }

      // page id of this lane's page, read two tiles ahead into registers
      // (unconditionally, the index clamped into the request's row of the table, so
      // that nothing waits for it; ids past the split's end are never used)
      const int32_t* table = a.page_table + (size_t)c * a.max_pages;
      auto page_of = [&](int local) -> int {
        const int t = c_begin + local * TT + 16 * q16;
        const int idx = pshift >= 0 ? t >> pshift : t / a.page_size;
        return table[idx < a.max_pages ? idx : a.max_pages - 1];
      };
      int pid0 = page_of(0), pid1 = page_of(1);

      for (int local = 0; local < n_tiles && ok; ++local, ++tile_i) {
        const int pid = pid0;
        pid0 = pid1;
        pid1 = page_of(local + 2);
        const int s = tile_i % NS;
        if (lane == 0) ok = tc::mbar_wait(&kv_empty[s], ((tile_i / NS) & 1) ^ 1, err);
        ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
        if (!ok) break;
        uint8_t* kd = sKV + s * L::STAGE;
        uint8_t* vd = kd + L::K_BYTES;
        const bool block = local >= n_ctx_tiles;
        const int bt = local - n_ctx_tiles;  // block tiles: keys [bt TT, bt TT + TT) of the block
        const int t0 = c_begin + local * TT;
        const int valid = block ? min(TT, a.K - bt * TT) : min(TT, c_end - t0);
        const int groups = (valid + 15) / 16;  // 16-row boxes with keys
        if (pw == 0 && lane == 0) {
          volatile TileMeta& m = meta[s];
          m.c = c, m.g = g, m.split = split, m.rb = rb, m.valid = valid, m.local = local;
          m.n_tiles = n_tiles, m.block = block ? 1 : 0, m.qslot = slot, m.qseq = seq, m.end = 0;
          m.bt = block ? bt : 0;
        }
        // this lane's box: what it loads and how many bytes
        uint32_t bytes = 0;
        if (has_box && q16 < groups) {
          if (!block) bytes = k_box ? 2048u : (uint32_t)L::V_PAGE;
          else if (k_box ? q16 == 0 : true) bytes = k_box ? (uint32_t)(16 * 128) * PPT : (uint32_t)L::V_PAGE;
        }
        // block tiles: K of column block bk is one TT-row box (lanes with q16 == 0)
        const uint32_t warp_bytes = __reduce_add_sync(0xffffffffu, bytes);
        if (lane == 0) tc::mbar_arrive_expect_tx(&kv_full[s], warp_bytes);  // also this warp's arrival
        __syncwarp();
        if (bytes) {
          if (!block) {
            int pg = pid;
            if (pg < 0 || pg >= a.num_pages) {
              flag_error(err, kErrPageOOB);
              pg = 0;  // keep the copy in bounds; the request's output is flagged as invalid
            }
            const int tt = t0 + 16 * q16;
            const int z = pg * a.page_size + (pshift >= 0 ? (tt & (a.page_size - 1)) : tt % a.page_size);
            if (k_box)
              tc::tma_load_3d(kd + bk * L::KV_BLK + q16 * 2048, &maps.k, &kv_full[s], bk * 64, g, z);
            else
              tc::tma_load_4d(vd + q16 * L::V_PAGE, &maps.v, &kv_full[s], 0, z, g, 0);
          } else {
            const int row0 = c * a.K + bt * TT;
            if (k_box)
              tc::tma_load_3d(kd + bk * L::KV_BLK, &maps.kb, &kv_full[s], bk * 64, g, row0);
            else
              tc::tma_load_4d(vd + q16 * L::V_PAGE, &maps.vb, &kv_full[s], 0, row0 + 16 * q16, g, 0);
          }
        }
        __syncwarp();
      }
      if (!ok) *s_stop = 1;
    }
    // sentinel stage: no more work
    if (!*s_stop) {
      const int s = tile_i % NS;
      bool fine = true;
      if (lane == 0) fine = tc::mbar_wait(&kv_empty[s], ((tile_i / NS) & 1) ^ 1, err);
      if (lane == 0 && fine) {
        if (pw == 0) meta[s].end = 1;
        tc::mbar_arrive(&kv_full[s]);
      }
    }
  } else if (warp == QK_WARP) {
    if (lane == 0) {
      // ---------------------------------------------------------- Q.K^T issuer
      // S_b = Q . K_i^T into S buffer b = i % NSB once tile i has landed, S_b is free
      // (the P.V of tile i - NSB has read its P) and the item's Q is loaded.  Issuing
      // P.V from another thread keeps either kind of MMA from waiting behind the other.
      constexpr uint32_t idesc_qk = tc::idesc_bf16_f32(ROWS, TT);
      int q_seen[2] = {-1, -1};
      for (int qk = 0;; ++qk) {
        const int s = qk % NS, b = qk & (NSB - 1);
        if (qk >= NSB && !tc::mbar_wait(&s_free[b], ((qk / NSB) - 1) & 1, err)) break;
        if (!tc::mbar_wait(&kv_full[s], (qk / NS) & 1, err)) break;
        if (meta[s].end) {
          *end_tile = qk;
          break;
        }
        const int slot = meta[s].qslot, seq = meta[s].qseq;
        if (seq > q_seen[slot]) {
          if (!tc::mbar_wait(&q_full[slot], (seq >> 1) & 1, err)) break;
          q_seen[slot] = seq;
        }
        tc::tc_fence_after();
        const uint32_t q = tc::smem_u32(sQ + slot * L::Q_BYTES), k = tc::smem_u32(sKV + s * L::STAGE);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk)
          tc::mma_bf16(tmem + L::S_COL(b), tc::sdesc_k128(q + (kk / 4) * L::Q_BLK + (kk % 4) * 32),
                       tc::sdesc_k128(k + (kk / 4) * L::KV_BLK + (kk % 4) * 32), idesc_qk, kk > 0);
        tc::mma_commit(&s_full[b]);
        if (meta[s].local == meta[s].n_tiles - 1) tc::mma_commit(&q_empty[slot]);  // item's last QK
      }
      // no MMA or commit arrival may land after the CTA has finished
      tc::mma_commit(&drain[0]);
      tc::mbar_wait(&drain[0], 0, err);
    }
  } else if (warp == PV_WARP) {
    if (lane == 0) {
      // ---------------------------------------------------------- P.V issuer
      // O_w += P_i . V_i as soon as the P of tile i is in TMEM (group w = i % 2).  Tile
      // i's Q.K^T finished before its softmax began, so the commit after P.V frees the
      // whole stage.
      constexpr uint32_t idesc_pv = tc::idesc_bf16_f32(ROWS, D) | (1u << 16);  // B (= V) MN-major
      bool ok = true;
      int pv = 0;
      uint64_t idle_since = 0;
      while (pv < *end_tile) {
        // try_wait suspends the thread until the phase completes or a short time passes
        // (no busy polling against the softmax warps' issue slots), then end_tile is
        // checked again
        if (tc::mbar_try_wait(&p_full[pv & (NSB - 1)], (pv / NSB) & 1)) {
          tc::tc_fence_after();
          const int w = pv & 1, s = pv % NS;
          const bool first = meta[s].local < 2;  // this group's first tile of the item
          const uint32_t pt = tmem + L::S_COL(pv & (NSB - 1));  // P of the tile, in its S buffer
          const uint32_t v = tc::smem_u32(sKV + s * L::STAGE + L::K_BYTES);
          // K slice kk = the 16 keys of page kk: V [column block][16 tokens] blocks 2 KB apart
#pragma unroll
          for (int kk = 0; kk < PPT; ++kk)
            tc::mma_bf16_ts(tmem + L::O_COL(w), pt + kk * 8, tc::sdesc_mn128(v + kk * L::V_PAGE, 2048), idesc_pv,
                            (kk > 0 || !first) ? 1u : 0u);
          tc::mma_commit(&kv_empty[s]);
          tc::mma_commit(&pv_done[w]);
          tc::mma_commit(&s_free[pv & (NSB - 1)]);  // P read: S buffer free for tile pv + NSB
          ++pv;
          idle_since = 0;
        } else {
          const uint64_t t = tc::global_ns();
          if (idle_since == 0) {
            idle_since = t;
          } else if (t - idle_since > tc::kWaitLimitNs) {
            flag_error(err, tc::kErrTimeout);
            ok = false;
            break;
          }
        }
      }
      if (ok) {
        // wake both softmax groups: their next tiles are end_at and end_at + 1 (every
        // earlier tile's softmax is done, so those S buffers' earlier phases are complete)
        const int end_at = pv;
        *end_tile = end_at;  // (again, by this thread, before its arrivals release it)
        tc::mbar_arrive(&s_full[end_at & (NSB - 1)]);
        tc::mbar_arrive(&s_full[(end_at + 1) & (NSB - 1)]);
      }
      tc::mma_commit(&drain[1]);
      tc::mbar_wait(&drain[1], 0, err);
    }
  } else {
    // ------------------------------------------------------------ softmax warpgroups
    const int wg = (warp - SM_WARP0) >> 2;  // 0: first four softmax warps, 1: the next four
    const int quarter = warp & 3;           // TMEM lanes this warp may access
    const int lane128 = quarter * 32 + lane;
    const int r_local = row_of_lane(lane128, spread);
    const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
    const uint32_t tOw = tmem + lane_off + L::O_COL(wg);
    const int gthread = (warp - SM_WARP0 - 4 * wg) * 32 + lane;  // 0..127 within the group

    float m_used = -INFINITY, l = 0.f;
    bool ok = true;
    for (int i = wg; ok; i += 2) {
      const int n = i >> 1;                 // this group's tile count so far
      const int b = i & (NSB - 1);
      ok = __all_sync(0xffffffffu, tc::mbar_wait(&s_full[b], (i / NSB) & 1, err));
      if (!ok || i >= *end_tile) break;
      tc::tc_fence_after();
      const int s = i % NS;
      // acquire the producer's description of the tile (this phase completed long ago;
      // the stage cannot move on before this group's P.V of the tile)
      ok = __all_sync(0xffffffffu, tc::mbar_wait(&kv_full[s], (i / NS) & 1, err));
      if (!ok) break;
      const int c = meta[s].c, g = meta[s].g, split = meta[s].split, rb = meta[s].rb;
      const int local = meta[s].local, n_tiles = meta[s].n_tiles, valid = meta[s].valid;
      const bool block_tile = meta[s].block != 0;
      const int bt = meta[s].bt;
      const int gr = rb * ROWS + (r_local < 0 ? 0 : r_local);
      const bool active = r_local >= 0 && gr < R;
      const int jq = active ? gr / G : 0;
      if (local < 2) {  // this group's first tile of a new item
        m_used = -INFINITY;
        l = 0.f;
      }
      float sv[TT];
      tc::tmem_ld(tmem + lane_off + L::S_COL(b), sv);
      // raw scores; the scale (> 0) is applied inside the exponent below
      float mx = -INFINITY;
      if (valid == TT && !(block_tile && a.causal_block)) {
#pragma unroll
        for (int j = 0; j < TT; ++j) mx = fmaxf(mx, sv[j]);
      } else {
        // causal block: query position jq sees the block keys 0..jq
        const int vis_end = (block_tile && a.causal_block) ? min(valid, jq + 1 - bt * TT) : valid;
#pragma unroll
        for (int j = 0; j < TT; ++j) {
          sv[j] = j < vis_end ? sv[j] : -INFINITY;
          mx = fmaxf(mx, sv[j]);
        }
      }
      const float m_new = fmaxf(m_used, mx * scale_log2);  // running max in the exp2 domain
      float alpha = 1.f;
      bool rescale = false;
      if (m_new > m_used + 8.f) {
        if (local >= 2 && m_used != -INFINITY) {
          alpha = exp2f(m_used - m_new);
          rescale = true;
          l *= alpha;
        }
        m_used = m_new;
      }
      // with no visible key yet (m = -inf) every s is -inf: subtract 0 so p = 0, not NaN
      const float mu = m_used == -INFINITY ? 0.f : m_used;
      float2 psum = make_float2(0.f, 0.f);
      uint32_t pk[TT / 2];
      const float2 sc2 = make_float2(scale_log2, scale_log2), nm2 = make_float2(-mu, -mu);
#pragma unroll
      for (int j = 0; j < TT; j += 2) {
        // p = 2^(s scale - m): the exponents of a pair in one packed FFMA, then one ex2
        // each (flushing results below 2^-126 to zero); 2^(-inf) = 0 for masked columns
        const float2 e = tc::ffma2(make_float2(sv[j], sv[j + 1]), sc2, nm2);
        const float2 pp = make_float2(tc::ex2_ftz(e.x), tc::ex2_ftz(e.y));
        psum = tc::fadd2(psum, pp);
        __nv_bfloat162 h2 = __floats2bfloat162_rn(pp.x, pp.y);
        pk[j / 2] = *reinterpret_cast<uint32_t*>(&h2);
      }
      l += psum.x + psum.y;
      // P over the first half of S_b
      tc::tmem_stu(tmem + lane_off + L::S_COL(b), pk);
      // The group's previous P.V (before O_w may be rescaled).  It is waited for at
      // every tile, not only before a rescale: softmax may run several tiles ahead of
      // the P.V's, and a parity wait is only unambiguous while its waiter is at most
      // one phase behind the barrier.
      if (n >= 1) {
        ok = __all_sync(0xffffffffu, tc::mbar_wait(&pv_done[wg], (n - 1) & 1, err));
        if (!ok) break;
        tc::tc_fence_after();
      }
      if (__any_sync(0xffffffffu, rescale)) {
        // O_w holds this group's earlier tiles of the item
#pragma unroll
        for (int cb = 0; cb < D / 32; ++cb) {
          float v[32];
          tc::tmem_ld32(tOw + cb * 32, v);
#pragma unroll
          for (int e = 0; e < 32; ++e) v[e] *= alpha;
          tc::tmem_st32(tOw + cb * 32, v);
        }
      }
      if (valid < TT) {
        // V rows past the last valid token may hold stale data: zero them (P is 0 there)
        uint8_t* vbase = sKV + s * L::STAGE + L::K_BYTES;
        const int n_chunks = (TT - valid) * L::DB * 8;
        for (int e = gthread; e < n_chunks; e += 128) {
          const int r2 = valid + e / (L::DB * 8), rest = e % (L::DB * 8);
          const int ck = rest / 8, cc = rest % 8, rr = r2 & 15;
          *(uint4*)(vbase + (r2 >> 4) * L::V_PAGE + ck * 2048 + rr * 128 + ((cc ^ (rr & 7)) << 4)) =
              make_uint4(0, 0, 0, 0);
        }
        tc::fence_proxy_async();
      }
      tc::tc_fence_before();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(&p_full[b]);

      if (local >= n_tiles - 2) {
        // this group's last tile of the item: write its partial (half of the split)
        ok = __all_sync(0xffffffffu, tc::mbar_wait(&pv_done[wg], n & 1, err));
        if (!ok) break;
        tc::tc_fence_after();
        // half (local & 1): the item's even or odd tiles, whichever group ran them,
        // so the result does not depend on how items were scheduled
        const size_t base = ((((size_t)c * a.Hkv + g) * a.n_splits + split) * 2 + (local & 1)) * R + gr;
#pragma unroll
        for (int cb = 0; cb < D / 32; ++cb) {
          float v[32];
          tc::tmem_ld32(tOw + cb * 32, v);
          if (active) {
            float* o = a.ws_acc + base * D + cb * 32;
#pragma unroll
            for (int e = 0; e < 32; e += 4) *(float4*)(o + e) = make_float4(v[e], v[e + 1], v[e + 2], v[e + 3]);
          }
        }
        if (active) {
          a.ws_ml[base * 2] = m_used;
          a.ws_ml[base * 2 + 1] = l;
        }
        tc::tc_fence_before();
      }
    }
  }
  __syncthreads();
  if (warp == QK_WARP) {
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

// 4-D map of [rows][Hkv][D] seen as (x = 64 elements, y = token row, z = kv head,
// w = 64-element column block, 128 B apart) with box 64 x 16 x 1 x D/64: one box
// holds 16 token rows of one head in both column blocks, stored [column block][row].
bool make_kv_map4(CUtensorMap* m, const void* base, long rows, int Hkv, int D, long row_stride_elems) {
  EncodeTiledFn fn = encode_fn_attn();
  if (!fn) return false;
  cuuint64_t dims[4] = {64, (cuuint64_t)rows, (cuuint64_t)Hkv, (cuuint64_t)(D / 64)};
  cuuint64_t strides[3] = {(cuuint64_t)row_stride_elems * 2, (cuuint64_t)D * 2, 128};
  cuuint32_t box[4] = {64, 16, 1, (cuuint32_t)(D / 64)};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 3-D map of q [positions][Hq][D] with box 64 x G x pos_rows, 128-byte swizzle.
bool make_q_map(CUtensorMap* m, const void* base, long positions, int Hq, int D, long row_stride_elems, int G,
                int pos_rows) {
  EncodeTiledFn fn = encode_fn_attn();
  if (!fn) return false;
  cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)Hq, (cuuint64_t)positions};
  cuuint64_t strides[2] = {(cuuint64_t)D * 2, (cuuint64_t)row_stride_elems * 2};
  cuuint32_t box[3] = {64, (cuuint32_t)G, (cuuint32_t)pos_rows};
  cuuint32_t estr[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int D>
bool launch_tc(const AttnArgs& a, cudaStream_t s) {
  static bool attr_set[64] = {};
  static int n_sm[64] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 64 && !attr_set[dev]) {
    if (cudaFuncSetAttribute(attn_tc_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, Lay<D>::SMEM) !=
        cudaSuccess) {
      set_error("cudaFuncSetAttribute(attn_tc_kernel) failed");
      return false;
    }
    cudaDeviceGetAttribute(&n_sm[dev], cudaDevAttrMultiProcessorCount, dev);
    attr_set[dev] = true;
  }
  TcMaps maps;
  const long pool_rows = (long)a.num_pages * a.page_size;
  bool ok = make_kv_map(&maps.k, a.k_pool, pool_rows, a.Hkv, D, (long)a.Hkv * D, 16) &&
            make_kv_map4(&maps.v, a.v_pool, pool_rows, a.Hkv, D, (long)a.Hkv * D) &&
            make_kv_map(&maps.kb, a.kb, (long)a.C * a.K, a.Hkv, D, a.kb_rs, TT) &&
            make_kv_map4(&maps.vb, a.vb, (long)a.C * a.K, a.Hkv, D, a.vb_rs);
  // Q as [C*K positions][Hq heads][D]: a box holds G heads x (16 / G or 128 / G) positions
  const int G = a.Hq / a.Hkv;
  const int Rq = a.K * G;
  ok = ok && make_q_map(&maps.q, a.q, (long)a.C * a.K, a.Hq, D, a.q_rs, G, Rq <= 64 ? 16 / G : ROWS / G);
  if (!ok) {
    set_error("cuTensorMapEncodeTiled failed for the attention K/V maps");
    return false;
  }
  const int R = a.K * (a.Hq / a.Hkv);
  const int n_rb = (R + ROWS - 1) / ROWS;
  if (a.sub_splits != 2) {
    set_error("tensor-core attention writes two partials per split");
    return false;
  }
  // after the partials: the work counter and unit count (256 bytes), then the unit list
  const size_t pairs = (size_t)a.C * a.Hkv * a.n_splits * 2 * R;
  int* sched = (int*)(a.ws_ml + pairs * 2);
  int2* units = (int2*)(sched + 64);
  attn_sched_kernel<<<1, 1024, 0, s>>>(a.ctx_lens, a.C, a.split_tokens, (long)a.max_pages * a.page_size,
                                       (a.K + TT - 1) / TT, sched, units, a.err);
  note_launch();
  const long max_items = (long)a.C * a.n_splits * n_rb * a.Hkv;
  const int sms = dev < 64 && n_sm[dev] > 0 ? n_sm[dev] : 148;
  const int grid = max_items < sms ? (int)max_items : sms;
  const float scale_log2 = 1.4426950408889634f / sqrtf((float)D);
  attn_tc_kernel<D><<<grid, THREADS, Lay<D>::SMEM, s>>>(maps, a, scale_log2, n_rb, sched, units);
  note_launch();
  return true;
}

}  // namespace

bool attn_tc_supported(const AttnArgs& a, const char** why) {
  if (a.D != 64 && a.D != 128) return *why = "head_dim must be 64 or 128", false;
  if (a.page_size % 16) return *why = "page_size must be a multiple of 16", false;
  if (a.K > 64) return *why = "K must be <= 64", false;
  const int G = a.Hq / a.Hkv;
  if (G > 16 || (G & (G - 1))) return *why = "the GQA group Hq/Hkv must be a power of two <= 16", false;
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
