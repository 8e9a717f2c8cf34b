// Paged in-place GQA attention on the 5th-generation tensor cores (bf16, D = 64 or
// 128).  H-Spec (arXiv 2609.24197) Abstract: the drafter's attention modules reuse
// the target KVs in place -- here the K/V pages are streamed by TMA straight out of
// the target's pool through the page table, never copied to a drafter-side cache.
//
// Work partition (stream-K over the tile space): each (request c, row block rb, kv
// head g) is a sequence of t_c 64-token tiles (the context's, then the block's own
// keys).  On a line of work units the sequences are laid end to end, request by
// request, each as kAttnSeqUnits units for its start (a piece's Q load, the page ids of
// its first tiles and its partials cost about as much as five or six tiles) followed by
// one unit per tile.  A one-CTA schedule kernel sums them (T units) and cuts the line into
// chunks of Z = ceil(T / grid) units, one per CTA of the persistent kernel (or of a
// requested length, CTA b then taking chunks b, b + grid, ...), so that every SM gets
// the same work whatever the mix of context lengths: with tiles alone a CTA whose
// chunk crossed many short sequences finished up to 20% after the others.  A CTA
// walks its chunk as pieces, one per sequence whose tiles it crosses; the piece of
// sequence q in chunk k writes its partial to slot q + k (distinct for every piece: a
// later sequence never starts in an earlier chunk), and the merge kernel finds the
// pieces of a sequence from T, Z and the request's offset on the line.
// The R = K*G queries of kv head g (block position j, query head g*G + i) form the rows
// of a 128-row Q tile, so every K/V byte read from HBM feeds all R queries; with R <= 64
// the rows are spread 16 per 32-lane TMEM quarter so that all four SM sub-partitions
// share the softmax work; rows without a query are zero.
// Warp roles (480 threads, one CTA per SM):
//   warps 0..3  producers: all four walk the CTA's pieces.  Warp 0 loads each piece's
//               Q tile (TMA) into one of two Q buffers.  Page ids are read two tiles
//               ahead.  The 64-token K/V tiles stream through a ring of 6 stages (5 for
//               M = 128) -- per tile one 3-D K box per page and 64-dim column block
//               (16 tokens x 64 dims of head g, 128-byte swizzle) and one 4-D V box per
//               page (both column blocks), box x issued by warp x % 4, all boxes of a
//               tile at once, with an L2 evict-first policy (read once) -- and warp 0
//               writes the tile's description next to it.
//               A sequence's last tiles are the block's own keys (one more tile for
//               K <= 64).
//   warps 4, 14 Q.K^T issuers (warp 4 also owns TMEM): S_b = Q . K_i^T (N = 64, K = D)
//               into S buffer b = i % 4 as soon as tile i has landed and the P.V of
//               tile i - 4 has read S_b, so that the S of a group's next tile is ready
//               while the group still works on the current one.  Warp 4 takes the even
//               tiles, warp 14 the odd ones (one per softmax group): two chains of
//               dependent MMAs in flight instead of one.
//   warp 5      P.V issuer: O_w += P_i . V_i (N = D, K = 64) as soon as the P of tile
//               i is in TMEM, with P (the A operand) read from TMEM, as two products
//               (its bf16 high and low parts); its commit frees the K/V stage and the S
//               buffer, and at a piece's last tile it frees the piece's Q buffer (every
//               Q.K^T of the piece finished before that tile's softmax began).
//   warps 6..9  softmax warpgroup 0 (tiles i even), warps 10..13 warpgroup 1 (i odd):
//               one query row per thread (M = 64: two threads per row, one in each
//               half-warp, 32 scores each); mask, running max in the exp2 domain,
//               P = exp2(s - m) written back over S as bf16 hi = bf16(P) and lo =
//               bf16(P - hi), which carry P to about 16 bits; O_w is rescaled in
//               TMEM only when the running max grows by more than 8, after the group's
//               previous P.V.
//               Each group keeps its own (m, l, O) per piece and writes its own partial
//               -- the half of the piece made of its even (or odd) tiles, so the
//               arithmetic does not depend on timing -- while it works on its next tile:
//               after that tile's softmax and before its P.V may overwrite O_w, so that
//               the wait for the piece's last P.V (queued behind the Q.K^T products of
//               the tiles ahead) overlaps useful work.  The merge kernel combines the
//               halves and the pieces.
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
constexpr int NSB = TT == 64 ? 4 : 8;   // S buffers in TMEM (half the columns)
constexpr int NPW = 4;           // producer warps
constexpr int THREADS = 32 * (NPW + 3 + 8);  // producers, 3 MMA warps, 2 softmax warpgroups
constexpr int ROWS = 128;     // MMA M

struct TileMeta {  // written by the producer before the stage's barrier arrive
  int c, g, slot, rb;  // slot: the partial slot of the piece
  int valid;       // keys in the tile
  int local;       // tile index within the piece
  int n_tiles;     // tiles of the piece
  int block;       // 1: the block's own keys
  int qslot, qseq; // Q buffer of the piece and the piece's use count of that buffer
  int end;         // 1: no more work
  int bt;          // block tiles: index among the block's tiles
  int end_at;      // sentinel stages: the first tile index past the work
};

// SP: the R <= 64 queries of a kv head in an M = 64 tile (rows 16 per TMEM lane
// quarter, lanes 0..15); else an M = 128 tile.  The 64-row Q buffers leave room for a
// sixth K/V stage.
template <int D, bool SP>
struct Lay {
  static constexpr int MR = SP ? 64 : ROWS;             // MMA M (rows of the Q tile)
  static constexpr int NS = SP ? 6 : 5;                 // K/V ring stages (TT = 64)
  static constexpr int DB = D / 64;                     // 64-element column blocks
  static constexpr int Q_BLK = MR * 128;                // per Q column block
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
  // TMEM columns: S_b [TT b, TT b + TT) for b < NSB (P of the tile as bf16 pairs
  // overwrites it: hi = bf16(p) in its first TT / 2 columns, lo = bf16(p - hi) in the
  // rest), O_w [256 + 128w, 256 + 128w + D)
  static constexpr uint32_t TMEM_COLS = 512;
  __host__ __device__ static constexpr uint32_t S_COL(int b) { return (uint32_t)(b * TT); }
  __host__ __device__ static constexpr uint32_t O_COL(int w) { return (uint32_t)(256 + w * 128); }
};

struct TcMaps {
  CUtensorMap k, v, kb, vb, q;
};

// Units of each sequence of a request on the partition's line: kAttnSeqUnits for its
// start, then one per tile -- its context tiles and the block's own keys (nbt tiles);
// none for an invalid context length (the merge writes zero rows).
__device__ __forceinline__ int seq_units(int ctx, long max_ctx, int nbt) {
  return ctx < 0 || ctx > max_ctx ? 0 : kAttnSeqUnits + (ctx + TT - 1) / TT + nbt;
}

// One CTA: off[c] = units of all sequences of requests before c (spr sequences of
// seq_units each per request), off[C] = T; sched[1] = T, sched[2] = Z (the chunk
// length in units: ceil(T / grid), or z_req; at least ceil(T / max_chunks)),
// sched[3] = the number of chunks.
__global__ void __launch_bounds__(1024) attn_sched_kernel(const int32_t* ctx_lens, int C, long max_ctx, int nbt,
                                                          int spr, int grid, int z_req, int max_chunks, int* sched,
                                                          int* off, int* err) {
  pdl_wait();  // the previous kernel on the stream is complete from here on
  pdl_trigger();
  __shared__ int part[1024];
  const int per = (C + 1023) / 1024;
  const int c0 = min(C, (int)threadIdx.x * per), c1 = min(C, c0 + per);
  int sum = 0;
  for (int c = c0; c < c1; ++c) {
    const int ctx = ctx_lens[c];
    if (ctx < 0 || ctx > max_ctx) flag_error(err, kErrCtxOOB);
    sum += seq_units(ctx, max_ctx, nbt) * spr;
  }
  part[threadIdx.x] = sum;
  __syncthreads();
  for (int o = 1; o < 1024; o <<= 1) {  // inclusive scan of the per-thread sums
    const int v = threadIdx.x >= (unsigned)o ? part[threadIdx.x - o] : 0;
    __syncthreads();
    part[threadIdx.x] += v;
    __syncthreads();
  }
  int run = threadIdx.x > 0 ? part[threadIdx.x - 1] : 0;
  for (int c = c0; c < c1; ++c) {
    off[c] = run;
    run += seq_units(ctx_lens[c], max_ctx, nbt) * spr;
  }
  if (threadIdx.x == 1023) {
    const int T = part[1023];
    int Z = z_req > 0 ? z_req : (T + grid - 1) / grid;
    Z = max(max(Z, (T + max_chunks - 1) / max_chunks), 1);
    off[C] = T;
    sched[1] = T;
    sched[2] = Z;
    sched[3] = (T + Z - 1) / Z;
  }
}

template <int D, bool SP>
__global__ void __launch_bounds__(THREADS, 1)
    attn_tc_kernel(const __grid_constant__ TcMaps maps, AttnArgs a, float scale_log2, int n_rb) {
  using L = Lay<D, SP>;
  constexpr int NS = L::NS;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = tc::smem_u32(smem_raw);
  uint8_t* smem = smem_raw + (((raw + 1023) & ~1023u) - raw);
  uint8_t* sQ = smem + L::OFF_Q;
  uint8_t* sKV = smem + L::OFF_KV;
  volatile TileMeta* meta = (volatile TileMeta*)(smem + L::OFF_META);
  uint64_t* kv_full = (uint64_t*)(smem + L::OFF_BAR);  // one arrival per producer warp
  uint64_t* kv_empty = kv_full + NS;
  uint64_t* s_full = kv_empty + NS;   // [NSB] S_b written by Q.K^T
  uint64_t* s_free = s_full + NSB;    // [NSB] P.V of S_b's tile finished (S_b / P free, O_w
                                      // holds that tile)
  // P of S_b's tile written (one barrier per S buffer: a group's next tile may finish
  // its softmax before the MMA thread has taken this one, and the phases of one
  // barrier must not run two ahead of its waiter)
  uint64_t* p_full = s_free + NSB;    // [NSB]
  uint64_t* q_full = p_full + NSB;    // [2]
  uint64_t* q_empty = q_full + 2;     // [2]
  uint64_t* drain = q_empty + 2;      // [3] every MMA of an issuer (and its arrivals) finished
  uint32_t* tmem_slot = (uint32_t*)(drain + 3);
  volatile int* end_tile = (volatile int*)(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int G = a.Hq / a.Hkv, R = a.K * G;
  const int RB = R < ROWS ? R : ROWS;  // rows of a row block's partial
  constexpr bool spread = SP;
  int* err = a.err;
  const uint64_t lim = a.wait_ns ? (uint64_t)a.wait_ns : tc::kWaitLimitNs;  // pipeline waits
  // Q.K^T issuers: QK_WARP for the even tiles (and the TMEM owner), QK_WARP2 for the odd
  constexpr int QK_WARP = NPW, PV_WARP = NPW + 1, SM_WARP0 = NPW + 2, QK_WARP2 = NPW + 2 + 8;

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
      tc::mbar_init(&q_full[w], 1);
      tc::mbar_init(&q_empty[w], 1);
    }
    tc::mbar_init(&drain[0], 1);
    tc::mbar_init(&drain[1], 1);
    tc::mbar_init(&drain[2], 1);
    *end_tile = 0x7fffffff;
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
  pdl_wait();  // the previous kernel on the stream is complete from here on
  pdl_trigger();

  if (warp < NPW) {
    // ------------------------------------------------------------ producers
    // A tile's TMA boxes are spread over the NPW producer warps (the issue of one box
    // takes a warp tens of nanoseconds; in parallel the boxes keep up with HBM):
    // box bx < KB is K page bx / DB, column block bx % DB (16 tokens x 64 dims of head
    // g, 128-byte swizzle); box KB + q is V page q (one 4-D box, both column blocks).
    // Box bx is issued by lane bx / NPW of warp bx % NPW.  All producer warps walk the
    // same tiles; warp 0 loads the Q tiles.
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
    const int spr = a.Hkv * n_rb;         // sequences per request
    const int pshift = (a.page_size & (a.page_size - 1)) == 0 ? __ffs(a.page_size) - 1 : -1;
    const int T = a.sched[1], Z = a.sched[2], n_chunks = a.sched[3];
    const int* off = a.sched + 64;
    // the request holding tile p of the line: the last c with off[c] <= p
    auto locate = [&](int p) -> int {
      int lo = 0, hi = a.C - 1;
      while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (off[mid] <= p) lo = mid;
        else hi = mid - 1;
      }
      return lo;
    };
    // the K/V tiles are read once: first out of L2, so that the pieces' partials stay
    // there until the end of the kernel reads them back
    const uint64_t once = tc::l2_evict_first();
    int k = blockIdx.x;  // this CTA's chunk
    int pos = k < n_chunks ? k * Z : 0, end = k < n_chunks ? min(T, pos + Z) : 0;
    int c = pos < end ? locate(pos) : 0;
    int tile_i = 0;   // K/V tiles this warp has armed (its arrival on their stage)
    int q_last = -1;  // warp 0: the last piece whose Q load it armed
    bool ok = true;
    // Every producer warp walks the same pieces and passes the same barriers: the loop
    // ends only at one, when the work is done or a producer has given up waiting (the
    // barrier ORs the warps' `ok`, so all of them take the same decision).
    bool stopped = false;
    for (int seq = 0;; ++seq) {
      if (tc::bar_or<1, 32 * NPW>(!ok)) {
        stopped = true;
        break;
      }
      // the next piece: tiles [lt0, lt0 + n_tiles) of sequence r = rb Hkv + g of
      // request c within the chunk (a span that holds only a sequence's start units
      // has no tiles and is passed over without a piece)
      int r = 0, lt0 = 0, n_tiles = 0;
      bool done = false;
      while (n_tiles == 0) {
        if (pos >= end) {  // the CTA's next chunk
          k += gridDim.x;
          if (k >= n_chunks) {
            done = true;
            break;
          }
          pos = k * Z;
          end = min(T, pos + Z);
          c = locate(pos);
        }
        while (off[c + 1] <= pos) ++c;
        // units [u0, u1) of the sequence: kAttnSeqUnits start units, then its tiles
        const int tw = (off[c + 1] - off[c]) / spr;
        const int rel = pos - off[c];
        r = rel / tw;
        const int u0 = rel - r * tw, u1 = min(tw, u0 + (end - pos));
        pos += u1 - u0;
        lt0 = max(u0 - kAttnSeqUnits, 0);
        n_tiles = max(u1 - kAttnSeqUnits - lt0, 0);
      }
      if (done) break;
      const int g = r % a.Hkv, rb = r / a.Hkv;
      const int pslot = c * spr + r + k;  // partial slot of the piece
      const int ctx = a.ctx_lens[c];
      const int ct = (ctx + TT - 1) / TT;  // context tiles of the sequence
      const int slot = seq & 1;

      // Q tile of the piece into Q buffer `slot` once the piece two back is done with it
      if (pw == 0) {
        if (lane == 0) ok = tc::mbar_wait(&q_empty[slot], ((seq >> 1) & 1) ^ 1, err, lim);
        ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
        if (ok) {
          uint8_t* qbuf = sQ + slot * L::Q_BYTES;
          q_last = seq;
          if (lane == 0)
            tc::mbar_arrive_expect_tx(&q_full[slot], (uint32_t)(q_boxes * L::DB * q_pos * G * 128));
          __syncwarp();
          if (lane < q_boxes * L::DB) {
            const int qb = lane / L::DB, qk = lane % L::DB;
            const int pos0 = c * a.K + (spread ? qb * q_pos : rb * q_pos);
            tc::tma_load_3d(qbuf + qk * L::Q_BLK + qb * 16 * 128, &maps.q, &q_full[slot], qk * 64, g * G, pos0);
          }
          __syncwarp();
        }
      }

      // page id of this lane's page, read two tiles ahead into registers
      // (unconditionally, the index clamped into the request's row of the table, so
      // that nothing waits for it; ids past the context's end are never used)
      const int32_t* table = a.page_table + (size_t)c * a.max_pages;
      auto page_of = [&](int local) -> int {
        const int t = (lt0 + local) * TT + 16 * q16;
        const int idx = pshift >= 0 ? t >> pshift : t / a.page_size;
        return table[idx < a.max_pages ? idx : a.max_pages - 1];
      };
      int pid0 = page_of(0), pid1 = page_of(1);

      for (int local = 0; local < n_tiles && ok; ++local, ++tile_i) {
        const int pid = pid0;
        pid0 = pid1;
        pid1 = page_of(local + 2);
        const int s = tile_i % NS;
        if (lane == 0) ok = tc::mbar_wait(&kv_empty[s], ((tile_i / NS) & 1) ^ 1, err, lim);
        ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
        if (!ok) break;
        uint8_t* kd = sKV + s * L::STAGE;
        uint8_t* vd = kd + L::K_BYTES;
        const int st = lt0 + local;  // tile of the sequence
        const bool block = st >= ct;
        const int bt = st - ct;      // block tiles: keys [bt TT, bt TT + TT) of the block
        const int t0 = st * TT;
        const int valid = block ? min(TT, a.K - bt * TT) : min(TT, ctx - t0);
        const int groups = (valid + 15) / 16;  // 16-row boxes with keys
        if (pw == 0 && lane == 0) {
          volatile TileMeta& m = meta[s];
          m.c = c, m.g = g, m.slot = pslot, m.rb = rb, m.valid = valid, m.local = local;
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
              tc::tma_load_3d_hint(kd + bk * L::KV_BLK + q16 * 2048, &maps.k, &kv_full[s], bk * 64, g, z, once);
            else
              tc::tma_load_4d_hint(vd + q16 * L::V_PAGE, &maps.v, &kv_full[s], 0, z, g, 0, once);
          } else {
            const int row0 = c * a.K + bt * TT;
            if (k_box)
              tc::tma_load_3d_hint(kd + bk * L::KV_BLK, &maps.kb, &kv_full[s], bk * 64, g, row0, once);
            else
              tc::tma_load_4d_hint(vd + q16 * L::V_PAGE, &maps.vb, &kv_full[s], 0, row0 + 16 * q16, g, 0, once);
          }
        }
        __syncwarp();
      }
    }
    // No copy may land after the CTA has finished: wait, with the full limit, for the
    // last filling of every stage this warp armed (complete once the copies of all four
    // warps have landed, whatever the consumers do; unless a wait gave up it is complete
    // already), and warp 0 for its last two Q loads.  This comes before the sentinel
    // below, which completes the next phase of one of these stages: a parity wait is
    // unambiguous only while the barrier is at most one phase past it.
    if (lane == 0) {
      for (int j = tile_i > NS ? tile_i - NS : 0; j < tile_i; ++j)
        tc::mbar_wait(&kv_full[j % NS], (j / NS) & 1, err);
      for (int q = q_last > 0 ? q_last - 1 : 0; q <= q_last; ++q) tc::mbar_wait(&q_full[q & 1], (q >> 1) & 1, err);
    }
    __syncwarp();
    // sentinel stages: no more work (two, one for each Q.K^T issuer)
    if (!stopped) {
      const int end_at = tile_i;
      for (int e = 0; e < 2; ++e) {
        const int ti = end_at + e, s = ti % NS;
        bool fine = true;
        if (lane == 0) fine = tc::mbar_wait(&kv_empty[s], ((ti / NS) & 1) ^ 1, err, lim);
        fine = __shfl_sync(0xffffffffu, fine ? 1 : 0, 0) != 0;
        if (!fine) break;
        if (lane == 0) {
          if (pw == 0) meta[s].end = 1, meta[s].end_at = end_at;
          tc::mbar_arrive(&kv_full[s]);
        }
      }
    }
  } else if (warp == QK_WARP || warp == QK_WARP2) {
    if (lane == 0) {
      const int qw = warp == QK_WARP2 ? 1 : 0;
      // ---------------------------------------------------------- Q.K^T issuer
      // S_b = Q . K_i^T into S buffer b = i % NSB once tile i has landed, S_b is free
      // (the P.V of tile i - NSB has read its P) and the piece's Q is loaded.  Issuing
      // P.V from another thread keeps either kind of MMA from waiting behind the other.
      constexpr uint32_t idesc_qk = tc::idesc_bf16_f32(L::MR, TT);
      int q_seen[2] = {-1, -1};
      for (int qk = qw;; qk += 2) {
        const int s = qk % NS, b = qk & (NSB - 1);
        if (qk >= NSB && !tc::mbar_wait(&s_free[b], ((qk / NSB) - 1) & 1, err, lim)) break;
        if (!tc::mbar_wait(&kv_full[s], (qk / NS) & 1, err, lim)) break;
        if (meta[s].end) {
          *end_tile = meta[s].end_at;
          break;
        }
        const int slot = meta[s].qslot, seq = meta[s].qseq;
        if (seq > q_seen[slot]) {
          if (!tc::mbar_wait(&q_full[slot], (seq >> 1) & 1, err, lim)) break;
          q_seen[slot] = seq;
        }
        tc::tc_fence_after();
        const uint32_t q = tc::smem_u32(sQ + slot * L::Q_BYTES), k = tc::smem_u32(sKV + s * L::STAGE);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk)
          tc::mma_bf16(tmem + L::S_COL(b), tc::sdesc_k128(q + (kk / 4) * L::Q_BLK + (kk % 4) * 32),
                       tc::sdesc_k128(k + (kk / 4) * L::KV_BLK + (kk % 4) * 32), idesc_qk, kk > 0);
        tc::mma_commit(&s_full[b]);
      }
      // no MMA or commit arrival may land after the CTA has finished
      tc::mma_commit(&drain[qw == 0 ? 0 : 2]);
      tc::mbar_wait(&drain[qw == 0 ? 0 : 2], 0, err);
    }
  } else if (warp == PV_WARP) {
    if (lane == 0) {
      // ---------------------------------------------------------- P.V issuer
      // O_w += P_i . V_i as soon as the P of tile i is in TMEM (group w = i % 2).  Tile
      // i's Q.K^T finished before its softmax began, so the commit after P.V frees the
      // whole stage.
      constexpr uint32_t idesc_pv = tc::idesc_bf16_f32(L::MR, D) | (1u << 16);  // B (= V) MN-major
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
          const bool first = meta[s].local < 2;  // this group's first tile of the piece
          const uint32_t pt = tmem + L::S_COL(pv & (NSB - 1));  // P of the tile, in its S buffer
          const uint32_t v = tc::smem_u32(sKV + s * L::STAGE + L::K_BYTES);
          // K slice kk = the 16 keys of page kk: V [column block][16 tokens] blocks 2 KB apart
#pragma unroll
          for (int kk = 0; kk < PPT; ++kk)
            tc::mma_bf16_ts(tmem + L::O_COL(w), pt + kk * 8, tc::sdesc_mn128(v + kk * L::V_PAGE, 2048), idesc_pv,
                            (kk > 0 || !first) ? 1u : 0u);
          // the low halves of P (columns TT / 2 on)
#pragma unroll
          for (int kk = 0; kk < PPT; ++kk)
            tc::mma_bf16_ts(tmem + L::O_COL(w), pt + TT / 2 + kk * 8, tc::sdesc_mn128(v + kk * L::V_PAGE, 2048),
                            idesc_pv, 1u);
          // the piece's last tile: every Q.K^T of the piece has finished (each before its
          // tile's softmax began), so its Q buffer is free
          if (meta[s].local == meta[s].n_tiles - 1) tc::mbar_arrive(&q_empty[meta[s].qslot]);
          tc::mma_commit(&kv_empty[s]);
          tc::mma_commit(&s_free[pv & (NSB - 1)]);  // P read: S buffer free for tile pv + NSB
          ++pv;
          idle_since = 0;
        } else {
          const uint64_t t = tc::global_ns();
          if (idle_since == 0) {
            idle_since = t;
          } else if (t - idle_since > lim) {
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
    // SP: row quarter * 16 + (lane & 15), the two half-warps taking columns
    // [0, TT / 2) and [TT / 2, TT) of S (and halves of O); else row quarter * 32 + lane
    constexpr int CW = SP ? TT / 2 : TT;  // score columns per thread
    const int hf = SP ? lane >> 4 : 0;    // which half of the row's columns
    const int r_local = SP ? quarter * 16 + (lane & 15) : quarter * 32 + lane;
    const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
    const uint32_t tOw = tmem + lane_off + L::O_COL(wg);
    const int gthread = (warp - SM_WARP0 - 4 * wg) * 32 + lane;  // 0..127 within the group
    // the thread's O columns: SP, halves [hf D / 2, hf D / 2 + D / 2) read as 32-column
    // chunks cb (16x32bx2 with offset D / 2); else all D
    auto o_ld = [&](int cb, float (&v)[32]) {
      if constexpr (SP) tc::tmem_ld16x2_32<D / 2>(tOw + cb * 32, v);
      else tc::tmem_ld32(tOw + cb * 32, v);
    };
    constexpr int OCB = SP ? D / 64 : D / 32;  // 32-column chunks of O per thread
    auto o_col = [&](int cb) { return SP ? hf * (D / 2) + cb * 32 : cb * 32; };

    // The partial of a piece's half: O_w as the P.V of tile ti (the half's last) left
    // it, with its (m, l), into rows `base` of the workspace.  The parity of s_free is
    // unambiguous as for the rescale below: the phase before (tile ti - NSB) completed
    // before the Q.K^T of tile ti, and the one after needs the P of tile ti + NSB, which
    // this group writes only after this call.
    auto write_partial = [&](int ti, size_t base, float pm, float plsum, bool act) -> bool {
      if (!__all_sync(0xffffffffu, tc::mbar_wait(&s_free[ti & (NSB - 1)], (ti / NSB) & 1, err, lim))) return false;
      tc::tc_fence_after();
#pragma unroll
      for (int cb = 0; cb < OCB; ++cb) {
        float v[32];
        o_ld(cb, v);
        if (act) {
          float* o = a.ws_acc + base * D + o_col(cb);
#pragma unroll
          for (int e = 0; e < 32; e += 4) *(float4*)(o + e) = make_float4(v[e], v[e + 1], v[e + 2], v[e + 3]);
        }
      }
      if (act && hf == 0) {
        a.ws_ml[base * 2] = pm;
        a.ws_ml[base * 2 + 1] = plsum;
      }
      return true;
    };
    // a partial not yet written: the group's last tile of its previous piece
    bool pend = false, pend_act = false;
    int pend_i = 0;
    size_t pend_base = 0;
    float pend_m = 0.f, pend_l = 0.f;

    float m_used = -INFINITY, l = 0.f;
    bool ok = true;
    for (int i = wg; ok; i += 2) {
      const int b = i & (NSB - 1);
      ok = __all_sync(0xffffffffu, tc::mbar_wait(&s_full[b], (i / NSB) & 1, err, lim));
      if (!ok || i >= *end_tile) break;
      tc::tc_fence_after();
      const int s = i % NS;
      // acquire the producer's description of the tile (this phase completed long ago;
      // the stage cannot move on before this group's P.V of the tile)
      ok = __all_sync(0xffffffffu, tc::mbar_wait(&kv_full[s], (i / NS) & 1, err, lim));
      if (!ok) break;
      const int c = meta[s].c, g = meta[s].g, pslot = meta[s].slot, rb = meta[s].rb;
      const int local = meta[s].local, n_tiles = meta[s].n_tiles, valid = meta[s].valid;
      const bool block_tile = meta[s].block != 0;
      const int bt = meta[s].bt;
      const int gr = rb * ROWS + r_local;
      const bool active = gr < R;
      const int jq = active ? gr / G : 0;
      if (local < 2) {  // this group's first tile of a new piece
        m_used = -INFINITY;
        l = 0.f;
      }
      float sv[CW];
      if constexpr (SP) tc::tmem_ld16x2_32<TT / 2>(tmem + lane_off + L::S_COL(b), sv);
      else tc::tmem_ld(tmem + lane_off + L::S_COL(b), sv);
      // raw scores; the scale (> 0) is applied inside the exponent below
      float mx = -INFINITY;
      if (valid == TT && !(block_tile && a.causal_block)) {
#pragma unroll
        for (int j = 0; j < CW; ++j) mx = fmaxf(mx, sv[j]);
      } else {
        // causal block: query position jq sees the block keys 0..jq
        const int vis_end = ((block_tile && a.causal_block) ? min(valid, jq + 1 - bt * TT) : valid) - hf * CW;
#pragma unroll
        for (int j = 0; j < CW; ++j) {
          sv[j] = j < vis_end ? sv[j] : -INFINITY;
          mx = fmaxf(mx, sv[j]);
        }
      }
      if constexpr (SP) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
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
      uint32_t pk[CW / 2], pl[CW / 2];
      const float2 sc2 = make_float2(scale_log2, scale_log2), nm2 = make_float2(-mu, -mu);
      const float2 neg1 = make_float2(-1.f, -1.f);
#pragma unroll
      for (int j = 0; j < CW; j += 2) {
        // p = 2^(s scale - m): the exponents of a pair in one packed FFMA, then one ex2
        // each (flushing results below 2^-126 to zero); 2^(-inf) = 0 for masked columns
        const float2 e = tc::ffma2(make_float2(sv[j], sv[j + 1]), sc2, nm2);
        const float2 pp = make_float2(tc::ex2_ftz(e.x), tc::ex2_ftz(e.y));
        psum = tc::fadd2(psum, pp);
        // p = hi + lo with hi = bf16(p) and lo = bf16(p - hi): the P.V products of both
        // halves are exact in the fp32 accumulator, so P carries about 16 bits
        __nv_bfloat162 h2 = __floats2bfloat162_rn(pp.x, pp.y);
        const uint32_t hb = *reinterpret_cast<uint32_t*>(&h2);
        pk[j / 2] = hb;
        const float2 hf2 = make_float2(__uint_as_float(hb << 16), __uint_as_float(hb & 0xFFFF0000u));
        const float2 r = tc::ffma2(hf2, neg1, pp);  // p - hi, exact in fp32
        __nv_bfloat162 l2 = __floats2bfloat162_rn(r.x, r.y);
        pl[j / 2] = *reinterpret_cast<uint32_t*>(&l2);
      }
      float ps = psum.x + psum.y;
      if constexpr (SP) ps += __shfl_xor_sync(0xffffffffu, ps, 16);  // the row's other half
      l += ps;
      // P over S_b (bf16 pairs: the row's keys 2c, 2c + 1 in column c): hi in the first
      // quarter of the columns, lo in the second
      if constexpr (SP) {
        tc::tmem_st16x2_16u<TT / 4>(tmem + lane_off + L::S_COL(b), pk);
        tc::tmem_st16x2_16u<TT / 4>(tmem + lane_off + L::S_COL(b) + TT / 2, pl);
      } else {
        tc::tmem_stu(tmem + lane_off + L::S_COL(b), pk);
        tc::tmem_stu(tmem + lane_off + L::S_COL(b) + TT / 2, pl);
      }
      if (__any_sync(0xffffffffu, rescale)) {
        // O_w may be rescaled only once the group's previous P.V (tile i - 2, S buffer
        // (i - 2) % NSB) has finished.  Its phase of s_free is unambiguous here: the
        // phase before it (tile i - 2 - NSB) completed before the Q.K^T of tile i - 2
        // was issued, and the one after it needs a P this group has not written yet.
        ok = __all_sync(0xffffffffu, tc::mbar_wait(&s_free[(i - 2) & (NSB - 1)], ((i - 2) / NSB) & 1, err, lim));
        if (!ok) break;
        tc::tc_fence_after();
        // O_w holds this group's earlier tiles of the piece
#pragma unroll
        for (int cb = 0; cb < OCB; ++cb) {
          float v[32];
          o_ld(cb, v);
#pragma unroll
          for (int e = 0; e < 32; ++e) v[e] *= alpha;
          if constexpr (SP) tc::tmem_st16x2_32<D / 2>(tOw + cb * 32, v);
          else tc::tmem_st32(tOw + cb * 32, v);
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
      if (pend) {
        // the previous piece's partial, now that the P of this tile (the first of a new
        // piece for this group, so no rescale above) is written and before its P.V may
        // overwrite O_w: by now the P.V of that piece's last tile has left the tensor
        // pipe's queue, so the wait for it overlaps this tile's softmax
        pend = false;
        ok = write_partial(pend_i, pend_base, pend_m, pend_l, pend_act);
        if (!ok) break;
      }
      tc::tc_fence_before();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(&p_full[b]);

      if (local >= n_tiles - 2) {
        // this group's last tile of the piece: its partial is the half of the piece
        // made of tiles of parity (local & 1), whichever group ran them, so the result
        // does not depend on timing; rows of the row block.  It is written during the
        // group's next tile, or after the loop.
        pend = true;
        pend_i = i;
        pend_base = ((size_t)pslot * 2 + (local & 1)) * RB + r_local;
        pend_m = m_used;
        pend_l = l;
        pend_act = active;
      }
    }
    if (pend && ok) write_partial(pend_i, pend_base, pend_m, pend_l, pend_act);
    tc::tc_fence_before();
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

template <int D, bool SP>
bool launch_tc(const AttnArgs& a, cudaStream_t s) {
  static bool attr_set[64] = {};
  static int n_sm[64] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 64 && !attr_set[dev]) {
    if (cudaFuncSetAttribute(attn_tc_kernel<D, SP>, cudaFuncAttributeMaxDynamicSharedMemorySize, Lay<D, SP>::SMEM) !=
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
    set_error("tensor-core attention writes two partials per piece");
    return false;
  }
  const int sms = dev < 64 && n_sm[dev] > 0 ? n_sm[dev] : 148;
  const int grid = min(sms, kAttnMaxChunksAuto);
  const int z_req = a.split_tokens > 0 ? (a.split_tokens + TT - 1) / TT : 0;
  launch_pdl(attn_sched_kernel, 1, 1024, 0, s, a.ctx_lens, a.C, (long)a.max_pages * a.page_size, (a.K + TT - 1) / TT,
                                       a.Hkv * n_rb, grid, z_req, a.max_chunks, a.sched, a.sched + 64, a.err);
  note_launch();
  const float scale_log2 = 1.4426950408889634f / sqrtf((float)D);
  launch_pdl(attn_tc_kernel<D, SP>, grid, THREADS, Lay<D, SP>::SMEM, s, maps, a, scale_log2, n_rb);
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
  // the tile line (all sequences end to end) is indexed in 32 bits
  const long n_rb = (a.K * G + ROWS - 1) / ROWS;
  const long line = (long)a.C * a.Hkv * n_rb * (((long)a.max_pages * a.page_size + TT - 1) / TT + (a.K + TT - 1) / TT);
  if (line >= (1L << 30)) return *why = "too many context tiles in one call", false;
  return true;
}

bool attn_tc_launch(const AttnArgs& a, cudaStream_t s) {
  // R = K * G query rows per kv head: up to 64 in one M = 64 tile
  const bool sp = a.K * (a.Hq / a.Hkv) <= 64;
  if (a.D == 128) return sp ? launch_tc<128, true>(a, s) : launch_tc<128, false>(a, s);
  return sp ? launch_tc<64, true>(a, s) : launch_tc<64, false>(a, s);
}

}  // namespace hspec
