// C-ABI of libhspec.so (declared in include/hspec.h): host-side validation,
// workspace carving, launch sequencing of the draft step, and status reporting.
// Every computation runs in this library's kernels; this file only checks
// arguments and launches.
#include <math.h>
#include <stdarg.h>
#include <stdio.h>
#include <string.h>

#include <atomic>
#include <cstdlib>
#include <map>
#include <mutex>
#include <string>
#include <vector>

#include "../../include/hspec.h"
#include "common.cuh"
#include "kernels.cuh"

// Device error word shared by all kernels of the library (OR of hspec::kErr* bits).
__device__ int g_hspec_device_error;

namespace hspec {

static std::atomic<unsigned long long> g_launches{0};
static thread_local char g_last_error[512] = "";

void note_launch(int n) { g_launches.fetch_add((unsigned long long)n, std::memory_order_relaxed); }

// Programmatic dependent launch: HSPEC_PDL=1 or 0 in the environment forces it on or off
// for every launch.  Otherwise it is on for the draft step's own launches when the batch
// has at most kPdlMaxRows block rows: with the GEMMs requesting their first weight tiles
// before the wait, steps at 8-32 requests measured 2-4% faster; at 128 requests (2048
// rows) there was no consistent gain (without the early weight requests it had measured
// 2% slower there: more overlap under the power cap).
constexpr int kPdlMaxRows = 1024;
static thread_local bool t_step_pdl = false;
static int pdl_env() {  // -1 unset, 0 off, 1 on
  static const int mode = [] {
    const char* e = getenv("HSPEC_PDL");
    return e && (e[0] == '0' || e[0] == '1') ? e[0] - '0' : -1;
  }();
  return mode;
}
bool pdl_enabled() {
  const int env = pdl_env();
  return env >= 0 ? env == 1 : t_step_pdl;
}
// Scope of one draft step's launches.
struct StepPdl {
  explicit StepPdl(int rows) { t_step_pdl = rows <= kPdlMaxRows; }
  ~StepPdl() { t_step_pdl = false; }
};

void set_error(const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_last_error, sizeof(g_last_error), fmt, ap);
  va_end(ap);
}

// The current thread's CUDA context (the driver's handle), or NULL.  Device
// addresses of this library's static arrays are cached per context: a context that
// is destroyed and created again (cudaDeviceReset) maps its modules afresh.
void* current_context() {
  using CtxGetCurrentFn = int (*)(void**);
  static CtxGetCurrentFn fn = [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return (CtxGetCurrentFn) nullptr;
    return (CtxGetCurrentFn)p;
  }();
  void* ctx = nullptr;
  if (!fn || fn(&ctx) != 0) return nullptr;
  return ctx;
}

// Device address of the static device array `symbol` in the current context, looked
// up once per context (cudaGetSymbolAddress maps the array's module on first use and
// allocates nothing else).  NULL with the message recorded on failure.
void* symbol_address(const void* symbol, const char* what) {
  struct Entry {
    void* ctx;
    const void* sym;
    void* addr;
  };
  static std::mutex mu;
  static std::vector<Entry> cache;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    set_error("%s: no current CUDA device", what);
    return nullptr;
  }
  void* ctx = current_context();  // NULL before the runtime has made a context current
  std::lock_guard<std::mutex> lock(mu);
  if (ctx)
    for (const Entry& e : cache)
      if (e.ctx == ctx && e.sym == symbol) return e.addr;
  void* p = nullptr;
  const cudaError_t e = cudaGetSymbolAddress(&p, symbol);
  if (e != cudaSuccess) {
    if (e == cudaErrorMemoryAllocation)
      set_error("%s: out of device memory while loading the library's static device arrays on device %d "
                "(cudaGetSymbolAddress: %s)", what, dev, cudaGetErrorString(e));
    else
      set_error("%s: cudaGetSymbolAddress failed on device %d: %s", what, dev, cudaGetErrorString(e));
    cudaGetLastError();
    return nullptr;
  }
  if (!ctx) ctx = current_context();  // the lookup made the device's primary context current
  if (ctx) cache.push_back({ctx, symbol, p});
  return p;
}

// Address of the device error word in the current context.
int* device_error_word() { return (int*)symbol_address((const void*)&g_hspec_device_error, "device error word"); }

// ---------------------------------------------------------------- profiling
// Event pairs recorded around kernel groups of the draft step when enabled.
struct Profiler {
  std::mutex mu;
  bool on = false;
  std::vector<cudaEvent_t> pool;
  struct Rec {
    const char* name;
    int a, b;
  };
  std::vector<Rec> recs;
  size_t used = 0;
  int take() {
    if (used == pool.size()) {
      cudaEvent_t e;
      if (cudaEventCreate(&e) != cudaSuccess) return -1;
      pool.push_back(e);
    }
    return (int)used++;
  }
};
static Profiler g_prof;

struct ProfScope {
  cudaStream_t s;
  const char* name;
  int a = -1;
  ProfScope(const char* n, cudaStream_t st) : s(st), name(n) {
    if (!g_prof.on) return;
    std::lock_guard<std::mutex> lock(g_prof.mu);
    a = g_prof.take();
    if (a >= 0) cudaEventRecord(g_prof.pool[a], s);
  }
  ~ProfScope() {
    if (a < 0) return;
    std::lock_guard<std::mutex> lock(g_prof.mu);
    int b = g_prof.take();
    if (b < 0) return;
    cudaEventRecord(g_prof.pool[b], s);
    g_prof.recs.push_back({name, a, b});
  }
};

}  // namespace hspec

using namespace hspec;

struct hspec_drafter {
  hspec_cfg cfg;
  hspec_model_weights w;
};

namespace {

#define FAIL(code, ...)     \
  do {                      \
    set_error(__VA_ARGS__); \
    return (code);          \
  } while (0)

size_t elem_bytes(const hspec_cfg* c) { return c->dtype == HSPEC_DTYPE_BF16 ? 2 : 4; }
size_t align256(size_t b) { return (b + 255) & ~(size_t)255; }

bool has_kind(const hspec_cfg* c, char k) {
  for (int i = 0; i < c->n_layers; ++i)
    if (c->layer_kinds[i] == k) return true;
  return false;
}

hspec_status check_launch(const char* what) {
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) FAIL(HSPEC_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
  return HSPEC_OK;
}

hspec_status validate_cfg(const hspec_cfg* c, bool need_attn, bool need_ssm) {
  if (!c) FAIL(HSPEC_ERR_INVALID_ARG, "cfg is NULL");
  if (c->dtype != HSPEC_DTYPE_F32 && c->dtype != HSPEC_DTYPE_BF16)
    FAIL(HSPEC_ERR_INVALID_ARG, "dtype %d is neither HSPEC_DTYPE_F32 nor HSPEC_DTYPE_BF16", c->dtype);
  if (c->flags & ~(HSPEC_FLAG_ROPE | HSPEC_FLAG_GATE | HSPEC_FLAG_CAUSAL_BLOCK | HSPEC_FLAG_FUSE_INJECT))
    FAIL(HSPEC_ERR_INVALID_ARG, "unknown flag bits 0x%x", c->flags);
  if (c->d_model <= 0) FAIL(HSPEC_ERR_INVALID_ARG, "d_model must be positive");
  if (need_attn) {
    if (c->n_q_heads <= 0 || c->n_kv_heads <= 0 || c->head_dim <= 0 || c->page_size <= 0)
      FAIL(HSPEC_ERR_INVALID_ARG, "attention dims and page_size must be positive");
    if (c->n_q_heads % c->n_kv_heads)
      FAIL(HSPEC_ERR_SHAPE_MISMATCH, "n_q_heads %d is not a multiple of n_kv_heads %d", c->n_q_heads,
           c->n_kv_heads);
    if (c->head_dim % 2) FAIL(HSPEC_ERR_SHAPE_MISMATCH, "head_dim must be even (rotate-half RoPE)");
    if (c->attn_split_tokens < 0 || c->attn_split_tokens % 16)
      FAIL(HSPEC_ERR_INVALID_ARG, "attn_split_tokens must be 0 or a positive multiple of 16");
  }
  if (need_ssm) {
    if (c->n_ssm_heads <= 0 || c->ssm_head_dim <= 0 || c->d_state <= 0)
      FAIL(HSPEC_ERR_INVALID_ARG, "Mamba-2 dims must be positive");
    if (c->ssd_chunk < 0) FAIL(HSPEC_ERR_INVALID_ARG, "ssd_chunk must be >= 0");
  }
  if (c->norm_eps < 0.f) FAIL(HSPEC_ERR_INVALID_ARG, "norm_eps must be >= 0");
  if (c->wait_limit_ns < 0) FAIL(HSPEC_ERR_INVALID_ARG, "wait_limit_ns must be >= 0");
  return HSPEC_OK;
}

// The kernels' pipeline wait limit (0 passes the kernels' default).
unsigned long long wait_ns(const hspec_cfg* c) { return (unsigned long long)c->wait_limit_ns; }

int ssd_chunk_len(const hspec_cfg* c, int K) { return (c->ssd_chunk > 0 && c->ssd_chunk < K) ? c->ssd_chunk : K; }

hspec_status validate_ssd_shape(const hspec_cfg* c, int K) {
  if (K < 1 || K > 64) FAIL(HSPEC_ERR_UNSUPPORTED, "K=%d outside 1..64", K);
  if (ssd_smem_bytes(c->ssm_head_dim, c->d_state, ssd_chunk_len(c, K)) > 227 * 1024)
    FAIL(HSPEC_ERR_UNSUPPORTED, "SSD tile P=%d N=%d chunk=%d exceeds shared memory", c->ssm_head_dim, c->d_state,
         ssd_chunk_len(c, K));
  return HSPEC_OK;
}

hspec_status validate_kv(const hspec_cfg* c, const hspec_kv_view* kv) {
  if (!kv) FAIL(HSPEC_ERR_INVALID_ARG, "kv view is NULL");
  if (!kv->k_pool || !kv->v_pool || !kv->page_table)
    FAIL(HSPEC_ERR_INVALID_ARG, "kv pools and page table must be non-NULL");
  if (kv->num_pages <= 0 || kv->max_pages <= 0)
    FAIL(HSPEC_ERR_PAGE_OOB, "num_pages (%d) and max_pages (%d) must be positive", kv->num_pages, kv->max_pages);
  if ((long)kv->max_pages * c->page_size > (1L << 30))
    FAIL(HSPEC_ERR_UNSUPPORTED, "max_pages * page_size exceeds 2^30 tokens");
  return HSPEC_OK;
}

struct AttnPlan {
  int split_tokens, n_splits, max_chunks;
  size_t rows;  // partial rows
  size_t ws;
};

AttnPlan attn_plan(const hspec_cfg* c, int C, int K, int max_pages) {
  AttnPlan p;
  const int max_ctx = max_pages * c->page_size;
  p.split_tokens = attn_split_tokens(c->dtype, C, c->n_kv_heads, K, max_ctx, c->attn_split_tokens);
  p.n_splits = attn_num_splits(c->dtype, K, max_ctx, p.split_tokens);
  p.max_chunks = p.split_tokens > 0 ? kAttnMaxChunksExplicit : kAttnMaxChunksAuto;
  const int G = c->n_q_heads / c->n_kv_heads;
  p.rows = attn_partial_rows(c->dtype, C, c->n_kv_heads, K, G, p.n_splits, p.max_chunks);
  p.ws = align256(attn_ws_bytes(c->dtype, C, c->n_kv_heads, K, G, c->head_dim, p.n_splits, p.max_chunks));
  return p;
}

// Fills AttnArgs for one launch; partials carved from `ws`.
AttnArgs attn_args(const hspec_cfg* c, const AttnPlan& p, const hspec_kv_view* kv, const int32_t* ctx_lens,
                   int C, int K, void* ws) {
  AttnArgs a;
  a.C = C;
  a.K = K;
  a.Hq = c->n_q_heads;
  a.Hkv = c->n_kv_heads;
  a.D = c->head_dim;
  a.k_pool = kv->k_pool;
  a.v_pool = kv->v_pool;
  a.num_pages = kv->num_pages;
  a.page_size = c->page_size;
  a.page_table = kv->page_table;
  a.max_pages = kv->max_pages;
  a.ctx_lens = ctx_lens;
  a.split_tokens = p.split_tokens;
  a.n_splits = p.n_splits;
  a.max_chunks = p.max_chunks;
  a.causal_block = (c->flags & HSPEC_FLAG_CAUSAL_BLOCK) != 0;
  a.tile_pieces = c->dtype == HSPEC_DTYPE_BF16;
  a.sub_splits = attn_sub_splits(c->dtype);
  a.ws_acc = (float*)ws;
  a.ws_ml = a.ws_acc + p.rows * a.D;
  a.sched = (int*)(a.ws_ml + p.rows * 2);
  a.err = device_error_word();
  a.wait_ns = wait_ns(c);
  return a;
}

// bf16 draft step with HSPEC_FLAG_FUSE_INJECT: the injected state's share of the SSD
// output is added in the injection GEMM's epilogue (h0 never stored; the scan runs
// from a zero state).  Default: h0 stored, read by the tensor-core scan -- measured
// faster from 8 requests up (the epilogue's L2 reads of C stall the weight stream, and
// the zero-state CUDA-core scan costs more than the tensor-core readout it replaces).
bool step_fuses_inject(const hspec_cfg* c) {
  const int N = c->d_state;
  const long HP = (long)c->n_ssm_heads * c->ssm_head_dim;
  const long n_in = 2 * HP + 2L * N + c->n_ssm_heads;
  return c->dtype == HSPEC_DTYPE_BF16 && (c->flags & HSPEC_FLAG_FUSE_INJECT) && N == 128 && c->ssm_head_dim % 2 == 0 &&
         n_in % 8 == 0 && (2 * HP + N) % 8 == 0 && HP % 2 == 0;
}

// Step workspace layout (all sub-buffers 256-byte aligned).
struct StepPlan {
  size_t x, xn, big, y, g, h0, attn, pval, pidx, gpart, gcnt, rope, total;
  AttnPlan ap;
  int n_parts;
  size_t gpart_bytes;  // partials of the projection / MLP GEMMs with a cut K loop
  int gmax_tiles;      // tile counters that follow them (per call site)
  int gcnt_sites;      // call sites with their own counter slice
};

StepPlan step_plan(const hspec_cfg* c, int C, int K, int max_pages) {
  StepPlan s = {};
  const size_t M = (size_t)C * K, E = elem_bytes(c), d = c->d_model;
  const size_t HP = (size_t)c->n_ssm_heads * c->ssm_head_dim;
  const size_t HPN = HP * c->d_state;
  const size_t n_in = 2 * HP + 2 * (size_t)c->d_state + c->n_ssm_heads;
  const size_t n_qkv = (size_t)(c->n_q_heads + 2 * c->n_kv_heads) * c->head_dim;
  const bool ssm = has_kind(c, 'M'), att = has_kind(c, 'A');
  size_t big = 0, gw = 0;
  if (ssm) big = n_in, gw = HP;
  if (att) big = big > n_qkv ? big : n_qkv, gw = gw > (size_t)c->n_q_heads * c->head_dim ? gw : (size_t)c->n_q_heads * c->head_dim;
  if (c->d_ff > 0) big = big > (size_t)c->d_ff ? big : (size_t)c->d_ff;
  size_t off = 0;
  s.x = off, off += align256(M * d * 4);
  s.xn = off, off += align256(M * d * E);
  s.big = off, off += align256(M * big * E);
  s.y = off, off += align256(ssm ? M * HP * 4 : 0);
  s.g = off, off += align256(M * gw * E);
  s.h0 = off, off += align256(ssm && !step_fuses_inject(c) ? (size_t)C * HPN * 4 : 0);
  s.attn = off;
  if (att) {
    s.ap = attn_plan(c, C, K, max_pages);
    off += s.ap.ws;
  }
  const int head_rows = c->draft_vocab > 0 ? c->draft_vocab : c->vocab;
  s.n_parts = c->vocab > 0 ? cdiv(head_rows, argmax_tile_n(c->dtype)) : 0;
  s.pval = off, off += align256(M * s.n_parts * 4);
  s.pidx = off, off += align256(M * s.n_parts * 4);
  // RoPE (cos, sin) table of the step's rows, read by the attention projections' epilogue
  s.rope = off, off += align256(att && (c->flags & HSPEC_FLAG_ROPE) ? M * (size_t)(c->head_dim / 2) * 8 : 0);
  // split-K workspace: the largest need of the step's projection and MLP GEMMs
  {
    const int Mi = (int)M;
    struct Shape { GemmEpi e; int n, k; bool on; } shapes[] = {
        {kEpiStore, (int)n_in, (int)d, ssm}, {kEpiResid, (int)d, (int)HP, ssm},
        {kEpiStore, (int)n_qkv, (int)d, att}, {kEpiResid, (int)d, c->n_q_heads * c->head_dim, att},
        {kEpiSwiGLU, c->d_ff, (int)d, c->d_ff > 0}, {kEpiResid, (int)d, c->d_ff, c->d_ff > 0}};
    for (const Shape& sh : shapes) {
      if (!sh.on) continue;
      const size_t b = gemm_kcut_bytes(c->dtype, sh.e, Mi, sh.n, sh.k);
      if (b > s.gpart_bytes) s.gpart_bytes = b;
      if (b > 0) {
        const int nt = gemm_tile_count(c->dtype, sh.e, Mi, sh.n);
        if (nt > s.gmax_tiles) s.gmax_tiles = nt;
      }
    }
  }
  s.gpart = off, off += align256(s.gpart_bytes);
  // one slice of tile counters per K-cut GEMM call of the step (at most 4 per layer),
  // all zeroed once at the start of the step
  s.gcnt_sites = 4 * c->n_layers;
  s.gcnt = off, off += align256((size_t)s.gmax_tiles * s.gcnt_sites * 4);
  s.total = off;
  return s;
}

GemmArgs gemm_args(int M, int N, int K, const void* A, long lda, const void* B, long ldb, void* out, long ldo) {
  GemmArgs g = {};
  g.M = M, g.N = N, g.K = K;
  g.A = A, g.lda = lda, g.B = B, g.ldb = ldb, g.out = out, g.ldo = ldo;
  return g;
}

}  // namespace

extern "C" {

const char* hspec_version(void) { return "hspec-b200 0.1.0 (sm_100a)"; }

hspec_status hspec_profile_enable(int on) {
  std::lock_guard<std::mutex> lock(g_prof.mu);
  g_prof.on = on != 0;
  if (on) {
    g_prof.recs.clear();
    g_prof.used = 0;
  }
  return HSPEC_OK;
}

int hspec_profile_read(char* names, double* total_ms, int* count, int max_entries) {
  std::lock_guard<std::mutex> lock(g_prof.mu);
  std::vector<std::string> order;
  std::map<std::string, std::pair<double, int>> agg;
  for (const auto& r : g_prof.recs) {
    if (cudaEventSynchronize(g_prof.pool[r.b]) != cudaSuccess) return -1;
    float ms = 0.f;
    if (cudaEventElapsedTime(&ms, g_prof.pool[r.a], g_prof.pool[r.b]) != cudaSuccess) return -1;
    auto it = agg.find(r.name);
    if (it == agg.end()) {
      order.push_back(r.name);
      agg[r.name] = {ms, 1};
    } else {
      it->second.first += ms;
      it->second.second += 1;
    }
  }
  int n = 0;
  for (const auto& k : order) {
    if (n >= max_entries) break;
    if (names) {
      strncpy(names + 32 * n, k.c_str(), 31);
      names[32 * n + 31] = 0;
    }
    if (total_ms) total_ms[n] = agg[k].first;
    if (count) count[n] = agg[k].second;
    ++n;
  }
  return n;
}

const char* hspec_last_error(void) { return g_last_error; }

unsigned long long hspec_launch_count(void) { return g_launches.load(); }

const char* hspec_status_string(hspec_status s) {
  switch (s) {
    case HSPEC_OK: return "ok";
    case HSPEC_ERR_INVALID_ARG: return "invalid argument";
    case HSPEC_ERR_SHAPE_MISMATCH: return "shape mismatch";
    case HSPEC_ERR_PAGE_OOB: return "page table / pool inconsistent";
    case HSPEC_ERR_UNSUPPORTED: return "unsupported shape";
    case HSPEC_ERR_CUDA: return "CUDA error";
    case HSPEC_ERR_DEVICE_CHECK: return "device-side check failed (page id, context length or token id)";
    case HSPEC_ERR_WORKSPACE: return "workspace missing, too small or misaligned";
  }
  return "unknown status";
}

hspec_status hspec_sync_status(void* stream) {
  cudaError_t e = cudaStreamSynchronize((cudaStream_t)stream);
  if (e != cudaSuccess) FAIL(HSPEC_ERR_CUDA, "stream: %s", cudaGetErrorString(e));
  int* w = device_error_word();
  if (!w) FAIL(HSPEC_ERR_CUDA, "device error word unavailable");
  int bits = 0;
  e = cudaMemcpy(&bits, w, sizeof(int), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) FAIL(HSPEC_ERR_CUDA, "reading device error word: %s", cudaGetErrorString(e));
  if (bits) {
    cudaMemset(w, 0, sizeof(int));
    FAIL(HSPEC_ERR_DEVICE_CHECK, "device check bits 0x%x (1 page id, 2 context length, 4 token id, 8 timeout)",
         bits);
  }
  return HSPEC_OK;
}

hspec_status hspec_inject_state(const hspec_cfg* cfg, const void* W_inj, const void* h_last, int C, float* h0,
                                void* stream) {
  hspec_status st = validate_cfg(cfg, false, true);
  if (st) return st;
  if (!W_inj || !h_last || !h0) FAIL(HSPEC_ERR_INVALID_ARG, "W_inj, h_last and h0 must be non-NULL");
  if (C < 1) FAIL(HSPEC_ERR_INVALID_ARG, "C must be >= 1");
  const long HPN = (long)cfg->n_ssm_heads * cfg->ssm_head_dim * cfg->d_state;
  if (HPN > (1L << 31) - 1) FAIL(HSPEC_ERR_UNSUPPORTED, "H*P*N too large");
  GemmArgs g = gemm_args(C, (int)HPN, cfg->d_model, h_last, cfg->d_model, W_inj, cfg->d_model, h0, HPN);
  g.out_f32 = true;
  g.wait_ns = wait_ns(cfg);
  if (!gemm(cfg->dtype, kEpiStore, g, (cudaStream_t)stream)) return HSPEC_ERR_UNSUPPORTED;
  return check_launch("hspec_inject_state");
}

hspec_status hspec_ssd_block_scan(const hspec_cfg* cfg, const void* x, const float* dt, const float* A,
                                  const void* B, const void* Cm, const float* D, const float* h0, int C, int K,
                                  float* y, float* hK, void* stream) {
  hspec_status st = validate_cfg(cfg, false, true);
  if (st) return st;
  if (!x || !dt || !A || !B || !Cm || !D || !y) FAIL(HSPEC_ERR_INVALID_ARG, "x, dt, A, B, Cm, D, y must be non-NULL");
  if (C < 1) FAIL(HSPEC_ERR_INVALID_ARG, "C must be >= 1");
  if ((st = validate_ssd_shape(cfg, K))) return st;
  SsdArgs a = {};
  a.C = C, a.K = K, a.H = cfg->n_ssm_heads, a.P = cfg->ssm_head_dim, a.N = cfg->d_state;
  a.Q = ssd_chunk_len(cfg, K);
  a.x = x, a.x_rs = (long)a.H * a.P;
  a.dt = dt, a.dt_rs = a.H, a.dt_bias = nullptr;
  a.A = A, a.D = D;
  a.B = B, a.Cm = Cm, a.bc_rs = a.N;
  a.h0 = h0, a.y = y, a.y_rs = (long)a.H * a.P, a.hK = hK;
  a.wait_ns = wait_ns(cfg);
  ssd_scan(cfg->dtype, a, (cudaStream_t)stream);
  return check_launch("hspec_ssd_block_scan");
}

}  // extern "C"

namespace hspec {
// Device address of the allocation-free attention's static scratch (noalloc.cu).
void* noalloc_scratch_address();
}  // namespace hspec

extern "C" {

hspec_status hspec_attn_paged_block_noalloc(const hspec_cfg* cfg, const void* q, const hspec_kv_view* kv,
                                            const int32_t* ctx_lens, const void* k_blk, const void* v_blk, int C,
                                            int K, void* out, void* stream) {
  hspec_status st = validate_cfg(cfg, true, false);
  if (st) return st;
  if ((st = validate_kv(cfg, kv))) return st;
  if (!q || !ctx_lens || !k_blk || !v_blk || !out)
    FAIL(HSPEC_ERR_INVALID_ARG, "q, ctx_lens, k_blk, v_blk, out must be non-NULL");
  if (C < 1 || K < 1 || K > 64) FAIL(HSPEC_ERR_UNSUPPORTED, "C=%d K=%d (need C >= 1, 1 <= K <= 64)", C, K);
  const int G = cfg->n_q_heads / cfg->n_kv_heads;
  const char* why = "";
  if (!attn_supported(cfg->dtype, K, G, cfg->head_dim, &why)) FAIL(HSPEC_ERR_UNSUPPORTED, "attention: %s", why);
  AttnPlan p = attn_plan(cfg, C, K, kv->max_pages);
  if (p.ws > HSPEC_NOALLOC_SCRATCH_BYTES)
    FAIL(HSPEC_ERR_WORKSPACE, "allocation-free attention needs %zu bytes of split partials; its static scratch holds %zu",
         p.ws, (size_t)HSPEC_NOALLOC_SCRATCH_BYTES);
  void* scratch = noalloc_scratch_address();
  if (!scratch) return HSPEC_ERR_CUDA;
  AttnArgs a = attn_args(cfg, p, kv, ctx_lens, C, K, scratch);
  const long qrow = (long)cfg->n_q_heads * cfg->head_dim, krow = (long)cfg->n_kv_heads * cfg->head_dim;
  a.q = q, a.q_rs = qrow;
  a.kb = k_blk, a.kb_rs = krow;
  a.vb = v_blk, a.vb_rs = krow;
  a.out = out, a.o_rs = qrow;
  if (!attn_paged(cfg->dtype, a, (cudaStream_t)stream)) return HSPEC_ERR_UNSUPPORTED;
  return check_launch("hspec_attn_paged_block_noalloc");
}

size_t hspec_attn_workspace_size(const hspec_cfg* cfg, int C, int K, int max_pages) {
  if (validate_cfg(cfg, true, false) || C < 1 || K < 1 || max_pages < 1) return 0;
  return attn_plan(cfg, C, K, max_pages).ws;
}

hspec_status hspec_attn_paged_block(const hspec_cfg* cfg, const void* q, const hspec_kv_view* kv,
                                    const int32_t* ctx_lens, const void* k_blk, const void* v_blk, int C, int K,
                                    void* out, void* workspace, size_t ws_bytes, void* stream) {
  hspec_status st = validate_cfg(cfg, true, false);
  if (st) return st;
  if ((st = validate_kv(cfg, kv))) return st;
  if (!q || !ctx_lens || !k_blk || !v_blk || !out) FAIL(HSPEC_ERR_INVALID_ARG, "q, ctx_lens, k_blk, v_blk, out must be non-NULL");
  if (C < 1 || K < 1 || K > 64) FAIL(HSPEC_ERR_UNSUPPORTED, "C=%d K=%d (need C >= 1, 1 <= K <= 64)", C, K);
  const int G = cfg->n_q_heads / cfg->n_kv_heads;
  const char* why = "";
  if (!attn_supported(cfg->dtype, K, G, cfg->head_dim, &why)) FAIL(HSPEC_ERR_UNSUPPORTED, "attention: %s", why);
  AttnPlan p = attn_plan(cfg, C, K, kv->max_pages);
  if (!workspace || ((uintptr_t)workspace & 255) || ws_bytes < p.ws)
    FAIL(HSPEC_ERR_WORKSPACE, "attention needs a 256-byte aligned workspace of %zu bytes (got %zu)", p.ws, ws_bytes);
  AttnArgs a = attn_args(cfg, p, kv, ctx_lens, C, K, workspace);
  const long qrow = (long)cfg->n_q_heads * cfg->head_dim, krow = (long)cfg->n_kv_heads * cfg->head_dim;
  a.q = q, a.q_rs = qrow;
  a.kb = k_blk, a.kb_rs = krow;
  a.vb = v_blk, a.vb_rs = krow;
  a.out = out, a.o_rs = qrow;
  if (!attn_paged(cfg->dtype, a, (cudaStream_t)stream)) return HSPEC_ERR_UNSUPPORTED;
  return check_launch("hspec_attn_paged_block");
}

size_t hspec_verify_workspace_size(const hspec_cfg* cfg, int C, int K) {
  if (!cfg || cfg->vocab < 1 || C < 1 || K < 1 || K > 64) return 0;
  return align256(verify_ws_bytes(cfg->dtype, C, K, cfg->vocab));
}

hspec_status hspec_verify_greedy(const hspec_cfg* cfg, const void* logits, const int32_t* drafts, int C, int K,
                                 int32_t* accepted, int32_t* next_token, int32_t* ctx_lens, void* workspace,
                                 size_t ws_bytes, void* stream) {
  if (!cfg) FAIL(HSPEC_ERR_INVALID_ARG, "cfg is NULL");
  if (cfg->dtype != HSPEC_DTYPE_F32 && cfg->dtype != HSPEC_DTYPE_BF16)
    FAIL(HSPEC_ERR_INVALID_ARG, "dtype %d is neither HSPEC_DTYPE_F32 nor HSPEC_DTYPE_BF16", cfg->dtype);
  if (cfg->vocab < 1) FAIL(HSPEC_ERR_INVALID_ARG, "verification needs cfg->vocab >= 1");
  if (!logits || !drafts || !accepted || !next_token)
    FAIL(HSPEC_ERR_INVALID_ARG, "logits, drafts, accepted and next_token must be non-NULL");
  if (C < 1 || K < 1 || K > 64) FAIL(HSPEC_ERR_UNSUPPORTED, "C=%d K=%d (need C >= 1, 1 <= K <= 64)", C, K);
  if ((long)C * (K + 1) > 0x7fffffffL || cfg->vocab > 65535L * 16384) FAIL(HSPEC_ERR_UNSUPPORTED, "too many rows or logits");
  const size_t need = hspec_verify_workspace_size(cfg, C, K);
  if (!workspace || ((uintptr_t)workspace & 255) || ws_bytes < need)
    FAIL(HSPEC_ERR_WORKSPACE, "verification needs a 256-byte aligned workspace of %zu bytes (got %zu)", need, ws_bytes);
  verify_greedy(cfg->dtype, logits, cfg->vocab, drafts, C, K, accepted, next_token, ctx_lens, workspace,
                (cudaStream_t)stream);
  return check_launch("hspec_verify_greedy");
}

hspec_status hspec_drafter_create(const hspec_cfg* cfg, const hspec_model_weights* w, hspec_drafter** out) {
  if (!out || !w) FAIL(HSPEC_ERR_INVALID_ARG, "weights and out must be non-NULL");
  *out = nullptr;
  if (!cfg) FAIL(HSPEC_ERR_INVALID_ARG, "cfg is NULL");
  if (cfg->n_layers < 1 || cfg->n_layers > HSPEC_MAX_LAYERS)
    FAIL(HSPEC_ERR_INVALID_ARG, "n_layers %d outside 1..%d", cfg->n_layers, HSPEC_MAX_LAYERS);
  for (int i = 0; i < cfg->n_layers; ++i)
    if (cfg->layer_kinds[i] != 'M' && cfg->layer_kinds[i] != 'A')
      FAIL(HSPEC_ERR_INVALID_ARG, "layer_kinds[%d] is neither 'M' nor 'A'", i);
  hspec_status st = validate_cfg(cfg, has_kind(cfg, 'A'), has_kind(cfg, 'M'));
  if (st) return st;
  if (cfg->d_ff < 0 || cfg->vocab < 0) FAIL(HSPEC_ERR_INVALID_ARG, "d_ff and vocab must be >= 0");
  if (cfg->draft_vocab < 0 || (cfg->draft_vocab > 0 && cfg->vocab == 0))
    FAIL(HSPEC_ERR_INVALID_ARG, "draft_vocab must be >= 0, and needs a vocab (the embedding table)");
  if (cfg->dtype == HSPEC_DTYPE_BF16) {
    // tensor-core GEMM operands are streamed by TMA: every GEMM reduction dimension
    // (= operand row stride) must be a multiple of 8 elements (16 bytes)
    const long HP = (long)cfg->n_ssm_heads * cfg->ssm_head_dim;
    const long dims[] = {cfg->d_model, HP, (long)cfg->n_q_heads * cfg->head_dim, cfg->d_ff};
    for (long v : dims)
      if (v % 8) FAIL(HSPEC_ERR_UNSUPPORTED, "bf16 drafter dims must be multiples of 8 (got %ld)", v);
  }
  for (int i = 0; i < cfg->n_layers; ++i) {
    const hspec_layer_weights& L = w->layers[i];
    if (!L.norm) FAIL(HSPEC_ERR_INVALID_ARG, "layer %d: norm weight is NULL", i);
    if (cfg->layer_kinds[i] == 'M') {
      if (!L.W_in || !L.dt_bias || !L.A || !L.D || !L.W_out || !L.W_inj ||
          (!L.gnorm && (cfg->flags & HSPEC_FLAG_GATE)))
        FAIL(HSPEC_ERR_INVALID_ARG, "layer %d: a Mamba-2 weight is NULL", i);
    } else if (!L.W_qkv || !L.W_o) {
      FAIL(HSPEC_ERR_INVALID_ARG, "layer %d: an attention weight is NULL", i);
    }
    if (cfg->d_ff > 0 && (!L.mlp_norm || !L.W_gate || !L.W_up || !L.W_down))
      FAIL(HSPEC_ERR_INVALID_ARG, "layer %d: an MLP weight is NULL", i);
  }
  if (cfg->vocab > 0 && (!w->final_norm || !w->W_lm)) FAIL(HSPEC_ERR_INVALID_ARG, "final_norm / W_lm is NULL");
  if (cfg->draft_vocab > 0 && (!w->W_lm_draft || !w->draft_to_target))
    FAIL(HSPEC_ERR_INVALID_ARG, "W_lm_draft / draft_to_target is NULL (draft_vocab > 0)");
  hspec_drafter* d = new hspec_drafter;
  d->cfg = *cfg;
  d->w = *w;
  *out = d;
  return HSPEC_OK;
}

void hspec_drafter_destroy(hspec_drafter* d) { delete d; }

size_t hspec_step_workspace_size(const hspec_cfg* cfg, int C, int K, int max_pages) {
  if (!cfg || C < 1 || K < 1 || (has_kind(cfg, 'A') && max_pages < 1)) return 0;
  return step_plan(cfg, C, K, max_pages > 0 ? max_pages : 1).total;
}

hspec_status hspec_draft_step(hspec_drafter* dr, const hspec_step_in* in, const hspec_step_out* out,
                              void* workspace, size_t ws_bytes, void* stream) {
  if (!dr || !in || !out) FAIL(HSPEC_ERR_INVALID_ARG, "drafter, in and out must be non-NULL");
  const hspec_cfg* c = &dr->cfg;
  const hspec_model_weights& W = dr->w;
  const int C = in->C, K = in->K, d = c->d_model;
  if (C < 1 || K < 1 || K > 64) FAIL(HSPEC_ERR_UNSUPPORTED, "C=%d K=%d (need C >= 1, 1 <= K <= 64)", C, K);
  const bool ssm = has_kind(c, 'M'), att = has_kind(c, 'A');
  hspec_status st;
  if (ssm && (st = validate_ssd_shape(c, K))) return st;
  if (ssm && !in->h_last) FAIL(HSPEC_ERR_INVALID_ARG, "h_last is NULL");
  if (c->vocab > 0 && (!in->tokens || !out->draft_tokens))
    FAIL(HSPEC_ERR_INVALID_ARG, "tokens and draft_tokens are required with an LM head");
  if (c->vocab == 0 && !in->x_in) FAIL(HSPEC_ERR_INVALID_ARG, "x_in is required without an LM head");
  int max_pages = 1, n_att = 0;
  if (att) {
    if (!in->ctx_lens) FAIL(HSPEC_ERR_INVALID_ARG, "ctx_lens is NULL");
    const char* why = "";
    if (!attn_supported(c->dtype, K, c->n_q_heads / c->n_kv_heads, c->head_dim, &why))
      FAIL(HSPEC_ERR_UNSUPPORTED, "attention: %s", why);
    for (int i = 0; i < c->n_layers; ++i) {
      if (c->layer_kinds[i] != 'A') continue;
      if ((st = validate_kv(c, &in->kv[n_att]))) return st;
      if (in->kv[n_att].max_pages > max_pages) max_pages = in->kv[n_att].max_pages;
      ++n_att;
    }
  }
  const StepPlan sp = step_plan(c, C, K, max_pages);
  if (!workspace || ((uintptr_t)workspace & 255) || ws_bytes < sp.total)
    FAIL(HSPEC_ERR_WORKSPACE, "draft step needs a 256-byte aligned workspace of %zu bytes (got %zu)", sp.total,
         ws_bytes);

  cudaStream_t s = (cudaStream_t)stream;
  uint8_t* ws = (uint8_t*)workspace;
  const int M = C * K;
  StepPdl pdl_scope(M);
  const int dtype = c->dtype;
  const float eps = c->norm_eps;
  const int H = c->n_ssm_heads, P = c->ssm_head_dim, N = c->d_state, HP = H * P;
  const long HPN = (long)HP * N;
  const int n_in = 2 * HP + 2 * N + H;
  const int Hq = c->n_q_heads, Hkv = c->n_kv_heads, Dh = c->head_dim;
  const int n_qkv = (Hq + 2 * Hkv) * Dh;
  const size_t E = elem_bytes(c);
  float* x = (float*)(ws + sp.x);
  uint8_t* xn = ws + sp.xn;
  uint8_t* big = ws + sp.big;
  float* y = (float*)(ws + sp.y);
  uint8_t* g = ws + sp.g;
  float* h0 = (float*)(ws + sp.h0);
  int* err = device_error_word();
  if (sp.gmax_tiles > 0 && cudaMemsetAsync(ws + sp.gcnt, 0, (size_t)sp.gmax_tiles * sp.gcnt_sites * 4, s) != cudaSuccess)
    FAIL(HSPEC_ERR_CUDA, "clearing the GEMM tile counters failed");
  // the projection and MLP GEMMs may split K over the step workspace
  int site = 0;  // the K-cut GEMM calls take the counter slices in turn
  auto split = [&](GemmArgs ga) {
    ga.wait_ns = wait_ns(c);
    ga.part = (float*)(ws + sp.gpart);
    ga.tile_cnt = site < sp.gcnt_sites ? (int*)(ws + sp.gcnt) + (size_t)site * sp.gmax_tiles : nullptr;
    ++site;
    ga.part_bytes = sp.gpart_bytes, ga.max_tiles = sp.gmax_tiles;
    return ga;
  };

  {
    ProfScope p("embed", s);
    if (c->vocab > 0) embed_rows(dtype, in->tokens, W.W_lm, c->vocab, x, M, d, err, s);
    else rows_to_f32(dtype, in->x_in, x, (long)M * d, s);
  }
  // RoPE: in the attention projections' epilogue (bf16, head dim 64 or 128, no split-K),
  // from one (cos, sin) table per step shared by every attention layer; else the row
  // kernel after each projection
  const bool rope = att && (c->flags & HSPEC_FLAG_ROPE) != 0;
  const bool rope_fused = rope && gemm_rope_fusable(dtype, M, n_qkv, d, Dh);
  if (rope_fused) {
    ProfScope p("rope", s);
    rope_table((float2*)(ws + sp.rope), in->ctx_lens, C, K, Dh, c->rope_theta, s);
  }

  int ai = 0;
  for (int li = 0; li < c->n_layers; ++li) {
    const hspec_layer_weights& L = W.layers[li];
    {
      ProfScope p("rmsnorm", s);
      rmsnorm_rows(dtype, x, L.norm, xn, M, d, eps, s);
    }
    if (c->layer_kinds[li] == 'M') {
      // in_proj -> [z | x | B | C | dt_raw]
      {
        ProfScope p("in_proj", s);
        if (!gemm(dtype, kEpiStore, split(gemm_args(M, n_in, d, xn, d, L.W_in, d, big, n_in)), s))
          return HSPEC_ERR_UNSUPPORTED;
      }
      SsdArgs a = {};
      a.C = C, a.K = K, a.H = H, a.P = P, a.N = N, a.Q = ssd_chunk_len(c, K);
      a.x = big + (size_t)HP * E, a.x_rs = n_in;
      a.dt = big + (size_t)(2 * HP + 2 * N) * E, a.dt_rs = n_in, a.dt_bias = L.dt_bias;
      a.A = L.A, a.D = L.D;
      a.B = big + (size_t)(2 * HP) * E, a.Cm = big + (size_t)(2 * HP + N) * E, a.bc_rs = n_in;
      a.y = y, a.y_rs = HP, a.hK = nullptr;
      a.wait_ns = wait_ns(c);
      if (step_fuses_inject(c)) {
        // y = the scan from a zero state (in-block terms, D x), then the injection GEMM
        // adds exp(cum_t) C_t . h0 from its accumulator: h0 = W_inj h_last is never stored
        a.h0 = nullptr;
        {
          ProfScope p("ssd_scan", s);
          ssd_scan(dtype, a, s);
        }
        GemmArgs gi = gemm_args(C, (int)HPN, d, in->h_last, d, L.W_inj, d, nullptr, 0);
        gi.ssd.K = K, gi.ssd.P = P, gi.ssd.N = N;
        gi.ssd.Cm = a.Cm, gi.ssd.c_rs = n_in;
        gi.ssd.dt_raw = a.dt, gi.ssd.dt_rs = n_in, gi.ssd.dt_bias = L.dt_bias, gi.ssd.A = L.A;
        gi.ssd.y = y, gi.ssd.y_rs = HP;
        gi.wait_ns = wait_ns(c);
        {
          ProfScope p("inject", s);
          if (!gemm(dtype, kEpiSsdRead, gi, s)) return HSPEC_ERR_UNSUPPORTED;
        }
      } else {
        // injected initial state h0 = W_inj h_last, stored, then the scan from it
        GemmArgs gi = gemm_args(C, (int)HPN, d, in->h_last, d, L.W_inj, d, h0, HPN);
        gi.out_f32 = true;
        gi.wait_ns = wait_ns(c);
        {
          ProfScope p("inject", s);
          if (!gemm(dtype, kEpiStore, gi, s)) return HSPEC_ERR_UNSUPPORTED;
        }
        a.h0 = h0;
        {
          ProfScope p("ssd_scan", s);
          ssd_scan(dtype, a, s);
        }
      }
      {
        ProfScope p("gated_norm", s);
        gated_rmsnorm_rows(dtype, y, big, n_in, L.gnorm, g, M, HP, eps, (c->flags & HSPEC_FLAG_GATE) != 0, s);
      }
      {
        ProfScope p("out_proj", s);
        if (!gemm(dtype, kEpiResid, split(gemm_args(M, d, HP, g, HP, L.W_out, HP, x, d)), s))
          return HSPEC_ERR_UNSUPPORTED;
      }
    } else {
      // q, k, v projections; RoPE on q and the block keys in the GEMM's epilogue where the
      // tensor-core GEMM can take it (the step's (cos, sin) table is written once, below the
      // embedding), else by the row kernel after it
      {
        ProfScope p("qkv_proj", s);
        GemmArgs gq = split(gemm_args(M, n_qkv, d, xn, d, L.W_qkv, d, big, n_qkv));
        if (rope_fused) gq.rope = {(const float2*)(ws + sp.rope), Dh, (Hq + Hkv) * Dh};
        if (!gemm(dtype, rope_fused ? kEpiRope : kEpiStore, gq, s)) return HSPEC_ERR_UNSUPPORTED;
      }
      if (rope && !rope_fused) {
        ProfScope p("rope", s);
        rope_rows(dtype, big, n_qkv, in->ctx_lens, C, K, Hq + Hkv, Dh, c->rope_theta, s);
      }
      const hspec_kv_view* kv = &in->kv[ai++];
      AttnPlan ap = attn_plan(c, C, K, kv->max_pages);
      AttnArgs a = attn_args(c, ap, kv, in->ctx_lens, C, K, ws + sp.attn);
      a.q = big, a.q_rs = n_qkv;
      a.kb = big + (size_t)Hq * Dh * E, a.kb_rs = n_qkv;
      a.vb = big + (size_t)(Hq + Hkv) * Dh * E, a.vb_rs = n_qkv;
      a.out = g, a.o_rs = (long)Hq * Dh;
      {
        ProfScope p("attn_paged", s);
        if (!attn_paged(dtype, a, s)) return HSPEC_ERR_UNSUPPORTED;
      }
      {
        ProfScope p("o_proj", s);
        if (!gemm(dtype, kEpiResid, split(gemm_args(M, d, Hq * Dh, g, (long)Hq * Dh, L.W_o, (long)Hq * Dh, x, d)), s))
          return HSPEC_ERR_UNSUPPORTED;
      }
    }
    if (c->d_ff > 0) {
      const int F = c->d_ff;
      {
        ProfScope p("rmsnorm", s);
        rmsnorm_rows(dtype, x, L.mlp_norm, xn, M, d, eps, s);
      }
      GemmArgs gs = gemm_args(M, F, d, xn, d, L.W_gate, d, big, F);
      gs.B2 = L.W_up;
      {
        ProfScope p("mlp_gate_up", s);
        if (!gemm(dtype, kEpiSwiGLU, split(gs), s)) return HSPEC_ERR_UNSUPPORTED;
      }
      {
        ProfScope p("mlp_down", s);
        if (!gemm(dtype, kEpiResid, split(gemm_args(M, d, F, big, F, L.W_down, F, x, d)), s))
          return HSPEC_ERR_UNSUPPORTED;
      }
    }
    if (out->layer_hidden)
      cudaMemcpyAsync(out->layer_hidden + (size_t)li * M * d, x, (size_t)M * d * 4, cudaMemcpyDeviceToDevice, s);
  }
  if (c->vocab > 0) {
    {
      ProfScope p("rmsnorm", s);
      rmsnorm_rows(dtype, x, W.final_norm, xn, M, d, eps, s);
    }
    if (out->final_normed) cudaMemcpyAsync(out->final_normed, xn, (size_t)M * d * E, cudaMemcpyDeviceToDevice, s);
    const bool reduced = c->draft_vocab > 0;
    GemmArgs ga = gemm_args(M, reduced ? c->draft_vocab : c->vocab, d, xn, d, reduced ? W.W_lm_draft : W.W_lm, d,
                            nullptr, 0);
    ga.pval = (float*)(ws + sp.pval);
    ga.pidx = (int32_t*)(ws + sp.pidx);
    ga.n_parts = sp.n_parts;
    ga.wait_ns = wait_ns(c);
    {
      ProfScope p("lm_head_argmax", s);
      if (!gemm(dtype, kEpiArgmax, ga, s)) return HSPEC_ERR_UNSUPPORTED;
    }
    {
      ProfScope p("argmax_reduce", s);
      argmax_reduce(ga.pval, ga.pidx, M, sp.n_parts, out->draft_tokens, out->top_logit,
                    reduced ? W.draft_to_target : nullptr, c->vocab, err, s);
    }
  }
  if (out->hidden) cudaMemcpyAsync(out->hidden, x, (size_t)M * d * 4, cudaMemcpyDeviceToDevice, s);
  return check_launch("hspec_draft_step");
}

}  // extern "C"
