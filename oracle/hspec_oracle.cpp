// CPU oracle of the H-Spec block-parallel draft step -- TEST INFRASTRUCTURE ONLY.
// See hspec_oracle.h for what each entry computes and where it comes from.
// Only tests, the package smoke check and the benchmark's CPU-baseline leg use it.
// Parallel loops (OpenMP) only split independent output elements across threads;
// every individual sum runs in its natural index order, in double.
#include "hspec_oracle.h"

#include <cmath>
#include <cstdint>
#include <cstring>
#include <vector>

namespace {

double load(const void* p, int type, size_t i) {
  if (type == ORACLE_F32) return (double)((const float*)p)[i];
  uint32_t bits = (uint32_t)((const uint16_t*)p)[i] << 16;  // bf16 = upper half of a float
  float f;
  std::memcpy(&f, &bits, 4);
  return (double)f;
}

// bf16 keeps 8 significant bits (1 implicit + 7 stored) with float's exponent range.
double bf16_round(double x) {
  if (!std::isfinite(x) || x == 0.0) return x;
  int e;
  std::frexp(x, &e);                       // |x| = m 2^e, m in [0.5, 1)
  int quantum = (e - 1 < -126) ? -133 : e - 8;  // subnormal range: fixed spacing 2^-133
  double y = std::ldexp(std::nearbyint(std::ldexp(x, -quantum)), quantum);  // ties to even
  const double kMax = 3.38953138925153547590470800371487866880e38;  // (2 - 2^-7) 2^127
  if (std::fabs(y) > kMax) y = x > 0 ? INFINITY : -INFINITY;
  return y;
}

double softplus(double v) { return v > 30.0 ? v : std::log1p(std::exp(v)); }
double silu(double v) { return v / (1.0 + std::exp(-v)); }

// ---------------------------------------------------------------- projections
// out[t][r] = sum_j W[r][j] a[t][j] for t < T, r < R (W row-major [R, n]).
void matvec_rows(int T, int R, int n, const void* W, int w_type, const double* a, double* out) {
#pragma omp parallel for schedule(static)
  for (int r = 0; r < R; ++r) {
    for (int t = 0; t < T; ++t) {
      double s = 0.0;
      for (int j = 0; j < n; ++j) s += load(W, w_type, (size_t)r * n + j) * a[(size_t)t * n + j];
      out[(size_t)t * R + r] = s;
    }
  }
}

void rmsnorm_row(int n, const double* x, const float* w, double eps, double* out) {
  double ss = 0.0;
  for (int i = 0; i < n; ++i) ss += x[i] * x[i];
  double inv = 1.0 / std::sqrt(ss / n + eps);
  for (int i = 0; i < n; ++i) out[i] = x[i] * inv * (double)w[i];
}

// Rotate-half ("neox") rotary embedding: pairs (i, i + D/2) turn by pos * theta^(-2i/D).
void rope_vec(int D, double theta, long pos, const double* v, double* out) {
  int half = D / 2;
  for (int i = 0; i < half; ++i) {
    double ang = (double)pos * std::pow(theta, -2.0 * i / D);
    double c = std::cos(ang), s = std::sin(ang);
    double a = v[i], b = v[i + half];
    out[i] = a * c - b * s;
    out[i + half] = a * s + b * c;
  }
}

// ---------------------------------------------------------------- SSD recurrence
// One request, sequential over t (Mamba-2 recurrence written out):
//   h <- exp(dt_t A_h) h + dt_t x_t[h] B_t^T   ([P,N] per head)
//   y_t[h][p] = sum_n C_t[n] h[p][n] + D_h x_t[h][p]
// x [K][H][P], dt [K][H], B/Cm [K][N], h0 [H][P][N] (NULL = zero state).
void ssd_one_request(int K, int H, int P, int N, const double* x, const double* dt,
                     const double* A, const double* B, const double* Cm, const double* Dv,
                     const double* h0, double* y, double* hK) {
  std::vector<double> h((size_t)P * N);
  for (int hh = 0; hh < H; ++hh) {
    for (size_t i = 0; i < h.size(); ++i) h[i] = h0 ? h0[(size_t)hh * P * N + i] : 0.0;
    for (int t = 0; t < K; ++t) {
      double d_t = dt[(size_t)t * H + hh];
      double decay = std::exp(d_t * A[hh]);
      for (int p = 0; p < P; ++p) {
        double xv = x[((size_t)t * H + hh) * P + p];
        for (int n = 0; n < N; ++n) {
          double& s = h[(size_t)p * N + n];
          s = decay * s + d_t * xv * B[(size_t)t * N + n];
        }
      }
      for (int p = 0; p < P; ++p) {
        double acc = 0.0;
        for (int n = 0; n < N; ++n) acc += Cm[(size_t)t * N + n] * h[(size_t)p * N + n];
        y[((size_t)t * H + hh) * P + p] = acc + Dv[hh] * x[((size_t)t * H + hh) * P + p];
      }
    }
    if (hK)
      for (size_t i = 0; i < h.size(); ++i) hK[(size_t)hh * P * N + i] = h[i];
  }
}

// ---------------------------------------------------------------- attention
// Dense softmax attention of K block queries over keys[0..T) of one request,
// GQA: query head h reads kv head h / (Hq / Hkv).  Keys/values are [T][Hkv][D];
// the last K of them are the block's own keys.  With causal_block, block query j
// sees block key i only when i <= j.  q and out are [K][Hq][D].
void attend_one_request(int K, int Hq, int Hkv, int D, int ctx, const double* q, const double* keys,
                        const double* vals, int causal_block, double* out) {
  int T = ctx + K;
  int G = Hq / Hkv;
  double scale = 1.0 / std::sqrt((double)D);
#pragma omp parallel for collapse(2) schedule(static)
  for (int j = 0; j < K; ++j) {
    for (int h = 0; h < Hq; ++h) {
      int g = h / G;
      std::vector<double> s(T);
      int visible = causal_block ? ctx + j + 1 : T;
      double m = -INFINITY;
      for (int t = 0; t < visible; ++t) {
        double acc = 0.0;
        for (int e = 0; e < D; ++e)
          acc += q[((size_t)j * Hq + h) * D + e] * keys[((size_t)t * Hkv + g) * D + e];
        s[t] = acc * scale;
        if (s[t] > m) m = s[t];
      }
      double l = 0.0;
      for (int t = 0; t < visible; ++t) {
        s[t] = std::exp(s[t] - m);
        l += s[t];
      }
      for (int e = 0; e < D; ++e) {
        double acc = 0.0;
        for (int t = 0; t < visible; ++t) acc += s[t] * vals[((size_t)t * Hkv + g) * D + e];
        out[((size_t)j * Hq + h) * D + e] = acc / l;
      }
    }
  }
}

// Copies request c's context out of the pool: token t lives in page
// page_table[c][t / page] at slot t % page.  Returns false on a bad page id.
bool gather_context(int c, int ctx, int Hkv, int D, int page, const void* k_pool,
                    const void* v_pool, int dtype, int num_pages, const int32_t* page_table,
                    int max_pages, double* keys, double* vals) {
  if (ctx < 0 || ctx > max_pages * page) return false;
  size_t row = (size_t)Hkv * D;
  for (int t = 0; t < ctx; ++t) {
    int32_t pg = page_table[(size_t)c * max_pages + t / page];
    if (pg < 0 || pg >= num_pages) return false;
    size_t src = ((size_t)pg * page + t % page) * row;
    for (size_t e = 0; e < row; ++e) {
      keys[(size_t)t * row + e] = load(k_pool, dtype, src + e);
      vals[(size_t)t * row + e] = load(v_pool, dtype, src + e);
    }
  }
  return true;
}

// logits[r][v] = sum_j W_lm[v][j] a[r][j]; argmax with the lowest id winning a tie,
// plus the top logit and the largest logit among the other ids.
void lm_head_argmax(int rows, int d, int V, const double* a, const void* W_lm, int w_type,
                    int32_t* argmax, double* top1, double* top2) {
  std::vector<double> logits((size_t)rows * V);
  matvec_rows(rows, V, d, W_lm, w_type, a, logits.data());
  for (int r = 0; r < rows; ++r) {
    const double* lg = logits.data() + (size_t)r * V;
    int best = 0;
    for (int v = 1; v < V; ++v)
      if (lg[v] > lg[best]) best = v;  // strict: the lowest id wins a tie
    double second = -INFINITY;
    for (int v = 0; v < V; ++v)
      if (v != best && lg[v] > second) second = lg[v];
    argmax[r] = best;
    if (top1) top1[r] = lg[best];
    if (top2) top2[r] = second;
  }
}

}  // namespace

extern "C" {

double oracle_bf16_round(double x) { return bf16_round(x); }

void oracle_bf16_round_array(long n, const double* in, double* out) {
  for (long i = 0; i < n; ++i) out[i] = bf16_round(in[i]);
}

void oracle_inject(int HPN, int d, const void* W_inj, int w_type, const void* h_last, int h_type,
                   int C, double* h0) {
  std::vector<double> a((size_t)C * d);
  for (size_t i = 0; i < a.size(); ++i) a[i] = load(h_last, h_type, i);
  matvec_rows(C, HPN, d, W_inj, w_type, a.data(), h0);
}

void oracle_ssd_scan(int C, int K, int H, int P, int N, const void* x, int x_type, const float* dt,
                     const float* A, const void* B, const void* Cm, int bc_type, const float* D,
                     const float* h0, double* y, double* hK) {
  std::vector<double> Ad(H), Dd(H);
  for (int h = 0; h < H; ++h) Ad[h] = A[h], Dd[h] = D[h];
#pragma omp parallel for schedule(dynamic)
  for (int c = 0; c < C; ++c) {
    size_t nx = (size_t)K * H * P, nb = (size_t)K * N, ns = (size_t)H * P * N;
    std::vector<double> xd(nx), dtd((size_t)K * H), Bd(nb), Cd(nb), h0d(h0 ? ns : 0);
    for (size_t i = 0; i < nx; ++i) xd[i] = load(x, x_type, (size_t)c * nx + i);
    for (size_t i = 0; i < (size_t)K * H; ++i) dtd[i] = dt[(size_t)c * K * H + i];
    for (size_t i = 0; i < nb; ++i) {
      Bd[i] = load(B, bc_type, (size_t)c * nb + i);
      Cd[i] = load(Cm, bc_type, (size_t)c * nb + i);
    }
    for (size_t i = 0; i < h0d.size(); ++i) h0d[i] = h0[(size_t)c * ns + i];
    ssd_one_request(K, H, P, N, xd.data(), dtd.data(), Ad.data(), Bd.data(), Cd.data(), Dd.data(),
                    h0 ? h0d.data() : nullptr, y + (size_t)c * nx, hK ? hK + (size_t)c * ns : nullptr);
  }
}

int oracle_attn_paged(int C, int K, int Hq, int Hkv, int D, int page, const void* q,
                      const void* k_pool, const void* v_pool, int dtype, int num_pages,
                      const int32_t* page_table, int max_pages, const int32_t* ctx_lens,
                      const void* k_blk, const void* v_blk, int causal_block, double* out) {
  size_t row = (size_t)Hkv * D, qn = (size_t)K * Hq * D;
  for (int c = 0; c < C; ++c) {
    int ctx = ctx_lens[c];
    if (ctx < 0 || ctx > max_pages * page) return -1;
    std::vector<double> keys((size_t)(ctx + K) * row), vals((size_t)(ctx + K) * row), qd(qn);
    if (!gather_context(c, ctx, Hkv, D, page, k_pool, v_pool, dtype, num_pages, page_table,
                        max_pages, keys.data(), vals.data()))
      return -1;
    for (size_t e = 0; e < (size_t)K * row; ++e) {
      keys[(size_t)ctx * row + e] = load(k_blk, dtype, (size_t)c * K * row + e);
      vals[(size_t)ctx * row + e] = load(v_blk, dtype, (size_t)c * K * row + e);
    }
    for (size_t e = 0; e < qn; ++e) qd[e] = load(q, dtype, (size_t)c * qn + e);
    attend_one_request(K, Hq, Hkv, D, ctx, qd.data(), keys.data(), vals.data(), causal_block,
                       out + (size_t)c * qn);
  }
  return 0;
}

void oracle_attn_contiguous(int C, int K, int Hq, int Hkv, int D, const void* q,
                            const void* k_ctx, const void* v_ctx, int dtype, int max_ctx,
                            const int32_t* ctx_lens, const void* k_blk, const void* v_blk,
                            int causal_block, double* out) {
  size_t row = (size_t)Hkv * D, qn = (size_t)K * Hq * D;
  for (int c = 0; c < C; ++c) {
    int ctx = ctx_lens[c];
    std::vector<double> keys((size_t)(ctx + K) * row), vals((size_t)(ctx + K) * row), qd(qn);
    for (size_t e = 0; e < (size_t)ctx * row; ++e) {
      keys[e] = load(k_ctx, dtype, (size_t)c * max_ctx * row + e);
      vals[e] = load(v_ctx, dtype, (size_t)c * max_ctx * row + e);
    }
    for (size_t e = 0; e < (size_t)K * row; ++e) {
      keys[(size_t)ctx * row + e] = load(k_blk, dtype, (size_t)c * K * row + e);
      vals[(size_t)ctx * row + e] = load(v_blk, dtype, (size_t)c * K * row + e);
    }
    for (size_t e = 0; e < qn; ++e) qd[e] = load(q, dtype, (size_t)c * qn + e);
    attend_one_request(K, Hq, Hkv, D, ctx, qd.data(), keys.data(), vals.data(), causal_block,
                       out + (size_t)c * qn);
  }
}

void oracle_rmsnorm(int rows, int n, const double* x, const float* w, double eps, double* out) {
  for (int r = 0; r < rows; ++r) rmsnorm_row(n, x + (size_t)r * n, w, eps, out + (size_t)r * n);
}

void oracle_rope(int D, double theta, long pos, const double* v, double* out) {
  rope_vec(D, theta, pos, v, out);
}

void oracle_lm_head_argmax(int rows, int d, int V, const void* hn, int hn_type, const void* W_lm,
                           int w_type, int32_t* argmax, double* top1, double* top2) {
  std::vector<double> a((size_t)rows * d);
  for (size_t i = 0; i < a.size(); ++i) a[i] = load(hn, hn_type, i);
  lm_head_argmax(rows, d, V, a.data(), W_lm, w_type, argmax, top1, top2);
}

// Greedy verification: the target's argmax per row, the longest prefix of drafts that
// matches it, and the target's token after that prefix.
void oracle_verify_greedy(int C, int K, int V, const void* logits, int ltype, const int32_t* drafts,
                          int32_t* accepted, int32_t* next_token, int32_t* ctx_lens) {
  for (int c = 0; c < C; ++c) {
    std::vector<int32_t> t(K + 1);
    for (int j = 0; j <= K; ++j) {
      const size_t base = ((size_t)c * (K + 1) + j) * V;
      int32_t best = -1;
      double bv = 0.0;
      for (int v = 0; v < V; ++v) {
        const double x = load(logits, ltype, base + v);
        if (std::isnan(x)) continue;
        if (best < 0 || x > bv) best = v, bv = x;
      }
      t[j] = best;
    }
    int a = 0;
    while (a < K && drafts[(size_t)c * K + a] == t[a]) ++a;
    accepted[c] = a;
    next_token[c] = t[a];
    if (ctx_lens) ctx_lens[c] += a + 1;
  }
}

// One draft step.  Per layer (pre-norm residual blocks):
//   M: xn = R(rmsnorm(x) w); [z, xs, B, C, dt_raw] = R(xn W_in^T); dt = softplus(dt_raw + dt_bias);
//      h0 = W_inj h_last (reshaped [H,P,N]); y = SSD recurrence from h0;
//      g = R(rmsnorm(y * silu(z)) w_g) (or R(y) without the gate); x += g W_out^T
//   A: xn = R(rmsnorm(x) w); [q, k, v] = R(xn W_qkv^T); q, k = R(rope(., ctx_c + j));
//      o = R(attention over the paged context then the block keys); x += o W_o^T
//   MLP (d_ff > 0): xn = R(rmsnorm(x) w_m); a = R(silu(xn W_g^T) * (xn W_u^T)); x += a W_d^T
// then hn = R(rmsnorm(x) w_f), logits = hn W_lm^T, draft token = argmax.
// R() rounds to bf16 in a bf16 step and is the identity in an fp32 step.
int oracle_draft_step(const oracle_cfg* cfg, const oracle_layer* layers, oracle_step* io) {
  const int d = cfg->d, K = io->K, C = io->C, dtype = cfg->dtype;
  const int H = cfg->H, P = cfg->P, N = cfg->N, HP = H * P, HPN = H * P * N;
  const int Hq = cfg->Hq, Hkv = cfg->Hkv, Dh = cfg->D;
  const int n_in = 2 * HP + 2 * N + H, n_qkv = (Hq + 2 * Hkv) * Dh;
  auto R = [dtype](double v) { return dtype == ORACLE_BF16 ? bf16_round(v) : v; };

  for (int c = 0; c < C; ++c) {
    const int ctx = io->ctx_lens[c];
    std::vector<double> x((size_t)K * d), xn((size_t)K * d), tmp;
    // block input: embedding of the block tokens (tied LM head) or the direct input
    for (int j = 0; j < K; ++j)
      for (int e = 0; e < d; ++e)
        x[(size_t)j * d + e] = cfg->vocab > 0
            ? load(io->W_lm, dtype, (size_t)io->tokens[(size_t)c * K + j] * d + e)
            : load(io->x_in, io->x_in_type, ((size_t)c * K + j) * d + e);
    std::vector<double> hl(d);
    for (int e = 0; e < d; ++e) hl[e] = load(io->h_last, dtype, (size_t)c * d + e);

    for (int li = 0; li < cfg->n_layers; ++li) {
      const oracle_layer& L = layers[li];
      for (int j = 0; j < K; ++j) {
        rmsnorm_row(d, &x[(size_t)j * d], L.norm, cfg->eps, &xn[(size_t)j * d]);
        for (int e = 0; e < d; ++e) xn[(size_t)j * d + e] = R(xn[(size_t)j * d + e]);
      }
      if (cfg->kinds[li] == 'M') {
        std::vector<double> zx((size_t)K * n_in);
        matvec_rows(K, n_in, d, L.W_in, dtype, xn.data(), zx.data());
        for (auto& v : zx) v = R(v);
        std::vector<double> xs((size_t)K * HP), dt((size_t)K * H), Bm((size_t)K * N),
            Cm((size_t)K * N), A(H), Dv(H), h0(HPN), y((size_t)K * HP);
        for (int j = 0; j < K; ++j) {
          const double* row = &zx[(size_t)j * n_in];
          for (int i = 0; i < HP; ++i) xs[(size_t)j * HP + i] = row[HP + i];
          for (int n = 0; n < N; ++n) {
            Bm[(size_t)j * N + n] = row[2 * HP + n];
            Cm[(size_t)j * N + n] = row[2 * HP + N + n];
          }
          for (int h = 0; h < H; ++h)
            dt[(size_t)j * H + h] = softplus(row[2 * HP + 2 * N + h] + (double)L.dt_bias[h]);
        }
        for (int h = 0; h < H; ++h) A[h] = L.A[h], Dv[h] = L.D[h];
        matvec_rows(1, HPN, d, L.W_inj, dtype, hl.data(), h0.data());  // injected initial state
        ssd_one_request(K, H, P, N, xs.data(), dt.data(), A.data(), Bm.data(), Cm.data(), Dv.data(),
                        h0.data(), y.data(), nullptr);
        std::vector<double> g((size_t)K * HP);
        for (int j = 0; j < K; ++j) {
          if (cfg->use_gate) {
            std::vector<double> gz(HP);
            for (int i = 0; i < HP; ++i)
              gz[i] = y[(size_t)j * HP + i] * silu(zx[(size_t)j * n_in + i]);
            rmsnorm_row(HP, gz.data(), L.gnorm, cfg->eps, &g[(size_t)j * HP]);
          } else {
            for (int i = 0; i < HP; ++i) g[(size_t)j * HP + i] = y[(size_t)j * HP + i];
          }
          for (int i = 0; i < HP; ++i) g[(size_t)j * HP + i] = R(g[(size_t)j * HP + i]);
        }
        tmp.assign((size_t)K * d, 0.0);
        matvec_rows(K, d, HP, L.W_out, dtype, g.data(), tmp.data());
        for (size_t i = 0; i < x.size(); ++i) x[i] += tmp[i];
      } else {
        std::vector<double> qkv((size_t)K * n_qkv);
        matvec_rows(K, n_qkv, d, L.W_qkv, dtype, xn.data(), qkv.data());
        for (auto& v : qkv) v = R(v);
        std::vector<double> q((size_t)K * Hq * Dh), kb((size_t)K * Hkv * Dh), vb((size_t)K * Hkv * Dh);
        std::vector<double> rot(Dh);
        for (int j = 0; j < K; ++j) {
          const double* row = &qkv[(size_t)j * n_qkv];
          long pos = (long)ctx + j;
          for (int h = 0; h < Hq; ++h) {
            const double* src = row + (size_t)h * Dh;
            double* dst = &q[((size_t)j * Hq + h) * Dh];
            if (cfg->use_rope) rope_vec(Dh, cfg->rope_theta, pos, src, rot.data());
            for (int e = 0; e < Dh; ++e) dst[e] = cfg->use_rope ? R(rot[e]) : src[e];
          }
          for (int g = 0; g < Hkv; ++g) {
            const double* src = row + (size_t)(Hq + g) * Dh;
            double* dst = &kb[((size_t)j * Hkv + g) * Dh];
            if (cfg->use_rope) rope_vec(Dh, cfg->rope_theta, pos, src, rot.data());
            for (int e = 0; e < Dh; ++e) dst[e] = cfg->use_rope ? R(rot[e]) : src[e];
            for (int e = 0; e < Dh; ++e)
              vb[((size_t)j * Hkv + g) * Dh + e] = row[(size_t)(Hq + Hkv + g) * Dh + e];
          }
        }
        size_t krow = (size_t)Hkv * Dh;
        std::vector<double> keys((size_t)(ctx + K) * krow), vals((size_t)(ctx + K) * krow);
        if (!gather_context(c, ctx, Hkv, Dh, cfg->page, L.k_pool, L.v_pool, dtype, L.num_pages,
                            L.page_table, L.max_pages, keys.data(), vals.data()))
          return -1;
        for (size_t e = 0; e < (size_t)K * krow; ++e) {
          keys[(size_t)ctx * krow + e] = kb[e];
          vals[(size_t)ctx * krow + e] = vb[e];
        }
        std::vector<double> o((size_t)K * Hq * Dh);
        attend_one_request(K, Hq, Hkv, Dh, ctx, q.data(), keys.data(), vals.data(),
                           cfg->causal_block, o.data());
        for (auto& v : o) v = R(v);
        tmp.assign((size_t)K * d, 0.0);
        matvec_rows(K, d, Hq * Dh, L.W_o, dtype, o.data(), tmp.data());
        for (size_t i = 0; i < x.size(); ++i) x[i] += tmp[i];
      }
      if (cfg->d_ff > 0) {
        const int F = cfg->d_ff;
        for (int j = 0; j < K; ++j) {
          rmsnorm_row(d, &x[(size_t)j * d], L.mlp_norm, cfg->eps, &xn[(size_t)j * d]);
          for (int e = 0; e < d; ++e) xn[(size_t)j * d + e] = R(xn[(size_t)j * d + e]);
        }
        std::vector<double> gt((size_t)K * F), up((size_t)K * F);
        matvec_rows(K, F, d, L.W_gate, dtype, xn.data(), gt.data());
        matvec_rows(K, F, d, L.W_up, dtype, xn.data(), up.data());
        for (size_t i = 0; i < gt.size(); ++i) gt[i] = R(silu(gt[i]) * up[i]);
        tmp.assign((size_t)K * d, 0.0);
        matvec_rows(K, d, F, L.W_down, dtype, gt.data(), tmp.data());
        for (size_t i = 0; i < x.size(); ++i) x[i] += tmp[i];
      }
      if (io->layer_out)
        for (size_t i = 0; i < x.size(); ++i)
          io->layer_out[(((size_t)li * C + c) * K) * d + i] = x[i];
    }
    if (io->hidden)
      for (size_t i = 0; i < x.size(); ++i) io->hidden[(size_t)c * K * d + i] = x[i];
    if (cfg->vocab > 0) {
      for (int j = 0; j < K; ++j) {
        rmsnorm_row(d, &x[(size_t)j * d], io->final_norm, cfg->eps, &xn[(size_t)j * d]);
        for (int e = 0; e < d; ++e) xn[(size_t)j * d + e] = R(xn[(size_t)j * d + e]);
      }
      if (io->final_normed)
        for (size_t i = 0; i < xn.size(); ++i) io->final_normed[(size_t)c * K * d + i] = xn[i];
      std::vector<int32_t> am(K);
      std::vector<double> t1(K), t2(K);
      // full head, or the reduced draft head whose row r stands for target token
      // draft_to_target[r] (argmax over the draft rows, lowest row on ties)
      const bool reduced = io->draft_vocab > 0;
      lm_head_argmax(K, d, reduced ? io->draft_vocab : cfg->vocab, xn.data(), reduced ? io->W_lm_draft : io->W_lm,
                     dtype, am.data(), t1.data(), t2.data());
      for (int j = 0; j < K; ++j) {
        if (io->draft_tokens) io->draft_tokens[(size_t)c * K + j] = reduced ? io->draft_to_target[am[j]] : am[j];
        if (io->top1) io->top1[(size_t)c * K + j] = t1[j];
        if (io->top2) io->top2[(size_t)c * K + j] = t2[j];
      }
    }
  }
  return 0;
}

}  // extern "C"
