// gpt2_oracle.cpp -- plain float64 CPU reference of the GPT-2 pre-LN training step.
//
// TEST INFRASTRUCTURE ONLY. Nothing on the product path may call this file: only
// the tests, the package's smoke check and the benchmark's CPU-baseline leg load
// it. It shares no code with the CUDA library (no headers, helpers or tables).
//
// What it computes, with the passages it follows (pages named by title/section):
//  * Embedding x = wte[tok] + wpe[t]: "gpt/docs/LLM.md", Architecture Details /
//    Embedding Layer; "GPT From Scratch", Architecture diagram (wte + wpe).
//  * Pre-LN block x += Attn(LN1(x)); x += MLP(LN2(x)), 4x tanh-GELU MLP:
//    "gpt/docs/LLM.md", Transformer Blocks; "GPT From Scratch", Key decisions
//    (pre-norm, tanh-GELU, 4x); "Genesis", Model Specs (GELU tanh, Pre-LayerNorm).
//  * Causal multi-head attention as the explicit masked softmax; a second, blocked
//    online-softmax formulation is kept only for the check that the two agree:
//    "GPT From Scratch", Key decisions.
//  * Final LN and a bias-free head tied to wte (or a separate head):
//    "gpt/docs/LLM.md", Output Layer; "AxonLM", Key Features (weight tying);
//    "Genesis", Model Specs (untied, 163,009,536 parameters).
//  * Mean next-token cross-entropy over all B*T positions.
//  * AdamW with betas (0.9, 0.95), decay only on >=2-D tensors, global-norm clip
//    1.0: "AxonLM", Training Recipe; "GPT From Scratch", Key decisions.
//  * Init N(0, 0.02), residual projections scaled by 1/sqrt(2L): "AxonLM", Key
//    Features; "GPT From Scratch", Key decisions.
// Readings where the pages are silent, taken here: LN eps 1e-5 with the biased
// variance; Adam eps 1e-8 with bias correction; clip coefficient 1 / (norm + 1e-6)
// capped at 1; padded vocabulary rows excluded from the softmax; the init random
// stream of init_params below.
//
// Parity pins: parity of this file is pinned by tests/test_oracle_*.py against
// numbers the pages print (parameter counts, ln 65 initial loss), closed forms,
// finite differences, invariants and float64 library routines.
#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstdio>
#include <cstring>
#include <string>
#include <vector>
#ifdef _OPENMP
#include <omp.h>
#endif

namespace {

struct Cfg {
  int L, H, C, T, V, tied, qkv_bias;
};

// ---------------------------------------------------------------------------
// Parameter table in canonical order (PyTorch Linear convention W[out][in]).
// ---------------------------------------------------------------------------
struct Tensor {
  std::string name;
  int64_t rows, cols;  // cols == 1 and ndim == 1 for vectors
  int ndim;
  double sigma;        // init std; 0 -> constant init (value `fill`)
  double fill;
  int64_t offset;
};

std::vector<Tensor> tensor_table(const Cfg& c) {
  std::vector<Tensor> t;
  const int64_t C = c.C, F = 4 * (int64_t)c.C;
  const double s = 0.02, sr = 0.02 / std::sqrt(2.0 * c.L);
  auto add = [&](const std::string& n, int64_t r, int64_t cc, int nd, double sg, double fill) {
    t.push_back(Tensor{n, r, cc, nd, sg, fill, 0});
  };
  add("wte", c.V, C, 2, s, 0);
  add("wpe", c.T, C, 2, s, 0);
  for (int l = 0; l < c.L; ++l) {
    std::string p = "h" + std::to_string(l) + ".";
    add(p + "ln1_g", C, 1, 1, 0, 1);
    add(p + "ln1_b", C, 1, 1, 0, 0);
    add(p + "qkv_w", 3 * C, C, 2, s, 0);
    if (c.qkv_bias) add(p + "qkv_b", 3 * C, 1, 1, 0, 0);
    add(p + "ao_w", C, C, 2, sr, 0);
    add(p + "ao_b", C, 1, 1, 0, 0);
    add(p + "ln2_g", C, 1, 1, 0, 1);
    add(p + "ln2_b", C, 1, 1, 0, 0);
    add(p + "fc_w", F, C, 2, s, 0);
    add(p + "fc_b", F, 1, 1, 0, 0);
    add(p + "pj_w", C, F, 2, sr, 0);
    add(p + "pj_b", C, 1, 1, 0, 0);
  }
  add("lnf_g", C, 1, 1, 0, 1);
  add("lnf_b", C, 1, 1, 0, 0);
  if (!c.tied) add("head_w", c.V, C, 2, s, 0);
  int64_t off = 0;
  for (auto& x : t) {
    x.offset = off;
    off += x.rows * x.cols;
  }
  return t;
}

int64_t total_params(const std::vector<Tensor>& t) {
  return t.back().offset + t.back().rows * t.back().cols;
}

// ---------------------------------------------------------------------------
// splitmix64 (S. Vigna): state advance by the golden-ratio increment, then the
// published finaliser. Used only for the init stream (init_params).
// ---------------------------------------------------------------------------
uint64_t splitmix64_at(uint64_t x) {
  uint64_t z = x + 0x9E3779B97F4A7C15ull;
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

// ---------------------------------------------------------------------------
// Building blocks, each the textbook definition in float64.
// ---------------------------------------------------------------------------

// LayerNorm of each row: y = (x - mean) / sqrt(var + eps) * g + b, biased var.
void layernorm_fwd(const double* x, const double* g, const double* b, int64_t N, int C,
                   double* y, double* mean, double* rstd) {
#pragma omp parallel for schedule(static)
  for (int64_t n = 0; n < N; ++n) {
    const double* xr = x + n * C;
    double mu = 0;
    for (int i = 0; i < C; ++i) mu += xr[i];
    mu /= C;
    double var = 0;
    for (int i = 0; i < C; ++i) var += (xr[i] - mu) * (xr[i] - mu);
    var /= C;
    double rs = 1.0 / std::sqrt(var + 1e-5);
    for (int i = 0; i < C; ++i) y[n * C + i] = (xr[i] - mu) * rs * g[i] + b[i];
    mean[n] = mu;
    rstd[n] = rs;
  }
}

// Reverse mode of the above. dx is OVERWRITTEN; dg, db are ACCUMULATED.
// With xh = (x - mean) * rstd and dxh = dy * g:
//   dx = rstd * (dxh - mean(dxh) - xh * mean(dxh * xh)),  dg += sum dy*xh,  db += sum dy.
void layernorm_bwd(const double* dy, const double* x, const double* g, const double* mean,
                   const double* rstd, int64_t N, int C, double* dx, double* dg, double* db) {
#pragma omp parallel for schedule(static)
  for (int64_t n = 0; n < N; ++n) {
    const double* dyr = dy + n * C;
    const double* xr = x + n * C;
    double m1 = 0, m2 = 0;
    for (int i = 0; i < C; ++i) {
      double xh = (xr[i] - mean[n]) * rstd[n];
      double dxh = dyr[i] * g[i];
      m1 += dxh;
      m2 += dxh * xh;
    }
    m1 /= C;
    m2 /= C;
    for (int i = 0; i < C; ++i) {
      double xh = (xr[i] - mean[n]) * rstd[n];
      double dxh = dyr[i] * g[i];
      dx[n * C + i] = rstd[n] * (dxh - m1 - xh * m2);
    }
  }
  // parameter gradients: a plain sum over rows, per column
#pragma omp parallel for schedule(static)
  for (int i = 0; i < C; ++i) {
    double sg = 0, sb = 0;
    for (int64_t n = 0; n < N; ++n) {
      double xh = (x[n * C + i] - mean[n]) * rstd[n];
      sg += dy[n * C + i] * xh;
      sb += dy[n * C + i];
    }
    dg[i] += sg;
    db[i] += sb;
  }
}

// Y[n][o] = sum_k X[n][k] W[o][k] + b[o]   (b may be null)
void linear_fwd(const double* X, const double* W, const double* b, int64_t N, int K, int O, double* Y) {
#pragma omp parallel for schedule(static)
  for (int64_t n = 0; n < N; ++n) {
    const double* xr = X + n * K;
    for (int o = 0; o < O; ++o) {
      const double* wr = W + (int64_t)o * K;
      double s = 0;
      for (int k = 0; k < K; ++k) s += xr[k] * wr[k];
      Y[n * O + o] = s + (b ? b[o] : 0.0);
    }
  }
}

// dX = dY W (overwritten); dW += dY^T X; db += colsum(dY) (db may be null)
void linear_bwd(const double* dY, const double* X, const double* W, int64_t N, int K, int O,
                double* dX, double* dW, double* db) {
#pragma omp parallel for schedule(static)
  for (int64_t n = 0; n < N; ++n) {
    double* dxr = dX + n * K;
    for (int k = 0; k < K; ++k) dxr[k] = 0;
    for (int o = 0; o < O; ++o) {
      double d = dY[n * O + o];
      const double* wr = W + (int64_t)o * K;
      for (int k = 0; k < K; ++k) dxr[k] += d * wr[k];
    }
  }
#pragma omp parallel for schedule(static)
  for (int o = 0; o < O; ++o) {
    double* dwr = dW + (int64_t)o * K;
    double sb = 0;
    for (int64_t n = 0; n < N; ++n) {
      double d = dY[n * O + o];
      sb += d;
      const double* xr = X + n * K;
      for (int k = 0; k < K; ++k) dwr[k] += d * xr[k];
    }
    if (db) db[o] += sb;
  }
}

// GELU, tanh form (Hendrycks & Gimpel): 0.5 u (1 + tanh(sqrt(2/pi) (u + 0.044715 u^3)))
inline double gelu(double u) {
  const double k = std::sqrt(2.0 / M_PI);
  return 0.5 * u * (1.0 + std::tanh(k * (u + 0.044715 * u * u * u)));
}
// its analytic derivative
inline double gelu_grad(double u) {
  const double k = std::sqrt(2.0 / M_PI);
  double inner = k * (u + 0.044715 * u * u * u);
  double th = std::tanh(inner);
  double dinner = k * (1.0 + 3.0 * 0.044715 * u * u);
  return 0.5 * (1.0 + th) + 0.5 * u * (1.0 - th * th) * dinner;
}

// Causal attention over qkv [B*T, 3C] (q | k | v column blocks; head h uses
// columns [h*hd, (h+1)*hd) of each block). out [B*T, C]; lse [B, NH, T].
// mode 0: explicit scores over all keys, future keys set to -inf, then softmax.
// mode 1: keys in blocks of 16 with a running max and sum (online softmax).
void attention_fwd(const double* qkv, int B, int T, int NH, int hd, int mode, double* out, double* lse) {
  const int C = NH * hd;
  const double scale = 1.0 / std::sqrt((double)hd);
#pragma omp parallel for collapse(2) schedule(static)
  for (int b = 0; b < B; ++b)
    for (int h = 0; h < NH; ++h) {
      std::vector<double> s(T), acc(hd);
      for (int i = 0; i < T; ++i) {
        const double* q = qkv + ((int64_t)b * T + i) * 3 * C + h * hd;
        double* o = out + ((int64_t)b * T + i) * C + h * hd;
        if (mode == 0) {
          double mx = -INFINITY;
          for (int j = 0; j < T; ++j) {
            if (j > i) {
              s[j] = -INFINITY;
              continue;
            }
            const double* k = qkv + ((int64_t)b * T + j) * 3 * C + C + h * hd;
            double d = 0;
            for (int e = 0; e < hd; ++e) d += q[e] * k[e];
            s[j] = d * scale;
            mx = std::max(mx, s[j]);
          }
          double den = 0;
          for (int j = 0; j < T; ++j) {
            s[j] = (j > i) ? 0.0 : std::exp(s[j] - mx);
            den += s[j];
          }
          for (int e = 0; e < hd; ++e) acc[e] = 0;
          for (int j = 0; j <= i; ++j) {
            const double* v = qkv + ((int64_t)b * T + j) * 3 * C + 2 * C + h * hd;
            double p = s[j] / den;
            for (int e = 0; e < hd; ++e) acc[e] += p * v[e];
          }
          for (int e = 0; e < hd; ++e) o[e] = acc[e];
          if (lse) lse[((int64_t)b * NH + h) * T + i] = mx + std::log(den);
        } else {
          const int BLK = 16;
          double m = -INFINITY, l = 0;
          for (int e = 0; e < hd; ++e) acc[e] = 0;
          for (int j0 = 0; j0 <= i; j0 += BLK) {
            int j1 = std::min(j0 + BLK, i + 1);
            double bm = -INFINITY;
            for (int j = j0; j < j1; ++j) {
              const double* k = qkv + ((int64_t)b * T + j) * 3 * C + C + h * hd;
              double d = 0;
              for (int e = 0; e < hd; ++e) d += q[e] * k[e];
              s[j] = d * scale;
              bm = std::max(bm, s[j]);
            }
            double mnew = std::max(m, bm);
            double corr = std::exp(m - mnew);  // m = -inf on the first block -> 0
            l *= corr;
            for (int e = 0; e < hd; ++e) acc[e] *= corr;
            for (int j = j0; j < j1; ++j) {
              double p = std::exp(s[j] - mnew);
              l += p;
              const double* v = qkv + ((int64_t)b * T + j) * 3 * C + 2 * C + h * hd;
              for (int e = 0; e < hd; ++e) acc[e] += p * v[e];
            }
            m = mnew;
          }
          for (int e = 0; e < hd; ++e) o[e] = acc[e] / l;
          if (lse) lse[((int64_t)b * NH + h) * T + i] = m + std::log(l);
        }
      }
    }
}

// Reverse mode of causal attention (probabilities recomputed from q, k):
//   dV = P^T dY,  dP = dY V^T,  dS = P o (dP - rowsum(dP o P)),  dQ = dS K / sqrt(hd),
//   dK = dS^T Q / sqrt(hd).  dqkv is OVERWRITTEN.
void attention_bwd(const double* qkv, const double* dout, int B, int T, int NH, int hd, double* dqkv) {
  const int C = NH * hd;
  const double scale = 1.0 / std::sqrt((double)hd);
#pragma omp parallel for collapse(2) schedule(static)
  for (int b = 0; b < B; ++b)
    for (int h = 0; h < NH; ++h) {
      std::vector<double> P((size_t)T * T, 0.0), dS((size_t)T * T, 0.0);
      auto q = [&](int i) { return qkv + ((int64_t)b * T + i) * 3 * C + h * hd; };
      auto k = [&](int j) { return qkv + ((int64_t)b * T + j) * 3 * C + C + h * hd; };
      auto v = [&](int j) { return qkv + ((int64_t)b * T + j) * 3 * C + 2 * C + h * hd; };
      auto dy = [&](int i) { return dout + ((int64_t)b * T + i) * C + h * hd; };
      auto dq = [&](int i) { return dqkv + ((int64_t)b * T + i) * 3 * C + h * hd; };
      auto dk = [&](int j) { return dqkv + ((int64_t)b * T + j) * 3 * C + C + h * hd; };
      auto dv = [&](int j) { return dqkv + ((int64_t)b * T + j) * 3 * C + 2 * C + h * hd; };
      for (int i = 0; i < T; ++i) {
        double mx = -INFINITY;
        for (int j = 0; j <= i; ++j) {
          double d = 0;
          for (int e = 0; e < hd; ++e) d += q(i)[e] * k(j)[e];
          P[(size_t)i * T + j] = d * scale;
          mx = std::max(mx, d * scale);
        }
        double den = 0;
        for (int j = 0; j <= i; ++j) {
          P[(size_t)i * T + j] = std::exp(P[(size_t)i * T + j] - mx);
          den += P[(size_t)i * T + j];
        }
        for (int j = 0; j <= i; ++j) P[(size_t)i * T + j] /= den;
        // dP_ij = dy_i . v_j ; dS = P (dP - sum_j dP P)
        double rs = 0;
        for (int j = 0; j <= i; ++j) {
          double d = 0;
          for (int e = 0; e < hd; ++e) d += dy(i)[e] * v(j)[e];
          dS[(size_t)i * T + j] = d;
          rs += d * P[(size_t)i * T + j];
        }
        for (int j = 0; j <= i; ++j) dS[(size_t)i * T + j] = P[(size_t)i * T + j] * (dS[(size_t)i * T + j] - rs);
      }
      for (int i = 0; i < T; ++i) {
        for (int e = 0; e < hd; ++e) dq(i)[e] = 0;
        for (int j = 0; j <= i; ++j)
          for (int e = 0; e < hd; ++e) dq(i)[e] += dS[(size_t)i * T + j] * k(j)[e] * scale;
      }
      for (int j = 0; j < T; ++j) {
        for (int e = 0; e < hd; ++e) {
          dk(j)[e] = 0;
          dv(j)[e] = 0;
        }
        for (int i = j; i < T; ++i)
          for (int e = 0; e < hd; ++e) {
            dk(j)[e] += dS[(size_t)i * T + j] * q(i)[e] * scale;
            dv(j)[e] += P[(size_t)i * T + j] * dy(i)[e];
          }
      }
    }
}

// Cross-entropy over the first V logits of each row (padding columns are
// storage only). row_loss[n] = logsumexp(z_n) - z_n[target]. If dlogits is
// given, dlogits[n][v] = (softmax(z_n)_v - [v == target]) * scale for v < V and
// 0 for V <= v < ld.  Returns sum_n row_loss[n].
double cross_entropy(const double* logits, int64_t N, int V, int64_t ld, const int32_t* tgt, double scale,
                     double* dlogits, double* row_loss) {
  double total = 0;
#pragma omp parallel for schedule(static) reduction(+ : total)
  for (int64_t n = 0; n < N; ++n) {
    const double* z = logits + n * ld;
    double mx = -INFINITY;
    for (int v = 0; v < V; ++v) mx = std::max(mx, z[v]);
    double den = 0;
    for (int v = 0; v < V; ++v) den += std::exp(z[v] - mx);
    double lse = mx + std::log(den);
    double rl = lse - z[tgt[n]];
    if (row_loss) row_loss[n] = rl;
    total += rl;
    if (dlogits) {
      for (int v = 0; v < V; ++v) dlogits[n * ld + v] = (std::exp(z[v] - lse) - (v == tgt[n] ? 1.0 : 0.0)) * scale;
      for (int64_t v = V; v < ld; ++v) dlogits[n * ld + v] = 0.0;
    }
  }
  return total;
}

// Counting sort of token positions by id (stable: positions ascend within an id).
void token_buckets(const int32_t* tok, int64_t N, int V, int64_t* counts, int64_t* offsets, int32_t* positions) {
  for (int v = 0; v < V; ++v) counts[v] = 0;
  for (int64_t n = 0; n < N; ++n) counts[tok[n]]++;
  int64_t run = 0;
  for (int v = 0; v < V; ++v) {
    offsets[v] = run;
    run += counts[v];
  }
  std::vector<int64_t> cursor(offsets, offsets + V);
  for (int64_t n = 0; n < N; ++n) positions[cursor[tok[n]]++] = (int32_t)n;
}

// x0[b*T + t] = wte[tok[b*T + t]] + wpe[t]: the token row plus the row of its
// position within its own sequence.
void embedding_fwd(const int32_t* tok, const double* wte, const double* wpe, int B, int T, int C, double* x0) {
  for (int b = 0; b < B; ++b)
    for (int t = 0; t < T; ++t) {
      const int64_t n = (int64_t)b * T + t;
      for (int i = 0; i < C; ++i) x0[n * C + i] = wte[(int64_t)tok[n] * C + i] + wpe[(int64_t)t * C + i];
    }
}

// dwte[v] += sum over positions n with tok[n] == v of dx0[n];  dwpe[t] += sum_b dx0[b, t]
void embedding_bwd(const int32_t* tok, const double* dx0, int B, int T, int C, double* dwte, double* dwpe) {
  for (int64_t n = 0; n < (int64_t)B * T; ++n) {
    double* r = dwte + (int64_t)tok[n] * C;
    for (int c = 0; c < C; ++c) r[c] += dx0[n * C + c];
  }
  for (int b = 0; b < B; ++b)
    for (int t = 0; t < T; ++t)
      for (int c = 0; c < C; ++c) dwpe[(int64_t)t * C + c] += dx0[((int64_t)b * T + t) * C + c];
}

// ---------------------------------------------------------------------------
// The model: forward with the caches the backward needs, then the backward.
// ---------------------------------------------------------------------------
struct Model {
  Cfg c;
  std::vector<Tensor> tab;
  int64_t P;
  explicit Model(const Cfg& cfg) : c(cfg), tab(tensor_table(cfg)), P(total_params(tab)) {}

  const Tensor& find(const std::string& n) const {
    for (auto& t : tab)
      if (t.name == n) return t;
    std::fprintf(stderr, "oracle: no tensor %s\n", n.c_str());
    std::abort();
  }
  template <class Ptr>
  Ptr at(Ptr base, const std::string& n) const {
    return base + find(n).offset;
  }
  template <class Ptr>
  Ptr at_opt(Ptr base, const std::string& n) const {
    for (auto& t : tab)
      if (t.name == n) return base + t.offset;
    return nullptr;
  }
};

struct Cache {
  int B, T;
  std::vector<double> x0;                        // [N, C] embedding output
  std::vector<std::vector<double>> xin, h1, m1, r1, qkv, att, xmid, h2, m2, r2, u, a;
  std::vector<double> xL, xf, mf, rf, logits;
};

double forward_impl(const Model& M, const double* p, const int32_t* tok, const int32_t* tgt, int B, int T,
                    int attn_mode, Cache& K, double* logits_out, double* dlogits_scale_out) {
  const Cfg& c = M.c;
  const int C = c.C, F = 4 * c.C, NH = c.H, hd = c.C / c.H;
  const int64_t N = (int64_t)B * T;
  K.B = B;
  K.T = T;
  const double* wte = M.at(p, "wte");
  const double* wpe = M.at(p, "wpe");
  K.x0.assign(N * C, 0.0);
  embedding_fwd(tok, wte, wpe, B, T, C, K.x0.data());
  std::vector<double> x = K.x0;
  auto L = c.L;
  K.xin.assign(L, {});
  K.h1 = K.m1 = K.r1 = K.qkv = K.att = K.xmid = K.h2 = K.m2 = K.r2 = K.u = K.a = K.xin;
  std::vector<double> tmp(N * C);
  for (int l = 0; l < L; ++l) {
    std::string pre = "h" + std::to_string(l) + ".";
    K.xin[l] = x;
    K.h1[l].resize(N * C);
    K.m1[l].resize(N);
    K.r1[l].resize(N);
    layernorm_fwd(x.data(), M.at(p, pre + "ln1_g"), M.at(p, pre + "ln1_b"), N, C, K.h1[l].data(), K.m1[l].data(),
                  K.r1[l].data());
    K.qkv[l].resize(N * 3 * C);
    linear_fwd(K.h1[l].data(), M.at(p, pre + "qkv_w"), M.at_opt(p, pre + "qkv_b"), N, C, 3 * C, K.qkv[l].data());
    K.att[l].resize(N * C);
    attention_fwd(K.qkv[l].data(), B, T, NH, hd, attn_mode, K.att[l].data(), nullptr);
    linear_fwd(K.att[l].data(), M.at(p, pre + "ao_w"), M.at(p, pre + "ao_b"), N, C, C, tmp.data());
    for (int64_t i = 0; i < N * C; ++i) x[i] += tmp[i];
    K.xmid[l] = x;
    K.h2[l].resize(N * C);
    K.m2[l].resize(N);
    K.r2[l].resize(N);
    layernorm_fwd(x.data(), M.at(p, pre + "ln2_g"), M.at(p, pre + "ln2_b"), N, C, K.h2[l].data(), K.m2[l].data(),
                  K.r2[l].data());
    K.u[l].resize(N * F);
    linear_fwd(K.h2[l].data(), M.at(p, pre + "fc_w"), M.at(p, pre + "fc_b"), N, C, F, K.u[l].data());
    K.a[l].resize(N * F);
    for (int64_t i = 0; i < N * F; ++i) K.a[l][i] = gelu(K.u[l][i]);
    linear_fwd(K.a[l].data(), M.at(p, pre + "pj_w"), M.at(p, pre + "pj_b"), N, F, C, tmp.data());
    for (int64_t i = 0; i < N * C; ++i) x[i] += tmp[i];
  }
  K.xL = x;
  K.xf.resize(N * C);
  K.mf.resize(N);
  K.rf.resize(N);
  layernorm_fwd(x.data(), M.at(p, "lnf_g"), M.at(p, "lnf_b"), N, C, K.xf.data(), K.mf.data(), K.rf.data());
  const double* head = c.tied ? wte : M.at(p, "head_w");
  K.logits.resize(N * (int64_t)c.V);
  linear_fwd(K.xf.data(), head, nullptr, N, C, c.V, K.logits.data());
  if (logits_out) std::memcpy(logits_out, K.logits.data(), sizeof(double) * N * c.V);
  double total = cross_entropy(K.logits.data(), N, c.V, c.V, tgt, 1.0, nullptr, nullptr);
  if (dlogits_scale_out) *dlogits_scale_out = 1.0 / (double)N;
  return total / (double)N;
}

void backward_impl(const Model& M, const double* p, const int32_t* tok, const int32_t* tgt, Cache& K, double* g) {
  const Cfg& c = M.c;
  const int C = c.C, F = 4 * c.C, NH = c.H, hd = c.C / c.H;
  const int B = K.B, T = K.T;
  const int64_t N = (int64_t)B * T;
  std::memset(g, 0, sizeof(double) * M.P);
  // loss = mean over N rows
  std::vector<double> dz(N * (int64_t)c.V);
  cross_entropy(K.logits.data(), N, c.V, c.V, tgt, 1.0 / (double)N, dz.data(), nullptr);
  const double* head = c.tied ? M.at(p, "wte") : M.at(p, "head_w");
  double* dhead = c.tied ? M.at(g, "wte") : M.at(g, "head_w");
  std::vector<double> dxf(N * C), dx(N * C), tmp(N * C), dtmp(N * C);
  linear_bwd(dz.data(), K.xf.data(), head, N, C, c.V, dxf.data(), dhead, nullptr);
  layernorm_bwd(dxf.data(), K.xL.data(), M.at(p, "lnf_g"), K.mf.data(), K.rf.data(), N, C, dx.data(),
                M.at(g, "lnf_g"), M.at(g, "lnf_b"));
  std::vector<double> da(N * F), dqkv(N * 3 * C);
  for (int l = c.L - 1; l >= 0; --l) {
    std::string pre = "h" + std::to_string(l) + ".";
    // x_out = x_mid + pj(a)
    linear_bwd(dx.data(), K.a[l].data(), M.at(p, pre + "pj_w"), N, F, C, da.data(), M.at(g, pre + "pj_w"),
               M.at(g, pre + "pj_b"));
    for (int64_t i = 0; i < N * F; ++i) da[i] *= gelu_grad(K.u[l][i]);
    linear_bwd(da.data(), K.h2[l].data(), M.at(p, pre + "fc_w"), N, C, F, tmp.data(), M.at(g, pre + "fc_w"),
               M.at(g, pre + "fc_b"));
    layernorm_bwd(tmp.data(), K.xmid[l].data(), M.at(p, pre + "ln2_g"), K.m2[l].data(), K.r2[l].data(), N, C,
                  dtmp.data(), M.at(g, pre + "ln2_g"), M.at(g, pre + "ln2_b"));
    for (int64_t i = 0; i < N * C; ++i) dx[i] += dtmp[i];
    // x_mid = x_in + ao(att)
    linear_bwd(dx.data(), K.att[l].data(), M.at(p, pre + "ao_w"), N, C, C, tmp.data(), M.at(g, pre + "ao_w"),
               M.at(g, pre + "ao_b"));
    attention_bwd(K.qkv[l].data(), tmp.data(), B, T, NH, hd, dqkv.data());
    linear_bwd(dqkv.data(), K.h1[l].data(), M.at(p, pre + "qkv_w"), N, C, 3 * C, tmp.data(), M.at(g, pre + "qkv_w"),
               M.at_opt(g, pre + "qkv_b"));
    layernorm_bwd(tmp.data(), K.xin[l].data(), M.at(p, pre + "ln1_g"), K.m1[l].data(), K.r1[l].data(), N, C,
                  dtmp.data(), M.at(g, pre + "ln1_g"), M.at(g, pre + "ln1_b"));
    for (int64_t i = 0; i < N * C; ++i) dx[i] += dtmp[i];
  }
  embedding_bwd(tok, dx.data(), B, T, C, M.at(g, "wte"), M.at(g, "wpe"));
}

Cfg to_cfg(const int* c) { return Cfg{c[0], c[1], c[2], c[3], c[4], c[5], c[6]}; }

}  // namespace

// ---------------------------------------------------------------------------
// C entry points for the tests (ctypes). A configuration is passed as
// int[7] = {L, H, C, T, V, tied, qkv_bias}; V is the logical vocabulary (the
// oracle never pads).
// ---------------------------------------------------------------------------
extern "C" {

void orc_set_threads(int n) {
#ifdef _OPENMP
  omp_set_num_threads(n);
#else
  (void)n;
#endif
}

int orc_get_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}

int64_t orc_num_params(const int* cfg) { return total_params(tensor_table(to_cfg(cfg))); }

int orc_num_tensors(const int* cfg) { return (int)tensor_table(to_cfg(cfg)).size(); }

// name (NUL-terminated, truncated to name_len), rows, cols, ndim, offset, decay flag
int orc_tensor_info(const int* cfg, int i, char* name, int name_len, int64_t* rows, int64_t* cols, int* ndim,
                    int64_t* offset, int* decay) {
  auto t = tensor_table(to_cfg(cfg));
  if (i < 0 || i >= (int)t.size()) return -1;
  std::snprintf(name, name_len, "%s", t[i].name.c_str());
  *rows = t[i].rows;
  *cols = t[i].cols;
  *ndim = t[i].ndim;
  *offset = t[i].offset;
  *decay = t[i].ndim >= 2 ? 1 : 0;
  return 0;
}

// Init stream: element j of tensor i draws x1 = splitmix64(seed ^ (i << 40) ^ 2j)
// and x2 = splitmix64(seed ^ (i << 40) ^ (2j + 1)); u1 = (top53(x1) + 1) * 2^-53 in
// (0, 1], u2 = top53(x2) * 2^-53 in [0, 1); z = sqrt(-2 ln u1) cos(2 pi u2);
// value = float(sigma * z). Constant tensors take their fill value.
void orc_init_params(const int* cfg, uint64_t seed, float* out) {
  auto t = tensor_table(to_cfg(cfg));
  for (size_t i = 0; i < t.size(); ++i) {
    const int64_t n = t[i].rows * t[i].cols;
    float* o = out + t[i].offset;
    if (t[i].sigma == 0) {
      for (int64_t j = 0; j < n; ++j) o[j] = (float)t[i].fill;
      continue;
    }
    const uint64_t base = seed ^ ((uint64_t)i << 40);
#pragma omp parallel for schedule(static)
    for (int64_t j = 0; j < n; ++j) {
      uint64_t x1 = splitmix64_at(base ^ (uint64_t)(2 * j));
      uint64_t x2 = splitmix64_at(base ^ (uint64_t)(2 * j + 1));
      double u1 = ((double)(x1 >> 11) + 1.0) * 0x1.0p-53;
      double u2 = (double)(x2 >> 11) * 0x1.0p-53;
      double z = std::sqrt(-2.0 * std::log(u1)) * std::cos(2.0 * M_PI * u2);
      o[j] = (float)(t[i].sigma * z);
    }
  }
}

// Mean cross-entropy of one batch; logits [B*T, V] written when non-null.
// attn_mode 0 is the explicit masked softmax (the default of the Python wrapper);
// mode 1, the blocked online softmax, exists for the equivalence check of the two.
double orc_forward(const int* cfg, const double* params, const int32_t* tok, const int32_t* tgt, int B, int T,
                   int attn_mode, double* logits) {
  Model M(to_cfg(cfg));
  Cache K;
  return forward_impl(M, params, tok, tgt, B, T, attn_mode, K, logits, nullptr);
}

// Mean cross-entropy and its gradient w.r.t. every parameter (grads [P], overwritten).
double orc_forward_backward(const int* cfg, const double* params, const int32_t* tok, const int32_t* tgt, int B,
                            int T, double* grads) {
  Model M(to_cfg(cfg));
  Cache K;
  // the explicit masked softmax (mode 0): the plain definition of causal attention
  double loss = forward_impl(M, params, tok, tgt, B, T, 0, K, nullptr, nullptr);
  backward_impl(M, params, tok, tgt, K, grads);
  return loss;
}

// One optimizer step (torch AdamW semantics) on the averaged gradient G:
//   ||G|| = sqrt(sum G^2);  c = 1/(||G|| + 1e-6);  if c < 1: G <- c G
//   for >=2-D tensors: p <- p (1 - lr wd);  t <- t (already incremented by caller)
//   m <- b1 m + (1-b1) G;  v <- b2 v + (1-b2) G^2
//   p <- p - lr (m / (1 - b1^t)) / (sqrt(v / (1 - b2^t)) + 1e-8)
// clipped_out (nullable) receives the clipped G.
void orc_adamw_step(const int* cfg, double* params, const double* grads, double* m, double* v, int t, double lr,
                    double wd, double b1, double b2, double* gnorm_out, double* clipped_out) {
  Model M(to_cfg(cfg));
  double ss = 0;
  for (int64_t i = 0; i < M.P; ++i) ss += grads[i] * grads[i];
  double norm = std::sqrt(ss);
  double coef = 1.0 / (norm + 1e-6);
  if (coef > 1.0) coef = 1.0;
  if (gnorm_out) *gnorm_out = norm;
  const double bc1 = 1.0 - std::pow(b1, t), bc2 = 1.0 - std::pow(b2, t);
  for (auto& ten : M.tab) {
    const int64_t n = ten.rows * ten.cols;
    for (int64_t j = ten.offset; j < ten.offset + n; ++j) {
      double gj = grads[j] * coef;
      if (clipped_out) clipped_out[j] = gj;
      if (ten.ndim >= 2) params[j] *= (1.0 - lr * wd);
      m[j] = b1 * m[j] + (1.0 - b1) * gj;
      v[j] = b2 * v[j] + (1.0 - b2) * gj * gj;
      params[j] -= lr * (m[j] / bc1) / (std::sqrt(v[j] / bc2) + 1e-8);
    }
  }
}

// ---- single operations, for the per-kernel parity tests --------------------
void orc_layernorm_fwd(const double* x, const double* g, const double* b, int64_t N, int C, double* y, double* mean,
                       double* rstd) {
  layernorm_fwd(x, g, b, N, C, y, mean, rstd);
}
void orc_layernorm_bwd(const double* dy, const double* x, const double* g, const double* mean, const double* rstd,
                       int64_t N, int C, double* dx, double* dg, double* db) {
  layernorm_bwd(dy, x, g, mean, rstd, N, C, dx, dg, db);
}
void orc_linear_fwd(const double* X, const double* W, const double* b, int64_t N, int K, int O, double* Y) {
  linear_fwd(X, W, b, N, K, O, Y);
}
void orc_linear_bwd(const double* dY, const double* X, const double* W, int64_t N, int K, int O, double* dX,
                    double* dW, double* db) {
  linear_bwd(dY, X, W, N, K, O, dX, dW, db);
}
void orc_gelu_fwd(const double* u, int64_t n, double* a) {
  for (int64_t i = 0; i < n; ++i) a[i] = gelu(u[i]);
}
void orc_gelu_bwd(const double* u, const double* da, int64_t n, double* du) {
  for (int64_t i = 0; i < n; ++i) du[i] = da[i] * gelu_grad(u[i]);
}
void orc_attention_fwd(const double* qkv, int B, int T, int NH, int hd, int mode, double* out, double* lse) {
  attention_fwd(qkv, B, T, NH, hd, mode, out, lse);
}
void orc_attention_bwd(const double* qkv, const double* dout, int B, int T, int NH, int hd, double* dqkv) {
  attention_bwd(qkv, dout, B, T, NH, hd, dqkv);
}
double orc_cross_entropy(const double* logits, int64_t N, int V, int64_t ld, const int32_t* tgt, double scale,
                         double* dlogits, double* row_loss) {
  return cross_entropy(logits, N, V, ld, tgt, scale, dlogits, row_loss);
}
void orc_token_buckets(const int32_t* tok, int64_t N, int V, int64_t* counts, int64_t* offsets, int32_t* positions) {
  token_buckets(tok, N, V, counts, offsets, positions);
}
void orc_embedding_bwd(const int32_t* tok, const double* dx0, int B, int T, int C, double* dwte, double* dwpe) {
  embedding_bwd(tok, dx0, B, T, C, dwte, dwpe);
}
// the model's own embedding step (the one forward_impl runs)
void orc_embedding_fwd(const int32_t* tok, const double* wte, const double* wpe, int B, int T, int C, double* x0) {
  embedding_fwd(tok, wte, wpe, B, T, C, x0);
}

}  // extern "C"
