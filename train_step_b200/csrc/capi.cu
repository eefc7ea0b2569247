// capi.cu -- the C ABI of include/gpt2.h: handle, device arena, initialisation and
// the orchestration of one micro-batch (forward, backward) and of the optimizer
// step, all enqueued on one CUDA stream.
#include <cmath>
#include <cstring>
#include <mutex>
#include <string>
#include <vector>

#include "launch.cuh"

using namespace g2;

namespace {

constexpr int HEAD_CHUNK_ROWS = 4096;  // rows of logits materialised at once

struct TensorSlot {
  std::string name;
  int64_t rows, cols;       // logical shape (cols = 1 for vectors)
  int ndim;
  double sigma, fill;       // init
  int64_t canon_off;        // offset in the canonical (logical) flat order
  int64_t dev_off;          // offset in device storage
  int64_t dev_rows;         // rows in storage (vocabulary tensors padded to Vp)
};

struct LayerP {
  float *ln1_g, *ln1_b, *qkv_w, *qkv_b, *ao_w, *ao_b, *ln2_g, *ln2_b, *fc_w, *fc_b, *pj_w, *pj_b;
};

thread_local std::string g_op_error;

uint64_t splitmix64_at(uint64_t x) {
  uint64_t z = x + 0x9E3779B97F4A7C15ull;
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

}  // namespace

struct gpt2 {
  gpt2_config cfg{};
  int Vp = 0, C = 0, F = 0, NH = 0, hd = 0, L = 0, T = 0, Nmax = 0;
  int act_bytes = 4;
  std::vector<TensorSlot> tensors;
  int64_t n_logical = 0, n_store = 0, n_decay = 0;
  // one-shot: events the next backward pass records as gradient buckets complete
  std::vector<cudaEvent_t> grad_events;
  // parameter state (device)
  float *p = nullptr, *g = nullptr, *m = nullptr, *v = nullptr;
  bf16* shadow = nullptr;
  // views into p (master) and g, and the GEMM operand view (shadow or master)
  float *wte = nullptr, *wpe = nullptr, *lnf_g = nullptr, *lnf_b = nullptr, *head = nullptr;
  std::vector<LayerP> lp, lg;
  float *g_wte = nullptr, *g_wpe = nullptr, *g_lnf_g = nullptr, *g_lnf_b = nullptr, *g_head = nullptr;
  // activations
  char* arena = nullptr;
  size_t arena_bytes = 0;
  float *x = nullptr, *stat_mean = nullptr, *stat_rstd = nullptr, *lse = nullptr;
  char *h1 = nullptr, *qkv = nullptr, *att = nullptr, *h2 = nullptr, *u = nullptr, *a = nullptr, *xf = nullptr;
  char *logits = nullptr, *dres_act = nullptr, *du = nullptr, *datt = nullptr, *dqkv = nullptr;
  float *dres = nullptr, *dh = nullptr, *Dattn = nullptr, *row_loss = nullptr, *part = nullptr, *splitk = nullptr;
  float2* ce_stats = nullptr;  // softmax partials of one head chunk, [chunk rows][2 * ceil(Vp / 128)]
  float* splitk2 = nullptr;    // second split-K workspace (dW reductions alternate on the side stream)
  float* part_bias = nullptr;  // bias-gradient column-sum partials (GELU-backward epilogue, attention backward)
  void* attn_ds = nullptr;     // bf16: the attention backward's stored dS^T tiles (one layer at a time)
  size_t part_bias_floats = 0;
  SideStream side;             // reductions of gradient partials overlapping the backward pass
  size_t part_floats = 0, splitk_floats = 0;
  int *tok = nullptr, *tgt = nullptr;
  void* emb_scratch = nullptr;
  // generation: key/value cache [L][B_max][T][2C] bf16 (allocated by the first prefill)
  bf16* kv = nullptr;
  int kv_B = 0, kv_len = 0;
  int* d_pos = nullptr;        // device copy of the next cache position (read by captured steps)
  float* dec_part = nullptr;   // split-key partial attention results
  cudaGraphExec_t dec_graph = nullptr;  // captured decode step, for (dec_B, dec_logits, dec_ld)
  int dec_B = 0;
  float* dec_logits = nullptr;
  int64_t dec_ld = 0;
  long long dec_graph_launches = 0;
  // scalars
  int* d_err = nullptr;
  float* d_loss = nullptr;
  float* d_gnorm = nullptr;
  double* d_norm_part = nullptr;
  int norm_parts = 0;
  // state
  cudaStream_t stream = nullptr;
  bool own_stream = false;
  int k = 0, k_B = 0, k_T = 0;
  int64_t t = 0;
  long long launches = 0;
  int num_sms = 148;
  std::string err;
  Profiler prof;

  LaunchCtx ctx() {
    LaunchCtx c;
    c.prof = &prof;
    c.stream = stream;
    c.d_err = d_err;
    c.msg = &err;
    c.launches = &launches;
    c.splitk_ws = splitk;
    c.splitk_cap = splitk_floats;
    c.ws_buf = SIDE_WS0;
    c.num_sms = num_sms;
    return c;
  }
  float* P(const std::string& n) { return p + find(n).dev_off; }
  float* G(const std::string& n) { return g + find(n).dev_off; }
  const TensorSlot& find(const std::string& n) const {
    for (auto& s : tensors)
      if (s.name == n) return s;
    static TensorSlot none{};
    return none;
  }
  bool has(const std::string& n) const {
    for (auto& s : tensors)
      if (s.name == n) return true;
    return false;
  }
  // GEMM operand for a weight: the bf16 shadow in bf16 mode, the master otherwise
  const void* W(const float* master) const {
    if (cfg.dtype == GPT2_BF16) return shadow + (master - p);
    return master;
  }
  char* act(char* base, int64_t layer, int64_t per_layer_elems) const {
    return base + layer * per_layer_elems * act_bytes;
  }
};

namespace {

int set_err(gpt2* m, int code, const std::string& msg) {
  if (m) m->err = msg;
  return code;
}

int cuda_err(gpt2* m, cudaError_t e, const char* what) {
  return set_err(m, GPT2_ERR_CUDA, std::string(what) + ": " + cudaGetErrorString(e));
}

#define CK(m, call)                                  \
  do {                                               \
    cudaError_t e_ = (call);                         \
    if (e_ != cudaSuccess) return cuda_err(m, e_, #call); \
  } while (0)
#define RK(call)            \
  do {                      \
    int r_ = (call);        \
    if (r_) return r_;      \
  } while (0)

int64_t align64(int64_t x) { return (x + 63) & ~int64_t(63); }

void build_tensors(gpt2* m) {
  const gpt2_config& c = m->cfg;
  const int64_t C = c.C, F = 4LL * c.C;
  const double s = 0.02, sr = 0.02 / std::sqrt(2.0 * c.L);
  auto& t = m->tensors;
  t.clear();
  auto add = [&](const std::string& n, int64_t r, int64_t cc, int nd, double sg, double fill, int64_t dev_rows) {
    t.push_back(TensorSlot{n, r, cc, nd, sg, fill, 0, 0, dev_rows});
  };
  add("wte", c.V, C, 2, s, 0, m->Vp);
  add("wpe", c.T, C, 2, s, 0, c.T);
  for (int l = 0; l < c.L; ++l) {
    std::string p = "h" + std::to_string(l) + ".";
    add(p + "ln1_g", C, 1, 1, 0, 1, C);
    add(p + "ln1_b", C, 1, 1, 0, 0, C);
    add(p + "qkv_w", 3 * C, C, 2, s, 0, 3 * C);
    if (c.qkv_bias) add(p + "qkv_b", 3 * C, 1, 1, 0, 0, 3 * C);
    add(p + "ao_w", C, C, 2, sr, 0, C);
    add(p + "ao_b", C, 1, 1, 0, 0, C);
    add(p + "ln2_g", C, 1, 1, 0, 1, C);
    add(p + "ln2_b", C, 1, 1, 0, 0, C);
    add(p + "fc_w", F, C, 2, s, 0, F);
    add(p + "fc_b", F, 1, 1, 0, 0, F);
    add(p + "pj_w", C, F, 2, sr, 0, C);
    add(p + "pj_b", C, 1, 1, 0, 0, C);
  }
  add("lnf_g", C, 1, 1, 0, 1, C);
  add("lnf_b", C, 1, 1, 0, 0, C);
  if (!c.tied) add("head_w", c.V, C, 2, s, 0, m->Vp);
  int64_t off = 0;
  for (auto& x : t) {
    x.canon_off = off;
    off += x.rows * x.cols;
  }
  m->n_logical = off;
  // storage: all >= 2-D tensors first (weight decay and the bf16 shadow cover
  // exactly that prefix), each tensor 64-element aligned
  int64_t d = 0;
  for (auto& x : t)
    if (x.ndim == 2) {
      x.dev_off = d;
      d = align64(d + x.dev_rows * x.cols);
    }
  m->n_decay = d;
  for (auto& x : t)
    if (x.ndim == 1) {
      x.dev_off = d;
      d = align64(d + x.dev_rows * x.cols);
    }
  // a multiple of 4096 floats, so that the storage splits into equal 64-aligned shards for
  // up to 64 data-parallel ranks (the tail is zero and stays zero under AdamW)
  m->n_store = (d + 4095) / 4096 * 4096;
}

// Gradient bucket of canonical tensor i: layer l's tensors form bucket l, everything else
// (embeddings, final LayerNorm, untied head) bucket L. The backward pass completes the
// buckets in the order L-1, ..., 0, L.
int tensor_bucket(const gpt2* m, size_t i) {
  const std::string& n = m->tensors[i].name;
  if (n.size() > 1 && n[0] == 'h' && n[1] >= '0' && n[1] <= '9') return std::atoi(n.c_str() + 1);
  return m->cfg.L;
}

// Record grad_events[b] once bucket b's gradients are complete: on the side stream (after
// everything the main stream has enqueued) when there is one, so the main stream never waits.
int mark_bucket(gpt2* m, const std::vector<cudaEvent_t>& ev, const LaunchCtx& cb, int b) {
  if (ev.empty()) return GPT2_OK;
  cudaStream_t s = cb.stream;
  if (cb.side) {
    CK(m, cudaEventRecord(cb.side->ready, cb.stream));
    CK(m, cudaStreamWaitEvent(cb.side->s, cb.side->ready, 0));
    s = cb.side->s;
  }
  CK(m, cudaEventRecord(ev[b], s));
  return GPT2_OK;
}

void host_init(const gpt2* m, uint64_t seed, std::vector<float>& out) {
  out.assign(m->n_logical, 0.f);
  for (size_t i = 0; i < m->tensors.size(); ++i) {
    const TensorSlot& t = m->tensors[i];
    const int64_t n = t.rows * t.cols;
    float* o = out.data() + t.canon_off;
    if (t.sigma == 0) {
      for (int64_t j = 0; j < n; ++j) o[j] = (float)t.fill;
      continue;
    }
    const uint64_t base = seed ^ ((uint64_t)i << 40);
    for (int64_t j = 0; j < n; ++j) {
      const uint64_t x1 = splitmix64_at(base ^ (uint64_t)(2 * j));
      const uint64_t x2 = splitmix64_at(base ^ (uint64_t)(2 * j + 1));
      const double u1 = ((double)(x1 >> 11) + 1.0) * 0x1.0p-53;
      const double u2 = (double)(x2 >> 11) * 0x1.0p-53;
      const double z = std::sqrt(-2.0 * std::log(u1)) * std::cos(2.0 * M_PI * u2);
      o[j] = (float)(t.sigma * z);
    }
  }
}

int check_device_error(gpt2* m) {
  int h = 0;
  CK(m, cudaMemcpyAsync(&h, m->d_err, sizeof(int), cudaMemcpyDeviceToHost, m->stream));
  CK(m, cudaStreamSynchronize(m->stream));
  if (h) {
    CK(m, cudaMemsetAsync(m->d_err, 0, sizeof(int), m->stream));
    if (h == DEV_TOKEN_RANGE) return set_err(m, GPT2_ERR_TOKEN_RANGE, "a token or target id is outside [0, V)");
    if (h == DEV_TIMEOUT) return set_err(m, GPT2_ERR_TIMEOUT, "a bounded device-side wait gave up");
    return set_err(m, GPT2_ERR_CUDA, "device error word set");
  }
  return GPT2_OK;
}

int copy_tokens(gpt2* m, int* dst, const int32_t* src, size_t n) {
  cudaPointerAttributes at;
  cudaMemcpyKind kind = cudaMemcpyHostToDevice;
  if (cudaPointerGetAttributes(&at, src) == cudaSuccess &&
      (at.type == cudaMemoryTypeDevice || at.type == cudaMemoryTypeManaged))
    kind = cudaMemcpyDeviceToDevice;
  cudaGetLastError();
  CK(m, cudaMemcpyAsync(dst, src, n * sizeof(int32_t), kind, m->stream));
  return GPT2_OK;
}

// Forward of the embedding, the L blocks and the final LayerNorm for B sequences of T
// tokens already in m->tok: leaves every activation the backward pass reads, the keys and
// values of each layer in its qkv activation, and ln_f's output in m->xf.
int forward_layers(gpt2* m, int B, int T) {
  LaunchCtx c = m->ctx();
  const int dt = m->cfg.dtype;
  // bf16: the tensor-core and LayerNorm kernels launch as programmatic dependents, so each
  // one's set-up (barriers, TMEM allocation) overlaps the tail of the kernel before it
  c.pdl = dt == GPT2_BF16 && !m->prof.on;
  const int N = B * T, C = m->C, F = m->F, L = m->L, NH = m->NH, hd = m->hd;
  const int64_t NC = (int64_t)m->Nmax * C, NF = (int64_t)m->Nmax * F, N3C = 3 * NC;
  const int64_t NLSE = (int64_t)m->cfg.B_max * NH * m->T;
  const int ab = m->act_bytes;
  auto xs = [&](int i) { return m->x + (int64_t)i * NC; };
  auto mean = [&](int i) { return m->stat_mean + (int64_t)i * m->Nmax; };
  auto rstd = [&](int i) { return m->stat_rstd + (int64_t)i * m->Nmax; };
  auto ACT = [&](char* base, int l, int64_t per) -> void* { return base + (int64_t)l * per * ab; };
  auto LN_F = [&](const float* x, const float* gg, const float* bb, void* y, float* mu, float* rs) {
    return dt == GPT2_BF16 ? layernorm_fwd_t<bf16>(c, x, gg, bb, N, C, (bf16*)y, mu, rs)
                           : layernorm_fwd_t<float>(c, x, gg, bb, N, C, (float*)y, mu, rs);
  };

  RK(embedding_fwd(c, m->tok, m->wte, m->wpe, N, T, C, m->cfg.V, xs(0)));
  for (int l = 0; l < L; ++l) {
    const LayerP& w = m->lp[l];
    void* h1 = ACT(m->h1, l, NC);
    void* qkv = ACT(m->qkv, l, N3C);
    void* att = ACT(m->att, l, NC);
    void* h2 = ACT(m->h2, l, NC);
    void* u = ACT(m->u, l, NF);
    void* a = ACT(m->a, l, NF);
    float* lse = m->lse + l * NLSE;
    RK(LN_F(xs(2 * l), w.ln1_g, w.ln1_b, h1, mean(2 * l), rstd(2 * l)));
    RK(gemm(c, dt, GemmDesc{h1, C, false, m->W(w.qkv_w), C, false, N, 3 * C, C, EPI_BF16, qkv, 3 * C, nullptr, 0,
                            w.qkv_b, nullptr, 0, 0, 1}));
    RK(attention_fwd(c, dt, qkv, B, T, NH, hd, att, lse));
    RK(gemm(c, dt, GemmDesc{att, C, false, m->W(w.ao_w), C, false, N, C, C, EPI_F32_RESID, xs(2 * l + 1), C, nullptr,
                            0, w.ao_b, xs(2 * l), C, 0, 1}));
    RK(LN_F(xs(2 * l + 1), w.ln2_g, w.ln2_b, h2, mean(2 * l + 1), rstd(2 * l + 1)));
    RK(gemm(c, dt, GemmDesc{h2, C, false, m->W(w.fc_w), C, false, N, F, C, EPI_BF16_GELU, u, F, a, F, w.fc_b, nullptr,
                            0, 0, 1}));
    RK(gemm(c, dt, GemmDesc{a, F, false, m->W(w.pj_w), F, false, N, C, F, EPI_F32_RESID, xs(2 * l + 2), C, nullptr, 0,
                            w.pj_b, xs(2 * l + 1), C, 0, 1}));
  }
  RK(LN_F(xs(2 * L), m->lnf_g, m->lnf_b, m->xf, mean(2 * L), rstd(2 * L)));

  return GPT2_OK;
}

// Forward of one micro-batch; with `backward`, also the backward pass that adds
// the gradients of this micro-batch's mean loss into m->g.
int run_micro_batch(gpt2* m, int B, int T, bool backward) {
  LaunchCtx c = m->ctx();
  const int dt = m->cfg.dtype;
  c.pdl = dt == GPT2_BF16 && !m->prof.on;  // programmatic dependent launches, as in forward_layers
  const int N = B * T, C = m->C, F = m->F, L = m->L, NH = m->NH, hd = m->hd, Vp = m->Vp;
  const int64_t NC = (int64_t)m->Nmax * C, NF = (int64_t)m->Nmax * F, N3C = 3 * NC;
  const int64_t NLSE = (int64_t)m->cfg.B_max * NH * m->T;
  const int ab = m->act_bytes;
  auto xs = [&](int i) { return m->x + (int64_t)i * NC; };
  auto mean = [&](int i) { return m->stat_mean + (int64_t)i * m->Nmax; };
  auto rstd = [&](int i) { return m->stat_rstd + (int64_t)i * m->Nmax; };
  auto ACT = [&](char* base, int l, int64_t per) -> void* { return base + (int64_t)l * per * ab; };

  // bf16 backward: reductions of gradient partials run on the side stream (cb); they
  // overlap, except while per-kernel times are being recorded (an event pair around a
  // kernel that shares the GPU would charge it the overlap)
  LaunchCtx cb = c;
  if (backward && dt == GPT2_BF16 && !m->prof.on) cb.side = &m->side;
  // the gradient-bucket events armed for this backward pass (one-shot: taken now, so that a
  // call that fails part-way leaves none behind for a later one)
  std::vector<cudaEvent_t> bucket_ev;
  if (backward) bucket_ev.swap(m->grad_events);
  EmbScratch es = emb_scratch_carve(m->emb_scratch, N, C);
  if (backward && cb.side) {
    // the embedding backward's sort of the token ids needs only the tokens: it runs on the
    // side stream (one CTA) under the forward pass; the embedding backward waits for it
    RK(token_sort(side_ctx(cb), m->tok, N, m->cfg.V, es));
    side_mark_free(cb, SIDE_EMB);
  }

  // ---------------- forward ----------------
  RK(forward_layers(m, B, T));

  // ---------------- head + cross-entropy, chunk by chunk ----------------
  const float* headw = m->cfg.tied ? m->wte : m->head;
  float* g_head = m->cfg.tied ? m->g_wte : m->g_head;
  const int chunk = N < HEAD_CHUNK_ROWS ? N : HEAD_CHUNK_ROWS;
  for (int r0 = 0; r0 < N; r0 += chunk) {
    const int rows = (N - r0) < chunk ? (N - r0) : chunk;
    char* xf_c = m->xf + (int64_t)r0 * C * ab;
    GemmDesc hd{xf_c, C, false, m->W(headw), C, false, rows, Vp, C, EPI_BF16, m->logits, Vp, nullptr, 0,
                nullptr, nullptr, 0, 0, 1, CAT_GEMM_HEAD};
    if (dt == GPT2_BF16) {
      // the head GEMM's epilogue leaves each row's softmax partials for the cross-entropy
      hd.rowstats = m->ce_stats;
      hd.stats_ncols = m->cfg.V;
    }
    RK(gemm(c, dt, hd));
    if (dt == GPT2_BF16)
      RK(cross_entropy_stats(c, (bf16*)m->logits, Vp, rows, m->cfg.V, m->tgt + r0, 1.0f / (float)N,
                             m->row_loss + r0, m->ce_stats, gemm_rowstats_count(hd), nullptr));
    else
      RK(cross_entropy(c, dt, m->logits, Vp, rows, m->cfg.V, m->tgt + r0, 1.0f / (float)N, m->row_loss + r0));
    if (backward) {
      // dxf = dlogits W ; dW += dlogits^T xf
      RK(gemm(cb, dt, GemmDesc{m->logits, Vp, false, m->W(headw), C, true, rows, C, Vp, EPI_F32, m->dh + (int64_t)r0 * C,
                               C, nullptr, 0, nullptr, nullptr, 0, 0, 0, CAT_GEMM_HEAD}));
      RK(gemm(cb, dt, GemmDesc{m->logits, Vp, true, xf_c, C, true, Vp, C, rows, EPI_F32, g_head, C, nullptr, 0, nullptr,
                               nullptr, 0, 1, 0, CAT_GEMM_HEAD}));
    }
  }
  sum_rows_kernel<<<1, 1024, 0, m->stream>>>(m->row_loss, N, 1.0f / (float)N, m->d_loss, 0);
  RK(check_launch(c, "sum_rows"));
  if (!backward) return GPT2_OK;

  // ---------------- backward ----------------
  void* dres_act = dt == GPT2_BF16 ? (void*)m->dres_act : (void*)m->dres;
  // LN backward; its column sums of the new dres are the bias gradient of the
  // linear layer that produced this residual (dbias_next, nullable)
  auto LN_B = [&](const float* dy, const float* x, const float* gg, float* mu, float* rs, int accumulate, float* dg,
                  float* db, float* dbias_next) -> int {
    return dt == GPT2_BF16 ? layernorm_bwd_t<bf16>(cb, dy, x, gg, mu, rs, N, C, m->dres, (bf16*)m->dres_act,
                                                   accumulate, m->part, dg, db, dbias_next, 1, SIDE_LN)
                           : layernorm_bwd_t<float>(c, dy, x, gg, mu, rs, N, C, m->dres, (float*)nullptr, accumulate,
                                                    m->part, dg, db, dbias_next, 1);
  };
  // bf16 mode: the dX GEMMs in front of the per-layer LayerNorms write dh in bf16 (half the
  // bytes for the GEMM to store and the LayerNorm to read), in the fp32 dh buffer's storage;
  // the final LayerNorm's dh stays fp32 (the head's dX accumulates over the logit chunks)
  bf16* dh16 = reinterpret_cast<bf16*>(m->dh);
  auto LN_B16 = [&](const float* x, const float* gg, float* mu, float* rs, float* dg, float* db,
                    float* dbias_next) -> int {
    return layernorm_bwd_t<bf16, bf16>(cb, dh16, x, gg, mu, rs, N, C, m->dres, (bf16*)m->dres_act, 1, m->part, dg,
                                       db, dbias_next, 1, SIDE_LN);
  };
  auto COLSUM_ACT = [&](const void* y, int ncols, float* out) -> int {
    return dt == GPT2_BF16 ? colsum_t<bf16>(c, (const bf16*)y, ncols, N, ncols, m->part, out)
                           : colsum_t<float>(c, (const float*)y, ncols, N, ncols, m->part, out);
  };
  // weight-gradient GEMMs alternate between two split-K workspaces, each reduced on the
  // side stream while the next GEMMs run
  int dw_i = 0;
  auto DW = [&](const GemmDesc& d) -> int {
    LaunchCtx cw = cb;
    if (cb.side) {
      cw.splitk_ws = (dw_i & 1) ? m->splitk2 : m->splitk;
      cw.ws_buf = (dw_i & 1) ? SIDE_WS1 : SIDE_WS0;
      cw.reduce_on_side = true;
      ++dw_i;
    }
    return gemm(cw, dt, d);
  };
  // a bias-gradient reduction of m->part_bias on the side stream (in order when there is none)
  auto BIAS_RED = [&](int P, int ncols, float* out) -> int {
    if (!cb.side) return reduce_partials(cb, m->part_bias, P, ncols, 1, out, nullptr, nullptr, 1);
    const int r = reduce_partials(side_ctx(cb), m->part_bias, P, ncols, 1, out, nullptr, nullptr, 1);
    side_mark_free(cb, SIDE_BIAS);
    return r;
  };
  RK(LN_B(m->dh, xs(2 * L), m->lnf_g, mean(2 * L), rstd(2 * L), 0, m->g_lnf_g, m->g_lnf_b, m->lg[L - 1].pj_b));
  for (int l = L - 1; l >= 0; --l) {
    const LayerP& w = m->lp[l];
    const LayerP& gw = m->lg[l];
    void* h1 = ACT(m->h1, l, NC);
    void* qkv = ACT(m->qkv, l, N3C);
    void* att = ACT(m->att, l, NC);
    void* h2 = ACT(m->h2, l, NC);
    void* u = ACT(m->u, l, NF);
    void* a = ACT(m->a, l, NF);
    float* lse = m->lse + l * NLSE;
    // MLP: x_out = x_mid + pj(gelu(fc(ln2(x_mid))))
    RK(DW(GemmDesc{dres_act, C, true, a, F, true, C, F, N, EPI_F32, gw.pj_w, F, nullptr, 0, nullptr, nullptr,
                   0, 1, 0, CAT_GEMM_DW}));
    {
      // bf16: the GELU-backward epilogue leaves the column sums of du (fc's bias gradient)
      // per 32-row block in m->part_bias
      GemmDesc d{dres_act, C, false, m->W(w.pj_w), F, true, N, F, C, EPI_BF16_DGELU, m->du, F, nullptr, 0,
                 nullptr, u, F, 0, 1, CAT_GEMM_DX};
      if (dt == GPT2_BF16) {
        d.colsum = m->part_bias;
        RK(side_wait_free(cb, SIDE_BIAS));
      }
      RK(gemm(cb, dt, d));
    }
    if (dt == GPT2_BF16) RK(BIAS_RED((N + 31) / 32, F, gw.fc_b));
    RK(DW(GemmDesc{m->du, F, true, h2, C, true, F, C, N, EPI_F32, gw.fc_w, C, nullptr, 0, nullptr, nullptr, 0,
                   1, 0, CAT_GEMM_DW}));
    if (dt != GPT2_BF16) RK(COLSUM_ACT(m->du, F, gw.fc_b));
    if (dt == GPT2_BF16) {
      RK(gemm(c, dt, GemmDesc{m->du, F, false, m->W(w.fc_w), C, true, N, C, F, EPI_BF16, dh16, C, nullptr, 0,
                              nullptr, nullptr, 0, 0, 1, CAT_GEMM_DX}));
      RK(LN_B16(xs(2 * l + 1), w.ln2_g, mean(2 * l + 1), rstd(2 * l + 1), gw.ln2_g, gw.ln2_b, gw.ao_b));
    } else {
      RK(gemm(c, dt, GemmDesc{m->du, F, false, m->W(w.fc_w), C, true, N, C, F, EPI_F32, m->dh, C, nullptr, 0,
                              nullptr, nullptr, 0, 0, 1, CAT_GEMM_DX}));
      RK(LN_B(m->dh, xs(2 * l + 1), w.ln2_g, mean(2 * l + 1), rstd(2 * l + 1), 1, gw.ln2_g, gw.ln2_b, gw.ao_b));
    }
    // attention: x_mid = x_in + ao(attn(ln1(x_in)))
    RK(DW(GemmDesc{dres_act, C, true, att, C, true, C, C, N, EPI_F32, gw.ao_w, C, nullptr, 0, nullptr, nullptr,
                   0, 1, 0, CAT_GEMM_DW}));
    RK(gemm(c, dt, GemmDesc{dres_act, C, false, m->W(w.ao_w), C, true, N, C, C, EPI_BF16, m->datt, C, nullptr, 0,
                            nullptr, nullptr, 0, 0, 1, CAT_GEMM_DX}));
    // bf16: the attention backward leaves the column sums of dqkv (the qkv bias gradient)
    // per 32-row block in m->part_bias
    const bool qkvb_fused = gw.qkv_b && dt == GPT2_BF16;
    if (qkvb_fused) RK(side_wait_free(cb, SIDE_BIAS));
    RK(attention_bwd(c, dt, qkv, att, m->datt, lse, B, T, NH, hd, m->dqkv, m->Dattn,
                     qkvb_fused ? m->part_bias : nullptr, dt == GPT2_BF16 ? m->attn_ds : nullptr));
    if (qkvb_fused) RK(BIAS_RED(attn_colsum_blocks(B, T), 3 * C, gw.qkv_b));
    RK(DW(GemmDesc{m->dqkv, 3 * C, true, h1, C, true, 3 * C, C, N, EPI_F32, gw.qkv_w, C, nullptr, 0, nullptr,
                   nullptr, 0, 1, 0, CAT_GEMM_DW}));
    if (gw.qkv_b && !qkvb_fused) RK(COLSUM_ACT(m->dqkv, 3 * C, gw.qkv_b));
    if (dt == GPT2_BF16) {
      RK(gemm(c, dt, GemmDesc{m->dqkv, 3 * C, false, m->W(w.qkv_w), C, true, N, C, 3 * C, EPI_BF16, dh16, C, nullptr,
                              0, nullptr, nullptr, 0, 0, 1, CAT_GEMM_DX}));
      RK(LN_B16(xs(2 * l), w.ln1_g, mean(2 * l), rstd(2 * l), gw.ln1_g, gw.ln1_b, l > 0 ? m->lg[l - 1].pj_b : nullptr));
    } else {
      RK(gemm(c, dt, GemmDesc{m->dqkv, 3 * C, false, m->W(w.qkv_w), C, true, N, C, 3 * C, EPI_F32, m->dh, C, nullptr,
                              0, nullptr, nullptr, 0, 0, 1, CAT_GEMM_DX}));
      RK(LN_B(m->dh, xs(2 * l), w.ln1_g, mean(2 * l), rstd(2 * l), 1, gw.ln1_g, gw.ln1_b,
              l > 0 ? m->lg[l - 1].pj_b : nullptr));
    }
    RK(mark_bucket(m, bucket_ev, cb, l));  // layer l's pj_b came from layer l + 1's LayerNorm (or ln_f)
  }
  RK(side_wait_free(cb, SIDE_EMB));  // the token sort (side stream) has finished
  RK(embedding_bwd(c, m->tok, m->dres, B, T, C, m->cfg.V, m->g_wte, m->g_wpe, es, cb.side != nullptr));
  RK(side_join(cb));  // every gradient is complete on the main stream from here on
  RK(mark_bucket(m, bucket_ev, c, L));
  return GPT2_OK;
}

int validate_batch(gpt2* m, const int32_t* tokens, const int32_t* targets, int B, int T) {
  if (!m) return GPT2_ERR_CONFIG;
  if (!tokens || !targets) return set_err(m, GPT2_ERR_CONFIG, "tokens and targets are required");
  if (T <= 0 || B <= 0) return set_err(m, GPT2_ERR_CONFIG, "B and T must be positive");
  if (T > m->cfg.T) return set_err(m, GPT2_ERR_SEQ_TOO_LONG, "sequence length exceeds the block size");
  if (B > m->cfg.B_max) return set_err(m, GPT2_ERR_BATCH, "B exceeds B_max");
  return GPT2_OK;
}

}  // namespace

extern "C" {

int gpt2_create(const gpt2_config* cfg, uint64_t seed, gpt2** out) {
  if (!out) return GPT2_ERR_CONFIG;
  *out = nullptr;
  if (!cfg) return GPT2_ERR_CONFIG;
  const gpt2_config c = *cfg;
  if (c.L <= 0 || c.H <= 0 || c.C <= 0 || c.T <= 0 || c.V <= 0 || c.B_max <= 0 || c.C % c.H ||
      (c.dtype != GPT2_FP32 && c.dtype != GPT2_BF16) || c.C % 64 || c.V > (1 << 17))
    return GPT2_ERR_CONFIG;
  const int hd = c.C / c.H;
  if (c.dtype == GPT2_BF16 && hd != 64) return GPT2_ERR_CONFIG;
  if (c.dtype == GPT2_FP32 && (hd % 32 || hd > 128)) return GPT2_ERR_CONFIG;
  if ((int64_t)c.B_max * c.T > EMB_MAX_TOKENS) return GPT2_ERR_BATCH;
  gpt2* m = new gpt2();
  m->cfg = c;
  m->C = c.C;
  m->F = 4 * c.C;
  m->NH = c.H;
  m->hd = hd;
  m->L = c.L;
  m->T = c.T;
  m->Vp = (c.V + 63) / 64 * 64;
  m->Nmax = c.B_max * c.T;
  m->act_bytes = c.dtype == GPT2_BF16 ? 2 : 4;
  m->num_sms = device_sm_count();
  build_tensors(m);
  auto bail = [&](int code, const char* what) {
    (void)what;
    gpt2_destroy(m);
    // a failed cudaMalloc leaves its error as the runtime's last error: clear it so that
    // it is not reported by the next launch check of another handle
    cudaGetLastError();
    return code;
  };
  if (cudaStreamCreateWithFlags(&m->stream, cudaStreamNonBlocking) != cudaSuccess) return bail(GPT2_ERR_CUDA, "stream");
  m->own_stream = true;
  if (cudaStreamCreateWithFlags(&m->side.s, cudaStreamNonBlocking) != cudaSuccess ||
      cudaEventCreateWithFlags(&m->side.ready, cudaEventDisableTiming) != cudaSuccess ||
      cudaEventCreateWithFlags(&m->side.joined, cudaEventDisableTiming) != cudaSuccess)
    return bail(GPT2_ERR_CUDA, "side stream");
  for (auto& e : m->side.freed)
    if (cudaEventCreateWithFlags(&e, cudaEventDisableTiming) != cudaSuccess) return bail(GPT2_ERR_CUDA, "side events");
  const size_t S = (size_t)m->n_store;
  if (cudaMalloc(&m->p, S * 4) || cudaMalloc(&m->g, S * 4) || cudaMalloc(&m->m, S * 4) || cudaMalloc(&m->v, S * 4))
    return bail(GPT2_ERR_OOM, "state");
  if (c.dtype == GPT2_BF16 && cudaMalloc(&m->shadow, (size_t)m->n_decay * 2)) return bail(GPT2_ERR_OOM, "shadow");
  cudaMemset(m->p, 0, S * 4);
  cudaMemset(m->g, 0, S * 4);
  cudaMemset(m->m, 0, S * 4);
  cudaMemset(m->v, 0, S * 4);
  // views
  m->wte = m->P("wte");
  m->wpe = m->P("wpe");
  m->lnf_g = m->P("lnf_g");
  m->lnf_b = m->P("lnf_b");
  m->head = c.tied ? nullptr : m->P("head_w");
  m->g_wte = m->G("wte");
  m->g_wpe = m->G("wpe");
  m->g_lnf_g = m->G("lnf_g");
  m->g_lnf_b = m->G("lnf_b");
  m->g_head = c.tied ? nullptr : m->G("head_w");
  m->lp.resize(c.L);
  m->lg.resize(c.L);
  for (int l = 0; l < c.L; ++l) {
    const std::string p = "h" + std::to_string(l) + ".";
    auto fill = [&](LayerP& L, bool grad) {
      auto X = [&](const char* n) -> float* {
        if (!m->has(p + n)) return nullptr;
        return grad ? m->G(p + n) : m->P(p + n);
      };
      L = LayerP{X("ln1_g"), X("ln1_b"), X("qkv_w"), X("qkv_b"), X("ao_w"), X("ao_b"),
                 X("ln2_g"), X("ln2_b"), X("fc_w"),  X("fc_b"),  X("pj_w"), X("pj_b")};
    };
    fill(m->lp[l], false);
    fill(m->lg[l], true);
  }
  // activation arena
  const int64_t N = m->Nmax, C = c.C, F = m->F, L = c.L, ab = m->act_bytes;
  const int64_t chunk = N < HEAD_CHUNK_ROWS ? N : HEAD_CHUNK_ROWS;
  int gx, R, rp;
  colsum_shape((int)N, (int)(3 * C > F ? 3 * C : F), gx, R, rp);
  const int64_t colsum_floats = (int64_t)(R + 1) * (3 * C > F ? 3 * C : F);
  // colsum partials never exceed 1184 row chunks x 2048 columns per chunk of columns
  m->part_floats = (size_t)std::max<int64_t>(
      std::max<int64_t>(std::max<int64_t>(3LL * ln_bwd_grid((int)N, (int)C, m->num_sms) * C, colsum_floats),
                        1184LL * 2048 + 4096),
      std::max<int64_t>((N + 31) / 32 * F,                         // the GELU-backward epilogue's column sums
                        (int64_t)(c.B_max * ((c.T + 127) / 128) * 4) * 3 * C));  // the attention backward's
  m->splitk_floats = (size_t)std::max<int64_t>(16LL * F * C, 16LL * chunk * C);
  m->part_bias_floats = (size_t)std::max<int64_t>((N + 31) / 32 * F, (int64_t)c.B_max * ((c.T + 127) / 128) * 4 * 3 * C);
  std::vector<std::pair<void**, size_t>> plan = {
      {(void**)&m->x, (size_t)(2 * L + 1) * N * C * 4},
      {(void**)&m->stat_mean, (size_t)(2 * L + 1) * N * 4},
      {(void**)&m->stat_rstd, (size_t)(2 * L + 1) * N * 4},
      {(void**)&m->lse, (size_t)L * c.B_max * c.H * c.T * 4},
      {(void**)&m->h1, (size_t)L * N * C * ab},
      {(void**)&m->qkv, (size_t)L * N * 3 * C * ab},
      {(void**)&m->att, (size_t)L * N * C * ab},
      {(void**)&m->h2, (size_t)L * N * C * ab},
      {(void**)&m->u, (size_t)L * N * F * ab},
      {(void**)&m->a, (size_t)L * N * F * ab},
      {(void**)&m->xf, (size_t)N * C * ab},
      {(void**)&m->logits, (size_t)chunk * m->Vp * ab},
      {(void**)&m->ce_stats, (size_t)chunk * 2 * ((m->Vp + 127) / 128) * sizeof(float2)},
      {(void**)&m->dres_act, (size_t)N * C * ab},
      {(void**)&m->du, (size_t)N * F * ab},
      {(void**)&m->datt, (size_t)N * C * ab},
      {(void**)&m->dqkv, (size_t)N * 3 * C * ab},
      {(void**)&m->dres, (size_t)N * C * 4},
      {(void**)&m->dh, (size_t)N * C * 4},
      {(void**)&m->Dattn, (size_t)c.B_max * c.H * c.T * 4},
      {(void**)&m->attn_ds, c.dtype == GPT2_BF16 ? attn_ds_bytes(c.B_max, c.T, c.H) : 0},
      {(void**)&m->row_loss, (size_t)N * 4},
      {(void**)&m->part, m->part_floats * 4},
      {(void**)&m->splitk, m->splitk_floats * 4},
      {(void**)&m->splitk2, m->splitk_floats * 4},
      {(void**)&m->part_bias, m->part_bias_floats * 4},
      {(void**)&m->tok, (size_t)N * 4},
      {(void**)&m->tgt, (size_t)N * 4},
      {(void**)&m->emb_scratch, emb_scratch_bytes((int)N, (int)C)},
      {(void**)&m->d_err, 256},
      {(void**)&m->d_loss, 256},
      {(void**)&m->d_gnorm, 256},
  };
  m->norm_parts = 8 * m->num_sms;
  plan.push_back({(void**)&m->d_norm_part, (size_t)m->norm_parts * 8});
  size_t total = 0;
  for (auto& e : plan) total += (e.second + 255) & ~size_t(255);
  if (cudaMalloc(&m->arena, total) != cudaSuccess) return bail(GPT2_ERR_OOM, "arena");
  m->arena_bytes = total;
  cudaMemset(m->arena, 0, total);
  size_t off = 0;
  for (auto& e : plan) {
    *e.first = m->arena + off;
    off += (e.second + 255) & ~size_t(255);
  }
  std::vector<float> init;
  host_init(m, seed, init);
  int r = gpt2_set_params(m, init.data(), m->n_logical);
  if (r) {
    gpt2_destroy(m);
    return r;
  }
  *out = m;
  return GPT2_OK;
}

int gpt2_set_stream(gpt2* m, void* stream) {
  if (!m) return GPT2_ERR_CONFIG;
  cudaStream_t s = (cudaStream_t)stream;
  if (!s) {
    if (!m->own_stream) {
      CK(m, cudaStreamCreateWithFlags(&m->stream, cudaStreamNonBlocking));
      m->own_stream = true;
    }
    return GPT2_OK;
  }
  if (m->own_stream) {
    CK(m, cudaStreamSynchronize(m->stream));
    cudaStreamDestroy(m->stream);
    m->own_stream = false;
  }
  m->stream = s;
  return GPT2_OK;
}

int gpt2_forward_backward(gpt2* m, const int32_t* tokens, const int32_t* targets, int B, int T, float* loss_out) {
  RK(validate_batch(m, tokens, targets, B, T));
  if (m->k > 0 && (B != m->k_B || T != m->k_T))
    return set_err(m, GPT2_ERR_BATCH, "all accumulated micro-batches must have the same B and T");
  RK(copy_tokens(m, m->tok, tokens, (size_t)B * T));
  RK(copy_tokens(m, m->tgt, targets, (size_t)B * T));
  RK(run_micro_batch(m, B, T, true));
  m->k += 1;
  m->k_B = B;
  m->k_T = T;
  if (loss_out) {
    CK(m, cudaMemcpyAsync(loss_out, m->d_loss, 4, cudaMemcpyDeviceToHost, m->stream));
    RK(check_device_error(m));
  }
  return GPT2_OK;
}

int gpt2_forward(gpt2* m, const int32_t* tokens, const int32_t* targets, int B, int T, float* loss_out) {
  RK(validate_batch(m, tokens, targets, B, T));
  RK(copy_tokens(m, m->tok, tokens, (size_t)B * T));
  RK(copy_tokens(m, m->tgt, targets, (size_t)B * T));
  RK(run_micro_batch(m, B, T, false));
  if (loss_out) {
    CK(m, cudaMemcpyAsync(loss_out, m->d_loss, 4, cudaMemcpyDeviceToHost, m->stream));
    RK(check_device_error(m));
  }
  return GPT2_OK;
}

int gpt2_read_loss(gpt2* m, float* loss_out) {
  if (!m || !loss_out) return GPT2_ERR_CONFIG;
  CK(m, cudaMemcpyAsync(loss_out, m->d_loss, 4, cudaMemcpyDeviceToHost, m->stream));
  return check_device_error(m);
}

int gpt2_step(gpt2* m, float lr, float wd, float beta1, float beta2, float* grad_norm_out) {
  if (!m) return GPT2_ERR_CONFIG;
  if (m->k == 0) return set_err(m, GPT2_ERR_NO_GRAD, "step without an accumulated micro-batch");
  LaunchCtx c = m->ctx();
  m->t += 1;
  ProfScope ps(c, CAT_ADAMW, 0.0, (double)m->n_store * 36 + (m->cfg.dtype == GPT2_BF16 ? 2.0 * m->n_decay : 0.0));
  sumsq_partial_kernel<<<m->norm_parts, ADAM_THREADS, 0, m->stream>>>(m->g, m->n_store, m->d_norm_part);
  RK(check_launch(c, "sumsq_partial"));
  AdamArgs a{};
  a.p = m->p;
  a.g = m->g;
  a.m = m->m;
  a.v = m->v;
  a.shadow = m->cfg.dtype == GPT2_BF16 ? m->shadow : nullptr;
  a.n = m->n_store;
  a.n_decay = m->n_decay;
  a.partial = m->d_norm_part;
  a.nparts = m->norm_parts;
  a.inv_k = 1.0f / (float)m->k;
  a.lr = lr;
  a.wd = wd;
  a.b1 = beta1;
  a.b2 = beta2;
  a.step_size = (float)(lr / (1.0 - std::pow((double)beta1, (double)m->t)));
  a.inv_sqrt_bc2 = (float)(1.0 / std::sqrt(1.0 - std::pow((double)beta2, (double)m->t)));
  a.gnorm_out = m->d_gnorm;
  a.sumsq_total = nullptr;
  a.zero_grad = 1;
  adamw_kernel<<<8 * m->num_sms, ADAM_THREADS, 0, m->stream>>>(a);
  RK(check_launch(c, "adamw"));
  m->k = 0;
  if (grad_norm_out) {
    CK(m, cudaMemcpyAsync(grad_norm_out, m->d_gnorm, 4, cudaMemcpyDeviceToHost, m->stream));
    RK(check_device_error(m));
  }
  return GPT2_OK;
}

int gpt2_grad_sumsq(gpt2* m, int64_t lo, int64_t hi, double* dev_out) {
  if (!m || !dev_out) return GPT2_ERR_CONFIG;
  if (lo < 0 || hi < lo || hi > m->n_store || lo % 64 || hi % 64)
    return set_err(m, GPT2_ERR_CONFIG, "0 <= lo <= hi <= storage length, both multiples of 64");
  LaunchCtx c = m->ctx();
  ProfScope ps(c, CAT_ADAMW, 0.0, 4.0 * (double)(hi - lo));
  sumsq_partial_kernel<<<m->norm_parts, ADAM_THREADS, 0, m->stream>>>(m->g + lo, hi - lo, m->d_norm_part);
  RK(check_launch(c, "sumsq_partial"));
  sum_partials_kernel<<<1, 32, 0, m->stream>>>(m->d_norm_part, m->norm_parts, dev_out);
  return check_launch(c, "sum_partials");
}

int gpt2_step_range(gpt2* m, float lr, float wd, float beta1, float beta2, int64_t lo, int64_t hi,
                    const double* dev_sumsq, float* grad_norm_out) {
  if (!m || !dev_sumsq) return GPT2_ERR_CONFIG;
  if (lo < 0 || hi < lo || hi > m->n_store || lo % 64 || hi % 64)
    return set_err(m, GPT2_ERR_CONFIG, "0 <= lo <= hi <= storage length, both multiples of 64");
  if (m->k == 0) return set_err(m, GPT2_ERR_NO_GRAD, "step without an accumulated micro-batch");
  LaunchCtx c = m->ctx();
  m->t += 1;
  const int64_t n = hi - lo;
  const int64_t nd = std::min<int64_t>(std::max<int64_t>(m->n_decay - lo, 0), n);
  {
    ProfScope ps(c, CAT_ADAMW, 0.0, (double)n * 32 + (m->cfg.dtype == GPT2_BF16 ? 2.0 * nd : 0.0));
    AdamArgs a{};
    a.p = m->p + lo;
    a.g = m->g + lo;
    a.m = m->m + lo;
    a.v = m->v + lo;
    a.shadow = m->cfg.dtype == GPT2_BF16 ? m->shadow + lo : nullptr;
    a.n = n;
    a.n_decay = nd;
    a.partial = nullptr;
    a.nparts = 0;
    a.inv_k = 1.0f / (float)m->k;
    a.lr = lr;
    a.wd = wd;
    a.b1 = beta1;
    a.b2 = beta2;
    a.step_size = (float)(lr / (1.0 - std::pow((double)beta1, (double)m->t)));
    a.inv_sqrt_bc2 = (float)(1.0 / std::sqrt(1.0 - std::pow((double)beta2, (double)m->t)));
    a.gnorm_out = m->d_gnorm;
    a.sumsq_total = dev_sumsq;
    a.zero_grad = 0;
    adamw_kernel<<<8 * m->num_sms, ADAM_THREADS, 0, m->stream>>>(a);
    RK(check_launch(c, "adamw_range"));
  }
  m->k = 0;
  if (grad_norm_out) {
    CK(m, cudaMemcpyAsync(grad_norm_out, m->d_gnorm, 4, cudaMemcpyDeviceToHost, m->stream));
    RK(check_device_error(m));
  }
  return GPT2_OK;
}

int gpt2_param_buffer(gpt2* m, float** dev, int64_t* n) {
  if (!m || !dev || !n) return GPT2_ERR_CONFIG;
  *dev = m->p;
  *n = m->n_store;
  return GPT2_OK;
}

int gpt2_refresh_shadow(gpt2* m) {
  if (!m) return GPT2_ERR_CONFIG;
  if (m->cfg.dtype != GPT2_BF16) return GPT2_OK;
  LaunchCtx c = m->ctx();
  ProfScope ps(c, CAT_ADAMW, 0.0, 6.0 * (double)m->n_decay);
  cast_shadow_kernel<<<8 * m->num_sms, 256, 0, m->stream>>>(m->p, m->shadow, m->n_decay);
  return check_launch(c, "cast_shadow");
}

int gpt2_zero_grad(gpt2* m) {
  if (!m) return GPT2_ERR_CONFIG;
  CK(m, cudaMemsetAsync(m->g, 0, (size_t)m->n_store * 4, m->stream));
  m->k = 0;
  return GPT2_OK;
}

int gpt2_num_params(const gpt2* m, int64_t* out) {
  if (!m || !out) return GPT2_ERR_CONFIG;
  *out = m->n_logical;
  return GPT2_OK;
}

int gpt2_tensor_info(const gpt2* m, int i, char* name, int name_len, int64_t* rows, int64_t* cols, int* ndim,
                     int64_t* offset) {
  if (!m || i < 0 || i >= (int)m->tensors.size()) return GPT2_ERR_CONFIG;
  const TensorSlot& t = m->tensors[i];
  if (name && name_len > 0) std::snprintf(name, name_len, "%s", t.name.c_str());
  if (rows) *rows = t.rows;
  if (cols) *cols = t.cols;
  if (ndim) *ndim = t.ndim;
  if (offset) *offset = t.canon_off;
  return GPT2_OK;
}

namespace {
// Copy between canonical host order and device storage for one state buffer.
int xfer(gpt2* m, float* dev, float* host, const float* host_in, int64_t n, bool to_host, float scale) {
  if (n != m->n_logical) return set_err(m, GPT2_ERR_CONFIG, "n must equal the logical parameter count");
  for (auto& t : m->tensors) {
    const size_t bytes = (size_t)(t.rows * t.cols) * 4;
    if (to_host)
      CK(m, cudaMemcpyAsync(host + t.canon_off, dev + t.dev_off, bytes, cudaMemcpyDeviceToHost, m->stream));
    else
      CK(m, cudaMemcpyAsync(dev + t.dev_off, host_in + t.canon_off, bytes, cudaMemcpyHostToDevice, m->stream));
  }
  CK(m, cudaStreamSynchronize(m->stream));
  if (to_host && scale != 1.0f)
    for (int64_t i = 0; i < n; ++i) host[i] *= scale;
  return GPT2_OK;
}
}  // namespace

int gpt2_get_params(gpt2* m, float* host, int64_t n) {
  if (!m || !host) return GPT2_ERR_CONFIG;
  RK(xfer(m, m->p, host, nullptr, n, true, 1.0f));
  return check_device_error(m);
}

int gpt2_set_params(gpt2* m, const float* host, int64_t n) {
  if (!m || !host) return GPT2_ERR_CONFIG;
  RK(xfer(m, m->p, nullptr, host, n, false, 1.0f));
  if (m->cfg.dtype == GPT2_BF16) {
    cast_shadow_kernel<<<8 * m->num_sms, 256, 0, m->stream>>>(m->p, m->shadow, m->n_decay);
    LaunchCtx c = m->ctx();
    RK(check_launch(c, "cast_shadow"));
    CK(m, cudaStreamSynchronize(m->stream));
  }
  return GPT2_OK;
}

int gpt2_get_grads(gpt2* m, float* host, int64_t n) {
  if (!m || !host) return GPT2_ERR_CONFIG;
  if (m->k == 0) return set_err(m, GPT2_ERR_NO_GRAD, "no accumulated micro-batch");
  RK(xfer(m, m->g, host, nullptr, n, true, 1.0f / (float)m->k));
  return check_device_error(m);
}

int gpt2_get_adam(gpt2* m, float* m_host, float* v_host, int64_t n, int64_t* t_out) {
  if (!m || !m_host || !v_host) return GPT2_ERR_CONFIG;
  RK(xfer(m, m->m, m_host, nullptr, n, true, 1.0f));
  RK(xfer(m, m->v, v_host, nullptr, n, true, 1.0f));
  if (t_out) *t_out = m->t;
  return check_device_error(m);
}

int gpt2_set_adam(gpt2* m, const float* m_host, const float* v_host, int64_t n, int64_t t) {
  if (!m || !m_host || !v_host || t < 0) return GPT2_ERR_CONFIG;
  RK(xfer(m, m->m, nullptr, m_host, n, false, 1.0f));
  RK(xfer(m, m->v, nullptr, v_host, n, false, 1.0f));
  m->t = t;
  return check_device_error(m);
}

// ---------------- generation ----------------
namespace {
int64_t kv_seq_elems(const gpt2* m) { return (int64_t)m->T * 2 * m->C; }
bf16* kv_layer(gpt2* m, int l) { return m->kv + (int64_t)l * m->cfg.B_max * kv_seq_elems(m); }

// fp32 logits of B rows against the head weight: rows of ln_f output (bf16, row stride
// ldx), or with ln, fp32 residual rows that ln_f is applied to on the fly.
int head_logits(gpt2* m, const LaunchCtx& c, const void* rows, int64_t ldx, int B, float* logits_out, int64_t ld,
                bool ln = false) {
  const float* headw = m->cfg.tied ? m->wte : m->head;
  return gemv_bf16(c, EPI_F32, rows, ldx, B, (const bf16*)m->W(headw), m->cfg.V, m->C, nullptr, logits_out, ld,
                   nullptr, 0, ln ? m->lnf_g : nullptr, ln ? m->lnf_b : nullptr);
}

int check_generation(gpt2* m, float* logits_out, int64_t ld, int B) {
  if (!m) return GPT2_ERR_CONFIG;
  if (m->cfg.dtype != GPT2_BF16) return set_err(m, GPT2_ERR_CONFIG, "generation needs a bf16 model");
  if (m->hd != DEC_HD) return set_err(m, GPT2_ERR_CONFIG, "generation needs head size 64");
  if (!logits_out || ld < m->cfg.V) return set_err(m, GPT2_ERR_CONFIG, "logits_out with ld >= V required");
  if (B < 1 || B > m->cfg.B_max || B > DEC_MAX_B) return set_err(m, GPT2_ERR_BATCH, "1 <= B <= min(B_max, 16)");
  return GPT2_OK;
}
}  // namespace

int gpt2_prefill(gpt2* m, const int32_t* tokens, int B, int T0, float* logits_out, int64_t ld) {
  RK(check_generation(m, logits_out, ld, B));
  if (!tokens) return set_err(m, GPT2_ERR_CONFIG, "tokens required");
  if (T0 < 1 || T0 > m->T) return set_err(m, GPT2_ERR_SEQ_TOO_LONG, "1 <= T0 <= block size");
  if (m->k > 0) return set_err(m, GPT2_ERR_BATCH, "prefill between micro-batches of an accumulation");
  if (!m->kv) {
    const size_t bytes = (size_t)m->L * m->cfg.B_max * kv_seq_elems(m) * sizeof(bf16);
    const size_t part = (size_t)m->cfg.B_max * m->NH * DEC_MAX_SPLIT * DEC_PART * sizeof(float);
    if (cudaMalloc(&m->kv, bytes) != cudaSuccess || cudaMalloc(&m->d_pos, 256) != cudaSuccess ||
        cudaMalloc(&m->dec_part, part) != cudaSuccess) {
      cudaGetLastError();
      cudaFree(m->kv);
      cudaFree(m->d_pos);
      m->kv = nullptr;
      m->d_pos = nullptr;
      m->dec_part = nullptr;
      return set_err(m, GPT2_ERR_OOM, "key/value cache");
    }
  }
  RK(copy_tokens(m, m->tok, tokens, (size_t)B * T0));
  RK(forward_layers(m, B, T0));
  LaunchCtx c = m->ctx();
  const int64_t N3C = 3 * (int64_t)m->Nmax * m->C;
  for (int l = 0; l < m->L; ++l)
    RK(kv_fill(c, (const bf16*)(m->qkv + (int64_t)l * N3C * m->act_bytes), B, T0, m->C, kv_layer(m, l),
               kv_seq_elems(m)));
  // the last position of each prompt: rows b*T0 + T0-1 of ln_f's output
  RK(head_logits(m, c, (const bf16*)m->xf + (int64_t)(T0 - 1) * m->C, (int64_t)T0 * m->C, B, logits_out, ld));
  set_pos_kernel<<<1, 1, 0, m->stream>>>(m->d_pos, T0);
  RK(check_launch(c, "set_pos"));
  m->kv_B = B;
  m->kv_len = T0;
  return check_device_error(m);
}

namespace {
// Enqueue one decode step for the B tokens in m->tok at the position in m->d_pos (which
// the step then advances): no synchronisation, so that it can be captured.
int decode_body(gpt2* m, int B, float* logits_out, int64_t ld) {
  LaunchCtx c = m->ctx();
  const int C = m->C, F = m->F;
  float* x0 = m->x;
  float* x1 = m->x + (int64_t)B * C;
  bf16* qkv = (bf16*)m->qkv;
  bf16* att = (bf16*)m->att;
  bf16* a = (bf16*)m->a;
  const int S = decode_splits(B, m->NH, m->num_sms);
  {
    ProfScope ps(c, CAT_EMB_FWD, 0.0, 12.0 * B * C);
    embed_decode_kernel<<<(B * 32 + 255) / 256, 256, 0, m->stream>>>(m->tok, m->wte, m->wpe, m->d_pos, x0, B, C,
                                                                    m->cfg.V, m->d_err);
    RK(check_launch(c, "embed_decode"));
  }
  // every later kernel of the step starts as a programmatic dependent of the one before:
  // it fetches its weights while that one finishes and waits for it before reading
  // activations or writing anything
  c.pdl = true;
  // each LayerNorm is applied inside the product that consumes it
  for (int l = 0; l < m->L; ++l) {
    const LayerP& w = m->lp[l];
    RK(gemv_bf16(c, EPI_BF16, x0, C, B, (const bf16*)m->W(w.qkv_w), 3 * C, C, w.qkv_b, qkv, 3 * C, nullptr, 0,
                 w.ln1_g, w.ln1_b));
    RK(decode_attention(c, qkv, kv_layer(m, l), kv_seq_elems(m), m->T, B, C, m->NH, m->d_pos, S, att, m->dec_part,
                        (double)m->kv_len + 1.0));
    RK(gemv_bf16(c, EPI_F32_RESID, att, C, B, (const bf16*)m->W(w.ao_w), C, C, w.ao_b, x1, C, x0, C));
    RK(gemv_bf16(c, EPI_BF16_GELU, x1, C, B, (const bf16*)m->W(w.fc_w), F, C, w.fc_b, a, F, nullptr, 0, w.ln2_g,
                 w.ln2_b));
    RK(gemv_bf16(c, EPI_F32_RESID, a, F, B, (const bf16*)m->W(w.pj_w), C, F, w.pj_b, x0, C, x1, C));
  }
  RK(head_logits(m, c, x0, C, B, logits_out, ld, true));
  set_pos_kernel<<<1, 1, 0, m->stream>>>(m->d_pos, -1);
  return check_launch(c, "set_pos");
}

// Capture decode_body into a CUDA graph for (B, logits_out, ld).
int capture_decode(gpt2* m, int B, float* logits_out, int64_t ld) {
  if (m->dec_graph) {
    cudaGraphExecDestroy(m->dec_graph);
    m->dec_graph = nullptr;
  }
  const long long before = m->launches;
  gemv_prepare();  // function attributes are set outside the capture
  CK(m, cudaStreamBeginCapture(m->stream, cudaStreamCaptureModeThreadLocal));
  const int r = decode_body(m, B, logits_out, ld);
  cudaGraph_t g = nullptr;
  const cudaError_t e = cudaStreamEndCapture(m->stream, &g);
  if (r || e != cudaSuccess) {
    if (g) cudaGraphDestroy(g);
    cudaGetLastError();
    return r ? r : cuda_err(m, e, "decode step capture");
  }
  const cudaError_t ei = cudaGraphInstantiate(&m->dec_graph, g, 0);
  cudaGraphDestroy(g);
  if (ei != cudaSuccess) {
    m->dec_graph = nullptr;
    return cuda_err(m, ei, "decode step graph");
  }
  m->dec_graph_launches = m->launches - before;
  m->launches = before;
  m->dec_B = B;
  m->dec_logits = logits_out;
  m->dec_ld = ld;
  return GPT2_OK;
}
}  // namespace

int gpt2_decode_step(gpt2* m, const int32_t* tokens, int B, float* logits_out, int64_t ld) {
  RK(check_generation(m, logits_out, ld, B));
  if (!tokens) return set_err(m, GPT2_ERR_CONFIG, "tokens required");
  if (!m->kv || m->kv_len == 0) return set_err(m, GPT2_ERR_CONFIG, "decode step before a prefill");
  if (B != m->kv_B) return set_err(m, GPT2_ERR_BATCH, "B must equal the prefill's B");
  if (m->kv_len >= m->T) return set_err(m, GPT2_ERR_SEQ_TOO_LONG, "the cache holds block-size positions");
  RK(copy_tokens(m, m->tok, tokens, (size_t)B));
  if (m->prof.on) {
    RK(decode_body(m, B, logits_out, ld));  // launch by launch, so that each kernel is timed
  } else {
    if (!m->dec_graph || m->dec_B != B || m->dec_logits != logits_out || m->dec_ld != ld)
      RK(capture_decode(m, B, logits_out, ld));
    CK(m, cudaGraphLaunch(m->dec_graph, m->stream));
    m->launches += m->dec_graph_launches;
  }
  m->kv_len += 1;
  return GPT2_OK;
}

int gpt2_sample_topk(gpt2* m, const float* logits, int64_t ld, int rows, int k, float temperature, float top_p,
                     const double* u, int32_t* idx_out) {
  if (!m) return GPT2_ERR_CONFIG;
  if (!logits || !u || !idx_out) return set_err(m, GPT2_ERR_CONFIG, "logits, u and idx_out are required");
  return sample_topk(m->ctx(), logits, ld, rows, m->cfg.V, k, temperature, top_p, u, idx_out);
}

int gpt2_synchronize(gpt2* m) {
  if (!m) return GPT2_ERR_CONFIG;
  return check_device_error(m);
}

int gpt2_kv_length(const gpt2* m, int* out) {
  if (!m || !out) return GPT2_ERR_CONFIG;
  *out = m->kv_len;
  return GPT2_OK;
}

int gpt2_grad_buffer(gpt2* m, float** dev, int64_t* n) {
  if (!m || !dev || !n) return GPT2_ERR_CONFIG;
  *dev = m->g;
  *n = m->n_store;
  return GPT2_OK;
}

int gpt2_storage_layout(const gpt2_config* cfg, int i, char* name, int name_len, int64_t* offset, int64_t* n,
                        int* bucket, int64_t* n_store) {
  if (!cfg || cfg->L <= 0 || cfg->C <= 0 || cfg->V <= 0 || cfg->T <= 0 || cfg->C % 64) return GPT2_ERR_CONFIG;
  gpt2 m;  // host-side layout only: no device state
  m.cfg = *cfg;
  m.Vp = (cfg->V + 63) / 64 * 64;
  build_tensors(&m);
  if (n_store) *n_store = m.n_store;
  if (i < 0 || i >= (int)m.tensors.size()) return GPT2_ERR_CONFIG;
  const TensorSlot& t = m.tensors[i];
  if (name && name_len > 0) std::snprintf(name, name_len, "%s", t.name.c_str());
  if (offset) *offset = t.dev_off;
  if (n) *n = t.dev_rows * t.cols;
  if (bucket) *bucket = tensor_bucket(&m, i);
  return GPT2_OK;
}

int gpt2_set_grad_events(gpt2* m, void* const* events, int n) {
  if (!m) return GPT2_ERR_CONFIG;
  if (n == 0) {
    m->grad_events.clear();
    return GPT2_OK;
  }
  if (n != m->cfg.L + 1 || !events) return set_err(m, GPT2_ERR_CONFIG, "expected L + 1 events");
  for (int i = 0; i < n; ++i)
    if (!events[i]) return set_err(m, GPT2_ERR_CONFIG, "null event");
  m->grad_events.assign(reinterpret_cast<const cudaEvent_t*>(events),
                        reinterpret_cast<const cudaEvent_t*>(events) + n);
  return GPT2_OK;
}

int gpt2_profile(gpt2* m, int enable) {
  if (!m) return GPT2_ERR_CONFIG;
  if (enable) m->prof.reset();
  m->prof.on = enable != 0;
  return GPT2_OK;
}

int gpt2_profile_read(gpt2* m, int cat, char* name, int name_len, double* ms, int64_t* launches, double* flops,
                      double* bytes) {
  if (!m || cat < 0 || cat >= CAT_COUNT) return GPT2_ERR_CONFIG;
  CK(m, cudaStreamSynchronize(m->stream));
  double t = 0, f = 0, b = 0;
  int64_t n = 0;
  for (auto& r : m->prof.recs) {
    if (r.cat != cat) continue;
    float e = 0.f;
    CK(m, cudaEventElapsedTime(&e, r.a, r.b));
    t += e;
    f += r.flops;
    b += r.bytes;
    ++n;
  }
  if (name && name_len > 0) std::snprintf(name, name_len, "%s", prof_cat_name(cat));
  if (ms) *ms = t;
  if (launches) *launches = n;
  if (flops) *flops = f;
  if (bytes) *bytes = b;
  return GPT2_OK;
}

int gpt2_launch_count(const gpt2* m, int64_t* out) {
  if (!m || !out) return GPT2_ERR_CONFIG;
  *out = m->launches;
  return GPT2_OK;
}

const char* gpt2_last_error(const gpt2* m) { return m ? m->err.c_str() : "null handle"; }

void gpt2_destroy(gpt2* m) {
  if (!m) return;
  if (m->stream) cudaStreamSynchronize(m->stream);
  cudaFree(m->arena);
  cudaFree(m->kv);
  cudaFree(m->d_pos);
  cudaFree(m->dec_part);
  if (m->dec_graph) cudaGraphExecDestroy(m->dec_graph);
  cudaFree(m->p);
  cudaFree(m->g);
  cudaFree(m->m);
  cudaFree(m->v);
  cudaFree(m->shadow);
  if (m->own_stream && m->stream) cudaStreamDestroy(m->stream);
  if (m->side.s) {
    cudaStreamSynchronize(m->side.s);
    cudaStreamDestroy(m->side.s);
  }
  if (m->side.ready) cudaEventDestroy(m->side.ready);
  if (m->side.joined) cudaEventDestroy(m->side.joined);
  for (auto& e : m->side.freed)
    if (e) cudaEventDestroy(e);
  delete m;
}

// ---------------------------------------------------------------------------
// op-level entry points
// ---------------------------------------------------------------------------
namespace {
struct OpCtx {
  LaunchCtx c;
  int* d_err = nullptr;
  cudaStream_t s;
  explicit OpCtx(void* stream) : s((cudaStream_t)stream) {
    c.stream = s;
    c.msg = &g_op_error;
    c.num_sms = device_sm_count();
  }
  int alloc_err() {
    if (cudaMallocAsync((void**)&d_err, sizeof(int), s) != cudaSuccess) return GPT2_ERR_OOM;
    cudaMemsetAsync(d_err, 0, sizeof(int), s);
    c.d_err = d_err;
    return GPT2_OK;
  }
  // synchronise and translate the device error word; frees it
  int finish() {
    int h = 0;
    if (d_err) {
      cudaMemcpyAsync(&h, d_err, sizeof(int), cudaMemcpyDeviceToHost, s);
      cudaFreeAsync(d_err, s);
      d_err = nullptr;
    }
    return sync_and_translate(s, h);
  }
  // after a device-to-host copy of the error word into h was enqueued on s
  static int sync_and_translate(cudaStream_t s, const int& h) {
    cudaError_t e = cudaStreamSynchronize(s);
    if (e != cudaSuccess) {
      g_op_error = cudaGetErrorString(e);
      return GPT2_ERR_CUDA;
    }
    if (h == DEV_TOKEN_RANGE) {
      g_op_error = "token or target id outside [0, V)";
      return GPT2_ERR_TOKEN_RANGE;
    }
    if (h == DEV_TIMEOUT) {
      g_op_error = "a bounded device-side wait gave up";
      return GPT2_ERR_TIMEOUT;
    }
    if (h) {
      g_op_error = "device error word set";
      return GPT2_ERR_CUDA;
    }
    return GPT2_OK;
  }
};
}  // namespace

int gpt2_op_gemm(int dtype, const void* A, int64_t lda, int a_mn, const void* B, int64_t ldb, int b_mn, int M, int N,
                 int K, int epilogue, void* out, int64_t ldo, void* out2, int64_t ldo2, const float* bias,
                 const void* aux, int64_t ld_aux, int accumulate, int ksplit, void* stream) {
  OpCtx o(stream);
  RK(o.alloc_err());
  float* ws = nullptr;
  if (dtype == GPT2_BF16 && epilogue == EPI_F32 && ksplit > 1) {
    const size_t n = (size_t)ksplit * M * N;
    if (cudaMallocAsync((void**)&ws, n * 4, o.s) != cudaSuccess) return GPT2_ERR_OOM;
    o.c.splitk_ws = ws;
    o.c.splitk_cap = n;
  }
  int r = gemm(o.c, dtype,
               GemmDesc{A, lda, a_mn != 0, B, ldb, b_mn != 0, M, N, K, epilogue, out, ldo, out2, ldo2, bias, aux,
                        ld_aux, accumulate, ksplit <= 0 ? 1 : ksplit});
  if (ws) cudaFreeAsync(ws, o.s);
  int r2 = o.finish();
  return r ? r : r2;
}

int gpt2_op_gemm_bench(const void* A, int64_t lda, int a_mn, const void* B, int64_t ldb, int b_mn, int M, int N, int K,
                       int epilogue, void* out, int64_t ldo, void* out2, int64_t ldo2, const float* bias,
                       const void* aux, int64_t ld_aux, int accumulate, int ksplit, int bn, int pair, int iters,
                       float* ms_out, void* stream) {
  if (iters <= 0 || !ms_out) {
    g_op_error = "gemm_bench: iters > 0 and ms_out required";
    return GPT2_ERR_CONFIG;
  }
  OpCtx o(stream);
  RK(o.alloc_err());
  float* ws = nullptr;
  if (epilogue == EPI_F32 && ksplit != 1) {
    const size_t n = (size_t)(ksplit > 1 ? ksplit : 16) * M * N;
    if (cudaMallocAsync((void**)&ws, n * 4, o.s) != cudaSuccess) return GPT2_ERR_OOM;
    o.c.splitk_ws = ws;
    o.c.splitk_cap = n;
  }
  GemmDesc d{A, lda, a_mn != 0, B, ldb, b_mn != 0, M, N, K, epilogue, out, ldo, out2, ldo2, bias, aux, ld_aux,
             accumulate, ksplit < 0 ? 1 : ksplit};
  d.bn = bn;
  d.pair = pair;
  int r = gemm_tc(o.c, d);  // warm-up (also sets kernel attributes)
  cudaEvent_t e0, e1;
  cudaEventCreate(&e0);
  cudaEventCreate(&e1);
  cudaEventRecord(e0, o.s);
  for (int i = 0; i < iters && !r; ++i) r = gemm_tc(o.c, d);
  cudaEventRecord(e1, o.s);
  if (ws) cudaFreeAsync(ws, o.s);
  int r2 = o.finish();
  float ms = 0.f;
  cudaEventElapsedTime(&ms, e0, e1);
  cudaEventDestroy(e0);
  cudaEventDestroy(e1);
  *ms_out = ms / iters;
  return r ? r : r2;
}

int gpt2_op_gemv(const void* x, int64_t ldx, int B, const void* W, int N, int K, int epilogue, const float* bias,
                 void* out, int64_t ldo, const float* resid, int64_t ldr, const float* ln_g, const float* ln_b,
                 int iters, int pdl, float* ms_out, void* stream) {
  if (!x || !W || !out || iters < 1 || (iters > 1 && !ms_out)) {
    g_op_error = "gemv: x, W, out required; iters >= 1 (ms_out with iters > 1)";
    return GPT2_ERR_CONFIG;
  }
  OpCtx o(stream);
  RK(o.alloc_err());
  auto one = [&]() {
    return gemv_bf16(o.c, epilogue, x, ldx, B, (const bf16*)W, N, K, bias, out, ldo, resid, ldr, ln_g, ln_b);
  };
  int r = one();  // warm-up (sets kernel attributes)
  if (!r && iters > 1) {
    o.c.pdl = pdl != 0;
    cudaEvent_t e0, e1;
    cudaEventCreate(&e0);
    cudaEventCreate(&e1);
    cudaEventRecord(e0, o.s);
    for (int i = 0; i < iters && !r; ++i) r = one();
    cudaEventRecord(e1, o.s);
    cudaEventSynchronize(e1);
    float ms = 0.f;
    cudaEventElapsedTime(&ms, e0, e1);
    cudaEventDestroy(e0);
    cudaEventDestroy(e1);
    *ms_out = ms / iters;
  }
  int r2 = o.finish();
  return r ? r : r2;
}

int gpt2_op_layernorm_fwd(int dtype, const float* x, const float* g, const float* b, int N, int C, void* y,
                          float* mean, float* rstd, void* stream) {
  OpCtx o(stream);
  if (C % 4 || C > 2048 || N <= 0) {
    g_op_error = "layernorm: C % 4 == 0, C <= 2048, N > 0 required";
    return GPT2_ERR_CONFIG;
  }
  if (((uintptr_t)x | (uintptr_t)g | (uintptr_t)b | (uintptr_t)y) & 15) {
    g_op_error = "layernorm: x, g, b and y must start on 16-byte boundaries";
    return GPT2_ERR_CONFIG;
  }
  return dtype == GPT2_BF16 ? layernorm_fwd_t<bf16>(o.c, x, g, b, N, C, (bf16*)y, mean, rstd)
                            : layernorm_fwd_t<float>(o.c, x, g, b, N, C, (float*)y, mean, rstd);
}

int gpt2_op_layernorm_bwd(int dtype, const float* dy, const float* x, const float* g, const float* mean,
                          const float* rstd, int N, int C, float* dres, void* dres_act, int accumulate, float* dg,
                          float* db, int accumulate_params, void* stream) {
  OpCtx o(stream);
  if (C % 4 || C > 2048 || N <= 0) {
    g_op_error = "layernorm: C % 4 == 0, C <= 2048, N > 0 required";
    return GPT2_ERR_CONFIG;
  }
  {
    const uintptr_t any = (uintptr_t)dy | (uintptr_t)x | (uintptr_t)g | (uintptr_t)dres | (uintptr_t)dres_act;
    if (any & 15) {
      g_op_error = "layernorm: dy, x, g, dres and dres_act must start on 16-byte boundaries";
      return GPT2_ERR_CONFIG;
    }
  }
  const int grid = ln_bwd_grid(N, C, o.c.num_sms);
  float* part = nullptr;
  if (cudaMallocAsync((void**)&part, (size_t)3 * grid * C * 4, o.s) != cudaSuccess) return GPT2_ERR_OOM;
  int r = dtype == GPT2_BF16
              ? layernorm_bwd_t<bf16>(o.c, dy, x, g, mean, rstd, N, C, dres, (bf16*)dres_act, accumulate, part, dg, db,
                                      nullptr, accumulate_params)
              : layernorm_bwd_t<float>(o.c, dy, x, g, mean, rstd, N, C, dres, (float*)dres_act, accumulate, part, dg,
                                       db, nullptr, accumulate_params);
  cudaFreeAsync(part, o.s);
  return r;
}

int gpt2_op_attention_fwd(int dtype, const void* qkv, int B, int T, int NH, int hd, void* out, float* lse,
                          void* stream) {
  OpCtx o(stream);
  if (B <= 0 || T <= 0 || NH <= 0) {
    g_op_error = "attention: empty shape";
    return GPT2_ERR_CONFIG;
  }
  RK(o.alloc_err());
  int r = attention_fwd(o.c, dtype, qkv, B, T, NH, hd, out, lse);
  int r2 = o.finish();
  return r ? r : r2;
}

int gpt2_op_attention_bwd(int dtype, const void* qkv, const void* out, const void* dout, const float* lse, int B,
                          int T, int NH, int hd, void* dqkv, void* stream) {
  OpCtx o(stream);
  if (B <= 0 || T <= 0 || NH <= 0) {
    g_op_error = "attention: empty shape";
    return GPT2_ERR_CONFIG;
  }
  RK(o.alloc_err());
  float* D = nullptr;
  if (cudaMallocAsync((void**)&D, (size_t)B * NH * T * 4, o.s) != cudaSuccess) {
    o.finish();
    return GPT2_ERR_OOM;
  }
  int r = attention_bwd(o.c, dtype, qkv, out, dout, lse, B, T, NH, hd, dqkv, D);
  cudaFreeAsync(D, o.s);
  int r2 = o.finish();
  return r ? r : r2;
}

int gpt2_op_attention_bwd_stored(const void* qkv, const void* out, const void* dout, const float* lse, int B, int T,
                                 int NH, int hd, void* dqkv, void* ds, void* stream) {
  OpCtx o(stream);
  if (B <= 0 || T <= 0 || NH <= 0) {
    g_op_error = "attention: empty shape";
    return GPT2_ERR_CONFIG;
  }
  if (!ds) {
    g_op_error = "attention_bwd_stored: no dS workspace";
    return GPT2_ERR_CONFIG;
  }
  RK(o.alloc_err());
  float* D = nullptr;
  if (cudaMallocAsync((void**)&D, (size_t)B * NH * T * 4, o.s) != cudaSuccess) {
    o.finish();
    return GPT2_ERR_OOM;
  }
  int r = attention_bwd(o.c, GPT2_BF16, qkv, out, dout, lse, B, T, NH, hd, dqkv, D, nullptr, ds);
  cudaFreeAsync(D, o.s);
  int r2 = o.finish();
  return r ? r : r2;
}

size_t gpt2_attention_ds_bytes(int B, int T, int NH) {
  return B > 0 && T > 0 && NH > 0 ? attn_ds_bytes(B, T, NH) : 0;
}

int gpt2_op_embedding_fwd(const int32_t* tokens, const float* wte, const float* wpe, int B, int T, int C, int V,
                          float* x0, void* stream) {
  OpCtx o(stream);
  RK(o.alloc_err());
  int r = embedding_fwd(o.c, tokens, wte, wpe, B * T, T, C, V, x0);
  int r2 = o.finish();
  return r ? r : r2;
}

int gpt2_op_token_buckets(const int32_t* tokens, int N, int V, int32_t* sorted_pos, int32_t* seg_id,
                          int32_t* seg_start, int32_t* nseg_out, void* stream) {
  OpCtx o(stream);
  if (N <= 0 || N > EMB_MAX_TOKENS) {
    g_op_error = "token_buckets: 0 < N <= 32768 required";
    return GPT2_ERR_BATCH;
  }
  RK(o.alloc_err());
  void* scratch = nullptr;
  if (cudaMallocAsync(&scratch, emb_scratch_bytes(N, 4), o.s) != cudaSuccess) return GPT2_ERR_OOM;
  EmbScratch es = emb_scratch_carve(scratch, N, 4);
  int r = token_sort(o.c, tokens, N, V, es);
  int counts[2] = {0, 0};
  std::vector<int> chunk_start, seg_chunk0;
  if (!r) {
    cudaMemcpyAsync(counts, es.counts, 8, cudaMemcpyDeviceToHost, o.s);
    cudaStreamSynchronize(o.s);
    chunk_start.resize(counts[1] + 1);
    seg_chunk0.resize(counts[0] + 1);
    cudaMemcpyAsync(chunk_start.data(), es.chunk_start, (counts[1] + 1) * 4, cudaMemcpyDeviceToHost, o.s);
    cudaMemcpyAsync(seg_chunk0.data(), es.seg_chunk0, (counts[0] + 1) * 4, cudaMemcpyDeviceToHost, o.s);
    cudaMemcpyAsync(sorted_pos, es.sorted_pos, (size_t)N * 4, cudaMemcpyDeviceToDevice, o.s);
    cudaMemcpyAsync(seg_id, es.seg_id, (size_t)counts[0] * 4, cudaMemcpyDeviceToDevice, o.s);
    cudaStreamSynchronize(o.s);
    std::vector<int> starts(counts[0] + 1);
    for (int s = 0; s <= counts[0]; ++s) starts[s] = chunk_start[seg_chunk0[s]];
    cudaMemcpyAsync(seg_start, starts.data(), (counts[0] + 1) * 4, cudaMemcpyHostToDevice, o.s);
    if (nseg_out) *nseg_out = counts[0];
  }
  cudaFreeAsync(scratch, o.s);
  int r2 = o.finish();
  return r ? r : r2;
}

int gpt2_op_embedding_bwd(const int32_t* tokens, const float* dx0, int B, int T, int C, int V, float* dwte,
                          float* dwpe, void* stream) {
  OpCtx o(stream);
  const int N = B * T;
  if (N <= 0 || N > EMB_MAX_TOKENS || C % 4) {
    g_op_error = "embedding_bwd: 0 < B*T <= 32768 and C % 4 == 0 required";
    return GPT2_ERR_CONFIG;
  }
  RK(o.alloc_err());
  void* scratch = nullptr;
  if (cudaMallocAsync(&scratch, emb_scratch_bytes(N, C), o.s) != cudaSuccess) return GPT2_ERR_OOM;
  EmbScratch es = emb_scratch_carve(scratch, N, C);
  int r = embedding_bwd(o.c, tokens, dx0, B, T, C, V, dwte, dwpe, es);
  cudaFreeAsync(scratch, o.s);
  int r2 = o.finish();
  return r ? r : r2;
}

int gpt2_op_cross_entropy(int dtype, void* logits, int64_t ld, int N, int V, const int32_t* targets, float scale,
                          float* row_loss, void* stream) {
  OpCtx o(stream);
  RK(o.alloc_err());
  int r;
  if (dtype == GPT2_BF16 && N > 0) {
    // the training step's bf16 path: per-row softmax partials (here from the logits
    // themselves), then the one-pass gradient
    float2* stats = nullptr;
    if (cudaMallocAsync((void**)&stats, (size_t)N * sizeof(float2), o.s) != cudaSuccess) {
      o.finish();
      return GPT2_ERR_OOM;
    }
    r = cross_entropy_stats(o.c, (bf16*)logits, ld, N, V, targets, scale, row_loss, nullptr, 0, stats);
    cudaFreeAsync(stats, o.s);
  } else {
    r = cross_entropy(o.c, dtype, logits, ld, N, V, targets, scale, row_loss);
  }
  int r2 = o.finish();
  return r ? r : r2;
}

int gpt2_op_sample_topk(const float* logits, int64_t ld, int rows, int V, int k, float temperature, float top_p,
                        const double* u, int32_t* idx_out, void* stream) {
  if (!logits || !u || !idx_out) {
    g_op_error = "sample_topk: logits, u and idx_out are required";
    return GPT2_ERR_CONFIG;
  }
  OpCtx o(stream);
  RK(o.alloc_err());
  int r = sample_topk(o.c, logits, ld, rows, V, k, temperature, top_p, u, idx_out);
  int r2 = o.finish();
  return r ? r : r2;
}

int gpt2_op_bounded_wait_check(int arrive, unsigned long long limit_ns, void* stream) {
  if (limit_ns > 1000000000ull) {
    g_op_error = "bounded_wait_check: limit_ns must be at most 1e9";
    return GPT2_ERR_CONFIG;
  }
  OpCtx o(stream);
  RK(o.alloc_err());
  bounded_wait_check_kernel<<<1, 32, 0, o.s>>>(arrive, limit_ns, o.d_err);
  int r = check_launch(o.c, "bounded_wait_check");
  int r2 = o.finish();
  return r ? r : r2;
}

const char* gpt2_op_last_error(void) { return g_op_error.c_str(); }

}  // extern "C"

// ---------------------------------------------------------------------------
// Attention backward without any allocation. Its one scratch buffer (the
// per-row dot products D = rowsum(dO * O), B*NH*T floats) lives in a fixed
// file-scope device array instead of memory from cudaMallocAsync, for callers
// whose device memory is wholly owned by their own allocator or budget and who
// therefore may not allocate, or who cannot pay for an allocation per call.
// Every GPU that loads this library holds the array (4 MiB) until the process
// exits. All calls on a device share it and each call overwrites all of it that
// it uses before reading it; calls whose kernels overlap on the GPU (different
// streams or threads, no ordering between them) race on it. A second fixed word
// carries the kernels' error flag (a bounded wait that gave up): each call clears
// it before its kernels and reads it back after them, so the call synchronises
// its stream and reports a timeout like every other entry point.
// The first call on each device looks up both addresses (with that device
// current) and caches them; make that first call before any stream capture.
// ---------------------------------------------------------------------------
namespace {
constexpr long long kNoAllocAttnRows = 1LL << 20;  // max B*NH*T
static __device__ __align__(256) float g_noalloc_attn_D[kNoAllocAttnRows];
static __device__ __align__(256) int g_noalloc_attn_err;
std::mutex g_noalloc_mu;
constexpr int kMaxDevices = 64;
float* g_noalloc_attn_ptr[kMaxDevices] = {};
int* g_noalloc_err_ptr[kMaxDevices] = {};

int noalloc_attn_scratch(float** out, int** err_out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) {
    g_op_error = std::string("cudaGetDevice: ") + cudaGetErrorString(e);
    return GPT2_ERR_CUDA;
  }
  if (dev < 0 || dev >= kMaxDevices) {
    g_op_error = "attention_bwd_noalloc: device ordinal beyond 63";
    return GPT2_ERR_CONFIG;
  }
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  if (!g_noalloc_attn_ptr[dev]) {
    void* p = nullptr;
    void* q = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_attn_D);
    if (e == cudaSuccess) e = cudaGetSymbolAddress(&q, g_noalloc_attn_err);
    if (e != cudaSuccess || !p || !q) {
      g_op_error = std::string("cudaGetSymbolAddress: ") + cudaGetErrorString(e);
      return GPT2_ERR_CUDA;
    }
    g_noalloc_err_ptr[dev] = static_cast<int*>(q);
    g_noalloc_attn_ptr[dev] = static_cast<float*>(p);
  }
  *out = g_noalloc_attn_ptr[dev];
  *err_out = g_noalloc_err_ptr[dev];
  return GPT2_OK;
}
}  // namespace

extern "C" int gpt2_op_attention_bwd_noalloc(int dtype, const void* qkv, const void* out, const void* dout,
                                             const float* lse, int B, int T, int NH, int hd, void* dqkv,
                                             void* stream) {
  OpCtx o(stream);
  if (B <= 0 || T <= 0 || NH <= 0) {
    g_op_error = "attention: empty shape";
    return GPT2_ERR_CONFIG;
  }
  if ((long long)B * NH * T > kNoAllocAttnRows) {
    g_op_error = "attention_bwd_noalloc: B*NH*T = " + std::to_string((long long)B * NH * T) +
                 " exceeds the fixed scratch of " + std::to_string(kNoAllocAttnRows) + " rows";
    return GPT2_ERR_CONFIG;
  }
  float* D = nullptr;
  int* err = nullptr;
  RK(noalloc_attn_scratch(&D, &err));
  cudaError_t e = cudaMemsetAsync(err, 0, sizeof(int), o.s);
  if (e != cudaSuccess) {
    g_op_error = std::string("attention_bwd_noalloc: clearing the error word: ") + cudaGetErrorString(e);
    return GPT2_ERR_CUDA;
  }
  o.c.d_err = err;
  const int r = attention_bwd(o.c, dtype, qkv, out, dout, lse, B, T, NH, hd, dqkv, D);
  int h = 0;
  e = cudaMemcpyAsync(&h, err, sizeof(int), cudaMemcpyDeviceToHost, o.s);
  const int r2 = OpCtx::sync_and_translate(o.s, h);
  if (r) return r;
  if (e != cudaSuccess) {
    g_op_error = std::string("attention_bwd_noalloc: reading the error word: ") + cudaGetErrorString(e);
    return GPT2_ERR_CUDA;
  }
  return r2;
}
