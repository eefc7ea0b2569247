/* gpt2.h -- C ABI of the B200 (sm_100a) GPT-2 pre-LayerNorm training step.
 *
 * The library computes one training step of a GPT-2 decoder: token + position
 * embedding, L pre-LN blocks (causal multi-head attention, 4x tanh-GELU MLP,
 * residual connections), final LayerNorm, a bias-free head tied to the token
 * embedding (or a separate head), mean next-token cross-entropy, the backward
 * pass, gradient accumulation over micro-batches, global-norm clipping at 1.0 and
 * AdamW with weight decay on >= 2-D tensors only; and, for generation, the
 * forward of the last position with a key/value cache and temperature / top-k /
 * top-p sampling.
 * Sources (page titles and sections): "gpt/docs/LLM.md" Architecture Details
 * (Embedding Layer, Transformer Blocks, Output Layer); "GPT From Scratch" Key
 * decisions (pre-norm blocks, tanh-GELU, tying, padding 50,257 -> 50,304, decay
 * groups, clipping, accumulation); "AxonLM" Key Features and Training Recipe
 * (1/sqrt(2L) init, betas 0.9/0.95, decay 0.1, clip 1.0); "Genesis" Model Specs
 * (untied head, 163,009,536 parameters).
 *
 * Conventions for every call:
 *  - Return value: 0 (GPT2_OK) or a negative GPT2_ERR_* code; the message of the
 *    last failure on a handle is in gpt2_last_error(). Op-level calls (gpt2_op_*)
 *    have no handle; their last message is in gpt2_op_last_error().
 *  - Pointers are plain host or device addresses; sizes are element counts. No
 *    call keeps a caller pointer after it returns.
 *  - A handle is not thread-safe: one thread at a time per handle. Handles on
 *    different devices may be used from one process; kernel attributes are set
 *    once per device, under a lock.
 *  - All GPU work of a handle is enqueued on its stream (gpt2_set_stream); calls
 *    that return data to host memory synchronise that stream.
 *  - Kernels never trap. Bad token ids are caught on the device (recorded in a
 *    device error word and replaced by id 0 so that all accesses stay in bounds)
 *    and reported as GPT2_ERR_TOKEN_RANGE at the next call that synchronises.
 *    Every mbarrier wait inside a kernel is bounded; one that gives up is
 *    reported as GPT2_ERR_TIMEOUT.
 */
#ifndef GPT2_B200_H
#define GPT2_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

enum {
  GPT2_OK = 0,
  GPT2_ERR_CONFIG = -1,       /* invalid configuration or argument */
  GPT2_ERR_OOM = -2,          /* device allocation failed */
  GPT2_ERR_SEQ_TOO_LONG = -3, /* T > cfg.T (the block size) */
  GPT2_ERR_TOKEN_RANGE = -4,  /* a token or target id outside [0, V) */
  GPT2_ERR_BATCH = -5,        /* B > B_max, B differs between accumulated micro-batches, or B*T too large */
  GPT2_ERR_NO_GRAD = -6,      /* gpt2_step / gpt2_get_grads with no accumulated micro-batch */
  GPT2_ERR_CUDA = -7,         /* a CUDA runtime or driver call failed */
  GPT2_ERR_TIMEOUT = -8       /* a bounded device-side wait gave up */
};

enum { GPT2_FP32 = 0, GPT2_BF16 = 1 };

/* Model configuration.
 *  L layers, H heads, C width (C % H == 0; bf16 mode needs C / H == 64), T block
 *  size (maximum sequence length), V logical vocabulary (stored padded to a
 *  multiple of 64; padding rows are zero, excluded from the softmax, receive no
 *  gradient and are not counted as parameters), tied = 1 ties the head to wte,
 *  qkv_bias = 1 gives the QKV projection a bias (0 matches the untied
 *  163,009,536-parameter count), dtype GPT2_FP32 (fp32 everywhere) or GPT2_BF16
 *  (bf16 GEMM/attention operands, fp32 residual stream, LayerNorm, softmax and
 *  cross-entropy statistics, fp32 gradients, master weights and Adam state),
 *  B_max the largest micro-batch the handle's activation arena is sized for. */
typedef struct {
  int L, H, C, T, V, tied, qkv_bias, dtype, B_max;
} gpt2_config;

typedef struct gpt2 gpt2; /* opaque; the library owns all device memory it uses */

/* Create a model on the current CUDA device. Weights: N(0, 0.02), attention-out
 * and MLP-projection weights N(0, 0.02 / sqrt(2L)), biases 0, LayerNorm gains 1
 * and biases 0 ("AxonLM", Key Features: 1/sqrt(2L) for residual projections).
 * The draws: element j of tensor i
 * (canonical order) takes two splitmix64 outputs of seed ^ (i << 40) ^ 2j and
 * ^ (2j + 1), maps them to u1 in (0, 1] and u2 in [0, 1), and uses the cos branch
 * of Box-Muller, computed on the host in double and rounded to fp32.
 * Allocates parameters, gradients, Adam state, the bf16 shadow and the
 * activation arena for B_max * T tokens (in bf16 mode it includes one layer's
 * attention dS workspace, gpt2_attention_ds_bytes(B_max, T, H) bytes, which grows
 * with T^2: 384 MiB at B_max = 16, T = 1024, H = 12). On failure *out is NULL and an
 * arena larger than the free device memory returns GPT2_ERR_OOM. */
int gpt2_create(const gpt2_config* cfg, uint64_t seed, gpt2** out);

/* Use `stream` (a cudaStream_t, e.g. torch.cuda.current_stream().cuda_stream) for
 * all later work; NULL selects the library's own stream. */
int gpt2_set_stream(gpt2* m, void* stream);

/* Forward + backward of one micro-batch of B sequences of length T (T <= cfg.T).
 * The forward is the pre-LN stack of "gpt/docs/LLM.md", Architecture Details
 * (embedding, blocks x += attn(ln_1(x)); x += mlp(ln_2(x)), final LayerNorm, head);
 * the loss is the mean next-token cross-entropy over all B*T positions ("GPT From
 * Scratch", Architecture diagram: the train loop and estimate_loss use the model's
 * loss); gradients are accumulated over micro-batches ("GPT From Scratch", Key
 * decisions: accumulation equals one large batch; "AxonLM", Key Features: gradient
 * accumulation set by the total and micro batch sizes, and Training Recipe: an
 * effective batch of 524,288 tokens).
 * tokens, targets: int32 [B, T], host or device memory (detected), copied in
 * before the call returns. Gradients of the micro-batch's mean cross-entropy
 * are ADDED to the accumulated gradients; the micro-batch count k grows by 1.
 * All micro-batches accumulated before one step must have the same B and T.
 * loss_out (nullable, host): mean cross-entropy of this micro-batch; when
 * given, the call synchronises the stream. */
int gpt2_forward_backward(gpt2* m, const int32_t* tokens, const int32_t* targets, int B, int T, float* loss_out);

/* Forward only (no gradients, no change to k): the same forward and loss as
 * gpt2_forward_backward, for evaluation ("GPT From Scratch", Architecture diagram:
 * estimate_loss on held-out batches). loss_out as above (nullable). */
int gpt2_forward(gpt2* m, const int32_t* tokens, const int32_t* targets, int B, int T, float* loss_out);

/* The mean loss of the most recent gpt2_forward_backward or gpt2_forward call, read
 * later (for a call made with loss_out = NULL so that it did not wait for the GPU).
 * Synchronises the handle's stream; GPT2_ERR_CONFIG for a NULL loss_out; a device
 * error raised since the last check is returned as in gpt2_forward_backward. */
int gpt2_read_loss(gpt2* m, float* loss_out);

/* Optimizer step ("AxonLM", Training Recipe: betas (0.9, 0.95), weight decay 0.1
 * on 2-D tensors only, gradient clip 1.0; "GPT From Scratch", Key decisions: AdamW
 * decays only parameters of two or more dimensions, clipping at 1.0) on the
 * accumulated gradients: G = (sum of micro-batch
 * gradients) / k; global-norm clip to 1.0 (coefficient 1 / (||G|| + 1e-6) when
 * below 1); AdamW with eps 1e-8, bias correction, decoupled decay
 * p <- p (1 - lr wd) on >= 2-D tensors only; t += 1; gradients zeroed; k = 0.
 * grad_norm_out (nullable, host): the pre-clip ||G||; when given, the call
 * synchronises. Returns GPT2_ERR_NO_GRAD when k == 0. */
int gpt2_step(gpt2* m, float lr, float wd, float beta1, float beta2, float* grad_norm_out);

/* Zero the accumulated gradients; k = 0. */
int gpt2_zero_grad(gpt2* m);

/* ------------------------------------------------------------------------
 * Sharded optimizer step for data parallelism (ZeRO stage 1: each of W ranks keeps
 * the full parameters, updates only its shard of parameters and optimizer state, and
 * the ranks exchange the updated shards). It computes exactly gpt2_step's update
 * ("AxonLM", Key Features: DDP multi-GPU; Training Recipe: clip 1.0, AdamW 0.9 /
 * 0.95, decay 0.1 on 2-D tensors), split by storage range. Ranges index the library's
 * flat storage (gpt2_grad_buffer, gpt2_param_buffer), whose length is a multiple of
 * 4096 floats; lo and hi must be multiples of 64 with 0 <= lo <= hi <= that length
 * (GPT2_ERR_CONFIG otherwise). Sequence per step: reduce-scatter the gradient buffer,
 * gpt2_grad_sumsq on the shard, sum the scalars over the ranks, gpt2_step_range on the
 * shard, all-gather the parameter shards, gpt2_refresh_shadow, gpt2_zero_grad.
 *
 * gpt2_grad_sumsq: *dev_out (DEVICE double) = sum over [lo, hi) of g^2, g the
 * accumulated gradient SUM over the k micro-batches (not divided by k). Asynchronous.
 * gpt2_step_range: gpt2_step restricted to [lo, hi), with the squared norm of the
 * whole accumulated gradient read from *dev_sumsq (DEVICE double: the sum of every
 * shard's gpt2_grad_sumsq): ||G|| = sqrt(sumsq) / k, the same clip, AdamW on [lo, hi)
 * (decay where the range overlaps the >= 2-D tensors), the bf16 shadow of [lo, hi)
 * refreshed; t += 1; k = 0. The gradient buffer is left unchanged (zero it with
 * gpt2_zero_grad). grad_norm_out as in gpt2_step; GPT2_ERR_NO_GRAD when k == 0.
 * gpt2_param_buffer: device address and length of the flat fp32 parameter storage
 * (owned by the handle, valid until gpt2_destroy).
 * gpt2_refresh_shadow: recast the whole bf16 weight shadow from the fp32 parameters
 * (after the parameter shards were exchanged). Asynchronous. */
int gpt2_grad_sumsq(gpt2* m, int64_t lo, int64_t hi, double* dev_out);
int gpt2_step_range(gpt2* m, float lr, float wd, float beta1, float beta2, int64_t lo, int64_t hi,
                    const double* dev_sumsq, float* grad_norm_out);
int gpt2_param_buffer(gpt2* m, float** dev, int64_t* n);
int gpt2_refresh_shadow(gpt2* m);

/* Logical parameter count (V rows, not the padded rows). */
int gpt2_num_params(const gpt2* m, int64_t* out);

/* Canonical tensor i: name (NUL-terminated, truncated to name_len), shape
 * (rows, cols; cols = 1 and ndim = 1 for vectors), offset in the canonical flat
 * order. Canonical order (PyTorch Linear convention W[out][in]): wte[V,C],
 * wpe[T,C]; per layer ln1_g, ln1_b, qkv_w[3C,C], qkv_b[3C] (if qkv_bias),
 * ao_w[C,C], ao_b, ln2_g, ln2_b, fc_w[4C,C], fc_b[4C], pj_w[C,4C], pj_b; lnf_g,
 * lnf_b; head_w[V,C] if untied. Returns GPT2_ERR_CONFIG past the last tensor. */
int gpt2_tensor_info(const gpt2* m, int i, char* name, int name_len, int64_t* rows, int64_t* cols, int* ndim,
                     int64_t* offset);

/* Copy parameters, averaged gradients ((1/k) sum, GPT2_ERR_NO_GRAD if k == 0)
 * or Adam moments between the device and n floats of HOST memory in canonical
 * order; n must equal gpt2_num_params. Synchronises. */
int gpt2_get_params(gpt2* m, float* host, int64_t n);
int gpt2_set_params(gpt2* m, const float* host, int64_t n); /* also refreshes the bf16 shadow */
int gpt2_get_grads(gpt2* m, float* host, int64_t n);
int gpt2_get_adam(gpt2* m, float* m_host, float* v_host, int64_t n, int64_t* t_out);
/* Restore the Adam moments and step count t (>= 0) from HOST memory, canonical order, for
 * resuming from a checkpoint (with gpt2_set_params). Returns GPT2_ERR_CONFIG on a NULL
 * pointer, n != gpt2_num_params or t < 0. Synchronises. */
int gpt2_set_adam(gpt2* m, const float* m_host, const float* v_host, int64_t n, int64_t t);

/* Device address and length (floats) of the flat fp32 gradient storage (the
 * library's internal, padded layout), e.g. for a data-parallel all-reduce of the
 * accumulated gradients between gpt2_forward_backward and gpt2_step. The buffer
 * holds the SUM over the k accumulated micro-batches; padding entries are zero.
 * Owned by the handle; valid until gpt2_destroy. */
int gpt2_grad_buffer(gpt2* m, float** dev, int64_t* n);

/* Storage layout, computed on the host from a configuration alone (no device, no
 * handle): for canonical tensor i (the order of gpt2_tensor_info), its offset and
 * length in floats in the flat device storage of parameters, gradients and Adam
 * moments (vocabulary tensors include their padding rows), and its gradient bucket:
 * layer l's tensors are bucket l, the embeddings, final LayerNorm and untied head
 * bucket L. *n_store (nullable) receives the storage length, also for an i past the
 * last tensor, which returns GPT2_ERR_CONFIG. The buckets exist for a data-parallel
 * exchange that overlaps the backward pass ("AxonLM", Key Features and Quick Start:
 * data-parallel training over several GPUs); see gpt2_set_grad_events. */
int gpt2_storage_layout(const gpt2_config* cfg, int i, char* name, int name_len, int64_t* offset, int64_t* n,
                        int* bucket, int64_t* n_store);

/* One-shot completion events for the gradient buckets of the NEXT gpt2_forward_backward
 * call (the last micro-batch before an exchange): events[b] (cudaEvent_t handles the
 * caller created on this handle's device, caller-owned, n = L + 1) is recorded as soon
 * as every gradient of bucket b is final in the gradient buffer, in the order L-1, ...,
 * 0, then L. A stream that waits on events[b] may read (and all-reduce in place) bucket
 * b's ranges while the rest of the backward pass runs; it must not write other buckets
 * before their own events. n = 0 cancels. The events are recorded once, then
 * forgotten. Returns GPT2_ERR_CONFIG for n other than 0 or L + 1, or a null event. */
int gpt2_set_grad_events(gpt2* m, void* const* events, int n);

/* Per-kernel-category timing with CUDA events on the handle's stream.
 * gpt2_profile(m, 1) clears old records and starts recording an event pair around
 * every launch; gpt2_profile(m, 0) stops. gpt2_profile_read(m, cat, ...) waits for
 * the stream and returns, for category cat (0 .. count-1), its name, total device
 * milliseconds, launch count and the algorithmic FLOPs and bytes of those launches
 * (2*M*N*K per GEMM; causal attention 4*B*H*hd*T(T+1)/2 forward and 2.5 times
 * that backward; bytes a kernel must move for the memory-bound ones). Returns
 * GPT2_ERR_CONFIG past the last category. While recording, the gradient reductions
 * that normally overlap on a second stream run in order on the handle's stream, so
 * that each kernel's time is its own. */
int gpt2_profile(gpt2* m, int enable);
int gpt2_profile_read(gpt2* m, int cat, char* name, int name_len, double* ms, int64_t* launches, double* flops,
                      double* bytes);

/* Number of kernel launches the handle has issued since creation (for reports). */
int gpt2_launch_count(const gpt2* m, int64_t* out);

/* ------------------------------------------------------------------------
 * Generation with a key/value cache. "GPT From Scratch" (Architecture diagram)
 * samples with temperature and top-k; "Genesis" (Project Structure; What I built
 * from scratch) adds top-p, and lists a key/value cache under Roadmap; the cache is
 * the incremental form of causal attention: keys and values of earlier positions do
 * not change when a token is appended. bf16 models with head size
 * 64 only (others: GPT2_ERR_CONFIG); 1 <= B <= min(B_max, 16) sequences of equal
 * length. The cache ([L][B_max][T][2C] bf16, keys then values per row) is
 * allocated by the first prefill and lives with the handle. Generation calls reuse
 * the training activation memory: make them between optimizer steps, not between
 * the micro-batches of one accumulation. Asynchronous on the handle's stream
 * unless stated otherwise.
 *
 * gpt2_prefill: forward of B prompts of T0 tokens (tokens: host or device int32
 * [B][T0], 1 <= T0 <= T), keys and values of every layer into cache positions
 * 0..T0-1, and the fp32 logits of each prompt's last position into logits_out
 * (DEVICE, caller-owned, row b at logits_out + b*ld, ld >= V). Synchronises and
 * reports token-range errors.
 * gpt2_decode_step: feed one token per sequence (tokens: host or device int32 [B],
 * B equal to the prefill's) at the next position p = gpt2_kv_length; appends its
 * keys and values at p and writes the fp32 logits of position p to logits_out.
 * GPT2_ERR_SEQ_TOO_LONG once the cache holds T positions. A token id outside
 * [0, V) raises the device error word (reported by the next synchronising call).
 * gpt2_sample_topk: one index per row of fp32 logits [rows][ld] on the DEVICE:
 * order the V logits by value descending, ties by lower index; keep the first k
 * (1 <= k <= min(V, 1024)); weights w_j = exp((z_j - z_max)/temperature) in
 * float64 (temperature > 0); running sums c_j taken in that order; with top_p < 1
 * keep only the prefix up to the first j with c_j >= top_p * c_{k-1} (0 < top_p
 * <= 1); return the index at the first kept j with c_j > u[row] * c_last, else the
 * last kept one. u: DEVICE float64 [rows] in [0, 1), the caller's random draws.
 * idx_out: DEVICE int32 [rows]. Logits must not be NaN. */
int gpt2_prefill(gpt2* m, const int32_t* tokens, int B, int T0, float* logits_out, int64_t ld);
int gpt2_decode_step(gpt2* m, const int32_t* tokens, int B, float* logits_out, int64_t ld);
int gpt2_sample_topk(gpt2* m, const float* logits, int64_t ld, int rows, int k, float temperature, float top_p,
                     const double* u, int32_t* idx_out);
/* Wait for the handle's stream and report the device error word (e.g. a token id
 * outside [0, V) fed to gpt2_decode_step). */
int gpt2_synchronize(gpt2* m);
/* Positions held in the key/value cache (0 before the first prefill). */
int gpt2_kv_length(const gpt2* m, int* out);

const char* gpt2_last_error(const gpt2* m);
void gpt2_destroy(gpt2* m);

/* ------------------------------------------------------------------------
 * Op-level entry points: single kernels on caller-owned DEVICE buffers, for
 * per-kernel checks and measurement. `stream` is a cudaStream_t (NULL = the
 * legacy default stream). dtype selects the activation type: GPT2_BF16 for
 * bf16 (__nv_bfloat16) buffers, GPT2_FP32 for float. fp32 buffers named f32_*
 * are float in both modes. Calls are asynchronous unless stated otherwise;
 * those that need scratch memory allocate it with cudaMallocAsync on the stream
 * and free it the same way.
 * ------------------------------------------------------------------------ */

/* Epilogues of gpt2_op_gemm (D = accumulator, fp32):
 *  0 out(act) = D + bias                     qkv / logits
 *  1 out(act) = D + bias, out2(act) = gelu_tanh(D + bias)   fc + GELU
 *  2 out(f32) = aux(f32) + D + bias          residual add
 *  3 out(act) = D * gelu_tanh'(aux(act))     GELU backward
 *  4 out(f32) = D, or out += D when accumulate   dX / dW
 * D[M, N] = sum_k A(m, k) B(n, k), with A(m, k) = A[m*lda + k] (a_mn = 0) or
 * A[k*lda + m] (a_mn = 1), and B(n, k) likewise with b_mn. bias (nullable) is
 * f32 [N]. ksplit > 1 (bf16 only, epilogue 4 only) splits K into ksplit slices
 * reduced in a fixed order. bf16 needs lda, ldb, ldo multiples of 8 and 16-byte
 * aligned base pointers (tensor-memory-accelerator tiles). */
int gpt2_op_gemm(int dtype, const void* A, int64_t lda, int a_mn, const void* B, int64_t ldb, int b_mn, int M, int N,
                 int K, int epilogue, void* out, int64_t ldo, void* out2, int64_t ldo2, const float* bias,
                 const void* aux, int64_t ld_aux, int accumulate, int ksplit, void* stream);

/* Time the bf16 tensor-core GEMM of gpt2_op_gemm (same arguments) over `iters`
 * back-to-back launches after one warm-up launch, with CUDA events on `stream`;
 * *ms_out = average milliseconds per call (split-K reduction included).
 * ksplit 0 lets the library choose the split as inside the training step; bn is
 * the tile width (0 = the library's choice, or 128 / 256); pair selects 256-row
 * tiles computed by a cluster of two CTAs whose MMAs span both SMs (-1 = the
 * library's choice, 0 = one CTA per 128-row tile, 1 = pairs; needs tile width
 * 256). Returns GPT2_ERR_CONFIG for iters <= 0 or a NULL ms_out. Synchronises. */
int gpt2_op_gemm_bench(const void* A, int64_t lda, int a_mn, const void* B, int64_t ldb, int b_mn, int M, int N, int K,
                       int epilogue, void* out, int64_t ldo, void* out2, int64_t ldo2, const float* bias,
                       const void* aux, int64_t ld_aux, int accumulate, int ksplit, int bn, int pair, int iters,
                       float* ms_out, void* stream);

/* LayerNorm forward over rows of f32_x [N, C]: y(act) [N, C], f32 mean and rstd
 * [N]. eps 1e-5, biased variance. C % 4 == 0, C <= 2048, and x, g, b, y start on
 * 16-byte boundaries; otherwise GPT2_ERR_CONFIG. */
int gpt2_op_layernorm_fwd(int dtype, const float* f32_x, const float* f32_g, const float* f32_b, int N, int C, void* y,
                          float* f32_mean, float* f32_rstd, void* stream);

/* LayerNorm backward: f32_dres (+)= dx (accumulate = 1 adds), dres_act (nullable)
 * = copy of the new f32_dres in the activation type, f32_dg and f32_db (+)= the
 * parameter gradients (accumulate_params = 1 adds). C % 4 == 0, C <= 2048, and the
 * row arrays (dy, x, g, dres, dres_act) start on 16-byte boundaries; otherwise
 * GPT2_ERR_CONFIG. */
int gpt2_op_layernorm_bwd(int dtype, const float* f32_dy, const float* f32_x, const float* f32_g,
                          const float* f32_mean, const float* f32_rstd, int N, int C, float* f32_dres, void* dres_act,
                          int accumulate, float* f32_dg, float* f32_db, int accumulate_params, void* stream);

/* Causal attention forward: qkv(act) [B*T, 3*NH*hd] -> out(act) [B*T, NH*hd],
 * f32_lse [B, NH, T] (natural log). bf16 requires hd == 64; fp32 requires hd a
 * multiple of 32, at most 128. Synchronises the stream and reports a bounded wait
 * that gave up as GPT2_ERR_TIMEOUT. */
int gpt2_op_attention_fwd(int dtype, const void* qkv, int B, int T, int NH, int hd, void* out, float* f32_lse,
                          void* stream);

/* Causal attention backward: dqkv(act) [B*T, 3*NH*hd] from qkv, out, dout(act)
 * and f32_lse. Deterministic (no atomics). Synchronises the stream and reports a
 * bounded wait that gave up as GPT2_ERR_TIMEOUT. */
int gpt2_op_attention_bwd(int dtype, const void* qkv, const void* out, const void* dout, const float* f32_lse, int B,
                          int T, int NH, int hd, void* dqkv, void* stream);

/* The training step's form of the causal attention backward (bf16, hd == 64): the
 * dK/dV kernel also stores the bf16 dS^T tiles it feeds to its dK product into the
 * caller's workspace ds (DEVICE, gpt2_attention_ds_bytes(B, T, NH) bytes, 16-byte
 * aligned: B*NH*nqb*nqb tiles of 32 KB, nqb = T / 128 rounded up, tile (b*NH + h, key
 * block, query block) = two halves [128 keys][64 queries]; only the causal tiles are
 * written), and dQ = dS K is then computed from them instead of
 * recomputing the scores ("GPT From Scratch", Key decisions: the same gradients as the
 * plain masked-softmax attention). Same arguments and results as gpt2_op_attention_bwd
 * otherwise (deterministic, not bitwise equal to it: the dQ sums run in another order);
 * ds == NULL returns GPT2_ERR_CONFIG. Synchronises the stream and reports a bounded wait
 * that gave up as GPT2_ERR_TIMEOUT. */
int gpt2_op_attention_bwd_stored(const void* qkv, const void* out, const void* dout, const float* f32_lse, int B,
                                 int T, int NH, int hd, void* dqkv, void* ds, void* stream);

/* Bytes of the dS^T workspace gpt2_op_attention_bwd_stored needs (0 for an empty shape). */
size_t gpt2_attention_ds_bytes(int B, int T, int NH);

/* Embedding forward: f32_x0[b*T + t, :] = wte[tokens[b*T + t], :] + wpe[t, :]
 * (wte [V, C], wpe [>= T, C], f32). Ids outside [0, V) raise
 * GPT2_ERR_TOKEN_RANGE (this call synchronises to report it). */
int gpt2_op_embedding_fwd(const int32_t* tokens, const float* f32_wte, const float* f32_wpe, int B, int T, int C, int V,
                          float* f32_x0, void* stream);

/* Stable bucketing of token positions by id (the atomic-free embedding
 * backward's first stage). tokens [N] device, N <= 32768, ids in [0, V).
 * Outputs (device): sorted_pos [N] (positions ordered by (id, position)),
 * seg_id [N] and seg_start [N + 1] (distinct ids in increasing order and the
 * index in sorted_pos where each id's positions begin; seg_start[nseg] = N).
 * *nseg_out (host) = number of distinct ids. Synchronises. */
int gpt2_op_token_buckets(const int32_t* tokens, int N, int V, int32_t* sorted_pos, int32_t* seg_id,
                          int32_t* seg_start, int32_t* nseg_out, void* stream);

/* Embedding backward, atomic-free and deterministic: f32_dwte[v] += sum of
 * f32_dx0 rows at positions with tokens == v; f32_dwpe[t] += sum_b
 * f32_dx0[b*T + t]. B*T <= 32768. */
int gpt2_op_embedding_bwd(const int32_t* tokens, const float* f32_dx0, int B, int T, int C, int V, float* f32_dwte,
                          float* f32_dwpe, void* stream);

/* Cross-entropy over rows of logits(act) [N, ld] (first V columns; bf16 needs
 * ld % 8 == 0): f32_row_loss[n] = logsumexp - z[target]; logits overwritten by
 * (softmax - onehot) * scale (padding columns set to 0). bf16 runs the training
 * step's path: per-row softmax partials (here computed from the logits; in the step
 * the head GEMM's epilogue leaves them), then one streaming pass. Synchronises. */
int gpt2_op_cross_entropy(int dtype, void* logits, int64_t ld, int N, int V, const int32_t* targets, float scale,
                          float* f32_row_loss, void* stream);

/* Attention backward that allocates nothing (no counterpart on the pages: an
 * interface addition for callers whose device memory is wholly owned by their
 * own allocator or fixed budget, so they may not call cudaMalloc/cudaMallocAsync,
 * or who cannot pay for an allocation per call). Same arguments and results as
 * gpt2_op_attention_bwd. Its scratch (B*NH*T floats) is a fixed device array of
 * 2^20 floats (4 MiB) that every GPU loading the library holds until exit;
 * B*NH*T > 1,048,576 returns GPT2_ERR_CONFIG with a message. A second fixed word
 * holds the kernels' error flag: the call clears it, runs the kernels, reads it
 * back (so the call synchronises the stream) and reports a bounded wait that gave
 * up as GPT2_ERR_TIMEOUT. The first call on a device looks up both addresses and
 * caches them: make that first call before any stream capture. All calls on a
 * device share the array and the word (each overwrites what it uses before reading
 * it); calls whose kernels overlap on the GPU race. */
int gpt2_op_attention_bwd_noalloc(int dtype, const void* qkv, const void* out, const void* dout,
                                  const float* f32_lse, int B, int T, int NH, int hd, void* dqkv, void* stream);

/* Skinny product of a generation step, all DEVICE pointers: out[b][n] = epilogue(sum_k
 * x[b][k] W[n][k]) for b < B <= 16, n < N; W bf16 [N][K] row-major; epilogue 0 (bf16 out,
 * + bias), 1 (bf16 gelu_tanh(acc + bias)), 2 (fp32 out = resid + acc + bias) or 4 (fp32
 * out = acc). x is bf16 rows of stride ldx, or, when ln_g and ln_b are given, fp32 rows that
 * are layer-normalised first (eps 1e-5, result rounded to bf16). K a multiple of 32 with
 * 16 * (K + 8) * 2 bytes <= 200 KB (K <= 6392), ldx a multiple of 8, 16-byte aligned x, W,
 * ln_g, ln_b; GPT2_ERR_BATCH for B outside [1, 16], GPT2_ERR_CONFIG for the rest. Runs on
 * the tensor cores (m16n8k16 products, fp32 accumulation). With iters > 1 the product is then
 * launched iters more times back to back (as programmatic dependents when pdl != 0) and
 * *ms_out receives the mean milliseconds per launch. Synchronises. */
int gpt2_op_gemv(const void* x, int64_t ldx, int B, const void* W, int N, int K, int epilogue, const float* bias,
                 void* out, int64_t ldo, const float* resid, int64_t ldr, const float* ln_g, const float* ln_b,
                 int iters, int pdl, float* ms_out, void* stream);

/* gpt2_sample_topk without a handle, for V given explicitly (same rules and
 * arguments, all DEVICE pointers). Synchronises. */
int gpt2_op_sample_topk(const float* logits, int64_t ld, int rows, int V, int k, float temperature, float top_p,
                        const double* u, int32_t* idx_out, void* stream);

/* Check of the device-side timeout path (no counterpart on the pages: it tests the
 * library's error reporting). One thread initialises an mbarrier of count 1,
 * completes it when arrive != 0, then waits for it with the same bounded wait as every
 * kernel of the library, giving up after limit_ns nanoseconds (at most 1e9). Returns
 * GPT2_OK when the barrier completed and GPT2_ERR_TIMEOUT when the wait gave up (always
 * the case for arrive == 0). Nothing else is in flight during the wait. Synchronises. */
int gpt2_op_bounded_wait_check(int arrive, unsigned long long limit_ns, void* stream);

const char* gpt2_op_last_error(void);

#ifdef __cplusplus
}
#endif
#endif /* GPT2_B200_H */
