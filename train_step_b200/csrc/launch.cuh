// launch.cuh -- host-side launchers for the kernels (shape checks, grid sizing,
// tensor-map encoding). Every launcher returns 0 or a negative GPT2_ERR_* code
// and writes a message into `msg` on failure.
#pragma once
#include <cudaTypedefs.h>

#include <algorithm>
#include <cstdio>
#include <map>
#include <mutex>
#include <string>
#include <utility>
#include <vector>

#include "../../include/gpt2.h"
#include "adamw.cuh"
#include "attention.cuh"
#include "attention_tc.cuh"
#include "common.cuh"
#include "cross_entropy.cuh"
#include "decode.cuh"
#include "embedding.cuh"
#include "gemm_simt.cuh"
#include "gemm_tc.cuh"
#include "layernorm.cuh"
#include "sample.cuh"

namespace g2 {

// Kernel categories for the per-launch CUDA-event profiler.
enum ProfCat : int {
  CAT_GEMM = 0,   // forward linears (qkv, attention-out, fc, proj)
  CAT_GEMM_HEAD,  // lm_head logits, dxf, dW
  CAT_GEMM_DX,    // backward input gradients
  CAT_GEMM_DW,    // backward weight gradients
  CAT_SPLITK,
  CAT_ATTN_FWD,
  CAT_ATTN_BWD,
  CAT_LN_FWD,
  CAT_LN_BWD,
  CAT_REDUCE,
  CAT_EMB_FWD,
  CAT_EMB_BWD,
  CAT_CE,
  CAT_ADAMW,
  CAT_DEC_GEMV,
  CAT_DEC_ATTN,
  CAT_SAMPLE,
  CAT_COUNT
};
inline const char* prof_cat_name(int c) {
  static const char* n[CAT_COUNT] = {"gemm_tc_fwd",   "gemm_tc_head",  "gemm_tc_dx",    "gemm_tc_dw",
                                     "splitk_reduce", "attention_fwd", "attention_bwd", "layernorm_fwd",
                                     "layernorm_bwd", "reductions",    "embedding_fwd", "embedding_bwd",
                                     "cross_entropy", "adamw",         "decode_gemv",   "decode_attention",
                                     "sample_topk"};
  return (c >= 0 && c < CAT_COUNT) ? n[c] : "?";
}

// Records a start/stop event pair around each profiled launch; totals are read
// after a synchronisation. Off by default (no events are recorded).
struct Profiler {
  bool on = false;
  struct Rec {
    int cat;
    cudaEvent_t a, b;
    double flops, bytes;
  };
  std::vector<Rec> recs;
  std::vector<cudaEvent_t> pool;
  size_t used = 0;
  cudaEvent_t get() {
    if (used == pool.size()) {
      cudaEvent_t e;
      cudaEventCreate(&e);
      pool.push_back(e);
    }
    return pool[used++];
  }
  void begin(cudaStream_t s, int cat, double flops, double bytes) {
    Rec r{cat, get(), get(), flops, bytes};
    cudaEventRecord(r.a, s);
    recs.push_back(r);
  }
  void end(cudaStream_t s) { cudaEventRecord(recs.back().b, s); }
  void reset() {
    recs.clear();
    used = 0;
  }
  ~Profiler() {
    for (auto e : pool) cudaEventDestroy(e);
  }
};

// A second stream for work that nothing on the main stream needs before a later join:
// the reductions of gradient partials into parameter gradients, which then overlap the
// next GEMM (they fit beside a GEMM's CTA on each SM). A partial buffer is written again
// only after the reduction that reads it has finished (its `freed` event); the main
// stream joins the side stream at the end of a micro-batch's backward pass.
enum SideBuf : int { SIDE_LN = 0, SIDE_BIAS = 1, SIDE_WS0 = 2, SIDE_WS1 = 3, SIDE_EMB = 4, SIDE_NBUF = 5 };
struct SideStream {
  cudaStream_t s = nullptr;
  cudaEvent_t ready = nullptr;  // recorded on the main stream before side work is enqueued
  cudaEvent_t joined = nullptr;
  cudaEvent_t freed[SIDE_NBUF] = {};
  bool used[SIDE_NBUF] = {};
};

struct LaunchCtx {
  Profiler* prof = nullptr;
  cudaStream_t stream = nullptr;
  int* d_err = nullptr;           // device error word
  std::string* msg = nullptr;     // where failures are described
  long long* launches = nullptr;  // launch counter (nullable)
  float* splitk_ws = nullptr;     // split-K workspace (nullable: split-K disabled)
  size_t splitk_cap = 0;          // floats
  int num_sms = 148;
  bool pdl = false;  // launch as programmatic dependents of the previous kernel (kernels that support it)
  SideStream* side = nullptr;     // nullable: every reduction on `stream`
  int ws_buf = -1;                // the side buffer id of splitk_ws (-1: none)
  bool reduce_on_side = false;    // a split-K reduction goes to the side stream
};

// The main stream waits until the last reduction that read side buffer b has finished.
inline int side_wait_free(const LaunchCtx& c, int b) {
  if (!c.side || b < 0 || !c.side->used[b]) return GPT2_OK;
  if (cudaStreamWaitEvent(c.stream, c.side->freed[b], 0) != cudaSuccess) {
    if (c.msg) *c.msg = "cudaStreamWaitEvent failed";
    return GPT2_ERR_CUDA;
  }
  return GPT2_OK;
}
// A context that launches on the side stream, after everything enqueued on c.stream so far.
inline LaunchCtx side_ctx(const LaunchCtx& c) {
  LaunchCtx r = c;
  cudaEventRecord(c.side->ready, c.stream);
  cudaStreamWaitEvent(c.side->s, c.side->ready, 0);
  r.stream = c.side->s;
  r.side = nullptr;
  r.pdl = false;
  return r;
}
// After the side-stream launches that read side buffer b.
inline void side_mark_free(const LaunchCtx& c, int b) {
  cudaEventRecord(c.side->freed[b], c.side->s);
  c.side->used[b] = true;
}
// The main stream waits for all side-stream work enqueued so far.
inline int side_join(const LaunchCtx& c) {
  if (!c.side) return GPT2_OK;
  if (cudaEventRecord(c.side->joined, c.side->s) != cudaSuccess ||
      cudaStreamWaitEvent(c.stream, c.side->joined, 0) != cudaSuccess) {
    if (c.msg) *c.msg = "side stream join failed";
    return GPT2_ERR_CUDA;
  }
  return GPT2_OK;
}

// Launch `kern` on c.stream; with c.pdl as a programmatic dependent of the stream's
// previous kernel (the kernel must call pdl_wait before reading that kernel's results and
// before any write).
template <typename... KArgs, typename... Args>
inline cudaError_t launch_k(const LaunchCtx& c, void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem,
                            Args... args) {
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = c.stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = c.pdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kern, args...);
}

struct ProfScope {
  const LaunchCtx& c;
  bool on;
  ProfScope(const LaunchCtx& ctx, int cat, double flops, double bytes) : c(ctx), on(ctx.prof && ctx.prof->on) {
    if (on) c.prof->begin(c.stream, cat, flops, bytes);
  }
  ~ProfScope() {
    if (on) c.prof->end(c.stream);
  }
};

inline int fail(const LaunchCtx& c, int code, const std::string& m) {
  if (c.msg) *c.msg = m;
  return code;
}

inline int check_launch(const LaunchCtx& c, const char* what) {
  cudaError_t e = cudaGetLastError();
  if (c.launches) ++*c.launches;
  if (e != cudaSuccess) return fail(c, GPT2_ERR_CUDA, std::string(what) + ": " + cudaGetErrorString(e));
  return GPT2_OK;
}

// One-time set-up per (device, key), thread-safe. Function attributes such as the
// dynamic shared-memory opt-in (cudaFuncSetAttribute) apply only on the device that is
// current when they are set, so each device that launches a kernel needs its own. The
// value `setup` returns (>= 0) is kept and returned on later calls for that device and
// key; a negative value is returned without being kept, so the set-up is tried again.
struct DeviceOnce {
  std::mutex mu;
  std::map<std::pair<int, const void*>, int> val;
};
inline DeviceOnce& device_once_registry() {
  static DeviceOnce r;
  return r;
}
template <class F>
inline int per_device_once(const void* key, F&& setup) {
  int dev = 0;
  cudaGetDevice(&dev);
  DeviceOnce& r = device_once_registry();
  std::lock_guard<std::mutex> lk(r.mu);
  auto it = r.val.find({dev, key});
  if (it != r.val.end()) return it->second;
  const int v = setup();
  if (v >= 0) r.val[{dev, key}] = v;
  return v;
}
// The dynamic shared-memory opt-in of `kern` on the current device (once per device).
template <class K>
inline bool smem_optin(K kern, int bytes) {
  return per_device_once(reinterpret_cast<const void*>(kern), [&]() -> int {
           return cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) == cudaSuccess ? 0
                                                                                                                : -1;
         }) >= 0;
}

inline int device_sm_count() {
  int dev = 0, n = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  return n;
}

// ---------------------------------------------------------------------------
// TMA descriptors through the driver entry point (no link-time libcuda).
// ---------------------------------------------------------------------------
inline PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  return fn;
}

// 2-D bf16 tensor [outer][inner] with row stride ld elements; box {64, box_outer};
// 128-byte swizzle; out-of-bounds elements read as zero.
inline bool encode_bf16_map(CUtensorMap* map, const void* ptr, long long inner, long long outer, long long ld,
                            int box_outer) {
  auto enc = tensor_map_encoder();
  if (!enc) return false;
  cuuint64_t dims[2] = {(cuuint64_t)inner, (cuuint64_t)outer};
  cuuint64_t strides[1] = {(cuuint64_t)(ld * 2)};
  cuuint32_t box[2] = {64u, (cuuint32_t)box_outer};
  cuuint32_t estr[2] = {1u, 1u};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// Epilogue maps: rows x cols tensor (row stride ld elements), box of box_cols x 32
// rows, matching the epilogue's 2 KB chunk layout: 64-byte rows (16 fp32 or 32 bf16
// columns) with 64-byte swizzle.
inline bool encode_out_map(CUtensorMap* map, const void* ptr, long long cols, long long rows, long long ld,
                           bool is_f32, int box_cols) {
  auto enc = tensor_map_encoder();
  if (!enc) return false;
  const int es = is_f32 ? 4 : 2;
  cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)(ld * es)};
  cuuint32_t box[2] = {(cuuint32_t)box_cols, 32u};
  cuuint32_t estr[2] = {1u, 1u};
  const int row_bytes = box_cols * es;
  CUresult r = enc(map, is_f32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
                   const_cast<void*>(ptr), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                   row_bytes == 64 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_NONE,
                   CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// Split-K partial workspace [ksplit][rows][cols] fp32 as a 3-D map, box 16 x 32 x 1.
inline bool encode_partial_map(CUtensorMap* map, const void* ptr, long long cols, long long rows, int ksplit) {
  auto enc = tensor_map_encoder();
  if (!enc) return false;
  cuuint64_t dims[3] = {(cuuint64_t)cols, (cuuint64_t)rows, (cuuint64_t)ksplit};
  cuuint64_t strides[2] = {(cuuint64_t)(cols * 4), (cuuint64_t)(rows * cols * 4)};
  cuuint32_t box[3] = {16u, 32u, 1u};
  cuuint32_t estr[3] = {1u, 1u, 1u};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, const_cast<void*>(ptr), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B, CU_TENSOR_MAP_L2_PROMOTION_NONE,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// qkv [B][T][3C] bf16 as a 3-D map {3C, T, B}; box {64, rows, 1} (one head's 64
// columns of `rows` positions), 128-byte swizzle; positions past T read as zero.
inline bool encode_qkv_map(CUtensorMap* map, const void* ptr, long long cols, long long T, long long B,
                           unsigned rows = 128, unsigned box_cols = 64) {
  auto enc = tensor_map_encoder();
  if (!enc) return false;
  cuuint64_t dims[3] = {(cuuint64_t)cols, (cuuint64_t)T, (cuuint64_t)B};
  cuuint64_t strides[2] = {(cuuint64_t)(cols * 2), (cuuint64_t)(T * cols * 2)};
  cuuint32_t box[3] = {box_cols, rows, 1u};
  cuuint32_t estr[3] = {1u, 1u, 1u};
  // 64-column boxes: 128-byte rows, 128-byte swizzle; 16-column boxes: 32-byte rows, unswizzled
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(ptr), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, box_cols == 64 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
                   box_cols == 64 ? CU_TENSOR_MAP_L2_PROMOTION_L2_256B : CU_TENSOR_MAP_L2_PROMOTION_NONE,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// ---------------------------------------------------------------------------
// GEMM
// ---------------------------------------------------------------------------
struct GemmDesc {
  const void* A;
  long long lda;
  bool a_mn;
  const void* B;
  long long ldb;
  bool b_mn;
  int M, N, K;
  int epi;
  void* out;
  long long ldo;
  void* out2;
  long long ldo2;
  const float* bias;
  const void* aux;
  long long ld_aux;
  int accumulate;
  int ksplit;  // 0 = choose, 1 = none, > 1 = forced
  int role = CAT_GEMM;  // profiler category
  int bn = 0;           // tile width: 0 = choose (256 when N >= 256), else 128 or 256
  int pair = -1;        // 2-CTA tiles (256 x 256): -1 = choose, 0 = off, 1 = on (needs BN 256)
  float* colsum = nullptr;  // EPI_BF16_DGELU: per-32-row-block column sums [ceil(M/32)][N] (nullable)
  float2* rowstats = nullptr;  // EPI_BF16: softmax partials per row and half tile (nullable)
  int stats_ncols = 0;         // columns counted by rowstats
};

// Tile width of a tensor-core GEMM: 256 when N >= 256 unless forced.
inline int gemm_bn(const GemmDesc& d) { return d.bn == 128 || d.bn == 256 ? d.bn : (d.N >= 256 ? 256 : 128); }
// Softmax partials per row that a GEMM with rowstats writes.
inline int gemm_rowstats_count(const GemmDesc& d) {
  return (tc_epi_warps<EPI_BF16>() / 4) * ((d.N + gemm_bn(d) - 1) / gemm_bn(d));
}

struct TcMaps {
  CUtensorMap a, b, o, o2;
};

template <int BN, bool AM, bool BM_, int EPI, bool PAIR>
int launch_tc_inst(const LaunchCtx& c, const TcMaps& tm, const GemmParams& p) {
  auto kern = gemm_tc_kernel<BN, AM, BM_, EPI, PAIR>;
  using Cfg = TcCfg<BN, PAIR, tc_has_aux<EPI>(), tc_epi_warps<EPI>()>;
  constexpr int smem = Cfg::SMEM;
  constexpr int threads = Cfg::THREADS;
  // shared-memory opt-in and, for pairs, the co-resident clusters: once per device
  const int max_clusters = per_device_once(reinterpret_cast<const void*>(kern), [&]() -> int {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess) return -1;
    if (!PAIR) return 0;
    cudaLaunchConfig_t q{};
    q.gridDim = dim3(2 * (c.num_sms / 2));
    q.blockDim = dim3(threads);
    q.dynamicSmemBytes = smem;
    cudaLaunchAttribute qa[1];
    qa[0].id = cudaLaunchAttributeClusterDimension;
    qa[0].val.clusterDim.x = 2;
    qa[0].val.clusterDim.y = 1;
    qa[0].val.clusterDim.z = 1;
    q.attrs = qa;
    q.numAttrs = 1;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, kern, &q) != cudaSuccess || n < 1) return -2;
    return n;
  });
  if (max_clusters == -1) return fail(c, GPT2_ERR_CUDA, "cudaFuncSetAttribute(gemm_tc) failed");
  if (max_clusters < 0) return fail(c, GPT2_ERR_CUDA, "gemm_tc: no 2-CTA cluster fits");
  if (!PAIR) {
    const int grid = p.num_units < c.num_sms ? p.num_units : c.num_sms;
    if (launch_k(c, kern, dim3(grid), dim3(threads), smem, tm.a, tm.b, tm.o, tm.o2, p) != cudaSuccess)
      return fail(c, GPT2_ERR_CUDA, "gemm_tc: launch failed");
    return check_launch(c, "gemm_tc");
  }
  const int clusters = p.num_units < max_clusters ? p.num_units : max_clusters;
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(2 * clusters);
  cfg.blockDim = dim3(threads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = c.stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;  // see launch_k
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = c.pdl ? 2 : 1;
  if (cudaLaunchKernelEx(&cfg, kern, tm.a, tm.b, tm.o, tm.o2, p) != cudaSuccess)
    return fail(c, GPT2_ERR_CUDA, "gemm_tc: cluster launch failed");
  return check_launch(c, "gemm_tc_pair");
}

template <int BN, bool AM, bool BM_, bool PAIR>
int launch_tc_epi(const LaunchCtx& c, int epi, const TcMaps& tm, const GemmParams& p) {
  switch (epi) {
    case EPI_BF16: return launch_tc_inst<BN, AM, BM_, EPI_BF16, PAIR>(c, tm, p);
    case EPI_BF16_GELU: return launch_tc_inst<BN, AM, BM_, EPI_BF16_GELU, PAIR>(c, tm, p);
    case EPI_F32_RESID: return launch_tc_inst<BN, AM, BM_, EPI_F32_RESID, PAIR>(c, tm, p);
    case EPI_BF16_DGELU: return launch_tc_inst<BN, AM, BM_, EPI_BF16_DGELU, PAIR>(c, tm, p);
    case EPI_F32: return launch_tc_inst<BN, AM, BM_, EPI_F32, PAIR>(c, tm, p);
  }
  return fail(c, GPT2_ERR_CONFIG, "gemm: unknown epilogue");
}

inline int gemm_tc(const LaunchCtx& c, const GemmDesc& d) {
  if (d.M <= 0 || d.N <= 0 || d.K <= 0) return fail(c, GPT2_ERR_CONFIG, "gemm: empty shape");
  if (d.a_mn && !d.b_mn) return fail(c, GPT2_ERR_CONFIG, "gemm: MN-major A needs MN-major B");
  if ((d.lda % 8) || (d.ldb % 8) || (reinterpret_cast<uintptr_t>(d.A) & 15) || (reinterpret_cast<uintptr_t>(d.B) & 15))
    return fail(c, GPT2_ERR_CONFIG, "gemm: bf16 operands need 16-byte aligned rows");
  const int BN = gemm_bn(d);
  if (d.pair == 1 && BN != 256) return fail(c, GPT2_ERR_CONFIG, "gemm: 2-CTA tiles need tile width 256");
  // 2-CTA tiles halve each SM's B-operand traffic; measured on B200 they lose where a short
  // main loop (K < 1536) meets an epilogue that reads an auxiliary tile (residual / GELU
  // input), and where the output is too small to keep 74 pairs busy
  const bool aux_epi = d.epi == EPI_F32_RESID || d.epi == EPI_BF16_DGELU;
  const bool pair = BN == 256 && (d.pair == 1 || (d.pair < 0 && d.M >= 2 * TC_BM && (!aux_epi || d.K >= 1536) &&
                                                  (long long)d.M * d.N >= (1LL << 20)));
  const int unit_m = pair ? 2 * TC_BM : TC_BM;
  const int tiles_m = (d.M + unit_m - 1) / unit_m, tiles_n = (d.N + BN - 1) / BN;
  const int num_kb = (d.K + TC_BK - 1) / TC_BK;
  int ksplit = d.ksplit;
  if (d.epi != EPI_F32 || !c.splitk_ws) {
    if (ksplit > 1) return fail(c, GPT2_ERR_CONFIG, "gemm: split-K needs epilogue 4 and a workspace");
    ksplit = 1;
  } else if (ksplit == 0) {
    // Choose the split that minimises (waves of units) x (k-blocks per unit) plus the
    // split-K reduction's traffic. A k-block of a 128-row x BN tile costs about
    // 128 * BN * 64 * 2 / 8192 tensor cycles per SM (~0.14 us at BN 256 per 128 rows);
    // the reduction moves (ksplit + 1 + accumulate) M N fp32 words at ~5 TB/s. Wave
    // quantisation matters: 36 tiles split 5 ways are 180 units, 2.4 waves of 74 pairs
    // (3 waves), where a split of 2 or 4 fills 1 or 2 waves exactly.
    const long long tiles = (long long)tiles_m * tiles_n;
    const long long slots = pair ? c.num_sms / 2 : c.num_sms;  // units in flight at once
    const double kb_us = (double)(pair ? 2 * TC_BM : TC_BM) * BN * TC_BK * 2.0 / 8192.0 / (pair ? 2.0 : 1.0) / 1.8e3;
    double best = 1e30;
    ksplit = 1;
    const int kmax = std::min(16, std::max(1, num_kb / 4));
    for (int k = 1; k <= kmax; ++k) {
      const int per = (num_kb + k - 1) / k;
      const int kk = (num_kb + per - 1) / per;  // no empty slices
      const long long waves = (tiles * kk + slots - 1) / slots;
      double t = (double)waves * per * kb_us;
      if (kk > 1) {
        if ((size_t)kk * d.M * d.N > c.splitk_cap) continue;
        t += (double)(kk + 1 + d.accumulate) * d.M * d.N * 4.0 / 5.0e6;  // us at 5 TB/s
      }
      if (t < best * 0.999) {
        best = t;
        ksplit = kk;
      }
    }
  }
  int kb_per = (num_kb + ksplit - 1) / ksplit;
  ksplit = (num_kb + kb_per - 1) / kb_per;  // no empty slices
  if (ksplit > 1 && (size_t)ksplit * d.M * d.N > c.splitk_cap) {
    ksplit = 1;
    kb_per = num_kb;
  }
  if (ksplit > 1 && (d.N % 4)) return fail(c, GPT2_ERR_CONFIG, "gemm: split-K needs N % 4 == 0");
  GemmParams p{};
  p.M = d.M;
  p.N = d.N;
  p.K = d.K;
  p.tiles_m = tiles_m;
  p.tiles_n = tiles_n;
  p.ksplit = ksplit;
  p.kb_per_split = kb_per;
  p.num_kb = num_kb;
  p.num_units = tiles_m * tiles_n * ksplit;
  p.out = d.out;
  p.ldo = d.ldo;
  p.out2 = d.out2;
  p.ldo2 = d.ldo2;
  p.bias = d.bias;
  p.aux = d.aux;
  p.ld_aux = d.ld_aux;
  p.accumulate = d.accumulate;
  p.partial = ksplit > 1 ? c.splitk_ws : nullptr;
  p.colsum = d.epi == EPI_BF16_DGELU ? d.colsum : nullptr;
  p.rowstats = d.epi == EPI_BF16 ? d.rowstats : nullptr;
  p.stats_ncols = d.stats_ncols;
  p.err = c.d_err;
  p.timeout_ns = 4000000000ull;
  const bool out_f32 = (d.epi == EPI_F32 || d.epi == EPI_F32_RESID);
  const int oes = out_f32 ? 4 : 2;
  if ((reinterpret_cast<uintptr_t>(d.out) & 15) || (d.ldo * oes) % 16 ||
      (d.epi == EPI_BF16_GELU && ((reinterpret_cast<uintptr_t>(d.out2) & 15) || (d.ldo2 * 2) % 16)))
    return fail(c, GPT2_ERR_CONFIG, "gemm: outputs need 16-byte aligned rows");
  TcMaps tm;
  bool ok = d.a_mn ? encode_bf16_map(&tm.a, d.A, d.M, d.K, d.lda, 64)
                   : encode_bf16_map(&tm.a, d.A, d.K, d.M, d.lda, 128);
  ok = ok && (d.b_mn ? encode_bf16_map(&tm.b, d.B, d.N, d.K, d.ldb, 64)
                     : encode_bf16_map(&tm.b, d.B, d.K, d.N, d.ldb, pair ? BN / 2 : BN));
  const int cw = (d.epi == EPI_F32 || d.epi == EPI_F32_RESID) ? 16 : 32;  // epilogue chunk columns
  ok = ok && encode_out_map(&tm.o, d.out, d.N, d.M, d.ldo, out_f32, cw);
  if (ksplit > 1) {
    ok = ok && encode_partial_map(&tm.o2, c.splitk_ws, d.N, d.M, ksplit);
  } else if (d.epi == EPI_BF16_GELU) {
    ok = ok && encode_out_map(&tm.o2, d.out2, d.N, d.M, d.ldo2, false, 32);
  } else if (d.epi == EPI_F32_RESID || d.epi == EPI_BF16_DGELU) {  // the auxiliary input, read by TMA
    if ((reinterpret_cast<uintptr_t>(d.aux) & 15) || (d.ld_aux * (d.epi == EPI_F32_RESID ? 4 : 2)) % 16)
      return fail(c, GPT2_ERR_CONFIG, "gemm: the auxiliary input needs 16-byte aligned rows");
    ok = ok && encode_out_map(&tm.o2, d.aux, d.N, d.M, d.ld_aux, d.epi == EPI_F32_RESID, cw);
  } else {
    tm.o2 = tm.o;
  }
  if (!ok) return fail(c, GPT2_ERR_CUDA, "gemm: cuTensorMapEncodeTiled failed");
  if (ksplit > 1) {  // the workspace's previous reduction has read it
    const int rw = side_wait_free(c, c.ws_buf);
    if (rw) return rw;
  }
  int r;
  {
  ProfScope ps(c, d.role, 2.0 * d.M * d.N * d.K, 0.0);
  if (pair) {
    if (!d.a_mn && !d.b_mn) r = launch_tc_epi<256, false, false, true>(c, d.epi, tm, p);
    else if (!d.a_mn) r = launch_tc_epi<256, false, true, true>(c, d.epi, tm, p);
    else r = launch_tc_epi<256, true, true, true>(c, d.epi, tm, p);
  } else if (BN == 256) {
    if (!d.a_mn && !d.b_mn) r = launch_tc_epi<256, false, false, false>(c, d.epi, tm, p);
    else if (!d.a_mn) r = launch_tc_epi<256, false, true, false>(c, d.epi, tm, p);
    else r = launch_tc_epi<256, true, true, false>(c, d.epi, tm, p);
  } else {
    if (!d.a_mn && !d.b_mn) r = launch_tc_epi<128, false, false, false>(c, d.epi, tm, p);
    else if (!d.a_mn) r = launch_tc_epi<128, false, true, false>(c, d.epi, tm, p);
    else r = launch_tc_epi<128, true, true, false>(c, d.epi, tm, p);
  }
  }
  if (r || ksplit == 1) return r;
  const bool on_side = c.side && c.reduce_on_side && c.ws_buf >= 0;
  const LaunchCtx rc = on_side ? side_ctx(c) : c;
  {
    ProfScope ps(rc, CAT_SPLITK, 0.0, 4.0 * d.M * d.N * (ksplit + 1 + d.accumulate));
    const long long n4 = (long long)d.M * (d.N / 4);
    long long blocks = (n4 + 255) / 256;
    if (blocks > 8LL * c.num_sms) blocks = 8LL * c.num_sms;
    splitk_reduce_kernel<<<(int)blocks, 256, 0, rc.stream>>>(c.splitk_ws, ksplit, d.M, d.N, (float*)d.out, d.ldo,
                                                              d.accumulate);
  }
  r = check_launch(rc, "splitk_reduce");
  if (on_side) side_mark_free(c, c.ws_buf);
  else if (c.side && c.ws_buf >= 0) c.side->used[c.ws_buf] = false;  // read on the main stream already
  return r;
}

inline int gemm_simt(const LaunchCtx& c, const GemmDesc& d) {
  if (d.M <= 0 || d.N <= 0 || d.K <= 0) return fail(c, GPT2_ERR_CONFIG, "gemm: empty shape");
  SimtGemmArgs a{};
  a.A = (const float*)d.A;
  a.lda = d.lda;
  a.a_mn = d.a_mn;
  a.B = (const float*)d.B;
  a.ldb = d.ldb;
  a.b_mn = d.b_mn;
  a.M = d.M;
  a.N = d.N;
  a.K = d.K;
  a.ep.out = d.out;
  a.ep.ldo = d.ldo;
  a.ep.out2 = d.out2;
  a.ep.ldo2 = d.ldo2;
  a.ep.bias = d.bias;
  a.ep.aux = d.aux;
  a.ep.ld_aux = d.ld_aux;
  a.ep.accumulate = d.accumulate;
  dim3 grid((d.N + 63) / 64, (d.M + 63) / 64);
  ProfScope ps(c, d.role, 2.0 * d.M * d.N * d.K, 0.0);
  switch (d.epi) {
    case EPI_BF16: gemm_simt_kernel<EPI_BF16><<<grid, 256, 0, c.stream>>>(a); break;
    case EPI_BF16_GELU: gemm_simt_kernel<EPI_BF16_GELU><<<grid, 256, 0, c.stream>>>(a); break;
    case EPI_F32_RESID: gemm_simt_kernel<EPI_F32_RESID><<<grid, 256, 0, c.stream>>>(a); break;
    case EPI_BF16_DGELU: gemm_simt_kernel<EPI_BF16_DGELU><<<grid, 256, 0, c.stream>>>(a); break;
    case EPI_F32: gemm_simt_kernel<EPI_F32><<<grid, 256, 0, c.stream>>>(a); break;
    default: return fail(c, GPT2_ERR_CONFIG, "gemm: unknown epilogue");
  }
  return check_launch(c, "gemm_simt");
}

inline int gemm(const LaunchCtx& c, int dtype, const GemmDesc& d) {
  return dtype == GPT2_BF16 ? gemm_tc(c, d) : gemm_simt(c, d);
}

// ---------------------------------------------------------------------------
// LayerNorm
// ---------------------------------------------------------------------------
inline int ln_nv(int C) { return (C + 127) / 128; }

template <class T>
int layernorm_fwd_t(const LaunchCtx& c, const float* x, const float* g, const float* b, int N, int C, T* y, float* mean,
                    float* rstd) {
  const int blocks = (N + LN_WARPS - 1) / LN_WARPS;
  const int nv = ln_nv(C);
  ProfScope ps(c, CAT_LN_FWD, 0.0, (double)N * C * (4 + sizeof(T)) + 8.0 * N);
  cudaError_t e = cudaSuccess;
#define LNF(NV)                                                                                           \
  e = c.pdl ? launch_k(c, layernorm_fwd_kernel<T, NV, true>, dim3(blocks), dim3(LN_WARPS * 32), 0, x, g, b, y, \
                       mean, rstd, N, C)                                                                  \
            : (layernorm_fwd_kernel<T, NV><<<blocks, LN_WARPS * 32, 0, c.stream>>>(x, g, b, y, mean, rstd, N, C), \
               cudaSuccess)
  if (nv <= 1) LNF(1);
  else if (nv <= 2) LNF(2);
  else if (nv <= 4) LNF(4);
  else if (nv <= 6) LNF(6);
  else if (nv <= 8) LNF(8);
  else if (nv <= 13) LNF(13);
  else LNF(16);
#undef LNF
  if (e != cudaSuccess) return fail(c, GPT2_ERR_CUDA, std::string("layernorm_fwd: ") + cudaGetErrorString(e));
  return check_launch(c, "layernorm_fwd");
}

// LayerNorm backward grid: the CTAs resident at once (so that none waits for a second
// wave). A CTA holds LN_WARPS x 3 x C fp32 column accumulators in shared memory and the
// kernel is built for three CTAs per SM of registers: 3 per SM at C = 768, 2 at 1024,
// 1 at 1600.
inline int ln_bwd_grid(int N, int C, int num_sms) {
  const long long per_cta = (long long)LN_WARPS * 3 * C * 4 + 1024;
  long long resident = 233472 / per_cta;
  if (resident > 8) resident = 8;
  if (resident < 1) resident = 1;
  const long long cap = resident * num_sms;
  const long long g = (N + LN_WARPS - 1) / LN_WARPS;
  return (int)(g < cap ? g : cap);
}

// out_v (+)= column sums of partial set v, for the non-null outputs out[0..nv).
inline int reduce_partials(const LaunchCtx& c, const float* part, int P, int ncols, int nv, float* out0, float* out1,
                           float* out2, int accumulate) {
  ProfScope ps(c, CAT_REDUCE, 0.0, 4.0 * nv * P * ncols + 8.0 * nv * ncols);
  ReduceOuts o{{out0, out1, out2}};
  reduce_partials_kernel<<<dim3((ncols + 7) / 8, nv), 256, 0, c.stream>>>(part, P, ncols, o, accumulate);
  return check_launch(c, "reduce_partials");
}

template <class T, int NV, class DY>
void launch_ln_bwd(const LaunchCtx& c, int grid, size_t smem, const DY* dy, const float* x, const float* g,
                   const float* mean, const float* rstd, float* dres, T* dres_act, int accumulate, float* part,
                   int with_rsum, int N, int C) {
  smem_optin(layernorm_bwd_kernel<T, NV, DY>, 200 * 1024);
  layernorm_bwd_kernel<T, NV, DY><<<grid, LN_WARPS * 32, smem, c.stream>>>(dy, x, g, mean, rstd, dres, dres_act,
                                                                           accumulate, part, with_rsum, N, C);
}

// Slots per warp of the staged backward: as many rows (dy, x, dres: 12 C bytes each) as
// fit in the shared memory of one CTA, at most 3; 0 when fewer than 2 fit (the staged
// kernel needs a row in flight while it computes one, so wide rows use the other kernel).
inline int ln_ring_stages(int C) {
  const long long slot = 12LL * C + 8;
  long long st = (232448 - 1024) / ((long long)LNR_WARPS * slot);
  if (st > 3) st = 3;
  return st >= 2 ? (int)st : 0;
}
inline size_t ln_ring_smem(int C, int stages) { return (size_t)LNR_WARPS * stages * (12 * (size_t)C + 8); }

template <class T, int NV, class DY>
int launch_ln_bwd_ring(const LaunchCtx& c, int grid, int stages, const DY* dy, const float* x, const float* g,
                       const float* mean, const float* rstd, float* dres, T* dres_act, int accumulate, float* part,
                       int with_rsum, int N, int C) {
  const size_t smem = ln_ring_smem(C, stages);
  // opted in once per device for the largest ring any C can ask for
  if (!smem_optin(layernorm_bwd_ring_kernel<T, NV, DY>, 232448 - 1024))
    return fail(c, GPT2_ERR_CUDA, "layernorm_bwd: shared-memory opt-in");
  const cudaError_t e = launch_k(c, layernorm_bwd_ring_kernel<T, NV, DY>, dim3(grid), dim3(LNR_WARPS * 32), smem, dy, x,
                                 g, mean, rstd, dres, dres_act, accumulate, part, with_rsum, N, C, stages, c.d_err,
                                 4000000000ull);
  if (e != cudaSuccess) return fail(c, GPT2_ERR_CUDA, std::string("layernorm_bwd: ") + cudaGetErrorString(e));
  return 0;
}

// LayerNorm backward plus the reduction of its parameter gradients: dg, db (+)=;
// dbias_next (nullable) (+)= column sums of the updated dres.
// dy: fp32, or bf16 (the dX GEMMs' output in bf16 mode)
template <class T, class DY = float>
int layernorm_bwd_t(const LaunchCtx& c, const DY* dy, const float* x, const float* g, const float* mean,
                    const float* rstd, int N, int C, float* dres, T* dres_act, int accumulate,
                    float* part /*3*grid*C*/, float* dg, float* db, float* dbias_next, int accumulate_params,
                    int side_buf = -1) {
  const int stages = ln_ring_stages(C);
  const int nv = ln_nv(C);
  // staged kernel: one CTA per SM (fewer if there are fewer row groups)
  const int grid = stages && nv <= 8 ? (int)std::min<long long>(c.num_sms, ((long long)N + LNR_WARPS - 1) / LNR_WARPS)
                                     : ln_bwd_grid(N, C, c.num_sms);
  const int with_rsum = dbias_next != nullptr;
  {
    const int rw = side_wait_free(c, side_buf);  // the partials' previous reduction has read them
    if (rw) return rw;
  }
  {
    ProfScope ps(c, CAT_LN_BWD, 0.0,
                 (double)N * C * (sizeof(DY) + 8 + 4 * accumulate + (dres_act ? sizeof(T) : 0)) + 8.0 * N +
                     4.0 * (2 + with_rsum) * grid * C);
    const size_t smem = (size_t)LN_WARPS * 3 * C * 4;
    int rr = 0;
    if (stages && nv <= 4) rr = launch_ln_bwd_ring<T, 4, DY>(c, grid, stages, dy, x, g, mean, rstd, dres, dres_act, accumulate, part, with_rsum, N, C);
    else if (stages && nv <= 6) rr = launch_ln_bwd_ring<T, 6, DY>(c, grid, stages, dy, x, g, mean, rstd, dres, dres_act, accumulate, part, with_rsum, N, C);
    else if (stages && nv <= 8) rr = launch_ln_bwd_ring<T, 8, DY>(c, grid, stages, dy, x, g, mean, rstd, dres, dres_act, accumulate, part, with_rsum, N, C);
    else if (nv <= 1) launch_ln_bwd<T, 1, DY>(c, grid, smem, dy, x, g, mean, rstd, dres, dres_act, accumulate, part, with_rsum, N, C);
    else if (nv <= 2) launch_ln_bwd<T, 2, DY>(c, grid, smem, dy, x, g, mean, rstd, dres, dres_act, accumulate, part, with_rsum, N, C);
    else if (nv <= 4) launch_ln_bwd<T, 4, DY>(c, grid, smem, dy, x, g, mean, rstd, dres, dres_act, accumulate, part, with_rsum, N, C);
    else if (nv <= 6) launch_ln_bwd<T, 6, DY>(c, grid, smem, dy, x, g, mean, rstd, dres, dres_act, accumulate, part, with_rsum, N, C);
    else if (nv <= 8) launch_ln_bwd<T, 8, DY>(c, grid, smem, dy, x, g, mean, rstd, dres, dres_act, accumulate, part, with_rsum, N, C);
    else if (nv <= 13) launch_ln_bwd<T, 13, DY>(c, grid, smem, dy, x, g, mean, rstd, dres, dres_act, accumulate, part, with_rsum, N, C);
    else launch_ln_bwd<T, 16, DY>(c, grid, smem, dy, x, g, mean, rstd, dres, dres_act, accumulate, part, with_rsum, N, C);
    if (rr) return rr;
  }
  int r = check_launch(c, "layernorm_bwd");
  if (r) return r;
  if (c.side && side_buf >= 0) {  // the parameter-gradient reduction overlaps what follows
    r = reduce_partials(side_ctx(c), part, grid, C, 2 + with_rsum, dg, db, dbias_next, accumulate_params);
    side_mark_free(c, side_buf);
    return r;
  }
  return reduce_partials(c, part, grid, C, 2 + with_rsum, dg, db, dbias_next, accumulate_params);
}

// column sums of y [N, ncols] (ncols % 8 == 0) into out (+=), through a partial
// buffer of R x ncols floats
inline void colsum_shape(int N, int ncols, int& gx, int& R, int& rows_per) {
  gx = (ncols + 2047) / 2048;  // 256 threads x 8 columns
  R = 1184 / gx;
  if (R < 1) R = 1;
  if (R > N) R = N;
  rows_per = (N + R - 1) / R;
  R = (N + rows_per - 1) / rows_per;
}

template <class T>
int colsum_t(const LaunchCtx& c, const T* y, long long ld, int N, int ncols, float* part, float* out) {
  if (ncols % 8) return fail(c, GPT2_ERR_CONFIG, "colsum: ncols % 8 != 0");
  int gx, R, rows_per;
  colsum_shape(N, ncols, gx, R, rows_per);
  {
    ProfScope ps(c, CAT_REDUCE, 0.0, (double)N * ncols * sizeof(T) + 4.0 * R * ncols);
    colsum_partial_kernel<T><<<dim3(gx, R), 256, 0, c.stream>>>(y, ld, N, ncols, rows_per, part);
  }
  int r = check_launch(c, "colsum_partial");
  if (r) return r;
  return reduce_partials(c, part, R, ncols, 1, out, nullptr, nullptr, 1);
}

// ---------------------------------------------------------------------------
// attention
// ---------------------------------------------------------------------------
inline int attention_fwd(const LaunchCtx& c, int dtype, const void* qkv, int B, int T, int NH, int hd, void* out,
                         float* lse) {
  const float scale = 1.0f / sqrtf((float)hd);
  ProfScope ps(c, CAT_ATTN_FWD, 4.0 * B * NH * hd * (0.5 * T * (T + 1.0)), 0.0);
  if (dtype == GPT2_BF16) {
    if (hd != 64) return fail(c, GPT2_ERR_CONFIG, "attention (bf16): head dim must be 64");
    if ((reinterpret_cast<uintptr_t>(qkv) & 15) || (reinterpret_cast<uintptr_t>(out) & 15))
      return fail(c, GPT2_ERR_CONFIG, "attention: qkv and out must be 16-byte aligned");
    CUtensorMap tqkv, tout;  // 128-row tiles of Q, K and V; 128-row output tiles
    if (!encode_qkv_map(&tqkv, qkv, 3LL * NH * 64, T, B) || !encode_qkv_map(&tout, out, (long long)NH * 64, T, B))
      return fail(c, GPT2_ERR_CUDA, "attention: tensor map");
    if (!smem_optin(attn_fwd_tc_kernel, FX_SMEM)) return fail(c, GPT2_ERR_CUDA, "attention: shared-memory opt-in");
    // persistent: one CTA per SM loops over (pair of query tiles, batch*head) items
    const long long items = (long long)((T + 255) / 256) * B * NH;
    const int grid = items < c.num_sms ? (int)items : c.num_sms;
    const cudaError_t e = launch_k(c, attn_fwd_tc_kernel, dim3(grid), dim3(FX_THREADS), FX_SMEM, tqkv, tout, lse, T,
                                   NH, B * NH, scale, c.d_err, 4000000000ull);
    if (e != cudaSuccess) return fail(c, GPT2_ERR_CUDA, std::string("attn_fwd_tc: ") + cudaGetErrorString(e));
    return check_launch(c, "attn_fwd_tc");
  }
  if (hd % 32 || hd > 128) return fail(c, GPT2_ERR_CONFIG, "attention (fp32): head dim must be 32, 64, 96 or 128");
  const long long warps = (long long)B * NH * T;
  attn_fwd_f32_kernel<<<(int)((warps * 32 + 255) / 256), 256, 0, c.stream>>>((const float*)qkv, (float*)out, lse, B,
                                                                             T, NH, hd, scale);
  return check_launch(c, "attn_fwd_f32");
}

// colsum (nullable, bf16 only): the kernels also leave the column sums of dqkv per 32-row
// block, [B * ceil(T / 128) * 4][3 * NH * hd] (the qkv bias gradient after a reduction).
inline int attn_colsum_blocks(int B, int T) { return B * ((T + FA_BM - 1) / FA_BM) * 4; }
// dS^T workspace of the stored-dS backward: B*NH*nqb*nqb contiguous 32 KB tiles (nqb = T / 128
// rounded up), tile (bh, key block, query block) = two halves of [128 keys][64 queries] bf16
inline size_t attn_ds_bytes(int B, int T, int NH) {
  const size_t nqb = (size_t)((T + FA_BM - 1) / FA_BM);
  return (size_t)B * NH * nqb * nqb * 2 * FA_BN * 64 * 2;
}
// ds (nullable, bf16 only, attn_ds_bytes(B, T, NH) bytes, 16-byte aligned): when given, the
// dK/dV kernel stores its dS^T tiles there and dQ is computed from them
// (attn_bwd_dq_stored_kernel); otherwise the dQ kernel recomputes S, dP and dS.
inline int attention_bwd(const LaunchCtx& c, int dtype, const void* qkv, const void* out, const void* dout,
                         const float* lse, int B, int T, int NH, int hd, void* dqkv, float* Dbuf,
                         float* colsum = nullptr, void* ds = nullptr) {
  const float scale = 1.0f / sqrtf((float)hd);
  ProfScope ps(c, CAT_ATTN_BWD, 2.5 * 4.0 * B * NH * hd * (0.5 * T * (T + 1.0)), 0.0);
  const long long warps = (long long)B * NH * T;
  const int dblocks = (int)((warps * 32 + 255) / 256);
  if (dtype == GPT2_BF16) {
    if (hd != 64) return fail(c, GPT2_ERR_CONFIG, "attention (bf16): head dim must be 64");
    if ((reinterpret_cast<uintptr_t>(qkv) & 15) || (reinterpret_cast<uintptr_t>(dout) & 15) ||
        (reinterpret_cast<uintptr_t>(out) & 15))
      return fail(c, GPT2_ERR_CONFIG, "attention: qkv, out and dout must be 16-byte aligned");
    const cudaError_t e = launch_k(c, attn_bwd_dot64_bf16_kernel, dim3((unsigned)((warps * 8 + 255) / 256)), dim3(256), 0,
                                   (const bf16*)out, (const bf16*)dout, Dbuf, B, T, NH);
    if (e != cudaSuccess) return fail(c, GPT2_ERR_CUDA, std::string("attn_bwd_dot: ") + cudaGetErrorString(e));
    int r = check_launch(c, "attn_bwd_dot");
    if (r) return r;
    CUtensorMap tq, td, tout;  // 128-row tiles of qkv, dout and dqkv
    if (!encode_qkv_map(&tq, qkv, 3LL * NH * 64, T, B) || !encode_qkv_map(&td, dout, (long long)NH * 64, T, B) ||
        !encode_qkv_map(&tout, dqkv, 3LL * NH * 64, T, B))
      return fail(c, GPT2_ERR_CUDA, "attention: tensor map");
    if (reinterpret_cast<uintptr_t>(dqkv) & 15) return fail(c, GPT2_ERR_CONFIG, "attention: dqkv must be 16-byte aligned");
    if (reinterpret_cast<uintptr_t>(ds) & 15) return fail(c, GPT2_ERR_CONFIG, "attention: dS workspace must be 16-byte aligned");
    // dS^T tiles as rows of 64 bf16: 128-key boxes for the dK/dV kernel's stores, 64-key
    // boxes for the loads
    const long long nqb = (T + FA_BM - 1) / FA_BM, ds_rows = (long long)B * NH * nqb * nqb * 2 * FA_BN;
    if (ds && ds_rows >= (1LL << 31)) return fail(c, GPT2_ERR_CONFIG, "attention: dS workspace too large");
    CUtensorMap tds_st = tq, tds_ld = tq;  // placeholders when dS is not stored (never read)
    if (ds && (!encode_out_map(&tds_st, ds, 64, ds_rows, 64, false, 32) || !encode_bf16_map(&tds_ld, ds, 64, ds_rows, 64, 64)))
      return fail(c, GPT2_ERR_CUDA, "attention: tensor map");
    CUtensorMap tout16;  // dqkv in boxes of 16 columns x 32 rows: the dK/dV kernel's per-warp stores
    if (!encode_qkv_map(&tout16, dqkv, 3LL * NH * 64, T, B, 32, 16)) return fail(c, GPT2_ERR_CUDA, "attention: tensor map");
    if (!smem_optin(attn_bwd_dkdv_tc_kernel<true>, BK_SMEM) || !smem_optin(attn_bwd_dkdv_tc_kernel<false>, BK_SMEM) ||
        !smem_optin(attn_bwd_dq_tc_kernel, BQ_SMEM) || !smem_optin(attn_bwd_dq_stored_kernel, DQS_SMEM))
      return fail(c, GPT2_ERR_CUDA, "attention: shared-memory opt-in");
    // persistent: one CTA per SM loops over (block, batch*head) items
    const long long items = (long long)((T + FA_BM - 1) / FA_BM) * B * NH;
    const int grid = items < c.num_sms ? (int)items : c.num_sms;
    cudaError_t e2 = launch_k(c, ds ? attn_bwd_dkdv_tc_kernel<true> : attn_bwd_dkdv_tc_kernel<false>, dim3(grid),
                              dim3(BK_THREADS), BK_SMEM, tq, td, ds ? tout16 : tout, tds_st, lse, (const float*)Dbuf,
                              colsum, T, NH, B * NH, scale, c.d_err, 4000000000ull);
    if (e2 != cudaSuccess) return fail(c, GPT2_ERR_CUDA, std::string("attn_bwd_dkdv_tc: ") + cudaGetErrorString(e2));
    r = check_launch(c, "attn_bwd_dkdv_tc");
    if (r) return r;
    if (ds) {
      e2 = launch_k(c, attn_bwd_dq_stored_kernel, dim3(grid), dim3(DQS_THREADS), DQS_SMEM, tq, tds_ld, tout, colsum, T,
                    NH, B * NH, scale, c.d_err, 4000000000ull);
      if (e2 != cudaSuccess) return fail(c, GPT2_ERR_CUDA, std::string("attn_bwd_dq_stored: ") + cudaGetErrorString(e2));
      return check_launch(c, "attn_bwd_dq_stored");
    }
    e2 = launch_k(c, attn_bwd_dq_tc_kernel, dim3(grid), dim3(BQ_THREADS), BQ_SMEM, tq, td, tout, lse, (const float*)Dbuf,
                  colsum, T, NH, B * NH, scale, c.d_err, 4000000000ull);
    if (e2 != cudaSuccess) return fail(c, GPT2_ERR_CUDA, std::string("attn_bwd_dq_tc: ") + cudaGetErrorString(e2));
    return check_launch(c, "attn_bwd_dq_tc");
  }
  if (hd % 32 || hd > 128) return fail(c, GPT2_ERR_CONFIG, "attention (fp32): head dim must be 32, 64, 96 or 128");
  attn_bwd_dot_kernel<float><<<dblocks, 256, 0, c.stream>>>((const float*)out, (const float*)dout, Dbuf, B, T, NH, hd);
  int r = check_launch(c, "attn_bwd_dot");
  if (r) return r;
  attn_bwd_dq_f32_kernel<<<dblocks, 256, 0, c.stream>>>((const float*)qkv, (const float*)dout, lse, Dbuf,
                                                        (float*)dqkv, B, T, NH, hd, scale);
  r = check_launch(c, "attn_bwd_dq_f32");
  if (r) return r;
  attn_bwd_dkdv_f32_kernel<<<dblocks, 256, 0, c.stream>>>((const float*)qkv, (const float*)dout, lse, Dbuf,
                                                          (float*)dqkv, B, T, NH, hd, scale);
  return check_launch(c, "attn_bwd_dkdv_f32");
}

// ---------------------------------------------------------------------------
// embedding
// ---------------------------------------------------------------------------
inline int embedding_fwd(const LaunchCtx& c, const int* tok, const float* wte, const float* wpe, int N, int T, int C,
                         int V, float* x0) {
  if (C % 4) return fail(c, GPT2_ERR_CONFIG, "embedding: C % 4 != 0");
  ProfScope ps(c, CAT_EMB_FWD, 0.0, 12.0 * N * C + 4.0 * N);
  embed_fwd_kernel<<<(int)(((long long)N * 32 + 255) / 256), 256, 0, c.stream>>>(tok, wte, wpe, x0, N, T, C, V, c.d_err);
  return check_launch(c, "embed_fwd");
}

// Scratch for the embedding backward, all device memory.
struct EmbScratch {
  int* sorted_pos;   // [N]
  int* chunk_start;  // [N + 1]
  int* seg_id;       // [N]
  int* seg_chunk0;   // [N + 1]
  int* counts;       // [2]
  float* partial;    // [N * C]
};
inline size_t emb_scratch_bytes(int N, int C) {
  return (size_t)N * 4 * 4 + 2 * 4 + 64 + (size_t)N * C * 4 + 6 * 256;
}
inline EmbScratch emb_scratch_carve(void* base, int N, int C) {
  auto al = [](uintptr_t x) { return (x + 255) & ~uintptr_t(255); };
  uintptr_t p = al(reinterpret_cast<uintptr_t>(base));
  EmbScratch s;
  s.partial = reinterpret_cast<float*>(p);
  p = al(p + (size_t)N * C * 4);
  s.sorted_pos = reinterpret_cast<int*>(p);
  p = al(p + (size_t)N * 4);
  s.chunk_start = reinterpret_cast<int*>(p);
  p = al(p + (size_t)(N + 1) * 4);
  s.seg_id = reinterpret_cast<int*>(p);
  p = al(p + (size_t)N * 4);
  s.seg_chunk0 = reinterpret_cast<int*>(p);
  p = al(p + (size_t)(N + 1) * 4);
  s.counts = reinterpret_cast<int*>(p);
  return s;
}

inline int token_sort(const LaunchCtx& c, const int* tok, int N, int V, const EmbScratch& s) {
  if (N > EMB_MAX_TOKENS) return fail(c, GPT2_ERR_BATCH, "embedding backward: B*T must be <= 32768");
  if (V > (1 << 17)) return fail(c, GPT2_ERR_CONFIG, "embedding backward: V must be <= 131072");
  int NP = 1;
  while (NP < N) NP <<= 1;
  smem_optin(token_sort_kernel, EMB_MAX_TOKENS * 4);
  token_sort_kernel<<<1, EMB_SORT_THREADS, NP * 4, c.stream>>>(tok, N, V, NP, s.sorted_pos, s.chunk_start, s.seg_id,
                                                              s.seg_chunk0, s.counts, c.d_err);
  return check_launch(c, "token_sort");
}

// sorted: the scratch already holds this batch's token sort (run earlier, e.g. on a side
// stream that the caller has waited for)
inline int embedding_bwd(const LaunchCtx& c, const int* tok, const float* dx0, int Bsz, int T, int C, int V,
                         float* dwte, float* dwpe, const EmbScratch& s, bool sorted = false) {
  const int N = Bsz * T;
  if (C % 4) return fail(c, GPT2_ERR_CONFIG, "embedding: C % 4 != 0");
  ProfScope ps(c, CAT_EMB_BWD, 0.0, 8.0 * N * C + 8.0 * T * C + 4.0 * N);
  int r = sorted ? GPT2_OK : token_sort(c, tok, N, V, s);
  if (r) return r;
  const int grid = 8 * c.num_sms;
  // a float4 of the row per thread: 192 threads cover C = 768 in one pass
  const int threads = std::min(256, std::max(32, (C / 4 + 31) / 32 * 32));
  embed_chunk_sum_kernel<<<grid, threads, 0, c.stream>>>(dx0, s.sorted_pos, s.chunk_start, s.counts, C, s.partial);
  if ((r = check_launch(c, "embed_chunk_sum"))) return r;
  embed_seg_sum_kernel<<<grid, threads, 0, c.stream>>>(s.partial, s.seg_id, s.seg_chunk0, s.counts, C, dwte);
  if ((r = check_launch(c, "embed_seg_sum"))) return r;
  const long long n4 = (long long)T * C / 4;
  embed_pos_grad_kernel<<<(int)((n4 + 255) / 256), 256, 0, c.stream>>>(dx0, Bsz, T, C, dwpe);
  return check_launch(c, "embed_pos_grad");
}

// ---------------------------------------------------------------------------
// cross-entropy
// ---------------------------------------------------------------------------
// fp32 parity path (one CTA per row, exact expf / logf); bf16 goes through
// cross_entropy_stats below.
inline int cross_entropy(const LaunchCtx& c, int dtype, void* logits, long long ld, int N, int V, const int* tgt,
                         float scale, float* row_loss) {
  if (N <= 0) return GPT2_OK;
  if (dtype != GPT2_FP32) return fail(c, GPT2_ERR_CONFIG, "cross_entropy: the bf16 path needs softmax partials");
  ProfScope ps(c, CAT_CE, 0.0, 2.0 * N * ld * 4);
  cross_entropy_f32_kernel<<<N, CE_THREADS, 0, c.stream>>>((float*)logits, ld, V, tgt, scale, row_loss, c.d_err);
  return check_launch(c, "cross_entropy");
}

// bf16 cross-entropy from softmax partials (nstats per row). With stats == nullptr the
// partials are computed first from the logits themselves (one per row) into `scratch`
// (rows float2).
inline int cross_entropy_stats(const LaunchCtx& c, bf16* logits, long long ld, int N, int V, const int* tgt,
                               float scale, float* row_loss, const float2* stats, int nstats, float2* scratch) {
  if (N <= 0) return GPT2_OK;
  if (ld % 8) return fail(c, GPT2_ERR_CONFIG, "cross_entropy: ld must be a multiple of 8");
  if (!stats) {
    if (!scratch) return fail(c, GPT2_ERR_CONFIG, "cross_entropy: no softmax partials");
    {
      ProfScope ps(c, CAT_CE, 0.0, 2.0 * N * V + 8.0 * N);
      ce_row_stats_kernel<<<(N + 7) / 8, 256, 0, c.stream>>>(logits, ld, V, N, scratch);
    }
    int r = check_launch(c, "ce_row_stats");
    if (r) return r;
    stats = scratch;
    nstats = 1;
  }
  ProfScope ps(c, CAT_CE, 0.0, 2.0 * N * ld * 2 + 8.0 * N * nstats);
  cross_entropy_stats_kernel<<<(N + CE_SROWS - 1) / CE_SROWS, CE_STHREADS, 0, c.stream>>>(
      logits, ld, V, N, tgt, scale, stats, nstats, row_loss, c.d_err);
  return check_launch(c, "cross_entropy_stats");
}

// ---------------------------------------------------------------------------
// generation: skinny GEMMs, single-query attention, key/value cache, sampling
// ---------------------------------------------------------------------------
constexpr int DEC_GEMV_MAX_SMEM = 200 * 1024;  // staged x: 16 * (K + 8) bf16

template <int KW, bool LN>
void gemv_attrs() {
  cudaFuncSetAttribute(gemv_bf16_kernel<EPI_BF16, KW, LN>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                       DEC_GEMV_MAX_SMEM);
  cudaFuncSetAttribute(gemv_bf16_kernel<EPI_BF16_GELU, KW, LN>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                       DEC_GEMV_MAX_SMEM);
  cudaFuncSetAttribute(gemv_bf16_kernel<EPI_F32_RESID, KW, LN>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                       DEC_GEMV_MAX_SMEM);
  cudaFuncSetAttribute(gemv_bf16_kernel<EPI_F32, KW, LN>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                       DEC_GEMV_MAX_SMEM);
}

// Shared-memory limits of every GEMV variant, set once per device before any launch
// (and so before a decode step is captured).
inline void gemv_prepare() {
  per_device_once(reinterpret_cast<const void*>(&gemv_prepare), []() -> int {
    gemv_attrs<1, false>();
    gemv_attrs<2, false>();
    gemv_attrs<4, false>();
    gemv_attrs<8, false>();
    gemv_attrs<1, true>();
    gemv_attrs<2, true>();
    gemv_attrs<4, true>();
    gemv_attrs<8, true>();
    return 0;
  });
}

template <int KW, bool LN>
int gemv_inst(const LaunchCtx& c, int epi, int grid, size_t smem, const void* x, int64_t ldx, int B, const bf16* W,
              int N, int K, const float* bias, void* out, int64_t ldo, const float* resid, int64_t ldr,
              const float* ln_g, const float* ln_b) {
  cudaError_t e = cudaSuccess;
  const dim3 g(grid), blk(DEC_WARPS * 32);
  switch (epi) {
    case EPI_BF16:
      e = launch_k(c, gemv_bf16_kernel<EPI_BF16, KW, LN>, g, blk, smem, x, ldx, B, W, N, K, bias, out, ldo, resid,
                   ldr, ln_g, ln_b);
      break;
    case EPI_BF16_GELU:
      e = launch_k(c, gemv_bf16_kernel<EPI_BF16_GELU, KW, LN>, g, blk, smem, x, ldx, B, W, N, K, bias, out, ldo,
                   resid, ldr, ln_g, ln_b);
      break;
    case EPI_F32_RESID:
      e = launch_k(c, gemv_bf16_kernel<EPI_F32_RESID, KW, LN>, g, blk, smem, x, ldx, B, W, N, K, bias, out, ldo,
                   resid, ldr, ln_g, ln_b);
      break;
    case EPI_F32:
      e = launch_k(c, gemv_bf16_kernel<EPI_F32, KW, LN>, g, blk, smem, x, ldx, B, W, N, K, bias, out, ldo, resid,
                   ldr, ln_g, ln_b);
      break;
    default: return fail(c, GPT2_ERR_CONFIG, "gemv: epilogue must be 0, 1, 2 or 4");
  }
  if (e != cudaSuccess) return fail(c, GPT2_ERR_CUDA, std::string("gemv_bf16: ") + cudaGetErrorString(e));
  return check_launch(c, "gemv_bf16");
}

// out[b][n] = epilogue(x[b] . W[n]) for B <= 16 rows (see gemv_bf16_kernel). With ln_g and
// ln_b set, x is the fp32 residual stream and is layer-normalised on the fly (ldx in
// floats); otherwise x is bf16.
inline int gemv_bf16(const LaunchCtx& c, int epi, const void* x, int64_t ldx, int B, const bf16* W, int N, int K,
                     const float* bias, void* out, int64_t ldo, const float* resid, int64_t ldr,
                     const float* ln_g = nullptr, const float* ln_b = nullptr) {
  const bool ln = ln_g != nullptr;
  if (B < 1 || B > DEC_MAX_B) return fail(c, GPT2_ERR_BATCH, "gemv: 1 <= B <= 16 rows");
  if (N <= 0 || K <= 0 || (K % 32) || (ldx % 8) || (reinterpret_cast<uintptr_t>(x) & 15) ||
      (reinterpret_cast<uintptr_t>(W) & 15) || (ln && (!ln_b || (reinterpret_cast<uintptr_t>(ln_g) & 15) ||
                                                      (reinterpret_cast<uintptr_t>(ln_b) & 15))))
    return fail(c, GPT2_ERR_CONFIG, "gemv: K % 32 == 0, ldx % 8 == 0, 16-byte aligned x, W and LayerNorm vectors");
  if (epi == EPI_F32_RESID && !resid) return fail(c, GPT2_ERR_CONFIG, "gemv: residual epilogue needs resid");
  const size_t smem = (size_t)DEC_MAX_B * (K + 8) * sizeof(bf16);
  if (smem > (size_t)DEC_GEMV_MAX_SMEM) return fail(c, GPT2_ERR_CONFIG, "gemv: K too large for the staged rows");
  gemv_prepare();
  // 8-column tiles; split K over up to 8 warps until there are about 8 warps per SM
  const int tiles = (N + 7) / 8;
  int kw = 1;
  while (kw < DEC_WARPS && (long long)tiles * kw < 8LL * c.num_sms && K / 32 >= 2 * kw) kw *= 2;
  const int nw = DEC_WARPS / kw;
  const int grid = (tiles + nw - 1) / nw;
  const bool f32o = epi == EPI_F32_RESID || epi == EPI_F32;
  ProfScope ps(c, CAT_DEC_GEMV, 2.0 * B * N * K,
               2.0 * N * K + (ln ? 4.0 : 2.0) * B * K + (double)B * N * (f32o ? 4 : 2) +
                   (epi == EPI_F32_RESID ? 4.0 * B * N : 0.0));
#define GEMV_KW(KWV)                                                                                          \
  return ln ? gemv_inst<KWV, true>(c, epi, grid, smem, x, ldx, B, W, N, K, bias, out, ldo, resid, ldr, ln_g, ln_b) \
            : gemv_inst<KWV, false>(c, epi, grid, smem, x, ldx, B, W, N, K, bias, out, ldo, resid, ldr, ln_g, ln_b)
  switch (kw) {
    case 1: GEMV_KW(1);
    case 2: GEMV_KW(2);
    case 4: GEMV_KW(4);
    default: GEMV_KW(8);
  }
#undef GEMV_KW
}

// Key splits per (sequence, head) for a generation step: none once every SM has a
// (sequence, head); else enough splits for two blocks per SM.
inline int decode_splits(int B, int NH, int num_sms) {
  const int bh = B * NH;
  if (bh >= num_sms) return 1;
  int S = (2 * num_sms + bh - 1) / bh;
  return S < 1 ? 1 : (S > DEC_MAX_SPLIT ? DEC_MAX_SPLIT : S);
}

// Single-query attention of one generation step (head size 64) at the position held in
// device memory (*pos_ptr < Tc); part: B*NH*S*DEC_PART floats when S > 1.
inline int decode_attention(const LaunchCtx& c, const bf16* qkv, bf16* cache, int64_t cache_seq, int Tc, int B, int C,
                            int NH, const int* pos_ptr, int S, bf16* att, float* part, double mean_keys) {
  if (B < 1 || NH < 1 || C != NH * DEC_HD) return fail(c, GPT2_ERR_CONFIG, "decode attention: head size must be 64");
  if (S < 1 || S > DEC_MAX_SPLIT || (S > 1 && !part)) return fail(c, GPT2_ERR_CONFIG, "decode attention: splits");
  const size_t smem = (size_t)Tc * 4;
  if (smem > 200 * 1024) return fail(c, GPT2_ERR_SEQ_TOO_LONG, "decode attention: more than 51200 positions");
  if (smem > 48 * 1024) smem_optin(decode_attn_kernel, 200 * 1024);
  ProfScope ps(c, CAT_DEC_ATTN, 4.0 * B * C * mean_keys, 4.0 * B * C * mean_keys + 10.0 * B * C);
  const float scale_log2 = 1.4426950408889634f / sqrtf((float)DEC_HD);
  cudaError_t e = launch_k(c, decode_attn_kernel, dim3(B * NH * S), dim3(DEC_ATT_THREADS), smem, qkv, cache,
                           cache_seq, C, NH, pos_ptr, S, scale_log2, att, part);
  if (e != cudaSuccess) return fail(c, GPT2_ERR_CUDA, std::string("decode_attention: ") + cudaGetErrorString(e));
  int r = check_launch(c, "decode_attention");
  if (r || S == 1) return r;
  e = launch_k(c, decode_attn_combine_kernel, dim3(B * NH), dim3(DEC_HD), 0, (const float*)part, S, C, NH, att);
  if (e != cudaSuccess) return fail(c, GPT2_ERR_CUDA, std::string("decode_combine: ") + cudaGetErrorString(e));
  return check_launch(c, "decode_attention_combine");
}

// Keys and values of a prompt's forward pass (qkv rows b*T0 + t) into cache rows t.
inline int kv_fill(const LaunchCtx& c, const bf16* qkv, int B, int T0, int C, bf16* cache, int64_t cache_seq) {
  if (C % 4) return fail(c, GPT2_ERR_CONFIG, "kv_fill: C % 4 != 0");
  const long long vec = (long long)B * T0 * (2 * C / 8);
  const int grid = (int)std::min<long long>((vec + 255) / 256, 8LL * c.num_sms);
  ProfScope ps(c, CAT_DEC_ATTN, 0.0, 8.0 * B * T0 * C);
  kv_fill_kernel<<<grid, 256, 0, c.stream>>>(qkv, B, T0, C, cache, cache_seq);
  return check_launch(c, "kv_fill");
}

// One sampled index per logits row (see sample_topk_kernel); u: [rows] doubles in [0, 1).
inline int sample_topk(const LaunchCtx& c, const float* logits, int64_t ld, int rows, int V, int k, float temperature,
                       float top_p, const double* u, int* out) {
  if (rows < 1 || V < 1 || ld < V || k < 1 || k > V || k > TOPK_MAX_K || !(temperature > 0.f) || !(top_p > 0.f) ||
      top_p > 1.f)
    return fail(c, GPT2_ERR_CONFIG, "sample_topk: 1 <= k <= min(V, 1024), temperature > 0, 0 < top_p <= 1");
  ProfScope ps(c, CAT_SAMPLE, 0.0, 5.0 * 4 * rows * V);
  sample_topk_kernel<<<rows, TOPK_THREADS, 0, c.stream>>>(logits, ld, V, k, temperature, top_p, u, out);
  return check_launch(c, "sample_topk");
}

}  // namespace g2
