// cross_entropy.cuh -- softmax cross-entropy over one chunk of logit rows, in
// place: logits in, d(loss)/d(logits) out ("gpt/docs/LLM.md", Output Layer:
// linear projection to the vocabulary; next-token loss on the shifted targets).
//
// For each row n: lse = logsumexp over the first V columns (padding columns V..ld
// are storage only); row_loss[n] = lse - z[target]; then
//   z[v] <- (exp(z[v] - lse) - [v == target]) * scale  for v < V,  0 for v >= V.
// HBM sees each logit once in and once out.
#pragma once
#include "common.cuh"

namespace g2 {

constexpr int CE_THREADS = 512;
constexpr float LOG2E_CE = 1.4426950408889634f;
constexpr float LN2_CE = 0.6931471805599453f;

__device__ __forceinline__ float block_reduce_ce(float v, bool is_max, float* buf) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  v = is_max ? warp_max(v) : warp_sum(v);
  __syncthreads();
  if (lane == 0) buf[warp] = v;
  __syncthreads();
  float r = buf[0];
  for (int w = 1; w < CE_THREADS / 32; ++w) r = is_max ? fmaxf(r, buf[w]) : r + buf[w];
  return r;
}

__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// bf16: persistent, one CTA per SM, rows r = blockIdx.x + k * gridDim.x. Two
// shared-memory row buffers: row k+1 arrives by a 1-D bulk copy while row k is
// processed. Each thread keeps a running (max, sum of exp) over its share of the
// row (one pass), the block combines them, and a second pass writes the gradient
// row to global memory with coalesced 16-byte stores, so the buffer is free for
// the next-but-one row as soon as the pass ends. HBM sees each logit once in and
// once out. ld * 2 bytes per buffer (ld % 8 == 0).
constexpr int CE_PERSIST_THREADS = 512;
__global__ void __launch_bounds__(CE_PERSIST_THREADS, 1) cross_entropy_bf16_kernel(
    bf16* __restrict__ logits, long long ld, int V, int rows, const int* __restrict__ tgt, float scale,
    float* __restrict__ row_loss, int* err, unsigned long long timeout_ns) {
  extern __shared__ __align__(128) uint8_t ce_smem[];
  __shared__ float red_m[CE_PERSIST_THREADS / 32], red_s[CE_PERSIST_THREADS / 32];
  __shared__ __align__(8) uint64_t bar[2];
  __shared__ int s_abort;
  const uint32_t row_bytes = (uint32_t)(ld * 2);
  bf16* buf[2] = {reinterpret_cast<bf16*>(ce_smem), reinterpret_cast<bf16*>(ce_smem + row_bytes)};
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int nvec = (int)(ld / 8);
  if (tid == 0) {
    mbar_init(&bar[0], 1);
    mbar_init(&bar[1], 1);
    s_abort = 0;
    fence_barrier_init();
  }
  __syncthreads();
  int row = blockIdx.x;
  if (tid == 0 && row < rows) {
    mbar_arrive_expect_tx(&bar[0], row_bytes);
    bulk_load_1d(buf[0], logits + (long long)row * ld, row_bytes, &bar[0]);
  }
  for (int k = 0; row < rows; ++k, row += gridDim.x) {
    const int cur = k & 1;
    const int nxt_row = row + gridDim.x;
    // buf[cur ^ 1] was last read in the previous iteration, which every thread has
    // finished (the __syncthreads at its end)
    if (tid == 0 && nxt_row < rows) {
      fence_proxy_async_smem();  // order the generic reads of that buffer before the async write
      mbar_arrive_expect_tx(&bar[cur ^ 1], row_bytes);
      bulk_load_1d(buf[cur ^ 1], logits + (long long)nxt_row * ld, row_bytes, &bar[cur ^ 1]);
    }
    if (tid == 0) {
      int never = 0;
      if (!mbar_wait_bounded(&bar[cur], (k >> 1) & 1, reinterpret_cast<volatile int*>(&never), timeout_ns)) {
        raise_device_error(err, DEV_TIMEOUT);
        s_abort = 1;
      }
    }
    __syncthreads();
    if (s_abort) break;
    mbar_try_wait(&bar[cur], (k >> 1) & 1);  // every thread observes the completed phase
    const bf16* z = buf[cur];
    int t = tgt[row];
    if (t < 0 || t >= V) {
      if (tid == 0) raise_device_error(err, DEV_TOKEN_RANGE);
      t = 0;
    }
    // Three passes over the row in shared memory, one exponential per logit:
    //   1. the row maximum M (log2 units);
    //   2. p = 2^(x*log2e - M) and its sum S; p (<= 1) replaces the logit in place as bf16;
    //   3. dlogits = (p / S - onehot(t)) * scale. The target column is recomputed in fp32,
    //      since p / S - 1 cancels there.
    const float xt = __bfloat162float(z[t]) * LOG2E_CE;  // read before pass 2 overwrites it
    bf16* zw = buf[cur];
    float m = -INFINITY;
    for (int vi = tid; vi < nvec; vi += CE_PERSIST_THREADS) {
      const uint4 u = reinterpret_cast<const uint4*>(z)[vi];
      const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const float2 f = unpack_bf16x2(w[q]);
        if (vi * 8 + 2 * q < V) m = fmaxf(m, f.x);
        if (vi * 8 + 2 * q + 1 < V) m = fmaxf(m, f.y);
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    if (lane == 0) red_m[warp] = m;
    __syncthreads();
    float M = red_m[0];
#pragma unroll
    for (int w = 1; w < CE_PERSIST_THREADS / 32; ++w) M = fmaxf(M, red_m[w]);
    M *= LOG2E_CE;
    float sacc = 0.f;
    for (int vi = tid; vi < nvec; vi += CE_PERSIST_THREADS) {
      const uint4 u = reinterpret_cast<const uint4*>(z)[vi];
      const uint32_t w[4] = {u.x, u.y, u.z, u.w};
      uint32_t o[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const float2 f = unpack_bf16x2(w[q]);
        const int c = vi * 8 + 2 * q;
        const float a = c < V ? ex2_approx(fmaf(f.x, LOG2E_CE, -M)) : 0.f;
        const float b = c + 1 < V ? ex2_approx(fmaf(f.y, LOG2E_CE, -M)) : 0.f;
        sacc += a + b;
        o[q] = pack_bf16x2(a, b);
      }
      reinterpret_cast<uint4*>(zw)[vi] = make_uint4(o[0], o[1], o[2], o[3]);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) sacc += __shfl_xor_sync(0xffffffffu, sacc, o);
    if (lane == 0) red_s[warp] = sacc;
    __syncthreads();
    float S = 0.f;
#pragma unroll
    for (int w = 0; w < CE_PERSIST_THREADS / 32; ++w) S += red_s[w];
    const float ll2 = M + __log2f(S);  // lse in the log2 domain
    if (tid == 0) row_loss[row] = (ll2 - xt) * LN2_CE;
    const float ps = scale / S;
    const float dt_val = (ex2_approx(xt - M) / S - 1.f) * scale;
    bf16* dst = logits + (long long)row * ld;
    for (int vi = tid; vi < nvec; vi += CE_PERSIST_THREADS) {
      const uint4 u = reinterpret_cast<const uint4*>(zw)[vi];
      const uint32_t w[4] = {u.x, u.y, u.z, u.w};
      uint32_t o[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const float2 f = unpack_bf16x2(w[q]);  // p, zero on padding columns
        const int c = vi * 8 + 2 * q;
        const float a = c == t ? dt_val : f.x * ps;
        const float b = c + 1 == t ? dt_val : f.y * ps;
        o[q] = pack_bf16x2(a, b);
      }
      reinterpret_cast<uint4*>(dst)[vi] = make_uint4(o[0], o[1], o[2], o[3]);
    }
    __syncthreads();  // everyone is done with buf[cur] and red_* before they are reused
  }
}

// fp32 parity mode: exact expf/logf, one CTA per row, strided (rows are short).
__global__ void __launch_bounds__(CE_THREADS) cross_entropy_f32_kernel(float* __restrict__ logits, long long ld, int V,
                                                                       const int* __restrict__ tgt, float scale,
                                                                       float* __restrict__ row_loss, int* err) {
  __shared__ float buf[CE_THREADS / 32];
  const long long row = blockIdx.x;
  float* z = logits + row * ld;
  int t = tgt[row];
  if (t < 0 || t >= V) {
    if (threadIdx.x == 0) raise_device_error(err, DEV_TOKEN_RANGE);
    t = 0;
  }
  const float zt = z[t];
  float mx = -INFINITY;
  for (int c = threadIdx.x; c < V; c += CE_THREADS) mx = fmaxf(mx, z[c]);
  mx = block_reduce_ce(mx, true, buf);
  float se = 0.f;
  for (int c = threadIdx.x; c < V; c += CE_THREADS) se += expf(z[c] - mx);
  se = block_reduce_ce(se, false, buf);
  const float lse = mx + logf(se);
  if (threadIdx.x == 0) row_loss[row] = lse - zt;
  __syncthreads();  // every thread has read z before any overwrite
  for (long long c = threadIdx.x; c < ld; c += CE_THREADS)
    z[c] = c < V ? (expf(z[c] - lse) - (c == t ? 1.f : 0.f)) * scale : 0.f;
}

// loss_acc[0] (+)= scale * sum_n row_loss[n], summed in a fixed tree order by one CTA.
__global__ void __launch_bounds__(1024) sum_rows_kernel(const float* __restrict__ row_loss, int N, float scale,
                                                        float* __restrict__ out, int accumulate) {
  __shared__ double buf[1024];
  double s = 0.0;
  for (int i = threadIdx.x; i < N; i += 1024) s += (double)row_loss[i];
  buf[threadIdx.x] = s;
  __syncthreads();
  for (int w = 512; w > 0; w >>= 1) {
    if (threadIdx.x < w) buf[threadIdx.x] += buf[threadIdx.x + w];
    __syncthreads();
  }
  if (threadIdx.x == 0) out[0] = (accumulate ? out[0] : 0.f) + (float)(buf[0] * (double)scale);
}

}  // namespace g2
