// cross_entropy.cuh -- softmax cross-entropy over one chunk of logit rows, in
// place: logits in, d(loss)/d(logits) out ("gpt/docs/LLM.md", Output Layer:
// linear projection to the vocabulary; next-token loss on the shifted targets).
//
// For each row n: lse = logsumexp over the first V columns (padding columns V..ld
// are storage only); row_loss[n] = lse - z[target]; then
//   z[v] <- (exp(z[v] - lse) - [v == target]) * scale  for v < V,  0 for v >= V.
// HBM sees each logit once in and once out: in bf16 the row statistics come from the
// producer of the logits (softmax partials), so one streaming pass remains.
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

// bf16, from per-row softmax partials. The producer of the logits leaves, per row, pairs
// (m_i, s_i) over disjoint column ranges with s_i = sum of exp(z - m_i) over the range's
// columns < V (the head GEMM's epilogue, or ce_row_stats_kernel). Then
//   lse = M + ln(sum_i s_i exp(m_i - M)), M = max_i m_i;  row_loss = lse - z[target];
//   z[v] <- (exp(z[v] - lse) - [v == target]) * scale for v < V, 0 for V <= v < ld,
// one pass over the row: each logit is read once and written once, with 16-byte
// accesses, and nothing waits for a row to be staged.
constexpr int CE_SROWS = 4;       // rows per CTA
constexpr int CE_STHREADS = 512;
__global__ void __launch_bounds__(CE_STHREADS) cross_entropy_stats_kernel(
    bf16* __restrict__ logits, long long ld, int V, int rows, const int* __restrict__ tgt, float scale,
    const float2* __restrict__ stats, int nstats, float* __restrict__ row_loss, int* err) {
  __shared__ float s_lse2[CE_SROWS];
  __shared__ int s_tgt[CE_SROWS];
  pdl_launch_dependents();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long r0 = (long long)blockIdx.x * CE_SROWS;
  if (warp < CE_SROWS && r0 + warp < rows) {
    const long long row = r0 + warp;
    const float2* st = stats + row * nstats;
    float m = -INFINITY;
    for (int i = lane; i < nstats; i += 32) m = fmaxf(m, st[i].x);
    m = warp_max(m);
    const float m2 = m * LOG2E_CE;
    float ssum = 0.f;
    for (int i = lane; i < nstats; i += 32) {
      const float2 x = st[i];
      if (x.x != -INFINITY) ssum += x.y * ex2_approx(fmaf(x.x, LOG2E_CE, -m2));
    }
    ssum = warp_sum(ssum);
    int t = tgt[row];
    if (t < 0 || t >= V) {
      if (lane == 0) raise_device_error(err, DEV_TOKEN_RANGE);
      t = 0;
    }
    const float lse2 = m2 + __log2f(ssum);  // log2 units
    if (lane == 0) {
      const float zt = __bfloat162float(logits[row * ld + t]);  // read before the row is overwritten
      row_loss[row] = (lse2 - zt * LOG2E_CE) * LN2_CE;
      s_lse2[warp] = lse2;
      s_tgt[warp] = t;
    }
  }
  __syncthreads();
  const int nvec = (int)(ld / 8);
  const int nrows = (int)min((long long)CE_SROWS, (long long)rows - r0);
  for (int rr = 0; rr < nrows; ++rr) {
    const float lse2 = s_lse2[rr];
    const int t = s_tgt[rr];
    uint4* rowv = reinterpret_cast<uint4*>(logits + (r0 + rr) * ld);
    // dlogits of the 8 columns of vector vi
    auto grad8 = [&](const uint4 u, int vi) -> uint4 {
      const uint32_t w[4] = {u.x, u.y, u.z, u.w};
      uint32_t o[4];
      const int c0 = vi * 8;
      if (c0 + 8 <= V && (unsigned)(t - c0) >= 8u) {
        // the common vector: all 8 columns inside the vocabulary, none of them the target
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const float2 f = unpack_bf16x2(w[q]);
          o[q] = pack_bf16x2(ex2_approx(fmaf(f.x, LOG2E_CE, -lse2)) * scale,
                             ex2_approx(fmaf(f.y, LOG2E_CE, -lse2)) * scale);
        }
      } else {
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const float2 f = unpack_bf16x2(w[q]);
          const int c = c0 + 2 * q;
          float a = 0.f, b = 0.f;
          if (c < V) a = (ex2_approx(fmaf(f.x, LOG2E_CE, -lse2)) - (c == t ? 1.f : 0.f)) * scale;
          if (c + 1 < V) b = (ex2_approx(fmaf(f.y, LOG2E_CE, -lse2)) - (c + 1 == t ? 1.f : 0.f)) * scale;
          o[q] = pack_bf16x2(a, b);
        }
      }
      return make_uint4(o[0], o[1], o[2], o[3]);
    };
    // two vectors per thread and iteration: both loads are in flight before either is used
    for (int vi = threadIdx.x; vi < nvec; vi += 2 * CE_STHREADS) {
      const int vj = vi + CE_STHREADS;
      const uint4 u0 = rowv[vi];
      const uint4 u1 = vj < nvec ? rowv[vj] : make_uint4(0u, 0u, 0u, 0u);
      rowv[vi] = grad8(u0, vi);
      if (vj < nvec) rowv[vj] = grad8(u1, vj);
    }
  }
}

// Softmax partials of whole bf16 rows (one pair per row), for rows whose producer left
// none: one warp per row, the maximum first, then the sum of exp(z - max) over v < V.
__global__ void __launch_bounds__(256) ce_row_stats_kernel(const bf16* __restrict__ logits, long long ld, int V,
                                                           int rows, float2* __restrict__ stats) {
  const long long row = (long long)blockIdx.x * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= rows) return;
  const bf16* z = logits + row * ld;
  float m = -INFINITY;
  for (int c = lane; c < V; c += 32) m = fmaxf(m, __bfloat162float(z[c]));
  m = warp_max(m);
  const float m2 = m * LOG2E_CE;
  float ssum = 0.f;
  for (int c = lane; c < V; c += 32) ssum += ex2_approx(fmaf(__bfloat162float(z[c]), LOG2E_CE, -m2));
  ssum = warp_sum(ssum);
  if (lane == 0) stats[row] = make_float2(m, ssum);
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
