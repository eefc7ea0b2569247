// cross_entropy.cuh -- softmax cross-entropy over one chunk of logit rows, in
// place: logits in, d(loss)/d(logits) out ("gpt/docs/LLM.md", Output Layer:
// linear projection to the vocabulary; next-token loss on the shifted targets).
//
// For each row n: lse = logsumexp over the first V columns (padding columns V..ld
// are storage only); row_loss[n] = lse - z[target]; then
//   z[v] <- (exp(z[v] - lse) - [v == target]) * scale  for v < V,  0 for v >= V.
// One CTA of CE_THREADS threads per row; the row stays in registers between the
// statistics pass and the write pass, so HBM sees one read and one write.
#pragma once
#include "common.cuh"

namespace g2 {

constexpr int CE_THREADS = 512;
constexpr int CE_MAXVEC = 16;  // per thread: 16 x 8 bf16 -> rows up to 65536 columns

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

__global__ void __launch_bounds__(CE_THREADS) cross_entropy_bf16_kernel(bf16* __restrict__ logits, long long ld, int V,
                                                                        const int* __restrict__ tgt, float scale,
                                                                        float* __restrict__ row_loss, int* err) {
  __shared__ float buf[CE_THREADS / 32];
  const long long row = blockIdx.x;
  bf16* z = logits + row * ld;
  int t = tgt[row];
  if (t < 0 || t >= V) {
    if (threadIdx.x == 0) raise_device_error(err, DEV_TOKEN_RANGE);
    t = 0;
  }
  const float zt = __bfloat162float(z[t]);
  const int nvec = (int)(ld / 8);
  uint4 r[CE_MAXVEC];
  float mx = -INFINITY;
#pragma unroll
  for (int i = 0; i < CE_MAXVEC; ++i) {
    const int vi = threadIdx.x + i * CE_THREADS;
    if (vi < nvec) {
      r[i] = *reinterpret_cast<const uint4*>(z + (long long)vi * 8);
      const uint32_t w[4] = {r[i].x, r[i].y, r[i].z, r[i].w};
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const float2 f = unpack_bf16x2(w[q]);
        const int c = vi * 8 + 2 * q;
        if (c < V) mx = fmaxf(mx, f.x);
        if (c + 1 < V) mx = fmaxf(mx, f.y);
      }
    }
  }
  mx = block_reduce_ce(mx, true, buf);
  float se = 0.f;
#pragma unroll
  for (int i = 0; i < CE_MAXVEC; ++i) {
    const int vi = threadIdx.x + i * CE_THREADS;
    if (vi < nvec) {
      const uint32_t w[4] = {r[i].x, r[i].y, r[i].z, r[i].w};
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const float2 f = unpack_bf16x2(w[q]);
        const int c = vi * 8 + 2 * q;
        if (c < V) se += __expf(f.x - mx);
        if (c + 1 < V) se += __expf(f.y - mx);
      }
    }
  }
  se = block_reduce_ce(se, false, buf);
  const float lse = mx + __logf(se);
  if (threadIdx.x == 0) row_loss[row] = lse - zt;
#pragma unroll
  for (int i = 0; i < CE_MAXVEC; ++i) {
    const int vi = threadIdx.x + i * CE_THREADS;
    if (vi < nvec) {
      const uint32_t w[4] = {r[i].x, r[i].y, r[i].z, r[i].w};
      uint32_t o[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const float2 f = unpack_bf16x2(w[q]);
        const int c = vi * 8 + 2 * q;
        float a = c < V ? (__expf(f.x - lse) - (c == t ? 1.f : 0.f)) * scale : 0.f;
        float b = c + 1 < V ? (__expf(f.y - lse) - (c + 1 == t ? 1.f : 0.f)) * scale : 0.f;
        o[q] = pack_bf16x2(a, b);
      }
      *reinterpret_cast<uint4*>(z + (long long)vi * 8) = make_uint4(o[0], o[1], o[2], o[3]);
    }
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
