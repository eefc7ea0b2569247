// attention.cuh -- causal multi-head self-attention, forward and backward, that
// never materialises the T x T score matrix ("AxonLM", Key Features: Flash
// Attention; "GPT From Scratch", Key decisions: written-out masked softmax and the
// fused path must agree). Softmax is taken online over key blocks; the forward
// saves lse = logsumexp of each query's scaled scores for the backward.
//
// Layout: qkv [B*T, 3C] (q | k | v column blocks; head h uses columns
// [h*hd, (h+1)*hd) of each), out [B*T, C], lse [B, NH, T] fp32.
//
// The bf16 path (tcgen05 tensor cores) is in attention_tc.cuh; this file holds
// the per-row dO.O sums the backward needs and the fp32 path: one warp per query
// (or key) row, exact expf, for the parity mode. Both backward paths are
// deterministic (no atomics).
#pragma once
#include "common.cuh"

namespace g2 {

constexpr float LOG2E = 1.4426950408889634f;
constexpr float LN2 = 0.6931471805599453f;

// ----------------------------------------------------------------------------
// backward: D_i = rowsum(dO_i * O_i) per (row, head)
// ----------------------------------------------------------------------------
template <class T>
__global__ void attn_bwd_dot_kernel(const T* __restrict__ out, const T* __restrict__ dout, float* __restrict__ D,
                                    int Bsz, int Tn, int NH, int hd) {
  const long long gw = (blockIdx.x * (long long)blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  const long long total = (long long)Bsz * Tn * NH;
  if (gw >= total) return;
  const int h = (int)(gw % NH);
  const long long row = gw / NH;  // b*T + t
  const int C = NH * hd;
  const T* o = out + row * C + h * hd;
  const T* d = dout + row * C + h * hd;
  float s = 0.f;
  for (int e = lane; e < hd; e += 32) s += to_f32<T>(o[e]) * to_f32<T>(d[e]);
  s = warp_sum(s);
  if (lane == 0) {
    const int b = (int)(row / Tn), t = (int)(row % Tn);
    D[((long long)b * NH + h) * Tn + t] = s;
  }
}

// bf16, hd = 64: eight threads per (row, head), each one 16-byte piece of O and of dO
// (consecutive threads read consecutive 16 bytes, so a warp's loads are 512 contiguous
// bytes of each tensor), the eight partial dot products combined by three shuffles in a
// fixed order.
__global__ void attn_bwd_dot64_bf16_kernel(const bf16* __restrict__ out, const bf16* __restrict__ dout,
                                           float* __restrict__ D, int Bsz, int Tn, int NH) {
  pdl_launch_dependents();
  pdl_wait();
  const long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x;  // 16-byte piece
  const long long npieces = (long long)Bsz * Tn * NH * 8;
  const bool in = i < npieces;
  float s = 0.f;
  if (in) {
    const uint4 a = __ldg(reinterpret_cast<const uint4*>(out) + i), b = __ldg(reinterpret_cast<const uint4*>(dout) + i);
    const uint32_t wa[4] = {a.x, a.y, a.z, a.w}, wb[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const float2 fa = unpack_bf16x2(wa[q]), fb = unpack_bf16x2(wb[q]);
      s += fa.x * fb.x + fa.y * fb.y;
    }
  }
  s += __shfl_xor_sync(0xffffffffu, s, 1);
  s += __shfl_xor_sync(0xffffffffu, s, 2);
  s += __shfl_xor_sync(0xffffffffu, s, 4);
  if (in && (i & 7) == 0) {
    const long long rh = i >> 3;  // (row, head)
    const int h = (int)(rh % NH);
    const long long row = rh / NH;
    const int b = (int)(row / Tn), t = (int)(row % Tn);
    D[((long long)b * NH + h) * Tn + t] = s;
  }
}

// ----------------------------------------------------------------------------
// fp32 SIMT attention (parity mode): one warp per row, hd a multiple of 32, <= 128
// ----------------------------------------------------------------------------
__global__ void attn_fwd_f32_kernel(const float* __restrict__ qkv, float* __restrict__ out, float* __restrict__ lse,
                                    int Bsz, int T, int NH, int hd, float scale) {
  const long long gw = (blockIdx.x * (long long)blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (gw >= (long long)Bsz * NH * T) return;
  const int i = (int)(gw % T);
  const int bh = (int)(gw / T), b = bh / NH, h = bh % NH;
  const int C = NH * hd, R = hd / 32;
  const long long ld = 3LL * C;
  const float* q = qkv + ((long long)b * T + i) * ld + h * hd;
  float qv[4], acc[4] = {0.f, 0.f, 0.f, 0.f};
  for (int r = 0; r < R; ++r) qv[r] = q[lane + 32 * r];
  float m = -INFINITY, l = 0.f;
  for (int j = 0; j <= i; ++j) {
    const float* k = qkv + ((long long)b * T + j) * ld + C + h * hd;
    const float* v = k + C;
    float d = 0.f;
    for (int r = 0; r < R; ++r) d += qv[r] * k[lane + 32 * r];
    const float s = warp_sum(d) * scale;
    const float mn = fmaxf(m, s);
    const float corr = expf(m - mn), p = expf(s - mn);
    l = l * corr + p;
    for (int r = 0; r < R; ++r) acc[r] = acc[r] * corr + p * v[lane + 32 * r];
    m = mn;
  }
  float* o = out + ((long long)b * T + i) * C + h * hd;
  for (int r = 0; r < R; ++r) o[lane + 32 * r] = acc[r] / l;
  if (lane == 0) lse[((long long)b * NH + h) * T + i] = m + logf(l);
}

__global__ void attn_bwd_dq_f32_kernel(const float* __restrict__ qkv, const float* __restrict__ dout,
                                       const float* __restrict__ lse, const float* __restrict__ Dg,
                                       float* __restrict__ dqkv, int Bsz, int T, int NH, int hd, float scale) {
  const long long gw = (blockIdx.x * (long long)blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (gw >= (long long)Bsz * NH * T) return;
  const int i = (int)(gw % T);
  const int bh = (int)(gw / T), b = bh / NH, h = bh % NH;
  const int C = NH * hd, R = hd / 32;
  const long long ld = 3LL * C;
  const float* q = qkv + ((long long)b * T + i) * ld + h * hd;
  const float* dy = dout + ((long long)b * T + i) * C + h * hd;
  const float L = lse[((long long)b * NH + h) * T + i], Di = Dg[((long long)b * NH + h) * T + i];
  float qv[4], dyv[4], acc[4] = {0.f, 0.f, 0.f, 0.f};
  for (int r = 0; r < R; ++r) {
    qv[r] = q[lane + 32 * r];
    dyv[r] = dy[lane + 32 * r];
  }
  for (int j = 0; j <= i; ++j) {
    const float* k = qkv + ((long long)b * T + j) * ld + C + h * hd;
    const float* v = k + C;
    float d = 0.f, e = 0.f;
    for (int r = 0; r < R; ++r) {
      d += qv[r] * k[lane + 32 * r];
      e += dyv[r] * v[lane + 32 * r];
    }
    const float p = expf(warp_sum(d) * scale - L);
    const float ds = p * (warp_sum(e) - Di);
    for (int r = 0; r < R; ++r) acc[r] += ds * k[lane + 32 * r];
  }
  float* dq = dqkv + ((long long)b * T + i) * ld + h * hd;
  for (int r = 0; r < R; ++r) dq[lane + 32 * r] = acc[r] * scale;
}

__global__ void attn_bwd_dkdv_f32_kernel(const float* __restrict__ qkv, const float* __restrict__ dout,
                                         const float* __restrict__ lse, const float* __restrict__ Dg,
                                         float* __restrict__ dqkv, int Bsz, int T, int NH, int hd, float scale) {
  const long long gw = (blockIdx.x * (long long)blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (gw >= (long long)Bsz * NH * T) return;
  const int j = (int)(gw % T);
  const int bh = (int)(gw / T), b = bh / NH, h = bh % NH;
  const int C = NH * hd, R = hd / 32;
  const long long ld = 3LL * C;
  const float* k = qkv + ((long long)b * T + j) * ld + C + h * hd;
  const float* v = k + C;
  float kv[4], vv[4], dk[4] = {0.f, 0.f, 0.f, 0.f}, dv[4] = {0.f, 0.f, 0.f, 0.f};
  for (int r = 0; r < R; ++r) {
    kv[r] = k[lane + 32 * r];
    vv[r] = v[lane + 32 * r];
  }
  for (int i = j; i < T; ++i) {
    const float* q = qkv + ((long long)b * T + i) * ld + h * hd;
    const float* dy = dout + ((long long)b * T + i) * C + h * hd;
    const float L = lse[((long long)b * NH + h) * T + i], Di = Dg[((long long)b * NH + h) * T + i];
    float d = 0.f, e = 0.f;
    for (int r = 0; r < R; ++r) {
      d += q[lane + 32 * r] * kv[r];
      e += dy[lane + 32 * r] * vv[r];
    }
    const float p = expf(warp_sum(d) * scale - L);
    const float ds = p * (warp_sum(e) - Di);
    for (int r = 0; r < R; ++r) {
      dk[r] += ds * q[lane + 32 * r];
      dv[r] += p * dy[lane + 32 * r];
    }
  }
  float* dkr = dqkv + ((long long)b * T + j) * ld + C + h * hd;
  float* dvr = dkr + C;
  for (int r = 0; r < R; ++r) {
    dkr[lane + 32 * r] = dk[r] * scale;
    dvr[lane + 32 * r] = dv[r];
  }
}

}  // namespace g2
