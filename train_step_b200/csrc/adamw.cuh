// adamw.cuh -- global-norm clip + AdamW over all parameters, one flat buffer
// ("AxonLM", Training Recipe: betas 0.9/0.95, weight decay 0.1 on 2D tensors
// only, gradient clip 1.0; "GPT From Scratch", Key decisions: decay only on
// parameters with two or more dimensions).
//
// The library stores every >= 2-D tensor first, so decay applies to the prefix
// [0, n_decay) of the flat buffer; the bf16 shadow copy that feeds the GEMMs
// covers the same prefix. With G = grad / k (k accumulated micro-batches):
//   ||G|| = sqrt(sum G^2);  c = min(1, 1 / (||G|| + 1e-6));  g = c G
//   p <- p (1 - lr wd) on the decayed prefix
//   m <- b1 m + (1 - b1) g;  v <- b2 v + (1 - b2) g^2
//   p <- p - (lr / (1 - b1^t)) m / (sqrt(v) / sqrt(1 - b2^t) + 1e-8)
// and the gradient buffer is zeroed for the next accumulation.
// The norm is a two-launch deterministic reduction: fixed per-CTA ranges summed
// in double, then every CTA of the update kernel re-adds the partials in order.
#pragma once
#include "common.cuh"

namespace g2 {

constexpr int ADAM_THREADS = 256;

__global__ void __launch_bounds__(ADAM_THREADS) sumsq_partial_kernel(const float* __restrict__ g, long long n,
                                                                     double* __restrict__ partial) {
  __shared__ double buf[ADAM_THREADS];
  const long long per = (n + gridDim.x - 1) / gridDim.x;
  const long long a = blockIdx.x * per, b = min(n, a + per);
  double s = 0.0;
  for (long long i = a + threadIdx.x; i < b; i += ADAM_THREADS) {
    const double x = (double)g[i];
    s += x * x;
  }
  buf[threadIdx.x] = s;
  __syncthreads();
  for (int w = ADAM_THREADS / 2; w > 0; w >>= 1) {
    if (threadIdx.x < w) buf[threadIdx.x] += buf[threadIdx.x + w];
    __syncthreads();
  }
  if (threadIdx.x == 0) partial[blockIdx.x] = buf[0];
}

struct AdamArgs {
  float* p;
  float* g;
  float* m;
  float* v;
  bf16* shadow;  // nullable (fp32 mode)
  long long n, n_decay;
  const double* partial;
  int nparts;
  float inv_k, lr, wd, b1, b2;
  float step_size;     // lr / (1 - b1^t)
  float inv_sqrt_bc2;  // 1 / sqrt(1 - b2^t)
  float* gnorm_out;    // device scalar: pre-clip ||G||
  const double* sumsq_total;  // nullable: the global sum of raw squared gradients, in place of the partials
  int zero_grad;              // zero the gradients that were read
};

__global__ void __launch_bounds__(ADAM_THREADS) adamw_kernel(const AdamArgs a) {
  __shared__ float s_coef;
  if (threadIdx.x == 0) {
    double ss = 0.0;
    if (a.sumsq_total)
      ss = *a.sumsq_total;
    else
      for (int i = 0; i < a.nparts; ++i) ss += a.partial[i];
    const double norm = sqrt(ss) * (double)a.inv_k;
    double coef = 1.0 / (norm + 1e-6);
    if (coef > 1.0) coef = 1.0;
    s_coef = (float)(coef * (double)a.inv_k);
    if (blockIdx.x == 0 && a.gnorm_out) *a.gnorm_out = (float)norm;
  }
  __syncthreads();
  const float gs = s_coef;
  const float decay = 1.0f - a.lr * a.wd;
  const long long n4 = a.n / 4;
  for (long long i = blockIdx.x * (long long)ADAM_THREADS + threadIdx.x; i < n4; i += (long long)gridDim.x * ADAM_THREADS) {
    const long long e = i * 4;
    float4 p = *reinterpret_cast<float4*>(a.p + e);
    float4 g = *reinterpret_cast<float4*>(a.g + e);
    float4 m = *reinterpret_cast<float4*>(a.m + e);
    float4 v = *reinterpret_cast<float4*>(a.v + e);
    const bool dec = e < a.n_decay;  // n_decay is a multiple of 4
    float* pp = &p.x;
    float* gg = &g.x;
    float* mm = &m.x;
    float* vv = &v.x;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float gj = gg[j] * gs;
      if (dec) pp[j] *= decay;
      mm[j] = a.b1 * mm[j] + (1.0f - a.b1) * gj;
      vv[j] = a.b2 * vv[j] + (1.0f - a.b2) * gj * gj;
      const float denom = sqrtf(vv[j]) * a.inv_sqrt_bc2 + 1e-8f;
      pp[j] -= a.step_size * (mm[j] / denom);
    }
    *reinterpret_cast<float4*>(a.p + e) = p;
    *reinterpret_cast<float4*>(a.m + e) = m;
    *reinterpret_cast<float4*>(a.v + e) = v;
    if (a.zero_grad) *reinterpret_cast<float4*>(a.g + e) = make_float4(0.f, 0.f, 0.f, 0.f);
    if (a.shadow && dec)
      *reinterpret_cast<uint2*>(a.shadow + e) = make_uint2(pack_bf16x2(p.x, p.y), pack_bf16x2(p.z, p.w));
  }
}

// out[0] = sum of the partials in index order (the sum of squares of a storage range).
__global__ void sum_partials_kernel(const double* __restrict__ partial, int nparts, double* __restrict__ out) {
  if (threadIdx.x == 0 && blockIdx.x == 0) {
    double s = 0.0;
    for (int i = 0; i < nparts; ++i) s += partial[i];
    out[0] = s;
  }
}

// bf16 shadow of the decayed prefix (after set_params / create).
__global__ void cast_shadow_kernel(const float* __restrict__ p, bf16* __restrict__ shadow, long long n) {
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n; i += (long long)gridDim.x * blockDim.x)
    shadow[i] = __float2bfloat16_rn(p[i]);
}

}  // namespace g2
