// layernorm.cuh -- LayerNorm forward/backward, one warp per row, float4 loads,
// warp-shuffle reductions ("gpt/docs/LLM.md", Transformer Blocks: layer
// normalization before attention and before the MLP; Output Layer: final LN).
// y = (x - mean) / sqrt(var + 1e-5) * g + b with the biased variance; mean and
// 1/sqrt(var + eps) are kept for the backward pass.
#pragma once
#include "common.cuh"

namespace g2 {

constexpr int LN_WARPS = 8;  // rows per CTA in the forward kernel

template <class T>
__device__ __forceinline__ void store4(T* dst, float a, float b, float c, float d);
template <>
__device__ __forceinline__ void store4<float>(float* dst, float a, float b, float c, float d) {
  *reinterpret_cast<float4*>(dst) = make_float4(a, b, c, d);
}
template <>
__device__ __forceinline__ void store4<bf16>(bf16* dst, float a, float b, float c, float d) {
  *reinterpret_cast<uint2*>(dst) = make_uint2(pack_bf16x2(a, b), pack_bf16x2(c, d));
}

// Four consecutive values of a row of type D as floats (16-byte fp32 or 8-byte bf16 load).
template <class D>
__device__ __forceinline__ float4 load4(const D* p);
template <>
__device__ __forceinline__ float4 load4<float>(const float* p) {
  return *reinterpret_cast<const float4*>(p);
}
template <>
__device__ __forceinline__ float4 load4<bf16>(const bf16* p) {
  const uint2 u = *reinterpret_cast<const uint2*>(p);
  const float2 a = unpack_bf16x2(u.x), b = unpack_bf16x2(u.y);
  return make_float4(a.x, a.y, b.x, b.y);
}

// x: fp32 [N, C]; y: T [N, C]; mean, rstd: fp32 [N]. C % 4 == 0, C <= 128 * NV.
// PDL: launched as a programmatic dependent (generation steps), it waits for the
// previous kernel before reading x.
template <class T, int NV, bool PDL = false>
__global__ void __launch_bounds__(LN_WARPS * 32) layernorm_fwd_kernel(const float* __restrict__ x,
                                                                      const float* __restrict__ g,
                                                                      const float* __restrict__ b, T* __restrict__ y,
                                                                      float* __restrict__ mean,
                                                                      float* __restrict__ rstd, int N, int C) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  pdl_launch_dependents();
  if (PDL) pdl_wait();
  const long long row = (long long)blockIdx.x * LN_WARPS + warp;
  if (row >= N) return;
  const float* xr = x + row * C;
  float4 v[NV];
  float s = 0.f;
#pragma unroll
  for (int i = 0; i < NV; ++i) {
    const int c = (i * 32 + lane) * 4;
    if (c < C) {
      v[i] = *reinterpret_cast<const float4*>(xr + c);
      s += (v[i].x + v[i].y) + (v[i].z + v[i].w);
    }
  }
  const float mu = warp_sum(s) / (float)C;
  float ss = 0.f;
#pragma unroll
  for (int i = 0; i < NV; ++i) {
    const int c = (i * 32 + lane) * 4;
    if (c < C) {
      float a = v[i].x - mu, bb = v[i].y - mu, cc = v[i].z - mu, d = v[i].w - mu;
      ss += (a * a + bb * bb) + (cc * cc + d * d);
    }
  }
  const float var = warp_sum(ss) / (float)C;
  const float rs = 1.0f / sqrtf(var + 1e-5f);
  T* yr = y + row * C;
#pragma unroll
  for (int i = 0; i < NV; ++i) {
    const int c = (i * 32 + lane) * 4;
    if (c < C) {
      float4 gg = __ldg(reinterpret_cast<const float4*>(g + c));
      float4 bb = __ldg(reinterpret_cast<const float4*>(b + c));
      store4<T>(yr + c, (v[i].x - mu) * rs * gg.x + bb.x, (v[i].y - mu) * rs * gg.y + bb.y,
                (v[i].z - mu) * rs * gg.z + bb.z, (v[i].w - mu) * rs * gg.w + bb.w);
    }
  }
  if (lane == 0) {
    mean[row] = mu;
    rstd[row] = rs;
  }
}

// Backward. With xh = (x - mean) * rstd and dxh = dy * g:
//   dx = rstd * (dxh - mean(dxh) - xh * mean(dxh * xh))
// dres (+)= dx (accumulate selects += vs =), dres_act (nullable) gets a copy of
// the updated dres in the activation type. Per-CTA partial column sums go to
// part [3][gridDim.x][C]: dy*xh (gain grad), dy (bias grad) and, when
// with_rsum, the updated dres itself (the bias gradient of the linear layer whose
// output this residual is). Rows are assigned to CTAs in a fixed pattern, so the
// reduction order never changes between runs.
template <class T, int NV, class DY = float>
__global__ void __launch_bounds__(LN_WARPS * 32) layernorm_bwd_kernel(
    const DY* __restrict__ dy, const float* __restrict__ x, const float* __restrict__ g,
    const float* __restrict__ mean, const float* __restrict__ rstd, float* __restrict__ dres,
    T* __restrict__ dres_act, int accumulate, float* __restrict__ part, int with_rsum, int N, int C) {
  // per-warp column accumulators [warp][3][C] in dynamic shared memory; lane l owns
  // the float4 slots (i*32 + l), so there are no bank conflicts and no atomics
  extern __shared__ float4 ln_acc[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int C4 = C / 4;
  float4* accw = ln_acc + (size_t)warp * 3 * C4;
#pragma unroll
  for (int i = 0; i < NV; ++i) {
    const int c4 = i * 32 + lane;
    if (c4 < C4) accw[c4] = accw[C4 + c4] = accw[2 * C4 + c4] = make_float4(0.f, 0.f, 0.f, 0.f);
  }
  for (long long row = (long long)blockIdx.x * LN_WARPS + warp; row < N; row += (long long)gridDim.x * LN_WARPS) {
    const float mu = mean[row], rs = rstd[row];
    const DY* dyr = dy + row * C;
    const float* xr = x + row * C;
    float4 vd[NV], vx[NV], vr[NV];
    float m1 = 0.f, m2 = 0.f;
    float* dr = dres + row * C;
    if (accumulate) {  // issued now, so its latency overlaps the row statistics
#pragma unroll
      for (int i = 0; i < NV; ++i) {
        const int c = (i * 32 + lane) * 4;
        if (c < C) vr[i] = *reinterpret_cast<const float4*>(dr + c);
      }
    }
#pragma unroll
    for (int i = 0; i < NV; ++i) {
      const int c = (i * 32 + lane) * 4;
      if (c < C) {
        vd[i] = load4<DY>(dyr + c);
        float4 xx = *reinterpret_cast<const float4*>(xr + c);
        float4 gg = __ldg(reinterpret_cast<const float4*>(g + c));
        vx[i] = make_float4((xx.x - mu) * rs, (xx.y - mu) * rs, (xx.z - mu) * rs, (xx.w - mu) * rs);
        float a = vd[i].x * gg.x, b = vd[i].y * gg.y, cc = vd[i].z * gg.z, d = vd[i].w * gg.w;
        m1 += (a + b) + (cc + d);
        m2 += (a * vx[i].x + b * vx[i].y) + (cc * vx[i].z + d * vx[i].w);
        float4 ag = accw[i * 32 + lane], ab = accw[C4 + i * 32 + lane];
        ag.x += vd[i].x * vx[i].x;
        ag.y += vd[i].y * vx[i].y;
        ag.z += vd[i].z * vx[i].z;
        ag.w += vd[i].w * vx[i].w;
        ab.x += vd[i].x;
        ab.y += vd[i].y;
        ab.z += vd[i].z;
        ab.w += vd[i].w;
        accw[i * 32 + lane] = ag;
        accw[C4 + i * 32 + lane] = ab;
      }
    }
    m1 = warp_sum(m1) / (float)C;
    m2 = warp_sum(m2) / (float)C;
#pragma unroll
    for (int i = 0; i < NV; ++i) {
      const int c = (i * 32 + lane) * 4;
      if (c < C) {
        float4 gg = __ldg(reinterpret_cast<const float4*>(g + c));
        float4 o = make_float4(rs * (vd[i].x * gg.x - m1 - vx[i].x * m2), rs * (vd[i].y * gg.y - m1 - vx[i].y * m2),
                               rs * (vd[i].z * gg.z - m1 - vx[i].z * m2), rs * (vd[i].w * gg.w - m1 - vx[i].w * m2));
        if (accumulate) {
          o.x += vr[i].x;
          o.y += vr[i].y;
          o.z += vr[i].z;
          o.w += vr[i].w;
        }
        *reinterpret_cast<float4*>(dr + c) = o;
        if (dres_act) store4<T>(dres_act + row * C + c, o.x, o.y, o.z, o.w);
        if (with_rsum) {
          float4 ar = accw[2 * C4 + i * 32 + lane];
          ar.x += o.x;
          ar.y += o.y;
          ar.z += o.z;
          ar.w += o.w;
          accw[2 * C4 + i * 32 + lane] = ar;
        }
      }
    }
  }
  __syncthreads();
  // CTA partials: sum the warps' accumulators in a fixed order
  const int nsum = with_rsum ? 3 : 2;
  const float* accf = reinterpret_cast<const float*>(ln_acc);
  for (int idx = threadIdx.x; idx < nsum * C; idx += blockDim.x) {
    const int which = idx / C, col = idx - which * C;
    float sacc = 0.f;
#pragma unroll
    for (int w = 0; w < LN_WARPS; ++w) sacc += accf[((size_t)w * 3 + which) * C + col];
    part[((long long)which * gridDim.x + blockIdx.x) * C + col] = sacc;
  }
}

// Backward, staged through shared memory (the same mathematics and partial layout as
// layernorm_bwd_kernel). One CTA of LNR_WARPS warps per SM; warp w of CTA b takes rows
// b * LNR_WARPS + w + k * gridDim.x * LNR_WARPS, k = 0, 1, ... Each warp owns a ring of
// `stages` slots, a slot holding one row of dy, x and (when accumulating) dres; lane 0
// fills slot k % stages with 1-D bulk copies `stages` rows ahead of the row computed, so
// a warp always has rows in flight while it computes (an HBM-bound kernel needs bytes in
// flight, not threads). Column accumulators live in registers (lane l owns the float4
// columns i * 32 + l); at the end the warps' accumulators pass through shared memory and
// are summed in warp order, so the reduction order is fixed.
constexpr int LNR_WARPS = 8;
template <class T, int NV, class DY = float>
__global__ void __launch_bounds__(LNR_WARPS * 32, 1) layernorm_bwd_ring_kernel(
    const DY* __restrict__ dy, const float* __restrict__ x, const float* __restrict__ g,
    const float* __restrict__ mean, const float* __restrict__ rstd, float* __restrict__ dres,
    T* __restrict__ dres_act, int accumulate, float* __restrict__ part, int with_rsum, int N, int C, int stages,
    int* err, unsigned long long limit_ns) {
  extern __shared__ __align__(128) uint8_t lnr_smem[];
  __shared__ int s_abort;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int C4 = C / 4;
  const size_t slot_floats = (size_t)3 * C;  // dy | x | dres
  float* ring = reinterpret_cast<float*>(lnr_smem);
  float* mine = ring + (size_t)warp * stages * slot_floats;
  uint64_t* bars = reinterpret_cast<uint64_t*>(lnr_smem + (size_t)LNR_WARPS * stages * slot_floats * 4) + warp * stages;
  pdl_launch_dependents();
  if (threadIdx.x == 0) s_abort = 0;
  if (lane == 0) {
    for (int st = 0; st < stages; ++st) mbar_init(&bars[st], 1);
    fence_barrier_init();
  }
  __syncthreads();
  pdl_wait();  // programmatic dependent launch: global memory only from here on
  const long long first = (long long)blockIdx.x * LNR_WARPS + warp;
  const long long stride = (long long)gridDim.x * LNR_WARPS;
  const uint32_t row_bytes = (uint32_t)C * 4, dy_bytes = (uint32_t)(C * sizeof(DY));
  const uint32_t slot_bytes = dy_bytes + row_bytes * (accumulate ? 2u : 1u);
  // lane 0: request row k of this warp into slot k % stages
  auto issue = [&](long long k) {
    const long long row = first + k * stride;
    if (row >= N) return;
    float* slot = mine + (size_t)(k % stages) * slot_floats;
    uint64_t* bar = &bars[k % stages];
    mbar_arrive_expect_tx(bar, slot_bytes);
    bulk_load_1d(slot, dy + row * C, dy_bytes, bar);  // a bf16 row fills the first half of its part
    bulk_load_1d(slot + C, x + row * C, row_bytes, bar);
    if (accumulate) bulk_load_1d(slot + 2 * C, dres + row * C, row_bytes, bar);
  };
  if (lane == 0)
    for (int k = 0; k < stages; ++k) issue(k);
  float4 gv[NV], ag[NV], ab[NV], ar[NV];
#pragma unroll
  for (int i = 0; i < NV; ++i) {
    const int c4 = i * 32 + lane;
    gv[i] = c4 < C4 ? __ldg(reinterpret_cast<const float4*>(g) + c4) : make_float4(0.f, 0.f, 0.f, 0.f);
    ag[i] = ab[i] = ar[i] = make_float4(0.f, 0.f, 0.f, 0.f);
  }
  long long k = 0;
  bool ok = true;
  // the row statistics are fetched one row ahead, so their latency is not on the row's path
  float mu_next = first < N ? mean[first] : 0.f, rs_next = first < N ? rstd[first] : 0.f;
  for (;; ++k) {
    const long long row = first + k * stride;
    if (row >= N) break;
    const float mu = mu_next, rs = rs_next;
    if (row + stride < N) {
      mu_next = mean[row + stride];
      rs_next = rstd[row + stride];
    }
    const int st = (int)(k % stages);
    const uint32_t par = (uint32_t)((k / stages) & 1);
    int got = 1;
    if (lane == 0) got = mbar_wait_bounded(&bars[st], par, &s_abort, limit_ns) ? 1 : 0;
    got = __shfl_sync(0xffffffffu, got, 0);
    if (!got) {
      if (lane == 0) {
        raise_device_error(err, DEV_TIMEOUT);
        s_abort = 1;
      }
      ok = false;
      break;
    }
    mbar_try_wait(&bars[st], par);  // every lane observes the completed phase
    const DY* sdy = reinterpret_cast<const DY*>(mine + (size_t)st * slot_floats);
    const float4* sx = reinterpret_cast<const float4*>(mine + (size_t)st * slot_floats) + C4;
    const float4* sr = sx + C4;
    float m1 = 0.f, m2 = 0.f;
#pragma unroll
    for (int i = 0; i < NV; ++i) {
      const int c4 = i * 32 + lane;
      if (c4 < C4) {
        const float4 d = load4<DY>(sdy + c4 * 4), xx = sx[c4];
        const float4 xh = make_float4((xx.x - mu) * rs, (xx.y - mu) * rs, (xx.z - mu) * rs, (xx.w - mu) * rs);
        const float a = d.x * gv[i].x, b = d.y * gv[i].y, cc = d.z * gv[i].z, e = d.w * gv[i].w;
        m1 += (a + b) + (cc + e);
        m2 += (a * xh.x + b * xh.y) + (cc * xh.z + e * xh.w);
        ag[i].x += d.x * xh.x;
        ag[i].y += d.y * xh.y;
        ag[i].z += d.z * xh.z;
        ag[i].w += d.w * xh.w;
        ab[i].x += d.x;
        ab[i].y += d.y;
        ab[i].z += d.z;
        ab[i].w += d.w;
      }
    }
    m1 = warp_sum(m1) / (float)C;
    m2 = warp_sum(m2) / (float)C;
    float* dr = dres + row * C;
#pragma unroll
    for (int i = 0; i < NV; ++i) {
      const int c4 = i * 32 + lane;
      if (c4 < C4) {
        const float4 d = load4<DY>(sdy + c4 * 4), xx = sx[c4];
        const float4 xh = make_float4((xx.x - mu) * rs, (xx.y - mu) * rs, (xx.z - mu) * rs, (xx.w - mu) * rs);
        float4 o = make_float4(rs * (d.x * gv[i].x - m1 - xh.x * m2), rs * (d.y * gv[i].y - m1 - xh.y * m2),
                               rs * (d.z * gv[i].z - m1 - xh.z * m2), rs * (d.w * gv[i].w - m1 - xh.w * m2));
        if (accumulate) {
          const float4 r = sr[c4];
          o.x += r.x;
          o.y += r.y;
          o.z += r.z;
          o.w += r.w;
        }
        reinterpret_cast<float4*>(dr)[c4] = o;
        if (dres_act) store4<T>(dres_act + row * C + c4 * 4, o.x, o.y, o.z, o.w);
        if (with_rsum) {
          ar[i].x += o.x;
          ar[i].y += o.y;
          ar[i].z += o.z;
          ar[i].w += o.w;
        }
      }
    }
    __syncwarp();  // every lane has read the slot before it is refilled
    if (lane == 0) issue(k + stages);
  }
  if (!ok) {
    // rows already requested land before the CTA exits: wait (bounded) for each
    if (lane == 0) {
      int never = 0;
      for (long long kk = k + 1; kk < k + stages; ++kk)
        if (first + kk * stride < N)
          mbar_wait_bounded(&bars[kk % stages], (uint32_t)((kk / stages) & 1),
                            reinterpret_cast<volatile int*>(&never), limit_ns);
    }
  }
  __syncthreads();  // every warp arrives, including one that gave up (s_abort is set by then)
  if (s_abort) return;
  // every copy was consumed: the ring is free for the warps' accumulators [warp][3][C4]
  float4* accs = reinterpret_cast<float4*>(lnr_smem) + (size_t)warp * 3 * C4;
#pragma unroll
  for (int i = 0; i < NV; ++i) {
    const int c4 = i * 32 + lane;
    if (c4 < C4) {
      accs[c4] = ag[i];
      accs[C4 + c4] = ab[i];
      accs[2 * C4 + c4] = ar[i];
    }
  }
  __syncthreads();
  const int nsum = with_rsum ? 3 : 2;
  const float* accf = reinterpret_cast<const float*>(lnr_smem);
  for (int idx = threadIdx.x; idx < nsum * C; idx += blockDim.x) {
    const int which = idx / C, col = idx - which * C;
    float sacc = 0.f;
#pragma unroll
    for (int w = 0; w < LNR_WARPS; ++w) sacc += accf[((size_t)w * 3 + which) * C + col];
    part[((long long)which * gridDim.x + blockIdx.x) * C + col] = sacc;
  }
}

// Deterministic column reduction of up to three partial sets at once:
// out_v[c] (+)= sum_{p < P} part[(v*P + p)*ncols + c] for v = blockIdx.y. Each CTA
// owns 8 columns: thread t sums column t % 8 over rows p = t / 8, t / 8 + 32, ...
// (four loads in flight), then the 32 row-group sums are added in order.
struct ReduceOuts {
  float* out[3];
};
__global__ void __launch_bounds__(256) reduce_partials_kernel(const float* __restrict__ part, int P, int ncols,
                                                              ReduceOuts outs, int accumulate) {
  __shared__ float sm[32][9];
  const int v = blockIdx.y;
  const int cl = threadIdx.x & 7, rg = threadIdx.x >> 3;
  const int c = blockIdx.x * 8 + cl;
  const float* base = part + (long long)v * P * ncols + c;
  float s = 0.f;
  if (c < ncols) {
    int p = rg;
    for (; p + 96 < P; p += 128) {
      const float a0 = base[(long long)p * ncols], a1 = base[(long long)(p + 32) * ncols];
      const float a2 = base[(long long)(p + 64) * ncols], a3 = base[(long long)(p + 96) * ncols];
      s += a0;
      s += a1;
      s += a2;
      s += a3;
    }
    for (; p < P; p += 32) s += base[(long long)p * ncols];
  }
  sm[rg][cl] = s;
  __syncthreads();
  if (threadIdx.x < 8 && c < ncols) {
    float t = 0.f;
#pragma unroll
    for (int w = 0; w < 32; ++w) t += sm[w][cl];
    float* o = outs.out[v];
    o[c] = accumulate ? o[c] + t : t;
  }
}

// Column sums of an activation matrix y [N, ncols] (row stride ld), stage 1:
// CTA (bx, by) sums rows [by*rows_per, (by+1)*rows_per) of 8 * blockDim.x
// columns, 8 consecutive columns per thread (one 16-byte load of bf16, or two of fp32).
template <class T>
__global__ void colsum_partial_kernel(const T* __restrict__ y, long long ld, int N, int ncols, int rows_per,
                                      float* __restrict__ part) {
  const int c = (blockIdx.x * blockDim.x + threadIdx.x) * 8;
  if (c >= ncols) return;
  const int r0 = blockIdx.y * rows_per, r1 = min(N, r0 + rows_per);
  float s[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
  int r = r0;
  if (sizeof(T) == 2) {  // eight rows in flight per iteration; same summation order as one at a time
    for (; r + 8 <= r1; r += 8) {
      uint4 u[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) u[j] = *reinterpret_cast<const uint4*>(y + (long long)(r + j) * ld + c);
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const uint32_t w[4] = {u[j].x, u[j].y, u[j].z, u[j].w};
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const float2 f = unpack_bf16x2(w[q]);
          s[2 * q] += f.x;
          s[2 * q + 1] += f.y;
        }
      }
    }
  }
  for (; r < r1; ++r) {
    const T* p = y + (long long)r * ld + c;
    if (sizeof(T) == 2) {
      const uint4 u = *reinterpret_cast<const uint4*>(p);
      const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const float2 f = unpack_bf16x2(w[q]);
        s[2 * q] += f.x;
        s[2 * q + 1] += f.y;
      }
    } else {
      const float4 a = *reinterpret_cast<const float4*>(p);
      const float4 b = *reinterpret_cast<const float4*>(p + 4);
      s[0] += a.x; s[1] += a.y; s[2] += a.z; s[3] += a.w;
      s[4] += b.x; s[5] += b.y; s[6] += b.z; s[7] += b.w;
    }
  }
  float* o = part + (long long)blockIdx.y * ncols + c;
#pragma unroll
  for (int q = 0; q < 8; ++q) o[q] = s[q];
}

}  // namespace g2
