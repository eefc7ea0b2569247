// decode.cuh -- kernels of one generation step with a key/value cache.
//
// A step advances B <= 16 sequences by one token. Its linear layers are skinny
// products (B rows against a [N, K] weight), bound by reading each weight once and by
// the latency of a chain of small kernels: they use register-level m16n8k16 tensor-core
// products with the batch rows as the 16-row operand and 16-byte weight loads spread over
// every SM, not 128-row tcgen05 tiles that would sit at least 7/8 empty behind a TMEM and
// barrier set-up. Attention is one query row per (sequence, head) against the cached keys
// and values of positions 0..pos.
#pragma once
#include "common.cuh"
#include "gemm_tc.cuh"

namespace g2 {

constexpr int DEC_MAX_B = 16;  // sequences advanced by one step
constexpr int DEC_WARPS = 8;
constexpr int DEC_PF = 8;  // weight slices in flight per warp in the skinny product
constexpr int DEC_ATT_THREADS = 256;
constexpr int DEC_HD = 64;  // head size the attention kernel is written for

__device__ __forceinline__ void dec_unpack8(const uint4& r, float* f) {
  const float2 a = unpack_bf16x2(r.x), b = unpack_bf16x2(r.y), c = unpack_bf16x2(r.z), d = unpack_bf16x2(r.w);
  f[0] = a.x; f[1] = a.y; f[2] = b.x; f[3] = b.y;
  f[4] = c.x; f[5] = c.y; f[6] = d.x; f[7] = d.y;
}

// Weight rows are read once per step: bypass L1 and do not keep them in it.
__device__ __forceinline__ uint4 dec_ld_stream(const void* p) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p));
  return r;
}

// One m16n8k16 bf16 tensor-core product with fp32 accumulation (D += A B): A is 16 x 16
// (rows x k), B is 16 x 8 (k x columns), fragments as the PTX ISA lays them out.
__device__ __forceinline__ void dec_mma(float* d, uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3, uint32_t b0,
                                        uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// out[b][n] = epilogue(sum_k x[b][k] * W[n][k] (+ bias[n])) for b < B <= 16, n < N.
// W: bf16 [N][K] row-major (the K-major layout the training GEMMs read), K % 32 == 0.
// x: bf16 rows of stride ldx; or, with LN, fp32 rows of the residual stream that the kernel
// layer-normalises itself (y = (x - mean) * rstd * ln_g + ln_b with the biased variance and
// eps 1e-5, rounded to bf16 as the LayerNorm kernel stores it), so that no LayerNorm launch
// sits between two products.
// The batch rows are the 16-row operand of m16n8k16 tensor-core products: each block stages
// the B rows of x in shared memory as bf16 rows of K + 8 (the 16-byte pad spreads the
// fragment loads over all banks; rows B..15 enter the products as zero registers), and each
// warp accumulates one 16 x 8 output tile (8 weight rows) over its share of K, with up to 8
// weight slices in flight; KW warps split K and their tiles are summed through shared
// memory. For a 32-wide slice of K a lane loads 16 bytes of one weight row (row n0 + lane/4,
// k = 8 (lane % 4) ... + 7) and 16 bytes of x rows lane/4 and lane/4 + 8 at the same k; the
// slice's k positions are assigned to the two k16 products so that these registers are
// exactly the A and B fragments (any one-to-one assignment of k gives the same sum).
// Epilogues: EPI_BF16 (bf16 out), EPI_BF16_GELU (bf16 gelu_tanh(acc + bias)), EPI_F32_RESID
// (fp32 out = resid + acc + bias), EPI_F32 (fp32 out = acc).
template <int EPI, int KW, bool LN>
__global__ void __launch_bounds__(DEC_WARPS * 32)
    gemv_bf16_kernel(const void* __restrict__ xin, int64_t ldx, int B, const bf16* __restrict__ W, int N, int K,
                     const float* __restrict__ bias, void* __restrict__ out, int64_t ldo,
                     const float* __restrict__ resid, int64_t ldr, const float* __restrict__ ln_g,
                     const float* __restrict__ ln_b) {
  constexpr int NW = DEC_WARPS / KW;  // 8-column tiles per block
  extern __shared__ __align__(16) unsigned char dec_smem[];
  bf16* xs = reinterpret_cast<bf16*>(dec_smem);  // [16][K + 8]
  __shared__ float red[DEC_WARPS][4][32];
  __shared__ float stat[DEC_MAX_B][2];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int kw = warp % KW, nw = warp / KW;
  const int g = lane >> 2, q = lane & 3;
  const int n0 = (blockIdx.x * NW + nw) * 8;
  const int xstride = K + 8;  // rows 0..B-1 staged; the 16-byte pad spreads fragment loads over the banks
  const bf16* wrow = W + (int64_t)(n0 + g) * K + q * 8;
  const bool wok = n0 + g < N;
  // this warp's 32-wide slices of K are kw, kw + KW, ...; weights do not depend on the
  // previous kernel, so the first DEC_PF slices are fetched before waiting for it, and
  // each slot is refilled DEC_PF slices ahead as it is consumed
  const int nslices = (K / 32 - kw + KW - 1) / KW;
  uint4 wbuf[DEC_PF];
#pragma unroll
  for (int j = 0; j < DEC_PF; ++j) {
    wbuf[j] = make_uint4(0u, 0u, 0u, 0u);
    if (wok && j < nslices) wbuf[j] = dec_ld_stream(wrow + (kw + j * KW) * 32);
  }
  pdl_launch_dependents();
  pdl_wait();
  // stage the B rows of x as bf16
  if (LN) {
    const float* xf = static_cast<const float*>(xin);
    for (int b = warp; b < B; b += DEC_WARPS) {  // row statistics, K % 4 == 0
      const float* xr = xf + (int64_t)b * ldx;
      float s = 0.f;
      for (int c = lane * 4; c < K; c += 128) {
        const float4 v = *reinterpret_cast<const float4*>(xr + c);
        s += (v.x + v.y) + (v.z + v.w);
      }
      const float mu = warp_sum(s) / (float)K;
      float ss = 0.f;
      for (int c = lane * 4; c < K; c += 128) {
        const float4 v = *reinterpret_cast<const float4*>(xr + c);
        const float e0 = v.x - mu, e1 = v.y - mu, e2 = v.z - mu, e3 = v.w - mu;
        ss += (e0 * e0 + e1 * e1) + (e2 * e2 + e3 * e3);
      }
      const float var = warp_sum(ss) / (float)K;
      if (lane == 0) {
        stat[b][0] = mu;
        stat[b][1] = 1.0f / sqrtf(var + 1e-5f);
      }
    }
    __syncthreads();
    const int per_row = K / 4;
    for (int i = threadIdx.x; i < B * per_row; i += DEC_WARPS * 32) {
      const int b = i / per_row, c = (i % per_row) * 4;
      const float4 v = *reinterpret_cast<const float4*>(xf + (int64_t)b * ldx + c);
      const float4 gg = __ldg(reinterpret_cast<const float4*>(ln_g + c));
      const float4 bb = __ldg(reinterpret_cast<const float4*>(ln_b + c));
      const float mu = stat[b][0], rs = stat[b][1];
      *reinterpret_cast<uint2*>(xs + b * xstride + c) =
          make_uint2(pack_bf16x2((v.x - mu) * rs * gg.x + bb.x, (v.y - mu) * rs * gg.y + bb.y),
                     pack_bf16x2((v.z - mu) * rs * gg.z + bb.z, (v.w - mu) * rs * gg.w + bb.w));
    }
  } else {
    const bf16* x = static_cast<const bf16*>(xin);
    const int per_row = K / 8;
    for (int i = threadIdx.x; i < B * per_row; i += DEC_WARPS * 32) {
      const int b = i / per_row, c = (i % per_row) * 8;
      *reinterpret_cast<uint4*>(xs + b * xstride + c) = *reinterpret_cast<const uint4*>(x + (int64_t)b * ldx + c);
    }
  }
  __syncthreads();
  float d[4] = {0.f, 0.f, 0.f, 0.f};
  const bool rlo = g < B, rhi = g + 8 < B;  // rows g and g + 8 exist (others enter as zeros)
  const bf16* xa = xs + g * xstride + q * 8;
  const bf16* xb = xa + 8 * xstride;
  for (int base = 0; base < nslices; base += DEC_PF) {
#pragma unroll
    for (int j = 0; j < DEC_PF; ++j) {
      const int sl = base + j;
      if (sl < nslices) {
        const uint4 w = wbuf[j];
        const int sn = sl + DEC_PF;
        if (wok && sn < nslices) wbuf[j] = dec_ld_stream(wrow + (kw + sn * KW) * 32);
        const int kb = (kw + sl * KW) * 32;
        const uint4 z = make_uint4(0u, 0u, 0u, 0u);
        const uint4 a = rlo ? *reinterpret_cast<const uint4*>(xa + kb) : z;
        const uint4 c = rhi ? *reinterpret_cast<const uint4*>(xb + kb) : z;
        dec_mma(d, a.x, c.x, a.y, c.y, w.x, w.y);  // k = 8q + {0,1} and 8q + {2,3} of the slice
        dec_mma(d, a.z, c.z, a.w, c.w, w.z, w.w);  // k = 8q + {4,5} and 8q + {6,7}
      }
    }
  }
  if (KW > 1) {
#pragma unroll
    for (int i = 0; i < 4; ++i) red[warp][i][lane] = d[i];
    __syncthreads();
    if (kw != 0) return;
#pragma unroll
    for (int j = 1; j < KW; ++j)
#pragma unroll
      for (int i = 0; i < 4; ++i) d[i] += red[warp + j][i][lane];
  }
  // d[0], d[1]: row g, columns 2q, 2q+1; d[2], d[3]: row g + 8, the same columns
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int b = g + (i >> 1) * 8, n = n0 + 2 * q + (i & 1);
    if (b >= B || n >= N) continue;
    const float v = d[i] + ((EPI != EPI_F32 && bias) ? bias[n] : 0.f);
    if (EPI == EPI_BF16) static_cast<bf16*>(out)[(int64_t)b * ldo + n] = __float2bfloat16_rn(v);
    if (EPI == EPI_BF16_GELU) static_cast<bf16*>(out)[(int64_t)b * ldo + n] = __float2bfloat16_rn(gelu_tanh(v));
    if (EPI == EPI_F32_RESID) static_cast<float*>(out)[(int64_t)b * ldo + n] = resid[(int64_t)b * ldr + n] + v;
    if (EPI == EPI_F32) static_cast<float*>(out)[(int64_t)b * ldo + n] = v;
  }
}

// One generation step of causal attention (head size 64), split over S blocks per
// (sequence b, head h) along the keys. The position p = *pos_ptr comes from device memory
// so that a captured step can be replayed. Keys 0..p are cut into S contiguous ranges;
// the block whose range holds p first appends the step's key and value (columns C.. and
// 2C.. of its qkv row) to the cache at p. Each block forms scores s_j = scale * q.k_j in
// log2 units, m = max s_j, l = sum 2^(s_j - m) and o = sum 2^(s_j - m) v_j in fp32; with
// S = 1 it writes att = o / l directly, otherwise (m, l, o) to part[(b*NH + h)*S + s]
// for decode_attn_combine_kernel.
// qkv: bf16 [B][3C]; cache: bf16, sequence b at cache + b*cache_seq, row t at +t*2C,
// keys in columns [0, C), values in [C, 2C); att: bf16 [B][C].
// 8 warps; a warp covers 4 keys per load (8 lanes x 8 elements), two loads in flight.
// Dynamic shared memory holds one range's scores (at most the cache length).
constexpr int DEC_PART = DEC_HD + 2;  // floats of one partial result: m, l, o[64]
constexpr int DEC_MAX_SPLIT = 16;

__device__ __forceinline__ float dec_dot8(const float* q, const uint4& r) {
  float k[8];
  dec_unpack8(r, k);
  float d = 0.f;
#pragma unroll
  for (int e = 0; e < 8; ++e) d = fmaf(q[e], k[e], d);
  return d;
}

__global__ void __launch_bounds__(DEC_ATT_THREADS)
    decode_attn_kernel(const bf16* __restrict__ qkv, bf16* __restrict__ cache, int64_t cache_seq, int C, int NH,
                       const int* __restrict__ pos_ptr, int S, float scale_log2, bf16* __restrict__ att,
                       float* __restrict__ part) {
  extern __shared__ float sc[];
  __shared__ float red[DEC_ATT_THREADS / 32][DEC_HD];
  __shared__ float wred[DEC_ATT_THREADS / 32];
  constexpr int NWARP = DEC_ATT_THREADS / 32;
  pdl_launch_dependents();
  pdl_wait();
  const int bh = blockIdx.x / S, split = blockIdx.x % S;
  const int b = bh / NH, h = bh % NH;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int g = lane >> 3, c8 = (lane & 7) * 8;
  const int64_t C2 = 2 * (int64_t)C;
  const int pos = *pos_ptr, nkeys = pos + 1;
  const int chunk = (nkeys + S - 1) / S;
  const int j0 = split * chunk, j1 = min(nkeys, j0 + chunk);
  const bf16* row = qkv + (int64_t)b * 3 * C;
  bf16* kc = cache + (int64_t)b * cache_seq + h * DEC_HD;
  bf16* vc = kc + C;
  if (j0 <= pos && pos < j1) {
    if (tid < 16) {
      const int which = tid >> 3, off = (tid & 7) * 8;  // 0: key, 1: value
      const uint4 val = *reinterpret_cast<const uint4*>(row + (1 + which) * C + h * DEC_HD + off);
      *reinterpret_cast<uint4*>((which ? vc : kc) + pos * C2 + off) = val;
    }
    __syncthreads();
  }
  float q[8];
  dec_unpack8(*reinterpret_cast<const uint4*>(row + h * DEC_HD + c8), q);
#pragma unroll
  for (int e = 0; e < 8; ++e) q[e] *= scale_log2;
  // scores; the loop bound is uniform over the warp (shuffles inside)
  for (int jb = j0 + warp * 4; jb < j1; jb += 2 * NWARP * 4) {
    const int ja = jb + g, jc = jb + NWARP * 4 + g;
    uint4 ra = make_uint4(0u, 0u, 0u, 0u), rc = make_uint4(0u, 0u, 0u, 0u);
    if (ja < j1) ra = *reinterpret_cast<const uint4*>(kc + ja * C2 + c8);
    if (jc < j1) rc = *reinterpret_cast<const uint4*>(kc + jc * C2 + c8);
    float da = dec_dot8(q, ra), dc = dec_dot8(q, rc);
#pragma unroll
    for (int o = 1; o < 8; o <<= 1) {
      da += __shfl_xor_sync(0xffffffffu, da, o);
      dc += __shfl_xor_sync(0xffffffffu, dc, o);
    }
    if ((lane & 7) == 0) {
      if (ja < j1) sc[ja - j0] = da;
      if (jc < j1) sc[jc - j0] = dc;
    }
  }
  __syncthreads();
  const int n = j1 > j0 ? j1 - j0 : 0;
  float mx = -INFINITY;
  for (int j = tid; j < n; j += DEC_ATT_THREADS) mx = fmaxf(mx, sc[j]);
  mx = warp_max(mx);
  if (lane == 0) wred[warp] = mx;
  __syncthreads();
  mx = wred[0];
#pragma unroll
  for (int w = 1; w < NWARP; ++w) mx = fmaxf(mx, wred[w]);
  __syncthreads();
  float sum = 0.f;
  for (int j = tid; j < n; j += DEC_ATT_THREADS) {
    const float p = exp2f(sc[j] - mx);
    sc[j] = p;
    sum += p;
  }
  sum = warp_sum(sum);
  if (lane == 0) wred[warp] = sum;
  __syncthreads();
  sum = 0.f;
#pragma unroll
  for (int w = 0; w < NWARP; ++w) sum += wred[w];
  float o[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
  for (int jb = j0 + warp * 4; jb < j1; jb += 2 * NWARP * 4) {
    const int ja = jb + g, jc = jb + NWARP * 4 + g;
    uint4 ra = make_uint4(0u, 0u, 0u, 0u), rc = make_uint4(0u, 0u, 0u, 0u);
    float pa = 0.f, pc = 0.f;
    if (ja < j1) {
      ra = *reinterpret_cast<const uint4*>(vc + ja * C2 + c8);
      pa = sc[ja - j0];
    }
    if (jc < j1) {
      rc = *reinterpret_cast<const uint4*>(vc + jc * C2 + c8);
      pc = sc[jc - j0];
    }
    float va[8], vv[8];
    dec_unpack8(ra, va);
    dec_unpack8(rc, vv);
#pragma unroll
    for (int e = 0; e < 8; ++e) o[e] = fmaf(pa, va[e], fmaf(pc, vv[e], o[e]));
  }
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    o[e] += __shfl_xor_sync(0xffffffffu, o[e], 8);
    o[e] += __shfl_xor_sync(0xffffffffu, o[e], 16);
  }
  if (lane < 8) {
#pragma unroll
    for (int e = 0; e < 8; ++e) red[warp][c8 + e] = o[e];
  }
  __syncthreads();
  if (tid < DEC_HD) {
    float acc = 0.f;
#pragma unroll
    for (int w = 0; w < NWARP; ++w) acc += red[w][tid];
    if (S == 1) {
      att[(int64_t)b * C + h * DEC_HD + tid] = __float2bfloat16_rn(acc / sum);
    } else {
      float* pp = part + (int64_t)blockIdx.x * DEC_PART;
      pp[2 + tid] = acc;
      if (tid == 0) {
        pp[0] = mx;  // -inf for an empty range
        pp[1] = sum;
      }
    }
  }
}

// att[b][h*64 + d] from the S partial results of (b, h): rescale each to the largest m.
__global__ void decode_attn_combine_kernel(const float* __restrict__ part, int S, int C, int NH,
                                           bf16* __restrict__ att) {
  pdl_launch_dependents();
  pdl_wait();
  const int bh = blockIdx.x, d = threadIdx.x;
  const float* pp = part + (int64_t)bh * S * DEC_PART;
  float M = -INFINITY;
  for (int s = 0; s < S; ++s) M = fmaxf(M, pp[s * DEC_PART]);
  float l = 0.f, o = 0.f;
  for (int s = 0; s < S; ++s) {
    const float ms = pp[s * DEC_PART];
    if (ms == -INFINITY) continue;
    const float w = exp2f(ms - M);
    l = fmaf(w, pp[s * DEC_PART + 1], l);
    o = fmaf(w, pp[s * DEC_PART + 2 + d], o);
  }
  const int b = bh / NH, h = bh % NH;
  att[(int64_t)b * C + h * DEC_HD + d] = __float2bfloat16_rn(o / l);
}

// x0[b] = wte[tok[b]] + wpe[*pos_ptr] (one warp per row; ids outside [0, V) raise the
// device error word and read row 0).
__global__ void embed_decode_kernel(const int* __restrict__ tok, const float* __restrict__ wte,
                                    const float* __restrict__ wpe, const int* __restrict__ pos_ptr,
                                    float* __restrict__ x0, int B, int C, int V, int* err) {
  const int b = (blockIdx.x * blockDim.x + threadIdx.x) >> 5, lane = threadIdx.x & 31;
  if (b >= B) return;
  int id = tok[b];
  if (id < 0 || id >= V) {
    if (lane == 0) raise_device_error(err, DEV_TOKEN_RANGE);
    id = 0;
  }
  const float* a = wte + (int64_t)id * C;
  const float* p = wpe + (int64_t)(*pos_ptr) * C;
  float* o = x0 + (int64_t)b * C;
  for (int c = lane * 4; c < C; c += 128) {
    const float4 u = __ldg(reinterpret_cast<const float4*>(a + c));
    const float4 w = __ldg(reinterpret_cast<const float4*>(p + c));
    *reinterpret_cast<float4*>(o + c) = make_float4(u.x + w.x, u.y + w.y, u.z + w.z, u.w + w.w);
  }
}

// *p = v (v >= 0), or *p += 1 (v < 0): the cache position of a captured step.
__global__ void set_pos_kernel(int* p, int v) {
  if (threadIdx.x == 0 && blockIdx.x == 0) *p = v >= 0 ? v : *p + 1;
}

// Copy the keys and values of a prompt's forward pass into the cache: source row
// b*T0 + t of qkv (bf16 [B*T0][3C], columns C..3C) -> cache row t of sequence b.
__global__ void kv_fill_kernel(const bf16* __restrict__ qkv, int B, int T0, int C, bf16* __restrict__ cache,
                               int64_t cache_seq) {
  const int per_row = (2 * C) / 8;  // 16-byte vectors
  const int64_t total = (int64_t)B * T0 * per_row;
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < total; i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t r = i / per_row;
    const int v = (int)(i % per_row);
    const int b = (int)(r / T0), t = (int)(r % T0);
    const uint4 val = *reinterpret_cast<const uint4*>(qkv + r * 3 * C + C + v * 8);
    *reinterpret_cast<uint4*>(cache + b * cache_seq + (int64_t)t * 2 * C + v * 8) = val;
  }
}

}  // namespace g2
