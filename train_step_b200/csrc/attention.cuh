// attention.cuh -- causal multi-head self-attention, forward and backward, that
// never materialises the T x T score matrix ("AxonLM", Key Features: Flash
// Attention; "GPT From Scratch", Key decisions: written-out masked softmax and the
// fused path must agree). Softmax is taken online over key blocks; the forward
// saves lse = logsumexp of each query's scaled scores for the backward.
//
// Layout: qkv [B*T, 3C] (q | k | v column blocks; head h uses columns
// [h*hd, (h+1)*hd) of each), out [B*T, C], lse [B, NH, T] fp32.
//
// bf16 path (hd = 64): tensor-core tiles of 64 queries x 64 keys, 4 warps of 16
// rows, mma.sync m16n8k16 with fp32 accumulation, K/V tiles double-buffered by
// cp.async into XOR-swizzled shared memory.
// Backward is deterministic: one kernel per key block accumulates dK, dV over the
// query blocks; a second kernel per query block accumulates dQ over the key
// blocks (scores are recomputed; no atomics).
// fp32 path: one warp per query (or key) row, exact expf; for the parity mode.
#pragma once
#include "common.cuh"

namespace g2 {

constexpr float LOG2E = 1.4426950408889634f;
constexpr float LN2 = 0.6931471805599453f;

__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void cp_async16(uint32_t smem_addr, const void* gptr, bool valid) {
  const int sz = valid ? 16 : 0;  // zero-fill rows past the end of the sequence
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_addr), "l"(gptr), "r"(sz) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// A 64 x 64 bf16 tile: row r, 16-byte chunk c lives at r*128 + ((c ^ (r & 7)) * 16).
__device__ __forceinline__ uint32_t sw_off(int r, int c) { return (uint32_t)(r * 128 + ((c ^ (r & 7)) << 4)); }

// Load rows [row0, row0+64) of a head's 64 columns (row stride ld elements).
__device__ __forceinline__ void load_tile64(uint32_t sbase, const bf16* gbase, long long ld, int row0, int T,
                                            int tid) {
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int idx = tid + i * 128;  // 512 chunks of 16 bytes
    const int r = idx >> 3, c = idx & 7;
    const int gr = row0 + r;
    const bool ok = gr < T;
    const bf16* src = gbase + (long long)(ok ? gr : 0) * ld + c * 8;
    cp_async16(sbase + sw_off(r, c), src, ok);
  }
}

// A fragments (16 rows x 64 cols) of rows [r0, r0+16) from a swizzled tile.
__device__ __forceinline__ void load_afrag_rows(uint32_t sbase, int r0, int lane, uint32_t (&f)[4][4]) {
#pragma unroll
  for (int ks = 0; ks < 4; ++ks) {
    const int r = r0 + (lane & 15);
    const int c = ks * 2 + (lane >> 4);
    ldsm_x4(sbase + sw_off(r, c), f[ks][0], f[ks][1], f[ks][2], f[ks][3]);
  }
}

// acc[8][4] (16 x 64) += A(16 x 64, registers) * Tile^T where the tile holds the
// 64 "n" rows (keys or queries) with the contraction along its columns.
__device__ __forceinline__ void mma_rows_x_tileT(float (&acc)[8][4], const uint32_t (&a)[4][4], uint32_t sbase,
                                                 int lane) {
#pragma unroll
  for (int ks = 0; ks < 4; ++ks) {
#pragma unroll
    for (int np = 0; np < 4; ++np) {
      const int r = np * 16 + ((lane >> 4) << 3) + (lane & 7);
      const int c = ks * 2 + ((lane >> 3) & 1);
      uint32_t b0, b1, b2, b3;
      ldsm_x4(sbase + sw_off(r, c), b0, b1, b2, b3);
      mma_bf16_16816(acc[2 * np], a[ks], b0, b1);
      mma_bf16_16816(acc[2 * np + 1], a[ks], b2, b3);
    }
  }
}

// acc[8][4] (16 x 64 dims) += P(16 x 64, fp32 accumulators as bf16) * Tile where
// the tile's rows are the contraction index and its columns the output dims.
__device__ __forceinline__ void mma_p_x_tile(float (&acc)[8][4], const float (&p)[8][4], uint32_t sbase, int lane) {
#pragma unroll
  for (int kk = 0; kk < 4; ++kk) {
    uint32_t a[4];
    a[0] = pack_bf16x2(p[2 * kk][0], p[2 * kk][1]);
    a[1] = pack_bf16x2(p[2 * kk][2], p[2 * kk][3]);
    a[2] = pack_bf16x2(p[2 * kk + 1][0], p[2 * kk + 1][1]);
    a[3] = pack_bf16x2(p[2 * kk + 1][2], p[2 * kk + 1][3]);
#pragma unroll
    for (int np = 0; np < 4; ++np) {
      const int r = kk * 16 + (((lane >> 3) & 1) << 3) + (lane & 7);
      const int c = np * 2 + (lane >> 4);
      uint32_t b0, b1, b2, b3;
      ldsm_x4_t(sbase + sw_off(r, c), b0, b1, b2, b3);
      mma_bf16_16816(acc[2 * np], a, b0, b1);
      mma_bf16_16816(acc[2 * np + 1], a, b2, b3);
    }
  }
}

// ----------------------------------------------------------------------------
// forward
// ----------------------------------------------------------------------------
__global__ void __launch_bounds__(128) attn_fwd_bf16_kernel(const bf16* __restrict__ qkv, bf16* __restrict__ out,
                                                            float* __restrict__ lse, int T, int NH, float scale) {
  __shared__ __align__(128) bf16 sQ[64 * 64];
  __shared__ __align__(128) bf16 sK[2][64 * 64];
  __shared__ __align__(128) bf16 sV[2][64 * 64];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int qb = gridDim.x - 1 - blockIdx.x;  // longest rows first
  const int bh = blockIdx.y, b = bh / NH, h = bh % NH;
  const int C = NH * 64;
  const long long ld = 3LL * C;
  const bf16* qg = qkv + (long long)b * T * ld + h * 64;
  const bf16* kg = qg + C;
  const bf16* vg = qg + 2 * C;
  const uint32_t sq = smem_u32(sQ), sk0 = smem_u32(sK[0]), sv0 = smem_u32(sV[0]);
  const uint32_t KV_STRIDE = 64 * 64 * 2;

  load_tile64(sq, qg, ld, qb * 64, T, tid);
  load_tile64(sk0, kg, ld, 0, T, tid);
  load_tile64(sv0, vg, ld, 0, T, tid);
  cp_async_commit();

  const float sl2 = scale * LOG2E;
  float o[8][4];
#pragma unroll
  for (int i = 0; i < 8; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;
  float mrow[2] = {-INFINITY, -INFINITY}, lrow[2] = {0.f, 0.f};
  uint32_t qf[4][4];
  const int g = lane >> 2, t4 = lane & 3;
  const int qrow0 = qb * 64 + warp * 16 + g;  // this thread's rows: qrow0, qrow0 + 8

  const int nkb = qb + 1;
  for (int j = 0; j < nkb; ++j) {
    const int st = j & 1;
    if (j + 1 < nkb) {
      load_tile64(sk0 + (st ^ 1) * KV_STRIDE, kg, ld, (j + 1) * 64, T, tid);
      load_tile64(sv0 + (st ^ 1) * KV_STRIDE, vg, ld, (j + 1) * 64, T, tid);
      cp_async_commit();
      cp_async_wait<1>();
    } else {
      cp_async_wait<0>();
    }
    __syncthreads();
    if (j == 0) load_afrag_rows(sq, warp * 16, lane, qf);
    float s[8][4];
#pragma unroll
    for (int i = 0; i < 8; ++i) s[i][0] = s[i][1] = s[i][2] = s[i][3] = 0.f;
    mma_rows_x_tileT(s, qf, sk0 + st * KV_STRIDE, lane);
    // scale into the log2 domain, causal mask on the diagonal block
    float mx[2] = {-INFINITY, -INFINITY};
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int key = j * 64 + nt * 8 + 2 * t4 + (e & 1);
        const int qr = qrow0 + ((e >> 1) << 3);
        float v = s[nt][e] * sl2;
        if (j == qb && key > qr) v = -INFINITY;
        s[nt][e] = v;
        mx[e >> 1] = fmaxf(mx[e >> 1], v);
      }
    }
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      mx[r] = fmaxf(mx[r], __shfl_xor_sync(0xffffffffu, mx[r], 1));
      mx[r] = fmaxf(mx[r], __shfl_xor_sync(0xffffffffu, mx[r], 2));
    }
    float mnew[2], corr[2], rsum[2] = {0.f, 0.f};
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      mnew[r] = fmaxf(mrow[r], mx[r]);
      corr[r] = exp2f(mrow[r] - mnew[r]);
      mrow[r] = mnew[r];
    }
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float pv = exp2f(s[nt][e] - mnew[e >> 1]);
        s[nt][e] = pv;
        rsum[e >> 1] += pv;
      }
      o[nt][0] *= corr[0];
      o[nt][1] *= corr[0];
      o[nt][2] *= corr[1];
      o[nt][3] *= corr[1];
    }
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      rsum[r] += __shfl_xor_sync(0xffffffffu, rsum[r], 1);
      rsum[r] += __shfl_xor_sync(0xffffffffu, rsum[r], 2);
      lrow[r] = lrow[r] * corr[r] + rsum[r];
    }
    mma_p_x_tile(o, s, sv0 + st * KV_STRIDE, lane);
    __syncthreads();
  }
  // write O and lse
#pragma unroll
  for (int r = 0; r < 2; ++r) {
    const int qr = qrow0 + r * 8;
    if (qr >= T) continue;
    const float inv = 1.0f / lrow[r];
    bf16* orow = out + ((long long)b * T + qr) * C + h * 64;
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) {
      *reinterpret_cast<uint32_t*>(orow + nt * 8 + 2 * t4) = pack_bf16x2(o[nt][2 * r] * inv, o[nt][2 * r + 1] * inv);
    }
    if (t4 == 0) lse[((long long)b * NH + h) * T + qr] = (mrow[r] + __log2f(lrow[r])) * LN2;
  }
}

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

// bf16, hd = 64: one thread per (row, head), 128-byte vector loads of O and dO.
__global__ void attn_bwd_dot64_bf16_kernel(const bf16* __restrict__ out, const bf16* __restrict__ dout,
                                           float* __restrict__ D, int Bsz, int Tn, int NH) {
  const long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x;
  if (i >= (long long)Bsz * Tn * NH) return;
  const int h = (int)(i % NH);
  const long long row = i / NH;
  const long long off = row * NH * 64 + h * 64;
  const uint4* o = reinterpret_cast<const uint4*>(out + off);
  const uint4* d = reinterpret_cast<const uint4*>(dout + off);
  float s = 0.f;
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    const uint4 a = o[k], b = d[k];
    const uint32_t wa[4] = {a.x, a.y, a.z, a.w}, wb[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const float2 fa = unpack_bf16x2(wa[q]), fb = unpack_bf16x2(wb[q]);
      s += fa.x * fb.x + fa.y * fb.y;
    }
  }
  const int b = (int)(row / Tn), t = (int)(row % Tn);
  D[((long long)b * NH + h) * Tn + t] = s;
}

// dK, dV for one block of 64 keys; loops over query blocks qb >= kb.
__global__ void __launch_bounds__(128) attn_bwd_dkdv_bf16_kernel(const bf16* __restrict__ qkv,
                                                                 const bf16* __restrict__ dout,
                                                                 const float* __restrict__ lse,
                                                                 const float* __restrict__ Dg,
                                                                 bf16* __restrict__ dqkv, int T, int NH, float scale) {
  __shared__ __align__(128) bf16 sQ[2][64 * 64];
  __shared__ __align__(128) bf16 sdO[2][64 * 64];
  __shared__ __align__(128) bf16 sKV[64 * 64];
  __shared__ float sL[2][64], sD[2][64];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int kb = blockIdx.x;
  const int bh = blockIdx.y, b = bh / NH, h = bh % NH;
  const int C = NH * 64;
  const long long ld = 3LL * C;
  const bf16* qg = qkv + (long long)b * T * ld + h * 64;
  const bf16* kg = qg + C;
  const bf16* vg = qg + 2 * C;
  const bf16* dog = dout + (long long)b * T * C + h * 64;
  const float* lseg = lse + ((long long)b * NH + h) * T;
  const float* Dgh = Dg + ((long long)b * NH + h) * T;
  const uint32_t sq0 = smem_u32(sQ[0]), sdo0 = smem_u32(sdO[0]), skv = smem_u32(sKV);
  const uint32_t STR = 64 * 64 * 2;
  const int nqb = (T + 63) / 64;
  const int g = lane >> 2, t4 = lane & 3;

  // K rows of this warp as A fragments, then V rows
  uint32_t kf[4][4], vf[4][4];
  load_tile64(skv, kg, ld, kb * 64, T, tid);
  cp_async_commit();
  cp_async_wait<0>();
  __syncthreads();
  load_afrag_rows(skv, warp * 16, lane, kf);
  __syncthreads();
  load_tile64(skv, vg, ld, kb * 64, T, tid);
  cp_async_commit();
  cp_async_wait<0>();
  __syncthreads();
  load_afrag_rows(skv, warp * 16, lane, vf);

  auto load_q = [&](int qb, int st) {
    load_tile64(sq0 + st * STR, qg, ld, qb * 64, T, tid);
    load_tile64(sdo0 + st * STR, dog, C, qb * 64, T, tid);
    if (tid < 64) {
      const int q = qb * 64 + tid;
      sL[st][tid] = q < T ? lseg[q] * LOG2E : 0.f;
      sD[st][tid] = q < T ? Dgh[q] : 0.f;
    }
  };
  load_q(kb, 0);
  cp_async_commit();

  float dk[8][4], dv[8][4];
#pragma unroll
  for (int i = 0; i < 8; ++i)
#pragma unroll
    for (int e = 0; e < 4; ++e) dk[i][e] = dv[i][e] = 0.f;
  const float sl2 = scale * LOG2E;
  const int key0 = kb * 64 + warp * 16 + g;  // this thread's keys: key0, key0 + 8

  for (int qb = kb; qb < nqb; ++qb) {
    const int st = (qb - kb) & 1;
    __syncthreads();  // previous iteration done with stage st^1
    if (qb + 1 < nqb) {
      load_q(qb + 1, st ^ 1);
      cp_async_commit();
      cp_async_wait<1>();
    } else {
      cp_async_wait<0>();
    }
    __syncthreads();
    const uint32_t sq = sq0 + st * STR, sdo = sdo0 + st * STR;
    // S^T (16 keys x 64 queries) and dP^T
    float s[8][4], dp[8][4];
#pragma unroll
    for (int i = 0; i < 8; ++i)
#pragma unroll
      for (int e = 0; e < 4; ++e) s[i][e] = dp[i][e] = 0.f;
    mma_rows_x_tileT(s, kf, sq, lane);
    mma_rows_x_tileT(dp, vf, sdo, lane);
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int ql = nt * 8 + 2 * t4 + (e & 1);
        const int q = qb * 64 + ql;
        const int key = key0 + ((e >> 1) << 3);
        float pv = exp2f(s[nt][e] * sl2 - sL[st][ql]);
        if (q < key || q >= T) pv = 0.f;
        s[nt][e] = pv;                            // P^T
        dp[nt][e] = pv * (dp[nt][e] - sD[st][ql]);  // dS^T
      }
    }
    mma_p_x_tile(dv, s, sdo, lane);
    mma_p_x_tile(dk, dp, sq, lane);
  }
  // write dK (scaled) and dV
#pragma unroll
  for (int r = 0; r < 2; ++r) {
    const int key = key0 + r * 8;
    if (key >= T) continue;
    bf16* dkr = dqkv + ((long long)b * T + key) * ld + C + h * 64;
    bf16* dvr = dkr + C;
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) {
      *reinterpret_cast<uint32_t*>(dkr + nt * 8 + 2 * t4) = pack_bf16x2(dk[nt][2 * r] * scale, dk[nt][2 * r + 1] * scale);
      *reinterpret_cast<uint32_t*>(dvr + nt * 8 + 2 * t4) = pack_bf16x2(dv[nt][2 * r], dv[nt][2 * r + 1]);
    }
  }
}

// dQ for one block of 64 queries; loops over key blocks kb <= qb.
__global__ void __launch_bounds__(128) attn_bwd_dq_bf16_kernel(const bf16* __restrict__ qkv,
                                                               const bf16* __restrict__ dout,
                                                               const float* __restrict__ lse,
                                                               const float* __restrict__ Dg, bf16* __restrict__ dqkv,
                                                               int T, int NH, float scale) {
  __shared__ __align__(128) bf16 sK[2][64 * 64];
  __shared__ __align__(128) bf16 sV[2][64 * 64];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int qb = gridDim.x - 1 - blockIdx.x;
  const int bh = blockIdx.y, b = bh / NH, h = bh % NH;
  const int C = NH * 64;
  const long long ld = 3LL * C;
  const bf16* qg = qkv + (long long)b * T * ld + h * 64;
  const bf16* kg = qg + C;
  const bf16* vg = qg + 2 * C;
  const bf16* dog = dout + (long long)b * T * C + h * 64;
  const float* lseg = lse + ((long long)b * NH + h) * T;
  const float* Dgh = Dg + ((long long)b * NH + h) * T;
  const uint32_t sk0 = smem_u32(sK[0]), sv0 = smem_u32(sV[0]);
  const uint32_t STR = 64 * 64 * 2;
  const int g = lane >> 2, t4 = lane & 3;
  const int q0 = qb * 64 + warp * 16 + g;

  // Q and dO rows of this warp as A fragments (staged through the K/V buffers)
  uint32_t qf[4][4], dof[4][4];
  load_tile64(sk0, qg, ld, qb * 64, T, tid);
  load_tile64(sv0, dog, C, qb * 64, T, tid);
  cp_async_commit();
  cp_async_wait<0>();
  __syncthreads();
  load_afrag_rows(sk0, warp * 16, lane, qf);
  load_afrag_rows(sv0, warp * 16, lane, dof);
  float lrow[2], drow[2];
#pragma unroll
  for (int r = 0; r < 2; ++r) {
    const int q = q0 + r * 8;
    lrow[r] = q < T ? lseg[q] * LOG2E : 0.f;
    drow[r] = q < T ? Dgh[q] : 0.f;
  }
  __syncthreads();
  load_tile64(sk0, kg, ld, 0, T, tid);
  load_tile64(sv0, vg, ld, 0, T, tid);
  cp_async_commit();

  float dq[8][4];
#pragma unroll
  for (int i = 0; i < 8; ++i) dq[i][0] = dq[i][1] = dq[i][2] = dq[i][3] = 0.f;
  const float sl2 = scale * LOG2E;
  for (int kb = 0; kb <= qb; ++kb) {
    const int st = kb & 1;
    if (kb + 1 <= qb) {
      load_tile64(sk0 + (st ^ 1) * STR, kg, ld, (kb + 1) * 64, T, tid);
      load_tile64(sv0 + (st ^ 1) * STR, vg, ld, (kb + 1) * 64, T, tid);
      cp_async_commit();
      cp_async_wait<1>();
    } else {
      cp_async_wait<0>();
    }
    __syncthreads();
    float s[8][4], dp[8][4];
#pragma unroll
    for (int i = 0; i < 8; ++i)
#pragma unroll
      for (int e = 0; e < 4; ++e) s[i][e] = dp[i][e] = 0.f;
    mma_rows_x_tileT(s, qf, sk0 + st * STR, lane);
    mma_rows_x_tileT(dp, dof, sv0 + st * STR, lane);
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int key = kb * 64 + nt * 8 + 2 * t4 + (e & 1);
        const int r = e >> 1;
        const int q = q0 + r * 8;
        float pv = exp2f(s[nt][e] * sl2 - lrow[r]);
        if (key > q) pv = 0.f;
        dp[nt][e] = pv * (dp[nt][e] - drow[r]);  // dS
      }
    }
    mma_p_x_tile(dq, dp, sk0 + st * STR, lane);
    __syncthreads();
  }
#pragma unroll
  for (int r = 0; r < 2; ++r) {
    const int q = q0 + r * 8;
    if (q >= T) continue;
    bf16* dqr = dqkv + ((long long)b * T + q) * ld + h * 64;
#pragma unroll
    for (int nt = 0; nt < 8; ++nt)
      *reinterpret_cast<uint32_t*>(dqr + nt * 8 + 2 * t4) = pack_bf16x2(dq[nt][2 * r] * scale, dq[nt][2 * r + 1] * scale);
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
