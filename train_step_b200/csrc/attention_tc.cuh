// attention_tc.cuh -- causal flash attention on the 5th-generation tensor cores
// (tcgen05, accumulators in TMEM, tiles by TMA), head dim 64, bf16 operands.
//
// Same mathematics as attention.cuh ("AxonLM", Key Features: Flash Attention;
// "GPT From Scratch", Key decisions): per (batch, head) and per 128-query block,
// online softmax over 128-key blocks; lse = logsumexp of the scaled scores.
//
// Forward, one CTA per (query block, batch*head), 320 threads:
//   warp 0     TMA producer: Q once, then K_j and V_j into a 3-stage ring
//   warp 1     one thread issues tcgen05.mma:
//                S_j  = Q K_j^T  (M=128, N=128, K=64)  into TMEM S[j % 2]
//                PV_j = P_j V_j  (M=128, N=64,  K=128) into TMEM PV[j % 2]
//   warps 2-9  softmax: each query row is shared by two threads (TMEM lane, one
//              per half of the 128 key columns; the halves swap row maxima
//              through shared memory). P_j = 2^(S_j*scale*log2e - m_j) goes to
//              shared memory as bf16 (128-byte swizzled, K-major); row sums and
//              the running output O = O * 2^(m_{j-1} - m_j) + PV_j (each thread
//              keeps 32 of the 64 output columns) stay in registers.
// S, P and PV are double-buffered so the tensor cores compute S_{j+1} and PV_j
// while the softmax warps work on block j.
// Every mbarrier wait is bounded (device error word + early exit, no trap).
#pragma once
#include "attention.cuh"
#include "common.cuh"

namespace g2 {

constexpr int FA_BM = 128;  // queries per CTA
constexpr int FA_BN = 128;  // keys per block
constexpr int FA_THREADS = 320;
constexpr int FA_TILE = FA_BM * 64 * 2;  // 16 KB: 128 rows x 64 bf16
constexpr int FA_P = FA_BM * FA_BN * 2;  // 32 KB: P tile
constexpr int FA_KV_STAGES = 3;
// shared memory: Q | K0 V0 | K1 V1 | K2 V2 | P0 | P1 | barriers | exchange
constexpr int FA_OFF_Q = 0;
constexpr int FA_OFF_KV = FA_TILE;
constexpr int FA_OFF_P = FA_OFF_KV + 2 * FA_KV_STAGES * FA_TILE;
constexpr int FA_OFF_BAR = FA_OFF_P + 2 * FA_P;
constexpr int FA_OFF_RED = FA_OFF_BAR + 256;  // row-max / row-sum exchange, 3 x 2 x 128 floats
constexpr int FA_SMEM = FA_OFF_RED + 3 * 2 * 128 * 4 + 1024;
constexpr uint32_t FA_TMEM_COLS = 512;  // S0 0..127, S1 128..255, PV0 256..319, PV1 320..383

// P row r, key column c (0..127): 128-byte-swizzled K-major tile in two 64-key halves.
__device__ __forceinline__ uint32_t fa_p_off(int r, int chunk16 /*0..15*/) {
  const int half = chunk16 >> 3, c8 = chunk16 & 7;
  return (uint32_t)(half * (FA_BM * 128) + r * 128 + ((c8 ^ (r & 7)) << 4));
}

__global__ void __launch_bounds__(FA_THREADS, 1)
    attn_fwd_tc_kernel(const __grid_constant__ CUtensorMap tm_qkv, bf16* __restrict__ out, float* __restrict__ lse,
                       int T, int NH, float scale, int* err, unsigned long long timeout_ns) {
  extern __shared__ uint8_t fa_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(fa_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bar = reinterpret_cast<uint64_t*>(sm + FA_OFF_BAR);
  uint64_t* q_full = bar + 0;
  uint64_t* kv_full = bar + 1;   // [3]
  uint64_t* kv_empty = bar + 4;  // [3]
  uint64_t* s_full = bar + 7;    // [2]
  uint64_t* s_empty = bar + 9;   // [2]
  uint64_t* p_full = bar + 11;   // [2]
  uint64_t* pv_full = bar + 13;  // [2]
  uint64_t* drain = bar + 15;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bar + 16);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(bar + 17);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int qb = gridDim.x - 1 - blockIdx.x;  // longest rows first
  const int bh = blockIdx.y, b = bh / NH, h = bh % NH;
  const int C = NH * 64;
  const int nkb = qb + 1;
  const uint64_t lim = timeout_ns;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int i = 0; i < FA_KV_STAGES; ++i) {
      mbar_init(&kv_full[i], 1);
      mbar_init(&kv_empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s_full[i], 1);
      mbar_init(&s_empty[i], 8);
      mbar_init(&p_full[i], 8);
      mbar_init(&pv_full[i], 1);
    }
    mbar_init(drain, 1);  // for the abort path
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, FA_TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      // ---------------- TMA producer ----------------
      tma_prefetch_desc(&tm_qkv);
      bool ok = true;
      mbar_arrive_expect_tx(q_full, FA_TILE);
      tma_load_3d(sm + FA_OFF_Q, &tm_qkv, q_full, h * 64, qb * FA_BM, b);
      uint32_t issued = 0, par = 0;  // bit s: stage s has a load issued / parity of its last load
      for (int j = 0; j < nkb && ok; ++j) {
        const int st = j % FA_KV_STAGES;
        const uint32_t ph = (uint32_t)((j / FA_KV_STAGES) & 1);
        if (!mbar_wait_bounded(&kv_empty[st], ph ^ 1, abort_flag, lim)) {
          ok = false;
          break;
        }
        mbar_arrive_expect_tx(&kv_full[st], 2 * FA_TILE);
        uint8_t* kd = sm + FA_OFF_KV + st * 2 * FA_TILE;  // stage st: K then V
        tma_load_3d(kd, &tm_qkv, &kv_full[st], C + h * 64, j * FA_BN, b);
        tma_load_3d(kd + FA_TILE, &tm_qkv, &kv_full[st], 2 * C + h * 64, j * FA_BN, b);
        issued |= 1u << st;
        par = (par & ~(1u << st)) | (ph << st);
      }
      if (!ok) {
        raise_device_error(err, DEV_TIMEOUT);
        *abort_flag = 1;
        int never = 0;
        mbar_wait_bounded(q_full, 0, reinterpret_cast<volatile int*>(&never), lim);
        for (int s = 0; s < FA_KV_STAGES; ++s)
          if ((issued >> s) & 1u)
            mbar_wait_bounded(&kv_full[s], (par >> s) & 1u, reinterpret_cast<volatile int*>(&never), lim);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ---------------- MMA issuer ----------------
      constexpr uint32_t idesc_s = make_idesc_bf16(128, 128, false, false);
      constexpr uint32_t idesc_o = make_idesc_bf16(128, 64, false, true);
      const uint32_t q_addr = smem_u32(sm + FA_OFF_Q);
      bool ok = mbar_wait_bounded(q_full, 0, abort_flag, lim);
      bool any = false;
      for (int j = 0; j <= nkb && ok; ++j) {
        if (j < nkb) {  // S_j = Q K_j^T
          const int st = j & 1, ks = j % FA_KV_STAGES;
          if (!mbar_wait_bounded(&kv_full[ks], (j / FA_KV_STAGES) & 1, abort_flag, lim) ||
              !mbar_wait_bounded(&s_empty[st], ((j >> 1) & 1) ^ 1, abort_flag, lim)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t k_addr = smem_u32(sm + FA_OFF_KV + ks * 2 * FA_TILE);
#pragma unroll
          for (int k = 0; k < 4; ++k)
            umma_bf16(tmem + st * 128, make_sw128_desc(q_addr + k * 32, 16, 1024),
                      make_sw128_desc(k_addr + k * 32, 16, 1024), idesc_s, k > 0 ? 1u : 0u);
          umma_commit(&s_full[st]);
          any = true;
        }
        if (j >= 1) {  // PV_{j-1} = P_{j-1} V_{j-1}
          const int i = j - 1, st = i & 1, ks = i % FA_KV_STAGES;
          if (!mbar_wait_bounded(&p_full[st], (i >> 1) & 1, abort_flag, lim)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t p_addr = smem_u32(sm + FA_OFF_P + st * FA_P);
          const uint32_t v_addr = smem_u32(sm + FA_OFF_KV + ks * 2 * FA_TILE + FA_TILE);
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            umma_bf16(tmem + 256 + st * 64,
                      make_sw128_desc(p_addr + (kk >> 2) * (FA_BM * 128) + (kk & 3) * 32, 16, 1024),
                      make_sw128_desc(v_addr + kk * 2048, 8192, 1024), idesc_o, kk > 0 ? 1u : 0u);
          umma_commit(&pv_full[st]);
          umma_commit(&kv_empty[ks]);
        }
      }
      if (!ok) {
        raise_device_error(err, DEV_TIMEOUT);
        *abort_flag = 1;
        if (any) {
          int never = 0;
          umma_commit(drain);
          mbar_wait_bounded(drain, 0, reinterpret_cast<volatile int*>(&never), lim);
        }
      }
    }
  } else {
    // ---------------- softmax warps ----------------
    // warps 2-5 take S columns 0-63, warps 6-9 columns 64-127 of the same rows; the
    // two halves exchange their row maxima through shared memory once per block
    const int hf = (warp - 2) >> 2;       // column half
    const int q4 = warp & 3;              // TMEM lane quarter
    const int r = q4 * 32 + lane;         // row within the query block
    const int qrow = qb * FA_BM + r;      // query position
    const uint32_t lane_base = tmem + ((uint32_t)(q4 * 32) << 16);
    float* red = reinterpret_cast<float*>(sm + FA_OFF_RED);  // [3 buffers][2 halves][128 rows]
    const float sl2 = scale * LOG2E;
    float o[32];
#pragma unroll
    for (int i = 0; i < 32; ++i) o[i] = 0.f;
    float m_run = -INFINITY, l_run = 0.f, c_prev = 0.f, c_cur = 0.f;
    // A failed (timed-out) wait never makes a warp leave on its own: every softmax
    // warp reaches each named barrier, and the barrier's OR decides for all.
    bool fail = false;
    for (int j = 0; j <= nkb; ++j) {
      if (j < nkb) {
        const int st = j & 1;
        if (!fail && !mbar_wait_bounded(&s_full[st], (j >> 1) & 1, abort_flag, lim)) fail = true;
        uint32_t sv[64];
        if (!fail) {
          tc_fence_after();
          tmem_ld_32x32b_x32(lane_base + st * 128 + hf * 64, *reinterpret_cast<uint32_t(*)[32]>(&sv[0]));
          tmem_ld_32x32b_x32(lane_base + st * 128 + hf * 64 + 32, *reinterpret_cast<uint32_t(*)[32]>(&sv[32]));
          tmem_ld_wait();
        } else {
#pragma unroll
          for (int e = 0; e < 64; ++e) sv[e] = 0u;
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&s_empty[st]);  // S[st] is free for S_{j+2}
        const bool diag = (j == qb);
        const int kbase = j * FA_BN + hf * 64;
        if (diag) {  // causal mask: keys after the query get -inf (only on the diagonal block)
#pragma unroll
          for (int e = 0; e < 64; ++e)
            if (kbase + e > qrow) sv[e] = __float_as_uint(-INFINITY);
        }
        float mx;
        {
          float m8[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) m8[e] = __uint_as_float(sv[e]);
#pragma unroll
          for (int e = 8; e < 64; ++e) m8[e & 7] = fmaxf(m8[e & 7], __uint_as_float(sv[e]));
          mx = fmaxf(fmaxf(fmaxf(m8[0], m8[1]), fmaxf(m8[2], m8[3])), fmaxf(fmaxf(m8[4], m8[5]), fmaxf(m8[6], m8[7])));
        }
        red[(st * 2 + hf) * FA_BM + r] = mx;
        if (named_barrier_or(1, 256, fail || *abort_flag)) {
          fail = true;
          break;
        }
        mx = fmaxf(mx, red[(st * 2 + (hf ^ 1)) * FA_BM + r]);
        const float m_new = fmaxf(m_run, mx * sl2);
        const float corr = (m_run == -INFINITY) ? 0.f : ex2_fast(m_run - m_new);
        float rs8[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
        uint8_t* pbuf = sm + FA_OFF_P + st * FA_P;
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          float p[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            p[e] = ex2_fast(fmaf(__uint_as_float(sv[8 * k + e]), sl2, -m_new));  // 2^-inf = 0 for masked keys
            rs8[e] += p[e];
          }
          uint4 w = make_uint4(pack_bf16x2(p[0], p[1]), pack_bf16x2(p[2], p[3]), pack_bf16x2(p[4], p[5]),
                               pack_bf16x2(p[6], p[7]));
          *reinterpret_cast<uint4*>(pbuf + fa_p_off(r, hf * 8 + k)) = w;
        }
        const float rs = ((rs8[0] + rs8[1]) + (rs8[2] + rs8[3])) + ((rs8[4] + rs8[5]) + (rs8[6] + rs8[7]));
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&p_full[st]);
        l_run = l_run * corr + rs;
        m_run = m_new;
        c_cur = corr;
      }
      // fold PV_{j-1} into O with the correction of block j-1
      if (j >= 1) {
        const int i = j - 1, sp = i & 1;
        if (!fail && !mbar_wait_bounded(&pv_full[sp], (i >> 1) & 1, abort_flag, lim)) fail = true;
        if (!fail) {
          tc_fence_after();
          uint32_t v[32];
          tmem_ld_32x32b_x32(lane_base + 256 + sp * 64 + hf * 32, v);
          tmem_ld_wait();
#pragma unroll
          for (int e = 0; e < 32; ++e) o[e] = fmaf(o[e], c_prev, __uint_as_float(v[e]));
        }
      }
      c_prev = c_cur;
    }
    // combine the two halves' row sums; the barrier also decides success for all
    red[(4 + hf) * FA_BM + r] = l_run;
    if (named_barrier_or(1, 256, fail || *abort_flag)) {
      if (lane == 0) {
        raise_device_error(err, DEV_TIMEOUT);
        *abort_flag = 1;
      }
    } else {
      const float l = l_run + red[(4 + (hf ^ 1)) * FA_BM + r];
      if (qrow < T) {
        const float inv = 1.0f / l;
        bf16* orow = out + ((long long)b * T + qrow) * C + h * 64 + hf * 32;
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          uint4 w = make_uint4(pack_bf16x2(o[8 * k] * inv, o[8 * k + 1] * inv),
                               pack_bf16x2(o[8 * k + 2] * inv, o[8 * k + 3] * inv),
                               pack_bf16x2(o[8 * k + 4] * inv, o[8 * k + 5] * inv),
                               pack_bf16x2(o[8 * k + 6] * inv, o[8 * k + 7] * inv));
          *reinterpret_cast<uint4*>(orow + 8 * k) = w;
        }
        if (hf == 0) lse[((long long)b * NH + h) * T + qrow] = (m_run + __log2f(l)) * LN2;
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, FA_TMEM_COLS);
  }
}

// ---------------------------------------------------------------------------
// Backward on tcgen05. Two deterministic kernels (no atomics):
//   dK/dV: one CTA per (128-key block, batch*head), looping over query blocks i:
//     S^T = K Q_i^T, dP^T = V dO_i^T                  (M=128, N=128, K=64)
//     P^T = 2^(S^T*scale*log2e - lse_q*log2e), dS^T = P^T (dP^T - D_q)   (softmax warps)
//     dV += P^T dO_i, dK += dS^T Q_i                    (M=128, N=64, K=128)
//   dQ: one CTA per (128-query block, batch*head), looping over key blocks j:
//     S = Q K_j^T, dP = dO V_j^T; P, dS as above; dQ += dS K_j
// Warp roles as in the forward (producer, MMA issuer, 8 element-wise warps that
// split the 128 columns in halves). D_q = rowsum(dO * O) comes precomputed.
// ---------------------------------------------------------------------------
constexpr int FB_STAGES = 3;
constexpr int FB_THREADS = 320;
// dK/dV kernel shared memory: K | V | stages (Q_i, dO_i) | P^T | dS^T | L/D [2][2][128] | barriers
constexpr int FBK_OFF_K = 0;
constexpr int FBK_OFF_V = FA_TILE;
constexpr int FBK_OFF_ST = 2 * FA_TILE;
constexpr int FBK_OFF_P = FBK_OFF_ST + FB_STAGES * 2 * FA_TILE;
constexpr int FBK_OFF_DS = FBK_OFF_P + FA_P;
constexpr int FBK_OFF_LD = FBK_OFF_DS + FA_P;
constexpr int FBK_OFF_BAR = FBK_OFF_LD + 2 * 2 * 128 * 4;
constexpr int FBK_SMEM = FBK_OFF_BAR + 256 + 1024;
// dQ kernel shared memory: Q | dO | stages (K_j, V_j) | dS | barriers
constexpr int FBQ_OFF_Q = 0;
constexpr int FBQ_OFF_DO = FA_TILE;
constexpr int FBQ_OFF_ST = 2 * FA_TILE;
constexpr int FBQ_OFF_DS = FBQ_OFF_ST + FB_STAGES * 2 * FA_TILE;
constexpr int FBQ_OFF_BAR = FBQ_OFF_DS + FA_P;
constexpr int FBQ_SMEM = FBQ_OFF_BAR + 256 + 1024;
// TMEM columns: S (or S^T) 0..127, dP (or dP^T) 128..255, accumulators from 256
constexpr uint32_t FB_TMEM_COLS = 512;

// 8 consecutive columns (chunk k of half hf) of row r of an element-wise tile.
__device__ __forceinline__ void fb_store_chunk(uint8_t* buf, int r, int hf, int k, const float (&v)[8]) {
  uint4 w = make_uint4(pack_bf16x2(v[0], v[1]), pack_bf16x2(v[2], v[3]), pack_bf16x2(v[4], v[5]),
                       pack_bf16x2(v[6], v[7]));
  *reinterpret_cast<uint4*>(buf + fa_p_off(r, hf * 8 + k)) = w;
}

__global__ void __launch_bounds__(FB_THREADS, 1)
    attn_bwd_dkdv_tc_kernel(const __grid_constant__ CUtensorMap tm_qkv, const __grid_constant__ CUtensorMap tm_do,
                            const float* __restrict__ lse, const float* __restrict__ Dg, bf16* __restrict__ dqkv, int T,
                            int NH, float scale, int* err, unsigned long long timeout_ns) {
  extern __shared__ uint8_t fb_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(fb_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bar = reinterpret_cast<uint64_t*>(sm + FBK_OFF_BAR);
  uint64_t* kv_full = bar + 0;
  uint64_t* st_full = bar + 1;   // [3]
  uint64_t* st_empty = bar + 4;  // [3]
  uint64_t* s_full = bar + 7;
  uint64_t* s_empty = bar + 8;
  uint64_t* p_full = bar + 9;
  uint64_t* p_free = bar + 10;
  uint64_t* acc_full = bar + 11;
  uint64_t* drain = bar + 12;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bar + 13);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(bar + 14);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int kb = blockIdx.x;
  const int bh = blockIdx.y, b = bh / NH, h = bh % NH;
  const int C = NH * 64;
  const int nqb = (T + FA_BM - 1) / FA_BM;
  const int n = nqb - kb;  // query blocks kb .. nqb-1
  const uint64_t lim = timeout_ns;

  if (threadIdx.x == 0) {
    mbar_init(kv_full, 1);
    for (int i = 0; i < FB_STAGES; ++i) {
      mbar_init(&st_full[i], 1);
      mbar_init(&st_empty[i], 1);
    }
    mbar_init(s_full, 1);
    mbar_init(s_empty, 8);
    mbar_init(p_full, 8);
    mbar_init(p_free, 1);
    mbar_init(acc_full, 1);
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, FB_TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      tma_prefetch_desc(&tm_qkv);
      tma_prefetch_desc(&tm_do);
      mbar_arrive_expect_tx(kv_full, 2 * FA_TILE);
      tma_load_3d(sm + FBK_OFF_K, &tm_qkv, kv_full, C + h * 64, kb * FA_BN, b);
      tma_load_3d(sm + FBK_OFF_V, &tm_qkv, kv_full, 2 * C + h * 64, kb * FA_BN, b);
      bool ok = true;
      uint32_t issued = 0, par = 0;
      for (int t = 0; t < n; ++t) {
        const int qi = kb + t, st = t % FB_STAGES;
        const uint32_t ph = (uint32_t)((t / FB_STAGES) & 1);
        if (!mbar_wait_bounded(&st_empty[st], ph ^ 1, abort_flag, lim)) {
          ok = false;
          break;
        }
        uint8_t* d = sm + FBK_OFF_ST + st * 2 * FA_TILE;
        mbar_arrive_expect_tx(&st_full[st], 2 * FA_TILE);
        tma_load_3d(d, &tm_qkv, &st_full[st], h * 64, qi * FA_BM, b);
        tma_load_3d(d + FA_TILE, &tm_do, &st_full[st], h * 64, qi * FA_BM, b);
        issued |= 1u << st;
        par = (par & ~(1u << st)) | (ph << st);
      }
      if (!ok) {
        raise_device_error(err, DEV_TIMEOUT);
        *abort_flag = 1;
        int never = 0;
        mbar_wait_bounded(kv_full, 0, reinterpret_cast<volatile int*>(&never), lim);
        for (int s2 = 0; s2 < FB_STAGES; ++s2)
          if ((issued >> s2) & 1u)
            mbar_wait_bounded(&st_full[s2], (par >> s2) & 1u, reinterpret_cast<volatile int*>(&never), lim);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t idesc_s = make_idesc_bf16(128, 128, false, false);
      constexpr uint32_t idesc_o = make_idesc_bf16(128, 64, false, true);
      const uint32_t k_addr = smem_u32(sm + FBK_OFF_K), v_addr = smem_u32(sm + FBK_OFF_V);
      const uint32_t p_addr = smem_u32(sm + FBK_OFF_P), ds_addr = smem_u32(sm + FBK_OFF_DS);
      bool ok = mbar_wait_bounded(kv_full, 0, abort_flag, lim);
      bool any = false;
      for (int t = 0; t <= n && ok; ++t) {
        if (t < n) {  // S^T = K Q_t^T, dP^T = V dO_t^T
          const int st = t % FB_STAGES;
          if (!mbar_wait_bounded(&st_full[st], (t / FB_STAGES) & 1, abort_flag, lim) ||
              !mbar_wait_bounded(s_empty, (t & 1) ^ 1, abort_flag, lim)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t q_addr = smem_u32(sm + FBK_OFF_ST + st * 2 * FA_TILE), do_addr = q_addr + FA_TILE;
#pragma unroll
          for (int k = 0; k < 4; ++k)
            umma_bf16(tmem, make_sw128_desc(k_addr + k * 32, 16, 1024), make_sw128_desc(q_addr + k * 32, 16, 1024),
                      idesc_s, k > 0 ? 1u : 0u);
#pragma unroll
          for (int k = 0; k < 4; ++k)
            umma_bf16(tmem + 128, make_sw128_desc(v_addr + k * 32, 16, 1024),
                      make_sw128_desc(do_addr + k * 32, 16, 1024), idesc_s, k > 0 ? 1u : 0u);
          umma_commit(s_full);
          any = true;
        }
        if (t >= 1) {  // dV += P^T dO, dK += dS^T Q for the previous query block
          const int i = t - 1, st = i % FB_STAGES;
          if (!mbar_wait_bounded(p_full, i & 1, abort_flag, lim)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t q_addr = smem_u32(sm + FBK_OFF_ST + st * 2 * FA_TILE), do_addr = q_addr + FA_TILE;
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            umma_bf16(tmem + 256, make_sw128_desc(p_addr + (kk >> 2) * (FA_BM * 128) + (kk & 3) * 32, 16, 1024),
                      make_sw128_desc(do_addr + kk * 2048, 8192, 1024), idesc_o, (i > 0 || kk > 0) ? 1u : 0u);
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            umma_bf16(tmem + 320, make_sw128_desc(ds_addr + (kk >> 2) * (FA_BM * 128) + (kk & 3) * 32, 16, 1024),
                      make_sw128_desc(q_addr + kk * 2048, 8192, 1024), idesc_o, (i > 0 || kk > 0) ? 1u : 0u);
          umma_commit(p_free);
          umma_commit(&st_empty[st]);
        }
      }
      if (ok) umma_commit(acc_full);
      if (!ok) {
        raise_device_error(err, DEV_TIMEOUT);
        *abort_flag = 1;
        if (any) {
          int never = 0;
          umma_commit(drain);
          mbar_wait_bounded(drain, 0, reinterpret_cast<volatile int*>(&never), lim);
        }
      }
    }
  } else {
    // element-wise warps: thread = key row r, queries [hf*64, hf*64 + 64) of the block
    const int hf = (warp - 2) >> 2, q4 = warp & 3;
    const int r = q4 * 32 + lane;
    const int key = kb * FA_BN + r;
    const uint32_t lane_base = tmem + ((uint32_t)(q4 * 32) << 16);
    float* ldb = reinterpret_cast<float*>(sm + FBK_OFF_LD);  // [2][L or D][128]
    const float* lse_bh = lse + (long long)bh * T;
    const float* D_bh = Dg + (long long)bh * T;
    const float sl2 = scale * LOG2E;
    const int tid8 = threadIdx.x - 64;  // 0..255
    bool fail = false;
    for (int t = 0; t < n; ++t) {
      const int qi = kb + t, buf = t & 1;
      {  // stage this query block's lse (log2 units) and D in shared memory
        const int idx = tid8 & 127, which = tid8 >> 7;
        const int q = qi * FA_BM + idx;
        float v = 0.f;
        if (q < T) v = which == 0 ? lse_bh[q] * LOG2E : D_bh[q];
        ldb[(buf * 2 + which) * 128 + idx] = v;
      }
      if (!fail && !mbar_wait_bounded(s_full, t & 1, abort_flag, lim)) fail = true;
      uint32_t sv[64], dv[64];
      if (!fail) {
        tc_fence_after();
        tmem_ld_32x32b_x32(lane_base + hf * 64, *reinterpret_cast<uint32_t(*)[32]>(&sv[0]));
        tmem_ld_32x32b_x32(lane_base + hf * 64 + 32, *reinterpret_cast<uint32_t(*)[32]>(&sv[32]));
        tmem_ld_32x32b_x32(lane_base + 128 + hf * 64, *reinterpret_cast<uint32_t(*)[32]>(&dv[0]));
        tmem_ld_32x32b_x32(lane_base + 128 + hf * 64 + 32, *reinterpret_cast<uint32_t(*)[32]>(&dv[32]));
        tmem_ld_wait();
      } else {
#pragma unroll
        for (int e = 0; e < 64; ++e) sv[e] = dv[e] = 0u;
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(s_empty);
      if (named_barrier_or(1, 256, fail || *abort_flag)) {  // also publishes the L/D stage
        fail = true;
        break;
      }
      const float* Lq = ldb + (buf * 2 + 0) * 128 + hf * 64;
      const float* Dq = ldb + (buf * 2 + 1) * 128 + hf * 64;
      const bool diag = (t == 0);  // queries qi*128 + c with qi == kb
      if (!fail && !mbar_wait_bounded(p_free, (t & 1) ^ 1, abort_flag, lim)) fail = true;
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        float pv[8], dsv[8];
#pragma unroll
        for (int e8 = 0; e8 < 8; ++e8) {
          const int e = 8 * k + e8;
          float pe = ex2_fast(fmaf(__uint_as_float(sv[e]), sl2, -Lq[e]));
          if (diag && hf * 64 + e < r) pe = 0.f;  // query before key
          pv[e8] = pe;
          dsv[e8] = pe * (__uint_as_float(dv[e]) - Dq[e]);
        }
        fb_store_chunk(sm + FBK_OFF_P, r, hf, k, pv);
        fb_store_chunk(sm + FBK_OFF_DS, r, hf, k, dsv);
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(p_full);
    }
    if (!fail && !mbar_wait_bounded(acc_full, 0, abort_flag, lim)) fail = true;
    if (named_barrier_or(1, 256, fail || *abort_flag)) {
      if (lane == 0) {
        raise_device_error(err, DEV_TIMEOUT);
        *abort_flag = 1;
      }
    } else {
      tc_fence_after();
      uint32_t v[32], k[32];
      tmem_ld_32x32b_x32(lane_base + 256 + hf * 32, v);
      tmem_ld_32x32b_x32(lane_base + 320 + hf * 32, k);
      tmem_ld_wait();
      if (key < T) {
        bf16* dk = dqkv + ((long long)b * T + key) * 3 * C + C + h * 64 + hf * 32;
        bf16* dvp = dk + C;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int e = 8 * q;
          *reinterpret_cast<uint4*>(dvp + e) =
              make_uint4(pack_bf16x2(__uint_as_float(v[e]), __uint_as_float(v[e + 1])),
                         pack_bf16x2(__uint_as_float(v[e + 2]), __uint_as_float(v[e + 3])),
                         pack_bf16x2(__uint_as_float(v[e + 4]), __uint_as_float(v[e + 5])),
                         pack_bf16x2(__uint_as_float(v[e + 6]), __uint_as_float(v[e + 7])));
          *reinterpret_cast<uint4*>(dk + e) =
              make_uint4(pack_bf16x2(__uint_as_float(k[e]) * scale, __uint_as_float(k[e + 1]) * scale),
                         pack_bf16x2(__uint_as_float(k[e + 2]) * scale, __uint_as_float(k[e + 3]) * scale),
                         pack_bf16x2(__uint_as_float(k[e + 4]) * scale, __uint_as_float(k[e + 5]) * scale),
                         pack_bf16x2(__uint_as_float(k[e + 6]) * scale, __uint_as_float(k[e + 7]) * scale));
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, FB_TMEM_COLS);
  }
}

__global__ void __launch_bounds__(FB_THREADS, 1)
    attn_bwd_dq_tc_kernel(const __grid_constant__ CUtensorMap tm_qkv, const __grid_constant__ CUtensorMap tm_do,
                          const float* __restrict__ lse, const float* __restrict__ Dg, bf16* __restrict__ dqkv, int T,
                          int NH, float scale, int* err, unsigned long long timeout_ns) {
  extern __shared__ uint8_t fb_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(fb_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bar = reinterpret_cast<uint64_t*>(sm + FBQ_OFF_BAR);
  uint64_t* q_full = bar + 0;
  uint64_t* st_full = bar + 1;   // [3]
  uint64_t* st_empty = bar + 4;  // [3]
  uint64_t* s_full = bar + 7;
  uint64_t* s_empty = bar + 8;
  uint64_t* ds_full = bar + 9;
  uint64_t* ds_free = bar + 10;
  uint64_t* acc_full = bar + 11;
  uint64_t* drain = bar + 12;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bar + 13);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(bar + 14);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int qb = gridDim.x - 1 - blockIdx.x;  // longest rows first
  const int bh = blockIdx.y, b = bh / NH, h = bh % NH;
  const int C = NH * 64;
  const int nkb = qb + 1;
  const uint64_t lim = timeout_ns;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int i = 0; i < FB_STAGES; ++i) {
      mbar_init(&st_full[i], 1);
      mbar_init(&st_empty[i], 1);
    }
    mbar_init(s_full, 1);
    mbar_init(s_empty, 8);
    mbar_init(ds_full, 8);
    mbar_init(ds_free, 1);
    mbar_init(acc_full, 1);
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, FB_TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      tma_prefetch_desc(&tm_qkv);
      tma_prefetch_desc(&tm_do);
      mbar_arrive_expect_tx(q_full, 2 * FA_TILE);
      tma_load_3d(sm + FBQ_OFF_Q, &tm_qkv, q_full, h * 64, qb * FA_BM, b);
      tma_load_3d(sm + FBQ_OFF_DO, &tm_do, q_full, h * 64, qb * FA_BM, b);
      bool ok = true;
      uint32_t issued = 0, par = 0;
      for (int j = 0; j < nkb; ++j) {
        const int st = j % FB_STAGES;
        const uint32_t ph = (uint32_t)((j / FB_STAGES) & 1);
        if (!mbar_wait_bounded(&st_empty[st], ph ^ 1, abort_flag, lim)) {
          ok = false;
          break;
        }
        uint8_t* d = sm + FBQ_OFF_ST + st * 2 * FA_TILE;
        mbar_arrive_expect_tx(&st_full[st], 2 * FA_TILE);
        tma_load_3d(d, &tm_qkv, &st_full[st], C + h * 64, j * FA_BN, b);
        tma_load_3d(d + FA_TILE, &tm_qkv, &st_full[st], 2 * C + h * 64, j * FA_BN, b);
        issued |= 1u << st;
        par = (par & ~(1u << st)) | (ph << st);
      }
      if (!ok) {
        raise_device_error(err, DEV_TIMEOUT);
        *abort_flag = 1;
        int never = 0;
        mbar_wait_bounded(q_full, 0, reinterpret_cast<volatile int*>(&never), lim);
        for (int s2 = 0; s2 < FB_STAGES; ++s2)
          if ((issued >> s2) & 1u)
            mbar_wait_bounded(&st_full[s2], (par >> s2) & 1u, reinterpret_cast<volatile int*>(&never), lim);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t idesc_s = make_idesc_bf16(128, 128, false, false);
      constexpr uint32_t idesc_o = make_idesc_bf16(128, 64, false, true);
      const uint32_t q_addr = smem_u32(sm + FBQ_OFF_Q), do_addr = smem_u32(sm + FBQ_OFF_DO);
      const uint32_t ds_addr = smem_u32(sm + FBQ_OFF_DS);
      bool ok = mbar_wait_bounded(q_full, 0, abort_flag, lim);
      bool any = false;
      for (int j = 0; j <= nkb && ok; ++j) {
        if (j < nkb) {  // S = Q K_j^T, dP = dO V_j^T
          const int st = j % FB_STAGES;
          if (!mbar_wait_bounded(&st_full[st], (j / FB_STAGES) & 1, abort_flag, lim) ||
              !mbar_wait_bounded(s_empty, (j & 1) ^ 1, abort_flag, lim)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t k_addr = smem_u32(sm + FBQ_OFF_ST + st * 2 * FA_TILE), v_addr = k_addr + FA_TILE;
#pragma unroll
          for (int k = 0; k < 4; ++k)
            umma_bf16(tmem, make_sw128_desc(q_addr + k * 32, 16, 1024), make_sw128_desc(k_addr + k * 32, 16, 1024),
                      idesc_s, k > 0 ? 1u : 0u);
#pragma unroll
          for (int k = 0; k < 4; ++k)
            umma_bf16(tmem + 128, make_sw128_desc(do_addr + k * 32, 16, 1024),
                      make_sw128_desc(v_addr + k * 32, 16, 1024), idesc_s, k > 0 ? 1u : 0u);
          umma_commit(s_full);
          any = true;
        }
        if (j >= 1) {  // dQ += dS K for the previous key block
          const int i = j - 1, st = i % FB_STAGES;
          if (!mbar_wait_bounded(ds_full, i & 1, abort_flag, lim)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t k_addr = smem_u32(sm + FBQ_OFF_ST + st * 2 * FA_TILE);
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            umma_bf16(tmem + 256, make_sw128_desc(ds_addr + (kk >> 2) * (FA_BM * 128) + (kk & 3) * 32, 16, 1024),
                      make_sw128_desc(k_addr + kk * 2048, 8192, 1024), idesc_o, (i > 0 || kk > 0) ? 1u : 0u);
          umma_commit(ds_free);
          umma_commit(&st_empty[st]);
        }
      }
      if (ok) umma_commit(acc_full);
      if (!ok) {
        raise_device_error(err, DEV_TIMEOUT);
        *abort_flag = 1;
        if (any) {
          int never = 0;
          umma_commit(drain);
          mbar_wait_bounded(drain, 0, reinterpret_cast<volatile int*>(&never), lim);
        }
      }
    }
  } else {
    // element-wise warps: thread = query row r, keys [hf*64, hf*64 + 64) of the block
    const int hf = (warp - 2) >> 2, q4 = warp & 3;
    const int r = q4 * 32 + lane;
    const int qrow = qb * FA_BM + r;
    const uint32_t lane_base = tmem + ((uint32_t)(q4 * 32) << 16);
    const float sl2 = scale * LOG2E;
    const float L2 = qrow < T ? lse[(long long)bh * T + qrow] * LOG2E : 0.f;
    const float Dr = qrow < T ? Dg[(long long)bh * T + qrow] : 0.f;
    bool fail = false;
    for (int j = 0; j < nkb; ++j) {
      if (!fail && !mbar_wait_bounded(s_full, j & 1, abort_flag, lim)) fail = true;
      uint32_t sv[64], dv[64];
      if (!fail) {
        tc_fence_after();
        tmem_ld_32x32b_x32(lane_base + hf * 64, *reinterpret_cast<uint32_t(*)[32]>(&sv[0]));
        tmem_ld_32x32b_x32(lane_base + hf * 64 + 32, *reinterpret_cast<uint32_t(*)[32]>(&sv[32]));
        tmem_ld_32x32b_x32(lane_base + 128 + hf * 64, *reinterpret_cast<uint32_t(*)[32]>(&dv[0]));
        tmem_ld_32x32b_x32(lane_base + 128 + hf * 64 + 32, *reinterpret_cast<uint32_t(*)[32]>(&dv[32]));
        tmem_ld_wait();
      } else {
#pragma unroll
        for (int e = 0; e < 64; ++e) sv[e] = dv[e] = 0u;
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(s_empty);
      const bool diag = (j == qb);
      const int kbase = j * FA_BN + hf * 64;
      if (!fail && !mbar_wait_bounded(ds_free, (j & 1) ^ 1, abort_flag, lim)) fail = true;
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        float dsv[8];
#pragma unroll
        for (int e8 = 0; e8 < 8; ++e8) {
          const int e = 8 * k + e8;
          float pe = ex2_fast(fmaf(__uint_as_float(sv[e]), sl2, -L2));
          if (diag && kbase + e > qrow) pe = 0.f;
          dsv[e8] = pe * (__uint_as_float(dv[e]) - Dr);
        }
        fb_store_chunk(sm + FBQ_OFF_DS, r, hf, k, dsv);
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(ds_full);
    }
    if (!fail && !mbar_wait_bounded(acc_full, 0, abort_flag, lim)) fail = true;
    if (named_barrier_or(1, 256, fail || *abort_flag)) {
      if (lane == 0) {
        raise_device_error(err, DEV_TIMEOUT);
        *abort_flag = 1;
      }
    } else {
      tc_fence_after();
      uint32_t v[32];
      tmem_ld_32x32b_x32(lane_base + 256 + hf * 32, v);
      tmem_ld_wait();
      if (qrow < T) {
        bf16* dq = dqkv + ((long long)b * T + qrow) * 3 * C + h * 64 + hf * 32;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int e = 8 * q;
          *reinterpret_cast<uint4*>(dq + e) =
              make_uint4(pack_bf16x2(__uint_as_float(v[e]) * scale, __uint_as_float(v[e + 1]) * scale),
                         pack_bf16x2(__uint_as_float(v[e + 2]) * scale, __uint_as_float(v[e + 3]) * scale),
                         pack_bf16x2(__uint_as_float(v[e + 4]) * scale, __uint_as_float(v[e + 5]) * scale),
                         pack_bf16x2(__uint_as_float(v[e + 6]) * scale, __uint_as_float(v[e + 7]) * scale));
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, FB_TMEM_COLS);
  }
}

}  // namespace g2
