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
// Backward on tcgen05. Two deterministic kernels (no atomics). Both are
// persistent (one CTA per SM looping over work items, so an item's loads overlap
// the previous item's tail) and work in 64-wide units:
//
//   dK/dV: item = (128-key block kb, batch*head); units = 64-query halves of the
//     query blocks kb .. nqb-1, in key-row orientation:
//       S^T = K Q_u^T, dP^T = V dO_u^T                 (M=128 keys, N=64 queries, K=64)
//       P^T = 2^(S^T*scale*log2e - lse*log2e), dS^T = P^T (dP^T - D)   (element-wise)
//       dV += P^T dO_u, dK += dS^T Q_u                 (M=128 keys, N=64, K=64 queries)
//     lse*log2e and D of a unit's queries are staged in shared memory by the producer warp.
//   dQ: item = (128-query block qb, batch*head); units = 64-key halves of the key
//     blocks 0 .. qb, in query-row orientation (lse and D are registers):
//       S = Q K_u^T, dP = dO V_u^T                     (M=128 queries, N=64 keys, K=64)
//       dQ += dS K_u                                   (M=128 queries, N=64, K=64 keys)
//
// Operands. With both MMA operands in shared memory these small products are
// bound by shared-memory bandwidth (a 128 x 64 x 16 MMA re-reads a 4 KB A tile
// for 2 KB of B). So every A operand lives in TMEM: the item's fixed 128-row tiles
// (Q and dO, or K and V) are copied there once per item by the element-wise warps,
// which also write P^T / dS^T (dS) there directly; only the 64-row B tiles of each
// unit are read from shared memory.
// Pipelining. Every unit streams its own 16 KB stage (two 64-row tiles) through a
// 7- or 8-deep ring, released as soon as that unit's accumulation MMAs complete,
// so a stage's copy is issued several units before it is needed (tile loads take
// 1-3 us under load). The score tiles are double-buffered in TMEM.
// MMA issue. One thread can issue a 1-SM tcgen05.mma only every ~96 cycles whatever
// its N (measured on B200), while the tensor pipe overlaps the streams of several
// threads. So each product has its own issuing thread (lane 0 of its own warp):
// dK/dV: S^T, dP^T, dV, dK; dQ: S, dP, dQ. The score threads never wait behind the
// accumulation threads, which wait for the element-wise warps.
// Warps: 0 TMA producer (lane 0 issues the copies), then the MMA warps (warp 1 owns
// the TMEM allocation), then 16 element-wise warps: warp w reads TMEM lane quarter
// w % 4 (32 rows) and column group (w - first) / 4 (16 of the 64 unit columns).
// D = rowsum(dO * O) comes precomputed. Every wait is bounded (device error word,
// no trap).
// ---------------------------------------------------------------------------
constexpr int FB_EW_WARPS = 16;
constexpr int FBK_EW0 = 5;  // dK/dV: producer, S^T, dP^T, dV, dK issuers, then element-wise warps
constexpr int FBQ_EW0 = 4;  // dQ: producer, S, dP, dQ issuers, then element-wise warps
constexpr int FBK_THREADS = 32 * (FBK_EW0 + FB_EW_WARPS);  // 672
constexpr int FBQ_THREADS = 32 * (FBQ_EW0 + FB_EW_WARPS);  // 640
constexpr int FB_HALF = 64 * 128;                  // 8 KB: 64 rows x 64 bf16 (128-byte rows)
constexpr int FB_UNIT = 2 * FB_HALF;               // 16 KB: a stage (two half tiles) or a 128 x 64 tile
constexpr int FB_BARS = 512;
// dK/dV kernel shared memory: K/V [2 items] | stages (Q_u, dO_u) | lse/D per stage |
// output staging (dK, dV tiles for one TMA store each) | barriers
constexpr int FBK_NST = 6;
constexpr int FBK_OFF_KV = 0;
constexpr int FBK_OFF_ST = 4 * FA_TILE;
constexpr int FBK_OFF_LD = FBK_OFF_ST + FBK_NST * FB_UNIT;
constexpr int FBK_OFF_OUT = FBK_OFF_LD + 4096;  // FBK_NST x 512 bytes, rounded up
constexpr int FBK_OFF_BAR = FBK_OFF_OUT + 2 * FA_TILE;
constexpr int FBK_SMEM = FBK_OFF_BAR + FB_BARS + 1024;
// dQ kernel shared memory: Q/dO [2 items] | stages (K_u, V_u) | output staging (dQ) | barriers
constexpr int FBQ_NST = 8;
constexpr int FBQ_OFF_QD = 0;
constexpr int FBQ_OFF_ST = 4 * FA_TILE;
constexpr int FBQ_OFF_OUT = FBQ_OFF_ST + FBQ_NST * FB_UNIT;
constexpr int FBQ_OFF_BAR = FBQ_OFF_OUT + FA_TILE;
constexpr int FBQ_SMEM = FBQ_OFF_BAR + FB_BARS + 1024;
static_assert(FBK_NST * 512 <= 4096, "lse/D staging");
static_assert(FBQ_SMEM <= 232448 && FBK_SMEM <= 232448, "shared memory per CTA");
// TMEM columns (512): score tiles [2 units] x (S 64 | dP 64) at 0 and 128, then
//   dK/dV: K | V A operands (32 + 32) at 256, P^T at 320, dS^T at 352 (32 each), dV | dK at 384
//   dQ:    Q | dO A operands (32 + 32) at 256, dS [2 units] at 320 (32 each), dQ [2 items] at 384
constexpr int FB_SBUF = 2;
constexpr uint32_t FBK_TM_KV = 256, FBK_TM_P = 320, FBK_TM_DS = 352, FBK_TM_ACC = 384;
constexpr uint32_t FBQ_TM_Q = 256, FBQ_TM_DS = 320, FBQ_TM_ACC = 384;
constexpr uint32_t FB_TMEM_COLS = 512;

// 16 bf16 values (two 16-byte chunks, chunk index c16 and c16 + 1 of a 64-column row)
// into row r of a 128-byte-swizzled tile with 128-byte rows.
__device__ __forceinline__ void fb_store16(uint8_t* tile, int r, int c16, const float (&v)[16]) {
#pragma unroll
  for (int k = 0; k < 2; ++k) {
    const int e = 8 * k;
    uint4 w = make_uint4(pack_bf16x2(v[e], v[e + 1]), pack_bf16x2(v[e + 2], v[e + 3]),
                         pack_bf16x2(v[e + 4], v[e + 5]), pack_bf16x2(v[e + 6], v[e + 7]));
    *reinterpret_cast<uint4*>(tile + r * 128 + (((c16 + k) ^ (r & 7)) << 4)) = w;
  }
}

// 16 accumulator values (x mul) of row r into a 128-row output staging tile laid out
// as the 128-byte-swizzled box of a TMA store
__device__ __forceinline__ void fb_stage_row16(uint8_t* tile, int r, int cg, const uint32_t (&v)[16], float mul) {
  float f[16];
#pragma unroll
  for (int e = 0; e < 16; ++e) f[e] = __uint_as_float(v[e]) * mul;
  fb_store16(tile, r, cg * 2, f);
}

// Bounded wait whose result is the same for every lane of the warp (lane 0 waits).
__device__ __forceinline__ bool fb_warp_wait(uint64_t* bar, uint32_t parity, volatile int* abort, uint64_t lim,
                                             int lane) {
  int ok = 1;
  if (lane == 0) ok = mbar_wait_bounded(bar, parity, abort, lim) ? 1 : 0;
  return __shfl_sync(0xffffffffu, ok, 0) != 0;
}

// Copy 16 bf16 (columns [cg*16, cg*16 + 16)) of row r of a 128-byte-swizzled tile
// with 128-byte rows into 8 TMEM columns of the thread's lane, as an MMA A operand.
__device__ __forceinline__ void fb_row_to_tmem(const uint8_t* tile, int r, int cg, uint32_t taddr) {
  const uint4 a = *reinterpret_cast<const uint4*>(tile + r * 128 + (((cg * 2) ^ (r & 7)) << 4));
  const uint4 b = *reinterpret_cast<const uint4*>(tile + r * 128 + (((cg * 2 + 1) ^ (r & 7)) << 4));
  const uint32_t w[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
  tmem_st_32x32b_x8(taddr, w);
}
// 16 values as 8 packed bf16 pairs into 8 TMEM columns of the thread's lane
__device__ __forceinline__ void fb_vals_to_tmem(const float (&v)[16], uint32_t taddr) {
  uint32_t w[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) w[i] = pack_bf16x2(v[2 * i], v[2 * i + 1]);
  tmem_st_32x32b_x8(taddr, w);
}


__global__ void __launch_bounds__(FBK_THREADS, 1)
    attn_bwd_dkdv_tc_kernel(const __grid_constant__ CUtensorMap tm_kv, const __grid_constant__ CUtensorMap tm_q64,
                            const __grid_constant__ CUtensorMap tm_do64, const __grid_constant__ CUtensorMap tm_out,
                            const float* __restrict__ lse, const float* __restrict__ Dg, int T, int NH, int BH,
                            float scale, int* err, unsigned long long timeout_ns) {
  extern __shared__ uint8_t fb_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(fb_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bar = reinterpret_cast<uint64_t*>(sm + FBK_OFF_BAR);
  uint64_t* kv_full = bar;                    // [2] K/V tiles landed in shared memory
  uint64_t* kv_empty = kv_full + 2;           // [2] copied into TMEM by the element-wise warps
  uint64_t* kva_full = kv_empty + 2;          // K/V A operands written to TMEM (once per item)
  uint64_t* st_full = kva_full + 1;           // [FBK_NST]
  uint64_t* st_empty = st_full + FBK_NST;     // [FBK_NST]
  uint64_t* s_full = st_empty + FBK_NST;      // [FB_SBUF]
  uint64_t* s_empty = s_full + FB_SBUF;       // [FB_SBUF]
  uint64_t* p_full = s_empty + FB_SBUF;
  uint64_t* p_free = p_full + 1;
  uint64_t* acc_full = p_free + 1;
  uint64_t* acc_empty = acc_full + 1;
  uint64_t* out_full = acc_empty + 1;         // output tiles staged (element-wise warps)
  uint64_t* out_free = out_full + 1;          // the previous item's TMA stores have read the staging
  uint64_t* drain = out_free + 1;             // [4]: one per MMA thread (abort path)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 4);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(drain + 5);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int C = NH * 64;
  const int nqb = (T + FA_BM - 1) / FA_BM;
  const int nitems = nqb * BH;  // item = kb * BH + bh: the longest rows (kb = 0) come first
  const uint64_t lim = timeout_ns;

  if (threadIdx.x == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(&kv_full[i], 1);
      mbar_init(&kv_empty[i], FB_EW_WARPS);
    }
    for (int i = 0; i < 4; ++i) mbar_init(&drain[i], 1);
    mbar_init(kva_full, FB_EW_WARPS);
    for (int i = 0; i < FBK_NST; ++i) {
      mbar_init(&st_full[i], 32);  // the producer warp's lanes (lane 0 with the copy bytes)
      mbar_init(&st_empty[i], 2);  // the dV and dK threads
    }
    for (int i = 0; i < FB_SBUF; ++i) {
      mbar_init(&s_full[i], 2);  // the S^T and dP^T threads
      mbar_init(&s_empty[i], FB_EW_WARPS);
    }
    mbar_init(p_full, FB_EW_WARPS);
    mbar_init(p_free, 2);  // the dV and dK threads
    mbar_init(acc_full, 2);
    mbar_init(acc_empty, FB_EW_WARPS);
    mbar_init(out_full, FB_EW_WARPS);
    mbar_init(out_free, 1);
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
    // ---------------- producer: K/V per item; (Q_u, dO_u, lse, D) per unit ----------------
    if (lane == 0) {
      tma_prefetch_desc(&tm_kv);
      tma_prefetch_desc(&tm_q64);
      tma_prefetch_desc(&tm_do64);
    }
    bool ok = true;
    uint32_t kv_iss = 0, kv_par = 0, st_iss = 0, st_par = 0;  // lane 0: copies in flight, for the abort path
    int U = 0;                                                 // unit (= stage use) counter over all items
    for (int it = 0, item = blockIdx.x; item < nitems && ok; ++it, item += gridDim.x) {
      const int kb = item / BH, bh = item - kb * BH, b = bh / NH, h = bh - b * NH;
      const int kvb = it & 1;
      if (!(ok = fb_warp_wait(&kv_empty[kvb], ((it >> 1) & 1) ^ 1, abort_flag, lim, lane))) break;
      if (lane == 0) {
        uint8_t* kd = sm + FBK_OFF_KV + kvb * 2 * FA_TILE;
        mbar_arrive_expect_tx(&kv_full[kvb], 2 * FA_TILE);
        tma_load_3d(kd, &tm_kv, &kv_full[kvb], C + h * 64, kb * FA_BN, b);
        tma_load_3d(kd + FA_TILE, &tm_kv, &kv_full[kvb], 2 * C + h * 64, kb * FA_BN, b);
        kv_iss |= 1u << kvb;
        kv_par = (kv_par & ~(1u << kvb)) | ((uint32_t)((it >> 1) & 1) << kvb);
      }
      const float* lse_bh = lse + (long long)bh * T;
      const float* D_bh = Dg + (long long)bh * T;
      for (int q0 = kb * FA_BM; q0 < nqb * FA_BM; q0 += 64, ++U) {
        const int s = U % FBK_NST;
        const uint32_t ph = (uint32_t)((U / FBK_NST) & 1);
        if (!(ok = fb_warp_wait(&st_empty[s], ph ^ 1, abort_flag, lim, lane))) break;
        float* ld = reinterpret_cast<float*>(sm + FBK_OFF_LD + s * 512);  // [lse*log2e 64][D 64]
#pragma unroll
        for (int k = 0; k < 2; ++k) {
          const int c = lane * 2 + k, q = q0 + c;
          ld[c] = q < T ? lse_bh[q] * LOG2E : INFINITY;  // P = 0 for queries past the end
          ld[64 + c] = q < T ? D_bh[q] : 0.f;
        }
        if (lane == 0) {
          uint8_t* d = sm + FBK_OFF_ST + s * FB_UNIT;
          mbar_arrive_expect_tx(&st_full[s], FB_UNIT);
          tma_load_3d(d, &tm_q64, &st_full[s], h * 64, q0, b);
          tma_load_3d(d + FB_HALF, &tm_do64, &st_full[s], h * 64, q0, b);
          st_iss |= 1u << s;
          st_par = (st_par & ~(1u << s)) | (ph << s);
        } else {
          mbar_arrive(&st_full[s]);
        }
      }
    }
    if (!ok && lane == 0) {
      raise_device_error(err, DEV_TIMEOUT);
      *abort_flag = 1;
      int never = 0;  // let the copies in flight land before the CTA's shared memory goes away
      for (int i = 0; i < 2; ++i)
        if ((kv_iss >> i) & 1u)
          mbar_wait_bounded(&kv_full[i], (kv_par >> i) & 1u, reinterpret_cast<volatile int*>(&never), lim);
      for (int i = 0; i < FBK_NST; ++i)
        if ((st_iss >> i) & 1u)
          mbar_wait_bounded(&st_full[i], (st_par >> i) & 1u, reinterpret_cast<volatile int*>(&never), lim);
    }
  } else if (warp == 1 || warp == 2) {
    if (lane == 0) {
      // ---------------- score MMAs: S^T = K Q_u^T (warp 1), dP^T = V dO_u^T (warp 2); A from TMEM ----------------
      const int part = warp - 1;
      constexpr uint32_t idesc_s = make_idesc_bf16(128, 64, false, false);
      bool ok = true, any = false;
      int U = 0;
      for (int it = 0, item = blockIdx.x; item < nitems && ok; ++it, item += gridDim.x) {
        const int nu = 2 * (nqb - item / BH);
        if (!mbar_wait_bounded(kva_full, it & 1, abort_flag, lim)) {
          ok = false;
          break;
        }
        for (int u = 0; u < nu; ++u, ++U) {
          const int s = U % FBK_NST, sb = U % FB_SBUF;
          if (!mbar_wait_bounded(&st_full[s], (U / FBK_NST) & 1, abort_flag, lim) ||
              !mbar_wait_bounded(&s_empty[sb], ((U / FB_SBUF) & 1) ^ 1, abort_flag, lim)) {
            ok = false;
            break;
          }
          tc_fence_after();
          // B = Q_u (part 0) or dO_u (part 1): 64 rows, K-major
          const uint32_t b_addr = smem_u32(sm + FBK_OFF_ST + s * FB_UNIT) + part * FB_HALF;
          const uint32_t d = tmem + (uint32_t)(sb * 128 + part * 64);
#pragma unroll
          for (int k = 0; k < 4; ++k)
            umma_bf16_ts(d, tmem + FBK_TM_KV + part * 32 + k * 8, make_sw128_desc(b_addr + k * 32, 16, 1024), idesc_s,
                         k > 0 ? 1u : 0u);
          umma_commit(&s_full[sb]);
          any = true;
        }
      }
      if (!ok) {
        raise_device_error(err, DEV_TIMEOUT);
        *abort_flag = 1;
        if (any) {  // wait for the MMAs already issued before the TMEM is freed
          int never = 0;
          umma_commit(&drain[part]);
          mbar_wait_bounded(&drain[part], 0, reinterpret_cast<volatile int*>(&never), lim);
        }
      }
    }
  } else if (warp == 3 || warp == 4) {
    if (lane == 0) {
      // ---------------- accumulation MMAs: dV += P^T dO_u (warp 3), dK += dS^T Q_u (warp 4); A from TMEM ----------------
      const int part = warp - 3;
      constexpr uint32_t idesc_a = make_idesc_bf16(128, 64, false, true);  // B = dO_u / Q_u, MN-major
      bool ok = true, any = false;
      int U = 0;
      for (int it = 0, item = blockIdx.x; item < nitems && ok; ++it, item += gridDim.x) {
        const int nu = 2 * (nqb - item / BH);
        // the element-wise warps have read the previous item's dV / dK
        if (!mbar_wait_bounded(acc_empty, (it & 1) ^ 1, abort_flag, lim)) {
          ok = false;
          break;
        }
        for (int u = 0; u < nu; ++u, ++U) {
          const int s = U % FBK_NST;
          if (!mbar_wait_bounded(&st_full[s], (U / FBK_NST) & 1, abort_flag, lim) ||
              !mbar_wait_bounded(p_full, U & 1, abort_flag, lim)) {
            ok = false;
            break;
          }
          tc_fence_after();
          // K = 64 queries: A = P^T (part 0) or dS^T (part 1); B = 16 query rows of dO_u (part 0)
          // or Q_u (part 1) per step (MN-major)
          const uint32_t b_addr = smem_u32(sm + FBK_OFF_ST + s * FB_UNIT) + (1 - part) * FB_HALF;
          const uint32_t a_tm = tmem + (part == 0 ? FBK_TM_P : FBK_TM_DS);
          const uint32_t acc = tmem + FBK_TM_ACC + part * 64;
#pragma unroll
          for (int k = 0; k < 4; ++k)
            umma_bf16_ts(acc, a_tm + k * 8, make_sw128_desc(b_addr + k * 2048, 8192, 1024), idesc_a,
                         (u > 0 || k > 0) ? 1u : 0u);
          any = true;
          umma_commit(p_free);
          // the unit's scores were consumed before P^T was written: its score MMAs are complete
          umma_commit(&st_empty[s]);
          if (u == nu - 1) umma_commit(acc_full);
        }
      }
      if (!ok) {
        raise_device_error(err, DEV_TIMEOUT);
        *abort_flag = 1;
        if (any) {
          int never = 0;
          umma_commit(&drain[2 + part]);
          mbar_wait_bounded(&drain[2 + part], 0, reinterpret_cast<volatile int*>(&never), lim);
        }
      }
    }
  } else {
    // ---------------- element-wise warps: key row r, query columns [cg*16, cg*16 + 16) of each unit ----------------
    const int q4 = warp & 3, cg = (warp - FBK_EW0) >> 2;
    const int r = q4 * 32 + lane;
    const bool issuer = (warp == FBK_EW0 && lane == 0);  // issues the output tiles' TMA stores
    const uint32_t lane_off = (uint32_t)(q4 * 32) << 16;
    const float sl2 = scale * LOG2E;
    bool fail = false;
    int U = 0;
    // K and V rows of item `it` into the TMEM A operands (after the previous item's score
    // MMAs, whose results this warp has all seen)
    auto load_operands = [&](int it) -> bool {
      const int kvb = it & 1;
      if (!mbar_wait_bounded(&kv_full[kvb], (it >> 1) & 1, abort_flag, lim)) return false;
      const uint8_t* kd = sm + FBK_OFF_KV + kvb * 2 * FA_TILE;
      fb_row_to_tmem(kd, r, cg, tmem + lane_off + FBK_TM_KV + cg * 8);
      fb_row_to_tmem(kd + FA_TILE, r, cg, tmem + lane_off + FBK_TM_KV + 32 + cg * 8);
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(kva_full);
        mbar_arrive(&kv_empty[kvb]);
      }
      return true;
    };
    if ((int)blockIdx.x < nitems) fail = !load_operands(0);
    for (int it = 0, item = blockIdx.x; item < nitems && !fail; ++it, item += gridDim.x) {
      const int kb = item / BH, bh = item - kb * BH, b = bh / NH, h = bh - b * NH;
      const int nu = 2 * (nqb - kb);
      for (int u = 0; u < nu; ++u, ++U) {
        const int sb = U % FB_SBUF, s = U % FBK_NST;
        // the producer's lse / D of this unit (acquired directly from its lanes), then the scores
        if (!mbar_wait_bounded(&st_full[s], (U / FBK_NST) & 1, abort_flag, lim) ||
            !mbar_wait_bounded(&s_full[sb], (U / FB_SBUF) & 1, abort_flag, lim)) {
          fail = true;
          break;
        }
        tc_fence_after();
        uint32_t sv[16], dv[16];
        tmem_ld_32x32b_x16(tmem + lane_off + (uint32_t)(sb * 128 + cg * 16), sv);
        tmem_ld_32x32b_x16(tmem + lane_off + (uint32_t)(sb * 128 + 64 + cg * 16), dv);
        tmem_ld_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&s_empty[sb]);
        const float* ld = reinterpret_cast<const float*>(sm + FBK_OFF_LD + s * 512) + cg * 16;
        float p[16], ds[16];
        const int qcol0 = (u & 1) * 64 + cg * 16;  // query index within the block of column 0
        const bool diag = u < 2;                    // the query block kb itself
#pragma unroll
        for (int e4 = 0; e4 < 4; ++e4) {
          const float4 L4 = *reinterpret_cast<const float4*>(ld + 4 * e4);
          const float4 D4 = *reinterpret_cast<const float4*>(ld + 64 + 4 * e4);
          const float Lv[4] = {L4.x, L4.y, L4.z, L4.w}, Dv[4] = {D4.x, D4.y, D4.z, D4.w};
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const int e = 4 * e4 + i;
            float pe = ex2_fast(fmaf(__uint_as_float(sv[e]), sl2, -Lv[i]));
            if (diag && r > qcol0 + e) pe = 0.f;  // key after query
            p[e] = pe;
            ds[e] = pe * (__uint_as_float(dv[e]) - Dv[i]);
          }
        }
        // the previous unit's dV / dK MMAs have finished reading P^T and dS^T
        if (!mbar_wait_bounded(p_free, (U & 1) ^ 1, abort_flag, lim)) {
          fail = true;
          break;
        }
        fb_vals_to_tmem(p, tmem + lane_off + FBK_TM_P + cg * 8);
        fb_vals_to_tmem(ds, tmem + lane_off + FBK_TM_DS + cg * 8);
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(p_full);
      }
      if (fail) break;
      // the next item's K / V first (lets its score MMAs start), then this item's dV / dK
      if (item + (int)gridDim.x < nitems && !load_operands(it + 1)) {
        fail = true;
        break;
      }
      if (!mbar_wait_bounded(acc_full, it & 1, abort_flag, lim)) {
        fail = true;
        break;
      }
      tc_fence_after();
      uint32_t v[16], k[16];
      tmem_ld_32x32b_x16(tmem + lane_off + FBK_TM_ACC + (uint32_t)(cg * 16), v);
      tmem_ld_32x32b_x16(tmem + lane_off + FBK_TM_ACC + (uint32_t)(64 + cg * 16), k);
      tmem_ld_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(acc_empty);
      // dK (scaled) and dV through shared memory, one TMA store per tile (rows past T are clipped)
      if (issuer && it > 0) {
        bulk_wait_read<0>();
        mbar_arrive(out_free);
      }
      if (!mbar_wait_bounded(out_free, (it & 1) ^ 1, abort_flag, lim)) {
        fail = true;
        break;
      }
      fb_stage_row16(sm + FBK_OFF_OUT, r, cg, k, scale);
      fb_stage_row16(sm + FBK_OFF_OUT + FA_TILE, r, cg, v, 1.0f);
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(out_full);
      if (issuer) {
        if (!mbar_wait_bounded(out_full, it & 1, abort_flag, lim)) {
          fail = true;
          break;
        }
        tma_store_3d(&tm_out, sm + FBK_OFF_OUT, C + h * 64, kb * FA_BN, b);
        tma_store_3d(&tm_out, sm + FBK_OFF_OUT + FA_TILE, 2 * C + h * 64, kb * FA_BN, b);
        bulk_commit();
      }
    }
    if (issuer) bulk_wait_all();  // the staging must outlive the stores' reads
    if (fail && lane == 0) {
      raise_device_error(err, DEV_TIMEOUT);
      *abort_flag = 1;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, FB_TMEM_COLS);
  }
}

__global__ void __launch_bounds__(FBQ_THREADS, 1)
    attn_bwd_dq_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_do,
                          const __grid_constant__ CUtensorMap tm_kv64, const __grid_constant__ CUtensorMap tm_out,
                          const float* __restrict__ lse, const float* __restrict__ Dg, int T, int NH, int BH,
                          float scale, int* err, unsigned long long timeout_ns) {
  extern __shared__ uint8_t fb_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(fb_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bar = reinterpret_cast<uint64_t*>(sm + FBQ_OFF_BAR);
  uint64_t* qd_full = bar;                    // [2] Q/dO tiles landed in shared memory
  uint64_t* qd_empty = qd_full + 2;           // [2] copied into TMEM by the element-wise warps
  uint64_t* qa_full = qd_empty + 2;           // Q/dO A operands written to TMEM (once per item)
  uint64_t* st_full = qa_full + 1;            // [FBQ_NST]
  uint64_t* st_empty = st_full + FBQ_NST;     // [FBQ_NST]
  uint64_t* s_full = st_empty + FBQ_NST;      // [FB_SBUF]
  uint64_t* s_empty = s_full + FB_SBUF;       // [FB_SBUF]
  uint64_t* ds_full = s_empty + FB_SBUF;      // [2]
  uint64_t* ds_free = ds_full + 2;            // [2]
  uint64_t* acc_full = ds_free + 2;           // [2]
  uint64_t* acc_empty = acc_full + 2;         // [2]
  uint64_t* out_full = acc_empty + 2;         // output tile staged (element-wise warps)
  uint64_t* out_free = out_full + 1;          // the previous item's TMA store has read the staging
  uint64_t* drain = out_free + 1;             // [3]: one per MMA thread (abort path)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 3);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(drain + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int C = NH * 64;
  const int nqb = (T + FA_BM - 1) / FA_BM;
  const int nitems = nqb * BH;  // item w: query block nqb - 1 - w / BH (longest rows first), bh = w % BH
  const uint64_t lim = timeout_ns;

  if (threadIdx.x == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(&qd_full[i], 1);
      mbar_init(&qd_empty[i], FB_EW_WARPS);
      mbar_init(&ds_full[i], FB_EW_WARPS);
      mbar_init(&ds_free[i], 1);
      mbar_init(&acc_full[i], 1);
      mbar_init(&acc_empty[i], FB_EW_WARPS);
    }
    for (int i = 0; i < 3; ++i) mbar_init(&drain[i], 1);
    mbar_init(out_full, FB_EW_WARPS);
    mbar_init(out_free, 1);
    mbar_init(qa_full, FB_EW_WARPS);
    for (int i = 0; i < FBQ_NST; ++i) {
      mbar_init(&st_full[i], 1);
      mbar_init(&st_empty[i], 1);
    }
    for (int i = 0; i < FB_SBUF; ++i) {
      mbar_init(&s_full[i], 2);  // the S and dP threads
      mbar_init(&s_empty[i], FB_EW_WARPS);
    }
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
      // ---------------- producer: Q/dO per item, (K_u, V_u) per unit ----------------
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_do);
      tma_prefetch_desc(&tm_kv64);
      bool ok = true;
      uint32_t qd_iss = 0, qd_par = 0, st_iss = 0, st_par = 0;
      int U = 0;
      for (int it = 0, item = blockIdx.x; item < nitems && ok; ++it, item += gridDim.x) {
        const int qb = nqb - 1 - item / BH, bh = item % BH, b = bh / NH, h = bh - b * NH;
        const int qdb = it & 1;
        if (!mbar_wait_bounded(&qd_empty[qdb], ((it >> 1) & 1) ^ 1, abort_flag, lim)) {
          ok = false;
          break;
        }
        uint8_t* qd = sm + FBQ_OFF_QD + qdb * 2 * FA_TILE;
        mbar_arrive_expect_tx(&qd_full[qdb], 2 * FA_TILE);
        tma_load_3d(qd, &tm_q, &qd_full[qdb], h * 64, qb * FA_BM, b);
        tma_load_3d(qd + FA_TILE, &tm_do, &qd_full[qdb], h * 64, qb * FA_BM, b);
        qd_iss |= 1u << qdb;
        qd_par = (qd_par & ~(1u << qdb)) | ((uint32_t)((it >> 1) & 1) << qdb);
        for (int k0 = 0; k0 < (qb + 1) * FA_BN; k0 += 64, ++U) {
          const int s = U % FBQ_NST;
          const uint32_t ph = (uint32_t)((U / FBQ_NST) & 1);
          if (!mbar_wait_bounded(&st_empty[s], ph ^ 1, abort_flag, lim)) {
            ok = false;
            break;
          }
          uint8_t* d = sm + FBQ_OFF_ST + s * FB_UNIT;
          mbar_arrive_expect_tx(&st_full[s], FB_UNIT);
          tma_load_3d(d, &tm_kv64, &st_full[s], C + h * 64, k0, b);
          tma_load_3d(d + FB_HALF, &tm_kv64, &st_full[s], 2 * C + h * 64, k0, b);
          st_iss |= 1u << s;
          st_par = (st_par & ~(1u << s)) | (ph << s);
        }
      }
      if (!ok) {
        raise_device_error(err, DEV_TIMEOUT);
        *abort_flag = 1;
        int never = 0;
        for (int i = 0; i < 2; ++i)
          if ((qd_iss >> i) & 1u)
            mbar_wait_bounded(&qd_full[i], (qd_par >> i) & 1u, reinterpret_cast<volatile int*>(&never), lim);
        for (int i = 0; i < FBQ_NST; ++i)
          if ((st_iss >> i) & 1u)
            mbar_wait_bounded(&st_full[i], (st_par >> i) & 1u, reinterpret_cast<volatile int*>(&never), lim);
      }
    }
  } else if (warp == 1 || warp == 2) {
    if (lane == 0) {
      // ---------------- score MMAs: S = Q K_u^T (warp 1), dP = dO V_u^T (warp 2); A from TMEM ----------------
      const int part = warp - 1;
      constexpr uint32_t idesc_s = make_idesc_bf16(128, 64, false, false);
      bool ok = true, any = false;
      int U = 0;
      for (int it = 0, item = blockIdx.x; item < nitems && ok; ++it, item += gridDim.x) {
        const int nu = 2 * (nqb - item / BH);
        if (!mbar_wait_bounded(qa_full, it & 1, abort_flag, lim)) {
          ok = false;
          break;
        }
        for (int u = 0; u < nu; ++u, ++U) {
          const int s = U % FBQ_NST, sb = U % FB_SBUF;
          if (!mbar_wait_bounded(&st_full[s], (U / FBQ_NST) & 1, abort_flag, lim) ||
              !mbar_wait_bounded(&s_empty[sb], ((U / FB_SBUF) & 1) ^ 1, abort_flag, lim)) {
            ok = false;
            break;
          }
          tc_fence_after();
          // B = K_u (part 0) or V_u (part 1): 64 rows, K-major
          const uint32_t b_addr = smem_u32(sm + FBQ_OFF_ST + s * FB_UNIT) + part * FB_HALF;
          const uint32_t d = tmem + (uint32_t)(sb * 128 + part * 64);
#pragma unroll
          for (int k = 0; k < 4; ++k)
            umma_bf16_ts(d, tmem + FBQ_TM_Q + part * 32 + k * 8, make_sw128_desc(b_addr + k * 32, 16, 1024), idesc_s,
                         k > 0 ? 1u : 0u);
          umma_commit(&s_full[sb]);
          any = true;
        }
      }
      if (!ok) {
        raise_device_error(err, DEV_TIMEOUT);
        *abort_flag = 1;
        if (any) {
          int never = 0;
          umma_commit(&drain[part]);
          mbar_wait_bounded(&drain[part], 0, reinterpret_cast<volatile int*>(&never), lim);
        }
      }
    }
  } else if (warp == 3) {
    if (lane == 0) {
      // ---------------- accumulation MMAs: dQ += dS K_u (A = dS from TMEM) ----------------
      constexpr uint32_t idesc_q = make_idesc_bf16(128, 64, false, true);  // B = K_u, MN-major
      bool ok = true, any = false;
      int U = 0;
      for (int it = 0, item = blockIdx.x; item < nitems && ok; ++it, item += gridDim.x) {
        const int ab = it & 1, nu = 2 * (nqb - item / BH);
        if (!mbar_wait_bounded(&acc_empty[ab], ((it >> 1) & 1) ^ 1, abort_flag, lim)) {
          ok = false;
          break;
        }
        for (int u = 0; u < nu; ++u, ++U) {
          const int s = U % FBQ_NST, dsb = U & 1;
          if (!mbar_wait_bounded(&st_full[s], (U / FBQ_NST) & 1, abort_flag, lim) ||
              !mbar_wait_bounded(&ds_full[dsb], (U >> 1) & 1, abort_flag, lim)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t k_addr = smem_u32(sm + FBQ_OFF_ST + s * FB_UNIT);
          const uint32_t acc = tmem + FBQ_TM_ACC + (uint32_t)(ab * 64);
          // K = 64 keys: B = 16 key rows of K_u per step (MN-major)
#pragma unroll
          for (int k = 0; k < 4; ++k)
            umma_bf16_ts(acc, tmem + FBQ_TM_DS + dsb * 32 + k * 8, make_sw128_desc(k_addr + k * 2048, 8192, 1024),
                         idesc_q, (u > 0 || k > 0) ? 1u : 0u);
          any = true;
          umma_commit(&ds_free[dsb]);
          umma_commit(&st_empty[s]);  // the unit's score MMAs completed before dS was written
          if (u == nu - 1) umma_commit(&acc_full[ab]);
        }
      }
      if (!ok) {
        raise_device_error(err, DEV_TIMEOUT);
        *abort_flag = 1;
        if (any) {
          int never = 0;
          umma_commit(&drain[2]);
          mbar_wait_bounded(&drain[2], 0, reinterpret_cast<volatile int*>(&never), lim);
        }
      }
    }
  } else {
    // ---------------- element-wise warps: query row r, key columns [cg*16, cg*16 + 16) of each unit ----------------
    const int q4 = warp & 3, cg = (warp - FBQ_EW0) >> 2;
    const int r = q4 * 32 + lane;
    const bool issuer = (warp == FBQ_EW0 && lane == 0);  // issues the output tile's TMA store
    const uint32_t lane_off = (uint32_t)(q4 * 32) << 16;
    const float sl2 = scale * LOG2E;
    bool fail = false;
    int U = 0;
    // Q and dO rows of item `it` (in shared memory) into the TMEM A operands. The score
    // MMAs of the previous item, the only readers of that TMEM, are complete: this warp
    // has seen all of their results.
    auto load_operands = [&](int it) -> bool {
      const int qdb = it & 1;
      if (!mbar_wait_bounded(&qd_full[qdb], (it >> 1) & 1, abort_flag, lim)) return false;
      const uint8_t* qd = sm + FBQ_OFF_QD + qdb * 2 * FA_TILE;
      fb_row_to_tmem(qd, r, cg, tmem + lane_off + FBQ_TM_Q + cg * 8);
      fb_row_to_tmem(qd + FA_TILE, r, cg, tmem + lane_off + FBQ_TM_Q + 32 + cg * 8);
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(qa_full);
        mbar_arrive(&qd_empty[qdb]);
      }
      return true;
    };
    // lse (log2 units) and D of this thread's query row, one item ahead
    float lse2 = INFINITY, Dr = 0.f;
    if ((int)blockIdx.x < nitems) {
      const int item = blockIdx.x, qrow = (nqb - 1 - item / BH) * FA_BM + r;
      const long long o = (long long)(item % BH) * T + qrow;
      if (qrow < T) {
        lse2 = lse[o] * LOG2E;
        Dr = Dg[o];
      }
      fail = !load_operands(0);
    }
    for (int it = 0, item = blockIdx.x; item < nitems && !fail; ++it, item += gridDim.x) {
      const int qb = nqb - 1 - item / BH, bh = item % BH, b = bh / NH, h = bh - b * NH;
      const int nu = 2 * (qb + 1);
      // the next item's lse / D: loads issued now, first used at the item switch
      float lse_n = INFINITY, Dr_n = 0.f;
      if (item + (int)gridDim.x < nitems) {
        const int item2 = item + gridDim.x, qrow2 = (nqb - 1 - item2 / BH) * FA_BM + r;
        const long long o = (long long)(item2 % BH) * T + qrow2;
        if (qrow2 < T) {
          lse_n = __ldg(lse + o);
          Dr_n = __ldg(Dg + o);
        }
      }
      for (int u = 0; u < nu; ++u, ++U) {
        const int sb = U % FB_SBUF, dsb = U & 1;
        if (!mbar_wait_bounded(&s_full[sb], (U / FB_SBUF) & 1, abort_flag, lim)) {
          fail = true;
          break;
        }
        tc_fence_after();
        uint32_t sv[16], dv[16];
        tmem_ld_32x32b_x16(tmem + lane_off + (uint32_t)(sb * 128 + cg * 16), sv);
        tmem_ld_32x32b_x16(tmem + lane_off + (uint32_t)(sb * 128 + 64 + cg * 16), dv);
        tmem_ld_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&s_empty[sb]);
        float ds[16];
        const int kcol0 = (u & 1) * 64 + cg * 16;  // key index within the block of column 0
        const bool diag = u >= nu - 2;             // the key block qb itself
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          float pe = ex2_fast(fmaf(__uint_as_float(sv[e]), sl2, -lse2));
          if (diag && kcol0 + e > r) pe = 0.f;  // key after query
          ds[e] = pe * (__uint_as_float(dv[e]) - Dr);
        }
        // the dQ MMAs of unit U - 2 have finished reading this dS buffer
        if (!mbar_wait_bounded(&ds_free[dsb], ((U >> 1) & 1) ^ 1, abort_flag, lim)) {
          fail = true;
          break;
        }
        fb_vals_to_tmem(ds, tmem + lane_off + FBQ_TM_DS + dsb * 32 + cg * 8);
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&ds_full[dsb]);
      }
      if (fail) break;
      // the next item's operands first (lets its score MMAs start), then this item's dQ
      if (item + (int)gridDim.x < nitems && !load_operands(it + 1)) {
        fail = true;
        break;
      }
      const int ab = it & 1;
      if (!mbar_wait_bounded(&acc_full[ab], (it >> 1) & 1, abort_flag, lim)) {
        fail = true;
        break;
      }
      tc_fence_after();
      uint32_t v[16];
      tmem_ld_32x32b_x16(tmem + lane_off + FBQ_TM_ACC + (uint32_t)(ab * 64 + cg * 16), v);
      tmem_ld_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acc_empty[ab]);
      // dQ (scaled) through shared memory, one TMA store (rows past T are clipped)
      if (issuer && it > 0) {
        bulk_wait_read<0>();
        mbar_arrive(out_free);
      }
      if (!mbar_wait_bounded(out_free, (it & 1) ^ 1, abort_flag, lim)) {
        fail = true;
        break;
      }
      fb_stage_row16(sm + FBQ_OFF_OUT, r, cg, v, scale);
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(out_full);
      if (issuer) {
        if (!mbar_wait_bounded(out_full, it & 1, abort_flag, lim)) {
          fail = true;
          break;
        }
        tma_store_3d(&tm_out, sm + FBQ_OFF_OUT, h * 64, qb * FA_BM, b);
        bulk_commit();
      }
      lse2 = lse_n * LOG2E;
      Dr = Dr_n;
    }
    if (issuer) bulk_wait_all();  // the staging must outlive the store's read
    if (fail && lane == 0) {
      raise_device_error(err, DEV_TIMEOUT);
      *abort_flag = 1;
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
