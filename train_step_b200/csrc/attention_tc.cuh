// attention_tc.cuh -- causal flash attention on the 5th-generation tensor cores
// (tcgen05, accumulators and A operands in TMEM, tiles by TMA), head dim 64, bf16.
//
// Same mathematics as attention.cuh ("AxonLM", Key Features: Flash Attention;
// "GPT From Scratch", Key decisions): per (batch, head), online softmax over key
// blocks; lse = logsumexp of the scaled scores; the backward recomputes P from lse.
//
// Three persistent kernels (one CTA per SM looping over (block, batch*head) items,
// longest first): the forward, and a deterministic backward split into a dK/dV
// kernel (per key block) and a dQ kernel (per query block). They share one design,
// set by what B200 measurements showed:
//  * a thread can issue a 1-SM tcgen05.mma only every ~96 cycles whatever its N,
//    but the tensor pipe overlaps the streams of several threads, so every product
//    has its own issuing thread;
//  * A operands live in TMEM (the item's fixed 128-row tile, and the P / dS tiles
//    written there by the element-wise warps), so only 64-row B tiles are read from
//    shared memory;
//  * each 64-wide unit streams its own 16 KB stage through a deep TMA ring, so a
//    tile is requested several units before it is needed;
//  * outputs leave through a shared-memory tile and one TMA store per tile.
// Every mbarrier wait is bounded (device error word, early exit, no trap).
#pragma once
#include "attention.cuh"
#include "common.cuh"

namespace g2 {

constexpr int FA_BM = 128;  // queries per CTA
constexpr int FA_BN = 128;  // keys per block
constexpr int FA_TILE = FA_BM * 64 * 2;  // 16 KB: 128 rows x 64 bf16

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

// Bounded wait whose result is the same for every lane of the warp: lane 0 waits,
// broadcasts the outcome, and on success every lane observes the completed phase
// (its own acquire). Warps that go on to warp-collective tcgen05 instructions must
// never split on a wait's outcome.
__device__ __forceinline__ bool fb_warp_wait(uint64_t* bar, uint32_t parity, volatile int* abort, uint64_t lim,
                                             int lane) {
  int ok = 1;
  if (lane == 0) ok = mbar_wait_bounded(bar, parity, abort, lim) ? 1 : 0;
  ok = __shfl_sync(0xffffffffu, ok, 0);
  if (ok) mbar_try_wait(bar, parity);
  return ok != 0;
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
      if (!fb_warp_wait(&kv_full[kvb], (it >> 1) & 1, abort_flag, lim, lane)) return false;
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
        if (!fb_warp_wait(&st_full[s], (U / FBK_NST) & 1, abort_flag, lim, lane) ||
            !fb_warp_wait(&s_full[sb], (U / FB_SBUF) & 1, abort_flag, lim, lane)) {
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
        if (!fb_warp_wait(p_free, (U & 1) ^ 1, abort_flag, lim, lane)) {
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
      if (!fb_warp_wait(acc_full, it & 1, abort_flag, lim, lane)) {
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
      if (!fb_warp_wait(out_free, (it & 1) ^ 1, abort_flag, lim, lane)) {
        fail = true;
        break;
      }
      fb_stage_row16(sm + FBK_OFF_OUT, r, cg, k, scale);
      fb_stage_row16(sm + FBK_OFF_OUT + FA_TILE, r, cg, v, 1.0f);
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(out_full);
      if (issuer) {
        if (mbar_wait_bounded(out_full, it & 1, abort_flag, lim)) {
          tma_store_3d(&tm_out, sm + FBK_OFF_OUT, C + h * 64, kb * FA_BN, b);
          tma_store_3d(&tm_out, sm + FBK_OFF_OUT + FA_TILE, 2 * C + h * 64, kb * FA_BN, b);
          bulk_commit();
        } else {
          fail = true;
        }
      }
      if (__shfl_sync(0xffffffffu, fail ? 1 : 0, 0)) {  // the issuer's warp leaves together
        fail = true;
        break;
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
      if (!fb_warp_wait(&qd_full[qdb], (it >> 1) & 1, abort_flag, lim, lane)) return false;
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
        if (!fb_warp_wait(&s_full[sb], (U / FB_SBUF) & 1, abort_flag, lim, lane)) {
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
        if (!fb_warp_wait(&ds_free[dsb], ((U >> 1) & 1) ^ 1, abort_flag, lim, lane)) {
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
      if (!fb_warp_wait(&acc_full[ab], (it >> 1) & 1, abort_flag, lim, lane)) {
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
      if (!fb_warp_wait(out_free, (it & 1) ^ 1, abort_flag, lim, lane)) {
        fail = true;
        break;
      }
      fb_stage_row16(sm + FBQ_OFF_OUT, r, cg, v, scale);
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(out_full);
      if (issuer) {
        if (mbar_wait_bounded(out_full, it & 1, abort_flag, lim)) {
          tma_store_3d(&tm_out, sm + FBQ_OFF_OUT, h * 64, qb * FA_BM, b);
          bulk_commit();
        } else {
          fail = true;
        }
      }
      if (__shfl_sync(0xffffffffu, fail ? 1 : 0, 0)) {  // the issuer's warp leaves together
        fail = true;
        break;
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

// ---------------------------------------------------------------------------
// Forward on tcgen05, persistent (one CTA per SM looping over items). Item =
// (128-query block qb, batch*head), longest rows first; units = 64-key halves of
// the key blocks 0 .. qb, each streamed through the same 16 KB stage ring as the
// backward kernels.
//   S_u  = Q K_u^T     (M=128 queries, N=64 keys, K=64; A = Q in TMEM, B = K_u)
//   O_g += P_u V_u     (M=128, N=64, K=64 keys;     A = P_u in TMEM, B = V_u)
// Two softmax groups (4 warps each) take alternate units. Each thread owns one
// query row of its group's units, so a unit needs no exchange between threads;
// each group keeps its own running max m, row sum l and output accumulator O_g,
// and the two are merged when the item ends:
//   m = max(m_0, m_1), O = (O_0 2^(m_0-m) + O_1 2^(m_1-m)) / (l_0 2^(m_0-m) + l_1 2^(m_1-m)).
// A group re-bases its running max only when the new block maximum exceeds it by
// more than 8 (log2 units); otherwise its probabilities are taken against the
// stale max (at most 2^8, exact in fp32 and representable in bf16) and O_g and l
// stay consistent because both use the same reference. A re-base rescales the
// thread's row of O_g in TMEM once the previous P V product has completed.
// Warps: 0 TMA producer, 1 S MMAs, 2 P V MMAs, 3-6 softmax group 0, 7-10 group 1.
// Every wait is bounded (device error word, no trap).
// ---------------------------------------------------------------------------
constexpr int FF_THREADS = 352;
constexpr int FF_NST = 8;
constexpr int FF_OFF_Q = 0;                                  // Q tiles [2 items]
constexpr int FF_OFF_ST = 2 * FA_TILE;                       // stages (K_u | V_u)
constexpr int FF_OFF_OUT = FF_OFF_ST + FF_NST * FB_UNIT;     // output staging tile
constexpr int FF_OFF_X = FF_OFF_OUT + FA_TILE;               // (m, l) exchange [2 items][2 groups][128]
constexpr int FF_OFF_BAR = FF_OFF_X + 2 * 2 * 128 * 8;
constexpr int FF_SMEM = FF_OFF_BAR + FB_BARS + 1024;
static_assert(FF_SMEM <= 232448, "shared memory per CTA");
// TMEM: S [group][2] x 64 at 0..255, O [group] x 64 at 256, Q (32) at 384, P [group] x 32 at 416
constexpr uint32_t FF_TM_O = 256, FF_TM_Q = 384, FF_TM_P = 416, FF_TMEM_COLS = 512;
constexpr float FF_REBASE = 8.0f;

__global__ void __launch_bounds__(FF_THREADS, 1)
    attn_fwd_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_kv64,
                       const __grid_constant__ CUtensorMap tm_out, float* __restrict__ lse, int T, int NH, int BH,
                       float scale, int* err, unsigned long long timeout_ns) {
  extern __shared__ uint8_t ff_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(ff_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bar = reinterpret_cast<uint64_t*>(sm + FF_OFF_BAR);
  uint64_t* q_full = bar;                  // [2] Q tile landed
  uint64_t* q_empty = q_full + 2;          // [2] Q copied into TMEM (8 softmax warps)
  uint64_t* qa_full = q_empty + 2;         // the TMEM Q operand is written (8 softmax warps)
  uint64_t* st_full = qa_full + 1;         // [FF_NST]
  uint64_t* st_empty = st_full + FF_NST;   // [FF_NST]
  uint64_t* s_full = st_empty + FF_NST;    // [group][2]
  uint64_t* s_empty = s_full + 4;          // [group][2] (the group's 4 warps)
  uint64_t* p_full = s_empty + 4;          // [group] (4 warps)
  uint64_t* o_done = p_full + 2;           // [group] P V product complete
  uint64_t* x_full = o_done + 2;           // (m, l) of both groups written (8 warps), once per item
  uint64_t* o_read = x_full + 1;           // both groups have read O_0 and O_1 (8 warps), once per item
  uint64_t* out_full = o_read + 1;         // output tile staged (8 warps)
  uint64_t* out_free = out_full + 1;       // the previous item's TMA store has read the staging
  uint64_t* drain = out_free + 1;          // [2]: one per MMA thread (abort path)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 2);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(drain + 3);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int C = NH * 64;
  const int nqb = (T + FA_BM - 1) / FA_BM;
  const int nitems = nqb * BH;  // item w: query block nqb - 1 - w / BH, bh = w % BH
  const uint64_t lim = timeout_ns;

  if (threadIdx.x == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(&q_full[i], 1);
      mbar_init(&q_empty[i], 8);
      mbar_init(&p_full[i], 4);
      mbar_init(&o_done[i], 1);
      mbar_init(&drain[i], 1);
    }
    mbar_init(qa_full, 8);
    for (int i = 0; i < FF_NST; ++i) {
      mbar_init(&st_full[i], 1);
      mbar_init(&st_empty[i], 1);
    }
    for (int i = 0; i < 4; ++i) {
      mbar_init(&s_full[i], 1);
      mbar_init(&s_empty[i], 4);
    }
    mbar_init(x_full, 8);
    mbar_init(o_read, 8);
    mbar_init(out_full, 8);
    mbar_init(out_free, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, FF_TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      // ---------------- producer: Q per item, (K_u, V_u) per unit ----------------
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_kv64);
      bool ok = true;
      uint32_t q_iss = 0, q_par = 0, st_iss = 0, st_par = 0;
      int U = 0;
      for (int it = 0, item = blockIdx.x; item < nitems && ok; ++it, item += gridDim.x) {
        const int qb = nqb - 1 - item / BH, bh = item % BH, b = bh / NH, h = bh - b * NH;
        const int qbuf = it & 1;
        if (!mbar_wait_bounded(&q_empty[qbuf], ((it >> 1) & 1) ^ 1, abort_flag, lim)) {
          ok = false;
          break;
        }
        mbar_arrive_expect_tx(&q_full[qbuf], FA_TILE);
        tma_load_3d(sm + FF_OFF_Q + qbuf * FA_TILE, &tm_q, &q_full[qbuf], h * 64, qb * FA_BM, b);
        q_iss |= 1u << qbuf;
        q_par = (q_par & ~(1u << qbuf)) | ((uint32_t)((it >> 1) & 1) << qbuf);
        for (int k0 = 0; k0 < (qb + 1) * FA_BN; k0 += 64, ++U) {
          const int s = U % FF_NST;
          const uint32_t ph = (uint32_t)((U / FF_NST) & 1);
          if (!mbar_wait_bounded(&st_empty[s], ph ^ 1, abort_flag, lim)) {
            ok = false;
            break;
          }
          uint8_t* d = sm + FF_OFF_ST + s * FB_UNIT;
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
          if ((q_iss >> i) & 1u)
            mbar_wait_bounded(&q_full[i], (q_par >> i) & 1u, reinterpret_cast<volatile int*>(&never), lim);
        for (int i = 0; i < FF_NST; ++i)
          if ((st_iss >> i) & 1u)
            mbar_wait_bounded(&st_full[i], (st_par >> i) & 1u, reinterpret_cast<volatile int*>(&never), lim);
      }
    }
  } else if (warp == 1 || warp == 2) {
    if (lane == 0) {
      // ---------------- MMAs: S_u = Q K_u^T (warp 1); O_g += P_u V_u (warp 2) ----------------
      const bool is_s = warp == 1;
      constexpr uint32_t idesc_s = make_idesc_bf16(128, 64, false, false);
      constexpr uint32_t idesc_o = make_idesc_bf16(128, 64, false, true);  // B = V_u, MN-major
      bool ok = true, any = false;
      int U = 0;  // unit counter over all items; unit U belongs to group U % 2 (items have even unit counts)
      for (int it = 0, item = blockIdx.x; item < nitems && ok; ++it, item += gridDim.x) {
        const int nu = 2 * (nqb - item / BH);
        if (is_s && !mbar_wait_bounded(qa_full, it & 1, abort_flag, lim)) {
          ok = false;
          break;
        }
        for (int u = 0; u < nu; ++u, ++U) {
          const int s = U % FF_NST, g = U & 1, Ug = U >> 1;  // Ug: the unit's index within its group
          if (!mbar_wait_bounded(&st_full[s], (U / FF_NST) & 1, abort_flag, lim)) {
            ok = false;
            break;
          }
          const uint32_t k_addr = smem_u32(sm + FF_OFF_ST + s * FB_UNIT), v_addr = k_addr + FB_HALF;
          if (is_s) {
            const int sg = g * 2 + (Ug & 1);
            if (!mbar_wait_bounded(&s_empty[sg], ((Ug >> 1) & 1) ^ 1, abort_flag, lim)) {
              ok = false;
              break;
            }
            tc_fence_after();
#pragma unroll
            for (int k = 0; k < 4; ++k)
              umma_bf16_ts(tmem + sg * 64, tmem + FF_TM_Q + k * 8, make_sw128_desc(k_addr + k * 32, 16, 1024), idesc_s,
                           k > 0 ? 1u : 0u);
            umma_commit(&s_full[sg]);
          } else {
            if (!mbar_wait_bounded(&p_full[g], Ug & 1, abort_flag, lim)) {
              ok = false;
              break;
            }
            tc_fence_after();
            // K = 64 keys: B = 16 key rows of V_u per step (MN-major); each group's first unit
            // of an item starts its accumulator
#pragma unroll
            for (int k = 0; k < 4; ++k)
              umma_bf16_ts(tmem + FF_TM_O + g * 64, tmem + FF_TM_P + g * 32 + k * 8,
                           make_sw128_desc(v_addr + k * 2048, 8192, 1024), idesc_o, (u >= 2 || k > 0) ? 1u : 0u);
            umma_commit(&o_done[g]);
            umma_commit(&st_empty[s]);  // the unit's S MMAs completed before its P was written
          }
          any = true;
        }
      }
      if (!ok) {
        raise_device_error(err, DEV_TIMEOUT);
        *abort_flag = 1;
        if (any) {
          int never = 0;
          umma_commit(&drain[warp - 1]);
          mbar_wait_bounded(&drain[warp - 1], 0, reinterpret_cast<volatile int*>(&never), lim);
        }
      }
    }
  } else {
    // ---------------- softmax: group g, query row r ----------------
    const int g = (warp - 3) >> 2, q4 = warp & 3;
    const int r = q4 * 32 + lane;
    const uint32_t lane_off = (uint32_t)(q4 * 32) << 16;
    const float sl2 = scale * LOG2E;
    const bool issuer = (warp == 3 && lane == 0);  // issues the output tile's TMA store
    float* xb = reinterpret_cast<float*>(sm + FF_OFF_X);  // [item parity][group][row] x (m, l)
    bool fail = false;
    // the Q rows of item `it` into the TMEM A operand: this group copies head dims [g*32, g*32 + 32)
    auto load_q = [&](int it) -> bool {
      const int qbuf = it & 1;
      if (!fb_warp_wait(&q_full[qbuf], (it >> 1) & 1, abort_flag, lim, lane)) return false;
      const uint8_t* qt = sm + FF_OFF_Q + qbuf * FA_TILE;
      fb_row_to_tmem(qt, r, 2 * g, tmem + lane_off + FF_TM_Q + (2 * g) * 8);
      fb_row_to_tmem(qt, r, 2 * g + 1, tmem + lane_off + FF_TM_Q + (2 * g + 1) * 8);
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(qa_full);
        mbar_arrive(&q_empty[qbuf]);
      }
      return true;
    };
    if ((int)blockIdx.x < nitems) fail = !load_q(0);
    int U0 = 0;  // first global unit of the current item
    for (int it = 0, item = blockIdx.x; item < nitems && !fail; ++it, item += gridDim.x) {
      const int qb = nqb - 1 - item / BH, bh = item % BH, b = bh / NH, h = bh - b * NH;
      const int nu = 2 * (qb + 1);
      float m_run = -INFINITY, l_run = 0.f;
      for (int u = g; u < nu; u += 2) {
        const int U = U0 + u, Ug = U >> 1, sg = g * 2 + (Ug & 1);
        if (!fb_warp_wait(&s_full[sg], (Ug >> 1) & 1, abort_flag, lim, lane)) {
          fail = true;
          break;
        }
        tc_fence_after();
        uint32_t sv[64];
        tmem_ld_32x32b_x32(tmem + lane_off + (uint32_t)(sg * 64), *reinterpret_cast<uint32_t(*)[32]>(&sv[0]));
        tmem_ld_32x32b_x32(tmem + lane_off + (uint32_t)(sg * 64 + 32), *reinterpret_cast<uint32_t(*)[32]>(&sv[32]));
        tmem_ld_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&s_empty[sg]);
        if (u >= nu - 2) {  // the diagonal key block: keys after the query get -inf
          const int kbase = (u & 1) * 64;
#pragma unroll
          for (int e = 0; e < 64; ++e)
            if (kbase + e > r) sv[e] = __float_as_uint(-INFINITY);
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
        const float m_blk = mx * sl2;
        // re-base only when the block maximum exceeds the reference by more than FF_REBASE
        const bool rebase = m_blk > m_run + FF_REBASE;
        const float m_use = rebase ? m_blk : m_run;
        const float m_ref = m_use == -INFINITY ? 0.f : m_use;  // fully masked so far: P = 0
        float rs8[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
        uint32_t pw[32];
#pragma unroll
        for (int e2 = 0; e2 < 32; ++e2) {
          const float p0 = ex2_fast(fmaf(__uint_as_float(sv[2 * e2]), sl2, -m_ref));
          const float p1 = ex2_fast(fmaf(__uint_as_float(sv[2 * e2 + 1]), sl2, -m_ref));
          rs8[(2 * e2) & 7] += p0;
          rs8[(2 * e2 + 1) & 7] += p1;
          pw[e2] = pack_bf16x2(p0, p1);
        }
        const float rs = ((rs8[0] + rs8[1]) + (rs8[2] + rs8[3])) + ((rs8[4] + rs8[5]) + (rs8[6] + rs8[7]));
        // the group's previous P V product has finished reading P_g (and updating O_g)
        if (Ug > 0 && !fb_warp_wait(&o_done[g], (Ug - 1) & 1, abort_flag, lim, lane)) {
          fail = true;
          break;
        }
        tc_fence_after();
        // rescale rows of O_g to their new reference. tcgen05.ld / st are warp-collective
        // (.sync.aligned), so the whole warp takes this path when any of its rows re-bases;
        // the other rows use the factor 1.
        const bool my_rescale = rebase && m_run != -INFINITY;
        if (__any_sync(0xffffffffu, my_rescale)) {
          const float corr = my_rescale ? ex2_fast(m_run - m_use) : 1.0f;
          uint32_t ov[32];
#pragma unroll
          for (int hh = 0; hh < 2; ++hh) {
            tmem_ld_32x32b_x32(tmem + lane_off + FF_TM_O + g * 64 + hh * 32, ov);
            tmem_ld_wait();
            uint32_t a[16], c[16];
#pragma unroll
            for (int e = 0; e < 16; ++e) {
              a[e] = __float_as_uint(__uint_as_float(ov[e]) * corr);
              c[e] = __float_as_uint(__uint_as_float(ov[16 + e]) * corr);
            }
            tmem_st_32x32b_x16(tmem + lane_off + FF_TM_O + g * 64 + hh * 32, a);
            tmem_st_32x32b_x16(tmem + lane_off + FF_TM_O + g * 64 + hh * 32 + 16, c);
          }
          l_run *= corr;
        }
        l_run += rs;
        m_run = m_use;
        // the first unit of an item (after the first item) starts a fresh O_g: both groups
        // must have read the previous item's accumulators
        if (u < 2 && it > 0 && !fb_warp_wait(o_read, (it - 1) & 1, abort_flag, lim, lane)) {
          fail = true;
          break;
        }
        tmem_st_32x32b_x16(tmem + lane_off + FF_TM_P + g * 32, *reinterpret_cast<uint32_t(*)[16]>(&pw[0]));
        tmem_st_32x32b_x16(tmem + lane_off + FF_TM_P + g * 32 + 16, *reinterpret_cast<uint32_t(*)[16]>(&pw[16]));
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&p_full[g]);
      }
      if (fail) break;
      // the other group's last S product of this item is complete too: then no MMA
      // still reads the TMEM Q operand, and the next item's Q can be written
      {
        const int uo = nu - 1 - g, Uo = U0 + uo, Ugo = Uo >> 1;
        if (!fb_warp_wait(&s_full[(1 - g) * 2 + (Ugo & 1)], (Ugo >> 1) & 1, abort_flag, lim, lane)) {
          fail = true;
          break;
        }
      }
      if (item + (int)gridDim.x < nitems && !load_q(it + 1)) {
        fail = true;
        break;
      }
      // merge the two groups' rows
      float* xm = xb + ((it & 1) * 2 + g) * 256;
      xm[r] = m_run;
      xm[128 + r] = l_run;
      __syncwarp();
      if (lane == 0) mbar_arrive(x_full);
      // both groups' last P V products complete
      const int Ug_last = (U0 + nu - 2 + g) >> 1, Ugo_last = (U0 + nu - 1 - g) >> 1;
      if (!fb_warp_wait(x_full, it & 1, abort_flag, lim, lane) ||
          !fb_warp_wait(&o_done[g], Ug_last & 1, abort_flag, lim, lane) ||
          !fb_warp_wait(&o_done[1 - g], Ugo_last & 1, abort_flag, lim, lane)) {
        fail = true;
        break;
      }
      const float* xo = xb + ((it & 1) * 2 + (1 - g)) * 256;
      const float m_o = xo[r], l_o = xo[128 + r];
      const float m = fmaxf(m_run, m_o);
      const float a_s = m_run == -INFINITY ? 0.f : ex2_fast(m_run - m);
      const float a_o = m_o == -INFINITY ? 0.f : ex2_fast(m_o - m);
      const float l = l_run * a_s + l_o * a_o;
      const float inv = 1.0f / l;
      const float a0 = (g == 0 ? a_s : a_o) * inv, a1 = (g == 0 ? a_o : a_s) * inv;
      // this thread's output columns [g*32, g*32 + 32) from O_0 and O_1
      tc_fence_after();
      uint32_t o0[32], o1[32];
      tmem_ld_32x32b_x32(tmem + lane_off + FF_TM_O + g * 32, o0);
      tmem_ld_32x32b_x32(tmem + lane_off + FF_TM_O + 64 + g * 32, o1);
      tmem_ld_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(o_read);
      const int qrow = qb * FA_BM + r;
      if (g == 0 && qrow < T) lse[(long long)bh * T + qrow] = (m + __log2f(l)) * LN2;
      if (issuer && it > 0) {
        bulk_wait_read<0>();
        mbar_arrive(out_free);
      }
      if (!fb_warp_wait(out_free, (it & 1) ^ 1, abort_flag, lim, lane)) {
        fail = true;
        break;
      }
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        float f[16];
#pragma unroll
        for (int e = 0; e < 16; ++e)
          f[e] = __uint_as_float(o0[hh * 16 + e]) * a0 + __uint_as_float(o1[hh * 16 + e]) * a1;
        fb_store16(sm + FF_OFF_OUT, r, g * 4 + hh * 2, f);
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(out_full);
      if (issuer) {
        if (mbar_wait_bounded(out_full, it & 1, abort_flag, lim)) {
          tma_store_3d(&tm_out, sm + FF_OFF_OUT, h * 64, qb * FA_BM, b);
          bulk_commit();
        } else {
          fail = true;
        }
      }
      if (__shfl_sync(0xffffffffu, fail ? 1 : 0, 0)) {  // the issuer's warp leaves together
        fail = true;
        break;
      }
      U0 += nu;
    }
    if (issuer) bulk_wait_all();
    if (fail && lane == 0) {
      raise_device_error(err, DEV_TIMEOUT);
      *abort_flag = 1;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, FF_TMEM_COLS);
  }
}

}  // namespace g2
