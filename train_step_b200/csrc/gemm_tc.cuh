// gemm_tc.cuh -- bf16 tensor-core GEMM for sm_100a (tcgen05 + TMEM + TMA).
//
// D[M, N] = sum_k A(m, k) * B(n, k), fp32 accumulate, fused epilogue.
// Every Linear of the pre-LN block and the tied/untied lm_head runs here
// ("gpt/docs/LLM.md", Architecture Details; "GPT From Scratch", Key decisions):
//   forward  Y  = X W^T         A = X  (K-major),   B = W  (K-major)
//   backward dX = dY W          A = dY (K-major),   B = W  (MN-major)
//   backward dW += dY^T X       A = dY (MN-major),  B = X  (MN-major)
//
// Design: one persistent CTA per SM (1 CTA/SM by shared memory), warp-specialised.
//   warp 0      TMA producer: 128-byte-swizzled tiles into a STAGES-deep ring
//   warp 1      one thread issues tcgen05.mma (M=128, N=BN, K=16) into TMEM;
//               the warp also owns the TMEM allocation
//   warps 2..    epilogue (8 or 16 warps): tcgen05.ld 32 lanes x 32 columns, fused
//               bias / GELU / residual / GELU' math, TMA stores. Two TMEM accumulators
//               (2 x BN columns) let the epilogue of one tile overlap the main
//               loop of the next.
// No cluster multicast is used (tiles are fetched per CTA from L2).
// Every mbarrier wait is bounded: on timeout the kernel records DEV_TIMEOUT in the
// device error word, stops issuing work, drains its in-flight copies and MMAs with
// bounded waits, frees its TMEM and returns.
#pragma once
#include "common.cuh"

namespace g2 {

enum Epi : int {
  EPI_BF16 = 0,        // out(bf16)  = acc + bias
  EPI_BF16_GELU = 1,   // out(bf16)  = u = acc + bias ; out2(bf16) = gelu(u)
  EPI_F32_RESID = 2,   // out(f32)   = aux(f32) + acc + bias
  EPI_BF16_DGELU = 3,  // out(bf16)  = acc * gelu'(aux(bf16))
  EPI_F32 = 4,         // out(f32)   = acc (+ out when accumulate)
};

struct GemmParams {
  int M, N, K;
  int tiles_m, tiles_n;
  int ksplit, kb_per_split, num_kb;
  int num_units;
  void* out;
  long long ldo;
  void* out2;
  long long ldo2;
  const float* bias;
  const void* aux;
  long long ld_aux;
  int accumulate;
  float* partial;  // split-K workspace [ksplit][M][N] fp32, used when ksplit > 1
  float* colsum;   // EPI_BF16_DGELU (nullable): column sums of the output per 32-row block, [ceil(M/32)][N]
  float2* rowstats;  // EPI_BF16 (nullable): per row and half tile, (max, sum of exp(z - max)) of the bf16
                     // outputs in columns < stats_ncols, [M][2 * tiles_n]
  int stats_ncols;
  int* err;
  unsigned long long timeout_ns;
};

constexpr int TC_BM = 128;
constexpr int TC_BK = 64;
// Epilogue warps: 8 (two per TMEM lane quarter, each draining half of the tile's columns),
// or 16 where that measured faster on B200: the residual add (fp32 in and out, latency-bound
// on its chunk chain; 16384 x 768 x 768: 39.1 -> 36.3 us) and GELU with two outputs (81.9 ->
// 79.8 us). GELU backward with the bias column sums is issue-bound and lost with 16 (88.6 ->
// 95.5 us), so it keeps 8.
template <int EPI>
__host__ __device__ constexpr int tc_epi_warps() {
  return (EPI == EPI_BF16_GELU || EPI == EPI_F32_RESID) ? 16 : 8;
}

// PAIR: a 2-CTA cluster computes one (2 * TC_BM) x BN tile with M = 256 MMAs that
// span both SMs' tensor cores. Each CTA stages its own 128 rows of A and its own
// BN / 2 rows of B, so a CTA moves 2/3 of the shared-memory and L2 bytes per FLOP
// that the single-CTA form (128 rows of A, BN rows of B) does.
// AUX: the epilogue reads an auxiliary tile (residual or GELU input) per chunk; it gets
// four 2 KB chunk buffers per epilogue warp so that the auxiliary tile of chunk n + 3 is
// in flight while chunk n is computed (one chunk of lookahead left the epilogue waiting
// on every load), at the price of one main-loop stage.
template <int BN, bool PAIR = false, bool AUX = false, int EPW = 8>
struct TcCfg {
  static constexpr int THREADS = (2 + EPW) * 32;
  static constexpr int A_BYTES = TC_BM * TC_BK * 2;
  static constexpr int B_ROWS = PAIR ? BN / 2 : BN;  // B rows staged by one CTA
  static constexpr int B_BYTES = B_ROWS * TC_BK * 2;
  static constexpr int UNIT_M = PAIR ? 2 * TC_BM : TC_BM;
  static constexpr int STAGE = A_BYTES + B_BYTES;
  // 2 KB chunk buffers per epilogue warp: with 8 warps an auxiliary tile gets 3 chunks of
  // lookahead; 16 warps keep as many chunks in flight with one each
  static constexpr int NBUF = (AUX && EPW == 8) ? 4 : 2;
  static constexpr int STAGING = EPW * NBUF * 2048;
  static constexpr int BARS = 512;                           // mbarriers, TMEM slot, abort flag
  static constexpr int STAGES = (232448 - 1024 - BARS - STAGING) / STAGE;
  static_assert(8 * (2 * STAGES + 6 + NBUF * EPW) <= BARS, "barrier space");
  static constexpr int TMEM_COLS = 2 * BN <= 256 ? 256 : 512;
  static constexpr int SMEM = STAGES * STAGE + STAGING + 1024 + BARS;
};

// tanh-GELU and its derivative on a PAIR of values with the packed fp32 instructions of
// sm_100 (f2_fma / f2_mul, common.cuh), t = u^2
// shared, constants folded (k = sqrt(2/pi), c = 0.044715, z = u (k + k c t)):
//   gelu(u)  = h + h tanh(z),  h = u / 2
//   gelu'(u) = (1 + tanh z) / 2 + u (1 - tanh^2 z) (k + 3 k c t) / 2
__device__ __forceinline__ float tanh_approx(float z) {
  float th;
  asm("tanh.approx.f32 %0, %1;" : "=f"(th) : "f"(z));
  return th;
}
constexpr float GELU_K = 0.7978845608028654f, GELU_KC = 0.7978845608028654f * 0.044715f;
// tanh(z) of both lanes of Z
__device__ __forceinline__ uint64_t f2_tanh(uint64_t Z) {
  const float2 z = f2_unpack(Z);
  return f2_pack(tanh_approx(z.x), tanh_approx(z.y));
}
__device__ __forceinline__ float2 gelu2_fast(float u0, float u1) {
  const uint64_t U = f2_pack(u0, u1);
  const uint64_t T = f2_mul(U, U);
  const uint64_t TH = f2_tanh(f2_mul(U, f2_fma(T, f2_pack(GELU_KC, GELU_KC), f2_pack(GELU_K, GELU_K))));
  const uint64_t H = f2_mul(U, f2_pack(0.5f, 0.5f));
  return f2_unpack(f2_fma(H, TH, H));
}
// g * gelu'(u) for both lanes (g: the incoming gradient)
__device__ __forceinline__ float2 gelu_grad2_mul(float u0, float u1, float g0, float g1) {
  const uint64_t U = f2_pack(u0, u1);
  const uint64_t T = f2_mul(U, U);
  const uint64_t TH = f2_tanh(f2_mul(U, f2_fma(T, f2_pack(GELU_KC, GELU_KC), f2_pack(GELU_K, GELU_K))));
  const uint64_t A = f2_fma(TH, f2_pack(0.5f, 0.5f), f2_pack(0.5f, 0.5f));             // (1 + th) / 2
  const uint64_t NB = f2_fma(TH, TH, f2_pack(-1.0f, -1.0f));                           // th^2 - 1
  const uint64_t NW = f2_mul(U, f2_fma(T, f2_pack(-1.5f * GELU_KC, -1.5f * GELU_KC),
                                       f2_pack(-0.5f * GELU_K, -0.5f * GELU_K)));     // -u dz/2
  const uint64_t GP = f2_fma(NW, NB, A);                                               // gelu'(u)
  return f2_unpack(f2_mul(GP, f2_pack(g0, g1)));
}

// Epilogue chunks: each epilogue warp turns 32 accumulator rows (one per lane) into
// one 2 KB output tile at a time, staged in shared memory in exactly the layout
// of the output tensor map's box:
//   "row64": 64-byte rows (16 fp32 or 32 bf16 columns), 64-byte swizzle: 16-byte
//            piece k of row r sits at piece k ^ ((r >> 1) & 3)
// It puts the 8 lanes of a 16-byte access phase in distinct banks. When the
// epilogue reads an auxiliary tile (the residual, or the pre-GELU input), TMA
// loads it into the same buffer beforehand and the result overwrites it in place.
template <int EPI>
__host__ __device__ constexpr int tc_chunk_cols() {
  return (EPI == EPI_BF16 || EPI == EPI_BF16_DGELU || EPI == EPI_BF16_GELU) ? 32 : 16;
}
// GELU writes two 2 KB outputs per chunk: one 4 KB buffer per warp, no alternation
template <int EPI>
__host__ __device__ constexpr bool tc_single_buffer() {
  return EPI == EPI_BF16_GELU;
}
template <int EPI>
__host__ __device__ constexpr bool tc_has_aux() {
  return EPI == EPI_F32_RESID || EPI == EPI_BF16_DGELU;
}
__device__ __forceinline__ uint8_t* row64_at(uint8_t* buf, int r, int k) {
  return buf + r * 64 + ((k ^ ((r >> 1) & 3)) << 4);
}
template <int EPI, int CW>
__device__ __forceinline__ void tc_epilogue_chunk(const GemmParams& p, int col0, int lane, float (&v)[CW],
                                                  uint8_t* buf) {
  const bool full = (col0 + CW <= p.N);
  if (p.ksplit > 1 || EPI == EPI_F32) {  // fp32, 16 columns, row64
#pragma unroll
    for (int k = 0; k < 4; ++k)
      *reinterpret_cast<float4*>(row64_at(buf, lane, k)) = make_float4(v[4 * k], v[4 * k + 1], v[4 * k + 2], v[4 * k + 3]);
    return;
  }
  if (EPI == EPI_BF16 || EPI == EPI_BF16_GELU || EPI == EPI_F32_RESID) {
    if (p.bias) {
      if (full) {
#pragma unroll
        for (int j = 0; j < CW; j += 4) {
          float4 b = __ldg(reinterpret_cast<const float4*>(p.bias + col0 + j));
          v[j] += b.x;
          v[j + 1] += b.y;
          v[j + 2] += b.z;
          v[j + 3] += b.w;
        }
      } else {
#pragma unroll
        for (int j = 0; j < CW; ++j)
          if (col0 + j < p.N) v[j] += p.bias[col0 + j];
      }
    }
  }
  if (EPI == EPI_F32_RESID) {  // fp32, 16 columns: out = residual (staged by TMA) + acc + bias
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      float4* q = reinterpret_cast<float4*>(row64_at(buf, lane, k));
      const float4 x = *q;
      *q = make_float4(x.x + v[4 * k], x.y + v[4 * k + 1], x.z + v[4 * k + 2], x.w + v[4 * k + 3]);
    }
  } else if (EPI == EPI_BF16) {  // bf16, 32 columns, row64
#pragma unroll
    for (int k = 0; k < 4; ++k)
      *reinterpret_cast<uint4*>(row64_at(buf, lane, k)) =
          make_uint4(pack_bf16x2(v[8 * k], v[8 * k + 1]), pack_bf16x2(v[8 * k + 2], v[8 * k + 3]),
                     pack_bf16x2(v[8 * k + 4], v[8 * k + 5]), pack_bf16x2(v[8 * k + 6], v[8 * k + 7]));
  } else if (EPI == EPI_BF16_DGELU) {  // bf16, 32 columns: out = acc * gelu'(u), u staged by TMA
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      uint4* q = reinterpret_cast<uint4*>(row64_at(buf, lane, k));
      const uint4 uu = *q;
      const uint32_t w[4] = {uu.x, uu.y, uu.z, uu.w};
      uint32_t o[4];
#pragma unroll
      for (int t = 0; t < 4; ++t) {
        const float2 f = unpack_bf16x2(w[t]);
        const float2 d = gelu_grad2_mul(f.x, f.y, v[8 * k + 2 * t], v[8 * k + 2 * t + 1]);
        v[8 * k + 2 * t] = d.x;  // kept in v for the column sums
        v[8 * k + 2 * t + 1] = d.y;
        o[t] = pack_bf16x2(d.x, d.y);
      }
      *q = make_uint4(o[0], o[1], o[2], o[3]);
    }
  } else if (EPI == EPI_BF16_GELU) {  // bf16, 32 columns: u at buf, gelu(u) at buf + 2 KB, row64
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      *reinterpret_cast<uint4*>(row64_at(buf, lane, k)) =
          make_uint4(pack_bf16x2(v[8 * k], v[8 * k + 1]), pack_bf16x2(v[8 * k + 2], v[8 * k + 3]),
                     pack_bf16x2(v[8 * k + 4], v[8 * k + 5]), pack_bf16x2(v[8 * k + 6], v[8 * k + 7]));
    }
#pragma unroll
    for (int j = 0; j < CW; j += 2) {
      const float2 gg = gelu2_fast(v[j], v[j + 1]);
      v[j] = gg.x;
      v[j + 1] = gg.y;
    }
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      *reinterpret_cast<uint4*>(row64_at(buf + 2048, lane, k)) =
          make_uint4(pack_bf16x2(v[8 * k], v[8 * k + 1]), pack_bf16x2(v[8 * k + 2], v[8 * k + 3]),
                     pack_bf16x2(v[8 * k + 4], v[8 * k + 5]), pack_bf16x2(v[8 * k + 6], v[8 * k + 7]));
    }
  }
}

// Column sums of a 32 x 32 block held one row per lane (v[j] = column j of the lane's
// row): after the exchange lane j holds the sum of column j over the 32 rows. Each
// stage halves the columns a lane keeps and adds its partner's half; the summation
// order is fixed, so the result is the same on every run.
__device__ __forceinline__ float warp_colsum32(float (&v)[32], int lane) {
#pragma unroll
  for (int w = 16; w >= 1; w >>= 1) {
    const bool upper = (lane & w) != 0;
#pragma unroll
    for (int j = 0; j < w; ++j) {
      const float send = upper ? v[j] : v[j + w];
      const float keep = upper ? v[j + w] : v[j];
      v[j] = keep + __shfl_xor_sync(0xffffffffu, send, w);
    }
  }
  return v[0];
}

__device__ __forceinline__ void tc_decode_unit(const GemmParams& p, int unit, int& tm, int& tn, int& ks) {
  const int per_split = p.tiles_m * p.tiles_n;
  ks = unit / per_split;
  const int t = unit - ks * per_split;
  tm = t / p.tiles_n;
  tn = t - tm * p.tiles_n;
}

// PAIR = true runs as clusters of two CTAs (launch attribute cluster dim 2 x 1 x 1):
// rank 0 (the leader) issues the M = 256 MMAs for both; both ranks load their halves
// of each stage, completing on the leader's `full` barrier; the leader's commits
// arrive on both ranks' `empty` / `tfull` barriers; both ranks' epilogue warps
// arrive on the leader's `tempty`. No load is multicast.
template <int BN, bool A_MN, bool B_MN, int EPI, bool PAIR>
__global__ void __launch_bounds__((2 + tc_epi_warps<EPI>()) * 32, 1)
    gemm_tc_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                   const __grid_constant__ CUtensorMap tmO, const __grid_constant__ CUtensorMap tmO2,
                   const GemmParams p) {
  constexpr int EPW = tc_epi_warps<EPI>();
  using Cfg = TcCfg<BN, PAIR, tc_has_aux<EPI>(), EPW>;
  constexpr int STAGES = Cfg::STAGES;
  constexpr int UNIT_M = Cfg::UNIT_M;
  const uint32_t rank = PAIR ? cluster_ctarank() : 0u;
  const int cid = PAIR ? (int)(blockIdx.x >> 1) : (int)blockIdx.x;  // cluster (or CTA) index
  const int ncl = PAIR ? (int)(gridDim.x >> 1) : (int)gridDim.x;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* staging = smem + STAGES * Cfg::STAGE;  // 1024-aligned
  uint64_t* full = reinterpret_cast<uint64_t*>(staging + Cfg::STAGING);
  uint64_t* empty = full + STAGES;
  uint64_t* tfull = empty + STAGES;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  uint64_t* auxbar = drain + 2;  // [EPW][NBUF]: auxiliary tile landed in chunk buffer b

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  pdl_launch_dependents();  // the next kernel may start its own set-up once every CTA is running

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], PAIR ? 2 * EPW : EPW);
    }
    mbar_init(drain, 1);
    for (int i = 0; i < Cfg::NBUF * EPW; ++i) mbar_init(&auxbar[i], 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
  }
  if (warp == 1) {
    if (PAIR) {
      tmem_alloc_pair(tmem_slot, Cfg::TMEM_COLS);
      tmem_relinquish_pair();
    } else {
      tmem_alloc(tmem_slot, Cfg::TMEM_COLS);
      tmem_relinquish();
    }
  }
  tc_fence_before();
  if (PAIR)
    cluster_sync();  // the peer's barriers are initialised before anything arrives on them
  else
    __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  // launched as a programmatic dependent (training step): the set-up above overlapped the
  // previous kernel's tail; nothing in global memory is touched before this wait (a no-op
  // for an ordinary launch)
  pdl_wait();
  const uint64_t lim = p.timeout_ns;

  if (warp == 0) {
    if (lane == 0) {
      // ---------------- TMA producer ----------------
      int stage = 0;
      uint32_t phase = 0;
      uint32_t issued = 0, last_par = 0;  // bit s: stage s has a copy issued / its parity
      bool ok = true;
      for (int unit = cid; unit < p.num_units && ok; unit += ncl) {
        int tm, tn, ks;
        tc_decode_unit(p, unit, tm, tn, ks);
        const int kb0 = ks * p.kb_per_split;
        const int kb1 = min(kb0 + p.kb_per_split, p.num_kb);
        const int arow = tm * UNIT_M + (int)rank * TC_BM;        // this CTA's rows of A
        const int brow = tn * BN + (int)rank * Cfg::B_ROWS;      // this CTA's rows of B
        for (int kb = kb0; kb < kb1; ++kb) {
          if (!mbar_wait_bounded(&empty[stage], phase ^ 1, abort_flag, lim)) {
            ok = false;
            break;
          }
          // the leader expects both CTAs' bytes; the peer's copies complete on the leader's barrier
          if (rank == 0) mbar_arrive_expect_tx(&full[stage], PAIR ? 2 * Cfg::STAGE : Cfg::STAGE);
          uint8_t* sa = smem + stage * Cfg::STAGE;
          uint8_t* sb = sa + Cfg::A_BYTES;
          const int kx = kb * TC_BK;
          if (PAIR) {
            const uint32_t fb = cluster_addr(&full[stage], 0);
            if (!A_MN) {
              tma_load_2d_pair(sa, &tmA, fb, kx, arow);
            } else {
              tma_load_2d_pair(sa, &tmA, fb, arow, kx);
              tma_load_2d_pair(sa + 8192, &tmA, fb, arow + 64, kx);
            }
            if (!B_MN) {
              tma_load_2d_pair(sb, &tmB, fb, kx, brow);
            } else {
#pragma unroll
              for (int j = 0; j < Cfg::B_ROWS / 64; ++j) tma_load_2d_pair(sb + j * 8192, &tmB, fb, brow + j * 64, kx);
            }
          } else {
            if (!A_MN) {
              tma_load_2d(sa, &tmA, &full[stage], kx, arow);
            } else {
              tma_load_2d(sa, &tmA, &full[stage], arow, kx);
              tma_load_2d(sa + 8192, &tmA, &full[stage], arow + 64, kx);
            }
            if (!B_MN) {
              tma_load_2d(sb, &tmB, &full[stage], kx, brow);
            } else {
#pragma unroll
              for (int j = 0; j < Cfg::B_ROWS / 64; ++j) tma_load_2d(sb + j * 8192, &tmB, &full[stage], brow + j * 64, kx);
            }
          }
          issued |= 1u << stage;
          last_par = (last_par & ~(1u << stage)) | (phase << stage);
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1;
          }
        }
      }
      if (!ok) {
        raise_device_error(p.err, DEV_TIMEOUT);
        *abort_flag = 1;
        // let every copy already issued land before the CTA's shared memory goes away
        int never = 0;
        if (rank == 0) {
          for (int s = 0; s < STAGES; ++s)
            if ((issued >> s) & 1u)
              mbar_wait_bounded(&full[s], (last_par >> s) & 1u, reinterpret_cast<volatile int*>(&never), lim);
        } else if (issued) {
          // the peer's copies complete on the leader's barriers, which it cannot wait on:
          // give them a fixed grace period (a tile copy lands in microseconds)
          spin_for_ns(2000000ull);
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0 && rank == 0) {
      // ---------------- MMA issuer (the leader alone, for a pair) ----------------
      constexpr uint32_t idesc = make_idesc_bf16(UNIT_M, BN, A_MN, B_MN);
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool ok = true, any = false;
      for (int unit = cid; unit < p.num_units && ok; unit += ncl) {
        int tm, tn, ks;
        tc_decode_unit(p, unit, tm, tn, ks);
        const int kb0 = ks * p.kb_per_split;
        const int kb1 = min(kb0 + p.kb_per_split, p.num_kb);
        if (!mbar_wait_bounded(&tempty[acc], acc_phase ^ 1, abort_flag, lim)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + (uint32_t)(acc * BN);
        for (int kb = kb0; kb < kb1; ++kb) {
          if (!mbar_wait_bounded(&full[stage], phase, abort_flag, lim)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a_addr = smem_u32(smem + stage * Cfg::STAGE);
          const uint32_t b_addr = a_addr + Cfg::A_BYTES;
#pragma unroll
          for (int k = 0; k < TC_BK / 16; ++k) {
            const uint64_t ad = A_MN ? make_sw128_desc(a_addr + k * 2048, 8192, 1024)
                                     : make_sw128_desc(a_addr + k * 32, 16, 1024);
            const uint64_t bd = B_MN ? make_sw128_desc(b_addr + k * 2048, 8192, 1024)
                                     : make_sw128_desc(b_addr + k * 32, 16, 1024);
            if (PAIR)
              umma_bf16_pair(d_tmem, ad, bd, idesc, (kb > kb0 || k > 0) ? 1u : 0u);
            else
              umma_bf16(d_tmem, ad, bd, idesc, (kb > kb0 || k > 0) ? 1u : 0u);
          }
          any = true;
          if (PAIR)
            umma_commit_pair_mc(&empty[stage], 0x3);  // frees the stage in both CTAs
          else
            umma_commit(&empty[stage]);
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1;
          }
        }
        if (!ok) break;
        if (PAIR)
          umma_commit_pair_mc(&tfull[acc], 0x3);
        else
          umma_commit(&tfull[acc]);
        acc ^= 1;
        if (acc == 0) acc_phase ^= 1;
      }
      if (!ok) {
        raise_device_error(p.err, DEV_TIMEOUT);
        *abort_flag = 1;
        if (any) {  // wait for the MMAs already issued before the TMEM is freed
          int never = 0;
          if (PAIR)
            umma_commit_pair(drain);
          else
            umma_commit(drain);
          mbar_wait_bounded(drain, 0, reinterpret_cast<volatile int*>(&never), lim);
        }
      }
    }
  } else {
    // ---------------- epilogue warps ----------------
    constexpr int CW = tc_chunk_cols<EPI>();
    constexpr bool HAS_AUX = tc_has_aux<EPI>();
    constexpr int NPART = EPW / 4;   // column parts of the tile (one warp per lane quarter each)
    const int ew = warp - 2;         // 0 .. EPW - 1
    const int q = warp & 3;          // TMEM lane quarter this warp may access
    const int part = ew >> 2;        // which part of the BN columns
    const int c_begin = part * (BN / NPART), c_end = (part + 1) * (BN / NPART);
    constexpr int NBUF = Cfg::NBUF;
    uint8_t* wbuf = staging + ew * (NBUF * 2048);  // chunk buffers: wbuf + b * 2048
    uint64_t* abar = auxbar + NBUF * ew;
    if (lane == 0) {
      if (EPI == EPI_BF16_GELU || p.ksplit > 1 || HAS_AUX) tma_prefetch_desc(&tmO2);
      tma_prefetch_desc(&tmO);
    }
    // auxiliary tiles (tmO2 is the auxiliary map for these epilogues): chunk g of this
    // warp's sequence goes to buffer g % NBUF, NBUF - 1 chunks ahead of the one computed;
    // lane 0 tracks the loads in flight (bit b: buffer b) for the abort path
    uint32_t aux_pending = 0, aux_par = 0;
    const int rbase = (int)rank * TC_BM + q * 32;  // this warp's first row within a unit
    constexpr int CPU_ = (BN / NPART) / CW;         // chunks per unit for this warp
    // issue the auxiliary load of this warp's chunk g (g counted over all its units)
    auto aux_load = [&](int g) {
      const int unit_g = cid + (g / CPU_) * ncl;
      if (unit_g >= p.num_units) return;
      int tmg, tng, ksg;
      tc_decode_unit(p, unit_g, tmg, tng, ksg);
      const int b = g % NBUF;
      mbar_arrive_expect_tx(&abar[b], 2048);
      tma_load_2d(wbuf + b * 2048, &tmO2, &abar[b], tng * BN + c_begin + (g % CPU_) * CW, tmg * UNIT_M + rbase);
      aux_pending |= 1u << b;
      aux_par = (aux_par & ~(1u << b)) | ((uint32_t)((g / NBUF) & 1) << b);
    };
    if (HAS_AUX && lane == 0)
      for (int g = 0; g < NBUF - 1; ++g) aux_load(g);
    int acc = 0;
    uint32_t acc_phase = 0;
    int n = 0;  // chunks processed by this warp
    bool ok = true;
    const bool stats = EPI == EPI_BF16 && p.rowstats != nullptr;
    for (int unit = cid; unit < p.num_units && ok; unit += ncl) {
      int tm, tn, ks;
      tc_decode_unit(p, unit, tm, tn, ks);
      float st_m = -INFINITY, st_s = 0.f;  // this lane's row over this warp's part of the tile
      if (!mbar_wait_bounded(&tfull[acc], acc_phase, abort_flag, lim)) {
        if (lane == 0) {
          raise_device_error(p.err, DEV_TIMEOUT);
          *abort_flag = 1;
        }
        break;
      }
      tc_fence_after();
      const int row0 = tm * UNIT_M + rbase;
#pragma unroll 1
      for (int c = c_begin; c < c_end; c += CW, ++n) {
        const int b = tc_single_buffer<EPI>() ? 0 : (n % NBUF);
        uint8_t* cur = wbuf + b * 2048;
        if (lane == 0) {
          if (HAS_AUX) {
            // nothing to wait for: the auxiliary tile of this chunk was requested NBUF - 1
            // chunks ago, into the buffer it is computed and stored from
          } else if (tc_single_buffer<EPI>()) {
            // GELU: u and gelu(u) go out as two bulk groups; the u half is free once the
            // previous chunk's u store has been read (its gelu store may still be reading)
            bulk_wait_read<1>();
          } else {
            bulk_wait_read<1>();  // this buffer's previous store (two chunks ago) has been read out
          }
        }
        __syncwarp();
        float v[CW];
        {
          uint32_t r[CW];
          if (CW == 32)
            tmem_ld_32x32b_x32(tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(acc * BN + c),
                               *reinterpret_cast<uint32_t(*)[32]>(&r[0]));
          else
            tmem_ld_32x32b_x16(tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(acc * BN + c),
                               *reinterpret_cast<uint32_t(*)[16]>(&r[0]));
          tmem_ld_wait();
#pragma unroll
          for (int j = 0; j < CW; ++j) v[j] = __uint_as_float(r[j]);
        }
        if (c + CW == c_end) {  // last read of this accumulator: hand it back to the MMA warp
          tc_fence_before();
          __syncwarp();
          if (lane == 0) {
            if (PAIR)
              mbar_arrive_cluster(cluster_addr(&tempty[acc], 0));
            else
              mbar_arrive(&tempty[acc]);
          }
        }
        if (HAS_AUX) {
          int got = 1;
          if (lane == 0) {
            got = mbar_wait_bounded(&abar[b], (n / NBUF) & 1, abort_flag, lim) ? 1 : 0;
            if (got) aux_pending &= ~(1u << b);
          }
          got = __shfl_sync(0xffffffffu, got, 0);
          if (!got) {
            if (lane == 0) {
              raise_device_error(p.err, DEV_TIMEOUT);
              *abort_flag = 1;
            }
            ok = false;
            break;
          }
          mbar_try_wait(&abar[b], (n / NBUF) & 1);  // every lane observes the completed phase
        }
        const int col0 = tn * BN + c;
        if (EPI == EPI_BF16_GELU) {
          // u = acc + bias into the first half, stored as its own group; gelu(u) into the
          // second half once the previous chunk's gelu store has read it
          if (col0 < p.N) tc_epilogue_chunk<EPI_BF16, CW>(p, col0, lane, v, cur);
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {
            if (col0 < p.N && row0 < p.M) tma_store_2d(&tmO, cur, col0, row0);
            bulk_commit();
            bulk_wait_read<1>();
          }
          __syncwarp();
          if (col0 < p.N) {
#pragma unroll
            for (int j = 0; j < CW; j += 2) {
              const float2 gg = gelu2_fast(v[j], v[j + 1]);
              v[j] = gg.x;
              v[j + 1] = gg.y;
            }
#pragma unroll
            for (int k = 0; k < 4; ++k)
              *reinterpret_cast<uint4*>(row64_at(cur + 2048, lane, k)) =
                  make_uint4(pack_bf16x2(v[8 * k], v[8 * k + 1]), pack_bf16x2(v[8 * k + 2], v[8 * k + 3]),
                             pack_bf16x2(v[8 * k + 4], v[8 * k + 5]), pack_bf16x2(v[8 * k + 6], v[8 * k + 7]));
          }
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {
            if (col0 < p.N && row0 < p.M) tma_store_2d(&tmO2, cur + 2048, col0, row0);
            bulk_commit();
          }
          continue;
        }
        if (col0 < p.N) tc_epilogue_chunk<EPI, CW>(p, col0, lane, v, cur);
        if (EPI == EPI_BF16 && stats) {
          // softmax statistics of the stored (bf16-rounded) values, for the cross-entropy
          // that reads them: running max and sum of exp(z - max) over columns < stats_ncols
          float cm = -INFINITY;
#pragma unroll
          for (int j = 0; j < CW; ++j) {
            v[j] = col0 + j < p.stats_ncols ? __bfloat162float(__float2bfloat16_rn(v[j])) : -INFINITY;
            cm = fmaxf(cm, v[j]);
          }
          const float nm = fmaxf(st_m, cm);
          if (nm != -INFINITY) {
            const float nm2 = nm * 1.4426950408889634f;
            float cs = 0.f;
#pragma unroll
            for (int j = 0; j < CW; ++j) cs += ex2_fast(fmaf(v[j], 1.4426950408889634f, -nm2));
            st_s = st_s * ex2_fast((st_m - nm) * 1.4426950408889634f) + cs;
            st_m = nm;
          }
          if (c + CW == c_end && row0 + lane < p.M)
            p.rowstats[(long long)(row0 + lane) * (NPART * p.tiles_n) + tn * NPART + part] = make_float2(st_m, st_s);
        }
        if (EPI == EPI_BF16_DGELU && CW == 32 && p.colsum != nullptr && col0 < p.N && row0 < p.M) {
          // the bias gradient of the layer that produced the GELU input: column sums of this
          // chunk's 32 rows (rows past M hold zeros), one partial per 32-row block
          float vv[32];
#pragma unroll
          for (int j = 0; j < 32; ++j) vv[j] = v[j % CW];
          const float cs = warp_colsum32(vv, lane);
          if (col0 + lane < p.N) p.colsum[(long long)(row0 >> 5) * p.N + col0 + lane] = cs;
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          if (col0 < p.N && row0 < p.M) {
            if (p.ksplit > 1) {
              tma_store_3d(&tmO2, cur, col0, row0, ks);
            } else if (EPI == EPI_F32 && p.accumulate) {
              tma_reduce_add_2d(&tmO, cur, col0, row0);
            } else {
              tma_store_2d(&tmO, cur, col0, row0);
              if (EPI == EPI_BF16_GELU) tma_store_2d(&tmO2, cur + 2048, col0, row0);
            }
          }
          bulk_commit();  // one group per chunk (possibly empty) keeps the buffer accounting exact
          if (HAS_AUX) {
            // the store of chunk n - 1 (committed a chunk ago) has read its buffer out: fetch
            // the auxiliary tile of chunk n + NBUF - 1, which uses that buffer next; the store
            // just committed may still be reading
            bulk_wait_read<1>();
            aux_load(n + NBUF - 1);
          }
        }
      }
      acc ^= 1;
      if (acc == 0) acc_phase ^= 1;
    }
    if (lane == 0) {
      bulk_wait_all();
      int never = 0;  // auxiliary loads still in flight (abort path only) land before the CTA exits
      for (int bb = 0; bb < NBUF; ++bb)
        if ((aux_pending >> bb) & 1u)
          mbar_wait_bounded(&abar[bb], (aux_par >> bb) & 1u, reinterpret_cast<volatile int*>(&never), lim);
    }
    __syncwarp();
  }

  tc_fence_before();
  if (PAIR)
    cluster_sync();  // the leader's MMAs into the peer's TMEM, and remote arrivals, are done
  else
    __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    if (PAIR)
      tmem_dealloc_pair(tmem_base, Cfg::TMEM_COLS);
    else
      tmem_dealloc(tmem_base, Cfg::TMEM_COLS);
  }
}

// Split-K reduction in a fixed order: out (+)= sum_s partial[s].
__global__ void splitk_reduce_kernel(const float* __restrict__ partial, int ksplit, long long M, int N,
                                     float* __restrict__ out, long long ldo, int accumulate) {
  const long long n4 = (long long)M * (N / 4);
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n4; i += (long long)gridDim.x * blockDim.x) {
    const long long row = i / (N / 4);
    const int c = (int)(i - row * (N / 4)) * 4;
    float4 s = *reinterpret_cast<const float4*>(partial + row * N + c);
#pragma unroll 4
    for (int k = 1; k < ksplit; ++k) {  // loads of several slices in flight; sums still in slice order
      float4 t = *reinterpret_cast<const float4*>(partial + ((long long)k * M + row) * N + c);
      s.x += t.x;
      s.y += t.y;
      s.z += t.z;
      s.w += t.w;
    }
    float* dst = out + row * ldo + c;
    if (accumulate) {
      float4 o = *reinterpret_cast<const float4*>(dst);
      s.x += o.x;
      s.y += o.y;
      s.z += o.z;
      s.w += o.w;
    }
    *reinterpret_cast<float4*>(dst) = s;
  }
}

}  // namespace g2
