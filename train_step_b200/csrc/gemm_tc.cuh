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
//   warps 2..9  epilogue: tcgen05.ld 32 lanes x 32 columns, fused bias / GELU /
//               residual / GELU' math, global stores. Two TMEM accumulators
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
  int* err;
  unsigned long long timeout_ns;
};

constexpr int TC_BM = 128;
constexpr int TC_BK = 64;
constexpr int TC_THREADS = 320;
constexpr int TC_EPI_WARPS = 8;

template <int BN>
struct TcCfg {
  static constexpr int A_BYTES = TC_BM * TC_BK * 2;
  static constexpr int B_BYTES = BN * TC_BK * 2;
  static constexpr int STAGE = A_BYTES + B_BYTES;
  static constexpr int STAGES = (192 * 1024) / STAGE;
  static constexpr int TMEM_COLS = 2 * BN <= 256 ? 256 : 512;
  static constexpr int STAGING = TC_EPI_WARPS * 4096;  // one 4 KB store buffer per epilogue warp
  static constexpr int SMEM = STAGES * STAGE + STAGING + 1024 + 256;
};

__device__ __forceinline__ float gelu_tanh_fast(float u) {
  const float k = 0.7978845608028654f;
  float inner = k * (u + 0.044715f * u * u * u);
  float th;
  asm("tanh.approx.f32 %0, %1;" : "=f"(th) : "f"(inner));
  return 0.5f * u * (1.0f + th);
}
__device__ __forceinline__ float gelu_tanh_grad_fast(float u) {
  const float k = 0.7978845608028654f;
  float inner = k * (u + 0.044715f * u * u * u);
  float th;
  asm("tanh.approx.f32 %0, %1;" : "=f"(th) : "f"(inner));
  float dinner = k * (1.0f + 3.0f * 0.044715f * u * u);
  return 0.5f * (1.0f + th) + 0.5f * u * (1.0f - th * th) * dinner;
}

// Output tile of one epilogue warp and chunk: 32 rows (one per lane) x 32 columns,
// staged in shared memory in the layout of the output tensor map's box:
//   bf16: 64-byte rows, 64-byte swizzle (16-byte chunk k of row r at chunk k ^ ((r >> 1) & 3))
//   fp32: 128-byte rows, 128-byte swizzle (chunk k of row r at chunk k ^ (r & 7))
// Both patterns put the 8 lanes of a 16-byte store phase in distinct banks.
__device__ __forceinline__ void stage_bf16_row(uint8_t* buf, int r, const float (&v)[32]) {
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const int j = k * 8;
    uint4 w = make_uint4(pack_bf16x2(v[j], v[j + 1]), pack_bf16x2(v[j + 2], v[j + 3]), pack_bf16x2(v[j + 4], v[j + 5]),
                         pack_bf16x2(v[j + 6], v[j + 7]));
    *reinterpret_cast<uint4*>(buf + r * 64 + ((k ^ ((r >> 1) & 3)) << 4)) = w;
  }
}
__device__ __forceinline__ void stage_f32_row(uint8_t* buf, int r, const float (&v)[32]) {
#pragma unroll
  for (int k = 0; k < 8; ++k)
    *reinterpret_cast<float4*>(buf + r * 128 + ((k ^ (r & 7)) << 4)) =
        make_float4(v[4 * k], v[4 * k + 1], v[4 * k + 2], v[4 * k + 3]);
}

// Epilogue math on 32 consecutive columns [col0, col0+32) of one row, written into
// the staging buffer(s) (row `lane`). Columns past N hold don't-care values: the
// tensor-map store clips them.
template <int EPI>
__device__ __forceinline__ void tc_epilogue_stage(const GemmParams& p, int row, int col0, int lane, float (&v)[32],
                                                  uint8_t* buf) {
  const bool full = (col0 + 32 <= p.N);
  const bool row_ok = row < p.M;
  if (p.ksplit > 1 || EPI == EPI_F32) {
    stage_f32_row(buf, lane, v);
    return;
  }
  if (EPI == EPI_BF16 || EPI == EPI_BF16_GELU || EPI == EPI_F32_RESID) {
    if (p.bias) {
      if (full) {
#pragma unroll
        for (int j = 0; j < 32; j += 4) {
          float4 b = __ldg(reinterpret_cast<const float4*>(p.bias + col0 + j));
          v[j] += b.x;
          v[j + 1] += b.y;
          v[j + 2] += b.z;
          v[j + 3] += b.w;
        }
      } else {
#pragma unroll
        for (int j = 0; j < 32; ++j)
          if (col0 + j < p.N) v[j] += p.bias[col0 + j];
      }
    }
  }
  if (EPI == EPI_BF16) {
    stage_bf16_row(buf, lane, v);
  } else if (EPI == EPI_BF16_GELU) {
    stage_bf16_row(buf, lane, v);
#pragma unroll
    for (int j = 0; j < 32; ++j) v[j] = gelu_tanh_fast(v[j]);
    stage_bf16_row(buf + 2048, lane, v);
  } else if (EPI == EPI_F32_RESID) {
    if (row_ok) {
      const float* res = reinterpret_cast<const float*>(p.aux) + (long long)row * p.ld_aux + col0;
      if (full) {
#pragma unroll
        for (int j = 0; j < 32; j += 4) {
          float4 x = *reinterpret_cast<const float4*>(res + j);
          v[j] += x.x;
          v[j + 1] += x.y;
          v[j + 2] += x.z;
          v[j + 3] += x.w;
        }
      } else {
#pragma unroll
        for (int j = 0; j < 32; ++j)
          if (col0 + j < p.N) v[j] += res[j];
      }
    }
    stage_f32_row(buf, lane, v);
  } else if (EPI == EPI_BF16_DGELU) {
    if (row_ok) {
      const bf16* u = reinterpret_cast<const bf16*>(p.aux) + (long long)row * p.ld_aux + col0;
      if (full) {
#pragma unroll
        for (int j = 0; j < 32; j += 8) {
          uint4 uu = *reinterpret_cast<const uint4*>(u + j);
          const uint32_t w[4] = {uu.x, uu.y, uu.z, uu.w};
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const float2 f = unpack_bf16x2(w[q]);
            v[j + 2 * q] *= gelu_tanh_grad_fast(f.x);
            v[j + 2 * q + 1] *= gelu_tanh_grad_fast(f.y);
          }
        }
      } else {
#pragma unroll
        for (int j = 0; j < 32; ++j)
          if (col0 + j < p.N) v[j] *= gelu_tanh_grad_fast(__bfloat162float(u[j]));
      }
    }
    stage_bf16_row(buf, lane, v);
  }
}

__device__ __forceinline__ void tc_decode_unit(const GemmParams& p, int unit, int& tm, int& tn, int& ks) {
  const int per_split = p.tiles_m * p.tiles_n;
  ks = unit / per_split;
  const int t = unit - ks * per_split;
  tm = t / p.tiles_n;
  tn = t - tm * p.tiles_n;
}

template <int BN, bool A_MN, bool B_MN, int EPI>
__global__ void __launch_bounds__(TC_THREADS, 1)
    gemm_tc_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                   const __grid_constant__ CUtensorMap tmO, const __grid_constant__ CUtensorMap tmO2,
                   const GemmParams p) {
  using Cfg = TcCfg<BN>;
  constexpr int STAGES = Cfg::STAGES;
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

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], TC_EPI_WARPS);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, Cfg::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const uint64_t lim = p.timeout_ns;

  if (warp == 0) {
    if (lane == 0) {
      // ---------------- TMA producer ----------------
      int stage = 0;
      uint32_t phase = 0;
      uint32_t issued = 0, last_par = 0;  // bit s: stage s has a copy issued / its parity
      bool ok = true;
      for (int unit = blockIdx.x; unit < p.num_units && ok; unit += gridDim.x) {
        int tm, tn, ks;
        tc_decode_unit(p, unit, tm, tn, ks);
        const int kb0 = ks * p.kb_per_split;
        const int kb1 = min(kb0 + p.kb_per_split, p.num_kb);
        for (int kb = kb0; kb < kb1; ++kb) {
          if (!mbar_wait_bounded(&empty[stage], phase ^ 1, abort_flag, lim)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&full[stage], Cfg::STAGE);
          uint8_t* sa = smem + stage * Cfg::STAGE;
          uint8_t* sb = sa + Cfg::A_BYTES;
          const int kx = kb * TC_BK;
          if (!A_MN) {
            tma_load_2d(sa, &tmA, &full[stage], kx, tm * TC_BM);
          } else {
            tma_load_2d(sa, &tmA, &full[stage], tm * TC_BM, kx);
            tma_load_2d(sa + 8192, &tmA, &full[stage], tm * TC_BM + 64, kx);
          }
          if (!B_MN) {
            tma_load_2d(sb, &tmB, &full[stage], kx, tn * BN);
          } else {
#pragma unroll
            for (int j = 0; j < BN / 64; ++j) tma_load_2d(sb + j * 8192, &tmB, &full[stage], tn * BN + j * 64, kx);
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
        for (int s = 0; s < STAGES; ++s)
          if ((issued >> s) & 1u) mbar_wait_bounded(&full[s], (last_par >> s) & 1u, reinterpret_cast<volatile int*>(&never), lim);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ---------------- MMA issuer ----------------
      constexpr uint32_t idesc = make_idesc_bf16(TC_BM, BN, A_MN, B_MN);
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool ok = true, any = false;
      for (int unit = blockIdx.x; unit < p.num_units && ok; unit += gridDim.x) {
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
            umma_bf16(d_tmem, ad, bd, idesc, (kb > kb0 || k > 0) ? 1u : 0u);
          }
          any = true;
          umma_commit(&empty[stage]);
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1;
          }
        }
        if (!ok) break;
        umma_commit(&tfull[acc]);
        acc ^= 1;
        if (acc == 0) acc_phase ^= 1;
      }
      if (!ok) {
        raise_device_error(p.err, DEV_TIMEOUT);
        *abort_flag = 1;
        if (any) {  // wait for the MMAs already issued before the TMEM is freed
          int never = 0;
          umma_commit(drain);
          mbar_wait_bounded(drain, 0, reinterpret_cast<volatile int*>(&never), lim);
        }
      }
    }
  } else {
    // ---------------- epilogue warps ----------------
    const int ew = warp - 2;         // 0..7
    const int q = warp & 3;          // TMEM lane quarter this warp may access
    const int half = ew >> 2;        // which half of the BN columns
    uint8_t* buf = staging + ew * 4096;
    // bf16 single-output chunks take 2 KB: two buffers alternate; others take 4 KB
    constexpr bool two_bufs = (EPI == EPI_BF16 || EPI == EPI_BF16_DGELU);
    if (lane == 0) {
      if (EPI == EPI_BF16_GELU || p.ksplit > 1) tma_prefetch_desc(&tmO2);
      tma_prefetch_desc(&tmO);
    }
    int acc = 0;
    uint32_t acc_phase = 0;
    int nchunk = 0;
    for (int unit = blockIdx.x; unit < p.num_units; unit += gridDim.x) {
      int tm, tn, ks;
      tc_decode_unit(p, unit, tm, tn, ks);
      if (!mbar_wait_bounded(&tfull[acc], acc_phase, abort_flag, lim)) {
        if (lane == 0) {
          raise_device_error(p.err, DEV_TIMEOUT);
          *abort_flag = 1;
        }
        break;
      }
      tc_fence_after();
      const int row0 = tm * TC_BM + q * 32;
      const int c_begin = half * (BN / 2), c_end = (half + 1) * (BN / 2);
#pragma unroll 1
      for (int c = c_begin; c < c_end; c += 32, ++nchunk) {
        uint32_t r[32];
        tmem_ld_32x32b_x32(tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(acc * BN + c), r);
        tmem_ld_wait();
        if (c + 32 == c_end) {  // last read of this accumulator: hand it back to the MMA warp
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&tempty[acc]);
        }
        const int col0 = tn * BN + c;
        uint8_t* b = (two_bufs && (nchunk & 1)) ? buf + 2048 : buf;
        // the staging buffer must have been read out by the previous store
        if (lane == 0) {
          if (two_bufs) bulk_wait_read<1>();
          else bulk_wait_read<0>();
        }
        __syncwarp();
        float v[32];
#pragma unroll
        for (int j = 0; j < 32; ++j) v[j] = __uint_as_float(r[j]);
        if (col0 < p.N) tc_epilogue_stage<EPI>(p, row0 + lane, col0, lane, v, b);
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          if (col0 < p.N && row0 < p.M) {
            if (p.ksplit > 1) {
              tma_store_3d(&tmO2, b, col0, row0, ks);
            } else if (EPI == EPI_F32 && p.accumulate) {
              tma_reduce_add_2d(&tmO, b, col0, row0);
            } else {
              tma_store_2d(&tmO, b, col0, row0);
              if (EPI == EPI_BF16_GELU) tma_store_2d(&tmO2, b + 2048, col0, row0);
            }
          }
          bulk_commit();  // one group per chunk (possibly empty) keeps the buffer accounting exact
        }
      }
      acc ^= 1;
      if (acc == 0) acc_phase ^= 1;
    }
    if (lane == 0) bulk_wait_all();
    __syncwarp();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
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
    for (int k = 1; k < ksplit; ++k) {
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
