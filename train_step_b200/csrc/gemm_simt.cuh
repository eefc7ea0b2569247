// gemm_simt.cuh -- fp32 CUDA-core GEMM with the same operand conventions and
// epilogues as the tensor-core kernel. It serves the fp32 parity mode only (the
// tiny character-level configuration, where the tolerance is 1e-5 on the loss and
// 1e-4 on gradients, which TF32 tensor cores would miss).
#pragma once
#include "common.cuh"
#include "gemm_tc.cuh"

namespace g2 {

struct SimtGemmArgs {
  const float* A;
  long long lda;
  int a_mn;
  const float* B;
  long long ldb;
  int b_mn;
  int M, N, K;
  GemmParams ep;  // epilogue fields (out, ldo, out2, bias, aux, accumulate)
};

// 64x64 tile, 16-deep K slices, 256 threads with a 4x4 micro-tile each.
template <int EPI>
__global__ void __launch_bounds__(256) gemm_simt_kernel(const SimtGemmArgs a) {
  __shared__ float As[16][64 + 1];
  __shared__ float Bs[16][64 + 1];
  const int tid = threadIdx.x;
  const int m0 = blockIdx.y * 64, n0 = blockIdx.x * 64;
  const int tx = tid % 16, ty = tid / 16;
  float acc[4][4] = {};
  for (int k0 = 0; k0 < a.K; k0 += 16) {
    for (int i = tid; i < 64 * 16; i += 256) {
      int mm, kk;
      if (a.a_mn) {
        mm = i % 64;
        kk = i / 64;
      } else {
        kk = i % 16;
        mm = i / 16;
      }
      const int gm = m0 + mm, gk = k0 + kk;
      float v = 0.f;
      if (gm < a.M && gk < a.K) v = a.a_mn ? a.A[(long long)gk * a.lda + gm] : a.A[(long long)gm * a.lda + gk];
      As[kk][mm] = v;
      int nn;
      if (a.b_mn) {
        nn = i % 64;
        kk = i / 64;
      } else {
        kk = i % 16;
        nn = i / 16;
      }
      const int gn = n0 + nn, gk2 = k0 + kk;
      float w = 0.f;
      if (gn < a.N && gk2 < a.K) w = a.b_mn ? a.B[(long long)gk2 * a.ldb + gn] : a.B[(long long)gn * a.ldb + gk2];
      Bs[kk][nn] = w;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < 16; ++kk) {
      float av[4], bv[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        av[i] = As[kk][ty * 4 + i];
        bv[i] = Bs[kk][tx * 4 + i];
      }
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(av[i], bv[j], acc[i][j]);
    }
    __syncthreads();
  }
  const GemmParams& p = a.ep;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int m = m0 + ty * 4 + i;
    if (m >= a.M) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int n = n0 + tx * 4 + j;
      if (n >= a.N) continue;
      float v = acc[i][j];
      if (EPI == EPI_BF16 || EPI == EPI_BF16_GELU || EPI == EPI_F32_RESID)
        if (p.bias) v += p.bias[n];
      if (EPI == EPI_BF16) {
        reinterpret_cast<float*>(p.out)[(long long)m * p.ldo + n] = v;
      } else if (EPI == EPI_BF16_GELU) {
        reinterpret_cast<float*>(p.out)[(long long)m * p.ldo + n] = v;
        reinterpret_cast<float*>(p.out2)[(long long)m * p.ldo2 + n] = gelu_tanh(v);
      } else if (EPI == EPI_F32_RESID) {
        reinterpret_cast<float*>(p.out)[(long long)m * p.ldo + n] =
            reinterpret_cast<const float*>(p.aux)[(long long)m * p.ld_aux + n] + v;
      } else if (EPI == EPI_BF16_DGELU) {
        reinterpret_cast<float*>(p.out)[(long long)m * p.ldo + n] =
            v * gelu_tanh_grad(reinterpret_cast<const float*>(p.aux)[(long long)m * p.ld_aux + n]);
      } else {
        float* d = reinterpret_cast<float*>(p.out) + (long long)m * p.ldo + n;
        *d = p.accumulate ? *d + v : v;
      }
    }
  }
}

}  // namespace g2
