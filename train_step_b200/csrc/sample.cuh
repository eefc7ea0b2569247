// sample.cuh -- exact temperature / top-k / top-p sampling of logits rows (generation).
//
// Per row (the pages give temperature and top-k sampling but no tie or precision rule;
// this is the reading used): order the V logits by value, descending, ties by lower
// index; keep the first k; weights w_j = exp((z_j - z_max) / temperature) in float64;
// running sums c_j = w_0 + ... + w_j taken left to right; with top_p < 1 keep only the
// prefix up to the first j with c_j >= top_p * c_{k-1}; draw: the first kept j with
// c_j > u * c_last, else the last kept one. -0.0 ranks equal to +0.0. Logits must not be NaN.
//
// One CTA of 1024 threads per row. The k-th largest value comes from a most-significant-
// digit radix select over order-preserving 32-bit keys (four 8-bit passes over the row,
// each digit found by one warp's scan of the 256-bin histogram); the k candidates are
// gathered (equal keys taken in index order), sorted by (value desc, index asc) with a
// bitonic sort in shared memory, weighted in parallel, and one thread forms the running
// sums in order.
#pragma once
#include "common.cuh"

namespace g2 {

constexpr int TOPK_THREADS = 1024;
constexpr int TOPK_MAX_K = 1024;

// order-preserving map of a float onto uint32 (larger float -> larger key; -0 == +0)
__device__ __forceinline__ uint32_t topk_key(float f) {
  uint32_t b = __float_as_uint(f);
  if (b == 0x80000000u) b = 0u;
  return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}

// index of candidate j (clamped into the row, although exactly k candidates are gathered)
__device__ __forceinline__ int topk_index(unsigned long long code, int V) {
  const unsigned i = (unsigned)(code & 0xFFFFFFFFull);
  return i < (unsigned)V ? (int)i : V - 1;
}

__global__ void __launch_bounds__(TOPK_THREADS)
    sample_topk_kernel(const float* __restrict__ logits, int64_t ld, int V, int k, float temperature, float top_p,
                       const double* __restrict__ u, int* __restrict__ out) {
  __shared__ unsigned int hist[256];
  __shared__ unsigned long long cand[TOPK_MAX_K];  // (~key << 32 | index): ascending = value desc, index asc
  __shared__ double w[TOPK_MAX_K];
  __shared__ uint32_t s_prefix, s_need, s_count;
  __shared__ int warp_cnt[TOPK_THREADS / 32];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const float* z = logits + (int64_t)blockIdx.x * ld;
  if (tid == 0) {
    s_prefix = 0u;
    s_need = (uint32_t)k;  // how many keys under the fixed prefix are still wanted
  }
  __syncthreads();
  // radix select: after pass d the top 8(d+1) bits of the k-th largest key are fixed
  for (int d = 0; d < 4; ++d) {
    const int shift = 24 - 8 * d;
    const uint32_t pmask = d == 0 ? 0u : (0xFFFFFFFFu << (shift + 8));
    for (int i = tid; i < 256; i += TOPK_THREADS) hist[i] = 0u;
    __syncthreads();
    const uint32_t prefix = s_prefix;
    for (int i = tid; i < V; i += TOPK_THREADS) {
      const uint32_t key = topk_key(z[i]);
      if ((key & pmask) == prefix) atomicAdd(&hist[(key >> shift) & 255u], 1u);
    }
    __syncthreads();
    if (warp == 0) {
      // lane l holds digits 255-8l .. 248-8l (descending); an inclusive scan over lanes
      // finds the digit at which the running count of larger keys reaches `need`
      uint32_t cnt[8], tot = 0u;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        cnt[i] = hist[255 - (lane * 8 + i)];
        tot += cnt[i];
      }
      uint32_t incl = tot;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const uint32_t v = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += v;
      }
      const uint32_t need = s_need, excl = incl - tot;
      if (excl < need && need <= incl) {  // exactly one lane: need <= keys under the prefix
        uint32_t acc = excl;
        int i = 0;
        for (; i < 7; ++i) {
          if (acc + cnt[i] >= need) break;
          acc += cnt[i];
        }
        s_prefix = prefix | ((uint32_t)(255 - (lane * 8 + i)) << shift);
        s_need = need - acc;  // keys wanted among those that share the new prefix
      }
    }
    __syncthreads();
  }
  // every key above the k-th, and the first s_need keys equal to it in index order: each
  // warp owns a contiguous range of the row, counts its equal keys, and after one scan of
  // those counts walks its range again placing candidates
  const uint32_t kth = s_prefix, n_eq = s_need;
  constexpr int NWARP = TOPK_THREADS / 32;
  const int seg = ((V + NWARP - 1) / NWARP + 31) & ~31;
  const int r0 = min(V, warp * seg), r1 = min(V, r0 + seg);
  if (tid == 0) s_count = 0u;
  uint32_t n_mine = 0u;
  for (int i0 = r0; i0 < r1; i0 += 32) {
    const int i = i0 + lane;
    const bool eq = i < r1 && topk_key(z[i]) == kth;
    n_mine += (uint32_t)__popc(__ballot_sync(0xffffffffu, eq));
  }
  if (lane == 0) warp_cnt[warp] = (int)n_mine;
  __syncthreads();
  uint32_t before = 0u;  // equal keys at lower indices than this warp's range
  for (int q = 0; q < warp; ++q) before += (uint32_t)warp_cnt[q];
  for (int i0 = r0; i0 < r1; i0 += 32) {
    const int i = i0 + lane;
    uint32_t key = 0u;
    bool gt = false, eq = false;
    if (i < r1) {
      key = topk_key(z[i]);
      gt = key > kth;
      eq = key == kth;
    }
    const unsigned ballot = __ballot_sync(0xffffffffu, eq);
    const uint32_t rank = before + (uint32_t)__popc(ballot & ((1u << lane) - 1u));
    if (gt || (eq && rank < n_eq)) {
      const uint32_t slot = atomicAdd(&s_count, 1u);
      if (slot < (uint32_t)TOPK_MAX_K) cand[slot] = ((unsigned long long)(~key) << 32) | (unsigned)i;
    }
    before += (uint32_t)__popc(ballot);
  }
  __syncthreads();
  // bitonic sort of the candidates, padded to a power of two with the largest code
  int np = 1;
  while (np < k) np <<= 1;
  for (int i = tid + k; i < np; i += TOPK_THREADS) cand[i] = ~0ull;
  __syncthreads();
  for (int kk = 2; kk <= np; kk <<= 1) {
    for (int j = kk >> 1; j > 0; j >>= 1) {
      for (int i = tid; i < np; i += TOPK_THREADS) {
        const int ixj = i ^ j;
        if (ixj > i) {
          const unsigned long long a = cand[i], b = cand[ixj];
          if ((a > b) == ((i & kk) == 0)) {
            cand[i] = b;
            cand[ixj] = a;
          }
        }
      }
      __syncthreads();
    }
  }
  const double zmax = (double)z[topk_index(cand[0], V)];
  for (int j = tid; j < k; j += TOPK_THREADS)
    w[j] = exp(((double)z[topk_index(cand[j], V)] - zmax) / (double)temperature);
  __syncthreads();
  if (tid == 0) {
    double total = 0.0;
    for (int j = 0; j < k; ++j) total += w[j];
    int last = k - 1;
    if (top_p < 1.0f) {
      const double cut = (double)top_p * total;
      double run = 0.0;
      for (int j = 0; j < k; ++j) {
        run += w[j];
        if (run >= cut) {
          last = j;
          total = run;
          break;
        }
      }
    }
    const double target = u[blockIdx.x] * total;
    double run = 0.0;
    int pick = last;
    for (int j = 0; j <= last; ++j) {
      run += w[j];
      if (run > target) {
        pick = j;
        break;
      }
    }
    out[blockIdx.x] = topk_index(cand[pick], V);
  }
}

}  // namespace g2
