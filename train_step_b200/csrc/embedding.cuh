// embedding.cuh -- token + position embedding, forward and atomic-free backward
// ("gpt/docs/LLM.md", Embedding Layer: token embeddings wte and position
// embeddings wpe; "GPT From Scratch", Architecture diagram: wte + wpe).
//
// Forward: x0[n, :] = wte[tok[n], :] + wpe[n mod T, :] in fp32.
// Backward: dwte[v] += sum over positions n with tok[n] == v of dx0[n], and
// dwpe[t] += sum_b dx0[b*T + t]. No floating-point atomics: positions are
// bucketed by token id with a stable sort (a single-CTA bitonic sort of the keys
// (id << 15) | position, which equals the stable counting sort because the keys
// are distinct), long buckets are cut into chunks of EMB_CHUNK rows, each chunk
// is summed in position order, and the chunks of a bucket are added in order.
#pragma once
#include "common.cuh"

namespace g2 {

constexpr int EMB_CHUNK = 32;          // rows per summed chunk
constexpr int EMB_SORT_THREADS = 1024;
constexpr int EMB_MAX_TOKENS = 32768;  // positions fit 15 bits of the sort key

__global__ void embed_fwd_kernel(const int* __restrict__ tok, const float* __restrict__ wte,
                                 const float* __restrict__ wpe, float* __restrict__ x0, int N, int T, int C, int V,
                                 int* err) {
  const long long gw = (blockIdx.x * (long long)blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (gw >= N) return;
  int id = tok[gw];
  if (id < 0 || id >= V) {
    if (lane == 0) raise_device_error(err, DEV_TOKEN_RANGE);
    id = 0;
  }
  const int t = (int)(gw % T);
  const float* a = wte + (long long)id * C;
  const float* b = wpe + (long long)t * C;
  float* o = x0 + gw * C;
  for (int c = lane * 4; c < C; c += 128) {
    float4 u = __ldg(reinterpret_cast<const float4*>(a + c));
    float4 w = __ldg(reinterpret_cast<const float4*>(b + c));
    *reinterpret_cast<float4*>(o + c) = make_float4(u.x + w.x, u.y + w.y, u.z + w.z, u.w + w.w);
  }
}

// Block-wide inclusive scan helpers over EMB_SORT_THREADS threads.
template <class Op>
__device__ __forceinline__ int block_scan_incl(int v, Op op, int identity, int* warp_buf) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    int y = __shfl_up_sync(0xffffffffu, v, o);
    if (lane >= o) v = op(v, y);
  }
  __syncthreads();
  if (lane == 31) warp_buf[warp] = v;
  __syncthreads();
  if (warp == 0) {
    int w = lane < (EMB_SORT_THREADS / 32) ? warp_buf[lane] : identity;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      int y = __shfl_up_sync(0xffffffffu, w, o);
      if (lane >= o) w = op(w, y);
    }
    warp_buf[lane] = w;
  }
  __syncthreads();
  if (warp > 0) v = op(v, warp_buf[warp - 1]);
  __syncthreads();
  return v;
}

struct OpMax {
  __device__ int operator()(int a, int b) const { return a > b ? a : b; }
};
struct OpAdd {
  __device__ int operator()(int a, int b) const { return a + b; }
};

// Bitonic sort of NP = 1024 * E keys (ascending) with the keys in registers: key
// i = (warp * E + e) * 32 + lane sits in register e of that lane. Partners i ^ j with
// j < 32 are in another lane (shuffle), with 32 <= j < 32 E in another register of the
// same thread, and only j >= 32 E crosses warps (one shared-memory pass). The sequence of
// compare-exchanges is the textbook network, so the result is the same sorted array.
template <int JE, int E>
__device__ __forceinline__ void bitonic_reg_stage(uint32_t (&v)[E], int k, int base, int lane) {
#pragma unroll
  for (int e = 0; e < E; ++e) {
    if ((e & JE) == 0) {
      const int e2 = e | JE;
      const bool up = (((base + e) * 32 + lane) & k) == 0;
      const uint32_t a = v[e], b = v[e2];
      if ((a > b) == up) {
        v[e] = b;
        v[e2] = a;
      }
    }
  }
}
template <int E>
__device__ void bitonic_sort_regs(uint32_t* keys, int tid) {
  constexpr int NP = 1024 * E;
  const int lane = tid & 31, base = (tid >> 5) * E;
  uint32_t v[E];
#pragma unroll
  for (int e = 0; e < E; ++e) v[e] = keys[(base + e) * 32 + lane];
  for (int k = 2; k <= NP; k <<= 1) {
    for (int j = k >> 1; j > 0; j >>= 1) {
      if (j >= 32 * E) {  // across warps, through shared memory
#pragma unroll
        for (int e = 0; e < E; ++e) keys[(base + e) * 32 + lane] = v[e];
        __syncthreads();
        for (int t = tid; t < NP / 2; t += 1024) {
          const int i = ((t & ~(j - 1)) << 1) | (t & (j - 1)), ixj = i | j;
          const uint32_t a = keys[i], b = keys[ixj];
          if ((a > b) == ((i & k) == 0)) {
            keys[i] = b;
            keys[ixj] = a;
          }
        }
        __syncthreads();
#pragma unroll
        for (int e = 0; e < E; ++e) v[e] = keys[(base + e) * 32 + lane];
      } else if (j >= 32) {  // another register of this thread
        switch (j >> 5) {
          case 1: bitonic_reg_stage<1, E>(v, k, base, lane); break;
          case 2: bitonic_reg_stage<2, E>(v, k, base, lane); break;
          case 4: bitonic_reg_stage<4, E>(v, k, base, lane); break;
          case 8: bitonic_reg_stage<8, E>(v, k, base, lane); break;
          case 16: bitonic_reg_stage<16, E>(v, k, base, lane); break;
        }
      } else {  // another lane of this warp
#pragma unroll
        for (int e = 0; e < E; ++e) {
          const uint32_t other = __shfl_xor_sync(0xffffffffu, v[e], j);
          const bool up = ((((base + e) * 32) + lane) & k) == 0;
          const bool lower = (lane & j) == 0;  // this lane holds the smaller index of the pair
          v[e] = (lower == up) ? min(v[e], other) : max(v[e], other);
        }
      }
    }
  }
#pragma unroll
  for (int e = 0; e < E; ++e) keys[(base + e) * 32 + lane] = v[e];
  __syncthreads();
}

// One CTA. Outputs:
//   sorted_pos[i]        position of the i-th entry in (id, position) order
//   chunk_start[c]       first sorted index of chunk c (chunks never straddle ids)
//   seg_id[s], seg_chunk0[s]  id of bucket s and its first chunk; seg_chunk0[nseg] = nchunks
//   counts[0] = nseg, counts[1] = nchunks
// Dynamic shared memory: NP * 4 bytes, NP = next power of two >= N.
__global__ void __launch_bounds__(EMB_SORT_THREADS) token_sort_kernel(const int* __restrict__ tok, int N, int V, int NP,
                                                                     int* __restrict__ sorted_pos,
                                                                     int* __restrict__ chunk_start,
                                                                     int* __restrict__ seg_id,
                                                                     int* __restrict__ seg_chunk0,
                                                                     int* __restrict__ counts, int* err) {
  extern __shared__ uint32_t keys[];
  __shared__ int warp_buf[32];
  const int tid = threadIdx.x;
  for (int i = tid; i < NP; i += EMB_SORT_THREADS) {
    if (i < N) {
      int id = tok[i];
      if (id < 0 || id >= V) {
        raise_device_error(err, DEV_TOKEN_RANGE);
        id = 0;
      }
      keys[i] = ((uint32_t)id << 15) | (uint32_t)i;
    } else {
      keys[i] = 0xFFFFFFFFu;
    }
  }
  __syncthreads();
  // bitonic sort, ascending
  if (NP == 1024 * 16) {
    bitonic_sort_regs<16>(keys, tid);
  } else if (NP == 1024 * 32) {
    bitonic_sort_regs<32>(keys, tid);
  } else {
    for (int k = 2; k <= NP; k <<= 1) {
      for (int j = k >> 1; j > 0; j >>= 1) {
        for (int i = tid; i < NP; i += EMB_SORT_THREADS) {
          const int ixj = i ^ j;
          if (ixj > i) {
            const uint32_t a = keys[i], b = keys[ixj];
            const bool up = (i & k) == 0;
            if ((a > b) == up) {
              keys[i] = b;
              keys[ixj] = a;
            }
          }
        }
        __syncthreads();
      }
    }
  }
  // each thread owns E consecutive sorted entries
  const int E = (N + EMB_SORT_THREADS - 1) / EMB_SORT_THREADS;
  const int i0 = tid * E, i1 = min(N, i0 + E);
  // segment heads and the start index of each entry's segment (max-scan)
  int local_max = -1;
  for (int i = i0; i < i1; ++i) {
    sorted_pos[i] = (int)(keys[i] & 0x7FFFu);
    const bool head = (i == 0) || ((keys[i] >> 15) != (keys[i - 1] >> 15));
    if (head) local_max = i;
  }
  const int run_max = block_scan_incl(local_max, OpMax(), -1, warp_buf);
  // exclusive max for this thread = inclusive max of the previous thread
  __shared__ int excl_max_buf[EMB_SORT_THREADS];
  excl_max_buf[tid] = run_max;
  __syncthreads();
  int cur_head = tid > 0 ? excl_max_buf[tid - 1] : -1;
  // count chunk heads and segment heads in this thread's range
  int nchunk_local = 0, nseg_local = 0;
  for (int i = i0; i < i1; ++i) {
    const bool head = (i == 0) || ((keys[i] >> 15) != (keys[i - 1] >> 15));
    if (head) cur_head = i;
    if ((i - cur_head) % EMB_CHUNK == 0) ++nchunk_local;
    if (head) ++nseg_local;
  }
  const int chunk_incl = block_scan_incl(nchunk_local, OpAdd(), 0, warp_buf);
  const int seg_incl = block_scan_incl(nseg_local, OpAdd(), 0, warp_buf);
  int c = chunk_incl - nchunk_local, s = seg_incl - nseg_local;
  cur_head = tid > 0 ? excl_max_buf[tid - 1] : -1;
  for (int i = i0; i < i1; ++i) {
    const bool head = (i == 0) || ((keys[i] >> 15) != (keys[i - 1] >> 15));
    if (head) cur_head = i;
    if ((i - cur_head) % EMB_CHUNK == 0) {
      chunk_start[c] = i;
      if (head) {
        seg_id[s] = (int)(keys[i] >> 15);
        seg_chunk0[s] = c;
        ++s;
      }
      ++c;
    }
  }
  if (tid == EMB_SORT_THREADS - 1) {
    counts[0] = seg_incl;
    counts[1] = chunk_incl;
    seg_chunk0[seg_incl] = chunk_incl;
    chunk_start[chunk_incl] = N;
  }
}

// Stage 1: partial[c][:] = sum of dx0 rows of chunk c, in sorted order. The rows of a
// chunk are fetched 8 at a time (independent loads in flight) and added in index order,
// so the sum is the plain sequential one.
__global__ void embed_chunk_sum_kernel(const float* __restrict__ dx0, const int* __restrict__ sorted_pos,
                                       const int* __restrict__ chunk_start, const int* __restrict__ counts, int C,
                                       float* __restrict__ partial) {
  const int nchunks = counts[1];
  for (int ch = blockIdx.x; ch < nchunks; ch += gridDim.x) {
    const int a = chunk_start[ch], b = chunk_start[ch + 1];
    for (int c = threadIdx.x * 4; c < C; c += blockDim.x * 4) {
      float4 s = make_float4(0.f, 0.f, 0.f, 0.f);
      for (int i = a; i < b; i += 8) {
        float4 v[8];
#pragma unroll
        for (int u = 0; u < 8; ++u)
          if (i + u < b) v[u] = __ldg(reinterpret_cast<const float4*>(dx0 + (long long)sorted_pos[i + u] * C + c));
#pragma unroll
        for (int u = 0; u < 8; ++u)
          if (i + u < b) {
            s.x += v[u].x;
            s.y += v[u].y;
            s.z += v[u].z;
            s.w += v[u].w;
          }
      }
      *reinterpret_cast<float4*>(partial + (long long)ch * C + c) = s;
    }
  }
}

// Stage 2: dwte[id] += sum over the bucket's chunks, in order.
__global__ void embed_seg_sum_kernel(const float* __restrict__ partial, const int* __restrict__ seg_id,
                                     const int* __restrict__ seg_chunk0, const int* __restrict__ counts, int C,
                                     float* __restrict__ dwte) {
  const int nseg = counts[0];
  for (int sg = blockIdx.x; sg < nseg; sg += gridDim.x) {
    const int c0 = seg_chunk0[sg], c1 = seg_chunk0[sg + 1];
    float* dst = dwte + (long long)seg_id[sg] * C;
    for (int c = threadIdx.x * 4; c < C; c += blockDim.x * 4) {
      float4 s = *reinterpret_cast<const float4*>(partial + (long long)c0 * C + c);
      for (int k = c0 + 1; k < c1; ++k) {
        const float4 v = *reinterpret_cast<const float4*>(partial + (long long)k * C + c);
        s.x += v.x;
        s.y += v.y;
        s.z += v.z;
        s.w += v.w;
      }
      float4 o = *reinterpret_cast<const float4*>(dst + c);
      *reinterpret_cast<float4*>(dst + c) = make_float4(o.x + s.x, o.y + s.y, o.z + s.z, o.w + s.w);
    }
  }
}

// dwpe[t, :] += sum_b dx0[b*T + t, :] (the Bsz rows fetched 8 at a time, added in order)
__global__ void embed_pos_grad_kernel(const float* __restrict__ dx0, int Bsz, int T, int C, float* __restrict__ dwpe) {
  const long long i = (blockIdx.x * (long long)blockDim.x + threadIdx.x) * 4;
  if (i >= (long long)T * C) return;
  const int t = (int)(i / C), c = (int)(i % C);
  float4 s = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int b0 = 0; b0 < Bsz; b0 += 8) {
    float4 v[8];
#pragma unroll
    for (int u = 0; u < 8; ++u)
      if (b0 + u < Bsz) v[u] = __ldg(reinterpret_cast<const float4*>(dx0 + ((long long)(b0 + u) * T + t) * C + c));
#pragma unroll
    for (int u = 0; u < 8; ++u)
      if (b0 + u < Bsz) {
        s.x += v[u].x;
        s.y += v[u].y;
        s.z += v[u].z;
        s.w += v[u].w;
      }
  }
  float4 o = *reinterpret_cast<float4*>(dwpe + i);
  *reinterpret_cast<float4*>(dwpe + i) = make_float4(o.x + s.x, o.y + s.y, o.z + s.z, o.w + s.w);
}

}  // namespace g2
