// topk.cuh -- global top-k over documents (MSA, b-lab.team summary item 1:
// the k most relevant documents are selected; Evermind sec. 2).
// Order: score descending, then document id ascending (ties go to the lower
// id).  Each (score, id) pair is packed into one order-preserving 64-bit key,
// so the top-k is a selection of the k largest keys -- exact and
// deterministic.  Phase 1: one CTA per (query, 4096-document slice) selects
// its slice's k largest keys; phase 2 merges the slices' candidates.
#pragma once
#include "common.cuh"

namespace msa {

constexpr int kTopkThreads = 256;
constexpr int kTopkPerThread = 16;
constexpr int kTopkSlice = kTopkThreads * kTopkPerThread;  // documents per CTA

__device__ __forceinline__ unsigned long long umax64(unsigned long long a, unsigned long long b) {
  return a > b ? a : b;
}

// Block-wide max of one key per thread (kTopkThreads threads).
__device__ __forceinline__ unsigned long long block_max_key(unsigned long long v,
                                                            unsigned long long *red) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = umax64(v, __shfl_xor_sync(0xffffffffu, v, o));
  if (lane == 0) red[warp] = v;
  __syncthreads();
  if (warp == 0) {
    v = lane < kTopkThreads / 32 ? red[lane] : 0ull;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = umax64(v, __shfl_xor_sync(0xffffffffu, v, o));
    if (lane == 0) red[kTopkThreads / 32] = v;
  }
  __syncthreads();
  return red[kTopkThreads / 32];
}

// k rounds of "take the block's largest key"; only the owner rescans.
// Key 0 means "no document" (never a valid key).
__device__ __forceinline__ void select_topk(unsigned long long (&key)[kTopkPerThread], int k,
                                            unsigned long long *out, unsigned long long *red) {
  unsigned long long m = 0ull;
#pragma unroll
  for (int j = 0; j < kTopkPerThread; ++j) m = umax64(m, key[j]);
  for (int r = 0; r < k; ++r) {
    const unsigned long long w = block_max_key(m, red);
    if (threadIdx.x == 0) out[r] = w;
    if (w != 0ull && m == w) {
      m = 0ull;
#pragma unroll
      for (int j = 0; j < kTopkPerThread; ++j) {
        if (key[j] == w) key[j] = 0ull;
        m = umax64(m, key[j]);
      }
    }
  }
  __syncthreads();
}

__device__ __forceinline__ void write_topk(const unsigned long long *sel, int k, int32_t *ids,
                                           float *scores) {
  for (int r = threadIdx.x; r < k; r += kTopkThreads) {
    const unsigned long long key = sel[r];
    ids[r] = key ? topk_key_id(key) : -1;
    scores[r] = key ? topk_key_score(key) : -INFINITY;
  }
}

// grid (n_split, B).  With n_split == 1 the result goes straight to ids/scores.
__global__ void __launch_bounds__(kTopkThreads)
topk_partial_kernel(const float *__restrict__ state, const uint8_t *__restrict__ exclude,
                    int n_docs, int k, int n_split, unsigned long long *__restrict__ cand,
                    int32_t *__restrict__ ids, float *__restrict__ scores) {
  __shared__ unsigned long long red[kTopkThreads / 32 + 1];
  __shared__ unsigned long long sel[kMaxTopK];
  const int b = blockIdx.y, split = blockIdx.x;
  const int64_t row = static_cast<int64_t>(b) * n_docs;
  unsigned long long key[kTopkPerThread];
#pragma unroll
  for (int j = 0; j < kTopkPerThread; ++j) {
    const int d = split * kTopkSlice + j * kTopkThreads + threadIdx.x;
    bool ok = d < n_docs;
    if (ok && exclude != nullptr) ok = exclude[row + d] == 0;
    key[j] = ok ? topk_key(state[row + d], d) : 0ull;
  }
  select_topk(key, k, sel, red);
  if (n_split == 1) {
    write_topk(sel, k, ids + static_cast<int64_t>(b) * k, scores + static_cast<int64_t>(b) * k);
  } else {
    unsigned long long *dst = cand + (static_cast<int64_t>(b) * n_split + split) * k;
    for (int r = threadIdx.x; r < k; r += kTopkThreads) dst[r] = sel[r];
  }
}

// grid (B).  n_cand = n_split * k <= kTopkSlice.
__global__ void __launch_bounds__(kTopkThreads)
topk_merge_kernel(const unsigned long long *__restrict__ cand, int n_cand, int k,
                  int32_t *__restrict__ ids, float *__restrict__ scores) {
  __shared__ unsigned long long red[kTopkThreads / 32 + 1];
  __shared__ unsigned long long sel[kMaxTopK];
  const int b = blockIdx.x;
  unsigned long long key[kTopkPerThread];
#pragma unroll
  for (int j = 0; j < kTopkPerThread; ++j) {
    const int i = j * kTopkThreads + threadIdx.x;
    key[j] = i < n_cand ? cand[static_cast<int64_t>(b) * n_cand + i] : 0ull;
  }
  select_topk(key, k, sel, red);
  write_topk(sel, k, ids + static_cast<int64_t>(b) * k, scores + static_cast<int64_t>(b) * k);
}

__global__ void fill_kernel(float *__restrict__ p, int64_t n, float v) {
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < n;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x)
    p[i] = v;
}

}  // namespace msa
