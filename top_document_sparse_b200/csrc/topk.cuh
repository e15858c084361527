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
constexpr int kTopkWarps = kTopkThreads / 32;
constexpr int kTopkPerThread = 16;
constexpr int kTopkSlice = kTopkThreads * kTopkPerThread;  // documents per CTA

__device__ __forceinline__ unsigned long long umax64(unsigned long long a, unsigned long long b) {
  return a > b ? a : b;
}

// Warp-wide max of one 64-bit key per lane: max of the high words, then max of
// the low words among the lanes holding that high word (two redux.sync).
__device__ __forceinline__ unsigned long long warp_max_key(unsigned long long v) {
  const unsigned hi = static_cast<unsigned>(v >> 32), lo = static_cast<unsigned>(v);
  const unsigned hmax = __reduce_max_sync(0xffffffffu, hi);
  const unsigned lmax = __reduce_max_sync(0xffffffffu, hi == hmax ? lo : 0u);
  return (static_cast<unsigned long long>(hmax) << 32) | lmax;
}

// k rounds of "take the warp's largest key" over the lanes' key[] registers;
// only the owner lane rescans.  Key 0 means "no document" (never a valid key).
// Lane 0 writes the selection, largest first, to out[0..k).
__device__ __forceinline__ void warp_select_topk(unsigned long long (&key)[kTopkPerThread], int k,
                                                 unsigned long long *out) {
  const int lane = threadIdx.x & 31;
  unsigned long long m = 0ull;
#pragma unroll
  for (int j = 0; j < kTopkPerThread; ++j) m = umax64(m, key[j]);
  for (int r = 0; r < k; ++r) {
    const unsigned long long w = warp_max_key(m);
    if (lane == 0) out[r] = w;
    if (w != 0ull && m == w) {
      m = 0ull;
#pragma unroll
      for (int j = 0; j < kTopkPerThread; ++j) {
        if (key[j] == w) key[j] = 0ull;
        m = umax64(m, key[j]);
      }
    }
  }
}

// Block top-k of the threads' key[] registers: every warp selects its own k,
// then warp 0 selects k among the kTopkWarps * k candidates.  The result is
// left in sel[0..k) (shared).
__device__ __forceinline__ void block_select_topk(unsigned long long (&key)[kTopkPerThread], int k,
                                                  unsigned long long *cand,
                                                  unsigned long long *sel) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  warp_select_topk(key, k, cand + warp * k);
  __syncthreads();
  if (warp == 0) {
#pragma unroll
    for (int j = 0; j < kTopkPerThread; ++j) {
      const int i = j * 32 + lane;
      key[j] = i < kTopkWarps * k ? cand[i] : 0ull;
    }
    warp_select_topk(key, k, sel);
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

// grid (n_split, B).  Warp w of split s holds documents s*kTopkSlice + w*512 +
// j*32 + lane.  With n_split == 1 the result goes straight to ids/scores.
__global__ void __launch_bounds__(kTopkThreads)
topk_partial_kernel(const float *__restrict__ state, const uint8_t *__restrict__ exclude,
                    int n_docs, int k, int n_split, unsigned long long *__restrict__ cand,
                    int32_t *__restrict__ ids, float *__restrict__ scores) {
  __shared__ unsigned long long wc[kTopkWarps * kMaxTopK];
  __shared__ unsigned long long sel[kMaxTopK];
  const int b = blockIdx.y, split = blockIdx.x;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t row = static_cast<int64_t>(b) * n_docs;
  unsigned long long key[kTopkPerThread];
#pragma unroll
  for (int j = 0; j < kTopkPerThread; ++j) {
    const int d = split * kTopkSlice + warp * (32 * kTopkPerThread) + j * 32 + lane;
    bool ok = d < n_docs;
    if (ok && exclude != nullptr) ok = exclude[row + d] == 0;
    key[j] = ok ? topk_key(state[row + d], d) : 0ull;
  }
  block_select_topk(key, k, wc, sel);
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
  __shared__ unsigned long long wc[kTopkWarps * kMaxTopK];
  __shared__ unsigned long long sel[kMaxTopK];
  const int b = blockIdx.x;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  unsigned long long key[kTopkPerThread];
#pragma unroll
  for (int j = 0; j < kTopkPerThread; ++j) {
    const int i = warp * (32 * kTopkPerThread) + j * 32 + lane;
    key[j] = i < n_cand ? cand[static_cast<int64_t>(b) * n_cand + i] : 0ull;
  }
  block_select_topk(key, k, wc, sel);
  write_topk(sel, k, ids + static_cast<int64_t>(b) * k, scores + static_cast<int64_t>(b) * k);
}

__global__ void fill_kernel(float *__restrict__ p, int64_t n, float v) {
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < n;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x)
    p[i] = v;
}

}  // namespace msa
