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

// --- sorting-network selection ------------------------------------------
// Each lane keeps a list of KL keys sorted in descending order.  Two lanes'
// lists are combined into the KL largest of their union by reversing one list,
// taking elementwise maxima (a bitonic sequence holding the KL largest) and
// sorting that with a bitonic merge network.  Five such butterfly rounds over
// the warp leave every lane with the warp's KL largest keys; no step depends
// on k serially.

template <int KL>
__device__ __forceinline__ void cas_desc(unsigned long long (&a)[KL], int i, int j) {
  const unsigned long long x = a[i], y = a[j];
  a[i] = x > y ? x : y;
  a[j] = x > y ? y : x;
}

// full bitonic sort, descending, of a[0..KL)
template <int KL>
__device__ __forceinline__ void sort_desc(unsigned long long (&a)[KL]) {
#pragma unroll
  for (int size = 2; size <= KL; size <<= 1)
#pragma unroll
    for (int stride = size >> 1; stride > 0; stride >>= 1)
#pragma unroll
      for (int i = 0; i < KL; ++i) {
        const int j = i ^ stride;
        if (j > i) {
          // descending within blocks whose (i & size) == 0, ascending otherwise
          if ((i & size) == 0) cas_desc<KL>(a, i, j); else cas_desc<KL>(a, j, i);
        }
      }
}

// a bitonic sequence -> sorted descending
template <int KL>
__device__ __forceinline__ void bitonic_merge_desc(unsigned long long (&a)[KL]) {
#pragma unroll
  for (int stride = KL >> 1; stride > 0; stride >>= 1)
#pragma unroll
    for (int i = 0; i < KL; ++i) {
      const int j = i ^ stride;
      if (j > i) cas_desc<KL>(a, i, j);
    }
}

// the KL largest of this lane's list and the list of lane ^ offset
template <int KL>
__device__ __forceinline__ void merge_with_lane(unsigned long long (&a)[KL], int offset) {
  unsigned long long b[KL];
#pragma unroll
  for (int i = 0; i < KL; ++i) b[i] = __shfl_xor_sync(0xffffffffu, a[KL - 1 - i], offset);
#pragma unroll
  for (int i = 0; i < KL; ++i) a[i] = a[i] > b[i] ? a[i] : b[i];
  bitonic_merge_desc<KL>(a);
}

// Block top-k (k <= KL) of the threads' key[] registers (kTopkPerThread each):
// per-lane sort, warp butterflies, then warp 0 merges the warps' lists.  The
// k largest keys, descending, end in sel[0..k).
template <int KL>
__device__ __forceinline__ void block_select_topk(const unsigned long long (&key)[kTopkPerThread],
                                                  int k, unsigned long long *cand,
                                                  unsigned long long *sel) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  unsigned long long a[KL];
#pragma unroll
  for (int i = 0; i < KL; ++i) a[i] = i < kTopkPerThread ? key[i] : 0ull;
  sort_desc<KL>(a);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) merge_with_lane<KL>(a, o);
  if (lane == 0) {
#pragma unroll
    for (int i = 0; i < KL; ++i) cand[warp * KL + i] = a[i];
  }
  __syncthreads();
  if (warp == 0) {
#pragma unroll
    for (int i = 0; i < KL; ++i) a[i] = lane < kTopkWarps ? cand[lane * KL + i] : 0ull;
#pragma unroll
    for (int o = kTopkWarps >> 1; o > 0; o >>= 1) merge_with_lane<KL>(a, o);
    if (lane == 0)
      for (int i = 0; i < k; ++i) sel[i] = a[i];
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
template <int KL>
__global__ void __launch_bounds__(kTopkThreads)
topk_partial_kernel(const float *__restrict__ state, const uint8_t *__restrict__ exclude,
                    int n_docs, int k, int n_split, unsigned long long *__restrict__ cand,
                    int32_t *__restrict__ ids, float *__restrict__ scores) {
  __shared__ unsigned long long wc[kTopkWarps * KL];
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
  block_select_topk<KL>(key, k, wc, sel);
  if (n_split == 1) {
    write_topk(sel, k, ids + static_cast<int64_t>(b) * k, scores + static_cast<int64_t>(b) * k);
  } else {
    unsigned long long *dst = cand + (static_cast<int64_t>(b) * n_split + split) * k;
    for (int r = threadIdx.x; r < k; r += kTopkThreads) dst[r] = sel[r];
  }
}

// grid (B).  n_cand = n_split * k <= kTopkSlice.
template <int KL>
__global__ void __launch_bounds__(kTopkThreads)
topk_merge_kernel(const unsigned long long *__restrict__ cand, int n_cand, int k,
                  int32_t *__restrict__ ids, float *__restrict__ scores) {
  __shared__ unsigned long long wc[kTopkWarps * KL];
  __shared__ unsigned long long sel[kMaxTopK];
  const int b = blockIdx.x;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  unsigned long long key[kTopkPerThread];
#pragma unroll
  for (int j = 0; j < kTopkPerThread; ++j) {
    const int i = warp * (32 * kTopkPerThread) + j * 32 + lane;
    key[j] = i < n_cand ? cand[static_cast<int64_t>(b) * n_cand + i] : 0ull;
  }
  block_select_topk<KL>(key, k, wc, sel);
  write_topk(sel, k, ids + static_cast<int64_t>(b) * k, scores + static_cast<int64_t>(b) * k);
}

__global__ void fill_kernel(float *__restrict__ p, int64_t n, float v) {
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < n;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x)
    p[i] = v;
}

}  // namespace msa
