// topk.cuh -- global top-k over documents (MSA, b-lab.team summary item 1:
// the k most relevant documents are selected; Evermind sec. 2).
// Order: score descending, then document id ascending (ties go to the lower
// id).  Each (score, id) pair is packed into one order-preserving 64-bit key,
// so the top-k is a selection of the k largest keys -- exact and
// deterministic.  Phase 1: one CTA per (query, 4096-document slice) selects
// its slice's k largest keys (a memory of at most 2,048 documents: one
// 128-thread CTA per query, no phase 2); phase 2 merges the slices'
// candidates.  Both filter first (block_select_topk_fast) and sort only the
// few survivors.  topk_merge_shards_kernel merges the candidates of several
// memory shards (Memory Parallel).
#pragma once
#include "common.cuh"
#include "ptx.cuh"

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
// k largest keys, descending, end in sel[0..k).  NTHR: the block's threads (a
// multiple of 32, at most 1024); cand holds NTHR / 32 lists of KL keys.
template <int KL, int NTHR = kTopkThreads>
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
    constexpr int NW = NTHR / 32;
    constexpr int NWP = NW <= 1 ? 1 : NW <= 2 ? 2 : NW <= 4 ? 4 : NW <= 8 ? 8 : NW <= 16 ? 16 : 32;
#pragma unroll
    for (int i = 0; i < KL; ++i) a[i] = lane < NW ? cand[lane * KL + i] : 0ull;
#pragma unroll
    for (int o = NWP >> 1; o > 0; o >>= 1) merge_with_lane<KL>(a, o);
    if (lane == 0)
      for (int i = 0; i < k; ++i) sel[i] = a[i];
  }
  __syncthreads();
}

// --- filtered selection ------------------------------------------------------
// For k <= 32 most keys cannot be in the top k and need no sorting.  Each lane
// takes the max of its keys; each warp sorts its 32 lane maxima (a 15-step
// shuffle network) and its k-th largest t_w bounds the warp's own top k from
// below: at least k of its keys are >= t_w (t_w = 1, i.e. every valid key,
// when fewer than k lanes hold a key).  So the block holds at least k keys >=
// T = max_w t_w and its top k are among them.  Those candidates (usually a few
// more than k) are compacted into shared memory and ranked by counting (keys
// are unique).  When they overflow kTopkCandCap (an adversarial layout of the
// keys over the lanes) the block falls back to the sorting network above, so
// the result is exact either way.
constexpr int kTopkCandCap = 512;

// descending bitonic sort of one key per lane across the warp
__device__ __forceinline__ unsigned long long warp_sort_desc(unsigned long long v, int lane) {
#pragma unroll
  for (int size = 2; size <= 32; size <<= 1)
#pragma unroll
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      const unsigned long long o = __shfl_xor_sync(0xffffffffu, v, stride);
      const bool keep_max = ((lane & stride) == 0) == ((lane & size) == 0);
      v = keep_max ? (v > o ? v : o) : (v < o ? v : o);
    }
  return v;
}

// Same contract as block_select_topk.  Shared scratch: wt[NTHR / 32] and
// cbuf[kTopkCandCap] besides block_select_topk's.
template <int KL, int NTHR = kTopkThreads>
__device__ __forceinline__ void block_select_topk_fast(
    const unsigned long long (&key)[kTopkPerThread], int k, unsigned long long *cand,
    unsigned long long *sel, unsigned long long *wt, unsigned long long *cbuf) {
  constexpr int NW = NTHR / 32;
  if (k > 32) {
    block_select_topk<KL, NTHR>(key, k, cand, sel);
    return;
  }
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  unsigned long long m = 0ull;
#pragma unroll
  for (int j = 0; j < kTopkPerThread; ++j) m = key[j] > m ? key[j] : m;
  m = warp_sort_desc(m, lane);
  const unsigned long long tw = __shfl_sync(0xffffffffu, m, k - 1);
  if (lane == 0) wt[warp] = tw ? tw : 1ull;
  __syncthreads();
  unsigned long long T = 1ull;
#pragma unroll
  for (int w = 0; w < NW; ++w) T = wt[w] > T ? wt[w] : T;
  // compact the keys >= T: per-thread counts, a warp scan and a block prefix
  // over the warps' totals give every thread its first slot (no atomics)
  __shared__ unsigned warp_n[NW];
  unsigned c = 0;
#pragma unroll
  for (int j = 0; j < kTopkPerThread; ++j) c += key[j] >= T ? 1u : 0u;
  unsigned inc = c;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const unsigned v = __shfl_up_sync(0xffffffffu, inc, o);
    if (lane >= o) inc += v;
  }
  if (lane == 31) warp_n[warp] = inc;
  __syncthreads();
  unsigned n = 0, pos = inc - c;
#pragma unroll
  for (int w = 0; w < NW; ++w) {
    const unsigned x = warp_n[w];
    pos += w < warp ? x : 0u;
    n += x;
  }
  if (n > kTopkCandCap) {  // uniform: every thread summed the same totals
    block_select_topk<KL, NTHR>(key, k, cand, sel);
    return;
  }
#pragma unroll
  for (int j = 0; j < kTopkPerThread; ++j)
    if (key[j] >= T) cbuf[pos++] = key[j];
  __syncthreads();
  // rank by counting: every thread reads the same cbuf entry at once (a
  // shared-memory broadcast)
  for (unsigned i = threadIdx.x; i < n; i += NTHR) {
    const unsigned long long x = cbuf[i];
    int r = 0;
#pragma unroll 8
    for (unsigned j2 = 0; j2 < n; ++j2) r += cbuf[j2] > x ? 1 : 0;
    if (r < k) sel[r] = x;
  }
  for (int r = static_cast<int>(n) + threadIdx.x; r < k; r += NTHR) sel[r] = 0ull;
  __syncthreads();
}

template <int NTHR = kTopkThreads>
__device__ __forceinline__ void write_topk(const unsigned long long *sel, int k, int32_t *ids,
                                           float *scores) {
  for (int r = threadIdx.x; r < k; r += NTHR) {
    const unsigned long long key = sel[r];
    ids[r] = key ? topk_key_id(key) : -1;
    scores[r] = key ? topk_key_score(key) : -INFINITY;
  }
}

// grid (n_split, B).  Warp w of split s holds documents s*kTopkSlice + w*512 ..
// + 511 (lane l: four runs of 4 from 4 l when the row can be read as float4,
// else l + 32 j).  With n_split == 1 the result goes straight to ids/scores.
// NTHR threads per CTA (a slice of NTHR x kTopkPerThread documents): 128 for a
// memory of at most 2,048 documents, so no warp joins the barriers empty-handed.
template <int KL, int NTHR = kTopkThreads>
__global__ void __launch_bounds__(NTHR)
topk_partial_kernel(const float *__restrict__ state, const uint8_t *__restrict__ exclude,
                    int n_docs, int k, int n_split, unsigned long long *__restrict__ cand,
                    int32_t *__restrict__ ids, float *__restrict__ scores) {
  __shared__ unsigned long long wc[(NTHR / 32) * KL];
  __shared__ unsigned long long sel[kMaxTopK];
  __shared__ unsigned long long wt[NTHR / 32 + 1], cbuf[kTopkCandCap];
  const int b = blockIdx.y, split = blockIdx.x;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t row = static_cast<int64_t>(b) * n_docs;
  griddep_wait();
  griddep_launch();
  unsigned long long key[kTopkPerThread];
  const int dw = split * (NTHR * kTopkPerThread) + warp * (32 * kTopkPerThread);
  if (exclude == nullptr && (n_docs & 3) == 0 && (reinterpret_cast<uintptr_t>(state) & 15) == 0) {
    // four 16-byte loads per thread: lane takes documents dw + 128 j4 + 4 lane + 0..3
    // (n_docs % 4 == 0, so a vector is either wholly inside the row or wholly past it)
#pragma unroll
    for (int j4 = 0; j4 < kTopkPerThread / 4; ++j4) {
      const int d = dw + j4 * 128 + lane * 4;
      float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
      if (d < n_docs) v = *reinterpret_cast<const float4 *>(state + row + d);
      const bool ok = d < n_docs;
      key[4 * j4 + 0] = ok ? topk_key(v.x, d + 0) : 0ull;
      key[4 * j4 + 1] = ok ? topk_key(v.y, d + 1) : 0ull;
      key[4 * j4 + 2] = ok ? topk_key(v.z, d + 2) : 0ull;
      key[4 * j4 + 3] = ok ? topk_key(v.w, d + 3) : 0ull;
    }
  } else if (exclude == nullptr) {
#pragma unroll
    for (int j = 0; j < kTopkPerThread; ++j) {
      const int d = dw + j * 32 + lane;
      key[j] = d < n_docs ? topk_key(state[row + d], d) : 0ull;
    }
  } else {
#pragma unroll
    for (int j = 0; j < kTopkPerThread; ++j) {
      const int d = dw + j * 32 + lane;
      const bool ok = d < n_docs && exclude[row + d] == 0;
      key[j] = ok ? topk_key(state[row + d], d) : 0ull;
    }
  }
  block_select_topk_fast<KL, NTHR>(key, k, wc, sel, wt, cbuf);
  if (n_split == 1) {
    write_topk<NTHR>(sel, k, ids + static_cast<int64_t>(b) * k,
                     scores + static_cast<int64_t>(b) * k);
  } else {
    unsigned long long *dst = cand + (static_cast<int64_t>(b) * n_split + split) * k;
    for (int r = threadIdx.x; r < k; r += NTHR) dst[r] = sel[r];
  }
}

// grid (B).  n_cand = n_split * k <= kTopkSlice.
template <int KL>
__global__ void __launch_bounds__(kTopkThreads)
topk_merge_kernel(const unsigned long long *__restrict__ cand, int n_cand, int k,
                  int32_t *__restrict__ ids, float *__restrict__ scores) {
  __shared__ unsigned long long wc[kTopkWarps * KL];
  __shared__ unsigned long long sel[kMaxTopK];
  __shared__ unsigned long long wt[kTopkWarps + 1], cbuf[kTopkCandCap];
  const int b = blockIdx.x;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  griddep_wait();
  griddep_launch();
  unsigned long long key[kTopkPerThread];
#pragma unroll
  for (int j = 0; j < kTopkPerThread; ++j) {
    const int i = warp * (32 * kTopkPerThread) + j * 32 + lane;
    key[j] = i < n_cand ? cand[static_cast<int64_t>(b) * n_cand + i] : 0ull;
  }
  block_select_topk_fast<KL>(key, k, wc, sel, wt, cbuf);
  write_topk(sel, k, ids + static_cast<int64_t>(b) * k, scores + static_cast<int64_t>(b) * k);
}

// --- Memory Parallel ------------------------------------------------------------
// The memory's documents are split into contiguous ranges (shards, one per GPU
// in the pages' engine: Evermind summary sec. 4B "Memory Parallel & Tiered
// Storage"; b-lab.team item 2); each shard routes its own documents and keeps
// its top k_cand as (score, local id).  The global top-k is the k largest
// (score, base + local id) keys over all shards' candidates: the global top-k
// documents are each in their own shard's top k_cand (k_cand >= k), and the
// keys order exactly as the single-memory top-k orders them, so the result is
// bit-identical to routing the whole memory at once.
constexpr int kMaxShards = 64;
struct ShardBases {
  int32_t base[kMaxShards];  // global id of each shard's document 0
};

// grid (B).  cand_* [n_shards][B][k_cand]; ids < 0 are padding.  n_shards *
// k_cand <= kTopkSlice.
template <int KL>
__global__ void __launch_bounds__(kTopkThreads)
topk_merge_shards_kernel(const float *__restrict__ cand_scores,
                         const int32_t *__restrict__ cand_ids, int n_shards, int B, int k_cand,
                         ShardBases bases, int k, int32_t *__restrict__ ids,
                         float *__restrict__ scores) {
  __shared__ unsigned long long wc[kTopkWarps * KL];
  __shared__ unsigned long long sel[kMaxTopK];
  __shared__ unsigned long long wt[kTopkWarps + 1], cbuf[kTopkCandCap];
  const int b = blockIdx.x;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  griddep_wait();
  griddep_launch();
  const int n_cand = n_shards * k_cand;
  unsigned long long key[kTopkPerThread];
#pragma unroll
  for (int j = 0; j < kTopkPerThread; ++j) {
    const int i = warp * (32 * kTopkPerThread) + j * 32 + lane;
    key[j] = 0ull;
    if (i < n_cand) {
      const int s = i / k_cand, r = i - s * k_cand;
      const int64_t src = (static_cast<int64_t>(s) * B + b) * k_cand + r;
      const int32_t id = cand_ids[src];
      if (id >= 0) key[j] = topk_key(cand_scores[src], bases.base[s] + id);
    }
  }
  block_select_topk_fast<KL>(key, k, wc, sel, wt, cbuf);
  write_topk(sel, k, ids + static_cast<int64_t>(b) * k, scores + static_cast<int64_t>(b) * k);
}

__global__ void fill_kernel(float *__restrict__ p, int64_t n, float v) {
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < n;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x)
    p[i] = v;
}

}  // namespace msa
