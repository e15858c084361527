// tier.cuh -- host tier of the pooled content (MSA, Evermind summary sec. 4B
// "Memory Parallel & Tiered Storage": routing keys stay in GPU memory, the
// content K/V lives in host DRAM and only the selected top-k documents are
// brought to the GPU, asynchronously; b-lab.team item 2, KV cache compression).
//
// A fetcher keeps a device slot cache: slot s holds one document's pooled rows
// (max_doc_chunks rows of [2][H_kv][D]) at slot_cache + s * slot_bytes.  Its
// bookkeeping lives in device memory, so a fetch needs no host round trip:
// fetch_assign_kernel (one CTA, on the caller's stream after the top-k) finds
// the documents already resident, gives every missing document a victim slot
// (a clock over the slots this call does not use) and writes the list of
// copies; fetch_gather_kernel (on the fetch stream) copies every missing
// document's contiguous rows from the pinned host content through its device
// mapping, one CTA per document, over the host link.  The attention kernels
// read rank r of query b from slot slots[b][r].
#pragma once
#include "common.cuh"
#include "ptx.cuh"

struct msa_fetcher {
  const msa_memory *mem = nullptr;
  const uint8_t *content_host = nullptr;  // pinned, [C][2][H_kv][D]
  const uint8_t *content_dev = nullptr;   // its device mapping
  uint8_t *slot_cache = nullptr;          // device, n_slots * slot_bytes
  int32_t n_slots = 0, max_batch = 0, max_k = 0;
  uint32_t flags = 0;
  size_t row_bytes = 0, slot_bytes = 0;
  // device bookkeeping
  int32_t *d_doc_slot = nullptr;    // [n_docs] -> slot or -1
  int32_t *d_claim = nullptr;       // [n_docs] lowest (query, rank) index missing it this call
  int32_t *d_slot_doc = nullptr;    // [n_slots] -> doc or -1
  int32_t *d_slot_stamp = nullptr;  // [n_slots] last call that used the slot
  int64_t *d_ctl = nullptr;         // kCtl* below
  int32_t *d_slots = nullptr;       // [max_batch * max_k] slot of each (query, rank)
  int64_t *d_list = nullptr;        // [max_batch * max_k][3]: source, bytes, destination
  int32_t *d_scratch = nullptr;     // [kAssignScratch] the assignment kernel's scratch
  cudaEvent_t ev_ids = nullptr, ev_fetch = nullptr;
};

namespace msa {

// d_ctl entries: call stamp, clock hand, copies of the last call, and the
// totals hits / misses (= copies) / bytes since creation.
enum { kCtlStamp = 0, kCtlHand, kCtlCopies, kCtlHits, kCtlMisses, kCtlBytes, kCtlN };
constexpr int kAssignThreads = 256;
constexpr int kAssignMaxIds = 4096;  // batch * k of one call

// Scratch of the assignment kernel, in device memory (kAssignScratch ints):
// the block scan's warp totals, the victim slots, and three words.  The kernel
// uses no shared memory, so it can run beside a route kernel that holds an
// SM's whole shared memory (a fetch that overlaps the next layer's routing).
constexpr int kAssignScratch = kAssignThreads / 32 + kAssignMaxIds + 4;

// Exclusive prefix sum over the block of one flag per thread; returns this
// thread's offset and sets *total.  `scr` holds kAssignThreads / 32 ints of
// device memory (a __syncthreads makes them visible to the whole block).
__device__ __forceinline__ int block_scan(int flag, volatile int *scr, int *total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int v = flag;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int u = __shfl_up_sync(0xffffffffu, v, o);
    if (lane >= o) v += u;
  }
  if (lane == 31) scr[warp] = v;
  __syncthreads();
  int before = 0, all = 0;
  for (int w = 0; w < kAssignThreads / 32; ++w) {
    const int x = scr[w];
    before += w < warp ? x : 0;
    all += x;
  }
  __syncthreads();  // scr may be reused
  *total = all;
  return before + v - flag;
}

// grid 1, block kAssignThreads.  ids [n] (n <= kAssignMaxIds) -> slots [n].
// Ids outside [0, n_docs) get slot 0 and no copy (the attention skips them
// and raises MSA_DEVERR_BAD_DOC_ID).
__global__ void __launch_bounds__(kAssignThreads)
fetch_assign_kernel(const int32_t *__restrict__ ids, int n, int n_docs,
                    const int64_t *__restrict__ doc_chunk_off, int64_t row_bytes,
                    int64_t slot_bytes, int n_slots, int cold, int32_t *__restrict__ doc_slot,
                    int32_t *__restrict__ claim, int32_t *__restrict__ slot_doc,
                    int32_t *__restrict__ slot_stamp, int64_t *__restrict__ ctl,
                    int64_t *__restrict__ list, int32_t *__restrict__ slots,
                    int *__restrict__ scratch) {
  volatile int *scr = scratch;
  volatile int *victim = scratch + kAssignThreads / 32;
  volatile int *words = victim + kAssignMaxIds;  // call stamp, clock hand, last victim position
  volatile int &s_now = words[0], &s_hand = words[1], &s_last = words[2];
  constexpr int P = kAssignMaxIds / kAssignThreads;  // ids per thread
  const int tid = threadIdx.x;
  griddep_wait();
  griddep_launch();
  if (tid == 0) {
    s_now = static_cast<int>(ctl[kCtlStamp] + 1);
    ctl[kCtlStamp] = s_now;
    s_hand = static_cast<int>(ctl[kCtlHand]);
  }
  if (cold)  // forget every resident document: each one is copied again
    for (int s = tid; s < n_slots; s += kAssignThreads) {
      const int d = slot_doc[s];
      if (d >= 0) doc_slot[d] = -1;
      slot_doc[s] = -1;
    }
  __syncthreads();
  const int now = s_now;
  int d[P];
  bool valid[P], miss[P];
#pragma unroll
  for (int u = 0; u < P; ++u) {
    const int i = tid + u * kAssignThreads;
    d[u] = i < n ? ids[i] : -1;
    valid[u] = d[u] >= 0 && d[u] < n_docs;
    miss[u] = false;
    if (valid[u]) {
      const int s = doc_slot[d[u]];
      if (s >= 0) {
        slot_stamp[s] = now;  // resident: keeps its slot
      } else {
        miss[u] = true;
        atomicMin(claim + d[u], i);  // the lowest index missing the document copies it
      }
    }
  }
  __syncthreads();
  // winners (one per missing document) numbered in index order
  int win_rank[P], n_win = 0;
#pragma unroll
  for (int u = 0; u < P; ++u) {
    const int i = tid + u * kAssignThreads;
    const bool win = miss[u] && claim[d[u]] == i;
    int tot;
    const int r = block_scan(win ? 1 : 0, scr, &tot);
    win_rank[u] = win ? n_win + r : -1;
    n_win += tot;
  }
  // victims: the slots this call does not use, in clock order from the hand
  // (n_slots >= n, so there are at least as many as missing documents)
  if (tid == 0) s_last = -1;
  int found = 0;
  for (int p0 = 0; p0 < n_slots && found < n_win; p0 += kAssignThreads) {
    const int p = p0 + tid;
    const int s = p < n_slots ? (s_hand + p) % n_slots : 0;
    const bool ev = p < n_slots && slot_stamp[s] != now;
    int tot;
    const int r = found + block_scan(ev ? 1 : 0, scr, &tot);
    if (ev && r < n_win) {
      victim[r] = s;
      if (r == n_win - 1) s_last = p;
    }
    found += tot;
  }
  __syncthreads();
  // every winner takes its victim slot and lists its copy
#pragma unroll
  for (int u = 0; u < P; ++u) {
    const int j = win_rank[u];
    if (j < 0) continue;
    const int s = victim[j];
    const int old = slot_doc[s];
    if (old >= 0) doc_slot[old] = -1;  // (a missing document is in no slot)
    slot_doc[s] = d[u];
    doc_slot[d[u]] = s;
    slot_stamp[s] = now;
    const int64_t c0 = doc_chunk_off[d[u]], c1 = doc_chunk_off[d[u] + 1];
    list[3 * j] = c0 * row_bytes;
    list[3 * j + 1] = (c1 - c0) * row_bytes;
    list[3 * j + 2] = static_cast<int64_t>(s) * slot_bytes;
  }
  __syncthreads();
  int64_t copied = 0;
  int n_valid = 0;
#pragma unroll
  for (int u = 0; u < P; ++u) {
    const int i = tid + u * kAssignThreads;
    if (i < n) slots[i] = valid[u] ? doc_slot[d[u]] : 0;
    n_valid += valid[u] ? 1 : 0;
    if (win_rank[u] >= 0) copied += list[3 * win_rank[u] + 1];
  }
  __syncthreads();
#pragma unroll
  for (int u = 0; u < P; ++u)
    if (win_rank[u] >= 0) claim[d[u]] = 0x7FFFFFFF;  // ready for the next call
  // totals
  int tot_valid;
  block_scan(n_valid, scr, &tot_valid);
  unsigned long long cb = static_cast<unsigned long long>(copied);
  cb += __shfl_xor_sync(0xffffffffu, cb, 16);
  cb += __shfl_xor_sync(0xffffffffu, cb, 8);
  cb += __shfl_xor_sync(0xffffffffu, cb, 4);
  cb += __shfl_xor_sync(0xffffffffu, cb, 2);
  cb += __shfl_xor_sync(0xffffffffu, cb, 1);
  if ((tid & 31) == 0 && cb) atomicAdd(reinterpret_cast<unsigned long long *>(ctl + kCtlBytes), cb);
  if (tid == 0) {
    if (n_win > 0) ctl[kCtlHand] = (s_hand + s_last + 1) % n_slots;
    ctl[kCtlCopies] = n_win;
    ctl[kCtlMisses] += n_win;
    ctl[kCtlHits] += tot_valid - n_win;
  }
}

// grid (batch * k), block 256: block i copies document i of the last
// assignment's list when i < its copy count; 16-byte loads from the
// host-mapped content, four in flight per thread.
__global__ void __launch_bounds__(256)
fetch_gather_kernel(const uint8_t *__restrict__ content, uint8_t *__restrict__ slot_cache,
                    const int64_t *__restrict__ list, const int64_t *__restrict__ ctl) {
  if (static_cast<int64_t>(blockIdx.x) >= ctl[kCtlCopies]) return;
  const int64_t src = list[3 * blockIdx.x], n16 = list[3 * blockIdx.x + 1] / 16,
                dst = list[3 * blockIdx.x + 2];
  const uint4 *s = reinterpret_cast<const uint4 *>(content + src);
  uint4 *d = reinterpret_cast<uint4 *>(slot_cache + dst);
  int64_t i = threadIdx.x;
  for (; i + 3 * 256 < n16; i += 4 * 256) {
    uint4 v[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) v[u] = s[i + u * 256];
#pragma unroll
    for (int u = 0; u < 4; ++u) d[i + u * 256] = v[u];
  }
  for (; i < n16; i += 256) d[i] = s[i];
}

}  // namespace msa
