// tier.cuh -- host tier of the pooled content (MSA, Evermind summary sec. 4B
// "Memory Parallel & Tiered Storage": routing keys stay in GPU memory, the
// content K/V lives in host DRAM and only the selected top-k documents are
// brought to the GPU, asynchronously; b-lab.team item 2, KV cache compression).
//
// A fetcher owns the bookkeeping of a device slot cache: slot s holds one
// document's pooled rows (max_doc_chunks rows of [2][H_kv][D]) at
// slot_cache + s * slot_bytes.  For a batch of top-k ids it reads the ids back
// (one small device-to-host copy), finds the documents already resident,
// chooses victim slots for the rest (a clock over slots not used by this
// call), and on the fetch stream uploads the list of missing documents and
// the per-(query, rank) slot table, then copies every missing document with
// one gather kernel that reads the pinned content through its device mapping
// (each CTA pulls one document's contiguous rows over the host link; per-
// document cudaMemcpyAsync calls cost several microseconds each and capped the
// link at a few GB/s).  When the content is not mapped into the device address
// space it falls back to one cudaMemcpyAsync per document.  The main stream
// then waits for the fetch stream; the attention kernels read rank r of query
// b from slot slots[b][r].
#pragma once
#include <vector>

#include "common.cuh"

struct msa_fetcher {
  const msa_memory *mem = nullptr;
  const uint8_t *content_host = nullptr;  // pinned, [C][2][H_kv][D]
  uint8_t *slot_cache = nullptr;          // device, n_slots * slot_bytes
  int32_t n_slots = 0, max_batch = 0, max_k = 0;
  uint32_t flags = 0;
  size_t row_bytes = 0, slot_bytes = 0;
  std::vector<int32_t> doc_slot;    // [n_docs] -> slot or -1
  std::vector<int32_t> slot_doc;    // [n_slots] -> doc or -1
  std::vector<int64_t> slot_stamp;  // [n_slots] last call that used the slot
  int64_t stamp = 0;
  int32_t hand = 0;
  int32_t *h_ids = nullptr, *h_slots = nullptr;  // pinned [max_batch * max_k]
  int32_t *d_slots = nullptr;                     // device [max_batch * max_k]
  const uint8_t *content_dev = nullptr;  // device address of content_host (null: not mapped)
  int64_t *h_list = nullptr, *d_list = nullptr;  // [max_batch * max_k][3]: src, bytes, dst
  cudaEvent_t ev_ids = nullptr, ev_fetch = nullptr;
  int64_t hits = 0, misses = 0, bytes = 0, copies = 0;
};

namespace msa {

// grid (missing documents), block 256: document i's rows, list[i] = {source
// byte offset in the content, bytes, destination byte offset in the slot
// cache}; 16-byte loads from the host-mapped content, four in flight per
// thread.
__global__ void __launch_bounds__(256)
fetch_gather_kernel(const uint8_t *__restrict__ content, uint8_t *__restrict__ slots,
                    const int64_t *__restrict__ list) {
  const int64_t src = list[3 * blockIdx.x], n16 = list[3 * blockIdx.x + 1] / 16,
                dst = list[3 * blockIdx.x + 2];
  const uint4 *s = reinterpret_cast<const uint4 *>(content + src);
  uint4 *d = reinterpret_cast<uint4 *>(slots + dst);
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
