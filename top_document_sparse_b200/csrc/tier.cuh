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
// call), issues one cudaMemcpyAsync per missing document on the fetch stream,
// uploads the per-(query, rank) slot table, and makes the main stream wait for
// the fetch stream.  The attention kernels then read rank r of query b from
// slot slots[b][r].
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
  cudaEvent_t ev_ids = nullptr, ev_fetch = nullptr;
  int64_t hits = 0, misses = 0, bytes = 0, copies = 0;
};
