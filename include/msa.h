/*
 * msa.h -- C ABI of libmsa.so, the B200 (sm_100a) hot path of Memory Sparse
 * Attention (MSA).
 *
 * The method (MSA: "Memory Sparse Attention for Efficient End-to-End Memory
 * Model Scaling to 100M Tokens"):
 *   - offline memory encoding: documents are cut into fixed-length chunks and
 *     each chunk's K, V and router key K_r are mean-pooled; keys carry
 *     document-wise RoPE (positions restart at 0 in each document)
 *     [Evermind summary sec. 2; b-lab.team summary item 1 and pipeline stage
 *     "Global Memory Encoding"];
 *   - online routing: cosine similarity between the query's router projection
 *     Q_r and every pooled router key, averaged over router heads, maxed over
 *     query tokens and over a document's chunks, then the top-k documents
 *     [b-lab.team item 1, Scalable Sparse Attention; pipeline stage "Online
 *     Routing & Context Assembly"];
 *   - sparse generation: the selected documents' pooled K/V are placed ahead
 *     of the query's local K/V, the query's positions start at k (Global RoPE),
 *     and attention runs over that context [b-lab.team item 1, Global RoPE;
 *     pipeline stage "Sparse Generation"].
 *
 * Conventions for every call:
 *   - Memory: the CALLER owns every buffer it passes (device memory, or pinned
 *     host memory where stated).  The library never frees caller memory and
 *     allocates device memory only inside msa_memory_create (small index and
 *     RoPE tables, freed by msa_memory_destroy).  Scratch space for a call is
 *     passed in as `workspace`; its size comes from the matching *_workspace_size
 *     query.  Device pointers must be 16-byte aligned.
 *   - Layouts are dense row-major; "token-major" means [token][head][dim].
 *     Element type is the memory's dtype (fp32 or bf16) unless stated;
 *     scores and running states are fp32, ids int32.
 *   - Asynchrony: arguments are validated on the host before anything is
 *     enqueued; work is then enqueued on `stream` and the call returns.  A
 *     rejected call enqueues nothing.
 *   - Errors: every call returns an msa_status; nothing aborts or throws.
 *     msa_last_error() gives a thread-local message for the last failure.
 *     Conditions that only the device can see (an id >= n_docs, a local cache
 *     that would overflow, a bounded wait that ran out) are recorded in a
 *     device error word and skipped; msa_device_error() reads and clears it.
 *   - Threads: a msa_memory handle is immutable after creation and may be
 *     used from several threads; calls that share output buffers must be
 *     ordered by the caller.
 */
#ifndef MSA_H_
#define MSA_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define MSA_API __attribute__((visibility("default")))
#else
#define MSA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* cudaStream_t; NULL means the legacy default stream. */
typedef struct CUstream_st *msa_stream;

typedef enum {
  MSA_OK = 0,
  MSA_ERR_INVALID_ARG = 1,   /* a bad argument; nothing was enqueued */
  MSA_ERR_UNSUPPORTED = 2,   /* a shape this build has no kernel for */
  MSA_ERR_CUDA = 3,          /* a CUDA runtime error (launch or copy) */
  MSA_ERR_OUT_OF_MEMORY = 4, /* msa_memory_create could not allocate its tables */
  MSA_ERR_TIMEOUT = 5,       /* a bounded device wait ran out (device error word) */
  MSA_ERR_STATE = 6,         /* a device-side bounds check fired (device error word) */
} msa_status;

typedef enum { MSA_F32 = 0, MSA_BF16 = 1 } msa_dtype;

/* Device error word bits reported by msa_device_error(). */
#define MSA_DEVERR_BAD_DOC_ID 0x1u      /* an id outside [0, n_docs) reached attention */
#define MSA_DEVERR_CACHE_OVERFLOW 0x2u  /* cache_len + tokens > cache_capacity */
#define MSA_DEVERR_WAIT_TIMEOUT 0x4u    /* a pipeline barrier wait ran out */

/*
 * The memory's shape.  Documents [Evermind sec. 2: the corpus is split into
 * documents, each cut into fixed-length chunks]:
 *   doc_token_offsets : HOST array [n_docs + 1], offsets[0] = 0, strictly
 *                       increasing (no empty document); copied at create.
 *   chunk_len         : tokens per chunk (2..64); the last chunk of a document
 *                       may be shorter and is averaged over its own length.
 * Content K/V: n_kv_heads x head_dim (head_dim 64 or 128).  Router keys:
 * n_router_heads x router_dim (router_dim 16..128, a power of two;
 * n_router_heads * router_dim a multiple of 64 for bf16).
 * rope_theta: RoPE base (NeoX rotate-half); the pages give none, 1e6 is the
 * Qwen3 value.  max_local_position: local (query/decode) RoPE positions must
 * stay below this; document positions are covered automatically.
 */
typedef struct {
  int32_t n_docs;
  const int64_t *doc_token_offsets;
  int32_t chunk_len;
  int32_t n_kv_heads;
  int32_t head_dim;
  int32_t n_router_heads;
  int32_t router_dim;
  msa_dtype dtype;
  double rope_theta;
  int32_t max_local_position;
} msa_memory_config;

typedef struct msa_memory msa_memory;

typedef struct {
  int64_t n_tokens;
  int64_t n_chunks;          /* total chunks C */
  int32_t max_doc_chunks;    /* chunks of the longest document */
  int64_t max_doc_tokens;
  size_t elem_bytes;         /* 4 (fp32) or 2 (bf16) */
  size_t router_key_bytes;   /* router store [C][H_r][d_r] */
  size_t content_bytes;      /* content store [C][2][H_kv][D]: K then V per chunk */
  size_t doc_content_stride; /* bytes of one document's content at max_doc_chunks */
} msa_memory_info;

/* Build the memory description and its device tables (chunk->document map,
 * document offsets, fp32 RoPE cos/sin table computed in fp64) on the current
 * CUDA device.  Errors: INVALID_ARG (bad config), UNSUPPORTED (shape without a
 * kernel), OUT_OF_MEMORY, CUDA. */
MSA_API msa_status msa_memory_create(const msa_memory_config *cfg, msa_memory **out);
MSA_API msa_status msa_memory_destroy(msa_memory *mem);
MSA_API msa_status msa_memory_get_info(const msa_memory *mem, msa_memory_info *out);
/* First chunk of every document, written to the HOST array out[n_docs + 1]. */
MSA_API msa_status msa_memory_doc_chunk_offsets(const msa_memory *mem, int64_t *out);

/*
 * Offline encoding of documents [doc_begin, doc_begin + doc_count)
 * [b-lab.team pipeline stage "Global Memory Encoding"; Evermind sec. 2 chunk
 * mean pooling; b-lab.team item 1 Document-wise RoPE].
 *   K, V   : device, token-major [n][n_kv_heads][head_dim], K before RoPE
 *   Kr     : device, token-major [n][n_router_heads][router_dim]
 *            where n = tokens of those documents; row 0 is the first token of
 *            document doc_begin.
 * Writes, for every chunk c of those documents:
 *   content[c][0] = mean over the chunk of RoPE(K_t, t - doc_start)
 *   content[c][1] = mean of V_t
 *   router_keys[c][h] = mean of Kr_t over the chunk, divided by
 *                       max(|mean|, 1e-12) per router head: the pooled router
 *                       key stored with unit norm, so routing needs no norms
 *   router_mean[c][h] (optional, may be NULL) = the un-normalised mean.
 * content may be device memory or pinned host memory (written in place over
 * the host link).  Sums are fp32 pairwise trees; stores round to nearest even.
 */
MSA_API msa_status msa_encode_memory(const msa_memory *mem, int32_t doc_begin,
                             int32_t doc_count, const void *K, const void *V,
                             const void *Kr, void *router_keys, void *content,
                             void *router_mean, msa_stream stream);

/* Fill a running routing state (fp32, `count` entries) with -inf. */
MSA_API msa_status msa_route_reset(float *state, int64_t count, msa_stream stream);

/* Scratch bytes msa_route needs for this batch / tokens / k. */
MSA_API size_t msa_route_workspace_size(const msa_memory *mem, int32_t batch,
                                int32_t tokens, int32_t k);

/*
 * Online routing [b-lab.team item 1 and stage "Online Routing & Context
 * Assembly"]:
 *   s[b,t,c]   = (1/H_r) sum_h <Qr[b,t,h], Kr_c,h> / (|Qr[b,t,h]| |Kr_c,h|)
 *   state[b,d] = max(state[b,d], max_{t < tokens, c in chunks(d)} s[b,t,c])
 *   ids[b,:]   = the k documents with the largest state[b,.] by (score
 *                descending, id ascending), excluding documents whose
 *                exclude[b,d] != 0; scores[b,:] their states.
 *   router_keys : device [C][H_r][d_r] as written by msa_encode_memory
 *   Qr          : device [batch][tokens][H_r][d_r]; tokens may be 0 (top-k
 *                 of the state only).  Read as soon as the call's first
 *                 kernel starts, which can be before the previous kernel of
 *                 this library on the stream has completed (programmatic
 *                 dependent launch): Qr must not be an output of the
 *                 previous msa_* call on the same stream
 *   state       : device [batch][n_docs] fp32, read and updated (the running
 *                 max over every token routed so far; reset with -inf)
 *   exclude     : device [batch][n_docs] uint8 or NULL
 *   ids, scores : device [batch][k]; k in [1, min(n_docs, 64)]
 * Errors: INVALID_ARG (k out of range, fewer eligible documents than k is NOT
 * checked: excluded documents then fill the tail with -inf scores), CUDA.
 */
MSA_API msa_status msa_route(const msa_memory *mem, const void *router_keys,
                     const void *Qr, int32_t batch, int32_t tokens, int32_t k,
                     const uint8_t *exclude, float *state, int32_t *ids,
                     float *scores, void *workspace, size_t workspace_bytes,
                     msa_stream stream);

/* Scratch bytes msa_sparse_attend needs. */
MSA_API size_t msa_attend_workspace_size(const msa_memory *mem, int32_t batch,
                                 int32_t tokens, int32_t k, int32_t n_q_heads);

/*
 * Sparse generation [b-lab.team item 1 Scalable Sparse Attention and Global
 * RoPE; stage "Sparse Generation"].  For query b, its `tokens` new tokens are
 * appended to the local cache and attend over
 *   [pooled K/V of every chunk of ids[b,0..k-1], in rank order, all visible]
 *   ++ [local cache rows 0..j] (causal: new token i sits at local index
 *      j = cache_len[b] + i)
 * with Q and the new K rotated at position pos_offset + j (pos_offset = k is
 * the pages' Global RoPE), softmax scale 1/sqrt(head_dim), and query head h
 * reading kv head h / (n_q_heads / n_kv_heads).
 *   content        : device [C][2][H_kv][D] (msa_encode_memory's store)
 *   ids            : device [batch][k] int32
 *   Q              : device [batch][tokens][n_q_heads][D], before RoPE
 *   K_new, V_new   : device [batch][tokens][H_kv][D], K before RoPE
 *   K_cache, V_cache : device [batch][cache_capacity][H_kv][D]; rows below
 *                    cache_len[b] are read (K already rotated), the new rows
 *                    are written
 *   cache_len      : device [batch] int32, advanced by `tokens` when the work
 *                    completes (stream order)
 *   O              : device [batch][tokens][n_q_heads][D]
 * Requires pos_offset >= 0 and pos_offset + cache_capacity <=
 * max_local_position; n_q_heads a multiple of n_kv_heads with a group of at
 * most 16.  A cache that would overflow or an id out of range is skipped and
 * flagged in the device error word.
 */
MSA_API msa_status msa_sparse_attend(const msa_memory *mem, const void *content,
                             const int32_t *ids, int32_t batch, int32_t k,
                             int32_t tokens, int32_t n_q_heads, const void *Q,
                             const void *K_new, const void *V_new,
                             void *K_cache, void *V_cache, int32_t *cache_len,
                             int32_t cache_capacity, int32_t pos_offset,
                             void *O, void *workspace, size_t workspace_bytes,
                             msa_stream stream);

/*
 * msa_sparse_attend_static -- the same attention as msa_sparse_attend, for
 * callers that cannot allocate device memory: for example a plugin inside a
 * host engine that reserved the whole device memory budget up front and
 * forbids any further allocation, or a C caller with no allocator of its own
 * to size a workspace.  The pages have no counterpart to this call; it is an
 * engineering entry point of this library.
 *
 * Arguments are those of msa_sparse_attend without `workspace` and
 * `workspace_bytes`; the caller still passes every input and output buffer.
 * The call allocates nothing.  Its scratch (the partial results of the split
 * attention context) lives in one fixed device array of 4 MiB (4194304 bytes)
 * inside the library; every GPU that loads the library holds that array until
 * the process exits.  A call whose scratch would exceed 4 MiB (the size
 * msa_attend_workspace_size reports for the same arguments, with
 * cache_capacity in place of max_local_position) is rejected with
 * MSA_ERR_UNSUPPORTED and enqueues nothing.
 *
 * The first call on a device looks up that device's address of the array
 * (cudaGetSymbolAddress, with the device current); make that first call before
 * any stream capture.  All calls share the one array and each call overwrites
 * it: calls that may run at the same time on the GPU (different streams, or
 * different host threads) race and must be ordered by the caller.  Nothing in
 * the array needs clearing: every scratch entry a call reads was written by
 * the same call.
 */
MSA_API msa_status msa_sparse_attend_static(
    const msa_memory *mem, const void *content, const int32_t *ids, int32_t batch,
    int32_t k, int32_t tokens, int32_t n_q_heads, const void *Q, const void *K_new,
    const void *V_new, void *K_cache, void *V_cache, int32_t *cache_len,
    int32_t cache_capacity, int32_t pos_offset, void *O, msa_stream stream);

/* Per-layer decode state, every buffer owned by the caller (see msa_step). */
typedef struct {
  int32_t batch;
  int32_t top_k;
  int32_t n_q_heads;
  int32_t cache_capacity;
  int32_t pos_offset;        /* Global RoPE offset, normally top_k */
  float *state;              /* device [batch][n_docs] running max */
  int32_t *ids;              /* device [batch][top_k] */
  float *scores;             /* device [batch][top_k] */
  void *k_cache;             /* device [batch][cache_capacity][H_kv][D] */
  void *v_cache;
  int32_t *cache_len;        /* device [batch] */
  void *workspace;
  size_t workspace_bytes;    /* >= msa_step_workspace_size(...) */
} msa_decode_state;

MSA_API size_t msa_step_workspace_size(const msa_memory *mem, int32_t batch, int32_t k,
                               int32_t n_q_heads);

/*
 * One routed decode step of one layer for every query of the batch
 * [b-lab.team stages "Online Routing & Context Assembly" and "Sparse
 * Generation", run per generated token]: route the new token with the running
 * state (so the result equals routing over every token so far), take the
 * top-k, then attend with the new token appended to the local cache.
 *   Qr_tok : device [batch][H_r][d_r];  Q_tok : [batch][n_q_heads][D]
 *   K_tok, V_tok : [batch][H_kv][D];     O_tok : [batch][n_q_heads][D]
 * Qr_tok is read early, as msa_route's Qr: it must not be an output of the
 * previous msa_* call on the same stream.
 */
MSA_API msa_status msa_step(const msa_memory *mem, const void *router_keys,
                    const void *content, const msa_decode_state *st,
                    const void *Qr_tok, const void *Q_tok, const void *K_tok,
                    const void *V_tok, void *O_tok, msa_stream stream);

/*
 * Memory Interleave [Evermind summary sec. 4C; b-lab.team item 3: generative
 * retrieval -> context expansion -> generation, repeated; the documents
 * retrieved in one round become part of the query of the next].  Runs
 * `rounds` routing rounds for every query of the batch:
 *   round 0 routes Qr [batch][tokens][H_r][d_r];
 *   round r > 0 routes the unit router rows (every chunk, every head) of the
 *   documents retrieved in round r-1;
 * each with the running state carried over, and each round's top-k taken
 * among the documents not yet in the context (taken[b][d] == 0).
 *   state  : device [batch][n_docs] fp32, reset to -inf here
 *   taken  : device [batch][n_docs] uint8, reset to 0 here; on return it marks
 *            every document retrieved in rounds 0..rounds-2
 *   ids, scores : device [rounds][batch][k]
 * The next round's row count is read back to the host once per round.  A
 * query with no new rows in a round (it retrieved nothing) keeps its state
 * through that round; when no query has new rows, the remaining rounds' ids /
 * scores are -1 / -inf.
 */
MSA_API size_t msa_interleave_workspace_size(const msa_memory *mem, int32_t batch,
                                             int32_t tokens, int32_t k);
MSA_API msa_status msa_interleave(const msa_memory *mem, const void *router_keys,
                                  const void *Qr, int32_t batch, int32_t tokens, int32_t k,
                                  int32_t rounds, float *state, uint8_t *taken, int32_t *ids,
                                  float *scores, void *workspace, size_t workspace_bytes,
                                  msa_stream stream);

/*
 * Adaptive Memory Interleave [same passages; the pages leave the number of
 * rounds to the model, which decides when the context holds enough -- here a
 * stopping score stands in for that decision]: msa_interleave with at most
 * `max_rounds` rounds, in which a query stops after the first round whose
 * best new document scores below stop_score.  That round's retrievals do not
 * enter its context: its ids / scores of that round and every later one are
 * -1 / -inf, and its state stays as it was after its last kept round.
 *   n_rounds : device [batch] int32 out, the rounds whose retrievals were kept
 *              (0 .. max_rounds)
 *   stop_score : any value but NaN (-inf: never stop = msa_interleave)
 * Workspace: msa_interleave_workspace_size.  Errors: INVALID_ARG for a null
 * n_rounds or a NaN stop_score, else as msa_interleave.
 */
MSA_API msa_status msa_interleave_adaptive(const msa_memory *mem, const void *router_keys,
                                           const void *Qr, int32_t batch, int32_t tokens,
                                           int32_t k, int32_t max_rounds, float stop_score,
                                           float *state, uint8_t *taken, int32_t *ids,
                                           float *scores, int32_t *n_rounds, void *workspace,
                                           size_t workspace_bytes, msa_stream stream);

/*
 * Host tier of the pooled content [Evermind summary sec. 4B "Memory Parallel &
 * Tiered Storage": routing keys stay in GPU memory, the content K/V stays in
 * host DRAM and only the selected documents are fetched, asynchronously;
 * b-lab.team item 2, KV cache compression].
 *
 * A fetcher manages a device slot cache for one layer's content:
 *   content_host : PINNED host memory [C][2][H_kv][D] written by
 *                  msa_encode_memory (it may write host memory directly); it
 *                  must be mapped into the device address space (pinned memory
 *                  is, on every 64-bit system with unified addressing)
 *   slot_cache   : device memory of n_slots * doc_content_stride bytes
 *                  (msa_memory_get_info), one document per slot
 *   n_slots      : >= max_batch * max_k, so one call's documents always fit;
 *                  max_batch * max_k <= 4096
 *   flags        : MSA_FETCH_COLD forgets every resident document at each
 *                  fetch (every selected document crosses the host link)
 * The fetcher's bookkeeping lives in device memory it allocates (the document
 * -> slot map and a claim word per document, the slot -> document map and use
 * stamps per slot, the slot of each (query, rank), the copy list, a small
 * scratch array), so no fetch
 * reads anything back to the host; it also creates two events.  It does not
 * own content_host or slot_cache.  msa_fetcher_destroy frees what it made.
 */
typedef struct msa_fetcher msa_fetcher;
#define MSA_FETCH_COLD 0x1u

MSA_API msa_status msa_fetcher_create(const msa_memory *mem, const void *content_host,
                                      void *slot_cache, int32_t n_slots, int32_t max_batch,
                                      int32_t max_k, uint32_t flags, msa_fetcher **out);
MSA_API msa_status msa_fetcher_destroy(msa_fetcher *f);
/* Totals since creation: (query, rank) hits, misses (documents copied),
 * documents copied, bytes copied over the host link.  Synchronises the device
 * to read them. */
MSA_API msa_status msa_fetcher_stats(const msa_fetcher *f, int64_t *hits, int64_t *misses,
                                     int64_t *copies, int64_t *bytes);

/*
 * Make the documents ids[batch][k] (device) resident in the slot cache, with
 * no host round trip: on `stream` (after the kernel that writes ids) one kernel
 * keeps the resident documents, gives every missing document a victim slot (a
 * clock over the slots not used by this call; a document wanted by several
 * (query, rank) entries is copied once, by the lowest entry) and writes the
 * slot of every (query, rank) and the list of copies; then, on `fetch_stream`,
 * one gather kernel copies every missing document's contiguous chunk rows from
 * content_host through its device mapping (one CTA per document) over the host
 * link.  `stream` then waits for `fetch_stream`.  fetch_stream may equal
 * stream.  Ids outside [0, n_docs) get slot 0 and are skipped by the attention
 * (device error word).  Calls of one fetcher must be ordered (they share its
 * bookkeeping); a whole step can be captured in a CUDA graph.
 */
MSA_API msa_status msa_fetch(msa_fetcher *f, const int32_t *ids, int32_t batch, int32_t k,
                             msa_stream stream, msa_stream fetch_stream);

/* msa_sparse_attend over the memory rows the last msa_fetch of `f` placed in
 * its slot cache (same ids, batch and k). */
MSA_API msa_status msa_sparse_attend_fetched(
    const msa_memory *mem, const msa_fetcher *f, const int32_t *ids, int32_t batch, int32_t k,
    int32_t tokens, int32_t n_q_heads, const void *Q, const void *K_new, const void *V_new,
    void *K_cache, void *V_cache, int32_t *cache_len, int32_t cache_capacity,
    int32_t pos_offset, void *O, void *workspace, size_t workspace_bytes, msa_stream stream);

/* msa_step with the content in the host tier: route, msa_fetch, then the
 * attention over the fetched rows.  Nothing is read back to the host. */
MSA_API msa_status msa_step_host(const msa_memory *mem, const void *router_keys, msa_fetcher *f,
                                 const msa_decode_state *st, const void *Qr_tok,
                                 const void *Q_tok, const void *K_tok, const void *V_tok,
                                 void *O_tok, msa_stream stream, msa_stream fetch_stream);

/*
 * Memory Parallel [Evermind summary sec. 4B "Memory Parallel & Tiered Storage":
 * the routing keys are split over GPUs, the query goes to every GPU, each scores
 * its own part and the results are reduced to one global top-k; b-lab.team item
 * 2, the inference engine serving 100M tokens on two GPUs].  The memory's
 * documents are cut into contiguous ranges ("shards"); each shard is an
 * msa_memory over its range (document 0 of shard s is global document
 * shard_doc_base[s]) and routes with msa_route as usual, keeping its top k_cand
 * as (score, shard-local id).  msa_topk_merge merges every shard's candidates
 * into the global top-k:
 *   cand_scores, cand_ids : device [n_shards][batch][k_cand], each shard's
 *                 msa_route output (ids < 0 are padding and are skipped)
 *   shard_doc_base : HOST array [n_shards], non-decreasing, >= 0
 *   ids, scores : device [batch][k] out, global document ids by (score
 *                 descending, global id ascending); padded with -1 / -inf when
 *                 fewer than k candidates are valid
 * With k_cand >= k the result is bit-identical to msa_route over the whole
 * memory: a document's score does not depend on the partition, and the merge
 * orders (score, global id) exactly as the single-memory top-k does.  The
 * candidates reach this GPU by any means -- an all-gather of batch * k_cand *
 * 8 bytes per shard over NCCL, or, for logical shards on one GPU, the shards'
 * own output buffers.  Errors: INVALID_ARG (bad counts, k > n_shards * k_cand,
 * bases out of order), UNSUPPORTED (more than 4096 candidates per query), CUDA.
 */
MSA_API msa_status msa_topk_merge(const float *cand_scores, const int32_t *cand_ids,
                                  int32_t n_shards, int32_t batch, int32_t k_cand,
                                  const int32_t *shard_doc_base, int32_t k, int32_t *ids,
                                  float *scores, msa_stream stream);

/*
 * Backward of the routing score [Evermind summary sec. 4A: continued
 * pre-training supervises the router with an auxiliary routing loss L_aux; the
 * training itself is outside this library].  For one routing call of `tokens`
 * query rows with no carried state, doc_score[b][d] = max over tokens t and
 * chunks c of document d of (1/H_r) sum_h cos(Qr[b,t,h], M[c,h]), M the pooled
 * (un-normalised) router keys.  Given d_score = dL/d doc_score, the gradient
 * of each document's max reaches its first maximising (token, chunk) pair, in
 * (token, chunk) order:
 *   d cos(q, m)/dq = m / (|q| |m|) - cos q / |q|^2   (and symmetrically for m;
 *   a norm clamped at 1e-12 contributes no term).
 *   router_mean   : device [C][H_r][d_r], msa_encode_memory's router_mean
 *   Qr            : device [batch][tokens][H_r][d_r]
 *   d_score       : device [batch][n_docs] fp32 (zeros skip their pairs)
 *   d_Qr          : device [batch][tokens][H_r][d_r] fp32, overwritten
 *   d_router_mean : device [C][H_r][d_r] fp32, overwritten
 * The pooling's own backward (each chunk token receives d_router_mean / chunk
 * length) is left to the caller.  CUDA-core kernel, one warp per (query,
 * document) with a nonzero gradient.
 */
MSA_API msa_status msa_route_backward(const msa_memory *mem, const void *router_mean,
                                      const void *Qr, int32_t batch, int32_t tokens,
                                      const float *d_score, float *d_Qr, float *d_router_mean,
                                      msa_stream stream);

/*
 * Backward of msa_sparse_attend [b-lab.team item 1 and stage "Sparse
 * Generation"; the same context, masking, Global RoPE and GQA mapping].  With
 * p = softmax(z) over the context rows of (b, i, h), z = <RoPE(Q), key> /
 * sqrt(D), O = sum p value, and dO given:
 *   dz = p (<dO, value> - <dO, O>);  dQ = RoPE^T(sum dz key) / sqrt(D);
 *   dkey += dz RoPE(Q) / sqrt(D);    dvalue += p dO.
 *   content, ids, Q, pos_offset, cache_capacity : as msa_sparse_attend
 *   K_cache, V_cache : device [batch][cache_capacity][H_kv][D] as the forward
 *                 left them (K rotated; the call's tokens appended)
 *   cache_len0  : device [batch] int32, the lengths BEFORE the forward call
 *   dO          : device [batch][tokens][n_q_heads][D]
 *   dQ          : device fp32 [batch][tokens][n_q_heads][D], overwritten,
 *                 with respect to Q before its RoPE
 *   d_cache_k, d_cache_v : device fp32 [batch][cache_capacity][H_kv][D],
 *                 overwritten, with respect to the cache rows as stored
 *   d_content   : device fp32 [C][2][H_kv][D], overwritten, with respect to
 *                 the pooled memory rows as stored
 * n_q_heads <= 32.  CUDA-core kernel, one warp per (query, token, head).
 */
MSA_API msa_status msa_sparse_attend_backward(const msa_memory *mem, const void *content,
                                              const int32_t *ids, int32_t batch, int32_t k,
                                              int32_t tokens, int32_t n_q_heads, const void *Q,
                                              const void *K_cache, const void *V_cache,
                                              const int32_t *cache_len0, int32_t cache_capacity,
                                              int32_t pos_offset, const void *dO, float *dQ,
                                              float *d_cache_k, float *d_cache_v,
                                              float *d_content, msa_stream stream);

/* Read and clear the device error word of the current device (synchronises/* Read and clear the device error word of the current device (synchronises/* Read and clear the device error word of the current device (synchronises
 * `stream`).  *bits receives the MSA_DEVERR_* bits; returns MSA_ERR_TIMEOUT or
 * MSA_ERR_STATE when a bit was set, else MSA_OK. */
MSA_API msa_status msa_device_error(uint32_t *bits, msa_stream stream);

MSA_API const char *msa_status_string(msa_status s);
MSA_API const char *msa_last_error(void);
/* Number of kernels this library has enqueued from this process so far, over
 * all threads and devices.  A launch made while a stream is being captured
 * into a CUDA graph counts once, at capture, not per replay.  No counterpart
 * in the method: it lets a caller count the kernels of a timed region. */
MSA_API uint64_t msa_launch_count(void);
/* Library version as major*10000 + minor*100 + patch. */
MSA_API int32_t msa_version(void);

#ifdef __cplusplus
}
#endif
#endif /* MSA_H_ */
