"""Memory Parallel: the memory's documents split over GPUs ("shards"), each routing its own part.

The pages' inference engine serves a 100M-token memory on two GPUs this way (Evermind summary
sec. 4B "Memory Parallel & Tiered Storage"; b-lab.team item 2): the routing keys are split over
the GPUs, the query goes to every GPU, each scores its own documents, and the per-GPU results
are reduced to one global top-k.  The pooled content stays in the host tier and is fetched by
whichever GPU generates.  Here:

* ``shard_ranges`` cuts the documents into contiguous ranges of about equal token counts;
* ``MemoryShard`` is one shard: an ``msa.Memory`` over its range, whose document 0 is global
  document ``doc_base``; its ``route`` keeps the shard's top k as (score, shard-local id);
* ``gather_candidates`` is the one exchange, an all-gather of every shard's (score, id)
  candidates -- batch x k x 8 bytes per shard -- over a ``torch.distributed`` process group
  (NCCL between GPUs);
* ``msa.topk_merge`` merges them on the device into the global top-k, bit-identical to routing
  the whole memory at once.

Host logic only (argument marshalling and the collective); every score and every merge runs in
the library's CUDA kernels.
"""
from __future__ import annotations

import numpy as np
import torch


def shard_ranges(doc_token_offsets, n_shards: int) -> np.ndarray:
    """Document boundaries [n_shards + 1] of n_shards contiguous ranges with about equal token
    counts; every range holds at least one document."""
    off = np.asarray(doc_token_offsets, dtype=np.int64)
    n_docs = off.size - 1
    if not 1 <= n_shards <= n_docs:
        raise ValueError(f"n_shards={n_shards} must be in [1, n_docs={n_docs}]")
    targets = off[-1] * np.arange(1, n_shards, dtype=np.float64) / n_shards
    cuts = np.searchsorted(off, targets, side="left")
    bounds = np.concatenate([[0], cuts, [n_docs]]).astype(np.int64)
    for s in range(1, n_shards + 1):  # at least one document per shard, in order
        bounds[s] = max(bounds[s], bounds[s - 1] + 1)
    for s in range(n_shards - 1, -1, -1):
        bounds[s] = min(bounds[s], bounds[s + 1] - 1)
    return bounds


def shard_token_offsets(doc_token_offsets, d0: int, d1: int) -> np.ndarray:
    """Token offsets of documents [d0, d1), rebased to start at 0."""
    off = np.asarray(doc_token_offsets, dtype=np.int64)
    return off[d0:d1 + 1] - off[d0]


class MemoryShard:
    """One shard of a memory: documents [d0, d1) of the whole memory as their own msa.Memory."""

    def __init__(self, doc_token_offsets, bounds, shard: int, chunk_len: int, n_kv_heads: int,
                 head_dim: int, n_router_heads: int, router_dim: int, dtype: torch.dtype,
                 rope_theta: float, max_local_position: int):
        from . import msa
        self.shard = shard
        self.d0, self.d1 = int(bounds[shard]), int(bounds[shard + 1])
        self.doc_base = self.d0
        off = np.asarray(doc_token_offsets, dtype=np.int64)
        self.tok0, self.tok1 = int(off[self.d0]), int(off[self.d1])
        self.mem = msa.Memory(shard_token_offsets(off, self.d0, self.d1), chunk_len, n_kv_heads,
                              head_dim, n_router_heads, router_dim, dtype, rope_theta,
                              max_local_position)

    def encode(self, K, V, Kr, router_keys, content, stream=None):
        """Encode the shard's documents from the whole memory's token-major K, V, Kr."""
        t0, t1 = self.tok0, self.tok1
        self.mem.encode(0, self.mem.n_docs, K[t0:t1], V[t0:t1], Kr[t0:t1], router_keys, content,
                        stream=stream)

    def route(self, router_keys, Qr, k: int, state, ids, scores, workspace, stream=None):
        """This shard's top-k candidates for the query rows Qr [B][T][H_r][d_r] into ids /
        scores [B][k] (shard-local ids), with the shard's running state [B][shard documents]
        carried over (msa_route)."""
        if k > self.mem.n_docs:
            raise ValueError(f"k={k} exceeds the {self.mem.n_docs} documents of shard {self.shard}")
        self.mem.route(router_keys, Qr, k, state, ids, scores, workspace, stream=stream)


def gather_candidates(scores, ids, group=None):
    """All-gather every shard's candidates (rank r holds shard r): returns (scores, ids) of
    shape [world][B][k], ordered by rank.  Works for CPU tensors over gloo and device tensors
    over NCCL."""
    import torch.distributed as dist
    world = dist.get_world_size(group)
    sc = [torch.empty_like(scores) for _ in range(world)]
    ii = [torch.empty_like(ids) for _ in range(world)]
    dist.all_gather(sc, scores.contiguous(), group=group)
    dist.all_gather(ii, ids.contiguous(), group=group)
    return torch.stack(sc), torch.stack(ii)
