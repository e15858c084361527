"""Named synthetic workloads for the MSA hot path.

Each workload fixes the memory shape (documents, chunk length, head shapes), the query batch,
the decode schedule and the planted-relevance recipe.  The shapes follow the MSA papers'
setting: a Qwen3-4B-shaped attention layer (32 query heads, 8 KV heads, head_dim 128), 8 router
heads of width 128, 64-token chunks, memories of 16K, 1M and 100M tokens.  Values the pages do
not state (batch of the tiny check, lognormal sigma, the planted cosine of the 16K workload,
RoPE base) are marked "proposed" and recorded in the design notes.
"""
from __future__ import annotations

from dataclasses import dataclass, field


@dataclass(frozen=True)
class Workload:
    name: str
    description: str
    dtype: str                 # "f32" or "bf16": storage and input type of the path
    n_docs: int
    doc_len: int               # fixed length; 0 when lengths are lognormal
    chunk_len: int
    n_q_heads: int
    n_kv_heads: int
    head_dim: int
    n_router_heads: int
    router_dim: int
    top_k: int
    batch: int                 # independent queries
    query_tokens: int          # local query length (prefill)
    decode_steps: int
    n_layers: int              # routed layers, each with its own memory
    planted_per_query: int
    planted_cos: float
    rope_theta: float = 1.0e6  # proposed (Qwen3 family default); not stated by the pages
    content_on_host: bool = False
    lognormal: tuple = field(default=())   # (median, sigma, lo, hi, total_tokens) for ragged docs
    rounds: int = 0            # Memory Interleave rounds (0 = plain routing)

    @property
    def chunks_per_doc(self) -> int:
        return -(-self.doc_len // self.chunk_len) if self.doc_len else 0

    @property
    def n_tokens(self) -> int:
        return self.n_docs * self.doc_len if self.doc_len else self.lognormal[4]


WORKLOADS = {
    "tiny_f32": Workload(
        name="tiny_f32",
        description="tiny fp32 check: 64 docs x 512 tokens, chunk 64; router 8x128; "
                    "attention 8 Q / 2 KV heads, head_dim 64; 32-token queries; top-4",
        dtype="f32", n_docs=64, doc_len=512, chunk_len=64, n_q_heads=8, n_kv_heads=2,
        head_dim=64, n_router_heads=8, router_dim=128, top_k=4, batch=4, query_tokens=32,
        decode_steps=0, n_layers=1, planted_per_query=4, planted_cos=0.6),
    "mem16k_bf16": Workload(
        name="mem16k_bf16",
        description="16K-token memory, one Qwen3-4B-shaped layer: 32 docs x 512 tokens, "
                    "k=16, 128-token query then 64 decode steps at batch 1",
        dtype="bf16", n_docs=32, doc_len=512, chunk_len=64, n_q_heads=32, n_kv_heads=8,
        head_dim=128, n_router_heads=8, router_dim=128, top_k=16, batch=1, query_tokens=128,
        decode_steps=64, n_layers=1, planted_per_query=8, planted_cos=0.6),
    "mem1m_bf16": Workload(
        name="mem1m_bf16",
        description="1M-token memory: 2,048 docs x 512 tokens (16,384 chunks), 16 routed "
                    "layers resident in HBM, 64 queries x 256 tokens, 128 decode steps, k=16",
        dtype="bf16", n_docs=2048, doc_len=512, chunk_len=64, n_q_heads=32, n_kv_heads=8,
        head_dim=128, n_router_heads=8, router_dim=128, top_k=16, batch=64, query_tokens=256,
        decode_steps=128, n_layers=16, planted_per_query=16, planted_cos=0.5),
    "mem100m_bf16": Workload(
        name="mem100m_bf16",
        description="100M-token memory: 195,313 docs x 512 tokens (1,562,504 chunks); router keys "
                    "in HBM, pooled content in pinned host DRAM; 4 routed layers, 16 queries x "
                    "256 tokens, 64 decode steps, k=16",
        dtype="bf16", n_docs=195_313, doc_len=512, chunk_len=64, n_q_heads=32, n_kv_heads=8,
        head_dim=128, n_router_heads=8, router_dim=128, top_k=16, batch=16, query_tokens=256,
        decode_steps=64, n_layers=4, planted_per_query=16, planted_cos=0.5,
        content_on_host=True),
    "interleave_bf16": Workload(
        name="interleave_bf16",
        description="Memory Interleave: 1M-token memory of lognormal-length docs (median 512, "
                    "sigma 1.0, clipped to 64..8192, ragged last chunks), chunk 64, k=8, "
                    "256 queries x 256 tokens, 3 rounds over a planted 3-hop chain",
        dtype="bf16", n_docs=0, doc_len=0, chunk_len=64, n_q_heads=32, n_kv_heads=8,
        head_dim=128, n_router_heads=8, router_dim=128, top_k=8, batch=256, query_tokens=256,
        decode_steps=0, n_layers=1, planted_per_query=3, planted_cos=0.6,
        lognormal=(512, 1.0, 64, 8192, 1 << 20), rounds=3),
}
