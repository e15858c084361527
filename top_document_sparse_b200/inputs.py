"""Seeded synthetic inputs for the MSA hot path.

This module only draws random numbers and places them; it computes nothing the method computes
(no pooling, no RoPE, no scoring, no top-k, no attention).  Both the CUDA path and the oracle
consume the tensors it returns, so they see the same bytes.

Recipe (shared by tests and the benchmark):

* Raw per-token K, V and router keys K_r are i.i.d. N(0, 1), rounded to the workload's dtype.
* Query router projections Q_r and local Q/K/V are i.i.d. N(0, 1).
* Planted relevance: for query b, planted document d and one of its full chunks j, a query token
  t is chosen and a target pooled router row m is built per router head h as
  ``m_h = rho * (c * u_h + sqrt(1 - c^2) * n_h)`` with ``u_h`` the unit direction of
  ``Q_r[b, t, h]`` and ``n_h`` a unit vector orthogonal to it, rho = sqrt(d_r / chunk_len) (the
  typical norm of a chunk mean of N(0,1) rows).  The chunk's raw rows are ``m + a_i`` where the
  noise rows come in antithetic pairs ``a_{2i} = g_i``, ``a_{2i+1} = -g_i`` (g_i ~ N(0,1)), so the
  chunk mean is m up to input rounding and the planted cosine is c.
* Memory Interleave chain: per query three documents h1, h2, h3; with w_0 the query token's
  direction and w_1..w_3 document-unique unit directions (each orthogonal to the ones before),
  hop i's planted chunk has pooled row rho * (0.6 w_{i-1} + 0.8 w_i).  Hop i+1 then scores 0.48
  against hop i's pooled row and ~0 against the query, so it only surfaces once hop i's rows
  are appended to the query.
"""
from __future__ import annotations

import math

import numpy as np
import torch

from .workloads import Workload

_TORCH_DTYPE = {"f32": torch.float32, "bf16": torch.bfloat16}


def torch_dtype(name: str) -> torch.dtype:
    return _TORCH_DTYPE[name]


def doc_offsets(w: Workload, seed: int = 0) -> np.ndarray:
    """Token offsets of the documents, int64 [n_docs + 1]."""
    if w.doc_len:
        return np.arange(w.n_docs + 1, dtype=np.int64) * w.doc_len
    median, sigma, lo, hi, total = w.lognormal
    rng = np.random.default_rng(np.random.SeedSequence([seed, 0x10C]))
    lens = []
    acc = 0
    while acc < total:
        n = int(np.clip(round(median * math.exp(sigma * rng.standard_normal())), lo, hi))
        n = min(n, total - acc) if total - acc >= lo else n
        lens.append(n)
        acc += n
    off = np.zeros(len(lens) + 1, dtype=np.int64)
    off[1:] = np.cumsum(lens)
    return off


def generator(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed) & 0x7FFFFFFFFFFFFFFF)
    return g


def gaussian(shape, gen: torch.Generator, device, dtype: torch.dtype) -> torch.Tensor:
    """N(0, 1) drawn in fp32 and rounded (round-to-nearest-even) to ``dtype``."""
    return torch.randn(*shape, generator=gen, device=device, dtype=torch.float32).to(dtype)


def raw_memory(w: Workload, n_tok: int, seed: int, device="cpu"):
    """Raw token-major K [n_tok][H_kv][D], V (same), K_r [n_tok][H_r][d_r]."""
    g = generator(seed, device)
    dt = torch_dtype(w.dtype)
    K = gaussian((n_tok, w.n_kv_heads, w.head_dim), g, device, dt)
    V = gaussian((n_tok, w.n_kv_heads, w.head_dim), g, device, dt)
    Kr = gaussian((n_tok, w.n_router_heads, w.router_dim), g, device, dt)
    return K, V, Kr


def queries(w: Workload, batch: int, tokens: int, seed: int, device="cpu"):
    """Local query block: Q_r [B][T][H_r][d_r], Q [B][T][H_q][D], K_new, V_new [B][T][H_kv][D]."""
    g = generator(seed, device)
    dt = torch_dtype(w.dtype)
    Qr = gaussian((batch, tokens, w.n_router_heads, w.router_dim), g, device, dt)
    Q = gaussian((batch, tokens, w.n_q_heads, w.head_dim), g, device, dt)
    Kn = gaussian((batch, tokens, w.n_kv_heads, w.head_dim), g, device, dt)
    Vn = gaussian((batch, tokens, w.n_kv_heads, w.head_dim), g, device, dt)
    return Qr, Q, Kn, Vn


def choose_plants(w: Workload, doc_tok_off: np.ndarray, batch: int, tokens: int, per_query: int,
                  seed: int):
    """Planted (query, doc, full chunk, query token) tuples; documents are distinct across the
    whole batch when the memory has enough of them.  Returns int64 arrays b, doc, chunk, tok."""
    rng = np.random.default_rng(np.random.SeedSequence([seed, 0x9A7]))
    n_docs = doc_tok_off.size - 1
    full = (doc_tok_off[1:] - doc_tok_off[:-1]) // w.chunk_len
    cand = np.nonzero(full >= 1)[0]
    need = batch * per_query
    replace = need > cand.size
    docs = rng.choice(cand, size=need, replace=replace)
    b = np.repeat(np.arange(batch, dtype=np.int64), per_query)
    if replace:  # keep documents distinct within one query
        for q in range(batch):
            docs[q * per_query:(q + 1) * per_query] = rng.choice(cand, size=per_query,
                                                                 replace=False)
    chunk = np.array([rng.integers(0, full[d]) for d in docs], dtype=np.int64)
    tok = rng.integers(0, tokens, size=need).astype(np.int64)
    assert n_docs > 0
    return b, docs.astype(np.int64), chunk, tok


def _unit(x: torch.Tensor) -> torch.Tensor:
    return x / x.norm(dim=-1, keepdim=True)


def _orthogonal_unit(x: torch.Tensor, against: list) -> torch.Tensor:
    for a in against:
        x = x - (x * a).sum(-1, keepdim=True) * a
    return _unit(x)


def write_chunk_rows(Kr: torch.Tensor, doc_tok_off: np.ndarray, chunk_len: int,
                     docs: np.ndarray, chunks: np.ndarray, target: torch.Tensor, seed: int):
    """Overwrite full chunk (doc, j) of the raw router keys with rows m + a_i, antithetic noise,
    so that the chunk mean is ``target`` [P][H_r][d_r] (up to rounding to Kr's dtype)."""
    assert chunk_len % 2 == 0
    dev = Kr.device
    P = len(docs)
    g = generator(seed ^ 0x5EED, dev)
    half = torch.randn(P, chunk_len // 2, Kr.shape[1], Kr.shape[2], generator=g, device=dev,
                       dtype=torch.float64)
    noise = torch.stack([half, -half], dim=2).reshape(P, chunk_len, Kr.shape[1], Kr.shape[2])
    rows = target.to(dev, torch.float64)[:, None] + noise
    start = torch.as_tensor(doc_tok_off[docs] + chunks * chunk_len, device=dev)
    idx = start[:, None] + torch.arange(chunk_len, device=dev)[None]
    Kr[idx.reshape(-1)] = rows.reshape(-1, Kr.shape[1], Kr.shape[2]).to(Kr.dtype)


def plant(w: Workload, Kr: torch.Tensor, Qr: torch.Tensor, doc_tok_off: np.ndarray, plants,
          cos: float, seed: int, tok_base: int = 0):
    """Plant the (b, doc, chunk, tok) tuples: the pooled router row of each planted chunk has
    cosine ``cos`` with every router head of Q_r[b, tok].  ``Kr`` holds the raw router keys of the
    tokens starting at global token ``tok_base``."""
    b, docs, chunks, tok = plants
    if len(docs) == 0:
        return
    dev = Kr.device
    q = Qr[torch.as_tensor(b, device=Qr.device), torch.as_tensor(tok, device=Qr.device)]
    u = _unit(q.to(dev, torch.float64))                                  # [P][H_r][d_r]
    g = generator(seed ^ 0x0DD, dev)
    n = torch.randn(u.shape, generator=g, device=dev, dtype=torch.float64)
    n = _orthogonal_unit(n, [u])
    rho = math.sqrt(w.router_dim / w.chunk_len)
    target = rho * (cos * u + math.sqrt(1.0 - cos * cos) * n)
    write_chunk_rows(Kr, doc_tok_off - tok_base, w.chunk_len, docs, chunks, target, seed)


def plant_chain(w: Workload, Kr: torch.Tensor, Qr: torch.Tensor, doc_tok_off: np.ndarray,
                hops: int, seed: int, a: float = 0.6, b: float = 0.8):
    """Plant a ``hops``-long chain per query (Memory Interleave workload).  Returns the chain
    documents, int64 [B][hops]."""
    B, T = Qr.shape[0], Qr.shape[1]
    rng = np.random.default_rng(np.random.SeedSequence([seed, 0xC4A]))
    full = (doc_tok_off[1:] - doc_tok_off[:-1]) // w.chunk_len
    cand = np.nonzero(full >= 1)[0]
    docs = rng.choice(cand, size=B * hops, replace=False).reshape(B, hops)
    chunks = np.array([[rng.integers(0, full[d]) for d in row] for row in docs], dtype=np.int64)
    tok = rng.integers(0, T, size=B)
    dev = Kr.device
    g = generator(seed ^ 0xC4A1, dev)
    w_prev = [_unit(Qr[torch.arange(B), torch.as_tensor(tok)].to(dev, torch.float64))]
    targets = []
    rho = math.sqrt(w.router_dim / w.chunk_len)
    for _ in range(hops):
        wi = torch.randn(w_prev[0].shape, generator=g, device=dev, dtype=torch.float64)
        wi = _orthogonal_unit(wi, w_prev)
        targets.append(rho * (a * w_prev[-1] + b * wi))
        w_prev.append(wi)
    target = torch.stack(targets, dim=1).reshape(B * hops, *w_prev[0].shape[1:])
    write_chunk_rows(Kr, doc_tok_off, w.chunk_len, docs.reshape(-1), chunks.reshape(-1), target,
                     seed)
    return docs
