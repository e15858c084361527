"""Shared test helpers: seeded memories, tolerance scales, comparisons."""
from __future__ import annotations

import math

import numpy as np
import torch

from top_document_sparse_b200 import inputs
from top_document_sparse_b200.workloads import Workload


def small_workload(**kw) -> Workload:
    base = dict(name="t", description="", dtype="bf16", n_docs=8, doc_len=256, chunk_len=64,
                n_q_heads=8, n_kv_heads=2, head_dim=128, n_router_heads=8, router_dim=128,
                top_k=4, batch=2, query_tokens=16, decode_steps=0, n_layers=1,
                planted_per_query=2, planted_cos=0.6)
    base.update(kw)
    return Workload(**base)


def memory_inputs(w: Workload, seed: int, device="cpu", plant_batch=None, plant_tokens=None,
                  lognormal_seed=None):
    """Raw K, V, Kr (with planted chunks against the returned query Q_r) and doc offsets."""
    off = inputs.doc_offsets(w, seed if lognormal_seed is None else lognormal_seed)
    n_tok = int(off[-1])
    K, V, Kr = inputs.raw_memory(w, n_tok, seed, device)
    B = w.batch if plant_batch is None else plant_batch
    T = w.query_tokens if plant_tokens is None else plant_tokens
    Qr, Q, Kn, Vn = inputs.queries(w, B, T, seed + 1, device)
    plants = inputs.choose_plants(w, off, B, T, w.planted_per_query, seed + 2)
    inputs.plant(w, Kr, Qr, off, plants, w.planted_cos, seed + 3)
    return dict(off=off, K=K, V=V, Kr=Kr, Qr=Qr, Q=Q, Kn=Kn, Vn=Vn, plants=plants)


def bf16_ulp(x: np.ndarray) -> np.ndarray:
    """Spacing of bf16 numbers at |x| (8 significant bits)."""
    a = np.maximum(np.abs(x), np.finfo(np.float32).tiny)
    return np.exp2(np.floor(np.log2(a)) - 7)


def chunk_abs_mean(x: np.ndarray, doc_tok_off, chunk_len: int) -> np.ndarray:
    """Per chunk and element, the mean of |x| over the chunk's tokens: the scale of the
    summation error bound of a chunk mean.  x: [n_tok][...]."""
    rows = []
    for d in range(len(doc_tok_off) - 1):
        for t0 in range(int(doc_tok_off[d]), int(doc_tok_off[d + 1]), chunk_len):
            t1 = min(t0 + chunk_len, int(doc_tok_off[d + 1]))
            rows.append(np.abs(x[t0:t1]).mean(axis=0))
    return np.stack(rows)


def rope_scale(K: np.ndarray, doc_tok_off, chunk_len: int) -> np.ndarray:
    """Error scale of a pooled rotated key: mean over the chunk of |k_i| + |k_{i+-D/2}|."""
    D = K.shape[-1]
    a = np.abs(K)
    pair = np.concatenate([a[..., D // 2:], a[..., :D // 2]], axis=-1)
    return chunk_abs_mean(a + pair, doc_tok_off, chunk_len)


def to64(t) -> np.ndarray:
    if isinstance(t, torch.Tensor):
        return t.detach().to("cpu", torch.float64).numpy()
    return np.asarray(t, dtype=np.float64)


def assert_close(got, want, tol, what):
    got, want = to64(got), to64(want)
    err = np.abs(got - want)
    bad = err > tol
    if np.any(bad):
        i = np.unravel_index(np.argmax(err - tol), err.shape)
        raise AssertionError(f"{what}: {bad.sum()} of {bad.size} elements out of tolerance; "
                             f"worst at {i}: got {got[i]!r} want {want[i]!r} "
                             f"err {err[i]:.3e} tol {np.broadcast_to(tol, err.shape)[i]:.3e}")
    return float(err.max()) if err.size else 0.0
