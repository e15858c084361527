"""fp64 CPU oracle for the Memory Sparse Attention hot path.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` import this package.  It shares no code with
the CUDA library in ``top_document_sparse_b200``: the arithmetic lives in
``msa_oracle.c`` (plain double-precision loops), and this module only converts
arrays and composes those functions in the order the pages give.

Sources are cited by page title and section:

* "Evermind & Shanda Group -- MSA: Memory Sparse Attention for Efficient
  End-to-End Memory Model Scaling" (medium summary), sec. 2 (architecture),
  sec. 4B (tiered storage), sec. 4C (Memory Interleave).
* "MSA: Memory Sparse Attention" (b-lab.team summary), item 1 (the MSA layer:
  scalable sparse attention, document-wise RoPE, global RoPE), item 3 (Memory
  Interleave) and the three-stage inference pipeline.

Parity status of each function is recorded in the header of ``msa_oracle.c``
and in the design notes; the functions below whose reading the pages do not
fix (chunk-to-document max, RoPE base and style, no RoPE on router vectors,
the global-RoPE offset, cumulative routing during decode, the interleave
append rule) are "parity unpinned" beyond the wording of the problem statement.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "msa_oracle.c")
_LIB = os.path.join(_HERE, "libmsa_oracle.so")

_dp = ctypes.POINTER(ctypes.c_double)
_i64p = ctypes.POINTER(ctypes.c_int64)
_i32p = ctypes.POINTER(ctypes.c_int32)


def build(force: bool = False) -> str:
    """Compile msa_oracle.c into libmsa_oracle.so (gcc, -O2, OpenMP, no FMA contraction)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call([
            "gcc", "-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math", "-fopenmp",
            "-shared", "-fPIC", _SRC, "-o", tmp, "-lm",
        ])
        os.replace(tmp, _LIB)
    return _LIB


_lib = None


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        lib.msa_oracle_doc_chunks.restype = ctypes.c_int64
        lib.msa_oracle_doc_chunks.argtypes = [_i64p, ctypes.c_int32, ctypes.c_int32, _i64p]
        lib.msa_oracle_rope_rows.restype = None
        lib.msa_oracle_rope_rows.argtypes = [_dp, ctypes.c_int64, ctypes.c_int32, ctypes.c_int32,
                                             _i64p, ctypes.c_double]
        lib.msa_oracle_encode.restype = None
        lib.msa_oracle_encode.argtypes = [_dp, _dp, _dp, _i64p, ctypes.c_int32, ctypes.c_int32,
                                          ctypes.c_int32, ctypes.c_int32, ctypes.c_int32,
                                          ctypes.c_int32, ctypes.c_double, _dp, _dp, _dp]
        lib.msa_oracle_chunk_score.restype = ctypes.c_double
        lib.msa_oracle_chunk_score.argtypes = [_dp, _dp, ctypes.c_int32, ctypes.c_int32]
        lib.msa_oracle_route.restype = None
        lib.msa_oracle_route.argtypes = [_dp, ctypes.c_int32, ctypes.c_int32, _dp, _i64p,
                                         ctypes.c_int32, ctypes.c_int32, ctypes.c_int32, _dp]
        lib.msa_oracle_topk.restype = None
        lib.msa_oracle_topk.argtypes = [_dp, ctypes.c_int32, ctypes.c_int32, ctypes.c_int32,
                                        _i32p, _dp]
        lib.msa_oracle_attend.restype = None
        lib.msa_oracle_attend.argtypes = [_dp, ctypes.c_int32, ctypes.c_int32, ctypes.c_int32,
                                          _dp, _dp, ctypes.c_int32, ctypes.c_int32, _dp, _dp,
                                          _i64p, _i32p, ctypes.c_int32, ctypes.c_int32,
                                          ctypes.c_int32, ctypes.c_int32, ctypes.c_double,
                                          _dp, _dp, _dp]
        lib.msa_oracle_route_backward.restype = None
        lib.msa_oracle_route_backward.argtypes = [_dp, ctypes.c_int32, ctypes.c_int32, _dp, _i64p,
                                                  ctypes.c_int32, ctypes.c_int32, ctypes.c_int32,
                                                  _dp, _dp, _dp]
        lib.msa_oracle_attend_backward.restype = None
        lib.msa_oracle_attend_backward.argtypes = [_dp, ctypes.c_int32, ctypes.c_int32,
                                                   ctypes.c_int32, _dp, _dp, ctypes.c_int32,
                                                   ctypes.c_int32, _dp, _dp, _i64p, _i32p,
                                                   ctypes.c_int32, ctypes.c_int32, ctypes.c_int32,
                                                   ctypes.c_int32, ctypes.c_double, _dp,
                                                   ctypes.c_int64, _dp, _dp, _dp, _dp, _dp]
        _lib = lib
    return _lib


def f64(x) -> np.ndarray:
    """Exact upcast of an fp32 / bf16 / fp64 array (numpy or torch, any device) to fp64."""
    try:
        import torch
        if isinstance(x, torch.Tensor):
            return np.ascontiguousarray(x.detach().to("cpu", torch.float64).numpy())
    except ImportError:  # pragma: no cover
        pass
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def _i64(x) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(x, dtype=np.int64))


def _i32(x) -> np.ndarray:
    try:
        import torch
        if isinstance(x, torch.Tensor):
            x = x.detach().cpu().numpy()
    except ImportError:  # pragma: no cover
        pass
    return np.ascontiguousarray(np.asarray(x, dtype=np.int32))


def _p(a: np.ndarray, t):
    return a.ctypes.data_as(t)


def doc_chunks(doc_tok_off, chunk_len: int) -> np.ndarray:
    """Fixed-length chunking: first chunk index of every document, [n_docs + 1]."""
    off = _i64(doc_tok_off)
    n_docs = off.size - 1
    out = np.zeros(n_docs + 1, dtype=np.int64)
    n = _load().msa_oracle_doc_chunks(_p(off, _i64p), n_docs, chunk_len, _p(out, _i64p))
    if n < 0:
        raise ValueError("empty document")
    return out


def rope_rows(x, pos, theta: float) -> np.ndarray:
    """RoPE (NeoX rotate-half) of rows x[n][H][dim] at positions pos[n]; returns a new array."""
    y = f64(x).copy()
    n, h, dim = y.shape
    p = _i64(pos)
    _load().msa_oracle_rope_rows(_p(y, _dp), n, h, dim, _p(p, _i64p), theta)
    return y


def encode(K, V, Kr, doc_tok_off, chunk_len: int, theta: float):
    """Offline encoding: chunk-mean pooled (Kbar, Vbar, Krbar) with document-wise RoPE on K."""
    K, V, Kr = f64(K), f64(V), f64(Kr)
    off = _i64(doc_tok_off)
    n_docs = off.size - 1
    n_tok, H_kv, D = K.shape
    _, H_r, d_r = Kr.shape
    C = int(doc_chunks(off, chunk_len)[-1])
    Kbar = np.zeros((C, H_kv, D))
    Vbar = np.zeros((C, H_kv, D))
    Krbar = np.zeros((C, H_r, d_r))
    _load().msa_oracle_encode(_p(K, _dp), _p(V, _dp), _p(Kr, _dp), _p(off, _i64p), n_docs,
                              chunk_len, H_kv, D, H_r, d_r, theta, _p(Kbar, _dp),
                              _p(Vbar, _dp), _p(Krbar, _dp))
    return Kbar, Vbar, Krbar


def chunk_score(qr_tok, krbar_chunk) -> float:
    """Mean over router heads of the cosine between one query token and one pooled chunk."""
    q, k = f64(qr_tok), f64(krbar_chunk)
    H_r, d_r = q.shape
    return _load().msa_oracle_chunk_score(_p(q, _dp), _p(k, _dp), H_r, d_r)


def route(Qr, Krbar, doc_chunk_off, state=None) -> np.ndarray:
    """Document relevance: max over query tokens and the document's chunks of chunk_score,
    max-merged into ``state`` ([B][n_docs], -inf when None)."""
    Q = f64(Qr)
    if Q.ndim == 3:
        Q = Q[:, None]
    B, T, H_r, d_r = Q.shape
    K = f64(Krbar)
    off = _i64(doc_chunk_off)
    n_docs = off.size - 1
    out = np.full((B, n_docs), -np.inf) if state is None else f64(state).copy()
    _load().msa_oracle_route(_p(Q, _dp), B, T, _p(K, _dp), _p(off, _i64p), n_docs, H_r, d_r,
                             _p(out, _dp))
    return out


def topk(score, k: int):
    """Top-k documents by (score descending, id ascending): (ids [B][k] int32, scores [B][k])."""
    s = f64(score)
    B, n_docs = s.shape
    if not 1 <= k <= n_docs:
        raise ValueError("k out of range")
    ids = np.zeros((B, k), dtype=np.int32)
    top = np.zeros((B, k))
    _load().msa_oracle_topk(_p(s, _dp), B, n_docs, k, _p(ids, _i32p), _p(top, _dp))
    return ids, top


def attend(Q, K_loc, V_loc, q_start: int, Kbar, Vbar, doc_chunk_off, ids, pos_offset: int,
           theta: float):
    """Sparse GQA attention of the new tokens over [retrieved memory rows | causal local rows].

    Returns (O [B][T][H_q][D], lse [B][T][H_q], rowsum [B][T][H_q])."""
    Q, Kl, Vl = f64(Q), f64(K_loc), f64(V_loc)
    B, T, H_q, D = Q.shape
    _, L_loc, H_kv, _ = Kl.shape
    if q_start + T > L_loc:
        raise ValueError("local history shorter than q_start + T")
    Kb, Vb = f64(Kbar), f64(Vbar)
    off = _i64(doc_chunk_off)
    idx = _i32(ids)
    k = idx.shape[1]
    O = np.zeros((B, T, H_q, D))
    lse = np.zeros((B, T, H_q))
    rs = np.zeros((B, T, H_q))
    _load().msa_oracle_attend(_p(Q, _dp), B, T, H_q, _p(Kl, _dp), _p(Vl, _dp), L_loc, q_start,
                              _p(Kb, _dp), _p(Vb, _dp), _p(off, _i64p), _p(idx, _i32p), k, H_kv,
                              D, pos_offset, theta, _p(O, _dp), _p(lse, _dp), _p(rs, _dp))
    return O, lse, rs


def decode_step(state, Qr_tok, Q_tok, K_hist, V_hist, q_index: int, Krbar, Kbar, Vbar,
                doc_chunk_off, k: int, pos_offset: int, theta: float):
    """One routed decode step for every query: route the new token with the running state
    (the max over all tokens so far), take the top-k, then attend with the new token at local
    index ``q_index`` (K_hist / V_hist hold the local history including the new token).

    Returns (new_state, ids, top_scores, O [B][H_q][D])."""
    st = route(np.asarray(f64(Qr_tok))[:, None], Krbar, doc_chunk_off, state)
    ids, top = topk(st, k)
    O, _, _ = attend(f64(Q_tok)[:, None], K_hist, V_hist, q_index, Kbar, Vbar, doc_chunk_off,
                     ids, pos_offset, theta)
    return st, ids, top, O[:, 0]


def interleave(Qr, Krbar, doc_chunk_off, k: int, rounds: int, stop_score=None):
    """Memory Interleave (retrieval -> context expansion, repeated): each round routes the new
    query rows with the state carried over, takes the top-k among the documents not yet in the
    context, adds them to the context, and appends their pooled router rows (every chunk, every
    head) as the next round's query rows.

    stop_score (adaptive interleave; the pages leave the round count to the model, a score
    threshold stands in for its decision): a query whose best new document in a round scores
    below it stops there -- that round's documents do not enter its context, its ids / scores
    from that round on are -1 / -inf, and it routes nothing more.

    Qr: [B][T][H_r][d_r].  Returns the list of (ids [B][k], top_scores [B][k]) per round; with
    stop_score also the final state [B][n_docs] and n_rounds [B] (rounds kept per query)."""
    off = _i64(doc_chunk_off)
    K = f64(Krbar)
    Q = f64(Qr)
    B = Q.shape[0]
    n_docs = off.size - 1
    state = np.full((B, n_docs), -np.inf)
    taken = np.zeros((B, n_docs), dtype=bool)
    active = np.ones(B, dtype=bool)
    n_rounds = np.zeros(B, dtype=np.int64)
    new_rows = [Q[b] for b in range(B)]
    out = []
    for _ in range(rounds):
        for b in range(B):
            if active[b] and new_rows[b].shape[0] > 0:
                state[b:b + 1] = route(new_rows[b][None], K, off, state[b:b + 1])
        eligible = np.where(taken, -np.inf, state)
        ids, top = topk(eligible, k)
        # a document already in the context cannot be retrieved again: with fewer than k
        # eligible documents the round's list is padded with -1 / -inf
        excluded = np.take_along_axis(taken, ids.astype(np.int64), axis=1)
        ids[excluded] = -1
        top[excluded] = -np.inf
        if stop_score is not None:
            active &= top[:, 0] >= stop_score
            ids[~active] = -1
            top[~active] = -np.inf
            n_rounds += active
        out.append((ids, top))
        for b in range(B):
            taken[b, ids[b][ids[b] >= 0]] = True
        new_rows = [np.concatenate([K[off[d]:off[d + 1]] for d in ids[b] if d >= 0] or
                                   [np.zeros((0,) + K.shape[1:])], axis=0)
                    for b in range(B)]
    if stop_score is not None:
        return out, state, n_rounds
    return out


def route_backward(Qr, Krbar, doc_chunk_off, G):
    """Gradients of sum_{b,d} G[b,d] * doc_score[b,d] (one routing call, no carried state) with
    respect to the query router rows and the pooled router keys: (dQr [B][T][H_r][d_r],
    dKrbar [C][H_r][d_r]).  The gradient of a max reaches its maximising (token, chunk) pair,
    the first in (token, chunk) order among equal maxima."""
    Q = f64(Qr)
    if Q.ndim == 3:
        Q = Q[:, None]
    B, T, H_r, d_r = Q.shape
    K = f64(Krbar)
    off = _i64(doc_chunk_off)
    g = f64(G)
    dQ = np.zeros_like(Q)
    dK = np.zeros_like(K)
    _load().msa_oracle_route_backward(_p(Q, _dp), B, T, _p(K, _dp), _p(off, _i64p), off.size - 1,
                                      H_r, d_r, _p(g, _dp), _p(dQ, _dp), _p(dK, _dp))
    return dQ, dK


def attend_backward(Q, K_loc, V_loc, q_start: int, Kbar, Vbar, doc_chunk_off, ids,
                    pos_offset: int, theta: float, dO):
    """Gradients of sum(dO * O) for the attention of ``attend`` with respect to Q (before RoPE),
    the local keys (before RoPE) and values, and the pooled memory rows Kbar / Vbar:
    (dQ, dK_loc, dV_loc, dKbar, dVbar)."""
    Q, Kl, Vl, g = f64(Q), f64(K_loc), f64(V_loc), f64(dO)
    B, T, H_q, D = Q.shape
    _, L_loc, H_kv, _ = Kl.shape
    if q_start + T > L_loc:
        raise ValueError("local history shorter than q_start + T")
    Kb, Vb = f64(Kbar), f64(Vbar)
    off = _i64(doc_chunk_off)
    idx = _i32(ids)
    k = idx.shape[1]
    dQ = np.zeros_like(Q)
    dK = np.zeros_like(Kl)
    dV = np.zeros_like(Vl)
    dKb = np.zeros_like(Kb)
    dVb = np.zeros_like(Vb)
    _load().msa_oracle_attend_backward(_p(Q, _dp), B, T, H_q, _p(Kl, _dp), _p(Vl, _dp), L_loc,
                                       q_start, _p(Kb, _dp), _p(Vb, _dp), _p(off, _i64p),
                                       _p(idx, _i32p), k, H_kv, D, pos_offset, theta, _p(g, _dp),
                                       Kb.shape[0], _p(dQ, _dp), _p(dK, _dp), _p(dV, _dp),
                                       _p(dKb, _dp), _p(dVb, _dp))
    return dQ, dK, dV, dKb, dVb
