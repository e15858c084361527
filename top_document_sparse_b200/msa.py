"""ctypes binding of libmsa.so (C ABI in include/msa.h).

Argument marshalling only: tensors become device pointers, streams become cudaStream_t handles,
statuses become exceptions.  Every step of the hot path runs in the library's CUDA kernels; there
is no CPU fallback, and importing this module fails loudly when the library cannot be loaded.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np
import torch

from . import build as _build

_HERE = os.path.dirname(os.path.abspath(__file__))

MSA_F32, MSA_BF16 = 0, 1
DEVERR_BAD_DOC_ID, DEVERR_CACHE_OVERFLOW, DEVERR_WAIT_TIMEOUT = 0x1, 0x2, 0x4
STATUS = {0: "MSA_OK", 1: "MSA_ERR_INVALID_ARG", 2: "MSA_ERR_UNSUPPORTED", 3: "MSA_ERR_CUDA",
          4: "MSA_ERR_OUT_OF_MEMORY", 5: "MSA_ERR_TIMEOUT", 6: "MSA_ERR_STATE"}
_DTYPE = {torch.float32: MSA_F32, torch.bfloat16: MSA_BF16}
_TORCH = {MSA_F32: torch.float32, MSA_BF16: torch.bfloat16}


class MsaError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"{STATUS.get(status, status)}: {message}")
        self.status = status


class MemoryConfig(ctypes.Structure):
    _fields_ = [("n_docs", ctypes.c_int32), ("doc_token_offsets", ctypes.POINTER(ctypes.c_int64)),
                ("chunk_len", ctypes.c_int32), ("n_kv_heads", ctypes.c_int32),
                ("head_dim", ctypes.c_int32), ("n_router_heads", ctypes.c_int32),
                ("router_dim", ctypes.c_int32), ("dtype", ctypes.c_int),
                ("rope_theta", ctypes.c_double), ("max_local_position", ctypes.c_int32)]


class MemoryInfo(ctypes.Structure):
    _fields_ = [("n_tokens", ctypes.c_int64), ("n_chunks", ctypes.c_int64),
                ("max_doc_chunks", ctypes.c_int32), ("max_doc_tokens", ctypes.c_int64),
                ("elem_bytes", ctypes.c_size_t), ("router_key_bytes", ctypes.c_size_t),
                ("content_bytes", ctypes.c_size_t), ("doc_content_stride", ctypes.c_size_t)]


class DecodeState(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int32), ("top_k", ctypes.c_int32),
                ("n_q_heads", ctypes.c_int32), ("cache_capacity", ctypes.c_int32),
                ("pos_offset", ctypes.c_int32), ("state", ctypes.c_void_p),
                ("ids", ctypes.c_void_p), ("scores", ctypes.c_void_p),
                ("k_cache", ctypes.c_void_p), ("v_cache", ctypes.c_void_p),
                ("cache_len", ctypes.c_void_p), ("workspace", ctypes.c_void_p),
                ("workspace_bytes", ctypes.c_size_t)]


_P = ctypes.c_void_p
_I32 = ctypes.c_int32
_I64 = ctypes.c_int64
_SZ = ctypes.c_size_t

# name -> (restype, argtypes); must match include/msa.h
SIGNATURES = {
    "msa_memory_create": (ctypes.c_int, [ctypes.POINTER(MemoryConfig), ctypes.POINTER(_P)]),
    "msa_memory_destroy": (ctypes.c_int, [_P]),
    "msa_memory_get_info": (ctypes.c_int, [_P, ctypes.POINTER(MemoryInfo)]),
    "msa_memory_doc_chunk_offsets": (ctypes.c_int, [_P, ctypes.POINTER(ctypes.c_int64)]),
    "msa_encode_memory": (ctypes.c_int, [_P, _I32, _I32, _P, _P, _P, _P, _P, _P, _P]),
    "msa_route_reset": (ctypes.c_int, [_P, _I64, _P]),
    "msa_route_workspace_size": (_SZ, [_P, _I32, _I32, _I32]),
    "msa_route": (ctypes.c_int, [_P, _P, _P, _I32, _I32, _I32, _P, _P, _P, _P, _P, _SZ, _P]),
    "msa_attend_workspace_size": (_SZ, [_P, _I32, _I32, _I32, _I32]),
    "msa_sparse_attend": (ctypes.c_int, [_P, _P, _P, _I32, _I32, _I32, _I32, _P, _P, _P, _P, _P,
                                         _P, _I32, _I32, _P, _P, _SZ, _P]),
    "msa_sparse_attend_static": (ctypes.c_int, [_P, _P, _P, _I32, _I32, _I32, _I32, _P, _P, _P,
                                                _P, _P, _P, _I32, _I32, _P, _P]),
    "msa_step_workspace_size": (_SZ, [_P, _I32, _I32, _I32]),
    "msa_step": (ctypes.c_int, [_P, _P, _P, ctypes.POINTER(DecodeState), _P, _P, _P, _P, _P, _P]),
    "msa_fetcher_create": (ctypes.c_int, [_P, _P, _P, _I32, _I32, _I32, ctypes.c_uint32,
                                          ctypes.POINTER(_P)]),
    "msa_fetcher_destroy": (ctypes.c_int, [_P]),
    "msa_fetcher_stats": (ctypes.c_int, [_P, ctypes.POINTER(_I64), ctypes.POINTER(_I64),
                                         ctypes.POINTER(_I64), ctypes.POINTER(_I64)]),
    "msa_fetch": (ctypes.c_int, [_P, _P, _I32, _I32, _P, _P]),
    "msa_sparse_attend_fetched": (ctypes.c_int, [_P, _P, _P, _I32, _I32, _I32, _I32, _P, _P, _P,
                                                 _P, _P, _P, _I32, _I32, _P, _P, _SZ, _P]),
    "msa_step_host": (ctypes.c_int, [_P, _P, _P, ctypes.POINTER(DecodeState), _P, _P, _P, _P, _P,
                                     _P, _P]),
    "msa_interleave_workspace_size": (_SZ, [_P, _I32, _I32, _I32]),
    "msa_interleave": (ctypes.c_int, [_P, _P, _P, _I32, _I32, _I32, _I32, _P, _P, _P, _P, _P, _SZ,
                                      _P]),
    "msa_interleave_adaptive": (ctypes.c_int, [_P, _P, _P, _I32, _I32, _I32, _I32, ctypes.c_float,
                                               _P, _P, _P, _P, _P, _P, _SZ, _P]),
    "msa_topk_merge": (ctypes.c_int, [_P, _P, _I32, _I32, _I32, ctypes.POINTER(_I32), _I32, _P,
                                      _P, _P]),
    "msa_route_backward": (ctypes.c_int, [_P, _P, _P, _I32, _I32, _P, _P, _P, _P]),
    "msa_sparse_attend_backward": (ctypes.c_int, [_P, _P, _P, _I32, _I32, _I32, _I32, _P, _P,
                                                  _P, _P, _I32, _I32, _P, _P, _P, _P, _P, _P]),
    "msa_device_error": (ctypes.c_int, [ctypes.POINTER(ctypes.c_uint32), _P]),
    "msa_status_string": (ctypes.c_char_p, [ctypes.c_int]),
    "msa_last_error": (ctypes.c_char_p, []),
    "msa_version": (ctypes.c_int32, []),
    "msa_launch_count": (ctypes.c_uint64, []),
}


def load_library(path: str | None = None) -> ctypes.CDLL:
    """Load (building first when stale) libmsa.so; raises if it cannot be loaded."""
    if path is None:
        path = _build.LIB
        if _build.stale():
            _build.build()
    lib = ctypes.CDLL(path)
    for name, (res, args) in SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib


_lib = load_library()


def lib() -> ctypes.CDLL:
    return _lib


def launch_count() -> int:
    """Kernels the library has enqueued (graph captures count once, at capture)."""
    return int(_lib.msa_launch_count())


def _check(status: int):
    if status != 0:
        raise MsaError(status, _lib.msa_last_error().decode())


def _ptr(t) -> int | None:
    if t is None:
        return None
    if not isinstance(t, torch.Tensor):
        raise TypeError("expected a torch.Tensor")
    if not t.is_contiguous():
        raise ValueError("tensors must be contiguous")
    return t.data_ptr()


def _stream(stream) -> int:
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream


def device_error(stream=None) -> int:
    """Read and clear the device error word (MSA_DEVERR_* bits)."""
    bits = ctypes.c_uint32(0)
    _lib.msa_device_error(ctypes.byref(bits), _stream(stream))
    return bits.value


class Memory:
    """One memory layout (documents, chunking, head shapes) and its device tables.

    Router keys and pooled content live in caller tensors: ``router_keys`` [C][H_r][d_r] and
    ``content`` [C][2][H_kv][D] (device, or pinned host for content)."""

    def __init__(self, doc_token_offsets, chunk_len: int, n_kv_heads: int, head_dim: int,
                 n_router_heads: int, router_dim: int, dtype: torch.dtype, rope_theta: float,
                 max_local_position: int):
        off = np.ascontiguousarray(np.asarray(doc_token_offsets, dtype=np.int64))
        self._off = off
        cfg = MemoryConfig(n_docs=off.size - 1,
                           doc_token_offsets=off.ctypes.data_as(ctypes.POINTER(ctypes.c_int64)),
                           chunk_len=chunk_len, n_kv_heads=n_kv_heads, head_dim=head_dim,
                           n_router_heads=n_router_heads, router_dim=router_dim,
                           dtype=_DTYPE[dtype], rope_theta=rope_theta,
                           max_local_position=max_local_position)
        h = _P()
        _check(_lib.msa_memory_create(ctypes.byref(cfg), ctypes.byref(h)))
        self.handle = h
        self.dtype = dtype
        self.n_docs = off.size - 1
        self.chunk_len, self.n_kv_heads, self.head_dim = chunk_len, n_kv_heads, head_dim
        self.n_router_heads, self.router_dim = n_router_heads, router_dim
        info = MemoryInfo()
        _check(_lib.msa_memory_get_info(h, ctypes.byref(info)))
        self.info = info
        self.n_chunks = info.n_chunks
        co = np.zeros(self.n_docs + 1, dtype=np.int64)
        _check(_lib.msa_memory_doc_chunk_offsets(h, co.ctypes.data_as(ctypes.POINTER(ctypes.c_int64))))
        self.doc_chunk_offsets = co

    def close(self):
        if getattr(self, "handle", None):
            _check(_lib.msa_memory_destroy(self.handle))
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    # -- storage -----------------------------------------------------------------------------
    def new_router_keys(self, device="cuda") -> torch.Tensor:
        return torch.empty(self.n_chunks, self.n_router_heads, self.router_dim, dtype=self.dtype,
                           device=device)

    def new_content(self, device="cuda", pin_memory=False) -> torch.Tensor:
        t = torch.empty(self.n_chunks, 2, self.n_kv_heads, self.head_dim, dtype=self.dtype,
                        device=device, pin_memory=pin_memory)
        return t

    # -- calls -------------------------------------------------------------------------------
    def encode(self, doc_begin: int, doc_count: int, K, V, Kr, router_keys, content,
               router_mean=None, stream=None):
        _check(_lib.msa_encode_memory(self.handle, doc_begin, doc_count, _ptr(K), _ptr(V), _ptr(Kr),
                                      _ptr(router_keys), _ptr(content), _ptr(router_mean),
                                      _stream(stream)))

    def route_workspace_size(self, batch: int, tokens: int, k: int) -> int:
        return _lib.msa_route_workspace_size(self.handle, batch, tokens, k)

    def route(self, router_keys, Qr, k: int, state, ids, scores, workspace, exclude=None,
              stream=None):
        B = state.shape[0]
        T = Qr.shape[1] if Qr is not None else 0
        ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
        _check(_lib.msa_route(self.handle, _ptr(router_keys), _ptr(Qr), B, T, k, _ptr(exclude),
                              _ptr(state), _ptr(ids), _ptr(scores), _ptr(workspace), ws_bytes,
                              _stream(stream)))

    def attend_workspace_size(self, batch: int, tokens: int, k: int, n_q_heads: int) -> int:
        return _lib.msa_attend_workspace_size(self.handle, batch, tokens, k, n_q_heads)

    def sparse_attend(self, content, ids, Q, K_new, V_new, K_cache, V_cache, cache_len,
                      pos_offset: int, O, workspace, stream=None):
        B, T, H_q, _ = Q.shape
        k = ids.shape[1] if ids is not None else 0
        ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
        _check(_lib.msa_sparse_attend(self.handle, _ptr(content), _ptr(ids), B, k, T, H_q, _ptr(Q),
                                      _ptr(K_new), _ptr(V_new), _ptr(K_cache), _ptr(V_cache),
                                      _ptr(cache_len), K_cache.shape[1], pos_offset, _ptr(O),
                                      _ptr(workspace), ws_bytes, _stream(stream)))

    def sparse_attend_static(self, content, ids, Q, K_new, V_new, K_cache, V_cache, cache_len,
                             pos_offset: int, O, stream=None):
        """msa_sparse_attend without a workspace: scratch from the library's fixed array."""
        B, T, H_q, _ = Q.shape
        k = ids.shape[1] if ids is not None else 0
        _check(_lib.msa_sparse_attend_static(self.handle, _ptr(content), _ptr(ids), B, k, T, H_q,
                                             _ptr(Q), _ptr(K_new), _ptr(V_new), _ptr(K_cache),
                                             _ptr(V_cache), _ptr(cache_len), K_cache.shape[1],
                                             pos_offset, _ptr(O), _stream(stream)))

    def interleave(self, router_keys, Qr, k: int, rounds: int, stream=None):
        """Memory Interleave rounds (msa_interleave): returns (ids [rounds][B][k], scores,
        state [B][n_docs], taken [B][n_docs])."""
        B, T = Qr.shape[0], Qr.shape[1]
        dev = Qr.device
        state = torch.empty(B, self.n_docs, dtype=torch.float32, device=dev)
        taken = torch.empty(B, self.n_docs, dtype=torch.uint8, device=dev)
        ids = torch.empty(rounds, B, k, dtype=torch.int32, device=dev)
        scores = torch.empty(rounds, B, k, dtype=torch.float32, device=dev)
        ws = workspace(_lib.msa_interleave_workspace_size(self.handle, B, T, k), dev)
        _check(_lib.msa_interleave(self.handle, _ptr(router_keys), _ptr(Qr), B, T, k, rounds,
                                   _ptr(state), _ptr(taken), _ptr(ids), _ptr(scores), _ptr(ws),
                                   ws.numel(), _stream(stream)))
        return ids, scores, state, taken

    def interleave_adaptive(self, router_keys, Qr, k: int, max_rounds: int, stop_score: float,
                            stream=None):
        """Adaptive Memory Interleave (msa_interleave_adaptive): returns (ids [max_rounds][B][k],
        scores, state [B][n_docs], taken [B][n_docs], n_rounds [B])."""
        B, T = Qr.shape[0], Qr.shape[1]
        dev = Qr.device
        state = torch.empty(B, self.n_docs, dtype=torch.float32, device=dev)
        taken = torch.empty(B, self.n_docs, dtype=torch.uint8, device=dev)
        ids = torch.empty(max_rounds, B, k, dtype=torch.int32, device=dev)
        scores = torch.empty(max_rounds, B, k, dtype=torch.float32, device=dev)
        n_rounds = torch.empty(B, dtype=torch.int32, device=dev)
        ws = workspace(_lib.msa_interleave_workspace_size(self.handle, B, T, k), dev)
        _check(_lib.msa_interleave_adaptive(self.handle, _ptr(router_keys), _ptr(Qr), B, T, k,
                                            max_rounds, float(stop_score), _ptr(state),
                                            _ptr(taken), _ptr(ids), _ptr(scores), _ptr(n_rounds),
                                            _ptr(ws), ws.numel(), _stream(stream)))
        return ids, scores, state, taken, n_rounds

    def route_backward(self, router_mean, Qr, d_score, stream=None):
        """Gradients of sum(d_score * doc_score) of one routing call of Qr [B][T][H_r][d_r]
        (msa_route_backward): (d_Qr, d_router_mean), fp32."""
        B, T = Qr.shape[0], Qr.shape[1]
        dQr = torch.empty(Qr.shape, dtype=torch.float32, device=Qr.device)
        dM = torch.empty(router_mean.shape, dtype=torch.float32, device=Qr.device)
        _check(_lib.msa_route_backward(self.handle, _ptr(router_mean), _ptr(Qr), B, T,
                                       _ptr(d_score), _ptr(dQr), _ptr(dM), _stream(stream)))
        return dQr, dM

    def sparse_attend_backward(self, content, ids, Q, K_cache, V_cache, cache_len0,
                               pos_offset: int, dO, stream=None):
        """Gradients of sum(dO * O) of a msa_sparse_attend call (msa_sparse_attend_backward):
        (dQ, d_cache_k, d_cache_v, d_content), fp32."""
        B, T, H_q, _ = Q.shape
        k = ids.shape[1] if ids is not None else 0
        dev = Q.device
        dQ = torch.empty(Q.shape, dtype=torch.float32, device=dev)
        dKc = torch.empty(K_cache.shape, dtype=torch.float32, device=dev)
        dVc = torch.empty(V_cache.shape, dtype=torch.float32, device=dev)
        dC = torch.empty(content.shape, dtype=torch.float32, device=dev)
        _check(_lib.msa_sparse_attend_backward(
            self.handle, _ptr(content), _ptr(ids), B, k, T, H_q, _ptr(Q), _ptr(K_cache),
            _ptr(V_cache), _ptr(cache_len0), K_cache.shape[1], pos_offset, _ptr(dO), _ptr(dQ),
            _ptr(dKc), _ptr(dVc), _ptr(dC), _stream(stream)))
        return dQ, dKc, dVc, dC

    def step_workspace_size(self, batch: int, k: int, n_q_heads: int) -> int:
        return _lib.msa_step_workspace_size(self.handle, batch, k, n_q_heads)

    def step(self, router_keys, content, st: "LayerDecode", Qr_tok, Q_tok, K_tok, V_tok, O_tok,
             stream=None):
        _check(_lib.msa_step(self.handle, _ptr(router_keys), _ptr(content), ctypes.byref(st.c),
                             _ptr(Qr_tok), _ptr(Q_tok), _ptr(K_tok), _ptr(V_tok), _ptr(O_tok),
                             _stream(stream)))


FETCH_COLD = 0x1


class Fetcher:
    """Host tier of one layer's pooled content: pinned host content plus a device slot cache
    (msa_fetcher_*).  Owns neither buffer; keeps references so they outlive it."""

    def __init__(self, mem: Memory, content_host: torch.Tensor, n_slots: int, max_batch: int,
                 max_k: int, cold: bool = False, device="cuda"):
        if not content_host.is_pinned():
            raise ValueError("content_host must be pinned host memory")
        self.mem = mem
        self.content_host = content_host
        self.slot_cache = torch.empty(n_slots * mem.info.doc_content_stride, dtype=torch.uint8,
                                      device=device)
        h = _P()
        _check(_lib.msa_fetcher_create(mem.handle, content_host.data_ptr(),
                                       self.slot_cache.data_ptr(), n_slots, max_batch, max_k,
                                       FETCH_COLD if cold else 0, ctypes.byref(h)))
        self.handle = h

    def close(self):
        if getattr(self, "handle", None):
            _check(_lib.msa_fetcher_destroy(self.handle))
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def stats(self) -> dict:
        v = [_I64() for _ in range(4)]
        _check(_lib.msa_fetcher_stats(self.handle, *[ctypes.byref(x) for x in v]))
        return dict(zip(("hits", "misses", "copies", "bytes"), (x.value for x in v)))

    def fetch(self, ids, stream=None, fetch_stream=None):
        B, k = ids.shape
        _check(_lib.msa_fetch(self.handle, _ptr(ids), B, k, _stream(stream),
                              _stream(fetch_stream) if fetch_stream is not None else _stream(stream)))

    def sparse_attend(self, ids, Q, K_new, V_new, K_cache, V_cache, cache_len, pos_offset: int,
                      O, workspace, stream=None):
        B, T, H_q, _ = Q.shape
        k = ids.shape[1]
        ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
        _check(_lib.msa_sparse_attend_fetched(self.mem.handle, self.handle, _ptr(ids), B, k, T, H_q,
                                              _ptr(Q), _ptr(K_new), _ptr(V_new), _ptr(K_cache),
                                              _ptr(V_cache), _ptr(cache_len), K_cache.shape[1],
                                              pos_offset, _ptr(O), _ptr(workspace), ws_bytes,
                                              _stream(stream)))

    def step(self, router_keys, st: "LayerDecode", Qr_tok, Q_tok, K_tok, V_tok, O_tok,
             stream=None, fetch_stream=None):
        _check(_lib.msa_step_host(self.mem.handle, _ptr(router_keys), self.handle,
                                  ctypes.byref(st.c), _ptr(Qr_tok), _ptr(Q_tok), _ptr(K_tok),
                                  _ptr(V_tok), _ptr(O_tok), _stream(stream),
                                  _stream(fetch_stream) if fetch_stream is not None
                                  else _stream(stream)))


def topk_merge(cand_scores, cand_ids, shard_doc_base, k: int, stream=None):
    """Global top-k from every memory shard's candidates (msa_topk_merge).

    cand_scores / cand_ids: device [n_shards][B][k_cand] (each shard's msa_route output, ids
    local to the shard); shard_doc_base: the global id of each shard's document 0.  Returns
    (ids [B][k] global, scores [B][k])."""
    n_shards, B, kc = cand_ids.shape
    base = (ctypes.c_int32 * n_shards)(*[int(x) for x in shard_doc_base])
    ids = torch.empty(B, k, dtype=torch.int32, device=cand_ids.device)
    scores = torch.empty(B, k, dtype=torch.float32, device=cand_ids.device)
    _check(_lib.msa_topk_merge(_ptr(cand_scores), _ptr(cand_ids), n_shards, B, kc, base, k,
                               _ptr(ids), _ptr(scores), _stream(stream)))
    return ids, scores


def workspace(nbytes: int, device="cuda") -> torch.Tensor:
    return torch.empty(max(int(nbytes), 16), dtype=torch.uint8, device=device)


class LayerDecode:
    """Per-layer decode buffers (all torch-allocated) bundled as an msa_decode_state."""

    def __init__(self, mem: Memory, batch: int, k: int, n_q_heads: int, cache_capacity: int,
                 pos_offset: int | None = None, device="cuda", cache_len=None):
        self.state = torch.full((batch, mem.n_docs), float("-inf"), dtype=torch.float32,
                                device=device)
        self.ids = torch.zeros(batch, k, dtype=torch.int32, device=device)
        self.scores = torch.zeros(batch, k, dtype=torch.float32, device=device)
        self.k_cache = torch.zeros(batch, cache_capacity, mem.n_kv_heads, mem.head_dim,
                                   dtype=mem.dtype, device=device)
        self.v_cache = torch.zeros_like(self.k_cache)
        # cache_len may be a caller's view (e.g. one row of a [layers][batch] tensor, so that
        # every layer's length can be set by one copy)
        if cache_len is None:
            cache_len = torch.zeros(batch, dtype=torch.int32, device=device)
        if cache_len.shape != (batch,) or cache_len.dtype != torch.int32:
            raise ValueError("cache_len must be int32 [batch]")
        self.cache_len = cache_len
        self.workspace = workspace(mem.step_workspace_size(batch, k, n_q_heads), device)
        self.pos_offset = k if pos_offset is None else pos_offset
        self.c = DecodeState(batch=batch, top_k=k, n_q_heads=n_q_heads,
                             cache_capacity=cache_capacity, pos_offset=self.pos_offset,
                             state=_ptr(self.state), ids=_ptr(self.ids), scores=_ptr(self.scores),
                             k_cache=_ptr(self.k_cache), v_cache=_ptr(self.v_cache),
                             cache_len=_ptr(self.cache_len), workspace=_ptr(self.workspace),
                             workspace_bytes=self.workspace.numel())
