"""Per-stage timing of the MSA hot path at a workload's sizes (one routed layer, one decode token).

    python -m top_document_sparse_b200.kernel_bench [--workload mem1m_bf16] [--stage all]
                                                    [--reps 20]

Stages: ``route`` (msa_route: query normalisation, route score, top-k), ``topk`` (msa_route with
no query rows), ``attend`` (msa_sparse_attend of one token over k retrieved documents plus the
local cache), ``prefill`` (msa_sparse_attend of the workload's query tokens), and the widening
calls: ``backward`` (msa_route_backward and msa_sparse_attend_backward of one decode token),
``merge`` (msa_topk_merge of four shards' candidates) and ``update`` (msa_encode_memory of one
512-token document).  The router keys are random unit vectors and the pooled content random bf16, so
no encode pass is needed.  Calls are captured in a CUDA graph and timed with CUDA events; each
call reads more than the 126 MB L2 only for memories of 64K+ chunks, so small workloads report
L2-warm figures (printed as "l2_warm").  Used for the ncu captures summarised under profiles/.
"""
from __future__ import annotations

import argparse
import json

import numpy as np
import torch

from . import msa
from .inputs import doc_offsets
from .workloads import WORKLOADS


def _graph_time(fn, reps):
    s = torch.cuda.Stream()
    torch.cuda.synchronize()
    with torch.cuda.stream(s):
        fn()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        for _ in range(reps):
            fn()
    g.replay()
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    g.replay()
    b.record()
    torch.cuda.synchronize()
    return a.elapsed_time(b) / reps * 1e3  # us per call


STAGES = ["all", "route", "topk", "attend", "prefill", "backward", "merge", "update"]


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--workload", default="mem1m_bf16")
    ap.add_argument("--stage", default="all", choices=STAGES)
    ap.add_argument("--reps", type=int, default=20)
    ap.add_argument("--seed", type=int, default=0)
    a = ap.parse_args(argv)
    print(json.dumps(run(a.workload, [a.stage], a.reps, a.seed)))


def run(workload: str, stages, reps: int = 20, seed: int = 0) -> dict:
    """Time the given stages (names from STAGES; "all" = route, topk and attend) and return
    their figures as one dict."""
    st_set = set(stages)
    if "all" in st_set:
        st_set |= {"route", "topk", "attend"}
    w = WORKLOADS[workload]
    torch.cuda.set_device(0)
    gen = torch.Generator(device="cuda")
    gen.manual_seed(seed)
    off = doc_offsets(w, seed)
    B, k, H_q, D, H_kv = w.batch, w.top_k, w.n_q_heads, w.head_dim, w.n_kv_heads
    cap = w.query_tokens + max(w.decode_steps, 1)
    mem = msa.Memory(off, w.chunk_len, H_kv, D, w.n_router_heads, w.router_dim, torch.bfloat16,
                     w.rope_theta, k + cap)
    W = w.n_router_heads * w.router_dim
    out = {"workload": w.name, "chunks": int(mem.n_chunks), "batch": B, "top_k": k,
           "l2_warm": mem.n_chunks * W * 2 < (126 << 20)}
    if st_set & {"route", "topk"}:
        rk = torch.randn(mem.n_chunks, w.n_router_heads, w.router_dim, device="cuda",
                         generator=gen)
        rk = (rk / rk.norm(dim=-1, keepdim=True)).to(torch.bfloat16)
        Qr = torch.randn(B, 1, w.n_router_heads, w.router_dim, device="cuda",
                         generator=gen).to(torch.bfloat16)
        st = torch.full((B, mem.n_docs), float("-inf"), device="cuda")
        ids = torch.zeros(B, k, dtype=torch.int32, device="cuda")
        sc = torch.zeros(B, k, device="cuda")
        ws = msa.workspace(mem.route_workspace_size(B, 1, k))
        byts = mem.n_chunks * W * 2 + 2 * B * mem.n_docs * 4
        if "route" in st_set:
            t = _graph_time(lambda: mem.route(rk, Qr, k, st, ids, sc, ws), reps)
            out["route_us"] = round(t, 2)
            out["route_gbs"] = round(byts / (t * 1e-6) / 1e9, 1)
        if "topk" in st_set:
            out["topk_us"] = round(_graph_time(lambda: mem.route(None, None, k, st, ids, sc, ws),
                                               reps), 2)
        del rk
    if "attend" in st_set:
        ct = torch.randn(mem.n_chunks, 2, H_kv, D, device="cuda", generator=gen).to(torch.bfloat16)
        ids = torch.from_numpy(np.stack([np.random.default_rng(b).choice(mem.n_docs, k, replace=False)
                                         for b in range(B)]).astype(np.int32)).cuda()
        Kc = torch.randn(B, cap, H_kv, D, device="cuda", generator=gen).to(torch.bfloat16)
        Vc = torch.randn(B, cap, H_kv, D, device="cuda", generator=gen).to(torch.bfloat16)
        Q = torch.randn(B, 1, H_q, D, device="cuda", generator=gen).to(torch.bfloat16)
        Kn = torch.randn(B, 1, H_kv, D, device="cuda", generator=gen).to(torch.bfloat16)
        O = torch.empty_like(Q)
        L0 = w.query_tokens + max(w.decode_steps, 1) // 2
        clen = torch.full((B,), L0, dtype=torch.int32, device="cuda")
        ws = msa.workspace(mem.attend_workspace_size(B, 1, k, H_q))

        def att():
            clen.fill_(L0)
            mem.sparse_attend(ct, ids, Q, Kn, Kn, Kc, Vc, clen, k, O, ws)

        t = _graph_time(att, reps)
        n_mem = int(sum(mem.doc_chunk_offsets[d + 1] - mem.doc_chunk_offsets[d]
                        for d in ids.cpu().numpy().ravel()))
        byts = (n_mem + B * (L0 + 1)) * H_kv * 2 * D * 2
        out["attend_us"] = round(t, 2)
        out["attend_gbs"] = round(byts / (t * 1e-6) / 1e9, 1)
    if "prefill" in st_set:
        # one layer's multi-token attention: the query's T tokens over [k documents | themselves]
        T = w.query_tokens
        ct = torch.randn(mem.n_chunks, 2, H_kv, D, device="cuda", generator=gen).to(torch.bfloat16)
        ids = torch.from_numpy(np.stack([np.random.default_rng(b).choice(mem.n_docs, k, replace=False)
                                         for b in range(B)]).astype(np.int32)).cuda()
        Kc = torch.zeros(B, cap, H_kv, D, dtype=torch.bfloat16, device="cuda")
        Vc = torch.zeros_like(Kc)
        Q = torch.randn(B, T, H_q, D, device="cuda", generator=gen).to(torch.bfloat16)
        Kn = torch.randn(B, T, H_kv, D, device="cuda", generator=gen).to(torch.bfloat16)
        O = torch.empty_like(Q)
        clen = torch.zeros(B, dtype=torch.int32, device="cuda")
        ws = msa.workspace(mem.attend_workspace_size(B, T, k, H_q))

        def pre():
            clen.zero_()
            mem.sparse_attend(ct, ids, Q, Kn, Kn, Kc, Vc, clen, k, O, ws)

        t = _graph_time(pre, reps)
        n_mem = np.array([sum(mem.doc_chunk_offsets[d + 1] - mem.doc_chunk_offsets[d] for d in row)
                          for row in ids.cpu().numpy()], dtype=np.float64)
        # QK^T and PV over every visible (token, context row) pair: 2 x 2 x D flops each
        pairs = float(np.sum(n_mem * T + T * (T + 1) / 2)) * H_q
        out["prefill_us"] = round(t, 2)
        out["prefill_tflops"] = round(4.0 * D * pairs / (t * 1e-6) / 1e12, 1)
    if "backward" in st_set:
        # gradients of one decode token's routing and attention (the plain CUDA-core kernels):
        # bytes = the inputs each call reads once + the fp32 gradient buffers it zeroes and adds to
        rmean = torch.randn(mem.n_chunks, w.n_router_heads, w.router_dim, device="cuda",
                            generator=gen).to(torch.bfloat16)
        Qr = torch.randn(B, 1, w.n_router_heads, w.router_dim, device="cuda",
                         generator=gen).to(torch.bfloat16)
        G = torch.randn(B, mem.n_docs, device="cuda", generator=gen)
        G[:, k:] = 0.0  # the auxiliary loss reaches the k retrieved documents of each query
        t = _graph_time(lambda: mem.route_backward(rmean, Qr, G), reps)
        per_doc = mem.n_chunks / mem.n_docs
        byts = (B * k * per_doc * W * 2 + B * W * 2 + B * mem.n_docs * 4
                + (mem.n_chunks + B) * W * 4)
        out["route_backward_us"] = round(t, 2)
        out["route_backward_gbs"] = round(byts / (t * 1e-6) / 1e9, 1)
        ct = torch.randn(mem.n_chunks, 2, H_kv, D, device="cuda", generator=gen).to(torch.bfloat16)
        ids = torch.from_numpy(np.stack([np.random.default_rng(b).choice(mem.n_docs, k, replace=False)
                                         for b in range(B)]).astype(np.int32)).cuda()
        L0 = w.query_tokens + max(w.decode_steps, 1) // 2
        Kc = torch.randn(B, cap, H_kv, D, device="cuda", generator=gen).to(torch.bfloat16)
        Vc = torch.randn(B, cap, H_kv, D, device="cuda", generator=gen).to(torch.bfloat16)
        Q = torch.randn(B, 1, H_q, D, device="cuda", generator=gen).to(torch.bfloat16)
        dO = torch.randn(B, 1, H_q, D, device="cuda", generator=gen).to(torch.bfloat16)
        len0 = torch.full((B,), L0, dtype=torch.int32, device="cuda")
        t = _graph_time(lambda: mem.sparse_attend_backward(ct, ids, Q, Kc, Vc, len0, k, dO), reps)
        n_mem = int(sum(mem.doc_chunk_offsets[d + 1] - mem.doc_chunk_offsets[d]
                        for d in ids.cpu().numpy().ravel()))
        rows = n_mem + B * (L0 + 1)
        byts = (rows * H_kv * 2 * D * 2 + 2 * B * H_q * D * 2
                + (ct.numel() + 2 * Kc.numel() + Q.numel()) * 4)
        out["attend_backward_us"] = round(t, 2)
        out["attend_backward_gbs"] = round(byts / (t * 1e-6) / 1e9, 1)
    if "merge" in st_set:
        # Memory Parallel: four shards' top-k candidates merged into the global top-k
        n_sh = 4
        cs = torch.randn(n_sh, B, k, device="cuda", generator=gen).sort(dim=-1, descending=True).values
        ci = torch.randint(0, max(mem.n_docs // n_sh, 1), (n_sh, B, k), dtype=torch.int32,
                           device="cuda", generator=gen)
        base = [i * (mem.n_docs // n_sh) for i in range(n_sh)]
        out["merge_us"] = round(_graph_time(lambda: msa.topk_merge(cs, ci, base, k), reps), 2)
    if "update" in st_set:
        # incremental memory update: one document's 512 tokens re-encoded in place
        n_tok = 512
        d = mem.n_docs // 2
        K = torch.randn(n_tok, H_kv, D, device="cuda", generator=gen).to(torch.bfloat16)
        V = torch.randn(n_tok, H_kv, D, device="cuda", generator=gen).to(torch.bfloat16)
        Kr = torch.randn(n_tok, w.n_router_heads, w.router_dim, device="cuda",
                         generator=gen).to(torch.bfloat16)
        rk = mem.new_router_keys()
        ctt = mem.new_content()
        n_doc_tok = int(off[d + 1] - off[d])
        if n_doc_tok != n_tok:
            raise SystemExit(f"document {d} has {n_doc_tok} tokens, not {n_tok}")
        t = _graph_time(lambda: mem.encode(d, 1, K, V, Kr, rk, ctt), reps)
        chunks = (n_tok + w.chunk_len - 1) // w.chunk_len
        byts = n_tok * (2 * H_kv * D + W) * 2 + chunks * (2 * H_kv * D + W) * 2
        out["update_us"] = round(t, 2)
        out["update_gbs"] = round(byts / (t * 1e-6) / 1e9, 1)
    out["device_error"] = msa.device_error()
    return out


if __name__ == "__main__":
    main()
