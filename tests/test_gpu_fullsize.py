"""Full-size parity on sampled outputs, in the launch configuration bench.py times: one routed
layer of the 1M-token workload (device-resident content) and of the 100M-token workload (content
in pinned host memory, fetched per step).  The oracle cannot hold these memories, so it checks
what it can compute one by one: sampled documents are encoded alone (document-wise RoPE makes
that exact) and scored against sampled queries; the planted documents must be the retrieved set;
a decode step's attention output is recomputed for sampled queries over the planted documents."""
import numpy as np
import pytest
import torch

import oracle
from top_document_sparse_b200 import inputs
from top_document_sparse_b200.workloads import WORKLOADS

from helpers import assert_close, bf16_ulp, chunk_abs_mean, to64

pytestmark = pytest.mark.gpu


def _build_layer(w, msa, seed, sample_docs, host_tier, q_sample):
    """Encode one layer exactly as bench.py does (device generation in ~256K-token blocks) and
    keep the raw tokens of `sample_docs` on the host."""
    off = inputs.doc_offsets(w, seed)
    B, T, k = w.batch, w.query_tokens, w.top_k
    mem = msa.Memory(off, w.chunk_len, w.n_kv_heads, w.head_dim, w.n_router_heads, w.router_dim,
                     torch.bfloat16, w.rope_theta, k + T + w.decode_steps)
    rk = mem.new_router_keys()
    ct = mem.new_content(device="cpu", pin_memory=True) if host_tier else mem.new_content()
    Qr, Q, Kn, Vn = inputs.queries(w, B, T, seed=seed * 1000 + 1, device="cuda")
    plants = inputs.choose_plants(w, off, B, T, w.planted_per_query, seed=seed * 1000)
    pb, pd, pc, pt = plants
    block = max(1, (1 << 18) // int(off[1] - off[0]))
    keep = {}
    want = set(int(d) for d in sample_docs) | set(int(d) for d in pd[np.isin(pb, q_sample)])
    for d0 in range(0, mem.n_docs, block):
        d1 = min(mem.n_docs, d0 + block)
        t0, t1 = int(off[d0]), int(off[d1])
        K, V, Kr = inputs.raw_memory(w, t1 - t0, seed=(seed * 1000) * 100003 + d0, device="cuda")
        sel = (pd >= d0) & (pd < d1)
        if sel.any():
            inputs.plant(w, Kr, Qr, off, (pb[sel], pd[sel], pc[sel], pt[sel]), w.planted_cos,
                         seed=seed * 1000, tok_base=t0)
        mem.encode(d0, d1 - d0, K, V, Kr, rk, ct)
        for d in want:
            if d0 <= d < d1:
                a, b = int(off[d]) - t0, int(off[d + 1]) - t0
                keep[d] = (K[a:b].cpu(), V[a:b].cpu(), Kr[a:b].cpu())
        del K, V, Kr
    torch.cuda.synchronize()
    return off, mem, rk, ct, (Qr, Q, Kn, Vn), plants, keep


def _oracle_doc(keep, d, w):
    K, V, Kr = keep[d]
    return oracle.encode(K, V, Kr, np.array([0, K.shape[0]]), w.chunk_len, w.rope_theta)


@pytest.mark.parametrize("name", ["mem1m_bf16", "mem100m_bf16"])
def test_full_size_route_and_decode_on_sampled_outputs(name):
    from top_document_sparse_b200 import msa
    w = WORKLOADS[name]
    host = w.content_on_host
    rng = np.random.default_rng(5)
    off_probe = inputs.doc_offsets(w, 11)
    sample = rng.choice(off_probe.size - 1, size=24, replace=False)
    q_sample = [0, w.batch - 1]
    off, mem, rk, ct, (Qr, Q, Kn, Vn), plants, keep = _build_layer(w, msa, 11, sample, host,
                                                                   q_sample)
    pb, pd, _, _ = plants
    B, T, k, H_q, D = w.batch, w.query_tokens, w.top_k, w.n_q_heads, w.head_dim
    layer = msa.LayerDecode(mem, B, k, H_q, T + w.decode_steps)
    # prefill route + attend (bench launch configuration)
    mem.route(rk, Qr, k, layer.state, layer.ids, layer.scores,
              msa.workspace(mem.route_workspace_size(B, T, k)))
    O = torch.empty(B, T, H_q, D, dtype=torch.bfloat16, device="cuda")
    ws_a = msa.workspace(mem.attend_workspace_size(B, T, k, H_q))
    f = None
    if host:
        f = msa.Fetcher(mem, ct, n_slots=4 * B * k, max_batch=B, max_k=k)
        f.fetch(layer.ids)
        f.sparse_attend(layer.ids, Q, Kn, Vn, layer.k_cache, layer.v_cache, layer.cache_len, k, O,
                        ws_a)
    else:
        mem.sparse_attend(ct, layer.ids, Q, Kn, Vn, layer.k_cache, layer.v_cache, layer.cache_len,
                          k, O, ws_a)
    # one decode step
    dec = inputs.queries(w, B, 1, seed=99)
    Ot = torch.empty(B, H_q, D, dtype=torch.bfloat16, device="cuda")
    args = (dec[0][:, 0].cuda().contiguous(), dec[1][:, 0].cuda().contiguous(),
            dec[2][:, 0].cuda().contiguous(), dec[3][:, 0].cuda().contiguous(), Ot)
    if host:
        f.step(rk, layer, *args)
    else:
        mem.step(rk, ct, layer, *args)
    torch.cuda.synchronize()
    assert msa.device_error() == 0
    assert layer.cache_len.cpu().tolist() == [T + 1] * B  # prefill, then one decode token
    ids = layer.ids.cpu().numpy()
    state = to64(layer.state)

    # 1. every query retrieves exactly its planted documents (planted 0.5 vs background < 0.3)
    for b in range(B):
        assert set(ids[b].tolist()) == set(pd[pb == b].tolist()), f"query {b}"

    # 2. sampled documents: pooled content and document scores against the oracle
    Qr_all = torch.cat([Qr.cpu(), dec[0].cpu()], dim=1)          # prefill + decode tokens
    cho = mem.doc_chunk_offsets
    for d in sample:
        Kb, Vb, Krb = _oracle_doc(keep, int(d), w)
        got = ct[cho[d]:cho[d + 1]]
        sV = chunk_abs_mean(to64(keep[int(d)][1]), np.array([0, keep[int(d)][1].shape[0]]),
                            w.chunk_len)
        assert_close(got[:, 1], Vb, 1e-6 * sV + bf16_ulp(Vb), f"pooled V of doc {d}")
        ref = oracle.route(Qr_all[q_sample], Krb, np.array([0, Krb.shape[0]]))
        assert_close(state[q_sample, d], ref[:, 0], 2e-3, f"score of doc {d}")

    # 3. decode attention of sampled queries over their planted documents
    for b in q_sample:
        docs = [int(d) for d in ids[b]]                 # == the planted set, checked above
        assert set(docs) == set(pd[pb == b].tolist())
        enc = [_oracle_doc(keep, d, w) for d in docs]
        Kb = np.concatenate([e[0] for e in enc])
        Vb = np.concatenate([e[1] for e in enc])
        mini_off = np.concatenate([[0], np.cumsum([e[0].shape[0] for e in enc])])
        Khist = torch.cat([Kn[b:b + 1].cpu(), dec[2][b:b + 1]], dim=1)
        Vhist = torch.cat([Vn[b:b + 1].cpu(), dec[3][b:b + 1]], dim=1)
        ref, _, _ = oracle.attend(dec[1][b:b + 1], Khist, Vhist, T, Kb, Vb, mini_off,
                                  np.arange(len(docs), dtype=np.int32)[None], k, w.rope_theta)
        assert_close(Ot[b:b + 1], ref[:, 0], 1e-2 + 0.5 * bf16_ulp(ref[:, 0]),
                     f"decode attention of query {b}")
    if f is not None:
        f.close()
