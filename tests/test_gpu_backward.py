"""Backward passes on the GPU (msa_route_backward, msa_sparse_attend_backward) against the fp64
oracle's gradients (tests/test_oracle_backward.py pins those by finite differences), stage-wise:
the oracle consumes exactly the GPU's inputs -- the stored pooled router means and memory rows,
and the local cache rows as the forward stored them (rotated back to their pre-RoPE values in
fp64 for the oracle, whose key gradients are then rotated forward).  The kernels accumulate in
fp32 on the same inputs, so the bound is fp32 summation: 2e-4 of the largest expected magnitude
of each gradient (n ~ a few hundred terms of mixed sign)."""
import numpy as np
import pytest
import torch

import oracle
from top_document_sparse_b200 import inputs

from helpers import memory_inputs, small_workload, to64

pytestmark = pytest.mark.gpu


def _close(got, want, what, rel=2e-4):
    got, want = to64(got), np.asarray(want, dtype=np.float64)
    tol = rel * max(np.abs(want).max(), 1e-30) + 1e-7
    err = np.abs(got - want)
    assert err.max() <= tol, f"{what}: max err {err.max():.3e} > {tol:.3e}"
    return err.max()


@pytest.mark.parametrize("dt", ["bf16", "f32"])
def test_route_backward_matches_oracle(dt):
    from top_document_sparse_b200 import msa
    w = small_workload(dtype=dt, n_docs=0, doc_len=0, lognormal=(150, 1.0, 5, 600, 6000), batch=3,
                       query_tokens=5, top_k=4, head_dim=64 if dt == "f32" else 128,
                       planted_per_query=2)
    inp = memory_inputs(w, seed=80)
    mem = msa.Memory(inp["off"], w.chunk_len, w.n_kv_heads, w.head_dim, w.n_router_heads,
                     w.router_dim, inputs.torch_dtype(dt), w.rope_theta, 64)
    rk, ct = mem.new_router_keys(), mem.new_content()
    rmean = torch.empty_like(rk)
    mem.encode(0, mem.n_docs, inp["K"].cuda(), inp["V"].cuda(), inp["Kr"].cuda(), rk, ct, rmean)
    rng = np.random.default_rng(1)
    G = rng.standard_normal((w.batch, mem.n_docs)).astype(np.float32)
    G[rng.random(G.shape) < 0.3] = 0.0
    Qr = inp["Qr"].cuda()
    dQ, dM = mem.route_backward(rmean, Qr, torch.from_numpy(G).cuda())
    torch.cuda.synchronize()
    rQ, rM = oracle.route_backward(inp["Qr"], rmean, mem.doc_chunk_offsets, G)
    _close(dQ, rQ, "d_Qr")
    _close(dM, rM, "d_router_mean")
    assert msa.device_error() == 0


@pytest.mark.parametrize("dt,D,H_q,H_kv,T0,T1,k", [("bf16", 128, 8, 2, 20, 6, 3),
                                                  ("bf16", 128, 32, 8, 9, 1, 4),
                                                  ("f32", 64, 4, 4, 5, 3, 2),
                                                  ("bf16", 64, 8, 4, 7, 2, 0)])
def test_attend_backward_matches_oracle(dt, D, H_q, H_kv, T0, T1, k):
    from top_document_sparse_b200 import msa
    w = small_workload(dtype=dt, head_dim=D, n_q_heads=H_q, n_kv_heads=H_kv, n_docs=0, doc_len=0,
                       lognormal=(150, 0.8, 3, 600, 5000), batch=2, query_tokens=T0 + T1,
                       top_k=max(k, 1))
    inp = memory_inputs(w, seed=81 + D + H_q)
    mem = msa.Memory(inp["off"], w.chunk_len, H_kv, D, w.n_router_heads, w.router_dim,
                     inputs.torch_dtype(dt), w.rope_theta, k + T0 + T1 + 8)
    rk, ct = mem.new_router_keys(), mem.new_content()
    mem.encode(0, mem.n_docs, inp["K"].cuda(), inp["V"].cuda(), inp["Kr"].cuda(), rk, ct)
    B = w.batch
    rng = np.random.default_rng(2)
    ids_np = np.stack([rng.choice(mem.n_docs, size=k, replace=False) for _ in range(B)]).astype(np.int32)
    ids = torch.from_numpy(ids_np).cuda() if k else torch.zeros(B, 0, dtype=torch.int32, device="cuda")
    cap = T0 + T1 + 2
    dtt = inputs.torch_dtype(dt)
    Kc = torch.zeros(B, cap, H_kv, D, dtype=dtt, device="cuda")
    Vc = torch.zeros_like(Kc)
    clen = torch.zeros(B, dtype=torch.int32, device="cuda")
    Q, Kn, Vn = inp["Q"].cuda(), inp["Kn"].cuda(), inp["Vn"].cuda()
    for a, b_ in ((0, T0), (T0, T0 + T1)):  # a prefill call, then the call to differentiate
        O = torch.empty(B, b_ - a, H_q, D, dtype=dtt, device="cuda")
        mem.sparse_attend(ct, ids, Q[:, a:b_].contiguous(), Kn[:, a:b_].contiguous(),
                          Vn[:, a:b_].contiguous(), Kc, Vc, clen, k, O,
                          msa.workspace(mem.attend_workspace_size(B, b_ - a, k, H_q)))
        if a == 0:
            len0 = clen.clone()
    dO = torch.randn(B, T1, H_q, D, generator=torch.Generator(device="cuda").manual_seed(3),
                     device="cuda").to(dtt)
    dQ, dKc, dVc, dC = mem.sparse_attend_backward(ct, ids, Q[:, T0:].contiguous(), Kc, Vc, len0,
                                                  k, dO)
    torch.cuda.synchronize()
    # the oracle on the GPU's stored rows: the cache keys rotated back to before their RoPE
    L = T0 + T1
    pos = k + np.arange(L)
    Kst = to64(Kc[:, :L])
    Kpre = np.stack([oracle.rope_rows(Kst[b], -pos, w.rope_theta) for b in range(B)])
    Kb, Vb = to64(ct[:, 0]), to64(ct[:, 1])
    rQ, rK, rV, rKb, rVb = oracle.attend_backward(to64(Q[:, T0:]), Kpre, to64(Vc[:, :L]), T0, Kb,
                                                  Vb, mem.doc_chunk_offsets, ids_np, k,
                                                  w.rope_theta, to64(dO))
    rK_stored = np.stack([oracle.rope_rows(rK[b], pos, w.rope_theta) for b in range(B)])
    _close(dQ, rQ, "dQ")
    _close(dKc[:, :L], rK_stored, "d cache keys")
    _close(dVc[:, :L], rV, "d cache values")
    assert torch.all(dKc[:, L:] == 0) and torch.all(dVc[:, L:] == 0)
    _close(dC[:, 0], rKb, "d memory keys")
    _close(dC[:, 1], rVb, "d memory values")
    assert msa.device_error() == 0
