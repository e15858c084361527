"""msa_sparse_attend_static: the attention entry point for callers that cannot allocate device
memory (for example a plugin inside a host engine that reserved the whole device budget up front).
It takes no workspace; its scratch is a fixed 4 MiB array inside the library.  This file runs last
(pytest collects it after the others) and must pass both alone in a fresh process and after the
rest of the suite: two calls in a row must give the same outputs and the same local cache as the
workspace entry point on the same inputs."""
import numpy as np
import pytest
import torch

from helpers import assert_close, memory_inputs, small_workload

pytestmark = pytest.mark.gpu


def test_static_scratch_attention_matches_workspace_entry_point():
    from top_document_sparse_b200 import msa
    w = small_workload(n_q_heads=32, n_kv_heads=8, head_dim=128, batch=3, query_tokens=8,
                       top_k=4, n_docs=12, doc_len=448)
    inp = memory_inputs(w, seed=910)
    B, k, H_q, D, cap = w.batch, w.top_k, w.n_q_heads, w.head_dim, 128
    mem = msa.Memory(inp["off"], w.chunk_len, w.n_kv_heads, w.head_dim, w.n_router_heads,
                     w.router_dim, torch.bfloat16, w.rope_theta, k + cap)
    rk, ct = mem.new_router_keys(), mem.new_content()
    mem.encode(0, mem.n_docs, inp["K"].cuda(), inp["V"].cuda(), inp["Kr"].cuda(), rk, ct)
    rng = np.random.default_rng(3)
    ids = torch.from_numpy(np.stack([rng.choice(mem.n_docs, k, replace=False)
                                     for _ in range(B)]).astype(np.int32)).cuda()
    # decode calls use the split context, so the scratch is really used
    assert mem.attend_workspace_size(B, 1, k, H_q) > 0

    def cache():
        Kc = torch.zeros(B, cap, w.n_kv_heads, D, dtype=torch.bfloat16, device="cuda")
        return Kc, torch.zeros_like(Kc), torch.zeros(B, dtype=torch.int32, device="cuda")

    Ka, Va, la = cache()
    Kb, Vb, lb = cache()
    ws = msa.workspace(mem.attend_workspace_size(B, 1, k, H_q))
    for t in range(2):  # two calls in a row on each path
        Q = inp["Q"][:, t:t + 1].cuda().contiguous()
        Kn = inp["Kn"][:, t:t + 1].cuda().contiguous()
        Vn = inp["Vn"][:, t:t + 1].cuda().contiguous()
        Oa = torch.empty(B, 1, H_q, D, dtype=torch.bfloat16, device="cuda")
        Ob = torch.empty_like(Oa)
        mem.sparse_attend(ct, ids, Q, Kn, Vn, Ka, Va, la, k, Oa, ws)
        mem.sparse_attend_static(ct, ids, Q, Kn, Vn, Kb, Vb, lb, k, Ob)
        torch.cuda.synchronize()
        assert_close(Ob, Oa, 1e-2, f"static-scratch attention, call {t}")
        assert torch.equal(Kb, Ka) and torch.equal(Vb, Va) and torch.equal(lb, la)
    assert lb.cpu().tolist() == [2] * B
    assert msa.device_error() == 0


def test_static_scratch_rejects_calls_beyond_its_size():
    """A call whose split-context scratch would exceed the 4 MiB array is refused on the host
    and enqueues nothing (every buffer below is sized for the call all the same).  The split
    count aims at about three CTAs per SM, so the largest scratch comes from a call with just
    fewer (query, token, kv head) CTAs than that and 16 query heads per kv head."""
    from top_document_sparse_b200 import msa
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    B, k, H_kv, D, cap = 4, 4, 1, 128, 512
    H_q = 16 * H_kv
    T = (3 * sms - 1) // (B * H_kv)            # B * T * H_kv just under 3 CTAs per SM: 2 splits
    w = small_workload(n_q_heads=H_q, n_kv_heads=H_kv, head_dim=D, batch=B, top_k=k,
                       n_docs=12, doc_len=448)
    inp = memory_inputs(w, seed=911)
    mem = msa.Memory(inp["off"], w.chunk_len, H_kv, D, w.n_router_heads, w.router_dim,
                     torch.bfloat16, w.rope_theta, k + cap)
    need = mem.attend_workspace_size(B, T, k, H_q)
    assert need > (4 << 20)
    ct = torch.zeros(mem.n_chunks, 2, H_kv, D, dtype=torch.bfloat16, device="cuda")
    Q = torch.zeros(B, T, H_q, D, dtype=torch.bfloat16, device="cuda")
    Kn = torch.zeros(B, T, H_kv, D, dtype=torch.bfloat16, device="cuda")
    Kc = torch.zeros(B, cap, H_kv, D, dtype=torch.bfloat16, device="cuda")
    Vc = torch.zeros_like(Kc)
    O = torch.full((B, T, H_q, D), 7.0, dtype=torch.bfloat16, device="cuda")
    ids = torch.zeros(B, k, dtype=torch.int32, device="cuda")
    ids[:, 1:] = torch.arange(1, k, dtype=torch.int32)
    lens = torch.zeros(B, dtype=torch.int32, device="cuda")
    with pytest.raises(msa.MsaError) as e:
        mem.sparse_attend_static(ct, ids, Q, Kn, Kn.clone(), Kc, Vc, lens, k, O)
    assert e.value.status == 2 and "static scratch" in str(e.value)
    torch.cuda.synchronize()
    assert lens.cpu().tolist() == [0] * B and bool((O == 7.0).all())
    assert msa.device_error() == 0


def test_static_scratch_reports_bad_shapes_before_sizing_its_scratch():
    """The shape checks of every attention call run before the static scratch is sized: a query
    head count that is not a multiple of the kv heads is an invalid argument (not a scratch size
    refusal) even when the call's split-context scratch would not fit the array, and nothing is
    enqueued."""
    from top_document_sparse_b200 import msa
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    B, k, H_kv, D, cap = 4, 4, 2, 128, 512
    T = (3 * sms - 1) // (B * H_kv)
    w = small_workload(n_q_heads=32, n_kv_heads=H_kv, head_dim=D, batch=B, top_k=k,
                       n_docs=12, doc_len=448)
    inp = memory_inputs(w, seed=912)
    mem = msa.Memory(inp["off"], w.chunk_len, H_kv, D, w.n_router_heads, w.router_dim,
                     torch.bfloat16, w.rope_theta, k + cap)
    assert mem.attend_workspace_size(B, T, k, 32) > (4 << 20)
    ct = torch.zeros(mem.n_chunks, 2, H_kv, D, dtype=torch.bfloat16, device="cuda")
    Kn = torch.zeros(B, T, H_kv, D, dtype=torch.bfloat16, device="cuda")
    Kc = torch.zeros(B, cap, H_kv, D, dtype=torch.bfloat16, device="cuda")
    ids = torch.zeros(B, k, dtype=torch.int32, device="cuda")
    lens = torch.zeros(B, dtype=torch.int32, device="cuda")
    Q = torch.zeros(B, T, 33, D, dtype=torch.bfloat16, device="cuda")
    O = torch.full_like(Q, 7.0)
    for H_q in (33, 0):  # 33 query heads over 2 kv heads; no query head
        st = msa.lib().msa_sparse_attend_static(
            mem.handle, ct.data_ptr(), ids.data_ptr(), B, k, T, H_q, Q.data_ptr(), Kn.data_ptr(),
            Kn.data_ptr(), Kc.data_ptr(), Kc.data_ptr(), lens.data_ptr(), cap, k, O.data_ptr(),
            torch.cuda.current_stream().cuda_stream)
        assert st == 1, msa.lib().msa_last_error()
        assert b"multiple of n_kv_heads" in msa.lib().msa_last_error()
    torch.cuda.synchronize()
    assert lens.cpu().tolist() == [0] * B and bool((O == 7.0).all())
    assert msa.device_error() == 0
