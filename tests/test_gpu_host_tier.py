"""Host tier of the pooled content (content in pinned host DRAM, top-k documents fetched into a
device slot cache): the fetched path must give exactly the results of the device-resident path,
and the encoder may write the content straight into pinned host memory."""
import numpy as np
import pytest
import torch

from helpers import memory_inputs, small_workload

pytestmark = pytest.mark.gpu


def _setup(seed, n_docs=40, doc_len=None, lognormal=None, B=3, k=5, T=6):
    from top_document_sparse_b200 import msa
    kw = dict(n_q_heads=32, n_kv_heads=8, head_dim=128, batch=B, query_tokens=T, top_k=k,
              planted_per_query=2)
    if lognormal:
        kw.update(n_docs=0, doc_len=0, lognormal=lognormal)
    else:
        kw.update(n_docs=n_docs, doc_len=doc_len or 320)
    w = small_workload(**kw)
    inp = memory_inputs(w, seed=seed)
    mem = msa.Memory(inp["off"], w.chunk_len, w.n_kv_heads, w.head_dim, w.n_router_heads,
                     w.router_dim, torch.bfloat16, w.rope_theta, 256)
    K, V, Kr = inp["K"].cuda(), inp["V"].cuda(), inp["Kr"].cuda()
    rk = mem.new_router_keys()
    ct_dev = mem.new_content()
    ct_host = mem.new_content(device="cpu", pin_memory=True)
    mem.encode(0, mem.n_docs, K, V, Kr, rk, ct_dev)
    rk2 = mem.new_router_keys()
    mem.encode(0, mem.n_docs, K, V, Kr, rk2, ct_host)  # pooled content written over the host link
    torch.cuda.synchronize()
    return msa, w, inp, mem, rk, ct_dev, ct_host


def test_encode_writes_pinned_host_content_identically():
    msa, w, inp, mem, rk, ct_dev, ct_host = _setup(200, lognormal=(150, 1.0, 5, 700, 9000))
    assert torch.equal(ct_host, ct_dev.cpu())
    assert msa.device_error() == 0


@pytest.mark.parametrize("cold", [False, True])
def test_fetched_attention_equals_device_resident_attention(cold):
    msa, w, inp, mem, rk, ct_dev, ct_host = _setup(201, lognormal=(150, 1.0, 5, 700, 9000))
    B, k, H_q, D = w.batch, w.top_k, w.n_q_heads, w.head_dim
    f = msa.Fetcher(mem, ct_host, n_slots=B * k + 3, max_batch=B, max_k=k, cold=cold)
    rng = np.random.default_rng(0)
    cap = 16
    caches = {}
    for name in ("dev", "host"):
        Kc = torch.zeros(B, cap, w.n_kv_heads, D, dtype=torch.bfloat16, device="cuda")
        caches[name] = (Kc, torch.zeros_like(Kc), torch.zeros(B, dtype=torch.int32, device="cuda"))
    fetch_stream = torch.cuda.Stream()
    prev = None
    distinct = []
    for t in range(3):
        ids_np = np.stack([rng.choice(mem.n_docs, size=k, replace=False) for _ in range(B)])
        if prev is not None:
            ids_np[:, :2] = prev[:, :2]  # some documents stay resident between calls
        prev = ids_np
        distinct.append(len(set(ids_np.ravel().tolist())))
        ids = torch.from_numpy(ids_np.astype(np.int32)).cuda()
        Q = inp["Q"][:, t:t + 1].cuda().contiguous()
        Kn = inp["Kn"][:, t:t + 1].cuda().contiguous()
        Vn = inp["Vn"][:, t:t + 1].cuda().contiguous()
        ws = msa.workspace(mem.attend_workspace_size(B, 1, k, H_q))
        O1 = torch.empty(B, 1, H_q, D, dtype=torch.bfloat16, device="cuda")
        O2 = torch.empty_like(O1)
        mem.sparse_attend(ct_dev, ids, Q, Kn, Vn, *caches["dev"], k, O1, ws)
        f.fetch(ids, fetch_stream=fetch_stream)
        f.sparse_attend(ids, Q, Kn, Vn, *caches["host"], k, O2, ws)
        torch.cuda.synchronize()
        assert torch.equal(O1, O2), f"call {t}"
    st = f.stats()
    assert st["hits"] + st["misses"] == 3 * B * k
    assert st["copies"] == st["misses"] and st["bytes"] > 0
    if cold:  # every call copies each of its distinct documents once
        assert st["misses"] == sum(distinct)
    else:     # documents carried from the previous call stay resident
        assert st["misses"] <= sum(distinct) - 2 * 2
    assert msa.device_error() == 0


def test_host_tier_decode_steps_equal_device_tier():
    msa, w, inp, mem, rk, ct_dev, ct_host = _setup(202, n_docs=48, doc_len=384, B=2, k=4, T=10)
    B, k, H_q, D = w.batch, w.top_k, w.n_q_heads, w.head_dim
    f = msa.Fetcher(mem, ct_host, n_slots=B * k * 2, max_batch=B, max_k=k)
    lay_d = msa.LayerDecode(mem, B, k, H_q, 12)
    lay_h = msa.LayerDecode(mem, B, k, H_q, 12)
    fs = torch.cuda.Stream()
    for t in range(10):
        Qr = inp["Qr"][:, t].cuda().contiguous()
        Q = inp["Q"][:, t].cuda().contiguous()
        Kt = inp["Kn"][:, t].cuda().contiguous()
        Vt = inp["Vn"][:, t].cuda().contiguous()
        Od = torch.empty(B, H_q, D, dtype=torch.bfloat16, device="cuda")
        Oh = torch.empty_like(Od)
        mem.step(rk, ct_dev, lay_d, Qr, Q, Kt, Vt, Od)
        f.step(rk, lay_h, Qr, Q, Kt, Vt, Oh, fetch_stream=fs)
        torch.cuda.synchronize()
        assert torch.equal(lay_d.ids, lay_h.ids) and torch.equal(Od, Oh), f"step {t}"
    s = f.stats()
    assert s["misses"] >= 1 and s["hits"] >= 1  # the running max keeps retrieved documents
    assert msa.device_error() == 0


def test_fetcher_rejects_bad_arguments():
    msa, w, inp, mem, rk, ct_dev, ct_host = _setup(203, n_docs=10, B=2, k=3)
    with pytest.raises(ValueError):
        msa.Fetcher(mem, ct_dev.cpu(), n_slots=8, max_batch=2, max_k=3)   # not pinned
    with pytest.raises(msa.MsaError):
        msa.Fetcher(mem, ct_host, n_slots=5, max_batch=2, max_k=3)        # fewer slots than B*k
    f = msa.Fetcher(mem, ct_host, n_slots=6, max_batch=2, max_k=3)
    with pytest.raises(msa.MsaError):
        f.fetch(torch.zeros(3, 3, dtype=torch.int32, device="cuda"))      # batch beyond max


def test_host_tier_step_captured_in_a_cuda_graph_equals_eager_steps():
    """The fetch reads nothing back to the host (slots are assigned on the device), so a whole
    host-tier decode step -- route, slot assignment, gather over the host link, attention --
    can be captured in a CUDA graph; replayed step by step it gives exactly the eager steps,
    which give exactly the device-resident steps.  Few slots, so documents are evicted."""
    msa, w, inp, mem, rk, ct_dev, ct_host = _setup(204, n_docs=48, doc_len=384, B=2, k=4, T=8)
    B, k, H_q, D = w.batch, w.top_k, w.n_q_heads, w.head_dim
    f_e = msa.Fetcher(mem, ct_host, n_slots=B * k + 1, max_batch=B, max_k=k)
    f_g = msa.Fetcher(mem, ct_host, n_slots=B * k + 1, max_batch=B, max_k=k)
    lay_d, lay_e, lay_g = (msa.LayerDecode(mem, B, k, H_q, 10) for _ in range(3))
    fs = torch.cuda.Stream()
    cur = torch.cuda.Stream()
    tok = [inp[n][:, 0].cuda().contiguous() for n in ("Qr", "Q", "Kn", "Vn")]  # static inputs
    Og = torch.empty(B, H_q, D, dtype=torch.bfloat16, device="cuda")
    with torch.cuda.stream(cur):  # one eager call on this stream first (kernel attributes)
        f_g.step(rk, lay_g, *tok, Og, fetch_stream=fs)
    torch.cuda.synchronize()
    lay_g.state.fill_(float("-inf"))
    lay_g.cache_len.zero_()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=cur):
        f_g.step(rk, lay_g, *tok, Og, fetch_stream=fs)
    for t in range(8):
        x = [inp[n][:, t].cuda().contiguous() for n in ("Qr", "Q", "Kn", "Vn")]
        Od = torch.empty(B, H_q, D, dtype=torch.bfloat16, device="cuda")
        Oe = torch.empty_like(Od)
        mem.step(rk, ct_dev, lay_d, *x, Od)
        f_e.step(rk, lay_e, *x, Oe, fetch_stream=fs)
        for dst, src in zip(tok, x):
            dst.copy_(src)
        torch.cuda.synchronize()
        g.replay()
        torch.cuda.synchronize()
        assert torch.equal(lay_e.ids, lay_d.ids) and torch.equal(Oe, Od), f"eager, step {t}"
        assert torch.equal(lay_g.ids, lay_e.ids) and torch.equal(Og, Oe), f"graph, step {t}"
    assert lay_g.cache_len.cpu().tolist() == [8] * B
    s_e, s_g = f_e.stats(), f_g.stats()
    assert s_e["misses"] >= B * k and s_e["hits"] >= 1
    assert msa.device_error() == 0
    del g
