"""GPU parity: the CUDA path through the C ABI against the fp64 oracle on the same seeded inputs.

Tolerances (floating point): pooled means within 1e-6 x (mean |x| over the chunk) in fp32, plus
one bf16 ulp when stored in bf16; routing scores 1e-5 (fp32) / 2e-3 (bf16) absolute; attention
outputs 1e-5 (fp32) / 1e-2 (bf16) max-abs, the bf16 bound taken before the output's own rounding
to bf16 (so + half a bf16 ulp of the expected value).  Top-k ids are compared exactly (as sets when the
oracle's k-th / (k+1)-th gap is wider than twice the score tolerance, else checked for validity).
"""
import numpy as np
import pytest
import torch

import oracle
from top_document_sparse_b200 import inputs
from top_document_sparse_b200.workloads import WORKLOADS

from helpers import (assert_close, bf16_ulp, chunk_abs_mean, memory_inputs, rope_scale,
                     small_workload, to64)

pytestmark = pytest.mark.gpu

SCORE_TOL = {"f32": 1e-5, "bf16": 2e-3}
ATTN_TOL = {"f32": 1e-5, "bf16": 1e-2}


def attn_tol(dt, want):
    """The attention bound applies before the output is stored: a bf16 output adds up to half a
    bf16 ulp of its own rounding (0.0078 at |O| ~ 2.6, where short local contexts put it)."""
    if dt == "f32":
        return ATTN_TOL["f32"]
    return ATTN_TOL["bf16"] + 0.5 * bf16_ulp(to64(want))


def _msa():
    from top_document_sparse_b200 import msa
    return msa


def _workload(case):
    if case in WORKLOADS:
        return WORKLOADS[case]
    if case == "ragged_bf16":
        return small_workload(n_docs=0, doc_len=0, lognormal=(100, 1.0, 1, 700, 20000), batch=5,
                              query_tokens=40, top_k=6, planted_per_query=3)
    if case == "ragged_f32":
        return small_workload(dtype="f32", n_docs=0, doc_len=0, head_dim=64,
                              lognormal=(80, 1.0, 1, 400, 6000), batch=3, query_tokens=9,
                              top_k=5, planted_per_query=2)
    raise KeyError(case)


def _build(w, inp, max_local=4096):
    msa = _msa()
    dt = inputs.torch_dtype(w.dtype)
    mem = msa.Memory(inp["off"], w.chunk_len, w.n_kv_heads, w.head_dim, w.n_router_heads,
                     w.router_dim, dt, w.rope_theta, max_local)
    return mem


def _encode(mem, inp, blocks=1):
    K, V, Kr = (inp[n].cuda() for n in ("K", "V", "Kr"))
    rk = mem.new_router_keys()
    ct = mem.new_content()
    rmean = torch.empty_like(rk)
    edges = np.linspace(0, mem.n_docs, blocks + 1).astype(int)
    off = inp["off"]
    for a, b in zip(edges[:-1], edges[1:]):
        if b <= a:
            continue
        t0, t1 = int(off[a]), int(off[b])
        mem.encode(int(a), int(b - a), K[t0:t1], V[t0:t1], Kr[t0:t1], rk, ct, rmean)
    torch.cuda.synchronize()
    return rk, ct, rmean


def _check_pool(w, inp, ct, rk, rmean, oracle_out):
    Kb, Vb, Krb = oracle_out
    off, L = inp["off"], w.chunk_len
    bf16 = w.dtype == "bf16"
    sK = rope_scale(to64(inp["K"]), off, L)
    sV = chunk_abs_mean(to64(inp["V"]), off, L)
    sR = chunk_abs_mean(to64(inp["Kr"]), off, L)
    tK = 1e-6 * sK + (bf16_ulp(Kb) if bf16 else 0)
    tV = 1e-6 * sV + (bf16_ulp(Vb) if bf16 else 0)
    tR = 1e-6 * sR + (bf16_ulp(Krb) if bf16 else 0)
    assert_close(ct[:, 0], Kb, tK, "pooled K (document-wise RoPE)")
    assert_close(ct[:, 1], Vb, tV, "pooled V")
    assert_close(rmean, Krb, tR, "pooled router keys")
    nrm = np.linalg.norm(Krb, axis=-1, keepdims=True)
    unit = Krb / np.maximum(nrm, 1e-12)
    d_r = Krb.shape[-1]
    tU = (np.sqrt(d_r) + 1) * 1e-6 * sR.max(axis=-1, keepdims=True) / np.maximum(nrm, 1e-12) \
        + 4 * 2.0 ** -24 + (bf16_ulp(unit) if bf16 else 0)
    assert_close(rk, unit, tU, "unit router keys")


@pytest.mark.parametrize("case,blocks", [("tiny_f32", 1), ("mem16k_bf16", 1), ("ragged_bf16", 3),
                                         ("ragged_f32", 2)])
def test_encode_matches_oracle(case, blocks):
    w = _workload(case)
    inp = memory_inputs(w, seed=100)
    mem = _build(w, inp)
    rk, ct, rmean = _encode(mem, inp, blocks)
    ref = oracle.encode(inp["K"], inp["V"], inp["Kr"], inp["off"], w.chunk_len, w.rope_theta)
    _check_pool(w, inp, ct, rk, rmean, ref)
    assert mem.doc_chunk_offsets.tolist() == oracle.doc_chunks(inp["off"], w.chunk_len).tolist()


@pytest.mark.parametrize("case", ["ragged_bf16", "tiny_f32"])
def test_document_encoded_alone_is_byte_identical(case):
    w = _workload(case)
    inp = memory_inputs(w, seed=101)
    mem = _build(w, inp)
    rk, ct, rmean = _encode(mem, inp)
    off, cho = inp["off"], mem.doc_chunk_offsets
    for d in (0, mem.n_docs // 2, mem.n_docs - 1):
        t0, t1 = int(off[d]), int(off[d + 1])
        sub = dict(off=np.array([0, t1 - t0]), K=inp["K"][t0:t1], V=inp["V"][t0:t1],
                   Kr=inp["Kr"][t0:t1])
        m1 = _build(w, sub)
        rk1, ct1, rm1 = _encode(m1, sub)
        assert torch.equal(ct1, ct[cho[d]:cho[d + 1]])
        assert torch.equal(rk1, rk[cho[d]:cho[d + 1]])
        assert torch.equal(rm1, rmean[cho[d]:cho[d + 1]])


@pytest.mark.parametrize("case", ["ragged_bf16", "tiny_f32"])
def test_incremental_update_of_one_document_equals_full_encode(case):
    """Replacing one document's tokens and re-encoding only that document gives exactly the rows
    a full encode of the updated memory gives, and leaves every other document's rows untouched:
    document-wise RoPE makes a document's pooled rows depend on its own tokens alone."""
    w = _workload(case)
    inp = memory_inputs(w, seed=102)
    mem = _build(w, inp)
    rk, ct, rmean = _encode(mem, inp)
    off, cho = inp["off"], mem.doc_chunk_offsets
    d = mem.n_docs // 3
    t0, t1 = int(off[d]), int(off[d + 1])
    gen = torch.Generator().manual_seed(7)
    new = {}
    for n in ("K", "V", "Kr"):
        x = inp[n].clone()
        x[t0:t1] = torch.randn(x[t0:t1].shape, generator=gen).to(x.dtype)
        new[n] = x
    before = (rk.clone(), ct.clone(), rmean.clone())
    mem.encode(d, 1, new["K"][t0:t1].cuda(), new["V"][t0:t1].cuda(), new["Kr"][t0:t1].cuda(), rk,
               ct, rmean)
    torch.cuda.synchronize()
    full = _encode(mem, dict(inp, **new))
    keep = torch.ones(rk.shape[0], dtype=torch.bool, device="cuda")
    keep[int(cho[d]):int(cho[d + 1])] = False
    for got, ref, old in zip((rk, ct, rmean), full, before):
        assert torch.equal(got, ref)
        assert torch.equal(got[keep], old[keep])
        assert not torch.equal(got[~keep], old[~keep])
    # the re-encoded rows against the oracle's encoding of the new tokens, at the pooling bound
    sub = dict(off=np.array([0, t1 - t0]), K=new["K"][t0:t1], V=new["V"][t0:t1],
               Kr=new["Kr"][t0:t1])
    ref = oracle.encode(sub["K"], sub["V"], sub["Kr"], sub["off"], w.chunk_len, w.rope_theta)
    c0, c1 = int(cho[d]), int(cho[d + 1])
    _check_pool(w, sub, ct[c0:c1], rk[c0:c1], rmean[c0:c1], ref)


def _check_topk(ids, scores, state, ref_state, k, tol, eligible=None):
    """ids/scores from the GPU; ref_state from the oracle (fp64)."""
    ids, scores, state = ids.cpu().numpy(), scores.cpu().numpy(), state.cpu().numpy()
    B = ids.shape[0]
    for b in range(B):
        ref = ref_state[b].copy()
        if eligible is not None:
            ref[~eligible[b]] = -np.inf
        order = np.lexsort((np.arange(ref.size), -ref))
        kth = ref[order[k - 1]]
        nxt = ref[order[k]] if ref.size > k else -np.inf
        # the GPU's own order is (score desc, id asc) over its own state
        assert np.all(scores[b] == state[b, ids[b]])
        pairs = list(zip(-scores[b], ids[b]))
        assert pairs == sorted(pairs)
        assert len(set(ids[b].tolist())) == k
        if kth - nxt > 2 * tol:
            assert set(ids[b].tolist()) == set(order[:k].tolist()), f"query {b}"
        else:  # several top-k sets are correct: check validity against the oracle
            assert all(ref[d] >= kth - tol for d in ids[b])
            assert all(d in ids[b] for d in np.nonzero(ref > kth + tol)[0])


@pytest.mark.parametrize("case", ["tiny_f32", "mem16k_bf16", "ragged_bf16", "ragged_f32"])
def test_route_matches_oracle(case):
    msa = _msa()
    w = _workload(case)
    inp = memory_inputs(w, seed=102)
    mem = _build(w, inp)
    rk, ct, _ = _encode(mem, inp)
    B, T, k = w.batch, w.query_tokens, w.top_k
    Qr = inp["Qr"].cuda()
    state = torch.full((B, mem.n_docs), float("-inf"), device="cuda")
    ids = torch.zeros(B, k, dtype=torch.int32, device="cuda")
    scores = torch.zeros(B, k, device="cuda")
    ws = msa.workspace(mem.route_workspace_size(B, T, k))
    mem.route(rk, Qr, k, state, ids, scores, ws)
    torch.cuda.synchronize()
    _, _, Krb = oracle.encode(inp["K"], inp["V"], inp["Kr"], inp["off"], w.chunk_len,
                              w.rope_theta)
    ref = oracle.route(inp["Qr"], Krb, mem.doc_chunk_offsets)
    tol = SCORE_TOL[w.dtype]
    err = assert_close(state, ref, tol, "document scores")
    assert np.all(np.abs(to64(state)) <= 1.0 + tol)
    _check_topk(ids, scores, state, ref, k, tol)
    # every planted document is retrieved by its query
    pb, pd, _, _ = inp["plants"]
    got = ids.cpu().numpy()
    for b, d in zip(pb, pd):
        assert d in got[b]
    assert msa.device_error() == 0
    print(f"{case}: max |score err| = {err:.2e}")


@pytest.mark.parametrize("n_docs,k,excl", [(1, 1, False), (7, 3, True), (4096, 16, False),
                                           (4097, 64, True), (20000, 16, True), (30011, 1, False)])
def test_topk_is_exact_on_identical_scores(n_docs, k, excl):
    msa = _msa()
    B = 3
    rng = np.random.default_rng(n_docs + k)
    st = (rng.integers(-50, 50, size=(B, n_docs)) / 64.0).astype(np.float32)  # many exact ties
    ex = (rng.random((B, n_docs)) < 0.3) if excl else np.zeros((B, n_docs), dtype=bool)
    ex[:, :k] = False  # keep at least k eligible documents
    off = np.arange(n_docs + 1, dtype=np.int64) * 2
    mem = msa.Memory(off, 2, 1, 64, 1, 64, torch.bfloat16, 1e4, 16)
    state = torch.from_numpy(st).cuda()
    ids = torch.zeros(B, k, dtype=torch.int32, device="cuda")
    scores = torch.zeros(B, k, device="cuda")
    exclude = torch.from_numpy(ex.astype(np.uint8)).cuda() if excl else None
    ws = msa.workspace(mem.route_workspace_size(B, 0, k))
    mem.route(None, None, k, state, ids, scores, ws, exclude=exclude)
    ref = np.where(ex, -np.inf, st.astype(np.float64))
    want_ids, want_sc = oracle.topk(ref, k)
    assert np.array_equal(ids.cpu().numpy(), want_ids)
    assert np.array_equal(scores.cpu().numpy().astype(np.float64), want_sc)
    assert torch.equal(state.cpu(), torch.from_numpy(st))  # top-k alone leaves the state


def test_topk_with_too_few_eligible_documents_pads_with_minus_one():
    msa = _msa()
    off = np.arange(11, dtype=np.int64) * 2
    mem = msa.Memory(off, 2, 1, 64, 1, 64, torch.bfloat16, 1e4, 16)
    state = torch.arange(10, dtype=torch.float32, device="cuda")[None].contiguous()
    ex = torch.ones(1, 10, dtype=torch.uint8, device="cuda")
    ex[0, 3] = 0
    ex[0, 7] = 0
    ids = torch.zeros(1, 4, dtype=torch.int32, device="cuda")
    scores = torch.zeros(1, 4, device="cuda")
    mem.route(None, None, 4, state, ids, scores, msa.workspace(mem.route_workspace_size(1, 0, 4)),
              exclude=ex)
    assert ids.cpu().tolist() == [[7, 3, -1, -1]]
    assert scores.cpu()[0, :2].tolist() == [7.0, 3.0]
    assert torch.isinf(scores.cpu()[0, 2:]).all()


ATTN_CASES = [
    # dtype, head_dim, H_q, H_kv, prefill tokens, then tokens, k
    ("f32", 64, 8, 2, 32, 1, 4),
    ("f32", 128, 4, 4, 5, 3, 2),
    ("bf16", 128, 32, 8, 24, 1, 6),
    ("bf16", 128, 32, 8, 40, 17, 4),
    ("bf16", 64, 16, 16, 7, 1, 3),
    ("bf16", 128, 16, 1, 9, 2, 5),
    ("bf16", 64, 8, 4, 33, 1, 0),
    # tensor-core prefill (head_dim 128, 128-row tiles in pairs): GQA group 1 (70 tokens, one
    # partial tile), 2 (150 tokens: three 64-token tiles, the second pair's second tile empty,
    # local blocks two whole and one ragged), 8 (33 tokens: three 16-token tiles); each then a
    # second multi-token call over the filled cache
    ("bf16", 128, 8, 8, 70, 5, 3),
    ("bf16", 128, 16, 8, 150, 3, 4),
    ("bf16", 128, 64, 8, 33, 31, 2),
    # one-token decode kernel (head_dim 128, GQA group 2..16), with and without memory rows
    ("bf16", 128, 16, 8, 20, 1, 3),
    ("bf16", 128, 64, 8, 11, 1, 2),
    ("bf16", 128, 32, 2, 5, 1, 4),
    ("bf16", 128, 32, 8, 40, 1, 0),
]


@pytest.mark.parametrize("dt,D,H_q,H_kv,T0,T1,k", ATTN_CASES)
def test_attend_matches_oracle(dt, D, H_q, H_kv, T0, T1, k):
    _attend_calls_match_oracle(dt, D, H_q, H_kv, (T0, T1), k, batch=3)


def test_one_split_decode_in_clusters_matches_oracle():
    """A batch with B * H_kv >= 3 CTAs per SM: each one-token call runs with one context split,
    as clusters of a query's kv-head CTAs that advance cache_len themselves."""
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    B, H_kv = 64, 8
    assert B * H_kv >= 3 * sms, "batch too small to take the one-split path on this device"
    _attend_calls_match_oracle("bf16", 128, 32, H_kv, (6, 1, 1, 1), 3, batch=B)


def _attend_calls_match_oracle(dt, D, H_q, H_kv, Ts, k, batch):
    msa = _msa()
    w = small_workload(dtype=dt, head_dim=D, n_q_heads=H_q, n_kv_heads=H_kv, n_docs=0, doc_len=0,
                       lognormal=(150, 0.8, 3, 600, 5000), batch=batch, query_tokens=sum(Ts),
                       top_k=max(k, 1))
    inp = memory_inputs(w, seed=103 + D + H_q)
    mem = _build(w, inp, max_local=k + sum(Ts) + 8)
    rk, ct, _ = _encode(mem, inp)
    Kb, Vb, _ = oracle.encode(inp["K"], inp["V"], inp["Kr"], inp["off"], w.chunk_len, w.rope_theta)
    B = w.batch
    rng = np.random.default_rng(7)
    ids_np = np.stack([rng.choice(mem.n_docs, size=k, replace=False) for _ in range(B)]).astype(np.int32)
    ids = torch.from_numpy(ids_np).cuda() if k else torch.zeros(B, 0, dtype=torch.int32, device="cuda")
    cap = sum(Ts) + 3
    dtt = inputs.torch_dtype(dt)
    Kc = torch.zeros(B, cap, H_kv, D, dtype=dtt, device="cuda")
    Vc = torch.zeros_like(Kc)
    clen = torch.zeros(B, dtype=torch.int32, device="cuda")
    Q, Kn, Vn = inp["Q"], inp["Kn"], inp["Vn"]
    pos_offset = k
    tol = ATTN_TOL[dt]
    start = 0
    for T in Ts:
        sl = slice(start, start + T)
        O = torch.empty(B, T, H_q, D, dtype=dtt, device="cuda")
        ws = msa.workspace(mem.attend_workspace_size(B, T, k, H_q))
        mem.sparse_attend(ct, ids, Q[:, sl].cuda().contiguous(), Kn[:, sl].cuda().contiguous(),
                          Vn[:, sl].cuda().contiguous(), Kc, Vc, clen, pos_offset, O, ws)
        torch.cuda.synchronize()
        ref, _, rs = oracle.attend(Q[:, sl], Kn[:, :start + T], Vn[:, :start + T], start, Kb, Vb,
                                   mem.doc_chunk_offsets, ids_np, pos_offset, w.rope_theta)
        np.testing.assert_allclose(rs, 1.0, atol=1e-12)
        assert_close(O, ref, attn_tol(dt, ref), f"attention output (tokens {start}..{start + T})")
        start += T
        assert clen.cpu().tolist() == [start] * B
    assert msa.device_error() == 0


def test_decode_steps_match_oracle():
    """16K-token workload at its stated configuration (8 planted documents per query, k = 16, a
    128-token query, then all 64 decode steps at batch 1) through msa_step, stage by stage: at
    every step the running state is the oracle's route of the new token over the oracle's own
    running state; the retrieved set is checked by the validity rule for near-ties at rank k
    (only 8 documents are planted, so ranks 9..16 are background documents whose scores may be
    within the tolerance of each other); the step's attention output is the oracle's attention
    over the documents the GPU retrieved."""
    msa = _msa()
    w = WORKLOADS["mem16k_bf16"]
    assert (w.planted_per_query, w.top_k, w.decode_steps, w.batch) == (8, 16, 64, 1)
    n_steps = w.decode_steps
    inp = memory_inputs(w, seed=104)
    mem = _build(w, inp, max_local=w.top_k + w.query_tokens + n_steps + 4)
    rk, ct, _ = _encode(mem, inp)
    Kb, Vb, Krb = oracle.encode(inp["K"], inp["V"], inp["Kr"], inp["off"], w.chunk_len,
                                w.rope_theta)
    B, T, k, H_q = w.batch, w.query_tokens, w.top_k, w.n_q_heads
    cho = mem.doc_chunk_offsets
    cap = T + n_steps + 2
    layer = msa.LayerDecode(mem, B, k, H_q, cap)
    # prefill: route the whole query block, attend it
    ws = msa.workspace(mem.route_workspace_size(B, T, k))
    mem.route(rk, inp["Qr"].cuda(), k, layer.state, layer.ids, layer.scores, ws)
    O = torch.empty(B, T, H_q, w.head_dim, dtype=torch.bfloat16, device="cuda")
    mem.sparse_attend(ct, layer.ids, inp["Q"].cuda(), inp["Kn"].cuda(), inp["Vn"].cuda(),
                      layer.k_cache, layer.v_cache, layer.cache_len, k, O,
                      msa.workspace(mem.attend_workspace_size(B, T, k, H_q)))
    torch.cuda.synchronize()
    st = oracle.route(inp["Qr"], Krb, cho)
    _check_topk(layer.ids, layer.scores, layer.state, st, k, SCORE_TOL["bf16"])
    pb, pd, _, _ = inp["plants"]
    ref, _, _ = oracle.attend(inp["Q"], inp["Kn"], inp["Vn"], 0, Kb, Vb, cho,
                              layer.ids.cpu().numpy(), k, w.rope_theta)
    assert_close(O, ref, attn_tol("bf16", ref), "prefill attention output")
    dec = inputs.queries(w, B, n_steps, seed=777)
    Khist = torch.cat([inp["Kn"], dec[2]], dim=1)
    Vhist = torch.cat([inp["Vn"], dec[3]], dim=1)
    near_ties = 0
    for s in range(n_steps):
        Ot = torch.empty(B, H_q, w.head_dim, dtype=torch.bfloat16, device="cuda")
        mem.step(rk, ct, layer, dec[0][:, s].cuda().contiguous(), dec[1][:, s].cuda().contiguous(),
                 dec[2][:, s].cuda().contiguous(), dec[3][:, s].cuda().contiguous(), Ot)
        torch.cuda.synchronize()
        st = oracle.route(dec[0][:, s:s + 1], Krb, cho, st)
        assert_close(layer.state, st, SCORE_TOL["bf16"], f"running state, step {s}")
        _check_topk(layer.ids, layer.scores, layer.state, st, k, SCORE_TOL["bf16"])
        ids_gpu = layer.ids.cpu().numpy()
        ids_o, _ = oracle.topk(st, k)
        near_ties += int(set(ids_gpu[0].tolist()) != set(ids_o[0].tolist()))
        for b, d in zip(pb, pd):  # the planted documents stay retrieved
            assert d in ids_gpu[b], f"planted document {d} lost at step {s}"
        O_ref, _, rs = oracle.attend(dec[1][:, s:s + 1], Khist, Vhist, T + s, Kb, Vb, cho, ids_gpu,
                                     k, w.rope_theta)
        np.testing.assert_allclose(rs, 1.0, atol=1e-12)
        assert_close(Ot, O_ref[:, 0], attn_tol("bf16", O_ref[:, 0]), f"decode output, step {s}")
    assert layer.cache_len.cpu().tolist() == [T + n_steps]
    assert msa.device_error() == 0
    print(f"64 decode steps: {near_ties} steps with a different (valid) set at rank k")


def test_device_bounds_checks_raise_the_error_word():
    msa = _msa()
    w = small_workload(batch=2, query_tokens=2)
    inp = memory_inputs(w, seed=105)
    mem = _build(w, inp, max_local=64)
    rk, ct, _ = _encode(mem, inp)
    assert msa.device_error() == 0
    B, H_q, D = 2, w.n_q_heads, w.head_dim
    ids = torch.tensor([[0, 99], [1, 2]], dtype=torch.int32, device="cuda")  # 99 >= n_docs
    Kc = torch.zeros(B, 4, w.n_kv_heads, D, dtype=torch.bfloat16, device="cuda")
    Vc = torch.zeros_like(Kc)
    clen = torch.tensor([0, 3], dtype=torch.int32, device="cuda")  # query 1 overflows with T=2
    Q = inp["Q"][:, :2].cuda().contiguous()
    O = torch.empty(B, 2, H_q, D, dtype=torch.bfloat16, device="cuda")
    mem.sparse_attend(ct, ids, Q, inp["Kn"][:, :2].cuda().contiguous(),
                      inp["Vn"][:, :2].cuda().contiguous(), Kc, Vc, clen, 2, O,
                      msa.workspace(mem.attend_workspace_size(B, 2, 2, H_q)))
    bits = msa.device_error()
    assert bits & msa.DEVERR_BAD_DOC_ID and bits & msa.DEVERR_CACHE_OVERFLOW
    assert msa.device_error() == 0  # cleared by the read


def test_host_validation_rejects_bad_calls_on_a_gpu():
    msa = _msa()
    w = small_workload()
    inp = memory_inputs(w, seed=106)
    mem = _build(w, inp, max_local=64)
    rk, ct, _ = _encode(mem, inp)
    state = torch.full((2, mem.n_docs), float("-inf"), device="cuda")
    ids = torch.zeros(2, 4, dtype=torch.int32, device="cuda")
    sc = torch.zeros(2, 4, device="cuda")
    ws = msa.workspace(mem.route_workspace_size(2, 16, 4))
    with pytest.raises(msa.MsaError) as e:
        mem.route(rk, inp["Qr"].cuda(), mem.n_docs + 1, state, ids, sc, ws)
    assert e.value.status == 1
    with pytest.raises(msa.MsaError):
        mem.route(rk, inp["Qr"].cuda(), 4, state, ids, sc, ws[:16])  # workspace too small
    with pytest.raises(msa.MsaError):
        mem.route(rk, inp["Qr"].cuda(), 0, state, ids, sc, ws)  # k = 0
    Q = inp["Q"][:, :1].cuda().contiguous()
    Kc = torch.zeros(2, 8, w.n_kv_heads, w.head_dim, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(msa.MsaError):  # pos_offset + capacity beyond the RoPE table
        mem.sparse_attend(ct, ids, Q, Q[:, :, :w.n_kv_heads].contiguous(),
                          Q[:, :, :w.n_kv_heads].contiguous(), Kc, Kc.clone(),
                          torch.zeros(2, dtype=torch.int32, device="cuda"), 60, torch.empty_like(Q),
                          msa.workspace(1 << 20))
    assert msa.device_error() == 0
