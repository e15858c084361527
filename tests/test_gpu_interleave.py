"""Memory Interleave on the GPU (msa_interleave) against the oracle's rounds: each round routes the
previous round's retrieved documents' pooled router rows with the state carried over and takes
the top-k among documents not yet in the context; a planted 3-hop chain must surface hop by hop."""
import numpy as np
import pytest
import torch

import oracle
from top_document_sparse_b200 import inputs

from helpers import small_workload, to64

pytestmark = pytest.mark.gpu


def _valid_topk(ids_b, ref_b, k, tol, what):
    """ids_b is a correct top-k of the scores ref_b (-inf = not eligible) up to ties within tol:
    every document scoring clearly above the k-th best is in it, none clearly below."""
    order = np.lexsort((np.arange(ref_b.size), -ref_b))
    kth = ref_b[order[k - 1]]
    assert len(set(ids_b.tolist())) == k, what
    assert all(ref_b[d] >= kth - tol for d in ids_b), what
    assert all(d in ids_b for d in np.nonzero(ref_b > kth + tol)[0]), what


def _replay_rounds(Qr, Krb, cho, got, sc, k, R, stop, tol):
    """The oracle replays adaptive interleave rounds on the GPU's own picks (stage by stage):
    round r routes the rows the GPU's round r-1 retrieved, over the oracle's running state; the
    GPU's ids of round r must be a valid top-k of the oracle's state among documents not yet in
    the context, their scores the oracle's, and the stop decisions the oracle's.  Returns the
    oracle's final state, rounds kept per query and the ids of every kept round."""
    Q = to64(Qr)
    B = Q.shape[0]
    n_docs = cho.size - 1
    state = np.full((B, n_docs), -np.inf)
    taken = np.zeros((B, n_docs), dtype=bool)
    active = np.ones(B, dtype=bool)
    n_rounds = np.zeros(B, dtype=np.int64)
    rows = [Q[b] for b in range(B)]
    kept = [[] for _ in range(B)]
    for r in range(R):
        for b in range(B):
            if active[b] and rows[b].shape[0] > 0:
                state[b:b + 1] = oracle.route(rows[b][None], Krb, cho, state[b:b + 1])
        elig = np.where(taken, -np.inf, state)
        best = elig.max(axis=1)
        for b in range(B):
            if active[b]:
                assert abs(best[b] - stop) > 2 * tol, f"stop decision too close, query {b}"
        active &= best >= stop
        n_rounds += active
        for b in range(B):
            if not active[b]:
                assert np.all(got[r, b] == -1) and np.all(np.isneginf(sc[r, b])), (r, b)
                rows[b] = np.zeros((0,) + Krb.shape[1:])
                continue
            _valid_topk(got[r, b], elig[b], k, tol, f"round {r}, query {b}")
            assert np.all(np.abs(sc[r, b] - elig[b, got[r, b]]) <= tol), (r, b)
            kept[b].append(got[r, b].tolist())
            taken[b, got[r, b]] = True
            rows[b] = np.concatenate([Krb[cho[d]:cho[d + 1]] for d in got[r, b]], axis=0)
    return state, n_rounds, kept


def _chain_memory(seed, dtype, B, T, n_docs_lognormal, k):
    from top_document_sparse_b200 import msa
    w = small_workload(dtype=dtype, n_docs=0, doc_len=0, lognormal=n_docs_lognormal, batch=B,
                       query_tokens=T, top_k=k, head_dim=64 if dtype == "f32" else 128,
                       n_kv_heads=2, n_q_heads=8, rounds=3)
    off = inputs.doc_offsets(w, seed)
    K, V, Kr = inputs.raw_memory(w, int(off[-1]), seed)
    Qr, _, _, _ = inputs.queries(w, B, T, seed + 1)
    chain = inputs.plant_chain(w, Kr, Qr, off, hops=3, seed=seed + 2)
    mem = msa.Memory(off, w.chunk_len, w.n_kv_heads, w.head_dim, w.n_router_heads, w.router_dim,
                     inputs.torch_dtype(dtype), w.rope_theta, 64)
    rk, ct = mem.new_router_keys(), mem.new_content()
    mem.encode(0, mem.n_docs, K.cuda(), V.cuda(), Kr.cuda(), rk, ct)
    torch.cuda.synchronize()
    _, _, Krb = oracle.encode(K, V, Kr, off, w.chunk_len, w.rope_theta)
    return msa, w, off, Qr, chain, mem, rk, Krb


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_interleave_k1_follows_the_chain_exactly(dtype):
    msa, w, off, Qr, chain, mem, rk, Krb = _chain_memory(300, dtype, B=4, T=12,
                                                          n_docs_lognormal=(200, 1.0, 64, 900, 30000),
                                                          k=1)
    ids, scores, state, taken = mem.interleave(rk, Qr.cuda(), k=1, rounds=3)
    torch.cuda.synchronize()
    ref = oracle.interleave(Qr, Krb, mem.doc_chunk_offsets, k=1, rounds=3)
    got = ids.cpu().numpy()
    for r in range(3):
        assert np.array_equal(got[r], ref[r][0]), f"round {r}"
        assert np.array_equal(got[r][:, 0], chain[:, r])
        tol = 2e-3 if dtype == "bf16" else 1e-5
        assert np.all(np.abs(to64(scores[r]) - ref[r][1]) <= tol)
    tk = taken.cpu().numpy()
    for b in range(4):  # documents of rounds 0 and 1 are in the context
        assert set(np.nonzero(tk[b])[0].tolist()) == {chain[b, 0], chain[b, 1]}
    assert msa.device_error() == 0


def test_interleave_k4_retrieves_each_hop_in_its_round():
    msa, w, off, Qr, chain, mem, rk, Krb = _chain_memory(301, "bf16", B=5, T=16,
                                                          n_docs_lognormal=(300, 1.0, 64, 1500, 60000),
                                                          k=4)
    ids, scores, state, taken = mem.interleave(rk, Qr.cuda(), k=4, rounds=3)
    torch.cuda.synchronize()
    ref = oracle.interleave(Qr, Krb, mem.doc_chunk_offsets, k=4, rounds=3)
    got = ids.cpu().numpy()
    sc = scores.cpu().numpy()
    for b in range(5):
        seen = set()
        for r in range(3):
            row = got[r, b].tolist()
            assert chain[b, r] in row, f"query {b} round {r}"
            assert not (set(row) & seen)               # each round adds new documents
            seen |= set(row)
            pairs = list(zip(-sc[r, b], row))
            assert pairs == sorted(pairs)              # (score desc, id asc)
        # round 0 has no exclusion: compare with the oracle when its k-th / (k+1)-th gap is clear
        o_ids, o_top = ref[0]
        assert chain[b, 0] in o_ids[b]
    assert msa.device_error() == 0


@pytest.mark.parametrize("mode,rounds", [("never", 3), ("split", 3), ("chain_end", 4),
                                         ("always", 3)])
def test_adaptive_interleave_matches_oracle(mode, rounds):
    """msa_interleave_adaptive against the oracle's stop rule: a query stops after the first
    round whose best new document scores below stop_score.  Thresholds: -inf (the fixed rounds),
    +inf (every query stops after round 0), the midpoint of the widest gap between the per-round
    best scores (the planted hops score ~0.6 in round 0 and ~0.48 after: stop after round 0's
    documents), and 0.35 over 4 rounds (keep the three hops, stop on the background).  Every
    finite threshold is at least 4 x the score tolerance from every decision value, so bf16
    rounding cannot flip a stop."""
    msa, w, off, Qr, chain, mem, rk, Krb = _chain_memory(302, "bf16", B=6, T=12,
                                                          n_docs_lognormal=(200, 1.0, 64, 900, 30000),
                                                          k=1)
    tol = 2e-3
    fixed = oracle.interleave(Qr, Krb, mem.doc_chunk_offsets, k=1, rounds=rounds)
    vals = np.unique(np.concatenate([r[1][:, 0] for r in fixed]))
    vals = vals[np.isfinite(vals)]
    gap, mid = max((vals[i + 1] - vals[i], 0.5 * (vals[i] + vals[i + 1]))
                   for i in range(vals.size - 1))
    stop = {"never": -np.inf, "always": np.inf, "split": mid, "chain_end": 0.35}[mode]
    if np.isfinite(stop):
        assert np.min(np.abs(vals - stop)) > 4 * tol
    ids, scores, state, taken, n = mem.interleave_adaptive(rk, Qr.cuda(), k=1, max_rounds=rounds,
                                                           stop_score=stop)
    torch.cuda.synchronize()
    out, st_ref, n_ref = oracle.interleave(Qr, Krb, mem.doc_chunk_offsets, k=1, rounds=rounds,
                                           stop_score=stop)
    assert n.cpu().tolist() == n_ref.tolist()
    got, sc = ids.cpu().numpy(), to64(scores)
    for r in range(rounds):
        assert np.array_equal(got[r], out[r][0]), f"round {r}"
        fin = np.isfinite(out[r][1])
        assert np.array_equal(np.isfinite(sc[r]), fin)
        assert np.all(np.abs(sc[r][fin] - out[r][1][fin]) <= tol)
    st = to64(state)
    fin = np.isfinite(st_ref)
    assert np.array_equal(np.isfinite(st), fin)
    assert np.all(np.abs(st[fin] - st_ref[fin]) <= tol)
    if mode == "never":
        assert n_ref.tolist() == [rounds] * 6
    elif mode == "always":
        assert n_ref.tolist() == [0] * 6
    else:  # the threshold stops queries before the last round
        assert np.all(n_ref < rounds) and np.all(n_ref >= 1)
    assert msa.device_error() == 0


def test_interleave_when_queries_run_out_of_documents():
    """A memory of 3 documents, k = 1, 5 rounds: the last two rounds have nothing eligible left,
    so their ids / scores are -1 / -inf, and a query with no new rows keeps its state."""
    from top_document_sparse_b200 import msa
    from helpers import small_workload as sw
    w = sw(n_docs=3, doc_len=128, batch=2, query_tokens=4, top_k=1)
    off = inputs.doc_offsets(w, 5)
    K, V, Kr = inputs.raw_memory(w, int(off[-1]), 5)
    Qr, _, _, _ = inputs.queries(w, 2, 4, 6)
    mem = msa.Memory(off, w.chunk_len, w.n_kv_heads, w.head_dim, w.n_router_heads, w.router_dim,
                     inputs.torch_dtype(w.dtype), w.rope_theta, 16)
    rk, ct = mem.new_router_keys(), mem.new_content()
    mem.encode(0, mem.n_docs, K.cuda(), V.cuda(), Kr.cuda(), rk, ct)
    torch.cuda.synchronize()
    _, _, Krb = oracle.encode(K, V, Kr, off, w.chunk_len, w.rope_theta)
    ids, scores, state, taken = mem.interleave(rk, Qr.cuda(), k=1, rounds=5)
    torch.cuda.synchronize()
    ref = oracle.interleave(Qr, Krb, mem.doc_chunk_offsets, k=1, rounds=5)
    got = ids.cpu().numpy()
    for r in range(5):
        fin = np.isfinite(ref[r][1])
        # rounds 0-2: each query takes the three documents one by one; the ranking is the oracle's
        # wherever its top two scores are apart (bf16 keys); rounds 3-4: nothing left
        if r >= 3:
            assert np.all(got[r] == -1) and np.all(ref[r][0] == -1)
            assert np.all(np.isneginf(to64(scores[r])))
        else:
            assert np.all(fin) and np.all(got[r] >= 0)
    assert all(sorted(got[:3, b, 0].tolist()) == [0, 1, 2] for b in range(2))
    assert np.all(taken.cpu().numpy() == 1)
    # the state after the last routed round (round 3 routes round 2's document; round 4 has no
    # rows) is the oracle's route of the GPU's own picks, whatever their order
    st, st_ref = to64(state), oracle.route(Qr, Krb, mem.doc_chunk_offsets)
    for r in range(3):
        rows = [np.concatenate([Krb[mem.doc_chunk_offsets[d]:mem.doc_chunk_offsets[d + 1]]
                                for d in got[r, b]])[None] for b in range(2)]
        st_ref = np.concatenate([oracle.route(rows[b], Krb, mem.doc_chunk_offsets,
                                              st_ref[b:b + 1]) for b in range(2)])
    assert np.all(np.abs(st - st_ref) <= 2e-3)
    assert msa.device_error() == 0


def test_adaptive_interleave_k4_with_mixed_stops_matches_oracle():
    """k = 4 and a threshold under which, in the same round, some queries stop and the others go
    on: the stopped queries route zero padding rows with their state saved and restored, the
    active ones route their new documents' rows.  The oracle runs on the GPU's stored unit router
    keys (stage-wise), so ids match exactly; the threshold lies between the per-query best
    background scores of the round after the chain ends, at least 4 x the score tolerance from
    every best score of every round."""
    msa, w, off, Qr, chain, mem, rk, _ = _chain_memory(303, "bf16", B=8, T=12,
                                                        n_docs_lognormal=(200, 1.0, 64, 900, 40000),
                                                        k=4)
    tol, R = 2e-3, 5
    Krb = to64(rk)
    cho = mem.doc_chunk_offsets
    fixed = oracle.interleave(Qr, Krb, cho, k=4, rounds=R)
    best = np.stack([r[1][:, 0] for r in fixed])            # [round][query]
    every = np.unique(best[np.isfinite(best)])
    # candidate thresholds: midpoints between consecutive best scores of rounds 3 and 4 that
    # split round 3's queries; take the one farthest from every decision value
    b3 = best[3]
    bg = np.unique(best[3:][np.isfinite(best[3:])])
    cands = [(np.min(np.abs(every - m)), m) for m in 0.5 * (bg[1:] + bg[:-1])
             if np.any(b3 < m) and np.any(b3 > m)]
    margin, stop = max(cands)
    assert margin > 4 * tol, "no clear threshold in this memory"
    ids, scores, state, taken, n = mem.interleave_adaptive(rk, Qr.cuda(), k=4, max_rounds=R,
                                                           stop_score=stop)
    torch.cuda.synchronize()
    got, sc = ids.cpu().numpy(), to64(scores)
    st_ref, n_ref, kept = _replay_rounds(Qr, Krb, cho, got, sc, 4, R, stop, tol)
    assert n.cpu().numpy().tolist() == n_ref.tolist()
    assert 3 in n_ref and np.any(n_ref > 3), "some queries stop after round 2, others go on"
    st = to64(state)
    fin = np.isfinite(st_ref)
    assert np.array_equal(np.isfinite(st), fin)
    assert np.all(np.abs(st[fin] - st_ref[fin]) <= tol)
    tk = taken.cpu().numpy().astype(bool)
    for b in range(8):  # the context holds the documents of every kept round but the last round
        in_ctx = [d for r in kept[b][:R - 1] for d in r]
        assert set(np.nonzero(tk[b])[0].tolist()) == set(in_ctx), f"query {b}"
    assert msa.device_error() == 0
