"""Pins of the fp64 oracle against facts fixed by the pages and by mathematics.

Each test targets a plausible mistake in the oracle: a wrong chunk boundary, RoPE with the wrong
partner, sign or position, pooling before RoPE, cosine of the concatenated heads instead of the
mean of per-head cosines, a wrong GQA mapping, a missing causal mask or offset, a lost running
state, and so on.  None of them compares the oracle with itself.
"""
import itertools
import json
import math
import os

import numpy as np
import pytest

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def rope_complex(x, pos, theta):
    """Independent restatement of rotate-half RoPE through complex multiplication:
    (x_i + i x_{i+D/2}) * exp(i p theta^(-2i/D))."""
    x = np.asarray(x, dtype=np.float64)
    D = x.shape[-1]
    half = D // 2
    z = x[..., :half] + 1j * x[..., half:]
    freq = theta ** (-2.0 * np.arange(half) / D)
    pos = np.asarray(pos, dtype=np.float64).reshape(-1, *([1] * (x.ndim - 1)))
    z = z * np.exp(1j * pos * freq)
    return np.concatenate([z.real, z.imag], axis=-1)


# ----------------------------------------------------------------------------- chunking
def test_chunking_ragged_by_hand():
    # lengths 100, 128, 72, 1 with chunk 64 -> 2, 2, 2, 1 chunks
    off = np.array([0, 100, 228, 300, 301])
    assert oracle.doc_chunks(off, 64).tolist() == [0, 2, 4, 6, 7]


def test_chunking_rejects_empty_doc():
    with pytest.raises(ValueError):
        oracle.doc_chunks(np.array([0, 5, 5, 9]), 4)


# ----------------------------------------------------------------------------- RoPE
def test_rope_position_zero_is_identity():
    x = np.random.default_rng(1).standard_normal((5, 3, 16))
    y = oracle.rope_rows(x, np.zeros(5, dtype=np.int64), 1e4)
    assert np.array_equal(x, y)


def test_rope_matches_complex_rotation():
    rng = np.random.default_rng(2)
    x = rng.standard_normal((7, 2, 8))
    pos = np.array([0, 1, 2, 5, 17, 511, 8191])
    np.testing.assert_allclose(oracle.rope_rows(x, pos, 1e6), rope_complex(x, pos, 1e6),
                               rtol=0, atol=1e-12)


def test_rope_preserves_pair_norms_and_is_relative():
    rng = np.random.default_rng(3)
    q, k = rng.standard_normal((2, 1, 1, 32))
    theta = 1e6
    y = oracle.rope_rows(q, [123], theta)[0, 0]
    np.testing.assert_allclose(y[:16] ** 2 + y[16:] ** 2, q[0, 0, :16] ** 2 + q[0, 0, 16:] ** 2,
                               rtol=1e-12)
    dots = []
    for m, n in [(10, 3), (110, 103), (7007, 7000)]:
        a = oracle.rope_rows(q, [m], theta)[0, 0]
        b = oracle.rope_rows(k, [n], theta)[0, 0]
        dots.append(a @ b)
    np.testing.assert_allclose(dots, dots[0], rtol=1e-9)


# ----------------------------------------------------------------------------- encoding
def _tiny_memory(seed, lens, H_kv=2, D=8, H_r=2, d_r=4):
    rng = np.random.default_rng(seed)
    off = np.concatenate([[0], np.cumsum(lens)]).astype(np.int64)
    n = int(off[-1])
    K = rng.standard_normal((n, H_kv, D))
    V = rng.standard_normal((n, H_kv, D))
    Kr = rng.standard_normal((n, H_r, d_r))
    return off, K, V, Kr


def test_pool_v_and_kr_are_chunk_means_with_ragged_tail():
    off, K, V, Kr = _tiny_memory(4, [10, 4, 7])
    Kb, Vb, Krb = oracle.encode(K, V, Kr, off, 4, 1e4)
    # chunk token ranges by hand: doc0 [0,4) [4,8) [8,10); doc1 [10,14); doc2 [14,18) [18,21)
    ranges = [(0, 4), (4, 8), (8, 10), (10, 14), (14, 18), (18, 21)]
    assert Vb.shape[0] == len(ranges)
    for c, (a, b) in enumerate(ranges):
        np.testing.assert_allclose(Vb[c], V[a:b].mean(axis=0), rtol=0, atol=1e-14)
        np.testing.assert_allclose(Krb[c], Kr[a:b].mean(axis=0), rtol=0, atol=1e-14)


def test_pool_constant_chunk_gives_constant():
    off = np.array([0, 64], dtype=np.int64)
    V = np.full((64, 1, 4), 2.5)
    Kr = np.full((64, 1, 4), -0.75)
    K = np.zeros((64, 1, 4))
    _, Vb, Krb = oracle.encode(K, V, Kr, off, 64, 1e4)
    assert np.all(Vb == 2.5) and np.all(Krb == -0.75)


def test_pool_k_rope_then_mean_closed_form():
    # A doc whose every token has the same key (1, 0) in a 2-dim head: the rotated keys are
    # exp(i p) for p = 0..n-1 (theta^0 = 1), so the chunk mean is a geometric series,
    # (1/n) * (1 - e^{i n}) / (1 - e^{i}) -- positions restart at 0 in each document.
    L = 6
    off = np.array([0, 9, 14], dtype=np.int64)  # doc0: chunks of 6 and 3; doc1: 5 tokens
    K = np.zeros((14, 1, 2))
    K[:, 0, 0] = 1.0
    V = np.zeros_like(K)
    Kr = np.zeros((14, 1, 2))
    Kb, _, _ = oracle.encode(K, V, Kr, off, L, 1e4)

    def mean_rot(p0, n):
        z = np.exp(1j * p0) * (1 - np.exp(1j * n)) / (1 - np.exp(1j)) / n
        return [z.real, z.imag]

    np.testing.assert_allclose(Kb[0, 0], mean_rot(0, 6), atol=1e-14)
    np.testing.assert_allclose(Kb[1, 0], mean_rot(6, 3), atol=1e-14)
    np.testing.assert_allclose(Kb[2, 0], mean_rot(0, 5), atol=1e-14)


def test_doc_encoded_alone_equals_doc_inside_memory():
    off, K, V, Kr = _tiny_memory(5, [70, 33, 128, 9], H_kv=2, D=16, H_r=2, d_r=8)
    full = oracle.encode(K, V, Kr, off, 32, 1e6)
    cho = oracle.doc_chunks(off, 32)
    for d in range(4):
        a, b = off[d], off[d + 1]
        alone = oracle.encode(K[a:b], V[a:b], Kr[a:b], np.array([0, b - a]), 32, 1e6)
        for x, y in zip(full, alone):
            assert np.array_equal(x[cho[d]:cho[d + 1]], y)


# ----------------------------------------------------------------------------- scoring
def test_cosine_bounds_identity_and_negation():
    rng = np.random.default_rng(6)
    q = rng.standard_normal((8, 16))
    assert oracle.chunk_score(q, q) == pytest.approx(1.0, abs=1e-14)
    assert oracle.chunk_score(q, -q) == pytest.approx(-1.0, abs=1e-14)
    assert oracle.chunk_score(q, 3.5 * q) == pytest.approx(1.0, abs=1e-14)
    for _ in range(50):
        k = rng.standard_normal((8, 16))
        s = oracle.chunk_score(q, k)
        assert -1.0 <= s <= 1.0
        assert oracle.chunk_score(7.0 * q, 0.01 * k) == pytest.approx(s, abs=1e-14)


def test_score_is_mean_of_per_head_cosines_not_cosine_of_concat():
    q = np.array([[10.0, 0.0], [0.0, 1.0]])
    k = np.array([[10.0, 0.0], [1.0, 0.0]])
    # head 0: cos 1, head 1: cos 0 -> mean 0.5 (the cosine of the concatenation would be ~0.99)
    assert oracle.chunk_score(q, k) == pytest.approx(0.5, abs=1e-15)
    k2 = np.array([[10.0, 0.0], [0.0, -1.0]])
    assert oracle.chunk_score(q, k2) == pytest.approx(0.0, abs=1e-15)


def test_zero_vector_scores_zero():
    q = np.array([[1.0, 2.0]])
    assert oracle.chunk_score(q, np.zeros((1, 2))) == 0.0


def test_route_is_max_over_tokens_and_chunks_brute_force():
    rng = np.random.default_rng(7)
    off = np.array([0, 3, 4, 8, 10])  # chunk offsets of 4 docs
    Kr = rng.standard_normal((10, 2, 5))
    Qr = rng.standard_normal((3, 4, 2, 5))
    got = oracle.route(Qr, Kr, off)
    for b in range(3):
        for d in range(4):
            best = max(oracle.chunk_score(Qr[b, t], Kr[c])
                       for t in range(4) for c in range(off[d], off[d + 1]))
            assert got[b, d] == best


def test_route_running_state_equals_all_tokens_at_once():
    rng = np.random.default_rng(8)
    off = np.array([0, 2, 5, 6])
    Kr = rng.standard_normal((6, 2, 4))
    Qr = rng.standard_normal((2, 9, 2, 4))
    once = oracle.route(Qr, Kr, off)
    st = oracle.route(Qr[:, :5], Kr, off)
    for t in range(5, 9):
        st = oracle.route(Qr[:, t], Kr, off, st)
    assert np.array_equal(st, once)


def test_planted_chunk_scores_the_planted_cosine():
    import torch
    from top_document_sparse_b200 import inputs
    from top_document_sparse_b200.workloads import Workload
    w = Workload(name="t", description="", dtype="f32", n_docs=6, doc_len=128, chunk_len=32,
                 n_q_heads=2, n_kv_heads=1, head_dim=8, n_router_heads=3, router_dim=16,
                 top_k=2, batch=2, query_tokens=5, decode_steps=0, n_layers=1,
                 planted_per_query=2, planted_cos=0.6)
    off = inputs.doc_offsets(w)
    g = inputs.generator(11, "cpu")
    Kr = torch.randn(int(off[-1]), 3, 16, generator=g, dtype=torch.float64)
    Qr = torch.randn(2, 5, 3, 16, generator=g, dtype=torch.float64)
    plants = inputs.choose_plants(w, off, 2, 5, 2, seed=3)
    inputs.plant(w, Kr, Qr, off, plants, 0.6, seed=3)
    K = np.zeros((Kr.shape[0], 1, 8))
    _, _, Krb = oracle.encode(K, K, Kr.numpy(), off, 32, 1e4)
    cho = oracle.doc_chunks(off, 32)
    for b, d, j, t in zip(*plants):
        assert oracle.chunk_score(Qr[b, t].numpy(), Krb[cho[d] + j]) == pytest.approx(0.6,
                                                                                     abs=1e-12)


# ----------------------------------------------------------------------------- top-k
def test_topk_matches_brute_force_with_ties():
    rng = np.random.default_rng(9)
    for trial in range(30):
        n = int(rng.integers(3, 9))
        k = int(rng.integers(1, n + 1))
        s = rng.integers(0, 4, size=(2, n)).astype(np.float64)  # many exact ties
        ids, top = oracle.topk(s, k)
        for b in range(2):
            # brute force: among all k-subsets in increasing-id order, the best is the one whose
            # sorted (-score, id) sequence is lexicographically smallest
            best = min(itertools.combinations(range(n), k),
                       key=lambda c: sorted((-s[b, d], d) for d in c))
            want = [d for _, d in sorted((-s[b, d], d) for d in best)]
            assert ids[b].tolist() == want
            assert top[b].tolist() == [s[b, d] for d in want]


def test_topk_tie_goes_to_lower_id():
    ids, _ = oracle.topk(np.array([[0.5, 0.9, 0.9, 0.1, 0.9]]), 2)
    assert ids.tolist() == [[1, 2]]


# ----------------------------------------------------------------------------- attention
def _attn_case(seed, B=2, T=3, H_q=4, H_kv=2, D=8, L_loc=6, q_start=2, n_docs=5, k=2):
    rng = np.random.default_rng(seed)
    doc_chunk_off = np.array([0, 2, 3, 6, 7, 9])[: n_docs + 1]
    C = int(doc_chunk_off[-1])
    Q = rng.standard_normal((B, T, H_q, D))
    Kl = rng.standard_normal((B, L_loc, H_kv, D))
    Vl = rng.standard_normal((B, L_loc, H_kv, D))
    Kb = rng.standard_normal((C, H_kv, D))
    Vb = rng.standard_normal((C, H_kv, D))
    ids = np.stack([rng.choice(n_docs, size=k, replace=False) for _ in range(B)]).astype(np.int32)
    return Q, Kl, Vl, q_start, Kb, Vb, doc_chunk_off, ids


def dense_reference(Q, Kl, Vl, q_start, Kb, Vb, doc_chunk_off, ids, pos_offset, theta):
    """Textbook causal softmax attention over an explicitly built context (k = all docs case
    reduces the sparse layer to this)."""
    B, T, H_q, D = Q.shape
    H_kv = Kl.shape[2]
    O = np.zeros_like(Q)
    for b in range(B):
        mem_c = np.concatenate([np.arange(doc_chunk_off[d], doc_chunk_off[d + 1]) for d in ids[b]])
        for i in range(T):
            j = q_start + i
            for h in range(H_q):
                g = h // (H_q // H_kv)
                keys = np.concatenate([Kb[mem_c, g],
                                       rope_complex(Kl[b, :j + 1, g], pos_offset + np.arange(j + 1),
                                                    theta)])
                vals = np.concatenate([Vb[mem_c, g], Vl[b, :j + 1, g]])
                q = rope_complex(Q[b, i, h][None], [pos_offset + j], theta)[0]
                z = keys @ q / math.sqrt(D)
                p = np.exp(z - z.max())
                O[b, i, h] = (p / p.sum()) @ vals
    return O


def test_attention_rows_sum_to_one():
    args = _attn_case(10)
    _, _, rs = oracle.attend(*args, pos_offset=2, theta=1e4)
    np.testing.assert_allclose(rs, 1.0, atol=1e-13)


def test_attention_single_key_returns_its_value():
    Q, Kl, Vl, _, Kb, Vb, off, _ = _attn_case(11)
    ids = np.zeros((2, 0), dtype=np.int32)
    O, _, _ = oracle.attend(Q[:, :1], Kl, Vl, 0, Kb, Vb, off, ids, pos_offset=0, theta=1e4)
    for h in range(4):
        np.testing.assert_allclose(O[:, 0, h], Vl[:, 0, h // 2], atol=1e-15)


def test_attention_equal_logits_average_the_values():
    Q, Kl, Vl, q_start, Kb, Vb, off, ids = _attn_case(12)
    Q = np.zeros_like(Q)
    O, _, _ = oracle.attend(Q, Kl, Vl, q_start, Kb, Vb, off, ids, pos_offset=5, theta=1e4)
    for b in range(2):
        mem_c = np.concatenate([np.arange(off[d], off[d + 1]) for d in ids[b]])
        for i in range(Q.shape[1]):
            for h in range(4):
                vals = np.concatenate([Vb[mem_c, h // 2], Vl[b, :q_start + i + 1, h // 2]])
                np.testing.assert_allclose(O[b, i, h], vals.mean(axis=0), atol=1e-14)


def test_attention_gqa_equals_mha_with_repeated_kv_heads():
    Q, Kl, Vl, q_start, Kb, Vb, off, ids = _attn_case(13)
    rep = [0, 0, 1, 1]
    O_gqa, _, _ = oracle.attend(Q, Kl, Vl, q_start, Kb, Vb, off, ids, 3, 1e4)
    O_mha, _, _ = oracle.attend(Q, Kl[:, :, rep], Vl[:, :, rep], q_start, Kb[:, rep], Vb[:, rep],
                                off, ids, 3, 1e4)
    np.testing.assert_allclose(O_gqa, O_mha, atol=1e-14)


def test_attention_all_docs_is_dense_attention_in_any_order():
    Q, Kl, Vl, q_start, Kb, Vb, off, _ = _attn_case(14, k=5)
    all_ids = np.tile(np.arange(5, dtype=np.int32), (2, 1))
    perm = np.stack([np.random.default_rng(0).permutation(5) for _ in range(2)]).astype(np.int32)
    O1, _, _ = oracle.attend(Q, Kl, Vl, q_start, Kb, Vb, off, all_ids, 5, 1e4)
    O2, _, _ = oracle.attend(Q, Kl, Vl, q_start, Kb, Vb, off, perm, 5, 1e4)
    ref = dense_reference(Q, Kl, Vl, q_start, Kb, Vb, off, all_ids, 5, 1e4)
    np.testing.assert_allclose(O1, ref, atol=1e-12)
    np.testing.assert_allclose(O2, ref, atol=1e-12)


def test_attention_global_rope_offset_and_causality():
    Q, Kl, Vl, q_start, Kb, Vb, off, ids = _attn_case(15)
    for pos_offset in (0, 2, 37):
        O, _, _ = oracle.attend(Q, Kl, Vl, q_start, Kb, Vb, off, ids, pos_offset, 1e4)
        ref = dense_reference(Q, Kl, Vl, q_start, Kb, Vb, off, ids, pos_offset, 1e4)
        np.testing.assert_allclose(O, ref, atol=1e-12)
    # causality: local rows after the query token do not matter
    Kl2, Vl2 = Kl.copy(), Vl.copy()
    Kl2[:, q_start + 1:] = 99.0
    Vl2[:, q_start + 1:] = -99.0
    O_a, _, _ = oracle.attend(Q[:, :1], Kl, Vl, q_start, Kb, Vb, off, ids, 2, 1e4)
    O_b, _, _ = oracle.attend(Q[:, :1], Kl2, Vl2, q_start, Kb, Vb, off, ids, 2, 1e4)
    assert np.array_equal(O_a, O_b)


# ----------------------------------------------------------------------------- composition
def test_decode_step_state_equals_route_over_all_tokens():
    rng = np.random.default_rng(16)
    off = np.array([0, 2, 4, 6, 8])
    Kr = rng.standard_normal((8, 2, 4))
    Qr = rng.standard_normal((2, 6, 2, 4))
    Q, Kl, Vl, _, Kb, Vb, _, _ = _attn_case(16, B=2, T=6, L_loc=6, n_docs=4)
    st = oracle.route(Qr[:, :4], Kr, off)
    for t in range(4, 6):
        st, ids, top, O = oracle.decode_step(st, Qr[:, t], Q[:, t], Kl, Vl, t, Kr, Kb, Vb, off,
                                            k=2, pos_offset=2, theta=1e4)
    want = oracle.route(Qr, Kr, off)
    assert np.array_equal(st, want)
    ids_all, _ = oracle.topk(want, 2)
    assert np.array_equal(ids, ids_all)


def test_interleave_retrieves_planted_chain_hop_by_hop():
    import torch
    from top_document_sparse_b200 import inputs
    from top_document_sparse_b200.workloads import Workload
    w = Workload(name="t", description="", dtype="f32", n_docs=40, doc_len=64, chunk_len=16,
                 n_q_heads=2, n_kv_heads=1, head_dim=8, n_router_heads=4, router_dim=32,
                 top_k=3, batch=3, query_tokens=4, decode_steps=0, n_layers=1,
                 planted_per_query=3, planted_cos=0.6, rounds=3)
    off = inputs.doc_offsets(w)
    g = inputs.generator(21, "cpu")
    Kr = torch.randn(int(off[-1]), 4, 32, generator=g, dtype=torch.float64)
    Qr = torch.randn(3, 4, 4, 32, generator=g, dtype=torch.float64)
    chain = inputs.plant_chain(w, Kr, Qr, off, hops=3, seed=5)
    K0 = np.zeros((Kr.shape[0], 1, 8))
    _, _, Krb = oracle.encode(K0, K0, Kr.numpy(), off, 16, 1e4)
    cho = oracle.doc_chunks(off, 16)
    rounds = oracle.interleave(Qr.numpy(), Krb, cho, k=3, rounds=3)
    for b in range(3):
        seen = set()
        for r, (ids, _) in enumerate(rounds):
            seen |= set(ids[b].tolist())
            assert chain[b, r] in ids[b]                  # hop r+1 surfaces in round r+1
            for later in chain[b, r + 1:]:
                assert later not in seen                  # and not before
        assert len(seen) == 9                             # each round adds new documents


def _adaptive_docs():
    """Four one-chunk documents (H_r = 1, d_r = 4): D0 = e0, D1 = 0.6 e0 + 0.8 e1, D2 = e1,
    D3 = -e0, and one query token e0.  With k = 1: round 0 takes D0 (cos 1); round 1 routes D0's
    row (= e0, nothing new) and takes D1 (0.6); round 2 routes D1's row, which raises D2 to 0.8
    and takes it."""
    e0, e1 = np.eye(4)[0], np.eye(4)[1]
    Krb = np.stack([e0, 0.6 * e0 + 0.8 * e1, e1, -e0])[:, None, :]   # [C][H_r][d_r]
    off = np.arange(5, dtype=np.int64)                                # one chunk per document
    Qr = e0[None, None, None, :]                                       # [B=1][T=1][H_r][d_r]
    return Qr, Krb, off


def test_adaptive_interleave_stop_rule_on_a_hand_worked_chain():
    Qr, Krb, off = _adaptive_docs()
    out, state, n = oracle.interleave(Qr, Krb, off, k=1, rounds=3, stop_score=0.5)
    assert [int(r[0][0, 0]) for r in out] == [0, 1, 2]
    np.testing.assert_allclose([r[1][0, 0] for r in out], [1.0, 0.6, 0.8], atol=1e-12)
    assert n.tolist() == [3]
    np.testing.assert_allclose(state[0], [1.0, 1.0, 0.8, -0.6], atol=1e-12)  # D3: cos(-e0, D1) = -0.6
    # 0.7: round 1's best (0.6) is below it -> stop after one kept round; nothing of round 1 or 2
    out, state, n = oracle.interleave(Qr, Krb, off, k=1, rounds=3, stop_score=0.7)
    assert [int(r[0][0, 0]) for r in out] == [0, -1, -1]
    assert np.all(np.isneginf([r[1][0, 0] for r in out[1:]]))
    assert n.tolist() == [1]
    np.testing.assert_allclose(state[0], [1.0, 0.6, 0.0, -1.0], atol=1e-12)  # D1's row unrouted


def test_adaptive_interleave_keeps_a_round_whose_best_score_equals_the_threshold():
    Qr, Krb, off = _adaptive_docs()                     # round 1's best is exactly 0.6
    _, _, n = oracle.interleave(Qr, Krb, off, k=1, rounds=3, stop_score=0.6)
    assert n.tolist() == [3]                            # "below" stops; equal does not


def test_adaptive_interleave_limits_reduce_to_fixed_rounds_and_to_round_zero():
    Qr, Krb, off = _adaptive_docs()
    fixed = oracle.interleave(Qr, Krb, off, k=2, rounds=3)
    out, _, n = oracle.interleave(Qr, Krb, off, k=2, rounds=3, stop_score=-np.inf)
    for (a_ids, a_sc), (b_ids, b_sc) in zip(fixed, out):
        assert np.array_equal(a_ids, b_ids) and np.array_equal(a_sc, b_sc)
    assert n.tolist() == [3]
    out, state, n = oracle.interleave(Qr, Krb, off, k=2, rounds=3, stop_score=np.inf)
    assert n.tolist() == [0] and all(np.all(r[0] == -1) for r in out)
    np.testing.assert_allclose(state, oracle.route(Qr, Krb, off), atol=0)  # only round 0 routed


def test_interleave_pads_with_minus_one_once_every_document_is_in_the_context():
    Qr, Krb, off = _adaptive_docs()                     # four documents, k = 1
    out = oracle.interleave(Qr, Krb, off, k=1, rounds=6)
    ids = [int(r[0][0, 0]) for r in out]
    assert sorted(ids[:4]) == [0, 1, 2, 3] and ids[4:] == [-1, -1]
    assert all(np.isneginf(r[1][0, 0]) for r in out[4:])
    # rounds 1-4 route the rows of the documents taken in rounds 0-3; round 5 has no rows, so the
    # final state is the max of the query's and those four documents' cosines: every document
    # matches its own row exactly, so the state is 1 everywhere
    _, state, _ = oracle.interleave(Qr, Krb, off, k=1, rounds=6, stop_score=-np.inf)
    np.testing.assert_allclose(state[0], np.ones(4), atol=1e-12)


# ----------------------------------------------------------------------------- golden example
def test_golden_hand_worked_example():
    with open(os.path.join(GOLDEN, "hand_worked_route_attend.json")) as f:
        g = json.load(f)
    off = np.array(g["doc_token_offsets"])
    Kr = np.array(g["router_key_tokens"], dtype=np.float64)
    K = np.array(g["key_tokens"], dtype=np.float64)
    V = np.array(g["value_tokens"], dtype=np.float64)
    Kb, Vb, Krb = oracle.encode(K, V, Kr, off, g["chunk_len"], g["rope_theta"])
    np.testing.assert_allclose(Krb, np.array(g["expect_pooled_router_keys"]), atol=1e-15)
    np.testing.assert_allclose(Vb, np.array(g["expect_pooled_values"]), atol=1e-15)
    cho = oracle.doc_chunks(off, g["chunk_len"])
    assert cho.tolist() == g["expect_doc_chunk_offsets"]
    Qr = np.array(g["query_router_tokens"], dtype=np.float64)
    scores = oracle.route(Qr, Krb, cho)
    np.testing.assert_allclose(scores, np.array(g["expect_doc_scores"]), atol=1e-15)
    ids, _ = oracle.topk(scores, g["top_k"])
    assert ids.tolist() == g["expect_topk_ids"]
    Q = np.array(g["query_tokens"], dtype=np.float64)
    Kl = np.array(g["local_keys"], dtype=np.float64)
    Vl = np.array(g["local_values"], dtype=np.float64)
    O, _, _ = oracle.attend(Q, Kl, Vl, 0, Kb, Vb, cho, ids, g["pos_offset"], g["rope_theta"])
    np.testing.assert_allclose(O, np.array(g["expect_output"]), atol=1e-12)
